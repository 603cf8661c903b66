"""CPU checks of the GPU parity harness itself (``tests/parity.py``): the
production-path replay and the teacher-forced driver, fed with decisions
taken from the oracle (so they must pass) and with decisions altered in the
ways a faulty decoder could alter them (so they must fail).  No GPU: the
"device" side is the oracle's own trace, or a stand-in object whose
``step_debug`` answers with the oracle's step.
"""
from types import SimpleNamespace

import numpy as np
import pytest

from kv_cache_decode_dualcache_b200 import synth
from oracle.decode import generate, step
from oracle.model import Model
from tests.parity import replay_gpu_trace, teacher_forced

SHAPE = synth.TINY
MASK = SHAPE.mask_id
P, G, B, TAU = 20, 32, 8, 0.9


@pytest.fixture(scope="module")
def tiny():
    return Model(SHAPE.as_dict(), synth.make_weights(SHAPE, device="cpu"))


@pytest.fixture(scope="module")
def prompt():
    return synth.make_prompt(SHAPE, P, salt=3).numpy()


def _stats(res):
    """The per-step trace the decoder's generate returns, built from the
    oracle's run (confidences as float32, as the decoder reports them)."""
    return SimpleNamespace(
        trace_block=np.array([r.block for r in res.trace], np.int32),
        trace_conf=np.stack([r.conf for r in res.trace]).astype(np.float32),
        trace_tok=np.stack([r.tok for r in res.trace]).astype(np.int32),
        trace_unmask=np.stack([r.unmask for r in res.trace]))


def _run(tiny, prompt, mode):
    res = generate(tiny, prompt, G, B, TAU, mode)
    assert res.steps > G // B
    return res, _stats(res)


@pytest.mark.parametrize("mode", ["dual", "prefix", "none"])
def test_replay_of_the_oracles_own_decisions_passes(tiny, prompt, mode):
    res, st = _run(tiny, prompt, mode)
    rep = replay_gpu_trace(tiny, prompt, G, B, TAU, mode, res.tokens, st)
    assert rep.steps == res.steps
    assert not rep.mismatches and rep.exempt == 0
    assert rep.max_dconf < 1e-6                       # float32 rounding of the trace only


def test_replay_limits_the_compared_steps(tiny, prompt):
    res, st = _run(tiny, prompt, "dual")
    one = replay_gpu_trace(tiny, prompt, G, B, TAU, "dual", res.tokens, st, max_steps_per_block=1)
    assert one.steps == G // B and not one.mismatches
    two = replay_gpu_trace(tiny, prompt, G, B, TAU, "dual", res.tokens, st, max_steps_per_block=2)
    assert two.steps == sum(min(2, n) for n in res.steps_per_block) and not two.mismatches
    only = replay_gpu_trace(tiny, prompt, G, B, TAU, "dual", res.tokens, st, blocks={1})
    assert only.steps == res.steps_per_block[1] and not only.mismatches


def test_replay_catches_a_block_left_with_masked_positions(tiny, prompt):
    # block 1's last step is dropped from the trace: block 2 starts while
    # block 1 still holds the mask id
    res, st = _run(tiny, prompt, "dual")
    last0 = int(np.flatnonzero(st.trace_block == 1)[-1])
    keep = np.ones(len(st.trace_block), bool)
    keep[last0] = False
    cut = SimpleNamespace(trace_block=st.trace_block[keep], trace_conf=st.trace_conf[keep],
                          trace_tok=st.trace_tok[keep], trace_unmask=st.trace_unmask[keep])
    tokens = res.tokens.copy()
    tokens[B + np.flatnonzero(res.trace[last0].unmask)] = MASK
    rep = replay_gpu_trace(tiny, prompt, G, B, TAU, "dual", tokens, cut)
    assert any("block 1 left masked positions" in m for m in rep.mismatches)


def _first_cached_step(res):
    return next(i for i, r in enumerate(res.trace) if r.kind != "refresh")


def test_replay_catches_a_wrong_token(tiny, prompt):
    res, st = _run(tiny, prompt, "dual")
    i = _first_cached_step(res)
    j = int(np.flatnonzero(st.trace_unmask[i])[0])
    st.trace_tok[i, j] = (st.trace_tok[i, j] + 1) % MASK
    tokens = res.tokens.copy()
    tokens[(res.trace[i].block * B) + j] = st.trace_tok[i, j]
    rep = replay_gpu_trace(tiny, prompt, G, B, TAU, "dual", tokens, st)
    assert any(f"row {j} token" in m for m in rep.mismatches)
    assert not any("returned tokens differ" in m for m in rep.mismatches)


def test_replay_catches_a_confidence_off_by_more_than_1e3(tiny, prompt):
    res, st = _run(tiny, prompt, "none")
    st.trace_conf[_first_cached_step(res)] += 2e-3
    rep = replay_gpu_trace(tiny, prompt, G, B, TAU, "none", res.tokens, st)
    assert len(rep.mismatches) == 1 and "conf max-abs" in rep.mismatches[0]


def test_replay_catches_a_changed_unmask_set(tiny, prompt):
    res, st = _run(tiny, prompt, "prefix")
    i = _first_cached_step(res)
    b = res.trace[i].block
    # also unmask a still-masked position whose confidence is far from tau
    u = st.trace_unmask[i].copy()
    masked_now = np.ones(B, bool)
    for r in res.trace[:i]:
        if r.block == b:
            masked_now &= ~r.unmask
    extra = [k for k in np.flatnonzero(masked_now & ~u) if abs(res.trace[i].conf[k] - TAU) > 1e-2]
    assert extra, "no masked position left to add"
    st.trace_unmask[i, extra[0]] = True
    rep = replay_gpu_trace(tiny, prompt, G, B, TAU, "prefix", res.tokens, st)
    assert any("unmask sets differ" in m for m in rep.mismatches)


def test_replay_catches_a_step_that_unmasks_a_decoded_position(tiny, prompt):
    res, st = _run(tiny, prompt, "dual")
    i = _first_cached_step(res)
    decoded = np.flatnonzero(st.trace_unmask[i - 1])[0]   # unmasked by the refresh step
    st.trace_unmask[i, decoded] = True
    rep = replay_gpu_trace(tiny, prompt, G, B, TAU, "dual", res.tokens, st)
    assert any("already decoded" in m for m in rep.mismatches)


def test_replay_catches_returned_tokens_that_differ_from_the_trace(tiny, prompt):
    res, st = _run(tiny, prompt, "dual")
    tokens = res.tokens.copy()
    tokens[-1] = (tokens[-1] + 1) % MASK
    rep = replay_gpu_trace(tiny, prompt, G, B, TAU, "dual", tokens, st)
    assert any("returned tokens differ" in m for m in rep.mismatches)


def test_replay_catches_blocks_out_of_order_and_empty_steps(tiny, prompt):
    res, st = _run(tiny, prompt, "dual")
    swapped = SimpleNamespace(**vars(st))
    swapped.trace_block = st.trace_block.copy()
    first_b1 = int(np.flatnonzero(st.trace_block == 1)[0])
    swapped.trace_block[first_b1] = 2
    rep = replay_gpu_trace(tiny, prompt, G, B, TAU, "dual", res.tokens, swapped)
    assert any("after block" in m for m in rep.mismatches)
    empty = SimpleNamespace(**vars(st))
    empty.trace_unmask = st.trace_unmask.copy()
    empty.trace_unmask[_first_cached_step(res)] = False
    rep = replay_gpu_trace(tiny, prompt, G, B, TAU, "dual", res.tokens, empty)
    assert any("unmasked nothing" in m for m in rep.mismatches)


def test_replay_catches_a_generation_that_stops_early(tiny, prompt):
    # the last step is missing and the returned tokens still hold the mask id
    # where it would have unmasked: only the left-over masks are wrong
    res, st = _run(tiny, prompt, "dual")
    last = res.trace[-1]
    short = SimpleNamespace(trace_block=st.trace_block[:-1], trace_conf=st.trace_conf[:-1],
                            trace_tok=st.trace_tok[:-1], trace_unmask=st.trace_unmask[:-1])
    tokens = res.tokens.copy()
    tokens[last.block * B + np.flatnonzero(last.unmask)] = MASK
    rep = replay_gpu_trace(tiny, prompt, G, B, TAU, "dual", tokens, short)
    assert rep.mismatches and all("masked positions left" in m for m in rep.mismatches)


class _OracleStandIn:
    """Answers ``step_debug`` with the oracle's step, optionally shifted."""

    def __init__(self, model, dz=0.0, dconf=0.0):
        self.model, self.dz, self.dconf = model, dz, dconf

    def step_debug(self, snap, x, s, block, tau, mode):
        out = step(self.model, snap, x, s, block, tau, mode)
        return {"z": out["z"].astype(np.float32) + self.dz,
                "conf": out["conf"].astype(np.float32) + self.dconf,
                "tok": out["tok"], "unmask": out["unmask"]}


@pytest.mark.parametrize("mode", ["dual", "prefix", "none"])
def test_teacher_forced_driver(tiny, prompt, mode):
    ref = generate(tiny, prompt, G, B, TAU, mode, keep_logits=True)
    ok = teacher_forced(_OracleStandIn(tiny), tiny, ref.trace, prompt, G, B, TAU, mode, MASK,
                        z_tol=1e-4)
    assert ok.steps == ref.steps and not ok.mismatches and ok.max_dz < 1e-4
    bad_z = teacher_forced(_OracleStandIn(tiny, dz=2e-4), tiny, ref.trace, prompt, G, B, TAU,
                           mode, MASK, z_tol=1e-4)
    assert any("logits" in m for m in bad_z.mismatches)
    bad_c = teacher_forced(_OracleStandIn(tiny, dconf=2e-3), tiny, ref.trace, prompt, G, B, TAU,
                           mode, MASK, z_tol=1e-4)
    assert any("conf" in m for m in bad_c.mismatches)
    some = teacher_forced(_OracleStandIn(tiny), tiny, ref.trace, prompt, G, B, TAU, mode, MASK,
                          z_tol=1e-4, max_steps=2)
    assert some.steps == 2 and not some.mismatches
    every3 = teacher_forced(_OracleStandIn(tiny), tiny, ref.trace, prompt, G, B, TAU, mode, MASK,
                            z_tol=1e-4, stride=3)
    assert every3.steps == -(-ref.steps // 3) and not every3.mismatches
