"""fdllm_generate_batch: independent sequences of different prompt lengths
(variable-length serving, BASELINE's batched configuration in small), each on
its own block schedule, decoded together with one shared weight stream per
global step (continuous batching over the context's sequence slots: more
sequences than slots, so sequences join as others finish).

Tiny fp32 model: every sequence's tokens and step count equal the
single-sequence path's bit for bit, and that path matches the float64 oracle
step by step (and free-running for non-empty prompts), in every cache mode.
bf16 models: every step of every sequence, as the batched path took it, is
recomputed by the oracle on that sequence's own tokens (confidences within
1e-3, tokens and unmask sets identical except counted near ties), and the
returned tokens equal the traced decisions."""
import numpy as np
import pytest
import torch

from kv_cache_decode_dualcache_b200 import synth
from oracle.decode import generate
from oracle.model import Model
from tests.gpu_util import make_decoder, require_gpu
from tests.parity import replay_gpu_trace

pytestmark = pytest.mark.gpu


def _prompts(shape, lens, salt0=10):
    return [synth.make_prompt(shape, n, salt=salt0 + i).numpy() for i, n in enumerate(lens)]


class _Seq:
    """One sequence's slice of a batched trace, shaped like GenerateStats."""

    def __init__(self, st, i):
        self.trace_block = st.trace_block[i]
        self.trace_conf = st.trace_conf[i]
        self.trace_tok = st.trace_tok[i]
        self.trace_unmask = st.trace_unmask[i]


@pytest.mark.parametrize("mode", ["dual", "prefix", "none"])
@pytest.mark.parametrize("slots", [2, 4])
def test_batch_tiny_matches_single_and_oracle(mode, slots):
    # 5 sequences over 2 or 4 slots: sequences join as others finish.  The
    # fp32 kernels sum in a fixed order per output, so the batched path must
    # equal the single-sequence path bit for bit; that path is checked
    # against the oracle step by step, and, for non-empty prompts, as a
    # free-running sequence.  (With an empty prompt every position holds the
    # mask token, the block's confidences tie to ~1e-6 and the fallback
    # pick is a near tie, which the step-by-step rule counts.)
    require_gpu()
    shape = synth.TINY
    w = synth.make_weights(shape, device="cpu")
    dec = make_decoder(shape, w, 96, max_batch=slots)
    lens, G, B, tau = [20, 32, 9, 0, 27], 48, 16, 0.9
    prompts = _prompts(shape, lens)
    out, steps, stats = dec.generate_batch(prompts, G, B, tau, mode)
    model = Model(shape.as_dict(), w)
    assert stats.steps == int(steps.sum())
    for i, p in enumerate(prompts):
        one, n1, st1 = dec.generate(p, G, B, tau, mode, trace=True)
        assert np.array_equal(out[i], one), i
        assert steps[i] == n1
        assert stats.steps_per_block[i * (G // B):(i + 1) * (G // B)] == st1.steps_per_block
        rep = replay_gpu_trace(model, p, G, B, tau, mode, one, st1, label=f"tiny seq {i}")
        print(f"tiny {mode} seq {i} (P={lens[i]}): {rep.summary()}")
        assert not rep.mismatches, rep.mismatches[:5]
        if lens[i] > 0:
            ref = generate(model, p, G, B, tau, mode)
            assert np.array_equal(one, ref.tokens), i
            assert n1 == ref.steps
    dec.close()


@pytest.mark.parametrize("name", ["small-bf16", "small-gqa-bf16"])
@pytest.mark.parametrize("mode", ["dual", "prefix"])
@pytest.mark.parametrize("blk", ["1", "0"], ids=["attn-tc", "attn-mma"])
def test_batch_bf16_steps_match_oracle(name, mode, blk):
    """Block segments through the tcgen05 block attention (default) and the
    mma.sync one (FDLLM_ATTN_BLK=0)."""
    require_gpu()
    shape = synth.SHAPES[name]
    w = synth.make_weights(shape, device="cpu")
    dec = make_decoder(shape, w, 256, max_batch=3, env={"FDLLM_ATTN_BLK": blk})
    lens, G, B, tau = [128, 40, 71, 200, 0], 32, 16, 0.9
    prompts = _prompts(shape, lens, salt0=30)
    out, steps, st = dec.generate_batch(prompts, G, B, tau, mode, trace=True)
    dec.close()
    model = Model(shape.as_dict(), w)
    same_as_single = 0
    for i, p in enumerate(prompts):
        rep = replay_gpu_trace(model, p, G, B, tau, mode, out[i], _Seq(st, i),
                               label=f"{name} {mode} seq {i}")
        print(f"{name} {mode} seq {i} (P={lens[i]}): {rep.summary()}")
        assert rep.steps == steps[i]
        assert not rep.mismatches, rep.mismatches[:5]


def test_batch_llada8b_2layer_steps_match_oracle():
    # full LLaDA-8B layer width, vocabulary and heads; three sequences of
    # different lengths in two slots
    require_gpu()
    shape = synth.with_layers(synth.LLADA_8B, 2)
    w = synth.make_weights(shape, device="cuda")
    lens, G, B, tau = [96, 33, 160], 64, 32, 0.9
    dec = make_decoder(shape, w, max(lens) + G, max_batch=2)
    w_host = {k: v.cpu() for k, v in w.items()}
    del w
    torch.cuda.empty_cache()
    prompts = _prompts(shape, lens, salt0=50)
    out, steps, st = dec.generate_batch(prompts, G, B, tau, "dual", trace=True)
    dec.close()
    model = Model(shape.as_dict(), w_host)
    for i, p in enumerate(prompts):
        rep = replay_gpu_trace(model, p, G, B, tau, "dual", out[i], _Seq(st, i),
                               label=f"llada8b-2layer seq {i}")
        print(f"llada8b-2layer batched seq {i} (P={lens[i]}): {rep.summary()}")
        assert rep.steps == steps[i]
        assert not rep.mismatches, rep.mismatches[:5]


def test_batch_rejects_any_bad_sequence():
    require_gpu()
    from kv_cache_decode_dualcache_b200.fdllm import FdllmError
    shape = synth.TINY
    dec = make_decoder(shape, synth.make_weights(shape, device="cpu"), 96, max_batch=2)
    good = synth.make_prompt(shape, 16).numpy()
    bad = good.copy()
    bad[3] = shape.mask_id
    with pytest.raises(FdllmError):
        dec.generate_batch([good, bad], 32, 16, 0.9, "dual")
    too_long = synth.make_prompt(shape, 80).numpy()
    with pytest.raises(FdllmError):
        dec.generate_batch([good, too_long], 32, 16, 0.9, "dual")
    dec.close()
