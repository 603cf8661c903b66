"""Pins for the oracle's block decode loop and cache modes (tiny fp32 model).

The invariants come from what the pages fix:
* cache off with tau > 1 is the plain sequential greedy masked-diffusion
  decode, one token per step (the baseline of the long-generation figure);
* the block-end refresh stores exactly a full recompute of the K/V;
* with block size 1 every block is a single refresh step, so all cache modes
  coincide;
* tau <= 0 finishes a block per step, tau > 1 takes one step per token;
* DualCache steps read prefix and suffix from the cache, prefix-cache steps
  read only the prefix from it.
"""
import numpy as np
import pytest
import torch

from kv_cache_decode_dualcache_b200 import synth
from oracle.decode import generate, step
from oracle.model import Model

SHAPE = synth.TINY


@pytest.fixture(scope="module")
def tiny():
    w = synth.make_weights(SHAPE, device="cpu")
    return Model(SHAPE.as_dict(), w)


@pytest.fixture(scope="module")
def prompt():
    return synth.make_prompt(SHAPE, 32).numpy()


def _plain_sequential_greedy(model, prompt, gen_len, block):
    """Sequential greedy masked-diffusion decode written out independently:
    full forward every step, softmax over the non-mask ids with torch, unmask
    the single most confident masked position of the current block."""
    mask = model.spec.mask_id
    x = np.concatenate([prompt, np.full(gen_len, mask)])
    P = len(prompt)
    for b in range(gen_len // block):
        s = P + b * block
        for _ in range(block):
            z = torch.from_numpy(model.forward(x, range(len(x))))[s:s + block]
            z = torch.cat([z[:, :mask], z[:, mask + 1:]], dim=1)
            p = torch.softmax(z, dim=1)
            c, t = p.max(dim=1)
            t = torch.where(t >= mask, t + 1, t)
            c = torch.where(torch.from_numpy(x[s:s + block] == mask), c, torch.full_like(c, -1))
            i = int(torch.argmax(c))
            x[s + i] = int(t[i])
    return x[P:]


def test_p1_cache_off_tau_above_one_is_sequential_greedy(tiny, prompt):
    res = generate(tiny, prompt, 64, 16, 1.01, "none")
    assert res.steps == 64
    assert all(int(r.unmask.sum()) == 1 for r in res.trace)
    np.testing.assert_array_equal(res.tokens, _plain_sequential_greedy(tiny, prompt, 64, 16))


@pytest.mark.parametrize("mode", ["none", "prefix", "dual"])
def test_p4_threshold_extremes(tiny, prompt, mode):
    assert generate(tiny, prompt, 64, 16, 0.0, mode).steps == 64 // 16
    assert generate(tiny, prompt, 64, 16, -1.0, mode).steps == 64 // 16
    assert generate(tiny, prompt[:8], 32, 16, 1.01, mode).steps == 32


def test_p3_block_size_one_all_modes_equal(tiny, prompt):
    outs = [generate(tiny, prompt[:12], 8, 1, 0.9, m) for m in ("none", "prefix", "dual")]
    for o in outs[1:]:
        np.testing.assert_array_equal(o.tokens, outs[0].tokens)
        assert o.steps == outs[0].steps == 8


def test_p3_first_step_of_each_block_same_in_all_modes(tiny, prompt):
    runs = {m: generate(tiny, prompt, 64, 16, 0.9, m, keep_logits=True)
            for m in ("none", "prefix", "dual")}
    firsts = {m: [r for i, r in enumerate(res.trace) if r.kind == "refresh" or
                  (m == "none" and (i == 0 or res.trace[i - 1].block != r.block))]
              for m, res in runs.items()}
    # The first block starts from the same x in every mode.
    for m in ("prefix", "dual"):
        np.testing.assert_array_equal(firsts[m][0].z, firsts["none"][0].z)


def test_p2_dual_steps_use_a_full_recompute_of_the_block_start(tiny, prompt):
    class Recorder:
        def __init__(self, m):
            self.m, self.spec, self.calls = m, m.spec, []

        def forward(self, x, rows, cache=None, **kw):
            self.calls.append((np.array(x), np.array(rows), cache))
            return self.m.forward(x, rows, cache=cache, **kw)

    rec = Recorder(tiny)
    snaps = []
    res = generate(rec, prompt, 64, 16, 0.9, "dual", on_refresh=lambda x, kv: snaps.append((x, kv)))
    assert len(snaps) == 4
    L = len(prompt) + 64
    for x, kv in snaps:
        _, fresh = tiny.forward(x, range(L), return_kv=True)
        for (k1, v1), (k2, v2) in zip(kv, fresh):
            np.testing.assert_array_equal(k1, k2)
            np.testing.assert_array_equal(v1, v2)
    # Every cached call used the very K/V object stored by its own block's refresh.
    cached_calls = [c for c in rec.calls if c[2] is not None]
    assert len(cached_calls) == res.steps - 4
    for x, rows, cache in cached_calls:
        block = (int(rows[0]) - len(prompt)) // 16
        assert cache is snaps[block][1]


def test_exact_cache_gives_full_forward(tiny, prompt):
    rng = np.random.default_rng(0)
    x = np.concatenate([prompt, rng.integers(0, 511, 64)])
    x[40:60] = 511
    L = len(x)
    z_full, kv = tiny.forward(x, range(L), return_kv=True)
    s, e = 48, 64
    z_dual = tiny.forward(x, range(s, e), cache=kv)
    np.testing.assert_allclose(z_dual, z_full[s:e], rtol=1e-12, atol=1e-12)
    z_pre = tiny.forward(x, range(s, L), cache=kv)
    np.testing.assert_allclose(z_pre, z_full[s:], rtol=1e-12, atol=1e-12)


def test_dual_reads_prefix_and_suffix_from_cache_only(tiny, prompt):
    rng = np.random.default_rng(1)
    x = np.concatenate([prompt, np.full(64, 511)])
    L = len(x)
    _, kv = tiny.forward(x, range(L), return_kv=True)
    s, e = 48, 64
    x2 = x.copy()
    x2[s:s + 3] = [5, 6, 7]
    z = tiny.forward(x2, range(s, e), cache=kv)
    x3 = x2.copy()
    x3[:s] = rng.integers(0, 511, s)     # prefix tokens changed, cache not refreshed
    x3[e:] = rng.integers(0, 511, L - e)  # suffix tokens changed, cache not refreshed
    np.testing.assert_array_equal(tiny.forward(x3, range(s, e), cache=kv), z)
    x4 = x2.copy()
    x4[s + 5] = 9                         # a block token changed: output changes
    assert np.abs(tiny.forward(x4, range(s, e), cache=kv) - z).max() > 1e-6


def test_prefix_mode_reads_only_prefix_from_cache(tiny, prompt):
    rng = np.random.default_rng(2)
    x = np.concatenate([prompt, np.full(64, 511)])
    L = len(x)
    _, kv = tiny.forward(x, range(L), return_kv=True)
    s = 48
    z = tiny.forward(x, range(s, L), cache=kv)
    x3 = x.copy()
    x3[:s] = rng.integers(0, 511, s)
    np.testing.assert_array_equal(tiny.forward(x3, range(s, L), cache=kv), z)
    x4 = x.copy()
    x4[L - 1] = 3                         # a suffix token: recomputed fresh in prefix mode
    assert np.abs(tiny.forward(x4, range(s, L), cache=kv)[:16] - z[:16]).max() > 1e-6


def test_step_matches_generate_trace(tiny, prompt):
    res = generate(tiny, prompt, 64, 16, 0.9, "dual", keep_logits=True)
    # Replay the trace: every step's teacher-forced result equals the free run.
    mask = 511
    P = len(prompt)
    x = np.concatenate([prompt, np.full(64, mask)])
    snap = None
    for r in res.trace:
        s = P + 16 * r.block
        if r.kind == "refresh":
            snap = x.copy()
        out = step(tiny, snap, x, s, 16, 0.9, "dual")
        assert out["kind"] == r.kind
        np.testing.assert_array_equal(out["z"], r.z)
        np.testing.assert_array_equal(out["unmask"], r.unmask)
        x[s:s + 16][r.unmask] = r.tok[r.unmask]
    np.testing.assert_array_equal(x[P:], res.tokens)


def test_generated_tokens_never_mask_and_blocks_bounded(tiny, prompt):
    for mode in ("none", "prefix", "dual"):
        res = generate(tiny, prompt, 64, 16, 0.9, mode)
        assert not np.any(res.tokens == 511)
        assert all(1 <= n <= 16 for n in res.steps_per_block)
