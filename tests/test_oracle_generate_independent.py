"""Pins of the oracle's decode loop wiring: which rows each cache mode
recomputes, which K/V it reads, which rows feed the LM head.

1. Against an independently written decode loop built on the separately
   written torch forward of ``test_oracle_forward_independent`` (the block
   procedure of the techwalker.com Fast-dLLM article, section
   "核心创新：适合扩散模型的KV缓存": a block's first step is a full forward whose
   K/V is kept; DualCache steps recompute the block rows over the kept K/V of
   every other position; prefix-cache steps recompute every position from the
   block start on over the kept prefix; the threshold rule of the ccyt168.com
   overview, section 一, item 2).  Every step's logits must agree to 1e-10,
   and the unmask sets, tokens and step counts exactly.
2. A property that needs no second implementation: in a one-layer model the
   K and V of a position depend on that position's token alone (they are
   projections of its normalised embedding), and within a block only the
   block's tokens change, so the K/V kept at the block start stays exact for
   every position outside the block.  DualCache, prefix-cache and cache-off
   decoding must then take the same steps with the same logits (up to
   rounding order) and return the same tokens.
"""
import numpy as np
import pytest
import torch

from oracle.decode import generate, step
from oracle.model import Model
from tests.test_oracle_forward_independent import SPEC, _weights, reference_forward

MASK = SPEC["mask_id"]


def _reference_decode(w, prompt, gen_len, block, tau, mode):
    """Block-wise threshold decode written out on the torch reference forward.
    Returns the tokens and, per step, (kind, logits of the block rows, unmask)."""
    P = len(prompt)
    L = P + gen_len
    x = np.concatenate([np.asarray(prompt), np.full(gen_len, MASK)]).astype(np.int64)
    steps = []
    for s in range(P, L, block):
        e = s + block
        kept = None
        while (x[s:e] == MASK).any():
            if kept is None:
                z_all, kept = reference_forward(w, x, np.arange(L))
                z, kind = z_all[s:e], "refresh"
            elif mode == "none":
                z_all, _ = reference_forward(w, x, np.arange(L))
                z, kind = z_all[s:e], "full"
            elif mode == "dual":
                z, _ = reference_forward(w, x, np.arange(s, e), kv=kept)
                kind = "dual"
            else:
                z_all, _ = reference_forward(w, x, np.arange(s, L), kv=kept)
                z, kind = z_all[:block], "prefix"
            probs = torch.softmax(torch.cat([z[:, :MASK], z[:, MASK + 1:]], dim=1), dim=1)
            conf, tok = probs.max(dim=1)
            tok = torch.where(tok >= MASK, tok + 1, tok).numpy()
            conf = conf.numpy()
            masked = x[s:e] == MASK
            u = masked & (conf >= tau)
            if not u.any():
                best = max(np.flatnonzero(masked), key=lambda i: conf[i])
                u[best] = True
            x[s:e][u] = tok[u]
            steps.append((kind, z.numpy(), u.copy()))
    return x[P:], steps


def _prompt(seed, n):
    return np.random.default_rng(seed).integers(0, MASK, size=n)


@pytest.mark.parametrize("mode", ["dual", "prefix", "none"])
@pytest.mark.parametrize("tau", [0.9, 1.01])
def test_generate_matches_independent_decode(mode, tau):
    w = _weights(7)
    model = Model(SPEC, {k: v.numpy() for k, v in w.items()})
    prompt = _prompt(8, 5)
    res = generate(model, prompt, 12, 4, tau, mode, keep_logits=True)
    tokens, ref_steps = _reference_decode(w, prompt, 12, 4, tau, mode)
    assert res.steps == len(ref_steps)
    assert res.steps > 12 // 4                       # cached steps happen
    if tau < 1:                                      # and parallel unmasking
        assert any(int(r.unmask.sum()) > 1 for r in res.trace)
    for r, (kind, z, u) in zip(res.trace, ref_steps):
        assert r.kind == kind
        np.testing.assert_allclose(r.z, z, rtol=1e-10, atol=1e-10)
        np.testing.assert_array_equal(r.unmask, u)
    np.testing.assert_array_equal(res.tokens, tokens)


@pytest.mark.parametrize("mode", ["prefix", "none"])
def test_teacher_forced_step_matches_generate_in_every_mode(mode):
    w = _weights(9)
    model = Model(SPEC, {k: v.numpy() for k, v in w.items()})
    prompt = _prompt(10, 6)
    res = generate(model, prompt, 12, 4, 0.9, mode, keep_logits=True)
    assert res.steps > 12 // 4
    P = len(prompt)
    x = np.concatenate([prompt, np.full(12, MASK)]).astype(np.int64)
    snap = None
    for r in res.trace:
        s = P + 4 * r.block
        if r.kind == "refresh":
            snap = x.copy()
        out = step(model, snap, x, s, 4, 0.9, mode)
        np.testing.assert_allclose(out["z"], r.z, rtol=1e-12, atol=1e-12)
        np.testing.assert_array_equal(out["unmask"], r.unmask)
        x[s:s + 4][r.unmask] = r.tok[r.unmask]
    np.testing.assert_array_equal(x[P:], res.tokens)


def test_one_layer_model_caches_are_exact_so_all_modes_agree():
    spec = dict(SPEC, n_layers=1)
    g = torch.Generator().manual_seed(11)
    d, hd, H, Hkv, F, V = (spec["d_model"], spec["head_dim"], spec["n_heads"],
                           spec["n_kv_heads"], spec["ffn_dim"], spec["vocab"])
    rnd = lambda *s, std=0.3: (torch.randn(*s, generator=g, dtype=torch.float64) * std).numpy()
    w = {"embed": rnd(V, d, std=1.0), "lm_head": rnd(V, d), "final_norm": 1.0 + rnd(d, std=0.2),
         "layers.0.attn_norm": 1.0 + rnd(d, std=0.2), "layers.0.ffn_norm": 1.0 + rnd(d, std=0.2),
         "layers.0.wq": rnd(H * hd, d), "layers.0.wk": rnd(Hkv * hd, d),
         "layers.0.wv": rnd(Hkv * hd, d), "layers.0.wo": rnd(d, H * hd),
         "layers.0.w_gate": rnd(F, d), "layers.0.w_up": rnd(F, d), "layers.0.w_down": rnd(d, F)}
    model = Model(spec, w)
    prompt = _prompt(12, 7)
    for tau in (0.9, 1.01):
        runs = {m: generate(model, prompt, 16, 4, tau, m, keep_logits=True)
                for m in ("none", "prefix", "dual")}
        ref = runs["none"]
        assert ref.steps > 16 // 4          # cached steps happen
        for m in ("prefix", "dual"):
            assert runs[m].steps == ref.steps
            np.testing.assert_array_equal(runs[m].tokens, ref.tokens)
            for a, b in zip(runs[m].trace, ref.trace):
                np.testing.assert_allclose(a.z, b.z, rtol=1e-11, atol=1e-11)
                np.testing.assert_array_equal(a.unmask, b.unmask)
