"""Pin of the oracle's whole-forward composition against an independently
written forward.

The per-layer pins (RMSNorm, RoPE, attention, SiLU) check each routine alone;
this file checks how ``oracle.model.Model.forward`` wires them together: which
normalised activation feeds which projection, which gain goes where, gate
versus up inside SwiGLU, RoPE on q and on k, where the residual additions
happen, the final norm, the LM-head scale, and how cached and fresh K/V meet in
a partial forward.  The reference below is a second, separately written float64
forward built only from torch library routines
(``torch.nn.functional.rms_norm / linear / scaled_dot_product_attention /
silu``, RoPE as a complex multiply with ``torch.polar``) following the layer
the pages attribute to LLaDA / Dream (techwalker.com Fast-dLLM article,
section "核心创新：适合扩散模型的KV缓存": a bidirectional transformer, every
position attends to every other one; ccyt168.com overview, section 一, item 1).

Every weight here is random and no gain is 1, so swapping two projections,
two gains, the gate and up matrices, or dropping RoPE from q or k changes the
logits by far more than the 1e-10 tolerance.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle.model import Model

SPEC = dict(n_layers=2, d_model=32, n_heads=4, n_kv_heads=2, head_dim=16, ffn_dim=48, vocab=37,
            mask_id=36, rope_theta=500.0, rms_eps=1e-5, logit_scale=7.0)


def _weights(seed=0):
    g = torch.Generator().manual_seed(seed)
    s = SPEC
    d, hd, H, Hkv, Fd, V = (s["d_model"], s["head_dim"], s["n_heads"], s["n_kv_heads"],
                           s["ffn_dim"], s["vocab"])

    def rnd(*shape, std=0.3):
        return torch.randn(*shape, generator=g, dtype=torch.float64) * std

    w = {"embed": rnd(V, d, std=1.0), "lm_head": rnd(V, d), "final_norm": 1.0 + rnd(d, std=0.2)}
    for i in range(s["n_layers"]):
        p = f"layers.{i}."
        w[p + "attn_norm"] = 1.0 + rnd(d, std=0.2)
        w[p + "ffn_norm"] = 1.0 + rnd(d, std=0.2)
        w[p + "wq"] = rnd(H * hd, d)
        w[p + "wk"] = rnd(Hkv * hd, d)
        w[p + "wv"] = rnd(Hkv * hd, d)
        w[p + "wo"] = rnd(d, H * hd)
        w[p + "w_gate"] = rnd(Fd, d)
        w[p + "w_up"] = rnd(Fd, d)
        w[p + "w_down"] = rnd(d, Fd)
    return w


def _rotary(t, pos, theta):
    """t: [n, heads, hd]; pairs (i, i + hd/2) rotated by pos * theta^(-2i/hd)."""
    hd = t.shape[-1]
    freqs = theta ** (-torch.arange(0, hd, 2, dtype=torch.float64) / hd)
    ang = torch.outer(pos.to(torch.float64), freqs)
    z = torch.complex(t[..., : hd // 2], t[..., hd // 2:]) * torch.polar(torch.ones_like(ang),
                                                                          ang)[:, None, :]
    return torch.cat([z.real, z.imag], dim=-1)


def reference_forward(w, x, rows, kv=None):
    """Logits of ``rows`` and the per-layer (K, V) over all positions.

    ``kv``: per layer (K [L, Hkv, hd], V [L, Hkv, hd]) for the positions not
    in ``rows`` (a partial forward); the rows' own K/V replace their entries.
    """
    s = SPEC
    d, hd, H, Hkv = s["d_model"], s["head_dim"], s["n_heads"], s["n_kv_heads"]
    x = torch.as_tensor(np.asarray(x), dtype=torch.long)
    rows = torch.as_tensor(np.asarray(rows), dtype=torch.long)
    hidden = w["embed"][x[rows]]
    out_kv = []
    for i in range(s["n_layers"]):
        p = f"layers.{i}."
        attn_in = F.rms_norm(hidden, (d,), w[p + "attn_norm"], eps=s["rms_eps"])
        q = _rotary(F.linear(attn_in, w[p + "wq"]).view(-1, H, hd), rows, s["rope_theta"])
        k = _rotary(F.linear(attn_in, w[p + "wk"]).view(-1, Hkv, hd), rows, s["rope_theta"])
        v = F.linear(attn_in, w[p + "wv"]).view(-1, Hkv, hd)
        if kv is None:
            K, V = k, v
        else:
            K, V = kv[i][0].clone(), kv[i][1].clone()
            K[rows], V[rows] = k, v
        out_kv.append((K, V))
        ctx = F.scaled_dot_product_attention(
            q.transpose(0, 1), K.transpose(0, 1).repeat_interleave(H // Hkv, dim=0),
            V.transpose(0, 1).repeat_interleave(H // Hkv, dim=0), is_causal=False)
        hidden = hidden + F.linear(ctx.transpose(0, 1).reshape(-1, H * hd), w[p + "wo"])
        ffn_in = F.rms_norm(hidden, (d,), w[p + "ffn_norm"], eps=s["rms_eps"])
        act = F.silu(F.linear(ffn_in, w[p + "w_gate"])) * F.linear(ffn_in, w[p + "w_up"])
        hidden = hidden + F.linear(act, w[p + "w_down"])
    final = F.rms_norm(hidden, (d,), w["final_norm"], eps=s["rms_eps"])
    return s["logit_scale"] * F.linear(final, w["lm_head"]), out_kv


def _model(w):
    return Model(SPEC, {k: v.numpy() for k, v in w.items()})


def _tokens(seed, L):
    rng = np.random.default_rng(seed)
    return rng.integers(0, SPEC["vocab"] - 1, size=L)


def test_full_forward_matches_independent_reference():
    w = _weights(0)
    x = _tokens(1, 19)
    z, kv = _model(w).forward(x, range(19), return_kv=True)
    z_ref, kv_ref = reference_forward(w, x, np.arange(19))
    np.testing.assert_allclose(z, z_ref.numpy(), rtol=1e-10, atol=1e-10)
    for (k, v), (kr, vr) in zip(kv, kv_ref):
        np.testing.assert_allclose(k, kr.numpy(), rtol=1e-10, atol=1e-10)
        np.testing.assert_allclose(v, vr.numpy(), rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("rows", [np.arange(8, 12), np.arange(8, 19), np.array([0, 5, 18])])
def test_partial_forward_with_stale_cache_matches_reference(rows):
    # K/V of the other positions come from an earlier sequence (the cache of a
    # previous step): both sides must take exactly those, plus fresh rows.
    w = _weights(2)
    L = 19
    x_old = _tokens(3, L)
    x_new = x_old.copy()
    x_new[rows] = _tokens(4, len(rows))
    _, kv_old = reference_forward(w, x_old, np.arange(L))
    cache = [(k.numpy(), v.numpy()) for k, v in kv_old]
    z = _model(w).forward(x_new, rows, cache=cache)
    z_ref, _ = reference_forward(w, x_new, rows, kv=kv_old)
    np.testing.assert_allclose(z, z_ref.numpy(), rtol=1e-10, atol=1e-10)
    # the cache really is stale: a full forward on x_new differs on these rows
    z_full, _ = reference_forward(w, x_new, np.arange(L))
    assert np.abs(z_full.numpy()[rows] - z).max() > 1e-6


def test_head_rows_select_lm_head_rows():
    w = _weights(5)
    x = _tokens(6, 11)
    z = _model(w).forward(x, range(11), head_rows=[3, 4, 9])
    z_ref, _ = reference_forward(w, x, np.arange(11))
    np.testing.assert_allclose(z, z_ref.numpy()[[3, 4, 9]], rtol=1e-10, atol=1e-10)
