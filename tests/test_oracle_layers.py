"""Pins for the oracle's layer math (RMSNorm, RoPE, attention) against torch
CPU float64 library routines, closed forms and invariants."""
import numpy as np
import torch

from oracle.model import attention, rmsnorm, rope


def test_rmsnorm_matches_torch():
    rng = np.random.default_rng(0)
    h = rng.standard_normal((9, 256)) * 3
    g = rng.standard_normal(256)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(h), (256,), torch.from_numpy(g), eps=1e-5)
    np.testing.assert_allclose(rmsnorm(h, g, 1e-5), ref.numpy(), rtol=1e-13)


def test_rmsnorm_eps_inside_sqrt_closed_form():
    h = np.array([[2.0, 0.0, 0.0, 0.0]])  # mean(h^2) = 1
    out = rmsnorm(h, np.ones(4), 0.25)
    np.testing.assert_allclose(out, [[2.0 / np.sqrt(1.25), 0, 0, 0]], rtol=1e-15)


def _rope_complex(x, pos, theta):
    """Same rotation written as a complex multiply of (x[i] + i x[i+hd/2])."""
    hd = x.shape[-1]
    half = hd // 2
    xt = torch.from_numpy(x)
    zc = torch.complex(xt[..., :half], xt[..., half:])
    freqs = 1.0 / (theta ** (torch.arange(0, hd, 2, dtype=torch.float64) / hd))
    ang = torch.outer(torch.from_numpy(pos).double(), freqs)
    rot = torch.polar(torch.ones_like(ang), ang)[:, None, :]
    r = zc * rot
    return torch.cat([r.real, r.imag], dim=-1).numpy()


def test_rope_matches_complex_rotation():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((11, 3, 64))
    pos = np.array([0, 1, 2, 7, 31, 32, 100, 511, 1000, 2047, 4095])
    for theta in (1e4, 1e6):
        np.testing.assert_allclose(rope(x, pos, theta), _rope_complex(x, pos, theta),
                                   rtol=1e-12, atol=1e-12)


def test_rope_identity_at_zero_and_norm_preserving():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 2, 32))
    np.testing.assert_array_equal(rope(x, np.zeros(5, dtype=np.int64), 1e4), x)
    y = rope(x, np.arange(5) * 13, 1e4)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)


def test_rope_scores_depend_only_on_relative_position():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 1, 128))
    k = rng.standard_normal((1, 1, 128))
    base = (rope(q, np.array([40]), 1e4) * rope(k, np.array([17]), 1e4)).sum()
    shifted = (rope(q, np.array([140]), 1e4) * rope(k, np.array([117]), 1e4)).sum()
    np.testing.assert_allclose(base, shifted, rtol=1e-10)


def test_attention_matches_torch_sdpa_no_mask_gqa():
    rng = np.random.default_rng(4)
    M, L, H, Hkv, hd = 7, 23, 8, 2, 16
    q = rng.standard_normal((M, H, hd))
    k = rng.standard_normal((L, Hkv, hd))
    v = rng.standard_normal((L, Hkv, hd))
    qt = torch.from_numpy(q).permute(1, 0, 2)                       # [H, M, hd]
    kt = torch.from_numpy(k).permute(1, 0, 2).repeat_interleave(H // Hkv, dim=0)
    vt = torch.from_numpy(v).permute(1, 0, 2).repeat_interleave(H // Hkv, dim=0)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=False)
    np.testing.assert_allclose(attention(q, k, v), ref.permute(1, 0, 2).numpy(), rtol=1e-12,
                               atol=1e-12)


def test_attention_equal_keys_average_all_values_bidirectionally():
    # With identical keys every query weights every position equally, including
    # positions after it: the output is the plain mean of all values.
    rng = np.random.default_rng(5)
    L, hd = 9, 8
    k = np.tile(rng.standard_normal((1, 1, hd)), (L, 1, 1))
    v = rng.standard_normal((L, 1, hd))
    q = rng.standard_normal((3, 1, hd))
    out = attention(q, k, v)
    for m in range(3):
        np.testing.assert_allclose(out[m, 0], v[:, 0, :].mean(axis=0), rtol=1e-13)


def test_attention_is_stable_for_large_scores():
    # scores of several thousand (far beyond exp's range) must give the same
    # softmax as torch's float64 attention: the max shift is per query row
    rng = np.random.default_rng(6)
    M, L, H, hd = 5, 13, 2, 8
    q = rng.standard_normal((M, H, hd)) * 300.0
    k = rng.standard_normal((L, H, hd)) * 30.0
    v = rng.standard_normal((L, H, hd))
    qt = torch.from_numpy(q).permute(1, 0, 2)
    kt = torch.from_numpy(k).permute(1, 0, 2)
    vt = torch.from_numpy(v).permute(1, 0, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=False)
    out = attention(q, k, v)
    assert np.isfinite(out).all()
    np.testing.assert_allclose(out, ref.permute(1, 0, 2).numpy(), rtol=1e-9, atol=1e-9)
