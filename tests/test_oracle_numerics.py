"""Pins for oracle.numerics against independent library routines."""
import numpy as np
import pytest
import torch

from oracle.numerics import logsumexp, round_bf16, round_f32, silu


def test_round_bf16_matches_torch_rne():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(200_000) * 10.0 ** rng.integers(-6, 6, 200_000),
        # exact halfway cases between two bf16 neighbours (ties to even both ways)
        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 2.0 ** -130 * 1.5]),
    ])
    got = round_bf16(x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(got, ref)


def test_round_bf16_is_idempotent_and_representable():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(10_000)
    r = round_bf16(x)
    np.testing.assert_array_equal(round_bf16(r), r)
    u = r.astype(np.float32).view(np.uint32)
    assert np.all((u & 0xFFFF) == 0)


def test_round_f32_matches_numpy_cast():
    x = np.random.default_rng(2).standard_normal(1000) * 1e3
    np.testing.assert_array_equal(round_f32(x), x.astype(np.float32).astype(np.float64))


def test_silu_matches_torch():
    x = np.linspace(-800, 800, 100_001)
    ref = torch.nn.functional.silu(torch.from_numpy(x)).numpy()
    np.testing.assert_allclose(silu(x), ref, rtol=1e-14, atol=1e-300)
    assert silu(np.array([0.0]))[0] == 0.0


def test_logsumexp_matches_torch_and_ignores_minus_inf():
    rng = np.random.default_rng(3)
    z = rng.standard_normal((7, 333)) * 50
    ref = torch.logsumexp(torch.from_numpy(z), dim=1).numpy()
    np.testing.assert_allclose(logsumexp(z, axis=1), ref, rtol=1e-13)
    z2 = z.copy()
    z2[:, 5] = -np.inf
    ref2 = torch.logsumexp(torch.from_numpy(np.delete(z, 5, axis=1)), dim=1).numpy()
    np.testing.assert_allclose(logsumexp(z2, axis=1), ref2, rtol=1e-13)
