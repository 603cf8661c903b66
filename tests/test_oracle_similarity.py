"""Pins of the oracle's K/V similarity (oracle/similarity.py): closed forms,
a brute-force loop on a tiny input, and what the model's structure fixes."""
import math

import numpy as np

from kv_cache_decode_dualcache_b200 import synth
from oracle.model import Model
from oracle.similarity import kv_cosine, step_kv_cosine


def _kv(k, v):
    return [(np.asarray(k, dtype=np.float64), np.asarray(v, dtype=np.float64))]


def test_closed_forms():
    # positions: parallel, 45 degrees, orthogonal, opposite; one KV head of 2 dims
    a = [[[1.0, 0.0]], [[1.0, 0.0]], [[1.0, 0.0]], [[1.0, 2.0]]]
    b = [[[3.0, 0.0]], [[1.0, 1.0]], [[0.0, 5.0]], [[-2.0, -4.0]]]
    c = kv_cosine(_kv(a, a), _kv(b, a))
    assert c.shape == (1, 2, 4)
    np.testing.assert_allclose(c[0, 0], [1.0, 1.0 / math.sqrt(2.0), 0.0, -1.0], atol=1e-15)
    np.testing.assert_allclose(c[0, 1], [1.0, 1.0, 1.0, 1.0], atol=1e-15)


def test_invariant_to_positive_scale_at_any_norm():
    # cos(s a, t b) = cos(a, b) for s, t > 0, also when the norms' product is
    # below 1 (K/V of N(0, 0.02) weights have small norms)
    rng = np.random.default_rng(7)
    a = rng.standard_normal((6, 2, 4))
    b = rng.standard_normal((6, 2, 4))
    ref = kv_cosine(_kv(a, b), _kv(b, a))
    for s, t in ((1e-3, 1.0), (1e-3, 2e-4), (50.0, 1e-2)):
        np.testing.assert_allclose(kv_cosine(_kv(s * a, t * b), _kv(t * b, s * a)), ref,
                                   rtol=1e-12, atol=1e-14)


def test_zero_vectors():
    z = np.zeros((2, 1, 3))
    nz = np.ones((2, 1, 3))
    np.testing.assert_array_equal(kv_cosine(_kv(z, z), _kv(z, nz))[0], [[1.0, 1.0], [0.0, 0.0]])


def test_against_a_plain_loop():
    rng = np.random.default_rng(5)
    kv_a = [(rng.standard_normal((5, 2, 4)), rng.standard_normal((5, 2, 4))) for _ in range(3)]
    kv_b = [(rng.standard_normal((5, 2, 4)), rng.standard_normal((5, 2, 4))) for _ in range(3)]
    c = kv_cosine(kv_a, kv_b)
    for li in range(3):
        for kv in range(2):
            for p in range(5):
                x = [float(t) for t in kv_a[li][kv][p].ravel()]
                y = [float(t) for t in kv_b[li][kv][p].ravel()]
                dot = sum(i * j for i, j in zip(x, y))
                ref = dot / (math.sqrt(sum(i * i for i in x)) * math.sqrt(sum(j * j for j in y)))
                assert abs(c[li, kv, p] - ref) < 1e-14


def _tiny():
    shape = synth.TINY
    return shape, Model(shape.as_dict(), synth.make_weights(shape, device="cpu"))


def test_same_sequence_is_identical():
    shape, model = _tiny()
    x = np.concatenate([synth.make_prompt(shape, 32).numpy(), np.full(16, shape.mask_id)])
    np.testing.assert_allclose(step_kv_cosine(model, x, x), 1.0, atol=1e-14)


def test_layer0_changes_only_where_the_token_changed():
    # layer-0 K/V of a position depend only on its token and its position;
    # from layer 1 on, bidirectional attention carries the change to every
    # position (the prefix too, not only the positions after it)
    shape, model = _tiny()
    prompt = synth.make_prompt(shape, 32).numpy()
    x_a = np.concatenate([prompt, np.full(16, shape.mask_id)])
    x_b = x_a.copy()
    x_b[[33, 36, 40]] = [7, 100, 200]
    c = step_kv_cosine(model, x_a, x_b)
    same = np.setdiff1d(np.arange(48), [33, 36, 40])
    np.testing.assert_allclose(c[0, :, same], 1.0, atol=1e-14)
    assert (c[0, :, [33, 36, 40]] < 1.0 - 1e-6).all()
    assert (c[1, :, :32] < 1.0 - 1e-12).all()
