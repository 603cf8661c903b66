"""Reduced bfloat16 models on the tensor-core path against the float64 oracle
(teacher-forced per step): logits within 3e-2, confidences within 1e-3,
tokens and unmask sets identical outside near ties.
Sizes span several GEMM tiles, ragged vocab / FFN tails, a prompt and
blocks that are not aligned to the 64-position KV pages, MHA and GQA."""
import numpy as np
import pytest

from kv_cache_decode_dualcache_b200 import synth
from oracle.decode import generate
from oracle.model import Model
from tests.gpu_util import make_decoder, require_gpu
from tests.parity import teacher_forced

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", params=["small-bf16", "small-gqa-bf16"])
def setup(request):
    require_gpu()
    shape = synth.SHAPES[request.param]
    w = synth.make_weights(shape, device="cpu")
    model = Model(shape.as_dict(), w)
    dec = make_decoder(shape, w, 256)
    prompt = synth.make_prompt(shape, 40).numpy()
    return shape, model, dec, prompt


@pytest.mark.parametrize("mode", ["dual", "prefix", "none"])
def test_teacher_forced_bf16(setup, mode):
    shape, model, dec, prompt = setup
    ref = generate(model, prompt, 64, 32, 0.9, mode, keep_logits=True)
    rep = teacher_forced(dec, model, ref.trace, prompt, 64, 32, 0.9, mode, shape.mask_id,
                         z_tol=3e-2)
    print(f"{shape.name} {mode}: steps {rep.steps} max|dz| {rep.max_dz:.3g} "
          f"max|dconf| {rep.max_dconf:.3g} exempt {rep.exempt}")
    assert not rep.mismatches, rep.mismatches[:5]


def test_refresh_kv_is_a_full_recompute(setup):
    shape, model, dec, prompt = setup
    L = 104
    rng = np.random.default_rng(0)
    x = np.concatenate([prompt, np.full(64, shape.mask_id)])
    cur = x.copy()
    cur[40:50] = rng.integers(0, shape.vocab - 1, 10)
    dec.step_debug(x, x, 40, 32, 0.9, "dual", logits=False)
    kv1 = [dec.read_kv(l, 0, L) for l in range(shape.n_layers)]
    dec.step_debug(x, cur, 40, 32, 0.9, "dual", logits=False)   # overwrites block rows
    dec.step_debug(x, x, 40, 32, 0.9, "dual", logits=False)     # refresh again
    kv2 = [dec.read_kv(l, 0, L) for l in range(shape.n_layers)]
    for (k1, v1), (k2, v2) in zip(kv1, kv2):
        np.testing.assert_array_equal(k1, k2)
        np.testing.assert_array_equal(v1, v2)
    _, okv = model.forward(x, range(L), return_kv=True)
    for (k, v), (ok, ov) in zip(kv1, okv):
        assert np.abs(k - ok).max() <= 2e-4 * max(1.0, np.abs(ok).max())
        assert np.abs(v - ov).max() <= 2e-4 * max(1.0, np.abs(ov).max())
