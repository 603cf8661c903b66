"""fdllm_kv_similarity (full forward over each of two sequences, cosine of
their K/V per layer and position) against the float64 oracle's
step_kv_cosine, on the tiny float32 and the reduced bfloat16 models."""
import numpy as np
import pytest

from kv_cache_decode_dualcache_b200 import synth
from oracle.decode import step
from oracle.model import Model
from oracle.similarity import step_kv_cosine
from tests.gpu_util import make_decoder, require_gpu

pytestmark = pytest.mark.gpu


def _sequences(shape, model, P, G, B):
    """The sequence at the first block's start and the one after its first
    step (the oracle's own unmask decisions)."""
    prompt = synth.make_prompt(shape, P).numpy()
    x_a = np.concatenate([prompt, np.full(G, shape.mask_id)])
    r = step(model, x_a, x_a, P, B, 0.9, "dual")
    x_b = x_a.copy()
    x_b[P:P + B][r["unmask"]] = r["tok"][r["unmask"]]
    assert (x_b != x_a).any()
    return x_a, x_b


@pytest.mark.parametrize("name,P,G,B,tol", [("tiny-fp32", 32, 64, 16, 1e-5),
                                            ("small-bf16", 40, 64, 32, 1e-4),
                                            ("small-gqa-bf16", 40, 64, 32, 1e-4)])
def test_kv_similarity_matches_oracle(name, P, G, B, tol):
    require_gpu()
    shape = synth.SHAPES[name]
    w = synth.make_weights(shape, device="cpu")
    model = Model(shape.as_dict(), w)
    dec = make_decoder(shape, w, P + G)
    x_a, x_b = _sequences(shape, model, P, G, B)
    got = dec.kv_similarity(x_a, x_b)
    ref = step_kv_cosine(model, x_a, x_b)
    assert got.shape == ref.shape == (shape.n_layers, 2, P + G)
    err = float(np.abs(got - ref).max())
    print(f"{name}: max |dcos| {err:.3g}; min cos per layer (K) {ref[:, 0].min(axis=1)}")
    assert err <= tol
    # layer 0: unchanged tokens keep bit-identical K/V
    same = np.nonzero(x_a == x_b)[0]
    np.testing.assert_allclose(got[0][:, same], 1.0, atol=1e-12)
    # the same sequence twice: identical K/V everywhere
    np.testing.assert_allclose(dec.kv_similarity(x_b, x_b), 1.0, atol=1e-12)
    dec.close()


def test_kv_similarity_rejects_bad_arguments():
    require_gpu()
    from kv_cache_decode_dualcache_b200 import fdllm
    shape = synth.TINY
    dec = make_decoder(shape, synth.make_weights(shape, device="cpu"), 64)
    x = np.zeros(64, dtype=np.int32)
    with pytest.raises(fdllm.FdllmError):
        dec.kv_similarity(x, np.full(64, shape.vocab, dtype=np.int32))   # id out of range
    with pytest.raises(fdllm.FdllmError):
        dec.kv_similarity(np.zeros(65, dtype=np.int32), np.zeros(65, dtype=np.int32))  # L > max_seq
    dec.close()
