"""fdllm_generate_fixed_k against the float64 oracle: the tiny fp32 model
decoded free-running with k = 1, 3 and the whole block, in DualCache and
cache-off modes, gives the oracle's tokens and step counts exactly; the
reduced bf16 model gives ceil(B / k) steps per block and k = 1 the same
sequence as tau > 1 (both pick the single most confident position)."""
import numpy as np
import pytest

from kv_cache_decode_dualcache_b200 import synth
from oracle.decode import generate
from oracle.model import Model
from tests.gpu_util import make_decoder, require_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode", ["dual", "none"])
@pytest.mark.parametrize("k", [1, 3, 16])
def test_fixed_k_tiny_matches_oracle(mode, k):
    require_gpu()
    shape = synth.TINY
    w = synth.make_weights(shape, device="cpu")
    dec = make_decoder(shape, w, 96)
    prompt = synth.make_prompt(shape, 32).numpy()
    out, steps, st = dec.generate(prompt, 64, 16, 0.9, mode, fixed_k=k)
    ref = generate(Model(shape.as_dict(), w), prompt, 64, 16, 0.9, mode, fixed_k=k)
    assert np.array_equal(out, ref.tokens)
    assert steps == ref.steps and st.steps_per_block == ref.steps_per_block
    dec.close()


def test_fixed_k_bf16_step_counts():
    require_gpu()
    shape = synth.SMALL_BF16
    dec = make_decoder(shape, synth.make_weights(shape, device="cpu"), 256)
    prompt = synth.make_prompt(shape, 64).numpy()
    G, B = 64, 32
    for k in (4, 7):
        out, steps, st = dec.generate(prompt, G, B, 0.9, "dual", fixed_k=k)
        assert st.steps_per_block == [-(-B // k)] * (G // B)
        assert not np.any(out == shape.mask_id)
    one, _, _ = dec.generate(prompt, G, B, 0.9, "dual", fixed_k=1)
    greedy, _, _ = dec.generate(prompt, G, B, 1.01, "dual")
    assert np.array_equal(one, greedy)
    dec.close()
