"""fdllm_generate_batch: independent sequences of different prompt lengths
(variable-length serving) give exactly the single-sequence results.

Tiny fp32 model: every sequence's tokens and step count equal the float64
oracle's free-running decode of that sequence alone (the oracle's own
batched-decode reading: per-sequence block schedules, nothing shared).
Reduced bf16 model: the batch equals fdllm_generate run on each sequence
alone, bit for bit."""
import numpy as np
import pytest

from kv_cache_decode_dualcache_b200 import synth
from oracle.decode import generate
from oracle.model import Model
from tests.gpu_util import make_decoder, require_gpu

pytestmark = pytest.mark.gpu


def _prompts(shape, lens, salt0=10):
    return [synth.make_prompt(shape, n, salt=salt0 + i).numpy() for i, n in enumerate(lens)]


def test_batch_tiny_matches_oracle():
    require_gpu()
    shape = synth.TINY
    w = synth.make_weights(shape, device="cpu")
    dec = make_decoder(shape, w, 96)
    lens, G, B, tau = [20, 32, 9], 48, 16, 0.9
    prompts = _prompts(shape, lens)
    out, steps, stats = dec.generate_batch(prompts, G, B, tau, "dual")
    model = Model(shape.as_dict(), w)
    for i, p in enumerate(prompts):
        ref = generate(model, p, G, B, tau, "dual")
        assert np.array_equal(out[i], ref.tokens), i
        assert steps[i] == ref.steps
    assert stats.steps == int(steps.sum())
    assert len(stats.steps_per_block) == len(lens) * (G // B)
    dec.close()


@pytest.mark.parametrize("mode", ["dual", "prefix"])
def test_batch_bf16_equals_single(mode):
    require_gpu()
    shape = synth.SMALL_BF16
    dec = make_decoder(shape, synth.make_weights(shape, device="cpu"), 256)
    lens, G, B, tau = [128, 40, 71, 200], 32, 16, 0.9
    prompts = _prompts(shape, lens, salt0=30)
    out, steps, _ = dec.generate_batch(prompts, G, B, tau, mode)
    for i, p in enumerate(prompts):
        one, n1, _ = dec.generate(p, G, B, tau, mode)
        assert np.array_equal(out[i], one), i
        assert steps[i] == n1
    dec.close()


def test_batch_rejects_any_bad_sequence():
    require_gpu()
    from kv_cache_decode_dualcache_b200.fdllm import FdllmError
    shape = synth.TINY
    dec = make_decoder(shape, synth.make_weights(shape, device="cpu"), 96)
    good = synth.make_prompt(shape, 16).numpy()
    bad = good.copy()
    bad[3] = shape.mask_id
    with pytest.raises(FdllmError):
        dec.generate_batch([good, bad], 32, 16, 0.9, "dual")
    too_long = synth.make_prompt(shape, 80).numpy()
    with pytest.raises(FdllmError):
        dec.generate_batch([good, too_long], 32, 16, 0.9, "dual")
    dec.close()
