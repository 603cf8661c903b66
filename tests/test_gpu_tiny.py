"""Tiny float32 model: the CUDA decoder against the oracle.

Free-running sequences and step counts must be identical in every cache
mode for tau = 0.9 and tau = 1.01; teacher-forced steps must match the
oracle's logits within 1e-4 and confidences within 1e-3."""
import numpy as np
import pytest

from kv_cache_decode_dualcache_b200 import synth
from oracle.decode import generate
from oracle.model import Model
from tests.gpu_util import make_decoder, require_gpu
from tests.parity import teacher_forced

pytestmark = pytest.mark.gpu
SHAPE = synth.TINY


@pytest.fixture(scope="module")
def setup():
    require_gpu()
    w = synth.make_weights(SHAPE, device="cpu")
    model = Model(SHAPE.as_dict(), w)
    dec = make_decoder(SHAPE, w, 128)
    prompt = synth.make_prompt(SHAPE, 32).numpy()
    return model, dec, prompt


@pytest.mark.parametrize("mode", ["dual", "prefix", "none"])
@pytest.mark.parametrize("tau", [0.9, 1.01])
def test_free_running_identical(setup, mode, tau):
    model, dec, prompt = setup
    ref = generate(model, prompt, 64, 16, tau, mode)
    out, steps, stats = dec.generate(prompt, 64, 16, tau, mode)
    np.testing.assert_array_equal(out, ref.tokens)
    assert steps == ref.steps
    assert stats.steps_per_block == ref.steps_per_block


@pytest.mark.parametrize("mode", ["dual", "prefix", "none"])
def test_teacher_forced_logits(setup, mode):
    model, dec, prompt = setup
    ref = generate(model, prompt, 64, 16, 0.9, mode, keep_logits=True)
    rep = teacher_forced(dec, model, ref.trace, prompt, 64, 16, 0.9, mode, SHAPE.mask_id,
                         z_tol=1e-4, stride=3)
    assert not rep.mismatches, rep.mismatches[:5]
    assert rep.max_dz <= 1e-4


def test_threshold_extremes_and_block_size_one(setup):
    model, dec, prompt = setup
    out, steps, _ = dec.generate(prompt, 64, 16, 0.0, "dual")
    assert steps == 4
    np.testing.assert_array_equal(out, generate(model, prompt, 64, 16, 0.0, "dual").tokens)
    outs = [dec.generate(prompt[:12], 8, 1, 0.9, m)[0] for m in ("none", "prefix", "dual")]
    assert all(np.array_equal(outs[0], o) for o in outs[1:])


def test_ragged_prompt_and_odd_positions(setup):
    model, dec, prompt = setup
    p = prompt[:13]
    ref = generate(model, p, 48, 16, 0.9, "dual")
    out, steps, _ = dec.generate(p, 48, 16, 0.9, "dual")
    np.testing.assert_array_equal(out, ref.tokens)
    assert steps == ref.steps
