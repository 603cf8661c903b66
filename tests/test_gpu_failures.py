"""Failure detection without a GPU fault: a device wait that runs out, an
allocator that refuses, truncated weights.  Each is reported as a status
code by the call that met it, and the context (or a new one) keeps working:
the next generation matches the float64 oracle."""
import time

import numpy as np
import pytest

from kv_cache_decode_dualcache_b200 import fdllm, synth
from oracle.decode import generate
from oracle.model import Model
from tests.gpu_util import make_decoder, require_gpu

pytestmark = pytest.mark.gpu

SHAPE = synth.TINY


def _reference():
    w = synth.make_weights(SHAPE, device="cpu")
    prompt = synth.make_prompt(SHAPE, 32).numpy()
    ref = generate(Model(SHAPE.as_dict(), w), prompt, 64, 16, 0.9, "dual")
    return w, prompt, ref


def _decodes_correctly(dec, prompt, ref):
    out, steps, _ = dec.generate(prompt, 64, 16, 0.9, "dual")
    return np.array_equal(out, ref.tokens) and steps == ref.steps


def test_device_wait_that_runs_out_is_reported_and_the_context_stays_usable():
    require_gpu()
    w, prompt, ref = _reference()
    dec = make_decoder(SHAPE, w, 96)
    lib = fdllm.load_library()
    t0 = time.perf_counter()
    rc = lib.fdllm_selftest_wait_timeout(dec.ctx)
    took = time.perf_counter() - t0
    assert rc == fdllm.FDLLM_ERR_TIMEOUT
    assert "timed out" in fdllm.fdllm_last_error(dec.ctx)
    assert 1.5 < took < 30.0          # the wait's limit is 2 s
    assert _decodes_correctly(dec, prompt, ref)
    dec.close()


class _RefusingAllocator(fdllm.TorchAllocator):
    """Torch's allocator, except that it answers NULL while `refuse` is set."""

    def __init__(self, device):
        super().__init__(device)
        self.refuse = False

    def _alloc(self, nbytes, user):
        return None if self.refuse else super()._alloc(nbytes, user)


def test_allocator_refusal_is_reported_as_oom():
    require_gpu()
    from kv_cache_decode_dualcache_b200 import build
    build.build()
    w, prompt, ref = _reference()
    # refused during creation: no context comes back
    alloc = _RefusingAllocator(0)
    alloc.refuse = True
    with pytest.raises(fdllm.FdllmError) as e:
        fdllm.fdllm_create(SHAPE, 96, 0, None, alloc)
    assert e.value.code == fdllm.FDLLM_ERR_OOM
    # refused for the weights: that call fails, the context stays usable
    alloc.refuse = False
    ctx = fdllm.fdllm_create(SHAPE, 96, 0, None, alloc)
    alloc.refuse = True
    with pytest.raises(fdllm.FdllmError) as e:
        fdllm.fdllm_load_weights(ctx, w, SHAPE.dtype)
    assert e.value.code == fdllm.FDLLM_ERR_OOM
    with pytest.raises(fdllm.FdllmError) as e:      # nothing to decode with yet
        fdllm.fdllm_generate(ctx, prompt, 64, 16, 0.9, "dual")
    assert e.value.code == fdllm.FDLLM_ERR_STATE
    alloc.refuse = False
    fdllm.fdllm_load_weights(ctx, w, SHAPE.dtype)
    out, steps = fdllm.fdllm_generate(ctx, prompt, 64, 16, 0.9, "dual")
    assert np.array_equal(out, ref.tokens) and steps == ref.steps
    fdllm.fdllm_destroy(ctx)


def test_truncated_or_missing_weights_are_rejected():
    require_gpu()
    import os

    from kv_cache_decode_dualcache_b200 import build
    build.build(checks=os.environ.get("FDLLM_CHECKS") == "1")
    w, prompt, ref = _reference()
    dec = fdllm.Decoder(SHAPE, 96)                          # no weights yet
    bad = dict(w)
    bad["lm_head"] = w["lm_head"].reshape(-1)[:-1]          # one value short
    with pytest.raises(fdllm.FdllmError) as e:
        dec.load_weights(bad)
    assert e.value.code == fdllm.FDLLM_ERR_SHAPE
    missing = {k: v for k, v in w.items() if k != "layers.1.w_down"}
    with pytest.raises(fdllm.FdllmError) as e:
        dec.load_weights(missing)
    assert e.value.code == fdllm.FDLLM_ERR_SHAPE
    dec.load_weights(w)                                     # a correct set still loads
    assert _decodes_correctly(dec, prompt, ref)
    dec.close()
