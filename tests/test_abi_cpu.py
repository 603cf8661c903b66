"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point the header declares, and rejects bad arguments before
touching the device."""
import ctypes
import os
import re

import pytest

from kv_cache_decode_dualcache_b200 import build, fdllm, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return fdllm.load_library()


def _declared():
    text = open(os.path.join(ROOT, "include", "fdllm.h")).read()
    return sorted(set(re.findall(r"FDLLM_API\s+[\w\s\*]+?\b(fdllm_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("fdllm_create", "fdllm_load_weights", "fdllm_generate", "fdllm_destroy",
              "fdllm_step_debug", "fdllm_last_error"):
        assert n in names
    assert sorted(fdllm.EXPORTED) == names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_create_rejects_bad_configs_without_a_device(lib):
    ctx = ctypes.c_void_p()
    assert lib.fdllm_create(None, 0, None, None, ctypes.byref(ctx)) == fdllm.FDLLM_ERR_ARG
    assert b"NULL" in lib.fdllm_last_error(None)
    good = synth.TINY
    cases = {
        "d_model": 100, "head_dim": 48, "n_kv_heads": 3, "mask_id": 512, "vocab": 1,
        "ffn_dim": 0, "n_layers": 0,
    }
    for field, value in cases.items():
        cfg = fdllm.make_config(good, 96)
        setattr(cfg, field, value)
        assert lib.fdllm_create(ctypes.byref(cfg), 0, None, None, ctypes.byref(ctx)) == \
            fdllm.FDLLM_ERR_ARG, field
        assert b"device" not in lib.fdllm_last_error(None), field  # rejected before CUDA
    cfg = fdllm.make_config(good, 96)
    cfg.max_batch = 2
    assert lib.fdllm_create(ctypes.byref(cfg), 0, None, None, ctypes.byref(ctx)) == \
        fdllm.FDLLM_ERR_ARG
    cfg = fdllm.make_config(synth.SMALL_BF16, 96)
    cfg.head_dim = 32
    cfg.n_heads = 16
    assert lib.fdllm_create(ctypes.byref(cfg), 0, None, None, ctypes.byref(ctx)) == \
        fdllm.FDLLM_ERR_ARG
    # the remaining limits the header states for fdllm_config
    more = {"d_model": 8256, "max_seq": 0, "max_batch": 65, "rope_theta": 0.0,
            "rms_eps": -1.0, "logit_scale": float("nan")}
    for field, value in more.items():
        cfg = fdllm.make_config(good, 96)
        setattr(cfg, field, value)
        assert lib.fdllm_create(ctypes.byref(cfg), 0, None, None, ctypes.byref(ctx)) == \
            fdllm.FDLLM_ERR_ARG, field
        assert b"device" not in lib.fdllm_last_error(None), field
    cfg = fdllm.make_config(good, (1 << 20) + 1)
    assert lib.fdllm_create(ctypes.byref(cfg), 0, None, None, ctypes.byref(ctx)) == \
        fdllm.FDLLM_ERR_ARG
    cfg = fdllm.make_config(good, 96)
    cfg.n_heads, cfg.n_kv_heads = 3, 3                  # 3 x 32 is not a multiple of 64
    assert lib.fdllm_create(ctypes.byref(cfg), 0, None, None, ctypes.byref(ctx)) == \
        fdllm.FDLLM_ERR_ARG


def test_null_ctx_calls_are_rejected(lib):
    assert lib.fdllm_destroy(None) == 0
    assert lib.fdllm_load_weights(None, None, 0) == fdllm.FDLLM_ERR_ARG
    steps = ctypes.c_int()
    assert lib.fdllm_generate(None, None, 0, 16, 16, 0.9, 2, None, ctypes.byref(steps), None) == \
        fdllm.FDLLM_ERR_ARG
    assert lib.fdllm_launch_count(None, 0) == 0
