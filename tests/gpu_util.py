"""Helpers for GPU tests: build the library, create a decoder with weights."""
from __future__ import annotations

import pytest


def require_gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def make_decoder(shape, weights, max_seq: int, max_batch: int = 1):
    import os
    from kv_cache_decode_dualcache_b200 import build, fdllm
    build.build(checks=os.environ.get("FDLLM_CHECKS") == "1")
    dec = fdllm.Decoder(shape, max_seq, max_batch=max_batch)
    dec.load_weights(weights)
    return dec
