"""The allocation-free GEMM entry point (fdllm_gemm_noalloc).

Callers that cannot allocate device memory (a host framework that has
reserved the GPU's memory up front, or a path that must not take an
allocation's implicit synchronisation) call the GEMM through this entry
point: its split-K scratch is a fixed device array inside the library.  The
test calls it through the C ABI twice in a row and checks both results
against the context-based fdllm_gemm on the same operands, within the
tolerance the GEMM tests use.  This file is collected last, so a run that
stops at its first failure has already run every other test."""
import numpy as np
import pytest
import torch

from kv_cache_decode_dualcache_b200 import fdllm, synth
from tests.bf16_layout import pair_rows
from tests.gpu_util import make_decoder, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dec():
    require_gpu()
    shape = synth.with_layers(synth.SMALL_BF16, 1)
    return make_decoder(shape, synth.make_weights(shape, device="cpu"), 256)


@pytest.mark.parametrize("N,M,K,splits", [(384, 32, 4096, 4), (1000, 17, 512, 0),
                                          (4096, 100, 1024, 3)])
def test_noalloc_matches_context_gemm_twice(dec, N, M, K, splits):
    g = torch.Generator(device="cuda").manual_seed(N + M + K)
    w = (torch.randn(N, K, generator=g, device="cuda") * 0.05).to(torch.bfloat16)
    x = torch.randn(M, K, generator=g, device="cuda")
    xp = pair_rows(x)
    torch.cuda.synchronize()
    ref = torch.empty(M, N, device="cuda")
    fdllm.fdllm_gemm(dec.ctx, w, xp, ref, splits)
    tol = 2e-5 * np.sqrt(K) * float(w.float().abs().max()) * float(x.abs().max())
    for _ in range(2):
        y = torch.full((M, N), float("nan"), device="cuda")
        fdllm.fdllm_gemm_noalloc(w, xp, y, splits)
        torch.cuda.synchronize()
        err = float((y - ref).abs().max())
        assert np.isfinite(err) and err <= tol, (err, tol)


def test_noalloc_rejects_requests_beyond_its_scratch():
    require_gpu()
    w = torch.zeros(4096, 4096, dtype=torch.bfloat16, device="cuda")
    x = torch.zeros(2 * 4096, 4096, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(4096, 4096, device="cuda")
    with pytest.raises(fdllm.FdllmError) as e:
        fdllm.fdllm_gemm_noalloc(w, x, y, splits=16)   # 16 x 32 x 32 partial tiles > 8 MiB
    assert e.value.code == fdllm.FDLLM_ERR_ARG
    assert "8 MiB" in fdllm.fdllm_last_error(None)
