"""The decoder's GEMM (tcgen05 on the bf16 model) against a float64 matmul of
the same operands: bf16 weights times two-term (hi + lo) activations, over
token-tile widths, K splits and ragged N / M."""
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


@pytest.mark.parametrize("N,M,K,splits", [
    (128, 32, 64, 1), (256, 32, 512, 0), (1000, 17, 512, 1), (384, 32, 4096, 4),
    (130, 64, 256, 0), (512, 100, 512, 0), (640, 256, 1024, 0), (256, 300, 512, 3),
    (4096, 32, 1024, 0), (257, 5, 128, 2), (12288, 32, 4096, 0), (4096, 512, 4096, 0),
])
def test_gemm_matches_float64(dec, N, M, K, splits):
    g = torch.Generator(device="cuda").manual_seed(N * 7 + M * 3 + K)
    w = (torch.randn(N, K, generator=g, device="cuda") * 0.05).to(torch.bfloat16)
    x = torch.randn(M, K, generator=g, device="cuda")
    xp = pair_rows(x)
    y = torch.full((M, N), float("nan"), device="cuda")
    fdllm.fdllm_gemm(dec.ctx, w, xp, y, splits)
    torch.cuda.synchronize()
    ref = x.double().cpu().numpy() @ w.double().cpu().numpy().T
    got = y.cpu().numpy()
    assert np.isfinite(got).all()
    err = np.abs(got - ref).max()
    # float32 accumulation plus the 2^-17 relative two-term representation
    tol = 2e-5 * np.sqrt(K) * np.abs(w.float().cpu().numpy()).max() * np.abs(x.cpu().numpy()).max()
    assert err <= tol, (err, tol)


def test_gemm_split_results_are_deterministic(dec):
    g = torch.Generator(device="cuda").manual_seed(5)
    w = (torch.randn(384, 2048, generator=g, device="cuda") * 0.05).to(torch.bfloat16)
    x = pair_rows(torch.randn(32, 2048, generator=g, device="cuda"))
    outs = []
    for _ in range(3):
        y = torch.empty(32, 384, device="cuda")
        fdllm.fdllm_gemm(dec.ctx, w, x, y, 8)
        outs.append(y.cpu())
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])


def test_gemm_accumulate_adds_into_y(dec):
    g = torch.Generator(device="cuda").manual_seed(9)
    w = (torch.randn(640, 1024, generator=g, device="cuda") * 0.05).to(torch.bfloat16)
    x = torch.randn(48, 1024, generator=g, device="cuda")
    y0 = torch.randn(48, 640, generator=g, device="cuda")
    for splits in (1, 4):
        y = y0.clone()
        fdllm.fdllm_gemm(dec.ctx, w, pair_rows(x), y, splits, accumulate=True)
        torch.cuda.synchronize()
        ref = y0.double().cpu().numpy() + x.double().cpu().numpy() @ w.double().cpu().numpy().T
        assert np.abs(y.cpu().numpy() - ref).max() <= 2e-5 * np.sqrt(1024) * 0.3 * 5
