"""The decoder's GEMM (tcgen05 on the bf16 model) against a float64 matmul of
the same operands: bf16 weights times two-term (hi + lo) activations, over
token-tile widths, K splits and ragged N / M."""
import numpy as np
import pytest
import torch

from kv_cache_decode_dualcache_b200 import fdllm, synth
from tests.bf16_layout import from_pair_rows, pair_rows
from tests.gpu_util import make_decoder, require_gpu

pytestmark = pytest.mark.gpu


def _decoder(pair):
    require_gpu()
    shape = synth.with_layers(synth.SMALL_BF16, 1)
    # 2 x 1024 rows: tile counters for the 24576 x 512-token case
    return make_decoder(shape, synth.make_weights(shape, device="cpu"), 1024, max_batch=2,
                        env={"FDLLM_GEMM_PAIR": "1" if pair else "0"})


@pytest.fixture(scope="module")
def dec():
    """The default context: shapes with N % 256 == 0 and M > 64 run on SM pairs."""
    return _decoder(True)


@pytest.fixture(scope="module")
def dec_single():
    """Every shape on the single-SM kernel."""
    return _decoder(False)


SHAPES = [
    (128, 32, 64, 1), (256, 32, 512, 0), (1000, 17, 512, 1), (384, 32, 4096, 4),
    (130, 64, 256, 0), (512, 100, 512, 0), (640, 256, 1024, 0), (256, 300, 512, 3),
    (4096, 32, 1024, 0), (257, 5, 128, 2), (12288, 32, 4096, 0), (4096, 512, 4096, 0),
    # SM-pair shapes: ragged token tiles, forced and planned K splits, the
    # LLaDA-8B QKV / gate-up / down shapes at 512 tokens
    (256, 65, 64, 0), (768, 129, 1024, 0), (512, 200, 2048, 5), (1024, 1000, 512, 0),
    (12288, 512, 4096, 0), (24576, 512, 4096, 0), (4096, 512, 12288, 0),
]


@pytest.mark.parametrize("N,M,K,splits", SHAPES)
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


@pytest.mark.parametrize("N,M,K,splits", [(512, 100, 512, 0), (768, 129, 1024, 0),
                                         (512, 200, 2048, 5), (4096, 512, 4096, 0)])
def test_gemm_pair_agrees_with_single_sm(dec, dec_single, N, M, K, splits):
    """The SM-pair kernel and the single-SM kernel on the same operands: the
    same sums up to float32 rounding order."""
    g = torch.Generator(device="cuda").manual_seed(N + M + K)
    w = (torch.randn(N, K, generator=g, device="cuda") * 0.05).to(torch.bfloat16)
    x = pair_rows(torch.randn(M, K, generator=g, device="cuda"))
    ys = []
    for d in (dec, dec_single):
        y = torch.full((M, N), float("nan"), device="cuda")
        fdllm.fdllm_gemm(d.ctx, w, x, y, splits)
        torch.cuda.synchronize()
        ys.append(y.cpu().double())
    assert torch.isfinite(ys[0]).all()
    scale = ys[1].abs().max().item()
    assert (ys[0] - ys[1]).abs().max().item() <= 1e-5 * scale


@pytest.mark.parametrize("N,M,K,splits", [(128, 32, 64, 1), (1000, 17, 512, 1), (384, 32, 4096, 4),
                                         (512, 100, 512, 0), (768, 129, 1024, 0),
                                         (512, 200, 2048, 5), (12288, 512, 4096, 0)])
def test_gemm_f16_operands_match_float64(dec, N, M, K, splits):
    """The decoder's operand form: fp16 weights (N(0, 0.05), exact in fp16)
    times two-term fp16 activations, against a float64 matmul of exactly
    those values, on the single-SM and SM-pair kernels."""
    g = torch.Generator(device="cuda").manual_seed(N * 11 + M * 5 + K)
    w = (torch.randn(N, K, generator=g, device="cuda") * 0.05).to(torch.float16)
    x = torch.randn(M, K, generator=g, device="cuda")
    xp = pair_rows(x, torch.float16)
    y = torch.full((M, N), float("nan"), device="cuda")
    fdllm.fdllm_gemm_f16(dec.ctx, w, xp, y, splits)
    torch.cuda.synchronize()
    xv = from_pair_rows(xp, M).double().cpu().numpy()     # the two-term value the kernel sees
    ref = xv @ w.double().cpu().numpy().T
    got = y.cpu().numpy()
    assert np.isfinite(got).all()
    tol = 2e-5 * np.sqrt(K) * np.abs(w.float().cpu().numpy()).max() * np.abs(xv).max()
    assert np.abs(got - ref).max() <= tol


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


@pytest.mark.parametrize("N,M", [(640, 48), (768, 200)])
def test_gemm_accumulate_adds_into_y(dec, N, M):
    g = torch.Generator(device="cuda").manual_seed(9)
    w = (torch.randn(N, 1024, generator=g, device="cuda") * 0.05).to(torch.bfloat16)
    x = torch.randn(M, 1024, generator=g, device="cuda")
    y0 = torch.randn(M, N, generator=g, device="cuda")
    for splits in (1, 4):
        y = y0.clone()
        fdllm.fdllm_gemm(dec.ctx, w, pair_rows(x), y, splits, accumulate=True)
        torch.cuda.synchronize()
        ref = y0.double().cpu().numpy() + x.double().cpu().numpy() @ w.double().cpu().numpy().T
        assert np.abs(y.cpu().numpy() - ref).max() <= 2e-5 * np.sqrt(1024) * 0.3 * 5
