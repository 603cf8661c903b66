"""Builders for the two-term (hi + lo) layouts of the bf16 model, written
with plain torch ops for the GPU kernel tests: bf16 pairs for the stand-alone
GEMM entry points, fp16 pairs for the decoder's own storage."""
import torch


def split(x: torch.Tensor, dtype=torch.bfloat16):
    hi = x.to(dtype)
    lo = (x - hi.float()).to(dtype)
    return hi, lo


def pair_rows(x: torch.Tensor, dtype=torch.bfloat16) -> torch.Tensor:
    """[M, K] float -> [2*ceil(M/32)*32, K] of dtype (bf16 for the stand-alone
    GEMM, fp16 for the decoder's own form): per group of 32 tokens the 32 hi
    rows, then the 32 lo rows."""
    M, K = x.shape
    G = (M + 31) // 32
    pad = torch.zeros(G * 32, K, device=x.device, dtype=x.dtype)
    pad[:M] = x
    hi, lo = split(pad, dtype)
    return torch.stack([hi.view(G, 32, K), lo.view(G, 32, K)], dim=1).reshape(G * 64, K)


def from_pair_rows(y: torch.Tensor, M: int) -> torch.Tensor:
    """Inverse of pair_rows: hi + lo as float [M, K]."""
    G = y.shape[0] // 64
    v = y.float().view(G, 2, 32, -1)
    return (v[:, 0] + v[:, 1]).reshape(G * 32, -1)[:M]
