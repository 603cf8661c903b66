"""The decoder's attention kernel in isolation: random queries against the
K/V the GPU cached for a sequence, checked against the oracle's attention
(float64) on exactly those K/V.  Covers the no-split path (many rows) and
the split-KV path (block-sized M), MHA and GQA, ragged key counts.  Every
query set runs the tcgen05 + TMA kernel (block-sized ones with the keys
split over a thread-block cluster); with FDLLM_ATTN_BLK=0 the block-sized
ones run the mma.sync key-split kernel instead (the batched forward's
block tiles use that one), and both are checked."""
import numpy as np
import pytest
import torch

from kv_cache_decode_dualcache_b200 import fdllm, synth
from oracle.model import attention
from tests.bf16_layout import from_pair_rows, split
from tests.gpu_util import make_decoder, require_gpu

pytestmark = pytest.mark.gpu


def _decoder(shape, max_seq, blk):
    return make_decoder(shape, synth.make_weights(shape, device="cpu"), max_seq,
                        env={"FDLLM_ATTN_BLK": "1" if blk else "0"})


PARAMS = [("small-bf16", True), ("small-gqa-bf16", True), ("small-bf16", False),
          ("small-gqa-bf16", False)]


@pytest.fixture(scope="module", params=PARAMS, ids=lambda p: f"{p[0]}-{'tc' if p[1] else 'mma'}")
def setup(request):
    require_gpu()
    shape = synth.SHAPES[request.param[0]]
    dec = _decoder(shape, 256, request.param[1])
    prompt = synth.make_prompt(shape, 150).numpy()
    x = np.concatenate([prompt, np.full(50, shape.mask_id)])
    dec.step_debug(x, x, 150, 32, 0.9, "dual", logits=False)   # fills the cache for 200 positions
    return shape, dec


@pytest.mark.parametrize("M,L", [(32, 200), (200, 200), (7, 65), (64, 128), (100, 37)])
@pytest.mark.parametrize("qscale", [1.0, 4.0, 16.0])
def test_attention_matches_oracle(setup, M, L, qscale):
    shape, dec = setup
    H, hd = shape.n_heads, shape.head_dim
    g = torch.Generator(device="cuda").manual_seed(M * 1000 + L)
    q = torch.randn(M, H, hd, generator=g, device="cuda") * qscale
    qh, ql = split(q, torch.float16)
    qd = torch.stack([qh, ql]).contiguous()
    rows = 2 * ((M + 31) // 32) * 32
    o = torch.full((rows, H * hd), float("nan"), device="cuda", dtype=torch.float16)
    fdllm.fdllm_attention(dec.ctx, qd, o, 0, L)
    torch.cuda.synchronize()
    k, v = dec.read_kv(0, 0, L)
    qx = (qh.double() + ql.double()).cpu().numpy()
    ref = attention(qx, k.astype(np.float64), v.astype(np.float64)).reshape(M, H * hd)
    got = from_pair_rows(o, M).double().cpu().numpy()
    assert np.isfinite(got).all()
    err = np.abs(got - ref).max()
    tol = 1e-4 * max(1.0, np.abs(ref).max())
    assert err <= tol, (err, tol)


@pytest.fixture(scope="module", params=PARAMS, ids=lambda p: f"{p[0]}-{'tc' if p[1] else 'mma'}")
def long_setup(request):
    require_gpu()
    shape = synth.SHAPES[request.param[0]]
    dec = _decoder(shape, 1024, request.param[1])
    prompt = synth.make_prompt(shape, 700).numpy()
    x = np.concatenate([prompt, np.full(60, shape.mask_id)])
    dec.step_debug(x, x, 700, 32, 0.9, "dual", logits=False)   # caches 760 positions
    return shape, dec


@pytest.mark.parametrize("M,L", [(32, 760), (7, 700), (64, 760), (16, 577), (256, 760),
                                 (130, 577), (760, 760)])
def test_attention_long_keys_split_path(long_setup, M, L):
    shape, dec = long_setup
    H, hd = shape.n_heads, shape.head_dim
    g = torch.Generator(device="cuda").manual_seed(M + L)
    q = torch.randn(M, H, hd, generator=g, device="cuda") * 4.0
    qh, ql = split(q, torch.float16)
    qd = torch.stack([qh, ql]).contiguous()
    rows = 2 * ((M + 31) // 32) * 32
    o = torch.full((rows, H * hd), float("nan"), device="cuda", dtype=torch.float16)
    for _ in range(2):  # the split counters reset themselves between calls
        fdllm.fdllm_attention(dec.ctx, qd, o, 1, L)
        torch.cuda.synchronize()
        k, v = dec.read_kv(1, 0, L)
        qx = (qh.double() + ql.double()).cpu().numpy()
        ref = attention(qx, k.astype(np.float64), v.astype(np.float64)).reshape(M, H * hd)
        got = from_pair_rows(o, M).double().cpu().numpy()
        assert np.isfinite(got).all()
        assert np.abs(got - ref).max() <= 1e-4 * max(1.0, np.abs(ref).max())


@pytest.fixture(scope="module", params=PARAMS, ids=lambda p: f"{p[0]}-{'tc' if p[1] else 'mma'}")
def very_long_setup(request):
    require_gpu()
    shape = synth.SHAPES[request.param[0]]
    dec = _decoder(shape, 1280, request.param[1])
    prompt = synth.make_prompt(shape, 1150).numpy()
    x = np.concatenate([prompt, np.full(50, shape.mask_id)])
    dec.step_debug(x, x, 1150, 32, 0.9, "dual", logits=False)   # caches 1200 positions
    return shape, dec


@pytest.mark.parametrize("M,L", [(32, 1200), (16, 1100), (64, 1200), (5, 1030)])
def test_attention_many_chunks_per_cta(very_long_setup, M, L):
    """More 128-key chunks than a cluster has CTAs: every split of the block
    attention runs several chunks with the online softmax between them."""
    shape, dec = very_long_setup
    H, hd = shape.n_heads, shape.head_dim
    g = torch.Generator(device="cuda").manual_seed(7 * M + L)
    q = torch.randn(M, H, hd, generator=g, device="cuda") * 8.0
    qh, ql = split(q, torch.float16)
    qd = torch.stack([qh, ql]).contiguous()
    rows = 2 * ((M + 31) // 32) * 32
    o = torch.full((rows, H * hd), float("nan"), device="cuda", dtype=torch.float16)
    fdllm.fdllm_attention(dec.ctx, qd, o, 1, L)
    torch.cuda.synchronize()
    k, v = dec.read_kv(1, 0, L)
    qx = (qh.double() + ql.double()).cpu().numpy()
    ref = attention(qx, k.astype(np.float64), v.astype(np.float64)).reshape(M, H * hd)
    got = from_pair_rows(o, M).double().cpu().numpy()
    assert np.isfinite(got).all()
    assert np.abs(got - ref).max() <= 1e-4 * max(1.0, np.abs(ref).max())
