"""Production generate path (bf16 models) at block sizes other than 32, with
an empty prompt, and at the largest block, against the oracle.

The block size decides which kernels a step runs: blocks of at most 32
tokens take the persistent chain kernel with a partly filled 32-token tile
(8 and 16 here), 64-token blocks the separate launches with the tcgen05
block attention over 64-row query tiles, 128 and 256-token blocks the SM-pair
GEMMs and the many-query attention.  Every step the production call took is
recomputed by the float64 oracle on the same sequence and compared
(confidence, token, unmask set; the block procedure of the techwalker.com
Fast-dLLM article, section "核心创新：适合扩散模型的KV缓存"; the threshold rule of
the ccyt168.com overview, section 一, item 2).
"""
import numpy as np
import pytest

from kv_cache_decode_dualcache_b200 import synth
from oracle.model import Model
from tests.gpu_util import make_decoder, require_gpu
from tests.parity import replay_gpu_trace

pytestmark = pytest.mark.gpu

P, G = 40, 128


@pytest.fixture(scope="module", params=["small-bf16", "small-gqa-bf16"])
def small(request):
    require_gpu()
    shape = synth.SHAPES[request.param]
    w = synth.make_weights(shape, device="cpu")
    dec = make_decoder(shape, w, P + 256)
    yield shape, dec, Model(shape.as_dict(), w)
    dec.close()


def _check(shape, dec, model, prompt, gen_len, block, tau, mode, label):
    out, steps, st = dec.generate(prompt, gen_len, block, tau, mode, trace=True)
    assert steps == len(st.trace_block) == st.steps
    assert len(st.steps_per_block) == gen_len // block
    rep = replay_gpu_trace(model, prompt, gen_len, block, tau, mode, out, st, label=label)
    print(f"{label}: {rep.summary()}")
    assert rep.steps == steps
    assert not rep.mismatches, rep.mismatches[:5]


# tau 0.99 for the large blocks: at 0.9 the reduced models unmask most of a
# 64 or 128-token block in its first (refresh) step, leaving few cached steps
@pytest.mark.parametrize("mode", ["dual", "prefix"])
@pytest.mark.parametrize("block,tau", [(8, 0.9), (16, 0.9), (64, 0.99), (128, 0.99)])
def test_block_sizes_match_oracle(small, block, tau, mode):
    shape, dec, model = small
    prompt = synth.make_prompt(shape, P, salt=11).numpy()
    _check(shape, dec, model, prompt, G, block, tau, mode, f"{shape.name} B={block} {mode}")


@pytest.mark.parametrize("mode", ["dual", "prefix", "none"])
def test_empty_prompt_matches_oracle(small, mode):
    shape, dec, model = small
    prompt = np.zeros(0, dtype=np.int32)
    _check(shape, dec, model, prompt, 64, 32, 0.9, mode, f"{shape.name} P=0 {mode}")


def test_largest_block_fills_max_seq(small):
    # one block of 256 tokens (the largest block the decoder takes) ending
    # exactly at max_seq
    shape, dec, model = small
    prompt = synth.make_prompt(shape, P, salt=13).numpy()
    _check(shape, dec, model, prompt, 256, 256, 0.99, "dual", f"{shape.name} B=256")
