"""Parity of the production generate path (bf16 models) with the oracle.

``fdllm_generate`` replays each step kind from a captured CUDA graph, chains
its kernels with programmatic dependent launches and runs DualCache block
steps through the persistent chain kernel: a different launch sequence from
the un-graphed one ``fdllm_step_debug`` uses.  Here the production call runs
with its per-step trace on, and every step it took is recomputed by the
float64 oracle on the same sequence (the block procedure of the techwalker.com
Fast-dLLM article, section "核心创新：适合扩散模型的KV缓存"; the threshold rule
of the ccyt168.com overview, section 一, item 2): confidences within 1e-3,
tokens and unmask sets identical except counted near ties, and the returned
tokens equal to the traced decisions.
"""
import numpy as np
import pytest
import torch

from kv_cache_decode_dualcache_b200 import synth
from oracle.model import Model
from tests.gpu_util import make_decoder, require_gpu
from tests.parity import replay_gpu_trace

pytestmark = pytest.mark.gpu

LLADA_2L = synth.with_layers(synth.LLADA_8B, 2)
DREAM_2L = synth.with_layers(synth.DREAM_7B, 2)


@pytest.fixture(scope="module", params=["small-bf16", "small-gqa-bf16"])
def small(request):
    require_gpu()
    shape = synth.SHAPES[request.param]
    w = synth.make_weights(shape, device="cpu")
    dec = make_decoder(shape, w, 40 + 64)
    yield shape, dec, Model(shape.as_dict(), w)
    dec.close()


@pytest.mark.parametrize("mode", ["dual", "prefix", "none"])
def test_small_generate_path_matches_oracle(small, mode):
    shape, dec, model = small
    prompt = synth.make_prompt(shape, 40, salt=7).numpy()     # blocks start mid-page
    out, steps, st = dec.generate(prompt, 64, 32, 0.9, mode, trace=True)
    assert steps == len(st.trace_block) == st.steps
    rep = replay_gpu_trace(model, prompt, 64, 32, 0.9, mode, out, st, label=f"{shape.name} {mode}")
    print(f"{shape.name} {mode}: {rep.summary()}")
    assert rep.steps == steps
    assert not rep.mismatches, rep.mismatches[:5]


@pytest.mark.parametrize("mode", ["dual", "prefix", "none"])
def test_device_resident_generate_equals_the_host_call(small, mode):
    # fdllm_generate_device (prompt and tokens in device memory; the call the
    # benchmark times) runs the same decode as the host-buffer call
    shape, dec, model = small
    prompt = synth.make_prompt(shape, 40, salt=9).numpy()
    host, steps, _ = dec.generate(prompt, 64, 32, 0.9, mode)
    p_dev = torch.as_tensor(prompt, dtype=torch.int32).cuda()
    out_dev = torch.full((64,), -1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    dev_steps = dec.generate_device(p_dev, 64, 32, 0.9, out_dev, mode)
    torch.cuda.synchronize()
    assert dev_steps == steps
    np.testing.assert_array_equal(out_dev.cpu().numpy(), host)


@pytest.mark.parametrize("shape", [LLADA_2L, DREAM_2L], ids=["llada8b-2layer", "dream7b-2layer"])
def test_full_width_generate_path_matches_oracle(shape):
    # the LLaDA-8B / Dream-7B layer widths, vocabularies and head layouts
    # (MHA 32 x 128; GQA 28 / 4 x 128) with two layers, so the oracle runs
    # every step of two blocks in seconds
    require_gpu()
    w = synth.make_weights(shape, device="cuda")
    P, G, B = 64, 64, 32
    dec = make_decoder(shape, w, P + G)
    w_host = {k: v.cpu() for k, v in w.items()}
    del w
    torch.cuda.empty_cache()
    model = Model(shape.as_dict(), w_host)
    prompt = synth.make_prompt(shape, P).numpy()
    out, steps, st = dec.generate(prompt, G, B, 0.9, "dual", trace=True)
    rep = replay_gpu_trace(model, prompt, G, B, 0.9, "dual", out, st, label=shape.name)
    print(f"{shape.name} dual: {rep.summary()}")
    dec.close()
    assert rep.steps == steps
    assert not rep.mismatches, rep.mismatches[:5]


def test_inexact_weight_count_matches_host_count():
    # GEMM weights (not the embedding table, which stays bf16) whose fp16
    # value differs from the bf16 value: non-zero values under 2^-17
    require_gpu()
    shape = synth.SMALL_BF16
    w = synth.make_weights(shape, device="cpu")
    dec = make_decoder(shape, w, 128)
    gemm = [n for n in w if n.endswith(("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down"))
            or n == "lm_head"]
    want = sum(int((w[n].to(torch.float16).float() != w[n].float()).sum()) for n in gemm)
    got = dec.inexact_weight_count()
    dec.close()
    print(f"inexact bf16 -> fp16 weights: {got} of {sum(w[n].numel() for n in gemm)}")
    assert got == want and got > 0
