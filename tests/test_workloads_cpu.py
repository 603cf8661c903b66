"""The workload definitions the benchmark and the parity tests run: model
shapes and (prompt, generation, block, tau) of each configuration, pinned
to figures stated independently of the code: the LLaDA-8B and Dream-7B
layer shapes (layers, width, heads, FFN width, vocabulary, RoPE base, norm
epsilon), their parameter counts per layer and per LM head, and the bytes
one DualCache block step must read (the weights once plus K and V of every
position once)."""
import pytest

from kv_cache_decode_dualcache_b200 import synth

# name: (layers, d_model, heads, kv heads, head dim, ffn, vocab, mask id, rope theta,
#        rms eps, logit scale, dtype)
SHAPES = {
    "tiny-fp32": (2, 128, 4, 4, 32, 384, 512, 511, 1e4, 1e-5, 8.0, "fp32"),
    "llada-8b-shape": (32, 4096, 32, 32, 128, 12288, 126464, 126463, 1e4, 1e-5, 30.0, "bf16"),
    "dream-7b-shape": (28, 3584, 28, 4, 128, 18944, 152064, 152063, 1e6, 1e-6, 30.0, "bf16"),
    # reduced test models: vocabulary and FFN widths off the tile sizes on purpose
    "small-bf16": (2, 512, 4, 4, 128, 1344, 1000, 999, 1e4, 1e-5, 30.0, "bf16"),
    "small-gqa-bf16": (2, 512, 8, 2, 64, 1408, 2051, 2050, 1e6, 1e-6, 30.0, "bf16"),
}
SEEDS = {"tiny-fp32": 0, "llada-8b-shape": 1, "dream-7b-shape": 2}

# name: (prompt, generation, block, tau, cache mode, batch)
WORKLOADS = {
    "tiny": (32, 64, 16, 0.9, "dual", 1),
    "llada8b-p256-g256": (256, 256, 32, 0.9, "dual", 1),
    "llada8b-p1024-g256": (1024, 256, 32, 0.9, "dual", 1),
    "llada8b-p1024-g512": (1024, 512, 32, 0.9, "dual", 1),
    "llada8b-p1024-g1024": (1024, 1024, 32, 0.9, "dual", 1),
    "dream7b-p512-g512": (512, 512, 32, 0.9, "dual", 1),
    "llada8b-batch16": (0, 256, 32, 0.9, "dual", 16),
}


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_model_shapes(name):
    s = synth.SHAPES[name]
    got = (s.n_layers, s.d_model, s.n_heads, s.n_kv_heads, s.head_dim, s.ffn_dim, s.vocab,
           s.mask_id, s.rope_theta, s.rms_eps, s.logit_scale, s.dtype)
    assert got == SHAPES[name]
    if name in SEEDS:
        assert s.seed == SEEDS[name]


# two layers of the LLaDA-8B shape: every per-launch shape of the full model
TWO_LAYER = {
    "llada8b-2layer-p256-g32": (256, 32, 32, 0.9, "dual", 1),
    "llada8b-2layer-p256-g256": (256, 256, 32, 0.9, "dual", 1),
    "llada8b-2layer-batch16": (0, 256, 32, 0.9, "dual", 16),
}


@pytest.mark.parametrize("name", sorted(TWO_LAYER))
def test_two_layer_workloads(name):
    w = synth.WORKLOADS[name]
    assert (w.prompt_len, w.gen_len, w.block_size, w.tau, w.cache_mode, w.batch) == \
        TWO_LAYER[name]
    full = synth.LLADA_8B
    assert w.shape.n_layers == 2
    for f in ("d_model", "n_heads", "n_kv_heads", "head_dim", "ffn_dim", "vocab", "mask_id",
              "rope_theta", "rms_eps", "logit_scale", "dtype", "seed"):
        assert getattr(w.shape, f) == getattr(full, f), f


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_workloads(name):
    w = synth.WORKLOADS[name]
    assert (w.prompt_len, w.gen_len, w.block_size, w.tau, w.cache_mode, w.batch) == \
        WORKLOADS[name]


def test_weights_a_block_step_reads():
    # LLaDA-8B shape: 218.1 M parameters per layer (q, k, v, o 4 x 4096^2 and
    # gate, up, down 3 x 4096 x 12288) and a 518.0 M LM head: 7.497 B, i.e.
    # 14.995 GB in bf16; Dream-7B shape: 233.0 M per layer (GQA: q and o
    # 2 x 3584^2, k and v 2 x 3584 x 512, FFN 3 x 3584 x 18944) and a 545.0 M
    # head: 7.070 B, 14.141 GB
    llada = synth.step_weight_params(synth.LLADA_8B)
    assert llada == 32 * (4 * 4096 ** 2 + 3 * 4096 * 12288) + 126464 * 4096
    assert round(llada / 1e9, 3) == 7.497 and round(2 * llada / 1e9, 3) == 14.995
    dream = synth.step_weight_params(synth.DREAM_7B)
    assert dream == 28 * (2 * 3584 ** 2 + 2 * 3584 * 512 + 3 * 3584 * 18944) + 152064 * 3584
    assert round(2 * dream / 1e9, 3) == 14.141


def test_parameter_counts_include_embedding_and_norms():
    s = synth.LLADA_8B
    per_layer = 4 * 4096 ** 2 + 3 * 4096 * 12288 + 2 * 4096
    assert s.n_params == 2 * 126464 * 4096 + 32 * per_layer + 4096
    t = synth.TINY
    assert t.n_params == 2 * 512 * 128 + 2 * (4 * 128 * 128 + 3 * 128 * 384 + 2 * 128) + 128
