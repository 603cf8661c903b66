"""The seeded input recipe both sides consume (``synth``): shapes, weights,
prompts and batch lengths are what the recipe states, and reproducible."""
import torch

from kv_cache_decode_dualcache_b200 import synth


def test_every_shape_reserves_the_last_id_as_the_mask():
    for shape in synth.SHAPES.values():
        assert shape.mask_id == shape.vocab - 1, shape.name


def test_prompts_are_seeded_uniform_ids_that_are_never_the_mask():
    for shape in (synth.TINY, synth.SMALL_BF16, synth.SMALL_GQA_BF16):
        p = synth.make_prompt(shape, 4000)
        assert p.dtype == torch.int32
        assert int(p.min()) >= 0 and int(p.max()) <= shape.vocab - 2
        assert int(p.max()) >= shape.vocab - 2 - shape.vocab // 50   # spans the range
        assert torch.equal(p, synth.make_prompt(shape, 4000))          # reproducible
        assert not torch.equal(p, synth.make_prompt(shape, 4000, salt=1))


def test_batch_lengths_follow_the_recipe():
    lens = synth.make_batch_prompt_lengths(16)
    assert lens == synth.make_batch_prompt_lengths(16)
    assert len(lens) == 16 and all(128 <= n <= 1024 for n in lens)
    assert synth.make_batch_prompt_lengths(16, seed=4) != lens


def test_weights_follow_the_recipe():
    for shape, dt in ((synth.TINY, torch.float32), (synth.SMALL_BF16, torch.bfloat16)):
        w = synth.make_weights(shape, device="cpu")
        shapes = synth.weight_shapes(shape)
        assert list(w) == synth.weight_names(shape) and set(w) == set(shapes)
        for name, t in w.items():
            assert tuple(t.shape) == shapes[name] and t.dtype == dt, name
            if name.endswith("norm"):
                assert bool((t == 1).all()), name                    # gains are 1
        big = torch.cat([w[n].float().flatten() for n in w if not n.endswith("norm")])
        assert abs(float(big.mean())) < 1e-3 and abs(float(big.std()) - 0.02) < 5e-4
        w2 = synth.make_weights(shape, device="cpu")
        assert all(torch.equal(w[n], w2[n]) for n in w)              # reproducible


def test_bf16_weights_are_the_rounded_float32_draw():
    # bf16 models round the float32 draw of the same generator (RNE)
    shape = synth.SMALL_BF16
    w = synth.make_weights(shape, device="cpu")
    gen = torch.Generator().manual_seed(shape.seed)
    first = torch.empty(synth.weight_shapes(shape)["embed"]).normal_(0.0, 0.02, generator=gen)
    assert torch.equal(w["embed"], first.to(torch.bfloat16))


def test_prompt_and_length_draws_are_the_stated_generators():
    # prompts: ids uniform in [0, vocab - 2] from a CPU generator seeded with
    # 1000 + model seed + salt; batch lengths: uniform in [128, 1024] from one
    # seeded with 3
    for shape, salt in ((synth.TINY, 0), (synth.LLADA_8B, 0), (synth.LLADA_8B, 5)):
        gen = torch.Generator().manual_seed(1000 + shape.seed + salt)
        want = torch.randint(0, shape.vocab - 1, (64,), generator=gen, dtype=torch.int64)
        assert torch.equal(synth.make_prompt(shape, 64, salt=salt), want.to(torch.int32))
    gen = torch.Generator().manual_seed(3)
    assert synth.make_batch_prompt_lengths(16) == \
        [int(v) for v in torch.randint(128, 1025, (16,), generator=gen)]


def test_batched_workload_lengths_are_the_recorded_ones():
    # the 16 prompt lengths this generator gave the batched workload when its
    # measurements were taken (listed beside them in the design notes)
    assert synth.make_batch_prompt_lengths(16) == [1014, 199, 510, 989, 570, 1022, 419, 988, 789,
                                                   615, 588, 323, 913, 952, 341, 552]


def test_element_sizes():
    assert synth.TINY.elem_bytes == 4 and synth.LLADA_8B.elem_bytes == 2
