"""The fixed-count strategy (k most confident masked positions per step) in
the oracle, pinned by its special cases: k = 1 is the one-token-per-step
greedy decode (the same decisions as tau > 1), k = block unmasks a whole
block in one step (as tau <= 0), and a block of B positions takes exactly
ceil(B / k) steps."""
import numpy as np
import pytest

from kv_cache_decode_dualcache_b200 import synth
from oracle.decode import generate, select_top_k, select_unmask
from oracle.model import Model


def test_select_top_k_order_and_ties():
    masked = np.array([1, 1, 0, 1, 1, 1], bool)
    conf = np.array([0.2, 0.7, 0.99, 0.7, 0.1, 0.5])
    # position 2 is not masked; 1 and 3 tie (lower first), then 5
    assert list(np.flatnonzero(select_top_k(masked, conf, 3))) == [1, 3, 5]
    assert list(np.flatnonzero(select_top_k(masked, conf, 1))) == [1]
    assert select_top_k(masked, conf, 9).tolist() == masked.tolist()
    assert not select_top_k(np.zeros(4, bool), conf[:4], 2).any()
    assert not select_top_k(masked, conf, 0).any() and not select_top_k(masked, conf, -2).any()
    # k = 1 is the threshold rule's fallback pick
    assert np.array_equal(select_top_k(masked, conf, 1), select_unmask(masked, conf, 2.0))


@pytest.fixture(scope="module")
def tiny():
    shape = synth.TINY
    return shape, Model(shape.as_dict(), synth.make_weights(shape, device="cpu"))


@pytest.mark.parametrize("mode", ["dual", "none"])
def test_fixed_k_special_cases(tiny, mode):
    shape, model = tiny
    prompt = synth.make_prompt(shape, 24).numpy()
    G, B = 32, 8
    one = generate(model, prompt, G, B, 0.9, mode, fixed_k=1)
    greedy = generate(model, prompt, G, B, 1.01, mode)
    assert np.array_equal(one.tokens, greedy.tokens) and one.steps == G
    whole = generate(model, prompt, G, B, 0.9, mode, fixed_k=B)
    at_once = generate(model, prompt, G, B, -1.0, mode)
    assert np.array_equal(whole.tokens, at_once.tokens) and whole.steps == G // B
    for k in (3, 5):
        r = generate(model, prompt, G, B, 0.9, mode, fixed_k=k)
        assert r.steps_per_block == [-(-B // k)] * (G // B)
        assert not np.any(r.tokens == shape.mask_id)
