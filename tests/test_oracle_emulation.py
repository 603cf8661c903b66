"""Pins for the oracle's bfloat16 storage-point emulation."""
import numpy as np

from kv_cache_decode_dualcache_b200 import synth
from oracle.model import Model
from oracle.numerics import round_bf16


def test_emulated_kv_is_bf16_and_close_to_exact():
    shape = synth.with_layers(synth.SMALL_BF16, 1)
    w = synth.make_weights(shape, device="cpu")
    x = synth.make_prompt(shape, 40).numpy()
    exact = Model(shape.as_dict(), w, emulate_bf16=False)
    emu = Model(shape.as_dict(), w, emulate_bf16=True)
    z0, kv0 = exact.forward(x, range(40), return_kv=True)
    z1, kv1 = emu.forward(x, range(40), return_kv=True)
    for k, v in kv1:
        np.testing.assert_array_equal(round_bf16(k), k)
        np.testing.assert_array_equal(round_bf16(v), v)
    # Rounding changes the logits, but only by a bf16-sized relative amount.
    rel = np.abs(z1 - z0).max() / np.abs(z0).max()
    assert 0 < rel < 2e-2
