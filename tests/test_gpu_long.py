"""Long-sequence parity: the LLaDA-8B layer shapes (2 layers, so the float64
oracle finishes in tens of seconds) at the long-generation configuration's
length, prompt 1024 + generation 1024 (L = 2048, 32 pages of keys, the
block-step attention split into a 4-CTA cluster per KV head).

Teacher-forced on the last block (s = 2016: the whole sequence before it is
cached prefix) and on a middle block (s = 1536: prefix and suffix both
cached): the refresh step and one DualCache step each, logits <= 3e-2,
confidences <= 1e-3, tokens and unmask sets identical except at counted
near ties."""
import numpy as np
import pytest
import torch

from kv_cache_decode_dualcache_b200 import synth
from oracle.decode import confidence, select_unmask
from oracle.model import Model
from tests.gpu_util import make_decoder, require_gpu
from tests.parity import StepReport, compare_step

pytestmark = pytest.mark.gpu

SHAPE = synth.with_layers(synth.LLADA_8B, 2)
P, G, B, TAU = 1024, 1024, 32, 0.9


@pytest.fixture(scope="module")
def long_model():
    require_gpu()
    w = synth.make_weights(SHAPE, device="cuda")
    dec = make_decoder(SHAPE, w, P + G)
    w_host = {k: v.cpu() for k, v in w.items()}
    del w
    torch.cuda.empty_cache()
    yield dec, Model(SHAPE.as_dict(), w_host)
    dec.close()


@pytest.mark.parametrize("s", [P + 512, P + G - B])
def test_long_sequence_teacher_forced(long_model, s):
    dec, model = long_model
    mask = SHAPE.mask_id
    L = P + G
    rng = np.random.default_rng(7)
    prompt = synth.make_prompt(SHAPE, P).numpy()
    x0 = np.concatenate([prompt, np.full(G, mask)]).astype(np.int64)
    # blocks before s already decoded (arbitrary non-mask ids)
    x0[P:s] = rng.integers(0, SHAPE.vocab - 1, s - P)
    rep = StepReport()
    z, kv = model.forward(x0, range(L), return_kv=True, head_rows=range(s, s + B))
    conf, tok = confidence(z, mask)
    ref = {"z": z, "conf": conf, "tok": tok, "unmask": select_unmask(np.ones(B, bool), conf, TAU)}
    g = dec.step_debug(x0, x0, s, B, TAU, "dual")
    compare_step(g, ref, np.ones(B, bool), TAU, mask, rep, z_tol=3e-2, label="refresh")
    x = x0.copy()
    x[s:s + B][ref["unmask"]] = ref["tok"][ref["unmask"]]
    masked = x[s:s + B] == mask
    if masked.any():
        z = model.forward(x, range(s, s + B), cache=kv)
        conf, tok = confidence(z, mask)
        ref = {"z": z, "conf": conf, "tok": tok, "unmask": select_unmask(masked, conf, TAU)}
        g = dec.step_debug(x0, x, s, B, TAU, "dual")
        compare_step(g, ref, masked, TAU, mask, rep, z_tol=3e-2, label="dual step")
    print(f"long s={s}: steps {rep.steps} max|dz| {rep.max_dz:.3g} "
          f"max|dconf| {rep.max_dconf:.3g} near-tie exemptions {rep.exempt}")
    assert not rep.mismatches, rep.mismatches[:5]
