"""Full-size parity on the Dream-7B shape (Qwen2.5-7B-like GQA: 28 layers,
d=3584, 28 query / 4 KV heads of 128, FFN 18944, V=152064, RoPE theta 1e6),
against the float64 oracle.

Teacher-forced on one block: the block-start full forward (refresh step) and
two DualCache steps on the sequence the oracle's own unmask decisions
produce, with a 224-token prompt (L = 256, so the float64 full forward
stays near a minute on the host).  Each step: logits max-abs <= 3e-2 over
all 32 x 152064 logits, confidences <= 1e-3, tokens and unmask sets
identical except at counted near ties."""
import numpy as np
import pytest
import torch

from kv_cache_decode_dualcache_b200 import synth
from oracle.decode import confidence, select_unmask
from oracle.model import Model
from tests.gpu_util import make_decoder, require_gpu
from tests.parity import StepReport, compare_step

pytestmark = pytest.mark.gpu

P, G, B, TAU = 224, 32, 32, 0.9


@pytest.fixture(scope="module")
def dream():
    require_gpu()
    shape = synth.DREAM_7B
    w = synth.make_weights(shape, device="cuda")
    dec = make_decoder(shape, w, P + G)
    w_host = {k: v.cpu() for k, v in w.items()}
    del w
    torch.cuda.empty_cache()
    model = Model(shape.as_dict(), w_host)
    yield shape, dec, model
    dec.close()


def test_dream7b_first_block_teacher_forced(dream):
    shape, dec, model = dream
    mask = shape.mask_id
    L = P + G
    s = P
    prompt = synth.make_prompt(shape, P).numpy()
    x0 = np.concatenate([prompt, np.full(G, mask)]).astype(np.int64)
    rep = StepReport()

    z, kv = model.forward(x0, range(L), return_kv=True, head_rows=range(s, s + B))
    conf, tok = confidence(z, mask)
    ref = {"z": z, "conf": conf, "tok": tok,
           "unmask": select_unmask(np.ones(B, bool), conf, TAU)}
    g = dec.step_debug(x0, x0, s, B, TAU, "dual")
    compare_step(g, ref, np.ones(B, bool), TAU, mask, rep, z_tol=3e-2, label="refresh")

    x = x0.copy()
    for i in range(2):
        x[s:s + B][ref["unmask"]] = ref["tok"][ref["unmask"]]
        masked = x[s:s + B] == mask
        if not masked.any():
            break
        z = model.forward(x, range(s, s + B), cache=kv)
        conf, tok = confidence(z, mask)
        ref = {"z": z, "conf": conf, "tok": tok, "unmask": select_unmask(masked, conf, TAU)}
        g = dec.step_debug(x0, x, s, B, TAU, "dual")
        compare_step(g, ref, masked, TAU, mask, rep, z_tol=3e-2, label=f"dual step {i + 1}")

    print(f"dream7b: steps {rep.steps} max|dz| {rep.max_dz:.3g} max|dconf| {rep.max_dconf:.3g} "
          f"near-tie exemptions {rep.exempt}")
    assert rep.steps >= 2
    assert not rep.mismatches, rep.mismatches[:5]
