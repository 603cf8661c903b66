"""Full-size parity: the LLaDA-8B shape (32 layers, d=4096, V=126464) in the
workload bench.py times (prompt 256, block 32, tau 0.9, DualCache), against
the float64 oracle.

Teacher-forced on the first block: the block-start full forward (refresh
step), then two DualCache steps on the sequence the oracle's own unmask
decisions produce.  Each step: logits max-abs <= 3e-2 over all 32 x 126464
logits, confidences <= 1e-3, tokens and unmask sets identical except at
counted near ties.  The oracle runs one float64 full forward (~40 s on 16
host cores) and two block steps (~20 s each).

A later block through the production path: the generation bench.py times
(CUDA-graph replay, programmatic dependent launches, the chain kernel) runs
with its per-step trace, and the oracle recomputes the first two steps of
block 3 (a decoded prefix of prompt + three blocks, a masked suffix of four
blocks) on the GPU's own sequence."""
import numpy as np
import pytest
import torch

from kv_cache_decode_dualcache_b200 import synth
from oracle.decode import confidence, select_unmask
from oracle.model import Model
from tests.gpu_util import make_decoder, require_gpu
from tests.parity import StepReport, compare_step, replay_gpu_trace

pytestmark = pytest.mark.gpu

WL = synth.WORKLOADS["llada8b-p256-g256"]


@pytest.fixture(scope="module")
def full_size():
    require_gpu()
    shape = WL.shape
    w = synth.make_weights(shape, device="cuda")
    dec = make_decoder(shape, w, WL.prompt_len + WL.gen_len)
    w_host = {k: v.cpu() for k, v in w.items()}
    del w
    torch.cuda.empty_cache()
    model = Model(shape.as_dict(), w_host)
    return shape, dec, model


def test_llada8b_first_block_teacher_forced(full_size):
    shape, dec, model = full_size
    P, G, B, tau = WL.prompt_len, WL.gen_len, WL.block_size, WL.tau
    mask = shape.mask_id
    L = P + G
    s = P
    prompt = synth.make_prompt(shape, P).numpy()
    x0 = np.concatenate([prompt, np.full(G, mask)]).astype(np.int64)
    rep = StepReport()

    # refresh step: full forward of x0, logits for the block rows
    z, kv = model.forward(x0, range(L), return_kv=True, head_rows=range(s, s + B))
    conf, tok = confidence(z, mask)
    ref = {"z": z, "conf": conf, "tok": tok,
           "unmask": select_unmask(np.ones(B, bool), conf, tau)}
    g = dec.step_debug(x0, x0, s, B, tau, "dual")
    compare_step(g, ref, np.ones(B, bool), tau, mask, rep, z_tol=3e-2, label="refresh")

    # two DualCache steps on the oracle's decisions, cache from x0's refresh
    x = x0.copy()
    for i in range(2):
        x[s:s + B][ref["unmask"]] = ref["tok"][ref["unmask"]]
        masked = x[s:s + B] == mask
        if not masked.any():
            break
        z = model.forward(x, range(s, s + B), cache=kv)
        conf, tok = confidence(z, mask)
        ref = {"z": z, "conf": conf, "tok": tok, "unmask": select_unmask(masked, conf, tau)}
        g = dec.step_debug(x0, x, s, B, tau, "dual")
        compare_step(g, ref, masked, tau, mask, rep, z_tol=3e-2, label=f"dual step {i + 1}")

    print(f"llada8b first block: {rep.summary()}")
    assert rep.steps >= 2
    assert not rep.mismatches, rep.mismatches[:5]


def test_llada8b_later_block_production_path(full_size):
    shape, dec, model = full_size
    P, G, B, tau = WL.prompt_len, WL.gen_len, WL.block_size, WL.tau
    prompt = synth.make_prompt(shape, P).numpy()
    out, steps, st = dec.generate(prompt, G, B, tau, "dual", trace=True)
    assert len(st.trace_block) == steps and list(np.bincount(st.trace_block)) == st.steps_per_block
    rep = replay_gpu_trace(model, prompt, G, B, tau, "dual", out, st, blocks={3},
                           max_steps_per_block=2, label="llada8b block 3")
    print(f"llada8b block 3 (production path): {rep.summary()}")
    assert rep.steps >= 1
    assert not rep.mismatches, rep.mismatches[:5]
