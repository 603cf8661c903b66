"""Closed-form pin of the oracle's whole forward and confidence rule.

A hand-built one-layer model whose output can be worked out by hand:

* Wq = 0, so every attention score is 0 and each query averages the values of
  ALL positions (before and after it: no causal mask).
* Wv = Wo = identity, so the attention branch adds mean_j RMSNorm(E[x_j]).
* W_gate = 0, so silu(0) * up = 0 and the FFN adds nothing.
* W_head rows: e0, e1, e2, e3, e0 again (a tie with id 0), and 10 * e0 for the
  mask id (largest logit, must be excluded).

So for position i: h = E[x_i] + mean_j E[x_j] / rms_j with
rms_j = sqrt(mean(E[x_j]^2) + eps); a = h / sqrt(mean(h^2) + eps);
z[v] = scale * <a, W_head[v]>.
"""
import numpy as np

from oracle.decode import confidence, select_unmask
from oracle.model import Model

EPS = 1e-5
SCALE = 3.0
SPEC = dict(n_layers=1, d_model=4, n_heads=1, n_kv_heads=1, head_dim=4, ffn_dim=4, vocab=6,
            mask_id=5, rope_theta=1e4, rms_eps=EPS, logit_scale=SCALE)


def _weights():
    I4 = np.eye(4)
    E = np.array([[2.0, 0, 0, 0], [0, 2.0, 0, 0], [0, 0, 2.0, 0], [0, 0, 0, 2.0],
                  [1.0, 1.0, 0, 0], [0, 0, 0, 1.0]])
    head = np.vstack([I4, I4[0], 10.0 * I4[0]])
    rng = np.random.default_rng(0)
    return {
        "embed": E, "final_norm": np.ones(4), "lm_head": head,
        "layers.0.attn_norm": np.ones(4), "layers.0.ffn_norm": np.ones(4),
        "layers.0.wq": np.zeros((4, 4)), "layers.0.wk": rng.standard_normal((4, 4)),
        "layers.0.wv": I4, "layers.0.wo": I4, "layers.0.w_gate": np.zeros((4, 4)),
        "layers.0.w_up": rng.standard_normal((4, 4)), "layers.0.w_down": rng.standard_normal((4, 4)),
    }


def _by_hand(x):
    E = _weights()["embed"]
    rows = E[x]
    normed = [r / np.sqrt(np.mean(r ** 2) + EPS) for r in rows]
    mean_v = sum(normed) / len(normed)
    out = []
    for r in rows:
        h = r + mean_v
        a = h / np.sqrt(np.mean(h ** 2) + EPS)
        out.append(SCALE * np.array([a[0], a[1], a[2], a[3], a[0], 10 * a[0]]))
    return np.array(out)


def test_forward_matches_hand_derivation():
    m = Model(SPEC, _weights())
    x = [0, 2, 4, 5, 5, 1]
    z = m.forward(x, range(len(x)))
    np.testing.assert_allclose(z, _by_hand(x), rtol=1e-13)


def test_suffix_positions_change_every_row():
    # Bidirectional: changing the last token changes the first row's logits.
    m = Model(SPEC, _weights())
    z1 = m.forward([0, 1, 2], range(3))
    z2 = m.forward([0, 1, 3], range(3))
    assert np.abs(z1[0] - z2[0]).max() > 1e-3


def test_confidence_excludes_mask_and_breaks_ties_low():
    m = Model(SPEC, _weights())
    x = [0, 0, 5]
    z = m.forward(x, range(3))
    conf, tok = confidence(z, SPEC["mask_id"])
    # Row 0: coordinate 0 dominates; ids 0 and 4 tie, the mask id (10x) is excluded.
    assert tok[0] == 0
    zr = _by_hand(x)[0]
    zz = zr[:5]
    expect = np.exp(zz[0]) / np.sum(np.exp(zz))    # softmax over the five non-mask ids
    np.testing.assert_allclose(conf[0], expect, rtol=1e-12)
    # Row 2 is the mask embedding (e3 direction mixed with the mean); by hand:
    assert tok[2] == int(np.argmax(_by_hand(x)[2][:5]))


def test_select_rule_threshold_and_fallback():
    masked = np.array([True, True, False, True])
    conf = np.array([0.95, 0.5, 0.99, 0.9])
    np.testing.assert_array_equal(select_unmask(masked, conf, 0.9), [True, False, False, True])
    # Nothing passes: the single most confident masked position (not position 2,
    # which is not masked).
    np.testing.assert_array_equal(select_unmask(masked, conf, 0.97), [True, False, False, False])
    # Ties in the fallback go to the lowest position.
    np.testing.assert_array_equal(
        select_unmask(np.array([False, True, True]), np.array([0.9, 0.4, 0.4]), 0.5),
        [False, True, False])
    # Nothing masked: nothing to unmask.
    assert not select_unmask(np.zeros(3, bool), np.ones(3), 0.5).any()
    # tau <= 0 unmasks every masked position.
    np.testing.assert_array_equal(select_unmask(masked, conf, 0.0), masked)
