"""CPU checks of the GPU-vs-oracle acceptance rule in tests/parity.py.

The rule (tolerances from the decoder's specification): token ids may differ
only where the oracle's top-2 logit margin is below 1e-3; unmask sets may
differ only at positions whose oracle confidence is within 1e-3 of tau, or in
the fallback pick between two candidates within 1e-3 of each other when the
oracle had no position reaching tau.
"""
import numpy as np

from tests.parity import StepReport, compare_step, top2_margin

MASK = 7
TAU = 0.9


def _ref(conf, unmask, tok=None, z=None):
    B = len(conf)
    if z is None:
        z = np.zeros((B, 8))
        z[:, 1] = 5.0            # clear argmax 1, margin 5
    return {"z": z, "conf": np.asarray(conf, np.float64),
            "tok": np.ones(B, np.int64) if tok is None else np.asarray(tok),
            "unmask": np.asarray(unmask, bool)}


def _gpu(ref, unmask=None, tok=None, conf=None):
    return {"z": None, "conf": ref["conf"] if conf is None else np.asarray(conf),
            "tok": ref["tok"] if tok is None else np.asarray(tok),
            "unmask": ref["unmask"] if unmask is None else np.asarray(unmask, bool)}


def _run(gpu, ref, masked):
    rep = StepReport()
    compare_step(gpu, ref, np.asarray(masked, bool), TAU, MASK, rep, z_tol=3e-2)
    return rep


def test_identical_step_passes_without_exemptions():
    ref = _ref([0.95, 0.2, 0.91], [True, False, True])
    rep = _run(_gpu(ref), ref, [True, True, True])
    assert not rep.mismatches and rep.exempt == 0


def test_threshold_difference_far_from_tau_fails_even_with_unrelated_close_confidences():
    # positions 1 and 3 have near-equal low confidences, which must not excuse a
    # mismatch at position 0 (conf 0.95, far from tau)
    ref = _ref([0.95, 0.30, 0.10, 0.3004], [True, False, False, False])
    gpu = _gpu(ref, unmask=[False, False, False, False])
    rep = _run(gpu, ref, [True, True, True, True])
    assert rep.mismatches and rep.exempt == 0


def test_difference_within_1e3_of_tau_is_exempt_and_counted():
    ref = _ref([0.9004, 0.95, 0.2], [True, True, False])
    gpu = _gpu(ref, unmask=[False, True, False])
    rep = _run(gpu, ref, [True, True, True])
    assert not rep.mismatches and rep.exempt == 1 and rep.exempt_log


def test_near_tau_exemption_covers_only_near_tau_positions():
    # position 0 differs within 1e-3 of tau (exempt on its own), position 1
    # differs far from it: the step fails
    ref = _ref([0.9004, 0.95, 0.2], [True, True, False])
    gpu = _gpu(ref, unmask=[False, False, False])
    rep = _run(gpu, ref, [True, True, True])
    assert rep.mismatches and rep.exempt == 0


def test_fallback_pick_between_near_equal_candidates_is_exempt():
    # nothing reaches tau: the oracle picks position 2 (0.4003), the GPU position 0 (0.4)
    ref = _ref([0.4, 0.1, 0.4003], [False, False, True])
    gpu = _gpu(ref, unmask=[True, False, False])
    rep = _run(gpu, ref, [True, True, True])
    assert not rep.mismatches and rep.exempt == 2


def test_fallback_pick_between_distinct_candidates_fails():
    ref = _ref([0.4, 0.1, 0.45], [False, False, True])
    gpu = _gpu(ref, unmask=[True, False, False])
    assert _run(gpu, ref, [True, True, True]).mismatches


def test_fallback_exemption_needs_the_fallback_rule_in_play():
    # position 1 reaches tau in the oracle, so there is no fallback to excuse
    ref = _ref([0.4, 0.95, 0.4002], [False, True, False])
    gpu = _gpu(ref, unmask=[False, True, True])
    assert _run(gpu, ref, [True, True, True]).mismatches


def test_token_difference_needs_a_near_tie():
    z = np.zeros((2, 8))
    z[0, 1], z[0, 3] = 5.0, 5.0 - 5e-4   # near tie in row 0
    z[1, 1], z[1, 3] = 5.0, 4.0          # clear winner in row 1
    ref = _ref([0.5, 0.5], [False, False], tok=[1, 1], z=z)
    rep = _run(_gpu(ref, tok=[3, 1]), ref, [False, False])
    assert not rep.mismatches and rep.exempt == 1
    rep = _run(_gpu(ref, tok=[1, 3]), ref, [False, False])
    assert rep.mismatches


def test_confidence_tolerance():
    ref = _ref([0.5, 0.6], [False, True])
    assert _run(_gpu(ref, conf=[0.5, 0.6011]), ref, [True, True]).mismatches
    assert not _run(_gpu(ref, conf=[0.5, 0.6009]), ref, [True, True]).mismatches


def test_exemptions_stop_at_1e3():
    # 1.5e-3 from tau is not a near-tau difference
    ref = _ref([0.9015, 0.95, 0.2], [True, True, False])
    gpu = _gpu(ref, unmask=[False, True, False])
    rep = _run(gpu, ref, [True, True, True])
    assert rep.mismatches and rep.exempt == 0


def test_top2_margin_is_the_gap_between_the_two_largest_non_mask_logits():
    rng = np.random.default_rng(8)
    for width in (8, 1000):                  # a vocabulary-sized row as well
        z = rng.standard_normal((40, width))
        srt = np.sort(np.delete(z, MASK, axis=1), axis=1)
        np.testing.assert_array_equal(top2_margin(z, MASK), srt[:, -1] - srt[:, -2])
        z[:, MASK] = 100.0                   # the mask id's logit never counts
        np.testing.assert_array_equal(top2_margin(z, MASK), srt[:, -1] - srt[:, -2])


def test_report_summary_and_maxima():
    ref = _ref([0.9004, 0.95, 0.2], [True, True, False])
    gpu = _gpu(ref, unmask=[False, True, False], conf=[0.9004, 0.9502, 0.2])
    rep = _run(gpu, ref, [True, True, True])
    assert abs(rep.max_dconf - 2e-4) < 1e-12 and rep.max_dz == 0.0
    text = rep.summary()
    assert text.startswith("1 steps, ") and "exemptions 1 (" in text
    assert StepReport().summary() == "0 steps, max|dz| 0, max|dconf| 0, exemptions 0"
