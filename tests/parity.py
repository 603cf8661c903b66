"""Shared helpers for the GPU parity tests (teacher-forced per-step compare).

The acceptance rule: per step, logits max-abs within ``z_tol`` (1e-4 for the
float32 model, 3e-2 for the bf16 model, both against the exact float64
oracle), confidences within 1e-3, and token ids / unmask sets identical
except at positions where the oracle's top-2 logit margin or |conf - tau| is
below 1e-3; those positions are counted and returned.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List

import numpy as np

NEAR = 1e-3


@dataclass
class StepReport:
    max_dz: float = 0.0
    max_dconf: float = 0.0
    exempt: int = 0
    steps: int = 0
    mismatches: List[str] = field(default_factory=list)


def top2_margin(z: np.ndarray, mask_id: int) -> np.ndarray:
    zz = np.array(z, dtype=np.float64, copy=True)
    zz[:, mask_id] = -np.inf
    part = np.partition(zz, -2, axis=1)
    return part[:, -1] - part[:, -2]


def compare_step(gpu: dict, ref: dict, masked: np.ndarray, tau: float, mask_id: int,
                 rep: StepReport, z_tol: float, conf_tol: float = 1e-3, label: str = "") -> None:
    rep.steps += 1
    if gpu.get("z") is not None:
        dz = float(np.abs(gpu["z"].astype(np.float64) - ref["z"]).max())
        rep.max_dz = max(rep.max_dz, dz)
        if dz > z_tol:
            rep.mismatches.append(f"{label}: logits max-abs {dz:.3g} > {z_tol}")
    dc = float(np.abs(gpu["conf"].astype(np.float64) - ref["conf"]).max())
    rep.max_dconf = max(rep.max_dconf, dc)
    if dc > conf_tol:
        rep.mismatches.append(f"{label}: conf max-abs {dc:.3g} > {conf_tol}")
    margin = top2_margin(ref["z"], mask_id)
    near_tie = margin < NEAR
    near_tau = np.abs(ref["conf"] - tau) < NEAR
    for i in range(len(ref["tok"])):
        tok_ok = int(gpu["tok"][i]) == int(ref["tok"][i])
        if not tok_ok:
            if near_tie[i]:
                rep.exempt += 1
            else:
                rep.mismatches.append(f"{label}: row {i} token {gpu['tok'][i]} != {ref['tok'][i]}")
    if not np.array_equal(gpu["unmask"], ref["unmask"]):
        diff = np.flatnonzero(gpu["unmask"] != ref["unmask"])
        if np.all(near_tau[diff] | near_tie[diff]) or _fallback_tie(ref, masked, diff):
            rep.exempt += len(diff)
        else:
            rep.mismatches.append(f"{label}: unmask sets differ at {diff.tolist()}")


def _fallback_tie(ref: dict, masked: np.ndarray, diff: np.ndarray) -> bool:
    """A fallback pick may differ when the top two masked confidences are
    within the tolerance."""
    c = np.where(masked, ref["conf"], -np.inf)
    if np.sum(masked) < 2:
        return False
    top = np.sort(c)[-2:]
    return (top[1] - top[0]) < NEAR


def teacher_forced(dec, model, trace, prompt, gen_len: int, block: int, tau: float, mode: str,
                   mask_id: int, z_tol: float, max_steps=None, stride: int = 1) -> StepReport:
    """Replay the oracle's free-running trace step by step on the GPU."""
    from oracle.decode import step as oracle_step
    rep = StepReport()
    P = len(prompt)
    x = np.concatenate([np.asarray(prompt, np.int64), np.full(gen_len, mask_id, np.int64)])
    snap = None
    for idx, r in enumerate(trace):
        s = P + block * r.block
        if r.kind == "refresh" or (mode == "none" and snap is None):
            snap = x.copy()
        if mode == "none" and (idx == 0 or trace[idx - 1].block != r.block):
            snap = x.copy()
        if idx % stride == 0 and (max_steps is None or rep.steps < max_steps):
            ref = {"z": r.z, "conf": r.conf, "tok": r.tok, "unmask": r.unmask}
            if ref["z"] is None:
                ref = oracle_step(model, snap, x, s, block, tau, mode)
            g = dec.step_debug(snap, x, s, block, tau, mode)
            compare_step(g, ref, x[s:s + block] == mask_id, tau, mask_id, rep, z_tol,
                         label=f"step {idx} ({r.kind}, block {r.block})")
        x[s:s + block][r.unmask] = r.tok[r.unmask]
    return rep
