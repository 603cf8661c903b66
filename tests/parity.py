"""Shared helpers for the GPU parity tests (teacher-forced per-step compare).

The acceptance rule: per step, logits max-abs within ``z_tol`` (1e-4 for the
float32 model, 3e-2 for the bf16 model, both against the exact float64
oracle), confidences within 1e-3, and token ids and unmask sets identical,
with two counted exemptions:

* a token id may differ where the oracle's top-2 logit margin is below 1e-3
  (the argmax is a near tie);
* an unmask set may differ at positions whose oracle confidence is within
  1e-3 of tau (membership depends on conf >= tau alone), or, when the oracle
  had no masked position reaching tau (the fallback rule picked its single
  most confident one), where the two sides' fallback picks differ and the
  oracle's confidences of those two picks are within 1e-3 of each other.

Each exemption is counted and described in ``StepReport.exempt_log``.
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
    exempt_log: List[str] = field(default_factory=list)

    def summary(self) -> str:
        return (f"{self.steps} steps, max|dz| {self.max_dz:.3g}, max|dconf| {self.max_dconf:.3g}, "
                f"exemptions {self.exempt}" + (f" ({'; '.join(self.exempt_log)})"
                                                if self.exempt_log else ""))


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
    near_tau = np.abs(np.asarray(ref["conf"], np.float64) - tau) < NEAR
    for i in range(len(ref["tok"])):
        if int(gpu["tok"][i]) != int(ref["tok"][i]):
            if near_tie[i]:
                rep.exempt += 1
                rep.exempt_log.append(f"{label}: row {i} token (top-2 margin {margin[i]:.2g})")
            else:
                rep.mismatches.append(f"{label}: row {i} token {gpu['tok'][i]} != {ref['tok'][i]}")
    g_u = np.asarray(gpu["unmask"], bool)
    r_u = np.asarray(ref["unmask"], bool)
    if not np.array_equal(g_u, r_u):
        diff = np.flatnonzero(g_u != r_u)
        if np.all(near_tau[diff]):
            rep.exempt += len(diff)
            rep.exempt_log.append(f"{label}: unmask {diff.tolist()} (|conf - tau| < {NEAR})")
        elif _fallback_tie(ref, g_u, r_u, masked, tau, diff):
            rep.exempt += len(diff)
            rep.exempt_log.append(f"{label}: fallback pick {diff.tolist()} (confidences within "
                                  f"{NEAR})")
        else:
            rep.mismatches.append(f"{label}: unmask sets differ at {diff.tolist()}")


def _fallback_tie(ref: dict, g_u: np.ndarray, r_u: np.ndarray, masked: np.ndarray, tau: float,
                  diff: np.ndarray) -> bool:
    """True when the difference is only the fallback rule's choice between two
    near-equal candidates: the oracle had no masked position with conf >= tau,
    each side unmasked exactly one position, those two positions are the whole
    difference, and the oracle's confidences of them are within NEAR."""
    conf = np.asarray(ref["conf"], np.float64)
    masked = np.asarray(masked, bool)
    if np.any(masked & (conf >= tau)):
        return False
    if g_u.sum() != 1 or r_u.sum() != 1:
        return False
    o, g = int(np.flatnonzero(r_u)[0]), int(np.flatnonzero(g_u)[0])
    if sorted(diff.tolist()) != sorted([o, g]) or not masked[g]:
        return False
    return abs(conf[o] - conf[g]) < NEAR


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


def replay_gpu_trace(model, prompt, gen_len: int, block: int, tau: float, mode: str, tokens,
                     stats, z_tol: float = float("inf"), blocks=None, max_steps_per_block=None,
                     label: str = "") -> StepReport:
    """Check a production generate (``Decoder.generate(..., trace=True)``)
    against the oracle on the GPU's own decisions.

    Every step the GPU took is recomputed by the oracle on the same current
    sequence (the K/V cache is the oracle's full forward of the sequence at
    the block's first step, as the decode procedure fixes), compared with
    ``compare_step`` (confidence, token, unmask set; the trace has no
    logits), and then the GPU's unmask decisions are applied, so later steps
    see the GPU's sequence.  ``blocks`` limits the oracle to those block
    indices (the other blocks only replay the GPU's decisions);
    ``max_steps_per_block`` limits the compared steps of a block.  Finally the
    replayed sequence must equal the tokens the GPU returned, every block must
    end with nothing masked, and the blocks must run in order.
    """
    from oracle.decode import confidence, select_unmask
    mask_id = model.spec.mask_id
    P = len(prompt)
    L = P + gen_len
    x = np.concatenate([np.asarray(prompt, np.int64), np.full(gen_len, mask_id, np.int64)])
    rep = StepReport()
    kv = None
    cur = -1
    in_block = 0
    for i in range(len(stats.trace_block)):
        b = int(stats.trace_block[i])
        s, e = P + b * block, P + (b + 1) * block
        first = b != cur
        if first:
            if cur >= 0 and np.any(x[P + cur * block:P + (cur + 1) * block] == mask_id):
                rep.mismatches.append(f"{label}: block {cur} left masked positions")
            if b != cur + 1:
                rep.mismatches.append(f"{label}: block {b} after block {cur}")
            cur, in_block = b, 0
        masked = x[s:e] == mask_id
        g = {"z": None, "conf": stats.trace_conf[i], "tok": stats.trace_tok[i],
             "unmask": np.asarray(stats.trace_unmask[i], bool)}
        check = (blocks is None or b in blocks) and (max_steps_per_block is None
                                                     or in_block < max_steps_per_block)
        if check:
            if mode == "none" or first:
                z, kv_full = model.forward(x, range(L), return_kv=True, head_rows=range(s, e))
                if first:
                    kv = kv_full
            elif mode == "dual":
                z = model.forward(x, range(s, e), cache=kv)
            else:
                z = model.forward(x, range(s, L), cache=kv, head_rows=range(block))
            conf, tok = confidence(z, mask_id)
            ref = {"z": z, "conf": conf, "tok": tok, "unmask": select_unmask(masked, conf, tau)}
            compare_step(g, ref, masked, tau, mask_id, rep, z_tol,
                         label=f"{label} step {i} (block {b}, {'first' if first else mode})")
        elif first and mode != "none":
            kv = None   # a later checked step of this block would need its refresh
        if np.any(g["unmask"] & ~masked):
            rep.mismatches.append(f"{label}: step {i} unmasked an already decoded position")
        if not g["unmask"].any():
            rep.mismatches.append(f"{label}: step {i} unmasked nothing")
        x[s:e][g["unmask"]] = g["tok"][g["unmask"]]
        in_block += 1
    if np.any(x[P:] == mask_id):
        rep.mismatches.append(f"{label}: masked positions left after the last step")
    if not np.array_equal(x[P:], np.asarray(tokens, np.int64)):
        rep.mismatches.append(f"{label}: returned tokens differ from the traced decisions")
    return rep
