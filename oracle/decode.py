"""Block-wise decoding with confidence thresholding and KV-cache modes (oracle).

Test infrastructure only; see ``oracle/__init__.py``.

The procedure, in the order the pages give it:

* Generation is split into blocks decoded left to right; before a block is
  decoded the K/V of the other blocks is computed and kept for reuse, and once
  the block is finished the K/V of all blocks is recomputed (techwalker.com
  Fast-dLLM article, section "核心创新：适合扩散模型的KV缓存", the two numbered
  items).  DualCache keeps both the prefix (prompt and finished blocks) and the
  suffix (still-masked blocks) (same section, last paragraph; ccyt168.com
  overview, section 一, item 1 "双向缓存策略").
* In each step, every masked position of the current block whose confidence
  (the probability the model gives the token; ccyt168.com overview, section
  一, item 2) reaches the threshold is unmasked in parallel; the others wait
  (same item, "阈值激活策略"; techwalker.com article, section
  "解决并行解码的质量下降问题").

Readings taken where the pages are silent (each one is listed in the design
notes of this repository):

* The block-start full forward is the block's first step: its logits for the
  block rows are used to unmask, and it counts as a step.  There is no
  refresh after the last block.
* ``conf >= tau`` unmasks.  When no masked position of the block passes, the
  single most confident one is unmasked (lowest position on ties), so each
  step unmasks at least one token and a block takes at most ``block`` steps.
* The mask id is excluded from both the argmax and the softmax.  Argmax ties
  go to the lowest token id.
* Only masked positions of the current block are candidates.
* DualCache steps recompute only the block rows; their fresh K/V is used in
  that step's attention and is not kept (the next refresh rewrites every
  position anyway).  Prefix-cache steps recompute rows [s, L) over the cached
  prefix [0, s).  Cache mode "none" runs a full forward every step.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence

import numpy as np

from .numerics import logsumexp

CACHE_NONE, CACHE_PREFIX, CACHE_DUAL = 0, 1, 2
_MODE_NAMES = {"none": CACHE_NONE, "prefix": CACHE_PREFIX, "dual": CACHE_DUAL}


def cache_mode_id(mode) -> int:
    if isinstance(mode, str):
        return _MODE_NAMES[mode]
    if mode not in (CACHE_NONE, CACHE_PREFIX, CACHE_DUAL):
        raise ValueError(f"unknown cache mode {mode!r}")
    return int(mode)


def confidence(z: np.ndarray, mask_id: int):
    """Per row: token = argmax over ids != mask_id (lowest id on ties) and
    confidence = its softmax probability over ids != mask_id.

    z: [rows, vocab].  Returns (conf float64 [rows], tok int64 [rows]).
    """
    z = np.array(z, dtype=np.float64, copy=True)
    z[:, mask_id] = -np.inf
    tok = np.argmax(z, axis=1)  # numpy returns the first (lowest) index of the max
    lse = logsumexp(z, axis=1)
    conf = np.exp(z[np.arange(z.shape[0]), tok] - lse)
    return conf, tok.astype(np.int64)


def select_unmask(masked: np.ndarray, conf: np.ndarray, tau: float) -> np.ndarray:
    """Unmask set of one step: masked positions with conf >= tau; if none, the
    single most confident masked position (lowest position on ties).  Empty
    when nothing is masked."""
    masked = np.asarray(masked, dtype=bool)
    u = masked & (np.asarray(conf) >= tau)
    if not u.any() and masked.any():
        cand = np.flatnonzero(masked)
        best = cand[np.argmax(np.asarray(conf)[cand])]
        u[best] = True
    return u


def select_top_k(masked: np.ndarray, conf: np.ndarray, k: int) -> np.ndarray:
    """Unmask set of one step of the fixed-count strategy that the threshold
    rule replaces (techwalker.com Fast-dLLM article, section
    "解决并行解码的质量下降问题": earlier methods unmask a fixed number of
    tokens per step): the k most confident masked positions, the lower
    position first among equal confidences; every masked position when fewer
    than k are masked."""
    masked = np.asarray(masked, dtype=bool)
    conf = np.asarray(conf, dtype=np.float64)
    cand = [int(i) for i in np.flatnonzero(masked)]
    cand.sort(key=lambda i: (-conf[i], i))
    u = np.zeros(masked.shape, dtype=bool)
    u[cand[:max(0, int(k))]] = True
    return u


@dataclass
class StepRecord:
    block: int
    kind: str                  # "refresh", "dual", "prefix", "full"
    conf: np.ndarray           # [B] confidence of every block row
    tok: np.ndarray            # [B] argmax token of every block row
    unmask: np.ndarray         # [B] bool
    z: Optional[np.ndarray] = None


@dataclass
class GenerateResult:
    tokens: np.ndarray         # [gen_len]
    steps: int
    steps_per_block: List[int]
    trace: List[StepRecord] = field(default_factory=list)


def generate(model, prompt: Sequence[int], gen_len: int, block_size: int, tau: float,
             cache_mode="dual", keep_logits: bool = False, on_refresh=None,
             fixed_k: Optional[int] = None) -> GenerateResult:
    """Block-wise generation (see module docstring).  With ``fixed_k`` every
    step unmasks the fixed_k most confident masked positions of the block
    (``select_top_k``) instead of applying the threshold rule; tau is unused.

    ``model`` is anything with ``spec.mask_id`` and
    ``forward(x, rows, cache=None, return_kv=False, head_rows=None)``; the
    (n+1)*eps toy of ``oracle.theorem`` plugs in here.  ``on_refresh(x, kv)``
    is called after every block-start full forward with the K/V it stored.
    """
    mode = cache_mode_id(cache_mode)
    mask_id = model.spec.mask_id
    prompt = np.asarray(prompt, dtype=np.int64)
    P = prompt.shape[0]
    if gen_len % block_size != 0:
        raise ValueError("gen_len must be a multiple of block_size")
    L = P + gen_len
    x = np.concatenate([prompt, np.full(gen_len, mask_id, dtype=np.int64)])
    all_rows = np.arange(L)
    res = GenerateResult(tokens=np.empty(0, np.int64), steps=0, steps_per_block=[])
    for b in range(gen_len // block_size):
        s = P + b * block_size
        e = s + block_size
        block_rows = np.arange(s, e)
        cache = None
        first = True
        n_steps = 0
        while np.any(x[s:e] == mask_id):
            if first or mode == CACHE_NONE:
                z, kv = model.forward(x, all_rows, return_kv=True, head_rows=block_rows)
                kind = "refresh" if first else "full"
                if first and mode != CACHE_NONE:
                    cache = kv
                    if on_refresh is not None:
                        on_refresh(x.copy(), kv)
            elif mode == CACHE_DUAL:
                z = model.forward(x, block_rows, cache=cache)
                kind = "dual"
            else:  # CACHE_PREFIX: rows [s, L) fresh over the cached prefix [0, s)
                rows = np.arange(s, L)
                z = model.forward(x, rows, cache=cache, head_rows=np.arange(block_size))
                kind = "prefix"
            first = False
            conf, tok = confidence(z, mask_id)
            masked = x[s:e] == mask_id
            u = select_top_k(masked, conf, fixed_k) if fixed_k else select_unmask(masked, conf, tau)
            x[s:e][u] = tok[u]
            n_steps += 1
            res.trace.append(StepRecord(b, kind, conf, tok, u, z if keep_logits else None))
        res.steps_per_block.append(n_steps)
        res.steps += n_steps
    res.tokens = x[P:].copy()
    return res


def step(model, snapshot_ids: Sequence[int], current_ids: Sequence[int], block_start: int,
         block_size: int, tau: float, cache_mode="dual") -> Dict[str, np.ndarray]:
    """One teacher-forced decode step.

    The K/V cache is the full forward of ``snapshot_ids`` (the sequence when
    the block started).  When ``current_ids`` equals the snapshot the step is
    the block's first (refresh) step and its logits come from that full
    forward; otherwise the step runs in ``cache_mode`` on ``current_ids``.
    Mode "none" always runs a full forward on ``current_ids``.

    Returns dict with z [B, V], conf [B], tok [B], unmask [B] (bool) and kind.
    """
    mode = cache_mode_id(cache_mode)
    mask_id = model.spec.mask_id
    snap = np.asarray(snapshot_ids, dtype=np.int64)
    cur = np.asarray(current_ids, dtype=np.int64)
    L = cur.shape[0]
    s, e = block_start, block_start + block_size
    block_rows = np.arange(s, e)
    all_rows = np.arange(L)
    if mode == CACHE_NONE:
        z = model.forward(cur, all_rows, head_rows=block_rows)
        kind = "full"
    elif np.array_equal(snap, cur):
        z = model.forward(cur, all_rows, head_rows=block_rows)
        kind = "refresh"
    else:
        _, kv = model.forward(snap, all_rows, return_kv=True, head_rows=np.arange(0))
        if mode == CACHE_DUAL:
            z = model.forward(cur, block_rows, cache=kv)
            kind = "dual"
        else:
            z = model.forward(cur, np.arange(s, L), cache=kv, head_rows=np.arange(block_size))
            kind = "prefix"
    conf, tok = confidence(z, mask_id)
    u = select_unmask(cur[s:e] == mask_id, conf, tau)
    return {"z": z, "conf": conf, "tok": tok, "unmask": u, "kind": kind}
