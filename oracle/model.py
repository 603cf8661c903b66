"""The bidirectional masked-diffusion transformer ``f`` in float64 (oracle).

Test infrastructure only; see ``oracle/__init__.py``.

What the pages fix about ``f``: a masked-diffusion LLM (LLaDA / Dream) is a
transformer whose attention is bidirectional: every position attends to every
other position, with no causal mask (techwalker.com Fast-dLLM article, section
"核心创新：适合扩散模型的KV缓存": the diffusion model looks at all parts of the
text at once, which is why autoregressive KV caching does not apply directly).
The layer itself (pre-norm RMSNorm, rotary position embedding, multi-head or
grouped-query attention, SwiGLU FFN, untied LM head) is the LLaDA / Dream
architecture the pages name; its shapes come from the workload definitions.

Plain readings taken where the pages say nothing:
  * RoPE is the rotate-half form: the pair (x[i], x[i + hd/2]) of each head is
    rotated by angle pos * theta**(-2i/hd).
  * RMSNorm: h / sqrt(mean(h^2) + eps) * g, eps inside the square root.
  * GQA: query head j reads KV head j // (H / Hkv).
  * Attention scale 1/sqrt(hd); no bias terms anywhere; the LM head output is
    multiplied by ``logit_scale``.

K and V are carried explicitly per position: ``forward`` computes fresh K/V
for the query ``rows`` only and takes every other position's K/V from
``cache``.  This is the one place cached and fresh keys meet, so a full
forward (rows = all positions), a DualCache block step (rows = the block,
cache = prefix + suffix) and a prefix-cache step (rows = [s, L), cache =
prefix) all run the same code.

``emulate_bf16`` rounds to bfloat16 (via float32, RNE) exactly where a
bfloat16 device path stores values: every GEMM input activation (the three
RMSNorm outputs, the attention output, the SwiGLU product), the rotated q and
k and the v that enter attention (k and v are what the KV cache stores), and
the residual stream is rounded to float32.  Accumulation, softmax and the
logits stay float64.
"""
from __future__ import annotations

from dataclasses import dataclass, fields
from typing import Dict, List, Mapping, Optional, Sequence, Tuple

import numpy as np

from .numerics import round_bf16, round_f32, silu

KV = Tuple[np.ndarray, np.ndarray]  # (K [L, Hkv, hd], V [L, Hkv, hd]) of one layer


@dataclass(frozen=True)
class Spec:
    n_layers: int
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn_dim: int
    vocab: int
    mask_id: int
    rope_theta: float
    rms_eps: float
    logit_scale: float

    @staticmethod
    def from_mapping(m: Mapping) -> "Spec":
        names = {f.name for f in fields(Spec)}
        return Spec(**{k: m[k] for k in names})


def to_f64(w) -> np.ndarray:
    """Host float64 copy of a numpy array or a CPU torch tensor (any dtype)."""
    if hasattr(w, "detach"):
        w = w.detach()
        if w.is_cuda:
            raise ValueError("oracle weights must be host tensors")
        return w.float().numpy().astype(np.float64)
    return np.asarray(w, dtype=np.float64)


def rmsnorm(h: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    ms = np.mean(h * h, axis=-1, keepdims=True)
    return h / np.sqrt(ms + eps) * g


def rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half RoPE.  x: [M, heads, hd]; pos: [M] absolute positions."""
    hd = x.shape[-1]
    half = hd // 2
    i = np.arange(half, dtype=np.float64)
    inv_freq = theta ** (-2.0 * i / hd)
    ang = pos.astype(np.float64)[:, None] * inv_freq[None, :]  # [M, half]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1 = x[..., :half]
    x2 = x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """softmax(q k^T / sqrt(hd)) v per head, no mask.

    q: [M, H, hd]; k, v: [L, Hkv, hd]; returns [M, H, hd].
    """
    m, h, hd = q.shape
    hkv = k.shape[1]
    rep = h // hkv
    out = np.empty_like(q)
    scale = 1.0 / np.sqrt(hd)
    for j in range(h):
        g = j // rep
        s = (q[:, j, :] @ k[:, g, :].T) * scale          # [M, L]
        s = s - np.max(s, axis=-1, keepdims=True)
        p = np.exp(s)
        p = p / np.sum(p, axis=-1, keepdims=True)
        out[:, j, :] = p @ v[:, g, :]
    return out


class Model:
    """Float64 forward of ``f`` with explicit K/V (see module docstring)."""

    def __init__(self, spec, weights: Mapping[str, object], emulate_bf16: bool = False,
                 keep_f64: Optional[bool] = None):
        self.spec = spec if isinstance(spec, Spec) else Spec.from_mapping(spec)
        self.w = weights
        self.emulate_bf16 = bool(emulate_bf16)
        s = self.spec
        n_params = s.n_layers * (s.d_model * (s.n_heads + 2 * s.n_kv_heads) * s.head_dim
                                 + s.n_heads * s.head_dim * s.d_model + 3 * s.d_model * s.ffn_dim)
        # Small models keep their float64 copies; large ones convert one layer at a time.
        self.keep_f64 = (n_params < 50_000_000) if keep_f64 is None else keep_f64
        self._cache: Dict[str, np.ndarray] = {}

    # -- weights -----------------------------------------------------------
    def _get(self, name: str) -> np.ndarray:
        if name in self._cache:
            return self._cache[name]
        a = to_f64(self.w[name])
        if self.keep_f64:
            self._cache[name] = a
        return a

    def _embed_rows(self, ids: np.ndarray) -> np.ndarray:
        e = self.w["embed"]
        if hasattr(e, "detach"):
            import torch  # host tensors only; plain CPU indexing
            return e[torch.as_tensor(np.asarray(ids, dtype=np.int64))].float().numpy().astype(np.float64)
        return np.asarray(e, dtype=np.float64)[np.asarray(ids)]

    def _rb(self, x: np.ndarray) -> np.ndarray:
        return round_bf16(x) if self.emulate_bf16 else x

    def _rf(self, x: np.ndarray) -> np.ndarray:
        return round_f32(x) if self.emulate_bf16 else x

    # -- forward -----------------------------------------------------------
    def forward(self, x: Sequence[int], rows: Sequence[int], cache: Optional[List[KV]] = None,
                return_kv: bool = False, return_hidden: bool = False,
                head_rows: Optional[Sequence[int]] = None):
        """Logits z for the query ``rows`` of the token sequence ``x``.

        Positions in ``rows`` get fresh K/V computed from their hidden states;
        every other position takes its K/V from ``cache`` (required unless
        ``rows`` covers the whole sequence).  Returns ``z`` of shape
        [len(rows), vocab], plus, with ``return_kv``, the list of per-layer
        K/V over the whole sequence as used by attention (fresh rows merged
        into the cached ones).  ``head_rows`` (indices into ``rows``) limits
        the LM head to those rows; the default is every row.
        """
        s = self.spec
        x = np.asarray(x, dtype=np.int64)
        rows = np.asarray(rows, dtype=np.int64)
        L = x.shape[0]
        M = rows.shape[0]
        full = (M == L) and np.array_equal(rows, np.arange(L))
        if cache is None and not full:
            raise ValueError("a partial forward needs cached K/V for the other positions")
        H, Hkv, hd = s.n_heads, s.n_kv_heads, s.head_dim

        h = self._rf(self._embed_rows(x[rows]))
        kv_out: List[KV] = []
        for li in range(s.n_layers):
            p = f"layers.{li}."
            a = self._rb(rmsnorm(h, self._get(p + "attn_norm"), s.rms_eps))
            q = (a @ self._get(p + "wq").T).reshape(M, H, hd)
            k = (a @ self._get(p + "wk").T).reshape(M, Hkv, hd)
            v = (a @ self._get(p + "wv").T).reshape(M, Hkv, hd)
            q = self._rb(rope(q, rows, s.rope_theta))
            k = self._rb(rope(k, rows, s.rope_theta))
            v = self._rb(v)
            if full:
                k_all, v_all = k, v
            else:
                k_all = np.array(cache[li][0], dtype=np.float64, copy=True)
                v_all = np.array(cache[li][1], dtype=np.float64, copy=True)
                k_all[rows] = k
                v_all[rows] = v
            if return_kv:
                kv_out.append((k_all, v_all))
            o = self._rb(attention(q, k_all, v_all)).reshape(M, H * hd)
            h = self._rf(h + o @ self._get(p + "wo").T)
            b = self._rb(rmsnorm(h, self._get(p + "ffn_norm"), s.rms_eps))
            f = self._rb(silu(b @ self._get(p + "w_gate").T) * (b @ self._get(p + "w_up").T))
            h = self._rf(h + f @ self._get(p + "w_down").T)
        if head_rows is not None:
            h = h[np.asarray(head_rows, dtype=np.int64)]
        a = self._rb(rmsnorm(h, self._get("final_norm"), s.rms_eps))
        z = s.logit_scale * (a @ self._get("lm_head").T)
        out = [z]
        if return_kv:
            out.append(kv_out)
        if return_hidden:
            out.append(a)
        return out[0] if len(out) == 1 else tuple(out)
