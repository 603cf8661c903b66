"""Seeded synthetic inputs: model shapes, random weights and prompts.

This module is the only thing the oracle and the CUDA library both consume.
It holds none of the decoder's arithmetic: it only names shapes and draws
random numbers.

Recipe (one line per workload; the shapes are the LLaDA-8B / Dream-7B shapes
the Fast-dLLM pages evaluate on, with random weights since no trained weights
are available):

* weights ~ N(0, 0.02) drawn tensor by tensor in the fixed order embed, then
  per layer wq, wk, wv, wo, w_gate, w_up, w_down, then lm_head, from one
  ``torch.Generator`` seeded with the workload seed; RMSNorm gains are 1.
  float32 models keep the float32 draw; bfloat16 models round it (RNE).
  Small models draw on the CPU generator.  Multi-billion-parameter models
  draw on a CUDA generator (the CPU generator runs at ~16 M values/s, i.e.
  minutes for 8 B values); the oracle then receives a host copy of exactly
  those tensors.
* prompt ids uniform in [0, vocab - 2] (the last id is the mask id) from a
  CPU generator seeded with 1000 + seed; batched prompt lengths uniform in
  [128, 1024] from a CPU generator seeded with the batch seed.
"""
from __future__ import annotations

from dataclasses import asdict, dataclass, replace
from typing import Dict, List, Optional

import torch


@dataclass(frozen=True)
class ModelShape:
    name: str
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
    dtype: str          # "fp32" or "bf16"
    seed: int

    def as_dict(self) -> dict:
        return asdict(self)

    @property
    def n_params(self) -> int:
        d, hd = self.d_model, self.head_dim
        per_layer = (d * (self.n_heads + 2 * self.n_kv_heads) * hd + self.n_heads * hd * d
                     + 3 * d * self.ffn_dim + 2 * d)
        return 2 * self.vocab * d + self.n_layers * per_layer + d

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "fp32" else 2


TINY = ModelShape("tiny-fp32", 2, 128, 4, 4, 32, 384, 512, 511, 1e4, 1e-5, 8.0, "fp32", 0)
LLADA_8B = ModelShape("llada-8b-shape", 32, 4096, 32, 32, 128, 12288, 126464, 126463,
                      1e4, 1e-5, 30.0, "bf16", 1)
DREAM_7B = ModelShape("dream-7b-shape", 28, 3584, 28, 4, 128, 18944, 152064, 152063,
                      1e6, 1e-6, 30.0, "bf16", 2)
# Reduced bf16 models for parity tests the oracle finishes in seconds.  The
# sizes are chosen to span several GEMM tiles and leave ragged tails (vocab
# and FFN not multiples of 128).
SMALL_BF16 = ModelShape("small-bf16", 2, 512, 4, 4, 128, 1344, 1000, 999, 1e4, 1e-5, 30.0,
                        "bf16", 11)
SMALL_GQA_BF16 = ModelShape("small-gqa-bf16", 2, 512, 8, 2, 64, 1408, 2051, 2050, 1e6, 1e-6,
                            30.0, "bf16", 12)

SHAPES = {s.name: s for s in (TINY, LLADA_8B, DREAM_7B, SMALL_BF16, SMALL_GQA_BF16)}


@dataclass(frozen=True)
class Workload:
    name: str
    shape: ModelShape
    prompt_len: int
    gen_len: int
    block_size: int
    tau: float
    cache_mode: str
    batch: int = 1


WORKLOADS = {
    "tiny": Workload("tiny", TINY, 32, 64, 16, 0.9, "dual"),
    "llada8b-p256-g256": Workload("llada8b-p256-g256", LLADA_8B, 256, 256, 32, 0.9, "dual"),
    "llada8b-p1024-g256": Workload("llada8b-p1024-g256", LLADA_8B, 1024, 256, 32, 0.9, "dual"),
    "llada8b-p1024-g512": Workload("llada8b-p1024-g512", LLADA_8B, 1024, 512, 32, 0.9, "dual"),
    "llada8b-p1024-g1024": Workload("llada8b-p1024-g1024", LLADA_8B, 1024, 1024, 32, 0.9, "dual"),
    "dream7b-p512-g512": Workload("dream7b-p512-g512", DREAM_7B, 512, 512, 32, 0.9, "dual"),
    "llada8b-batch16": Workload("llada8b-batch16", LLADA_8B, 0, 256, 32, 0.9, "dual", batch=16),
    # Two layers of the LLaDA-8B shape (~3 GB of weights): the same GEMM,
    # attention and LM-head shapes per launch, small enough for a full ncu
    # capture of single launches.
    "llada8b-2layer-p256-g32": Workload("llada8b-2layer-p256-g32",
                                        ModelShape("llada-8b-shape-2layer", 2, 4096, 32, 32, 128,
                                                   12288, 126464, 126463, 1e4, 1e-5, 30.0, "bf16",
                                                   1),
                                        256, 32, 32, 0.9, "dual"),
    # The same two layers with the full prompt and generation lengths (L = 512):
    # the refresh-step GEMM and attention shapes of the LLaDA-8B workload.
    "llada8b-2layer-p256-g256": Workload("llada8b-2layer-p256-g256",
                                         ModelShape("llada-8b-shape-2layer", 2, 4096, 32, 32,
                                                    128, 12288, 126464, 126463, 1e4, 1e-5, 30.0,
                                                    "bf16", 1),
                                         256, 256, 32, 0.9, "dual"),
    # The batched-serving workload on the 2-layer model (every GEMM, attention
    # and LM-head shape of one global step of the batch-16 workload per layer).
    "llada8b-2layer-batch16": Workload("llada8b-2layer-batch16",
                                       ModelShape("llada-8b-shape-2layer", 2, 4096, 32, 32, 128,
                                                  12288, 126464, 126463, 1e4, 1e-5, 30.0,
                                                  "bf16", 1),
                                       0, 256, 32, 0.9, "dual", batch=16),
}


def step_weight_params(shape: ModelShape) -> int:
    """Weights a DualCache block step reads: every layer's QKV, O, gate, up
    and down matrices and the LM head (the embedding only for the block's
    rows, negligible)."""
    d, hd = shape.d_model, shape.head_dim
    per_layer = (d * (shape.n_heads + 2 * shape.n_kv_heads) * hd + shape.n_heads * hd * d
                 + 3 * d * shape.ffn_dim)
    return shape.n_layers * per_layer + shape.vocab * d


def weight_names(shape: ModelShape) -> List[str]:
    names = ["embed"]
    for i in range(shape.n_layers):
        p = f"layers.{i}."
        names += [p + n for n in ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm",
                                  "w_gate", "w_up", "w_down")]
    names += ["final_norm", "lm_head"]
    return names


def weight_shapes(shape: ModelShape) -> Dict[str, tuple]:
    d, hd, f, v = shape.d_model, shape.head_dim, shape.ffn_dim, shape.vocab
    out = {"embed": (v, d), "final_norm": (d,), "lm_head": (v, d)}
    for i in range(shape.n_layers):
        p = f"layers.{i}."
        out.update({
            p + "attn_norm": (d,), p + "ffn_norm": (d,),
            p + "wq": (shape.n_heads * hd, d), p + "wk": (shape.n_kv_heads * hd, d),
            p + "wv": (shape.n_kv_heads * hd, d), p + "wo": (d, shape.n_heads * hd),
            p + "w_gate": (f, d), p + "w_up": (f, d), p + "w_down": (d, f),
        })
    return out


def _draw_order(shape: ModelShape) -> List[str]:
    order = ["embed"]
    for i in range(shape.n_layers):
        p = f"layers.{i}."
        order += [p + n for n in ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down")]
    return order + ["lm_head"]


def default_device(shape: ModelShape) -> str:
    return "cuda" if shape.n_params > 200_000_000 else "cpu"


def make_weights(shape: ModelShape, device: Optional[str] = None, std: float = 0.02
                 ) -> Dict[str, torch.Tensor]:
    """Random weights for ``shape`` (see the module docstring for the recipe)."""
    device = device or default_device(shape)
    gen = torch.Generator(device=device).manual_seed(shape.seed)
    dt = torch.float32 if shape.dtype == "fp32" else torch.bfloat16
    shapes = weight_shapes(shape)
    out: Dict[str, torch.Tensor] = {}
    for name in _draw_order(shape):
        w = torch.empty(shapes[name], dtype=torch.float32, device=device)
        w.normal_(0.0, std, generator=gen)
        out[name] = w if dt == torch.float32 else w.to(dt)
        del w
    for name, shp in shapes.items():
        if name.endswith("norm"):
            out[name] = torch.ones(shp, dtype=dt, device=device)
    return {n: out[n] for n in weight_names(shape)}


def make_prompt(shape: ModelShape, length: int, salt: int = 0) -> torch.Tensor:
    """int32 prompt ids uniform in [0, vocab - 2] (never the mask id)."""
    gen = torch.Generator().manual_seed(1000 + shape.seed + salt)
    return torch.randint(0, shape.vocab - 1, (length,), generator=gen, dtype=torch.int64).to(
        torch.int32)


def make_batch_prompt_lengths(batch: int, seed: int = 3, lo: int = 128, hi: int = 1024) -> List[int]:
    gen = torch.Generator().manual_seed(seed)
    return [int(v) for v in torch.randint(lo, hi + 1, (batch,), generator=gen)]


def with_layers(shape: ModelShape, n_layers: int) -> ModelShape:
    """Same shape with fewer layers (used only where a test says so)."""
    return replace(shape, n_layers=n_layers, name=f"{shape.name}-{n_layers}l")
