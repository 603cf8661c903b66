"""ctypes binding of ``libfdllm.so`` (argument marshalling only).

The module-level functions carry the C names (``fdllm_create``,
``fdllm_load_weights``, ``fdllm_generate``, ...) and take Python / torch /
numpy arguments; every step of the decode runs inside the library's CUDA
kernels.  ``Decoder`` is a small convenience wrapper around one context.

PyTorch is used only for device memory: by default the context's device
buffers come from torch's caching allocator through the C allocator hook.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Dict, Mapping, Optional

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
# FDLLM_CHECKS=1 selects the self-checking build (bounds-checked device accesses).
LIB_PATH = os.path.join(HERE, "libfdllm_checks.so" if os.environ.get("FDLLM_CHECKS") == "1"
                        else "libfdllm.so")

FDLLM_OK, FDLLM_ERR_ARG, FDLLM_ERR_OOM, FDLLM_ERR_CUDA = 0, -1, -2, -3
FDLLM_ERR_STATE, FDLLM_ERR_TIMEOUT, FDLLM_ERR_SHAPE = -4, -5, -6
CACHE_MODES = {"none": 0, "prefix": 1, "dual": 2}
DTYPES = {"fp32": 0, "bf16": 1}

EXPORTED = ("fdllm_create", "fdllm_load_weights", "fdllm_generate", "fdllm_generate_device",
            "fdllm_generate_batch", "fdllm_generate_fixed_k",
            "fdllm_step_debug", "fdllm_read_kv", "fdllm_kv_similarity", "fdllm_selftest_wait_timeout",
            "fdllm_gemm", "fdllm_gemm_f16", "fdllm_attention",
            "fdllm_gemm_noalloc", "fdllm_profile_enable", "fdllm_profile_read",
            "fdllm_last_error", "fdllm_launch_count", "fdllm_inexact_weight_count",
            "fdllm_destroy")


class FdllmConfig(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("d_model", ctypes.c_int32),
                ("n_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("ffn_dim", ctypes.c_int32),
                ("vocab", ctypes.c_int32), ("mask_id", ctypes.c_int32),
                ("rope_theta", ctypes.c_float), ("rms_eps", ctypes.c_float),
                ("logit_scale", ctypes.c_float), ("dtype", ctypes.c_int32),
                ("max_batch", ctypes.c_int32), ("max_seq", ctypes.c_int32)]


class FdllmTensor(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("data", ctypes.c_void_p), ("numel", ctypes.c_int64),
                ("on_device", ctypes.c_int32), ("dtype", ctypes.c_int32)]


ALLOC_FN = ctypes.CFUNCTYPE(ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p)
FREE_FN = ctypes.CFUNCTYPE(None, ctypes.c_void_p, ctypes.c_void_p)


class FdllmAllocator(ctypes.Structure):
    _fields_ = [("alloc", ALLOC_FN), ("free", FREE_FN), ("user", ctypes.c_void_p)]


class FdllmStats(ctypes.Structure):
    _fields_ = [("steps", ctypes.c_int32), ("refresh_steps", ctypes.c_int32),
                ("cached_steps", ctypes.c_int32), ("n_blocks", ctypes.c_int32),
                ("steps_per_block", ctypes.POINTER(ctypes.c_int32)),
                ("collect_timing", ctypes.c_int32), ("refresh_ms", ctypes.c_double),
                ("cached_ms", ctypes.c_double), ("trace_cap", ctypes.c_int32),
                ("trace_block", ctypes.POINTER(ctypes.c_int32)),
                ("trace_conf", ctypes.POINTER(ctypes.c_float)),
                ("trace_tok", ctypes.POINTER(ctypes.c_int32)),
                ("trace_unmask", ctypes.POINTER(ctypes.c_uint8))]


class FdllmKernelStat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("launches", ctypes.c_int64),
                ("total_ms", ctypes.c_double), ("bytes", ctypes.c_double),
                ("flops", ctypes.c_double)]


class FdllmError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"fdllm error {code}: {msg}")
        self.code = code


_lib: Optional[ctypes.CDLL] = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libfdllm.so.  Raises (never falls back) when it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m kv_cache_decode_dualcache_b200.build` "
            "(the decoder has no CPU fallback)")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER
    vp, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.fdllm_create.argtypes = [P(FdllmConfig), i32, vp, P(FdllmAllocator), P(vp)]
    lib.fdllm_load_weights.argtypes = [vp, P(FdllmTensor), i32]
    lib.fdllm_generate.argtypes = [vp, P(ctypes.c_int32), i32, i32, i32, f32, i32,
                                   P(ctypes.c_int32), P(i32), P(FdllmStats)]
    lib.fdllm_generate_device.argtypes = [vp, vp, i32, i32, i32, f32, i32, vp, P(i32),
                                          P(FdllmStats)]
    lib.fdllm_generate_fixed_k.argtypes = [vp, P(ctypes.c_int32), i32, i32, i32, i32, i32,
                                           P(ctypes.c_int32), P(i32), P(FdllmStats)]
    lib.fdllm_generate_batch.argtypes = [vp, i32, P(P(ctypes.c_int32)), P(i32), i32, i32, f32,
                                         i32, P(ctypes.c_int32), P(i32), P(FdllmStats)]
    lib.fdllm_step_debug.argtypes = [vp, P(ctypes.c_int32), P(ctypes.c_int32), i32, i32, i32, f32,
                                     i32, P(ctypes.c_float), P(ctypes.c_float),
                                     P(ctypes.c_int32), P(ctypes.c_uint8)]
    lib.fdllm_read_kv.argtypes = [vp, i32, i32, i32, P(ctypes.c_float), P(ctypes.c_float)]
    lib.fdllm_kv_similarity.argtypes = [vp, P(ctypes.c_int32), P(ctypes.c_int32), i32,
                                        P(ctypes.c_double)]
    lib.fdllm_selftest_wait_timeout.argtypes = [vp]
    lib.fdllm_gemm.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32]
    lib.fdllm_gemm_f16.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32]
    lib.fdllm_attention.argtypes = [vp, vp, vp, i32, i32, i32]
    lib.fdllm_gemm_noalloc.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp]
    lib.fdllm_profile_enable.argtypes = [vp, i32]
    lib.fdllm_profile_read.argtypes = [vp, P(FdllmKernelStat), i32, P(i32)]
    lib.fdllm_last_error.argtypes = [vp]
    lib.fdllm_last_error.restype = ctypes.c_char_p
    lib.fdllm_launch_count.argtypes = [vp, i32]
    lib.fdllm_launch_count.restype = ctypes.c_int64
    lib.fdllm_inexact_weight_count.argtypes = [vp]
    lib.fdllm_inexact_weight_count.restype = ctypes.c_int64
    lib.fdllm_destroy.argtypes = [vp]
    for name in ("fdllm_create", "fdllm_load_weights", "fdllm_generate", "fdllm_generate_device",
                 "fdllm_generate_batch", "fdllm_generate_fixed_k", "fdllm_step_debug", "fdllm_read_kv",
                 "fdllm_kv_similarity", "fdllm_selftest_wait_timeout", "fdllm_gemm",
                 "fdllm_gemm_f16", "fdllm_attention", "fdllm_gemm_noalloc",
                 "fdllm_profile_enable", "fdllm_profile_read", "fdllm_destroy"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def _check(code: int, ctx) -> None:
    if code != FDLLM_OK:
        msg = load_library().fdllm_last_error(ctx).decode(errors="replace")
        raise FdllmError(code, msg)


def _i32_ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def make_config(shape, max_seq: int, max_batch: int = 1) -> FdllmConfig:
    s = shape.as_dict() if hasattr(shape, "as_dict") else dict(shape)
    return FdllmConfig(s["n_layers"], s["d_model"], s["n_heads"], s["n_kv_heads"], s["head_dim"],
                       s["ffn_dim"], s["vocab"], s["mask_id"], s["rope_theta"], s["rms_eps"],
                       s["logit_scale"], DTYPES[s["dtype"]], int(max_batch), max_seq)


class TorchAllocator:
    """Hands torch caching-allocator blocks to the library (device memory
    plumbing only)."""

    def __init__(self, device: int):
        import torch
        self._torch = torch
        self.device = device
        self.blocks: Dict[int, object] = {}
        self.c_alloc = ALLOC_FN(self._alloc)
        self.c_free = FREE_FN(self._free)
        self.struct = FdllmAllocator(self.c_alloc, self.c_free, None)

    def _alloc(self, nbytes, _user):
        try:
            t = self._torch.empty(int(nbytes), dtype=self._torch.uint8,
                                  device=f"cuda:{self.device}")
        except Exception:  # out of memory: report NULL to the library
            return None
        ptr = t.data_ptr()
        self.blocks[ptr] = t
        return ptr

    def _free(self, ptr, _user):
        self.blocks.pop(int(ptr), None)


# ------------------------------------------------------------------ C names
def fdllm_create(shape, max_seq: int, device: int = 0, stream=None, allocator=None,
                 max_batch: int = 1):
    lib = load_library()
    cfg = make_config(shape, max_seq, max_batch)
    ctx = ctypes.c_void_p()
    alloc_ptr = ctypes.byref(allocator.struct) if allocator is not None else None
    stream_ptr = ctypes.c_void_p(stream) if stream else None
    _check(lib.fdllm_create(ctypes.byref(cfg), device, stream_ptr, alloc_ptr, ctypes.byref(ctx)),
           None)
    return ctx


def fdllm_load_weights(ctx, weights: Mapping[str, object], dtype: str) -> None:
    """``weights``: name -> torch tensor (CPU or CUDA) or numpy array, contiguous."""
    lib = load_library()
    keep = []
    arr = (FdllmTensor * len(weights))()
    for i, (name, w) in enumerate(weights.items()):
        if hasattr(w, "data_ptr"):
            w = w.contiguous()
            ptr, numel, on_dev = w.data_ptr(), w.numel(), int(w.is_cuda)
        else:
            w = np.ascontiguousarray(w)
            ptr, numel, on_dev = w.ctypes.data, w.size, 0
        keep.append(w)
        arr[i] = FdllmTensor(name.encode(), ptr, numel, on_dev, DTYPES[dtype])
    _check(lib.fdllm_load_weights(ctx, arr, len(weights)), ctx)
    del keep


def fdllm_generate(ctx, prompt, gen_len: int, block_size: int, tau: float, cache_mode,
                   stats: Optional[FdllmStats] = None):
    lib = load_library()
    p = np.ascontiguousarray(np.asarray(prompt, dtype=np.int32))
    out = np.empty(gen_len, dtype=np.int32)
    steps = ctypes.c_int()
    mode = CACHE_MODES[cache_mode] if isinstance(cache_mode, str) else int(cache_mode)
    _check(lib.fdllm_generate(ctx, _i32_ptr(p), int(p.size), gen_len, block_size, float(tau), mode,
                              _i32_ptr(out), ctypes.byref(steps),
                              ctypes.byref(stats) if stats is not None else None), ctx)
    return out, steps.value


def fdllm_generate_fixed_k(ctx, prompt, gen_len: int, block_size: int, k: int, cache_mode,
                           stats: Optional[FdllmStats] = None):
    lib = load_library()
    p = np.ascontiguousarray(np.asarray(prompt, dtype=np.int32))
    out = np.empty(gen_len, dtype=np.int32)
    steps = ctypes.c_int()
    mode = CACHE_MODES[cache_mode] if isinstance(cache_mode, str) else int(cache_mode)
    _check(lib.fdllm_generate_fixed_k(ctx, _i32_ptr(p), int(p.size), gen_len, block_size, int(k),
                                      mode, _i32_ptr(out), ctypes.byref(steps),
                                      ctypes.byref(stats) if stats is not None else None), ctx)
    return out, steps.value


def fdllm_generate_batch(ctx, prompts, gen_len: int, block_size: int, tau: float, cache_mode,
                         stats: Optional[FdllmStats] = None):
    """prompts: a list of 1-D id arrays (any lengths).  Returns (tokens
    [batch, gen_len] int32, steps [batch] int32)."""
    lib = load_library()
    ps = [np.ascontiguousarray(np.asarray(p, dtype=np.int32)) for p in prompts]
    n = len(ps)
    ptrs = (ctypes.POINTER(ctypes.c_int32) * max(1, n))(*[_i32_ptr(p) for p in ps])
    lens = (ctypes.c_int * max(1, n))(*[int(p.size) for p in ps])
    out = np.empty((n, gen_len), dtype=np.int32)
    steps = np.empty(n, dtype=np.int32)
    mode = CACHE_MODES[cache_mode] if isinstance(cache_mode, str) else int(cache_mode)
    _check(lib.fdllm_generate_batch(ctx, n, ptrs, lens, gen_len, block_size, float(tau), mode,
                                    _i32_ptr(out), steps.ctypes.data_as(ctypes.POINTER(ctypes.c_int)),
                                    ctypes.byref(stats) if stats is not None else None), ctx)
    return out, steps


def fdllm_generate_device(ctx, prompt_dev, gen_len: int, block_size: int, tau: float, cache_mode,
                          out_dev, stats: Optional[FdllmStats] = None) -> int:
    """``prompt_dev`` / ``out_dev``: contiguous int32 CUDA tensors."""
    lib = load_library()
    steps = ctypes.c_int()
    mode = CACHE_MODES[cache_mode] if isinstance(cache_mode, str) else int(cache_mode)
    _check(lib.fdllm_generate_device(ctx, prompt_dev.data_ptr(), int(prompt_dev.numel()), gen_len,
                                     block_size, float(tau), mode, out_dev.data_ptr(),
                                     ctypes.byref(steps),
                                     ctypes.byref(stats) if stats is not None else None), ctx)
    return steps.value


def fdllm_step_debug(ctx, snapshot_ids, current_ids, block_start: int, block_size: int,
                     tau: float, cache_mode, vocab: Optional[int] = None):
    lib = load_library()
    snap = np.ascontiguousarray(np.asarray(snapshot_ids, dtype=np.int32))
    cur = np.ascontiguousarray(np.asarray(current_ids, dtype=np.int32))
    B = block_size
    conf = np.empty(B, dtype=np.float32)
    tok = np.empty(B, dtype=np.int32)
    unmask = np.empty(B, dtype=np.uint8)
    logits = np.empty((B, vocab), dtype=np.float32) if vocab else None
    mode = CACHE_MODES[cache_mode] if isinstance(cache_mode, str) else int(cache_mode)
    _check(lib.fdllm_step_debug(
        ctx, _i32_ptr(snap), _i32_ptr(cur), int(snap.size), block_start, B, float(tau), mode,
        logits.ctypes.data_as(ctypes.POINTER(ctypes.c_float)) if logits is not None else None,
        conf.ctypes.data_as(ctypes.POINTER(ctypes.c_float)), _i32_ptr(tok),
        unmask.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))), ctx)
    return {"z": logits, "conf": conf, "tok": tok, "unmask": unmask.astype(bool)}


def fdllm_read_kv(ctx, layer: int, pos0: int, n: int, n_kv_heads: int, head_dim: int):
    lib = load_library()
    k = np.empty((n, n_kv_heads, head_dim), dtype=np.float32)
    v = np.empty_like(k)
    _check(lib.fdllm_read_kv(ctx, layer, pos0, n,
                             k.ctypes.data_as(ctypes.POINTER(ctypes.c_float)),
                             v.ctypes.data_as(ctypes.POINTER(ctypes.c_float))), ctx)
    return k, v


def fdllm_kv_similarity(ctx, ids_a, ids_b, n_layers: int):
    """Cosines [n_layers, 2 (K, V), L] of the two sequences' K/V activations
    (full forward over each; see the header)."""
    lib = load_library()
    a = np.ascontiguousarray(np.asarray(ids_a, dtype=np.int32))
    b = np.ascontiguousarray(np.asarray(ids_b, dtype=np.int32))
    if a.shape != b.shape or a.ndim != 1:
        raise ValueError("ids_a and ids_b must be 1-D sequences of the same length")
    out = np.empty((n_layers, 2, a.size), dtype=np.float64)
    _check(lib.fdllm_kv_similarity(ctx, _i32_ptr(a), _i32_ptr(b), int(a.size),
                                   out.ctypes.data_as(ctypes.POINTER(ctypes.c_double))), ctx)
    return out


def _pair_rows(m: int) -> int:
    return 2 * ((m + 31) // 32) * 32


def fdllm_gemm(ctx, w_dev, x_dev, y_dev, splits: int = 0, accumulate: bool = False) -> None:
    """y_dev[M, N] (float32 CUDA tensor) = x @ w_dev[N, K]^T (+= when accumulate).

    M is y_dev's row count.  x_dev is [M, K] float32 (fp32 model) or the
    two-term bf16 pair-row layout with 2*ceil(M/32)*32 rows (bf16 model)."""
    N, K = w_dev.shape
    M = int(y_dev.shape[0])
    if tuple(y_dev.shape) != (M, N) or not y_dev.is_contiguous():
        raise ValueError("y_dev must be a contiguous [M, N] tensor")
    need = _pair_rows(M) if x_dev.element_size() == 2 else M
    if x_dev.shape[0] < need or x_dev.shape[1] != K or not x_dev.is_contiguous():
        raise ValueError(f"x_dev must be a contiguous [{need}, {K}] tensor")
    _check(load_library().fdllm_gemm(ctx, w_dev.data_ptr(), x_dev.data_ptr(), y_dev.data_ptr(), N,
                                     M, K, splits, int(accumulate)), ctx)


def fdllm_gemm_f16(ctx, w_dev, x_dev, y_dev, splits: int = 0, accumulate: bool = False) -> None:
    """fdllm_gemm with fp16 operands (bf16 model): w_dev [N, K] float16, x_dev
    the two-term float16 pair rows [2*ceil(M/32)*32, K]; y_dev [M, N] float32."""
    N, K = w_dev.shape
    M = int(y_dev.shape[0])
    if tuple(y_dev.shape) != (M, N) or not y_dev.is_contiguous():
        raise ValueError("y_dev must be a contiguous [M, N] tensor")
    need = _pair_rows(M)
    if x_dev.shape[0] < need or x_dev.shape[1] != K or not x_dev.is_contiguous():
        raise ValueError(f"x_dev must be a contiguous [{need}, {K}] tensor")
    _check(load_library().fdllm_gemm_f16(ctx, w_dev.data_ptr(), x_dev.data_ptr(), y_dev.data_ptr(),
                                         N, M, K, splits, int(accumulate)), ctx)


def fdllm_gemm_noalloc(w_dev, x_dev, y_dev, splits: int = 0, stream=None) -> None:
    """Allocation-free variant of fdllm_gemm (bf16 model only; no ctx): same
    operands and layouts, scratch from the library's fixed device array.
    Runs on the current device and the given stream handle (None = legacy
    default stream)."""
    N, K = w_dev.shape
    M = int(y_dev.shape[0])
    if tuple(y_dev.shape) != (M, N) or not y_dev.is_contiguous():
        raise ValueError("y_dev must be a contiguous [M, N] tensor")
    need = _pair_rows(M)
    if x_dev.shape[0] < need or x_dev.shape[1] != K or not x_dev.is_contiguous():
        raise ValueError(f"x_dev must be a contiguous [{need}, {K}] tensor")
    _check(load_library().fdllm_gemm_noalloc(w_dev.data_ptr(), x_dev.data_ptr(),
                                             y_dev.data_ptr(), N, M, K, splits,
                                             ctypes.c_void_p(stream) if stream else None), None)


def fdllm_attention(ctx, q_dev, o_dev, layer: int, L: int) -> None:
    """Attention of M queries over cached keys [0, L) of ``layer``.

    fp32 model: q_dev [M, H, hd], o_dev [M, H*hd] float32.  bf16 model:
    q_dev [2, M, H, hd] fp16 (hi plane, lo plane), o_dev two-term fp16 pair
    rows [2*ceil(M/32)*32, H*hd]."""
    two_term = q_dev.dim() == 4
    M = int(q_dev.shape[1] if two_term else q_dev.shape[0])
    need = _pair_rows(M) if two_term else M
    if o_dev.shape[0] < need or not (q_dev.is_contiguous() and o_dev.is_contiguous()):
        raise ValueError(f"o_dev needs {need} contiguous rows")
    _check(load_library().fdllm_attention(ctx, q_dev.data_ptr(), o_dev.data_ptr(), layer, M, L),
           ctx)


def fdllm_profile_enable(ctx, enable: bool = True) -> None:
    _check(load_library().fdllm_profile_enable(ctx, int(enable)), ctx)


def fdllm_profile_read(ctx, max_stats: int = 64):
    """List of dicts {name, launches, total_ms, bytes, flops} per kernel class."""
    arr = (FdllmKernelStat * max_stats)()
    n = ctypes.c_int()
    _check(load_library().fdllm_profile_read(ctx, arr, max_stats, ctypes.byref(n)), ctx)
    return [{"name": arr[i].name.decode(), "launches": int(arr[i].launches),
             "total_ms": float(arr[i].total_ms), "bytes": float(arr[i].bytes),
             "flops": float(arr[i].flops)} for i in range(min(n.value, max_stats))]


def fdllm_last_error(ctx=None) -> str:
    return load_library().fdllm_last_error(ctx).decode(errors="replace")


def fdllm_launch_count(ctx, reset: bool = False) -> int:
    return int(load_library().fdllm_launch_count(ctx, int(reset)))


def fdllm_destroy(ctx) -> None:
    if ctx:
        _check(load_library().fdllm_destroy(ctx), None)


# ------------------------------------------------------------------ wrapper
@dataclass
class GenerateStats:
    steps: int
    refresh_steps: int
    cached_steps: int
    steps_per_block: list
    refresh_ms: float
    cached_ms: float
    # per-step trace (generate(..., trace=True)): block index [steps] and, per
    # step, the block rows' confidence / argmax / unmask flag [steps, block]
    trace_block: Optional[np.ndarray] = None
    trace_conf: Optional[np.ndarray] = None
    trace_tok: Optional[np.ndarray] = None
    trace_unmask: Optional[np.ndarray] = None


def fdllm_inexact_weight_count(ctx) -> int:
    return int(load_library().fdllm_inexact_weight_count(ctx))


class Decoder:
    """One decoder context (convenience wrapper over the C calls)."""

    def __init__(self, shape, max_seq: int, device: int = 0, stream=None, torch_alloc: bool = True,
                 max_batch: int = 1):
        self.shape = shape
        self.max_seq = max_seq
        self.max_batch = max_batch
        self.device = device
        self.allocator = TorchAllocator(device) if torch_alloc else None
        self.ctx = fdllm_create(shape, max_seq, device, stream, self.allocator, max_batch)

    def load_weights(self, weights: Mapping[str, object]) -> None:
        fdllm_load_weights(self.ctx, weights, self.shape.dtype)

    def generate(self, prompt, gen_len: int, block_size: int, tau: float, cache_mode="dual",
                 timing: bool = False, fixed_k: Optional[int] = None, trace: bool = False):
        """Threshold decoding (tau), or with fixed_k the fixed-count strategy.
        With trace, the returned stats carry every step's block index and the
        block rows' confidence, argmax token and unmask flag."""
        n_blocks = gen_len // block_size if block_size > 0 else 0
        spb = (ctypes.c_int32 * max(1, n_blocks))()
        st = FdllmStats(0, 0, 0, 0, ctypes.cast(spb, ctypes.POINTER(ctypes.c_int32)), int(timing),
                        0.0, 0.0)
        if trace:
            cap = max(1, gen_len)                      # every step unmasks >= 1 token
            tb = np.zeros(cap, np.int32)
            tc = np.zeros((cap, block_size), np.float32)
            tt = np.zeros((cap, block_size), np.int32)
            tu = np.zeros((cap, block_size), np.uint8)
            st.trace_cap = cap
            st.trace_block = _i32_ptr(tb)
            st.trace_conf = tc.ctypes.data_as(ctypes.POINTER(ctypes.c_float))
            st.trace_tok = _i32_ptr(tt)
            st.trace_unmask = tu.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))
        if fixed_k is not None:
            out, steps = fdllm_generate_fixed_k(self.ctx, prompt, gen_len, block_size, fixed_k,
                                                cache_mode, st)
        else:
            out, steps = fdllm_generate(self.ctx, prompt, gen_len, block_size, tau, cache_mode, st)
        gs = GenerateStats(st.steps, st.refresh_steps, st.cached_steps, list(spb)[:n_blocks],
                           st.refresh_ms, st.cached_ms)
        if trace:
            n = min(steps, cap)
            gs.trace_block, gs.trace_conf = tb[:n].copy(), tc[:n].copy()
            gs.trace_tok, gs.trace_unmask = tt[:n].copy(), tu[:n].astype(bool)
        return out, steps, gs

    def inexact_weight_count(self) -> int:
        return fdllm_inexact_weight_count(self.ctx)

    def generate_batch(self, prompts, gen_len: int, block_size: int, tau: float,
                       cache_mode="dual", timing: bool = False, trace: bool = False):
        """Variable-length batch: returns (tokens [batch, gen_len], steps [batch],
        GenerateStats of the totals, steps_per_block sequence by sequence).
        With trace, the stats carry per-sequence traces: trace_block[i] [steps_i],
        trace_conf[i] / trace_tok[i] / trace_unmask[i] [steps_i, block]."""
        n = len(prompts)
        n_blocks = gen_len // block_size if block_size > 0 else 0
        spb = (ctypes.c_int32 * max(1, n_blocks * n))()
        st = FdllmStats(0, 0, 0, 0, ctypes.cast(spb, ctypes.POINTER(ctypes.c_int32)), int(timing),
                        0.0, 0.0)
        if trace:
            cap = max(1, gen_len)
            tb = np.zeros((n, cap), np.int32)
            tc = np.zeros((n, cap, block_size), np.float32)
            tt = np.zeros((n, cap, block_size), np.int32)
            tu = np.zeros((n, cap, block_size), np.uint8)
            st.trace_cap = cap
            st.trace_block = _i32_ptr(tb)
            st.trace_conf = tc.ctypes.data_as(ctypes.POINTER(ctypes.c_float))
            st.trace_tok = _i32_ptr(tt)
            st.trace_unmask = tu.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))
        out, steps = fdllm_generate_batch(self.ctx, prompts, gen_len, block_size, tau, cache_mode,
                                          st)
        gs = GenerateStats(st.steps, st.refresh_steps, st.cached_steps,
                           list(spb)[:n_blocks * n], st.refresh_ms, st.cached_ms)
        if trace:
            k = [min(int(v), cap) for v in steps]
            gs.trace_block = [tb[i, :k[i]].copy() for i in range(n)]
            gs.trace_conf = [tc[i, :k[i]].copy() for i in range(n)]
            gs.trace_tok = [tt[i, :k[i]].copy() for i in range(n)]
            gs.trace_unmask = [tu[i, :k[i]].astype(bool) for i in range(n)]
        return out, steps, gs

    def generate_device(self, prompt_dev, gen_len: int, block_size: int, tau: float, out_dev,
                        cache_mode="dual") -> int:
        return fdllm_generate_device(self.ctx, prompt_dev, gen_len, block_size, tau, cache_mode,
                                     out_dev)

    def step_debug(self, snapshot_ids, current_ids, block_start: int, block_size: int,
                   tau: float, cache_mode="dual", logits: bool = True):
        return fdllm_step_debug(self.ctx, snapshot_ids, current_ids, block_start, block_size, tau,
                                cache_mode, self.shape.vocab if logits else None)

    def kv_similarity(self, ids_a, ids_b):
        return fdllm_kv_similarity(self.ctx, ids_a, ids_b, self.shape.n_layers)

    def read_kv(self, layer: int, pos0: int, n: int):
        return fdllm_read_kv(self.ctx, layer, pos0, n, self.shape.n_kv_heads, self.shape.head_dim)

    def launch_count(self, reset: bool = False) -> int:
        return fdllm_launch_count(self.ctx, reset)

    def close(self) -> None:
        if self.ctx:
            fdllm_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
