/*
 * fdllm.h - C ABI of the B200 (sm_100a) Fast-dLLM block-wise DualCache decoder.
 *
 * What the library computes (sources: the techwalker.com article
 * "Fast-dLLM：NVIDIA研究团队通过KV缓存和并行解码实现扩散大语言模型的无训练加速",
 * sections "核心创新：适合扩散模型的KV缓存" and "解决并行解码的质量下降问题";
 * the ccyt168.com Fast-dLLM overview, section 一 "核心技术", items 1 and 2):
 *
 *   A masked-diffusion LLM (LLaDA / Dream shape: bidirectional transformer,
 *   RMSNorm, RoPE, MHA or GQA, SwiGLU, untied scaled LM head) generates
 *   gen_len tokens after a prompt.  All generated positions start as the mask
 *   id.  Generation proceeds block by block, left to right.  Each block
 *   starts with a full forward over the whole sequence that refreshes the
 *   K/V cache of every layer and every position (prefix = prompt + finished
 *   blocks, block, suffix = masked future blocks).  That forward's logits
 *   for the block rows make the block's first step.  Later steps of the
 *   block (DualCache) recompute only the block rows: QKV for the block,
 *   attention of the block queries over cached prefix K/V + fresh block K/V
 *   + cached suffix K/V (no causal mask), O-projection, FFN, LM head.  Per
 *   masked block position the LM head yields the argmax token and its
 *   softmax probability (the confidence), with the mask id excluded.  Every
 *   masked position with confidence >= tau is unmasked; if none passes, the
 *   single most confident one is (lowest position on ties).
 *
 *   cache_mode NONE runs the full forward on every step; PREFIX recomputes
 *   rows [s, L) over the cached prefix [0, s); DUAL is the method above.
 *
 * Conventions for every entry point:
 *   - The return value is an fdllm_status; nothing throws or aborts.  On an
 *     error, fdllm_last_error(ctx) returns a message that stays valid until
 *     the next call on that ctx.
 *   - "host" pointers belong to the caller and are read or written only
 *     during the call.  "device" pointers are CUDA device addresses on the
 *     ctx's device; the caller keeps ownership.
 *   - Calls are synchronous: when a call returns, its work on the ctx's
 *     stream has completed (or failed).  A ctx is not thread-safe; use one
 *     ctx per host thread.
 *   - Token ids are int32 in [0, vocab).  The prompt must not contain the
 *     mask id.
 */
#ifndef FDLLM_H
#define FDLLM_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FDLLM_API __attribute__((visibility("default")))
#else
#define FDLLM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct fdllm_ctx fdllm_ctx;

typedef enum {
  FDLLM_OK = 0,
  FDLLM_ERR_ARG = -1,      /* invalid argument (see each call) */
  FDLLM_ERR_OOM = -2,      /* device allocation failed */
  FDLLM_ERR_CUDA = -3,     /* a CUDA runtime/driver call failed */
  FDLLM_ERR_STATE = -4,    /* call made in the wrong state (e.g. no weights) */
  FDLLM_ERR_TIMEOUT = -5,  /* a device-side bounded wait ran out; results invalid */
  FDLLM_ERR_SHAPE = -6     /* weight tensor name/shape/dtype mismatch */
} fdllm_status;

typedef enum {
  FDLLM_CACHE_NONE = 0,
  FDLLM_CACHE_PREFIX = 1,
  FDLLM_CACHE_DUAL = 2
} fdllm_cache_mode;

typedef enum {
  FDLLM_DTYPE_F32 = 0,     /* float32 weights and activations, CUDA cores */
  FDLLM_DTYPE_BF16 = 1     /* bfloat16 weights, run on tensor cores: the GEMM weights
                              are held as fp16 on the device (exact for every bf16
                              value of magnitude in [2^-17, 65504]); activations, q,
                              the K/V cache and the softmax weights stored as two fp16
                              terms (hi + lo, ~22 significant bits); float32
                              accumulation and residual stream */
} fdllm_dtype;

/* Model shape and numerics.  Requirements (FDLLM_ERR_ARG otherwise):
 * n_layers >= 1; d_model a multiple of 64 in [64, 8192]; ffn_dim and
 * n_heads*head_dim multiples of 64; head_dim in {32, 64, 128} (bf16: 64 or
 * 128, and n_kv_heads*head_dim a multiple of 64); n_heads a multiple of
 * n_kv_heads; 0 <= mask_id < vocab; vocab >= 2; 1 <= max_seq <= 2^20;
 * 1 <= max_batch <= 64; rope_theta finite and > 0, rms_eps >= 0,
 * logit_scale finite. */
typedef struct {
  int32_t n_layers;
  int32_t d_model;
  int32_t n_heads;
  int32_t n_kv_heads;
  int32_t head_dim;
  int32_t ffn_dim;
  int32_t vocab;
  int32_t mask_id;
  float rope_theta;    /* RoPE base; rotate-half pairs (i, i + head_dim/2) */
  float rms_eps;       /* RMSNorm: h / sqrt(mean(h^2) + eps) * g */
  float logit_scale;   /* z = logit_scale * (RMSNorm(h) W_head^T) */
  int32_t dtype;       /* fdllm_dtype */
  int32_t max_batch;   /* sequence slots: sequences fdllm_generate_batch decodes at once
                          (each slot holds a K/V cache of max_seq positions) */
  int32_t max_seq;     /* largest prompt_len + gen_len */
} fdllm_config;

/* One weight tensor for fdllm_load_weights.  Names and shapes ([rows, cols],
 * row-major, y = x W^T convention):
 *   "embed" [vocab, d]  "lm_head" [vocab, d]  "final_norm" [d]
 *   "layers.{i}.attn_norm" [d]        "layers.{i}.ffn_norm" [d]
 *   "layers.{i}.wq" [H*hd, d]         "layers.{i}.wk" [Hkv*hd, d]
 *   "layers.{i}.wv" [Hkv*hd, d]       "layers.{i}.wo" [d, H*hd]
 *   "layers.{i}.w_gate" [F, d]        "layers.{i}.w_up" [F, d]
 *   "layers.{i}.w_down" [d, F]
 * dtype is the config dtype (fdllm_dtype) of the data. */
typedef struct {
  const char* name;
  const void* data;    /* host or device pointer, see on_device */
  int64_t numel;
  int32_t on_device;   /* 1: data is a device pointer on the ctx's device */
  int32_t dtype;       /* fdllm_dtype of data */
} fdllm_tensor;

/* Optional device allocator.  When given to fdllm_create, every device
 * buffer of the ctx is obtained from alloc and returned through free (e.g. a
 * framework's caching allocator).  alloc returns NULL on failure.  The
 * returned memory must be 256-byte aligned. */
typedef struct {
  void* (*alloc)(size_t bytes, void* user);
  void (*free)(void* ptr, void* user);
  void* user;
} fdllm_allocator;

/* Optional statistics filled by fdllm_generate*.  steps_per_block, when not
 * NULL, must hold gen_len / block_size entries (caller-owned). */
typedef struct {
  int32_t steps;            /* total denoising steps */
  int32_t refresh_steps;    /* steps that ran a full forward */
  int32_t cached_steps;     /* steps that ran on cached K/V */
  int32_t n_blocks;
  int32_t* steps_per_block;
  int32_t collect_timing;   /* in: 1 = time each step with CUDA events */
  double refresh_ms;        /* out (timing only): summed time of full-forward steps */
  double cached_ms;         /* out (timing only): summed time of cached steps */
  /* Optional per-step trace (in: caller-owned host arrays, trace_cap > 0 to
   * enable; filled by fdllm_generate, fdllm_generate_device and
   * fdllm_generate_fixed_k, not by fdllm_generate_batch).  For denoising step
   * i < trace_cap of the generation: trace_block[i] = its block index and,
   * for row j < block_size of that block, trace_conf[i * block_size + j] =
   * the confidence, trace_tok[...] = the argmax token and trace_unmask[...]
   * = 1 when the step unmasked the row.  Steps beyond trace_cap are not
   * recorded.  The values are read back after each step from the buffers the
   * step's own kernels wrote, so the trace does not change the launches. */
  int32_t trace_cap;
  int32_t* trace_block;
  float* trace_conf;
  int32_t* trace_tok;
  uint8_t* trace_unmask;
} fdllm_stats;

/* Create a decoder context on CUDA device `device`.  cuda_stream is a
 * cudaStream_t to run on (borrowed; NULL = the ctx creates its own blocking
 * stream, which is ordered after work on the legacy default stream).  alloc
 * may be NULL (cudaMalloc/cudaFree).  Allocates the KV cache for max_seq
 * positions and the activation buffers.  Errors: ARG (bad config), OOM, CUDA. */
FDLLM_API int fdllm_create(const fdllm_config* cfg, int device, void* cuda_stream,
                 const fdllm_allocator* alloc, fdllm_ctx** out);

/* Copy the model weights into ctx-owned device memory in the kernels' layout
 * (Wq/Wk/Wv fused and W_gate/W_up interleaved, rows reordered within 32-row
 * groups so that the rotate-half and gate/up partners meet in one warp; the
 * bf16 model's GEMM weights stored as fp16, exact for |w| >= 2^-17).  Every tensor
 * named above must appear exactly once.  The caller keeps ownership of the
 * inputs.  Errors: SHAPE (unknown/missing/duplicate name, wrong numel or
 * dtype), OOM, CUDA. */
FDLLM_API int fdllm_load_weights(fdllm_ctx* ctx, const fdllm_tensor* tensors, int n_tensors);

/* Number of GEMM weights of the bf16 model whose conversion to fp16 at
 * fdllm_load_weights was not exact (non-zero bf16 values below 2^-17 in
 * magnitude, where the fp16 grid spacing is 2^-24; each such weight is off by
 * at most 2^-25).  0 for the fp32 model or before weights are loaded.
 * Returns -1 for a NULL ctx. */
FDLLM_API int64_t fdllm_inexact_weight_count(const fdllm_ctx* ctx);

/* Generate gen_len tokens after prompt_ids (host, prompt_len ids) with block
 * size block_size, threshold tau and cache mode cache_mode; writes the
 * gen_len generated ids to out_tokens (host) and the number of denoising
 * steps to *out_steps.  tau > 1 decodes one token per step; tau <= 0
 * unmasks a whole block per step.  Errors: ARG (gen_len or block_size < 1,
 * gen_len % block_size != 0, prompt_len < 0, prompt_len + gen_len > max_seq,
 * an id out of range or equal to the mask id in the prompt, NaN tau, unknown
 * cache_mode, NULL outputs), STATE (no weights), CUDA, TIMEOUT.
 * Precondition of the bf16 DualCache block steps: their persistent kernel
 * runs one CTA on every SM and its phases wait on every CTA, so the decoder
 * needs the GPU's SMs to itself while a step runs; if another stream or
 * process holds SMs for longer than the 2 s bound, the step ends with
 * FDLLM_ERR_TIMEOUT (the context stays usable) instead of running slower. */
FDLLM_API int fdllm_generate(fdllm_ctx* ctx, const int32_t* prompt_ids, int prompt_len, int gen_len,
                   int block_size, float tau, int cache_mode, int32_t* out_tokens,
                   int* out_steps, fdllm_stats* stats);

/* Same as fdllm_generate, but prompt_ids and out_tokens are device pointers
 * (no host copies of the ids; the prompt is not range-checked on the host:
 * ids outside [0, vocab) or equal to the mask id give FDLLM_ERR_ARG after
 * the call from a device-side check). */
FDLLM_API int fdllm_generate_device(fdllm_ctx* ctx, const int32_t* prompt_ids_dev, int prompt_len,
                          int gen_len, int block_size, float tau, int cache_mode,
                          int32_t* out_tokens_dev, int* out_steps, fdllm_stats* stats);

/* Fixed-count decoding, the strategy that the confidence threshold replaces
 * (techwalker.com Fast-dLLM article, section "解决并行解码的质量下降问题":
 * earlier methods unmask a fixed number of tokens per step): as
 * fdllm_generate, but every step unmasks the k most confident masked
 * positions of the block (the lower position first among equal
 * confidences; all remaining ones when fewer than k are masked), so a block
 * of B positions takes ceil(B / k) steps.  Errors as fdllm_generate; ARG for
 * k < 1. */
FDLLM_API int fdllm_generate_fixed_k(fdllm_ctx* ctx, const int32_t* prompt_ids, int prompt_len,
                                     int gen_len, int block_size, int k, int cache_mode,
                                     int32_t* out_tokens, int* out_steps, fdllm_stats* stats);

/* Variable-length batch: `batch` independent sequences, prompts[i] (host)
 * holding prompt_lens[i] ids, each generating gen_len tokens with the same
 * block size, tau and cache mode on its own block schedule (its blocks start
 * at its own prompt end; the readings of the block procedure are those of
 * fdllm_generate, per sequence).  out_tokens (host, caller-owned, batch *
 * gen_len) receives sequence i's tokens at [i * gen_len, (i + 1) * gen_len);
 * out_steps (host, batch) its step counts; stats (optional) the totals over
 * the batch (steps = the sequences' denoising steps summed; refresh_steps /
 * cached_steps = the global steps that did / did not hold a full forward of
 * some sequence, refresh_ms / cached_ms their summed times with timing),
 * with steps_per_block (when not NULL) holding batch * gen_len /
 * block_size entries, sequence by sequence, and the trace (when trace_cap >
 * 0) of sequence i's step k at index i * trace_cap + k.
 *
 * With max_batch > 1 the sequences share the weight stream: up to max_batch
 * of them occupy the context's slots at once, and every global step runs ONE
 * forward over the rows all of them need (a full forward for a sequence at a
 * block start, or every step with the cache off; its block rows in a
 * DualCache step; rows [s, L) in a prefix-cache step), with per-row RoPE
 * positions and K/V destinations, attention per sequence over its own cache
 * pages, and the unmask rule per sequence.  A sequence that finishes frees
 * its slot for the next waiting one (continuous batching).  Each sequence's
 * decode is the single-sequence algorithm; its results equal fdllm_generate
 * on it alone up to the rounding of the batched GEMM's reduction order (the
 * fp32 model's kernels sum in a fixed order per output, so there they are
 * identical).  With max_batch == 1 the sequences run one after another
 * through the single-sequence path.  Every sequence's arguments are checked
 * before any work (errors as fdllm_generate; ARG for batch < 1 or NULL
 * arrays). */
FDLLM_API int fdllm_generate_batch(fdllm_ctx* ctx, int batch, const int32_t* const* prompts,
                                   const int* prompt_lens, int gen_len, int block_size, float tau,
                                   int cache_mode, int32_t* out_tokens, int* out_steps,
                                   fdllm_stats* stats);

/* Teacher-forced single step (parity checking).  Runs the block-start full
 * forward on snapshot_ids (host, L ids), which fills the K/V cache, then one
 * step on current_ids (host, L ids) for the block [block_start,
 * block_start + block_size).  If current_ids equals snapshot_ids the step is
 * the block's first (refresh) step and uses the full forward's logits.
 * Outputs (host, caller-owned, block_size entries each; logits may be NULL,
 * else block_size * vocab floats with the mask id's logit included):
 * logits z, confidence, argmax token, and the unmask flags (0/1) the
 * threshold rule picks among the positions of the block that are masked in
 * current_ids.  Errors as fdllm_generate. */
FDLLM_API int fdllm_step_debug(fdllm_ctx* ctx, const int32_t* snapshot_ids, const int32_t* current_ids,
                     int L, int block_start, int block_size, float tau, int cache_mode,
                     float* logits, float* conf, int32_t* tok, uint8_t* unmask);

/* Similarity of the K/V activations of two token sequences (diagnostic).
 * The approximate block cache rests on the observation that the K/V
 * activations of adjacent denoising steps are nearly identical (cosine
 * similarity close to 1): ccyt168.com Fast-dLLM overview, section 一
 * "核心技术", item 1 (双向缓存策略 / 高相似度验证, Fig. 2), and the
 * techwalker.com Fast-dLLM article, section "核心创新：适合扩散模型的KV缓存".
 * This call measures it for the loaded weights: a full forward over ids_a
 * (e.g. the sequence at the block start, whose K/V a DualCache step reuses)
 * and one over ids_b (e.g. the sequence some steps later), both of L tokens,
 * then writes cos_out[(layer * 2 + kv) * L + pos] (caller-owned, 2 *
 * n_layers * L doubles): the cosine of the two sequences' K (kv = 0) or V
 * (kv = 1) at that layer and position, over its n_kv_heads * head_dim
 * values (float64 accumulation; 1 for two zero vectors).  The first call
 * allocates a device copy of the K/V cache.  Leaves the cache holding
 * ids_b's K/V.  Errors: ARG (NULL, L out of range, id out of range), STATE
 * (no weights), OOM, CUDA. */
FDLLM_API int fdllm_kv_similarity(fdllm_ctx* ctx, const int32_t* ids_a, const int32_t* ids_b,
                                  int L, double* cos_out);

/* Failure-path self-test.  Every device-side wait of the library (TMA and
 * MMA barriers, the block-step kernel's phase and row waits) is bounded: a
 * wait that runs past its limit (2 s) records a timeout in the context's
 * device error word and its kernel returns, and the call that launched it
 * returns FDLLM_ERR_TIMEOUT.  This call runs one wait that nothing can
 * complete through that same bounded wait and returns what a real timeout
 * returns: FDLLM_ERR_TIMEOUT, after about 2 s, with the error word cleared
 * and the context still usable.  No fault, trap or hang is involved.  The
 * pages have no counterpart; it tests the library's own failure detection.
 * Errors: ARG (NULL ctx), CUDA. */
FDLLM_API int fdllm_selftest_wait_timeout(fdllm_ctx* ctx);

/* Copy K and V of one layer for positions [pos0, pos0 + n) from the cache to
 * host float buffers k_out, v_out ([n, n_kv_heads, head_dim] each).  Used to
 * check that the cache after a refresh equals a full recompute.  Errors: ARG
 * (range), STATE, CUDA. */
FDLLM_API int fdllm_read_kv(fdllm_ctx* ctx, int layer, int pos0, int n, float* k_out, float* v_out);

/* Kernel-level check of the GEMM the decoder runs (tcgen05 on the bf16
 * model, CUDA cores on the fp32 one): y = x W^T with a plain float output.
 * w_dev [N, K] is a device pointer in the ctx dtype (row-major); the bf16
 * model's decoder runs the same tcgen05 kernel on fp16 operands.  x_dev
 * holds the M x K activations as the decoder stores them: fp32 model, plain
 * [M, K] float rows; bf16 model, two-term bf16 rows (x = hi + lo with
 * hi = bf16(x), lo = bf16(x - hi)) grouped by 32 tokens: group j occupies
 * rows [64j, 64j+32) with the hi terms of tokens 32j.. and rows
 * [64j+32, 64j+64) with their lo terms (2 * ceil(M/32) * 32 rows in all).
 * y_dev is a device [M, N] float buffer: y = x W^T, or y += x W^T when
 * accumulate != 0 (the residual-add epilogue of the decoder's O and down
 * projections).  splits = 0 lets the planner pick the K split; splits > 0
 * forces it (bf16 only).  Needs K % 64 == 0 and 16-byte aligned w_dev /
 * x_dev on the bf16 model.  Like the decoder, the bf16 model runs shapes
 * with N % 256 == 0 and M > 64 on pairs of SMs (tcgen05 cta_group::2, a
 * 256-row weight tile per pair) unless FDLLM_GEMM_PAIR=0 was set when the
 * ctx was created; the result is the same up to float32 rounding order.
 * Errors: ARG, CUDA, TIMEOUT. */
FDLLM_API int fdllm_gemm(fdllm_ctx* ctx, const void* w_dev, const void* x_dev, float* y_dev,
                         int N, int M, int K, int splits, int accumulate);

/* fdllm_gemm with the decoder's own operand type on the bf16 model: w_dev
 * [N, K] fp16 and x_dev the two-term fp16 pair rows (hi = fp16(x),
 * lo = fp16(x - hi)) in the layout described for fdllm_gemm; the same
 * kernels, tile plans, splits and float y.  The bf16 model's decoder keeps
 * its weights and activations in exactly this form (bf16 weights are held
 * as the fp16 values equal to them).  Errors: ARG (also on the fp32 model),
 * CUDA, TIMEOUT. */
FDLLM_API int fdllm_gemm_f16(fdllm_ctx* ctx, const void* w_dev, const void* x_dev, float* y_dev,
                             int N, int M, int K, int splits, int accumulate);

/* Kernel-level check of the decoder's attention over the ctx's KV cache:
 * o = softmax(q K^T / sqrt(head_dim)) V with keys [0, L) of layer `layer`
 * (as left by the last forward), no mask: the bidirectional attention of
 * the block queries over cached prefix, block and cached suffix K/V
 * (techwalker.com Fast-dLLM article, section "核心创新：适合扩散模型的KV缓存";
 * ccyt168.com overview, section 一, item 1).  fp32 model: q_dev [M, n_heads,
 * head_dim] and o_dev [M, n_heads * head_dim] float.  bf16 model: q_dev is
 * two planes of fp16 [M, n_heads, head_dim] (hi terms, then lo terms) and
 * o_dev receives two-term fp16 rows of n_heads * head_dim in the 32-token
 * grouping described for fdllm_gemm (the decoder's storage format).  The
 * same kernel choice (and key split for M <= 64) as a decode step.
 * Errors: ARG, STATE, CUDA. */
FDLLM_API int fdllm_attention(fdllm_ctx* ctx, const void* q_dev, void* o_dev, int layer, int M,
                              int L);

/* The same GEMM as fdllm_gemm on the bf16 model (tcgen05, two-term x in
 * the 32-token pair-row layout described there, float y), for callers that
 * cannot allocate device memory: code that runs inside a host framework
 * which has reserved the device memory up front (a cudaMalloc here would
 * fail or break its accounting), or that must not take the implicit
 * synchronisation an allocation can cause.  It needs no ctx and allocates
 * nothing: the split-K scratch (8 MiB of partial tiles, 4096 tile counters,
 * an error word) is a fixed device array inside the library, present on
 * every GPU that loads the library until the process exits.  The Fast-dLLM
 * pages have no counterpart of this call; it is an interface convenience.
 *   - Runs on the current CUDA device, on stream cuda_stream (NULL = the
 *     legacy default stream), and returns when the result is in y_dev.
 *   - The first call on each device looks the scratch array's address up
 *     and caches it; make that first call before any stream capture.
 *   - Every call on a device shares the same scratch array: calls whose GPU
 *     work overlaps (two host threads, or two streams) race and give wrong
 *     results.  The tile counters and the error word are cleared on the
 *     stream at the start of every call.
 *   - Maximum size: the planned (or forced) K splits must fit their partial
 *     tiles in 8 MiB (units x tokens-per-tile x 128 floats) and the output
 *     must have at most 4096 tiles of 128 features x one token tile; larger
 *     requests return FDLLM_ERR_ARG (message via fdllm_last_error(NULL)).
 * Errors: ARG (NULL pointers, sizes <= 0, K % 64 != 0, misaligned operands,
 * too many splits, beyond the maximum, not an sm_100 GPU), CUDA, TIMEOUT. */
FDLLM_API int fdllm_gemm_noalloc(const void* w_dev, const void* x_dev, float* y_dev, int N, int M,
                                 int K, int splits, void* cuda_stream);

/* Per-kernel-class timing.  While enabled, every launch the ctx makes is
 * bracketed by CUDA events on the ctx's stream and accumulated per class
 * (e.g. "gemm.ffn_up.step", "attn.full"), together with the launch's
 * algorithmic DRAM bytes (weights + activations read + outputs written +
 * K/V read, each once) and FLOPs.  Enabling resets the counters.  Timing
 * adds event records between launches, so a run meant for throughput should
 * keep it off. */
typedef struct {
  char name[48];
  int64_t launches;
  double total_ms;     /* summed event-to-event device time */
  double bytes;        /* summed algorithmic bytes */
  double flops;        /* summed FLOPs */
} fdllm_kernel_stat;

FDLLM_API int fdllm_profile_enable(fdllm_ctx* ctx, int enable);

/* Copy up to max_stats class records to out (caller-owned); *n_stats gets
 * the number of classes.  Errors: ARG. */
FDLLM_API int fdllm_profile_read(fdllm_ctx* ctx, fdllm_kernel_stat* out, int max_stats,
                                 int* n_stats);

/* Message for the last failing call on ctx (or on creation when ctx is
 * NULL).  Never NULL. */
FDLLM_API const char* fdllm_last_error(const fdllm_ctx* ctx);

/* Number of this library's kernels launched since creation (or since the
 * last call with reset != 0, which also zeroes it). */
FDLLM_API int64_t fdllm_launch_count(fdllm_ctx* ctx, int reset);

/* Free every device buffer of ctx and ctx itself.  NULL is accepted. */
FDLLM_API int fdllm_destroy(fdllm_ctx* ctx);

#ifdef __cplusplus
}
#endif

#endif /* FDLLM_H */
