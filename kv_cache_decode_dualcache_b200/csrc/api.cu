// Host side of the decoder: context, weight layout, the forward pass over a
// contiguous range of rows, the block-wise decode loop and the C ABI.
//
// One forward covers rows [r0, r0 + M) of the sequence and attends over keys
// [0, L) taken from the paged KV cache (its own rows are written there first,
// by the QKV epilogue):
//   block-start refresh / cache-off step   r0 = 0, M = L
//   DualCache block step                   r0 = s, M = block
//   prefix-cache step                      r0 = s, M = L - s
// The LM head then runs on `n_lm` rows starting at row `lm0` of the forward
// and a single-CTA kernel merges its partials and applies the unmask rule.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <string>
#include <tuple>
#include <vector>

#include "../../include/fdllm.h"
#include "common.cuh"
#include "kernels.h"

using namespace fd;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

const int kNtChoices[3] = {64, 128, 256};   // token-tile rows (two-term: rows/2 tokens)
constexpr size_t kWorkspaceBytes = 64ull << 20;
constexpr int kMaxLmRows = 256;
constexpr int kMaxAttnSplit = 8;   // key splits = CTAs of one thread-block cluster
constexpr int kAttnSplitMaxM = 64;
constexpr int kSpRing = 8;
constexpr int kMaxBatch = 64;      // sequence slots of a context
constexpr int kMaxLmChunk = 512;   // LM-head rows per launch of a batched step

thread_local std::string g_create_error = "no error";

struct LayerW {
  void* wqkv = nullptr;
  void* wo = nullptr;
  void* wgu = nullptr;
  void* wd = nullptr;
  float* attn_norm = nullptr;
  float* ffn_norm = nullptr;
  CUtensorMap m_qkv, m_o, m_gu, m_d;
};

int nt_index(int nt) {
  for (int i = 0; i < 3; ++i)
    if (kNtChoices[i] == nt) return i;
  return -1;
}

// Rows of a two-term activation matrix holding `tokens` tokens.
size_t pair_rows(size_t tokens) { return 2 * ((tokens + 31) / 32) * 32; }

}  // namespace

struct fdllm_ctx {
  fdllm_config cfg{};
  int device = 0;
  cudaStream_t stream = nullptr;
  bool own_stream = false;
  fdllm_allocator alloc{};
  bool custom_alloc = false;
  std::string err = "no error";
  std::vector<void*> allocations;
  bool weights_loaded = false;
  int num_sms = 0;
  bool tc = false;          // bf16 model on tensor cores
  int f32 = 0;              // fp32 model
  size_t esz = 2;           // bytes per weight / activation element
  EncodeTiledFn encode = nullptr;

  void* weights = nullptr;
  void* embed = nullptr;
  void* lm_head = nullptr;
  float* final_norm = nullptr;
  std::vector<LayerW> layers;
  CUtensorMap m_head;

  void* kv_pool = nullptr;
  void* kv_snap = nullptr;          // fdllm_kv_similarity: copy of the K/V pool
  double* kv_cos = nullptr;         // fdllm_kv_similarity: [n_layers][2][max_seq] cosines
  int kv_planes = 2;        // fp32: K, V; bf16: K hi, K lo, V hi, V lo
  int n_pages = 0;          // pages per layer over every sequence slot
  int pages_per_seq = 0;    // slot q owns pages [q * pages_per_seq, (q + 1) * pages_per_seq)
  int rows_cap = 0;         // forward rows the activation buffers hold (max_batch * max_seq)
  size_t q_plane = 0;       // elements per q plane (bf16 two-term q)
  int* page_table = nullptr;
  float2* rope = nullptr;
  int* x = nullptr;
  float* h = nullptr;
  void* a = nullptr;
  void* q = nullptr;
  void* o = nullptr;
  void* f = nullptr;
  float* ws = nullptr;
  int* counters = nullptr;
  int n_counters = 0;
  float* lm_part = nullptr;
  size_t lm_part_cap = 0;   // SoftmaxState entries
  float* conf = nullptr;
  int* tok = nullptr;
  uint8_t* unmask = nullptr;
  float* dbg = nullptr;
  size_t dbg_cap = 0;
  DecodeState* state = nullptr;
  DecodeState* state_host = nullptr;
  int* err_dev = nullptr;
  int* err_host = nullptr;
  unsigned long long* inexact_dev = nullptr;  // bf16 -> fp16 weight conversions that changed a value
  int64_t inexact_weights = 0;
  int* check = nullptr;        // self-check record (FDLLM_CHECKS builds)
  size_t cap_h = 0, cap_q = 0, cap_kv = 0, cap_f = 0;
  CUtensorMap m_a[3], m_o[3], m_f[3];
  // tcgen05 attention of many-query forwards: q (3-D, hi plane then lo
  // plane) and K/V pool (2-D, one row per (layer, page, plane, head, slot))
  CUtensorMap m_q3, m_kv;
  bool use_attn_tc = true;
  bool use_attn_blk = true;     // block steps' attention: tcgen05 kernel with key splits
  bool use_tc2 = true;          // SM-pair GEMM for the many-token forwards
  int tc2_pairs = 0;            // resident SM pairs of that kernel (0 = not used)
  std::map<std::tuple<int, int, int, int>, GemmShape> plans;
  int64_t launches = 0;
  bool pdl = true;              // programmatic dependent launch between kernels
  bool graphs = true;           // replay each step kind from a captured CUDA graph
  // batched decode (fdllm_generate_batch): per-slot decode states and the
  // per-step row / tile / select tables (one device buffer, one pinned
  // staging copy, one upload per step)
  DecodeState* states = nullptr;
  DecodeState* states_host = nullptr;
  uint8_t* btab = nullptr;
  uint8_t* btab_host = nullptr;
  size_t btab_bytes = 0;
  StepParams* sp = nullptr;     // device step scalars (read by the kernels)
  StepParams* sp_host = nullptr;  // pinned ring of kSpRing slots: a pending async copy
  int sp_slot = 0;                // never reads a slot overwritten after it was queued
  int fixed_k = 0;                // > 0 during fdllm_generate_fixed_k
  struct StepGraph {
    cudaGraphExec_t exec;
    int n_part;
    int launches;
  };
  std::map<std::tuple<int, int, int>, StepGraph> step_graphs;
  // DualCache block steps of at most 32 tokens (bf16 model) run as one
  // attention launch plus one chain-kernel launch per layer (chain.cu).
  bool use_chain = true;
  int* chain_sync = nullptr;        // per-phase done counters of one step, then the abort word
  int chain_sync_cap = 0;
  float* norm_ss = nullptr;         // chain NORM phases: partial sums of squares [32][8]
  struct ChainProg {
    std::vector<ChainArgs> launches;           // kernel arguments per launch
    std::vector<int> first;                    // index of each launch's first phase in the step
    std::vector<double> bytes, flops;          // algorithmic bytes / flops per launch
    int n_phases = 0;
  };
  std::map<std::tuple<int, int, uintptr_t>, ChainProg> chain_progs;
  // per-kernel-class timing (fdllm_profile_enable)
  struct ProfPending {
    cudaEvent_t a, b;
    int cls;
    double bytes, flops;
  };
  bool prof = false;
  std::vector<cudaEvent_t> ev_pool;
  std::vector<ProfPending> prof_pending;
  std::vector<fdllm_kernel_stat> prof_stats;
};

namespace {

int fail(fdllm_ctx* c, int code, const std::string& msg) {
  if (c) c->err = msg; else g_create_error = msg;
  return code;
}

int prof_class(fdllm_ctx* ctx, const std::string& name) {
  for (size_t i = 0; i < ctx->prof_stats.size(); ++i)
    if (name == ctx->prof_stats[i].name) return (int)i;
  fdllm_kernel_stat st{};
  std::snprintf(st.name, sizeof(st.name), "%s", name.c_str());
  ctx->prof_stats.push_back(st);
  return (int)ctx->prof_stats.size() - 1;
}

cudaEvent_t prof_event(fdllm_ctx* ctx) {
  if (!ctx->ev_pool.empty()) {
    cudaEvent_t e = ctx->ev_pool.back();
    ctx->ev_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) e = nullptr;
  return e;
}

// Bracket one launch with events when profiling is on.
struct ProfScope {
  fdllm_ctx* ctx;
  cudaEvent_t a = nullptr;
  int cls = -1;
  double bytes, flops;
  ProfScope(fdllm_ctx* c, const std::string& name, double by, double fl)
      : ctx(c), bytes(by), flops(fl) {
    if (!ctx->prof) return;
    a = prof_event(ctx);
    if (!a) return;
    cls = prof_class(ctx, name);
    cudaEventRecord(a, ctx->stream);
  }
  ~ProfScope() {
    if (!ctx->prof || !a) return;
    cudaEvent_t b = prof_event(ctx);
    if (!b) { ctx->ev_pool.push_back(a); return; }
    cudaEventRecord(b, ctx->stream);
    ctx->prof_pending.push_back({a, b, cls, bytes, flops});
  }
};

// Called after the stream has been synchronised.
void prof_harvest(fdllm_ctx* ctx) {
  for (auto& p : ctx->prof_pending) {
    float ms = 0.0f;
    if (cudaEventElapsedTime(&ms, p.a, p.b) == cudaSuccess) {
      fdllm_kernel_stat& st = ctx->prof_stats[p.cls];
      st.launches += 1;
      st.total_ms += ms;
      st.bytes += p.bytes;
      st.flops += p.flops;
    }
    ctx->ev_pool.push_back(p.a);
    ctx->ev_pool.push_back(p.b);
  }
  ctx->prof_pending.clear();
}

#define CK(call)                                                                       \
  do {                                                                                 \
    cudaError_t e_ = (call);                                                           \
    if (e_ != cudaSuccess)                                                             \
      return fail(ctx, FDLLM_ERR_CUDA, std::string(#call) + ": " + cudaGetErrorString(e_)); \
  } while (0)

#define KL(call)                                                                       \
  do {                                                                                 \
    cudaError_t e_ = (call);                                                           \
    ++ctx->launches;                                                                   \
    if (e_ != cudaSuccess)                                                             \
      return fail(ctx, FDLLM_ERR_CUDA, std::string(#call) + ": " + cudaGetErrorString(e_)); \
  } while (0)

void* dalloc(fdllm_ctx* ctx, size_t bytes) {
  if (bytes == 0) bytes = 256;
  bytes = (bytes + 255) & ~(size_t)255;
  void* p = nullptr;
  if (ctx->custom_alloc) {
    p = ctx->alloc.alloc(bytes, ctx->alloc.user);
  } else if (cudaMalloc(&p, bytes) != cudaSuccess) {
    cudaGetLastError();
    p = nullptr;
  }
  if (p) ctx->allocations.push_back(p);
  return p;
}

void dfree_all(fdllm_ctx* ctx) {
  for (void* p : ctx->allocations) {
    if (ctx->custom_alloc) ctx->alloc.free(p, ctx->alloc.user);
    else cudaFree(p);
  }
  ctx->allocations.clear();
}

// 2-byte row-major [rows, cols] operand, boxes of box_rows x 64 elements with
// the 128-byte swizzle.  f16: fp16 (the decoder's storage), else bf16.
bool make_map(fdllm_ctx* ctx, CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
              uint32_t box_rows, bool f16 = true) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = ctx->encode(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                           2, const_cast<void*>(base), dims,
                           strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// q planes [2 * rows][heads][hd] (hi plane rows, then lo plane rows) as a
// 3-D map with boxes of {64 dims, rep heads, 128 / rep positions}.
bool make_q_map(fdllm_ctx* ctx, CUtensorMap* m, const void* q, uint64_t rows_per_plane) {
  const fdllm_config& c = ctx->cfg;
  const int rep = c.n_heads / c.n_kv_heads;
  if (rep < 1 || rep > 128) return false;
  cuuint64_t dims[3] = {(cuuint64_t)c.head_dim, (cuuint64_t)c.n_heads, 2 * rows_per_plane};
  cuuint64_t strides[2] = {(cuuint64_t)c.head_dim * 2, (cuuint64_t)c.n_heads * c.head_dim * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)rep, (cuuint32_t)(128 / rep)};
  cuuint32_t es[3] = {1, 1, 1};
  return ctx->encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(q), dims, strides,
                     box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int check_config(const fdllm_config* c, std::string* why) {
  auto bad = [&](const char* m) { *why = m; return FDLLM_ERR_ARG; };
  if (!c) return bad("config is NULL");
  if (c->n_layers < 1) return bad("n_layers must be >= 1");
  if (c->d_model < 64 || c->d_model % 64 || c->d_model > 8192)
    return bad("d_model must be a multiple of 64 in [64, 8192]");
  if (c->ffn_dim < 64 || c->ffn_dim % 64) return bad("ffn_dim must be a positive multiple of 64");
  if (!(c->head_dim == 32 || c->head_dim == 64 || c->head_dim == 128))
    return bad("head_dim must be 32, 64 or 128");
  if (c->n_heads < 1 || c->n_kv_heads < 1 || c->n_heads % c->n_kv_heads)
    return bad("n_heads must be a positive multiple of n_kv_heads");
  if ((c->n_heads * c->head_dim) % 64) return bad("n_heads * head_dim must be a multiple of 64");
  if (c->vocab < 2) return bad("vocab must be >= 2");
  if (c->mask_id < 0 || c->mask_id >= c->vocab) return bad("mask_id must be in [0, vocab)");
  if (!(c->dtype == FDLLM_DTYPE_F32 || c->dtype == FDLLM_DTYPE_BF16)) return bad("unknown dtype");
  if (c->dtype == FDLLM_DTYPE_BF16 && c->head_dim == 32)
    return bad("the bf16 attention kernel needs head_dim 64 or 128");
  if (c->dtype == FDLLM_DTYPE_BF16 && (c->n_kv_heads * c->head_dim) % 64)
    return bad("n_kv_heads * head_dim must be a multiple of 64");
  if (c->max_batch < 1 || c->max_batch > kMaxBatch) return bad("max_batch must be in [1, 64]");
  if (c->max_seq < 1 || c->max_seq > (1 << 20)) return bad("max_seq out of range");
  if (!(c->rms_eps >= 0.0f) || !std::isfinite(c->rope_theta) || !(c->rope_theta > 0.0f) ||
      !std::isfinite(c->logit_scale))
    return bad("rope_theta, rms_eps and logit_scale must be finite (theta > 0, eps >= 0)");
  return FDLLM_OK;
}

// --------------------------------------------------------------- GEMM plan
// fp32 model: CUDA-core tiles of 128 features x 32 tokens.  bf16 model:
// token tile of nt rows (nt/2 tokens, two-term), the K split chosen to
// balance the per-CTA K blocks over the persistent grid (deterministic
// reduction of the splits).  Plans are memoised per shape.
GemmShape make_plan(const fdllm_ctx* ctx, int N, int M, int K, bool allow_split, bool lm) {
  if (ctx->tc) return plan_gemm_tc(ctx->num_sms, N, M, K, allow_split, kWorkspaceBytes, lm ? 128 : 256);
  GemmShape g{};
  g.N = N;
  g.M = M;
  g.K = K;
  g.n_tiles = (N + 127) / 128;
  g.kb_total = (K + 63) / 64;
  g.nt = 32;
  g.splits = 1;
  g.n_tt = (M + 31) / 32;
  g.units = g.n_tiles * g.n_tt;
  g.grid = g.units;
  return g;
}

GemmShape plan_gemm(fdllm_ctx* ctx, int N, int M, int K, bool allow_split, bool lm = false,
                    bool pair = false) {
  const auto key = std::make_tuple(N, M, K, (allow_split ? 1 : 0) + (lm ? 2 : 0) + (pair ? 4 : 0));
  auto it = ctx->plans.find(key);
  if (it != ctx->plans.end()) return it->second;
  GemmShape g = pair ? plan_gemm_tc2(ctx->tc2_pairs, N, M, K, kWorkspaceBytes)
                     : make_plan(ctx, N, M, K, allow_split, lm);
  ctx->plans[key] = g;
  return g;
}

// The many-token GEMMs of the bf16 model run on SM pairs where the shape
// allows it (N a multiple of 256, more than 64 tokens, not the LM head).
bool use_pair_gemm(const fdllm_ctx* ctx, int N, int M, bool lm) {
  return ctx->tc && ctx->tc2_pairs > 0 && !lm && N % 256 == 0 && M > 64;
}

const CUtensorMap* act_map(CUtensorMap* maps, int nt) { return &maps[nt_index(nt)]; }

int run_gemm(fdllm_ctx* ctx, const char* tag, const void* w, const CUtensorMap* wmap,
             const void* act, CUtensorMap* amaps, int act_row0, int N, int M, int K,
             const EpiParams& ep_in, int* n_part_out = nullptr) {
  const bool lm = ep_in.kind == EPI_LMHEAD;
  const bool pair = use_pair_gemm(ctx, N, M, lm);
  GemmShape gs = plan_gemm(ctx, N, M, K, !lm, lm, pair);
  gs.f16 = ctx->tc ? 1 : 0;  // fp16 weights and two-term fp16 activations
  EpiParams ep = ep_in;
  ep.N = N;
  ep.M = M;
  ep.act_f32 = ctx->f32;
  if (lm && (size_t)gs.grid * M > ctx->lm_part_cap)
    return fail(ctx, FDLLM_ERR_CUDA, "LM-head partial buffer too small");
  if (gs.n_tiles * gs.n_tt > ctx->n_counters)
    return fail(ctx, FDLLM_ERR_CUDA, "split-K counter buffer too small");
  const double es = (double)ctx->esz;
  double out_bytes = 0.0;
  switch (ep.kind) {
    case EPI_QKV: out_bytes = (double)M * N * es; break;
    case EPI_RESID: out_bytes = 2.0 * M * N * 4.0; break;
    case EPI_SWIGLU: out_bytes = (double)M * (N / 2) * es; break;
    case EPI_STORE: out_bytes = (double)M * N * 4.0; break;
    default: break;
  }
  ProfScope ps(ctx, std::string("gemm.") + tag + (M <= 64 ? ".step" : ".full"),
               (double)N * K * es + (double)M * K * es + out_bytes, 2.0 * M * N * K);
  if (ctx->tc) {
    GemmScratch sc{ctx->ws, ctx->counters, ctx->err_dev, kWorkspaceBytes / sizeof(float),
                   ctx->n_counters};
    if (pair)
      KL(launch_gemm_tc2(wmap, act_map(amaps, 128), gs, ep, sc, ctx->stream, ctx->pdl));
    else
      KL(launch_gemm_tc(wmap, act_map(amaps, gs.nt), gs, ep, sc, ctx->stream, ctx->pdl));
  } else {
    KL(launch_gemm_simt((const float*)w, (const float*)act, act_row0, K, gs, ep, ctx->stream,
                        ctx->pdl));
  }
  if (n_part_out) *n_part_out = gs.grid;
  return FDLLM_OK;
}

EpiParams epi_base(fdllm_ctx* ctx, int kind) {
  EpiParams ep{};
  ep.kind = kind;
  ep.check = ctx->check;
  ep.cap_h = ctx->cap_h;
  ep.cap_q = ctx->cap_q;
  ep.cap_kv = ctx->cap_kv;
  ep.cap_f = ctx->cap_f;
  ep.cap_dbg = ctx->dbg_cap;
  ep.cap_lm = ctx->lm_part_cap;
  ep.sp = ctx->sp;
  ep.kv_pool = ctx->kv_pool;
  ep.kv_planes = ctx->kv_planes;
  ep.q_plane = ctx->q_plane;
  ep.page_table = ctx->page_table;
  ep.n_pages = ctx->n_pages;
  ep.rope = ctx->rope;
  ep.n_heads = ctx->cfg.n_heads;
  ep.n_kv_heads = ctx->cfg.n_kv_heads;
  ep.head_dim = ctx->cfg.head_dim;
  ep.logit_scale = ctx->cfg.logit_scale;
  ep.mask_id = ctx->cfg.mask_id;
  return ep;
}

int run_attention(fdllm_ctx* ctx, int layer, int M, int L, const void* q = nullptr,
                  void* o = nullptr) {
  const fdllm_config& c = ctx->cfg;
  AttnParams ap{};
  ap.q = q ? q : ctx->q;
  ap.q_plane = q ? (size_t)M * c.n_heads * c.head_dim : ctx->q_plane;
  ap.o = o ? o : ctx->o;
  ap.kv_pool = ctx->kv_pool;
  ap.kv_planes = ctx->kv_planes;
  ap.page_table = ctx->page_table;
  ap.n_pages = ctx->n_pages;
  ap.layer = layer;
  ap.M = M;
  ap.L = L;
  ap.n_heads = c.n_heads;
  ap.n_kv_heads = c.n_kv_heads;
  ap.head_dim = c.head_dim;
  ap.n_split = 1;
  ap.keys_per_split = ((L + 63) / 64) * 64;
  ap.err = ctx->err_dev;
  const double es = (double)ctx->esz;
  const double kv_bytes = (double)ctx->kv_planes * L * c.n_kv_heads * c.head_dim * es;
  const double qo_bytes = (ctx->f32 ? 2.0 : 4.0) * M * c.n_heads * c.head_dim * es;
  const double att_flops = 4.0 * M * c.n_heads * (double)L * c.head_dim;
  const std::string att_tag = M <= 64 ? "attn.step" : "attn.full";
  const int rep = c.n_heads / c.n_kv_heads;
  const int tc_ctas = rep <= 128 ? ((M + 128 / rep - 1) / (128 / rep)) * c.n_kv_heads : 0;
  if (ctx->tc && ctx->use_attn_tc && ctx->use_attn_blk && M <= kAttnSplitMaxM) {
    // block steps: tcgen05 attention over 128-key chunks, the keys split over
    // a cluster of up to 8 CTAs per (query-row tile, KV head) so that the
    // grid fills the SMs once
    AttnParams bp = ap;
    const int rows = M * rep, rp = rows <= 32 ? 32 : 64;
    const int ctas = ((rows + rp - 1) / rp) * c.n_kv_heads;
    const int chunks = (L + 127) / 128;
    const int want = std::min(std::min(8, chunks), std::max(1, ctx->num_sms / ctas));
    const int cps = (chunks + want - 1) / want;
    bp.keys_per_split = cps * 128;
    bp.n_split = (chunks + cps - 1) / cps;
    if (attn_blk_supported(bp)) {
      ProfScope ps(ctx, att_tag, kv_bytes + qo_bytes, att_flops);
      KL(launch_attn_blk(&ctx->m_kv, bp, ctx->stream, ctx->pdl));
      return FDLLM_OK;
    }
  }
  const bool tc_path = ctx->tc && ctx->use_attn_tc && M * rep >= 128 &&
                       (M > kAttnSplitMaxM || 2 * tc_ctas >= ctx->num_sms) &&
                       attn_tc_supported(ap);
  if (tc_path) {
    // tcgen05 + TMA attention
    CUtensorMap qm;
    const CUtensorMap* qmap = &ctx->m_q3;
    int q_lo_rows = ctx->rows_cap;
    if (q) {
      q_lo_rows = M;
      if (!make_q_map(ctx, &qm, q, (uint64_t)M))
        return fail(ctx, FDLLM_ERR_CUDA, "cuTensorMapEncodeTiled failed for q");
      qmap = &qm;
    }
    ProfScope ps(ctx, att_tag, kv_bytes + qo_bytes, att_flops);
    KL(launch_attn_tc(qmap, &ctx->m_kv, ap, q_lo_rows, ctx->err_dev, ctx->stream, ctx->pdl));
    return FDLLM_OK;
  }
  if (!ctx->tc) {
    ProfScope ps(ctx, att_tag, kv_bytes + qo_bytes, att_flops);
    KL(launch_attn_simt(ap, ctx->stream, ctx->pdl));
    return FDLLM_OK;
  }
  // Few query rows (block steps): split the keys so that the (row tile, KV
  // head, split) CTAs fill the SMs once, at least 2 key tiles per split
  // (measured: one key tile per split, with two single-buffered CTAs per SM
  // and clusters of 8, is slower).
  const int rows_per_cta = attn_rows_per_cta(M, c.n_heads, c.n_kv_heads);
  const int ctas = ((M * rep + rows_per_cta - 1) / rows_per_cta) * c.n_kv_heads;
  const int key_tiles = (L + 63) / 64;
  if (M <= kAttnSplitMaxM && key_tiles >= 4) {
    int want = std::max(1, ctx->num_sms / std::max(1, ctas));
    want = std::min(want, std::min(kMaxAttnSplit, key_tiles / 2));
    if (want > 1) {
      const int tiles_per = (key_tiles + want - 1) / want;
      ap.keys_per_split = tiles_per * 64;
      ap.n_split = (key_tiles + tiles_per - 1) / tiles_per;
    }
  }
  {
    ProfScope ps(ctx, att_tag, kv_bytes + qo_bytes, att_flops);
    KL(launch_attn_mma(&ctx->m_kv, ap, ctx->stream, ctx->pdl));
  }
  return FDLLM_OK;
}

// Forward over rows [r0, r0+M) with keys [0, L); LM head on rows
// [lm0, lm0+n_lm) of the forward.  Returns the number of LM partials.
int forward(fdllm_ctx* ctx, int r0, int M, int L, int lm0, int n_lm, float* dbg, int* n_part) {
  const fdllm_config& c = ctx->cfg;
  const int d = c.d_model, hq = c.n_heads * c.head_dim, hkv = c.n_kv_heads * c.head_dim;
  const int nqkv = hq + 2 * hkv;
  const double es = (double)ctx->esz;
  {
    ProfScope ps(ctx, "embed_rmsnorm", (double)M * d * (2.0 * es + 4.0), 0.0);
    KL(launch_embed_rmsnorm(ctx->x, r0, M, ctx->embed, d, c.vocab, ctx->layers[0].attn_norm,
                            c.rms_eps, ctx->h, ctx->a, ctx->f32, ctx->err_dev, ctx->sp,
                            ctx->stream, ctx->pdl));
  }
  int rc;
  for (int l = 0; l < c.n_layers; ++l) {
    LayerW& lw = ctx->layers[l];
    EpiParams ep = epi_base(ctx, EPI_QKV);
    ep.q_out = ctx->q;
    ep.layer = l;
    ep.pos0 = r0;
    if ((rc = run_gemm(ctx, "qkv", lw.wqkv, &lw.m_qkv, ctx->a, ctx->m_a, 0, nqkv, M, d, ep))) return rc;
    if ((rc = run_attention(ctx, l, M, L))) return rc;
    ep = epi_base(ctx, EPI_RESID);
    ep.h = ctx->h;
    if ((rc = run_gemm(ctx, "o", lw.wo, &lw.m_o, ctx->o, ctx->m_o, 0, d, M, hq, ep))) return rc;
    {
      ProfScope ps(ctx, "rmsnorm", (double)M * d * (es + 4.0), 0.0);
      KL(launch_rmsnorm(ctx->h, 0, M, d, lw.ffn_norm, c.rms_eps, ctx->a, ctx->f32, nullptr, false,
                        ctx->stream, ctx->pdl));
    }
    ep = epi_base(ctx, EPI_SWIGLU);
    ep.f_out = ctx->f;
    if ((rc = run_gemm(ctx, "ffn_up", lw.wgu, &lw.m_gu, ctx->a, ctx->m_a, 0, 2 * c.ffn_dim, M, d, ep)))
      return rc;
    ep = epi_base(ctx, EPI_RESID);
    ep.h = ctx->h;
    if ((rc = run_gemm(ctx, "ffn_down", lw.wd, &lw.m_d, ctx->f, ctx->m_f, 0, d, M, c.ffn_dim, ep))) return rc;
    // next layer's attention norm over all rows, or the final norm over the
    // LM-head rows only (written to rows [0, n_lm) of the activation buffer)
    const bool last = l + 1 == c.n_layers;
    const int nr = last ? n_lm : M;
    {
      ProfScope ps(ctx, "rmsnorm", (double)nr * d * (es + 4.0), 0.0);
      KL(launch_rmsnorm(ctx->h, last ? lm0 : 0, nr, d,
                        last ? ctx->final_norm : ctx->layers[l + 1].attn_norm, c.rms_eps, ctx->a,
                        ctx->f32, ctx->sp, last, ctx->stream, ctx->pdl));
    }
  }
  EpiParams ep = epi_base(ctx, EPI_LMHEAD);
  ep.lm_part = ctx->lm_part;
  ep.dbg_logits = dbg;
  return run_gemm(ctx, "lm_head", ctx->lm_head, &ctx->m_head, ctx->a, ctx->m_a, 0, c.vocab, n_lm,
                  d, ep, n_part);
}

int sync_state(fdllm_ctx* ctx);

// ----------------------------------------------------- batched steps
// One forward over the rows of several sequences (slots) at once, so every
// GEMM streams the weights once for all of them.  The host writes the
// step's tables into ctx->btab: per forward row its position and slot, the
// attention tiles (each within one sequence, keys [0, L) of that slot), the
// LM-head rows (each sequence's block rows) and the select segments.
struct BatchFwd {
  int M = 0;                       // forward rows
  const RowInfo* rows = nullptr;   // [M]
  const RowChunk* row_chunks = nullptr;  // [M / 32]
  const AttnTile* tiles = nullptr;     // key-split kernel (block-sized segments)
  int n_tiles = 0;
  const AttnTile* tc_tiles = nullptr;  // tcgen05 kernel (segments of >= 128 query rows per KV head)
  int n_tc_tiles = 0;
  int max_L = 0;
  const int* lm_src = nullptr;     // [m_lm]: forward row of LM-head row k
  int m_lm = 0;
  const SelectSeg* segs = nullptr; // [n_segs], in LM-row order
  std::vector<std::pair<int, int>> chunks;  // LM-head launches: segments [first, last)
  std::vector<SelectSeg> host_segs;
  float tau = 0.0f;
  int fixed_k = 0;
};

int run_attention_batched(fdllm_ctx* ctx, int layer, const BatchFwd& bf) {
  const fdllm_config& c = ctx->cfg;
  AttnParams ap{};
  ap.q = ctx->q;
  ap.q_plane = ctx->q_plane;
  ap.o = ctx->o;
  ap.kv_pool = ctx->kv_pool;
  ap.kv_planes = ctx->kv_planes;
  ap.page_table = ctx->page_table;
  ap.n_pages = ctx->n_pages;
  ap.layer = layer;
  ap.M = bf.M;
  ap.L = bf.max_L;
  ap.n_heads = c.n_heads;
  ap.n_kv_heads = c.n_kv_heads;
  ap.head_dim = c.head_dim;
  ap.n_split = 1;
  ap.keys_per_split = ((bf.max_L + 63) / 64) * 64;
  ap.err = ctx->err_dev;
  ap.tiles = bf.tiles;
  ap.n_tiles = bf.n_tiles;
  ap.pages_per_seq = ctx->pages_per_seq;
  const double es = (double)ctx->esz;
  ProfScope ps(ctx, "attn.batch",
               (double)ctx->kv_planes * bf.max_L * c.n_kv_heads * c.head_dim * es,
               4.0 * bf.M * c.n_heads * (double)bf.max_L * c.head_dim);
  if (!ctx->tc) {
    KL(launch_attn_simt(ap, ctx->stream, ctx->pdl));
    return FDLLM_OK;
  }
  if (bf.n_tc_tiles > 0) {
    AttnParams at = ap;
    at.tiles = bf.tc_tiles;
    at.n_tiles = bf.n_tc_tiles;
    KL(launch_attn_tc(&ctx->m_q3, &ctx->m_kv, at, ctx->rows_cap, ctx->err_dev, ctx->stream,
                      ctx->pdl));
  }
  if (bf.n_tiles > 0) {
    // the block segments: tcgen05 block attention (64-row tiles, every key
    // of the segment's sequence per CTA), else the mma.sync kernel
    AttnParams bp = ap;
    bp.keys_per_split = ((bf.max_L + 127) / 128) * 128;
    if (ctx->use_attn_blk && attn_blk_supported(bp))
      KL(launch_attn_blk(&ctx->m_kv, bp, ctx->stream, ctx->pdl));
    else
      KL(launch_attn_mma(&ctx->m_kv, ap, ctx->stream, ctx->pdl));
  }
  return FDLLM_OK;
}

// The batched forward, then per LM chunk: final norm of its rows, LM head,
// merge + select of its sequences.
int forward_batched(fdllm_ctx* ctx, const BatchFwd& bf) {
  const fdllm_config& c = ctx->cfg;
  const int d = c.d_model, hq = c.n_heads * c.head_dim, hkv = c.n_kv_heads * c.head_dim;
  const int nqkv = hq + 2 * hkv;
  const int M = bf.M;
  const double es = (double)ctx->esz;
  const RowMap gather{bf.rows, c.max_seq, nullptr};
  {
    ProfScope ps(ctx, "embed_rmsnorm", (double)M * d * (2.0 * es + 4.0), 0.0);
    KL(launch_embed_rmsnorm(ctx->x, 0, M, ctx->embed, d, c.vocab, ctx->layers[0].attn_norm,
                            c.rms_eps, ctx->h, ctx->a, ctx->f32, ctx->err_dev, nullptr,
                            ctx->stream, ctx->pdl, gather));
  }
  int rc;
  for (int l = 0; l < c.n_layers; ++l) {
    LayerW& lw = ctx->layers[l];
    EpiParams ep = epi_base(ctx, EPI_QKV);
    ep.sp = nullptr;
    ep.pos0 = 0;
    ep.rows = bf.rows;
    ep.chunks = bf.row_chunks;
    ep.pages_per_seq = ctx->pages_per_seq;
    ep.q_out = ctx->q;
    ep.layer = l;
    if ((rc = run_gemm(ctx, "qkv", lw.wqkv, &lw.m_qkv, ctx->a, ctx->m_a, 0, nqkv, M, d, ep))) return rc;
    if ((rc = run_attention_batched(ctx, l, bf))) return rc;
    ep = epi_base(ctx, EPI_RESID);
    ep.sp = nullptr;
    ep.h = ctx->h;
    if ((rc = run_gemm(ctx, "o", lw.wo, &lw.m_o, ctx->o, ctx->m_o, 0, d, M, hq, ep))) return rc;
    {
      ProfScope ps(ctx, "rmsnorm", (double)M * d * (es + 4.0), 0.0);
      KL(launch_rmsnorm(ctx->h, 0, M, d, lw.ffn_norm, c.rms_eps, ctx->a, ctx->f32, nullptr, false,
                        ctx->stream, ctx->pdl));
    }
    ep = epi_base(ctx, EPI_SWIGLU);
    ep.sp = nullptr;
    ep.f_out = ctx->f;
    if ((rc = run_gemm(ctx, "ffn_up", lw.wgu, &lw.m_gu, ctx->a, ctx->m_a, 0, 2 * c.ffn_dim, M, d, ep)))
      return rc;
    ep = epi_base(ctx, EPI_RESID);
    ep.sp = nullptr;
    ep.h = ctx->h;
    if ((rc = run_gemm(ctx, "ffn_down", lw.wd, &lw.m_d, ctx->f, ctx->m_f, 0, d, M, c.ffn_dim, ep)))
      return rc;
    if (l + 1 < c.n_layers) {
      ProfScope ps(ctx, "rmsnorm", (double)M * d * (es + 4.0), 0.0);
      KL(launch_rmsnorm(ctx->h, 0, M, d, ctx->layers[l + 1].attn_norm, c.rms_eps, ctx->a,
                        ctx->f32, nullptr, false, ctx->stream, ctx->pdl));
    }
  }
  // LM head per chunk of sequences; partials of chunk j after those of chunks < j
  size_t part_off = 0;
  for (const auto& ch : bf.chunks) {
    const int k0 = bf.host_segs[ch.first].k0;
    const int k1 = bf.host_segs[ch.second - 1].k0 + bf.host_segs[ch.second - 1].n;
    const int mc = k1 - k0;
    {
      ProfScope ps(ctx, "rmsnorm", (double)mc * d * (es + 4.0), 0.0);
      KL(launch_rmsnorm(ctx->h, 0, mc, d, ctx->final_norm, c.rms_eps, ctx->a, ctx->f32, nullptr,
                        false, ctx->stream, ctx->pdl, RowMap{nullptr, 0, bf.lm_src + k0}));
    }
    const GemmShape gs = plan_gemm(ctx, c.vocab, mc, d, false, true);
    if (part_off + (size_t)gs.grid * mc > ctx->lm_part_cap)
      return fail(ctx, FDLLM_ERR_CUDA, "LM-head partial buffer too small");
    float* part = reinterpret_cast<float*>(reinterpret_cast<SoftmaxState*>(ctx->lm_part) + part_off);
    EpiParams ep = epi_base(ctx, EPI_LMHEAD);
    ep.sp = nullptr;
    ep.lm_part = part;
    int n_part = 0;
    if ((rc = run_gemm(ctx, "lm_head", ctx->lm_head, &ctx->m_head, ctx->a, ctx->m_a, 0, c.vocab, mc,
                       d, ep, &n_part)))
      return rc;
    ProfScope ps(ctx, "merge_select", (double)n_part * mc * 12.0, 0.0);
    // segment k0 relative to the chunk; conf / tok / unmask by global LM row
    KL(launch_merge_select_seg(part, n_part, mc, bf.segs + ch.first, ch.second - ch.first, ctx->x,
                               c.max_seq, c.mask_id, bf.tau, bf.fixed_k, ctx->conf + k0,
                               ctx->tok + k0, ctx->unmask + k0, ctx->states, ctx->stream,
                               ctx->pdl));
    part_off += (size_t)n_part * mc;
  }
  return FDLLM_OK;
}

// Continuous batching over the context's sequence slots: every global step
// runs one batched forward over all active sequences (each in its own block
// schedule: a full forward at a block start or with the cache off, the block
// rows in DualCache steps, rows [s, L) in prefix-cache steps); a sequence
// that finishes leaves its slot to the next waiting one.
int generate_batch_impl(fdllm_ctx* ctx, int batch, const int32_t* const* prompts,
                        const int* prompt_lens, int G, int B, float tau, int mode, int fixed_k,
                        int32_t* out_tokens, int* out_steps, fdllm_stats* stats) {
  const fdllm_config& c = ctx->cfg;
  const int n_slots = std::min(batch, c.max_batch);
  const int n_blocks = G / B;
  const int rep = c.n_heads / c.n_kv_heads;
  const int rpc = attn_rows_per_cta(-1, c.n_heads, c.n_kv_heads);
  struct Slot {
    int seq = -1, P = 0, L = 0, b = 0, nb = 0, steps = 0;
    bool first = true;
  };
  std::vector<Slot> slots(n_slots);
  int next = 0;
  CK(cudaSetDevice(ctx->device));
  auto admit = [&](int q) -> int {
    Slot& S = slots[q];
    S = Slot();
    if (next >= batch) return FDLLM_OK;
    S.seq = next++;
    S.P = prompt_lens[S.seq];
    S.L = S.P + G;
    int* xq = ctx->x + (size_t)q * c.max_seq;
    if (S.P > 0)
      CK(cudaMemcpyAsync(xq, prompts[S.seq], sizeof(int32_t) * S.P, cudaMemcpyHostToDevice,
                         ctx->stream));
    KL(launch_fill_masked(xq, S.P, S.L, c.mask_id, ctx->stream));
    CK(cudaMemsetAsync(ctx->states + q, 0, sizeof(DecodeState), ctx->stream));
    return FDLLM_OK;
  };
  int rc;
  for (int q = 0; q < n_slots; ++q)
    if ((rc = admit(q))) return rc;
  const bool timing = stats && stats->collect_timing;
  const bool trace = stats && stats->trace_cap > 0;
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  if (timing) {
    CK(cudaEventCreate(&e0));
    CK(cudaEventCreate(&e1));
  }
  int refresh = 0, cached = 0;
  double refresh_ms = 0, cached_ms = 0;
  std::vector<RowInfo> rows;
  std::vector<RowChunk> rchunks;
  std::vector<AttnTile> tiles, tc_tiles;
  std::vector<int> lm_src;
  const int tc_mp = 128 / rep;   // positions per tcgen05 attention tile
  const bool tc_ok = ctx->tc && ctx->use_attn_tc && rep <= 128;
  std::vector<float> h_conf;
  std::vector<int32_t> h_tok;
  std::vector<uint8_t> h_unmask;
  for (;;) {
    BatchFwd bf;
    bf.tau = tau;
    bf.fixed_k = fixed_k;
    rows.clear();
    rchunks.clear();
    tiles.clear();
    tc_tiles.clear();
    lm_src.clear();
    bool any_full = false;
    for (int q = 0; q < n_slots; ++q) {
      const Slot& S = slots[q];
      if (S.seq < 0) continue;
      const int s = S.P + S.b * B;
      const bool full = S.first || mode == FDLLM_CACHE_NONE;
      any_full = any_full || full;
      const int r_lo = full ? 0 : s;
      const int r_hi = (full || mode == FDLLM_CACHE_PREFIX) ? S.L : s + B;
      const int q0 = (int)rows.size(), m = r_hi - r_lo;
      for (int pos = r_lo; pos < r_hi; ++pos) rows.push_back(RowInfo{pos, q});
      // pad to a multiple of 32 rows: every 32-row chunk is one sequence's
      for (int c0 = q0; c0 < (int)rows.size(); c0 += 32)
        rchunks.push_back(RowChunk{rows[c0].pos, q, std::min(32, (int)rows.size() - c0), 0});
      while (rows.size() % 32) rows.push_back(RowInfo{-1, q});
      if (tc_ok && m * rep >= 128) {
        // many query rows (a full forward or a long prefix-cache segment)
        for (int p0 = 0; p0 < m; p0 += tc_mp)
          tc_tiles.push_back(AttnTile{q0, m, p0 * rep, S.L, q, {0, 0, 0}});
      } else if (ctx->tc) {
        for (int r0 = 0; r0 < m * rep; r0 += rpc) tiles.push_back(AttnTile{q0, m, r0, S.L, q, {0, 0, 0}});
      } else {
        for (int j = 0; j < m; ++j) tiles.push_back(AttnTile{q0 + j, 1, 0, S.L, q, {0, 0, 0}});
      }
      bf.max_L = std::max(bf.max_L, S.L);
      bf.host_segs.push_back(SelectSeg{(int)lm_src.size(), B, q, s});
      for (int j = 0; j < B; ++j) lm_src.push_back(q0 + (s - r_lo) + j);
    }
    if (bf.host_segs.empty()) break;
    // LM-head chunks of at most kMaxLmChunk rows; select k0 relative to the chunk
    std::vector<SelectSeg> dev_segs = bf.host_segs;
    for (int i = 0; i < (int)bf.host_segs.size();) {
      int j = i, rows_c = 0;
      while (j < (int)bf.host_segs.size() && rows_c + bf.host_segs[j].n <= kMaxLmChunk)
        rows_c += bf.host_segs[j++].n;
      for (int k = i; k < j; ++k) dev_segs[k].k0 -= bf.host_segs[i].k0;
      bf.chunks.push_back({i, j});
      i = j;
    }
    // one upload of the step's tables
    auto align = [](size_t v) { return (v + 255) & ~(size_t)255; };
    const size_t o_rows = 0, o_chunks = align(rows.size() * sizeof(RowInfo));
    const size_t o_tiles = o_chunks + align(rchunks.size() * sizeof(RowChunk));
    const size_t o_tc = o_tiles + align(tiles.size() * sizeof(AttnTile));
    const size_t o_lm = o_tc + align(tc_tiles.size() * sizeof(AttnTile));
    const size_t o_seg = o_lm + align(lm_src.size() * sizeof(int));
    const size_t used = o_seg + dev_segs.size() * sizeof(SelectSeg);
    if (used > ctx->btab_bytes) return fail(ctx, FDLLM_ERR_CUDA, "batched-step tables too large");
    std::memcpy(ctx->btab_host + o_rows, rows.data(), rows.size() * sizeof(RowInfo));
    std::memcpy(ctx->btab_host + o_chunks, rchunks.data(), rchunks.size() * sizeof(RowChunk));
    std::memcpy(ctx->btab_host + o_tiles, tiles.data(), tiles.size() * sizeof(AttnTile));
    std::memcpy(ctx->btab_host + o_tc, tc_tiles.data(), tc_tiles.size() * sizeof(AttnTile));
    std::memcpy(ctx->btab_host + o_lm, lm_src.data(), lm_src.size() * sizeof(int));
    std::memcpy(ctx->btab_host + o_seg, dev_segs.data(), dev_segs.size() * sizeof(SelectSeg));
    CK(cudaMemcpyAsync(ctx->btab, ctx->btab_host, used, cudaMemcpyHostToDevice, ctx->stream));
    bf.M = (int)rows.size();
    bf.rows = reinterpret_cast<const RowInfo*>(ctx->btab + o_rows);
    bf.row_chunks = reinterpret_cast<const RowChunk*>(ctx->btab + o_chunks);
    bf.tiles = reinterpret_cast<const AttnTile*>(ctx->btab + o_tiles);
    bf.n_tiles = (int)tiles.size();
    bf.tc_tiles = reinterpret_cast<const AttnTile*>(ctx->btab + o_tc);
    bf.n_tc_tiles = (int)tc_tiles.size();
    bf.lm_src = reinterpret_cast<const int*>(ctx->btab + o_lm);
    bf.m_lm = (int)lm_src.size();
    bf.segs = reinterpret_cast<const SelectSeg*>(ctx->btab + o_seg);
    if (timing) CK(cudaEventRecord(e0, ctx->stream));
    if ((rc = forward_batched(ctx, bf))) return rc;
    if (timing) CK(cudaEventRecord(e1, ctx->stream));
    CK(cudaMemcpyAsync(ctx->states_host, ctx->states, sizeof(DecodeState) * n_slots,
                       cudaMemcpyDeviceToHost, ctx->stream));
    if ((rc = sync_state(ctx))) return rc;  // also the error word
    (any_full ? refresh : cached) += 1;
    if (timing) {
      float ms = 0;
      CK(cudaEventElapsedTime(&ms, e0, e1));
      (any_full ? refresh_ms : cached_ms) += ms;
    }
    if (trace) {
      h_conf.resize(bf.m_lm);
      h_tok.resize(bf.m_lm);
      h_unmask.resize(bf.m_lm);
      CK(cudaMemcpy(h_conf.data(), ctx->conf, sizeof(float) * bf.m_lm, cudaMemcpyDeviceToHost));
      CK(cudaMemcpy(h_tok.data(), ctx->tok, sizeof(int32_t) * bf.m_lm, cudaMemcpyDeviceToHost));
      CK(cudaMemcpy(h_unmask.data(), ctx->unmask, bf.m_lm, cudaMemcpyDeviceToHost));
    }
    for (const SelectSeg& sg : bf.host_segs) {
      Slot& S = slots[sg.seq];
      const DecodeState& st = ctx->states_host[sg.seq];
      if (trace && S.steps < stats->trace_cap) {
        const size_t idx = (size_t)S.seq * stats->trace_cap + S.steps;
        if (stats->trace_block) stats->trace_block[idx] = S.b;
        if (stats->trace_conf) std::memcpy(stats->trace_conf + idx * B, &h_conf[sg.k0], 4 * B);
        if (stats->trace_tok) std::memcpy(stats->trace_tok + idx * B, &h_tok[sg.k0], 4 * B);
        if (stats->trace_unmask) std::memcpy(stats->trace_unmask + idx * B, &h_unmask[sg.k0], B);
      }
      S.steps += 1;
      S.nb += 1;
      S.first = false;
      if (st.remaining == 0) {
        if (stats && stats->steps_per_block)
          stats->steps_per_block[(size_t)S.seq * n_blocks + S.b] = S.nb;
        S.b += 1;
        S.nb = 0;
        S.first = true;
        if (S.b == n_blocks) {
          out_steps[S.seq] = S.steps;
          CK(cudaMemcpy(out_tokens + (size_t)S.seq * G, ctx->x + (size_t)sg.seq * c.max_seq + S.P,
                        sizeof(int32_t) * G, cudaMemcpyDeviceToHost));
          if ((rc = admit(sg.seq))) return rc;
        }
      } else if (st.unmasked < 1 || S.nb >= B) {
        return fail(ctx, FDLLM_ERR_CUDA, "decode step made no progress");
      }
    }
  }
  CK(cudaStreamSynchronize(ctx->stream));
  if (timing) {
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
  }
  if (stats) {
    int total = 0;
    for (int i = 0; i < batch; ++i) total += out_steps[i];
    stats->steps = total;
    stats->refresh_steps = refresh;
    stats->cached_steps = cached;
    stats->n_blocks = n_blocks * batch;
    stats->refresh_ms = refresh_ms;
    stats->cached_ms = cached_ms;
  }
  return FDLLM_OK;
}

// ----------------------------------------------------- block-step chains
bool chain_applicable(const fdllm_ctx* ctx, int M, int lm0, int n_lm) {
  return ctx->tc && ctx->use_chain && ctx->weights_loaded && M >= 1 && M <= 32 && lm0 == 0 &&
         n_lm == M && ctx->cfg.d_model % 512 == 0 && ctx->cfg.d_model <= CHAIN_NORM_GROUPS * 512;
}

// The phases of one block step over M rows with keys [0, L): launch 0 =
// [EMBED_NORM, QKV_0]; launch l + 1 = [O_l, NORM, gate/up_l, down_l, NORM,
// QKV_{l+1} or LM head].  The attention of layer l runs between launches l
// and l + 1.
int build_chain(fdllm_ctx* ctx, int M, int L, float* dbg, fdllm_ctx::ChainProg* out) {
  const fdllm_config& c = ctx->cfg;
  const int d = c.d_model, hq = c.n_heads * c.head_dim, hkv = c.n_kv_heads * c.head_dim;
  const int nl = c.n_layers;
  const CUtensorMap& amap_a = ctx->m_a[0];   // 64-row token tiles
  const CUtensorMap& amap_o = ctx->m_o[0];
  const CUtensorMap& amap_f = ctx->m_f[0];
  const int G = ctx->num_sms;
  const double es = 2.0;
  std::vector<ChainPhase> ph;
  fdllm_ctx::ChainProg pr;
  int rot = 0;
  double bytes = 0, flops = 0;
  std::vector<std::pair<int, int>> chains;   // (first phase, phase count)
  auto begin_chain = [&]() {
    chains.push_back({(int)ph.size(), 0});
    rot = 0;
    bytes = flops = 0;
  };
  auto end_chain = [&]() {
    chains.back().second = (int)ph.size() - chains.back().first;
    pr.bytes.push_back(bytes);
    pr.flops.push_back(flops);
  };
  auto norm = [&](int type, const float* gain) {
    ChainPhase P{};
    P.type = type;
    P.gain = gain;
    P.rot = rot;
    rot = (rot + M * (d / 512)) % G;
    if (!ph.empty() && ph.back().type == CH_GEMM && ph.back().ep.kind == EPI_RESID)
      P.resid_splits = ph.back().splits;
    ph.push_back(P);
    bytes += (double)M * d * (4.0 + 4.0 + 2.0 * es);
  };
  auto gemm = [&](const CUtensorMap& wmap, const CUtensorMap& amap, int N, int K, EpiParams ep,
                  bool lm) -> bool {
    // Split count: inside one launch a phase ends with its slowest CTA, so
    // balance comes first: the largest per-CTA share of K blocks (units go
    // round robin), plus a small charge per split for the partial tiles
    // (residual GEMMs: read by the next norm) or for the last-arriver
    // reduction (the other epilogues).
    const int T = (N + 127) / 128, KB = (K + 63) / 64;
    int best_s = 1;
    double best = 1e300;
    for (int sp = 1; sp <= (lm ? 1 : 16) && sp <= KB; ++sp) {
      const long long units = (long long)T * sp;
      if ((size_t)units * 32 * 128 * sizeof(float) > kWorkspaceBytes) break;
      const double load = (double)((units + G - 1) / G) * ((KB + sp - 1) / sp);
      const double cost = load + (ep.kind == EPI_RESID ? 0.25 * sp : (sp > 1 ? 4.0 : 0.0) + 0.5 * sp);
      if (cost < best) {
        best = cost;
        best_s = sp;
      }
    }
    if (T > ctx->n_counters) return false;
    ChainPhase P{};
    P.type = CH_GEMM;
    P.N = N;
    P.K = K;
    P.kb_total = KB;
    P.n_tiles = T;
    P.splits = best_s;
    P.units = T * best_s;
    P.kc = 8;
    P.rot = rot;
    rot = (rot + P.units) % G;
    P.wmap = wmap;
    P.amap = amap;
    ep.N = N;
    ep.M = M;
    ep.act_f32 = 0;
    P.ep = ep;
    ph.push_back(P);

    double out_b = 0;
    switch (ep.kind) {
      case EPI_QKV: out_b = (double)M * N * es * 2; break;
      case EPI_RESID: out_b = 2.0 * M * N * 4.0; break;
      case EPI_SWIGLU: out_b = (double)M * (N / 2) * es * 2; break;
      default: break;
    }
    bytes += (double)N * K * es + 2.0 * M * K * es + out_b;
    flops += 2.0 * M * N * K;
    return true;
  };
  auto qkv = [&](int l) {
    EpiParams ep = epi_base(ctx, EPI_QKV);
    ep.q_out = ctx->q;
    ep.layer = l;
    return gemm(ctx->layers[l].m_qkv, amap_a, hq + 2 * hkv, d, ep, false);
  };
  bool ok = true;
  begin_chain();
  norm(CH_EMBED_NORM, ctx->layers[0].attn_norm);
  ok = ok && qkv(0);
  end_chain();
  for (int l = 0; l < nl && ok; ++l) {
    LayerW& lw = ctx->layers[l];
    begin_chain();
    EpiParams ep = epi_base(ctx, EPI_RESID);
    ep.h = ctx->h;
    ok = ok && gemm(lw.m_o, amap_o, d, hq, ep, false);
    norm(CH_NORM, lw.ffn_norm);
    ep = epi_base(ctx, EPI_SWIGLU);
    ep.f_out = ctx->f;
    ok = ok && gemm(lw.m_gu, amap_a, 2 * c.ffn_dim, d, ep, false);
    ep = epi_base(ctx, EPI_RESID);
    ep.h = ctx->h;
    ok = ok && gemm(lw.m_d, amap_f, d, c.ffn_dim, ep, false);
    if (l + 1 < nl) {
      norm(CH_NORM, ctx->layers[l + 1].attn_norm);
      ok = ok && qkv(l + 1);
    } else {
      norm(CH_NORM, ctx->final_norm);
      ep = epi_base(ctx, EPI_LMHEAD);
      ep.lm_part = ctx->lm_part;
      ep.dbg_logits = dbg;
      ok = ok && gemm(ctx->m_head, amap_a, c.vocab, d, ep, true);
    }
    end_chain();
  }
  if (!ok) return fail(ctx, FDLLM_ERR_CUDA, "block-step chain: unexpected GEMM plan");
  if ((size_t)G * M > ctx->lm_part_cap)
    return fail(ctx, FDLLM_ERR_CUDA, "LM-head partial buffer too small");
  pr.n_phases = (int)ph.size();
  for (const auto& ch : chains) {
    if (ch.second > CHAIN_MAX_PHASES) return fail(ctx, FDLLM_ERR_CUDA, "chain too long");
    ChainArgs A{};
    for (int i = 0; i < ch.second; ++i) A.ph[i] = ph[ch.first + i];
    A.n_phases = ch.second;
    A.M = M;
    A.d = c.d_model;
    A.vocab = c.vocab;
    A.eps = c.rms_eps;
    A.x = ctx->x;
    A.embed = ctx->embed;
    A.h = ctx->h;
    A.a = ctx->a;
    A.sp = ctx->sp;
    A.sc = GemmScratch{ctx->ws, ctx->counters, ctx->err_dev, kWorkspaceBytes / sizeof(float),
                       ctx->n_counters};
    pr.launches.push_back(A);
    pr.first.push_back(ch.first);
  }
  const int n_sync = (pr.n_phases + 1) * CHAIN_DONE_STRIDE + pr.n_phases * 32 +
                     pr.n_phases * CHAIN_DONE_STRIDE;
  if (n_sync > ctx->chain_sync_cap) {
    ctx->chain_sync = (int*)dalloc(ctx, sizeof(int) * n_sync);
    if (!ctx->chain_sync) return fail(ctx, FDLLM_ERR_OOM, "chain counter allocation failed");
    ctx->chain_sync_cap = n_sync;
  }
  if (!ctx->norm_ss) {
    ctx->norm_ss = (float*)dalloc(ctx, sizeof(float) * 32 * CHAIN_NORM_GROUPS);
    if (!ctx->norm_ss) return fail(ctx, FDLLM_ERR_OOM, "chain norm scratch allocation failed");
  }
  *out = pr;
  return FDLLM_OK;
}

// One block step (rows [sp->r0, sp->r0 + M), keys [0, L)) through the chain
// kernel: n_layers + 1 chain launches with the attention launches between
// them.  The LM partials come from every CTA of the grid.
int forward_chain(fdllm_ctx* ctx, int M, int L, float* dbg, int* n_part) {
  const auto key = std::make_tuple(M, L, (uintptr_t)dbg);
  auto it = ctx->chain_progs.find(key);
  if (it == ctx->chain_progs.end()) {
    fdllm_ctx::ChainProg pr;
    int rc = build_chain(ctx, M, L, dbg, &pr);
    if (rc) return rc;
    it = ctx->chain_progs.emplace(key, pr).first;
  }
  const fdllm_ctx::ChainProg& pr = it->second;
  const fdllm_config& c = ctx->cfg;
  // counters of one step: [done per phase, abort word][NORM row counters][unit claims]
  const int rowcnt0 = (pr.n_phases + 1) * CHAIN_DONE_STRIDE;
  const int next0 = rowcnt0 + pr.n_phases * 32;
  CK(cudaMemsetAsync(ctx->chain_sync, 0,
                     sizeof(int) * (next0 + pr.n_phases * CHAIN_DONE_STRIDE), ctx->stream));
  for (size_t ci = 0; ci < pr.launches.size(); ++ci) {
    ChainArgs A = pr.launches[ci];
    A.done = ctx->chain_sync + pr.first[ci] * CHAIN_DONE_STRIDE;
    A.gabort = ctx->chain_sync + pr.n_phases * CHAIN_DONE_STRIDE;
    A.rowcnt = ctx->chain_sync + rowcnt0 + pr.first[ci] * 32;
    A.norm_ss = ctx->norm_ss;
    A.next = ctx->chain_sync + next0 + pr.first[ci] * CHAIN_DONE_STRIDE;
    {
      ProfScope ps(ctx, "chain.step", pr.bytes[ci], pr.flops[ci]);
      KL(launch_chain(A, ctx->num_sms, ctx->stream, ctx->pdl && ci > 0));
    }
    if ((int)ci < c.n_layers) {
      int rc = run_attention(ctx, (int)ci, M, L);
      if (rc) return rc;
    }
  }
  *n_part = ctx->num_sms;
  return FDLLM_OK;
}

int sync_state(fdllm_ctx* ctx) {
  CK(cudaMemcpyAsync(ctx->state_host, ctx->state, sizeof(DecodeState), cudaMemcpyDeviceToHost,
                     ctx->stream));
  CK(cudaMemcpyAsync(ctx->err_host, ctx->err_dev, sizeof(int), cudaMemcpyDeviceToHost,
                     ctx->stream));
  CK(cudaStreamSynchronize(ctx->stream));
  if (!ctx->prof_pending.empty()) prof_harvest(ctx);
#ifdef FDLLM_CHECKS
  {
    int chk[4] = {0, 0, 0, 0};
    CK(cudaMemcpy(chk, ctx->check, sizeof(chk), cudaMemcpyDeviceToHost));
    if (chk[0]) {
      const int zero4[4] = {0, 0, 0, 0};
      cudaMemcpy(ctx->check, zero4, sizeof(zero4), cudaMemcpyHostToDevice);
      return fail(ctx, FDLLM_ERR_CUDA,
                  "device self-check failed: " + std::to_string(chk[0]) + " violations, first code " +
                      std::to_string(chk[1]) + " index " + std::to_string(chk[2]) + " limit " +
                      std::to_string(chk[3]));
    }
  }
#endif
  const int e = *ctx->err_host;
  if (e) {
    int zero = 0;
    cudaMemcpy(ctx->err_dev, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (e & DEV_ERR_TIMEOUT)
      return fail(ctx, FDLLM_ERR_TIMEOUT, "a device-side wait timed out; results are invalid");
    if (e & DEV_ERR_TOKEN)
      return fail(ctx, FDLLM_ERR_ARG, "a token id is out of range or the prompt holds the mask id");
    return fail(ctx, FDLLM_ERR_CUDA, "device kernel reported an error");
  }
  return FDLLM_OK;
}

// Write the step scalars the kernels read (r0, lm0, s, tau).  Each update
// uses the next slot of a pinned ring; every call path synchronises the
// stream before kSpRing updates are outstanding.
int set_step_params(fdllm_ctx* ctx, int r0, int lm0, int s, float tau) {
  StepParams* slot = ctx->sp_host + ctx->sp_slot;
  ctx->sp_slot = (ctx->sp_slot + 1) % kSpRing;
  *slot = StepParams{r0, lm0, s, tau, ctx->fixed_k};
  CK(cudaMemcpyAsync(ctx->sp, slot, sizeof(StepParams), cudaMemcpyHostToDevice, ctx->stream));
  return FDLLM_OK;
}

// The launches of one step: forward over rows [r0, r0+M) (r0 and lm0 come
// from the step scalars) and the merge/select kernel.
int enqueue_step(fdllm_ctx* ctx, int r0, int M, int L, int lm0, int B, float tau, float* dbg,
                 int* n_part) {
  int rc = chain_applicable(ctx, M, lm0, B) ? forward_chain(ctx, M, L, dbg, n_part)
                                            : forward(ctx, r0, M, L, lm0, B, dbg, n_part);
  if (rc) return rc;
  ProfScope ps(ctx, "merge_select", (double)*n_part * B * 12.0, 0.0);
  KL(launch_merge_select(ctx->lm_part, *n_part, B, ctx->x, 0, ctx->cfg.mask_id, tau, 1, ctx->conf,
                         ctx->tok, ctx->unmask, ctx->state, ctx->sp, ctx->stream, ctx->pdl));
  return FDLLM_OK;
}

// One denoising step: forward for the mode + merge/select.  first = block
// start.  Steps of the same shape replay one captured CUDA graph (the kernel
// sequence depends only on the row count, the key count and the block size;
// the per-step scalars live in device memory).
int run_step(fdllm_ctx* ctx, int mode, bool first, int s, int B, int L, float tau, float* dbg) {
  int r0, M, lm0;
  if (first || mode == FDLLM_CACHE_NONE) {
    r0 = 0; M = L; lm0 = s;
  } else if (mode == FDLLM_CACHE_DUAL) {
    r0 = s; M = B; lm0 = 0;
  } else {
    r0 = s; M = L - s; lm0 = 0;
  }
  int rc = set_step_params(ctx, r0, lm0, s, tau);
  if (rc) return rc;
  int n_part = 0;
  if (!ctx->graphs || ctx->prof || dbg) return enqueue_step(ctx, r0, M, L, lm0, B, tau, dbg, &n_part);
  const auto key = std::make_tuple(M, L, B);
  auto it = ctx->step_graphs.find(key);
  if (it == ctx->step_graphs.end()) {
    cudaGraph_t g = nullptr;
    CK(cudaStreamBeginCapture(ctx->stream, cudaStreamCaptureModeRelaxed));
    const int64_t before = ctx->launches;
    rc = enqueue_step(ctx, r0, M, L, lm0, B, tau, nullptr, &n_part);
    cudaError_t e = cudaStreamEndCapture(ctx->stream, &g);
    if (rc) {
      if (g) cudaGraphDestroy(g);
      return rc;
    }
    if (e != cudaSuccess)
      return fail(ctx, FDLLM_ERR_CUDA, std::string("graph capture: ") + cudaGetErrorString(e));
    fdllm_ctx::StepGraph sg{};
    e = cudaGraphInstantiate(&sg.exec, g, 0);
    cudaGraphDestroy(g);
    if (e != cudaSuccess)
      return fail(ctx, FDLLM_ERR_CUDA, std::string("graph instantiate: ") + cudaGetErrorString(e));
    sg.n_part = n_part;
    sg.launches = (int)(ctx->launches - before);
    ctx->launches = before;
    it = ctx->step_graphs.emplace(key, sg).first;
  }
  CK(cudaGraphLaunch(it->second.exec, ctx->stream));
  ctx->launches += it->second.launches;
  return FDLLM_OK;
}

int check_gen_args(fdllm_ctx* ctx, int prompt_len, int gen_len, int block_size, float tau,
                   int cache_mode) {
  if (!ctx->weights_loaded) return fail(ctx, FDLLM_ERR_STATE, "weights are not loaded");
  if (gen_len < 1 || block_size < 1 || gen_len % block_size)
    return fail(ctx, FDLLM_ERR_ARG, "gen_len and block_size must be >= 1 with gen_len % block_size == 0");
  if (block_size > kMaxLmRows) return fail(ctx, FDLLM_ERR_ARG, "block_size must be <= 256");
  if (prompt_len < 0 || (long long)prompt_len + gen_len > ctx->cfg.max_seq)
    return fail(ctx, FDLLM_ERR_ARG, "prompt_len + gen_len exceeds max_seq (or prompt_len < 0)");
  if (std::isnan(tau)) return fail(ctx, FDLLM_ERR_ARG, "tau is NaN");
  if (cache_mode < FDLLM_CACHE_NONE || cache_mode > FDLLM_CACHE_DUAL)
    return fail(ctx, FDLLM_ERR_ARG, "unknown cache_mode");
  return FDLLM_OK;
}

int generate_impl(fdllm_ctx* ctx, const int32_t* prompt, bool prompt_dev, int P, int G, int B,
                  float tau, int mode, int32_t* out, bool out_dev, int* out_steps,
                  fdllm_stats* stats) {
  int rc = check_gen_args(ctx, P, G, B, tau, mode);
  if (rc) return rc;
  if (!out || !out_steps) return fail(ctx, FDLLM_ERR_ARG, "NULL output pointer");
  if (P > 0 && !prompt) return fail(ctx, FDLLM_ERR_ARG, "NULL prompt");
  const fdllm_config& c = ctx->cfg;
  if (!prompt_dev) {
    for (int i = 0; i < P; ++i)
      if (prompt[i] < 0 || prompt[i] >= c.vocab || prompt[i] == c.mask_id)
        return fail(ctx, FDLLM_ERR_ARG, "prompt id out of range or equal to the mask id");
  }
  CK(cudaSetDevice(ctx->device));
  const int L = P + G;
  if (P > 0)
    CK(cudaMemcpyAsync(ctx->x, prompt, sizeof(int32_t) * P,
                       prompt_dev ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice,
                       ctx->stream));
  if (prompt_dev) KL(launch_check_prompt(ctx->x, P, c.vocab, c.mask_id, ctx->err_dev, ctx->stream));
  KL(launch_fill_masked(ctx->x, P, L, c.mask_id, ctx->stream));
  CK(cudaMemsetAsync(ctx->state, 0, sizeof(DecodeState), ctx->stream));
  const int n_blocks = G / B;
  int total = 0, refresh = 0, cached = 0;
  double refresh_ms = 0, cached_ms = 0;
  const bool timing = stats && stats->collect_timing;
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  if (timing) {
    CK(cudaEventCreate(&e0));
    CK(cudaEventCreate(&e1));
  }
  for (int b = 0; b < n_blocks; ++b) {
    const int s = P + b * B;
    int nb = 0;
    bool first = true;
    for (;;) {
      if (timing) CK(cudaEventRecord(e0, ctx->stream));
      if ((rc = run_step(ctx, mode, first, s, B, L, tau, nullptr))) return rc;
      if (timing) CK(cudaEventRecord(e1, ctx->stream));
      if ((rc = sync_state(ctx))) return rc;
      if (stats && stats->trace_cap > 0 && total + nb < stats->trace_cap) {
        // the step's own outputs (the stream is idle after sync_state)
        const size_t at = (size_t)(total + nb) * B;
        if (stats->trace_block) stats->trace_block[total + nb] = b;
        if (stats->trace_conf)
          CK(cudaMemcpy(stats->trace_conf + at, ctx->conf, sizeof(float) * B, cudaMemcpyDeviceToHost));
        if (stats->trace_tok)
          CK(cudaMemcpy(stats->trace_tok + at, ctx->tok, sizeof(int32_t) * B, cudaMemcpyDeviceToHost));
        if (stats->trace_unmask)
          CK(cudaMemcpy(stats->trace_unmask + at, ctx->unmask, B, cudaMemcpyDeviceToHost));
      }
      const bool full = first || mode == FDLLM_CACHE_NONE;
      if (timing) {
        float ms = 0;
        CK(cudaEventElapsedTime(&ms, e0, e1));
        (full ? refresh_ms : cached_ms) += ms;
      }
      (full ? refresh : cached) += 1;
      first = false;
      ++nb;
      if (ctx->state_host->remaining == 0) break;
      if (ctx->state_host->unmasked < 1 || nb >= B)
        return fail(ctx, FDLLM_ERR_CUDA, "decode step made no progress");
    }
    total += nb;
    if (stats && stats->steps_per_block) stats->steps_per_block[b] = nb;
  }
  CK(cudaMemcpyAsync(out, ctx->x + P, sizeof(int32_t) * G,
                     out_dev ? cudaMemcpyDeviceToDevice : cudaMemcpyDeviceToHost, ctx->stream));
  CK(cudaStreamSynchronize(ctx->stream));
  if (timing) {
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
  }
  *out_steps = total;
  if (stats) {
    stats->steps = total;
    stats->refresh_steps = refresh;
    stats->cached_steps = cached;
    stats->n_blocks = n_blocks;
    stats->refresh_ms = refresh_ms;
    stats->cached_ms = cached_ms;
  }
  return FDLLM_OK;
}

}  // namespace

namespace fd {

// Error message for calls without a ctx (fdllm_last_error(NULL)).
void set_thread_error(const std::string& msg) { g_create_error = msg; }

GemmShape plan_gemm_tc(int num_sms, int N, int M, int K, bool allow_split, size_t ws_bytes,
                       int max_nt) {
  GemmShape g{};
  g.N = N;
  g.M = M;
  g.K = K;
  g.n_tiles = (N + 127) / 128;
  g.kb_total = (K + 63) / 64;
  int nt = 64;
  while (nt / 2 < M && nt < max_nt) nt *= 2;
  g.nt = nt;
  g.n_tt = (M + nt / 2 - 1) / (nt / 2);
  const int base_units = g.n_tiles * g.n_tt;
  const int max_split = allow_split ? std::min(16, std::max(1, g.kb_total / 4)) : 1;
  double best = 1e300;
  int best_s = 1;
  for (int s = 1; s <= max_split; ++s) {
    const long long units = (long long)base_units * s;
    if (s > 1 && (size_t)units * (nt / 2) * 128 * sizeof(float) > ws_bytes) break;
    const int grid = (int)std::min<long long>(units, num_sms);
    // per-CTA cost in K blocks of its units, +2 per unit (pipeline fill and
    // epilogue); a split unit also writes its float partial tile and the last
    // one reads all of them back: (1 + s) tiles of nt/2 x 128 floats, costed
    // in K blocks of the same bytes (one K block moves (128 + nt) x 64 bf16).
    const double kb_bytes = (128.0 + nt) * 64 * 2;
    const double split_cost = s > 1 ? (1.0 + s) * (nt / 2) * 128 * 4 / kb_bytes : 0.0;
    std::vector<double> load(grid, 0.0);
    for (long long u = 0; u < units; ++u) {
      const int sp = (int)(u % s);
      const int kb = (int)((long long)(sp + 1) * g.kb_total / s - (long long)sp * g.kb_total / s);
      load[u % grid] += kb + 2.0 + split_cost;
    }
    double mx = 0.0;
    for (double v : load) mx = std::max(mx, v);
    if (mx < best * 0.9) {
      best = mx;
      best_s = s;
    }
  }
  g.splits = best_s;
  g.units = base_units * best_s;
  g.grid = std::min(g.units, num_sms);
  // K blocks per TMEM accumulation chain.  The tensor core's float32
  // accumulation rounds toward zero: measured on B200, every K block of 64
  // added to a running TMEM accumulator biases it by about -5e-8 relative
  // (-3.8e-6 after K = 4096, -1.2e-5 after K = 12288).  Chains of 8 blocks
  // keep that near -4e-7, the level of a plain float32 dot product; the
  // epilogue warps sum the chains with round-to-nearest float32 adds.
  g.kc = nt == 256 ? 16 : 8;
  return g;
}

// Plan of the SM-pair GEMM (N a multiple of 256): 256-feature x 128-token
// units over at most max_pairs resident pairs, the K split balancing the
// per-pair K blocks as in plan_gemm_tc.  A unit's split partials are two
// 128 x 128 float tiles (one per CTA); one K block moves 2 x 32 KB.
GemmShape plan_gemm_tc2(int max_pairs, int N, int M, int K, size_t ws_bytes) {
  GemmShape g{};
  g.N = N;
  g.M = M;
  g.K = K;
  g.n_tiles = N / 128;
  g.kb_total = (K + 63) / 64;
  g.nt = 256;
  g.n_tt = (M + 127) / 128;
  const int base_units = g.n_tiles / 2 * g.n_tt;
  const int max_split = std::min(16, std::max(1, g.kb_total / 4));
  const double tile_bytes = 128.0 * 128 * 4;
  double best = 1e300;
  int best_s = 1;
  for (int s = 1; s <= max_split; ++s) {
    const long long units = (long long)base_units * s;
    if (s > 1 && (size_t)units * 2 * (size_t)tile_bytes > ws_bytes) break;
    const int pairs = (int)std::min<long long>(units, max_pairs);
    const double split_cost = s > 1 ? (1.0 + s) * tile_bytes / (256.0 * 64 * 2) : 0.0;
    std::vector<double> load(pairs, 0.0);
    for (long long u = 0; u < units; ++u) {
      const int sp = (int)(u % s);
      const int kb = (int)((long long)(sp + 1) * g.kb_total / s - (long long)sp * g.kb_total / s);
      load[u % pairs] += kb + 2.0 + split_cost;
    }
    double mx = 0.0;
    for (double v : load) mx = std::max(mx, v);
    if (mx < best * 0.9) {
      best = mx;
      best_s = s;
    }
  }
  g.splits = best_s;
  g.units = base_units * best_s;
  g.grid = 2 * std::min(g.units, max_pairs);
  g.kc = 16;
  return g;
}

}  // namespace fd

// =============================================================== C ABI
extern "C" {

int fdllm_create(const fdllm_config* cfg, int device, void* cuda_stream,
                 const fdllm_allocator* alloc, fdllm_ctx** out) {
  std::string why;
  if (!out) return fail(nullptr, FDLLM_ERR_ARG, "out is NULL");
  *out = nullptr;
  int rc = check_config(cfg, &why);
  if (rc) return fail(nullptr, rc, why);
  if (alloc && (!alloc->alloc || !alloc->free))
    return fail(nullptr, FDLLM_ERR_ARG, "allocator needs both alloc and free");
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) {
    cudaGetLastError();
    return fail(nullptr, FDLLM_ERR_ARG, "no such CUDA device");
  }
  fdllm_ctx* ctx = new fdllm_ctx();
  ctx->cfg = *cfg;
  ctx->device = device;
  if (alloc) {
    ctx->alloc = *alloc;
    ctx->custom_alloc = true;
  }
  ctx->f32 = cfg->dtype == FDLLM_DTYPE_F32;
  if (const char* ch = std::getenv("FDLLM_CHAIN")) ctx->use_chain = std::strcmp(ch, "0") != 0;
  if (const char* at = std::getenv("FDLLM_ATTN_TC")) ctx->use_attn_tc = std::strcmp(at, "0") != 0;
  if (const char* gp = std::getenv("FDLLM_GEMM_PAIR")) ctx->use_tc2 = std::strcmp(gp, "0") != 0;
  if (const char* ab = std::getenv("FDLLM_ATTN_BLK")) ctx->use_attn_blk = std::strcmp(ab, "0") != 0;
  ctx->tc = !ctx->f32;
  ctx->esz = ctx->f32 ? 4 : 2;
  auto bail = [&](int code, const std::string& m) {
    g_create_error = m;
    dfree_all(ctx);
    if (ctx->own_stream && ctx->stream) cudaStreamDestroy(ctx->stream);
    if (ctx->state_host) cudaFreeHost(ctx->state_host);
    if (ctx->states_host) cudaFreeHost(ctx->states_host);
    if (ctx->btab_host) cudaFreeHost(ctx->btab_host);
    if (ctx->err_host) cudaFreeHost(ctx->err_host);
    if (ctx->sp_host) cudaFreeHost(ctx->sp_host);
    delete ctx;
    return code;
  };
  if (cudaSetDevice(device) != cudaSuccess) return bail(FDLLM_ERR_CUDA, "cudaSetDevice failed");
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, device) != cudaSuccess)
    return bail(FDLLM_ERR_CUDA, "cudaGetDeviceProperties failed");
  ctx->num_sms = prop.multiProcessorCount;
  if (ctx->tc && prop.major != 10)
    return bail(FDLLM_ERR_ARG, "the bf16 path needs an sm_100 (B200-class) GPU");
  if (cuda_stream) {
    ctx->stream = static_cast<cudaStream_t>(cuda_stream);
  } else {
    // A blocking stream: ordered after work on the legacy default stream, so
    // inputs a caller produced there are complete before the decoder reads them.
    if (cudaStreamCreate(&ctx->stream) != cudaSuccess)
      return bail(FDLLM_ERR_CUDA, "cudaStreamCreate failed");
    ctx->own_stream = true;
  }
  if (ctx->tc) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess || !fn)
      return bail(FDLLM_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    ctx->encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  const fdllm_config& c = *cfg;
  const int S = c.max_seq;
  const int hq = c.n_heads * c.head_dim, hkv = c.n_kv_heads * c.head_dim;
  ctx->pages_per_seq = (S + KV_PAGE - 1) / KV_PAGE;
  ctx->n_pages = ctx->pages_per_seq * c.max_batch;
  ctx->kv_planes = ctx->f32 ? 2 : 4;
  const size_t kv_elems =
      (size_t)c.n_layers * ctx->n_pages * ctx->kv_planes * c.n_kv_heads * KV_PAGE * c.head_dim;
  // a batched forward holds up to every slot's whole sequence, each padded to
  // a multiple of 32 rows
  const size_t rows = (size_t)((S + 31) / 32 * 32) * c.max_batch;
  ctx->rows_cap = (int)rows;
  // activation matrices: plain rows (fp32) or two-term pair rows (bf16)
  const size_t arows = ctx->f32 ? rows : pair_rows(rows);
  ctx->q_plane = ctx->f32 ? 0 : rows * hq;
  ctx->kv_pool = dalloc(ctx, kv_elems * ctx->esz);
  ctx->page_table = (int*)dalloc(ctx, sizeof(int) * ctx->n_pages);
  ctx->rope = (float2*)dalloc(ctx, sizeof(float2) * S * (c.head_dim / 2));
  ctx->x = (int*)dalloc(ctx, sizeof(int) * rows);
  ctx->h = (float*)dalloc(ctx, sizeof(float) * rows * c.d_model);
  ctx->a = dalloc(ctx, ctx->esz * arows * c.d_model);
  ctx->q = dalloc(ctx, ctx->esz * rows * hq * (ctx->f32 ? 1 : 2));
  ctx->o = dalloc(ctx, ctx->esz * arows * hq);
  ctx->f = dalloc(ctx, ctx->esz * arows * c.ffn_dim);
  const int max_n = std::max(std::max(c.vocab, 2 * c.ffn_dim), std::max(hq + 2 * hkv, c.d_model));
  ctx->n_counters = (int)(((max_n + 127) / 128) * ((rows + 31) / 32));
  ctx->counters = (int*)dalloc(ctx, sizeof(int) * ctx->n_counters);
  if (ctx->tc) ctx->ws = (float*)dalloc(ctx, kWorkspaceBytes);
  // LM-head rows per launch: a block (<= kMaxLmRows) or a batched chunk
  const int lm_rows = c.max_batch > 1 ? kMaxLmChunk : kMaxLmRows;
  const size_t max_parts = std::max<size_t>((size_t)ctx->num_sms,
                                            (size_t)((c.vocab + 127) / 128) * ((lm_rows + 31) / 32));
  // per-launch partials; a batched step keeps every chunk's partials at once
  const int lm_total = c.max_batch * kMaxLmRows;
  ctx->lm_part_cap = max_parts * (size_t)std::max(lm_rows, lm_total);
  ctx->lm_part = (float*)dalloc(ctx, sizeof(SoftmaxState) * ctx->lm_part_cap);
  ctx->conf = (float*)dalloc(ctx, sizeof(float) * lm_total);
  ctx->tok = (int*)dalloc(ctx, sizeof(int) * lm_total);
  ctx->unmask = (uint8_t*)dalloc(ctx, lm_total);
  ctx->state = (DecodeState*)dalloc(ctx, sizeof(DecodeState));
  ctx->states = (DecodeState*)dalloc(ctx, sizeof(DecodeState) * c.max_batch);
  // batched-step tables: rows, attention tiles (one per query row at most),
  // LM-head row sources, select segments
  ctx->btab_bytes = rows * sizeof(RowInfo) + (rows / 32) * sizeof(RowChunk) +
                    2 * rows * sizeof(AttnTile) +
                    (size_t)lm_total * sizeof(int) + (size_t)c.max_batch * sizeof(SelectSeg) + 1024;
  ctx->btab = (uint8_t*)dalloc(ctx, ctx->btab_bytes);
  ctx->err_dev = (int*)dalloc(ctx, sizeof(int));
  ctx->check = (int*)dalloc(ctx, 4 * sizeof(int));
  ctx->sp = (StepParams*)dalloc(ctx, sizeof(StepParams));
  ctx->cap_h = rows * c.d_model;
  ctx->cap_q = ctx->esz == 4 ? rows * hq : 2 * rows * hq;
  ctx->cap_kv = kv_elems;
  ctx->cap_f = arows * c.ffn_dim;
  for (void* p : {(void*)ctx->kv_pool, (void*)ctx->page_table, (void*)ctx->rope, (void*)ctx->x,
                  (void*)ctx->h, ctx->a, ctx->q, ctx->o, ctx->f, (void*)ctx->counters,
                  (void*)ctx->lm_part,
                  (void*)ctx->conf, (void*)ctx->tok, (void*)ctx->unmask, (void*)ctx->state,
                  (void*)ctx->states, (void*)ctx->btab,
                  (void*)ctx->err_dev, (void*)ctx->check, (void*)ctx->sp})
    if (!p) return bail(FDLLM_ERR_OOM, "device allocation failed");
  if (ctx->tc && !ctx->ws) return bail(FDLLM_ERR_OOM, "device allocation failed");
  if (cudaMallocHost(&ctx->state_host, sizeof(DecodeState)) != cudaSuccess ||
      cudaMallocHost(&ctx->states_host, sizeof(DecodeState) * c.max_batch) != cudaSuccess ||
      cudaMallocHost(&ctx->btab_host, ctx->btab_bytes) != cudaSuccess ||
      cudaMallocHost(&ctx->err_host, sizeof(int)) != cudaSuccess ||
      cudaMallocHost(&ctx->sp_host, kSpRing * sizeof(StepParams)) != cudaSuccess)
    return bail(FDLLM_ERR_OOM, "pinned host allocation failed");
  if (ctx->tc && init_kernel_attributes() != cudaSuccess)
    return bail(FDLLM_ERR_CUDA, "setting kernel shared-memory limits failed");
  // SM pairs for the many-token GEMM: at most one per TPC, as many as can be
  // resident at once (a persistent grid of pairs)
  if (ctx->tc && ctx->use_tc2) ctx->tc2_pairs = std::min(gemm_tc2_max_pairs(), ctx->num_sms / 2);
  // page table (identity for one sequence), RoPE table (angles in double)
  std::vector<int> pt(ctx->n_pages);
  for (int i = 0; i < ctx->n_pages; ++i) pt[i] = i;
  const int half = c.head_dim / 2;
  std::vector<float2> rt((size_t)S * half);
  for (size_t p = 0; p < (size_t)S; ++p)
    for (int i = 0; i < half; ++i) {
      const double inv = std::pow((double)c.rope_theta, -2.0 * i / c.head_dim);
      const double ang = (double)p * inv;
      rt[p * half + i] = make_float2((float)std::cos(ang), (float)std::sin(ang));
    }
  bool ok = cudaMemcpy(ctx->page_table, pt.data(), sizeof(int) * pt.size(),
                       cudaMemcpyHostToDevice) == cudaSuccess &&
            cudaMemcpy(ctx->rope, rt.data(), sizeof(float2) * rt.size(),
                       cudaMemcpyHostToDevice) == cudaSuccess &&
            cudaMemset(ctx->counters, 0, sizeof(int) * ctx->n_counters) == cudaSuccess &&
            cudaMemset(ctx->err_dev, 0, sizeof(int)) == cudaSuccess &&
            cudaMemset(ctx->check, 0, 4 * sizeof(int)) == cudaSuccess &&
            cudaMemset(ctx->kv_pool, 0, kv_elems * ctx->esz) == cudaSuccess &&
            cudaMemset(ctx->a, 0, ctx->esz * arows * c.d_model) == cudaSuccess &&
            cudaMemset(ctx->o, 0, ctx->esz * arows * hq) == cudaSuccess &&
            cudaMemset(ctx->f, 0, ctx->esz * arows * c.ffn_dim) == cudaSuccess;
  if (!ok) return bail(FDLLM_ERR_CUDA, "initialising device buffers failed");
  if (ctx->tc) {
    for (int i = 0; i < 3; ++i) {
      const int nt = kNtChoices[i];
      if (!make_map(ctx, &ctx->m_a[i], ctx->a, arows, c.d_model, nt) ||
          !make_map(ctx, &ctx->m_o[i], ctx->o, arows, hq, nt) ||
          !make_map(ctx, &ctx->m_f[i], ctx->f, arows, c.ffn_dim, nt))
        return bail(FDLLM_ERR_CUDA, "cuTensorMapEncodeTiled failed for an activation buffer");
    }
    // K/V pool rows of head_dim elements: (layer, page, plane, KV head, slot)
    const uint64_t kv_rows = (uint64_t)c.n_layers * ctx->n_pages * ctx->kv_planes * c.n_kv_heads *
                             KV_PAGE;
    if (!make_q_map(ctx, &ctx->m_q3, ctx->q, rows) ||
        !make_map(ctx, &ctx->m_kv, ctx->kv_pool, kv_rows, c.head_dim, 64))
      return bail(FDLLM_ERR_CUDA, "cuTensorMapEncodeTiled failed for q or the K/V cache");
  }
  *out = ctx;
  return FDLLM_OK;
}

int fdllm_load_weights(fdllm_ctx* ctx, const fdllm_tensor* tensors, int n_tensors) {
  if (!ctx) return FDLLM_ERR_ARG;
  if (!tensors || n_tensors < 1) return fail(ctx, FDLLM_ERR_ARG, "no tensors");
  if (ctx->weights_loaded) return fail(ctx, FDLLM_ERR_STATE, "weights are already loaded");
  const fdllm_config& c = ctx->cfg;
  const int d = c.d_model, hd = c.head_dim, F = c.ffn_dim, V = c.vocab;
  const int hq = c.n_heads * hd, hkv = c.n_kv_heads * hd;
  struct Want { std::string name; int64_t numel; const fdllm_tensor* got; };
  std::vector<Want> want;
  want.push_back({"embed", (int64_t)V * d, nullptr});
  for (int l = 0; l < c.n_layers; ++l) {
    const std::string p = "layers." + std::to_string(l) + ".";
    want.push_back({p + "attn_norm", d, nullptr});
    want.push_back({p + "wq", (int64_t)hq * d, nullptr});
    want.push_back({p + "wk", (int64_t)hkv * d, nullptr});
    want.push_back({p + "wv", (int64_t)hkv * d, nullptr});
    want.push_back({p + "wo", (int64_t)d * hq, nullptr});
    want.push_back({p + "ffn_norm", d, nullptr});
    want.push_back({p + "w_gate", (int64_t)F * d, nullptr});
    want.push_back({p + "w_up", (int64_t)F * d, nullptr});
    want.push_back({p + "w_down", (int64_t)d * F, nullptr});
  }
  want.push_back({"final_norm", d, nullptr});
  want.push_back({"lm_head", (int64_t)V * d, nullptr});
  for (int i = 0; i < n_tensors; ++i) {
    const fdllm_tensor& t = tensors[i];
    if (!t.name || !t.data) return fail(ctx, FDLLM_ERR_SHAPE, "tensor with NULL name or data");
    bool found = false;
    for (Want& w : want) {
      if (w.name != t.name) continue;
      if (w.got) return fail(ctx, FDLLM_ERR_SHAPE, "duplicate tensor " + w.name);
      if (t.numel != w.numel)
        return fail(ctx, FDLLM_ERR_SHAPE, "wrong numel for " + w.name);
      if (t.dtype != c.dtype) return fail(ctx, FDLLM_ERR_SHAPE, "wrong dtype for " + w.name);
      w.got = &t;
      found = true;
      break;
    }
    if (!found) return fail(ctx, FDLLM_ERR_SHAPE, std::string("unknown tensor ") + t.name);
  }
  for (Want& w : want)
    if (!w.got) return fail(ctx, FDLLM_ERR_SHAPE, "missing tensor " + w.name);
  CK(cudaSetDevice(ctx->device));
  if (ctx->tc) {
    if (!ctx->inexact_dev) {
      ctx->inexact_dev = (unsigned long long*)dalloc(ctx, sizeof(unsigned long long));
      if (!ctx->inexact_dev) return fail(ctx, FDLLM_ERR_OOM, "counter allocation failed");
    }
    CK(cudaMemset(ctx->inexact_dev, 0, sizeof(unsigned long long)));
  }
  const size_t es = ctx->esz;
  const size_t per_layer = ((size_t)(hq + 2 * hkv) * d + (size_t)d * hq + 2ull * F * d +
                            (size_t)d * F) * es + 2 * sizeof(float) * d;
  const size_t total = 2ull * V * d * es + sizeof(float) * d + c.n_layers * (per_layer + 1024);
  uint8_t* arena = (uint8_t*)dalloc(ctx, total + 4096);
  if (!arena) return fail(ctx, FDLLM_ERR_OOM, "weight allocation failed");
  size_t off = 0;
  auto take = [&](size_t bytes) {
    void* p = arena + off;
    off += (bytes + 255) & ~(size_t)255;
    return p;
  };
  auto find = [&](const std::string& n) {
    for (Want& w : want) if (w.name == n) return w.got;
    return (const fdllm_tensor*)nullptr;
  };
  auto copy_to = [&](void* dst, const std::string& n, size_t bytes) {
    return cudaMemcpy(dst, find(n)->data, bytes, cudaMemcpyDefault);
  };
  auto norm_to = [&](float* dst, const std::string& n) -> cudaError_t {
    const fdllm_tensor* t = find(n);
    std::vector<float> hv(d);
    if (ctx->f32) {
      cudaError_t e = cudaMemcpy(hv.data(), t->data, sizeof(float) * d, cudaMemcpyDefault);
      if (e != cudaSuccess) return e;
    } else {
      std::vector<uint16_t> raw(d);
      cudaError_t e = cudaMemcpy(raw.data(), t->data, 2 * d, cudaMemcpyDefault);
      if (e != cudaSuccess) return e;
      for (int i = 0; i < d; ++i) {
        uint32_t u = (uint32_t)raw[i] << 16;
        std::memcpy(&hv[i], &u, 4);
      }
    }
    return cudaMemcpy(dst, hv.data(), sizeof(float) * d, cudaMemcpyHostToDevice);
  };
  ctx->embed = take((size_t)V * d * es);
  ctx->lm_head = take((size_t)V * d * es);
  ctx->final_norm = (float*)take(sizeof(float) * d);
  CK(copy_to(ctx->embed, "embed", (size_t)V * d * es));
  CK(copy_to(ctx->lm_head, "lm_head", (size_t)V * d * es));
  // The GEMM weights of the bf16 model are held as fp16 (exact for every
  // bf16 value of magnitude in [2^-17, 65504]; below 2^-17 the fp16 grid
  // spacing 2^-24 applies), so that the tensor-core products with the
  // two-term fp16 activations keep 22 significant bits.  The embedding
  // table stays bf16 (read directly into the float32 residual stream).
  auto to_f16 = [&](void* p, size_t n) -> cudaError_t {
    return ctx->tc ? launch_bf16_to_f16(p, n, ctx->err_dev, ctx->inexact_dev, nullptr)
                   : cudaSuccess;
  };
  CK(to_f16(ctx->lm_head, (size_t)V * d));
  CK(norm_to(ctx->final_norm, "final_norm"));
  ctx->layers.assign(c.n_layers, LayerW());
  for (int l = 0; l < c.n_layers; ++l) {
    const std::string p = "layers." + std::to_string(l) + ".";
    LayerW& lw = ctx->layers[l];
    lw.wqkv = take((size_t)(hq + 2 * hkv) * d * es);
    lw.wo = take((size_t)d * hq * es);
    lw.wgu = take(2ull * F * d * es);
    lw.wd = take((size_t)d * F * es);
    lw.attn_norm = (float*)take(sizeof(float) * d);
    lw.ffn_norm = (float*)take(sizeof(float) * d);
    uint8_t* qkv = (uint8_t*)lw.wqkv;
    const size_t row = (size_t)d * es;  // bytes per weight row
    if (ctx->tc) {
      // q and k heads: within each head, slab s (32 rows) holds dims
      // 16s .. 16s+15 then their rotate-half partners dims + hd/2 (the
      // epilogue's rope_slab_dim); 2-D copies over the heads.
      auto put_heads = [&](uint8_t* dst, const std::string& n, int heads) -> cudaError_t {
        const uint8_t* src = (const uint8_t*)find(n)->data;
        for (int sl = 0; sl < hd / 32; ++sl)
          for (int half = 0; half < 2; ++half) {
            cudaError_t e = cudaMemcpy2D(dst + (32 * sl + 16 * half) * row, hd * row,
                                         src + (16 * sl + half * (hd / 2)) * row, hd * row,
                                         16 * row, heads, cudaMemcpyDefault);
            if (e != cudaSuccess) return e;
          }
        return cudaSuccess;
      };
      CK(put_heads(qkv, p + "wq", c.n_heads));
      CK(put_heads(qkv + (size_t)hq * row, p + "wk", c.n_kv_heads));
      CK(copy_to(qkv + (size_t)(hq + hkv) * row, p + "wv", (size_t)hkv * row));
      // gate / up: slab s holds gate rows 16s .. 16s+15 then the matching up rows
      CK(cudaMemcpy2D(lw.wgu, 32 * row, find(p + "w_gate")->data, 16 * row, 16 * row, F / 16,
                      cudaMemcpyDefault));
      CK(cudaMemcpy2D((uint8_t*)lw.wgu + 16 * row, 32 * row, find(p + "w_up")->data, 16 * row,
                      16 * row, F / 16, cudaMemcpyDefault));
    } else {
      CK(copy_to(qkv, p + "wq", (size_t)hq * row));
      CK(copy_to(qkv + (size_t)hq * row, p + "wk", (size_t)hkv * row));
      CK(copy_to(qkv + (size_t)(hq + hkv) * row, p + "wv", (size_t)hkv * row));
      // gate/up interleaved in groups of 64 rows: [g0..g63, u0..u63, g64..g127, ...]
      const size_t grp = 64 * row;
      CK(cudaMemcpy2D(lw.wgu, 2 * grp, find(p + "w_gate")->data, grp, grp, F / 64,
                      cudaMemcpyDefault));
      CK(cudaMemcpy2D((uint8_t*)lw.wgu + grp, 2 * grp, find(p + "w_up")->data, grp, grp, F / 64,
                      cudaMemcpyDefault));
    }
    CK(copy_to(lw.wo, p + "wo", (size_t)d * hq * es));
    CK(copy_to(lw.wd, p + "w_down", (size_t)d * F * es));
    CK(norm_to(lw.attn_norm, p + "attn_norm"));
    CK(norm_to(lw.ffn_norm, p + "ffn_norm"));
    CK(to_f16(lw.wqkv, (size_t)(hq + 2 * hkv) * d));
    CK(to_f16(lw.wo, (size_t)d * hq));
    CK(to_f16(lw.wgu, 2ull * F * d));
    CK(to_f16(lw.wd, (size_t)d * F));
    if (ctx->tc) {
      if (!make_map(ctx, &lw.m_qkv, lw.wqkv, hq + 2 * hkv, d, 128) ||
          !make_map(ctx, &lw.m_o, lw.wo, d, hq, 128) ||
          !make_map(ctx, &lw.m_gu, lw.wgu, 2 * F, d, 128) ||
          !make_map(ctx, &lw.m_d, lw.wd, d, F, 128))
        return fail(ctx, FDLLM_ERR_CUDA, "cuTensorMapEncodeTiled failed for a weight");
    }
  }
  if (ctx->tc && !make_map(ctx, &ctx->m_head, ctx->lm_head, V, d, 128))
    return fail(ctx, FDLLM_ERR_CUDA, "cuTensorMapEncodeTiled failed for lm_head");

  CK(cudaDeviceSynchronize());
  {
    int e = 0;
    CK(cudaMemcpy(&e, ctx->err_dev, sizeof(int), cudaMemcpyDeviceToHost));
    if (e) {
      const int zero = 0;
      cudaMemcpy(ctx->err_dev, &zero, sizeof(int), cudaMemcpyHostToDevice);
      return fail(ctx, FDLLM_ERR_SHAPE,
                  "a GEMM weight is NaN or outside the fp16 range (|w| > 65504)");
    }
  }
  if (ctx->tc) {
    unsigned long long n_inexact = 0;
    CK(cudaMemcpy(&n_inexact, ctx->inexact_dev, sizeof(n_inexact), cudaMemcpyDeviceToHost));
    ctx->inexact_weights = (int64_t)n_inexact;
  }
  ctx->weights = arena;
  ctx->weights_loaded = true;
  return FDLLM_OK;
}

int64_t fdllm_inexact_weight_count(const fdllm_ctx* ctx) {
  if (!ctx) return -1;
  return ctx->weights_loaded ? ctx->inexact_weights : 0;
}

int fdllm_generate(fdllm_ctx* ctx, const int32_t* prompt_ids, int prompt_len, int gen_len,
                   int block_size, float tau, int cache_mode, int32_t* out_tokens,
                   int* out_steps, fdllm_stats* stats) {
  if (!ctx) return FDLLM_ERR_ARG;
  return generate_impl(ctx, prompt_ids, false, prompt_len, gen_len, block_size, tau, cache_mode,
                       out_tokens, false, out_steps, stats);
}

int fdllm_generate_device(fdllm_ctx* ctx, const int32_t* prompt_ids_dev, int prompt_len,
                          int gen_len, int block_size, float tau, int cache_mode,
                          int32_t* out_tokens_dev, int* out_steps, fdllm_stats* stats) {
  if (!ctx) return FDLLM_ERR_ARG;
  return generate_impl(ctx, prompt_ids_dev, true, prompt_len, gen_len, block_size, tau,
                       cache_mode, out_tokens_dev, true, out_steps, stats);
}

int fdllm_generate_fixed_k(fdllm_ctx* ctx, const int32_t* prompt_ids, int prompt_len,
                           int gen_len, int block_size, int k, int cache_mode,
                           int32_t* out_tokens, int* out_steps, fdllm_stats* stats) {
  if (!ctx) return FDLLM_ERR_ARG;
  if (k < 1) return fail(ctx, FDLLM_ERR_ARG, "k must be >= 1");
  ctx->fixed_k = k;
  const int rc = generate_impl(ctx, prompt_ids, false, prompt_len, gen_len, block_size, 0.0f,
                               cache_mode, out_tokens, false, out_steps, stats);
  ctx->fixed_k = 0;
  return rc;
}

int fdllm_generate_batch(fdllm_ctx* ctx, int batch, const int32_t* const* prompts,
                         const int* prompt_lens, int gen_len, int block_size, float tau,
                         int cache_mode, int32_t* out_tokens, int* out_steps, fdllm_stats* stats) {
  if (!ctx) return FDLLM_ERR_ARG;
  if (batch < 1 || !prompts || !prompt_lens || !out_tokens || !out_steps)
    return fail(ctx, FDLLM_ERR_ARG, "batch < 1 or a NULL array");
  // every sequence's arguments before any work
  const fdllm_config& c = ctx->cfg;
  for (int i = 0; i < batch; ++i) {
    int rc = check_gen_args(ctx, prompt_lens[i], gen_len, block_size, tau, cache_mode);
    if (rc) return rc;
    if (prompt_lens[i] > 0 && !prompts[i]) return fail(ctx, FDLLM_ERR_ARG, "NULL prompt");
    for (int j = 0; j < prompt_lens[i]; ++j)
      if (prompts[i][j] < 0 || prompts[i][j] >= c.vocab || prompts[i][j] == c.mask_id)
        return fail(ctx, FDLLM_ERR_ARG, "prompt id out of range or equal to the mask id");
  }
  const int n_blocks = gen_len / block_size;
  if (c.max_batch > 1 && batch > 1)
    return generate_batch_impl(ctx, batch, prompts, prompt_lens, gen_len, block_size, tau,
                               cache_mode, 0, out_tokens, out_steps, stats);
  // one slot: each sequence in turn through the single-sequence path
  fdllm_stats tot{};
  if (stats) tot.collect_timing = stats->collect_timing;
  for (int i = 0; i < batch; ++i) {
    fdllm_stats one{};
    one.collect_timing = stats ? stats->collect_timing : 0;
    one.steps_per_block = (stats && stats->steps_per_block)
                              ? stats->steps_per_block + (size_t)i * n_blocks : nullptr;
    int rc = generate_impl(ctx, prompts[i], false, prompt_lens[i], gen_len, block_size, tau,
                           cache_mode, out_tokens + (size_t)i * gen_len, false, &out_steps[i],
                           stats ? &one : nullptr);
    if (rc) return rc;
    tot.steps += one.steps;
    tot.refresh_steps += one.refresh_steps;
    tot.cached_steps += one.cached_steps;
    tot.n_blocks += one.n_blocks;
    tot.refresh_ms += one.refresh_ms;
    tot.cached_ms += one.cached_ms;
  }
  if (stats) {
    int32_t* spb = stats->steps_per_block;
    *stats = tot;
    stats->steps_per_block = spb;
  }
  return FDLLM_OK;
}

int fdllm_step_debug(fdllm_ctx* ctx, const int32_t* snapshot_ids, const int32_t* current_ids,
                     int L, int block_start, int block_size, float tau, int cache_mode,
                     float* logits, float* conf, int32_t* tok, uint8_t* unmask) {
  if (!ctx) return FDLLM_ERR_ARG;
  if (!ctx->weights_loaded) return fail(ctx, FDLLM_ERR_STATE, "weights are not loaded");
  const fdllm_config& c = ctx->cfg;
  if (!snapshot_ids || !current_ids || !conf || !tok || !unmask)
    return fail(ctx, FDLLM_ERR_ARG, "NULL argument");
  if (L < 1 || L > c.max_seq || block_size < 1 || block_size > kMaxLmRows || block_start < 0 ||
      block_start + block_size > L)
    return fail(ctx, FDLLM_ERR_ARG, "bad L / block range");
  if (std::isnan(tau)) return fail(ctx, FDLLM_ERR_ARG, "tau is NaN");
  if (cache_mode < FDLLM_CACHE_NONE || cache_mode > FDLLM_CACHE_DUAL)
    return fail(ctx, FDLLM_ERR_ARG, "unknown cache_mode");
  for (int i = 0; i < L; ++i)
    if (snapshot_ids[i] < 0 || snapshot_ids[i] >= c.vocab || current_ids[i] < 0 ||
        current_ids[i] >= c.vocab)
      return fail(ctx, FDLLM_ERR_ARG, "token id out of range");
  CK(cudaSetDevice(ctx->device));
  const int B = block_size, s = block_start;
  float* dbg = nullptr;
  if (logits) {
    const size_t need = (size_t)B * c.vocab;
    if (need > ctx->dbg_cap) {
      ctx->dbg = (float*)dalloc(ctx, sizeof(float) * need);
      if (!ctx->dbg) return fail(ctx, FDLLM_ERR_OOM, "debug logits allocation failed");
      ctx->dbg_cap = need;
    }
    dbg = ctx->dbg;
  }
  const bool same = std::memcmp(snapshot_ids, current_ids, sizeof(int32_t) * L) == 0;
  CK(cudaMemsetAsync(ctx->state, 0, sizeof(DecodeState), ctx->stream));
  CK(cudaMemcpyAsync(ctx->x, snapshot_ids, sizeof(int32_t) * L, cudaMemcpyHostToDevice,
                     ctx->stream));
  int rc, n_part = 0;
  if (same || cache_mode == FDLLM_CACHE_NONE) {
    if (!same)
      CK(cudaMemcpyAsync(ctx->x, current_ids, sizeof(int32_t) * L, cudaMemcpyHostToDevice,
                         ctx->stream));
    if ((rc = set_step_params(ctx, 0, s, s, tau))) return rc;
    if ((rc = enqueue_step(ctx, 0, L, L, s, B, tau, dbg, &n_part))) return rc;
  } else {
    if ((rc = set_step_params(ctx, 0, s, s, tau))) return rc;
    if ((rc = forward(ctx, 0, L, L, s, B, nullptr, &n_part))) return rc;
    CK(cudaMemcpyAsync(ctx->x, current_ids, sizeof(int32_t) * L, cudaMemcpyHostToDevice,
                       ctx->stream));
    if (cache_mode == FDLLM_CACHE_DUAL) {
      if ((rc = set_step_params(ctx, s, 0, s, tau))) return rc;
      rc = enqueue_step(ctx, s, B, L, 0, B, tau, dbg, &n_part);
    } else {
      if ((rc = set_step_params(ctx, s, 0, s, tau))) return rc;
      rc = enqueue_step(ctx, s, L - s, L, 0, B, tau, dbg, &n_part);
    }
    if (rc) return rc;
  }
  if ((rc = sync_state(ctx))) return rc;
  CK(cudaMemcpy(conf, ctx->conf, sizeof(float) * B, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(tok, ctx->tok, sizeof(int32_t) * B, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(unmask, ctx->unmask, B, cudaMemcpyDeviceToHost));
  if (logits) CK(cudaMemcpy(logits, dbg, sizeof(float) * B * c.vocab, cudaMemcpyDeviceToHost));
  return FDLLM_OK;
}

int fdllm_selftest_wait_timeout(fdllm_ctx* ctx) {
  if (!ctx) return FDLLM_ERR_ARG;
  CK(cudaSetDevice(ctx->device));
  KL(launch_wait_timeout(ctx->err_dev, ctx->stream));
  return sync_state(ctx);  // DEV_ERR_TIMEOUT -> FDLLM_ERR_TIMEOUT; clears the error word
}

int fdllm_kv_similarity(fdllm_ctx* ctx, const int32_t* ids_a, const int32_t* ids_b, int L,
                        double* cos_out) {
  if (!ctx) return FDLLM_ERR_ARG;
  if (!ctx->weights_loaded) return fail(ctx, FDLLM_ERR_STATE, "weights are not loaded");
  const fdllm_config& c = ctx->cfg;
  if (!ids_a || !ids_b || !cos_out) return fail(ctx, FDLLM_ERR_ARG, "NULL argument");
  if (L < 1 || L > c.max_seq) return fail(ctx, FDLLM_ERR_ARG, "bad L");
  for (int i = 0; i < L; ++i)
    if (ids_a[i] < 0 || ids_a[i] >= c.vocab || ids_b[i] < 0 || ids_b[i] >= c.vocab)
      return fail(ctx, FDLLM_ERR_ARG, "token id out of range");
  CK(cudaSetDevice(ctx->device));
  const size_t kv_bytes = ctx->cap_kv * ctx->esz;
  if (!ctx->kv_snap) {
    ctx->kv_snap = dalloc(ctx, kv_bytes);
    ctx->kv_cos = (double*)dalloc(ctx, sizeof(double) * 2 * c.n_layers * c.max_seq);
    if (!ctx->kv_snap || !ctx->kv_cos)
      return fail(ctx, FDLLM_ERR_OOM, "similarity scratch allocation failed");
  }
  // a full forward over each sequence writes the K/V of every position
  int rc, n_part = 0;
  CK(cudaMemsetAsync(ctx->state, 0, sizeof(DecodeState), ctx->stream));
  CK(cudaMemcpyAsync(ctx->x, ids_a, sizeof(int32_t) * L, cudaMemcpyHostToDevice, ctx->stream));
  if ((rc = set_step_params(ctx, 0, 0, 0, 1.0f))) return rc;
  if ((rc = forward(ctx, 0, L, L, 0, 1, nullptr, &n_part))) return rc;
  CK(cudaMemcpyAsync(ctx->kv_snap, ctx->kv_pool, kv_bytes, cudaMemcpyDeviceToDevice, ctx->stream));
  CK(cudaMemcpyAsync(ctx->x, ids_b, sizeof(int32_t) * L, cudaMemcpyHostToDevice, ctx->stream));
  if ((rc = forward(ctx, 0, L, L, 0, 1, nullptr, &n_part))) return rc;
  KL(launch_kv_cosine(ctx->kv_snap, ctx->kv_pool, ctx->page_table, ctx->n_pages, ctx->kv_planes,
                      c.n_layers, c.n_kv_heads, c.head_dim, ctx->f32 ? 1 : 0, L, ctx->kv_cos,
                      ctx->stream));
  if ((rc = sync_state(ctx))) return rc;
  CK(cudaMemcpy(cos_out, ctx->kv_cos, sizeof(double) * 2 * c.n_layers * L,
                cudaMemcpyDeviceToHost));
  return FDLLM_OK;
}

int fdllm_read_kv(fdllm_ctx* ctx, int layer, int pos0, int n, float* k_out, float* v_out) {
  if (!ctx) return FDLLM_ERR_ARG;
  const fdllm_config& c = ctx->cfg;
  if (layer < 0 || layer >= c.n_layers || pos0 < 0 || n < 1 || pos0 + n > c.max_seq || !k_out ||
      !v_out)
    return fail(ctx, FDLLM_ERR_ARG, "bad layer / position range");
  CK(cudaSetDevice(ctx->device));
  CK(cudaStreamSynchronize(ctx->stream));
  const int Hkv = c.n_kv_heads, hd = c.head_dim;
  const int P = ctx->kv_planes;
  const size_t page_elems = (size_t)P * Hkv * KV_PAGE * hd;
  std::vector<int> pt(ctx->n_pages);
  CK(cudaMemcpy(pt.data(), ctx->page_table, sizeof(int) * pt.size(), cudaMemcpyDeviceToHost));
  std::vector<uint8_t> page(page_elems * ctx->esz);
  int cur = -1;
  for (int i = 0; i < n; ++i) {
    const int pos = pos0 + i;
    const int pg = pt[pos / KV_PAGE], slot = pos % KV_PAGE;
    if (pg != cur) {
      const size_t off = ((size_t)layer * ctx->n_pages + pg) * page_elems * ctx->esz;
      CK(cudaMemcpy(page.data(), (uint8_t*)ctx->kv_pool + off, page.size(),
                    cudaMemcpyDeviceToHost));
      cur = pg;
    }
    auto elem = [&](int plane, int hh, int dd) -> float {
      const size_t e = (((size_t)plane * Hkv + hh) * KV_PAGE + slot) * hd + dd;
      float val;
      if (ctx->f32) {
        std::memcpy(&val, page.data() + e * 4, 4);
        return val;
      }
      uint16_t raw;
      std::memcpy(&raw, page.data() + e * 2, 2);
      __half_raw hr;  // fp16 K and V terms
      hr.x = raw;
      return __half2float(__half(hr));
    };
    for (int hh = 0; hh < Hkv; ++hh)
      for (int dd = 0; dd < hd; ++dd) {
        const size_t o = ((size_t)i * Hkv + hh) * hd + dd;
        if (ctx->f32) {
          k_out[o] = elem(0, hh, dd);
          v_out[o] = elem(1, hh, dd);
        } else {  // two-term: the stored value is hi + lo
          k_out[o] = elem(0, hh, dd) + elem(1, hh, dd);
          v_out[o] = elem(2, hh, dd) + elem(3, hh, dd);
        }
      }
  }
  return FDLLM_OK;
}

}  // extern "C"

namespace {

// fdllm_gemm (operand_f16 false: bf16 operands) and fdllm_gemm_f16 (true:
// the decoder's fp16 operands, bf16 model only).
int gemm_entry(fdllm_ctx* ctx, const void* w_dev, const void* x_dev, float* y_dev, int N, int M,
               int K, int splits, int accumulate, bool operand_f16) {
  if (!ctx) return FDLLM_ERR_ARG;
  if (operand_f16 && !ctx->tc)
    return fail(ctx, FDLLM_ERR_ARG, "fp16 operands need the bf16 model's tensor-core path");
  if (!w_dev || !x_dev || !y_dev || N < 1 || M < 1 || K < 1)
    return fail(ctx, FDLLM_ERR_ARG, "bad GEMM arguments");
  if (ctx->tc && (K % 64 || ((uintptr_t)w_dev | (uintptr_t)x_dev) % 16))
    return fail(ctx, FDLLM_ERR_ARG, "bf16 GEMM needs K % 64 == 0 and 16-byte aligned operands");
  if (splits < 0 || (splits > 0 && !ctx->tc))
    return fail(ctx, FDLLM_ERR_ARG, "bad split count");
  CK(cudaSetDevice(ctx->device));
  const bool pair = use_pair_gemm(ctx, N, M, false);
  GemmShape gs = plan_gemm(ctx, N, M, K, true, false, pair);
  if (splits > 0) {
    if (splits > gs.kb_total) return fail(ctx, FDLLM_ERR_ARG, "more splits than K blocks");
    gs.splits = splits;
    if (pair) {
      gs.units = gs.n_tiles / 2 * gs.n_tt * splits;
      gs.grid = 2 * std::min(gs.units, ctx->tc2_pairs);
    } else {
      gs.units = gs.n_tiles * gs.n_tt * splits;
      gs.grid = std::min(gs.units, ctx->num_sms);
    }
    if ((size_t)gs.n_tiles * gs.n_tt * splits * (gs.nt / 2) * 128 * sizeof(float) >
        kWorkspaceBytes)
      return fail(ctx, FDLLM_ERR_ARG, "split workspace too large");
  }
  if (gs.n_tiles * gs.n_tt > ctx->n_counters)
    return fail(ctx, FDLLM_ERR_ARG, "GEMM too large for the counter buffer");
  EpiParams ep = epi_base(ctx, accumulate ? EPI_RESID : EPI_STORE);
  ep.N = N;
  ep.M = M;
  ep.out = y_dev;
  ep.ld_out = N;
  ep.cap_out = (size_t)M * N;
  ep.h = y_dev;
  ep.cap_h = (size_t)M * N;
  ep.act_f32 = ctx->f32;
  {
    ProfScope ps(ctx, "gemm.check",
                 (double)N * K * ctx->esz + 2.0 * M * K * ctx->esz + 4.0 * M * N,
                 2.0 * (ctx->tc ? 2 : 1) * M * N * K);
    if (ctx->tc) {
      CUtensorMap wm, xm;
      gs.f16 = operand_f16 ? 1 : 0;  // bf16 or fp16 operands (see the header)
      if (!make_map(ctx, &wm, w_dev, N, K, 128, operand_f16) ||
          !make_map(ctx, &xm, x_dev, pair_rows(M), K, pair ? 128 : gs.nt, operand_f16))
        return fail(ctx, FDLLM_ERR_CUDA, "cuTensorMapEncodeTiled failed");
      GemmScratch sc{ctx->ws, ctx->counters, ctx->err_dev, kWorkspaceBytes / sizeof(float),
                     ctx->n_counters};
      if (pair)
        KL(launch_gemm_tc2(&wm, &xm, gs, ep, sc, ctx->stream));
      else
        KL(launch_gemm_tc(&wm, &xm, gs, ep, sc, ctx->stream));
    } else {
      KL(launch_gemm_simt((const float*)w_dev, (const float*)x_dev, 0, K, gs, ep, ctx->stream));
    }
  }
  return sync_state(ctx);
}

}  // namespace

extern "C" {

int fdllm_gemm(fdllm_ctx* ctx, const void* w_dev, const void* x_dev, float* y_dev, int N, int M,
               int K, int splits, int accumulate) {
  return gemm_entry(ctx, w_dev, x_dev, y_dev, N, M, K, splits, accumulate, false);
}

int fdllm_gemm_f16(fdllm_ctx* ctx, const void* w_dev, const void* x_dev, float* y_dev, int N,
                   int M, int K, int splits, int accumulate) {
  return gemm_entry(ctx, w_dev, x_dev, y_dev, N, M, K, splits, accumulate, true);
}

int fdllm_attention(fdllm_ctx* ctx, const void* q_dev, void* o_dev, int layer, int M, int L) {
  if (!ctx) return FDLLM_ERR_ARG;
  const fdllm_config& c = ctx->cfg;
  if (!q_dev || !o_dev || layer < 0 || layer >= c.n_layers || M < 1 || L < 1 || L > c.max_seq)
    return fail(ctx, FDLLM_ERR_ARG, "bad attention arguments");
  CK(cudaSetDevice(ctx->device));
  int rc = run_attention(ctx, layer, M, L, q_dev, o_dev);
  if (rc) return rc;
  return sync_state(ctx);
}

int fdllm_profile_enable(fdllm_ctx* ctx, int enable) {
  if (!ctx) return FDLLM_ERR_ARG;
  if (ctx->stream) cudaStreamSynchronize(ctx->stream);
  prof_harvest(ctx);
  ctx->prof = enable != 0;
  if (ctx->prof) ctx->prof_stats.clear();
  return FDLLM_OK;
}

int fdllm_profile_read(fdllm_ctx* ctx, fdllm_kernel_stat* out, int max_stats, int* n_stats) {
  if (!ctx || !n_stats || (max_stats > 0 && !out)) return FDLLM_ERR_ARG;
  if (ctx->stream) cudaStreamSynchronize(ctx->stream);
  prof_harvest(ctx);
  *n_stats = (int)ctx->prof_stats.size();
  for (int i = 0; i < max_stats && i < *n_stats; ++i) out[i] = ctx->prof_stats[i];
  return FDLLM_OK;
}

const char* fdllm_last_error(const fdllm_ctx* ctx) {
  return ctx ? ctx->err.c_str() : g_create_error.c_str();
}

int64_t fdllm_launch_count(fdllm_ctx* ctx, int reset) {
  if (!ctx) return 0;
  const int64_t n = ctx->launches;
  if (reset) ctx->launches = 0;
  return n;
}

int fdllm_destroy(fdllm_ctx* ctx) {
  if (!ctx) return FDLLM_OK;
  cudaSetDevice(ctx->device);
  if (ctx->stream) cudaStreamSynchronize(ctx->stream);
  prof_harvest(ctx);
  for (cudaEvent_t e : ctx->ev_pool) cudaEventDestroy(e);
  for (auto& kv : ctx->step_graphs) cudaGraphExecDestroy(kv.second.exec);
  ctx->step_graphs.clear();
  dfree_all(ctx);
  if (ctx->state_host) cudaFreeHost(ctx->state_host);
  if (ctx->states_host) cudaFreeHost(ctx->states_host);
  if (ctx->btab_host) cudaFreeHost(ctx->btab_host);
  if (ctx->err_host) cudaFreeHost(ctx->err_host);
  if (ctx->sp_host) cudaFreeHost(ctx->sp_host);
  if (ctx->own_stream && ctx->stream) cudaStreamDestroy(ctx->stream);
  delete ctx;
  return FDLLM_OK;
}

}  // extern "C"
