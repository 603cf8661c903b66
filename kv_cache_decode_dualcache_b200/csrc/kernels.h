// Internal interface between the host orchestration (api.cu) and the kernel
// translation units.  Not part of the public C ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace fd {

enum EpiKind : int {
  EPI_STORE = 0,   // out[t, n] = y (float)
  EPI_QKV = 1,     // RoPE on q and k; q -> q buffer, k and v -> KV cache pages
  EPI_RESID = 2,   // h[t, n] += y  (float residual stream)
  EPI_SWIGLU = 3,  // 64-row gate/up groups: f[t, j] = silu(gate) * up
  EPI_LMHEAD = 4,  // online max / argmax / sum-exp over vocab tiles
};

// Per-step scalars read by the kernels from device memory, so that one
// captured CUDA graph serves every block of a generation: the host writes
// them (one small copy) before each replay.
struct StepParams {
  int r0;            // absolute position of the forward's first row
  int lm0;           // first LM-head row within the forward
  int s;             // block start position (unmask target)
  float tau;         // confidence threshold
  int fixed_k;       // > 0: unmask the fixed_k most confident masked positions instead
};

// Batched forward (rows of several sequences in one pass): the sequence
// slot and absolute position of every row of the forward.  Slot q's token ids
// live at x[q * seq_stride ..], its K/V pages at page_table[q * pages_per_seq ..].
// Every sequence's rows start at a multiple of 32 forward rows and are padded
// to one (pos = -1), so each 32-row chunk belongs to one sequence and holds
// consecutive positions: RowChunk {first position, slot, real rows}.
struct RowInfo {
  int pos;
  int seq;
};
struct RowChunk {
  int pos0, seq, n, pad;
};

// Everything a GEMM epilogue needs.  Token index t is the row within the
// GEMM's activation operand (0..M-1); feature index n is the output column.
struct EpiParams {
  int kind;
  int N;             // output features (rows of the weight matrix)
  int M;             // valid token rows
  int act_f32;       // 1: activations / outputs are float (fp32 model); 0: two-term fp16
  // EPI_STORE
  float* out;
  int ld_out;
  // EPI_QKV
  void* q_out;       // fp32: [M, H*hd]; bf16 model: fp16 hi plane then lo plane, each [rows, H*hd]
  size_t q_plane;    // elements per q plane (bf16 model)
  void* kv_pool;     // [layers][pages][planes][Hkv][KV_PAGE][hd]; planes: fp32 K,V;
                     // bf16 model: K hi, K lo, V hi, V lo (all fp16)
  int kv_planes;
  const int* page_table;
  int n_pages;
  int layer;
  int pos0;          // absolute position of token row 0
  const float2* rope;  // [max_seq][hd/2] (cos, sin)
  int n_heads, n_kv_heads, head_dim;
  // EPI_RESID
  float* h;          // [M, N]
  // EPI_SWIGLU
  void* f_out;       // [M, N/2] (fp32) or two-term fp16 pair rows (bf16 model)
  // EPI_LMHEAD
  float logit_scale;
  int mask_id;
  float* lm_part;    // [n_part][M] of (m, s, arg) triples
  float* dbg_logits; // optional [M, N] float logits (mask id included)
  const StepParams* sp;  // when set, pos0 = sp->r0 (device-side step scalars)
  const RowInfo* rows;   // batched forward: row t has position rows[t].pos in slot rows[t].seq
                         // (NULL: one sequence, row t at position pos0 + t)
  const RowChunk* chunks;  // batched forward: the 32-row chunks of rows
  int pages_per_seq;     // batched forward: page-table entries per slot
  // Capacities (elements) of the output buffers, used only by builds with
  // FDLLM_CHECKS, where every store is bounds-checked and a violation is
  // recorded in check[0..3] (count, code, index, aux) instead of performed.
  size_t cap_out, cap_h, cap_q, cap_kv, cap_f, cap_dbg, cap_lm;
  int* check;
};

// Bookkeeping shared by both GEMM implementations.
struct GemmShape {
  int N, M, K;
  int nt;            // token tile width
  int splits;        // K splits (deterministic reduction when > 1)
  int n_tiles;       // ceil(N / 128)
  int n_tt;          // ceil(M / nt)
  int kb_total;      // ceil(K / 64)
  int units;         // n_tiles * n_tt * splits
  int grid;          // CTAs launched
  int f16;           // tcgen05 operands: 1 = fp16 (the decoder), 0 = bf16
  int kc;            // K blocks per TMEM accumulation chain (tcgen05 GEMM)
};

struct GemmScratch {
  float* ws;         // split-K partial tiles
  int* counters;     // per tile arrival counters (self-resetting)
  int* err;          // device error word
  size_t ws_elems;   // capacities (checked in FDLLM_CHECKS builds)
  int n_counters;
};

// Tile / split plan of the tcgen05 GEMM for N output features, M tokens and
// reduction length K on a GPU with num_sms SMs: token tile of nt <= max_nt
// rows (nt/2 tokens of two-term activations), K split chosen to balance the
// per-CTA K blocks over the persistent grid, within ws_bytes of split-K
// workspace.  The LM-head epilogue needs max_nt <= 128.
GemmShape plan_gemm_tc(int num_sms, int N, int M, int K, bool allow_split, size_t ws_bytes,
                       int max_nt = 256);

// Launch with the programmatic stream-serialization attribute (when pdl).
template <typename... KArgs, typename... Args>
cudaError_t launch_k(bool pdl, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                     cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Sets the dynamic shared-memory limits of every kernel (call once per
// device before any launch, outside stream capture).
cudaError_t init_kernel_attributes();

// Launchers (return cudaError_t of the launch).
// bf16 model: activations in two-term pair rows, token tiles of nt/2 tokens;
// operand type fp16 or bf16 by gs.f16.
cudaError_t launch_gemm_tc(const CUtensorMap* w_map, const CUtensorMap* act_map,
                           const GemmShape& gs, const EpiParams& ep, const GemmScratch& sc,
                           cudaStream_t st, bool pdl = false);
// fp32 model: plain [M, K] activations starting at row act_row0.
cudaError_t launch_gemm_simt(const float* w, const float* act, int act_row0, int K,
                             const GemmShape& gs, const EpiParams& ep, cudaStream_t st,
                             bool pdl = false);
int gemm_tc_smem_bytes(int nt);

// The same GEMM on pairs of SMs (gemm_tc2.cu, tcgen05 cta_group::2):
// 256-feature x 128-token output tiles, any epilogue but the LM head.  gs comes from plan_gemm_tc2; act_map has 128-row boxes (each CTA
// of a pair loads half of a 256-row token tile).
GemmShape plan_gemm_tc2(int max_pairs, int N, int M, int K, size_t ws_bytes);
cudaError_t launch_gemm_tc2(const CUtensorMap* w_map, const CUtensorMap* act_map,
                            const GemmShape& gs, const EpiParams& ep, const GemmScratch& sc,
                            cudaStream_t st, bool pdl = false);
int gemm_tc2_smem_bytes();
// Pairs of CTAs that can be resident at once (0 if none or on error).
int gemm_tc2_max_pairs();

// Batched attention: CTA x-index i covers query rows [r0, r0 + rows) (rows
// of (position, head-in-group) pairs) of one sequence's segment, whose
// positions are rows q0 .. q0 + m - 1 of the forward; its keys are [0, L) of
// slot seq.
struct AttnTile {
  int q0, m, r0, L, seq;
  int pad[3];
};

struct AttnParams {
  const void* q;       // [M, H, hd] (fp32) or fp16 hi/lo planes of [M, H, hd] (bf16 model)
  size_t q_plane;      // elements per q plane (bf16 model)
  void* o;             // [M, H*hd] (fp32) or two-term fp16 pair rows (bf16 model)
  const void* kv_pool;
  int kv_planes;
  const int* page_table;
  int n_pages, layer;
  int M;               // query positions
  int L;               // keys [0, L)
  int n_heads, n_kv_heads, head_dim;
  int n_split;         // key splits, <= 8: one thread-block cluster per (row tile, KV head)
  int keys_per_split;  // multiple of 64
  const AttnTile* tiles;  // batched forward: one entry per CTA along x (NULL: one sequence)
  int n_tiles;
  int pages_per_seq;
  int* err;               // device error word (a bounded wait that runs out)
};

// kvmap: the 2-D K/V pool map of launch_attn_tc (boxes {64, 64}); the K/V
// tiles are staged by TMA, the queries gathered with cp.async.
cudaError_t launch_attn_mma(const CUtensorMap* kvmap, const AttnParams& p, cudaStream_t st,
                            bool pdl = false);
// tcgen05 + TMA attention for many query rows (see attn_tc.cu); with
// p.tiles, one CTA per table entry: r0 / rep = the tile's first position in
// its segment, 128 / rep positions per tile.  qmap: 3-D
// map {head_dim, n_heads, 2 * q_lo_rows} over the q hi plane followed by the
// lo plane (boxes {64, rep, 128 / rep}); kvmap: 2-D map {head_dim, rows} over
// the K/V pool, one row per (layer, page, plane, KV head, slot) (boxes
// {64, 64}); both with the 128-byte swizzle.
bool attn_tc_supported(const AttnParams& p);
cudaError_t launch_attn_tc(const CUtensorMap* qmap, const CUtensorMap* kvmap, const AttnParams& p,
                           int q_lo_rows, int* err, cudaStream_t st, bool pdl = false);
cudaError_t attn_tc_init_attributes();
// tcgen05 + TMA attention of block queries (see attn_blk.cu).  One
// sequence: at most 64 query positions, n_split <= 8 key splits of
// keys_per_split (a multiple of 128) keys each, one thread-block cluster per
// (query-row tile, KV head).  Batched forward (p.tiles): one CTA per table
// entry of 64 query rows, n_split = 1, keys_per_split >= every segment's L.
// kvmap as for launch_attn_tc.
bool attn_blk_supported(const AttnParams& p);
cudaError_t launch_attn_blk(const CUtensorMap* kvmap, const AttnParams& p, cudaStream_t st,
                            bool pdl = false);
cudaError_t attn_blk_init_attributes();
// Query rows per CTA of launch_attn_mma for M query positions (16, 32 or 64).
int attn_rows_per_cta(int M, int n_heads, int n_kv_heads);
cudaError_t launch_attn_simt(const AttnParams& p, cudaStream_t st, bool pdl = false);

// Row sources of the norm kernels in a batched forward (all NULL: one
// sequence).  rows: the embedding gather reads x[rows[i].seq * seq_stride +
// rows[i].pos]; src: RMSNorm output row i reads h row src[i].
struct RowMap {
  const RowInfo* rows;
  int seq_stride;
  const int* src;
};

// h[i] = embed[x[r0+i]]; a[i] = RMSNorm(h[i]) * g, i in [0, M).  With sp,
// r0 = sp->r0.  bf16 model: bf16 embedding rows, a in two-term fp16 pair rows.
cudaError_t launch_embed_rmsnorm(const int* x, int r0, int M, const void* embed, int d,
                                 int vocab, const float* g, float eps, float* h, void* a,
                                 int f32, int* err, const StepParams* sp, cudaStream_t st,
                                 bool pdl = false, RowMap rm = RowMap{nullptr, 0, nullptr});
// a[i] = RMSNorm(h[h_row0 + i]) * g, i in [0, M).  bf16 model: two-term fp16
// pair rows.
// With sp and rows_from_lm0, h_row0 = sp->lm0.
cudaError_t launch_rmsnorm(const float* h, int h_row0, int M, int d, const float* g, float eps,
                           void* a, int f32, const StepParams* sp, bool rows_from_lm0,
                           cudaStream_t st, bool pdl = false,
                           RowMap rm = RowMap{nullptr, 0, nullptr});

// ------------------------------------------------ block-step chain kernel
// One launch runs a program of phases of the DualCache block step (bf16
// model, at most 32 block tokens), see chain.cu.
enum ChainPhaseType : int {
  CH_GEMM = 0,        // tcgen05 GEMM, one token tile, fused epilogue ep
  CH_NORM = 1,        // a = RMSNorm(h) * gain over the block rows
  CH_EMBED_NORM = 2,  // h = E[x[r0 + row]], then as CH_NORM
};
constexpr int CHAIN_NORM_GROUPS = 8;  // d_model: a multiple of 512, at most 8 * 512
constexpr int CHAIN_DONE_STRIDE = 32;  // ints between phase counters (one 128-byte line each)

constexpr int CHAIN_MAX_PHASES = 6;

struct ChainPhase {
  CUtensorMap wmap;         // weight map (GEMM)
  CUtensorMap amap;         // activation map, 64-row token tile (GEMM)
  int type;
  int N, K, kb_total, n_tiles, splits, units, rot, kc;
  const float* gain;        // norm gains (NORM, EMBED_NORM)
  int resid_splits;         // NORM: split partials of the preceding residual GEMM to add
                            // into h first (its EPI_RESID epilogue only stores partials)
  EpiParams ep;             // GEMM epilogue (ep.M = block rows)
};

// Passed by value (kernel parameter space: read-only, so the compiler never
// has to re-read a phase field after the kernel's own global stores); larger
// than the classic 4 KB parameter limit, which CUDA 12.1+ lifts to 32 KB.
struct ChainArgs {
  ChainPhase ph[CHAIN_MAX_PHASES];
  int n_phases;
  int* done;                // CTAs finished per phase, phase p at done[p * CHAIN_DONE_STRIDE];
                            // zero at launch
  int* gabort;              // grid-wide abort word; zero at launch
  int M;                    // block rows (<= 32)
  int d, vocab;
  float eps;
  const int* x;             // token ids (EMBED_NORM: rows x[sp->r0 + row])
  const void* embed;        // bf16 [vocab, d]
  float* h;                 // residual stream [M, d]
  void* a;                  // normed activations, two-term fp16 pair rows
  const StepParams* sp;
  GemmScratch sc;           // split-K partials and per-tile counters
  int* rowcnt;              // NORM phases: per-row group arrivals, phase p at rowcnt[p * 32];
                            // zero at launch
  float* norm_ss;           // NORM phases: partial sums of squares [32][CHAIN_NORM_GROUPS]
  int* next;                // GEMM phases: unit claim counters, phase p at next[p *
                            // CHAIN_DONE_STRIDE]; zero at launch
};
static_assert(sizeof(ChainArgs) <= 32764, "kernel parameters are limited to 32 KB");

// Launch of grid CTAs (one per SM): cooperative, or with after_kernel a
// programmatic dependent launch behind the preceding kernel of the stream
// (the program must then begin with a GEMM phase, whose activation loads
// wait for that kernel).
cudaError_t launch_chain(const ChainArgs& args, int grid, cudaStream_t st, bool after_kernel);
cudaError_t chain_init_attributes();
int chain_smem_bytes();

struct DecodeState {
  int remaining;     // masked positions left in the block after the step
  int unmasked;      // positions unmasked by the step
  int steps;         // steps taken so far (incremented by every select)
  int pad;
};

// A bounded device wait that runs out (see fdllm_selftest_wait_timeout).
cudaError_t launch_wait_timeout(int* err, cudaStream_t st);

// out[(layer * 2 + kv) * L + pos], pos < L: cosine of K (kv = 0) / V (kv = 1)
// of cache a and cache b (same paged layout and page table), float64.
cudaError_t launch_kv_cosine(const void* a, const void* b, const int* page_table, int n_pages,
                             int planes, int n_layers, int Hkv, int hd, int f32, int L,
                             double* out, cudaStream_t st);

// Merge LM-head partials into conf/tok for n rows and, when select != 0,
// apply the threshold-or-fallback unmask rule to x[s .. s+n).
// With sp, s = sp->s and tau = sp->tau.
cudaError_t launch_merge_select(const float* lm_part, int n_part, int n, int* x, int s,
                                int mask_id, float tau, int select, float* conf, int* tok,
                                uint8_t* unmask, DecodeState* state, const StepParams* sp,
                                cudaStream_t st, bool pdl = false);

// Batched decode: LM-head rows [k0, k0 + n) belong to the block [s, s + n)
// of the sequence in slot seq.
struct SelectSeg {
  int k0, n, seq, s;
};

// merge + select per sequence: block i of the grid handles segs[i] (n <= 256)
// with the partials of all m_lm LM-head rows, the slot's token ids at
// x + seq * seq_stride and its state states[seq]; conf / tok / unmask are
// indexed by LM-head row.  fixed_k > 0 selects the fixed-count rule.
cudaError_t launch_merge_select_seg(const float* lm_part, int n_part, int m_lm,
                                    const SelectSeg* segs, int n_segs, int* x, int seq_stride,
                                    int mask_id, float tau, int fixed_k, float* conf, int* tok,
                                    uint8_t* unmask, DecodeState* states, cudaStream_t st,
                                    bool pdl = false);

cudaError_t launch_fill_masked(int* x, int from, int to, int mask_id, cudaStream_t st,
                               bool pdl = false);
cudaError_t launch_check_prompt(const int* x, int n, int vocab, int mask_id, int* err,
                                cudaStream_t st, bool pdl = false);
// In place: n bf16 values -> fp16 (round to nearest even).  A value outside
// the fp16 range sets DEV_ERR_RANGE in *err; values the conversion changes
// are counted into *inexact (may be NULL).
cudaError_t launch_bf16_to_f16(void* p, size_t n, int* err, unsigned long long* inexact,
                               cudaStream_t st);

}  // namespace fd
