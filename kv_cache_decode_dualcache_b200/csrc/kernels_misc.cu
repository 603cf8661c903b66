// CUDA-core kernels: embedding + RMSNorm, RMSNorm, the LM-head partial
// merge fused with the threshold/unmask/scatter step, and the float32 GEMM
// and attention of the fp32 model.
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"

namespace fd {

namespace {

constexpr int RMS_VPT = 32;   // values per thread: d_model up to 8192 with 256 threads

// Deterministic block sum (fixed tree) for blockDim.x a multiple of 32.
FD_DEV float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.0f;
  for (int i = 0; i < nw; ++i) t += red[i];
  return t;
}

FD_DEV float block_max(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = -INFINITY;
  for (int i = 0; i < nw; ++i) t = fmaxf(t, red[i]);
  return t;
}

// ------------------------------------------------------------------ RMSNorm
// a[row] = h[h_row0 + row] / sqrt(mean(h^2) + eps) * g; one CTA per row.  With
// `x` given, h[row] is first gathered from the embedding table at token
// x[r0 + row].  fp32 model: a is [M, d] float; bf16 model (bf16 embedding
// rows): a is two-term fp16 in pair rows.
template <typename T>
__global__ void __launch_bounds__(256) rmsnorm_kernel(const int* __restrict__ x, int r0,
                                                      const T* __restrict__ embed, int vocab,
                                                      float* __restrict__ h, int h_row0, int d,
                                                      const float* __restrict__ g, float eps,
                                                      void* __restrict__ a, int* err,
                                                      const StepParams* sp, int rows_from_lm0,
                                                      RowMap rm) {
  // The row stays in registers (d <= 256 * RMS_VPT): every load is issued
  // before any store.
  constexpr int VPT = RMS_VPT;
  __shared__ float red[32];
  pdl_trigger();
  pdl_wait();
  const int row = blockIdx.x;
  if (sp) {
    if (x) r0 = sp->r0;
    if (rows_from_lm0) h_row0 = sp->lm0;
  }
  // batched forward: the output row's h row and token come from the row map
  float* hr = h + (size_t)(rm.src ? rm.src[row] : h_row0 + row) * d;
  float v[VPT];
  if (x) {
    // (a padding row of a batched forward, pos < 0, takes token 0)
    const int rpos = rm.rows ? rm.rows[row].pos : 0;
    int tok = rm.rows ? (rpos < 0 ? 0 : x[(size_t)rm.rows[row].seq * rm.seq_stride + rpos])
                      : x[r0 + row];
    if (tok < 0 || tok >= vocab) {
      if (threadIdx.x == 0) atomicOr(err, DEV_ERR_TOKEN);
      tok = 0;
    }
    const T* er = embed + (size_t)tok * d;
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      const int j = threadIdx.x + k * 256;
      v[k] = j < d ? to_f(er[j]) : 0.0f;
    }
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      const int j = threadIdx.x + k * 256;
      if (j < d) hr[j] = v[k];
    }
  } else {
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      const int j = threadIdx.x + k * 256;
      v[k] = j < d ? hr[j] : 0.0f;
    }
  }
  float ss = 0.0f;
#pragma unroll
  for (int k = 0; k < VPT; ++k) ss += v[k] * v[k];
  ss = block_sum(ss, red);
  const float inv = 1.0f / sqrtf(ss / (float)d + eps);
  if (std::is_same<T, float>::value) {
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      const int j = threadIdx.x + k * 256;
      if (j < d) reinterpret_cast<float*>(a)[(size_t)row * d + j] = v[k] * inv * __ldg(&g[j]);
    }
  } else {
    __half* ab = reinterpret_cast<__half*>(a);
    const size_t r_hi = (size_t)pair_row(row) * d, r_lo = r_hi + (size_t)PAIR_LO * d;
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      const int j = threadIdx.x + k * 256;
      if (j < d) {
        __half hi, lo;
        split_f16(v[k] * inv * __ldg(&g[j]), hi, lo);
        ab[r_hi + j] = hi;
        ab[r_lo + j] = lo;
      }
    }
  }
}

// bf16 model with d % 4 == 0: as rmsnorm_kernel<__nv_bfloat16>, four
// consecutive features per thread and access (16-byte h loads and stores,
// 8-byte embedding loads and two-term stores).
__global__ void __launch_bounds__(256) rmsnorm_v4_kernel(const int* __restrict__ x, int r0,
                                                         const __nv_bfloat16* __restrict__ embed,
                                                         int vocab, float* __restrict__ h,
                                                         int h_row0, int d,
                                                         const float* __restrict__ g, float eps,
                                                         __half* __restrict__ a, int* err,
                                                         const StepParams* sp, int rows_from_lm0,
                                                         RowMap rm) {
  constexpr int V4 = RMS_VPT / 4;
  __shared__ float red[32];
  pdl_trigger();
  pdl_wait();
  const int row = blockIdx.x;
  if (sp) {
    if (x) r0 = sp->r0;
    if (rows_from_lm0) h_row0 = sp->lm0;
  }
  // batched forward: the output row's h row and token come from the row map
  float* hr = h + (size_t)(rm.src ? rm.src[row] : h_row0 + row) * d;
  float4 v[V4];
  if (x) {
    // (a padding row of a batched forward, pos < 0, takes token 0)
    const int rpos = rm.rows ? rm.rows[row].pos : 0;
    int tok = rm.rows ? (rpos < 0 ? 0 : x[(size_t)rm.rows[row].seq * rm.seq_stride + rpos])
                      : x[r0 + row];
    if (tok < 0 || tok >= vocab) {
      if (threadIdx.x == 0) atomicOr(err, DEV_ERR_TOKEN);
      tok = 0;
    }
    const __nv_bfloat16* er = embed + (size_t)tok * d;
#pragma unroll
    for (int k = 0; k < V4; ++k) {
      const int j = (threadIdx.x + k * 256) * 4;
      if (j < d) {
        const uint2 raw = __ldg(reinterpret_cast<const uint2*>(er + j));
        const __nv_bfloat162 p0 = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
        const __nv_bfloat162 p1 = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
        v[k] = make_float4(__low2float(p0), __high2float(p0), __low2float(p1), __high2float(p1));
      } else {
        v[k] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      }
    }
#pragma unroll
    for (int k = 0; k < V4; ++k) {
      const int j = (threadIdx.x + k * 256) * 4;
      if (j < d) *reinterpret_cast<float4*>(hr + j) = v[k];
    }
  } else {
#pragma unroll
    for (int k = 0; k < V4; ++k) {
      const int j = (threadIdx.x + k * 256) * 4;
      v[k] = j < d ? *reinterpret_cast<const float4*>(hr + j) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
  }
  float ss = 0.0f;
#pragma unroll
  for (int k = 0; k < V4; ++k) ss += v[k].x * v[k].x + v[k].y * v[k].y + v[k].z * v[k].z + v[k].w * v[k].w;
  ss = block_sum(ss, red);
  const float inv = 1.0f / sqrtf(ss / (float)d + eps);
  const size_t r_hi = (size_t)pair_row(row) * d, r_lo = r_hi + (size_t)PAIR_LO * d;
#pragma unroll
  for (int k = 0; k < V4; ++k) {
    const int j = (threadIdx.x + k * 256) * 4;
    if (j < d) {
      const float4 gn = __ldg(reinterpret_cast<const float4*>(g + j));
      __half h0, l0, h1, l1, h2, l2, h3, l3;
      split_f16(v[k].x * inv * gn.x, h0, l0);
      split_f16(v[k].y * inv * gn.y, h1, l1);
      split_f16(v[k].z * inv * gn.z, h2, l2);
      split_f16(v[k].w * inv * gn.w, h3, l3);
      __half2 hh[2] = {__halves2half2(h0, h1), __halves2half2(h2, h3)};
      __half2 ll[2] = {__halves2half2(l0, l1), __halves2half2(l2, l3)};
      *reinterpret_cast<uint2*>(a + r_hi + j) = *reinterpret_cast<const uint2*>(hh);
      *reinterpret_cast<uint2*>(a + r_lo + j) = *reinterpret_cast<const uint2*>(ll);
    }
  }
}

// ------------------------------------------------------- failure path
// One wait that nothing completes (an mbarrier expecting an arrival that no
// thread makes), through the same bounded mbar_wait the tcgen05 kernels use:
// after its limit it records DEV_ERR_TIMEOUT in the error word and returns.
__global__ void wait_timeout_kernel(int* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, err, nullptr);
}

// ------------------------------------------------------- K/V similarity
// out[(layer * 2 + kv) * L + pos] = cosine of the K (kv = 0) or V (kv = 1)
// activations of one position and layer in two caches of the same layout,
// over its n_kv_heads * head_dim values (two-term fp16 terms summed for the
// bf16 model), accumulated in float64 in a fixed order.  One CTA per
// (position, kv, layer).
__global__ void __launch_bounds__(128) kv_cosine_kernel(const void* __restrict__ a,
                                                        const void* __restrict__ b,
                                                        const int* __restrict__ page_table,
                                                        int n_pages, int planes, int Hkv, int hd,
                                                        int f32, int L, double* __restrict__ out) {
  __shared__ double red[3][4];
  const int pos = blockIdx.x, kv = blockIdx.y, layer = blockIdx.z;
  const int page = page_table[pos / KV_PAGE], slot = pos % KV_PAGE;
  const size_t plane_elems = (size_t)Hkv * KV_PAGE * hd;
  const size_t base = ((size_t)layer * n_pages + page) * planes * plane_elems;
  double dot = 0.0, na = 0.0, nb = 0.0;
  for (int i = threadIdx.x; i < Hkv * hd; i += blockDim.x) {
    const int h = i / hd, d = i - h * hd;
    const size_t off = (size_t)h * KV_PAGE * hd + (size_t)slot * hd + d;
    double x, y;
    if (f32) {
      const size_t e = base + (size_t)kv * plane_elems + off;
      x = reinterpret_cast<const float*>(a)[e];
      y = reinterpret_cast<const float*>(b)[e];
    } else {
      const size_t hi = base + (size_t)(2 * kv) * plane_elems + off, lo = hi + plane_elems;
      const __half* ha = reinterpret_cast<const __half*>(a);
      const __half* hb = reinterpret_cast<const __half*>(b);
      x = (double)__half2float(ha[hi]) + (double)__half2float(ha[lo]);
      y = (double)__half2float(hb[hi]) + (double)__half2float(hb[lo]);
    }
    dot += x * y;
    na += x * x;
    nb += y * y;
  }
  for (int o = 16; o > 0; o >>= 1) {
    dot += __shfl_xor_sync(0xffffffffu, dot, o);
    na += __shfl_xor_sync(0xffffffffu, na, o);
    nb += __shfl_xor_sync(0xffffffffu, nb, o);
  }
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    red[0][w] = dot;
    red[1][w] = na;
    red[2][w] = nb;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double s[3];
    for (int q = 0; q < 3; ++q) s[q] = ((red[q][0] + red[q][1]) + red[q][2]) + red[q][3];
    // two zero vectors are identical; a zero and a non-zero one are not alike
    const double den = sqrt(s[1]) * sqrt(s[2]);
    out[((size_t)layer * 2 + kv) * L + pos] =
        den > 0.0 ? s[0] / den : ((s[1] == 0.0 && s[2] == 0.0) ? 1.0 : 0.0);
  }
}

// ------------------------------------------------------- merge + select
// Merge of the LM-head partials of n rows (row t's partial of producer q at
// part[q * stride + t]) into conf / tok, then, when select is set, the
// unmask rule on the block x[s .. s + n): every masked position with
// conf >= tau (or, with fixed_k > 0, the fixed_k most confident masked
// ones), else the single most confident masked position; the chosen
// positions take their argmax token.  One CTA of at least n threads.
FD_DEV void merge_select_body(const SoftmaxState* part, int n_part, int stride, int n, int* x,
                              int s, int mask_id, float tau, int fixed_k, int select,
                              float* conf, int* tok, uint8_t* unmask, DecodeState* state,
                              float* s_conf, int* s_tok, int* s_best) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int t = warp; t < n; t += blockDim.x >> 5) {
    SoftmaxState st = sm_empty();
    for (int q = lane; q < n_part; q += 32) st = sm_merge(st, part[(size_t)q * stride + t]);
    st = warp_sm_merge(st);
    if (lane == 0) {
      // conf = exp(z_max - logsumexp) = 1 / sum exp(z - z_max)
      const float c = (st.s > 0.0f) ? 1.0f / st.s : 0.0f;
      s_conf[t] = c;
      s_tok[t] = st.arg;
      conf[t] = c;
      tok[t] = st.arg;
    }
  }
  __syncthreads();
  if (!select) return;
  const int i = threadIdx.x;
  const bool valid = i < n;
  const bool masked = valid && x[s + i] == mask_id;
  const float ci = valid ? s_conf[i] : 0.0f;
  bool pass = masked && (ci >= tau);
  if (fixed_k > 0) {
    // fixed-count strategy: the fixed_k most confident masked positions,
    // the lower position first among equal confidences (NaN counts as -1)
    const float mine = (ci == ci) ? ci : -1.0f;
    int rank = 0;
    for (int j = 0; j < n; ++j) {
      if (j == i || x[s + j] != mask_id) continue;
      const float cj = (s_conf[j] == s_conf[j]) ? s_conf[j] : -1.0f;
      rank += (cj > mine || (cj == mine && j < i)) ? 1 : 0;
    }
    pass = masked && rank < fixed_k;
  }
  const int n_pass = __syncthreads_count(pass);
  if (threadIdx.x == 0) {
    int best = -1;
    float bc = -INFINITY;
    if (n_pass == 0) {
      for (int j = 0; j < n; ++j) {
        if (x[s + j] != mask_id) continue;
        const float cj = (s_conf[j] == s_conf[j]) ? s_conf[j] : -1.0f;  // NaN last
        if (best < 0 || cj > bc) { best = j; bc = cj; }
      }
    }
    *s_best = best;
  }
  __syncthreads();
  const bool u = pass || (n_pass == 0 && i == *s_best);
  if (valid) unmask[i] = u ? 1 : 0;
  const int n_left = __syncthreads_count(masked && !u);
  const int n_un = __syncthreads_count(u);
  if (u) x[s + i] = s_tok[i];
  if (threadIdx.x == 0) {
    state->remaining = n_left;
    state->unmasked = n_un;
    state->steps += 1;
  }
}

__global__ void merge_select_kernel(const SoftmaxState* part, int n_part, int n, int* x, int s,
                                    int mask_id, float tau, int select, float* conf, int* tok,
                                    uint8_t* unmask, DecodeState* state, const StepParams* sp) {
  __shared__ float s_conf[256];
  __shared__ int s_tok[256];
  __shared__ int s_best;
  pdl_trigger();
  pdl_wait();
  int fixed_k = 0;
  if (sp) {
    s = sp->s;
    tau = sp->tau;
    fixed_k = sp->fixed_k;
  }
  merge_select_body(part, n_part, n, n, x, s, mask_id, tau, fixed_k, select, conf, tok, unmask,
                    state, s_conf, s_tok, &s_best);
}

// Batched decode: CTA i merges and selects the block of segs[i].
__global__ void merge_select_seg_kernel(const SoftmaxState* part, int n_part, int m_lm,
                                        const SelectSeg* segs, int* x, int seq_stride,
                                        int mask_id, float tau, int fixed_k, float* conf,
                                        int* tok, uint8_t* unmask, DecodeState* states) {
  __shared__ float s_conf[256];
  __shared__ int s_tok[256];
  __shared__ int s_best;
  pdl_trigger();
  pdl_wait();
  const SelectSeg sg = segs[blockIdx.x];
  merge_select_body(part + sg.k0, n_part, m_lm, sg.n, x + (size_t)sg.seq * seq_stride, sg.s,
                    mask_id, tau, fixed_k, 1, conf + sg.k0, tok + sg.k0, unmask + sg.k0,
                    states + sg.seq, s_conf, s_tok, &s_best);
}

// In place bf16 -> fp16 (round to nearest even).  Values outside the fp16
// range (and NaN) set DEV_ERR_RANGE; conversions that change the value (bf16
// values below 2^-17 in magnitude, under the fp16 subnormal grid) are counted
// into *inexact, one atomic per warp and iteration that saw any.
__global__ void bf16_to_f16_kernel(uint16_t* p, size_t n, int* err,
                                   unsigned long long* inexact) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  const size_t n_iter = (n + stride - 1) / stride;
  const size_t i0 = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  // every thread runs the same number of iterations, so the ballot below is
  // taken by the full warp
  for (size_t k = 0; k < n_iter; ++k) {
    const size_t i = i0 + k * stride;
    bool changed = false;
    if (i < n) {
      const float v = __uint_as_float((uint32_t)p[i] << 16);
      if (!(fabsf(v) <= 65504.0f)) atomicOr(err, DEV_ERR_RANGE);  // also NaN
      const __half h = __float2half_rn(v);
      changed = __half2float(h) != v && v == v;
      p[i] = __half_as_ushort(h);
    }
    const unsigned b = __ballot_sync(0xffffffffu, changed);
    if (b && (threadIdx.x & 31) == 0 && inexact) atomicAdd(inexact, (unsigned long long)__popc(b));
  }
}

__global__ void fill_kernel(int* x, int from, int to, int v) {
  pdl_trigger();
  pdl_wait();
  const int i = from + blockIdx.x * blockDim.x + threadIdx.x;
  if (i < to) x[i] = v;
}

__global__ void check_prompt_kernel(const int* x, int n, int vocab, int mask_id, int* err) {
  pdl_trigger();
  pdl_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    const int t = x[i];
    if (t < 0 || t >= vocab || t == mask_id) atomicOr(err, DEV_ERR_TOKEN);
  }
}

// ------------------------------------------------------- CUDA-core GEMM
// One CTA computes one 128-feature x 32-token chunk; 128 threads, thread e
// owns feature n0 + e.  Used by the float32 model (float32 FMAs; tensor-core
// tf32 would round the inputs to 10 significant bits).
__global__ void __launch_bounds__(128)
    gemm_simt_kernel(const float* w, const float* act, int act_row0, int K, GemmShape gs,
                     EpiParams ep) {
  __shared__ float ws_[32][129];
  __shared__ float as_[32][33];
  __shared__ float tile[32 * 128];
  __shared__ SoftmaxState lm[32];
  pdl_trigger();
  pdl_wait();
  const int e = threadIdx.x;
  const int tile_idx = blockIdx.x % gs.n_tiles;
  const int tt = blockIdx.x / gs.n_tiles;
  const int n0 = tile_idx * 128, t0 = tt * 32;
  float acc[32];
#pragma unroll
  for (int t = 0; t < 32; ++t) acc[t] = 0.0f;
  for (int k0 = 0; k0 < K; k0 += 32) {
    for (int idx = e; idx < 128 * 32; idx += 128) {
      const int r = idx / 32, kk = idx % 32;
      const int n = n0 + r, k = k0 + kk;
      ws_[kk][r] = (n < gs.N && k < K) ? w[(size_t)n * K + k] : 0.0f;
    }
    for (int idx = e; idx < 32 * 32; idx += 128) {
      const int t = idx / 32, kk = idx % 32;
      const int k = k0 + kk;
      as_[t][kk] = (t0 + t < gs.M && k < K) ? act[(size_t)(act_row0 + t0 + t) * K + k] : 0.0f;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < 32; ++kk) {
      const float wv = ws_[kk][e];
#pragma unroll
      for (int t = 0; t < 32; ++t) acc[t] = fmaf(wv, as_[t][kk], acc[t]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int t = 0; t < 32; ++t) tile[t * 128 + e] = acc[t];
  SoftmaxState* lmp = lm - t0;  // index by absolute token row
  if (ep.kind == EPI_LMHEAD && e < 32) lm[e] = sm_empty();
  __syncthreads();
  epi_chunk(ep, tile, n0, t0, e, lmp);
  __syncthreads();
  if (ep.kind == EPI_LMHEAD) {
    SoftmaxState* out = reinterpret_cast<SoftmaxState*>(ep.lm_part) + (size_t)blockIdx.x * gs.M;
    for (int t = e; t < gs.M; t += 128) out[t] = (t >= t0 && t < t0 + 32) ? lm[t - t0] : sm_empty();
  }
}

// ------------------------------------------------------- CUDA-core attention
// One CTA per (query row, head): softmax(q K^T / sqrt(hd)) V over keys [0, L),
// float32 model (K and V planes of float).
__global__ void __launch_bounds__(128) attn_simt_kernel(AttnParams p) {
  using T = float;
  using VT = float;
  extern __shared__ float sh[];
  __shared__ float red[32];
  pdl_trigger();
  pdl_wait();
  float* qs = sh;               // [hd]
  float* sc = sh + p.head_dim;  // [L]
  const int head = blockIdx.y;
  const int hd = p.head_dim, H = p.n_heads, Hkv = p.n_kv_heads;
  // batched forward: one tile per query row (its forward row, keys, slot)
  int m = blockIdx.x, L = p.L;
  const int* ptab = p.page_table;
  if (p.tiles) {
    const AttnTile tl = p.tiles[blockIdx.x];
    m = tl.q0;
    L = tl.L;
    ptab = p.page_table + (size_t)tl.seq * p.pages_per_seq;
  }
  const int g = head / (H / Hkv);
  const T* q = reinterpret_cast<const T*>(p.q) + ((size_t)m * H + head) * hd;
  for (int d = threadIdx.x; d < hd; d += blockDim.x) qs[d] = to_f(q[d]);
  __syncthreads();
  const float scale = 1.0f / sqrtf((float)hd);
  const T* kp = reinterpret_cast<const T*>(p.kv_pool);
  const VT* vp = reinterpret_cast<const VT*>(p.kv_pool);
  auto off = [&](int pos, int kv) {
    const int page = ptab[pos / KV_PAGE];
    return ((((size_t)p.layer * p.n_pages + page) * p.kv_planes + kv) * Hkv + g) *
               (size_t)(KV_PAGE * hd) +
           (size_t)(pos % KV_PAGE) * hd;
  };
  float mx = -INFINITY;
  for (int j = threadIdx.x; j < L; j += blockDim.x) {
    const T* kr = kp + off(j, 0);
    float dot = 0.0f;
    for (int d = 0; d < hd; ++d) dot = fmaf(qs[d], to_f(kr[d]), dot);
    sc[j] = dot * scale;
    mx = fmaxf(mx, sc[j]);
  }
  mx = block_max(mx, red);
  float sum = 0.0f;
  for (int j = threadIdx.x; j < L; j += blockDim.x) {
    const float e = expf(sc[j] - mx);
    sc[j] = e;
    sum += e;
  }
  sum = block_sum(sum, red);
  __syncthreads();
  T* o = reinterpret_cast<T*>(p.o) + ((size_t)m * H + head) * hd;
  for (int d = threadIdx.x; d < hd; d += blockDim.x) {
    float acc = 0.0f;
    for (int j = 0; j < L; ++j) acc = fmaf(sc[j], to_f(vp[off(j, 1) + d]), acc);
    o[d] = from_f<T>(acc / sum);
  }
}

}  // namespace

cudaError_t launch_embed_rmsnorm(const int* x, int r0, int M, const void* embed, int d,
                                 int vocab, const float* g, float eps, float* h, void* a,
                                 int f32, int* err, const StepParams* sp, cudaStream_t st,
                                 bool pdl, RowMap rm) {
  if (M <= 0) return cudaSuccess;
  if (f32)
    return launch_k(pdl, rmsnorm_kernel<float>, dim3(M), dim3(256), 0, st, x, r0,
                    (const float*)embed, vocab, h, 0, d, g, eps, a, err, sp, 0, rm);
  if (d % 4 == 0)
    return launch_k(pdl, rmsnorm_v4_kernel, dim3(M), dim3(256), 0, st, x, r0,
                    (const __nv_bfloat16*)embed, vocab, h, 0, d, g, eps, (__half*)a, err, sp, 0,
                    rm);
  return launch_k(pdl, rmsnorm_kernel<__nv_bfloat16>, dim3(M), dim3(256), 0, st, x, r0,
                  (const __nv_bfloat16*)embed, vocab, h, 0, d, g, eps, a, err, sp, 0, rm);
}

cudaError_t launch_rmsnorm(const float* h, int h_row0, int M, int d, const float* g, float eps,
                           void* a, int f32, const StepParams* sp, bool rows_from_lm0,
                           cudaStream_t st, bool pdl, RowMap rm) {
  if (M <= 0) return cudaSuccess;
  const int* nx = nullptr;
  if (f32)
    return launch_k(pdl, rmsnorm_kernel<float>, dim3(M), dim3(256), 0, st, nx, 0,
                    (const float*)nullptr, 0, const_cast<float*>(h), h_row0, d, g, eps, a,
                    (int*)nullptr, sp, rows_from_lm0 ? 1 : 0, rm);
  if (d % 4 == 0)
    return launch_k(pdl, rmsnorm_v4_kernel, dim3(M), dim3(256), 0, st, nx, 0,
                    (const __nv_bfloat16*)nullptr, 0, const_cast<float*>(h), h_row0, d, g, eps,
                    (__half*)a, (int*)nullptr, sp, rows_from_lm0 ? 1 : 0, rm);
  return launch_k(pdl, rmsnorm_kernel<__nv_bfloat16>, dim3(M), dim3(256), 0, st, nx, 0,
                  (const __nv_bfloat16*)nullptr, 0, const_cast<float*>(h), h_row0, d, g, eps, a,
                  (int*)nullptr, sp, rows_from_lm0 ? 1 : 0, rm);
}

cudaError_t launch_wait_timeout(int* err, cudaStream_t st) {
  wait_timeout_kernel<<<1, 32, 0, st>>>(err);
  return cudaGetLastError();
}

cudaError_t launch_kv_cosine(const void* a, const void* b, const int* page_table, int n_pages,
                             int planes, int n_layers, int Hkv, int hd, int f32, int L,
                             double* out, cudaStream_t st) {
  if (L < 1 || n_layers < 1 || Hkv < 1 || hd < 1) return cudaErrorInvalidValue;
  kv_cosine_kernel<<<dim3(L, 2, n_layers), 128, 0, st>>>(a, b, page_table, n_pages, planes, Hkv,
                                                          hd, f32, L, out);
  return cudaGetLastError();
}

cudaError_t launch_merge_select(const float* lm_part, int n_part, int n, int* x, int s,
                                int mask_id, float tau, int select, float* conf, int* tok,
                                uint8_t* unmask, DecodeState* state, const StepParams* sp,
                                cudaStream_t st, bool pdl) {
  if (n <= 0 || n > 256) return cudaErrorInvalidValue;
  return launch_k(pdl, merge_select_kernel, dim3(1), dim3(256), 0, st,
                  reinterpret_cast<const SoftmaxState*>(lm_part), n_part, n, x, s, mask_id, tau,
                  select, conf, tok, unmask, state, sp);
}

cudaError_t launch_merge_select_seg(const float* lm_part, int n_part, int m_lm,
                                    const SelectSeg* segs, int n_segs, int* x, int seq_stride,
                                    int mask_id, float tau, int fixed_k, float* conf, int* tok,
                                    uint8_t* unmask, DecodeState* states, cudaStream_t st,
                                    bool pdl) {
  if (n_segs <= 0) return cudaSuccess;
  return launch_k(pdl, merge_select_seg_kernel, dim3(n_segs), dim3(256), 0, st,
                  reinterpret_cast<const SoftmaxState*>(lm_part), n_part, m_lm, segs, x,
                  seq_stride, mask_id, tau, fixed_k, conf, tok, unmask, states);
}

cudaError_t launch_bf16_to_f16(void* p, size_t n, int* err, unsigned long long* inexact,
                               cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const size_t blocks = std::min<size_t>((n + 255) / 256, 4096);
  bf16_to_f16_kernel<<<(unsigned)blocks, 256, 0, st>>>(reinterpret_cast<uint16_t*>(p), n, err,
                                                       inexact);
  return cudaGetLastError();
}

cudaError_t launch_fill_masked(int* x, int from, int to, int mask_id, cudaStream_t st, bool pdl) {
  if (to <= from) return cudaSuccess;
  return launch_k(pdl, fill_kernel, dim3((to - from + 255) / 256), dim3(256), 0, st, x, from, to,
                  mask_id);
}

cudaError_t launch_check_prompt(const int* x, int n, int vocab, int mask_id, int* err,
                                cudaStream_t st, bool pdl) {
  if (n <= 0) return cudaSuccess;
  return launch_k(pdl, check_prompt_kernel, dim3((n + 255) / 256), dim3(256), 0, st, x, n, vocab,
                  mask_id, err);
}

cudaError_t launch_gemm_simt(const float* w, const float* act, int act_row0, int K,
                             const GemmShape& gs, const EpiParams& ep, cudaStream_t st, bool pdl) {
  const int grid = gs.n_tiles * ((gs.M + 31) / 32);
  return launch_k(pdl, gemm_simt_kernel, dim3(grid), dim3(128), 0, st, w, act, act_row0, K, gs,
                  ep);
}

cudaError_t launch_attn_simt(const AttnParams& p, cudaStream_t st, bool pdl) {
  if (p.kv_planes != 2) return cudaErrorInvalidValue;
  const size_t smem = (size_t)(p.head_dim + p.L) * sizeof(float);
  if (smem > 48 * 1024) return cudaErrorInvalidValue;
  // batched forward: p.L is the largest key count of the tiles
  return launch_k(pdl, attn_simt_kernel, dim3(p.tiles ? p.n_tiles : p.M, p.n_heads), dim3(128),
                  smem, st, p);
}


}  // namespace fd
