// Bidirectional attention of the bfloat16 model on the 5th-generation tensor
// cores (tcgen05, accumulators in tensor memory), K/V staged by TMA: the
// many-query forwards (block-start refresh, cache off, prefix cache).
//
// o = softmax(q K^T / sqrt(hd)) V over keys [0, L), no mask (every query
// position attends to every cached position, before and after it).
//
// CTA = (tile of 128 query rows, KV head g).  A query row is a (position,
// head-in-group) pair: a tile holds MP = 128 / rep consecutive positions x
// the rep query heads that share KV head g, so GQA heads share every K/V
// tile.  The whole Q tile (hi and lo planes) is staged once by a 3-D TMA
// load; the K/V pages of 64 keys (one cache page: K hi, K lo, V hi, V lo)
// stream through two 2-stage TMA rings, K's released as soon as its S
// product is done, V's after its PV product.  Per key tile j:
//   S_j  = Qhi Khi^T + Qhi Klo^T + Qlo Khi^T    (tcgen05, 128 x 64, TMEM)
//   softmax warps: one thread per query row reads its 64 scores from TMEM,
//         keeps the running max m and sum l (fp32, exp2 domain), writes
//         P = exp2(S - m) as two fp16 terms (hi + lo) to shared memory;
//   O   += Phi Vhi + Phi Vlo + Plo Vhi          (tcgen05, 128 x hd, TMEM)
// so every product keeps the three significant cross terms of the two-term
// storage (~22 significant bits, as everywhere in the bf16 model).  S is
// double-buffered in TMEM, so S_{j+1} runs on the tensor core while the
// softmax of tile j does.  The running max moves only when a row's max grows
// by more than 2^8 (then that row of O is rescaled in TMEM before the next
// PV product); P stays below 2^8, inside the fp16 range, and the result is
// the same softmax.  The output rows are divided by l and stored as
// two-term fp16 pair rows.
//
// Warp roles (192 threads): warp 0 = TMA producer, warp 1 = TMEM owner and
// MMA issuer, warps 2..5 = softmax / epilogue (TMEM lane quadrant = warp %
// 4; thread = query row).  Every wait is bounded (WAIT_LIMIT_NS): a timeout
// sets DEV_ERR_TIMEOUT and ends the CTA.
#include "common.cuh"
#include "kernels.h"

namespace fd {

namespace {

template <int HD>
struct AtLayout {
  static constexpr int KH = HD / 64;                  // 64-dim sub-tiles (128-byte rows)
  static constexpr int Q_SUB = 128 * 64 * 2;          // [128 rows][64 dims] fp16
  static constexpr int KV_SUB = 64 * 64 * 2;          // [64 keys][64 dims] fp16
  static constexpr int STAGES = 2;
  static constexpr int HALF_STAGE = 2 * KH * KV_SUB;  // K hi + K lo, or V hi + V lo
  static constexpr int P_SUB = 128 * 64 * 2;          // [128 rows][64 keys] fp16
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + 2 * KH * Q_SUB;
  static constexpr int V_OFF = K_OFF + STAGES * HALF_STAGE;
  static constexpr int P_OFF = V_OFF + STAGES * HALF_STAGE;
  static constexpr int BAR_OFF = P_OFF + 2 * P_SUB;
  // q_full, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2], s_empty[2],
  // p_full, o_done, mma_done
  static constexpr int N_BARS = 1 + 4 * STAGES + 4 + 3;
  static constexpr int MISC_OFF = BAR_OFF + N_BARS * 8;
  static constexpr int SMEM = MISC_OFF + 16 + 1024;   // slack for 1024-byte alignment
  static constexpr uint32_t TMEM_COLS = 256;          // S: 2 x 64 columns, O: HD columns
  static constexpr uint32_t O_COL = 128;
  static_assert(SMEM <= 232448, "exceeds the 227 KB per-CTA shared memory limit");
  static_assert(O_COL + HD <= TMEM_COLS, "O does not fit in the TMEM allocation");
};

constexpr int AT_THREADS = 192;

struct AtArgs {
  AttnParams p;
  int q_lo_rows;   // row offset of the q lo plane in the q map (rows of H * hd)
  int rep, mp;     // query heads per KV head; positions per tile (128 / rep)
  int* err;
};

template <int HD>
__global__ void __launch_bounds__(AT_THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kvmap,
                   const AtArgs A) {
  using Lay = AtLayout<HD>;
  constexpr int KH = Lay::KH;
  const AttnParams& p = A.p;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::BAR_OFF);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + Lay::STAGES;
  uint64_t* v_full = k_empty + Lay::STAGES;
  uint64_t* v_empty = v_full + Lay::STAGES;
  uint64_t* s_full = v_empty + Lay::STAGES;
  uint64_t* s_empty = s_full + 2;
  uint64_t* p_full = s_empty + 2;
  uint64_t* o_done = p_full + 1;
  uint64_t* mma_done = o_done + 1;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Lay::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.y;
  const int rep = A.rep, MP = A.mp;
  // one sequence: tile x covers positions [x MP, x MP + MP) of the M query
  // positions over keys [0, p.L); batched forward: the tile table gives the
  // segment (forward rows q0 .. q0 + m - 1 of slot seq, keys [0, L)) and the
  // tile's first position r0 / rep within it
  int m0 = blockIdx.x * MP, qbase = 0, m_seg = p.M, L = p.L;
  const int* ptab = p.page_table;
  if (p.tiles) {
    const AttnTile tl = p.tiles[blockIdx.x];
    m0 = tl.r0 / rep;
    qbase = tl.q0;
    m_seg = tl.m;
    L = tl.L;
    ptab = p.page_table + (size_t)tl.seq * p.pages_per_seq;
  }
  const int n_kt = (L + 63) / 64;
  int* err = A.err;

  if (threadIdx.x == 0) {
    // s_empty and p_full collect the 128 softmax threads; the others one
    // arrival (an expect_tx or a tcgen05.commit)
    for (int i = 0; i < Lay::N_BARS; ++i) {
      uint64_t* bar = &bars[i];
      mbar_init(bar, (bar == s_empty || bar == s_empty + 1 || bar == p_full) ? 128 : 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(misc, Lay::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  pdl_trigger();
  pdl_wait();  // q and the K/V cache come from the preceding kernels

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------- TMA producer
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&kvmap);
      // Q: 2 planes x KH boxes of {64 dims, rep heads, MP positions}
      mbar_arrive_expect_tx(q_full, 2 * KH * 128 * MP * rep);
      for (int pl = 0; pl < 2; ++pl)
        for (int kh = 0; kh < KH; ++kh)
          tma_load_3d(smem + Lay::Q_OFF + (pl * KH + kh) * Lay::Q_SUB, &qmap, q_full, kh * 64,
                      g * rep, (pl ? A.q_lo_rows : 0) + qbase + m0);
      // K tile j is free once S_j is done, V tile j once PV_j is: K runs a
      // tile ahead of V through its own ring, so S_{j+1} never waits for a
      // load issued after PV_{j-1}
      int j = 0;
      bool ok = true;
      for (; j < n_kt && ok; ++j) {
        const int st = j % Lay::STAGES;
        const uint32_t par = ((j / Lay::STAGES) & 1u) ^ 1u;
        const int page = ptab[j];   // keys [64 j, 64 j + 64) = one cache page
        for (int kv = 0; kv < 2 && ok; ++kv) {
          uint64_t* full = kv ? &v_full[st] : &k_full[st];
          if (!mbar_wait(kv ? &v_empty[st] : &k_empty[st], par, err, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full, Lay::HALF_STAGE);
          uint8_t* dst = smem + (kv ? Lay::V_OFF : Lay::K_OFF) + st * Lay::HALF_STAGE;
          for (int t = 0; t < 2; ++t) {   // hi, lo planes
            const int pl = 2 * kv + t;
            const int row = (((p.layer * p.n_pages + page) * 4 + pl) * p.n_kv_heads + g) * 64;
            for (int kh = 0; kh < KH; ++kh)
              tma_load_2d(dst + (t * KH + kh) * Lay::KV_SUB, &kvmap, full, kh * 64, row);
          }
        }
      }
      if (!ok) {
        // let the copies already issued land before the CTA can exit
        *abort_flag = 1;
        mbar_wait(q_full, 0, err, nullptr);
        for (int jj = (j > Lay::STAGES ? j - Lay::STAGES : 0); jj < j; ++jj) {
          mbar_wait(&k_full[jj % Lay::STAGES], (jj / Lay::STAGES) & 1u, err, nullptr);
          mbar_wait(&v_full[jj % Lay::STAGES], (jj / Lay::STAGES) & 1u, err, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------- MMA issuer
      const uint32_t idesc_s = idesc_f32acc(64, true);      // 128 x 64 scores
      const uint32_t idesc_o = idesc_f32acc_bmn(HD, true);  // 128 x HD, V MN-major
      const uint32_t q0 = smem_u32(smem + Lay::Q_OFF);
      const uint32_t p0 = smem_u32(smem + Lay::P_OFF);
      bool ok = mbar_wait(q_full, 0, err, abort_flag);
      for (int j = 0; j <= n_kt && ok; ++j) {
        if (j < n_kt) {
          const int st = j % Lay::STAGES, b = j & 1;
          if (!mbar_wait(&k_full[st], (j / Lay::STAGES) & 1u, err, abort_flag) ||
              !mbar_wait(&s_empty[b], ((j >> 1) & 1u) ^ 1u, err, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t kv0 = smem_u32(smem + Lay::K_OFF + st * Lay::HALF_STAGE);
          const uint32_t d = tmem + b * 64;
#pragma unroll
          for (int kh = 0; kh < KH; ++kh) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint32_t qh = q0 + kh * Lay::Q_SUB + k * 32;
              const uint32_t ql = qh + KH * Lay::Q_SUB;
              const uint32_t kh_ = kv0 + kh * Lay::KV_SUB + k * 32;          // K hi
              const uint32_t kl_ = kh_ + KH * Lay::KV_SUB;                    // K lo
              tc_mma(d, smem_desc_sw128(qh), smem_desc_sw128(kh_), idesc_s,
                     (kh > 0 || k > 0) ? 1u : 0u);
              tc_mma(d, smem_desc_sw128(qh), smem_desc_sw128(kl_), idesc_s, 1u);
              tc_mma(d, smem_desc_sw128(ql), smem_desc_sw128(kh_), idesc_s, 1u);
            }
          }
          tc_commit(&s_full[b]);
          tc_commit(&k_empty[st]);
        }
        if (j > 0) {
          const int jj = j - 1, st = jj % Lay::STAGES;
          if (!mbar_wait(p_full, jj & 1u, err, abort_flag) ||
              !mbar_wait(&v_full[st], (jj / Lay::STAGES) & 1u, err, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t v0 = smem_u32(smem + Lay::V_OFF + st * Lay::HALF_STAGE);  // V hi
#pragma unroll
          for (int k = 0; k < 4; ++k) {   // 16 keys per MMA
            const uint32_t ph = p0 + k * 32, pl = ph + Lay::P_SUB;
            const uint64_t vh = smem_desc_sw128_mn(v0 + k * 2048, Lay::KV_SUB, 1024);
            const uint64_t vl = smem_desc_sw128_mn(v0 + KH * Lay::KV_SUB + k * 2048, Lay::KV_SUB,
                                                   1024);
            tc_mma(tmem + Lay::O_COL, smem_desc_sw128(ph), vh, idesc_o,
                   (jj > 0 || k > 0) ? 1u : 0u);
            tc_mma(tmem + Lay::O_COL, smem_desc_sw128(ph), vl, idesc_o, 1u);
            tc_mma(tmem + Lay::O_COL, smem_desc_sw128(pl), vh, idesc_o, 1u);
          }
          tc_commit(o_done);
          tc_commit(&v_empty[st]);
        }
      }
      if (!ok) *abort_flag = 1;
      // every MMA issued has completed before TMEM is released
      tc_commit(mma_done);
      mbar_wait(mma_done, 0, err, nullptr);
    }
  } else {
    // ------------------------------------------------------ softmax / epilogue
    const int quad = warp & 3;
    const int row = quad * 32 + lane;             // query row of the tile = TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    const float sl2 = rsqrtf((float)HD) * 1.4426950408889634f;  // 1/sqrt(hd) * log2(e)
    uint8_t* p_hi = smem + Lay::P_OFF;
    uint8_t* p_lo = p_hi + Lay::P_SUB;
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true;
    for (int j = 0; j < n_kt && ok; ++j) {
      const int b = j & 1;
      // TMEM loads and stores are warp-collective: every decision that guards
      // one is made uniform across the warp
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[b], (j >> 1) & 1u, err, abort_flag));
      tc_fence_after();
      float s[64];
      if (ok) tmem_ld64(lane_base + b * 64, s);
      tc_fence_before();
      mbar_arrive(&s_empty[b]);
      if (!ok) break;
      const int k_valid = min(64, L - j * 64);
      float mt = -INFINITY;
#pragma unroll
      for (int k = 0; k < 64; ++k) {
        s[k] = k < k_valid ? s[k] * sl2 : -INFINITY;
        mt = fmaxf(mt, s[k]);
      }
      // the reference max moves only when the row max grows by more than 2^8
      const bool move = mt > m_run + 8.0f;
      const float m_use = move ? mt : m_run;
      float rs = 0.0f;
      uint32_t hw[32], lw[32];   // P hi / lo, two fp16 per word
#pragma unroll
      for (int k = 0; k < 64; k += 2) {
        const float e0 = exp2f(s[k] - m_use), e1 = exp2f(s[k + 1] - m_use);
        rs += e0 + e1;
        const __half2 h = __floats2half2_rn(e0, e1);
        const float2 hf = __half22float2(h);
        const __half2 l = __floats2half2_rn(e0 - hf.x, e1 - hf.y);
        hw[k >> 1] = *reinterpret_cast<const uint32_t*>(&h);
        lw[k >> 1] = *reinterpret_cast<const uint32_t*>(&l);
      }
      // the P buffer and O are free once the previous tile's PV product is done
      if (j > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(o_done, (j - 1) & 1u, err, abort_flag));
        tc_fence_after();
        const bool rescale = move && m_run != -INFINITY;
        if (ok && __any_sync(0xffffffffu, rescale)) {
          // rows that keep their reference max multiply by exactly 1
          const float alpha = rescale ? exp2f(m_run - m_use) : 1.0f;
          l_run *= alpha;
#pragma unroll
          for (int c = 0; c < HD; c += 32) {
            float o[32];
            tmem_ld32(lane_base + Lay::O_COL + c, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(lane_base + Lay::O_COL + c, o);
          }
        }
      }
      m_run = m_use;
      l_run += rs;
      // row `row` of the [128][64] K-major, 128-byte-swizzled P tiles
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t off = row * 128 + ((c ^ (row & 7)) << 4);
        *reinterpret_cast<uint4*>(p_hi + off) =
            make_uint4(hw[4 * c], hw[4 * c + 1], hw[4 * c + 2], hw[4 * c + 3]);
        *reinterpret_cast<uint4*>(p_lo + off) =
            make_uint4(lw[4 * c], lw[4 * c + 1], lw[4 * c + 2], lw[4 * c + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok) ok = mbar_wait(o_done, (n_kt - 1) & 1u, err, abort_flag);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    if (!ok) *abort_flag = 1;
    // ---- epilogue: O / l as two-term fp16 pair rows
    const int pos_local = row / rep, jj = row - pos_local * rep;
    const int m = qbase + m0 + pos_local;   // forward row
    const bool valid = ok && pos_local < MP && m0 + pos_local < m_seg;
    if (ok) {   // warp-uniform; the stores are per row
      const float inv = valid ? 1.0f / l_run : 0.0f;
      const int hq = p.n_heads * HD, head = g * rep + jj;
      __half* ob = reinterpret_cast<__half*>(p.o);
      const size_t hi_off = (size_t)pair_row(m) * hq + (size_t)head * HD;
      const size_t lo_off = hi_off + (size_t)PAIR_LO * hq;
      for (int c0 = 0; c0 < HD; c0 += 32) {
        float o[32];
        tmem_ld32(lane_base + Lay::O_COL + c0, o);
        if (!valid) continue;
#pragma unroll
        for (int c = 0; c < 32; c += 8) {
          uint32_t hv[4], lv[4];
#pragma unroll
          for (int i = 0; i < 8; i += 2) {
            __half h0, l0, h1, l1;
            split_f16(o[c + i] * inv, h0, l0);
            split_f16(o[c + i + 1] * inv, h1, l1);
            const __half2 hh = __halves2half2(h0, h1), ll = __halves2half2(l0, l1);
            hv[i >> 1] = *reinterpret_cast<const uint32_t*>(&hh);
            lv[i >> 1] = *reinterpret_cast<const uint32_t*>(&ll);
          }
          *reinterpret_cast<uint4*>(ob + hi_off + c0 + c) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
          *reinterpret_cast<uint4*>(ob + lo_off + c0 + c) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
        }
      }
    }
  }

  // lanes 1..31 of the single-thread role warps reach this point long before
  // their lane 0: reconverge every warp first
  __syncwarp();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, Lay::TMEM_COLS);
  }
}

template <int HD>
cudaError_t launch_hd(const CUtensorMap* qmap, const CUtensorMap* kvmap, const AtArgs& a,
                      cudaStream_t st, bool pdl) {
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<HD>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         AtLayout<HD>::SMEM);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const int tiles = a.p.tiles ? a.p.n_tiles : (a.p.M + a.mp - 1) / a.mp;
  return launch_k(pdl, attn_tc_kernel<HD>, dim3(tiles, a.p.n_kv_heads), dim3(AT_THREADS),
                  (size_t)AtLayout<HD>::SMEM, st, *qmap, *kvmap, a);
}

}  // namespace

bool attn_tc_supported(const AttnParams& p) {
  const int rep = p.n_kv_heads > 0 ? p.n_heads / p.n_kv_heads : 0;
  return p.kv_planes == 4 && (p.head_dim == 64 || p.head_dim == 128) && rep >= 1 && rep <= 128 &&
         p.n_split == 1 && p.M >= 1 && p.L >= 1 && (p.tiles == nullptr || p.n_tiles >= 1);
}

cudaError_t launch_attn_tc(const CUtensorMap* qmap, const CUtensorMap* kvmap, const AttnParams& p,
                           int q_lo_rows, int* err, cudaStream_t st, bool pdl) {
  if (!attn_tc_supported(p)) return cudaErrorInvalidValue;
  AtArgs a{};
  a.p = p;
  a.q_lo_rows = q_lo_rows;
  a.rep = p.n_heads / p.n_kv_heads;
  a.mp = 128 / a.rep;
  a.err = err;
  switch (p.head_dim) {
    case 64: return launch_hd<64>(qmap, kvmap, a, st, pdl);
    case 128: return launch_hd<128>(qmap, kvmap, a, st, pdl);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t attn_tc_init_attributes() {
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<64>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       AtLayout<64>::SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attn_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             AtLayout<128>::SMEM);
  return e;
}

}  // namespace fd
