// Bidirectional attention of the block queries of a DualCache step (bf16
// model) on the 5th-generation tensor cores: o = softmax(q K^T / sqrt(hd)) V
// over keys [0, L), no mask, for at most 64 query positions (a block step,
// or the block segments of a batched step).
//
// A block step attends 32 positions to all L cached positions: little
// arithmetic, a K/V stream of L positions per head, and a latency chain per
// CTA.  This kernel keeps that chain short: a CTA takes one chunk of 128
// keys at a time and runs ONE score product, ONE softmax and ONE PV product
// per chunk, and the keys are split over the CTAs of a thread-block cluster
// (one cluster per (query-row tile, KV head)) that merge their partial
// results over distributed shared memory.
//
// CTA = (tile of RP = 32 or 64 query rows, KV head g, key split z).  A query
// row is a (position, head-in-group) pair, so GQA heads share each K/V
// chunk.  Per chunk (128 keys = two cache pages, K and V hi/lo planes staged
// by TMA with the 128-byte swizzle):
//   S^T = K_hi Qs^T + K_lo Qs^T,  Qs = [q_hi rows; q_lo rows]   (tcgen05,
//         M = 128 keys, N = 2 RP, TMEM) -- the keys are the MMA's M, so
//         one chunk is one chain of 2 hd / 16 instructions; the score of
//         (row r, key k) is column r plus column RP + r of lane k;
//   the scores go through shared memory (transposed) to the softmax: 8
//         threads per row, 16 keys each, fp32, exp2 domain; P = exp2(s - m)
//         as two fp16 terms (hi + lo) in the rows [P_hi; P_lo] of the PV
//         product's A operand;
//   O += [P_hi; P_lo] V_hi + [P_hi; P_lo] V_lo                 (tcgen05,
//         M = 128 (2 RP rows used), N = hd, V MN-major, TMEM);
// every product carries the three significant cross terms of the two-term
// storage (and the negligible lo x lo one), ~22 significant bits as
// everywhere in the bf16 model; O row r = TMEM row r + TMEM row RP + r.
// Across chunks of one CTA the reference max moves only when a row's max
// grows by more than 2^8 (then O and l are rescaled), so P < 2^8 stays in
// the fp16 range and the result is the same softmax.
//
// Key splits: each split writes its rows' unnormalised O, reference max m
// and sum l to its own shared memory; after a cluster barrier the 8-feature
// groups of O are merged round-robin by the splits (group j by split
// j % n_split), each from every split in split order
// (O = sum_r 2^(m_r - M) O_r, l likewise, M = max_r m_r), divided by l and
// stored as two-term fp16 pair rows: the result does not depend on timing
// or on which CTA merges it.
//
// 256 threads (the two warps of each TMEM lane quadrant split the rows of a
// score read-out and the features of O); thread 0 issues the TMA loads and
// the MMAs.  Every wait is bounded (WAIT_LIMIT_NS): a timeout sets
// DEV_ERR_TIMEOUT and the CTA skips its remaining work but still reaches
// both cluster barriers.
#include "common.cuh"
#include "kernels.h"

namespace fd {

namespace {

constexpr int BLK_THREADS = 256;
constexpr int BLK_WARPS = BLK_THREADS / 32;
constexpr int CHUNK = 128;   // keys per chunk: two cache pages

template <int HD, int RP>
struct BlkLayout {
  static constexpr int KH = HD / 64;                  // 64-dim sub-tiles (128-byte rows)
  static constexpr int PAGE_SUB = 64 * 128;           // [64 keys][64 dims] fp16
  static constexpr int PLANE = KH * 2 * PAGE_SUB;     // [128 keys][HD] fp16, as KH sub-tiles
  static constexpr int KV_OFF = 0;                    // planes K hi, K lo, V hi, V lo
  static constexpr int Q_SUB = 2 * RP * 128;          // [2 RP rows][64 dims] fp16
  static constexpr int Q_OFF = KV_OFF + 4 * PLANE;
  static constexpr int P_SUB = 128 * 128;             // [128 rows][64 keys] fp16
  static constexpr int P_OFF = Q_OFF + KH * Q_SUB;
  // per-row statistics: red_max[8][RP], red_sum[8][RP], m_ref[RP], l[RP], alpha[RP]
  static constexpr int RED_OFF = P_OFF + 2 * P_SUB;
  static constexpr int RED_BYTES = (2 * BLK_WARPS + 3) * RP * 4;
  static constexpr int BAR_OFF = RED_OFF + RED_BYTES;
  static constexpr int N_BARS = 4;                    // k_full, v_full, s_done, pv_done
  static constexpr int MISC_OFF = BAR_OFF + N_BARS * 8;
  static constexpr int SMEM = MISC_OFF + 16 + 1024;   // slack for 1024-byte alignment
  static constexpr uint32_t TMEM_COLS = 256;          // S^T: 2 RP columns; O: HD at O_COL
  static constexpr uint32_t O_COL = 128;
  static constexpr int XCH_ROW = HD + 4;              // split exchange row (floats)
  static_assert(Q_SUB % 1024 == 0 && PLANE % 1024 == 0, "swizzled tiles stay 1024-aligned");
  static_assert(RP * 128 * 4 <= 2 * P_SUB, "score transpose exceeds the P area");
  static_assert(RP * HD * 4 <= 2 * P_SUB, "O exchange exceeds the P area");
  static_assert(RP * XCH_ROW * 4 <= 4 * PLANE, "split exchange exceeds the K/V area");
  static_assert(2 * RP <= 128 && 2 * RP <= (int)O_COL, "scores exceed their TMEM columns");
  static_assert(SMEM <= 232448, "exceeds the 227 KB per-CTA shared memory limit");
};

struct BlkArgs {
  AttnParams p;
  int rp;            // query rows per CTA (32 or 64)
  int chunks_per_split;
};

FD_DEV void cp_async16_zfill(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}

// 16-byte load from distributed shared memory: volatile (ordered with the
// cluster barriers), no memory clobber, so a run of them issues back to back.
FD_DEV float4 ld_dsmem16(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr));
  return v;
}

// Two-term fp16 store of n (multiple of 8) output features x * inv.
template <int N>
FD_DEV void store_two_term(__half* ob, size_t hi_off, size_t lo_off, const float* x, float inv) {
#pragma unroll
  for (int c = 0; c < N; c += 8) {
    uint32_t hv[4], lv[4];
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      __half h0, l0, h1, l1;
      split_f16(x[c + i] * inv, h0, l0);
      split_f16(x[c + i + 1] * inv, h1, l1);
      const __half2 hh = __halves2half2(h0, h1), ll = __halves2half2(l0, l1);
      hv[i >> 1] = *reinterpret_cast<const uint32_t*>(&hh);
      lv[i >> 1] = *reinterpret_cast<const uint32_t*>(&ll);
    }
    *reinterpret_cast<uint4*>(ob + hi_off + c) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
    *reinterpret_cast<uint4*>(ob + lo_off + c) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
  }
}

template <int HD, int RP>
__global__ void __launch_bounds__(BLK_THREADS, 1)
    attn_blk_kernel(const __grid_constant__ CUtensorMap kvmap, const BlkArgs A) {
  using Lay = BlkLayout<HD, RP>;
  constexpr int KH = Lay::KH;
  const AttnParams& p = A.p;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::BAR_OFF);
  uint64_t* k_full = bars;
  uint64_t* v_full = bars + 1;
  uint64_t* s_done = bars + 2;
  uint64_t* pv_done = bars + 3;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Lay::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  float* red_max = reinterpret_cast<float*>(smem + Lay::RED_OFF);   // [8][RP]
  float* red_sum = red_max + BLK_WARPS * RP;                        // [8][RP]
  float* row_m = red_sum + BLK_WARPS * RP;                          // [RP]
  float* row_l = row_m + RP;                                        // [RP]
  float* row_a = row_l + RP;                                        // [RP]
  float* sT = reinterpret_cast<float*>(smem + Lay::P_OFF);          // [RP][128] scores, swizzled

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // TMEM lane quadrant of this warp, and which half of the columns (scores:
  // rows; O: features) it takes of that quadrant
  const int quad = warp & 3, half = warp >> 2;
  const int g = blockIdx.y;
  const int H = p.n_heads, Hkv = p.n_kv_heads, rep = H / Hkv;
  // one sequence: row tile x of the M block positions over keys [0, p.L);
  // batched forward: the tile table gives the segment (forward rows q0 ..
  // q0 + m - 1 of slot seq, keys [0, L)) and the tile's first query row r0
  int rows_total = p.M * rep, row0 = blockIdx.x * RP, qbase = 0, L = p.L;
  const int* ptab = p.page_table;
  if (p.tiles) {
    const AttnTile tl = p.tiles[blockIdx.x];
    rows_total = tl.m * rep;
    row0 = tl.r0;
    qbase = tl.q0;
    L = tl.L;
    ptab = p.page_table + (size_t)tl.seq * p.pages_per_seq;
  }
  const int n_split = p.n_split;
  const int n_chunks_all = (L + CHUNK - 1) / CHUNK;
  const int ch_lo = blockIdx.z * A.chunks_per_split;
  const int n_ch = max(0, min(n_chunks_all, ch_lo + A.chunks_per_split) - ch_lo);
  const int valid_pages = (L + KV_PAGE - 1) / KV_PAGE;
  int* err = p.err;

  if (tid == 0) {
    for (int i = 0; i < Lay::N_BARS; ++i) mbar_init(&bars[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(misc, Lay::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
  pdl_trigger();
  pdl_wait();   // q and the step's own K/V come from the preceding kernel

  // ---- K/V chunk loads (thread 0): planes {hi, lo} of K or V, KH sub-tiles
  // of [128 keys][64 dims], two pages each; pages past the sequence are
  // clamped to its last page (their keys are masked below)
  auto load_half = [&](int c, int kv, uint64_t* bar) {
    const int k0 = (ch_lo + c) * CHUNK;
    mbar_arrive_expect_tx(bar, 2 * KH * 2 * Lay::PAGE_SUB);
    for (int pg = 0; pg < 2; ++pg) {
      const int page = ptab[min(k0 / KV_PAGE + pg, valid_pages - 1)];
      for (int t = 0; t < 2; ++t) {
        const int pl = 2 * kv + t;
        const int row = (((p.layer * p.n_pages + page) * 4 + pl) * Hkv + g) * KV_PAGE;
        uint8_t* dst = smem + Lay::KV_OFF + pl * Lay::PLANE + pg * Lay::PAGE_SUB;
        for (int kh = 0; kh < KH; ++kh)
          tma_load_2d(dst + kh * 2 * Lay::PAGE_SUB, &kvmap, bar, kh * 64, row);
      }
    }
  };
  int k_issued = 0, v_issued = 0, k_seen = 0, v_seen = 0;   // chunks (thread 0)
  if (tid == 0 && n_ch > 0) {
    tma_prefetch_desc(&kvmap);
    load_half(0, 0, k_full);
    load_half(0, 1, v_full);
    k_issued = v_issued = 1;
  }

  // ---- Q rows [q_hi; q_lo] of the tile (zero past the last query row)
  {
    const __half* qg = reinterpret_cast<const __half*>(p.q);
    const uint32_t qs = smem_u32(smem + Lay::Q_OFF);
    for (int idx = tid; idx < 2 * RP * (HD / 8); idx += BLK_THREADS) {
      const int i = idx / (HD / 8), ch = idx % (HD / 8);
      const int r = row0 + (i < RP ? i : i - RP);
      const bool ok = r < rows_total;
      const int pos = ok ? qbase + r / rep : 0, jj = ok ? r % rep : 0;   // forward row
      const __half* src = qg + (i < RP ? 0 : p.q_plane) + ((size_t)pos * H + g * rep + jj) * HD +
                          ch * 8;
      const int kh = ch >> 3, c = ch & 7;
      cp_async16_zfill(qs + kh * Lay::Q_SUB + i * 128 + ((c ^ (i & 7)) << 4), src, ok ? 16 : 0);
    }
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
    fence_proxy_async_smem();
    __syncthreads();
  }

  const float sl2 = rsqrtf((float)HD) * 1.4426950408889634f;   // 1/sqrt(hd) * log2(e)
  // S^T = K Qs^T of chunk c (thread 0): once its K has landed; everyone
  // waits on s_done for it.  Chunk 0's is issued here, chunk c + 1's right
  // behind chunk c's PV product, so that it runs while the threads finish
  // chunk c and its K was loaded during chunk c's softmax.
  auto issue_s = [&](int c) {
    if (!mbar_wait(k_full, c & 1u, err, abort_flag)) {
      *abort_flag = 1;
      return;
    }
    ++k_seen;
    tc_fence_after();
    const uint32_t idesc = idesc_f32acc(2 * RP, true);
    const uint32_t kbase = smem_u32(smem + Lay::KV_OFF);
    const uint32_t qb = smem_u32(smem + Lay::Q_OFF);
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int kh = 0; kh < KH; ++kh)
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc_mma(tmem, smem_desc_sw128(kbase + t * Lay::PLANE + kh * 2 * Lay::PAGE_SUB + k * 32),
                 smem_desc_sw128(qb + kh * Lay::Q_SUB + k * 32), idesc,
                 (t > 0 || kh > 0 || k > 0) ? 1u : 0u);
    tc_commit(s_done);
  };
  bool ok = true;
  if (tid == 0 && n_ch > 0) issue_s(0);
  for (int c = 0; c < n_ch && ok; ++c) {
    const uint32_t ph = c & 1u;
    __syncthreads();
    ok = *abort_flag == 0;
    if (ok) ok = mbar_wait(s_done, ph, err, abort_flag);
    // the score transpose goes over P: the previous chunk's PV product (which
    // reads P) must be done; it also frees O for the rescale below
    if (ok && c > 0) ok = mbar_wait(pv_done, (c - 1) & 1u, err, abort_flag);
    ok = __syncthreads_and(ok);
    if (!ok) break;
    tc_fence_after();
    // the K planes are free: the next chunk's K streams in during this softmax
    if (tid == 0 && c + 1 < n_ch) {
      load_half(c + 1, 0, k_full);
      ++k_issued;
    }

    // ---- scores: lane = key; transpose into sT[row][key ^ (row & 31)]; the
    // two warps of a lane quadrant take half of the rows each
    {
      constexpr int RH = RP / 2;
      const int kl = quad * 32 + lane;
      const bool kvalid = (ch_lo + c) * CHUNK + kl < L;
      float hi[32], lo[32];
      if (RH == 16) {
        tmem_ld16x2<RP>(lane_base + half * RH, hi, lo);
      } else {
        tmem_ld32(lane_base + half * RH, hi);
        tmem_ld32(lane_base + RP + half * RH, lo);
      }
#pragma unroll
      for (int i = 0; i < RH; ++i) {
        const int r = half * RH + i;
        sT[r * 128 + (kl ^ (r & 31))] = kvalid ? (hi[i] + lo[i]) * sl2 : -INFINITY;
      }
    }
    tc_fence_before();
    __syncthreads();

    // ---- softmax: thread (warp w, lane) = keys [16 w, 16 w + 16) of rows
    // lane and lane + 32 (RP = 64); 8 threads per row
    constexpr int NR = RP / 32;
    constexpr int KPT = CHUNK / BLK_WARPS;   // keys per thread
    float s[NR][KPT];
#pragma unroll
    for (int q = 0; q < NR; ++q) {
      const int r = lane + 32 * q;
      float mloc = -INFINITY;
#pragma unroll
      for (int i = 0; i < KPT; ++i) {
        s[q][i] = sT[r * 128 + ((warp * KPT + i) ^ (r & 31))];
        mloc = fmaxf(mloc, s[q][i]);
      }
      red_max[warp * RP + r] = mloc;
    }
    __syncthreads();
    float m_use[NR];
    bool moved_any = false;
#pragma unroll
    for (int q = 0; q < NR; ++q) {
      const int r = lane + 32 * q;
      float mt = red_max[r];
#pragma unroll
      for (int w = 1; w < BLK_WARPS; ++w) mt = fmaxf(mt, red_max[w * RP + r]);
      const float m_old = c == 0 ? -INFINITY : row_m[r];
      // the reference max moves only when the row max grows by more than 2^8
      const bool move = c == 0 || mt > m_old + 8.0f;
      m_use[q] = move ? mt : m_old;
      moved_any |= (c > 0 && move);
      float rs = 0.0f;
#pragma unroll
      for (int i = 0; i < KPT; ++i) {
        s[q][i] = m_use[q] == -INFINITY ? 0.0f : exp2f(s[q][i] - m_use[q]);
        rs += s[q][i];
      }
      red_sum[warp * RP + r] = rs;
    }
    moved_any = __syncthreads_or(moved_any);
    if (warp == 0) {
#pragma unroll
      for (int q = 0; q < NR; ++q) {
        const int r = lane + 32 * q;
        const float m_old = c == 0 ? -INFINITY : row_m[r];
        const float a = (c == 0 || m_use[q] == m_old) ? 1.0f : exp2f(m_old - m_use[q]);
        const float l_old = c == 0 ? 0.0f : row_l[r];
        float rs = 0.0f;
#pragma unroll
        for (int w = 0; w < BLK_WARPS; ++w) rs += red_sum[w * RP + r];
        row_l[r] = l_old * a + rs;
        row_a[r] = a;
        row_m[r] = m_use[q];
      }
    }
    __syncthreads();   // sT (under P) has been read by every thread; row_a is written
    if (c > 0) {
      if (moved_any && quad < 2 * NR) {
        // TMEM rows r and RP + r of O (this quadrant's lanes, this warp's
        // half of the features) times alpha_r
        const int lr = quad * 32 + lane;
        const float a = row_a[lr < RP ? lr : lr - RP];
#pragma unroll
        for (int c0 = half * (HD / 2); c0 < (half + 1) * (HD / 2); c0 += 32) {
          float o[32];
          tmem_ld32(lane_base + Lay::O_COL + c0, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= a;
          tmem_st32(lane_base + Lay::O_COL + c0, o);
        }
      }
    }
    // ---- P = [P_hi; P_lo] rows of the [128 rows][128 keys] K-major tile
    {
      uint8_t* pb = smem + Lay::P_OFF + (warp * KPT / 64) * Lay::P_SUB;
#pragma unroll
      for (int q = 0; q < NR; ++q) {
        const int r = lane + 32 * q;
#pragma unroll
        for (int cc = 0; cc < KPT / 8; ++cc) {
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int i = 0; i < 8; i += 2) {
            const float e0 = s[q][cc * 8 + i], e1 = s[q][cc * 8 + i + 1];
            const __half2 h = __floats2half2_rn(e0, e1);
            const float2 hf = __half22float2(h);
            const __half2 l = __floats2half2_rn(e0 - hf.x, e1 - hf.y);
            hw[i >> 1] = *reinterpret_cast<const uint32_t*>(&h);
            lw[i >> 1] = *reinterpret_cast<const uint32_t*>(&l);
          }
          // 16-byte chunk of the 128-byte (64-key) row
          const int chk = ((warp * KPT) % 64) / 8 + cc;
          const int rh = r, rl = RP + r;
          *reinterpret_cast<uint4*>(pb + rh * 128 + ((chk ^ (rh & 7)) << 4)) =
              make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(pb + rl * 128 + ((chk ^ (rl & 7)) << 4)) =
              make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- O += [P_hi; P_lo] (V_hi + V_lo)
    if (tid == 0) {
      if (!mbar_wait(v_full, ph, err, abort_flag)) {
        *abort_flag = 1;
      } else {
        ++v_seen;
        tc_fence_after();
        const uint32_t idesc = idesc_f32acc_bmn(HD, true);
        const uint32_t pbase = smem_u32(smem + Lay::P_OFF);
        const uint32_t vbase = smem_u32(smem + Lay::KV_OFF + 2 * Lay::PLANE);
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int k = 0; k < CHUNK / 16; ++k)
            tc_mma(tmem + Lay::O_COL,
                   smem_desc_sw128(pbase + (k >> 2) * Lay::P_SUB + (k & 3) * 32),
                   smem_desc_sw128_mn(vbase + t * Lay::PLANE + k * 2048, 2 * Lay::PAGE_SUB, 1024),
                   idesc, (c > 0 || t > 0 || k > 0) ? 1u : 0u);
        tc_commit(pv_done);
        if (c + 1 < n_ch) {
          // the next chunk's scores (their TMEM columns were read out before
          // this chunk's softmax), then its V once this product is done
          issue_s(c + 1);
          if (*abort_flag == 0 && mbar_wait(pv_done, c & 1u, err, abort_flag)) {
            load_half(c + 1, 1, v_full);
            ++v_issued;
          } else {
            *abort_flag = 1;
          }
        }
      }
    }
  }
  // a failed wait may leave copies in flight: they land before the K/V area
  // is reused or the CTA exits
  if (tid == 0 && *abort_flag) {
    if (k_issued > k_seen) mbar_wait(k_full, (k_issued - 1) & 1u, err, nullptr);
    if (v_issued > v_seen) mbar_wait(v_full, (v_issued - 1) & 1u, err, nullptr);
  }
  // ---- O rows: TMEM row r + TMEM row RP + r, unnormalised; rows past the
  // partner's lanes go through shared memory (over P)
  ok = ok && *abort_flag == 0 && n_ch > 0;
  if (ok) ok = mbar_wait(pv_done, (n_ch - 1) & 1u, err, abort_flag);
  ok = __syncthreads_and(ok) != 0;
  tc_fence_after();
  // lane quadrants [0, NQ) hold rows [0, RP), quadrants [NQ, 2 NQ) rows
  // RP.. (the lo products); each warp takes half of the features
  constexpr int NQ = RP / 32;
  constexpr int HH = HD / 2;
  float* xo = reinterpret_cast<float*>(smem + Lay::P_OFF);   // [RP][HD], 16-byte chunks swizzled
  if (ok && quad >= NQ && quad < 2 * NQ) {
    const int r = quad * 32 + lane - RP;
#pragma unroll
    for (int c0 = half * HH; c0 < half * HH + HH; c0 += 32) {
      float o[32];
      tmem_ld32(lane_base + Lay::O_COL + c0, o);
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        const int chk = (c0 + i) >> 2;
        *reinterpret_cast<float4*>(xo + r * HD + ((chk ^ (r & 7)) << 2)) =
            make_float4(o[i], o[i + 1], o[i + 2], o[i + 3]);
      }
    }
  }
  __syncthreads();
  const int my_row = quad * 32 + lane;   // owners (quad < NQ): rows [0, RP)
  const int qr = row0 + my_row;
  const bool valid = qr < rows_total;
  const int pos = valid ? qbase + qr / rep : 0, head = g * rep + (valid ? qr % rep : 0);
  const int hq = H * HD;
  __half* ob = reinterpret_cast<__half*>(p.o);
  const size_t hi_off = (size_t)pair_row(pos) * hq + (size_t)head * HD;
  const size_t lo_off = hi_off + (size_t)PAIR_LO * hq;
  float* xch = reinterpret_cast<float*>(smem + Lay::KV_OFF);   // [RP][XCH_ROW] (n_split > 1)
  if (quad < NQ) {
    const float l_row = ok ? row_l[my_row] : 0.0f;
    const float inv = (ok && valid) ? 1.0f / l_row : 0.0f;
#pragma unroll
    for (int c0 = half * HH; c0 < half * HH + HH; c0 += 32) {
      float o[32];
      if (ok) {
        tmem_ld32(lane_base + Lay::O_COL + c0, o);
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const int chk = (c0 + i) >> 2;
          const float4 v =
              *reinterpret_cast<const float4*>(xo + my_row * HD + ((chk ^ (my_row & 7)) << 2));
          o[i] += v.x;
          o[i + 1] += v.y;
          o[i + 2] += v.z;
          o[i + 3] += v.w;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0.0f;
      }
      if (n_split == 1) {
        if (ok && valid) store_two_term<32>(ob, hi_off + c0, lo_off + c0, o, inv);
      } else {
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(xch + my_row * Lay::XCH_ROW + c0 + i) =
              make_float4(o[i], o[i + 1], o[i + 2], o[i + 3]);
      }
    }
    if (n_split > 1 && half == 0)
      *reinterpret_cast<float4*>(xch + my_row * Lay::XCH_ROW + HD) =
          make_float4(ok ? row_m[my_row] : -INFINITY, ok ? row_l[my_row] : 0.0f, 0.0f, 0.0f);
  }

  if (n_split > 1) {
    // ---- merge the splits: 8-feature group j of every row by split j % n_split
    __syncwarp();
    __syncthreads();
    cluster_sync();
    if (__syncthreads_and(*abort_flag == 0)) {
      const int me = (int)blockIdx.z;
      const int groups = (HD / 8 - me + n_split - 1) / n_split;   // groups of this split
      const uint32_t xbase = smem_u32(xch);
      for (int item = tid; item < RP * groups; item += BLK_THREADS) {
        const int r = item % RP, grp = me + (item / RP) * n_split;
        const int q = row0 + r;
        if (q >= rows_total) continue;
        const uint32_t rowa = xbase + (uint32_t)(r * Lay::XCH_ROW) * 4;
        float4 ml[8], lo4[8], hi4[8];
#pragma unroll
        for (int s2 = 0; s2 < 8; ++s2) {
          if (s2 < n_split) {
            const uint32_t a = cluster_map(rowa, s2);
            ml[s2] = ld_dsmem16(a + HD * 4);
            lo4[s2] = ld_dsmem16(a + grp * 32);
            hi4[s2] = ld_dsmem16(a + grp * 32 + 16);
          } else {
            ml[s2] = make_float4(-INFINITY, 0.0f, 0.0f, 0.0f);
            lo4[s2] = hi4[s2] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
          }
        }
        float mt = -INFINITY;
#pragma unroll
        for (int s2 = 0; s2 < 8; ++s2) mt = fmaxf(mt, ml[s2].x);
        float o[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
        float l_tot = 0.0f;
#pragma unroll
        for (int s2 = 0; s2 < 8; ++s2) {
          const float a = ml[s2].x == -INFINITY ? 0.0f : exp2f(ml[s2].x - mt);
          l_tot += a * ml[s2].y;
          o[0] += a * lo4[s2].x;
          o[1] += a * lo4[s2].y;
          o[2] += a * lo4[s2].z;
          o[3] += a * lo4[s2].w;
          o[4] += a * hi4[s2].x;
          o[5] += a * hi4[s2].y;
          o[6] += a * hi4[s2].z;
          o[7] += a * hi4[s2].w;
        }
        const int pq = qbase + q / rep, hh = g * rep + q % rep;
        const size_t ho = (size_t)pair_row(pq) * hq + (size_t)hh * HD + grp * 8;
        store_two_term<8>(ob, ho, ho + (size_t)PAIR_LO * hq, o, 1.0f / l_tot);
      }
    }
    __syncwarp();
    cluster_sync();   // every split's shared memory has been read
  }

  __syncwarp();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, Lay::TMEM_COLS);
  }
}

template <int HD, int RP>
cudaError_t launch_blk(const CUtensorMap* kvmap, const BlkArgs& a, cudaStream_t st, bool pdl) {
  const int tiles = a.p.tiles ? a.p.n_tiles
                              : (a.p.M * (a.p.n_heads / a.p.n_kv_heads) + RP - 1) / RP;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles, a.p.n_kv_heads, a.p.n_split);
  cfg.blockDim = dim3(BLK_THREADS);
  cfg.dynamicSmemBytes = (size_t)BlkLayout<HD, RP>::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute la[2];
  int na = 0;
  if (a.p.n_split > 1) {   // the key splits of a (row tile, KV head) form one cluster
    la[na].id = cudaLaunchAttributeClusterDimension;
    la[na].val.clusterDim.x = 1;
    la[na].val.clusterDim.y = 1;
    la[na].val.clusterDim.z = a.p.n_split;
    ++na;
  }
  if (pdl) {
    la[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    la[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = la;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, attn_blk_kernel<HD, RP>, *kvmap, a);
}

template <int HD, int RP>
cudaError_t set_blk_attr() {
  return cudaFuncSetAttribute(attn_blk_kernel<HD, RP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              BlkLayout<HD, RP>::SMEM);
}

}  // namespace

int attn_blk_rows(const AttnParams& p) {
  const int rep = p.n_kv_heads > 0 ? p.n_heads / p.n_kv_heads : 0;
  return (p.tiles == nullptr && p.M * rep <= 32) ? 32 : 64;
}

bool attn_blk_supported(const AttnParams& p) {
  const int rep = p.n_kv_heads > 0 ? p.n_heads / p.n_kv_heads : 0;
  if (!(p.kv_planes == 4 && (p.head_dim == 64 || p.head_dim == 128) && rep >= 1 &&
        p.n_heads == rep * p.n_kv_heads && p.M >= 1 && p.L >= 1 &&
        p.keys_per_split >= CHUNK && p.keys_per_split % CHUNK == 0 &&
        p.n_split >= 1 && p.n_split <= 8))
    return false;
  // batched forward: one CTA per table entry (64 query rows of a segment),
  // no key split, keys_per_split covering every segment's keys
  if (p.tiles) return p.n_tiles >= 1 && p.n_split == 1 && p.keys_per_split >= p.L;
  // one sequence: at most 64 block positions; every split holds at least
  // one key and together they cover [0, L)
  return p.M <= 64 && (long long)(p.n_split - 1) * p.keys_per_split < p.L &&
         (long long)p.n_split * p.keys_per_split >= p.L;
}

cudaError_t launch_attn_blk(const CUtensorMap* kvmap, const AttnParams& p, cudaStream_t st,
                            bool pdl) {
  if (!attn_blk_supported(p)) return cudaErrorInvalidValue;
  BlkArgs a{};
  a.p = p;
  a.rp = attn_blk_rows(p);
  a.chunks_per_split = p.keys_per_split / CHUNK;
  if (p.head_dim == 128)
    return a.rp == 32 ? launch_blk<128, 32>(kvmap, a, st, pdl) : launch_blk<128, 64>(kvmap, a, st, pdl);
  return a.rp == 32 ? launch_blk<64, 32>(kvmap, a, st, pdl) : launch_blk<64, 64>(kvmap, a, st, pdl);
}

cudaError_t attn_blk_init_attributes() {
  cudaError_t e = set_blk_attr<128, 32>();
  if (e == cudaSuccess) e = set_blk_attr<128, 64>();
  if (e == cudaSuccess) e = set_blk_attr<64, 32>();
  if (e == cudaSuccess) e = set_blk_attr<64, 64>();
  return e;
}

}  // namespace fd
