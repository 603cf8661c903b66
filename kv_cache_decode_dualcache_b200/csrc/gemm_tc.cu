// Persistent tcgen05 GEMM: Y[t, n] = sum_k X[t, k] W[n, k], W and X both fp16
// (the decoder's storage) or both bf16 (the stand-alone GEMM entry points).
//
// The weight matrix is the 128-row A operand (the "swap-AB" arrangement: the
// model's output features fill the MMA's M = 128; the few block tokens are
// the MMA's N), so a block step with 32 tokens still issues full 128-row
// MMAs while it streams the weights once from HBM.  The activations are
// two-term (hi + lo) in pair rows: every 64 rows hold the hi and the lo term
// of 32 tokens, so a token tile of NT rows covers NT/2 tokens and the lo term
// costs tensor work only (the weights are read once).  Both operands are
// K-major, staged by TMA with the 128-byte swizzle into a STAGES-deep ring of
// shared-memory buffers; one thread issues tcgen05.mma into a ring of NBUF
// TMEM accumulators (128 lanes x NT columns each), one per accumulation chain
// of at most KC K blocks.  The epilogue warps read each chain with
// tcgen05.ld (64 columns: hi and lo of 32 tokens, summed), add the chains up
// in float32 registers and hand the buffer back at once, so the next unit's
// MMAs overlap the epilogue's global-memory work.  The epilogue itself
// (RoPE + KV-cache write, residual add, SwiGLU) runs from registers on the
// permuted weight rows of epi_regs; the fused LM-head max/argmax/sum-exp
// goes through a shared tile (epi_chunk).
//
// Work units are (feature tile, token tile, K split).  CTAs loop over units
// with a stride of gridDim.x.  With more than one split, each split writes
// its float partial tile to a workspace and the last split to arrive (an
// atomic counter per tile, reset by that CTA) sums the partials in split
// order, so results do not depend on arrival order.
//
// Warp roles: warp 0 = TMA producer, warp 1 = TMEM owner and MMA issuer,
// warps 2.. = EG epilogue warpgroups (TMEM lane quadrant = warp % 4; group g
// takes tokens [g * TOK / EG, (g + 1) * TOK / EG) of each tile).  NT = 256
// runs two epilogue warpgroups (320 threads) to hold its 128 tokens of
// accumulators in registers.
#include <type_traits>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"

namespace fd {

namespace {

constexpr int BK = 64;                    // K elements per stage (128 bytes of bf16)
constexpr int A_STAGE_BYTES = 128 * BK * 2;
constexpr int LM_MAX_ROWS = 512;          // largest M for the LM-head epilogue


template <int NT> struct TcCfg;
template <> struct TcCfg<64> { static constexpr int STAGES = 8, NBUF = 4, EG = 1; };
template <> struct TcCfg<128> { static constexpr int STAGES = 6, NBUF = 4, EG = 1; };
template <> struct TcCfg<256> { static constexpr int STAGES = 4, NBUF = 2, EG = 2; };

template <int NT>
struct TcLayout {
  static constexpr int STAGES = TcCfg<NT>::STAGES;
  static constexpr int NBUF = TcCfg<NT>::NBUF;   // TMEM accumulator buffers
  static constexpr int EG = TcCfg<NT>::EG;       // epilogue warpgroups
  static constexpr bool LM = EG == 1;            // LM-head epilogue available
  static constexpr int THREADS = 64 + 128 * EG;
  static constexpr int B_STAGE_BYTES = NT * BK * 2;
  static constexpr int A_OFF = 0;
  static constexpr int B_OFF = A_OFF + STAGES * A_STAGE_BYTES;
  static constexpr int TILE_OFF = B_OFF + STAGES * B_STAGE_BYTES;
  static constexpr int BAR_OFF = TILE_OFF + (LM ? CHUNK_T * 128 * 4 : 0);
  static constexpr int N_BARS = 2 * STAGES + 2 * NBUF;
  static constexpr int MISC_OFF = BAR_OFF + N_BARS * 8;
  static constexpr int LM_OFF = MISC_OFF + 16;
  // staging of the two-term SwiGLU output (epi_staged_f16): 16 KB per
  // epilogue warpgroup; where the LM-head tile exists it serves the one group
  static constexpr int STG_OFF = LM_OFF + (LM ? LM_MAX_ROWS * (int)sizeof(SoftmaxState) : 0);
  static constexpr int STG_BYTES = CHUNK_T * 128 * 2 * 2;
  static constexpr int END = STG_OFF + (LM ? 0 : EG * STG_BYTES);
  static constexpr int SMEM = END + 1024;  // slack for 1024-byte alignment
  static_assert(B_STAGE_BYTES % 1024 == 0, "B stages must stay 1024-byte aligned");
  static_assert(SMEM <= 232448, "exceeds the 227 KB per-CTA shared memory limit");
  static_assert(NBUF * NT <= 512, "TMEM holds 512 columns");
};

struct UnitCoord {
  int tile, tt, split, kb_lo, kb_hi;
};

FD_DEV UnitCoord decode_unit(const GemmShape& gs, int u) {
  UnitCoord c;
  c.split = u % gs.splits;
  const int rest = u / gs.splits;
  c.tt = rest % gs.n_tt;
  c.tile = rest / gs.n_tt;
  c.kb_lo = (int)((long long)c.split * gs.kb_total / gs.splits);
  c.kb_hi = (int)((long long)(c.split + 1) * gs.kb_total / gs.splits);
  return c;
}

// Epilogue variants, one kernel instantiation each (so every variant's
// registers are allocated for its own path only): direct stores from
// registers (and the LM head), the same with the batched forward's per-row
// positions, and the SwiGLU output staged through shared memory.
enum EpiVariant : int { EV_REGS = 0, EV_ROWS = 1, EV_STAGED = 2 };

template <int NT, int EV>
__global__ void __launch_bounds__(TcLayout<NT>::THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap wmap,
                   const __grid_constant__ CUtensorMap amap, GemmShape gs, EpiParams ep,
                   GemmScratch sc) {
  constexpr int TOK = NT / 2;  // tokens per token tile
  using Lay = TcLayout<NT>;
  constexpr int STAGES = Lay::STAGES;
  constexpr int NBUF = Lay::NBUF;
  constexpr int EPI_ALL = 128 * Lay::EG;   // epilogue threads
  constexpr int GT = TOK / Lay::EG;        // tokens per epilogue warpgroup
  // operand type: fp16 (the decoder's weights and two-term activations) or bf16
  const uint32_t idesc = gs.f16 ? idesc_f32acc(NT, true) : idesc_f32acc(NT, false);
  constexpr uint32_t TMEM_COLS = NBUF * NT;
  constexpr uint32_t STAGE_TX = A_STAGE_BYTES + Lay::B_STAGE_BYTES;
  const int KC = gs.kc;  // K blocks per TMEM accumulation chain (see plan_gemm_tc)

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* a_st = smem + Lay::A_OFF;
  uint8_t* b_st = smem + Lay::B_OFF;
  float* tile = reinterpret_cast<float*>(smem + Lay::TILE_OFF);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::BAR_OFF);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* acc_full = bars + 2 * STAGES;
  uint64_t* acc_empty = bars + 2 * STAGES + NBUF;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Lay::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(misc + 2);
  SoftmaxState* lm = reinterpret_cast<SoftmaxState*>(smem + Lay::LM_OFF);
  __half* stage = reinterpret_cast<__half*>(
      Lay::LM ? smem + Lay::TILE_OFF
              : smem + Lay::STG_OFF + ((threadIdx.x >= 64 ? (threadIdx.x - 64) >> 7 : 0) *
                                       Lay::STG_BYTES));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool lmhead = Lay::LM && ep.kind == EPI_LMHEAD;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < NBUF; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], EPI_ALL);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&wmap);
    tma_prefetch_desc(&amap);
  }
  if (warp == 1) tmem_alloc(misc, TMEM_COLS);
  if (lmhead && warp >= 2) {
    for (int t = threadIdx.x - 64; t < gs.M && t < LM_MAX_ROWS; t += EPI_ALL)
      lm[t] = sm_empty();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  pdl_trigger();  // the next kernel may launch onto SMs this grid is not using

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      // The weight tiles do not depend on the previous kernel: the first
      // STAGES of them are requested before waiting for it; activation tiles
      // only after.
      uint32_t it = 0;
      bool ok = true;
      int pre = 0;  // stages whose weight tile was prefetched
      {
        int u = blockIdx.x, kb = 0;
        if (u < gs.units) kb = decode_unit(gs, u).kb_lo;
        while (u < gs.units && pre < STAGES) {
          const UnitCoord c = decode_unit(gs, u);
          if (kb >= c.kb_hi) {
            u += gridDim.x;
            if (u < gs.units) kb = decode_unit(gs, u).kb_lo;
            continue;
          }
          mbar_arrive_expect_tx(&full[pre], STAGE_TX);
          tma_load_2d(a_st + pre * A_STAGE_BYTES, &wmap, &full[pre], kb * BK, c.tile * 128);
          ++pre;
          ++kb;
        }
      }
      pdl_wait();
      for (int u = blockIdx.x; u < gs.units && ok; u += gridDim.x) {
        const UnitCoord c = decode_unit(gs, u);
        for (int kb = c.kb_lo; kb < c.kb_hi; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (it < (uint32_t)pre) {  // weight tile already requested
            tma_load_2d(b_st + s * Lay::B_STAGE_BYTES, &amap, &full[s], kb * BK, c.tt * NT);
            continue;
          }
          if (!mbar_wait(&empty[s], ph ^ 1u, sc.err, abort_flag)) { ok = false; break; }
          FD_CHECK(kb >= 0 && kb < gs.kb_total && c.tile < gs.n_tiles && c.tt < gs.n_tt, ep.check,
                   20, kb, c.tile * 65536 + c.tt);
          mbar_arrive_expect_tx(&full[s], STAGE_TX);
          tma_load_2d(a_st + s * A_STAGE_BYTES, &wmap, &full[s], kb * BK, c.tile * 128);
          tma_load_2d(b_st + s * Lay::B_STAGE_BYTES, &amap, &full[s], kb * BK, c.tt * NT);
        }
      }
      if (!ok || *abort_flag) {
        // Let every copy already issued land before the CTA can exit.
        const uint32_t n = it < (uint32_t)STAGES ? it : (uint32_t)STAGES;
        for (uint32_t j = 0; j < n; ++j) {
          const uint32_t i2 = it - 1 - j;
          mbar_wait(&full[i2 % STAGES], (i2 / STAGES) & 1u, sc.err, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      // Each unit's K range is accumulated in TMEM in chains of at most KC
      // K blocks (one accumulator buffer per chain, NBUF buffers in
      // rotation); the epilogue warps add the chains up in float32 registers
      // and release each buffer as soon as they have read it.
      uint32_t it = 0, chain = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < gs.units && ok; u += gridDim.x) {
        const UnitCoord c = decode_unit(gs, u);
        for (int k0 = c.kb_lo; k0 < c.kb_hi && ok; k0 += KC, ++chain) {
          const uint32_t buf = chain % NBUF;
          if (!mbar_wait(&acc_empty[buf], ((chain / NBUF) & 1u) ^ 1u, sc.err, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem + buf * NT;
          const int k1 = min(k0 + KC, c.kb_hi);
          for (int kb = k0; kb < k1; ++kb, ++it) {
            const int s = it % STAGES;
            if (!mbar_wait(&full[s], (it / STAGES) & 1u, sc.err, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t a0 = smem_u32(a_st + s * A_STAGE_BYTES);
            const uint32_t b0 = smem_u32(b_st + s * Lay::B_STAGE_BYTES);
#pragma unroll
            for (int k = 0; k < BK / 16; ++k) {
              tc_mma(d, smem_desc_sw128(a0 + k * 32), smem_desc_sw128(b0 + k * 32), idesc,
                     (kb > k0 || k > 0) ? 1u : 0u);
            }
            tc_commit(&empty[s]);
          }
          tc_commit(&acc_full[buf]);
        }
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    // Warpgroup grp handles tokens [grp * GT, (grp + 1) * GT) of each token
    // tile; its warps read TMEM lane quadrant warp % 4 (feature rows).
    const int grp = (warp - 2) >> 2;
    const int quad = warp & 3;
    const int e = quad * 32 + lane;  // feature row = TMEM lane
    const bool leader = warp == 2 && lane == 0;
    pdl_wait();                      // reads / writes of the previous kernel's data follow
    uint32_t chain = 0;
    for (int u = blockIdx.x; u < gs.units; u += gridDim.x) {
      const UnitCoord c = decode_unit(gs, u);
      // acc[t] = this lane's feature for token grp * GT + t of the tile: the
      // sum over the unit's accumulation chains of the hi- and lo-term
      // columns (columns [64g, 64g+32) of a chain buffer hold the hi term of
      // tokens 32g.., the next 32 their lo term).
      float acc[GT];
#pragma unroll
      for (int t = 0; t < GT; ++t) acc[t] = 0.0f;
      bool got = true;
      for (int k0 = c.kb_lo; k0 < c.kb_hi; k0 += KC, ++chain) {
        const uint32_t buf = chain % NBUF;
        got = mbar_wait(&acc_full[buf], (chain / NBUF) & 1u, sc.err, abort_flag) && got;
        tc_fence_after();
        const uint32_t col = tmem + ((uint32_t)(quad * 32) << 16) + buf * NT + grp * 2 * GT;
#pragma unroll
        for (int g = 0; g < GT / 32; ++g) {
          float v[64];
          tmem_ld64(col + g * 64, v);
#pragma unroll
          for (int t = 0; t < 32; ++t) acc[g * 32 + t] += v[t] + v[t + 32];
        }
        tc_fence_before();
        mbar_arrive(&acc_empty[buf]);
      }
      const int n0 = c.tile * 128;
      const int tile_id = c.tile * gs.n_tt + c.tt;
      const int tg0 = c.tt * TOK + grp * GT;  // first token row of this warpgroup
      if (lmhead || gs.splits > 1) {
        // the paths below have named barriers: agree on `got` first (one
        // thread samples the flags), so a failed wait in one thread cannot
        // leave the others at a barrier
        if (!got) *abort_flag = 1;
        named_bar(1, EPI_ALL);
        if (threadIdx.x == 64) misc[3] = *abort_flag == 0;
        named_bar(1, EPI_ALL);
        got = misc[3] != 0;
      }
      bool run_epi = gs.splits == 1;
      if (gs.splits > 1) {
        // float partial tile [TOK][128] of this split; the last split to
        // arrive sums all of them in split order and runs the epilogue.
        float* ws_unit = sc.ws + ((size_t)tile_id * gs.splits + c.split) * (TOK * 128);
        const size_t wi = (size_t)(ws_unit - sc.ws) + (size_t)(grp * GT + GT - 1) * 128 + e;
        if (FD_CHECK(wi < sc.ws_elems, ep.check, 22, wi, sc.ws_elems)) {
#pragma unroll
          for (int t = 0; t < GT; ++t) ws_unit[(grp * GT + t) * 128 + e] = acc[t];
        }
        __threadfence();
        named_bar(1, EPI_ALL);
        if (leader) {
          int prev = -1;
          if (FD_CHECK(tile_id < sc.n_counters, ep.check, 23, tile_id, sc.n_counters))
            prev = atomicAdd(&sc.counters[tile_id], 1);
          *last_flag = (prev == gs.splits - 1);
        }
        named_bar(1, EPI_ALL);
        run_epi = *last_flag;
        if (run_epi) {
          __threadfence();
          const float* ws_tile = sc.ws + (size_t)tile_id * gs.splits * (TOK * 128);
#pragma unroll
          for (int t = 0; t < GT; ++t) acc[t] = 0.0f;
          for (int sp = 0; sp < gs.splits; ++sp) {
            const float* p = ws_tile + (size_t)sp * (TOK * 128) + (size_t)grp * GT * 128 + e;
            const size_t pi = (size_t)(p - sc.ws) + (size_t)(GT - 1) * 128;
            if (!FD_CHECK(pi < sc.ws_elems, ep.check, 24, pi, sc.ws_elems)) continue;
#pragma unroll
            for (int t = 0; t < GT; ++t) acc[t] += __ldcg(p + t * 128);
          }
          if (leader) sc.counters[tile_id] = 0;
        }
      }
      if (run_epi && got) {
#pragma unroll
        for (int ch = 0; ch < GT / CHUNK_T; ++ch) {
          float v[CHUNK_T];
#pragma unroll
          for (int t = 0; t < CHUNK_T; ++t) v[t] = acc[ch * CHUNK_T + t];
          if (lmhead) {
            // all 128 features of a token meet in the shared tile
            named_bar(1, EPI_ALL);  // previous chunk's reduction is done with `tile`
#pragma unroll
            for (int t = 0; t < CHUNK_T; ++t) tile[t * 128 + e] = v[t];
            named_bar(1, EPI_ALL);
            epi_chunk(ep, tile, n0, tg0 + ch * CHUNK_T, e, lm);
          } else if (EV == EV_STAGED) {
            // 16-byte stores through shared memory (measured: gate/up 7 %
            // faster; the QKV epilogue is faster with its direct stores)
            epi_staged_f16(ep, v, n0, tg0 + ch * CHUNK_T, e, stage, 2 + grp);
          } else {
            epi_regs<EV == EV_ROWS>(ep, v, n0, tg0 + ch * CHUNK_T, e);
          }
        }
      }
      if (gs.splits > 1) named_bar(1, EPI_ALL);  // last_flag is read before the next unit
    }
  }

  // lanes 1..31 of the single-thread role warps reach this point long before
  // their lane 0: reconverge every warp first, so that the CTA barrier below
  // counts each warp once, with all of its threads
  __syncwarp();
  __syncthreads();
  if (lmhead && warp >= 2) {
    SoftmaxState* out = reinterpret_cast<SoftmaxState*>(ep.lm_part) + (size_t)blockIdx.x * gs.M;
    for (int t = threadIdx.x - 64; t < gs.M && t < LM_MAX_ROWS; t += EPI_ALL) {
      const size_t i = (size_t)blockIdx.x * gs.M + t;
      if (FD_CHECK(i < ep.cap_lm, ep.check, 25, i, ep.cap_lm)) out[t] = lm[t];
    }
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int NT>
cudaError_t set_attr_nt() {
  cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<NT, EV_REGS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       TcLayout<NT>::SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gemm_tc_kernel<NT, EV_ROWS>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, TcLayout<NT>::SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gemm_tc_kernel<NT, EV_STAGED>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, TcLayout<NT>::SMEM);
  return e;
}

template <int NT>
cudaError_t launch_nt(const CUtensorMap* w_map, const CUtensorMap* act_map, const GemmShape& gs,
                      const EpiParams& ep, const GemmScratch& sc, cudaStream_t st, bool pdl) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = set_attr_nt<NT>();
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  auto* kern = ep.kind == EPI_SWIGLU ? gemm_tc_kernel<NT, EV_STAGED>
               : (ep.rows && ep.kind == EPI_QKV) ? gemm_tc_kernel<NT, EV_ROWS>
                                                 : gemm_tc_kernel<NT, EV_REGS>;
  return launch_k(pdl, kern, dim3(gs.grid), dim3(TcLayout<NT>::THREADS),
                  (size_t)TcLayout<NT>::SMEM, st, *w_map, *act_map, gs, ep, sc);
}

}  // namespace

int gemm_tc_smem_bytes(int nt) {
  switch (nt) {
    case 64: return TcLayout<64>::SMEM;
    case 128: return TcLayout<128>::SMEM;
    case 256: return TcLayout<256>::SMEM;
    default: return -1;
  }
}

cudaError_t launch_gemm_tc(const CUtensorMap* w_map, const CUtensorMap* act_map,
                           const GemmShape& gs, const EpiParams& ep, const GemmScratch& sc,
                           cudaStream_t st, bool pdl) {
  if (ep.kind == EPI_LMHEAD && (gs.M > LM_MAX_ROWS || gs.nt > 128)) return cudaErrorInvalidValue;
  switch (gs.nt) {
    case 64: return launch_nt<64>(w_map, act_map, gs, ep, sc, st, pdl);
    case 128: return launch_nt<128>(w_map, act_map, gs, ep, sc, st, pdl);
    case 256: return launch_nt<256>(w_map, act_map, gs, ep, sc, st, pdl);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t gemm_tc_init_attributes() {
  cudaError_t e = set_attr_nt<64>();
  if (e == cudaSuccess) e = set_attr_nt<128>();
  if (e == cudaSuccess) e = set_attr_nt<256>();
  return e;
}

}  // namespace fd
