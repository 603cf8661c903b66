// The many-token GEMM on pairs of SMs (tcgen05 cta_group::2):
// Y[t, n] = sum_k X[t, k] W[n, k] with W and the two-term X in fp16 (the
// decoder's storage; bf16 for the stand-alone GEMM entry point), for the
// forwards over whole sequences (block-start refresh, cache off, prefix
// cache, batched admission).
//
// A cluster of two CTAs (the two SMs of a TPC) computes one output tile of
// 256 features x 128 tokens per work unit.  The pair's MMA is M = 256 weight
// rows by N = 256 activation rows: CTA r stages weight rows
// [128 r, 128 r + 128) of the tile (its half of A) and activation rows
// [128 r, 128 r + 128) of the token tile (its half of B: the hi and lo terms
// of 64 tokens), and its TMEM receives its 128 weight rows against all 256
// activation rows.  Each CTA's epilogue therefore sees exactly the
// 128-feature x 128-token accumulator of the single-SM kernel (gemm_tc.cu)
// and runs the same epilogues.  Per SM and K block the pair moves 16 KB of
// weights and 16 KB of activations for the tensor work that the single-SM
// 128 x 256 tile needs 16 + 32 KB for: a third less shared-memory fill per
// FLOP, and six K blocks of look-ahead in the space that held four.
//
// Protocol (the even CTA of the pair leads):
//  * TMEM: warp 1 of both CTAs allocates 512 columns with cta_group::2 (the
//    same warp, the same destination word in each CTA).
//  * loads: each CTA's producer waits for its own stage to be free and
//    issues its two TMA loads with cta_group::2, completing on the LEADER's
//    full barrier; the leader's producer alone posts the expected bytes of
//    both halves (the barrier's transaction count may run negative while
//    the peer's bytes arrive first).
//  * MMA: the leader's MMA thread waits on its full barrier, issues the
//    M = 256 MMAs and frees the stage in both CTAs with one commit that
//    arrives on both CTAs' empty barriers; a finished accumulation chain
//    is signalled to both CTAs' epilogues the same way.
//  * epilogue: each CTA drains its own TMEM; lane 0 of each epilogue warp
//    then arrives on the leader's accumulator-empty barrier.
// Every wait is bounded (WAIT_LIMIT_NS) and no role returns early, so both
// CTAs always reach the closing cluster barrier; the leader's MMA thread
// waits for its last MMAs before the pair releases TMEM.  Split-K partial
// tiles and their last-arriver reduction are per CTA (per 128-feature
// tile), with the single-SM kernel's workspace layout.
#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"

namespace fd {

namespace {

constexpr int BK = 64;
constexpr int ROWS = 128;                       // A rows and B rows per CTA
constexpr int A_BYTES = ROWS * BK * 2;          // 16 KB
constexpr int B_BYTES = ROWS * BK * 2;          // 16 KB
constexpr int STAGES = 6;
constexpr int NBUF = 2;                         // TMEM accumulators of 256 columns
constexpr int NCOL = 256;                       // activation rows of the pair's tile
constexpr int TOK = NCOL / 2;                   // tokens per tile
constexpr int EG = 2;                           // epilogue warpgroups
constexpr int EPI_ALL = 128 * EG;
constexpr int EPI_WARPS = EPI_ALL / 32;
constexpr int GT = TOK / EG;                    // tokens per epilogue warpgroup
constexpr int THREADS = 64 + EPI_ALL;
constexpr int A_OFF = 0;
constexpr int B_OFF = A_OFF + STAGES * A_BYTES;
constexpr int STG_OFF = B_OFF + STAGES * B_BYTES;   // SwiGLU staging, 16 KB per group
constexpr int STG_BYTES = CHUNK_T * 128 * 2 * 2;
constexpr int BAR_OFF = STG_OFF + EG * STG_BYTES;
constexpr int N_BARS = 2 * STAGES + 2 * NBUF + 1;
constexpr int MISC_OFF = BAR_OFF + N_BARS * 8;
constexpr int SMEM = MISC_OFF + 16 + 1024;          // slack for 1024-byte alignment
constexpr uint32_t TMEM_COLS = NBUF * NCOL;
constexpr uint32_t PAIR_TX = 2 * (A_BYTES + B_BYTES);   // bytes landing per stage, both CTAs
static_assert(SMEM <= 232448, "exceeds the 227 KB per-CTA shared memory limit");
static_assert(TMEM_COLS <= 512, "TMEM holds 512 columns");
static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "stages stay 1024-byte aligned");

// Epilogue variants, one instantiation each (as in the single-SM kernel).
enum PairEpi : int { PE_REGS = 0, PE_ROWS = 1, PE_STAGED = 2 };

// ------------------------------------------------------------ pair helpers
FD_DEV void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

FD_DEV void tmem_dealloc_pair(uint32_t base, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(ncols)
               : "memory");
}

// D[256 x N] (+)= A[256 x 16] B[N x 16]^T over the pair: A's rows 0..127 and
// B's rows 0..N/2-1 from this CTA's shared memory at the descriptors'
// addresses, the rest from the peer CTA at the same addresses.
FD_DEV void tc_mma_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5, %5, %5, %5, %5}, p;"
      "\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u)
      : "memory");
}

// Arrive once on the mbarrier at this shared-memory offset in every CTA of
// cta_mask when all tcgen05.mma issued so far by this thread are complete.
FD_DEV void tc_commit_pair_mask(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}

// The same, arriving on this CTA's barrier only.
FD_DEV void tc_commit_pair_local(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// TMA tile load into this CTA's shared memory whose completed bytes count
// on the mbarrier at shared::cluster address bar_cluster (the leader's).
FD_DEV void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                             int c1, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}

FD_DEV uint64_t make_policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Arrive on an mbarrier given by its shared::cluster address (this CTA's or
// the peer's), releasing this thread's prior writes at cluster scope.
FD_DEV void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
               : "memory");
}

// Instruction descriptor of the pair MMA: D f32, A and B both fp16 (the
// decoder) or both bf16 (the stand-alone GEMM entry point), K-major,
// N = 256, M = 256.
__host__ __device__ constexpr uint32_t idesc_pair(bool f16) {
  return (1u << 4) | ((f16 ? 0u : 1u) << 7) | ((f16 ? 0u : 1u) << 10) |
         ((uint32_t)(NCOL >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
}

struct PairUnit {
  int ptile, tt, split, kb_lo, kb_hi;
};

// Units are (256-feature pair tile, 128-token tile, K split), numbered like
// the single-SM kernel's (split fastest).
FD_DEV PairUnit pair_unit(const GemmShape& gs, int u) {
  PairUnit c;
  c.split = u % gs.splits;
  const int rest = u / gs.splits;
  c.tt = rest % gs.n_tt;
  c.ptile = rest / gs.n_tt;
  c.kb_lo = (int)((long long)c.split * gs.kb_total / gs.splits);
  c.kb_hi = (int)((long long)(c.split + 1) * gs.kb_total / gs.splits);
  return c;
}

// gs: n_tiles = 128-feature tiles (even), n_tt = 128-token tiles, units =
// n_tiles / 2 * n_tt * splits, grid = 2 x (pairs launched).
template <int EV>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap wmap,
                    const __grid_constant__ CUtensorMap amap, GemmShape gs, EpiParams ep,
                    GemmScratch sc) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* a_st = smem + A_OFF;
  uint8_t* b_st = smem + B_OFF;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* acc_full = bars + 2 * STAGES;
  uint64_t* acc_empty = bars + 2 * STAGES + NBUF;
  uint64_t* mma_done = bars + 2 * STAGES + 2 * NBUF;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(misc + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();   // 0 = the pair's leader
  const bool lead = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < NBUF; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 2 * EPI_WARPS);   // every epilogue warp of both CTAs
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&wmap);
    tma_prefetch_desc(&amap);
  }
  if (warp == 1) tmem_alloc_pair(misc, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // both CTAs' barriers are initialised before any cross-CTA use
  tc_fence_after();
  const uint32_t tmem = misc[0];
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      // The weight tiles do not depend on the previous kernel: the first
      // STAGES of them are requested before waiting for it.
      const uint64_t pol = make_policy_evict_normal();
      uint32_t it = 0;
      bool ok = true;
      int pre = 0;
      {
        int u = pair, kb = 0;
        if (u < gs.units) kb = pair_unit(gs, u).kb_lo;
        while (u < gs.units && pre < STAGES) {
          const PairUnit c = pair_unit(gs, u);
          if (kb >= c.kb_hi) {
            u += n_pairs;
            if (u < gs.units) kb = pair_unit(gs, u).kb_lo;
            continue;
          }
          if (lead) mbar_arrive_expect_tx(&full[pre], PAIR_TX);
          tma_load_2d_pair(a_st + pre * A_BYTES, &wmap, cluster_map(smem_u32(&full[pre]), 0),
                           kb * BK, (c.ptile * 2 + (int)rank) * ROWS, pol);
          ++pre;
          ++kb;
        }
      }
      pdl_wait();   // the activations are the previous kernel's output
      for (int u = pair; u < gs.units && ok; u += n_pairs) {
        const PairUnit c = pair_unit(gs, u);
        const int a_row = (c.ptile * 2 + (int)rank) * ROWS;
        const int b_row = c.tt * NCOL + (int)rank * ROWS;
        for (int kb = c.kb_lo; kb < c.kb_hi; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t bar_lead = cluster_map(smem_u32(&full[s]), 0);
          if (it < (uint32_t)pre) {   // weight half already requested
            tma_load_2d_pair(b_st + s * B_BYTES, &amap, bar_lead, kb * BK, b_row, pol);
            continue;
          }
          if (!mbar_wait(&empty[s], ((it / STAGES) & 1u) ^ 1u, sc.err, abort_flag)) {
            ok = false;
            break;
          }
          FD_CHECK(kb >= 0 && kb < gs.kb_total && 2 * c.ptile + 1 < gs.n_tiles && c.tt < gs.n_tt,
                   ep.check, 26, kb, c.ptile * 65536 + c.tt);
          if (lead) mbar_arrive_expect_tx(&full[s], PAIR_TX);
          tma_load_2d_pair(a_st + s * A_BYTES, &wmap, bar_lead, kb * BK, a_row, pol);
          tma_load_2d_pair(b_st + s * B_BYTES, &amap, bar_lead, kb * BK, b_row, pol);
        }
      }
      if (lead && (!ok || *abort_flag)) {
        // the copies in flight (both CTAs') land before the pair can exit:
        // the peer waits for the leader at the closing cluster barrier
        const uint32_t n = it < (uint32_t)STAGES ? it : (uint32_t)STAGES;
        for (uint32_t j = 0; j < n; ++j) {
          const uint32_t i2 = it - 1 - j;
          mbar_wait(&full[i2 % STAGES], (i2 / STAGES) & 1u, sc.err, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && lead) {
      // ------------------------------------------------------- MMA (leader)
      const uint32_t idesc = idesc_pair(gs.f16 != 0);
      const int KC = gs.kc;
      uint32_t it = 0, chain = 0;
      bool ok = true, issued = false;
      for (int u = pair; u < gs.units && ok; u += n_pairs) {
        const PairUnit c = pair_unit(gs, u);
        for (int k0 = c.kb_lo; k0 < c.kb_hi && ok; k0 += KC, ++chain) {
          const uint32_t buf = chain % NBUF;
          if (!mbar_wait(&acc_empty[buf], ((chain / NBUF) & 1u) ^ 1u, sc.err, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem + buf * NCOL;
          const int k1 = min(k0 + KC, c.kb_hi);
          for (int kb = k0; kb < k1; ++kb, ++it) {
            const int s = it % STAGES;
            if (!mbar_wait(&full[s], (it / STAGES) & 1u, sc.err, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t a0 = smem_u32(a_st + s * A_BYTES);
            const uint32_t b0 = smem_u32(b_st + s * B_BYTES);
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              tc_mma_pair(d, smem_desc_sw128(a0 + k * 32), smem_desc_sw128(b0 + k * 32), idesc,
                          (kb > k0 || k > 0) ? 1u : 0u);
            issued = true;
            tc_commit_pair_mask(&empty[s], 0x3);
          }
          tc_commit_pair_mask(&acc_full[buf], 0x3);
        }
      }
      if (!ok) *abort_flag = 1;
      if (issued) {
        // every MMA of this kernel is complete before the pair frees TMEM
        tc_commit_pair_local(mma_done);
        mbar_wait(mma_done, 0, sc.err, nullptr);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int grp = (warp - 2) >> 2;
    const int quad = warp & 3;
    const int e = quad * 32 + lane;      // feature row = TMEM lane
    const bool leader_thr = threadIdx.x == 64;
    __half* stage = reinterpret_cast<__half*>(smem + STG_OFF + grp * STG_BYTES);
    pdl_wait();
    uint32_t chain = 0;
    for (int u = pair; u < gs.units; u += n_pairs) {
      const PairUnit c = pair_unit(gs, u);
      float acc[GT];
#pragma unroll
      for (int t = 0; t < GT; ++t) acc[t] = 0.0f;
      bool got = true;
      for (int k0 = c.kb_lo; k0 < c.kb_hi; k0 += gs.kc, ++chain) {
        const uint32_t buf = chain % NBUF;
        got = mbar_wait(&acc_full[buf], (chain / NBUF) & 1u, sc.err, abort_flag) && got;
        tc_fence_after();
        // columns [64 g, 64 g + 32) hold the hi term of 32 tokens, the next
        // 32 their lo term; this warpgroup's tokens are [grp GT, grp GT + GT)
        const uint32_t col = tmem + ((uint32_t)(quad * 32) << 16) + buf * NCOL + grp * 2 * GT;
#pragma unroll
        for (int g = 0; g < GT / 32; ++g) {
          float v[64];
          tmem_ld64(col + g * 64, v);
#pragma unroll
          for (int t = 0; t < 32; ++t) acc[g * 32 + t] += v[t] + v[t + 32];
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(cluster_map(smem_u32(&acc_empty[buf]), 0));
      }
      const int tile = c.ptile * 2 + (int)rank;   // this CTA's 128-feature tile
      const int n0 = tile * 128;
      const int tile_id = tile * gs.n_tt + c.tt;
      const int tg0 = c.tt * TOK + grp * GT;
      if (gs.splits > 1) {
        // agree on `got` before the named barriers below
        if (!got) *abort_flag = 1;
        named_bar(1, EPI_ALL);
        if (leader_thr) misc[3] = *abort_flag == 0;
        named_bar(1, EPI_ALL);
        got = misc[3] != 0;
      }
      bool run_epi = gs.splits == 1;
      if (gs.splits > 1) {
        float* ws_unit = sc.ws + ((size_t)tile_id * gs.splits + c.split) * (TOK * 128);
        const size_t wi = (size_t)(ws_unit - sc.ws) + (size_t)(grp * GT + GT - 1) * 128 + e;
        if (FD_CHECK(wi < sc.ws_elems, ep.check, 22, wi, sc.ws_elems)) {
#pragma unroll
          for (int t = 0; t < GT; ++t) ws_unit[(grp * GT + t) * 128 + e] = acc[t];
        }
        __threadfence();
        named_bar(1, EPI_ALL);
        if (leader_thr) {
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
          if (leader_thr) sc.counters[tile_id] = 0;
        }
      }
      if (run_epi && got) {
#pragma unroll
        for (int ch = 0; ch < GT / CHUNK_T; ++ch) {
          float v[CHUNK_T];
#pragma unroll
          for (int t = 0; t < CHUNK_T; ++t) v[t] = acc[ch * CHUNK_T + t];
          if (EV == PE_STAGED)
            epi_staged_f16(ep, v, n0, tg0 + ch * CHUNK_T, e, stage, 2 + grp);
          else
            epi_regs<EV == PE_ROWS>(ep, v, n0, tg0 + ch * CHUNK_T, e);
        }
      }
      if (gs.splits > 1) named_bar(1, EPI_ALL);   // last_flag is read before the next unit
    }
  }

  // Every role of both CTAs arrives here; then the pair releases its TMEM
  // (the leader's MMA thread has seen its last MMAs complete).
  __syncwarp();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

template <int EV>
cudaError_t launch_ev(const CUtensorMap* w_map, const CUtensorMap* act_map, const GemmShape& gs,
                      const EpiParams& ep, const GemmScratch& sc, cudaStream_t st, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(gs.grid);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = SMEM;
  cfg.stream = st;
  cudaLaunchAttribute la[2];
  int na = 0;
  la[na].id = cudaLaunchAttributeClusterDimension;
  la[na].val.clusterDim.x = 2;
  la[na].val.clusterDim.y = 1;
  la[na].val.clusterDim.z = 1;
  ++na;
  if (pdl) {
    la[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    la[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = la;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, gemm_tc2_kernel<EV>, *w_map, *act_map, gs, ep, sc);
}

}  // namespace

int gemm_tc2_smem_bytes() { return SMEM; }

cudaError_t gemm_tc2_init_attributes() {
  for (auto kern : {gemm_tc2_kernel<PE_REGS>, gemm_tc2_kernel<PE_ROWS>,
                    gemm_tc2_kernel<PE_STAGED>}) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

int gemm_tc2_max_pairs() {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = SMEM;
  cudaLaunchAttribute la[1];
  la[0].id = cudaLaunchAttributeClusterDimension;
  la[0].val.clusterDim.x = 2;
  la[0].val.clusterDim.y = 1;
  la[0].val.clusterDim.z = 1;
  cfg.attrs = la;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_tc2_kernel<PE_REGS>, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  return n;
}

cudaError_t launch_gemm_tc2(const CUtensorMap* w_map, const CUtensorMap* act_map,
                            const GemmShape& gs, const EpiParams& ep, const GemmScratch& sc,
                            cudaStream_t st, bool pdl) {
  if (ep.kind == EPI_LMHEAD || gs.nt != NCOL || (gs.n_tiles & 1) || gs.grid < 2 ||
      (gs.grid & 1) || gs.units != gs.n_tiles / 2 * gs.n_tt * gs.splits)
    return cudaErrorInvalidValue;
  if (ep.kind == EPI_SWIGLU) return launch_ev<PE_STAGED>(w_map, act_map, gs, ep, sc, st, pdl);
  if (ep.rows && ep.kind == EPI_QKV) return launch_ev<PE_ROWS>(w_map, act_map, gs, ep, sc, st, pdl);
  return launch_ev<PE_REGS>(w_map, act_map, gs, ep, sc, st, pdl);
}

}  // namespace fd
