// Persistent multi-phase kernel of the DualCache block step (bf16 model,
// block of at most 32 tokens): one launch runs a short program of phases
//   EMBED_NORM  h = E[x[r0 ..]], a = RMSNorm(h) * g
//   NORM        a = RMSNorm(h) * g
//   GEMM        tcgen05 GEMM with a fused epilogue (QKV + RoPE + KV write,
//               residual add, SwiGLU, or the LM-head max/argmax/sum-exp)
// for example [O-proj, NORM, gate/up, down, NORM, next layer's QKV], so that
// the only launch boundary left per layer is the attention kernel.
//
// Why: at 32 tokens every GEMM of the step is a weight stream from HBM of
// 33-200 MB, and a separate launch per GEMM pays a pipeline fill, a split-K
// reduction tail and a grid drain each time.  Here the weight tiles of every
// GEMM of the program stream through one shared-memory ring without a break:
// the weight producer never waits for a phase, so while the grid finishes a
// phase (its last reductions, a norm) the next GEMM's weights are already in
// flight.  Only the activation producer and the worker warps wait for the
// previous phase.
//
// Phase completion: each CTA adds 1 to done[p] once its workers have
// finished (and fenced) all of its work of phase p; phase p + 1's
// activation loads and its non-GEMM work wait until done[p] == gridDim.x.
// Every phase has at least one CTA that waits for its predecessor, so
// done[p] == gridDim.x implies that every earlier phase is complete.  The
// grid must be co-resident (one CTA per SM, cooperative launch); every wait
// is bounded (WAIT_LIMIT_NS) and a timeout sets DEV_ERR_TIMEOUT, raises a
// grid-wide abort word and ends the kernel.
//
// GEMM work units are (feature tile of 128 weight rows, K split) over the
// single token tile (64 two-term rows = 32 tokens); unit u of a phase runs
// on CTA (u + rot) % gridDim.x, the rotation continuing from the previous
// phase so that CTAs left idle by one phase get the next one's first units.
// Split-K partials are reduced by the last split to arrive, in split order.
//
// Warp roles (224 threads): warp 0 = weight (A) producer, warp 1 = TMEM
// owner and MMA issuer, warp 2 = activation (B) producer, warps 3..6 =
// workers (TMEM lane quadrant = warp % 4): accumulator drain and epilogue,
// norms.
#include <climits>

#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.h"

namespace fd {

namespace {

constexpr int BK = 64;                   // K elements per stage
constexpr int NT = 64;                   // token-tile rows (32 tokens, two-term)
constexpr int TOK = 32;
constexpr int STAGES = 8;
constexpr int NBUF = 4;                  // TMEM accumulator buffers (64 columns each)
constexpr int WORKERS = 128;
constexpr int THREADS = 96 + WORKERS;
constexpr uint32_t A_BYTES = 128 * BK * 2;
constexpr uint32_t B_BYTES = NT * BK * 2;
constexpr int A_OFF = 0;
constexpr int B_OFF = A_OFF + STAGES * A_BYTES;
constexpr int TILE_OFF = B_OFF + STAGES * B_BYTES;       // [32][128] float (LM head)
constexpr int RED_OFF = TILE_OFF + CHUNK_T * 128 * 4;    // norm reduction (4 floats)
constexpr int LM_OFF = RED_OFF + 64;                     // [TOK] softmax states
constexpr int BAR_OFF = LM_OFF + TOK * (int)sizeof(SoftmaxState);
constexpr int UQ = 16;                   // unit queue entries (weight producer -> other roles)
constexpr int N_BARS = 3 * STAGES + 2 * NBUF + 1 + 2 * UQ;
constexpr int MISC_OFF = BAR_OFF + N_BARS * 8;
constexpr int UQ_OFF = MISC_OFF + 16;  // [UQ] unit ids, then the workers' broadcast word
constexpr int PH_OFF = (UQ_OFF + (UQ + 1) * 4 + 127) / 128 * 128;  // workers' copy of the phase
constexpr int SMEM = PH_OFF + (int)sizeof(ChainPhase) + 1024;
static_assert(SMEM <= 232448, "exceeds the 227 KB per-CTA shared memory limit");
static_assert(BAR_OFF % 8 == 0, "mbarriers need 8-byte alignment");

struct Unit {
  int tile, split, kb_lo, kb_hi;
};

// The fields of a phase the producer and MMA loops use, read once per phase
// into registers.
struct Geom {
  int type, units, splits, kb_total, rot, kc;
};

FD_DEV Geom geom_of(const ChainPhase& P) {
  return Geom{P.type, P.units, P.splits, P.kb_total, P.rot, P.kc};
}

FD_DEV Unit unit_of(const Geom& P, int u) {
  Unit c;
  c.split = u % P.splits;
  c.tile = u / P.splits;
  c.kb_lo = (int)((long long)c.split * P.kb_total / P.splits);
  c.kb_hi = (int)((long long)(c.split + 1) * P.kb_total / P.splits);
  return c;
}

// First unit of phase P that runs on CTA c.
FD_DEV int first_unit(const Geom& P, int c, int G) {
  int u = (c - P.rot) % G;
  return u < 0 ? u + G : u;
}

// Release add at gpu scope, no return value: publishes the writes ordered
// before it (after a CTA barrier, the whole CTA's) without a separate fence.
FD_DEV void red_add_release_gpu(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

FD_DEV int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

FD_DEV int ld_relaxed(const int* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Bounded wait until *ctr >= target (every CTA of the grid has finished the
// phase), then an acquire load of it (it synchronizes with the arrivals'
// release reductions; measured 3 % less block-step time than a fence on
// either side of relaxed operations).  Relaxed polls with a growing sleep keep
// the counter's L2 slice free for the arrivals and for the data traffic.
// false on timeout (DEV_ERR_TIMEOUT, grid abort raised) or abort.
FD_DEV bool grid_wait(const int* ctr, int target, int* err, int* gabort) {
  if (ld_relaxed(ctr) < target) {
    const uint64_t t0 = global_timer_ns();
    uint32_t ns = 64;
    for (uint32_t it = 1;; ++it) {
      __nanosleep(ns);
      if (ns < 256) ns *= 2;
      if (ld_relaxed(ctr) >= target) break;
      if ((it & 7u) == 0) {
        if (*(volatile int*)gabort) return false;
        if (global_timer_ns() - t0 > (uint64_t)WAIT_LIMIT_NS) {
          atomicOr(err, DEV_ERR_TIMEOUT);
          atomicExch(gabort, 1);
          return false;
        }
      }
    }
  }
  (void)ld_acquire(ctr);
  return true;
}

// Generic-proxy writes of other CTAs (made visible by grid_wait's acquire)
// are read next through the async proxy (TMA).
FD_DEV void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// NORM / EMBED_NORM phase: a[row] = RMSNorm(h[row]) * g as two-term fp16
// pair rows, spread over every CTA.  Work items are (row, 512-feature group)
// pairs, item i on CTA (i + rot) % G; a worker thread owns 4 consecutive
// features of an item.  First every item of the CTA loads its features
// (EMBED_NORM: gathers them from the bf16 embedding table; NORM with
// resid_splits: adds the preceding residual GEMM's split partials, in split
// order, and stores h back), all loads of an item in flight at once, and
// publishes its partial sum of squares (ss[row][group], then one arrival on
// the row's counter).  Only then does any item wait for its row's other
// groups, so no CTA can wait on an item that waits on it.  The row total
// sums the groups in group order.
constexpr int NORM_MAX_ITEMS = 4;   // per CTA: M * (d / 512) <= 4 * gridDim.x
constexpr int NORM_MAX_SPLITS = 16;

FD_DEV bool norm_phase(const ChainArgs& A, const ChainPhase& P, int p, int cta, int G, int wt,
                       float* red, volatile int* flag, int* err) {
  const int d = A.d;
  const int ng = d >> 9;
  const int n_items = A.M * ng;
  const bool leader = wt == 0;
  int* rowcnt = A.rowcnt + p * 32;
  int first = (cta - P.rot) % G;
  if (first < 0) first += G;
  float4 v[NORM_MAX_ITEMS];
  // ---- load, partial sum of squares, publish
  int k = 0;
  for (int item = first; item < n_items && k < NORM_MAX_ITEMS; item += G, ++k) {
    const int row = item / ng, g = item - row * ng;
    const int j = g * 512 + wt * 4;
    float* hj = A.h + (size_t)row * d + j;
    float4 x;
    if (P.type == CH_EMBED_NORM) {
      const int r0 = A.sp ? A.sp->r0 : 0;
      int tok = A.x[r0 + row];
      if (tok < 0 || tok >= A.vocab) {
        if (leader) atomicOr(err, DEV_ERR_TOKEN);
        tok = 0;
      }
      const uint2 raw = __ldg(reinterpret_cast<const uint2*>(
          reinterpret_cast<const __nv_bfloat16*>(A.embed) + (size_t)tok * d + j));
      const __nv_bfloat162 lo2 = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
      const __nv_bfloat162 hi2 = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
      x = make_float4(__low2float(lo2), __high2float(lo2), __low2float(hi2), __high2float(hi2));
      *reinterpret_cast<float4*>(hj) = x;
    } else {
      const int S = P.resid_splits;
      // partial tiles [tile][split][token][128]; feature j lies in tile j / 128
      const float* pp = A.sc.ws + (((size_t)(j >> 7) * S) * TOK + row) * 128 + (j & 127);
      float4 pv[NORM_MAX_SPLITS];
      x = __ldcg(reinterpret_cast<const float4*>(hj));
#pragma unroll
      for (int sp = 0; sp < NORM_MAX_SPLITS; ++sp)
        if (sp < S) pv[sp] = __ldcg(reinterpret_cast<const float4*>(pp + (size_t)sp * TOK * 128));
#pragma unroll
      for (int sp = 0; sp < NORM_MAX_SPLITS; ++sp) {
        if (sp < S) {
          x.x += pv[sp].x;
          x.y += pv[sp].y;
          x.z += pv[sp].z;
          x.w += pv[sp].w;
        }
      }
      if (S > 0) *reinterpret_cast<float4*>(hj) = x;
    }
    v[k] = x;
    float ss = warp_sum(x.x * x.x + x.y * x.y + x.z * x.z + x.w * x.w);
    named_bar(2, WORKERS);  // red is free
    if ((wt & 31) == 0) red[wt >> 5] = ss;
    named_bar(2, WORKERS);
    if (leader) {
      A.norm_ss[row * CHAIN_NORM_GROUPS + g] = (red[0] + red[1]) + (red[2] + red[3]);
      red_add_release_gpu(rowcnt + row, 1);
    }
  }
  // ---- per item: wait for the row's groups, normalise, store
  bool ok = true;
  k = 0;
  for (int item = first; item < n_items && k < NORM_MAX_ITEMS; item += G, ++k) {
    const int row = item / ng, g = item - row * ng;
    const int j = g * 512 + wt * 4;
    if (leader) *flag = grid_wait(rowcnt + row, ng, err, A.gabort) ? 1 : 0;
    named_bar(2, WORKERS);
    ok = *flag != 0;
    named_bar(2, WORKERS);
    if (!ok) break;
    float tot = 0.0f;
    for (int q = 0; q < ng; ++q) tot += __ldcg(A.norm_ss + row * CHAIN_NORM_GROUPS + q);
    const float inv = 1.0f / sqrtf(tot / (float)d + A.eps);
    const float4 gn = __ldg(reinterpret_cast<const float4*>(P.gain + j));
    const float4 x = v[k];
    __half h0, l0, h1, l1, h2, l2, h3, l3;
    split_f16(x.x * inv * gn.x, h0, l0);
    split_f16(x.y * inv * gn.y, h1, l1);
    split_f16(x.z * inv * gn.z, h2, l2);
    split_f16(x.w * inv * gn.w, h3, l3);
    __half2 hh[2] = {__halves2half2(h0, h1), __halves2half2(h2, h3)};
    __half2 ll[2] = {__halves2half2(l0, l1), __halves2half2(l2, l3)};
    __half* ab = reinterpret_cast<__half*>(A.a);
    const size_t r_hi = (size_t)pair_row(row) * d, r_lo = r_hi + (size_t)PAIR_LO * d;
    *reinterpret_cast<uint2*>(ab + r_hi + j) = *reinterpret_cast<const uint2*>(hh);
    *reinterpret_cast<uint2*>(ab + r_lo + j) = *reinterpret_cast<const uint2*>(ll);
  }
  return ok;
}

__global__ void __launch_bounds__(THREADS, 1) chain_kernel(const __grid_constant__ ChainArgs A) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* a_st = smem + A_OFF;
  uint8_t* b_st = smem + B_OFF;
  float* tile = reinterpret_cast<float*>(smem + TILE_OFF);
  float* red = reinterpret_cast<float*>(smem + RED_OFF);
  SoftmaxState* lm = reinterpret_cast<SoftmaxState*>(smem + LM_OFF);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* full_a = bars;
  uint64_t* full_b = bars + STAGES;
  uint64_t* empty = bars + 2 * STAGES;
  uint64_t* acc_full = bars + 3 * STAGES;
  uint64_t* acc_empty = bars + 3 * STAGES + NBUF;
  uint64_t* mma_done = bars + 3 * STAGES + 2 * NBUF;
  uint64_t* uq_full = mma_done + 1;
  uint64_t* uq_empty = uq_full + UQ;
  volatile int* uq = reinterpret_cast<volatile int*>(smem + UQ_OFF);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + MISC_OFF);
  ChainPhase* sph = reinterpret_cast<ChainPhase*>(smem + PH_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(misc + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int cta = blockIdx.x;
  int* err = A.sc.err;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full_a[i], 1);
      mbar_init(&full_b[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < NBUF; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], WORKERS);
    }
    mbar_init(mma_done, 1);
    for (int i = 0; i < UQ; ++i) {
      mbar_init(&uq_full[i], 1);
      mbar_init(&uq_empty[i], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(misc, NBUF * NT);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------- weight (A) producer
      // Also the unit scheduler: it claims each GEMM phase's units (from the
      // phase's global counter, so CTAs that stream faster take more units;
      // the LM head keeps its static round-robin assignment, since the
      // merge of its per-CTA softmax states must not depend on timing) and
      // queues each unit id, then -1 at the phase end, for the other roles.
      uint32_t it = 0, qi = 0;
      bool ok = true;
      const uint64_t stream_once = make_policy_evict_first();
      auto push = [&](int u) -> bool {
        const int slot = qi % UQ;
        if (!mbar_wait(&uq_empty[slot], ((qi / UQ) & 1u) ^ 1u, err, abort_flag)) return false;
        uq[slot] = u;
        mbar_arrive(&uq_full[slot]);  // release: the write above is visible to its waiters
        ++qi;
        return true;
      };
      for (int p = 0; p < A.n_phases && ok; ++p) {
        const Geom P = geom_of(A.ph[p]);
        if (P.type != CH_GEMM) continue;
        const bool dyn = A.ph[p].ep.kind != EPI_LMHEAD;
        int* next = A.next + p * CHAIN_DONE_STRIDE;
        const CUtensorMap* wmap = &A.ph[p].wmap;
        tma_prefetch_desc(wmap);
        int u = dyn ? atomicAdd(next, 1) : first_unit(P, cta, G);
        while (u < P.units && ok) {
          if (!push(u)) { ok = false; break; }
          const Unit c = unit_of(P, u);
          int u_next = P.units;
          for (int kb = c.kb_lo; kb < c.kb_hi; ++kb, ++it) {
            // claim the next unit while this unit's last stages are in flight
            if (kb == c.kb_hi - 1) u_next = dyn ? atomicAdd(next, 1) : u + G;
            const int s = it % STAGES;
            if (!mbar_wait(&empty[s], ((it / STAGES) & 1u) ^ 1u, err, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full_a[s], A_BYTES);
            tma_load_2d_hint(a_st + s * A_BYTES, wmap, &full_a[s], kb * BK, c.tile * 128,
                             stream_once);
          }
          u = u_next;
        }
        if (ok && !push(-1)) ok = false;  // end of this CTA's share of phase p
        if (*(volatile int*)A.gabort) ok = false;
      }
      if (!ok) {
        *abort_flag = 1;
        const uint32_t n = it < (uint32_t)STAGES ? it : (uint32_t)STAGES;
        for (uint32_t j = 0; j < n; ++j) {
          const uint32_t i2 = it - 1 - j;
          mbar_wait(&full_a[i2 % STAGES], (i2 / STAGES) & 1u, err, nullptr);
        }
      }
    }
  } else if (warp == 2) {
    if (lane == 0) {
      // ---------------------------------------------- activation (B) producer
      uint32_t it = 0, qi = 0;
      bool ok = true;
      for (int p = 0; p < A.n_phases && ok; ++p) {
        const Geom P = geom_of(A.ph[p]);
        if (P.type != CH_GEMM) continue;
        const CUtensorMap* amap = &A.ph[p].amap;
        // phase 0 reads the previous kernel's output (programmatic launch:
        // wait until that kernel has completed)
        bool ready = p == 0;
        if (p == 0) pdl_wait();
        for (;;) {
          const int slot = qi % UQ;
          if (!mbar_wait(&uq_full[slot], (qi / UQ) & 1u, err, abort_flag)) { ok = false; break; }
          const int u = uq[slot];
          ++qi;
          if (u < 0) break;
          if (!ready) {
            // the activations of phase p are complete once every CTA has
            // finished phase p - 1
            tma_prefetch_desc(amap);
            if (!grid_wait(A.done + (p - 1) * CHAIN_DONE_STRIDE, G, err, A.gabort)) {
              ok = false;
              break;
            }
            fence_proxy_async_global();
            ready = true;
          }
          const Unit c = unit_of(P, u);
          for (int kb = c.kb_lo; kb < c.kb_hi; ++kb, ++it) {
            const int s = it % STAGES;
            if (!mbar_wait(&empty[s], ((it / STAGES) & 1u) ^ 1u, err, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full_b[s], B_BYTES);
            tma_load_2d(b_st + s * B_BYTES, amap, &full_b[s], kb * BK, 0);
          }
          if (!ok) break;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        const uint32_t n = it < (uint32_t)STAGES ? it : (uint32_t)STAGES;
        for (uint32_t j = 0; j < n; ++j) {
          const uint32_t i2 = it - 1 - j;
          mbar_wait(&full_b[i2 % STAGES], (i2 / STAGES) & 1u, err, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------- MMA issuer
      const uint32_t idesc = idesc_f32acc(NT, true);
      uint32_t it = 0, chain = 0, qi = 0;
      bool ok = true;
      for (int p = 0; p < A.n_phases && ok; ++p) {
        const Geom P = geom_of(A.ph[p]);
        if (P.type != CH_GEMM) continue;
        for (;;) {
          const int slot = qi % UQ;
          if (!mbar_wait(&uq_full[slot], (qi / UQ) & 1u, err, abort_flag)) { ok = false; break; }
          const int u = uq[slot];
          ++qi;
          if (u < 0) break;
          const Unit c = unit_of(P, u);
          for (int k0 = c.kb_lo; k0 < c.kb_hi && ok; k0 += P.kc, ++chain) {
            const uint32_t buf = chain % NBUF;
            if (!mbar_wait(&acc_empty[buf], ((chain / NBUF) & 1u) ^ 1u, err, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t d = tmem + buf * NT;
            const int k1 = min(k0 + P.kc, c.kb_hi);
            for (int kb = k0; kb < k1; ++kb, ++it) {
              const int s = it % STAGES;
              const uint32_t ph = (it / STAGES) & 1u;
              if (!mbar_wait(&full_a[s], ph, err, abort_flag) ||
                  !mbar_wait(&full_b[s], ph, err, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t a0 = smem_u32(a_st + s * A_BYTES);
              const uint32_t b0 = smem_u32(b_st + s * B_BYTES);
#pragma unroll
              for (int k = 0; k < BK / 16; ++k)
                tc_mma(d, smem_desc_sw128(a0 + k * 32), smem_desc_sw128(b0 + k * 32), idesc,
                       (kb > k0 || k > 0) ? 1u : 0u);
              tc_commit(&empty[s]);
            }
            tc_commit(&acc_full[buf]);
          }
        }
      }
      if (!ok) *abort_flag = 1;
      // every MMA this thread issued has completed before TMEM is released
      tc_commit(mma_done);
      mbar_wait(mma_done, 0, err, nullptr);
    }
  } else {
    // -------------------------------------------------- workers
    const int wt = threadIdx.x - 96;   // 0 .. 127
    const int quad = warp & 3;
    const int e = quad * 32 + lane;    // feature row = TMEM lane
    const bool leader = wt == 0;
    uint32_t chain = 0, wq = 0;
    bool ok = true;
    for (int p = 0; p < A.n_phases; ++p) {
      // the epilogues and norms read the phase from shared memory: loads
      // through a runtime-indexed address into parameter space are slow
      {
        const uint4* src = reinterpret_cast<const uint4*>(&A.ph[p]);
        uint4* dst = reinterpret_cast<uint4*>(sph);
        for (int i = wt; i < (int)(sizeof(ChainPhase) / 16); i += WORKERS) dst[i] = src[i];
        named_bar(1, WORKERS);
      }
      const ChainPhase& P = *sph;
      const Geom PG = geom_of(P);
      if (ok && P.type == CH_GEMM) {
        const bool lmh = P.ep.kind == EPI_LMHEAD;
        if (lmh) {
          for (int t = wt; t < TOK; t += WORKERS) lm[t] = sm_empty();
          named_bar(1, WORKERS);
        }
        for (;;) {
          // next unit from the weight producer's queue (the leader waits and
          // broadcasts it, so every worker takes the same path)
          const int slot = wq % UQ;
          if (leader)
            uq[UQ] = mbar_wait(&uq_full[slot], (wq / UQ) & 1u, err, abort_flag) ? uq[slot]
                                                                                : INT_MIN;
          named_bar(1, WORKERS);
          const int u = uq[UQ];
          if (u == INT_MIN) {
            ok = false;
            break;
          }
          if (u < 0) {  // end of this CTA's share of the phase
            named_bar(1, WORKERS);
            if (leader) mbar_arrive(&uq_empty[slot]);
            ++wq;
            break;
          }
          {
          const Unit c = unit_of(PG, u);
          float acc[TOK];
#pragma unroll
          for (int t = 0; t < TOK; ++t) acc[t] = 0.0f;
          bool got = true;
          for (int k0 = c.kb_lo; k0 < c.kb_hi; k0 += P.kc, ++chain) {
            const uint32_t buf = chain % NBUF;
            got = got && mbar_wait(&acc_full[buf], (chain / NBUF) & 1u, err, abort_flag);
            tc_fence_after();
            if (got) {
              // columns [0, 32) hold the hi term of the 32 tokens, [32, 64) the
              // lo term; 16 tokens at a time keeps 32 registers in flight
              const uint32_t col = tmem + ((uint32_t)(quad * 32) << 16) + buf * NT;
#pragma unroll
              for (int h = 0; h < TOK; h += 16) {
                float hi[16], lo[16];
                tmem_ld16x2<32>(col + h, hi, lo);
#pragma unroll
                for (int t = 0; t < 16; ++t) acc[h + t] += hi[t] + lo[t];
              }
            }
            tc_fence_before();
            mbar_arrive(&acc_empty[buf]);
          }
          if (!got) ok = false;
          const int n0 = c.tile * 128;
          if (P.ep.kind == EPI_RESID) {
            // residual GEMM: every split stores its partial tile; the next
            // NORM phase adds h and the partials in split order
            float* ws_unit = A.sc.ws + ((size_t)c.tile * P.splits + c.split) * (TOK * 128);
            if (ok && FD_CHECK((size_t)(ws_unit - A.sc.ws) + (TOK - 1) * 128 + e < A.sc.ws_elems,
                               P.ep.check, 22, (size_t)(ws_unit - A.sc.ws), A.sc.ws_elems)) {
#pragma unroll
              for (int t = 0; t < TOK; ++t) ws_unit[t * 128 + e] = acc[t];
            }
            goto unit_done;
          }
          if (!lmh) {
            // QKV / SwiGLU: with splits, the last split to arrive at a tile
            // sums all partials in split order and runs the epilogue
            if (!ok) *abort_flag = 1;
            bool run_epi = true;
            if (P.splits > 1) {
              float* ws_unit = A.sc.ws + ((size_t)c.tile * P.splits + c.split) * (TOK * 128);
              if (*abort_flag == 0) {
#pragma unroll
                for (int t = 0; t < TOK; ++t) ws_unit[t * 128 + e] = acc[t];
              }
              named_bar(1, WORKERS);
              if (leader) {
                int prev = -1;
                // releases this split's partial tile and acquires the other
                // splits' (one acquire-release atomic: measured 3 % less
                // chain time than a fence on either side of a relaxed add)
                if (FD_CHECK(c.tile < A.sc.n_counters, P.ep.check, 23, c.tile, A.sc.n_counters))
                  prev = atom_add_acq_rel_gpu(&A.sc.counters[c.tile], 1);
                if (prev == P.splits - 1) A.sc.counters[c.tile] = 0;
                // only the leader samples the abort flag: every worker then
                // takes the same branch through the barriers below
                *last_flag = (prev == P.splits - 1) && *abort_flag == 0;
              }
              named_bar(1, WORKERS);
              run_epi = *last_flag != 0;
              if (run_epi) {
                const float* ws_tile = A.sc.ws + (size_t)c.tile * P.splits * (TOK * 128) + e;
#pragma unroll
                for (int t = 0; t < TOK; ++t) acc[t] = __ldcg(ws_tile + t * 128);
                for (int sp = 1; sp < P.splits; ++sp) {
                  const float* q = ws_tile + (size_t)sp * (TOK * 128);
#pragma unroll
                  for (int t = 0; t < TOK; ++t) acc[t] += __ldcg(q + t * 128);
                }
              }
            } else {
              if (leader) *last_flag = *abort_flag == 0;
              named_bar(1, WORKERS);
              run_epi = *last_flag != 0;
            }
            if (run_epi)
              epi_staged_f16(P.ep, acc, n0, 0, e, reinterpret_cast<__half*>(tile), 1);
            named_bar(1, WORKERS);  // last_flag / tile are free for the next unit
            goto unit_done;
          }
          // LM head: no splits, reduced into this CTA's softmax states.  The
          // barriers run in every thread; a failed wait anywhere skips the work.
          if (!ok) *abort_flag = 1;
          named_bar(1, WORKERS);  // previous unit's reduction is done with `tile`
          if (leader) *last_flag = *abort_flag == 0;
          named_bar(1, WORKERS);
          const bool fine = *last_flag != 0;
          if (fine) {
#pragma unroll
            for (int t = 0; t < TOK; ++t) tile[t * 128 + e] = acc[t];
          }
          named_bar(1, WORKERS);
          if (fine) epi_chunk(P.ep, tile, n0, 0, e, lm);
                  }
        unit_done:
          named_bar(1, WORKERS);  // every worker is done with the entry and the unit
          if (leader) mbar_arrive(&uq_empty[slot]);
          ++wq;
        }
        if (lmh) {
          named_bar(1, WORKERS);
          SoftmaxState* out = reinterpret_cast<SoftmaxState*>(P.ep.lm_part) + (size_t)cta * P.ep.M;
          for (int t = wt; t < P.ep.M; t += WORKERS) out[t] = lm[t];
        }
      } else if (ok && (P.type == CH_NORM || P.type == CH_EMBED_NORM)) {
        int first = (cta - P.rot) % G;
        if (first < 0) first += G;
        const bool has_items = first < A.M * (A.d >> 9);
        if (p > 0 && has_items) {
          // one poller per CTA (thousands of polling threads would queue
          // behind the arrivals at the counter's L2 slice)
          if (leader) *last_flag = grid_wait(A.done + (p - 1) * CHAIN_DONE_STRIDE, G, err, A.gabort) ? 1 : 0;
          named_bar(1, WORKERS);
          ok = *last_flag != 0;
          named_bar(1, WORKERS);
        }
        if (ok && has_items) ok = norm_phase(A, P, p, cta, G, wt, red, last_flag, err);
      }
      // this CTA's share of phase p is complete: release it to the grid.
      // ok leaves here the same in every worker thread.
      if (!ok) *abort_flag = 1;
      named_bar(1, WORKERS);
      if (leader) {
        if (*abort_flag) atomicExch(A.gabort, 1);
        red_add_release_gpu(A.done + p * CHAIN_DONE_STRIDE, 1);
        misc[3] = ld_relaxed(A.gabort) | *abort_flag;
      }
      named_bar(1, WORKERS);
      ok = misc[3] == 0;
    }
    if (!ok) *abort_flag = 1;
  }

  // lanes 1..31 of the single-thread role warps reach this point long before
  // their lane 0: reconverge every warp first, so that the CTA barrier below
  // counts each warp once, with all of its threads
  __syncwarp();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, NBUF * NT);
  }
}

}  // namespace

int chain_smem_bytes() { return SMEM; }

cudaError_t chain_init_attributes() {
  return cudaFuncSetAttribute(chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
}

cudaError_t launch_chain(const ChainArgs& args, int grid, cudaStream_t st, bool after_kernel) {
  if (args.M < 1 || args.M > TOK || args.d % 512 || args.d > CHAIN_NORM_GROUPS * 512 ||
      args.M * (args.d / 512) > NORM_MAX_ITEMS * grid ||
      args.n_phases < 1 || args.n_phases > CHAIN_MAX_PHASES ||
      (after_kernel && args.ph[0].type != CH_GEMM))
    return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = SMEM;
  cfg.stream = st;
  cudaLaunchAttribute la[1];
  if (after_kernel) {
    // Programmatic launch after the attention kernel: CTAs start as its CTAs
    // retire, and the weight stream begins at once; only the first phase's
    // activation loads wait for the attention output (pdl_wait).  Phases
    // wait on every CTA of the grid, so all grid CTAs must become resident:
    // the grid is one CTA per SM (the shared memory admits no second), and
    // the preceding kernel's CTAs never wait on this one, so every SM frees
    // up; if that assumption is ever broken the bounded phase waits end the
    // launch with DEV_ERR_TIMEOUT instead of hanging.
    la[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    la[0].val.programmaticStreamSerializationAllowed = 1;
  } else {
    la[0].id = cudaLaunchAttributeCooperative;  // phases wait on every CTA of the grid
    la[0].val.cooperative = 1;
  }
  cfg.attrs = la;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, chain_kernel, args);
}

}  // namespace fd
