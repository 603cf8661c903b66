// Shared device helpers for the sm_100a decoder kernels: type conversions,
// warp reductions, bounded mbarrier waits, TMA and tcgen05 wrappers.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

#define FD_DEV __device__ __forceinline__

namespace fd {

// Error bits written by kernels into the ctx's device error word.
enum : int {
  DEV_ERR_TIMEOUT = 1,   // a bounded wait gave up
  DEV_ERR_TOKEN = 2,     // a token id outside [0, vocab) or a mask id in the prompt
  DEV_ERR_SHAPE = 4,     // a kernel was launched with a shape it cannot handle
  DEV_ERR_RANGE = 8,     // a weight outside the fp16 range
};

constexpr int KV_PAGE = 64;             // positions per KV-cache page
constexpr long long WAIT_LIMIT_NS = 2000000000ll;  // 2 s for any single wait

// ---------------------------------------------------------------- numerics
template <typename T> FD_DEV float to_f(T v);
template <> FD_DEV float to_f<float>(float v) { return v; }
template <> FD_DEV float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <> FD_DEV float to_f<__half>(__half v) { return __half2float(v); }

template <typename T> FD_DEV T from_f(float v);
template <> FD_DEV float from_f<float>(float v) { return v; }
template <> FD_DEV __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }
template <> FD_DEV __half from_f<__half>(float v) { return __float2half_rn(v); }

// Two-term storage of the bf16 model's activations and K/V: x = hi + lo with
// hi = round(x) and lo = round(x - hi) in the storage type.  The decoder
// stores fp16 pairs (22 significant bits together; the GEMM weights are
// converted to fp16 at load, exactly for every bf16 weight of magnitude
// >= 2^-17).  A single 16-bit term puts a rounding flip of 2^-9 (bf16) or
// 2^-12 (fp16) relative into every stored element whose float32 and float64
// values straddle a rounding boundary, and 32 layers of a random-weight
// network amplify those flips into logit errors far above 3e-2; bf16 pairs
// (16 bits) still left confidence errors of ~1.3e-3 at the LLaDA-8B shape.
// split_bf16 serves the bf16 operands of the stand-alone GEMM entry points.
FD_DEV void split_bf16(float x, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}
FD_DEV void split_f16(float x, __half& hi, __half& lo) {
  hi = __float2half_rn(x);
  lo = __float2half_rn(x - __half2float(hi));
}

// Row of token t's hi term in a two-term activation matrix: tokens come in
// groups of 32, each group stored as 32 hi rows followed by 32 lo rows, so a
// 64-row tile always holds both terms of the same 32 tokens.
FD_DEV __host__ int pair_row(int t) { return ((t >> 5) << 6) + (t & 31); }
constexpr int PAIR_LO = 32;  // lo row = hi row + 32

FD_DEV float silu_f(float g) { return g / (1.0f + expf(-g)); }
// SiLU with the fast exponential and division intrinsics (relative error of
// order 1e-6, under the bf16 model's tolerances; the fp32 model keeps
// silu_f).  g -> -inf gives g / inf = 0.
FD_DEV float silu_fast(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

FD_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

FD_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// (max, argmax) with the lowest index winning ties.
FD_DEV void warp_argmax(float& v, int& i) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float ov = __shfl_xor_sync(0xffffffffu, v, o);
    int oi = __shfl_xor_sync(0xffffffffu, i, o);
    if (ov > v || (ov == v && oi < i)) { v = ov; i = oi; }
  }
}

// Online-softmax state over a set of logits: running max m, sum of
// exp(z - m) s, and the lowest index attaining the max.
struct SoftmaxState {
  float m;
  float s;
  int arg;
};

FD_DEV SoftmaxState sm_empty() { return {-INFINITY, 0.0f, 0x7fffffff}; }

FD_DEV SoftmaxState sm_merge(SoftmaxState a, SoftmaxState b) {
  SoftmaxState r;
  r.m = fmaxf(a.m, b.m);
  r.arg = (b.m > a.m || (b.m == a.m && b.arg < a.arg)) ? b.arg : a.arg;
  if (r.m == -INFINITY) {
    r.s = 0.0f;
  } else {
    r.s = (a.m == -INFINITY ? 0.0f : a.s * expf(a.m - r.m)) +
          (b.m == -INFINITY ? 0.0f : b.s * expf(b.m - r.m));
  }
  return r;
}

FD_DEV SoftmaxState warp_sm_merge(SoftmaxState st) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    SoftmaxState other;
    other.m = __shfl_xor_sync(0xffffffffu, st.m, o);
    other.s = __shfl_xor_sync(0xffffffffu, st.s, o);
    other.arg = __shfl_xor_sync(0xffffffffu, st.arg, o);
    st = sm_merge(st, other);
  }
  return st;
}

// ---------------------------------------------------------------- self-checks
// Builds with FDLLM_CHECKS bounds-check device accesses: a failed check
// records (count, code, index, aux) in check[0..3] (first failure kept) and
// the access is skipped.  Normal builds compile the checks away.
FD_DEV bool check_fail(int* check, int code, long long idx, long long aux) {
  if (check && atomicAdd(check, 1) == 0) {
    check[1] = code;
    check[2] = (int)idx;
    check[3] = (int)aux;
  }
  return false;
}
#ifdef FDLLM_CHECKS
#define FD_CHECK(cond, chk, code, idx, aux) \
  ((cond) ? true : ::fd::check_fail((chk), (code), (long long)(idx), (long long)(aux)))
#else
#define FD_CHECK(cond, chk, code, idx, aux) true
#endif

// ---------------------------------------------------------------- address helpers
FD_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

FD_DEV uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- dependent launch
// Programmatic dependent launch: a kernel launched with the programmatic
// stream-serialization attribute may start while the previous kernel in the
// stream is still running.  pdl_wait() blocks until that kernel has completed
// and its memory is visible: every read of data the previous kernel wrote,
// and every write the previous kernel might still read, comes after it.
// pdl_trigger() lets the next kernel launch once every CTA of this grid has
// issued it (or exited).  Without the attribute both are no-ops.
FD_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
FD_DEV void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------- mbarrier
FD_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

FD_DEV void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

FD_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

FD_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

FD_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint: a thread whose phase is not complete
// sleeps (up to the hint) and is woken when it completes, instead of
// re-polling the barrier through the shared-memory pipe.
FD_DEV bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
      : "memory");
  return ok != 0;
}

// Bounded wait: returns false (and sets DEV_ERR_TIMEOUT) if the phase with the
// given parity has not completed within WAIT_LIMIT_NS, or if *abort is set.
FD_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, int* err, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_sleep(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (abort_flag && *abort_flag) return false;
      if (global_timer_ns() - t0 > (uint64_t)WAIT_LIMIT_NS) {
        atomicOr(err, DEV_ERR_TIMEOUT);
        if (abort_flag) *abort_flag = 1;
        return false;
      }
    }
  }
}

// ---------------------------------------------------------------- TMA
FD_DEV void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// As tma_load_2d, with an L2 eviction-priority policy (make_policy_*).
FD_DEV void tma_load_2d_hint(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                             uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}

FD_DEV void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                        int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Shared-memory writes of this thread (generic proxy) become visible to the
// tensor core's and TMA's reads of shared memory (async proxy).
FD_DEV void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// L2 policy for data read once (streamed weights): evicted first, so the
// activations, partial tiles and K/V the step re-reads stay in L2.
FD_DEV uint64_t make_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

FD_DEV void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- tcgen05
FD_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
FD_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Allocate ncols TMEM columns (power of two >= 32); the base address is
// written to *dst_smem.  Executed by one full warp.
FD_DEV void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

FD_DEV void tmem_dealloc(uint32_t base, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(ncols)
               : "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile stored with the
// 128-byte swizzle (rows of 128 bytes, 8-row / 1024-byte swizzle atoms).
//   bits [0,14)  start address >> 4
//   bits [16,30) leading byte offset >> 4 (unused for swizzled K-major; 1)
//   bits [32,46) stride byte offset >> 4 (1024 bytes between 8-row groups)
//   bits [46,48) descriptor version (1 on sm_100)
//   bits [61,64) layout: 2 = 128-byte swizzle
FD_DEV uint64_t smem_desc_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

// Descriptor of an MN-major operand tile stored with the 128-byte swizzle:
// rows of 128 bytes hold 64 consecutive MN elements for one K index, 8 rows
// (8 K indices) form a 1024-byte swizzle atom.  lbo_bytes = distance between
// 64-element atoms along MN, sbo_bytes = distance between 8-row groups
// along K.
FD_DEV uint64_t smem_desc_sw128_mn(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

// Instruction descriptor, kind::f16: D f32, A and B both fp16 (f16 = true)
// or both bf16, both K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_f32acc(int n, bool f16) {
  return (1u << 4)                          // D format f32
         | ((f16 ? 0u : 1u) << 7)           // A format: 0 fp16, 1 bf16
         | ((f16 ? 0u : 1u) << 10)          // B format: the same as A
         | ((uint32_t)(n >> 3) << 17)       // N >> 3
         | ((uint32_t)(128 >> 4) << 24);    // M >> 4
}

// As idesc_f32acc with the B operand MN-major (its N elements contiguous).
__host__ __device__ constexpr uint32_t idesc_f32acc_bmn(int n, bool f16) {
  return idesc_f32acc(n, f16) | (1u << 16);
}

FD_DEV void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on an mbarrier once every previously issued tcgen05.mma of this
// thread has completed.
FD_DEV void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Load 32 consecutive TMEM columns of this warp's 32 lanes (one lane per
// thread) into v[0..31].
FD_DEV void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Load TMEM columns [c, c + 16) into a[0..15] and [c + off, c + off + 16)
// into b[0..15] for this warp's 32 lanes; both loads and their wait in one
// statement, so no use of the registers can be scheduled before the wait.
template <int OFF>
FD_DEV void tmem_ld16x2(uint32_t taddr, float* a, float* b) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%32];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%33];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr), "r"(taddr + OFF)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    a[i] = __uint_as_float(r[i]);
    b[i] = __uint_as_float(r[16 + i]);
  }
}

// Load 64 consecutive TMEM columns of this warp's 32 lanes into v[0..63]
// (one instruction, one wait).
FD_DEV void tmem_ld64(uint32_t taddr, float* v) {
  uint32_t r[64];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]),
        "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]),
        "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]),
        "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]),
        "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]),
        "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}

// Store v[0..31] into 32 consecutive TMEM columns of this warp's 32 lanes
// and wait for the store to complete.
FD_DEV void tmem_st32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- clusters
// Barrier over every thread of every CTA of the thread-block cluster, with
// release / acquire ordering of shared-memory writes.
FD_DEV void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
FD_DEV uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory location in cluster CTA `rank`.
FD_DEV uint32_t cluster_map(uint32_t smem_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
  return r;
}
FD_DEV void ld_cluster_v4(uint32_t addr, float* v) {
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3])
               : "r"(addr)
               : "memory");
}

// Named barrier among `count` threads (a multiple of 32).
// Atomic add at gpu scope with acquire-release semantics: releases the
// writes ordered before it (after a CTA barrier, the whole CTA's) and
// acquires those released by the earlier additions, in one instruction.
FD_DEV int atom_add_acq_rel_gpu(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

FD_DEV void named_bar(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

}  // namespace fd
