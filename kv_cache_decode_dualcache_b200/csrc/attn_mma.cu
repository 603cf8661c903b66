// Bidirectional attention of the bfloat16 model on tensor cores (mma.sync).
//
// o = softmax(q K^T / sqrt(hd)) V over keys [0, L), no mask: block queries
// (DualCache step), rows [s, L) (prefix-cache step) or every position (full
// forward) all attend to the whole sequence, whose K/V come from the paged
// cache (the step's own rows were written there by the QKV epilogue just
// before).
//
// CTA = (row tile of up to 64 query rows, KV head, key split).  A query row
// is a (position, head-in-group) pair, so the query heads that share a KV
// head in GQA share the K/V tiles.  K/V tiles of 64 keys (one cache page)
// are double-buffered in shared memory with cp.async, in a 16-byte-chunk XOR
// swizzle so ldmatrix is conflict-free.  The NW warps (4, or 8 for full
// forwards with many query rows, so that twice the warps share each K/V
// tile) are NKG key groups x (NW / NKG) row groups of 16 rows: with few
// query rows (a 32-token block, MHA: NKG = 2) the warps split every key
// tile between them instead of
// idling, and merge their online-softmax states through shared memory at
// the end.
//
// Every operand is two-term (hi + lo fp16 pairs): q, K, V and the softmax
// weights P.  Each product takes the three significant cross terms:
//   S  = q_hi K_hi + q_hi K_lo + q_lo K_hi        (fp16 MMAs, f32 accumulate)
//   PV = P_hi V_hi + P_hi V_lo + P_lo V_hi
// so the attention output carries ~22 significant bits like every other
// stored activation of the bf16 model (see split_f16).  Online softmax in
// f32, exp2 domain.
//
// With n_split > 1 (block steps: few query rows, so the keys are split to
// fill the SMs) the n_split CTAs of a (row tile, KV head) run as one
// thread-block cluster; each keeps its unnormalised partial output and
// (max, sum) per row in shared memory and cluster rank 0 merges them in
// split order over distributed shared memory and writes o.
#include "common.cuh"
#include "kernels.h"

namespace fd {

namespace {

constexpr int kMaxSplit = 8;  // portable thread-block cluster size

FD_DEV void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
FD_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
FD_DEV void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

FD_DEV void ldsm_x4(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
FD_DEV void ldsm_x4_t(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

FD_DEV void mma_f16(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte offset of 16-byte chunk `ch` of row `r` in a [ROWS][HD] 2-byte tile
// stored as HD / 64 sub-tiles of [ROWS][64] (128-byte rows whose 16-byte
// chunks are XOR-swizzled by row % 8: the layout TMA writes with the
// 128-byte swizzle, and conflict-free for ldmatrix).
template <int HD, int ROWS>
FD_DEV uint32_t swz(int r, int ch) {
  return (uint32_t)((ch >> 3) * (ROWS * 128) + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
}

template <int HD, int NKG, int NW>
__global__ void __launch_bounds__(NW * 32)
    attn_mma_kernel(const __grid_constant__ CUtensorMap kvmap, AttnParams p) {
  constexpr int NT = NW * 32;        // threads
  constexpr int TILE = 64 * HD * 2;  // bytes of one [64][HD] 2-byte tile
  constexpr int CH = HD / 8;         // 16-byte chunks per row
  constexpr int NRG = NW / NKG;      // row groups of 16 rows
  constexpr int QR = 16 * NRG;          // query rows of the tile
  constexpr int QT = QR * HD * 2;        // bytes of one Q plane
  constexpr int KEYS = 64 / NKG;     // keys of a tile per key group
  constexpr int NNT = KEYS / 8;      // 8-key n-tiles per key group
  extern __shared__ __align__(128) uint8_t sm_raw[];
  __shared__ uint64_t kv_bar[2];   // one per K/V buffer (TMA completion)
  // layout (1024-byte aligned for the TMA swizzle): Q hi, Q lo, then per
  // buffer b: K hi, K lo, V hi, V lo
  uint8_t* sm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t q_s = smem_u32(sm);
  auto kv_s = [&](int buf, int plane) { return q_s + 2 * QT + (buf * 4 + plane) * TILE; };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rg = warp % NRG, kg = warp / NRG;
  const int H = p.n_heads, Hkv = p.n_kv_heads, rep = H / Hkv;
  const int g = blockIdx.y;
  if (tid == 0) {
    mbar_init(&kv_bar[0], 1);
    mbar_init(&kv_bar[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  pdl_trigger();
  pdl_wait();
  // one sequence: row tiles of the M query positions over keys [0, p.L);
  // batched forward: this CTA's tile of one sequence's segment
  int rows_total = p.M * rep, row0 = blockIdx.x * (16 * NRG), qbase = 0, L = p.L;
  const int* ptab = p.page_table;
  if (p.tiles) {
    const AttnTile tl = p.tiles[blockIdx.x];
    rows_total = tl.m * rep;
    row0 = tl.r0;
    qbase = tl.q0;
    L = tl.L;
    ptab = p.page_table + (size_t)tl.seq * p.pages_per_seq;
  }
  const int key_lo = blockIdx.z * p.keys_per_split;
  const int key_hi = min(L, key_lo + p.keys_per_split);
  const int n_kt = (key_hi - key_lo + 63) / 64;

  const __half* qg = reinterpret_cast<const __half*>(p.q);
  const uint16_t* pool = reinterpret_cast<const uint16_t*>(p.kv_pool);

  // ---- Q tiles (hi and lo planes), 16 * NRG rows
  for (int idx = tid; idx < 16 * NRG * CH; idx += NT) {
    const int i = idx / CH, ch = idx % CH;
    const int r = row0 + i;
    const bool ok = r < rows_total;
    const int m = ok ? qbase + r / rep : 0, jj = ok ? r % rep : 0;
    const __half* src = qg + ((size_t)m * H + g * rep + jj) * HD + ch * 8;
    cp_async16(q_s + swz<HD, QR>(i, ch), src, ok ? 16 : 0);
    cp_async16(q_s + QT + swz<HD, QR>(i, ch), src + p.q_plane, ok ? 16 : 0);
  }
  cp_async_commit();
  // K/V: one cache page (64 keys) per tile, each plane [64][HD] as HD / 64
  // TMA boxes of [64][64]; keys past key_hi are loaded and masked below
  auto load_kv = [&](int kt, int buf) {
    const int k0 = key_lo + kt * 64;          // key_lo is a multiple of 64
    const int page = ptab[k0 / KV_PAGE];
    fence_proxy_async_smem();                 // the buffer's earlier reads come first
    mbar_arrive_expect_tx(&kv_bar[buf], 4 * TILE);
#pragma unroll
    for (int pl = 0; pl < 4; ++pl) {
      const int row = (((p.layer * p.n_pages + page) * 4 + pl) * Hkv + g) * 64;
#pragma unroll
      for (int kh = 0; kh < HD / 64; ++kh)
        tma_load_2d(sm + (kv_s(buf, pl) - q_s) + kh * 64 * 128, &kvmap, &kv_bar[buf], kh * 64,
                    row);
    }
  };
  if (tid == 0 && n_kt > 0) load_kv(0, 0);

  const bool warp_active = row0 + rg * 16 < rows_total;
  const float sl2 = rsqrtf((float)HD) * 1.4426950408889634f;  // 1/sqrt(hd) * log2(e)
  float oacc[HD / 8][4];
#pragma unroll
  for (int j = 0; j < HD / 8; ++j) oacc[j][0] = oacc[j][1] = oacc[j][2] = oacc[j][3] = 0.0f;
  float mrow[2] = {-INFINITY, -INFINITY};
  float lrow[2] = {0.0f, 0.0f};

  for (int kt = 0; kt < n_kt; ++kt) {
    // buffer (kt + 1) & 1 was last read in iteration kt - 1 (CTA barrier since)
    if (tid == 0 && kt + 1 < n_kt) load_kv(kt + 1, (kt + 1) & 1);
    if (kt == 0) cp_async_wait<0>();
    mbar_wait(&kv_bar[kt & 1], (kt >> 1) & 1u, p.err, nullptr);
    __syncthreads();
    const int buf = kt & 1;
    if (warp_active) {
      // ---- S = Q K^T for this warp's KEYS keys of the tile
      float s[NNT][4];
#pragma unroll
      for (int nt = 0; nt < NNT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.0f;
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
        uint32_t qh[4], ql[4];
        const uint32_t qa = swz<HD, QR>(rg * 16 + (lane & 15), 2 * kk + (lane >> 4));
        ldsm_x4(q_s + qa, qh);
        ldsm_x4(q_s + QT + qa, ql);
#pragma unroll
        for (int np = 0; np < NNT / 2; ++np) {
          uint32_t kh[4], kl[4];
          const int key = kg * KEYS + np * 16 + (lane & 7) + ((lane >> 4) << 3);
          const uint32_t ka = swz<HD, 64>(key, 2 * kk + ((lane >> 3) & 1));
          ldsm_x4(kv_s(buf, 0) + ka, kh);
          ldsm_x4(kv_s(buf, 1) + ka, kl);
          mma_f16(s[2 * np], qh, kh[0], kh[1]);
          mma_f16(s[2 * np + 1], qh, kh[2], kh[3]);
          mma_f16(s[2 * np], qh, kl[0], kl[1]);
          mma_f16(s[2 * np + 1], qh, kl[2], kl[3]);
          mma_f16(s[2 * np], ql, kh[0], kh[1]);
          mma_f16(s[2 * np + 1], ql, kh[2], kh[3]);
        }
      }
      // ---- online softmax (rows lane/4 and lane/4 + 8)
      const int kbase = key_lo + kt * 64 + kg * KEYS + 2 * (lane & 3);
      float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < NNT; ++nt) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const bool ok = kbase + nt * 8 + (c & 1) < key_hi;
          s[nt][c] = ok ? s[nt][c] * sl2 : -INFINITY;
          tmax[c >> 1] = fmaxf(tmax[c >> 1], s[nt][c]);
        }
      }
      float alpha[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        tmax[r] = fmaxf(tmax[r], __shfl_xor_sync(0xffffffffu, tmax[r], 1));
        tmax[r] = fmaxf(tmax[r], __shfl_xor_sync(0xffffffffu, tmax[r], 2));
        const float mnew = fmaxf(mrow[r], tmax[r]);
        // a key group may see only masked keys in a ragged last tile
        alpha[r] = (mrow[r] == -INFINITY) ? 0.0f : exp2f(mrow[r] - mnew);
        mrow[r] = mnew;
        lrow[r] *= alpha[r];
      }
#pragma unroll
      for (int j = 0; j < HD / 8; ++j) {
        oacc[j][0] *= alpha[0];
        oacc[j][1] *= alpha[0];
        oacc[j][2] *= alpha[1];
        oacc[j][3] *= alpha[1];
      }
      uint32_t ph[NNT][2], pl[NNT][2];
#pragma unroll
      for (int nt = 0; nt < NNT; ++nt) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const float p0 = mrow[r] == -INFINITY ? 0.0f : exp2f(s[nt][2 * r] - mrow[r]);
          const float p1 = mrow[r] == -INFINITY ? 0.0f : exp2f(s[nt][2 * r + 1] - mrow[r]);
          const __half2 hi = __floats2half2_rn(p0, p1);
          const float2 hf = __half22float2(hi);
          const __half2 lo = __floats2half2_rn(p0 - hf.x, p1 - hf.y);
          ph[nt][r] = *reinterpret_cast<const uint32_t*>(&hi);
          pl[nt][r] = *reinterpret_cast<const uint32_t*>(&lo);
          lrow[r] += p0 + p1;
        }
      }
      // ---- O += P V
#pragma unroll
      for (int kk2 = 0; kk2 < NNT / 2; ++kk2) {
        const uint32_t ah[4] = {ph[2 * kk2][0], ph[2 * kk2][1], ph[2 * kk2 + 1][0],
                                ph[2 * kk2 + 1][1]};
        const uint32_t al[4] = {pl[2 * kk2][0], pl[2 * kk2][1], pl[2 * kk2 + 1][0],
                                pl[2 * kk2 + 1][1]};
#pragma unroll
        for (int j = 0; j < HD / 8; j += 2) {
          uint32_t vh[4], vl[4];
          const int key = kg * KEYS + kk2 * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
          const uint32_t va = swz<HD, 64>(key, j + (lane >> 4));
          ldsm_x4_t(kv_s(buf, 2) + va, vh);
          ldsm_x4_t(kv_s(buf, 3) + va, vl);
          mma_f16(oacc[j], ah, vh[0], vh[1]);
          mma_f16(oacc[j + 1], ah, vh[2], vh[3]);
          mma_f16(oacc[j], ah, vl[0], vl[1]);
          mma_f16(oacc[j + 1], ah, vl[2], vl[3]);
          mma_f16(oacc[j], al, vh[0], vh[1]);
          mma_f16(oacc[j + 1], al, vh[2], vh[3]);
        }
      }
    }
    __syncthreads();
  }

  // ---- merge the key groups of each row group (shared memory, fixed order)
  if (NKG > 1) {
    // per warp: 32 lanes x (HD/2 accumulators + 2 max + 2 sums) floats,
    // placed over the (now unused) K/V buffers
    constexpr int PER_LANE = HD / 2 + 4;
    float* xch = reinterpret_cast<float*>(sm + 2 * QT);
    float* mine = xch + (size_t)(warp * 32 + lane) * PER_LANE;
    if (kg > 0) {
#pragma unroll
      for (int j = 0; j < HD / 8; ++j)
#pragma unroll
        for (int c = 0; c < 4; ++c) mine[j * 4 + c] = oacc[j][c];
      mine[HD / 2] = mrow[0];
      mine[HD / 2 + 1] = mrow[1];
      mine[HD / 2 + 2] = lrow[0];
      mine[HD / 2 + 3] = lrow[1];
    }
    __syncthreads();
    if (kg == 0) {
      for (int k = 1; k < NKG; ++k) {
        const float* other = xch + (size_t)((k * NRG + rg) * 32 + lane) * PER_LANE;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const float mo = other[HD / 2 + r], lo_ = other[HD / 2 + 2 + r];
          const float mn = fmaxf(mrow[r], mo);
          const float a = (mrow[r] == -INFINITY) ? 0.0f : exp2f(mrow[r] - mn);
          const float b = (mo == -INFINITY) ? 0.0f : exp2f(mo - mn);
#pragma unroll
          for (int j = 0; j < HD / 8; ++j) {
            oacc[j][2 * r] = oacc[j][2 * r] * a + other[j * 4 + 2 * r] * b;
            oacc[j][2 * r + 1] = oacc[j][2 * r + 1] * a + other[j * 4 + 2 * r + 1] * b;
          }
          lrow[r] = lrow[r] * a + lo_ * b;
          mrow[r] = mn;
        }
      }
    }
  }
  const bool writer = warp_active && kg == 0;

  // ---- merge the key splits of this (row tile, KV head): the n_split CTAs
  // form one thread-block cluster (cluster rank = split index); rank 0 folds
  // ranks 1, 2, ... in order through distributed shared memory, so the
  // result does not depend on timing.
  if (p.n_split > 1) {
    constexpr int PER_LANE = HD / 2 + 4;
    float* xch = reinterpret_cast<float*>(sm + 2 * QT);
    float* mine = xch + (size_t)(warp * 32 + lane) * PER_LANE;
    __syncthreads();  // the key-group merge above is done with xch
    if (writer) {
#pragma unroll
      for (int j = 0; j < HD / 8; ++j)
#pragma unroll
        for (int c = 0; c < 4; ++c) mine[j * 4 + c] = oacc[j][c];
      mine[HD / 2] = mrow[0];
      mine[HD / 2 + 1] = mrow[1];
      mine[HD / 2 + 2] = lrow[0];
      mine[HD / 2 + 3] = lrow[1];
    }
    cluster_sync();  // every split's state is in its shared memory
    if (cluster_rank() == 0 && writer) {
      for (int k = 1; k < p.n_split; ++k) {
        const uint32_t rem = cluster_map(smem_u32(mine), k);
        float other[PER_LANE];
#pragma unroll
        for (int i = 0; i < PER_LANE; i += 4) ld_cluster_v4(rem + 4 * i, other + i);
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const float mo = other[HD / 2 + r], lo_ = other[HD / 2 + 2 + r];
          const float mn = fmaxf(mrow[r], mo);
          const float a = (mrow[r] == -INFINITY) ? 0.0f : exp2f(mrow[r] - mn);
          const float b = (mo == -INFINITY) ? 0.0f : exp2f(mo - mn);
#pragma unroll
          for (int j = 0; j < HD / 8; ++j) {
            oacc[j][2 * r] = oacc[j][2 * r] * a + other[j * 4 + 2 * r] * b;
            oacc[j][2 * r + 1] = oacc[j][2 * r + 1] * a + other[j * 4 + 2 * r + 1] * b;
          }
          lrow[r] = lrow[r] * a + lo_ * b;
          mrow[r] = mn;
        }
      }
    }
    cluster_sync();  // ranks 1.. keep their shared memory until rank 0 has read it
    if (cluster_rank() != 0) return;
  }

#pragma unroll
  for (int r = 0; r < 2; ++r) {
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 1);
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 2);
  }
  const int hq = H * HD;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    if (!writer) break;
    const int rr = row0 + rg * 16 + (lane >> 2) + 8 * r;
    if (rr >= rows_total) continue;
    const int m = qbase + rr / rep, head = g * rep + rr % rep;
    const float inv = 1.0f / lrow[r];
    __half* o = reinterpret_cast<__half*>(p.o);
    const size_t hi_off = (size_t)pair_row(m) * hq + (size_t)head * HD;
    const size_t lo_off = hi_off + (size_t)PAIR_LO * hq;
#pragma unroll
    for (int j = 0; j < HD / 8; ++j) {
      const int d = j * 8 + 2 * (lane & 3);
      __half h0, l0, h1, l1;
      split_f16(oacc[j][2 * r] * inv, h0, l0);
      split_f16(oacc[j][2 * r + 1] * inv, h1, l1);
      *reinterpret_cast<__half2*>(o + hi_off + d) = __halves2half2(h0, h1);
      *reinterpret_cast<__half2*>(o + lo_off + d) = __halves2half2(l0, l1);
    }
  }
}

// Shared memory: Q hi and lo planes of 16 * NW / NKG rows, then nbuf
// buffers of the four K/V planes of a 64-key tile (one buffer when a CTA
// has a single key tile), which the key-group and split merges reuse.
template <int HD, int NKG, int NW>
constexpr int attn_smem(int nbuf = 2) {
  return 2 * (16 * (NW / NKG) * HD * 2) +
         (nbuf * 4 * 64 * HD * 2 > NW * 32 * (HD / 2 + 4) * 4 ? nbuf * 4 * 64 * HD * 2
                                                               : NW * 32 * (HD / 2 + 4) * 4);
}

template <int HD, int NKG, int NW>
cudaError_t set_attr() {
  static_assert(attn_smem<HD, NKG, NW>() + 1024 <= 232448, "exceeds the 227 KB shared memory limit");
  return cudaFuncSetAttribute(attn_mma_kernel<HD, NKG, NW>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              attn_smem<HD, NKG, NW>() + 1024);
}

template <int HD, int NKG, int NW>
cudaError_t launch_hd(const CUtensorMap* kvmap, const AttnParams& p, cudaStream_t st, bool pdl) {
  // a single key tile per CTA needs one K/V buffer: two CTAs fit on an SM
  // (+1 KB: the tiles start at a 1024-byte boundary for the TMA swizzle)
  const int smem = attn_smem<HD, NKG, NW>(p.keys_per_split <= 64 ? 1 : 2) + 1024;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = set_attr<HD, NKG, NW>();
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const int rows = p.M * (p.n_heads / p.n_kv_heads);
  const int rows_per_cta = 16 * (NW / NKG);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.tiles ? p.n_tiles : (rows + rows_per_cta - 1) / rows_per_cta,
                     p.n_kv_heads, p.n_split);
  cfg.blockDim = dim3(NW * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute la[2];
  int na = 0;
  if (pdl) {
    la[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    la[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (p.n_split > 1) {  // the splits of a (row tile, KV head) form one cluster
    la[na].id = cudaLaunchAttributeClusterDimension;
    la[na].val.clusterDim.x = 1;
    la[na].val.clusterDim.y = 1;
    la[na].val.clusterDim.z = p.n_split;
    ++na;
  }
  cfg.attrs = la;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, attn_mma_kernel<HD, NKG, NW>, *kvmap, p);
}

template <int HD>
cudaError_t launch_nkg(const CUtensorMap* kvmap, const AttnParams& p, cudaStream_t st, bool pdl) {
  // batched forwards tile every segment into 64-row tiles (attn_rows_per_cta(-1, ..))
  if (p.tiles) return launch_hd<HD, 1, 4>(kvmap, p, st, pdl);
  const int rows = p.M * (p.n_heads / p.n_kv_heads);
  if (rows <= 16) return launch_hd<HD, 4, 4>(kvmap, p, st, pdl);
  if (rows <= 32) return launch_hd<HD, 2, 4>(kvmap, p, st, pdl);
  if (rows <= 64) return launch_hd<HD, 1, 4>(kvmap, p, st, pdl);
  // many query rows (full forwards, GQA): eight warps share each K/V tile
  return launch_hd<HD, 1, 8>(kvmap, p, st, pdl);
}

}  // namespace

int attn_rows_per_cta(int M, int n_heads, int n_kv_heads) {
  if (M < 0) return 64;  // batched forwards (AttnParams::tiles)
  const int rows = M * (n_heads / n_kv_heads);
  return rows <= 16 ? 16 : rows <= 32 ? 32 : rows <= 64 ? 64 : 128;
}

cudaError_t launch_attn_mma(const CUtensorMap* kvmap, const AttnParams& p, cudaStream_t st,
                            bool pdl) {
  if (p.kv_planes != 4 || p.n_split < 1 || p.n_split > kMaxSplit ||
      (p.tiles && (p.n_split != 1 || p.n_tiles < 1)))
    return cudaErrorInvalidValue;
  switch (p.head_dim) {
    case 64: return launch_nkg<64>(kvmap, p, st, pdl);
    case 128: return launch_nkg<128>(kvmap, p, st, pdl);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t gemm_tc_init_attributes();
cudaError_t gemm_tc2_init_attributes();
cudaError_t attn_blk_init_attributes();

cudaError_t init_kernel_attributes() {
  cudaError_t e = set_attr<64, 1, 4>();
  if (e == cudaSuccess) e = set_attr<64, 2, 4>();
  if (e == cudaSuccess) e = set_attr<64, 4, 4>();
  if (e == cudaSuccess) e = set_attr<64, 1, 8>();
  if (e == cudaSuccess) e = set_attr<128, 1, 4>();
  if (e == cudaSuccess) e = set_attr<128, 2, 4>();
  if (e == cudaSuccess) e = set_attr<128, 4, 4>();
  if (e == cudaSuccess) e = set_attr<128, 1, 8>();
  if (e == cudaSuccess) e = gemm_tc_init_attributes();
  if (e == cudaSuccess) e = gemm_tc2_init_attributes();
  if (e == cudaSuccess) e = attn_blk_init_attributes();
  if (e == cudaSuccess) e = chain_init_attributes();
  if (e == cudaSuccess) e = attn_tc_init_attributes();
  return e;
}

}  // namespace fd
