// GEMM epilogues.
//
// epi_chunk: output tiles of 128 features x 32 tokens staged in shared
// memory as float tile[t * 128 + e] (t = token row in the chunk, e = feature
// within the 128-feature tile); the 128 epilogue threads call it with e =
// their feature index.  It serves every epilogue of the CUDA-core GEMM (fp32
// model, natural weight-row order) and the LM-head reduction of the tcgen05
// GEMM.  Control flow is uniform within each warp (the LM-head reduction
// uses warp shuffles).
//
// epi_regs: the other epilogues of the tcgen05 GEMM (bf16 model), straight
// from the registers the accumulator was read into, on the permuted weight
// rows described at rope_slab_dim.  Its stores are two-term fp16 (hi + lo,
// see split_f16): the q planes, the K/V cache planes and the SwiGLU output
// in pair rows.
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace fd {

constexpr int EPI_THREADS = 128;
constexpr int CHUNK_T = 32;

// Element offset of (position, plane, kv head, dim) in the paged cache, with
// the position's page already looked up.
FD_DEV size_t kv_offset_pg(const EpiParams& ep, int page, int pos, int plane, int head, int dim) {
  const int slot = pos % KV_PAGE;
  return ((((size_t)ep.layer * ep.n_pages + page) * ep.kv_planes + plane) * ep.n_kv_heads +
          head) * (size_t)(KV_PAGE * ep.head_dim) +
         (size_t)slot * ep.head_dim + dim;
}

// Batched forward (ep.rows set): position (-1 for a padding row) and K/V
// page of token row tok.
FD_DEV int row_pos(const EpiParams& ep, int tok) { return __ldg(&ep.rows[tok].pos); }
FD_DEV int row_page(const EpiParams& ep, int tok, int pos) {
  return __ldg(&ep.page_table[__ldg(&ep.rows[tok].seq) * ep.pages_per_seq + pos / KV_PAGE]);
}

// One 32-token chunk of a 128-feature output tile.
//   tile: [32][128] float in shared memory, fully written before the call.
//   n0:   first feature of the tile; t0: token row of tile row 0.
//   lm:   per-token softmax states of this CTA (EPI_LMHEAD only).
FD_DEV void epi_chunk(const EpiParams& ep, const float* tile, int n0, int t0, int e,
                      SoftmaxState* lm) {
  const int n = n0 + e;
  switch (ep.kind) {
    case EPI_STORE: {
      if (n < ep.N)
        for (int t = 0; t < CHUNK_T && t0 + t < ep.M; ++t) {
          const size_t i = (size_t)(t0 + t) * ep.ld_out + n;
          if (FD_CHECK(i < ep.cap_out, ep.check, 1, i, ep.cap_out)) ep.out[i] = tile[t * 128 + e];
        }
      break;
    }
    case EPI_RESID: {
      // All 32 loads of h are issued before any store: interleaving them
      // would serialise one memory round trip per token row (the compiler
      // cannot prove the stores do not alias the next loads).
      if (n < ep.N) {
        const int nt = min(CHUNK_T, ep.M - t0);
        float hv[CHUNK_T];
#pragma unroll
        for (int t = 0; t < CHUNK_T; ++t)
          hv[t] = (t < nt) ? ep.h[(size_t)(t0 + t) * ep.N + n] : 0.0f;
#pragma unroll
        for (int t = 0; t < CHUNK_T; ++t) {
          if (t >= nt) break;
          const size_t i = (size_t)(t0 + t) * ep.N + n;
          if (FD_CHECK(i < ep.cap_h, ep.check, 2, i, ep.cap_h)) ep.h[i] = hv[t] + tile[t * 128 + e];
        }
      }
      break;
    }
    case EPI_SWIGLU: {
      // fp32 model: rows [128j, 128j+64) of the fused weight are gate rows
      // [64j, 64j+64), rows [128j+64, 128j+128) the matching up rows.
      const int F = ep.N / 2;
      const int j = (n0 / 128) * 64 + e;
      if (e < 64 && j < F)
        for (int t = 0; t < CHUNK_T && t0 + t < ep.M; ++t) {
          const float g = tile[t * 128 + e];
          const float u = tile[t * 128 + e + 64];
          const size_t i = (size_t)(t0 + t) * F + j;
          if (FD_CHECK(i < ep.cap_f, ep.check, 3, i, ep.cap_f))
            reinterpret_cast<float*>(ep.f_out)[i] = silu_f(g) * u;
        }
      break;
    }
    case EPI_QKV: {
      // fp32 model: natural row order, RoPE partners through the tile
      if (n >= ep.N) break;
      if (ep.rows) {
        // batched forward: every row has its own position and slot
        const int hd = ep.head_dim, half = hd / 2;
        const int hq = ep.n_heads * hd, hk = ep.n_kv_heads * hd;
        const int dh = n % hd;
        const bool is_q = n < hq, is_v = n >= hq + hk;
        float* kv = reinterpret_cast<float*>(ep.kv_pool);
        for (int t = 0; t < CHUNK_T && t0 + t < ep.M; ++t) {
          const int tok = t0 + t;
          const int pos = row_pos(ep, tok);
          if (pos < 0) continue;   // padding row of the batched forward
          float y = tile[t * 128 + e];
          if (!is_v) {
            const float2 c = __ldg(&ep.rope[(size_t)pos * half + (dh % half)]);
            y = dh < half ? y * c.x - tile[t * 128 + e + half] * c.y
                          : y * c.x + tile[t * 128 + e - half] * c.y;
          }
          if (is_q) {
            const size_t i = (size_t)tok * hq + n;
            if (FD_CHECK(i < ep.cap_q, ep.check, 4, i, ep.cap_q))
              reinterpret_cast<float*>(ep.q_out)[i] = y;
          } else {
            const int page = row_page(ep, tok, pos);
            const size_t i = is_v ? kv_offset_pg(ep, page, pos, 1, (n - hq - hk) / hd, dh)
                                  : kv_offset_pg(ep, page, pos, 0, (n - hq) / hd, dh);
            if (FD_CHECK(i < ep.cap_kv, ep.check, 5, i, ep.cap_kv)) kv[i] = y;
          }
        }
        break;
      }
      const int hd = ep.head_dim, half = hd / 2;
      const int hq = ep.n_heads * hd, hk = ep.n_kv_heads * hd;
      const int dh = n % hd;
      const bool is_q = n < hq, is_v = n >= hq + hk;
      const int pos0 = ep.sp ? ep.sp->r0 : ep.pos0;
      const int nt = min(CHUNK_T, ep.M - t0);
      if (nt <= 0) break;  // chunk past the last token row of the tile
      // Loads first (RoPE table for the chunk's 32 positions), stores after:
      // see EPI_RESID.
      float2 cs[CHUNK_T];
      if (!is_v) {
#pragma unroll
        for (int t = 0; t < CHUNK_T; ++t)
          cs[t] = (t < nt) ? __ldg(&ep.rope[(size_t)(pos0 + t0 + t) * half + (dh % half)])
                           : make_float2(1.0f, 0.0f);
      }
      // the chunk's 32 positions span at most two cache pages
      const int pidx0 = (pos0 + t0) / KV_PAGE;
      int page0 = 0, page1 = 0;
      if (!is_q) {
        page0 = __ldg(&ep.page_table[pidx0]);
        page1 = __ldg(&ep.page_table[(pos0 + t0 + nt - 1) / KV_PAGE]);
      }
      float* kv = reinterpret_cast<float*>(ep.kv_pool);
#pragma unroll
      for (int t = 0; t < CHUNK_T; ++t) {
        if (t >= nt) break;
        const int tok = t0 + t;
        const int pos = pos0 + tok;
        float y = tile[t * 128 + e];
        if (!is_v) {
          if (dh < half) {
            const float x2 = tile[t * 128 + e + half];
            y = y * cs[t].x - x2 * cs[t].y;
          } else {
            const float x1 = tile[t * 128 + e - half];
            y = y * cs[t].x + x1 * cs[t].y;
          }
        }
        const int page = (pos / KV_PAGE == pidx0) ? page0 : page1;
        if (is_q) {
          const size_t i = (size_t)tok * hq + n;
          if (FD_CHECK(i < ep.cap_q, ep.check, 4, i, ep.cap_q))
            reinterpret_cast<float*>(ep.q_out)[i] = y;
        } else {
          const size_t i = is_v ? kv_offset_pg(ep, page, pos, 1, (n - hq - hk) / hd, dh)
                                : kv_offset_pg(ep, page, pos, 0, (n - hq) / hd, dh);
          if (FD_CHECK(i < ep.cap_kv, ep.check, 5, i, ep.cap_kv)) kv[i] = y;
        }
      }
      break;
    }
    case EPI_LMHEAD: {
      const int warp = e >> 5, lane = e & 31;
      for (int t = warp; t < CHUNK_T; t += EPI_THREADS / 32) {
        const int tok = t0 + t;
        if (tok >= ep.M) break;  // uniform across the warp
        float z[4];
        float mx = -INFINITY;
        int arg = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = lane + 32 * j;
          const int nn = n0 + r;
          z[j] = ep.logit_scale * tile[t * 128 + r];
          if (ep.dbg_logits && nn < ep.N) {
            const size_t i = (size_t)tok * ep.N + nn;
            if (FD_CHECK(i < ep.cap_dbg, ep.check, 7, i, ep.cap_dbg)) ep.dbg_logits[i] = z[j];
          }
          const bool ok = nn < ep.N && nn != ep.mask_id;
          if (!ok) z[j] = -INFINITY;
          if (z[j] > mx) { mx = z[j]; arg = nn; }  // j ascending: lowest id kept on ties
        }
        warp_argmax(mx, arg);
        float s = 0.0f;
        if (mx != -INFINITY) {
#pragma unroll
          for (int j = 0; j < 4; ++j) s += (z[j] == -INFINITY) ? 0.0f : expf(z[j] - mx);
        }
        s = warp_sum(s);
        if (lane == 0) lm[tok] = sm_merge(lm[tok], SoftmaxState{mx, s, arg});
      }
      break;
    }
    default:
      break;
  }
}

// Weight-row order of the tensor-core path inside every 32-row slab (one
// warp's TMEM lanes), so that the two rows an epilogue output needs sit 16
// lanes apart in the same warp and meet through one shuffle:
//   q / k heads: slab s of a head (rows 32s .. 32s+31) holds dims
//                16s .. 16s+15 in lanes 0..15 and their rotate-half partners
//                (dim + hd/2) in lanes 16..31; rope_slab_dim maps the row
//                r within the head to its dim;
//   gate / up:   slab s of the fused matrix holds gate features
//                16s .. 16s+15 in lanes 0..15 and the matching up features
//                in lanes 16..31.
// The V rows and every other weight keep their natural order.
FD_DEV __host__ int rope_slab_dim(int r, int hd) {
  return 16 * (r >> 5) + (r & 15) + ((r >> 4) & 1) * (hd / 2);
}

// Epilogue of one 32-token chunk held in registers by the 128 threads of an
// epilogue warpgroup: v[t] = output feature n0 + e of token row t0 + t.
// e = tile row = 32 * (warp % 4) + lane.  Shuffles stay within a warp and
// control flow is warp-uniform (N and the q / k / v region boundaries are
// multiples of 64 for the QKV and SwiGLU layouts).  EPI_LMHEAD is not
// handled here: it needs all 128 features of a token (epi_chunk).  ROWS:
// the batched forward's per-row positions (a separate instantiation, so the
// one-sequence code is compiled without that path).
template <bool ROWS = false>
FD_DEV void epi_regs(const EpiParams& ep, const float (&v)[CHUNK_T], int n0, int t0, int e) {
  const int lane = e & 31;
  const int n = n0 + e;
  int nt = min(CHUNK_T, ep.M - t0);
  if (nt <= 0) return;
  switch (ep.kind) {
    case EPI_STORE: {
      if (n >= ep.N) break;
#pragma unroll
      for (int t = 0; t < CHUNK_T; ++t) {
        if (t >= nt) break;
        const size_t i = (size_t)(t0 + t) * ep.ld_out + n;
        if (FD_CHECK(i < ep.cap_out, ep.check, 1, i, ep.cap_out)) ep.out[i] = v[t];
      }
      break;
    }
    case EPI_RESID: {
      // all loads of h before any store (see epi_chunk); through L2, since
      // in the chain kernel other SMs wrote h earlier in the same launch
      if (n >= ep.N) break;
      float hv[CHUNK_T];
#pragma unroll
      for (int t = 0; t < CHUNK_T; ++t)
        hv[t] = (t < nt) ? __ldcg(ep.h + (size_t)(t0 + t) * ep.N + n) : 0.0f;
#pragma unroll
      for (int t = 0; t < CHUNK_T; ++t) {
        if (t >= nt) break;
        const size_t i = (size_t)(t0 + t) * ep.N + n;
        if (FD_CHECK(i < ep.cap_h, ep.check, 2, i, ep.cap_h)) ep.h[i] = hv[t] + v[t];
      }
      break;
    }
    case EPI_SWIGLU: {
      if (n >= ep.N) break;  // warp-uniform
      const int F = ep.N / 2;
      const int j = 16 * (n >> 5) + (lane & 15);  // FFN feature of this lane pair
      const bool up = lane >= 16;
      __half* f = reinterpret_cast<__half*>(ep.f_out);
#pragma unroll
      for (int t = 0; t < CHUNK_T; ++t) {
        if (t >= nt) break;
        const float p = __shfl_xor_sync(0xffffffffu, v[t], 16);
        const float g = up ? p : v[t];
        const float u = up ? v[t] : p;
        __half hi, lo;
        split_f16(silu_f(g) * u, hi, lo);
        // lanes 0..15 store the hi term, lanes 16..31 the lo term
        const size_t i = ((size_t)pair_row(t0 + t) + (up ? PAIR_LO : 0)) * F + j;
        if (FD_CHECK(i < ep.cap_f, ep.check, 3, i, ep.cap_f)) f[i] = up ? lo : hi;
      }
      break;
    }
    case EPI_QKV: {
      if (n >= ep.N) break;  // warp-uniform
      const int hd = ep.head_dim, half = hd / 2;
      const int hq = ep.n_heads * hd, hk = ep.n_kv_heads * hd;
      const int region = n < hq ? 0 : (n < hq + hk ? 1 : 2);  // q, k, v (uniform per warp)
      const int rn = n - (region == 0 ? 0 : (region == 1 ? hq : hq + hk));
      const int head = rn / hd;
      const int r = rn - head * hd;
      const int dim = region < 2 ? rope_slab_dim(r, hd) : r;
      // one sequence: rows t0.. at positions pos0.. of its pages; batched
      // forward: the chunk's sequence and first position (t0 is a multiple
      // of 32, and a chunk's real rows come first)
      int pos0;
      const int* ptab = ep.page_table;
      if constexpr (ROWS) {
        const RowChunk ck = ep.chunks[t0 >> 5];
        pos0 = ck.pos0;
        ptab += ck.seq * ep.pages_per_seq;
        nt = min(nt, ck.n);
      } else {
        pos0 = (ep.sp ? ep.sp->r0 : ep.pos0) + t0;
      }
      const bool second = lane >= 16;  // holds dim + hd/2 of the rotate-half pair
      int page0 = 0, page1 = 0;
      if (region > 0) {
        page0 = __ldg(&ptab[pos0 / KV_PAGE]);
        page1 = __ldg(&ptab[(pos0 + nt - 1) / KV_PAGE]);
      }
      // 16 tokens at a time: the RoPE table loads of a half are issued
      // before its stores (see EPI_RESID), in fewer registers than 32.
      // Stores: lanes 4k .. 4k + 3 hold dims d .. d + 3 (the slab
      // permutation keeps 16-lane runs of consecutive dims); per 4 tokens
      // they transpose their (hi, lo) values in two shuffle rounds, so that
      // lane 4k + j stores dims d .. d + 3 of token j: 8-byte stores, a
      // quarter of the store instructions of one 2-byte store per value
      // (the narrow stores, each waiting for write credits, are what bound
      // this epilogue).
      const int l4 = lane & 3;
      const int dim4 = dim - l4;   // first dim of the lane quad (a multiple of 4)
#pragma unroll
      for (int h16 = 0; h16 < CHUNK_T; h16 += 16) {
        if (h16 >= nt) break;
        float2 cs[16];
        if (region < 2) {
#pragma unroll
          for (int t = 0; t < 16; ++t)
            cs[t] = (h16 + t < nt)
                        ? __ldg(&ep.rope[(size_t)(pos0 + h16 + t) * half + (dim % half)])
                        : make_float2(1.0f, 0.0f);
        }
#pragma unroll
        for (int t = 0; t < 16; t += 4) {
          if (h16 + t >= nt) break;
          // x[j] = (hi, lo) of token t + j at this lane's dim
          uint32_t x[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float y = v[h16 + t + j];
            if (region < 2) {
              const float p = __shfl_xor_sync(0xffffffffu, y, 16);
              y = second ? (y * cs[t + j].x + p * cs[t + j].y) : (y * cs[t + j].x - p * cs[t + j].y);
            }
            __half hi, lo;
            split_f16(y, hi, lo);
            const __half2 hl = __halves2half2(hi, lo);
            x[j] = *reinterpret_cast<const uint32_t*>(&hl);
          }
          // 4 x 4 transpose over the lane quad: swap bit 0, then bit 1, of
          // (lane, token); afterwards x[k] = token t + l4 at dim dim4 + k
          {
            const bool b0 = l4 & 1;
            const uint32_t s0 = __shfl_xor_sync(0xffffffffu, b0 ? x[0] : x[1], 1);
            const uint32_t s1 = __shfl_xor_sync(0xffffffffu, b0 ? x[2] : x[3], 1);
            if (b0) { x[0] = s0; x[2] = s1; } else { x[1] = s0; x[3] = s1; }
            const bool b1 = l4 & 2;
            const uint32_t s2 = __shfl_xor_sync(0xffffffffu, b1 ? x[0] : x[2], 2);
            const uint32_t s3 = __shfl_xor_sync(0xffffffffu, b1 ? x[1] : x[3], 2);
            if (b1) { x[0] = s2; x[1] = s3; } else { x[2] = s2; x[3] = s3; }
          }
          const uint2 hi4 = make_uint2(__byte_perm(x[0], x[1], 0x5410), __byte_perm(x[2], x[3], 0x5410));
          const uint2 lo4 = make_uint2(__byte_perm(x[0], x[1], 0x7632), __byte_perm(x[2], x[3], 0x7632));
          const int tt = h16 + t + l4;
          if (tt >= nt) continue;
          const int tok = t0 + tt;
          const int pos = pos0 + tt;
          if (region == 0) {
            __half* q = reinterpret_cast<__half*>(ep.q_out);
            const size_t i = (size_t)tok * hq + head * hd + dim4;
            if (FD_CHECK(ep.q_plane + i + 3 < ep.cap_q, ep.check, 4, ep.q_plane + i, ep.cap_q)) {
              *reinterpret_cast<uint2*>(q + i) = hi4;
              *reinterpret_cast<uint2*>(q + ep.q_plane + i) = lo4;
            }
          } else {
            const int page = (pos / KV_PAGE == pos0 / KV_PAGE) ? page0 : page1;
            const int plane = region == 1 ? 0 : 2;
            __half* kv = reinterpret_cast<__half*>(ep.kv_pool);
            const size_t i0 = kv_offset_pg(ep, page, pos, plane, head, dim4);
            const size_t i1 = kv_offset_pg(ep, page, pos, plane + 1, head, dim4);
            if (FD_CHECK(i1 + 3 < ep.cap_kv, ep.check, 5, i1, ep.cap_kv)) {
              *reinterpret_cast<uint2*>(kv + i0) = hi4;
              *reinterpret_cast<uint2*>(kv + i1) = lo4;
            }
          }
        }
      }
      break;
    }
    default:
      break;
  }
}

}  // namespace fd

namespace fd {

// epi_regs for the QKV and SwiGLU epilogues, with the two-term fp16 output
// staged in shared memory and written back as 16-byte stores: a thread
// stores 8 chunks of 16 bytes per tile instead of 64 scattered 2-byte
// values, and those narrow stores are what limits an SM's epilogue (each
// store instruction waits for write credits toward L2).  Called by the 128
// threads of one warpgroup, which sync on named barrier `bar`; st is 16 KB
// of shared memory that the caller does not use until the call returns.
// v[t] = output feature n0 + e of token row t0 + t (see epi_regs).
FD_DEV void epi_staged_f16(const EpiParams& ep, const float (&v)[CHUNK_T], int n0, int t0, int e,
                           __half* st, int bar) {
  const int lane = e & 31;
  const int n = n0 + e;
  const int nt = min(CHUNK_T, ep.M - t0);
  if (nt <= 0) return;
  __half* st_hi = st;                 // [32 tokens][128 features]
  __half* st_lo = st + CHUNK_T * 128;
  if (ep.kind == EPI_SWIGLU) {
    // 64 outputs per tile: feature j0 + f, f = 16 * (e / 32) + lane % 16.
    // Lane l < 16 holds the gate and lane l + 16 the up value of feature f;
    // per pair of tokens they swap one value, so that the gate lane computes
    // token t and the up lane token t + 1: every lane of a SiLU instruction
    // does useful work.
    const int F = ep.N / 2;
    const bool up = lane >= 16;
    const int f = 16 * (e >> 5) + (lane & 15);
#pragma unroll
    for (int t = 0; t < CHUNK_T; t += 2) {
      const float recv = __shfl_xor_sync(0xffffffffu, up ? v[t] : v[t + 1], 16);
      const float g = up ? recv : v[t];        // gate lane: (g_t, u_t); up lane: (g_t+1, u_t+1)
      const float u = up ? v[t + 1] : recv;
      __half hi, lo;
      split_f16(silu_fast(g) * u, hi, lo);
      const int tt = t + (up ? 1 : 0);
      st_hi[tt * 128 + f] = hi;
      st_lo[tt * 128 + f] = lo;
    }
    named_bar(bar, EPI_THREADS);
    // rows: 32 tokens x {hi, lo}; 64 features = 8 chunks of 8 per row
    const int j0 = n0 / 2;  // 64 FFN features per 128-row tile
    __half* fo = reinterpret_cast<__half*>(ep.f_out);
    for (int c = e; c < CHUNK_T * 2 * 8; c += EPI_THREADS) {
      const int t = c >> 4, term = (c >> 3) & 1, ch = c & 7;
      if (t >= nt || n0 >= ep.N) continue;
      const __half* src = (term ? st_lo : st_hi) + t * 128 + ch * 8;
      const size_t i = ((size_t)pair_row(t0 + t) + (term ? PAIR_LO : 0)) * F + j0 + ch * 8;
      if (FD_CHECK(i + 7 < ep.cap_f, ep.check, 3, i, ep.cap_f))
        *reinterpret_cast<uint4*>(fo + i) = *reinterpret_cast<const uint4*>(src);
    }
    named_bar(bar, EPI_THREADS);
    return;
  }
  // EPI_QKV (one sequence: the chain kernel's block rows): the tile is
  // 128 / hd heads of one region (q, k or v); N and the region bounds are
  // multiples of 64, so a warp is wholly inside or outside
  const int hd = ep.head_dim, half = hd / 2;
  const int hq = ep.n_heads * hd, hk = ep.n_kv_heads * hd;
  const bool valid = n < ep.N;
  const int region = n0 < hq ? 0 : (n0 < hq + hk ? 1 : 2);
  const int rbase = region == 0 ? 0 : (region == 1 ? hq : hq + hk);
  const int rn = n - rbase;
  const int head = rn / hd;
  const int r = rn - head * hd;
  const int dim = region < 2 ? rope_slab_dim(r, hd) : r;
  const int col = (head - (n0 - rbase) / hd) * hd + dim;  // natural column within the tile
  const int pos0 = (ep.sp ? ep.sp->r0 : ep.pos0) + t0;
  const bool second = lane >= 16;
  if (valid) {
#pragma unroll
    for (int h16 = 0; h16 < CHUNK_T; h16 += 16) {
      float2 cs[16];
      if (region < 2) {
#pragma unroll
        for (int t = 0; t < 16; ++t)
          cs[t] = (h16 + t < nt) ? __ldg(&ep.rope[(size_t)(pos0 + h16 + t) * half + (dim % half)])
                                 : make_float2(1.0f, 0.0f);
      }
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        float y = v[h16 + t];
        if (region < 2) {
          const float p = __shfl_xor_sync(0xffffffffu, y, 16);
          y = second ? (y * cs[t].x + p * cs[t].y) : (y * cs[t].x - p * cs[t].y);
        }
        __half hi, lo;
        split_f16(y, hi, lo);
        st_hi[(h16 + t) * 128 + col] = hi;
        st_lo[(h16 + t) * 128 + col] = lo;
      }
    }
  }
  named_bar(bar, EPI_THREADS);
  {
    const int head0 = (n0 - rbase) / hd;  // first head of the tile
    const int pg0 = region > 0 ? __ldg(&ep.page_table[pos0 / KV_PAGE]) : 0;
    const int pg1 = region > 0 ? __ldg(&ep.page_table[(pos0 + nt - 1) / KV_PAGE]) : 0;
    // 32 tokens x 2 terms x 16 chunks of 8 features
    for (int c = e; c < CHUNK_T * 2 * 16; c += EPI_THREADS) {
      const int t = c >> 5, term = (c >> 4) & 1, ch = c & 15;
      if (t >= nt || n0 + ch * 8 >= ep.N) continue;
      const uint4 val = *reinterpret_cast<const uint4*>((term ? st_lo : st_hi) + t * 128 + ch * 8);
      const int cf = ch * 8;                 // natural column within the tile
      const int hh = head0 + cf / hd, dd = cf % hd;
      if (region == 0) {
        __half* q = reinterpret_cast<__half*>(ep.q_out);
        const size_t i = (size_t)(t0 + t) * hq + (size_t)hh * hd + dd + (term ? ep.q_plane : 0);
        if (FD_CHECK(i + 7 < ep.cap_q, ep.check, 4, i, ep.cap_q))
          *reinterpret_cast<uint4*>(q + i) = val;
      } else {
        const int pos = pos0 + t;
        const int page = (pos / KV_PAGE == pos0 / KV_PAGE) ? pg0 : pg1;
        const int plane = (region == 1 ? 0 : 2) + term;
        __half* kv = reinterpret_cast<__half*>(ep.kv_pool);
        const size_t i = kv_offset_pg(ep, page, pos, plane, hh, dd);
        if (FD_CHECK(i + 7 < ep.cap_kv, ep.check, 5, i, ep.cap_kv))
          *reinterpret_cast<uint4*>(kv + i) = val;
      }
    }
  }
  named_bar(bar, EPI_THREADS);
}

}  // namespace fd
