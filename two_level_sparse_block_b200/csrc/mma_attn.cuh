// Warp-level tensor-core attention pieces of the mma attention kernels
// (decode_attn_mma.cu): 16-token chunks of 128-wide K and V rows staged by
// cp.async into 128B-swizzled tiles, S = Q.K^T and O += P.V on mma.sync
// m16n8k16 (bf16 -> fp32), an fp32 online softmax in base 2, and the fold of
// a CTA's warps (for any warp count).
#pragma once

#include <cooperative_groups.h>

#include "attn_common.cuh"
#include "device_common.cuh"

namespace tls {

constexpr int kMmaWarps = 4;
constexpr int kChunk = 16;           // tokens per chunk
constexpr int kChunkBytes = 8192;    // K (4 KB) + V (4 KB) of 16 tokens
constexpr int kMmaDv = 128;          // K and V row width of these kernels

// the two bf16 halves of a 32-bit word as floats
__device__ __forceinline__ float bf16_lo_f(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi_f(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// 2^x with the hardware approximation (relative error ~2^-22, far below the
// 2e-3 output tolerance); 2^-inf = 0
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_f16(float a, float b) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
  return r;
}
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) { return pack_f16(bf16_lo_f(w), bf16_hi_f(w)); }

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// byte offset of 16-byte unit c (0..15) of token row r (0..15) inside a 4 KB
// tile of 256-byte rows; the low 3 bits of c are XORed with r so that the 8
// rows an ldmatrix reads hit 8 different bank groups
__device__ __forceinline__ uint32_t tile_off(int r, int c) {
  return (uint32_t)(r * 256 + (((c & 8) | ((c & 7) ^ (r & 7))) << 4));
}

struct MmaLayout {
  int off_comb, off_stat, bytes;
};
// ring stages per warp: 3 (two chunks in flight while one is computed), so
// that two CTAs (eight warps) fit on an SM: instruction latency, not memory
// depth, is what limits a warp here
__host__ __device__ constexpr int mma_stages(int g) { return 3; }
__host__ __device__ inline MmaLayout mma_layout(int g) {
  MmaLayout L;
  L.off_comb = kMmaWarps * mma_stages(g) * kChunkBytes;    // [warp][h][128] fp32
  L.off_stat = L.off_comb + kMmaWarps * g * 128 * 4;        // [warp][h] m, then l; [h] M, then l
  L.bytes = L.off_stat + (2 * kMmaWarps + 2) * 16 * 4 + 16;
  return L;
}

// Q fragments (the A operand of S = Q.K^T, 8 k-steps of 16) of heads
// h0 .. h0+g-1 of the group of row (b, kvh); fragment rows >= g are zero.
__device__ __forceinline__ void mma_load_q(const AttnParams& p, int b, int kvh, int h0, int g, int lane,
                                           uint32_t (&qa)[8][4]) {
  const int gq = lane >> 2, tq = lane & 3;
  const uint16_t* q0 = p.q + ((int64_t)b * p.n_q_heads + (int64_t)kvh * p.group + h0 + gq) * p.dqk;
  const uint16_t* q8 = q0 + (int64_t)8 * p.dqk;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int d0 = ks * 16 + 2 * tq;
    qa[ks][0] = gq < g ? *reinterpret_cast<const uint32_t*>(q0 + d0) : 0u;
    qa[ks][1] = gq + 8 < g ? *reinterpret_cast<const uint32_t*>(q8 + d0) : 0u;
    qa[ks][2] = gq < g ? *reinterpret_cast<const uint32_t*>(q0 + d0 + 8) : 0u;
    qa[ks][3] = gq + 8 < g ? *reinterpret_cast<const uint32_t*>(q8 + d0 + 8) : 0u;
  }
}

// Raw list entry (lane & 15) of chunk x of the row's list, or -1 past the
// end of the list: the token (a token list), the position (every position),
// or the block holding the position (a block list).  Nothing is computed on
// the loaded value here: the load runs a chunk ahead of its use, and any
// arithmetic on it would make the warp wait for it at once.  RAGGED covers
// every list form; otherwise the list is a token list.
template <bool RAGGED>
__device__ __forceinline__ int mma_list_raw(const AttnParams& p, int row, int x, int lane) {
  const int t = x * kChunk + (lane & 15);
  if (t >= p.k_sel) return -1;
  // L2 loads: the list is written by the preceding kernel while this grid is
  // already resident (programmatic dependent launch)
  if (!RAGGED || p.list_mode == kListTokens) return __ldcg(p.token_idx + (int64_t)row * p.k_sel + t);
  if (p.list_mode == kListAll) return t;
  return __ldcg(p.blocks + (int64_t)row * p.K_b + t / p.bs);
}

// Token of a raw entry of chunk x (lane & 15), or -1 when it is none of the
// sequence's len tokens (list padding, past the list end, out of range).
template <bool RAGGED>
__device__ __forceinline__ int mma_list_token(const AttnParams& p, int raw, int x, int lane, int64_t len) {
  if (raw < 0) return -1;
  int64_t tok = raw;
  if (RAGGED && p.list_mode == kListBlocks) tok = (int64_t)raw * p.bs + (x * kChunk + (lane & 15)) % p.bs;
  return tok < len ? (int)tok : -1;
}

// The chunk's 16 entries that are tokens (bit e: entry e), from the lane
// values of mma_list_token; all lanes of the warp call it.
__device__ __forceinline__ uint32_t mma_valid_mask(int tok) {
  return __ballot_sync(0xffffffffu, tok >= 0) & 0xFFFFu;
}

// cp.async of the K and V rows of one chunk into the ring stage at shared
// address kb (K tile; V tile at kb + 4096).  Entry lane & 15 holds token
// `tok` in [0, N) (-1: the rows are zero-filled and the scores masked);
// slots are clamped to the pool.  The caller commits the group.
__device__ __forceinline__ void mma_issue_rows(const AttnParams& p, int row, int tok, uint32_t kb, int lane) {
  const int64_t rid = tok >= 0 ? attn_row_id(p, row, tok) : -1;
  const uint32_t vb = kb + 4096;
  const int c = lane & 15;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int r = (lane >> 4) + 2 * j;
    const int64_t rr = __shfl_sync(0xffffffffu, rid, r);
    const bool v = rr >= 0;
    const uint32_t off = tile_off(r, c);
    cp_async16(kb + off, p.k + (v ? rr * p.k_stride : 0) + c * 8, v ? 16u : 0u);
    cp_async16(vb + off, p.v + (v ? rr * p.v_stride : 0) + c * 8, v ? 16u : 0u);
  }
}

// One chunk of 16 list entries for the fragment rows gq (m0, l0) and gq + 8
// (m1, l1): S = Q.K^T scaled to base 2 and masked where the entry is no token
// (bit e of vm clear: past the list end, or padding), the online softmax
// update, and O += P.V in fp16.  K and V tiles of the chunk at shared
// address kb / kb + 4096.
__device__ __forceinline__ void mma_chunk(const AttnParams& p, const uint32_t (&qa)[8][4], float (&o)[16][4],
                                          float& m0, float& m1, float& l0, float& l1, uint32_t kb, uint32_t vm,
                                          int lane) {
  const int tq = lane & 3;
  const uint32_t vb = kb + 4096;
  // S = Q . K^T for 16 tokens (two n-tiles of 8)
  float s[2][4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.0f;
#pragma unroll
    for (int ks = 0; ks < 8; ks += 2) {
      // matrices: (k-step ks, units 2ks, 2ks+1), (ks+1, units 2ks+2, 2ks+3)
      const int mtx = lane >> 3;
      const uint32_t addr = kb + tile_off(nt * 8 + (lane & 7), ks * 2 + mtx);
      uint32_t b0, b1, b2, b3;
      ldsm_x4(addr, b0, b1, b2, b3);
      mma_bf16_16816(s[nt], qa[ks], b0, b1);
      mma_bf16_16816(s[nt], qa[ks + 1], b2, b3);
    }
  }
  // scale (and mask the tail of the list), online softmax
  // (rows gq: elements 0,1; rows gq+8: elements 2,3)
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) s[nt][e] *= p.scale_log2;
  if (vm != 0xFFFFu) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (!((vm >> (nt * 8 + 2 * tq + (e & 1))) & 1u)) s[nt][e] = -INFINITY;
  }
  float mx0 = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
  float mx1 = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
  const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
  // the O rescale is skipped (warp-uniformly) when no row maximum moved
  if (!__all_sync(0xffffffffu, n0 == m0 && n1 == m1)) {
    // 0 on a row's first token; 1 where the maximum did not move (also while
    // a row has seen no token at all: both -inf)
    const float c0 = n0 == m0 ? 1.0f : fast_exp2(m0 - n0), c1 = n1 == m1 ? 1.0f : fast_exp2(m1 - n1);
    l0 *= c0;
    l1 *= c1;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      o[j][0] *= c0;
      o[j][1] *= c0;
      o[j][2] *= c1;
      o[j][3] *= c1;
    }
    m0 = n0;
    m1 = n1;
  }
  // a row with no token so far keeps max -inf: its masked scores give 2^-inf = 0
  const float z0 = n0 == -INFINITY ? 0.0f : n0, z1 = n1 == -INFINITY ? 0.0f : n1;
  float pr[2][4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) pr[nt][e] = fast_exp2(s[nt][e] - (e < 2 ? z0 : z1));
  l0 += (pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]);
  l1 += (pr[0][2] + pr[0][3]) + (pr[1][2] + pr[1][3]);
  // P as the A operand (k = the 16 tokens) in fp16: P in [0, 1] rounds with
  // relative error <= 2^-11, and V's bf16 pairs convert to fp16 exactly
  // within fp16's range, so one MMA per n-tile replaces a bf16 hi + lo pair
  uint32_t pf[4];
  {
    const float a[4][2] = {{pr[0][0], pr[0][1]}, {pr[0][2], pr[0][3]}, {pr[1][0], pr[1][1]}, {pr[1][2], pr[1][3]}};
#pragma unroll
    for (int r = 0; r < 4; ++r) pf[r] = pack_f16(a[r][0], a[r][1]);
  }
  // O += P . V over 16 n-tiles of 8 value columns
#pragma unroll
  for (int j = 0; j < 16; j += 2) {
    // matrices: tokens 0-7 / 8-15 of unit j, then of unit j+1
    const int mtx = lane >> 3;
    const uint32_t addr = vb + tile_off((mtx & 1) * 8 + (lane & 7), j + (mtx >> 1));
    uint32_t b0, b1, b2, b3;
    ldsm_x4_t(addr, b0, b1, b2, b3);
    mma_f16_16816(o[j], pf, bf16x2_to_f16x2(b0), bf16x2_to_f16x2(b1));
    mma_f16_16816(o[j + 1], pf, bf16x2_to_f16x2(b2), bf16x2_to_f16x2(b3));
  }
}

// The CTA's warps fold their (m, l, O) for one row: they write them to
// shared memory (comb [warp][h][128], cm / cl [warp][16]) and, after a
// barrier, put(h, e, v) receives for every head h < g the CTA's combined
// values relative to its own maximum M: e = 0 -> M, e = 1 -> l,
// e = 2 + d -> O[d].  All threads of the CTA must call it.
template <typename Put>
__device__ __forceinline__ void mma_fold(int g, float m0, float m1, float l0, float l1, const float (&o)[16][4],
                                         float* comb, float* cm, float* cl, Put put) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  if (tq == 0) {
    if (gq < g) {
      cm[warp * 16 + gq] = m0;
      cl[warp * 16 + gq] = l0;
    }
    if (gq + 8 < g) {
      cm[warp * 16 + gq + 8] = m1;
      cl[warp * 16 + gq + 8] = l1;
    }
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int d = j * 8 + 2 * tq;
    if (gq < g) {
      comb[(warp * g + gq) * 128 + d] = o[j][0];
      comb[(warp * g + gq) * 128 + d + 1] = o[j][1];
    }
    if (gq + 8 < g) {
      comb[(warp * g + gq + 8) * 128 + d] = o[j][2];
      comb[(warp * g + gq + 8) * 128 + d + 1] = o[j][3];
    }
  }
  __syncthreads();
  for (int idx = tid; idx < g * 130; idx += kMmaWarps * 32) {
    const int h = idx / 130, e = idx % 130;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kMmaWarps; ++w) M = fmaxf(M, cm[w * 16 + h]);
    float val = 0.0f;
    if (e == 0) {
      val = M;
    } else if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kMmaWarps; ++w) {
        const float mw = cm[w * 16 + h];
        if (mw == -INFINITY) continue;
        const float f = exp2f(mw - M);
        val += f * (e == 1 ? cl[w * 16 + h] : comb[(w * g + h) * 128 + (e - 2)]);
      }
    }
    put(h, e, val);
  }
}

// The CTA's warps fold their (m, l) for one row into factors: afterwards
// comb [warp][h][128] holds each warp's O (relative to its own maximum),
// cm [warp][h] the factor 2^(m_w - M) that brings it to the CTA's maximum
// M = hm[h] (0 for a warp that saw no token), and hl[h] the CTA's l
// relative to M.  All threads of the CTA call it.
template <int NW = kMmaWarps>
__device__ __forceinline__ void mma_fold_factors(int g, float m0, float m1, float l0, float l1,
                                                 const float (&o)[16][4], float* comb, float* cm, float* cl,
                                                 float* hm, float* hl) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  if (tq == 0) {
    if (gq < g) {
      cm[warp * 16 + gq] = m0;
      cl[warp * 16 + gq] = l0;
    }
    if (gq + 8 < g) {
      cm[warp * 16 + gq + 8] = m1;
      cl[warp * 16 + gq + 8] = l1;
    }
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int d = j * 8 + 2 * tq;
    if (gq < g) *reinterpret_cast<float2*>(comb + (warp * g + gq) * 128 + d) = make_float2(o[j][0], o[j][1]);
    if (gq + 8 < g) *reinterpret_cast<float2*>(comb + (warp * g + gq + 8) * 128 + d) = make_float2(o[j][2], o[j][3]);
  }
  __syncthreads();
  if (tid < g) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, cm[w * 16 + tid]);
    float L = 0.0f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float mw = cm[w * 16 + tid];
      const float f = mw == -INFINITY ? 0.0f : exp2f(mw - M);
      cm[w * 16 + tid] = f;
      L += f * cl[w * 16 + tid];
    }
    hm[tid] = M;
    hl[tid] = L;
  }
  __syncthreads();
}

__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

}  // namespace tls
