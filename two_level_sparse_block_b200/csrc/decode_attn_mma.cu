// Attention over the chosen tokens for small head groups (G <= 16) with
// 128-wide K and V rows (AsyncTLS, Italian summary 2.A.2: attention runs on
// the selected tokens only).
//
// At G <= 16 the gather does ~G flop per byte, so the kernel is HBM-bound; the
// design follows the bandwidth: persistent CTAs (two per SM) over contiguous
// ranges of 16-token chunks, every warp streaming its own chunks through a
// 3-stage cp.async ring with no CTA-wide barrier in the steady state.  The
// dot products run on the tensor cores through warp-level mma.sync
// (m16n8k16, bf16 -> fp32), whose results stay in registers:
//   S  = Q . K^T   A = q of the group's heads (rows >= G are zero), B = K rows
//                  via ldmatrix from a 128B-swizzled stage
//   softmax        online per head in fp32 registers, base 2
//   O += P . V     A = P from the S accumulators, split into bf16 hi + lo
//                  parts (two MMAs: P keeps ~16 significant bits), B = V rows
//                  via ldmatrix.trans
// At the end of each (row) segment of its range the CTA folds its warps in
// shared memory and writes (m, l, O) to the split workspace; the last CTA to
// finish a row merges the splits by log-sum-exp (attn_common.cuh).

#include <cooperative_groups.h>

#include "attn_common.cuh"
#include "device_common.cuh"
#include "host_common.h"

namespace tls {

constexpr int kMmaWarps = 4;
constexpr int kChunk = 16;           // tokens per chunk
constexpr int kChunkBytes = 8192;    // K (4 KB) + V (4 KB) of 16 tokens
constexpr int kMmaDv = 128;          // K and V row width of these kernels

// two floats -> bf16x2 (round to nearest even); `a` goes to the low half
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
  return r;
}
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
// update, and O += P.V with P split into bf16 hi + lo parts.  K and V tiles
// of the chunk at shared address kb / kb + 4096.
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
  // P as the A operand (k = the 16 tokens), hi and lo parts
  uint32_t ph[4], pl[4];
  {
    const float a[4][2] = {{pr[0][0], pr[0][1]}, {pr[0][2], pr[0][3]}, {pr[1][0], pr[1][1]}, {pr[1][2], pr[1][3]}};
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      ph[r] = pack_bf16(a[r][0], a[r][1]);
      pl[r] = pack_bf16(a[r][0] - bf16_lo_f(ph[r]), a[r][1] - bf16_hi_f(ph[r]));
    }
  }
  // O += P . V over 16 n-tiles of 8 value columns
#pragma unroll
  for (int j = 0; j < 16; j += 2) {
    // matrices: tokens 0-7 / 8-15 of unit j, then of unit j+1
    const int mtx = lane >> 3;
    const uint32_t addr = vb + tile_off((mtx & 1) * 8 + (lane & 7), j + (mtx >> 1));
    uint32_t b0, b1, b2, b3;
    ldsm_x4_t(addr, b0, b1, b2, b3);
    mma_bf16_16816(o[j], ph, b0, b1);
    mma_bf16_16816(o[j], pl, b0, b1);
    mma_bf16_16816(o[j + 1], ph, b2, b3);
    mma_bf16_16816(o[j + 1], pl, b2, b3);
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
    for (int w = 0; w < kMmaWarps; ++w) M = fmaxf(M, cm[w * 16 + tid]);
    float L = 0.0f;
#pragma unroll
    for (int w = 0; w < kMmaWarps; ++w) {
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

// Persistent form: every CTA owns a contiguous range of the (row, chunk)
// items; a row spread over several CTAs is merged by the last of them
// through the split workspace (attn_common.cuh).
template <int NS, bool RAGGED>
__global__ void __launch_bounds__(kMmaWarps * 32, 2) sparse_attn_mma_kernel(AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const int HPC = p.heads_per_cta, HG = p.head_groups;  // heads of a CTA item, head groups per row
  const MmaLayout L = mma_layout(HPC);
  float* comb = reinterpret_cast<float*>(sm + L.off_comb);
  float* cm = reinterpret_cast<float*>(sm + L.off_stat);
  float* cl = cm + kMmaWarps * 16;
  __shared__ int s_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int CPR = p.tiles_per_pair;  // chunks per row
  const int64_t C = p.n_items;
  const int64_t cta = blockIdx.x;
  const int64_t c_lo = cta * C / p.n_ctas, c_hi = (cta + 1) * C / p.n_ctas;
  const uint32_t ring_s = smem_u32(sm + warp * NS * kChunkBytes);

  // this warp's stream: chunks c_lo + warp + 4i
  const int64_t x0 = c_lo + warp;
  const int n_mine = x0 < c_hi ? (int)((c_hi - 1 - x0) / kMmaWarps + 1) : 0;
  // items are (virtual row, chunk); virtual row vr = (row, head group vr % HG)
  auto load_tok = [&](int i) -> int {
    if (i >= n_mine) return -1;
    const int64_t x = x0 + (int64_t)kMmaWarps * i;
    return mma_list_raw<RAGGED>(p, (int)(x / CPR) / HG, (int)(x % CPR), lane);
  };
  // issues chunk i from its raw list entry; returns the chunk's token mask
  auto issue = [&](int i, int raw, int st) -> uint32_t {
    int tok = -1;
    if (i < n_mine) {
      const int64_t x = x0 + (int64_t)kMmaWarps * i;
      const int r = (int)(x / CPR) / HG;
      tok = mma_list_token<RAGGED>(p, raw, (int)(x % CPR), lane,
                                   RAGGED ? seq_len_of(p.seq_lens, r / p.n_kv_heads, p.ctx_len) : p.ctx_len);
      mma_issue_rows(p, r, tok, ring_s + st * kChunkBytes, lane);
    }
    cp_async_commit();
    return mma_valid_mask(tok);
  };

  uint32_t qa[8][4];
  float o[16][4];
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f;  // fragment rows gq and gq + 8

  grid_launch_dependents();
  if (tid == 0 && c_lo < c_hi) {
    // what the first row end writes (split partials, the row's ticket, the
    // output and lse rows): prefetching them now also warms their address
    // translations while the token lists are still being selected
    const int v0 = (int)(c_lo / CPR), r0 = v0 / HG, h00 = (v0 % HG) * HPC;
    const int64_t f0 = attn_owner((int64_t)v0 * CPR, C, p.n_ctas);
    prefetch_l2(p.partial + (((int64_t)r0 * p.group + h00) * p.splits + (cta - f0)) * 130);
    prefetch_l2(p.counters + v0);
    const int64_t oh = (int64_t)(r0 / p.n_kv_heads) * p.n_q_heads + (int64_t)(r0 % p.n_kv_heads) * p.group + h00;
    prefetch_l2(reinterpret_cast<const uint8_t*>(p.out) + oh * p.dv * (p.out_bf16 ? 2 : 4));
    if (p.lse != nullptr) prefetch_l2(p.lse + oh);
  }
  grid_dependency_wait();  // token lists come from the preceding kernel

  // prologue: stages 0 .. S-2; token indices one chunk further ahead; vq
  // queues the issued chunks' token masks, 16 bits each, oldest lowest
  int tok_ahead[NS];
#pragma unroll
  for (int s = 0; s < NS; ++s) tok_ahead[s] = load_tok(s);
  uint64_t vq = 0;
#pragma unroll
  for (int s = 0; s < NS - 1; ++s) vq |= (uint64_t)issue(s, tok_ahead[s], s) << (16 * s);
  int tok_next = tok_ahead[NS - 1];  // for chunk S-1

  const int vrow_first = (int)(c_lo / CPR);
  const int vrow_last = (int)((c_hi - 1) / CPR);
  int i = 0;  // position in this warp's stream
  for (int vr = vrow_first; vr <= vrow_last; ++vr) {
    const int row = vr / HG, h0 = (vr % HG) * HPC, g = min(HPC, p.group - h0);
    const int b = row / p.n_kv_heads, kvh = row % p.n_kv_heads;
    // this virtual row's chunks inside the CTA range
    const int64_t seg_end = min(c_hi, (int64_t)(vr + 1) * CPR);
    mma_load_q(p, b, kvh, h0, g, lane, qa);
#pragma unroll
    for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.0f;
    m0 = m1 = -INFINITY;
    l0 = l1 = 0.0f;

    for (; i < n_mine && x0 + (int64_t)kMmaWarps * i < seg_end; ++i) {
      // keep S-1 chunks in flight; indices run one chunk further ahead
      const int tok_after = load_tok(i + NS);
      vq |= (uint64_t)issue(i + NS - 1, tok_next, (i + NS - 1) % NS) << (16 * (NS - 1));
      tok_next = tok_after;
      cp_async_wait<NS - 1>();
      __syncwarp();
      const uint32_t vm = (uint32_t)(vq & 0xFFFFu);
      vq >>= 16;
      mma_chunk(p, qa, o, m0, m1, l0, l1, ring_s + (i % NS) * kChunkBytes, vm, lane);
      __syncwarp();
    }

    // fold the warps of the CTA for this virtual row into its split of the workspace
    const int64_t first = attn_owner((int64_t)vr * CPR, C, p.n_ctas);
    const int n_part = (int)(attn_owner((int64_t)vr * CPR + CPR - 1, C, p.n_ctas) - first + 1);
    const int slot = (int)(cta - first);
    float* part = p.partial + (((int64_t)row * p.group + h0) * p.splits + slot) * 130;
    mma_fold(g, m0, m1, l0, l1, o, comb, cm, cl,
             [&](int h, int e, float v) { part[(int64_t)h * p.splits * 130 + e] = v; });
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicInc(&p.counters[vr], (unsigned)(n_part - 1)) == (unsigned)(n_part - 1);
    __syncthreads();
    if (s_last) {
      __threadfence();
      merge_splits(p, row, b, kvh, h0, g, n_part, comb, kMmaWarps * HPC * 128);
    }
    __syncthreads();  // the fold area is rewritten for the next row
  }
  cp_async_wait<0>();
}

// Cluster form: one cluster of CL = gridDim.x CTAs per row (row =
// blockIdx.y).  CTA r streams chunks [r * CPR / CL, (r + 1) * CPR / CL) of
// the row as above; then every CTA folds its warps, and CTA j merges output
// columns [j * 128 / CL, (j + 1) * 128 / CL) of every head by log-sum-exp:
// each CTA writes that slice of its folded O, with its (M, l) per head, into
// CTA j's drained cp.async ring over distributed shared memory.  Two cluster
// barriers; no workspace, ticket or device-wide fence.
template <int NS, bool RAGGED>
__global__ void __launch_bounds__(kMmaWarps * 32, 2) sparse_attn_mma_cluster_kernel(AttnParams p) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const int HPC = p.heads_per_cta, HG = p.head_groups;
  const MmaLayout L = mma_layout(HPC);
  float* comb = reinterpret_cast<float*>(sm + L.off_comb);
  float* cm = reinterpret_cast<float*>(sm + L.off_stat);
  float* cl = cm + kMmaWarps * 16;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // blockIdx.y is the virtual row (row, head group): heads h0 .. h0+g-1
  const int CL = (int)gridDim.x, rank = (int)blockIdx.x, vr = (int)blockIdx.y;
  const int row = vr / HG, h0 = (vr % HG) * HPC, g = min(HPC, p.group - h0);
  const int b = row / p.n_kv_heads, kvh = row % p.n_kv_heads;
  const int CPR = p.tiles_per_pair;
  const int c_lo = rank * CPR / CL, c_hi = (rank + 1) * CPR / CL;
  const uint32_t ring_s = smem_u32(sm + warp * NS * kChunkBytes);
  const int x0 = c_lo + warp;
  const int n_mine = x0 < c_hi ? (c_hi - 1 - x0) / kMmaWarps + 1 : 0;
  const int64_t len = RAGGED ? seq_len_of(p.seq_lens, b, p.ctx_len) : p.ctx_len;
  auto load_tok = [&](int i) -> int { return i < n_mine ? mma_list_raw<RAGGED>(p, row, x0 + kMmaWarps * i, lane) : -1; };
  // issues chunk i from its raw list entry; returns the chunk's token mask
  auto issue = [&](int i, int raw, int st) -> uint32_t {
    int tok = -1;
    if (i < n_mine) {
      tok = mma_list_token<RAGGED>(p, raw, x0 + kMmaWarps * i, lane, len);
      mma_issue_rows(p, row, tok, ring_s + st * kChunkBytes, lane);
    }
    cp_async_commit();
    return mma_valid_mask(tok);
  };
  const int64_t oh = (int64_t)b * p.n_q_heads + (int64_t)kvh * p.group + h0;  // first output head

  grid_launch_dependents();
  if (tid == 0) {
    // every CTA writes its column slice of the output rows last (the leader
    // the lse values too): warm them now
    prefetch_l2(reinterpret_cast<const uint8_t*>(p.out) + (oh * kMmaDv + rank * (kMmaDv / CL)) * (p.out_bf16 ? 2 : 4));
    if (p.lse != nullptr && rank == 0) prefetch_l2(p.lse + oh);
  }
  uint32_t qa[8][4];
  mma_load_q(p, b, kvh, h0, g, lane, qa);  // q is an input of the step, not of the preceding kernel
  grid_dependency_wait();           // token lists come from the preceding kernel

  float o[16][4];
#pragma unroll
  for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.0f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f;
  int tok_ahead[NS];
#pragma unroll
  for (int s = 0; s < NS; ++s) tok_ahead[s] = load_tok(s);
  uint64_t vq = 0;  // token masks of the issued chunks, 16 bits each, oldest lowest
#pragma unroll
  for (int s = 0; s < NS - 1; ++s) vq |= (uint64_t)issue(s, tok_ahead[s], s) << (16 * s);
  int tok_next = tok_ahead[NS - 1];
  for (int i = 0; i < n_mine; ++i) {
    const int tok_after = load_tok(i + NS);
    vq |= (uint64_t)issue(i + NS - 1, tok_next, (i + NS - 1) % NS) << (16 * (NS - 1));
    tok_next = tok_after;
    cp_async_wait<NS - 1>();
    __syncwarp();
    const uint32_t vm = (uint32_t)(vq & 0xFFFFu);
    vq >>= 16;
    mma_chunk(p, qa, o, m0, m1, l0, l1, ring_s + (i % NS) * kChunkBytes, vm, lane);
    __syncwarp();
  }
  cp_async_wait<0>();
  // barrier 1, split: arrive once this CTA's ring is drained, fold the warps
  // meanwhile, and wait before writing into the other CTAs' rings
  cluster_arrive_release();
  float* hm = cl + kMmaWarps * 16;
  float* hl = hm + 16;
  mma_fold_factors(g, m0, m1, l0, l1, o, comb, cm, cl, hm, hl);
  // CTA j merges output columns [j W, (j + 1) W) of every head: it receives
  // from every CTA r that slice of r's folded O and r's (M, l), in its own
  // drained ring
  const int W = kMmaDv / CL;
  float* recv = reinterpret_cast<float*>(sm);  // [CL][g][W]
  float* recv_ml = recv + CL * g * W;          // [CL][g] (M, l)
  cluster_wait_acquire();
  for (int idx = tid; idx < g * kMmaDv; idx += kMmaWarps * 32) {
    const int h = idx / kMmaDv, e = idx - h * kMmaDv;
    float v = 0.0f;
#pragma unroll
    for (int w = 0; w < kMmaWarps; ++w) v += cm[w * 16 + h] * comb[(w * g + h) * kMmaDv + e];
    const int j = e / W;
    cluster.map_shared_rank(recv, j)[(rank * g + h) * W + (e - j * W)] = v;
  }
  for (int idx = tid; idx < g * CL; idx += kMmaWarps * 32) {
    const int j = idx / g, h = idx - j * g;
    float* dst = cluster.map_shared_rank(recv_ml, j) + (rank * g + h) * 2;
    dst[0] = hm[h];
    dst[1] = hl[h];
  }
  cluster_arrive_release();
  cluster_wait_acquire();  // every slice has landed; nothing remote is touched after this

  for (int idx = tid; idx < g * W; idx += kMmaWarps * 32) {
    const int h = idx / W, c = idx - h * W;
    float M = -INFINITY;
    for (int r = 0; r < CL; ++r) M = fmaxf(M, recv_ml[(r * g + h) * 2]);
    float lsum = 0.0f, acc = 0.0f;
    if (M != -INFINITY) {
      for (int r = 0; r < CL; ++r) {
        const float mr = recv_ml[(r * g + h) * 2];
        if (mr == -INFINITY) continue;
        const float f = exp2f(mr - M);
        lsum += f * recv_ml[(r * g + h) * 2 + 1];
        acc += f * recv[(r * g + h) * W + c];
      }
    }
    const float val = lsum > 0.0f ? acc / lsum : 0.0f;
    const int64_t oe = (oh + h) * kMmaDv + rank * W + c;
    if (p.out_bf16) reinterpret_cast<uint16_t*>(p.out)[oe] = f32_to_bf16_rn(val);
    else reinterpret_cast<float*>(p.out)[oe] = val;
    if (rank == 0 && c == 0 && p.lse != nullptr)
      p.lse[oh + h] = lsum > 0.0f ? (M + log2f(lsum)) * 0.69314718055994531f : -INFINITY;
  }
}

// 128-wide K and V rows, any group size: groups above 16 heads are split
// into head groups of at most 16, each its own virtual row.
bool attn_mma_supported(const tls_shape& s) { return s.qk_dim == 128 && s.v_dim == 128 && s.v_offset < 0; }

// Work partition: chunks of 16 entries of every row's token list, contiguous
// ranges over two CTAs per SM.  Returns the largest number of CTAs sharing a row.
int attn_mma_plan(int rows, int k, int* chunks_per_row, int* n_items, int* n_ctas) {
  const int CPR = (k + kChunk - 1) / kChunk;
  const int64_t C = (int64_t)rows * CPR;
  const int64_t want = 2 * (int64_t)kNumSMs;
  const int64_t byw = (C + kMmaWarps - 1) / kMmaWarps;  // at least a chunk per warp
  int64_t n = want < byw ? want : byw;
  if (n > 63 * (int64_t)rows) n = 63 * (int64_t)rows;  // at most 64 splits per row
  int max_part = 1;
  for (int64_t r = 0; r < rows; ++r) {
    const int64_t parts = attn_owner(r * CPR + CPR - 1, C, n) - attn_owner(r * CPR, C, n) + 1;
    if (parts > max_part) max_part = (int)parts;
  }
  *chunks_per_row = CPR;
  *n_items = (int)C;
  *n_ctas = (int)n;
  return max_part;
}

// Cluster size of the cluster form for `rows` virtual rows of `hpc` heads:
// the largest of 16, 8, 4, 2 whose grid (rows x CL CTAs) fits two CTAs per
// SM and whose merge slices fit a CTA's ring (hpc * (128 + 2 CL) floats);
// 0 when even CL = 2 does not fit (many rows: the persistent form).
int attn_mma_cluster_size(int rows, int hpc) {
  const int ring_floats = kMmaWarps * mma_stages(hpc) * kChunkBytes / 4;
  for (int cl = 16; cl >= 2; cl /= 2) {
    if ((int64_t)rows * cl > 2 * (int64_t)kNumSMs) continue;
    if ((int64_t)hpc * (kMmaDv + 2 * cl) > ring_floats) continue;
    return cl;
  }
  return 0;
}

template <int NS, bool RAGGED>
static tls_status launch_mma(const AttnParams& p, int rows, cudaStream_t stream, bool pdl) {
  const MmaLayout L = mma_layout(p.heads_per_cta);
  const size_t smem = 128 + (size_t)L.bytes;
  rows *= p.head_groups;  // virtual rows (row, head group)
  const int cl = attn_mma_cluster_size(rows, p.heads_per_cta);
  if (cl > 0) {
    // 16-CTA clusters are beyond the portable size
    cudaError_t e = kernel_attrs((const void*)sparse_attn_mma_cluster_kernel<NS, RAGGED>, smem, cl > 8);
    if (e != cudaSuccess) return cuda_check(e, "sparse_decode_attn: set cluster attributes");
    return cuda_check(launch_ex(sparse_attn_mma_cluster_kernel<NS, RAGGED>, dim3(cl, rows), dim3(kMmaWarps * 32), smem,
                                stream, pdl, (unsigned)cl, p),
                      "sparse_decode_attn: mma cluster launch");
  }
  cudaError_t e = kernel_attrs((const void*)sparse_attn_mma_kernel<NS, RAGGED>, smem);
  if (e != cudaSuccess) return cuda_check(e, "sparse_decode_attn: set smem attribute");
  return cuda_check(
      launch_ex(sparse_attn_mma_kernel<NS, RAGGED>, dim3(p.n_ctas), dim3(kMmaWarps * 32), smem, stream, pdl, 0u, p),
      "sparse_decode_attn: mma launch");
}

// A token list with every sequence full (no per-sequence lengths) takes the
// kernels built for that case alone; the others read the list form and the
// lengths at run time.  Both skip entries that are no token.
tls_status launch_attn_mma(const AttnParams& p, int rows, cudaStream_t stream, bool pdl) {
  if (p.seq_lens == nullptr && p.list_mode == kListTokens) return launch_mma<3, false>(p, rows, stream, pdl);
  return launch_mma<3, true>(p, rows, stream, pdl);
}

}  // namespace tls
