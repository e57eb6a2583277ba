// Attention over the chosen tokens for the MLA latent cache (AsyncTLS,
// Italian summary 2.A.2: attention on the chosen tokens only; the pages
// validate the method on MLA): one latent row of 576 bf16 per token serves
// as the key, and its first 512 values as the value; all query heads of the
// row share it.
//
// At G = 128 heads the attention is ~240 flop per byte, so it runs on the
// tensor cores (warp-level mma.sync bf16 -> fp32).  CTA = (row, block of 16
// heads, 1/8 of the token list); the 8 token splits of a (row, head block)
// form a thread-block cluster.  Per 16-token chunk (18 KB, a CTA-shared
// 3-stage cp.async ring, rows of 72 16-byte units swizzled in groups of 8):
//   S = Q.K^T   each warp takes a quarter of the 576 dims (9 k-steps) into
//               a partial S; the four partials are summed in a fixed order
//               through shared memory, so every warp holds the same S
//   softmax     online, base 2, fp32, identical in the four warps
//   O += P.V    each warp its own 128 of the 512 value dims, in fp16 (P
//               rounded to fp16, V converted exactly)
// The split merge needs no workspace: each CTA leaves (m, l, O) in its
// drained ring, and after a cluster barrier CTA r merges output dims
// [64r, 64r + 64) of the 16 heads by log-sum-exp over the 8 CTAs, reading
// their partials through distributed shared memory.

#include <cooperative_groups.h>

#include "attn_common.cuh"
#include "device_common.cuh"
#include "host_common.h"

namespace tls {

constexpr int kMlaQk = 576, kMlaV = 512;
constexpr int kMlaWarps = 4;
constexpr int kMlaHeads = 16;                  // heads of a CTA (the m16n8k16 M)
constexpr int kMlaChunk = 16;                  // tokens per chunk
constexpr int kMlaUnits = kMlaQk * 2 / 16;     // 16-byte units of a latent row (72)
constexpr int kMlaRowBytes = kMlaQk * 2;       // 1152
constexpr int kMlaStageBytes = kMlaChunk * kMlaRowBytes;  // 18432
constexpr int kMlaStages = 3;
constexpr int kMlaSplits = 8;                  // CTAs per cluster = token splits
constexpr int kMlaKsteps = kMlaQk / 16 / kMlaWarps;       // k-steps of 16 dims per warp (9)

// byte offset of unit u (0..71) of token row r (0..15) inside a stage: within
// each group of 8 units (128 B) the unit index is XORed with the row, so the
// 8 rows an ldmatrix reads hit 8 different bank groups
__device__ __forceinline__ uint32_t mla_off(int r, int u) {
  return (uint32_t)(r * kMlaRowBytes + (((u & ~7) | ((u & 7) ^ (r & 7))) << 4));
}

// shared memory: ring [kMlaStages][kMlaStageBytes], then the partial-S
// exchange [2][kMlaWarps][16 x 16] fp32, then m/l [16] x 2
constexpr int kMlaOffS = kMlaStages * kMlaStageBytes;
constexpr int kMlaOffStat = kMlaOffS + 2 * kMlaWarps * 256 * 4;
constexpr int kMlaOffRid = kMlaOffStat + 2 * kMlaHeads * 4;  // then the split's row ids, int64 each
constexpr int kMlaSmem = kMlaOffRid;
// after the loop the ring holds this CTA's partial O [16][512] fp32 (rows
// padded to 520 floats, so the 8 rows a warp store touches hit 8 banks)
constexpr int kMlaOStride = kMlaV + 8;
static_assert(kMlaHeads * kMlaOStride * 4 <= kMlaStages * kMlaStageBytes, "partial O must fit the ring");

__device__ __forceinline__ float mla_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void mla_mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// O += P.V in fp16: P (in [0, 1]) rounds to fp16 with 11 significant bits
// (relative error <= 2^-11), and a pair of bf16 values of V converts to fp16
// exactly within fp16's range (bf16 carries 8 significant bits), so one MMA
// replaces the bf16 hi + lo pair at well under the output tolerance
__device__ __forceinline__ uint32_t mla_pack_f16(float a, float b) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
  return r;
}
__device__ __forceinline__ uint32_t mla_bf16x2_to_f16x2(uint32_t w) {
  return mla_pack_f16(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
__device__ __forceinline__ void mla_mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mla_ldsm4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mla_ldsm2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
__device__ __forceinline__ void mla_ldsm4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// cp.async of chunk c's 16 latent rows into the stage at shared address
// stage; every thread copies 9 of the 1152 units.  Row ids come from lanes
// 0..15 of the calling warp (rid, -1 = zero-fill).
__device__ __forceinline__ void mla_issue(const AttnParams& p, int64_t rid, uint32_t stage) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int i = 0; i < (kMlaChunk * kMlaUnits) / (kMlaWarps * 32); ++i) {
    const int idx = tid + i * kMlaWarps * 32;
    const int r = idx / kMlaUnits, u = idx - r * kMlaUnits;
    const int64_t rr = __shfl_sync(0xffffffffu, rid, r);
    const bool v = rr >= 0;
    cp_async16(stage + mla_off(r, u), p.k + (v ? rr * p.k_stride : 0) + u * 8, v ? 16u : 0u);
  }
}

// Row id (index into the K/V rows) of list entry t of the row (t < k), or -1
// when the entry is no token of the sequence (len tokens).
__device__ __forceinline__ int64_t mla_rid(const AttnParams& p, int row, int t, int64_t len) {
  const int tok = attn_token(p, row, t, len);
  return tok < 0 ? (int64_t)-1 : attn_row_id(p, row, tok);
}

template <int NS>
__global__ void __launch_bounds__(kMlaWarps * 32, 2) sparse_attn_mla_kernel(AttnParams p) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const uint32_t ring = smem_u32(sm);
  float* sS = reinterpret_cast<float*>(sm + kMlaOffS);     // [2][warp][i * 32 + lane]
  float* sM = reinterpret_cast<float*>(sm + kMlaOffStat);  // m [16], then l [16]
  float* sO = reinterpret_cast<float*>(sm);                // after the loop: O [16][kMlaOStride]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const int split = (int)cluster.block_rank(), row = (int)blockIdx.z;
  const int b = row / p.n_kv_heads, kvh = row % p.n_kv_heads, h0 = (int)blockIdx.y * kMlaHeads;
  const int t_lo = min(p.k_sel, split * p.tokens_per_split);
  const int t_hi = min(p.k_sel, t_lo + p.tokens_per_split);
  const int n_chunks = (t_hi - t_lo + kMlaChunk - 1) / kMlaChunk;
  const int64_t oh = (int64_t)b * p.n_q_heads + (int64_t)kvh * p.group + h0;  // first output head

  grid_launch_dependents();
  if (tid == 0) {
    // the output and lse rows are written last: warm their translations now
    prefetch_l2(reinterpret_cast<const uint8_t*>(p.out) + (oh * kMlaV + 64 * split) * (p.out_bf16 ? 2 : 4));
    if (p.lse != nullptr) prefetch_l2(p.lse + oh);
  }
  // Q fragments of this warp's 9 k-steps (dims 144 w .. 144 w + 143), 16 heads
  uint32_t qa[kMlaKsteps][4];
  {
    const uint16_t* q0 = p.q + (oh + gq) * p.dqk;
    const uint16_t* q8 = q0 + (int64_t)8 * p.dqk;
#pragma unroll
    for (int ks = 0; ks < kMlaKsteps; ++ks) {
      const int d0 = (warp * kMlaKsteps + ks) * 16 + 2 * tq;
      qa[ks][0] = *reinterpret_cast<const uint32_t*>(q0 + d0);
      qa[ks][1] = *reinterpret_cast<const uint32_t*>(q8 + d0);
      qa[ks][2] = *reinterpret_cast<const uint32_t*>(q0 + d0 + 8);
      qa[ks][3] = *reinterpret_cast<const uint32_t*>(q8 + d0 + 8);
    }
  }
  const int64_t len = seq_len_of(p.seq_lens, b, p.ctx_len);
  grid_dependency_wait();  // token lists come from the preceding kernel
  // a token list: the row ids of this split's entries, padded with -1
  // (zero-fill) to whole chunks -- one round trip to the list now instead of
  // one per chunk in the loop; other lists are computed where they are used
  int64_t* srid = reinterpret_cast<int64_t*>(sm + kMlaOffRid);
  const bool staged = p.list_mode == kListTokens;
  if (staged) {
    for (int i = tid; i < n_chunks * kMlaChunk; i += kMlaWarps * 32)
      srid[i] = t_lo + i < t_hi ? mla_rid(p, row, t_lo + i, len) : (int64_t)-1;
    __syncthreads();
  }
  // row id of entry i of this split (-1: no token, rows zero-filled and masked)
  auto rid_at = [&](int i) -> int64_t {
    if (staged) return srid[i];
    return t_lo + i < t_hi ? mla_rid(p, row, t_lo + i, len) : (int64_t)-1;
  };

  float o[16][4];
#pragma unroll
  for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.0f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f;  // fragment rows gq and gq + 8

#pragma unroll
  for (int s = 0; s < NS - 1; ++s) {
    if (s < n_chunks) mla_issue(p, rid_at(s * kMlaChunk + (lane & 15)), ring + s * kMlaStageBytes);
    cp_async_commit();
  }
  for (int c = 0; c < n_chunks; ++c) {
    cp_async_wait<NS - 2>();  // this thread's copies of chunk c have landed
    __syncthreads();          // everyone's have; every warp is past chunk c - 1
    {
      const int cn = c + NS - 1;  // refill the stage chunk c - 1 used
      if (cn < n_chunks) mla_issue(p, rid_at(cn * kMlaChunk + (lane & 15)), ring + (cn % NS) * kMlaStageBytes);
      cp_async_commit();
    }
    const uint32_t st = ring + (c % NS) * kMlaStageBytes;
    // the chunk's entries that are tokens (bit e: entry e)
    const uint32_t vm = __ballot_sync(0xffffffffu, rid_at(c * kMlaChunk + (lane & 15)) >= 0) & 0xFFFFu;

    // partial S over this warp's 144 dims: 16 heads x 16 tokens
    float s[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.0f;
      const int r = nt * 8 + (lane & 7);
#pragma unroll
      for (int ks = 0; ks + 1 < kMlaKsteps; ks += 2) {
        const int u0 = (warp * kMlaKsteps + ks) * 2;  // units of k-steps ks, ks + 1
        uint32_t b0, b1, b2, b3;
        mla_ldsm4(st + mla_off(r, u0 + (lane >> 3)), b0, b1, b2, b3);
        mla_mma(s[nt], qa[ks], b0, b1);
        mla_mma(s[nt], qa[ks + 1], b2, b3);
      }
      {
        const int ks = kMlaKsteps - 1;
        const int u0 = (warp * kMlaKsteps + ks) * 2;
        uint32_t b0, b1;
        mla_ldsm2(st + mla_off(r, u0 + ((lane >> 3) & 1)), b0, b1);
        mla_mma(s[nt], qa[ks], b0, b1);
      }
    }
    // the four partial S summed in a fixed order: every warp holds the same S
    // (element i of lane l at [i][l]: consecutive lanes, consecutive banks)
    float* mine = sS + ((c & 1) * kMlaWarps + warp) * 256 + lane;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) mine[(nt * 4 + e) * 32] = s[nt][e];
    __syncthreads();
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < kMlaWarps; ++w) v += sS[((c & 1) * kMlaWarps + w) * 256 + (nt * 4 + e) * 32 + lane];
        s[nt][e] = v * p.scale_log2;
      }
    if (vm != 0xFFFFu) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (!((vm >> (nt * 8 + 2 * tq + (e & 1))) & 1u)) s[nt][e] = -INFINITY;
    }
    // online softmax (rows gq: elements 0, 1; rows gq + 8: elements 2, 3)
    float mx0 = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
    float mx1 = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
    if (!__all_sync(0xffffffffu, n0 == m0 && n1 == m1)) {
      // 1 where the maximum did not move (also while a row has seen no token)
      const float c0 = n0 == m0 ? 1.0f : mla_exp2(m0 - n0), c1 = n1 == m1 ? 1.0f : mla_exp2(m1 - n1);
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
    // a row with no token so far keeps max -inf: its masked scores give 0
    const float z0 = n0 == -INFINITY ? 0.0f : n0, z1 = n1 == -INFINITY ? 0.0f : n1;
    float pr[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) pr[nt][e] = mla_exp2(s[nt][e] - (e < 2 ? z0 : z1));
    l0 += (pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]);
    l1 += (pr[0][2] + pr[0][3]) + (pr[1][2] + pr[1][3]);
    uint32_t pf[4];
    {
      const float a[4][2] = {{pr[0][0], pr[0][1]}, {pr[0][2], pr[0][3]}, {pr[1][0], pr[1][1]}, {pr[1][2], pr[1][3]}};
#pragma unroll
      for (int r = 0; r < 4; ++r) pf[r] = mla_pack_f16(a[r][0], a[r][1]);
    }
    // O += P . V over this warp's 128 value dims (units 16 w .. 16 w + 15), fp16
#pragma unroll
    for (int j = 0; j < 16; j += 2) {
      const int mtx = lane >> 3;
      uint32_t b0, b1, b2, b3;
      mla_ldsm4_t(st + mla_off((mtx & 1) * 8 + (lane & 7), 16 * warp + j + (mtx >> 1)), b0, b1, b2, b3);
      mla_mma_f16(o[j], pf, mla_bf16x2_to_f16x2(b0), mla_bf16x2_to_f16x2(b1));
      mla_mma_f16(o[j + 1], pf, mla_bf16x2_to_f16x2(b2), mla_bf16x2_to_f16x2(b3));
    }
  }
  cp_async_wait<0>();
  __syncthreads();  // the ring is free: it takes this CTA's partial O

  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int d = 128 * warp + j * 8 + 2 * tq;
    sO[gq * kMlaOStride + d] = o[j][0];
    sO[gq * kMlaOStride + d + 1] = o[j][1];
    sO[(gq + 8) * kMlaOStride + d] = o[j][2];
    sO[(gq + 8) * kMlaOStride + d + 1] = o[j][3];
  }
  if (warp == 0 && tq == 0) {
    sM[gq] = m0;
    sM[gq + 8] = m1;
    sM[kMlaHeads + gq] = l0;
    sM[kMlaHeads + gq + 8] = l1;
  }
  cluster.sync();  // every CTA's partial is in place

  // CTA r merges output dims [64 r, 64 r + 64) of the 16 heads over the cluster
  float* sW = sS;  // [16 heads][kMlaSplits] weights, then [16] lse
  const int CL = (int)cluster.num_blocks();
  if (tid < kMlaHeads) {
    float mj[kMlaSplits], lj[kMlaSplits];
    float M = -INFINITY;
#pragma unroll
    for (int j = 0; j < kMlaSplits; ++j) {
      mj[j] = -INFINITY;
      lj[j] = 0.0f;
      if (j < CL) {
        const float* rm = cluster.map_shared_rank(sM, j);
        mj[j] = rm[tid];
        lj[j] = rm[kMlaHeads + tid];
      }
      M = fmaxf(M, mj[j]);
    }
    float L = 0.0f;
#pragma unroll
    for (int j = 0; j < kMlaSplits; ++j) {
      const float f = mj[j] == -INFINITY ? 0.0f : exp2f(mj[j] - M);
      mj[j] = f;
      L += f * lj[j];
    }
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
#pragma unroll
    for (int j = 0; j < kMlaSplits; ++j) sW[tid * kMlaSplits + j] = mj[j] * inv;
    sW[kMlaHeads * kMlaSplits + tid] = (M + log2f(L)) * 0.69314718055994531f;
  }
  __syncthreads();
  for (int idx = tid; idx < kMlaHeads * 64; idx += kMlaWarps * 32) {
    const int h = idx >> 6, d = 64 * split + (idx & 63);
    float v[kMlaSplits];
#pragma unroll
    for (int j = 0; j < kMlaSplits; ++j) v[j] = j < CL ? cluster.map_shared_rank(sO, j)[h * kMlaOStride + d] : 0.0f;
    float acc = 0.0f;
#pragma unroll
    for (int j = 0; j < kMlaSplits; ++j) acc = fmaf(sW[h * kMlaSplits + j], v[j], acc);
    const int64_t oe = (oh + h) * kMlaV + d;
    if (p.out_bf16) reinterpret_cast<uint16_t*>(p.out)[oe] = f32_to_bf16_rn(acc);
    else reinterpret_cast<float*>(p.out)[oe] = acc;
    if (split == 0 && (idx & 63) == 0 && p.lse != nullptr) p.lse[oh + h] = sW[kMlaHeads * kMlaSplits + h];
  }
  cluster.sync();  // the other CTAs may still be reading this CTA's partial
}

bool attn_mla_supported(const tls_shape& s) {
  return s.qk_dim == kMlaQk && s.v_dim == kMlaV && s.v_offset == 0 && group_of(s) % kMlaHeads == 0;
}

int attn_mla_tokens_per_split(int k) {
  const int per = (k + kMlaSplits - 1) / kMlaSplits;
  return (per + kMlaChunk - 1) / kMlaChunk * kMlaChunk;
}

tls_status launch_attn_mla(const AttnParams& p, int rows, cudaStream_t stream, bool pdl) {
  // staged row ids only for a token list
  const size_t smem = 128 + (size_t)kMlaSmem + (p.list_mode == kListTokens ? (size_t)p.tokens_per_split * 8 : 0);
  cudaError_t e = kernel_attrs((const void*)sparse_attn_mla_kernel<kMlaStages>, smem);
  if (e != cudaSuccess) return cuda_check(e, "sparse_decode_attn: set smem attribute");
  const dim3 grid(kMlaSplits, (unsigned)(p.group / kMlaHeads), (unsigned)rows);
  return cuda_check(launch_ex(sparse_attn_mla_kernel<kMlaStages>, grid, dim3(kMlaWarps * 32), smem, stream, pdl,
                              (unsigned)kMlaSplits, p),
                    "sparse_decode_attn: mla launch");
}

}  // namespace tls
