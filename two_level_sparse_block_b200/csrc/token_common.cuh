// Level-2 pieces shared by the token-select kernels (AsyncTLS, English
// summary 2.A Stage 2).
#pragma once

#include "device_common.cuh"

namespace tls {

struct TokenParams {
  const uint16_t* q;
  const int32_t* label_ch;
  const uint8_t* codes;
  const float* scales;
  const int32_t* block_idx;
  int n_q_heads, n_kv_heads, group, dqk, bs, nb;
  int64_t ctx_len;
  int K_b, k, n_cand, chunk;
  float* tscore;        // workspace [rows, n_cand]
  float* token_score;   // optional copy
  unsigned* counters;   // workspace [rows]
  int32_t* token_idx;   // [rows, k]
  const int32_t* seq_lens;  // optional [B]: tokens per sequence (later positions are not candidates)
};

template <int R>
__device__ __forceinline__ void load_codes(const uint8_t* p, float (&c)[R]) {
  uint32_t w[(R + 7) / 8];
  if constexpr (R == 2) {
    w[0] = p[0];
  } else if constexpr (R == 4) {
    w[0] = *reinterpret_cast<const uint16_t*>(p);
  } else if constexpr (R == 8) {
    w[0] = *reinterpret_cast<const uint32_t*>(p);
  } else if constexpr (R == 16) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    w[0] = v.x;
    w[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < R / 32; ++i) {
      const uint4 v = reinterpret_cast<const uint4*>(p)[i];
      w[4 * i + 0] = v.x;
      w[4 * i + 1] = v.y;
      w[4 * i + 2] = v.z;
      w[4 * i + 3] = v.w;
    }
  }
  // sign-extend the 4-bit two's complement codes without integer-to-float
  // conversions: with v = nibble ^ 8, the float bit pattern 0x4B000000 | v is
  // 2^23 + v, and subtracting 2^23 + 8 leaves v - 8 exactly
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const uint32_t v = ((w[r / 8] >> (4 * (r % 8))) & 15u) ^ 8u;
    c[r] = __uint_as_float(0x4B000000u | v) - 8388616.0f;
  }
}

// Candidate position -> absolute token position (block list in shared
// memory); shift and mask when the block size is a power of two.
struct CandidateToken {
  const int32_t* bidx;
  int bs;
  __device__ __forceinline__ int operator()(int i) const {
    if ((bs & (bs - 1)) == 0) {
      const int sh = __ffs(bs) - 1;
      return (bidx[i >> sh] << sh) | (i & (bs - 1));
    }
    return bidx[i / bs] * bs + (i % bs);
  }
};

// q values of the label channels of the row's group, float [G][R] in smem.
template <int R, int NT>
__device__ __forceinline__ void load_qlab(const TokenParams& p, int row, float* qlab) {
  const int g = p.group;
  const int b = row / p.n_kv_heads, kvh = row % p.n_kv_heads;
  const uint16_t* qg = p.q + ((int64_t)b * p.n_q_heads + (int64_t)kvh * g) * p.dqk;
  for (int i = threadIdx.x; i < g * R; i += NT) {
    const int h = i / R, r = i % R;
    const int ch = min(max(p.label_ch[kvh * R + r], 0), p.dqk - 1);  // clamped: never out of bounds
    qlab[i] = __uint_as_float((uint32_t)qg[(int64_t)h * p.dqk + ch] << 16);
  }
}

// The row's chosen blocks, clamped into [0, NB) so a bad list can never
// address outside the index, copied to shared memory (block_idx NULL: every
// block, 0 .. K_b - 1).  Returns how many entries are blocks (not the -1 that
// ends a list); every thread of the CTA must call it, and it ends with a CTA
// barrier, after which sb is complete.
// `pre` runs once in every thread while the first list loads are in flight,
// before the barrier (work that waits on other loads of the same thread).
template <int NT, typename Pre>
__device__ __forceinline__ int load_block_list(const TokenParams& p, int row, int32_t* sb, Pre pre) {
  int nvb = 0;
  for (int base = 0; base < p.K_b; base += NT) {
    const int i = base + (int)threadIdx.x;
    int v = -1;
    // L2 loads: the list is written by the preceding kernel while this grid
    // may already be resident (programmatic dependent launch)
    if (i < p.K_b) v = p.block_idx == nullptr ? i : __ldcg(p.block_idx + (int64_t)row * p.K_b + i);
    if (base == 0) pre();
    if (i < p.K_b) sb[i] = min(max(v, 0), p.nb - 1);
    nvb += __syncthreads_count(i < p.K_b && v >= 0);
  }
  return nvb;
}
template <int NT>
__device__ __forceinline__ int load_block_list(const TokenParams& p, int row, int32_t* sb) {
  return load_block_list<NT>(p, row, sb, [] {});
}

// The group's query rows (G x Dqk bf16, contiguous in q) copied into shared
// memory by 16-byte async copies, committed as one group (q 16-byte aligned,
// Dqk a multiple of 8).
template <int NT>
__device__ __forceinline__ void stage_query_rows(const TokenParams& p, int row, uint16_t* sq) {
  const int g = p.group, b = row / p.n_kv_heads, kvh = row % p.n_kv_heads;
  const uint16_t* qg = p.q + ((int64_t)b * p.n_q_heads + (int64_t)kvh * g) * p.dqk;
  const uint32_t s0 = smem_addr32(sq);
  for (int i = threadIdx.x; i < g * p.dqk / 8; i += NT) cp_async16(s0 + (uint32_t)i * 16u, qg + (int64_t)i * 8, 16u);
  cp_async_commit();
}

// Candidates of a row that are tokens of its sequence: the lists are
// ascending with any -1 at the end and only the sequence's last block can be
// partial, so they are a prefix of the candidate order -- every position of
// the nvb listed blocks, less the part of the highest one past the sequence.
__device__ __forceinline__ int valid_candidates(const TokenParams& p, int row, const int32_t* sb, int nvb) {
  if (nvb <= 0) return 0;
  const int64_t len = seq_len_of(p.seq_lens, row / p.n_kv_heads, p.ctx_len);
  const int64_t all = (int64_t)nvb * p.bs;
  const int64_t end = (int64_t)(sb[nvb - 1] + 1) * p.bs;  // one past the highest listed block
  const int64_t n = all - (end > len ? end - len : 0);
  return (int)(n < 0 ? 0 : n);
}

// Scores of candidates [c0, c1) of one row (candidates in ascending token
// order), score(t) = s_t * max_h sum_r qlab[h, r] * code_{t, r}, stored as
// order-preserving keys at keys[i - c0] (n_valid: candidates that are tokens
// of the sequence; the optional score copy gets -inf past them).
template <int R, int NT>
__device__ __forceinline__ void score_candidates(const TokenParams& p, int row, const float* qlab,
                                                 const int32_t* bidx, int c0, int c1, uint32_t* keys, int n_valid) {
  constexpr int U = 4;  // candidates per thread whose loads are in flight together
  const int g = p.group;
  const int tid = threadIdx.x;
  for (int base = c0; base < c1; base += NT * U) {
    float c[U][R];
    float sc[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + u * NT + tid;
      if (i < c1) {
        const int64_t at = (int64_t)row * p.ctx_len + (int64_t)bidx[i / p.bs] * p.bs + (i % p.bs);
        load_codes<R>(p.codes + at * (R / 2), c[u]);
        sc[u] = p.scales[at];
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + u * NT + tid;
      if (i < c1) {
        float best = -INFINITY;
        for (int h = 0; h < g; ++h) {
          const float* qh = qlab + h * R;
          float acc = 0.0f;
#pragma unroll
          for (int r = 0; r < R; ++r) acc = fmaf(qh[r], c[u][r], acc);
          best = fmaxf(best, acc);
        }
        const float score = sc[u] * best;
        keys[i - c0] = float_key(score);
        if (p.token_score != nullptr) p.token_score[(int64_t)row * p.n_cand + i] = i < n_valid ? score : -INFINITY;
      }
    }
  }
}

// Codes and scales of every candidate of a row copied to shared memory in
// candidate order (block by block, 16-byte asynchronous copies, all in flight
// at once), so that scoring waits on one round trip to memory instead of one
// per batch of candidates.  Needs bs * R / 2 and bs * 4 to be multiples of 16
// and 16-byte aligned codes and scales (token_row_kernel_fits).
// Blocks [j0, j1) of the row's list are staged; candidate j0 * bs lands at
// index 0.
template <int R, int NT>
__device__ __forceinline__ void stage_candidate_codes(const TokenParams& p, int row, const int32_t* bidx, int j0,
                                                      int j1, uint8_t* scodes, float* sscales) {
  const int cpb = p.bs * (R / 2) / 16;  // 16-byte chunks of codes per block
  const int per = cpb + p.bs * 4 / 16;  // ... and of scales
  const uint32_t sc0 = smem_addr32(scodes), ss0 = smem_addr32(sscales);
  for (int i = threadIdx.x; i < (j1 - j0) * per; i += NT) {
    const int j = i / per, c = i - j * per;
    const int64_t tok0 = (int64_t)row * p.ctx_len + (int64_t)bidx[j0 + j] * p.bs;
    if (c < cpb)
      cp_async16(sc0 + (uint32_t)(j * p.bs * (R / 2) + c * 16), p.codes + tok0 * (R / 2) + c * 16, 16u);
    else
      cp_async16(ss0 + (uint32_t)(j * p.bs * 4 + (c - cpb) * 16),
                 reinterpret_cast<const uint8_t*>(p.scales + tok0) + (c - cpb) * 16, 16u);
  }
  cp_async_commit();
  cp_async_wait<0>();
}

// Token scores on the tensor cores for wide groups (G >= 16, R = 16 or 32):
// per warp step 16 candidates, S[cand, head] = code[cand, :] . qlab[head, :]
// as m16n8k16 bf16 MMAs with fp32 accumulation (M = 16 candidates, N = 8
// heads per n-tile, K = the R label channels).  INT4 codes are integers in
// [-7, 7], exact in bf16, and qlab holds bf16 values, so every product is
// exact.  Then the max over the group's heads (n-tiles and lanes), times the
// token's scale.  Same output as score_candidates.
__device__ __forceinline__ uint32_t tok_pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// the two INT4 codes of one byte (low nibble = even channel) as bf16x2,
// without integer-to-float conversions: with v = nibble ^ 8, the bf16 bit
// pattern 0x4300 | v is 128 + v (v < 128 fits the 7 mantissa bits at
// exponent 7), and subtracting 136 (bf16 0x4308) leaves v - 8, the two's
// complement code, exactly
__device__ __forceinline__ uint32_t tok_codes_bf16x2(uint32_t byte) {
  const uint32_t t = ((byte & 0xFu) | ((byte & 0xF0u) << 12)) ^ 0x43084308u;
  uint32_t r;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(t), "r"(0x43084308u));
  return r;
}
__device__ __forceinline__ void tok_mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// STAGED: the codes and scales of candidates [c0, c1) were copied, in
// candidate order from index 0, to shared memory (scodes, sscales) by
// stage_candidate_codes.
template <int R, int NT, int NTILE, bool STAGED = false>
__device__ __forceinline__ void score_candidates_tc(const TokenParams& p, int row, const float* qlab,
                                                    const int32_t* bidx, int c0, int c1, uint32_t* keys,
                                                    int n_valid, const uint8_t* scodes = nullptr,
                                                    const float* sscales = nullptr) {
  static_assert(R == 16 || R == 32, "label channels for the tensor-core scorer");
  constexpr int KS = R / 16, NW = NT / 32;
  const int g = p.group;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
  // B fragments: n-tile j holds heads 8j .. 8j + 7 (zero beyond G)
  uint32_t bq[NTILE][KS][2];
#pragma unroll
  for (int j = 0; j < NTILE; ++j) {
    const int h = 8 * j + gq;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const float* qh = qlab + h * R + ks * 16 + 2 * tq;
      bq[j][ks][0] = h < g ? tok_pack_bf16(qh[0], qh[1]) : 0u;
      bq[j][ks][1] = h < g ? tok_pack_bf16(qh[8], qh[9]) : 0u;
    }
  }
  const CandidateToken map{bidx, p.bs};
  // U steps of 16 candidates per warp iteration: all their code and scale
  // loads are in flight before the first MMA (fewer in 1024-thread CTAs,
  // which have 64 registers a thread)
  constexpr int U = STAGED ? 2 : NT >= 1024 ? 2 : 4;
  for (int base0 = c0 + warp * 16; base0 < c1; base0 += NW * 16 * U) {
    uint32_t w[U][2][KS * 2];  // code words of fragment rows gq, gq + 8
    float sc[U][2];
    bool ok[U][2];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int base = base0 + u * NW * 16;
#pragma unroll
      for (int hlf = 0; hlf < 2; ++hlf) {
        const int i = base + gq + 8 * hlf;
        ok[u][hlf] = i < c1;
        const int64_t at = STAGED ? (ok[u][hlf] ? i - c0 : 0) : (int64_t)row * p.ctx_len + (ok[u][hlf] ? map(i) : 0);
        const uint8_t* cb = STAGED ? scodes : p.codes;
        const float* sb = STAGED ? sscales : p.scales;
        if constexpr (R == 16) {
          const uint2 c = ok[u][hlf] ? *reinterpret_cast<const uint2*>(cb + at * 8) : make_uint2(0u, 0u);
          w[u][hlf][0] = c.x;
          w[u][hlf][1] = c.y;
        } else {
          const uint4 c = ok[u][hlf] ? *reinterpret_cast<const uint4*>(cb + at * 16) : make_uint4(0u, 0u, 0u, 0u);
          w[u][hlf][0] = c.x;
          w[u][hlf][1] = c.y;
          w[u][hlf][2] = c.z;
          w[u][hlf][3] = c.w;
        }
        sc[u][hlf] = ok[u][hlf] ? sb[at] : 0.0f;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int base = base0 + u * NW * 16;
      if (base >= c1) break;  // warp-uniform
      float acc[NTILE][4];
#pragma unroll
      for (int j = 0; j < NTILE; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        // channels 16 ks + 2 tq, +1 are byte 8 ks + tq; channels + 8, + 9 are byte 8 ks + tq + 4
        const uint32_t lo0 = (w[u][0][2 * ks] >> (8 * tq)) & 0xFFu, hi0 = (w[u][0][2 * ks + 1] >> (8 * tq)) & 0xFFu;
        const uint32_t lo1 = (w[u][1][2 * ks] >> (8 * tq)) & 0xFFu, hi1 = (w[u][1][2 * ks + 1] >> (8 * tq)) & 0xFFu;
        const uint32_t a[4] = {tok_codes_bf16x2(lo0), tok_codes_bf16x2(lo1), tok_codes_bf16x2(hi0),
                               tok_codes_bf16x2(hi1)};
#pragma unroll
        for (int j = 0; j < NTILE; ++j) tok_mma(acc[j], a, bq[j][ks][0], bq[j][ks][1]);
      }
      // max over the group's heads: fragment columns 2 tq, 2 tq + 1 of every n-tile, then the 4 lanes of a row
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int j = 0; j < NTILE; ++j) {
        const int h = 8 * j + 2 * tq;
        if (h < g) {
          mx0 = fmaxf(mx0, acc[j][0]);
          mx1 = fmaxf(mx1, acc[j][2]);
        }
        if (h + 1 < g) {
          mx0 = fmaxf(mx0, acc[j][1]);
          mx1 = fmaxf(mx1, acc[j][3]);
        }
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      if (tq == 0) {
#pragma unroll
        for (int hlf = 0; hlf < 2; ++hlf) {
          if (!ok[u][hlf]) continue;
          const int i = base + gq + 8 * hlf;
          const float score = sc[u][hlf] * (hlf == 0 ? mx0 : mx1);
          keys[i - c0] = float_key(score);
          if (p.token_score != nullptr)
            p.token_score[(int64_t)row * p.n_cand + i] = i < n_valid ? score : -INFINITY;
        }
      }
    }
  }
}

// Whether level 2 runs as the row-cluster kernel: tensor-core scoring of a
// narrow group (G <= 16, 16 or 32 label channels) over at most 8192
// candidates, kept in registers by the leader's top-k, with the candidates'
// codes and scales staged in shared memory by 16-byte copies (block size a
// multiple of 4; the caller also checks 16-byte aligned codes and scales).
__host__ __device__ inline bool token_row_kernel_fits(int group, int n_label, int n_cand, int bs) {
  return group <= 16 && (n_label == 16 || n_label == 32) && n_cand <= 8192 && bs % 4 == 0;
}

// CTAs per row of the row-cluster kernel: 4, 2 or 1, as many as keep every
// CTA at 8 blocks or more and the grid within `max_ctas` CTAs.
__host__ __device__ inline int token_row_cluster_size(int rows, int K_b, int max_ctas) {
  int cl = 4;
  while (cl > 1 && ((int64_t)rows * cl > max_ctas || K_b < 8 * cl)) cl /= 2;
  return cl;
}

// CTAs per row of the cluster kernel: 4, or (tensor-core scoring only) 8 / 16
// while the rows leave most SMs idle and every CTA keeps 512 candidates or more.
// Rows whose candidates exceed 4 * kTokMaxPerCta take more CTAs still (up to
// 16), so that a CTA's keys stay within kTokMaxPerCta.
constexpr int kTokMaxPerCta = 8192;
__host__ __device__ inline int token_cluster_size(int rows, int n_cand, bool tc) {
  int cl = 4;
  while (tc && cl < 16 && (int64_t)rows * cl * 2 <= 148 && n_cand >= cl * 2 * 512) cl *= 2;
  while (cl < 16 && n_cand > cl * kTokMaxPerCta) cl *= 2;
  return cl;
}

// Candidates per row above which the cluster kernel's degenerate fallback
// gathers the keys in the workspace instead of the leader's shared memory, and
// above which the chunked kernel (all keys of a row in one CTA) is not used.
constexpr int kTokSmemKeysMax = 24576;
// Largest candidate count level 2 takes (16 CTAs of 4 * kTokMaxPerCta keys).
constexpr int kTokMaxCand = 16 * 4 * kTokMaxPerCta;

// Whether level 2 of a row is light enough for one 4-CTA cluster (the
// scores of all candidates in shared memory, no device-wide exchange).
__host__ __device__ inline bool token_cluster_fits(int group, int n_label, int n_cand) {
  return (int64_t)group * n_label * n_cand <= ((int64_t)1 << 20);
}

}  // namespace tls
