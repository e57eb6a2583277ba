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
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int nib = (int)((w[r / 8] >> (4 * (r % 8))) & 15u);
    c[r] = (float)((nib ^ 8) - 8);  // sign-extend the 4-bit two's complement code
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
// address outside the index, copied to shared memory.
template <int NT>
__device__ __forceinline__ void load_block_list(const TokenParams& p, int row, int32_t* sb) {
  // L2 loads: the list is written by the preceding kernel while this grid may
  // already be resident (programmatic dependent launch)
  for (int i = threadIdx.x; i < p.K_b; i += NT)
    sb[i] = min(max(__ldcg(p.block_idx + (int64_t)row * p.K_b + i), 0), p.nb - 1);
}

// Scores of candidates [c0, c1) of one row (candidates in ascending token
// order), score(t) = s_t * max_h sum_r qlab[h, r] * code_{t, r}, stored as
// order-preserving keys at keys[i - c0].
template <int R, int NT>
__device__ __forceinline__ void score_candidates(const TokenParams& p, int row, const float* qlab,
                                                 const int32_t* bidx, int c0, int c1, uint32_t* keys) {
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
        if (p.token_score != nullptr) p.token_score[(int64_t)row * p.n_cand + i] = score;
      }
    }
  }
}

// Whether level 2 of a row is light enough for one 4-CTA cluster (the
// scores of all candidates in shared memory, no device-wide exchange).
__host__ __device__ inline bool token_cluster_fits(int group, int n_label, int n_cand) {
  return (int64_t)group * n_label * n_cand <= ((int64_t)1 << 20);
}

}  // namespace tls
