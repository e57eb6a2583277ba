// Level 2 of the two-level selection (AsyncTLS, English summary 2.A Stage 2:
// Double-Sparsity token selection inside the chosen blocks, from selected
// key channels quantised to INT4, then the top-K_t tokens).
//
// Candidates of a row are the bs tokens of each of its K_b chosen blocks, in
// ascending token order.  A grid of (chunks, rows) CTAs scores them:
//     score(t) = s_t * max_h sum_r qlab[h, r] * code_{t, r}
// (s_t >= 0, so scaling after the max is the same as taking the max of the
// scaled dots), writes the scores to the workspace, and the last CTA of each
// row to finish runs the deterministic top-k over the row's scores.

#include <cstdlib>

#include "device_common.cuh"
#include "host_common.h"

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

template <int R, int NT>
__global__ void __launch_bounds__(NT) token_select_kernel(TokenParams p) {
  extern __shared__ float sm[];
  float* qlab = sm;  // [G][R]
  __shared__ int last;
  const int tid = threadIdx.x;
  const int row = blockIdx.y;
  const int g = p.group;
  const int b = row / p.n_kv_heads, kvh = row % p.n_kv_heads;
  const uint16_t* qg = p.q + ((int64_t)b * p.n_q_heads + (int64_t)kvh * g) * p.dqk;
  for (int i = tid; i < g * R; i += NT) {
    const int h = i / R, r = i % R;
    const int ch = min(max(p.label_ch[kvh * R + r], 0), p.dqk - 1);  // clamped: never out of bounds
    qlab[i] = __uint_as_float((uint32_t)qg[(int64_t)h * p.dqk + ch] << 16);
  }
  __syncthreads();

  const int32_t* bidx = p.block_idx + (int64_t)row * p.K_b;
  const int c0 = blockIdx.x * p.chunk;
  const int c1 = min(p.n_cand, c0 + p.chunk);
  float* out = p.tscore + (int64_t)row * p.n_cand;
  for (int i = c0 + tid; i < c1; i += NT) {
    const int64_t blk = min(max(bidx[i / p.bs], 0), p.nb - 1);  // clamped: never out of bounds
    const int64_t tok = blk * p.bs + (i % p.bs);
    const int64_t at = (int64_t)row * p.ctx_len + tok;
    float c[R];
    load_codes<R>(p.codes + at * (R / 2), c);
    const float s = p.scales[at];
    float best = -INFINITY;
    for (int h = 0; h < g; ++h) {
      const float* qh = qlab + h * R;
      float acc = 0.0f;
#pragma unroll
      for (int r = 0; r < R; ++r) acc = fmaf(qh[r], c[r], acc);
      best = fmaxf(best, acc);
    }
    const float score = s * best;
    out[i] = score;
    if (p.token_score != nullptr) p.token_score[(int64_t)row * p.n_cand + i] = score;
  }

  __threadfence();
  __syncthreads();
  if (tid == 0) last = atomicInc(&p.counters[row], gridDim.x - 1) == gridDim.x - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  uint32_t* keys = reinterpret_cast<uint32_t*>(sm + g * R);
  TopkScratch* ts = reinterpret_cast<TopkScratch*>(keys + p.n_cand);
  for (int i = tid; i < p.n_cand; i += NT) keys[i] = float_key(__ldcg(out + i));
  __syncthreads();
  const int bs = p.bs;
  cta_topk_ascending<NT>(keys, p.n_cand, p.k, p.token_idx + (int64_t)row * p.k, *ts,
                         [bidx, bs](int i) { return bidx[i / bs] * bs + (i % bs); });
}

tls_status select_tokens_impl(const tls_shape& s, const void* q, const int32_t* label_ch, const uint8_t* codes,
                              const float* scales, const int32_t* block_idx, int K_b, int k, int32_t* token_idx,
                              float* token_score, uint8_t* ws, const WsLayout& L, cudaStream_t stream) {
  constexpr int NT = 256;
  const int rows = rows_of(s);
  TokenParams p;
  p.q = (const uint16_t*)q;
  p.label_ch = label_ch;
  p.codes = codes;
  p.scales = scales;
  p.block_idx = block_idx;
  p.n_q_heads = s.n_q_heads;
  p.n_kv_heads = s.n_kv_heads;
  p.group = group_of(s);
  p.dqk = s.qk_dim;
  p.bs = s.block_size;
  p.nb = (int)n_blocks(s);
  p.ctx_len = s.ctx_len;
  p.K_b = K_b;
  p.k = k;
  p.n_cand = K_b * s.block_size;
  // enough CTAs for about two waves, at least one candidate per thread
  int chunks = (2 * kNumSMs + rows - 1) / rows;
  int chunk = (p.n_cand + chunks - 1) / chunks;
  chunk = (int)align_up((size_t)chunk, 32);
  if (chunk < NT) chunk = NT;
  p.chunk = chunk;
  chunks = (p.n_cand + chunk - 1) / chunk;
  p.tscore = reinterpret_cast<float*>(ws + L.tscore);
  p.token_score = token_score;
  p.counters = reinterpret_cast<unsigned*>(ws + L.tok_counter);
  p.token_idx = token_idx;

  const size_t smem = (size_t)p.group * s.n_label * 4 + (size_t)p.n_cand * 4 + sizeof(TopkScratch) + 16;
  dim3 grid((unsigned)chunks, (unsigned)rows);
  switch (s.n_label) {
#define TLS_TS_CASE(RR)                                                                                     \
  case RR: {                                                                                                \
    cudaError_t e =                                                                                         \
        cudaFuncSetAttribute(token_select_kernel<RR, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
    if (e != cudaSuccess) return cuda_check(e, "select_tokens: set smem attribute");                        \
    token_select_kernel<RR, NT><<<grid, NT, smem, stream>>>(p);                                             \
    break;                                                                                                  \
  }
    TLS_TS_CASE(2)
    TLS_TS_CASE(4)
    TLS_TS_CASE(8)
    TLS_TS_CASE(16)
    TLS_TS_CASE(32)
    TLS_TS_CASE(64)
#undef TLS_TS_CASE
    default:
      return fail(TLS_ERR_UNSUPPORTED, "select_tokens: n_label %d not built (2,4,8,16,32,64)", s.n_label);
  }
  return launch_check("select_tokens launch");
}

}  // namespace tls
