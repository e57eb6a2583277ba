// Index build for the two-level selection (AsyncTLS, English summary 2.A
// Stage 1 block-level index, Italian summary 2.A.1 max/min of the keys, and
// 2.A Stage 2 channel selection with INT4 keys).
//
//   build_block_meta_kernel   per-block channel max and min of K (exact)
//   quant_label_kernel        per-token symmetric INT4 codes of R label channels
//
// Both are single memory-bound passes over K run at prefill (or when a range
// of tokens is appended); neither is part of the per-step hot path.

#include "device_common.cuh"
#include "host_common.h"

namespace tls {

// One CTA per (block, row).  VPR = Dqk/8 vector lanes per token row; the
// CTA's RP sub-rows stride over the block's tokens with 16-byte loads and a
// shared-memory reduction finishes the max/min.
__global__ void build_block_meta_kernel(const uint16_t* __restrict__ k, int64_t k_row_stride, int dqk,
                                        int bs, int64_t ctx_len, int64_t nb, int64_t blk0,
                                        uint16_t* __restrict__ meta) {
  extern __shared__ float red[];  // [RP][dqk] max, then [RP][dqk] min
  const int vpr = dqk / 8;
  const int rp = blockDim.x / vpr;
  const int tid = threadIdx.x;
  const int v = tid % vpr, sub = tid / vpr;
  const int64_t row = blockIdx.y;
  const int64_t blk = blk0 + blockIdx.x;
  const uint16_t* base = k + (row * ctx_len + blk * bs) * k_row_stride + v * 8;

  float mx[8], mn[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    mx[e] = -INFINITY;
    mn[e] = INFINITY;
  }
  if (sub < rp) {
    for (int t = sub; t < bs; t += rp) {
      uint4 w = *reinterpret_cast<const uint4*>(base + (int64_t)t * k_row_stride);
      float f[8];
      unpack8(w, f);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        mx[e] = fmaxf(mx[e], f[e]);
        mn[e] = fminf(mn[e], f[e]);
      }
    }
    float* rmx = red + (size_t)sub * dqk + v * 8;
    float* rmn = red + (size_t)(rp + sub) * dqk + v * 8;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      rmx[e] = mx[e];
      rmn[e] = mn[e];
    }
  }
  __syncthreads();
  uint16_t* out = meta + (row * nb + blk) * (int64_t)(2 * dqk);
  for (int c = tid; c < dqk; c += blockDim.x) {
    float a = -INFINITY, b = INFINITY;
    for (int r = 0; r < rp; ++r) {
      a = fmaxf(a, red[(size_t)r * dqk + c]);
      b = fminf(b, red[(size_t)(rp + r) * dqk + c]);
    }
    // max/min return one of the bf16 inputs, so the narrowing is exact
    out[c] = (uint16_t)(__float_as_uint(a) >> 16);
    out[dqk + c] = (uint16_t)(__float_as_uint(b) >> 16);
  }
}

// One thread per token.  s = max|x|/7 and code = rint(x/s) with IEEE float32
// division and round-half-even, exactly as the definition states.
template <int R>
__global__ void quant_label_kernel(const uint16_t* __restrict__ k, int64_t k_row_stride,
                                   const int32_t* __restrict__ label_ch, int dqk, int n_kv_heads, int64_t ctx_len,
                                   int64_t t0, int64_t t1, uint8_t* __restrict__ codes,
                                   float* __restrict__ scales) {
  __shared__ int lab[R];
  const int64_t row = blockIdx.y;
  const int kvh = (int)(row % n_kv_heads);
  // channel indices are clamped into the row so a bad index cannot read out of bounds
  if (threadIdx.x < R) lab[threadIdx.x] = min(max(label_ch[kvh * R + threadIdx.x], 0), dqk - 1);
  __syncthreads();
  const int64_t t = t0 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= t1) return;
  const uint16_t* src = k + (row * ctx_len + t) * k_row_stride;
  float x[R];
  float m = 0.0f;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    x[r] = __uint_as_float((uint32_t)src[lab[r]] << 16);
    m = fmaxf(m, fabsf(x[r]));
  }
  const float s = __fdiv_rn(m, 7.0f);
  uint8_t packed[R / 2];
#pragma unroll
  for (int r = 0; r < R; r += 2) {
    int c0 = 0, c1 = 0;
    if (s > 0.0f) {
      c0 = __float2int_rn(__fdiv_rn(x[r], s));
      c1 = __float2int_rn(__fdiv_rn(x[r + 1], s));
      c0 = max(-7, min(7, c0));
      c1 = max(-7, min(7, c1));
    }
    packed[r / 2] = (uint8_t)((c0 & 15) | ((c1 & 15) << 4));
  }
  uint8_t* dst = codes + (row * ctx_len + t) * (R / 2);
#pragma unroll
  for (int j = 0; j < R / 2; ++j) dst[j] = packed[j];
  scales[row * ctx_len + t] = s;
}

}  // namespace tls

using namespace tls;

extern "C" tls_status tls_build_block_meta(const tls_shape* shape, const void* k, int64_t k_row_stride,
                                           int64_t t0, int64_t t1, void* meta, void* stream) {
  clear_error();
  tls_status st = check_shape(shape);
  if (st != TLS_OK) return st;
  const tls_shape& s = *shape;
  if (k == nullptr || meta == nullptr) return fail(TLS_ERR_INVALID_ARG, "build_block_meta: null pointer");
  if (!aligned16(k)) return fail(TLS_ERR_INVALID_ARG, "build_block_meta: k must be 16-byte aligned");
  if (k_row_stride < s.qk_dim || k_row_stride % 8 != 0)
    return fail(TLS_ERR_INVALID_ARG, "build_block_meta: k_row_stride %lld must be >= qk_dim and a multiple of 8",
                (long long)k_row_stride);
  if (t0 < 0 || t1 > s.ctx_len || t0 >= t1 || t0 % s.block_size || t1 % s.block_size)
    return fail(TLS_ERR_INVALID_ARG, "build_block_meta: range [%lld, %lld) must be block aligned inside [0, N)",
                (long long)t0, (long long)t1);
  const int vpr = s.qk_dim / 8;
  const int rp = vpr >= 256 ? 1 : 256 / vpr;
  const int threads = rp * vpr;
  const size_t smem = (size_t)2 * rp * s.qk_dim * sizeof(float);
  dim3 grid((unsigned)((t1 - t0) / s.block_size), (unsigned)rows_of(s));
  build_block_meta_kernel<<<grid, threads, smem, (cudaStream_t)stream>>>(
      (const uint16_t*)k, k_row_stride, s.qk_dim, s.block_size, s.ctx_len, n_blocks(s), t0 / s.block_size,
      (uint16_t*)meta);
  return launch_check("build_block_meta launch");
}

extern "C" tls_status tls_quant_label_cache(const tls_shape* shape, const void* k, int64_t k_row_stride,
                                            const int32_t* label_ch, int64_t t0, int64_t t1, uint8_t* codes,
                                            float* scales, void* stream) {
  clear_error();
  tls_status st = check_shape(shape);
  if (st != TLS_OK) return st;
  const tls_shape& s = *shape;
  if (k == nullptr || label_ch == nullptr || codes == nullptr || scales == nullptr)
    return fail(TLS_ERR_INVALID_ARG, "quant_label_cache: null pointer");
  if (k_row_stride < s.qk_dim)
    return fail(TLS_ERR_INVALID_ARG, "quant_label_cache: k_row_stride must be >= qk_dim");
  if (t0 < 0 || t1 > s.ctx_len || t0 >= t1)
    return fail(TLS_ERR_INVALID_ARG, "quant_label_cache: bad token range [%lld, %lld)", (long long)t0,
                (long long)t1);
  dim3 grid((unsigned)((t1 - t0 + 255) / 256), (unsigned)rows_of(s));
  cudaStream_t cs = (cudaStream_t)stream;
  const uint16_t* kk = (const uint16_t*)k;
  switch (s.n_label) {
#define TLS_QL_CASE(RR)                                                                              \
  case RR:                                                                                           \
    quant_label_kernel<RR><<<grid, 256, 0, cs>>>(kk, k_row_stride, label_ch, s.qk_dim, s.n_kv_heads, s.ctx_len, \
                                                 t0, t1, codes, scales);                             \
    break;
    TLS_QL_CASE(2)
    TLS_QL_CASE(4)
    TLS_QL_CASE(8)
    TLS_QL_CASE(16)
    TLS_QL_CASE(32)
    TLS_QL_CASE(64)
#undef TLS_QL_CASE
    default:
      return fail(TLS_ERR_UNSUPPORTED, "quant_label_cache: n_label %d not built (2,4,8,16,32,64)", s.n_label);
  }
  return launch_check("quant_label_cache launch");
}
