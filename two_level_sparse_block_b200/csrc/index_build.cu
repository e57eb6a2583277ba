// Index build for the two-level selection (AsyncTLS, English summary 2.A
// Stage 1 block-level index, Italian summary 2.A.1 max/min of the keys, and
// 2.A Stage 2 channel selection with INT4 keys).
//
//   build_block_meta_kernel   per-block channel max and min of K (exact)
//   quant_label_kernel        per-token symmetric INT4 codes of R label channels
//   append_kv_kernel          one decoded token per sequence: its K/V rows, the
//                             running max/min of its block, its INT4 codes
//
// The first two are single memory-bound passes over K run at prefill (or when
// a range of tokens is appended); the third is the per-step update.  A
// sequence's tokens are its first len_b positions (seq_lens); a block holding
// fewer than bs of them (the last one) has the max/min of those it holds.

#include "device_common.cuh"
#include "host_common.h"

namespace tls {

// One CTA per (block, row).  VPR = Dqk/8 vector lanes per token row; the
// CTA's RP sub-rows stride over the block's tokens with 16-byte loads and a
// shared-memory reduction finishes the max/min.
__global__ void build_block_meta_kernel(const uint16_t* __restrict__ k, int64_t k_row_stride, int dqk,
                                        int bs, int64_t ctx_len, int64_t nb, int64_t blk0, int64_t t1,
                                        const int32_t* __restrict__ seq_lens, int n_kv_heads,
                                        uint16_t* __restrict__ meta) {
  extern __shared__ float red[];  // [RP][dqk] max, then [RP][dqk] min
  const int vpr = dqk / 8;
  const int rp = blockDim.x / vpr;
  const int tid = threadIdx.x;
  const int v = tid % vpr, sub = tid / vpr;
  const int64_t row = blockIdx.y;
  const int64_t blk = blk0 + blockIdx.x;
  const uint16_t* base = k + (row * ctx_len + blk * bs) * k_row_stride + v * 8;
  // the block's tokens below min(t1, len): all bs, fewer for a partial block,
  // none past the sequence (then the block is left as it is)
  const int64_t end = min(t1, seq_len_of(seq_lens, (int)(row / n_kv_heads), ctx_len));
  const int nt = (int)max((int64_t)0, min((int64_t)bs, end - blk * bs));
  if (nt == 0) return;

  float mx[8], mn[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    mx[e] = -INFINITY;
    mn[e] = INFINITY;
  }
  if (sub < rp) {
    for (int t = sub; t < nt; t += rp) {
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

// Symmetric INT4 codes of one token's R label channels: s = max|x|/7 and
// code = rint(x/s) with IEEE float32 division and round-half-even, exactly as
// the definition states (s = 0: all codes 0).  lab: the R channel indices.
template <int R>
__device__ __forceinline__ void quant_token(const uint16_t* __restrict__ src, const int* lab, uint8_t* dst,
                                            float* scale) {
  float x[R];
  float m = 0.0f;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    x[r] = __uint_as_float((uint32_t)src[lab[r]] << 16);
    m = fmaxf(m, fabsf(x[r]));
  }
  const float s = __fdiv_rn(m, 7.0f);
#pragma unroll
  for (int r = 0; r < R; r += 2) {
    int c0 = 0, c1 = 0;
    if (s > 0.0f) {
      c0 = __float2int_rn(__fdiv_rn(x[r], s));
      c1 = __float2int_rn(__fdiv_rn(x[r + 1], s));
      c0 = max(-7, min(7, c0));
      c1 = max(-7, min(7, c1));
    }
    dst[r / 2] = (uint8_t)((c0 & 15) | ((c1 & 15) << 4));
  }
  *scale = s;
}

// One thread per token.
template <int R>
__global__ void quant_label_kernel(const uint16_t* __restrict__ k, int64_t k_row_stride,
                                   const int32_t* __restrict__ label_ch, int dqk, int n_kv_heads, int64_t ctx_len,
                                   int64_t t0, int64_t t1, const int32_t* __restrict__ seq_lens,
                                   uint8_t* __restrict__ codes, float* __restrict__ scales) {
  __shared__ int lab[R];
  const int64_t row = blockIdx.y;
  const int kvh = (int)(row % n_kv_heads);
  // channel indices are clamped into the row so a bad index cannot read out of bounds
  if (threadIdx.x < R) lab[threadIdx.x] = min(max(label_ch[kvh * R + threadIdx.x], 0), dqk - 1);
  __syncthreads();
  const int64_t t = t0 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= min(t1, seq_len_of(seq_lens, (int)(row / n_kv_heads), ctx_len))) return;
  quant_token<R>(k + (row * ctx_len + t) * k_row_stride, lab, codes + (row * ctx_len + t) * (R / 2),
                 scales + row * ctx_len + t);
}

// One CTA per sequence b: with t = seq_lens[b] (< N), for every KV head the
// new K row (and V row) is stored as token t, the index of block t / bs takes
// it in -- (k, k) when t starts the block, else the channel-wise max / min --
// and its label channels are quantised; then seq_lens[b] = t + 1.
struct AppendParams {
  const uint16_t* k_new;  // [B, Hkv, Dqk]
  const uint16_t* v_new;  // [B, Hkv, Dv] or NULL
  uint16_t* k;            // K rows (dense or the slot pool)
  uint16_t* v;            // V rows, or NULL
  int64_t k_stride, v_stride;
  const int32_t* slot_of_block;  // NULL: dense
  int n_slots;
  uint16_t* meta;
  const int32_t* label_ch;
  uint8_t* codes;
  float* scales;
  int n_kv_heads, dqk, dv, bs, nb;
  int64_t ctx_len;
};

template <int R>
__global__ void __launch_bounds__(128) append_kv_kernel(int32_t* seq_lens, AppendParams p) {
  __shared__ int lab[R];
  const int b = blockIdx.x, tid = threadIdx.x;
  const int t = seq_lens[b];
  __syncthreads();  // every thread has read the length before it changes
  if (t < 0 || t >= p.ctx_len) return;  // a full (or invalid) sequence is left unchanged
  const int j = t / p.bs;
  const bool first = t % p.bs == 0;
  for (int h = 0; h < p.n_kv_heads; ++h) {
    const int64_t row = (int64_t)b * p.n_kv_heads + h;
    const uint16_t* kn = p.k_new + row * p.dqk;
    int64_t rid = row * p.ctx_len + t;
    if (p.slot_of_block != nullptr) {
      const int slot = p.slot_of_block[row * p.nb + j];
      rid = slot >= 0 && slot < p.n_slots ? (int64_t)slot * p.bs + t % p.bs : -1;  // no slot: no row to write
    }
    if (rid >= 0) {
      uint4* kd = reinterpret_cast<uint4*>(p.k + rid * p.k_stride);
      for (int i = tid; i < p.dqk / 8; i += blockDim.x) kd[i] = reinterpret_cast<const uint4*>(kn)[i];
      if (p.v_new != nullptr && p.v != nullptr) {
        uint4* vd = reinterpret_cast<uint4*>(p.v + rid * p.v_stride);
        const uint4* vs = reinterpret_cast<const uint4*>(p.v_new + row * p.dv);
        for (int i = tid; i < p.dv / 8; i += blockDim.x) vd[i] = vs[i];
      }
    }
    // the block's max / min take the new key in (exact: max/min picks an input)
    uint16_t* mrow = p.meta + (row * p.nb + j) * (int64_t)(2 * p.dqk);
    for (int c = tid; c < p.dqk; c += blockDim.x) {
      const uint16_t x = kn[c];
      if (first) {
        mrow[c] = x;
        mrow[p.dqk + c] = x;
      } else {
        const float xf = __uint_as_float((uint32_t)x << 16);
        const float hi = fmaxf(__uint_as_float((uint32_t)mrow[c] << 16), xf);
        const float lo = fminf(__uint_as_float((uint32_t)mrow[p.dqk + c] << 16), xf);
        mrow[c] = (uint16_t)(__float_as_uint(hi) >> 16);
        mrow[p.dqk + c] = (uint16_t)(__float_as_uint(lo) >> 16);
      }
    }
    if (tid < R) lab[tid] = min(max(p.label_ch[h * R + tid], 0), p.dqk - 1);
    __syncthreads();
    if (tid == 0) quant_token<R>(kn, lab, p.codes + (row * p.ctx_len + t) * (R / 2), p.scales + row * p.ctx_len + t);
    __syncthreads();  // lab is rewritten for the next head
  }
  if (tid == 0) seq_lens[b] = t + 1;
}

}  // namespace tls

using namespace tls;

extern "C" tls_status tls_build_block_meta(const tls_shape* shape, const void* k, int64_t k_row_stride,
                                           int64_t t0, int64_t t1, void* meta, void* stream) {
  NvtxRange nvtx_range("tls_build_block_meta");
  clear_error();
  tls_status st = check_shape(shape);
  if (st != TLS_OK) return st;
  const tls_shape& s = *shape;
  if (k == nullptr || meta == nullptr) return fail(TLS_ERR_INVALID_ARG, "build_block_meta: null pointer");
  if (!aligned16(k)) return fail(TLS_ERR_INVALID_ARG, "build_block_meta: k must be 16-byte aligned");
  if (k_row_stride < s.qk_dim || k_row_stride % 8 != 0)
    return fail(TLS_ERR_INVALID_ARG, "build_block_meta: k_row_stride %lld must be >= qk_dim and a multiple of 8",
                (long long)k_row_stride);
  if (t0 < 0 || t1 > s.ctx_len || t0 >= t1 || t0 % s.block_size)
    return fail(TLS_ERR_INVALID_ARG, "build_block_meta: range [%lld, %lld) must start on a block inside [0, N)",
                (long long)t0, (long long)t1);
  const int vpr = s.qk_dim / 8;
  const int rp = vpr >= 256 ? 1 : 256 / vpr;
  const int threads = rp * vpr;
  const size_t smem = (size_t)2 * rp * s.qk_dim * sizeof(float);
  dim3 grid((unsigned)((t1 - t0 + s.block_size - 1) / s.block_size), (unsigned)rows_of(s));
  build_block_meta_kernel<<<grid, threads, smem, (cudaStream_t)stream>>>(
      (const uint16_t*)k, k_row_stride, s.qk_dim, s.block_size, s.ctx_len, n_blocks(s), t0 / s.block_size, t1,
      s.seq_lens, s.n_kv_heads, (uint16_t*)meta);
  return launch_check("build_block_meta launch");
}

extern "C" tls_status tls_quant_label_cache(const tls_shape* shape, const void* k, int64_t k_row_stride,
                                            const int32_t* label_ch, int64_t t0, int64_t t1, uint8_t* codes,
                                            float* scales, void* stream) {
  NvtxRange nvtx_range("tls_quant_label_cache");
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
                                                 t0, t1, s.seq_lens, codes, scales);                 \
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

extern "C" tls_status tls_append_kv(const tls_shape* shape, int32_t* seq_lens, const void* k_new, const void* v_new,
                                    const tls_kv_view* kv, void* meta, const int32_t* label_ch, uint8_t* codes,
                                    float* scales, void* stream) {
  NvtxRange nvtx_range("tls_append_kv");
  clear_error();
  tls_status st = check_shape(shape);
  if (st != TLS_OK) return st;
  const tls_shape& s = *shape;
  if (seq_lens == nullptr || k_new == nullptr || kv == nullptr || kv->k == nullptr || meta == nullptr ||
      label_ch == nullptr || codes == nullptr || scales == nullptr)
    return fail(TLS_ERR_INVALID_ARG, "append_kv: null pointer");
  const bool own_v = s.v_offset < 0;
  if (own_v && (v_new == nullptr || kv->v == nullptr))
    return fail(TLS_ERR_INVALID_ARG, "append_kv: v_new and kv.v are needed when V is its own tensor");
  if (!aligned16(k_new) || !aligned16(kv->k) || (own_v && (!aligned16(v_new) || !aligned16(kv->v))))
    return fail(TLS_ERR_INVALID_ARG, "append_kv: k_new / v_new / kv.k / kv.v must be 16-byte aligned");
  if (kv->k_row_stride < s.qk_dim || kv->k_row_stride % 8 != 0 ||
      (own_v && (kv->v_row_stride < s.v_dim || kv->v_row_stride % 8 != 0)))
    return fail(TLS_ERR_INVALID_ARG, "append_kv: bad row strides");
  if (kv->slot_of_block != nullptr && kv->n_slots < 1)
    return fail(TLS_ERR_INVALID_ARG, "append_kv: n_slots must be >= 1 with a slot table");
  AppendParams p;
  p.k_new = (const uint16_t*)k_new;
  p.v_new = own_v ? (const uint16_t*)v_new : nullptr;
  p.k = (uint16_t*)const_cast<void*>(kv->k);
  p.v = own_v ? (uint16_t*)const_cast<void*>(kv->v) : nullptr;
  p.k_stride = kv->k_row_stride;
  p.v_stride = kv->v_row_stride;
  p.slot_of_block = kv->slot_of_block;
  p.n_slots = kv->n_slots;
  p.meta = (uint16_t*)meta;
  p.label_ch = label_ch;
  p.codes = codes;
  p.scales = scales;
  p.n_kv_heads = s.n_kv_heads;
  p.dqk = s.qk_dim;
  p.dv = s.v_dim;
  p.bs = s.block_size;
  p.nb = (int)n_blocks(s);
  p.ctx_len = s.ctx_len;
  cudaStream_t cs = (cudaStream_t)stream;
  switch (s.n_label) {
#define TLS_AP_CASE(RR)                                                    \
  case RR:                                                                 \
    append_kv_kernel<RR><<<s.batch, 128, 0, cs>>>(seq_lens, p);            \
    break;
    TLS_AP_CASE(2)
    TLS_AP_CASE(4)
    TLS_AP_CASE(8)
    TLS_AP_CASE(16)
    TLS_AP_CASE(32)
    TLS_AP_CASE(64)
#undef TLS_AP_CASE
    default:
      return fail(TLS_ERR_UNSUPPORTED, "append_kv: n_label %d not built (2,4,8,16,32,64)", s.n_label);
  }
  return launch_check("append_kv launch");
}
