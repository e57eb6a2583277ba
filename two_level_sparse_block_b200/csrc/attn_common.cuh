// Parameters and the split merge shared by the attention kernels.
#pragma once

#include "device_common.cuh"
#include "host_common.h"

namespace tls {

struct AttnParams {
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  int64_t k_stride, v_stride;
  const int32_t* slot_of_block;
  int bs, nb, n_slots;
  int64_t ctx_len;
  const int32_t* token_idx;
  int k_sel;
  int n_q_heads, n_kv_heads, group, dqk, dv;
  float scale_log2;
  int tokens_per_split, splits, head_groups, heads_per_cta;
  int tiles_per_pair, n_items, n_ctas;  // mma attention: chunks per (virtual) row, items, persistent CTAs
  int* err;            // workspace error word
  float* partial;      // workspace [rows][G][splits][dv + 2]
  unsigned* counters;  // workspace [rows * head_groups]
  void* out;
  int out_bf16;
  float* lse;
  const int32_t* seq_lens;  // optional [B]: tokens per sequence (later positions are skipped)
  int list_mode;            // kListTokens, kListAll or kListBlocks
  const int32_t* blocks;    // kListBlocks: [rows, K_b] block list
  int K_b;
};

// Token of entry t (< k_sel) of row `row`'s list, or -1 when the entry is no
// token of the sequence (padding of a selection, a position >= len).  List
// reads go through L2: the list may be written by the preceding kernel while
// this grid is already resident (programmatic dependent launch).
__device__ __forceinline__ int attn_token(const AttnParams& p, int row, int t, int64_t len) {
  int64_t tok;
  if (p.list_mode == kListAll) {
    tok = t;
  } else if (p.list_mode == kListBlocks) {
    const int blk = __ldcg(p.blocks + (int64_t)row * p.K_b + t / p.bs);
    tok = blk < 0 ? -1 : (int64_t)blk * p.bs + t % p.bs;
  } else {
    tok = __ldcg(p.token_idx + (int64_t)row * p.k_sel + t);
  }
  return (tok >= 0 && tok < len) ? (int)tok : -1;
}

// Row id (index of the K/V row) of token `tok` of row `row` (tok >= 0): the
// dense layout, or its block's slot in the pool (clamped into the pool).
__device__ __forceinline__ int64_t attn_row_id(const AttnParams& p, int row, int64_t tok) {
  if (p.slot_of_block != nullptr) {
    const int64_t slot = min(max(__ldg(p.slot_of_block + (int64_t)row * p.nb + tok / p.bs), 0), p.n_slots - 1);
    return slot * p.bs + tok % p.bs;
  }
  return (int64_t)row * p.ctx_len + tok;
}

// Owner of work item `item` when CTA c takes items [c*W/n, (c+1)*W/n).
__host__ __device__ inline int64_t attn_owner(int64_t item, int64_t n_items, int64_t n_ctas) {
  return ((item + 1) * n_ctas + n_items - 1) / n_items - 1;
}

// Last CTA of a (row, head group): log-sum-exp merge of the splits of heads
// h0 .. h0+nh-1, then the normalised output and the natural-log lse.
// Partials are [row][head][split][m, l, acc[0..dv)] with m in log2 units;
// only the first n_splits of the p.splits slots of each head are read.
// All threads of the CTA must call it (it synchronises).  Every load is
// issued in a batch with the others it does not depend on: (m, l) of all
// splits in one round into `scratch` (shared memory the caller no longer
// needs, >= 2 * kMergeStride floats per head), then per output the
// accumulators of 8 splits at a time.
constexpr int kMergeMaxSplits = 64;
constexpr int kMergeStride = kMergeMaxSplits + 1;

static __device__ __noinline__ void merge_splits(const AttnParams& p, int row, int b, int kvh, int h0, int nh,
                                                 int n_splits, float* scratch, int scratch_floats) {
  const int g = p.group, dv = p.dv;
  const int tid = threadIdx.x, nt = blockDim.x;
  const int64_t sstride = dv + 2;
  const int per = max(1, scratch_floats / (2 * kMergeStride));  // heads per pass
  float* wm = scratch;                        // [per][kMergeStride]: m, then the weight; [.][64] = lse
  float* wl = scratch + per * kMergeStride;   // [per][kMergeStride]: l
  for (int base = 0; base < nh; base += per) {
    const int hn = min(per, nh - base);
    for (int i = tid; i < hn * n_splits; i += nt) {
      const int hh = i / n_splits, s = i % n_splits;
      const float* pp = p.partial + (((int64_t)row * g + h0 + base + hh) * p.splits + s) * sstride;
      const float m = __ldcg(pp), l = __ldcg(pp + 1);
      wm[hh * kMergeStride + s] = m;
      wl[hh * kMergeStride + s] = l;
    }
    __syncthreads();
    for (int hh = tid; hh < hn; hh += nt) {
      float* m = wm + hh * kMergeStride;
      const float* l = wl + hh * kMergeStride;
      float M = -INFINITY;
      for (int s = 0; s < n_splits; ++s) M = fmaxf(M, m[s]);
      float L = 0.0f;
      for (int s = 0; s < n_splits; ++s) {
        const float f = m[s] == -INFINITY ? 0.0f : exp2f(m[s] - M);
        L += f * l[s];
        m[s] = f;
      }
      const float inv = L > 0.0f ? 1.0f / L : 0.0f;  // a row with no token: zero output
      for (int s = 0; s < n_splits; ++s) m[s] *= inv;
      m[kMergeMaxSplits] = (M + log2f(L)) * 0.69314718055994531f;
    }
    __syncthreads();
    const float* __restrict__ part = p.partial;
    for (int idx0 = tid; idx0 < hn * dv; idx0 += 4 * nt) {
      // four outputs per thread at a time, eight splits each: 32 loads in flight
      float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      for (int s0 = 0; s0 < n_splits; s0 += 8) {
        float v[4][8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int idx = idx0 + j * nt;
          const int hh = idx / dv, e = idx % dv;
          const float* pp = part + ((int64_t)row * g + h0 + base + hh) * p.splits * sstride + 2 + e;
#pragma unroll
          for (int u = 0; u < 8; ++u)
            v[j][u] = (idx < hn * dv && s0 + u < n_splits) ? __ldcg(pp + (s0 + u) * sstride) : 0.0f;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int idx = idx0 + j * nt;
          const int hh = min(idx / dv, hn - 1);
#pragma unroll
          for (int u = 0; u < 8; ++u)
            if (s0 + u < n_splits) acc[j] = fmaf(wm[hh * kMergeStride + s0 + u], v[j][u], acc[j]);
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int idx = idx0 + j * nt;
        if (idx >= hn * dv) break;
        const int hh = idx / dv, e = idx % dv;
        const int64_t oh = (int64_t)b * p.n_q_heads + kvh * g + h0 + base + hh;
        if (p.out_bf16) reinterpret_cast<uint16_t*>(p.out)[oh * dv + e] = f32_to_bf16_rn(acc[j]);
        else reinterpret_cast<float*>(p.out)[oh * dv + e] = acc[j];
        if (e == 0 && p.lse != nullptr) p.lse[oh] = wm[hh * kMergeStride + kMergeMaxSplits];
      }
    }
    __syncthreads();
  }
}

// Warp-streaming attention for groups of <= 16 heads (decode_attn_mma.cu).
bool attn_mma_supported(const tls_shape& s);
tls_status launch_attn_mma(const AttnParams& p, int rows, cudaStream_t stream, bool pdl);
// MLA latent attention (decode_attn_mla.cu): Dqk 576, Dv 512 = the row's first 512, G % 16 == 0.
bool attn_mla_supported(const tls_shape& s);
int attn_mla_tokens_per_split(int k);
tls_status launch_attn_mla(const AttnParams& p, int rows, cudaStream_t stream, bool pdl);
int attn_mma_cluster_size(int rows, int hpc);

}  // namespace tls
