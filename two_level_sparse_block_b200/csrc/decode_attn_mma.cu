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
//   O += P . V     in fp16: A = P from the S accumulators rounded to fp16
//                  (relative error <= 2^-11), B = V rows via ldmatrix.trans,
//                  their bf16 pairs converted to fp16 exactly
// At the end of each (row) segment of its range the CTA folds its warps in
// shared memory and writes (m, l, O) to the split workspace; the last CTA to
// finish a row merges the splits by log-sum-exp (attn_common.cuh).

#include <cooperative_groups.h>

#include "attn_common.cuh"
#include "device_common.cuh"
#include "host_common.h"
#include "mma_attn.cuh"

namespace tls {

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
