// Level 1 of the two-level selection (AsyncTLS, English summary 2.A Stage 1:
// the Quest block score recast as a GEMM so the heads sharing a KV head use
// the tensor cores, then the top-K_b blocks; Italian summary 2.A.1: the block
// index is the max/min of the keys).
//
// Per row (batch, KV head) the scores form one GEMM
//     S[j, h] = sum_k  meta[j, k] * Q'[h, k],   Q' = [relu(q_h), min(q_h, 0)]
// with meta[j] = [kmax_j ; kmin_j] (K = 2*Dqk).  The blocks are the MMA's M
// dimension (128 per CTA) and the G heads its N dimension (padded to a
// multiple of 16), so even G = 4 fills an M = 128 tcgen05 tile.
//
// CTA roles (128 threads):
//   warp 0 lane 0   TMA producer: 128 x 64 bf16 metadata tiles, 128B swizzle
//   warp 1 lane 0   MMA issuer: tcgen05.mma kind::f16, fp32 accumulator in TMEM
//   warps 2-3       build the Q' tile of each stage in the same swizzled layout
//                   (for 64 padded heads or more a prep kernel writes Q' once
//                   per step and warp 0 loads it by TMA as well)
//   all warps       epilogue: tcgen05.ld one accumulator row per thread,
//                   max over the G real heads -> agg[row, j]
// The deterministic top-K_b over the row's NB scores: a row of one tile is
// selected by its CTA; the 2, 4 or 8 CTAs of a longer row form a cluster and
// push their keys into the leader's shared memory, which selects; longer
// rows go through the workspace, and the last CTA of the row to finish
// (atomic ticket) selects from the scores read back from L2.
//
// Every mbarrier wait is bounded (2 s); on expiry the workspace error word
// is set and the CTA skips the rest of its work, frees its TMEM and returns.

#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include <cooperative_groups.h>

#include "cluster_topk.cuh"
#include "device_common.cuh"
#include "host_common.h"

namespace tls {

constexpr int kBsTile = 128;     // blocks per CTA (MMA M)
constexpr int kBsChunk = 64;     // K elements per pipeline stage (128 B of bf16)
constexpr int kBsStages = 4;
constexpr uint64_t kWaitNs = 2000000000ull;

struct BlockScoreParams {
  const uint16_t* q;
  int n_q_heads, n_kv_heads, group, dqk;
  int nb, K_b;
  float* agg;          // workspace [rows, nb]
  float* block_score;  // optional copy of agg
  unsigned* counters;  // workspace [rows]
  int32_t* block_idx;  // [rows, K_b]
  int* err;            // workspace error word
  const int32_t* seq_lens;  // optional [B]: tokens per sequence (blocks past them do not compete)
  int64_t ctx_len;
  int bs;
};

template <int NPAD>
struct BsSmem {
  static constexpr int A_BYTES = kBsTile * 128;
  static constexpr int B_BYTES = NPAD * 128;
  static constexpr int STAGE_BYTES = kBsStages * (A_BYTES + B_BYTES);
};

// Shared-memory bytes the body of a block-score CTA needs: the pipeline
// stages, which the selection reuses once the MMAs are done (this CTA's
// keys, the row's keys for a one-CTA selection, the selection scratch).
template <int CL>
__host__ __device__ inline int bs_body_bytes(int stage_bytes, int nb) {
  const int sel = (kBsTile + nb) * 4 + (int)sizeof(TopkScratch);
  return stage_bytes > sel ? stage_bytes : sel;
}

// CL: how the row's top-K_b is taken.  1: the row is one tile, its CTA
// selects; 2, 4, 8: the row's CTAs form a cluster, push their keys into the
// leader's shared memory, and the leader selects (cta_topk_regs); 0: the last
// CTA of the row (a ticket) selects from the scores in the workspace.
// Q' = [relu(q_h), min(q_h, 0)] of every row, bf16 [rows * npad][2 * Dqk]
// (rows h >= G zero): the level-1 B operand, written once per step for wide
// groups so that each level-1 CTA loads it by TMA instead of rebuilding it.
// One CTA per (row, padded head): eight bf16 per thread, one 16-byte load and
// two 16-byte stores (Dqk is a multiple of 32).
__global__ void __launch_bounds__(128) block_query_prep_kernel(const uint16_t* q, int n_q_heads, int n_kv_heads,
                                                                int g, int dqk, int npad, uint16_t* qp) {
  const int row = blockIdx.x, h = blockIdx.y, b = row / n_kv_heads, kvh = row % n_kv_heads;
  const uint4* src = reinterpret_cast<const uint4*>(q + ((int64_t)b * n_q_heads + (int64_t)kvh * g + h) * dqk);
  uint4* out = reinterpret_cast<uint4*>(qp + ((int64_t)row * npad + h) * 2 * dqk);
  const int n8 = dqk / 8;
  for (int i = threadIdx.x; i < n8; i += blockDim.x) {
    const uint4 x = h < g ? src[i] : make_uint4(0u, 0u, 0u, 0u);
    out[i] = make_uint4(relu_bf16x2(x.x), relu_bf16x2(x.y), relu_bf16x2(x.z), relu_bf16x2(x.w));
    out[n8 + i] = make_uint4(min0_bf16x2(x.x), min0_bf16x2(x.y), min0_bf16x2(x.z), min0_bf16x2(x.w));
  }
}

// QT: the B operand (Q') comes from global memory by TMA (wide groups)
// instead of being built by warps 2-3 in every CTA.
template <int NPAD, int CL>
__global__ void __launch_bounds__(128, 1)
    block_score_tc_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap qmap,
                          BlockScoreParams p) {
  constexpr bool QT = NPAD >= 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  using L = BsSmem<NPAD>;
  const int body = bs_body_bytes<CL>(L::STAGE_BYTES, p.nb);
  uint8_t* sA = smem;
  uint8_t* sB = smem + kBsStages * L::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + ((body + 7) & ~7));
  uint64_t* empty = full + kBsStages;
  uint64_t* done = empty + kBsStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* flags = reinterpret_cast<volatile int*>(tmem_slot + 1);  // [0] last CTA, [1] failed

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row = blockIdx.y, mt = blockIdx.x;
  const int nk = (2 * p.dqk) / kBsChunk;
  // blocks of this row's sequence: only they compete (a suffix of the row)
  const int nbr = (int)((seq_len_of(p.seq_lens, row / p.n_kv_heads, p.ctx_len) + p.bs - 1) / p.bs);
  const int kk = min(p.K_b, nbr);  // entries selected; the rest of the list is -1
  constexpr uint32_t kCols = NPAD < 32 ? 32u : (uint32_t)NPAD;
  if constexpr (CL >= 2) cluster_arrive_relaxed();  // completes once every CTA of the cluster has started
  grid_launch_dependents();  // level 2 may be scheduled now; it waits for this grid before reading

  if (tid == 0) {
    for (int s = 0; s < kBsStages; ++s) {
      mbar_init(&full[s], QT ? 1 : 1 + 64);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    flags[0] = 0;
    flags[1] = 0;
    fence_barrier_init();
  } else if (tid == 32) {
    // what the epilogue and the row's top-K_b write: prefetching them now
    // also warms their address translations during the metadata loads
    prefetch_l2(p.agg + (int64_t)row * p.nb + mt * kBsTile);
    prefetch_l2(p.counters + row);
    prefetch_l2(p.block_idx + (int64_t)row * p.K_b);
  }
  if (warp == 0) tmem_alloc(tmem_slot, kCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      for (int kc = 0; kc < nk; ++kc) {
        const int s = kc % kBsStages, r = kc / kBsStages;
        if (r > 0 && !mbar_wait_bounded(&empty[s], (r - 1) & 1, kWaitNs)) {
          report_error(p.err, kErrTimeout, 101);
          flags[1] = 1;
          break;
        }
        mbar_arrive_expect_tx(&full[s], L::A_BYTES + (QT ? L::B_BYTES : 0));
        tma_load_2d(sA + s * L::A_BYTES, &tmap, &full[s], kc * kBsChunk, row * p.nb + mt * kBsTile);
        if constexpr (QT) tma_load_2d(sB + s * L::B_BYTES, &qmap, &full[s], kc * kBsChunk, row * NPAD);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBsTile, NPAD);
      bool ok = true;
      for (int kc = 0; kc < nk; ++kc) {
        const int s = kc % kBsStages, r = kc / kBsStages;
        if (!mbar_wait_bounded(&full[s], r & 1, kWaitNs)) {
          report_error(p.err, kErrTimeout, 102);
          flags[1] = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + s * L::A_BYTES);
        const uint32_t b0 = smem_u32(sB + s * L::B_BYTES);
#pragma unroll
        for (int k16 = 0; k16 < kBsChunk / 16; ++k16)
          tc_mma_bf16(tmem, sw128_kmajor_desc(a0 + k16 * 32), sw128_kmajor_desc(b0 + k16 * 32), idesc,
                      (kc | k16) != 0);
        tc_commit(&empty[s]);
      }
      if (ok) tc_commit(done);
    }
  } else if (!QT) {
    // Q' producers: row h of a stage holds Q'[h, kc*64 .. kc*64+63] as eight
    // 16-byte chunks, chunk c stored at position c ^ (h % 8) (128B swizzle).
    const int t = tid - 64;
    const int g = p.group;
    const int b = row / p.n_kv_heads, kvh = row % p.n_kv_heads;
    const uint16_t* qg = p.q + ((int64_t)b * p.n_q_heads + (int64_t)kvh * g) * p.dqk;
    for (int kc = 0; kc < nk; ++kc) {
      const int s = kc % kBsStages, r = kc / kBsStages;
      if (r > 0 && !mbar_wait_bounded(&empty[s], (r - 1) & 1, kWaitNs)) {
        report_error(p.err, kErrTimeout, 103);
        flags[1] = 1;
        break;
      }
      uint8_t* dst = sB + s * L::B_BYTES;
      for (int v = t; v < NPAD * 8; v += 64) {
        const int h = v >> 3, c = v & 7;
        const int e0 = kc * kBsChunk + c * 8;
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if (h < g) {
          const bool lo_half = e0 < p.dqk;
          const uint4 x = *reinterpret_cast<const uint4*>(qg + (int64_t)h * p.dqk + (lo_half ? e0 : e0 - p.dqk));
          if (lo_half) w = make_uint4(relu_bf16x2(x.x), relu_bf16x2(x.y), relu_bf16x2(x.z), relu_bf16x2(x.w));
          else w = make_uint4(min0_bf16x2(x.x), min0_bf16x2(x.y), min0_bf16x2(x.z), min0_bf16x2(x.w));
        }
        *reinterpret_cast<uint4*>(dst + h * 128 + ((c ^ (h & 7)) << 4)) = w;
      }
      fence_proxy_async_smem();
      mbar_arrive(&full[s]);
    }
  }
  __syncwarp();

  // Epilogue: thread (warp w, lane l) owns accumulator row m = 32w + l.
  bool ok = mbar_wait_bounded(done, 0, kWaitNs) && flags[1] == 0;
  ok = __all_sync(0xffffffffu, ok);
  tc_fence_after();
  float best = -INFINITY;
  if (ok) {
    const int j = mt * kBsTile + warp * 32 + lane;
#pragma unroll
    for (int c0 = 0; c0 < NPAD; c0 += 16) {
      float v[16];
      tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (c0 + i < p.group) best = fmaxf(best, v[i]);
    }
    if (j < p.nb) {
      if (CL == 0) p.agg[(int64_t)row * p.nb + j] = best;
      if (p.block_score != nullptr) p.block_score[(int64_t)row * p.nb + j] = j < nbr ? best : -INFINITY;
    }
  } else if (lane == 0) {
    report_error(p.err, kErrTimeout, 104);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }

  int32_t* out = p.block_idx + (int64_t)row * p.K_b;
  if constexpr (CL == 0) {
    // Last CTA of this row selects the top-K_b blocks.
    __threadfence();
    __syncthreads();
    if (tid == 0) {
      unsigned prev = atomicInc(&p.counters[row], gridDim.x - 1);
      flags[0] = (prev == gridDim.x - 1) ? 1 : 0;
    }
    __syncthreads();
    if (flags[0] == 0) return;
    __threadfence();
    uint32_t* keys = reinterpret_cast<uint32_t*>(smem);
    TopkScratch* ts = reinterpret_cast<TopkScratch*>(keys + p.nb);
    const float* arow = p.agg + (int64_t)row * p.nb;
    for (int i = tid; i < nbr; i += 128) keys[i] = float_key(__ldcg(arow + i));
    pad_list(out, kk, p.K_b);
    __syncthreads();
    if (kk == 0) return;
    if (nbr <= 128 * 16) cta_topk_regs<128, 16>(keys, nbr, kk, out, *ts, [](int i) { return i; });
    else cta_topk_ascending<128>(keys, nbr, kk, out, *ts, [](int i) { return i; });
  } else {
    // the drained stages hold the selection: this CTA's keys, then the row's
    uint32_t* mine = reinterpret_cast<uint32_t*>(smem);  // [kBsTile]
    uint32_t* all = mine + kBsTile;                       // [nb]
    TopkScratch* ts = reinterpret_cast<TopkScratch*>(all + p.nb);
    const int n_loc = max(0, min(kBsTile, nbr - mt * kBsTile));  // this CTA's competing blocks
    if (tid < n_loc) mine[tid] = float_key(best);
    if (mt == 0) pad_list(out, kk, p.K_b);
    __syncthreads();
    if constexpr (CL == 1) {
      if (kk > 0) cta_topk_ascending<128>(mine, n_loc, kk, out, *ts, [](int i) { return i; });
    } else {
      // every CTA pushes its keys into the leader's row array; after one
      // cluster barrier the leader selects alone with the keys in registers
      namespace cg = cooperative_groups;
      cg::cluster_group cluster = cg::this_cluster();
      cluster_wait();
      uint32_t* dst = cluster.map_shared_rank(all, 0) + mt * kBsTile;
      if (tid < n_loc) dst[tid] = mine[tid];
      cluster.sync();  // the leader's keys are complete; no remote access after this
      if (mt != 0 || kk == 0) return;
      cta_topk_regs<128, CL>(all, nbr, kk, out, *ts, [](int i) { return i; });
    }
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

tls_status get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (g_encode == nullptr) return fail(TLS_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  return TLS_OK;
}

template <int NPAD, int CL>
tls_status launch_tc(const CUtensorMap& tmap, const CUtensorMap& qmap, const BlockScoreParams& p, int rows,
                     cudaStream_t stream) {
  using L = BsSmem<NPAD>;
  const int body = bs_body_bytes<CL>(L::STAGE_BYTES, p.nb);
  const size_t smem = 1024 + (size_t)((body + 7) & ~7) + (2 * kBsStages + 1) * 8 + 16;
  cudaError_t e = kernel_attrs((const void*)block_score_tc_kernel<NPAD, CL>, smem);
  if (e != cudaSuccess) return cuda_check(e, "select_blocks: set smem attribute");
  const dim3 grid((unsigned)((p.nb + kBsTile - 1) / kBsTile), (unsigned)rows);
  if constexpr (CL >= 2)
    return cuda_check(launch_cluster(block_score_tc_kernel<NPAD, CL>, grid, dim3(128), smem, stream, (unsigned)CL,
                                     tmap, qmap, p),
                      "select_blocks: block_score_tc launch");
  block_score_tc_kernel<NPAD, CL><<<grid, 128, smem, stream>>>(tmap, qmap, p);
  return launch_check("select_blocks: block_score_tc launch");
}

template <int CL>
tls_status launch_tc_group(const CUtensorMap& tmap, const CUtensorMap& qmap, const BlockScoreParams& p, int rows,
                           cudaStream_t stream) {
  const int g = p.group;
  if (g <= 16) return launch_tc<16, CL>(tmap, qmap, p, rows, stream);
  if (g <= 32) return launch_tc<32, CL>(tmap, qmap, p, rows, stream);
  if (g <= 64) return launch_tc<64, CL>(tmap, qmap, p, rows, stream);
  if (g <= 128) return launch_tc<128, CL>(tmap, qmap, p, rows, stream);
  if (g <= 256) return launch_tc<256, CL>(tmap, qmap, p, rows, stream);
  return fail(TLS_ERR_UNSUPPORTED, "select_blocks: group size %d > 256", g);
}

}  // namespace

// Level 1: block scores and the top-K_b of every row.
tls_status select_blocks_impl(const tls_shape& s, const void* q, const void* meta, int K_b, int32_t* block_idx,
                              float* block_score, uint8_t* ws, const WsLayout& L, cudaStream_t stream) {
  const int rows = rows_of(s);
  const int nb = (int)n_blocks(s);
  BlockScoreParams p;
  p.q = (const uint16_t*)q;
  p.n_q_heads = s.n_q_heads;
  p.n_kv_heads = s.n_kv_heads;
  p.group = group_of(s);
  p.dqk = s.qk_dim;
  p.nb = nb;
  p.K_b = K_b;
  p.agg = reinterpret_cast<float*>(ws + L.agg);
  p.block_score = block_score;
  p.counters = reinterpret_cast<unsigned*>(ws + L.blk_counter);
  p.block_idx = block_idx;
  p.err = reinterpret_cast<int*>(ws + L.err);
  p.seq_lens = s.seq_lens;
  p.ctx_len = s.ctx_len;
  p.bs = s.block_size;

  tls_status st = get_encoder();
  if (st != TLS_OK) return st;
  CUtensorMap tmap;
  const cuuint64_t dims[2] = {(cuuint64_t)(2 * s.qk_dim), (cuuint64_t)rows * (cuuint64_t)nb};
  const cuuint64_t strides[1] = {(cuuint64_t)(2 * s.qk_dim) * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kBsChunk, (cuuint32_t)kBsTile};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(meta), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TLS_ERR_CUDA, "select_blocks: cuTensorMapEncodeTiled failed (%d)", (int)r);
  // wide groups: Q' written once per step, loaded by TMA in every CTA
  CUtensorMap qmap = tmap;  // unused below 64 padded heads
  const int npad = block_score_npad(p.group);
  if (npad >= 64) {
    uint16_t* qp = reinterpret_cast<uint16_t*>(ws + L.qprime);
    block_query_prep_kernel<<<dim3(rows, npad), 128, 0, stream>>>((const uint16_t*)q, s.n_q_heads, s.n_kv_heads,
                                                                   p.group, s.qk_dim, npad, qp);
    tls_status lst = launch_check("select_blocks: query prep launch");
    if (lst != TLS_OK) return lst;
    const cuuint64_t qdims[2] = {(cuuint64_t)(2 * s.qk_dim), (cuuint64_t)rows * (cuuint64_t)npad};
    const cuuint64_t qstrides[1] = {(cuuint64_t)(2 * s.qk_dim) * 2};
    const cuuint32_t qbox[2] = {(cuuint32_t)kBsChunk, (cuuint32_t)npad};
    r = g_encode(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, qp, qdims, qstrides, qbox, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(TLS_ERR_CUDA, "select_blocks: cuTensorMapEncodeTiled (Q') failed (%d)", (int)r);
  }

  // the row's tiles select together when they fit one cluster
  const int tiles = (nb + kBsTile - 1) / kBsTile;
  if (tiles == 1) return launch_tc_group<1>(tmap, qmap, p, rows, stream);
  if (tiles == 2) return launch_tc_group<2>(tmap, qmap, p, rows, stream);
  if (tiles == 4) return launch_tc_group<4>(tmap, qmap, p, rows, stream);
  if (tiles == 8) return launch_tc_group<8>(tmap, qmap, p, rows, stream);
  return launch_tc_group<0>(tmap, qmap, p, rows, stream);
}

}  // namespace tls
