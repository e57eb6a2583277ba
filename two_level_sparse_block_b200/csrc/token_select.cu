// Level 2 of the two-level selection (AsyncTLS, English summary 2.A Stage 2:
// Double-Sparsity token selection inside the chosen blocks, from selected
// key channels quantised to INT4, then the top-K_t tokens).
//
// Candidates of a row are the bs tokens of each of its K_b chosen blocks, in
// ascending token order, scored as
//     score(t) = s_t * max_h sum_r qlab[h, r] * code_{t, r}
// (s_t >= 0, so scaling after the max is the same as taking the max of the
// scaled dots), then the deterministic top-k.  Three kernels, chosen by
// token_dispatch:
//   token_select_row_kernel      narrow groups (G <= 16, 16 or 32 label
//                                channels, <= 8192 candidates): up to 4 CTAs
//                                a row stage and score, the leader selects
//   token_select_cluster_kernel  wider groups or other channel counts: a
//                                cluster of 4 to 16 CTAs scores and selects
//                                together over distributed shared memory
//   token_select_kernel          the rest: a grid of (chunks, rows) CTAs
//                                writes the scores to the workspace and the
//                                last CTA of each row selects

#include <cooperative_groups.h>
#include <cstdlib>

#include "cluster_topk.cuh"
#include "device_common.cuh"
#include "host_common.h"
#include "token_common.cuh"

namespace tls {

template <int R, int NT>
__global__ void __launch_bounds__(NT) token_select_kernel(TokenParams p) {
  extern __shared__ float sm[];
  float* qlab = sm;                                                 // [G][R]
  int32_t* sb = reinterpret_cast<int32_t*>(sm + p.group * R);       // [K_b]
  uint32_t* keys = reinterpret_cast<uint32_t*>(sb + p.K_b);         // [n_cand] (last CTA)
  TopkScratch* ts = reinterpret_cast<TopkScratch*>(
      (reinterpret_cast<uintptr_t>(keys + p.n_cand) + 15) & ~uintptr_t(15));
  __shared__ int last;
  const int tid = threadIdx.x;
  const int row = blockIdx.y;
  load_qlab<R, NT>(p, row, qlab);
  const int nvb = load_block_list<NT>(p, row, sb);  // ends with a CTA barrier
  const int n_valid = valid_candidates(p, row, sb, nvb);

  const int c0 = blockIdx.x * p.chunk;
  const int c1 = min(p.n_cand, c0 + p.chunk);
  float* out = p.tscore + (int64_t)row * p.n_cand;
  const int g = p.group;
  for (int i = c0 + tid; i < c1; i += NT) {
    const int64_t tok = (int64_t)sb[i / p.bs] * p.bs + (i % p.bs);
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
    if (p.token_score != nullptr) p.token_score[(int64_t)row * p.n_cand + i] = i < n_valid ? score : -INFINITY;
  }

  __threadfence();
  __syncthreads();
  if (tid == 0) last = atomicInc(&p.counters[row], gridDim.x - 1) == gridDim.x - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  for (int i = tid; i < n_valid; i += NT) keys[i] = float_key(__ldcg(out + i));
  const int kk = min(p.k, n_valid);
  int32_t* dst = p.token_idx + (int64_t)row * p.k;
  pad_list(dst, kk, p.k);
  __syncthreads();
  if (kk == 0) return;
  cta_topk_ascending<NT>(keys, n_valid, kk, dst, *ts, CandidateToken{sb, p.bs});
}

// A cluster of CTAs per row when scoring is light: every CTA scores a
// contiguous share of the candidates into its own shared memory and the
// cluster selects the top-k together over distributed shared memory
// (cluster_topk.cuh).  When the scores are degenerate (a wide run of equal
// keys at the threshold), the leader CTA gathers all keys and selects alone.
constexpr int kTokThreads = 256;

// NTILE > 0: scores on the tensor cores (score_candidates_tc, heads in
// NTILE n-tiles of 8); 0: on the CUDA cores.  CL CTAs (the launch's cluster
// size) share a row: 4 when there are enough rows to fill the GPU, up to 16
// when a few long rows would leave it idle.
// BIG: the row has too many candidates for one CTA's shared memory to hold
// all their keys; the degenerate fallback then gathers them in the workspace
// (tscore, as keys) instead of the leader's shared memory.
template <int R, int NTILE, int CL, bool BIG>
__global__ void __launch_bounds__(kTokThreads) token_select_cluster_kernel(TokenParams p) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ float sm[];
  const int rank = (int)cluster.block_rank();
  const int row = blockIdx.y;
  const int per = (p.n_cand + CL - 1) / CL;
  float* qlab = sm;                                                   // [G][R]
  int32_t* bidx = reinterpret_cast<int32_t*>(sm + p.group * R);       // [K_b]
  uint32_t* mine = reinterpret_cast<uint32_t*>(bidx + p.K_b);         // [per]
  uint32_t* all = mine + per;                                         // [n_cand] (leader, fallback; not BIG)
  TopkScratch* ts = reinterpret_cast<TopkScratch*>(BIG ? all : all + p.n_cand);
  ClusterTopkScratch<CL>* cts =
      reinterpret_cast<ClusterTopkScratch<CL>*>((reinterpret_cast<uintptr_t>(ts + 1) + 15) & ~uintptr_t(15));
  cluster_arrive_relaxed();  // completes once every CTA of the cluster has started
  grid_launch_dependents();
  load_qlab<R, kTokThreads>(p, row, qlab);
  if (threadIdx.x == 0) prefetch_l2(p.token_idx + (int64_t)row * p.k + (int64_t)rank * p.k / CL);
  grid_dependency_wait();  // the block lists come from the preceding kernel
  const int nvb = load_block_list<kTokThreads>(p, row, bidx);  // ends with a CTA barrier
  const int n_valid = valid_candidates(p, row, bidx, nvb);
  const int c0 = min(p.n_cand, rank * per), c1 = min(p.n_cand, c0 + per);
  if constexpr (NTILE > 0) score_candidates_tc<R, kTokThreads, NTILE>(p, row, qlab, bidx, c0, c1, mine, n_valid);
  else score_candidates<R, kTokThreads>(p, row, qlab, bidx, c0, c1, mine, n_valid);
  __syncthreads();
  cluster_wait();
  int* out = p.token_idx + (int64_t)row * p.k;
  const CandidateToken map{bidx, p.bs};
  // only the candidates that are tokens of the sequence compete (a prefix)
  const int kk = min(p.k, n_valid);
  const int n_loc = max(0, min(c1, n_valid) - c0);
  if (rank == 0) pad_list(out, kk, p.k);
  if (kk == 0) {
    cluster.sync();  // no CTA leaves while another may still read its shared memory
    return;
  }
  if (cluster_topk_ascending<kTokThreads, CL>(mine, n_loc, c0, kk, out, *cts, map)) return;
  uint32_t* keys = all;
  if constexpr (BIG) {
    // every CTA writes its keys into the row's workspace scores (as keys)
    keys = reinterpret_cast<uint32_t*>(p.tscore + (int64_t)row * p.n_cand);
    for (int i = threadIdx.x; i < n_loc; i += kTokThreads) keys[c0 + i] = mine[i];
    __threadfence();
  } else if (rank == 0) {
    // gather the other CTAs' keys through distributed shared memory, eight
    // independent loads in flight per thread
    for (int r = 0; r < CL; ++r) {
      const uint32_t* __restrict__ src = cluster.map_shared_rank(mine, r);
      const int b0 = min(n_valid, r * per), b1 = min(n_valid, b0 + per);
      for (int i0 = 0; i0 < b1 - b0; i0 += 8 * kTokThreads) {
        uint32_t v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = i0 + u * kTokThreads + (int)threadIdx.x;
          v[u] = i < b1 - b0 ? src[i] : 0u;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = i0 + u * kTokThreads + (int)threadIdx.x;
          if (i < b1 - b0) all[b0 + i] = v[u];
        }
      }
    }
  }
  cluster.sync();  // the other CTAs' shared memory (or workspace keys) may be released / read after this
  if (rank != 0) return;
  cta_topk_ascending<kTokThreads>(keys, n_valid, kk, out, *ts, map);
}

// A small cluster per row (the launch's cluster size CL, 1 to 4): each CTA
// stages the codes and scales of its share of the row's blocks in shared
// memory (16-byte copies, all in flight at once), scores them on the tensor
// cores and pushes the keys into the leader's shared memory; the leader then
// selects with the register-resident top-k (cta_topk_regs), CTA barriers
// only.  For narrow groups (G <= 16) and rows of at most 8192 candidates.
constexpr int kRowThreads = 512;  // the default CTA; 1024 when a row has one CTA of its own (`lean`)

template <int R, int NTILE, int KPT, int NT>
__global__ void __launch_bounds__(NT, NT >= 1024 || KPT > 8 ? 1 : 2) token_select_row_kernel(TokenParams p) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int cl = (int)cluster.num_blocks(), rank = (int)cluster.block_rank();
  const int row = blockIdx.y;
  const int bpc = (p.K_b + cl - 1) / cl;  // blocks per CTA
  const int j0 = min(p.K_b, rank * bpc), j1 = min(p.K_b, j0 + bpc);
  const int c0 = j0 * p.bs, c1 = j1 * p.bs;
  extern __shared__ __align__(16) uint32_t smw[];
  uint32_t* keys = smw;                                                           // [KPT * NT]
  uint8_t* scodes = reinterpret_cast<uint8_t*>(smw + KPT * NT);          // [bpc * bs][R / 2]
  float* sscales = reinterpret_cast<float*>(scodes + (size_t)bpc * p.bs * (R / 2));  // [bpc * bs]
  float* qlab = sscales + bpc * p.bs;                                             // [G][R]
  int32_t* bidx = reinterpret_cast<int32_t*>(qlab + p.group * R);                 // [K_b]
  TopkScratch* ts = reinterpret_cast<TopkScratch*>(bidx + ((p.K_b + 3) & ~3));
  int32_t* slab = reinterpret_cast<int32_t*>(ts + 1);                             // [R] label channels
  uint16_t* sq = reinterpret_cast<uint16_t*>(
      (reinterpret_cast<uintptr_t>(slab + R) + 15) & ~uintptr_t(15));             // [G][Dqk] query rows
  if (cl > 1) cluster_arrive_relaxed();  // completes once every CTA of the cluster has started
  // the query rows and the label channels (inputs of the step) are loaded
  // while the block list is: one memory round trip for the three
  stage_query_rows<NT>(p, row, sq);
  const int kvh = row % p.n_kv_heads;
  const int lab = threadIdx.x < R ? __ldg(p.label_ch + kvh * R + threadIdx.x) : 0;
  if (threadIdx.x == 0 && rank == 0) prefetch_l2(p.token_idx + (int64_t)row * p.k);
  grid_dependency_wait();  // the block lists come from the preceding kernel
  const int nvb = load_block_list<NT>(p, row, bidx, [&] {
    if (threadIdx.x < R) slab[threadIdx.x] = min(max(lab, 0), p.dqk - 1);  // clamped: never out of bounds
    cp_async_wait<0>();
  });  // ends with a CTA barrier
  for (int i = threadIdx.x; i < p.group * R; i += NT) {
    const int h = i / R, r = i - h * R;
    qlab[i] = __uint_as_float((uint32_t)sq[h * p.dqk + slab[r]] << 16);
  }
  const int n_valid = valid_candidates(p, row, bidx, nvb);
  stage_candidate_codes<R, NT>(p, row, bidx, j0, j1, scodes, sscales);
  __syncthreads();
  score_candidates_tc<R, NT, NTILE, true>(p, row, qlab, bidx, c0, c1, keys, n_valid, scodes, sscales);
  // the next grid (the attention) may become resident from here: only the
  // selection is left, and earlier it would hold SMs a concurrent level 1
  // needs
  grid_launch_dependents();
  __syncthreads();
  if (cl > 1) {
    cluster_wait();
    if (rank != 0) {
      // keys of [c0, c1) into the leader's array (bs is a multiple of 4: whole 16-byte units)
      uint4* dst = reinterpret_cast<uint4*>(cluster.map_shared_rank(keys, 0) + c0);
      const uint4* src = reinterpret_cast<const uint4*>(keys);
      for (int i = threadIdx.x; i < (c1 - c0) / 4; i += NT) dst[i] = src[i];
    }
    cluster.sync();  // the leader's keys are complete; no remote access after this
    if (rank != 0) return;
  }
  // only the candidates that are tokens of the sequence compete (a prefix)
  const int kk = min(p.k, n_valid);
  int32_t* out = p.token_idx + (int64_t)row * p.k;
  pad_list(out, kk, p.k);
  if (kk == 0) return;
  const CandidateToken map{bidx, p.bs};
  cta_topk_regs<NT, KPT>(keys, n_valid, kk, out, *ts, map);
}

// Dynamic shared memory of the row kernel with cl CTAs of nt threads a row:
// keys, staged codes and scales, qlab, the block list, the top-k scratch,
// the label channels and the group's query rows.
size_t token_row_smem(const tls_shape& s, int K_b, int cl, int nt) {
  const int n_cand = K_b * s.block_size, g = group_of(s);
  const int kpt = n_cand <= 2 * nt ? 2 : n_cand <= 4 * nt ? 4 : n_cand <= 8 * nt ? 8 : 16;
  const int bpc = (K_b + cl - 1) / cl;
  return (size_t)kpt * nt * 4 + (size_t)bpc * s.block_size * (s.n_label / 2 + 4) +
         ((size_t)g * s.n_label + ((K_b + 3) & ~3)) * 4 + sizeof(TopkScratch) + (size_t)s.n_label * 4 + 16 +
         (size_t)g * s.qk_dim * 2;
}

// Which level-2 kernel a call takes, its CTAs per row and threads per CTA
// (`lean` as in select_tokens_impl; `aligned`: q, codes and scales 16-byte
// aligned).  The one place the choice is made.
TokenDispatch token_dispatch(const tls_shape& s, int K_b, bool lean, bool aligned) {
  const int rows = rows_of(s), g = group_of(s), n_cand = K_b * s.block_size;
  if (aligned && token_row_kernel_fits(g, s.n_label, n_cand, s.block_size)) {
    const int cl = token_row_cluster_size(rows, K_b, lean ? kNumSMs / 2 : 2 * kNumSMs);
    // a row alone in its CTA gets 1024 threads: twice the warps to score it
    const int nt = (cl == 1 && n_cand <= 8 * 1024) ? 1024 : kRowThreads;
    if (token_row_smem(s, K_b, cl, nt) <= kMaxDynSmem) return {TokenDispatch::kRow, "token_select_row_kernel", cl, nt};
  }
  const bool tc = g >= 16 && g <= 128 && (s.n_label == 16 || s.n_label == 32);
  // rows too long for one CTA's shared memory go to clusters whatever the
  // scoring load (each CTA keeps at most kTokMaxPerCta * 4 keys)
  if (tc || token_cluster_fits(g, s.n_label, n_cand) || n_cand > kTokSmemKeysMax)
    return {TokenDispatch::kCluster, "token_select_cluster_kernel", token_cluster_size(rows, n_cand, tc), kTokThreads};
  return {TokenDispatch::kChunked, "token_select_kernel", 1, 256};
}

void fill_token_params(TokenParams& p, const tls_shape& s, const void* q, const int32_t* label_ch,
                       const uint8_t* codes, const float* scales, const int32_t* block_idx, int K_b, int k,
                       int32_t* token_idx, float* token_score, uint8_t* ws, const WsLayout& L) {
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
  p.chunk = 0;
  p.tscore = reinterpret_cast<float*>(ws + L.tscore);
  p.token_score = token_score;
  p.counters = reinterpret_cast<unsigned*>(ws + L.tok_counter);
  p.token_idx = token_idx;
  p.seq_lens = s.seq_lens;
}

// `lean`: the row kernel on at most half the SMs (the other half is left to
// a level-1 grid running beside it, as in the resident stagger).
// `pdl`: the preceding kernel of the stream is this library's level-1 kernel,
// which writes only the block lists (the one input the cluster kernel reads
// after its dependency wait), so the launch may overlap its tail.
tls_status select_tokens_impl(const tls_shape& s, const void* q, const int32_t* label_ch, const uint8_t* codes,
                              const float* scales, const int32_t* block_idx, int K_b, int k, int32_t* token_idx,
                              float* token_score, uint8_t* ws, const WsLayout& L, cudaStream_t stream, bool pdl,
                              bool lean) {
  constexpr int NT = 256;
  const int rows = rows_of(s);
  TokenParams p;
  fill_token_params(p, s, q, label_ch, codes, scales, block_idx, K_b, k, token_idx, token_score, ws, L);
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

  const size_t smem = ((size_t)p.group * s.n_label + K_b + p.n_cand) * 4 + sizeof(TopkScratch) + 32;
  const TokenDispatch d = token_dispatch(s, K_b, lean,
                                         ((reinterpret_cast<uintptr_t>(codes) | reinterpret_cast<uintptr_t>(scales) |
                                           reinterpret_cast<uintptr_t>(q)) & 15u) == 0);
  if (d.kind == TokenDispatch::kRow) {
    const int cl = d.cl, nt = d.threads;
    const int kpt = p.n_cand <= 2 * nt ? 2 : p.n_cand <= 4 * nt ? 4 : p.n_cand <= 8 * nt ? 8 : 16;
    const size_t rsmem = token_row_smem(s, K_b, cl, nt);
    auto launch = [&](auto kernel) -> tls_status {
      cudaError_t e = kernel_attrs((const void*)kernel, rsmem);
      if (e != cudaSuccess) return cuda_check(e, "select_tokens: set kernel attributes");
      return cuda_check(launch_ex(kernel, dim3((unsigned)cl, (unsigned)rows), dim3((unsigned)nt), rsmem, stream, pdl,
                                  (unsigned)cl, p),
                        "select_tokens launch");
    };
    auto by_kpt = [&](auto k2, auto k4, auto k8, auto k16, auto w2, auto w4, auto w8) -> tls_status {
      if (nt == 1024) return kpt == 2 ? launch(w2) : kpt == 4 ? launch(w4) : launch(w8);
      return kpt == 2 ? launch(k2) : kpt == 4 ? launch(k4) : kpt == 8 ? launch(k8) : launch(k16);
    };
#define TLS_ROW(RR, NN)                                                                                     \
  by_kpt(token_select_row_kernel<RR, NN, 2, 512>, token_select_row_kernel<RR, NN, 4, 512>,                  \
         token_select_row_kernel<RR, NN, 8, 512>, token_select_row_kernel<RR, NN, 16, 512>,                 \
         token_select_row_kernel<RR, NN, 2, 1024>, token_select_row_kernel<RR, NN, 4, 1024>,                \
         token_select_row_kernel<RR, NN, 8, 1024>)
    if (s.n_label == 16) return p.group <= 8 ? TLS_ROW(16, 1) : TLS_ROW(16, 2);
    return p.group <= 8 ? TLS_ROW(32, 1) : TLS_ROW(32, 2);
#undef TLS_ROW
  }
  // wide groups score on the tensor cores, which keeps any candidate count in one cluster
  const bool tc = p.group >= 16 && p.group <= 128 && (s.n_label == 16 || s.n_label == 32);
  if (d.kind == TokenDispatch::kCluster) {
    const int cl = d.cl;
    const int per = (p.n_cand + cl - 1) / cl;
    const bool big = p.n_cand > kTokSmemKeysMax;  // the fallback gathers keys in the workspace
    const size_t cts_bytes = cl == 16 ? sizeof(ClusterTopkScratch<16>)
                             : cl == 8 ? sizeof(ClusterTopkScratch<8>)
                                       : sizeof(ClusterTopkScratch<4>);
    const size_t csmem = ((size_t)p.group * s.n_label + K_b + per + (big ? 0 : p.n_cand)) * 4 +
                         sizeof(TopkScratch) + cts_bytes + 32;
    const int ntile = p.group <= 16 ? 2 : p.group <= 32 ? 4 : p.group <= 64 ? 8 : 16;
    auto launch = [&](auto kernel) -> tls_status {
      // 16-CTA clusters are beyond the portable size
      cudaError_t e = kernel_attrs((const void*)kernel, csmem, cl > 8);
      if (e != cudaSuccess) return cuda_check(e, "select_tokens: set kernel attributes");
      return cuda_check(launch_ex(kernel, dim3((unsigned)cl, (unsigned)rows), dim3(kTokThreads), csmem, stream, pdl,
                                  (unsigned)cl, p),
                        "select_tokens launch");
    };
    auto by_cl = [&](auto k4, auto k8, auto k16, auto b4, auto b8, auto b16) -> tls_status {
      if (big) return cl == 16 ? launch(b16) : cl == 8 ? launch(b8) : launch(b4);
      return cl == 16 ? launch(k16) : cl == 8 ? launch(k8) : launch(k4);
    };
#define TLS_TC(RR, NN)                                                                                      \
  by_cl(token_select_cluster_kernel<RR, NN, 4, false>, token_select_cluster_kernel<RR, NN, 8, false>,       \
        token_select_cluster_kernel<RR, NN, 16, false>, token_select_cluster_kernel<RR, NN, 4, true>,        \
        token_select_cluster_kernel<RR, NN, 8, true>, token_select_cluster_kernel<RR, NN, 16, true>)
    if (tc) {
      if (s.n_label == 16) {
        if (ntile == 2) return TLS_TC(16, 2);
        if (ntile == 4) return TLS_TC(16, 4);
        if (ntile == 8) return TLS_TC(16, 8);
        return TLS_TC(16, 16);
      }
      if (ntile == 2) return TLS_TC(32, 2);
      if (ntile == 4) return TLS_TC(32, 4);
      if (ntile == 8) return TLS_TC(32, 8);
      return TLS_TC(32, 16);
    }
    switch (s.n_label) {
      case 2: return TLS_TC(2, 0);
      case 4: return TLS_TC(4, 0);
      case 8: return TLS_TC(8, 0);
      case 16: return TLS_TC(16, 0);
      case 32: return TLS_TC(32, 0);
      case 64: return TLS_TC(64, 0);
      default:
        return fail(TLS_ERR_UNSUPPORTED, "select_tokens: n_label %d not built (2,4,8,16,32,64)", s.n_label);
    }
#undef TLS_TC
  }
  dim3 grid((unsigned)chunks, (unsigned)rows);
  switch (s.n_label) {
#define TLS_TS_CASE(RR)                                                                                     \
  case RR: {                                                                                                \
    cudaError_t e = kernel_attrs((const void*)token_select_kernel<RR, NT>, smem);                          \
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
