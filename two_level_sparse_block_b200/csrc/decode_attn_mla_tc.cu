// Attention over the chosen tokens for the MLA latent cache on the tcgen05
// tensor cores (AsyncTLS, Italian summary 2.A.2: attention on the chosen
// tokens only; English summary 2.A Stage 1: the query heads that share a KV
// head form the M dimension of the tensor-core products, which is what makes
// shared-KV layouts such as MLA efficient).
//
// One latent row of 576 bf16 per token is the key, its first 512 values the
// value; the 128 heads of a group share it.  With the heads as M = 128:
//   S = Q . K^T     M = 128 heads, N = 32 tokens, K = 576      -> TMEM (fp32)
//   O += P . V      M = 128 heads, N = 256 value dims, K = 32  -> TMEM (fp32)
// O for all 512 value dims would fill TMEM, so a CTA owns one value half
// (256 columns) and computes S for it (the two halves' CTAs compute the same
// S).  CTA = (row, 128-head group, value half, token split); the token
// splits of a (row, group, half) form a thread-block cluster and merge their
// partial (max, sum, O) by log-sum-exp over distributed shared memory.
//
// Shared memory (1024-aligned):
//   Q      nine 128 x 64 k-block tiles, 128-byte swizzled, K-major, loaded
//          once by TMA (147,456 B)
//   ring   16 tiles of one 64-dim k-block of a 32-token chunk (32 rows of
//          128 B, swizzled as the K-major canonical layout), filled with
//          16-byte cp.async copies of the gathered latent rows; a chunk's nine
//          k-blocks enter in an order that puts the value half's four last, so
//          those four tiles are still resident when O += P . V reads them (as
//          the MN-major B operand: rows = tokens, 64 value dims a row)
//   P      128 rows of 128 B: P as bf16 hi (bytes 0-63) and the bf16 residual
//          lo (64-127) of the 32 tokens, so that P keeps ~16 significant bits
// Warps:  0-3 softmax (thread = head = TMEM lane), 4-7 gather, 8 MMA issue.
// Per chunk c: S(c) into TMEM buffer c % 2; softmax reads it, keeps a lazy
// running maximum (O is rescaled in TMEM only when the maximum grows by more
// than 2^8, so P <= 256 and no rescale happens for most chunks), writes P;
// O += P . V.  Every mbarrier wait is bounded (2 s); on expiry the error word
// is set, the CTA stops its loop, still takes part in the cluster barriers and
// frees its TMEM.

#include <cooperative_groups.h>
#include <cuda.h>
#include <cudaTypedefs.h>

#include "attn_common.cuh"
#include "device_common.cuh"
#include "host_common.h"

namespace tls {

constexpr int kTcQk = 576;
constexpr int kTcHeads = 128;              // MMA M: one group of 128 heads
constexpr int kTcChunk = 32;               // tokens per chunk (the S product's N)
constexpr int kTcKb = kTcQk / 64;          // 64-dim k-blocks of a latent row (9)
constexpr int kTcTile = kTcChunk * 128;    // a chunk's k-block tile: 32 rows x 128 B
constexpr int kTcRing = 16;                // ring tiles
constexpr int kTcOffRing = kTcHeads * kTcQk * 2;         // after Q (147,456)
constexpr int kTcOffP = kTcOffRing + kTcRing * kTcTile;  // 212,992
constexpr int kTcOffBar = kTcOffP + kTcHeads * 128;      // 229,376
constexpr int kTcSmem = kTcOffBar + 512;                 // barriers, TMEM slot, flag
constexpr int kTcThreads = 288;
constexpr uint32_t kTcCols = 512;          // O half: columns 0..255; S buffers: 256..319
constexpr int kTcOStride = 260;            // floats per row of the partial O (merge)
constexpr int kTcOffW = kTcHeads * kTcOStride * 4 + 2 * kTcHeads * 4;  // merge weights after O, m, l
constexpr uint64_t kTcWaitNs = 2000000000ull;
static_assert(kTcOffW + kTcHeads * 17 * 4 <= kTcOffRing, "merge scratch must fit in the Q region");

__device__ __forceinline__ float tc_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t tc_pack_bf16(float a, float b) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
  return r;
}

// k-block of position i (0..8) of a chunk: value half 0 -> 4 5 6 7 8 0 1 2 3,
// value half 1 -> 0 1 2 3 8 4 5 6 7 (the half's own four k-blocks last)
__device__ __forceinline__ int tc_kblock(int i, int vh) {
  if (i < 4) return vh ? i : 4 + i;
  if (i == 4) return 8;
  return vh ? i - 1 : i - 5;
}

__global__ void __launch_bounds__(kTcThreads, 1)
    sparse_attn_mla_tc_kernel(const __grid_constant__ CUtensorMap qmap, AttnParams p) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* q_full = reinterpret_cast<uint64_t*>(sm + kTcOffBar);
  uint64_t* full = q_full + 1;          // [kTcRing]: a tile's copies landed (128 gather threads)
  uint64_t* empty = full + kTcRing;     // [kTcRing]: the MMAs reading a tile are done
  uint64_t* s_full = empty + kTcRing;   // [2]: S of a chunk is in TMEM
  uint64_t* p_full = s_full + 2;        // P of a chunk written (128 softmax threads)
  uint64_t* p_free = p_full + 1;        // O += P . V of a chunk done (P free, O stable)
  uint64_t* mma_done = p_free + 1;      // every MMA of the CTA is complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* failed = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = (int)cluster.block_rank(), CL = (int)cluster.num_blocks();
  const int hg = (int)blockIdx.y >> 1, vh = (int)blockIdx.y & 1, row = (int)blockIdx.z;
  const int b = row / p.n_kv_heads, kvh = row % p.n_kv_heads;
  const int t_lo = min(p.k_sel, split * p.tokens_per_split);
  const int t_hi = min(p.k_sel, t_lo + p.tokens_per_split);
  const int n_chunks = (t_hi - t_lo + kTcChunk - 1) / kTcChunk;
  const int64_t len = seq_len_of(p.seq_lens, b, p.ctx_len);
  const int64_t oh = (int64_t)b * p.n_q_heads + (int64_t)kvh * p.group + hg * kTcHeads;  // first output head
  const uint32_t q_s = smem_u32(sm), ring_s = smem_u32(sm + kTcOffRing), p_s = smem_u32(sm + kTcOffP);

  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kTcRing; ++s) {
      mbar_init(&full[s], 128);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(p_full, 128);
    mbar_init(p_free, 1);
    mbar_init(mma_done, 1);
    *failed = 0;
    fence_barrier_init();
  } else if (tid == 32) {
    // the output and lse rows are written last: warm their translations now
    prefetch_l2(reinterpret_cast<const uint8_t*>(p.out) + (oh * p.dv + vh * 256) * (p.out_bf16 ? 2 : 4));
    if (p.lse != nullptr) prefetch_l2(p.lse + oh);
  }
  if (warp == 8) tmem_alloc(tmem_slot, kTcCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_launch_dependents();
  float my_m = -INFINITY, my_l = 0.0f;  // softmax threads: the head's running maximum (log2 units) and sum

  if (warp == 8) {
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      // Q: nine 128 x 64 tiles by TMA (an input of the step, not of the preceding kernel)
      mbar_arrive_expect_tx(q_full, (uint32_t)kTcOffRing);
      for (int j = 0; j < kTcKb; ++j) tma_load_2d(sm + j * 16384, &qmap, q_full, j * 64, (int)oh);
      bool ok = mbar_wait_bounded(q_full, 0, kTcWaitNs);
      const uint32_t id_s = idesc_bf16_f32(128, kTcChunk);
      const uint32_t id_pv = idesc_bf16_f32(128, 64, /*a_mn=*/false, /*b_mn=*/true);
      auto issue_s = [&](int c) -> bool {
        const uint32_t d = tmem + 256u + 32u * (uint32_t)(c & 1);
        for (int i = 0; i < kTcKb; ++i) {
          const int n = c * kTcKb + i, s = n % kTcRing;
          if (!mbar_wait_bounded(&full[s], (uint32_t)((n / kTcRing) & 1), kTcWaitNs)) return false;
          tc_fence_after();
          const uint32_t a0 = q_s + (uint32_t)tc_kblock(i, vh) * 16384u, b0 = ring_s + (uint32_t)s * kTcTile;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc_mma_bf16(d, sw128_kmajor_desc(a0 + kk * 32), sw128_kmajor_desc(b0 + kk * 32), id_s, (i | kk) != 0);
        }
        tc_commit(&s_full[c & 1]);
        for (int i = 0; i < 5; ++i) tc_commit(&empty[(c * kTcKb + i) % kTcRing]);  // the S-only tiles
        return true;
      };
      auto issue_pv = [&](int c) -> bool {
        if (!mbar_wait_bounded(p_full, (uint32_t)(c & 1), kTcWaitNs)) return false;
        tc_fence_after();
        for (int jv = 0; jv < 4; ++jv) {
          const uint32_t vt = ring_s + (uint32_t)((c * kTcKb + 5 + jv) % kTcRing) * kTcTile;
          const uint32_t d = tmem + 64u * (uint32_t)jv;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            // V: 16 token rows (two 8-row groups, 1024 B apart) of 64 value dims
            const uint64_t bd = sw128_mnmajor_desc(vt + kk * 2048, kTcTile, 1024);
            tc_mma_bf16(d, sw128_kmajor_desc(p_s + kk * 32), bd, id_pv, (c > 0 || kk > 0) ? 1u : 0u);
            tc_mma_bf16(d, sw128_kmajor_desc(p_s + 64 + kk * 32), bd, id_pv, 1u);
          }
        }
        tc_commit(p_free);
        for (int jv = 0; jv < 4; ++jv) tc_commit(&empty[(c * kTcKb + 5 + jv) % kTcRing]);  // the V tiles
        return true;
      };
      if (ok && n_chunks > 0) ok = issue_s(0);
      if (ok && n_chunks > 1) ok = issue_s(1);
      for (int c = 0; ok && c < n_chunks; ++c) {
        ok = issue_pv(c);
        if (ok && c + 2 < n_chunks) ok = issue_s(c + 2);
      }
      if (!ok) {
        *failed = 1;
        report_error(p.err, kErrTimeout, 301);
      }
      tc_commit(mma_done);  // after whatever was issued, on every path
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- gather
    // thread: token row r of the chunk, 16-byte units 2 qt, 2 qt + 1 of each k-block
    const int lt = tid - 128, r = lt & 31, qt = lt >> 5;
    grid_dependency_wait();  // token lists come from the preceding kernel
    auto rid_of = [&](int c) -> int64_t {
      const int t = t_lo + c * kTcChunk + r;
      if (t >= t_hi) return -1;
      const int tok = attn_token(p, row, t, len);
      return tok < 0 ? (int64_t)-1 : attn_row_id(p, row, tok);
    };
    bool ok = true;
    int64_t rid_next = n_chunks > 0 ? rid_of(0) : -1;
    for (int c = 0; c < n_chunks && ok; ++c) {
      const int64_t rid = rid_next;
      rid_next = c + 1 < n_chunks ? rid_of(c + 1) : -1;  // a chunk ahead: its latency hides behind the waits
      const bool v = rid >= 0;
      const uint16_t* src = p.k + (v ? rid * p.k_stride : 0);
      for (int i = 0; i < kTcKb; ++i) {
        // each tile as soon as its slot is free
        const int n = c * kTcKb + i, use = n / kTcRing;
        if (use > 0 && !mbar_wait_bounded(&empty[n % kTcRing], (uint32_t)((use - 1) & 1), kTcWaitNs)) {
          ok = false;
          break;
        }
        const uint32_t dst = ring_s + (uint32_t)(n % kTcRing) * kTcTile + (uint32_t)r * 128;
        const int kb = tc_kblock(i, vh);
#pragma unroll
        for (int uu = 0; uu < 2; ++uu) {
          const int u = 2 * qt + uu;
          cp_async16(dst + (uint32_t)((u ^ (r & 7)) << 4), src + kb * 64 + u * 8, v ? 16u : 0u);
        }
      }
      cp_async_commit();
      if (!ok) break;
      if (c > 0) {
        // chunk c - 1 has landed: publish it to the async proxy, then to the MMA
        cp_async_wait<1>();
        fence_proxy_async_smem();
        for (int i = 0; i < kTcKb; ++i) mbar_arrive(&full[((c - 1) * kTcKb + i) % kTcRing]);
      }
    }
    cp_async_wait<0>();
    fence_proxy_async_smem();
    if (ok && n_chunks > 0)
      for (int i = 0; i < kTcKb; ++i) mbar_arrive(&full[((n_chunks - 1) * kTcKb + i) % kTcRing]);
    if (!ok) {
      *failed = 1;
      report_error(p.err, kErrTimeout, 302);
    }
  } else {
    // ---------------------------------------------------------------- softmax
    const int h = tid;  // head within the group = TMEM lane
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    grid_dependency_wait();  // token lists come from the preceding kernel
    auto tok_of = [&](int c) -> int {
      const int t = t_lo + c * kTcChunk + lane;
      return t < t_hi ? attn_token(p, row, t, len) : -1;
    };
    float m_ref = -INFINITY, l_sum = 0.0f;
    bool ok = true;
    int tok_next = n_chunks > 0 ? tok_of(0) : -1;
    uint8_t* prow = sm + kTcOffP + (h >> 3) * 1024 + (h & 7) * 128;
    for (int c = 0; c < n_chunks; ++c) {
      const uint32_t vm = __ballot_sync(0xffffffffu, tok_next >= 0);  // entries of the chunk that are tokens
      tok_next = c + 1 < n_chunks ? tok_of(c + 1) : -1;
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&s_full[c & 1], (uint32_t)((c >> 1) & 1), kTcWaitNs));
      if (!ok) break;
      tc_fence_after();
      float sv[32];
      {
        float lo16[16], hi16[16];
        tmem_ld16(tmem + lane_base + 256u + 32u * (uint32_t)(c & 1), lo16);
        tmem_ld16(tmem + lane_base + 256u + 32u * (uint32_t)(c & 1) + 16u, hi16);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          sv[i] = lo16[i];
          sv[16 + i] = hi16[i];
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        sv[i] = ((vm >> i) & 1u) ? sv[i] * p.scale_log2 : -INFINITY;
        mx = fmaxf(mx, sv[i]);
      }
      // lazy maximum: moved only when the chunk's maximum passes it by 2^8
      const bool grow = mx > m_ref + 8.0f;
      const bool rescale = grow && m_ref != -INFINITY;
      const float ref = grow ? mx : m_ref;
      const float corr = rescale ? tc_exp2(m_ref - ref) : 1.0f;
      uint32_t ph[16], pl[16];
      float ps = 0.0f;
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const float p0 = ref == -INFINITY ? 0.0f : tc_exp2(sv[i] - ref);
        const float p1 = ref == -INFINITY ? 0.0f : tc_exp2(sv[i + 1] - ref);
        ps += p0 + p1;
        const uint32_t w = tc_pack_bf16(p0, p1);
        ph[i / 2] = w;
        pl[i / 2] = tc_pack_bf16(p0 - __uint_as_float(w << 16), p1 - __uint_as_float(w & 0xFFFF0000u));
      }
      l_sum = l_sum * corr + ps;
      m_ref = ref;
      // the P buffer is free and O stable once the previous chunk's O += P . V is done
      if (c > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(p_free, (uint32_t)((c - 1) & 1), kTcWaitNs));
        if (!ok) break;
        tc_fence_after();
      }
      if (__any_sync(0xffffffffu, rescale)) {
        for (int c0 = 0; c0 < 256; c0 += 16) {
          float o[16];
          tmem_ld16(tmem + lane_base + (uint32_t)c0, o);
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] *= corr;
          tmem_st16(tmem + lane_base + (uint32_t)c0, o);
        }
      }
      // row h of P: hi in 16-byte units 0-3, lo in 4-7, 128-byte swizzle
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        *reinterpret_cast<uint4*>(prow + ((cc ^ (h & 7)) << 4)) =
            make_uint4(ph[4 * cc], ph[4 * cc + 1], ph[4 * cc + 2], ph[4 * cc + 3]);
        *reinterpret_cast<uint4*>(prow + (((cc + 4) ^ (h & 7)) << 4)) =
            make_uint4(pl[4 * cc], pl[4 * cc + 1], pl[4 * cc + 2], pl[4 * cc + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (!ok) {
      *failed = 1;
      if (lane == 0) report_error(p.err, kErrTimeout, 303);
    }
    my_m = m_ref;
    my_l = l_sum;
  }
  // every MMA of the CTA is complete before TMEM and the Q region are reused
  if (warp < 4) {
    if (!__all_sync(0xffffffffu, mbar_wait_bounded(mma_done, 0, kTcWaitNs))) {
      *failed = 1;
      if (lane == 0) report_error(p.err, kErrTimeout, 304);
    }
    tc_fence_after();
  }

  // ---------------------------------------------------------------- partial (m, l, O) of this CTA
  // every MMA is complete (the last p_free) or the CTA failed; Q's region
  // holds the partial: O [128][kTcOStride], then m [128], l [128]
  __syncthreads();
  float* o_part = reinterpret_cast<float*>(sm);
  float* m_part = o_part + kTcHeads * kTcOStride;
  float* l_part = m_part + kTcHeads;
  const bool good = *failed == 0 && n_chunks > 0;
  if (warp < 4) {
    const int h = tid;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    m_part[h] = good ? my_m : -INFINITY;
    l_part[h] = good ? my_l : 0.0f;
    for (int c0 = 0; c0 < 256; c0 += 16) {
      float o[16];
      if (good) {
        tmem_ld16(tmem + lane_base + (uint32_t)c0, o);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) o[i] = 0.0f;
      }
#pragma unroll
      for (int i = 0; i < 16; i += 4)
        *reinterpret_cast<float4*>(o_part + h * kTcOStride + c0 + i) = make_float4(o[i], o[i + 1], o[i + 2], o[i + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, kTcCols);
  }
  cluster.sync();  // every CTA's partial is in place

  // ---------------------------------------------------------------- merge
  // CTA r of the cluster merges value dims [r * 256 / CL, (r + 1) * 256 / CL)
  // of the half for all 128 heads, by log-sum-exp over the CTAs' (m, l, O)
  // (m in log2 units, the reference l and O were summed against).
  float* w_s = reinterpret_cast<float*>(sm + kTcOffW);  // [128][17]: the CTAs' weights, then lse
  if (tid < kTcHeads) {
    float M = -INFINITY;
    for (int j = 0; j < CL; ++j) M = fmaxf(M, cluster.map_shared_rank(m_part, j)[tid]);
    float L = 0.0f, wj[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      wj[j] = 0.0f;
      if (j < CL) {
        const float mj = cluster.map_shared_rank(m_part, j)[tid];
        wj[j] = mj == -INFINITY ? 0.0f : exp2f(mj - M);
        L += wj[j] * cluster.map_shared_rank(l_part, j)[tid];
      }
    }
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) w_s[tid * 17 + j] = wj[j] * inv;
    w_s[tid * 17 + 16] = (M + log2f(L)) * 0.69314718055994531f;
  }
  __syncthreads();
  const int dspan = 256 / CL, d0 = split * dspan;
  for (int idx = tid; idx < kTcHeads * dspan; idx += kTcThreads) {
    const int h = idx / dspan, d = d0 + idx % dspan;
    float acc = 0.0f;
    for (int j = 0; j < CL; ++j) acc = fmaf(w_s[h * 17 + j], cluster.map_shared_rank(o_part, j)[h * kTcOStride + d], acc);
    const int64_t oe = (oh + h) * p.dv + vh * 256 + d;
    if (p.out_bf16) reinterpret_cast<uint16_t*>(p.out)[oe] = f32_to_bf16_rn(acc);
    else reinterpret_cast<float*>(p.out)[oe] = acc;
  }
  if (vh == 0 && split == 0 && p.lse != nullptr && tid < kTcHeads) p.lse[oh + tid] = w_s[tid * 17 + 16];
  cluster.sync();  // the other CTAs may still be reading this CTA's partial
}

bool attn_mla_tc_supported(const tls_shape& s) {
  return s.qk_dim == kTcQk && s.v_dim == 512 && s.v_offset == 0 && group_of(s) % kTcHeads == 0;
}

// CTAs per cluster (token splits of a row, group and value half): 16 when
// the grid of 16-CTA clusters fits the GPU at once, else 8.
int attn_mla_tc_splits(int rows, int groups) {
  static int cl16_ok = -1;
  if (cl16_ok < 0) {
    cl16_ok = 0;
    const size_t smem = 1024 + (size_t)kTcSmem;
    if (kernel_attrs((const void*)sparse_attn_mla_tc_kernel, smem, true) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(16, 1, 1);
      cfg.blockDim = dim3(kTcThreads);
      cfg.dynamicSmemBytes = smem;
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = 16;
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, (const void*)sparse_attn_mla_tc_kernel, &cfg) == cudaSuccess)
        cl16_ok = n;
      cudaGetLastError();
    }
  }
  return (cl16_ok >= rows * groups * 2 && rows * groups * 2 * 16 <= kNumSMs) ? 16 : 8;
}

tls_status launch_attn_mla_tc(const AttnParams& p, int rows, cudaStream_t stream, bool pdl) {
  alignas(64) CUtensorMap qmap;
  tls_status st = encode_bf16_2d_sw128(&qmap, p.q, (uint64_t)kTcQk, (uint64_t)rows / p.n_kv_heads * p.n_q_heads,
                                       64u, (uint32_t)kTcHeads);
  if (st != TLS_OK) return st;
  const size_t smem = 1024 + (size_t)kTcSmem;
  const int groups = p.group / kTcHeads;
  const int cl = attn_mla_tc_splits(rows, groups);
  AttnParams q = p;
  // a cluster's CTAs split the list into ranges of whole 32-token chunks
  q.tokens_per_split = ((p.k_sel + cl - 1) / cl + kTcChunk - 1) / kTcChunk * kTcChunk;
  cudaError_t e = kernel_attrs((const void*)sparse_attn_mla_tc_kernel, smem, cl > 8);
  if (e != cudaSuccess) return cuda_check(e, "sparse_decode_attn: set smem attribute");
  const dim3 grid((unsigned)cl, (unsigned)(2 * groups), (unsigned)rows);
  return cuda_check(launch_ex(sparse_attn_mla_tc_kernel, grid, dim3(kTcThreads), smem, stream, pdl, (unsigned)cl,
                              qmap, q),
                    "sparse_decode_attn: mla tc launch");
}

}  // namespace tls
