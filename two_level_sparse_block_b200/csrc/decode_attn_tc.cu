// Attention over the chosen tokens on the tcgen05 tensor cores (AsyncTLS,
// Italian summary 2.A.2: attention runs on the selected tokens only), for
// 128-wide key and value rows.
//
// Persistent, software-pipelined: one CTA per SM walks a contiguous range of
// work items, an item being one tile of 128 entries of a row's token list for
// one head group (<= 64 heads) of the row.  Tokens are the MMA's M dimension,
// so any group size fills the M = 128 tile.  Per item:
//   gather   (issued NS-1 items ahead) cp.async 16-byte copies of the chosen
//            K and V rows into a 64 KB ring stage of 128B-swizzled tiles
//            ([64-column panel][token][128 B]); missing rows are zero-filled
//   QK       S^T[tok, h] = K_tile (K-major) . Q^T (K-major)       -> TMEM
//   softmax  fp32, base 2, online across the CTA's tiles of the same row
//            (running max and sum per head; O rescaled in TMEM when the max
//            moves); scores pass through shared memory to reduce per head
//   PV       O^T[d, h] += V^T (MN-major view of the V tile) . P^T, with P split
//            into bf16 hi + lo parts (two MMAs) so that P keeps ~16
//            significant bits; one bf16 P could move an output by 2^-8.
// At the end of its part of a row a CTA writes (m, l, O) to the split
// workspace; the last part to finish merges them by log-sum-exp.
// Tensor-core waits are bounded (2 s) and report through the workspace
// error word; the CTA then stops and releases its TMEM.

#include "attn_common.cuh"
#include "device_common.cuh"
#include "host_common.h"

namespace tls {

constexpr int kAttnTile = 128;
constexpr uint64_t kAttnWaitNs = 2000000000ull;
constexpr int kStageBytes = 65536;  // K tile (32 KB) + V tile (32 KB)

struct AttnTcLayout {
  int off_q, off_s, off_row, off_stat, off_bar, bytes;
};

__host__ __device__ inline AttnTcLayout attn_tc_layout(int npad, int heads, int stages) {
  AttnTcLayout L;
  L.off_q = stages * kStageBytes;       // Q panel: 2 x npad x 128 B
  L.off_s = L.off_q + 2 * npad * 128;   // scores: heads x 128 floats
  L.off_row = L.off_s + heads * 128 * 4;
  L.off_stat = L.off_row + 128 * 8;     // m[64], l[64], corr[64]
  L.off_bar = L.off_stat + 3 * 64 * 4;  // 2 mbarriers, tmem slot, flags
  L.bytes = L.off_bar + 32;
  return L;
}

template <int NPAD, int NS>
__global__ void __launch_bounds__(128, 1) sparse_attn_tc_kernel(AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int HG = p.heads_per_cta;
  const AttnTcLayout L = attn_tc_layout(NPAD, HG, NS);
  uint8_t* sQ = sm + L.off_q;
  float* sS = reinterpret_cast<float*>(sm + L.off_s);
  int64_t* srow = reinterpret_cast<int64_t*>(sm + L.off_row);
  float* s_m = reinterpret_cast<float*>(sm + L.off_stat);
  float* s_l = s_m + 64;
  float* s_corr = s_m + 128;
  uint64_t* bar_s = reinterpret_cast<uint64_t*>(sm + L.off_bar);
  uint64_t* bar_o = bar_s + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_o + 1);
  volatile int* s_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);  // [0] merge, [1] rescale
  constexpr uint32_t kCols = (2 * NPAD <= 32) ? 32u : (2 * NPAD <= 64 ? 64u : 128u);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = p.group;
  const int T = p.tiles_per_pair;
  const int64_t W = p.n_items;
  const int64_t c = blockIdx.x;
  const int64_t i0 = c * W / p.n_ctas, i1 = (c + 1) * W / p.n_ctas;

  if (tid == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, kCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;

  // storage row of entry `tid` of item `it` (-1: past the token list); indices are clamped
  auto row_of_entry = [&](int64_t it) -> int64_t {
    const int64_t pair = it / T;
    const int row = (int)(pair / p.head_groups);
    const int t = (int)(it % T) * kAttnTile + tid;
    if (t >= p.k_sel) return -1;
    const int64_t tok =
        min(max((int64_t)__ldcg(p.token_idx + (int64_t)row * p.k_sel + t), (int64_t)0), p.ctx_len - 1);
    if (p.slot_of_block != nullptr) {
      const int64_t slot = min(max(__ldg(p.slot_of_block + (int64_t)row * p.nb + tok / p.bs), 0), p.n_slots - 1);
      return slot * p.bs + tok % p.bs;
    }
    return (int64_t)row * p.ctx_len + tok;
  };
  // cp.async of the K and V rows listed in srow into ring stage `st`
  auto issue_gather = [&](int st) {
    const int cc = tid & 15;
    const uint32_t kb = smem_u32(sm + st * kStageBytes), vb = kb + 32768;
#pragma unroll 4
    for (int it = 0; it < 16; ++it) {
      const int r = (tid >> 4) + 8 * it;
      const int64_t rid = srow[r];
      const uint32_t off = (uint32_t)((cc >> 3) * 16384 + r * 128 + (((cc & 7) ^ (r & 7)) << 4));
      const bool v = rid >= 0;
      cp_async16(kb + off, p.k + (v ? rid * p.k_stride : 0) + cc * 8, v ? 16u : 0u);
      cp_async16(vb + off, p.v + (v ? rid * p.v_stride : 0) + cc * 8, v ? 16u : 0u);
    }
  };

  grid_launch_dependents();
  grid_dependency_wait();  // token lists come from the preceding kernel

  // prologue: gathers for the first NS-1 items
  for (int j = 0; j < NS - 1; ++j) {
    const int64_t it = i0 + j;
    if (it < i1) {
      srow[tid] = row_of_entry(it);
      __syncthreads();
      issue_gather(j);
      __syncthreads();
    }
    cp_async_commit();
  }

  int hgp = 4;
  int64_t cur_pair = -1;
  bool first_tile = true;
  bool ok = true;
  int phase = 0;
  for (int64_t it = i0; it < i1; ++it, phase ^= 1) {
    const int j = (int)(it - i0);
    const int st = j % NS;
    uint8_t* sK = sm + st * kStageBytes;
    const uint32_t kaddr = smem_u32(sK), vaddr = kaddr + 32768;
    const int64_t pair = it / T;
    const int row = (int)(pair / p.head_groups), hg = (int)(pair % p.head_groups);
    const int b = row / p.n_kv_heads, kvh = row % p.n_kv_heads;
    const int h0 = hg * HG;
    const int nh = min(HG, g - h0);
    const int t_begin = (int)(it % T) * kAttnTile;
    const int n_valid = min(kAttnTile, p.k_sel - t_begin);
    const bool last_of_part = (it + 1 == i1) || ((it + 1) / T != pair);

    if (pair != cur_pair) {
      // a new (row, head group): load its Q panel, reset the running softmax
      for (int i = tid; i < NPAD * 16; i += 128) {
        const int h = i >> 4, cq = i & 15;
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if (h < nh)
          w = *reinterpret_cast<const uint4*>(p.q + ((int64_t)b * p.n_q_heads + kvh * g + h0 + h) * p.dqk + cq * 8);
        *reinterpret_cast<uint4*>(sQ + (cq >> 3) * (NPAD * 128) + h * 128 + (((cq & 7) ^ (h & 7)) << 4)) = w;
      }
      if (tid < 64) {
        s_m[tid] = -INFINITY;
        s_l[tid] = 0.0f;
      }
      hgp = 4;
      while (hgp < nh) hgp <<= 1;
      cur_pair = pair;
      first_tile = true;
    }
    // the index of the item NS-1 ahead is read now; its gather is issued after QK
    const int64_t nxt = it + NS - 1;
    const int64_t nxt_row = nxt < i1 ? row_of_entry(nxt) : -1;

    cp_async_wait<NS - 2>();
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16_f32(128, NPAD);
#pragma unroll
      for (int kb = 0; kb < 2; ++kb)
#pragma unroll
        for (int k16 = 0; k16 < 4; ++k16)
          tc_mma_bf16(tmem, sw128_kmajor_desc(kaddr + kb * 16384 + k16 * 32),
                      sw128_kmajor_desc(smem_u32(sQ) + kb * NPAD * 128 + k16 * 32), idesc, (kb | k16) != 0);
      tc_commit(bar_s);
    }
    srow[tid] = nxt_row;  // read by the gather below, after two barriers
    __syncwarp();
    ok = __syncthreads_and(mbar_wait_bounded(bar_s, phase, kAttnWaitNs)) != 0;
    if (!ok) break;
    tc_fence_after();
    {
      const bool tv = tid < n_valid;
#pragma unroll
      for (int c0 = 0; c0 < NPAD; c0 += 16) {
        float v[16];
        tmem_ld16(tmem + lane_base + (uint32_t)c0, v);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (c0 + i < nh) sS[(c0 + i) * 128 + tid] = tv ? v[i] * p.scale_log2 : -INFINITY;
      }
    }
    __syncthreads();

    // per head: tph threads, hgp consecutive tokens each
    const int tph = 128 / hgp;
    const int h = tid / tph, part = tid % tph;
    float m_new = -INFINITY;
    {
      float m_t = -INFINITY;
      if (h < nh)
        for (int i = 0; i < hgp; ++i) m_t = fmaxf(m_t, sS[h * 128 + part * hgp + i]);
      for (int o = tph >> 1; o > 0; o >>= 1) m_t = fmaxf(m_t, __shfl_xor_sync(0xffffffffu, m_t, o));
      const float m_old = h < nh ? s_m[h] : -INFINITY;
      m_new = fmaxf(m_old, m_t);
      float l_t = 0.0f;
      if (h < nh)
        for (int i = 0; i < hgp; ++i) l_t += exp2f(sS[h * 128 + part * hgp + i] - m_new);
      for (int o = tph >> 1; o > 0; o >>= 1) l_t += __shfl_xor_sync(0xffffffffu, l_t, o);
      __syncthreads();  // every thread has read s_m
      if (part == 0 && h < nh) {
        const float corr = (m_old == -INFINITY) ? 0.0f : exp2f(m_old - m_new);
        s_corr[h] = corr;
        s_m[h] = m_new;
        s_l[h] = s_l[h] * corr + l_t;
      }
      if (tid == 0) s_flag[1] = 0;
      // P^T (the PV B operand, K-major over tokens) overwrites the consumed K tile
      for (int i = tid; i < NPAD * 32; i += 128) reinterpret_cast<uint4*>(sK)[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    __syncthreads();
    if (!first_tile && tid < nh && s_corr[tid] != 1.0f) s_flag[1] = 1;
    if (h < nh) {
      uint8_t* plo = sK + NPAD * 256;
      for (int i = 0; i < hgp; ++i) {
        const int t = part * hgp + i;
        const float pv = exp2f(sS[h * 128 + t] - m_new);
        const uint16_t hi = f32_to_bf16_rn(pv);
        const uint16_t lo = f32_to_bf16_rn(pv - __uint_as_float((uint32_t)hi << 16));
        const int off = (t >> 6) * (NPAD * 128) + h * 128 + ((((t & 63) >> 3) ^ (h & 7)) << 4) + (t & 7) * 2;
        *reinterpret_cast<uint16_t*>(sK + off) = hi;
        *reinterpret_cast<uint16_t*>(plo + off) = lo;
      }
    }
    // the stage of item it-1 is free: gather item it+NS-1 into it
    if (nxt < i1) issue_gather((j + NS - 1) % NS);
    cp_async_commit();
    __syncthreads();
    if (s_flag[1]) {
      // the running max moved: rescale O^T (lane d, one column per head)
      tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < NPAD; c0 += 16) {
        float v[16];
        tmem_ld16(tmem + lane_base + (uint32_t)(NPAD + c0), v);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (c0 + i < nh) v[i] *= s_corr[c0 + i];
        tmem_st16(tmem + lane_base + (uint32_t)(NPAD + c0), v);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16_f32(128, NPAD, /*a_mn=*/true, false);
      const uint32_t pb = kaddr;
#pragma unroll
      for (int step = 0; step < 8; ++step) {
        const uint64_t a = sw128_mnmajor_desc(vaddr + step * 2048, 16384, 1024);
        const uint32_t boff = (uint32_t)((step >> 2) * NPAD * 128 + (step & 3) * 32);
        tc_mma_bf16(tmem + NPAD, a, sw128_kmajor_desc(pb + boff), idesc, (!first_tile || step > 0) ? 1u : 0u);
        tc_mma_bf16(tmem + NPAD, a, sw128_kmajor_desc(pb + NPAD * 256 + boff), idesc, 1u);
      }
      tc_commit(bar_o);
    }
    __syncwarp();
    ok = __syncthreads_and(mbar_wait_bounded(bar_o, phase, kAttnWaitNs)) != 0;
    if (!ok) break;
    tc_fence_after();
    first_tile = false;

    if (last_of_part) {
      // this CTA's share of (row, head group) ends here: write its partial
      const int64_t first = attn_owner(pair * T, W, p.n_ctas);
      const int n_part = (int)(attn_owner(pair * T + T - 1, W, p.n_ctas) - first + 1);
      const int slot = (int)(c - first);
      const int dv = p.dv;
      float* part_base = p.partial + (((int64_t)row * g + h0) * p.splits + slot) * (dv + 2);
      const int64_t hstride = (int64_t)p.splits * (dv + 2);
#pragma unroll
      for (int c0 = 0; c0 < NPAD; c0 += 16) {
        float v[16];
        tmem_ld16(tmem + lane_base + (uint32_t)(NPAD + c0), v);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (c0 + i < nh) part_base[(c0 + i) * hstride + 2 + tid] = v[i];
      }
      if (tid < nh) {
        part_base[tid * hstride + 0] = s_m[tid];
        part_base[tid * hstride + 1] = s_l[tid];
      }
      __threadfence();
      __syncthreads();
      if (tid == 0)
        s_flag[0] = atomicInc(&p.counters[pair], (unsigned)(n_part - 1)) == (unsigned)(n_part - 1);
      __syncthreads();
      if (s_flag[0]) {
        __threadfence();
        merge_splits(p, row, b, kvh, h0, nh, n_part, sS, HG * 128);
      }
    }
    tc_fence_before();
    __syncthreads();
  }
  if (!ok && lane == 0) report_error(p.err, kErrTimeout, 201);
  cp_async_wait<0>();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

bool attn_tc_supported(const tls_shape& s) {
  return s.qk_dim == 128 && s.v_dim == 128 && s.v_offset < 0;
}

static int attn_tc_npad(int heads) { return heads <= 16 ? 16 : heads <= 32 ? 32 : 64; }

// Work partition of the persistent kernel: items = rows x head groups x tiles,
// one CTA per SM.  Returns the largest number of CTAs that share one
// (row, head group), which sizes the split workspace.
int attn_tc_plan(int rows, int head_groups, int k, int* tiles, int* n_items, int* n_ctas) {
  const int T = (k + kAttnTile - 1) / kAttnTile;
  const int64_t W = (int64_t)rows * head_groups * T;
  int64_t n = W < kNumSMs ? W : kNumSMs;
  if (n > 63 * (int64_t)rows * head_groups) n = 63 * (int64_t)rows * head_groups;  // <= 64 splits per pair
  int max_part = 1;
  for (int64_t q = 0; q < (int64_t)rows * head_groups; ++q) {
    const int64_t parts = attn_owner(q * T + T - 1, W, n) - attn_owner(q * T, W, n) + 1;
    if (parts > max_part) max_part = (int)parts;
  }
  *tiles = T;
  *n_items = (int)W;
  *n_ctas = (int)n;
  return max_part;
}

template <int NPAD, int NS>
static tls_status launch_tc(const AttnParams& p, cudaStream_t stream, bool pdl) {
  const AttnTcLayout L = attn_tc_layout(NPAD, p.heads_per_cta, NS);
  const size_t smem = 1024 + (size_t)L.bytes;
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_tc_kernel<NPAD, NS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return cuda_check(e, "sparse_decode_attn: set smem attribute");
  return cuda_check(launch_ex(sparse_attn_tc_kernel<NPAD, NS>, dim3(p.n_ctas), dim3(128), smem, stream, pdl, 0u, p),
                    "sparse_decode_attn: tc launch");
}

tls_status launch_attn_tc(const AttnParams& p, int rows, cudaStream_t stream, bool pdl) {
  (void)rows;
  switch (attn_tc_npad(p.heads_per_cta)) {
    case 16: return launch_tc<16, 3>(p, stream, pdl);
    case 32: return launch_tc<32, 3>(p, stream, pdl);
    default: return launch_tc<64, 2>(p, stream, pdl);
  }
}

}  // namespace tls
