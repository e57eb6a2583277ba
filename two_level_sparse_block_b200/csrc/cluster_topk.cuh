// Deterministic top-k over keys spread across the CTAs of a thread-block
// cluster (sm_100a, distributed shared memory).
//
// CTA r of the cluster holds keys[0..n_loc) (its own shared memory) for the
// positions pos0 .. pos0 + n_loc - 1; the CTAs' ranges are contiguous in rank
// order.  The selection is the one cta_topk_ascending makes on the
// concatenated keys: the k largest, ties towards the lower position, written
// as out[j] = map(position) in ascending position order.
//
// Every exchange is a push: a CTA stores what the others need into their
// scratch (one array per step, written once) and a cluster barrier publishes
// it, so after the last barrier no CTA touches another's shared memory and
// any of them may exit.
//
//   1. key range: local min / max, pushed; barrier
//   2. 256 value bins over the range: local histogram, pushed; barrier
//   3. every CTA sums the histograms and finds the bin of the k-th key; if
//      that bin holds more than kTopkRankMax keys, steps 2-3 repeat with 256
//      sub-bins of it (at most kTopkLevels levels in all)
//   4. the local keys of that bin are compacted and pushed; barrier
//   5. every CTA ranks the (few) candidates pairwise: tau and how many keys
//      equal to tau to take
//   6. per-warp counts above / equal to tau; CTA totals pushed; barrier
//   7. output slots: CTAs before this one, warps before this one, lanes
//      before this one (ballot prefix counts), then the stores
//
// Returns false, uniformly over the cluster and with nothing written, when
// the keys cannot be binned (not finite, or all equal) or the threshold bin
// still holds more than kTopkRankMax keys after the last level of sub-bins
// (keys equal over a wide run); the caller then selects with one CTA.
// On both return paths the other CTAs' shared memory is still alive until
// the caller's next cluster barrier.
//
// Precondition: every CTA of the cluster has started (a cluster barrier has
// completed since launch, e.g. cluster_arrive_relaxed early and cluster_wait
// before the call), and all of them call this with the same k.
#pragma once

#include <cooperative_groups.h>

#include "device_common.cuh"

namespace tls {

template <int CL>
struct alignas(16) ClusterTopkScratch {
  // written by the cluster's CTAs (index = writer's rank)
  uint32_t lo[CL], hi[CL];
  int hist[2][CL][256];  // alternate levels use alternate halves
  int ncand[CL];
  alignas(16) uint32_t cand[CL][kTopkRankMax];  // rows read as uint4
  int tot_gt[CL], tot_eq[CL];
  // this CTA's own
  int hsum[256];
  uint32_t wlo[32], whi[32];
  int wgt[32], weq[32];
  int tbin, need, tcount, nloc, take;
  uint32_t tau;
  float lmin[kTopkLevels], linv[kTopkLevels];
  int lbin[kTopkLevels];
  uint32_t lcand[kTopkRankMax];
};

// Arrive / wait halves of the cluster barrier.  An early relaxed arrive
// followed by a wait before the first remote access guarantees that every
// CTA of the cluster has started, at no cost on the critical path.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

template <int NT, int CL, typename MapFn>
__device__ bool cluster_topk_ascending(const uint32_t* keys, int n_loc, int pos0, int k, int* out,
                                       ClusterTopkScratch<CL>& sm, MapFn map) {
  static_assert(NT % 32 == 0 && NT >= kTopkRankMax && NT <= 1024, "CTA size");
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  constexpr int NW = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rank = (int)cluster.block_rank();
  const unsigned below = (1u << lane) - 1u;

  // 1. key range
  {
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
    for (int i = tid; i < n_loc; i += NT) {
      lo = min(lo, keys[i]);
      hi = max(hi, keys[i]);
    }
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    if (lane == 0) {
      sm.wlo[warp] = lo;
      sm.whi[warp] = hi;
    }
    __syncthreads();
    if (tid < CL) {
      for (int w = 0; w < NW; ++w) {
        lo = min(lo, sm.wlo[w]);
        hi = max(hi, sm.whi[w]);
      }
      ClusterTopkScratch<CL>* dst = cluster.map_shared_rank(&sm, tid);
      dst->lo[rank] = lo;
      dst->hi[rank] = hi;
    }
  }
  cluster.sync();
  uint32_t glo = 0xFFFFFFFFu, ghi = 0u;
#pragma unroll
  for (int j = 0; j < CL; ++j) {
    glo = min(glo, sm.lo[j]);
    ghi = max(ghi, sm.hi[j]);
  }
  const float fmin = key_float(glo), fmax = key_float(ghi);
  const float span = fmax - fmin;
  if (!(glo != ghi && isfinite(fmin) && isfinite(fmax) && isfinite(span) && span > 0.0f)) return false;
  if (tid == 0) {
    sm.lmin[0] = fmin;
    sm.linv[0] = 256.0f / span;
  }
  // whether a key lies in the threshold bins of levels 0 .. upto - 1
  auto in_cell = [&](uint32_t key, int upto) {
    bool m = true;
    for (int l = 0; l < upto; ++l) m = m && topk_sub_bin(key, sm.lmin[l], sm.linv[l]) == sm.lbin[l];
    return m;
  };

  int lv = 0, need = k;
  for (;;) {
    // 2. local histogram of the keys in the current cell, pushed to every CTA
    for (int i = tid; i < 256; i += NT) sm.hsum[i] = 0;
    __syncthreads();
    const float lmin = sm.lmin[lv], linv = sm.linv[lv];
    for (int i = tid; i < n_loc; i += NT) {
      const uint32_t key = keys[i];
      if (in_cell(key, lv)) atomicAdd(&sm.hsum[topk_sub_bin(key, lmin, linv)], 1);
    }
    __syncthreads();
    for (int i = tid; i < 256 * CL; i += NT) {
      const int j = i >> 8, b = i & 255;
      *cluster.map_shared_rank(&sm.hist[lv & 1][rank][b], j) = sm.hsum[b];
    }
    cluster.sync();

    // 3. the bin of the need-th largest key of the cell (every CTA finds the same)
    for (int b = tid; b < 256; b += NT) {
      int s = 0;
#pragma unroll
      for (int j = 0; j < CL; ++j) s += sm.hist[lv & 1][j][b];
      sm.hsum[b] = s;
    }
    __syncthreads();
    if (tid < 32) {
      int local[8];
      int s = 0;
#pragma unroll
      for (int d = 0; d < 8; ++d) {
        local[d] = sm.hsum[255 - (tid * 8 + d)];
        s += local[d];
      }
      int incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += y;
      }
      int above = incl - s;
      if (above < need && incl >= need) {
        int d = 0;
        for (; d < 8; ++d) {
          if (above + local[d] >= need) break;
          above += local[d];
        }
        const int tb = 255 - (tid * 8 + d);
        sm.tbin = tb;
        sm.need = need - above;
        sm.tcount = local[d];
        sm.lbin[lv] = tb;
        if (lv + 1 < kTopkLevels) {
          // sub-bins of the threshold bin for the next level
          sm.lmin[lv + 1] = lmin + (float)tb / linv;
          sm.linv[lv + 1] = linv * 256.0f;
        }
      }
      if (tid == 0) sm.nloc = 0;
    }
    __syncthreads();
    // (hsum is cleared by the next level before every thread could read it,
    // so the bin's count travels in its own field)
    need = sm.need;
    if (sm.tcount <= kTopkRankMax) break;  // uniform over the cluster
    if (lv + 1 == kTopkLevels || !isfinite(sm.lmin[lv + 1]) || !isfinite(sm.linv[lv + 1])) return false;
    ++lv;
  }
  const int tbin = sm.tbin;
  const float bmin = sm.lmin[lv], binv = sm.linv[lv];

  // 4. local keys of that bin, pushed to every CTA
  for (int base = 0; base < n_loc; base += NT) {
    const int i = base + tid;
    const uint32_t key = i < n_loc ? keys[i] : 0u;
    const bool hit = i < n_loc && topk_sub_bin(key, bmin, binv) == tbin && in_cell(key, lv);
    const unsigned bal = __ballot_sync(0xffffffffu, hit);
    if (bal == 0u) continue;  // warp-uniform
    int slot0 = 0;
    if (lane == 0) slot0 = atomicAdd(&sm.nloc, __popc(bal));
    slot0 = __shfl_sync(0xffffffffu, slot0, 0);
    if (hit) {
      const int slot = slot0 + __popc(bal & below);
      if (slot < kTopkRankMax) sm.lcand[slot] = key;
    }
  }
  __syncthreads();
  {
    const int nl = sm.nloc, nlc = min(nl, kTopkRankMax);
    for (int i = tid; i < CL * nlc; i += NT) {
      const int j = i / nlc, t = i - j * nlc;
      *cluster.map_shared_rank(&sm.cand[rank][t], j) = sm.lcand[t];
    }
    if (tid < CL) *cluster.map_shared_rank(&sm.ncand[rank], tid) = nl;
  }
  cluster.sync();

  // 5. pairwise ranking of the candidates (every CTA, the same result)
  int nc = 0;
#pragma unroll
  for (int j = 0; j < CL; ++j) nc += sm.ncand[j];
  if (nc > kTopkRankMax) return false;
  if (tid < nc) {
    int t = tid, jj = 0;
    while (t >= sm.ncand[jj]) t -= sm.ncand[jj++];
    const uint32_t mine = sm.cand[jj][t];
    int gt = 0, eq = 0;
    // four candidates per 16-byte load; compact loops, since this code runs
    // once per call and its size (instruction fetch) costs more than the
    // latency that unrolling would hide
#pragma unroll 1
    for (int j = 0; j < CL; ++j) {
      const int m = sm.ncand[j];
      const uint4* c4 = reinterpret_cast<const uint4*>(sm.cand[j]);
#pragma unroll 1
      for (int q = 0; q < m; q += 4) {
        const uint4 v = c4[q >> 2];
        const uint32_t o[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          gt += (int)(q + u < m && o[u] > mine);
          eq += (int)(q + u < m && o[u] == mine);
        }
      }
    }
    if (gt < need && need <= gt + eq) {
      sm.tau = mine;  // every thread that holds tau writes the same values
      sm.take = need - gt;
    }
  }
  __syncthreads();
  const uint32_t tau = sm.tau;
  const int take_eq = sm.take;  // keys equal to tau to take, lowest positions first

  // 6. counts above / equal to tau over each warp's contiguous range
  const int per_w = ((n_loc + NW - 1) / NW + 31) & ~31;
  const int w_lo = min(n_loc, warp * per_w), w_hi = min(n_loc, w_lo + per_w);
  int cgt = 0, ceq = 0;
  for (int base = w_lo; base < w_hi; base += 32) {
    const int i = base + lane;
    const bool valid = i < w_hi;
    const uint32_t key = valid ? keys[i] : 0u;
    cgt += __popc(__ballot_sync(0xffffffffu, valid && key > tau));
    ceq += __popc(__ballot_sync(0xffffffffu, valid && key == tau));
  }
  if (lane == 0) {
    sm.wgt[warp] = cgt;
    sm.weq[warp] = ceq;
  }
  __syncthreads();
  if (tid < CL) {
    int g = 0, e = 0;
    for (int w = 0; w < NW; ++w) {
      g += sm.wgt[w];
      e += sm.weq[w];
    }
    *cluster.map_shared_rank(&sm.tot_gt[rank], tid) = g;
    *cluster.map_shared_rank(&sm.tot_eq[rank], tid) = e;
  }
  cluster.sync();  // last barrier: no remote access after this one

  // 7. output slots in position order
  int e_run = 0, p_run = 0;
  for (int j = 0; j < rank; ++j) {
    const int e = sm.tot_eq[j];
    p_run += sm.tot_gt[j] + min(e, max(0, take_eq - e_run));
    e_run += e;
  }
  for (int w = 0; w < warp; ++w) {
    const int e = sm.weq[w];
    p_run += sm.wgt[w] + min(e, max(0, take_eq - e_run));
    e_run += e;
  }
  for (int base = w_lo; base < w_hi; base += 32) {
    const int i = base + lane;
    const bool valid = i < w_hi;
    const uint32_t key = valid ? keys[i] : 0u;
    const bool q = valid && key == tau;
    const unsigned eb = __ballot_sync(0xffffffffu, q);
    const bool take = (valid && key > tau) || (q && e_run + __popc(eb & below) < take_eq);
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    const int pos = p_run + __popc(tb & below);
    if (take && pos < k) out[pos] = map(pos0 + i);
    e_run += __popc(eb);
    p_run += __popc(tb);
  }
  return true;
}

}  // namespace tls
