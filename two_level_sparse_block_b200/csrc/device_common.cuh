// Device helpers shared by the libtls kernels (sm_100a only).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace tls {

// ----------------------------------------------------------------------------
// Workspace header: word 0 is the error word set by kernels whose bounded
// waits ran out; word 1 records where.
// ----------------------------------------------------------------------------
constexpr int kErrTimeout = 4;

__device__ __forceinline__ void report_error(int* err, int code, int where) {
  if (err != nullptr) {
    atomicCAS(err, 0, code);
    atomicCAS(err + 1, 0, where);
  }
}

// Programmatic dependent launch: wait for the preceding kernel of the stream
// (no-op when the launch carried no programmatic dependency), and let the
// next kernel be scheduled early.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Tokens sequence b holds: seq_lens[b] clamped into [0, cap], or cap when
// there is no length array.  Read through L2 (an earlier kernel of the stream
// may have written it).
__device__ __forceinline__ int64_t seq_len_of(const int32_t* seq_lens, int b, int64_t cap) {
  if (seq_lens == nullptr) return cap;
  const int64_t v = __ldcg(seq_lens + b);
  return v < 0 ? 0 : (v > cap ? cap : v);
}

// -1 into out[from, to) (the padding of a selection with fewer valid entries
// than asked for); all threads of the CTA may call it.
__device__ __forceinline__ void pad_list(int32_t* out, int from, int to) {
  for (int i = from + (int)threadIdx.x; i < to; i += (int)blockDim.x) out[i] = -1;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// ----------------------------------------------------------------------------
// bf16 helpers
// ----------------------------------------------------------------------------
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  f[0] = bf16lo(v.x); f[1] = bf16hi(v.x);
  f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
  f[4] = bf16lo(v.z); f[5] = bf16hi(v.z);
  f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
}

__device__ __forceinline__ uint16_t f32_to_bf16_rn(float x) {
  __nv_bfloat16 b = __float2bfloat16_rn(x);
  return *reinterpret_cast<uint16_t*>(&b);
}

// ----------------------------------------------------------------------------
// Order-preserving map float -> uint32 (larger float -> larger key).
// -0 is folded onto +0 and NaN onto -inf so that equal values tie.
// ----------------------------------------------------------------------------
// Prefetches the line at p into L2.  Issued early for a buffer a kernel
// writes only at its end, it also brings the buffer's address translation
// into the SM's TLBs while the kernel still waits for its inputs.
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ uint32_t float_key(float f) {
  if (f != f) f = -INFINITY;
  if (f == 0.0f) f = 0.0f;
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ----------------------------------------------------------------------------
// CTA-wide deterministic top-k.
//
// keys[0..n) (shared memory) hold float_key(score).  Selects the k largest
// keys, ties broken towards the lower position, and writes
// out[j] = map(position) for the selected positions in ascending order.
//
// 1. The smallest and largest key bound the scores.  If they are finite and
//    differ, one pass bins every key by value into 256 equal-width bins over
//    [min, max] (a monotone map, so bins never reorder keys) and finds the
//    bin that holds the k-th largest key.  Float keys are log-scaled, so this
//    splits a few-octave range far better than the top bits of the key.
// 2. The keys of that bin are compacted and the exact threshold tau and the
//    number of keys equal to tau to take are found among them: by ranking
//    them pairwise when they are few, else by radix passes (8 bits at a time)
//    over the compacted keys, or over all keys if they do not fit.
// 3. Every warp owns a contiguous range of positions.  One ballot pass counts
//    the keys above and equal to tau per warp; a second one hands out output
//    slots in position order (ballot prefix counts inside a warp, the warps'
//    counts before it across warps).
//
// The scans of steps 2 and 3 read the keys of four 32-key steps before they
// vote, so a warp has four shared-memory loads in flight instead of one.
// ----------------------------------------------------------------------------
constexpr int kTopkCand = 512;
constexpr int kTopkRankMax = 128;  // at most this many compacted keys are ranked pairwise
struct TopkScratch {
  int hist[256];
  uint32_t wlo[32], whi[32];
  int wgt[32], weq[32];
  uint32_t prefix, mask;
  int need;   // how many more keys must be taken at the current prefix
  int ncand;  // keys still in contention, compacted into cand[]
  int tbin;   // value bin of the k-th largest key
  uint32_t lo, hi;
  uint32_t tau;  // threshold found by the pairwise ranking
  int take;      // keys equal to tau to take, found by the pairwise ranking
  int tcount;    // keys in the threshold bin (cta_topk_regs)
  uint32_t cand[kTopkCand];
};

__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// 256 value bins of a (finite) key over [fmin, fmin + 256 / inv]
__device__ __forceinline__ int topk_value_bin(uint32_t key, float fmin, float inv) {
  return min(255, (int)((key_float(key) - fmin) * inv));
}

__device__ __forceinline__ uint32_t smem_addr32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

constexpr int kTopkLevels = 3;  // levels of 256 sub-bins before a selection gives up on value bins

// bin of a key at a sub-bin level: the bounds are rounded, so a key of the
// parent bin may fall just outside [fmin, fmin + 256 / inv]; clamping keeps
// the map monotone in the key, which is all the selection relies on
__device__ __forceinline__ int topk_sub_bin(uint32_t key, float fmin, float inv) {
  return max(0, min(255, (int)((key_float(key) - fmin) * inv)));
}

// Out of line: it is the fallback of the other selections, and its code
// inlined into their kernels would sit between their hot phases and the
// instruction fetch.
template <int NT, typename MapFn>
__device__ __noinline__ void cta_topk_ascending(const uint32_t* keys, int n, int k, int* out, TopkScratch& sm,
                                   MapFn map) {
  static_assert(NT % 32 == 0 && NT >= kTopkRankMax && NT <= 1024, "CTA size");
  constexpr int NW = NT / 32;
  constexpr int U = 4;  // 32-key steps batched per warp iteration
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned below = (1u << lane) - 1u;
  // this warp's contiguous range of positions
  const int per_w = ((n + NW - 1) / NW + 31) & ~31;
  const int w_lo = min(n, warp * per_w), w_hi = min(n, w_lo + per_w);

  // 0. smallest and largest key
  {
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
#pragma unroll 4
    for (int i = tid; i < n; i += NT) {
      const uint32_t key = keys[i];
      lo = min(lo, key);
      hi = max(hi, key);
    }
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    if (lane == 0) {
      sm.wlo[warp] = lo;
      sm.whi[warp] = hi;
    }
    __syncthreads();
    if (tid == 0) {
      for (int w = 1; w < NW; ++w) {
        lo = min(lo, sm.wlo[w]);
        hi = max(hi, sm.whi[w]);
      }
      const uint32_t diff = lo ^ hi;
      const uint32_t undecided = diff == 0 ? 0u : (0xFFFFFFFFu >> __clz(diff));
      sm.mask = ~undecided;
      sm.prefix = lo & ~undecided;
      sm.need = k;
      sm.lo = lo;
      sm.hi = hi;
      sm.ncand = -1;  // no compacted set yet
    }
    __syncthreads();
  }

  // 1. value bins over [min, max]
  const float fmin = key_float(sm.lo), fmax = key_float(sm.hi);
  const float span = fmax - fmin;
  bool ranked = false;
  if (sm.lo != sm.hi && isfinite(fmin) && isfinite(fmax) && isfinite(span) && span > 0.0f) {
    const float inv = 256.0f / span;
    for (int i = tid; i < 256; i += NT) sm.hist[i] = 0;
    __syncthreads();
    // value bins are spread over the range, so plain shared atomics rarely collide
#pragma unroll 4
    for (int i = tid; i < n; i += NT) atomicAdd(&sm.hist[topk_value_bin(keys[i], fmin, inv)], 1);
    __syncthreads();
    if (tid < 32) {
      int local[8];
      int s = 0;
#pragma unroll
      for (int d = 0; d < 8; ++d) {
        local[d] = sm.hist[255 - (tid * 8 + d)];
        s += local[d];
      }
      int incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += y;
      }
      int above = incl - s;
      if (above < k && incl >= k) {
        int d = 0;
        for (; d < 8; ++d) {
          if (above + local[d] >= k) break;
          above += local[d];
        }
        sm.tbin = 255 - (tid * 8 + d);
        sm.need = k - above;
      }
      if (tid == 0) sm.ncand = 0;
    }
    __syncthreads();
    const int tbin = sm.tbin;
    // 2. compact the keys of the threshold bin (slot order is irrelevant)
    for (int base = w_lo; base < w_hi; base += 32 * U) {
      uint32_t kv[U];
      unsigned bal[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = base + 32 * u + lane;
        kv[u] = i < w_hi ? keys[i] : 0u;
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = base + 32 * u + lane;
        bal[u] = __ballot_sync(0xffffffffu, i < w_hi && topk_value_bin(kv[u], fmin, inv) == tbin);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (bal[u] == 0u) continue;  // warp-uniform
        int slot0 = 0;
        if (lane == 0) slot0 = atomicAdd(&sm.ncand, __popc(bal[u]));
        slot0 = __shfl_sync(0xffffffffu, slot0, 0);
        if ((bal[u] >> lane) & 1u) {
          const int slot = slot0 + __popc(bal[u] & below);
          if (slot < kTopkCand) sm.cand[slot] = kv[u];
        }
      }
    }
    __syncthreads();
    const int nc = sm.ncand;
    if (nc <= kTopkRankMax) {
      // few keys: thread t ranks compacted key t against all of them
      ranked = true;
      if (tid < kTopkRankMax) {
        const int need = sm.need;
        const uint32_t mine = tid < nc ? sm.cand[tid] : 0u;
        int gt = 0, eq = 0, c = 0;
        for (; c + 4 <= nc; c += 4) {
          const uint32_t o0 = sm.cand[c], o1 = sm.cand[c + 1], o2 = sm.cand[c + 2], o3 = sm.cand[c + 3];
          gt += (int)(o0 > mine) + (int)(o1 > mine) + (int)(o2 > mine) + (int)(o3 > mine);
          eq += (int)(o0 == mine) + (int)(o1 == mine) + (int)(o2 == mine) + (int)(o3 == mine);
        }
        for (; c < nc; ++c) {
          const uint32_t o = sm.cand[c];
          gt += (int)(o > mine);
          eq += (int)(o == mine);
        }
        if (tid < nc && gt < need && need <= gt + eq) {
          sm.tau = mine;  // every thread that holds tau writes the same values
          sm.take = need - gt;
        }
      }
    }
  }

  // radix passes for whatever is still undecided
  __syncthreads();
  uint32_t tau;
  int take_eq;  // keys equal to tau to take, lowest positions first
  if (ranked) {
    tau = sm.tau;
    take_eq = sm.take;
  } else {
    const uint32_t* src = keys;
    int nsrc = n;
    if (sm.ncand > 0 && sm.ncand <= kTopkCand) {
      // restart the radix select inside the compacted bin
      src = sm.cand;
      nsrc = sm.ncand;
    }
    if (tid == 0) {
      // over all keys the common prefix of min and max is skipped; inside a
      // compacted bin all 32 bits are decided (sm.need already counts there)
      uint32_t lo = 0u, hi = 0xFFFFFFFFu;
      if (src == keys) {
        lo = sm.lo;
        hi = sm.hi;
        sm.need = k;
      }
      const uint32_t diff = lo ^ hi;
      const uint32_t undecided = diff == 0 ? 0u : (0xFFFFFFFFu >> __clz(diff));
      sm.mask = ~undecided;
      sm.prefix = lo & ~undecided;
    }
    __syncthreads();
    int top = 31 - __clz(~sm.mask);  // highest undecided bit, -1 if none (clz(0) = 32)
#pragma unroll 1
    while (top >= 0) {
      const int shift = top >= 7 ? top - 7 : 0;
      const int width = top - shift + 1;
      const uint32_t dmask = (1u << width) - 1u;
      for (int i = tid; i < 256; i += NT) sm.hist[i] = 0;
      __syncthreads();
      const uint32_t prefix = sm.prefix, mask = sm.mask;
      for (int base = 0; base < nsrc; base += NT) {
        const int i = base + tid;
        uint32_t key = 0;
        bool valid = false;
        if (i < nsrc) {
          key = src[i];
          valid = (key & mask) == prefix;
        }
        const uint32_t d = valid ? ((key >> shift) & dmask) : 0xFFFFFFFFu;
        const unsigned peers = __match_any_sync(0xffffffffu, d);
        if (valid && lane == __ffs(peers) - 1) atomicAdd(&sm.hist[d], __popc(peers));
      }
      __syncthreads();
      if (tid < 32) {
        int local[8];
        int s = 0;
#pragma unroll
        for (int d = 0; d < 8; ++d) {
          local[d] = sm.hist[255 - (tid * 8 + d)];
          s += local[d];
        }
        int incl = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (tid >= o) incl += y;
        }
        const int need = sm.need;
        int above = incl - s;
        if (above < need && incl >= need) {
          int d = 0;
          for (; d < 8; ++d) {
            if (above + local[d] >= need) break;
            above += local[d];
          }
          const uint32_t digit = 255u - (uint32_t)(tid * 8 + d);
          sm.prefix = prefix | (digit << shift);
          sm.mask = mask | (dmask << shift);
          sm.need = need - above;
        }
      }
      __syncthreads();
      top = shift - 1;
    }
    tau = sm.prefix;
    take_eq = sm.need;
  }

  // 3. per-warp counts above / equal to tau
  int cgt = 0, ceq = 0;
  for (int base = w_lo; base < w_hi; base += 32 * U) {
    uint32_t kv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + 32 * u + lane;
      kv[u] = i < w_hi ? keys[i] : 0u;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const bool valid = base + 32 * u + lane < w_hi;
      cgt += __popc(__ballot_sync(0xffffffffu, valid && kv[u] > tau));
      ceq += __popc(__ballot_sync(0xffffffffu, valid && kv[u] == tau));
    }
  }
  if (lane == 0) {
    sm.wgt[warp] = cgt;
    sm.weq[warp] = ceq;
  }
  __syncthreads();
  // keys equal to tau and output slots used by the warps before this one
  int e_run = 0, p_run = 0;
  for (int w = 0; w < warp; ++w) {
    const int e = sm.weq[w];
    p_run += sm.wgt[w] + min(e, max(0, take_eq - e_run));
    e_run += e;
  }
  // slots in position order
  for (int base = w_lo; base < w_hi; base += 32 * U) {
    uint32_t kv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + 32 * u + lane;
      kv[u] = i < w_hi ? keys[i] : 0u;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + 32 * u + lane;
      const bool valid = i < w_hi;
      const bool q = valid && kv[u] == tau;
      const unsigned eb = __ballot_sync(0xffffffffu, q);
      const bool take = (valid && kv[u] > tau) || (q && e_run + __popc(eb & below) < take_eq);
      const unsigned tb = __ballot_sync(0xffffffffu, take);
      const int pos = p_run + __popc(tb & below);
      if (take && pos < k) out[pos] = map(i);
      e_run += __popc(eb);
      p_run += __popc(tb);
    }
  }
}

// Same selection as cta_topk_ascending for n <= KPT * NT keys, with every
// thread holding KPT consecutive positions in registers: a handful of CTA
// barriers, prefix counts by warp scans instead of shared counters, and
// sub-bins (up to three levels of 256) instead of radix passes.
//   0. key range (warp reductions, every thread folds the warp results)
//   1. value-bin histogram of the keys still in the threshold cell; the bin
//      of the need-th key narrows the cell; repeat while it holds > 128 keys
//   2. the cell's keys compacted at scanned offsets
//   3. pairwise ranking of those: tau and how many keys equal to it to take
//   4. counts above / equal to tau scanned over the CTA, then each thread
//      writes its own taken positions
// Degenerate keys (all equal, not finite, or a wide run of equal keys at the
// threshold) go to cta_topk_ascending.  `keys` is shared memory (read with
// 16-byte loads when it is 16-byte aligned and KPT a multiple of 4); its first
// k words are overwritten (the output is staged there).
template <int NT, int KPT, typename MapFn>
__device__ void cta_topk_regs(const uint32_t* keys, int n, int k, int* out, TopkScratch& sm, MapFn map) {
  static_assert(NT % 32 == 0 && NT >= kTopkRankMax && NT <= 1024 && KPT >= 1 && KPT <= 32, "shape");
  constexpr int NW = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int p0 = tid * KPT;
  uint32_t kv[KPT];
  uint32_t cell = 0u;  // bit j: key j is valid and still in the threshold cell
  if constexpr (KPT % 4 == 0) {
    if (p0 + KPT <= n && (smem_addr32(keys) & 15u) == 0u) {
#pragma unroll
      for (int j = 0; j < KPT; j += 4) {
        const uint4 v = *reinterpret_cast<const uint4*>(keys + p0 + j);
        kv[j] = v.x;
        kv[j + 1] = v.y;
        kv[j + 2] = v.z;
        kv[j + 3] = v.w;
      }
      cell = KPT == 32 ? 0xFFFFFFFFu : (1u << KPT) - 1u;
    } else {
#pragma unroll
      for (int j = 0; j < KPT; ++j) {
        kv[j] = p0 + j < n ? keys[p0 + j] : 0u;
        if (p0 + j < n) cell |= 1u << j;
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
      kv[j] = p0 + j < n ? keys[p0 + j] : 0u;
      if (p0 + j < n) cell |= 1u << j;
    }
  }

  // 0. key range
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    if ((cell >> j) & 1u) {
      lo = min(lo, kv[j]);
      hi = max(hi, kv[j]);
    }
  }
  lo = __reduce_min_sync(0xffffffffu, lo);
  hi = __reduce_max_sync(0xffffffffu, hi);
  if (lane == 0) {
    sm.wlo[warp] = lo;
    sm.whi[warp] = hi;
  }
  for (int i = tid; i < 256; i += NT) sm.hist[i] = 0;
  __syncthreads();
  // every warp folds the warp results, one per lane
  lo = __reduce_min_sync(0xffffffffu, lane < NW ? sm.wlo[lane] : 0xFFFFFFFFu);
  hi = __reduce_max_sync(0xffffffffu, lane < NW ? sm.whi[lane] : 0u);
  const float fmin = key_float(lo), fmax = key_float(hi);
  const float span = fmax - fmin;
  bool ok = lo != hi && isfinite(fmin) && isfinite(fmax) && isfinite(span) && span > 0.0f;  // uniform
  float lmin = fmin, linv = ok ? 256.0f / span : 0.0f;
  int need = k;

  // 1. levels of value bins
  for (int lv = 0; ok; ++lv) {
#pragma unroll
    for (int j = 0; j < KPT; ++j)
      if ((cell >> j) & 1u) atomicAdd(&sm.hist[topk_sub_bin(kv[j], lmin, linv)], 1);
    __syncthreads();
    if (warp == 0) {
      int local[8];
      int s = 0;
#pragma unroll
      for (int d = 0; d < 8; ++d) {
        local[d] = sm.hist[255 - (lane * 8 + d)];
        s += local[d];
      }
      int incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int above = incl - s;
      if (above < need && incl >= need) {
        int d = 0;
        for (; d < 8; ++d) {
          if (above + local[d] >= need) break;
          above += local[d];
        }
        sm.tbin = 255 - (lane * 8 + d);
        sm.need = need - above;
        sm.tcount = local[d];
      }
    }
    __syncthreads();
    const int tb = sm.tbin;
    need = sm.need;
#pragma unroll
    for (int j = 0; j < KPT; ++j)
      if (((cell >> j) & 1u) && topk_sub_bin(kv[j], lmin, linv) != tb) cell &= ~(1u << j);
    if (sm.tcount <= kTopkRankMax) break;
    // sub-bins of the threshold bin
    lmin = lmin + (float)tb / linv;
    linv = linv * 256.0f;
    ok = lv + 1 < kTopkLevels && isfinite(lmin) && isfinite(linv);
    // every thread has read the scan results; the histogram is free again
    for (int i = tid; i < 256; i += NT) sm.hist[i] = 0;
    __syncthreads();
  }
  if (!ok) {
    __syncthreads();  // the scratch fields read above are rewritten by the fallback
    cta_topk_ascending<NT>(keys, n, k, out, sm, map);
    return;
  }

  // 2. compaction of the threshold cell at scanned offsets
  {
    const int c = __popc(cell);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) sm.wgt[warp] = incl;
    __syncthreads();
    int off = incl - c + (int)__reduce_add_sync(0xffffffffu, lane < warp ? (unsigned)sm.wgt[lane] : 0u);
#pragma unroll
    for (int j = 0; j < KPT; ++j)
      if ((cell >> j) & 1u) sm.cand[off++] = kv[j];
    __syncthreads();
  }

  // 3. pairwise ranking inside the cell: TPC adjacent threads per key, thread
  // `part` comparing the 16-byte chunks part, part + TPC, ... that hold
  // candidates (the TPC lanes of a key read adjacent chunks: no bank
  // conflicts), four chunk loads in flight at a time
  {
    constexpr int TPC = NT / kTopkRankMax;  // 1, 2, 4 or 8
    const int nc = sm.tcount;
    const int c = tid / TPC, part = tid % TPC;
    if (c < nc) {
      const uint32_t mine = sm.cand[c];
      const int nq = (nc + 4 * TPC - 1) / (4 * TPC);  // chunks per thread
      const bool vec = (smem_addr32(sm.cand) & 15u) == 0u;  // (the scratch may sit anywhere 4-byte aligned)
      int gt = 0, eq = 0;
      for (int q0 = 0; q0 < nq; q0 += 4) {
        uint32_t o[4][4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i0 = 4 * ((q0 + u) * TPC + part);
          if (q0 + u < nq && vec) {
            const uint4 v = *reinterpret_cast<const uint4*>(sm.cand + i0);
            o[u][0] = v.x; o[u][1] = v.y; o[u][2] = v.z; o[u][3] = v.w;
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) o[u][e] = q0 + u < nq ? sm.cand[i0 + e] : 0u;
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const bool in = q0 + u < nq && 4 * ((q0 + u) * TPC + part) + e < nc;
            gt += (int)(in && o[u][e] > mine);
            eq += (int)(in && o[u][e] == mine);
          }
      }
      // the TPC lanes of a key are adjacent and all inside the c < nc branch
      const unsigned grp = TPC == 32 ? 0xffffffffu : (((1u << TPC) - 1u) << (lane & ~(TPC - 1)));
#pragma unroll
      for (int o = 1; o < TPC; o <<= 1) {
        gt += __shfl_xor_sync(grp, gt, o);
        eq += __shfl_xor_sync(grp, eq, o);
      }
      if (part == 0 && gt < need && need <= gt + eq) {
        sm.tau = mine;  // every thread that holds tau writes the same values
        sm.take = need - gt;
      }
    }
  }
  __syncthreads();
  const uint32_t tau = sm.tau;
  const int take_eq = sm.take;

  // 4. counts above / equal to tau before this thread, then the stores
  int gt = 0, eq = 0;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    const bool valid = p0 + j < n;
    gt += (int)(valid && kv[j] > tau);
    eq += (int)(valid && kv[j] == tau);
  }
  const int v = gt | (eq << 16);  // n <= 32768: neither half overflows
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sm.weq[warp] = incl;
  __syncthreads();
  const int pre = incl - v + (int)__reduce_add_sync(0xffffffffu, lane < warp ? (unsigned)sm.weq[lane] : 0u);
  int e_run = pre >> 16;
  int slot = (pre & 0xFFFF) + min(e_run, take_eq);
  // taken positions staged in shared memory (over the keys, which every
  // thread holds in registers by now), then written out coalesced
  int* stage = reinterpret_cast<int*>(const_cast<uint32_t*>(keys));
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    if (p0 + j >= n) continue;
    bool take = kv[j] > tau;
    if (kv[j] == tau) {
      take = e_run < take_eq;
      ++e_run;
    }
    if (take) {
      if (slot < k) stage[slot] = p0 + j;
      ++slot;
    }
  }
  __syncthreads();
  for (int i = tid; i < k; i += NT) out[i] = map(stage[i]);
}

// The two halves of a block score's query operand [relu(q), min(q, 0)] on a
// pair of bf16 values (exact: a sign test per half).
__device__ __forceinline__ uint32_t relu_bf16x2(uint32_t w) {
  uint32_t neg = (w & 0x80008000u) >> 15;  // 1 in each negative half
  return w & ~(neg * 0xFFFFu);
}
__device__ __forceinline__ uint32_t min0_bf16x2(uint32_t w) {
  uint32_t neg = (w & 0x80008000u) >> 15;
  return w & (neg * 0xFFFFu);
}

// ----------------------------------------------------------------------------
// mbarrier / TMA / tcgen05 wrappers (PTX ISA 8.7, sm_100a)
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0]; }" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1; }" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete; gives up after
// `limit_ns` nanoseconds and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > limit_ns) return false;
  }
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 2-D tiled TMA load (no multicast) completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::
          "r"(smem_u32(dst)),
      "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
               "r"(ncols));
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major operand in the 128-byte
// swizzled canonical layout: rows of 128 B, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);        // start address
  d |= (uint64_t)1 << 16;                           // leading byte offset (unused here)
  d |= (uint64_t)(1024 >> 4) << 32;                 // stride byte offset: 8 rows * 128 B
  d |= (uint64_t)1 << 46;                           // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                           // layout: 128-byte swizzle
  return d;
}

// Instruction descriptor: kind::f16, bf16 x bf16 -> f32; K-major operands
// unless a_mn / b_mn select MN-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn = false, bool b_mn = false) {
  return (1u << 4)                      // D format f32
         | (1u << 7)                    // A format bf16
         | (1u << 10)                   // B format bf16
         | ((a_mn ? 1u : 0u) << 15)     // A major
         | ((b_mn ? 1u : 0u) << 16)     // B major
         | ((uint32_t)(N >> 3) << 17)   // N / 8
         | ((uint32_t)(M >> 4) << 24);  // M / 16
}

// 16-byte asynchronous global -> shared copy (L2 only); src_bytes = 0 fills zeros.
__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* gptr, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(saddr), "l"(gptr), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void tc_mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(
          tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// 32 lanes x 32 bit, 16 consecutive columns per thread.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

}  // namespace tls
