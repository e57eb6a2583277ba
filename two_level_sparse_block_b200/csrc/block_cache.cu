// HBM block cache with incremental transfer (AsyncTLS, English summary 2.B:
// only the blocks of the new candidate set that are not resident,
// T_t = M_t \ C_t, cross PCIe; the copies overlap the running attention).
//
// Host state: a mirror of the device slot table (block -> slot), the owner
// of every slot and its last use.  Planning is pure host code; the prefetch
// issues one cudaMemcpyAsync per run of blocks that are adjacent both in host
// memory and in the slot pool, then updates the device slot table.  The first
// transfer writes the whole table (nothing is resident, so nothing reads it);
// later ones change only the entries of the copied and the evicted blocks,
// which the running attention (reading M_{t-1}) never reads, so the update
// may run concurrently with it.

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <vector>

#include "device_common.cuh"
#include "host_common.h"

struct tls_block_cache {
  tls_shape shape;
  int rows = 0;
  int nb = 0;
  const uint8_t* host_k = nullptr;
  const uint8_t* host_v = nullptr;
  int64_t hk_stride = 0, hv_stride = 0;
  int n_slots = 0;
  uint8_t* slot_k = nullptr;
  uint8_t* slot_v = nullptr;
  int32_t* table_dev = nullptr;
  std::vector<int32_t> table;       // [rows * nb] -> slot or -1
  std::vector<int64_t> owner;       // [n_slots] -> row * nb + block, or -1
  std::vector<int64_t> last_use;    // [n_slots] planning step of the last use
  int64_t step = 0;
  int32_t* staging[2] = {nullptr, nullptr};  // pinned, mapped: the first table, then (entry, value) pairs
  cudaEvent_t staged[2] = {nullptr, nullptr};
  int cur = 0;
  bool published = false;                     // the device table has been written once
  // Pull path: when K/V are pinned host memory mapped into the device address
  // space, one kernel reads the planned blocks over PCIe into their slots.
  const uint8_t* dev_host_k = nullptr;        // device addresses of host_k / host_v
  const uint8_t* dev_host_v = nullptr;
  int4* jobs[2] = {nullptr, nullptr};         // pinned, mapped: {tok0 lo, tok0 hi, slot, 0} per copy
  // set when a transfer failed after some of its device work was queued: the
  // slots may no longer hold what the host mirror says, so every later
  // transfer or plan returns this status
  tls_status failed = TLS_OK;
  // Device planning (tls_prefetch_diff_device, the engine): the plan kernel
  // keeps the owner and last-use arrays on the device; while `device_owned`
  // the device copies (and the device slot table) are the cache state, and a
  // host path first downloads them.
  bool device_owned = false;
  int64_t* owner_dev = nullptr;
  int64_t* last_use_dev = nullptr;
  int4* jobs_dev = nullptr;      // [rows * K_b max] {tok0 lo, tok0 hi, slot, list entry}
  int32_t* n_jobs_dev = nullptr;
  int32_t* dev_failed = nullptr;  // pinned, mapped: set by a plan that found too few evictable slots
  int32_t* dev_failed_dptr = nullptr;  // its device address
  int max_entries = 0;            // rows * K_b the device arrays were sized for
};

namespace tls {
namespace {

struct Copy {
  int32_t row, block, slot;
};

// Device address of [p, p + bytes) when the whole range is pinned host memory
// mapped into the device address space as one contiguous range; else NULL.
const uint8_t* mapped_host_range(const void* p, size_t bytes) {
  if (p == nullptr || bytes == 0) return nullptr;
  cudaPointerAttributes a, b;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess ||
      cudaPointerGetAttributes(&b, (const uint8_t*)p + (bytes - 1)) != cudaSuccess) {
    cudaGetLastError();  // clear the sticky-free error of an unknown pointer
    return nullptr;
  }
  if (a.type != cudaMemoryTypeHost || b.type != cudaMemoryTypeHost || a.devicePointer == nullptr ||
      b.devicePointer == nullptr)
    return nullptr;
  if ((const uint8_t*)b.devicePointer - (const uint8_t*)a.devicePointer != (ptrdiff_t)(bytes - 1)) return nullptr;
  return (const uint8_t*)a.devicePointer;
}

bool fault_injected_copy() {
  const char* e = std::getenv("TLS_FAULT_INJECT");
  return e != nullptr && std::strcmp(e, "copy") == 0;
}

// Plans T_t and its victim slots without changing the cache.
tls_status plan(const tls_block_cache& c, const int32_t* new_idx, const int32_t* in_use, int K_b,
                std::vector<Copy>* copies, std::vector<int32_t>* victims) {
  const int64_t total = (int64_t)c.rows * c.nb;
  std::vector<char> keep(c.n_slots, 0);
  std::vector<char> seen(total, 0);
  copies->clear();
  for (int r = 0; r < c.rows; ++r) {
    for (int i = 0; i < K_b; ++i) {
      const int32_t blk = new_idx[(int64_t)r * K_b + i];
      if (blk < 0) continue;  // the -1 padding of a sequence with fewer than K_b blocks
      if (blk >= c.nb) return fail(TLS_ERR_INVALID_ARG, "plan: block %d out of range in row %d", blk, r);
      const int64_t key = (int64_t)r * c.nb + blk;
      if (seen[key]) return fail(TLS_ERR_INVALID_ARG, "plan: block %d repeated in row %d", blk, r);
      seen[key] = 1;
      const int32_t s = c.table[key];
      if (s >= 0) keep[s] = 1;
      else copies->push_back({r, blk, -1});
    }
    if (in_use != nullptr) {
      for (int i = 0; i < K_b; ++i) {
        const int32_t blk = in_use[(int64_t)r * K_b + i];
        if (blk < 0 || blk >= c.nb) continue;
        const int32_t s = c.table[(int64_t)r * c.nb + blk];
        if (s >= 0) keep[s] = 1;
      }
    }
  }
  // free slots first (ascending), then least recently used, then lower slot
  std::vector<int32_t> cand;
  for (int s = 0; s < c.n_slots; ++s)
    if (!keep[s] && c.owner[s] < 0) cand.push_back(s);
  std::vector<int32_t> used;
  for (int s = 0; s < c.n_slots; ++s)
    if (!keep[s] && c.owner[s] >= 0) used.push_back(s);
  std::stable_sort(used.begin(), used.end(), [&](int32_t a, int32_t b) {
    if (c.last_use[a] != c.last_use[b]) return c.last_use[a] < c.last_use[b];
    return a < b;
  });
  cand.insert(cand.end(), used.begin(), used.end());
  if (cand.size() < copies->size())
    return fail(TLS_ERR_CAPACITY, "plan: %zu blocks to copy but only %zu evictable slots", copies->size(),
                cand.size());
  // copy i (row, then list order) takes the i-th victim in slot order
  victims->assign(cand.begin(), cand.begin() + copies->size());
  std::sort(victims->begin(), victims->end());
  return TLS_OK;
}

// The slot-table changes a plan makes, as (entry, value) pairs, without
// changing the cache: each copied block's entry gets its victim slot, and the
// block a victim held (if any) loses its entry.  The new blocks are not
// resident and the evicted ones are, so no entry appears twice.
void assign_slots(const tls_block_cache& c, std::vector<Copy>& copies, const std::vector<int32_t>& victims,
                  std::vector<int2>* changes) {
  changes->clear();
  for (size_t i = 0; i < copies.size(); ++i) {
    const int32_t s = victims[i];
    if (c.owner[s] >= 0) changes->push_back(make_int2((int)c.owner[s], -1));
    changes->push_back(make_int2((int)((int64_t)copies[i].row * c.nb + copies[i].block), s));
    copies[i].slot = s;
  }
}

// Applies a plan to the host mirror (after its device work was queued).
void commit(tls_block_cache& c, const int32_t* new_idx, int K_b, const std::vector<Copy>& copies) {
  c.step += 1;
  for (const Copy& cp : copies) {
    if (c.owner[cp.slot] >= 0) c.table[c.owner[cp.slot]] = -1;
    const int64_t key = (int64_t)cp.row * c.nb + cp.block;
    c.owner[cp.slot] = key;
    c.table[key] = cp.slot;
  }
  for (int r = 0; r < c.rows; ++r)
    for (int i = 0; i < K_b; ++i) {
      const int32_t blk = new_idx[(int64_t)r * K_b + i];
      if (blk < 0) continue;
      c.last_use[c.table[(int64_t)r * c.nb + blk]] = c.step;
    }
}

// Copies planned blocks from mapped pinned host memory into their slots: CTA
// j takes job j (a block's bs rows of K and of V, contiguous on both sides),
// 16-byte loads, eight in flight per thread; then the slot-table changes.
// The consumers (the next attention) start after the whole kernel, so the
// order of the two parts does not matter.
constexpr int kPullThreads = 256;
// One job: the block's bs rows of K (and of V) from host memory into its
// slot.  The loads of both parts are issued together (one PCIe round trip
// for a block when the CTA's loads cover it), 32 bytes each where every
// address and size is 32-byte aligned, else 16.
__device__ __forceinline__ void pull_block(const uint8_t* host_k, const uint8_t* host_v, uint8_t* slot_k,
                                           uint8_t* slot_v, int64_t kblk, int64_t vblk, int64_t k_row_bytes,
                                           int64_t v_row_bytes, int4 jb) {
  const int64_t tok0 = (int64_t)(uint32_t)jb.x | ((int64_t)jb.y << 32);
  const int64_t slot = jb.z;
  const uint8_t* src0 = host_k + tok0 * k_row_bytes;
  uint8_t* dst0 = slot_k + slot * kblk;
  const bool with_v = host_v != nullptr && slot_v != nullptr;
  const uint8_t* src1 = with_v ? host_v + tok0 * v_row_bytes : src0;
  uint8_t* dst1 = with_v ? slot_v + slot * vblk : dst0;
  const int64_t n1 = with_v ? vblk : 0;
  const uintptr_t al = reinterpret_cast<uintptr_t>(src0) | reinterpret_cast<uintptr_t>(dst0) |
                       reinterpret_cast<uintptr_t>(src1) | reinterpret_cast<uintptr_t>(dst1) | (uintptr_t)kblk |
                       (uintptr_t)n1;
  if ((al & 31u) == 0) {
    // 32-byte units: K's first, then V's
    const int64_t a0 = kblk / 32, tot = a0 + n1 / 32;
    for (int64_t i0 = threadIdx.x; i0 < tot; i0 += 4 * kPullThreads) {
      uint32_t v[4][8];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t i = i0 + (int64_t)u * kPullThreads;
        if (i < tot) {
          const uint8_t* sp = i < a0 ? src0 + i * 32 : src1 + (i - a0) * 32;
          asm volatile("ld.global.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                       : "=r"(v[u][0]), "=r"(v[u][1]), "=r"(v[u][2]), "=r"(v[u][3]), "=r"(v[u][4]), "=r"(v[u][5]),
                         "=r"(v[u][6]), "=r"(v[u][7])
                       : "l"(sp));
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t i = i0 + (int64_t)u * kPullThreads;
        if (i < tot) {
          uint4* d = reinterpret_cast<uint4*>(i < a0 ? dst0 + i * 32 : dst1 + (i - a0) * 32);
          d[0] = make_uint4(v[u][0], v[u][1], v[u][2], v[u][3]);
          d[1] = make_uint4(v[u][4], v[u][5], v[u][6], v[u][7]);
        }
      }
    }
    return;
  }
  // 16-byte units (rows 16-byte aligned: checked at cache creation)
  const int64_t a0 = kblk / 16, tot = a0 + n1 / 16;
  for (int64_t i0 = threadIdx.x; i0 < tot; i0 += 8 * kPullThreads) {
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int64_t i = i0 + (int64_t)u * kPullThreads;
      if (i < tot)
        v[u] = __ldcv(reinterpret_cast<const uint4*>(i < a0 ? src0 + i * 16 : src1 + (i - a0) * 16));
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int64_t i = i0 + (int64_t)u * kPullThreads;
      if (i < tot) *reinterpret_cast<uint4*>(i < a0 ? dst0 + i * 16 : dst1 + (i - a0) * 16) = v[u];
    }
  }
}

__global__ void __launch_bounds__(kPullThreads) block_pull_kernel(const uint8_t* host_k, const uint8_t* host_v,
                                                                  uint8_t* slot_k, uint8_t* slot_v, int64_t kblk,
                                                                  int64_t vblk, int64_t k_row_bytes,
                                                                  int64_t v_row_bytes, const int4* jobs, int n_jobs,
                                                                  int32_t* table, const int2* pairs, int n_pairs) {
  if ((int)blockIdx.x < n_jobs)
    pull_block(host_k, host_v, slot_k, slot_v, kblk, vblk, k_row_bytes, v_row_bytes, jobs[blockIdx.x]);
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < n_pairs; i += kPullThreads) table[pairs[i].x] = pairs[i].y;
}

// The device plan's jobs: a fixed grid strides over the *n_jobs jobs the
// plan kernel wrote (the table is already updated).
__global__ void __launch_bounds__(kPullThreads) block_pull_jobs_kernel(const uint8_t* host_k, const uint8_t* host_v,
                                                                       uint8_t* slot_k, uint8_t* slot_v, int64_t kblk,
                                                                       int64_t vblk, int64_t k_row_bytes,
                                                                       int64_t v_row_bytes, const int4* jobs,
                                                                       const int32_t* n_jobs) {
  grid_dependency_wait();  // the plan kernel's jobs (programmatic dependent launch)
  const int n = *n_jobs;
  for (int j = blockIdx.x; j < n; j += gridDim.x)
    pull_block(host_k, host_v, slot_k, slot_v, kblk, vblk, k_row_bytes, v_row_bytes, jobs[j]);
}

// Applies (entry, value) pairs (mapped pinned memory) to the device slot table.
__global__ void slot_table_update_kernel(int32_t* table, const int2* pairs, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int2 pr = pairs[i];
    table[pr.x] = pr.y;
  }
}

// ---------------------------------------------------------------------------
// Device planning: the same plan as plan() + assign_slots() + commit(), made
// by one CTA from the device block lists, so no host wait sits between level
// 1 and the transfer.  Victims are the host plan's set: a slot's key is
// highest when it is free, then higher the longer it has not been used, and
// 0 when a block of M_t or M_{t-1} holds it; the n_copy largest keys win,
// ties to the lower slot (the CTA top-k's rule).  Copy i (in row, then list
// order) takes the i-th victim in slot order, as in the host plan, so both
// leave the same table.
constexpr int kPlanThreads = 512;  // small enough to start beside the step's other kernels
constexpr int kPlanMaxSlots = 32768;    // keys in shared memory
constexpr int kPlanMaxEntries = 65536;  // rows * K_b

struct PlanParams {
  int32_t* table;
  int64_t* owner;
  int64_t* last_use;
  const int32_t* new_idx;  // M_t [rows, K_b]
  const int32_t* in_use;   // M_{t-1} [rows, K_b] or NULL
  int rows, nb, K_b, n_slots, bs;
  int keep_prev;           // 1: the slots the previous plan used are kept (its list was M_{t-1})
  int64_t ctx_len, step;   // step: the plan's number (last use of M_t's slots)
  int4* jobs;
  int32_t* n_jobs;
  int32_t* n_out;    // optional: n_copy, or -1 when the plan failed
  int32_t* failed;   // mapped pinned flag, sticky
};

// Dynamic shared memory of the plan kernel (byte offsets): the slots' keys,
// the kept bits, the victims in slot order, the state of every list entry
// and the top-k scratch.
struct PlanSmem {
  size_t keys, kept, vic, ent, ts, total;
};
__host__ __device__ inline PlanSmem plan_smem(int n_slots, int n_entries) {
  auto a16 = [](size_t x) { return (x + 15) & ~(size_t)15; };
  PlanSmem m;
  const int nv = n_entries < n_slots ? n_entries : n_slots;
  m.keys = 0;
  m.kept = m.keys + a16((size_t)n_slots * 4);
  m.vic = m.kept + a16((size_t)((n_slots + 31) / 32) * 4);
  m.ent = m.vic + a16((size_t)nv * 4);
  m.ts = m.ent + a16((size_t)n_entries * 4);
  m.total = m.ts + a16(sizeof(TopkScratch));
  return m;
}

// Exclusive prefix of v over the CTA, with the total and the CTA's largest
// x.  All threads call it; three barriers.
__device__ __forceinline__ unsigned long long plan_scan_max(unsigned long long v, uint32_t x,
                                                            unsigned long long* wsum, uint32_t* wmax,
                                                            unsigned long long* total, uint32_t* xmax) {
  constexpr int NW = kPlanThreads / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned long long s = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xffffffffu, s, o);
    if (lane >= o) s += y;
  }
  x = __reduce_max_sync(0xffffffffu, x);
  if (lane == 31) wsum[warp] = s;
  if (lane == 0) wmax[warp] = x;
  __syncthreads();
  if (warp == 0) {
    unsigned long long w = lane < NW ? wsum[lane] : 0ull;
    uint32_t m = lane < NW ? wmax[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    m = __reduce_max_sync(0xffffffffu, m);
    if (lane < NW) wsum[lane] = w;  // inclusive
    if (lane == 0) wmax[NW] = m;
  }
  __syncthreads();
  const unsigned long long before = (warp > 0 ? wsum[warp - 1] : 0ull) + s - v;
  *total = wsum[NW - 1];
  *xmax = wmax[NW];
  __syncthreads();  // wsum / wmax may be reused
  return before;
}

// One CTA plans T_t and applies it.  The memory round trips on the path are
// few on purpose (the kernel runs beside the attention, which keeps DRAM busy
// and each round trip long): the first slot's state, the first list entries
// and the sticky flag are loaded together; then the table entries of M_t
// (and M_{t-1}); everything else is shared memory until the evicted slots'
// owners are read.  A list entry's state: its slot when resident, -1 when not
// a block (padding), -2 - block when it must be copied.
__global__ void __launch_bounds__(kPlanThreads, 1) block_plan_kernel(PlanParams p) {
  extern __shared__ __align__(16) uint8_t psm[];
  constexpr int NT = kPlanThreads;
  const int E = p.rows * p.K_b, nsl = p.n_slots;
  const PlanSmem L = plan_smem(nsl, E);
  uint32_t* pkeys = reinterpret_cast<uint32_t*>(psm + L.keys);
  uint32_t* kept = reinterpret_cast<uint32_t*>(psm + L.kept);
  int* vic = reinterpret_cast<int*>(psm + L.vic);
  int* ent = reinterpret_cast<int*>(psm + L.ent);
  TopkScratch* ts = reinterpret_cast<TopkScratch*>(psm + L.ts);
  __shared__ unsigned long long wsum[NT / 32];
  __shared__ uint32_t wmax[NT / 32 + 1];
  __shared__ int bad, failed_s, thr_bin, thr_above;
  const int tid = threadIdx.x;
  const int32_t* __restrict__ new_idx = p.new_idx;
  const int32_t* __restrict__ in_use = p.in_use;
  const uint32_t kFree = float_key(33554432.0f), kKept = float_key(0.0f);

  // 1. loads that depend on nothing: this thread's first slot and first list entry, the flag
  int64_t own0 = -1, lu0 = 0;
  if (tid < nsl) {
    own0 = p.owner[tid];
    lu0 = p.last_use[tid];
  }
  int blk0 = -1, prv0 = -1, ub0 = -1;
  if (tid < E) {
    blk0 = new_idx[tid];
    prv0 = tid % p.K_b > 0 ? new_idx[tid - 1] : -1;
    ub0 = in_use != nullptr ? in_use[tid] : -1;
  }
  const int32_t failed0 = tid == 0 ? *reinterpret_cast<volatile int32_t*>(p.failed) : 0;
  for (int w = tid; w < (nsl + 31) / 32; w += NT) kept[w] = 0u;
  if (tid < 256) ts->hist[tid] = 0;
  if (tid == 0) bad = 0;
  __syncthreads();
  // 2. the slots of M_t and M_{t-1} are kept; M_t must list distinct blocks
  //    in [0, NB) in ascending order (as level 1 writes it)
  for (int j = tid; j < E; j += NT) {
    int blk = blk0, prv = prv0, ub = ub0;
    if (j != tid) {
      blk = new_idx[j];
      prv = j % p.K_b > 0 ? new_idx[j - 1] : -1;
      ub = in_use != nullptr ? in_use[j] : -1;
    }
    const int64_t r = j / p.K_b;
    const bool ok = blk >= 0 && blk < p.nb;
    if (blk >= p.nb || (blk >= 0 && j % p.K_b > 0 && (prv >= blk || prv < 0))) bad = 1;
    const int s = ok ? p.table[r * p.nb + blk] : -1;
    const int su = (ub >= 0 && ub < p.nb) ? p.table[r * p.nb + ub] : -1;
    if (s >= 0 && s < nsl) atomicOr(&kept[s >> 5], 1u << (s & 31));
    if (su >= 0 && su < nsl) atomicOr(&kept[su >> 5], 1u << (su & 31));
    ent[j] = !ok ? -1 : s < 0 ? -2 - blk : s < nsl ? s : -1;
  }
  //    and the keys: free slots highest, then by the age of their last use
  for (int s = tid; s < nsl; s += NT) {
    int64_t own = own0, lu = lu0;
    if (s != tid) {
      own = p.owner[s];
      lu = p.last_use[s];
    }
    const int64_t age = p.step - lu;
    pkeys[s] = own < 0 ? kFree
                       : (p.keep_prev && age == 1) ? kKept
                                                   : float_key((float)(age < 1 ? 1 : (age > 16777215 ? 16777215 : age)));
  }
  if (tid == 0) failed_s = failed0;
  __syncthreads();
  if (failed_s != 0) {
    if (tid == 0) {
      *p.n_jobs = 0;
      if (p.n_out != nullptr) *p.n_out = -1;
    }
    return;
  }
  // 3. counts: blocks to copy (this thread's contiguous range of entries),
  //    evictable and free slots, and the oldest age
  const int per = (E + NT - 1) / NT;
  const int j0 = min(E, tid * per), j1 = min(E, j0 + per);
  int cnt = 0, avail = 0, nfree = 0;
  uint32_t kmax = 0u;
  for (int j = j0; j < j1; ++j) cnt += ent[j] <= -2;
  for (int s = tid; s < nsl; s += NT) {
    uint32_t k = pkeys[s];
    if ((kept[s >> 5] >> (s & 31)) & 1u) pkeys[s] = k = kKept;
    avail += k != kKept;
    nfree += k == kFree;
    if (k != kFree && k != kKept) kmax = max(kmax, k);
  }
  unsigned long long tot = 0ull;
  uint32_t amax_key = 0u;
  const unsigned long long before =
      plan_scan_max(((unsigned long long)cnt << 40) | ((unsigned long long)avail << 20) | (unsigned long long)nfree,
                    kmax, wsum, wmax, &tot, &amax_key);
  const int n_copy = (int)(tot >> 40), n_avail = (int)((tot >> 20) & 0xFFFFFu), n_free = (int)(tot & 0xFFFFFu);
  if (bad != 0 || n_copy > n_avail) {
    // nothing changes; the cache refuses later plans
    if (tid == 0) {
      *reinterpret_cast<volatile int32_t*>(p.failed) = bad != 0 ? 2 : 1;
      *p.n_jobs = 0;
      if (p.n_out != nullptr) *p.n_out = -1;
    }
    return;
  }
  if (tid == 0) {
    *p.n_jobs = n_copy;
    if (p.n_out != nullptr) *p.n_out = n_copy;
  }
  // 4. the victims: the n_copy largest keys (ties: lower slot), in slot
  //    order.  Free slots first; ages are small integers with many ties, so
  //    the threshold among used slots is found from a histogram of ages below
  //    the oldest (256 of them); wider spreads take the generic CTA top-k.
  uint32_t thr = kFree;
  int eq_take = n_copy;  // keys equal to thr to take, the first ones in slot order
  bool generic = false;
  const int need_used = n_copy - n_free;
  if (n_copy > 0 && need_used > 0) {
    const float amax = key_float(amax_key);
    for (int s = tid; s < nsl; s += NT) {
      const uint32_t k = pkeys[s];
      if (k == kFree || k == kKept) continue;
      const float d = amax - key_float(k);
      if (d < 256.0f) atomicAdd(&ts->hist[(int)d], 1);
    }
    __syncthreads();
    if (tid < 32) {
      // the bin (age below the oldest) where the count from the oldest reaches need_used
      int run = 0, bin = -1, above = 0;
      for (int c = 0; c < 256 && bin < 0; c += 32) {
        const int v = ts->hist[c + tid];
        int x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, x, o);
          if (tid >= o) x += y;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, run + x >= need_used);
        if (hit != 0u) {
          const int l = __ffs(hit) - 1;
          bin = c + l;
          above = run + __shfl_sync(0xffffffffu, x - v, l);
        }
        run += __shfl_sync(0xffffffffu, x, 31);
      }
      if (tid == 0) {
        thr_bin = bin;
        thr_above = above;
      }
    }
    __syncthreads();
    if (thr_bin < 0) {
      generic = true;
    } else {
      thr = float_key(amax - (float)thr_bin);
      eq_take = need_used - thr_above;
    }
  }
  if (generic) {
    cta_topk_ascending<NT>(pkeys, nsl, n_copy, vic, *ts, [](int i) { return i; });
  } else if (n_copy > 0) {
    // keys above thr and the first eq_take keys equal to it, compacted in
    // slot order (a contiguous range of slots per thread)
    const int sp = (nsl + NT - 1) / NT;
    const int s0 = min(nsl, tid * sp), s1 = min(nsl, s0 + sp);
    int above = 0, eq = 0;
    for (int s = s0; s < s1; ++s) {
      const uint32_t k = pkeys[s];
      above += k > thr && k != kKept;
      eq += k == thr;
    }
    unsigned long long t2 = 0ull;
    uint32_t unused = 0u;
    const unsigned long long b2 =
        plan_scan_max(((unsigned long long)above << 32) | (unsigned long long)eq, 0u, wsum, wmax, &t2, &unused);
    int e = (int)(b2 & 0xFFFFFFFFu);
    int pos = (int)(b2 >> 32) + min(eq_take, e);
    for (int s = s0; s < s1; ++s) {
      const uint32_t k = pkeys[s];
      const bool v = k == thr ? e++ < eq_take : (k > thr && k != kKept);
      if (v && pos < n_copy) vic[pos++] = s;
    }
  }
  __syncthreads();
  // the pull kernel may become resident from here (it waits for this grid)
  grid_launch_dependents();
  // 5. copy i (row, then list order) takes victim i: the evicted block loses
  //    its entry, the copied one gets the slot (no entry is touched twice:
  //    copied blocks are not resident, evicted ones are); every slot of M_t
  //    was used at this step
  int pos = (int)(before >> 40);
  for (int j = j0; j < j1; ++j) {
    int s = ent[j];
    if (s == -1) continue;
    const int64_t r = j / p.K_b;
    if (s <= -2) {
      const int blk = -2 - s;
      const int i = pos++;
      s = vic[i];
      if (s < 0 || s >= nsl) continue;  // unreachable: n_copy victims were chosen
      const int64_t key = r * p.nb + blk;
      const int64_t old = p.owner[s];
      if (old >= 0) p.table[old] = -1;
      p.table[key] = s;
      p.owner[s] = key;
      const int64_t tok0 = r * p.ctx_len + (int64_t)blk * p.bs;
      p.jobs[i] = make_int4((int)(uint32_t)(tok0 & 0xFFFFFFFF), (int)(tok0 >> 32), s, j);
    }
    p.last_use[s] = p.step;
  }
}

// The host mirror follows the device state again (after device plans): the
// device work is drained and the table, owners and last uses are copied back.
tls_status sync_host_mirror(tls_block_cache& c) {
  if (!c.device_owned) return TLS_OK;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess)
    e = cudaMemcpy(c.table.data(), c.table_dev, c.table.size() * sizeof(int32_t), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess)
    e = cudaMemcpy(c.owner.data(), c.owner_dev, c.owner.size() * sizeof(int64_t), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess)
    e = cudaMemcpy(c.last_use.data(), c.last_use_dev, c.last_use.size() * sizeof(int64_t), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) {
    c.failed = TLS_ERR_COPY;
    return fail(TLS_ERR_COPY, "block cache: reading the device state back failed: %s", cudaGetErrorString(e));
  }
  c.device_owned = false;
  return TLS_OK;
}

// A device plan that failed leaves the flag set: the cache is failed from then on.
tls_status device_plan_status(tls_block_cache& c) {
  if (c.dev_failed != nullptr && c.failed == TLS_OK) {
    const int32_t f = *reinterpret_cast<volatile int32_t*>(c.dev_failed);
    if (f != 0) c.failed = f == 2 ? TLS_ERR_INVALID_ARG : TLS_ERR_CAPACITY;
  }
  if (c.failed != TLS_OK)
    return fail(c.failed, c.failed == TLS_ERR_CAPACITY
                              ? "block cache: a device plan found too few evictable slots"
                              : c.failed == TLS_ERR_INVALID_ARG
                                    ? "block cache: a device plan got a block list that is not ascending and in range"
                                    : "block cache: an earlier transfer failed; the slots no longer match the block lists");
  return TLS_OK;
}

}  // namespace

// Whether device planning serves this cache for K_b blocks per row, and its
// device arrays (allocated once, sized for the largest K_b asked for); the
// host mirror's state is uploaded when the device takes over.
tls_status block_cache_device_ready(tls_block_cache* c, int K_b) {
  if (c->dev_host_k == nullptr || c->slot_k == nullptr || c->table_dev == nullptr)
    return fail(TLS_ERR_UNSUPPORTED, "device planning needs K/V in mapped pinned host memory and device slots");
  const int64_t entries = (int64_t)c->rows * K_b;
  if (c->n_slots > kPlanMaxSlots || entries > kPlanMaxEntries)
    return fail(TLS_ERR_UNSUPPORTED, "device planning takes at most %d slots and %d list entries", kPlanMaxSlots,
                kPlanMaxEntries);
  const size_t smem = plan_smem(c->n_slots, (int)entries).total;
  if (smem > kMaxDynSmem)
    return fail(TLS_ERR_UNSUPPORTED, "device planning of %d slots and %lld list entries needs %zu bytes of shared "
                "memory (at most %zu)", c->n_slots, (long long)entries, smem, kMaxDynSmem);
  cudaError_t e = cudaSuccess;
  if (c->owner_dev == nullptr) {
    e = cudaMalloc((void**)&c->owner_dev, (size_t)c->n_slots * sizeof(int64_t));
    if (e == cudaSuccess) e = cudaMalloc((void**)&c->last_use_dev, (size_t)c->n_slots * sizeof(int64_t));
    if (e == cudaSuccess) e = cudaMalloc((void**)&c->n_jobs_dev, sizeof(int32_t));
    if (e == cudaSuccess)
      e = cudaHostAlloc((void**)&c->dev_failed, sizeof(int32_t), cudaHostAllocMapped | cudaHostAllocPortable);
    if (e == cudaSuccess) *c->dev_failed = 0;
    if (e == cudaSuccess) e = cudaHostGetDevicePointer((void**)&c->dev_failed_dptr, c->dev_failed, 0);
  }
  if (e == cudaSuccess && entries > c->max_entries) {
    if (c->jobs_dev != nullptr) cudaFree(c->jobs_dev);
    c->jobs_dev = nullptr;
    e = cudaMalloc((void**)&c->jobs_dev, (size_t)entries * sizeof(int4));
    if (e == cudaSuccess) c->max_entries = (int)entries;
  }
  if (e == cudaSuccess && !c->device_owned) {
    e = cudaDeviceSynchronize();  // queued host-planned transfers land first
    if (e == cudaSuccess)
      e = cudaMemcpy(c->table_dev, c->table.data(), c->table.size() * sizeof(int32_t), cudaMemcpyHostToDevice);
    if (e == cudaSuccess)
      e = cudaMemcpy(c->owner_dev, c->owner.data(), c->owner.size() * sizeof(int64_t), cudaMemcpyHostToDevice);
    if (e == cudaSuccess)
      e = cudaMemcpy(c->last_use_dev, c->last_use.data(), c->last_use.size() * sizeof(int64_t),
                     cudaMemcpyHostToDevice);
    if (e == cudaSuccess) {
      c->device_owned = true;
      c->published = true;
    }
  }
  if (e != cudaSuccess) return cuda_check(e, "block cache: device planning state");
  return TLS_OK;
}

// The cache's status: a failed transfer or device plan (sticky).
tls_status block_cache_check(tls_block_cache* c) { return device_plan_status(*c); }

// Bytes one block occupies in the pool (K and, when the cache has them, V rows).
int64_t block_cache_block_bytes(const tls_block_cache* c) {
  const int64_t kblk = (int64_t)c->shape.block_size * c->hk_stride * 2;
  const int64_t vblk = (int64_t)c->shape.block_size * c->hv_stride * 2;
  return kblk + (c->host_v != nullptr && c->slot_v != nullptr ? vblk : 0);
}

// The incremental prefetch planned on the device: one plan kernel (one CTA)
// reads M_t (and M_{t-1}) from device memory and updates the slot table, the
// owners and the last uses; a pull kernel copies its jobs.  keep_prev: the
// slots the previous plan used are kept instead of those of in_use_dev (the
// engine, whose previous plan was for M_{t-1}: the plan then no longer reads
// M_{t-1}, and level 1 may overwrite it while the plan runs).  n_out (device
// or mapped memory, may be NULL) receives the number of copied blocks, or -1
// when the plan failed (the cache is failed from then on).
tls_status prefetch_device_impl(tls_block_cache* c, const int32_t* new_dev, const int32_t* in_use_dev, int K_b,
                                cudaStream_t cs, int32_t* n_out, bool keep_prev) {
  tls_status st = device_plan_status(*c);
  if (st != TLS_OK) return st;
  if (fault_injected_copy()) return fail(TLS_ERR_COPY, "prefetch_diff: copy failure injected (TLS_FAULT_INJECT=copy)");
  st = block_cache_device_ready(c, K_b);
  if (st != TLS_OK) return st;
  c->step += 1;
  PlanParams p;
  p.table = c->table_dev;
  p.owner = c->owner_dev;
  p.last_use = c->last_use_dev;
  p.new_idx = new_dev;
  p.in_use = keep_prev ? nullptr : in_use_dev;
  p.keep_prev = keep_prev ? 1 : 0;
  p.rows = c->rows;
  p.nb = c->nb;
  p.K_b = K_b;
  p.n_slots = c->n_slots;
  p.bs = c->shape.block_size;
  p.ctx_len = c->shape.ctx_len;
  p.step = c->step;
  p.jobs = c->jobs_dev;
  p.n_jobs = c->n_jobs_dev;
  p.n_out = n_out;
  p.failed = c->dev_failed_dptr;
  const size_t smem = plan_smem(c->n_slots, c->rows * K_b).total;
  cudaError_t e = kernel_attrs((const void*)block_plan_kernel, smem);
  if (e != cudaSuccess) return cuda_check(e, "prefetch_diff_device: plan kernel setup");
  block_plan_kernel<<<1, kPlanThreads, smem, cs>>>(p);
  e = cudaGetLastError();
  const int64_t kblk = (int64_t)c->shape.block_size * c->hk_stride * 2;
  const int64_t vblk = (int64_t)c->shape.block_size * c->hv_stride * 2;
  const bool with_v = c->host_v != nullptr && c->slot_v != nullptr;
  // one CTA an SM at most: the grid becomes resident while the plan kernel
  // still runs (programmatic launch), beside the step's other kernels
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((int64_t)c->rows * K_b, (int64_t)kNumSMs));
  if (e == cudaSuccess)
    e = launch_ex(block_pull_jobs_kernel, dim3(grid), dim3(kPullThreads), 0, cs, /*pdl=*/true, 0u,
                  (const uint8_t*)c->dev_host_k, (const uint8_t*)(with_v ? c->dev_host_v : nullptr), c->slot_k,
                  (uint8_t*)(with_v ? c->slot_v : nullptr), kblk, vblk, c->hk_stride * 2, c->hv_stride * 2,
                  (const int4*)c->jobs_dev, (const int32_t*)c->n_jobs_dev);
  if (e != cudaSuccess) {
    c->failed = TLS_ERR_COPY;
    return fail(TLS_ERR_COPY, "prefetch_diff_device: launch failed: %s", cudaGetErrorString(e));
  }
  return TLS_OK;
}

// The incremental prefetch of tls_prefetch_diff without the argument checks
// (also used by the staggered engine).  *bytes = host -> device bytes of the
// block copies.
tls_status prefetch_diff_impl(tls_block_cache* c, const int32_t* new_idx, const int32_t* in_use, int K_b,
                              cudaStream_t cs, int32_t* n_copied, int64_t* bytes) {
  tls_status st = device_plan_status(*c);
  if (st != TLS_OK) return st;
  if (fault_injected_copy()) return fail(TLS_ERR_COPY, "prefetch_diff: copy failure injected (TLS_FAULT_INJECT=copy)");
  st = sync_host_mirror(*c);
  if (st != TLS_OK) return st;
  std::vector<Copy> copies;
  std::vector<int32_t> victims;
  st = plan(*c, new_idx, in_use, K_b, &copies, &victims);
  if (st != TLS_OK) return st;
  std::vector<int2> changes;
  assign_slots(*c, copies, victims, &changes);

  const int bs = c->shape.block_size;
  const int64_t n = c->shape.ctx_len;
  const size_t kblk = (size_t)bs * c->hk_stride * 2, vblk = (size_t)bs * c->hv_stride * 2;
  const bool with_v = c->host_v != nullptr && c->slot_v != nullptr;
  const int b = c->cur;
  // the staging buffers' previous use is done
  st = wait_event_deadline(c->staged[b], host_wait_ms(), "prefetch_diff: staging buffers");
  if (st != TLS_OK) return st;
  cudaError_t e = cudaSuccess;
  // from here on device work is queued: a failure leaves the cache failed
  auto queue_failed = [&](const char* what, cudaError_t err) {
    c->failed = TLS_ERR_COPY;
    return fail(TLS_ERR_COPY, "prefetch_diff: %s: %s", what, cudaGetErrorString(err));
  };
  // the first transfer publishes the whole table (nothing is resident, so nothing reads it)
  const bool first = !c->published;
  if (first) {
    std::memcpy(c->staging[b], c->table.data(), c->table.size() * sizeof(int32_t));
    for (const int2& ch : changes) c->staging[b][ch.x] = ch.y;
    e = cudaMemcpyAsync(c->table_dev, c->staging[b], c->table.size() * sizeof(int32_t), cudaMemcpyHostToDevice, cs);
    if (e != cudaSuccess) return queue_failed("slot table copy failed", e);
  }
  const int n_pairs = first ? 0 : (int)changes.size();
  if (c->dev_host_k != nullptr) {
    // one kernel pulls every planned block over PCIe and applies the table changes
    int4* jobs = c->jobs[b];
    for (size_t i = 0; i < copies.size(); ++i) {
      const int64_t tok0 = (int64_t)copies[i].row * n + (int64_t)copies[i].block * bs;
      jobs[i] = make_int4((int)(uint32_t)(tok0 & 0xFFFFFFFF), (int)(tok0 >> 32), copies[i].slot, 0);
    }
    int2* pairs = first ? nullptr : reinterpret_cast<int2*>(c->staging[b]);
    if (pairs != nullptr) std::memcpy(pairs, changes.data(), (size_t)n_pairs * sizeof(int2));
    const int grid = copies.empty() ? 1 : (int)copies.size();
    if (!copies.empty() || n_pairs > 0) {
      block_pull_kernel<<<grid, kPullThreads, 0, cs>>>(c->dev_host_k, with_v ? c->dev_host_v : nullptr, c->slot_k,
                                                        with_v ? c->slot_v : nullptr, (int64_t)kblk, (int64_t)vblk,
                                                        c->hk_stride * 2, c->hv_stride * 2, jobs,
                                                        (int)copies.size(), c->table_dev, pairs, n_pairs);
      e = cudaGetLastError();
      if (e != cudaSuccess) return queue_failed("pull kernel launch failed", e);
    }
  } else {
    // one cudaMemcpyAsync per run of blocks adjacent in host memory and in the pool
    size_t i = 0;
    while (i < copies.size()) {
      size_t j = i + 1;
      while (j < copies.size() && copies[j].row == copies[i].row &&
             copies[j].block == copies[j - 1].block + 1 && copies[j].slot == copies[j - 1].slot + 1)
        ++j;
      const size_t len = j - i;
      const int64_t tok0 = (int64_t)copies[i].row * n + (int64_t)copies[i].block * bs;
      e = cudaMemcpyAsync(c->slot_k + (size_t)copies[i].slot * kblk, c->host_k + (size_t)tok0 * c->hk_stride * 2,
                          len * kblk, cudaMemcpyHostToDevice, cs);
      if (e == cudaSuccess && with_v)
        e = cudaMemcpyAsync(c->slot_v + (size_t)copies[i].slot * vblk, c->host_v + (size_t)tok0 * c->hv_stride * 2,
                            len * vblk, cudaMemcpyHostToDevice, cs);
      if (e != cudaSuccess) return queue_failed("block copy failed", e);
      i = j;
    }
    if (n_pairs > 0) {
      int2* pairs = reinterpret_cast<int2*>(c->staging[b]);
      std::memcpy(pairs, changes.data(), (size_t)n_pairs * sizeof(int2));
      slot_table_update_kernel<<<(n_pairs + 255) / 256, 256, 0, cs>>>(c->table_dev, pairs, n_pairs);
      e = cudaGetLastError();
      if (e != cudaSuccess) return queue_failed("table update launch failed", e);
    }
  }
  e = cudaEventRecord(c->staged[b], cs);
  if (e != cudaSuccess) return queue_failed("staging event", e);
  // everything is queued: the host mirror follows
  if (first) c->published = true;
  commit(*c, new_idx, K_b, copies);
  c->cur ^= 1;
  *n_copied = (int32_t)copies.size();
  if (bytes != nullptr) *bytes = (int64_t)copies.size() * (int64_t)(kblk + (with_v ? vblk : 0));
  return TLS_OK;
}

// The attention's view of the slot pool of a cache created with device buffers.
tls_status block_cache_view(const tls_block_cache* c, tls_kv_view* kv) {
  if (c->slot_k == nullptr || c->table_dev == nullptr || c->host_k == nullptr)
    return fail(TLS_ERR_INVALID_ARG, "block cache was created without device buffers");
  const bool own_v = c->shape.v_offset < 0;
  if (own_v && c->slot_v == nullptr) return fail(TLS_ERR_INVALID_ARG, "block cache has no V slots");
  kv->k = c->slot_k;
  kv->v = own_v ? c->slot_v : c->slot_k;
  kv->k_row_stride = c->hk_stride;
  kv->v_row_stride = own_v ? c->hv_stride : c->hk_stride;
  kv->slot_of_block = c->table_dev;
  kv->n_slots = c->n_slots;
  return TLS_OK;
}

}  // namespace tls

using namespace tls;

extern "C" tls_status tls_block_cache_create(const tls_shape* shape, const void* host_k, const void* host_v,
                                             int64_t host_k_row_stride, int64_t host_v_row_stride, int32_t n_slots,
                                             void* slot_k, void* slot_v, int32_t* slot_table_dev,
                                             tls_block_cache** out) {
  clear_error();
  tls_status st = check_shape(shape);
  if (st != TLS_OK) return st;
  if (out == nullptr) return fail(TLS_ERR_INVALID_ARG, "block_cache_create: out is NULL");
  if (n_slots < 1) return fail(TLS_ERR_INVALID_ARG, "block_cache_create: n_slots must be >= 1");
  if (host_k_row_stride < shape->qk_dim)
    return fail(TLS_ERR_INVALID_ARG, "block_cache_create: host_k_row_stride must be >= qk_dim");
  if (shape->v_offset < 0 && host_v != nullptr && host_v_row_stride < shape->v_dim)
    return fail(TLS_ERR_INVALID_ARG, "block_cache_create: host_v_row_stride must be >= v_dim");
  auto* c = new tls_block_cache();
  c->shape = *shape;
  c->rows = rows_of(*shape);
  c->nb = (int)n_blocks(*shape);
  c->host_k = (const uint8_t*)host_k;
  c->host_v = shape->v_offset < 0 ? (const uint8_t*)host_v : nullptr;
  c->hk_stride = host_k_row_stride;
  c->hv_stride = host_v_row_stride;
  c->n_slots = n_slots;
  c->slot_k = (uint8_t*)slot_k;
  c->slot_v = (uint8_t*)slot_v;
  c->table_dev = slot_table_dev;
  c->table.assign((size_t)c->rows * c->nb, -1);
  c->owner.assign(n_slots, -1);
  c->last_use.assign(n_slots, 0);
  if (slot_table_dev != nullptr && host_k != nullptr && slot_k != nullptr) {
    // the pull path needs 16-byte-aligned rows and both tensors mapped
    const size_t tokens = (size_t)c->rows * (size_t)shape->ctx_len;
    const bool aligned = aligned16(host_k) && host_k_row_stride % 8 == 0 &&
                         (c->host_v == nullptr || (aligned16(host_v) && host_v_row_stride % 8 == 0));
    const uint8_t* dk = aligned ? mapped_host_range(host_k, tokens * (size_t)host_k_row_stride * 2) : nullptr;
    const uint8_t* dv =
        (dk != nullptr && c->host_v != nullptr) ? mapped_host_range(host_v, tokens * (size_t)host_v_row_stride * 2)
                                                : nullptr;
    if (dk != nullptr && (c->host_v == nullptr || dv != nullptr)) {
      cudaError_t e = cudaSuccess;
      for (int i = 0; i < 2 && e == cudaSuccess; ++i)
        e = cudaHostAlloc((void**)&c->jobs[i], (size_t)n_slots * sizeof(int4), cudaHostAllocMapped | cudaHostAllocPortable);
      if (e != cudaSuccess) {
        tls_block_cache_destroy(c);
        return cuda_check(e, "block_cache_create: pinned job lists");
      }
      c->dev_host_k = dk;
      c->dev_host_v = dv;
    }
  }
  if (slot_table_dev != nullptr) {
    // a plan changes at most two entries per copied block and copies at most n_slots blocks
    const size_t words = std::max(c->table.size(), (size_t)4 * (size_t)n_slots);
    for (int i = 0; i < 2; ++i) {
      cudaError_t e = cudaHostAlloc((void**)&c->staging[i], words * sizeof(int32_t),
                                    cudaHostAllocMapped | cudaHostAllocPortable);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->staged[i], cudaEventDisableTiming);
      if (e != cudaSuccess) {
        tls_block_cache_destroy(c);
        return cuda_check(e, "block_cache_create: pinned staging");
      }
    }
  }
  *out = c;
  return TLS_OK;
}

extern "C" void tls_block_cache_destroy(tls_block_cache* c) {
  if (c == nullptr) return;
  for (int i = 0; i < 2; ++i) {
    if (c->staged[i] != nullptr) {
      cudaEventSynchronize(c->staged[i]);
      cudaEventDestroy(c->staged[i]);
    }
    if (c->staging[i] != nullptr) cudaFreeHost(c->staging[i]);
    if (c->jobs[i] != nullptr) cudaFreeHost(c->jobs[i]);
  }
  if (c->owner_dev != nullptr) {
    cudaDeviceSynchronize();  // no plan or pull kernel may still use the arrays
    cudaFree(c->owner_dev);
    cudaFree(c->last_use_dev);
    cudaFree(c->n_jobs_dev);
    cudaFreeHost(c->dev_failed);
  }
  if (c->jobs_dev != nullptr) cudaFree(c->jobs_dev);
  delete c;
}

extern "C" tls_status tls_block_cache_plan(tls_block_cache* c, const int32_t* new_block_idx,
                                           const int32_t* in_use_block_idx, int32_t K_b, int32_t* copy_row,
                                           int32_t* copy_block, int32_t* copy_slot, int32_t* n_copy) {
  NvtxRange nvtx_range("tls_block_cache_plan");
  clear_error();
  if (c == nullptr || new_block_idx == nullptr || n_copy == nullptr)
    return fail(TLS_ERR_INVALID_ARG, "block_cache_plan: NULL argument");
  if (K_b < 1 || K_b > c->nb) return fail(TLS_ERR_INVALID_ARG, "block_cache_plan: K_b out of range");
  tls_status st = device_plan_status(*c);
  if (st != TLS_OK) return st;
  st = sync_host_mirror(*c);
  if (st != TLS_OK) return st;
  std::vector<Copy> copies;
  std::vector<int32_t> victims;
  st = plan(*c, new_block_idx, in_use_block_idx, K_b, &copies, &victims);
  if (st != TLS_OK) return st;
  std::vector<int2> changes;
  assign_slots(*c, copies, victims, &changes);
  commit(*c, new_block_idx, K_b, copies);
  for (size_t i = 0; i < copies.size(); ++i) {
    if (copy_row) copy_row[i] = copies[i].row;
    if (copy_block) copy_block[i] = copies[i].block;
    if (copy_slot) copy_slot[i] = copies[i].slot;
  }
  *n_copy = (int32_t)copies.size();
  return TLS_OK;
}

extern "C" tls_status tls_prefetch_diff(tls_block_cache* c, const int32_t* new_block_idx_host,
                                        const int32_t* in_use_block_idx_host, int32_t K_b, void* copy_stream,
                                        void* done_event, int32_t* n_copied) {
  NvtxRange nvtx_range("tls_prefetch_diff");
  clear_error();
  if (c == nullptr || new_block_idx_host == nullptr || n_copied == nullptr)
    return fail(TLS_ERR_INVALID_ARG, "prefetch_diff: NULL argument");
  if (c->host_k == nullptr || c->slot_k == nullptr || c->table_dev == nullptr)
    return fail(TLS_ERR_INVALID_ARG, "prefetch_diff: cache was created without device buffers");
  if (K_b < 1 || K_b > c->nb) return fail(TLS_ERR_INVALID_ARG, "prefetch_diff: K_b out of range");
  tls_status st = prefetch_diff_impl(c, new_block_idx_host, in_use_block_idx_host, K_b, (cudaStream_t)copy_stream,
                                     n_copied, nullptr);
  if (st != TLS_OK || done_event == nullptr) return st;
  cudaError_t e = cudaEventRecord((cudaEvent_t)done_event, (cudaStream_t)copy_stream);
  return e == cudaSuccess ? TLS_OK : cuda_check(e, "prefetch_diff: done event");
}

extern "C" tls_status tls_block_cache_table(const tls_block_cache* c, int32_t* table) {
  clear_error();
  if (c == nullptr || table == nullptr) return fail(TLS_ERR_INVALID_ARG, "block_cache_table: NULL argument");
  if (c->device_owned) {
    // the device table is the state: read it once the queued work is done
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess)
      e = cudaMemcpy(table, c->table_dev, c->table.size() * sizeof(int32_t), cudaMemcpyDeviceToHost);
    return e == cudaSuccess ? TLS_OK : cuda_check(e, "block_cache_table: reading the device table");
  }
  std::memcpy(table, c->table.data(), c->table.size() * sizeof(int32_t));
  return TLS_OK;
}

extern "C" tls_status tls_prefetch_diff_device(tls_block_cache* c, const int32_t* new_block_idx_dev,
                                               const int32_t* in_use_block_idx_dev, int32_t K_b, void* copy_stream,
                                               void* done_event, int32_t* n_copied_dev) {
  NvtxRange nvtx_range("tls_prefetch_diff_device");
  clear_error();
  if (c == nullptr || new_block_idx_dev == nullptr) return fail(TLS_ERR_INVALID_ARG, "prefetch_diff_device: NULL argument");
  if (K_b < 1 || K_b > c->nb) return fail(TLS_ERR_INVALID_ARG, "prefetch_diff_device: K_b out of range");
  tls_status st = prefetch_device_impl(c, new_block_idx_dev, in_use_block_idx_dev, K_b, (cudaStream_t)copy_stream,
                                       n_copied_dev, /*keep_prev=*/false);
  if (st != TLS_OK || done_event == nullptr) return st;
  cudaError_t e = cudaEventRecord((cudaEvent_t)done_event, (cudaStream_t)copy_stream);
  return e == cudaSuccess ? TLS_OK : cuda_check(e, "prefetch_diff_device: done event");
}
