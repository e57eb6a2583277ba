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
__device__ __forceinline__ uint32_t float_key(float f) {
  if (f != f) f = -INFINITY;
  if (f == 0.0f) f = 0.0f;
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ----------------------------------------------------------------------------
// Block-wide exclusive scan of one int per thread.  `scratch` holds >= 33 ints.
// Returns the exclusive prefix; *total receives the sum over the block.
// ----------------------------------------------------------------------------
template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int v, int* scratch, int* total) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < NW ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < NW) scratch[lane] = w;  // inclusive warp totals
    if (lane == NW - 1) scratch[32] = w;
  }
  __syncthreads();
  int before = (warp > 0 ? scratch[warp - 1] : 0) + x - v;
  *total = scratch[32];
  __syncthreads();
  return before;
}

// ----------------------------------------------------------------------------
// CTA-wide deterministic top-k.
//
// keys[0..n) (shared memory) hold float_key(score).  Selects the k largest
// keys, ties broken towards the lower position, and writes
// out[j] = map(position) for the selected positions in ascending order.
// Radix select (four 8-bit digits, most significant first) finds the k-th
// largest key tau and how many of the keys equal to tau to take; one
// index-ordered scan then marks the selection and a second one compacts it.
// ----------------------------------------------------------------------------
struct TopkScratch {
  int hist[256];
  int scan[33];
  uint32_t prefix;
  int need;  // how many more keys must be taken at the current prefix
};

template <int NT, typename MapFn>
__device__ void cta_topk_ascending(const uint32_t* keys, int n, int k, int* out, TopkScratch& sm,
                                   MapFn map) {
  const int tid = threadIdx.x;
  if (tid == 0) {
    sm.prefix = 0;
    sm.need = k;
  }
  uint32_t mask = 0;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += NT) sm.hist[i] = 0;
    __syncthreads();
    const uint32_t prefix = sm.prefix;
    for (int i = tid; i < n; i += NT) {
      uint32_t key = keys[i];
      if ((key & mask) == prefix) atomicAdd(&sm.hist[(key >> shift) & 255u], 1);
    }
    __syncthreads();
    if (tid < 32) {
      // lane L owns digits [248 - 8L, 255 - 8L] (lane 0 holds the largest)
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
        int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += y;
      }
      const int need = sm.need;
      int above = incl - s;  // keys in digits larger than this lane's range
      bool mine = (above < need) && (incl >= need);
      unsigned ballot = __ballot_sync(0xffffffffu, mine);
      if (mine) {
        int d = 0;
        for (; d < 8; ++d) {
          if (above + local[d] >= need) break;
          above += local[d];
        }
        uint32_t digit = 255u - (uint32_t)(tid * 8 + d);
        sm.prefix = prefix | (digit << shift);
        sm.need = need - above;
      }
      (void)ballot;
    }
    mask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t tau = sm.prefix;
  const int take_eq = sm.need;  // keys equal to tau to take, lowest positions first

  // contiguous chunk per thread keeps the scans in position order
  const int per = (n + NT - 1) / NT;
  const int lo = min(n, tid * per), hi = min(n, lo + per);
  int eq = 0;
  for (int i = lo; i < hi; ++i) eq += (keys[i] == tau);
  int total;
  int eq_before = block_exclusive_scan<NT>(eq, sm.scan, &total);
  int sel = 0;
  {
    int e = eq_before;
    for (int i = lo; i < hi; ++i) {
      uint32_t key = keys[i];
      if (key > tau) ++sel;
      else if (key == tau) { if (e < take_eq) ++sel; ++e; }
    }
  }
  int pos = block_exclusive_scan<NT>(sel, sm.scan, &total);
  {
    int e = eq_before;
    for (int i = lo; i < hi; ++i) {
      uint32_t key = keys[i];
      bool take = false;
      if (key > tau) take = true;
      else if (key == tau) { take = e < take_eq; ++e; }
      if (take && pos < k) out[pos++] = map(i);
    }
  }
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

// Instruction descriptor: kind::f16, bf16 x bf16 -> f32, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4)                      // D format f32
         | (1u << 7)                    // A format bf16
         | (1u << 10)                   // B format bf16
         | ((uint32_t)(N >> 3) << 17)   // N / 8
         | ((uint32_t)(M >> 4) << 24);  // M / 16
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
