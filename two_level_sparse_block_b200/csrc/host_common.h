// Host-side helpers shared by the libtls entry points.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>
#include <unordered_map>

#include "tls.h"

namespace tls {

// Sets the thread-local error message and returns `st`.
tls_status fail(tls_status st, const char* fmt, ...);
void clear_error();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Validates the fields every call depends on.
tls_status check_shape(const tls_shape* s);

inline int64_t n_blocks(const tls_shape& s) { return s.ctx_len / s.block_size; }
inline int rows_of(const tls_shape& s) { return s.batch * s.n_kv_heads; }
inline int group_of(const tls_shape& s) { return s.n_q_heads / s.n_kv_heads; }
// Heads of a KV group padded to the level-1 GEMM's N (16, 32, 64, 128 or 256).
inline int block_score_npad(int g) { return g <= 16 ? 16 : g <= 32 ? 32 : g <= 64 ? 64 : g <= 128 ? 128 : 256; }

inline tls_status cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return TLS_OK;
  return fail(TLS_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Launch-time error (configuration or earlier sticky error).
inline tls_status launch_check(const char* what) { return cuda_check(cudaGetLastError(), what); }

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace layout shared by the selection and attention entry points.
struct WsLayout {
  size_t err;          // int[64] header: error word, location word
  size_t blk_counter;  // unsigned[rows]
  size_t tok_counter;  // unsigned[rows]
  size_t att_counter;  // unsigned[rows]
  size_t agg;          // float[rows * NB]
  size_t qprime;       // bf16[rows * NPAD * 2 * Dqk] when NPAD >= 64 (level-1 B operand), else empty
  size_t tscore;       // float[rows * K_b * bs]
  size_t partial;      // float[rows * G * splits * (Dv + 2)]
  size_t total;
  int splits;          // attention split count along the token list
  int head_groups;     // attention CTAs along the heads of a group
  int heads_per_cta;
  int tokens_per_split;
  int tiles_per_pair, n_items, n_ctas;  // mma attention: chunks per (virtual) row, items, persistent CTAs
};

// Device address of the scratch-free entry point's static array on the
// current device and context (looked up once per device and context).
tls_status noalloc_scratch(void** out);

// Plans the attention launch and the workspace for (shape, K_b, k).
tls_status plan_workspace(const tls_shape& s, int K_b, int k, WsLayout* out);

constexpr int kNumSMs = 148;

// Launches `kernel` with programmatic stream serialization: it may start while
// the preceding kernel of the stream finishes, and must call
// griddepcontrol.wait (grid_dependency_wait) before touching that kernel's
// outputs.  Hides the launch gap between dependent kernels of one step.
// cudaLaunchKernelEx with optional programmatic dependent launch (the grid
// may start before the preceding kernel of the stream ends; it calls
// griddepcontrol.wait before reading that kernel's output) and optional
// thread-block clusters of cluster_x CTAs along x (cluster_x <= 1: none).
// The level-2 kernel a call takes (token_select.cu decides it).
struct TokenDispatch {
  enum Kind { kRow, kCluster, kChunked } kind;
  const char* name;  // static string
  int cl;            // CTAs per row (a cluster when > 1)
  int threads;       // threads per CTA
};
TokenDispatch token_dispatch(const tls_shape& s, int K_b, bool lean, bool aligned);

// cudaFuncSetAttribute once per kernel, device and value (the dynamic shared
// memory limit only ever rises): a launch path that runs every decode step
// should not pay the driver calls each time.
inline cudaError_t kernel_attrs(const void* fn, size_t smem_bytes, bool nonportable_cluster = false) {
  struct Key {
    const void* fn;
    int dev;
    bool operator==(const Key& o) const { return fn == o.fn && dev == o.dev; }
  };
  struct KeyHash {
    size_t operator()(const Key& k) const { return std::hash<const void*>()(k.fn) * 31u + (size_t)k.dev; }
  };
  static std::mutex mu;
  static std::unordered_map<Key, std::pair<size_t, bool>, KeyHash> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  auto& d = done[Key{fn, dev}];
  if (smem_bytes > d.first) {
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes);
    if (e != cudaSuccess) return e;
    d.first = smem_bytes;
  }
  if (nonportable_cluster && !d.second) {
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    d.second = true;
  }
  return cudaSuccess;
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                             bool pdl, unsigned cluster_x, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// A kernel whose CTAs form clusters of cluster_x along x (no PDL).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                                  unsigned cluster_x, Args... args) {
  return launch_ex(kernel, grid, block, smem, stream, false, cluster_x, args...);
}

}  // namespace tls
