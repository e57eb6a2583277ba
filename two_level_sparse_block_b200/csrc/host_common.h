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
#include <nvtx3/nvToolsExt.h>

namespace tls {

// An NVTX range around one library call, named for the entry point (seen by
// Nsight Systems and other NVTX tools; a few nanoseconds without a tool).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Sets the thread-local error message and returns `st`.
tls_status fail(tls_status st, const char* fmt, ...);
void clear_error();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Validates the fields every call depends on.
tls_status check_shape(const tls_shape* s);

inline int64_t n_blocks(const tls_shape& s) { return s.ctx_len / s.block_size; }
// Largest candidate count of level 2 (K_b * bs) and list length of the attention.
constexpr int64_t kMaxCandidates = (int64_t)1 << 19;
constexpr int64_t kMaxListLen = (int64_t)1 << 24;
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

// Host waits with a deadline.  wait_event_deadline polls cudaEventQuery,
// yielding the thread between polls, until the event has completed
// (TLS_OK), the runtime reports an error (TLS_ERR_CUDA) or timeout_ms have
// passed (TLS_ERR_TIMEOUT; the device work it waited for keeps running and
// completes on its own).  host_wait_ms: the deadline the library's host waits
// use, TLS_HOST_WAIT_MS from the environment when set (> 0), else 10 s.
tls_status wait_event_deadline(cudaEvent_t ev, double timeout_ms, const char* what);
double host_wait_ms();

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
constexpr size_t kMaxDynSmem = 227 * 1024;  // dynamic shared memory a CTA may opt into

// Where entry t of a row's attention list comes from: the token list
// (token_idx), every position in order (t itself: full attention), or the
// tokens of a block list in order (blocks[t / bs] * bs + t % bs: block
// selection alone).
enum { kListTokens = 0, kListAll = 1, kListBlocks = 2 };

// The launch paths behind the entry points (arguments already checked).
// Level 1: scores and top-K_b of every row into block_idx.
tls_status select_blocks_impl(const tls_shape& s, const void* q, const void* meta, int K_b, int32_t* block_idx,
                              float* block_score, uint8_t* ws, const WsLayout& L, cudaStream_t stream);
// Level 2 within block_idx (NULL: every block, K_b = NB).  `lean`: on at most
// half the SMs (beside a level-1 grid); `pdl`: launched as a programmatic
// dependent of the stream's preceding kernel.
tls_status select_tokens_impl(const tls_shape& s, const void* q, const int32_t* label_ch, const uint8_t* codes,
                              const float* scales, const int32_t* block_idx, int K_b, int k, int32_t* token_idx,
                              float* token_score, uint8_t* ws, const WsLayout& L, cudaStream_t stream,
                              bool pdl = false, bool lean = false);
// Attention over k list entries per row; list_mode 0: token_idx, 1: every
// position (full attention), 2: the tokens of the block list `blocks` [rows, K_b].
tls_status sparse_attn_impl(const tls_shape& s, const void* q, const tls_kv_view& kv, const int32_t* token_idx,
                            int k, int out_dtype, void* out, float* lse, uint8_t* ws, const WsLayout& L,
                            cudaStream_t stream, bool pdl = true, int list_mode = 0, const int32_t* blocks = nullptr,
                            int K_b = 0);

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
// should not pay the driver calls each time.  Every kernel also prefers the
// largest shared-memory carve-out: an SM configured for a kernel with little
// shared memory cannot take a CTA of a concurrent kernel that needs more (the
// staggered step runs level 1 beside level 2), and none of these kernels
// keeps data in L1.
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
  struct Set {
    size_t smem = 0;
    bool nonportable = false, carveout = false;
  };
  static std::unordered_map<Key, Set, KeyHash> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  Set& d = done[Key{fn, dev}];
  if (!d.carveout) {
    e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    d.carveout = true;
  }
  if (smem_bytes > d.smem) {
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes);
    if (e != cudaSuccess) return e;
    d.smem = smem_bytes;
  }
  if (nonportable_cluster && !d.nonportable) {
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    d.nonportable = true;
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
