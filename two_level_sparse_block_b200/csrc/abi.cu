// C-ABI entry points of libtls for the per-step path, argument validation and
// the workspace plan.  Kernels live in block_select.cu, token_select.cu and
// decode_attn.cu; the index build in index_build.cu; the block cache and
// incremental prefetch in block_cache.cu.

#include <chrono>
#include <cstdlib>
#include <cstring>
#include <thread>

#include "host_common.h"
#include "token_common.cuh"

namespace tls {

int attn_heads_per_cta(const tls_shape& s);
bool attn_mma_supported(const tls_shape& s);
int attn_mma_plan(int rows, int k, int* chunks_per_row, int* n_items, int* n_ctas);
int attn_mma_cluster_size(int rows, int hpc);
bool attn_mla_supported(const tls_shape& s);
int attn_mla_tokens_per_split(int k);

namespace {
thread_local char g_err[512] = {0};
}

tls_status fail(tls_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

void clear_error() { g_err[0] = 0; }

tls_status wait_event_deadline(cudaEvent_t ev, double timeout_ms, const char* what) {
  const auto t0 = std::chrono::steady_clock::now();
  for (;;) {
    const cudaError_t e = cudaEventQuery(ev);
    if (e == cudaSuccess) return TLS_OK;
    if (e != cudaErrorNotReady) return cuda_check(e, what);
    const double ms = std::chrono::duration<double, std::milli>(std::chrono::steady_clock::now() - t0).count();
    if (ms > timeout_ms) return fail(TLS_ERR_TIMEOUT, "%s: no completion within %.0f ms", what, timeout_ms);
    std::this_thread::yield();
  }
}

double host_wait_ms() {
  const char* v = std::getenv("TLS_HOST_WAIT_MS");
  if (v != nullptr) {
    const double x = std::atof(v);
    if (x > 0.0) return x;
  }
  return 10000.0;
}

tls_status check_shape(const tls_shape* p) {
  if (p == nullptr) return fail(TLS_ERR_INVALID_ARG, "shape is NULL");
  const tls_shape& s = *p;
  if (s.batch < 1 || s.n_kv_heads < 1 || s.n_q_heads < 1 || s.n_q_heads % s.n_kv_heads != 0)
    return fail(TLS_ERR_INVALID_ARG, "bad heads/batch: B=%d Hq=%d Hkv=%d", s.batch, s.n_q_heads, s.n_kv_heads);
  if (s.qk_dim < 32 || s.qk_dim % 32 != 0 || s.qk_dim > 640)
    return fail(TLS_ERR_INVALID_ARG, "qk_dim %d must be a multiple of 32 in [32, 640]", s.qk_dim);
  if (s.v_dim < 8 || s.v_dim % 8 != 0 || s.v_dim > 512)
    return fail(TLS_ERR_INVALID_ARG, "v_dim %d must be a multiple of 8 in [8, 512]", s.v_dim);
  if (s.v_offset >= 0 && (s.v_offset % 8 != 0 || s.v_offset + s.v_dim > s.qk_dim))
    return fail(TLS_ERR_INVALID_ARG, "v_offset %d: V slice must be 8-aligned and inside the K row", s.v_offset);
  if (s.v_offset < -1) return fail(TLS_ERR_INVALID_ARG, "v_offset must be -1 or >= 0");
  if (s.block_size < 8 || s.block_size > 256 || s.block_size % 8 != 0)
    return fail(TLS_ERR_INVALID_ARG, "block_size %d must be a multiple of 8 in [8, 256]", s.block_size);
  if (s.n_label < 2 || s.n_label > 64 || s.n_label % 2 != 0 || s.n_label > s.qk_dim)
    return fail(TLS_ERR_INVALID_ARG, "n_label %d must be even, in [2, 64] and <= qk_dim", s.n_label);
  if (s.ctx_len < s.block_size || s.ctx_len % s.block_size != 0)
    return fail(TLS_ERR_INVALID_ARG, "ctx_len %lld must be a positive multiple of block_size",
                (long long)s.ctx_len);
  if (s.ctx_len > (int64_t)1 << 31) return fail(TLS_ERR_INVALID_ARG, "ctx_len above 2^31");
  if (!(s.softmax_scale > 0.0f)) return fail(TLS_ERR_INVALID_ARG, "softmax_scale must be > 0");
  return TLS_OK;
}

tls_status plan_workspace(const tls_shape& s, int K_b, int k, WsLayout* out) {
  const int rows = rows_of(s);
  const int64_t nb = n_blocks(s);
  const int g = group_of(s);
  if (K_b < 1 || K_b > nb) return fail(TLS_ERR_INVALID_ARG, "K_b %d must be in [1, NB=%lld]", K_b, (long long)nb);
  if (nb > 16384) return fail(TLS_ERR_UNSUPPORTED, "NB %lld above 16384", (long long)nb);
  const int64_t n_cand = (int64_t)K_b * s.block_size;
  if (n_cand > kMaxListLen) return fail(TLS_ERR_UNSUPPORTED, "K_b*block_size %lld above %lld", (long long)n_cand,
                                        (long long)kMaxListLen);
  if (k < 1 || k > n_cand) return fail(TLS_ERR_INVALID_ARG, "k %d must be in [1, K_b*bs=%lld]", k, (long long)n_cand);
  WsLayout L;
  L.heads_per_cta = attn_heads_per_cta(s);
  L.head_groups = (g + L.heads_per_cta - 1) / L.heads_per_cta;
  L.tiles_per_pair = L.n_items = L.n_ctas = 0;
  if (attn_mma_supported(s)) {
    // warp-streaming attention: persistent CTAs over 16-token chunks
    L.tokens_per_split = 16;
    L.splits = attn_mma_plan(rows * L.head_groups, k, &L.tiles_per_pair, &L.n_items, &L.n_ctas);
  } else if (attn_mla_supported(s)) {
    // MLA: 8 token splits per (row, head block) merged inside a cluster; no workspace partials
    L.tokens_per_split = attn_mla_tokens_per_split(k);
    L.splits = 1;
  } else {
    const int target = 4 * kNumSMs;
    int splits = (target + rows * L.head_groups - 1) / (rows * L.head_groups);
    int max_splits = (k + 15) / 16;
    if (max_splits > 64) max_splits = 64;  // the split merge reads at most 64 splits
    if (splits > max_splits) splits = max_splits;
    if (splits < 1) splits = 1;
    int tps = (k + splits - 1) / splits;
    L.tokens_per_split = (int)align_up((size_t)tps, 8);
    L.splits = (k + L.tokens_per_split - 1) / L.tokens_per_split;
  }
  size_t off = 0;
  L.err = off;
  off += 256;
  L.blk_counter = off;
  off = align_up(off + (size_t)rows * 4, 256);
  L.tok_counter = off;
  off = align_up(off + (size_t)rows * 4, 256);
  L.att_counter = off;
  off = align_up(off + (size_t)rows * L.head_groups * 4, 256);
  if (L.splits > 64) return fail(TLS_ERR_UNSUPPORTED, "attention plan needs %d splits (> 64)", L.splits);
  // regions that depend on fewer arguments come first, so that the offsets
  // a call uses do not depend on arguments it is not given
  L.agg = off;
  off = align_up(off + (size_t)rows * nb * 4, 256);
  const int npad = block_score_npad(g);
  L.qprime = off;
  if (npad >= 64) off = align_up(off + (size_t)rows * npad * 2 * s.qk_dim * 2, 256);
  L.partial = off;
  off = align_up(off + (size_t)rows * g * L.splits * (s.v_dim + 2) * 4, 256);
  L.tscore = off;
  off = align_up(off + (size_t)rows * n_cand * 4, 256);
  L.total = off;
  *out = L;
  return TLS_OK;
}

static tls_status check_ws(const tls_shape& s, int K_b, int k, void* ws, size_t ws_bytes, WsLayout* L) {
  tls_status st = plan_workspace(s, K_b, k, L);
  if (st != TLS_OK) return st;
  if (ws == nullptr || !aligned16(ws)) return fail(TLS_ERR_INVALID_ARG, "workspace NULL or not 16-byte aligned");
  if (ws_bytes < L->total)
    return fail(TLS_ERR_INVALID_ARG, "workspace %zu bytes < required %zu", ws_bytes, L->total);
  return TLS_OK;
}

// Level 2 takes at most kMaxCandidates candidates per row.
static tls_status check_candidates(const tls_shape& s, int K_b) {
  const int64_t n_cand = (int64_t)K_b * s.block_size;
  if (n_cand > kMaxCandidates)
    return fail(TLS_ERR_UNSUPPORTED, "level 2 takes at most %lld candidates per row (K_b*bs = %lld)",
                (long long)kMaxCandidates, (long long)n_cand);
  return TLS_OK;
}

static tls_status check_kv(const tls_shape& s, const tls_kv_view* kv) {
  if (kv == nullptr || kv->k == nullptr) return fail(TLS_ERR_INVALID_ARG, "kv view or kv.k is NULL");
  if (!aligned16(kv->k)) return fail(TLS_ERR_INVALID_ARG, "kv.k must be 16-byte aligned");
  if (kv->k_row_stride < s.qk_dim || kv->k_row_stride % 8 != 0)
    return fail(TLS_ERR_INVALID_ARG, "kv.k_row_stride must be >= qk_dim and a multiple of 8");
  if (s.v_offset < 0) {
    if (kv->v == nullptr || !aligned16(kv->v)) return fail(TLS_ERR_INVALID_ARG, "kv.v NULL or not 16-byte aligned");
    if (kv->v_row_stride < s.v_dim || kv->v_row_stride % 8 != 0)
      return fail(TLS_ERR_INVALID_ARG, "kv.v_row_stride must be >= v_dim and a multiple of 8");
  }
  if (kv->slot_of_block != nullptr && kv->n_slots < 1)
    return fail(TLS_ERR_INVALID_ARG, "kv.n_slots must be >= 1 with a slot table");
  return TLS_OK;
}

}  // namespace tls

using namespace tls;

extern "C" const char* tls_last_error(void) { return g_err; }

extern "C" int32_t tls_version(void) { return 100; }

extern "C" const char* tls_attn_kernel(const tls_shape* shape) {
  if (check_shape(shape) != TLS_OK) return nullptr;
  if (attn_mma_supported(*shape)) {
    const int g = group_of(*shape), hpc = g < 16 ? g : 16, head_groups = (g + hpc - 1) / hpc;
    return attn_mma_cluster_size(rows_of(*shape) * head_groups, hpc) > 0 ? "sparse_attn_mma_cluster_kernel"
                                                                          : "sparse_attn_mma_kernel";
  }
  if (attn_mla_supported(*shape)) return "sparse_attn_mla_kernel";
  return "sparse_attn_kernel";
}

extern "C" const char* tls_token_kernel(const tls_shape* shape, int32_t K_b, int32_t k, int32_t staggered,
                                        int32_t* cluster_ctas, int32_t* cta_threads) {
  clear_error();
  if (check_shape(shape) != TLS_OK) return nullptr;
  WsLayout L;
  if (plan_workspace(*shape, K_b, k, &L) != TLS_OK) return nullptr;
  const TokenDispatch d = token_dispatch(*shape, K_b, staggered != 0, true);
  if (cluster_ctas != nullptr) *cluster_ctas = d.cl;
  if (cta_threads != nullptr) *cta_threads = d.threads;
  return d.name;
}

extern "C" size_t tls_workspace_bytes(const tls_shape* shape, int32_t K_b, int32_t k) {
  if (check_shape(shape) != TLS_OK) return 0;
  WsLayout L;
  if (plan_workspace(*shape, K_b, k, &L) != TLS_OK) return 0;
  return L.total;
}

extern "C" tls_status tls_workspace_error(const void* ws, int32_t clear, int32_t* code, void* stream) {
  clear_error();
  if (code == nullptr) return fail(TLS_ERR_INVALID_ARG, "workspace_error: NULL code");
  if (ws == nullptr) {
    // the scratch-free attention's array on the current device
    void* base = nullptr;
    tls_status st = noalloc_scratch(&base);
    if (st != TLS_OK) return st;
    ws = base;
  }
  int32_t words[2] = {0, 0};
  cudaStream_t cs = (cudaStream_t)stream;
  tls_status st = cuda_check(cudaMemcpyAsync(words, ws, sizeof(words), cudaMemcpyDeviceToHost, cs),
                             "workspace_error: copy");
  if (st != TLS_OK) return st;
  if (clear) {
    st = cuda_check(cudaMemsetAsync(const_cast<void*>(ws), 0, sizeof(words), cs), "workspace_error: clear");
    if (st != TLS_OK) return st;
  }
  st = cuda_check(cudaStreamSynchronize(cs), "workspace_error: sync");
  if (st != TLS_OK) return st;
  *code = words[0];
  if (words[0] != 0) fail((tls_status)words[0], "kernel error %d at site %d", words[0], words[1]);
  return TLS_OK;
}

extern "C" tls_status tls_select_blocks(const tls_shape* shape, const void* q, const void* meta, int32_t K_b,
                                        int32_t* block_idx, float* block_score, void* ws, size_t ws_bytes,
                                        void* stream) {
  NvtxRange nvtx_range("tls_select_blocks");
  clear_error();
  tls_status st = check_shape(shape);
  if (st != TLS_OK) return st;
  if (q == nullptr || meta == nullptr || block_idx == nullptr)
    return fail(TLS_ERR_INVALID_ARG, "select_blocks: null pointer");
  if (!aligned16(q) || !aligned16(meta)) return fail(TLS_ERR_INVALID_ARG, "select_blocks: q/meta not 16-byte aligned");
  WsLayout L;
  st = check_ws(*shape, K_b, 1, ws, ws_bytes, &L);
  if (st != TLS_OK) return st;
  return select_blocks_impl(*shape, q, meta, K_b, block_idx, block_score, (uint8_t*)ws, L, (cudaStream_t)stream);
}

extern "C" tls_status tls_select_tokens(const tls_shape* shape, const void* q, const int32_t* label_ch,
                                        const uint8_t* codes, const float* scales, const int32_t* block_idx,
                                        int32_t K_b, int32_t k, int32_t* token_idx, float* token_score, void* ws,
                                        size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("tls_select_tokens");
  clear_error();
  tls_status st = check_shape(shape);
  if (st != TLS_OK) return st;
  if (q == nullptr || label_ch == nullptr || codes == nullptr || scales == nullptr || block_idx == nullptr ||
      token_idx == nullptr)
    return fail(TLS_ERR_INVALID_ARG, "select_tokens: null pointer");
  if (!aligned16(q) || !aligned16(codes)) return fail(TLS_ERR_INVALID_ARG, "select_tokens: q/codes not 16-byte aligned");
  WsLayout L;
  st = check_ws(*shape, K_b, k, ws, ws_bytes, &L);
  if (st != TLS_OK) return st;
  st = check_candidates(*shape, K_b);
  if (st != TLS_OK) return st;
  return select_tokens_impl(*shape, q, label_ch, codes, scales, block_idx, K_b, k, token_idx, token_score,
                            (uint8_t*)ws, L, (cudaStream_t)stream);
}

extern "C" tls_status tls_sparse_decode_attn(const tls_shape* shape, const void* q, const tls_kv_view* kv,
                                             const int32_t* token_idx, int32_t k, int32_t out_dtype, void* out,
                                             float* lse, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("tls_sparse_decode_attn");
  clear_error();
  tls_status st = check_shape(shape);
  if (st != TLS_OK) return st;
  st = check_kv(*shape, kv);
  if (st != TLS_OK) return st;
  if (q == nullptr || token_idx == nullptr || out == nullptr)
    return fail(TLS_ERR_INVALID_ARG, "sparse_decode_attn: null pointer");
  if (!aligned16(q)) return fail(TLS_ERR_INVALID_ARG, "sparse_decode_attn: q not 16-byte aligned");
  if (out_dtype != TLS_OUT_F32 && out_dtype != TLS_OUT_BF16)
    return fail(TLS_ERR_INVALID_ARG, "sparse_decode_attn: out_dtype must be TLS_OUT_F32 or TLS_OUT_BF16");
  if (k < 1 || k > shape->ctx_len) return fail(TLS_ERR_INVALID_ARG, "sparse_decode_attn: k %d out of range", k);
  // the attention plan depends on k only; take K_b as large as the context allows
  const int64_t nb = n_blocks(*shape);
  int K_b = (int)((k + shape->block_size - 1) / shape->block_size);
  if (K_b > nb) K_b = (int)nb;
  WsLayout L;
  st = check_ws(*shape, K_b, k, ws, ws_bytes, &L);
  if (st != TLS_OK) return st;
  return sparse_attn_impl(*shape, q, *kv, token_idx, k, out_dtype, out, lse, (uint8_t*)ws, L,
                          (cudaStream_t)stream);
}

// Levels 1 and 2 (the second launched with programmatic dependent launch).
static tls_status select_impl(const tls_shape* shape, const void* q, const void* meta, const int32_t* label_ch,
                              const uint8_t* codes, const float* scales, int32_t K_b, int32_t k, int32_t* block_idx,
                              int32_t* token_idx, void* ws, size_t ws_bytes, void* stream) {
  tls_status st = check_shape(shape);
  if (st != TLS_OK) return st;
  if (q == nullptr || meta == nullptr || label_ch == nullptr || codes == nullptr || scales == nullptr ||
      block_idx == nullptr || token_idx == nullptr)
    return fail(TLS_ERR_INVALID_ARG, "select: null pointer");
  if (!aligned16(q) || !aligned16(meta) || !aligned16(codes))
    return fail(TLS_ERR_INVALID_ARG, "select: q/meta/codes not 16-byte aligned");
  WsLayout L;
  st = check_ws(*shape, K_b, k, ws, ws_bytes, &L);
  if (st != TLS_OK) return st;
  st = check_candidates(*shape, K_b);
  if (st != TLS_OK) return st;
  st = select_blocks_impl(*shape, q, meta, K_b, block_idx, nullptr, (uint8_t*)ws, L, (cudaStream_t)stream);
  if (st != TLS_OK) return st;
  return select_tokens_impl(*shape, q, label_ch, codes, scales, block_idx, K_b, k, token_idx, nullptr,
                            (uint8_t*)ws, L, (cudaStream_t)stream, /*pdl=*/true);
}

extern "C" tls_status tls_select(const tls_shape* shape, const void* q, const void* meta, const int32_t* label_ch,
                                 const uint8_t* codes, const float* scales, int32_t K_b, int32_t k,
                                 int32_t* block_idx, int32_t* token_idx, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("tls_select");
  clear_error();
  return select_impl(shape, q, meta, label_ch, codes, scales, K_b, k, block_idx, token_idx, ws, ws_bytes, stream);
}

extern "C" tls_status tls_decode_step(const tls_shape* shape, const void* q, const void* meta,
                                      const int32_t* label_ch, const uint8_t* codes, const float* scales,
                                      const tls_kv_view* kv, int32_t K_b, int32_t k, int32_t* block_idx,
                                      int32_t* token_idx, int32_t out_dtype, void* out, float* lse, void* ws,
                                      size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("tls_decode_step");
  clear_error();
  // everything the attention checks is checked before anything is launched
  tls_status st = check_shape(shape);
  if (st != TLS_OK) return st;
  st = check_kv(*shape, kv);
  if (st != TLS_OK) return st;
  if (out == nullptr) return fail(TLS_ERR_INVALID_ARG, "decode_step: out is NULL");
  if (out_dtype != TLS_OUT_F32 && out_dtype != TLS_OUT_BF16)
    return fail(TLS_ERR_INVALID_ARG, "decode_step: out_dtype must be TLS_OUT_F32 or TLS_OUT_BF16");
  st = select_impl(shape, q, meta, label_ch, codes, scales, K_b, k, block_idx, token_idx, ws, ws_bytes, stream);
  if (st != TLS_OK) return st;
  return tls_sparse_decode_attn(shape, q, kv, token_idx, k, out_dtype, out, lse, ws, ws_bytes, stream);
}

// ---------------------------------------------------------------------------
// Operator baselines: full attention, block selection alone, token selection
// alone (English summary 4, Efficiency).
// ---------------------------------------------------------------------------

static tls_status check_attn_args(const tls_shape* shape, const void* q, const tls_kv_view* kv, int32_t out_dtype,
                                  const void* out, const char* who) {
  tls_status st = check_shape(shape);
  if (st != TLS_OK) return st;
  st = check_kv(*shape, kv);
  if (st != TLS_OK) return st;
  if (q == nullptr || out == nullptr) return fail(TLS_ERR_INVALID_ARG, "%s: null pointer", who);
  if (!aligned16(q)) return fail(TLS_ERR_INVALID_ARG, "%s: q not 16-byte aligned", who);
  if (out_dtype != TLS_OUT_F32 && out_dtype != TLS_OUT_BF16)
    return fail(TLS_ERR_INVALID_ARG, "%s: out_dtype must be TLS_OUT_F32 or TLS_OUT_BF16", who);
  return TLS_OK;
}

extern "C" tls_status tls_dense_decode_attn(const tls_shape* shape, const void* q, const tls_kv_view* kv,
                                            int32_t out_dtype, void* out, float* lse, void* ws, size_t ws_bytes,
                                            void* stream) {
  NvtxRange nvtx_range("tls_dense_decode_attn");
  clear_error();
  tls_status st = check_attn_args(shape, q, kv, out_dtype, out, "dense_decode_attn");
  if (st != TLS_OK) return st;
  const int nb = (int)n_blocks(*shape);
  if (shape->ctx_len > kMaxListLen) return fail(TLS_ERR_UNSUPPORTED, "dense_decode_attn: ctx_len above 2^24");
  WsLayout L;
  st = check_ws(*shape, nb, (int)shape->ctx_len, ws, ws_bytes, &L);
  if (st != TLS_OK) return st;
  return sparse_attn_impl(*shape, q, *kv, nullptr, (int)shape->ctx_len, out_dtype, out, lse, (uint8_t*)ws, L,
                          (cudaStream_t)stream, /*pdl=*/true, kListAll);
}

extern "C" tls_status tls_quest_decode_step(const tls_shape* shape, const void* q, const void* meta,
                                            const tls_kv_view* kv, int32_t K_b, int32_t* block_idx,
                                            int32_t out_dtype, void* out, float* lse, void* ws, size_t ws_bytes,
                                            void* stream) {
  NvtxRange nvtx_range("tls_quest_decode_step");
  clear_error();
  tls_status st = check_attn_args(shape, q, kv, out_dtype, out, "quest_decode_step");
  if (st != TLS_OK) return st;
  if (meta == nullptr || block_idx == nullptr) return fail(TLS_ERR_INVALID_ARG, "quest_decode_step: null pointer");
  if (!aligned16(meta)) return fail(TLS_ERR_INVALID_ARG, "quest_decode_step: meta not 16-byte aligned");
  const int64_t k = (int64_t)K_b * shape->block_size;
  if (K_b < 1 || k > kMaxListLen) return fail(TLS_ERR_INVALID_ARG, "quest_decode_step: K_b %d out of range", K_b);
  WsLayout L;
  st = check_ws(*shape, K_b, (int)k, ws, ws_bytes, &L);
  if (st != TLS_OK) return st;
  st = select_blocks_impl(*shape, q, meta, K_b, block_idx, nullptr, (uint8_t*)ws, L, (cudaStream_t)stream);
  if (st != TLS_OK) return st;
  return sparse_attn_impl(*shape, q, *kv, nullptr, (int)k, out_dtype, out, lse, (uint8_t*)ws, L,
                          (cudaStream_t)stream, /*pdl=*/true, kListBlocks, block_idx, K_b);
}

extern "C" tls_status tls_ds_decode_step(const tls_shape* shape, const void* q, const int32_t* label_ch,
                                         const uint8_t* codes, const float* scales, const tls_kv_view* kv, int32_t k,
                                         int32_t* token_idx, int32_t out_dtype, void* out, float* lse, void* ws,
                                         size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("tls_ds_decode_step");
  clear_error();
  tls_status st = check_attn_args(shape, q, kv, out_dtype, out, "ds_decode_step");
  if (st != TLS_OK) return st;
  if (label_ch == nullptr || codes == nullptr || scales == nullptr || token_idx == nullptr)
    return fail(TLS_ERR_INVALID_ARG, "ds_decode_step: null pointer");
  if (!aligned16(codes)) return fail(TLS_ERR_INVALID_ARG, "ds_decode_step: codes not 16-byte aligned");
  const int nb = (int)n_blocks(*shape);
  WsLayout L;
  st = check_ws(*shape, nb, k, ws, ws_bytes, &L);
  if (st != TLS_OK) return st;
  st = check_candidates(*shape, nb);
  if (st != TLS_OK) return st;
  // level 2 over every block (no list), then the attention over its choice
  st = select_tokens_impl(*shape, q, label_ch, codes, scales, nullptr, nb, k, token_idx, nullptr, (uint8_t*)ws, L,
                          (cudaStream_t)stream);
  if (st != TLS_OK) return st;
  return sparse_attn_impl(*shape, q, *kv, token_idx, k, out_dtype, out, lse, (uint8_t*)ws, L, (cudaStream_t)stream);
}
