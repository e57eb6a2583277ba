// Staggered decode engine over an HBM block cache (AsyncTLS, English summary
// 2.B; Italian 2.B; Japanese 2.B): step t selects its tokens and attends
// within the blocks chosen at step t-1 (M_{t-1}, already resident), while
// level 1 chooses M_t on a second stream; only the blocks of M_t that are not
// resident, T_t = M_t \ C_t, cross PCIe on a copy stream, overlapping step
// t's attention, and must land before step t+1 attends.
//
// Streams: the caller's stream A runs level 2 and the attention; the engine's
// stream B runs level 1 and the device -> host copy of M_t; stream C copies
// blocks and updates the slot table.  Per step t (cur = t & 1 holds M_t):
//   A: event q_t; level 2 over M_{t-1}; event ready_t; wait copy_end_{t-1};
//      attention over the slot pool; event attn_t
//   B: wait q_t; level 1 -> M_t; M_t -> pinned host; event sel_t
//   host: wait sel_t, plan T_t against C_t with M_{t-1} kept (host mirror)
//   C: wait attn_{t-1} (its slots may be victims now); event copy_start_t;
//      block copies; slot-table update; event copy_end_t
// The table update changes only entries of copied and evicted blocks, none of
// which step t's attention reads, so C may run alongside it.
//
// Planned on the device (where the cache allows it) the step has no host wait:
//   A: wait sel_{t-1}; event q_t; level 2 over M_{t-1} (half the SMs);
//      event ready_t; wait copy_end_{t-1}; attention over the slot pool
//   B: wait q_t; level 1 -> M_t; event sel_t
//   C: wait sel_t (level 1 started after q_t, so the attention of step t-1
//      is done too); event copy_start_t; plan kernel (T_t, its victims, the
//      table; the slots the previous plan used are kept); pull kernel;
//      event copy_end_t
//
// A resident engine (K/V in HBM, no cache) keeps only the stagger, with no
// host wait: A: event q_t, level 2 over M_{t-1}; B: wait q_t, level 1 -> M_t,
// event sel_t; A: attention, wait sel_t.  Level 1 of step t overwrites the list
// level 2 read at step t-1, which A finished before recording q_t; level 2 of
// step t+1 reads M_t, which the join at the end of step t completes.  Every
// step forks and joins within itself, so it can be captured into a graph.

#include <cstdlib>
#include <cstring>
#include <vector>

#include "host_common.h"

namespace tls {
tls_status plan_workspace(const tls_shape& s, int K_b, int k, WsLayout* out);
tls_status prefetch_diff_impl(tls_block_cache* c, const int32_t* new_idx, const int32_t* in_use, int K_b,
                              cudaStream_t cs, int32_t* n_copied, int64_t* bytes);
tls_status block_cache_view(const tls_block_cache* c, tls_kv_view* kv);
tls_status block_cache_device_ready(tls_block_cache* c, int K_b);
tls_status prefetch_device_impl(tls_block_cache* c, const int32_t* new_dev, const int32_t* in_use_dev, int K_b,
                                cudaStream_t cs, int32_t* n_out, bool keep_prev);
int64_t block_cache_block_bytes(const tls_block_cache* c);
tls_status block_cache_check(tls_block_cache* c);
}  // namespace tls

namespace {
constexpr int kRing = 256;  // steps whose timing events are kept
}

struct tls_engine {
  tls_shape shape;
  int K_b = 0, k = 0, rows = 0;
  const void* meta = nullptr;
  const int32_t* label_ch = nullptr;
  const uint8_t* codes = nullptr;
  const float* scales = nullptr;
  tls_block_cache* cache = nullptr;  // null: resident K/V (kv is a dense view)
  tls_kv_view kv;
  uint8_t* ws = nullptr;
  tls::WsLayout L;
  int32_t* bidx[2] = {nullptr, nullptr};       // caller's device [rows, K_b] x 2
  int32_t* token_idx = nullptr;                // caller's device [rows, k]
  int32_t* host_bidx[2] = {nullptr, nullptr};  // pinned mirrors of bidx
  cudaStream_t sel = nullptr, copy = nullptr;
  cudaEvent_t ev_q = nullptr, ev_sel = nullptr, ev_attn[2] = {nullptr, nullptr};
  cudaEvent_t ready[kRing] = {}, copy_start[kRing] = {}, copy_end[kRing] = {};
  int32_t n_copied[kRing] = {};
  int64_t bytes[kRing] = {};
  // device planning: the plan kernel writes each step's block count here
  bool device_plan = false;
  int32_t* n_copied_map = nullptr;  // pinned, mapped [kRing]
  int32_t* n_copied_dev = nullptr;  // its device address
  int64_t t = 0;
  tls_status failed = TLS_OK;
  double wait_ms = 10000.0;  // deadline of the host waits (TLS_HOST_WAIT_MS)
};

using namespace tls;

namespace {

void release(tls_engine* e) {
  if (e->sel != nullptr) cudaStreamSynchronize(e->sel);
  if (e->copy != nullptr) cudaStreamSynchronize(e->copy);
  for (cudaEvent_t* ev : {&e->ev_q, &e->ev_sel, &e->ev_attn[0], &e->ev_attn[1]})
    if (*ev != nullptr) cudaEventDestroy(*ev);
  if (e->n_copied_map != nullptr) cudaFreeHost(e->n_copied_map);
  for (int i = 0; i < kRing; ++i)
    for (cudaEvent_t ev : {e->ready[i], e->copy_start[i], e->copy_end[i]})
      if (ev != nullptr) cudaEventDestroy(ev);
  for (int i = 0; i < 2; ++i)
    if (e->host_bidx[i] != nullptr) cudaFreeHost(e->host_bidx[i]);
  if (e->sel != nullptr) cudaStreamDestroy(e->sel);
  if (e->copy != nullptr) cudaStreamDestroy(e->copy);
  delete e;
}

}  // namespace

namespace {

tls_status engine_create(const tls_shape* shape, int32_t K_b, int32_t k, const void* meta, const int32_t* label_ch,
                         const uint8_t* codes, const float* scales, tls_block_cache* cache, const tls_kv_view* dense,
                         int32_t* block_idx, int32_t* token_idx, void* ws, size_t ws_bytes, tls_engine** out) {
  clear_error();
  tls_status st = check_shape(shape);
  if (st != TLS_OK) return st;
  if (out == nullptr || meta == nullptr || label_ch == nullptr || codes == nullptr || scales == nullptr ||
      (cache == nullptr && dense == nullptr) || block_idx == nullptr || token_idx == nullptr)
    return fail(TLS_ERR_INVALID_ARG, "engine_create: NULL argument");
  if (!aligned16(meta) || !aligned16(codes)) return fail(TLS_ERR_INVALID_ARG, "engine_create: meta/codes not 16-byte aligned");
  WsLayout L;
  st = plan_workspace(*shape, K_b, k, &L);
  if (st != TLS_OK) return st;
  if (ws == nullptr || !aligned16(ws)) return fail(TLS_ERR_INVALID_ARG, "engine_create: workspace NULL or not 16-byte aligned");
  if (ws_bytes < L.total) return fail(TLS_ERR_INVALID_ARG, "engine_create: workspace %zu bytes < required %zu", ws_bytes, L.total);
  tls_kv_view kv;
  if (cache != nullptr) {
    st = block_cache_view(cache, &kv);
    if (st != TLS_OK) return st;
  } else {
    kv = *dense;
    if (kv.k == nullptr || kv.slot_of_block != nullptr || !aligned16(kv.k) || (kv.v != nullptr && !aligned16(kv.v)))
      return fail(TLS_ERR_INVALID_ARG, "engine_create_resident: kv must be a dense view with 16-byte aligned K/V");
  }

  auto* e = new tls_engine();
  e->shape = *shape;
  e->K_b = K_b;
  e->k = k;
  e->rows = rows_of(*shape);
  e->meta = meta;
  e->label_ch = label_ch;
  e->codes = codes;
  e->scales = scales;
  e->cache = cache;
  e->kv = kv;
  e->ws = (uint8_t*)ws;
  e->L = L;
  e->wait_ms = host_wait_ms();
  e->bidx[0] = block_idx;
  e->bidx[1] = block_idx + (size_t)e->rows * K_b;
  e->token_idx = token_idx;
  cudaError_t ce = cudaSuccess;
  for (int i = 0; i < 2 && ce == cudaSuccess && cache != nullptr; ++i)
    ce = cudaHostAlloc((void**)&e->host_bidx[i], (size_t)e->rows * K_b * sizeof(int32_t), cudaHostAllocDefault);
  // the select and copy streams get the highest priority: their small grids
  // are on the critical path of the next step, the attention is not
  int least = 0, greatest = 0;
  if (ce == cudaSuccess) ce = cudaDeviceGetStreamPriorityRange(&least, &greatest);
  if (ce == cudaSuccess) ce = cudaStreamCreateWithPriority(&e->sel, cudaStreamNonBlocking, greatest);
  if (ce == cudaSuccess && cache != nullptr) ce = cudaStreamCreateWithPriority(&e->copy, cudaStreamNonBlocking, greatest);
  for (cudaEvent_t* ev : {&e->ev_q, &e->ev_sel, &e->ev_attn[0], &e->ev_attn[1]})
    if (ce == cudaSuccess) ce = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
  for (int i = 0; i < kRing && ce == cudaSuccess && cache != nullptr; ++i) {
    ce = cudaEventCreate(&e->ready[i]);
    if (ce == cudaSuccess) ce = cudaEventCreate(&e->copy_start[i]);
    if (ce == cudaSuccess) ce = cudaEventCreate(&e->copy_end[i]);
  }
  if (ce != cudaSuccess) {
    release(e);
    return cuda_check(ce, "engine_create: streams, events or pinned mirrors");
  }
  // the transfer is planned on the device when the cache allows it (K/V in
  // mapped pinned memory, pool and lists within the plan kernel's sizes);
  // TLS_ENGINE_PLANNER=host keeps the host planner
  const char* planner = std::getenv("TLS_ENGINE_PLANNER");
  if (cache != nullptr && !(planner != nullptr && std::strcmp(planner, "host") == 0)) {
    st = block_cache_device_ready(cache, K_b);
    if (st == TLS_OK) {
      ce = cudaHostAlloc((void**)&e->n_copied_map, kRing * sizeof(int32_t), cudaHostAllocMapped | cudaHostAllocPortable);
      if (ce == cudaSuccess) ce = cudaHostGetDevicePointer((void**)&e->n_copied_dev, e->n_copied_map, 0);
      if (ce != cudaSuccess) {
        release(e);
        return cuda_check(ce, "engine_create: device planning buffers");
      }
      for (int i = 0; i < kRing; ++i) e->n_copied_map[i] = 0;
      e->device_plan = true;
    } else if (st == TLS_ERR_UNSUPPORTED) {
      clear_error();  // the host planner serves this cache
    } else {
      release(e);
      return st;
    }
  }
  *out = e;
  return TLS_OK;
}

}  // namespace

extern "C" tls_status tls_engine_create(const tls_shape* shape, int32_t K_b, int32_t k, const void* meta,
                                        const int32_t* label_ch, const uint8_t* codes, const float* scales,
                                        tls_block_cache* cache, int32_t* block_idx, int32_t* token_idx, void* ws,
                                        size_t ws_bytes, tls_engine** out) {
  if (cache == nullptr) {
    clear_error();
    return fail(TLS_ERR_INVALID_ARG, "engine_create: NULL cache (resident K/V: tls_engine_create_resident)");
  }
  return engine_create(shape, K_b, k, meta, label_ch, codes, scales, cache, nullptr, block_idx, token_idx, ws,
                       ws_bytes, out);
}

extern "C" tls_status tls_engine_create_resident(const tls_shape* shape, int32_t K_b, int32_t k, const void* meta,
                                                 const int32_t* label_ch, const uint8_t* codes, const float* scales,
                                                 const tls_kv_view* kv, int32_t* block_idx, int32_t* token_idx,
                                                 void* ws, size_t ws_bytes, tls_engine** out) {
  if (kv == nullptr) {
    clear_error();
    return fail(TLS_ERR_INVALID_ARG, "engine_create_resident: NULL kv");
  }
  return engine_create(shape, K_b, k, meta, label_ch, codes, scales, nullptr, kv, block_idx, token_idx, ws, ws_bytes,
                       out);
}

extern "C" void tls_engine_destroy(tls_engine* e) {
  if (e != nullptr) release(e);
}

namespace {

tls_status resident_step(tls_engine* e, const void* q, int32_t out_dtype, void* out, float* lse, cudaStream_t A) {
  const tls_shape& s = e->shape;
  const int cur = (int)(e->t & 1), prev = cur ^ 1;
  tls_status st;
  // prologue: M_{-1} from q_0
  if (e->t == 0) {
    st = select_blocks_impl(s, q, e->meta, e->K_b, e->bidx[prev], nullptr, e->ws, e->L, A);
    if (st != TLS_OK) return st;
  }
  // level 2 within M_{t-1} first, on A (it is on the critical path; launched
  // first, its CTAs are placed first), on at most half the SMs, which leaves
  // level 1 the other half
  cudaError_t ce = cudaEventRecord(e->ev_q, A);
  if (ce != cudaSuccess) return cuda_check(ce, "engine_step: q event");
  st = select_tokens_impl(s, q, e->label_ch, e->codes, e->scales, e->bidx[prev], e->K_b, e->k, e->token_idx, nullptr,
                          e->ws, e->L, A, /*pdl=*/false, /*lean=*/true);
  if (st != TLS_OK) return st;
  // fork: level 1 for q_t on the select stream, after what A had issued
  // before level 2 (it writes M_t, which no kernel of this step reads)
  ce = cudaStreamWaitEvent(e->sel, e->ev_q, 0);
  if (ce != cudaSuccess) return cuda_check(ce, "engine_step: select stream");
  st = select_blocks_impl(s, q, e->meta, e->K_b, e->bidx[cur], nullptr, e->ws, e->L, e->sel);
  if (st != TLS_OK) return st;
  ce = cudaEventRecord(e->ev_sel, e->sel);
  if (ce != cudaSuccess) return cuda_check(ce, "engine_step: select stream");
  // programmatic launch: level 2 lets the attention's CTAs in only once it has
  // scored, so they do not hold the SMs level 1 needs for long
  st = sparse_attn_impl(s, q, e->kv, e->token_idx, e->k, out_dtype, out, lse, e->ws, e->L, A, /*pdl=*/true);
  if (st != TLS_OK) return st;
  // join: M_t is complete before anything A issues next
  ce = cudaStreamWaitEvent(A, e->ev_sel, 0);
  if (ce != cudaSuccess) return cuda_check(ce, "engine_step: join");
  e->t += 1;
  return TLS_OK;
}

// The offloaded step with the transfer planned on the device: no host wait.
// Beside the host-planned order, one device-side wait takes the place of the
// host's: level 2 waits for the level 1 of the step before (it reads M_{t-1}).
// The plan of step t keeps the slots the plan of step t-1 used (M_{t-1}'s)
// without reading M_{t-1}, so level 1 of step t+1 may overwrite that list
// while the plan runs.
tls_status device_step(tls_engine* e, const void* q, int32_t out_dtype, void* out, float* lse, cudaStream_t A) {
  const tls_shape& s = e->shape;
  const int cur = (int)(e->t & 1), prev = cur ^ 1;
  const int ri = (int)(e->t % kRing), rp = (int)((e->t + kRing - 1) % kRing);
  tls_status st = block_cache_check(e->cache);  // a failed plan of an earlier step stops the engine
  if (st != TLS_OK) return st;
  cudaError_t ce;
  if (e->t == 0) {
    // prologue: M_{-1} from q_0 on A, pulled in on the copy stream
    st = select_blocks_impl(s, q, e->meta, e->K_b, e->bidx[prev], nullptr, e->ws, e->L, A);
    if (st != TLS_OK) return st;
    ce = cudaEventRecord(e->ev_sel, A);
    if (ce == cudaSuccess) ce = cudaStreamWaitEvent(e->copy, e->ev_sel, 0);
    if (ce == cudaSuccess) ce = cudaEventRecord(e->copy_start[rp], e->copy);
    if (ce != cudaSuccess) return cuda_check(ce, "engine_step: prologue");
    e->n_copied_map[rp] = 0;
    st = prefetch_device_impl(e->cache, e->bidx[prev], nullptr, e->K_b, e->copy, e->n_copied_dev + rp,
                              /*keep_prev=*/false);
    if (st != TLS_OK) return st;
    ce = cudaEventRecord(e->copy_end[rp], e->copy);
    if (ce != cudaSuccess) return cuda_check(ce, "engine_step: prologue");
  }
  // M_{t-1} (written by level 1 of the step before) is complete before level 2
  ce = cudaStreamWaitEvent(A, e->ev_sel, 0);
  if (ce == cudaSuccess) ce = cudaEventRecord(e->ev_q, A);
  if (ce != cudaSuccess) return cuda_check(ce, "engine_step: q event");
  // level 2 within M_{t-1} first, on A, on at most half the SMs (as in the
  // resident step: launched first, its CTAs are placed first, and level 1
  // keeps the other half)
  st = select_tokens_impl(s, q, e->label_ch, e->codes, e->scales, e->bidx[prev], e->K_b, e->k, e->token_idx, nullptr,
                          e->ws, e->L, A, /*pdl=*/false, /*lean=*/true);
  if (st != TLS_OK) return st;
  // level 1 for q_t on the select stream: M_t
  ce = cudaStreamWaitEvent(e->sel, e->ev_q, 0);
  if (ce != cudaSuccess) return cuda_check(ce, "engine_step: select stream");
  st = select_blocks_impl(s, q, e->meta, e->K_b, e->bidx[cur], nullptr, e->ws, e->L, e->sel);
  if (st != TLS_OK) return st;
  ce = cudaEventRecord(e->ev_sel, e->sel);
  if (ce != cudaSuccess) return cuda_check(ce, "engine_step: select stream");
  // the attention over the slot pool, on A, once T_{t-1} has landed (a
  // plain launch: as a programmatic one, its CTAs would wait on SMs the pull
  // of T_t needs; measured once, the transfer-bound 36-layer workload's layer
  // ran about 10 % slower that way, for about 1 us gained on the MQA offload
  // workload)
  ce = cudaEventRecord(e->ready[ri], A);
  if (ce == cudaSuccess) ce = cudaStreamWaitEvent(A, e->copy_end[rp], 0);  // T_{t-1} has landed
  if (ce != cudaSuccess) return cuda_check(ce, "engine_step: wait for the transfer");
  st = sparse_attn_impl(s, q, e->kv, e->token_idx, e->k, out_dtype, out, lse, e->ws, e->L, A, /*pdl=*/false);
  if (st != TLS_OK) return st;
  // T_t on the copy stream once M_t is chosen, alongside the attention of
  // step t.  The attention of step t-1 (whose slots may be evicted now) is
  // done by then: level 1 started after q_t, which A records after it.
  ce = cudaStreamWaitEvent(e->copy, e->ev_sel, 0);
  if (ce == cudaSuccess) ce = cudaEventRecord(e->copy_start[ri], e->copy);
  if (ce != cudaSuccess) return cuda_check(ce, "engine_step: copy stream");
  e->n_copied_map[ri] = 0;
  st = prefetch_device_impl(e->cache, e->bidx[cur], nullptr, e->K_b, e->copy, e->n_copied_dev + ri,
                            /*keep_prev=*/true);
  if (st != TLS_OK) return st;
  ce = cudaEventRecord(e->copy_end[ri], e->copy);
  if (ce != cudaSuccess) return cuda_check(ce, "engine_step: copy stream");
  e->t += 1;
  return TLS_OK;
}

tls_status engine_step(tls_engine* e, const void* q, int32_t out_dtype, void* out, float* lse, cudaStream_t A) {
  if (e->cache == nullptr) return resident_step(e, q, out_dtype, out, lse, A);
  if (e->device_plan) return device_step(e, q, out_dtype, out, lse, A);
  const tls_shape& s = e->shape;
  const size_t list_bytes = (size_t)e->rows * e->K_b * sizeof(int32_t);
  const int cur = (int)(e->t & 1), prev = cur ^ 1;
  const int ri = (int)(e->t % kRing), rp = (int)((e->t + kRing - 1) % kRing);
  tls_status st;
  if (e->t == 0) {
    // prologue: M_{-1} from q_0, made resident before the first attention
    st = select_blocks_impl(s, q, e->meta, e->K_b, e->bidx[prev], nullptr, e->ws, e->L, A);
    if (st != TLS_OK) return st;
    cudaError_t ce = cudaMemcpyAsync(e->host_bidx[prev], e->bidx[prev], list_bytes, cudaMemcpyDeviceToHost, A);
    if (ce == cudaSuccess) ce = cudaEventRecord(e->ev_sel, A);
    if (ce != cudaSuccess) return cuda_check(ce, "engine_step: prologue");
    st = wait_event_deadline(e->ev_sel, e->wait_ms, "engine_step: prologue block list");
    if (st != TLS_OK) return st;
    ce = cudaEventRecord(e->copy_start[rp], e->copy);
    if (ce != cudaSuccess) return cuda_check(ce, "engine_step: prologue");
    st = prefetch_diff_impl(e->cache, e->host_bidx[prev], nullptr, e->K_b, e->copy, &e->n_copied[rp], &e->bytes[rp]);
    if (st != TLS_OK) return st;
    ce = cudaEventRecord(e->copy_end[rp], e->copy);
    if (ce != cudaSuccess) return cuda_check(ce, "engine_step: prologue");
  }
  // level 1 for q_t on the select stream: M_t
  cudaError_t ce = cudaEventRecord(e->ev_q, A);
  if (ce == cudaSuccess) ce = cudaStreamWaitEvent(e->sel, e->ev_q, 0);
  if (ce != cudaSuccess) return cuda_check(ce, "engine_step: select stream");
  st = select_blocks_impl(s, q, e->meta, e->K_b, e->bidx[cur], nullptr, e->ws, e->L, e->sel);
  if (st != TLS_OK) return st;
  ce = cudaMemcpyAsync(e->host_bidx[cur], e->bidx[cur], list_bytes, cudaMemcpyDeviceToHost, e->sel);
  if (ce == cudaSuccess) ce = cudaEventRecord(e->ev_sel, e->sel);
  if (ce != cudaSuccess) return cuda_check(ce, "engine_step: block list to host");
  // level 2 within M_{t-1} and the attention over the slot pool, on A
  st = select_tokens_impl(s, q, e->label_ch, e->codes, e->scales, e->bidx[prev], e->K_b, e->k, e->token_idx, nullptr,
                          e->ws, e->L, A, /*pdl=*/false);
  if (st != TLS_OK) return st;
  ce = cudaEventRecord(e->ready[ri], A);
  if (ce == cudaSuccess) ce = cudaStreamWaitEvent(A, e->copy_end[rp], 0);  // T_{t-1} has landed
  if (ce != cudaSuccess) return cuda_check(ce, "engine_step: wait for the transfer");
  // a plain launch: an early-resident attention would hold every SM while it
  // waits, starving level 1 on the select stream and the block pulls
  st = sparse_attn_impl(s, q, e->kv, e->token_idx, e->k, out_dtype, out, lse, e->ws, e->L, A, /*pdl=*/false);
  if (st != TLS_OK) return st;
  ce = cudaEventRecord(e->ev_attn[cur], A);
  // T_t = M_t \ C_t on the copy stream, after the attention of step t-1 (its
  // slots may be evicted now), alongside the attention of step t
  if (ce != cudaSuccess) return cuda_check(ce, "engine_step: attention event");
  st = wait_event_deadline(e->ev_sel, e->wait_ms, "engine_step: level 1 of this step");
  if (st != TLS_OK) return st;
  ce = cudaStreamWaitEvent(e->copy, e->ev_attn[prev], 0);
  if (ce == cudaSuccess) ce = cudaEventRecord(e->copy_start[ri], e->copy);
  if (ce != cudaSuccess) return cuda_check(ce, "engine_step: copy stream");
  st = prefetch_diff_impl(e->cache, e->host_bidx[cur], e->host_bidx[prev], e->K_b, e->copy, &e->n_copied[ri],
                          &e->bytes[ri]);
  if (st != TLS_OK) return st;
  ce = cudaEventRecord(e->copy_end[ri], e->copy);
  if (ce != cudaSuccess) return cuda_check(ce, "engine_step: copy stream");
  e->t += 1;
  return TLS_OK;
}

}  // namespace

extern "C" tls_status tls_engine_step(tls_engine* e, const void* q, int32_t out_dtype, void* out, float* lse,
                                      void* stream) {
  NvtxRange nvtx_range("tls_engine_step");
  clear_error();
  if (e == nullptr || q == nullptr || out == nullptr) return fail(TLS_ERR_INVALID_ARG, "engine_step: NULL argument");
  if (!aligned16(q)) return fail(TLS_ERR_INVALID_ARG, "engine_step: q not 16-byte aligned");
  if (out_dtype != TLS_OUT_F32 && out_dtype != TLS_OUT_BF16)
    return fail(TLS_ERR_INVALID_ARG, "engine_step: out_dtype must be TLS_OUT_F32 or TLS_OUT_BF16");
  if (e->failed != TLS_OK)
    return fail(e->failed, "engine_step: an earlier step failed; the cache no longer matches the block lists");
  const tls_status st = engine_step(e, q, out_dtype, out, lse, (cudaStream_t)stream);
  if (st != TLS_OK) e->failed = st;
  return st;
}

extern "C" int64_t tls_engine_steps(const tls_engine* e) { return e == nullptr ? -1 : e->t; }

extern "C" int32_t tls_engine_step_kernels(const tls_engine* e) {
  if (e == nullptr) return -1;
  // level 1 (with its query preparation for groups padded to 64 heads or
  // more), level 2, the attention; offloaded: the transfer's plan and pull
  // (device planner) or its one pull kernel (host planner)
  const int n = 3 + (group_of(e->shape) > 32 ? 1 : 0);
  if (e->cache == nullptr) return n;
  return n + (e->device_plan ? 2 : 1);
}

extern "C" tls_status tls_engine_stats(tls_engine* e, int64_t step, tls_engine_step_stats* out) {
  clear_error();
  if (e == nullptr || out == nullptr) return fail(TLS_ERR_INVALID_ARG, "engine_stats: NULL argument");
  if (step < -1 || step >= e->t || step < e->t - (kRing - 1))
    return fail(TLS_ERR_INVALID_ARG, "engine_stats: step %lld not among the last %d steps taken",
                (long long)step, kRing - 1);
  if (e->cache == nullptr) {  // resident K/V: nothing is transferred
    out->step = step;
    out->n_copied = 0;
    out->bytes_copied = 0;
    out->copy_ms = 0.0f;
    out->exposed_ms = step + 1 < e->t ? 0.0f : -1.0f;
    return TLS_OK;
  }
  const int si = (int)((step + kRing) % kRing);
  tls_status st = wait_event_deadline(e->copy_end[si], e->wait_ms, "engine_stats: transfer");
  if (st != TLS_OK) return st;
  int32_t n_copied = e->n_copied[si];
  int64_t bytes_copied = e->bytes[si];
  if (e->device_plan) {
    // written by the step's plan kernel, which ran before copy_end
    n_copied = *reinterpret_cast<volatile int32_t*>(e->n_copied_map + si);
    if (n_copied < 0) {
      st = block_cache_check(e->cache);
      return st != TLS_OK ? st : fail(TLS_ERR_CAPACITY, "engine_stats: the plan of step %lld failed", (long long)step);
    }
    bytes_copied = (int64_t)n_copied * block_cache_block_bytes(e->cache);
  }
  float copy_ms = 0.0f, exposed_ms = -1.0f;
  cudaError_t ce = cudaEventElapsedTime(&copy_ms, e->copy_start[si], e->copy_end[si]);
  if (ce == cudaSuccess && step + 1 < e->t) {
    const int ni = (int)((step + 1) % kRing);
    st = wait_event_deadline(e->ready[ni], e->wait_ms, "engine_stats: next step");
    if (st != TLS_OK) return st;
    ce = cudaEventElapsedTime(&exposed_ms, e->ready[ni], e->copy_end[si]);
    if (exposed_ms < 0.0f) exposed_ms = 0.0f;
  }
  if (ce != cudaSuccess) return cuda_check(ce, "engine_stats: events");
  out->step = step;
  out->n_copied = n_copied;
  out->bytes_copied = bytes_copied;
  out->copy_ms = copy_ms;
  out->exposed_ms = exposed_ms;
  return TLS_OK;
}
