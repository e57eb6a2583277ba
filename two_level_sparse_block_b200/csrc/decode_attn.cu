// Attention over the chosen tokens only (AsyncTLS, Italian summary 2.A.2; the
// token list comes from level 2, English summary 2.A Stage 2).
//
// Split-K flash decoding.  Grid (splits, head groups, rows); a CTA takes a
// contiguous slice of the row's token list and HG heads of the group.  Each
// half-warp handles one token at a time: its 16 lanes load the token's K row
// (and V row) with 16-byte loads, reduce the per-head dot products with
// shuffles, and keep an online softmax (base-2 exponentials, fp32) plus an
// fp32 accumulator.  The CTA folds its 8 half-warps, writes (m, l, acc) to
// the workspace, and the last CTA of each (row, head group) merges the splits
// by log-sum-exp and writes the output (fp32 or bf16) and the natural-log lse.

#include <mutex>
#include <utility>
#include <vector>

#include "attn_common.cuh"
#include "device_common.cuh"
#include "host_common.h"

namespace tls {



template <int PK, int PV, int HG, int U>
__global__ void __launch_bounds__(128) sparse_attn_kernel(AttnParams p) {
  extern __shared__ float red[];  // [8][HG] m, [8][HG] l, [8][HG][dv] acc
  __shared__ int last;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int l16 = lane & 15, half = lane >> 4;
  const int hw = warp * 2 + half;  // half-warp id 0..7
  const int split = blockIdx.x, hg = blockIdx.y, row = blockIdx.z;
  const int g = p.group;
  const int b = row / p.n_kv_heads, kvh = row % p.n_kv_heads;
  const int h0 = hg * HG;

  // q slice of this lane: element e = pass*128 + l16*8 + i
  float qf[HG][PK][8];
#pragma unroll
  for (int hh = 0; hh < HG; ++hh) {
    const int h = h0 + hh;
#pragma unroll
    for (int ps = 0; ps < PK; ++ps) {
      const int e = ps * 128 + l16 * 8;
      if (h < g && e < p.dqk) {
        const uint4 w = *reinterpret_cast<const uint4*>(p.q + ((int64_t)b * p.n_q_heads + kvh * g + h) * p.dqk + e);
        unpack8(w, qf[hh][ps]);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) qf[hh][ps][i] = 0.0f;
      }
    }
  }

  float m[HG], l[HG], acc[HG][PV][8];
#pragma unroll
  for (int hh = 0; hh < HG; ++hh) {
    m[hh] = -INFINITY;
    l[hh] = 0.0f;
#pragma unroll
    for (int ps = 0; ps < PV; ++ps)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[hh][ps][i] = 0.0f;
  }

  const int t_begin = split * p.tokens_per_split;
  const int t_end = min(p.k_sel, t_begin + p.tokens_per_split);
  const int64_t len = seq_len_of(p.seq_lens, b, p.ctx_len);
  grid_dependency_wait();  // token lists come from the preceding kernel (read through L2)

  for (int base = t_begin; base < t_end; base += 8 * U) {
    uint4 kw[U][PK], vw[U][PV];
    bool valid[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int t = base + u * 8 + hw;
      // entries that are no token of the sequence are skipped, so a bad list
      // can never address outside the cache
      const int tok = t < t_end ? attn_token(p, row, t, len) : -1;
      valid[u] = tok >= 0;
      int64_t krow = 0, vrow = 0;
      if (valid[u]) {
        const int64_t r = attn_row_id(p, row, tok);
        krow = r * p.k_stride;
        vrow = r * p.v_stride;
      }
#pragma unroll
      for (int ps = 0; ps < PK; ++ps) {
        const int e = ps * 128 + l16 * 8;
        kw[u][ps] = (valid[u] && e < p.dqk) ? __ldg(reinterpret_cast<const uint4*>(p.k + krow + e))
                                            : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int ps = 0; ps < PV; ++ps) {
        const int e = ps * 128 + l16 * 8;
        vw[u][ps] = (valid[u] && e < p.dv) ? __ldg(reinterpret_cast<const uint4*>(p.v + vrow + e))
                                           : make_uint4(0u, 0u, 0u, 0u);
      }
    }

    float sc[U][HG];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float part[HG];
#pragma unroll
      for (int hh = 0; hh < HG; ++hh) part[hh] = 0.0f;
#pragma unroll
      for (int ps = 0; ps < PK; ++ps) {
        float kf[8];
        unpack8(kw[u][ps], kf);
#pragma unroll
        for (int hh = 0; hh < HG; ++hh)
#pragma unroll
          for (int i = 0; i < 8; ++i) part[hh] = fmaf(qf[hh][ps][i], kf[i], part[hh]);
      }
#pragma unroll
      for (int hh = 0; hh < HG; ++hh) {
        float x = part[hh];
        x += __shfl_xor_sync(0xffffffffu, x, 8);
        x += __shfl_xor_sync(0xffffffffu, x, 4);
        x += __shfl_xor_sync(0xffffffffu, x, 2);
        x += __shfl_xor_sync(0xffffffffu, x, 1);
        sc[u][hh] = valid[u] ? x * p.scale_log2 : -INFINITY;
      }
    }

#pragma unroll
    for (int hh = 0; hh < HG; ++hh) {
      float mn = m[hh];
#pragma unroll
      for (int u = 0; u < U; ++u) mn = fmaxf(mn, sc[u][hh]);
      if (mn == -INFINITY) continue;
      const float corr = (m[hh] == -INFINITY) ? 0.0f : exp2f(m[hh] - mn);
      float pu[U];
      float psum = 0.0f;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        pu[u] = valid[u] ? exp2f(sc[u][hh] - mn) : 0.0f;
        psum += pu[u];
      }
      l[hh] = l[hh] * corr + psum;
      m[hh] = mn;
#pragma unroll
      for (int ps = 0; ps < PV; ++ps) {
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[hh][ps][i] *= corr;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          float vf[8];
          unpack8(vw[u][ps], vf);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[hh][ps][i] = fmaf(pu[u], vf[i], acc[hh][ps][i]);
        }
      }
    }
  }

  // fold the 8 half-warps of the CTA
  const int dv = p.dv;
  float* rm = red;
  float* rl = red + 8 * HG;
  float* ra = red + 16 * HG;
#pragma unroll
  for (int hh = 0; hh < HG; ++hh) {
    if (l16 == 0) {
      rm[hw * HG + hh] = m[hh];
      rl[hw * HG + hh] = l[hh];
    }
#pragma unroll
    for (int ps = 0; ps < PV; ++ps) {
      const int e = ps * 128 + l16 * 8;
      if (e < dv) {
#pragma unroll
        for (int i = 0; i < 8; ++i) ra[((size_t)hw * HG + hh) * dv + e + i] = acc[hh][ps][i];
      }
    }
  }
  __syncthreads();
  const int nh = min(HG, g - h0);
  for (int idx = tid; idx < nh * (dv + 2); idx += 128) {
    const int hh = idx / (dv + 2), e = idx % (dv + 2);
    float M = -INFINITY;
    for (int w = 0; w < 8; ++w) M = fmaxf(M, rm[w * HG + hh]);
    float val = 0.0f;
    if (e == 0) {
      val = M;
    } else if (M != -INFINITY) {
      for (int w = 0; w < 8; ++w) {
        const float mw = rm[w * HG + hh];
        if (mw == -INFINITY) continue;
        const float f = exp2f(mw - M);
        val += f * (e == 1 ? rl[w * HG + hh] : ra[((size_t)w * HG + hh) * dv + (e - 2)]);
      }
    }
    p.partial[(((int64_t)row * g + h0 + hh) * p.splits + split) * (dv + 2) + e] = val;
  }

  __threadfence();
  __syncthreads();
  if (tid == 0)
    last = atomicInc(&p.counters[row * p.head_groups + hg], p.splits - 1) == (unsigned)(p.splits - 1);
  __syncthreads();
  if (!last) return;
  __threadfence();

  merge_splits(p, row, b, kvh, h0, nh, p.splits, red, 16 * HG + 8 * HG * dv);
}

template <int PK, int PV, int HG>
tls_status launch_attn(const AttnParams& p, int rows, cudaStream_t stream) {
  constexpr int U = (PK + PV <= 2) ? 4 : 1;
  const size_t smem = (size_t)(16 * HG + 8 * HG * p.dv) * sizeof(float);
  cudaError_t e = kernel_attrs((const void*)sparse_attn_kernel<PK, PV, HG, U>, smem);
  if (e != cudaSuccess) return cuda_check(e, "sparse_decode_attn: set smem attribute");
  dim3 grid((unsigned)p.splits, (unsigned)p.head_groups, (unsigned)rows);
  sparse_attn_kernel<PK, PV, HG, U><<<grid, 128, smem, stream>>>(p);
  return launch_check("sparse_decode_attn launch");
}

tls_status sparse_attn_impl(const tls_shape& s, const void* q, const tls_kv_view& kv, const int32_t* token_idx,
                            int k, int out_dtype, void* out, float* lse, uint8_t* ws, const WsLayout& L,
                            cudaStream_t stream, bool pdl, int list_mode, const int32_t* blocks, int K_b) {
  AttnParams p;
  p.q = (const uint16_t*)q;
  p.k = (const uint16_t*)kv.k;
  p.v = s.v_offset >= 0 ? (const uint16_t*)kv.k + s.v_offset : (const uint16_t*)kv.v;
  p.k_stride = kv.k_row_stride;
  p.v_stride = s.v_offset >= 0 ? kv.k_row_stride : kv.v_row_stride;
  p.slot_of_block = kv.slot_of_block;
  p.n_slots = kv.n_slots;
  p.bs = s.block_size;
  p.nb = (int)n_blocks(s);
  p.ctx_len = s.ctx_len;
  p.token_idx = token_idx;
  p.k_sel = k;
  p.n_q_heads = s.n_q_heads;
  p.n_kv_heads = s.n_kv_heads;
  p.group = group_of(s);
  p.dqk = s.qk_dim;
  p.dv = s.v_dim;
  p.scale_log2 = s.softmax_scale * 1.4426950408889634f;
  p.tokens_per_split = L.tokens_per_split;
  p.splits = L.splits;
  p.head_groups = L.head_groups;
  p.partial = reinterpret_cast<float*>(ws + L.partial);
  p.counters = reinterpret_cast<unsigned*>(ws + L.att_counter);
  p.out = out;
  p.out_bf16 = out_dtype == TLS_OUT_BF16;
  p.lse = lse;
  p.heads_per_cta = L.heads_per_cta;
  p.tiles_per_pair = L.tiles_per_pair;
  p.n_items = L.n_items;
  p.n_ctas = L.n_ctas;
  p.err = reinterpret_cast<int*>(ws + L.err);
  p.seq_lens = s.seq_lens;
  p.list_mode = list_mode;
  p.blocks = blocks;
  p.K_b = K_b;
  const int rows = rows_of(s);
  if (attn_mma_supported(s)) return launch_attn_mma(p, rows, stream, pdl);
  if (attn_mla_supported(s)) return launch_attn_mla(p, rows, stream, pdl);
  const int pk = (s.qk_dim + 127) / 128, pv = (s.v_dim + 127) / 128;
  const int hg = L.heads_per_cta;
  if (pk == 1 && pv == 1) {
    if (hg == 1) return launch_attn<1, 1, 1>(p, rows, stream);
    if (hg == 2) return launch_attn<1, 1, 2>(p, rows, stream);
    if (hg == 4) return launch_attn<1, 1, 4>(p, rows, stream);
    if (hg == 8) return launch_attn<1, 1, 8>(p, rows, stream);
  } else if (pk <= 2 && pv <= 2) {
    if (hg == 1) return launch_attn<2, 2, 1>(p, rows, stream);
    if (hg == 2) return launch_attn<2, 2, 2>(p, rows, stream);
    if (hg == 4) return launch_attn<2, 2, 4>(p, rows, stream);
  } else if (pk <= 5 && pv <= 4) {
    if (hg == 1) return launch_attn<5, 4, 1>(p, rows, stream);
    if (hg == 2) return launch_attn<5, 4, 2>(p, rows, stream);
  }
  return fail(TLS_ERR_UNSUPPORTED, "sparse_decode_attn: no kernel for qk_dim %d, v_dim %d, %d heads per CTA",
              s.qk_dim, s.v_dim, hg);
}

// Heads per CTA for the attention kernel.  The tensor-core kernel takes up to
// 64 heads (its TMEM and shared-memory budget); for the CUDA-core kernel the
// register budget allows 8 heads at 128-wide rows, 4 at 256 and 2 above.
int attn_heads_per_cta(const tls_shape& s) {
  const int g = group_of(s);
  if (attn_mma_supported(s)) return g < 16 ? g : 16;
  if (attn_mla_supported(s)) return 16;
  const int pk = (s.qk_dim + 127) / 128, pv = (s.v_dim + 127) / 128;
  int cap = (pk == 1 && pv == 1) ? 8 : (pk <= 2 && pv <= 2) ? 4 : 2;
  int hg = 1;
  while (hg < g && hg < cap) hg <<= 1;
  return hg;
}

}  // namespace tls

// ---------------------------------------------------------------------------
// Scratch-free variant of the attention entry point.
//
// Some callers cannot hand the library a workspace: code that runs as a
// plug-in inside a serving runtime that owns the whole HBM budget and exposes
// no allocator, and latency-critical decode loops where a cudaMalloc (which can
// synchronise the device and take milliseconds) is not allowed.  For them the
// split-K partials and the merge tickets live in one file-scope device array
// of fixed size.  Every GPU that loads the library holds this array until the
// process exits.  Host code must not pass the array's name to a kernel (on the
// host it is only a stand-in symbol); the device address is looked up once per
// device with cudaGetSymbolAddress, on the first call made on that device.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_attn_scratch[TLS_NOALLOC_SCRATCH_BYTES];

namespace {
// The array's device address, looked up once per (device, CUDA context): a
// context created anew (the primary context after cudaDeviceReset, or a
// context of the caller's own) loads the module again at another address.
struct ScratchKey {
  int dev;
  void* ctx;
};
std::mutex g_scratch_mu;
std::vector<std::pair<ScratchKey, void*>> g_scratch_ptr;
using CtxGetCurrentFn = int (*)(void**);
CtxGetCurrentFn g_ctx_current = nullptr;
std::once_flag g_ctx_once;
}  // namespace

namespace tls {
tls_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_check(e, "sparse_decode_attn_noalloc: cudaGetDevice");
  std::call_once(g_ctx_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_current = reinterpret_cast<CtxGetCurrentFn>(fn);
  });
  if (g_ctx_current == nullptr) return fail(TLS_ERR_CUDA, "sparse_decode_attn_noalloc: cuCtxGetCurrent unavailable");
  void* ctx = nullptr;
  if (g_ctx_current(&ctx) != 0) return fail(TLS_ERR_CUDA, "sparse_decode_attn_noalloc: cuCtxGetCurrent failed");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (ctx != nullptr)
    for (auto& kv : g_scratch_ptr)
      if (kv.first.dev == dev && kv.first.ctx == ctx) {
        *out = kv.second;
        return TLS_OK;
      }
  // the lookup also makes the device's primary context current when no
  // context was; the context it ran in keys the cached address
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_attn_scratch);
  if (e != cudaSuccess || p == nullptr)
    return cuda_check(e != cudaSuccess ? e : cudaErrorInvalidSymbol, "sparse_decode_attn_noalloc: cudaGetSymbolAddress");
  if (g_ctx_current(&ctx) != 0 || ctx == nullptr)
    return fail(TLS_ERR_CUDA, "sparse_decode_attn_noalloc: no current context after the lookup");
  g_scratch_ptr.push_back({ScratchKey{dev, ctx}, p});
  *out = p;
  return TLS_OK;
}
}  // namespace tls

extern "C" tls_status tls_sparse_decode_attn_noalloc(const tls_shape* shape, const void* q, const tls_kv_view* kv,
                                                     const int32_t* token_idx, int32_t k, int32_t out_dtype,
                                                     void* out, float* lse, void* stream) {
  tls::NvtxRange nvtx_range("tls_sparse_decode_attn_noalloc");
  using namespace tls;
  clear_error();
  tls_status st = check_shape(shape);
  if (st != TLS_OK) return st;
  const tls_shape& s = *shape;
  if (q == nullptr || token_idx == nullptr || out == nullptr || kv == nullptr || kv->k == nullptr)
    return fail(TLS_ERR_INVALID_ARG, "sparse_decode_attn_noalloc: null pointer");
  if (!aligned16(q) || !aligned16(kv->k) || (s.v_offset < 0 && (kv->v == nullptr || !aligned16(kv->v))))
    return fail(TLS_ERR_INVALID_ARG, "sparse_decode_attn_noalloc: q/k/v NULL or not 16-byte aligned");
  if (kv->k_row_stride < s.qk_dim || kv->k_row_stride % 8 != 0 ||
      (s.v_offset < 0 && (kv->v_row_stride < s.v_dim || kv->v_row_stride % 8 != 0)))
    return fail(TLS_ERR_INVALID_ARG, "sparse_decode_attn_noalloc: bad row strides");
  if (kv->slot_of_block != nullptr && kv->n_slots < 1)
    return fail(TLS_ERR_INVALID_ARG, "sparse_decode_attn_noalloc: n_slots must be >= 1 with a slot table");
  if (out_dtype != TLS_OUT_F32 && out_dtype != TLS_OUT_BF16)
    return fail(TLS_ERR_INVALID_ARG, "sparse_decode_attn_noalloc: bad out_dtype");
  if (k < 1 || k > s.ctx_len) return fail(TLS_ERR_INVALID_ARG, "sparse_decode_attn_noalloc: k %d out of range", k);
  const int64_t nb = n_blocks(s);
  int K_b = (int)((k + s.block_size - 1) / s.block_size);
  if (K_b > nb) K_b = (int)nb;
  WsLayout L;
  st = plan_workspace(s, K_b, k, &L);
  if (st != TLS_OK) return st;
  // the error word (256-byte header), the tickets, then the partials, inside the static array
  const size_t header = 256;
  const size_t ticket_bytes = align_up((size_t)rows_of(s) * L.head_groups * sizeof(unsigned), 256);
  const size_t partial_bytes = (size_t)rows_of(s) * group_of(s) * L.splits * (s.v_dim + 2) * sizeof(float);
  if (header + ticket_bytes + partial_bytes > (size_t)TLS_NOALLOC_SCRATCH_BYTES)
    return fail(TLS_ERR_CAPACITY,
                "sparse_decode_attn_noalloc: this shape needs %zu bytes of scratch, above the fixed %u-byte "
                "array; use tls_sparse_decode_attn with a workspace",
                header + ticket_bytes + partial_bytes, (unsigned)TLS_NOALLOC_SCRATCH_BYTES);
  void* base = nullptr;
  st = noalloc_scratch(&base);
  if (st != TLS_OK) return st;
  // the array keeps the previous call's contents: error word and tickets must start at zero
  cudaError_t e = cudaMemsetAsync(base, 0, header + ticket_bytes, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_check(e, "sparse_decode_attn_noalloc: clear tickets");
  WsLayout S = L;
  S.err = 0;
  S.att_counter = header;
  S.partial = header + ticket_bytes;
  return sparse_attn_impl(s, q, *kv, token_idx, k, out_dtype, out, lse, (uint8_t*)base, S, (cudaStream_t)stream,
                          /*pdl=*/true);
}
