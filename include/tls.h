/*
 * tls.h -- C ABI of libtls, the two-level sparse decode step of AsyncTLS on
 * NVIDIA B200 (sm_100a).
 *
 * Source of the method: "AsyncTLS: Efficient Generative LLM Inference with
 * Asynchronous Two-level Sparse Attention" (gist.science technical summaries
 * in English, Italian and Japanese).  Section names below refer to the
 * English summary unless another page is named:
 *   2.A Stage 1  coarse block filtering: blocks, a block-level index, the
 *                Quest score recast as a GEMM, top-K_b blocks;
 *                (Italian 2.A.1: the block index is the max/min of the keys)
 *   2.A Stage 2  fine token selection inside the chosen blocks (Double
 *                Sparsity): selected channels, INT4 keys, top-K_t tokens;
 *                (Italian 2.A.2: attention runs on the chosen tokens only)
 *   2.B          asynchronous offloading engine: temporal locality, staggered
 *                execution, incremental transfer T_t = M_t \ C_t.
 *
 * Conventions for every call
 *   - Pointers named "device" point to GPU memory (cudaMalloc / torch CUDA
 *     tensors); "host" pointers point to CPU memory.  The caller owns every
 *     buffer; the library keeps no pointer after a call returns, except the
 *     handles of tls_block_cache_create and tls_engine_create, which keep the
 *     pointers given to them until destroyed.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Kernel calls are asynchronous on that stream.
 *   - bf16 is IEEE bfloat16 stored as 16-bit words; all tensors are dense,
 *     row-major and C-contiguous unless a row stride is given (in elements).
 *   - Arguments are validated before anything is launched.  A rejected call
 *     returns TLS_ERR_INVALID_ARG or TLS_ERR_UNSUPPORTED, launches nothing,
 *     and tls_last_error() describes why.  A failed launch returns
 *     TLS_ERR_CUDA.  Errors inside kernels that use bounded waits are
 *     reported through the workspace error word (tls_workspace_error).
 *   - Shapes: B batch, Hq query heads, Hkv KV heads (Hq % Hkv == 0,
 *     G = Hq / Hkv heads share one KV head), Dqk key dim, Dv value dim,
 *     N context capacity, bs block size, NB = N / bs, R label channels,
 *     "row" = one (batch, KV head) pair, rows = B * Hkv.
 *   - Ragged batches and partial blocks: sequence b holds len_b tokens,
 *     positions 0 .. len_b - 1 (tls_shape.seq_lens; all N when NULL).  Its
 *     blocks are j < ceil(len_b / bs); the last one may be partial.  Positions
 *     >= len_b are never scored, selected or attended.  When a sequence has
 *     fewer blocks than K_b, or its chosen blocks fewer tokens than k, the
 *     valid entries of its list come first (ascending) and the rest are -1.
 *     A sequence with len_b = 0 gets empty (all -1) lists, a zero output and
 *     lse = -inf.
 */
#ifndef TLS_H
#define TLS_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TLS_API __attribute__((visibility("default")))
#else
#define TLS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum tls_status {
  TLS_OK = 0,
  TLS_ERR_INVALID_ARG = 1,  /* bad shape, pointer, alignment or size */
  TLS_ERR_UNSUPPORTED = 2,  /* valid but not built (e.g. a head dim with no kernel) */
  TLS_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
  TLS_ERR_TIMEOUT = 4,      /* a bounded wait ran out (device word or host deadline) */
  TLS_ERR_CAPACITY = 5,     /* block cache has too few free slots */
  TLS_ERR_COPY = 6          /* a host->device block copy failed (or was failed on purpose) */
} tls_status;

typedef struct tls_shape {
  int32_t batch;        /* B >= 1 */
  int32_t n_q_heads;    /* Hq, a multiple of n_kv_heads */
  int32_t n_kv_heads;   /* Hkv >= 1 */
  int32_t qk_dim;       /* Dqk: multiple of 32, <= 640 */
  int32_t v_dim;        /* Dv: multiple of 8, <= 512 */
  int32_t v_offset;     /* -1: V is its own tensor; >= 0: V of a token is its K row
                           slice [v_offset, v_offset + v_dim) (MLA shared latent) */
  int32_t block_size;   /* bs: tokens per block, multiple of 8, <= 256 */
  int32_t n_label;      /* R: label channels, even, 2..64, <= qk_dim */
  int64_t ctx_len;      /* N: capacity of every sequence in tokens (the row stride of K/V and
                           of the index), a multiple of block_size */
  float softmax_scale;  /* logits are softmax_scale * q.k (e.g. 1/sqrt(Dqk)) */
  const int32_t* seq_lens; /* optional device int32 [B]: tokens present in each sequence, 0..N
                              (values outside are clamped); NULL: every sequence holds N */
} tls_shape;

/* Output element type of tls_sparse_decode_attn. */
enum { TLS_OUT_F32 = 0, TLS_OUT_BF16 = 1 };

/* Where the attention kernel finds K/V rows. */
typedef struct tls_kv_view {
  const void* k;           /* device bf16 K rows */
  const void* v;           /* device bf16 V rows; unused when v_offset >= 0 */
  int64_t k_row_stride;    /* elements between consecutive K rows (>= Dqk, multiple of 8) */
  int64_t v_row_stride;    /* elements between consecutive V rows (>= Dv, multiple of 8) */
  const int32_t* slot_of_block; /* NULL: dense cache, row r = b*Hkv + h, token t at
                                   k + (r*N + t) * k_row_stride.
                                   Else device int32 [B, Hkv, NB]: block -> slot in a
                                   shared pool; token t of block j at
                                   k + (slot*bs + t % bs) * k_row_stride. */
  int32_t n_slots;         /* pool size when slot_of_block != NULL */
} tls_kv_view;

/* Thread-local description of the last rejected or failed call ("" if none). */
TLS_API const char* tls_last_error(void);

/* Library version, major*10000 + minor*100 + patch. */
TLS_API int32_t tls_version(void);

/*
 * Copies `bytes` from pinned host memory that the device can address
 * (cudaHostAlloc, cudaHostRegister'd or pinned torch buffers) into device
 * memory with one kernel on `stream`, whose 16-byte loads cross PCIe: for a
 * decode step's small inputs (q), it starts sooner than a copy-engine
 * transfer, most of all inside a captured step.  src (host), dst (device) and
 * bytes must be multiples of 16 bytes; bytes = 0 does nothing.  The source
 * range is checked once per (address, size) (cudaPointerGetAttributes at
 * both ends; the result is remembered, so a captured call does not repeat
 * it): memory that is not pinned and mapped returns TLS_ERR_INVALID_ARG and
 * launches nothing.  The source must stay allocated while the copy runs.
 */
TLS_API tls_status tls_copy_from_host(void* dst_device, const void* src_host, size_t bytes, void* stream);

/*
 * Name of the attention kernel tls_sparse_decode_attn launches for this
 * shape: "sparse_attn_mma_cluster_kernel" or "sparse_attn_mma_kernel" for
 * 128-wide K and V rows (one cluster of CTAs per row and head group of <= 16
 * heads while such a grid fits two CTAs per SM; else persistent CTAs),
 * "sparse_attn_mla_kernel" for the MLA latent cache (Dqk 576, Dv 512 taken
 * from the same row, G a multiple of 16), and "sparse_attn_kernel" for every
 * other shape.  A
 * static string owned by the library; NULL if the shape is invalid
 * (tls_last_error says why).  Host only, no device work.
 */
TLS_API const char* tls_attn_kernel(const tls_shape* shape);

/*
 * Name of the level-2 kernel tls_select_tokens (staggered = 0: as in
 * tls_select and tls_decode_step) or an engine's step (staggered != 0: the
 * resident step and the device-planned offloaded step, which keep level 2 to
 * half the SMs) takes for this shape, K_b and k,
 * for 16-byte aligned codes and scales: "token_select_row_kernel",
 * "token_select_cluster_kernel" or "token_select_kernel".  cluster_ctas and
 * cta_threads (nullable, host) receive its CTAs per row (a thread-block
 * cluster when more than one) and threads per CTA.  A static string owned by
 * the library; NULL if the arguments are invalid (tls_last_error says why).
 * Host only, no device work.
 */
TLS_API const char* tls_token_kernel(const tls_shape* shape, int32_t K_b, int32_t k, int32_t staggered,
                                     int32_t* cluster_ctas, int32_t* cta_threads);

/*
 * Bytes of device workspace needed by tls_select_blocks, tls_select_tokens,
 * tls_sparse_decode_attn and tls_decode_step for this shape, K_b and k.
 * The workspace must be zero-filled once after allocation; every call that
 * completes leaves its counters at zero again, so it can be reused without
 * clearing.  Calls that run concurrently on different streams may share one
 * workspace only if they are different entry points (each uses its own
 * region); two concurrent calls of the same entry point need two workspaces.
 * Returns 0 if the shape is invalid.
 */
TLS_API size_t tls_workspace_bytes(const tls_shape* shape, int32_t K_b, int32_t k);

/*
 * Reads (and, if clear != 0, zeroes) the workspace error word on `stream`,
 * synchronising that stream.  *code = 0 when no kernel reported an error;
 * otherwise a TLS_ERR_* value set by a kernel whose bounded wait ran out.
 * ws = NULL reads the error word of tls_sparse_decode_attn_noalloc's fixed
 * array on the current device instead (each call of that entry point clears
 * it first, so it reports the last call's kernels).
 */
TLS_API tls_status tls_workspace_error(const void* ws, int32_t clear, int32_t* code, void* stream);

/*
 * Index build, part 1 (Stage 1 block-level index; Italian 2.A.1 max/min of
 * the keys).  For every row and every block j with t0 <= j*bs < t1 that
 * holds a token below e = min(t1, len_b):
 *   meta[row, j, c]       = max over the block's tokens t < e of K[row, t, c]
 *   meta[row, j, Dqk + c] = min over the block's tokens t < e of K[row, t, c]
 * (so a partial last block covers the tokens it holds; blocks with none are
 * left untouched).  k: device bf16, row r's token t at
 * k + (r*N + t) * k_row_stride.  meta: device bf16 [B, Hkv, NB, 2*Dqk].
 * t0 a multiple of bs, 0 <= t0 < t1 <= N.  The values are exact (max/min
 * picks an input).
 */
TLS_API tls_status tls_build_block_meta(const tls_shape* shape, const void* k, int64_t k_row_stride,
                                int64_t t0, int64_t t1, void* meta, void* stream);

/*
 * Index build, part 2 (Stage 2: channel selection + INT4 keys).  For every
 * row and token t0 <= t < min(t1, len_b), with x_r = K[row, t, label_ch[h, r]]:
 *   s = max_r |x_r| / 7                  (float32, IEEE division)
 *   code_r = rint(x_r / s) in [-7, 7]    (float32, ties to even; s = 0 -> 0)
 * codes: device uint8 [B, Hkv, N, R/2]; byte j holds code 2j in its low
 * nibble and code 2j+1 in its high nibble, two's complement.
 * scales: device float32 [B, Hkv, N].  label_ch: device int32 [Hkv, R],
 * each in [0, Dqk).  Codes and scales are bit-exact by this definition.
 */
TLS_API tls_status tls_quant_label_cache(const tls_shape* shape, const void* k, int64_t k_row_stride,
                                 const int32_t* label_ch, int64_t t0, int64_t t1,
                                 uint8_t* codes, float* scales, void* stream);

/*
 * Level 1 (Stage 1): block scores as one GEMM per row on tcgen05 tensor cores,
 *   S[h, j] = [relu(q_h), min(q_h, 0)] . [kmax_j ; kmin_j]   (fp32 accumulate)
 * which equals Quest's sum_c max(q_hc*kmax_jc, q_hc*kmin_jc); the G heads of
 * a row combine by max: agg[row, j] = max_h S[h, j].  Then the K_b blocks
 * with the largest agg (ties: lower block index) are written ascending.
 * q: device bf16 [B, Hq, Dqk] (16-byte aligned); meta as built above
 * (16-byte aligned).  block_idx: device int32 [B, Hkv, K_b]; only blocks
 * holding tokens of the sequence compete (the list is padded with -1 past
 * them).  block_score: optional device float32 [B, Hkv, NB] receiving agg
 * (-inf for blocks past the sequence).  1 <= K_b <= NB, NB <= 16384.
 */
TLS_API tls_status tls_select_blocks(const tls_shape* shape, const void* q, const void* meta, int32_t K_b,
                             int32_t* block_idx, float* block_score,
                             void* ws, size_t ws_bytes, void* stream);

/*
 * Level 2 (Stage 2): for each candidate token t of the row's K_b chosen
 * blocks (candidates in ascending token order),
 *   score(t) = max_h  s_t * sum_r q_h[label_ch[h_kv, r]] * code_{t, r}
 * then the k best candidates (ties: lower token index) are written
 * ascending as absolute token positions.  Candidates are the positions
 * below len_b of the listed blocks; entries -1 of the list end it.
 * block_idx: device int32 [B, Hkv, K_b], ascending per row with any -1 at
 * the end (as written by tls_select_blocks).  token_idx: device int32
 * [B, Hkv, k], padded with -1 past the candidates.  token_score: optional
 * device float32 [B, Hkv, K_b*bs] receiving the candidate scores (-inf past
 * the candidates).  1 <= k <= K_b*bs <= 524288.
 */
TLS_API tls_status tls_select_tokens(const tls_shape* shape, const void* q, const int32_t* label_ch,
                             const uint8_t* codes, const float* scales, const int32_t* block_idx,
                             int32_t K_b, int32_t k, int32_t* token_idx, float* token_score,
                             void* ws, size_t ws_bytes, void* stream);

/*
 * Attention over the chosen tokens only (Italian 2.A.2).  For each query
 * head h of row (b, kv) with its row's token list T (token_idx, k entries):
 *   p = softmax(softmax_scale * q_h . K[T]^T),  out[b, h] = p . V[T]
 *   lse[b, h] = log(sum_t exp(softmax_scale * q_h . K_t))   (natural log)
 * bf16 inputs, fp32 products, fp32 softmax and accumulation; split-K over
 * the token list with a log-sum-exp merge inside the same launch.
 * out: device [B, Hq, Dv], float32 (out_dtype TLS_OUT_F32) or bf16
 * (TLS_OUT_BF16, round to nearest even).  lse: optional device float32 [B, Hq].
 * Entries outside [0, len_b) (the -1 padding of a selection) are skipped;
 * with a slot table, every block a valid entry falls in must map to a slot
 * in [0, n_slots) (slots are clamped into the pool on the device).  A row
 * with no valid entry gets a zero output and lse = -inf.  1 <= k <= N.
 */
TLS_API tls_status tls_sparse_decode_attn(const tls_shape* shape, const void* q, const tls_kv_view* kv,
                                  const int32_t* token_idx, int32_t k, int32_t out_dtype,
                                  void* out, float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * Levels 1 and 2 together: tls_select_blocks followed by tls_select_tokens
 * on `stream` (two kernel launches, one shared workspace); the same results
 * as the two calls.  Arguments as in the two calls.
 */
TLS_API tls_status tls_select(const tls_shape* shape, const void* q, const void* meta, const int32_t* label_ch,
                              const uint8_t* codes, const float* scales, int32_t K_b, int32_t k,
                              int32_t* block_idx, int32_t* token_idx, void* ws, size_t ws_bytes, void* stream);

/*
 * One decode step: tls_select then tls_sparse_decode_attn on `stream` (three
 * kernel launches), sharing one workspace; the same results as those calls.
 * block_idx / token_idx are outputs as above.  Every argument either call
 * would reject is checked before anything is launched.
 */
TLS_API tls_status tls_decode_step(const tls_shape* shape, const void* q, const void* meta,
                           const int32_t* label_ch, const uint8_t* codes, const float* scales,
                           const tls_kv_view* kv, int32_t K_b, int32_t k,
                           int32_t* block_idx, int32_t* token_idx, int32_t out_dtype,
                           void* out, float* lse, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Operator baselines (English summary 4, Efficiency: the method is compared
 * with full attention and with each level alone -- Quest's block selection,
 * Double Sparsity's token selection).  Same numerics and output conventions
 * as tls_sparse_decode_attn; each takes a workspace of the size given.
 * ------------------------------------------------------------------------ */

/*
 * Full attention: every token a sequence holds (positions 0 .. len_b - 1),
 * with no selection.  Workspace: tls_workspace_bytes(shape, NB, N).
 */
TLS_API tls_status tls_dense_decode_attn(const tls_shape* shape, const void* q, const tls_kv_view* kv,
                                         int32_t out_dtype, void* out, float* lse, void* ws, size_t ws_bytes,
                                         void* stream);

/*
 * Block selection alone (Quest): level 1 as tls_select_blocks writes
 * block_idx, then attention over every token of the K_b chosen blocks
 * (K_b * bs positions, no level 2).  Two launches.  Workspace:
 * tls_workspace_bytes(shape, K_b, K_b * bs).
 */
TLS_API tls_status tls_quest_decode_step(const tls_shape* shape, const void* q, const void* meta,
                                         const tls_kv_view* kv, int32_t K_b, int32_t* block_idx,
                                         int32_t out_dtype, void* out, float* lse, void* ws, size_t ws_bytes,
                                         void* stream);

/*
 * Token selection alone (Double Sparsity): level 2 over every token of the
 * sequence (K_b = NB, no level 1) writes token_idx (k entries), then the
 * attention over them.  Two launches.  Workspace:
 * tls_workspace_bytes(shape, NB, k).
 */
TLS_API tls_status tls_ds_decode_step(const tls_shape* shape, const void* q, const int32_t* label_ch,
                                      const uint8_t* codes, const float* scales, const tls_kv_view* kv, int32_t k,
                                      int32_t* token_idx, int32_t out_dtype, void* out, float* lse, void* ws,
                                      size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Appending the decoded token (English summary 2.A: the KV cache is split
 * into blocks with a block-level index and an INT4 label cache; a decode step
 * adds one token to each sequence, and with it to the index).
 * ------------------------------------------------------------------------ */

/*
 * For every sequence b with t = seq_lens[b] < N and every KV head h: writes
 * k_new[b, h] as K row t and v_new[b, h] as V row t (through kv: dense, or
 * the slot of block t / bs in the slot table, which must be >= 0), updates
 * the block-level index of block t / bs -- meta = (k, k) when t starts the
 * block, else the channel-wise max / min with k -- quantises the token's
 * label channels into codes / scales (as tls_quant_label_cache), and then
 * sets seq_lens[b] = t + 1.  A full sequence (seq_lens[b] >= N) is left
 * unchanged.  One launch; the result equals building the index over the
 * grown sequence.
 * seq_lens: device int32 [B] (in/out; shape->seq_lens is ignored).
 * k_new: device bf16 [B, Hkv, Dqk]; v_new: device bf16 [B, Hkv, Dv], NULL
 * when v_offset >= 0 (the value is the K row slice).  kv.k / kv.v are written.
 */
TLS_API tls_status tls_append_kv(const tls_shape* shape, int32_t* seq_lens, const void* k_new, const void* v_new,
                                 const tls_kv_view* kv, void* meta, const int32_t* label_ch, uint8_t* codes,
                                 float* scales, void* stream);

/*
 * Scratch-free variant of tls_sparse_decode_attn (no counterpart in the
 * paper; it is a convenience of this library).  Same inputs, outputs and
 * numerics, but it takes no workspace and allocates nothing: the split-K
 * partials and merge tickets live in one fixed device array of
 * TLS_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads
 * the library holds until the process exits.
 * Meant for callers that cannot allocate device memory: a plug-in inside a
 * serving runtime that owns the whole HBM budget and offers no allocator, or
 * a latency-critical decode loop where cudaMalloc (which may synchronise the
 * device) is not allowed.
 *   - The first call in a device's CUDA context looks up the array's device
 *     address (cudaGetSymbolAddress) with that device current and keeps it for
 *     that device and context; make that first call before any stream
 *     capture.  A context created later (e.g. after cudaDeviceReset) is looked
 *     up again on its own first call.
 *   - Each call clears the error word and the tickets with cudaMemsetAsync on
 *     `stream`; it calls no cudaMalloc, cudaFree or allocating library routine.
 *   - tls_workspace_error(NULL, ...) reads the error word of the last call.
 *   - All calls share the one array: two calls whose kernels overlap on the
 *     GPU (e.g. on different streams) race and give wrong results.  Issue them
 *     on one stream, or use tls_sparse_decode_attn with separate workspaces.
 *   - Shapes whose scratch exceeds the array (a 256-byte error header, the
 *     tickets and rows * G * splits * (Dv + 2) floats) return
 *     TLS_ERR_CAPACITY and launch nothing.
 */
#define TLS_NOALLOC_SCRATCH_BYTES (4u << 20)
TLS_API tls_status tls_sparse_decode_attn_noalloc(const tls_shape* shape, const void* q, const tls_kv_view* kv,
                                                  const int32_t* token_idx, int32_t k, int32_t out_dtype,
                                                  void* out, float* lse, void* stream);

/* ------------------------------------------------------------------------
 * Offloaded KV: HBM block cache with incremental transfer (section 2.B).
 * ------------------------------------------------------------------------ */
typedef struct tls_block_cache tls_block_cache;

/*
 * Creates the host-side state of a block cache.  Full K/V live in host
 * memory (pinned, for asynchronous copies): row r's token t at
 * host_k + (r*N + t) * host_k_row_stride (likewise V; host_v may be NULL when
 * v_offset >= 0).  The device pool holds n_slots blocks:
 * slot_k [n_slots, bs, host_k_row_stride] and slot_v [n_slots, bs,
 * host_v_row_stride] (bf16).  slot_table_dev: device int32 [B, Hkv, NB],
 * written by the library (-1 = not resident); the attention kernel reads it
 * through tls_kv_view.slot_of_block.  The handle allocates two small mapped
 * pinned staging buffers (max(B*Hkv*NB, 4*n_slots) int32 each) and nothing
 * on the device.
 * Any pointer may be NULL only for host-only use of tls_block_cache_plan.
 */
TLS_API tls_status tls_block_cache_create(const tls_shape* shape, const void* host_k, const void* host_v,
                                  int64_t host_k_row_stride, int64_t host_v_row_stride,
                                  int32_t n_slots, void* slot_k, void* slot_v,
                                  int32_t* slot_table_dev, tls_block_cache** out);
TLS_API void tls_block_cache_destroy(tls_block_cache* cache);

/*
 * Host-only planning of one incremental transfer (section 2.B): for every
 * row, T_t = M_t \ C_t where M_t = new_block_idx[row] and C_t is the set of
 * resident blocks.  Each block of T_t gets a victim slot that holds no block
 * of in_use_block_idx[row] (the blocks the running attention reads, M_{t-1})
 * nor of M_t, preferring free slots, then the least recently used, then the
 * lower slot; copy i (in row, then list order) takes the i-th victim in slot
 * order.  The plan is committed to the cache's host mirror.
 * new_block_idx, in_use_block_idx: host int32 [B, Hkv, K_b] (in_use may be
 * NULL for none).  copy_row/copy_block/copy_slot: host int32 arrays of
 * capacity B*Hkv*K_b receiving the plan (may be NULL); *n_copy = |T_t| summed
 * over rows.  Returns TLS_ERR_CAPACITY (and commits nothing) if victims run out.
 */
TLS_API tls_status tls_block_cache_plan(tls_block_cache* cache, const int32_t* new_block_idx,
                                const int32_t* in_use_block_idx, int32_t K_b,
                                int32_t* copy_row, int32_t* copy_block, int32_t* copy_slot,
                                int32_t* n_copy);

/*
 * Incremental prefetch (section 2.B): plans as tls_block_cache_plan, then
 * queues on copy_stream the copies of the planned blocks (K and V) from host
 * memory into their slots -- one kernel that reads them from mapped pinned
 * memory, or else one cudaMemcpyAsync per run of adjacent blocks -- and the
 * slot-table update: the first call writes the whole table, later calls
 * change only the entries of the copied and the evicted blocks.  Neither
 * touches a slot or an entry of in_use_block_idx_host, so an attention
 * reading those blocks may run concurrently.  The caller must order
 * copy_stream after every other kernel still reading a slot that may be
 * evicted (e.g. the attention of the step before).
 * done_event: optional cudaEvent_t (as void*), recorded on copy_stream after
 * the copies and the table update; a stream that makes the next attention
 * waits on it (cudaStreamWaitEvent) before reading the new blocks.  NULL:
 * the caller orders its work after copy_stream itself.
 * The host mirror is updated only once all device work is queued.  A failure
 * after some of it was queued marks the cache failed: that call and every
 * later tls_prefetch_diff or tls_block_cache_plan return TLS_ERR_COPY.
 * *n_copied = blocks copied.  Setting the environment variable
 * TLS_FAULT_INJECT=copy makes the copy step fail with TLS_ERR_COPY before
 * anything is issued (host-side fault injection for tests).
 */
TLS_API tls_status tls_prefetch_diff(tls_block_cache* cache, const int32_t* new_block_idx_host,
                             const int32_t* in_use_block_idx_host, int32_t K_b,
                             void* copy_stream, void* done_event, int32_t* n_copied);

/*
 * Incremental prefetch planned on the device (section 2.B), for block lists
 * that live on the device (as level 1 writes them): one kernel of one CTA
 * plans T_t = M_t \ C_t and its victims from new_block_idx_dev (M_t) and
 * in_use_block_idx_dev (M_{t-1}, may be NULL), updates the device slot table
 * and the cache state, and a second kernel pulls the planned blocks from
 * mapped pinned host memory into their slots -- both on copy_stream, with no
 * host wait.  The plan is the one tls_block_cache_plan makes (the same
 * victims and slots; the tables of the two paths are equal).
 * Each row of new_block_idx_dev must hold distinct blocks in [0, NB),
 * ascending, with any -1 at the end.  n_copied_dev: optional int32 in device
 * or mapped pinned memory, written on the device with the number of copied
 * blocks, or -1 when the plan failed (a list that breaks the rule above:
 * TLS_ERR_INVALID_ARG; too few evictable slots: TLS_ERR_CAPACITY); a failed
 * plan changes nothing, and the cache then returns that status from every
 * later transfer, plan or engine step.  done_event as in tls_prefetch_diff.
 * Needs a cache whose K/V are mapped pinned host memory (the pull path),
 * n_slots <= 32768, B*Hkv*K_b <= 65536, and the plan's shared memory within
 * 227 KB: 4 bytes per slot, per list entry and per possible victim
 * (min(n_slots, B*Hkv*K_b)), plus about 4 KB (else TLS_ERR_UNSUPPORTED).  From
 * the first call on, the device holds the cache state: the host calls
 * (tls_block_cache_plan, tls_prefetch_diff, tls_block_cache_table) first
 * wait for the device to finish (cudaDeviceSynchronize) and read it back.
 * TLS_FAULT_INJECT=copy fails the call with TLS_ERR_COPY before anything is
 * queued.
 */
TLS_API tls_status tls_prefetch_diff_device(tls_block_cache* cache, const int32_t* new_block_idx_dev,
                                            const int32_t* in_use_block_idx_dev, int32_t K_b, void* copy_stream,
                                            void* done_event, int32_t* n_copied_dev);

/* Copies the slot table (int32 [B, Hkv, NB]) into `table`: the host mirror,
 * or, once the device plans the cache, the device table after a
 * cudaDeviceSynchronize. */
TLS_API tls_status tls_block_cache_table(const tls_block_cache* cache, int32_t* table);

/* ------------------------------------------------------------------------
 * Staggered decode engine over a block cache (section 2.B: staggered
 * execution with incremental transfer).
 * ------------------------------------------------------------------------ */
typedef struct tls_engine tls_engine;

/* Transfer figures of one engine step (see tls_engine_stats). */
typedef struct tls_engine_step_stats {
  int64_t step;          /* the step whose transfer T_step these describe; -1 = the prologue (M_{-1}) */
  int32_t n_copied;      /* blocks copied, summed over rows */
  int64_t bytes_copied;  /* host -> device bytes of K and V */
  float copy_ms;         /* copy-stream time of the transfer (block copies and slot-table update) */
  float exposed_ms;      /* how long the attention of step+1 waited for this transfer past the point it
                            was otherwise ready to start; -1 when step+1 has not been issued */
} tls_engine_step_stats;

/*
 * Creates an engine for one attention layer whose K/V live in `cache` (created
 * with device buffers).  meta, label_ch, codes, scales: the resident index, as
 * in tls_select_blocks / tls_select_tokens.  block_idx: device int32
 * [2, B, Hkv, K_b], the engine's two block lists (M_t and M_{t-1}, alternating).
 * token_idx: device int32 [B, Hkv, k].  ws/ws_bytes: a workspace of
 * tls_workspace_bytes(shape, K_b, k) bytes, zero-filled, used by no other call
 * while the engine lives.  The engine keeps every pointer until destroyed and
 * allocates two streams, its events and two pinned host copies of a block list.
 */
TLS_API tls_status tls_engine_create(const tls_shape* shape, int32_t K_b, int32_t k, const void* meta,
                             const int32_t* label_ch, const uint8_t* codes, const float* scales,
                             tls_block_cache* cache, int32_t* block_idx, int32_t* token_idx, void* ws,
                             size_t ws_bytes, tls_engine** out);

/*
 * Creates an engine whose K/V are resident in HBM (`kv`, a dense view as in
 * tls_sparse_decode_attn; no block cache, no transfers): the staggered
 * schedule alone.  Other arguments and ownership as tls_engine_create; the
 * engine allocates one stream and its events.  Its steps never wait on the
 * host, so a step may be captured into a CUDA graph on its stream (each step
 * forks level 1 onto the engine's stream and joins it back before returning).
 * A captured step keeps the block-list parity of the step it was captured
 * at (it writes M_t into one of the two lists and reads M_{t-1} from the
 * other): capture two consecutive steps and replay the two graphs
 * alternately.  Captures count as steps in tls_engine_steps; replays do not.
 */
TLS_API tls_status tls_engine_create_resident(const tls_shape* shape, int32_t K_b, int32_t k, const void* meta,
                                      const int32_t* label_ch, const uint8_t* codes, const float* scales,
                                      const tls_kv_view* kv, int32_t* block_idx, int32_t* token_idx, void* ws,
                                      size_t ws_bytes, tls_engine** out);

/*
 * One decode step t with query q (device bf16 [B, Hq, Dqk], ready on
 * `stream`).  Output as tls_sparse_decode_attn (device memory), written on
 * `stream`.  Level 2
 * and the attention use the blocks chosen at step t-1 (M_{t-1}, resident in
 * the cache) with q; level 1 chooses M_t from q on the engine's second stream,
 * and the blocks of M_t not yet resident are copied from host memory on the
 * engine's copy stream while the attention runs; step t+1's attention waits
 * for them.  The first step selects M_{-1} from its own q and makes it
 * resident before attending.  When the cache allows it (as for
 * tls_prefetch_diff_device), the transfer is planned on the device
 * (tls_prefetch_diff_device on the copy stream, after level 1 and after the
 * attention of step t-1) and the call does not wait on the host at all; else,
 * or with TLS_ENGINE_PLANNER=host in the environment at engine creation, the
 * call waits on the host for level 1 of step t to plan it (tls_prefetch_diff).
 * A failed device plan is seen by the next step (or tls_engine_stats), which
 * returns its status.  A resident
 * engine (tls_engine_create_resident) has no transfer and no host wait: on
 * `stream` it records q_t, runs level 2 over M_{t-1} and the attention, and
 * waits for level 1 of step t (engine stream, after q_t) before returning, so
 * the next step's level 2 finds M_t complete.  The host waits (for level 1
 * of the step, and for the prologue's block list) have a deadline:
 * TLS_HOST_WAIT_MS milliseconds from the environment at engine creation, else
 * 10 s; when it passes the step returns TLS_ERR_TIMEOUT (the device work
 * completes on its own).  After a failed step (a timeout, a copy failure,
 * TLS_ERR_CAPACITY, a launch error) the cache no longer matches the block
 * lists: every later step returns the same error and the engine must be
 * destroyed.
 */
TLS_API tls_status tls_engine_step(tls_engine* engine, const void* q, int32_t out_dtype, void* out, float* lse,
                           void* stream);

/* Number of steps taken (-1 for a NULL engine). */
TLS_API int64_t tls_engine_steps(const tls_engine* engine);

/*
 * Kernel launches of one steady-state step (-1 for a NULL engine): level 1,
 * level 2 and the attention (plus level 1's query preparation for groups of
 * more than 32 heads); an offloaded engine adds the transfer's plan and pull
 * kernels (device planner) or its pull kernel (host planner).
 */
TLS_API int32_t tls_engine_step_kernels(const tls_engine* engine);

/*
 * Transfer figures of step `step` (-1 .. steps-1, among the last 255 steps);
 * waits for the events they need.  A resident engine reports no transfer
 * (zero blocks, bytes and times).
 */
TLS_API tls_status tls_engine_stats(tls_engine* engine, int64_t step, tls_engine_step_stats* out);

/* Waits for the engine's streams and releases it (not the caller's buffers). */
TLS_API void tls_engine_destroy(tls_engine* engine);

#ifdef __cplusplus
}
#endif

#endif /* TLS_H */
