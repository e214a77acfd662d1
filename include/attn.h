/*
 * attn.h — C ABI of libattn.so: exact long-context attention on NVIDIA B200 (sm_100a).
 *
 * The library computes exact scaled-dot-product attention
 *     O = softmax(scale * Q K^T + causal mask) V
 * with grouped-query heads, tile by tile with an online softmax so the S x T score
 * matrix never exists in memory; decode splits the key range into partials that a
 * log-sum-exp reduce merges exactly, over bf16, FP8 E4M3, INT8 or INT4 caches (contiguous or
 * paged) whose dequantisation happens inside the tile load; a host streamer feeds (query block, key chunk)
 * sub-tasks from pinned host memory under a device-memory budget and merges their
 * partials the same way.
 *
 * Sources for the operations (web pages; titles and sections):
 *   [CQSA]  "Stream-CQSA: avoiding out-of-memory in attention computation through flexible
 *           workload scheduling" (euno.news summary of arXiv 2604.20819), Methodology 1-4,
 *           Results.
 *   [COOPT] "LLM-CoOpt: a co-design and optimization framework for efficient LLM inference on
 *           heterogeneous platforms" (euno.news summary of arXiv 2602.09323), Methodology 1-3.
 *   [ORT-CPU] "ONNX Runtime CPU GQA optimization: Flash Attention and Flash Decoding"
 *           (analysis of onnxruntime PR 28695), Code analysis 1-2, Reviewer feedback.
 *   [ORT-QSA] "ONNX Runtime CUDA packed sparse attention optimization" (analysis of
 *           onnxruntime PR 33328), Code analysis 1 (packed tokens, positions) and 2 (multi-token
 *           verification).
 *
 * Conventions for every entry point
 *   - Device pointers are plain CUDA device addresses owned by the caller; the library never
 *     frees or keeps them.  Host pointers are used only during the call.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).  Device
 *     calls enqueue work and return without synchronising, except attn_chunked_stream, which
 *     returns after its last device-to-host copy has completed.
 *   - Every argument is validated before any CUDA call; an invalid call returns an error
 *     status, launches nothing and never aborts or prints.
 *   - Layouts are row-major.  Q and O are token-major [B, S, Hq, D]; K and V are
 *     [B, T, Hkv, D]; the row log-sum-exp LSE is float32 [B, S, Hq] (same row order as O),
 *     natural log, including the score scale.  Query head h reads KV head h / (Hq / Hkv).
 *   - Supported: D in {64, 128}; bf16 Q/K/V; FP8 E4M3, INT8 and INT4 K/V codes with per-token
 *     float32 scales (decode, D = 128); Hq % Hkv == 0; Hq / Hkv <= 16 for decode.  All base
 *     pointers 16-byte aligned.
 *   - Thread safety: calls may be made from several host threads at once.
 */
#ifndef ATTN_H_
#define ATTN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1, /* bad pointer, size, alignment or combination */
  ATTN_ERR_UNSUPPORTED = 2, /* valid request outside what the kernels implement (e.g. D=96) */
  ATTN_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed; see attn_last_cuda_error() */
  ATTN_ERR_BUDGET = 4,      /* the streamer's smallest plan does not fit the device budget */
  ATTN_ERR_TIMEOUT = 5,     /* a kernel's bounded wait ran out (device status word) */
  ATTN_ERR_INJECTED = 6     /* a host-side injected failure (tests of the error paths) */
} attn_status_t;

/* Element types.  ATTN_INT8 / ATTN_INT4 are KV-cache codes only ([ORT-CPU] INT8/INT4 KV cache,
 * V dequantised on the fly in the SV accumulation; the page gives no encoding, so the reading is
 * two's complement with one float32 scale per (token, KV head)): INT8 one signed byte per element;
 * INT4 two signed 4-bit elements per byte, element 2i in the low nibble of byte i, so a row of D
 * elements is D/2 bytes. */
typedef enum { ATTN_BF16 = 0, ATTN_FP8_E4M3 = 1, ATTN_F32 = 2, ATTN_INT8 = 3, ATTN_INT4 = 4 } attn_dtype_t;

typedef struct {
  int B;       /* batch */
  int Hq;      /* query heads */
  int Hkv;     /* key/value heads; Hq % Hkv == 0 ([COOPT] Opt-GQA: heads share K/V in groups) */
  int D;       /* head dimension, 64 or 128 */
  float scale; /* score scale > 0, normally 1/sqrt(D) */
} attn_dims_t;

/* ------------------------------------------------------------------------------------------
 * attn_prefill — exact (optionally causal) GQA attention of S query rows over T keys.
 *
 * Follows [ORT-CPU] Code analysis 1 (tiled computation: per key block, score block, online
 * softmax running max and sum, fused P·V accumulation) on tcgen05 tensor cores, with the
 * definition of [CQSA] Methodology 2.  Query row i sits at absolute position q_pos0 + i, key j
 * at kv_pos0 + j ([ORT-QSA] Code analysis 1: position = past length + local index); with
 * causal != 0 row i sees key j iff kv_pos0 + j <= q_pos0 + i.  Tiles wholly above the
 * diagonal or past T are never computed.
 *
 *   q    device bf16 [B, S, Hq, D]     k, v  device bf16 [B, T, Hkv, D]
 *   o    device [B, S, Hq, D], bf16 (o_dtype = ATTN_BF16) or float32 (ATTN_F32)
 *   lse  device float32 [B, S, Hq] (always packed) or NULL.  Rows that see no key get O = 0,
 *        LSE = -inf.
 *   S, T >= 0 (S = 0 or B = 0 is a no-op); q_pos0, kv_pos0 >= 0.
 *   strides  host array of 12 element strides, or NULL for packed [B, S, H, D] tensors:
 *        {q_b, q_s, q_h, k_b, k_s, k_h, v_b, v_s, v_h, o_b, o_s, o_h}, the distance in elements
 *        between consecutive batches, tokens and heads of q, k, v and o; the D elements of a head
 *        are always contiguous.  Views such as one slice of a fused [B, S, Hq + 2 Hkv, D] QKV
 *        tensor, a subset of heads, or a [B, H, S, D] tensor seen as [B, S, H, D] are read in
 *        place, with no copy ([ORT-QSA] Code analysis 1: Q, K and V packed in one tensor).  Each
 *        stride must be positive and a whole number of 16-byte units (a multiple of 8 elements;
 *        of 4 for a float32 o); the array is read during the call only.  The caller keeps the
 *        rows o addresses disjoint.
 * Errors: ATTN_ERR_INVALID_ARG for bad sizes, strides, null or misaligned pointers;
 * ATTN_ERR_UNSUPPORTED for other head dims; ATTN_ERR_CUDA if the driver refuses a tensor map.
 * Returns ATTN_OK after enqueueing on `stream`.
 * ------------------------------------------------------------------------------------------ */
ATTN_API attn_status_t attn_prefill(const void* q, const void* k, const void* v, void* o, attn_dtype_t o_dtype,
                           float* lse, attn_dims_t dims, int S, int T, int causal, long long q_pos0,
                           long long kv_pos0, const long long* strides, void* stream);

/* ------------------------------------------------------------------------------------------
 * attn_prefill_varlen — attn_prefill over a packed batch of sequences of different lengths,
 * with no padding.
 *
 * [ORT-QSA] Code analysis 1: tokens of all sequences are packed along one axis and cut by
 * cumulative sequence lengths; a new token's position is the sequence's past length plus its
 * index among the new tokens.  Sequence b's queries are rows cu_seqlens_q[b] ..
 * cu_seqlens_q[b+1]-1 of q, o and lse; its keys are rows cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1
 * of k and v (past tokens first, then the new ones), so query i of a sequence with Sq queries and
 * Sk keys sits at position Sk - Sq + i and, when causal, sees keys [0, Sk - Sq + i].  Rows with no
 * visible key get O = 0, LSE = -inf.
 *
 *   q, o          device [total_q, Hq, D] (q bf16; o bf16 or float32 per o_dtype)
 *   k, v          device bf16 [total_k, Hkv, D]
 *   lse           device float32 [total_q, Hq] or NULL
 *   cu_seqlens_q  device int32 [B + 1], non-decreasing, cu_seqlens_q[0] = 0, cu_seqlens_q[B] = total_q
 *   cu_seqlens_k  device int32 [B + 1], likewise ending at total_k
 *   max_seqlen_q  the largest query count of any sequence (host value: sizes the grid; the device
 *                 lengths are never read back)
 *   dims.B        number of sequences; D in {64, 128}; scale as in dims
 * Errors: ATTN_ERR_INVALID_ARG for bad sizes, null or misaligned pointers; ATTN_ERR_UNSUPPORTED for
 * other head dims.  Cumulative lengths that break the rules above give rows with no keys, never an
 * out-of-bounds read (TMA boxes past the packed tensors land as zeros).
 * ------------------------------------------------------------------------------------------ */
ATTN_API attn_status_t attn_prefill_varlen(const void* q, const void* k, const void* v, void* o, attn_dtype_t o_dtype,
                                  float* lse, attn_dims_t dims, const int* cu_seqlens_q, const int* cu_seqlens_k,
                                  int total_q, int total_k, int max_seqlen_q, int causal, void* stream);

/* ------------------------------------------------------------------------------------------
 * attn_decode_splitkv — one query token per sequence over a ragged KV cache.
 *
 * Flash Decoding ([ORT-CPU] Code analysis 2): the key range of each (sequence, KV head) is cut
 * into num_splits chunks, each producing a partial softmax state, and a log-sum-exp reduce
 * merges them.  Sequence b's query sits at position kv_lens[b] - 1 and sees keys
 * [0, kv_lens[b]).  Lengths stay on the device (no host read-back).  Cache slots at or past
 * kv_lens[b] are never used, whatever they hold (NaN included).  kv_lens[b] == 0 gives O = 0,
 * LSE = -inf.
 *
 *   q        device bf16 [B, Hq, D]
 *   k, v     device [B, Tmax, Hkv, D]: bf16 (kv_dtype = ATTN_BF16), E4M3 codes (ATTN_FP8_E4M3) or
 *            INT8 codes (ATTN_INT8); [B, Tmax, Hkv, D/2] packed INT4 codes (ATTN_INT4)
 *   k_scale, v_scale  device float32 [B, Tmax, Hkv] dequantisation multipliers for the FP8 and
 *            integer caches ([COOPT] Opt-KV FP8 cache, [ORT-CPU] INT8/INT4 cache); must be NULL for
 *            bf16.  Dequantised value = code * scale.  Integer caches: |v_scale| is clamped to
 *            [2^-100, 2^100] and |q| must stay below 2^114 (each query row is carried as f16
 *            scaled by a power of two).
 *   kv_lens  device int32 [B], each in [0, Tmax]
 *   num_splits  0 = automatic (fills the GPU), else 1..4096
 *   o        device bf16 [B, Hq, D];  lse  device float32 [B, Hq] or NULL
 *   ws       device workspace of at least attn_decode_workspace_bytes(dims, Tmax, num_splits)
 *            bytes, owned by the caller; may be NULL when that size is 0.
 * ------------------------------------------------------------------------------------------ */
ATTN_API size_t attn_decode_workspace_bytes(attn_dims_t dims, int Tmax, int num_splits);
ATTN_API int attn_decode_num_splits(attn_dims_t dims, int Tmax, int num_splits); /* the split count used */
ATTN_API attn_status_t attn_decode_splitkv(const void* q, const void* k, const void* v, attn_dtype_t kv_dtype,
                                  const float* k_scale, const float* v_scale, const int* kv_lens, int Tmax,
                                  attn_dims_t dims, int num_splits, void* o, float* lse, void* ws,
                                  size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------------------------
 * attn_decode_multi — n_q query tokens per sequence over one KV cache (multi-token decode,
 * e.g. verifying n_q draft tokens).
 *
 * [ORT-QSA] Code analysis 2 (multi-token verification; positions of packed tokens): a new
 * token's absolute position is the past length plus its index among the new tokens.  Here the cache already holds the n_q
 * new tokens, so token i of sequence b sits at position kv_lens[b] - n_q + i and sees keys
 * [0, kv_lens[b] - n_q + i + 1) (a token with no visible key gets O = 0, LSE = -inf).  One pass
 * over the cache serves all n_q tokens: their n_q * Hq/Hkv query rows share each K/V tile, which
 * requires n_q * Hq/Hkv <= 16.  n_q = 1 is attn_decode_splitkv.
 *
 *   q      device bf16 [B, n_q, Hq, D];  o device bf16 [B, n_q, Hq, D];  lse float32 [B, n_q, Hq]
 *   ws     at least attn_decode_multi_workspace_bytes(dims, Tmax, n_q, num_splits) bytes
 *   other arguments, layouts and errors as for attn_decode_splitkv, except that the cache is
 *   bf16 or FP8: integer caches (ATTN_INT8, ATTN_INT4) give ATTN_ERR_UNSUPPORTED
 * ------------------------------------------------------------------------------------------ */
ATTN_API size_t attn_decode_multi_workspace_bytes(attn_dims_t dims, int Tmax, int n_q, int num_splits);
ATTN_API attn_status_t attn_decode_multi(const void* q, const void* k, const void* v, attn_dtype_t kv_dtype,
                                const float* k_scale, const float* v_scale, const int* kv_lens, int Tmax, int n_q,
                                attn_dims_t dims, int num_splits, void* o, float* lse, void* ws, size_t ws_bytes,
                                void* stream);

/* ------------------------------------------------------------------------------------------
 * attn_decode_paged — attn_decode_splitkv over a paged KV cache.
 *
 * [COOPT] Opt-Pa: sequences are cut into fixed-size pages (e.g. 512 tokens) and only pages that
 * are mapped are ever touched ("lazy mapping").  Here the cache is a pool of pages shared by all
 * sequences and a page table maps sequence b's logical page i (tokens i*page_size .. +page_size-1)
 * to a pool page.  Only the pages covering [0, kv_lens[b]) are read; table entries past them are
 * never read and may hold anything (-1 for unmapped).  Same split-KV method, outputs, scaling and
 * workspace rule as attn_decode_splitkv, with Tmax = max_pages * page_size.
 *
 *   q                 device bf16 [B, Hq, D]
 *   k_pool, v_pool    device [num_pages, page_size, Hkv, D]: bf16, E4M3 or INT8 codes (kv_dtype);
 *                     [num_pages, page_size, Hkv, D/2] packed INT4 codes
 *   k_scale_pool, v_scale_pool  device float32 [num_pages, page_size, Hkv] for the FP8 and integer
 *                     caches, else NULL
 *   page_table        device int32 [B, max_pages]; entries used must lie in [0, num_pages)
 *   page_size         a multiple of 128 (a 128-token tile never straddles two pages)
 *   kv_lens           device int32 [B], each in [0, max_pages * page_size]
 *   num_splits, o, lse, ws, ws_bytes, stream  as for attn_decode_splitkv; the workspace size is
 *                     attn_decode_workspace_bytes(dims, max_pages * page_size, num_splits)
 * Errors: ATTN_ERR_INVALID_ARG for bad sizes, null or misaligned pointers; a page-table entry
 * outside [0, num_pages) met on the device is never dereferenced (its tokens read as zeros) and
 * is reported later by attn_device_status as ATTN_ERR_INVALID_ARG (site 44).
 * ------------------------------------------------------------------------------------------ */
ATTN_API attn_status_t attn_decode_paged(const void* q, const void* k_pool, const void* v_pool, attn_dtype_t kv_dtype,
                                const float* k_scale_pool, const float* v_scale_pool, const int* page_table,
                                int max_pages, int page_size, int num_pages, const int* kv_lens, attn_dims_t dims,
                                int num_splits, void* o, float* lse, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------------------------
 * attn_decode_splitkv_noalloc — the same split-KV decode, for callers that cannot allocate.
 *
 * The pages have no counterpart to this entry point; it is an integration aid.  Some callers
 * cannot call cudaMalloc or hand out a workspace: a serving engine that has reserved nearly
 * all device memory for its own pool, or a latency-critical decode loop in which an allocation
 * (which may synchronise the device) is not allowed.  This variant takes the same arguments as
 * attn_decode_splitkv minus the workspace, and keeps the split partials in one static device
 * array of ATTN_NOALLOC_SCRATCH_BYTES that every GPU which loads the library holds until the
 * process exits.  It allocates nothing.
 *
 *   - The first call on a device (with that device current) looks up the array's device
 *     address; make that first call before any stream capture.  The address is kept with the
 *     device's context and looked up again if that context changes (e.g. after cudaDeviceReset,
 *     which reloads the library's device code).
 *   - The arguments are checked first, exactly as attn_decode_splitkv checks them (an invalid or
 *     unsupported call gets that status whatever its size); the scratch limit after them.
 *   - Requests whose partials need more than ATTN_NOALLOC_SCRATCH_BYTES
 *     (attn_decode_workspace_bytes(dims, Tmax, num_splits) > the limit) return ATTN_ERR_BUDGET
 *     without launching anything; lower num_splits or use attn_decode_splitkv.
 *   - All calls share the array and it keeps the last call's contents.  Nothing in it needs to
 *     start at zero (every partial is written before it is read), but calls whose work
 *     overlaps on the GPU (other streams, other host threads) race on it: serialise them.
 * ------------------------------------------------------------------------------------------ */
#define ATTN_NOALLOC_SCRATCH_BYTES (4u << 20)
ATTN_API attn_status_t attn_decode_splitkv_noalloc(const void* q, const void* k, const void* v, attn_dtype_t kv_dtype,
                                          const float* k_scale, const float* v_scale, const int* kv_lens,
                                          int Tmax, attn_dims_t dims, int num_splits, void* o, float* lse,
                                          void* stream);

/* ------------------------------------------------------------------------------------------
 * attn_merge_lse — exact log-sum-exp merge of P partial results per row.
 *
 * [ORT-CPU] Code analysis 2 (the reduce phase that merges per-chunk partial softmax states by
 * log-sum-exp) and [CQSA] Methodology 2-3 (sub-results recombine to the full result):
 * lse = log sum_p exp(lse_p),
 * o = sum_p exp(lse_p - lse) o_p; parts with lse_p = -inf add nothing; a row with every part
 * empty gets o = 0, lse = -inf.
 *
 *   o_parts   device float32 [P, R, D];  lse_parts device float32 [P, R]
 *   o_out     device [R, D], bf16 or float32 (o_dtype);  lse_out device float32 [R] or NULL
 *   accumulate != 0: (o_out, lse_out) already hold a partial (o_out float32, lse_out non-NULL)
 *             that is merged in place with the P parts.
 *   P >= 1 (P = 0 valid only with accumulate), R >= 0, D in {64, 128}.
 * ------------------------------------------------------------------------------------------ */
ATTN_API attn_status_t attn_merge_lse(const float* o_parts, const float* lse_parts, int P, long long R, int D,
                             void* o_out, attn_dtype_t o_dtype, float* lse_out, int accumulate, void* stream);

/* ------------------------------------------------------------------------------------------
 * Streamer: exact causal (or full) self-attention over S tokens whose Q, K, V, O, LSE live in
 * host memory, computed under a device-memory budget.
 *
 * [CQSA] Methodology 2-4: attention is split into independent sub-tasks — here (query block,
 * key chunk) rectangles that cover every visible (query, key) pair exactly once — queued and
 * streamed host->device on a copy stream, computed on the compute stream, and recombined by
 * the log-sum-exp merge (inside each task's kernel); finished blocks are swapped back to host
 * memory on a stream of their own.  A controller picks the block sizes from the budget ([CQSA]
 * Methodology 4; its Limitations section calls the block-size rule a plain heuristic): the query
 * block that fits and sends the fewest key chunks across the host link.
 *
 *   q_h, k_h, v_h  host bf16 [B, S, Hq, D] / [B, S, Hkv, D]; pinned memory lets copies overlap
 *   o_h            host bf16 [B, S, Hq, D];  lse_h host float32 [B, S, Hq] or NULL
 *   chunk_tokens   key chunk length (0 = the controller picks); multiple of 128
 *   device_budget_bytes  upper bound on every device allocation the call makes
 *   compute_stream, copy_stream: cudaStream_t or NULL (the call then creates its own)
 *   stats          optional out-parameter
 * Allocates device buffers (counted against the budget) and frees them before returning.
 * Returns ATTN_ERR_BUDGET, without allocating, if the smallest plan does not fit.
 * ------------------------------------------------------------------------------------------ */
typedef struct {
  long long q_block;      /* query rows per block */
  long long kv_chunk;     /* keys per chunk */
  long long n_tasks;      /* (query block, key chunk) sub-tasks */
  long long device_bytes; /* bytes the plan allocates on the device */
} attn_stream_plan_t;

/* Timings are CUDA-event times on the stream that runs each step (0 when the call failed). */
typedef struct {
  attn_stream_plan_t plan;
  long long h2d_bytes;     /* host->device bytes copied */
  long long d2h_bytes;     /* device->host bytes copied */
  double ms_total;         /* wall time of the call (host clock), set-up and frees included */
  double ms_compute;       /* compute stream, from its first launch to its last */
  double ms_device;        /* device span from the first upload to the end of the last copy back */
  double ms_compute_busy;  /* summed time of the compute steps (prefill tasks and block finishes):
                              the span the call would take with every copy hidden */
  double ms_h2d;           /* summed time of the host->device copies (copy stream) */
  double ms_d2h;           /* summed time of the device->host copies (their own stream) */
} attn_stream_stats_t;

ATTN_API attn_status_t attn_stream_plan(attn_dims_t dims, long long S, int causal, long long chunk_tokens,
                               size_t device_budget_bytes, attn_stream_plan_t* plan);
/* The idx-th task of a plan in execution order: first query row and first key of its rectangle. */
ATTN_API attn_status_t attn_stream_task(const attn_stream_plan_t* plan, long long S, int causal, long long idx,
                               long long* q_start, long long* kv_start);
ATTN_API attn_status_t attn_chunked_stream(const void* q_h, const void* k_h, const void* v_h, void* o_h, float* lse_h,
                                  attn_dims_t dims, long long S, int causal, long long chunk_tokens,
                                  size_t device_budget_bytes, void* compute_stream, void* copy_stream,
                                  attn_stream_stats_t* stats);

/* ------------------------------------------------------------------------------------------
 * Status and diagnostics
 * ------------------------------------------------------------------------------------------ */
ATTN_API const char* attn_status_string(attn_status_t status);
/* Last CUDA error code seen by this host thread inside the library (0 = none). */
ATTN_API int attn_last_cuda_error(void);
/* Reads the device status word of the current device (synchronises the device).  Returns
 * ATTN_ERR_TIMEOUT if a kernel's bounded wait ran out since the last reset, ATTN_ERR_INVALID_ARG
 * if a decode kernel met a page-table entry outside the pool, and stores the site in *site when
 * site != NULL.  reset != 0 clears the word. */
ATTN_API attn_status_t attn_device_status(int reset, int* site);
/* Upper bound of any single in-kernel wait, in nanoseconds (default 2e9). */
ATTN_API attn_status_t attn_set_wait_limit_ns(unsigned long long ns);
/* Launches one tiny kernel that waits on an mbarrier nothing ever arrives at, with the given
 * limit; the wait runs out, the kernel records ATTN_ERR_TIMEOUT and returns.  Used to test
 * the timeout path without faulting or hanging the GPU.  Synchronises the device. */
ATTN_API attn_status_t attn_debug_wait_probe(unsigned long long limit_ns);
/* Evaluates the kernels' exp2 on n device floats: mode 0 = the FMA-pipe polynomial the prefill
 * softmax uses for one exponential pair in eight, mode 1 = the MUFU ex2.approx.  For tests. */
ATTN_API attn_status_t attn_debug_exp2(const float* x, float* y, long long n, int mode, void* stream);
/* Host-side fault injection for the streamer: the nth (1-based) host->device copy (what = 1)
 * or device allocation (what = 2) of the next attn_chunked_stream call fails with
 * ATTN_ERR_INJECTED.  what = 0 disarms. */
ATTN_API attn_status_t attn_debug_inject(int what, long long nth);

#ifdef __cplusplus
}
#endif
#endif /* ATTN_H_ */
