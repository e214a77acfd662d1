// Host side of libattn.so: argument validation, TMA tensor maps, launch configuration and
// the status/diagnostic entry points.  Every device kernel of the library is compiled in
// this one translation unit, so the device status word exists once per device.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <algorithm>
#include <cstring>
#include <mutex>

#include "../../include/attn.h"
#include "internal.h"
#include "decode.cuh"
#include "decode_fp8.cuh"
#include "decode_int.cuh"
#include "merge.cuh"
#include "prefill.cuh"

namespace attn {

static thread_local int t_last_cuda_error = 0;

static attn_status_t cuda_fail(cudaError_t e) {
  t_last_cuda_error = (int)e;
  return ATTN_ERR_CUDA;
}

#define ATTN_CUDA(call)                          \
  do {                                           \
    cudaError_t e_ = (call);                     \
    if (e_ != cudaSuccess) return cuda_fail(e_); \
  } while (0)

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// ---------------------------------------------------------------- tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 4-D tiled map over a row-major [d3][d2][d1][d0] tensor, 128-byte swizzle (or `swz`), zero fill out
// of bounds.
// A 4-D tiled map over (D, heads, tokens, batch).  `strides` gives the element strides of the
// three outer dimensions (NULL: packed row-major, as the dimensions imply).
static attn_status_t make_map_4d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int elem_bytes,
                                 const uint64_t dims[4], const uint32_t box[4],
                                 CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B,
                                 const long long* strides = nullptr) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cuda_fail(cudaErrorNotSupported);
  cuuint64_t gdim[4] = {dims[0], dims[1], dims[2], dims[3]};
  cuuint64_t gstride[3] = {dims[0] * elem_bytes, dims[0] * dims[1] * elem_bytes,
                           dims[0] * dims[1] * dims[2] * elem_bytes};
  if (strides)
    for (int i = 0; i < 3; ++i) gstride[i] = (cuuint64_t)strides[i] * (cuuint64_t)elem_bytes;
  cuuint32_t bx[4] = {box[0], box[1], box[2], box[3]};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = fn(map, dt, 4, const_cast<void*>(base), gdim, gstride, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    t_last_cuda_error = (int)r;
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

// Opt a kernel into more than 48 KB of dynamic shared memory, once per device.
template <typename K>
static attn_status_t ensure_smem(K kernel, int bytes, std::atomic<uint64_t>& done_mask) {
  int dev = 0;
  ATTN_CUDA(cudaGetDevice(&dev));
  const uint64_t bit = 1ull << (dev & 63);
  if (done_mask.load(std::memory_order_acquire) & bit) return ATTN_OK;
  ATTN_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  done_mask.fetch_or(bit, std::memory_order_acq_rel);
  return ATTN_OK;
}

static bool dims_ok(const attn_dims_t& d) {
  return d.B >= 0 && d.Hq > 0 && d.Hkv > 0 && d.Hq % d.Hkv == 0 && d.D > 0 && std::isfinite(d.scale) &&
         d.scale > 0.f;
}

static constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------- prefill

// Dense batch: q [B, S, Hq, D], k/v [B, T, Hkv, D].  Packed batch (cu_q non-null): q/o/lse rows
// [total_q] and k/v rows [total_k] (S = total_q, T = total_k, a single TMA batch), the sequences
// cut by the device cumulative lengths, and max_s the longest query count (grid size).
// strides: NULL (packed [B, S, H, D] tensors) or 12 element strides, (batch, token, head) for
// q, k, v and o in that order; already validated.
// A kernel whose warpgroups trade registers with setmaxnreg must be launched with at least the
// registers the split hands out, or the increasing warpgroups wait forever: check the compiled
// per-thread count once (per kernel) before the first launch.
template <typename K>
static attn_status_t check_register_split(K kernel, int threads, int split_total, std::atomic<int>& state) {
  int s = state.load(std::memory_order_acquire);
  if (s == 0) {
    cudaFuncAttributes a{};
    ATTN_CUDA(cudaFuncGetAttributes(&a, kernel));
    s = (a.numRegs * threads >= split_total) ? 1 : 2;
    state.store(s, std::memory_order_release);
  }
  return s == 1 ? ATTN_OK : ATTN_ERR_UNSUPPORTED;
}

template <int D>
static attn_status_t launch_prefill(const void* q, const void* k, const void* v, void* o, int o_f32, float* lse,
                                    const attn_dims_t& d, int S, int T, int causal, long long q_pos0,
                                    long long kv_pos0, cudaStream_t stream, const int* cu_q = nullptr,
                                    const int* cu_k = nullptr, int max_s = 0, const long long* strides = nullptr,
                                    int accumulate = 0) {
  using C = PrefillCfg<D>;
  static std::atomic<uint64_t> smem_done{0};
  static std::atomic<int> regs_state{0};
  attn_status_t st = ensure_smem(prefill_fwd_sm100<D>, C::SMEM_BYTES, smem_done);
  if (st != ATTN_OK) return st;
  st = check_register_split(prefill_fwd_sm100<D>, C::THREADS, C::REGS_CTRL * 128 + C::REGS_SOFTMAX * 256,
                            regs_state);
  if (st != ATTN_OK) return st;
  CUtensorMap mq, mk, mv;
  const uint64_t nb = cu_q ? 1 : (uint64_t)d.B;
  const uint64_t dq[4] = {(uint64_t)D, (uint64_t)d.Hq, (uint64_t)std::max(S, 1), nb};
  const uint64_t dk[4] = {(uint64_t)D, (uint64_t)d.Hkv, (uint64_t)std::max(T, 1), nb};
  const uint32_t box[4] = {64, 1, 128, 1};
  // The map's outer strides run (head, token, batch); the argument lists (batch, token, head).
  long long sq[3], sk[3], sv[3];
  if (strides) {
    for (int i = 0; i < 3; ++i) {
      sq[i] = strides[2 - i];
      sk[i] = strides[5 - i];
      sv[i] = strides[8 - i];
    }
  }
  const CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B;
  if ((st = make_map_4d(&mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dq, box, swz, strides ? sq : nullptr)) != ATTN_OK)
    return st;
  if ((st = make_map_4d(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dk, box, swz, strides ? sk : nullptr)) != ATTN_OK)
    return st;
  if ((st = make_map_4d(&mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dk, box, swz, strides ? sv : nullptr)) != ATTN_OK)
    return st;
  PrefillParams p{};
  p.B = d.B;
  p.Hq = d.Hq;
  p.Hkv = d.Hkv;
  p.D = D;
  p.S = S;
  p.T = T;
  p.G = d.Hq / d.Hkv;
  p.causal = causal ? 1 : 0;
  p.q_pos0 = q_pos0;
  p.kv_pos0 = kv_pos0;
  p.scale_log2 = d.scale * kLog2e;
  p.n_qtiles = ((cu_q ? max_s : S) + 127) / 128;
  p.pair_heads = (p.G % 2 == 0) ? 1 : 0;
  p.n_head_units = p.pair_heads ? d.Hq / 2 : d.Hq;
  p.n_q_units = p.pair_heads ? p.n_qtiles : (p.n_qtiles + 1) / 2;
  const long long items = (long long)d.B * p.n_head_units * p.n_q_units;
  if (items > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  p.n_items = (int)items;
  p.o = o;
  p.o_f32 = o_f32;
  p.o_sb = strides ? strides[9] : (long long)S * d.Hq * D;
  p.o_ss = strides ? strides[10] : (long long)d.Hq * D;
  p.o_sh = strides ? strides[11] : (long long)D;
  p.lse = lse;
  p.accumulate = accumulate;
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  if (p.n_items == 0) return ATTN_OK;
  // Persistent: one CTA per SM (shared memory and TMEM allow one), at most one per work item.
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = std::min(p.n_items, std::max(sms, 1));
  prefill_fwd_sm100<D><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, p);
  ATTN_CUDA(cudaGetLastError());
  return ATTN_OK;
}

// ---------------------------------------------------------------- decode planning

static int decode_splits(const attn_dims_t& d, int Tmax, int requested) {
  if (Tmax <= 0) return 1;
  const int max_splits = (Tmax + 127) / 128;
  int P = requested;
  if (P <= 0) {
    // One CTA per SM at a time (shared memory).  Take the split count, with every split at least
    // 2048 tokens, whose CTAs fill whole waves best (at least ~4 waves, so the tail is short),
    // preferring fewer splits on ties.
    int sms = 148;
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long units = (long long)std::max(d.B, 1) * d.Hkv;
    const int p_cap = std::max(1, std::min(max_splits, Tmax / 2048));
    const int p_min = (int)std::min<long long>(p_cap, std::max(1LL, (4LL * sms + units - 1) / units));
    double best = -1.0;
    P = p_min;
    for (int c = p_min; c <= std::min(p_cap, 2 * p_min + 8); ++c) {
      const long long ctas = units * c;
      const long long waves = (ctas + sms - 1) / sms;
      const double fill = (double)ctas / (double)(waves * sms);
      if (fill > best + 0.02) {
        best = fill;
        P = c;
      }
    }
  }
  P = std::min(P, max_splits);
  // Round the split length up to whole tiles, then recompute how many splits cover Tmax.
  const int per = ((Tmax + P - 1) / P + 127) / 128 * 128;
  return (Tmax + per - 1) / per;
}

static int decode_split_tokens(int Tmax, int P) {
  if (Tmax <= 0) return 128;
  return ((Tmax + P - 1) / P + 127) / 128 * 128;
}

static size_t decode_ws_bytes(const attn_dims_t& d, int P, int n_q = 1) {
  if (P <= 1) return 0;
  const size_t rows = (size_t)P * d.B * n_q * d.Hq;
  return rows * d.D * sizeof(float) + rows * sizeof(float) + 256;
}

template <bool FP8, int GP, bool MULTI>
static attn_status_t launch_decode_gp(const CUtensorMap& mk, const CUtensorMap& mv, const DecodeParams& p,
                                      dim3 grid, cudaStream_t stream) {
  static std::atomic<uint64_t> smem_done{0};
  if (FP8) {
    attn_status_t st = ensure_smem(decode_fp8_sm100<GP, MULTI>, DecodeFp8Cfg<GP>::SMEM_BYTES, smem_done);
    if (st != ATTN_OK) return st;
    // Persistent: one CTA per SM (at most one per work item), each walking items c, c + grid, ...
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long items = (long long)grid.x * grid.y * grid.z;
    const dim3 pgrid((unsigned)std::min<long long>(items, std::max(sms, 1)));
    decode_fp8_sm100<GP, MULTI><<<pgrid, DecodeFp8Cfg<GP>::THREADS, DecodeFp8Cfg<GP>::SMEM_BYTES, stream>>>(mk, mv, p);
  } else {
    attn_status_t st = ensure_smem(decode_split_sm100<GP, MULTI>, DecodeCfg::SMEM_BYTES, smem_done);
    if (st != ATTN_OK) return st;
    decode_split_sm100<GP, MULTI><<<grid, DecodeCfg::THREADS, DecodeCfg::SMEM_BYTES, stream>>>(mk, mv, p);
  }
  ATTN_CUDA(cudaGetLastError());
  return ATTN_OK;
}

// Where the cache lives: a padded [B, Tmax] cache is the page table-free case (one page of Tmax
// tokens per sequence); a paged pool is [num_pages, page_size] with a device page table.
struct DecodePaging {
  const int* table;
  int max_pages, page_size, num_pages;
};

template <int GP, int BITS>
static attn_status_t launch_decode_int_gp(const CUtensorMap& mk, const CUtensorMap& mv, const DecodeParams& p,
                                          dim3 grid, cudaStream_t stream) {
  static std::atomic<uint64_t> smem_done{0};
  attn_status_t st = ensure_smem(decode_int_sm100<GP, BITS>, DecodeIntCfg<BITS>::SMEM_BYTES, smem_done);
  if (st != ATTN_OK) return st;
  decode_int_sm100<GP, BITS><<<grid, DecodeIntCfg<BITS>::THREADS, DecodeIntCfg<BITS>::SMEM_BYTES, stream>>>(mk, mv, p);
  ATTN_CUDA(cudaGetLastError());
  return ATTN_OK;
}

template <int BITS>
static attn_status_t launch_decode_int(const CUtensorMap& mk, const CUtensorMap& mv, const DecodeParams& p, int R,
                                       dim3 grid, cudaStream_t stream) {
  if (R <= 1) return launch_decode_int_gp<1, BITS>(mk, mv, p, grid, stream);
  if (R <= 2) return launch_decode_int_gp<2, BITS>(mk, mv, p, grid, stream);
  if (R <= 4) return launch_decode_int_gp<4, BITS>(mk, mv, p, grid, stream);
  if (R <= 8) return launch_decode_int_gp<8, BITS>(mk, mv, p, grid, stream);
  return launch_decode_int_gp<16, BITS>(mk, mv, p, grid, stream);
}

// Cache element kinds of the decode launcher.
enum DecodeKv { KV_BF16 = 0, KV_FP8 = 1, KV_INT8 = 2, KV_INT4 = 3 };

template <int KV>
static attn_status_t launch_decode(const void* q, const void* k, const void* v, const float* ks, const float* vs,
                                   const int* kv_lens, int Tmax, const attn_dims_t& d, int P, int split_tokens,
                                   void* o, float* lse, void* ws, cudaStream_t stream, const DecodePaging& pg,
                                   int n_q = 1) {
  constexpr bool FP8 = KV == KV_FP8;
  attn_status_t st;
  CUtensorMap mk, mv;
  // With Tmax == 0 every split is empty and no map is read; it still needs a valid base and extent.
  const uint64_t row = KV == KV_INT4 ? 64 : 128;  // elements (bytes for the 8-bit and 4-bit caches) per row
  const uint64_t dk[4] = {row, (uint64_t)d.Hkv, (uint64_t)std::max(pg.page_size, 1), (uint64_t)std::max(pg.num_pages, 1)};
  const void* kb = Tmax > 0 ? k : q;
  const void* vb = Tmax > 0 ? v : q;
  if (KV == KV_INT8 || KV == KV_INT4) {
    const uint32_t box[4] = {(uint32_t)row, 1, 128, 1};
    const CUtensorMapSwizzle swz = KV == KV_INT4 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
    if ((st = make_map_4d(&mk, kb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, dk, box, swz)) != ATTN_OK) return st;
    if ((st = make_map_4d(&mv, vb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, dk, box, swz)) != ATTN_OK) return st;
  } else if (FP8) {
    const uint32_t box[4] = {128, 1, 128, 1};
    if ((st = make_map_4d(&mk, kb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, dk, box)) != ATTN_OK) return st;
    if ((st = make_map_4d(&mv, vb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, dk, box)) != ATTN_OK) return st;
  } else {
    const uint32_t box[4] = {64, 1, 128, 1};
    if ((st = make_map_4d(&mk, kb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dk, box)) != ATTN_OK) return st;
    if ((st = make_map_4d(&mv, vb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dk, box)) != ATTN_OK) return st;
  }
  DecodeParams p{};
  p.B = d.B;
  p.Hq = d.Hq;
  p.Hkv = d.Hkv;
  p.G = d.Hq / d.Hkv;
  p.n_q = n_q;
  p.Tmax = Tmax;
  p.split_tokens = split_tokens;
  p.n_splits = P;
  p.scale_log2 = d.scale * kLog2e;
  p.q = reinterpret_cast<const __nv_bfloat16*>(q);
  p.k_scale = ks;
  p.v_scale = vs;
  p.kv_lens = kv_lens;
  p.v_codes = FP8 ? reinterpret_cast<const uint8_t*>(v) : nullptr;
  p.page_table = pg.table;
  p.max_pages = pg.max_pages;
  p.page_size = std::max(pg.page_size, 1);
  p.num_pages = pg.num_pages;
  float* ws_f = reinterpret_cast<float*>(ws);
  const size_t rows = (size_t)P * d.B * n_q * d.Hq;
  p.o_part = P > 1 ? ws_f : nullptr;
  p.lse_part = P > 1 ? ws_f + rows * 128 : nullptr;
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  dim3 grid(P, d.Hkv, d.B);
  if ((long long)P * d.Hkv * d.B > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;  // work items are int-indexed
  // The query group is padded to the next power of two (<= 16) so the kernels' per-row loops unroll.
  const int R = p.G * n_q;  // MMA rows of one (sequence, KV head)
  // Single-token decode runs instances without per-row key limits (one compare per token).
  if (KV == KV_INT8 || KV == KV_INT4) {
    if (n_q != 1) return ATTN_ERR_UNSUPPORTED;
    st = launch_decode_int<KV == KV_INT8 ? 8 : 4>(mk, mv, p, R, grid, stream);
  } else if (n_q == 1) {
    if (R <= 1) st = launch_decode_gp<FP8, 1, false>(mk, mv, p, grid, stream);
    else if (R <= 2) st = launch_decode_gp<FP8, 2, false>(mk, mv, p, grid, stream);
    else if (R <= 4) st = launch_decode_gp<FP8, 4, false>(mk, mv, p, grid, stream);
    else if (R <= 8) st = launch_decode_gp<FP8, 8, false>(mk, mv, p, grid, stream);
    else st = launch_decode_gp<FP8, 16, false>(mk, mv, p, grid, stream);
  } else {
    if (R <= 2) st = launch_decode_gp<FP8, 2, true>(mk, mv, p, grid, stream);
    else if (R <= 4) st = launch_decode_gp<FP8, 4, true>(mk, mv, p, grid, stream);
    else if (R <= 8) st = launch_decode_gp<FP8, 8, true>(mk, mv, p, grid, stream);
    else st = launch_decode_gp<FP8, 16, true>(mk, mv, p, grid, stream);
  }
  if (st != ATTN_OK) return st;
  if (P > 1) {
    MergeParams mp{};
    mp.o_parts = p.o_part;
    mp.lse_parts = p.lse_part;
    mp.P = P;
    mp.R = (long long)d.B * n_q * d.Hq;
    mp.o_out = o;
    mp.o_f32 = 0;
    mp.lse_out = lse;
    mp.accumulate = 0;
    const long long blocks = (mp.R + 7) / 8;
    merge_lse_kernel<128><<<(unsigned)blocks, 256, 0, stream>>>(mp);
    ATTN_CUDA(cudaGetLastError());
  }
  return ATTN_OK;
}

static bool kv_dtype_ok(attn_dtype_t t) {
  return t == ATTN_BF16 || t == ATTN_FP8_E4M3 || t == ATTN_INT8 || t == ATTN_INT4;
}

// Single-token decode over a cache of any supported element kind.
static attn_status_t launch_decode_kind(attn_dtype_t kv, const void* q, const void* k, const void* v, const float* ks,
                                        const float* vs, const int* kv_lens, int Tmax, const attn_dims_t& d, int P,
                                        int per, void* o, float* lse, void* ws, cudaStream_t st,
                                        const DecodePaging& pg) {
  switch (kv) {
    case ATTN_FP8_E4M3: return launch_decode<KV_FP8>(q, k, v, ks, vs, kv_lens, Tmax, d, P, per, o, lse, ws, st, pg);
    case ATTN_INT8: return launch_decode<KV_INT8>(q, k, v, ks, vs, kv_lens, Tmax, d, P, per, o, lse, ws, st, pg);
    case ATTN_INT4: return launch_decode<KV_INT4>(q, k, v, ks, vs, kv_lens, Tmax, d, P, per, o, lse, ws, st, pg);
    default: return launch_decode<KV_BF16>(q, k, v, nullptr, nullptr, kv_lens, Tmax, d, P, per, o, lse, ws, st, pg);
  }
}

// ---------------------------------------------------------------- diagnostics

__global__ void exp2_probe_kernel(const float* x, float* y, long long n, int mode) {
  const long long i = 2 * ((long long)blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 >= n + 1) return;
  const float a = x[i], b = (i + 1 < n) ? x[i + 1] : 0.f;
  float2 r;
  if (mode == 0) {
    r = exp2_poly2(make_float2(a, b));
  } else {
    r.x = ex2_approx(a);
    r.y = ex2_approx(b);
  }
  y[i] = r.x;
  if (i + 1 < n) y[i + 1] = r.y;
}

__global__ void wait_probe_kernel() {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, SITE_PROBE);  // nothing arrives: runs out and records
  __syncthreads();
}

}  // namespace attn

using namespace attn;

extern "C" {

const char* attn_status_string(attn_status_t s) {
  switch (s) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported configuration";
    case ATTN_ERR_CUDA: return "CUDA error";
    case ATTN_ERR_BUDGET: return "device budget too small for the smallest plan";
    case ATTN_ERR_TIMEOUT: return "a kernel wait ran out of time";
    case ATTN_ERR_INJECTED: return "injected failure";
  }
  return "unknown status";
}

int attn_last_cuda_error(void) { return t_last_cuda_error; }

// The 12 element strides of attn_prefill: each positive, a whole number of 16-byte units (TMA
// strides and the 16-byte output stores need it) and below TMA's 2^40-byte stride limit.
static bool prefill_strides_ok(const long long* s, int o_f32) {
  for (int i = 0; i < 12; ++i) {
    const long long unit = (i >= 9 && o_f32) ? 4 : 8;  // elements per 16 bytes
    if (s[i] <= 0 || s[i] % unit != 0 || s[i] >= (1LL << 38)) return false;
  }
  return true;
}

attn_status_t attn_prefill(const void* q, const void* k, const void* v, void* o, attn_dtype_t o_dtype, float* lse,
                           attn_dims_t dims, int S, int T, int causal, long long q_pos0, long long kv_pos0,
                           const long long* strides, void* stream) {
  if (!dims_ok(dims) || S < 0 || T < 0 || q_pos0 < 0 || kv_pos0 < 0) return ATTN_ERR_INVALID_ARG;
  if (o_dtype != ATTN_BF16 && o_dtype != ATTN_F32) return ATTN_ERR_INVALID_ARG;
  if (strides && !prefill_strides_ok(strides, o_dtype == ATTN_F32)) return ATTN_ERR_INVALID_ARG;
  if (dims.B == 0 || S == 0) return ATTN_OK;
  if (!q || !o || (T > 0 && (!k || !v))) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || (T > 0 && (!aligned16(k) || !aligned16(v))) || (lse && !aligned4(lse)))
    return ATTN_ERR_INVALID_ARG;
  if (dims.D != 64 && dims.D != 128) return ATTN_ERR_UNSUPPORTED;
  long long s_nokv[12];
  if (T == 0 && strides) {
    // No keys and a strided output: the kernel itself writes the empty rows (O = 0, LSE = -inf)
    // and never reads a key; its K/V maps only need a valid base, so they point at q.
    for (int i = 0; i < 12; ++i) s_nokv[i] = strides[i < 9 ? i % 3 : i];
    k = v = q;
    strides = s_nokv;
  } else if (T == 0) {
    // No keys: every row is empty.  O = 0, LSE = -inf, written by the merge kernel with no parts.
    MergeParams mp{};
    mp.P = 0;
    mp.R = (long long)dims.B * S * dims.Hq;
    mp.o_out = o;
    mp.o_f32 = o_dtype == ATTN_F32;
    mp.lse_out = lse;
    mp.accumulate = 0;
    const long long blocks = (mp.R + 7) / 8;
    if (blocks > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dims.D == 128) merge_lse_kernel<128><<<(unsigned)blocks, 256, 0, st>>>(mp);
    else merge_lse_kernel<64><<<(unsigned)blocks, 256, 0, st>>>(mp);
    ATTN_CUDA(cudaGetLastError());
    return ATTN_OK;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int f32 = o_dtype == ATTN_F32;
  if (dims.D == 128)
    return launch_prefill<128>(q, k, v, o, f32, lse, dims, S, T, causal, q_pos0, kv_pos0, st, nullptr, nullptr, 0,
                               strides);
  return launch_prefill<64>(q, k, v, o, f32, lse, dims, S, T, causal, q_pos0, kv_pos0, st, nullptr, nullptr, 0,
                            strides);
}

attn_status_t attn_prefill_varlen(const void* q, const void* k, const void* v, void* o, attn_dtype_t o_dtype,
                                  float* lse, attn_dims_t dims, const int* cu_seqlens_q, const int* cu_seqlens_k,
                                  int total_q, int total_k, int max_seqlen_q, int causal, void* stream) {
  if (!dims_ok(dims) || total_q < 0 || total_k < 0 || max_seqlen_q < 0) return ATTN_ERR_INVALID_ARG;
  if (o_dtype != ATTN_BF16 && o_dtype != ATTN_F32) return ATTN_ERR_INVALID_ARG;
  if (dims.B == 0 || total_q == 0 || max_seqlen_q == 0) return ATTN_OK;
  if (!q || !o || !cu_seqlens_q || !cu_seqlens_k || (total_k > 0 && (!k || !v))) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || (total_k > 0 && (!aligned16(k) || !aligned16(v))) ||
      (lse && !aligned4(lse)) || !aligned4(cu_seqlens_q) || !aligned4(cu_seqlens_k))
    return ATTN_ERR_INVALID_ARG;
  if (dims.D != 64 && dims.D != 128) return ATTN_ERR_UNSUPPORTED;
  if (total_k == 0) {  // no keys anywhere: every row is empty (O = 0, LSE = -inf)
    MergeParams mp{};
    mp.P = 0;
    mp.R = (long long)total_q * dims.Hq;
    mp.o_out = o;
    mp.o_f32 = o_dtype == ATTN_F32;
    mp.lse_out = lse;
    mp.accumulate = 0;
    const long long blocks = (mp.R + 7) / 8;
    if (blocks > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dims.D == 128) merge_lse_kernel<128><<<(unsigned)blocks, 256, 0, st>>>(mp);
    else merge_lse_kernel<64><<<(unsigned)blocks, 256, 0, st>>>(mp);
    ATTN_CUDA(cudaGetLastError());
    return ATTN_OK;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int f32 = o_dtype == ATTN_F32;
  if (dims.D == 128)
    return launch_prefill<128>(q, k, v, o, f32, lse, dims, total_q, total_k, causal, 0, 0, st, cu_seqlens_q,
                               cu_seqlens_k, max_seqlen_q);
  return launch_prefill<64>(q, k, v, o, f32, lse, dims, total_q, total_k, causal, 0, 0, st, cu_seqlens_q,
                            cu_seqlens_k, max_seqlen_q);
}

}  // extern "C"

namespace attn {

attn_status_t prefill_accumulate_f32(const void* q, const void* k, const void* v, float* o, float* lse,
                                     attn_dims_t dims, int S, int T, int causal, long long q_pos0, long long kv_pos0,
                                     void* stream) {
  if (!dims_ok(dims) || S < 0 || T < 0 || q_pos0 < 0 || kv_pos0 < 0) return ATTN_ERR_INVALID_ARG;
  if (dims.B == 0 || S == 0 || T == 0) return ATTN_OK;  // no key: every stored partial stands
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse)) return ATTN_ERR_INVALID_ARG;
  if (dims.D != 64 && dims.D != 128) return ATTN_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dims.D == 128)
    return launch_prefill<128>(q, k, v, o, 1, lse, dims, S, T, causal, q_pos0, kv_pos0, st, nullptr, nullptr, 0,
                               nullptr, 1);
  return launch_prefill<64>(q, k, v, o, 1, lse, dims, S, T, causal, q_pos0, kv_pos0, st, nullptr, nullptr, 0, nullptr,
                            1);
}

}  // namespace attn

extern "C" {

int attn_decode_num_splits(attn_dims_t dims, int Tmax, int num_splits) {
  if (!dims_ok(dims) || Tmax < 0) return 0;
  return decode_splits(dims, Tmax, num_splits);
}

size_t attn_decode_workspace_bytes(attn_dims_t dims, int Tmax, int num_splits) {
  if (!dims_ok(dims) || Tmax < 0) return 0;
  return decode_ws_bytes(dims, decode_splits(dims, Tmax, num_splits));
}

}  // extern "C"

// Every check of attn_decode_splitkv that does not involve the workspace, in its order.  ATTN_OK
// with *empty set means a valid call with nothing to do (B = 0).
static attn_status_t decode_splitkv_args(const void* q, const void* k, const void* v, attn_dtype_t kv_dtype,
                                         const float* k_scale, const float* v_scale, const int* kv_lens, int Tmax,
                                         const attn_dims_t& dims, int num_splits, void* o, float* lse, bool* empty) {
  *empty = false;
  if (!dims_ok(dims) || Tmax < 0 || num_splits < 0 || num_splits > 4096) return ATTN_ERR_INVALID_ARG;
  if (!kv_dtype_ok(kv_dtype)) return ATTN_ERR_INVALID_ARG;
  if (dims.B == 0) {
    *empty = true;
    return ATTN_OK;
  }
  if (!q || !o || !kv_lens || (Tmax > 0 && (!k || !v))) return ATTN_ERR_INVALID_ARG;
  const bool quant = kv_dtype != ATTN_BF16;  // codes + per-token scales
  if (quant != (k_scale != nullptr) || quant != (v_scale != nullptr)) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || !aligned4(kv_lens) || (lse && !aligned4(lse))) return ATTN_ERR_INVALID_ARG;
  if (Tmax > 0 && (!aligned16(k) || !aligned16(v))) return ATTN_ERR_INVALID_ARG;
  if (quant && (!aligned4(k_scale) || !aligned4(v_scale))) return ATTN_ERR_INVALID_ARG;
  if (dims.D != 128 || dims.Hq / dims.Hkv > 16) return ATTN_ERR_UNSUPPORTED;
  if (dims.B > 65535 || dims.Hkv > 65535) return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

extern "C" {

attn_status_t attn_decode_splitkv(const void* q, const void* k, const void* v, attn_dtype_t kv_dtype,
                                  const float* k_scale, const float* v_scale, const int* kv_lens, int Tmax,
                                  attn_dims_t dims, int num_splits, void* o, float* lse, void* ws, size_t ws_bytes,
                                  void* stream) {
  bool empty = false;
  const attn_status_t a = decode_splitkv_args(q, k, v, kv_dtype, k_scale, v_scale, kv_lens, Tmax, dims, num_splits,
                                              o, lse, &empty);
  if (a != ATTN_OK || empty) return a;
  const int P = decode_splits(dims, Tmax, num_splits);
  const size_t need = decode_ws_bytes(dims, P);
  if (need > 0 && (!ws || ws_bytes < need || !aligned16(ws))) return ATTN_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int per = decode_split_tokens(Tmax, P);
  const DecodePaging pg{nullptr, 1, Tmax, dims.B};
  return launch_decode_kind(kv_dtype, q, k, v, k_scale, v_scale, kv_lens, Tmax, dims, P, per, o, lse, ws, st, pg);
}

attn_status_t attn_decode_paged(const void* q, const void* k_pool, const void* v_pool, attn_dtype_t kv_dtype,
                                const float* k_scale_pool, const float* v_scale_pool, const int* page_table,
                                int max_pages, int page_size, int num_pages, const int* kv_lens, attn_dims_t dims,
                                int num_splits, void* o, float* lse, void* ws, size_t ws_bytes, void* stream) {
  if (!dims_ok(dims) || num_splits < 0 || num_splits > 4096) return ATTN_ERR_INVALID_ARG;
  if (!kv_dtype_ok(kv_dtype)) return ATTN_ERR_INVALID_ARG;
  if (max_pages < 1 || page_size < 128 || page_size % 128 != 0 || num_pages < 1) return ATTN_ERR_INVALID_ARG;
  if ((long long)max_pages * page_size > 0x7fffffffLL || (long long)num_pages * page_size > 0x7fffffffLL)
    return ATTN_ERR_UNSUPPORTED;
  if (dims.B == 0) return ATTN_OK;
  if (!q || !o || !kv_lens || !page_table || !k_pool || !v_pool) return ATTN_ERR_INVALID_ARG;
  const bool quant = kv_dtype != ATTN_BF16;  // codes + per-token scales
  if (quant != (k_scale_pool != nullptr) || quant != (v_scale_pool != nullptr)) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || !aligned4(kv_lens) || !aligned4(page_table) || (lse && !aligned4(lse)))
    return ATTN_ERR_INVALID_ARG;
  if (!aligned16(k_pool) || !aligned16(v_pool)) return ATTN_ERR_INVALID_ARG;
  if (quant && (!aligned4(k_scale_pool) || !aligned4(v_scale_pool))) return ATTN_ERR_INVALID_ARG;
  if (dims.D != 128 || dims.Hq / dims.Hkv > 16) return ATTN_ERR_UNSUPPORTED;
  if (dims.B > 65535 || dims.Hkv > 65535) return ATTN_ERR_UNSUPPORTED;
  const int Tmax = max_pages * page_size;
  const int P = decode_splits(dims, Tmax, num_splits);
  const size_t need = decode_ws_bytes(dims, P);
  if (need > 0 && (!ws || ws_bytes < need || !aligned16(ws))) return ATTN_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int per = decode_split_tokens(Tmax, P);
  const DecodePaging pg{page_table, max_pages, page_size, num_pages};
  return launch_decode_kind(kv_dtype, q, k_pool, v_pool, k_scale_pool, v_scale_pool, kv_lens, Tmax, dims, P, per, o,
                            lse, ws, st, pg);
}

size_t attn_decode_multi_workspace_bytes(attn_dims_t dims, int Tmax, int n_q, int num_splits) {
  if (!dims_ok(dims) || Tmax < 0 || n_q < 1) return 0;
  return decode_ws_bytes(dims, decode_splits(dims, Tmax, num_splits), n_q);
}

attn_status_t attn_decode_multi(const void* q, const void* k, const void* v, attn_dtype_t kv_dtype,
                                const float* k_scale, const float* v_scale, const int* kv_lens, int Tmax, int n_q,
                                attn_dims_t dims, int num_splits, void* o, float* lse, void* ws, size_t ws_bytes,
                                void* stream) {
  if (!dims_ok(dims) || Tmax < 0 || num_splits < 0 || num_splits > 4096 || n_q < 1) return ATTN_ERR_INVALID_ARG;
  if (!kv_dtype_ok(kv_dtype)) return ATTN_ERR_INVALID_ARG;
  if (kv_dtype == ATTN_INT8 || kv_dtype == ATTN_INT4) return ATTN_ERR_UNSUPPORTED;
  if (dims.B == 0) return ATTN_OK;
  if (!q || !o || !kv_lens || (Tmax > 0 && (!k || !v))) return ATTN_ERR_INVALID_ARG;
  const bool fp8 = kv_dtype == ATTN_FP8_E4M3;
  if (fp8 != (k_scale != nullptr) || fp8 != (v_scale != nullptr)) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || !aligned4(kv_lens) || (lse && !aligned4(lse))) return ATTN_ERR_INVALID_ARG;
  if (Tmax > 0 && (!aligned16(k) || !aligned16(v))) return ATTN_ERR_INVALID_ARG;
  if (fp8 && (!aligned4(k_scale) || !aligned4(v_scale))) return ATTN_ERR_INVALID_ARG;
  if (dims.D != 128 || (long long)(dims.Hq / dims.Hkv) * n_q > 16) return ATTN_ERR_UNSUPPORTED;
  if (dims.B > 65535 || dims.Hkv > 65535) return ATTN_ERR_UNSUPPORTED;
  const int P = decode_splits(dims, Tmax, num_splits);
  const size_t need = decode_ws_bytes(dims, P, n_q);
  if (need > 0 && (!ws || ws_bytes < need || !aligned16(ws))) return ATTN_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int per = decode_split_tokens(Tmax, P);
  const DecodePaging pg{nullptr, 1, Tmax, dims.B};
  if (fp8) return launch_decode<KV_FP8>(q, k, v, k_scale, v_scale, kv_lens, Tmax, dims, P, per, o, lse, ws, st, pg, n_q);
  return launch_decode<KV_BF16>(q, k, v, nullptr, nullptr, kv_lens, Tmax, dims, P, per, o, lse, ws, st, pg, n_q);
}

// Split-KV decode without allocation: the split partials live in this static device array
// (ATTN_NOALLOC_SCRATCH_BYTES per device, held until the process exits).  Host code must not pass
// the array's name to a kernel — on the host it is only a stand-in — so its device address is
// looked up with cudaGetSymbolAddress, with the device current, once per device and context: the
// address is cached with the context it belongs to, and looked up again if the device's context
// changes (after a cudaDeviceReset the module, and with it the array, is loaded anew).
static __device__ __align__(256) unsigned char g_noalloc_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

static CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

static attn_status_t noalloc_scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[64] = {};
  static CUcontext owner[64] = {};
  int dev = 0;
  ATTN_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return ATTN_ERR_UNSUPPORTED;
  CtxGetCurrentFn get = ctx_get_current_fn();
  if (!get) return cuda_fail(cudaErrorNotSupported);
  CUcontext ctx = nullptr;
  if (get(&ctx) != CUDA_SUCCESS) ctx = nullptr;  // none yet: the lookup below makes it current
  std::lock_guard<std::mutex> lock(mu);
  if (!ctx || !addr[dev] || owner[dev] != ctx) {
    void* p = nullptr;
    ATTN_CUDA(cudaGetSymbolAddress(&p, g_noalloc_scratch));
    if (get(&ctx) != CUDA_SUCCESS || !ctx) return cuda_fail(cudaErrorNotSupported);
    addr[dev] = p;
    owner[dev] = ctx;
  }
  *out = addr[dev];
  return ATTN_OK;
}

attn_status_t attn_decode_splitkv_noalloc(const void* q, const void* k, const void* v, attn_dtype_t kv_dtype,
                                          const float* k_scale, const float* v_scale, const int* kv_lens, int Tmax,
                                          attn_dims_t dims, int num_splits, void* o, float* lse, void* stream) {
  // Argument checks first, in attn_decode_splitkv's order; the scratch limit after them.
  bool empty = false;
  const attn_status_t a = decode_splitkv_args(q, k, v, kv_dtype, k_scale, v_scale, kv_lens, Tmax, dims, num_splits,
                                              o, lse, &empty);
  if (a != ATTN_OK || empty) return a;
  const size_t need = decode_ws_bytes(dims, decode_splits(dims, Tmax, num_splits));
  if (need > ATTN_NOALLOC_SCRATCH_BYTES) return ATTN_ERR_BUDGET;
  void* ws = nullptr;
  if (need > 0) {
    const attn_status_t s = noalloc_scratch_address(&ws);
    if (s != ATTN_OK) return s;
  }
  return attn_decode_splitkv(q, k, v, kv_dtype, k_scale, v_scale, kv_lens, Tmax, dims, num_splits, o, lse, ws,
                             need > 0 ? (size_t)ATTN_NOALLOC_SCRATCH_BYTES : 0, stream);
}

attn_status_t attn_merge_lse(const float* o_parts, const float* lse_parts, int P, long long R, int D, void* o_out,
                             attn_dtype_t o_dtype, float* lse_out, int accumulate, void* stream) {
  if (P < 0 || R < 0 || (P == 0 && !accumulate)) return ATTN_ERR_INVALID_ARG;
  if (o_dtype != ATTN_BF16 && o_dtype != ATTN_F32) return ATTN_ERR_INVALID_ARG;
  if (accumulate && (o_dtype != ATTN_F32 || !lse_out)) return ATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  if (R == 0) return ATTN_OK;
  if (!o_out || (P > 0 && (!o_parts || !lse_parts))) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(o_out) || (P > 0 && (!aligned16(o_parts) || !aligned4(lse_parts))) || (lse_out && !aligned4(lse_out)))
    return ATTN_ERR_INVALID_ARG;
  const long long blocks = (R + 7) / 8;
  if (blocks > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  MergeParams mp{};
  mp.o_parts = o_parts;
  mp.lse_parts = lse_parts;
  mp.P = P;
  mp.R = R;
  mp.o_out = o_out;
  mp.o_f32 = o_dtype == ATTN_F32;
  mp.lse_out = lse_out;
  mp.accumulate = accumulate ? 1 : 0;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (D == 128) merge_lse_kernel<128><<<(unsigned)blocks, 256, 0, st>>>(mp);
  else merge_lse_kernel<64><<<(unsigned)blocks, 256, 0, st>>>(mp);
  ATTN_CUDA(cudaGetLastError());
  return ATTN_OK;
}

attn_status_t attn_device_status(int reset, int* site) {
  uint32_t v = 0;
  ATTN_CUDA(cudaDeviceSynchronize());
  ATTN_CUDA(cudaMemcpyFromSymbol(&v, g_dev_status, sizeof(v)));
  if (reset) {
    const uint32_t z = 0;
    ATTN_CUDA(cudaMemcpyToSymbol(g_dev_status, &z, sizeof(z)));
  }
  if (site) *site = (int)(v & 0xFFFFu);
  if (v == 0) return ATTN_OK;
  if ((v >> 16) == ATTN_DEV_TIMEOUT) return ATTN_ERR_TIMEOUT;
  if ((v >> 16) == ATTN_DEV_BAD_PAGE) return ATTN_ERR_INVALID_ARG;
  return ATTN_ERR_CUDA;
}

attn_status_t attn_set_wait_limit_ns(unsigned long long ns) {
  if (ns == 0) return ATTN_ERR_INVALID_ARG;
  const uint64_t v = ns;
  ATTN_CUDA(cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v)));
  return ATTN_OK;
}

#ifdef ATTN_PROF
// Profile builds only: point the cycle counters at a device buffer of 64 unsigned 64-bit words.
ATTN_API attn_status_t attn_debug_set_prof(void* dev_ptr) {
  unsigned long long* p = static_cast<unsigned long long*>(dev_ptr);
  ATTN_CUDA(cudaMemcpyToSymbol(g_prof, &p, sizeof(p)));
  return ATTN_OK;
}
ATTN_API attn_status_t attn_debug_set_evt(void* dev_ptr) {
  long long* p = static_cast<long long*>(dev_ptr);
  ATTN_CUDA(cudaMemcpyToSymbol(g_evt, &p, sizeof(p)));
  return ATTN_OK;
}
#endif

#ifdef ATTN_TRACE
// Trace builds only: point the progress trace at host-mapped memory (device address).
ATTN_API attn_status_t attn_debug_set_trace(void* dev_ptr) {
  uint32_t* p = static_cast<uint32_t*>(dev_ptr);
  ATTN_CUDA(cudaMemcpyToSymbol(g_trace, &p, sizeof(p)));
  return ATTN_OK;
}
#endif

attn_status_t attn_debug_exp2(const float* x, float* y, long long n, int mode, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y)) || (mode != 0 && mode != 1)) return ATTN_ERR_INVALID_ARG;
  if (n == 0) return ATTN_OK;
  const long long pairs = (n + 1) / 2;
  const long long blocks = (pairs + 255) / 256;
  if (blocks > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  exp2_probe_kernel<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n, mode);
  ATTN_CUDA(cudaGetLastError());
  return ATTN_OK;
}

attn_status_t attn_debug_wait_probe(unsigned long long limit_ns) {
  if (limit_ns == 0 || limit_ns > 10ull * 1000 * 1000 * 1000) return ATTN_ERR_INVALID_ARG;
  uint64_t old = 0;
  ATTN_CUDA(cudaMemcpyFromSymbol(&old, g_wait_limit_ns, sizeof(old)));
  const uint64_t v = limit_ns;
  ATTN_CUDA(cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v)));
  wait_probe_kernel<<<1, 32>>>();
  const cudaError_t e1 = cudaGetLastError();
  const cudaError_t e2 = cudaDeviceSynchronize();
  ATTN_CUDA(cudaMemcpyToSymbol(g_wait_limit_ns, &old, sizeof(old)));
  if (e1 != cudaSuccess) return cuda_fail(e1);
  if (e2 != cudaSuccess) return cuda_fail(e2);
  return attn_device_status(0, nullptr);
}

}  // extern "C"
