// Split-KV GQA decode on tcgen05 with the KV tokens on the MMA's M axis.
//
// Flash Decoding (ONNX Runtime CPU GQA analysis, "Flash Decoding"): the keys of one
// (sequence, KV head) are cut into chunks; each chunk yields a partial softmax state
// (o_s normalised by its own sum, lse_s) that a log-sum-exp reduce merges exactly.
//
// One CTA = (split, KV head, sequence).  Per 128-token tile j:
//   S^T_j [128 tokens x 16]  = K_j [128 x D] . Q^T [D x 16]        (G query rows, zero-padded to 16)
//   O^T   [D x 16]          += V_j^T [D x 128] . P_j^T [128 x 16]
// so every thread of the softmax warpgroup owns one token (one TMEM lane): per-token
// dequantisation scales multiply that thread's score and probability, masking is a per-thread
// compare, and only the G row maxima need a cross-thread reduction.  O^T rows are D, so the
// same thread later owns output element d.
//
// This file holds the bf16-cache kernel and what the decode kernels share (parameters, page
// cursor, softmax steps, epilogue).  Coded caches have their own kernels: decode_fp8.cuh
// (E4M3 codes fed to the MMA as they land) and decode_int.cuh (INT8 / INT4 codes widened to
// f16 inside the tile load).
//
// Roles of the bf16 kernel (192 threads): warp 0 TMA producer, warp 1 TMEM allocator + MMA issuer,
// warps 2..5 softmax / epilogue (128 threads).  The query group is padded to GP (a power of two
// <= 16, a template parameter) so the per-row loops unroll and run side by side.
#pragma once

#include "ptx.cuh"

namespace attn {

struct DecodeParams {
  int B, Hq, Hkv, G, Tmax;
  // Query tokens per sequence (1 for plain decode).  With n_q > 1 (multi-token decode / draft
  // verification, ORT GQA analysis "Verification"), token i of sequence b sits at position
  // len_b - n_q + i and sees keys [0, len_b - n_q + i + 1); its G heads are MMA rows
  // r = i * G + g, so the rows of one (sequence, KV head) are n_q * G <= 16.
  int n_q;
  int split_tokens;  // tokens per split, multiple of 128
  int n_splits;
  float scale_log2;
  const __nv_bfloat16* q;  // [B, n_q, Hq, 128]
  const float* k_scale;    // [B, Tmax, Hkv] (FP8) or null
  const float* v_scale;
  const int* kv_lens;       // [B]
  const uint8_t* v_codes;   // FP8 V pool [num_pages, page_size, Hkv, 128] (partial tiles are copied without TMA)
  // Paged cache (LLM-CoOpt summary, "Opt-Pa"): token t of sequence b lives in pool page
  // page_table[b * max_pages + t / page_size] at offset t % page_size.  Without a table the cache
  // is one page of Tmax tokens per sequence (page_size = Tmax, num_pages = B, page of b = b).
  const int* page_table;    // device int32 [B, max_pages] or null
  int max_pages, page_size, num_pages;
  float* o_part;            // [n_splits, B * n_q * Hq, 128] when n_splits > 1
  float* lse_part;          // [n_splits, B * n_q * Hq]
  __nv_bfloat16* o;         // [B, n_q, Hq, 128] when n_splits == 1
  float* lse;               // [B, n_q, Hq] or null
};

// Rows of one (sequence, KV head): n_q query tokens x G heads.
__device__ __forceinline__ int decode_rows(const DecodeParams& p) { return p.n_q * p.G; }

// Row r = i * G + g of (sequence b, KV head kvh) in the [B, n_q, Hq] order of q, o and lse.
__device__ __forceinline__ long long decode_row_index(const DecodeParams& p, int b, int kvh, int r) {
  const int i = r / p.G, g = r - i * p.G;
  return ((long long)b * p.n_q + i) * p.Hq + (long long)kvh * p.G + g;
}

// Exclusive key limit of row r within a split ending at t1: the token's causal limit, and t1.
__device__ __forceinline__ int decode_row_limit(const DecodeParams& p, int len, int t1, int r) {
  const int lim = len - p.n_q + 1 + r / p.G;
  return lim < t1 ? lim : t1;
}

// Pool page of the tile of sequence b that starts at token tok (a multiple of 128; with a table,
// page_size is a multiple of 128, so a tile never straddles two pages).  Table entries are read
// one page ahead of their use, so the load latency stays off the copy issue; an entry outside
// [0, num_pages) is reported through the device status word and gives page -1, which the callers
// never dereference (a TMA box at page -1 lands as zeros).
struct PageCursor {
  int b = -1, lp = -1, page = 0;  // the page in use
  int nb = -1, nlp = -1, nraw = 0;  // the next page of the same sequence, loaded ahead
  __device__ __forceinline__ int offset(const DecodeParams& p, int tok) const {
    return p.page_table ? tok % p.page_size : tok;
  }
  __device__ __forceinline__ int get(const DecodeParams& p, int b_, int tok) {
    if (!p.page_table) return b_;
    const int l = tok / p.page_size;
    if (b_ == b && l == lp) return page;
    int raw;
    if (b_ == nb && l == nlp) raw = nraw;
    else raw = __ldg(p.page_table + (long long)b_ * p.max_pages + l);
    if (raw < 0 || raw >= p.num_pages) {
      record_device_error(ATTN_DEV_BAD_PAGE, SITE_DC_PAGE);
      raw = -1;
    }
    b = b_;
    lp = l;
    page = raw;
    nb = b_;
    nlp = l + 1;
    nraw = nlp < p.max_pages ? __ldg(p.page_table + (long long)b_ * p.max_pages + nlp) : -1;
    return page;
  }
};

struct DecodeCfg {
  static constexpr int D = 128;
  static constexpr int NST = 3;
  static constexpr int KV_TILE = 2 * 128 * 128;  // bytes of one bf16 K (or V) tile: two 64-wide boxes
  static constexpr int QBOX = 16 * 128;          // 16 rows x 64 16-bit elements
  static constexpr int Q_BYTES = 2 * QBOX;
  static constexpr int P_BYTES = 2 * QBOX;       // P^T: 16 rows x 128 tokens
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + NST * KV_TILE;
  static constexpr int OFF_Q = OFF_V + NST * KV_TILE;
  static constexpr int OFF_P = OFF_Q + Q_BYTES;
  static constexpr int OFF_RED = OFF_P + 2 * P_BYTES;  // [2][4 warps][16] maxima + [4][16] sums
  static constexpr int OFF_BAR = OFF_RED + (2 * 4 * 16 + 4 * 16) * 4;
  static constexpr int N_BARS = 4 * NST + 1 + 2 + 2 + 1 + 1 + 2 + 1 + 1;
  static constexpr int SMEM_BYTES = OFF_BAR + N_BARS * 8 + 16 + 1024;
  static constexpr int THREADS = 192;
  static constexpr uint32_t TMEM_COLS = 64;  // S^T double buffer (2 x 16) + O^T (16)
  static constexpr float RESCALE_THRESHOLD = 8.0f;
};

// Order-preserving integer image of a float (an involution), so a warp max is one redux.sync.
__device__ __forceinline__ int float_to_ordered(float f) {
  const int i = __float_as_int(f);
  return i ^ ((i >> 31) & 0x7fffffff);
}
__device__ __forceinline__ float ordered_to_float(int i) { return __int_as_float(i ^ ((i >> 31) & 0x7fffffff)); }
__device__ __forceinline__ float warp_max_redux(float v) {
  int r;
  asm volatile("redux.sync.max.s32 %0, %1, 0xffffffff;" : "=r"(r) : "r"(float_to_ordered(v)));
  return ordered_to_float(r);
}

template <int GP>
struct DecodeRows {
  float m_used[GP];  // log2-domain reference max per query row (lazy: moves by > threshold only)
  float l_part[GP];  // this thread's share of the row sums, relative to m_used
};

// One tile of the decode softmax on the thread that owns token t (= TMEM lane t of S^T and, for
// the O^T rescale, output element d = t), from this token's scores x[g] (log2 domain, -inf for a
// token past the length): row maxima (warp redux, then a bounded cross-warp exchange) -> lazy O
// rescale -> this token's entries of P^T (scaled by vs).  Returns false, warp-uniformly, if a
// bounded wait ran out.
// j counts the tiles this warpgroup has processed (it selects the phases of red_bar); has_prev
// says O^T already holds earlier tiles of the same split.  prev_pv / prev_pv_parity name the
// barrier phase that completes when the previous PV has finished (the O^T rescale must wait for
// it); the caller picks them so that the wait is unambiguous.
template <int GP, bool F16P>
__device__ __forceinline__ bool decode_softmax_core(DecodeRows<GP>& rows, const float (&x)[GP], int j,
                                                    bool has_prev, int lane, int wq, int t, float vs,
                                                    uint32_t tO_lane, float* red_max, uint64_t* red_bar,
                                                    uint64_t* prev_pv, uint32_t prev_pv_parity, uint8_t* p_tile,
                                                    float threshold) {
  float* rm = red_max + (j & 1) * 64;
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    const float m = warp_max_redux(x[g]);
    if (lane == 0) rm[wq * 16 + g] = m;
  }
  mbar_arrive(&red_bar[j & 1]);
  if (!mbar_wait_warp(&red_bar[j & 1], (j >> 1) & 1, SITE_DC_SM_S)) return false;
  bool need = false;
  float alpha[GP];
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    const float tm = fmaxf(fmaxf(rm[g], rm[16 + g]), fmaxf(rm[32 + g], rm[48 + g]));
    const float mn = fmaxf(rows.m_used[g], tm);
    alpha[g] = 1.f;
    if (mn > rows.m_used[g] + threshold) {  // the same decision on every thread of the CTA
      alpha[g] = ex2_approx(rows.m_used[g] - mn);
      rows.m_used[g] = mn;
      rows.l_part[g] *= alpha[g];
      need = true;
    }
  }
  if (need && has_prev) {  // rescale O^T row t once the previous PV is done
    if (!mbar_wait_warp(prev_pv, prev_pv_parity, SITE_DC_SM_O)) return false;
    tc_fence_after();
    uint32_t orow[16];
    tmem_ld16(tO_lane, orow);
    tmem_wait_ld();
#pragma unroll
    for (int g = 0; g < GP; ++g) orow[g] = __float_as_uint(__uint_as_float(orow[g]) * alpha[g]);
    tmem_st16(tO_lane, orow);
    tmem_wait_st();
  }
  uint8_t* prow = p_tile + (t >> 6) * (16 * 128);
  const uint32_t pchunk = (t & 63) >> 3, pbyte = (t & 7) * 2;
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    const float pr = (x[g] == -INFINITY) ? 0.f : ex2_approx(x[g] - rows.m_used[g]);
    rows.l_part[g] += pr;
    const float pv = pr * vs;
    const uint16_t bits = F16P ? __half_as_ushort(__float2half_rn(pv)) : __bfloat16_as_ushort(__float2bfloat16_rn(pv));
    *reinterpret_cast<uint16_t*>(prow + sw128_offset(g, pchunk) + pbyte) = bits;
  }
  return true;
}

// bf16 decode: the 16 S^T columns of this lane, scaled by sc (log2 domain), then the shared core.
// MULTI: several query tokens share the rows, each with its own key limit rlim[g]; otherwise every
// row's limit is t1 (kept as one compare).
template <int GP, bool F16P, bool MULTI>
__device__ __forceinline__ bool decode_softmax_tile(DecodeRows<GP>& rows, int j, bool has_prev, int lane, int wq,
                                                    int t, int tok, int t1, const int (&rlim)[GP], float sc, float vs,
                                                    uint32_t tS_lane,
                                                    uint32_t tO_lane, float* red_max, uint64_t* red_bar,
                                                    uint64_t* prev_pv, uint32_t prev_pv_parity, uint8_t* p_tile,
                                                    float threshold) {
  uint32_t sv[16];
  tmem_ld16(tS_lane, sv);
  tmem_wait_ld();
  float x[GP];
#pragma unroll
  for (int g = 0; g < GP; ++g)
    x[g] = (MULTI ? tok < rlim[g] : tok < t1) ? __uint_as_float(sv[g]) * sc : -INFINITY;
  return decode_softmax_core<GP, F16P>(rows, x, j, has_prev, lane, wq, t, vs, tO_lane, red_max, red_bar, prev_pv,
                                       prev_pv_parity, p_tile, threshold);
}

// Epilogue shared by the decode kernels: reduce the row sums over the warpgroup, wait for the last
// PV, then thread t (= output element d) writes o[g][t] = O^T[t][g] / l_g and, for t < G, lse_t.
// The last PV is awaited on a barrier that completes once per split (o_final, phase o_parity): on
// a per-tile barrier two phases can still be pending here, and a parity wait could be satisfied
// by the older one.  sum_parity is the phase of sum_bar; o_free (if not null) is arrived on once
// O^T has been read, so the accumulator can take the next split.
template <int GP, bool MULTI>
__device__ __forceinline__ bool decode_epilogue(DecodeRows<GP>& rows, const DecodeParams& p, int G, int split,
                                                int kvh, int b, int lane, int wq, int t, uint32_t tO_lane,
                                                float* red_sum, uint64_t* sum_bar, uint32_t sum_parity,
                                                uint64_t* o_final, uint32_t o_parity, uint64_t* o_free,
                                                int d_out = -1) {
  constexpr int D = 128;
  if (d_out < 0) d_out = t;  // the head-dimension element that TMEM lane t of O^T holds
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    const float s = warp_sum(rows.l_part[g]);
    if (lane == 0) red_sum[wq * 16 + g] = s;
  }
  mbar_arrive(sum_bar);
  if (!mbar_wait_warp(sum_bar, sum_parity, SITE_DC_SM_S)) return false;
  if (!mbar_wait_warp(o_final, o_parity, SITE_DC_SM_O)) return false;
  tc_fence_after();
  uint32_t orow[16];
  tmem_ld16(tO_lane, orow);
  tmem_wait_ld();
  if (o_free) {
    tc_fence_before();
    mbar_arrive(o_free);
  }
  float my_lse = -INFINITY;
  const int R = decode_rows(p);
  const long long rows_all = (long long)p.B * p.n_q * p.Hq;
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    if (g < R) {
      const float l = red_sum[g] + red_sum[16 + g] + red_sum[32 + g] + red_sum[48 + g];
      const float ov = (l > 0.f) ? __uint_as_float(orow[g]) / l : 0.f;
      const float lse = (l > 0.f) ? (rows.m_used[g] + log2f(l)) * 0.69314718055994531f : -INFINITY;
      if (g == t) my_lse = lse;
      const long long h = MULTI ? decode_row_index(p, b, kvh, g) : (long long)b * p.Hq + (long long)kvh * p.G + g;
      if (p.n_splits == 1) {
        p.o[h * D + d_out] = __float2bfloat16_rn(ov);
      } else {
        p.o_part[((long long)split * rows_all + h) * D + d_out] = ov;
      }
    }
  }
  if (t < R) {
    const long long h = MULTI ? decode_row_index(p, b, kvh, t) : (long long)b * p.Hq + (long long)kvh * p.G + t;
    if (p.n_splits == 1) {
      if (p.lse) p.lse[h] = my_lse;
    } else {
      p.lse_part[(long long)split * rows_all + h] = my_lse;
    }
  }
  return true;
}

// Empty split: o = 0, lse = -inf, written by threads tid = 0..nthreads-1 (no barrier or TMEM use).
__device__ __forceinline__ void decode_write_empty(const DecodeParams& p, int G, int split, int kvh, int b, int tid,
                                                   int nthreads) {
  constexpr int D = 128;
  const long long rows_all = (long long)p.B * p.n_q * p.Hq;
  for (int i = tid; i < decode_rows(p) * D; i += nthreads) {
    const int g = i / D, d = i % D;
    const long long h = decode_row_index(p, b, kvh, g);
    if (p.n_splits == 1) {
      p.o[h * D + d] = __float2bfloat16_rn(0.f);
      if (d == 0 && p.lse) p.lse[h] = -INFINITY;
    } else {
      p.o_part[((long long)split * rows_all + h) * D + d] = 0.f;
      if (d == 0) p.lse_part[(long long)split * rows_all + h] = -INFINITY;
    }
  }
}

// Chunk c (< 256) of the query rows: row r = c / 16, elements 8 (c % 16) .. + 7 (zero for r past
// the n_q * G rows).
__device__ __forceinline__ uint4 decode_q_chunk_load(const DecodeParams& p, int G, int kvh, int b, int c) {
  constexpr int D = 128;
  const int r = c >> 4, cc = c & 15;
  uint4 x = make_uint4(0u, 0u, 0u, 0u);
  if (r < p.n_q * G) x = *reinterpret_cast<const uint4*>(p.q + decode_row_index(p, b, kvh, r) * D + cc * 8);
  return x;
}

// Q^T rows of the group into the 128B-swizzled bf16 B operand: two 64-wide boxes of 16 rows
// (rows >= G zero).  Threads tid = 0..nthreads-1 share the work.
__device__ __forceinline__ void decode_stage_q(const DecodeParams& p, int G, int kvh, int b, int tid, int nthreads,
                                               uint8_t* q_smem) {
  for (int c = tid; c < 256; c += nthreads) {
    const int g = c >> 4, cc = c & 15;
    *reinterpret_cast<uint4*>(q_smem + (cc >> 3) * (16 * 128) + sw128_offset(g, cc & 7)) =
        decode_q_chunk_load(p, G, kvh, b, c);
  }
}

template <int GP, bool MULTI>
__global__ void __launch_bounds__(192, 1)
    decode_split_sm100(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const DecodeParams p) {
  using C = DecodeCfg;
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int len = p.kv_lens[b];
  len = len < 0 ? 0 : (len > p.Tmax ? p.Tmax : len);
  const int t0 = split * p.split_tokens;
  const int t1 = min(len, t0 + p.split_tokens);
  const int n = t1 > t0 ? (t1 - t0 + 127) / 128 : 0;
  const int G = p.G;
  if (n == 0) {
    decode_write_empty(p, G, split, kvh, b, threadIdx.x, blockDim.x);
    return;
  }

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* k_full = bars;
  uint64_t* k_empty = k_full + C::NST;
  uint64_t* v_full = k_empty + C::NST;
  uint64_t* v_empty = v_full + C::NST;
  uint64_t* q_ready = v_empty + C::NST;
  uint64_t* s_full = q_ready + 1;  // [2]
  uint64_t* p_full = s_full + 2;   // [2]
  uint64_t* o_ready = p_full + 2;
  uint64_t* drain = o_ready + 1;
  uint64_t* red_bar = drain + 1;  // [2] cross-warp exchange of the tile maxima
  uint64_t* sum_bar = red_bar + 2;
  uint64_t* o_final = sum_bar + 1;  // single phase: every PV of the split has completed
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(o_final + 1);
  float* red_max = reinterpret_cast<float*>(smem + C::OFF_RED);  // [2][4][16]
  float* red_sum = red_max + 2 * 4 * 16;                         // [4][16]

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    mbar_init(q_ready, 128);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 128);
      mbar_init(&red_bar[s], 128);
    }
    mbar_init(o_ready, 1);
    mbar_init(drain, 1);
    mbar_init(sum_bar, 128);
    mbar_init(o_final, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tS0 = tmem, tO = tmem + 32;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int issued = 0;
      bool ok = true;
      PageCursor pc;
      for (int j = 0; j < n; ++j) {
        const int st = j % C::NST;
        const uint32_t ph = (j / C::NST) & 1;
        const int tok = t0 + j * 128;
        const int pg = pc.get(p, b, tok), off = pc.offset(p, tok);
        if (!(ok = mbar_wait(&k_empty[st], ph ^ 1, SITE_DC_LOAD_EMPTY))) break;
        mbar_arrive_expect_tx(&k_full[st], C::KV_TILE);
        tma_load_4d(smem + C::OFF_K + st * C::KV_TILE, &tmK, &k_full[st], 0, kvh, off, pg);
        tma_load_4d(smem + C::OFF_K + st * C::KV_TILE + 128 * 128, &tmK, &k_full[st], 64, kvh, off, pg);
        issued = 2 * j + 1;
        if (!(ok = mbar_wait(&v_empty[st], ph ^ 1, SITE_DC_LOAD_EMPTY))) break;
        mbar_arrive_expect_tx(&v_full[st], C::KV_TILE);
        tma_load_4d(smem + C::OFF_V + st * C::KV_TILE, &tmV, &v_full[st], 0, kvh, off, pg);
        tma_load_4d(smem + C::OFF_V + st * C::KV_TILE + 128 * 128, &tmV, &v_full[st], 64, kvh, off, pg);
        issued = 2 * j + 2;
      }
      if (!ok) {
        const int nk = (issued + 1) / 2, nv = issued / 2;
        for (int j = (nk > C::NST ? nk - C::NST : 0); j < nk; ++j)
          mbar_wait_drain(&k_full[j % C::NST], (j / C::NST) & 1, SITE_DC_DRAIN);
        for (int j = (nv > C::NST ? nv - C::NST : 0); j < nv; ++j)
          mbar_wait_drain(&v_full[j % C::NST], (j / C::NST) & 1, SITE_DC_DRAIN);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = make_idesc_f16(128, 16, false, false, true);
      constexpr uint32_t idesc_pv = make_idesc_f16(128, 16, true, false, true);
      const uint32_t sQ = smem_u32(smem + C::OFF_Q);
      const uint32_t sP = smem_u32(smem + C::OFF_P);
      const uint32_t sK = smem_u32(smem + C::OFF_K);
      const uint32_t sV = smem_u32(smem + C::OFF_V);
      auto issue_s = [&](uint32_t kbase, int buf) {  // S^T(j) = K_j . Q^T
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
          const uint32_t qoff = (kk >> 2) * C::QBOX + (kk & 3) * 32;
          mma_ss(tS0 + buf * 16, make_sdesc_sw128(kbase + koff, 16, 1024), make_sdesc_sw128(sQ + qoff, 16, 1024),
                 idesc_qk, kk > 0);
        }
      };
      auto issue_pv = [&](uint32_t vbase, int pbuf, bool acc) {  // O^T += V_j^T . P_j^T
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t da = make_sdesc_sw128(vbase + kk * 16 * 128, 128 * 128, 1024);
          const uint64_t db =
              make_sdesc_sw128(sP + pbuf * C::P_BYTES + (kk >> 2) * C::QBOX + (kk & 3) * 32, 16, 1024);
          mma_ss(tO, da, db, idesc_pv, (acc || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(q_ready, 0, SITE_DC_MMA_K);
      for (int jj = 0; jj < 2 && jj < n && ok; ++jj) {
        if (!(ok = mbar_wait(&k_full[jj % C::NST], (jj / C::NST) & 1, SITE_DC_MMA_K))) break;
        tc_fence_after();
        issue_s(sK + (jj % C::NST) * C::KV_TILE, jj & 1);
        mma_commit(&s_full[jj & 1]);
        mma_commit(&k_empty[jj % C::NST]);
      }
      for (int j = 0; j < n && ok; ++j) {
        const int st = j % C::NST;
        if (!(ok = mbar_wait(&v_full[st], (j / C::NST) & 1, SITE_DC_MMA_V))) break;
        if (!(ok = mbar_wait(&p_full[j & 1], (j >> 1) & 1, SITE_DC_MMA_P))) break;
        tc_fence_after();
        issue_pv(sV + st * C::KV_TILE, j & 1, j > 0);
        mma_commit(o_ready);
        mma_commit(&v_empty[st]);
        if (j + 2 < n) {
          const int st2 = (j + 2) % C::NST;
          if (!(ok = mbar_wait(&k_full[st2], ((j + 2) / C::NST) & 1, SITE_DC_MMA_K))) break;
          tc_fence_after();
          issue_s(sK + st2 * C::KV_TILE, j & 1);
          mma_commit(&s_full[j & 1]);
          mma_commit(&k_empty[st2]);
        }
      }
      if (ok) mma_commit(o_final);
      mma_commit(drain);
      mbar_wait_drain(drain, 0, SITE_DC_DRAIN);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax warpgroup
    const int wq = warp & 3;
    const int t = wq * 32 + lane;  // token of the tile / TMEM lane / output element d
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const int wg_tid = threadIdx.x - 64;
    for (int i = wg_tid; i < 2 * C::P_BYTES / 16; i += 128)  // P^T rows >= GP stay zero
      reinterpret_cast<uint4*>(smem + C::OFF_P)[i] = make_uint4(0u, 0u, 0u, 0u);
    decode_stage_q(p, G, kvh, b, wg_tid, 128, smem + C::OFF_Q);
    fence_proxy_async_smem();
    mbar_arrive(q_ready);

    DecodeRows<GP> rows;
    int rlim[GP];  // per-row exclusive key limits (a query token sees its own causal prefix)
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      rows.m_used[g] = -INFINITY;
      rows.l_part[g] = 0.f;
      rlim[g] = g < decode_rows(p) ? decode_row_limit(p, len, t1, g) : t1;
    }
    bool ok = true;
    for (int j = 0; j < n && ok; ++j) {
      const int st = j % C::NST;
      const uint32_t ph = (j / C::NST) & 1;
      const int tok = t0 + j * 128 + t;
      const bool valid = tok < t1;
      // tcgen05.ld/st are warp-collective: every lane takes the same branch around them.
      if (!(ok = mbar_wait_warp(&s_full[j & 1], (j >> 1) & 1, SITE_DC_SM_S))) break;
      tc_fence_after();
      // PV(j-1) is the j-th completion of o_ready; S(j) completing implies PV(j-2) done, so at
      // most one phase is pending and the parity wait is unambiguous.
      if (!(ok = decode_softmax_tile<GP, false, MULTI>(rows, j, j > 0, lane, wq, t, tok, t1, rlim, p.scale_log2, 1.f,
                                                tS0 + (j & 1) * 16 + lane_off, tO + lane_off, red_max, red_bar,
                                                o_ready, (j - 1) & 1, smem + C::OFF_P + (j & 1) * C::P_BYTES,
                                                C::RESCALE_THRESHOLD)))
        break;
      if (t1 - (t0 + j * 128) < 128) {
        // last, partial tile: cache slots past the length may hold anything (NaN included);
        // zero those V rows so a 0-probability x slot product cannot poison the sum.
        if (!(ok = mbar_wait_warp(&v_full[st], ph, SITE_DC_SM_V))) break;
        if (!valid) {
          uint4* r0 = reinterpret_cast<uint4*>(smem + C::OFF_V + st * C::KV_TILE + t * 128);
          uint4* r1 = reinterpret_cast<uint4*>(smem + C::OFF_V + st * C::KV_TILE + 128 * 128 + t * 128);
#pragma unroll
          for (int i = 0; i < 8; ++i) r0[i] = r1[i] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[j & 1]);
    }
    if (ok)
      decode_epilogue<GP, MULTI>(rows, p, G, split, kvh, b, lane, wq, t, tO + lane_off, red_sum, sum_bar, 0, o_final, 0,
                          nullptr);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace attn
