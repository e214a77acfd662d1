// Split-KV GQA decode over an FP8 E4M3 KV cache (LLM-CoOpt summary, "Opt-KV": the cache is
// stored in FP8 to halve the bytes per token; ONNX Runtime CPU GQA analysis, "Flash Decoding":
// split the key range, merge the partial softmax states by log-sum-exp).
//
// Same arithmetic as the bf16 kernel (KV tokens on the MMA's M axis: S^T = K.Q^T and
// O^T += V^T.P^T), but both MMAs run on the E4M3 codes exactly as the TMA brings them
// (kind::f8f6f4, K = 32 per instruction); no code is ever converted:
//   * Q as three E4M3 pieces per query row: the row is scaled by 2^e (its largest magnitude lands
//     in (224, 448]), x = q 2^e, and x = p1 + p2 / 16 + p3 / 256 with p1 = e4m3(x),
//     p2 = e4m3(16 (x - p1)), p3 = e4m3(16 (16 (x - p1) - p2)).  This is exact for a bf16 q unless
//     an element lies some 2^14 below the row maximum (the E4M3 residual of a bf16 value has at
//     most 4 significant bits).  The pieces are the B rows of the score MMA, whose A operand is
//     the K code tile; the tensor core sums code x piece products exactly in fp32, and the
//     softmax combines the three score columns, undoes 2^e and applies k_scale;
//   * P^T as four E4M3 pieces per query row, written by the softmax: pv = p v_scale (the token's
//     V dequant scale folded into its probability) = p1 + p2 / 16 + p3 / 256 + p4 / 4096 (relative
//     error 2^-16, absolute floor 2^-23).  The PV MMA reads V^T straight from the code tile
//     (an MN-major A operand) and accumulates one O^T column per (piece, row); the epilogue
//     combines them.  To keep pv inside E4M3's range the running maximum is taken over
//     y = x + log2(v_scale) instead of the score x: then pv = 2^(y - m) <= 2^threshold, while
//     l = sum 2^(x - m) is still the softmax denominator for the same m.
//
// Persistent CTAs: CTA c takes the work items (split, KV head, sequence) c, c + grid, c + 2 grid,
// ... and every role runs straight from one item into the next, so the next item's loads, Q
// staging and first score tiles overlap the current item's last tiles and epilogue.  A tile is
// named by its index in the CTA's whole sequence of tiles (all its items, empty items skipped).
//
// Roles (256 threads):
//   warp 0       TMA producer of the raw K code tiles (NCS_K-stage ring, freed by S completing)
//   warp 1       TMEM allocator; lane 0 issues the S MMAs (as soon as K lands and a buffer is free)
//   warp 2       Q stager (whole warp, double-buffered, loads one item ahead) and, on lane 0, TMA
//                producer of the raw V code tiles (NCS_V-stage ring, freed by PV completing)
//   warps 3..6   softmax + epilogue: thread = token (and later = output element d)
//   warp 7       lane 0 issues the PV MMAs
// S and PV have separate issuing threads (each commit tracks its own thread's MMAs), so a late K
// copy never holds up a PV and a late P never holds up the S that frees a K stage.  S^T and P^T
// rotate through NS buffers (more than either stage count); O^T is double-buffered per item.
// A tcgen05.commit or a barrier wait costs an issuing thread tens of cycles, so completions are
// shared: S(j) done (s_full) frees K stage j % NCS_K; PV(j) done (pv_done) frees V stage j % NCS_V
// and P^T buffer j % NS; the V copy of tile j completes its bytes on p_full(j), which the
// softmax's P(j) arrivals also complete, so PV(j) waits on one barrier.
// TMEM columns: S^T NS buffers of NQ = 3 GP (rounded up to 16) columns from 0, O^T two buffers of
// NP = 4 GP (rounded up to 16) columns from 256.
#pragma once

#include "decode.cuh"

namespace attn {

// Shared-memory and TMEM layout for a query group padded to GP rows.  A V stage is held from its
// copy until PV of its tile completes, which trails the softmax, while the copy itself takes
// microseconds under a full HBM load; so V gets as many stages as shared memory allows, and NS
// (S^T / P^T buffers) stays one above the stage counts, which lets completions free stages.
template <int GP>
struct DecodeFp8Cfg {
  static constexpr int D = 128;
  static constexpr int NQ = ((3 * GP + 15) / 16) * 16;  // S^T columns per buffer = B rows of the Q pieces
  static constexpr int NP = ((4 * GP + 15) / 16) * 16;  // O^T columns per buffer = B rows of the P pieces
  static constexpr int NCS_K = 4;                       // stages of raw K code tiles
  static constexpr int NCS_V = GP <= 4 ? 8 : (GP <= 8 ? 7 : 5);  // stages of raw V code tiles
  static constexpr int NS = NCS_V + 1;                  // S^T (TMEM) and P^T (shared) buffers
  static constexpr int CODE_TILE = 128 * 128;           // 128 tokens x 128 one-byte codes
  static constexpr int Q_BYTES = ((NQ * 128 + 1023) / 1024) * 1024;  // Q pieces: rows of 128 codes (d)
  static constexpr int P_BYTES = ((NP * 128 + 1023) / 1024) * 1024;  // P pieces: rows of 128 codes (tokens)
  static constexpr int OFF_KCODE = 0;
  static constexpr int OFF_VCODE = OFF_KCODE + NCS_K * CODE_TILE;
  static constexpr int OFF_Q = OFF_VCODE + NCS_V * CODE_TILE;
  static constexpr int OFF_P = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_QEXP = OFF_P + NS * P_BYTES;  // [2][16] row exponents e
  static constexpr int OFF_RED = OFF_QEXP + 2 * 16 * 4;
  static constexpr int OFF_SCALE = OFF_RED + (2 * 4 * 16 + 4 * 16) * 4;  // [NCS_V][k, v][128] per-token scales
  static constexpr int OFF_BAR = OFF_SCALE + NCS_V * 2 * 128 * 4;
  static constexpr int N_BARS = NCS_K + 4 * NS + 10 + 4 + NCS_V;
  static constexpr int SMEM_BYTES = OFF_BAR + N_BARS * 8 + 16 + 1024;
  static constexpr int THREADS = 256;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_O = NS * NQ;
  static constexpr float RESCALE_THRESHOLD = 8.0f;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");
  static_assert(NS > NCS_K && NS > NCS_V, "freeing a stage by a shared S / PV completion needs NS > stages");
  static_assert(COL_O + 2 * NP <= TMEM_COLS, "TMEM columns");
  // Each CTA allocates all 512 TMEM columns; its shared memory keeps a second CTA off the SM.
  static_assert(2 * SMEM_BYTES > 228 * 1024, "one CTA per SM");
  static_assert(OFF_Q % 1024 == 0 && OFF_P % 1024 == 0, "128B-swizzled operands start on 1024-byte boundaries");
};

// One work item of the persistent decode: a split of one (sequence, KV head).
struct DecodeItem {
  int split, kvh, b;
  int len;     // the sequence's length
  int t0, t1;  // token range [t0, t1)
  int n;       // 128-token tiles (0: empty split)
};

__device__ __forceinline__ DecodeItem decode_item(const DecodeParams& p, int w) {
  DecodeItem it;
  it.split = w % p.n_splits;
  it.kvh = (w / p.n_splits) % p.Hkv;
  it.b = w / (p.n_splits * p.Hkv);
  int len = __ldg(p.kv_lens + it.b);
  len = len < 0 ? 0 : (len > p.Tmax ? p.Tmax : len);
  it.len = len;
  it.t0 = it.split * p.split_tokens;
  it.t1 = min(len, it.t0 + p.split_tokens);
  it.n = it.t1 > it.t0 ? (it.t1 - it.t0 + 127) / 128 : 0;
  return it;
}

// Walks this CTA's items with tiles, in order (empty items are skipped: the softmax warpgroup
// writes their results itself).
struct DecodeItemIter {
  int w, n_items;
  DecodeItem cur;
  __device__ __forceinline__ explicit DecodeItemIter(const DecodeParams& p)
      : w((int)blockIdx.x - (int)gridDim.x), n_items(p.n_splits * p.Hkv * p.B) {}
  __device__ __forceinline__ bool next(const DecodeParams& p) {
    for (w += gridDim.x; w < n_items; w += gridDim.x) {
      cur = decode_item(p, w);
      if (cur.n > 0) return true;
    }
    return false;
  }
};

// 2^e as a float, e in [-126, 127].
__device__ __forceinline__ float pow2i(int e) { return __int_as_float((e + 127) << 23); }

// Exponent e that puts the row maximum m (>= 0) into (224, 448]: m = 1.f x 2^E with
// 1.f <= 1.75 -> e = 8 - E, else e = 7 - E; clamped to [-126, 100] (0 for an all-zero row).
__device__ __forceinline__ int q_row_exponent(float m) {
  const uint32_t bits = __float_as_uint(m);
  const int eb = (int)(bits >> 23) & 255;
  if (eb == 0) return m > 0.f ? 100 : 0;  // zero or subnormal row maximum
  const int e = ((bits & 0x7FFFFFu) <= 0x600000u ? 135 : 134) - eb;
  return e < -126 ? -126 : (e > 100 ? 100 : e);
}

// Eight scaled query elements -> the eight codes of each of the three E4M3 pieces.
__device__ __forceinline__ void q_pieces8(const uint4 x, float scale, uint2& p1, uint2& p2, uint2& p3) {
  const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
  uint32_t c1[2], c2[2], c3[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t w1 = 0, w2 = 0, w3 = 0;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint32_t v = xw[2 * h + i];
      const float a = __uint_as_float(v << 16) * scale, b = __uint_as_float(v & 0xFFFF0000u) * scale;
      const uint16_t q1 = f32x2_to_e4m3x2(a, b);
      const uint32_t d1w = e4m3x2_to_f16x2(q1);
      const __half2 d1 = *reinterpret_cast<const __half2*>(&d1w);
      const float ra = (a - __low2float(d1)) * 16.f, rb = (b - __high2float(d1)) * 16.f;
      const uint16_t q2 = f32x2_to_e4m3x2(ra, rb);
      const uint32_t d2w = e4m3x2_to_f16x2(q2);
      const __half2 d2 = *reinterpret_cast<const __half2*>(&d2w);
      const uint16_t q3 = f32x2_to_e4m3x2((ra - __low2float(d2)) * 16.f, (rb - __high2float(d2)) * 16.f);
      w1 |= (uint32_t)q1 << (16 * i);
      w2 |= (uint32_t)q2 << (16 * i);
      w3 |= (uint32_t)q3 << (16 * i);
    }
    c1[h] = w1;
    c2[h] = w2;
    c3[h] = w3;
  }
  p1 = make_uint2(c1[0], c1[1]);
  p2 = make_uint2(c2[0], c2[1]);
  p3 = make_uint2(c3[0], c3[1]);
}


// N (16, 32, 48 or 64) consecutive TMEM columns of this warp's 32 lanes.
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&v)[N]) {
  static_assert(N == 16 || N == 32 || N == 48 || N == 64, "column count");
  if constexpr (N == 16) {
    tmem_ld16(taddr, v);
    tmem_wait_ld_regs(v);
  } else if constexpr (N == 32) {
    tmem_ld32(taddr, v);
    tmem_wait_ld_regs(v);
  } else {
    uint32_t a[32], b[N - 32];
    tmem_ld32(taddr, a);
    if constexpr (N == 48) tmem_ld16(taddr + 32, b);
    else tmem_ld32(taddr + 32, b);
    tmem_wait_ld_regs(a);
    tmem_wait_ld_regs(b);
#pragma unroll
    for (int c = 0; c < 32; ++c) v[c] = a[c];
#pragma unroll
    for (int c = 0; c < N - 32; ++c) v[32 + c] = b[c];
  }
}

template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t (&v)[N]) {
  static_assert(N == 16 || N == 32 || N == 64, "column count");
  if constexpr (N == 16) {
    tmem_st16(taddr, v);
  } else if constexpr (N == 32) {
    tmem_st32(taddr, v);
  } else {
    uint32_t a[32], b[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      a[c] = v[c];
      b[c] = v[32 + c];
    }
    tmem_st32(taddr, a);
    tmem_st32(taddr + 32, b);
  }
}

// Four E4M3 pieces of a and b (|a|, |b| <= 448): piece k holds 16^k times the residual left by
// pieces 0 .. k-1, so a = c0 + c1 / 16 + c2 / 256 + c3 / 4096 up to 2^-16 relative (2^-23 absolute
// below E4M3's normal range).  c[k] carries a in its low byte and b in its high byte.
__device__ __forceinline__ void e4m3_pieces4(float a, float b, uint16_t (&c)[4]) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    c[k] = f32x2_to_e4m3x2(a, b);
    if (k < 3) {
      const uint32_t dw = e4m3x2_to_f16x2(c[k]);
      const __half2 d = *reinterpret_cast<const __half2*>(&dw);
      a = (a - __low2float(d)) * 16.f;
      b = (b - __high2float(d)) * 16.f;
    }
  }
}

// Byte of P^T row r (a 128-byte row of tokens, 128B swizzle) for token t.
__device__ __forceinline__ uint32_t p8_offset(int r, int t) {
  return (uint32_t)r * 128u + ((((uint32_t)t >> 4) ^ ((uint32_t)r & 7u)) << 4) + ((uint32_t)t & 15u);
}

// One tile of the FP8 decode softmax on the thread that owns token t (= TMEM lane t of S^T and,
// for the O^T rescale, output element d = t).  Scores x (log2 domain) from the three piece columns;
// the row maxima are taken over y = x + log2 |v_scale| (warp redux, then a bounded cross-warp
// exchange); lazy O^T rescale; p = 2^(x - m) into l and pv = p v_scale (<= 2^threshold) as four
// E4M3 pieces into P^T.  j counts this warpgroup's tiles (phases of red_bar); has_prev says O^T
// already holds earlier tiles of the item; prev_pv / prev_pv_parity name the unambiguous phase
// that completes with the previous PV.  Returns false, warp-uniformly, if a bounded wait ran out.
template <int GP, int NQ, int NP, int NS, bool MULTI>
__device__ __forceinline__ bool fp8_softmax_tile(DecodeRows<GP>& rows, int j, bool has_prev, int lane, int wq, int t,
                                                 int tok, int t1, const int (&rlim)[GP], float sck, float vs,
                                                 const float (&fq)[GP],
                                                 uint32_t tS_lane, uint32_t tO_lane, float* red_max,
                                                 uint64_t* red_bar, uint64_t* s_free, uint64_t* pv_done,
                                                 uint8_t* p_tile, float threshold) {
  uint32_t sv[NQ];
  tmem_ld_cols<NQ>(tS_lane, sv);
  tc_fence_before();
  mbar_arrive(&s_free[j % NS]);  // S^T buffer j % NS may take S(j + NS)
  const float lv = __log2f(fmaxf(fabsf(vs), 7.8886091e-31f));  // 2^-100 floor keeps 2^(x - m) finite
  float x[GP], y[GP];
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    const float s12 = fmaf(__uint_as_float(sv[2 * GP + g]), 0.0625f, __uint_as_float(sv[GP + g]));
    const float s = fmaf(s12, 0.0625f, __uint_as_float(sv[g]));
    x[g] = (MULTI ? tok < rlim[g] : tok < t1) ? s * (sck * fq[g]) : -INFINITY;
    y[g] = x[g] + lv;
  }
  float* rm = red_max + (j & 1) * 64;
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    const float m = warp_max_redux(y[g]);
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
  if (need && has_prev) {  // rescale O^T row t (every piece column) once the previous PV is done
    // PV(j-1) is completion (j-1)/NS of pv_done[(j-1)%NS]; PV(j-1-NS) was awaited before P(j-1)
    // was written, so this is the one pending phase.
    if (!mbar_wait_warp(&pv_done[(j - 1) % NS], (uint32_t)((j - 1) / NS) & 1, SITE_DC_SM_O)) return false;
    tc_fence_after();
    uint32_t o[NP];
    tmem_ld_cols<NP>(tO_lane, o);
#pragma unroll
    for (int c = 0; c < NP; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha[c % GP]);
    tmem_st_cols<NP>(tO_lane, o);
    tmem_wait_st();
  }
  float pv[GP + (GP & 1)];
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    const float pr = (x[g] == -INFINITY) ? 0.f : ex2_approx(x[g] - rows.m_used[g]);
    rows.l_part[g] += pr;
    pv[g] = pr * vs;
  }
  if (GP & 1) pv[GP] = 0.f;
  // P^T buffer j % NS last held P(j - NS): wait for PV(j - NS) to have read it (one phase pending:
  // PV(j - 2 NS) was awaited here NS tiles ago, and PV(j) needs this P).
  if (j >= NS && !mbar_wait_warp(&pv_done[j % NS], (uint32_t)((j / NS) & 1) ^ 1, SITE_DC_SM_P)) return false;
#pragma unroll
  for (int g = 0; g < GP; g += 2) {
    uint16_t c[4];
    e4m3_pieces4(pv[g], pv[g + 1], c);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      p_tile[p8_offset(k * GP + g, t)] = (uint8_t)(c[k] & 0xFF);
      if (g + 1 < GP) p_tile[p8_offset(k * GP + g + 1, t)] = (uint8_t)(c[k] >> 8);
    }
  }
  return true;
}

// Epilogue of an item: reduce the row sums over the warpgroup, wait for the item's last PV
// (o_full, phase o_parity), read O^T (then release it through o_free), and thread t (= output
// element d) writes o[g][t] = (sum over pieces k of O^T[t][k GP + g] / 16^k) / l_g and, for t < G,
// lse_t = ln 2 (m_g + log2 l_g).
template <int GP, int NP, bool MULTI>
__device__ __forceinline__ bool fp8_epilogue(DecodeRows<GP>& rows, const DecodeParams& p, int G, int split, int kvh,
                                             int b, int lane, int wq, int t, uint32_t tO_lane, float* red_sum,
                                             uint64_t* sum_bar, uint32_t sum_parity, uint64_t* o_full,
                                             uint32_t o_parity, uint64_t* o_free) {
  constexpr int D = 128;
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    const float s = warp_sum(rows.l_part[g]);
    if (lane == 0) red_sum[wq * 16 + g] = s;
  }
  mbar_arrive(sum_bar);
  if (!mbar_wait_warp(sum_bar, sum_parity, SITE_DC_SM_S)) return false;
  if (!mbar_wait_warp(o_full, o_parity, SITE_DC_SM_O)) return false;
  tc_fence_after();
  uint32_t o[NP];
  tmem_ld_cols<NP>(tO_lane, o);
  tc_fence_before();
  mbar_arrive(o_free);
  float my_lse = -INFINITY;
  const int R = decode_rows(p);
  const long long rows_all = (long long)p.B * p.n_q * p.Hq;
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    if (g < R) {
      const float l = red_sum[g] + red_sum[16 + g] + red_sum[32 + g] + red_sum[48 + g];
      const float c23 = fmaf(__uint_as_float(o[3 * GP + g]), 0.0625f, __uint_as_float(o[2 * GP + g]));
      const float c123 = fmaf(c23, 0.0625f, __uint_as_float(o[GP + g]));
      const float acc = fmaf(c123, 0.0625f, __uint_as_float(o[g]));
      const float ov = (l > 0.f) ? acc / l : 0.f;
      const float lse = (l > 0.f) ? (rows.m_used[g] + log2f(l)) * 0.69314718055994531f : -INFINITY;
      if (g == t) my_lse = lse;
      const long long h = MULTI ? decode_row_index(p, b, kvh, g) : (long long)b * p.Hq + (long long)kvh * p.G + g;
      if (p.n_splits == 1) {
        p.o[h * D + t] = __float2bfloat16_rn(ov);
      } else {
        p.o_part[((long long)split * rows_all + h) * D + t] = ov;
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

template <int GP, bool MULTI>
__global__ void __launch_bounds__(256, 1)
    decode_fp8_sm100(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const DecodeParams p) {
  using C = DecodeFp8Cfg<GP>;
  constexpr int NS = C::NS, NCS_K = C::NCS_K, NCS_V = C::NCS_V, NQ = C::NQ, NP = C::NP;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.G;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* k_full = bars;             // [NCS_K] raw K codes landed
  uint64_t* s_full = k_full + NCS_K;   // [NS] S^T(j) in TMEM; K stage j % NCS_K read
  uint64_t* p_full = s_full + NS;      // [NS] P^T(j) written (128 arrivals) and V(j) landed (1 + bytes)
  uint64_t* pv_done = p_full + NS;     // [NS] PV(j) completed: P^T(j) and V stage j % NCS_V read
  uint64_t* s_free = pv_done + NS;     // [NS] the softmax has read S^T(j)
  uint64_t* q_full = s_free + NS;      // [2] Q pieces of an item staged
  uint64_t* q_free = q_full + 2;       // [2] the item's S MMAs have read them
  uint64_t* o_full = q_free + 2;       // [2] every PV of an item has completed
  uint64_t* o_free = o_full + 2;       // [2] the epilogue has read O^T
  uint64_t* red_bar = o_free + 2;      // [2]
  uint64_t* sum_bar = red_bar + 2;
  uint64_t* drain = sum_bar + 1;       // S issuer's MMAs completed
  uint64_t* drain_pv = drain + 1;      // PV issuer's MMAs completed
  uint64_t* exp_bar = drain_pv + 1;    // the softmax's row exponents of an item are in q_exp
  uint64_t* sc_full = exp_bar + 1;     // [NCS_V] the per-token scales of V stage j % NCS_V landed
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sc_full + NCS_V);
  float* scales = reinterpret_cast<float*>(smem + C::OFF_SCALE);  // [NCS_V][2][128]
  int* q_exp = reinterpret_cast<int*>(smem + C::OFF_QEXP);       // [2][16] softmax's row exponents
  float* red_max = reinterpret_cast<float*>(smem + C::OFF_RED);  // [2][4][16]
  float* red_sum = red_max + 2 * 4 * 16;                         // [4][16]

  if (threadIdx.x == 0) {
    for (int i = 0; i < NCS_K; ++i) mbar_init(&k_full[i], 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128 + 1);
      mbar_init(&pv_done[i], 1);
      mbar_init(&s_free[i], 128);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_free[i], 1);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_free[i], 128);
      mbar_init(&red_bar[i], 128);
    }
    mbar_init(sum_bar, 128);
    mbar_init(drain, 1);
    mbar_init(drain_pv, 1);
    mbar_init(exp_bar, 128);
    for (int i = 0; i < NCS_V; ++i) mbar_init(&sc_full[i], 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::TMEM_COLS);
    tmem_relinquish();
  }
  // Zero both Q piece buffers (rows past 3 GP stay zero) and the P^T buffers (rows past 4 GP).
  for (int i = threadIdx.x; i < 2 * C::Q_BYTES / 16; i += C::THREADS)
    reinterpret_cast<uint4*>(smem + C::OFF_Q)[i] = make_uint4(0u, 0u, 0u, 0u);
  for (int i = threadIdx.x; i < NS * C::P_BYTES / 16; i += C::THREADS)
    reinterpret_cast<uint4*>(smem + C::OFF_P)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tS0 = tmem, tO0 = tmem + C::COL_O;
  ATTN_EVT_INIT();

  if (warp == 0) {
    // ------------------------------------------------------------------ K producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      DecodeItemIter it(p);
      int j = 0;  // tiles issued
      bool ok = true;
      PageCursor pc;
      while (ok && it.next(p)) {
        for (int l = 0; l < it.cur.n; ++l, ++j) {
          const int st = j % NCS_K;
          const int tok0 = it.cur.t0 + l * 128;
          const int pg = pc.get(p, it.cur.b, tok0);
          // Stage st last held tile j - NCS_K: S(j - NCS_K) completing frees it.  That barrier phase
          // is unambiguous: S(j - NCS_K - NS) completed before tile j - NS was loaded, and the next
          // S on the barrier, S(j - NCS_K + NS), needs a later load (NS > NCS_K).
          if (j >= NCS_K && !(ok = mbar_wait(&s_full[(j - NCS_K) % NS], ((j - NCS_K) / NS) & 1, SITE_DC_LOAD_EMPTY)))
            break;
          mbar_arrive_expect_tx(&k_full[st], C::CODE_TILE);
          ATTN_EVT(j, 0);
          tma_load_4d(smem + C::OFF_KCODE + st * C::CODE_TILE, &tmK, &k_full[st], 0, it.cur.kvh,
                      pc.offset(p, tok0), pg);
        }
      }
      if (!ok)  // wait (bounded) for the copies still in flight before the CTA exits
        for (int jj = (j > NCS_K ? j - NCS_K : 0); jj < j; ++jj)
          mbar_wait_drain(&k_full[jj % NCS_K], (jj / NCS_K) & 1, SITE_DC_DRAIN);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------------ Q stager + V producer
    // Lane l holds the query chunks c = l + 32 i (row g = 2 i + l / 16, elements 8 (l % 16) ..
    // + 7) of the next item, loaded one item ahead.  At the start of an item the warp turns them
    // into the E4M3 pieces in Q buffer (item & 1), once that buffer has been released.
    if (lane == 0) tma_prefetch_desc(&tmV);
    DecodeItemIter it(p), ahead(p);
    uint4 qx[8];
    if (ahead.next(p)) {
#pragma unroll
      for (int i = 0; i < 8; ++i) qx[i] = decode_q_chunk_load(p, G, ahead.cur.kvh, ahead.cur.b, lane + 32 * i);
    }
    int j = 0, ie = 0;
    bool ok = true;
    PageCursor vpc;
    while (ok && it.next(p)) {
      const int qb = ie & 1;
      if (!(ok = mbar_wait_warp(&q_free[qb], ((ie >> 1) & 1) ^ 1, SITE_DC_Q))) break;
      uint8_t* qs = smem + C::OFF_Q + qb * C::Q_BYTES;
      const int cc = lane & 15;  // 8-element chunk of the row
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int g = 2 * i + (lane >> 4);
        if (2 * i >= GP) break;  // rows >= GP do not exist in this layout
        float m = 0.f;
        const uint32_t xw[4] = {qx[i].x, qx[i].y, qx[i].z, qx[i].w};
#pragma unroll
        for (int k = 0; k < 4; ++k)
          m = fmaxf(m, fmaxf(fabsf(__uint_as_float(xw[k] << 16)), fabsf(__uint_as_float(xw[k] & 0xFFFF0000u))));
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const int e = q_row_exponent(m);
        if (g < GP) {
          uint2 p1, p2, p3;
          q_pieces8(qx[i], pow2i(e), p1, p2, p3);
          const uint32_t off = (uint32_t)(cc & 1) * 8;
          *reinterpret_cast<uint2*>(qs + sw128_offset(g, cc >> 1) + off) = p1;
          *reinterpret_cast<uint2*>(qs + sw128_offset(GP + g, cc >> 1) + off) = p2;
          *reinterpret_cast<uint2*>(qs + sw128_offset(2 * GP + g, cc >> 1) + off) = p3;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&q_full[qb]);
      if (ahead.next(p)) {
#pragma unroll
        for (int i = 0; i < 8; ++i) qx[i] = decode_q_chunk_load(p, G, ahead.cur.kvh, ahead.cur.b, lane + 32 * i);
      }
      for (int l = 0; l < it.cur.n; ++l, ++j) {
        const int st = j % NCS_V;
        // Stage st last held tile j - NCS_V: PV(j - NCS_V) completing frees it (one phase pending, as
        // for K: NS > NCS_V).  The copy completes on p_full(j), whose previous phase (tile j - NS)
        // has completed: PV(j - NS) was issued before PV(j - NCS_V) completed.
        if (j >= NCS_V && !(ok = mbar_wait_warp(&pv_done[(j - NCS_V) % NS], ((j - NCS_V) / NS) & 1, SITE_DC_LOAD_EMPTY)))
          break;
        uint8_t* dst = smem + C::OFF_VCODE + st * C::CODE_TILE;
        const int tok0 = it.cur.t0 + l * 128;
        const int pg = vpc.get(p, it.cur.b, tok0), off = vpc.offset(p, tok0);
        {
          // The tile's k and v scales go into the scale stage with the codes, so the softmax reads
          // them from shared memory (no global load, no page lookup on its path).  Tokens past the
          // split (or on an invalid page) get 0, which their masked scores never use.
          const long long base = ((long long)(pg >= 0 ? pg : 0) * p.page_size + off) * p.Hkv + it.cur.kvh;
          float* sdst = scales + st * 256;
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const int i = lane + 32 * m, tk = i & 127;
            const bool in = pg >= 0 && tok0 + tk < it.cur.t1;
            const float* src = (i < 128 ? p.k_scale : p.v_scale) + (in ? base + (long long)tk * p.Hkv : 0);
            cp_async_4_zfill(sdst + i, src, in ? 4u : 0u);
          }
          cp_async_mbar_arrive(&sc_full[st]);
          __syncwarp();
          if (lane == 0) mbar_arrive(&sc_full[st]);
        }
        if (tok0 + 128 <= it.cur.t1) {
          if (lane == 0) {
            mbar_arrive_expect_tx(&p_full[j % NS], C::CODE_TILE);
            ATTN_EVT(j, 8);
            tma_load_4d(dst, &tmV, &p_full[j % NS], 0, it.cur.kvh, off, pg);
          }
        } else {
          // The split's last, partial tile: the PV MMA reads the codes as they are, and cache
          // slots past the length may hold anything (NaN codes included), so the tile comes in
          // through zero-filling 16-byte copies laid out like the TMA's 128-byte swizzle.
          // (an invalid page, already reported, reads nothing: every row is zero-filled)
          const int nvalid = pg >= 0 ? it.cur.t1 - tok0 : 0;
          const uint8_t* src = reinterpret_cast<const uint8_t*>(p.v_codes) +
                               (((long long)(pg >= 0 ? pg : 0) * p.page_size + off) * p.Hkv + it.cur.kvh) * 128;
#pragma unroll 4
          for (int i = 0; i < 32; ++i) {
            const int c = lane + 32 * i, r = c >> 3, ch = c & 7;
            const bool in = r < nvalid;
            cp_async_16_zfill(dst + r * 128 + ((ch ^ (r & 7)) << 4), src + (in ? (long long)r * p.Hkv * 128 + ch * 16 : 0),
                              in ? 16u : 0u);
          }
          cp_async_mbar_arrive(&p_full[j % NS]);
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[j % NS]);
        }
      }
      ++ie;
    }
    // On an error the copies in flight may land on barriers whose phase never completes (the
    // softmax gave up); the bounded drain then waits out the time limit, far longer than a copy.
    if (lane == 0 && !ok)
      for (int jj = (j > NCS_V ? j - NCS_V : 0); jj < j; ++jj)
        mbar_wait_drain(&p_full[jj % NS], (jj / NS) & 1, SITE_DC_DRAIN);
    if (!ok) asm volatile("cp.async.wait_all;" ::: "memory");
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ S issuer
    // S(j) needs K(j) landed, the item's Q pieces, and S^T / P^T buffer j % NS released by the
    // softmax (s_free, after it read S(j - NS)).  It runs ahead of the softmax by up to NS tiles, so
    // the K stages it frees go straight back to the producer.  An item's Q buffer is released
    // (q_free) by the commit after its last S.
    if (lane == 0) {
      constexpr uint32_t idesc_s = make_idesc_e4m3(128, NQ);  // A = K codes (K-major)
      const uint32_t sK = smem_u32(smem + C::OFF_KCODE);
      const uint32_t sQ = smem_u32(smem + C::OFF_Q);
      DecodeItemIter its(p);
      bool s_more = its.next(p);
      int js = 0, ls = 0, ies = 0;  // next S: CTA tile, tile within its item, item number
      bool ok = true;
      while (ok && s_more) {
        const int st = js % NCS_K, bs = js % NS, qb = ies & 1;
        ok = mbar_wait(&k_full[st], (js / NCS_K) & 1, SITE_DC_MMA_K) &&
             (ls > 0 || mbar_wait(&q_full[qb], (ies >> 1) & 1, SITE_DC_Q)) &&
             (js < NS || mbar_wait(&s_free[bs], ((js / NS) & 1) ^ 1, SITE_DC_MMA_S));
        if (!ok) break;
        ATTN_EVT(js, 3);
        tc_fence_after();
        // S^T(js) [128 x NQ] = K codes_js . Q pieces^T (4 steps of 32 codes)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f8_ss(tS0 + bs * NQ, make_sdesc_sw128(sK + st * C::CODE_TILE + kk * 32, 16, 1024),
                    make_sdesc_sw128(sQ + qb * C::Q_BYTES + kk * 32, 16, 1024), idesc_s, kk > 0);
        mma_commit(&s_full[bs]);
        ATTN_EVT(js, 10);
        if (++ls == its.cur.n) {
          mma_commit(&q_free[qb]);
          ls = 0;
          ++ies;
          s_more = its.next(p);
        }
        ++js;
      }
      mma_commit(drain);
      mbar_wait_drain(drain, 0, SITE_DC_DRAIN);
    }
    __syncwarp();
  } else if (warp == 7) {
    // ------------------------------------------------------------------ PV issuer
    // PV(j) needs P^T(j) and V(j) (both on p_full) and, for an item's first tile, the O^T buffer
    // released by the epilogue two items back.
    if (lane == 0) {
      constexpr uint32_t idesc_pv = make_idesc_e4m3(128, NP, true);  // A = V^T codes (MN-major)
      const uint32_t sV = smem_u32(smem + C::OFF_VCODE);
      const uint32_t sP = smem_u32(smem + C::OFF_P);
      DecodeItemIter itp(p);
      bool p_more = itp.next(p);
      int jp = 0, lp = 0, iep = 0;  // next PV: CTA tile, tile within its item, item number
      bool ok = true;
      while (ok && p_more) {
        const int st = jp % NCS_V, bp = jp % NS, ob = iep & 1;
        ok = mbar_wait(&p_full[bp], (jp / NS) & 1, SITE_DC_MMA_P) &&
             (lp > 0 || mbar_wait(&o_free[ob], ((iep >> 1) & 1) ^ 1, SITE_DC_MMA_O));
        if (!ok) break;
        ATTN_EVT(jp, 6);
        // a partial tile's codes came through generic-proxy copies: order them before the MMA reads
        if (itp.cur.t0 + (lp + 1) * 128 > itp.cur.t1) fence_proxy_async_smem();
        tc_fence_after();
        // O^T(item) [128 x NP] += V codes_jp^T . P pieces_jp^T (4 steps of 32 tokens)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f8_ss(tO0 + ob * NP, make_sdesc_sw128(sV + st * C::CODE_TILE + kk * 32 * 128, 16384, 1024),
                    make_sdesc_sw128(sP + bp * C::P_BYTES + kk * 32, 16, 1024), idesc_pv, (lp > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&pv_done[bp]);
        ATTN_EVT(jp, 11);
        if (++lp == itp.cur.n) {
          mma_commit(&o_full[ob]);
          lp = 0;
          ++iep;
          p_more = itp.next(p);
        }
        ++jp;
      }
      mma_commit(drain_pv);
      mbar_wait_drain(drain_pv, 0, SITE_DC_DRAIN);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax warpgroup
    const int wq = warp & 3;
    const int t = wq * 32 + lane;  // token of the tile / TMEM lane / output element d
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const int wg_tid = threadIdx.x - 96;  // warps 3..6
    const int n_items = p.n_splits * p.Hkv * p.B;
    // The row exponents e are recomputed here (the same function of the same bf16 query as the Q
    // stager's): thread wg_tid takes elements 16 (wg_tid % 8) .. + 15 of row wg_tid / 8, loaded
    // one item ahead, and the row maxima meet in shared memory.
    const int erow = wg_tid >> 3, epart = wg_tid & 7;
    auto load_q16 = [&](const DecodeItem& it, uint4& a, uint4& b) {
      a = decode_q_chunk_load(p, G, it.kvh, it.b, erow * 16 + 2 * epart);
      b = decode_q_chunk_load(p, G, it.kvh, it.b, erow * 16 + 2 * epart + 1);
    };
    DecodeItem cur;
    cur.n = 0;
    int w = blockIdx.x;
    if (w < n_items) cur = decode_item(p, w);
    uint4 qa = make_uint4(0u, 0u, 0u, 0u), qb = qa;
    if (w < n_items && cur.n > 0) load_q16(cur, qa, qb);
    int j = 0, ie = 0;  // tiles and non-empty items processed by this CTA
    bool ok = true;
    for (; w < n_items && ok; w += gridDim.x) {
      DecodeItem nxt;
      nxt.n = 0;
      if (w + (int)gridDim.x < n_items) nxt = decode_item(p, w + gridDim.x);
      if (cur.n == 0) {
        decode_write_empty(p, G, cur.split, cur.kvh, cur.b, wg_tid, 128);
        if (nxt.n > 0) load_q16(nxt, qa, qb);
        cur = nxt;
        continue;
      }
      {
        const uint32_t xw[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
        float m = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          m = fmaxf(m, fmaxf(fabsf(__uint_as_float(xw[k] << 16)), fabsf(__uint_as_float(xw[k] & 0xFFFF0000u))));
#pragma unroll
        for (int o = 4; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (epart == 0) q_exp[(ie & 1) * 16 + erow] = q_row_exponent(m);
      }
      mbar_arrive(exp_bar);
      if (!(ok = mbar_wait_warp(exp_bar, ie & 1, SITE_DC_Q))) break;
      float fq[GP];  // 2^-e per query row
#pragma unroll
      for (int g = 0; g < GP; ++g) fq[g] = pow2i(-q_exp[(ie & 1) * 16 + g]);
      if (nxt.n > 0) load_q16(nxt, qa, qb);
      DecodeRows<GP> rows;
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        rows.m_used[g] = -INFINITY;
        rows.l_part[g] = 0.f;
      }
      const uint32_t tO = tO0 + (ie & 1) * NP + lane_off;
      int rlim[GP];  // per-row exclusive key limits (a query token sees its own causal prefix)
#pragma unroll
      for (int g = 0; g < GP; ++g) rlim[g] = g < decode_rows(p) ? decode_row_limit(p, cur.len, cur.t1, g) : cur.t1;
      for (int l = 0; l < cur.n; ++l, ++j) {
        const int bs = j % NS;
        const int tok = cur.t0 + l * 128 + t;
        // scales of tile j: staged with V(j); the V producer refills the stage only after PV(j),
        // i.e. after this tile's P, so one phase is pending
        const int sst = j % NCS_V;
        if (!(ok = mbar_wait_warp(&sc_full[sst], (j / NCS_V) & 1, SITE_DC_SM_V))) break;
        const float ks = scales[sst * 256 + t], vs = scales[sst * 256 + 128 + t];
        if (!(ok = mbar_wait_warp(&s_full[bs], (j / NS) & 1, SITE_DC_SM_S))) break;
        if (t == 0) ATTN_EVT(j, 4);
        tc_fence_after();
        if (!(ok = fp8_softmax_tile<GP, NQ, NP, NS, MULTI>(rows, j, l > 0, lane, wq, t, tok, cur.t1, rlim,
                                                           p.scale_log2 * ks, vs, fq,
                                                    tS0 + bs * NQ + lane_off, tO, red_max, red_bar, s_free, pv_done,
                                                    smem + C::OFF_P + bs * C::P_BYTES, C::RESCALE_THRESHOLD)))
          break;
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&p_full[bs]);
        if (t == 0) ATTN_EVT(j, 5);
      }
      if (!ok) break;
      ok = fp8_epilogue<GP, NP, MULTI>(rows, p, G, cur.split, cur.kvh, cur.b, lane, wq, t, tO, red_sum, sum_bar, ie & 1,
                                &o_full[ie & 1], (ie >> 1) & 1, &o_free[ie & 1]);
      ++ie;
      cur = nxt;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace attn
