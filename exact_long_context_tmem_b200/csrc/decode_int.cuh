// Split-KV GQA decode over an INT8 or INT4 KV cache (ORT CPU GQA analysis: the KV cache is held
// as INT8 / INT4 codes and V is dequantised on the fly inside the SV accumulation; "Flash
// Decoding": the key range is split and the partial softmax states are merged by log-sum-exp).
//
// Codes: INT8 is one two's complement byte per element; INT4 is two 4-bit two's complement
// elements per byte, element 2i in the low nibble of byte i (a 128-element row is 64 bytes).  Each
// (token, KV head) has one float32 scale for K and one for V; value = code * scale.
//
// The dequantisation is fused into the tile load, and the scales stay out of the operands: k_scale
// multiplies the token's score and v_scale its probability, on the thread that owns the token.
// TMA brings the raw code tiles into shared memory.
//  * Scores, INT8: the K code tile is, as it lands, the K-major A operand of an integer MMA
//    (kind::i8, int32 accumulation) against Q as three signed 8-bit digits per element: the row
//    scaled by 2^e (absmax in [2^21, 2^22)) and rounded, q = 65536 d0 + 256 d1 + d2; the softmax
//    recombines the three digit columns exactly, so the score is (K . q) 2^-e with no conversion of
//    K at all.
//  * Scores, INT4: converter warps widen K to f16 (exact) straight into TMEM, the A operand of
//    S^T = K . Q^T, against Q as one f16 row per head scaled by 2^e (absmax in [2^14, 2^15)).
//  * Values (both): converter warps widen V to f16 in shared memory, the MN-major A operand of
//    O^T += V^T . P^T.  The running max is taken over y = x + log2(v_scale) (x the log2-domain score),
// so the probability that enters P, 2^(y - m) = 2^(x - m) * v_scale, stays below 2^threshold
// whatever the scale; the row sum l adds 2^(x - m) = P / v_scale.
//
// Roles (512 threads, one CTA per (split, KV head, sequence)):
//   warp 0       TMA producer of the raw K code tiles (NCS-stage ring)
//   warp 14      TMA producer of the raw V code tiles (NCS-stage ring)
//   warp 1       TMEM allocator; lane 0 issues the S MMAs
//   warp 15      lane 0 issues the PV MMAs
//   warps 2..5   K converter (INT4): thread = token; codes -> f16 into TMEM
//   warps 6..9   V converter: thread = token; codes -> f16 in shared memory (MN-major operand)
//   warps 10..13 Q staging, softmax, epilogue: thread = token (later = output element d)
// Issuing a tcgen05.mma costs its thread tens of cycles, so the S and PV chains (8 MMAs each per
// tile) go to two threads, ordered only through barriers: S(j+NB) waits until the softmax has read
// S(j) (s_free), and the softmax writes P(j+NB) once PV(j) has completed.  The softmax takes two
// tiles per step; scores, probabilities and converted K rotate through NB = 4 buffers, converted V
// through NV (4 for INT4, 3 for INT8).  TMEM columns: S^T [0, 64) (16-column buffers), O^T
// [64, 80), converted K [128, 384) (64-column buffers, 128 f16 per lane).
#pragma once

#include "decode.cuh"

namespace attn {

template <int BITS>
struct DecodeIntCfg {
  static constexpr int D = 128;
  static constexpr int ROW = BITS == 8 ? 128 : 64;  // code bytes per token row
  static constexpr int NCS = 3;                     // stages of raw code tiles
  // The softmax runs over two tiles per step (one maxima exchange and rescale decision per 256
  // tokens, up to eight query rows per KV head); S^T, P^T and converted K then rotate in fours.
  // Converted V tiles (32 KB each) get four buffers for INT4 and three for INT8, whose raw code
  // stages take twice the shared memory.
  static constexpr int STEP = 2;
  static constexpr int NB = 4;                      // S / P / converted-K buffers
  static constexpr int NV = BITS == 4 ? 4 : 3;      // converted-V buffers
  static constexpr int CODE_TILE = 128 * ROW;
  static constexpr int VC_TILE = 2 * 128 * 128;     // 128 tokens x 128 f16, two 64-wide boxes
  static constexpr int QBOX = 16 * 128;             // 16 rows x 64 f16
  // INT8: the score MMA takes the K codes as TMA lands them (kind::i8) against Q as three signed
  // 8-bit digits per element (up to 48 rows of 128 bytes); INT4: Q as f16 rows (two boxes).
  static constexpr bool K_I8 = BITS == 8;
  static constexpr int Q_BYTES = K_I8 ? 48 * 128 : 2 * QBOX;
  static constexpr int PBOX = 16 * 128;
  static constexpr int P_BYTES = 2 * PBOX;
  static constexpr int OFF_KCODE = 0;
  static constexpr int OFF_VCODE = OFF_KCODE + NCS * CODE_TILE;
  static constexpr int OFF_VC = OFF_VCODE + NCS * CODE_TILE;
  static constexpr int OFF_Q = OFF_VC + NV * VC_TILE;
  static constexpr int OFF_P = OFF_Q + Q_BYTES;
  static constexpr int OFF_RED = OFF_P + NB * P_BYTES;
  static constexpr int OFF_QSC = OFF_RED + (2 * 4 * 16 + 4 * 16) * 4;  // [16] 2^-e per query row
  static constexpr int OFF_BAR = OFF_QSC + 16 * 4;
  static constexpr int N_BARS = 4 * NCS + 1 + 6 * NB + 2 * NV + 2 + 2 + 1 + 1;
  static constexpr int SMEM_BYTES = OFF_BAR + N_BARS * 8 + 16 + 1024;
  static constexpr int THREADS = 512;
  static constexpr uint32_t TMEM_COLS = 512;
  // S^T from column 0 (NB buffers of 16 columns, or for INT8 of 16 / 32 / 48: three digit columns
  // per query row), O^T at 64 (INT4) or 256 (INT8), converted K (INT4) from 128.
  static constexpr uint32_t COL_S = 0, COL_O = K_I8 ? 256 : NB * 16, COL_K = 128;
  static_assert(K_I8 ? NB * 48 <= (int)COL_O : (COL_O + 16 <= COL_K && COL_K + NB * 64 <= TMEM_COLS), "TMEM columns");
  static constexpr float RESCALE_THRESHOLD = 8.0f;
};
static_assert(DecodeIntCfg<8>::SMEM_BYTES <= 227 * 1024, "shared memory per CTA");
static_assert(DecodeIntCfg<4>::SMEM_BYTES <= 227 * 1024, "shared memory per CTA");
static_assert(DecodeIntCfg<8>::OFF_VCODE % 1024 == 0 && DecodeIntCfg<4>::OFF_VCODE % 1024 == 0, "TMA tile alignment");

// Byte offset of 16-byte chunk c of token row t in a TMA code tile: 128-byte rows with the 128B
// swizzle (INT8), 64-byte rows with the 64B swizzle (INT4: chunk c ^ bits 7..8 of the address).
template <int BITS>
__device__ __forceinline__ uint32_t int_code_offset(uint32_t t, uint32_t c) {
  if (BITS == 8) return sw128_offset(t, c);
  return t * 64u + ((c ^ ((t >> 1) & 3u)) << 4);
}

__device__ __forceinline__ uint32_t sub_f16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Four INT8 codes -> f16 pairs (elements 0,1) and (2,3), exact: code + 128 becomes the low 8
// mantissa bits of an f16 in [1024, 2048), whose unit in the last place is 1; 1152 is subtracted.
__device__ __forceinline__ void i8x4_to_f16(uint32_t w, uint32_t& h01, uint32_t& h23) {
  const uint32_t u = w ^ 0x80808080u;
  h01 = sub_f16x2(__byte_perm(u, 0x64646464u, 0x5150u), 0x64806480u);
  h23 = sub_f16x2(__byte_perm(u, 0x64646464u, 0x5352u), 0x64806480u);
}

// INT8 scores on the tensor core: S^T = K codes . Q digits^T with int32 accumulation (kind::i8,
// K = 32 per instruction).  Instruction descriptor: s32 accumulator (format 2 at bit 4), A and B
// signed 8-bit (format 1 at bits 7 and 10), both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t make_idesc_s8(int M, int N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_s8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// S^T columns per buffer for a group padded to GP rows: 16, or for INT8 3 GP digit columns
// rounded up to 16.
template <int GP, int BITS>
__host__ __device__ constexpr int int_score_cols() {
  return BITS == 8 ? ((3 * GP + 15) / 16) * 16 : 16;
}

// N consecutive TMEM columns of this warp's lanes (N = 16, 32 or 48), waited for.
template <int N>
__device__ __forceinline__ void int_tmem_ld(uint32_t taddr, uint32_t (&v)[N]) {
  static_assert(N == 16 || N == 32 || N == 48, "column count");
  if constexpr (N == 16) {
    tmem_ld16(taddr, v);
    tmem_wait_ld_regs(v);
  } else if constexpr (N == 32) {
    tmem_ld32(taddr, v);
    tmem_wait_ld_regs(v);
  } else {
    uint32_t a[32], b[16];
    tmem_ld32(taddr, a);
    tmem_ld16(taddr + 32, b);
    tmem_wait_ld_regs(a);
    tmem_wait_ld_regs(b);
#pragma unroll
    for (int c = 0; c < 32; ++c) v[c] = a[c];
#pragma unroll
    for (int c = 0; c < 16; ++c) v[32 + c] = b[c];
  }
}

__device__ __forceinline__ uint32_t lop3_and_xor(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(b), "r"(c));  // (a & b) ^ c
  return d;
}
__device__ __forceinline__ uint32_t fma_f16x2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Eight INT4 codes (one word; element k in nibble k) -> four f16 pairs (0,4), (1,5), (2,6), (3,7),
// exact, in five integer instructions: one lop3 per pair puts code + 8 (the nibble with its top bit
// flipped) into the mantissa of an f16 in [1024, 1040) (low nibbles) or, at 16x, in [1024, 1264)
// (high nibbles), which a subtraction or an fma by 1/16 takes back to the code.  The pairing is not
// element order: a kernel using it permutes the other operand of each product the same way.
__device__ __forceinline__ void i4x8_to_f16_paired(uint32_t w, uint32_t* h) {
  const uint32_t w8 = w >> 8;
  h[0] = sub_f16x2(lop3_and_xor(w, 0x000F000Fu, 0x64086408u), 0x64086408u);                // 0, 4
  h[1] = fma_f16x2(lop3_and_xor(w, 0x00F000F0u, 0x64806480u), 0x2C002C00u, 0xD480D480u);   // 1, 5
  h[2] = sub_f16x2(lop3_and_xor(w8, 0x000F000Fu, 0x64086408u), 0x64086408u);               // 2, 6
  h[3] = fma_f16x2(lop3_and_xor(w8, 0x00F000F0u, 0x64806480u), 0x2C002C00u, 0xD480D480u);  // 3, 7
}

// Position within each group of eight head-dimension elements of the INT4 path: the f16 pair at
// positions (2i, 2i+1) holds elements (i, i + 4).  Element of position q: (q >> 1) + 4 (q & 1).
__device__ __forceinline__ int int4_paired_element(int q) { return (q & ~7) | (((q & 7) >> 1) + 4 * (q & 1)); }

// Elements [64 half, 64 half + 64) of token row t of a code tile as 32 f16 pairs (zeros when the
// token is not valid); INT4 rows come out in the paired order of i4x8_to_f16_paired.
template <int BITS>
__device__ __forceinline__ void int_row_half_to_f16(const uint8_t* tile, int t, int half, bool valid,
                                                    uint32_t (&h)[32]) {
  constexpr int CH = BITS == 8 ? 4 : 2;  // 16-byte code chunks per 64 elements
#pragma unroll
  for (int k = 0; k < CH; ++k) {
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (valid) w = *reinterpret_cast<const uint4*>(tile + int_code_offset<BITS>(t, half * CH + k));
    const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (BITS == 8) i8x4_to_f16(wd[i], h[k * 8 + 2 * i], h[k * 8 + 2 * i + 1]);
      else i4x8_to_f16_paired(wd[i], &h[k * 16 + 4 * i]);
    }
  }
}

// One arrival per warp: every lane's prior writes (and the fences each lane issued) are ordered
// before lane 0's release-arrive by the warp barrier.  Barriers fed this way count warps, which
// keeps the same-address shared-memory atomics at one per warp instead of one per thread.
__device__ __forceinline__ void warp_arrive(uint64_t* bar, int lane) {
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
}

// Index of the (token, KV head) scale of sequence b's token tok, or -1 for an unmapped page.
__device__ __forceinline__ long long int_scale_index(const DecodeParams& p, int b, int tok, int kvh) {
  long long page = b;
  int off = tok;
  if (p.page_table) {
    const int raw = __ldg(p.page_table + (long long)b * p.max_pages + tok / p.page_size);
    if (raw < 0 || raw >= p.num_pages) return -1;
    page = raw;
    off = tok % p.page_size;
  }
  return (page * p.page_size + off) * p.Hkv + kvh;
}

// Query rows of the group, staged as the B operand of the score MMA; 2^-e of row g goes to qsc[g].
// 128 threads: chunk c = tid + 128 k is row c / 16, elements 8 (c % 16).., so the 16 threads of a
// row are 16 consecutive lanes of one warp, which find the row's absmax together.
//  INT4: f16 rows scaled by 2^e (absmax in [2^14, 2^15); every bf16 element within 2^31 of it is
//    then exact) into the 128B-swizzled K-major operand (two 64-wide boxes of 16 rows), elements in
//    the paired order of the widened K rows.
//  INT8: integers q = rn(x 2^e) with the absmax in [2^21, 2^22) (exact for every element within
//    2^14 of it), written as three balanced signed 8-bit digits q = 65536 d0 + 256 d1 + d2
//    (|d0| <= 64): digit k of row g is operand row k GP + g, one 128-byte row of 128 elements.
//  e is clamped to [-100, 100].
template <int BITS, int GP>
__device__ __forceinline__ void int_stage_q(const DecodeParams& p, int G, int kvh, int b, int tid, uint8_t* q_smem,
                                            float* qsc) {
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int c = tid + 128 * k;
    const int g = c >> 4, cc = c & 15;
    const uint4 x = decode_q_chunk_load(p, G, kvh, b, c);
    const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
    float f[8];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(xw[i] << 16);
      f[2 * i + 1] = __uint_as_float(xw[i] & 0xFFFF0000u);
      amax = fmaxf(amax, fmaxf(fabsf(f[2 * i]), fabsf(f[2 * i + 1])));
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    int e = (BITS == 8 ? 21 : 14) - ((int)((__float_as_uint(amax) >> 23) & 0xFFu) - 127);
    e = e < -100 ? -100 : (e > 100 ? 100 : e);
    const float up = __uint_as_float((uint32_t)(e + 127) << 23);
    if constexpr (BITS == 8) {
      uint32_t dw[3][2] = {{0u, 0u}, {0u, 0u}, {0u, 0u}};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int q = __float2int_rn(f[i] * up);
        const int d2 = ((q + 128) & 255) - 128;
        const int r = (q - d2) >> 8;
        const int d1 = ((r + 128) & 255) - 128;
        const int d0 = (r - d1) >> 8;
        const int sh = 8 * (i & 3);
        dw[0][i >> 2] |= ((uint32_t)d0 & 0xFFu) << sh;
        dw[1][i >> 2] |= ((uint32_t)d1 & 0xFFu) << sh;
        dw[2][i >> 2] |= ((uint32_t)d2 & 0xFFu) << sh;
      }
      if (g < GP) {
#pragma unroll
        for (int dk = 0; dk < 3; ++dk) {
          const uint32_t row = (uint32_t)(dk * GP + g);
          *reinterpret_cast<uint2*>(q_smem + row * 128u + ((((uint32_t)cc >> 1) ^ (row & 7u)) << 4) +
                                    ((uint32_t)cc & 1u) * 8u) = make_uint2(dw[dk][0], dw[dk][1]);
        }
      }
    } else {
      uint32_t hv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) hv[i] = pack_f16x2(f[i] * up, f[i + 4] * up);  // the paired order of the K rows
      *reinterpret_cast<uint4*>(q_smem + (cc >> 3) * (16 * 128) + sw128_offset(g, cc & 7)) =
          make_uint4(hv[0], hv[1], hv[2], hv[3]);
    }
    if (cc == 0) qsc[g] = __uint_as_float((uint32_t)(127 - e) << 23);
  }
}

// One softmax step over NT tiles (one or, for INT4, two) on the thread that owns token t of each,
// with the running max over y = x + log2(v_scale): row maxima over the step's tokens (warp redux,
// then the cross-warp exchange number e) -> lazy O rescale -> this thread's entries of each tile's
// P^T (2^(y - m), f16).  nt (warp-uniform) is how many of the NT tiles exist (the last step of an
// odd tile count has one).  Returns false, warp-uniformly, if a bounded wait ran out.  The S^T of
// every tile is read first and its s_free arrived on at once, so the next S into the same buffer
// can be issued; a P^T buffer is written only after p_reuse (the PV that last read it, if any) has
// completed.
template <int GP, int NT, int BITS>
__device__ __forceinline__ bool int_softmax_step(DecodeRows<GP>& rows, int e, int j, int nt, int lane, int wq, int t,
                                                 const bool (&valid)[NT], const float (&scq)[GP], const float (&ks)[NT],
                                                 const float (&vs)[NT], const uint32_t (&tS_lane)[NT],
                                                 uint64_t* const (&s_free)[NT], uint32_t tO_lane, float* red_max,
                                                 uint64_t* red_bar, uint64_t* prev_pv, uint32_t prev_pv_parity,
                                                 uint64_t* const (&p_reuse)[NT], const uint32_t (&p_reuse_parity)[NT],
                                                 uint8_t* const (&p_tile)[NT], float threshold,
                                                 long long* evt_base_ = nullptr) {
  constexpr int SC = int_score_cols<GP, BITS>();
  uint32_t sv[NT][SC];
  if constexpr (SC == 16) {
#pragma unroll
    for (int k = 0; k < NT; ++k)
      if (k < nt) tmem_ld16(tS_lane[k], sv[k]);
#pragma unroll
    for (int k = 0; k < NT; ++k)
      if (k < nt) tmem_wait_ld_regs(sv[k]);
  } else {
#pragma unroll
    for (int k = 0; k < NT; ++k)
      if (k < nt) int_tmem_ld<SC>(tS_lane[k], sv[k]);
  }
  if (t == 0) ATTN_EVT(j, 10);
  if (lane == 0 && j < 31) ATTN_EVT(32 + j, 4 + wq);
  tc_fence_before();
#pragma unroll
  for (int k = 0; k < NT; ++k)
    if (k < nt) warp_arrive(s_free[k], lane);
  float lvs[NT], ivs[NT];
  bool neg[NT];
  float y[NT][GP];
#pragma unroll
  for (int k = 0; k < NT; ++k) {
    const float avs = fminf(fmaxf(fabsf(vs[k]), 0x1p-100f), 0x1p100f);
    lvs[k] = __log2f(avs);
    ivs[k] = __fdividef(1.f, avs);
    neg[k] = vs[k] < 0.f;
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      float raw;  // Q.K of row g in units of 2^-e
      if constexpr (BITS == 8)  // digits: 65536 S0 + (256 S1 + S2), each partial an exact int32
        raw = fmaf((float)(int)sv[k][g], 65536.f, (float)((int)sv[k][GP + g] * 256 + (int)sv[k][2 * GP + g]));
      else
        raw = __uint_as_float(sv[k][g]);
      y[k][g] = (k < nt && valid[k]) ? fmaf(raw * scq[g], ks[k], lvs[k]) : -INFINITY;
    }
  }
  float* rm = red_max + (e & 1) * 64;
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    float ym = y[0][g];
#pragma unroll
    for (int k = 1; k < NT; ++k) ym = fmaxf(ym, y[k][g]);
    const float m = warp_max_redux(ym);
    if (lane == 0) rm[wq * 16 + g] = m;
  }
  if (lane == 0 && j < 31) ATTN_EVT(32 + j, wq);
  warp_arrive(&red_bar[e & 1], lane);  // lane 0 wrote this warp's maxima
  if (!mbar_wait_warp(&red_bar[e & 1], (e >> 1) & 1, SITE_DC_SM_S)) return false;
  if (t == 0) ATTN_EVT(j, 11);
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
  if (need && j > 0) {  // rescale O^T row t once the previous PV is done
    if (t == 0) ATTN_EVT(j, 14);
    if (!mbar_wait_warp(prev_pv, prev_pv_parity, SITE_DC_SM_O)) return false;
    tc_fence_after();
    uint32_t orow[16];
    tmem_ld16(tO_lane, orow);
    tmem_wait_ld_regs(orow);
#pragma unroll
    for (int g = 0; g < GP; ++g) orow[g] = __float_as_uint(__uint_as_float(orow[g]) * alpha[g]);
    tmem_st16(tO_lane, orow);
    tmem_wait_st();
  }
#pragma unroll
  for (int k = 0; k < NT; ++k)
    if (k < nt && p_reuse[k] && !mbar_wait_warp(p_reuse[k], p_reuse_parity[k], SITE_DC_SM_P)) return false;
  if (t == 0) ATTN_EVT(j, 12);
  const uint32_t pchunk = (t & 63) >> 3, pbyte = (t & 7) * 2;
#pragma unroll
  for (int k = 0; k < NT; ++k) {
    if (k >= nt) break;
    uint8_t* prow = p_tile[k] + (t >> 6) * (16 * 128);
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      const float pe = (y[k][g] == -INFINITY) ? 0.f : ex2_approx(y[k][g] - rows.m_used[g]);
      rows.l_part[g] += pe * ivs[k];
      *reinterpret_cast<uint16_t*>(prow + sw128_offset(g, pchunk) + pbyte) =
          __half_as_ushort(__float2half_rn(neg[k] ? -pe : pe));
    }
  }
  return true;
}

template <int GP, int BITS>
__global__ void __launch_bounds__(512, 1)
    decode_int_sm100(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const DecodeParams p) {
  using C = DecodeIntCfg<BITS>;
  constexpr int NB = C::NB;
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
#ifdef ATTN_PROF
  // Event timeline of the grid's first CTA only (profile builds).
  long long* const evt_base_ = (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) ? g_evt : nullptr;
#endif
  ATTN_EVT(63, 0);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* k_full = bars;              // [NCS] raw K codes landed
  uint64_t* k_empty = k_full + C::NCS;  // [NCS] converter done with the raw K stage
  uint64_t* v_full = k_empty + C::NCS;
  uint64_t* v_empty = v_full + C::NCS;
  uint64_t* q_ready = v_empty + C::NCS;
  uint64_t* s_full = q_ready + 1;    // [NB] S^T(j) in TMEM
  uint64_t* p_full = s_full + NB;    // [NB] P^T(j) in shared memory
  uint64_t* pv_done = p_full + NB;   // [NB] PV(j) completed
  uint64_t* kc_full = pv_done + NB;  // [NB] converted K in TMEM
  uint64_t* kc_empty = kc_full + NB; // [NB] S MMA done reading it
  uint64_t* vc_full = kc_empty + NB;     // [NV] converted V in shared memory
  uint64_t* vc_empty = vc_full + C::NV;  // [NV] PV MMA done reading it
  uint64_t* s_free = vc_empty + C::NV;   // [NB] the softmax has read S^T(j)
  uint64_t* drain = s_free + NB;     // [2] each MMA issuer's own MMAs completed
  uint64_t* red_bar = drain + 2;     // [2]
  uint64_t* sum_bar = red_bar + 2;
  uint64_t* o_final = sum_bar + 1;  // single phase: every PV of the split has completed
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(o_final + 1);
  float* red_max = reinterpret_cast<float*>(smem + C::OFF_RED);  // [2][4][16]
  float* red_sum = red_max + 2 * 4 * 16;                         // [4][16]
  float* qsc = reinterpret_cast<float*>(smem + C::OFF_QSC);

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NCS; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], C::K_I8 ? 1 : 4);  // the S MMA's commit, or the K converter warps
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 4);
    }
    mbar_init(q_ready, 4);
    for (int s = 0; s < NB; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 4);
      mbar_init(&pv_done[s], 1);
      mbar_init(&kc_full[s], 4);
      mbar_init(&kc_empty[s], 1);
      mbar_init(&s_free[s], 4);
    }
    for (int s = 0; s < C::NV; ++s) {
      mbar_init(&vc_full[s], 4);
      mbar_init(&vc_empty[s], 1);
    }
    mbar_init(&red_bar[0], 4);
    mbar_init(&red_bar[1], 4);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
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
  const uint32_t tS0 = tmem + C::COL_S, tO = tmem + C::COL_O, tK0 = tmem + C::COL_K;

  if (warp == 0 || warp == 14) {
    // ------------------------------------------------------------------ TMA producers (K: warp 0, V: warp 14)
    if (lane == 0) {
      const bool is_k = warp == 0;
      const CUtensorMap* tm = is_k ? &tmK : &tmV;
      uint64_t* full = is_k ? k_full : v_full;
      uint64_t* empty = is_k ? k_empty : v_empty;
      uint8_t* ring = smem + (is_k ? C::OFF_KCODE : C::OFF_VCODE);
      tma_prefetch_desc(tm);
      PageCursor pc;
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < n; ++j) {
        const int st = j % C::NCS;
        if (!(ok = mbar_wait(&empty[st], ((j / C::NCS) & 1) ^ 1, SITE_DC_LOAD_EMPTY))) break;
        const int tok = t0 + j * 128;
        const int page = pc.get(p, b, tok);
        mbar_arrive_expect_tx(&full[st], C::CODE_TILE);
        tma_load_4d(ring + st * C::CODE_TILE, tm, &full[st], 0, kvh, pc.offset(p, tok), page);
        ATTN_EVT(j, is_k ? 0 : 1);
        issued = j + 1;
      }
      if (!ok)  // wait (bounded) for the copies still in flight before the CTA exits
        for (int j = (issued > C::NCS ? issued - C::NCS : 0); j < issued; ++j)
          mbar_wait_drain(&full[j % C::NCS], (j / C::NCS) & 1, SITE_DC_DRAIN);
    }
    __syncwarp();
  } else if (warp == 1 || warp == 15) {
    // ------------------------------------------------------------------ MMA issuers (S: warp 1, PV: warp 15)
    if (lane == 0) {
      bool ok = true;
      if (warp == 1 && C::K_I8) {
        // S^T(j) [128 x SC] = K codes_j (as TMA landed them) . Q digits^T, int32 (4 steps of 32
        // codes); the commit after it frees the raw K stage.
        constexpr int SC = int_score_cols<GP, BITS>();
        constexpr uint32_t idesc_qk = make_idesc_s8(128, SC);
        const uint32_t sQ = smem_u32(smem + C::OFF_Q), sK = smem_u32(smem + C::OFF_KCODE);
        ok = mbar_wait(q_ready, 0, SITE_DC_MMA_K);
        for (int j = 0; j < n && ok; ++j) {
          const int bj = j % NB, st = j % C::NCS;
          const uint32_t ph = (j / NB) & 1;
          if (!(ok = mbar_wait(&k_full[st], (j / C::NCS) & 1, SITE_DC_MMA_K))) break;
          if (j >= NB && !(ok = mbar_wait(&s_free[bj], ph ^ 1, SITE_DC_MMA_S))) break;  // S(j-NB) read
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_s8_ss(tS0 + bj * SC, make_sdesc_sw128(sK + st * C::CODE_TILE + kk * 32, 16, 1024),
                      make_sdesc_sw128(sQ + kk * 32, 16, 1024), idesc_qk, kk > 0);
          ATTN_EVT(j, 4);
          mma_commit(&s_full[bj]);
          mma_commit(&k_empty[st]);
        }
        mma_commit(&drain[0]);
        mbar_wait_drain(&drain[0], 0, SITE_DC_DRAIN);
      } else if (warp == 1) {
        // S^T(j) [128 x 16] = K_j (TMEM, f16) . Q^T
        constexpr uint32_t idesc_qk = make_idesc_f16(128, 16, false, false, false);
        const uint32_t sQ = smem_u32(smem + C::OFF_Q);
        ok = mbar_wait(q_ready, 0, SITE_DC_MMA_K);
        for (int j = 0; j < n && ok; ++j) {
          const int bj = j % NB;
          const uint32_t ph = (j / NB) & 1;
          if (!(ok = mbar_wait(&kc_full[bj], ph, SITE_DC_MMA_K))) break;
          if (j >= NB && !(ok = mbar_wait(&s_free[bj], ph ^ 1, SITE_DC_MMA_S))) break;  // S(j-NB) read
          tc_fence_after();
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t qoff = (kk >> 2) * C::QBOX + (kk & 3) * 32;
            mma_ts(tS0 + bj * 16, tK0 + bj * 64 + kk * 8, make_sdesc_sw128(sQ + qoff, 16, 1024), idesc_qk, kk > 0);
          }
          ATTN_EVT(j, 4);
          mma_commit(&s_full[bj]);
          mma_commit(&kc_empty[bj]);
        }
        mma_commit(&drain[0]);
        mbar_wait_drain(&drain[0], 0, SITE_DC_DRAIN);
      } else {
        // O^T += V_j^T . P_j^T
        constexpr uint32_t idesc_pv = make_idesc_f16(128, 16, true, false, false);
        const uint32_t sP = smem_u32(smem + C::OFF_P);
        const uint32_t sVc = smem_u32(smem + C::OFF_VC);
        for (int j = 0; j < n && ok; ++j) {
          const int bj = j % NB, bv = j % C::NV;
          const uint32_t ph = (j / NB) & 1, phv = (j / C::NV) & 1;
          ATTN_EVT(j, 8);
          if (!(ok = mbar_wait(&vc_full[bv], phv, SITE_DC_MMA_V))) break;
          ATTN_EVT(j, 9);
          if (!(ok = mbar_wait(&p_full[bj], ph, SITE_DC_MMA_P))) break;
          tc_fence_after();
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t da = make_sdesc_sw128(sVc + bv * C::VC_TILE + kk * 16 * 128, 128 * 128, 1024);
            const uint64_t db = make_sdesc_sw128(sP + bj * C::P_BYTES + (kk >> 2) * C::PBOX + (kk & 3) * 32, 16, 1024);
            mma_ss(tO, da, db, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
          }
          ATTN_EVT(j, 7);
          mma_commit(&pv_done[bj]);
          mma_commit(&vc_empty[bv]);
        }
        if (ok) mma_commit(o_final);
        mma_commit(&drain[1]);
        mbar_wait_drain(&drain[1], 0, SITE_DC_DRAIN);
      }
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------------ K converter warpgroup
    // (INT4 only: the INT8 score MMA reads the codes directly)
    const int wq = warp & 3;
    const int t = wq * 32 + lane;  // token row of the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    for (int j = 0; j < (C::K_I8 ? 0 : n); ++j) {
      const int st = j % C::NCS;
      const uint32_t ph = (j / C::NCS) & 1;
      const int bj = j % NB;
      const uint32_t phb = (j / NB) & 1;
      const bool valid = t0 + j * 128 + t < t1;
      if (!mbar_wait_warp(&k_full[st], ph, SITE_DC_SM_K)) break;
      if (!mbar_wait_warp(&kc_empty[bj], phb ^ 1, SITE_DC_SM_K)) break;  // S(j-NB) has read it
      tc_fence_after();
      const uint8_t* ktile = smem + C::OFF_KCODE + st * C::CODE_TILE;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t h[32];
        int_row_half_to_f16<BITS>(ktile, t, half, valid, h);
        tmem_st32(tK0 + bj * 64 + half * 32 + lane_off, h);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&k_empty[st]);
        mbar_arrive(&kc_full[bj]);
      }
      if (t == 0) ATTN_EVT(j, 2);
    }
  } else if (warp < 10) {
    // ------------------------------------------------------------------ V converter warpgroup
    const int t = (warp & 3) * 32 + lane;  // token row of the tile
    for (int j = 0; j < n; ++j) {
      const int st = j % C::NCS;
      const uint32_t ph = (j / C::NCS) & 1;
      const int bv = j % C::NV;
      const uint32_t phv = (j / C::NV) & 1;
      const bool valid = t0 + j * 128 + t < t1;
      if (!mbar_wait_warp(&v_full[st], ph, SITE_DC_SM_V)) break;
      if (!mbar_wait_warp(&vc_empty[bv], phv ^ 1, SITE_DC_SM_V)) break;  // PV(j-NV) has read it
      const uint8_t* vtile = smem + C::OFF_VCODE + st * C::CODE_TILE;
      uint8_t* vc = smem + C::OFF_VC + bv * C::VC_TILE;
#pragma unroll
      for (int half = 0; half < 2; ++half) {  // elements [64 half, +64) = box `half` of the operand
        uint32_t h[32];
        int_row_half_to_f16<BITS>(vtile, t, half, valid, h);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          *reinterpret_cast<uint4*>(vc + half * (128 * 128) + sw128_offset(t, k)) =
              make_uint4(h[4 * k], h[4 * k + 1], h[4 * k + 2], h[4 * k + 3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&v_empty[st]);
        mbar_arrive(&vc_full[bv]);
      }
      if (t == 0) ATTN_EVT(j, 3);
    }
  } else {
    // ------------------------------------------------------------------ softmax warpgroup
    const int wq = warp & 3;
    const int t = wq * 32 + lane;  // token of the tile / TMEM lane / output element d
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const int wg_tid = threadIdx.x - 320;
    for (int i = wg_tid; i < NB * C::P_BYTES / 16; i += 128)  // P^T rows >= GP stay zero
      reinterpret_cast<uint4*>(smem + C::OFF_P)[i] = make_uint4(0u, 0u, 0u, 0u);
    if constexpr (C::K_I8)  // operand rows past the 3 GP digit rows stay zero
      for (int i = 3 * GP * 128 / 16 + wg_tid; i < C::Q_BYTES / 16; i += 128)
        reinterpret_cast<uint4*>(smem + C::OFF_Q)[i] = make_uint4(0u, 0u, 0u, 0u);
    int_stage_q<BITS, GP>(p, G, kvh, b, wg_tid, smem + C::OFF_Q, qsc);
    fence_proxy_async_smem();
    warp_arrive(q_ready, lane);
    named_barrier_sync(1, 128);  // every row's 2^-e is in qsc
    if (t == 0) ATTN_EVT(63, 1);
    float scq[GP];
#pragma unroll
    for (int g = 0; g < GP; ++g) scq[g] = p.scale_log2 * qsc[g];

    DecodeRows<GP> rows;
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      rows.m_used[g] = -INFINITY;
      rows.l_part[g] = 0.f;
    }
    bool ok = true;
    // Per-token scales are loaded SPF tiles ahead into a register ring: under full HBM streaming a
    // plain global load takes longer than one tile, and the scores wait on k_scale.  An unmapped
    // page leaves them at 1 (its codes land as zeros).
    constexpr int SPF = 4;
    float ksr[SPF], vsr[SPF];
#pragma unroll
    for (int i = 0; i < SPF; ++i) {
      ksr[i] = 1.f;
      vsr[i] = 1.f;
      const int tk = t0 + i * 128 + t;
      if (tk < t1) {
        const long long x = int_scale_index(p, b, tk, kvh);
        if (x >= 0) {
          ksr[i] = __ldg(p.k_scale + x);
          vsr[i] = __ldg(p.v_scale + x);
        }
      }
    }
    // Groups whose tile scores fill 32 or more columns (16 rows; 8 rows of INT8 digits) keep a
    // one-tile step, so two tiles' scores need not be live at once.
    constexpr int ST = int_score_cols<GP, BITS>() * GP <= 128 && GP <= 8 ? C::STEP : 1;
    for (int j = 0; j < n && ok; j += ST) {
      const int nt = n - j < ST ? n - j : ST;  // tiles in this step (warp-uniform)
      bool valid[ST];
      float ks[ST], vs[ST];
      uint32_t tSl[ST], prp[ST];
      uint64_t* sfr[ST];
      uint64_t* prb[ST];
      uint8_t* ptl[ST];
#pragma unroll
      for (int k = 0; k < ST; ++k) {
        const int jk = j + k;
        const int bk = jk % NB;
        valid[k] = t0 + jk * 128 + t < t1;
        ks[k] = ksr[k];
        vs[k] = vsr[k];
        tSl[k] = tS0 + bk * int_score_cols<GP, BITS>() + lane_off;
        sfr[k] = &s_free[bk];
        // PV(i) is completion number i/NB of pv_done[i%NB]; PV(jk-NB), the last reader of P buffer
        // bk, is the oldest pending phase of its barrier (PV(jk) needs this step's P first).
        prb[k] = jk >= NB ? &pv_done[bk] : nullptr;
        prp[k] = ((uint32_t)(jk / NB) & 1) ^ 1;
        ptl[k] = smem + C::OFF_P + bk * C::P_BYTES;
      }
      // Per-token scales: the ring holds SPF tiles; this step consumes ST of them and refills the
      // same number SPF tiles ahead.
#pragma unroll
      for (int i = 0; i + ST < SPF; ++i) {
        ksr[i] = ksr[i + ST];
        vsr[i] = vsr[i + ST];
      }
#pragma unroll
      for (int k = 0; k < ST; ++k) {
        const int tk = t0 + (j + k + SPF) * 128 + t;
        ksr[SPF - ST + k] = 1.f;
        vsr[SPF - ST + k] = 1.f;
        if (tk < t1) {
          const long long x = int_scale_index(p, b, tk, kvh);
          if (x >= 0) {
            ksr[SPF - ST + k] = __ldg(p.k_scale + x);
            vsr[SPF - ST + k] = __ldg(p.v_scale + x);
          }
        }
      }
      if (t == 0) ATTN_EVT(j, 13);
      if (lane == 0 && j < 31) ATTN_EVT(32 + j, 8 + wq);
#pragma unroll
      for (int k = 0; k < ST; ++k)
        if (k < nt && !(ok = mbar_wait_warp(&s_full[(j + k) % NB], (uint32_t)((j + k) / NB) & 1, SITE_DC_SM_S))) break;
      if (!ok) break;
      if (t == 0) ATTN_EVT(j, 5);
      tc_fence_after();
      // PV(j-1) is the oldest pending phase of its barrier (PV(j-1+NB) needs a later P).
      const int jp = j > 0 ? j - 1 : 0;
      if (!(ok = int_softmax_step<GP, ST, BITS>(rows, j / ST, j, nt, lane, wq, t, valid, scq, ks, vs, tSl, sfr,
                                          tO + lane_off, red_max, red_bar, &pv_done[jp % NB],
                                          (uint32_t)(jp / NB) & 1, prb, prp, ptl, C::RESCALE_THRESHOLD
#ifdef ATTN_PROF
                                          , evt_base_
#endif
                                          )))
        break;
      fence_proxy_async_smem();
      tc_fence_before();
#pragma unroll
      for (int k = 0; k < ST; ++k)
        if (k < nt) warp_arrive(&p_full[(j + k) % NB], lane);
      if (t == 0) ATTN_EVT(j, 6);
      if (lane == 0 && j < 31) ATTN_EVT(32 + j, 12 + wq);
    }
    if (t == 0) ATTN_EVT(63, 2);
    if (ok)
      decode_epilogue<GP, false>(rows, p, G, split, kvh, b, lane, wq, t, tO + lane_off, red_sum, sum_bar, 0, o_final,
                                 0, nullptr, BITS == 4 ? int4_paired_element(t) : t);  // O^T lane t: V's paired order
    if (t == 0) ATTN_EVT(63, 3);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace attn
