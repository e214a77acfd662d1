// Split-KV GQA decode over an FP8 E4M3 KV cache (LLM-CoOpt summary, "Opt-KV": the cache is
// stored in FP8 to halve the bytes per token; ONNX Runtime CPU GQA analysis, "Flash Decoding":
// split the key range, merge the partial softmax states by log-sum-exp).
//
// Same arithmetic as the bf16 kernel (KV tokens on the MMA's M axis:
// S^T = K.Q^T and O^T += V^T.P^T), with the dequantisation fused into the tile load:
//   * E4M3 -> f16 is exact (every E4M3 value is an f16 value), so the MMAs run in f16 and the
//     fp32 scales stay out of the operands: k_scale multiplies the token's score and v_scale its
//     probability, both on the thread that owns the token;
//   * Q is carried as an f16 pair hi + lo (hi = f16(q), lo = f16(q - hi)) over the same K
//     columns, so the score keeps float32-level accuracy.
//
// Roles (320 threads):
//   warp 0      TMA producer: raw K and V code tiles through an NCS-stage ring
//   warp 1      TMEM allocator; lane 0 issues every MMA
//   warps 2..5  converter: thread = token; K codes -> f16 straight into TMEM (the A operand of
//               the S MMA), V codes -> f16 in shared memory (the A operand of the PV MMA);
//               both double-buffered so conversion runs a tile ahead of the softmax
//   warps 6..9  softmax + epilogue: thread = token (and later = output element d)
// TMEM columns: S^T [0,32) (two 16-column buffers), O^T [32,48), K tiles [64,128) and [128,192).
#pragma once

#include "decode.cuh"

namespace attn {

struct DecodeFp8Cfg {
  static constexpr int D = 128;
  static constexpr int NCS = 3;                 // stages of raw code tiles
  static constexpr int CODE_TILE = 128 * 128;   // 128 tokens x 128 one-byte codes
  static constexpr int VC_TILE = 2 * 128 * 128; // 128 tokens x 128 f16, two 64-wide boxes
  static constexpr int QBOX = 16 * 128;
  static constexpr int Q_BYTES = 2 * QBOX;      // one of hi / lo
  static constexpr int P_BYTES = 2 * QBOX;
  static constexpr int OFF_KCODE = 0;
  static constexpr int OFF_VCODE = OFF_KCODE + NCS * CODE_TILE;
  static constexpr int OFF_VC = OFF_VCODE + NCS * CODE_TILE;
  static constexpr int OFF_Q = OFF_VC + 2 * VC_TILE;
  static constexpr int OFF_P = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_RED = OFF_P + 2 * P_BYTES;
  static constexpr int OFF_BAR = OFF_RED + (2 * 4 * 16 + 4 * 16) * 4;
  static constexpr int N_BARS = 4 * NCS + 1 + 2 + 2 + 1 + 8 + 1 + 2 + 1;
  static constexpr int SMEM_BYTES = OFF_BAR + N_BARS * 8 + 16 + 1024;
  static constexpr int THREADS = 320;
  static constexpr uint32_t TMEM_COLS = 256;
  static constexpr float RESCALE_THRESHOLD = 8.0f;
};

__global__ void __launch_bounds__(320, 1)
    decode_fp8_sm100(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const DecodeParams p) {
  using C = DecodeFp8Cfg;
  constexpr int D = C::D;
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int len = p.kv_lens[b];
  len = len < 0 ? 0 : (len > p.Tmax ? p.Tmax : len);
  const int t0 = split * p.split_tokens;
  const int t1 = min(len, t0 + p.split_tokens);
  const int n = t1 > t0 ? (t1 - t0 + 127) / 128 : 0;
  const int G = p.G;

  if (n == 0) {  // empty split: o = 0, lse = -inf
    for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
      const int g = i / D, d = i % D;
      const long long h = (long long)kvh * G + g;
      if (p.n_splits == 1) {
        p.o[((long long)b * p.Hq + h) * D + d] = __float2bfloat16_rn(0.f);
        if (d == 0 && p.lse) p.lse[(long long)b * p.Hq + h] = -INFINITY;
      } else {
        p.o_part[(((long long)split * p.B + b) * p.Hq + h) * D + d] = 0.f;
        if (d == 0) p.lse_part[((long long)split * p.B + b) * p.Hq + h] = -INFINITY;
      }
    }
    return;
  }

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* k_full = bars;                 // [NCS] raw K codes landed
  uint64_t* k_empty = k_full + C::NCS;     // [NCS] converter done with the raw K stage
  uint64_t* v_full = k_empty + C::NCS;
  uint64_t* v_empty = v_full + C::NCS;
  uint64_t* q_ready = v_empty + C::NCS;
  uint64_t* s_full = q_ready + 1;          // [2]
  uint64_t* p_full = s_full + 2;           // [2]
  uint64_t* o_ready = p_full + 2;
  uint64_t* kc_full = o_ready + 1;         // [2] converted K in TMEM
  uint64_t* kc_empty = kc_full + 2;        // [2] S MMA done reading it
  uint64_t* vc_full = kc_empty + 2;        // [2] converted V in shared memory
  uint64_t* vc_empty = vc_full + 2;        // [2] PV MMA done reading it
  uint64_t* drain = vc_empty + 2;
  uint64_t* red_bar = drain + 1;           // [2]
  uint64_t* sum_bar = red_bar + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sum_bar + 1);
  float* red_max = reinterpret_cast<float*>(smem + C::OFF_RED);  // [2][4][16]
  float* red_sum = red_max + 2 * 4 * 16;                         // [4][16]

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NCS; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 128);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 128);
    }
    mbar_init(q_ready, 128);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 128);
      mbar_init(&kc_full[s], 128);
      mbar_init(&kc_empty[s], 1);
      mbar_init(&vc_full[s], 128);
      mbar_init(&vc_empty[s], 1);
      mbar_init(&red_bar[s], 128);
    }
    mbar_init(o_ready, 1);
    mbar_init(drain, 1);
    mbar_init(sum_bar, 128);
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
  const uint32_t tS0 = tmem, tO = tmem + 32, tK0 = tmem + 64;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < n; ++j) {
        const int st = j % C::NCS;
        const uint32_t ph = (j / C::NCS) & 1;
        const int tok = t0 + j * 128;
        if (!(ok = mbar_wait(&k_empty[st], ph ^ 1, SITE_DC_LOAD_EMPTY))) break;
        mbar_arrive_expect_tx(&k_full[st], C::CODE_TILE);
        tma_load_4d(smem + C::OFF_KCODE + st * C::CODE_TILE, &tmK, &k_full[st], 0, kvh, tok, b);
        issued = 2 * j + 1;
        if (!(ok = mbar_wait(&v_empty[st], ph ^ 1, SITE_DC_LOAD_EMPTY))) break;
        mbar_arrive_expect_tx(&v_full[st], C::CODE_TILE);
        tma_load_4d(smem + C::OFF_VCODE + st * C::CODE_TILE, &tmV, &v_full[st], 0, kvh, tok, b);
        issued = 2 * j + 2;
      }
      if (!ok) {
        const int nk = (issued + 1) / 2, nv = issued / 2;
        for (int j = (nk > C::NCS ? nk - C::NCS : 0); j < nk; ++j)
          mbar_wait_drain(&k_full[j % C::NCS], (j / C::NCS) & 1, SITE_DC_DRAIN);
        for (int j = (nv > C::NCS ? nv - C::NCS : 0); j < nv; ++j)
          mbar_wait_drain(&v_full[j % C::NCS], (j / C::NCS) & 1, SITE_DC_DRAIN);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = make_idesc_f16(128, 16, false, false, false);
      constexpr uint32_t idesc_pv = make_idesc_f16(128, 16, true, false, false);
      const uint32_t sQ = smem_u32(smem + C::OFF_Q);
      const uint32_t sP = smem_u32(smem + C::OFF_P);
      const uint32_t sVc = smem_u32(smem + C::OFF_VC);
      // S^T(j) = K_j (TMEM, f16) . [Q_hi; Q_lo]^T over the same K columns
      auto issue_s = [&](int buf) {
        for (int kk = 0; kk < 16; ++kk) {
          const int kd = kk & 7;
          const uint32_t qoff = (kk >> 3) * C::Q_BYTES + (kd >> 2) * C::QBOX + (kd & 3) * 32;
          mma_ts(tS0 + buf * 16, tK0 + buf * 64 + kd * 8, make_sdesc_sw128(sQ + qoff, 16, 1024), idesc_qk, kk > 0);
        }
      };
      auto issue_pv = [&](int buf, bool acc) {
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t da = make_sdesc_sw128(sVc + buf * C::VC_TILE + kk * 16 * 128, 128 * 128, 1024);
          const uint64_t db = make_sdesc_sw128(sP + buf * C::P_BYTES + (kk >> 2) * C::QBOX + (kk & 3) * 32, 16, 1024);
          mma_ss(tO, da, db, idesc_pv, (acc || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(q_ready, 0, SITE_DC_MMA_K);
      for (int jj = 0; jj < 2 && jj < n && ok; ++jj) {
        if (!(ok = mbar_wait(&kc_full[jj], 0, SITE_DC_MMA_K))) break;
        tc_fence_after();
        issue_s(jj);
        mma_commit(&s_full[jj]);
        mma_commit(&kc_empty[jj]);
      }
      for (int j = 0; j < n && ok; ++j) {
        const int b2 = j & 1;
        const uint32_t ph2 = (j >> 1) & 1;
        if (!(ok = mbar_wait(&vc_full[b2], ph2, SITE_DC_MMA_V))) break;
        if (!(ok = mbar_wait(&p_full[b2], ph2, SITE_DC_MMA_P))) break;
        tc_fence_after();
        issue_pv(b2, j > 0);
        mma_commit(o_ready);
        mma_commit(&vc_empty[b2]);
        if (j + 2 < n) {
          if (!(ok = mbar_wait(&kc_full[b2], ((j + 2) >> 1) & 1, SITE_DC_MMA_K))) break;
          tc_fence_after();
          issue_s(b2);
          mma_commit(&s_full[b2]);
          mma_commit(&kc_empty[b2]);
        }
      }
      mma_commit(drain);
      mbar_wait_drain(drain, 0, SITE_DC_DRAIN);
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------------ converter warpgroup
    const int wq = warp & 3;
    const int t = wq * 32 + lane;  // token row of the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    for (int j = 0; j < n; ++j) {
      const int st = j % C::NCS;
      const uint32_t ph = (j / C::NCS) & 1;
      const int b2 = j & 1;
      const uint32_t ph2 = (j >> 1) & 1;
      const bool valid = t0 + j * 128 + t < t1;
      // K_j -> f16 -> TMEM lane t (64 columns, two f16 per column)
      if (!mbar_wait_warp(&k_full[st], ph, SITE_DC_SM_K)) break;
      if (!mbar_wait_warp(&kc_empty[b2], ph2 ^ 1, SITE_DC_SM_K)) break;
      tc_fence_after();
      const uint8_t* ktile = smem + C::OFF_KCODE + st * C::CODE_TILE;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t h[32];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const int c = half * 4 + c4;
          uint4 w = make_uint4(0u, 0u, 0u, 0u);
          if (valid) w = *reinterpret_cast<const uint4*>(ktile + sw128_offset(t, c));
          const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            h[c4 * 8 + 2 * i] = e4m3x2_to_f16x2((uint16_t)(wd[i] & 0xFFFFu));
            h[c4 * 8 + 2 * i + 1] = e4m3x2_to_f16x2((uint16_t)(wd[i] >> 16));
          }
        }
        tmem_st32(tK0 + b2 * 64 + half * 32 + lane_off, h);
      }
      tmem_wait_st();
      mbar_arrive(&k_empty[st]);
      tc_fence_before();
      mbar_arrive(&kc_full[b2]);
      // V_j -> f16 in shared memory (zeros for tokens past the length)
      if (!mbar_wait_warp(&v_full[st], ph, SITE_DC_SM_V)) break;
      if (!mbar_wait_warp(&vc_empty[b2], ph2 ^ 1, SITE_DC_SM_V)) break;
      convert_row_e4m3(smem + C::OFF_VCODE + st * C::CODE_TILE, smem + C::OFF_VC + b2 * C::VC_TILE, t, valid);
      mbar_arrive(&v_empty[st]);
      fence_proxy_async_smem();
      mbar_arrive(&vc_full[b2]);
    }
  } else {
    // ------------------------------------------------------------------ softmax warpgroup
    const int wq = warp & 3;
    const int t = wq * 32 + lane;  // token of the tile / TMEM lane / output element d
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const int wg_tid = threadIdx.x - 192;
    for (int i = wg_tid; i < 2 * C::P_BYTES / 16; i += 128)
      reinterpret_cast<uint4*>(smem + C::OFF_P)[i] = make_uint4(0u, 0u, 0u, 0u);
    for (int c = wg_tid; c < 256; c += 128) {  // Q^T as f16 hi and lo, 16 rows (G real)
      const int g = c >> 4, cc = c & 15;
      uint4 x = make_uint4(0u, 0u, 0u, 0u);
      if (g < G) x = *reinterpret_cast<const uint4*>(p.q + ((long long)b * p.Hq + (long long)kvh * G + g) * D + cc * 8);
      const uint32_t off = (cc >> 3) * C::QBOX + sw128_offset(g, cc & 7);
      const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float f0 = __uint_as_float(xw[i] << 16), f1 = __uint_as_float(xw[i] & 0xFFFF0000u);
        const __half h0 = __float2half_rn(f0), h1 = __float2half_rn(f1);
        hi[i] = (uint32_t)__half_as_ushort(h0) | ((uint32_t)__half_as_ushort(h1) << 16);
        lo[i] = pack_f16x2(f0 - __half2float(h0), f1 - __half2float(h1));
      }
      *reinterpret_cast<uint4*>(smem + C::OFF_Q + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(smem + C::OFF_Q + C::Q_BYTES + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
    fence_proxy_async_smem();
    mbar_arrive(q_ready);

    float m_used[16], l_part[16];
#pragma unroll
    for (int g = 0; g < 16; ++g) {
      m_used[g] = -INFINITY;
      l_part[g] = 0.f;
    }
    bool ok = true;
    const long long kv_row0 = (long long)b * p.Tmax;
    for (int j = 0; j < n && ok; ++j) {
      const int b2 = j & 1;
      const uint32_t ph2 = (j >> 1) & 1;
      const int tok = t0 + j * 128 + t;
      const bool valid = tok < t1;
      float ks = 1.f, vs = 1.f;
      if (valid) {
        ks = p.k_scale[(kv_row0 + tok) * p.Hkv + kvh];
        vs = p.v_scale[(kv_row0 + tok) * p.Hkv + kvh];
      }
      if (!(ok = mbar_wait_warp(&s_full[b2], ph2, SITE_DC_SM_S))) break;
      tc_fence_after();
      uint32_t sv[16];
      tmem_ld16(tS0 + b2 * 16 + lane_off, sv);
      tmem_wait_ld();
      float x[16];
      const float sc = p.scale_log2 * ks;
#pragma unroll
      for (int g = 0; g < 16; ++g) x[g] = valid ? __uint_as_float(sv[g]) * sc : -INFINITY;
      float* rm = red_max + b2 * 64;
#pragma unroll
      for (int g = 0; g < 16; ++g) {
        if (g < G) {
          const float m = warp_max(x[g]);
          if (lane == 0) rm[wq * 16 + g] = m;
        }
      }
      mbar_arrive(&red_bar[b2]);
      if (!(ok = mbar_wait_warp(&red_bar[b2], ph2, SITE_DC_SM_S))) break;
      bool need = false;
      float alpha[16];
#pragma unroll
      for (int g = 0; g < 16; ++g) {
        alpha[g] = 1.f;
        if (g < G) {
          const float tm = fmaxf(fmaxf(rm[g], rm[16 + g]), fmaxf(rm[32 + g], rm[48 + g]));
          const float mn = fmaxf(m_used[g], tm);
          if (mn > m_used[g] + C::RESCALE_THRESHOLD) {
            alpha[g] = ex2_approx(m_used[g] - mn);
            m_used[g] = mn;
            l_part[g] *= alpha[g];
            need = true;
          }
        }
      }
      if (need && j > 0) {  // the decision is CTA-uniform (it follows the reduced maxima)
        if (!(ok = mbar_wait_warp(o_ready, (j - 1) & 1, SITE_DC_SM_O))) break;
        tc_fence_after();
        uint32_t orow[16];
        tmem_ld16(tO + lane_off, orow);
        tmem_wait_ld();
#pragma unroll
        for (int g = 0; g < 16; ++g) orow[g] = __float_as_uint(__uint_as_float(orow[g]) * alpha[g]);
        tmem_st16(tO + lane_off, orow);
        tmem_wait_st();
      }
      uint8_t* prow = smem + C::OFF_P + b2 * C::P_BYTES + (t >> 6) * C::QBOX;
      const uint32_t pchunk = (t & 63) >> 3, pbyte = (t & 7) * 2;
#pragma unroll
      for (int g = 0; g < 16; ++g) {
        if (g < G) {
          const float pr = (x[g] == -INFINITY) ? 0.f : ex2_approx(x[g] - m_used[g]);
          l_part[g] += pr;
          *reinterpret_cast<uint16_t*>(prow + sw128_offset(g, pchunk) + pbyte) =
              __half_as_ushort(__float2half_rn(pr * vs));
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[b2]);
    }
    if (ok) {
#pragma unroll
      for (int g = 0; g < 16; ++g) {
        if (g < G) {
          const float s = warp_sum(l_part[g]);
          if (lane == 0) red_sum[wq * 16 + g] = s;
        }
      }
      mbar_arrive(sum_bar);
      ok = mbar_wait_warp(sum_bar, 0, SITE_DC_SM_S) && mbar_wait_warp(o_ready, (n - 1) & 1, SITE_DC_SM_O);
    }
    if (ok) {
      tc_fence_after();
      uint32_t orow[16];
      tmem_ld16(tO + lane_off, orow);
      tmem_wait_ld();
      float my_lse = -INFINITY;
#pragma unroll
      for (int g = 0; g < 16; ++g) {
        if (g < G) {
          const float l = red_sum[g] + red_sum[16 + g] + red_sum[32 + g] + red_sum[48 + g];
          const float ov = (l > 0.f) ? __uint_as_float(orow[g]) / l : 0.f;
          const float lse = (l > 0.f) ? (m_used[g] + log2f(l)) * 0.69314718055994531f : -INFINITY;
          if (g == t) my_lse = lse;
          const long long h = (long long)kvh * G + g;
          if (p.n_splits == 1) {
            p.o[((long long)b * p.Hq + h) * D + t] = __float2bfloat16_rn(ov);
          } else {
            p.o_part[(((long long)split * p.B + b) * p.Hq + h) * D + t] = ov;
          }
        }
      }
      if (t < G) {
        const long long h = (long long)kvh * G + t;
        if (p.n_splits == 1) {
          if (p.lse) p.lse[(long long)b * p.Hq + h] = my_lse;
        } else {
          p.lse_part[((long long)split * p.B + b) * p.Hq + h] = my_lse;
        }
      }
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
