// Split-KV GQA decode over an FP8 E4M3 KV cache (LLM-CoOpt summary, "Opt-KV": the cache is
// stored in FP8 to halve the bytes per token; ONNX Runtime CPU GQA analysis, "Flash Decoding":
// split the key range, merge the partial softmax states by log-sum-exp).
//
// Same arithmetic as the bf16 kernel (KV tokens on the MMA's M axis:
// S^T = K.Q^T and O^T += V^T.P^T), with the dequantisation fused into the tile load:
//   * E4M3 -> f16 is exact (every E4M3 value is an f16 value), so the MMAs run in f16 and the
//     fp32 scales stay out of the operands: k_scale multiplies the token's score and v_scale its
//     probability, both on the thread that owns the token;
//   * Q is carried as an f16 pair hi + lo (hi = f16(q), lo = f16(q - hi)) stacked as the 32 rows of
//     one B operand, so a single 8-step MMA chain gives both products and the score keeps
//     float32-level accuracy.
//
// Roles (480 threads):
//   warp 0       TMA producer of the raw K code tiles (NCS-stage ring)
//   warp 14      TMA producer of the raw V code tiles (NCS-stage ring); a separate thread, so a
//                V stage still waiting for its converter never holds back the next K load
//   warp 1       TMEM allocator; lane 0 issues every MMA
//   warps 2..5   K converter: thread = token; K codes -> f16 straight into TMEM (the A operand of
//                the S MMA)
//   warps 6..9   V converter: thread = token; V codes -> f16 in shared memory (the A operand of
//                the PV MMA)
//   warps 10..13 softmax + epilogue: thread = token (and later = output element d)
// The two converters run side by side and ahead of the softmax.  Scores, probabilities and
// converted tiles rotate through NB = 3 buffers: S(j+3) is issued right after PV(j), so the
// softmax has two tiles of its own work to cover the PV -> S round trip of the tensor pipe.  PV
// completion has one barrier per buffer, so every wait on it is at most one phase behind.
// TMEM columns: S^T [0,96) (three 32-column buffers: Q_hi and Q_lo products), O^T [96,112),
// K tiles [128,320) (three 64-column buffers).
#pragma once

#include "decode.cuh"

namespace attn {

struct DecodeFp8Cfg {
  static constexpr int D = 128;
  static constexpr int NCS = 3;                 // stages of raw code tiles
  static constexpr int NB = 3;                  // S / P / converted-tile buffers
  static constexpr int CODE_TILE = 128 * 128;   // 128 tokens x 128 one-byte codes
  static constexpr int VC_TILE = 2 * 128 * 128; // 128 tokens x 128 f16, two 64-wide boxes
  static constexpr int QBOX = 32 * 128;         // Q_hi rows [0,16) + Q_lo rows [16,32), 64 wide
  static constexpr int Q_BYTES = 2 * QBOX;
  static constexpr int PBOX = 16 * 128;
  static constexpr int P_BYTES = 2 * PBOX;
  static constexpr int OFF_KCODE = 0;
  static constexpr int OFF_VCODE = OFF_KCODE + NCS * CODE_TILE;
  static constexpr int OFF_VC = OFF_VCODE + NCS * CODE_TILE;
  static constexpr int OFF_Q = OFF_VC + NB * VC_TILE;
  static constexpr int OFF_P = OFF_Q + Q_BYTES;
  static constexpr int OFF_RED = OFF_P + NB * P_BYTES;
  static constexpr int OFF_BAR = OFF_RED + (2 * 4 * 16 + 4 * 16) * 4;
  static constexpr int N_BARS = 4 * NCS + 1 + 7 * NB + 1 + 2 + 1 + 1;
  static constexpr int SMEM_BYTES = OFF_BAR + N_BARS * 8 + 16 + 1024;
  static constexpr int THREADS = 480;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S = 0, COL_O = 96, COL_K = 128;
  static constexpr float RESCALE_THRESHOLD = 8.0f;
};
static_assert(DecodeFp8Cfg::SMEM_BYTES <= 227 * 1024, "shared memory per CTA");

template <int GP>
__global__ void __launch_bounds__(480, 1)
    decode_fp8_sm100(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const DecodeParams p) {
  using C = DecodeFp8Cfg;
  constexpr int D = C::D;
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
    decode_write_empty(p, G, split, kvh, b);
    return;
  }
  ATTN_PROF_T0(cta_t0);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* k_full = bars;                 // [NCS] raw K codes landed
  uint64_t* k_empty = k_full + C::NCS;     // [NCS] converter done with the raw K stage
  uint64_t* v_full = k_empty + C::NCS;
  uint64_t* v_empty = v_full + C::NCS;
  uint64_t* q_ready = v_empty + C::NCS;
  uint64_t* s_full = q_ready + 1;          // [NB] S^T(j) in TMEM
  uint64_t* p_full = s_full + NB;          // [NB] P^T(j) in shared memory
  uint64_t* pv_done = p_full + NB;         // [NB] PV(j) completed
  uint64_t* kc_full = pv_done + NB;        // [NB] converted K in TMEM
  uint64_t* kc_empty = kc_full + NB;       // [NB] S MMA done reading it
  uint64_t* vc_full = kc_empty + NB;       // [NB] converted V in shared memory
  uint64_t* vc_empty = vc_full + NB;       // [NB] PV MMA done reading it
  uint64_t* drain = vc_empty + NB;
  uint64_t* red_bar = drain + 1;           // [2]
  uint64_t* sum_bar = red_bar + 2;
  uint64_t* o_final = sum_bar + 1;  // single phase: every PV of the split has completed
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(o_final + 1);
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
    for (int s = 0; s < NB; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 128);
      mbar_init(&pv_done[s], 1);
      mbar_init(&kc_full[s], 128);
      mbar_init(&kc_empty[s], 1);
      mbar_init(&vc_full[s], 128);
      mbar_init(&vc_empty[s], 1);
    }
    mbar_init(&red_bar[0], 128);
    mbar_init(&red_bar[1], 128);
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
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < n; ++j) {
        const int st = j % C::NCS;
        if (!(ok = mbar_wait(&empty[st], ((j / C::NCS) & 1) ^ 1, SITE_DC_LOAD_EMPTY))) break;
        mbar_arrive_expect_tx(&full[st], C::CODE_TILE);
        tma_load_4d(ring + st * C::CODE_TILE, tm, &full[st], 0, kvh, t0 + j * 128, b);
        issued = j + 1;
      }
      if (!ok)  // wait (bounded) for the copies still in flight before the CTA exits
        for (int j = (issued > C::NCS ? issued - C::NCS : 0); j < issued; ++j)
          mbar_wait_drain(&full[j % C::NCS], (j / C::NCS) & 1, SITE_DC_DRAIN);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = make_idesc_f16(128, 32, false, false, false);
      constexpr uint32_t idesc_pv = make_idesc_f16(128, 16, true, false, false);
      const uint32_t sQ = smem_u32(smem + C::OFF_Q);
      const uint32_t sP = smem_u32(smem + C::OFF_P);
      const uint32_t sVc = smem_u32(smem + C::OFF_VC);
      // S^T(j) [128 x 32] = K_j (TMEM, f16) . [Q_hi; Q_lo]^T
      auto issue_s = [&](int buf) {
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t qoff = (kk >> 2) * C::QBOX + (kk & 3) * 32;
          mma_ts(tS0 + buf * 32, tK0 + buf * 64 + kk * 8, make_sdesc_sw128(sQ + qoff, 16, 1024), idesc_qk, kk > 0);
        }
      };
      auto issue_pv = [&](int buf, bool acc) {  // O^T += V_j^T . P_j^T
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t da = make_sdesc_sw128(sVc + buf * C::VC_TILE + kk * 16 * 128, 128 * 128, 1024);
          const uint64_t db = make_sdesc_sw128(sP + buf * C::P_BYTES + (kk >> 2) * C::PBOX + (kk & 3) * 32, 16, 1024);
          mma_ss(tO, da, db, idesc_pv, (acc || kk > 0) ? 1u : 0u);
        }
      };
      ATTN_PROF_DECL(pw_vc);
      ATTN_PROF_DECL(pw_p);
      ATTN_PROF_DECL(pw_kc);
      bool ok = mbar_wait(q_ready, 0, SITE_DC_MMA_K);
      for (int jj = 0; jj < NB && jj < n && ok; ++jj) {
        if (!(ok = mbar_wait(&kc_full[jj], 0, SITE_DC_MMA_K))) break;
        tc_fence_after();
        issue_s(jj);
        mma_commit(&s_full[jj]);
        mma_commit(&kc_empty[jj]);
      }
      for (int j = 0; j < n && ok; ++j) {
        const int bj = j % NB;
        const uint32_t ph = (j / NB) & 1;
        ATTN_PROF_T0(q0);
        if (!(ok = mbar_wait(&vc_full[bj], ph, SITE_DC_MMA_V))) break;
        ATTN_PROF_ADD(pw_vc, q0);
        ATTN_PROF_T0(q1);
        if (!(ok = mbar_wait(&p_full[bj], ph, SITE_DC_MMA_P))) break;
        ATTN_PROF_ADD(pw_p, q1);
        tc_fence_after();
        issue_pv(bj, j > 0);
        mma_commit(&pv_done[bj]);
        mma_commit(&vc_empty[bj]);
        if (j + NB < n) {  // S(j+NB) reuses buffer bj: S(j) was read before P(j) was published
          ATTN_PROF_T0(q2);
          if (!(ok = mbar_wait(&kc_full[bj], ph ^ 1, SITE_DC_MMA_K))) break;
          ATTN_PROF_ADD(pw_kc, q2);
          tc_fence_after();
          issue_s(bj);
          mma_commit(&s_full[bj]);
          mma_commit(&kc_empty[bj]);
        }
      }
      if (ok) mma_commit(o_final);
      mma_commit(drain);
      mbar_wait_drain(drain, 0, SITE_DC_DRAIN);
      ATTN_PROF_FLUSH(0, pw_vc);
      ATTN_PROF_FLUSH(1, pw_p);
      ATTN_PROF_FLUSH(2, pw_kc);
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------------ K converter warpgroup
    const int wq = warp & 3;
    const int t = wq * 32 + lane;  // token row of the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    ATTN_PROF_DECL(cw_k);
    ATTN_PROF_DECL(cw_kce);
    ATTN_PROF_DECL(cc_k);
    for (int j = 0; j < n; ++j) {
      const int st = j % C::NCS;
      const uint32_t ph = (j / C::NCS) & 1;
      const int bj = j % NB;
      const uint32_t phb = (j / NB) & 1;
      const bool valid = t0 + j * 128 + t < t1;
      // K_j -> f16 -> TMEM lane t (64 columns, two f16 per column)
      ATTN_PROF_T0(c0);
      if (!mbar_wait_warp(&k_full[st], ph, SITE_DC_SM_K)) break;
      ATTN_PROF_ADD(cw_k, c0);
      ATTN_PROF_T0(c1);
      if (!mbar_wait_warp(&kc_empty[bj], phb ^ 1, SITE_DC_SM_K)) break;  // S(j-NB) has read it
      ATTN_PROF_ADD(cw_kce, c1);
      ATTN_PROF_T0(c2);
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
        tmem_st32(tK0 + bj * 64 + half * 32 + lane_off, h);
      }
      tmem_wait_st();
      mbar_arrive(&k_empty[st]);
      tc_fence_before();
      mbar_arrive(&kc_full[bj]);
      ATTN_PROF_ADD(cc_k, c2);
    }
    if (lane == 0 && wq == 2) {
      ATTN_PROF_FLUSH(3, cw_k);
      ATTN_PROF_FLUSH(4, cw_kce);
      ATTN_PROF_FLUSH(5, cc_k);
    }
  } else if (warp < 10) {
    // ------------------------------------------------------------------ V converter warpgroup
    const int t = (warp & 3) * 32 + lane;  // token row of the tile
    ATTN_PROF_DECL(cw_v);
    ATTN_PROF_DECL(cw_vce);
    ATTN_PROF_DECL(cc_v);
    for (int j = 0; j < n; ++j) {
      const int st = j % C::NCS;
      const uint32_t ph = (j / C::NCS) & 1;
      const int bj = j % NB;
      const uint32_t phb = (j / NB) & 1;
      const bool valid = t0 + j * 128 + t < t1;
      // V_j -> f16 in shared memory (zeros for tokens past the length)
      ATTN_PROF_T0(c3);
      if (!mbar_wait_warp(&v_full[st], ph, SITE_DC_SM_V)) break;
      ATTN_PROF_ADD(cw_v, c3);
      ATTN_PROF_T0(c4);
      if (!mbar_wait_warp(&vc_empty[bj], phb ^ 1, SITE_DC_SM_V)) break;  // PV(j-NB) has read it
      ATTN_PROF_ADD(cw_vce, c4);
      ATTN_PROF_T0(c5);
      convert_row_e4m3(smem + C::OFF_VCODE + st * C::CODE_TILE, smem + C::OFF_VC + bj * C::VC_TILE, t, valid);
      mbar_arrive(&v_empty[st]);
      fence_proxy_async_smem();
      mbar_arrive(&vc_full[bj]);
      ATTN_PROF_ADD(cc_v, c5);
    }
    if (lane == 0 && warp == 6) {
      ATTN_PROF_FLUSH(6, cw_v);
      ATTN_PROF_FLUSH(7, cw_vce);
      ATTN_PROF_FLUSH(8, cc_v);
    }
  } else {
    // ------------------------------------------------------------------ softmax warpgroup
    const int wq = warp & 3;
    const int t = wq * 32 + lane;  // token of the tile / TMEM lane / output element d
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const int wg_tid = threadIdx.x - 320;
    for (int i = wg_tid; i < NB * C::P_BYTES / 16; i += 128)  // P^T rows >= GP stay zero
      reinterpret_cast<uint4*>(smem + C::OFF_P)[i] = make_uint4(0u, 0u, 0u, 0u);
    decode_stage_q(p, G, kvh, b, wg_tid, smem + C::OFF_Q, true);
    fence_proxy_async_smem();
    mbar_arrive(q_ready);

    DecodeRows<GP> rows;
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      rows.m_used[g] = -INFINITY;
      rows.l_part[g] = 0.f;
    }
    bool ok = true;
    const long long kv_row0 = (long long)b * p.Tmax;
    // Per-token scales are prefetched one tile ahead so their global-memory latency stays off
    // the tile's critical path.
    float ks_next = 1.f, vs_next = 1.f;
    if (t0 + t < t1) {
      ks_next = __ldg(p.k_scale + (kv_row0 + t0 + t) * p.Hkv + kvh);
      vs_next = __ldg(p.v_scale + (kv_row0 + t0 + t) * p.Hkv + kvh);
    }
    ATTN_PROF_DECL(sw_s);
    ATTN_PROF_DECL(sc_all);
    for (int j = 0; j < n && ok; ++j) {
      ATTN_PROF_T0(s0);
      const int bj = j % NB;
      const uint32_t phb = (j / NB) & 1;
      const int tok = t0 + j * 128 + t;
      const bool valid = tok < t1;
      const float ks = ks_next, vs = vs_next;
      if (tok + 128 < t1) {
        ks_next = __ldg(p.k_scale + (kv_row0 + tok + 128) * p.Hkv + kvh);
        vs_next = __ldg(p.v_scale + (kv_row0 + tok + 128) * p.Hkv + kvh);
      }
      ATTN_PROF_T0(s1);
      if (!(ok = mbar_wait_warp(&s_full[bj], phb, SITE_DC_SM_S))) break;
      ATTN_PROF_ADD(sw_s, s1);
      tc_fence_after();
      // PV(j-1) is completion number (j-1)/NB of pv_done[(j-1)%NB]; S(j) completing implies PV(j-NB)
      // done (S(j) was issued after it), so that barrier has at most this one phase pending.
      const int jp = j > 0 ? j - 1 : 0;
      if (!(ok = decode_softmax_tile<GP, true, true>(rows, j, lane, wq, t, valid, p.scale_log2 * ks, vs,
                                                     tS0 + bj * 32 + lane_off, tO + lane_off, red_max, red_bar,
                                                     &pv_done[jp % NB], (uint32_t)(jp / NB) & 1,
                                                     smem + C::OFF_P + bj * C::P_BYTES, C::RESCALE_THRESHOLD)))
        break;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[bj]);
      ATTN_PROF_ADD(sc_all, s0);
    }
    ATTN_PROF_T0(ep0);
    if (ok) decode_epilogue<GP>(rows, p, G, split, kvh, b, lane, wq, t, tO + lane_off, red_sum, sum_bar, o_final);
    if (lane == 0 && wq == 2) {
      ATTN_PROF_FLUSH(9, sw_s);
      ATTN_PROF_FLUSH(11, sc_all);
      ATTN_PROF_FLUSH(12, (long long)n);
      ATTN_PROF_FLUSH(13, clock64() - ep0);
      ATTN_PROF_FLUSH(14, ep0 - cta_t0);
      ATTN_PROF_FLUSH(15, 1);
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
