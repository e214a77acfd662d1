// Exact GQA prefill on tcgen05: one CTA computes two 128-row query tiles ("slots") that
// share every K/V tile, so each K/V byte staged in shared memory feeds 256 query rows.
//
// Method (ONNX Runtime CPU GQA analysis, "Flash Attention tiling"): for each key block
// compute the score block, update the running row max and row sum (online softmax), and
// accumulate P.V into the output; the S x T score matrix never leaves the SM.
//
// Persistent: one CTA per SM walks the work items c, c + grid, ... (heaviest causal tiles first);
// TMEM stays allocated and every barrier keeps counting phases across items, so the next item's
// first QK^T overlaps the current epilogue and the K/V ring never drains between items.
//
// Roles (384 threads; warpgroup 0 hands most of its registers to warpgroups 1 and 2):
//   warp 0        TMA producer: per item the Q tiles, then K_j / V_j through an NST-stage ring
//   warp 1        TMEM allocator; MMA issuer (the warp runs the loop, one elected lane issues)
//   warps 4..7    softmax + epilogue for slot 0 (one thread per TMEM lane = query row)
//   warps 8..11   softmax + epilogue for slot 1
// TMEM columns: S0/P0 [0,128), S1/P1 [128,256), O0 [256,256+D), O1 [256+D,256+2D).
// P (bf16, two per column) overwrites the first 64 columns of its S region.  MMA order per
// key tile j: PV0(j), S0(j+1), PV1(j), S1(j+1) — so S_s(j+1) completing implies PV_s(j)
// completed, and the softmax warps may rescale O_s and overwrite P_s in place.
#pragma once

#include "ptx.cuh"

// Of every 8 exponential pairs of the softmax, this many are computed by polynomial on the FMA
// pipe instead of the MUFU (0: all on the MUFU).
#ifndef ATTN_PREFILL_POLY_PER8
#define ATTN_PREFILL_POLY_PER8 1
#endif

namespace attn {

constexpr int kPolyPer8 = ATTN_PREFILL_POLY_PER8;

struct PrefillParams {
  int B, Hq, Hkv, D, S, T, G;
  int causal;
  long long q_pos0, kv_pos0;
  float scale_log2;  // scale * log2(e)
  int n_qtiles;      // ceil(S / 128)
  int pair_heads;    // 1: the slots are heads 2u, 2u+1 of one KV group at one query tile
  int n_head_units;  // Hq/2 (paired heads) or Hq
  int n_q_units;     // n_qtiles (paired heads) or ceil(n_qtiles / 2)
  int n_items;       // B * n_head_units * n_q_units
  void* o;
  int o_f32;
  long long o_sb, o_ss, o_sh;  // element strides of o between batches, tokens and heads (D contiguous)
  float* lse;
  // 1: o (float32) and lse already hold the normalised output and log-sum-exp of earlier key chunks
  // for these rows; the kernel merges its own result into them by log-sum-exp (the exact merge of
  // partial softmax states), and leaves rows that see no key here unchanged.
  int accumulate;
  // Packed variable-length batch (ORT packed-QSA analysis, "Code analysis": cumulative sequence
  // lengths, and a token's position = past length + its index among the new tokens): sequence b's
  // queries are rows cu_q[b] .. cu_q[b+1]-1 of q/o/lse and its keys rows cu_k[b] .. cu_k[b+1]-1 of
  // k/v; query i sits at position (len_k - len_q) + i, key j at j.  Null for a dense batch.
  const int* cu_q;
  const int* cu_k;
};

template <int D>
struct PrefillCfg {
  static constexpr int BM = 128;                 // query rows per slot
  static constexpr int BN = 128;                 // keys per tile
  static constexpr int NST = (D == 128) ? 2 : 3;  // K/V ring stages
  static constexpr int BOX_BYTES = 128 * 128;     // one TMA box: 128 rows x 64 bf16
  static constexpr int NBOX = D / 64;             // boxes per tile along D
  static constexpr int TILE_BYTES = NBOX * BOX_BYTES;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * TILE_BYTES;
  static constexpr int OFF_V = OFF_K + NST * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_V + NST * TILE_BYTES;
  static constexpr int N_BARS = 2 + 4 * NST + 2 + 2 + 2 + 1;
  static constexpr int SMEM_BYTES = OFF_BAR + N_BARS * 8 + 16 + 1024;  // + alignment slack
  static constexpr int THREADS = 384;
  // Register split (setmaxnreg): the producer / MMA warpgroup gives registers to the two softmax
  // warpgroups, which hold a row's 128 scores and weights.  REGS_CTRL * 128 + REGS_SOFTMAX * 256
  // must not exceed the launch allocation (the host checks it against the compiled count).
  static constexpr int REGS_CTRL = 72;
  static constexpr int REGS_SOFTMAX = 216;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units: rescale O only when max grows > 2^8
};

struct PrefillItem {
  int b, head[2], q_lo[2];
  bool active[2];
  int n_tiles;
  int kvh;
  int S, T;                    // this sequence's query and key counts
  long long q_pos0, kv_pos0;   // absolute positions of its query row 0 and key 0
  int q_base, k_base, bc;      // TMA token offsets of its rows 0 and batch coordinate
  long long o_base;            // element offset of query 0's row in o
  long long lse_row0;          // row of query 0 in lse (rows of Hq heads)
};

__device__ __forceinline__ PrefillItem prefill_item(const PrefillParams& p, int idx) {
  PrefillItem it;
  const int per_q = p.B * p.n_head_units;
  const int qunit = p.n_q_units - 1 - idx / per_q;  // heaviest causal tiles first
  const int rem = idx % per_q;
  it.b = rem / p.n_head_units;
  const int hunit = rem % p.n_head_units;
  if (p.cu_q) {
    const int qs = __ldg(p.cu_q + it.b), qe = __ldg(p.cu_q + it.b + 1);
    const int ks = __ldg(p.cu_k + it.b), ke = __ldg(p.cu_k + it.b + 1);
    it.S = qe > qs ? qe - qs : 0;
    it.T = ke > ks ? ke - ks : 0;
    it.q_pos0 = (long long)it.T - it.S;  // the queries are the sequence's last S tokens
    it.kv_pos0 = 0;
    it.q_base = qs;
    it.k_base = ks;
    it.bc = 0;
    it.o_base = (long long)qs * p.o_ss;
    it.lse_row0 = qs;
  } else {
    it.S = p.S;
    it.T = p.T;
    it.q_pos0 = p.q_pos0;
    it.kv_pos0 = p.kv_pos0;
    it.q_base = 0;
    it.k_base = 0;
    it.bc = it.b;
    it.o_base = (long long)it.b * p.o_sb;
    it.lse_row0 = (long long)it.b * p.S;
  }
  for (int s = 0; s < 2; ++s) {
    int head, qt;
    if (p.pair_heads) {
      head = 2 * hunit + s;
      qt = qunit;
    } else {
      head = hunit;
      qt = 2 * qunit + s;
    }
    it.head[s] = head;
    it.q_lo[s] = qt * 128;
    it.active[s] = it.q_lo[s] < it.S;
  }
  it.kvh = it.head[0] / p.G;
  int n = 0;
  for (int s = 0; s < 2; ++s) {
    if (!it.active[s]) continue;
    long long kv_end = it.T;
    if (p.causal) {
      const long long q_last = (long long)min(it.S, it.q_lo[s] + 128) - 1;
      long long e = it.q_pos0 + q_last - it.kv_pos0 + 1;
      kv_end = e < kv_end ? e : kv_end;
    }
    if (kv_end < 0) kv_end = 0;
    const int ns = (int)((kv_end + 127) / 128);
    n = ns > n ? ns : n;
  }
  it.n_tiles = n;
  return it;
}

template <int D>
__global__ void __launch_bounds__(384, 1)
    prefill_fwd_sm100(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using C = PrefillCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  // Phases: q_* and o_* complete once per item with tiles (item counter qi), k/v_* once per ring
  // use (CTA-wide tile counter g), s_full / p_full once per tile (g).
  uint64_t* q_full = bars + 0;          // Q tiles of the item landed
  uint64_t* q_empty = bars + 1;         // the item's last QK^T has read them
  uint64_t* k_full = bars + 2;
  uint64_t* k_empty = k_full + C::NST;
  uint64_t* v_full = k_empty + C::NST;
  uint64_t* v_empty = v_full + C::NST;
  uint64_t* s_full = v_empty + C::NST;  // [2]
  uint64_t* p_full = s_full + 2;        // [2]
  uint64_t* o_full = p_full + 2;        // the item's last PV has completed
  uint64_t* o_empty = o_full + 1;       // the epilogue has read O out of TMEM (8 warps)
  uint64_t* drain = o_empty + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 4);  // one arrival per softmax warp of the slot
    }
    mbar_init(o_full, 1);
    mbar_init(o_empty, 8);  // one arrival per softmax warp
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    if (lane == 0) ATTN_TRACE_AT(1, 1, 0);
    tmem_alloc(tmem_holder, C::TMEM_COLS);
    tmem_relinquish();
    if (lane == 0) ATTN_TRACE_AT(1, 2, 0);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  ATTN_EVT_INIT();

  // Each role derives its work items after its register change.
  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    regs_dec<C::REGS_CTRL>();
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      // L2: a Q tile is read once (evict first); a K/V tile is read by every query tile of its
      // head group, so it is kept (evict last) against the streamed Q reads and O writes.
      const uint64_t pol_q = l2_policy_evict_first();
      const uint64_t pol_kv = l2_policy_evict_last();
      uint8_t* sQ = smem + C::OFF_Q;
      int g = 0, qi = 0;  // tiles loaded, items with tiles
      int nk = 0, nv = 0;  // K / V tiles issued
      bool ok = true, q_pending = false;
      for (int idx = blockIdx.x; idx < p.n_items && ok; idx += gridDim.x) {
        const PrefillItem it = prefill_item(p, idx);
        const int n = it.n_tiles;
        if (n == 0) continue;
        ATTN_TRACE_AT(0, 3, qi);
        if (qi > 0 && !(ok = mbar_wait<true>(q_empty, (qi - 1) & 1, SITE_PF_LOAD_EMPTY))) break;
        mbar_arrive_expect_tx(q_full, 2 * C::TILE_BYTES);
        for (int s = 0; s < 2; ++s)
          for (int bx = 0; bx < C::NBOX; ++bx)
            tma_load_4d_hint(sQ + s * C::TILE_BYTES + bx * C::BOX_BYTES, &tmQ, q_full, bx * 64, it.head[s],
                             it.q_base + it.q_lo[s], it.bc, pol_q);
        q_pending = true;
        for (int j = 0; j < n; ++j, ++g) {
          const int st = g % C::NST;
          const uint32_t ph = (g / C::NST) & 1;
          ATTN_TRACE_AT(0, 4, j);
          if (!(ok = mbar_wait<true>(&k_empty[st], ph ^ 1, SITE_PF_LOAD_EMPTY))) break;
          mbar_arrive_expect_tx(&k_full[st], C::TILE_BYTES);
          for (int bx = 0; bx < C::NBOX; ++bx)
            tma_load_4d_hint(smem + C::OFF_K + st * C::TILE_BYTES + bx * C::BOX_BYTES, &tmK, &k_full[st], bx * 64,
                             it.kvh, it.k_base + j * 128, it.bc, pol_kv);
          ++nk;
          ATTN_TRACE_AT(0, 5, j);
          if (!(ok = mbar_wait<true>(&v_empty[st], ph ^ 1, SITE_PF_LOAD_EMPTY))) break;
          mbar_arrive_expect_tx(&v_full[st], C::TILE_BYTES);
          for (int bx = 0; bx < C::NBOX; ++bx)
            tma_load_4d_hint(smem + C::OFF_V + st * C::TILE_BYTES + bx * C::BOX_BYTES, &tmV, &v_full[st], bx * 64,
                             it.kvh, it.k_base + j * 128, it.bc, pol_kv);
          ++nv;
        }
        if (ok) {
          ++qi;
          q_pending = false;
        }
      }
      ATTN_TRACE_AT(0, 6, nk);
      if (!ok) {
        // Let every copy already issued land before the CTA's shared memory is released.
        if (q_pending) mbar_wait_drain<true>(q_full, qi & 1, SITE_PF_DRAIN);
        for (int t = (nk > C::NST ? nk - C::NST : 0); t < nk; ++t)
          mbar_wait_drain<true>(&k_full[t % C::NST], (t / C::NST) & 1, SITE_PF_DRAIN);
        for (int t = (nv > C::NST ? nv - C::NST : 0); t < nv; ++t)
          mbar_wait_drain<true>(&v_full[t % C::NST], (t / C::NST) & 1, SITE_PF_DRAIN);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop in lockstep and one elected lane issues each MMA and commit:
    // descriptors are base values computed once plus compile-time offsets of their start-address
    // field (addresses stay below 2^18 bytes, so the field never carries), so an MMA costs the
    // issuing warp a couple of uniform instructions even while the softmax warps sharing its
    // sub-partition keep the issue slots busy.
    regs_dec<C::REGS_CTRL>();
    {
      constexpr uint32_t idesc_qk = make_idesc_f16(128, 128, false, false, true);
      constexpr uint32_t idesc_pv = make_idesc_f16(128, D, false, true, true);
      constexpr uint32_t HI = sdesc_sw128_hi(1024);  // every operand here: 8-row groups 1024 B apart
      const uint32_t q_lo = sdesc_sw128_lo(smem_u32(smem + C::OFF_Q), 16);
      const uint32_t k_lo = sdesc_sw128_lo(smem_u32(smem + C::OFF_K), 16);
      const uint32_t v_lo = sdesc_sw128_lo(smem_u32(smem + C::OFF_V), C::BOX_BYTES);
      auto issue_qk = [&](int s, int st) {
        const uint32_t a0 = q_lo + ((s * C::TILE_BYTES) >> 4), b0 = k_lo + ((st * C::TILE_BYTES) >> 4);
        const uint32_t d = tmem + s * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * C::BOX_BYTES + (kk & 3) * 32) >> 4;
          mma_ss_elect(d, sdesc_join(a0 + off, HI), sdesc_join(b0 + off, HI), idesc_qk, kk > 0);
        }
      };
      auto issue_pv = [&](int s, int st, bool acc) {
        const uint32_t b0 = v_lo + ((st * C::TILE_BYTES) >> 4);
        const uint32_t d = tmem + 256 + s * D, a = tmem + s * 128;
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          mma_ts_elect(d, a + kk * 8, sdesc_join(b0 + ((kk * 16 * 128) >> 4), HI), idesc_pv,
                       (acc || kk > 0) ? 1u : 0u);
      };
      int g = 0, qi = 0;
      bool ok = true;
      for (int idx = blockIdx.x; idx < p.n_items && ok; idx += gridDim.x) {
        const int n = prefill_item(p, idx).n_tiles;
        if (n == 0) continue;
        if (lane == 0) ATTN_TRACE_AT(1, 3, qi);
        if (!(ok = mbar_wait_warp<true>(q_full, qi & 1, SITE_PF_MMA_Q))) break;
        if (!(ok = mbar_wait_warp<true>(&k_full[g % C::NST], (g / C::NST) & 1, SITE_PF_MMA_K))) break;
        tc_fence_after();
        // S(0) of this item overwrites S/P regions the previous item's PVs read: those were issued
        // earlier by this warp and the tensor pipe executes in order.
        if (lane == 0 && qi == 0) ATTN_EVT(0, 0);
        issue_qk(0, g % C::NST);
        mma_commit_elect(&s_full[0]);
        if (lane == 0 && qi == 0) ATTN_EVT(0, 8);
        issue_qk(1, g % C::NST);
        mma_commit_elect(&s_full[1]);
        mma_commit_elect(&k_empty[g % C::NST]);
        if (n == 1) mma_commit_elect(q_empty);
        for (int j = 0; j < n; ++j) {
          const int gj = g + j;
          const int st = gj % C::NST;
          const uint32_t ph = (gj / C::NST) & 1;
          const bool more = j + 1 < n;
          const int st1 = (gj + 1) % C::NST;
          const uint32_t ph1 = ((gj + 1) / C::NST) & 1;
          const int ej = qi == 0 ? j : 64;  // timeline events: the CTA's first item only
          if (lane == 0) ATTN_TRACE_AT(1, 5, j);
          if (!(ok = mbar_wait_warp<true>(&v_full[st], ph, SITE_PF_MMA_V))) break;
          if (lane == 0) ATTN_TRACE_AT(1, 6, j);
          if (!(ok = mbar_wait_warp<true>(&p_full[0], gj & 1, SITE_PF_MMA_P))) break;
          // The first PV of an item overwrites O: the previous item's epilogue must have read it.
          if (j == 0 && qi > 0 && !(ok = mbar_wait_warp<true>(o_empty, (qi - 1) & 1, SITE_PF_MMA_P))) break;
          if (lane == 0) ATTN_TRACE_AT(1, 7, j);
          tc_fence_after();
          if (lane == 0) ATTN_EVT(ej, 3);
          issue_pv(0, st, j > 0);
          if (more) {
            if (!(ok = mbar_wait_warp<true>(&k_full[st1], ph1, SITE_PF_MMA_K))) break;
            tc_fence_after();
            if (lane == 0) ATTN_EVT(ej + 1, 0);
            issue_qk(0, st1);
            mma_commit_elect(&s_full[0]);
          }
          if (lane == 0) ATTN_TRACE_AT(1, 8, j);
          if (!(ok = mbar_wait_warp<true>(&p_full[1], gj & 1, SITE_PF_MMA_P))) break;
          if (lane == 0) ATTN_TRACE_AT(1, 9, j);
          tc_fence_after();
          if (lane == 0) ATTN_EVT(ej, 11);
          issue_pv(1, st, j > 0);
          mma_commit_elect(&v_empty[st]);
          if (more) {
            if (lane == 0) ATTN_EVT(ej + 1, 8);
            issue_qk(1, st1);
            mma_commit_elect(&s_full[1]);
            mma_commit_elect(&k_empty[st1]);
            if (j + 2 == n) mma_commit_elect(q_empty);  // that was the item's last QK^T
          }
        }
        if (!ok) break;
        mma_commit_elect(o_full);
        g += n;
        ++qi;
      }
      if (lane == 0) ATTN_TRACE_AT(1, 10, ok);
      // Drain: every MMA issued above completes before TMEM is released.
      mma_commit_elect(drain);
      const bool drained = mbar_wait_drain<true>(drain, 0, SITE_PF_DRAIN);
      if (lane == 0) ATTN_TRACE_AT(1, 11, drained);
    }
    __syncwarp();
  } else if (warp < 4) {
    regs_dec<C::REGS_CTRL>();  // idle warps of warpgroup 0: give their registers away
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    regs_inc<C::REGS_SOFTMAX>();
    const int slot = (warp - 4) >> 2;
    const int wq = warp & 3;  // TMEM lane quarter this warp may access
    const int r = wq * 32 + lane;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + slot * 128 + lane_off;
    const uint32_t tO = tmem + 256 + slot * D + lane_off;
    int g = 0, qi = 0;
    bool ok = true;
    for (int idx = blockIdx.x; idx < p.n_items && ok; idx += gridDim.x) {
      const PrefillItem it = prefill_item(p, idx);
      const int n = it.n_tiles;
      const int q_lo = it.q_lo[slot];
      const long long rel = it.q_pos0 + q_lo + r - it.kv_pos0;  // key index limit (inclusive) for causal
      float m_used = -INFINITY, l = 0.f;
      for (int j = 0; j < n; ++j) {
        const int gj = g + j;
        const int ej = qi == 0 ? j : 64;
        if (r == 0) ATTN_TRACE_AT(2 + slot, 1, j);
        // tcgen05.ld/st are warp-collective: every lane takes the same branch around them.
        if (!(ok = mbar_wait_warp<true>(&s_full[slot], gj & 1, SITE_PF_SM_S))) break;
        if (r == 0) ATTN_TRACE_AT(2 + slot, 2, j);
        if (r == 0) ATTN_EVT(ej, slot * 8 + 1);
        tc_fence_after();
        const int kv0 = j * 128;
        long long lim64 = (long long)it.T - kv0;  // column c is a visible key iff c < lim
        if (p.causal) {
          const long long c2 = rel + 1 - kv0;
          lim64 = c2 < lim64 ? c2 : lim64;
        }
        const int lim = lim64 < 0 ? 0 : (lim64 > 128 ? 128 : (int)lim64);
        // all 128 scores of the row in registers (one TMEM round trip)
        uint32_t sr[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_wait_ld_regs(*reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
        if (lim < 128) {
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i >= lim) sr[i] = __float_as_uint(-INFINITY);
        }
        float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
        for (int i = 0; i < 128; i += 8) {
          mx0 = max3(mx0, __uint_as_float(sr[i]), __uint_as_float(sr[i + 1]));
          mx1 = max3(mx1, __uint_as_float(sr[i + 2]), __uint_as_float(sr[i + 3]));
          mx2 = max3(mx2, __uint_as_float(sr[i + 4]), __uint_as_float(sr[i + 5]));
          mx3 = max3(mx3, __uint_as_float(sr[i + 6]), __uint_as_float(sr[i + 7]));
        }
        const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * p.scale_log2;
        const float m_new = fmaxf(m_used, m_tile);
        const bool need = m_new > m_used + C::RESCALE_THRESHOLD;
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = need ? ex2_approx(m_used - m_new) : 1.f;  // 0 when m_used = -inf
          if (need) {
            l *= alpha;
            m_used = m_new;
          }
          if (j > 0) {  // the whole warp rescales its 32 rows of O (factor 1 where unchanged)
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              uint32_t orow[32];
              tmem_ld32(tO + c * 32, orow);
              tmem_wait_ld_regs(orow);
#pragma unroll
              for (int i = 0; i < 32; ++i) orow[i] = __float_as_uint(__uint_as_float(orow[i]) * alpha);
              tmem_st32(tO + c * 32, orow);
            }
            tmem_wait_st();
          }
        }
        if (r == 0) ATTN_EVT(ej, slot * 8 + 2);
        const float neg_m = (m_used == -INFINITY) ? 0.f : -m_used;
        // p = 2^(s * scale * log2 e - m) in packed fp32 pairs; ATTN_PREFILL_POLY_PER8 pairs in 8 go
        // to the FMA pipe (polynomial) and the rest to the MUFU.  P is stored per 32 scores (16
        // packed columns, over S columns already read into registers).  The fp32 weights stay in
        // the score registers: the row sum is taken after P is handed to the MMA, off the critical
        // path.
        const float2 c2 = make_float2(p.scale_log2, p.scale_log2);
        const float2 nm2 = make_float2(neg_m, neg_m);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int k = c * 32 + 2 * i;
            const float2 x = fma2(make_float2(__uint_as_float(sr[k]), __uint_as_float(sr[k + 1])), c2, nm2);
            float2 e;
            if ((i & 7) >= 8 - kPolyPer8) {
              e = exp2_poly2(x);
            } else {
              e.x = ex2_approx(x.x);
              e.y = ex2_approx(x.y);
            }
            pk[i] = pack_bf16x2(e.x, e.y);
            sr[k] = __float_as_uint(e.x);
            sr[k + 1] = __float_as_uint(e.y);
          }
          tmem_st16(tS + c * 16, pk);
          if (c == 1 && r == 0) ATTN_EVT(ej, slot * 8 + 6);
        }
        if (r == 0) ATTN_TRACE_AT(2 + slot, 3, j);
        tmem_wait_st();
        if (r == 0) ATTN_EVT(ej, slot * 8 + 7);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[slot]);  // one arrival per warp
        if (r == 0) ATTN_EVT(ej, slot * 8 + 4);
        {
          float2 a0 = make_float2(0.f, 0.f), a1 = a0, a2 = a0, a3 = a0;
#pragma unroll
          for (int k = 0; k < 128; k += 8) {
            a0 = add2(a0, make_float2(__uint_as_float(sr[k]), __uint_as_float(sr[k + 1])));
            a1 = add2(a1, make_float2(__uint_as_float(sr[k + 2]), __uint_as_float(sr[k + 3])));
            a2 = add2(a2, make_float2(__uint_as_float(sr[k + 4]), __uint_as_float(sr[k + 5])));
            a3 = add2(a3, make_float2(__uint_as_float(sr[k + 6]), __uint_as_float(sr[k + 7])));
          }
          a0 = add2(add2(a0, a1), add2(a2, a3));
          l += a0.x + a0.y;
        }
        if (r == 0) ATTN_EVT(ej, slot * 8 + 5);
      }
      if (!ok) break;
      // ---- epilogue: O / l -> global, LSE = ln2 * (m + log2 l).  O comes out of TMEM first and
      // o_empty lets the next item's first PV overwrite it while this warp normalises and stores.
      const int row = q_lo + r;
      const bool row_ok = it.active[slot] && row < it.S;
      uint32_t ov[D];
      if (n > 0) {
        if (r == 0) ATTN_TRACE_AT(4 + slot, 1, qi);
        if (!(ok = mbar_wait_warp<true>(o_full, qi & 1, SITE_PF_EPI_O))) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) tmem_ld32(tO + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&ov[c * 32]));
#pragma unroll
        for (int c = 0; c < D / 32; ++c) tmem_wait_ld_regs(*reinterpret_cast<uint32_t(*)[32]>(&ov[c * 32]));
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(o_empty);
        if (r == 0) ATTN_TRACE_AT(4 + slot, 2, qi);
      } else {
#pragma unroll
        for (int i = 0; i < D; ++i) ov[i] = 0u;
      }
      float inv_l = (l > 0.f) ? 1.f / l : 0.f;
      float lse = (l > 0.f) ? (m_used + log2f(l)) * 0.69314718055994531f : -INFINITY;
      const long long lse_idx = (it.lse_row0 + row) * p.Hq + it.head[slot];
      float w_old = 0.f;  // weight of the stored partial (accumulate)
      bool store = row_ok;
      if (p.accumulate && row_ok) {
        const float lse_old = p.lse[lse_idx];
        if (lse == -INFINITY) {
          store = false;  // no key of this chunk is visible: the stored partial stands
        } else if (lse_old != -INFINITY) {
          const float mx = fmaxf(lse_old, lse);
          const float e_old = expf(lse_old - mx), e_new = expf(lse - mx);
          const float inv = 1.f / (e_old + e_new);
          w_old = e_old * inv;
          inv_l *= e_new * inv;
          lse = mx + logf(e_old + e_new);
        }
      }
      if (store) {
        const long long orow = it.o_base + (long long)row * p.o_ss + (long long)it.head[slot] * p.o_sh;
        if (p.o_f32) {
          float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.o) + orow);
#pragma unroll
          for (int i = 0; i < D / 4; ++i) {
            float4 v = make_float4(__uint_as_float(ov[4 * i]) * inv_l, __uint_as_float(ov[4 * i + 1]) * inv_l,
                                   __uint_as_float(ov[4 * i + 2]) * inv_l, __uint_as_float(ov[4 * i + 3]) * inv_l);
            if (w_old != 0.f) {  // the stored partial is read only when it has a weight
              const float4 old = dst[i];
              v.x = fmaf(w_old, old.x, v.x);
              v.y = fmaf(w_old, old.y, v.y);
              v.z = fmaf(w_old, old.z, v.z);
              v.w = fmaf(w_old, old.w, v.w);
            }
            st_global_cs_v4f(dst + i, v);
          }
        } else {
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.o) + orow);
#pragma unroll
          for (int i = 0; i < D / 8; ++i) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(ov[8 * i + 0]) * inv_l, __uint_as_float(ov[8 * i + 1]) * inv_l);
            w.y = pack_bf16x2(__uint_as_float(ov[8 * i + 2]) * inv_l, __uint_as_float(ov[8 * i + 3]) * inv_l);
            w.z = pack_bf16x2(__uint_as_float(ov[8 * i + 4]) * inv_l, __uint_as_float(ov[8 * i + 5]) * inv_l);
            w.w = pack_bf16x2(__uint_as_float(ov[8 * i + 6]) * inv_l, __uint_as_float(ov[8 * i + 7]) * inv_l);
            st_global_cs_v4(dst + i, w);
          }
        }
        if (p.lse) p.lse[lse_idx] = lse;
      }
      if (n > 0) {
        g += n;
        ++qi;
      }
    }
  }
  tc_fence_before();
  if (threadIdx.x == 0) ATTN_TRACE_AT(6, 1, 0);
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
    if (lane == 0) ATTN_TRACE_AT(6, 2, 0);
  }
}

}  // namespace attn
