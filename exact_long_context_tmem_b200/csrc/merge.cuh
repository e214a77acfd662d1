// Exact log-sum-exp merge of partial attention results (ONNX Runtime CPU GQA analysis,
// "Flash Decoding": the reduce phase merges the per-chunk partial softmax states; Stream-CQSA
// summary, "Methodology" 2-3: independent sub-results recombine into the full result).
//   lse = log sum_p exp(lse_p),  o = sum_p exp(lse_p - lse) * o_p
// Empty parts (lse_p = -inf) add nothing; a row whose parts are all empty gets o = 0, lse = -inf.
// One warp per row; each lane owns D/32 consecutive elements (vector loads of 16 or 8 bytes).
#pragma once

#include "ptx.cuh"

namespace attn {

struct MergeParams {
  const float* o_parts;    // [P, R, D]
  const float* lse_parts;  // [P, R]
  int P;
  long long R;
  void* o_out;  // [R, D] bf16 or f32
  int o_f32;
  float* lse_out;  // [R] or null
  int accumulate;  // (o_out f32, lse_out) hold a partial merged in place
};

template <int D>
__global__ void __launch_bounds__(256) merge_lse_kernel(const MergeParams p) {
  constexpr int V = D / 32;  // elements per lane
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= p.R) return;
  const float* own_o = p.accumulate ? reinterpret_cast<const float*>(p.o_out) + row * D : nullptr;
  const float own_lse = p.accumulate ? p.lse_out[row] : -INFINITY;

  float mx = own_lse;
  for (int q = lane; q < p.P; q += 32) mx = fmaxf(mx, p.lse_parts[(long long)q * p.R + row]);
  mx = warp_max(mx);
  float out_lse = -INFINITY;
  float acc[V];
#pragma unroll
  for (int i = 0; i < V; ++i) acc[i] = 0.f;
  if (mx != -INFINITY) {
    float sum = 0.f;
    for (int q = lane; q < p.P; q += 32) sum += expf(p.lse_parts[(long long)q * p.R + row] - mx);
    sum = warp_sum(sum);
    if (p.accumulate) sum += expf(own_lse - mx);
    out_lse = mx + logf(sum);
    const float inv = 1.f / sum;
    auto add_part = [&](const float* src, float lse_q) {
      const float w = expf(lse_q - mx) * inv;
      if (w == 0.f) return;
      if constexpr (V == 4) {
        const float4 x = reinterpret_cast<const float4*>(src)[lane];
        acc[0] += w * x.x; acc[1] += w * x.y; acc[2] += w * x.z; acc[3] += w * x.w;
      } else {
        const float2 x = reinterpret_cast<const float2*>(src)[lane];
        acc[0] += w * x.x; acc[1] += w * x.y;
      }
    };
    if (p.accumulate) add_part(own_o, own_lse);
    for (int q = 0; q < p.P; ++q) {
      const float lq = p.lse_parts[(long long)q * p.R + row];
      add_part(p.o_parts + ((long long)q * p.R + row) * D, lq);
    }
  }
  if (p.o_f32) {
    float* dst = reinterpret_cast<float*>(p.o_out) + row * D + lane * V;
#pragma unroll
    for (int i = 0; i < V; ++i) dst[i] = acc[i];
  } else {
    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.o_out) + row * D + lane * V;
    if constexpr (V == 4) {
      uint2 w;
      w.x = pack_bf16x2(acc[0], acc[1]);
      w.y = pack_bf16x2(acc[2], acc[3]);
      *reinterpret_cast<uint2*>(dst) = w;
    } else {
      *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0], acc[1]);
    }
  }
  if (p.lse_out && lane == 0) p.lse_out[row] = out_lse;
}

}  // namespace attn
