// The indexer's head reduction, shared by the tensor-core indexer and the fused indexer/top-k so
// that both produce the same bits for the same accumulators.
//
// sum_h w_h * relu(c_h * dot_h) with c_h = scale * (per-head scale, 1 without FP8).  The per-head
// scales are positive, so relu(c_h * x) = |c_h| * relu(sign(scale) * x): the weight w_h * |c_h| is
// folded once per query tile (wsc) and each accumulator column costs one max and one fma.
#pragma once
#include <stdint.h>

namespace dsa {

// Weighted relu sum of 32 accumulator columns v (fp32 bits) with folded weights wsc[0..31]
// (16-byte aligned shared memory), in four interleaved partial sums combined in a fixed order.
template <bool kNeg>
__device__ __forceinline__ float head_sum32(const uint32_t (&v)[32], const float* wsc) {
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    const float4 c = *reinterpret_cast<const float4*>(wsc + j);
    const float x0 = __uint_as_float(v[j]), x1 = __uint_as_float(v[j + 1]);
    const float x2 = __uint_as_float(v[j + 2]), x3 = __uint_as_float(v[j + 3]);
    s0 = fmaf(c.x, fmaxf(kNeg ? -x0 : x0, 0.f), s0);
    s1 = fmaf(c.y, fmaxf(kNeg ? -x1 : x1, 0.f), s1);
    s2 = fmaf(c.z, fmaxf(kNeg ? -x2 : x2, 0.f), s2);
    s3 = fmaf(c.w, fmaxf(kNeg ? -x3 : x3, 0.f), s3);
  }
  return (s0 + s1) + (s2 + s3);
}

}  // namespace dsa
