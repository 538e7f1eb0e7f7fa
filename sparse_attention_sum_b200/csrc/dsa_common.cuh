// Device helpers shared by the DSA kernels: element access, visibility, keys.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "dsa.h"

namespace dsa {

typedef __nv_bfloat16 bf16;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(bf16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float x) { return __float2bfloat16_rn(x); }

// Visible key range [lo, hi] of one query row (empty when hi < lo).
//   token mode (kpool == 0): kv_start <= s <= min(q_pos, kv_len - 1), s < n_kv
//   pool mode  (kpool >= 1): pool j visible iff its last token
//                            kv_start + (j+1)*kpool - 1 <= q_pos and < kv_len
struct KeyRange {
  int lo, hi;
  __device__ __forceinline__ int count() const { return hi >= lo ? hi - lo + 1 : 0; }
};

__device__ __forceinline__ KeyRange visible_range(int q_pos, int kv_start, int kv_len, int n_kv,
                                                  int kpool) {
  KeyRange r;
  if (kpool <= 0) {
    r.lo = kv_start < 0 ? 0 : kv_start;
    int hi = q_pos;
    if (hi > kv_len - 1) hi = kv_len - 1;
    if (hi > n_kv - 1) hi = n_kv - 1;
    r.hi = hi;
  } else {
    r.lo = 0;
    if (q_pos < kv_start) {
      r.hi = -1;
    } else {
      int by_pos = (q_pos - kv_start + 1) / kpool;
      int by_len = kv_len > kv_start ? (kv_len - kv_start) / kpool : 0;
      int n = by_pos < by_len ? by_pos : by_len;
      if (n > n_kv) n = n_kv;
      r.hi = n - 1;
    }
  }
  return r;
}

// Order-preserving map of a finite fp32 score to uint32 (-0.0 and +0.0 map to
// the same key): larger score <=> larger key.
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7fffffffu) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_score(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(u);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ void record_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

}  // namespace dsa
