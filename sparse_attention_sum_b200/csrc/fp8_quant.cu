// Per-vector e4m3 quantisation of the indexer operands (the FP8 indexer's input step).
//
// ik_llama.cpp PR #2063 ships the indexer tensors in F8_E4M3; the scaling is
// this library's reading: every vector of 128 values (a query head's q_idx row,
// a key's k_idx row) gets one fp32 scale s = amax / 448, and its codes are
// e4m3(x * fl(448 / amax)) with the reciprocal and the product rounded to fp32
// (round to nearest even everywhere, e4m3 saturating at 448).  A zero vector
// gets scale 1 and zero codes.  x ~= codes * s.
//
// One warp per vector: lane l holds values 4l..4l+3 (one 8- or 16-byte load),
// the amax is a warp maximum, and the lane writes its four codes as one 32-bit
// store, so a warp reads 256 (bf16) or 512 (fp32) contiguous bytes and writes
// 128.  Memory-bound: each vector is read once and its codes and scale written
// once.
#include <cuda_fp8.h>

#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {

namespace {

constexpr int kWarps = 8;

template <typename T>
__device__ __forceinline__ void load4(const T* p, float (&v)[4]);
template <>
__device__ __forceinline__ void load4<bf16>(const bf16* p, float (&v)[4]) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
  const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
  v[0] = __low2float(a);
  v[1] = __high2float(a);
  v[2] = __low2float(b);
  v[3] = __high2float(b);
}
template <>
__device__ __forceinline__ void load4<float>(const float* p, float (&v)[4]) {
  const float4 u = *reinterpret_cast<const float4*>(p);
  v[0] = u.x;
  v[1] = u.y;
  v[2] = u.z;
  v[3] = u.w;
}

template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
fp8_quantize_kernel(long long n, const T* __restrict__ x, long long stride, uint32_t* __restrict__ codes,
                    float* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * kWarps;
  for (long long r = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5); r < n; r += warps) {
    float v[4];
    load4<T>(x + r * stride + 4 * lane, v);
    float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
    amax = warp_max(amax);
    const float safe = amax > 0.f ? amax : 1.f;
    const float inv = __fdiv_rn(448.f, safe);
    const __nv_fp8x2_storage_t lo =
        __nv_cvt_float2_to_fp8x2(make_float2(__fmul_rn(v[0], inv), __fmul_rn(v[1], inv)), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t hi =
        __nv_cvt_float2_to_fp8x2(make_float2(__fmul_rn(v[2], inv), __fmul_rn(v[3], inv)), __NV_SATFINITE, __NV_E4M3);
    codes[r * 32 + lane] = (uint32_t)lo | ((uint32_t)hi << 16);
    if (lane == 0) scales[r] = amax > 0.f ? __fdiv_rn(safe, 448.f) : 1.f;
  }
}

}  // namespace

cudaError_t launch_fp8_quantize(long long n, bool in_bf16, const void* x, long long x_stride, void* codes,
                                float* scales, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  long long blocks = (n + kWarps - 1) / kWarps;
  const long long cap = (long long)sm_count() * 8;
  if (blocks > cap) blocks = cap;
  if (in_bf16)
    fp8_quantize_kernel<bf16><<<(unsigned)blocks, kWarps * 32, 0, st>>>(n, (const bf16*)x, x_stride,
                                                                         (uint32_t*)codes, scales);
  else
    fp8_quantize_kernel<float><<<(unsigned)blocks, kWarps * 32, 0, st>>>(n, (const float*)x, x_stride,
                                                                          (uint32_t*)codes, scales);
  return cudaGetLastError();
}

}  // namespace dsa
