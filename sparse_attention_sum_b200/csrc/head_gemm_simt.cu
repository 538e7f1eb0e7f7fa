// S8 — per-head GEMMs of the absorbed NoPE MLA on the CUDA cores.
//
// C[n,h,:] = A[n,h,:] x B[h] with bf16 operands, fp32 accumulation and a bf16
// result (metrale glm5next_dsa_ref expand_kv: K_h = W_UK,h c and V_h = W_UV,h c;
// absorbing W_UK into the query and W_UV into the output gives the same
// attention over the latent).  A 64x64 output tile per block, 16-deep K slices
// staged in shared memory, 4x4 outputs per thread.
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {

constexpr int kGT = 64, kGK = 16;

__global__ void __launch_bounds__(256)
head_gemm_simt_kernel(int n_rows, int H, int K, int N, const bf16* __restrict__ A,
                      const bf16* __restrict__ Bm, bool b_kn, bf16* __restrict__ C) {
  __shared__ float As[kGK][kGT + 4];
  __shared__ float Bs[kGK][kGT + 4];
  const int h = blockIdx.z;
  const int m0 = blockIdx.y * kGT, n0 = blockIdx.x * kGT;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += kGK) {
    for (int i = threadIdx.x; i < kGK * kGT; i += 256) {
      // A tile: element (m, kk) -> As[kk][m]
      int m = i / kGK, kk = i % kGK;
      int gm = m0 + m, gk = k0 + kk;
      As[kk][m] = (gm < n_rows && gk < K) ? __bfloat162float(A[((size_t)gm * H + h) * K + gk]) : 0.f;
      // B tile: element (kk, nn) -> Bs[kk][nn]
      int kk2 = i / kGT, nn = i % kGT;
      int gk2 = k0 + kk2, gn = n0 + nn;
      float bv = 0.f;
      if (gk2 < K && gn < N)
        bv = __bfloat162float(b_kn ? Bm[((size_t)h * K + gk2) * N + gn] : Bm[((size_t)h * N + gn) * K + gk2]);
      Bs[kk2][nn] = bv;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kGK; ++kk) {
      float a[4], bb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bb[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int gm = m0 + ty * 4 + i;
    if (gm >= n_rows) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int gn = n0 + tx * 4 + j;
      if (gn < N) C[((size_t)gm * H + h) * N + gn] = __float2bfloat16_rn(acc[i][j]);
    }
  }
}

cudaError_t launch_head_gemm(int n_rows, int heads, int K, int N, const void* A, const void* Bm,
                             bool b_kn, void* C, cudaStream_t st) {
  dim3 grid((N + kGT - 1) / kGT, (n_rows + kGT - 1) / kGT, heads);
  head_gemm_simt_kernel<<<grid, 256, 0, st>>>(n_rows, heads, K, N, (const bf16*)A, (const bf16*)Bm,
                                               b_kn, (bf16*)C);
  return cudaGetLastError();
}

}  // namespace dsa
