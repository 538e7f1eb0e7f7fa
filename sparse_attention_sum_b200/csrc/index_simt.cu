// S2 lightning-indexer scores on the CUDA cores (fp32 accumulation).
//
// I[b,t,s] = sum_h w[b,t,h] * relu(scale * q[b,t,h,:] . k[b,s,:])  for visible s, -inf otherwise
// (fak note "GLM-5.2: the DSA sparse attention moves onto the pure fak kernel",
// section 3; metrale glm5next_dsa_ref index_scores).
//
// One block per (query row, 128-key tile).  The query's H_I x D_I block and
// its weights sit in shared memory (broadcast reads); each thread owns one key
// row, staged in shared memory with a one-float pad so that a warp reading
// the same column of 32 different rows hits 32 different banks.  This path
// serves fp32 inputs (where the tensor cores would round to tf32) and shapes
// the tensor-core kernel does not take.
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {

constexpr int kIdxSimtKeys = 128;

template <typename T>
__global__ void __launch_bounds__(kIdxSimtKeys)
index_scores_simt_kernel(dsa_dims d, const T* __restrict__ q_idx, const T* __restrict__ k_idx,
                         const float* __restrict__ w, float scale, const int32_t* __restrict__ q_pos,
                         const int32_t* __restrict__ kv_start, const int32_t* __restrict__ kv_len,
                         float* __restrict__ scores) {
  extern __shared__ float smem[];
  const int HI = d.idx_heads, DI = d.idx_dim, S = d.n_kv;
  const int b = blockIdx.z, t = blockIdx.y;
  const int s0 = blockIdx.x * kIdxSimtKeys;
  const int s = s0 + threadIdx.x;
  const size_t row = (size_t)b * d.n_q + t;
  float* out_row = scores + row * S;

  KeyRange r = visible_range(q_pos[row], kv_start[b], kv_len[b], S, d.kpool);
  int tile_hi = s0 + kIdxSimtKeys - 1;
  if (r.count() == 0 || r.hi < s0 || r.lo > tile_hi) {  // whole tile invisible
    if (s < S) out_row[s] = -INFINITY;
    return;
  }

  float* qs = smem;                 // [HI][DI]
  float* wsm = qs + HI * DI;        // [HI]
  float* ks = wsm + HI;             // [128][DI+1]
  const T* qrow = q_idx + row * HI * DI;
  for (int i = threadIdx.x; i < HI * DI; i += blockDim.x) qs[i] = to_f32(qrow[i]);
  for (int i = threadIdx.x; i < HI; i += blockDim.x) wsm[i] = w[row * HI + i];
  // stage the tile's key rows (coalesced: consecutive threads read consecutive elements)
  const T* kb = k_idx + (size_t)b * S * DI;
  for (int i = threadIdx.x; i < kIdxSimtKeys * DI; i += blockDim.x) {
    int kr = i / DI, c = i - kr * DI;
    int sk = s0 + kr;
    ks[kr * (DI + 1) + c] = sk < S ? to_f32(kb[(size_t)sk * DI + c]) : 0.f;
  }
  __syncthreads();
  if (s >= S) return;
  if (s < r.lo || s > r.hi) {
    out_row[s] = -INFINITY;
    return;
  }
  const float* kr = ks + threadIdx.x * (DI + 1);
  float acc = 0.f;
  for (int h = 0; h < HI; ++h) {
    const float* qh = qs + h * DI;
    float dot = 0.f;
    for (int c = 0; c < DI; ++c) dot = fmaf(qh[c], kr[c], dot);
    float v = fmaxf(scale * dot, 0.f);
    acc = fmaf(wsm[h], v, acc);
  }
  out_row[s] = acc + 0.0f == 0.0f ? 0.0f : acc;  // signed zero -> +0
}

cudaError_t launch_index_scores_simt(const dsa_dims& d, const void* q_idx, const void* k_idx,
                                     const float* w, float scale, const int32_t* q_pos,
                                     const int32_t* kv_start, const int32_t* kv_len, float* scores,
                                     cudaStream_t st) {
  size_t smem = sizeof(float) * ((size_t)d.idx_heads * d.idx_dim + d.idx_heads +
                                 (size_t)kIdxSimtKeys * (d.idx_dim + 1));
  dim3 grid((d.n_kv + kIdxSimtKeys - 1) / kIdxSimtKeys, d.n_q, d.batch);
  if (d.dtype == DSA_F32) {
    auto kern = index_scores_simt_kernel<float>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kIdxSimtKeys, smem, st>>>(d, (const float*)q_idx, (const float*)k_idx, w, scale,
                                           q_pos, kv_start, kv_len, scores);
  } else {
    auto kern = index_scores_simt_kernel<bf16>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kIdxSimtKeys, smem, st>>>(d, (const bf16*)q_idx, (const bf16*)k_idx, w, scale,
                                           q_pos, kv_start, kv_len, scores);
  }
  return cudaGetLastError();
}

}  // namespace dsa
