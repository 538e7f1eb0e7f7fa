// S4 sparse attention on the CUDA cores (any head layout; fp32 or bf16 inputs).
//
// For each (b,t,h): U = distinct in-range entries of idx[b,t,:] (INVALID and
// out-of-range entries dropped, duplicates collapsed: metrale glm5next_dsa_ref
// topk_to_mask), then out = sum_{i in U} softmax_i(scale*q.K_i) V_i with an
// online (running max / running sum) softmax (fak note "GLM-5.2: the DSA
// sparse attention moves onto the pure fak kernel", "What changed": one block
// per query head with an online softmax and separate key/value widths).
//
// One block per query row; the row's index set is deduplicated once in shared
// memory (a bitmap over the key range, or a pairwise scan for very long
// caches) and compacted in index-row order, then each warp runs the online
// softmax for one head at a time: lanes split the key and value widths, the
// dot product is a warp reduction.  Accumulation and softmax are fp32.
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {

constexpr int kAttSimtThreads = 256;
constexpr int kAttSimtMaxC = 32;          // kd, vd <= 32 * 32
constexpr int kAttBitmapMaxKeys = 131072; // bitmap dedupe up to this many keys (16 KB)

template <typename T>
__global__ void __launch_bounds__(kAttSimtThreads)
attend_simt_kernel(dsa_dims d, const T* __restrict__ q, const T* __restrict__ k, int64_t k_stride,
                   const T* __restrict__ v, int64_t v_stride, const int32_t* __restrict__ idx,
                   int width, float scale, T* __restrict__ out, float* __restrict__ lse) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  int* U = reinterpret_cast<int*>(smem_raw);                 // [width]
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(U + width); // [ceil(S/32)] when used
  __shared__ int scan[kAttSimtThreads / 32];
  __shared__ int s_count;

  const int b = blockIdx.y, t = blockIdx.x;
  const size_t row = (size_t)b * d.n_q + t;
  const int S = d.n_kv, H = d.heads, Hk = d.kv_heads, kd = d.kd, vd = d.vd;
  const int32_t* irow = idx + row * width;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool use_bitmap = S <= kAttBitmapMaxKeys;

  if (use_bitmap) {
    for (int i = threadIdx.x; i < (S + 31) / 32; i += blockDim.x) bitmap[i] = 0u;
    __syncthreads();
  }
  if (threadIdx.x == 0) s_count = 0;
  __syncthreads();
  // keep entry e iff it is in range and the first of its value to claim the key
  for (int e0 = 0; e0 < width; e0 += blockDim.x) {
    const int e = e0 + threadIdx.x;
    int key = -1;
    bool keep = false;
    if (e < width) {
      key = irow[e];
      if (key >= 0 && key < S) {
        if (use_bitmap) {
          uint32_t bit = 1u << (key & 31);
          keep = (atomicOr(&bitmap[key >> 5], bit) & bit) == 0u;
        } else {
          keep = true;
          for (int j = 0; j < e; ++j)
            if (irow[j] == key) { keep = false; break; }
        }
      }
    }
    // order-preserving compaction of this chunk
    uint32_t m = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) scan[warp] = __popc(m);
    __syncthreads();
    int base = s_count, before = 0, total = 0;
    for (int w = 0; w < kAttSimtThreads / 32; ++w) {
      if (w < warp) before += scan[w];
      total += scan[w];
    }
    if (keep) U[base + before + __popc(m & ((1u << lane) - 1u))] = key;
    __syncthreads();
    if (threadIdx.x == 0) s_count = base + total;
    __syncthreads();
  }
  const int nU = s_count;

  for (int h = warp; h < H; h += kAttSimtThreads / 32) {
    const int g = h / (H / Hk);
    const T* qh = q + (row * H + h) * (size_t)kd;
    float qr[kAttSimtMaxC];
#pragma unroll
    for (int c = 0; c < kAttSimtMaxC; ++c) {
      int dd = c * 32 + lane;
      qr[c] = dd < kd ? to_f32(qh[dd]) : 0.f;
    }
    float acc[kAttSimtMaxC];
#pragma unroll
    for (int c = 0; c < kAttSimtMaxC; ++c) acc[c] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;
    for (int j = 0; j < nU; ++j) {
      const size_t key_row = (size_t)b * S + U[j];
      const T* kr = k + key_row * k_stride + (size_t)g * kd;
      const T* vr = v + key_row * v_stride + (size_t)g * vd;
      float part = 0.f;
#pragma unroll
      for (int c = 0; c < kAttSimtMaxC; ++c) {
        int dd = c * 32 + lane;
        if (dd < kd) part = fmaf(qr[c], to_f32(kr[dd]), part);
      }
      const float z = scale * warp_sum(part);
      const float m_new = fmaxf(m_run, z);
      const float corr = expf(m_run - m_new);   // 0 on the first key (m_run = -inf)
      const float p = expf(z - m_new);
      l_run = l_run * corr + p;
#pragma unroll
      for (int c = 0; c < kAttSimtMaxC; ++c) {
        int dd = c * 32 + lane;
        if (dd < vd) acc[c] = fmaf(p, to_f32(vr[dd]), acc[c] * corr);
      }
      m_run = m_new;
    }
    T* oh = out + (row * H + h) * (size_t)vd;
    const float inv = nU > 0 ? 1.f / l_run : 0.f;
#pragma unroll
    for (int c = 0; c < kAttSimtMaxC; ++c) {
      int dd = c * 32 + lane;
      if (dd < vd) oh[dd] = from_f32<T>(acc[c] * inv);
    }
    if (lse && lane == 0) lse[row * H + h] = nU > 0 ? m_run + logf(l_run) : -INFINITY;
  }
}

bool attend_simt_supported(const dsa_dims& d, int width) {
  return d.kd <= 32 * kAttSimtMaxC && d.vd <= 32 * kAttSimtMaxC && width <= 16384;
}

cudaError_t launch_attend_simt(const dsa_dims& d, const void* q, const void* k, int64_t k_stride,
                               const void* v, int64_t v_stride, const int32_t* idx, int width,
                               float scale, void* out, float* lse, cudaStream_t st) {
  size_t smem = (size_t)width * 4;
  if (d.n_kv <= kAttBitmapMaxKeys) smem += (size_t)((d.n_kv + 31) / 32) * 4;
  dim3 grid(d.n_q, d.batch);
  if (d.dtype == DSA_F32) {
    auto kern = attend_simt_kernel<float>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kAttSimtThreads, smem, st>>>(d, (const float*)q, (const float*)k, k_stride,
                                              (const float*)v, v_stride, idx, width, scale,
                                              (float*)out, lse);
  } else {
    auto kern = attend_simt_kernel<bf16>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kAttSimtThreads, smem, st>>>(d, (const bf16*)q, (const bf16*)k, k_stride,
                                              (const bf16*)v, v_stride, idx, width, scale,
                                              (bf16*)out, lse);
  }
  return cudaGetLastError();
}

}  // namespace dsa
