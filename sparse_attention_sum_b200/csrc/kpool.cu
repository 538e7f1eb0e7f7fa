// S6 / S7 — the kpool variant of the indexer (metrale glm5next_dsa_ref:
// layer_norm, pool_states, kept_pools, expand_selection and the module
// invariants).
//
// pool_states: one warp per pool.  Each of the kpool key rows is LayerNorm-ed
// (k_norm: subtract the mean, divide by the standard deviation, then w*x + b)
// with warp reductions; the gate softmax runs over the slot axis separately for
// each channel; lanes own channels.  Pooling starts at the first valid token
// and only complete pools exist; pooled rows past n_pools are zero-filled.
//
// expand_selection: one block per query row.  A block scan over the selected
// pool ids gives each valid pool its output slot, so pools keep rank order and
// their tokens are written ascending; the visible tail and the INVALID fill
// follow.  Every row is written for its full out_width.
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {

constexpr int kPoolMaxC = 8;  // D_I <= 256

template <typename T>
__global__ void pool_states_kernel(dsa_dims d, const T* __restrict__ k, const T* __restrict__ gate,
                                   const float* __restrict__ ln_w, const float* __restrict__ ln_b,
                                   float eps, const int32_t* __restrict__ kv_start,
                                   const int32_t* __restrict__ kv_len, T* __restrict__ pooled,
                                   int32_t* __restrict__ n_pools) {
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int pool = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int D = d.idx_dim, kp = d.kpool, S = d.n_kv;
  const int P = S / kp;
  const int f = kv_start[b];
  const int np = kv_len[b] > f ? (kv_len[b] - f) / kp : 0;
  if (pool == 0 && lane == 0) n_pools[b] = np;
  if (pool >= P) return;
  T* out = pooled + ((size_t)b * P + pool) * D;
  if (pool >= np) {
    for (int c = lane; c < D; c += 32) out[c] = from_f32<T>(0.f);
    return;
  }
  float num[kPoolMaxC], den[kPoolMaxC], gmax[kPoolMaxC];
#pragma unroll
  for (int c = 0; c < kPoolMaxC; ++c) {
    num[c] = 0.f;
    den[c] = 0.f;
    gmax[c] = -INFINITY;
  }
  const size_t tok0 = (size_t)b * S + f + (size_t)pool * kp;
  // per-channel max of the gate over the slots (softmax stabiliser)
  for (int r = 0; r < kp; ++r) {
    const T* g = gate + (tok0 + r) * D;
#pragma unroll
    for (int c = 0; c < kPoolMaxC; ++c)
      if (c * 32 + lane < D) gmax[c] = fmaxf(gmax[c], to_f32(g[c * 32 + lane]));
  }
  for (int r = 0; r < kp; ++r) {
    const T* kr = k + (tok0 + r) * D;
    const T* g = gate + (tok0 + r) * D;
    float x[kPoolMaxC];
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < kPoolMaxC; ++c) {
      x[c] = c * 32 + lane < D ? to_f32(kr[c * 32 + lane]) : 0.f;
      s += x[c];
    }
    const float mean = warp_sum(s) / (float)D;
    float s2 = 0.f;
#pragma unroll
    for (int c = 0; c < kPoolMaxC; ++c) {
      float dx = c * 32 + lane < D ? x[c] - mean : 0.f;
      s2 = fmaf(dx, dx, s2);
    }
    const float inv_std = 1.f / sqrtf(warp_sum(s2) / (float)D + eps);
#pragma unroll
    for (int c = 0; c < kPoolMaxC; ++c) {
      const int cc = c * 32 + lane;
      if (cc < D) {
        float kn = (x[c] - mean) * inv_std;
        if (ln_w) kn *= ln_w[cc];
        if (ln_b) kn += ln_b[cc];
        const float e = expf(to_f32(g[cc]) - gmax[c]);
        den[c] += e;
        num[c] = fmaf(e, kn, num[c]);
      }
    }
  }
#pragma unroll
  for (int c = 0; c < kPoolMaxC; ++c)
    if (c * 32 + lane < D) out[c * 32 + lane] = from_f32<T>(num[c] / den[c]);
}

cudaError_t launch_pool_states(const dsa_dims& d, const void* k, const void* gate,
                               const float* ln_w, const float* ln_b, float eps,
                               const int32_t* kv_start, const int32_t* kv_len, void* pooled,
                               int32_t* n_pools, cudaStream_t st) {
  const int P = d.n_kv / d.kpool;
  const int warps = 8;
  dim3 grid((P + warps - 1) / warps > 0 ? (P + warps - 1) / warps : 1, d.batch);
  if (d.dtype == DSA_F32)
    pool_states_kernel<float><<<grid, warps * 32, 0, st>>>(d, (const float*)k, (const float*)gate,
                                                           ln_w, ln_b, eps, kv_start, kv_len,
                                                           (float*)pooled, n_pools);
  else
    pool_states_kernel<bf16><<<grid, warps * 32, 0, st>>>(d, (const bf16*)k, (const bf16*)gate,
                                                          ln_w, ln_b, eps, kv_start, kv_len,
                                                          (bf16*)pooled, n_pools);
  return cudaGetLastError();
}

constexpr int kExpandThreads = 256;

__global__ void __launch_bounds__(kExpandThreads)
expand_selection_kernel(dsa_dims d, const int32_t* __restrict__ pool_idx,
                        const int32_t* __restrict__ q_pos, const int32_t* __restrict__ kv_start,
                        const int32_t* __restrict__ kv_len, const int32_t* __restrict__ n_pools,
                        int32_t* __restrict__ tok_idx) {
  __shared__ int scan[kExpandThreads / 32];
  __shared__ int s_base;
  const int b = blockIdx.y, t = blockIdx.x;
  const size_t row = (size_t)b * d.n_q + t;
  const int W = d.out_width, K = d.top_k, kp = d.kpool;
  const int f = kv_start[b], p = q_pos[row], np = n_pools[b];
  int32_t* orow = tok_idx + row * W;
  const int32_t* prow = pool_idx + row * K;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  if (p < f) {  // padded query row: all INVALID
    for (int i = threadIdx.x; i < W; i += blockDim.x) orow[i] = DSA_INVALID;
    return;
  }
  if (threadIdx.x == 0) s_base = 0;
  __syncthreads();
  for (int e0 = 0; e0 < K; e0 += blockDim.x) {
    const int e = e0 + threadIdx.x;
    int pid = e < K ? prow[e] : -1;
    bool ok = pid >= 0 && pid < np;
    uint32_t m = __ballot_sync(0xffffffffu, ok);
    if (lane == 0) scan[warp] = __popc(m);
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < kExpandThreads / 32; ++w) {
      if (w < warp) before += scan[w];
      total += scan[w];
    }
    const int base = s_base;
    if (ok) {
      int slot = base + before + __popc(m & ((1u << lane) - 1u));
      for (int j = 0; j < kp; ++j) orow[slot * kp + j] = f + pid * kp + j;
    }
    __syncthreads();
    if (threadIdx.x == 0) s_base = base + total;
    __syncthreads();
  }
  const int filled = s_base * kp;
  int nvis = (p - f + 1) / kp;
  if (nvis > np) nvis = np;
  int last = p < kv_len[b] - 1 ? p : kv_len[b] - 1;
  const int tail0 = f + nvis * kp;
  int ntail = last >= tail0 ? last - tail0 + 1 : 0;
  if (ntail > W - filled) ntail = W - filled;  // only reachable with an inconsistent n_pools
  for (int i = threadIdx.x; i < ntail; i += blockDim.x) orow[filled + i] = tail0 + i;
  for (int i = filled + ntail + threadIdx.x; i < W; i += blockDim.x) orow[i] = DSA_INVALID;
}

cudaError_t launch_expand_selection(const dsa_dims& d, const int32_t* pool_idx,
                                    const int32_t* q_pos, const int32_t* kv_start,
                                    const int32_t* kv_len, const int32_t* n_pools,
                                    int32_t* tok_idx, cudaStream_t st) {
  dim3 grid(d.n_q, d.batch);
  expand_selection_kernel<<<grid, kExpandThreads, 0, st>>>(d, pool_idx, q_pos, kv_start, kv_len,
                                                           n_pools, tok_idx);
  return cudaGetLastError();
}

}  // namespace dsa
