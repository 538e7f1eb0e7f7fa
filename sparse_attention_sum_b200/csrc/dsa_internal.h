// Host-side launchers of the DSA kernels (internal to libdsa; not part of the C ABI).
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "dsa.h"

namespace dsa {

// The current driver context (CUcontext) of the calling thread, or NULL.  Device addresses
// of __device__ variables are cached together with it: after a cudaDeviceReset the device's
// new context holds fresh copies of those variables at other addresses.
void* current_context();

// Records that the current entry point call launched kernel family `name`
// (returned by dsa_last_kernels).
void note_kernel(const char* name);

// Device address of the status word on the current device (bounded waits
// record DSA_ERR_TIMEOUT there).
int* device_status_ptr();

// Number of SMs of the current device.
int sm_count();

// Sets the message dsa_last_error() returns on this host thread.
void set_last_error(const char* msg);

// S2 on the CUDA cores (any D_I <= 256, H_I*D_I <= 16384), fp32 or bf16 inputs.
cudaError_t launch_index_scores_simt(const dsa_dims& d, const void* q_idx, const void* k_idx,
                                     const float* w, float scale, const int32_t* q_pos,
                                     const int32_t* kv_start, const int32_t* kv_len, float* scores,
                                     cudaStream_t st);
// S2 on the tensor cores (tcgen05, D_I == 128, H_I in {32,64,128}): bf16 operands, or e4m3
// codes with per-vector scales (f8; q_scale/k_scale non-NULL at launch).
bool index_scores_tc_supported(const dsa_dims& d, bool f8 = false);
cudaError_t launch_index_scores_tc(const dsa_dims& d, const void* q_idx, const void* k_idx,
                                   const float* w, float scale, const int32_t* q_pos,
                                   const int32_t* kv_start, const int32_t* kv_len, float* scores,
                                   cudaStream_t st, const float* q_scale = nullptr,
                                   const float* k_scale = nullptr);

// Per-vector e4m3 quantisation of n rows of 128 values (bf16 or fp32, row stride in elements):
// codes [n,128] bytes, scales [n] fp32.
cudaError_t launch_fp8_quantize(long long n, bool in_bf16, const void* x, long long x_stride, void* codes,
                                float* scales, cudaStream_t st);

// S2 + S3 fused (bf16, D_I == 128, H_I in {32,64,128}, n_kv <= 8 * 16384): one cluster per query
// row, scores kept in shared memory; writes the selection in ascending key order (dsa_topk_set's form).
// f8: e4m3 codes with per-vector scales (q_scale/k_scale non-NULL at launch).
bool index_topk_supported(const dsa_dims& d, int k, bool f8 = false);
cudaError_t launch_index_topk(const dsa_dims& d, const void* q_idx, const void* k_idx, const float* w, float scale,
                              const int32_t* q_pos, const int32_t* kv_start, const int32_t* kv_len, int k,
                              int32_t* idx, cudaStream_t st, const float* q_scale = nullptr,
                              const float* k_scale = nullptr);

// S3 radix select, then a rank sort (ranked) or an ascending-key-order listing of
// the same selection (!ranked, the fused layer's set).
cudaError_t launch_topk(const dsa_dims& d, const float* scores, const int32_t* q_pos,
                        const int32_t* kv_start, const int32_t* kv_len, int k, int32_t* idx,
                        float* vals, bool ranked, cudaStream_t st);

// S4 on the CUDA cores (generic shapes).
bool attend_simt_supported(const dsa_dims& d, int width);
cudaError_t launch_attend_simt(const dsa_dims& d, const void* q, const void* k, int64_t k_stride,
                               const void* v, int64_t v_stride, const int32_t* idx, int width,
                               float scale, void* out, float* lse, cudaStream_t st);
// S4 on the tensor cores (tcgen05, bf16 shared latent).
bool attend_tc_supported(const dsa_dims& d, int64_t k_stride, const void* k, const void* v,
                         int64_t v_stride, int width);
cudaError_t launch_attend_tc(const dsa_dims& d, const void* q, const void* k, int64_t k_stride,
                             const int32_t* idx, int width, float scale, void* out, float* lse,
                             cudaStream_t st);

// S6 / S7.
cudaError_t launch_pool_states(const dsa_dims& d, const void* k, const void* gate,
                               const float* ln_w, const float* ln_b, float eps,
                               const int32_t* kv_start, const int32_t* kv_len, void* pooled,
                               int32_t* n_pools, cudaStream_t st);
cudaError_t launch_expand_selection(const dsa_dims& d, const int32_t* pool_idx,
                                    const int32_t* q_pos, const int32_t* kv_start,
                                    const int32_t* kv_len, const int32_t* n_pools,
                                    int32_t* tok_idx, cudaStream_t st);

// S8: batched per-head GEMM C[n,h,:] = A[n,h,:] x B[h] (bf16 in, fp32 accumulate, bf16 out).
//   b_kn = true:  B[h] is [K, N] (N contiguous)    (absorb_q: w_uk[h] is [d, L])
//   b_kn = false: B[h] is [N, K] (K contiguous)    (absorb_out: w_uv[h] is [e, L])
cudaError_t launch_head_gemm(int n_rows, int heads, int K, int N, const void* A, const void* Bm,
                             bool b_kn, void* C, cudaStream_t st);
// The same on tcgen05 (n_rows >= 128, K % 64 == 0, K <= 512, B[h] <= 128 KB, 16-byte aligned).
bool head_gemm_tc_supported(int n_rows, int heads, int K, int N, const void* A, const void* Bm, bool b_kn,
                            const void* C);
cudaError_t launch_head_gemm_tc(int n_rows, int heads, int K, int N, const void* A, const void* Bm, bool b_kn,
                                void* C, cudaStream_t st);

// Indexer query / key preparation: optional LayerNorm, NEOX RoPE of the first
// n_rope values, optional orthonormal Walsh-Hadamard rotation, store to row
// out_rows[r] (or r) when that row is in [0, out_cap).  dim in {32, 64, 128}.
cudaError_t launch_index_rotate(int n_rows, int heads, int dim, int n_rope, float theta, bool layer_norm,
                                const float* ln_w, const float* ln_b, float eps, bool hadamard,
                                const int32_t* pos, bool in_bf16, const void* in, int64_t in_stride,
                                bool out_bf16, void* out, int64_t out_stride, const int32_t* out_rows,
                                int64_t out_cap, cudaStream_t st);

// Bounded-wait self test.
cudaError_t launch_wait_selftest(long long timeout_ns, cudaStream_t st);

}  // namespace dsa
