// dsa_layer_forward_static: the fused layer without any caller workspace.
//
// Some callers cannot allocate device memory at the point where they run the
// layer: a serving engine that plans every buffer up front and forbids
// allocation on its decode path, code that runs inside an allocator callback
// or an allocator-less embedding of the CUDA runtime, or a runtime whose only
// device memory is what it was handed at start-up.  For them this entry point
// takes the fused layer's scratch (the fp32 score matrix and the int32 index
// rows) from one fixed array that lives in the library's own device memory.
//
// The array is a file-scope __device__ variable of kStaticScratchBytes bytes.
// Every GPU that loads the library holds it until the process exits.  Its name
// in host code is only a host-side stand-in, so the device address is fetched
// with cudaGetSymbolAddress once per device (on the first call made with that
// device current) and cached together with the context it was read in; that
// first call should therefore happen before any stream capture.  After a
// cudaDeviceReset the device's new context has its own copy of the array, so
// the next call looks the address up again (make that call outside a capture
// too).  All calls share the array and it keeps the last call's
// contents: calls whose work overlaps on the GPU (on different streams, or on
// different host threads) race on it.  Nothing in the array has to start at
// zero: the index-score kernel writes every score of the rows it covers and
// the top-k kernel writes every index slot before either is read.
#include <cuda_runtime.h>

#include <mutex>

#include "dsa.h"
#include "dsa_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = 16u << 20;  // 16 MiB

__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

void* scratch_address(cudaError_t* err) {
  static std::mutex mu;
  static void* ctxs[128] = {};
  static void* ptrs[128] = {};
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= 128) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  void* ctx = dsa::current_context();
  std::lock_guard<std::mutex> lock(mu);
  if (ptrs[dev] && ctx && ctxs[dev] == ctx) return ptrs[dev];
  void* p = nullptr;
  *err = cudaGetSymbolAddress(&p, g_static_scratch);
  if (*err != cudaSuccess) return nullptr;
  ctxs[dev] = dsa::current_context();  // the lookup binds the primary context if none was current
  ptrs[dev] = p;
  return p;
}

}  // namespace

extern "C" dsa_status dsa_layer_forward_static(const dsa_dims* dims, const void* q_idx, const void* k_idx,
                                               const float* w, float idx_scale, const int32_t* q_pos,
                                               const int32_t* kv_start, const int32_t* kv_len, const void* q,
                                               const void* k, int64_t k_row_stride, const void* v,
                                               int64_t v_row_stride, float attn_scale, const int32_t* idx_in,
                                               int32_t* idx_out, void* out, float* lse, dsa_stream_t stream) {
  if (dims == nullptr) {
    dsa::set_last_error("dsa_layer_forward_static: dims is NULL");
    return DSA_ERR_INVALID_ARGUMENT;
  }
  const size_t need = idx_in ? 0 : dsa_workspace_size(dims, DSA_OP_LAYER_FORWARD);
  if (!idx_in && need == 0) {
    dsa::set_last_error("dsa_layer_forward_static: invalid dims (batch, n_q, n_kv and top_k must be >= 1)");
    return DSA_ERR_INVALID_ARGUMENT;
  }
  if (need > kStaticScratchBytes) {
    dsa::set_last_error(
        "dsa_layer_forward_static: the layer needs more scratch than the fixed 16 MiB array holds "
        "(scores batch*n_q*n_kv*4 bytes plus index rows batch*n_q*top_k*4 bytes); use dsa_layer_forward "
        "with a caller workspace");
    return DSA_ERR_WORKSPACE;
  }
  cudaError_t err = cudaSuccess;
  void* ws = scratch_address(&err);
  if (ws == nullptr) {
    dsa::set_last_error("dsa_layer_forward_static: cudaGetSymbolAddress of the scratch array failed");
    return DSA_ERR_CUDA;
  }
  return dsa_layer_forward(dims, q_idx, k_idx, w, idx_scale, q_pos, kv_start, kv_len, q, k, k_row_stride, v,
                           v_row_stride, attn_scale, idx_in, idx_out, out, lse, ws, kStaticScratchBytes, stream);
}
