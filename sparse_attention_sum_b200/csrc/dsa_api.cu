// C ABI of libdsa: argument validation, workspace layout and kernel dispatch.
// Declarations and contracts: include/dsa.h.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

#include "dsa.h"
#include "dsa_internal.h"
#include "dsa_sm100.cuh"

namespace {

thread_local std::string g_last_error;

// Kernel families launched by the current top-level entry point call of this host thread
// (entry points that call other entry points record into the outer call's list).
thread_local std::string g_kernels;
thread_local int g_call_depth = 0;

struct CallScope {
  CallScope() {
    if (g_call_depth++ == 0) g_kernels.clear();
  }
  ~CallScope() { --g_call_depth; }
};

__device__ int g_device_status;  // DSA_ERR_TIMEOUT recorded by bounded device waits

dsa_status fail(dsa_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

dsa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(DSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

dsa_status ok() {
  g_last_error.clear();
  return DSA_OK;
}

bool dtype_ok(int32_t dt) { return dt == DSA_F32 || dt == DSA_BF16; }

#define REQUIRE(cond, ...)                                   \
  do {                                                       \
    if (!(cond)) return fail(DSA_ERR_INVALID_ARGUMENT, __VA_ARGS__); \
  } while (0)

dsa_status check_rows(const dsa_dims* d) {
  REQUIRE(d != nullptr, "dims is NULL");
  REQUIRE(d->batch >= 1 && d->batch <= 65535, "batch must be in [1, 65535] (got %d)", d->batch);
  REQUIRE(d->n_q >= 1 && d->n_q <= 2147483647 / 1, "n_q must be >= 1 (got %d)", d->n_q);
  REQUIRE(d->n_kv >= 1, "n_kv must be >= 1 (got %d)", d->n_kv);
  REQUIRE(d->kpool >= 0, "kpool must be >= 0 (got %d)", d->kpool);
  return DSA_OK;
}

dsa_status check_visibility(const int32_t* q_pos, const int32_t* kv_start, const int32_t* kv_len) {
  REQUIRE(q_pos && kv_start && kv_len, "q_pos, kv_start and kv_len must be non-NULL");
  return DSA_OK;
}

dsa_status check_index(const dsa_dims* d, const void* q_idx, const void* k_idx, const float* w,
                       float scale, float* scores) {
  dsa_status s = check_rows(d);
  if (s) return s;
  REQUIRE(dtype_ok(d->dtype), "dtype must be DSA_F32 or DSA_BF16 (got %d)", d->dtype);
  REQUIRE(d->idx_heads >= 1 && d->idx_dim >= 1, "idx_heads and idx_dim must be >= 1");
  REQUIRE(q_idx && k_idx && w && scores, "q_idx, k_idx, w and scores must be non-NULL");
  REQUIRE(scale == scale, "scale must not be NaN");
  REQUIRE(d->n_q <= 65535, "n_q must be <= 65535 for dsa_index_scores (got %d)", d->n_q);
  return DSA_OK;
}

dsa_status check_topk(const dsa_dims* d, const float* scores, int32_t k, int32_t* idx) {
  dsa_status s = check_rows(d);
  if (s) return s;
  REQUIRE(scores && idx, "scores and idx must be non-NULL");
  REQUIRE(k >= 1 && k <= 4096, "k must be in [1, 4096] (got %d)", k);
  REQUIRE(d->n_q <= 2147483647, "n_q too large");
  return DSA_OK;
}

dsa_status check_attend(const dsa_dims* d, const void* q, const void* k, int64_t ks, const void* v,
                        int64_t vs, const int32_t* idx, int32_t width, void* out) {
  dsa_status s = check_rows(d);
  if (s) return s;
  REQUIRE(dtype_ok(d->dtype), "dtype must be DSA_F32 or DSA_BF16 (got %d)", d->dtype);
  REQUIRE(q && k && v && idx && out, "q, k, v, idx and out must be non-NULL");
  REQUIRE(d->heads >= 1 && d->kv_heads >= 1 && d->heads % d->kv_heads == 0,
          "kv_heads must divide heads (heads=%d kv_heads=%d)", d->heads, d->kv_heads);
  REQUIRE(d->kd >= 1 && d->vd >= 1, "kd and vd must be >= 1");
  REQUIRE(width >= 1, "width must be >= 1 (got %d)", width);
  REQUIRE(ks >= (int64_t)d->kv_heads * d->kd, "k_row_stride (%lld) < kv_heads*kd", (long long)ks);
  REQUIRE(vs >= (int64_t)d->kv_heads * d->vd, "v_row_stride (%lld) < kv_heads*vd", (long long)vs);
  REQUIRE(d->n_q <= 65535, "n_q must be <= 65535 for dsa_sparse_attend (got %d)", d->n_q);
  return DSA_OK;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// 0: tensor-core kernels where the shape allows; 1: CUDA-core kernels only.  Read by every entry point,
// possibly from several host threads while another sets it.
std::atomic<int> g_policy{0};
bool tc_policy() { return g_policy.load(std::memory_order_relaxed) == 0; }

}  // namespace

namespace dsa {

void* current_context() {
  typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
  static std::atomic<CtxGetCurrentFn> fn{nullptr};
  CtxGetCurrentFn f = fn.load(std::memory_order_acquire);
  if (!f) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    f = (CtxGetCurrentFn)ptr;
    fn.store(f, std::memory_order_release);
  }
  CUcontext c = nullptr;
  return f(&c) == CUDA_SUCCESS ? (void*)c : nullptr;
}

int* device_status_ptr() {
  static std::mutex mu;
  static void* ctxs[128] = {};
  static int* ptrs[128] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return nullptr;
  void* ctx = current_context();
  std::lock_guard<std::mutex> lock(mu);
  if (ptrs[dev] && ctx && ctxs[dev] == ctx) return ptrs[dev];
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
  ctxs[dev] = current_context();  // the lookup binds the primary context if none was current
  ptrs[dev] = (int*)p;
  return ptrs[dev];
}

void note_kernel(const char* name) {
  if (!g_kernels.empty()) g_kernels += ',';
  g_kernels += name;
}

void set_last_error(const char* msg) { g_last_error = msg; }

int sm_count() {
  static std::atomic<int> cached[128];  // zero-initialised (static storage); several threads may fill a slot
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 128) return 148;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (!n) {
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

__global__ void wait_selftest_kernel(long long timeout_ns, int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    sm100::mbar_init(sm100::smem_u32(&bar), 1);
    sm100::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing ever arrives on this barrier: the bounded wait must expire
    bool done = sm100::mbar_wait(sm100::smem_u32(&bar), 0, status, &abort_flag,
                                 (unsigned long long)timeout_ns);
    if (done) record_status(status, DSA_ERR_INVALID_ARGUMENT);  // impossible: flag it
  }
}

cudaError_t launch_wait_selftest(long long timeout_ns, cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(timeout_ns, device_status_ptr());
  return cudaGetLastError();
}

}  // namespace dsa

extern "C" {

const char* dsa_status_string(dsa_status s) {
  switch (s) {
    case DSA_OK: return "DSA_OK";
    case DSA_ERR_INVALID_ARGUMENT: return "DSA_ERR_INVALID_ARGUMENT";
    case DSA_ERR_UNSUPPORTED: return "DSA_ERR_UNSUPPORTED";
    case DSA_ERR_WORKSPACE: return "DSA_ERR_WORKSPACE";
    case DSA_ERR_CUDA: return "DSA_ERR_CUDA";
    case DSA_ERR_TIMEOUT: return "DSA_ERR_TIMEOUT";
  }
  return "DSA_ERR_UNKNOWN";
}

const char* dsa_last_error(void) { return g_last_error.c_str(); }

const char* dsa_last_kernels(void) { return g_kernels.c_str(); }

const char* dsa_version(void) { return "libdsa 0.1 (sm_100a)"; }

/* Selects which kernels serve shapes both families support: 0 (default) picks
 * the tensor-core kernels, 1 forces the CUDA-core kernels (used to compare the
 * two families on the same inputs).  Returns the previous policy. */
int dsa_set_kernel_policy(int policy) {
  return g_policy.exchange(policy == 1 ? 1 : 0, std::memory_order_relaxed);
}

size_t dsa_workspace_size(const dsa_dims* d, int op) {
  if (!d || d->batch < 1 || d->n_q < 1 || d->n_kv < 1) return 0;
  if (op == DSA_OP_TOPK) return 0;
  if (op == DSA_OP_LAYER_FORWARD) {
    if (d->top_k < 1) return 0;
    size_t rows = (size_t)d->batch * d->n_q;
    return align256(rows * d->n_kv * sizeof(float)) + align256(rows * d->top_k * sizeof(int32_t));
  }
  return 0;
}

dsa_status dsa_index_scores(const dsa_dims* d, const void* q_idx, const void* k_idx, const float* w,
                            float scale, const int32_t* q_pos, const int32_t* kv_start,
                            const int32_t* kv_len, float* scores, dsa_stream_t stream) {
  CallScope scope;
  dsa_status s = check_index(d, q_idx, k_idx, w, scale, scores);
  if (s) return s;
  if ((s = check_visibility(q_pos, kv_start, kv_len))) return s;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  const bool tc = tc_policy() && dsa::index_scores_tc_supported(*d);
  if (tc) {
    e = dsa::launch_index_scores_tc(*d, q_idx, k_idx, w, scale, q_pos, kv_start, kv_len, scores, st);
  } else {
    if (d->idx_dim > 256 || (int64_t)d->idx_heads * d->idx_dim > 16384)
      return fail(DSA_ERR_UNSUPPORTED, "dsa_index_scores: idx_dim <= 256 and idx_heads*idx_dim <= 16384 required");
    e = dsa::launch_index_scores_simt(*d, q_idx, k_idx, w, scale, q_pos, kv_start, kv_len, scores, st);
  }
  if (e != cudaSuccess) return cuda_fail(e, "dsa_index_scores launch");
  dsa::note_kernel(tc ? "index_tc" : "index_simt");
  return ok();
}

dsa_status dsa_fp8_quantize(int64_t n_vectors, int32_t dim, dsa_dtype in_dtype, const void* x,
                            int64_t x_row_stride, void* codes, float* scales, dsa_stream_t stream) {
  CallScope scope;
  REQUIRE(n_vectors >= 0, "n_vectors must be >= 0 (got %lld)", (long long)n_vectors);
  REQUIRE(dtype_ok(in_dtype), "in_dtype must be DSA_F32 or DSA_BF16 (got %d)", (int)in_dtype);
  if (dim != 128) return fail(DSA_ERR_UNSUPPORTED, "dsa_fp8_quantize: dim must be 128 (got %d)", dim);
  if (n_vectors == 0) return ok();
  REQUIRE(x && codes && scales, "x, codes and scales must be non-NULL");
  REQUIRE(x_row_stride >= dim, "x_row_stride (%lld) must be >= dim", (long long)x_row_stride);
  const size_t esz = in_dtype == DSA_BF16 ? 2 : 4;
  REQUIRE(x_row_stride % 4 == 0 && (uintptr_t)x % (4 * esz) == 0,
          "x and its row stride must be aligned to 4 values");
  REQUIRE((uintptr_t)codes % 4 == 0, "codes must be 4-byte aligned");
  cudaError_t e = dsa::launch_fp8_quantize((long long)n_vectors, in_dtype == DSA_BF16, x, (long long)x_row_stride,
                                           codes, scales, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "dsa_fp8_quantize launch");
  dsa::note_kernel("fp8_quantize");
  return ok();
}

dsa_status dsa_index_scores_fp8(const dsa_dims* d, const void* q_codes, const float* q_scales, const void* k_codes,
                                const float* k_scales, const float* w, float scale, const int32_t* q_pos,
                                const int32_t* kv_start, const int32_t* kv_len, float* scores,
                                dsa_stream_t stream) {
  CallScope scope;
  dsa_status s = check_rows(d);
  if (s) return s;
  REQUIRE(d->idx_heads >= 1 && d->idx_dim >= 1, "idx_heads and idx_dim must be >= 1");
  REQUIRE(q_codes && q_scales && k_codes && k_scales && w && scores,
          "q_codes, q_scales, k_codes, k_scales, w and scores must be non-NULL");
  REQUIRE(scale == scale, "scale must not be NaN");
  REQUIRE(d->n_q <= 65535, "n_q must be <= 65535 for dsa_index_scores_fp8 (got %d)", d->n_q);
  if ((s = check_visibility(q_pos, kv_start, kv_len))) return s;
  REQUIRE(((uintptr_t)q_codes & 15u) == 0 && ((uintptr_t)k_codes & 15u) == 0, "codes must be 16-byte aligned");
  if (!dsa::index_scores_tc_supported(*d, true))
    return fail(DSA_ERR_UNSUPPORTED,
                "dsa_index_scores_fp8: idx_dim 128, idx_heads in {32, 64, 128} and batch*n_kv >= 128 required");
  cudaError_t e = dsa::launch_index_scores_tc(*d, q_codes, k_codes, w, scale, q_pos, kv_start, kv_len, scores,
                                              (cudaStream_t)stream, q_scales, k_scales);
  if (e != cudaSuccess) return cuda_fail(e, "dsa_index_scores_fp8 launch");
  dsa::note_kernel("index_tc_fp8");
  return ok();
}

dsa_status dsa_index_topk(const dsa_dims* d, const void* q_idx, const void* k_idx, const float* w, float scale,
                          const int32_t* q_pos, const int32_t* kv_start, const int32_t* kv_len, int32_t k,
                          int32_t* idx, dsa_stream_t stream) {
  CallScope scope;
  dsa_status s = check_index(d, q_idx, k_idx, w, scale, (float*)1);
  if (s) return s;
  if ((s = check_visibility(q_pos, kv_start, kv_len))) return s;
  REQUIRE(idx != nullptr, "idx must be non-NULL");
  REQUIRE(k >= 1 && k <= 4096, "k must be in [1, 4096] (got %d)", k);
  REQUIRE(d->kpool == 0, "dsa_index_topk: kpool must be 0 (got %d)", d->kpool);
  if (!dsa::index_topk_supported(*d, k))
    return fail(DSA_ERR_UNSUPPORTED,
                "dsa_index_topk: bf16, idx_dim 128, idx_heads in {32, 64, 128} and n_kv <= 131072 required");
  cudaError_t e = dsa::launch_index_topk(*d, q_idx, k_idx, w, scale, q_pos, kv_start, kv_len, k, idx,
                                         (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "dsa_index_topk launch");
  dsa::note_kernel("index_topk");
  return ok();
}

dsa_status dsa_index_topk_fp8(const dsa_dims* d, const void* q_codes, const float* q_scales, const void* k_codes,
                              const float* k_scales, const float* w, float scale, const int32_t* q_pos,
                              const int32_t* kv_start, const int32_t* kv_len, int32_t k, int32_t* idx,
                              dsa_stream_t stream) {
  CallScope scope;
  dsa_status s = check_rows(d);
  if (s) return s;
  REQUIRE(d->idx_heads >= 1 && d->idx_dim >= 1, "idx_heads and idx_dim must be >= 1");
  REQUIRE(q_codes && q_scales && k_codes && k_scales && w && idx,
          "q_codes, q_scales, k_codes, k_scales, w and idx must be non-NULL");
  REQUIRE(scale == scale, "scale must not be NaN");
  REQUIRE(d->n_q <= 65535, "n_q must be <= 65535 (got %d)", d->n_q);
  if ((s = check_visibility(q_pos, kv_start, kv_len))) return s;
  REQUIRE(k >= 1 && k <= 4096, "k must be in [1, 4096] (got %d)", k);
  REQUIRE(d->kpool == 0, "dsa_index_topk_fp8: kpool must be 0 (got %d)", d->kpool);
  REQUIRE(((uintptr_t)q_codes & 15u) == 0 && ((uintptr_t)k_codes & 15u) == 0, "codes must be 16-byte aligned");
  if (!dsa::index_topk_supported(*d, k, true))
    return fail(DSA_ERR_UNSUPPORTED, "dsa_index_topk_fp8: idx_dim 128, idx_heads in {32, 64, 128} and n_kv <= 131072 required");
  cudaError_t e = dsa::launch_index_topk(*d, q_codes, k_codes, w, scale, q_pos, kv_start, kv_len, k, idx,
                                         (cudaStream_t)stream, q_scales, k_scales);
  if (e != cudaSuccess) return cuda_fail(e, "dsa_index_topk_fp8 launch");
  dsa::note_kernel("index_topk_fp8");
  return ok();
}

namespace {
dsa_status topk_checked(const dsa_dims* d, const float* scores, const int32_t* q_pos, const int32_t* kv_start,
                        const int32_t* kv_len, int32_t k, int32_t* idx, float* vals, bool ranked,
                        dsa_stream_t stream) {
  if (d->batch > 65535) return fail(DSA_ERR_UNSUPPORTED, "dsa_topk: grid too large");
  cudaError_t e = dsa::launch_topk(*d, scores, q_pos, kv_start, kv_len, k, idx, vals, ranked, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "dsa_topk launch");
  dsa::note_kernel(ranked ? "topk_ranked" : "topk_set");
  return ok();
}
}  // namespace

dsa_status dsa_topk(const dsa_dims* d, const float* scores, const int32_t* q_pos,
                    const int32_t* kv_start, const int32_t* kv_len, int32_t k, int32_t* idx,
                    float* vals, void* ws, size_t ws_bytes, dsa_stream_t stream) {
  CallScope scope;
  (void)ws;
  dsa_status s = check_topk(d, scores, k, idx);
  if (s) return s;
  if ((s = check_visibility(q_pos, kv_start, kv_len))) return s;
  if (ws_bytes < dsa_workspace_size(d, DSA_OP_TOPK))
    return fail(DSA_ERR_WORKSPACE, "dsa_topk: workspace too small");
  return topk_checked(d, scores, q_pos, kv_start, kv_len, k, idx, vals, true, stream);
}

dsa_status dsa_topk_set(const dsa_dims* d, const float* scores, const int32_t* q_pos, const int32_t* kv_start,
                        const int32_t* kv_len, int32_t k, int32_t* idx, float* vals, dsa_stream_t stream) {
  CallScope scope;
  dsa_status s = check_topk(d, scores, k, idx);
  if (s) return s;
  if ((s = check_visibility(q_pos, kv_start, kv_len))) return s;
  return topk_checked(d, scores, q_pos, kv_start, kv_len, k, idx, vals, false, stream);
}

dsa_status dsa_sparse_attend(const dsa_dims* d, const void* q, const void* k, int64_t k_row_stride,
                             const void* v, int64_t v_row_stride, const int32_t* idx, int32_t width,
                             float scale, void* out, float* lse, dsa_stream_t stream) {
  CallScope scope;
  dsa_status s = check_attend(d, q, k, k_row_stride, v, v_row_stride, idx, width, out);
  if (s) return s;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  const bool tc = tc_policy() && dsa::attend_tc_supported(*d, k_row_stride, k, v, v_row_stride, width);
  if (tc) {
    e = dsa::launch_attend_tc(*d, q, k, k_row_stride, idx, width, scale, out, lse, st);
  } else {
    if (!dsa::attend_simt_supported(*d, width))
      return fail(DSA_ERR_UNSUPPORTED, "dsa_sparse_attend: kd, vd <= 1024 and width <= 16384 required");
    e = dsa::launch_attend_simt(*d, q, k, k_row_stride, v, v_row_stride, idx, width, scale, out, lse, st);
  }
  if (e != cudaSuccess) return cuda_fail(e, "dsa_sparse_attend launch");
  dsa::note_kernel(tc ? "attend_tc" : "attend_simt");
  return ok();
}

dsa_status dsa_layer_forward(const dsa_dims* d, const void* q_idx, const void* k_idx, const float* w,
                             float idx_scale, const int32_t* q_pos, const int32_t* kv_start,
                             const int32_t* kv_len, const void* q, const void* k,
                             int64_t k_row_stride, const void* v, int64_t v_row_stride,
                             float attn_scale, const int32_t* idx_in, int32_t* idx_out, void* out,
                             float* lse, void* ws, size_t ws_bytes, dsa_stream_t stream) {
  CallScope scope;
  dsa_status s = check_rows(d);
  if (s) return s;
  REQUIRE(d->kpool == 0, "dsa_layer_forward: kpool must be 0 (got %d)", d->kpool);
  REQUIRE(d->top_k >= 1 && d->top_k <= 4096, "top_k must be in [1, 4096] (got %d)", d->top_k);
  if ((s = check_attend(d, q, k, k_row_stride, v, v_row_stride, idx_in ? idx_in : (const int32_t*)1,
                        d->top_k, out)))
    return s;
  const int32_t* sel = idx_in;
  if (!idx_in) {
    if ((s = check_index(d, q_idx, k_idx, w, idx_scale, (float*)1))) return s;
    if ((s = check_visibility(q_pos, kv_start, kv_len))) return s;
    const size_t need = dsa_workspace_size(d, DSA_OP_LAYER_FORWARD);
    REQUIRE(ws != nullptr || need == 0, "workspace is NULL");
    if (ws_bytes < need)
      return fail(DSA_ERR_WORKSPACE, "dsa_layer_forward: workspace %zu < %zu bytes", ws_bytes, need);
    const size_t rows = (size_t)d->batch * d->n_q;
    float* scores = (float*)ws;
    int32_t* idx_ws = (int32_t*)((char*)ws + align256(rows * d->n_kv * sizeof(float)));
    int32_t* idx = idx_out ? idx_out : idx_ws;
    if (tc_policy() && d->n_q == 1 && dsa::index_topk_supported(*d, d->top_k)) {
      // one query per sequence (decode): the fused selection keeps each row's scores on chip
      if ((s = dsa_index_topk(d, q_idx, k_idx, w, idx_scale, q_pos, kv_start, kv_len, d->top_k, idx, stream)))
        return s;
    } else {
      if ((s = dsa_index_scores(d, q_idx, k_idx, w, idx_scale, q_pos, kv_start, kv_len, scores, stream)))
        return s;
      // the attention reads the selection as a set: same keys as dsa_topk, listed in key order
      if ((s = dsa_topk_set(d, scores, q_pos, kv_start, kv_len, d->top_k, idx, nullptr, stream))) return s;
    }
    sel = idx;
  }
  return dsa_sparse_attend(d, q, k, k_row_stride, v, v_row_stride, sel, d->top_k, attn_scale, out,
                           lse, stream);
}

dsa_status dsa_pool_states(const dsa_dims* d, const void* k, const void* gate, const float* ln_w,
                           const float* ln_b, float ln_eps, const int32_t* kv_start,
                           const int32_t* kv_len, void* pooled, int32_t* n_pools,
                           dsa_stream_t stream) {
  CallScope scope;
  REQUIRE(d != nullptr, "dims is NULL");
  REQUIRE(d->batch >= 1 && d->batch <= 65535, "batch must be in [1, 65535]");
  REQUIRE(d->kpool >= 1, "dsa_pool_states: kpool must be >= 1 (got %d)", d->kpool);
  REQUIRE(d->n_kv >= d->kpool, "n_kv must be >= kpool");
  REQUIRE(dtype_ok(d->dtype), "dtype must be DSA_F32 or DSA_BF16");
  REQUIRE(d->idx_dim >= 1, "idx_dim must be >= 1");
  REQUIRE(k && gate && pooled && n_pools && kv_start && kv_len, "array arguments must be non-NULL");
  REQUIRE(ln_eps > 0.f, "ln_eps must be > 0 (got %g)", (double)ln_eps);
  if (d->idx_dim > 256) return fail(DSA_ERR_UNSUPPORTED, "dsa_pool_states: idx_dim <= 256 required");
  cudaError_t e = dsa::launch_pool_states(*d, k, gate, ln_w, ln_b, ln_eps, kv_start, kv_len, pooled,
                                          n_pools, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "dsa_pool_states launch");
  dsa::note_kernel("pool_states");
  return ok();
}

dsa_status dsa_expand_selection(const dsa_dims* d, const int32_t* pool_idx, const int32_t* q_pos,
                                const int32_t* kv_start, const int32_t* kv_len,
                                const int32_t* n_pools, int32_t* tok_idx, dsa_stream_t stream) {
  CallScope scope;
  REQUIRE(d != nullptr, "dims is NULL");
  REQUIRE(d->batch >= 1 && d->batch <= 65535, "batch must be in [1, 65535]");
  REQUIRE(d->n_q >= 1 && d->n_q <= 2147483647, "n_q must be >= 1");
  REQUIRE(d->kpool >= 1, "dsa_expand_selection: kpool must be >= 1 (got %d)", d->kpool);
  REQUIRE(d->top_k >= 1, "top_k must be >= 1");
  REQUIRE((int64_t)d->out_width >= (int64_t)d->top_k * d->kpool + d->kpool - 1,
          "out_width (%d) must be >= top_k*kpool + kpool - 1", d->out_width);
  REQUIRE(pool_idx && q_pos && kv_start && kv_len && n_pools && tok_idx,
          "array arguments must be non-NULL");
  cudaError_t e = dsa::launch_expand_selection(*d, pool_idx, q_pos, kv_start, kv_len, n_pools,
                                               tok_idx, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "dsa_expand_selection launch");
  dsa::note_kernel("expand_selection");
  return ok();
}

dsa_status dsa_index_rotate(int32_t n_rows, int32_t heads, int32_t dim, int32_t n_rope, float rope_theta,
                            int32_t layer_norm, const float* ln_w, const float* ln_b, float ln_eps,
                            int32_t hadamard, const int32_t* pos, dsa_dtype in_dtype, const void* in,
                            int64_t in_row_stride, dsa_dtype out_dtype, void* out, int64_t out_row_stride,
                            const int32_t* out_rows, int64_t out_capacity, dsa_stream_t stream) {
  CallScope scope;
  REQUIRE(n_rows >= 0, "n_rows must be >= 0 (got %d)", n_rows);
  REQUIRE(heads >= 1, "heads must be >= 1 (got %d)", heads);
  REQUIRE(dim == 32 || dim == 64 || dim == 128, "dim must be 32, 64 or 128 (got %d)", dim);
  const int E = dim / 32;
  REQUIRE(n_rope >= 0 && n_rope <= dim && n_rope % 2 == 0 && (n_rope / 2) % E == 0,
          "n_rope must be even, in [0, dim], with n_rope/2 a multiple of dim/32 (got %d)", n_rope);
  REQUIRE(n_rope == 0 || (rope_theta > 0.f && rope_theta < INFINITY), "rope_theta must be finite and > 0");
  REQUIRE(!layer_norm || ln_eps > 0.f, "ln_eps must be > 0 (got %g)", (double)ln_eps);
  REQUIRE(dtype_ok(in_dtype) && dtype_ok(out_dtype), "dtypes must be DSA_F32 or DSA_BF16");
  if (n_rows == 0) return ok();
  REQUIRE(in && out, "in and out must be non-NULL");
  REQUIRE(n_rope == 0 || pos, "pos must be non-NULL when n_rope > 0");
  const int64_t row = (int64_t)heads * dim;
  REQUIRE(in_row_stride >= row && out_row_stride >= row, "row strides must be >= heads*dim (%lld)",
          (long long)row);
  REQUIRE(in_row_stride % E == 0 && out_row_stride % E == 0, "row strides must be multiples of dim/32");
  const size_t in_align = (size_t)E * (in_dtype == DSA_BF16 ? 2 : 4);
  const size_t out_align = (size_t)E * (out_dtype == DSA_BF16 ? 2 : 4);
  REQUIRE((uintptr_t)in % in_align == 0 && (uintptr_t)out % out_align == 0,
          "in and out must be aligned to dim/32 values");
  REQUIRE(out_capacity >= 0, "out_capacity must be >= 0");
  REQUIRE(out_rows || out_capacity >= n_rows, "out_capacity must be >= n_rows when out_rows is NULL");
  cudaError_t e = dsa::launch_index_rotate(n_rows, heads, dim, n_rope, rope_theta, layer_norm != 0, ln_w, ln_b,
                                           ln_eps, hadamard != 0, pos, in_dtype == DSA_BF16, in, in_row_stride,
                                           out_dtype == DSA_BF16, out, out_row_stride, out_rows, out_capacity,
                                           (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "dsa_index_rotate launch");
  dsa::note_kernel("index_rotate");
  return ok();
}

static dsa_status check_absorb(const dsa_dims* d, const void* a, int32_t K, const void* w, int32_t N,
                               void* c) {
  REQUIRE(d != nullptr, "dims is NULL");
  REQUIRE(d->batch >= 1 && d->n_q >= 1 && d->heads >= 1, "batch, n_q and heads must be >= 1");
  REQUIRE(a && w && c, "array arguments must be non-NULL");
  REQUIRE(K >= 1 && N >= 1, "widths must be >= 1");
  if (d->dtype != DSA_BF16) return fail(DSA_ERR_UNSUPPORTED, "absorption is implemented for bf16 only");
  const int64_t rows = (int64_t)d->batch * d->n_q;
  REQUIRE(rows <= 65535LL * 64, "too many query rows");
  return DSA_OK;
}

dsa_status dsa_absorb_q(const dsa_dims* d, const void* q, int32_t dq, const void* w_uk, int32_t L,
                        void* q_lat, dsa_stream_t stream) {
  CallScope scope;
  dsa_status s = check_absorb(d, q, dq, w_uk, L, q_lat);
  if (s) return s;
  const int rows = d->batch * d->n_q;
  const bool tc = tc_policy() && dsa::head_gemm_tc_supported(rows, d->heads, dq, L, q, w_uk, true, q_lat);
  cudaError_t e = tc ? dsa::launch_head_gemm_tc(rows, d->heads, dq, L, q, w_uk, true, q_lat, (cudaStream_t)stream)
                     : dsa::launch_head_gemm(rows, d->heads, dq, L, q, w_uk, true, q_lat, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "dsa_absorb_q launch");
  dsa::note_kernel(tc ? "head_gemm_tc" : "head_gemm_simt");
  return ok();
}

dsa_status dsa_absorb_out(const dsa_dims* d, const void* o_lat, int32_t L, const void* w_uv,
                          int32_t dv, void* out, dsa_stream_t stream) {
  CallScope scope;
  dsa_status s = check_absorb(d, o_lat, L, w_uv, dv, out);
  if (s) return s;
  const int rows = d->batch * d->n_q;
  const bool tc = tc_policy() && dsa::head_gemm_tc_supported(rows, d->heads, L, dv, o_lat, w_uv, false, out);
  cudaError_t e = tc ? dsa::launch_head_gemm_tc(rows, d->heads, L, dv, o_lat, w_uv, false, out, (cudaStream_t)stream)
                     : dsa::launch_head_gemm(rows, d->heads, L, dv, o_lat, w_uv, false, out, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "dsa_absorb_out launch");
  dsa::note_kernel(tc ? "head_gemm_tc" : "head_gemm_simt");
  return ok();
}

dsa_status dsa_get_device_status(dsa_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "dsa_get_device_status: stream synchronize");
  int* p = dsa::device_status_ptr();
  if (!p) return fail(DSA_ERR_CUDA, "dsa_get_device_status: no status word on this device");
  int v = 0;
  e = cudaMemcpy(&v, p, sizeof v, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "dsa_get_device_status: read");
  int zero = 0;
  e = cudaMemcpy(p, &zero, sizeof zero, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "dsa_get_device_status: clear");
  if (v != 0) return fail((dsa_status)v, "device reported %s", dsa_status_string((dsa_status)v));
  return ok();
}

dsa_status dsa_selftest_wait_timeout(int64_t timeout_ns, dsa_stream_t stream) {
  CallScope scope;
  REQUIRE(timeout_ns >= 1000 && timeout_ns <= 10000000000LL, "timeout_ns must be in [1e3, 1e10]");
  cudaError_t e = dsa::launch_wait_selftest((long long)timeout_ns, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "dsa_selftest_wait_timeout launch");
  dsa::note_kernel("wait_selftest");
  return ok();
}

}  // extern "C"
