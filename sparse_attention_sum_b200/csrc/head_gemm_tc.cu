// S8 — per-head GEMMs of the absorbed NoPE MLA on the 5th-generation tensor cores.
//
// C[n,h,:] = A[n,h,:] x B[h]  (bf16 operands, fp32 accumulation in tensor memory,
// bf16 result; metrale glm5next_dsa_ref expand_kv: K_h = W_UK,h c and
// V_h = W_UV,h c, so absorbing W_UK into the query and W_UV into the output
// gives the same attention over the latent):
//   absorb_q:   A = q [n,H,128],     B[h] = w_uk[h] [128 x 512] (N contiguous: MN-major operand)
//   absorb_out: A = o_lat [n,H,512], B[h] = w_uv[h] [128 x 512] read as [N=128][K=512] (K-major)
//
// Both are HBM-bound (about 100 FLOP per byte): every A row and C row crosses
// HBM once.  A persistent CTA takes a contiguous range of (head, 128-row tile,
// N tile) items, so it loads a head's whole B (<= 128 KB) into shared memory
// once and reuses it for every row tile of that head.  Warp 0 streams A tiles
// (64 columns, 16 KB) by TMA through a 4-stage ring; warp 1 issues
// tcgen05.mma (M=128, N=NT<=256, K=16) into one of two TMEM accumulators;
// warps 2-5 drain the other accumulator through swizzled shared-memory boxes
// that TMA stores to global memory, so the epilogue of one tile overlaps the
// MMAs of the next.  Every wait is bounded.
#include <cuda.h>

#include "dsa_common.cuh"
#include "dsa_internal.h"
#include "dsa_sm100.cuh"

namespace dsa {
namespace {

using namespace sm100;

constexpr int kHgThreads = 192;
constexpr int kHgStages = 4;
constexpr int kHgABytes = 128 * 128;  // one A box: 128 rows x 64 bf16
constexpr int kHgMaxBBytes = 128 * 1024;
constexpr int kHgOutBox = 32 * 128;   // one output staging box: 32 rows x 64 bf16 (128-byte swizzle)

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"((uint64_t)map),
               "r"(src), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// wait until at most N committed bulk groups of this thread still read their shared memory
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

struct HgParams {
  int n_rows, H, K, N, NT;
  bool b_kn;
  bf16* C;
  int* status;
};

__global__ void __launch_bounds__(kHgThreads, 1)
head_gemm_tc_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                    const __grid_constant__ CUtensorMap map_c, HgParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t a_full[kHgStages], a_empty[kHgStages], b_full, b_free, d_full[2], d_empty[2];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sB = base;                          // B of the current head
  const uint32_t sA = base + kHgMaxBBytes;           // A ring
  const uint32_t sO = sA + kHgStages * kHgABytes;    // output staging: 4 warps x 2 boxes
  const int RT = (p.n_rows + 127) / 128, NTILES = p.N / p.NT;
  const long long total = (long long)p.H * RT * NTILES;
  const long long per = (total + gridDim.x - 1) / gridDim.x;
  const long long i0 = (long long)blockIdx.x * per, i1 = i0 + per < total ? i0 + per : total;
  const uint32_t b_bytes = (uint32_t)p.K * p.N * 2u;
  const int KC = p.K / 64;
  volatile int* abort_flag = &abort_flag_s;

  if (threadIdx.x == 0) {
    abort_flag_s = 0;
    for (int s = 0; s < kHgStages; ++s) {
      mbar_init(smem_u32(&a_full[s]), 1);
      mbar_init(smem_u32(&a_empty[s]), 1);
    }
    mbar_init(smem_u32(&b_full), 1);
    mbar_init(smem_u32(&b_free), 1);
    for (int d = 0; d < 2; ++d) {
      mbar_init(smem_u32(&d_full[d]), 1);
      mbar_init(smem_u32(&d_empty[d]), 4);
    }
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(&tmem_slot), 2 * p.NT);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&map_a);
      tma_prefetch_desc(&map_b);
      int cur_h = -1, nb = 0;
      long long na = 0;
      for (long long it = i0; it < i1; ++it) {
        const int h = (int)(it / ((long long)RT * NTILES));
        const int rt = (int)((it / NTILES) % RT);
        if (h != cur_h) {
          // the MMAs that read the previous head's B are complete
          if (nb > 0 && !mbar_wait(smem_u32(&b_free), (nb - 1) & 1, p.status, abort_flag)) break;
          mbar_arrive_expect_tx(smem_u32(&b_full), b_bytes);
          if (p.b_kn) {
            // w_uk[h]: [K rows][N cols]; one box per 64-column block: [K][64] (MN-major operand)
            for (int nbk = 0; nbk < p.N / 64; ++nbk)
              tma_load_2d(sB + nbk * p.K * 128, &map_b, smem_u32(&b_full), nbk * 64, h * p.K);
          } else {
            // w_uv[h]: [N rows][K cols]; one box per (N tile, 64-column K chunk): [NT][64] (K-major)
            for (int nt = 0; nt < NTILES; ++nt)
              for (int kc = 0; kc < KC; ++kc)
                tma_load_2d(sB + (nt * KC + kc) * p.NT * 128, &map_b, smem_u32(&b_full), kc * 64,
                            h * p.N + nt * p.NT);
          }
          cur_h = h;
          ++nb;
        }
        for (int kc = 0; kc < KC; ++kc, ++na) {
          const int s = (int)(na % kHgStages);
          if (!mbar_wait(smem_u32(&a_empty[s]), (uint32_t)(((na / kHgStages) & 1) ^ 1), p.status, abort_flag)) {
            it = i1;
            break;
          }
          mbar_arrive_expect_tx(smem_u32(&a_full[s]), kHgABytes);
          tma_load_2d(sA + s * kHgABytes, &map_a, smem_u32(&a_full[s]), h * p.K + kc * 64, rt * 128);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, p.NT, false, p.b_kn);
      int cur_h = -1, nb = 0;
      long long na = 0, nd = 0;
      bool ok = true;
      for (long long it = i0; ok && it < i1; ++it, ++nd) {
        const int h = (int)(it / ((long long)RT * NTILES));
        const int nt = (int)(it % NTILES);
        if (h != cur_h) {
          if (!(ok = mbar_wait(smem_u32(&b_full), nb & 1, p.status, abort_flag))) break;
          cur_h = h;
          ++nb;
        }
        const int d = (int)(nd & 1);
        if (!(ok = mbar_wait(smem_u32(&d_empty[d]), (uint32_t)(((nd >> 1) & 1) ^ 1), p.status, abort_flag))) break;
        tc_fence_after();
        const uint32_t dt = tmem + (uint32_t)(d * p.NT);
        for (int kc = 0; kc < KC; ++kc, ++na) {
          const int s = (int)(na % kHgStages);
          if (!(ok = mbar_wait(smem_u32(&a_full[s]), (uint32_t)((na / kHgStages) & 1), p.status, abort_flag))) break;
          tc_fence_after();
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint64_t ad = desc_sw128(sA + s * kHgABytes + j * 32);
            uint64_t bd;
            if (p.b_kn) {
              // MN-major B: 16 K-rows at (kc*4+j)*16; 64-column blocks are K*128 bytes apart
              bd = desc_sw128(sB + (nt * (p.NT / 64)) * p.K * 128 + (kc * 4 + j) * 16 * 128, 1024,
                              (uint32_t)p.K * 128u);
            } else {
              bd = desc_sw128(sB + (nt * KC + kc) * p.NT * 128 + j * 32);
            }
            mma_bf16_ss(dt, ad, bd, idesc, (kc | j) ? 1u : 0u);
          }
          mma_commit(smem_u32(&a_empty[s]));
        }
        if (!ok) break;
        mma_commit(smem_u32(&d_full[d]));
        // the next item starts another head (or there is none): B may be replaced once these MMAs end
        const bool last_of_head = it + 1 >= i1 || (int)((it + 1) / ((long long)RT * NTILES)) != h;
        if (last_of_head) mma_commit(smem_u32(&b_free));
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue: TMEM -> bf16 -> TMA store
    // Each warp converts its 32 rows, 64 columns at a time, into a 128-byte-swizzled staging box
    // and one lane stores the box by TMA (rows past n_rows are clipped by the store).
    const int q4 = warp & 3;                          // TMEM lane quarter of this warp
    const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
    const uint32_t stage0 = sO + (uint32_t)(q4 * 2 * kHgOutBox);
    long long nd = 0;
    int nbox = 0;
    for (long long it = i0; it < i1; ++it, ++nd) {
      const int h = (int)(it / ((long long)RT * NTILES));
      const int rt = (int)((it / NTILES) % RT);
      const int nt = (int)(it % NTILES);
      const int d = (int)(nd & 1);
      if (!mbar_wait(smem_u32(&d_full[d]), (uint32_t)((nd >> 1) & 1), p.status, abort_flag)) break;
      tc_fence_after();
      for (int c = 0; c < p.NT; c += 64, ++nbox) {
        uint32_t v[64];
        tmem_ld_32x32b_x32(tmem + lane_addr + (uint32_t)(d * p.NT + c), *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_ld_32x32b_x32(tmem + lane_addr + (uint32_t)(d * p.NT + c + 32), *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_ld_wait();
        const uint32_t box = stage0 + (uint32_t)((nbox & 1) * kHgOutBox);
        // the store issued from this buffer two boxes ago has read it
        if (lane == 0) bulk_wait_read<1>();
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 8; ++k) {                  // 16-byte chunk k of this row, swizzled by row
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[8 * k + 2 * e]), __uint_as_float(v[8 * k + 2 * e + 1]));
            w4[e] = *reinterpret_cast<uint32_t*>(&b2);
          }
          const uint32_t a = box + (uint32_t)(lane * 128) + (uint32_t)(((k ^ (lane & 7)) & 7) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(w4[0]), "r"(w4[1]), "r"(w4[2]),
                       "r"(w4[3])
                       : "memory");
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int y = rt * 128 + q4 * 32;
          if (y < p.n_rows) tma_store_2d(&map_c, box, h * p.N + nt * p.NT + c, y);  // a partial box is clipped
          bulk_commit();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&d_empty[d]));
    }
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");  // stores complete before exit
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * p.NT);
    tmem_relinquish();
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)ptr;
  }
  return fn;
}

int tile_n(int N) { return N > 256 ? 256 : N; }

}  // namespace

bool head_gemm_tc_supported(int n_rows, int heads, int K, int N, const void* A, const void* Bm, bool b_kn,
                            const void* C) {
  if (n_rows < 128 || heads < 1 || K % 64 != 0 || K > 512) return false;
  const int NT = tile_n(N);
  if (N % NT != 0 || NT % 64 != 0) return false;
  if ((long long)K * N * 2 > kHgMaxBBytes) return false;
  if (b_kn && K > 256) return false;                       // one [K][64] box per column block
  if ((((uintptr_t)A) | ((uintptr_t)Bm) | ((uintptr_t)C)) & 15u) return false;
  if ((long long)heads * K > (1LL << 31) / 2 || (long long)heads * N > (1LL << 31) / 2) return false;
  return encode_fn() != nullptr;
}

cudaError_t launch_head_gemm_tc(int n_rows, int heads, int K, int N, const void* A, const void* Bm, bool b_kn,
                                void* C, cudaStream_t st) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  const int NT = tile_n(N);
  // A viewed as [n_rows, H*K]; box = 64 columns x 128 rows (128-byte swizzle)
  CUtensorMap ma;
  cuuint64_t adims[2] = {(cuuint64_t)heads * K, (cuuint64_t)n_rows};
  cuuint64_t astr[1] = {(cuuint64_t)heads * K * 2};
  cuuint32_t abox[2] = {64u, 128u};
  cuuint32_t estr[2] = {1u, 1u};
  if (enc(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(A), adims, astr, abox, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  CUtensorMap mb;
  if (b_kn) {
    // B viewed as [H*K rows, N cols]; box = 64 columns x K rows
    cuuint64_t bdims[2] = {(cuuint64_t)N, (cuuint64_t)heads * K};
    cuuint64_t bstr[1] = {(cuuint64_t)N * 2};
    cuuint32_t bbox[2] = {64u, (cuuint32_t)K};
    if (enc(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(Bm), bdims, bstr, bbox, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {
    // B viewed as [H*N rows, K cols]; box = 64 columns x NT rows
    cuuint64_t bdims[2] = {(cuuint64_t)K, (cuuint64_t)heads * N};
    cuuint64_t bstr[1] = {(cuuint64_t)K * 2};
    cuuint32_t bbox[2] = {64u, (cuuint32_t)NT};
    if (enc(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(Bm), bdims, bstr, bbox, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  // C viewed as [n_rows, H*N]; box = 64 columns x 32 rows (one epilogue warp's rows), 128-byte swizzle
  CUtensorMap mc;
  cuuint64_t cdims[2] = {(cuuint64_t)heads * N, (cuuint64_t)n_rows};
  cuuint64_t cstr[1] = {(cuuint64_t)heads * N * 2};
  cuuint32_t cbox[2] = {64u, 32u};
  if (enc(&mc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, C, cdims, cstr, cbox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
      CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  HgParams p{n_rows, heads, K, N, NT, b_kn, (bf16*)C, device_status_ptr()};
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long items = (long long)heads * ((n_rows + 127) / 128) * (N / NT);
  const int grid = (int)(items < sms ? items : sms);
  const size_t smem = 1024 + kHgMaxBBytes + (size_t)kHgStages * kHgABytes + 4 * 2 * kHgOutBox;
  cudaError_t e = cudaFuncSetAttribute(head_gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  head_gemm_tc_kernel<<<grid, kHgThreads, smem, st>>>(ma, mb, mc, p);
  return cudaGetLastError();
}

}  // namespace dsa
