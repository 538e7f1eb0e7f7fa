// S2 lightning-indexer scores on the 5th-generation tensor cores (tcgen05).
//
// I[b,t,s] = sum_h w[b,t,h] * relu(scale * q[b,t,h,:] . k[b,s,:])   (fak note
// "GLM-5.2: the DSA sparse attention moves onto the pure fak kernel", section 3;
// metrale glm5next_dsa_ref index_scores), -inf for keys that are not visible.
//
// The contraction q.k is dense: keys x (queries*heads) x 128.  Layout:
//   M = 128 keys (one TMEM lane per key)          A: k_idx tile, K-major
//   N = NQ queries x H_I heads (<= 256 columns)   B: q_idx rows (t,h), K-major
//   K = D_I = 128 (two 64-wide swizzled blocks)
// so the non-linear head reduction sum_h w*relu(.) is a per-lane loop over the
// accumulator columns: no shuffles, and each warp stores 32 consecutive scores.
//
// One CTA owns a query tile (NQ consecutive queries of one sequence, loaded
// once by TMA) and a contiguous range of 128-key tiles.  Tiles that intersect
// the tile's visible key interval are computed; the rest are filled with -inf.
// Warp roles: warp 0 issues TMA loads into a ring of key stages, warp 1 issues
// tcgen05.mma into one of two TMEM accumulators, warps 2.. run the epilogue
// (tcgen05.ld -> relu/weight reduction -> coalesced fp32 stores).  Every
// mbarrier wait is bounded (records DSA_ERR_TIMEOUT and aborts the CTA).
//
// FP8 operands (kF8): q and k arrive as e4m3 codes with one fp32 scale per
// query-head vector and per key row (dsa_fp8_quantize).  A key row is then 128
// bytes, one 128-byte swizzle row, and the MMA is kind::f8f6f4 with K = 32 per
// instruction.  Since the scales are positive, relu(scale*sq*sk*dot) =
// sk*relu(scale*sq*dot): the epilogue folds scale*sq into each accumulator
// column and multiplies each key's sum by sk.  The producer warp brings each
// tile's 128 key scales into a shared-memory ring of stages + 2 slots (4-byte
// cp.async completing on the slot's own barrier, which the epilogue waits on),
// so no epilogue waits on a global load.  A slot is refilled only after the
// epilogue has finished the tile that used it: the producer runs at most
// `stages` tiles ahead of the MMA, and the MMA at most two ahead of the epilogue.
//
// The head reduction (index_epilogue.cuh) folds w_h * |scale| (* sq_h) into one
// weight per accumulator column, computed once per CTA.
#include <cuda.h>

#include "dsa_common.cuh"
#include "dsa_internal.h"
#include "dsa_sm100.cuh"
#include "index_epilogue.cuh"

namespace dsa {

namespace {

constexpr int kDI = 128;           // indexer head width served by this kernel
constexpr int kKeysPerTile = 128;  // M
constexpr int kMaxStages = 8;
// Bytes of one indexer vector and of one key stage: bf16 256 B / 32 KB, e4m3 128 B / 16 KB.
__host__ __device__ constexpr int row_bytes(bool f8) { return f8 ? kDI : 2 * kDI; }
__host__ __device__ constexpr int tile_bytes(bool f8) { return kKeysPerTile * row_bytes(f8); }

struct IdxTcParams {
  int B, T, S, HI, NQ, N;     // N = NQ * HI
  int kpool;
  int n_qtiles, n_ktiles, tiles_per_split;
  int stages, epi_warps;
  float scale;                // applied inside relu
  const float* q_scale;       // FP8: [B*T*H_I] per query-head vector
  const float* k_scale;       // FP8: [B*S] per key row
  const float* w;
  const int32_t* q_pos;
  const int32_t* kv_start;
  const int32_t* kv_len;
  float* scores;
  int* status;
};

template <bool kF8>
__global__ void __launch_bounds__(320, 1)
index_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                IdxTcParams p) {
  using namespace sm100;
  constexpr int kTileBytes = tile_bytes(kF8);
  constexpr uint32_t kRow = (uint32_t)row_bytes(kF8);
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* gbase = smem_raw + (base - raw);
  // [B operand: N x kRow B][stages x kTileBytes][wsc: NQ*HI floats][(FP8) key scales: (stages+2) x 128]
  // [lo/hi per query][barriers]
  const uint32_t sB = base;
  const uint32_t sA = sB + (uint32_t)p.N * kRow;
  const int sk_slots = p.stages + 2;
  float* wsc_s = reinterpret_cast<float*>(gbase + (sA - base) + (uint32_t)p.stages * kTileBytes);
  float* sk_s = wsc_s + p.N;                                      // FP8 only
  int* lohi = reinterpret_cast<int*>(sk_s + (kF8 ? sk_slots * kKeysPerTile : 0));  // [NQ][2]
  uint64_t* bars = reinterpret_cast<uint64_t*>(lohi + 2 * 16 + 2); // 8-byte aligned below
  bars = reinterpret_cast<uint64_t*>((reinterpret_cast<uintptr_t>(bars) + 7) & ~uintptr_t(7));
  uint64_t* full = bars;                  // [stages]
  uint64_t* empty = full + kMaxStages;    // [stages]
  uint64_t* tfull = empty + kMaxStages;   // [2]
  uint64_t* tempty = tfull + 2;           // [2]
  uint64_t* bfull = tempty + 2;           // [1]
  uint64_t* drain = bfull + 1;            // [1]
  uint64_t* skfull = drain + 1;           // [stages + 2] (FP8)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(skfull + kMaxStages + 2);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z;
  // later query tiles see more keys (causal): launch them first so the last wave is the cheap one
  const int qt = (int)gridDim.y - 1 - (int)blockIdx.y;
  const int t0 = qt * p.NQ;
  const int nq_here = min(p.NQ, p.T - t0);
  const int kt_begin = blockIdx.x * p.tiles_per_split;
  const int kt_end = min(p.n_ktiles, kt_begin + p.tiles_per_split);

  // visible interval of every query of the tile, and their union
  int u_lo = 0x7fffffff, u_hi = -1;
  for (int q = 0; q < nq_here; ++q) {
    const size_t row = (size_t)b * p.T + t0 + q;
    KeyRange r = visible_range(p.q_pos[row], p.kv_start[b], p.kv_len[b], p.S, p.kpool);
    if (r.count() > 0) {
      u_lo = min(u_lo, r.lo);
      u_hi = max(u_hi, r.hi);
    }
    if (threadIdx.x == 0) {
      lohi[2 * q] = r.lo;
      lohi[2 * q + 1] = r.hi;
    }
  }
  int c_begin = kt_end, c_end = kt_end;  // compute tiles [c_begin, c_end)
  if (u_hi >= u_lo) {
    c_begin = max(kt_begin, u_lo / kKeysPerTile);
    c_end = min(kt_end, u_hi / kKeysPerTile + 1);
    if (c_end < c_begin) c_end = c_begin;
  }
  const int n_compute = c_end - c_begin;

  const uint32_t ncols = p.N * 2 <= 32 ? 32 : (p.N * 2 <= 64 ? 64 : (p.N * 2 <= 128 ? 128 : (p.N * 2 <= 256 ? 256 : 512)));
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    if (kF8)
      for (int s = 0; s < sk_slots; ++s) mbar_init(smem_u32(&skfull[s]), 32);  // one cp.async arrival per lane
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&tfull[a]), 1);
      mbar_init(smem_u32(&tempty[a]), p.epi_warps);
    }
    mbar_init(smem_u32(bfull), 1);
    mbar_init(smem_u32(drain), 1);
    fence_barrier_init();
  }
  // folded weight of each accumulator column: w * |scale| (* sq with FP8 operands)
  const float ascale = fabsf(p.scale);
  for (int i = threadIdx.x; i < p.N; i += blockDim.x) {
    const int q = i / p.HI;
    const size_t col = ((size_t)b * p.T + t0 + q) * p.HI + (i - q * p.HI);
    wsc_s[i] = q < nq_here ? (kF8 ? p.w[col] * ascale * p.q_scale[col] : p.w[col] * ascale) : 0.f;
  }
  if (warp == 1 && n_compute > 0) tmem_alloc(smem_u32(tmem_slot), ncols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = n_compute > 0 ? *tmem_slot : 0u;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (n_compute > 0) {
      if (lane == 0) {
        tma_prefetch_desc(&map_q);
        tma_prefetch_desc(&map_k);
        const int qrow = (b * p.T + t0) * p.HI;
        mbar_arrive_expect_tx(smem_u32(bfull), (uint32_t)p.N * kRow);
        tma_load_2d(sB, &map_q, smem_u32(bfull), 0, qrow);
        if (!kF8) tma_load_2d(sB + (uint32_t)p.N * 128u, &map_q, smem_u32(bfull), 64, qrow);
      }
      int issued = 0;
      for (int i = 0; i < n_compute; ++i) {
        const int s = i % p.stages;
        bool ok = true;
        if (lane == 0) ok = mbar_wait(smem_u32(&empty[s]), ((i / p.stages) & 1) ^ 1, p.status, &abort_flag);
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        const int krow = b * p.S + (c_begin + i) * kKeysPerTile;
        if (lane == 0) {
          const uint32_t dst = sA + (uint32_t)s * kTileBytes;
          mbar_arrive_expect_tx(smem_u32(&full[s]), kTileBytes);
          tma_load_2d(dst, &map_k, smem_u32(&full[s]), 0, krow);
          if (!kF8) tma_load_2d(dst + kTileBytes / 2, &map_k, smem_u32(&full[s]), 64, krow);
        }
        if (kF8) {
          // the tile's 128 key scales, four per lane (keys past the sequence read its last scale)
          const int key0 = (c_begin + i) * kKeysPerTile + 4 * lane;
          const int slot = i % sk_slots;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int key = min(key0 + e, p.S - 1);
            cp_async_4(smem_u32(sk_s + slot * kKeysPerTile + 4 * lane + e), p.k_scale + (size_t)b * p.S + key);
          }
          cp_async_mbar_arrive(smem_u32(&skfull[slot]));
        }
        ++issued;
      }
      if (kF8) cp_async_wait_all();
      // on abort, let every issued copy land before the CTA exits
      if (lane == 0 && abort_flag) {
        mbar_wait(smem_u32(bfull), 0, nullptr, nullptr);
        for (int i = max(0, issued - p.stages); i < issued; ++i)
          mbar_wait(smem_u32(&full[i % p.stages]), (i / p.stages) & 1, nullptr, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_compute > 0) {
      const uint32_t idesc = kF8 ? idesc_e4m3(128, p.N) : idesc_bf16(128, p.N);
      bool ok = mbar_wait(smem_u32(bfull), 0, p.status, &abort_flag);
      for (int i = 0; ok && i < n_compute; ++i) {
        const int s = i % p.stages, a = i & 1;
        if (!mbar_wait(smem_u32(&tempty[a]), ((i >> 1) & 1) ^ 1, p.status, &abort_flag)) break;
        if (!mbar_wait(smem_u32(&full[s]), (i / p.stages) & 1, p.status, &abort_flag)) break;
        tc_fence_after();
        const uint32_t a0 = sA + (uint32_t)s * kTileBytes;
        const uint32_t d = tmem + (uint32_t)(a * p.N);
        if (kF8) {
          // one 128-byte row per key: K = 32 codes (32 bytes) per instruction
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t koff = (uint32_t)j * 32u;
            mma_f8_ss(d, desc_sw128(a0 + koff), desc_sw128(sB + koff), idesc, j > 0 ? 1u : 0u);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint32_t koff = (uint32_t)(j & 3) * 32u;
            const uint64_t ad = desc_sw128(a0 + (uint32_t)(j >> 2) * (kTileBytes / 2) + koff);
            const uint64_t bd = desc_sw128(sB + (uint32_t)(j >> 2) * (uint32_t)p.N * 128u + koff);
            mma_bf16_ss(d, ad, bd, idesc, j > 0 ? 1u : 0u);
          }
        }
        mma_commit(smem_u32(&empty[s]));
        mma_commit(smem_u32(&tfull[a]));
      }
      // every issued MMA has completed once this commit arrives
      mma_commit(smem_u32(drain));
      mbar_wait(smem_u32(drain), 0, nullptr, nullptr);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;                       // 0 .. epi_warps-1
    const int quarter = warp & 3;                  // TMEM lane quarter this warp may access
    const int group = ew >> 2;                     // 0 or 1 (two warps per quarter when 8 warps)
    const int ngroups = p.epi_warps >> 2;
    const int key_in_tile = quarter * 32 + lane;
    const bool neg = p.scale < 0.f;               // relu(scale * x) = |scale| * relu(-x)
    int ci = 0;  // compute-tile ordinal
    for (int kt = kt_begin; kt < kt_end; ++kt) {
      const int s = kt * kKeysPerTile + key_in_tile;
      const bool compute = kt >= c_begin && kt < c_end;
      if (!compute) {
        if (s < p.S)
          for (int q = group; q < nq_here; q += ngroups)
            p.scores[((size_t)b * p.T + t0 + q) * p.S + s] = -INFINITY;
        continue;
      }
      const int a = ci & 1;
      if (!mbar_wait(smem_u32(&tfull[a]), (ci >> 1) & 1, p.status, &abort_flag)) break;
      tc_fence_after();
      const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(a * p.N);
      // FP8: this lane's key scale, brought in with the tile
      float sk = 1.f;
      if (kF8) {
        const int slot = ci % sk_slots;
        if (!mbar_wait(smem_u32(&skfull[slot]), (uint32_t)((ci / sk_slots) & 1), p.status, &abort_flag)) break;
        sk = sk_s[slot * kKeysPerTile + key_in_tile];
      }
      for (int q = group; q < nq_here; q += ngroups) {
        float acc = 0.f;
        const float* wq = wsc_s + q * p.HI;
        for (int h0 = 0; h0 < p.HI; h0 += 32) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(trow + (uint32_t)(q * p.HI + h0), v);
          tmem_ld_wait();
          acc += neg ? head_sum32<true>(v, wq + h0) : head_sum32<false>(v, wq + h0);
        }
        if (kF8) acc *= sk;
        if (s < p.S) {
          const int lo = lohi[2 * q], hi = lohi[2 * q + 1];
          const float v = (s >= lo && s <= hi) ? (acc == 0.f ? 0.f : acc) : -INFINITY;
          p.scores[((size_t)b * p.T + t0 + q) * p.S + s] = v;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tempty[a]));
      ++ci;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1 && n_compute > 0) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
    tmem_relinquish();
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  }
  return fn;
}

// 2D tensor [rows, 128] (row-major) of bf16 (box [64 cols, box_rows]) or of e4m3 codes (box [128
// cols, box_rows]): 128-byte box rows in the 128-byte swizzle.
bool make_map_128(CUtensorMap* m, const void* ptr, uint64_t rows, uint32_t box_rows, bool f8) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kDI, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes(f8)};
  cuuint32_t box[2] = {f8 ? 128u : 64u, box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  return enc(m, f8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr),
             dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool index_scores_tc_supported(const dsa_dims& d, bool f8) {
  if ((!f8 && d.dtype != DSA_BF16) || d.idx_dim != kDI) return false;
  if (!(d.idx_heads == 32 || d.idx_heads == 64 || d.idx_heads == 128)) return false;
  if ((long long)d.batch * d.n_kv < 128) return false;  // the key TMA box is 128 rows
  return encode_fn() != nullptr;
}

cudaError_t launch_index_scores_tc(const dsa_dims& d, const void* q_idx, const void* k_idx,
                                   const float* w, float scale, const int32_t* q_pos,
                                   const int32_t* kv_start, const int32_t* kv_len, float* scores,
                                   cudaStream_t st, const float* q_scale, const float* k_scale) {
  const bool f8 = q_scale != nullptr;
  IdxTcParams p{};
  p.B = d.batch;
  p.T = d.n_q;
  p.S = d.n_kv;
  p.HI = d.idx_heads;
  p.NQ = 256 / p.HI;
  if (p.NQ > p.T) p.NQ = p.T;
  p.N = p.NQ * p.HI;
  p.kpool = d.kpool;
  p.n_qtiles = (p.T + p.NQ - 1) / p.NQ;
  p.n_ktiles = (p.S + kKeysPerTile - 1) / kKeysPerTile;
  const int sms = sm_count();
  // Narrow query tiles (N <= 128: decode, one query per sequence) stream many key tiles per CTA:
  // two CTAs per SM with two key stages each hide each other's start-up and keep four tiles
  // in flight per SM; wide tiles keep one CTA per SM with up to six stages.
  const int ctas_per_sm = p.N <= 128 ? 2 : 1;
  // Key-range splits per query tile: one CTA per SM, so the time is about (waves) x (tiles per
  // CTA + a fixed cost of ~3 tiles for the query load and pipeline fill).  Pick the split count
  // that minimises it; a count that leaves a nearly empty last wave loses to a finer one.
  const long long qt = (long long)p.B * p.n_qtiles;
  int splits = 1;
  long long best = -1;
  for (int s2 = 1; s2 <= p.n_ktiles && s2 <= 512; ++s2) {
    const int tps = (p.n_ktiles + s2 - 1) / s2;
    const int used = (p.n_ktiles + tps - 1) / tps;           // splits that get tiles
    const long long waves = (qt * used + (long long)sms * ctas_per_sm - 1) / ((long long)sms * ctas_per_sm);
    const long long cost = waves * (tps + 3);
    if (best < 0 || cost < best) {
      best = cost;
      splits = used;
    }
  }
  p.tiles_per_split = (p.n_ktiles + splits - 1) / splits;
  splits = (p.n_ktiles + p.tiles_per_split - 1) / p.tiles_per_split;
  p.epi_warps = p.NQ >= 2 ? 8 : 4;
  p.scale = scale;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.w = w;
  p.q_pos = q_pos;
  p.kv_start = kv_start;
  p.kv_len = kv_len;
  p.scores = scores;
  p.status = device_status_ptr();
  const size_t tb = (size_t)tile_bytes(f8);
  const size_t fixed = 1024 + (size_t)p.N * row_bytes(f8) + (size_t)p.N * 4 +
                       (f8 ? (kMaxStages + 2) * kKeysPerTile * 4 : 0) + 2 * 16 * 4 + 64 +
                       8 * (2 * kMaxStages + 8 + kMaxStages + 2) + 64;
  int stages = (int)((220 * 1024 - fixed) / tb);
  if (stages > (f8 ? kMaxStages : 6)) stages = f8 ? kMaxStages : 6;
  // two CTAs per SM: two 32 KB stages each (bf16), four 16 KB stages each (e4m3): 64 KB in flight per CTA
  if (ctas_per_sm == 2 && stages > (f8 ? 4 : 2)) stages = f8 ? 4 : 2;
  if (stages < 2) return cudaErrorInvalidConfiguration;
  p.stages = stages;
  const size_t smem = fixed + (size_t)stages * tb;

  CUtensorMap mq, mk;
  if (!make_map_128(&mq, q_idx, (uint64_t)d.batch * d.n_q * d.idx_heads, (uint32_t)p.N, f8))
    return cudaErrorInvalidValue;
  if (!make_map_128(&mk, k_idx, (uint64_t)d.batch * d.n_kv, kKeysPerTile, f8)) return cudaErrorInvalidValue;
  auto kern = f8 ? index_tc_kernel<true> : index_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(splits, p.n_qtiles, p.B);
  const int threads = 64 + 32 * p.epi_warps;
  kern<<<grid, threads, smem, st>>>(mq, mk, p);
  return cudaGetLastError();
}

}  // namespace dsa
