// Fused S2 -> S3: lightning-indexer scores and the deterministic top-k in one kernel, without
// writing the score matrix to memory.
//
// The score is I[s] = sum_h w[h] * relu(scale * q[h,:] . k[s,:]) (fak note "GLM-5.2: the DSA sparse
// attention moves onto the pure fak kernel", section 3: the selection is score dots followed by a
// top-k), and the selection takes the min(k, n_visible) visible keys of highest score, smaller key
// index first among equal scores (metrale glm5next_dsa_ref topk_pools).  The output lists the
// selected keys in ascending key order with DSA_INVALID after them: the set dsa_topk_set lists.
//
// One query row per thread-block cluster of C CTAs (C = 1, 2, 4 or 8).  CTA rank r scores the keys
// [r*chunk, (r+1)*chunk) of the row's sequence (chunk <= 16384, a multiple of 128) exactly as the
// tensor-core indexer does for a single query (M = 128 keys per tcgen05.mma, N = H_I heads, K =
// 128 in two 64-wide swizzled blocks, TMEM accumulators, the relu*w reduction per lane), and keeps
// each score as an order-preserving 32-bit key in shared memory.  The epilogue also counts the
// top 8 bits of every key (the first histogram of the selection).  Then the cluster selects:
//   1. four rounds of 8 bits: each CTA histograms its keys that match the prefix found so far and
//      stores the histogram into every CTA of the cluster (distributed shared memory; the freed key
//      stages hold the copies), so every CTA walks the same summed bins from the top, locally, and
//      all agree on the next 8 bits of the k-th largest key tau and on how many keys equal to tau
//      still have to be taken;
//   2. each CTA counts its keys above and equal to tau and stores the counts into every CTA, so each
//      knows the counts of the lower ranks: how many of its tau keys to take (ties go to the smaller
//      index, and lower ranks hold smaller indices) and where its keys start in the row;
//   3. each warp lists its contiguous segment of keys in order (ballots), at offsets from a scan of
//      the warps' counts.
// A row with at most k visible keys lists them all.  Nothing is written but the index rows.
//
// FP8 operands (kF8): the e4m3 codes and per-vector scales of dsa_fp8_quantize, scored as the FP8
// indexer does (kind::f8f6f4, K = 32 per instruction, one 128-byte row per key; the epilogue folds
// w * |scale| * sq into each head column and multiplies a key's sum by its scale sk, which the
// producer warp brings into a shared-memory ring with cp.async as in the FP8 indexer).  The head
// reduction is index_epilogue.cuh's, so the scores are the standalone indexer's bit for bit.
//
// Warp roles while scoring: warp 0 issues the TMA loads (the query's H_I x 128 block once, then a
// ring of 128-key stages), warp 1 issues the MMAs into two TMEM accumulators, warps 2-5 run the
// epilogue.  All six warps select.  Every mbarrier wait is bounded; a CTA whose wait expires still
// takes part in every cluster barrier (the selection of that row is then meaningless and the
// device status reports DSA_ERR_TIMEOUT), so no CTA of the cluster waits forever.
#include <cuda.h>

#include "dsa_common.cuh"
#include "dsa_internal.h"
#include "dsa_sm100.cuh"
#include "index_epilogue.cuh"

namespace dsa {

#ifdef DSA_TRACE
// Optional per-tile timeline of CTA 0 (build with -DDSA_TRACE): g_fused_trace[event][tile] = %globaltimer.
__device__ unsigned long long g_fused_trace[8][256];
#define FTRACE(ev, i)                                                                       \
  do {                                                                                      \
    if (blockIdx.x == 0 && (i) < 256) g_fused_trace[ev][(i)] = sm100::globaltimer();        \
  } while (0)
#else
#define FTRACE(ev, i) ((void)0)
#endif

namespace {

using namespace sm100;

constexpr int kDI = 128;
constexpr int kKeysPerTile = 128;
constexpr int kMaxStages = 6;
// Bytes of one indexer vector and of one key stage: bf16 256 B / 32 KB, e4m3 128 B / 16 KB.
__host__ __device__ constexpr int row_bytes(bool f8) { return f8 ? kDI : 2 * kDI; }
__host__ __device__ constexpr int tile_bytes(bool f8) { return kKeysPerTile * row_bytes(f8); }
constexpr int kMaxLocal = 16384;                     // keys a CTA holds (64 KB of 32-bit keys)
constexpr int kThreads = 192;                        // 6 warps
constexpr int kWarps = kThreads / 32;
constexpr int kLevels = 4;                           // 8-bit rounds of the radix select

struct FusedParams {
  int B, T, S, HI;
  int chunk;              // keys per CTA
  int stages;
  int k;
  float scale;
  const float* q_scale;   // FP8: [B*T*H_I]
  const float* k_scale;   // FP8: [B*S]
  const float* w;
  const int32_t* q_pos;
  const int32_t* kv_start;
  const int32_t* kv_len;
  int32_t* idx;           // [B*T, k]
  int* status;
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// 32-bit store into the shared memory of CTA `rank` of the cluster at the same offset as `local`.
__device__ __forceinline__ void st_cluster(void* local, uint32_t rank, uint32_t v) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(remote), "r"(v) : "memory");
}

template <bool kF8>
__global__ void __launch_bounds__(kThreads, 1)
index_topk_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                  FusedParams p) {
  constexpr int kTileBytes = tile_bytes(kF8);
  constexpr uint32_t kRow = (uint32_t)row_bytes(kF8);
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* gbase = smem_raw + (base - raw);
  // [q block: HI x kRow][stages x kTileBytes][keys: chunk x 4 B][hist: 4 x 256][wsc: HI]
  // [(FP8) key scales: (stages+2) x 128][misc][barriers]
  const uint32_t sB = base;
  const uint32_t sA = sB + (uint32_t)p.HI * kRow;
  const int sk_slots = p.stages + 2;
  uint32_t* keys = reinterpret_cast<uint32_t*>(gbase + (sA - base) + (uint32_t)p.stages * kTileBytes);
  uint32_t* hist = keys + p.chunk;                        // [kLevels][256]
  float* wsc_s = reinterpret_cast<float*>(hist + kLevels * 256);
  float* sk_s = wsc_s + p.HI;                              // FP8 only
  // misc: [0] bin, [1] remaining, [4..4+kWarps) warp gt counts, [16..16+kWarps) warp eq counts,
  // [32..32+2C) every rank's (gt, eq) totals, pushed by the ranks
  int* misc = reinterpret_cast<int*>(sk_s + (kF8 ? sk_slots * kKeysPerTile : 0));
  uint64_t* bars = reinterpret_cast<uint64_t*>(misc + 48);
  uint64_t* full = bars;
  uint64_t* empty = full + kMaxStages;
  uint64_t* tfull = empty + kMaxStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* bfull = tempty + 2;
  uint64_t* drain = bfull + 1;
  uint64_t* skfull = drain + 1;                            // [stages + 2] (FP8)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(skfull + kMaxStages + 2);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank(), C = cluster_size();
  const long long row = (long long)blockIdx.x / C;        // one query row per cluster
  const int b = (int)(row / p.T);
  const KeyRange vis = visible_range(p.q_pos[row], p.kv_start[b], p.kv_len[b], p.S, 0);
  const int n_vis = vis.count();
  // this CTA's visible keys [l0, l1] (absolute key indices; empty when l1 < l0)
  const int r0 = (int)rank * p.chunk;
  const int l0 = max(vis.lo, r0), l1 = min(vis.hi, r0 + p.chunk - 1);
  const int n_local = l1 >= l0 ? l1 - l0 + 1 : 0;
  const int t_begin = n_local ? l0 / kKeysPerTile : 0;
  const int n_tiles = n_local ? l1 / kKeysPerTile - t_begin + 1 : 0;
  const uint32_t ncols = p.HI * 2 <= 64 ? 64 : (p.HI * 2 <= 128 ? 128 : 256);

  for (int i = threadIdx.x; i < kLevels * 256; i += kThreads) hist[i] = 0u;
  const float ascale = fabsf(p.scale);
  for (int i = threadIdx.x; i < p.HI; i += kThreads) {
    const long long col = row * p.HI + i;
    wsc_s[i] = kF8 ? p.w[col] * ascale * p.q_scale[col] : p.w[col] * ascale;
  }
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&tfull[a]), 1);
      mbar_init(smem_u32(&tempty[a]), 4);
    }
    if (kF8)
      for (int s = 0; s < sk_slots; ++s) mbar_init(smem_u32(&skfull[s]), 32);  // one cp.async arrival per lane
    mbar_init(smem_u32(bfull), 1);
    mbar_init(smem_u32(drain), 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), ncols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // ---------------------------------------------------------------- scoring
  if (warp == 0) {
    if (n_tiles > 0) {
      if (lane == 0) {
        tma_prefetch_desc(&map_q);
        tma_prefetch_desc(&map_k);
        mbar_arrive_expect_tx(smem_u32(bfull), (uint32_t)p.HI * kRow);
        tma_load_2d(sB, &map_q, smem_u32(bfull), 0, (int)(row * p.HI));
        if (!kF8) tma_load_2d(sB + (uint32_t)p.HI * 128u, &map_q, smem_u32(bfull), 64, (int)(row * p.HI));
      }
      int issued = 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % p.stages;
        bool ok = true;
        if (lane == 0) ok = mbar_wait(smem_u32(&empty[s]), ((i / p.stages) & 1) ^ 1, p.status, &abort_flag);
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        const int krow = b * p.S + (t_begin + i) * kKeysPerTile;
        if (lane == 0) {
          FTRACE(0, i);
          const uint32_t dst = sA + (uint32_t)s * kTileBytes;
          mbar_arrive_expect_tx(smem_u32(&full[s]), kTileBytes);
          tma_load_2d(dst, &map_k, smem_u32(&full[s]), 0, krow);
          if (!kF8) tma_load_2d(dst + kTileBytes / 2, &map_k, smem_u32(&full[s]), 64, krow);
        }
        if (kF8) {
          // the tile's 128 key scales, four per lane (keys past the sequence read its last scale)
          const int key0 = (t_begin + i) * kKeysPerTile + 4 * lane;
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
      if (lane == 0 && abort_flag) {  // let every issued copy land before the shared memory is reused or freed
        mbar_wait(smem_u32(bfull), 0, nullptr, nullptr);
        for (int i = max(0, issued - p.stages); i < issued; ++i)
          mbar_wait(smem_u32(&full[i % p.stages]), (i / p.stages) & 1, nullptr, nullptr);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && n_tiles > 0) {
      const uint32_t idesc = kF8 ? idesc_e4m3(128, p.HI) : idesc_bf16(128, p.HI);
      bool ok = mbar_wait(smem_u32(bfull), 0, p.status, &abort_flag);
      for (int i = 0; ok && i < n_tiles; ++i) {
        const int s = i % p.stages, a = i & 1;
        if (!mbar_wait(smem_u32(&tempty[a]), ((i >> 1) & 1) ^ 1, p.status, &abort_flag)) break;
        if (!mbar_wait(smem_u32(&full[s]), (i / p.stages) & 1, p.status, &abort_flag)) break;
        FTRACE(1, i);
        tc_fence_after();
        const uint32_t a0 = sA + (uint32_t)s * kTileBytes;
        const uint32_t d = tmem + (uint32_t)(a * p.HI);
        if (kF8) {
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
            const uint64_t bd = desc_sw128(sB + (uint32_t)(j >> 2) * (uint32_t)p.HI * 128u + koff);
            mma_bf16_ss(d, ad, bd, idesc, j > 0 ? 1u : 0u);
          }
        }
        mma_commit(smem_u32(&empty[s]));
        mma_commit(smem_u32(&tfull[a]));
        FTRACE(2, i);
      }
      mma_commit(smem_u32(drain));
      mbar_wait(smem_u32(drain), 0, nullptr, nullptr);
    }
  } else {
    // epilogue: lane quarter (warp & 3) of each tile, one key per thread
    const int quarter = warp & 3;
    const bool neg = p.scale < 0.f;                      // relu(scale * x) = |scale| * relu(-x)
    for (int i = 0; i < n_tiles; ++i) {
      const int a = i & 1;
      if (!mbar_wait(smem_u32(&tfull[a]), (i >> 1) & 1, p.status, &abort_flag)) break;
      if (quarter == 0 && lane == 0) FTRACE(3, i);
      tc_fence_after();
      const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(a * p.HI);
      const int s = (t_begin + i) * kKeysPerTile + quarter * 32 + lane;
      float sk = 1.f;
      if (kF8) {
        const int slot = i % sk_slots;
        if (!mbar_wait(smem_u32(&skfull[slot]), (uint32_t)((i / sk_slots) & 1), p.status, &abort_flag)) break;
        sk = sk_s[slot * kKeysPerTile + quarter * 32 + lane];
      }
      float acc = 0.f;
      for (int h0 = 0; h0 < p.HI; h0 += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(trow + (uint32_t)h0, v);
        tmem_ld_wait();
        acc += neg ? head_sum32<true>(v, wsc_s + h0) : head_sum32<false>(v, wsc_s + h0);
      }
      if (kF8) acc *= sk;
      if (quarter == 0 && lane == 0) FTRACE(4, i);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tempty[a]));
      if (s >= l0 && s <= l1) {
        const uint32_t key = score_key(acc);            // -0 and +0 share a key
        keys[s - l0] = key;
        atomicAdd(&hist[key >> 24], 1u);
      }
      __syncwarp();
      if (quarter == 0 && lane == 0) FTRACE(5, i);
    }
  }
  tc_fence_before();
  __syncthreads();

  // ---------------------------------------------------------------- selection
  if (threadIdx.x == 0) FTRACE(6, 0);
  int32_t* orow = p.idx + row * p.k;
  if (n_vis <= p.k) {
    // every visible key: this CTA's keys sit at positions l0 - vis.lo .. in the ascending list
    for (int i = threadIdx.x; i < n_local; i += kThreads) orow[l0 - vis.lo + i] = l0 + i;
    if (rank == C - 1)
      for (int i = n_vis + threadIdx.x; i < p.k; i += kThreads) orow[i] = DSA_INVALID;
  } else {
    // After scoring, the key stages are free.  Every CTA pushes each round's histogram and its final
    // counts into every CTA of the cluster (remote stores into the stage area), so the walks read
    // only local shared memory.  A cluster barrier first makes sure no CTA is still scoring into
    // its stages.
    uint32_t* hall = reinterpret_cast<uint32_t*>(gbase + (sA - base));  // [kLevels][C][256]
    int* call = misc + 32;                                              // [C][2]: each rank's gt, eq
    cluster_sync();
    if (threadIdx.x == 0) FTRACE(7, 0);
    uint32_t prefix = 0u, mask = 0u;
    int remaining = p.k;                                 // keys still to take at and below the prefix
    for (int lev = 0; lev < kLevels; ++lev) {
      const int shift = 24 - 8 * lev;
      uint32_t* h = hist + lev * 256;
      if (lev > 0) {
        // four keys per thread in flight
        for (int i0 = threadIdx.x; i0 < n_local; i0 += 4 * kThreads) {
          uint32_t k4[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * kThreads;
            k4[u] = i < n_local ? keys[i] : 0u;
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * kThreads;
            if (i < n_local && (k4[u] & mask) == prefix) atomicAdd(&h[(k4[u] >> shift) & 255u], 1u);
          }
        }
        __syncthreads();                                 // this round's local histogram is complete
      }
      for (int bin = threadIdx.x; bin < 256; bin += kThreads) {
        const uint32_t v = h[bin];
        uint32_t* dst = hall + (lev * C + rank) * 256 + bin;
        for (uint32_t r = 0; r < C; ++r) st_cluster(dst, r, v);
      }
      if (threadIdx.x == 0) FTRACE(7, 3 * lev + 1);
      cluster_sync();                                    // every CTA holds every CTA's histogram
      if (warp == 0) {
        // bins from the top: lane l holds bins 255-8l .. 248-8l, summed over the cluster
        uint32_t c[8], tot = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int bin = 255 - 8 * lane - j;
          uint32_t v = 0;
          for (uint32_t r = 0; r < C; ++r) v += hall[(lev * C + r) * 256 + bin];
          c[j] = v;
          tot += v;
        }
        uint32_t incl = tot;                             // inclusive scan over lanes (from the top)
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const uint32_t excl = incl - tot;
        const uint32_t hit = __ballot_sync(0xffffffffu, excl < (uint32_t)remaining && incl >= (uint32_t)remaining);
        if (hit == 0u && lane == 0) {                    // only after an expired wait left keys unscored
          misc[0] = 0;
          misc[1] = 1;
        }
        if (lane == __ffs(hit) - 1) {
          uint32_t above = excl;
          int j = 0;
          while (above + c[j] < (uint32_t)remaining) above += c[j++];
          misc[0] = 255 - 8 * lane - j;                  // the bin holding the k-th largest key
          misc[1] = remaining - (int)above;              // keys to take inside that bin
        }
      }
      __syncthreads();
      if (threadIdx.x == 0) FTRACE(7, 3 * lev + 2);
      prefix |= (uint32_t)misc[0] << shift;
      mask |= 255u << shift;
      remaining = misc[1];
      __syncthreads();                                   // misc is rewritten in the next round
    }
    const uint32_t tau = prefix;                         // the k-th largest key
    const int need_eq = remaining;                       // keys equal to tau to take (>= 1)
    // per-warp counts over contiguous segments, in key order, 64 keys per step
    const int seg = (n_local + kWarps - 1) / kWarps;
    const int e0 = min(n_local, warp * seg), e1 = min(n_local, e0 + seg);
    int gt = 0, eq = 0;
    for (int i0 = e0; i0 < e1; i0 += 64) {
      const int ia = i0 + lane, ib = i0 + 32 + lane;
      const uint32_t ka = ia < e1 ? keys[ia] : 0u, kb = ib < e1 ? keys[ib] : 0u;
      gt += __popc(__ballot_sync(0xffffffffu, ia < e1 && ka > tau)) + __popc(__ballot_sync(0xffffffffu, ib < e1 && kb > tau));
      eq += __popc(__ballot_sync(0xffffffffu, ia < e1 && ka == tau)) + __popc(__ballot_sync(0xffffffffu, ib < e1 && kb == tau));
    }
    if (lane == 0) {
      misc[4 + warp] = gt;
      misc[16 + warp] = eq;
    }
    __syncthreads();
    int g_all = 0, e_all = 0;
    for (int k = 0; k < kWarps; ++k) {
      g_all += misc[4 + k];
      e_all += misc[16 + k];
    }
    if (threadIdx.x < C) {                               // push (gt, eq) to rank threadIdx.x
      st_cluster(&call[2 * rank], threadIdx.x, (uint32_t)g_all);
      st_cluster(&call[2 * rank + 1], threadIdx.x, (uint32_t)e_all);
    }
    if (threadIdx.x == 0) FTRACE(7, 12);
    cluster_sync();                                      // every CTA holds every CTA's totals
    if (threadIdx.x == 0) FTRACE(7, 13);
    int gt_before = 0, eq_before = 0;
    for (uint32_t r = 0; r < rank; ++r) {
      gt_before += call[2 * r];
      eq_before += call[2 * r + 1];
    }
    const int take = max(0, min(need_eq - eq_before, e_all));        // this CTA's tau keys to take
    int out = gt_before + min(eq_before, need_eq);                   // where this CTA's keys start
    int eq_rank = 0;                                                 // tau keys before this warp's segment
    for (int k = 0; k < warp; ++k) {
      out += misc[4 + k];
      eq_rank += misc[16 + k];
    }
    out += min(eq_rank, take);
    const uint32_t below = (1u << lane) - 1u;
    for (int i0 = e0; i0 < e1; i0 += 64) {
      const int ib = i0 + 32 + lane;
      const uint32_t kb = ib < e1 ? keys[ib] : 0u;       // the second half's keys load with the first's
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int i = i0 + 32 * half + lane;
        const uint32_t key = half ? kb : (i < e1 ? keys[i] : 0u);
        const bool is_gt = i < e1 && key > tau;
        const bool is_eq = i < e1 && key == tau;
        const uint32_t m_eq = __ballot_sync(0xffffffffu, is_eq);
        const int my_eq = eq_rank + __popc(m_eq & below);
        const bool sel = is_gt || (is_eq && my_eq < take);
        const uint32_t m_sel = __ballot_sync(0xffffffffu, sel);
        const int pos = out + __popc(m_sel & below);
        if (sel && pos < p.k) orow[pos] = l0 + i;      // always true unless an expired wait left keys unscored
        out += __popc(m_sel);
        eq_rank += __popc(m_eq);
      }
    }
  }
  if (threadIdx.x == 0) FTRACE(6, 1);
  cluster_sync();  // no CTA leaves while a peer may still read its shared memory
  if (warp == 1) {
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
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)ptr;
  }
  return fn;
}

// [rows, 128] of bf16 (box 64 columns) or e4m3 codes (box 128 columns), box_rows rows, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint32_t box_rows, bool f8) {
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

int cluster_for(int S) {
  int C = 1;
  while (C < 8 && ((S + C - 1) / C + kKeysPerTile - 1) / kKeysPerTile * kKeysPerTile > kMaxLocal) C *= 2;
  return C;
}

size_t fused_smem(int HI, int stages, int chunk, bool f8) {
  return 1024 + (size_t)HI * row_bytes(f8) + (size_t)stages * tile_bytes(f8) + (size_t)chunk * 4 +
         kLevels * 256 * 4 + (size_t)HI * 4 + (f8 ? (size_t)(stages + 2) * kKeysPerTile * 4 : 0) + 48 * 4 +
         8 * (2 * kMaxStages + 6 + kMaxStages + 2) + 16;
}

}  // namespace

bool index_topk_supported(const dsa_dims& d, int k, bool f8) {
  if ((!f8 && d.dtype != DSA_BF16) || d.idx_dim != kDI || d.kpool != 0) return false;
  if (!(d.idx_heads == 32 || d.idx_heads == 64 || d.idx_heads == 128)) return false;
  if ((long long)d.batch * d.n_kv < kKeysPerTile || (long long)d.batch * d.n_q * d.idx_heads > 2147483647LL ||
      (long long)d.batch * d.n_kv > 2147483647LL)
    return false;
  if (k < 1 || k > 1 << 20) return false;
  const int C = cluster_for(d.n_kv);
  const int chunk = ((d.n_kv + C - 1) / C + kKeysPerTile - 1) / kKeysPerTile * kKeysPerTile;
  if (chunk > kMaxLocal) return false;                  // more than 8 x 16384 keys
  if (fused_smem(d.idx_heads, 2, chunk, f8) > 227 * 1024) return false;
  return encode_fn() != nullptr;
}

cudaError_t launch_index_topk(const dsa_dims& d, const void* q_idx, const void* k_idx, const float* w, float scale,
                              const int32_t* q_pos, const int32_t* kv_start, const int32_t* kv_len, int k,
                              int32_t* idx, cudaStream_t st, const float* q_scale, const float* k_scale) {
  const bool f8 = q_scale != nullptr;
  FusedParams p{};
  p.B = d.batch;
  p.T = d.n_q;
  p.S = d.n_kv;
  p.HI = d.idx_heads;
  const int C = cluster_for(d.n_kv);
  p.chunk = ((d.n_kv + C - 1) / C + kKeysPerTile - 1) / kKeysPerTile * kKeysPerTile;
  p.k = k;
  p.scale = scale;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.w = w;
  p.q_pos = q_pos;
  p.kv_start = kv_start;
  p.kv_len = kv_len;
  p.idx = idx;
  p.status = device_status_ptr();
  // 128 KB of key stages in flight per CTA at most (four bf16 or six e4m3 stages)
  int stages = f8 ? kMaxStages : 4;
  while (stages > 2 && fused_smem(p.HI, stages, p.chunk, f8) > 227 * 1024) --stages;
  p.stages = stages;
  const size_t smem = fused_smem(p.HI, stages, p.chunk, f8);
  CUtensorMap mq, mk;
  if (!make_map(&mq, q_idx, (uint64_t)d.batch * d.n_q * d.idx_heads, (uint32_t)p.HI, f8)) return cudaErrorInvalidValue;
  if (!make_map(&mk, k_idx, (uint64_t)d.batch * d.n_kv, kKeysPerTile, f8)) return cudaErrorInvalidValue;
  auto kern = f8 ? index_topk_kernel<true> : index_topk_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((long long)d.batch * d.n_q * C));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, mq, mk, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace dsa

#ifdef DSA_TRACE
extern "C" int dsa_fused_trace_read(unsigned long long* host) {
  return (int)cudaMemcpyFromSymbol(host, dsa::g_fused_trace, sizeof(dsa::g_fused_trace));
}
#endif
