// S3 deterministic top-k: radix select in shared memory, then a rank sort.
//
// Per query row: the min(k, n_visible) visible keys with the highest score,
// ordered by higher score and then smaller key index (metrale
// glm5next_dsa_ref topk_pools; ik_llama.cpp #2045 ggml_top_k(min(top_k,
// n_tokens))).
//
// One block per row: 1024 threads for rows of more than 8192 keys, 512 up to 8192, and 256 (six
// blocks per SM, so that short rows overlap) up to 4096.  Scores become order-preserving uint32 keys (signed
// zeros merged) and are cached in shared memory when the visible range fits.
// One pass (16-byte loads) counts the top 12 bits of every key (plain shared atomics); the
// keys of the bin that holds the k-th largest become a small candidate set
// whose low 20 bits are resolved alone (12 + 8 bits).  That gives the exact
// k-th largest key tau and how many keys equal to tau are still needed.  A
// crowded bin (more keys than the candidate buffer holds, e.g. near-equal
// scores) resolves the same two digits with one filtered pass over the row
// each instead.  Each warp owns a
// contiguous segment of the row, walked 128 keys at a time (four per lane, their
// loads and ballots independent).  The pass that
// collects the candidates also counts, per warp, the keys above the bin, and
// tags each candidate with its warp, so the per-warp counts of keys > tau and
// == tau come from the candidates without another pass over the row (the
// crowded-bin path counts them in one more pass).  Ballots and a block-wide
// prefix sum of those counts place every key > tau and the lowest-index keys
// == tau, which keeps the tie rule exact.  Finally the (key, index) pairs are put in
// rank order by a stable four-pass LSD radix sort on the key (descending), so
// equal keys keep ascending index order.
//
// The unranked variant (the fused layer's selection, which the attention reads
// as a set) selects the same keys under the same rule and lists them in
// ascending key order: a row with at most k visible keys is its visible range,
// and a longer row needs the select passes and one ordered compaction, no sort.
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {

#ifdef DSA_TRACE
// Optional phase timeline of a few rows (build with -DDSA_TRACE): g_topk_trace[row][phase] = %globaltimer.
__device__ unsigned long long g_topk_trace[8][8];
#define TOPK_TRACE(ph)                                                                         \
  do {                                                                                         \
    if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.x < 8) {                               \
      unsigned long long t_;                                                                   \
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                                   \
      g_topk_trace[blockIdx.x][ph] = t_;                                                       \
    }                                                                                          \
  } while (0)
#else
#define TOPK_TRACE(ph) ((void)0)
#endif

constexpr int kTopkCacheMax = 40960;  // keys cached in shared memory (160 KB)
constexpr int kHist12 = 4096;         // first-pass histogram: the top 12 bits of a key
constexpr int kCand = 4096;           // keys of the threshold's 12-bit bin resolved on their own (at most)

// Block-wide exclusive scan of one int per thread; returns the block total.  One barrier: every
// warp scans the (at most 32) warp totals itself.  The caller reaches a barrier before `scratch`
// (>= BLOCK/32 ints) is written again.
template <int BLOCK>
__device__ __forceinline__ int block_exclusive_scan(int v, int* scratch, int& total) {
  constexpr int NW = BLOCK / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  const int w = lane < NW ? scratch[lane] : 0;
  int s = w;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, s, o);
    if (lane >= o) s += y;
  }
  total = __shfl_sync(0xffffffffu, s, NW - 1);
  const int warp_base = __shfl_sync(0xffffffffu, s - w, warp);
  return warp_base + x - v;
}

// Lanes of the warp holding the same 8-bit digit d (0..255) as this lane, from one ballot
// per bit (the address-divergence unit behind match.any is the bottleneck otherwise).
// Lanes with d < 0 take no part; their own result is meaningless.
__device__ __forceinline__ uint32_t same_digit_lanes(int d) {
  uint32_t m = __ballot_sync(0xffffffffu, d >= 0);
#pragma unroll
  for (int b = 0; b < 8; ++b) {
    const bool bit = (d >> b) & 1;
    const uint32_t bb = __ballot_sync(0xffffffffu, bit);
    m &= bit ? bb : ~bb;
  }
  return m;
}

// In a histogram of `nbins` bins (bin = a digit, counted over the keys still in play), find
// the digit holding the `kneed`-th largest key, scanning digits from the top: *s_bin gets
// the digit and *s_krem how many keys of that digit are still needed.  Block-wide.
template <int BLOCK>
__device__ void find_crossing(const uint32_t* hist, int nbins, uint32_t kneed, int* scan, uint32_t* s_bin,
                              uint32_t* s_krem) {
  const int per = nbins >= BLOCK ? nbins / BLOCK : 1;    // digits per thread (<= 8 from 512 threads up)
  const int owners = nbins / per;
  const int top = nbins - 1 - per * (int)threadIdx.x;   // this thread's digits: top, top - 1, ..., top - per + 1
  const bool own = (int)threadIdx.x < owners;
  const bool vec = (per & 3) == 0;                       // whole aligned groups of four: 16-byte loads
  const uint4* h4 = reinterpret_cast<const uint4*>(hist);
  if constexpr (BLOCK >= 512) {
    // at most eight digits: held in registers between the scan and the walk
    uint32_t cnt[8];
    if (vec) {
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        const uint4 v = (own && 4 * g < per) ? h4[(top - 3 - 4 * g) >> 2] : make_uint4(0u, 0u, 0u, 0u);
        cnt[4 * g] = v.w;                                // digit top - 4g
        cnt[4 * g + 1] = v.z;
        cnt[4 * g + 2] = v.y;
        cnt[4 * g + 3] = v.x;
      }
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u) cnt[u] = (u < per && own) ? hist[top - u] : 0u;
    }
    uint32_t lsum = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) lsum += cnt[u];
    int total;
    const uint32_t excl = (uint32_t)block_exclusive_scan<BLOCK>((int)lsum, scan, total);
    if (own && excl < kneed && excl + lsum >= kneed) {
      uint32_t c = excl;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (u < per && c + cnt[u] >= kneed) {
          *s_bin = (uint32_t)(top - u);
          *s_krem = kneed - c;
          break;
        }
        c += cnt[u];
      }
    }
  } else {
    // more digits per thread: summed first, walked again by the one thread holding the crossing
    uint32_t lsum = 0;
    if (own) {
      if (vec) {
        for (int g = 0; g < per; g += 4) {
          const uint4 v = h4[(top - 3 - g) >> 2];
          lsum += (v.x + v.y) + (v.z + v.w);
        }
      } else {
        for (int u = 0; u < per; ++u) lsum += hist[top - u];
      }
    }
    int total;
    const uint32_t excl = (uint32_t)block_exclusive_scan<BLOCK>((int)lsum, scan, total);
    if (own && excl < kneed && excl + lsum >= kneed) {
      uint32_t c = excl;
      for (int u = 0; u < per; ++u) {
        const uint32_t cnt = hist[top - u];
        if (c + cnt >= kneed) {
          *s_bin = (uint32_t)(top - u);
          *s_krem = kneed - c;
          break;
        }
        c += cnt;
      }
    }
  }
  __syncthreads();
}

// Zeroes the 4096-bin histogram (16-byte aligned) with 16-byte stores.
template <int BLOCK>
__device__ __forceinline__ void clear_hist12(uint32_t* hist12) {
  uint4* h4 = reinterpret_cast<uint4*>(hist12);
  for (int i = threadIdx.x; i < kHist12 / 4; i += BLOCK) h4[i] = make_uint4(0u, 0u, 0u, 0u);
}

// Stable LSD radix sort of m (key, index) pairs by key, descending: four 8-bit
// passes.  Each warp owns a contiguous segment and per-(digit, warp) offsets
// keep equal keys in their input order, so ties stay in ascending index order.
// a, b: ping-pong buffers of m uint64 (key << 32 | index); hist: NW*256 uint32.
// The result ends in `a`.
template <int BLOCK>
__device__ void radix_sort_desc(uint64_t* a, uint64_t* b, uint32_t* hist, int* scan, int m) {
  constexpr int NW = BLOCK / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int seg = ((m + NW - 1) / NW + 31) & ~31;
  const int w0 = warp * seg, w1 = min(m, w0 + seg);
  const uint32_t lt = (1u << lane) - 1u;
  for (int shift = 32; shift < 64; shift += 8) {
    for (int i = threadIdx.x; i < NW * 256; i += BLOCK) hist[i] = 0u;
    __syncthreads();
    uint32_t* h = hist + warp * 256;
    for (int g = w0; g < w1; g += 32) {
      const int i = g + lane;
      const int d = i < w1 ? 255 - (int)((a[i] >> shift) & 255u) : -1;
      const uint32_t peers = same_digit_lanes(d);
      if (d >= 0 && (peers & lt) == 0u) h[d] += __popc(peers);
      __syncwarp();
    }
    __syncthreads();
    // offset[w][d] = sum over digits < d of all counts + counts of warps < w at digit d
    int tot = 0;
    if (threadIdx.x < 256) {
      const int d = threadIdx.x;
      for (int w = 0; w < NW; ++w) {
        const uint32_t c = hist[w * 256 + d];
        hist[w * 256 + d] = tot;
        tot += c;
      }
    }
    int total;
    const int base = block_exclusive_scan<BLOCK>(threadIdx.x < 256 ? tot : 0, scan, total);
    if (threadIdx.x < 256)
      for (int w = 0; w < NW; ++w) hist[w * 256 + threadIdx.x] += base;
    __syncthreads();
    for (int g = w0; g < w1; g += 32) {
      const int i = g + lane;
      uint64_t e = 0;
      int d = -1;
      if (i < w1) {
        e = a[i];
        d = 255 - (int)((e >> shift) & 255u);
      }
      const uint32_t peers = same_digit_lanes(d);
      if (d >= 0) {
        b[h[d] + __popc(peers & lt)] = e;
      }
      __syncwarp();
      if (d >= 0 && (peers & lt) == 0u) h[d] += __popc(peers);
      __syncwarp();
    }
    __syncthreads();
    uint64_t* t = a;
    a = b;
    b = t;
  }
}

template <int BLOCK, bool RANKED>
__global__ void __launch_bounds__(BLOCK, BLOCK >= 1024 ? 1 : (BLOCK >= 512 ? 3 : 6))
topk_kernel(dsa_dims d, const float* __restrict__ scores, const int32_t* __restrict__ q_pos,
            const int32_t* __restrict__ kv_start, const int32_t* __restrict__ kv_len, int k,
            int cache_cap, int cand_cap_arg, int32_t* __restrict__ idx_out, float* __restrict__ vals_out) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int cand_cap = BLOCK >= 512 ? kCand : cand_cap_arg;         // a compile-time size from 512 threads up
  const int ksel = RANKED ? k : 0;                                   // the unranked variant keeps no pairs
  uint64_t* sel = reinterpret_cast<uint64_t*>(smem_raw);            // [k]   selected (key, index)
  uint64_t* tmp = sel + ksel;                                        // [k]   sort ping-pong
  uint32_t* rhist = reinterpret_cast<uint32_t*>(tmp + ksel);         // [BLOCK/32 * 256] (ranked only)
  uint32_t* hist = rhist + (RANKED ? (BLOCK / 32) * 256 : 0);        // [256]
  int* scan = reinterpret_cast<int*>(hist + 256);                    // [64]
  uint32_t* hist12 = reinterpret_cast<uint32_t*>(scan + 64);         // [kHist12]
  uint32_t* cand = hist12 + kHist12;                                 // [cand_cap] candidate keys
  uint8_t* candw = reinterpret_cast<uint8_t*>(cand + cand_cap);      // [cand_cap] their warps
  uint32_t* cache = reinterpret_cast<uint32_t*>(candw + cand_cap);   // [cache_cap] (cand_cap % 16 == 0)
  __shared__ uint32_t s_krem, s_bin;
  __shared__ int s_ncand;
  __shared__ int s_cgt[BLOCK / 32], s_ceq[BLOCK / 32];

  // later rows see more keys (causal): launch them first so the last wave is the cheap one
  const int b = blockIdx.y, t = (int)gridDim.x - 1 - (int)blockIdx.x;
  const size_t row = (size_t)b * d.n_q + t;
  const float* srow = scores + row * d.n_kv;
  int32_t* orow = idx_out + row * k;
  float* vrow = vals_out ? vals_out + row * k : nullptr;

  KeyRange r = visible_range(q_pos[row], kv_start[b], kv_len[b], d.n_kv, d.kpool);
  const int n = r.count();
  const bool cached = n <= cache_cap;

  if (!RANKED && n <= k) {
    // every visible key is selected: the visible range, in key order
    for (int i = threadIdx.x; i < k; i += BLOCK) {
      orow[i] = i < n ? r.lo + i : DSA_INVALID;
      if (vrow) vrow[i] = i < n ? key_score(score_key(srow[r.lo + i])) : -INFINITY;
    }
    return;
  }
  if (RANKED && n <= k) {
    // every visible key is selected: rank them (inputs in index order)
    for (int i = threadIdx.x; i < n; i += BLOCK)
      sel[i] = ((uint64_t)score_key(srow[r.lo + i]) << 32) | (uint32_t)(r.lo + i);
    __syncthreads();
    radix_sort_desc<BLOCK>(sel, tmp, rhist, scan, n);
    for (int i = threadIdx.x; i < k; i += BLOCK) {
      if (i < n) {
        const uint64_t c = sel[i];
        orow[i] = (int32_t)(uint32_t)c;
        if (vrow) vrow[i] = key_score((uint32_t)(c >> 32));
      } else {
        orow[i] = DSA_INVALID;
        if (vrow) vrow[i] = -INFINITY;
      }
    }
    return;
  }

  // ---- threshold: tau = the k-th largest key.  One pass over the row (filling the cache)
  // counts the top 12 bits; the keys of the bin holding the k-th largest then become a small
  // candidate set, and the low 20 bits are resolved over it alone (12 + 8 bits).
  TOPK_TRACE(0);
  clear_hist12<BLOCK>(hist12);
  if (threadIdx.x == 0) s_ncand = 0;
  __syncthreads();
  {
    // the row as 16-byte vectors (eight in flight per thread) between a scalar head and tail
    auto one = [&](int i) {
      const uint32_t key = score_key(__ldg(srow + r.lo + i));
      if (cached) cache[i] = key;
      atomicAdd(&hist12[key >> 20], 1u);
    };
    const int head = min(n, (int)(((16u - ((uint32_t)(uintptr_t)(srow + r.lo) & 15u)) & 15u) >> 2));
    const int nv = (n - head) >> 2;
    const float4* s4 = reinterpret_cast<const float4*>(srow + r.lo + head);
    if ((int)threadIdx.x < head) one(threadIdx.x);
    constexpr int kV = BLOCK >= 1024 ? 8 : 4;   // 16-byte loads in flight per thread (rows of n_kv <= 8192 take 512)
    for (int base = threadIdx.x; base < nv; base += BLOCK * kV) {
      float4 v[kV];
#pragma unroll
      for (int u = 0; u < kV; ++u) {
        const int j = base + u * BLOCK;
        v[u] = j < nv ? __ldg(s4 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kV; ++u) {
        const int j = base + u * BLOCK;
        if (j < nv) {
          const int i = head + 4 * j;
          const uint32_t k0 = score_key(v[u].x), k1 = score_key(v[u].y), k2 = score_key(v[u].z),
                         k3 = score_key(v[u].w);
          if (cached) {
            if (head == 0) {
              *reinterpret_cast<uint4*>(cache + i) = make_uint4(k0, k1, k2, k3);
            } else {
              cache[i] = k0;
              cache[i + 1] = k1;
              cache[i + 2] = k2;
              cache[i + 3] = k3;
            }
          }
          atomicAdd(&hist12[k0 >> 20], 1u);
          atomicAdd(&hist12[k1 >> 20], 1u);
          atomicAdd(&hist12[k2 >> 20], 1u);
          atomicAdd(&hist12[k3 >> 20], 1u);
        }
      }
    }
    const int t0 = head + 4 * nv;
    if ((int)threadIdx.x < n - t0) one(t0 + threadIdx.x);
  }
  __syncthreads();
  TOPK_TRACE(1);
  find_crossing<BLOCK>(hist12, kHist12, (uint32_t)k, scan, &s_bin, &s_krem);
  const uint32_t b1 = s_bin, krem1 = s_krem;
  TOPK_TRACE(2);
  const uint32_t nb1 = hist12[b1];
  // each warp owns a contiguous segment of the row, walked 128 keys at a time (the output order
  // of equal keys is their index order)
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int NW = BLOCK / 32;
  const int wseg = ((n + NW - 1) / NW + 31) & ~31;
  const int w0 = warp * wseg;
  const int w1 = min(n, w0 + wseg);
  const bool few = nb1 <= (uint32_t)cand_cap;
  int gt12 = 0;                                       // keys of this warp whose top 12 bits exceed b1
  uint32_t prefix = 0u;
  if (few) {
    // collect the bin's keys with their warp, and count the keys above the bin per warp
    if (threadIdx.x < NW) {
      s_cgt[threadIdx.x] = 0;
      s_ceq[threadIdx.x] = 0;
    }
    // four keys per lane per step (independent loads and ballots); the order of the candidates
    // does not matter, each carries its warp
    for (int b0 = w0; b0 < w1; b0 += 128) {
      uint32_t key[4], m[4];
      bool in[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = b0 + 32 * q + lane;
        key[q] = i < w1 ? (cached ? cache[i] : score_key(srow[r.lo + i])) : 0u;
        in[q] = i < w1 && (key[q] >> 20) == b1;
        gt12 += (i < w1 && (key[q] >> 20) > b1) ? 1 : 0;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) m[q] = __ballot_sync(0xffffffffu, in[q]);
      const int tot = __popc(m[0]) + __popc(m[1]) + __popc(m[2]) + __popc(m[3]);
      if (tot) {
        int slot = 0;
        if (lane == 0) slot = atomicAdd(&s_ncand, tot);
        slot = __shfl_sync(0xffffffffu, slot, 0);
        const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (in[q]) {
            const int c = slot + __popc(m[q] & lt);
            cand[c] = key[q];
            candw[c] = (uint8_t)warp;
          }
          slot += __popc(m[q]);
        }
      }
    }
    gt12 = __reduce_add_sync(0xffffffffu, gt12);
    __syncthreads();
    TOPK_TRACE(3);
    // bits 19..8 of the candidates
    clear_hist12<BLOCK>(hist12);
    __syncthreads();
    for (int c = threadIdx.x; c < (int)nb1; c += BLOCK) atomicAdd(&hist12[(cand[c] >> 8) & 4095u], 1u);
    __syncthreads();
    find_crossing<BLOCK>(hist12, kHist12, krem1, scan, &s_bin, &s_krem);
    const uint32_t b2 = s_bin, krem2 = s_krem;
    // bits 7..0 of the candidates whose bits 19..8 are b2
    for (int i = threadIdx.x; i < 256; i += BLOCK) hist[i] = 0u;
    __syncthreads();
    for (int c = threadIdx.x; c < (int)nb1; c += BLOCK)
      if (((cand[c] >> 8) & 4095u) == b2) atomicAdd(&hist[cand[c] & 255u], 1u);
    __syncthreads();
    find_crossing<BLOCK>(hist, 256, krem2, scan, &s_bin, &s_krem);
    prefix = (b1 << 20) | (b2 << 8) | s_bin;
    // per warp: the bin's keys above and equal to tau
    for (int c = threadIdx.x; c < (int)nb1; c += BLOCK) {
      if (cand[c] > prefix) atomicAdd(&s_cgt[candw[c]], 1);
      else if (cand[c] == prefix) atomicAdd(&s_ceq[candw[c]], 1);
    }
    __syncthreads();
  } else {
    // a crowded bin (more than cand_cap keys share the top 12 bits, e.g. near-equal scores): bits 19..8 of
    // the bin's keys, then bits 7..0 of the keys under that 24-bit prefix, each one filtered pass over
    // the row with plain shared atomics (the same digits the candidate path resolves)
    clear_hist12<BLOCK>(hist12);
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += BLOCK) {
      const uint32_t key = cached ? cache[i] : score_key(srow[r.lo + i]);
      if ((key >> 20) == b1) atomicAdd(&hist12[(key >> 8) & 4095u], 1u);
    }
    __syncthreads();
    find_crossing<BLOCK>(hist12, kHist12, krem1, scan, &s_bin, &s_krem);
    const uint32_t p24 = (b1 << 12) | s_bin, krem2 = s_krem;
    for (int i = threadIdx.x; i < 256; i += BLOCK) hist[i] = 0u;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += BLOCK) {
      const uint32_t key = cached ? cache[i] : score_key(srow[r.lo + i]);
      if ((key >> 8) == p24) atomicAdd(&hist[key & 255u], 1u);
    }
    __syncthreads();
    find_crossing<BLOCK>(hist, 256, krem2, scan, &s_bin, &s_krem);
    prefix = (p24 << 8) | s_bin;
  }
  TOPK_TRACE(4);
#ifdef DSA_TRACE
  if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.x < 8)
    g_topk_trace[blockIdx.x][7] = ((unsigned long long)few << 32) | nb1;
#endif
  const uint32_t tau = prefix;
  const int need_eq = (int)s_krem;  // keys equal to tau still to take (lowest indices first)
  const int n_gt = k - need_eq;

  // ---- gather: per-warp counts of keys > tau and == tau (from the collection pass, or one
  // more pass over a crowded row), then every warp places its keys
  int c_gt = 0, c_eq = 0;
  if (few) {
    c_gt = gt12 + s_cgt[warp];
    c_eq = s_ceq[warp];
  } else {
    for (int i = w0 + lane; i < w1; i += 32) {
      uint32_t key = cached ? cache[i] : score_key(srow[r.lo + i]);
      c_gt += key > tau;
      c_eq += key == tau;
    }
    c_gt = __reduce_add_sync(0xffffffffu, c_gt);
    c_eq = __reduce_add_sync(0xffffffffu, c_eq);
  }
  TOPK_TRACE(5);
  // the warps' counts, scanned by every warp itself (one barrier): keys of earlier warps above / equal to tau
  if (lane == 0) {
    scan[warp] = c_gt;
    scan[32 + warp] = c_eq;
  }
  __syncthreads();
  int gt_base, eq_base;
  {
    const int g = lane < NW ? scan[lane] : 0, e = lane < NW ? scan[32 + lane] : 0;
    int sg = g, se = e;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int yg = __shfl_up_sync(0xffffffffu, sg, o), ye = __shfl_up_sync(0xffffffffu, se, o);
      if (lane >= o) {
        sg += yg;
        se += ye;
      }
    }
    gt_base = __shfl_sync(0xffffffffu, sg - g, warp);
    eq_base = __shfl_sync(0xffffffffu, se - e, warp);
  }
  const uint32_t lt_mask = (1u << lane) - 1u;
  if constexpr (!RANKED) {
    if (c_eq == 0) {
      // no key of this warp equals tau (the usual case): a key is taken iff it is above tau, after
      // every taken key of the earlier warps; one ballot per four keys
      int base = gt_base + min(eq_base, need_eq);
      for (int b0 = w0; b0 < w1; b0 += 128) {
        uint32_t key[4], m[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int i = b0 + 32 * q + lane;
          key[q] = i < w1 ? (cached ? cache[i] : score_key(srow[r.lo + i])) : 0u;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) m[q] = __ballot_sync(0xffffffffu, b0 + 32 * q + lane < w1 && key[q] > tau);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if ((m[q] >> lane) & 1u) {
            const int pos = base + __popc(m[q] & lt_mask);
            orow[pos] = r.lo + b0 + 32 * q + lane;
            if (vrow) vrow[pos] = key_score(key[q]);
          }
          base += __popc(m[q]);
        }
      }
      TOPK_TRACE(6);
      return;
    }
    // ascending key order: key i goes to (#gt before i) + min(#eq before i, need_eq); four keys
    // per lane per step, their loads and ballots independent
    for (int b0 = w0; b0 < w1; b0 += 128) {
      uint32_t key[4], m_gt[4], m_eq[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = b0 + 32 * q + lane;
        key[q] = i < w1 ? (cached ? cache[i] : score_key(srow[r.lo + i])) : 0u;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = b0 + 32 * q + lane;
        m_gt[q] = __ballot_sync(0xffffffffu, i < w1 && key[q] > tau);
        m_eq[q] = __ballot_sync(0xffffffffu, i < w1 && key[q] == tau);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = b0 + 32 * q + lane;
        const bool is_gt = (m_gt[q] >> lane) & 1u, is_eq = (m_eq[q] >> lane) & 1u;
        const int gt_before = gt_base + __popc(m_gt[q] & lt_mask);
        const int eq_before = eq_base + __popc(m_eq[q] & lt_mask);
        if (is_gt || (is_eq && eq_before < need_eq)) {
          const int pos = gt_before + min(eq_before, need_eq);
          orow[pos] = r.lo + i;
          if (vrow) vrow[pos] = key_score(key[q]);
        }
        gt_base += __popc(m_gt[q]);
        eq_base += __popc(m_eq[q]);
      }
    }
    TOPK_TRACE(6);
  } else {
    for (int b0 = w0; b0 < w1; b0 += 32) {
      const int i = b0 + lane;
      uint32_t key = 0u;
      if (i < w1) key = cached ? cache[i] : score_key(srow[r.lo + i]);
      const bool is_gt = i < w1 && key > tau;
      const bool is_eq = i < w1 && key == tau;
      const uint32_t m_gt = __ballot_sync(0xffffffffu, is_gt);
      const uint32_t m_eq = __ballot_sync(0xffffffffu, is_eq);
      const uint64_t c = ((uint64_t)key << 32) | (uint32_t)(r.lo + i);
      if (is_gt) sel[gt_base + __popc(m_gt & lt_mask)] = c;
      if (is_eq) {
        int rank = eq_base + __popc(m_eq & lt_mask);
        if (rank < need_eq) sel[n_gt + rank] = c;
      }
      gt_base += __popc(m_gt);
      eq_base += __popc(m_eq);
    }
    __syncthreads();
    // gt keys came first in index order, then the taken tau keys in index order:
    // the stable sort keeps every run of equal keys in ascending index order
    radix_sort_desc<BLOCK>(sel, tmp, rhist, scan, k);
    for (int i = threadIdx.x; i < k; i += BLOCK) {
      const uint64_t c = sel[i];
      orow[i] = (int32_t)(uint32_t)c;
      if (vrow) vrow[i] = key_score((uint32_t)(c >> 32));
    }
  }
}

namespace {
template <int BLOCK, bool RANKED>
cudaError_t launch_topk_t(const dsa_dims& d, const float* scores, const int32_t* q_pos, const int32_t* kv_start,
                          const int32_t* kv_len, int k, int32_t* idx, float* vals, cudaStream_t st) {
  int cache_cap = d.n_kv < kTopkCacheMax ? d.n_kv : kTopkCacheMax;
  // short rows (256-thread blocks, six per SM) keep a candidate buffer of half a row, at least 1024 keys:
  // a threshold bin holding more takes the crowded-bin passes instead (the same result)
  int cand_cap = kCand;
  if (BLOCK <= 256) cand_cap = std::min(kCand, std::max(1024, ((d.n_kv / 2) + 15) & ~15));
  const size_t fixed = (RANKED ? (size_t)k * 16 + (size_t)(BLOCK / 32) * 256 * 4 : 0) + 256 * 4 + 64 * 4 +
                       (size_t)(kHist12 + cand_cap) * 4 + cand_cap;
  if (fixed + (size_t)cache_cap * 4 > 220 * 1024) cache_cap = (int)((220 * 1024 - fixed) / 4);
  const size_t smem = fixed + (size_t)cache_cap * 4;
  auto kern = topk_kernel<BLOCK, RANKED>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(d.n_q, d.batch), BLOCK, smem, st>>>(d, scores, q_pos, kv_start, kv_len, k, cache_cap, cand_cap, idx,
                                                  vals);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_topk(const dsa_dims& d, const float* scores, const int32_t* q_pos,
                        const int32_t* kv_start, const int32_t* kv_len, int k, int32_t* idx,
                        float* vals, bool ranked, cudaStream_t st) {
  if (d.n_kv > 8192)
    return ranked ? launch_topk_t<1024, true>(d, scores, q_pos, kv_start, kv_len, k, idx, vals, st)
                  : launch_topk_t<1024, false>(d, scores, q_pos, kv_start, kv_len, k, idx, vals, st);
  if (d.n_kv > 4096)
    return ranked ? launch_topk_t<512, true>(d, scores, q_pos, kv_start, kv_len, k, idx, vals, st)
                  : launch_topk_t<512, false>(d, scores, q_pos, kv_start, kv_len, k, idx, vals, st);
  return ranked ? launch_topk_t<256, true>(d, scores, q_pos, kv_start, kv_len, k, idx, vals, st)
                : launch_topk_t<256, false>(d, scores, q_pos, kv_start, kv_len, k, idx, vals, st);
}

}  // namespace dsa

#ifdef DSA_TRACE
extern "C" int dsa_topk_trace_read(unsigned long long* host) {
  return (int)cudaMemcpyFromSymbol(host, dsa::g_topk_trace, sizeof(dsa::g_topk_trace));
}
#endif
