// S4 sparse MLA attention on the 5th-generation tensor cores (tcgen05).
//
// out[b,t,h,:] = sum_{i in U} softmax_i(scale * q[b,t,h,:] . c_i) c_i[:vd], U = the
// distinct valid entries of idx[b,t,:] (fak note "GLM-5.2: the DSA sparse
// attention moves onto the pure fak kernel", "What changed": online softmax,
// key width kd != value width vd; metrale glm5next_dsa_ref topk_to_mask and
// mla_masked_attention).  The key is the shared latent row c_i (kd = 512 or
// 576 columns) and the value is its first vd = 512 columns.
//
// Heads are the MMA M dimension (128 rows; fewer heads leave rows unused).  A
// 128 x 512 fp32 output accumulator fills all of one SM's tensor memory, so a
// query is processed by a cluster of two CTAs, each owning half of the value
// columns and the matching half of the key columns:
//   rank 0: latent columns [0,256)   (+ rope columns [512,544) when kd = 576), O[:, 0:256)
//   rank 1: latent columns [256,512) (+ rope columns [544,576) when kd = 576), O[:, 256:512)
// Each CTA gathers only its own columns of every selected latent row (TMA
// tile::gather4, four rows per instruction, straight into the swizzled operand
// layout), so no byte is loaded twice.  Per 64-key chunk each CTA computes the q.k partial over its columns;
// the two fp32 partial tiles are exchanged through distributed shared memory
// and summed (fp32 addition is commutative, so both CTAs see bit-identical
// scores and take identical online-softmax decisions).  The exchange uses
// st.async, which completes the peer's barrier by byte count, so the sender
// never waits for a round trip.  A tile travels in two 16 KB halves (keys 0-31
// and 32-63), each with its own barriers, laid out by head quarter
// ([half][quarter][key/4][32 heads][4 keys] fp32): the first half also holds the
// chunk's P (below) and returns to the peer after P.V, the second returns as
// soon as the softmax has read it.
//
// Tensor memory (512 columns): score buffers 0-63 and 64-127, the CTA's four
// value-side query blocks 128-255 as the A operand of q.k (two bf16 per
// column), O 256-511.  The 32 rope columns of each CTA use a 64-byte-swizzled
// shared-memory operand.
// The bf16 probabilities go to the first 16 KB of the chunk's exchange tile (its
// fp32 partial scores are consumed by then), as a 128-byte-swizzled K-major
// operand of P.V: a score buffer is free again as soon as it has been read, so
// the q.k two chunks ahead never waits for P.V, and the exchange tile returns
// to the peer once P.V has read it.  Every tcgen05.mma here costs about
// 100 cycles whatever its N up to 128, so q.k uses N = 64 keys per instruction
// and P.V N = 256 value columns.  The running maximum only moves (and O is
// rescaled in TMEM) when it grows by more than 2^8.
//
// Warp roles per CTA: warps 0-3 and 13-16 run the softmax and the epilogue (one
// head row per thread, TMEM lanes 0-127; the two groups take the two halves of
// every chunk's keys and of O, and the two warps of a head quarter agree on its
// row maxima through their own barrier, after which the quarter's P rows
// overwrite exactly its consumed half-0 scores; with H = 64 the warps of the two
// padding quarters take part in no per-chunk barrier); warps 9-12 load the query columns into TMEM,
// read the same score rows and push them to the peer (buffer reuse is
// acknowledged by the peer); warp 4 issues tcgen05.mma from a polling scheduler
// (and loads the CTA's rope query columns by TMA); warps 5-8 stage and
// deduplicate the index row, then issue the TMA gathers of value blocks 0-2
// (TMA runs them off the load/store pipe that the softmax and exchange warps
// use, but each gather costs its issuing warp about 60 ns); warps 17-19 issue
// those of value block 3 and the rope columns, so that seven warps share the 80
// gathers of a chunk.
// Every mbarrier wait is bounded.
#include <cuda.h>

#include "dsa_common.cuh"
#include "dsa_internal.h"
#include "dsa_sm100.cuh"

namespace dsa {

#ifdef DSA_TRACE
// Optional per-chunk timeline of the first cluster (build with -DDSA_TRACE):
// g_attend_trace[cta rank][event][chunk] = %globaltimer.
__device__ unsigned long long g_attend_trace[2][16][512];
// g_attend_span[cta][0] = entry, [1] = exit (%globaltimer), every CTA
__device__ unsigned long long g_attend_span[1024][2];
#define TRACE(ev, j)                                                                             \
  do {                                                                                           \
    if (blockIdx.x < 2 && (j) < 512) g_attend_trace[blockIdx.x & 1][ev][(j)] = sm100::globaltimer(); \
  } while (0)
#else
#define TRACE(ev, j) ((void)0)
#endif

namespace {

using namespace sm100;

constexpr int kChunk = 64;             // keys per pipeline step (N of q.k, K of P.V)
constexpr int kStages = 4;             // gathered key/value stages
constexpr int kBlockBytes = kChunk * 128;                   // one 64-col block of a stage: 8 KB
constexpr int kRopeOff = 4 * kBlockBytes;                   // 32 rope columns after the 4 value blocks
constexpr int kStageBytes = kRopeOff + kChunk * 64;         // 36 KB
constexpr int kQRopeBytes = 128 * 64;                       // rope query columns in smem: 8 KB
// exchange tile, fp32 [key half][head quarter][key/4 within the half][32 heads][4 keys]: 32 KB; the P rows
// of a head quarter (128-byte rows at the start of the tile) cover exactly that quarter's half-0 scores
constexpr int kXBytes = kChunk * 128 * 4;
constexpr int kNarrowKeys = 65536;                          // key lists of 16-bit entries up to here
constexpr int kMaxKeys = kStageBytes * 8;                   // 294912: the dedupe bitmap fits one stage
constexpr int kQCol = 128;                                  // query columns in TMEM
constexpr int kOCol = 256;                                  // output accumulator
constexpr int kThreads = 640;          // 20 warps (registers are granted per 4 warps: 17 cost as much)
constexpr int kProducerThreads = 128;  // warps 5-8: key lists and TMA gathers of value blocks 0-2
constexpr int kCopyWarps = 3;          // warps 17-19: TMA gathers of value block 3 and the rope columns

struct AttTcParams {
  int B, T, S, H, kd, width;
  long long stride;          // latent row stride in elements
  const bf16* latent;
  const bf16* q;             // [B,T,H,kd]
  const int32_t* idx;
  float scale_log2;          // softmax scale * log2(e)
  bf16* out;                 // [B,T,H,512]
  float* lse;                // [B,T,H] or null
  int* status;
  int list_bitmap;           // 1: the dedupe bitmap fits in the key-list buffer
  int out_v8;                // 1: out is 32-byte aligned (256-bit stores)
  int list_nbytes;           // key-list buffer size in shared memory (list_bytes)
  int list_hi_off;           // byte offset of the high parts in the key-list buffer (S > 65536)
};

// Key-list buffer: width uint16 entries (the low 16 bits of each key) and, when S > 65536, width
// uint8 high parts after them; grown to hold the dedupe bitmap of S keys when `with_bitmap` (then
// the bitmap needs no gather stage).
inline size_t list_lo_bytes(int width) { return ((size_t)width * 2 + 15) & ~(size_t)15; }
inline size_t list_bytes(int width, int S, bool with_bitmap) {
  size_t b = list_lo_bytes(width) + (S > kNarrowKeys ? (((size_t)width + 15) & ~(size_t)15) : 0);
  const size_t bm = (size_t)((S + 31) / 32) * 4;
  if (with_bitmap && bm > b) b = bm;
  return (b + 15) & ~(size_t)15;
}

struct Smem {
  uint32_t kv, x, qrope;     // shared-window addresses
  uint16_t* list;            // deduplicated key rows of the row being gathered: low 16 bits (then
                             // bits 16-23 of each entry when S > 65536, see put_key)
  int* wcount;               // 4 per-warp counts of the list compaction
  float* mx;                 // [2 parities][2 groups][128 rows] half-row maxima
  float* lsum;               // [2 groups][128 rows] partial row sums for the epilogue
  uint64_t *qfull, *qrope_full, *list_ready, *list_taken, *kv_full, *kv_empty, *s_full, *s_read, *p_full, *o_done,
      *o_free, *xfull, *xfree, *xread1, *mxready, *lready, *drain, *list_free;
  uint32_t* tmem_slot;
  int* n_list;               // [2]: list length of the published row, by row parity
  int* dup_flag;
  int* abort_flag;
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t map_peer(uint32_t addr, uint32_t peer) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(peer));
  return r;
}
__device__ __forceinline__ void st_async_v4(uint32_t addr, const uint32_t* v, uint32_t remote_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(addr),
               "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(remote_bar)
               : "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, const uint32_t* v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3])
               : "memory");
}
__device__ __forceinline__ void st_global_v8(void* ptr, const uint32_t* v) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(ptr), "r"(v[0]), "r"(v[1]),
               "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
__device__ __forceinline__ void arrive_remote_relaxed(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ bool try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool wait_cluster(uint32_t bar, uint32_t parity, int* status, volatile int* abort_flag) {
  if (try_wait_cluster(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (try_wait_cluster(bar, parity)) return true;
    if ((it & 63u) == 0u) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > kWaitLimitNs) {
        record_status(status, DSA_ERR_TIMEOUT);
        *abort_flag = 1;
        return false;
      }
    }
  }
}
// Named barrier that also returns whether any participating thread passed `pred`
// (bar.red.or): the producer warps take every early exit together.
__device__ __forceinline__ bool named_any(int id, int n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}


// Row list construction, by the 128 producer threads (warps 5-8): the distinct in-range
// entries of the index row in index-row order.  Deterministic, so both CTAs of the
// cluster obtain the same list.  Entry e = w*q + 32*it + lane belongs to warp w; rows of
// up to 2176 entries are read from global memory once into registers.
constexpr int kListCache = 17;  // rows of up to 2176 entries (top_k 2048; kpool widths 2051)

struct RowKeys {
  int q, e0, e1;
  bool cached;
  int key[kListCache];
};

// The high parts sit after the low parts (list_lo_bytes(width) = p.list_hi_off bytes in).
template <bool kWide>
__device__ __forceinline__ void put_key(const AttTcParams& p, const Smem& sm, int pos, int key) {
  sm.list[pos] = (uint16_t)key;
  if (kWide) (reinterpret_cast<uint8_t*>(sm.list) + p.list_hi_off)[pos] = (uint8_t)(key >> 16);
}
template <bool kWide>
__device__ __forceinline__ int get_key(const AttTcParams& p, const Smem& sm, int pos) {
  if (!kWide) return (int)sm.list[pos];
  return ((int)(reinterpret_cast<const uint8_t*>(sm.list) + p.list_hi_off)[pos] << 16) | (int)sm.list[pos];
}

__device__ void load_row(const AttTcParams& p, const int32_t* irow, RowKeys& rk) {
  const int tid = threadIdx.x - 5 * 32, lane = threadIdx.x & 31, w = tid >> 5;
  rk.q = (((p.width + 3) >> 2) + 31) & ~31;
  rk.e0 = w * rk.q;
  rk.e1 = min(p.width, rk.e0 + rk.q);
  rk.cached = rk.q <= 32 * kListCache;
  if (rk.cached) {
#pragma unroll
    for (int it = 0; it < kListCache; ++it) {
      const int e = rk.e0 + 32 * it + lane;
      rk.key[it] = e < rk.e1 ? __ldg(irow + e) : -1;
    }
  }
}

// Marks every in-range key in `bitmap` (cleared first); returns whether any key repeats.
__device__ bool mark_keys(const AttTcParams& p, const int32_t* irow, const RowKeys& rk, uint32_t* bitmap) {
  const int tid = threadIdx.x - 5 * 32, lane = threadIdx.x & 31;
  const int words = (p.S + 31) >> 5;
  for (int i = tid; i < words; i += kProducerThreads) bitmap[i] = 0u;
  named_sync(1, kProducerThreads);
  bool dup = false;
  if (rk.cached) {
#pragma unroll
    for (int it = 0; it < kListCache; ++it) {
      const int key = rk.key[it];
      if (key >= 0 && key < p.S) {
        const uint32_t bit = 1u << (key & 31);
        dup |= (atomicOr(&bitmap[key >> 5], bit) & bit) != 0u;
      }
    }
  } else {
    for (int b = rk.e0; b < rk.e1; b += 32) {
      const int e = b + lane;
      const int key = e < rk.e1 ? __ldg(irow + e) : -1;
      if (key >= 0 && key < p.S) {
        const uint32_t bit = 1u << (key & 31);
        dup |= (atomicOr(&bitmap[key >> 5], bit) & bit) != 0u;
      }
    }
  }
  return named_any(1, kProducerThreads, dup);
}

// No repeated key: keep every in-range entry.  Each warp compacts its contiguous quarter of
// the row 32 entries at a time (ballots), after a scan of the four quarters' counts.
template <bool kWide>
__device__ int compact_unique(const AttTcParams& p, const Smem& sm, const int32_t* irow, const RowKeys& rk) {
  const int tid = threadIdx.x - 5 * 32, lane = threadIdx.x & 31, w = tid >> 5;
  const uint32_t below = (1u << lane) - 1u;
  int cnt = 0;
  if (rk.cached) {
#pragma unroll
    for (int it = 0; it < kListCache; ++it)
      cnt += __popc(__ballot_sync(0xffffffffu, rk.key[it] >= 0 && rk.key[it] < p.S));
  } else {
    for (int b = rk.e0; b < rk.e1; b += 32) {
      const int e = b + lane;
      const int key = e < rk.e1 ? __ldg(irow + e) : -1;
      cnt += __popc(__ballot_sync(0xffffffffu, key >= 0 && key < p.S));
    }
  }
  if (lane == 0) sm.wcount[w] = cnt;
  named_sync(1, kProducerThreads);   // counts visible; every thread is past the bitmap
  int base = 0;
  for (int k = 0; k < w; ++k) base += sm.wcount[k];
  const int total = sm.wcount[0] + sm.wcount[1] + sm.wcount[2] + sm.wcount[3];
  if (rk.cached) {
#pragma unroll
    for (int it = 0; it < kListCache; ++it) {
      const int key = rk.key[it];
      const bool keep = key >= 0 && key < p.S;
      const uint32_t m = __ballot_sync(0xffffffffu, keep);
      if (keep) put_key<kWide>(p, sm, base + __popc(m & below), key);
      base += __popc(m);
    }
  } else {
    for (int b = rk.e0; b < rk.e1; b += 32) {
      const int e = b + lane;
      const int key = e < rk.e1 ? __ldg(irow + e) : -1;
      const bool keep = key >= 0 && key < p.S;
      const uint32_t m = __ballot_sync(0xffffffffu, keep);
      if (keep) put_key<kWide>(p, sm, base + __popc(m & below), key);
      base += __popc(m);
    }
  }
  named_sync(1, kProducerThreads);   // the counts are read before the next row rewrites them
  return total;
}

// Repeated keys: order-preserving compaction by one warp, first occurrence only (not seen in
// an earlier group of 32, lowest lane within its group).  `bitmap` must not overlap the list.
template <bool kWide>
__device__ int compact_first(const AttTcParams& p, const Smem& sm, const int32_t* irow, uint32_t* bitmap) {
  const int tid = threadIdx.x - 5 * 32, lane = threadIdx.x & 31;
  const int words = (p.S + 31) >> 5;
  for (int i = tid; i < words; i += kProducerThreads) bitmap[i] = 0u;
  named_sync(1, kProducerThreads);
  if (tid < 32) {
    int n = 0;
    for (int e0 = 0; e0 < p.width; e0 += 32) {
      const int e = e0 + lane;
      const int key = e < p.width ? __ldg(irow + e) : -1;
      bool keep = key >= 0 && key < p.S;
      const uint32_t peers = __match_any_sync(0xffffffffu, keep ? key : -1);
      if (keep) keep = (bitmap[key >> 5] & (1u << (key & 31))) == 0u && lane == __ffs(peers) - 1;
      __syncwarp();
      if (keep) atomicOr(&bitmap[key >> 5], 1u << (key & 31));
      const uint32_t m = __ballot_sync(0xffffffffu, keep);
      if (keep) put_key<kWide>(p, sm, n + __popc(m & ((1u << lane) - 1u)), key);
      n += __popc(m);
      __syncwarp();
    }
    if (lane == 0) sm.wcount[0] = n;
  }
  named_sync(1, kProducerThreads);
  const int total = sm.wcount[0];
  named_sync(1, kProducerThreads);
  return total;
}

// Persistent: cluster c (of gridDim.x / 2) processes query rows c, c + #clusters, ...
// All per-chunk barriers run on a global chunk counter across the cluster's rows, so
// the next row's list build, query load and first gathers overlap the current row's
// last chunks, and a row's epilogue overlaps the next row's first q.k.
// kHalfHeads: H = 64, so the head rows 64-127 of the M = 128 tiles are padding; the warps that own
// them skip their softmax and exchange work (separate instantiation, so H = 128 pays nothing).
// kWide: S > 65536, so list entries carry an 8-bit high part (separate instantiation as well).
template <bool kHalfHeads, bool kWide>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
attend_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_kv,
                 const __grid_constant__ CUtensorMap map_rope, AttTcParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ int s_misc[5];
#ifdef DSA_TRACE
  if (threadIdx.x == 0 && blockIdx.x < 1024) g_attend_span[blockIdx.x][0] = sm100::globaltimer();
#endif
  __shared__ int s_wcount[4];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* gb = smem_raw + (base - raw);
  Smem sm;
  sm.x = base;                                   // peer-written: same offset in both CTAs
  sm.qrope = sm.x + 2 * kXBytes;
  sm.kv = sm.qrope + kQRopeBytes;
  uint32_t off = sm.kv + kStages * kStageBytes - base;
  sm.list = reinterpret_cast<uint16_t*>(gb + off);
  off += (uint32_t)p.list_nbytes;
  sm.mx = reinterpret_cast<float*>(gb + off);
  off += 2 * 2 * 128 * 4;
  sm.lsum = reinterpret_cast<float*>(gb + off);
  off += 2 * 128 * 4;
  uint64_t* bars = reinterpret_cast<uint64_t*>(gb + off);
  sm.qfull = bars;
  sm.qrope_full = bars + 1;
  sm.list_ready = bars + 2;
  sm.list_taken = bars + 3;
  sm.kv_full = bars + 4;
  sm.kv_empty = sm.kv_full + kStages;
  sm.s_full = sm.kv_empty + kStages;
  sm.s_read = sm.s_full + 2;
  sm.p_full = sm.s_read + 2;
  sm.o_done = sm.p_full + 2;
  sm.xfull = sm.o_done + 2;                      // [buffer][half]
  sm.xfree = sm.xfull + 4;                       // [buffer][half]
  sm.xread1 = sm.xfree + 4;
  sm.mxready = sm.xread1 + 2;                    // [buffer][head quarter]
  sm.o_free = sm.mxready + 8;
  sm.lready = sm.o_free + 1;
  sm.drain = sm.lready + 1;
  sm.list_free = sm.drain + 1;
  sm.tmem_slot = reinterpret_cast<uint32_t*>(sm.list_free + 1);
  sm.n_list = &s_misc[0];                        // [0], [1]
  sm.dup_flag = &s_misc[2];
  sm.abort_flag = &s_misc[3];
  sm.wcount = s_wcount;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const uint32_t peer = rank ^ 1u;
  const bool rope = p.kd == 576;                 // each CTA owns 32 of the 64 rope columns
  const int rope_col = 512 + 32 * (int)rank;
  const long long n_rows = (long long)p.B * p.T;
  const int ncl = (int)(gridDim.x >> 1), cid = (int)(blockIdx.x >> 1);
  const int my_rows = n_rows > cid ? (int)((n_rows - 1 - cid) / ncl + 1) : 0;
  auto row_of = [&](int i) { return (size_t)cid + (size_t)i * ncl; };

  if (threadIdx.x == 0) {
    *sm.abort_flag = 0;
    mbar_init(smem_u32(sm.qfull), 4);            // per row: each exchange warp's Q rows are in TMEM
    mbar_init(smem_u32(sm.qrope_full), 1);
    mbar_init(smem_u32(sm.list_ready), 1);       // per row: the producer published n_list
    mbar_init(smem_u32(sm.list_taken), 13);      // per row: MMA + 8 softmax + 4 exchange warps read it
    mbar_init(smem_u32(sm.o_free), 8);           // per non-empty row: the epilogue has read O
    mbar_init(smem_u32(sm.lready), 8);
    for (int s = 0; s < kStages; ++s) {
      // one expect-tx arrival per gathering warp set (warps 5-8, then each of warps 17-19); the
      // TMA gathers complete the bytes
      mbar_init(smem_u32(&sm.kv_full[s]), 1 + kCopyWarps);
      mbar_init(smem_u32(&sm.kv_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&sm.s_full[s]), 1);
      // softmax warps that own real head rows: all 8, or those of the first two quarters when H = 64
      const uint32_t n_sm = kHalfHeads ? 4u : 8u;
      mbar_init(smem_u32(&sm.s_read[s]), 4 + n_sm);  // the exchange and softmax warps have read the score buffer
      mbar_init(smem_u32(&sm.p_full[s]), n_sm);   // both softmax groups wrote their P columns
      for (int q = 0; q < 4; ++q) mbar_init(smem_u32(&sm.mxready[4 * s + q]), 2);  // the quarter's two softmax warps
      mbar_init(smem_u32(&sm.o_done[s]), 1);
      for (int h = 0; h < 2; ++h) {
        mbar_init(smem_u32(&sm.xfull[2 * s + h]), 1);  // armed by our softmax; completed by the peer's st.async bytes
        mbar_init(smem_u32(&sm.xfree[2 * s + h]), 4);  // one arrival per peer exchange warp
      }
      mbar_init(smem_u32(&sm.xread1[s]), n_sm / 2);  // the group-1 softmax warps have read half 1
    }
    mbar_init(smem_u32(sm.drain), 1);
    mbar_init(smem_u32(sm.list_free), kCopyWarps);  // per row: warps 17-19 are done with its list
    fence_barrier_init();
    for (int s = 0; s < 4; ++s) mbar_arrive_expect_tx(smem_u32(&sm.xfull[s]), 32u * p.H * 4u);  // first use of each half
  }
  if (warp == 4) tmem_alloc(smem_u32(sm.tmem_slot), 512);
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer's barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_slot;
  volatile int* abort_flag = sm.abort_flag;
  if (threadIdx.x == 0) TRACE(8, 0);

  if (warp >= 5 && warp <= 8) {
    // ---------------------------------------------------------------- lists + gathers
    const int w = warp - 5;                              // 0..3: gathers 12w..12w+11 of each chunk
    if (lane == 0) tma_prefetch_desc(&map_kv);
    long long gc = 0;                                    // global chunk counter
    bool ok = true;
    // a row's index entries are read into registers while the previous row's gathers are issued
    RowKeys rk;
    if (my_rows > 0) load_row(p, p.idx + row_of(0) * p.width, rk);
    for (int i = 0; i < my_rows; ++i) {
      const size_t row = row_of(i);
      const int32_t* irow = p.idx + row * p.width;
      // every consumer has read the previous row's length before this row's is published, and the
      // copy warps have issued the previous row's copies (they read its list)
      const int s0 = (int)(gc % kStages);
      bool got = true;
      if (w == 0 && lane == 0)
        got = i == 0 || (mbar_wait(smem_u32(sm.list_taken), (i - 1) & 1, p.status, abort_flag) &&
                         mbar_wait(smem_u32(sm.list_free), (i - 1) & 1, p.status, abort_flag));
      if (named_any(1, kProducerThreads, !got)) {
        ok = false;
        break;
      }
      // the dedupe bitmap: the list buffer (free once the previous row's gathers are issued) when
      // it fits, else the stage of this row's first chunk (free once its P.V is done)
      uint32_t* stage_bitmap = reinterpret_cast<uint32_t*>(gb + (sm.kv + s0 * kStageBytes - base));
      auto wait_stage = [&]() {
        bool g2 = true;
        if (w == 0 && lane == 0)
          g2 = mbar_wait(smem_u32(&sm.kv_empty[s0]), (uint32_t)(((gc / kStages) & 1) ^ 1), p.status, abort_flag);
        return !named_any(1, kProducerThreads, !g2);
      };
      if (!p.list_bitmap && !wait_stage()) {
        ok = false;
        break;
      }
      const bool dup = mark_keys(p, irow, rk, p.list_bitmap ? reinterpret_cast<uint32_t*>(sm.list) : stage_bitmap);
      int n;
      if (!dup) {
        n = compact_unique<kWide>(p, sm, irow, rk);
      } else {
        if (p.list_bitmap && !wait_stage()) {
          ok = false;
          break;
        }
        n = compact_first<kWide>(p, sm, irow, stage_bitmap);
      }
      fence_proxy_async_smem();                          // bitmap writes ordered before gathers into the stage
      named_sync(1, kProducerThreads);
      if (w == 0 && lane == 0) {
        sm.n_list[i & 1] = n;
        if (i < 100) TRACE(8, 402 + i);
        mbar_arrive(smem_u32(sm.list_ready));
      }
      const int nch = (n + kChunk - 1) / kChunk;
      const int rowbase = (int)(row / p.T) * p.S;        // latent row of key 0 of this query's sequence
      if (i + 1 < my_rows) load_row(p, p.idx + row_of(i + 1) * p.width, rk);  // the next row's entries
      for (int j = 0; j < nch; ++j, ++gc) {
        const int s = (int)(gc % kStages);
        if (!(ok = mbar_wait(smem_u32(&sm.kv_empty[s]), (uint32_t)(((gc / kStages) & 1) ^ 1), p.status, abort_flag)))
          break;
        if (w == 0 && lane == 0) {
          TRACE(0, gc);
          mbar_arrive_expect_tx(smem_u32(&sm.kv_full[s]), 3 * kBlockBytes);
        }
        const uint32_t stb = sm.kv + s * kStageBytes;
        const uint32_t bar = smem_u32(&sm.kv_full[s]);
        // TMA tile::gather4: four selected rows per instruction, written in the swizzled operand
        // layout.  Rows past the list repeat the list's first key (their scores are masked, P = 0).
        // Gather o = 12w + lane (lane < 12) brings the 64 columns of value block o / 16 of keys
        // 4g..4g+3, g = o % 16 (a gather costs its warp about 60 ns to issue, so the 48 gathers of
        // a chunk are spread over the four warps; block 3 and the rope columns are the copy warps').
        if (lane < 12) {
          const int o = 12 * w + lane, b = o >> 4, g = o & 15;
          int rr[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int li = j * kChunk + 4 * g + k;
            rr[k] = rowbase + get_key<kWide>(p, sm, li < n ? li : 0);
          }
          tma_gather4(stb + b * kBlockBytes + g * 512, &map_kv, bar, (4 * (int)rank + b) * 64, rr[0], rr[1], rr[2],
                      rr[3]);
        }
        if (w == 0 && lane == 0) TRACE(11, gc);
      }
      // the list buffer is rewritten for the next row only after these gathers were issued;
      // a failed wait in any producer warp ends the loop for all four
      if (named_any(1, kProducerThreads, !ok)) break;
    }
  } else if (warp == 4) {
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      const uint32_t id_qk = idesc_bf16(128, kChunk);
      const uint32_t id_pv = idesc_bf16(128, 256, false, true);
      // q.k position: row index qi (in this cluster's sequence), chunk qj of qn; pv likewise.
      // Rows without keys are skipped; ring[] keeps the chunk counts of the last non-empty rows.
      int qi = 0, qj = 0, qn = -1, q_ne = 0;
      int pj = 0, p_ne = 0;
      int ring[4] = {0, 0, 0, 0};
      long long gq = 0, gp = 0;
      bool ok = true;
      unsigned long long t_last = globaltimer();
      uint32_t spins = 0;
#ifdef DSA_TRACE
      bool trace_q = false, trace_kv = false;
#endif
      while (ok) {
        bool progressed = false;
        if (qn < 0 && qi < my_rows && mbar_test_wait(smem_u32(sm.list_ready), qi & 1)) {
          const int n = sm.n_list[qi & 1];
          mbar_arrive(smem_u32(sm.list_taken));
          qn = (n + kChunk - 1) / kChunk;
          qj = 0;
          if (qn == 0) {
            ++qi;
            qn = -1;
          } else {
            ring[q_ne & 3] = qn;
            ++q_ne;
          }
          progressed = true;
        }
#ifdef DSA_TRACE
        if (qn > 0 && qj == 0) {
          if (mbar_test_wait(smem_u32(sm.qfull), qi & 1) && !trace_q) {
            TRACE(12, gq);
            trace_q = true;
          }
          if (mbar_test_wait(smem_u32(&sm.kv_full[gq % kStages]), (uint32_t)((gq / kStages) & 1)) && !trace_kv) {
            TRACE(13, gq);
            trace_kv = true;
          }
        }
#endif
        // q.k of chunk gq: at a row start its query is loaded; its stage is loaded; the scores of
        // chunk gq-2 (same score buffer) have been read
        if (qn > 0 &&
            (qj > 0 || (mbar_test_wait(smem_u32(sm.qfull), qi & 1) &&
                        (!rope || mbar_test_wait(smem_u32(sm.qrope_full), qi & 1)))) &&
            mbar_test_wait(smem_u32(&sm.kv_full[gq % kStages]), (uint32_t)((gq / kStages) & 1)) &&
            mbar_test_wait(smem_u32(&sm.s_read[gq & 1]), (uint32_t)(((gq >> 1) & 1) ^ 1))) {
          tc_fence_after();
          const uint32_t st = sm.kv + (gq % kStages) * kStageBytes;
          const uint32_t d = tmem + (gq & 1) * kChunk;
          for (int lb = 0; lb < 4; ++lb) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_bf16_ts(d, tmem + kQCol + (lb * 4 + k) * 8, desc_sw128(st + lb * kBlockBytes + k * 32), id_qk,
                          (lb | k) ? 1u : 0u);
          }
          if (rope) {
#pragma unroll
            for (int k = 0; k < 2; ++k)
              mma_bf16_ss(d, desc_sw64(sm.qrope + k * 32), desc_sw64(st + kRopeOff + k * 32), id_qk, 1u);
          }
          mma_commit(smem_u32(&sm.s_full[gq & 1]));
          TRACE(1, gq);
#ifdef DSA_TRACE
          trace_q = trace_kv = false;
#endif
          ++gq;
          if (++qj == qn) {
            ++qi;
            qn = -1;
          }
          progressed = true;
        }
        // P.V of chunk gp: its P is in the exchange tile; at a row start the previous row's O has been read
        if (gp < gq && (pj > 0 || p_ne == 0 || mbar_test_wait(smem_u32(sm.o_free), (p_ne - 1) & 1)) &&
            mbar_test_wait(smem_u32(&sm.p_full[gp & 1]), (uint32_t)((gp >> 1) & 1))) {
          tc_fence_after();
          const uint32_t st = sm.kv + (gp % kStages) * kStageBytes;
          const uint32_t pt = sm.x + (uint32_t)(gp & 1) * kXBytes;   // P: 128 head rows x 64 keys, 128 B each
#pragma unroll
          for (int k = 0; k < kChunk / 16; ++k) {
            const uint64_t bd = desc_sw128(st + k * 2048, 1024, kBlockBytes);
            mma_bf16_ss(tmem + kOCol, desc_sw128(pt + k * 32), bd, id_pv, (pj | k) ? 1u : 0u);
          }
          mma_commit(smem_u32(&sm.kv_empty[gp % kStages]));
          mma_commit(smem_u32(&sm.o_done[gp & 1]));
          TRACE(2, gp);
          ++gp;
          if (++pj == ring[p_ne & 3]) {
            pj = 0;
            ++p_ne;
          }
          progressed = true;
        }
        if (qi >= my_rows && gp == gq) break;    // every row's lists read, every chunk's P.V issued
        if (progressed) {
          spins = 0;
          continue;
        }
        __nanosleep(32);  // keep the shared-memory pipe free for the other warps while polling
        if ((++spins & 255u) == 0u) {
          const unsigned long long now = globaltimer();
          if (*abort_flag) break;
          if (spins == 256u) t_last = now;
          else if (now - t_last > kWaitLimitNs) {
            record_status(p.status, DSA_ERR_TIMEOUT);
            *abort_flag = 1;
            break;
          }
        }
      }
      mma_commit(smem_u32(sm.drain));
      mbar_wait(smem_u32(sm.drain), 0, nullptr, nullptr);
    }
  } else if (warp >= 9 && warp <= 12) {
    // ---------------------------------------------------------------- score exchange
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
    const uint32_t dst0 = map_peer(sm.x + (uint32_t)(q4 * 4096 + lane * 16), peer);  // head r's 16 bytes of each key/4 row
    const bool real = r < p.H;
    const bool act = !kHalfHeads || q4 < 2;        // warp-uniform: this warp's head rows exist
    // Query of row i into TMEM: the CTA's 256 value-side columns of head r as bf16 pairs in
    // lane r, columns kQCol..kQCol+127, plus the rope columns by TMA.  Called only when every
    // q.k of earlier rows is complete (these warps have read all their scores).
    auto load_q = [&](int i) {
      const size_t qrow = row_of(i);
      if (warp == 9 && lane == 0 && i < 200) TRACE(8, 2 + 2 * i);
      if (warp == 9 && lane == 0 && rope) {
        mbar_arrive_expect_tx(smem_u32(sm.qrope_full), kQRopeBytes);
        tma_load_2d(sm.qrope, &map_q, smem_u32(sm.qrope_full), rope_col, (int)(qrow * p.H));
      }
      const uint4* qsrc = reinterpret_cast<const uint4*>(p.q + (qrow * p.H + (real ? r : 0)) * p.kd + rank * 256);
      // two batches of sixteen 16-byte loads (64 columns each): the rows' lines are in L2 (prefetched
      // during the previous row), so each batch costs one L2 round trip
#pragma unroll 1
      for (int c0 = 0; act && c0 < 128; c0 += 64) {      // 64 columns = 128 bf16 = 16 x 16 bytes
        uint32_t qv[64];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const uint4 u = real ? qsrc[c0 / 4 + k] : make_uint4(0, 0, 0, 0);
          qv[4 * k] = u.x;
          qv[4 * k + 1] = u.y;
          qv[4 * k + 2] = u.z;
          qv[4 * k + 3] = u.w;
        }
        tmem_st_32x32b_x32(tmem + lane_addr + kQCol + c0, *reinterpret_cast<const uint32_t(*)[32]>(&qv[0]));
        tmem_st_32x32b_x32(tmem + lane_addr + kQCol + c0 + 32, *reinterpret_cast<const uint32_t(*)[32]>(&qv[32]));
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (warp == 9 && lane == 0 && i < 200) TRACE(8, 3 + 2 * i);
      if (lane == 0) mbar_arrive(smem_u32(sm.qfull));
      // the following row's query lines are pulled into L2 meanwhile
      if (i + 1 < my_rows && real) {
        const bf16* nq = p.q + (row_of(i + 1) * p.H + r) * p.kd + rank * 256;
#pragma unroll
        for (int k = 0; k < 4; ++k) asm volatile("prefetch.global.L2 [%0];" ::"l"(nq + 64 * k) : "memory");
      }
    };
    if (my_rows > 0) load_q(0);
    long long gc = 0, pend = -1;   // pend: the chunk whose exchange tile still has to go back to the peer
    bool ok = true;
    // Exchange tile c & 1 goes back to the peer in two halves: half 1 (keys 32-63) once our group-1
    // softmax warps have read it, half 0 (keys 0-31, overwritten by P) once P.V of chunk c has read P.
    auto give_back = [&](long long c) {
      const uint32_t ph = (uint32_t)((c >> 1) & 1);
      if (!mbar_wait(smem_u32(&sm.xread1[c & 1]), ph, p.status, abort_flag)) return false;
      __syncwarp();
      if (lane == 0) arrive_remote_relaxed(map_peer(smem_u32(&sm.xfree[2 * (c & 1) + 1]), peer));
      if (!mbar_wait(smem_u32(&sm.o_done[c & 1]), ph, p.status, abort_flag)) return false;
      if (q4 == 1 && lane == 0) TRACE(14, c);
      __syncwarp();
      if (lane == 0) arrive_remote_relaxed(map_peer(smem_u32(&sm.xfree[2 * (c & 1)]), peer));
      return true;
    };
    for (int i = 0; ok && i < my_rows; ++i) {
      if (!(ok = mbar_wait(smem_u32(sm.list_ready), i & 1, p.status, abort_flag))) break;
      const int n = sm.n_list[i & 1];
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(sm.list_taken));
      const int nch = (n + kChunk - 1) / kChunk;
      if (nch == 0 && i + 1 < my_rows) load_q(i + 1);
      for (int j = 0; j < nch; ++j, ++gc) {
        const int sb = (int)(gc & 1);
        const uint32_t use = (uint32_t)((gc >> 1) & 1);
        if (!(ok = mbar_wait(smem_u32(&sm.s_full[sb]), use, p.status, abort_flag))) break;
        if (act) {
          tc_fence_after();
          uint32_t v[kChunk];
          tmem_ld_32x32b_x32(tmem + lane_addr + sb * kChunk, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
          tmem_ld_32x32b_x32(tmem + lane_addr + sb * kChunk + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&sm.s_read[sb]));
          if (q4 == 1 && lane == 0) TRACE(3, gc);
          // each store writes 4 keys of head r, the warp 512 contiguous
          // bytes; each store completes its bytes on the peer's barrier of that half (no round trip
          // here).  Half 1 first: the peer returns it as soon as its softmax has read it, half 0
          // only after its P.V (P overwrites half 0).
          const uint32_t dst = dst0 + (uint32_t)sb * kXBytes;
          if (!(ok = wait_cluster(smem_u32(&sm.xfree[2 * sb + 1]), use ^ 1u, p.status, abort_flag))) break;
          const uint32_t xbar1 = map_peer(smem_u32(&sm.xfull[2 * sb + 1]), peer);
#pragma unroll
          for (int c = 32; c < kChunk; c += 4) st_async_v4(dst + 16384 + (c - 32) * 128, &v[c], xbar1);
          if (!(ok = wait_cluster(smem_u32(&sm.xfree[2 * sb]), use ^ 1u, p.status, abort_flag))) break;
          const uint32_t xbar0 = map_peer(smem_u32(&sm.xfull[2 * sb]), peer);
#pragma unroll
          for (int c = 0; c < 32; c += 4) st_async_v4(dst + c * 128, &v[c], xbar0);
        } else {
          // head rows >= H: nothing to read or send
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&sm.s_read[sb]));
        }
        if (q4 == 1 && lane == 0) TRACE(4, gc);
        if (j + 1 == nch) break;                     // the row's last chunk continues below
        // the previous chunk's tile goes back after this chunk's push, which therefore never waits for a P.V
        if (pend >= 0 && !(ok = give_back(pend))) break;
        pend = gc;
      }
      if (ok && nch > 0) {
        // the row's last q.k is complete (its scores were just read): load the next row's query first
        if (i + 1 < my_rows) load_q(i + 1);
        if (pend >= 0 && !(ok = give_back(pend))) break;
        pend = gc;
        ++gc;
      }
    }
    if (ok && pend >= 0) give_back(pend);
  } else if (warp >= 17) {
    // ---------------------------------------------------------------- more TMA gathers
    // Gather o = 11 (warp - 17) + lane of the 16 of value block 3 (o < 16: keys 4o..4o+3, latent
    // columns (4 rank + 3) * 64 ..) and, when kd = 576, the 16 of the CTA's 32 rope columns (o - 16:
    // keys 4(o-16).., 64-byte swizzled rope block).  Each warp arms the stage's barrier with its
    // own bytes.
    const int cw = warp - 17;
    const int nops = rope ? 32 : 16;
    const int o = 11 * cw + lane;
    const bool mine = lane < 11 && o < nops;
    uint32_t bytes = 0;                               // this warp's bytes per chunk
    for (int k = 11 * cw; k < 11 * cw + 11 && k < nops; ++k) bytes += k < 16 ? 512u : 256u;
    if (lane == 0) {
      tma_prefetch_desc(&map_kv);
      if (rope) tma_prefetch_desc(&map_rope);
    }
    long long gc = 0;
    bool ok = true;
    for (int i = 0; ok && i < my_rows; ++i) {
      const size_t row = row_of(i);
      if (!(ok = mbar_wait(smem_u32(sm.list_ready), i & 1, p.status, abort_flag))) break;
      const int n = sm.n_list[i & 1];
      const int nch = (n + kChunk - 1) / kChunk;
      const int rowbase = (int)(row / p.T) * p.S;
      for (int j = 0; j < nch; ++j, ++gc) {
        const int s = (int)(gc % kStages);
        if (!(ok = mbar_wait(smem_u32(&sm.kv_empty[s]), (uint32_t)(((gc / kStages) & 1) ^ 1), p.status, abort_flag)))
          break;
        const uint32_t stb = sm.kv + s * kStageBytes;
        const uint32_t bar = smem_u32(&sm.kv_full[s]);
        if (lane == 0) mbar_arrive_expect_tx(bar, bytes);
        if (mine) {
          const int g = o & 15;
          int rr[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int li = j * kChunk + 4 * g + k;
            rr[k] = rowbase + get_key<kWide>(p, sm, li < n ? li : 0);
          }
          if (o < 16)
            tma_gather4(stb + 3 * kBlockBytes + g * 512, &map_kv, bar, (4 * (int)rank + 3) * 64, rr[0], rr[1], rr[2],
                        rr[3]);
          else
            tma_gather4(stb + kRopeOff + g * 256, &map_rope, bar, rope_col, rr[0], rr[1], rr[2], rr[3]);
        }
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(sm.list_free));   // this row's list may be rewritten
    }
  } else if (warp < 4 || warp >= 13) {
    // ---------------------------------------------------------------- softmax + epilogue
    // Group g (warps 0-3 or 13-16) takes keys 32g..32g+31 of every chunk and O columns 128g..128g+127.
    const int g = warp < 4 ? 0 : 1;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;                   // head row == TMEM lane
    const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
    const bool lead = g == 0 && q4 == 0 && lane == 0;
    const bool real = r < p.H;
    const bool act = !kHalfHeads || q4 < 2;         // warp-uniform: this warp's head rows exist
    // head r's 4-key groups in the exchange tile: quarter q4, lane
    const float4* xcol = reinterpret_cast<const float4*>(gb + (sm.x - base)) + q4 * 256 + lane;
    long long gc = 0;
    bool ok = true;
    // the epilogue of a row runs after the next row's query load, so it overlaps that row's first q.k
    bool pending = false;
    size_t p_row = 0;
    long long p_last = 0;
    float p_mref = 0.f, p_lsum = 0.f;
    int n_epi = 0;
    auto epilogue = [&]() {
      bf16* orow = p.out + (p_row * p.H + r) * 512 + rank * 256 + 128 * g;
      sm.lsum[g * 128 + r] = p_lsum;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(sm.lready));
      ok = mbar_wait(smem_u32(sm.lready), n_epi & 1, p.status, abort_flag) &&
           mbar_wait(smem_u32(&sm.o_done[p_last & 1]), (uint32_t)((p_last >> 1) & 1), p.status, abort_flag);
      const float l_all = p_lsum + sm.lsum[(1 - g) * 128 + r];
      tc_fence_after();
      const float inv = 1.f / l_all;
      for (int c = 0; act && c < 128; c += 32) {
        uint32_t o[32];
        tmem_ld_32x32b_x32(tmem + lane_addr + kOCol + 128 * g + c, o);
        tmem_ld_wait();
        if (real && ok) {
          uint32_t pk[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) pk[k] = pack_bf16(__uint_as_float(o[2 * k]) * inv, __uint_as_float(o[2 * k + 1]) * inv);
          if (p.out_v8) {
            // 32 contiguous bytes (one full sector) per store
            st_global_v8(orow + c, pk);
            st_global_v8(orow + c + 16, pk + 8);
          } else {
#pragma unroll
            for (int k = 0; k < 4; ++k)
              *reinterpret_cast<uint4*>(orow + c + 8 * k) = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
          }
        }
      }
      if (real && ok && rank == 0 && g == 0 && p.lse)
        p.lse[p_row * p.H + r] = (p_mref + log2f(l_all)) * 0.69314718055994531f;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(sm.o_free));  // P.V of the next row may overwrite O
      ++n_epi;
      pending = false;
    };
    for (int i = 0; ok && i < my_rows; ++i) {
      const size_t row = row_of(i);
      if (pending) {
        epilogue();
        if (!ok) break;
      }
      if (!(ok = mbar_wait(smem_u32(sm.list_ready), i & 1, p.status, abort_flag))) break;
      const int n = sm.n_list[i & 1];
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(sm.list_taken));
      const int nch = (n + kChunk - 1) / kChunk;
      if (nch == 0) {
        // no key selected: out = 0, lse = -inf
        if (real) {
          bf16* orow = p.out + (row * p.H + r) * 512 + rank * 256 + 128 * g;
          for (int c = 0; c < 128; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
          if (rank == 0 && g == 0 && p.lse) p.lse[row * p.H + r] = -INFINITY;
        }
        continue;
      }
      if (!act) {
        // head rows >= H (H = 64): no per-chunk work and no per-chunk barrier (nothing would keep
        // these warps from running chunks ahead); only the row's epilogue barriers count them
        gc += nch;
        pending = true;
        p_row = row;
        p_last = gc - 1;
        p_mref = 0.f;
        p_lsum = 0.f;
        continue;
      }
      float m_ref = -INFINITY, l_sum = 0.f;
      for (int j = 0; ok && j < nch; ++j, ++gc) {
        const int sb = (int)(gc & 1);
        const uint32_t use = (uint32_t)((gc >> 1) & 1);
        if (!(ok = mbar_wait(smem_u32(&sm.s_full[sb]), use, p.status, abort_flag))) break;
        tc_fence_after();
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + lane_addr + sb * kChunk + 32 * g, v);
        tmem_ld_wait();
        // the score buffer may be refilled by the q.k two chunks ahead
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.s_read[sb]));
        if (lead) TRACE(5, gc);
        // our half g of exchange tile sb (keys 32g..32g+31 of the peer's partial scores)
        if (!(ok = wait_cluster(smem_u32(&sm.xfull[2 * sb + g]), use, p.status, abort_flag))) break;
        if (q4 == 0 && lane == 0) {
          if (g == 0) TRACE(6, gc);
          mbar_arrive_expect_tx(smem_u32(&sm.xfull[2 * sb + g]), 32u * p.H * 4u);  // arm the next use (H rows)
        }
        const float4* xr = xcol + sb * (kXBytes / 16) + g * 1024;
        const int valid = n - j * kChunk - 32 * g;
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const float4 x4 = xr[(c / 4) * 32];
          const float xs[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float x = c + k < valid ? (__uint_as_float(v[c + k]) + xs[k]) * p.scale_log2 : -INFINITY;
            v[c + k] = __float_as_uint(x);
            mx = fmaxf(mx, x);
          }
        }
        if (g == 1) {
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&sm.xread1[sb]));   // half 1 may go back to the peer
        }
        // row maximum over both halves of the chunk, agreed by the two warps of this head quarter;
        // once both pass this barrier the quarter's half-0 scores have been read, and its P rows,
        // which occupy exactly those bytes, may be written
        float* mxb = sm.mx + sb * 256;
        mxb[g * 128 + r] = mx;
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.mxready[4 * sb + q4]));
        if (!(ok = mbar_wait(smem_u32(&sm.mxready[4 * sb + q4]), use, p.status, abort_flag))) break;
        mx = fmaxf(mx, mxb[(1 - g) * 128 + r]);
        if (lead) TRACE(9, gc);
        // move the reference maximum only when it grows by more than 2^8 (both groups agree)
        const bool grow = mx > m_ref + 8.f;
        const float new_ref = grow ? mx : m_ref;
        if (__any_sync(0xffffffffu, grow && j > 0)) {
          const long long pg = gc - 1;
          if (!(ok = mbar_wait(smem_u32(&sm.o_done[pg & 1]), (uint32_t)((pg >> 1) & 1), p.status, abort_flag))) break;
          tc_fence_after();
          const float f = (grow && j > 0) ? ex2(m_ref - new_ref) : 1.f;
          for (int c = 128 * g; c < 128 * g + 128; c += 16) {
            uint32_t o[16];
            tmem_ld_32x32b_x16(tmem + lane_addr + kOCol + c, o);
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * f);
            tmem_st_32x32b_x16(tmem + lane_addr + kOCol + c, o);
          }
          tmem_st_wait();
          l_sum *= f;
        }
        m_ref = new_ref;
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float p0 = ex2(__uint_as_float(v[c]) - m_ref);
          const float p1 = ex2(__uint_as_float(v[c + 1]) - m_ref);
          l_sum += p0 + p1;
          pk[c / 2] = pack_bf16(p0, p1);
        }
        if (lead) TRACE(10, gc);
        // P of keys 32g..32g+31: 16-byte chunks 4g..4g+3 of row r of the 128-byte-swizzled K-major
        // tile at the start of exchange tile sb (chunk c of row r sits at position c ^ (r & 7))
        {
          const uint32_t prow = sm.x + (uint32_t)sb * kXBytes + (uint32_t)r * 128u;
#pragma unroll
          for (int k = 0; k < 4; ++k) st_shared_v4(prow + ((uint32_t)((4 * g + k) ^ (r & 7)) << 4), &pk[4 * k]);
        }
        if (lead) TRACE(15, gc);
        fence_proxy_async_smem();                   // visible to the tensor core's operand reads
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.p_full[sb]));
        if (lead) TRACE(7, gc);
      }
      pending = true;
      p_row = row;
      p_last = gc - 1;
      p_mref = m_ref;
      p_lsum = l_sum;
    }
    if (ok && pending) epilogue();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no remote access to a CTA that has exited
#ifdef DSA_TRACE
  if (threadIdx.x == 0 && blockIdx.x < 1024) g_attend_span[blockIdx.x][1] = sm100::globaltimer();
#endif
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
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

size_t smem_bytes(int width, int S, bool with_bitmap) {
  return 1024 + 2 * (size_t)kXBytes + kQRopeBytes + (size_t)kStages * kStageBytes + list_bytes(width, S, with_bitmap) +
         2 * 2 * 128 * 4 + 2 * 128 * 4 + 8 * 48 + 16;
}

bool bitmap_in_list(int width, int S) { return smem_bytes(width, S, true) <= 227 * 1024; }

}  // namespace

bool attend_tc_supported(const dsa_dims& d, int64_t k_stride, const void* k, const void* v, int64_t v_stride,
                         int width) {
  if (d.dtype != DSA_BF16 || d.kv_heads != 1 || d.vd != 512) return false;
  if (!(d.kd == 512 || d.kd == 576)) return false;
  if (!(d.heads == 64 || d.heads == 128)) return false;
  if ((long long)d.batch * d.n_q * d.heads < 128) return false;  // the query TMA box is 128 rows
  if (k != v || k_stride != v_stride || k_stride < d.kd || (k_stride * 2) % 16 != 0) return false;
  if (((uintptr_t)k & 15u) != 0) return false;
  if (d.n_kv > kMaxKeys) return false;                     // the dedupe bitmap fits one gather stage
  if ((long long)d.batch * d.n_kv > 2147483647LL) return false;  // 32-bit TMA row coordinates
  if (width > 8192) return false;
  if (smem_bytes(width, d.n_kv, false) > 227 * 1024) return false;
  return encode_fn() != nullptr;
}

cudaError_t launch_attend_tc(const dsa_dims& d, const void* q, const void* k, int64_t k_stride,
                             const int32_t* idx, int width, float scale, void* out, float* lse,
                             cudaStream_t st) {
  AttTcParams p{};
  p.B = d.batch;
  p.T = d.n_q;
  p.S = d.n_kv;
  p.H = d.heads;
  p.kd = d.kd;
  p.width = width;
  p.stride = k_stride;
  p.latent = (const bf16*)k;
  p.q = (const bf16*)q;
  p.idx = idx;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.out = (bf16*)out;
  p.lse = lse;
  p.status = device_status_ptr();
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  // q viewed as [B*T*H rows, kd cols]; box = 32 cols x 128 rows, 64-byte swizzle (a CTA's rope columns)
  CUtensorMap mq;
  cuuint64_t qdims[2] = {(cuuint64_t)d.kd, (cuuint64_t)d.batch * d.n_q * d.heads};
  cuuint64_t qstrides[1] = {(cuuint64_t)d.kd * 2};
  cuuint32_t qbox[2] = {32u, 128u};
  cuuint32_t qestr[2] = {1u, 1u};
  if (enc(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(q), qdims, qstrides, qbox, qestr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  // latent viewed as [B*S rows, kd cols] with the caller's row stride; box = 64 cols x 1 row (gather4)
  CUtensorMap mkv, mrope;
  cuuint64_t kdims[2] = {(cuuint64_t)d.kd, (cuuint64_t)d.batch * d.n_kv};
  cuuint64_t kstrides[1] = {(cuuint64_t)k_stride * 2};
  cuuint32_t kbox[2] = {64u, 1u};
  cuuint32_t estr[2] = {1u, 1u};
  if (enc(&mkv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(k), kdims, kstrides, kbox, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  // the same rows, 32 rope columns per box with the 64-byte swizzle of the rope operand
  cuuint32_t rbox[2] = {32u, 1u};
  if (enc(&mrope, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(k), kdims, kstrides, rbox, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  p.list_bitmap = bitmap_in_list(width, d.n_kv) ? 1 : 0;
  p.list_nbytes = (int)list_bytes(width, d.n_kv, p.list_bitmap != 0);
  p.list_hi_off = (int)list_lo_bytes(width);
  p.out_v8 = ((uintptr_t)out & 31u) == 0 ? 1 : 0;
  const size_t smem = smem_bytes(width, d.n_kv, p.list_bitmap != 0);
  const bool wide = d.n_kv > kNarrowKeys;
  auto kern = d.heads == 64 ? (wide ? attend_tc_kernel<true, true> : attend_tc_kernel<true, false>)
                            : (wide ? attend_tc_kernel<false, true> : attend_tc_kernel<false, false>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // persistent clusters: one per SM pair (or one per row when there are fewer rows)
  const long long rows = (long long)d.batch * d.n_q;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long clusters = rows < sms / 2 ? rows : sms / 2;
  kern<<<dim3((unsigned)(2 * clusters)), kThreads, smem, st>>>(mq, mkv, mrope, p);
  return cudaGetLastError();
}

}  // namespace dsa

#ifdef DSA_TRACE
extern "C" int dsa_trace_read(unsigned long long* host) {
  return (int)cudaMemcpyFromSymbol(host, dsa::g_attend_trace, sizeof(dsa::g_attend_trace));
}
extern "C" int dsa_trace_span(unsigned long long* host) {
  return (int)cudaMemcpyFromSymbol(host, dsa::g_attend_span, sizeof(dsa::g_attend_span));
}
extern "C" int dsa_trace_clear() {
  static unsigned long long zero[2 * 16 * 512];
  return (int)cudaMemcpyToSymbol(dsa::g_attend_trace, zero, sizeof(zero));
}
#endif
