// Indexer query / key preparation ahead of the score (ik_llama.cpp PR #2063 with
// the PR #2045 commit messages: "What it does" (split rope/nope, NEOX RoPE of the
// rope part, concat; LayerNorm with bias on the key), the decode-cache commit
// (Walsh-Hadamard rotation of q and k, keys written into the indexer cache at
// their slot) and the K-shift commit (the cached key is H * concat(RoPE(k_pe,
// pos), k_nope); NEOX RoPE without scaling)).
//
// One block per row (token).  Each warp takes head vectors of `dim` values, up
// to four at a time so their loads are in flight together: lane l holds values
// l*E .. l*E+E-1 (E = dim/32) in registers, read with one vector load.  While
// the first loads are in flight, the block builds the row's RoPE table: the
// angle pos * f_i (f_i = theta^(-2i/n_rope), computed once on the host in
// double) is reduced modulo 2*pi in double, so the fp32 sine and cosine see an
// argument in [-pi, pi] whatever the position.
//   LayerNorm: a warp sum for the mean, then one for the biased variance of the
//     centred values.
//   NEOX RoPE: value d < n_rope/2 pairs with d + n_rope/2, which lives
//     n_rope/(2E) lanes higher; one shuffle down and one up give both partners.
//   Walsh-Hadamard: log2(E) butterfly stages inside the lane, five over the lane
//     bits with xor shuffles, then the 1/sqrt(dim) scale; the butterflies give
//     y[i] = sum_j (-1)^popcount(i & j) x[j], the Sylvester matrix.
// The row goes to out_rows[r] (its cache slot) or to r; a slot outside
// [0, capacity) is skipped.  Each vector is read once and written once, so the
// kernel is bound by HBM bandwidth.
//
// dim = 128 with n_rope in {0, 64, 128} (the indexer's shape), 16-byte aligned
// rows, takes a second kernel, index_rotate128_kernel, that spends fewer shuffles per vector: four
// lanes share a vector, lane t of the four holding values 32t .. 32t+31, so
// five of the seven Walsh-Hadamard stages run inside the lane and two cross
// lanes (xor 1 and 2), the RoPE partner of a value sits in lane t^1 (n_rope 64)
// or t^2 (n_rope 128) at the same register, and a LayerNorm sum takes two
// shuffles.  A block of 128 threads takes 32 consecutive head vectors of one row
// (rows of 32, 64, ... heads: the query step); the RoPE table holds that row.
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {

namespace {

constexpr int kRotWarps = 8;  // warps per block (fewer when a row has fewer heads)
constexpr int kRotBatch = 4;  // head vectors per warp in flight

constexpr double kTwoPi = 6.283185307179586;      // 2*pi rounded to double
constexpr double kInvTwoPi = 0.15915494309189535;  // 1/(2*pi) rounded to double

struct RotParams {
  double inv_freq[64];  // theta^(-2i/n_rope), i < n_rope/2
  const void* in;
  void* out;
  const int32_t* pos;
  const int32_t* out_rows;
  const float* ln_w;
  const float* ln_b;
  int64_t in_stride, out_stride, out_cap;
  int heads, n_rope, layer_norm, hadamard;
  float eps, hscale;
};

template <int E>
__device__ __forceinline__ void load_vals(const float* p, float (&v)[E]) {
  if constexpr (E == 4) {
    const float4 u = *reinterpret_cast<const float4*>(p);
    v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
  } else if constexpr (E == 2) {
    const float2 u = *reinterpret_cast<const float2*>(p);
    v[0] = u.x; v[1] = u.y;
  } else {
    v[0] = *p;
  }
}

template <int E>
__device__ __forceinline__ void load_vals(const bf16* p, float (&v)[E]) {
  if constexpr (E == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
  } else if constexpr (E == 2) {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
    v[0] = a.x; v[1] = a.y;
  } else {
    v[0] = __bfloat162float(*p);
  }
}

template <int E>
__device__ __forceinline__ void store_vals(float* p, const float (&v)[E]) {
  if constexpr (E == 4) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  } else if constexpr (E == 2) {
    *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
  } else {
    *p = v[0];
  }
}

template <int E>
__device__ __forceinline__ void store_vals(bf16* p, const float (&v)[E]) {
  if constexpr (E == 4) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
    __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&a);
    u.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = u;
  } else if constexpr (E == 2) {
    *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(v[0], v[1]);
  } else {
    *p = __float2bfloat16_rn(v[0]);
  }
}

template <typename Tin, typename Tout, int E>
__global__ void __launch_bounds__(kRotWarps * 32)
index_rotate_kernel(const __grid_constant__ RotParams p) {
  constexpr int D = 32 * E;
  __shared__ float2 tab[D / 2];  // (cos, sin) of each RoPE pair
  const int r = blockIdx.x;
  const int half = p.n_rope >> 1;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int d0 = lane * E;
  // no __restrict__: an exactly in-place call reads and writes the same vectors
  const Tin* src = static_cast<const Tin*>(p.in) + (int64_t)r * p.in_stride + d0;

  // first batch of head vectors: loads in flight while the table is built
  float v[kRotBatch][E];
#pragma unroll
  for (int u = 0; u < kRotBatch; ++u) {
    const int h = warp + u * nwarps;
    if (h < p.heads) load_vals<E>(src + (int64_t)h * D, v[u]);
  }
  if (half > 0) {
    const double pos = (double)p.pos[r];
    for (int i = threadIdx.x; i < half; i += blockDim.x) {
      const double a = pos * p.inv_freq[i];
      const double red = fma(-rint(a * kInvTwoPi), kTwoPi, a);  // a - 2*pi*k, |red| <= pi
      float s, c;
      sincosf((float)red, &s, &c);
      tab[i] = make_float2(c, s);
    }
  }
  __syncthreads();

  const int64_t dst = p.out_rows ? (int64_t)p.out_rows[r] : (int64_t)r;
  if (dst < 0 || dst >= p.out_cap) return;  // block-uniform; no barrier follows
  Tout* dstp = static_cast<Tout*>(p.out) + dst * p.out_stride + d0;

  float lw[E], lb[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    lw[e] = p.layer_norm && p.ln_w ? p.ln_w[d0 + e] : 1.f;
    lb[e] = p.layer_norm && p.ln_b ? p.ln_b[d0 + e] : 0.f;
  }
  const int off = half / E;  // lane distance between the two values of a RoPE pair
  const bool first_half = d0 < half, second_half = d0 >= half && d0 < p.n_rope;

  for (int h0 = warp; h0 < p.heads; h0 += nwarps * kRotBatch) {
    if (h0 != warp) {
#pragma unroll
      for (int u = 0; u < kRotBatch; ++u) {
        const int h = h0 + u * nwarps;
        if (h < p.heads) load_vals<E>(src + (int64_t)h * D, v[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < kRotBatch; ++u) {
      const int h = h0 + u * nwarps;
      if (h >= p.heads) break;  // warp-uniform
      if (p.layer_norm) {
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) s += v[u][e];
        const float mean = warp_sum(s) * (1.f / D);
        float s2 = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          v[u][e] -= mean;
          s2 = fmaf(v[u][e], v[u][e], s2);
        }
        const float inv_std = 1.f / sqrtf(warp_sum(s2) * (1.f / D) + p.eps);
#pragma unroll
        for (int e = 0; e < E; ++e) v[u][e] = fmaf(v[u][e] * inv_std, lw[e], lb[e]);
      }
      if (half > 0) {
        float up[E], dn[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
          up[e] = __shfl_down_sync(0xffffffffu, v[u][e], off);
          dn[e] = __shfl_up_sync(0xffffffffu, v[u][e], off);
        }
        if (first_half) {
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const float2 cs = tab[d0 + e];
            v[u][e] = v[u][e] * cs.x - up[e] * cs.y;
          }
        } else if (second_half) {
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const float2 cs = tab[d0 + e - half];
            v[u][e] = v[u][e] * cs.x + dn[e] * cs.y;
          }
        }
      }
      if (p.hadamard) {
#pragma unroll
        for (int m = 1; m < E; m <<= 1) {
#pragma unroll
          for (int e = 0; e < E; ++e) {
            if (!(e & m)) {
              const float a = v[u][e], b = v[u][e | m];
              v[u][e] = a + b;
              v[u][e | m] = a - b;
            }
          }
        }
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const float o = __shfl_xor_sync(0xffffffffu, v[u][e], m);
            v[u][e] = (lane & m) ? o - v[u][e] : v[u][e] + o;
          }
        }
#pragma unroll
        for (int e = 0; e < E; ++e) v[u][e] *= p.hscale;
      }
      store_vals<E>(dstp + (int64_t)h * D, v[u]);
    }
  }
}

constexpr int k128Vectors = 32;               // head vectors per block of the dim-128 kernel
constexpr int k128Threads = 4 * k128Vectors;  // four lanes per vector

// 32 consecutive values of a lane: 16-byte loads and stores.
__device__ __forceinline__ void load32(const bf16* p, float (&x)[32]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 u = reinterpret_cast<const uint4*>(p)[i];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
      x[8 * i + 2 * j] = f.x;
      x[8 * i + 2 * j + 1] = f.y;
    }
  }
}
__device__ __forceinline__ void load32(const float* p, float (&x)[32]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 u = reinterpret_cast<const float4*>(p)[i];
    x[4 * i] = u.x;
    x[4 * i + 1] = u.y;
    x[4 * i + 2] = u.z;
    x[4 * i + 3] = u.w;
  }
}
__device__ __forceinline__ void store32(bf16* p, const float (&x)[32]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      __nv_bfloat162 b = __floats2bfloat162_rn(x[8 * i + 2 * j], x[8 * i + 2 * j + 1]);
      w[j] = *reinterpret_cast<uint32_t*>(&b);
    }
    reinterpret_cast<uint4*>(p)[i] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}
__device__ __forceinline__ void store32(float* p, const float (&x)[32]) {
#pragma unroll
  for (int i = 0; i < 8; ++i)
    reinterpret_cast<float4*>(p)[i] = make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
}

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(k128Threads, 6)
index_rotate128_kernel(const __grid_constant__ RotParams p, long long n_vec) {
  // (cos, sin) per (row of the block, angle): one row when heads is a multiple of 32, up to 32
  // rows for other head counts
  __shared__ __align__(16) float2 tab[k128Vectors][64];
  __shared__ float lnw[128], lnb[128];
  const int lane = threadIdx.x & 31;
  const int t = lane & 3;                                   // quarter of the vector this lane holds
  const long long v0 = (long long)blockIdx.x * k128Vectors;
  const long long v = v0 + (threadIdx.x >> 2);
  const bool live = v < n_vec;
  const long long r0 = v0 / p.heads;                        // first row of the block
  // lanes past the last vector take the block's first row (table index 0) and store nothing
  const long long r = live ? v / p.heads : r0;
  const int h = live ? (int)(v - r * p.heads) : 0;
  const int half = p.n_rope >> 1;

  float x[32];
  if (live) {
    load32(static_cast<const Tin*>(p.in) + r * p.in_stride + (long long)h * 128 + 32 * t, x);
  } else {
#pragma unroll
    for (int e = 0; e < 32; ++e) x[e] = 0.f;
  }
  // the RoPE table of the block's rows (loads in flight meanwhile)
  if (half > 0) {
    const long long last = min(n_vec, v0 + k128Vectors) - 1;
    const int n_rows = (int)(last / p.heads - r0) + 1;
    for (int i = threadIdx.x; i < n_rows * half; i += k128Threads) {
      const int rr = i / half, a = i - rr * half;
      const double ang = (double)p.pos[r0 + rr] * p.inv_freq[a];
      const double red = fma(-rint(ang * kInvTwoPi), kTwoPi, ang);  // |red| <= pi
      float sn, cs;
      sincosf((float)red, &sn, &cs);
      tab[rr][a] = make_float2(cs, sn);
    }
  }
  if (p.layer_norm) {
    lnw[threadIdx.x] = p.ln_w ? p.ln_w[threadIdx.x] : 1.f;
    lnb[threadIdx.x] = p.ln_b ? p.ln_b[threadIdx.x] : 0.f;
  }
  __syncthreads();

  if (p.layer_norm) {
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < 32; ++e) s += x[e];
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    const float mean = s * (1.f / 128.f);
    float s2 = 0.f;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      x[e] -= mean;
      s2 = fmaf(x[e], x[e], s2);
    }
    s2 += __shfl_xor_sync(0xffffffffu, s2, 1);
    s2 += __shfl_xor_sync(0xffffffffu, s2, 2);
    const float inv_std = 1.f / sqrtf(s2 * (1.f / 128.f) + p.eps);
#pragma unroll
    for (int e = 0; e < 32; ++e) x[e] = fmaf(x[e] * inv_std, lnw[32 * t + e], lnb[32 * t + e]);
  }
  if (half > 0) {
    // NEOX pairs (i, i + half): half = 32 pairs lanes t^1 among t < 2; half = 64 pairs t^2.
    // first half: x cos - o sin; second half: x cos + o sin (the sign goes onto sin's bits)
    const int m = half >> 5;
    const bool in_rope = 32 * t < p.n_rope;
    const uint32_t neg = (t & m) == 0 ? 0x80000000u : 0u;
    const int a0 = half == 32 ? 0 : 32 * (t & 1);            // angle index of register e is a0 + e
    const float4* tr = reinterpret_cast<const float4*>(&tab[(int)(r - r0)][a0]);
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const float4 cs = tr[e >> 1];                           // (cos, sin) of angles a0+e, a0+e+1
      const float o0 = __shfl_xor_sync(0xffffffffu, x[e], m);
      const float o1 = __shfl_xor_sync(0xffffffffu, x[e + 1], m);
      if (in_rope) {
        x[e] = fmaf(o0, __uint_as_float(__float_as_uint(cs.y) ^ neg), x[e] * cs.x);
        x[e + 1] = fmaf(o1, __uint_as_float(__float_as_uint(cs.w) ^ neg), x[e + 1] * cs.z);
      }
    }
  }
  if (p.hadamard) {
    // bits 0-4 of the value index inside the lane, bits 5-6 across the four lanes:
    // x' = x + o on the lower lane of a pair, o - x on the upper one
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        if (!(e & m)) {
          const float a = x[e], b = x[e | m];
          x[e] = a + b;
          x[e | m] = a - b;
        }
      }
    }
#pragma unroll
    for (int m = 1; m < 4; m <<= 1) {
      const float sg = (t & m) ? -1.f : 1.f;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float o = __shfl_xor_sync(0xffffffffu, x[e], m);
        x[e] = fmaf(x[e], sg, o);
      }
    }
#pragma unroll
    for (int e = 0; e < 32; ++e) x[e] *= p.hscale;
  }
  if (!live) return;
  const long long dst = p.out_rows ? (long long)p.out_rows[r] : r;
  if (dst < 0 || dst >= p.out_cap) return;
  store32(static_cast<Tout*>(p.out) + dst * p.out_stride + (long long)h * 128 + 32 * t, x);
}

template <typename Tin, typename Tout>
cudaError_t launch_rotate_t(int n_rows, int dim, const RotParams& p, cudaStream_t st) {
  // the dim-128 kernel moves 16 bytes per access: rows and bases must allow it
  const auto al16 = [](const void* q) { return ((uintptr_t)q & 15u) == 0; };
  const bool aligned = al16(p.in) && al16(p.out) && p.in_stride % (16 / (int)sizeof(Tin)) == 0 &&
                       p.out_stride % (16 / (int)sizeof(Tout)) == 0;
  // one-head rows (keys) stay on the general kernel: there a block's 32 vectors span 32 rows, and
  // building 32 rows of angles per block costs more than the shuffles it saves
  if (dim == 128 && aligned && p.heads % k128Vectors == 0 && (p.n_rope == 0 || p.n_rope == 64 || p.n_rope == 128)) {
    const long long n_vec = (long long)n_rows * p.heads;
    const long long blocks = (n_vec + k128Vectors - 1) / k128Vectors;
    if (blocks < 2147483647LL) {
      index_rotate128_kernel<Tin, Tout><<<(unsigned)blocks, k128Threads, 0, st>>>(p, n_vec);
      return cudaGetLastError();
    }
  }
  const int warps = p.heads < kRotWarps ? p.heads : kRotWarps;
  const dim3 grid((unsigned)n_rows), block((unsigned)(32 * warps));
  switch (dim) {
    case 32: index_rotate_kernel<Tin, Tout, 1><<<grid, block, 0, st>>>(p); break;
    case 64: index_rotate_kernel<Tin, Tout, 2><<<grid, block, 0, st>>>(p); break;
    case 128: index_rotate_kernel<Tin, Tout, 4><<<grid, block, 0, st>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_index_rotate(int n_rows, int heads, int dim, int n_rope, float theta, bool layer_norm,
                                const float* ln_w, const float* ln_b, float eps, bool hadamard,
                                const int32_t* pos, bool in_bf16, const void* in, int64_t in_stride,
                                bool out_bf16, void* out, int64_t out_stride, const int32_t* out_rows,
                                int64_t out_cap, cudaStream_t st) {
  if (n_rows == 0) return cudaSuccess;
  RotParams p;
  for (int i = 0; i < 64; ++i) p.inv_freq[i] = i < n_rope / 2 ? pow((double)theta, -2.0 * i / n_rope) : 0.0;
  p.in = in;
  p.out = out;
  p.pos = pos;
  p.out_rows = out_rows;
  p.ln_w = ln_w;
  p.ln_b = ln_b;
  p.in_stride = in_stride;
  p.out_stride = out_stride;
  p.out_cap = out_cap;
  p.heads = heads;
  p.n_rope = n_rope;
  p.layer_norm = layer_norm ? 1 : 0;
  p.hadamard = hadamard ? 1 : 0;
  p.eps = eps;
  p.hscale = (float)(1.0 / sqrt((double)dim));
  if (in_bf16)
    return out_bf16 ? launch_rotate_t<bf16, bf16>(n_rows, dim, p, st) : launch_rotate_t<bf16, float>(n_rows, dim, p, st);
  return out_bf16 ? launch_rotate_t<float, bf16>(n_rows, dim, p, st) : launch_rotate_t<float, float>(n_rows, dim, p, st);
}

}  // namespace dsa
