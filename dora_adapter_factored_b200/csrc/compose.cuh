// Fused DoRA compose, forward and backward ("Scaling DoRA ...", section 3:
// one pass that reads base and lora once and writes the output once, with the
// near-unity correction (g - 1) formed in fp32; backward writes d_base and
// d_lora in one pass and reduces dm over tokens without atomics).
//
// Both kernels are HBM-bound streams: 16-byte vector loads/stores along
// d_out, each thread keeps its columns' coefficients in registers and walks
// rows; four rows are loaded before any is used so that enough bytes are in
// flight.  No tensor cores.
#pragma once

#include "common.cuh"

namespace dora {

// Grid shaping for the [T, d_out] streams.  Depends on the shape only (not on
// the device), so that the backward's partial layout -- and therefore dm's
// summation order -- is the same on every run.
constexpr int kStreamThreads = 256;
constexpr int kStreamRowUnroll = 4;
constexpr int kStreamTargetBlocks = 148 * 8;

struct StreamGrid {
  int bx, by;
  int gx, gy;
};

inline StreamGrid stream_grid(long long T, int ncv) {
  StreamGrid g;
  int best = 256;
  long long best_waste = -1;
  for (int bx = 256; bx >= 32; bx >>= 1) {
    const long long waste = ceil_div_ll(ncv, bx) * bx - ncv;
    if (best_waste < 0 || waste < best_waste) {
      best = bx;
      best_waste = waste;
    }
  }
  g.bx = best;
  g.by = kStreamThreads / best;
  g.gx = static_cast<int>(ceil_div_ll(ncv, g.bx));
  long long want_y = kStreamTargetBlocks / g.gx;
  if (want_y < 1) want_y = 1;
  const long long max_y = ceil_div_ll(T, static_cast<long long>(g.by) * kStreamRowUnroll);
  g.gy = static_cast<int>(want_y < max_y ? want_y : max_y);
  if (g.gy < 1) g.gy = 1;
  return g;
}

template <typename T, int VEC>
struct VecIO;

template <>
struct VecIO<__nv_bfloat16, 8> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 u = __ldcs(reinterpret_cast<const uint4*>(p));
    v[0] = bf16lo_to_f32(u.x); v[1] = bf16hi_to_f32(u.x);
    v[2] = bf16lo_to_f32(u.y); v[3] = bf16hi_to_f32(u.y);
    v[4] = bf16lo_to_f32(u.z); v[5] = bf16hi_to_f32(u.z);
    v[6] = bf16lo_to_f32(u.w); v[7] = bf16hi_to_f32(u.w);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&v)[8]) {
    uint4 u;
    u.x = pack_bf16x2_rn(v[0], v[1]);
    u.y = pack_bf16x2_rn(v[2], v[3]);
    u.z = pack_bf16x2_rn(v[4], v[5]);
    u.w = pack_bf16x2_rn(v[6], v[7]);
    __stcs(reinterpret_cast<uint4*>(p), u);
  }
};

template <>
struct VecIO<float, 4> {
  static __device__ __forceinline__ void load(const float* p, float (&v)[4]) {
    const float4 u = __ldcs(reinterpret_cast<const float4*>(p));
    v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
  }
  static __device__ __forceinline__ void store(float* p, const float (&v)[4]) {
    __stcs(reinterpret_cast<float4*>(p), make_float4(v[0], v[1], v[2], v[3]));
  }
};

template <>
struct VecIO<__nv_bfloat16, 1> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&v)[1]) {
    v[0] = __bfloat162float(*p);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&v)[1]) {
    *p = __float2bfloat16_rn(v[0]);
  }
};

template <>
struct VecIO<float, 1> {
  static __device__ __forceinline__ void load(const float* p, float (&v)[1]) { v[0] = *p; }
  static __device__ __forceinline__ void store(float* p, const float (&v)[1]) { *p = v[0]; }
};

// y = base + ((g - 1) base + (g s) lora), (g - 1) = (m - n_c)/n_c, g = m/n_c.
template <typename T, int VEC>
__global__ void __launch_bounds__(kStreamThreads)
    compose_fwd_kernel(const T* __restrict__ base, const T* __restrict__ lora,
                       const float* __restrict__ m, const float* __restrict__ n, float s,
                       float eps, long long T_rows, int d_out, T* y) {
  const int cv = blockIdx.x * blockDim.x + threadIdx.x;
  const int col0 = cv * VEC;
  if (col0 >= d_out) return;
  float gm1[VEC], gs[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    const float nc = fmaxf(__ldg(n + col0 + e), eps);
    const float mm = __ldg(m + col0 + e);
    gm1[e] = __fdiv_rn(mm - nc, nc);
    gs[e] = __fdiv_rn(mm, nc) * s;
  }
  const long long stride = static_cast<long long>(gridDim.y) * blockDim.y;
  long long t = static_cast<long long>(blockIdx.y) * blockDim.y + threadIdx.y;
  for (; t < T_rows; t += kStreamRowUnroll * stride) {
    float b[kStreamRowUnroll][VEC], l[kStreamRowUnroll][VEC];
#pragma unroll
    for (int u = 0; u < kStreamRowUnroll; ++u) {
      const long long tt = t + u * stride;
      if (tt < T_rows) {
        const size_t off = static_cast<size_t>(tt) * d_out + col0;
        VecIO<T, VEC>::load(base + off, b[u]);
        VecIO<T, VEC>::load(lora + off, l[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < kStreamRowUnroll; ++u) {
      const long long tt = t + u * stride;
      if (tt < T_rows) {
        float o[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) o[e] = b[u][e] + fmaf(gm1[e], b[u][e], gs[e] * l[u][e]);
        VecIO<T, VEC>::store(y + static_cast<size_t>(tt) * d_out + col0, o);
      }
    }
  }
}

// d_base = g dy, d_lora = (g s) dy, and per-block column partials of
// sum_t dy (base + s lora) written to partial[blockIdx.y][d_out].
template <typename T, int VEC>
__global__ void __launch_bounds__(kStreamThreads)
    compose_bwd_kernel(const T* dy, const T* __restrict__ base, const T* __restrict__ lora,
                       const float* __restrict__ m, const float* __restrict__ n, float s,
                       float eps, long long T_rows, int d_out, T* d_base, T* __restrict__ d_lora,
                       float* __restrict__ partial) {
  __shared__ float red[kStreamThreads * VEC];
  const int cv = blockIdx.x * blockDim.x + threadIdx.x;
  const int col0 = cv * VEC;
  const bool active = col0 < d_out;
  float g[VEC], gs[VEC], acc[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    acc[e] = 0.f;
    g[e] = gs[e] = 0.f;
    if (active) {
      const float nc = fmaxf(__ldg(n + col0 + e), eps);
      g[e] = __fdiv_rn(__ldg(m + col0 + e), nc);
      gs[e] = g[e] * s;
    }
  }
  if (active) {
    const long long stride = static_cast<long long>(gridDim.y) * blockDim.y;
    long long t = static_cast<long long>(blockIdx.y) * blockDim.y + threadIdx.y;
    for (; t < T_rows; t += kStreamRowUnroll * stride) {
      float d[kStreamRowUnroll][VEC], b[kStreamRowUnroll][VEC], l[kStreamRowUnroll][VEC];
#pragma unroll
      for (int u = 0; u < kStreamRowUnroll; ++u) {
        const long long tt = t + u * stride;
        if (tt < T_rows) {
          const size_t off = static_cast<size_t>(tt) * d_out + col0;
          VecIO<T, VEC>::load(dy + off, d[u]);
          VecIO<T, VEC>::load(base + off, b[u]);
          VecIO<T, VEC>::load(lora + off, l[u]);
        }
      }
#pragma unroll
      for (int u = 0; u < kStreamRowUnroll; ++u) {
        const long long tt = t + u * stride;
        if (tt < T_rows) {
          float ob[VEC], ol[VEC];
#pragma unroll
          for (int e = 0; e < VEC; ++e) {
            ob[e] = g[e] * d[u][e];
            ol[e] = gs[e] * d[u][e];
            acc[e] = fmaf(d[u][e], fmaf(s, l[u][e], b[u][e]), acc[e]);
          }
          const size_t off = static_cast<size_t>(tt) * d_out + col0;
          VecIO<T, VEC>::store(d_base + off, ob);
          VecIO<T, VEC>::store(d_lora + off, ol);
        }
      }
    }
  }
  // Reduce the block's rows (threadIdx.y) in a fixed order.
  const int tx = threadIdx.x, ty = threadIdx.y;
#pragma unroll
  for (int e = 0; e < VEC; ++e) red[(ty * blockDim.x + tx) * VEC + e] = acc[e];
  __syncthreads();
  if (ty == 0 && active) {
    for (int yy = 1; yy < static_cast<int>(blockDim.y); ++yy)
#pragma unroll
      for (int e = 0; e < VEC; ++e) acc[e] += red[(yy * blockDim.x + tx) * VEC + e];
    float* dst = partial + static_cast<size_t>(blockIdx.y) * d_out + col0;
#pragma unroll
    for (int e = 0; e < VEC; ++e) dst[e] = acc[e];
  }
}

// dm_j = (sum over row chunks, in chunk order) / max(n_j, eps).
__global__ void __launch_bounds__(256)
    colsum_finalize_kernel(const float* __restrict__ partial, int chunks, int d_out,
                           const float* __restrict__ n, float eps, float* __restrict__ dm) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= d_out) return;
  float s = 0.f;
  for (int c = 0; c < chunks; ++c) s += partial[static_cast<size_t>(c) * d_out + j];
  dm[j] = __fdiv_rn(s, fmaxf(__ldg(n + j), eps));
}

}  // namespace dora
