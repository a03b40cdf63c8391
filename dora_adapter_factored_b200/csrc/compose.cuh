// Fused DoRA compose, forward and backward ("Scaling DoRA ...", section 3:
// one pass that reads base and lora once and writes the output once, with the
// near-unity correction (g - 1) formed in fp32; backward writes d_base and
// d_lora in one pass and reduces dm over tokens without atomics).
//
// Both kernels are HBM-bound streams: 16-byte vector loads/stores along
// d_out, each thread keeps its columns' coefficients in registers and walks
// rows; several rows are loaded (as raw 16-byte registers) before any is
// used so that enough bytes are in flight.  No tensor cores.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace dora {

// Grid shaping for the [T, d_out] streams: a persistent grid of about two
// blocks per SM (one wave), each block walking rows.  It depends on the shape
// only (not on the device), so that the backward's partial layout -- and
// therefore dm's summation order -- is the same on every run.
constexpr int kStreamThreads = 256;
constexpr int kFwdRowUnroll = 8;
constexpr int kBwdRowUnroll = 4;
constexpr int kStreamSlots = 148 * 2;

struct StreamGrid {
  int bx, by;
  int gx, gy;
};

inline StreamGrid stream_grid(long long T, int ncv, int unroll) {
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
  long long want_y = kStreamSlots / g.gx;
  if (want_y < 1) want_y = 1;
  const long long max_y = ceil_div_ll(T, static_cast<long long>(g.by) * unroll);
  g.gy = static_cast<int>(want_y < max_y ? want_y : max_y);
  if (g.gy < 1) g.gy = 1;
  return g;
}

// Raw 16-byte (or scalar) register images of VEC consecutive elements, so that
// several rows can be in flight without unpacking them first.
template <typename T, int VEC>
struct Pack;

template <>
struct Pack<__nv_bfloat16, 8> {
  using raw = uint4;
  static __device__ __forceinline__ raw load(const __nv_bfloat16* p) {
    return __ldcs(reinterpret_cast<const uint4*>(p));
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const raw& u) {
    __stcs(reinterpret_cast<uint4*>(p), u);
  }
  static __device__ __forceinline__ void unpack(const raw& u, float (&v)[8]) {
    v[0] = bf16lo_to_f32(u.x); v[1] = bf16hi_to_f32(u.x);
    v[2] = bf16lo_to_f32(u.y); v[3] = bf16hi_to_f32(u.y);
    v[4] = bf16lo_to_f32(u.z); v[5] = bf16hi_to_f32(u.z);
    v[6] = bf16lo_to_f32(u.w); v[7] = bf16hi_to_f32(u.w);
  }
  static __device__ __forceinline__ raw pack(const float (&v)[8]) {
    uint4 u;
    u.x = pack_bf16x2_rn(v[0], v[1]);
    u.y = pack_bf16x2_rn(v[2], v[3]);
    u.z = pack_bf16x2_rn(v[4], v[5]);
    u.w = pack_bf16x2_rn(v[6], v[7]);
    return u;
  }
};

template <>
struct Pack<float, 4> {
  using raw = float4;
  static __device__ __forceinline__ raw load(const float* p) {
    return __ldcs(reinterpret_cast<const float4*>(p));
  }
  static __device__ __forceinline__ void store(float* p, const raw& u) {
    __stcs(reinterpret_cast<float4*>(p), u);
  }
  static __device__ __forceinline__ void unpack(const raw& u, float (&v)[4]) {
    v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
  }
  static __device__ __forceinline__ raw pack(const float (&v)[4]) {
    return make_float4(v[0], v[1], v[2], v[3]);
  }
};

template <>
struct Pack<__nv_bfloat16, 1> {
  using raw = __nv_bfloat16;
  static __device__ __forceinline__ raw load(const __nv_bfloat16* p) { return *p; }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const raw& u) { *p = u; }
  static __device__ __forceinline__ void unpack(const raw& u, float (&v)[1]) {
    v[0] = __bfloat162float(u);
  }
  static __device__ __forceinline__ raw pack(const float (&v)[1]) {
    return __float2bfloat16_rn(v[0]);
  }
};

template <>
struct Pack<float, 1> {
  using raw = float;
  static __device__ __forceinline__ raw load(const float* p) { return *p; }
  static __device__ __forceinline__ void store(float* p, const raw& u) { *p = u; }
  static __device__ __forceinline__ void unpack(const raw& u, float (&v)[1]) { v[0] = u; }
  static __device__ __forceinline__ raw pack(const float (&v)[1]) { return v[0]; }
};

// y = base + ((g - 1) base + (g s) lora), (g - 1) = (m - n_c)/n_c, g = m/n_c.
// Idx is the element-offset type: 32-bit when T * d_out < 2^31 (fewer live
// registers per in-flight row), 64-bit otherwise.
template <typename T, int VEC, typename Idx>
__global__ void __launch_bounds__(kStreamThreads, 2)
    compose_fwd_kernel(const T* __restrict__ base, const T* __restrict__ lora,
                       const float* __restrict__ m, const float* __restrict__ n, float s,
                       float eps, long long T_rows, int d_out, T* y) {
  using P = Pack<T, VEC>;
  grid_dependency_wait();
  grid_dependency_trigger();
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
  for (; t < T_rows; t += kFwdRowUnroll * stride) {
    typename P::raw rb[kFwdRowUnroll], rl[kFwdRowUnroll];
#pragma unroll
    for (int u = 0; u < kFwdRowUnroll; ++u) {
      const long long tt = t + u * stride;
      if (tt < T_rows) {
        const Idx off = static_cast<Idx>(tt) * static_cast<Idx>(d_out) + static_cast<Idx>(col0);
        rb[u] = P::load(base + off);
        rl[u] = P::load(lora + off);
      }
    }
#pragma unroll
    for (int u = 0; u < kFwdRowUnroll; ++u) {
      const long long tt = t + u * stride;
      if (tt < T_rows) {
        float b[VEC], l[VEC], o[VEC];
        P::unpack(rb[u], b);
        P::unpack(rl[u], l);
#pragma unroll
        for (int e = 0; e < VEC; ++e) o[e] = b[e] + fmaf(gm1[e], b[e], gs[e] * l[e]);
        const Idx off = static_cast<Idx>(tt) * static_cast<Idx>(d_out) + static_cast<Idx>(col0);
        P::store(y + off, P::pack(o));
      }
    }
  }
}

// d_base = g dy, d_lora = (g s) dy, and per-block column partials of
// sum_t dy (base + s lora) written to partial[blockIdx.y][d_out].
template <typename T, int VEC, typename Idx>
__global__ void __launch_bounds__(kStreamThreads, 2)
    compose_bwd_kernel(const T* dy, const T* __restrict__ base, const T* __restrict__ lora,
                       const float* __restrict__ m, const float* __restrict__ n, float s,
                       float eps, long long T_rows, int d_out, T* d_base, T* __restrict__ d_lora,
                       float* __restrict__ partial) {
  using P = Pack<T, VEC>;
  __shared__ float red[kStreamThreads * VEC];
  grid_dependency_wait();
  grid_dependency_trigger();
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
    for (; t < T_rows; t += kBwdRowUnroll * stride) {
      typename P::raw rd[kBwdRowUnroll], rb[kBwdRowUnroll], rl[kBwdRowUnroll];
#pragma unroll
      for (int u = 0; u < kBwdRowUnroll; ++u) {
        const long long tt = t + u * stride;
        if (tt < T_rows) {
          const Idx off = static_cast<Idx>(tt) * static_cast<Idx>(d_out) + static_cast<Idx>(col0);
          rd[u] = P::load(dy + off);
          rb[u] = P::load(base + off);
          rl[u] = P::load(lora + off);
        }
      }
#pragma unroll
      for (int u = 0; u < kBwdRowUnroll; ++u) {
        const long long tt = t + u * stride;
        if (tt < T_rows) {
          float d[VEC], b[VEC], l[VEC], ob[VEC], ol[VEC];
          P::unpack(rd[u], d);
          P::unpack(rb[u], b);
          P::unpack(rl[u], l);
#pragma unroll
          for (int e = 0; e < VEC; ++e) {
            ob[e] = g[e] * d[e];
            ol[e] = gs[e] * d[e];
            acc[e] = fmaf(d[e], fmaf(s, l[e], b[e]), acc[e]);
          }
          const Idx off = static_cast<Idx>(tt) * static_cast<Idx>(d_out) + static_cast<Idx>(col0);
          P::store(d_base + off, P::pack(ob));
          P::store(d_lora + off, P::pack(ol));
        }
      }
    }
  }
  // Reduce the block's rows (threadIdx.y) in a fixed order.
  const int tx = threadIdx.x, ty = threadIdx.y;
  if (blockDim.y > 1) {
#pragma unroll
    for (int e = 0; e < VEC; ++e) red[(ty * blockDim.x + tx) * VEC + e] = acc[e];
    __syncthreads();
    if (ty == 0 && active) {
      for (int yy = 1; yy < static_cast<int>(blockDim.y); ++yy)
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] += red[(yy * blockDim.x + tx) * VEC + e];
    }
  }
  if (ty == 0 && active) {
    float* dst = partial + static_cast<size_t>(blockIdx.y) * d_out + col0;
#pragma unroll
    for (int e = 0; e < VEC; ++e) dst[e] = acc[e];
  }
}

// dm_j = (sum over row chunks, in a fixed order) / max(n_j, eps).  Block
// (32, 8): thread (x, y) sums chunks y, y + 8, ... of column x, then the
// eight sums are added in y order.
__global__ void __launch_bounds__(256)
    colsum_finalize_kernel(const float* __restrict__ partial, int chunks, int d_out,
                           const float* __restrict__ n, float eps, float* __restrict__ dm) {
  __shared__ float red[8][33];
  grid_dependency_wait();
  grid_dependency_trigger();
  const int j = blockIdx.x * 32 + threadIdx.x;
  float s = 0.f;
  if (j < d_out)
    for (int c = threadIdx.y; c < chunks; c += 8) s += partial[static_cast<size_t>(c) * d_out + j];
  red[threadIdx.y][threadIdx.x] = s;
  __syncthreads();
  if (threadIdx.y == 0 && j < d_out) {
    float t = red[0][threadIdx.x];
#pragma unroll
    for (int y = 1; y < 8; ++y) t += red[y][threadIdx.x];
    dm[j] = __fdiv_rn(t, fmaxf(__ldg(n + j), eps));
  }
}

}  // namespace dora
