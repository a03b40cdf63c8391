// Factored DoRA row norm on CUDA cores, for fp32 modules (where bf16 or tf32
// tensor-core products would not meet fp32 accuracy) and for bf16 shapes the
// TMA path cannot describe (d_in or r not a multiple of 8, or unaligned
// pointers).  Same three terms as the tensor-core path ("Scaling DoRA ...",
// section 2): ||W0_i||^2 + 2 s B_i.(W0 A^T)_i + s^2 B_i G B_i^T, G = A A^T,
// all accumulated in fp32.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace dora {

template <typename T>
__device__ __forceinline__ float load_f32(const T* p);
template <>
__device__ __forceinline__ float load_f32<float>(const float* p) {
  return __ldg(p);
}
template <>
__device__ __forceinline__ float load_f32<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(__ldg(p));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Fixed-order block sum for 256 threads; result valid in every thread.
__device__ __forceinline__ float block_sum_256(float v, float* red /* [8] */) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) s += red[i];
  return s;
}

// G[i][j] = sum_k A[i][k] A[j][k]: one warp per (i, j), lanes split k.
template <typename T>
__global__ void __launch_bounds__(256)
    gram_simt_kernel(const T* __restrict__ A, int r, int d_in, float* __restrict__ G) {
  const int warp_global = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp_global >= r * r) return;
  const int i = warp_global / r, j = warp_global % r;
  if (j < i) return;  // upper triangle; mirrored below
  const T* ai = A + static_cast<size_t>(i) * d_in;
  const T* aj = A + static_cast<size_t>(j) * d_in;
  float s = 0.f;
  for (int k = lane; k < d_in; k += 32) s = fmaf(load_f32(ai + k), load_f32(aj + k), s);
  s = warp_sum(s);
  if (lane == 0) {
    G[static_cast<size_t>(i) * r + j] = s;
    G[static_cast<size_t>(j) * r + i] = s;
  }
}

// One block of 256 threads per output row.
template <typename T>
__global__ void __launch_bounds__(256)
    norm_simt_kernel(const T* __restrict__ W0, const T* __restrict__ A, const T* __restrict__ B,
                     const float* __restrict__ G, int d_out, int d_in, int r, float s,
                     const float* __restrict__ m, float eps, float* __restrict__ n_out,
                     float* __restrict__ g_out, int emit_sq) {
  __shared__ float U[DORA_MAX_RANK];
  __shared__ float Bi[DORA_MAX_RANK];
  __shared__ float red[8];
  const int i = blockIdx.x;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const T* wrow = W0 + static_cast<size_t>(i) * d_in;

  for (int c = tid; c < r; c += 256) Bi[c] = load_f32(B + static_cast<size_t>(i) * r + c);

  // base term ||W0_i||^2
  float ss = 0.f;
  for (int k = tid; k < d_in; k += 256) {
    const float v = load_f32(wrow + k);
    ss = fmaf(v, v, ss);
  }
  ss = block_sum_256(ss, red);

  // U_c = W0_i . A_c, one warp per c
  for (int c = w; c < r; c += 8) {
    const T* ac = A + static_cast<size_t>(c) * d_in;
    float u = 0.f;
    for (int k = lane; k < d_in; k += 32) u = fmaf(load_f32(wrow + k), load_f32(ac + k), u);
    u = warp_sum(u);
    if (lane == 0) U[c] = u;
  }
  __syncthreads();

  // cross term B_i . U  and Gram term B_i G B_i^T
  float cross = 0.f, gram = 0.f;
  for (int c = tid; c < r; c += 256) {
    cross = fmaf(Bi[c], U[c], cross);
    const float* gc = G + static_cast<size_t>(c) * r;
    float gb = 0.f;
    for (int d = 0; d < r; ++d) gb = fmaf(gc[d], Bi[d], gb);
    gram = fmaf(Bi[c], gb, gram);
  }
  cross = block_sum_256(cross, red);
  gram = block_sum_256(gram, red);

  if (tid == 0) {
    const float sq = ss + 2.f * s * cross + s * s * gram;
    if (emit_sq) {
      n_out[i] = sq;
      return;
    }
    const float n = __fsqrt_rn(fmaxf(sq, 0.f));
    n_out[i] = n;
    if (m != nullptr && g_out != nullptr) g_out[i] = __fdiv_rn(m[i], fmaxf(n, eps));
  }
}

// n_i = sqrt(max(sq_i, 0)), g_i = m_i / max(n_i, eps): the finalize of a norm
// whose squared sums were reduced across devices.
__global__ void __launch_bounds__(256)
    norm_finalize_sq_kernel(const float* __restrict__ sq, int d_out, const float* __restrict__ m,
                            float eps, float* __restrict__ n_out, float* __restrict__ g_out) {
  grid_dependency_wait();
  grid_dependency_trigger();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= d_out) return;
  const float n = __fsqrt_rn(fmaxf(sq[i], 0.f));
  n_out[i] = n;
  if (m != nullptr && g_out != nullptr) g_out[i] = __fdiv_rn(m[i], fmaxf(n, eps));
}

}  // namespace dora
