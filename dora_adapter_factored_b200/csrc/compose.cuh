// Fused DoRA compose, forward and backward ("Scaling DoRA ...", section 3:
// one pass that reads base and lora once and writes the output once, with the
// near-unity correction (g - 1) formed in fp32; backward writes d_base and
// d_lora in one pass and reduces dm over tokens without atomics).
//
// Variants ("Scaling DoRA ...", section 4, tiers 1 and 2, and section 6):
//   * forward, optionally also writing inner = base + s lora (the training
//     forward's second output, kept for the backward instead of base and lora);
//   * backward from base and lora (5 passes), from inner (4 passes: dy and
//     inner in, d_base and d_lora out), or with the magnitude frozen (3
//     passes, no dm);
//   * grouped: one launch over all the modules of a layer, each module its own
//     slice of the grid (the launch-latency regime of small activations).
//
// All kernels are HBM-bound streams: 16-byte vector loads/stores along
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
constexpr int kStreamCtasPerSm = 2;  // resident blocks per SM the kernels are built for
constexpr int kFwdRowUnroll = 8;
constexpr int kBwdRowUnroll = 4;
constexpr int kStreamSlots = 148 * kStreamCtasPerSm;

// Backward variants: what the pass reads besides dy, and whether dm is formed.
enum BwdMode : int {
  kBwdFromBaseLora = 0,  // dy, base, lora -> d_base, d_lora, dm partials
  kBwdFromInner = 1,     // dy, inner      -> d_base, d_lora, dm partials
  kBwdFrozen = 2,        // dy             -> d_base, d_lora
};
// Rows in flight per thread: fewer input streams leave room for more rows.
__host__ __device__ constexpr int bwd_row_unroll(int mode) {
  return mode == kBwdFromBaseLora ? kBwdRowUnroll : (mode == kBwdFromInner ? 6 : 8);
}

struct StreamGrid {
  int bx, by;
  int gx, gy;
};

// `slots`: blocks the grid aims at (a module of a grouped launch gets its
// share of the launch's slots).  `bx_fixed` > 0 sets the block's width in
// column vectors; otherwise the widest with the fewest idle columns.
inline StreamGrid stream_grid(long long T, int ncv, int unroll, long long slots = kStreamSlots,
                              int bx_fixed = 0) {
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
  g.bx = bx_fixed > 0 ? bx_fixed : best;
  g.by = kStreamThreads / g.bx;
  g.gx = static_cast<int>(ceil_div_ll(ncv, g.bx));
  long long want_y = slots / g.gx;
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

// ---------------------------------------------------------------------------
// Row loops shared by the single-module and grouped kernels.  A thread owns
// VEC consecutive columns from col0 and rows t, t + stride, ...
// ---------------------------------------------------------------------------

// Per-column coefficients: gm1 = (m - n_c)/n_c, gs = (m/n_c) s, n_c = max(n, eps).
template <int VEC>
__device__ __forceinline__ void fwd_coefficients(const float* __restrict__ m,
                                                 const float* __restrict__ n, float s, float eps,
                                                 int col0, float (&gm1)[VEC], float (&gs)[VEC]) {
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    const float nc = fmaxf(__ldg(n + col0 + e), eps);
    const float mm = __ldg(m + col0 + e);
    gm1[e] = __fdiv_rn(mm - nc, nc);
    gs[e] = __fdiv_rn(mm, nc) * s;
  }
}

// Outputs of the forward pass.
enum FwdOut : int {
  kFwdY = 0,       // y = base + ((g - 1) base + (g s) lora)
  kFwdYInner = 1,  // y, and inner = base + s lora
  kFwdDelta = 2,   // dY = (g - 1) base + (g s) lora only, for a caller that adds Y_base
};

template <typename T, int VEC, typename Idx, int kOut>
__device__ __forceinline__ void fwd_rows(const T* __restrict__ base, const T* __restrict__ lora,
                                         const float (&gm1)[VEC], const float (&gs)[VEC], float s,
                                         long long t, long long stride, long long T_rows,
                                         int d_out, int col0, T* y, T* inner) {
  using P = Pack<T, VEC>;
  // 64-bit offsets take twice the registers per row in flight: half the rows.
  constexpr int U = sizeof(Idx) == 8 ? kFwdRowUnroll / 2 : kFwdRowUnroll;
  for (; t < T_rows; t += U * stride) {
    typename P::raw rb[U], rl[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long tt = t + u * stride;
      if (tt < T_rows) {
        const Idx off = static_cast<Idx>(tt) * static_cast<Idx>(d_out) + static_cast<Idx>(col0);
        rb[u] = P::load(base + off);
        rl[u] = P::load(lora + off);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long tt = t + u * stride;
      if (tt < T_rows) {
        float b[VEC], l[VEC], o[VEC];
        P::unpack(rb[u], b);
        P::unpack(rl[u], l);
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          const float d = fmaf(gm1[e], b[e], gs[e] * l[e]);
          o[e] = kOut == kFwdDelta ? d : b[e] + d;
        }
        const Idx off = static_cast<Idx>(tt) * static_cast<Idx>(d_out) + static_cast<Idx>(col0);
        if (!DORA_BOUNDS_OK(col0 >= 0 && col0 + VEC <= d_out)) continue;
        P::store(y + off, P::pack(o));
        if (kOut == kFwdYInner) {
          float in[VEC];
#pragma unroll
          for (int e = 0; e < VEC; ++e) in[e] = fmaf(s, l[e], b[e]);
          P::store(inner + off, P::pack(in));
        }
      }
    }
  }
}

// d_base = g dy, d_lora = (g s) dy, and (unless frozen) the thread's column
// sums of dy (base + s lora), or of dy inner, accumulated into acc.
// x1 / x2: base / lora (kBwdFromBaseLora), inner / unused (kBwdFromInner).
template <typename T, int VEC, typename Idx, int kMode>
__device__ __forceinline__ void bwd_rows(const T* dy, const T* __restrict__ x1,
                                         const T* __restrict__ x2, const float (&g)[VEC],
                                         const float (&gs)[VEC], float s, long long t,
                                         long long stride, long long T_rows, int d_out, int col0,
                                         T* d_base, T* __restrict__ d_lora, float (&acc)[VEC]) {
  using P = Pack<T, VEC>;
  constexpr int U = sizeof(Idx) == 8 ? (bwd_row_unroll(kMode) + 1) / 2 : bwd_row_unroll(kMode);
  for (; t < T_rows; t += U * stride) {
    typename P::raw rd[U], r1[U], r2[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long tt = t + u * stride;
      if (tt < T_rows) {
        const Idx off = static_cast<Idx>(tt) * static_cast<Idx>(d_out) + static_cast<Idx>(col0);
        rd[u] = P::load(dy + off);
        if (kMode != kBwdFrozen) r1[u] = P::load(x1 + off);
        if (kMode == kBwdFromBaseLora) r2[u] = P::load(x2 + off);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long tt = t + u * stride;
      if (tt < T_rows) {
        float d[VEC], ob[VEC], ol[VEC];
        P::unpack(rd[u], d);
        if (kMode == kBwdFromBaseLora) {
          float b[VEC], l[VEC];
          P::unpack(r1[u], b);
          P::unpack(r2[u], l);
#pragma unroll
          for (int e = 0; e < VEC; ++e) acc[e] = fmaf(d[e], fmaf(s, l[e], b[e]), acc[e]);
        } else if (kMode == kBwdFromInner) {
          float in[VEC];
          P::unpack(r1[u], in);
#pragma unroll
          for (int e = 0; e < VEC; ++e) acc[e] = fmaf(d[e], in[e], acc[e]);
        }
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          ob[e] = g[e] * d[e];
          ol[e] = gs[e] * d[e];
        }
        const Idx off = static_cast<Idx>(tt) * static_cast<Idx>(d_out) + static_cast<Idx>(col0);
        if (!DORA_BOUNDS_OK(col0 >= 0 && col0 + VEC <= d_out)) continue;
        P::store(d_base + off, P::pack(ob));
        P::store(d_lora + off, P::pack(ol));
      }
    }
  }
}

// Sums acc over the block's rows (ty = 0 .. by-1, in that order) and writes
// the block's column partials to dst (row ty = 0 only).
template <int VEC>
__device__ __forceinline__ void bwd_block_partial(float (&acc)[VEC], float* red, int tx, int ty,
                                                  int bx, int by, bool active, float* dst) {
  if (by > 1) {
#pragma unroll
    for (int e = 0; e < VEC; ++e) red[(ty * bx + tx) * VEC + e] = acc[e];
    __syncthreads();
    if (ty == 0 && active) {
      for (int yy = 1; yy < by; ++yy)
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] += red[(yy * bx + tx) * VEC + e];
    }
  }
  if (ty == 0 && active) {
#pragma unroll
    for (int e = 0; e < VEC; ++e) dst[e] = acc[e];
  }
}

// dm_j = (sum of the chunk partials of column j, in a fixed order) / n_c,j.
// Block (32, 8): thread (x, y) sums chunks y, y + 8, ... of column x, then
// the eight sums are added in y order.
__device__ __forceinline__ void colsum_column(const float* __restrict__ partial, int chunks,
                                              int d_out, const float* __restrict__ n, float eps,
                                              float* __restrict__ dm, int j) {
  __shared__ float red[8][33];
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

// ---------------------------------------------------------------------------
// Single module
// ---------------------------------------------------------------------------

// y = base + ((g - 1) base + (g s) lora), (g - 1) = (m - n_c)/n_c, g = m/n_c;
// kOut adds inner = base + s lora, or writes dY = y - base alone (FwdOut).
// Idx is the element-offset type: 32-bit when T * d_out < 2^31 (fewer live
// registers per in-flight row), 64-bit otherwise.
template <typename T, int VEC, typename Idx, int kOut>
__global__ void __launch_bounds__(kStreamThreads, kStreamCtasPerSm)
    compose_fwd_kernel(const T* __restrict__ base, const T* __restrict__ lora,
                       const float* __restrict__ m, const float* __restrict__ n, float s,
                       float eps, long long T_rows, int d_out, T* y, T* inner) {
  grid_dependency_wait();
  grid_dependency_trigger();
  const int cv = blockIdx.x * blockDim.x + threadIdx.x;
  const int col0 = cv * VEC;
  if (col0 >= d_out) return;
  float gm1[VEC], gs[VEC];
  fwd_coefficients<VEC>(m, n, s, eps, col0, gm1, gs);
  const long long stride = static_cast<long long>(gridDim.y) * blockDim.y;
  const long long t = static_cast<long long>(blockIdx.y) * blockDim.y + threadIdx.y;
  fwd_rows<T, VEC, Idx, kOut>(base, lora, gm1, gs, s, t, stride, T_rows, d_out, col0, y, inner);
}

// d_base = g dy, d_lora = (g s) dy, and (unless frozen) per-block column
// partials of sum_t dy (base + s lora), or of sum_t dy inner, written to
// partial[blockIdx.y][d_out].
template <typename T, int VEC, typename Idx, int kMode>
__global__ void __launch_bounds__(kStreamThreads, kStreamCtasPerSm)
    compose_bwd_kernel(const T* dy, const T* __restrict__ x1, const T* __restrict__ x2,
                       const float* __restrict__ m, const float* __restrict__ n, float s,
                       float eps, long long T_rows, int d_out, T* d_base, T* __restrict__ d_lora,
                       float* __restrict__ partial) {
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
    const long long t = static_cast<long long>(blockIdx.y) * blockDim.y + threadIdx.y;
    bwd_rows<T, VEC, Idx, kMode>(dy, x1, x2, g, gs, s, t, stride, T_rows, d_out, col0, d_base,
                                 d_lora, acc);
  }
  if (kMode != kBwdFrozen)
    bwd_block_partial<VEC>(acc, red, threadIdx.x, threadIdx.y, blockDim.x, blockDim.y, active,
                           partial + static_cast<size_t>(blockIdx.y) * d_out + col0);
}

__global__ void __launch_bounds__(256)
    colsum_finalize_kernel(const float* __restrict__ partial, int chunks, int d_out,
                           const float* __restrict__ n, float eps, float* __restrict__ dm) {
  grid_dependency_wait();
  grid_dependency_trigger();
  colsum_column(partial, chunks, d_out, n, eps, dm, blockIdx.x * 32 + threadIdx.x);
}

// ---------------------------------------------------------------------------
// Grouped: one launch for several modules.  Module p owns blocks
// [blk_begin, blk_begin + gx gy) of a 1-D grid of 256-thread blocks, laid out
// as its own (gx, gy) grid of (bx, 256 / bx) blocks; the dm reduction owns
// blocks [cblk_begin, cblk_begin + ceil(d_out / 32)) of its launch.
// ---------------------------------------------------------------------------
constexpr int kMaxComposeGroup = 64;

struct ComposeItem {
  const void* in0;    // forward: base;  backward: dy
  const void* in1;    // forward: lora;  backward: base, or inner
  const void* in2;    // backward from base and lora: lora
  const float* m;
  const float* n;
  void* out0;         // forward: y;     backward: d_base
  void* out1;         // forward: inner (or null);  backward: d_lora
  float* partial;     // backward: [gy][d_out] column partials
  float* dm;          // backward: [d_out]
  long long T;
  int d_out;
  float s;
  int bx, gx, gy;     // threads along columns per block, module grid
  int blk_begin, cblk_begin;
};

struct ComposeGroup {
  int count;
  float eps;
  ComposeItem it[kMaxComposeGroup];
};

__device__ __forceinline__ int compose_item_of_block(const ComposeGroup& grp, int blk, bool dm) {
  int p = 0;
  while (p + 1 < grp.count && (dm ? grp.it[p + 1].cblk_begin : grp.it[p + 1].blk_begin) <= blk)
    ++p;
  return p;
}

template <typename T, int VEC, typename Idx>
__global__ void __launch_bounds__(kStreamThreads, kStreamCtasPerSm)
    compose_fwd_grouped_kernel(const __grid_constant__ ComposeGroup grp) {
  grid_dependency_wait();
  grid_dependency_trigger();
  const ComposeItem& it = grp.it[compose_item_of_block(grp, blockIdx.x, false)];
  const int local = static_cast<int>(blockIdx.x) - it.blk_begin;
  const int bx = it.bx, by = kStreamThreads / it.bx;
  const int tx = threadIdx.x % bx, ty = threadIdx.x / bx;
  const int col0 = ((local % it.gx) * bx + tx) * VEC;
  if (col0 >= it.d_out) return;
  float gm1[VEC], gs[VEC];
  fwd_coefficients<VEC>(it.m, it.n, it.s, grp.eps, col0, gm1, gs);
  const long long stride = static_cast<long long>(it.gy) * by;
  const long long t = static_cast<long long>(local / it.gx) * by + ty;
  const T* base = static_cast<const T*>(it.in0);
  const T* lora = static_cast<const T*>(it.in1);
  if (it.out1 != nullptr)
    fwd_rows<T, VEC, Idx, kFwdYInner>(base, lora, gm1, gs, it.s, t, stride, it.T, it.d_out, col0,
                                static_cast<T*>(it.out0), static_cast<T*>(it.out1));
  else
    fwd_rows<T, VEC, Idx, kFwdY>(base, lora, gm1, gs, it.s, t, stride, it.T, it.d_out, col0,
                                 static_cast<T*>(it.out0), nullptr);
}

template <typename T, int VEC, typename Idx, int kMode>
__global__ void __launch_bounds__(kStreamThreads, kStreamCtasPerSm)
    compose_bwd_grouped_kernel(const __grid_constant__ ComposeGroup grp) {
  __shared__ float red[kStreamThreads * VEC];
  grid_dependency_wait();
  grid_dependency_trigger();
  const ComposeItem& it = grp.it[compose_item_of_block(grp, blockIdx.x, false)];
  const int local = static_cast<int>(blockIdx.x) - it.blk_begin;
  const int bx = it.bx, by = kStreamThreads / it.bx;
  const int tx = threadIdx.x % bx, ty = threadIdx.x / bx;
  const int col0 = ((local % it.gx) * bx + tx) * VEC;
  const bool active = col0 < it.d_out;
  float g[VEC], gs[VEC], acc[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    acc[e] = 0.f;
    g[e] = gs[e] = 0.f;
    if (active) {
      const float nc = fmaxf(__ldg(it.n + col0 + e), grp.eps);
      g[e] = __fdiv_rn(__ldg(it.m + col0 + e), nc);
      gs[e] = g[e] * it.s;
    }
  }
  if (active) {
    const long long stride = static_cast<long long>(it.gy) * by;
    const long long t = static_cast<long long>(local / it.gx) * by + ty;
    bwd_rows<T, VEC, Idx, kMode>(static_cast<const T*>(it.in0), static_cast<const T*>(it.in1),
                                 static_cast<const T*>(it.in2), g, gs, it.s, t, stride, it.T,
                                 it.d_out, col0, static_cast<T*>(it.out0),
                                 static_cast<T*>(it.out1), acc);
  }
  if (kMode != kBwdFrozen)
    bwd_block_partial<VEC>(acc, red, tx, ty, bx, by, active,
                           it.partial + static_cast<size_t>(local / it.gx) * it.d_out + col0);
}

__global__ void __launch_bounds__(256)
    colsum_grouped_kernel(const __grid_constant__ ComposeGroup grp) {
  grid_dependency_wait();
  grid_dependency_trigger();
  const ComposeItem& it = grp.it[compose_item_of_block(grp, blockIdx.x, true)];
  const int j = (static_cast<int>(blockIdx.x) - it.cblk_begin) * 32 + threadIdx.x;
  colsum_column(it.partial, it.gy, it.d_out, it.n, grp.eps, it.dm, j);
}

}  // namespace dora
