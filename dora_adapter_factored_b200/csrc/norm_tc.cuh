// Factored DoRA row norm on the 5th-generation tensor cores (tcgen05 + TMEM,
// operands staged by TMA), following "Scaling DoRA: High-Rank Adaptation via
// Factored Norms and Fused Kernels", section 2: the squared norm of row i of
// W0 + s B A is ||W0_i||^2 + 2 s B_i.(W0 A^T)_i + s^2 B_i G B_i^T, G = A A^T,
// evaluated from [d_out, r] and [r, r] intermediates only.
//
// One persistent kernel on CTA pairs (after a tiny kernel that zeroes its
// counters) does the whole norm of one module, or of many (the grouped call):
//
//   Gram units   G = A A^T in pseudo-tiles of 256 rows of A: the A operand is
//                256 rows of A, the N-side operand the whole of A, k-blocks
//                over d_in.  A few pairs take these first; each posts its
//                fp32 partial, and once all of a pseudo-tile's partials are
//                posted, the pairs that posted them each sum a share of its
//                rows in a fixed order, scale by s/2 and write G' = (s/2) G
//                as two bf16 matrices, G'_hi = bf16(G') and
//                G'_lo = bf16(G' - G'_hi), so that the Gram term keeps
//                fp32-level accuracy (the pages' norm accumulates in fp32
//                whatever the weight dtype).  They store them transposed,
//                which the quadratic form B_i G' B_i^T does not see.
//   W0 units     per 256-row tile of W0, k-blocks over d_in: TMEM
//                accumulator += W0_tile A^T, while the reduction warps square
//                and sum the same W0 tile straight from shared memory
//                (||W0_i||^2), so W0 crosses HBM exactly once.
//   G units      per tile, k-blocks over r: accumulator += B_tile G'_hi, then
//                B_tile G'_lo; they wait until the module's G' is written.
//
// A segment (one pair's run of units on one tile) ends with an epilogue that
// drains TMEM, dots each row with B_i and posts the per-row partial
// ||W0_i||^2_part + 2 s B_i.acc_i: every term is linear in a k-range, so the
// partials of all segments of a tile simply add (B_i.acc_i over G units is
// (s/2) B_i G B_i^T).  The segment that posts a tile's partials last (an
// arrival counter per 32 rows) sums them in slot order and finalises those
// rows: n_i = sqrt(max(sum, 0)) and g_i = m_i / max(n_i, eps) (section 4,
// precision bullet).
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace dora {

constexpr int kTileM = 128;                  // W0 rows per CTA = TMEM lanes
constexpr int kPairM = 2 * kTileM;           // W0 rows per tile of a CTA pair
constexpr int kBlockK = 64;                  // bf16 of K per stage: one 128-byte swizzle row
constexpr int kMaxStages = 8;
constexpr int kEpiWarps = 8;                 // warps 0-7: reduction + epilogue
constexpr int kNormThreads = (kEpiWarps + 2) * 32;  // + warp 8 TMA, warp 9 MMA
constexpr int kMaxChunksPerHalf = 8;         // 32-column TMEM chunks per epilogue half (r <= 512)
constexpr int kPrefetchChunks = 6;           // of which B is prefetched into registers (r <= 384)
// Registers are granted to a block in groups of four warps, so the 10-warp
// kernel is charged as 12 warps: 65536 / 384 threads = 170 -> 168.
constexpr int kNormMaxRegs = 168;

constexpr uint32_t kTileABytes = kTileM * kBlockK * 2;  // 16 KiB
constexpr int kMaxDynSmem = 232448;          // 227 KiB opt-in per block on sm_100
constexpr int kTraceWords = 16;              // diagnostic trace words per CTA

enum NormPhase : int { kPhaseGram = 0, kPhaseW0 = 1, kPhaseG = 2 };

// ---------------------------------------------------------------------------
// Problem descriptors (built on the host; kernel parameter for one module,
// a workspace table for the grouped call).
// ---------------------------------------------------------------------------
struct alignas(64) NormProblemDev {
  CUtensorMap tm_w0;     // W0 [d_out, d_in], box 64 x 128
  CUtensorMap tm_arow;   // A  [r, d_in],     box 64 x 128: the Gram units' A operand
  CUtensorMap tm_a;      // A  as the N-side slab: box 64 x h0, or the 4-D view
                         //    {64, h0, 2 ranks, 2 chunks} with box {64, h0, 1, 2}
  CUtensorMap tm_b;      // B  [d_out, r],    box 64 x 128
  CUtensorMap tm_g;      // G'_hi (transposed) [r, r], like tm_a
  CUtensorMap tm_glo;    // G'_lo (transposed) [r, r], like tm_a
  const uint16_t* B;     // bf16 bits of B, for the epilogue dot
  uint16_t* g_hi;        // [r][r8] bf16 bits of (G'_hi)^T
  uint16_t* g_lo;        // [r][r8] bf16 bits of (G'_lo)^T
  float* partial;        // [tiles][seg_slots][256] per-row partials
  float* gram_part;      // [pg_tiles][gram_slots][n_pad][256] fp32 Gram partials
  int* tile_cnt;         // [tiles * 8] segments posted per 32-row quarter of each CTA's half
  int* gram_cnt;         // [pg_tiles * 2] Gram segments posted per pseudo-tile half
  int* g_ready;          // [1] rows of G' written (256 per pseudo-tile when complete)
  int* tile_w;           // [tiles] first pair | (pairs << 16) of each tile's W0 units
  const float* m;        // [d_out] or null
  float* n_out;          // [d_out]
  float* g_out;          // [d_out] or null
  long long begin[3];    // first unit of this module in its wave's Gram / W0 / G sequence
  int d_out, r, r8, n_pad;
  int n0, n1;            // N of the two pair-MMA chunks (n1 = 0: single chunk; else n1 = n0)
  int h0;                // slab rows of each chunk that one CTA stages: n0 / 2
  int slab4d;            // tm_a / tm_g / tm_glo are the 4-D view: one box per slab half
  int emit_sq;           // write the squared-norm sum itself to n_out (no clamp, sqrt or g)
  int kb_w, kb_r, tiles, pg_tiles, seg_slots, gram_slots;
  uint32_t pair_tx;      // bytes landing per stage in both CTAs together
  uint32_t idesc0, idesc1;
  float two_s, half_s;
};

// Units of phase `ph` per tile (per pseudo-tile for the Gram).
__host__ __device__ __forceinline__ int phase_per_tile(const NormProblemDev& P, int ph) {
  return ph == kPhaseG ? 2 * P.kb_r : P.kb_w;
}

// ---------------------------------------------------------------------------
// Schedule.  The grouped call splits its modules (in order) into waves whose
// re-read operands (A, G') fit in L2 together; one module alone is one wave.
// Within a wave every pair j takes, in this order, a contiguous range of the
// wave's Gram units, of its W0 units and of its G units:
//   Gram: pairs j < J share the n[0] Gram units evenly (the others have none),
//   G:    every pair gets an even share of the n[2] G units,
//   W0:   the rest of an even share of all units, where the Gram units count
//         as gw >= n[0] (the Gram pairs also post and reduce partials),
// so every pair has about the same work, the Gram is done early by a few
// pairs, and the G units (which need G') come last in every pair.  The
// boundaries are closed forms of j; the host checks that every pair's W0
// range is non-empty and the ranges are ordered.
// ---------------------------------------------------------------------------
constexpr int kMaxWaves = 64;
struct WaveInfo {
  long long n[3];  // units of the wave in the Gram, W0 and G sequences
  long long gw;    // what the Gram units weigh in the W0 split (>= n[0])
  int J;           // pairs that share the Gram units
  int m0, m1;      // modules [m0, m1) of the table
};
struct NormSched {
  int waves;
  int pairs;
  WaveInfo w[kMaxWaves];
};

// First unit of pair j's range of phase `ph` (j = pairs gives the total).
__host__ __device__ __forceinline__ long long sched_begin(const WaveInfo& w, int pairs, int ph,
                                                          int j) {
  const long long jj = j;
  const long long jg = jj < w.J ? jj : w.J;
  if (ph == kPhaseGram) return w.J > 0 ? jg * w.n[0] / w.J : 0;
  const long long gp = jj * w.n[2] / pairs;
  if (ph == kPhaseG) return gp;
  const long long gram_w = w.J > 0 ? jg * w.gw / w.J : 0;
  return jj * (w.gw + w.n[1] + w.n[2]) / pairs - gram_w - gp;
}

// The pair whose range of phase `ph` holds unit x (the last j with
// begin(j) <= x; pairs with empty ranges before it are skipped).
__host__ __device__ __forceinline__ int sched_pair_of(const WaveInfo& w, int pairs, int ph,
                                                      long long x) {
  int lo = 0, hi = pairs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) / 2;
    if (sched_begin(w, pairs, ph, mid) <= x)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

// The pair whose range holds unit x of a sequence of n units split evenly
// over q pairs (range j = [floor(j n / q), floor((j+1) n / q))).
__host__ __device__ __forceinline__ int even_owner(long long x, long long n, int q) {
  return static_cast<int>(((x + 1) * q - 1) / n);
}

// Slot of pair `me`'s segment among the segments of units [x0, x1) of a
// sequence of n units split evenly over q pairs (its segment starts at xs),
// and how many segments there are: consecutive pairs when every pair has a
// unit (n >= q), else one unit per pair.
__host__ __device__ __forceinline__ int even_segments(long long x0, long long x1, long long xs,
                                                      long long n, int q, int me, int* ord) {
  if (n >= q) {
    const int f = even_owner(x0, n, q);
    *ord = me - f;
    return even_owner(x1 - 1, n, q) - f + 1;
  }
  *ord = static_cast<int>(xs - x0);
  return static_cast<int>(x1 - x0);
}

// The segments of units [x0, x1) of phase `ph`, in order: returns how many
// there are and sets *ord to the position of pair `me`'s segment.
__host__ __device__ __forceinline__ int sched_segments(const WaveInfo& w, int pairs, int ph,
                                                       long long x0, long long x1, int me,
                                                       int* ord) {
  int nseg = 0;
  long long x = x0;
  while (x < x1) {
    const int j = sched_pair_of(w, pairs, ph, x);
    if (j == me && ord != nullptr) *ord = nseg;
    ++nseg;
    const long long e = sched_begin(w, pairs, ph, j + 1);
    x = e < x1 ? e : x1;
  }
  return nseg;
}

__device__ __forceinline__ float sumsq_bf16x8(uint4 v) {
  float a = 0.f, b = 0.f;
  a = fmaf(bf16lo_to_f32(v.x), bf16lo_to_f32(v.x), a);
  b = fmaf(bf16hi_to_f32(v.x), bf16hi_to_f32(v.x), b);
  a = fmaf(bf16lo_to_f32(v.y), bf16lo_to_f32(v.y), a);
  b = fmaf(bf16hi_to_f32(v.y), bf16hi_to_f32(v.y), b);
  a = fmaf(bf16lo_to_f32(v.z), bf16lo_to_f32(v.z), a);
  b = fmaf(bf16hi_to_f32(v.z), bf16hi_to_f32(v.z), b);
  a = fmaf(bf16lo_to_f32(v.w), bf16lo_to_f32(v.w), a);
  b = fmaf(bf16hi_to_f32(v.w), bf16hi_to_f32(v.w), b);
  return a + b;
}

__device__ __forceinline__ float dot_bf16x8(const float* acc, uint4 v) {
  float s = 0.f;
  s = fmaf(acc[0], bf16lo_to_f32(v.x), s);
  s = fmaf(acc[1], bf16hi_to_f32(v.x), s);
  s = fmaf(acc[2], bf16lo_to_f32(v.y), s);
  s = fmaf(acc[3], bf16hi_to_f32(v.y), s);
  s = fmaf(acc[4], bf16lo_to_f32(v.z), s);
  s = fmaf(acc[5], bf16hi_to_f32(v.z), s);
  s = fmaf(acc[6], bf16lo_to_f32(v.w), s);
  s = fmaf(acc[7], bf16hi_to_f32(v.w), s);
  return s;
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Waits (bounded) until *flag >= target, with acquire ordering.
__device__ __forceinline__ bool wait_counter_geq(const int* flag, int target,
                                                 uint64_t timeout_ns, const volatile int* abort) {
  const uint64_t t0 = global_timer_ns();
  while (true) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v >= target) return true;
    if (abort != nullptr && *abort) return false;
    if (global_timer_ns() - t0 > timeout_ns) return false;
    __nanosleep(64);
  }
}

// Orders this thread's generic-proxy accesses of global memory with its
// async-proxy (TMA) ones.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// The eight epilogue warps only (named barrier 1).
__device__ __forceinline__ void epi_bar_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");
}

// Walks one pair's segments of one phase of one wave: its range [x, end) of
// the wave's phase sequence, module by module, tile by tile.
template <bool kGrouped>
struct SegWalk {
  const NormProblemDev* single;
  const NormProblemDev* table;
  int m, m1, ph;
  long long x, end;
  // current segment: tile (pseudo-tile for the Gram), first unit in the tile, units
  const NormProblemDev* P;
  int tile, k0, n;
  long long xs;  // the segment's first unit in the wave's phase sequence

  __device__ __forceinline__ void start(const WaveInfo& w, int pairs, int pair, int phase) {
    ph = phase;
    m = w.m0;
    m1 = w.m1;
    x = sched_begin(w, pairs, ph, pair);
    end = sched_begin(w, pairs, ph, pair + 1);
  }
  // Moves to the segment starting at x; false when the range is done.
  __device__ __forceinline__ bool next() {
    if (x >= end) return false;
    if (kGrouped) {
      while (m + 1 < m1 && table[m + 1].begin[ph] <= x) ++m;
      P = &table[m];
    } else {
      P = single;
    }
    const int per = phase_per_tile(*P, ph);
    const long long local = x - P->begin[ph];
    tile = static_cast<int>(local / per);
    k0 = static_cast<int>(local % per);
    const long long left = end - x;
    n = static_cast<int>(left < per - k0 ? left : per - k0);
    xs = x;
    x += n;
    return true;
  }
};

// ---------------------------------------------------------------------------
// The fused kernel on CTA pairs
//
// A cluster of two CTAs owns a 256-row tile at a time: rank c stages rows
// [128 c, 128 c + 128) of the tile's A operand (W0, B, or A itself for the
// Gram) and half of the N-side slab (rows [c h0, c h0 + h0) of each
// accumulator chunk), and rank 0 issues one M = 256 MMA per 16-element K
// step and chunk for both.  Each CTA thus stages 16 KB of W0 and only half of
// the 64-column slab per k-block (24 KB at r = 384), so five stages fit in
// shared memory and the slab is fetched from L2 once per 256 rows.
//
// Barriers (per CTA, same offsets in both):
//   full[s]      rank 0 only: its producer's expected bytes plus the copies of
//                both CTAs (the peer's copies signal rank 0's barrier).
//   mma_done[s]  both: rank 0's commit after the MMAs reading stage s, sent to
//                both CTAs; the reduction warps then read the W0 rows
//                (||W0_i||^2) and release the stage.
//   empty[s]     both: one arrival per reduction warp; the producer refills.
//   acc_full     both: rank 0's commit at the end of a segment.
//   acc_empty    rank 0 only: one arrival per epilogue warp of both CTAs.
// ---------------------------------------------------------------------------
struct NormSmemTail {
  uint64_t full[kMaxStages];
  uint64_t mma_done[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t drain;
  uint64_t half_ready;         // upper epilogue half has posted its partial
  float half_part[2][kTileM];  // double-buffered by segment parity
  uint32_t tmem_slot;
  int abort_flag;
  int gram_ok;                 // every Gram segment of the pseudo-tile has posted
};

// Sets this CTA's and the peer's abort flags and records the timeout.
__device__ __forceinline__ void give_up_pair(volatile int* abort_flag, uint32_t peer_flag) {
  *abort_flag = 1;
  st_cluster_u32(peer_flag, 1u);
  record_error(DORA_ERR_TIMEOUT);
}

template <bool kGrouped>
__global__ void __cluster_dims__(2, 1, 1) __maxnreg__(kNormMaxRegs)
    norm_main_kernel(const __grid_constant__ NormProblemDev single,
                     const NormProblemDev* __restrict__ table,
                     const __grid_constant__ NormSched sched, int stages, uint32_t b_region,
                     uint32_t tmem_cols, float eps, unsigned long long timeout_ns,
                     unsigned long long* __restrict__ trace) {
  // trace (optional, diagnostics): per CTA kTraceWords words -- entry and
  // exit global time, MMA-issuer cycles waiting for data / for the
  // accumulator, issued k-blocks, segments, SM id, cycles waited for data
  // over the first four k-blocks; then global times: the MMA issuer starting
  // its W0 and its G units, and (first Gram segment) the epilogue holding the
  // accumulator, its partial posted, all partials posted, its rows of G'
  // written.
  const uint64_t t_entry = trace != nullptr ? global_timer_ns() : 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t stage_bytes = kTileABytes + b_region;
  NormSmemTail* tail = reinterpret_cast<NormSmemTail*>(smem + stages * stage_bytes);
  uint64_t* full = tail->full;
  uint64_t* mma_done = tail->mma_done;
  uint64_t* empty = tail->empty;
  volatile int* abort_flag = &tail->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pairs = sched.pairs;
  const int pair = blockIdx.x >> 1;
  const uint32_t peer_abort = mapa_shared(smem_addr(&tail->abort_flag), rank ^ 1u);

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&mma_done[s], 1);
      mbar_init(&empty[s], kEpiWarps);
    }
    mbar_init(&tail->acc_full, 1);
    mbar_init(&tail->acc_empty, 2 * kEpiWarps);
    mbar_init(&tail->drain, 1);
    mbar_init(&tail->half_ready, kTileM);
    tail->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(&tail->tmem_slot, tmem_cols);
    tmem_relinquish_pair();
  }
  if (!kGrouped && warp == kEpiWarps && lane == 0) {
    prefetch_tmap(&single.tm_w0);
    prefetch_tmap(&single.tm_arow);
    prefetch_tmap(&single.tm_a);
    prefetch_tmap(&single.tm_b);
    prefetch_tmap(&single.tm_g);
    prefetch_tmap(&single.tm_glo);
  }
  // Both CTAs' barriers are initialised (and their TMEM allocated) before
  // either CTA signals the other.
  tc_fence_before_sync();
  cluster_sync();
  tc_fence_after_sync();
  const uint32_t tmem_base = tail->tmem_slot;

  SegWalk<kGrouped> sw;
  sw.single = &single;
  sw.table = table;

  if (warp == kEpiWarps) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_last();
      const uint32_t full0 = mapa_shared(smem_addr(&full[0]), 0);  // rank 0's full[0]
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool dep_waited = false;
      const NormProblemDev* ready = nullptr;  // module whose G' is known to be written
      bool ok = true;
      for (int wv = 0; ok && wv < sched.waves; ++wv) {
        for (int ph = kPhaseGram; ok && ph <= kPhaseG; ++ph) {
          sw.start(sched.w[wv], pairs, pair, ph);
          while (ok && sw.next()) {
            const NormProblemDev* P = sw.P;
            if (ph == kPhaseG && P != ready) {
              // G' of this module is written by the pairs that reduce its
              // Gram; the count they raise was zeroed by the preceding kernel.
              if (!dep_waited) {
                grid_dependency_wait();
                grid_dependency_trigger();
                dep_waited = true;
              }
              if (!wait_counter_geq(P->g_ready, kPairM * P->pg_tiles, timeout_ns, abort_flag)) {
                give_up_pair(abort_flag, peer_abort);
                ok = false;
                break;
              }
              fence_proxy_async_global();
              ready = P;
            }
            const int row0 = sw.tile * kPairM + static_cast<int>(rank) * kTileM;
            for (int k = sw.k0; k < sw.k0 + sw.n; ++k) {
              if (!mbar_wait(&empty[stage], phase ^ 1u, timeout_ns, abort_flag)) {
                give_up_pair(abort_flag, peer_abort);
                ok = false;
                break;
              }
              uint8_t* sa = smem + stage * stage_bytes;
              uint8_t* sb = sa + kTileABytes;
              const uint32_t bar = full0 + stage * static_cast<uint32_t>(sizeof(uint64_t));
              if (rank == 0) mbar_arrive_expect_tx(&full[stage], P->pair_tx);
              const CUtensorMap* slab;
              int kx;
              if (ph == kPhaseG) {
                const bool lo = k >= P->kb_r;
                kx = (k - (lo ? P->kb_r : 0)) * kBlockK;
                tma_load_2d_pair(sa, &P->tm_b, bar, kx, row0, pol_keep);
                slab = lo ? &P->tm_glo : &P->tm_g;
              } else {
                kx = k * kBlockK;
                if (ph == kPhaseW0)
                  tma_load_2d_pair(sa, &P->tm_w0, bar, kx, row0, pol_stream);
                else
                  tma_load_2d_pair(sa, &P->tm_arow, bar, kx, row0, pol_keep);
                slab = &P->tm_a;
              }
              if (P->slab4d) {
                tma_load_4d_pair(sb, slab, bar, kx, 0, static_cast<int>(rank), 0, pol_keep);
              } else {
                tma_load_2d_pair(sb, slab, bar, kx, static_cast<int>(rank) * P->h0, pol_keep);
                if (P->n1 > 0)
                  tma_load_2d_pair(sb + P->h0 * 128, slab, bar, kx,
                                   P->n0 + static_cast<int>(rank) * P->h0, pol_keep);
              }
              ++issued;
              if (++stage == stages) {
                stage = 0;
                phase ^= 1u;
              }
            }
          }
        }
      }
      if (!dep_waited) {
        grid_dependency_wait();
        grid_dependency_trigger();
      }
      // Let every copy already issued land before the block can exit: rank 0
      // sees its full barriers complete; rank 1's copies complete on rank 0's
      // barriers, so it waits for its stages to be consumed (bounded: after
      // a give-up this only waits out the drain limit, by which time the
      // copies have long landed).
      const long long first = issued > stages ? issued - stages : 0;
      for (long long j = first; j < issued; ++j) {
        const uint32_t par = static_cast<uint32_t>((j / stages) & 1);
        if (rank == 0)
          mbar_wait(&full[j % stages], par, kDrainTimeoutNs, nullptr);
        else
          mbar_wait(&empty[j % stages], par, kDrainTimeoutNs, nullptr);
      }
    }
  } else if (warp == kEpiWarps + 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && rank == 0) {
      const bool tracing = trace != nullptr;
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool issued_any = false;
      long long wait_data = 0, wait_first = 0, wait_acc = 0, nseg = 0, nkb = 0;
      bool ok = true;
      for (int wv = 0; ok && wv < sched.waves; ++wv) {
        for (int ph = kPhaseGram; ok && ph <= kPhaseG; ++ph) {
          sw.start(sched.w[wv], pairs, pair, ph);
          if (tracing && wv == 0 && ph > kPhaseGram)
            trace[static_cast<size_t>(blockIdx.x) * kTraceWords + 7 + ph] = global_timer_ns();
          while (ok && sw.next()) {
            const NormProblemDev* P = sw.P;
            const long long c0 = tracing ? clock64() : 0;
            if (!mbar_wait(&tail->acc_empty, acc_phase ^ 1u, timeout_ns, abort_flag)) {
              give_up_pair(abort_flag, peer_abort);
              ok = false;
              break;
            }
            if (tracing) wait_acc += clock64() - c0;
            ++nseg;
            tc_fence_after_sync();
            const uint32_t idesc0 = P->idesc0, idesc1 = P->idesc1;
            const int n0 = P->n0, n1 = P->n1;
            const uint32_t b1_off = static_cast<uint32_t>(P->h0) * 128u;
            for (int i = 0; i < sw.n; ++i) {
              // The stage's copies completed on this barrier; the MMAs that
              // read it are issued straight after the wait.
              const long long c1 = tracing ? clock64() : 0;
              if (!mbar_wait(&full[stage], phase, timeout_ns, abort_flag)) {
                give_up_pair(abort_flag, peer_abort);
                ok = false;
                break;
              }
              if (tracing) {
                wait_data += clock64() - c1;
                if (nkb < 4) wait_first = wait_data;
              }
              ++nkb;
              const uint32_t a0 = smem_addr(smem + stage * stage_bytes);
              const uint32_t b0 = a0 + kTileABytes;
              // Two accumulator chains (chunks) when r > 256, interleaved per
              // K step; the chunk test stays outside the issue loops.
              if (n1 > 0) {
#pragma unroll
                for (int k = 0; k < kBlockK / 16; ++k) {
                  const uint64_t ad = sw128_kmajor_desc(a0 + k * 32);
                  const uint32_t acc = (i == 0 && k == 0) ? 0u : 1u;
                  umma_bf16_pair(tmem_base, ad, sw128_kmajor_desc(b0 + k * 32), idesc0, acc);
                  umma_bf16_pair(tmem_base + n0, ad, sw128_kmajor_desc(b0 + b1_off + k * 32),
                                 idesc1, acc);
                }
              } else {
#pragma unroll
                for (int k = 0; k < kBlockK / 16; ++k)
                  umma_bf16_pair(tmem_base, sw128_kmajor_desc(a0 + k * 32),
                                 sw128_kmajor_desc(b0 + k * 32), idesc0,
                                 (i == 0 && k == 0) ? 0u : 1u);
              }
              issued_any = true;
              umma_commit_pair(&mma_done[stage], 0x3);
              if (++stage == stages) {
                stage = 0;
                phase ^= 1u;
              }
            }
            if (!ok) break;
            umma_commit_pair(&tail->acc_full, 0x3);
            acc_phase ^= 1u;
          }
        }
      }
      if (issued_any) {
        umma_commit_pair(&tail->drain, 0x1);
        mbar_wait(&tail->drain, 0, kDrainTimeoutNs, nullptr);
      }
      if (trace != nullptr) {
        unsigned long long* tr = trace + static_cast<size_t>(blockIdx.x) * kTraceWords;
        tr[2] = static_cast<unsigned long long>(wait_data);
        tr[3] = static_cast<unsigned long long>(wait_acc);
        tr[4] = static_cast<unsigned long long>(nkb);
        tr[5] = static_cast<unsigned long long>(nseg);
        tr[7] = static_cast<unsigned long long>(wait_first);
      }
    }
  } else {
    // ------------------------------------ ||W0_i||^2 + epilogue (warps 0-7)
    // Thread (half h, row): TMEM lane `row`; half h of the row's 16-byte chunks
    // of each W0 stage and half h of the accumulator's 32-column chunks.
    const int half = warp / 4;
    const int row = threadIdx.x & (kTileM - 1);
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t acc_empty0 = mapa_shared(smem_addr(&tail->acc_empty), 0);
    int stage = 0;
    uint32_t phase = 0, acc_phase = 0, seg_count = 0;
    bool dep_waited = false;
    bool ok = true;
    for (int wv = 0; ok && wv < sched.waves; ++wv) {
      const WaveInfo& W = sched.w[wv];
      for (int ph = kPhaseGram; ok && ph <= kPhaseG; ++ph) {
        sw.start(W, pairs, pair, ph);
        while (ok && sw.next()) {
          const NormProblemDev* P = sw.P;
          const int t = sw.tile;
          const int r = P->r;
          // the row of W0 (or, for the Gram, of A) this thread finishes
          const int grow = t * kPairM + static_cast<int>(rank) * kTileM + row;
          const bool valid = grow < (ph == kPhaseGram ? r : P->d_out);
          // this half's 32-column chunks of the accumulator
          const int nchunks = (P->n0 + P->n1 + 31) / 32;
          const int c_lo = half == 0 ? 0 : (nchunks + 1) / 2;
          const int c_hi = half == 0 ? (nchunks + 1) / 2 : nchunks;
          // Prefetch B_i for (up to kPrefetchChunks of) those columns while
          // the MMAs of this segment run.
          const bool dotted = ph != kPhaseGram;
          const uint16_t* brow = P->B + static_cast<size_t>(dotted && valid ? grow : 0) * r;
          uint4 bq[kPrefetchChunks][4];
#pragma unroll
          for (int c = 0; c < kPrefetchChunks; ++c)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int col = (c_lo + c) * 32 + q * 8;
              bq[c][q] = (dotted && valid && c_lo + c < c_hi && col < r)
                             ? __ldg(reinterpret_cast<const uint4*>(brow + col))
                             : make_uint4(0u, 0u, 0u, 0u);
            }
          // Where this segment's partial goes among the tile's segments
          // (the Gram and G sequences are split evenly over their pairs; the
          // W0 segments of each tile come from consecutive pairs, found by
          // the preceding kernel).
          int ord = 0, nseg = 0;
          if (ph == kPhaseGram) {
            const long long x0 = P->begin[kPhaseGram] + static_cast<long long>(t) * P->kb_w;
            nseg = even_segments(x0, x0 + P->kb_w, sw.xs, W.n[kPhaseGram], W.J, pair, &ord);
          } else {
            const long long xg = P->begin[kPhaseG] + static_cast<long long>(t) * 2 * P->kb_r;
            int ord_g = 0;
            const int ng = even_segments(xg, xg + 2 * P->kb_r, sw.xs, W.n[kPhaseG], pairs, pair,
                                         &ord_g);
            nseg = ng;  // the W0 count and this pair's W0 slot follow once the table is visible
            ord = ord_g;
          }
          float ss = 0.f;
          for (int i = 0; i < sw.n; ++i) {
            // The MMAs that read this stage have completed, so its copies
            // (completed on rank 0's barrier) have landed here too.
            if (!mbar_wait(&mma_done[stage], phase, timeout_ns, abort_flag)) {
              give_up_pair(abort_flag, peer_abort);
              ok = false;
              break;
            }
            if (ph == kPhaseW0) {
              const uint8_t* rowp = smem + stage * stage_bytes + row * 128;
              float part = 0.f;
#pragma unroll
              for (int q = 0; q < 4; ++q)
                part += sumsq_bf16x8(
                    *reinterpret_cast<const uint4*>(rowp + (((half * 4 + q) ^ (row & 7)) << 4)));
              ss += part;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (++stage == stages) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          if (!mbar_wait(&tail->acc_full, acc_phase, timeout_ns, abort_flag)) {
            give_up_pair(abort_flag, peer_abort);
            ok = false;
            break;
          }
          tc_fence_after_sync();
          acc_phase ^= 1u;
          if (!dep_waited) {  // counters and the tile table come from the preceding kernel
            grid_dependency_wait();
            dep_waited = true;
          }
          if (ph != kPhaseGram) {
            const int tw = __ldcg(P->tile_w + t);
            const int nw = tw >> 16;
            if (ph == kPhaseW0) {
              ord = pair - (tw & 0xffff);
              nseg += nw;
            } else {
              ord += nw;
              nseg += nw;
            }
          }

          const bool gtrace = trace != nullptr && threadIdx.x == 0 && ph == kPhaseGram &&
                              trace[static_cast<size_t>(blockIdx.x) * kTraceWords + 10] == 0;
          if (gtrace) trace[static_cast<size_t>(blockIdx.x) * kTraceWords + 10] = global_timer_ns();
          if (ph == kPhaseGram) {
            // ---- Gram segment: post the raw accumulator (this CTA's 128
            // rows of G, all n_pad columns) as partial `ord`, column-major,
            // so that each store of a warp covers 32 consecutive rows.
            const int n_pad = P->n_pad;
            const size_t slot = static_cast<size_t>(n_pad) * kPairM;
            float* gbase = P->gram_part + static_cast<size_t>(t) * P->gram_slots * slot +
                           static_cast<int>(rank) * kTileM;
            float* gp = gbase + static_cast<size_t>(ord) * slot + row;
#pragma unroll 1
            for (int c = c_lo; c < c_hi; ++c) {
              float acc[32];
              tmem_load_32cols(tmem_base + lane_base + c * 32, acc);
#pragma unroll
              for (int q = 0; q < 32; ++q)
                if (c * 32 + q < n_pad) __stcg(gp + static_cast<size_t>(c * 32 + q) * kPairM, acc[q]);
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty0);
            // Once every segment of this pseudo-tile has posted (per CTA
            // half: the segments end together, since the Gram pairs start
            // at once), each sums a share of the rows over all partials in
            // slot order and writes those rows of G'_hi and G'_lo.
            __threadfence();
            epi_bar_sync();
            int* cnt = P->gram_cnt + t * 2 + static_cast<int>(rank);
            if (threadIdx.x == 0) {
              if (gtrace) trace[static_cast<size_t>(blockIdx.x) * kTraceWords + 11] = global_timer_ns();
              atomicAdd(cnt, 1);
              tail->gram_ok = wait_counter_geq(cnt, nseg, timeout_ns, abort_flag) ? 1 : 0;
              if (gtrace) trace[static_cast<size_t>(blockIdx.x) * kTraceWords + 12] = global_timer_ns();
            }
            epi_bar_sync();
            if (!tail->gram_ok) {
              give_up_pair(abort_flag, peer_abort);
              ok = false;
              break;
            }
            __threadfence();
            // This segment's share: rows [rb, re) of the CTA half, every
            // column.  Lanes take consecutive rows (32 at a time) and warps
            // interleaved columns, so every load and store of a warp covers
            // consecutive addresses; kU columns of every partial are in
            // flight per thread.
            const int rb = ord * kTileM / nseg, re = (ord + 1) * kTileM / nseg;
            constexpr int kU = 12;
            constexpr int kCs = kEpiWarps;  // column stride between a warp's columns
#pragma unroll 1
            for (int r0 = rb; r0 < re; r0 += 32) {
              const int rr = r0 + lane;
              const bool rv = rr < re;
              const int gr = t * kPairM + static_cast<int>(rank) * kTileM + rr;
              const float* src = gbase + rr;
#pragma unroll 1
              for (int c0 = warp; c0 < n_pad; c0 += kCs * kU) {
                float sum[kU];
#pragma unroll
                for (int u = 0; u < kU; ++u) sum[u] = 0.f;
#pragma unroll 1
                for (int o = 0; o < nseg; ++o) {
                  const float* so = src + static_cast<size_t>(o) * slot;
                  float v[kU];
#pragma unroll
                  for (int u = 0; u < kU; ++u) {
                    const int c = c0 + u * kCs;
                    v[u] = (rv && c < n_pad) ? __ldcg(so + static_cast<size_t>(c) * kPairM) : 0.f;
                  }
#pragma unroll
                  for (int u = 0; u < kU; ++u) sum[u] += v[u];
                }
                if (rv && gr < r) {
#pragma unroll
                  for (int u = 0; u < kU; ++u) {
                    const int c = c0 + u * kCs;
                    if (c >= r) break;
                    const float x = P->half_s * sum[u];
                    const uint16_t hi = f32_to_bf16_rn(x);
                    const uint16_t lo =
                        f32_to_bf16_rn(x - __uint_as_float(static_cast<uint32_t>(hi) << 16));
                    P->g_hi[static_cast<size_t>(c) * P->r8 + gr] = hi;
                    P->g_lo[static_cast<size_t>(c) * P->r8 + gr] = lo;
                  }
                }
              }
            }
            // Publish these rows of G' to the TMA reads of every pair's G units.
            __threadfence();
            fence_proxy_async_global();
            epi_bar_sync();
            if (threadIdx.x == 0) atomicAdd(P->g_ready, re - rb);
            if (gtrace) trace[static_cast<size_t>(blockIdx.x) * kTraceWords + 13] = global_timer_ns();
            continue;
          }

          // ---- W0 / G segment: dot each row's accumulator with B_i.
          float dot = 0.f;
#pragma unroll
          for (int c = 0; c < kMaxChunksPerHalf; ++c) {
            if (c_lo + c < c_hi) {  // warp-uniform
              float acc[32];
              tmem_load_32cols(tmem_base + lane_base + (c_lo + c) * 32, acc);
              if (c < kPrefetchChunks) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                  dot += dot_bf16x8(acc + q * 8, bq[c < kPrefetchChunks ? c : 0][q]);
              } else {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  const int col = (c_lo + c) * 32 + q * 8;
                  if (valid && col < r)
                    dot += dot_bf16x8(acc + q * 8,
                                      __ldg(reinterpret_cast<const uint4*>(brow + col)));
                }
              }
            }
          }
          tc_fence_before_sync();
          // Combine the two halves of the row in a fixed order (lower +
          // upper).  The lower half takes the upper half's value before it
          // releases the accumulator, so the next segment cannot overwrite it
          // early.
          const float part = fmaf(P->two_s, dot, ss);
          const int buf = seg_count & 1;
          if (half == 1) {
            tail->half_part[buf][row] = part;
            mbar_arrive(&tail->half_ready);
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty0);
          } else {
            const bool got_one =
                mbar_wait(&tail->half_ready, seg_count & 1u, timeout_ns, abort_flag);
            const float other = tail->half_part[buf][row];
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty0);
            if (!__all_sync(0xffffffffu, got_one)) {
              give_up_pair(abort_flag, peer_abort);
              ok = false;
              break;
            }
            float* part_t = P->partial + static_cast<size_t>(t) * P->seg_slots * kPairM +
                            static_cast<int>(rank) * kTileM + row;
            if (valid) part_t[static_cast<size_t>(ord) * kPairM] = part + other;
            // The last of the tile's segments to post its partials (per warp:
            // 32 rows) sums every slot in slot order and writes n and g.
            __threadfence();
            __syncwarp();
            int prev = 0;
            if (lane == 0)
              prev = atomicAdd(P->tile_cnt + (t * 2 + static_cast<int>(rank)) * 4 + warp, 1);
            prev = __shfl_sync(0xffffffffu, prev, 0);
            if (prev == nseg - 1) {
              __threadfence();
              if (valid) {
                float sum = 0.f;
                for (int c = 0; c < nseg; ++c)
                  sum += __ldcg(part_t + static_cast<size_t>(c) * kPairM);
                if (P->emit_sq) {
                  P->n_out[grow] = sum;
                } else {
                  const float n = __fsqrt_rn(fmaxf(sum, 0.f));
                  P->n_out[grow] = n;
                  if (P->m != nullptr && P->g_out != nullptr)
                    P->g_out[grow] = __fdiv_rn(__ldg(P->m + grow), fmaxf(n, eps));
                }
              }
            }
          }
          ++seg_count;
        }
      }
    }
  }

  // Neither CTA leaves (or frees TMEM) while the other may still signal it,
  // read its shared memory through the MMAs, or write its TMEM.
  __syncwarp();
  tc_fence_before_sync();
  cluster_sync();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem_base, tmem_cols);
  }
  if (trace != nullptr && threadIdx.x == 0) {
    unsigned long long* tr = trace + static_cast<size_t>(blockIdx.x) * kTraceWords;
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    tr[0] = t_entry;
    tr[1] = global_timer_ns();
    tr[6] = smid;
  }
}

// Before the fused kernel, once the preceding kernel has finished: zeroes
// its counters (every module's counters form one block of ints) and writes
// each tile's W0 segment table (first pair, number of pairs: the W0 ranges
// are not an even split, so this takes a search per tile), then lets the
// fused kernel launch; it waits for this grid before it reads either.
template <bool kGrouped>
__global__ void __launch_bounds__(256)
    norm_prep_kernel(int* __restrict__ cnt, int n_cnt, const __grid_constant__ NormProblemDev single,
                     const NormProblemDev* __restrict__ table, int count,
                     const __grid_constant__ NormSched sched) {
  grid_dependency_wait();
  grid_dependency_trigger();
  const int stride = gridDim.x * blockDim.x;
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  for (int i = tid; i < n_cnt; i += stride) cnt[i] = 0;
  for (int w = 0; w < sched.waves; ++w) {
    const WaveInfo& W = sched.w[w];
    for (int m = W.m0; m < W.m1; ++m) {
      const NormProblemDev* P = kGrouped ? &table[m] : &single;
      for (int t = tid; t < P->tiles; t += stride) {
        const long long x0 = P->begin[kPhaseW0] + static_cast<long long>(t) * P->kb_w;
        const int f = sched_pair_of(W, sched.pairs, kPhaseW0, x0);
        const int l = sched_pair_of(W, sched.pairs, kPhaseW0, x0 + P->kb_w - 1);
        P->tile_w[t] = f | ((l - f + 1) << 16);
      }
    }
  }
  (void)count;
}

}  // namespace dora
