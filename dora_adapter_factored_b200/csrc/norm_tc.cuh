// Factored DoRA row norm on the 5th-generation tensor cores (tcgen05 + TMEM,
// operands staged by TMA), following "Scaling DoRA: High-Rank Adaptation via
// Factored Norms and Fused Kernels", section 2: the squared norm of row i of
// W0 + s B A is ||W0_i||^2 + 2 s B_i.(W0 A^T)_i + s^2 B_i G B_i^T, G = A A^T,
// evaluated from [d_out, r] and [r, r] intermediates only.
//
// One persistent kernel on CTA pairs (after a tiny kernel that zeroes its
// counters) does the whole norm of one module, or of many (the grouped call):
//
//   Gram jobs    one block of G = A A^T each: 256 rows of A (a pseudo-tile)
//                against nc (<= 256) rows of A, over one of the gkp equal
//                parts of d_in.  A few pairs take one job each first; the
//                job scales its sum by s/2 and writes it as part p of S, in
//                two bf16 matrices S_hi = bf16(S_p) and S_lo = bf16(S_p -
//                S_hi), so that the Gram term keeps fp32-level accuracy (the
//                pages' norm accumulates in fp32 whatever the weight dtype).
//                Since G is symmetric, only one triangle is computed and
//                stored: S_p = G'_p on the diagonal, 2 G'_p below it and 0
//                above it (row gr, column c: c < gr), for which
//                B_i (sum_p S_p) B_i^T = B_i G' B_i^T, G' = (s/2) G.  The parts
//                are never added up: the G units sum them in their
//                accumulator, so no job waits for another.
//   W0 units     per 256-row tile of W0, k-blocks over d_in: TMEM
//                accumulator += W0_tile A^T, while the reduction warps square
//                and sum the same W0 tile straight from shared memory
//                (||W0_i||^2), so W0 crosses HBM exactly once.
//   G units      per tile, k-blocks over r, for every part p:
//                accumulator += B_tile S_hi,p^T, then B_tile S_lo,p^T; they wait
//                until every part of the module's S is written.
//
// A segment (one pair's run of units on one tile) ends with an epilogue that
// drains TMEM and dots each row with B_i; the per-row value
// ||W0_i||^2_part + 2 s B_i.acc_i is handed to a finisher warp, which posts it
// as the segment's partial: every term is linear in a k-range, so the
// partials of all segments of a tile simply add (B_i.acc_i over G units is
// (s/2) B_i G B_i^T).  The finisher of the segment that posts a tile's
// partials last (an arrival counter per CTA half of the tile) sums them in
// slot order and finalises those rows: n_i = sqrt(max(sum, 0)) and
// g_i = m_i / max(n_i, eps) (section 4, precision bullet).  Global round
// trips thus never hold up the warps that release pipeline stages.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace dora {

constexpr int kTileM = 128;                  // W0 rows per CTA = TMEM lanes
constexpr int kPairM = 2 * kTileM;           // W0 rows per tile of a CTA pair
constexpr int kBlockK = 64;                  // bf16 of K per stage: one 128-byte swizzle row
constexpr int kMaxStages = 8;
constexpr int kEpiWarps = 8;                 // warps 0-7: reduction + epilogue
constexpr int kProducerWarp = kEpiWarps;     // warp 8: TMA producer
constexpr int kMmaWarp = kEpiWarps + 1;      // warps 9, 10: MMA issuers, one per accumulator chunk
constexpr int kFinisherWarp = kEpiWarps + 3; // warp 11: posts partials, finalises rows
constexpr int kNormThreads = (kEpiWarps + 4) * 32;
constexpr int kMaxChunksPerHalf = 8;         // 32-column TMEM chunks per epilogue half (r <= 512)
constexpr int kPrefetchChunks = 6;           // of which B is prefetched into registers (r <= 384)
constexpr int kPartBufs = 4;                 // epilogue -> finisher hand-over buffers
constexpr int kFinBatch = 8;                 // partial slots loaded together when finalising
// k-blocks per W0 chunk of the pool (at most): a pool item costs a segment
// boundary (accumulator drain, operand refill), so chunks are large; on the
// 56-module stack 64 gave ~1530 us against ~1630 us with 16.
constexpr int kChunkKb = 64;
constexpr int kItemRing = 8;                 // pool items in flight between the roles of a pair
// Roles that read each pool item: rank 0's two MMA issuers, eight epilogue
// warps and finisher; rank 1's producer, eight epilogue warps and finisher.
constexpr int kItemConsumers = 2 + kEpiWarps + 1 + 1 + kEpiWarps + 1;
constexpr int kGramCols = 128;               // columns of G per Gram job (at most)
// 12 warps: 65536 / 384 threads = 170 -> 168 registers per thread.
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
  CUtensorMap tm_arow;   // A  [r, d_in],     box 64 x 128: the Gram jobs' A operand
  CUtensorMap tm_agram;  // A  [r, d_in],     box 64 x gh: the Gram jobs' N-side slab
  CUtensorMap tm_a;      // A  as the N-side slab: box 64 x h0, or the 4-D view
                         //    {64, h0, 2 ranks, 2 chunks} with box {64, h0, 1, 2}
  CUtensorMap tm_b;      // B  [d_out, r],    box 64 x 128
  CUtensorMap tm_g;      // S_hi [gkp][r][r8] as {r8, r, gkp} (or the 5-D pair view), box like tm_a
  CUtensorMap tm_glo;    // S_lo, like tm_g
  CUtensorMap tm_ghi_st; // S_hi as {r, r, gkp}, box 32 x 32 x 1, 64-byte swizzle: the Gram jobs' stores
  CUtensorMap tm_glo_st; // S_lo, like tm_ghi_st
  const uint16_t* B;     // bf16 bits of B, for the epilogue dot
  uint16_t* g_hi;        // [gkp][r][r8] bf16 bits of S_hi: S_p[gr][c] = 2 G'_p (c < gr), G'_p (c = gr), 0
  uint16_t* g_lo;        // [gkp][r][r8] bf16 bits of S_lo = bf16(S_p - S_hi)
  float* partial;        // [tiles][seg_slots][256] per-row partials
  int* tile_cnt;         // [tiles * 2] segments posted per CTA half of each tile
  int* g_ready;          // [1] epilogue warps of Gram jobs whose rows of S are written
  int* tile_w;           // [tiles] first pair | (pairs << 16) of each tile's W0 units
  const float* m;        // [d_out] or null
  float* n_out;          // [d_out]
  float* g_out;          // [d_out] or null
  long long begin[3];    // first job (Gram) / static W0 unit of this module in its wave
  long long dyn_begin;   // first W0-chunk item of this module in its wave's pool
  long long g_item_begin;  // first G item of this module among the wave's G items
  int dyn_t0;            // tiles [0, dyn_t0) are scheduled statically, the rest chunk by chunk
  int cpt;               // W0 chunks per pool tile
  int gpi, gipt;         // parts of S per G item, G items per tile
  int d_out, r, r8, n_pad;
  int n0, n1;            // N of the two pair-MMA chunks (n1 = 0: single chunk; else n1 = n0)
  int h0;                // slab rows of each chunk that one CTA stages: n0 / 2
  int slab4d;            // tm_a / tm_g / tm_glo are the 4-D view: one box per slab half
  int emit_sq;           // write the squared-norm sum itself to n_out (no clamp, sqrt or g)
  int kb_w, kb_r, tiles, pg_tiles, seg_slots;
  int nc;                // columns of G per Gram block: gchunks MMA chunks of gn
  int gchunks, gn, gh;   // each CTA stages gh = gn / 2 slab rows per chunk
  int gj0, gblocks;      // Gram blocks of pseudo-tile 0, of the module
  int gkp;               // parts of d_in (one job per block and part)
  uint32_t pair_tx;      // bytes landing per W0 / G stage in both CTAs together
  uint32_t gram_tx;      // bytes landing per Gram stage in both CTAs together
  uint32_t idesc0, idesc1, idesc_gram;
  float two_s, half_s;
};

// Units of phase `ph` per tile (per job for the Gram).
__host__ __device__ __forceinline__ int phase_per_tile(const NormProblemDev& P, int ph) {
  return ph == kPhaseG ? 2 * P.kb_r * P.gkp : P.kb_w;
}

// Gram jobs of pseudo-tile t of a module of rank r (nc columns each): the
// column blocks that reach the lower triangle, c <= row < min(r, 256 (t + 1)).
__host__ __device__ __forceinline__ int gram_jobs_of_tile(int r, int nc, int t) {
  const int rows_end = r < kPairM * (t + 1) ? r : kPairM * (t + 1);
  return (rows_end + nc - 1) / nc;
}

// ---------------------------------------------------------------------------
// Schedule.  The grouped call splits its modules (in order) into waves whose
// re-read operands (A, S) fit in L2 together; one module alone is one wave.
// Within a wave:
//   Gram: pairs j < J share the n[0] jobs evenly by count (a job is never
//         split), first;
//   W0:   the other pairs share the n[1] static W0 units (the wave's first
//         tiles) evenly;
//   pool: then every pair takes items from the wave's pool until it is
//         empty: the W0 units of the remaining tiles in chunks, then one item
//         per tile and part of S with its G units (which need S, written by
//         then),
// so the Gram is done early by a few pairs, and the pool evens out whatever
// the static split did not (the Gram pairs' work, segment overheads, slower
// pairs).  The static boundaries are closed forms of j.
// ---------------------------------------------------------------------------
constexpr int kMaxWaves = 64;
constexpr int kMaxGramRuns = 8;
struct WaveInfo {
  long long n[3];  // Gram jobs, static W0 units and (static) G units of the wave
  long long dyn_w0_items, dyn_items;  // pool: W0 chunks, then G items (gipt per tile)
  long long gw;    // cost of all the wave's Gram jobs, in W0 units
  int J;           // pairs that share the Gram jobs
  int m0, m1;      // modules [m0, m1) of the table
  int runs;                      // runs of consecutive jobs of equal cost
  int run_end[kMaxGramRuns];     // first job after each run
  int run_cost[kMaxGramRuns];    // cost of one job of the run, in W0 units
};
struct NormSched {
  int waves;
  int pairs;
  WaveInfo w[kMaxWaves];
};

// Cost, in W0 units, of the wave's first x Gram jobs.
__host__ __device__ __forceinline__ long long gram_cost_prefix(const WaveInfo& w, long long x) {
  long long c = 0, start = 0;
  for (int i = 0; i < w.runs && start < x; ++i) {
    const long long e = w.run_end[i];
    c += ((x < e ? x : e) - start) * w.run_cost[i];
    start = e;
  }
  return c;
}

// First unit (Gram: job) of pair j's static range of phase `ph` (j = pairs
// gives the total).  The Gram pairs j < J share the Gram jobs and take no
// static W0 units (they go on to the pool); the other pairs share the static
// W0 units evenly.  There are no static G units.
__host__ __device__ __forceinline__ long long sched_begin(const WaveInfo& w, int pairs, int ph,
                                                          int j) {
  const long long jj = j;
  if (ph == kPhaseGram) {
    const long long jg = jj < w.J ? jj : w.J;
    return w.J > 0 ? jg * w.n[0] / w.J : 0;
  }
  if (ph == kPhaseG) return 0;
  const long long q = pairs - w.J;
  if (q <= 0 || jj <= w.J) return 0;
  return (jj - w.J) * w.n[1] / q;
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

// The segments of units [x0, x1) of phase `ph` (W0 or G), in order: returns
// how many there are and sets *ord to the position of pair `me`'s segment.
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

// Splits two fp32 values into bf16 hi (round to nearest even) and bf16 lo
// (the residual, rounded the same way), each pair packed low half first.
__device__ __forceinline__ void split_bf16_hi_lo(float x0, float x1, uint32_t* hi, uint32_t* lo) {
  const uint32_t h = pack_bf16x2_rn(x0, x1);
  *hi = h;
  *lo = pack_bf16x2_rn(x0 - __uint_as_float(h << 16), x1 - __uint_as_float(h & 0xffff0000u));
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

// Atomic add with release semantics at GPU scope (no result).
__device__ __forceinline__ void red_add_release_gpu(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Atomic add with acquire-release semantics at GPU scope; returns the old value.
__device__ __forceinline__ int atom_add_acq_rel_gpu(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v)
               : "memory");
  return old;
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
// the wave's phase sequence, module by module, tile by tile (Gram: job by
// job).
template <bool kGrouped>
struct SegWalk {
  const NormProblemDev* single;
  const NormProblemDev* table;
  int m, m1, ph;
  long long x, end;
  // current segment: tile (pseudo-tile for the Gram), Gram block, its
  // column block and K part, first unit in the tile, units
  const NormProblemDev* P;
  int tile, blk, cb, kpart, k0, n;
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
    const long long local = x - P->begin[ph];
    xs = x;
    if (ph == kPhaseGram) {
      const int q = static_cast<int>(local);
      const int kp = P->gkp;
      blk = q / kp;
      kpart = q - blk * kp;
      tile = blk < P->gj0 ? 0 : 1;
      cb = blk - (tile ? P->gj0 : 0);
      k0 = kpart * P->kb_w / kp;
      n = (kpart + 1) * P->kb_w / kp - k0;
      x += 1;
      return true;
    }
    const int per = phase_per_tile(*P, ph);
    tile = static_cast<int>(local / per);
    cb = 0;
    k0 = static_cast<int>(local % per);
    const long long left = end - x;
    n = static_cast<int>(left < per - k0 ? left : per - k0);
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
//   mma_done[s]  both: rank 0's commits after the MMAs reading stage s, sent
//                to both CTAs; the reduction warps then read the W0 rows
//                (||W0_i||^2) and release the stage.
//   empty[s]     both: one arrival per reduction warp; the producer refills.
//   acc_full     both: rank 0's commits at the end of a segment.
//   acc_empty    rank 0 only: one arrival per epilogue warp of both CTAs.
//   part_full[b] both: the epilogue threads have written hand-over buffer b.
//   part_empty[b] both: the finisher has read it.
//   item_full[i] both: rank 0's producer has written pool item slot i.
//   item_empty[i] rank 0 only: every role of both CTAs has read it.
// ---------------------------------------------------------------------------
struct NormSmemTail {
  // per epilogue warp: 32 rows x 32 bf16 of S for one tiled store, in the
  // 64-byte swizzle of the store's tensor map (first, so 1024-byte aligned)
  alignas(1024) uint4 xpose[kEpiWarps][32 * 4];
  uint64_t full[kMaxStages];
  uint64_t mma_done[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t drain[2];                   // one per MMA issuer
  uint64_t part_full[kPartBufs];
  uint64_t part_empty[kPartBufs];
  float part[kPartBufs][2][kTileM];    // per buffer: the lower and upper half's value per row
  uint64_t item_full[kItemRing];
  uint64_t item_empty[kItemRing];
  int item[kItemRing];                 // pool items (-1: the wave's pool is empty)
  uint32_t tmem_slot;
  int abort_flag;
};

// Sets this CTA's and the peer's abort flags and records the timeout.
__device__ __forceinline__ void give_up_pair(volatile int* abort_flag, uint32_t peer_flag) {
  *abort_flag = 1;
  st_cluster_u32(peer_flag, 1u);
  record_error(DORA_ERR_TIMEOUT);
}

// One segment of a pair's work: a static range of one phase on one tile (or a
// Gram job), or an item of the wave's pool.
struct Seg {
  const NormProblemDev* P;
  int wv, ph, tile, blk, cb, kpart, k0, n;
  int chunk;  // pool items: the W0 chunk of the tile, or the tile's G item; -1: static
};

// A pair's segments in order, as one role sees them: per wave its static
// Gram jobs, its static W0 range, then pool items until the wave's pool is
// empty.  Rank 0's producer takes the items from the wave's queue counter
// (one taken ahead, so the round trip overlaps the copies) and writes each
// into both CTAs' item rings; every other role of either CTA reads them
// there, in the same order.  Items are handed out in order: a wave's W0
// chunks (tile by tile), then its G items, so a pair that runs fast takes
// more and the pairs end together.
template <bool kGrouped>
struct SegSource {
  SegWalk<kGrouped> sw;
  const NormSched* sched;
  const NormProblemDev* single;
  const NormProblemDev* table;
  NormSmemTail* tail;
  int* queues;
  int pairs, pair;
  bool grabber;     // rank 0's producer
  bool rank1;       // this CTA is rank 1: arrivals go to rank 0's item_empty
  bool warp_wide;   // the whole warp runs this source (one arrival per warp)
  uint32_t peer_item, peer_full, empty0;  // cluster addresses
  unsigned long long timeout_ns;
  const volatile int* abort;
  int wv, stage;    // stage: 0 static Gram, 1 static W0, 2 pool, 3 wave done
  bool started, have_nxt;
  int nxt;
  uint32_t d;       // item-ring slots used so far
  bool* dep;        // grabber: whether the preceding kernel is known to be done
  Seg s;

  __device__ __forceinline__ void init(const NormSched* sc, const NormProblemDev* sg,
                                       const NormProblemDev* tb, NormSmemTail* t, int* q, int pr,
                                       bool grab, uint32_t rank, bool ww,
                                       unsigned long long tmo, const volatile int* ab) {
    sched = sc;
    single = sg;
    table = tb;
    sw.single = sg;
    sw.table = tb;
    tail = t;
    queues = q;
    pairs = sc->pairs;
    pair = pr;
    grabber = grab;
    rank1 = rank != 0;
    warp_wide = ww;
    peer_item = mapa_shared(smem_addr(&t->item[0]), rank ^ 1u);
    peer_full = mapa_shared(smem_addr(&t->item_full[0]), rank ^ 1u);
    empty0 = mapa_shared(smem_addr(&t->item_empty[0]), 0);
    timeout_ns = tmo;
    abort = ab;
    wv = 0;
    stage = 0;
    started = false;
    have_nxt = false;
    d = 0;
    dep = nullptr;
  }

  // Takes the next item of the current wave's pool ahead (rank 0's producer;
  // after the counters were zeroed by the preceding kernel).
  __device__ __forceinline__ void take_ahead() {
    if (grabber && !have_nxt && wv < sched->waves) {
      if (!*dep) {
        grid_dependency_wait();
        grid_dependency_trigger();
        *dep = true;
      }
      nxt = atomicAdd(queues + wv, 1);
      have_nxt = true;
    }
  }

  // The pool item at position idx of wave W: a W0 chunk or a G item.
  __device__ __forceinline__ void decode(const WaveInfo& W, long long idx) {
    s.wv = wv;
    s.blk = s.cb = s.kpart = 0;
    if (idx < W.dyn_w0_items) {
      const NormProblemDev* P = single;
      if (kGrouped) {
        int m = W.m0;
        while (m + 1 < W.m1 && table[m + 1].dyn_begin <= idx) ++m;
        P = &table[m];
      }
      const int local = static_cast<int>(idx - P->dyn_begin);
      const int c = local % P->cpt;
      s.P = P;
      s.ph = kPhaseW0;
      s.tile = P->dyn_t0 + local / P->cpt;
      s.chunk = c;
      s.k0 = c * P->kb_w / P->cpt;
      s.n = (c + 1) * P->kb_w / P->cpt - s.k0;
    } else {
      const long long j = idx - W.dyn_w0_items;
      const NormProblemDev* P = single;
      if (kGrouped) {
        int m = W.m0;
        while (m + 1 < W.m1 && table[m + 1].g_item_begin <= j) ++m;
        P = &table[m];
      }
      const int local = static_cast<int>(j - P->g_item_begin);
      const int gi = local % P->gipt;
      const int p0 = gi * P->gpi;
      const int p1 = p0 + P->gpi < P->gkp ? p0 + P->gpi : P->gkp;
      s.P = P;
      s.ph = kPhaseG;
      s.tile = local / P->gipt;
      s.chunk = gi;
      s.k0 = p0 * 2 * P->kb_r;
      s.n = (p1 - p0) * 2 * P->kb_r;
    }
  }

  // Writes v into ring slot d of both CTAs (rank 0's producer).
  __device__ __forceinline__ bool publish(int v) {
    const int i = static_cast<int>(d % kItemRing);
    const uint32_t par = (d / kItemRing) & 1u;
    ++d;
    if (!mbar_wait(&tail->item_empty[i], par ^ 1u, timeout_ns, abort)) return false;
    tail->item[i] = v;
    st_cluster_u32(peer_item + 4u * i, static_cast<uint32_t>(v));
    mbar_arrive(&tail->item_full[i]);
    mbar_arrive_cluster(peer_full + 8u * i);
    return true;
  }

  // Reads ring slot d (every other role).
  __device__ __forceinline__ bool consume(int* v) {
    const int i = static_cast<int>(d % kItemRing);
    const uint32_t par = (d / kItemRing) & 1u;
    ++d;
    if (!mbar_wait_cluster(&tail->item_full[i], par, timeout_ns, abort)) return false;
    *v = *reinterpret_cast<volatile int*>(&tail->item[i]);
    if (warp_wide) __syncwarp();
    if (!warp_wide || (threadIdx.x & 31) == 0) {
      if (rank1)
        mbar_arrive_cluster(empty0 + 8u * i);
      else
        mbar_arrive(&tail->item_empty[i]);
    }
    return true;
  }

  // Moves to the next segment; false at the end, or with *ok = false after a
  // bounded wait gave up.
  __device__ __forceinline__ bool next(bool* ok) {
    while (wv < sched->waves) {
      const WaveInfo& W = sched->w[wv];
      if (stage < 2) {
        if (!started) {
          sw.start(W, pairs, pair, stage == 0 ? kPhaseGram : kPhaseW0);
          started = true;
        }
        if (sw.next()) {
          s.P = sw.P;
          s.wv = wv;
          s.ph = sw.ph;
          s.tile = sw.tile;
          s.blk = sw.blk;
          s.cb = sw.cb;
          s.kpart = sw.kpart;
          s.k0 = sw.k0;
          s.n = sw.n;
          s.chunk = -1;
          return true;
        }
        ++stage;
        started = false;
        continue;
      }
      if (stage == 2) {
        int idx;
        if (grabber) {
          take_ahead();
          idx = nxt;
          have_nxt = false;
          const bool end = idx >= W.dyn_items;
          if (!publish(end ? -1 : idx)) {
            *ok = false;
            return false;
          }
          if (!end) {
            take_ahead();
          } else if (wv + 1 < sched->waves) {
            ++wv;          // take the next wave's first item ahead, then come back
            take_ahead();
            --wv;
          }
          if (end) idx = -1;
        } else if (!consume(&idx)) {
          *ok = false;
          return false;
        }
        if (idx < 0) {
          stage = 3;
          continue;
        }
        decode(W, idx);
        return true;
      }
      ++wv;
      stage = 0;
      started = false;
    }
    return false;
  }
};

template <bool kGrouped>
__global__ void __cluster_dims__(2, 1, 1) __maxnreg__(kNormMaxRegs)
    norm_main_kernel(const __grid_constant__ NormProblemDev single,
                     const NormProblemDev* __restrict__ table,
                     const __grid_constant__ NormSched sched, int stages, uint32_t b_region,
                     uint32_t tmem_cols, float eps, unsigned long long timeout_ns,
                     int* __restrict__ queues, unsigned long long* __restrict__ trace) {
  // queues: one pool counter per wave, zeroed by the preceding kernel.
  // trace (optional, diagnostics): per CTA kTraceWords words -- entry and
  // exit global time, MMA-issuer cycles waiting for data / for the
  // accumulator, issued k-blocks, segments, SM id, cycles waited for data
  // over the first four k-blocks; then global times: the MMA issuer starting
  // its static W0 range and its first pool item, the epilogue holding its
  // first Gram job's accumulator and having written that block of S, and the
  // finisher done with its last segment.
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
  const int pair = blockIdx.x >> 1;
  const uint32_t peer_abort = mapa_shared(smem_addr(&tail->abort_flag), rank ^ 1u);

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&mma_done[s], 2);  // both issuers' commits
      mbar_init(&empty[s], kEpiWarps);
    }
    mbar_init(&tail->acc_full, 2);
    mbar_init(&tail->acc_empty, 2 * kEpiWarps);
    mbar_init(&tail->drain[0], 1);
    mbar_init(&tail->drain[1], 1);
    for (int b = 0; b < kPartBufs; ++b) {
      mbar_init(&tail->part_full[b], kEpiWarps * 32);
      mbar_init(&tail->part_empty[b], 1);
    }
    for (int i = 0; i < kItemRing; ++i) {
      mbar_init(&tail->item_full[i], 1);  // rank 0's producer (locally, or from the peer)
      mbar_init(&tail->item_empty[i], kItemConsumers);
    }
    tail->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(&tail->tmem_slot, tmem_cols);
    tmem_relinquish_pair();
  }
  if (!kGrouped && warp == kProducerWarp && lane == 0) {
    prefetch_tmap(&single.tm_w0);
    prefetch_tmap(&single.tm_arow);
    prefetch_tmap(&single.tm_agram);
    prefetch_tmap(&single.tm_a);
    prefetch_tmap(&single.tm_b);
    prefetch_tmap(&single.tm_g);
    prefetch_tmap(&single.tm_glo);
    prefetch_tmap(&single.tm_ghi_st);
    prefetch_tmap(&single.tm_glo_st);
  }
  // Both CTAs' barriers are initialised (and their TMEM allocated) before
  // either CTA signals the other.
  tc_fence_before_sync();
  cluster_sync();
  tc_fence_after_sync();
  const uint32_t tmem_base = tail->tmem_slot;

  SegSource<kGrouped> src;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_last();
      const uint32_t full0 = mapa_shared(smem_addr(&full[0]), 0);  // rank 0's full[0]
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool dep_waited = false;
      const NormProblemDev* ready = nullptr;  // module whose S is known to be written
      const NormProblemDev* fetched = nullptr;  // module whose tensor maps were prefetched
      bool ok = true;
      src.init(&sched, &single, table, tail, queues, pair, rank == 0, rank, false, timeout_ns,
               abort_flag);
      src.dep = &dep_waited;
      while (ok && src.next(&ok)) {
            const Seg& sg = src.s;
            const NormProblemDev* P = sg.P;
            const int ph = sg.ph;
            if (kGrouped && P != fetched) {
              // Each module has its own tensor maps in the table: fetch this
              // module's and the next one's into the TMA unit's descriptor
              // cache ahead of their copies.
              const NormProblemDev* Q[2] = {
                  P, static_cast<int>(P - table) + 1 < sched.w[sg.wv].m1 ? P + 1 : P};
              for (int i = 0; i < 2; ++i) {
                prefetch_tmap(&Q[i]->tm_w0);
                prefetch_tmap(&Q[i]->tm_a);
                prefetch_tmap(&Q[i]->tm_arow);
                prefetch_tmap(&Q[i]->tm_agram);
                prefetch_tmap(&Q[i]->tm_b);
                prefetch_tmap(&Q[i]->tm_g);
                prefetch_tmap(&Q[i]->tm_glo);
              }
              // (the Gram jobs' store maps are fetched by the epilogue's own stores)
              fetched = P;
            }
            if (ph == kPhaseG && P != ready) {
              // S of this module is written by the pairs that run its Gram
              // jobs (each epilogue warp of both CTAs counts its rows of each
              // job); the count they raise was zeroed by the preceding kernel.
              if (!dep_waited) {
                grid_dependency_wait();
                grid_dependency_trigger();
                dep_waited = true;
              }
              if (!wait_counter_geq(P->g_ready, 2 * kEpiWarps * P->gblocks * P->gkp, timeout_ns,
                                    abort_flag)) {
                give_up_pair(abort_flag, peer_abort);
                ok = false;
                break;
              }
              fence_proxy_async_global();
              ready = P;
            }
            const int row0 = sg.tile * kPairM + static_cast<int>(rank) * kTileM;
            for (int k = sg.k0; k < sg.k0 + sg.n; ++k) {
              if (!mbar_wait(&empty[stage], phase ^ 1u, timeout_ns, abort_flag)) {
                give_up_pair(abort_flag, peer_abort);
                ok = false;
                break;
              }
              uint8_t* sa = smem + stage * stage_bytes;
              uint8_t* sb = sa + kTileABytes;
              const uint32_t bar = full0 + stage * static_cast<uint32_t>(sizeof(uint64_t));
              if (ph == kPhaseGram) {
                if (rank == 0) mbar_arrive_expect_tx(&full[stage], P->gram_tx);
                const int kx = k * kBlockK;
                tma_load_2d_pair(sa, &P->tm_arow, bar, kx, row0, pol_keep);
                for (int q = 0; q < P->gchunks; ++q)
                  tma_load_2d_pair(sb + q * P->gh * 128, &P->tm_agram, bar, kx,
                                   sg.cb * P->nc + q * P->gn + static_cast<int>(rank) * P->gh,
                                   pol_keep);
              } else {
                if (rank == 0) mbar_arrive_expect_tx(&full[stage], P->pair_tx);
                const int rk = static_cast<int>(rank);
                if (ph == kPhaseG) {
                  // unit k: part p, then S_hi or S_lo, then the k-block of r
                  const int p = k / (2 * P->kb_r);
                  const int kk = k - p * 2 * P->kb_r;
                  const bool lo = kk >= P->kb_r;
                  const int kx = (kk - (lo ? P->kb_r : 0)) * kBlockK;
                  tma_load_2d_pair(sa, &P->tm_b, bar, kx, row0, pol_keep);
                  const CUtensorMap* slab = lo ? &P->tm_glo : &P->tm_g;
                  if (P->slab4d) {
                    tma_load_5d_pair(sb, slab, bar, kx, 0, rk, 0, p, pol_keep);
                  } else {
                    tma_load_3d_pair(sb, slab, bar, kx, rk * P->h0, p, pol_keep);
                    if (P->n1 > 0)
                      tma_load_3d_pair(sb + P->h0 * 128, slab, bar, kx, P->n0 + rk * P->h0, p,
                                       pol_keep);
                  }
                } else {
                  const int kx = k * kBlockK;
                  tma_load_2d_pair(sa, &P->tm_w0, bar, kx, row0, pol_stream);
                  if (P->slab4d) {
                    tma_load_4d_pair(sb, &P->tm_a, bar, kx, 0, rk, 0, pol_keep);
                  } else {
                    tma_load_2d_pair(sb, &P->tm_a, bar, kx, rk * P->h0, pol_keep);
                    if (P->n1 > 0)
                      tma_load_2d_pair(sb + P->h0 * 128, &P->tm_a, bar, kx, P->n0 + rk * P->h0,
                                       pol_keep);
                  }
                }
              }
              ++issued;
              if (++stage == stages) {
                stage = 0;
                phase ^= 1u;
              }
              // Once the first stages are in flight: wait for the preceding
              // kernel (it zeroes the counters) and take the first pool item
              // ahead.
              if (issued == stages) src.take_ahead();
            }
      }
      if (!ok) give_up_pair(abort_flag, peer_abort);
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
  } else if (warp == kMmaWarp || warp == kMmaWarp + 1) {
    // ------------------------------------------------------------ MMA issuers
    // Issuer q drives accumulator chunk q: the two chains go to the tensor
    // pipe from two threads, which halves the issue time per k-block.  Both
    // commit after every stage and at the end of every segment (issuer 1
    // without MMAs when there is a single chunk), so the barriers count two.
    const int issuer = warp - kMmaWarp;
    if (lane == 0 && rank == 0) {
      const bool tracing = trace != nullptr && issuer == 0;
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool issued_any = false;
      long long wait_data = 0, wait_first = 0, wait_acc = 0, nseg = 0, nkb = 0;
      bool ok = true;
      bool seen_w0 = false, seen_pool = false;
      src.init(&sched, &single, table, tail, queues, pair, false, rank, false, timeout_ns,
               abort_flag);
      while (ok && src.next(&ok)) {
            const Seg& sg = src.s;
            const NormProblemDev* P = sg.P;
            const int ph = sg.ph;
            if (tracing && !seen_w0 && sg.chunk < 0 && ph == kPhaseW0) {
              trace[static_cast<size_t>(blockIdx.x) * kTraceWords + 8] = global_timer_ns();
              seen_w0 = true;
            }
            if (tracing && !seen_pool && sg.chunk >= 0) {
              trace[static_cast<size_t>(blockIdx.x) * kTraceWords + 9] = global_timer_ns();
              seen_pool = true;
            }
            const long long c0 = tracing ? clock64() : 0;
            if (!mbar_wait(&tail->acc_empty, acc_phase ^ 1u, timeout_ns, abort_flag)) {
              give_up_pair(abort_flag, peer_abort);
              ok = false;
              break;
            }
            if (tracing) wait_acc += clock64() - c0;
            ++nseg;
            tc_fence_after_sync();
            // this issuer's chunk: accumulator columns, slab rows, shape
            const bool gram = ph == kPhaseGram;
            const bool active = issuer == 0 || (gram ? P->gchunks > 1 : P->n1 > 0);
            const uint32_t d_col =
                issuer == 0 ? 0u : static_cast<uint32_t>(gram ? P->gn : P->n0);
            const uint32_t b_off =
                issuer == 0 ? 0u : static_cast<uint32_t>(gram ? P->gh : P->h0) * 128u;
            const uint32_t idesc = gram ? P->idesc_gram : (issuer == 0 ? P->idesc0 : P->idesc1);
            for (int i = 0; i < sg.n; ++i) {
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
              if (active) {
                const uint32_t a0 = smem_addr(smem + stage * stage_bytes);
                const uint32_t b0 = a0 + kTileABytes + b_off;
#pragma unroll
                for (int k = 0; k < kBlockK / 16; ++k)
                  umma_bf16_pair(tmem_base + d_col, sw128_kmajor_desc(a0 + k * 32),
                                 sw128_kmajor_desc(b0 + k * 32), idesc,
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
      if (!ok) give_up_pair(abort_flag, peer_abort);
      if (tracing) trace[static_cast<size_t>(blockIdx.x) * kTraceWords + 15] = global_timer_ns();
      if (issued_any) {
        umma_commit_pair(&tail->drain[issuer], 0x1);
        mbar_wait(&tail->drain[issuer], 0, kDrainTimeoutNs, nullptr);
      }
      if (tracing) {
        unsigned long long* tr = trace + static_cast<size_t>(blockIdx.x) * kTraceWords;
        tr[2] = static_cast<unsigned long long>(wait_data);
        tr[3] = static_cast<unsigned long long>(wait_acc);
        tr[4] = static_cast<unsigned long long>(nkb);
        tr[5] = static_cast<unsigned long long>(nseg);
        tr[7] = static_cast<unsigned long long>(wait_first);
      }
    }
  } else if (warp == kFinisherWarp) {
    // ------------------------------------------- partials and finalisation
    // Gram jobs: only the hand-over buffer is passed on (the epilogue warps
    // publish their rows of S themselves).
    // W0 / G segments: lane l takes rows l, l + 32, l + 64, l + 96 of this
    // CTA's half of the tile: it adds the two epilogue halves' values of each
    // row (lower + upper), posts them as the segment's partial and counts the
    // arrival; when that was the tile's last arrival, it sums every slot in
    // slot order and writes n and g.  The arrival's result is looked at one
    // segment later (or at the end), so its round trip overlaps the next
    // segment's instead of holding up the hand-over buffers.
    uint32_t seg_count = 0;
    bool dep_waited = false;
    bool ok = true;
    // the previous segment, whose arrival count is still in flight
    bool pend = false;
    int pend_prev = 0, pend_nseg = 0, pend_row_base = 0;
    const NormProblemDev* pend_P = nullptr;
    const float* pend_part = nullptr;
    auto finish_pending = [&]() {
      if (!pend) return;
      pend = false;
      const int prev = __shfl_sync(0xffffffffu, pend_prev, 0);
      if (prev != pend_nseg - 1) return;
      __syncwarp();
      // All of a batch's loads (kFinBatch slots of the four rows) are in
      // flight together; absent slots add zero, so the sum is the same
      // fixed slot order whatever the batching.
      float sum[4] = {0.f, 0.f, 0.f, 0.f};
      for (int c0 = 0; c0 < pend_nseg; c0 += kFinBatch) {
        float v[4][kFinBatch];
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int u = 0; u < kFinBatch; ++u)
            v[q][u] = c0 + u < pend_nseg
                          ? __ldcg(pend_part + static_cast<size_t>(c0 + u) * kPairM + lane + 32 * q)
                          : 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int u = 0; u < kFinBatch; ++u) sum[q] += v[q][u];
      }
      const NormProblemDev* Q = pend_P;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int grow = pend_row_base + lane + 32 * q;
        if (grow >= Q->d_out) continue;
        if (Q->emit_sq) {
          Q->n_out[grow] = sum[q];
        } else {
          const float n = __fsqrt_rn(fmaxf(sum[q], 0.f));
          Q->n_out[grow] = n;
          if (Q->m != nullptr && Q->g_out != nullptr)
            Q->g_out[grow] = __fdiv_rn(__ldg(Q->m + grow), fmaxf(n, eps));
        }
      }
    };
    src.init(&sched, &single, table, tail, queues, pair, false, rank, true, timeout_ns,
             abort_flag);
    while (ok && src.next(&ok)) {
      const Seg& sg = src.s;
      const NormProblemDev* P = sg.P;
      const int ph = sg.ph;
      const int t = sg.tile;
      const int buf = static_cast<int>(seg_count % kPartBufs);
      const uint32_t par = (seg_count / kPartBufs) & 1u;
      ++seg_count;
      // A static tile's W0 segment table, requested before the hand-over wait
      // (it comes from the preceding kernel, waited for once before).
      const bool static_tile = ph != kPhaseGram && t < P->dyn_t0;
      int tw = 0;
      if (static_tile && dep_waited) tw = __ldcg(P->tile_w + t);
      if (!mbar_wait(&tail->part_full[buf], par, timeout_ns, abort_flag)) {
        ok = false;
        break;
      }
      if (ph == kPhaseGram) {  // published by the epilogue warps themselves
        __syncwarp();
        if (lane == 0) mbar_arrive(&tail->part_empty[buf]);
        continue;
      }
      float v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int row = lane + 32 * q;
        v[q] = tail->part[buf][0][row] + tail->part[buf][1][row];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&tail->part_empty[buf]);
      if (!dep_waited) {  // counters and the tile table come from the preceding kernel
        grid_dependency_wait();
        dep_waited = true;
        if (static_tile) tw = __ldcg(P->tile_w + t);
      }
      // Where this segment's partial goes among the tile's segments: first
      // its W0 segments -- on a static tile, consecutive pairs (found by the
      // preceding kernel), on a pool tile one per chunk -- then its G items.
      int nw, ord;
      if (static_tile) {
        nw = tw >> 16;
        ord = sg.chunk < 0 ? pair - (tw & 0xffff) : nw + sg.chunk;
      } else {
        nw = P->cpt;
        ord = ph == kPhaseW0 ? sg.chunk : nw + sg.chunk;
      }
      const int nseg = nw + P->gipt;
      const int row_base = t * kPairM + static_cast<int>(rank) * kTileM;
      float* part_t = P->partial + static_cast<size_t>(t) * P->seg_slots * kPairM +
                      static_cast<int>(rank) * kTileM;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (row_base + lane + 32 * q < P->d_out &&
            DORA_BOUNDS_OK(ord >= 0 && ord < P->seg_slots && nseg <= P->seg_slots))
          part_t[static_cast<size_t>(ord) * kPairM + lane + 32 * q] = v[q];
      // One acquire-release arrival per warp: it publishes the lanes'
      // partials (ordered before it by the warp barrier) and, for the last
      // arrival, orders the other segments' partials before the loads of the
      // finalisation.  The previous segment's arrival is looked at first.
      __syncwarp();
      int prev = 0;
      if (lane == 0) prev = atom_add_acq_rel_gpu(P->tile_cnt + t * 2 + static_cast<int>(rank), 1);
      finish_pending();
      pend = true;
      pend_prev = prev;
      pend_nseg = nseg;
      pend_row_base = row_base;
      pend_P = P;
      pend_part = part_t;
    }
    if (ok) finish_pending();
    if (!ok) give_up_pair(abort_flag, peer_abort);
    if (trace != nullptr && lane == 0)
      trace[static_cast<size_t>(blockIdx.x) * kTraceWords + 12] = global_timer_ns();
  } else if (warp < kEpiWarps) {
    // ------------------------------------ ||W0_i||^2 + epilogue (warps 0-7)
    // Thread (half h, row): TMEM lane `row`; half h of the row's 16-byte chunks
    // of each W0 stage and half h of the accumulator's 32-column chunks.
    const int half = warp / 4;
    const int row = threadIdx.x & (kTileM - 1);
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t acc_empty0 = mapa_shared(smem_addr(&tail->acc_empty), 0);
    int stage = 0;
    uint32_t phase = 0, acc_phase = 0, seg_count = 0;
    bool gram_traced = false;
    bool ok = true;
    src.init(&sched, &single, table, tail, queues, pair, false, rank, true, timeout_ns,
             abort_flag);
    while (ok && src.next(&ok)) {
          const Seg& sg = src.s;
          const NormProblemDev* P = sg.P;
          const int ph = sg.ph;
          const int t = sg.tile;
          const int r = P->r;
          // the row of W0 (or, for the Gram, of A) this thread finishes
          const int grow = t * kPairM + static_cast<int>(rank) * kTileM + row;
          const bool gram = ph == kPhaseGram;
          const bool valid = grow < (gram ? r : P->d_out);
          // this half's 32-column chunks of the accumulator
          const int nchunks = gram ? (P->nc + 31) / 32 : (P->n0 + P->n1 + 31) / 32;
          const int c_lo = half == 0 ? 0 : (nchunks + 1) / 2;
          const int c_hi = half == 0 ? (nchunks + 1) / 2 : nchunks;
          // Prefetch B_i for (up to kPrefetchChunks of) those columns while
          // the MMAs of this segment run.
          const uint16_t* brow = P->B + static_cast<size_t>(!gram && valid ? grow : 0) * r;
          uint4 bq[kPrefetchChunks][4];
#pragma unroll
          for (int c = 0; c < kPrefetchChunks; ++c)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int col = (c_lo + c) * 32 + q * 8;
              bq[c][q] = (!gram && valid && c_lo + c < c_hi && col < r)
                             ? __ldg(reinterpret_cast<const uint4*>(brow + col))
                             : make_uint4(0u, 0u, 0u, 0u);
            }
          float ss = 0.f;
          for (int i = 0; i < sg.n; ++i) {
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

          if (gram) {
            // ---- Gram job: this CTA's 128 rows gr of the block of G
            // (columns [cb nc, cb nc + nc)) over part kpart of d_in, scaled
            // into S_kpart (row gr, column c): 2 G' for c < gr, G' for c = gr,
            // 0 above.
            const bool first = trace != nullptr && threadIdx.x == 0 && !gram_traced;
            if (first) trace[static_cast<size_t>(blockIdx.x) * kTraceWords + 10] = global_timer_ns();
            const int col0 = sg.cb * P->nc;
            const int col_end = min(r, col0 + P->nc);
            const float hs = P->half_s;
            const float two_hs = 2.f * hs;
            // This warp's 32 rows of S_kpart (TMEM lanes (warp & 3) * 32 + i):
            // per 32 columns, hi then lo, the warp writes the 32 x 32 block
            // into its staging tile (16-byte units swizzled by row, the
            // store's 64-byte swizzle: no bank conflicts) and one lane stores
            // it with TMA; rows and columns past r are clipped by the store.
            const int wrow0 = t * kPairM + static_cast<int>(rank) * kTileM + (warp & 3) * 32;
            uint4* xp = tail->xpose[warp];
            bool pending = false;  // a store may still be reading the staging tile
            auto stage_store = [&](const uint32_t (&w)[16], const CUtensorMap* map, int colc) {
              if (pending) {
                if (lane == 0) bulk_wait_group_read0();
                __syncwarp();
              }
#pragma unroll
              for (int j = 0; j < 4; ++j)
                xp[lane * 4 + (j ^ ((lane >> 1) & 3))] =
                    make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0 && DORA_BOUNDS_OK(colc % 8 == 0 && sg.kpart < P->gkp)) {
                tma_store_3d(map, xp, colc, wrow0, sg.kpart);
                bulk_commit_group();
              }
              pending = true;
            };
#pragma unroll 1
            for (int c = c_lo; c < c_hi; ++c) {
              float acc[32];
              tmem_load_32cols(tmem_base + lane_base + c * 32, acc);
              const int colc = col0 + c * 32;
              uint32_t wh[16], wl[16];
              // The warp's 32 rows are wrow0 .. wrow0 + 31: a block of
              // columns wholly left of all of them is scaled by 2 G' as a
              // whole, one wholly right of them is zero, and the block that
              // holds the diagonal goes element by element.
              if (colc + 31 < wrow0) {
#pragma unroll
                for (int e = 0; e < 16; ++e)
                  split_bf16_hi_lo(two_hs * acc[2 * e], two_hs * acc[2 * e + 1], &wh[e], &wl[e]);
              } else if (colc > wrow0 + 31) {
#pragma unroll
                for (int e = 0; e < 16; ++e) wh[e] = wl[e] = 0u;
              } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                  float x[2];
#pragma unroll
                  for (int f = 0; f < 2; ++f) {
                    const int col = colc + 2 * e + f;
                    const float g = acc[2 * e + f];
                    x[f] = col < grow ? two_hs * g : (col == grow ? hs * g : 0.f);
                  }
                  split_bf16_hi_lo(x[0], x[1], &wh[e], &wl[e]);
                }
              }
              if (colc < col_end) {
                stage_store(wh, &P->tm_ghi_st, colc);
                stage_store(wl, &P->tm_glo_st, colc);
              }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster_relaxed(acc_empty0);
            // The pseudo-tile's last block also zeroes the columns past it
            // (all above the diagonal for these rows), 32 at a time, split
            // between the two halves.
            const int njt = gram_jobs_of_tile(r, P->nc, t);
            if (sg.cb == njt - 1) {
              const uint32_t zero[16] = {};
              for (int colc = njt * P->nc + half * 32; colc < r; colc += 64) {
                stage_store(zero, &P->tm_ghi_st, colc);
                stage_store(zero, &P->tm_glo_st, colc);
              }
            }
            // Once every store of this warp has written global memory, its
            // rows of S are published to the TMA reads of every pair's G
            // units: a release add on the count their producers wait for.
            if (lane == 0) {
              bulk_wait_group0();
              fence_proxy_async_global();
              if (first) trace[static_cast<size_t>(blockIdx.x) * kTraceWords + 14] = global_timer_ns();
              red_add_release_gpu(P->g_ready, 1);
              if (first) trace[static_cast<size_t>(blockIdx.x) * kTraceWords + 11] = global_timer_ns();
            }
            __syncwarp();
            const int buf = static_cast<int>(seg_count % kPartBufs);
            const uint32_t use = seg_count / kPartBufs;
            ++seg_count;
            if (!mbar_wait(&tail->part_empty[buf], (use & 1u) ^ 1u, timeout_ns, abort_flag)) {
              give_up_pair(abort_flag, peer_abort);
              ok = false;
              break;
            }
            mbar_arrive(&tail->part_full[buf]);
            if (first) gram_traced = true;
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
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster_relaxed(acc_empty0);
          // Hand this half's value of the row to the finisher warp.
          const int buf = static_cast<int>(seg_count % kPartBufs);
          const uint32_t use = seg_count / kPartBufs;
          ++seg_count;
          const long long cw = trace != nullptr ? clock64() : 0;
          const bool handed =
              mbar_wait(&tail->part_empty[buf], (use & 1u) ^ 1u, timeout_ns, abort_flag);
          if (trace != nullptr && threadIdx.x == 0)
            trace[static_cast<size_t>(blockIdx.x) * kTraceWords + 13] += clock64() - cw;
          if (!handed) {
            give_up_pair(abort_flag, peer_abort);
            ok = false;
            break;
          }
          tail->part[buf][half][row] = fmaf(P->two_s, dot, ss);
          mbar_arrive(&tail->part_full[buf]);
    }
    if (!ok) give_up_pair(abort_flag, peer_abort);
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
// fused kernel launch; it waits for this grid before it reads either.  One
// warp of at most 32 registers: it fits beside a fused-kernel CTA on the same
// SM (which leaves 1024 registers free), so no pair waits for it to finish.
template <bool kGrouped>
__global__ void __maxnreg__(32)
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
      for (int t = tid; t < P->dyn_t0; t += stride) {
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
