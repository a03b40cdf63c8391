// Factored DoRA row norm on the 5th-generation tensor cores (tcgen05 + TMEM,
// operands staged by TMA), following "Scaling DoRA: High-Rank Adaptation via
// Factored Norms and Fused Kernels", section 2: the squared norm of row i of
// W0 + s B A is ||W0_i||^2 + 2 s B_i.(W0 A^T)_i + s^2 B_i G B_i^T, G = A A^T,
// evaluated from [d_out, r] and [r, r] intermediates only.
//
// Three kernels per module (the grouped call runs each once for all modules):
//   gram_kernel      G' = (s/2) A A^T: 128x128 upper-triangle tiles, split
//                    over K, fp32 partial tiles in the workspace.
//   gram_reduce      sums the K splits in a fixed order and writes G' as two
//                    bf16 matrices, G'_hi = bf16(G') and G'_lo = bf16(G' - G'_hi),
//                    so that the Gram term keeps fp32-level accuracy (the pages'
//                    norm accumulates in fp32 whatever the weight dtype);
//                    mirrors the off-diagonal tiles; zeroes the norm GEMM's
//                    arrival counters.
//   norm_main_kernel one 128-row tile of W0 at a time, stream-K over the
//                    (tile, k-block) sequence.  Per tile the accumulator in
//                    TMEM collects  W0_tile A^T  (k-blocks over d_in) and then
//                    B_tile G'_hi and B_tile G'_lo  (k-blocks over r), so that
//                    B_i . acc_i = B_i.(W0 A^T)_i + (s/2) B_i G B_i^T.
//                    While the MMAs run, four warps square and sum the same
//                    W0 tile straight from shared memory (||W0_i||^2), so W0
//                    crosses HBM exactly once.  The epilogue (eight warps, each
//                    half of a row's columns, with B_i prefetched into registers
//                    while the MMAs run) drains TMEM, dots each row with B_i
//                    and writes the per-row partial ||W0_i||^2_part +
//                    2 s B_i.acc_i for its k-range.  The segment that posts a
//                    tile's partials last (an arrival counter per 32 rows)
//                    finalises those rows: n_i = sqrt(max(sum of partials, 0))
//                    with the partials summed in slot order, and
//                    g_i = m_i / max(n_i, eps)  (section 4, precision bullet).
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace dora {

constexpr int kTileM = 128;                  // W0 rows per tile = TMEM lanes
constexpr int kBlockK = 64;                  // bf16 of K per stage: one 128-byte swizzle row
constexpr int kMaxStages = 8;
constexpr int kTcThreads = 192;              // Gram: warps 0-3 epilogue, 4 TMA, 5 MMA
constexpr int kEpiWarps = 8;                 // norm: warps 0-7 reduction/epilogue
constexpr int kNormThreads = (kEpiWarps + 2) * 32;  // + warp 8 TMA, warp 9 MMA
constexpr int kMaxChunksPerHalf = 8;         // 32-column TMEM chunks per epilogue half (r <= 512)
constexpr int kPrefetchChunks = 6;           // of which B is prefetched into registers (r <= 384)
// Registers are granted to a block in groups of four warps, so the 10-warp
// norm kernel is charged as 12 warps: 65536 / 384 threads = 170 -> 168.
constexpr int kNormMaxRegs = 168;

constexpr uint32_t kTileABytes = kTileM * kBlockK * 2;  // 16 KiB
constexpr int kMaxDynSmem = 232448;          // 227 KiB opt-in per block on sm_100

// ---------------------------------------------------------------------------
// Problem descriptors (built on the host; kernel parameter for one module,
// a workspace table for the grouped call).
// ---------------------------------------------------------------------------
struct alignas(64) NormProblemDev {
  CUtensorMap tm_w0;     // W0 [d_out, d_in], box 64 x 128
  CUtensorMap tm_a;      // A  [r, d_in],     box 64 x box_rows
  CUtensorMap tm_b;      // B  [d_out, r],    box 64 x 128
  CUtensorMap tm_g;      // G'_hi [r, r],     box 64 x box_rows
  CUtensorMap tm_glo;    // G'_lo [r, r],     box 64 x box_rows
  const uint16_t* B;     // bf16 bits of B, for the epilogue dot
  float* partial;        // [tiles * seg_slots][128] per-row partials
  int* tile_cnt;         // [tiles * 4] segments posted per 32-row quarter of a tile
  const float* m;        // [d_out] or null
  float* n_out;          // [d_out]
  float* g_out;          // [d_out] or null
  long long unit_begin;  // first global stream-K unit of this problem
  long long wave_begin, wave_units;  // the stream-K wave holding this problem
  int d_out, r;
  int n0, n1;            // N of the two accumulator chunks (n1 = 0: single chunk)
  int box_rows, nbox;    // N-side operand: boxes per stage and rows per box
  int slab3d;            // tm_a / tm_g / tm_glo are 3-D {64, box_rows, nbox}: one box per slab
  int emit_sq;           // write the squared-norm sum itself to n_out (no clamp, sqrt or g)
  int kb_w, kb_r, kb_tile, tiles, seg_slots;  // kb_tile = kb_w + 2 kb_r (hi, then lo)
  uint32_t stage_tx;     // bytes landing per stage
  uint32_t idesc0, idesc1;
  float two_s;
};

struct alignas(64) GramProblemDev {
  CUtensorMap tm_a;      // A [r, d_in], box 64 x 128
  float* partial;        // [pairs * S][128 * 128]
  uint16_t* g_out;       // G'_hi [r][r8] bf16 bits
  uint16_t* g_lo;        // G'_lo [r][r8] bf16 bits
  int* tile_cnt;         // the norm GEMM's arrival counters, zeroed by the reduce
  int cnt_len;
  int r, r8, kb, tiles_r, pairs, S, job_begin;
  float half_s;
};

// Waves: the grouped call splits its modules (in order) into waves whose
// operands that every tile re-reads (A and G') fit in L2 together, and runs
// stream-K over one wave at a time across all CTAs.  begin[w] .. begin[w+1]
// are wave w's global units; one module alone is one wave.  Every wave has at
// least as many units as there are CTAs, so no CTA's share of a wave is empty.
constexpr int kMaxWaves = 64;
struct WaveList {
  int n;
  long long begin[kMaxWaves + 1];
};

// ---------------------------------------------------------------------------
// Stream-K bookkeeping (per wave, U = the wave's units, X relative to the
// wave's first unit).  CTA c of C owns units [c U / C, (c+1) U / C).
// The CTAs that touch the tile starting at unit X are first_cta(X) ..
// first_cta(X + kb_tile - 1); the segment of CTA c on that tile goes to slot
// c - first_cta(X).
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ int first_cta_of_unit(long long x, long long U, int C) {
  return static_cast<int>(((x + 1) * C - 1) / U);
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

__device__ __forceinline__ void give_up(volatile int* abort_flag) {
  *abort_flag = 1;
  record_error(DORA_ERR_TIMEOUT);
}

// Walks the global unit sequence of one CTA: which problem, tile and k-block.
template <bool kGrouped>
struct UnitCursor {
  const NormProblemDev* single;
  const NormProblemDev* table;
  int nprob;
  int p;
  const NormProblemDev* P;
  long long local;  // unit index inside problem p

  __device__ __forceinline__ void start(long long u) {
    if (kGrouped) {
      p = 0;
      while (p + 1 < nprob && table[p + 1].unit_begin <= u) ++p;
      P = &table[p];
    } else {
      p = 0;
      P = single;
    }
    local = u - P->unit_begin;
  }
  // Moves to the next problem when the current one is exhausted.
  __device__ __forceinline__ void settle(long long u) {
    if (kGrouped) {
      while (local >= static_cast<long long>(P->tiles) * P->kb_tile) {
        ++p;
        P = &table[p];
        local = u - P->unit_begin;
      }
    }
  }
  __device__ __forceinline__ int tile() const { return static_cast<int>(local / P->kb_tile); }
  __device__ __forceinline__ int kblock() const { return static_cast<int>(local % P->kb_tile); }
};

// ---------------------------------------------------------------------------
// Fused norm GEMM
// ---------------------------------------------------------------------------
struct NormSmemTail {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t drain;
  uint64_t half_ready;        // upper epilogue half has posted its partial
  float half_part[2][kTileM];  // double-buffered by segment parity
  uint32_t tmem_slot;
  int abort_flag;
};

template <bool kGrouped>
__global__ void __maxnreg__(kNormMaxRegs)
    norm_main_kernel(const __grid_constant__ NormProblemDev single,
                     const NormProblemDev* __restrict__ table, int nprob, long long total_units,
                     int stages, uint32_t b_region, uint32_t tmem_cols, float eps,
                     const __grid_constant__ WaveList waves, unsigned long long timeout_ns,
                     unsigned long long* __restrict__ trace) {
  // trace (optional, diagnostics): per CTA 8 words -- entry and exit global
  // time, MMA-issuer cycles waiting for data / for the accumulator, issued
  // k-blocks, segments, SM id.
  const uint64_t t_entry = trace != nullptr ? global_timer_ns() : 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t stage_bytes = kTileABytes + b_region;
  NormSmemTail* tail = reinterpret_cast<NormSmemTail*>(smem + stages * stage_bytes);
  uint64_t* full = tail->full;
  uint64_t* empty = tail->empty;
  volatile int* abort_flag = &tail->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int C = gridDim.x;
  const int cta = blockIdx.x;
  (void)total_units;
  // This CTA's units of wave w.
  auto wave_range = [&](int w, long long& ub, long long& ue) {
    const long long b = waves.begin[w], U = waves.begin[w + 1] - b;
    ub = b + static_cast<long long>(cta) * U / C;
    ue = b + static_cast<long long>(cta + 1) * U / C;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + kEpiWarps);  // MMA commit + one arrival per epilogue warp
    }
    mbar_init(&tail->acc_full, 1);
    mbar_init(&tail->acc_empty, kEpiWarps * 32);
    mbar_init(&tail->drain, 1);
    mbar_init(&tail->half_ready, kTileM);
    tail->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tail->tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  if (!kGrouped && warp == kEpiWarps && lane == 0) {
    prefetch_tmap(&single.tm_w0);
    prefetch_tmap(&single.tm_a);
    prefetch_tmap(&single.tm_b);
    prefetch_tmap(&single.tm_g);
    prefetch_tmap(&single.tm_glo);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = tail->tmem_slot;

  UnitCursor<kGrouped> cur;
  cur.single = &single;
  cur.table = table;
  cur.nprob = nprob;

  if (warp == kEpiWarps) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool waited = false;  // G' (written by the preceding kernel) is visible
      bool ok = true;
      for (int wv = 0; ok && wv < waves.n; ++wv) {
      long long u_begin, u_end;
      wave_range(wv, u_begin, u_end);
      if (u_begin < u_end) cur.start(u_begin);
      for (long long u = u_begin; u < u_end; ++u, ++cur.local) {
        cur.settle(u);
        const NormProblemDev* P = cur.P;
        const int t = cur.tile();
        const int kb = cur.kblock();
        if (!mbar_wait(&empty[stage], phase ^ 1u, timeout_ns, abort_flag)) {
          give_up(abort_flag);
          ok = false;
          break;
        }
        uint8_t* sa = smem + stage * stage_bytes;
        uint8_t* sb = sa + kTileABytes;
        if (kb < P->kb_w) {
          mbar_arrive_expect_tx(&full[stage], P->stage_tx);
          tma_load_2d(sa, &P->tm_w0, &full[stage], kb * kBlockK, t * kTileM, pol_stream);

          if (P->slab3d)
            tma_load_3d(sb, &P->tm_a, &full[stage], kb * kBlockK, 0, 0, pol_keep);
          else
            for (int j = 0; j < P->nbox; ++j)
              tma_load_2d(sb + j * P->box_rows * 128, &P->tm_a, &full[stage], kb * kBlockK,
                          j * P->box_rows, pol_keep);
        } else {
          if (!waited) {
            grid_dependency_wait();
            grid_dependency_trigger();
            waited = true;
          }
          const bool lo = kb >= P->kb_w + P->kb_r;
          const int kr = kb - P->kb_w - (lo ? P->kb_r : 0);
          const CUtensorMap* gm = lo ? &P->tm_glo : &P->tm_g;
          mbar_arrive_expect_tx(&full[stage], P->stage_tx);
          tma_load_2d(sa, &P->tm_b, &full[stage], kr * kBlockK, t * kTileM, pol_keep);
          if (P->slab3d)
            tma_load_3d(sb, gm, &full[stage], kr * kBlockK, 0, 0, pol_keep);
          else
            for (int j = 0; j < P->nbox; ++j)
              tma_load_2d(sb + j * P->box_rows * 128, gm, &full[stage], kr * kBlockK,
                          j * P->box_rows, pol_keep);
        }
        ++issued;
        if (++stage == stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      }
      if (!waited) {
        grid_dependency_wait();
        grid_dependency_trigger();
      }
      // Let every copy already issued land before the block can exit.
      const long long first = issued > stages ? issued - stages : 0;
      for (long long j = first; j < issued; ++j)
        mbar_wait(&full[j % stages], static_cast<uint32_t>((j / stages) & 1), kDrainTimeoutNs,
                  nullptr);
    }
  } else if (warp == kEpiWarps + 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool issued_any = false;
      long long wait_data = 0, wait_acc = 0, nseg = 0, nkb = 0;
      bool ok = true;
      for (int wv = 0; ok && wv < waves.n; ++wv) {
      long long u_begin, u_end;
      wave_range(wv, u_begin, u_end);
      if (u_begin >= u_end) continue;
      cur.start(u_begin);
      long long u = u_begin;
      while (ok && u < u_end) {
        cur.settle(u);
        const NormProblemDev* P = cur.P;
        const int kb0 = cur.kblock();
        const long long seg_end = min(u_end, u + (P->kb_tile - kb0));
        const long long c0 = clock64();
        if (!mbar_wait(&tail->acc_empty, acc_phase ^ 1u, timeout_ns, abort_flag)) {
          give_up(abort_flag);
          ok = false;
          break;
        }
        wait_acc += clock64() - c0;
        ++nseg;
        tc_fence_after_sync();
        const uint32_t idesc0 = P->idesc0, idesc1 = P->idesc1;
        const int n0 = P->n0, n1 = P->n1;
        bool first = true;
        for (; u < seg_end; ++u, ++cur.local) {
          const long long c1 = clock64();
          if (!mbar_wait(&full[stage], phase, timeout_ns, abort_flag)) {
            give_up(abort_flag);
            ok = false;
            break;
          }
          wait_data += clock64() - c1;
          ++nkb;
          tc_fence_after_sync();
          const uint32_t a0 = smem_addr(smem + stage * stage_bytes);
          const uint32_t b0 = a0 + kTileABytes;
#pragma unroll
          for (int k = 0; k < kBlockK / 16; ++k) {
            const uint64_t ad = sw128_kmajor_desc(a0 + k * 32);
            const uint32_t acc = (first && k == 0) ? 0u : 1u;
            umma_bf16(tmem_base, ad, sw128_kmajor_desc(b0 + k * 32), idesc0, acc);
            if (n1 > 0)
              umma_bf16(tmem_base + n0, ad, sw128_kmajor_desc(b0 + n0 * 128 + k * 32), idesc1,
                        acc);
          }
          first = false;
          issued_any = true;
          umma_commit(&empty[stage]);
          if (++stage == stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tail->acc_full);
        acc_phase ^= 1u;
      }
      }
      if (issued_any) {
        umma_commit(&tail->drain);
        mbar_wait(&tail->drain, 0, kDrainTimeoutNs, nullptr);
      }
      if (trace != nullptr) {
        unsigned long long* tr = trace + static_cast<size_t>(cta) * 8;
        tr[2] = static_cast<unsigned long long>(wait_data);
        tr[3] = static_cast<unsigned long long>(wait_acc);
        tr[4] = static_cast<unsigned long long>(nkb);
        tr[5] = static_cast<unsigned long long>(nseg);
      }
    }
  } else {
    // ------------------------------------ ||W0_i||^2 + epilogue (warps 0-7)
    // Thread (half h, row): TMEM lane `row`; half h of the row's 16-byte chunks
    // of each W0 stage and half h of the accumulator's 32-column chunks.
    const int half = warp / 4;
    const int row = threadIdx.x & (kTileM - 1);
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    int stage = 0;
    uint32_t phase = 0, acc_phase = 0, seg_count = 0;
    bool dep_waited = false;
    bool ok = true;
    for (int wv = 0; ok && wv < waves.n; ++wv) {
      long long u_begin, u_end;
      wave_range(wv, u_begin, u_end);
      if (u_begin >= u_end) continue;
      cur.start(u_begin);
      long long u = u_begin;
      while (ok && u < u_end) {
        cur.settle(u);
        const NormProblemDev* P = cur.P;
        const int t = cur.tile();
        const int kb0 = cur.kblock();
        const long long seg_end = min(u_end, u + (P->kb_tile - kb0));
        const int r = P->r;
        const int grow = t * kTileM + row;
        const bool valid = grow < P->d_out;
        // this half's 32-column chunks of the accumulator
        const int nchunks = (P->n0 + P->n1 + 31) / 32;
        const int c_lo = half == 0 ? 0 : (nchunks + 1) / 2;
        const int c_hi = half == 0 ? (nchunks + 1) / 2 : nchunks;
        // Prefetch B_i for (up to kPrefetchChunks of) those columns while the
        // MMAs of this segment run.
        const uint16_t* brow = P->B + static_cast<size_t>(valid ? grow : 0) * r;
        uint4 bq[kPrefetchChunks][4];
#pragma unroll
        for (int c = 0; c < kPrefetchChunks; ++c)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int col = (c_lo + c) * 32 + q * 8;
            bq[c][q] = (valid && c_lo + c < c_hi && col < r)
                           ? __ldg(reinterpret_cast<const uint4*>(brow + col))
                           : make_uint4(0u, 0u, 0u, 0u);
          }
        float ss = 0.f;
        int kb = kb0;
        for (; u < seg_end; ++u, ++cur.local, ++kb) {
          if (!mbar_wait(&full[stage], phase, timeout_ns, abort_flag)) {
            give_up(abort_flag);
            ok = false;
            break;
          }
          if (kb < P->kb_w) {
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
          give_up(abort_flag);
          ok = false;
          break;
        }
        tc_fence_after_sync();
        float dot = 0.f;
#pragma unroll
        for (int c = 0; c < kMaxChunksPerHalf; ++c) {
          if (c_lo + c < c_hi) {  // warp-uniform
            float acc[32];
            tmem_load_32cols(tmem_base + lane_base + (c_lo + c) * 32, acc);
            if (c < kPrefetchChunks) {
#pragma unroll
              for (int q = 0; q < 4; ++q) dot += dot_bf16x8(acc + q * 8, bq[c < kPrefetchChunks ? c : 0][q]);
            } else {
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int col = (c_lo + c) * 32 + q * 8;
                if (valid && col < r)
                  dot += dot_bf16x8(acc + q * 8, __ldg(reinterpret_cast<const uint4*>(brow + col)));
              }
            }
          }
        }
        tc_fence_before_sync();
        acc_phase ^= 1u;
        // Combine the two halves of the row in a fixed order (lower + upper).
        // The lower half takes the upper half's value before it releases the
        // accumulator, so the next segment cannot overwrite it early.
        const float part = fmaf(P->two_s, dot, ss);
        const int buf = seg_count & 1;
        if (half == 1) {
          tail->half_part[buf][row] = part;
          mbar_arrive(&tail->half_ready);
          mbar_arrive(&tail->acc_empty);
        } else {
          const bool got_one =
              mbar_wait(&tail->half_ready, seg_count & 1u, timeout_ns, abort_flag);
          const float other = tail->half_part[buf][row];
          mbar_arrive(&tail->acc_empty);
          if (!__all_sync(0xffffffffu, got_one)) {
            give_up(abort_flag);
            ok = false;
            break;
          }
          const long long x0 = P->unit_begin - P->wave_begin + static_cast<long long>(t) * P->kb_tile;
          const int c0 = first_cta_of_unit(x0, P->wave_units, C);
          const int nseg = first_cta_of_unit(x0 + P->kb_tile - 1, P->wave_units, C) - c0 + 1;
          float* part_t = P->partial + static_cast<size_t>(t) * P->seg_slots * kTileM + row;
          if (valid) part_t[static_cast<size_t>(cta - c0) * kTileM] = part + other;
          // The last of the tile's segments to post its partials (per warp:
          // 32 rows) sums every slot in slot order and writes n and g.
          __threadfence();
          __syncwarp();
          if (!dep_waited) {  // the counters are zeroed by the preceding kernel
            grid_dependency_wait();
            dep_waited = true;
          }
          int prev = 0;
          if (lane == 0) prev = atomicAdd(P->tile_cnt + t * 4 + warp, 1);
          prev = __shfl_sync(0xffffffffu, prev, 0);
          if (prev == nseg - 1) {
            __threadfence();
            if (valid) {
              float sum = 0.f;
              for (int c = 0; c < nseg; ++c) sum += __ldcg(part_t + static_cast<size_t>(c) * kTileM);
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

  __syncwarp();
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, tmem_cols);
  }
  if (trace != nullptr && threadIdx.x == 0) {
    unsigned long long* tr = trace + static_cast<size_t>(cta) * 8;
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    tr[0] = t_entry;
    tr[1] = global_timer_ns();
    tr[6] = smid;
  }
}

// ---------------------------------------------------------------------------
// Gram matrix G' = (s/2) A A^T
// ---------------------------------------------------------------------------
constexpr int kGramStages = 4;
constexpr uint32_t kGramStageBytes = 2 * kTileABytes;  // 128 rows of A for each operand

__device__ __forceinline__ void gram_pair(int pair, int tiles, int& a, int& b) {
  a = 0;
  int left = pair;
  while (left >= tiles - a) {
    left -= tiles - a;
    ++a;
  }
  b = a + left;
}

template <bool kGrouped>
__global__ void __launch_bounds__(kTcThreads, 1)
    gram_kernel(const __grid_constant__ GramProblemDev single,
                const GramProblemDev* __restrict__ table, int nprob,
                unsigned long long timeout_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGramStages * kGramStageBytes);
  uint64_t* empty = full + kGramStages;
  uint64_t* acc_full = empty + kGramStages;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // job -> (problem, tile pair, K split)
  const GramProblemDev* P = &single;
  int job = blockIdx.x;
  if (kGrouped) {
    int p = 0;
    while (p + 1 < nprob && table[p + 1].job_begin <= job) ++p;
    P = &table[p];
    job -= P->job_begin;
  }
  const int pair = job / P->S;
  const int split = job % P->S;
  int ta, tb;
  gram_pair(pair, P->tiles_r, ta, tb);
  const int kb_lo = split * P->kb / P->S;
  const int kb_hi = (split + 1) * P->kb / P->S;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGramStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  grid_dependency_wait();
  grid_dependency_trigger();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 4) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      for (int kb = kb_lo; kb < kb_hi; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, timeout_ns, abort_flag)) {
          give_up(abort_flag);
          break;
        }
        uint8_t* sa = smem + stage * kGramStageBytes;
        mbar_arrive_expect_tx(&full[stage], kGramStageBytes);
        tma_load_2d(sa, &P->tm_a, &full[stage], kb * kBlockK, ta * kTileM, pol);
        tma_load_2d(sa + kTileABytes, &P->tm_a, &full[stage], kb * kBlockK, tb * kTileM, pol);
        ++issued;
        if (++stage == kGramStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      const long long first = issued > kGramStages ? issued - kGramStages : 0;
      for (long long j = first; j < issued; ++j)
        mbar_wait(&full[j % kGramStages], static_cast<uint32_t>((j / kGramStages) & 1),
                  kDrainTimeoutNs, nullptr);
    }
  } else if (warp == 5) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kTileM, kTileM);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, issued_any = false;
      for (int kb = kb_lo; kb < kb_hi; ++kb) {
        if (!mbar_wait(&full[stage], phase, timeout_ns, abort_flag)) {
          give_up(abort_flag);
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t a0 = smem_addr(smem + stage * kGramStageBytes);
        const uint32_t b0 = a0 + kTileABytes;
#pragma unroll
        for (int k = 0; k < kBlockK / 16; ++k)
          umma_bf16(tmem_base, sw128_kmajor_desc(a0 + k * 32), sw128_kmajor_desc(b0 + k * 32),
                    idesc, (kb == kb_lo && k == 0) ? 0u : 1u);
        issued_any = true;
        umma_commit(&empty[stage]);
        if (++stage == kGramStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok && issued_any) umma_commit(acc_full);
      if (issued_any) {
        umma_commit(drain);
        mbar_wait(drain, 0, kDrainTimeoutNs, nullptr);
      }
    }
  } else {
    const int row = threadIdx.x;
    if (mbar_wait(acc_full, 0, timeout_ns, abort_flag)) {
      tc_fence_after_sync();
      float* dst = P->partial + (static_cast<size_t>(job) * kTileM + row) * kTileM;
      for (int col = 0; col < kTileM; col += 32) {
        float acc[32];
        tmem_load_32cols(tmem_base + (static_cast<uint32_t>(warp * 32) << 16) + col, acc);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          *reinterpret_cast<float4*>(dst + col + q * 4) =
              make_float4(acc[q * 4], acc[q * 4 + 1], acc[q * 4 + 2], acc[q * 4 + 3]);
      }
    } else {
      give_up(abort_flag);
    }
  }

  __syncwarp();
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, 128);
  }
}

// Sums the K splits of every tile pair in split order, scales by s/2, splits
// the fp32 value into bf16 hi + lo and writes G'[i][j] (and the mirrored
// G'[j][i] off the diagonal).
template <bool kGrouped>
__global__ void __launch_bounds__(256)
    gram_reduce_kernel(const __grid_constant__ GramProblemDev single,
                       const GramProblemDev* __restrict__ table) {
  // Let the norm GEMM launch now: its W0 k-blocks need nothing from the Gram,
  // and it waits for this grid before it reads G' or the arrival counters.
  grid_dependency_trigger();
  grid_dependency_wait();
  const GramProblemDev* P = kGrouped ? &table[blockIdx.z] : &single;
  if (blockIdx.x == 0 && blockIdx.y == 0)
    for (int k = threadIdx.x; k < P->cnt_len; k += blockDim.x) P->tile_cnt[k] = 0;
  const int pair = blockIdx.y;
  if (pair >= P->pairs) return;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;  // element of the 128x128 tile
  const int i = e / kTileM, j = e % kTileM;
  int ta, tb;
  gram_pair(pair, P->tiles_r, ta, tb);
  const int gi = ta * kTileM + i, gj = tb * kTileM + j;
  if (gi >= P->r || gj >= P->r) return;
  const float* src = P->partial + static_cast<size_t>(pair) * P->S * kTileM * kTileM + e;
  float sum = 0.f;
  for (int s = 0; s < P->S; ++s) sum += src[static_cast<size_t>(s) * kTileM * kTileM];
  const float x = P->half_s * sum;
  const uint16_t hi = f32_to_bf16_rn(x);
  const uint16_t lo = f32_to_bf16_rn(x - __uint_as_float(static_cast<uint32_t>(hi) << 16));
  P->g_out[static_cast<size_t>(gi) * P->r8 + gj] = hi;
  P->g_lo[static_cast<size_t>(gi) * P->r8 + gj] = lo;
  if (ta != tb) {
    P->g_out[static_cast<size_t>(gj) * P->r8 + gi] = hi;
    P->g_lo[static_cast<size_t>(gj) * P->r8 + gi] = lo;
  }
}

}  // namespace dora
