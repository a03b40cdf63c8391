// Merged DoRA weight W' = g (W0 + s B A), g = m / max(n, eps), for inference
// without the adapter branch ("LoRA & DoRA: The Math, Memory, and
// Trade-offs", section 6: the trained magnitude and direction fold into one
// dense weight; "Scaling DoRA ...", section 4 precision bullet for g).  n is
// the row norm the norm kernels produce; the merge does not recompute it.
//
// Two kernels:
//   transpose_bf16_kernel  A [r, d_in] -> A^T [d_in, r8] in the workspace, so
//                          that both MMA operands are K-major (K = r).
//   merge_kernel           persistent, on CTA pairs, over 256 x 256 tiles of
//                          W' in row-major order.  Per tile the tensor cores
//                          form acc = B_tile A^T_tile over K = r into a
//                          256-column TMEM accumulator of each CTA (its 128
//                          rows): one M = 256, N = 256 MMA per 16 of K,
//                          issued by rank 0 for both.  Eight epilogue warps
//                          per CTA read the whole accumulator into registers
//                          and free it at once (the next tile's MMAs then
//                          overlap the rest of the epilogue), read the W0
//                          tile (staged by TMA in one of two shared buffers),
//                          write g_i (W0_ij + s acc_ij) rounded once to bf16
//                          over it in place, and store their sub-boxes with
//                          TMA.  Each CTA keeps its rows of the row block's B
//                          tile (128 x r) resident in TMEM -- copied there
//                          once per row block (tcgen05.cp) and used as the
//                          MMAs' A operand -- while the pair walks that
//                          block's column tiles, so only A^T streams through
//                          the shared-memory k-block stages, each CTA staging
//                          half of it: 96 KiB of A^T per 64 KiB of W0 at
//                          r = 384, where a single CTA on 128 x 256 tiles
//                          would stage 192 KiB.
// HBM-bound: W0 is read once and W' written once (2 x 2 bytes per element);
// the 2 d_out d_in r MMA FLOPs overlap with that traffic.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace dora {

constexpr int kMergeM = 128;        // rows of W' per CTA (TMEM lanes)
constexpr int kMergePairM = 256;    // rows of W' per tile: a pair of CTAs
constexpr int kMergeN = 256;        // columns of W' per tile (accumulator columns)
constexpr int kMergeK = 64;         // r per k-block: one 128-byte swizzle row
constexpr int kMergeEpiWarps = 8;   // two per TMEM lane quadrant, each half of the columns
// + warp 8 (A^T / B copies), warp 9 (MMA), warp 10 (W0 copies)
constexpr int kMergeThreads = (kMergeEpiWarps + 3) * 32;
constexpr int kMergeMaxRegs = 168;  // 11 warps are charged as 12: 65536 / 384 -> 168
constexpr int kMergeMaxStages = 6;
constexpr int kMergeWBufs = 2;
constexpr uint32_t kMergeTmemCols = 512;   // the accumulator + B (r / 2 columns)
constexpr uint32_t kMergeTmemB = kMergeN;  // first TMEM column of the resident B tile
// One k-block stage of a CTA: its half (128 columns of W') of an A^T
// k-block, or its 128 rows of a B k-block.
constexpr uint32_t kMergeStageBytes = kMergeM * kMergeK * 2;    // 16 KiB
constexpr uint32_t kMergeTileBytes = kMergeM * kMergeN * 2;     // 64 KiB: W0 in, W' out
constexpr uint32_t kMergeBoxBytes = kMergeM * 64 * 2;           // 16 KiB: one 64-column box

struct alignas(64) MergeDev {
  CUtensorMap tm_w0;   // W0 [d_out, d_in], box 64 x 128 (load)
  CUtensorMap tm_out;  // W' [d_out, d_in], box 64 x 32 (store: one epilogue warp's rows)
  CUtensorMap tm_b;    // B  [d_out, r],    box 64 x 128
  CUtensorMap tm_at;   // A^T [d_in, r],    box 64 x 128
  const float* m;
  const float* n;
  float s, eps;
  int d_out, d_in, r;
  int kb;              // k-blocks over r
  int tiles_n, tiles;  // column tiles per 256-row block, all tiles
  uint32_t idesc;
};

// Barriers (per CTA, same offsets in both CTAs of a pair):
//   full[s]    rank 0 only: its producer's expected bytes plus both CTAs'
//              copies of k-block stage s (rank 1's copies signal rank 0's).
//   empty[s]   both: rank 0's commit after the copies or MMAs reading stage s.
//   b_swap     rank 0: every MMA reading the resident B tiles has completed.
//   w_full[b], w_empty[b]  both, local: W0 tile landed / W' stores read it.
//   acc_full   both: rank 0's commit after a tile's MMAs.
//   acc_empty  rank 0: one arrival per epilogue warp of both CTAs.
//   drain      rank 0: the last MMAs have completed.
struct MergeSmemTail {
  uint64_t full[kMergeMaxStages];
  uint64_t empty[kMergeMaxStages];
  uint64_t b_swap;
  uint64_t w_full[kMergeWBufs], w_empty[kMergeWBufs];
  uint64_t acc_full, acc_empty;
  uint64_t drain;
  uint32_t tmem_slot;
  int abort_flag;
};

// Sets this CTA's and the peer's abort flags and records the timeout.
__device__ __forceinline__ void merge_give_up(volatile int* abort_flag, uint32_t peer_flag) {
  *abort_flag = 1;
  st_cluster_u32(peer_flag, 1u);
  record_error(DORA_ERR_TIMEOUT);
}

// At[j][k] = A[k][j]: 32 x 32 tiles through shared memory, block (32, 8).
__global__ void __launch_bounds__(256)
    transpose_bf16_kernel(const uint16_t* __restrict__ A, int rows, int cols,
                          uint16_t* __restrict__ At, int ld_at) {
  __shared__ uint16_t tile[32][33];
  grid_dependency_wait();
  grid_dependency_trigger();
  const int x = blockIdx.x * 32 + threadIdx.x;  // column of A
  const int y = blockIdx.y * 32 + threadIdx.y;  // row of A
#pragma unroll
  for (int j = 0; j < 32; j += 8)
    if (x < cols && y + j < rows)
      tile[threadIdx.y + j][threadIdx.x] = A[static_cast<size_t>(y + j) * cols + x];
  __syncthreads();
  const int tx = blockIdx.y * 32 + threadIdx.x;  // column of At (= row of A)
  const int ty = blockIdx.x * 32 + threadIdx.y;  // row of At (= column of A)
#pragma unroll
  for (int j = 0; j < 32; j += 8)
    if (tx < rows && ty + j < cols)
      At[static_cast<size_t>(ty + j) * ld_at + tx] = tile[threadIdx.x][threadIdx.y + j];
}

__global__ void __cluster_dims__(2, 1, 1) __maxnreg__(kMergeMaxRegs)
    merge_kernel(const __grid_constant__ MergeDev P, int stages,
                 unsigned long long timeout_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* s_w = smem;                                  // 2 x 64 KiB W0 / W' tiles
  uint8_t* s_at = s_w + kMergeWBufs * kMergeTileBytes;  // stages x 16 KiB A^T (or B)
  MergeSmemTail* tail = reinterpret_cast<MergeSmemTail*>(s_at + stages * kMergeStageBytes);
  volatile int* abort_flag = &tail->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer_abort = mapa_shared(smem_addr(&tail->abort_flag), rank ^ 1u);
  // A pair of CTAs owns a 256-row tile of W': this CTA its rows
  // [128 rank, 128 rank + 128), half of each A^T k-block (columns
  // [128 rank, 128 rank + 128) of the tile) and its rows of B.
  const int pairs = static_cast<int>(gridDim.x >> 1);
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int t_begin = static_cast<int>(static_cast<long long>(pair) * P.tiles / pairs);
  const int t_end = static_cast<int>(static_cast<long long>(pair + 1) * P.tiles / pairs);
  const int row_off = static_cast<int>(rank) * kMergeM;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&tail->full[s], 1);
      mbar_init(&tail->empty[s], 1);
    }
    mbar_init(&tail->b_swap, 1);
    for (int b = 0; b < kMergeWBufs; ++b) {
      mbar_init(&tail->w_full[b], 1);
      mbar_init(&tail->w_empty[b], kMergeEpiWarps);  // each warp's stores have read its rows
    }
    mbar_init(&tail->acc_full, 1);
    mbar_init(&tail->acc_empty, 2 * kMergeEpiWarps);
    mbar_init(&tail->drain, 1);
    tail->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(&tail->tmem_slot, kMergeTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == kMergeEpiWarps && lane == 0) {
    prefetch_tmap(&P.tm_w0);
    prefetch_tmap(&P.tm_out);
    prefetch_tmap(&P.tm_b);
    prefetch_tmap(&P.tm_at);
  }
  // Both CTAs' barriers are initialised (and their TMEM allocated) before
  // either CTA signals the other.
  tc_fence_before_sync();
  cluster_sync();
  tc_fence_after_sync();
  const uint32_t tmem_base = tail->tmem_slot;
  // A^T is written by the transpose that precedes this kernel: only its
  // copies wait for that grid (the transpose itself waited for every kernel
  // before it, so W0, B, m and n are complete), and the next kernel may
  // launch now.
  grid_dependency_trigger();

  if (warp == kMergeEpiWarps) {
    // ------------------------------------------------- A^T / B copy producer
    // (the W0 tiles have a warp of their own, so that a k-block copy never
    // waits for a staging buffer to come free)
    if (lane == 0 && t_begin < t_end) {
      const uint64_t pol_keep = policy_evict_last();
      const uint32_t full0 = mapa_shared(smem_addr(&tail->full[0]), 0);  // rank 0's full[0]
      int stage = 0, cur_tm = -1;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      // This CTA's 16 KiB of one k-block into the next stage; both CTAs'
      // copies complete on rank 0's barrier.
      auto load_kblock = [&](const CUtensorMap* map, int kx, int row) -> bool {
        if (!mbar_wait(&tail->empty[stage], phase ^ 1u, timeout_ns, abort_flag)) {
          merge_give_up(abort_flag, peer_abort);
          return false;
        }
        if (rank == 0) mbar_arrive_expect_tx(&tail->full[stage], 2 * kMergeStageBytes);
        tma_load_2d_pair(s_at + stage * kMergeStageBytes, map,
                         full0 + stage * static_cast<uint32_t>(sizeof(uint64_t)), kx, row,
                         pol_keep);
        ++issued;
        if (++stage == stages) {
          stage = 0;
          phase ^= 1u;
        }
        return true;
      };
      bool at_ready = false;
      for (int t = t_begin; ok && t < t_end; ++t) {
        const int tm = t / P.tiles_n, tn = t % P.tiles_n;
        const int row0 = tm * kMergePairM + row_off;
        if (tm != cur_tm) {  // the row block's B tile, to be copied into TMEM
          for (int k = 0; ok && k < P.kb; ++k) ok = load_kblock(&P.tm_b, k * kMergeK, row0);
          cur_tm = tm;
        }
        if (!at_ready) {
          grid_dependency_wait();
          at_ready = true;
        }
        for (int k = 0; ok && k < P.kb; ++k)
          ok = load_kblock(&P.tm_at, k * kMergeK, tn * kMergeN + row_off);
      }
      // Let every operand copy already issued land before the block can exit:
      // rank 0 sees its full barriers complete; rank 1's copies complete on
      // rank 0's barriers, so it waits for its stages to be consumed.
      const long long first = issued > stages ? issued - stages : 0;
      for (long long j = first; j < issued; ++j) {
        const uint32_t par = static_cast<uint32_t>((j / stages) & 1);
        if (rank == 0)
          mbar_wait(&tail->full[j % stages], par, kDrainTimeoutNs, nullptr);
        else
          mbar_wait(&tail->empty[j % stages], par, kDrainTimeoutNs, nullptr);
      }
    }
  } else if (warp == kMergeEpiWarps + 2) {
    // ----------------------------------------------------- W0 copy producer
    // This CTA's rows of each tile's W0 into a staging buffer, as soon as
    // the W' stores of the tile it held have read it.
    if (lane == 0) {
      const uint64_t pol_stream = policy_evict_first();
      for (int t = t_begin, it = 0; t < t_end; ++t, ++it) {
        const int tm = t / P.tiles_n, tn = t % P.tiles_n;
        const int wb = it % kMergeWBufs;
        if (!mbar_wait(&tail->w_empty[wb], static_cast<uint32_t>(((it / kMergeWBufs) & 1) ^ 1),
                       timeout_ns, abort_flag)) {
          merge_give_up(abort_flag, peer_abort);
          break;
        }
        mbar_arrive_expect_tx(&tail->w_full[wb], kMergeTileBytes);
        for (int h = 0; h < kMergeN / 64; ++h)
          tma_load_2d(s_w + wb * kMergeTileBytes + h * kMergeBoxBytes, &P.tm_w0, &tail->w_full[wb],
                      tn * kMergeN + h * 64, tm * kMergePairM + row_off, pol_stream);
      }
    }
  } else if (warp == kMergeEpiWarps + 1) {
    // ------------------------------------------------------------ MMA issuer
    // Rank 0 issues for the pair: the copies of both CTAs' B rows into their
    // TMEM and one M = 256 MMA per 16 of K, whose A operand is that TMEM.
    if (lane == 0 && rank == 0 && t_begin < t_end) {
      int stage = 0, cur_tm = -1, swaps = 0;
      uint32_t phase = 0;
      bool issued_any = false, ok = true;
      const uint32_t b_tmem = tmem_base + kMergeTmemB;
      for (int t = t_begin, it = 0; ok && t < t_end; ++t, ++it) {
        const int tm = t / P.tiles_n;
        if (tm != cur_tm) {
          // Overwrite the resident B tiles only once every MMA reading them is done.
          if (issued_any) {
            umma_commit_pair(&tail->b_swap, 0x1);
            if (!mbar_wait(&tail->b_swap, static_cast<uint32_t>(swaps & 1), timeout_ns,
                           abort_flag)) {
              merge_give_up(abort_flag, peer_abort);
              break;
            }
            ++swaps;
            tc_fence_after_sync();
          }
          for (int k = 0; k < P.kb; ++k) {
            if (!mbar_wait(&tail->full[stage], phase, timeout_ns, abort_flag)) {
              merge_give_up(abort_flag, peer_abort);
              ok = false;
              break;
            }
            tc_fence_after_sync();
            const uint32_t b0 = smem_addr(s_at + stage * kMergeStageBytes);
#pragma unroll
            for (int kk = 0; kk < kMergeK / 16; ++kk)
              tmem_copy_128x32B_pair(b_tmem + static_cast<uint32_t>(k * 32 + kk * 8),
                                     sw128_kmajor_desc(b0 + kk * 32));
            umma_commit_pair(&tail->empty[stage], 0x3);
            if (++stage == stages) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          cur_tm = tm;
        }
        // The accumulator is free once both CTAs' epilogues have read it out.
        if (!mbar_wait(&tail->acc_empty, static_cast<uint32_t>((it & 1) ^ 1), timeout_ns,
                       abort_flag)) {
          merge_give_up(abort_flag, peer_abort);
          break;
        }
        tc_fence_after_sync();
        for (int k = 0; k < P.kb; ++k) {
          if (!mbar_wait(&tail->full[stage], phase, timeout_ns, abort_flag)) {
            merge_give_up(abort_flag, peer_abort);
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t b0 = smem_addr(s_at + stage * kMergeStageBytes);
#pragma unroll
          for (int kk = 0; kk < kMergeK / 16; ++kk)
            umma_bf16_pair_tmem_a(tmem_base, b_tmem + static_cast<uint32_t>(k * 32 + kk * 8),
                                  sw128_kmajor_desc(b0 + kk * 32), P.idesc,
                                  (k > 0 || kk > 0) ? 1u : 0u);
          issued_any = true;
          umma_commit_pair(&tail->empty[stage], 0x3);
          if (++stage == stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair(&tail->acc_full, 0x3);
      }
      if (issued_any) {
        umma_commit_pair(&tail->drain, 0x1);
        mbar_wait(&tail->drain, 0, kDrainTimeoutNs, nullptr);
      }
    }
  } else {
    // ------------------------------------------------ epilogue (warps 0-7)
    // Warp w: TMEM lanes 32 (w % 4) .. + 31 (its rows) and the 128 columns of
    // boxes 2 (w / 4) and 2 (w / 4) + 1.  It reads its 128 accumulator
    // columns into registers and frees the accumulator, then reads the rows'
    // W0 values from the 128-byte-swizzled staging buffer, writes W' over them
    // and stores its two 32 x 64 sub-boxes with TMA.  At its next tile, once
    // it has freed the accumulator, it hands the previous staging buffer back
    // when those stores have read it.
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const int half = warp >> 2;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t acc_empty0 = mapa_shared(smem_addr(&tail->acc_empty), 0);
    int g_tm = -1, prev_wb = -1;
    float g = 0.f;
    for (int t = t_begin, it = 0; t < t_end; ++t, ++it) {
      const int tm = t / P.tiles_n, tn = t % P.tiles_n;
      const int row0 = tm * kMergePairM + row_off;
      const int wb = it % kMergeWBufs;
      if (tm != g_tm) {
        const int grow = row0 + row;
        g = grow < P.d_out ? __fdiv_rn(__ldg(P.m + grow), fmaxf(__ldg(P.n + grow), P.eps)) : 0.f;
        g_tm = tm;
      }
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&tail->acc_full, static_cast<uint32_t>(it & 1), timeout_ns,
                                abort_flag))) {
        merge_give_up(abort_flag, peer_abort);
        break;
      }
      tc_fence_after_sync();
      float acc[4][32];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        tmem_load_32cols(tmem_base + lane_base + static_cast<uint32_t>(half * 128 + j * 32), acc[j]);
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(acc_empty0);
      // The previous tile's staging buffer goes back to the W0 copies once
      // its stores have read it (after the accumulator is released, so the
      // next tile's MMAs do not wait for this).
      if (lane == 0 && prev_wb >= 0) {
        bulk_wait_group_read0();
        mbar_arrive(&tail->w_empty[prev_wb]);
      }
      prev_wb = -1;
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&tail->w_full[wb], static_cast<uint32_t>((it / kMergeWBufs) & 1),
                                timeout_ns, abort_flag))) {
        merge_give_up(abort_flag, peer_abort);
        break;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        // chunk j: columns half * 128 + 32 j .. of the tile = box 2 half + j / 2,
        // 16-byte chunks 4 (j % 2) .. of the box's 128-byte row
        uint8_t* rowp = s_w + wb * kMergeTileBytes + (half * 2 + j / 2) * kMergeBoxBytes + row * 128;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int c = (j & 1) * 4 + q;
          uint4* p = reinterpret_cast<uint4*>(rowp + ((c ^ (row & 7)) << 4));
          const uint4 w = *p;
          const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float lo = g * fmaf(P.s, acc[j][q * 8 + 2 * e], bf16lo_to_f32(wv[e]));
            const float hi = g * fmaf(P.s, acc[j][q * 8 + 2 * e + 1], bf16hi_to_f32(wv[e]));
            o[e] = pack_bf16x2_rn(lo, hi);
          }
          *p = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        // rows 32 quad .. + 31 of boxes 2 half and 2 half + 1: 4 KiB each,
        // 1024-byte aligned, so the 128-byte swizzle pattern is the box's own
        for (int h = 0; h < 2; ++h)
          tma_store_2d(&P.tm_out,
                       s_w + wb * kMergeTileBytes + (half * 2 + h) * kMergeBoxBytes + quad * 32 * 128,
                       tn * kMergeN + (half * 2 + h) * 64, row0 + quad * 32);
        bulk_commit_group();
      }
      prev_wb = wb;
    }
    if (lane == 0) bulk_wait_group0();
  }

  // Neither CTA leaves (or frees TMEM) while the other may still signal it,
  // read its shared memory through the MMAs, or write its TMEM.
  __syncwarp();
  tc_fence_before_sync();
  cluster_sync();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem_base, kMergeTmemCols);
  }
}

}  // namespace dora
