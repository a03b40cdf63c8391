// Merged DoRA weight W' = g (W0 + s B A), g = m / max(n, eps), for inference
// without the adapter branch ("LoRA & DoRA: The Math, Memory, and
// Trade-offs", section 6: the trained magnitude and direction fold into one
// dense weight; "Scaling DoRA ...", section 4 precision bullet for g).  n is
// the row norm the norm kernels produce; the merge does not recompute it.
//
// Two kernels:
//   transpose_bf16_kernel  A [r, d_in] -> A^T [d_in, r8] in the workspace, so
//                          that both MMA operands are K-major (K = r).
//   merge_kernel           persistent, one CTA per SM over 128 x 256 tiles of
//                          W' in row-major order.  Per tile the tensor cores
//                          form acc = B_tile A^T_tile over K = r into a
//                          256-column TMEM accumulator: one N = 256 MMA per 16
//                          of K, since MMAs that accumulate into one
//                          accumulator run one after another at a fixed cost
//                          each, whatever their N.  Eight epilogue warps read
//                          the whole accumulator into registers and free it at
//                          once (the next tile's MMAs then overlap the rest of
//                          the epilogue), read the W0 tile (staged by TMA in
//                          one of two shared buffers), write g_i (W0_ij +
//                          s acc_ij) rounded once to bf16 over it in place,
//                          and store their sub-boxes with TMA.  The CTA keeps
//                          its row block's B tile (128 x r) resident in TMEM
//                          -- copied there once per row block (tcgen05.cp) and
//                          used as the MMAs' A operand -- while it walks that
//                          block's column tiles, so only A^T streams through
//                          the shared-memory k-block stages.
// HBM-bound: W0 is read once and W' written once (2 x 2 bytes per element);
// the 2 d_out d_in r MMA FLOPs overlap with that traffic.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace dora {

constexpr int kMergeM = 128;        // rows of W' per tile (TMEM lanes)
constexpr int kMergeN = 256;        // columns of W' per tile (accumulator columns)
constexpr int kMergeK = 64;         // r per k-block: one 128-byte swizzle row
constexpr int kMergeEpiWarps = 8;   // two per TMEM lane quadrant, each half of the columns
constexpr int kMergeThreads = (kMergeEpiWarps + 2) * 32;  // + warp 8 TMA, warp 9 MMA
constexpr int kMergeMaxRegs = 168;  // 10 warps are charged as 12: 65536 / 384 -> 168
constexpr int kMergeMaxStages = 4;
constexpr int kMergeWBufs = 2;
constexpr uint32_t kMergeTmemCols = 512;   // the accumulator + B (r / 2 columns)
constexpr uint32_t kMergeTmemB = kMergeN;  // first TMEM column of the resident B tile
constexpr uint32_t kMergeStageBytes = kMergeN * kMergeK * 2;    // 32 KiB: A^T (or B) k-block
constexpr uint32_t kMergeBBytes = kMergeM * kMergeK * 2;        // 16 KiB: B k-block
constexpr uint32_t kMergeTileBytes = kMergeM * kMergeN * 2;     // 64 KiB: W0 in, W' out
constexpr uint32_t kMergeBoxBytes = kMergeM * 64 * 2;           // 16 KiB: one 64-column box

struct alignas(64) MergeDev {
  CUtensorMap tm_w0;   // W0 [d_out, d_in], box 64 x 128 (load)
  CUtensorMap tm_out;  // W' [d_out, d_in], box 64 x 32 (store: one epilogue warp's rows)
  CUtensorMap tm_b;    // B  [d_out, r],    box 64 x 128
  CUtensorMap tm_at;   // A^T [d_in, r],    box 64 x 256
  const float* m;
  const float* n;
  float s, eps;
  int d_out, d_in, r;
  int kb;              // k-blocks over r
  int tiles_n, tiles;  // column tiles per row block, all tiles
  uint32_t idesc;
};

struct MergeSmemTail {
  uint64_t full[kMergeMaxStages];   // k-block landed (B when a row block starts, else A^T)
  uint64_t empty[kMergeMaxStages];  // copy or MMAs done with the k-block
  uint64_t b_swap;                  // every MMA reading the resident B tile has completed
  uint64_t w_full[kMergeWBufs], w_empty[kMergeWBufs];  // W0 landed / W' stored out
  uint64_t acc_full, acc_empty;
  uint64_t drain;
  uint32_t tmem_slot;
  int abort_flag;
};

__device__ __forceinline__ void merge_give_up(volatile int* abort_flag) {
  *abort_flag = 1;
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

__global__ void __maxnreg__(kMergeMaxRegs)
    merge_kernel(const __grid_constant__ MergeDev P, int stages,
                 unsigned long long timeout_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* s_w = smem;                                  // 2 x 64 KiB W0 / W' tiles
  uint8_t* s_at = s_w + kMergeWBufs * kMergeTileBytes;  // stages x 32 KiB A^T (or B)
  MergeSmemTail* tail = reinterpret_cast<MergeSmemTail*>(s_at + stages * kMergeStageBytes);
  volatile int* abort_flag = &tail->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int C = gridDim.x;
  const int t_begin = static_cast<int>(static_cast<long long>(blockIdx.x) * P.tiles / C);
  const int t_end = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * P.tiles / C);

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
    mbar_init(&tail->acc_empty, kMergeEpiWarps);
    mbar_init(&tail->drain, 1);
    tail->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tail->tmem_slot, kMergeTmemCols);
    tmem_relinquish();
  }
  if (warp == kMergeEpiWarps && lane == 0) {
    prefetch_tmap(&P.tm_w0);
    prefetch_tmap(&P.tm_out);
    prefetch_tmap(&P.tm_b);
    prefetch_tmap(&P.tm_at);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = tail->tmem_slot;
  // A^T is written by the transpose that precedes this kernel.
  grid_dependency_wait();
  grid_dependency_trigger();

  if (warp == kMergeEpiWarps) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && t_begin < t_end) {
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_last();
      int stage = 0, cur_tm = -1;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      // One k-block (bytes: 16 KiB of B or 32 KiB of A^T) into the next stage.
      auto load_kblock = [&](const CUtensorMap* map, int kx, int row, uint32_t bytes) -> bool {
        if (!mbar_wait(&tail->empty[stage], phase ^ 1u, timeout_ns, abort_flag)) {
          merge_give_up(abort_flag);
          return false;
        }
        mbar_arrive_expect_tx(&tail->full[stage], bytes);
        tma_load_2d(s_at + stage * kMergeStageBytes, map, &tail->full[stage], kx, row, pol_keep);
        ++issued;
        if (++stage == stages) {
          stage = 0;
          phase ^= 1u;
        }
        return true;
      };
      for (int t = t_begin, it = 0; ok && t < t_end; ++t, ++it) {
        const int tm = t / P.tiles_n, tn = t % P.tiles_n;
        if (tm != cur_tm) {  // the row block's B tile, to be copied into TMEM
          for (int k = 0; ok && k < P.kb; ++k)
            ok = load_kblock(&P.tm_b, k * kMergeK, tm * kMergeM, kMergeBBytes);
          cur_tm = tm;
        }
        const int wb = it % kMergeWBufs;
        if (!ok || !mbar_wait(&tail->w_empty[wb],
                              static_cast<uint32_t>(((it / kMergeWBufs) & 1) ^ 1), timeout_ns,
                              abort_flag)) {
          merge_give_up(abort_flag);
          break;
        }
        mbar_arrive_expect_tx(&tail->w_full[wb], kMergeTileBytes);
        for (int h = 0; h < kMergeN / 64; ++h)
          tma_load_2d(s_w + wb * kMergeTileBytes + h * kMergeBoxBytes, &P.tm_w0, &tail->w_full[wb],
                      tn * kMergeN + h * 64, tm * kMergeM, pol_stream);
        for (int k = 0; ok && k < P.kb; ++k)
          ok = load_kblock(&P.tm_at, k * kMergeK, tn * kMergeN, kMergeStageBytes);
      }
      // Let every operand copy already issued land before the block can exit.
      const long long first = issued > stages ? issued - stages : 0;
      for (long long j = first; j < issued; ++j)
        mbar_wait(&tail->full[j % stages], static_cast<uint32_t>((j / stages) & 1),
                  kDrainTimeoutNs, nullptr);
    }
  } else if (warp == kMergeEpiWarps + 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && t_begin < t_end) {
      int stage = 0, cur_tm = -1, swaps = 0;
      uint32_t phase = 0;
      bool issued_any = false, ok = true;
      const uint32_t b_tmem = tmem_base + kMergeTmemB;
      for (int t = t_begin, it = 0; ok && t < t_end; ++t, ++it) {
        const int tm = t / P.tiles_n;
        if (tm != cur_tm) {
          // Overwrite the resident B tile only once every MMA reading it is done.
          if (issued_any) {
            umma_commit(&tail->b_swap);
            if (!mbar_wait(&tail->b_swap, static_cast<uint32_t>(swaps & 1), timeout_ns,
                           abort_flag)) {
              merge_give_up(abort_flag);
              break;
            }
            ++swaps;
            tc_fence_after_sync();
          }
          for (int k = 0; k < P.kb; ++k) {
            if (!mbar_wait(&tail->full[stage], phase, timeout_ns, abort_flag)) {
              merge_give_up(abort_flag);
              ok = false;
              break;
            }
            tc_fence_after_sync();
            const uint32_t b0 = smem_addr(s_at + stage * kMergeStageBytes);
#pragma unroll
            for (int kk = 0; kk < kMergeK / 16; ++kk)
              tmem_copy_128x32B(b_tmem + static_cast<uint32_t>(k * 32 + kk * 8),
                                sw128_kmajor_desc(b0 + kk * 32));
            umma_commit(&tail->empty[stage]);
            if (++stage == stages) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          cur_tm = tm;
        }
        // The accumulator is free once the epilogue has read it out.
        if (!mbar_wait(&tail->acc_empty, static_cast<uint32_t>((it & 1) ^ 1), timeout_ns,
                       abort_flag)) {
          merge_give_up(abort_flag);
          break;
        }
        tc_fence_after_sync();
        for (int k = 0; k < P.kb; ++k) {
          if (!mbar_wait(&tail->full[stage], phase, timeout_ns, abort_flag)) {
            merge_give_up(abort_flag);
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t b0 = smem_addr(s_at + stage * kMergeStageBytes);
#pragma unroll
          for (int kk = 0; kk < kMergeK / 16; ++kk)
            umma_bf16_tmem_a(tmem_base, b_tmem + static_cast<uint32_t>(k * 32 + kk * 8),
                             sw128_kmajor_desc(b0 + kk * 32), P.idesc,
                             (k > 0 || kk > 0) ? 1u : 0u);
          issued_any = true;
          umma_commit(&tail->empty[stage]);
          if (++stage == stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tail->acc_full);
      }
      if (issued_any) {
        umma_commit(&tail->drain);
        mbar_wait(&tail->drain, 0, kDrainTimeoutNs, nullptr);
      }
    }
  } else {
    // ------------------------------------------------ epilogue (warps 0-7)
    // Warp w: TMEM lanes 32 (w % 4) .. + 31 (its rows) and the 128 columns of
    // boxes 2 (w / 4) and 2 (w / 4) + 1.  It reads its 128 accumulator
    // columns into registers and frees the accumulator, then reads the rows'
    // W0 values from the 128-byte-swizzled staging buffer, writes W' over them
    // and stores its two 32 x 64 sub-boxes with TMA.  At its next tile's start
    // it hands the previous staging buffer back once those stores have read it.
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const int half = warp >> 2;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    int g_tm = -1, prev_wb = -1;
    float g = 0.f;
    for (int t = t_begin, it = 0; t < t_end; ++t, ++it) {
      const int tm = t / P.tiles_n, tn = t % P.tiles_n;
      const int wb = it % kMergeWBufs;
      if (lane == 0 && prev_wb >= 0) {
        bulk_wait_group_read0();
        mbar_arrive(&tail->w_empty[prev_wb]);
      }
      prev_wb = -1;
      if (tm != g_tm) {
        const int grow = tm * kMergeM + row;
        g = grow < P.d_out ? __fdiv_rn(__ldg(P.m + grow), fmaxf(__ldg(P.n + grow), P.eps)) : 0.f;
        g_tm = tm;
      }
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&tail->acc_full, static_cast<uint32_t>(it & 1), timeout_ns,
                                abort_flag))) {
        merge_give_up(abort_flag);
        break;
      }
      tc_fence_after_sync();
      float acc[4][32];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        tmem_load_32cols(tmem_base + lane_base + static_cast<uint32_t>(half * 128 + j * 32), acc[j]);
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tail->acc_empty);
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&tail->w_full[wb], static_cast<uint32_t>((it / kMergeWBufs) & 1),
                                timeout_ns, abort_flag))) {
        merge_give_up(abort_flag);
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
                       tn * kMergeN + (half * 2 + h) * 64, tm * kMergeM + quad * 32);
        bulk_commit_group();
      }
      prev_wb = wb;
    }
    if (lane == 0) bulk_wait_group0();
  }

  __syncwarp();
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, kMergeTmemCols);
  }
}

}  // namespace dora
