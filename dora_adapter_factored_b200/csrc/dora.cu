// C ABI of the DoRA hot path (declared in include/dora.h).  Host code only:
// argument validation, tensor-map encoding, workspace carving and launches.
// The kernels live in the .cuh files included below (one translation unit).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "dora.h"
#include "common.cuh"
#include "compose.cuh"
#include "merge.cuh"
#include "norm_simt.cuh"
#include "norm_tc.cuh"

namespace dora {
namespace {

constexpr int kVersion = 100;  // 0.1.0
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;
constexpr int kMaxDevices = 64;

std::atomic<uint64_t> g_launches{0};
std::atomic<unsigned long long> g_timeout_ns{kDefaultTimeoutNs};

// One-shot timing events around the principal kernel of the next call.
thread_local cudaEvent_t t_ev_before = nullptr;
unsigned long long* g_trace = nullptr;  // optional norm-kernel trace (diagnostics)
thread_local cudaEvent_t t_ev_after = nullptr;

// While the stream is being captured into a graph, the events become event
// record nodes of the graph (so they time the kernel at each replay).
cudaError_t record_timing_event(cudaEvent_t ev, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    return cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal);
  return cudaEventRecord(ev, st);
}

struct TimedLaunch {
  cudaStream_t st;
  explicit TimedLaunch(cudaStream_t s) : st(s) {
    if (t_ev_before != nullptr) record_timing_event(t_ev_before, st);
  }
  ~TimedLaunch() {
    if (t_ev_after != nullptr) record_timing_event(t_ev_after, st);
    t_ev_before = t_ev_after = nullptr;
  }
};

struct DeviceInfo {
  bool init = false;
  bool supported = false;
  int sms = 0;
  bool attrs_set = false;
  int norm_pairs = 0;  // CTA pairs of the norm GEMM resident at once
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

// Current device's info; nullptr if the device cannot be queried.
const DeviceInfo* device_info() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.init) {
    int major = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return nullptr;
    d.supported = (major == 10);
    d.sms = sms;
    d.init = true;
  }
  return &d;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }
size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Whether [a, a + na) and [b, b + nb) share a byte; an absent (NULL) buffer
// overlaps nothing.
bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  if (a == nullptr || b == nullptr) return false;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// Launch with programmatic stream serialization: the kernel may start while
// its predecessor drains; every kernel of the library executes
// griddepcontrol.wait before it reads or writes anything a predecessor
// touches.  Most let their dependents launch only after that wait, so that a
// kernel's launch implies its predecessor's predecessor has completed; the
// Gram reduce lets the norm GEMM launch at once, which is safe because the
// GEMM waits for the reduce (hence for the Gram) before it touches their
// outputs.
// If the runtime rejects the programmatic attribute for this stream, the
// kernel is launched again without it (plain stream order).
thread_local char t_last_error[512] = "";
thread_local bool launch_failed = false;

void note_error(const char* where, cudaError_t e) {
  snprintf(t_last_error, sizeof(t_last_error), "%s: %s (%d)", where, cudaGetErrorString(e),
           static_cast<int>(e));
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    cfg.numAttrs = 0;
    e = cudaLaunchKernelEx(&cfg, kernel, args...);
    if (e != cudaSuccess) {
      // Describe the kernel that could not be launched.
      cudaFuncAttributes fa = {};
      cudaFuncGetAttributes(&fa, reinterpret_cast<const void*>(kernel));
      snprintf(t_last_error, sizeof(t_last_error),
               "launch of grid (%u,%u,%u) x block (%u,%u,%u), %zu B dynamic smem: %s (%d); "
               "kernel: %d regs, max %d threads/block, %zu B static smem, max %d B dynamic, "
               "%zu B local",
               grid.x, grid.y, grid.z, block.x, block.y, block.z, smem, cudaGetErrorString(e),
               static_cast<int>(e), fa.numRegs, fa.maxThreadsPerBlock, fa.sharedSizeBytes,
               fa.maxDynamicSharedSizeBytes, fa.localSizeBytes);
      cudaGetLastError();
      launch_failed = true;
    }
  }
  return e;
}

// The streaming kernels (the compose passes) keep many 16-byte global loads in
// flight per SM, and those need L1 capacity.  Without a stated preference a
// CTA may land on an SM still split for the shared-memory-heavy norm or merge
// kernel, with a small L1: the forward pass at [4096, 8192] then ran ~9 us
// (30 %) slower after a norm call than after another forward pass.  So each
// streaming kernel asks, once per device, for the smallest shared-memory
// split that still holds the kStreamCtasPerSm CTAs per SM it is built for
// (its static shared memory plus the per-block reserve, each) -- not simply
// the largest L1, which gave the backward pass's 8 KB reduction buffer a
// split with room for one CTA per SM (the [8192, 25600] backward went from
// 347 to 446 us).  It is a hint: if the runtime refuses it, the launch goes
// ahead without it.
void prefer_l1(const void* kernel) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return;
  }
  static std::mutex mu;
  static std::vector<std::pair<int, const void*>> done;
  std::lock_guard<std::mutex> lk(mu);
  const std::pair<int, const void*> key(dev, kernel);
  if (std::find(done.begin(), done.end(), key) != done.end()) return;
  cudaFuncAttributes fa = {};
  int sm_smem = 0, reserve = 0;
  if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess ||
      cudaDeviceGetAttribute(&sm_smem, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) !=
          cudaSuccess ||
      cudaDeviceGetAttribute(&reserve, cudaDevAttrReservedSharedMemoryPerBlock, dev) !=
          cudaSuccess ||
      sm_smem <= 0) {
    (void)cudaGetLastError();
    return;
  }
  const long long need = static_cast<long long>(kStreamCtasPerSm) *
                         (static_cast<long long>(fa.sharedSizeBytes) + reserve);
  const int percent =
      static_cast<int>(std::min<long long>(100, (100 * need + sm_smem - 1) / sm_smem));
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, percent) ==
      cudaSuccess)
    done.push_back(key);
  else
    (void)cudaGetLastError();
}

template <typename... KArgs, typename... Args>
cudaError_t launch_stream(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t st, Args&&... args) {
  prefer_l1(reinterpret_cast<const void*>(kernel));
  return launch_pdl(kernel, grid, block, smem, st, std::forward<Args>(args)...);
}

dora_status_t launch_status() {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  const cudaError_t e = cudaGetLastError();
  if (launch_failed) {
    launch_failed = false;  // the launch helper already described it
    return DORA_ERR_CUDA;
  }
  if (e == cudaSuccess) return DORA_OK;
  note_error("kernel launch", e);
  return DORA_ERR_CUDA;
}

// ------------------------------------------------------------ tensor maps

PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// The N-side slab of a CTA pair: a row-major bf16 matrix of exactly 4 h rows
// (two accumulator chunks of 2 h rows, each split between the two CTAs)
// viewed as 4-D {cols, h, rank, chunk}; one box {box_cols, h, 1, 2} at
// (x, 0, rank, 0) brings a CTA its h rows of both chunks (128-byte swizzle).
bool make_tmap_bf16_pairslab(CUtensorMap* map, const void* ptr, uint64_t h, uint64_t cols,
                             uint64_t ld, uint32_t box_cols) {
  auto enc = tmap_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[4] = {cols, h, 2, 2};
  cuuint64_t strides[3] = {ld * 2, h * ld * 2, 2 * h * ld * 2};
  cuuint32_t box[4] = {box_cols, static_cast<cuuint32_t>(h), 1, 2};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// `parts` stacked row-major bf16 matrices [rows, cols] (`ld` elements per
// row, rows x ld per part) as {cols, rows, parts}, loaded in boxes of
// box_cols x box_rows x 1 with 128-byte swizzle; out-of-range elements read
// as zero.
bool make_tmap_bf16_parts(CUtensorMap* map, const void* ptr, uint64_t rows, uint64_t cols,
                          uint64_t ld, uint64_t parts, uint32_t box_cols, uint32_t box_rows) {
  auto enc = tmap_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {cols, rows, parts};
  cuuint64_t strides[2] = {ld * 2, rows * ld * 2};
  cuuint32_t box[3] = {box_cols, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The pair-slab view of `parts` stacked [4 h, cols] matrices: {cols, h, 2, 2,
// parts}, box {box_cols, h, 1, 2, 1} (one CTA's halves of both chunks).
bool make_tmap_bf16_pairslab_parts(CUtensorMap* map, const void* ptr, uint64_t h, uint64_t cols,
                                   uint64_t ld, uint64_t parts, uint32_t box_cols) {
  auto enc = tmap_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[5] = {cols, h, 2, 2, parts};
  cuuint64_t strides[4] = {ld * 2, h * ld * 2, 2 * h * ld * 2, 4 * h * ld * 2};
  cuuint32_t box[5] = {box_cols, static_cast<cuuint32_t>(h), 1, 2, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// `parts` stacked [rows, cols] bf16 matrices (ld elements per row) as the
// destination of 32 x 32 tiled stores from shared memory staged in the
// 64-byte swizzle; elements past rows or cols are not written.
bool make_tmap_bf16_store32(CUtensorMap* map, void* ptr, uint64_t rows, uint64_t cols, uint64_t ld,
                            uint64_t parts) {
  auto enc = tmap_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {cols, rows, parts};
  cuuint64_t strides[2] = {ld * 2, rows * ld * 2};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, ptr, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row-major bf16 matrix [rows, cols] with `ld` elements per row, loaded in
// boxes of box_cols x box_rows with 128-byte swizzle; out-of-range elements
// read as zero.
bool make_tmap_bf16(CUtensorMap* map, const void* ptr, uint64_t rows, uint64_t cols, uint64_t ld,
                    uint32_t box_cols, uint32_t box_rows) {
  auto enc = tmap_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------ norm planning

struct ModulePlan {
  // N side (pair MMA chunks; each CTA stages h0 rows of each)
  int n_pad, n0, n1, h0, tmem_cols;
  uint32_t b_region;
  // K and tiles (tiles of 256 rows; Gram pseudo-tiles of 256 rows of A)
  int kb_w, kb_r, tiles, pg_tiles, r8;
  // Gram blocks: nc columns of G each (gchunks MMA chunks of gn), gj0 of
  // them for pseudo-tile 0; d_in is split into gkp parts (a job per block
  // and part), and a job costs `gram_cost` W0 units in the schedule
  int nc, gchunks, gn, gj0, gblocks, gkp, gram_cost;
  long long units[3];  // Gram jobs, W0 units and G units (all of them)
  // the pool: tiles [dyn_t0, tiles) go chunk by chunk (cpt chunks each), the
  // others are split statically; every tile's G units are pool items
  int dyn_t0, cpt, gpi, gipt;  // gpi parts of S per G item, gipt G items per tile
  long long dyn_begin, g_item_begin;  // first W0-chunk item / G item in the wave's pool
  // workspace (byte offsets from the workspace base) and counters (ints
  // from the start of the counter block)
  size_t off_g, off_np, off_tw, cnt_off;
};

// One accumulator chunk up to N = 256, else two equal chunks; each chunk's
// slab rows are split evenly between the two CTAs in 8-row swizzle groups.
void plan_n_side(int r, ModulePlan& p) {
  if (r <= 256) {
    p.n_pad = round_up_int(r, 16);
    p.n0 = p.n_pad;
    p.n1 = 0;
  } else {
    p.n_pad = round_up_int(r, 32);
    p.n0 = p.n1 = p.n_pad / 2;
  }
  p.h0 = p.n0 / 2;
  p.b_region = static_cast<uint32_t>(p.n_pad / 2 * 128);
  int tc = 32;
  while (tc < p.n_pad) tc <<= 1;
  p.tmem_cols = tc;
}

// What a Gram job costs in W0 units of its module: a k-block stages
// 256 + nc rows of A against 256 + n_pad rows (W0 and A) for a W0 unit, and
// the feed of a CTA's stages sets the pace; plus the job's epilogue.
constexpr int kGramJobCharge = 3;
constexpr int kMaxGramParts = 16;

// Splits d_in into kp parts: kp jobs per Gram block, and the G units run
// over every part of S.
// G items of at least kMinGItemKb k-blocks: one per part of S, parts grouped
// where a part has fewer (each pool item costs an epilogue and a hand-over).
constexpr int kMinGItemKb = 8;

void set_gram_split(ModulePlan& p, int kp) {
  p.gkp = kp;
  p.gpi = std::min(kp, std::max(1, (kMinGItemKb + 2 * p.kb_r - 1) / (2 * p.kb_r)));
  p.gipt = (kp + p.gpi - 1) / p.gpi;
  p.units[kPhaseGram] = static_cast<long long>(p.gblocks) * kp;
  p.units[kPhaseG] = static_cast<long long>(p.tiles) * 2 * p.kb_r * kp;
  p.gram_cost = static_cast<int>(
      ceil_div_ll(ceil_div_ll(p.kb_w, kp) * (256 + p.nc), 256 + p.n_pad) + kGramJobCharge);
}

void plan_module(int64_t d_out, int64_t d_in, int64_t r, bool wide_gram, ModulePlan& p) {
  plan_n_side(static_cast<int>(r), p);
  p.kb_w = static_cast<int>(ceil_div_ll(d_in, kBlockK));
  p.kb_r = static_cast<int>(ceil_div_ll(r, kBlockK));
  p.tiles = static_cast<int>(ceil_div_ll(d_out, kPairM));
  p.pg_tiles = static_cast<int>(ceil_div_ll(r, kPairM));
  p.r8 = round_up_int(static_cast<int>(r), 8);
  // Gram blocks.  A single module: blocks of up to 128 columns, one chunk
  // (one MMA issuer).  At r = 384 that is five blocks (two on the first
  // pseudo-tile, three on the second) where 256-column blocks made three: a
  // job's k-block stages 24 KiB instead of 32, the second pseudo-tile's
  // padded rows cost 128-column blocks instead of 256, and the jobs spread
  // over more pairs, so S is written sooner (headline: by ~32 us of the call
  // against ~40 us, the kernel 60 us against 64 us).  Several modules
  // (`wide_gram`): 256-column blocks as two chunks of 128 (one per MMA
  // issuer) where the slab region holds them -- a layer's nine modules would
  // otherwise make 45 jobs of its 74 pairs, leaving the static W0 units to
  // the other 29 (the 56-module stack took ~1680-1770 us against ~1640).
  if (wide_gram && p.n_pad >= 2 * kGramCols) {
    p.nc = 2 * kGramCols;
    p.gchunks = 2;
  } else {
    p.nc = std::min(kGramCols, p.n_pad);
    p.gchunks = 1;
  }
  p.gn = p.nc / p.gchunks;
  p.gj0 = gram_jobs_of_tile(static_cast<int>(r), p.nc, 0);
  p.gblocks = p.gj0 + (p.pg_tiles > 1 ? gram_jobs_of_tile(static_cast<int>(r), p.nc, 1) : 0);
  p.units[kPhaseW0] = static_cast<long long>(p.tiles) * p.kb_w;
  set_gram_split(p, 1);
  p.dyn_t0 = p.tiles;
  p.cpt = std::max(1, (p.kb_w + kChunkKb - 1) / kChunkKb);
  p.dyn_begin = p.g_item_begin = 0;
}

int module_counters(const ModulePlan& p) { return p.tiles * 2 + 1; }

// Re-read operands (A and S) of one wave of the grouped norm: well inside
// the 126 MB L2, which also carries the W0 stream.
constexpr size_t kWaveBudgetBytes = size_t(40) << 20;

// The static W0 units of a module (its tiles before the pool's).
long long static_w0(const ModulePlan& p) { return static_cast<long long>(p.dyn_t0) * p.kb_w; }

// Runs of equal Gram-job cost of modules [m0, m1), in order.
int gram_runs(const std::vector<ModulePlan>& plans, int m0, int m1) {
  int runs = 0, last = -1;
  for (int i = m0; i < m1; ++i) {
    if (plans[i].units[kPhaseGram] == 0) continue;
    if (plans[i].gram_cost != last) ++runs;
    last = plans[i].gram_cost;
  }
  return runs;
}

// Splits the modules, in order, into waves: a wave closes before a module
// that would take its re-read operands (A, S_hi, S_lo) past the budget,
// provided it already holds at least `min_w` W0 units, and before one that
// would give its Gram jobs more than kMaxGramRuns runs of equal cost; a last
// wave with fewer W0 units joins the one before where it can.  The budget
// is `budget` evened out over the waves it takes, so that no wave is left
// with a small remainder.  Returns the waves' first modules (and the module
// count at the end).
std::vector<int> plan_waves(const std::vector<ModulePlan>& plans, const int64_t* d_in,
                            const int64_t* r, long long min_w, size_t budget) {
  const int count = static_cast<int>(plans.size());
  std::vector<size_t> mbytes(count);
  size_t total = 0, largest = 0;
  for (int i = 0; i < count; ++i) {
    mbytes[i] = static_cast<size_t>(r[i]) * d_in[i] * 2 +
                2 * static_cast<size_t>(r[i]) * plans[i].r8 * 2;
    total += mbytes[i];
    largest = std::max(largest, mbytes[i]);
  }
  if (budget != SIZE_MAX && total > budget) {
    const size_t waves = (total + budget - 1) / budget;
    budget = std::max(largest, total / waves + total / waves / 12);
  }
  std::vector<int> begin{0};
  long long wunits = 0;
  size_t bytes = 0;
  for (int i = 0; i < count; ++i) {
    const size_t mb = mbytes[i];
    const bool over_budget = bytes + mb > budget && wunits >= min_w;
    const bool over_runs = gram_runs(plans, begin.back(), i + 1) > kMaxGramRuns;
    if (wunits > 0 && (over_budget || over_runs)) {
      begin.push_back(i);
      wunits = 0;
      bytes = 0;
    }
    wunits += plans[i].units[kPhaseW0];
    bytes += mb;
  }
  if (begin.size() > 1 && wunits < min_w &&
      gram_runs(plans, begin[begin.size() - 2], count) <= kMaxGramRuns)
    begin.pop_back();
  begin.push_back(count);
  return begin;
}

// Every phase's ranges in order, and every non-Gram pair's static W0 range
// non-empty when there are static W0 units (a tile's W0 segments then come
// from consecutive pairs).
bool sched_valid(const WaveInfo& w, int pairs) {
  for (int j = 0; j < pairs; ++j)
    for (int ph = kPhaseGram; ph <= kPhaseG; ++ph) {
      const long long a = sched_begin(w, pairs, ph, j), b = sched_begin(w, pairs, ph, j + 1);
      if (b < a || (ph == kPhaseW0 && w.n[1] > 0 && j >= w.J && b == a)) return false;
    }
  return true;
}

// The Gram jobs of a wave: one per pair while there are pairs enough (so
// the Gram is done early), as runs of equal cost for the W0 split.
// The share of a wave's W0 units its pool takes (whole tiles from its end).
constexpr double kPoolFraction = 0.25;

bool plan_gram(WaveInfo& w, std::vector<ModulePlan>& plans, int pairs) {
  // Each module's parts of d_in: the fewest (every part adds the module's G
  // units once more) for which a job ends, by the cost model, before the
  // other pairs finish their static W0 units (the G items that need S come
  // after those).
  const double frac = w.m1 - w.m0 > 1 ? kPoolFraction : 0.0;
  long long w0_all = 0;
  for (int i = w.m0; i < w.m1; ++i) {
    set_gram_split(plans[i], 1);
    w0_all += plans[i].units[kPhaseW0];
  }
  for (int i = w.m0; i < w.m1; ++i) {
    ModulePlan& p = plans[i];
    const int kp_max = std::max(1, std::min(kMaxGramParts, p.kb_w / 2));
    for (int kp = 1; kp <= kp_max; ++kp) {
      set_gram_split(p, kp);
      long long jobs = 0;
      for (int m = w.m0; m < w.m1; ++m) jobs += plans[m].units[kPhaseGram];
      const long long q = std::max<long long>(1, pairs - std::min<long long>(jobs, pairs));
      const double static_per_pair = static_cast<double>(w0_all) * (1.0 - frac) / q;
      if (p.gram_cost <= static_per_pair) break;
    }
  }
  for (int ph = 0; ph < 3; ++ph) {
    w.n[ph] = 0;
    for (int i = w.m0; i < w.m1; ++i) w.n[ph] += plans[i].units[ph];
  }
  w.runs = 0;
  w.gw = 0;
  long long jobs = 0;
  for (int i = w.m0; i < w.m1; ++i) {
    const ModulePlan& p = plans[i];
    if (p.units[kPhaseGram] == 0) continue;
    if (w.runs > 0 && w.run_cost[w.runs - 1] == p.gram_cost) {
      w.run_end[w.runs - 1] += static_cast<int>(p.units[kPhaseGram]);
    } else {
      if (w.runs == kMaxGramRuns) return false;
      w.run_cost[w.runs] = p.gram_cost;
      w.run_end[w.runs] = static_cast<int>(jobs + p.units[kPhaseGram]);
      ++w.runs;
    }
    jobs += p.units[kPhaseGram];
    w.gw += p.units[kPhaseGram] * p.gram_cost;
  }
  w.J = static_cast<int>(std::min<long long>(jobs, pairs));
  return sched_valid(w, pairs);
}

// The wave's pool: the static W0 units are the wave's first whole tiles (in
// module order) up to (1 - kPoolFraction) of its W0 units; the rest go to the
// pool chunk by chunk, then the G items (by then S is written).  No static W0
// at all when there would be less than one unit per non-Gram pair.
bool plan_pool(WaveInfo& w, std::vector<ModulePlan>& plans, int pairs) {
  long long w0_all = 0;
  for (int i = w.m0; i < w.m1; ++i) w0_all += plans[i].units[kPhaseW0];
  const long long q = pairs - w.J;
  // A wave of one module keeps all its W0 units static (its pool holds the G
  // items); a wave of several gives the pool the last kPoolFraction of them.
  const double frac = w.m1 - w.m0 > 1 ? kPoolFraction : 0.0;
  long long budget = q > 0 ? static_cast<long long>(w0_all * (1.0 - frac)) : 0;
  long long w0 = 0;
  bool open = true;  // static tiles are a prefix of the wave's tiles in module order
  for (int i = w.m0; i < w.m1; ++i) {
    ModulePlan& p = plans[i];
    p.dyn_t0 = 0;
    while (open && p.dyn_t0 < p.tiles && w0 + p.kb_w <= budget) {
      ++p.dyn_t0;
      w0 += p.kb_w;
    }
    if (p.dyn_t0 < p.tiles) open = false;
  }
  if (w0 < q) {  // too little for a static split: everything from the pool
    for (int i = w.m0; i < w.m1; ++i) plans[i].dyn_t0 = 0;
    w0 = 0;
  }
  long long items = 0, gitems = 0;
  for (int i = w.m0; i < w.m1; ++i) {
    ModulePlan& p = plans[i];
    p.dyn_begin = items;
    items += static_cast<long long>(p.tiles - p.dyn_t0) * p.cpt;
    p.g_item_begin = gitems;
    gitems += static_cast<long long>(p.tiles) * p.gipt;
  }
  w.n[kPhaseW0] = w0;
  w.n[kPhaseG] = 0;
  w.dyn_w0_items = items;
  w.dyn_items = items + gitems;
  return sched_valid(w, pairs);
}

struct GroupLayout {
  std::vector<ModulePlan> plans;
  NormSched sched;
  int seg_slots = 1;
  uint32_t b_region = 0;
  int tmem_cols = 32;
  int stages = 0;
  size_t smem_bytes = 0;
  size_t table_bytes = 0;  // descriptor table at the start of the workspace (grouped)
  size_t cnt_bytes = 0;    // the counter block, right after it
  int cnt_ints = 0;
  int queue_off = 0;       // the waves' pool counters, in ints from the counter block
  size_t total_bytes = 0;
};

// `workers`: the CTA pairs the norm kernel may run (one per two SMs that
// can hold a cluster).
bool layout_group(const int64_t* d_out, const int64_t* d_in, const int64_t* r, int count,
                  bool grouped, int workers, GroupLayout& L) {
  L.plans.resize(count);
  for (int i = 0; i < count; ++i) plan_module(d_out[i], d_in[i], r[i], count > 1, L.plans[i]);
  long long total_w = 0;
  for (const auto& p : L.plans) {
    L.b_region = std::max(L.b_region, p.b_region);
    L.tmem_cols = std::max(L.tmem_cols, p.tmem_cols);
    total_w += p.units[kPhaseW0];
  }
  // Pairs: about a dozen units each at least (every segment ends in an
  // epilogue), at most one per W0 unit; fewer if some wave cannot give every
  // pair a W0 range.
  long long total = 0;
  for (const auto& p : L.plans)
    total += p.units[kPhaseGram] * p.gram_cost + p.units[kPhaseW0] + p.units[kPhaseG];
  int pairs = static_cast<int>(std::min<long long>(
      std::max(1, workers), std::min<long long>(total_w, std::max(1ll, total / 12))));
  std::vector<int> wb;
  while (true) {
    for (auto& p : L.plans) set_gram_split(p, 1);
    size_t budget = grouped ? kWaveBudgetBytes : SIZE_MAX;
    const long long min_w = 3ll * pairs;
    wb = plan_waves(L.plans, d_in, r, min_w, budget);
    while (static_cast<int>(wb.size()) - 1 > kMaxWaves) {
      budget *= 2;
      wb = plan_waves(L.plans, d_in, r, min_w, budget);
    }
    bool ok = static_cast<int>(wb.size()) - 1 <= kMaxWaves;
    NormSched& S = L.sched;
    S.waves = static_cast<int>(wb.size()) - 1;
    S.pairs = pairs;
    for (int w = 0; w < S.waves && ok; ++w) {
      WaveInfo& wi = S.w[w];
      wi.m0 = wb[w];
      wi.m1 = wb[w + 1];
      wi.n[0] = wi.n[1] = wi.n[2] = 0;
      for (int i = wi.m0; i < wi.m1; ++i)
        for (int ph = 0; ph < 3; ++ph) wi.n[ph] += L.plans[i].units[ph];
      if (wi.n[kPhaseW0] < pairs || !plan_gram(wi, L.plans, pairs)) {
        ok = false;
        break;
      }
      if (!plan_pool(wi, L.plans, pairs)) ok = false;
    }
    if (ok) break;
    if (pairs == 1) return false;
    pairs = std::max(1, pairs * 3 / 4);
  }
  // Segment slots: the most segments any tile has -- its W0 segments (the
  // static pairs that share it, or its pool chunks) and one per part of S.
  const NormSched& S = L.sched;
  L.seg_slots = 1;
  for (int w = 0; w < S.waves; ++w) {
    long long at = 0;
    for (int i = S.w[w].m0; i < S.w[w].m1; ++i) {
      const ModulePlan& p = L.plans[i];
      for (int t = 0; t < p.dyn_t0; ++t) {
        const long long xw = at + static_cast<long long>(t) * p.kb_w;
        L.seg_slots = std::max(
            L.seg_slots,
            sched_segments(S.w[w], S.pairs, kPhaseW0, xw, xw + p.kb_w, -1, nullptr) + p.gipt);
      }
      if (p.dyn_t0 < p.tiles) L.seg_slots = std::max(L.seg_slots, p.cpt + p.gipt);
      at += static_w0(p);
    }
  }
  const uint32_t stage_bytes = kTileABytes + L.b_region;
  const int tail_bytes = static_cast<int>(align_up(sizeof(NormSmemTail), 128));
  L.stages = std::min<int>(kMaxStages, (kMaxDynSmem - 1024 - tail_bytes) / stage_bytes);
  if (L.stages < 2) return false;
  L.smem_bytes = 1024 + static_cast<size_t>(L.stages) * stage_bytes + tail_bytes;
  size_t off = grouped ? align_up(sizeof(NormProblemDev) * count, 256) : 0;
  L.table_bytes = off;
  int cnt = 0;
  for (auto& p : L.plans) {
    p.cnt_off = static_cast<size_t>(cnt);
    cnt += module_counters(p);
  }
  L.queue_off = cnt;  // one pool counter per wave after the modules' counters
  cnt += L.sched.waves;
  L.cnt_ints = cnt;
  L.cnt_bytes = align_up(static_cast<size_t>(cnt) * sizeof(int), 256);
  off += L.cnt_bytes;
  for (auto& p : L.plans) {
    p.off_g = off;
    off += align_up(static_cast<size_t>(2) * p.gkp * r[&p - L.plans.data()] * p.r8 * 2,
                    256);  // S_hi, S_lo: gkp parts each
    p.off_np = off;
    off += align_up(static_cast<size_t>(p.tiles) * L.seg_slots * kPairM * 4, 256);
    p.off_tw = off;
    off += align_up(static_cast<size_t>(p.tiles) * sizeof(int), 256);
  }
  L.total_bytes = off;
  return true;
}

bool ensure_tc_attrs() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (d.attrs_set) return true;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(norm_main_kernel<false>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem)) !=
          cudaSuccess ||
      (e = cudaFuncSetAttribute(norm_main_kernel<true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem)) !=
          cudaSuccess ||
      (e = cudaFuncSetAttribute(merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kMaxDynSmem)) != cudaSuccess) {
    note_error("cudaFuncSetAttribute", e);
    return false;
  }
  // How many CTA pairs of the norm kernel (one CTA per SM) can be resident at
  // once: all of them must be, since the pairs that take the G units wait for
  // the pairs that reduce the Gram.
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) sms = 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * std::max(1, sms / 2));
  cfg.blockDim = dim3(kNormThreads);
  cfg.dynamicSmemBytes = kMaxDynSmem;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, norm_main_kernel<false>, &cfg) != cudaSuccess ||
      clusters < 1) {
    (void)cudaGetLastError();
    clusters = std::max(1, sms / 2);
  }
  d.norm_pairs = std::min(clusters, std::max(1, sms / 2));
  d.attrs_set = true;
  return true;
}

// Stream-K workers (CTA pairs) of the norm kernel on the current device; half
// the SMs of a B200 when the device cannot be asked (workspace sizing on a
// host without one).
int norm_workers() {
  int dev = 0;
  if (ensure_tc_attrs() && cudaGetDevice(&dev) == cudaSuccess) return g_dev[dev].norm_pairs;
  (void)cudaGetLastError();
  return 74;
}

// Fills the device descriptor of module `i`; `phase_begin` are its first
// units in its wave's Gram, W0 and G sequences.
bool fill_descriptor(const dora_norm_problem_t& pr, const GroupLayout& L, int i,
                     const long long* phase_begin, uint8_t* ws_base, NormProblemDev& nd) {
  const ModulePlan& p = L.plans[i];
  std::memset(&nd, 0, sizeof(nd));
  uint16_t* g_hi = reinterpret_cast<uint16_t*>(ws_base + p.off_g);
  uint16_t* g_lo = g_hi + static_cast<size_t>(p.gkp) * pr.r * p.r8;
  bool ok = true;
  ok &= make_tmap_bf16(&nd.tm_w0, pr.W0, pr.d_out, pr.d_in, pr.d_in, kBlockK, kTileM);
  ok &= make_tmap_bf16(&nd.tm_arow, pr.A, pr.r, pr.d_in, pr.d_in, kBlockK, kTileM);
  ok &= make_tmap_bf16(&nd.tm_agram, pr.A, pr.r, pr.d_in, pr.d_in, kBlockK, p.gn / 2);
  // The N-side slab half of a CTA in one 4-D box when the two chunks are
  // equal and cover r exactly (no dimension of the view then reaches past the
  // matrix); otherwise one 2-D box of h0 rows per chunk (rows past r read 0).
  const bool slab4d = p.n1 > 0 && 2 * p.n0 == pr.r;
  nd.slab4d = slab4d ? 1 : 0;
  if (slab4d) {
    ok &= make_tmap_bf16_pairslab(&nd.tm_a, pr.A, p.h0, pr.d_in, pr.d_in, kBlockK);
    ok &= make_tmap_bf16_pairslab_parts(&nd.tm_g, g_hi, p.h0, pr.r, p.r8, p.gkp, kBlockK);
    ok &= make_tmap_bf16_pairslab_parts(&nd.tm_glo, g_lo, p.h0, pr.r, p.r8, p.gkp, kBlockK);
  } else {
    ok &= make_tmap_bf16(&nd.tm_a, pr.A, pr.r, pr.d_in, pr.d_in, kBlockK, p.h0);
    ok &= make_tmap_bf16_parts(&nd.tm_g, g_hi, pr.r, pr.r, p.r8, p.gkp, kBlockK, p.h0);
    ok &= make_tmap_bf16_parts(&nd.tm_glo, g_lo, pr.r, pr.r, p.r8, p.gkp, kBlockK, p.h0);
  }
  ok &= make_tmap_bf16(&nd.tm_b, pr.B, pr.d_out, pr.r, pr.r, kBlockK, kTileM);
  ok &= make_tmap_bf16_store32(&nd.tm_ghi_st, g_hi, pr.r, pr.r, p.r8, p.gkp);
  ok &= make_tmap_bf16_store32(&nd.tm_glo_st, g_lo, pr.r, pr.r, p.r8, p.gkp);
  int* cnt = reinterpret_cast<int*>(ws_base + L.table_bytes) + p.cnt_off;
  nd.B = static_cast<const uint16_t*>(pr.B);
  nd.g_hi = g_hi;
  nd.g_lo = g_lo;
  nd.partial = reinterpret_cast<float*>(ws_base + p.off_np);
  nd.tile_cnt = cnt;
  nd.g_ready = cnt + p.tiles * 2;
  nd.tile_w = reinterpret_cast<int*>(ws_base + p.off_tw);
  nd.m = pr.m;
  nd.n_out = pr.n_out;
  nd.g_out = pr.g_out;
  for (int ph = 0; ph < 3; ++ph) nd.begin[ph] = phase_begin[ph];
  nd.dyn_t0 = p.dyn_t0;
  nd.cpt = p.cpt;
  nd.gpi = p.gpi;
  nd.gipt = p.gipt;
  nd.dyn_begin = p.dyn_begin;
  nd.g_item_begin = p.g_item_begin;
  nd.d_out = static_cast<int>(pr.d_out);
  nd.r = static_cast<int>(pr.r);
  nd.r8 = p.r8;
  nd.n_pad = p.n_pad;
  nd.n0 = p.n0;
  nd.n1 = p.n1;
  nd.h0 = p.h0;
  nd.kb_w = p.kb_w;
  nd.kb_r = p.kb_r;
  nd.tiles = p.tiles;
  nd.pg_tiles = p.pg_tiles;
  nd.seg_slots = L.seg_slots;
  nd.nc = p.nc;
  nd.gchunks = p.gchunks;
  nd.gn = p.gn;
  nd.gh = p.gn / 2;
  nd.gj0 = p.gj0;
  nd.gblocks = p.gblocks;
  nd.gkp = p.gkp;
  nd.pair_tx = 2 * (kTileABytes + p.b_region);
  nd.gram_tx = 2 * (kTileABytes + static_cast<uint32_t>(p.nc / 2) * 128u);  // gchunks x gh rows
  nd.idesc0 = idesc_bf16_f32(kPairM, p.n0);
  nd.idesc1 = p.n1 > 0 ? idesc_bf16_f32(kPairM, p.n1) : 0u;
  nd.idesc_gram = idesc_bf16_f32(kPairM, p.gn);
  nd.two_s = 2.0f * pr.s;
  nd.half_s = 0.5f * pr.s;
  return ok;
}

bool tc_eligible(const dora_norm_problem_t& p) {
  return p.d_in % 8 == 0 && p.r % 8 == 0 && aligned16(p.W0) && aligned16(p.A) && aligned16(p.B);
}

dora_status_t check_problem(const dora_norm_problem_t& p) {
  if (p.W0 == nullptr || p.A == nullptr || p.B == nullptr || p.n_out == nullptr)
    return DORA_ERR_INVALID_ARG;
  if (p.d_out < 1 || p.d_in < 1 || p.r < 1) return DORA_ERR_INVALID_ARG;
  if (p.d_out > (1ll << 31) - 1 || p.d_in > (1ll << 31) - 1) return DORA_ERR_UNSUPPORTED;
  if (p.r > DORA_MAX_RANK) return DORA_ERR_UNSUPPORTED;
  if ((p.m == nullptr) != (p.g_out == nullptr)) return DORA_ERR_INVALID_ARG;
  const size_t nb = static_cast<size_t>(p.d_out) * 4;
  if (p.g_out != nullptr && overlaps(p.n_out, nb, p.g_out, nb)) return DORA_ERR_INVALID_ARG;
  return DORA_OK;
}

dora_status_t run_tc_group(const dora_norm_problem_t* probs, int count, bool grouped, float eps,
                           void* ws, size_t ws_bytes, cudaStream_t st, bool emit_sq = false) {
  const DeviceInfo* di = device_info();
  if (di == nullptr) return DORA_ERR_CUDA;
  if (!di->supported) return DORA_ERR_UNSUPPORTED;
  std::vector<int64_t> d_out(count), d_in(count), r(count);
  for (int i = 0; i < count; ++i) {
    d_out[i] = probs[i].d_out;
    d_in[i] = probs[i].d_in;
    r[i] = probs[i].r;
  }
  if (!ensure_tc_attrs()) return DORA_ERR_CUDA;
  static thread_local GroupLayout L;
  if (!layout_group(d_out.data(), d_in.data(), r.data(), count, grouped, norm_workers(), L))
    return DORA_ERR_UNSUPPORTED;
  if (ws == nullptr || ws_bytes < L.total_bytes || !aligned256(ws)) return DORA_ERR_WORKSPACE;

  uint8_t* base = static_cast<uint8_t*>(ws);
  std::vector<NormProblemDev> nds(count);
  for (int w = 0; w < L.sched.waves; ++w) {
    const WaveInfo& W = L.sched.w[w];
    long long at[3] = {0, 0, 0};
    for (int i = W.m0; i < W.m1; ++i) {
      if (!fill_descriptor(probs[i], L, i, at, base, nds[i])) return DORA_ERR_INVALID_ARG;
      nds[i].emit_sq = emit_sq ? 1 : 0;
      at[kPhaseGram] += L.plans[i].units[kPhaseGram];
      at[kPhaseW0] += static_w0(L.plans[i]);
    }
  }
  const unsigned long long tmo = g_timeout_ns.load();
  int* cnt = reinterpret_cast<int*>(base + L.table_bytes);
  const NormProblemDev* table = nullptr;
  if (grouped) {
    NormProblemDev* ntab = reinterpret_cast<NormProblemDev*>(base);
    if (cudaMemcpyAsync(ntab, nds.data(), sizeof(NormProblemDev) * count,
                        cudaMemcpyHostToDevice, st) != cudaSuccess)
      return DORA_ERR_CUDA;
    table = ntab;
  }
  // One-warp blocks (each fits beside a fused-kernel CTA), as many as the
  // counters and static tiles need at about 8 items per lane.
  long long static_tiles = 0;
  for (const auto& p : L.plans) static_tiles += p.dyn_t0;
  const unsigned prep_blocks = static_cast<unsigned>(std::min<long long>(
      64, std::max<long long>(1, ceil_div_ll(std::max<long long>(L.cnt_ints, static_tiles),
                                             32 * 8))));
  if (grouped)
    launch_pdl(norm_prep_kernel<true>, dim3(prep_blocks), dim3(32), 0, st, cnt, L.cnt_ints,
               nds[0], table, count, L.sched);
  else
    launch_pdl(norm_prep_kernel<false>, dim3(prep_blocks), dim3(32), 0, st, cnt, L.cnt_ints,
               nds[0], table, count, L.sched);
  dora_status_t s;
  if ((s = launch_status()) != DORA_OK) return s;
  TimedLaunch tl(st);
  if (grouped)
    launch_pdl(norm_main_kernel<true>, dim3(2 * L.sched.pairs), dim3(kNormThreads),
               L.smem_bytes, st, nds[0], table, L.sched, L.stages, L.b_region,
               static_cast<uint32_t>(L.tmem_cols), eps, tmo, cnt + L.queue_off, g_trace);
  else
    launch_pdl(norm_main_kernel<false>, dim3(2 * L.sched.pairs), dim3(kNormThreads),
               L.smem_bytes, st, nds[0], table, L.sched, L.stages, L.b_region,
               static_cast<uint32_t>(L.tmem_cols), eps, tmo, cnt + L.queue_off, g_trace);
  return launch_status();
}


// One thread waits on a barrier that nothing arrives on; the bounded wait
// gives up and records DORA_ERR_TIMEOUT.
__global__ void unsignalled_wait_kernel(unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbar_init();
  if (!mbar_wait(&bar, 0, timeout_ns, nullptr)) record_error(DORA_ERR_TIMEOUT);
}

size_t simt_workspace(int64_t r) { return align_up(static_cast<size_t>(r) * r * 4, 256); }

}  // namespace
}  // namespace dora

namespace dora {
namespace {
template <typename E, int VEC>
void launch_fwd(bool small, int64_t rows, int64_t d_out, const void* base, const void* lora,
                const float* m, const float* n, float s, float eps, void* y, void* inner,
                bool delta, cudaStream_t cs) {
  const StreamGrid g = stream_grid(rows, static_cast<int>(d_out / VEC), kFwdRowUnroll);
  const dim3 grid(g.gx, g.gy), block(g.bx, g.by);
  const E* b = static_cast<const E*>(base);
  const E* l = static_cast<const E*>(lora);
  E* yo = static_cast<E*>(y);
  E* io = static_cast<E*>(inner);
  const long long R = rows;
  const int D = static_cast<int>(d_out);
  auto go = [&](auto out) {
    constexpr int kOut = decltype(out)::value;
    if (small)
      launch_stream(compose_fwd_kernel<E, VEC, uint32_t, kOut>, grid, block, 0, cs, b, l, m, n,
                    s, eps, R, D, yo, io);
    else
      launch_stream(compose_fwd_kernel<E, VEC, uint64_t, kOut>, grid, block, 0, cs, b, l, m, n,
                    s, eps, R, D, yo, io);
  };
  if (delta)
    go(std::integral_constant<int, kFwdDelta>());
  else if (inner != nullptr)
    go(std::integral_constant<int, kFwdYInner>());
  else
    go(std::integral_constant<int, kFwdY>());
}

template <typename E, int VEC, int kMode>
void launch_bwd(bool small, const StreamGrid& g, int64_t rows, int64_t d_out, const void* dy,
                const void* x1, const void* x2, const float* m, const float* n, float s,
                float eps, void* d_base, void* d_lora, float* partial, cudaStream_t cs) {
  const dim3 grid(g.gx, g.gy), block(g.bx, g.by);
  const E* d = static_cast<const E*>(dy);
  const E* a1 = static_cast<const E*>(x1);
  const E* a2 = static_cast<const E*>(x2);
  E* ob = static_cast<E*>(d_base);
  E* ol = static_cast<E*>(d_lora);
  const long long R = rows;
  const int D = static_cast<int>(d_out);
  if (small)
    launch_stream(compose_bwd_kernel<E, VEC, uint32_t, kMode>, grid, block, 0, cs, d, a1, a2,
                  m, n, s, eps, R, D, ob, ol, partial);
  else
    launch_stream(compose_bwd_kernel<E, VEC, uint64_t, kMode>, grid, block, 0, cs, d, a1, a2,
                  m, n, s, eps, R, D, ob, ol, partial);
}

template <int kMode>
void launch_bwd_dt(dora_dtype_t dt, int vec, bool small, const StreamGrid& g, int64_t rows,
                   int64_t d_out, const void* dy, const void* x1, const void* x2, const float* m,
                   const float* n, float s, float eps, void* d_base, void* d_lora,
                   float* partial, cudaStream_t cs) {
  using B16 = __nv_bfloat16;
  if (dt == DORA_BF16) {
    if (vec == 8)
      launch_bwd<B16, 8, kMode>(small, g, rows, d_out, dy, x1, x2, m, n, s, eps, d_base, d_lora,
                                partial, cs);
    else
      launch_bwd<B16, 1, kMode>(small, g, rows, d_out, dy, x1, x2, m, n, s, eps, d_base, d_lora,
                                partial, cs);
  } else {
    if (vec == 4)
      launch_bwd<float, 4, kMode>(small, g, rows, d_out, dy, x1, x2, m, n, s, eps, d_base,
                                  d_lora, partial, cs);
    else
      launch_bwd<float, 1, kMode>(small, g, rows, d_out, dy, x1, x2, m, n, s, eps, d_base,
                                  d_lora, partial, cs);
  }
}
}  // namespace
}  // namespace dora

using namespace dora;

extern "C" {

size_t dora_factored_norm_workspace_size(int64_t d_out, int64_t d_in, int64_t r,
                                         dora_dtype_t dt) {
  if (d_out < 1 || d_in < 1 || r < 1 || r > DORA_MAX_RANK) return 0;
  if (dt == DORA_F32 || d_in % 8 != 0 || r % 8 != 0) return simt_workspace(r);
  static thread_local GroupLayout L;
  if (!layout_group(&d_out, &d_in, &r, 1, false, norm_workers(), L)) return 0;
  return std::max(L.total_bytes, simt_workspace(r));
}

}  // extern "C"

namespace {
// The single-module norm; with emit_sq the squared-norm sums (before the
// clamp and sqrt) go to n_out and g is not formed.
dora_status_t norm_impl(const void* W0, const void* A, const void* B, dora_dtype_t dt,
                        int64_t d_out, int64_t d_in, int64_t r, float s, const float* m, float eps,
                        float* n_out, float* g_out, void* ws, size_t ws_bytes,
                        dora_stream_t stream, bool emit_sq) {
  if (dt != DORA_F32 && dt != DORA_BF16) return DORA_ERR_INVALID_ARG;
  dora_norm_problem_t p{W0, A, B, m, n_out, g_out, d_out, d_in, r, s};
  dora_status_t st = check_problem(p);
  if (st != DORA_OK) return st;
  if (!(eps >= 0.f)) return DORA_ERR_INVALID_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (dt == DORA_BF16 && tc_eligible(p))
    return run_tc_group(&p, 1, false, eps, ws, ws_bytes, cs, emit_sq);

  const DeviceInfo* di = device_info();
  if (di == nullptr) return DORA_ERR_CUDA;
  if (!di->supported) return DORA_ERR_UNSUPPORTED;
  if (ws == nullptr || ws_bytes < simt_workspace(r) || !aligned256(ws)) return DORA_ERR_WORKSPACE;
  float* G = static_cast<float*>(ws);
  const long long warps = r * r;
  const unsigned gblocks = static_cast<unsigned>(ceil_div_ll(warps * 32, 256));
  const int esq = emit_sq ? 1 : 0;
  if (dt == DORA_F32) {
    gram_simt_kernel<float><<<gblocks, 256, 0, cs>>>(static_cast<const float*>(A), (int)r,
                                                     (int)d_in, G);
    if ((st = launch_status()) != DORA_OK) return st;
    norm_simt_kernel<float><<<(unsigned)d_out, 256, 0, cs>>>(
        static_cast<const float*>(W0), static_cast<const float*>(A),
        static_cast<const float*>(B), G, (int)d_out, (int)d_in, (int)r, s, m, eps, n_out, g_out,
        esq);
  } else {
    gram_simt_kernel<__nv_bfloat16><<<gblocks, 256, 0, cs>>>(
        static_cast<const __nv_bfloat16*>(A), (int)r, (int)d_in, G);
    if ((st = launch_status()) != DORA_OK) return st;
    norm_simt_kernel<__nv_bfloat16><<<(unsigned)d_out, 256, 0, cs>>>(
        static_cast<const __nv_bfloat16*>(W0), static_cast<const __nv_bfloat16*>(A),
        static_cast<const __nv_bfloat16*>(B), G, (int)d_out, (int)d_in, (int)r, s, m, eps, n_out,
        g_out, esq);
  }
  return launch_status();
}

// The schedule self-check behind dora_norm_plan_check: walks every segment
// the kernel's roles take (the same closed forms and item decoding) and
// checks coverage and partial-slot numbering.  Returns "" when every
// invariant holds, else the first one that failed.
std::string check_norm_plan(const GroupLayout& L) {
  char msg[256];
  const NormSched& S = L.sched;
  const int P = S.pairs;
  for (int w = 0; w < S.waves; ++w) {
    const WaveInfo& W = S.w[w];
    const int nm = W.m1 - W.m0;
    std::vector<long long> bw(nm), bg(nm);
    long long aw = 0, ag = 0;
    for (int i = 0; i < nm; ++i) {
      const ModulePlan& p = L.plans[W.m0 + i];
      bw[i] = aw;
      bg[i] = ag;
      aw += static_w0(p);
      if (W.n[kPhaseG] > 0) ag += p.units[kPhaseG];
    }
    if (aw != W.n[kPhaseW0] || ag != W.n[kPhaseG]) {
      snprintf(msg, sizeof(msg), "wave %d: static W0 / G totals %lld / %lld against %lld / %lld",
               w, aw, ag, W.n[kPhaseW0], W.n[kPhaseG]);
      return msg;
    }
    // Gram jobs: consecutive ranges of the wave's jobs, in pair order.
    long long gx = 0;
    for (int j = 0; j < P; ++j) {
      const long long a = sched_begin(W, P, kPhaseGram, j), b = sched_begin(W, P, kPhaseGram, j + 1);
      if (a != gx || b < a) {
        snprintf(msg, sizeof(msg), "wave %d: Gram range of pair %d is [%lld, %lld)", w, j, a, b);
        return msg;
      }
      gx = b;
    }
    if (gx != W.n[kPhaseGram]) {
      snprintf(msg, sizeof(msg), "wave %d: Gram ranges cover %lld of %lld jobs", w, gx,
               W.n[kPhaseGram]);
      return msg;
    }
    // Per tile of each module: (nseg, slot) of every segment; units covered.
    std::vector<std::vector<std::vector<std::pair<int, int>>>> slots(nm);
    std::vector<std::vector<long long>> cov_w(nm), cov_g(nm);
    for (int i = 0; i < nm; ++i) {
      const ModulePlan& p = L.plans[W.m0 + i];
      slots[i].assign(p.tiles, {});
      cov_w[i].assign(p.tiles, 0);
      cov_g[i].assign(p.tiles, 0);
    }
    auto module_of = [&](long long x, bool g) {
      int i = 0;
      while (i + 1 < nm && (g ? bg[i + 1] : bw[i + 1]) <= x) ++i;
      return i;
    };
    auto g_segments = [&](int i, int t, int me, int* gord) {
      const ModulePlan& p = L.plans[W.m0 + i];
      if (W.n[kPhaseG] > 0) {
        const int per = 2 * p.kb_r * p.gkp;
        const long long xg = bg[i] + static_cast<long long>(t) * per;
        return sched_segments(W, P, kPhaseG, xg, xg + per, me, gord);
      }
      return p.gipt;
    };
    auto w0_segments = [&](int i, int t, int* first) {
      const ModulePlan& p = L.plans[W.m0 + i];
      const long long xw = bw[i] + static_cast<long long>(t) * p.kb_w;
      const int f = sched_pair_of(W, P, kPhaseW0, xw);
      *first = f;
      return sched_pair_of(W, P, kPhaseW0, xw + p.kb_w - 1) - f + 1;
    };
    // each pair's static W0 and G ranges
    for (int j = 0; j < P; ++j) {
      for (int ph : {kPhaseW0, kPhaseG}) {
        long long x = sched_begin(W, P, ph, j);
        const long long e = sched_begin(W, P, ph, j + 1);
        while (x < e) {
          const int i = module_of(x, ph == kPhaseG);
          const ModulePlan& p = L.plans[W.m0 + i];
          const int per = ph == kPhaseG ? 2 * p.kb_r * p.gkp : p.kb_w;
          const long long local = x - (ph == kPhaseG ? bg[i] : bw[i]);
          const int t = static_cast<int>(local / per);
          const int k0 = static_cast<int>(local % per);
          const int len = static_cast<int>(std::min<long long>(e - x, per - k0));
          if (t >= p.tiles || (ph == kPhaseW0 && t >= p.dyn_t0)) {
            snprintf(msg, sizeof(msg), "wave %d pair %d: static unit %lld lands on tile %d", w,
                     j, x, t);
            return msg;
          }
          int gord = -1, f = 0;
          const int ng = g_segments(i, t, j, &gord);
          const int nw = w0_segments(i, t, &f);
          slots[i][t].push_back({nw + ng, ph == kPhaseW0 ? j - f : nw + gord});
          (ph == kPhaseG ? cov_g : cov_w)[i][t] += len;
          x += len;
        }
      }
    }
    // the pool items
    for (long long idx = 0; idx < W.dyn_items; ++idx) {
      if (idx < W.dyn_w0_items) {
        int i = 0;
        while (i + 1 < nm && L.plans[W.m0 + i + 1].dyn_begin <= idx) ++i;
        const ModulePlan& p = L.plans[W.m0 + i];
        const int local = static_cast<int>(idx - p.dyn_begin);
        const int c = local % p.cpt, t = p.dyn_t0 + local / p.cpt;
        if (t >= p.tiles) {
          snprintf(msg, sizeof(msg), "wave %d: pool item %lld lands on tile %d", w, idx, t);
          return msg;
        }
        int gord;
        slots[i][t].push_back({p.cpt + g_segments(i, t, -1, &gord), c});
        cov_w[i][t] += (c + 1) * p.kb_w / p.cpt - c * p.kb_w / p.cpt;
      } else {
        const long long jj = idx - W.dyn_w0_items;
        int i = 0;
        while (i + 1 < nm && L.plans[W.m0 + i + 1].g_item_begin <= jj) ++i;
        const ModulePlan& p = L.plans[W.m0 + i];
        const int local = static_cast<int>(jj - p.g_item_begin);
        const int gi = local % p.gipt, t = local / p.gipt;
        if (t >= p.tiles || W.n[kPhaseG] > 0) {
          snprintf(msg, sizeof(msg), "wave %d: G item %lld (tile %d) not expected", w, jj, t);
          return msg;
        }
        int f = 0;
        const int nw = t < p.dyn_t0 ? w0_segments(i, t, &f) : p.cpt;
        const int p0 = gi * p.gpi, p1 = std::min(p0 + p.gpi, p.gkp);
        slots[i][t].push_back({nw + p.gipt, nw + gi});
        cov_g[i][t] += static_cast<long long>(p1 - p0) * 2 * p.kb_r;
      }
    }
    for (int i = 0; i < nm; ++i) {
      const ModulePlan& p = L.plans[W.m0 + i];
      for (int t = 0; t < p.tiles; ++t) {
        const auto& v = slots[i][t];
        if (cov_w[i][t] != p.kb_w || cov_g[i][t] != 2LL * p.kb_r * p.gkp) {
          snprintf(msg, sizeof(msg), "wave %d module %d tile %d: %lld of %d W0 and %lld of %d G "
                   "units covered", w, W.m0 + i, t, cov_w[i][t], p.kb_w, cov_g[i][t],
                   2 * p.kb_r * p.gkp);
          return msg;
        }
        const int nseg = v.empty() ? 0 : v[0].first;
        std::vector<int> seen(std::max(nseg, 1), 0);
        bool ok = static_cast<int>(v.size()) == nseg && nseg <= L.seg_slots;
        for (const auto& q : v) {
          if (q.first != nseg || q.second < 0 || q.second >= nseg || seen[q.second]++) ok = false;
        }
        if (!ok) {
          snprintf(msg, sizeof(msg), "wave %d module %d tile %d: %zu segments, nseg %d, %d slots",
                   w, W.m0 + i, t, v.size(), nseg, L.seg_slots);
          return msg;
        }
      }
    }
  }
  return "";
}
}  // namespace

extern "C" {

dora_status_t dora_factored_norm(const void* W0, const void* A, const void* B, dora_dtype_t dt,
                                 int64_t d_out, int64_t d_in, int64_t r, float s, const float* m,
                                 float eps, float* n_out, float* g_out, void* ws, size_t ws_bytes,
                                 dora_stream_t stream) {
  return norm_impl(W0, A, B, dt, d_out, d_in, r, s, m, eps, n_out, g_out, ws, ws_bytes, stream,
                   false);
}

dora_status_t dora_factored_norm_sq(const void* W0, const void* A, const void* B, dora_dtype_t dt,
                                    int64_t d_out, int64_t d_in, int64_t r, float s,
                                    float* sq_out, void* ws, size_t ws_bytes,
                                    dora_stream_t stream) {
  return norm_impl(W0, A, B, dt, d_out, d_in, r, s, nullptr, 0.f, sq_out, nullptr, ws, ws_bytes,
                   stream, true);
}

dora_status_t dora_norm_finalize(const float* sq, const float* m, float eps, int64_t d_out,
                                 float* n_out, float* g_out, dora_stream_t stream) {
  if (sq == nullptr || n_out == nullptr || d_out < 1) return DORA_ERR_INVALID_ARG;
  if ((m == nullptr) != (g_out == nullptr)) return DORA_ERR_INVALID_ARG;
  if (!(eps >= 0.f)) return DORA_ERR_INVALID_ARG;
  if (d_out > (1ll << 31) - 1) return DORA_ERR_UNSUPPORTED;
  const size_t vb = static_cast<size_t>(d_out) * 4;
  if ((n_out != sq && overlaps(n_out, vb, sq, vb)) || overlaps(g_out, vb, sq, vb) ||
      overlaps(g_out, vb, n_out, vb) || overlaps(n_out, vb, m, vb) || overlaps(g_out, vb, m, vb))
    return DORA_ERR_INVALID_ARG;
  const DeviceInfo* di = device_info();
  if (di == nullptr) return DORA_ERR_CUDA;
  if (!di->supported) return DORA_ERR_UNSUPPORTED;
  launch_pdl(norm_finalize_sq_kernel, dim3((unsigned)ceil_div_ll(d_out, 256)), dim3(256), 0,
             reinterpret_cast<cudaStream_t>(stream), sq, (int)d_out, m, eps, n_out, g_out);
  return launch_status();
}

size_t dora_factored_norm_grouped_workspace_size(const dora_norm_problem_t* problems, int count,
                                                 dora_dtype_t dt) {
  if (problems == nullptr || count < 1 || count > DORA_MAX_GROUP || dt != DORA_BF16) return 0;
  std::vector<int64_t> d_out(count), d_in(count), r(count);
  for (int i = 0; i < count; ++i) {
    if (problems[i].d_out < 1 || problems[i].d_in < 1 || problems[i].r < 1 ||
        problems[i].r > DORA_MAX_RANK)
      return 0;
    d_out[i] = problems[i].d_out;
    d_in[i] = problems[i].d_in;
    r[i] = problems[i].r;
  }
  static thread_local GroupLayout L;
  if (!layout_group(d_out.data(), d_in.data(), r.data(), count, true, norm_workers(), L))
    return 0;
  return L.total_bytes;
}

dora_status_t dora_factored_norm_grouped(const dora_norm_problem_t* problems, int count,
                                         dora_dtype_t dt, float eps, void* ws, size_t ws_bytes,
                                         dora_stream_t stream) {
  if (problems == nullptr || count < 1) return DORA_ERR_INVALID_ARG;
  if (count > DORA_MAX_GROUP) return DORA_ERR_UNSUPPORTED;
  if (dt != DORA_BF16) return DORA_ERR_UNSUPPORTED;
  if (!(eps >= 0.f)) return DORA_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i) {
    dora_status_t st = check_problem(problems[i]);
    if (st != DORA_OK) return st;
    if (!tc_eligible(problems[i])) return DORA_ERR_UNSUPPORTED;
  }
  return run_tc_group(problems, count, true, eps, ws, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

// Forward with an optional second output.  Validation, then one launch.
dora_status_t compose_fwd_impl(const void* base, const void* lora, const float* m, const float* n,
                               float s, float eps, dora_dtype_t dt, int64_t T, int64_t d_out,
                               void* y, void* inner, bool want_inner, dora_stream_t stream,
                               bool delta = false) {
  if (dt != DORA_F32 && dt != DORA_BF16) return DORA_ERR_INVALID_ARG;
  if (T < 0 || d_out < 1) return DORA_ERR_INVALID_ARG;
  if (m == nullptr || n == nullptr) return DORA_ERR_INVALID_ARG;
  if (T > 0 && (base == nullptr || lora == nullptr || y == nullptr)) return DORA_ERR_INVALID_ARG;
  if (want_inner && T > 0 && inner == nullptr) return DORA_ERR_INVALID_ARG;
  if (d_out > (1ll << 31) - 1) return DORA_ERR_UNSUPPORTED;
  if (!(eps >= 0.f)) return DORA_ERR_INVALID_ARG;
  const size_t es = dt == DORA_BF16 ? 2 : 4;
  const size_t nbytes = static_cast<size_t>(T) * d_out * es;
  if (y != base && overlaps(y, nbytes, base, nbytes)) return DORA_ERR_INVALID_ARG;
  if (overlaps(y, nbytes, lora, nbytes)) return DORA_ERR_INVALID_ARG;
  if (want_inner) {
    if (inner != lora && overlaps(inner, nbytes, lora, nbytes)) return DORA_ERR_INVALID_ARG;
    if (overlaps(inner, nbytes, base, nbytes) || overlaps(inner, nbytes, y, nbytes))
      return DORA_ERR_INVALID_ARG;
  }
  const DeviceInfo* di = device_info();
  if (di == nullptr) return DORA_ERR_CUDA;
  if (!di->supported) return DORA_ERR_UNSUPPORTED;
  if (T == 0) return DORA_OK;
  void* in_out = want_inner ? inner : nullptr;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  TimedLaunch tl(cs);
  const bool al = aligned16(base) && aligned16(lora) && aligned16(y) &&
                  (in_out == nullptr || aligned16(in_out));
  const bool small = static_cast<unsigned long long>(T) * static_cast<unsigned long long>(d_out) <
                     (1ull << 31);
  if (dt == DORA_BF16) {
    using B16 = __nv_bfloat16;
    if (al && d_out % 8 == 0)
      launch_fwd<B16, 8>(small, T, d_out, base, lora, m, n, s, eps, y, in_out, delta, cs);
    else
      launch_fwd<B16, 1>(small, T, d_out, base, lora, m, n, s, eps, y, in_out, delta, cs);
  } else {
    if (al && d_out % 4 == 0)
      launch_fwd<float, 4>(small, T, d_out, base, lora, m, n, s, eps, y, in_out, delta, cs);
    else
      launch_fwd<float, 1>(small, T, d_out, base, lora, m, n, s, eps, y, in_out, delta, cs);
  }
  return launch_status();
}

struct BwdShape {
  int vec;
  StreamGrid g;
};
BwdShape bwd_shape(int64_t T, int64_t d_out, dora_dtype_t dt, bool aligned, int unroll) {
  BwdShape b;
  const int v = dt == DORA_BF16 ? 8 : 4;
  b.vec = (aligned && d_out % v == 0) ? v : 1;
  // Blocks 32 vectors wide when the columns divide evenly: the backward then
  // has few row chunks (9 at d_out = 8192 rather than 74), so the dm
  // finalize sums few partials per column; measured 0.3-7 % faster per call
  // than the widest blocks, most on [8192, 25600] and [2048, 4096].
  const int ncv = static_cast<int>(d_out / b.vec);
  b.g = stream_grid(T, ncv, unroll, kStreamSlots, ncv % 32 == 0 ? 32 : 0);
  return b;
}

// The three backward variants after their own validation: x1 / x2 are base /
// lora, inner / unused, or unused / unused.
dora_status_t compose_bwd_impl(int mode, const void* dy, const void* x1, const void* x2,
                               const float* m, const float* n, float s, float eps,
                               dora_dtype_t dt, int64_t T, int64_t d_out, void* d_base,
                               void* d_lora, float* dm, void* ws, size_t ws_bytes,
                               dora_stream_t stream) {
  const DeviceInfo* di = device_info();
  if (di == nullptr) return DORA_ERR_CUDA;
  if (!di->supported) return DORA_ERR_UNSUPPORTED;
  if (mode == kBwdFrozen && T == 0) return DORA_OK;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const bool al = aligned16(dy) && (mode == kBwdFrozen || aligned16(x1)) &&
                  (mode != kBwdFromBaseLora || aligned16(x2)) && aligned16(d_base) &&
                  aligned16(d_lora);
  const BwdShape b = bwd_shape(T, d_out, dt, al, bwd_row_unroll(mode));
  float* partial = nullptr;
  if (mode != kBwdFrozen) {
    const size_t need = static_cast<size_t>(b.g.gy) * d_out * 4;
    if (ws == nullptr || ws_bytes < need || !aligned256(ws)) return DORA_ERR_WORKSPACE;
    partial = static_cast<float*>(ws);
  }
  const bool small = static_cast<unsigned long long>(T) * static_cast<unsigned long long>(d_out) <
                     (1ull << 31);
  dora_status_t st;
  {
    TimedLaunch tl(cs);
    if (mode == kBwdFromBaseLora)
      launch_bwd_dt<kBwdFromBaseLora>(dt, b.vec, small, b.g, T, d_out, dy, x1, x2, m, n, s, eps,
                                      d_base, d_lora, partial, cs);
    else if (mode == kBwdFromInner)
      launch_bwd_dt<kBwdFromInner>(dt, b.vec, small, b.g, T, d_out, dy, x1, x2, m, n, s, eps,
                                   d_base, d_lora, partial, cs);
    else
      launch_bwd_dt<kBwdFrozen>(dt, b.vec, small, b.g, T, d_out, dy, x1, x2, m, n, s, eps,
                                d_base, d_lora, partial, cs);
    st = launch_status();
  }
  if (st != DORA_OK || mode == kBwdFrozen) return st;
  launch_pdl(colsum_finalize_kernel, dim3((unsigned)ceil_div_ll(d_out, 32)), dim3(32, 8), 0, cs,
             static_cast<const float*>(partial), b.g.gy, (int)d_out, n, eps, dm);
  return launch_status();
}

// Arguments shared by every backward variant.
dora_status_t check_bwd_common(const float* m, const float* n, float eps, dora_dtype_t dt,
                               int64_t T, int64_t d_out) {
  if (dt != DORA_F32 && dt != DORA_BF16) return DORA_ERR_INVALID_ARG;
  if (T < 0 || d_out < 1) return DORA_ERR_INVALID_ARG;
  if (m == nullptr || n == nullptr) return DORA_ERR_INVALID_ARG;
  if (d_out > (1ll << 31) - 1) return DORA_ERR_UNSUPPORTED;
  if (!(eps >= 0.f)) return DORA_ERR_INVALID_ARG;
  return DORA_OK;
}

}  // namespace

extern "C" {

dora_status_t dora_compose_fwd(const void* base, const void* lora, const float* m, const float* n,
                               float s, float eps, dora_dtype_t dt, int64_t T, int64_t d_out,
                               void* y, dora_stream_t stream) {
  return compose_fwd_impl(base, lora, m, n, s, eps, dt, T, d_out, y, nullptr, false, stream);
}

dora_status_t dora_compose_fwd_delta(const void* base, const void* lora, const float* m,
                                     const float* n, float s, float eps, dora_dtype_t dt,
                                     int64_t T, int64_t d_out, void* dy_out,
                                     dora_stream_t stream) {
  return compose_fwd_impl(base, lora, m, n, s, eps, dt, T, d_out, dy_out, nullptr, false, stream,
                          true);
}

dora_status_t dora_compose_fwd_train(const void* base, const void* lora, const float* m,
                                     const float* n, float s, float eps, dora_dtype_t dt,
                                     int64_t T, int64_t d_out, void* y, void* inner,
                                     dora_stream_t stream) {
  return compose_fwd_impl(base, lora, m, n, s, eps, dt, T, d_out, y, inner, true, stream);
}

size_t dora_compose_bwd_workspace_size(int64_t T, int64_t d_out, dora_dtype_t dt) {
  if (T < 0 || d_out < 1) return 0;
  // The chunk count does not depend on the vector width chosen at call time:
  // take the larger of the two layouts.  The variants that read fewer
  // streams keep more rows in flight per thread, so they need no more.
  const BwdShape a = bwd_shape(T, d_out, dt, true, kBwdRowUnroll);
  const BwdShape b = bwd_shape(T, d_out, dt, false, kBwdRowUnroll);
  const int chunks = std::max(a.g.gy, b.g.gy);
  return align_up(static_cast<size_t>(chunks) * d_out * 4, 256);
}

dora_status_t dora_compose_bwd(const void* dy, const void* base, const void* lora, const float* m,
                               const float* n, float s, float eps, dora_dtype_t dt, int64_t T,
                               int64_t d_out, void* d_base, void* d_lora, float* dm, void* ws,
                               size_t ws_bytes, dora_stream_t stream) {
  dora_status_t c = check_bwd_common(m, n, eps, dt, T, d_out);
  if (c != DORA_OK) return c;
  if (dm == nullptr) return DORA_ERR_INVALID_ARG;
  if (T > 0 && (dy == nullptr || base == nullptr || lora == nullptr || d_base == nullptr ||
                d_lora == nullptr))
    return DORA_ERR_INVALID_ARG;
  const size_t es = dt == DORA_BF16 ? 2 : 4;
  const size_t nbytes = static_cast<size_t>(T) * d_out * es;
  const size_t vb = static_cast<size_t>(d_out) * 4;
  if (d_base != dy && overlaps(d_base, nbytes, dy, nbytes)) return DORA_ERR_INVALID_ARG;
  if (overlaps(d_base, nbytes, base, nbytes) || overlaps(d_base, nbytes, lora, nbytes) ||
      overlaps(d_base, nbytes, d_lora, nbytes) || overlaps(d_lora, nbytes, dy, nbytes) ||
      overlaps(d_lora, nbytes, base, nbytes) || overlaps(d_lora, nbytes, lora, nbytes))
    return DORA_ERR_INVALID_ARG;
  if (overlaps(dm, vb, m, vb) || overlaps(dm, vb, n, vb)) return DORA_ERR_INVALID_ARG;
  return compose_bwd_impl(kBwdFromBaseLora, dy, base, lora, m, n, s, eps, dt, T, d_out, d_base,
                          d_lora, dm, ws, ws_bytes, stream);
}

dora_status_t dora_compose_bwd_inner(const void* dy, const void* inner, const float* m,
                                     const float* n, float s, float eps, dora_dtype_t dt,
                                     int64_t T, int64_t d_out, void* d_base, void* d_lora,
                                     float* dm, void* ws, size_t ws_bytes, dora_stream_t stream) {
  dora_status_t c = check_bwd_common(m, n, eps, dt, T, d_out);
  if (c != DORA_OK) return c;
  if (dm == nullptr) return DORA_ERR_INVALID_ARG;
  if (T > 0 && (dy == nullptr || inner == nullptr || d_base == nullptr || d_lora == nullptr))
    return DORA_ERR_INVALID_ARG;
  const size_t es = dt == DORA_BF16 ? 2 : 4;
  const size_t nbytes = static_cast<size_t>(T) * d_out * es;
  const size_t vb = static_cast<size_t>(d_out) * 4;
  if (d_base != dy && overlaps(d_base, nbytes, dy, nbytes)) return DORA_ERR_INVALID_ARG;
  if (overlaps(d_base, nbytes, inner, nbytes) || overlaps(d_base, nbytes, d_lora, nbytes) ||
      overlaps(d_lora, nbytes, dy, nbytes) || overlaps(d_lora, nbytes, inner, nbytes))
    return DORA_ERR_INVALID_ARG;
  if (overlaps(dm, vb, m, vb) || overlaps(dm, vb, n, vb)) return DORA_ERR_INVALID_ARG;
  return compose_bwd_impl(kBwdFromInner, dy, inner, nullptr, m, n, s, eps, dt, T, d_out, d_base,
                          d_lora, dm, ws, ws_bytes, stream);
}

dora_status_t dora_compose_bwd_frozen(const void* dy, const float* m, const float* n, float s,
                                      float eps, dora_dtype_t dt, int64_t T, int64_t d_out,
                                      void* d_base, void* d_lora, dora_stream_t stream) {
  dora_status_t c = check_bwd_common(m, n, eps, dt, T, d_out);
  if (c != DORA_OK) return c;
  if (T > 0 && (dy == nullptr || d_base == nullptr || d_lora == nullptr))
    return DORA_ERR_INVALID_ARG;
  const size_t es = dt == DORA_BF16 ? 2 : 4;
  const size_t nbytes = static_cast<size_t>(T) * d_out * es;
  if (d_base != dy && overlaps(d_base, nbytes, dy, nbytes)) return DORA_ERR_INVALID_ARG;
  if (overlaps(d_base, nbytes, d_lora, nbytes) || overlaps(d_lora, nbytes, dy, nbytes))
    return DORA_ERR_INVALID_ARG;
  return compose_bwd_impl(kBwdFrozen, dy, nullptr, nullptr, m, n, s, eps, dt, T, d_out, d_base,
                          d_lora, nullptr, nullptr, 0, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Merged inference weight.
// ---------------------------------------------------------------------------
namespace dora {
namespace {
struct MergeLayout {
  int kb, stages, tiles_m, tiles_n, r8;
  size_t smem_bytes, ws_bytes;
};

bool merge_layout(int64_t d_out, int64_t d_in, int64_t r, MergeLayout& L) {
  if (d_out < 1 || d_in < 1 || r < 1 || r > DORA_MAX_RANK) return false;
  L.kb = static_cast<int>(ceil_div_ll(r, kMergeK));
  L.r8 = round_up_int(static_cast<int>(r), 8);
  L.tiles_m = static_cast<int>(ceil_div_ll(d_out, kMergePairM));
  L.tiles_n = static_cast<int>(ceil_div_ll(d_in, kMergeN));
  // Shared memory: two W0 / W' staging tiles and as many 16 KiB k-block
  // stages (this CTA's half of A^T, or its B rows while a row block
  // starts) as fit: six.
  const size_t tail = align_up(sizeof(MergeSmemTail), 128);
  const size_t fixed = 1024 + static_cast<size_t>(kMergeWBufs) * kMergeTileBytes + tail;
  if (fixed + 2 * kMergeStageBytes > static_cast<size_t>(kMaxDynSmem)) return false;
  L.stages = static_cast<int>(std::min<size_t>(kMergeMaxStages,
                                               (kMaxDynSmem - fixed) / kMergeStageBytes));
  L.smem_bytes = fixed + static_cast<size_t>(L.stages) * kMergeStageBytes;
  L.ws_bytes = align_up(static_cast<size_t>(d_in) * L.r8 * 2, 256);
  return true;
}
}  // namespace
}  // namespace dora

extern "C" {

size_t dora_merge_weight_workspace_size(int64_t d_out, int64_t d_in, int64_t r) {
  MergeLayout L;
  return merge_layout(d_out, d_in, r, L) ? L.ws_bytes : 0;
}

dora_status_t dora_merge_weight(const void* W0, const void* A, const void* B, const float* m,
                                const float* n, float s, float eps, int64_t d_out, int64_t d_in,
                                int64_t r, void* W_out, void* ws, size_t ws_bytes,
                                dora_stream_t stream) {
  if (W0 == nullptr || A == nullptr || B == nullptr || m == nullptr || n == nullptr ||
      W_out == nullptr)
    return DORA_ERR_INVALID_ARG;
  if (d_out < 1 || d_in < 1 || r < 1) return DORA_ERR_INVALID_ARG;
  if (!(eps >= 0.f)) return DORA_ERR_INVALID_ARG;
  if (r > DORA_MAX_RANK || d_out > (1ll << 31) - 1 || d_in > (1ll << 31) - 1)
    return DORA_ERR_UNSUPPORTED;
  if (d_in % 8 != 0 || r % 8 != 0 || !aligned16(W0) || !aligned16(A) || !aligned16(B) ||
      !aligned16(W_out))
    return DORA_ERR_UNSUPPORTED;
  const size_t wb = static_cast<size_t>(d_out) * d_in * 2;
  if (W_out != W0 && overlaps(W_out, wb, W0, wb)) return DORA_ERR_INVALID_ARG;
  if (overlaps(W_out, wb, A, static_cast<size_t>(r) * d_in * 2) ||
      overlaps(W_out, wb, B, static_cast<size_t>(d_out) * r * 2) ||
      overlaps(W_out, wb, m, d_out * 4) || overlaps(W_out, wb, n, d_out * 4))
    return DORA_ERR_INVALID_ARG;
  MergeLayout L;
  if (!merge_layout(d_out, d_in, r, L)) return DORA_ERR_UNSUPPORTED;
  if (ws == nullptr || ws_bytes < L.ws_bytes || !aligned256(ws)) return DORA_ERR_WORKSPACE;
  if (overlaps(ws, L.ws_bytes, W_out, wb)) return DORA_ERR_INVALID_ARG;
  const DeviceInfo* di = device_info();
  if (di == nullptr) return DORA_ERR_CUDA;
  if (!di->supported) return DORA_ERR_UNSUPPORTED;
  if (!ensure_tc_attrs()) return DORA_ERR_CUDA;
  static thread_local MergeDev P;
  std::memset(&P, 0, sizeof(P));
  uint16_t* At = static_cast<uint16_t*>(ws);
  bool ok = true;
  ok &= make_tmap_bf16(&P.tm_w0, W0, d_out, d_in, d_in, 64, kMergeM);
  ok &= make_tmap_bf16(&P.tm_out, W_out, d_out, d_in, d_in, 64, 32);
  ok &= make_tmap_bf16(&P.tm_b, B, d_out, r, r, kMergeK, kMergeM);
  ok &= make_tmap_bf16(&P.tm_at, At, d_in, r, L.r8, kMergeK, kMergeM);  // a CTA's 128 rows
  if (!ok) return DORA_ERR_INVALID_ARG;
  P.m = m;
  P.n = n;
  P.s = s;
  P.eps = eps;
  P.d_out = static_cast<int>(d_out);
  P.d_in = static_cast<int>(d_in);
  P.r = static_cast<int>(r);
  P.kb = L.kb;
  P.tiles_n = L.tiles_n;
  P.tiles = L.tiles_m * L.tiles_n;
  P.idesc = idesc_bf16_f32(kMergePairM, kMergeN);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  launch_pdl(transpose_bf16_kernel, dim3((unsigned)ceil_div_ll(d_in, 32), (unsigned)ceil_div_ll(r, 32)),
             dim3(32, 8), 0, cs, static_cast<const uint16_t*>(A), static_cast<int>(r),
             static_cast<int>(d_in), At, L.r8);
  dora_status_t st = launch_status();
  if (st != DORA_OK) return st;
  const int pairs = std::max(1, std::min(di->sms / 2, P.tiles));
  TimedLaunch tl(cs);
  launch_pdl(merge_kernel, dim3(2 * pairs), dim3(kMergeThreads), L.smem_bytes, cs, P, L.stages,
             g_timeout_ns.load());
  return launch_status();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Grouped compose: the modules of a layer in one launch.
// ---------------------------------------------------------------------------
namespace dora {
namespace {
static_assert(kMaxComposeGroup == DORA_MAX_COMPOSE_GROUP, "group capacity");

struct ComposePlan {
  ComposeGroup grp;
  int blocks = 0, cblocks = 0;
  bool small = true;
  size_t ws_bytes = 0;
};

// Each module's grid is stream_grid() with its share of the launch's slots
// (by activation elements); its dm partial table follows the previous
// module's at a 256-byte boundary of the workspace.  Depends on the shapes,
// the vector width and the variant only, so dm's summation order is fixed.
void plan_compose_group(const dora_compose_problem_t* pr, int count, int vec, int unroll,
                        bool partials, uint8_t* ws, float eps, ComposePlan& P) {
  std::memset(&P.grp, 0, sizeof(P.grp));
  P.grp.count = count;
  P.grp.eps = eps;
  double total = 0.0;
  for (int p = 0; p < count; ++p) total += static_cast<double>(pr[p].T) * pr[p].d_out;
  int blk = 0, cblk = 0;
  size_t off = 0;
  P.small = true;
  for (int p = 0; p < count; ++p) {
    ComposeItem& it = P.grp.it[p];
    const double share = total > 0.0 ? static_cast<double>(pr[p].T) * pr[p].d_out / total : 0.0;
    const long long slots = std::max(1ll, std::llround(kStreamSlots * share));
    const StreamGrid g = stream_grid(pr[p].T, static_cast<int>(pr[p].d_out / vec), unroll, slots);
    it.T = pr[p].T;
    it.d_out = static_cast<int>(pr[p].d_out);
    it.s = pr[p].s;
    it.m = pr[p].m;
    it.n = pr[p].n;
    it.bx = g.bx;
    it.gx = g.gx;
    it.gy = g.gy;
    it.blk_begin = blk;
    it.cblk_begin = cblk;
    blk += g.gx * g.gy;
    cblk += static_cast<int>(ceil_div_ll(pr[p].d_out, 32));
    if (partials) {
      it.partial = ws != nullptr ? reinterpret_cast<float*>(ws + off) : nullptr;
      off += align_up(static_cast<size_t>(g.gy) * pr[p].d_out * 4, 256);
    }
    if (static_cast<unsigned long long>(pr[p].T) * static_cast<unsigned long long>(pr[p].d_out) >=
        (1ull << 31))
      P.small = false;
  }
  P.blocks = blk;
  P.cblocks = cblk;
  P.ws_bytes = off;
}

// Backward variant of a record list, or -1 if the records disagree.  dm
// (never empty) tells frozen from not; inner vs base and lora is read from the
// records with T > 0 (an empty record reads nothing and may leave them NULL).
int compose_group_mode(const dora_compose_problem_t* pr, int count) {
  const bool frozen = pr[0].dm == nullptr;
  for (int p = 1; p < count; ++p)
    if ((pr[p].dm == nullptr) != frozen) return -1;
  if (frozen) return kBwdFrozen;
  int mode = -1;
  for (int p = 0; p < count; ++p) {
    if (pr[p].T == 0) continue;
    const int mp = pr[p].inner != nullptr ? kBwdFromInner : kBwdFromBaseLora;
    if (mode >= 0 && mp != mode) return -1;
    mode = mp;
  }
  return mode >= 0 ? mode : kBwdFromBaseLora;
}

dora_status_t check_compose_record(const dora_compose_problem_t& q, dora_dtype_t dt, bool bwd,
                                   int mode) {
  if (q.T < 0 || q.d_out < 1) return DORA_ERR_INVALID_ARG;
  if (q.d_out > (1ll << 31) - 1) return DORA_ERR_UNSUPPORTED;
  if (q.m == nullptr || q.n == nullptr) return DORA_ERR_INVALID_ARG;
  const size_t es = dt == DORA_BF16 ? 2 : 4;
  const size_t nb = static_cast<size_t>(q.T) * q.d_out * es;
  const size_t vb = static_cast<size_t>(q.d_out) * 4;
  if (!bwd) {
    if (q.T > 0 && (q.base == nullptr || q.lora == nullptr || q.y == nullptr))
      return DORA_ERR_INVALID_ARG;
    if (q.y != q.base && overlaps(q.y, nb, q.base, nb)) return DORA_ERR_INVALID_ARG;
    if (overlaps(q.y, nb, q.lora, nb)) return DORA_ERR_INVALID_ARG;
    if (q.inner != nullptr) {
      if (q.inner != q.lora && overlaps(q.inner, nb, q.lora, nb)) return DORA_ERR_INVALID_ARG;
      if (overlaps(q.inner, nb, q.base, nb) || overlaps(q.inner, nb, q.y, nb))
        return DORA_ERR_INVALID_ARG;
    }
    return DORA_OK;
  }
  if (q.T > 0 && (q.dy == nullptr || q.d_base == nullptr || q.d_lora == nullptr))
    return DORA_ERR_INVALID_ARG;
  if (q.d_base != q.dy && overlaps(q.d_base, nb, q.dy, nb)) return DORA_ERR_INVALID_ARG;
  if (overlaps(q.d_base, nb, q.d_lora, nb) || overlaps(q.d_lora, nb, q.dy, nb))
    return DORA_ERR_INVALID_ARG;
  if (mode == kBwdFrozen) return DORA_OK;
  if (overlaps(q.dm, vb, q.m, vb) || overlaps(q.dm, vb, q.n, vb)) return DORA_ERR_INVALID_ARG;
  // The streams this variant reads besides dy: inner, or base and lora.
  const void* ins[2] = {mode == kBwdFromInner ? q.inner : q.base, q.lora};
  const int nin = mode == kBwdFromInner ? 1 : 2;
  for (int k = 0; k < nin; ++k) {
    if (q.T > 0 && ins[k] == nullptr) return DORA_ERR_INVALID_ARG;
    if (overlaps(q.d_base, nb, ins[k], nb) || overlaps(q.d_lora, nb, ins[k], nb))
      return DORA_ERR_INVALID_ARG;
  }
  return DORA_OK;
}

// Vector width usable by every record of the group.
int compose_group_vec(const dora_compose_problem_t* pr, int count, dora_dtype_t dt, bool bwd,
                      int mode) {
  const int v = dt == DORA_BF16 ? 8 : 4;
  for (int p = 0; p < count; ++p) {
    const dora_compose_problem_t& q = pr[p];
    if (q.d_out % v != 0) return 1;
    bool al;
    if (!bwd)
      al = aligned16(q.base) && aligned16(q.lora) && aligned16(q.y) &&
           (q.inner == nullptr || aligned16(q.inner));
    else
      al = aligned16(q.dy) && aligned16(q.d_base) && aligned16(q.d_lora) &&
           (mode != kBwdFromInner || aligned16(q.inner)) &&
           (mode != kBwdFromBaseLora || (aligned16(q.base) && aligned16(q.lora)));
    if (!al) return 1;
  }
  return v;
}

template <typename E, int VEC>
void launch_fwd_grouped(const ComposePlan& P, cudaStream_t cs) {
  if (P.small)
    launch_stream(compose_fwd_grouped_kernel<E, VEC, uint32_t>, dim3(P.blocks),
                  dim3(kStreamThreads), 0, cs, P.grp);
  else
    launch_stream(compose_fwd_grouped_kernel<E, VEC, uint64_t>, dim3(P.blocks),
                  dim3(kStreamThreads), 0, cs, P.grp);
}

template <typename E, int VEC, int kMode>
void launch_bwd_grouped(const ComposePlan& P, cudaStream_t cs) {
  if (P.small)
    launch_stream(compose_bwd_grouped_kernel<E, VEC, uint32_t, kMode>, dim3(P.blocks),
                  dim3(kStreamThreads), 0, cs, P.grp);
  else
    launch_stream(compose_bwd_grouped_kernel<E, VEC, uint64_t, kMode>, dim3(P.blocks),
                  dim3(kStreamThreads), 0, cs, P.grp);
}

template <int kMode>
void launch_bwd_grouped_dt(dora_dtype_t dt, int vec, const ComposePlan& P, cudaStream_t cs) {
  if (dt == DORA_BF16) {
    if (vec == 8)
      launch_bwd_grouped<__nv_bfloat16, 8, kMode>(P, cs);
    else
      launch_bwd_grouped<__nv_bfloat16, 1, kMode>(P, cs);
  } else {
    if (vec == 4)
      launch_bwd_grouped<float, 4, kMode>(P, cs);
    else
      launch_bwd_grouped<float, 1, kMode>(P, cs);
  }
}
}  // namespace
}  // namespace dora

extern "C" {

dora_status_t dora_compose_fwd_grouped(const dora_compose_problem_t* problems, int count,
                                       dora_dtype_t dt, float eps, dora_stream_t stream) {
  if (dt != DORA_F32 && dt != DORA_BF16) return DORA_ERR_INVALID_ARG;
  if (problems == nullptr || count < 1) return DORA_ERR_INVALID_ARG;
  if (count > DORA_MAX_COMPOSE_GROUP) return DORA_ERR_UNSUPPORTED;
  if (!(eps >= 0.f)) return DORA_ERR_INVALID_ARG;
  for (int p = 0; p < count; ++p) {
    const dora_status_t c = check_compose_record(problems[p], dt, false, 0);
    if (c != DORA_OK) return c;
  }
  const DeviceInfo* di = device_info();
  if (di == nullptr) return DORA_ERR_CUDA;
  if (!di->supported) return DORA_ERR_UNSUPPORTED;
  const int vec = compose_group_vec(problems, count, dt, false, 0);
  static thread_local ComposePlan P;
  plan_compose_group(problems, count, vec, kFwdRowUnroll, false, nullptr, eps, P);
  for (int p = 0; p < count; ++p) {
    ComposeItem& it = P.grp.it[p];
    it.in0 = problems[p].base;
    it.in1 = problems[p].lora;
    it.out0 = problems[p].y;
    it.out1 = problems[p].inner;
  }
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  TimedLaunch tl(cs);
  if (dt == DORA_BF16) {
    if (vec == 8)
      launch_fwd_grouped<__nv_bfloat16, 8>(P, cs);
    else
      launch_fwd_grouped<__nv_bfloat16, 1>(P, cs);
  } else {
    if (vec == 4)
      launch_fwd_grouped<float, 4>(P, cs);
    else
      launch_fwd_grouped<float, 1>(P, cs);
  }
  return launch_status();
}

size_t dora_compose_bwd_grouped_workspace_size(const dora_compose_problem_t* problems, int count,
                                               dora_dtype_t dt) {
  if (problems == nullptr || count < 1 || count > DORA_MAX_COMPOSE_GROUP) return 0;
  const int mode = compose_group_mode(problems, count);
  if (mode < 0 || mode == kBwdFrozen) return 0;
  for (int p = 0; p < count; ++p)
    if (problems[p].T < 0 || problems[p].d_out < 1) return 0;
  static thread_local ComposePlan P;
  size_t best = 0;
  for (int vec : {dt == DORA_BF16 ? 8 : 4, 1}) {
    bool ok = true;
    for (int p = 0; p < count; ++p) ok = ok && problems[p].d_out % vec == 0;
    if (!ok) continue;
    plan_compose_group(problems, count, vec, bwd_row_unroll(mode), true, nullptr, 0.f, P);
    best = std::max(best, P.ws_bytes);
  }
  return best;
}

dora_status_t dora_compose_bwd_grouped(const dora_compose_problem_t* problems, int count,
                                       dora_dtype_t dt, float eps, void* ws, size_t ws_bytes,
                                       dora_stream_t stream) {
  if (dt != DORA_F32 && dt != DORA_BF16) return DORA_ERR_INVALID_ARG;
  if (problems == nullptr || count < 1) return DORA_ERR_INVALID_ARG;
  if (count > DORA_MAX_COMPOSE_GROUP) return DORA_ERR_UNSUPPORTED;
  if (!(eps >= 0.f)) return DORA_ERR_INVALID_ARG;
  const int mode = compose_group_mode(problems, count);
  if (mode < 0) return DORA_ERR_INVALID_ARG;
  for (int p = 0; p < count; ++p) {
    const dora_status_t c = check_compose_record(problems[p], dt, true, mode);
    if (c != DORA_OK) return c;
  }
  const DeviceInfo* di = device_info();
  if (di == nullptr) return DORA_ERR_CUDA;
  if (!di->supported) return DORA_ERR_UNSUPPORTED;
  const int vec = compose_group_vec(problems, count, dt, true, mode);
  static thread_local ComposePlan P;
  const bool partials = mode != kBwdFrozen;
  plan_compose_group(problems, count, vec, bwd_row_unroll(mode), partials,
                     static_cast<uint8_t*>(ws), eps, P);
  if (partials && (ws == nullptr || ws_bytes < P.ws_bytes || !aligned256(ws)))
    return DORA_ERR_WORKSPACE;
  for (int p = 0; p < count; ++p) {
    ComposeItem& it = P.grp.it[p];
    it.in0 = problems[p].dy;
    it.in1 = mode == kBwdFromInner ? problems[p].inner : problems[p].base;
    it.in2 = mode == kBwdFromBaseLora ? problems[p].lora : nullptr;
    it.out0 = problems[p].d_base;
    it.out1 = problems[p].d_lora;
    it.dm = problems[p].dm;
  }
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  dora_status_t st;
  {
    TimedLaunch tl(cs);
    if (mode == kBwdFromBaseLora)
      launch_bwd_grouped_dt<kBwdFromBaseLora>(dt, vec, P, cs);
    else if (mode == kBwdFromInner)
      launch_bwd_grouped_dt<kBwdFromInner>(dt, vec, P, cs);
    else
      launch_bwd_grouped_dt<kBwdFrozen>(dt, vec, P, cs);
    st = launch_status();
  }
  if (st != DORA_OK || !partials) return st;
  launch_pdl(colsum_grouped_kernel, dim3(P.cblocks), dim3(32, 8), 0, cs, P.grp);
  return launch_status();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Compose backward without a caller-provided workspace.
//
// Some callers cannot hand the library a workspace: a plain C host program
// that links libdora.so without any device allocator of its own, or a
// latency-critical loop in which cudaMalloc is not allowed because it can
// synchronise the whole device.  For them, the column-partial table of the
// backward lives in a fixed array in device memory instead.  Every GPU that
// loads this library holds the array (4 MiB) until the process exits.
// ---------------------------------------------------------------------------
namespace dora {
namespace {
constexpr size_t kStaticScratchBytes = size_t(4) << 20;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch on the current device (the name is only
// a host-side stand-in in host code).  Looked up on every call, so that the
// address stays right after a device reset; the first lookup on a device can
// load the module, which must not happen inside a stream capture, so that
// first call is refused while `st` is capturing.
void* static_scratch_address() {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
  if (e != cudaSuccess) {
    note_error("cudaGetSymbolAddress(static scratch)", e);
    return nullptr;
  }
  return p;
}
}  // namespace
}  // namespace dora

extern "C" dora_status_t dora_compose_bwd_static(const void* dy, const void* base,
                                                 const void* lora, const float* m, const float* n,
                                                 float s, float eps, dora_dtype_t dt, int64_t T,
                                                 int64_t d_out, void* d_base, void* d_lora,
                                                 float* dm, dora_stream_t stream) {
  if (dt != DORA_F32 && dt != DORA_BF16) return DORA_ERR_INVALID_ARG;
  if (T < 0 || d_out < 1) return DORA_ERR_INVALID_ARG;
  const size_t need = dora_compose_bwd_workspace_size(T, d_out, dt);
  if (need > kStaticScratchBytes) {
    snprintf(t_last_error, sizeof(t_last_error),
             "dora_compose_bwd_static: this shape needs %zu bytes of scratch; the built-in array "
             "holds %zu (use dora_compose_bwd with a workspace)",
             need, kStaticScratchBytes);
    return DORA_ERR_UNSUPPORTED;
  }
  const DeviceInfo* di = device_info();
  if (di == nullptr) return DORA_ERR_CUDA;
  if (!di->supported) return DORA_ERR_UNSUPPORTED;
  void* scratch = static_scratch_address();
  if (scratch == nullptr) return DORA_ERR_CUDA;
  // Every slot of the partial table the kernels read is written by the same
  // call first, so nothing has to be cleared between calls.
  return dora_compose_bwd(dy, base, lora, m, n, s, eps, dt, T, d_out, d_base, d_lora, dm,
                          scratch, kStaticScratchBytes, stream);
}

extern "C" {

dora_status_t dora_get_device_status(dora_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DORA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return DORA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess)
      return DORA_ERR_CUDA;
  }
  return static_cast<dora_status_t>(v);
}

const char* dora_status_string(dora_status_t status) {
  switch (status) {
    case DORA_OK: return "ok";
    case DORA_ERR_INVALID_ARG: return "invalid argument";
    case DORA_ERR_UNSUPPORTED: return "unsupported size, dtype or device";
    case DORA_ERR_WORKSPACE: return "workspace missing, too small or not 256-byte aligned";
    case DORA_ERR_CUDA: return "CUDA runtime error";
    case DORA_ERR_TIMEOUT: return "a kernel gave up on a bounded wait";
    case DORA_ERR_BOUNDS: return "a kernel skipped an out-of-range store (debug build)";
    case DORA_ERR_INTERNAL: return "a schedule invariant does not hold";
  }
  return "unknown status";
}

int dora_version(void) { return kVersion; }

dora_status_t dora_debug_unsignalled_wait(uint64_t timeout_ns, dora_stream_t stream) {
  const DeviceInfo* di = device_info();
  if (di == nullptr) return DORA_ERR_CUDA;
  if (!di->supported) return DORA_ERR_UNSUPPORTED;
  const unsigned long long t = std::min<unsigned long long>(
      std::max<unsigned long long>(timeout_ns, 1000ull), 1000000000ull);
  unsignalled_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(t);
  return launch_status();
}

uint64_t dora_launch_count(void) { return g_launches.load(); }

const char* dora_last_error(void) { return t_last_error; }

void dora_set_trace_buffer(void* buf) { g_trace = static_cast<unsigned long long*>(buf); }

dora_status_t dora_norm_plan_check(const int64_t* d_out, const int64_t* d_in, const int64_t* r,
                                   int count, int grouped, int pairs) {
  if (d_out == nullptr || d_in == nullptr || r == nullptr || count < 1 || pairs < 1 ||
      pairs > 512 || (!grouped && count != 1))
    return DORA_ERR_INVALID_ARG;
  if (count > DORA_MAX_GROUP) return DORA_ERR_UNSUPPORTED;
  for (int i = 0; i < count; ++i) {
    if (d_out[i] < 1 || d_in[i] < 1 || r[i] < 1) return DORA_ERR_INVALID_ARG;
    if (r[i] > DORA_MAX_RANK || d_out[i] > (1ll << 31) - 1 || d_in[i] > (1ll << 31) - 1)
      return DORA_ERR_UNSUPPORTED;
  }
  static thread_local dora::GroupLayout L;
  if (!dora::layout_group(d_out, d_in, r, count, grouped != 0, pairs, L)) {
    snprintf(dora::t_last_error, sizeof(dora::t_last_error), "no schedule for these sizes");
    return DORA_ERR_UNSUPPORTED;
  }
  const std::string err = check_norm_plan(L);
  if (!err.empty()) {
    snprintf(dora::t_last_error, sizeof(dora::t_last_error), "%s", err.c_str());
    return DORA_ERR_INTERNAL;
  }
  return DORA_OK;
}

void dora_set_timing_events(void* before, void* after) {
  t_ev_before = static_cast<cudaEvent_t>(before);
  t_ev_after = static_cast<cudaEvent_t>(after);
}

void dora_set_wait_timeout_ns(uint64_t ns) {
  g_timeout_ns.store(ns == 0 ? kDefaultTimeoutNs : static_cast<unsigned long long>(ns));
}

}  // extern "C"
