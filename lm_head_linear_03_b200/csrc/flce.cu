// Host side of the FLCE library: argument checks, workspace carving, TMA
// descriptors, the launch plan and the C ABI declared in include/flce.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "flce.h"
#include "flce_kernels.cuh"

namespace {

using namespace flce;

// Vocabulary entries per pass-2 chunk.  The G chunk buffer is N x VC bf16, so
// the workspace stays independent of V.
constexpr int VC = 2048;
// Active k-blocks a paired dW item runs on its first half before it needs the
// second buffer: about one dX epilogue's time on the previous item.
constexpr int DW_LEAD = 16;
constexpr int MAX_SPLITS = 64;
constexpr unsigned long long DEFAULT_TIMEOUT_NS = 2000000000ull;  // 2 s per bounded wait

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// The last CUDA failure this library reported (FLCE_ERR_CUDA), per host thread:
// the source line of the failing step and the CUDA runtime's error.
thread_local int g_fail_line = 0;
thread_local cudaError_t g_fail_code = cudaSuccess;

flce_status_t cuda_fail(int line) {
  g_fail_line = line;
  g_fail_code = cudaPeekAtLastError();
  return FLCE_ERR_CUDA;
}

struct WsLayout {
  size_t ctrl, counters, counters_bytes, tile_cnt, tile_valid, perm, y_perm, g_perm, lse2, zy, part_m, part_l,
      blk_loss, blk_cnt, G, lo, xc, total;
  bool packed;  // holds xc, the packed copy of X that reordered rows need
};

// ctrl block: [0] status, [4] ticket, [8] n_valid, [12] inv_n, [16] loss,
// [20] reordered (1 when the token rows are reordered), [24] valid rows
struct Ctrl {
  int32_t status;
  uint32_t ticket;
  int32_t n_valid;
  float inv_n;
  float loss;
  int32_t reordered;
  int32_t n_rows;
};

// `packed`: with the N x H area for the packed copy of X (reordered rows).
WsLayout ws_layout(int64_t N, int64_t H, bool packed = false) {
  WsLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  const size_t n = static_cast<size_t>(N);
  const size_t nblk = (n + COMBINE_THREADS - 1) / COMBINE_THREADS;
  L.ctrl = take(256);
  // pass-2 completion counters: g_row[TM], x_row[TM], g_col[VC/BN], w_col[VC/BN]
  const size_t tm = (n + CM - 1) / CM;
  L.counters_bytes = (2 * tm + 2 * (VC / BN)) * 4;
  L.counters = take(L.counters_bytes);
  L.tile_cnt = take(tm * 4);
  L.tile_valid = take(tm * 4);
  L.perm = take(tm * CM * 4);
  L.y_perm = take(n * 4);
  L.g_perm = take(n * 4);
  L.lse2 = take(n * 4);
  L.zy = take(n * 4);
  L.part_m = take(static_cast<size_t>(MAX_SPLITS) * n * 4);
  L.part_l = take(static_cast<size_t>(MAX_SPLITS) * n * 4);
  L.blk_loss = take(nblk * 8);
  L.blk_cnt = take(nblk * 4);
  L.G = take(n * VC * 2);
  L.lo = take(n * static_cast<size_t>(H) * 2);
  L.packed = packed;
  L.xc = packed ? take(n * static_cast<size_t>(H) * 2) : 0;
  L.total = off;
  return L;
}

// Workspace of the cross-entropy-on-logits entry: depends on N only.
struct CeLayout {
  size_t ctrl, tile_valid, row_acc, blk_sum, total;
};
CeLayout ce_ws_layout(int64_t N) {
  CeLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  const size_t n = static_cast<size_t>(N);
  L.ctrl = take(256);
  L.tile_valid = take(((n + CM - 1) / CM) * 4);
  L.row_acc = take(n * 8);
  L.blk_sum = take(((n + COMBINE_THREADS - 1) / COMBINE_THREADS) * 8);
  L.total = off;
  return L;
}

// ------------------------------------------------------------ device info --
struct DevInfo {
  bool ok = false;
  bool sm100 = false;
  int num_sms = 0;
  int max_clusters = 0;  // SM pairs that can run a GEMM kernel at the same time
};

std::mutex g_mu;
DevInfo g_dev[64];
bool g_attr_set[64];

cudaError_t device_info(DevInfo* out, int* dev_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_dev[dev].ok) {
    int major = 0, minor = 0, sms = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    g_dev[dev].sm100 = (major == 10 && minor == 0);
    g_dev[dev].num_sms = sms;
    g_dev[dev].ok = true;
  }
  *out = g_dev[dev];
  *dev_out = dev;
  return cudaSuccess;
}

cudaError_t set_kernel_attrs(int dev) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_attr_set[dev]) return cudaSuccess;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(flce_pass1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, P1_SMEM_BYTES)) !=
      cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(flce_pass2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES)) !=
      cudaSuccess)
    return e;
  // How many SM pairs the GEMM kernels can occupy at once (persistent grids).
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * 1024, 1, 1);
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = CLUSTER;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int clusters = 0, clusters2 = 0;
  cfg.dynamicSmemBytes = P1_SMEM_BYTES;
  if ((e = cudaOccupancyMaxActiveClusters(&clusters, flce_pass1_kernel, &cfg)) != cudaSuccess) return e;
  cfg.dynamicSmemBytes = SMEM_BYTES;
  if ((e = cudaOccupancyMaxActiveClusters(&clusters2, flce_pass2_kernel, &cfg)) != cudaSuccess) return e;
  clusters = std::min(clusters, clusters2);
  if (clusters <= 0) return cudaErrorInvalidConfiguration;
  g_dev[dev].max_clusters = clusters;
  g_attr_set[dev] = true;
  return cudaSuccess;
}

// ------------------------------------------------------------ tensor maps --
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool get_encode() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode) return true;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fn == nullptr)
    return false;
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return true;
}

// 2-D bf16 row-major tensor [outer][inner], boxes of box_inner x box_outer
// elements with the 128-B swizzle (operands) or the 64-B one (the epilogues'
// 32 x 32 boxes); out-of-range elements read as zero.
enum class Swz { k128, k64 };

bool make_map(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint64_t row_bytes,
              uint32_t box_inner, uint32_t box_outer, Swz swz = Swz::k128) {
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              swz == Swz::k128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ plan --
struct Plan {
  int tiles_m;        // 256-token tiles (one per SM pair)
  int vtiles;         // 256-wide vocabulary tiles
  int splits;         // pass-1 vocabulary splits
  int lse_clusters;   // SM pairs of the pass-1 launch
  int num_chunks;
  int launches;
  int clusters;       // SM pairs available
};

// Pass 1: pick the number of vocabulary splits whose units, dealt round-robin
// to the persistent SM pairs, give the smallest largest per-pair load.  A unit
// walks its tiles in pairs (256 x 512), a pair costing about 1.6 lone tiles
// (an estimate from the tiles' k-block rates; counting one per tile measured
// the same), plus one tile's worth for its pipeline fill and partial write.
int choose_splits(int tiles_m, int vtiles, int sms) {
  int best = 1;
  long long best_cost = LLONG_MAX;
  const int smax = std::min(MAX_SPLITS, vtiles);
  std::vector<long long> load;
  for (int S = 1; S <= smax; ++S) {
    const long long units = static_cast<long long>(tiles_m) * S;
    const int grid = static_cast<int>(std::min<long long>(units, sms));
    load.assign(grid, 0);
    for (long long u = 0; u < units; ++u) {
      const long long s = u / tiles_m;
      const long long n = ((s + 1) * vtiles) / S - (s * vtiles) / S;
      load[u % grid] += 16 * (n / 2) + 10 * (n % 2) + 10;
    }
    const long long cost = *std::max_element(load.begin(), load.end());
    if (cost < best_cost) {
      best_cost = cost;
      best = S;
    }
  }
  return best;
}

Plan make_plan(int64_t N, int64_t H, int64_t V, int clusters) {
  (void)H;
  Plan p{};
  p.clusters = clusters;
  p.tiles_m = static_cast<int>((N + CM - 1) / CM);
  p.vtiles = static_cast<int>((V + BN - 1) / BN);
  p.splits = choose_splits(p.tiles_m, p.vtiles, clusters);
  p.lse_clusters =
      static_cast<int>(std::min<long long>(static_cast<long long>(p.tiles_m) * p.splits, clusters));
  p.num_chunks = static_cast<int>((V + VC - 1) / VC);
  // prep, row order, pass 1, combine, pass 2, dX scatter (plus the X row
  // packing on a workspace with the packed-X area)
  p.launches = 6;
  return p;
}

// ------------------------------------------------------------- profiling --
struct Prof {
  bool on = false;
  std::vector<cudaEvent_t> ev;  // pairs
  std::vector<int> kind;
  size_t used = 0;
};
Prof g_prof;
constexpr size_t PROF_PAIRS = 16384;

void prof_begin(cudaStream_t s, int k, size_t* slot) {
  *slot = SIZE_MAX;
  if (!g_prof.on || g_prof.used >= PROF_PAIRS) return;
  *slot = g_prof.used++;
  g_prof.kind[*slot] = k;
  cudaEventRecord(g_prof.ev[2 * *slot], s);
}
void prof_end(cudaStream_t s, size_t slot) {
  if (slot != SIZE_MAX) cudaEventRecord(g_prof.ev[2 * slot + 1], s);
}

// ---------------------------------------------------------------- checks --
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

flce_status_t check_sizes(int64_t N, int64_t H, int64_t V) {
  if (N <= 0 || H <= 0 || V <= 0) return FLCE_ERR_INVALID_ARGUMENT;
  if (N > (1ll << 30) || V > (1ll << 30) || H > (1ll << 20)) return FLCE_ERR_INVALID_ARGUMENT;
  if (H % 8 != 0) return FLCE_ERR_UNSUPPORTED;
  return FLCE_OK;
}

// dX and dW may both be NULL only when `forward_only_ok` (no gradient pass).
flce_status_t check_args(const void* X, const void* W, const void* y, int64_t N, int64_t H, int64_t V,
                         const void* dX, const void* dW, const void* ws, bool forward_only_ok = false) {
  const flce_status_t s = check_sizes(N, H, V);
  if (s != FLCE_OK) return s;
  if (!X || !W || !y || !ws) return FLCE_ERR_INVALID_ARGUMENT;
  const bool no_grads = !dX && !dW;
  if ((!dX || !dW) && !(no_grads && forward_only_ok)) return FLCE_ERR_INVALID_ARGUMENT;
  if (!aligned(X, 16) || !aligned(W, 16) || !aligned(dX, 16) || !aligned(dW, 16) || !aligned(y, 4) ||
      !aligned(ws, 256))
    return FLCE_ERR_UNSUPPORTED;
  return FLCE_OK;
}

// --------------------------------------------------------------- enqueue --
// Host-buffer calls overlap the PCIe copies with the kernels: W arrives in
// pieces on a copy stream and pass 1 runs piece by piece as they land; pass 2
// runs as a few launches over consecutive chunk sections of its item queue,
// and each section's finished dW rows go back on the copy stream while the
// next section computes.
constexpr int MAX_PIECES = 16;
struct PipeCtx {
  cudaStream_t copy = nullptr;
  int pieces = 0;                      // W pieces = pass-1 launches
  int64_t piece_v[MAX_PIECES + 1] = {};  // vocabulary rows [piece_v[i], piece_v[i+1]), multiples of BN
  cudaEvent_t w_ready[MAX_PIECES] = {};  // recorded on `copy` after piece i's copy
  int groups = 0;                      // pass-2 launches
  cudaEvent_t p2_done[MAX_PIECES] = {};
  uint16_t* h_dW = nullptr;            // host dW, filled group by group on `copy` (null: no copies)
  int64_t* section_rows = nullptr;     // if set: dW rows [section_rows[k], section_rows[k+1]) of section k
};

// Per-device copy stream and events of the host-buffer entry, made on first
// use and kept (like the device-property cache) for the life of the process.
struct PipeRes {
  std::mutex mu;
  cudaStream_t copy = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t ev[2 * MAX_PIECES] = {};
};
PipeRes g_pipe[64];

cudaError_t pipe_resources(PipeRes** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  PipeRes& r = g_pipe[dev];
  std::lock_guard<std::mutex> lk(g_mu);
  if (r.copy == nullptr) {
    if ((e = cudaStreamCreateWithFlags(&r.copy, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&r.start, cudaEventDisableTiming)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&r.done, cudaEventDisableTiming)) != cudaSuccess) return e;
    for (auto& ev : r.ev)
      if ((e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming)) != cudaSuccess) return e;
  }
  *out = &r;
  return cudaSuccess;
}

struct Options {
  int reduction = RED_MEAN;
  const float* grad_row_scale = nullptr;
  float* row_loss = nullptr;
  const int* mean_count = nullptr;
  // Vocabulary shard: this call's W holds rows [v0, v0 + V) of a vocabulary of
  // V_total entries (0 = V).  COMBINE_SHARD calls stop after writing the rows'
  // shard statistics; COMBINE_SHARDS_IN calls take every shard's statistics
  // instead of running pass 1.
  int combine = COMBINE_FULL;
  int64_t v0 = 0, V_total = 0;
  float* shard_lse = nullptr;
  float* shard_zy = nullptr;
  int shards = 0;
  const float* all_lse = nullptr;
  const float* all_zy = nullptr;
  const PipeCtx* pipe = nullptr;  // host-buffer call: pieces of pass 1, sections of pass 2
  // failure probe only: a shorter wait limit, and dW mainloops that wait for
  // one G tile more than the queue produces
  unsigned long long timeout_ns = DEFAULT_TIMEOUT_NS;
  int starve_dw = 0;
};

flce_status_t enqueue(const uint16_t* X, const uint16_t* W, const int32_t* y, int64_t N, int64_t H, int64_t V,
                      int32_t ignore_index, float* d_loss, int32_t* d_status, uint16_t* dX, uint16_t* dW,
                      void* workspace, size_t ws_bytes, cudaStream_t stream, const Options& opt = Options()) {
  DevInfo di;
  int dev;
  if (device_info(&di, &dev) != cudaSuccess) return cuda_fail(__LINE__);
  if (!di.sm100) return FLCE_ERR_UNSUPPORTED;
  if (set_kernel_attrs(dev) != cudaSuccess) return cuda_fail(__LINE__);
  if (!get_encode()) return cuda_fail(__LINE__);

  if (device_info(&di, &dev) != cudaSuccess) return cuda_fail(__LINE__);  // now with max_clusters
  // reordered rows need the packed-X area: only a large enough workspace has it
  // (vocabulary shards keep the caller's order: their statistics are per row)
  const WsLayout L = ws_layout(N, H, opt.combine == COMBINE_FULL && ws_bytes >= ws_layout(N, H, true).total);
  const Plan P = make_plan(N, H, V, di.max_clusters);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(ws + L.ctrl);
  float* lse2 = reinterpret_cast<float*>(ws + L.lse2);
  float* zy = reinterpret_cast<float*>(ws + L.zy);
  float* part_m = reinterpret_cast<float*>(ws + L.part_m);
  float* part_l = reinterpret_cast<float*>(ws + L.part_l);
  uint16_t* G = reinterpret_cast<uint16_t*>(ws + L.G);
  uint16_t* lo = reinterpret_cast<uint16_t*>(ws + L.lo);
  int* perm = reinterpret_cast<int*>(ws + L.perm);
  int32_t* y_perm = reinterpret_cast<int32_t*>(ws + L.y_perm);
  float* g_perm = reinterpret_cast<float*>(ws + L.g_perm);
  const float* g_rows = opt.grad_row_scale ? g_perm : nullptr;  // upstream weights in the rows' order
  uint16_t* Xc = L.packed ? reinterpret_cast<uint16_t*>(ws + L.xc) : nullptr;

  CUtensorMap mX_k, mW_k, mG_mn, mX_mn, mG_k, mW_mn, mXc_k, mXc_mn;
  const uint64_t n = static_cast<uint64_t>(N), h = static_cast<uint64_t>(H), v = static_cast<uint64_t>(V);
  bool ok = make_map(&mX_k, X, h, n, h * 2, BK, BM) && make_map(&mW_k, W, h, v, h * 2, BK, BNH) &&
            make_map(&mG_mn, G, VC, n, VC * 2, 64, BK) && make_map(&mX_mn, X, h, n, h * 2, 64, BK) &&
            make_map(&mG_k, G, VC, n, VC * 2, BK, BM) && make_map(&mW_mn, W, h, v, h * 2, 64, BK) &&
            // the packed copy of X (the caller's X stands in when there is none: never read then)
            make_map(&mXc_k, Xc ? Xc : X, h, n, h * 2, BK, BM) && make_map(&mXc_mn, Xc ? Xc : X, h, n, h * 2, 64, BK);
  // 32 x 32 output boxes of the epilogues (64-byte swizzle)
  CUtensorMap mGo, mDWo, mHio, mLoo;
  ok = ok && (dX == nullptr || (make_map(&mGo, G, VC, n, VC * 2, EPI_BOX, EPI_BOX, Swz::k64) &&
                                make_map(&mDWo, dW, h, v, h * 2, EPI_BOX, EPI_BOX, Swz::k64) &&
                                make_map(&mHio, dX, h, n, h * 2, EPI_BOX, EPI_BOX, Swz::k64) &&
                                make_map(&mLoo, lo, h, n, h * 2, EPI_BOX, EPI_BOX, Swz::k64)));
  if (!ok) return cuda_fail(__LINE__);

  // control words and pass-2 counters start at zero (they are contiguous)
  if (cudaMemsetAsync(ctrl, 0, L.counters + L.counters_bytes - L.ctrl, stream) != cudaSuccess) return cuda_fail(__LINE__);
  if (d_status != &ctrl->status && cudaMemsetAsync(d_status, 0, sizeof(int32_t), stream) != cudaSuccess)
    return cuda_fail(__LINE__);

  GemmArgs a{};
  a.N = static_cast<int>(N);
  a.H = static_cast<int>(H);
  a.V = static_cast<int>(V);
  a.ignore_index = ignore_index;
  a.Vc = VC;
  a.y = y_perm;
  a.part_m = part_m;
  a.part_l = part_l;
  a.zy = zy;
  a.lse2 = lse2;
  a.inv_n = &ctrl->inv_n;
  a.G = G;
  a.dW = dW;
  a.dX = dX;
  a.lo = lo;
  a.status = d_status;
  a.timeout_ns = opt.timeout_ns;
  a.starve_dw = opt.starve_dw;
  a.reduction = opt.reduction;
  a.grad_row_scale = g_rows;
  a.tile_valid = reinterpret_cast<const int*>(ws + L.tile_valid);
  a.perm = perm;
  a.reordered = &ctrl->reordered;

  // Valid rows per 256-row token tile, then the token-row order of both passes.
  {
    size_t slot;
    prof_begin(stream, KIND_PREP, &slot);
    flce_prep_kernel<<<P.tiles_m, CM, 0, stream>>>(y, static_cast<int>(N), ignore_index,
                                                   reinterpret_cast<int*>(ws + L.tile_cnt));
    prof_end(stream, slot);
    if (cudaGetLastError() != cudaSuccess) return cuda_fail(__LINE__);
    prof_begin(stream, KIND_ORDER, &slot);
    flce_row_order_kernel<<<P.tiles_m, CM, 0, stream>>>(
        y, opt.grad_row_scale, static_cast<int>(N), P.tiles_m, ignore_index,
        reinterpret_cast<const int*>(ws + L.tile_cnt), L.packed ? 1 : 0, static_cast<int>(opt.v0),
        static_cast<int>(V), static_cast<int>(opt.V_total ? opt.V_total : V),
        reinterpret_cast<int*>(ws + L.tile_valid), perm, y_perm, g_perm, &ctrl->reordered, &ctrl->n_rows, d_status);
    prof_end(stream, slot);
    if (cudaGetLastError() != cudaSuccess) return cuda_fail(__LINE__);
    if (L.packed) {  // X rows in the new order (returns at once when the order was kept)
      const int pgrid = static_cast<int>(std::min<int64_t>((N + 7) / 8, static_cast<int64_t>(di.num_sms) * 8));
      prof_begin(stream, KIND_PACK, &slot);
      flce_pack_rows_kernel<<<pgrid, 256, 0, stream>>>(X, Xc, perm, &ctrl->reordered, &ctrl->n_rows,
                                                        static_cast<int>(N), static_cast<int>(H));
      prof_end(stream, slot);
      if (cudaGetLastError() != cudaSuccess) return cuda_fail(__LINE__);
    }
  }

  // Pass 1: logits tile by tile, online log-sum-exp per (row, split); a call
  // given every vocabulary shard's statistics has its lse already.
  int total_splits = P.splits;
  if (opt.combine != COMBINE_SHARDS_IN && (opt.pipe == nullptr || opt.pipe->pieces == 0)) {
    GemmArgs p1 = a;
    p1.tiles_m = P.tiles_m;
    p1.tiles_n = P.vtiles;
    p1.k_blocks = static_cast<int>((H + BK - 1) / BK);
    p1.splits = P.splits;
    p1.num_units = P.tiles_m * P.splits;
    size_t slot;
    prof_begin(stream, KIND_LSE, &slot);
    flce_pass1_kernel<<<CLUSTER * P.lse_clusters, NUM_THREADS, P1_SMEM_BYTES, stream>>>(mX_k, mXc_k, mW_k, p1);
    prof_end(stream, slot);
    if (cudaGetLastError() != cudaSuccess) return cuda_fail(__LINE__);
  } else if (opt.combine != COMBINE_SHARDS_IN) {
    // one launch per W piece, after its copy; its splits fill the next partial slots
    const PipeCtx& pp = *opt.pipe;
    total_splits = 0;
    for (int i = 0; i < pp.pieces; ++i) {
      const int64_t v0 = pp.piece_v[i], vp = pp.piece_v[i + 1] - pp.piece_v[i];
      CUtensorMap mWp;
      if (!make_map(&mWp, W + v0 * H, h, static_cast<uint64_t>(vp), h * 2, BK, BNH)) return cuda_fail(__LINE__);
      GemmArgs p1 = a;
      p1.V = static_cast<int>(vp);
      p1.v_off = static_cast<int>(v0);
      p1.split_off = total_splits;
      p1.tiles_m = P.tiles_m;
      p1.tiles_n = static_cast<int>((vp + BN - 1) / BN);
      p1.k_blocks = static_cast<int>((H + BK - 1) / BK);
      p1.splits = std::min(choose_splits(P.tiles_m, p1.tiles_n, P.clusters), MAX_SPLITS / pp.pieces);
      p1.num_units = P.tiles_m * p1.splits;
      total_splits += p1.splits;
      const int grid = static_cast<int>(std::min<long long>(p1.num_units, P.clusters));
      if (cudaStreamWaitEvent(stream, pp.w_ready[i], 0) != cudaSuccess) return cuda_fail(__LINE__);
      size_t slot;
      prof_begin(stream, KIND_LSE, &slot);
      flce_pass1_kernel<<<CLUSTER * grid, NUM_THREADS, P1_SMEM_BYTES, stream>>>(mX_k, mXc_k, mWp, p1);
      prof_end(stream, slot);
      if (cudaGetLastError() != cudaSuccess) return cuda_fail(__LINE__);
    }
  }
  // Combine the splits: lse, loss, n_valid, 1/n.
  {
    CombineArgs c{};
    c.N = static_cast<int>(N);
    c.V = static_cast<int>(V);
    c.ignore_index = ignore_index;
    c.splits = total_splits;
    c.y = y_perm;
    c.perm = perm;
    c.part_m = part_m;
    c.part_l = part_l;
    c.zy = zy;
    c.lse2 = lse2;
    c.blk_loss = reinterpret_cast<double*>(ws + L.blk_loss);
    c.blk_cnt = reinterpret_cast<int*>(ws + L.blk_cnt);
    c.ticket = &ctrl->ticket;
    c.n_valid = &ctrl->n_valid;
    c.inv_n = &ctrl->inv_n;
    c.loss = d_loss;
    c.status = d_status;
    c.reduction = opt.reduction;
    c.grad_row_scale = g_rows;
    c.row_loss = opt.row_loss;
    c.mean_count = opt.mean_count;
    c.mode = opt.combine;
    c.shards = opt.shards;
    c.all_lse = opt.all_lse;
    c.all_zy = opt.all_zy;
    c.shard_lse = opt.shard_lse;
    c.shard_zy = opt.shard_zy;
    const int grid = static_cast<int>((N + COMBINE_THREADS - 1) / COMBINE_THREADS);
    size_t slot;
    prof_begin(stream, KIND_COMBINE, &slot);
    flce_combine_kernel<<<grid, COMBINE_THREADS, 0, stream>>>(c);
    prof_end(stream, slot);
    if (cudaGetLastError() != cudaSuccess) return cuda_fail(__LINE__);
  }
  // Pass 2: every chunk's logit recompute, dW and dX tiles in one persistent launch
  // (skipped for a forward-only call and for a shard's statistics).
  if (dX != nullptr && opt.combine != COMBINE_SHARD) {
    GemmArgs b = a;
    b.TM = P.tiles_m;
    b.HN = static_cast<int>((H + BN - 1) / BN);
    b.dw_lead = DW_LEAD;
    b.C = P.num_chunks;
    b.VTf = VC / BN;
    b.VT_last = static_cast<int>((V - static_cast<int64_t>(P.num_chunks - 1) * VC + BN - 1) / BN);
    if (b.C == 1) b.VTf = b.VT_last;
    // G tiles column by column when a chunk holds more than three rounds of
    // them for the SM pairs, else row by row (see the queue's description)
    b.g_cols_first = static_cast<long long>(b.TM) * b.VTf > 3ll * P.clusters ? b.VTf : 0;
    // dW items pair adjacent hidden tiles (256 x 512 in both accumulator
    // buffers) in the same regime; with fewer rounds a chunk's items are on the
    // critical path of the next chunk's G epilogues, and longer items only delay it
    b.HW = b.g_cols_first ? (b.HN + 1) / 2 : b.HN;
    // section_end[c]: end of the queue's section c (dX(c) dW(c) G(c+1)), after G(0)
    std::vector<long long> section_end(b.C);
    long long total = static_cast<long long>(b.C == 1 ? b.VT_last : b.VTf) * b.TM;  // G(0)
    for (int c = 0; c < b.C; ++c) {
      const long long vt = c == b.C - 1 ? b.VT_last : b.VTf;
      total += static_cast<long long>(b.TM) * b.HN + vt * b.HW;
      if (c + 1 < b.C) total += static_cast<long long>(c + 1 == b.C - 1 ? b.VT_last : b.VTf) * b.TM;
      section_end[c] = total;
    }
    b.total_items = total;
    int* ctr = reinterpret_cast<int*>(ws + L.counters);
    b.g_row = ctr;
    b.x_row = ctr + b.TM;
    b.g_col = ctr + 2 * b.TM;
    b.w_col = ctr + 2 * b.TM + VC / BN;
    Pass2Maps pm;
    pm.Xk = mX_k;
    pm.Wk = mW_k;
    pm.Gmn = mG_mn;
    pm.Xmn = mX_mn;
    pm.Gk = mG_k;
    pm.Wmn = mW_mn;
    pm.Go = mGo;
    pm.DWo = mDWo;
    pm.Hio = mHio;
    pm.Loo = mLoo;
    pm.Xck = mXc_k;
    pm.Xcmn = mXc_mn;
    // one launch over the whole queue; a host-buffer call splits it into
    // sections of whole chunks and sends each section's dW rows back
    const int groups = opt.pipe ? std::max(1, std::min(opt.pipe->groups, b.C)) : 1;
    // Sections of whole chunks; with several, the last one is a single chunk,
    // so that little of dW is left to copy or reduce after the last launch.
    auto section_chunk = [&](int k) {  // first chunk of section k (k = groups: the end)
      if (groups == 1 || k == groups) return k == groups ? b.C : 0;
      return static_cast<int>(static_cast<long long>(k) * (b.C - 1) / (groups - 1));
    };
    size_t slot;
    for (int k = 0; k < groups; ++k) {
      const int c0 = section_chunk(k);
      const int c1 = section_chunk(k + 1);
      b.item_begin = k == 0 ? 0 : section_end[c0 - 1];
      b.item_end = section_end[c1 - 1];
      const int grid = static_cast<int>(std::min<long long>(b.item_end - b.item_begin, P.clusters));
      if (grid > 0) {
        prof_begin(stream, KIND_PASS2, &slot);
        flce_pass2_kernel<<<CLUSTER * grid, NUM_THREADS, SMEM_BYTES, stream>>>(pm, b);
        prof_end(stream, slot);
        if (cudaGetLastError() != cudaSuccess) return cuda_fail(__LINE__);
      }
      if (opt.pipe) {  // dW rows of chunks c0 .. c1-1 are final
        const PipeCtx& pp = *opt.pipe;
        const int64_t r0 = static_cast<int64_t>(c0) * VC, r1 = std::min<int64_t>(V, static_cast<int64_t>(c1) * VC);
        if (pp.section_rows) {
          pp.section_rows[k] = r0;
          pp.section_rows[k + 1] = r1;
        }
        if (cudaEventRecord(pp.p2_done[k], stream) != cudaSuccess) return cuda_fail(__LINE__);
        if (pp.h_dW) {
          if (cudaStreamWaitEvent(pp.copy, pp.p2_done[k], 0) != cudaSuccess) return cuda_fail(__LINE__);
          prof_begin(pp.copy, KIND_D2H, &slot);
          if (cudaMemcpyAsync(pp.h_dW + r0 * H, dW + r0 * H, static_cast<size_t>(r1 - r0) * H * 2,
                              cudaMemcpyDeviceToHost, pp.copy) != cudaSuccess)
            return cuda_fail(__LINE__);
          prof_end(pp.copy, slot);
        }
      }
    }
    // reordered rows: the final dX rows go back in place (no-op otherwise)
    const int sgrid = static_cast<int>(std::min<int64_t>((N + 7) / 8, static_cast<int64_t>(di.num_sms) * 8));
    prof_begin(stream, KIND_SCATTER, &slot);
    flce_dx_scatter_kernel<<<sgrid, 256, 0, stream>>>(lo, dX, perm, &ctrl->reordered, &ctrl->n_rows,
                                                      static_cast<int>(N), static_cast<int>(H));
    prof_end(stream, slot);
    if (cudaGetLastError() != cudaSuccess) return cuda_fail(__LINE__);
  }
  return FLCE_OK;
}

// Synchronous call on a workspace of `ws_bytes` bytes: enqueue, then read the
// loss and the device status back.
flce_status_t sync_call(const uint16_t* X, const uint16_t* W, const int32_t* y, int64_t N, int64_t H, int64_t V,
                        int32_t ignore_index, float* loss, uint16_t* dX, uint16_t* dW, void* workspace,
                        size_t ws_bytes, cudaStream_t stream) {
  if (!loss) return FLCE_ERR_INVALID_ARGUMENT;
  flce_status_t s = check_args(X, W, y, N, H, V, dX, dW, workspace);
  if (s != FLCE_OK) return s;
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(workspace);  // the control block opens every layout
  s = enqueue(X, W, y, N, H, V, ignore_index, &ctrl->loss, &ctrl->status, dX, dW, workspace, ws_bytes, stream);
  if (s != FLCE_OK) return s;
  Ctrl host{};
  if (cudaMemcpyAsync(&host, ctrl, sizeof(Ctrl), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return cuda_fail(__LINE__);
  if (cudaStreamSynchronize(stream) != cudaSuccess) return cuda_fail(__LINE__);
  *loss = host.loss;
  return static_cast<flce_status_t>(host.status);
}

}  // namespace

// ================================================================== C ABI ==
extern "C" {

void flce_last_cuda_error(int32_t* line, int32_t* cuda_error, const char** text) {
  if (line) *line = g_fail_line;
  if (cuda_error) *cuda_error = static_cast<int32_t>(g_fail_code);
  if (text) *text = cudaGetErrorString(g_fail_code);
}

const char* flce_status_string(int s) {
  switch (s) {
    case FLCE_OK: return "FLCE_OK";
    case FLCE_ERR_INVALID_ARGUMENT: return "FLCE_ERR_INVALID_ARGUMENT";
    case FLCE_ERR_UNSUPPORTED: return "FLCE_ERR_UNSUPPORTED";
    case FLCE_ERR_WORKSPACE_TOO_SMALL: return "FLCE_ERR_WORKSPACE_TOO_SMALL";
    case FLCE_ERR_TARGET_OUT_OF_RANGE: return "FLCE_ERR_TARGET_OUT_OF_RANGE";
    case FLCE_ERR_TIMEOUT: return "FLCE_ERR_TIMEOUT";
    case FLCE_ERR_CUDA: return "FLCE_ERR_CUDA";
    default: return "FLCE_UNKNOWN_STATUS";
  }
}

size_t flce_workspace_size(int64_t N, int64_t H, int64_t V) {
  if (check_sizes(N, H, V == 0 ? 1 : V) != FLCE_OK) return 0;
  return ws_layout(N, H).total;
}

size_t flce_workspace_size_reorder(int64_t N, int64_t H) {
  if (check_sizes(N, H, 1) != FLCE_OK) return 0;
  return ws_layout(N, H, true).total;
}

flce_status_t flce_forward_backward(const uint16_t* X, const uint16_t* W, const int32_t* y, int64_t N, int64_t H,
                                    int64_t V, int32_t ignore_index, float* loss, uint16_t* dX, uint16_t* dW,
                                    void* workspace, cudaStream_t stream) {
  if (check_sizes(N, H, V) != FLCE_OK) return check_sizes(N, H, V);
  return sync_call(X, W, y, N, H, V, ignore_index, loss, dX, dW, workspace, ws_layout(N, H).total, stream);
}

flce_status_t flce_forward_backward_async(const uint16_t* X, const uint16_t* W, const int32_t* y, int64_t N,
                                          int64_t H, int64_t V, int32_t ignore_index, float* d_loss,
                                          int32_t* d_status, uint16_t* dX, uint16_t* dW, void* workspace,
                                          size_t workspace_bytes, cudaStream_t stream) {
  if (!d_loss || !d_status) return FLCE_ERR_INVALID_ARGUMENT;
  const flce_status_t s = check_args(X, W, y, N, H, V, dX, dW, workspace);
  if (s != FLCE_OK) return s;
  if (!aligned(d_status, 4) || !aligned(d_loss, 4)) return FLCE_ERR_UNSUPPORTED;
  if (workspace_bytes < ws_layout(N, H).total) return FLCE_ERR_WORKSPACE_TOO_SMALL;
  return enqueue(X, W, y, N, H, V, ignore_index, d_loss, d_status, dX, dW, workspace, workspace_bytes, stream);
}

flce_status_t flce_forward_backward_ex(const uint16_t* X, const uint16_t* W, const int32_t* y, int64_t N, int64_t H,
                                       int64_t V, int32_t ignore_index, int32_t reduction,
                                       const float* grad_row_scale, const int32_t* d_mean_count, float* d_loss,
                                       float* d_row_loss, int32_t* d_status, uint16_t* dX, uint16_t* dW,
                                       void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!d_loss || !d_status) return FLCE_ERR_INVALID_ARGUMENT;
  if (reduction != FLCE_REDUCTION_MEAN && reduction != FLCE_REDUCTION_SUM && reduction != FLCE_REDUCTION_NONE)
    return FLCE_ERR_INVALID_ARGUMENT;
  const flce_status_t s = check_args(X, W, y, N, H, V, dX, dW, workspace, true);
  if (s != FLCE_OK) return s;
  if (!aligned(d_status, 4) || !aligned(d_loss, 4) || !aligned(d_row_loss, 4) || !aligned(grad_row_scale, 4) ||
      !aligned(d_mean_count, 4))
    return FLCE_ERR_UNSUPPORTED;
  if (workspace_bytes < ws_layout(N, H).total) return FLCE_ERR_WORKSPACE_TOO_SMALL;
  Options opt;
  opt.reduction = reduction;
  opt.grad_row_scale = reduction == FLCE_REDUCTION_NONE ? grad_row_scale : nullptr;
  opt.row_loss = d_row_loss;
  opt.mean_count = reduction == FLCE_REDUCTION_MEAN ? d_mean_count : nullptr;
  return enqueue(X, W, y, N, H, V, ignore_index, d_loss, d_status, dX, dW, workspace, workspace_bytes, stream,
                 opt);
}

size_t flce_ce_workspace_size(int64_t N, int64_t V) {
  if (N <= 0 || V <= 0 || N > (1ll << 30) || V > (1ll << 30)) return 0;
  return ce_ws_layout(N).total;
}

flce_status_t flce_cross_entropy(const uint16_t* logits, const int32_t* y, int64_t N, int64_t V,
                                 int32_t ignore_index, int32_t reduction, const float* grad_row_scale,
                                 float* d_loss, float* d_row_loss, int32_t* d_status, uint16_t* dlogits,
                                 void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (N <= 0 || V <= 0 || N > (1ll << 30) || V > (1ll << 30)) return FLCE_ERR_INVALID_ARGUMENT;
  if (!logits || !y || !d_loss || !d_status || !workspace) return FLCE_ERR_INVALID_ARGUMENT;
  if (reduction != FLCE_REDUCTION_MEAN && reduction != FLCE_REDUCTION_SUM && reduction != FLCE_REDUCTION_NONE)
    return FLCE_ERR_INVALID_ARGUMENT;
  if (!aligned(logits, 2) || !aligned(dlogits, 2) || !aligned(y, 4) || !aligned(workspace, 256) ||
      !aligned(d_loss, 4) || !aligned(d_status, 4) || !aligned(d_row_loss, 4) || !aligned(grad_row_scale, 4))
    return FLCE_ERR_UNSUPPORTED;
  const CeLayout L = ce_ws_layout(N);
  if (workspace_bytes < L.total) return FLCE_ERR_WORKSPACE_TOO_SMALL;
  DevInfo di;
  int dev;
  if (device_info(&di, &dev) != cudaSuccess) return cuda_fail(__LINE__);
  if (!di.sm100) return FLCE_ERR_UNSUPPORTED;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int TM = static_cast<int>((N + CM - 1) / CM);
  if (cudaMemsetAsync(ws + L.ctrl, 0, 256, stream) != cudaSuccess ||
      cudaMemsetAsync(d_status, 0, sizeof(int32_t), stream) != cudaSuccess)
    return cuda_fail(__LINE__);
  CeArgs c{};
  c.logits = logits;
  c.dlogits = dlogits;
  c.y = y;
  c.N = static_cast<int>(N);
  c.V = static_cast<int>(V);
  c.ignore_index = ignore_index;
  c.reduction = reduction;
  c.TM = TM;
  c.grad_row_scale = reduction == FLCE_REDUCTION_NONE ? grad_row_scale : nullptr;
  c.tile_valid = reinterpret_cast<const int*>(ws + L.tile_valid);
  c.row_acc = reinterpret_cast<double*>(ws + L.row_acc);
  c.row_loss = d_row_loss;
  c.blk_sum = reinterpret_cast<double*>(ws + L.blk_sum);
  c.ticket = reinterpret_cast<unsigned int*>(ws + L.ctrl + 4);
  c.n_valid = reinterpret_cast<const int*>(ws + L.ctrl + 8);
  c.loss = d_loss;
  c.status = d_status;
  size_t slot;
  prof_begin(stream, KIND_PREP, &slot);
  flce_prep_kernel<<<TM, CM, 0, stream>>>(y, c.N, ignore_index, reinterpret_cast<int*>(ws + L.tile_valid),
                                          reinterpret_cast<int*>(ws + L.ctrl + 8));
  prof_end(stream, slot);
  if (cudaGetLastError() != cudaSuccess) return cuda_fail(__LINE__);
  const int grid = static_cast<int>(std::min<int64_t>(N, static_cast<int64_t>(di.num_sms) * 4 * 64));
  prof_begin(stream, KIND_CE, &slot);
  flce_ce_rows_kernel<<<grid, CE_THREADS, 0, stream>>>(c);
  prof_end(stream, slot);
  if (cudaGetLastError() != cudaSuccess) return cuda_fail(__LINE__);
  prof_begin(stream, KIND_COMBINE, &slot);
  flce_ce_reduce_kernel<<<static_cast<int>((N + COMBINE_THREADS - 1) / COMBINE_THREADS), COMBINE_THREADS, 0, stream>>>(c);
  prof_end(stream, slot);
  if (cudaGetLastError() != cudaSuccess) return cuda_fail(__LINE__);
  return FLCE_OK;
}

flce_status_t flce_count_valid(const int32_t* y, int64_t N, int32_t ignore_index, int32_t* d_count,
                               cudaStream_t stream) {
  if (!y || !d_count || N <= 0 || N > (1ll << 30)) return FLCE_ERR_INVALID_ARGUMENT;
  if (!aligned(y, 4) || !aligned(d_count, 4)) return FLCE_ERR_UNSUPPORTED;
  DevInfo di;
  int dev;
  if (device_info(&di, &dev) != cudaSuccess) return cuda_fail(__LINE__);
  if (!di.sm100) return FLCE_ERR_UNSUPPORTED;
  if (cudaMemsetAsync(d_count, 0, sizeof(int32_t), stream) != cudaSuccess) return cuda_fail(__LINE__);
  const int tiles = static_cast<int>((N + CM - 1) / CM);
  size_t slot;
  prof_begin(stream, KIND_PREP, &slot);
  flce_prep_kernel<<<tiles, CM, 0, stream>>>(y, static_cast<int>(N), ignore_index, nullptr, d_count);
  prof_end(stream, slot);
  return cudaGetLastError() == cudaSuccess ? FLCE_OK : cuda_fail(__LINE__);
}

flce_status_t flce_pairwise_logistic(const float* d_row_loss, const int32_t* y, int64_t N, int32_t ignore_index,
                                     const int32_t* d_seq_start, int32_t S, const int32_t* d_chosen,
                                     const int32_t* d_rejected, int32_t P, double beta, const double* d_ref_logp,
                                     double* d_loss, double* d_logp, double* d_grad_logp, float* d_row_weight,
                                     int32_t* d_status, cudaStream_t stream) {
  if (!d_row_loss || !y || !d_seq_start || !d_chosen || !d_rejected || !d_loss || !d_logp || !d_grad_logp ||
      !d_row_weight || !d_status)
    return FLCE_ERR_INVALID_ARGUMENT;
  if (N <= 0 || N > (1ll << 30) || S <= 0 || S > (1 << 24) || P <= 0 || P > (1 << 24) || !(beta == beta))
    return FLCE_ERR_INVALID_ARGUMENT;
  if (!aligned(d_row_loss, 4) || !aligned(y, 4) || !aligned(d_seq_start, 4) || !aligned(d_chosen, 4) ||
      !aligned(d_rejected, 4) || !aligned(d_ref_logp, 8) || !aligned(d_loss, 8) || !aligned(d_logp, 8) ||
      !aligned(d_grad_logp, 8) || !aligned(d_row_weight, 4) || !aligned(d_status, 4))
    return FLCE_ERR_UNSUPPORTED;
  DevInfo di;
  int dev;
  if (device_info(&di, &dev) != cudaSuccess) return cuda_fail(__LINE__);
  if (!di.sm100) return FLCE_ERR_UNSUPPORTED;
  if (cudaMemsetAsync(d_status, 0, sizeof(int32_t), stream) != cudaSuccess ||
      cudaMemsetAsync(d_row_weight, 0, static_cast<size_t>(N) * sizeof(float), stream) != cudaSuccess)
    return cuda_fail(__LINE__);
  PrefArgs a{};
  a.row_loss = d_row_loss;
  a.y = y;
  a.seq_start = d_seq_start;
  a.chosen = d_chosen;
  a.rejected = d_rejected;
  a.ref_logp = d_ref_logp;
  a.beta = beta;
  a.N = static_cast<int>(N);
  a.S = S;
  a.P = P;
  a.ignore_index = ignore_index;
  a.logp = d_logp;
  a.grad_logp = d_grad_logp;
  a.loss = d_loss;
  a.row_weight = d_row_weight;
  a.status = d_status;
  flce_pref_logp_kernel<<<S, PREF_THREADS, 0, stream>>>(a);
  if (cudaGetLastError() != cudaSuccess) return cuda_fail(__LINE__);
  flce_pref_pairs_kernel<<<1, PREF_THREADS, 0, stream>>>(a);
  if (cudaGetLastError() != cudaSuccess) return cuda_fail(__LINE__);
  flce_pref_weights_kernel<<<S, PREF_THREADS, 0, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? FLCE_OK : cuda_fail(__LINE__);
}

namespace {
flce_status_t check_shard(int64_t V_shard, int64_t v0, int64_t V) {
  if (v0 < 0 || V <= 0 || V > (1ll << 30) || v0 + V_shard > V) return FLCE_ERR_INVALID_ARGUMENT;
  return FLCE_OK;
}
}  // namespace

flce_status_t flce_vp_shard_stats(const uint16_t* X, const uint16_t* W_shard, const int32_t* y, int64_t N,
                                  int64_t H, int64_t V_shard, int64_t v0, int64_t V, int32_t ignore_index,
                                  float* d_shard_lse, float* d_shard_zy, int32_t* d_status, void* workspace,
                                  size_t workspace_bytes, cudaStream_t stream) {
  if (!d_shard_lse || !d_shard_zy || !d_status) return FLCE_ERR_INVALID_ARGUMENT;
  flce_status_t s = check_args(X, W_shard, y, N, H, V_shard, nullptr, nullptr, workspace, true);
  if (s == FLCE_OK) s = check_shard(V_shard, v0, V);
  if (s != FLCE_OK) return s;
  if (!aligned(d_shard_lse, 4) || !aligned(d_shard_zy, 4) || !aligned(d_status, 4)) return FLCE_ERR_UNSUPPORTED;
  if (workspace_bytes < ws_layout(N, H).total) return FLCE_ERR_WORKSPACE_TOO_SMALL;
  Options opt;
  opt.combine = COMBINE_SHARD;
  opt.v0 = v0;
  opt.V_total = V;
  opt.shard_lse = d_shard_lse;
  opt.shard_zy = d_shard_zy;
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(workspace);  // the loss slot is unused by this step
  return enqueue(X, W_shard, y, N, H, V_shard, ignore_index, &ctrl->loss, d_status, nullptr, nullptr, workspace,
                 workspace_bytes, stream, opt);
}

flce_status_t flce_vp_backward(const uint16_t* X, const uint16_t* W_shard, const int32_t* y, int64_t N, int64_t H,
                               int64_t V_shard, int64_t v0, int64_t V, int32_t ignore_index, int32_t shards,
                               const float* d_all_lse, const float* d_all_zy, const int32_t* d_mean_count,
                               float* d_loss, int32_t* d_status, uint16_t* dX_part, uint16_t* dW_shard,
                               void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!d_all_lse || !d_all_zy || !d_loss || !d_status || shards < 1) return FLCE_ERR_INVALID_ARGUMENT;
  flce_status_t s = check_args(X, W_shard, y, N, H, V_shard, dX_part, dW_shard, workspace, true);
  if (s == FLCE_OK) s = check_shard(V_shard, v0, V);
  if (s != FLCE_OK) return s;
  if (!aligned(d_all_lse, 4) || !aligned(d_all_zy, 4) || !aligned(d_loss, 4) || !aligned(d_status, 4) ||
      !aligned(d_mean_count, 4))
    return FLCE_ERR_UNSUPPORTED;
  if (workspace_bytes < ws_layout(N, H).total) return FLCE_ERR_WORKSPACE_TOO_SMALL;
  Options opt;
  opt.combine = COMBINE_SHARDS_IN;
  opt.v0 = v0;
  opt.V_total = V;
  opt.shards = shards;
  opt.all_lse = d_all_lse;
  opt.all_zy = d_all_zy;
  opt.mean_count = d_mean_count;
  return enqueue(X, W_shard, y, N, H, V_shard, ignore_index, d_loss, d_status, dX_part, dW_shard, workspace,
                 workspace_bytes, stream, opt);
}

flce_status_t flce_probe_bounded_wait(int64_t timeout_ns, int32_t* d_status, cudaStream_t stream) {
  if (!d_status || timeout_ns <= 0 || timeout_ns > 10000000000ll) return FLCE_ERR_INVALID_ARGUMENT;
  if (!aligned(d_status, 4)) return FLCE_ERR_UNSUPPORTED;
  DevInfo di;
  int dev;
  if (device_info(&di, &dev) != cudaSuccess) return cuda_fail(__LINE__);
  if (!di.sm100) return FLCE_ERR_UNSUPPORTED;
  // d_status[0], d_status[1]: the two waits' results; d_status[2]: the counter nobody sets
  if (cudaMemsetAsync(d_status, 0, 3 * sizeof(int32_t), stream) != cudaSuccess) return cuda_fail(__LINE__);
  flce_wait_probe_kernel<<<1, 32, 0, stream>>>(d_status, d_status + 2, static_cast<unsigned long long>(timeout_ns));
  return cudaGetLastError() == cudaSuccess ? FLCE_OK : cuda_fail(__LINE__);
}

flce_status_t flce_probe_pass2_timeout(const uint16_t* X, const uint16_t* W, const int32_t* y, int64_t N, int64_t H,
                                       int64_t V, int32_t ignore_index, float* d_loss, int32_t* d_status,
                                       uint16_t* dX, uint16_t* dW, void* workspace, size_t workspace_bytes,
                                       int64_t timeout_ns, cudaStream_t stream) {
  if (!d_loss || !d_status || timeout_ns <= 0 || timeout_ns > 10000000000ll) return FLCE_ERR_INVALID_ARGUMENT;
  const flce_status_t s = check_args(X, W, y, N, H, V, dX, dW, workspace);
  if (s != FLCE_OK) return s;
  if (!aligned(d_status, 4) || !aligned(d_loss, 4)) return FLCE_ERR_UNSUPPORTED;
  if (workspace_bytes < ws_layout(N, H).total) return FLCE_ERR_WORKSPACE_TOO_SMALL;
  Options opt;
  opt.timeout_ns = static_cast<unsigned long long>(timeout_ns);
  opt.starve_dw = 1;
  return enqueue(X, W, y, N, H, V, ignore_index, d_loss, d_status, dX, dW, workspace, workspace_bytes, stream, opt);
}

flce_status_t flce_forward_backward_host(const uint16_t* h_X, const uint16_t* h_W, const int32_t* h_y, int64_t N,
                                         int64_t H, int64_t V, int32_t ignore_index, float* h_loss, uint16_t* h_dX,
                                         uint16_t* h_dW, uint16_t* d_X, uint16_t* d_W, int32_t* d_y,
                                         uint16_t* d_dX, uint16_t* d_dW, void* workspace, size_t workspace_bytes,
                                         cudaStream_t stream) {
  if (!h_X || !h_W || !h_y || !h_loss || !h_dX || !h_dW) return FLCE_ERR_INVALID_ARGUMENT;
  flce_status_t s = check_args(d_X, d_W, d_y, N, H, V, d_dX, d_dW, workspace);
  if (s != FLCE_OK) return s;
  if (workspace_bytes < ws_layout(N, H).total) return FLCE_ERR_WORKSPACE_TOO_SMALL;
  PipeRes* pr = nullptr;
  if (pipe_resources(&pr) != cudaSuccess) return cuda_fail(__LINE__);
  std::lock_guard<std::mutex> lk(pr->mu);  // one host-buffer call per device at a time: shared copy stream
  const size_t xb = static_cast<size_t>(N) * H * 2, yb = N * 4;
  // X and y first, on the caller's stream: every kernel needs them
  size_t slot;
  prof_begin(stream, KIND_H2D, &slot);
  if (cudaMemcpyAsync(d_X, h_X, xb, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
      cudaMemcpyAsync(d_y, h_y, yb, cudaMemcpyHostToDevice, stream) != cudaSuccess)
    return cuda_fail(__LINE__);
  prof_end(stream, slot);
  // W in pieces on the copy stream, which starts after the caller's earlier work
  PipeCtx pp;
  pp.copy = pr->copy;
  const int64_t vt = (V + BN - 1) / BN;
  pp.pieces = static_cast<int>(std::min<int64_t>(MAX_PIECES, vt));
  for (int i = 0; i <= pp.pieces; ++i) pp.piece_v[i] = std::min<int64_t>(V, (vt * i / pp.pieces) * BN);
  pp.groups = MAX_PIECES;
  pp.h_dW = h_dW;
  if (cudaEventRecord(pr->start, stream) != cudaSuccess || cudaStreamWaitEvent(pr->copy, pr->start, 0) != cudaSuccess)
    return cuda_fail(__LINE__);
  for (int i = 0; i < pp.pieces; ++i) {
    const int64_t v0 = pp.piece_v[i], v1 = pp.piece_v[i + 1];
    pp.w_ready[i] = pr->ev[i];
    pp.p2_done[i] = pr->ev[MAX_PIECES + i];
    prof_begin(pr->copy, KIND_H2D, &slot);
    if (cudaMemcpyAsync(d_W + v0 * H, h_W + v0 * H, static_cast<size_t>(v1 - v0) * H * 2, cudaMemcpyHostToDevice,
                        pr->copy) != cudaSuccess)
      return cuda_fail(__LINE__);
    prof_end(pr->copy, slot);
    if (cudaEventRecord(pp.w_ready[i], pr->copy) != cudaSuccess) return cuda_fail(__LINE__);
  }
  for (int i = pp.pieces; i < MAX_PIECES; ++i) pp.p2_done[i] = pr->ev[MAX_PIECES + i];
  Options opt;
  opt.pipe = &pp;
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(workspace);  // the control block opens every layout
  s = enqueue(d_X, d_W, d_y, N, H, V, ignore_index, &ctrl->loss, &ctrl->status, d_dX, d_dW, workspace,
              workspace_bytes, stream, opt);
  if (s != FLCE_OK) {
    cudaStreamSynchronize(pr->copy);
    return s;
  }
  // dX and the control block on the caller's stream; dW went back section by section
  Ctrl host{};
  prof_begin(stream, KIND_D2H, &slot);
  if (cudaMemcpyAsync(h_dX, d_dX, xb, cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
      cudaMemcpyAsync(&host, ctrl, sizeof(Ctrl), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return cuda_fail(__LINE__);
  prof_end(stream, slot);
  if (cudaEventRecord(pr->done, pr->copy) != cudaSuccess || cudaStreamWaitEvent(stream, pr->done, 0) != cudaSuccess)
    return cuda_fail(__LINE__);
  if (cudaStreamSynchronize(stream) != cudaSuccess) return cuda_fail(__LINE__);
  *h_loss = host.loss;
  return static_cast<flce_status_t>(host.status);
}

flce_status_t flce_forward_backward_sections(const uint16_t* X, const uint16_t* W, const int32_t* y, int64_t N,
                                             int64_t H, int64_t V, int32_t ignore_index, const int32_t* d_mean_count,
                                             float* d_loss, int32_t* d_status, uint16_t* dX, uint16_t* dW,
                                             void* workspace, size_t workspace_bytes, int32_t sections,
                                             cudaEvent_t* section_done, int64_t* section_rows, cudaStream_t stream) {
  if (!d_loss || !d_status || !section_done || !section_rows || sections < 1 || sections > MAX_PIECES)
    return FLCE_ERR_INVALID_ARGUMENT;
  for (int k = 0; k < sections; ++k)
    if (!section_done[k]) return FLCE_ERR_INVALID_ARGUMENT;
  const flce_status_t s = check_args(X, W, y, N, H, V, dX, dW, workspace);
  if (s != FLCE_OK) return s;
  if (!aligned(d_status, 4) || !aligned(d_loss, 4) || !aligned(d_mean_count, 4)) return FLCE_ERR_UNSUPPORTED;
  if (workspace_bytes < ws_layout(N, H).total) return FLCE_ERR_WORKSPACE_TOO_SMALL;
  const int chunks = static_cast<int>((V + VC - 1) / VC);
  const int used = std::min(sections, chunks);
  PipeCtx pp;
  pp.pieces = 0;  // pass 1 in one launch: W is on the device already
  pp.groups = used;
  pp.section_rows = section_rows;
  for (int k = 0; k < used; ++k) pp.p2_done[k] = section_done[k];
  Options opt;
  opt.mean_count = d_mean_count;
  opt.pipe = &pp;
  const flce_status_t e = enqueue(X, W, y, N, H, V, ignore_index, d_loss, d_status, dX, dW, workspace,
                                  workspace_bytes, stream, opt);
  if (e != FLCE_OK) return e;
  // sections beyond the chunks hold no rows and are done with the last one
  for (int k = used; k < sections; ++k) {
    section_rows[k + 1] = V;
    if (cudaEventRecord(section_done[k], stream) != cudaSuccess) return cuda_fail(__LINE__);
  }
  return FLCE_OK;
}

flce_status_t flce_plan(int64_t N, int64_t H, int64_t V, flce_plan_t* out) {
  if (!out) return FLCE_ERR_INVALID_ARGUMENT;
  const flce_status_t s = check_sizes(N, H, V);
  if (s != FLCE_OK) return s;
  int sms = 148, clusters = 74;
  DevInfo di;
  int dev;
  if (device_info(&di, &dev) == cudaSuccess && di.num_sms > 0) {
    sms = di.num_sms;
    if (di.sm100 && set_kernel_attrs(dev) == cudaSuccess && device_info(&di, &dev) == cudaSuccess)
      clusters = di.max_clusters;
    else
      clusters = sms / CLUSTER;
  }
  const Plan P = make_plan(N, H, V, clusters);
  out->workspace_bytes = static_cast<int64_t>(ws_layout(N, H).total);
  out->workspace_reorder_bytes = static_cast<int64_t>(ws_layout(N, H, true).total);
  out->vocab_chunk = VC;
  out->num_chunks = P.num_chunks;
  out->lse_splits = P.splits;
  out->launches = P.launches;
  out->num_sms = sms;
  return FLCE_OK;
}

const char* flce_kernel_name(int kind) {
  switch (kind) {
    case KIND_LSE: return "pass1_logits_lse";
    case KIND_COMBINE: return "combine_lse_loss";
    case KIND_PASS2: return "pass2_grad_dw_dx";
    case KIND_PREP: return "prep_tile_valid";
    case KIND_CE: return "ce_on_logits_rows";
    case KIND_ORDER: return "prep_row_order";
    case KIND_SCATTER: return "dx_row_scatter";
    case KIND_PACK: return "prep_pack_rows";
    case KIND_H2D: return "copy_host_to_device";
    case KIND_D2H: return "copy_device_to_host";
    default: return "unknown";
  }
}

flce_status_t flce_profile_enable(int on) {
  if (on && g_prof.ev.empty()) {
    g_prof.ev.resize(2 * PROF_PAIRS);
    g_prof.kind.resize(PROF_PAIRS);
    for (auto& e : g_prof.ev)
      if (cudaEventCreate(&e) != cudaSuccess) return cuda_fail(__LINE__);
  }
  g_prof.on = on != 0;
  g_prof.used = 0;
  return FLCE_OK;
}

flce_status_t flce_row_order_info(const void* workspace, int32_t* reordered, int32_t* n_valid,
                                  cudaStream_t stream) {
  if (!workspace || !reordered || !n_valid || !aligned(workspace, 256)) return FLCE_ERR_INVALID_ARGUMENT;
  Ctrl host{};
  if (cudaMemcpyAsync(&host, workspace, sizeof(Ctrl), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
      cudaStreamSynchronize(stream) != cudaSuccess)
    return cuda_fail(__LINE__);
  *reordered = host.reordered;
  *n_valid = host.n_rows;
  return FLCE_OK;
}

flce_status_t flce_profile_read(int32_t* launches, double* total_ms) {
  if (!launches || !total_ms) return FLCE_ERR_INVALID_ARGUMENT;
  for (int k = 0; k < FLCE_NUM_KERNEL_KINDS; ++k) {
    launches[k] = 0;
    total_ms[k] = 0.0;
  }
  for (size_t i = 0; i < g_prof.used; ++i) {
    if (g_prof.kind[i] >= FLCE_NUM_KERNEL_KINDS) continue;  // copies: see flce_profile_timeline
    if (cudaEventSynchronize(g_prof.ev[2 * i + 1]) != cudaSuccess) return cuda_fail(__LINE__);
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, g_prof.ev[2 * i], g_prof.ev[2 * i + 1]) != cudaSuccess) return cuda_fail(__LINE__);
    launches[g_prof.kind[i]] += 1;
    total_ms[g_prof.kind[i]] += ms;
  }
  g_prof.used = 0;
  return FLCE_OK;
}

flce_status_t flce_profile_timeline(int32_t* kinds, double* begin_ms, double* end_ms, int32_t capacity,
                                    int32_t* count) {
  if (!kinds || !begin_ms || !end_ms || !count || capacity < 0) return FLCE_ERR_INVALID_ARGUMENT;
  *count = static_cast<int32_t>(g_prof.used);
  for (size_t i = 0; i < g_prof.used; ++i) {
    if (cudaEventSynchronize(g_prof.ev[2 * i + 1]) != cudaSuccess) return cuda_fail(__LINE__);
    if (static_cast<int64_t>(i) >= capacity) continue;
    float b = 0.f, e = 0.f;
    if (cudaEventElapsedTime(&b, g_prof.ev[0], g_prof.ev[2 * i]) != cudaSuccess ||
        cudaEventElapsedTime(&e, g_prof.ev[0], g_prof.ev[2 * i + 1]) != cudaSuccess)
      return cuda_fail(__LINE__);
    kinds[i] = g_prof.kind[i];
    begin_ms[i] = b;
    end_ms[i] = e;
  }
  g_prof.used = 0;
  return FLCE_OK;
}

}  // extern "C"

// ============================================================ no-alloc entry ==
// Scratch of flce_forward_backward_noalloc.  It is part of the library's device
// module, so a caller of that entry never needs an allocation.  In host code
// the name stands for a host-side shadow; the device address comes from
// cudaGetSymbolAddress, looked up once per device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[FLCE_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_noalloc_mu;
void* g_noalloc_addr[64];

cudaError_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return cudaSuccess;
}
}  // namespace

extern "C" flce_status_t flce_forward_backward_noalloc(const uint16_t* X, const uint16_t* W, const int32_t* y,
                                                       int64_t N, int64_t H, int64_t V, int32_t ignore_index,
                                                       float* loss, uint16_t* dX, uint16_t* dW,
                                                       cudaStream_t stream) {
  if (!loss) return FLCE_ERR_INVALID_ARGUMENT;
  const flce_status_t s = check_sizes(N, H, V);
  if (s != FLCE_OK) return s;
  if (ws_layout(N, H).total > static_cast<size_t>(FLCE_NOALLOC_SCRATCH_BYTES)) return FLCE_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  if (noalloc_scratch(&scratch) != cudaSuccess) return cuda_fail(__LINE__);
  return sync_call(X, W, y, N, H, V, ignore_index, loss, dX, dW, scratch, FLCE_NOALLOC_SCRATCH_BYTES, stream);
}
