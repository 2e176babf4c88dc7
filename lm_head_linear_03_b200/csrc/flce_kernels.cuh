// Device code of the fused linear + cross-entropy head.
//
// One persistent, warp-specialised tcgen05 GEMM template serves all four
// tensor-core steps; they differ in which operands the TMA engine streams in,
// in which of them are MN-major, and in the epilogue that turns the fp32
// accumulator tile in tensor memory into the step's output:
//
//   KIND_LSE  (pass 1)  z = X W^T per [128 tokens x 256 vocab] tile; the
//                       epilogue keeps an online row max and sum of
//                       exponentials over the tiles of one vocabulary split and
//                       picks out the target logit.  No logit leaves the chip.
//   KIND_GRAD (pass 2)  recomputes the logits of one vocabulary chunk and writes
//                       G = (softmax - onehot) / n in bf16 into the chunk buffer.
//   KIND_DW             dW[chunk rows] = G_c^T X       (K = tokens)
//   KIND_DX             dX += G_c W_c                  (K = chunk vocabulary)
//
// These follow the pages' description of the fused head: the loss and its
// gradient are computed chunk by chunk over the vocabulary, the logits are
// recomputed rather than stored ("Liger Kernel explained", cross-entropy head
// section), and the (batch, sequence, vocab) tensor is never allocated
// ("Liger-Kernel: Triton kernels that replace HF training ops", section "What
// actually gets replaced").
//
// The CTAs run in pairs (clusters of two on neighbouring SMs).  A pair owns one
// 256 x 256 accumulator tile: each CTA loads 128 rows of A and 128 columns of B
// into its own shared memory, the leader CTA issues cta_group::2 UMMAs that read
// both halves, and each CTA's tensor memory receives its 128 rows.  Per SM this
// halves the B-operand traffic of a 128 x 256 single-CTA tile.  Pass 1, and
// pass 2's dW items where its queue pairs them, take two adjacent 256-column
// tiles as one 256 x 512 tile in both accumulator buffers: two UMMAs per
// k-block share the A tile, so a k-block reads 48 KB of operands for twice
// the work of a 32 KB one (see the pass-1 issuer and the pass-2 queue).
//
// Warp roles (192 threads per CTA): warp 0 issues TMA loads, warp 1 issues UMMAs
// (leader CTA only) and owns the tensor-memory allocation, warps 2..5 run the
// epilogue (warp w reads TMEM lanes 32*(w%4) .. 32*(w%4)+31, one accumulator row
// per thread).
#pragma once

#include <cfloat>
#include <cstdint>

#include "sm100.cuh"

namespace flce {

constexpr int CLUSTER = 2;     // SM pair: the two CTAs of a cluster share one UMMA tile
constexpr int BM = 128;        // accumulator rows per CTA (TMEM lanes)
constexpr int CM = CLUSTER * BM;  // rows of the pair's tile (UMMA M = 256)
constexpr int BN = 256;        // accumulator columns (UMMA N)
constexpr int BNH = BN / CLUSTER; // B columns each CTA of the pair holds
constexpr int BK = 64;         // K per pipeline stage: one 128-B swizzle row of bf16
constexpr int UMMA_K = 16;     // K per tcgen05.mma kind::f16
constexpr int STAGES = 6;
constexpr int A_TILE_BYTES = BM * BK * 2;
constexpr int B_TILE_BYTES = BNH * BK * 2;
constexpr int STAGE_BYTES = A_TILE_BYTES + B_TILE_BYTES;
constexpr int MN_BOX_BYTES = 64 * BK * 2;  // one 64(MN) x 64(K) MN-major box
constexpr int NUM_THREADS = 192;
constexpr int EPI_WARPS = 4;
constexpr int ACC_COLS = BN;
constexpr int TMEM_COLS = 2 * ACC_COLS;    // double-buffered accumulator
// Epilogue staging: each epilogue warp owns two 4 KB buffers, each holding a
// 32-row x 32-column bf16 box of the output (and, for dX, of the low half of
// the running sum), stored with the 64-byte TMA swizzle.
constexpr int EPI_BOX = 32;
constexpr int EPI_BOX_BYTES = EPI_BOX * EPI_BOX * 2;
constexpr int EPI_BUF_BYTES = 2 * EPI_BOX_BYTES;
constexpr int EPI_WARP_BYTES = 2 * EPI_BUF_BYTES;
constexpr int EPI_BYTES = EPI_WARPS * EPI_WARP_BYTES;
// barrier slots: full[STAGES], empty[STAGES], tfull[2], tempty[2], fin, epilogue loads[2 per warp], drain
constexpr int BAR_DRAIN = 2 * STAGES + 5 + 2 * EPI_WARPS;
constexpr int NUM_BARRIERS = BAR_DRAIN + 1;
// words after the barriers: tensor-memory address, abort flag, ring positions
// the producer filled and the issuer consumed
constexpr int SLOT_WORDS = 4;
static_assert(NUM_BARRIERS * 8 + SLOT_WORDS * 4 <= 256, "barrier area");
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + 1024 /*alignment*/ + 256 /*barriers*/;
// Pass 1 takes adjacent vocabulary tiles in pairs, as one 256 x 512 tile in
// both accumulator buffers: its stages hold this CTA's X tile and the W tiles
// of both halves (48 KB), four of them in the same bytes as pass 2's six.  A
// stage thus holds 1024 tensor-core cycles of work instead of 512, and the
// loads in flight cover their latency.  Pass 1 stages nothing through shared
// memory in its epilogue and needs no staging area.
constexpr int P1_STAGES = 4;
constexpr int P1_STAGE_BYTES = A_TILE_BYTES + 2 * B_TILE_BYTES;
constexpr int P1_SMEM_BYTES = P1_STAGES * P1_STAGE_BYTES + 1024 /*alignment*/ + 256 /*barriers*/;
static_assert(P1_STAGES <= STAGES, "pass 1 uses the first barriers of pass 2's layout");
// k-blocks a tile pair runs on its first half alone (see the pass-1 issuer)
constexpr int P1_LEAD = 8;
constexpr float LOG2E = 1.4426950408889634f;
constexpr double LN2 = 0.6931471805599453;

// Reductions: the loss is sum_i s_i l_i over valid rows with s_i = 1/n, 1, or
// the caller's per-row upstream gradient.
enum : int { RED_MEAN = 0, RED_SUM = 1, RED_NONE = 2 };

// Per-row weight s_i of a valid row (the reduction's scale of its loss and of its G row).
__device__ __forceinline__ float row_weight(int reduction, const float* inv_n, const float* grad_row_scale, int row) {
  if (reduction == RED_MEAN) return *inv_n;
  if (reduction == RED_SUM) return 1.f;
  return grad_row_scale ? grad_row_scale[row] : 1.f;
}

// Target of a valid row whose vocabulary entry lies in another shard: far
// above any column index, and never equal to ignore_index.
__host__ __device__ __forceinline__ int target_elsewhere(int ignore_index) {
  return ignore_index == 0x7fffffff ? 0x7ffffffe : 0x7fffffff;
}

// Kinds of launch, as the profiler reports them.
enum : int {
  KIND_LSE = 0, KIND_COMBINE = 1, KIND_PASS2 = 2, KIND_PREP = 3, KIND_CE = 4, KIND_ORDER = 5, KIND_SCATTER = 6,
  KIND_PACK = 7, KIND_H2D = 8, KIND_D2H = 9  // the last two: copies of the host-buffer entry (profiling only)
};
enum : int { ST_TARGET_OUT_OF_RANGE = 4, ST_TIMEOUT = 5 };

struct GemmArgs {
  int N, H, V, ignore_index;
  int tiles_m, tiles_n;   // pass 1: 256-token tiles, 256-wide vocabulary tiles
  int k_blocks;           // pass 1: BK-wide steps along K = H
  int num_units;          // pass 1: tiles_m * splits
  int splits;             // pass 1: vocabulary splits
  int v_off;              // pass 1: vocabulary id of W's row 0 (a launch over a range of the vocabulary)
  int split_off;          // pass 1: first partial slot of this launch's splits
  int Vc;                 // pass 2: chunk width = row stride of the G buffer
  const int32_t* y;
  float* part_m;          // [splits][N] running max, log2 units
  float* part_l;          // [splits][N] running sum of 2^(s - m)
  float* zy;              // [N] target logit
  const float* lse2;      // [N] log2-sum-exp2 of z*log2(e)
  const float* inv_n;     // 1 / n_valid (0 when n_valid = 0)
  uint16_t* G;            // [N][Vc] bf16
  uint16_t* dW;           // [V][H] bf16
  uint16_t* dX;           // [N][H] bf16, also the high half of the dX accumulator
  uint16_t* lo;           // [N][H] bf16, low half of the dX accumulator
  int* status;
  unsigned long long timeout_ns;
  int starve_dw;          // failure probe only: dW mainloops wait for one G tile more than exist
  int g_cols_first;       // G(c): this many vocabulary tiles first, column by column; the rest row by row
  int reduction;                 // RED_MEAN, RED_SUM, RED_NONE
  const float* grad_row_scale;   // RED_NONE: per-row upstream gradient, or null for 1
  const int* tile_valid;         // [ceil(N/256)] valid rows per 256-row token tile (prep kernel)
  // Token-row order.  When the rows of ignored targets are scattered, the rows
  // are reordered so that every valid row comes first (a stable partition);
  // then perm[r] is the row of X behind row r, the GEMMs read a packed copy of
  // X in that order (same TMA tiles), and y, the upstream weights and every
  // output row of the workspace follow the new order.
  const int* perm;               // [ceil(N/256)*256] row of X behind each row
  const int* reordered;          // device word: 1 when the rows are reordered
  // pass 2 (one persistent launch over every chunk)
  int TM, HN;             // 256-row token tiles, 256-column hidden tiles
  int HW;                 // dW items per vocabulary tile: hidden tiles in pairs, the last alone when HN is odd
  int dw_lead;            // active k-blocks a paired dW item runs on its first half alone (see the issuer)
  int C;                  // vocabulary chunks
  int VTf, VT_last;       // 256-wide vocabulary tiles in a full / the last chunk
  long long total_items;
  long long item_begin, item_end;  // the items of the queue this launch runs
  int* g_row;             // [TM]  G tiles finished per token tile    (x EPI_WARPS*CLUSTER)
  int* g_col;             // [VTf] G tiles finished per chunk column  (x EPI_WARPS*CLUSTER)
  int* x_row;             // [TM]  dX tiles finished per token tile   (x EPI_WARPS*CLUSTER)
  int* w_col;             // [VTf] dW tiles finished per chunk column (x EPI_WARPS*CLUSTER)
};

__device__ __forceinline__ void raise_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// A wait of one CTA of an SM pair gave up: both CTAs wind down at once (the
// peer's roles see the flag in their next wait), so the pair reaches the
// end-of-kernel handshake together and neither CTA leaves while the other may
// still reach into its shared memory.  The handshake allows END_WAIT_LIMITS
// wait limits, more than the one wait a CTA can still be in when the other
// arrives.
constexpr unsigned long long END_WAIT_LIMITS = 4;
__device__ __forceinline__ void give_up_pair(volatile int* abort_flag, int rank, int* status) {
  *abort_flag = 1;
  st_cluster_u32(mapa_shared(smem_u32(const_cast<int*>(abort_flag)), static_cast<uint32_t>(rank ^ 1)), 1u);
  raise_status(status, ST_TIMEOUT);
}

// Pass-1 work unit u -> token tile mb, vocabulary split `split` and the range
// [nb_begin, nb_end) of 256-wide vocabulary tiles it walks.  Units are ordered
// split-major, so that SM pairs running at the same time share the same W
// tiles through L2.
__device__ __forceinline__ void unit_range(const GemmArgs& a, int u, int& mb, int& nb_begin, int& nb_end,
                                           int& split) {
  split = u / a.tiles_m;
  mb = u - split * a.tiles_m;
  nb_begin = static_cast<int>((static_cast<long long>(split) * a.tiles_n) / a.splits);
  nb_end = static_cast<int>((static_cast<long long>(split + 1) * a.tiles_n) / a.splits);
}

template <bool MN>
__device__ __forceinline__ uint64_t operand_desc(uint32_t base, int k) {
  if constexpr (MN)
    return sdesc_sw128(base + k * (UMMA_K * 128), MN_BOX_BYTES, 1024);
  else
    return sdesc_sw128(base + k * (UMMA_K * 2), 16, 1024);
}

// ------------------------------------------------------------- epilogues --

struct LseState {
  float run_m, run_l, zy_val;
  int yr, row;
  bool has_zy;
};

// Pass 1: fold one [128 x 256] logit tile into the running (max, sum) of the row.
__device__ __forceinline__ void epi_lse_tile(const GemmArgs& a, uint32_t taddr, int nb, LseState& st) {
  const int col_base = nb * BN;
#pragma unroll 1
  for (int c = 0; c < BN / 32; ++c) {
    uint32_t r[32];
    tmem_ld32(taddr + c * 32, r);
    tmem_ld_wait();
    const int col0 = col_base + c * 32;
    const int lim = a.V - col0;
    const int off = st.yr - col0;
    if (static_cast<unsigned>(off) < 32u) {
#pragma unroll
      for (int t = 0; t < 32; ++t)
        if (t == off) st.zy_val = __uint_as_float(r[t]);
      st.has_zy = true;
    }
    float s[32];
    float cmax = -INFINITY;
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      s[t] = (t < lim) ? __uint_as_float(r[t]) * LOG2E : -INFINITY;
      cmax = fmaxf(cmax, s[t]);
    }
    const float new_m = fmaxf(st.run_m, cmax);
    float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
#pragma unroll
    for (int t = 0; t < 32; t += 4) {
      acc0 += ex2_approx(s[t + 0] - new_m);
      acc1 += ex2_approx(s[t + 1] - new_m);
      acc2 += ex2_approx(s[t + 2] - new_m);
      acc3 += ex2_approx(s[t + 3] - new_m);
    }
    st.run_l = st.run_l * ex2_approx(st.run_m - new_m) + ((acc0 + acc1) + (acc2 + acc3));
    st.run_m = new_m;
  }
}

// Per-warp output staging.  A warp's 32 rows of one 32-column slice go through
// shared memory and leave (or, for the dX sum, also arrive) as one TMA box, so
// global memory sees whole 64-byte row segments instead of the one-row-per-
// thread pattern of the tensor-memory layout.
struct EpiStage {
  uint8_t* ptr;    // this warp's staging area (generic pointer)
  uint32_t addr;   // the same, shared address
  uint32_t bar;    // two mbarriers for boxes loaded into the buffers (dX only)
  uint32_t k;      // slices staged so far by this warp
};

// Byte offset of 16-byte chunk j (0..3) of row r in a 32 x 32 bf16 box stored
// with the 64-byte swizzle (16-byte chunk index XOR bits 1..2 of the row).
__device__ __forceinline__ uint32_t sw64(int r, int j) {
  return static_cast<uint32_t>(r * 64 + ((j ^ ((r >> 1) & 3)) << 4));
}

__device__ __forceinline__ void put_row32(uint8_t* box, int r, const float (&v)[32]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint4 w;
    w.x = pack_bf16x2(v[8 * j + 0], v[8 * j + 1]);
    w.y = pack_bf16x2(v[8 * j + 2], v[8 * j + 3]);
    w.z = pack_bf16x2(v[8 * j + 4], v[8 * j + 5]);
    w.w = pack_bf16x2(v[8 * j + 6], v[8 * j + 7]);
    *reinterpret_cast<uint4*>(box + sw64(r, j)) = w;
  }
}

// Store-only slice: make sure the buffer's previous store has read it, fill it
// with fill(v) for this thread's row, then one lane ships the box.
template <class Fill>
__device__ __forceinline__ void stage_and_store(EpiStage& es, int lane, const CUtensorMap* map, int x, int y,
                                                uint64_t policy, Fill fill) {
  const uint32_t b = es.k & 1u;
  if (lane == 0) bulk_wait_read<1>();
  __syncwarp();
  float v[32];
  fill(v);
  put_row32(es.ptr + b * EPI_BUF_BYTES, lane, v);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(map, es.addr + b * EPI_BUF_BYTES, x, y, policy);
    bulk_commit();
  }
  ++es.k;
}

// Pass 2: G = valid * (softmax - onehot) / n for one tile, stored as bf16.
__device__ __forceinline__ void epi_grad_tile(const GemmArgs& a, int vbase, uint32_t taddr, int row0, int nb,
                                              int row_local, EpiStage& es, const CUtensorMap* mapG) {
  const int row = row0 + row_local;
  const int lane = row_local & 31;
  const bool in_rows = row < a.N;
  const int yr = in_rows ? a.y[row] : a.ignore_index;
  const bool valid = in_rows && yr != a.ignore_index;
  const float l2 = valid ? a.lse2[row] : 0.f;
  const float scale = valid ? row_weight(a.reduction, a.inv_n, a.grad_row_scale, row) : 0.f;
  const int wrow0 = row0 + (row_local & ~31);
#pragma unroll 1
  for (int c = 0; c < BN / 32; ++c) {
    uint32_t r[32];
    tmem_ld32(taddr + c * 32, r);
    tmem_ld_wait();
    const int colg0 = vbase + nb * BN + c * 32;
    const int lim = a.V - colg0;
    stage_and_store(es, lane, mapG, nb * BN + c * 32, wrow0, l2_evict_normal(), [&](float (&g)[32]) {
#pragma unroll
      for (int t = 0; t < 32; ++t)
        g[t] = (valid && t < lim) ? ex2_approx(fmaf(__uint_as_float(r[t]), LOG2E, -l2)) * scale : 0.f;
      const int off = yr - colg0;
      if (valid && static_cast<unsigned>(off) < 32u) {
#pragma unroll
        for (int t = 0; t < 32; ++t)
          if (t == off) g[t] -= scale;
      }
    });
  }
}

// dW rows of this chunk: the K = tokens contraction is complete, round to bf16.
__device__ __forceinline__ void epi_dw_tile(int vbase, uint32_t taddr, int row0, int nb, int row_local,
                                            EpiStage& es, const CUtensorMap* mapDW) {
  const int lane = row_local & 31;
  const int wrow0 = vbase + row0 + (row_local & ~31);
#pragma unroll 1
  for (int c = 0; c < BN / 32; ++c) {
    uint32_t r[32];
    tmem_ld32(taddr + c * 32, r);
    tmem_ld_wait();
    stage_and_store(es, lane, mapDW, nb * BN + c * 32, wrow0, l2_evict_first(), [&](float (&v)[32]) {
#pragma unroll
      for (int t = 0; t < 32; ++t) v[t] = __uint_as_float(r[t]);
    });
  }
}

// Writes a tile of zeros (rows row0.., columns nb*BN..) without reading the
// accumulator: outputs of rows that are all ignored, or a contraction with
// no k-block left.
__device__ __forceinline__ void epi_zero_tile(uint32_t taddr, int row0, int nb, int row_local, EpiStage& es,
                                              const CUtensorMap* map) {
  (void)taddr;
  const int lane = row_local & 31;
  const int wrow0 = row0 + (row_local & ~31);
#pragma unroll 1
  for (int c = 0; c < BN / 32; ++c) {
    stage_and_store(es, lane, map, nb * BN + c * 32, wrow0, l2_evict_first(), [&](float (&v)[32]) {
#pragma unroll
      for (int t = 0; t < 32; ++t) v[t] = 0.f;
    });
  }
}

// dX += G_c W_c.  The running sum lives in two bf16 words, hi (in dX itself) and
// lo (workspace), with value = hi + lo: about 16 significant bits, enough for an
// fp32-grade sum over the chunks, at the memory cost of one bf16 copy of dX.
// Each 32-column slice of the warp's rows is read back (hi and lo boxes by TMA,
// one slice ahead), combined with the accumulator and written back by TMA.
// The last chunk writes the rounded sum through `mapFinal` (dX itself, or the
// workspace when the rows are reordered and a scatter puts them in place).
__device__ __forceinline__ void epi_dx_tile(const GemmArgs& a, bool first_chunk, bool last_chunk, uint32_t taddr,
                                            int row0, int nb, int row_local, EpiStage& es, const CUtensorMap* mapHi,
                                            const CUtensorMap* mapLo, const CUtensorMap* mapFinal,
                                            volatile int* abort_flag, bool& ok) {
  const int lane = row_local & 31;
  const int wrow0 = row0 + (row_local & ~31);
  const bool accumulate = !first_chunk;
  constexpr int SLICES = BN / 32;
  const uint64_t stream = l2_evict_first();  // the running sum is touched once per chunk
  auto fetch = [&](uint32_t b, int c) {  // lane 0: hi and lo boxes of slice c into buffer b
    bulk_wait_read<0>();                 // the buffer's previous store has read it
    fence_proxy_async_smem();
    const uint32_t bar = es.bar + 8u * b;
    mbar_arrive_expect_tx(bar, 2 * EPI_BOX_BYTES);
    tma_load_2d(es.addr + b * EPI_BUF_BYTES, mapHi, bar, nb * BN + c * 32, wrow0, stream);
    tma_load_2d(es.addr + b * EPI_BUF_BYTES + EPI_BOX_BYTES, mapLo, bar, nb * BN + c * 32, wrow0, stream);
  };
  if (accumulate && lane == 0) fetch(es.k & 1u, 0);
#pragma unroll 1
  for (int c = 0; c < SLICES; ++c) {
    const uint32_t b = es.k & 1u;
    if (accumulate) {
      if (c + 1 < SLICES && lane == 0) fetch(b ^ 1u, c + 1);
    } else {
      if (lane == 0) bulk_wait_read<1>();
    }
    __syncwarp();
    uint32_t r[32];
    tmem_ld32(taddr + c * 32, r);
    tmem_ld_wait();
    uint8_t* hbox = es.ptr + b * EPI_BUF_BYTES;
    uint8_t* lbox = hbox + EPI_BOX_BYTES;
    float v[32];
#pragma unroll
    for (int t = 0; t < 32; ++t) v[t] = __uint_as_float(r[t]);
    if (accumulate) {
      const bool got = mbar_wait(es.bar + 8u * b, (es.k >> 1) & 1u, abort_flag, a.timeout_ns);
      if (!__all_sync(0xffffffffu, got)) {
        // let the boxes still in flight land in this warp's buffers before it
        // leaves: this slice's, and the next slice's if it was fetched
        if (lane == 0) {
          volatile int never = 0;
          mbar_wait(es.bar + 8u * b, (es.k >> 1) & 1u, &never, 1000000ull);
          if (c + 1 < SLICES) mbar_wait(es.bar + 8u * (b ^ 1u), ((es.k + 1) >> 1) & 1u, &never, 1000000ull);
        }
        __syncwarp();
        ok = false;
        return;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 h = *reinterpret_cast<const uint4*>(hbox + sw64(lane, j));
        const uint4 l = *reinterpret_cast<const uint4*>(lbox + sw64(lane, j));
        const uint32_t hw[4] = {h.x, h.y, h.z, h.w};
        const uint32_t lw[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[8 * j + 2 * e] += bf16lo_to_f32(hw[e]) + bf16lo_to_f32(lw[e]);
          v[8 * j + 2 * e + 1] += bf16hi_to_f32(hw[e]) + bf16hi_to_f32(lw[e]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x0 = v[8 * j + 2 * e], x1 = v[8 * j + 2 * e + 1];
        hw[e] = pack_bf16x2(x0, x1);
        lw[e] = pack_bf16x2(x0 - bf16lo_to_f32(hw[e]), x1 - bf16hi_to_f32(hw[e]));
      }
      *reinterpret_cast<uint4*>(hbox + sw64(lane, j)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(lbox + sw64(lane, j)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(last_chunk ? mapFinal : mapHi, es.addr + b * EPI_BUF_BYTES, nb * BN + c * 32, wrow0, stream);
      if (!last_chunk)
        tma_store_2d(mapLo, es.addr + b * EPI_BUF_BYTES + EPI_BOX_BYTES, nb * BN + c * 32, wrow0, stream);
      bulk_commit();
    }
    ++es.k;
  }
}

// ------------------------------------------------------------- wind-down --

// Wind-down of both GEMM kernels: this CTA's work is done; tell the peer, wait
// (bounded) for the peer to say the same, then free the pair's tensor memory
// together.  What is known complete before the tensor memory is freed and the
// CTA exits:
//   - every UMMA: the leader's last commit (issued after all its UMMAs, also
//     after a give-up) arrives on the drain barrier of both CTAs once they
//     have all completed;
//   - every TMA store, and every epilogue TMA load: the epilogue warps wait
//     for them (bulk groups; the running-sum boxes' barriers);
//   - the operand loads: after a give-up, the leader waits on the full barrier
//     of every ring position its producer filled and its issuer did not
//     consume; each completes once both CTAs' bytes have landed, and only then
//     does the leader tell the peer it is done.  Only if the two producers
//     stopped at different positions can a load be left that no barrier
//     reports; a fixed 100 us grace period covers that case.
// Every wait here ends by completion or by its own time limit, not by the
// abort flag.  NST is the kernel's ring length (pass 1: P1_STAGES, pass 2:
// STAGES); both kernels lay their barriers out as pass 2 does, so the full
// barrier of ring position q is barrier q % NST and its empty barrier
// STAGES + q % NST.
template <int NST>
__device__ __forceinline__ void pair_wind_down(uint32_t bars, const uint32_t* slots, int rank, int warp,
                                               volatile int* abort_flag, int* status, unsigned long long timeout_ns) {
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile int never = 0;
    if (!mbar_wait(bar(BAR_DRAIN), 0u, &never, END_WAIT_LIMITS * timeout_ns)) raise_status(status, ST_TIMEOUT);
    if (*abort_flag && rank == 0) {
      const long long filled = slots[2], consumed = slots[3];
      bool all = true;
      for (long long q = consumed; q < filled; ++q)
        all = mbar_wait(bar(static_cast<int>(q % NST)), static_cast<uint32_t>((q / NST) & 1), &never,
                        1000000ull) && all;
      if (!all) {
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 100000ull) {
        }
      }
    }
    const uint32_t fin = bar(2 * STAGES + 4);
    mbar_arrive_cluster(mapa_shared(fin, static_cast<uint32_t>(rank ^ 1)));
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_cluster(fin, 0)) {
      if (globaltimer_ns() - t0 > END_WAIT_LIMITS * timeout_ns) {
        raise_status(status, ST_TIMEOUT);
        break;
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(slots[0], TMEM_COLS);
  }
}

// The producer's tail: wait for the UMMA commits still headed for this CTA's
// empty barriers, so none lands after the CTA has gone, and record how far it
// filled the ring.  After a give-up the peer's producer (which cannot see the
// leader's full barriers) lets copies in flight land for 100 us.  NST: the
// ring length, as for pair_wind_down (empty barriers at STAGES + stage).
template <int NST>
__device__ __forceinline__ void producer_tail(uint32_t bars, uint32_t* slots, long long filled, int& stage,
                                              uint32_t& phase, volatile int* abort_flag,
                                              unsigned long long timeout_ns, int rank, int* status) {
  slots[2] = static_cast<uint32_t>(filled);
  for (int i = 0; i < NST; ++i) {
    if (!mbar_wait(bars + 8u * static_cast<uint32_t>(STAGES + stage), phase ^ 1u, abort_flag, timeout_ns)) {
      give_up_pair(abort_flag, rank, status);
      break;
    }
    if (++stage == NST) {
      stage = 0;
      phase ^= 1u;
    }
  }
  if (*abort_flag && rank != 0) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 100000ull) {
    }
  }
}

// ------------------------------------------------------------ the kernel --

// Pass 1: z = X W^T tile by tile; each epilogue thread folds its row's logits
// into a running (max, sum of exponentials) over the vocabulary split of the
// unit, and picks out the target logit.  No logit leaves the chip.
__global__ void __cluster_dims__(CLUSTER, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    flce_pass1_kernel(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapXc,
                      const __grid_constant__ CUtensorMap mapW, const GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  // Same dynamic-smem base in both CTAs, so every offset below matches across the pair.
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;  // swizzle atoms need 1024-B alignment
  uint8_t* base_ptr = smem_raw + (base - raw_addr);
  // the ring of P1_STAGES stages, then the barriers (pass 2's layout; pass 1
  // uses the first P1_STAGES full and empty barriers)
  uint64_t* bars = reinterpret_cast<uint64_t*>(base_ptr + P1_STAGES * P1_STAGE_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NUM_BARRIERS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = static_cast<int>(cluster_ctarank());
  const bool leader = rank == 0;
  const int cid = blockIdx.x / CLUSTER;
  const int ncl = gridDim.x / CLUSTER;
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + STAGES + s); };
  auto tfull_bar = [&](int b) { return smem_u32(bars + 2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return smem_u32(bars + 2 * STAGES + 2 + b); };
  const uint32_t fin_bar = smem_u32(bars + 2 * STAGES + 4);
  // stage s: this CTA's X tile, then the W tiles of the pair's halves 0 and 1
  auto sA = [&](int s) { return base + s * P1_STAGE_BYTES; };
  auto sB = [&](int s, int h) { return base + s * P1_STAGE_BYTES + A_TILE_BYTES + h * B_TILE_BYTES; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < P1_STAGES; ++s) {
      mbar_init(full_bar(s), 1);    // leader: its producer's arrive + both CTAs' bytes
      mbar_init(empty_bar(s), 1);   // the leader's UMMA commit, multicast to both
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);                 // UMMA commit, multicast to both
      mbar_init(tempty_bar(b), CLUSTER * EPI_WARPS);  // leader: epilogue warps of both CTAs
    }
    mbar_init(fin_bar, 1);  // the peer's end-of-work signal
    mbar_init(smem_u32(bars + BAR_DRAIN), 1);  // the leader's last UMMA commit
    *abort_flag = 0;
    tmem_slot[2] = tmem_slot[3] = 0;
    fence_mbar_init();
  }
  // X rows in the token-row order: the caller's X, or its packed copy
  const CUtensorMap* mX = *a.reordered != 0 ? &mapXc : &mapX;
  if (warp == 0 && lane == 0) {
    prefetch_tmap(mX);
    prefetch_tmap(&mapW);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised before any cross-CTA use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  auto give_up = [&]() { give_up_pair(abort_flag, rank, a.status); };

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      const uint64_t keep = l2_evict_last(), stream = l2_evict_first();
      int stage = 0;
      uint32_t phase = 0;
      long long filled = 0;
      bool ok = true;
      // One stage: this CTA's X rows at k-block kb (read again by every
      // vocabulary tile: kept in L2) and its W rows of tile nb + h for each
      // half h in `halves` (bit h; W streams through once), all K-major.
      auto fill = [&](int mb, int nb, int kb, int halves) {
        if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, a.timeout_ns)) {
          give_up();
          return false;
        }
        const int nh = (halves & 1) + (halves >> 1);
        if (leader) mbar_arrive_expect_tx(full_bar(stage), CLUSTER * (A_TILE_BYTES + nh * B_TILE_BYTES));
        const uint32_t bar = mapa_shared(full_bar(stage), 0);
        tma_load_2d_pair(sA(stage), mX, bar, kb * BK, mb * CM + rank * BM, keep);
        for (int h = 0; h < 2; ++h)
          if ((halves >> h) & 1)
            tma_load_2d_pair(sB(stage, h), &mapW, bar, kb * BK, (nb + h) * BN + rank * BNH, stream);
        ++filled;
        if (++stage == P1_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
        return true;
      };
      const int le = min(P1_LEAD, a.k_blocks / 2);
      for (int u = cid; ok && u < a.num_units; u += ncl) {
        int mb, nb0, nb1, split;
        unit_range(a, u, mb, nb0, nb1, split);
        if (a.tile_valid[mb] == 0) continue;  // every row of the tile is ignored
        for (int nb = nb0; ok && nb < nb1;) {
          if (nb + 1 < nb1) {  // tiles nb and nb + 1 as one 256 x 512 tile (see the issuer)
            for (int kb = 0; ok && kb < le; ++kb) ok = fill(mb, nb, kb, 1);
            for (int kb = le; ok && kb < a.k_blocks; ++kb) ok = fill(mb, nb, kb, 3);
            for (int kb = 0; ok && kb < le; ++kb) ok = fill(mb, nb, kb, 2);
            nb += 2;
          } else {
            for (int kb = 0; ok && kb < a.k_blocks; ++kb) ok = fill(mb, nb, kb, 1);
            nb += 1;
          }
        }
      }
      producer_tail<P1_STAGES>(smem_u32(bars), tmem_slot, filled, stage, phase, abort_flag, a.timeout_ns, rank,
                               a.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ UMMA issuer (leader) --
    if (leader && lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(CM, BN, false, false);
      int stage = 0;
      uint32_t phase = 0;
      long long consumed = 0;
      int acc = 0;       // accumulator buffer of the next tile
      uint32_t tph = 0;  // bit b: phase of buffer b's tempty barrier (one flip per use)
      bool ok = true;
      // One stage: the X tile times the W tile of each half h in `halves`
      // into d[h]; f[h] says whether d[h] accumulates.
      auto step = [&](int halves, uint32_t d0, uint32_t& f0, uint32_t d1, uint32_t& f1) {
        if (!mbar_wait(full_bar(stage), phase, abort_flag, a.timeout_ns)) {
          give_up();
          return false;
        }
        ++consumed;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < BK / UMMA_K; ++k) {
          const uint64_t ad = operand_desc<false>(sA(stage), k);
          if (halves & 1) {
            umma_bf16_pair(d0, ad, operand_desc<false>(sB(stage, 0), k), IDESC, f0);
            f0 = 1;
          }
          if (halves & 2) {
            umma_bf16_pair(d1, ad, operand_desc<false>(sB(stage, 1), k), IDESC, f1);
            f1 = 1;
          }
        }
        umma_commit_pair(empty_bar(stage), 0x3);
        if (++stage == P1_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
        return true;
      };
      auto acquire = [&](int b) {  // the epilogue has released buffer b
        if (!mbar_wait<true>(tempty_bar(b), ((tph >> b) & 1u) ^ 1u, abort_flag, a.timeout_ns)) {
          give_up();
          return false;
        }
        tc_fence_after();
        return true;
      };
      const int le = min(P1_LEAD, a.k_blocks / 2);
      for (int u = cid; ok && u < a.num_units; u += ncl) {
        int mb, nb0, nb1, split;
        unit_range(a, u, mb, nb0, nb1, split);
        if (a.tile_valid[mb] == 0) continue;  // every row of the tile is ignored
        for (int nb = nb0; ok && nb < nb1;) {
          const int p = acc, q = acc ^ 1;
          const uint32_t dp = tmem_base + p * ACC_COLS, dq = tmem_base + q * ACC_COLS;
          uint32_t fp = 0, fq = 0;
          ok = acquire(p);
          if (ok && nb + 1 < nb1) {
            // Tiles nb (buffer p) and nb + 1 (buffer q) share each X tile.
            // q may still be in the epilogue of the previous tile: the lead's
            // k-blocks run on p alone meanwhile, and the same k-blocks run on
            // q alone at the end, after p is committed, so that the epilogue
            // folds tile nb while tile nb + 1 finishes.  The next tile takes
            // p again.
            for (int kb = 0; ok && kb < le; ++kb) ok = step(1, dp, fp, dq, fq);
            ok = ok && acquire(q);
            for (int kb = le; ok && kb < a.k_blocks; ++kb) ok = step(3, dp, fp, dq, fq);
            if (ok) {
              umma_commit_pair(tfull_bar(p), 0x3);
              tph ^= 1u << p;
            }
            for (int kb = 0; ok && kb < le; ++kb) ok = step(2, dp, fp, dq, fq);
            if (ok) {
              umma_commit_pair(tfull_bar(q), 0x3);
              tph ^= 1u << q;
            }
            nb += 2;
          } else if (ok) {
            for (int kb = 0; ok && kb < a.k_blocks; ++kb) ok = step(1, dp, fp, dq, fq);
            if (ok) {
              umma_commit_pair(tfull_bar(p), 0x3);
              tph ^= 1u << p;
            }
            acc ^= 1;
            nb += 1;
          }
        }
      }
      // Tail: both accumulators released by the epilogues of both CTAs, so all
      // UMMAs are done and no remote arrive is still on its way here.
      for (int b = 0; b < 2; ++b)
        if (!mbar_wait<true>(tempty_bar(b), ((tph >> b) & 1u) ^ 1u, abort_flag, a.timeout_ns)) {
          give_up();
          break;
        }
      // the positions consumed, and one last commit that completes when every UMMA has
      tmem_slot[3] = static_cast<uint32_t>(consumed);
      umma_commit_pair(smem_u32(bars + BAR_DRAIN), 0x3);
    }
  } else {
    // ---------------------------------------------------------- epilogue --
    const int q = warp & 3;
    const int row_local = q * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t tempty_leader0 = mapa_shared(tempty_bar(0), 0);
    const uint32_t tempty_leader1 = mapa_shared(tempty_bar(1), 0);
    int acc = 0;       // accumulator buffer of the next tile (the issuer's sequence)
    uint32_t eph = 0;  // bit b: phase of buffer b's tfull barrier (one flip per use)
    bool ok = true;
    for (int u = cid; ok && u < a.num_units; u += ncl) {
      int mb, nb0, nb1, split;
      unit_range(a, u, mb, nb0, nb1, split);
      if (a.tile_valid[mb] == 0) continue;  // every row of the tile is ignored
      LseState st;
      st.row = mb * CM + rank * BM + row_local;
      // the target's column in this launch's vocabulary range (-1: none; only the pick reads it)
      const int yrow = st.row < a.N ? a.y[st.row] : a.ignore_index;
      st.yr = yrow != a.ignore_index && yrow >= a.v_off ? yrow - a.v_off : -1;
      st.run_m = -1e30f;
      st.run_l = 0.f;
      st.zy_val = 0.f;
      st.has_zy = false;
      for (int nb = nb0; nb < nb1; ++nb) {
        // a pair of tiles (nb, nb + 1) sits in buffers acc and acc ^ 1, and the
        // tile after it in acc again (the issuer's sequence)
        const bool second = ((nb - nb0) & 1) != 0;
        const int buf = second ? acc ^ 1 : acc;
        const bool got = mbar_wait(tfull_bar(buf), (eph >> buf) & 1u, abort_flag, a.timeout_ns);
        if (!__all_sync(0xffffffffu, got)) {
          give_up();
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem_base + lane_addr + buf * ACC_COLS;
        epi_lse_tile(a, taddr, nb, st);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(buf == 0 ? tempty_leader0 : tempty_leader1);
        eph ^= 1u << buf;
        if (!second && nb + 1 == nb1) acc ^= 1;  // a lone last tile
      }
      if (ok && st.row < a.N) {
        a.part_m[static_cast<size_t>(split + a.split_off) * a.N + st.row] = st.run_m;
        a.part_l[static_cast<size_t>(split + a.split_off) * a.N + st.row] = st.run_l;
        if (st.has_zy) a.zy[st.row] = st.zy_val;
      }
    }
  }

  pair_wind_down<P1_STAGES>(smem_u32(bars), tmem_slot, rank, warp, abort_flag, a.status, a.timeout_ns);
}

// ===================================================== pass 2, one launch ==
//
// All of pass 2 runs as one persistent launch over a static queue of work
// items, dealt round-robin to the SM pairs:
//
//   G(0)  |  dX(0) dW(0) G(1)  |  dX(1) dW(1) G(2)  | ... |  dX(C-1) dW(C-1)
//
// where G(c) are the logit-recompute tiles of chunk c, dX(c) the
// dX += G_c W_c tiles and dW(c) the dW rows of chunk c.  The G tiles of a
// chunk go column by column (all token tiles of one vocabulary tile, then the
// next) when a chunk holds more than three rounds of them for the SM pairs:
// the dW(c) items that their epilogues wait for finish column by column.  With
// fewer rounds they go row by row, so that each token tile's G row is complete
// early and the dX(c) items that wait for it are not all held up by the last
// column.  There is one G buffer,
// so items wait for what they read and for the readers of what they overwrite:
//   dX(c) mainloop  after G(c) of its token tile (all its columns),
//   dX(c) epilogue  after dX(c-1) of its token tile (running sum),
//   dW(c) mainloop  after G(c) of its column (all token tiles),
//   G(c)  epilogue  after dX(c-1) of its token tile and dW(c-1) of its column.
// Every dependency points to an earlier item and all SM pairs are resident at
// once, so the queue always drains.  Completion is counted per token tile /
// column in monotonic counters: each epilogue warp adds one per 256x256 tile
// after its TMA stores have landed, so a finished tile adds EPI_WARPS * CLUSTER.
//
// A dW item covers two adjacent 256-column hidden tiles (the last one alone
// when the hidden tiles are odd in number): a 256 x 512 tile in both halves of
// the tensor memory, which reads its G^T operand once for both halves.  Its
// K = tokens contraction is long and its epilogue short, so the loss of the
// accumulator double buffer is confined to its two ends (see the issuer).

enum : int { ITEM_GRAD = 0, ITEM_DW = 1, ITEM_DX = 2 };

struct Item {
  int kind, c, a, b;  // G: (tm, vb)  dW: (vm, hidden tile pair)  dX: (tm, hn)
};

// A dW item with two hidden tiles (2b and 2b+1)?
__device__ __forceinline__ bool dw_paired(const GemmArgs& p, const Item& it) {
  return p.HW < p.HN && 2 * it.b + 1 < p.HN;
}

__device__ __forceinline__ int chunk_vtiles(const GemmArgs& p, int c) { return c == p.C - 1 ? p.VT_last : p.VTf; }

__device__ __forceinline__ long long section_size(const GemmArgs& p, int c) {
  long long n = static_cast<long long>(p.TM) * p.HN + static_cast<long long>(chunk_vtiles(p, c)) * p.HW;
  if (c + 1 < p.C) n += static_cast<long long>(chunk_vtiles(p, c + 1)) * p.TM;
  return n;
}

// Tile of the r-th G item of chunk c: the first g_cols_first vocabulary tiles
// column by column (every token tile of one column, then the next column),
// the remaining ones row by row.
__device__ __forceinline__ void grad_tile(const GemmArgs& p, int c, long long r, Item& it) {
  const int vt = chunk_vtiles(p, c);
  const int k = min(p.g_cols_first, vt);
  const long long head = static_cast<long long>(k) * p.TM;
  if (r < head) {
    it.b = static_cast<int>(r / p.TM);
    it.a = static_cast<int>(r - static_cast<long long>(it.b) * p.TM);
  } else {
    const long long r2 = r - head;
    const int w = vt - k;
    it.a = static_cast<int>(r2 / w);
    it.b = k + static_cast<int>(r2 - static_cast<long long>(it.a) * w);
  }
}

__device__ __forceinline__ Item decode_item(const GemmArgs& p, long long i) {
  Item it;
  const long long g0 = static_cast<long long>(chunk_vtiles(p, 0)) * p.TM;
  if (i < g0) {
    it.kind = ITEM_GRAD;
    it.c = 0;
    grad_tile(p, 0, i, it);
    return it;
  }
  // sections 0 .. C-3 all have the size of section 0; the last two may be shorter
  long long r = i - g0;
  int c = 0;
  if (p.C >= 3) {
    const long long full = section_size(p, 0);
    c = static_cast<int>(min(r / full, static_cast<long long>(p.C - 3)));
    r -= static_cast<long long>(c) * full;
  }
  while (c + 1 < p.C && r >= section_size(p, c)) {
    r -= section_size(p, c);
    ++c;
  }
  const long long nx = static_cast<long long>(p.TM) * p.HN;
  const long long nw = static_cast<long long>(chunk_vtiles(p, c)) * p.HW;
  it.c = c;
  if (r < nx) {
    it.kind = ITEM_DX;
    it.a = static_cast<int>(r / p.HN);
    it.b = static_cast<int>(r - static_cast<long long>(it.a) * p.HN);
  } else if (r < nx + nw) {
    r -= nx;
    it.kind = ITEM_DW;
    it.a = static_cast<int>(r / p.HW);
    it.b = static_cast<int>(r - static_cast<long long>(it.a) * p.HW);
  } else {
    r -= nx + nw;
    it.kind = ITEM_GRAD;
    it.c = c + 1;
    grad_tile(p, c + 1, r, it);
  }
  return it;
}

// First 256-column hidden tile of a dW item.
__device__ __forceinline__ int dw_first_tile(const GemmArgs& p, const Item& it) {
  return p.HW < p.HN ? 2 * it.b : it.b;
}

// A paired dW item runs its first `lead` active k-blocks on the first half
// alone and the same k-blocks on the second half last (see the issuer).  The
// k-blocks over token tiles whose rows are all ignored are not active.  Returns
// the raw k-block index just past the lead, with lead = min(dw_lead, active/2).
__device__ __forceinline__ int dw_lead_end(const GemmArgs& a) {
  const int kblocks = (a.N + BK - 1) / BK;
  int active = 0;
  for (int kb = 0; kb < kblocks; ++kb) active += a.tile_valid[kb / (CM / BK)] != 0 ? 1 : 0;
  const int lead = min(a.dw_lead, active / 2);
  int cnt = 0;
  for (int kb = 0; kb < kblocks && cnt < lead; ++kb)
    if (a.tile_valid[kb / (CM / BK)] != 0 && ++cnt == lead) return kb + 1;
  return 0;
}

constexpr int SIGNALS_PER_ITEM = EPI_WARPS * CLUSTER;

// Pass-2 tensor maps, in one struct so they travel as one kernel parameter.
struct Pass2Maps {
  CUtensorMap Xk, Wk;      // G: X rows and W rows, K-major
  CUtensorMap Gmn, Xmn;    // dW: G_c^T and X, MN-major
  CUtensorMap Gk, Wmn;     // dX: G_c rows K-major, W_c MN-major
  CUtensorMap Go, DWo;     // epilogue output boxes of G and dW
  CUtensorMap Hio, Loo;    // epilogue boxes of the dX running sum (hi = dX, lo)
  CUtensorMap Xck, Xcmn;   // the packed copy of X (reordered rows), K- and MN-major
};

__global__ void __cluster_dims__(CLUSTER, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    flce_pass2_kernel(const __grid_constant__ Pass2Maps m, const GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw_addr);
  uint8_t* epi_ptr = base_ptr + STAGES * STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(epi_ptr + EPI_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NUM_BARRIERS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = static_cast<int>(cluster_ctarank());
  const bool leader = rank == 0;
  const long long cid = blockIdx.x / CLUSTER;
  const long long ncl = gridDim.x / CLUSTER;
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + STAGES + s); };
  auto tfull_bar = [&](int b) { return smem_u32(bars + 2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return smem_u32(bars + 2 * STAGES + 2 + b); };
  const uint32_t fin_bar = smem_u32(bars + 2 * STAGES + 4);
  auto sA = [&](int s) { return base + s * STAGE_BYTES; };
  auto sB = [&](int s) { return base + s * STAGE_BYTES + A_TILE_BYTES; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), CLUSTER * EPI_WARPS);
    }
    mbar_init(fin_bar, 1);
    for (int e = 0; e < 2 * EPI_WARPS; ++e) mbar_init(smem_u32(bars + 2 * STAGES + 5 + e), 1);
    mbar_init(smem_u32(bars + BAR_DRAIN), 1);
    *abort_flag = 0;
    tmem_slot[2] = tmem_slot[3] = 0;
    fence_mbar_init();
  }
  // X rows in the token-row order: the caller's X, or its packed copy
  const bool reordered = *a.reordered != 0;
  const CUtensorMap* mXk = reordered ? &m.Xck : &m.Xk;
  const CUtensorMap* mXmn = reordered ? &m.Xcmn : &m.Xmn;
  if (warp == 0 && lane == 0) {
    prefetch_tmap(mXk);
    prefetch_tmap(&m.Wk);
    prefetch_tmap(&m.Gmn);
    prefetch_tmap(mXmn);
    prefetch_tmap(&m.Gk);
    prefetch_tmap(&m.Wmn);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  auto give_up = [&]() { give_up_pair(abort_flag, rank, a.status); };
  // cumulative G tiles of token tile tm after chunk c
  auto g_row_target = [&](int c) {
    return SIGNALS_PER_ITEM * (c < a.C - 1 ? (c + 1) * a.VTf : (a.C - 1) * a.VTf + a.VT_last);
  };

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      const uint64_t keep = l2_evict_last(), normal = l2_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      long long filled = 0;
      bool ok = true;
      const int dw_lead = dw_lead_end(a);
      for (long long u = a.item_begin + cid; ok && u < a.item_end; u += ncl) {
        const Item it = decode_item(a, u);
        const int vbase = it.c * a.Vc;
        const int vcount = min(a.Vc, a.V - vbase);
        // G and dX tiles of a token tile whose rows are all ignored are skipped
        const bool skip = it.kind != ITEM_DW && a.tile_valid[it.a] == 0;
        int kblocks;
        if (skip) {
          kblocks = 0;
        } else if (it.kind == ITEM_GRAD) {
          kblocks = (a.H + BK - 1) / BK;
        } else if (it.kind == ITEM_DW) {
          kblocks = (a.N + BK - 1) / BK;
          ok = wait_counter(a.g_col + it.a, SIGNALS_PER_ITEM * a.TM * (it.c + 1) + a.starve_dw, abort_flag,
                            a.timeout_ns);
        } else {
          kblocks = (vcount + BK - 1) / BK;
          ok = wait_counter(a.g_row + it.a, g_row_target(it.c), abort_flag, a.timeout_ns);
        }
        if (!ok) {
          give_up();
          break;
        }
        // G written by other CTAs' TMA stores is read below by TMA: order the
        // acquire above before those reads (G tiles read only X and W)
        if (it.kind != ITEM_GRAD) fence_proxy_async_global();
        const int m0 = it.a * CM + rank * BM;
        const int n0 = (it.kind == ITEM_DW ? dw_first_tile(a, it) : it.b) * BN + rank * BNH;
        if (it.kind == ITEM_DW && dw_paired(a, it)) {
          // one ring position: G^T (unless with_a is false) and the X columns from n
          auto fill_dw = [&](int kb, bool with_a, int n) {
            if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, a.timeout_ns)) {
              give_up();
              return false;
            }
            if (leader) mbar_arrive_expect_tx(full_bar(stage), CLUSTER * (with_a ? STAGE_BYTES : B_TILE_BYTES));
            const uint32_t bar = mapa_shared(full_bar(stage), 0);
            const int k0 = kb * BK;
            if (with_a) {
#pragma unroll
              for (int i = 0; i < BM / 64; ++i)
                tma_load_2d_pair(sA(stage) + i * MN_BOX_BYTES, &m.Gmn, bar, m0 + i * 64, k0, normal);
            }
#pragma unroll
            for (int i = 0; i < BNH / 64; ++i)
              tma_load_2d_pair(sB(stage) + i * MN_BOX_BYTES, mXmn, bar, n + i * 64, k0, keep);
            ++filled;
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
            return true;
          };
          // lead: first half alone; middle: both halves (two positions, G^T
          // once); tail: second half alone over the lead's k-blocks
          for (int kb = 0; ok && kb < dw_lead; ++kb)
            if (a.tile_valid[kb / (CM / BK)] != 0) ok = fill_dw(kb, true, n0);
          for (int kb = dw_lead; ok && kb < kblocks; ++kb)
            if (a.tile_valid[kb / (CM / BK)] != 0) ok = fill_dw(kb, true, n0) && fill_dw(kb, false, n0 + BN);
          for (int kb = 0; ok && kb < dw_lead; ++kb)
            if (a.tile_valid[kb / (CM / BK)] != 0) ok = fill_dw(kb, true, n0 + BN);
          continue;
        }
        for (int kb = 0; kb < kblocks; ++kb) {
          // dW: K runs over tokens; k-blocks of all-ignored token tiles add nothing
          if (it.kind == ITEM_DW && a.tile_valid[kb / (CM / BK)] == 0) continue;
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, a.timeout_ns)) {
            give_up();
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(full_bar(stage), CLUSTER * STAGE_BYTES);
          const uint32_t bar = mapa_shared(full_bar(stage), 0);
          const int k0 = kb * BK;
          if (it.kind == ITEM_GRAD) {
            tma_load_2d_pair(sA(stage), mXk, bar, k0, m0, keep);
            tma_load_2d_pair(sB(stage), &m.Wk, bar, k0, vbase + n0, normal);
          } else if (it.kind == ITEM_DW) {
#pragma unroll
            for (int i = 0; i < BM / 64; ++i)
              tma_load_2d_pair(sA(stage) + i * MN_BOX_BYTES, &m.Gmn, bar, m0 + i * 64, k0, normal);
#pragma unroll
            for (int i = 0; i < BNH / 64; ++i)
              tma_load_2d_pair(sB(stage) + i * MN_BOX_BYTES, mXmn, bar, n0 + i * 64, k0, keep);
          } else {
            tma_load_2d_pair(sA(stage), &m.Gk, bar, k0, m0, normal);
#pragma unroll
            for (int i = 0; i < BNH / 64; ++i)
              tma_load_2d_pair(sB(stage) + i * MN_BOX_BYTES, &m.Wmn, bar, n0 + i * 64, vbase + k0, normal);
          }
          ++filled;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      producer_tail<STAGES>(smem_u32(bars), tmem_slot, filled, stage, phase, abort_flag, a.timeout_ns, rank,
                            a.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ UMMA issuer (leader) --
    if (leader && lane == 0) {
      constexpr uint32_t ID_GRAD = idesc_bf16_f32(CM, BN, false, false);
      constexpr uint32_t ID_DW = idesc_bf16_f32(CM, BN, true, true);
      constexpr uint32_t ID_DX = idesc_bf16_f32(CM, BN, false, true);
      int stage = 0;
      uint32_t phase = 0;
      long long consumed = 0;
      int acc = 0;          // accumulator buffer of the next item
      uint32_t tph = 0;     // bit b: phase of buffer b's tempty barrier (one flip per use)
      bool ok = true;
      const int dw_lead = dw_lead_end(a);
      auto take = [&]() {  // wait for the next ring position to fill
        if (!mbar_wait(full_bar(stage), phase, abort_flag, a.timeout_ns)) {
          give_up();
          return -1;
        }
        ++consumed;
        tc_fence_after();
        const int s = stage;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
        return s;
      };
      auto mma_dw = [&](uint32_t d, int sa, int sb, uint32_t& accumulate) {
#pragma unroll
        for (int k = 0; k < BK / UMMA_K; ++k) {
          umma_bf16_pair(d, operand_desc<true>(sA(sa), k), operand_desc<true>(sB(sb), k), ID_DW, accumulate);
          accumulate = 1;
        }
      };
      for (long long u = a.item_begin + cid; ok && u < a.item_end; u += ncl) {
        const Item it = decode_item(a, u);
        if (it.kind == ITEM_DW && dw_paired(a, it)) {
          // 256 x 512: the first half in buffer p (the next in turn), the
          // second in q, which the previous item's epilogue may still be
          // reading.  The lead's k-blocks run on p alone meanwhile, and the
          // same k-blocks run on q alone at the end, after p is committed, so
          // that the epilogue drains p while q finishes; the next item then
          // takes p again.
          const int p = acc, q = acc ^ 1;
          const int kblocks = (a.N + BK - 1) / BK;
          uint32_t acc_p = 0, acc_q = 0;
          if (!mbar_wait<true>(tempty_bar(p), ((tph >> p) & 1u) ^ 1u, abort_flag, a.timeout_ns)) {
            give_up();
            break;
          }
          tc_fence_after();
          const uint32_t dp = tmem_base + p * ACC_COLS, dq = tmem_base + q * ACC_COLS;
          for (int kb = 0; ok && kb < dw_lead; ++kb) {
            if (a.tile_valid[kb / (CM / BK)] == 0) continue;
            const int s1 = take();
            if (s1 < 0) {
              ok = false;
              break;
            }
            mma_dw(dp, s1, s1, acc_p);
            umma_commit_pair(empty_bar(s1), 0x3);
          }
          if (!ok) break;
          if (!mbar_wait<true>(tempty_bar(q), ((tph >> q) & 1u) ^ 1u, abort_flag, a.timeout_ns)) {
            give_up();
            break;
          }
          tc_fence_after();
          for (int kb = dw_lead; ok && kb < kblocks; ++kb) {
            if (a.tile_valid[kb / (CM / BK)] == 0) continue;
            const int s1 = take();
            const int s2 = s1 < 0 ? -1 : take();
            if (s2 < 0) {
              ok = false;
              break;
            }
            mma_dw(dp, s1, s1, acc_p);
            mma_dw(dq, s1, s2, acc_q);
            umma_commit_pair(empty_bar(s1), 0x3);
            umma_commit_pair(empty_bar(s2), 0x3);
          }
          if (!ok) break;
          umma_commit_pair(tfull_bar(p), 0x3);
          tph ^= 1u << p;
          for (int kb = 0; ok && kb < dw_lead; ++kb) {
            if (a.tile_valid[kb / (CM / BK)] == 0) continue;
            const int s1 = take();
            if (s1 < 0) {
              ok = false;
              break;
            }
            mma_dw(dq, s1, s1, acc_q);
            umma_commit_pair(empty_bar(s1), 0x3);
          }
          if (!ok) break;
          umma_commit_pair(tfull_bar(q), 0x3);
          tph ^= 1u << q;
          continue;
        }
        const int vcount = min(a.Vc, a.V - it.c * a.Vc);
        const bool skip = it.kind != ITEM_DW && a.tile_valid[it.a] == 0;
        const int kblocks = skip                  ? 0
                            : it.kind == ITEM_GRAD ? (a.H + BK - 1) / BK
                            : it.kind == ITEM_DW   ? (a.N + BK - 1) / BK
                                                   : (vcount + BK - 1) / BK;
        const uint32_t idesc = it.kind == ITEM_GRAD ? ID_GRAD : it.kind == ITEM_DW ? ID_DW : ID_DX;
        const bool a_mn = it.kind == ITEM_DW;
        const bool b_mn = it.kind != ITEM_GRAD;
        if (!mbar_wait<true>(tempty_bar(acc), ((tph >> acc) & 1u) ^ 1u, abort_flag, a.timeout_ns)) {
          give_up();
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
        uint32_t accumulate = 0;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (it.kind == ITEM_DW && a.tile_valid[kb / (CM / BK)] == 0) continue;
          if (!mbar_wait(full_bar(stage), phase, abort_flag, a.timeout_ns)) {
            give_up();
            ok = false;
            break;
          }
          ++consumed;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k) {
            const uint64_t ad = a_mn ? operand_desc<true>(sA(stage), k) : operand_desc<false>(sA(stage), k);
            const uint64_t bd = b_mn ? operand_desc<true>(sB(stage), k) : operand_desc<false>(sB(stage), k);
            umma_bf16_pair(d_tmem, ad, bd, idesc, accumulate);
            accumulate = 1;
          }
          umma_commit_pair(empty_bar(stage), 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair(tfull_bar(acc), 0x3);
        tph ^= 1u << acc;
        acc ^= 1;
      }
      for (int b = 0; b < 2; ++b) {
        if (!mbar_wait<true>(tempty_bar(b), ((tph >> b) & 1u) ^ 1u, abort_flag, a.timeout_ns)) {
          give_up();
          break;
        }
      }
      // the positions consumed, and one last commit that completes when every UMMA has
      tmem_slot[3] = static_cast<uint32_t>(consumed);
      umma_commit_pair(smem_u32(bars + BAR_DRAIN), 0x3);
    }
  } else {
    // ---------------------------------------------------------- epilogue --
    const int q = warp & 3;
    const int row_local = q * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t tempty_leader0 = mapa_shared(tempty_bar(0), 0);
    const uint32_t tempty_leader1 = mapa_shared(tempty_bar(1), 0);
    EpiStage es;
    es.ptr = epi_ptr + q * EPI_WARP_BYTES;
    es.addr = smem_u32(es.ptr);
    es.bar = smem_u32(bars + 2 * STAGES + 5 + 2 * q);
    es.k = 0;
    // the rounded dX goes to the workspace when the rows are reordered
    const CUtensorMap* dx_final = reordered ? &m.Loo : &m.Hio;
    // with every token ignored the dW contraction has no k-block at all
    bool any_valid = false;
    for (int t = 0; t < a.TM && !any_valid; ++t) any_valid = a.tile_valid[t] != 0;
    int acc = 0;       // accumulator buffer of the next item (the issuer's sequence)
    uint32_t eph = 0;  // bit b: phase of buffer b's tfull barrier (one flip per use)
    bool ok = true;
    for (long long u = a.item_begin + cid; ok && u < a.item_end; u += ncl) {
      const Item it = decode_item(a, u);
      const int vbase = it.c * a.Vc;
      const int row0 = it.a * CM + rank * BM;
      // wait for the previous readers (G) / writers (dX) of what this tile writes
      if (lane == 0) {
        if (it.kind == ITEM_GRAD && it.c > 0) {
          ok = wait_counter(a.x_row + it.a, SIGNALS_PER_ITEM * it.c * a.HN, abort_flag, a.timeout_ns) &&
               wait_counter(a.w_col + it.b, SIGNALS_PER_ITEM * it.c * a.HN, abort_flag, a.timeout_ns);
        } else if (it.kind == ITEM_DX && it.c > 0) {
          ok = wait_counter(a.x_row + it.a, SIGNALS_PER_ITEM * it.c * a.HN, abort_flag, a.timeout_ns);
        }
        if (ok) fence_proxy_async_global();
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) {
        give_up();
        break;
      }
      if (it.kind == ITEM_DW && dw_paired(a, it)) {
        // a paired dW item: its first half in buffer acc, its second in acc ^ 1;
        // the next item takes acc again, the buffer freed first
        for (int h = 0; h < 2; ++h) {
          const int buf = acc ^ h;
          const bool got = mbar_wait(tfull_bar(buf), (eph >> buf) & 1u, abort_flag, a.timeout_ns);
          if (!__all_sync(0xffffffffu, got)) {
            give_up();
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t taddr = tmem_base + lane_addr + buf * ACC_COLS;
          const int nt = dw_first_tile(a, it) + h;
          if (any_valid)
            epi_dw_tile(vbase, taddr, row0, nt, row_local, es, &m.DWo);
          else
            epi_zero_tile(taddr, vbase + row0, nt, row_local, es, &m.DWo);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(buf == 0 ? tempty_leader0 : tempty_leader1);
          eph ^= 1u << buf;
        }
        if (!ok) break;
        if (lane == 0) {
          bulk_wait<0>();
          fence_proxy_async_global();
          red_release_gpu_add(a.w_col + it.a, 2);
        }
        continue;
      }
      const bool got = mbar_wait(tfull_bar(acc), (eph >> acc) & 1u, abort_flag, a.timeout_ns);
      if (!__all_sync(0xffffffffu, got)) {
        give_up();
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + lane_addr + acc * ACC_COLS;
      const bool skip = it.kind != ITEM_DW && a.tile_valid[it.a] == 0;
      if (skip) {
        // all rows ignored: nothing reads this tile's G rows; its dX rows are
        // zero, written once by the first chunk
        if (it.kind == ITEM_DX && it.c == 0) epi_zero_tile(taddr, row0, it.b, row_local, es, &m.Hio);
      } else if (it.kind == ITEM_GRAD) {
        epi_grad_tile(a, vbase, taddr, row0, it.b, row_local, es, &m.Go);
      } else if (it.kind == ITEM_DW) {
        const int nt = dw_first_tile(a, it);
        if (any_valid)
          epi_dw_tile(vbase, taddr, row0, nt, row_local, es, &m.DWo);
        else
          epi_zero_tile(taddr, vbase + row0, nt, row_local, es, &m.DWo);
      } else {
        epi_dx_tile(a, it.c == 0, it.c == a.C - 1, taddr, row0, it.b, row_local, es, &m.Hio, &m.Loo, dx_final,
                    abort_flag, ok);
        if (!ok) {
          give_up();
          break;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc == 0 ? tempty_leader0 : tempty_leader1);
      eph ^= 1u << acc;
      acc ^= 1;
      // this warp's boxes have landed: count the tile as done for its readers
      if (lane == 0) {
        bulk_wait<0>();
        fence_proxy_async_global();
        if (it.kind == ITEM_GRAD) {
          red_release_gpu_add(a.g_row + it.a, 1);
          red_release_gpu_add(a.g_col + it.b, 1);
        } else if (it.kind == ITEM_DW) {
          red_release_gpu_add(a.w_col + it.a, 1);
        } else {
          red_release_gpu_add(a.x_row + it.a, 1);
        }
      }
    }
    if (lane == 0) bulk_wait<0>();
  }

  pair_wind_down<STAGES>(smem_u32(bars), tmem_slot, rank, warp, abort_flag, a.status, a.timeout_ns);
}

// ---------------------------------------------------------------- prep --

// Valid (non-ignored) rows of each 256-row token tile, so that pass 1 and
// pass 2 can skip tiles whose rows are all ignored (a prompt mask).
// `tile_valid` may be null; a non-null `total` (zeroed beforehand) receives
// the count of every tile (an integer sum, the same in any order).
__global__ void __launch_bounds__(CM)
    flce_prep_kernel(const int32_t* y, int N, int ignore_index, int* tile_valid, int* total = nullptr) {
  const int r = blockIdx.x * CM + threadIdx.x;
  const int v = (r < N && y[r] != ignore_index) ? 1 : 0;
  const int cnt = __syncthreads_count(v);
  if (threadIdx.x == 0) {
    if (tile_valid) tile_valid[blockIdx.x] = cnt;
    if (total && cnt) atomicAdd(total, cnt);
  }
}

// Token-row order for the two passes (one CTA per 256-row tile of y).
// Ignored rows cost as much as valid ones unless a whole 256-row tile is
// ignored.  When the valid rows, packed first, fill fewer tiles than the
// tiles that hold any valid row, the rows are reordered: a stable partition
// with every valid row first, in their original order, then the ignored rows.
// Writes the row map `perm`, y and the upstream weights in that order, the
// per-tile valid counts of the new order, and the decision (`reordered_out`).
// `allow` = 0 keeps the caller's order (no room for the packed copy of X).
// Every CTA computes the same totals from `tile_cnt`, so they all decide alike.
// Targets are checked against the whole vocabulary [0, V_total) and stored
// relative to this call's W rows [v0, v0 + V): a target outside them (held by
// another vocabulary shard) becomes TARGET_ELSEWHERE, which no column matches.
__global__ void __launch_bounds__(CM)
    flce_row_order_kernel(const int32_t* y, const float* g, int N, int TM, int ignore_index, const int* tile_cnt,
                          int allow, int v0, int V, int V_total, int* tile_valid, int* perm, int32_t* y_perm,
                          float* g_perm, int* reordered_out, int* n_rows_out, int* status) {
  const int t = blockIdx.x;
  int total = 0, nonempty = 0, before = 0;
  for (int i = threadIdx.x; i < TM; i += CM) {
    const int c = tile_cnt[i];
    total += c;
    nonempty += c > 0 ? 1 : 0;
    before += i < t ? c : 0;
  }
  __shared__ int red[3][CM / 32];
  __shared__ int wrank[CM / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    total += __shfl_down_sync(0xffffffffu, total, o);
    nonempty += __shfl_down_sync(0xffffffffu, nonempty, o);
    before += __shfl_down_sync(0xffffffffu, before, o);
  }
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  if (lane == 0) {
    red[0][w] = total;
    red[1][w] = nonempty;
    red[2][w] = before;
  }
  const int r = t * CM + threadIdx.x;
  const bool in = r < N;
  const int yr = in ? y[r] : ignore_index;
  const bool v = in && yr != ignore_index;
  const unsigned bal = __ballot_sync(0xffffffffu, v);
  if (lane == 0) wrank[w] = __popc(bal);
  __syncthreads();
  total = nonempty = before = 0;
  int rank_v = __popc(bal & ((1u << lane) - 1u));
  for (int i = 0; i < CM / 32; ++i) {
    total += red[0][i];
    nonempty += red[1][i];
    before += red[2][i];
    rank_v += i < w ? wrank[i] : 0;
  }
  const bool reorder = allow != 0 && (total + CM - 1) / CM < nonempty;
  if (v && (yr < 0 || yr >= V_total)) raise_status(status, ST_TARGET_OUT_OF_RANGE);
  const int yl = !v ? ignore_index : (yr >= v0 && yr - v0 < V) ? yr - v0 : target_elsewhere(ignore_index);
  if (in) {
    int dest = r;
    if (reorder) {
      // ignored rows ahead of this one: those of the (full) earlier tiles plus
      // those earlier in this tile
      dest = v ? before + rank_v : total + (t * CM - before) + (static_cast<int>(threadIdx.x) - rank_v);
    }
    perm[dest] = r;
    y_perm[dest] = yl;
    if (g) g_perm[dest] = g[r];
  } else {
    perm[r] = 0;  // padding of the last tile: any in-range row (its outputs are never kept)
  }
  if (threadIdx.x == 0) tile_valid[t] = reorder ? max(0, min(CM, total - t * CM)) : tile_cnt[t];
  if (t == 0 && threadIdx.x == 0) {
    *reordered_out = reorder ? 1 : 0;
    *n_rows_out = total;
  }
}

// With reordered rows the GEMMs read X through a packed copy in the new order,
// Xc[r] = X[perm[r]], for every row of the 256-row tiles that hold a valid row
// (the ignored rows sharing the last such tile included, so that every row the
// tensor cores read is finite).  One warp per row, 16-byte accesses.
__global__ void __launch_bounds__(256)
    flce_pack_rows_kernel(const uint16_t* X, uint16_t* Xc, const int* perm, const int* reordered,
                          const int* n_rows, int N, int H) {
  if (*reordered == 0) return;
  const int rows = min(N, (*n_rows + CM - 1) / CM * CM);
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  const int h8 = H / 8;
  for (int r = blockIdx.x * wpb + (threadIdx.x >> 5); r < rows; r += gridDim.x * wpb) {
    const uint4* sr = reinterpret_cast<const uint4*>(X + static_cast<size_t>(perm[r]) * H);
    uint4* d = reinterpret_cast<uint4*>(Xc + static_cast<size_t>(r) * H);
    for (int j = lane; j < h8; j += 32) d[j] = sr[j];
  }
}

// With reordered rows the rounded dX sits in the workspace in the new order:
// put each row back in place and write zeros for the rows of ignored targets
// (one warp per row, 16-byte accesses; H is a multiple of 8).
__global__ void __launch_bounds__(256)
    flce_dx_scatter_kernel(const uint16_t* src, uint16_t* dX, const int* perm, const int* reordered,
                           const int* n_rows, int N, int H) {
  if (*reordered == 0) return;
  const int nr = *n_rows;
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  const int h8 = H / 8;
  for (int r = blockIdx.x * wpb + (threadIdx.x >> 5); r < N; r += gridDim.x * wpb) {
    uint4* d = reinterpret_cast<uint4*>(dX + static_cast<size_t>(perm[r]) * H);
    if (r < nr) {
      const uint4* sr = reinterpret_cast<const uint4*>(src + static_cast<size_t>(r) * H);
      for (int j = lane; j < h8; j += 32) d[j] = sr[j];
    } else {
      for (int j = lane; j < h8; j += 32) d[j] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

// ------------------------------------------------------------ combine --

// What the combine kernel does with the rows' statistics.
enum : int {
  COMBINE_FULL = 0,      // merge the pass-1 splits: lse, loss, 1/n
  COMBINE_SHARD = 1,     // merge the splits into this vocabulary shard's (lse, target logit) per row, no loss
  COMBINE_SHARDS_IN = 2  // lse and target logit from every shard's statistics, then loss and 1/n
};

struct CombineArgs {
  int N, V, ignore_index, splits;
  int mode;                // COMBINE_*
  int shards;              // COMBINE_SHARDS_IN: number of shards in all_lse / all_zy
  const float* all_lse;    // [shards][N] per-shard log-sum-exp (natural log)
  const float* all_zy;     // [shards][N] per-shard target logit (0 outside the shard)
  float* shard_lse;        // COMBINE_SHARD outputs, [N] each
  float* shard_zy;
  int reduction;
  const float* grad_row_scale;
  float* row_loss;  // optional per-row losses, in the caller's row order
  const int* perm;  // row of the caller behind each row of y, part_m, ... (token-row order)
  const int* mean_count;  // optional: divide the mean by this count instead of n_valid
  const int32_t* y;
  const float* part_m;
  const float* part_l;
  const float* zy;
  float* lse2;
  double* blk_loss;
  int* blk_cnt;
  unsigned int* ticket;
  int* n_valid;
  float* inv_n;
  float* loss;
  int* status;
};

constexpr int COMBINE_THREADS = 256;

// Merges the per-split (max, sum) pairs of each row into its log-sum-exp, forms
// the row loss lse_i - z_{i,y_i} for valid rows and reduces the token mean.
// Deterministic: a fixed tree inside each block, then the last block to finish
// adds the block sums in block order, in fp64.  (The target range was checked
// by the row-order kernel.)
// A vocabulary shard's call (COMBINE_SHARD) stops after writing its rows'
// (lse, target logit); the call after the exchange (COMBINE_SHARDS_IN) takes
// lse_i as the log-sum-exp of every shard's lse and z_{i,y_i} as the sum of
// their target logits, then goes on as the full head does.
__global__ void __launch_bounds__(COMBINE_THREADS) flce_combine_kernel(const CombineArgs a) {
  const int i = blockIdx.x * COMBINE_THREADS + threadIdx.x;
  double li = 0.0;
  int vi = 0;
  if (i < a.N) {
    const int yi = a.y[i];
    const bool valid = yi != a.ignore_index;
    float l2, zyi;
    if (a.mode == COMBINE_SHARDS_IN) {
      float M = -INFINITY;
      for (int s = 0; s < a.shards; ++s) M = fmaxf(M, a.all_lse[static_cast<size_t>(s) * a.N + i]);
      float S = 0.f;
      zyi = 0.f;
      for (int s = 0; s < a.shards; ++s) {
        S += expf(a.all_lse[static_cast<size_t>(s) * a.N + i] - M);
        zyi += a.all_zy[static_cast<size_t>(s) * a.N + i];
      }
      l2 = (M + logf(S)) * LOG2E;
    } else {
      float M = -INFINITY;
      for (int s = 0; s < a.splits; ++s) M = fmaxf(M, a.part_m[static_cast<size_t>(s) * a.N + i]);
      float L = 0.f;
      for (int s = 0; s < a.splits; ++s)
        L += a.part_l[static_cast<size_t>(s) * a.N + i] * exp2f(a.part_m[static_cast<size_t>(s) * a.N + i] - M);
      l2 = M + log2f(L);
      zyi = a.zy[i];
    }
    if (a.mode == COMBINE_SHARD) {
      // zy holds a value only for rows whose target this shard holds
      a.shard_lse[a.perm[i]] = static_cast<float>(static_cast<double>(l2) * LN2);
      a.shard_zy[a.perm[i]] = valid && yi >= 0 && yi < a.V ? zyi : 0.f;
      return;
    }
    a.lse2[i] = l2;
    double row = 0.0;
    if (valid) {
      row = static_cast<double>(l2) * LN2 - static_cast<double>(zyi);
      vi = 1;
      // mean and sum add the plain row losses (the mean divides at the end)
      li = a.reduction == RED_NONE && a.grad_row_scale ? row * static_cast<double>(a.grad_row_scale[i]) : row;
    }
    if (a.row_loss) a.row_loss[a.perm[i]] = static_cast<float>(row);
  } else if (a.mode == COMBINE_SHARD) {
    return;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    li += __shfl_down_sync(0xffffffffu, li, o);
    vi += __shfl_down_sync(0xffffffffu, vi, o);
  }
  __shared__ double wl[COMBINE_THREADS / 32];
  __shared__ int wc[COMBINE_THREADS / 32];
  __shared__ bool is_last;
  if ((threadIdx.x & 31) == 0) {
    wl[threadIdx.x >> 5] = li;
    wc[threadIdx.x >> 5] = vi;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double sl = 0.0;
    int sc = 0;
    for (int w = 0; w < COMBINE_THREADS / 32; ++w) {
      sl += wl[w];
      sc += wc[w];
    }
    a.blk_loss[blockIdx.x] = sl;
    a.blk_cnt[blockIdx.x] = sc;
    __threadfence();
    is_last = atomicAdd(a.ticket, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (is_last && threadIdx.x == 0) {
    __threadfence();
    const volatile double* bl = a.blk_loss;
    const volatile int* bc = a.blk_cnt;
    double tot = 0.0;
    long long cnt = 0;
    for (unsigned b = 0; b < gridDim.x; ++b) {
      tot += bl[b];
      cnt += bc[b];
    }
    *a.n_valid = static_cast<int>(cnt);
    // a data-parallel caller divides by the count over every rank's tokens
    const long long den = a.mean_count ? static_cast<long long>(*a.mean_count) : cnt;
    *a.inv_n = den > 0 ? static_cast<float>(1.0 / static_cast<double>(den)) : 0.f;
    if (a.reduction == RED_MEAN)
      *a.loss = den > 0 ? static_cast<float>(tot / static_cast<double>(den)) : 0.f;
    else
      *a.loss = static_cast<float>(tot);
    *a.ticket = 0u;
  }
}

// ================================================== bounded-wait probe ==
//
// Exercises the two bounded waits every kernel above relies on, on things that
// never happen: an mbarrier phase nobody arrives on and a global counter
// nobody increments.  Each wait must give up after `timeout_ns` and report
// ST_TIMEOUT in its own status slot, leaving the context usable.
__global__ void flce_wait_probe_kernel(int* status, const int* never, unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  mbar_init(smem_u32(&bar), 1);
  fence_mbar_init();
  if (!mbar_wait(smem_u32(&bar), 0, &abort_flag, timeout_ns)) status[0] = ST_TIMEOUT;
  if (!wait_counter(never, 1, &abort_flag, timeout_ns)) status[1] = ST_TIMEOUT;
}

// ======================================== cross-entropy on given logits ==
//
// The same loss and gradient from a logit tensor the caller already holds
// ("Complete Guide to Liger Kernel", section LigerCrossEntropyLoss).  Memory
// bound: one CTA per row reads the row once for its online (max, sum) and once
// more (an L2 hit while the row is in flight) to write the bf16 gradient,
// in place if the caller wishes.

constexpr int CE_THREADS = 512;
constexpr int CE_UNROLL = 4;  // 16-byte loads in flight per thread

struct CeArgs {
  const uint16_t* logits;  // [N][V] bf16
  uint16_t* dlogits;       // [N][V] bf16 or null (forward only); may equal logits
  const int32_t* y;
  int N, V, ignore_index, reduction, TM;
  const float* grad_row_scale;
  const int* tile_valid;   // [TM] valid rows per 256-row tile (prep kernel)
  const int* n_valid;      // valid rows of the whole call (prep kernel)
  double* row_acc;         // [N] weighted row losses for the deterministic sum
  float* row_loss;         // [N] or null
  double* blk_sum;         // [ceil(N / COMBINE_THREADS)]
  unsigned int* ticket;
  float* loss;
  int* status;
};

__device__ __forceinline__ void lse_merge(float& m, float& l, float m2, float l2) {
  const float mn = fmaxf(m, m2);
  l = l * ex2_approx(m - mn) + l2 * ex2_approx(m2 - mn);
  m = mn;
}

__device__ __forceinline__ void unpack_bf16x8(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = bf16lo_to_f32(w[e]);
    f[2 * e + 1] = bf16hi_to_f32(w[e]);
  }
}

__global__ void __launch_bounds__(CE_THREADS) flce_ce_rows_kernel(const CeArgs a) {
  __shared__ float sm_m[CE_THREADS / 32], sm_l[CE_THREADS / 32];
  __shared__ float s_zy, s_lse2;
  __shared__ int s_n;
  const int tid = threadIdx.x;
  if (tid == 0) s_n = *a.n_valid;
  const bool vec = (a.V & 7) == 0 && (reinterpret_cast<uintptr_t>(a.logits) & 15) == 0 &&
                   (a.dlogits == nullptr || (reinterpret_cast<uintptr_t>(a.dlogits) & 15) == 0);
#pragma unroll 1
  for (int row = blockIdx.x; row < a.N; row += gridDim.x) {
    const uint16_t* z = a.logits + static_cast<size_t>(row) * a.V;
    const int yi = a.y[row];
    const bool in_range = yi >= 0 && yi < a.V;
    const bool valid = yi != a.ignore_index && in_range;
    if (tid == 0 && yi != a.ignore_index && !in_range) raise_status(a.status, ST_TARGET_OUT_OF_RANGE);
    if (tid == 0) s_zy = 0.f;
    __syncthreads();
    // ---- online max and sum of 2^(z log2 e) over the row.  The row is read
    // again for the gradient: keep it in L2 (evict_last) until then; the
    // second read and the gradient stores are its last touch (evict_first).
    float m = -1e30f, l = 0.f;
    const uint64_t keep = l2_evict_last(), last = l2_evict_first();
    if (vec) {
      const uint4* zv = reinterpret_cast<const uint4*>(z);
      const int nv = a.V >> 3;
#pragma unroll 1
      for (int base = tid; base < nv; base += CE_THREADS * CE_UNROLL) {
        uint4 buf[CE_UNROLL];
#pragma unroll
        for (int u = 0; u < CE_UNROLL; ++u) {
          const int j = base + u * CE_THREADS;
          buf[u] = j < nv ? ld_l2hint_v4(zv + j, keep) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < CE_UNROLL; ++u) {
          const int j = base + u * CE_THREADS;
          if (j < nv) {
            float f[8];
            unpack_bf16x8(buf[u], f);
            if (static_cast<unsigned>(yi - 8 * j) < 8u) s_zy = f[yi - 8 * j];
            float cm = f[0];
#pragma unroll
            for (int e = 1; e < 8; ++e) cm = fmaxf(cm, f[e]);
            const float mn = fmaxf(m, cm * LOG2E);
            float acc = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc += ex2_approx(fmaf(f[e], LOG2E, -mn));
            l = l * ex2_approx(m - mn) + acc;
            m = mn;
          }
        }
      }
    } else {
#pragma unroll 1
      for (int j = tid; j < a.V; j += CE_THREADS) {
        const float f = __uint_as_float(static_cast<uint32_t>(z[j]) << 16);
        if (j == yi) s_zy = f;
        const float mn = fmaxf(m, f * LOG2E);
        l = l * ex2_approx(m - mn) + ex2_approx(fmaf(f, LOG2E, -mn));
        m = mn;
      }
    }
    // ---- block reduction of (m, l), fixed order
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
      const float l2 = __shfl_xor_sync(0xffffffffu, l, o);
      lse_merge(m, l, m2, l2);
    }
    if ((tid & 31) == 0) {
      sm_m[tid >> 5] = m;
      sm_l[tid >> 5] = l;
    }
    __syncthreads();
    if (tid == 0) {
      float M = sm_m[0], L = sm_l[0];
      for (int w = 1; w < CE_THREADS / 32; ++w) {
        const float mn = fmaxf(M, sm_m[w]);
        L = L * exp2f(M - mn) + sm_l[w] * exp2f(sm_m[w] - mn);
        M = mn;
      }
      const float lse2 = M + log2f(L);
      s_lse2 = lse2;
      const double row_l = valid ? static_cast<double>(lse2) * LN2 - static_cast<double>(s_zy) : 0.0;
      const double wgt = (a.reduction == RED_NONE && a.grad_row_scale && valid) ? a.grad_row_scale[row] : 1.0;
      a.row_acc[row] = row_l * wgt;
      if (a.row_loss) a.row_loss[row] = static_cast<float>(row_l);
    }
    __syncthreads();
    // ---- gradient: s_i (softmax - onehot), bf16
    if (a.dlogits) {
      uint16_t* g = a.dlogits + static_cast<size_t>(row) * a.V;
      const float inv_n = s_n ? 1.f / static_cast<float>(s_n) : 0.f;
      const float sc = valid ? row_weight(a.reduction, &inv_n, a.grad_row_scale, row) : 0.f;
      const float l2r = s_lse2;
      if (vec) {
        const uint4* zv = reinterpret_cast<const uint4*>(z);
        uint4* gv = reinterpret_cast<uint4*>(g);
        const int nv = a.V >> 3;
#pragma unroll 1
        for (int base = tid; base < nv; base += CE_THREADS * CE_UNROLL) {
          uint4 buf[CE_UNROLL];
#pragma unroll
          for (int u = 0; u < CE_UNROLL; ++u) {
            const int j = base + u * CE_THREADS;
            buf[u] = (j < nv && valid) ? ld_l2hint_v4(zv + j, last) : make_uint4(0, 0, 0, 0);
          }
#pragma unroll
          for (int u = 0; u < CE_UNROLL; ++u) {
            const int j = base + u * CE_THREADS;
            if (j < nv) {
              float f[8];
              unpack_bf16x8(buf[u], f);
              float o[8];
#pragma unroll
              for (int e = 0; e < 8; ++e)
                o[e] = valid ? ex2_approx(fmaf(f[e], LOG2E, -l2r)) * sc : 0.f;
              if (valid && static_cast<unsigned>(yi - 8 * j) < 8u) o[yi - 8 * j] -= sc;
              st_l2hint_v4(gv + j,
                           make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                                      pack_bf16x2(o[6], o[7])),
                           last);
            }
          }
        }
      } else {
#pragma unroll 1
        for (int j = tid; j < a.V; j += CE_THREADS) {
          float o = 0.f;
          if (valid) {
            const float f = __uint_as_float(static_cast<uint32_t>(z[j]) << 16);
            o = ex2_approx(fmaf(f, LOG2E, -l2r)) * sc;
            if (j == yi) o -= sc;
          }
          __nv_bfloat16 b = __float2bfloat16_rn(o);
          g[j] = *reinterpret_cast<uint16_t*>(&b);
        }
      }
    }
    __syncthreads();  // s_zy / s_lse2 are reused by the next row
  }
}

// Deterministic sum of the weighted row losses: fixed tree per block, then the
// last block adds the block sums in order (fp64); 'mean' divides by n_valid.
__global__ void __launch_bounds__(COMBINE_THREADS) flce_ce_reduce_kernel(const CeArgs a) {
  const int i = blockIdx.x * COMBINE_THREADS + threadIdx.x;
  double v = i < a.N ? a.row_acc[i] : 0.0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
  __shared__ double wsum[COMBINE_THREADS / 32];
  __shared__ bool is_last;
  if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < COMBINE_THREADS / 32; ++w) t += wsum[w];
    a.blk_sum[blockIdx.x] = t;
    __threadfence();
    is_last = atomicAdd(a.ticket, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (is_last && threadIdx.x == 0) {
    __threadfence();
    const volatile double* b = a.blk_sum;
    double tot = 0.0;
    for (unsigned k = 0; k < gridDim.x; ++k) tot += b[k];
    const long long n = *a.n_valid;
    if (a.reduction == RED_MEAN)
      *a.loss = n ? static_cast<float>(tot / static_cast<double>(n)) : 0.f;
    else
      *a.loss = static_cast<float>(tot);
    *a.ticket = 0u;
  }
}

// ------------------------------------------------- pairwise preference loss --
//
// The logistic (DPO-form) preference loss on per-row log-probabilities of the
// head ("Liger-Kernel: Triton kernels that replace HF training ops", section
// "Installation and the one-line patch": the fused-linear post-training losses
// take the LM-head weight, the hidden states and the targets and return the
// loss).  Sequence s holds the token rows [seq_start[s], seq_start[s+1]);
// logp_s = -sum of their row losses; pair k compares sequences chosen[k] and
// rejected[k]:
//   m_k  = beta ((logp_c - ref_c) - (logp_r - ref_r))
//   L    = (1/P) sum_k softplus(-m_k)          (= -mean log sigmoid(m_k))
//   dL/dlogp_s = (beta/P) sum_k sigmoid(-m_k) ([s == r_k] - [s == c_k])
// and each valid row i of sequence s gets the upstream weight
// w_i = -dL/dlogp_s of its own row loss (d logp_s / d l_i = -1).
// All sums are fp64 in a fixed order.

struct PrefArgs {
  const float* row_loss;    // [N]
  const int32_t* y;         // [N], for the valid mask of the weights
  const int32_t* seq_start; // [S + 1]
  const int32_t* chosen;    // [P]
  const int32_t* rejected;  // [P]
  const double* ref_logp;   // [S] or null
  double beta;
  int N, S, P, ignore_index;
  double* logp;             // [S]
  double* grad_logp;        // [S]
  double* loss;             // [1]
  float* row_weight;        // [N]
  int* status;
};

constexpr int PREF_THREADS = 256;

// One block per sequence: logp_s by a fixed-order block sum; checks the row ranges.
__global__ void __launch_bounds__(PREF_THREADS) flce_pref_logp_kernel(const PrefArgs a) {
  const int s = blockIdx.x;
  const int r0 = a.seq_start[s], r1 = a.seq_start[s + 1];
  const bool ok = r0 >= 0 && r0 <= r1 && r1 <= a.N;
  if (!ok) {
    if (threadIdx.x == 0) {
      raise_status(a.status, 1 /* FLCE_ERR_INVALID_ARGUMENT */);
      a.logp[s] = 0.0;
    }
    return;
  }
  double v = 0.0;
  for (int i = r0 + static_cast<int>(threadIdx.x); i < r1; i += PREF_THREADS) v += static_cast<double>(a.row_loss[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
  __shared__ double w[PREF_THREADS / 32];
  if ((threadIdx.x & 31) == 0) w[threadIdx.x >> 5] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int k = 0; k < PREF_THREADS / 32; ++k) t += w[k];
    a.logp[s] = -t;
  }
}

__device__ __forceinline__ double pref_margin(const PrefArgs& a, int k) {
  const int c = a.chosen[k], r = a.rejected[k];
  const double dc = a.logp[c] - (a.ref_logp ? a.ref_logp[c] : 0.0);
  const double dr = a.logp[r] - (a.ref_logp ? a.ref_logp[r] : 0.0);
  return a.beta * (dc - dr);
}

// One block: the loss (fixed-order block sum over the pairs) and, one thread
// per sequence, dL/dlogp_s summed over the pairs in pair order.
__global__ void __launch_bounds__(PREF_THREADS) flce_pref_pairs_kernel(const PrefArgs a) {
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  for (int k = threadIdx.x; k < a.P; k += PREF_THREADS) {
    const int c = a.chosen[k], r = a.rejected[k];
    if (c < 0 || c >= a.S || r < 0 || r >= a.S) bad = 1;
  }
  __syncthreads();
  if (bad) {
    if (threadIdx.x == 0) {
      raise_status(a.status, 1 /* FLCE_ERR_INVALID_ARGUMENT */);
      *a.loss = 0.0;
    }
    for (int s = threadIdx.x; s < a.S; s += PREF_THREADS) a.grad_logp[s] = 0.0;
    return;
  }
  const double invP = 1.0 / static_cast<double>(a.P);
  double v = 0.0;
  for (int k = threadIdx.x; k < a.P; k += PREF_THREADS) {
    const double m = pref_margin(a, k);
    v += fmax(-m, 0.0) + log1p(exp(-fabs(m)));  // softplus(-m)
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
  __shared__ double w[PREF_THREADS / 32];
  if ((threadIdx.x & 31) == 0) w[threadIdx.x >> 5] = v;
  for (int s = threadIdx.x; s < a.S; s += PREF_THREADS) {
    double g = 0.0;
    for (int k = 0; k < a.P; ++k) {
      const int c = a.chosen[k], r = a.rejected[k];
      if (c != s && r != s) continue;
      const double m = pref_margin(a, k);
      const double sg = 1.0 / (1.0 + exp(m));  // sigmoid(-m)
      if (r == s) g += a.beta * sg * invP;
      if (c == s) g -= a.beta * sg * invP;
    }
    a.grad_logp[s] = g;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int k = 0; k < PREF_THREADS / 32; ++k) t += w[k];
    *a.loss = t * invP;
  }
}

// One block per sequence: the upstream weights of its valid rows (the rest of
// row_weight was zeroed beforehand).
__global__ void __launch_bounds__(PREF_THREADS) flce_pref_weights_kernel(const PrefArgs a) {
  const int s = blockIdx.x;
  const int r0 = a.seq_start[s], r1 = a.seq_start[s + 1];
  if (!(r0 >= 0 && r0 <= r1 && r1 <= a.N)) return;
  const float wgt = static_cast<float>(-a.grad_logp[s]);
  for (int i = r0 + static_cast<int>(threadIdx.x); i < r1; i += PREF_THREADS)
    a.row_weight[i] = a.y[i] != a.ignore_index ? wgt : 0.f;
}

}  // namespace flce
