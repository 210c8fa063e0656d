// k_loss_gemm.cu — the candidate forward and its loss ("AWQ：为什么 4-bit 权重量化要先观察
// Activation" §4: every candidate is scored by the mean squared difference between the
// original output and the candidate output, the difference cast to FP32).
//
// One persistent kernel, six modes:
//   mode 0: Y = X_b W_b, written once to HBM in a tile-major layout;
//   mode 1: for every (candidate i, output tile): acc = X_b W_hat_i,b on the tensor
//           cores, and the epilogue adds (acc - Y)^2 over the tile and writes one fp64
//           partial sum. The candidate output Y_hat is never written to HBM. With
//           cand_inner the walk visits, for each column tile of a raster group, every
//           candidate before the next column tile, so each tile of Y is read from DRAM once
//           and by the other candidates from L2 (used when Y is larger than L2);
//   mode 2: a plain product A B^T (B stored K-major), written row-major in fp32 with
//           the ragged rows and columns masked (the packed artifact's consumer);
//   mode 4: modes 0 and 1 in one launch: units 0 .. tiles - 1 are the reference tiles
//           (B slot 0), the rest the candidates' (slot 1 + c). A reference tile's epilogue
//           publishes a per-tile flag after its Y stores; a candidate tile's epilogue waits
//           for the flag (bounded) before it reads Y. Every CTA finishes its reference tiles
//           before it starts a candidate tile, and the grid never exceeds the SMs (one CTA
//           each), so every flag a CTA waits for is set by a CTA that is running;
//   mode 3: the MLP block's first GEMM, B = [W_gate | W_up] interleaved by 128 columns so
//           that a 256-column tile holds the gate and up halves of 128 intermediate
//           columns; the epilogue writes h = bf16(silu(g) u) row-major and never stores
//           the fp32 halves;
//   mode 5: a plain product per candidate, rounded to bf16 and written row-major (the
//           attention block's Q, K and V^T operands), ragged rows and columns masked.
//
// Blackwell structure (sm_100a): 128 x 256 output tiles, K in 64-element (128-byte)
// slices; a 4-stage TMA -> shared-memory ring (128-byte swizzle, no multicast); one
// elected thread issues tcgen05.mma (M=128, N=256, K=16, bf16 -> fp32) into one of
// two 256-column tensor-memory accumulators, so the epilogue of tile t overlaps the
// main loop of tile t+1; four epilogue warps read the accumulator with tcgen05.ld
// (warp w % 4 owns TMEM lanes 32(w%4)..+31 = tile rows). Warp roles: 0 TMA producer,
// 1 MMA issuer, 2 TMEM allocator, 4-7 epilogue, and in loss_gemm_kernel<true> 8-15 the
// QDQ warps, which make the candidate operands (the tile routine of qdq_tile.cuh) while
// the tensor cores run, publishing each finished piece through a per-tile counter that
// the producer waits for. Units (candidate, tile) are walked in a grouped raster
// (group_m row tiles at a time) so the X row block and the W_hat column block of
// neighbouring CTAs stay in L2.
//
// Every wait is bounded (global timer); a wait that runs out sets the call's
// timeout bit, raises a CTA-wide abort flag, the producer waits for its own copies in
// flight, the MMA thread waits for its issued MMAs, and tensor memory is freed.
#include "awq_device.cuh"
#include "awq_kernels.h"
#include "qdq_tile.cuh"

#include <cudaTypedefs.h>
#include <cstdlib>
#include <cstdio>

namespace awq {
namespace {

constexpr int BM = kTileM, BN = kTileN, BK = kTileK;
constexpr int kStages = 4;
constexpr int kABytes = BM * BK * 2;  // 16 KB
constexpr int kBBytes = BN * BK * 2;  // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kTmemCols = 2 * BN;     // two fp32 accumulators of 256 columns
constexpr int kThreads = 256;
constexpr int kEpiThreads = 128;
constexpr int kBarrierBytes = 256;
constexpr int kSmemBytes = kStages * kStageBytes + kBarrierBytes + 1024;  // + alignment slack
// Row tiles per raster group (the host picks one per launch): 32 when a group's rows of A
// take at most 32 MB (K <= 4096), which keeps them and the group's W_hat column blocks in
// L2 (measured 3.8 % faster than 16 on the 4096^3 layer), else 16. On the 70B gate+up layer
// (K = 8192; one B200, 15 searches each, interleaved) 16 row tiles took 259.2 ms per launch,
// 32 took 266.3 ms (their 64 MB of rows of X do not stay in L2 while a candidate's column
// tiles are swept: 440 GB of DRAM reads per launch) and 8 took 267.5 ms; the MLP block's
// second GEMM (K = 11008) ran 2 % slower with 32.
constexpr int kGroupMLarge = 32, kGroupMSmall = 16;
inline int raster_group_m(int64_t K) {
  return static_cast<int64_t>(kGroupMLarge) * kTileM * K * 2 <= (int64_t(32) << 20) ? kGroupMLarge : kGroupMSmall;
}
constexpr uint64_t kDrainNs = 200ull * 1000 * 1000;  // bound on the waits of the abort path

struct GemmParams {
  int mode;
  int n_grid;
  int tiles_m, tiles_n;
  int nk;
  int64_t M, N, ldo;  // mode 2: output rows, columns and row pitch
  int f16;            // mode 2: operands are fp16 (else bf16)
  int group_m;        // row tiles per raster group
  int slot_base;      // B slot of candidate 0 (modes 1, 3) or the slot multiplied (mode 2)
  int cands;          // candidates this launch walks (modes 1 and 3)
  int b_per_cand;     // modes 1, 3: B slot = slot_base + c (1) or slot_base for every c (0)
  int a_slotted;      // A is a stack of slots (3-D map); candidate c reads slot a_slot_base + c
  int a_slot_base;
  float* Y;           // modes 0, 1, 4: the tiled reference output; mode 2: the row-major output
  int* ready;         // mode 4: per-tile flags, zero at launch, set once a reference tile is in Y
  __nv_bfloat16* H;   // mode 3: the row-major bf16 intermediate of candidate 0 (pitch ldo)
  int64_t h_stride;   // mode 3: elements between successive candidates' intermediates
  double* partial;
  int* err;
  uint64_t timeout_ns;
  int fault_mode;
  int cand_inner;     // mode 1: raster group -> column tile -> candidate -> row tile
  int64_t K;
  // QDQ warps (loss_gemm_kernel<true>): the candidate operand slots of a K x N bf16 W are
  // made by warps 8 .. 15 of the same CTAs while the tensor cores run, in pieces claimed
  // column-major from a counter that spans the launches of one search: a piece is a
  // 128 x 32 tile of W for a chunk of up to kQdqChunk candidates, qdq_ready[nt] counts the
  // finished pieces of the operand's 256-row tile nt, and a load of a candidate slot's
  // tile nt (mode 1, or modes 3 and 5 past slot 0) waits for that count. A second
  // operand (qdq_W2: another column range, no counters; the attention block's W_v) is
  // made after the first by the same claims. qdq_ready[ceil(qdq_N / 256)] is the claim
  // counter.
  const __nv_bfloat16* qdq_W;  // [qdq_K][qdq_N], row pitch qdq_ldw
  const float* qdq_S;          // [qdq_grid][qdq_K] candidate scales
  __nv_bfloat16* qdq_Wt;       // [qdq_grid + 1][qdq_N][qdq_K]
  int* qdq_ready;
  int qdq_cands;               // claim pieces: 1 until none is left, 2 while this CTA's GEMM runs
  int qdq_quantizer;
  int64_t qdq_K, qdq_N, qdq_interleave, qdq_ldw;
  int qdq_grid;
  const __nv_bfloat16* qdq_W2;  // [qdq_K][qdq_N2], row pitch qdq_ldw, or null
  __nv_bfloat16* qdq_Wt2;       // [qdq_grid + 1][qdq_N2][qdq_K]
  int64_t qdq_N2;
};

// QDQ warps: group 128, tiles of 128 rows x 32 columns (8 warps of 16 row-lanes x 2
// column-lanes, each lane 8 rows of 2 columns), up to kQdqChunk candidates staged per
// pass over a tile.
using QdqTile = Tile<128, 32>;
constexpr int kQdqTileCols = QdqTile::kCols;
constexpr int kQdqThreads = QdqTile::kThreads;  // 256
constexpr int kQdqChunk = 10;
constexpr int kQdqSmemBytes = kQdqTileCols * QdqTile::kPitch * 4 + 2 * kQdqChunk * QdqTile::kSkewPitch * 4 +
                              kQdqChunk * kQdqTileCols * 16 + 16;
static_assert(kQdqThreads == 256, "QDQ warps 8 .. 15");
static_assert((kQdqTileCols * QdqTile::kPitch * 4) % 16 == 0 && (QdqTile::kSkewPitch * 4 * 2) % 16 == 0,
              "16-byte aligned parameter sets");
constexpr int kQdqColsPerTileN = kTileN / kQdqTileCols;  // 8 QDQ column blocks per GEMM column tile

// Finished QDQ pieces a 256-row tile of the operand needs: its 32-column blocks of W (the
// last tile may be ragged; with the gate/up interleave every tile holds four of each
// half) times the groups of K times the candidate chunks.
__device__ __forceinline__ int qdq_target(const GemmParams& p, int nt) {
  const int64_t cols = min(static_cast<int64_t>(kTileN), p.qdq_N - static_cast<int64_t>(nt) * kTileN);
  return static_cast<int>(ceil_div(cols, static_cast<int64_t>(kQdqTileCols)) * (p.qdq_K / 128) *
                          ceil_div(p.qdq_grid, kQdqChunk));
}

// The column of W held by row `row` of the K-major candidate operand (the inverse of the
// QDQ tile's interleaved_column): with the MLP block's interleave F > 0 every 256 rows
// hold 128 gate columns, then the 128 up columns of the same outputs.
__device__ __forceinline__ int64_t qdq_w_column(int64_t row, int64_t interleave) {
  if (interleave <= 0) return row;
  const int64_t nt = row / kTileN, j = row - nt * kTileN;
  return j < kTileN / 2 ? nt * (kTileN / 2) + j : interleave + nt * (kTileN / 2) + (j - kTileN / 2);
}

struct QdqWarpsSync {
  __device__ __forceinline__ void operator()() const { asm volatile("bar.sync 5, 256;" ::: "memory"); }
};

__device__ __forceinline__ void unit_coords(int64_t u, const GemmParams& p, int& c, int& mt, int& nt) {
  if (p.cand_inner) {
    const int64_t group_units = static_cast<int64_t>(p.group_m) * p.tiles_n * p.cands;  // a full group
    const int64_t gi = u / group_units;
    const int first_m = static_cast<int>(gi * p.group_m);
    const int gm = min(p.group_m, p.tiles_m - first_m);
    const int64_t r = u - gi * group_units;
    const int64_t per_column = static_cast<int64_t>(gm) * p.cands;
    nt = static_cast<int>(r / per_column);
    const int rc = static_cast<int>(r - nt * per_column);
    c = rc / gm;
    mt = first_m + rc % gm;
    return;
  }
  const int64_t tiles = static_cast<int64_t>(p.tiles_m) * p.tiles_n;
  c = static_cast<int>(u / tiles);
  const int64_t t = u - static_cast<int64_t>(c) * tiles;
  const int64_t group_size = static_cast<int64_t>(p.group_m) * p.tiles_n;
  const int64_t gi = t / group_size;
  const int first_m = static_cast<int>(gi * p.group_m);
  const int gm = min(p.group_m, p.tiles_m - first_m);
  const int64_t r = t - gi * group_size;
  mt = first_m + static_cast<int>(r % gm);
  nt = static_cast<int>(r / gm);
}

__device__ __forceinline__ int named_barrier_or(uint32_t id, uint32_t nthreads, int pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %3, 0;\n\t"
      "bar.red.or.pred p, %1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(id), "r"(nthreads), "r"(pred)
      : "memory");
  return static_cast<int>(r);
}

template <bool kQdq>
__global__ void __launch_bounds__(kQdq ? kThreads + kQdqThreads : kThreads, 1)
    loss_gemm_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                     const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * kABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* full = bars;                    // [kStages] TMA landed
  uint64_t* empty = bars + kStages;         // [kStages] MMAs done reading the stage
  uint64_t* tfull = bars + 2 * kStages;     // [2] accumulator ready
  uint64_t* tempty = bars + 2 * kStages + 2;  // [2] accumulator drained by the epilogue
  uint64_t* drain = bars + 2 * kStages + 4;   // [1] abort path: all issued MMAs done
  double* red = reinterpret_cast<double*>(bars + 2 * kStages + 5);  // [2][4]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 13);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* gemm_done = reinterpret_cast<volatile int*>(bars + 2 * kStages + 14);  // the epilogue's last unit is done
  volatile int* qdq_claim = gemm_done + 1;  // the QDQ warps' current candidate tile

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull + a, 1);
      mbar_init(tempty + a, kEpiThreads);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    *gemm_done = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapA);
    tma_prefetch_desc(&mapB);
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int64_t tiles = static_cast<int64_t>(p.tiles_m) * p.tiles_n;
  const int64_t n_units =
      (p.mode == 1 || p.mode == 3 || p.mode == 5 ? p.cands : (p.mode == 4 ? p.n_grid + 1 : 1)) * tiles;
  const uint64_t budget = p.timeout_ns;

  auto fail = [&]() {
    *abort_flag = 1;
    atomicOr(p.err, kErrTimeout);
  };

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_parity = 0;  // per-stage bits
      bool ok = true;
      bool fault_pending = p.fault_mode == 1;
      int confirmed = -1;  // the last operand tile whose candidate slots were seen complete
      (void)confirmed;
      for (int64_t u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        int c, mt, nt;
        unit_coords(u, p, c, mt, nt);
        if constexpr (kQdq) {
          // a candidate operand: its tile nt must be complete for every candidate
          const bool cand = p.mode == 1 || ((p.mode == 3 || p.mode == 5) && p.slot_base + c >= 1);
          if (cand && confirmed != nt) {
            if (!counter_wait_bounded(p.qdq_ready + nt, qdq_target(p, nt), abort_flag, budget)) {
              ok = false;
              break;
            }
            fence_proxy_async_global();
            confirmed = nt;
          }
        }
        const int slot = p.mode == 0 ? 0
                         : p.mode == 4 ? c  // 0: bf16(W), then candidate c - 1 in slot c
                                       : p.slot_base +
                                             ((p.mode == 1 || p.mode == 3 || p.mode == 5) && p.b_per_cand ? c : 0);
        for (int kb = 0; kb < p.nk; ++kb) {
          if (!mbar_wait_bounded(empty + stage, phase ^ 1u, abort_flag, budget)) {
            ok = false;
            break;
          }
          // fault injection: the first candidate unit of the CTA loses its first copy
          const bool skip = fault_pending && (p.mode == 1 || (p.mode == 4 && c > 0)) && kb == 0;
          if (skip) fault_pending = false;
          if (!skip) {
            mbar_arrive_expect_tx(full + stage, kStageBytes);
            if (p.a_slotted)
              tma_load_3d(&mapA, full + stage, sA + stage * kABytes, kb * BK, mt * BM, p.a_slot_base + c);
            else
              tma_load_2d(&mapA, full + stage, sA + stage * kABytes, kb * BK, mt * BM);
            tma_load_3d(&mapB, full + stage, sB + stage * kBBytes, kb * BK, nt * BN, slot);
            issued |= 1u << stage;
            last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          }
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        fail();
        // let the copies this thread started land before the CTA goes away
        for (int s = 0; s < kStages; ++s)
          if (issued & (1u << s)) mbar_wait_bounded(full + s, (last_parity >> s) & 1u, nullptr, kDrainNs);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = p.f16 ? idesc_f16_f32(BM, BN) : idesc_bf16_f32(BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int local = 0;
      for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x, ++local) {
        const int acc = local & 1;
        const uint32_t acc_parity = (local >> 1) & 1;
        if (!mbar_wait_bounded(tempty + acc, acc_parity ^ 1u, abort_flag, budget)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < p.nk; ++kb) {
          if (!mbar_wait_bounded(full + stage, phase, abort_flag, budget)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = smem_desc_k_sw128(smem_u32(sA + stage * kABytes));
          const uint64_t bdesc = smem_desc_k_sw128(smem_u32(sB + stage * kBBytes));
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)  // K = 16 per MMA: advance 32 bytes = 2 descriptor units
            umma_bf16_f32(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
          umma_commit(empty + stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(tfull + acc);
      }
      if (!ok) {
        fail();
        umma_commit(drain);
        mbar_wait_bounded(drain, 0, nullptr, kDrainNs);
      }
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------- epilogue
    const int ew = warp - 4;  // == warp % 4: TMEM lanes 32*ew .. 32*ew+31
    const int row = ew * 32 + lane;
    int local = 0;
    for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x, ++local) {
      int c, mt, nt;
      unit_coords(u, p, c, mt, nt);
      const int acc = local & 1;
      const uint32_t acc_parity = (local >> 1) & 1;
      const bool ok = mbar_wait_bounded(tfull + acc, acc_parity, abort_flag, budget);
      if (named_barrier_or(1, kEpiThreads, !ok)) {
        if (!ok) fail();
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(ew * 32) << 16) + static_cast<uint32_t>(acc * BN);
      if (p.mode == 3) {
        // columns j (gate) and BN/2 + j (up) of the accumulator are the two halves of
        // intermediate column nt * BN/2 + j
        const int64_t grow = static_cast<int64_t>(mt) * BM + row;
#pragma unroll 1
        for (int j0 = 0; j0 < BN / 2; j0 += 32) {
          uint32_t g[32], up[32];
          tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(j0), g);
          tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(BN / 2 + j0), up);
          tmem_ld_wait();
          if (grow < p.M) {
            uint4* orow = reinterpret_cast<uint4*>(p.H + static_cast<int64_t>(c) * p.h_stride + grow * p.ldo +
                                                   static_cast<int64_t>(nt) * (BN / 2) + j0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int k = 8 * q + 2 * e;
                const __nv_bfloat162 hv =
                    __floats2bfloat162_rn(silu_mul_f32(__uint_as_float(g[k]), __uint_as_float(up[k])),
                                          silu_mul_f32(__uint_as_float(g[k + 1]), __uint_as_float(up[k + 1])));
                w[e] = *reinterpret_cast<const uint32_t*>(&hv);
              }
              orow[q] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(tempty + acc);
        continue;
      }
      if (p.mode == 5) {
        // the product of candidate c rounded to bf16, row-major with pitch ldo
        const int64_t grow = static_cast<int64_t>(mt) * BM + row;
#pragma unroll 1
        for (int j0 = 0; j0 < BN; j0 += 32) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(j0), v);
          tmem_ld_wait();
          const int64_t col0 = static_cast<int64_t>(nt) * BN + j0;
          if (grow < p.M) {
            uint4* orow = reinterpret_cast<uint4*>(p.H + static_cast<int64_t>(c) * p.h_stride + grow * p.ldo + col0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {  // N % 8 == 0: eight columns lie wholly inside or outside
              if (col0 + 8 * q >= p.N) continue;
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const __nv_bfloat162 hv = __floats2bfloat162_rn(__uint_as_float(v[8 * q + 2 * e]),
                                                                __uint_as_float(v[8 * q + 2 * e + 1]));
                w[e] = *reinterpret_cast<const uint32_t*>(&hv);
              }
              orow[q] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(tempty + acc);
        continue;
      }
      const int64_t tile = static_cast<int64_t>(mt) * p.tiles_n + nt;
      // mode 4: unit c = 0 is a reference tile, c > 0 candidate c - 1's
      const bool ref_tile = p.mode == 0 || (p.mode == 4 && c == 0);
      const bool loss_tile = p.mode == 1 || (p.mode == 4 && c > 0);
      const int lc = p.mode == 4 ? c - 1 : c;
      if (p.mode == 4 && c > 0) {
        // the reference tile this candidate tile is compared with must be in Y
        int ready = 1;
        if (ew == 0 && lane == 0) ready = flag_wait_bounded(p.ready + tile, abort_flag, budget);
        if (named_barrier_or(3, kEpiThreads, !ready)) {
          if (!ready) fail();
          break;
        }
      }
      float4* ytile = reinterpret_cast<float4*>(p.Y + tile * (BM * BN));
      float sq = 0.0f;
#pragma unroll 1
      for (int j0 = 0; j0 < BN; j0 += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(j0), v);
        tmem_ld_wait();
        float4* yrow = ytile + (j0 / 4) * BM + row;  // tile layout [BN/4][BM][4]
        if (p.mode == 2) {
          const int64_t grow = static_cast<int64_t>(mt) * BM + row;
          if (grow < p.M) {
            const int64_t col0 = static_cast<int64_t>(nt) * BN + j0;
            float4* orow = reinterpret_cast<float4*>(p.Y + grow * p.ldo + col0);
#pragma unroll
            for (int q = 0; q < 8; ++q)  // N % 8 == 0: a float4 lies wholly inside or outside
              if (col0 + 4 * q < p.N)
                orow[q] = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                      __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
          }
        } else if (ref_tile) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            yrow[q * BM] = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                       __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 y = __ldcg(yrow + q * BM);  // through L2: mode 4 wrote it in this launch
            const float d0 = __uint_as_float(v[4 * q]) - y.x;
            const float d1 = __uint_as_float(v[4 * q + 1]) - y.y;
            const float d2 = __uint_as_float(v[4 * q + 2]) - y.z;
            const float d3 = __uint_as_float(v[4 * q + 3]) - y.w;
            sq = fmaf(d0, d0, sq);
            sq = fmaf(d1, d1, sq);
            sq = fmaf(d2, d2, sq);
            sq = fmaf(d3, d3, sq);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(tempty + acc);
      if (p.mode == 4 && ref_tile) {
        // publish: every thread's Y stores, then the tile's flag
        __threadfence();
        named_barrier_sync(4, kEpiThreads);
        if (ew == 0 && lane == 0) st_release_gpu(p.ready + tile, 1);
      }
      if (loss_tile) {
        double ds = static_cast<double>(sq);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ds += __shfl_xor_sync(0xffffffffu, ds, o);
        if (lane == 0) red[acc * 4 + ew] = ds;
        named_barrier_sync(2, kEpiThreads);
        if (ew == 0 && lane == 0)
          p.partial[static_cast<int64_t>(lc) * tiles + tile] =
              ((red[acc * 4 + 0] + red[acc * 4 + 1]) + red[acc * 4 + 2]) + red[acc * 4 + 3];
      }
    }
    if (kQdq && ew == 0 && lane == 0) *gemm_done = 1;
    tc_fence_before();
  } else if constexpr (kQdq) {
    if (warp >= 8) {
      // --------------------------------------------------------------- QDQ warps
      // (128 x 32 tile of W, chunk of up to kQdqChunk candidates) pieces, claimed one at a
      // time in column-major order (the column tiles the GEMM reads first are finished
      // first) from a counter that spans the search's launches: the reference launch
      // claims while its own GEMM runs (a claim takes a few microseconds, so the launch
      // outlasts its GEMM by at most that), the candidate launch until none is left. Each
      // piece's stores are published by its column tile's count.
      const int tid = static_cast<int>(threadIdx.x) - kThreads;
      uint8_t* qs = smem + kSmemBytes - 1024;  // past the ring, the barriers and their slack
      float* sWT = reinterpret_cast<float*>(qs);
      float* sS = sWT + kQdqTileCols * QdqTile::kPitch;
      float* sR = sS + kQdqChunk * QdqTile::kSkewPitch;
      float4* sPar = reinterpret_cast<float4*>(sR + kQdqChunk * QdqTile::kSkewPitch);
      uint32_t* sRowsExact = reinterpret_cast<uint32_t*>(sPar + kQdqChunk * kQdqTileCols);
      const int64_t groups = p.qdq_K / 128;
      const int64_t chunks = ceil_div(p.qdq_grid, kQdqChunk);
      const int64_t pieces1 = ceil_div(p.qdq_N, static_cast<int64_t>(kQdqTileCols)) * groups * chunks;
      const int64_t pieces = pieces1 + (p.qdq_W2 ? ceil_div(p.qdq_N2, static_cast<int64_t>(kQdqTileCols)) * groups * chunks : 0);
      int* const next = p.qdq_ready + ceil_div(p.qdq_N, static_cast<int64_t>(kTileN));
      bool skip_publish = p.fault_mode == 3 && blockIdx.x == 0;  // fault injection: one count never arrives
      while (p.qdq_cands) {
        if (tid == 0) *qdq_claim = (p.qdq_cands == 2 && *gemm_done) ? -1 : atomicAdd(next, 1);
        QdqWarpsSync{}();
        const int64_t qq = *qdq_claim;
        if (qq < 0 || qq >= pieces) break;
        // q = (tile, chunk), chunk fastest; tiles in the order of the operand rows they
        // fill (32 rows = 32 columns of W, never straddling a 128-column block), rows major
        const bool first = qq < pieces1;
        const int64_t q = first ? qq : qq - pieces1;
        const int64_t t = q / chunks;
        const int64_t rb = t / groups, k0 = (t - rb * groups) * 128;
        const int c0 = static_cast<int>(q - t * chunks) * kQdqChunk;
        const int c1 = min(c0 + kQdqChunk, p.qdq_grid);
        const int64_t ldw = p.qdq_ldw > 0 ? p.qdq_ldw : p.qdq_N;
        if (first)
          qdq_tile<__nv_bfloat16, 128, QdqTile>(p.qdq_W, p.qdq_K, p.qdq_N, ldw, k0,
                                                qdq_w_column(rb * kQdqTileCols, p.qdq_interleave), p.qdq_S, c0, c1, true,
                                                false, p.qdq_Wt, p.err, p.qdq_quantizer, p.qdq_interleave, sWT, sS, sR,
                                                sPar, sRowsExact, tid, QdqWarpsSync{});
        else
          qdq_tile<__nv_bfloat16, 128, QdqTile>(p.qdq_W2, p.qdq_K, p.qdq_N2, ldw, k0, rb * kQdqTileCols, p.qdq_S, c0, c1,
                                                true, false, p.qdq_Wt2, p.err, p.qdq_quantizer, 0, sWT, sS, sR, sPar,
                                                sRowsExact, tid, QdqWarpsSync{});
        // publish: every thread's stores, then (first operand) the count of the operand
        // tile the rows are in; the second operand is read only by a later launch
        fence_proxy_async_global();
        __threadfence();
        QdqWarpsSync{}();
        if (tid == 0 && first) {
          if (skip_publish)
            skip_publish = false;
          else
            red_release_add_gpu(p.qdq_ready + rb / kQdqColsPerTileN, 1);
        }
      }
    }
  }

  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem_base, kTmemCols);
}

// ---------------------------------------------------------------------------------
// Loss reduction: one block per candidate, fixed summation order (strided per-thread
// sums, then a tree), divided by M*N and rounded once to fp32. The first argmin is
// taken by the pack kernel from these fp32 values.
// ---------------------------------------------------------------------------------
constexpr int kReduceThreads = 256;

__global__ void __launch_bounds__(kReduceThreads)
    loss_reduce_kernel(const double* __restrict__ partial, int64_t tiles, int64_t M, int64_t N,
                       float* __restrict__ losses) {
  __shared__ double buf[kReduceThreads];
  const int c = blockIdx.x;
  const double* row = partial + static_cast<int64_t>(c) * tiles;
  double s = 0.0;
  for (int64_t t = threadIdx.x; t < tiles; t += kReduceThreads) s += row[t];
  buf[threadIdx.x] = s;
  __syncthreads();
  for (int w = kReduceThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) buf[threadIdx.x] += buf[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0)
    losses[c] = __double2float_rn(buf[0] / (static_cast<double>(M) * static_cast<double>(N)));
}

// ---------------------------------------------------------------------------------
// Two-SM variant. A cluster of 2 CTAs (one TPC) computes 256 x 256 output tiles with
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16): each CTA loads its own 128 rows
// of X and 128 of the tile's 256 columns of W_hat (rows of the K-major operand), the
// even CTA issues the MMA over both CTAs' shared memory, and each CTA's tensor memory
// holds its 128 rows of the accumulator. A stage is 32 KB per CTA (16 KB of X, 16 KB of
// W_hat) instead of 48 KB, so 6 stages fit and each SM moves a third less operand data
// per flop. The even CTA owns the stage-full barriers (both CTAs' TMA loads count their
// bytes there) and the accumulator-empty barriers (both CTAs' epilogue warps arrive);
// the MMA's commits are multicast to both CTAs' stage-empty and accumulator-full
// barriers. Output sub-tiles, the Y layout and the partial sums are the 128 x 256 ones
// of the one-SM kernel.
// ---------------------------------------------------------------------------------
constexpr int kPairStages = 6;
constexpr int kPairBBytes = (BN / 2) * BK * 2;         // 16 KB
constexpr int kPairStageBytes = kABytes + kPairBBytes;  // 32 KB
constexpr int kPairSmemBytes = kPairStages * kPairStageBytes + kBarrierBytes + 1024;
constexpr int kGroupPairs = 8;                          // grouped raster: 8 pair rows
constexpr uint64_t kInFlightNs = 1000ull * 1000;        // abort path: let issued copies land

struct PairParams {
  int mode;
  int n_grid;
  int tiles_m, tiles_n, pairs_m;
  int nk;
  float* Y;
  double* partial;
  int* err;
  uint64_t timeout_ns;
  int fault_mode;
};

__device__ __forceinline__ void pair_unit_coords(int64_t u, const PairParams& p, int& c, int& pm, int& nt) {
  const int64_t ptiles = static_cast<int64_t>(p.pairs_m) * p.tiles_n;
  c = static_cast<int>(u / ptiles);
  const int64_t t = u - static_cast<int64_t>(c) * ptiles;
  const int64_t group_size = static_cast<int64_t>(kGroupPairs) * p.tiles_n;
  const int64_t gi = t / group_size;
  const int first = static_cast<int>(gi * kGroupPairs);
  const int gm = min(kGroupPairs, p.pairs_m - first);
  const int64_t r = t - gi * group_size;
  pm = first + static_cast<int>(r % gm);
  nt = static_cast<int>(r / gm);
}

__device__ __forceinline__ void spin_ns(uint64_t ns) {
  const uint64_t t0 = global_timer_ns();
  while (global_timer_ns() - t0 < ns) {
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    loss_gemm_pair_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                          const PairParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kPairStages * kABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kPairStages * kPairStageBytes);
  uint64_t* full = bars;                          // [kPairStages] in rank 0: both CTAs' loads landed
  uint64_t* empty = bars + kPairStages;           // [kPairStages] each CTA: the pair's MMAs read the stage
  uint64_t* tfull = bars + 2 * kPairStages;       // [2] each CTA: accumulator ready
  uint64_t* tempty = bars + 2 * kPairStages + 2;  // [2] in rank 0: both CTAs' epilogues drained it
  uint64_t* drain = bars + 2 * kPairStages + 4;   // [1] rank 0, abort path
  double* red = reinterpret_cast<double*>(bars + 2 * kPairStages + 5);  // [2][4]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kPairStages + 13);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int64_t cid = blockIdx.x >> 1, nclusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(full + s, 2);  // rank 0's expect_tx arrival + rank 1's arrival
      mbar_init(empty + s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull + a, 1);
      mbar_init(tempty + a, 8);  // one arrival per epilogue warp of both CTAs
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapA);
    tma_prefetch_desc(&mapB);
  }
  if (warp == 2) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int64_t tiles = static_cast<int64_t>(p.tiles_m) * p.tiles_n;
  const int64_t n_units = (p.mode == 0 ? 1 : p.n_grid) * static_cast<int64_t>(p.pairs_m) * p.tiles_n;
  const uint64_t budget = p.timeout_ns;
  const uint32_t full0 = mapa_shared(smem_u32(full), 0);      // rank 0's full[0]
  const uint32_t tempty0 = mapa_shared(smem_u32(tempty), 0);  // rank 0's tempty[0]

  auto fail = [&]() {
    *abort_flag = 1;
    atomicOr(p.err, kErrTimeout);
  };

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, issued_any = false;
      for (int64_t u = cid; u < n_units && ok; u += nclusters) {
        int c, pm, nt;
        pair_unit_coords(u, p, c, pm, nt);
        const int slot = p.mode == 0 ? 0 : c + 1;
        const int mt = 2 * pm + static_cast<int>(rank);
        for (int kb = 0; kb < p.nk; ++kb) {
          if (!mbar_wait_bounded(empty + stage, phase ^ 1u, abort_flag, budget)) {
            ok = false;
            break;
          }
          const bool skip = p.fault_mode == 1 && p.mode == 1 && leader && u == cid && kb == 0;
          if (!skip) {
            const uint32_t fbar = full0 + 8u * static_cast<uint32_t>(stage);
            if (leader)
              mbar_arrive_expect_tx(full + stage, 2 * kPairStageBytes);
            else
              mbar_arrive_cluster(fbar);
            tma_load_2d_pair(&mapA, fbar, sA + stage * kABytes, kb * BK, mt * BM);
            tma_load_3d_pair(&mapB, fbar, sB + stage * kPairBBytes, kb * BK, nt * BN + static_cast<int>(rank) * (BN / 2),
                             slot);
            issued_any = true;
          }
          if (++stage == kPairStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        fail();
        if (issued_any) spin_ns(kInFlightNs);  // copies already issued land within microseconds
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer (rank 0)
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = idesc_bf16_f32(2 * BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int local = 0;
      for (int64_t u = cid; u < n_units; u += nclusters, ++local) {
        const int acc = local & 1;
        const uint32_t acc_parity = (local >> 1) & 1;
        if (!mbar_wait_bounded(tempty + acc, acc_parity ^ 1u, abort_flag, budget)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < p.nk; ++kb) {
          if (!mbar_wait_bounded(full + stage, phase, abort_flag, budget)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = smem_desc_k_sw128(smem_u32(sA + stage * kABytes));
          const uint64_t bdesc = smem_desc_k_sw128(smem_u32(sB + stage * kPairBBytes));
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_bf16_f32_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
          umma_commit_pair(empty + stage, 0x3);
          if (++stage == kPairStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair(tfull + acc, 0x3);
      }
      if (!ok) {
        fail();
        umma_commit_pair(drain, 0x1);
        mbar_wait_bounded(drain, 0, nullptr, kDrainNs);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------- epilogue (both CTAs)
    const int ew = warp - 4;  // TMEM lanes 32*ew .. 32*ew+31 = rows of this CTA's half
    const int row = ew * 32 + lane;
    int local = 0;
    for (int64_t u = cid; u < n_units; u += nclusters, ++local) {
      int c, pm, nt;
      pair_unit_coords(u, p, c, pm, nt);
      const int mt = 2 * pm + static_cast<int>(rank);
      const bool valid = mt < p.tiles_m;  // an odd tile count leaves rank 1 of the last pair row empty
      const int acc = local & 1;
      const uint32_t acc_parity = (local >> 1) & 1;
      const bool ok = mbar_wait_bounded(tfull + acc, acc_parity, abort_flag, budget);
      if (named_barrier_or(1, kEpiThreads, !ok)) {
        if (!ok) fail();
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(ew * 32) << 16) + static_cast<uint32_t>(acc * BN);
      const int64_t tile = static_cast<int64_t>(valid ? mt : 0) * p.tiles_n + nt;
      float4* ytile = reinterpret_cast<float4*>(p.Y + tile * (BM * BN));
      float sq = 0.0f;
#pragma unroll 1
      for (int j0 = 0; j0 < BN; j0 += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(j0), v);
        tmem_ld_wait();
        if (!valid) continue;
        float4* yrow = ytile + (j0 / 4) * BM + row;  // tile layout [BN/4][BM][4]
        if (p.mode == 0) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            yrow[q * BM] = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                       __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 y = __ldg(yrow + q * BM);
            const float d0 = __uint_as_float(v[4 * q]) - y.x;
            const float d1 = __uint_as_float(v[4 * q + 1]) - y.y;
            const float d2 = __uint_as_float(v[4 * q + 2]) - y.z;
            const float d3 = __uint_as_float(v[4 * q + 3]) - y.w;
            sq = fmaf(d0, d0, sq);
            sq = fmaf(d1, d1, sq);
            sq = fmaf(d2, d2, sq);
            sq = fmaf(d3, d3, sq);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(tempty + acc);
        else
          mbar_arrive_cluster(tempty0 + 8u * static_cast<uint32_t>(acc));
      }
      if (p.mode == 1) {
        double ds = static_cast<double>(sq);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ds += __shfl_xor_sync(0xffffffffu, ds, o);
        if (lane == 0) red[acc * 4 + ew] = ds;
        named_barrier_sync(2, kEpiThreads);
        if (ew == 0 && lane == 0 && valid)
          p.partial[static_cast<int64_t>(c) * tiles + tile] =
              ((red[acc * 4 + 0] + red[acc * 4 + 1]) + red[acc * 4 + 2]) + red[acc * 4 + 3];
      }
    }
    tc_fence_before();
  }

  __syncthreads();
  cluster_sync_all();  // neither CTA leaves while the other may still touch its barriers or operands
  tc_fence_after();
  if (warp == 2) tmem_dealloc_pair(tmem_base, kTmemCols);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

}  // namespace

cudaError_t make_operand_maps(const LossGemmArgs& a, CUtensorMap* mapA, CUtensorMap* mapB, const char** why,
                              int b_box_rows) {
  auto fn = encode_fn();
  if (!fn) {
    *why = "cuTensorMapEncodeTiled unavailable";
    return cudaErrorNotSupported;
  }
  // A = X_b [M][K]: dims (K, M), box (64, 128), 128-byte swizzle; or a stack of a_slots
  // such operands [a_slots][M][K]: dims (K, M, slots), box (64, 128, 1)
  const cuuint64_t dimsA[3] = {static_cast<cuuint64_t>(a.K), static_cast<cuuint64_t>(a.M),
                               static_cast<cuuint64_t>(a.a_slots)};
  const cuuint64_t strideA[2] = {static_cast<cuuint64_t>(a.K) * 2, static_cast<cuuint64_t>(a.K) * a.M * 2};
  const cuuint32_t boxA[3] = {BK, BM, 1};
  const cuuint32_t ones[3] = {1, 1, 1};
  CUresult r = fn(mapA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.a_slotted ? 3 : 2, const_cast<__nv_bfloat16*>(a.Xb),
                  dimsA, strideA, boxA, ones, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    *why = "tensor map of X";
    return cudaErrorInvalidValue;
  }
  // B = W_hat^T slots [n_grid+1][N][K]: dims (K, N, slots), box (64, 256, 1)
  const cuuint64_t dimsB[3] = {static_cast<cuuint64_t>(a.K), static_cast<cuuint64_t>(a.N),
                               static_cast<cuuint64_t>(a.n_grid + 1)};
  const cuuint64_t strideB[2] = {static_cast<cuuint64_t>(a.K) * 2, static_cast<cuuint64_t>(a.K) * a.N * 2};
  const cuuint32_t boxB[3] = {BK, static_cast<cuuint32_t>(b_box_rows), 1};
  r = fn(mapB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<__nv_bfloat16*>(a.Wt), dimsB, strideB, boxB, ones,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    *why = "tensor map of the candidate weights";
    return cudaErrorInvalidValue;
  }
  return cudaSuccess;
}

cudaError_t launch_loss_gemm(const LossGemmArgs& a, const CUtensorMap& mapA, const CUtensorMap& mapB, int mode,
                             cudaStream_t s, int* launches) {
  const int tiles_m = static_cast<int>(ceil_div(a.M, BM));
  const int tiles_n = static_cast<int>(ceil_div(a.N, BN));
  if (mode == 4 && (a.slot_base != 1 || !a.ready || a.a_slotted || !a.b_per_cand)) return cudaErrorInvalidValue;
  if (a.variant == 2 && mode < 2 && a.slot_base == 1 && !a.a_slotted && a.b_per_cand && a.cands == 0) {
    static unsigned long long attr_done = 0;
    cudaError_t e = set_smem_limit_once(loss_gemm_pair_kernel, kPairSmemBytes, &attr_done);
    if (e != cudaSuccess) return e;
    PairParams p;
    p.mode = mode;
    p.n_grid = a.n_grid;
    p.tiles_m = tiles_m;
    p.tiles_n = tiles_n;
    p.pairs_m = (tiles_m + 1) / 2;
    p.nk = static_cast<int>(ceil_div(a.K, BK));
    p.Y = a.Y;
    p.partial = a.partial;
    p.err = a.err;
    p.timeout_ns = a.timeout_ns;
    p.fault_mode = a.fault_mode;
    const int64_t units = (mode == 0 ? 1 : a.n_grid) * static_cast<int64_t>(p.pairs_m) * tiles_n;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kPairSmemBytes;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int max_clusters = a.num_sms / 2;
    cfg.gridDim = dim3(static_cast<unsigned>(2 * max_clusters));
    int active = 0;
    if (cudaOccupancyMaxActiveClusters(&active, loss_gemm_pair_kernel, &cfg) == cudaSuccess && active > 0)
      max_clusters = std::min(max_clusters, active);
    else
      cudaGetLastError();
    cfg.gridDim = dim3(static_cast<unsigned>(2 * std::min<int64_t>(units, max_clusters)));
    if (getenv("AWQ_DEBUG_LAUNCH"))
      fprintf(stderr, "loss_gemm_pair_kernel: mode %d, %d clusters (occupancy query %d), %lld units\n", mode,
              cfg.gridDim.x / 2, active, static_cast<long long>(units));
    e = cudaLaunchKernelEx(&cfg, loss_gemm_pair_kernel, mapA, mapB, p);
    *launches += 1;
    return e != cudaSuccess ? e : cudaGetLastError();
  }
  const bool qdq = a.qdq_W != nullptr;
  // the launches that read candidate slots (mode 1, mode 3) must read the operand the QDQ
  // warps make, one B slot per candidate
  if (qdq && ((mode != 0 && mode != 1 && mode != 3 && mode != 5) || !a.qdq_ready || !a.qdq_S || !a.qdq_Wt || a.qdq_K % 128 ||
              (a.qdq_W2 && (!a.qdq_Wt2 || a.qdq_N2 % 8 || a.qdq_interleave)) ||
              (a.qdq_ldw && a.qdq_ldw < a.qdq_N + (a.qdq_W2 ? a.qdq_N2 : 0)) ||
              a.qdq_N % 8 || a.qdq_grid < 1 || (a.qdq_interleave && (a.qdq_interleave % 128 || a.qdq_N != 2 * a.qdq_interleave)) ||
              (mode != 0 && (a.qdq_N != a.N || a.qdq_K != a.K || a.qdq_Wt != a.Wt || a.a_slotted || !a.b_per_cand)) ||
              ceil_div(a.qdq_N, static_cast<int64_t>(kQdqTileCols)) * (a.qdq_K / 128) * ceil_div(a.qdq_grid, kQdqChunk) >=
                  (int64_t(1) << 30)))
    return cudaErrorInvalidValue;
  static unsigned long long attr_done = 0, attr_done_qdq = 0;
  cudaError_t e = qdq ? set_smem_limit_once(loss_gemm_kernel<true>, kSmemBytes + kQdqSmemBytes, &attr_done_qdq)
                      : set_smem_limit_once(loss_gemm_kernel<false>, kSmemBytes, &attr_done);
  if (e != cudaSuccess) return e;
  GemmParams p;
  p.mode = mode;
  p.n_grid = a.n_grid;
  p.tiles_m = tiles_m;
  p.tiles_n = tiles_n;
  p.nk = static_cast<int>(ceil_div(a.K, BK));
  p.M = a.M;
  p.N = a.N;
  p.ldo = mode == 3 ? a.N / 2 : a.N;
  p.group_m = raster_group_m(a.K);
  p.H = a.H;
  p.h_stride = a.h_stride;
  p.cands = a.cands > 0 ? a.cands : (mode == 1 ? a.n_grid : 1);
  p.b_per_cand = a.b_per_cand;
  p.a_slotted = a.a_slotted;
  p.a_slot_base = a.a_slot_base;
  p.f16 = a.f16;
  p.slot_base = a.slot_base;
  p.Y = a.Y;
  p.ready = a.ready;
  p.partial = a.partial;
  p.err = a.err;
  p.timeout_ns = a.timeout_ns;
  p.fault_mode = a.fault_mode;
  p.cand_inner = (mode == 1 || mode == 3 || mode == 5) ? a.cand_inner : 0;
  p.qdq_W = a.qdq_W;
  p.qdq_S = a.qdq_S;
  p.qdq_Wt = const_cast<__nv_bfloat16*>(a.qdq_Wt);
  p.qdq_ready = a.qdq_ready;
  p.qdq_cands = a.qdq_cands;
  p.qdq_quantizer = a.qdq_quantizer;
  p.qdq_K = a.qdq_K;
  p.qdq_N = a.qdq_N;
  p.qdq_interleave = a.qdq_interleave;
  p.qdq_grid = a.qdq_grid;
  p.qdq_ldw = a.qdq_ldw;
  p.qdq_W2 = a.qdq_W2;
  p.qdq_Wt2 = a.qdq_Wt2;
  p.qdq_N2 = a.qdq_N2;
  p.K = a.K;
  const int64_t tiles = static_cast<int64_t>(p.tiles_m) * p.tiles_n;
  const int64_t units = (mode == 1 || mode == 3 || mode == 5 ? p.cands : (mode == 4 ? a.n_grid + 1 : 1)) * tiles;
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(units, a.num_sms));
  if (qdq)
    loss_gemm_kernel<true><<<grid, kThreads + kQdqThreads, kSmemBytes + kQdqSmemBytes, s>>>(mapA, mapB, p);
  else
    loss_gemm_kernel<false><<<grid, kThreads, kSmemBytes, s>>>(mapA, mapB, p);
  *launches += 1;
  return cudaGetLastError();
}

cudaError_t launch_loss_reduce(const double* partial, int64_t tiles, int n_grid, int64_t M, int64_t N, float* losses,
                               cudaStream_t s, int* launches) {
  loss_reduce_kernel<<<n_grid, kReduceThreads, 0, s>>>(partial, tiles, M, N, losses);
  *launches += 1;
  return cudaGetLastError();
}

}  // namespace awq
