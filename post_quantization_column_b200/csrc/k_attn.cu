// k_attn.cu — the attention-block objective's module output and its loss ("AWQ：为什么
// 4-bit 权重量化要先观察 Activation" §4: a candidate is scored on the output of the module
// it belongs to, which may be an attention block holding several projections).
//
// For every candidate slot c, sequence b, head h and block of 128 queries i:
//   S = Q K^T over the causal key range (keys 0 .. 128 (i + 1) - 1 of the sequence);
//   m = row max of S (exact, over the whole range); e = exp((S - m) / sqrt(d));
//   l = row sum of e; P = bf16(e); O = (P V) / l;
// and either O is stored (the reference launch, slot 0 = the original weights) or the
// squared difference against the stored reference is summed over the unit and written
// as one fp64 partial (the candidates' launch). O never reaches HBM for a candidate.
//
// Operands (bf16, from the loss GEMM's mode 5): QK [slots][M][2D] row-major (Q in columns
// 0 .. D-1, K in D .. 2D-1) and VT [slots][D][M] (V transposed, so the keys of a head's
// value tile are contiguous, the K-major operand the second product needs). Heads are
// 128 wide; a sequence holds at most 512 tokens, so the scores of a block of queries fit
// the 512 tensor-memory columns of the SM and the row max is taken over all of them
// before any weight is formed (no running-max rescaling).
//
// Blackwell structure (sm_100a): one CTA per SM walks units (c, b, h, i), the longest
// query blocks first. Warp 0 issues TMA loads (128-byte swizzle, no multicast): the query
// tile, then the key tiles and the V^T tiles through a 4-stage ring. Warp 1 issues
// tcgen05.mma (M = 128, N = 128, K = 16, bf16 -> fp32): the score tiles into tensor-memory
// columns 128 j, then O += P_j V_j into columns 0 .. 127 (the first score tile's columns,
// free once its weights are formed). Warps 4-11 (two threads per query row, warp w on
// tensor-memory lanes 32 (w % 4) .., one half of the key columns each) read the scores with
// tcgen05.ld, 64 columns per wait, take the row max over the whole row, form the weights
// (one FMA and one ex2 per score) into shared memory in the swizzled K-major layout the MMA
// reads (two weight buffers, P_j in buffer j % 2 once the MMAs of tile j - 2 are done with
// it), and finish O, with the reference row prefetched into L2 when the unit starts. Every
// wait is bounded by the global timer; a wait that runs out sets the call's timeout bit,
// raises a CTA-wide abort flag and the CTA drains its copies and MMAs before it exits.
#include "awq_device.cuh"
#include "awq_kernels.h"

#include <cudaTypedefs.h>
#include <cmath>
#include <type_traits>

namespace awq {
namespace {

constexpr int kHd = kAttnHeadDim;            // head dimension = rows of the V^T tile
constexpr int kBlk = 128;                    // queries per unit, keys per key tile
constexpr int kAtomBytes = kBlk * 128;       // one 64-column (128-byte) swizzle atom of 128 rows
constexpr int kTileBytes = 2 * kAtomBytes;   // a 128 x 128 bf16 tile
constexpr int kRing = 4;                     // key / V^T tiles in flight
constexpr int kPBufs = 2;                    // weight tiles: P_j in buffer j % 2
constexpr int kSBufs = 3;                    // score tiles in tensor memory, columns 128 b
constexpr uint32_t kOCol = kSBufs * kBlk;    // O in tensor-memory columns 384 .. 511
constexpr int kThreads = 384;                // warps 0-3 roles, warps 4-11 weights and epilogue
constexpr int kEpi = 256;                    // two threads per query row, one per half of the key columns
constexpr int kTmemCols = 512;
constexpr int kSmemBytes = kTileBytes + kRing * kTileBytes + kPBufs * kTileBytes + 512 + 1024 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
static_assert(kOCol + kHd <= kTmemCols, "score buffers and O fit the tensor memory");
constexpr uint64_t kDrainNs = 200ull * 1000 * 1000;

struct AttnParams {
  int n_seq, n_heads, nqt;  // sequences, heads, query blocks per sequence
  int64_t T, M, D;          // tokens per sequence, all tokens, model width (n_heads * 128)
  int slots;                // slots this launch walks
  int slot0;                // stack index of its first slot
  int ref;                  // 1: store O into O_ref; 0: squared error against O_ref
  int rotate;               // gridDim % nqt == 0: rotate the query block of each position per wave
  float* O_ref;             // [M][D] fp32
  double* partial;          // [slots][n_seq * n_heads * nqt]
  int* err;
  uint64_t timeout_ns;
  float score_scale;        // log2(e) / sqrt(head_dim): exp(x / sqrt(d)) = exp2(x * score_scale)
  int fault_mode;           // 1: the producer skips its first ring tile (tests the bounded waits)
};

// Unit u -> (local slot c, sequence b, head h, query block i). The nqt query blocks of one
// (slot, sequence, head) are consecutive units, so a wave of gridDim CTAs works on them at the
// same time and their key and V^T tiles are read from DRAM once; when gridDim % nqt == 0 a
// wave holds whole groups and each position's block is rotated from wave to wave (a
// bijection within each group), so every CTA gets about as many long blocks as short ones.
// (32-bit arithmetic: the launcher keeps the number of units below 2^31.)
__device__ __forceinline__ void unit_coords(int64_t u64, const AttnParams& p, int& c, int& b, int& h, int& i) {
  const uint32_t u = static_cast<uint32_t>(u64), nqt = static_cast<uint32_t>(p.nqt);
  const uint32_t cbh = u / nqt;
  const uint32_t ir = u - cbh * nqt;
  i = static_cast<int>(p.rotate ? (ir + u / gridDim.x) % nqt : ir);
  const uint32_t bh = static_cast<uint32_t>(p.n_seq) * static_cast<uint32_t>(p.n_heads);
  const uint32_t cc = cbh / bh;
  const uint32_t g = cbh - cc * bh;
  c = static_cast<int>(cc);
  b = static_cast<int>(g / static_cast<uint32_t>(p.n_heads));
  h = static_cast<int>(g - static_cast<uint32_t>(b) * static_cast<uint32_t>(p.n_heads));
}

// Shared-memory writes of this thread become visible to the tensor cores (async proxy).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x by the special-function unit (PTX ex2.approx.f32: subnormal results kept, 2^-inf = 0).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// 64 consecutive columns of this thread's tensor-memory row: two loads, one wait.
__device__ __forceinline__ void load_row64(uint32_t taddr, uint32_t (&v)[2][32]) {
  tmem_ld_32x32b_x32(taddr, v[0]);
  tmem_ld_32x32b_x32(taddr + 32u, v[1]);
  tmem_ld_wait_tied(v[0]);
  tmem_ld_wait_tied(v[1]);
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_loss_kernel(const __grid_constant__ CUtensorMap mapQK, const __grid_constant__ CUtensorMap mapVT,
                     const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                              // the query tile
  uint8_t* sRing = sQ + kTileBytes;                // key / V^T tiles
  uint8_t* sP = sRing + kRing * kTileBytes;        // weight tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + kPBufs * kTileBytes);
  uint64_t* q_full = bars;              // the query tile landed
  uint64_t* q_empty = bars + 1;         // the unit's last score MMA is done with it
  uint64_t* kv_full = bars + 2;         // [kRing]
  uint64_t* kv_empty = bars + 6;        // [kRing]
  uint64_t* s_full = bars + 10;         // [kSBufs] a score tile is in tensor memory
  uint64_t* s_free = bars + 13;         // [kSBufs] its 256 readers are done with it
  uint64_t* p_ready = bars + 16;        // [kPBufs] a weight tile written (256 arrivals)
  uint64_t* p_empty = bars + 18;        // [kPBufs] the P V MMAs are done with a weight tile
  uint64_t* o_full = bars + 20;         // O of the unit is in tensor memory
  uint64_t* o_free = bars + 21;         // the epilogue has read O (256 arrivals)
  uint64_t* drain = bars + 22;          // abort path: every issued MMA has completed
  uint64_t* x_ready = bars + 23;        // both halves of every row wrote their normaliser (256)
  uint64_t* r_ready = bars + 24;        // the 8 warps wrote their loss partials (8)
  double* red = reinterpret_cast<double*>(bars + 25);  // [2][8] per-warp loss partials
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(red + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* xl = reinterpret_cast<float*>(sP + kPBufs * kTileBytes + 512);  // [2][128] half-row normalisers

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < kRing; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    for (int s = 0; s < kSBufs; ++s) {
      mbar_init(s_full + s, 1);
      mbar_init(s_free + s, kEpi);
    }
    for (int j = 0; j < kPBufs; ++j) {
      mbar_init(p_ready + j, kEpi);
      mbar_init(p_empty + j, 1);
    }
    mbar_init(o_full, 1);
    mbar_init(o_free, kEpi);
    mbar_init(drain, 1);
    mbar_init(x_ready, kEpi);
    mbar_init(r_ready, kEpi / 32);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapQK);
    tma_prefetch_desc(&mapVT);
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int64_t n_units = static_cast<int64_t>(p.nqt) * p.slots * p.n_seq * p.n_heads;
  const uint64_t budget = p.timeout_ns;
  auto fail = [&]() {
    *abort_flag = 1;
    atomicOr(p.err, kErrTimeout);
  };

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    // Per unit: the query tile, then through the ring in the MMAs' order: the key tiles
    // 0 .. i (pass A), then K_0, and for j = 0 .. i: K_{j+1} (if any), V^T_j (pass B).
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, qphase = 0;
      uint32_t issued = 0, last_parity = 0;  // ring stages with a copy in flight, and its parity
      bool q_issued = false;
      uint32_t q_parity = 0;
      bool ok = true;
      bool fault_pending = p.fault_mode == 1;
      for (int64_t u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        int c, b, h, i;
        unit_coords(u, p, c, b, h, i);
        const int z = p.slot0 + c;
        const int32_t row0 = static_cast<int32_t>(b * p.T);
        if (!mbar_wait_bounded(q_empty, qphase ^ 1u, abort_flag, budget)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(q_full, kTileBytes);
        tma_load_3d(&mapQK, q_full, sQ, h * kHd, row0 + i * kBlk, z);
        tma_load_3d(&mapQK, q_full, sQ + kAtomBytes, h * kHd + 64, row0 + i * kBlk, z);
        q_issued = true;
        q_parity = qphase;
        qphase ^= 1u;
        const int n_tiles = 3 * (i + 1);  // (i + 1) key tiles, the same again, (i + 1) V^T tiles
        for (int t = 0; t < n_tiles && ok; ++t) {
          // tile t of the unit's ring sequence: a key tile (is_v = false) or a V^T tile
          bool is_v;
          int j;
          if (t <= i) {
            is_v = false;
            j = t;
          } else {
            const int r = t - (i + 1);  // pass B: K_0, then (K_1, V_0), (K_2, V_1), ..., V_i
            if (r == 0) {
              is_v = false;
              j = 0;
            } else {
              const int pair = (r - 1) / 2, second = (r - 1) % 2;
              if (pair + 1 <= i && second == 0) {
                is_v = false;
                j = pair + 1;
              } else {
                is_v = true;
                j = pair + 1 <= i ? pair : r - 1 - i;
              }
            }
          }
          if (!mbar_wait_bounded(kv_empty + stage, phase ^ 1u, abort_flag, budget)) {
            ok = false;
            break;
          }
          const bool skip = fault_pending && t == 0;
          if (skip) {
            fault_pending = false;
          } else {
            uint8_t* dst = sRing + stage * kTileBytes;
            mbar_arrive_expect_tx(kv_full + stage, kTileBytes);
            if (!is_v) {  // K_j: columns D + h*128 .., rows of key tile j
              tma_load_3d(&mapQK, kv_full + stage, dst, static_cast<int32_t>(p.D) + h * kHd, row0 + j * kBlk, z);
              tma_load_3d(&mapQK, kv_full + stage, dst + kAtomBytes, static_cast<int32_t>(p.D) + h * kHd + 64,
                          row0 + j * kBlk, z);
            } else {      // V^T_j: rows h*128 .. of V^T, the keys of tile j
              tma_load_3d(&mapVT, kv_full + stage, dst, row0 + j * kBlk, h * kHd, z);
              tma_load_3d(&mapVT, kv_full + stage, dst + kAtomBytes, row0 + j * kBlk + 64, h * kHd, z);
            }
            issued |= 1u << stage;
            last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          }
          if (++stage == kRing) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        fail();
        // let the copies this thread started land before the CTA goes away
        if (q_issued) mbar_wait_bounded(q_full, q_parity, nullptr, kDrainNs);
        for (int s = 0; s < kRing; ++s)
          if (issued & (1u << s)) mbar_wait_bounded(kv_full + s, (last_parity >> s) & 1u, nullptr, kDrainNs);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBlk, kBlk);
      const uint64_t qdesc0 = smem_desc_k_sw128(smem_u32(sQ));
      const uint64_t qdesc1 = smem_desc_k_sw128(smem_u32(sQ + kAtomBytes));
      int stage = 0;
      uint32_t phase = 0;
      uint32_t pready_parity = 0;   // bit b: parity of weight buffer b's next p_ready phase
      uint32_t suse = 0u;  // bit b: parity of the uses of score buffer b so far
      int scount = 0;
      bool ok = true;
      int local = 0;
      // the next ring tile, once landed
      auto ring_wait = [&]() -> bool {
        if (!mbar_wait_bounded(kv_full + stage, phase, abort_flag, budget)) return false;
        tc_fence_after();
        return true;
      };
      auto ring_release = [&]() {
        umma_commit(kv_empty + stage);
        if (++stage == kRing) {
          stage = 0;
          phase ^= 1u;
        }
      };
      // S = Q K^T of the ring's next tile into the next score buffer
      auto score = [&]() -> bool {
        const int sb = scount % kSBufs;
        if (!mbar_wait_bounded(s_free + sb, ((suse >> sb) & 1u) ^ 1u, abort_flag, budget) || !ring_wait()) return false;
        const uint8_t* kt = sRing + stage * kTileBytes;
        const uint64_t kdesc0 = smem_desc_k_sw128(smem_u32(kt)), kdesc1 = smem_desc_k_sw128(smem_u32(kt + kAtomBytes));
#pragma unroll
        for (int k = 0; k < kHd / 16; ++k)  // 16 head dimensions per MMA: 32 bytes = 2 descriptor units
          umma_bf16_f32(tmem_base + static_cast<uint32_t>(sb * kBlk), (k < 4 ? qdesc0 : qdesc1) + 2 * (k & 3),
                        (k < 4 ? kdesc0 : kdesc1) + 2 * (k & 3), idesc, k > 0 ? 1u : 0u);
        ring_release();
        umma_commit(s_full + sb);
        suse ^= 1u << sb;
        ++scount;
        return true;
      };
      for (int64_t u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++local) {
        int c, b, h, i;
        unit_coords(u, p, c, b, h, i);
        const uint32_t up = static_cast<uint32_t>(local & 1);
        if (!mbar_wait_bounded(q_full, up, abort_flag, budget)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // pass A: the score tiles for the row max
        for (int j = 0; j <= i && ok; ++j) ok = score();
        // pass B: the score tiles again, one ahead of the P V product of the previous tile
        if (ok) ok = score();
        if (ok && i == 0) umma_commit(q_empty);
        for (int j = 0; j <= i && ok; ++j) {
          if (j + 1 <= i) {
            ok = score();
            if (ok && j + 1 == i) umma_commit(q_empty);  // the unit's last score MMA
            if (!ok) break;
          }
          const int pb = j & 1;
          // O += P_j V_j into columns 384 .. 511 once P_j is written (and, for the first
          // tile, once the previous unit's epilogue has read O)
          if ((j == 0 && !mbar_wait_bounded(o_free, up ^ 1u, abort_flag, budget)) ||
              !mbar_wait_bounded(p_ready + pb, (pready_parity >> pb) & 1u, abort_flag, budget) || !ring_wait()) {
            ok = false;
            break;
          }
          pready_parity ^= 1u << pb;
          const uint8_t* vt = sRing + stage * kTileBytes;
          const uint8_t* pt = sP + pb * kTileBytes;
          const uint64_t pdesc0 = smem_desc_k_sw128(smem_u32(pt)), pdesc1 = smem_desc_k_sw128(smem_u32(pt + kAtomBytes));
          const uint64_t vdesc0 = smem_desc_k_sw128(smem_u32(vt)), vdesc1 = smem_desc_k_sw128(smem_u32(vt + kAtomBytes));
#pragma unroll
          for (int k = 0; k < kBlk / 16; ++k)  // 16 keys per MMA
            umma_bf16_f32(tmem_base + kOCol, (k < 4 ? pdesc0 : pdesc1) + 2 * (k & 3),
                          (k < 4 ? vdesc0 : vdesc1) + 2 * (k & 3), idesc, (j | k) != 0 ? 1u : 0u);
          ring_release();
          umma_commit(p_empty + pb);
        }
        if (ok) umma_commit(o_full);
      }
      if (!ok) {
        fail();
        umma_commit(drain);
        mbar_wait_bounded(drain, 0, nullptr, kDrainNs);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------- weights and epilogue
    // Warps 4-11: warp w reads tensor-memory lanes 32 (w % 4) .. (its query rows); in pass
    // A it takes the max over the whole row, in pass B the key columns 64 hf .. 64 hf + 63 of
    // every key tile, hf = (w - 4) / 4, which is swizzle atom hf of the weight tile, and in the
    // epilogue O's columns 64 hf ..; the two threads of a row add their normalisers through
    // shared memory.
    const int ew = warp - 4;
    const int quarter = ew & 3, hf = ew >> 2;
    const int row = quarter * 32 + lane;  // query row of the unit = tensor-memory lane
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    const int64_t units_per_slot = static_cast<int64_t>(p.n_seq) * p.n_heads * p.nqt;
    const float2 scale2 = make_float2(p.score_scale, p.score_scale);
    uint32_t pc0 = 0u, pc1 = 0u;          // P V commits to weight buffers 0 and 1 so far (all units)
    uint32_t suse = 0u;  // bit b: parity of the uses of score buffer b so far
    uint32_t rphase = 0u;  // parity of r_ready's next phase (one per candidate unit)
    int scount = 0;
    bool ok = true;
    // Every wait of these warps is bounded and watches the CTA's abort flag, and a warp
    // takes one decision from its lanes' outcomes (a vote, so the warp stays converged for
    // the warp-wide tensor-memory loads): a warp that gives up leaves on its own and the
    // others follow at their next wait; no thread waits on a barrier that cannot time out.
    auto wait_or_fail = [&](uint64_t* bar, uint32_t parity) -> bool {
      const bool w = mbar_wait_bounded(bar, parity, abort_flag, budget);
      if (!w) fail();
      return !__any_sync(0xffffffffu, !w);
    };
    // the next score tile
    auto score_wait = [&](int& sb) -> bool {
      sb = scount % kSBufs;
      if (!wait_or_fail(s_full + sb, (suse >> sb) & 1u)) return false;
      tc_fence_after();
      return true;
    };
    auto score_release = [&](int sb) {
      tc_fence_before();
      mbar_arrive(s_free + sb);
      suse ^= 1u << sb;
      ++scount;
    };
    int local = 0;
    for (int64_t u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++local) {
      int c, b, h, i;
      unit_coords(u, p, c, b, h, i);
      const uint32_t up = static_cast<uint32_t>(local & 1);
      const int64_t grow = static_cast<int64_t>(b) * p.T + static_cast<int64_t>(i) * kBlk + row;
      float* orow = p.O_ref + grow * p.D + static_cast<int64_t>(h) * kHd + 64 * hf;
      if (!p.ref) {  // this thread's half of the reference row, read in the epilogue
        prefetch_l2(orow);
        prefetch_l2(orow + 32);
      }
      // pass A: the row max over the causal key range (keys <= this query), every column
      // of the row (four independent chains; max is exact in any order)
      float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      for (int j = 0; j <= i; ++j) {
        int sb;
        if (!score_wait(sb)) {
          ok = false;
          break;
        }
#pragma unroll 1
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t v[2][32];
          load_row64(tl + static_cast<uint32_t>(sb * kBlk + 64 * h2), v);
          if (j < i) {
#pragma unroll
            for (int q = 0; q < 2; ++q)
#pragma unroll
              for (int e = 0; e < 32; e += 4)
                mq[e / 8 % 4] = fmax3(mq[e / 8 % 4], fmaxf(__uint_as_float(v[q][e]), __uint_as_float(v[q][e + 1])),
                                      fmaxf(__uint_as_float(v[q][e + 2]), __uint_as_float(v[q][e + 3])));
          } else {
            const int lim = row + 1 - 64 * h2;  // diagonal tile: keys <= row
#pragma unroll
            for (int q = 0; q < 2; ++q)
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (32 * q + e < lim) mq[e % 4] = fmaxf(mq[e % 4], __uint_as_float(v[q][e]));
          }
        }
        score_release(sb);
      }
      if (!ok) break;
      const float m = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
      const float2 nms2 = make_float2(-__fmul_rn(m, p.score_scale), -__fmul_rn(m, p.score_scale));
      // pass B: e = 2^(s log2(e) / sqrt(d) - m log2(e) / sqrt(d)) for this thread's half of
      // each recomputed key tile, partial normalisers, and P = bf16(e) into atom hf of the
      // weight tile (16-byte chunk q of a row at position q ^ (row % 8) of its 128-byte
      // line), P_j in buffer j % 2 once the P V MMAs of tile j - 2 are done with it
      float2 lq[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      for (int j = 0; j <= i; ++j) {
        const int pb = j & 1;
        int sb;
        if (!score_wait(sb)) {
          ok = false;
          break;
        }
        uint32_t v[2][32];
        load_row64(tl + static_cast<uint32_t>(sb * kBlk + 64 * hf), v);
        score_release(sb);
        if (j >= 2 && !wait_or_fail(p_empty + pb, ((pb ? pc1 : pc0) - 1u) & 1u)) {
          ok = false;  // buffer pb is free once the P V MMAs of tile j - 2 are done
          break;
        }
        uint8_t* line = sP + pb * kTileBytes + hf * kAtomBytes + row * 128;
        // weights of 32 keys (2 x 16 pairs), masked from key index `lim` on when kMask
        auto weights = [&](auto mask_tag, int q, int lim) {
          constexpr bool kMask = decltype(mask_tag)::value;
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float2 x = __ffma2_rn(make_float2(__uint_as_float(v[q][e]), __uint_as_float(v[q][e + 1])), scale2, nms2);
            if (kMask) {
              if (32 * q + e >= lim) x.x = -INFINITY;
              if (32 * q + e + 1 >= lim) x.y = -INFINITY;
            }
            const float2 ev = make_float2(ex2(x.x), ex2(x.y));
            lq[e / 2 % 4] = __fadd2_rn(lq[e / 2 % 4], ev);
            w[e / 2] = pack_bf16x2(ev.x, ev.y);
          }
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int chunk = q * 4 + r;  // 16-byte chunk of the 128-byte line
            *reinterpret_cast<uint4*>(line + ((chunk ^ (row & 7)) << 4)) =
                make_uint4(w[4 * r], w[4 * r + 1], w[4 * r + 2], w[4 * r + 3]);
          }
        };
        if (j < i) {  // every key of the tile is in range
#pragma unroll
          for (int q = 0; q < 2; ++q) weights(std::false_type{}, q, 0);
        } else {      // the diagonal tile: keys 64 hf + k in range for k <= row - 64 hf
          const int lim = row + 1 - 64 * hf;
#pragma unroll
          for (int q = 0; q < 2; ++q) weights(std::true_type{}, q, lim);
        }
        fence_proxy_async_smem();  // the weights are read by the tensor cores
        mbar_arrive(p_ready + pb);
        if (pb) ++pc1; else ++pc0;  // P V_j commits to p_empty[pb]
      }
      if (!ok) break;
      // the row's normaliser: this half's partials in a fixed order, then half 0 + half 1
      const float lh = ((lq[0].x + lq[0].y) + (lq[1].x + lq[1].y)) + ((lq[2].x + lq[2].y) + (lq[3].x + lq[3].y));
      xl[hf * 128 + row] = lh;
      mbar_arrive(x_ready);
      if (!wait_or_fail(x_ready, up)) {
        ok = false;
        break;
      }
      const float l = __fadd_rn(xl[row], xl[128 + row]);
      // epilogue: O / l for this thread's 64 columns, stored (reference) or compared
      if (!wait_or_fail(o_full, up)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float inv_l = __frcp_rn(l);
      float sq = 0.0f;
      {
        uint32_t v[2][32];
        load_row64(tl + kOCol + static_cast<uint32_t>(64 * hf), v);
        tc_fence_before();
        mbar_arrive(o_free);  // O is in registers: the next unit's P V may overwrite it
        float4 r[16];
        if (!p.ref)
#pragma unroll
          for (int q = 0; q < 16; ++q) r[q] = __ldg(reinterpret_cast<const float4*>(orow) + q);
        float4* o4 = reinterpret_cast<float4*>(orow);
        const float2 il2 = make_float2(inv_l, inv_l);
        float2 sq2 = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const uint32_t* x = &v[q / 8][4 * (q % 8)];
          const float2 o01 = __fmul2_rn(make_float2(__uint_as_float(x[0]), __uint_as_float(x[1])), il2);
          const float2 o23 = __fmul2_rn(make_float2(__uint_as_float(x[2]), __uint_as_float(x[3])), il2);
          if (p.ref) {
            o4[q] = make_float4(o01.x, o01.y, o23.x, o23.y);
          } else {
            const float2 d01 = __fadd2_rn(o01, make_float2(-r[q].x, -r[q].y));
            const float2 d23 = __fadd2_rn(o23, make_float2(-r[q].z, -r[q].w));
            sq2 = __ffma2_rn(d01, d01, sq2);
            sq2 = __ffma2_rn(d23, d23, sq2);
          }
        }
        sq = sq2.x + sq2.y;
      }
      if (!p.ref) {
        double ds = static_cast<double>(sq);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ds += __shfl_xor_sync(0xffffffffu, ds, o);
        if (lane == 0) {
          red[up * 8 + ew] = ds;
          mbar_arrive(r_ready);
        }
        bool rfail = false;
        if (ew == 0 && lane == 0) {  // the unit's partial: the 8 warps' sums in a fixed order
          if (mbar_wait_bounded(r_ready, rphase, abort_flag, budget)) {
            double t = 0.0;
            for (int k = 0; k < 8; ++k) t += red[up * 8 + k];
            p.partial[static_cast<int64_t>(c) * units_per_slot + (static_cast<int64_t>(b) * p.n_heads + h) * p.nqt + i] =
                t;
          } else {
            fail();
            rfail = true;
          }
        }
        rphase ^= 1u;
        if (__any_sync(0xffffffffu, rfail)) {
          ok = false;
          break;
        }
      }
    }
    tc_fence_before();
  }

  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem_base, kTmemCols);
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

cudaError_t launch_attn_loss(const AttnLossArgs& a, int ref, cudaStream_t s, int* launches) {
  if (a.n_heads <= 0 || a.T <= 0 || a.T % kBlk || a.T > kAttnMaxSeq || a.M % a.T ||
      a.D != static_cast<int64_t>(a.n_heads) * kHd || a.slots <= 0)
    return cudaErrorInvalidValue;
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  // QK [slots][M][2D]: dims (2D, M, slots), box (64, 128, 1); VT [slots][D][M]: dims
  // (M, D, slots), box (64, 128, 1); both 128-byte swizzled, as the MMA descriptors expect
  CUtensorMap mQK, mVT;
  const cuuint32_t box[3] = {64, kBlk, 1};
  const cuuint32_t ones[3] = {1, 1, 1};
  const cuuint64_t dqk[3] = {static_cast<cuuint64_t>(2 * a.D), static_cast<cuuint64_t>(a.M),
                             static_cast<cuuint64_t>(a.total_slots)};
  const cuuint64_t sqk[2] = {static_cast<cuuint64_t>(2 * a.D) * 2, static_cast<cuuint64_t>(2 * a.D) * a.M * 2};
  CUresult r = fn(&mQK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<__nv_bfloat16*>(a.QK), dqk, sqk, box, ones,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  const cuuint64_t dvt[3] = {static_cast<cuuint64_t>(a.M), static_cast<cuuint64_t>(a.D),
                             static_cast<cuuint64_t>(a.total_slots)};
  const cuuint64_t svt[2] = {static_cast<cuuint64_t>(a.M) * 2, static_cast<cuuint64_t>(a.M) * a.D * 2};
  r = fn(&mVT, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<__nv_bfloat16*>(a.VT), dvt, svt, box, ones,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;

  static unsigned long long attr_done = 0;
  cudaError_t e = set_smem_limit_once(attn_loss_kernel, kSmemBytes, &attr_done);
  if (e != cudaSuccess) return e;
  AttnParams p;
  p.n_seq = static_cast<int>(a.M / a.T);
  p.n_heads = a.n_heads;
  p.nqt = static_cast<int>(a.T / kBlk);
  p.T = a.T;
  p.M = a.M;
  p.D = a.D;
  p.slots = a.slots;
  p.slot0 = a.slot0;
  p.ref = ref;
  p.O_ref = a.O_ref;
  p.partial = a.partial;
  p.err = a.err;
  p.timeout_ns = a.timeout_ns;
  p.score_scale = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(kHd)));
  p.fault_mode = a.fault_mode;
  const int64_t units = static_cast<int64_t>(p.nqt) * p.slots * p.n_seq * p.n_heads;
  if (units >= (int64_t(1) << 31)) return cudaErrorInvalidValue;  // unit indices are 32-bit in the kernel
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(units, a.num_sms));
  p.rotate = grid % static_cast<unsigned>(p.nqt) == 0 ? 1 : 0;
  attn_loss_kernel<<<grid, kThreads, kSmemBytes, s>>>(mQK, mVT, p);
  *launches += 1;
  return cudaGetLastError();
}

}  // namespace awq
