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

namespace awq {
namespace {

constexpr int kHd = kAttnHeadDim;            // head dimension = rows of the V^T tile
constexpr int kBlk = 128;                    // queries per unit, keys per key tile
static_assert(kAttnMaxSeq / kBlk * kBlk <= 512, "the scores of a unit fit the 512 tensor-memory columns");
constexpr int kAtomBytes = kBlk * 128;       // one 64-column (128-byte) swizzle atom of 128 rows
constexpr int kTileBytes = 2 * kAtomBytes;   // a 128 x 128 bf16 tile
constexpr int kRing = 4;                     // key / V^T tiles in flight
constexpr int kPBufs = 2;                    // weight tiles: P_j in buffer j % 2
constexpr int kThreads = 384;               // warps 0-3 roles, warps 4-11 weights and epilogue
constexpr int kEpi = 256;                   // two threads per query row, one per half of the key columns
constexpr int kTmemCols = 512;
constexpr int kSmemBytes = kTileBytes + kRing * kTileBytes + kPBufs * kTileBytes + 512 + 1024 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
constexpr uint64_t kDrainNs = 200ull * 1000 * 1000;

struct AttnParams {
  int n_seq, n_heads, nqt;  // sequences, heads, query blocks per sequence
  int64_t T, M, D;          // tokens per sequence, all tokens, model width (n_heads * 128)
  int slots;                // slots this launch walks
  int slot0;                // stack index of its first slot
  int ref;                  // 1: store O into O_ref; 0: squared error against O_ref
  float* O_ref;             // [M][D] fp32
  double* partial;          // [slots][n_seq * n_heads * nqt]
  int* err;
  uint64_t timeout_ns;
  float score_scale;        // log2(e) / sqrt(head_dim): exp(x / sqrt(d)) = exp2(x * score_scale)
  int fault_mode;           // 1: the producer skips the first key tile (tests the bounded waits)
};

// Unit u -> (local slot c, sequence b, head h, query block i), the longest blocks (largest
// i) first, so a CTA walking every gridDim-th unit gets about as many of each length as
// any other CTA.
__device__ __forceinline__ void unit_coords(int64_t u, const AttnParams& p, int& c, int& b, int& h, int& i) {
  const int64_t per_class = static_cast<int64_t>(p.slots) * p.n_seq * p.n_heads;
  const int cls = static_cast<int>(u / per_class);
  i = p.nqt - 1 - cls;
  const int64_t r = u - cls * per_class;
  const int64_t bh = static_cast<int64_t>(p.n_seq) * p.n_heads;
  c = static_cast<int>(r / bh);
  const int g = static_cast<int>(r - static_cast<int64_t>(c) * bh);
  b = g / p.n_heads;
  h = g - b * p.n_heads;
}

__device__ __forceinline__ int bar_or(uint32_t id, uint32_t nthreads, int pred) {
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
  uint64_t* q_empty = bars + 1;         // the score MMAs are done with it
  uint64_t* kv_full = bars + 2;         // [kRing]
  uint64_t* kv_empty = bars + 6;        // [kRing]
  uint64_t* s_full = bars + 10;         // every score tile of the unit is in tensor memory
  uint64_t* p_ready = bars + 11;        // [kPBufs] a weight tile written (128 arrivals)
  uint64_t* p_empty = bars + 13;        // [kPBufs] the P V MMAs are done with a weight tile
  uint64_t* o_full = bars + 15;         // O of the unit is in tensor memory
  uint64_t* tmem_free = bars + 16;      // the epilogue has read O (128 arrivals)
  uint64_t* drain = bars + 17;          // abort path: every issued MMA has completed
  double* red = reinterpret_cast<double*>(bars + 18);  // [2][8] per-warp loss partials
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(red + 16);
  float* xl = reinterpret_cast<float*>(sP + kPBufs * kTileBytes + 512);  // [2][128] half-row normalisers
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < kRing; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    mbar_init(s_full, 1);
    for (int j = 0; j < kPBufs; ++j) {
      mbar_init(p_ready + j, kEpi);
      mbar_init(p_empty + j, 1);
    }
    mbar_init(o_full, 1);
    mbar_init(tmem_free, kEpi);
    mbar_init(drain, 1);
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
        // the key tiles 0 .. i, then the V^T tiles 0 .. i, in the order the MMAs consume them
        for (int t = 0; t < 2 * (i + 1) && ok; ++t) {
          const int j = t <= i ? t : t - (i + 1);
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
            if (t <= i) {  // K_j: columns D + h*128 .., rows of key tile j
              tma_load_3d(&mapQK, kv_full + stage, dst, static_cast<int32_t>(p.D) + h * kHd, row0 + j * kBlk, z);
              tma_load_3d(&mapQK, kv_full + stage, dst + kAtomBytes, static_cast<int32_t>(p.D) + h * kHd + 64,
                          row0 + j * kBlk, z);
            } else {       // V^T_j: rows h*128 .. of V^T, the keys of tile j
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
      int stage = 0;
      uint32_t phase = 0, pready_parity = 0;  // bit j: parity of weight buffer j's next p_ready phase
      bool ok = true;
      int local = 0;
      for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x, ++local) {
        int c, b, h, i;
        unit_coords(u, p, c, b, h, i);
        const uint32_t up = static_cast<uint32_t>(local & 1);
        // tensor memory free (the previous unit's epilogue has read O), the query tile in
        if (!mbar_wait_bounded(tmem_free, up ^ 1u, abort_flag, budget) ||
            !mbar_wait_bounded(q_full, up, abort_flag, budget)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t qdesc0 = smem_desc_k_sw128(smem_u32(sQ));
        const uint64_t qdesc1 = smem_desc_k_sw128(smem_u32(sQ + kAtomBytes));
        // scores: S_j = Q K_j^T into columns 128 j
        for (int j = 0; j <= i && ok; ++j) {
          if (!mbar_wait_bounded(kv_full + stage, phase, abort_flag, budget)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint8_t* kt = sRing + stage * kTileBytes;
          const uint64_t kdesc0 = smem_desc_k_sw128(smem_u32(kt)), kdesc1 = smem_desc_k_sw128(smem_u32(kt + kAtomBytes));
#pragma unroll
          for (int k = 0; k < kHd / 16; ++k)  // 16 head dimensions per MMA: 32 bytes = 2 descriptor units
            umma_bf16_f32(tmem_base + static_cast<uint32_t>(j * kBlk), (k < 4 ? qdesc0 : qdesc1) + 2 * (k & 3),
                          (k < 4 ? kdesc0 : kdesc1) + 2 * (k & 3), idesc, k > 0 ? 1u : 0u);
          umma_commit(kv_empty + stage);
          if (++stage == kRing) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(s_full);
        umma_commit(q_empty);
        // O = sum_j P_j V_j into columns 0 .. 127, each P_j once its weights are written
        for (int j = 0; j <= i && ok; ++j) {
          const int pb = j & 1;
          if (!mbar_wait_bounded(kv_full + stage, phase, abort_flag, budget) ||
              !mbar_wait_bounded(p_ready + pb, (pready_parity >> pb) & 1u, abort_flag, budget)) {
            ok = false;
            break;
          }
          pready_parity ^= 1u << pb;
          tc_fence_after();
          const uint8_t* vt = sRing + stage * kTileBytes;
          const uint8_t* pt = sP + pb * kTileBytes;
          const uint64_t pdesc0 = smem_desc_k_sw128(smem_u32(pt)), pdesc1 = smem_desc_k_sw128(smem_u32(pt + kAtomBytes));
          const uint64_t vdesc0 = smem_desc_k_sw128(smem_u32(vt)), vdesc1 = smem_desc_k_sw128(smem_u32(vt + kAtomBytes));
#pragma unroll
          for (int k = 0; k < kBlk / 16; ++k)  // 16 keys per MMA
            umma_bf16_f32(tmem_base, (k < 4 ? pdesc0 : pdesc1) + 2 * (k & 3), (k < 4 ? vdesc0 : vdesc1) + 2 * (k & 3),
                          idesc, (j | k) != 0 ? 1u : 0u);
          umma_commit(kv_empty + stage);
          umma_commit(p_empty + pb);
          if (++stage == kRing) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(o_full);
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
    // Warps 4-11: warp w reads tensor-memory lanes 32 (w % 4) .. (its query rows) and takes
    // the key columns 64 hf .. 64 hf + 63 of every key tile, hf = (w - 4) / 4, which is
    // swizzle atom hf of the weight tile; the two threads of a row share its normaliser
    // through shared memory.
    const int ew = warp - 4;
    const int quarter = ew & 3, hf = ew >> 2;
    const int row = quarter * 32 + lane;  // query row of the unit = tensor-memory lane
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    const int64_t units_per_slot = static_cast<int64_t>(p.n_seq) * p.n_heads * p.nqt;
    const float2 scale2 = make_float2(p.score_scale, p.score_scale);
    uint32_t pc0 = 0u, pc1 = 0u;  // P V commits to weight buffers 0 and 1 so far (all units)
    int local = 0;
    for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x, ++local) {
      int c, b, h, i;
      unit_coords(u, p, c, b, h, i);
      const uint32_t up = static_cast<uint32_t>(local & 1);
      const int64_t grow = static_cast<int64_t>(b) * p.T + static_cast<int64_t>(i) * kBlk + row;
      float* orow = p.O_ref + grow * p.D + static_cast<int64_t>(h) * kHd + 64 * hf;
      if (!p.ref) {  // this thread's half of the reference row, read in the epilogue
        prefetch_l2(orow);
        prefetch_l2(orow + 32);
      }
      bool ok = mbar_wait_bounded(s_full, up, abort_flag, budget);
      if (bar_or(1, kEpi, !ok)) {
        if (!ok) fail();
        break;
      }
      tc_fence_after();
      // pass 1: the row max over the causal key range (keys <= this query), every column
      // of the row (four independent chains; max is exact in any order)
      float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      for (int j = 0; j <= i; ++j) {
#pragma unroll 1
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t v[2][32];
          load_row64(tl + static_cast<uint32_t>(j * kBlk + 64 * h2), v);
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
      }
      const float m = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
      const float ms = __fmul_rn(m, p.score_scale);
      const float2 nms2 = make_float2(-ms, -ms);
      // pass 2: e = 2^(s log2(e) / sqrt(d) - m log2(e) / sqrt(d)) for this thread's half of
      // each key tile, partial normalisers, and P = bf16(e) into atom hf of the weight tile
      // (16-byte chunk q of a row at position q ^ (row % 8) of its 128-byte line), P_j in
      // buffer j % 2 once the P V MMAs of tile j - 2 are done with it
      float2 lq[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      for (int j = 0; j <= i; ++j) {
        const int pb = j & 1;
        uint32_t v[2][32];
        load_row64(tl + static_cast<uint32_t>(j * kBlk + 64 * hf), v);
        if (j >= 2) {  // buffer pb free once the P V MMAs of tile j - 2 are done
          const bool w = mbar_wait_bounded(p_empty + pb, ((pb ? pc1 : pc0) - 1u) & 1u, abort_flag, budget);
          if (bar_or(1, kEpi, !w)) {
            if (!w) fail();
            ok = false;
            break;
          }
        }
        const int lim = j < i ? kBlk : row + 1 - 64 * hf;  // keys 64 hf + k, k < lim, are in range
        uint8_t* line = sP + pb * kTileBytes + hf * kAtomBytes + row * 128;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float2 x = __ffma2_rn(make_float2(__uint_as_float(v[q][e]), __uint_as_float(v[q][e + 1])), scale2, nms2);
            if (32 * q + e >= lim) x.x = -INFINITY;
            if (32 * q + e + 1 >= lim) x.y = -INFINITY;
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
        }
        fence_proxy_async_smem();  // the weights are read by the tensor cores
        tc_fence_before();         // and the score columns of tile j are no longer read
        mbar_arrive(p_ready + pb);
        if (pb) ++pc1; else ++pc0;  // P V_j commits to p_empty[pb]
      }
      if (!ok) break;
      // the row's normaliser: this half's partials in a fixed order, then half 0 + half 1
      const float lh = ((lq[0].x + lq[0].y) + (lq[1].x + lq[1].y)) + ((lq[2].x + lq[2].y) + (lq[3].x + lq[3].y));
      xl[hf * 128 + row] = lh;
      named_barrier_sync(3, kEpi);
      const float l = __fadd_rn(xl[row], xl[128 + row]);
      // epilogue: O / l for this thread's 64 columns, stored (reference) or compared
      ok = mbar_wait_bounded(o_full, up, abort_flag, budget);
      if (bar_or(1, kEpi, !ok)) {
        if (!ok) fail();
        break;
      }
      tc_fence_after();
      const float inv_l = __frcp_rn(l);
      float sq = 0.0f;
      {
        float4 r[16];
        if (!p.ref)
#pragma unroll
          for (int q = 0; q < 16; ++q) r[q] = __ldg(reinterpret_cast<const float4*>(orow) + q);
        uint32_t v[2][32];
        load_row64(tl + static_cast<uint32_t>(64 * hf), v);
        float4* o4 = reinterpret_cast<float4*>(orow);
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const uint32_t* x = &v[q / 8][4 * (q % 8)];
          const float4 o = make_float4(__fmul_rn(__uint_as_float(x[0]), inv_l), __fmul_rn(__uint_as_float(x[1]), inv_l),
                                       __fmul_rn(__uint_as_float(x[2]), inv_l), __fmul_rn(__uint_as_float(x[3]), inv_l));
          if (p.ref) {
            o4[q] = o;
          } else {
            const float d0 = o.x - r[q].x, d1 = o.y - r[q].y, d2 = o.z - r[q].z, d3 = o.w - r[q].w;
            sq = fmaf(d0, d0, sq);
            sq = fmaf(d1, d1, sq);
            sq = fmaf(d2, d2, sq);
            sq = fmaf(d3, d3, sq);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(tmem_free);
      if (!p.ref) {
        double ds = static_cast<double>(sq);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ds += __shfl_xor_sync(0xffffffffu, ds, o);
        if (lane == 0) red[up * 8 + ew] = ds;
        named_barrier_sync(2, kEpi);
        if (ew == 0 && lane == 0) {
          double t = 0.0;
          for (int k = 0; k < 8; ++k) t += red[up * 8 + k];
          p.partial[static_cast<int64_t>(c) * units_per_slot + (static_cast<int64_t>(b) * p.n_heads + h) * p.nqt + i] = t;
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
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(units, a.num_sms));
  attn_loss_kernel<<<grid, kThreads, kSmemBytes, s>>>(mQK, mVT, p);
  *launches += 1;
  return cudaGetLastError();
}

}  // namespace awq
