// k_w4a16.cu — the W4A16 consumer of the packed artifact ("AWQ：为什么 4-bit 权重量化要先
// 观察 Activation" §7: the artifact feeds a W4A16 kernel; §8: 4-bit weights, 16-bit
// activations; "model-quantization / 05 core modules" §5.3 for the int32 packing).
//
// Y = A w16, A the fp16 activations (already divided by the scales, §6), w16[k][n] =
// fp16((q - z) * step) with the artifact's fp16 step and zero; products exact in fp32,
// fp32 accumulation.
//
// The dequantization uses packed fp16 arithmetic: a nibble OR-ed into 0x6400 is the
// half 1024 + q, so (1024 + q) - (1024 + z) = q - z exactly and one fp16 multiply by
// the step rounds the exact product once — the definition, two values per instruction.
// The packing puts columns 8w .. 8w+7 of row k in word (k, w), nibble i = column 8w + i,
// so (word >> 4j) & 0x000F000F holds columns j and j + 4 in its two halves.
//
// gemv_kernel (decode, M <= 16): bound by the stream of codes (0.5 byte per weight +
// 4 bytes of step and zero per group and column). The weights are dequantized in
// registers straight into the B fragments of 16 x 8 x 16 fp16 MMAs whose A operand is
// the tokens (rows beyond M are zero); the MMA adds the exact products in fp32 without
// any fp16 -> fp32 conversion. The tensor work is small; the kernel is bound by the
// weight stream and the dequantization.
//
// dequant_kernel (M > 16): writes w16 transposed (N x K, K contiguous) so the
// tensor-core GEMM (k_loss_gemm.cu, mode 2, fp16 operands) can load it with TMA.
#include "awq_device.cuh"
#include "awq_kernels.h"

namespace awq {
namespace {

constexpr int kGemvThreads = 256;  // 8 warps
constexpr int kGemvCols = 64;      // columns per CTA (8 words)
constexpr int kRing = 8;           // steps each warp keeps in flight (a power of two)
constexpr int kRingPitch = 48;     // bytes per staged row (32 used)
constexpr int kRingStage = 16 * kRingPitch;
constexpr int kRingBytes = (kGemvThreads / 32) * kRing * kRingStage;  // 48 KB
constexpr int kDqThreads = 256;
constexpr int kDqK = 64;           // rows of k per dequant tile
constexpr int kDqN = 64;           // columns per dequant tile

__device__ __forceinline__ __half2 u32_as_half2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }
__device__ __forceinline__ uint32_t half2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }

// Column pairs (j, j + 4) of one group and 8-column word: 1024 + z and the step.
struct DqParams {
  __half2 z1024[4];
  __half2 step[4];
};

__device__ __forceinline__ DqParams load_pair_params(const __half* steps, const __half* zeros, int64_t at) {
  // 8 consecutive fp16 values of each (16-byte aligned: N % 8 == 0)
  const uint4 sv = __ldg(reinterpret_cast<const uint4*>(steps + at));
  const uint4 zv = __ldg(reinterpret_cast<const uint4*>(zeros + at));
  const __half* s = reinterpret_cast<const __half*>(&sv);
  const __half* z = reinterpret_cast<const __half*>(&zv);
  DqParams p;
  const __half k1024 = __float2half_rn(1024.0f);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    p.z1024[j] = __halves2half2(__hadd(z[j], k1024), __hadd(z[j + 4], k1024));  // exact: z is an integer <= 15
    p.step[j] = __halves2half2(s[j], s[j + 4]);
  }
  return p;
}

// The 8 dequantized weights of one word as fp16 pairs (columns j, j + 4).
__device__ __forceinline__ void dequant_word(uint32_t word, const DqParams& p, __half2 (&w)[4]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t biased = ((word >> (4 * j)) & 0x000F000Fu) | 0x64006400u;  // halves 1024 + q
    w[j] = __hmul2(__hsub2(u32_as_half2(biased), p.z1024[j]), p.step[j]);
  }
}

// One 16 x 8 x 16 fp16 MMA with fp32 accumulation. Lane (g, t) = (lane / 4, lane % 4):
// A (16 x 16, row-major) a0 = rows g, cols 2t..2t+1; a1 = rows g + 8; a2, a3 = cols + 8;
// B (16 x 8) b0 = rows 2t..2t+1 of col g, b1 = rows 2t+8..2t+9; D rows g / g + 8, cols 2t..2t+1.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// fp16 pair (w[row r][col], w[row r + 1][col]) of the lane's column: `sel` moves the
// byte holding its nibble from each row's word into bytes 0 and 2, `sh` (0 or 4) brings
// the nibble down, and OR-ing 0x6400 makes the halves 1024 + q.
__device__ __forceinline__ uint32_t dq_pair(uint32_t wlo, uint32_t whi, uint32_t sel, uint32_t sh, __half2 z1024,
                                            __half2 step) {
  const uint32_t both = __byte_perm(wlo, whi, sel) >> sh;
  const uint32_t biased = (both & 0x000F000Fu) | 0x64006400u;
  return half2_as_u32(__hmul2(__hsub2(u32_as_half2(biased), z1024), step));
}

// CTA: 64 columns (8 words) x one split of K (whole groups); warp w takes a contiguous
// run of the split's 16-row steps. Per step a lane loads the 8 words of rows 2t, 2t+1,
// 2t+8, 2t+9 (32 contiguous bytes each), builds the B fragments of the 8 column tiles
// from its own nibble (column 8 j + g of word j) and runs 8 MMAs against the tokens
// (A rows, zero beyond M). The warps' sums are combined in shared memory in a fixed
// order and the splits by a second launch.
template <int G>
__global__ void __launch_bounds__(kGemvThreads)
    gemv_kernel(const __half* __restrict__ A, int M, const int32_t* __restrict__ codes,
                const __half* __restrict__ steps, const __half* __restrict__ zeros, int64_t K, int64_t N,
                int64_t k_per_split, float* __restrict__ out) {
  __shared__ float red[kGemvThreads / 32][16][kGemvCols];
  extern __shared__ __align__(16) uint8_t gemv_ring[];  // [warp][kRing][16 rows x kRingPitch]

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int gq = lane >> 2, tq = lane & 3;
  const int64_t words = N / 8;
  const int64_t wc0 = static_cast<int64_t>(blockIdx.x) * (kGemvCols / 8);
  const int nw = static_cast<int>(min(static_cast<int64_t>(kGemvCols / 8), words - wc0));  // valid words of the tile
  const bool vec = nw == kGemvCols / 8 && (words % 4) == 0;                  // 16-byte row segments
  const int64_t k0 = static_cast<int64_t>(blockIdx.y) * k_per_split;
  const int64_t k1 = min(K, k0 + k_per_split);
  const int n_steps = static_cast<int>((k1 - k0) / 16);
  const int per_warp = (n_steps + kGemvThreads / 32 - 1) / (kGemvThreads / 32);
  const int s0 = warp * per_warp, s1 = min(n_steps, s0 + per_warp);
  const uint32_t byte = static_cast<uint32_t>(gq >> 1);
  const uint32_t sel = byte | ((byte + 4u) << 8);  // result byte 0 <- wlo.byte, byte 2 <- whi.byte
  const uint32_t sh = 4u * static_cast<uint32_t>(gq & 1);

  float acc[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;

  int64_t cur_group = -1;
  __half2 z2[8], st2[8];
  const __half k1024 = __float2half_rn(1024.0f);
  auto step_compute = [&](int64_t kb, const uint32_t (&wr)[4][8]) {
    const int64_t grp = kb / G;
    if (grp != cur_group) {
      cur_group = grp;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        __half st = __float2half_rn(0.0f), zr = __float2half_rn(0.0f);
        if (j < nw) {
          const int64_t at = grp * N + (wc0 + j) * 8 + gq;
          st = steps[at];
          zr = zeros[at];
        }
        st2[j] = __halves2half2(st, st);
        const __half zb = __hadd(zr, k1024);  // exact: z is an integer <= 15
        z2[j] = __halves2half2(zb, zb);
      }
    }
    // activations: tokens g and g + 8, k pairs 2t and 2t + 8
    uint32_t a0 = 0, a1 = 0, a2 = 0, a3 = 0;
    if (gq < M) {
      const __half* ar = A + static_cast<int64_t>(gq) * K + kb + 2 * tq;
      a0 = __ldg(reinterpret_cast<const uint32_t*>(ar));
      a2 = __ldg(reinterpret_cast<const uint32_t*>(ar + 8));
    }
    if (gq + 8 < M) {
      const __half* ar = A + static_cast<int64_t>(gq + 8) * K + kb + 2 * tq;
      a1 = __ldg(reinterpret_cast<const uint32_t*>(ar));
      a3 = __ldg(reinterpret_cast<const uint32_t*>(ar + 8));
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t b0 = dq_pair(wr[0][j], wr[1][j], sel, sh, z2[j], st2[j]);
      const uint32_t b1 = dq_pair(wr[2][j], wr[3][j], sel, sh, z2[j], st2[j]);
      mma_f16_16816(acc[j], a0, a1, a2, a3, b0, b1);
    }
  };
  const int rows[4] = {2 * tq, 2 * tq + 1, 2 * tq + 8, 2 * tq + 9};

  if (vec) {
    // Each warp streams its steps through a ring of kRing stages in shared memory: lane l
    // copies 16 bytes (row l / 2, half l % 2) of every step with cp.async, kRing - 1
    // steps ahead of the one it computes. Rows sit 48 bytes apart, so the four rows a
    // 16-byte read touches (2t, 2t+2, ...) fall in different banks.
    uint8_t* ring = gemv_ring + warp * (kRing * kRingStage);
    const int crow = lane >> 1, chalf = lane & 1;
    auto issue = [&](int s, int stage) {
      if (s < s1) {
        const int32_t* src = codes + (k0 + 16 * static_cast<int64_t>(s) + crow) * words + wc0 + 4 * chalf;
        const uint32_t dst = smem_u32(ring + stage * kRingStage + crow * kRingPitch + chalf * 16);
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
#pragma unroll
    for (int p = 0; p < kRing - 1; ++p) issue(s0 + p, p);
    int fill = kRing - 1, read = 0;  // ring stages being filled and read
    for (int s = s0; s < s1; ++s) {
      issue(s + kRing - 1, fill);
      fill = (fill + 1) & (kRing - 1);
      asm volatile("cp.async.wait_group %0;" ::"n"(kRing - 1) : "memory");
      __syncwarp();
      const uint8_t* st = ring + read * kRingStage;
      read = (read + 1) & (kRing - 1);
      uint32_t wr[4][8];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const uint4 v0 = *reinterpret_cast<const uint4*>(st + rows[r] * kRingPitch);
        const uint4 v1 = *reinterpret_cast<const uint4*>(st + rows[r] * kRingPitch + 16);
        wr[r][0] = v0.x; wr[r][1] = v0.y; wr[r][2] = v0.z; wr[r][3] = v0.w;
        wr[r][4] = v1.x; wr[r][5] = v1.y; wr[r][6] = v1.z; wr[r][7] = v1.w;
      }
      __syncwarp();  // every lane has read the stage before it is refilled
      step_compute(k0 + 16 * static_cast<int64_t>(s), wr);
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
  } else {
    for (int s = s0; s < s1; ++s) {
      const int64_t kb = k0 + 16 * static_cast<int64_t>(s);
      uint32_t wr[4][8];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int32_t* src = codes + (kb + rows[r]) * words + wc0;
#pragma unroll
        for (int j = 0; j < 8; ++j) wr[r][j] = j < nw ? static_cast<uint32_t>(__ldcs(src + j)) : 0u;
      }
      step_compute(kb, wr);
    }
  }
  // D of tile j: tokens g (acc 0, 1) and g + 8 (acc 2, 3), columns 8 j + 2 t, + 1
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    red[warp][gq][8 * j + 2 * tq] = acc[j][0];
    red[warp][gq][8 * j + 2 * tq + 1] = acc[j][1];
    red[warp][gq + 8][8 * j + 2 * tq] = acc[j][2];
    red[warp][gq + 8][8 * j + 2 * tq + 1] = acc[j][3];
  }
  __syncthreads();
  const int64_t col0 = wc0 * 8;
  for (int i = threadIdx.x; i < M * kGemvCols; i += kGemvThreads) {
    const int m = i / kGemvCols, c = i % kGemvCols;
    if (c >= nw * 8) continue;
    float sum = red[0][m][c];
#pragma unroll
    for (int q = 1; q < kGemvThreads / 32; ++q) sum = __fadd_rn(sum, red[q][m][c]);
    out[(static_cast<int64_t>(blockIdx.y) * M + m) * N + col0 + c] = sum;
  }
}

// Y[m][n] = sum over splits, in split order.
__global__ void split_sum_kernel(const float* __restrict__ part, int splits, int64_t MN, float* __restrict__ Y) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < MN;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float s = part[i];
    for (int q = 1; q < splits; ++q) s = __fadd_rn(s, part[static_cast<int64_t>(q) * MN + i]);
    Y[i] = s;
  }
}

// One 64 (k) x 64 (n) tile: codes -> fp16 weights in shared memory (transposed) ->
// 128-byte rows of Wt[n][k0 .. k0 + 63].
__global__ void __launch_bounds__(kDqThreads)
    dequant_kernel(const int32_t* __restrict__ codes, const __half* __restrict__ steps,
                   const __half* __restrict__ zeros, int64_t K, int64_t N, int group, __half* __restrict__ Wt) {
  constexpr int kPitch = kDqK + 8;  // halves; 16-byte aligned rows, staggered banks
  __shared__ __align__(16) __half T[kDqN][kPitch];
  const int64_t k0 = static_cast<int64_t>(blockIdx.y) * kDqK;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kDqN;
  const int64_t words = N / 8;
  // word (k, w): thread t takes k = t % 64 and words t / 64, t / 64 + 4 (8 words per tile row)
  const int kk = threadIdx.x % kDqK;
#pragma unroll
  for (int it = 0; it < 2; ++it) {
    const int ww = threadIdx.x / kDqK + 4 * it;
    const int64_t wcol = n0 / 8 + ww;
    __half2 wv[4];
    if (wcol < words && k0 + kk < K) {
      const int64_t k = k0 + kk;
      const DqParams pp = load_pair_params(steps, zeros, (k / group) * N + 8 * wcol);
      dequant_word(static_cast<uint32_t>(__ldg(codes + k * words + wcol)), pp, wv);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) wv[j] = __float2half2_rn(0.0f);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      T[8 * ww + j][kk] = __low2half(wv[j]);
      T[8 * ww + j + 4][kk] = __high2half(wv[j]);
    }
  }
  __syncthreads();
  // 64 rows of 64 halves = 8 vectors of 16 bytes per row
  for (int i = threadIdx.x; i < kDqN * 8; i += kDqThreads) {
    const int r = i / 8, v = i % 8;
    const int64_t n = n0 + r;
    if (n < N && k0 + 8 * v < K)  // K % 32 == 0: a vector of 8 rows lies wholly inside or outside
      *reinterpret_cast<uint4*>(Wt + n * K + k0 + 8 * v) = *reinterpret_cast<const uint4*>(&T[r][8 * v]);
  }
}

// ---- the consumer's repacked layout ---------------------------------------------------
// For decode the weights are the A operand of 16 x 8 x 16 MMAs (16 output columns by 16
// rows of K per MMA) and the codes are read in fragment order: for every 16-row step s,
// 64-column block cb and lane (g, t), 16 bytes (4 words) hold the lane's 32 nibbles.
// Word u serves the 16 columns 16u .. 16u + 15; its nibbles p and p + 4 (p = 0..3) are
// rows (r, r + 1) of column 16u + g + 8 (p & 1), r = 2t + 8 (p >> 1) — fragment register
// a_p. Pairs 0 and 1 sit in bits 0-7 of each half of the word, pairs 2 and 3 in bits
// 8-15, and a warp reads 512 contiguous bytes per step.
__global__ void repack_kernel(const int32_t* __restrict__ codes, int64_t K, int64_t N, uint32_t* __restrict__ P) {
  const int64_t words = N / 8, cbs = N / 64;
  const int64_t total = (K / 16) * cbs * 32 * 4;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int u = static_cast<int>(i % 4);
    const int lane = static_cast<int>((i / 4) % 32);
    const int64_t cb = (i / 128) % cbs, s = i / (128 * cbs);
    const int g = lane >> 2, t = lane & 3;
    uint32_t out = 0;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int64_t w = cb * 8 + 2 * u + (p & 1);  // column 16u + g + 8 (p & 1) is nibble g of this word
      const int64_t row = 16 * s + 2 * t + 8 * (p >> 1);
      const uint32_t lo = (static_cast<uint32_t>(__ldg(codes + row * words + w)) >> (4 * g)) & 0xFu;
      const uint32_t hi = (static_cast<uint32_t>(__ldg(codes + (row + 1) * words + w)) >> (4 * g)) & 0xFu;
      out |= (lo << (4 * p)) | (hi << (4 * (p + 4)));
    }
    P[i] = out;
  }
}

// The decode GEMV on the repacked codes, as a persistent stream. The work is the list of
// chunks (64-column block cb, group g), cb-major, split into equal contiguous runs, one
// per warp of a grid sized to the SMs: every warp streams the same number of weights (to
// one chunk), whatever the layer's shape, so no wave is left partly empty. A warp's run
// crosses column blocks: it keeps one accumulator set, and when its run leaves a block
// (or ends) it writes its partial sums to that block's slot for this warp, the block's
// "piece". A second launch adds each block's pieces in warp order (fixed order,
// deterministic).
//
// Per 16-row step a lane copies its 16 bytes (the repacked layout) into a per-warp ring
// of kPRing stages in shared memory (cp.async, kPRing - 1 steps ahead, continuing across
// chunks and blocks); a chunk's 64 steps and 64 zeros travel in the same ring with its
// first step. Each fp16 pair of the B fragments costs one logic op (plus one shift per
// two pairs, on the multiply pipe) before an exact packed q - z and the multiply by the
// step.
constexpr int kPRing = 8;                           // steps in flight per warp (a power of two)
constexpr int kSActBytes = 32 * 1024;               // the activations are staged when M K halves fit
constexpr int kPRingBytes = kPRing * 32 * 16;       // 4 KB of codes per warp
// Parameter buffers per warp: a chunk's steps and zeros are copied with its first step,
// up to kPRing - 1 steps before that step is computed, and must outlive the whole chunk,
// so PB * S > kPRing + S - 2 for S = G / 16 steps per chunk: 8, 4 and 2 for G = 32, 64, 128.
template <int G>
struct PackedSmem {
  static constexpr int S = G / 16;
  static constexpr int PB = G == 32 ? 8 : (G == 64 ? 4 : 2);
  static_assert(PB * S > kPRing + S - 2, "parameter buffers must outlive their chunk");
  static constexpr int kParamBytes = PB * 2 * 64 * 2;  // PB chunks of 64 steps + 64 zeros (fp16)
  static constexpr int kWarpBytes = kPRingBytes + kParamBytes;
  static constexpr int kSmem = (kGemvThreads / 32) * kWarpBytes;
};

// The warp whose run holds chunk l when T chunks are split over W warps (warp w starts at
// floor(w T / W)): the last warp whose start is <= l.
__host__ __device__ __forceinline__ int64_t chunk_owner(int64_t l, int64_t T, int64_t W) {
  return ((l + 1) * W - 1) / T;
}

template <int G, int NT>
__global__ void __launch_bounds__(kGemvThreads, NT == 1 ? 3 : 2)
    gemv_stream_kernel(const __half* __restrict__ A, int M, const uint4* __restrict__ P,
                       const __half* __restrict__ steps, const __half* __restrict__ zeros, int64_t K, int64_t N,
                       int64_t W, int pieces, float* __restrict__ part) {
  constexpr int S = G / 16;
  using PS = PackedSmem<G>;
  extern __shared__ __align__(16) uint8_t pdyn[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int gq = lane >> 2, tq = lane & 3;
  const int64_t cbs = N / 64, Gk = K / G, T = cbs * Gk;
  const int64_t wg = static_cast<int64_t>(blockIdx.x) * (kGemvThreads / 32) + warp;

  // the activations, staged once per CTA when they fit (M K halves)
  __half* sAct = reinterpret_cast<__half*>(pdyn + PS::kSmem);
  const bool staged = static_cast<int64_t>(M) * K * 2 <= kSActBytes;
  if (staged) {
    const int64_t vecs = static_cast<int64_t>(M) * K / 8;
    for (int64_t i = threadIdx.x; i < vecs; i += kGemvThreads)
      reinterpret_cast<uint4*>(sAct)[i] = __ldg(reinterpret_cast<const uint4*>(A) + i);
    __syncthreads();
  }
  if (wg >= W) return;  // W <= T: every warp below W has at least one chunk
  const int64_t l0 = wg * T / W, l1 = (wg + 1) * T / W;
  uint8_t* ring = pdyn + warp * PS::kWarpBytes;
  __half* params = reinterpret_cast<__half*>(ring + kPRingBytes);  // [PB][2][64]

  // ---- issue side: kPRing - 1 steps ahead of the compute side
  int64_t i_cb = l0 / Gk, i_g = l0 % Gk, i_l = l0;
  const uint4* i_ptr = P + (i_g * S * cbs + i_cb) * 32 + lane;
  // issue(ssi): the step at position ssi of its chunk (ssi is a constant once unrolled)
  auto issue = [&](int ssi) {
    if (i_l < l1) {
      const uint32_t dst = smem_u32(ring + ((i_l * S + ssi) & (kPRing - 1)) * 512 + lane * 16);
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(i_ptr) : "memory");
      if (ssi == 0 && lane < 16) {
        const __half* src = (lane < 8 ? steps : zeros) + i_g * N + i_cb * 64 + 8 * (lane & 7);
        const uint32_t pd = smem_u32(params + (i_l & (PS::PB - 1)) * 128 + (lane < 8 ? 0 : 64) + 8 * (lane & 7));
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(pd), "l"(src) : "memory");
      }
      i_ptr += cbs * 32;
      if (ssi == S - 1) {  // next chunk
        ++i_l;
        if (++i_g == Gk) {
          i_g = 0;
          ++i_cb;
          i_ptr = P + i_cb * 32 + lane;
        }
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
#pragma unroll
  for (int q = 0; q < kPRing - 1; ++q) issue(q % S);

  // ---- compute side: acc[i][u] is the 16 x 8 tile of columns 16u .. and tokens 8i ..
  float acc[NT][4][4];
#pragma unroll
  for (int i = 0; i < NT; ++i)
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[i][u][0] = acc[i][u][1] = acc[i][u][2] = acc[i][u][3] = 0.0f;
  const __half k1024 = __float2half_rn(1024.0f), k64 = __float2half_rn(64.0f);
  const __half2 sixteenth = __float2half2_rn(0.0625f);
  const __half* sArow0 = sAct + static_cast<int64_t>(gq) * K + 2 * tq;      // staged row of token g
  const __half* sArow1 = sArow0 + 8 * K;                                     // and of token g + 8
  const __half* gArow0 = A + static_cast<int64_t>(gq) * K + 2 * tq;
  const __half* gArow1 = gArow0 + 8 * K;
  int64_t c_cb = l0 / Gk, c_g = l0 % Gk;
#pragma unroll 1
  for (int64_t l = l0; l < l1; ++l) {
    // per word u: column 16u + g (even pairs: 1024 + z, step) and 16u + g + 8 (odd pairs:
    // -(64 + z), step)
    __half2 z2[4], zn2[4], st2[8];
#pragma unroll
    for (int ss = 0; ss < S; ++ss) {
      issue((ss + kPRing - 1) % S);
      asm volatile("cp.async.wait_group %0;" ::"n"(kPRing - 1) : "memory");
      __syncwarp();  // the chunk's steps and zeros were copied by other lanes
      if (ss == 0) {
        const __half* pr = params + (l & (PS::PB - 1)) * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) {  // column 8j + g of the block
          const __half st = pr[8 * j + gq];
          const __half z = pr[64 + 8 * j + gq];
          st2[j] = __halves2half2(st, st);
          if (j % 2 == 0) {
            const __half zb = __hadd(z, k1024);  // 1024 + z, exact: z is an integer <= 15
            z2[j / 2] = __halves2half2(zb, zb);
          } else {
            const __half zn = __hneg(__hadd(z, k64));  // -(64 + z), exact
            zn2[j / 2] = __halves2half2(zn, zn);
          }
        }
      }
      const uint4 v = *reinterpret_cast<const uint4*>(ring + ((l * S + ss) & (kPRing - 1)) * 512 + lane * 16);
      const int64_t kk = (c_g * S + ss) * 16;  // row of the step
      // B fragments: tokens g (and g + 8), rows 2t, 2t + 1 and 2t + 8, 2t + 9 of the step
      uint32_t b0 = 0, b1 = 0, b2 = 0, b3 = 0;
      if (staged) {
        if (gq < M) {
          b0 = *reinterpret_cast<const uint32_t*>(sArow0 + kk);
          b1 = *reinterpret_cast<const uint32_t*>(sArow0 + kk + 8);
        }
        if (NT == 2 && gq + 8 < M) {
          b2 = *reinterpret_cast<const uint32_t*>(sArow1 + kk);
          b3 = *reinterpret_cast<const uint32_t*>(sArow1 + kk + 8);
        }
      } else {
        if (gq < M) {
          b0 = __ldg(reinterpret_cast<const uint32_t*>(gArow0 + kk));
          b1 = __ldg(reinterpret_cast<const uint32_t*>(gArow0 + kk + 8));
        }
        if (NT == 2 && gq + 8 < M) {
          b2 = __ldg(reinterpret_cast<const uint32_t*>(gArow1 + kk));
          b3 = __ldg(reinterpret_cast<const uint32_t*>(gArow1 + kk + 8));
        }
      }
      const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        // pairs 0, 1 in bits 0-7 of each half, pairs 2, 3 after a shift by 8 (taken on the
        // multiply pipe as the high word of w * 2^24). Even pair: halves 1024 + q minus
        // (1024 + z); odd pair: halves 1024 + 16 q times 1/16 minus (64 + z) in one fused
        // step (every value exact); then times the step.
        const uint32_t w8 = __umulhi(wv[u], 1u << 24);
        uint32_t a[4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t src = h ? w8 : wv[u];
          const uint32_t lo = (src & 0x000F000Fu) | 0x64006400u;
          const uint32_t hi = (src & 0x00F000F0u) | 0x64006400u;
          a[2 * h] = half2_as_u32(__hmul2(__hsub2(u32_as_half2(lo), z2[u]), st2[2 * u]));
          a[2 * h + 1] = half2_as_u32(__hmul2(__hfma2(u32_as_half2(hi), sixteenth, zn2[u]), st2[2 * u + 1]));
        }
        mma_f16_16816(acc[0][u], a[0], a[1], a[2], a[3], b0, b1);
        if (NT == 2) mma_f16_16816(acc[NT - 1][u], a[0], a[1], a[2], a[3], b2, b3);
      }
    }
    // the chunk is done: leave the column block at its end or at the end of the run
    if (++c_g == Gk || l + 1 == l1) {
      const int64_t piece = wg - chunk_owner(c_cb * Gk, T, W);
      float* dst = part + (c_cb * pieces + piece) * static_cast<int64_t>(M) * 64;
#pragma unroll
      for (int i = 0; i < NT; ++i)
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          // D rows are columns 16u + g (+ 8), D columns are tokens 8i + 2t (+ 1)
          const int m0 = 8 * i + 2 * tq, n0 = 16 * u + gq;
          if (m0 < M) {
            dst[m0 * 64 + n0] = acc[i][u][0];
            dst[m0 * 64 + n0 + 8] = acc[i][u][2];
          }
          if (m0 + 1 < M) {
            dst[(m0 + 1) * 64 + n0] = acc[i][u][1];
            dst[(m0 + 1) * 64 + n0 + 8] = acc[i][u][3];
          }
          acc[i][u][0] = acc[i][u][1] = acc[i][u][2] = acc[i][u][3] = 0.0f;
        }
      c_g = 0;
      ++c_cb;
    }
    __syncwarp();  // all lanes are past this chunk's parameters before a later chunk overwrites them
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// Y[m][n] = the sum of column block n / 64's pieces, in warp order.
__global__ void piece_sum_kernel(const float* __restrict__ part, int pieces, int M, int64_t N, int64_t Gk, int64_t W,
                                 float* __restrict__ Y) {
  const int64_t MN = static_cast<int64_t>(M) * N, T = (N / 64) * Gk;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < MN;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = i / N, n = i % N, cb = n / 64;
    const int64_t count = chunk_owner(cb * Gk + Gk - 1, T, W) - chunk_owner(cb * Gk, T, W) + 1;
    const float* src = part + (cb * pieces * M + m) * 64 + n % 64;
    const int64_t stride = static_cast<int64_t>(M) * 64;  // one piece
    float s = src[0];
    // eight loads in flight at a time, the additions still in piece order
    for (int64_t q0 = 1; q0 < count; q0 += 8) {
      float v[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) v[k] = q0 + k < count ? src[(q0 + k) * stride] : 0.0f;
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (q0 + k < count) s = __fadd_rn(s, v[k]);
    }
    Y[i] = s;
  }
}

// Splits of whole groups so that the grid fills the SMs a few times over.
int64_t gemv_splits(int64_t K, int64_t N, int group, int num_sms) {
  const int64_t col_blocks = ceil_div(N, kGemvCols);
  const int64_t groups = K / group;
  int64_t splits = std::max<int64_t>(1, std::min<int64_t>(groups, ceil_div(8 * num_sms, col_blocks)));
  const int64_t gps = ceil_div(groups, splits);
  return ceil_div(groups, gps);
}

template <int G>
cudaError_t launch_gemv_g(const W4A16Args& a, int num_sms, float* part, cudaStream_t s, int* launches) {
  const int64_t col_blocks = ceil_div(a.N, kGemvCols);
  const int64_t splits = gemv_splits(a.K, a.N, G, num_sms);
  const int64_t k_per_split = ceil_div(a.K / G, splits) * G;
  float* dst = splits == 1 ? a.Y : part;
  static unsigned long long done = 0;
  cudaError_t e0 = set_smem_limit_once(gemv_kernel<G>, kRingBytes, &done);
  if (e0 != cudaSuccess) return e0;
  gemv_kernel<G><<<dim3(static_cast<unsigned>(col_blocks), static_cast<unsigned>(splits)), kGemvThreads, kRingBytes,
                   s>>>(
      a.A, static_cast<int>(a.M), a.codes, a.steps, a.zeros, a.K, a.N, k_per_split, dst);
  *launches += 1;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || splits == 1) return e;
  const int64_t mn = a.M * a.N;
  const unsigned blocks = static_cast<unsigned>(std::min<int64_t>(ceil_div(mn, 256), 4 * num_sms));
  split_sum_kernel<<<blocks, 256, 0, s>>>(part, static_cast<int>(splits), mn, a.Y);
  *launches += 1;
  return cudaGetLastError();
}

template <int G>
int stream_smem(int64_t M, int64_t K) {
  return PackedSmem<G>::kSmem + (M * K * 2 <= kSActBytes ? static_cast<int>(M * K * 2) : 0);
}

// Resident CTAs per SM of a decode variant (queried once, at the largest shared-memory
// size the launcher uses).
template <int G, int NT>
int stream_ctas_per_sm() {
  static const int per_sm = [] {
    static unsigned long long done = 0;
    int n = 0;
    if (set_smem_limit_once(gemv_stream_kernel<G, NT>, PackedSmem<G>::kSmem + kSActBytes, &done) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, gemv_stream_kernel<G, NT>, kGemvThreads,
                                                      PackedSmem<G>::kSmem + kSActBytes) != cudaSuccess) {
      cudaGetLastError();
      n = 1;
    }
    return std::max(n, 1);
  }();
  return per_sm;
}

// Warps of the streaming decode: as many CTAs of 8 warps as the SMs hold at once, and
// never more warps than chunks.
template <int G>
int64_t gemv_stream_warps(int64_t M, int64_t K, int64_t N, int num_sms) {
  const int per_sm = M <= 8 ? stream_ctas_per_sm<G, 1>() : stream_ctas_per_sm<G, 2>();
  const int64_t T = (N / 64) * (K / G);
  return std::max<int64_t>(1, std::min<int64_t>(T, static_cast<int64_t>(per_sm) * num_sms * (kGemvThreads / 32)));
}

// Slots per column block for its pieces: a block's Gk chunks meet at most
// ceil((Gk - 1) W / T) + 1 warps' runs (the sum kernel uses each block's exact count).
int gemv_stream_pieces(int64_t K, int64_t N, int group, int64_t W) {
  const int64_t Gk = K / group, T = (N / 64) * Gk;
  return static_cast<int>(ceil_div((Gk - 1) * W, T) + 1);
}

template <int G>
int64_t gemv_stream_part_floats(int64_t M, int64_t K, int64_t N, int num_sms) {
  return (N / 64) * gemv_stream_pieces(K, N, G, gemv_stream_warps<G>(M, K, N, num_sms)) * M * 64;
}

template <int G>
cudaError_t launch_gemv_packed_g(const W4A16Args& a, const uint32_t* packed, int num_sms, float* part,
                                 cudaStream_t s, int* launches) {
  const int64_t W = gemv_stream_warps<G>(a.M, a.K, a.N, num_sms);
  const int pieces = gemv_stream_pieces(a.K, a.N, G, W);
  const unsigned ctas = static_cast<unsigned>(ceil_div(W, static_cast<int64_t>(kGemvThreads / 32)));
  auto kernel = a.M <= 8 ? gemv_stream_kernel<G, 1> : gemv_stream_kernel<G, 2>;
  static unsigned long long done1 = 0, done2 = 0;  // the limit is per device
  cudaError_t e0 = set_smem_limit_once(kernel, PackedSmem<G>::kSmem + kSActBytes, a.M <= 8 ? &done1 : &done2);
  if (e0 != cudaSuccess) return e0;
  kernel<<<ctas, kGemvThreads, stream_smem<G>(a.M, a.K), s>>>(a.A, static_cast<int>(a.M),
                                                              reinterpret_cast<const uint4*>(packed), a.steps,
                                                              a.zeros, a.K, a.N, W, pieces, part);
  *launches += 1;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t mn = a.M * a.N;
  const unsigned blocks = static_cast<unsigned>(std::min<int64_t>(ceil_div(mn, 256), 4 * num_sms));
  piece_sum_kernel<<<blocks, 256, 0, s>>>(part, pieces, static_cast<int>(a.M), a.N, a.K / G, W, a.Y);
  *launches += 1;
  return cudaGetLastError();
}

}  // namespace

int64_t gemv_split_floats(int64_t M, int64_t K, int64_t N, int group, int num_sms, bool packed) {
  if (packed) {
    switch (group) {
      case 32: return gemv_stream_part_floats<32>(M, K, N, num_sms);
      case 64: return gemv_stream_part_floats<64>(M, K, N, num_sms);
      default: return gemv_stream_part_floats<128>(M, K, N, num_sms);
    }
  }
  const int64_t splits = gemv_splits(K, N, group, num_sms);
  return splits > 1 ? splits * M * N : 0;
}

cudaError_t launch_w4a16_gemv(const W4A16Args& a, int num_sms, float* part, cudaStream_t s, int* launches) {
  if (a.M < 1 || a.M > kW4A16GemvMaxM) return cudaErrorInvalidValue;
  switch (a.group) {
    case 32: return launch_gemv_g<32>(a, num_sms, part, s, launches);
    case 64: return launch_gemv_g<64>(a, num_sms, part, s, launches);
    default: return launch_gemv_g<128>(a, num_sms, part, s, launches);
  }
}

cudaError_t launch_w4a16_dequant(const int32_t* codes, const __half* steps, const __half* zeros, int64_t K, int64_t N,
                                 int group, __half* Wt, cudaStream_t s, int* launches) {
  dim3 grid(static_cast<unsigned>(ceil_div(N, kDqN)), static_cast<unsigned>(ceil_div(K, kDqK)));
  dequant_kernel<<<grid, kDqThreads, 0, s>>>(codes, steps, zeros, K, N, group, Wt);
  *launches += 1;
  return cudaGetLastError();
}

}  // namespace awq

namespace awq {
cudaError_t launch_w4a16_repack(const int32_t* codes, int64_t K, int64_t N, uint32_t* packed, cudaStream_t s,
                                int* launches) {
  const int64_t total = K * N / 8;
  const unsigned blocks = static_cast<unsigned>(std::min<int64_t>(ceil_div(total, 256), 148 * 16));
  repack_kernel<<<blocks, 256, 0, s>>>(codes, K, N, packed);
  *launches += 1;
  return cudaGetLastError();
}

cudaError_t launch_w4a16_gemv_packed(const W4A16Args& a, const uint32_t* packed, int num_sms, float* part,
                                     cudaStream_t s, int* launches) {
  if (a.M < 1 || a.M > kW4A16GemvMaxM || a.N % 64) return cudaErrorInvalidValue;
  switch (a.group) {
    case 32: return launch_gemv_packed_g<32>(a, packed, num_sms, part, s, launches);
    case 64: return launch_gemv_packed_g<64>(a, packed, num_sms, part, s, launches);
    default: return launch_gemv_packed_g<128>(a, packed, num_sms, part, s, launches);
  }
}
}  // namespace awq
