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
// For decode the codes are read in the order the MMA fragments use them: for every
// 16-row step s, 64-column block cb and lane (g, t), 16 bytes (4 words) hold the lane's
// 32 nibbles. Word u serves column tiles j = 2u and 2u + 1; its nibble p (0..3) and
// p + 4 are the pair (rows r, r + 1) of fragment p: tile 2u + (p >> 1), rows 2t (p even)
// or 2t + 8 (p odd), column 8 j + g. So (word >> 4p) & 0x000F000F puts the pair in the two
// halves, one shift and one logic op per two weights, and a warp reads 512 contiguous
// bytes per step.
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
      const int j = 2 * u + (p >> 1);
      const int64_t row = 16 * s + ((p & 1) ? 2 * t + 8 : 2 * t);
      const int64_t w = cb * 8 + j;
      const uint32_t lo = (static_cast<uint32_t>(__ldg(codes + row * words + w)) >> (4 * g)) & 0xFu;
      const uint32_t hi = (static_cast<uint32_t>(__ldg(codes + (row + 1) * words + w)) >> (4 * g)) & 0xFu;
      out |= (lo << (4 * p)) | (hi << (4 * (p + 4)));
    }
    P[i] = out;
  }
}

// The decode GEMV on the repacked codes: as gemv_kernel, but a step is one 16-byte copy per
// lane into a per-warp ring of kPRing stages in shared memory (cp.async, kPRing - 1 steps
// ahead, so about 8 KB per warp are in flight), the group's steps and zeros travel in the
// same ring (16 lanes copy the 64 columns' 128 + 128 bytes with the group's first step),
// and each fp16 pair costs one shift and one logic op before the packed (1024 + q) -
// (1024 + z) and the multiply by the step.
constexpr int kPRing = 16;                          // steps in flight per warp (a power of two)
constexpr int kPActBytes = 16 * 1024;               // activations staged per CTA when they fit (2 CTAs per SM)
constexpr int kPRingBytes = kPRing * 32 * 16;       // 8 KB of codes per warp
// Parameter buffers per warp: a group's steps and zeros are copied with its first step,
// up to kPRing - 1 steps before that step is computed, and must outlive the whole group,
// so PB * S > kPRing + S - 2 for S = G / 16 steps per group: 16, 8 and 4 for G = 32, 64, 128.
template <int G>
struct PackedSmem {
  static constexpr int S = G / 16;
  static constexpr int PB = G == 32 ? 16 : (G == 64 ? 8 : 4);
  static_assert(PB * S > kPRing + S - 2, "parameter buffers must outlive their group");
  static constexpr int kParamBytes = PB * 2 * 64 * 2;  // PB groups of 64 steps + 64 zeros (fp16)
  static constexpr int kWarpBytes = kPRingBytes + kParamBytes;
  static constexpr int kSmem = (kGemvThreads / 32) * kWarpBytes;
};

template <int G>
__global__ void __launch_bounds__(kGemvThreads)
    gemv_packed_kernel(const __half* __restrict__ A, int M, const uint4* __restrict__ P,
                       const __half* __restrict__ steps, const __half* __restrict__ zeros, int64_t K, int64_t N,
                       int64_t k_per_split, float* __restrict__ out) {
  __shared__ float red[kGemvThreads / 32][16][kGemvCols];
  extern __shared__ __align__(16) uint8_t pdyn[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int gq = lane >> 2, tq = lane & 3;
  const int64_t cbs = N / 64, cb = blockIdx.x;
  const int64_t k0 = static_cast<int64_t>(blockIdx.y) * k_per_split;
  const int64_t k1 = min(K, k0 + k_per_split);
  // warps take whole groups of the split (contiguous runs), so parameters change only
  // between the unrolled steps of one group
  constexpr int kStepsPerGroup = G / 16;
  const int n_groups = static_cast<int>((k1 - k0) / G);
  const int gpw = (n_groups + kGemvThreads / 32 - 1) / (kGemvThreads / 32);
  const int g_begin = min(n_groups, warp * gpw), g_end = min(n_groups, g_begin + gpw);
  const int s0 = g_begin * kStepsPerGroup, s1 = g_end * kStepsPerGroup;
  using PS = PackedSmem<G>;
  uint8_t* ring = pdyn + warp * PS::kWarpBytes;
  // the CTA's slice of the activations, staged once when it fits (M k_per_split halves)
  __half* sAct = reinterpret_cast<__half*>(pdyn + PS::kSmem);
  const bool staged = static_cast<int64_t>(M) * k_per_split * 2 <= kPActBytes;
  if (staged) {
    const int kn = static_cast<int>(k1 - k0);
    for (int i = threadIdx.x; i < M * (kn / 8); i += kGemvThreads) {
      const int m = i / (kn / 8), v = i % (kn / 8);
      *reinterpret_cast<uint4*>(sAct + m * k_per_split + 8 * v) =
          __ldg(reinterpret_cast<const uint4*>(A + static_cast<int64_t>(m) * K + k0 + 8 * v));
    }
    __syncthreads();
  }
  __half* params = reinterpret_cast<__half*>(ring + kPRingBytes);  // [PB][2][64]

  float acc[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;

  auto issue = [&](int s) {
    if (s < s1) {
      const int64_t gs = k0 / 16 + s;  // global step
      const uint32_t dst = smem_u32(ring + (s & (kPRing - 1)) * 512 + lane * 16);
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(P + (gs * cbs + cb) * 32 + lane)
                   : "memory");
      if (gs % kStepsPerGroup == 0 && lane < 16) {  // runs start on group boundaries
        const int64_t grp = (gs * 16) / G;
        const __half* src = (lane < 8 ? steps : zeros) + grp * N + cb * 64 + 8 * (lane & 7);
        const uint32_t pd = smem_u32(params + (grp & (PS::PB - 1)) * 128 + (lane < 8 ? 0 : 64) + 8 * (lane & 7));
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(pd), "l"(src) : "memory");
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
#pragma unroll 1
  for (int q = 0; q < kPRing - 1; ++q) issue(s0 + q);

  __half2 z2[8], st2[8];
  const __half k1024 = __float2half_rn(1024.0f);
  const __half* sArow0 = sAct + gq * k_per_split + 2 * tq;      // staged activations of token g
  const __half* sArow1 = sArow0 + 8 * k_per_split;              // and of token g + 8
#pragma unroll 1
  for (int gi = g_begin; gi < g_end; ++gi) {
    const int64_t grp = k0 / G + gi;
#pragma unroll
    for (int ss = 0; ss < kStepsPerGroup; ++ss) {
      const int s = gi * kStepsPerGroup + ss;
      issue(s + kPRing - 1);
      asm volatile("cp.async.wait_group %0;" ::"n"(kPRing - 1) : "memory");
      __syncwarp();  // the group's steps and zeros were copied by other lanes
      if (ss == 0) {
        const __half* pr = params + (grp & (PS::PB - 1)) * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const __half st = pr[8 * j + gq];
          const __half zb = __hadd(pr[64 + 8 * j + gq], k1024);  // exact: z is an integer <= 15
          st2[j] = __halves2half2(st, st);
          z2[j] = __halves2half2(zb, zb);
        }
      }
      const uint4 v = *reinterpret_cast<const uint4*>(ring + (s & (kPRing - 1)) * 512 + lane * 16);
      const int kk = 16 * s;  // row offset inside the split
      uint32_t a0 = 0, a1 = 0, a2 = 0, a3 = 0;
      if (staged) {
        if (gq < M) {
          a0 = *reinterpret_cast<const uint32_t*>(sArow0 + kk);
          a2 = *reinterpret_cast<const uint32_t*>(sArow0 + kk + 8);
        }
        if (gq + 8 < M) {
          a1 = *reinterpret_cast<const uint32_t*>(sArow1 + kk);
          a3 = *reinterpret_cast<const uint32_t*>(sArow1 + kk + 8);
        }
      } else {
        const int64_t kb = k0 + kk;
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
      }
      const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int j = 2 * u + h;
          uint32_t b[2];
#pragma unroll
          for (int which = 0; which < 2; ++which) {
            const int p = 2 * h + which;
            const uint32_t biased = ((wv[u] >> (4 * p)) & 0x000F000Fu) | 0x64006400u;  // halves 1024 + q
            b[which] = half2_as_u32(__hmul2(__hsub2(u32_as_half2(biased), z2[j]), st2[j]));
          }
          mma_f16_16816(acc[j], a0, a1, a2, a3, b[0], b[1]);
        }
      }
    }
    __syncwarp();  // all lanes are past this group's parameters before a later group overwrites them
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    red[warp][gq][8 * j + 2 * tq] = acc[j][0];
    red[warp][gq][8 * j + 2 * tq + 1] = acc[j][1];
    red[warp][gq + 8][8 * j + 2 * tq] = acc[j][2];
    red[warp][gq + 8][8 * j + 2 * tq + 1] = acc[j][3];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < M * kGemvCols; i += kGemvThreads) {
    const int m = i / kGemvCols, c = i % kGemvCols;
    float sum = red[0][m][c];
#pragma unroll
    for (int q = 1; q < kGemvThreads / 32; ++q) sum = __fadd_rn(sum, red[q][m][c]);
    out[(static_cast<int64_t>(blockIdx.y) * M + m) * N + cb * 64 + c] = sum;
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

// The repacked kernel gives its warps whole groups: a split holds at least 8 groups when
// the layer has that many.
int64_t gemv_packed_splits(int64_t K, int64_t N, int group, int num_sms) {
  const int64_t col_blocks = N / 64;
  const int64_t groups = K / group;
  int64_t splits = std::max<int64_t>(1, std::min<int64_t>(groups / 8, ceil_div(8 * num_sms, col_blocks)));
  const int64_t gps = ceil_div(groups, splits);
  return ceil_div(groups, gps);
}

template <int G>
cudaError_t launch_gemv_packed_g(const W4A16Args& a, const uint32_t* packed, int num_sms, float* part,
                                 cudaStream_t s, int* launches) {
  const int64_t col_blocks = a.N / 64;
  const int64_t splits = gemv_packed_splits(a.K, a.N, G, num_sms);
  const int64_t k_per_split = ceil_div(a.K / G, splits) * G;
  float* dst = splits == 1 ? a.Y : part;
  static unsigned long long done = 0;
  const int smem = PackedSmem<G>::kSmem +
                   (a.M * k_per_split * 2 <= kPActBytes ? static_cast<int>(a.M * k_per_split * 2) : 0);
  cudaError_t e0 = set_smem_limit_once(gemv_packed_kernel<G>, PackedSmem<G>::kSmem + kPActBytes, &done);
  if (e0 != cudaSuccess) return e0;
  gemv_packed_kernel<G><<<dim3(static_cast<unsigned>(col_blocks), static_cast<unsigned>(splits)), kGemvThreads,
                          smem, s>>>(a.A, static_cast<int>(a.M), reinterpret_cast<const uint4*>(packed), a.steps, a.zeros,
                               a.K, a.N, k_per_split, dst);
  *launches += 1;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || splits == 1) return e;
  const int64_t mn = a.M * a.N;
  const unsigned blocks = static_cast<unsigned>(std::min<int64_t>(ceil_div(mn, 256), 4 * num_sms));
  split_sum_kernel<<<blocks, 256, 0, s>>>(part, static_cast<int>(splits), mn, a.Y);
  *launches += 1;
  return cudaGetLastError();
}

}  // namespace

int64_t gemv_split_floats(int64_t M, int64_t K, int64_t N, int group, int num_sms, bool packed) {
  const int64_t splits = packed ? gemv_packed_splits(K, N, group, num_sms) : gemv_splits(K, N, group, num_sms);
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
