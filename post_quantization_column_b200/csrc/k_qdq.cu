// k_qdq.cu — candidate weights and the packed artifact.
//
// qdq_kernel: for every candidate scale vector s_i, W' = diag(s_i) W is quantized and
// dequantized group-wise along K with the asymmetric 4-bit zero-point quantizer and
// folded back, W_hat_i = diag(s_i)^-1 Q(W') ("AWQ：为什么 4-bit 权重量化要先观察
// Activation" §4 candidate loop, §7 quantizer). A CTA stages one `group` x 64 tile of
// W in shared memory once, keeps it in registers, and emits all n_grid candidates
// (plus the plain bf16 copy of W used for the reference output), so W is read from
// HBM once for the whole grid. Each lane owns 8 consecutive rows of 2 columns; the
// group/8 row-lanes that share a column finish its min/max with a shuffle butterfly,
// and each lane writes its 8 rows as one 16-byte run of the K-major operand (N x K,
// K contiguous) that the loss GEMM's TMA reads. With 16 elements per lane the kernel
// fits 64 registers, so 32 warps share an SM.
//
// Arithmetic. The definition is a chain of IEEE fp32 operations (see
// awq_device.cuh): q = clamp(rint(w'/step) + z), W_hat = bf16(((q - z) * step) / s).
// The two divisions per element are replaced by products with correctly rounded
// reciprocals (one per column, one per row), which are within 2^-22 relative of the
// exact quotients. The rounding decisions that follow are then provably the same as
// the definition's unless a quotient lies within 2^-15 of a half-integer (for rint)
// or within 8 fp32 ulps of a bf16 rounding midpoint (for the bf16 conversion); those
// rare elements (about 3 in 10^5) are recomputed with the exact divisions. Rounding to
// an integer uses (x + 1.5*2^23) - 1.5*2^23, exact round-half-to-even for |x| < 2^22.
//
// pack_kernel: the same tile walk for the chosen candidate only (the first argmin of
// the fp32 losses, computed by every CTA): codes go through shared memory and are
// packed eight per int32 along N (QUANT-P4 §5.3), steps and zeros are written as fp16,
// and the chosen scales are copied out.
#include "awq_device.cuh"
#include "awq_kernels.h"

namespace awq {
namespace {

constexpr int kQdqCols = 64;                          // columns per CTA
constexpr int kRowsPerLane = 8;                       // one 16-byte bf16 run per column
constexpr float kRoundMagic = 12582912.0f;            // 1.5 * 2^23
constexpr float kNearHalf = 0.5f - 1.0f / 32768.0f;   // |x - rint(x)| at or above this: recheck
constexpr float kTinyStep = 7.888609052210118e-31f;   // 2^-100: below this, the exact path
constexpr float kHugeRecip = 1.2676506002282294e30f;  // 2^100

// Thread layout for a group size G: RL row-lanes x CG column-lanes per warp, each
// lane 8 rows x 2 columns; a warp covers G rows x 2*CG columns.
template <int G>
struct Tile {
  static constexpr int RL = G / kRowsPerLane;       // 4, 8, 16
  static constexpr int CG = 32 / RL;                // 8, 4, 2
  static constexpr int kColsPerWarp = 2 * CG;       // 16, 8, 4
  static constexpr int kWarps = kQdqCols / kColsPerWarp;
  static constexpr int kThreads = 32 * kWarps;      // 128, 256, 512
  static constexpr int kPitch = G + 1;              // transposed W tile, odd pitch
  static constexpr int kSkewPitch = G + G / 16;     // candidate rows of scales, skewed
  static constexpr int kBlocksPerSm = 1024 / kThreads;
};

// Row r of a candidate's scales sits at r + r/16: row-lanes 8 rows apart hit
// distinct banks.
__device__ __forceinline__ int skew(int r) { return r + (r >> 4); }

__device__ __forceinline__ float round_small(float x) {
  return __fsub_rn(__fadd_rn(x, kRoundMagic), kRoundMagic);
}

// True when bf16 rounding of fp32 values within 8 ulps of v could differ, i.e. when
// the low 16 bits of v lie within 8 of 0x8000. Multiplying by 2^16 moves those bits
// to the top (a multiply-add, off the integer-compare pipe the rest of the kernel
// loads), so one unsigned compare decides: ((u - 0x7FF8) mod 2^16) << 16 <= 16 << 16.
__device__ __forceinline__ bool near_bf16_midpoint(float v) {
  const uint32_t x = __float_as_uint(v) * 65536u + 0x80080000u;  // 0x80080000 = -(0x7FF8 << 16) mod 2^32
  return x <= 0x00100000u;
}

__device__ __forceinline__ void store_bf16x8(__nv_bfloat16* dst, const float (&v)[8]) {
  uint32_t packed[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    packed[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  *reinterpret_cast<uint4*>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
}

// Stage a G x 64 tile of W transposed in shared memory (sWT[col][row]) from coalesced
// 16-byte global loads; columns at or beyond N read as 0. Returns whether a
// non-finite value was seen.
template <typename T, int G>
__device__ __forceinline__ bool stage_tile(const T* __restrict__ W, int64_t N, int64_t k0, int64_t n0, float* sWT) {
  constexpr int VEC = 16 / sizeof(T);
  constexpr int VPR = kQdqCols / VEC;
  bool bad = false;
  for (int idx = threadIdx.x; idx < G * VPR; idx += Tile<G>::kThreads) {
    const int r = idx / VPR, v = idx % VPR;
    const int64_t col = n0 + static_cast<int64_t>(v) * VEC;
    float vals[VEC];
    if (col < N) {  // N % 8 == 0: a vector lies wholly inside or outside
      const uint4 raw = __ldcs(reinterpret_cast<const uint4*>(W + (k0 + r) * N + col));
      const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
      for (int i = 0; i < VEC; ++i) {
        vals[i] = to_f32<T>(e[i]);
        bad |= !isfinite(vals[i]);
      }
    } else {
#pragma unroll
      for (int i = 0; i < VEC; ++i) vals[i] = 0.0f;
    }
#pragma unroll
    for (int i = 0; i < VEC; ++i) sWT[(v * VEC + i) * Tile<G>::kPitch + r] = vals[i];
  }
  return bad;
}

struct ColumnQdq {
  QdqParams p;
  float recip;  // correctly rounded 1/step
  bool exact;   // take the exact path for the whole column
};

// Finish both columns' group min/max across the RL row-lanes that share them (a
// butterfly over the low lane bits), then compute each column's parameters once per
// column-group — even row-lanes column 0, odd ones column 1 — and broadcast them.
template <int RL>
__device__ __forceinline__ void column_qdq(float (&mn)[2], float (&mx)[2], ColumnQdq (&cq)[2], int quantizer) {
#pragma unroll
  for (int o = 1; o < RL; o <<= 1) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      mn[j] = fminf(mn[j], __shfl_xor_sync(0xffffffffu, mn[j], o));
      mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], o));
    }
  }
  const int lane = threadIdx.x & 31;
  const int odd = lane & 1;
  const QdqParams p = qdq_params_q(odd ? mn[1] : mn[0], odd ? mx[1] : mx[0], quantizer);
  const float r = __frcp_rn(p.step);
  const int exact = !(p.step >= kTinyStep && r <= kHugeRecip);
  const int base = lane & ~(RL - 1);
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    cq[j].p.step = __shfl_sync(0xffffffffu, p.step, base + j);
    cq[j].p.zero = __shfl_sync(0xffffffffu, p.zero, base + j);
    cq[j].p.qmax = p.qmax;  // the same for every column of the launch
    cq[j].recip = __shfl_sync(0xffffffffu, r, base + j);
    cq[j].exact = __shfl_sync(0xffffffffu, exact, base + j) != 0;
  }
}

// Whether every scaled weight of a column rounds inside [-z, qmax - z] without
// clamping: t = w' * (1/step) is monotone in w', so its extremes are the range times
// the reciprocal, and a margin of 2^-15 covers the difference to the exact quotient.
__device__ __forceinline__ bool clamp_free(float mn, float mx, const ColumnQdq& c) {
  const float lo = -c.p.zero, hi = c.p.qmax - c.p.zero;
  return !c.exact && __fmul_rn(mn, c.recip) >= lo - kNearHalf && __fmul_rn(mx, c.recip) <= hi + kNearHalf;
}

// Codes (as q - z), reconstruction and fold-back of this lane's 8 rows of one column;
// returns whether any element needs the exact divisions.
template <bool kClamp>
__device__ __forceinline__ bool fold_back_8(const float (&s)[8], const float (&w)[8], const float* rs,
                                            const ColumnQdq& c, float (&out)[8]) {
  const float lo = -c.p.zero, hi = c.p.qmax - c.p.zero;
  bool need = false;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float t = __fmul_rn(__fmul_rn(s[i], w[i]), c.recip);
    if (kClamp) t = fminf(fmaxf(t, lo), hi);
    const float qz = round_small(t);  // q - z, an integer in [-z, qmax - z]
    need |= fabsf(__fsub_rn(t, qz)) >= kNearHalf;
    const float v = __fmul_rn(__fmul_rn(qz, c.p.step), rs[i]);
    need |= near_bf16_midpoint(v);
    out[i] = v;
  }
  return need;
}

template <typename T, int G>
__global__ void __launch_bounds__(Tile<G>::kThreads, Tile<G>::kBlocksPerSm)
    qdq_kernel(const T* __restrict__ W, int64_t K, int64_t N, int n_grid, const float* __restrict__ S,
               __nv_bfloat16* __restrict__ Wt, int* err, int64_t group0, int quantizer) {
  using L = Tile<G>;
  extern __shared__ float smem[];
  float* sWT = smem;                                 // [64][kPitch]
  float* sS = smem + kQdqCols * L::kPitch;           // [n_grid][kSkewPitch] scales
  float* sR = sS + n_grid * L::kSkewPitch;           // [n_grid][kSkewPitch] correctly rounded 1/s

  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kQdqCols;
  const int64_t k0 = (group0 + static_cast<int64_t>(blockIdx.y)) * G;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  if (stage_tile<T, G>(W, N, k0, n0, sWT)) atomicOr(err, kErrNonfiniteW);
  for (int idx = threadIdx.x; idx < n_grid * G; idx += L::kThreads) {
    const int c = idx / G, r = idx % G;
    const float s = S[static_cast<int64_t>(c) * K + k0 + r];
    sS[c * L::kSkewPitch + skew(r)] = s;
    sR[c * L::kSkewPitch + skew(r)] = __frcp_rn(s);
  }
  __syncthreads();

  const int rl = lane % L::RL, cg = lane / L::RL;
  const int col0 = warp * L::kColsPerWarp + cg * 2;  // this lane's two columns in the tile
  const int row0 = rl * kRowsPerLane;                 // this lane's 8 rows in the group
  const int64_t n = n0 + col0;
  const bool active = n < N;  // N is even, so columns n and n+1 are both in or both out

  float w[2][8];
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int i = 0; i < 8; ++i) w[j][i] = sWT[(col0 + j) * L::kPitch + row0 + i];

  // reference operand: bf16(W), transposed
  if (active) {
#pragma unroll
    for (int j = 0; j < 2; ++j) store_bf16x8(Wt + (n + j) * K + k0 + row0, w[j]);
  }

  const int srow = skew(row0);  // 8 rows never straddle a skew pad (pads every 16)
  for (int c = 0; c < n_grid; ++c) {
    const float* rs = sR + c * L::kSkewPitch + srow;
    float s[8];
    bool rows_exact = false;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      s[i] = sS[c * L::kSkewPitch + srow + i];
      rows_exact |= !(fabsf(rs[i]) <= kHugeRecip && fabsf(rs[i]) >= kTinyStep);
    }
    // pass 1: the group range of each column of W' = s * W
    float mn[2], mx[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      mn[j] = INFINITY;
      mx[j] = -INFINITY;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float wp = __fmul_rn(s[i], w[j][i]);
        mn[j] = fminf(mn[j], wp);
        mx[j] = fmaxf(mx[j], wp);
      }
    }
    ColumnQdq cq[2];
    column_qdq<L::RL>(mn, mx, cq, quantizer);
    const bool no_clamp =
        __all_sync(0xffffffffu, clamp_free(mn[0], mx[0], cq[0]) && clamp_free(mn[1], mx[1], cq[1]));

    // pass 2: codes, reconstruction and fold-back
    __nv_bfloat16* slot = Wt + static_cast<int64_t>(c + 1) * N * K;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float out[8];
      bool need = rows_exact || cq[j].exact;
      if (no_clamp)
        need |= fold_back_8<false>(s, w[j], rs, cq[j], out);
      else
        need |= fold_back_8<true>(s, w[j], rs, cq[j], out);
      if (__any_sync(0xffffffffu, need) && need) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          out[i] = qdq_fold_back(qdq_code(__fmul_rn(s[i], w[j][i]), cq[j].p), cq[j].p, s[i]);
      }
      if (active) store_bf16x8(slot + (n + j) * K + k0 + row0, out);
    }
  }
}

// Register-staged tile loads for the persistent pack kernel: each thread holds its
// share of the next G x 64 tile (16-byte vectors) while the current tile is computed.
template <typename T, int G>
struct TileLoad {
  static constexpr int VEC = 16 / sizeof(T);
  static constexpr int VPR = kQdqCols / VEC;
  static constexpr int kPerThread = G * VPR / Tile<G>::kThreads;  // 2 (bf16) or 4 (fp32)
  uint4 v[kPerThread];

  __device__ __forceinline__ void load(const T* __restrict__ W, int64_t N, int64_t k0, int64_t n0) {
#pragma unroll
    for (int it = 0; it < kPerThread; ++it) {
      const int idx = threadIdx.x + it * Tile<G>::kThreads;
      const int r = idx / VPR, vv = idx % VPR;
      const int64_t col = n0 + static_cast<int64_t>(vv) * VEC;
      v[it] = col < N ? __ldcs(reinterpret_cast<const uint4*>(W + (k0 + r) * N + col)) : make_uint4(0, 0, 0, 0);
    }
  }
  __device__ __forceinline__ void store(float* sWT) const {
#pragma unroll
    for (int it = 0; it < kPerThread; ++it) {
      const int idx = threadIdx.x + it * Tile<G>::kThreads;
      const int r = idx / VPR, vv = idx % VPR;
      const T* e = reinterpret_cast<const T*>(&v[it]);
#pragma unroll
      for (int i = 0; i < VEC; ++i) sWT[(vv * VEC + i) * Tile<G>::kPitch + r] = to_f32<T>(e[i]);
    }
  }
};

// Persistent: each CTA walks tiles blockIdx.x, + gridDim.x, ... (column tiles of one
// group are adjacent), loading the next tile into registers while it quantizes the
// current one, so HBM reads overlap the arithmetic.
template <typename T, int G>
__global__ void __launch_bounds__(Tile<G>::kThreads, Tile<G>::kBlocksPerSm)
    pack_kernel(const T* __restrict__ W, int64_t K, int64_t N, int n_grid, const float* __restrict__ S,
                const float* __restrict__ losses, int* __restrict__ best_out, int32_t* __restrict__ codes,
                __half* __restrict__ steps, __half* __restrict__ zeros, float* __restrict__ out_scales,
                int quantizer) {
  using L = Tile<G>;
  __shared__ float sWT[kQdqCols * L::kPitch];
  __shared__ __align__(16) uint8_t sQ[G][kQdqCols];
  __shared__ float sScale[G];
  __shared__ int sBest;

  const int64_t tiles_n = ceil_div(N, kQdqCols);
  const int64_t tiles = tiles_n * (K / G);
  const int64_t words = N / 8;

  // the chosen candidate: first minimum of the fp32 losses
  if (threadIdx.x == 0) {
    int b = 0;
    for (int c = 1; c < n_grid; ++c)
      if (losses[c] < losses[b]) b = c;
    sBest = b;
    if (blockIdx.x == 0) *best_out = b;
  }

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rl = lane % L::RL, cg = lane / L::RL;
  const int col0 = warp * L::kColsPerWarp + cg * 2;
  const int row0 = rl * kRowsPerLane;

  TileLoad<T, G> next;
  int64_t t = blockIdx.x;
  if (t < tiles) next.load(W, N, (t / tiles_n) * G, (t % tiles_n) * kQdqCols);
  __syncthreads();
  const float* Sbest = S + static_cast<int64_t>(sBest) * K;

  for (; t < tiles; t += gridDim.x) {
    const int64_t k0 = (t / tiles_n) * G, n0 = (t % tiles_n) * kQdqCols;
    next.store(sWT);
    for (int r = threadIdx.x; r < G; r += L::kThreads) {
      const float sv = Sbest[k0 + r];
      sScale[r] = sv;
      if (n0 == 0) out_scales[k0 + r] = sv;
    }
    __syncthreads();
    const int64_t tn = t + gridDim.x;
    if (tn < tiles) next.load(W, N, (tn / tiles_n) * G, (tn % tiles_n) * kQdqCols);

    float wp[2][8];
    float mn[2], mx[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      mn[j] = INFINITY;
      mx[j] = -INFINITY;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        wp[j][i] = __fmul_rn(sScale[row0 + i], sWT[(col0 + j) * L::kPitch + row0 + i]);
        mn[j] = fminf(mn[j], wp[j][i]);
        mx[j] = fmaxf(mx[j], wp[j][i]);
      }
    }
    ColumnQdq cq[2];
    column_qdq<L::RL>(mn, mx, cq, quantizer);

    float q[2][8];
    bool need = cq[0].exact || cq[1].exact;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float lo = -cq[j].p.zero, hi = cq[j].p.qmax - cq[j].p.zero;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float tc = fminf(fmaxf(__fmul_rn(wp[j][i], cq[j].recip), lo), hi);
        const float qz = round_small(tc);
        need |= fabsf(__fsub_rn(tc, qz)) >= kNearHalf;
        q[j][i] = __fadd_rn(qz, cq[j].p.zero);
      }
    }
    if (__any_sync(0xffffffffu, need) && need) {
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i) q[j][i] = qdq_code(wp[j][i], cq[j].p);
    }
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int i = 0; i < 8; ++i) sQ[row0 + i][col0 + j] = static_cast<uint8_t>(q[j][i]);

    const int64_t n = n0 + col0;
    if (rl == 0 && n < N) {
      const int64_t g = k0 / G;
      *reinterpret_cast<__half2*>(steps + g * N + n) = __halves2half2(__float2half_rn(cq[0].p.step),
                                                                      __float2half_rn(cq[1].p.step));
      *reinterpret_cast<__half2*>(zeros + g * N + n) = __halves2half2(__float2half_rn(cq[0].p.zero),
                                                                      __float2half_rn(cq[1].p.zero));
    }
    __syncthreads();
    // eight codes (one 8-byte run of a tile row) -> one int32, nibble i = column 8w + i
    for (int idx = threadIdx.x; idx < G * (kQdqCols / 8); idx += L::kThreads) {
      const int r = idx / (kQdqCols / 8), wd = idx % (kQdqCols / 8);
      const int64_t word = n0 / 8 + wd;
      if (word >= words) continue;
      const uint2 b = *reinterpret_cast<const uint2*>(&sQ[r][wd * 8]);
      uint32_t packed = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        packed |= ((b.x >> (8 * i)) & 0xFu) << (4 * i);
        packed |= ((b.y >> (8 * i)) & 0xFu) << (4 * (i + 4));
      }
      codes[(k0 + r) * words + word] = static_cast<int32_t>(packed);
    }
    __syncthreads();  // sWT, sQ and sScale are rewritten by the next tile
  }
}

template <typename T, int G>
cudaError_t launch_qdq_t(const T* W, int64_t K, int64_t N, int n_grid, const float* S, __nv_bfloat16* Wt,
                         int* err, int64_t group0, int64_t groups, cudaStream_t s, int quantizer) {
  using L = Tile<G>;
  const size_t smem = (static_cast<size_t>(kQdqCols) * L::kPitch + 2 * static_cast<size_t>(n_grid) * L::kSkewPitch) *
                      sizeof(float);
  // the limit is raised once, to what the largest grid (64 candidates) needs
  const int smem_max = (kQdqCols * L::kPitch + 2 * 64 * L::kSkewPitch) * static_cast<int>(sizeof(float));
  static unsigned long long attr_done = 0;
  cudaError_t e = set_smem_limit_once(qdq_kernel<T, G>, smem_max, &attr_done);
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(ceil_div(N, kQdqCols)), static_cast<unsigned>(groups));
  qdq_kernel<T, G><<<grid, L::kThreads, smem, s>>>(W, K, N, n_grid, S, Wt, err, group0, quantizer);
  return cudaGetLastError();
}

template <typename T, int G>
cudaError_t launch_pack_t(const T* W, int64_t K, int64_t N, int n_grid, const float* S, const float* losses,
                          int* best, int32_t* codes, __half* steps, __half* zeros, float* out_scales,
                          cudaStream_t s, int quantizer) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = ceil_div(N, kQdqCols) * (K / G);
  const int64_t per_sm = Tile<G>::kBlocksPerSm;  // resident CTAs per SM at <= 64 registers
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(tiles, per_sm * sms));
  pack_kernel<T, G><<<grid, Tile<G>::kThreads, 0, s>>>(W, K, N, n_grid, S, losses, best, codes, steps, zeros,
                                                       out_scales, quantizer);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_qdq_groups(const void* W, int in_dtype, int64_t K, int64_t N, int group, int n_grid,
                              const float* S, __nv_bfloat16* Wt, int* err, int64_t group0, int64_t groups,
                              cudaStream_t s, int* launches, int quantizer) {
  *launches += 1;
  if (in_dtype == 0) {
    const auto* w = static_cast<const __nv_bfloat16*>(W);
    switch (group) {
      case 32: return launch_qdq_t<__nv_bfloat16, 32>(w, K, N, n_grid, S, Wt, err, group0, groups, s, quantizer);
      case 64: return launch_qdq_t<__nv_bfloat16, 64>(w, K, N, n_grid, S, Wt, err, group0, groups, s, quantizer);
      default: return launch_qdq_t<__nv_bfloat16, 128>(w, K, N, n_grid, S, Wt, err, group0, groups, s, quantizer);
    }
  }
  const auto* w = static_cast<const float*>(W);
  switch (group) {
    case 32: return launch_qdq_t<float, 32>(w, K, N, n_grid, S, Wt, err, group0, groups, s, quantizer);
    case 64: return launch_qdq_t<float, 64>(w, K, N, n_grid, S, Wt, err, group0, groups, s, quantizer);
    default: return launch_qdq_t<float, 128>(w, K, N, n_grid, S, Wt, err, group0, groups, s, quantizer);
  }
}

cudaError_t launch_qdq(const void* W, int in_dtype, int64_t K, int64_t N, int group, int n_grid, const float* S,
                       __nv_bfloat16* Wt, int* err, cudaStream_t s, int* launches, int quantizer) {
  return launch_qdq_groups(W, in_dtype, K, N, group, n_grid, S, Wt, err, 0, K / group, s, launches, quantizer);
}

cudaError_t launch_pack(const void* W, int in_dtype, int64_t K, int64_t N, int group, int n_grid, const float* S,
                        const float* losses, int* best, int32_t* codes, __half* steps, __half* zeros,
                        float* out_scales, cudaStream_t s, int* launches, int quantizer) {
  *launches += 1;
  if (in_dtype == 0) {
    const auto* w = static_cast<const __nv_bfloat16*>(W);
    switch (group) {
      case 32: return launch_pack_t<__nv_bfloat16, 32>(w, K, N, n_grid, S, losses, best, codes, steps, zeros, out_scales, s, quantizer);
      case 64: return launch_pack_t<__nv_bfloat16, 64>(w, K, N, n_grid, S, losses, best, codes, steps, zeros, out_scales, s, quantizer);
      default: return launch_pack_t<__nv_bfloat16, 128>(w, K, N, n_grid, S, losses, best, codes, steps, zeros, out_scales, s, quantizer);
    }
  }
  const auto* w = static_cast<const float*>(W);
  switch (group) {
    case 32: return launch_pack_t<float, 32>(w, K, N, n_grid, S, losses, best, codes, steps, zeros, out_scales, s, quantizer);
    case 64: return launch_pack_t<float, 64>(w, K, N, n_grid, S, losses, best, codes, steps, zeros, out_scales, s, quantizer);
    default: return launch_pack_t<float, 128>(w, K, N, n_grid, S, losses, best, codes, steps, zeros, out_scales, s, quantizer);
  }
}

}  // namespace awq
