// k_qdq.cu — candidate weights and the packed artifact.
//
// qdq_kernel: for every candidate scale vector s_i, W' = diag(s_i) W is quantized and
// dequantized group-wise along K with the asymmetric 4-bit zero-point quantizer and
// folded back, W_hat_i = diag(s_i)^-1 Q(W') ("AWQ：为什么 4-bit 权重量化要先观察
// Activation" §4 candidate loop, §7 quantizer). A CTA stages one `group` x 64 tile of
// W in shared memory once, keeps it in registers, and emits all n_grid candidates
// (plus the plain bf16 copy of W used for the reference output), so W is read from
// HBM once for the whole grid. A warp owns 8 columns; within it, 8 row-lanes split
// the group's rows (group/8 consecutive rows each) and 4 column-lanes take 2 columns
// each, so a column's min/max is a 3-step warp-shuffle reduction and each lane
// writes group/8 consecutive elements of the K-major operand (N x K, K contiguous)
// that the loss GEMM's TMA reads.
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

constexpr int kQdqCols = 64;       // columns per CTA
constexpr int kQdqThreads = 256;   // 8 warps x 8 columns
constexpr float kRoundMagic = 12582912.0f;           // 1.5 * 2^23
constexpr float kNearHalf = 0.5f - 1.0f / 32768.0f;  // |x - rint(x)| at or above this: recheck
constexpr float kTinyStep = 7.888609052210118e-31f;  // 2^-100: below this, the exact path
constexpr float kHugeRecip = 1.2676506002282294e30f; // 2^100

__device__ __forceinline__ float round_small(float x) {
  return __fsub_rn(__fadd_rn(x, kRoundMagic), kRoundMagic);
}

// True when bf16 rounding of fp32 values within 8 ulps of v could differ.
__device__ __forceinline__ bool near_bf16_midpoint(float v) {
  const uint32_t u = __float_as_uint(v);
  return ((u - 0x7FF8u) & 0xFFFFu) <= 16u;
}

template <int RPL>
__device__ __forceinline__ void store_bf16_run(__nv_bfloat16* dst, const float (&v)[RPL]) {
  static_assert(RPL % 4 == 0, "runs of 4, 8 or 16 elements");
  uint32_t packed[RPL / 2];
#pragma unroll
  for (int i = 0; i < RPL / 2; ++i) {
    __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    packed[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  if constexpr (RPL == 4) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
  } else {
#pragma unroll
    for (int i = 0; i < RPL / 8; ++i)
      reinterpret_cast<uint4*>(dst)[i] =
          make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
  }
}

// Stage a G x 64 tile of W transposed in shared memory (sWT[col][row], odd pitch),
// from coalesced 16-byte global loads. Columns at or beyond N read as 0.
template <typename T, int G>
__device__ __forceinline__ bool stage_tile(const T* __restrict__ W, int64_t N, int64_t k0, int64_t n0, float* sWT) {
  constexpr int VEC = 16 / sizeof(T);
  constexpr int VPR = kQdqCols / VEC;
  constexpr int PITCH = G + 1;
  bool bad = false;
  for (int idx = threadIdx.x; idx < G * VPR; idx += kQdqThreads) {
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
    for (int i = 0; i < VEC; ++i) sWT[(v * VEC + i) * PITCH + r] = vals[i];
  }
  return bad;
}

// Finish a column's group min/max across the 8 row-lanes (lane bits 0-2) that
// share it: a 3-step butterfly, after which every lane holds both columns' range.
__device__ __forceinline__ void column_range_reduce(float (&mn)[2], float (&mx)[2]) {
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      mn[j] = fminf(mn[j], __shfl_xor_sync(0xffffffffu, mn[j], o));
      mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], o));
    }
  }
}

struct ColumnQdq {
  QdqParams p;
  float recip;  // correctly rounded 1/step
  bool exact;   // take the exact path for the whole column
};

// Lanes with even row-lane index compute column 0's parameters, odd ones column 1's;
// every lane then fetches both columns' parameters from its column-group.
__device__ __forceinline__ void column_params(const float (&mn)[2], const float (&mx)[2], ColumnQdq (&cq)[2]) {
  const int lane = threadIdx.x & 31;
  const int odd = lane & 1;
  const QdqParams p = qdq_params(odd ? mn[1] : mn[0], odd ? mx[1] : mx[0]);
  const float r = __frcp_rn(p.step);
  const int exact = !(p.step >= kTinyStep && r <= kHugeRecip);
  const int base = lane & ~7;
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    cq[j].p.step = __shfl_sync(0xffffffffu, p.step, base + j);
    cq[j].p.zero = __shfl_sync(0xffffffffu, p.zero, base + j);
    cq[j].recip = __shfl_sync(0xffffffffu, r, base + j);
    cq[j].exact = __shfl_sync(0xffffffffu, exact, base + j) != 0;
  }
}

// Skewed index of row r in a per-candidate row of scales (one padding float every 16
// rows), so the 8 row-lanes of a warp, 16 rows apart, read 8 different banks.
template <int G>
__device__ __forceinline__ int skew(int r) { return r + (r >> 4); }
template <int G>
__host__ __device__ constexpr int skewed_pitch() { return G + G / 16; }

// Whether every scaled weight of a column rounds inside [lo, hi] without clamping:
// t = w' * (1/step) is monotone in w', so its extremes are mn/mx times the reciprocal,
// and a margin of 2^-15 covers the difference to the exact quotient.
__device__ __forceinline__ bool clamp_free(float mn, float mx, const ColumnQdq& c) {
  const float lo = -c.p.zero, hi = 15.0f - c.p.zero;
  return !c.exact && __fmul_rn(mn, c.recip) >= lo - kNearHalf && __fmul_rn(mx, c.recip) <= hi + kNearHalf;
}

// Codes, reconstruction and fold-back of CH consecutive rows of one column. Returns
// whether any element needs the exact divisions (near a rounding boundary).
template <int CH, bool kClamp>
__device__ __forceinline__ bool fold_back_run(const float* s, const float* w, const float* rs, const ColumnQdq& c,
                                              float (&out)[CH]) {
  const float lo = -c.p.zero, hi = 15.0f - c.p.zero;
  bool need = false;
#pragma unroll
  for (int i = 0; i < CH; ++i) {
    float t = __fmul_rn(__fmul_rn(s[i], w[i]), c.recip);
    if (kClamp) t = fminf(fmaxf(t, lo), hi);
    const float qz = round_small(t);  // q - z, an integer in [-z, 15 - z]
    need |= fabsf(__fsub_rn(t, qz)) >= kNearHalf;
    const float v = __fmul_rn(__fmul_rn(qz, c.p.step), rs[i]);
    need |= near_bf16_midpoint(v);
    out[i] = v;
  }
  return need;
}

template <typename T, int G>
__global__ void __launch_bounds__(kQdqThreads, 2)
    qdq_kernel(const T* __restrict__ W, int64_t K, int64_t N, int n_grid, const float* __restrict__ S,
               __nv_bfloat16* __restrict__ Wt, int* err) {
  constexpr int RPL = G / 8;
  constexpr int CH = RPL < 8 ? RPL : 8;  // rows per store run
  constexpr int PITCH = G + 1;
  constexpr int SP = skewed_pitch<G>();
  extern __shared__ float smem[];
  float* sWT = smem;                        // [64][PITCH]
  float* sS = smem + kQdqCols * PITCH;      // [n_grid][SP] scales, skewed
  float* sR = sS + n_grid * SP;             // [n_grid][SP] correctly rounded 1/s, skewed

  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kQdqCols;
  const int64_t k0 = static_cast<int64_t>(blockIdx.y) * G;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  if (stage_tile<T, G>(W, N, k0, n0, sWT)) atomicOr(err, kErrNonfiniteW);
  for (int idx = threadIdx.x; idx < n_grid * G; idx += kQdqThreads) {
    const int c = idx / G, r = idx % G;
    const float s = S[static_cast<int64_t>(c) * K + k0 + r];
    sS[c * SP + skew<G>(r)] = s;
    sR[c * SP + skew<G>(r)] = __frcp_rn(s);
  }
  __syncthreads();

  const int rl = lane & 7, cg = lane >> 3;
  const int col0 = warp * 8 + cg * 2;  // this lane's two columns in the tile
  const int row0 = rl * RPL;           // this lane's rows in the group
  const int64_t n = n0 + col0;
  const bool active = n < N;           // N is even, so columns n and n+1 are both in or both out

  float w[2][RPL];
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int i = 0; i < RPL; ++i) w[j][i] = sWT[(col0 + j) * PITCH + row0 + i];

  // reference operand: bf16(W), transposed
  if (active) {
#pragma unroll
    for (int j = 0; j < 2; ++j) store_bf16_run<RPL>(Wt + (n + j) * K + k0 + row0, w[j]);
  }

  for (int c = 0; c < n_grid; ++c) {
    float s[RPL];
    // the row reciprocals stay in shared memory (16 rows = 16 + 1 floats, conflict-free)
    const float* rs = sR + c * SP + skew<G>(row0);
    bool rows_exact = false;
#pragma unroll
    for (int i = 0; i < RPL; ++i) {
      s[i] = sS[c * SP + skew<G>(row0 + i)];
      const float r = rs[skew<G>(row0 + i) - skew<G>(row0)];
      rows_exact |= !(fabsf(r) <= kHugeRecip && fabsf(r) >= kTinyStep);
    }
    // pass 1: the group range of each column of W' = s * W
    float mn[2], mx[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      mn[j] = INFINITY;
      mx[j] = -INFINITY;
#pragma unroll
      for (int i = 0; i < RPL; ++i) {
        const float wp = __fmul_rn(s[i], w[j][i]);
        mn[j] = fminf(mn[j], wp);
        mx[j] = fmaxf(mx[j], wp);
      }
    }
    column_range_reduce(mn, mx);
    ColumnQdq cq[2];
    column_params(mn, mx, cq);
    const bool no_clamp =
        __all_sync(0xffffffffu, clamp_free(mn[0], mx[0], cq[0]) && clamp_free(mn[1], mx[1], cq[1]));

    // pass 2: codes, reconstruction and fold-back, in runs of CH rows of one column
    __nv_bfloat16* slot = Wt + static_cast<int64_t>(c + 1) * N * K;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
#pragma unroll
      for (int h = 0; h < RPL; h += CH) {
        float out[CH];
        bool need = rows_exact || cq[j].exact;
        // rows h .. h+CH-1 of this lane never cross a skew pad (CH divides 16)
        const float* rsh = rs + skew<G>(row0 + h) - skew<G>(row0);
        if (no_clamp)
          need |= fold_back_run<CH, false>(s + h, w[j] + h, rsh, cq[j], out);
        else
          need |= fold_back_run<CH, true>(s + h, w[j] + h, rsh, cq[j], out);
        if (__any_sync(0xffffffffu, need) && need) {
#pragma unroll
          for (int i = 0; i < CH; ++i)
            out[i] = qdq_fold_back(qdq_code(__fmul_rn(s[h + i], w[j][h + i]), cq[j].p), cq[j].p, s[h + i]);
        }
        if (active) store_bf16_run<CH>(slot + (n + j) * K + k0 + row0 + h, out);
      }
    }
  }
}


template <typename T, int G>
__global__ void __launch_bounds__(kQdqThreads)
    pack_kernel(const T* __restrict__ W, int64_t K, int64_t N, int n_grid, const float* __restrict__ S,
                const float* __restrict__ losses, int* __restrict__ best_out, int32_t* __restrict__ codes,
                __half* __restrict__ steps, __half* __restrict__ zeros, float* __restrict__ out_scales) {
  constexpr int RPL = G / 8;
  constexpr int PITCH = G + 1;
  __shared__ float sWT[kQdqCols * PITCH];
  __shared__ __align__(16) uint8_t sQ[G][kQdqCols];
  __shared__ int sBest;

  // the chosen candidate: first minimum of the fp32 losses
  if (threadIdx.x == 0) {
    int b = 0;
    for (int c = 1; c < n_grid; ++c)
      if (losses[c] < losses[b]) b = c;
    sBest = b;
    if (blockIdx.x == 0 && blockIdx.y == 0) *best_out = b;
  }
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kQdqCols;
  const int64_t k0 = static_cast<int64_t>(blockIdx.y) * G;
  stage_tile<T, G>(W, N, k0, n0, sWT);
  __syncthreads();
  const int c = sBest;
  const float* srow = S + static_cast<int64_t>(c) * K + k0;
  if (blockIdx.x == 0)
    for (int r = threadIdx.x; r < G; r += kQdqThreads) out_scales[k0 + r] = srow[r];

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rl = lane & 7, cg = lane >> 3;
  const int col0 = warp * 8 + cg * 2;
  const int row0 = rl * RPL;
  float s[RPL];
#pragma unroll
  for (int i = 0; i < RPL; ++i) s[i] = srow[row0 + i];
  float wp[2][RPL];
  float mn[2], mx[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    mn[j] = INFINITY;
    mx[j] = -INFINITY;
#pragma unroll
    for (int i = 0; i < RPL; ++i) {
      wp[j][i] = __fmul_rn(s[i], sWT[(col0 + j) * PITCH + row0 + i]);
      mn[j] = fminf(mn[j], wp[j][i]);
      mx[j] = fmaxf(mx[j], wp[j][i]);
    }
  }
  column_range_reduce(mn, mx);
  ColumnQdq cq[2];
  column_params(mn, mx, cq);

  float q[2][RPL];
  bool need = cq[0].exact || cq[1].exact;
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const float lo = -cq[j].p.zero, hi = 15.0f - cq[j].p.zero;
#pragma unroll
    for (int i = 0; i < RPL; ++i) {
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
      for (int i = 0; i < RPL; ++i) q[j][i] = qdq_code(wp[j][i], cq[j].p);
  }
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int i = 0; i < RPL; ++i) sQ[row0 + i][col0 + j] = static_cast<uint8_t>(q[j][i]);

  const int64_t n = n0 + col0;
  if (rl == 0 && n < N) {
    const int64_t g = blockIdx.y;
    *reinterpret_cast<__half2*>(steps + g * N + n) = __halves2half2(__float2half_rn(cq[0].p.step),
                                                                    __float2half_rn(cq[1].p.step));
    *reinterpret_cast<__half2*>(zeros + g * N + n) = __halves2half2(__float2half_rn(cq[0].p.zero),
                                                                    __float2half_rn(cq[1].p.zero));
  }
  __syncthreads();
  // eight codes (one 8-byte run of a tile row) -> one int32, nibble i = column 8w + i
  const int64_t words = N / 8;
  for (int idx = threadIdx.x; idx < G * (kQdqCols / 8); idx += kQdqThreads) {
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
}

template <typename T, int G>
cudaError_t launch_qdq_t(const T* W, int64_t K, int64_t N, int n_grid, const float* S, __nv_bfloat16* Wt,
                         int* err, cudaStream_t s) {
  const size_t smem =
      (static_cast<size_t>(kQdqCols) * (G + 1) + 2 * static_cast<size_t>(n_grid) * skewed_pitch<G>()) * sizeof(float);
  // the limit is raised once, to what the largest grid (64 candidates) needs
  const int smem_max = (kQdqCols * (G + 1) + 2 * 64 * skewed_pitch<G>()) * static_cast<int>(sizeof(float));
  static unsigned long long attr_done = 0;
  cudaError_t e = set_smem_limit_once(qdq_kernel<T, G>, smem_max, &attr_done);
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(ceil_div(N, kQdqCols)), static_cast<unsigned>(K / G));
  qdq_kernel<T, G><<<grid, kQdqThreads, smem, s>>>(W, K, N, n_grid, S, Wt, err);
  return cudaGetLastError();
}

template <typename T, int G>
cudaError_t launch_pack_t(const T* W, int64_t K, int64_t N, int n_grid, const float* S, const float* losses,
                          int* best, int32_t* codes, __half* steps, __half* zeros, float* out_scales,
                          cudaStream_t s) {
  dim3 grid(static_cast<unsigned>(ceil_div(N, kQdqCols)), static_cast<unsigned>(K / G));
  pack_kernel<T, G><<<grid, kQdqThreads, 0, s>>>(W, K, N, n_grid, S, losses, best, codes, steps, zeros, out_scales);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_qdq(const void* W, int in_dtype, int64_t K, int64_t N, int group, int n_grid, const float* S,
                       __nv_bfloat16* Wt, int* err, cudaStream_t s, int* launches) {
  *launches += 1;
  if (in_dtype == 0) {
    const auto* w = static_cast<const __nv_bfloat16*>(W);
    switch (group) {
      case 32: return launch_qdq_t<__nv_bfloat16, 32>(w, K, N, n_grid, S, Wt, err, s);
      case 64: return launch_qdq_t<__nv_bfloat16, 64>(w, K, N, n_grid, S, Wt, err, s);
      default: return launch_qdq_t<__nv_bfloat16, 128>(w, K, N, n_grid, S, Wt, err, s);
    }
  }
  const auto* w = static_cast<const float*>(W);
  switch (group) {
    case 32: return launch_qdq_t<float, 32>(w, K, N, n_grid, S, Wt, err, s);
    case 64: return launch_qdq_t<float, 64>(w, K, N, n_grid, S, Wt, err, s);
    default: return launch_qdq_t<float, 128>(w, K, N, n_grid, S, Wt, err, s);
  }
}

cudaError_t launch_pack(const void* W, int in_dtype, int64_t K, int64_t N, int group, int n_grid, const float* S,
                        const float* losses, int* best, int32_t* codes, __half* steps, __half* zeros,
                        float* out_scales, cudaStream_t s, int* launches) {
  *launches += 1;
  if (in_dtype == 0) {
    const auto* w = static_cast<const __nv_bfloat16*>(W);
    switch (group) {
      case 32: return launch_pack_t<__nv_bfloat16, 32>(w, K, N, n_grid, S, losses, best, codes, steps, zeros, out_scales, s);
      case 64: return launch_pack_t<__nv_bfloat16, 64>(w, K, N, n_grid, S, losses, best, codes, steps, zeros, out_scales, s);
      default: return launch_pack_t<__nv_bfloat16, 128>(w, K, N, n_grid, S, losses, best, codes, steps, zeros, out_scales, s);
    }
  }
  const auto* w = static_cast<const float*>(W);
  switch (group) {
    case 32: return launch_pack_t<float, 32>(w, K, N, n_grid, S, losses, best, codes, steps, zeros, out_scales, s);
    case 64: return launch_pack_t<float, 64>(w, K, N, n_grid, S, losses, best, codes, steps, zeros, out_scales, s);
    default: return launch_pack_t<float, 128>(w, K, N, n_grid, S, losses, best, codes, steps, zeros, out_scales, s);
  }
}

}  // namespace awq
