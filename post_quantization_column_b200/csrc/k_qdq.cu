// k_qdq.cu — candidate weights and the packed artifact.
//
// qdq_kernel: for every candidate scale vector s_i, W' = diag(s_i) W is quantized and
// dequantized group-wise along K with the asymmetric 4-bit zero-point quantizer and
// folded back, W_hat_i = diag(s_i)^-1 Q(W') ("AWQ：为什么 4-bit 权重量化要先观察
// Activation" §4 candidate loop, §7 quantizer). A CTA stages one `group` x 64 tile of
// W in shared memory once, keeps it in registers, and emits all n_grid candidates
// (plus the plain bf16 copy of W used for the reference output), so W is read from
// HBM once for the whole grid. One warp owns one output column at a time: its 32
// lanes split the group's rows, the group min/max is a warp-shuffle reduction, and
// the warp writes the column's group as one contiguous run of the K-major operand
// that the loss GEMM's TMA reads (N x K, K contiguous).
//
// pack_kernel: recomputes the QDQ of the chosen candidate bit-for-bit and writes the
// artifact: 4-bit codes packed eight per int32 along N (QUANT-P4 §5.3), fp16 steps and
// fp16 zeros per (group, column), and the chosen scales.
#include "awq_device.cuh"
#include "awq_kernels.h"

namespace awq {
namespace {

constexpr int kQdqCols = 64;               // columns per CTA
constexpr int kQdqThreads = 256;           // 8 warps
constexpr int kColsPerWarp = kQdqCols / 8;  // 8
constexpr int kTilePitch = kQdqCols + 1;    // odd pitch: lanes reading one column hit distinct banks

template <typename T, int G>
__global__ void __launch_bounds__(kQdqThreads)
    qdq_kernel(const T* __restrict__ W, int64_t K, int64_t N, int n_grid, const float* __restrict__ S,
               __nv_bfloat16* __restrict__ Wt, int* err) {
  constexpr int RPL = G / 32;        // rows of the group per lane
  constexpr int VEC = 16 / sizeof(T);
  constexpr int VPR = kQdqCols / VEC;  // 16-byte vectors per tile row
  extern __shared__ float smem[];
  float* sW = smem;                    // [G][kTilePitch]
  float* sS = smem + G * kTilePitch;   // [n_grid][G]

  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kQdqCols;
  const int64_t k0 = static_cast<int64_t>(blockIdx.y) * G;
  const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;

  // 1. stage the W tile (coalesced 16-byte loads) and this group's scales
  bool bad = false;
  for (int idx = tid; idx < G * VPR; idx += kQdqThreads) {
    const int r = idx / VPR, v = idx % VPR;
    const int64_t col = n0 + static_cast<int64_t>(v) * VEC;
    float vals[VEC];
    if (col < N) {  // N % 8 == 0, so a vector lies wholly inside or outside
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
    for (int i = 0; i < VEC; ++i) sW[r * kTilePitch + v * VEC + i] = vals[i];
  }
  for (int idx = tid; idx < n_grid * G; idx += kQdqThreads) {
    const int c = idx / G, r = idx % G;
    sS[idx] = S[static_cast<int64_t>(c) * K + k0 + r];
  }
  if (bad) atomicOr(err, kErrNonfiniteW);
  __syncthreads();

  // 2. this warp's columns, rows lane + 32*i, into registers
  float w[kColsPerWarp][RPL];
#pragma unroll
  for (int j = 0; j < kColsPerWarp; ++j)
#pragma unroll
    for (int i = 0; i < RPL; ++i) w[j][i] = sW[(lane + 32 * i) * kTilePitch + warp + 8 * j];

  // 3. reference operand: bf16(W), transposed
#pragma unroll
  for (int j = 0; j < kColsPerWarp; ++j) {
    const int64_t n = n0 + warp + 8 * j;
    if (n >= N) continue;
    __nv_bfloat16* out = Wt + n * K + k0 + lane;
#pragma unroll
    for (int i = 0; i < RPL; ++i) out[32 * i] = __float2bfloat16_rn(w[j][i]);
  }

  // 4. every candidate
  for (int c = 0; c < n_grid; ++c) {
    float s[RPL];
#pragma unroll
    for (int i = 0; i < RPL; ++i) s[i] = sS[c * G + lane + 32 * i];
    __nv_bfloat16* slot = Wt + static_cast<int64_t>(c + 1) * N * K;
#pragma unroll
    for (int j = 0; j < kColsPerWarp; ++j) {
      const int64_t n = n0 + warp + 8 * j;
      if (n >= N) continue;  // warp-uniform
      float wp[RPL];
      float mn = INFINITY, mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < RPL; ++i) {
        wp[i] = __fmul_rn(s[i], w[j][i]);
        mn = fminf(mn, wp[i]);
        mx = fmaxf(mx, wp[i]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      const QdqParams p = qdq_params(mn, mx);
      __nv_bfloat16* out = slot + n * K + k0 + lane;
#pragma unroll
      for (int i = 0; i < RPL; ++i) {
        const float q = qdq_code(wp[i], p);
        out[32 * i] = __float2bfloat16_rn(qdq_fold_back(q, p, s[i]));
      }
    }
  }
}

constexpr int kPackThreads = 128;

// One thread = 8 consecutive columns of one group (one packed int32 per row).
template <typename T, int G>
__global__ void __launch_bounds__(kPackThreads)
    pack_kernel(const T* __restrict__ W, int64_t K, int64_t N, const float* __restrict__ S,
                const int* __restrict__ best, int32_t* __restrict__ codes, __half* __restrict__ steps,
                __half* __restrict__ zeros, float* __restrict__ out_scales) {
  const int64_t g = blockIdx.y;
  const int c = *best;
  const float* s = S + static_cast<int64_t>(c) * K + g * G;
  if (blockIdx.x == 0)
    for (int r = threadIdx.x; r < G; r += kPackThreads) out_scales[g * G + r] = s[r];
  const int64_t w8 = static_cast<int64_t>(blockIdx.x) * kPackThreads + threadIdx.x;
  const int64_t words = N / 8;
  if (w8 >= words) return;

  auto load8 = [&](int64_t k, float (&v)[8]) {
    const T* src = W + k * N + w8 * 8;
    if constexpr (sizeof(T) == 2) {
      const uint4 raw = *reinterpret_cast<const uint4*>(src);
      const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = to_f32<T>(e[i]);
    } else {
      const uint4 a = *reinterpret_cast<const uint4*>(src);
      const uint4 b = *reinterpret_cast<const uint4*>(src + 4);
      const float* ea = reinterpret_cast<const float*>(&a);
      const float* eb = reinterpret_cast<const float*>(&b);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[i] = ea[i];
        v[4 + i] = eb[i];
      }
    }
  };

  float mn[8], mx[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    mn[i] = INFINITY;
    mx[i] = -INFINITY;
  }
  for (int r = 0; r < G; ++r) {
    float v[8];
    load8(g * G + r, v);
    const float sr = s[r];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float wp = __fmul_rn(sr, v[i]);
      mn[i] = fminf(mn[i], wp);
      mx[i] = fmaxf(mx[i], wp);
    }
  }
  QdqParams p[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) p[i] = qdq_params(mn[i], mx[i]);

  for (int r = 0; r < G; ++r) {
    float v[8];
    load8(g * G + r, v);
    const float sr = s[r];
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float q = qdq_code(__fmul_rn(sr, v[i]), p[i]);
      word |= static_cast<uint32_t>(q) << (4 * i);
    }
    codes[(g * G + r) * words + w8] = static_cast<int32_t>(word);
  }
  __align__(16) __half st[8];
  __align__(16) __half zr[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    st[i] = __float2half_rn(p[i].step);
    zr[i] = __float2half_rn(p[i].zero);
  }
  *reinterpret_cast<uint4*>(steps + g * N + w8 * 8) = *reinterpret_cast<const uint4*>(st);
  *reinterpret_cast<uint4*>(zeros + g * N + w8 * 8) = *reinterpret_cast<const uint4*>(zr);
}

template <typename T, int G>
cudaError_t launch_qdq_t(const T* W, int64_t K, int64_t N, int n_grid, const float* S, __nv_bfloat16* Wt,
                         int* err, cudaStream_t s) {
  const size_t smem = (static_cast<size_t>(G) * kTilePitch + static_cast<size_t>(n_grid) * G) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(qdq_kernel<T, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(ceil_div(N, kQdqCols)), static_cast<unsigned>(K / G));
  qdq_kernel<T, G><<<grid, kQdqThreads, smem, s>>>(W, K, N, n_grid, S, Wt, err);
  return cudaGetLastError();
}

template <typename T, int G>
cudaError_t launch_pack_t(const T* W, int64_t K, int64_t N, const float* S, const int* best, int32_t* codes,
                          __half* steps, __half* zeros, float* out_scales, cudaStream_t s) {
  dim3 grid(static_cast<unsigned>(std::max<int64_t>(1, ceil_div(N / 8, kPackThreads))),
            static_cast<unsigned>(K / G));
  pack_kernel<T, G><<<grid, kPackThreads, 0, s>>>(W, K, N, S, best, codes, steps, zeros, out_scales);
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

cudaError_t launch_pack(const void* W, int in_dtype, int64_t K, int64_t N, int group, const float* S,
                        const int* best, int32_t* codes, __half* steps, __half* zeros, float* out_scales,
                        cudaStream_t s, int* launches) {
  *launches += 1;
  if (in_dtype == 0) {
    const auto* w = static_cast<const __nv_bfloat16*>(W);
    switch (group) {
      case 32: return launch_pack_t<__nv_bfloat16, 32>(w, K, N, S, best, codes, steps, zeros, out_scales, s);
      case 64: return launch_pack_t<__nv_bfloat16, 64>(w, K, N, S, best, codes, steps, zeros, out_scales, s);
      default: return launch_pack_t<__nv_bfloat16, 128>(w, K, N, S, best, codes, steps, zeros, out_scales, s);
    }
  }
  const auto* w = static_cast<const float*>(W);
  switch (group) {
    case 32: return launch_pack_t<float, 32>(w, K, N, S, best, codes, steps, zeros, out_scales, s);
    case 64: return launch_pack_t<float, 64>(w, K, N, S, best, codes, steps, zeros, out_scales, s);
    default: return launch_pack_t<float, 128>(w, K, N, S, best, codes, steps, zeros, out_scales, s);
  }
}

}  // namespace awq
