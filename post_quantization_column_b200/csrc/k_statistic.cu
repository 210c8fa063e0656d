// k_statistic.cu — the activation statistic a_j = mean_m |X[m, j]| ("AWQ：为什么 4-bit
// 权重量化要先观察 Activation" §1; "AWQ salient weight / GGUF compilation" §二), the
// candidate scale family (same AWQ page, §3 code and §4) and the fp32 -> bf16 operand
// copy for fp32 layers.
//
// The statistic is one coalesced pass over X: each thread owns a 16-byte column
// vector and walks rows, accumulating |x| in fp64; a second tiny pass adds the
// per-chunk partial sums in a fixed order and rounds once to fp32. HBM-bound: M*K*b
// bytes read.
#include "awq_device.cuh"
#include "awq_kernels.h"

namespace awq {
namespace {

constexpr int kStatCols = 64;  // column vectors per block
constexpr int kStatRows = 4;   // row lanes per block

template <typename T>
__global__ void __launch_bounds__(kStatCols * kStatRows)
    statistic_partial_kernel(const T* __restrict__ X, int64_t M, int64_t K, int64_t rows_per_chunk,
                             double* __restrict__ partial) {
  constexpr int VEC = 16 / sizeof(T);
  const int tx = threadIdx.x % kStatCols;
  const int ty = threadIdx.x / kStatCols;
  const int64_t c0 = (static_cast<int64_t>(blockIdx.x) * kStatCols + tx) * VEC;
  const int64_t r_begin = static_cast<int64_t>(blockIdx.y) * rows_per_chunk;
  const int64_t r_end = min(M, r_begin + rows_per_chunk);

  double acc[VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) acc[i] = 0.0;
  if (c0 < K) {
    const T* base = X + c0;
#pragma unroll 4
    for (int64_t r = r_begin + ty; r < r_end; r += kStatRows) {
      const uint4 raw = __ldcs(reinterpret_cast<const uint4*>(base + r * K));
      const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
      for (int i = 0; i < VEC; ++i) acc[i] += fabs(static_cast<double>(to_f32<T>(e[i])));
    }
  }
  __shared__ double red[kStatRows][kStatCols][VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) red[ty][tx][i] = acc[i];
  __syncthreads();
  if (ty == 0 && c0 < K) {
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
      double s = red[0][tx][i];
#pragma unroll
      for (int r = 1; r < kStatRows; ++r) s += red[r][tx][i];
      partial[static_cast<int64_t>(blockIdx.y) * K + c0 + i] = s;
    }
  }
}

__global__ void statistic_final_kernel(const double* __restrict__ partial, int row_chunks, int64_t K,
                                       int64_t M, float* __restrict__ a, int* err) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= K) return;
  double s = 0.0;
  for (int r = 0; r < row_chunks; ++r) s += partial[static_cast<int64_t>(r) * K + j];
  if (!isfinite(s)) atomicOr(err, kErrNonfiniteX);  // NaN/Inf anywhere in the column
  a[j] = __double2float_rn(s / static_cast<double>(M));
}

// One block per candidate i: alpha = i / n_grid; raw_j = max(a_j^alpha, 1e-4);
// s_j = raw_j / sqrt(max raw * min raw), in fp64, one rounding to fp32.
constexpr int kScaleThreads = 1024;

__global__ void __launch_bounds__(kScaleThreads)
    scales_kernel(const float* __restrict__ a, int64_t K, int n_grid, float* __restrict__ S) {
  const int i = blockIdx.x;
  const double alpha = static_cast<double>(i) / static_cast<double>(n_grid);
  double mx = 0.0, mn = INFINITY;
  for (int64_t j = threadIdx.x; j < K; j += blockDim.x) {
    const double raw = fmax(pow(static_cast<double>(a[j]), alpha), kClampMin);
    mx = fmax(mx, raw);
    mn = fmin(mn, raw);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    mn = fmin(mn, __shfl_xor_sync(0xffffffffu, mn, o));
  }
  __shared__ double smx[kScaleThreads / 32], smn[kScaleThreads / 32];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (lane == 0) {
    smx[warp] = mx;
    smn[warp] = mn;
  }
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x / 32;
    mx = lane < nw ? smx[lane] : 0.0;
    mn = lane < nw ? smn[lane] : INFINITY;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      mn = fmin(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    }
    if (lane == 0) {
      smx[0] = mx;
      smn[0] = mn;
    }
  }
  __syncthreads();
  const double normaliser = sqrt(__dmul_rn(smx[0], smn[0]));
  for (int64_t j = threadIdx.x; j < K; j += blockDim.x) {
    const double raw = fmax(pow(static_cast<double>(a[j]), alpha), kClampMin);
    S[static_cast<int64_t>(i) * K + j] = __double2float_rn(__ddiv_rn(raw, normaliser));
  }
}

__global__ void to_bf16_kernel(const float4* __restrict__ x, int64_t n4, uint2* __restrict__ out) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 v = __ldcs(x + i);
    __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(v.z, v.w);
    uint2 o;
    o.x = *reinterpret_cast<uint32_t*>(&lo);
    o.y = *reinterpret_cast<uint32_t*>(&hi);
    out[i] = o;
  }
}

}  // namespace

int statistic_row_chunks(int64_t M, int64_t K, int in_dtype, int num_sms) {
  const int vec = in_dtype == 0 ? 8 : 4;
  const int64_t col_blocks = ceil_div(K, static_cast<int64_t>(kStatCols) * vec);
  int64_t want = ceil_div(static_cast<int64_t>(num_sms) * 4, col_blocks);
  // at least 16 rows per chunk, at most 65535 chunks
  want = std::min<int64_t>(want, std::max<int64_t>(1, M / 16));
  want = std::min<int64_t>(want, 65535);
  return static_cast<int>(std::max<int64_t>(1, want));
}

cudaError_t launch_statistic(const void* X, int in_dtype, int64_t M, int64_t K, int row_chunks,
                             double* partial, float* a, int* err, cudaStream_t s, int* launches) {
  const int vec = in_dtype == 0 ? 8 : 4;
  const int64_t rows_per_chunk = ceil_div(M, row_chunks);
  dim3 grid(static_cast<unsigned>(ceil_div(K, static_cast<int64_t>(kStatCols) * vec)),
            static_cast<unsigned>(row_chunks));
  if (in_dtype == 0)
    statistic_partial_kernel<__nv_bfloat16><<<grid, kStatCols * kStatRows, 0, s>>>(
        static_cast<const __nv_bfloat16*>(X), M, K, rows_per_chunk, partial);
  else
    statistic_partial_kernel<float><<<grid, kStatCols * kStatRows, 0, s>>>(static_cast<const float*>(X), M, K,
                                                                           rows_per_chunk, partial);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  statistic_final_kernel<<<static_cast<unsigned>(ceil_div(K, 256)), 256, 0, s>>>(partial, row_chunks, K, M, a,
                                                                                 err);
  *launches += 2;
  return cudaGetLastError();
}

cudaError_t launch_scales(const float* a, int64_t K, int n_grid, float* S, cudaStream_t s, int* launches) {
  scales_kernel<<<n_grid, kScaleThreads, 0, s>>>(a, K, n_grid, S);
  *launches += 1;
  return cudaGetLastError();
}

cudaError_t launch_to_bf16(const float* x, int64_t n, __nv_bfloat16* out, cudaStream_t s, int* launches) {
  // n is a multiple of 4 (K % 32 == 0) and both buffers are 16-byte aligned
  const int64_t n4 = n / 4;
  const unsigned blocks = static_cast<unsigned>(std::min<int64_t>(ceil_div(n4, 256), 148 * 16));
  to_bf16_kernel<<<blocks, 256, 0, s>>>(reinterpret_cast<const float4*>(x), n4, reinterpret_cast<uint2*>(out));
  *launches += 1;
  return cudaGetLastError();
}

}  // namespace awq
