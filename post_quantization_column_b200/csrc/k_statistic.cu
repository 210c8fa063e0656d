// k_statistic.cu — the activation statistic a_j = mean_m |X[m, j]| ("AWQ：为什么 4-bit
// 权重量化要先观察 Activation" §1; "AWQ salient weight / GGUF compilation" §二), the
// candidate scale family (same AWQ page, §3 code and §4) and the fp32 -> bf16 operand
// copy for fp32 layers.
//
// Both reductions run as one launch of 8-CTA thread-block clusters and combine their
// partial results through distributed shared memory in a fixed order, so they need no
// global scratch and no second pass:
//  * statistic: a cluster owns 8 or 16 16-byte column vectors (64 or 128 bf16 columns,
//    32 or 64 fp32 ones; the wider form once the narrow grid would exceed a wave of
//    resident CTAs); its 8 CTAs split the rows, each thread walks rows with one column
//    vector, 8 loads in flight (fp64 accumulation), the CTA sums its row-threads, and
//    CTA rank 0 sums the 8 CTAs' partials, divides by M once in fp64 and rounds once to
//    fp32. HBM-bound: one read of X in 128- or 256-byte row segments.
//  * scales: a cluster owns one candidate alpha_i; its 8 CTAs split K, exchange their
//    max/min of raw = max(a^alpha, 1e-4) and each normalises its share by
//    sqrt(max * min) — fp64 throughout, one rounding to fp32.
#include "awq_device.cuh"
#include "awq_kernels.h"

#include <cooperative_groups.h>

namespace cg = cooperative_groups;

namespace awq {
namespace {

constexpr int kCluster = 8;       // CTAs per cluster (portable size)
constexpr int kStatThreads = 256;
constexpr int kStatBatch = 8;     // row loads in flight per thread
constexpr int kStatCtasPerSm = 4;  // resident statistic CTAs per SM (registers)

// VECS 16-byte column vectors per CTA: a warp reads 32 / VECS rows of 16 VECS bytes.
template <typename T, int VECS>
__global__ void __cluster_dims__(1, kCluster, 1) __launch_bounds__(kStatThreads)
    statistic_kernel(const T* __restrict__ X, int64_t M, int64_t K, float* __restrict__ a, int* err) {
  constexpr int VEC = 16 / sizeof(T);
  constexpr int kStatVecs = VECS;
  constexpr int kStatRows = kStatThreads / VECS;  // row-threads per column vector
  constexpr int kCols = kStatVecs * VEC;  // columns per cluster
  __shared__ double red[kStatRows][kStatVecs][VEC];
  __shared__ double part[kCols];          // this CTA's column sums, read by rank 0

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int tx = threadIdx.x % kStatVecs, ty = threadIdx.x / kStatVecs;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kCols + static_cast<int64_t>(tx) * VEC;

  double acc[VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) acc[i] = 0.0;
  if (c0 < K) {  // K % 32 == 0, so a vector lies wholly inside or outside
    // Rows r0, r0 + stride, ... in that order; kStatBatch loads are issued before any is
    // used, so a thread waits for one DRAM round trip per batch, not per row.
    const T* base = X + c0;
    const int64_t stride = static_cast<int64_t>(kStatRows) * kCluster;
    auto add = [&](const uint4& raw) {
      const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
      for (int i = 0; i < VEC; ++i) acc[i] += fabs(static_cast<double>(to_f32<T>(e[i])));
    };
    int64_t r = static_cast<int64_t>(rank) * kStatRows + ty;
    for (; r + (kStatBatch - 1) * stride < M; r += stride * kStatBatch) {
      uint4 raw[kStatBatch];
#pragma unroll
      for (int b = 0; b < kStatBatch; ++b) raw[b] = __ldcs(reinterpret_cast<const uint4*>(base + (r + b * stride) * K));
#pragma unroll
      for (int b = 0; b < kStatBatch; ++b) add(raw[b]);
    }
    for (; r < M; r += stride) add(__ldcs(reinterpret_cast<const uint4*>(base + r * K)));
  }
#pragma unroll
  for (int i = 0; i < VEC; ++i) red[ty][tx][i] = acc[i];
  __syncthreads();
  if (ty == 0) {
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
      double s = red[0][tx][i];
#pragma unroll
      for (int r = 1; r < kStatRows; ++r) s += red[r][tx][i];
      part[tx * VEC + i] = s;
    }
  }
  cluster.sync();
  if (rank == 0) {
    for (int j = threadIdx.x; j < kCols; j += kStatThreads) {
      const int64_t col = static_cast<int64_t>(blockIdx.x) * kCols + j;
      if (col >= K) continue;
      double s = 0.0;
      for (int q = 0; q < kCluster; ++q) s += cluster.map_shared_rank(part, q)[j];
      if (!isfinite(s)) atomicOr(err, kErrNonfiniteX);  // NaN/Inf anywhere in the column
      a[col] = __double2float_rn(s / static_cast<double>(M));
    }
  }
  cluster.sync();  // keep every CTA's partials alive until rank 0 has read them
}

constexpr int kScaleThreads = 256;

__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kScaleThreads)
    scales_kernel(const float* __restrict__ a, int64_t K, int n_grid, float* __restrict__ S) {
  __shared__ double smx[kScaleThreads / 32], smn[kScaleThreads / 32];
  __shared__ double cta_range[2];  // this CTA's max and min of raw, read by the cluster

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int i = blockIdx.y;  // candidate
  const double alpha = static_cast<double>(i) / static_cast<double>(n_grid);
  const int64_t share = ceil_div(K, kCluster);
  const int64_t j0 = rank * share, j1 = min(K, j0 + share);

  double mx = 0.0, mn = INFINITY;
  for (int64_t j = j0 + threadIdx.x; j < j1; j += kScaleThreads) {
    const double raw = fmax(pow(static_cast<double>(a[j]), alpha), kClampMin);
    mx = fmax(mx, raw);
    mn = fmin(mn, raw);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    mn = fmin(mn, __shfl_xor_sync(0xffffffffu, mn, o));
  }
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (lane == 0) {
    smx[warp] = mx;
    smn[warp] = mn;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kScaleThreads / 32; ++w) {
      mx = fmax(mx, smx[w]);
      mn = fmin(mn, smn[w]);
    }
    cta_range[0] = mx;
    cta_range[1] = mn;
  }
  cluster.sync();
  double gmx = 0.0, gmn = INFINITY;
  for (int q = 0; q < kCluster; ++q) {
    const double* r = cluster.map_shared_rank(cta_range, q);
    gmx = fmax(gmx, r[0]);
    gmn = fmin(gmn, r[1]);
  }
  cluster.sync();  // every CTA has read every range before any CTA exits
  const double normaliser = sqrt(__dmul_rn(gmx, gmn));
  for (int64_t j = j0 + threadIdx.x; j < j1; j += kScaleThreads) {
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

cudaError_t launch_statistic(const void* X, int in_dtype, int64_t M, int64_t K, float* a, int* err, cudaStream_t s,
                             int* launches) {
  // Clusters of 8 column vectors (64 bf16 / 32 fp32 columns, 128-byte row segments) while
  // they fit in one wave of resident CTAs; wider clusters of 16 vectors (256-byte
  // segments) for larger K, which halves the CTAs and keeps the grid to about one wave.
  int dev = 0, num_sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int vec = in_dtype == 0 ? 8 : 4;
  const bool wide = ceil_div(K, static_cast<int64_t>(8 * vec)) * kCluster > static_cast<int64_t>(kStatCtasPerSm) * num_sms;
  const int vecs = wide ? 16 : 8;
  dim3 grid(static_cast<unsigned>(ceil_div(K, static_cast<int64_t>(vecs) * vec)), kCluster);
  if (in_dtype == 0) {
    const auto* x = static_cast<const __nv_bfloat16*>(X);
    if (wide)
      statistic_kernel<__nv_bfloat16, 16><<<grid, kStatThreads, 0, s>>>(x, M, K, a, err);
    else
      statistic_kernel<__nv_bfloat16, 8><<<grid, kStatThreads, 0, s>>>(x, M, K, a, err);
  } else {
    const auto* x = static_cast<const float*>(X);
    if (wide)
      statistic_kernel<float, 16><<<grid, kStatThreads, 0, s>>>(x, M, K, a, err);
    else
      statistic_kernel<float, 8><<<grid, kStatThreads, 0, s>>>(x, M, K, a, err);
  }
  *launches += 1;
  return cudaGetLastError();
}

cudaError_t launch_scales(const float* a, int64_t K, int n_grid, float* S, cudaStream_t s, int* launches) {
  scales_kernel<<<dim3(kCluster, n_grid), kScaleThreads, 0, s>>>(a, K, n_grid, S);
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
