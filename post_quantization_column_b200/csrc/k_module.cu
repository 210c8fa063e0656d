// k_module.cu — pieces of the module-level objective for an MLP block ("AWQ：为什么 4-bit
// 权重量化要先观察 Activation" §4: a candidate may be scored on the output of the whole
// module it belongs to; here down(silu(X W_gate) * (X W_up)) with the gate and up
// projections searched jointly and the down projection kept as it is).
//
// silu_mul_kernel: the elementwise middle of the block. It reads the fp32 output of the
// first GEMM (the gate half and the up half of each row) and writes the bf16 operand of
// the second GEMM, h = bf16(fl32(silu(g) * u)), silu(g) = g / (1 + exp(-g)) in fp32.
// HBM-bound: 8 bytes read and 2 written per element of h.
//
// transpose_bf16_kernel: the down projection W (F x K_out) as the K-major operand
// Wt (K_out x F) of the second GEMM, through 32 x 32 shared-memory tiles.
#include "awq_device.cuh"
#include "awq_kernels.h"

namespace awq {
namespace {

constexpr int kActThreads = 256;

__global__ void __launch_bounds__(kActThreads)
    silu_mul_kernel(const float4* __restrict__ H, int64_t M, int64_t F4, uint2* __restrict__ h) {
  // F4 = F / 4: four consecutive columns per thread (16-byte loads of each half)
  const int64_t total = M * F4;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = i / F4, f = i % F4;
    const float4 g = __ldcs(H + m * 2 * F4 + f);
    const float4 u = __ldcs(H + m * 2 * F4 + F4 + f);
    float v[4] = {g.x, g.y, g.z, g.w};
    const float w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = silu_mul_f32(v[j], w[j]);
    const __nv_bfloat162 lo = __floats2bfloat162_rn(v[0], v[1]);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(v[2], v[3]);
    uint2 o;
    o.x = *reinterpret_cast<const uint32_t*>(&lo);
    o.y = *reinterpret_cast<const uint32_t*>(&hi);
    h[i] = o;
  }
}

template <typename T>
__global__ void transpose_bf16_kernel(const T* __restrict__ W, int64_t rows, int64_t cols,
                                      __nv_bfloat16* __restrict__ Wt) {
  __shared__ float tile[32][33];
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * 32, c0 = static_cast<int64_t>(blockIdx.x) * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int64_t r = r0 + i, c = c0 + threadIdx.x;
    tile[i][threadIdx.x] = (r < rows && c < cols) ? to_f32<T>(W[r * cols + c]) : 0.0f;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int64_t c = c0 + i, r = r0 + threadIdx.x;  // output row c, column r
    if (c < cols && r < rows) Wt[c * rows + r] = __float2bfloat16_rn(tile[threadIdx.x][i]);
  }
}

}  // namespace

cudaError_t launch_silu_mul(const float* H, int64_t M, int64_t F, __nv_bfloat16* h, cudaStream_t s, int* launches) {
  // F % 8 == 0 and both buffers 16-byte aligned
  const int64_t F4 = F / 4;
  const unsigned blocks = static_cast<unsigned>(std::min<int64_t>(ceil_div(M * F4, kActThreads), 148 * 16));
  silu_mul_kernel<<<blocks, kActThreads, 0, s>>>(reinterpret_cast<const float4*>(H), M, F4,
                                                  reinterpret_cast<uint2*>(h));
  *launches += 1;
  return cudaGetLastError();
}

cudaError_t launch_transpose_bf16(const void* W, int in_dtype, int64_t rows, int64_t cols, __nv_bfloat16* Wt,
                                  cudaStream_t s, int* launches) {
  dim3 grid(static_cast<unsigned>(ceil_div(cols, 32)), static_cast<unsigned>(ceil_div(rows, 32)));
  dim3 block(32, 8);
  if (in_dtype == 0)
    transpose_bf16_kernel<__nv_bfloat16><<<grid, block, 0, s>>>(static_cast<const __nv_bfloat16*>(W), rows, cols, Wt);
  else
    transpose_bf16_kernel<float><<<grid, block, 0, s>>>(static_cast<const float*>(W), rows, cols, Wt);
  *launches += 1;
  return cudaGetLastError();
}

}  // namespace awq
