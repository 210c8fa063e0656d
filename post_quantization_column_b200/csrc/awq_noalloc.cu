// awq_noalloc.cu — awq_search_noalloc: the same search for callers that must not
// allocate device memory.
//
// Who needs it: code that runs where cudaMalloc / cudaMallocAsync are off limits —
// an engine or plugin whose host framework owns every byte of device memory and
// forbids allocations behind its back, a process with a hard memory budget that was
// fixed at start-up, or a latency-critical loop that cannot risk an allocation's
// implicit synchronisation or failure in the middle of a run. Such a caller passes
// its inputs and outputs as usual; the library supplies the work space from one
// fixed-size array compiled into this file.
//
// The array is a file-scope __device__ variable: every GPU that loads the library
// holds AWQ_NOALLOC_SCRATCH_BYTES of it until the process exits. Host code cannot
// use the array's name as a device address, so the first call on each device looks
// the address up with cudaGetSymbolAddress (with that device current) and keeps it.
// All calls share the array and it keeps the previous call's contents: the status
// word is cleared at the start of every call and every other piece is overwritten
// before it is read. Two calls that overlap on the GPU (different streams, or
// different host threads on one device) race on the array and must be serialised by
// the caller. Nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include "../../include/awq_search.h"
#include "awq_device.cuh"
#include "awq_kernels.h"

#include <mutex>
#include <string>

namespace {

using namespace awq;

static __device__ __align__(256) unsigned char g_noalloc_scratch[AWQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// The message awq_last_error_message reports for this thread.
int noalloc_fail(int status, const std::string& msg) {
  record_error_message(msg.c_str());
  return status;
}

// Once per device, with that device current: the device address of the array.
int scratch_address(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return noalloc_fail(AWQ_ERR_CUDA, "device ordinal out of range");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return noalloc_fail(AWQ_ERR_CUDA, std::string("cudaGetSymbolAddress of the scratch array: ") +
                                            cudaGetErrorString(e));
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return AWQ_OK;
}

bool on_device(const void* p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
}

}  // namespace

extern "C" int awq_search_noalloc(const void* X, const void* W, int in_dtype, int64_t M, int64_t K, int64_t N,
                                  int group, int n_grid, float* out_scales, int32_t* out_codes, void* out_steps,
                                  void* out_zeros, float* out_losses, awq_stream_t stream) {
  record_error_message("");
  if (!X || !W || !out_scales || !out_codes || !out_steps || !out_zeros)
    return noalloc_fail(AWQ_ERR_INVALID_ARG, "a required pointer is NULL");
  if (in_dtype != AWQ_DTYPE_BF16 && in_dtype != AWQ_DTYPE_F32)
    return noalloc_fail(AWQ_ERR_INVALID_ARG, "in_dtype must be AWQ_DTYPE_BF16 or AWQ_DTYPE_F32");
  if (group != 32 && group != 64 && group != 128)
    return noalloc_fail(AWQ_ERR_INVALID_ARG, "group must be 32, 64 or 128");
  if (n_grid < 1 || n_grid > 64) return noalloc_fail(AWQ_ERR_INVALID_ARG, "n_grid must be in 1..64");
  if (M <= 0 || K <= 0 || N <= 0 || M >= (int64_t(1) << 31) || K >= (int64_t(1) << 31) || N >= (int64_t(1) << 31))
    return noalloc_fail(AWQ_ERR_SHAPE, "M, K and N must be in 1 .. 2^31-1");
  if (K % group || K / group > 65535) return noalloc_fail(AWQ_ERR_SHAPE, "group must divide K (K/group <= 65535)");
  if (N % 8) return noalloc_fail(AWQ_ERR_SHAPE, "N must be a multiple of 8");
  for (const void* p : {X, W, static_cast<const void*>(out_scales), static_cast<const void*>(out_codes),
                        static_cast<const void*>(out_steps), static_cast<const void*>(out_zeros)})
    if (reinterpret_cast<uintptr_t>(p) & 15u)
      return noalloc_fail(AWQ_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int dev = -1;
  if (s != nullptr && cudaStreamGetDevice(s, &dev) != cudaSuccess) {
    cudaGetLastError();
    dev = -1;
  }
  if (dev < 0) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, X) == cudaSuccess && at.type == cudaMemoryTypeDevice)
      dev = at.device;
    else
      cudaGetLastError();
  }
  if (dev >= 0) cudaSetDevice(dev);
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return noalloc_fail(AWQ_ERR_CUDA, "cudaGetDevice");
  int major = 0, minor = 0, num_sms = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
  if (major != 10 || minor != 0) return noalloc_fail(AWQ_ERR_UNSUPPORTED_DEVICE, "needs an sm_100 device");
  if (!on_device(X) || !on_device(W) || !on_device(out_scales) || !on_device(out_codes) || !on_device(out_steps) ||
      !on_device(out_zeros) || (out_losses && !on_device(out_losses)))
    return noalloc_fail(AWQ_ERR_INVALID_ARG, "inputs and outputs must be device memory");

  // carve the work space out of the fixed array (same pieces as the pooled entry points)
  const int64_t tiles = ceil_div(M, kTileM) * ceil_div(N, kTileN);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += round256(bytes);
    return at;
  };
  const size_t o_err = take(16), o_a = take(size_t(K) * 4),
               o_S = take(size_t(n_grid) * K * 4), o_best = take(16), o_loss = take(size_t(n_grid) * 4),
               o_Xb = in_dtype == AWQ_DTYPE_F32 ? take(size_t(M) * K * 2) : 0,
               o_Wt = take(size_t(n_grid + 1) * N * K * 2), o_Y = take(size_t(tiles) * kTileM * kTileN * 4),
               o_lp = take(size_t(n_grid) * tiles * 8);
  if (off > static_cast<size_t>(AWQ_NOALLOC_SCRATCH_BYTES))
    return noalloc_fail(AWQ_ERR_SHAPE, "this layer needs " + std::to_string(off) +
                                           " bytes of work space; awq_search_noalloc has " +
                                           std::to_string(static_cast<long long>(AWQ_NOALLOC_SCRATCH_BYTES)) +
                                           " (use awq_search for larger layers)");

  void* scratch = nullptr;
  int st = scratch_address(dev, &scratch);
  if (st != AWQ_OK) return st;
  uint8_t* base = static_cast<uint8_t*>(scratch);
  int* err = reinterpret_cast<int*>(base + o_err);
  float* a = reinterpret_cast<float*>(base + o_a);
  float* S = reinterpret_cast<float*>(base + o_S);
  int* best = reinterpret_cast<int*>(base + o_best);
  float* losses = reinterpret_cast<float*>(base + o_loss);
  __nv_bfloat16* Wt = reinterpret_cast<__nv_bfloat16*>(base + o_Wt);
  float* Y = reinterpret_cast<float*>(base + o_Y);
  double* loss_partial = reinterpret_cast<double*>(base + o_lp);
  __nv_bfloat16* Xb = in_dtype == AWQ_DTYPE_F32 ? reinterpret_cast<__nv_bfloat16*>(base + o_Xb)
                                                : const_cast<__nv_bfloat16*>(static_cast<const __nv_bfloat16*>(X));

  int launches = 0;
  const char* where = "";
  do {
    if ((e = cudaMemsetAsync(err, 0, 16, s)) != cudaSuccess) { where = "clearing the status word"; break; }
    if ((e = launch_statistic(X, in_dtype, M, K, a, err, s, &launches)) != cudaSuccess) {
      where = "statistic kernel";
      break;
    }
    if ((e = launch_scales(a, K, n_grid, S, s, &launches)) != cudaSuccess) { where = "scales kernel"; break; }
    if (in_dtype == AWQ_DTYPE_F32 &&
        (e = launch_to_bf16(static_cast<const float*>(X), M * K, Xb, s, &launches)) != cudaSuccess) {
      where = "bf16 operand kernel";
      break;
    }
    if ((e = launch_qdq(W, in_dtype, K, N, group, n_grid, S, Wt, err, s, &launches)) != cudaSuccess) {
      where = "qdq kernel";
      break;
    }
    LossGemmArgs ga;
    ga.Xb = Xb;
    ga.Wt = Wt;
    ga.M = M;
    ga.K = K;
    ga.N = N;
    ga.n_grid = n_grid;
    ga.Y = Y;
    ga.partial = loss_partial;
    ga.err = err;
    ga.timeout_ns = 2000ull * 1000 * 1000;
    ga.fault_mode = 0;
    ga.num_sms = num_sms;
    ga.variant = gemm_variant(M, K, N, n_grid);
    CUtensorMap mapA, mapB;
    const char* why = "";
    if ((e = make_operand_maps(ga, &mapA, &mapB, &why, operand_b_box_rows(ga.variant))) != cudaSuccess) { where = why; break; }
    if ((e = launch_loss_gemm(ga, mapA, mapB, 0, s, &launches)) != cudaSuccess) { where = "reference GEMM"; break; }
    if ((e = launch_loss_gemm(ga, mapA, mapB, 1, s, &launches)) != cudaSuccess) { where = "loss GEMM"; break; }
    if ((e = launch_loss_reduce(loss_partial, tiles, n_grid, M, N, losses, s, &launches)) != cudaSuccess) {
      where = "loss reduction kernel";
      break;
    }
    if ((e = launch_pack(W, in_dtype, K, N, group, n_grid, S, losses, best, out_codes, static_cast<__half*>(out_steps),
                         static_cast<__half*>(out_zeros), out_scales, s, &launches)) != cudaSuccess) {
      where = "pack kernel";
      break;
    }
    if (out_losses &&
        (e = cudaMemcpyAsync(out_losses, losses, size_t(n_grid) * 4, cudaMemcpyDeviceToDevice, s)) != cudaSuccess) {
      where = "copy of the losses";
      break;
    }
  } while (false);
  int h_err = 0;
  if (e == cudaSuccess) {
    e = cudaMemcpyAsync(&h_err, err, sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) where = "status read-back";
  }
  cudaError_t se = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return noalloc_fail(AWQ_ERR_CUDA, std::string(where) + ": " + cudaGetErrorString(e));
  if (se != cudaSuccess) return noalloc_fail(AWQ_ERR_CUDA, std::string("stream synchronize: ") + cudaGetErrorString(se));
  if (h_err & kErrTimeout) return noalloc_fail(AWQ_ERR_TIMEOUT, "a bounded wait in the loss GEMM ran out");
  if (h_err & (kErrNonfiniteX | kErrNonfiniteW)) return noalloc_fail(AWQ_ERR_NONFINITE, "non-finite value in X or W");
  if (h_err) return noalloc_fail(AWQ_ERR_CUDA, "device status word " + std::to_string(h_err));
  return AWQ_OK;
}
