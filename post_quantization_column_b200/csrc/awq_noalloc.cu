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
// The search itself is the one awq_search_ex runs (same argument checks, same
// kernels, same launch sequence, same work-space layout): this file only hands it the
// array instead of a block from the library's pool. A search given a fixed work space
// also reads its status word back into pageable host memory and records no profiling
// events, so nothing at all is allocated.
//
// The array is a file-scope __device__ variable. CUDA loads a module's device
// variables when the module is first used, so a GPU materialises the array on the
// first call made on it (which fails with AWQ_ERR_CUDA if that GPU has no room left
// for it); from then on the GPU holds AWQ_NOALLOC_SCRATCH_BYTES of it until the
// process exits. Host code cannot use the array's name as a device address, so the
// first call on each device looks the address up with cudaGetSymbolAddress (with that
// device current) and keeps it. All calls share the array and it keeps the previous
// call's contents: the status word and the per-tile flags are cleared at the start of
// every call and every other piece is overwritten before it is read. Two calls that
// overlap on the GPU (different streams, or different host threads on one device) race
// on the array and must be serialised by the caller.
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

// Once per device, with that device current (the search makes the call's device current
// before it asks): the device address of the array.
int scratch_address(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices) {
    record_error_message("device ordinal out of range for the fixed work space");
    return AWQ_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      record_error_message((std::string("cudaGetSymbolAddress of the fixed work space: ") + cudaGetErrorString(e))
                               .c_str());
      return AWQ_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return AWQ_OK;
}

}  // namespace

extern "C" int awq_search_noalloc(const void* X, const void* W, int in_dtype, int64_t M, int64_t K, int64_t N,
                                  int group, int n_grid, float* out_scales, int32_t* out_codes, void* out_steps,
                                  void* out_zeros, float* out_losses, int32_t* out_best, awq_stream_t stream) {
  const FixedWorkspace fixed{static_cast<size_t>(AWQ_NOALLOC_SCRATCH_BYTES), &scratch_address};
  return search_in_workspace(X, W, in_dtype, M, K, N, group, n_grid, out_scales, out_codes, out_steps, out_zeros,
                             out_losses, out_best, reinterpret_cast<cudaStream_t>(stream), fixed);
}
