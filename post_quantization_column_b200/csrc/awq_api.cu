// awq_api.cu — the C ABI of libawqsearch.so (declared in include/awq_search.h).
//
// Validates the call, carves the device work space from a library-owned
// stream-ordered memory pool, enqueues the search kernels on the caller's stream in
// the order of "AWQ：为什么 4-bit 权重量化要先观察 Activation" §4 (statistic -> scales ->
// QDQ of every candidate -> loss GEMM -> argmin) and §7 (artifact), synchronizes the
// stream and turns the kernels' device status word into an awq_status.
#include "../../include/awq_search.h"
#include "awq_device.cuh"
#include "awq_kernels.h"

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <unordered_map>

namespace {

using namespace awq;

constexpr int kVersion = 1;
constexpr int kMaxGrid = 64;
constexpr int kMaxShrink = 20;  // factor 1 - i/20 stays positive for i < 20
constexpr uint64_t kDefaultTimeoutNs = 2000ull * 1000 * 1000;

enum Phase { kPhStatistic, kPhScales, kPhConvert, kPhQdq, kPhGemmY, kPhGemmLoss, kPhReduce, kPhPack, kNumPhases };
const char* kPhaseNames[kNumPhases] = {"statistic", "scales", "to_bf16", "qdq",
                                       "gemm_reference", "gemm_loss", "loss_reduce", "pack"};

thread_local std::string t_last_error;
std::mutex g_mu;
std::unordered_map<int, cudaMemPool_t> g_pools;
bool g_profile = false;
float g_phase_ms[kNumPhases] = {0};
int g_last_launches = 0;
int g_fault_mode = 0;
uint64_t g_timeout_ns = kDefaultTimeoutNs;

int set_error(int status, const std::string& msg) {
  t_last_error = msg;
  return status;
}

int cuda_error(cudaError_t e, const char* where) {
  return set_error(AWQ_ERR_CUDA, std::string(where) + ": " + cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t x, size_t a = 256) { return (x + a - 1) / a * a; }

int get_pool(int dev, cudaMemPool_t* out) {
  std::lock_guard<std::mutex> lock(g_mu);
  auto it = g_pools.find(dev);
  if (it != g_pools.end()) {
    *out = it->second;
    return AWQ_OK;
  }
  cudaMemPoolProps props;
  std::memset(&props, 0, sizeof(props));
  props.allocType = cudaMemAllocationTypePinned;
  props.handleTypes = cudaMemHandleTypeNone;
  props.location.type = cudaMemLocationTypeDevice;
  props.location.id = dev;
  cudaMemPool_t pool;
  cudaError_t e = cudaMemPoolCreate(&pool, &props);
  if (e != cudaSuccess) return cuda_error(e, "cudaMemPoolCreate");
  uint64_t keep = UINT64_MAX;  // keep freed blocks for the next call
  e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
  if (e != cudaSuccess) return cuda_error(e, "cudaMemPoolSetAttribute");
  g_pools[dev] = pool;
  *out = pool;
  return AWQ_OK;
}

struct Layout {
  size_t err, a, S, best, losses, Xb, Wt, Y, loss_partial, total;
  int64_t tiles, tiles_n;
  size_t flag_bytes;  // the status word, the per-tile flags and the QDQ counters, zeroed per call
};

Layout plan(int in_dtype, int64_t M, int64_t K, int64_t N, int n_grid) {
  Layout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align_up(bytes);
    return at;
  };
  const int64_t tiles_m = ceil_div(M, kTileM), tiles_n = ceil_div(N, kTileN);
  L.tiles = tiles_m * tiles_n;
  L.tiles_n = tiles_n;
  // status word, then the loss GEMM's per-tile flags, then its QDQ warps' counters and
  // their claim counter
  L.flag_bytes = 16 + static_cast<size_t>(L.tiles + tiles_n + 1) * 4;
  L.err = take(L.flag_bytes);
  L.a = take(static_cast<size_t>(K) * 4);
  L.S = take(static_cast<size_t>(n_grid) * K * 4);
  L.best = take(16);
  L.losses = take(static_cast<size_t>(n_grid) * 4);
  L.Xb = in_dtype == AWQ_DTYPE_F32 ? take(static_cast<size_t>(M) * K * 2) : 0;
  L.Wt = take(static_cast<size_t>(n_grid + 1) * N * K * 2);
  L.Y = take(static_cast<size_t>(L.tiles) * kTileM * kTileN * 4);
  L.loss_partial = take(static_cast<size_t>(n_grid) * L.tiles * 8);
  L.total = off;
  return L;
}

int validate(const void* X, const void* W, int in_dtype, int64_t M, int64_t K, int64_t N, int group, int n_grid,
             const void* out_scales, const void* out_codes, const void* out_steps, const void* out_zeros,
             bool device_ptrs) {
  if (!X || !W || !out_scales || !out_codes || !out_steps || !out_zeros)
    return set_error(AWQ_ERR_INVALID_ARG, "a required pointer is NULL");
  if (in_dtype != AWQ_DTYPE_BF16 && in_dtype != AWQ_DTYPE_F32)
    return set_error(AWQ_ERR_INVALID_ARG, "in_dtype must be AWQ_DTYPE_BF16 or AWQ_DTYPE_F32");
  if (group != 32 && group != 64 && group != 128)
    return set_error(AWQ_ERR_INVALID_ARG, "group must be 32, 64 or 128");
  if (n_grid < 1 || n_grid > kMaxGrid) return set_error(AWQ_ERR_INVALID_ARG, "n_grid must be in 1..64");
  if (M <= 0 || K <= 0 || N <= 0) return set_error(AWQ_ERR_SHAPE, "M, K and N must be positive");
  if (M >= (int64_t(1) << 31) || K >= (int64_t(1) << 31) || N >= (int64_t(1) << 31))
    return set_error(AWQ_ERR_SHAPE, "M, K and N must be below 2^31");
  if (K % group) return set_error(AWQ_ERR_SHAPE, "group must divide K");
  if (K / group > 65535) return set_error(AWQ_ERR_SHAPE, "K / group must not exceed 65535");
  if (N % 8) return set_error(AWQ_ERR_SHAPE, "N must be a multiple of 8 (eight codes per int32)");
  if (device_ptrs && (!aligned16(X) || !aligned16(W) || !aligned16(out_scales) || !aligned16(out_codes) ||
                      !aligned16(out_steps) || !aligned16(out_zeros)))
    return set_error(AWQ_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  return AWQ_OK;
}

// Makes the device of `s` (or, for the legacy default stream, the device that owns
// `ptr`) current for this library's runtime, so calls from any host thread and any
// device work without a separate device-selection call.
void bind_device(cudaStream_t s, const void* ptr) {
  int dev = -1;
  if (s != nullptr && cudaStreamGetDevice(s, &dev) != cudaSuccess) {
    cudaGetLastError();
    dev = -1;
  }
  if (dev < 0 && ptr != nullptr) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, ptr) == cudaSuccess && at.type == cudaMemoryTypeDevice)
      dev = at.device;
    else
      cudaGetLastError();
  }
  if (dev >= 0) cudaSetDevice(dev);
}

bool is_device_memory(const void* p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
}

int check_device(int* dev, int* num_sms) {
  cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return cuda_error(e, "cudaGetDevice");
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, *dev);
  cudaDeviceGetAttribute(num_sms, cudaDevAttrMultiProcessorCount, *dev);
  if (major != 10 || minor != 0)
    return set_error(AWQ_ERR_UNSUPPORTED_DEVICE,
                     "this library is built for sm_100a (B200); device is sm_" + std::to_string(major * 10 + minor));
  return AWQ_OK;
}

// Phase events of profiled calls: a ring of event sets per device, created once, so
// that the times of an asynchronous call can still be read after later calls have been
// enqueued (until the ring wraps). Each profiled call takes the next set and a ticket.
constexpr int kEvRing = 256;
thread_local int64_t t_last_ticket = -1;

struct Events {
  static cudaEvent_t cache[64][kEvRing][kNumPhases + 1];
  static bool made[64];
  static int64_t next[64];
  cudaEvent_t* ev = nullptr;
  cudaStream_t s = nullptr;
  void create(bool enable, cudaStream_t stream) {
    s = stream;
    t_last_ticket = -1;  // an unprofiled call has no ticket
    if (!enable) return;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!made[dev]) {
      for (auto& set : cache[dev])
        for (auto& e : set)
          if (cudaEventCreate(&e) != cudaSuccess) return;
      made[dev] = true;
    }
    const int64_t ticket = next[dev]++;
    ev = cache[dev][ticket % kEvRing];
    t_last_ticket = ticket * 64 + dev;
  }
  void mark(int i) {
    if (ev) cudaEventRecord(ev[i], s);
  }
  void collect() {
    if (!ev) return;
    for (int i = 0; i < kNumPhases; ++i) cudaEventElapsedTime(&g_phase_ms[i], ev[i], ev[i + 1]);
  }
  // phase times of the call with this ticket, once its events have completed; false if
  // the ticket's set has been reused or its events are not complete
  static bool collect_ticket(int64_t ticket, float* ms) {
    if (ticket < 0) return false;
    const int dev = static_cast<int>(ticket % 64);
    const int64_t seq = ticket / 64;
    cudaEvent_t* set = nullptr;
    {
      std::lock_guard<std::mutex> lock(g_mu);
      if (!made[dev] || seq >= next[dev] || next[dev] - seq > kEvRing) return false;
      set = cache[dev][seq % kEvRing];
    }
    for (int i = 0; i < kNumPhases; ++i)
      if (cudaEventElapsedTime(&ms[i], set[i], set[i + 1]) != cudaSuccess) {
        cudaGetLastError();
        return false;
      }
    return true;
  }
};
cudaEvent_t Events::cache[64][kEvRing][kNumPhases + 1];
bool Events::made[64] = {false};
int64_t Events::next[64] = {0};

// A pinned host word per device for the kernels' status, so reading it back is one
// asynchronous copy followed by the stream synchronisation the call does anyway.
int* pinned_status_word(int dev) {
  static int* words[64] = {nullptr};
  if (dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!words[dev]) {
    void* p = nullptr;
    if (cudaHostAlloc(&p, 64, cudaHostAllocPortable) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    words[dev] = static_cast<int*>(p);
  }
  return words[dev];
}

// Events around the two launches of the clipping search (profiling only).
float g_clip_ms[2] = {0.0f, 0.0f};
cudaEvent_t* clip_events(int dev) {
  static cudaEvent_t ev[64][3];
  static bool made[64] = {false};
  if (dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!made[dev]) {
    for (auto& e : ev[dev])
      if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    made[dev] = true;
  }
  return ev[dev];
}

// Events around the kernels of the W4A16 consumer (profiling only).
bool g_w4a16_profiled = false;
cudaEvent_t* g_w4a16_last_ev = nullptr;
cudaEvent_t* w4a16_events(int dev) {
  static cudaEvent_t ev[64][2];
  static bool made[64] = {false};
  if (dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!made[dev]) {
    for (auto& e : ev[dev])
      if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    made[dev] = true;
  }
  g_w4a16_last_ev = ev[dev];
  return ev[dev];
}

// Per-device copy stream and events for awq_search_host, created on first use.
struct CopyLane {
  static constexpr int kChunks = 8;
  cudaStream_t stream = nullptr;
  cudaEvent_t alloc_done = nullptr, x_ready = nullptr, copies_done = nullptr;
  cudaEvent_t w_ready[kChunks] = {};
};

CopyLane* copy_lane(int dev) {
  static CopyLane lanes[64];
  static bool made[64] = {false};
  if (dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  CopyLane& L = lanes[dev];
  if (!made[dev]) {
    if (cudaStreamCreateWithFlags(&L.stream, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    bool ok = cudaEventCreateWithFlags(&L.alloc_done, cudaEventDisableTiming) == cudaSuccess &&
              cudaEventCreateWithFlags(&L.x_ready, cudaEventDisableTiming) == cudaSuccess &&
              cudaEventCreateWithFlags(&L.copies_done, cudaEventDisableTiming) == cudaSuccess;
    for (auto& ev : L.w_ready) ok = ok && cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) == cudaSuccess;
    if (!ok) return nullptr;
    made[dev] = true;
  }
  return &L;
}

// Streams, events and pinned status words of the batched host search, created once per
// device and reused; a batch holds the lane's mutex for its whole call.
struct BatchLane {
  struct Slot {
    cudaEvent_t x_ready = nullptr, in_free = nullptr, out_done = nullptr;
    cudaEvent_t w_ready[CopyLane::kChunks] = {};
  };
  std::mutex mu;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t alloc_done = nullptr, search_done = nullptr, h2d_done = nullptr, d2h_done = nullptr;
  Slot slots[2];
  int* words = nullptr;
  int words_cap = 0;
};

BatchLane* batch_lane(int dev) {
  static BatchLane lanes[64];
  static bool made[64] = {false};
  if (dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  BatchLane& L = lanes[dev];
  if (!made[dev]) {
    auto ev = [](cudaEvent_t* e) { return cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess; };
    bool ok = cudaStreamCreateWithFlags(&L.h2d, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&L.d2h, cudaStreamNonBlocking) == cudaSuccess && ev(&L.alloc_done) &&
              ev(&L.search_done) && ev(&L.h2d_done) && ev(&L.d2h_done);
    for (auto& sl : L.slots) {
      ok = ok && ev(&sl.x_ready) && ev(&sl.in_free) && ev(&sl.out_done);
      for (auto& w : sl.w_ready) ok = ok && ev(&w);
    }
    if (!ok) {
      cudaGetLastError();
      return nullptr;
    }
    made[dev] = true;
  }
  return &L;
}

// Inputs that are still arriving from the host: the search waits for X before the
// statistic and for each chunk of W's row groups before quantizing those groups.
struct HostFeed {
  cudaEvent_t x_ready = nullptr;
  const cudaEvent_t* w_ready = nullptr;  // one event per chunk
  int chunks = 0;
  int64_t groups_per_chunk = 0;
};

// The call's status from the device status word the kernels set.
int status_from_word(int h_err) {
  if (h_err & kErrTimeout) return set_error(AWQ_ERR_TIMEOUT, "a bounded wait in the loss GEMM ran out");
  if (h_err & (kErrNonfiniteX | kErrNonfiniteW))
    return set_error(AWQ_ERR_NONFINITE, (h_err & kErrNonfiniteX) ? "non-finite value in X" : "non-finite value in W");
  if (h_err) return set_error(AWQ_ERR_CUDA, "device status word " + std::to_string(h_err));
  return AWQ_OK;
}

// The whole search of one layer on `s`. `out_best` (device, may be NULL) receives the
// index the pack kernel chose. With `fixed` the work space is the caller's array
// instead of a pool block and nothing is allocated.
int search_device(const void* X, const void* W, int in_dtype, int64_t M, int64_t K, int64_t N, int group, int n_grid,
                  float* out_scales, int32_t* out_codes, void* out_steps, void* out_zeros, float* out_losses,
                  int32_t* out_best, double* out_tile_sq_err, int64_t tile_sq_err_len, cudaStream_t s,
                  const HostFeed* feed = nullptr, int quantizer = kQuantAsym, int* async_status = nullptr,
                  const FixedWorkspace* fixed = nullptr) {
  if (quantizer != kQuantAsym && quantizer != kQuantSym)
    return set_error(AWQ_ERR_INVALID_ARG, "quantizer must be AWQ_QUANT_ASYM or AWQ_QUANT_SYM");
  int st = validate(X, W, in_dtype, M, K, N, group, n_grid, out_scales, out_codes, out_steps, out_zeros, true);
  if (st != AWQ_OK) return st;
  // losses and the chosen index are written as plain 4-byte words
  if (out_losses && (reinterpret_cast<uintptr_t>(out_losses) & 3u))
    return set_error(AWQ_ERR_INVALID_ARG, "out_losses misaligned");
  if (out_best && (reinterpret_cast<uintptr_t>(out_best) & 3u))
    return set_error(AWQ_ERR_INVALID_ARG, "out_best misaligned");
  DeviceRestore restore_device;
  bind_device(s, X);
  int dev = 0, num_sms = 0;
  st = check_device(&dev, &num_sms);
  if (st != AWQ_OK) return st;
  if (!is_device_memory(X) || !is_device_memory(W) || !is_device_memory(out_scales) ||
      !is_device_memory(out_codes) || !is_device_memory(out_steps) || !is_device_memory(out_zeros) ||
      (out_losses && !is_device_memory(out_losses)) || (out_best && !is_device_memory(out_best)) ||
      (out_tile_sq_err && !is_device_memory(out_tile_sq_err)))
    return set_error(AWQ_ERR_INVALID_ARG, "inputs and outputs must be device memory (use awq_search_host for host buffers)");
  const Layout L = plan(in_dtype, M, K, N, n_grid);
  if (out_tile_sq_err && tile_sq_err_len < static_cast<int64_t>(n_grid) * L.tiles)
    return set_error(AWQ_ERR_INVALID_ARG, "out_tile_sq_err holds fewer than n_grid * tiles values");

  void* ws = nullptr;
  cudaError_t e = cudaSuccess;
  if (fixed) {
    if (L.total > fixed->bytes)
      return set_error(AWQ_ERR_SHAPE, "this layer needs " + std::to_string(L.total) + " bytes of work space; the " +
                                          "fixed array holds " + std::to_string(fixed->bytes) +
                                          " (use awq_search for larger layers)");
    if ((st = fixed->resolve(dev, &ws)) != AWQ_OK) return st;
  } else {
    cudaMemPool_t pool;
    st = get_pool(dev, &pool);
    if (st != AWQ_OK) return st;
    e = cudaMallocFromPoolAsync(&ws, L.total, pool, s);
    if (e != cudaSuccess || !ws) {
      cudaGetLastError();
      return set_error(AWQ_ERR_OOM, "work space of " + std::to_string(L.total) + " bytes: " + cudaGetErrorString(e));
    }
  }
  uint8_t* base = static_cast<uint8_t*>(ws);
  int* err = reinterpret_cast<int*>(base + L.err);
  float* a = reinterpret_cast<float*>(base + L.a);
  float* S = reinterpret_cast<float*>(base + L.S);
  int* best = reinterpret_cast<int*>(base + L.best);
  float* losses = reinterpret_cast<float*>(base + L.losses);
  __nv_bfloat16* Wt = reinterpret_cast<__nv_bfloat16*>(base + L.Wt);
  float* Y = reinterpret_cast<float*>(base + L.Y);
  double* loss_partial = reinterpret_cast<double*>(base + L.loss_partial);
  const __nv_bfloat16* Xb = in_dtype == AWQ_DTYPE_F32 ? reinterpret_cast<__nv_bfloat16*>(base + L.Xb)
                                                      : static_cast<const __nv_bfloat16*>(X);

  int launches = 0;
  Events ev;
  ev.create(g_profile && !fixed, s);
  const char* where = "";
  int status = AWQ_OK;
  do {
    // the status word, the loss GEMM's per-tile flags and its QDQ counters
    if ((e = cudaMemsetAsync(err, 0, L.flag_bytes, s)) != cudaSuccess) {
      where = "cudaMemsetAsync";
      break;
    }
    if (feed && (e = cudaStreamWaitEvent(s, feed->x_ready, 0)) != cudaSuccess) { where = "waiting for X"; break; }
    ev.mark(kPhStatistic);
    if ((e = launch_statistic(X, in_dtype, M, K, a, err, s, &launches)) != cudaSuccess) {
      where = "statistic kernel";
      break;
    }
    ev.mark(kPhScales);
    if ((e = launch_scales(a, K, n_grid, S, s, &launches)) != cudaSuccess) { where = "scales kernel"; break; }
    ev.mark(kPhConvert);
    if (in_dtype == AWQ_DTYPE_F32) {
      if ((e = launch_to_bf16(static_cast<const float*>(X), M * K, const_cast<__nv_bfloat16*>(Xb), s, &launches)) !=
          cudaSuccess) {
        where = "bf16 operand kernel";
        break;
      }
    }
    const int variant = gemm_variant(M, K, N, n_grid);
    // bf16 W, group 128: the candidate operands are made inside the loss GEMM's launches
    const bool qdq_in_gemm = !feed && qdq_in_loss_gemm(in_dtype, group, variant, M, K, N, n_grid);
    ev.mark(kPhQdq);
    if (qdq_in_gemm) {
      // the reference operand only: the loss GEMM's QDQ warps make the candidates'
      e = launch_qdq(W, in_dtype, K, N, group, 0, S, Wt, err, s, &launches, quantizer);
    } else if (feed) {
      // quantize each chunk of row groups as soon as it has arrived
      const int64_t groups = K / group;
      for (int c = 0; c < feed->chunks && e == cudaSuccess; ++c) {
        const int64_t g0 = c * feed->groups_per_chunk;
        const int64_t gn = std::min(feed->groups_per_chunk, groups - g0);
        if (gn <= 0) break;
        if ((e = cudaStreamWaitEvent(s, feed->w_ready[c], 0)) == cudaSuccess)
          e = launch_qdq_groups(W, in_dtype, K, N, group, n_grid, S, Wt, err, g0, gn, s, &launches, quantizer);
      }
    } else {
      e = launch_qdq(W, in_dtype, K, N, group, n_grid, S, Wt, err, s, &launches, quantizer);
    }
    if (e != cudaSuccess) {
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
    ga.timeout_ns = g_timeout_ns;
    ga.fault_mode = g_fault_mode;
    ga.num_sms = num_sms;
    ga.variant = variant;
    if (qdq_in_gemm) {
      ga.qdq_W = static_cast<const __nv_bfloat16*>(W);
      ga.qdq_S = S;
      ga.qdq_Wt = Wt;
      ga.qdq_ready = err + 4 + L.tiles;
      ga.qdq_quantizer = quantizer;
      ga.qdq_K = K;
      ga.qdq_N = N;
      ga.qdq_grid = n_grid;
    }
    CUtensorMap mapA, mapB;
    const char* why = "";
    if ((e = make_operand_maps(ga, &mapA, &mapB, &why, operand_b_box_rows(ga.variant))) != cudaSuccess) {
      status = set_error(AWQ_ERR_CUDA, std::string("TMA descriptor: ") + why);
      break;
    }
    ev.mark(kPhGemmY);
    int l2_bytes = 0;
    if ((e = cudaDeviceGetAttribute(&l2_bytes, cudaDevAttrL2CacheSize, dev)) != cudaSuccess) {
      where = "querying the L2 cache size";
      break;
    }
    if (ga.variant == 1 && !qdq_in_gemm && !reference_in_own_launch(M, N, l2_bytes)) {
      // one launch: the reference tiles first, each candidate tile waits for its tile of Y
      ga.ready = err + 4;
      ev.mark(kPhGemmLoss);
      if ((e = launch_loss_gemm(ga, mapA, mapB, 4, s, &launches)) != cudaSuccess) { where = "loss GEMM"; break; }
    } else if (ga.variant == 1) {
      // the reference in its own launch (its QDQ warps make candidate tiles while its GEMM
      // runs), then every candidate of a column tile while that tile of Y is in L2 (the
      // QDQ warps make the remaining candidate tiles, column tiles in the order the GEMM
      // reads them)
      ga.qdq_cands = 2;
      if ((e = launch_loss_gemm(ga, mapA, mapB, 0, s, &launches)) != cudaSuccess) { where = "reference GEMM"; break; }
      ev.mark(kPhGemmLoss);
      ga.cand_inner = 1;
      ga.qdq_cands = 1;
      if ((e = launch_loss_gemm(ga, mapA, mapB, 1, s, &launches)) != cudaSuccess) { where = "loss GEMM"; break; }
    } else {
      if ((e = launch_loss_gemm(ga, mapA, mapB, 0, s, &launches)) != cudaSuccess) { where = "reference GEMM"; break; }
      ev.mark(kPhGemmLoss);
      if ((e = launch_loss_gemm(ga, mapA, mapB, 1, s, &launches)) != cudaSuccess) { where = "loss GEMM"; break; }
    }
    ev.mark(kPhReduce);
    if ((e = launch_loss_reduce(loss_partial, L.tiles, n_grid, M, N, losses, s, &launches)) != cudaSuccess) {
      where = "loss reduction kernel";
      break;
    }
    ev.mark(kPhPack);
    if ((e = launch_pack(W, in_dtype, K, N, group, n_grid, S, losses, best, out_codes, static_cast<__half*>(out_steps),
                         static_cast<__half*>(out_zeros), out_scales, s, &launches, quantizer)) != cudaSuccess) {
      where = "pack kernel";
      break;
    }
    ev.mark(kNumPhases);
    if (out_losses &&
        (e = cudaMemcpyAsync(out_losses, losses, static_cast<size_t>(n_grid) * 4, cudaMemcpyDeviceToDevice, s)) !=
            cudaSuccess) {
      where = "copy of the losses";
      break;
    }
    if (out_best && (e = cudaMemcpyAsync(out_best, best, sizeof(int32_t), cudaMemcpyDeviceToDevice, s)) != cudaSuccess) {
      where = "copy of the chosen index";
      break;
    }
    if (out_tile_sq_err &&
        (e = cudaMemcpyAsync(out_tile_sq_err, loss_partial, static_cast<size_t>(n_grid) * L.tiles * 8,
                             cudaMemcpyDeviceToDevice, s)) != cudaSuccess) {
      where = "copy of the tile partials";
      break;
    }
  } while (false);

  if (async_status) {
    // the caller reads the device status word later (pinned host memory), after a sync
    if (status == AWQ_OK && e == cudaSuccess) {
      e = cudaMemcpyAsync(async_status, err, sizeof(int), cudaMemcpyDeviceToHost, s);
      if (e != cudaSuccess) where = "status read-back";
    }
    if (status == AWQ_OK && e != cudaSuccess) status = cuda_error(e, where);
    if (!fixed) cudaFreeAsync(ws, s);
    g_last_launches = launches;
    return status;
  }
  int h_err = 0;
  // a fixed work space's call reads its status into pageable memory (no pinned word)
  int* pinned = fixed ? nullptr : pinned_status_word(dev);
  int* status_dst = pinned ? pinned : &h_err;
  if (status == AWQ_OK && e == cudaSuccess) {
    e = cudaMemcpyAsync(status_dst, err, sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) where = "status read-back";
  }
  if (status == AWQ_OK && e != cudaSuccess) status = cuda_error(e, where);
  if (!fixed) cudaFreeAsync(ws, s);
  cudaError_t se = cudaStreamSynchronize(s);
  if (status == AWQ_OK && se != cudaSuccess) status = cuda_error(se, "stream synchronize");
  if (pinned) h_err = *pinned;
  if (status == AWQ_OK) {
    ev.collect();
    g_last_launches = launches;
    status = status_from_word(h_err);
  }
  return status;
}

}  // namespace

namespace awq {
void record_error_message(const char* msg) { t_last_error = msg; }

int search_in_workspace(const void* X, const void* W, int in_dtype, int64_t M, int64_t K, int64_t N, int group,
                        int n_grid, float* out_scales, int32_t* out_codes, void* out_steps, void* out_zeros,
                        float* out_losses, int32_t* out_best, cudaStream_t s, const FixedWorkspace& fixed) {
  t_last_error.clear();
  return search_device(X, W, in_dtype, M, K, N, group, n_grid, out_scales, out_codes, out_steps, out_zeros,
                       out_losses, out_best, nullptr, 0, s, nullptr, kQuantAsym, nullptr, &fixed);
}
}  // namespace awq

extern "C" {

int awq_search_ex(const void* X, const void* W, int in_dtype, int64_t M, int64_t K, int64_t N, int group, int n_grid,
                  float* out_scales, int32_t* out_codes, void* out_steps, void* out_zeros, float* out_losses,
                  int32_t* out_best, double* out_tile_sq_err, int64_t tile_sq_err_len, awq_stream_t stream) {
  t_last_error.clear();
  return search_device(X, W, in_dtype, M, K, N, group, n_grid, out_scales, out_codes, out_steps, out_zeros,
                       out_losses, out_best, out_tile_sq_err, tile_sq_err_len, reinterpret_cast<cudaStream_t>(stream));
}

int awq_search_async(const void* X, const void* W, int in_dtype, int64_t M, int64_t K, int64_t N, int group,
                     int n_grid, float* out_scales, int32_t* out_codes, void* out_steps, void* out_zeros,
                     float* out_losses, int32_t* out_best, int32_t* status_word, awq_stream_t stream) {
  t_last_error.clear();
  if (!status_word) return set_error(AWQ_ERR_INVALID_ARG, "status_word is NULL");
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, status_word) != cudaSuccess || attr.type != cudaMemoryTypeHost) {
    cudaGetLastError();
    return set_error(AWQ_ERR_INVALID_ARG, "status_word must be pinned host memory");
  }
  return search_device(X, W, in_dtype, M, K, N, group, n_grid, out_scales, out_codes, out_steps, out_zeros,
                       out_losses, out_best, nullptr, 0, reinterpret_cast<cudaStream_t>(stream), nullptr, kQuantAsym,
                       status_word);
}

int awq_search_status(int32_t status_word) {
  t_last_error.clear();
  return status_from_word(status_word);
}

int awq_search(const void* X, const void* W, int64_t M, int64_t K, int64_t N, int group, int n_grid,
               float* out_scales, int32_t* out_codes, void* out_steps, void* out_zeros, float* out_losses,
               awq_stream_t stream) {
  return awq_search_ex(X, W, AWQ_DTYPE_BF16, M, K, N, group, n_grid, out_scales, out_codes, out_steps, out_zeros,
                       out_losses, nullptr, nullptr, 0, stream);
}

int awq_search_f32(const float* X, const float* W, int64_t M, int64_t K, int64_t N, int group, int n_grid,
                   float* out_scales, int32_t* out_codes, void* out_steps, void* out_zeros, float* out_losses,
                   awq_stream_t stream) {
  return awq_search_ex(X, W, AWQ_DTYPE_F32, M, K, N, group, n_grid, out_scales, out_codes, out_steps, out_zeros,
                       out_losses, nullptr, nullptr, 0, stream);
}

int awq_search_quant(const void* X, const void* W, int in_dtype, int64_t M, int64_t K, int64_t N, int group,
                     int n_grid, int quantizer, float* out_scales, int32_t* out_codes, void* out_steps,
                     void* out_zeros, float* out_losses, int32_t* out_best, awq_stream_t stream) {
  t_last_error.clear();
  return search_device(X, W, in_dtype, M, K, N, group, n_grid, out_scales, out_codes, out_steps, out_zeros,
                       out_losses, out_best, nullptr, 0, reinterpret_cast<cudaStream_t>(stream), nullptr, quantizer);
}

int awq_search_host(const void* X_host, const void* W_host, int in_dtype, int64_t M, int64_t K, int64_t N, int group,
                    int n_grid, float* out_scales_host, int32_t* out_codes_host, void* out_steps_host,
                    void* out_zeros_host, float* out_losses_host, int32_t* out_best_host, awq_stream_t stream) {
  t_last_error.clear();
  int st = validate(X_host, W_host, in_dtype, M, K, N, group, n_grid, out_scales_host, out_codes_host,
                    out_steps_host, out_zeros_host, false);
  if (st != AWQ_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DeviceRestore restore_device;
  bind_device(s, nullptr);
  int dev = 0, num_sms = 0;
  st = check_device(&dev, &num_sms);
  if (st != AWQ_OK) return st;
  cudaMemPool_t pool;
  st = get_pool(dev, &pool);
  if (st != AWQ_OK) return st;
  CopyLane* lane = copy_lane(dev);
  if (!lane) return set_error(AWQ_ERR_CUDA, "could not create the host-copy stream");
  const size_t eb = in_dtype == AWQ_DTYPE_BF16 ? 2 : 4;
  const size_t G = static_cast<size_t>(K / group);
  const size_t bx = static_cast<size_t>(M) * K * eb, bw = static_cast<size_t>(K) * N * eb;
  const size_t bs = static_cast<size_t>(K) * 4, bc = static_cast<size_t>(K) * (N / 8) * 4;
  const size_t bst = G * N * 2, bl = static_cast<size_t>(n_grid) * 4;
  size_t off[8], total = 0;
  const size_t sizes[8] = {bx, bw, bs, bc, bst, bst, bl, sizeof(int32_t)};
  for (int i = 0; i < 8; ++i) {
    off[i] = total;
    total += align_up(sizes[i]);
  }
  void* buf = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(&buf, total, pool, s);
  if (e != cudaSuccess || !buf) {
    cudaGetLastError();
    return set_error(AWQ_ERR_OOM, "device buffers for the host call");
  }
  uint8_t* b = static_cast<uint8_t*>(buf);
  int status = AWQ_OK;
  // X first, then W in chunks of whole row groups, on the copy stream; the search on
  // `s` starts on X while W is still arriving and quantizes each chunk as it lands.
  HostFeed feed;
  feed.chunks = static_cast<int>(std::min<size_t>(CopyLane::kChunks, G));
  feed.groups_per_chunk = static_cast<int64_t>((G + feed.chunks - 1) / feed.chunks);
  feed.x_ready = lane->x_ready;
  feed.w_ready = lane->w_ready;
  const size_t chunk_bytes = static_cast<size_t>(feed.groups_per_chunk) * group * N * eb;
  do {
    if ((e = cudaEventRecord(lane->alloc_done, s)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(lane->stream, lane->alloc_done, 0)) != cudaSuccess)
      break;
    if ((e = cudaMemcpyAsync(b + off[0], X_host, bx, cudaMemcpyHostToDevice, lane->stream)) != cudaSuccess ||
        (e = cudaEventRecord(lane->x_ready, lane->stream)) != cudaSuccess)
      break;
    for (int c = 0; c < feed.chunks && e == cudaSuccess; ++c) {
      const size_t at = static_cast<size_t>(c) * chunk_bytes;
      const size_t n = std::min(chunk_bytes, bw - std::min(bw, at));
      if (n > 0)
        e = cudaMemcpyAsync(b + off[1] + at, static_cast<const uint8_t*>(W_host) + at, n, cudaMemcpyHostToDevice,
                            lane->stream);
      if (e == cudaSuccess) e = cudaEventRecord(lane->w_ready[c], lane->stream);
    }
  } while (false);
  if (e != cudaSuccess) status = cuda_error(e, "host-to-device copy");
  if (status == AWQ_OK)
    status = search_device(b + off[0], b + off[1], in_dtype, M, K, N, group, n_grid, reinterpret_cast<float*>(b + off[2]),
                           reinterpret_cast<int32_t*>(b + off[3]), b + off[4], b + off[5],
                           reinterpret_cast<float*>(b + off[6]), reinterpret_cast<int32_t*>(b + off[7]), nullptr, 0, s,
                           &feed);
  if (status == AWQ_OK) {
    if ((e = cudaMemcpyAsync(out_scales_host, b + off[2], bs, cudaMemcpyDeviceToHost, s)) != cudaSuccess ||
        (e = cudaMemcpyAsync(out_codes_host, b + off[3], bc, cudaMemcpyDeviceToHost, s)) != cudaSuccess ||
        (e = cudaMemcpyAsync(out_steps_host, b + off[4], bst, cudaMemcpyDeviceToHost, s)) != cudaSuccess ||
        (e = cudaMemcpyAsync(out_zeros_host, b + off[5], bst, cudaMemcpyDeviceToHost, s)) != cudaSuccess ||
        (out_losses_host &&
         (e = cudaMemcpyAsync(out_losses_host, b + off[6], bl, cudaMemcpyDeviceToHost, s)) != cudaSuccess) ||
        (out_best_host &&
         (e = cudaMemcpyAsync(out_best_host, b + off[7], sizeof(int32_t), cudaMemcpyDeviceToHost, s)) != cudaSuccess))
      status = cuda_error(e, "device-to-host copy");
  }
  // the copy stream must be done with the buffers before they return to the pool
  cudaEventRecord(lane->copies_done, lane->stream);
  cudaStreamWaitEvent(s, lane->copies_done, 0);
  cudaFreeAsync(buf, s);
  cudaError_t se = cudaStreamSynchronize(s);
  if (status == AWQ_OK && se != cudaSuccess) status = cuda_error(se, "stream synchronize");
  return status;
}

// ---- many layers from host memory, transfers overlapped with the searches -------------
// Inputs go through two device slots: while layer i is searched on `stream`, a copy stream
// uploads layer i + 1 into the other slot (X, then W in chunks the first search consumes
// as they land), and a third stream copies layer i's artifact back while layer i + 1 runs.
// The whole batch is enqueued without host waits (events order the slots' reuse); each
// layer's device status word lands in pinned memory and is read after the final sync.
int awq_search_host_batch(int n_layers, const void* const* X_hosts, const void* const* W_hosts, int in_dtype,
                          int64_t M, int64_t K, int64_t N, int group, int n_grid, float* const* out_scales_host,
                          int32_t* const* out_codes_host, void* const* out_steps_host, void* const* out_zeros_host,
                          float* const* out_losses_host, int32_t* const* out_best_host, awq_stream_t stream) {
  t_last_error.clear();
  if (n_layers < 1 || !X_hosts || !W_hosts || !out_scales_host || !out_codes_host || !out_steps_host ||
      !out_zeros_host)
    return set_error(AWQ_ERR_INVALID_ARG, "n_layers must be >= 1 and the pointer arrays non-null");
  for (int i = 0; i < n_layers; ++i) {
    const int st = validate(X_hosts[i], W_hosts[i], in_dtype, M, K, N, group, n_grid, out_scales_host[i],
                            out_codes_host[i], out_steps_host[i], out_zeros_host[i], false);
    if (st != AWQ_OK) return st;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DeviceRestore restore_device;
  bind_device(s, nullptr);
  int dev = 0, num_sms = 0;
  int st = check_device(&dev, &num_sms);
  if (st != AWQ_OK) return st;
  cudaMemPool_t pool;
  if ((st = get_pool(dev, &pool)) != AWQ_OK) return st;
  const size_t eb = in_dtype == AWQ_DTYPE_BF16 ? 2 : 4;
  const size_t G = static_cast<size_t>(K / group);
  const size_t bx = static_cast<size_t>(M) * K * eb, bw = static_cast<size_t>(K) * N * eb;
  const size_t bs = static_cast<size_t>(K) * 4, bc = static_cast<size_t>(K) * (N / 8) * 4;
  const size_t bst = G * N * 2, bl = static_cast<size_t>(n_grid) * 4;
  // per slot: X, W, scales, codes, steps, zeros, losses, chosen index
  const size_t sizes[8] = {bx, bw, bs, bc, bst, bst, bl, sizeof(int32_t)};
  size_t off[8], slot_bytes = 0;
  for (int k = 0; k < 8; ++k) {
    off[k] = slot_bytes;
    slot_bytes += align_up(sizes[k]);
  }
  constexpr int kChunks = CopyLane::kChunks;
  BatchLane* lane = batch_lane(dev);
  if (!lane) return set_error(AWQ_ERR_CUDA, "could not create the batch's streams and events");
  std::lock_guard<std::mutex> hold(lane->mu);  // one batch at a time per device
  BatchLane::Slot* slots = lane->slots;
  cudaStream_t h2d = lane->h2d, d2h = lane->d2h;
  cudaEvent_t alloc_done = lane->alloc_done, search_done = lane->search_done, h2d_done = lane->h2d_done,
              d2h_done = lane->d2h_done;
  void* buf = nullptr;
  int status = AWQ_OK;
  cudaError_t e = cudaSuccess;
  if (lane->words_cap < n_layers) {  // pinned: each layer's device status word, read after the final sync
    if (lane->words) cudaFreeHost(lane->words);
    lane->words = nullptr;
    lane->words_cap = 0;
    if (cudaMallocHost(reinterpret_cast<void**>(&lane->words), static_cast<size_t>(n_layers) * sizeof(int)) ==
        cudaSuccess)
      lane->words_cap = n_layers;
    else
      cudaGetLastError();
  }
  int* words = lane->words_cap >= n_layers ? lane->words : nullptr;
  if (!words) {
    status = set_error(AWQ_ERR_OOM, "pinned status words for the batch");
  } else if ((e = cudaMallocFromPoolAsync(&buf, 2 * slot_bytes, pool, s)) != cudaSuccess || !buf) {
    cudaGetLastError();
    buf = nullptr;
    status = set_error(AWQ_ERR_OOM, "device slots for the batch");
  }
  const int chunks = static_cast<int>(std::min<size_t>(kChunks, G));
  const int64_t groups_per_chunk = static_cast<int64_t>((G + chunks - 1) / chunks);
  const size_t chunk_bytes = static_cast<size_t>(groups_per_chunk) * group * N * eb;
  auto slot_ptr = [&](int i, int k) { return static_cast<uint8_t*>(buf) + (i & 1) * slot_bytes + off[k]; };
  // uploads of layer i into slot i % 2, once the search of layer i - 2 is done with it
  auto upload = [&](int i) -> cudaError_t {
    BatchLane::Slot& sl = slots[i & 1];
    cudaError_t r = i >= 2 ? cudaStreamWaitEvent(h2d, sl.in_free, 0) : cudaSuccess;
    if (r == cudaSuccess) r = cudaMemcpyAsync(slot_ptr(i, 0), X_hosts[i], bx, cudaMemcpyHostToDevice, h2d);
    if (r == cudaSuccess) r = cudaEventRecord(sl.x_ready, h2d);
    for (int c = 0; c < chunks && r == cudaSuccess; ++c) {
      const size_t at = static_cast<size_t>(c) * chunk_bytes;
      const size_t n = std::min(chunk_bytes, bw - std::min(bw, at));
      if (n > 0)
        r = cudaMemcpyAsync(slot_ptr(i, 1) + at, static_cast<const uint8_t*>(W_hosts[i]) + at, n,
                            cudaMemcpyHostToDevice, h2d);
      if (r == cudaSuccess) r = cudaEventRecord(sl.w_ready[c], h2d);
    }
    return r;
  };
  if (status == AWQ_OK) {
    if ((e = cudaEventRecord(alloc_done, s)) != cudaSuccess || (e = cudaStreamWaitEvent(h2d, alloc_done, 0)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(d2h, alloc_done, 0)) != cudaSuccess || (e = upload(0)) != cudaSuccess)
      status = cuda_error(e, "host-to-device copy");
  }
  for (int i = 0; i < n_layers && status == AWQ_OK; ++i) {
    BatchLane::Slot& sl = slots[i & 1];
    if (i + 1 < n_layers && (e = upload(i + 1)) != cudaSuccess) {
      status = cuda_error(e, "host-to-device copy");
      break;
    }
    if (i >= 2 && (e = cudaStreamWaitEvent(s, sl.out_done, 0)) != cudaSuccess) {
      status = cuda_error(e, "stream wait");
      break;
    }
    // the first layer is searched as its inputs land (X, then W chunk by chunk); later
    // layers were uploaded during the previous search, so they wait for their whole
    // upload and quantize W in one launch
    HostFeed feed;
    feed.chunks = chunks;
    feed.groups_per_chunk = groups_per_chunk;
    feed.x_ready = sl.x_ready;
    feed.w_ready = sl.w_ready;
    if (i > 0 && ((e = cudaStreamWaitEvent(s, sl.x_ready, 0)) != cudaSuccess ||
                  (e = cudaStreamWaitEvent(s, sl.w_ready[chunks - 1], 0)) != cudaSuccess)) {
      status = cuda_error(e, "stream wait");
      break;
    }
    status = search_device(slot_ptr(i, 0), slot_ptr(i, 1), in_dtype, M, K, N, group, n_grid,
                           reinterpret_cast<float*>(slot_ptr(i, 2)), reinterpret_cast<int32_t*>(slot_ptr(i, 3)),
                           slot_ptr(i, 4), slot_ptr(i, 5), reinterpret_cast<float*>(slot_ptr(i, 6)),
                           reinterpret_cast<int32_t*>(slot_ptr(i, 7)), nullptr, 0, s, i == 0 ? &feed : nullptr,
                           kQuantAsym, words + i);
    if (status != AWQ_OK) break;
    if ((e = cudaEventRecord(sl.in_free, s)) != cudaSuccess || (e = cudaEventRecord(search_done, s)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(d2h, search_done, 0)) != cudaSuccess ||
        (e = cudaMemcpyAsync(out_scales_host[i], slot_ptr(i, 2), bs, cudaMemcpyDeviceToHost, d2h)) != cudaSuccess ||
        (e = cudaMemcpyAsync(out_codes_host[i], slot_ptr(i, 3), bc, cudaMemcpyDeviceToHost, d2h)) != cudaSuccess ||
        (e = cudaMemcpyAsync(out_steps_host[i], slot_ptr(i, 4), bst, cudaMemcpyDeviceToHost, d2h)) != cudaSuccess ||
        (e = cudaMemcpyAsync(out_zeros_host[i], slot_ptr(i, 5), bst, cudaMemcpyDeviceToHost, d2h)) != cudaSuccess ||
        (out_losses_host && out_losses_host[i] &&
         (e = cudaMemcpyAsync(out_losses_host[i], slot_ptr(i, 6), bl, cudaMemcpyDeviceToHost, d2h)) != cudaSuccess) ||
        (out_best_host && out_best_host[i] &&
         (e = cudaMemcpyAsync(out_best_host[i], slot_ptr(i, 7), sizeof(int32_t), cudaMemcpyDeviceToHost, d2h)) !=
             cudaSuccess) ||
        (e = cudaEventRecord(sl.out_done, d2h)) != cudaSuccess) {
      status = cuda_error(e, "device-to-host copy");
      break;
    }
  }
  // both copy streams are done with the slots before they return to the pool
  {
    cudaEventRecord(h2d_done, h2d);
    cudaEventRecord(d2h_done, d2h);
    cudaStreamWaitEvent(s, h2d_done, 0);
    cudaStreamWaitEvent(s, d2h_done, 0);
  }
  if (buf) cudaFreeAsync(buf, s);
  cudaError_t se = cudaStreamSynchronize(s);
  if (h2d) cudaStreamSynchronize(h2d);
  if (d2h) cudaStreamSynchronize(d2h);
  if (status == AWQ_OK && se != cudaSuccess) status = cuda_error(se, "stream synchronize");
  // the first layer whose kernels reported a problem decides the status
  for (int i = 0; i < n_layers && status == AWQ_OK && words; ++i) status = status_from_word(words[i]);
  return status;
}

// ---- the steps one at a time (same kernels as the search) --------------------------
int awq_activation_statistic(const void* X, int in_dtype, int64_t M, int64_t K, float* out_a, awq_stream_t stream) {
  t_last_error.clear();
  static int dummy;
  int st = validate(X, &dummy, in_dtype, M, K, 8, 32, 1, out_a, &dummy, &dummy, &dummy, false);
  if (st != AWQ_OK) return st;
  if (!aligned16(X) || (reinterpret_cast<uintptr_t>(out_a) & 3u))
    return set_error(AWQ_ERR_INVALID_ARG, "X must be 16-byte aligned and out_a 4-byte aligned");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DeviceRestore restore_device;
  bind_device(s, X);
  int dev = 0, num_sms = 0;
  if ((st = check_device(&dev, &num_sms)) != AWQ_OK) return st;
  if (!is_device_memory(X) || !is_device_memory(out_a))
    return set_error(AWQ_ERR_INVALID_ARG, "X and out_a must be device memory");
  cudaMemPool_t pool;
  if ((st = get_pool(dev, &pool)) != AWQ_OK) return st;
  void* ws = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(&ws, 256, pool, s);  // the status word
  if (e != cudaSuccess || !ws) {
    cudaGetLastError();
    return set_error(AWQ_ERR_OOM, "statistic work space");
  }
  int* err = static_cast<int*>(ws);
  int launches = 0, h_err = 0;
  if ((e = cudaMemsetAsync(err, 0, 16, s)) == cudaSuccess &&
      (e = launch_statistic(X, in_dtype, M, K, out_a, err, s, &launches)) == cudaSuccess)
    e = cudaMemcpyAsync(&h_err, err, sizeof(int), cudaMemcpyDeviceToHost, s);
  cudaFreeAsync(ws, s);
  cudaError_t se = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_error(e, "statistic");
  if (se != cudaSuccess) return cuda_error(se, "stream synchronize");
  g_last_launches = launches;
  if (h_err & kErrNonfiniteX) return set_error(AWQ_ERR_NONFINITE, "non-finite value in X");
  return AWQ_OK;
}

int awq_candidate_scales(const float* a, int64_t K, int n_grid, float* out_S, awq_stream_t stream) {
  t_last_error.clear();
  if (!a || !out_S) return set_error(AWQ_ERR_INVALID_ARG, "a required pointer is NULL");
  if (K <= 0 || K >= (int64_t(1) << 31)) return set_error(AWQ_ERR_SHAPE, "K must be in 1 .. 2^31-1");
  if (n_grid < 1 || n_grid > kMaxGrid) return set_error(AWQ_ERR_INVALID_ARG, "n_grid must be in 1..64");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DeviceRestore restore_device;
  bind_device(s, a);
  int dev = 0, num_sms = 0, st;
  if ((st = check_device(&dev, &num_sms)) != AWQ_OK) return st;
  if (!is_device_memory(a) || !is_device_memory(out_S))
    return set_error(AWQ_ERR_INVALID_ARG, "a and out_S must be device memory");
  int launches = 0;
  cudaError_t e = launch_scales(a, K, n_grid, out_S, s, &launches);
  cudaError_t se = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_error(e, "scales");
  if (se != cudaSuccess) return cuda_error(se, "stream synchronize");
  g_last_launches = launches;
  return AWQ_OK;
}

int awq_qdq_candidates(const void* W, int in_dtype, int64_t K, int64_t N, int group, int n_grid, const float* S,
                       void* out_wt, awq_stream_t stream) {
  t_last_error.clear();
  static int dummy;
  int st = validate(&dummy, W, in_dtype, 1, K, N, group, n_grid, S, out_wt, &dummy, &dummy, false);
  if (st != AWQ_OK) return st;
  if (!aligned16(W) || !aligned16(out_wt) || (reinterpret_cast<uintptr_t>(S) & 3u))
    return set_error(AWQ_ERR_INVALID_ARG, "W and out_wt must be 16-byte aligned, S 4-byte aligned");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DeviceRestore restore_device;
  bind_device(s, W);
  int dev = 0, num_sms = 0;
  if ((st = check_device(&dev, &num_sms)) != AWQ_OK) return st;
  if (!is_device_memory(W) || !is_device_memory(S) || !is_device_memory(out_wt))
    return set_error(AWQ_ERR_INVALID_ARG, "W, S and out_wt must be device memory");
  cudaMemPool_t pool;
  if ((st = get_pool(dev, &pool)) != AWQ_OK) return st;
  void* ws = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(&ws, 256, pool, s);
  if (e != cudaSuccess || !ws) {
    cudaGetLastError();
    return set_error(AWQ_ERR_OOM, "status word");
  }
  int* err = static_cast<int*>(ws);
  int launches = 0, h_err = 0;
  if ((e = cudaMemsetAsync(err, 0, 16, s)) == cudaSuccess &&
      (e = launch_qdq(W, in_dtype, K, N, group, n_grid, S, static_cast<__nv_bfloat16*>(out_wt), err, s,
                      &launches)) == cudaSuccess)
    e = cudaMemcpyAsync(&h_err, err, sizeof(int), cudaMemcpyDeviceToHost, s);
  cudaFreeAsync(ws, s);
  cudaError_t se = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_error(e, "qdq");
  if (se != cudaSuccess) return cuda_error(se, "stream synchronize");
  g_last_launches = launches;
  if (h_err & kErrNonfiniteW) return set_error(AWQ_ERR_NONFINITE, "non-finite value in W");
  return AWQ_OK;
}

// ---- clipping search after the scaling ---------------------------------------------
int awq_clip_search(const void* X, const void* W, int in_dtype, const float* scales, int64_t M, int64_t K, int64_t N,
                    int group, int n_shrink, int64_t max_tokens, int quantizer, float* out_max_val, int32_t* out_best,
                    double* out_errors, int32_t* out_codes, void* out_steps, void* out_zeros, awq_stream_t stream) {
  t_last_error.clear();
  int st = validate(X, W, in_dtype, M, K, N, group, 1, out_max_val, out_codes, out_steps, out_zeros, false);
  if (st != AWQ_OK) return st;
  if (!scales) return set_error(AWQ_ERR_INVALID_ARG, "scales is NULL");
  if (n_shrink < 1 || n_shrink > kMaxShrink) return set_error(AWQ_ERR_INVALID_ARG, "n_shrink must be in 1..20");
  if (max_tokens < 1) return set_error(AWQ_ERR_INVALID_ARG, "max_tokens must be positive");
  if (quantizer != kQuantAsym && quantizer != kQuantSym)
    return set_error(AWQ_ERR_INVALID_ARG, "quantizer must be AWQ_QUANT_ASYM or AWQ_QUANT_SYM");
  if (!aligned16(X) || !aligned16(W) || (reinterpret_cast<uintptr_t>(scales) & 3u) ||
      (reinterpret_cast<uintptr_t>(out_max_val) & 3u) || (reinterpret_cast<uintptr_t>(out_best) & 3u) ||
      (reinterpret_cast<uintptr_t>(out_errors) & 7u) || (reinterpret_cast<uintptr_t>(out_codes) & 3u) ||
      (reinterpret_cast<uintptr_t>(out_steps) & 1u) || (reinterpret_cast<uintptr_t>(out_zeros) & 1u))
    return set_error(AWQ_ERR_INVALID_ARG, "X and W must be 16-byte aligned, the other pointers aligned to their type");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DeviceRestore restore_device;
  bind_device(s, X);
  int dev = 0, num_sms = 0;
  if ((st = check_device(&dev, &num_sms)) != AWQ_OK) return st;
  if (!is_device_memory(X) || !is_device_memory(W) || !is_device_memory(scales) || !is_device_memory(out_max_val) ||
      !is_device_memory(out_codes) || !is_device_memory(out_steps) || !is_device_memory(out_zeros) ||
      (out_best && !is_device_memory(out_best)) || (out_errors && !is_device_memory(out_errors)))
    return set_error(AWQ_ERR_INVALID_ARG, "inputs and outputs must be device memory");
  cudaMemPool_t pool;
  if ((st = get_pool(dev, &pool)) != AWQ_OK) return st;
  const size_t h_bytes = static_cast<size_t>(K / group) * group * group * sizeof(double);
  void* ws = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(&ws, 256 + align_up(h_bytes), pool, s);
  if (e != cudaSuccess || !ws) {
    cudaGetLastError();
    return set_error(AWQ_ERR_OOM, "clipping work space of " + std::to_string(256 + h_bytes) + " bytes");
  }
  ClipArgs a;
  a.X = X;
  a.W = W;
  a.in_dtype = in_dtype;
  a.s = scales;
  a.M = M;
  a.K = K;
  a.N = N;
  a.group = group;
  a.n_shrink = n_shrink;
  a.max_tokens = max_tokens;
  a.tokens = static_cast<int>(clip_token_count(M, max_tokens));
  a.err = static_cast<int*>(ws);
  a.H = reinterpret_cast<double*>(static_cast<uint8_t*>(ws) + 256);
  a.max_val = out_max_val;
  a.best = out_best;
  a.errors = out_errors;
  a.codes = out_codes;
  a.steps = static_cast<__half*>(out_steps);
  a.zeros = static_cast<__half*>(out_zeros);
  a.ev = g_profile ? clip_events(dev) : nullptr;
  a.quantizer = quantizer;
  int launches = 0, h_err = 0;
  int* pinned = pinned_status_word(dev);
  int* status_dst = pinned ? pinned : &h_err;
  if ((e = cudaMemsetAsync(a.err, 0, 16, s)) == cudaSuccess && (e = launch_clip(a, s, &launches)) == cudaSuccess)
    e = cudaMemcpyAsync(status_dst, a.err, sizeof(int), cudaMemcpyDeviceToHost, s);
  cudaFreeAsync(ws, s);
  cudaError_t se = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_error(e, "clipping search");
  if (se != cudaSuccess) return cuda_error(se, "stream synchronize");
  if (pinned) h_err = *pinned;
  g_last_launches = launches;
  if (a.ev) {
    cudaEventElapsedTime(&g_clip_ms[0], a.ev[0], a.ev[1]);
    cudaEventElapsedTime(&g_clip_ms[1], a.ev[1], a.ev[2]);
  }
  if (h_err & kErrBadScale) return set_error(AWQ_ERR_INVALID_ARG, "a scale is not a positive finite number");
  if (h_err & kErrNonfiniteX) return set_error(AWQ_ERR_NONFINITE, "non-finite value in X / s");
  if (h_err & kErrNonfiniteW) return set_error(AWQ_ERR_NONFINITE, "non-finite value in W");
  if (h_err) return set_error(AWQ_ERR_CUDA, "device status word " + std::to_string(h_err));
  return AWQ_OK;
}

// ---- W4A16 consumer of the artifact --------------------------------------------------
namespace {
int validate_w4a16(const void* A, const void* codes, const void* steps, const void* zeros, int64_t M, int64_t K,
                   int64_t N, int group, const void* Y) {
  if (!codes || !steps || !zeros || (M > 0 && (!A || !Y)))
    return set_error(AWQ_ERR_INVALID_ARG, "a required pointer is NULL");
  if (group != 32 && group != 64 && group != 128)
    return set_error(AWQ_ERR_INVALID_ARG, "group must be 32, 64 or 128");
  if (M <= 0 || K <= 0 || N <= 0) return set_error(AWQ_ERR_SHAPE, "M, K and N must be positive");
  if (M >= (int64_t(1) << 31) || K >= (int64_t(1) << 31) || N >= (int64_t(1) << 31))
    return set_error(AWQ_ERR_SHAPE, "M, K and N must be below 2^31");
  if (K % group) return set_error(AWQ_ERR_SHAPE, "group must divide K");
  if (K / group > 65535) return set_error(AWQ_ERR_SHAPE, "K / group must not exceed 65535");
  if (N % 8) return set_error(AWQ_ERR_SHAPE, "N must be a multiple of 8 (eight codes per int32)");
  if (!aligned16(A) || !aligned16(codes) || !aligned16(steps) || !aligned16(zeros) || !aligned16(Y))
    return set_error(AWQ_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  return AWQ_OK;
}
}  // namespace

int awq_w4a16_matmul(const void* A, const int32_t* codes, const void* steps, const void* zeros, int64_t M, int64_t K,
                     int64_t N, int group, float* Y, awq_stream_t stream) {
  t_last_error.clear();
  int st = validate_w4a16(A, codes, steps, zeros, M, K, N, group, Y);
  if (st != AWQ_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DeviceRestore restore_device;
  bind_device(s, codes);
  int dev = 0, num_sms = 0;
  if ((st = check_device(&dev, &num_sms)) != AWQ_OK) return st;
  if (!is_device_memory(A) || !is_device_memory(codes) || !is_device_memory(steps) || !is_device_memory(zeros) ||
      !is_device_memory(Y))
    return set_error(AWQ_ERR_INVALID_ARG, "inputs and outputs must be device memory");
  cudaMemPool_t pool;
  if ((st = get_pool(dev, &pool)) != AWQ_OK) return st;
  const bool gemv = M <= kW4A16GemvMaxM;
  const size_t ws_bytes = gemv ? 256 + align_up(static_cast<size_t>(gemv_split_floats(M, K, N, group, num_sms)) * 4)
                               : 256 + align_up(static_cast<size_t>(N) * K * 2);
  void* ws = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(&ws, ws_bytes, pool, s);
  if (e != cudaSuccess || !ws) {
    cudaGetLastError();
    return set_error(AWQ_ERR_OOM, "W4A16 work space of " + std::to_string(ws_bytes) + " bytes");
  }
  int* err = static_cast<int*>(ws);
  void* body = static_cast<uint8_t*>(ws) + 256;
  W4A16Args a;
  a.A = static_cast<const __half*>(A);
  a.codes = codes;
  a.steps = static_cast<const __half*>(steps);
  a.zeros = static_cast<const __half*>(zeros);
  a.M = M;
  a.K = K;
  a.N = N;
  a.group = group;
  a.Y = Y;
  int launches = 0, h_err = 0;
  cudaEvent_t* ev = g_profile ? w4a16_events(dev) : nullptr;
  if (gemv) {
    // asynchronous: no device-side error conditions, nothing to read back
    if (ev) cudaEventRecord(ev[0], s);
    e = launch_w4a16_gemv(a, num_sms, static_cast<float*>(body), s, &launches);
    if (ev) cudaEventRecord(ev[1], s);
    g_w4a16_profiled = ev != nullptr;
    cudaFreeAsync(ws, s);
    if (e != cudaSuccess) return cuda_error(e, "W4A16 GEMV");
    g_last_launches = launches;
    return AWQ_OK;
  }
  int* pinned = pinned_status_word(dev);
  int* status_dst = pinned ? pinned : &h_err;
  int status = AWQ_OK;
  const char* where = "";
  do {
    if ((e = cudaMemsetAsync(err, 0, 16, s)) != cudaSuccess) { where = "cudaMemsetAsync"; break; }
    if (ev) cudaEventRecord(ev[0], s);
    {
      __half* Wt = static_cast<__half*>(body);
      if ((e = launch_w4a16_dequant(codes, a.steps, a.zeros, K, N, group, Wt, s, &launches)) != cudaSuccess) {
        where = "W4A16 dequantization";
        break;
      }
      LossGemmArgs ga;
      ga.Xb = reinterpret_cast<const __nv_bfloat16*>(A);  // 2-byte elements; the MMA reads them as fp16
      ga.Wt = reinterpret_cast<const __nv_bfloat16*>(Wt);
      ga.M = M;
      ga.K = K;
      ga.N = N;
      ga.n_grid = 0;
      ga.Y = Y;
      ga.partial = nullptr;
      ga.err = err;
      ga.timeout_ns = g_timeout_ns;
      ga.fault_mode = 0;
      ga.num_sms = num_sms;
      ga.f16 = 1;
      ga.slot_base = 0;
      CUtensorMap mapA, mapB;
      const char* why = "";
      if ((e = make_operand_maps(ga, &mapA, &mapB, &why, kTileN)) != cudaSuccess) {
        status = set_error(AWQ_ERR_CUDA, std::string("TMA descriptor: ") + why);
        break;
      }
      if ((e = launch_loss_gemm(ga, mapA, mapB, 2, s, &launches)) != cudaSuccess) { where = "W4A16 GEMM"; break; }
      if (ev) cudaEventRecord(ev[1], s);
      g_w4a16_profiled = ev != nullptr;
    }
    e = cudaMemcpyAsync(status_dst, err, sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) where = "status read-back";
  } while (false);
  if (status == AWQ_OK && e != cudaSuccess) status = cuda_error(e, where);
  cudaFreeAsync(ws, s);
  cudaError_t se = cudaStreamSynchronize(s);
  if (status == AWQ_OK && se != cudaSuccess) status = cuda_error(se, "stream synchronize");
  if (pinned) h_err = *pinned;
  if (status == AWQ_OK) {
    g_last_launches = launches;
    if (h_err & kErrTimeout) status = set_error(AWQ_ERR_TIMEOUT, "a bounded wait in the W4A16 GEMM ran out");
    else if (h_err) status = set_error(AWQ_ERR_CUDA, "device status word " + std::to_string(h_err));
  }
  return status;
}

int awq_w4a16_repack(const int32_t* codes, int64_t K, int64_t N, int32_t* out_packed, awq_stream_t stream) {
  t_last_error.clear();
  if (!codes || !out_packed) return set_error(AWQ_ERR_INVALID_ARG, "a required pointer is NULL");
  if (K <= 0 || N <= 0 || K % 32 || N % 64 || K >= (int64_t(1) << 31) || N >= (int64_t(1) << 31))
    return set_error(AWQ_ERR_SHAPE, "K must be a positive multiple of 32 and N of 64");
  if (!aligned16(codes) || !aligned16(out_packed))
    return set_error(AWQ_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DeviceRestore restore_device;
  bind_device(s, codes);
  int dev = 0, num_sms = 0, st;
  if ((st = check_device(&dev, &num_sms)) != AWQ_OK) return st;
  if (!is_device_memory(codes) || !is_device_memory(out_packed))
    return set_error(AWQ_ERR_INVALID_ARG, "codes and out_packed must be device memory");
  int launches = 0;
  cudaError_t e = launch_w4a16_repack(codes, K, N, reinterpret_cast<uint32_t*>(out_packed), s, &launches);
  cudaError_t se = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_error(e, "repack");
  if (se != cudaSuccess) return cuda_error(se, "stream synchronize");
  g_last_launches = launches;
  return AWQ_OK;
}

int awq_w4a16_matmul_packed(const void* A, const int32_t* packed, const void* steps, const void* zeros, int64_t M,
                            int64_t K, int64_t N, int group, float* Y, awq_stream_t stream) {
  t_last_error.clear();
  int st = validate_w4a16(A, packed, steps, zeros, M, K, N, group, Y);
  if (st != AWQ_OK) return st;
  if (M > kW4A16GemvMaxM) return set_error(AWQ_ERR_SHAPE, "the repacked layout serves at most 16 tokens");
  if (N % 64) return set_error(AWQ_ERR_SHAPE, "the repacked layout needs N % 64 == 0");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DeviceRestore restore_device;
  bind_device(s, packed);
  int dev = 0, num_sms = 0;
  if ((st = check_device(&dev, &num_sms)) != AWQ_OK) return st;
  if (!is_device_memory(A) || !is_device_memory(packed) || !is_device_memory(steps) || !is_device_memory(zeros) ||
      !is_device_memory(Y))
    return set_error(AWQ_ERR_INVALID_ARG, "inputs and outputs must be device memory");
  cudaMemPool_t pool;
  if ((st = get_pool(dev, &pool)) != AWQ_OK) return st;
  const size_t ws_bytes = 256 + align_up(static_cast<size_t>(gemv_split_floats(M, K, N, group, num_sms, true)) * 4);
  void* ws = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(&ws, ws_bytes, pool, s);
  if (e != cudaSuccess || !ws) {
    cudaGetLastError();
    return set_error(AWQ_ERR_OOM, "W4A16 work space");
  }
  W4A16Args a;
  a.A = static_cast<const __half*>(A);
  a.codes = packed;
  a.steps = static_cast<const __half*>(steps);
  a.zeros = static_cast<const __half*>(zeros);
  a.M = M;
  a.K = K;
  a.N = N;
  a.group = group;
  a.Y = Y;
  int launches = 0;
  cudaEvent_t* ev = g_profile ? w4a16_events(dev) : nullptr;
  if (ev) cudaEventRecord(ev[0], s);
  e = launch_w4a16_gemv_packed(a, reinterpret_cast<const uint32_t*>(packed), num_sms,
                               reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + 256), s, &launches);
  if (ev) cudaEventRecord(ev[1], s);
  g_w4a16_profiled = ev != nullptr;
  cudaFreeAsync(ws, s);
  if (e != cudaSuccess) return cuda_error(e, "W4A16 GEMV (repacked)");
  g_last_launches = launches;
  return AWQ_OK;
}

float awq_w4a16_profile_last(void) {
  if (!g_w4a16_profiled || !g_w4a16_last_ev) return -1.0f;
  float ms = -1.0f;
  if (cudaEventSynchronize(g_w4a16_last_ev[1]) != cudaSuccess ||
      cudaEventElapsedTime(&ms, g_w4a16_last_ev[0], g_w4a16_last_ev[1]) != cudaSuccess) {
    cudaGetLastError();
    return -1.0f;
  }
  return ms;
}

int awq_w4a16_dequant(const int32_t* codes, const void* steps, const void* zeros, int64_t K, int64_t N, int group,
                      void* out_wt, awq_stream_t stream) {
  t_last_error.clear();
  static __align__(16) int dummy[4];
  int st = validate_w4a16(dummy, codes, steps, zeros, 1, K, N, group, out_wt);
  if (st != AWQ_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DeviceRestore restore_device;
  bind_device(s, codes);
  int dev = 0, num_sms = 0;
  if ((st = check_device(&dev, &num_sms)) != AWQ_OK) return st;
  if (!is_device_memory(codes) || !is_device_memory(steps) || !is_device_memory(zeros) || !is_device_memory(out_wt))
    return set_error(AWQ_ERR_INVALID_ARG, "inputs and outputs must be device memory");
  int launches = 0;
  cudaError_t e = launch_w4a16_dequant(codes, static_cast<const __half*>(steps), static_cast<const __half*>(zeros), K,
                                       N, group, static_cast<__half*>(out_wt), s, &launches);
  cudaError_t se = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_error(e, "W4A16 dequantization");
  if (se != cudaSuccess) return cuda_error(se, "stream synchronize");
  g_last_launches = launches;
  return AWQ_OK;
}

// ---- MLP-block objective --------------------------------------------------------------
int awq_search_mlp(const void* X, const void* W_gu, const void* W_down, int in_dtype, int64_t M, int64_t K,
                   int64_t F, int64_t K_out, int group, int n_grid, float* out_scales, int32_t* out_codes,
                   void* out_steps, void* out_zeros, float* out_losses, int32_t* out_best, awq_stream_t stream) {
  t_last_error.clear();
  int st = validate(X, W_gu, in_dtype, M, K, 2 * F, group, n_grid, out_scales, out_codes, out_steps, out_zeros, true);
  if (st != AWQ_OK) return st;
  if (!W_down || !aligned16(W_down)) return set_error(AWQ_ERR_INVALID_ARG, "W_down must be a 16-byte aligned pointer");
  if (F <= 0 || K_out <= 0 || F % 8 || K_out % 8 || K_out >= (int64_t(1) << 31))
    return set_error(AWQ_ERR_SHAPE, "F and K_out must be positive multiples of 8");
  if (out_losses && (reinterpret_cast<uintptr_t>(out_losses) & 3u))
    return set_error(AWQ_ERR_INVALID_ARG, "out_losses misaligned");
  if (out_best && (reinterpret_cast<uintptr_t>(out_best) & 3u))
    return set_error(AWQ_ERR_INVALID_ARG, "out_best misaligned");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DeviceRestore restore_device;
  bind_device(s, X);
  int dev = 0, num_sms = 0;
  if ((st = check_device(&dev, &num_sms)) != AWQ_OK) return st;
  if (!is_device_memory(X) || !is_device_memory(W_gu) || !is_device_memory(W_down) || !is_device_memory(out_scales) ||
      !is_device_memory(out_codes) || !is_device_memory(out_steps) || !is_device_memory(out_zeros) ||
      (out_losses && !is_device_memory(out_losses)) || (out_best && !is_device_memory(out_best)))
    return set_error(AWQ_ERR_INVALID_ARG, "inputs and outputs must be device memory");
  const int64_t N = 2 * F;
  const int64_t tiles2 = ceil_div(M, kTileM) * ceil_div(K_out, kTileN);
  // The silu-mul runs in the first GEMM's epilogue when its tiles can hold both halves of
  // 128 intermediate columns (F % 128 == 0); AWQ_MLP_UNFUSED=1 keeps the separate
  // elementwise kernel (the two give identical bits).
  const char* unfused_env = getenv("AWQ_MLP_UNFUSED");
  const bool fused = F % (kTileN / 2) == 0 && !(unfused_env && unfused_env[0] == '1');
  // The fused path runs each GEMM once for a batch of candidates (their intermediates h
  // side by side, up to 4 GiB), so the second GEMM's few hundred tiles of one candidate
  // do not each end in a partial wave.
  const int64_t h_bytes = M * F * 2;
  const int h_batch = fused ? static_cast<int>(std::max<int64_t>(
                                  1, std::min<int64_t>(n_grid, (int64_t(4) << 30) / std::max<int64_t>(h_bytes, 1))))
                            : 0;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align_up(bytes);
    return at;
  };
  // bf16 W with group 128: the candidate operands of [W_gate | W_up] are made by the
  // first GEMM's QDQ warps while the reference block runs and then while the candidates'
  // first GEMM walks every candidate of an operand tile before the next
  const bool qdq_warps = fused && qdq_in_loss_gemm(in_dtype, group, 1, M, K, N, n_grid);
  const size_t flag_bytes = 16 + static_cast<size_t>(ceil_div(N, kTileN) + 1) * 4;  // status word, QDQ counters
  const size_t o_err = take(flag_bytes), o_a = take(static_cast<size_t>(K) * 4), o_S = take(static_cast<size_t>(n_grid) * K * 4),
               o_best = take(16), o_losses = take(static_cast<size_t>(n_grid) * 4),
               o_Xb = in_dtype == AWQ_DTYPE_F32 ? take(static_cast<size_t>(M) * K * 2) : 0,
               o_Wt = take(static_cast<size_t>(n_grid + 1) * N * K * 2),
               o_H = fused ? 0 : take(static_cast<size_t>(M) * N * 4),
               o_h = take(static_cast<size_t>(1 + h_batch) * M * F * 2),
               o_WdT = take(static_cast<size_t>(K_out) * F * 2),
               o_Y = take(static_cast<size_t>(tiles2) * kTileM * kTileN * 4),
               o_part = take(static_cast<size_t>(n_grid) * tiles2 * 8);
  cudaMemPool_t pool;
  if ((st = get_pool(dev, &pool)) != AWQ_OK) return st;
  void* ws = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(&ws, off, pool, s);
  if (e != cudaSuccess || !ws) {
    cudaGetLastError();
    return set_error(AWQ_ERR_OOM, "work space of " + std::to_string(off) + " bytes");
  }
  uint8_t* b = static_cast<uint8_t*>(ws);
  int* err = reinterpret_cast<int*>(b + o_err);
  float* a = reinterpret_cast<float*>(b + o_a);
  float* S = reinterpret_cast<float*>(b + o_S);
  int* best = reinterpret_cast<int*>(b + o_best);
  float* losses = reinterpret_cast<float*>(b + o_losses);
  __nv_bfloat16* Wt = reinterpret_cast<__nv_bfloat16*>(b + o_Wt);
  float* H = fused ? nullptr : reinterpret_cast<float*>(b + o_H);
  __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(b + o_h);
  __nv_bfloat16* WdT = reinterpret_cast<__nv_bfloat16*>(b + o_WdT);
  float* Y = reinterpret_cast<float*>(b + o_Y);
  double* part = reinterpret_cast<double*>(b + o_part);
  const __nv_bfloat16* Xb = in_dtype == AWQ_DTYPE_F32 ? reinterpret_cast<__nv_bfloat16*>(b + o_Xb)
                                                      : static_cast<const __nv_bfloat16*>(X);
  int launches = 0, h_err = 0, status = AWQ_OK;
  const char* where = "";
  do {
    if ((e = cudaMemsetAsync(err, 0, flag_bytes, s)) != cudaSuccess) { where = "cudaMemsetAsync"; break; }
    if ((e = launch_statistic(X, in_dtype, M, K, a, err, s, &launches)) != cudaSuccess) {
      where = "statistic kernel";
      break;
    }
    if ((e = launch_scales(a, K, n_grid, S, s, &launches)) != cudaSuccess) { where = "scales kernel"; break; }
    if (in_dtype == AWQ_DTYPE_F32 &&
        (e = launch_to_bf16(static_cast<const float*>(X), M * K, const_cast<__nv_bfloat16*>(Xb), s, &launches)) !=
            cudaSuccess) {
      where = "bf16 operand kernel";
      break;
    }
    // every operand slot, or (QDQ warps) the reference slot alone
    if ((e = launch_qdq(W_gu, in_dtype, K, N, group, qdq_warps ? 0 : n_grid, S, Wt, err, s, &launches, 0,
                        fused ? F : 0)) != cudaSuccess) {
      where = "qdq kernel";
      break;
    }
    if ((e = launch_transpose_bf16(W_down, in_dtype, F, K_out, WdT, s, &launches)) != cudaSuccess) {
      where = "down-projection transpose";
      break;
    }
    // GEMM 1: h = bf16(silu(X_b W_gate) (X_b W_up)) with the silu-mul in the epilogue
    // (mode 3), or H = X_b [W_gate | W_up]_slot row-major fp32 (mode 2) and the
    // elementwise kernel
    LossGemmArgs g1;
    g1.Xb = Xb;
    g1.Wt = Wt;
    g1.M = M;
    g1.K = K;
    g1.N = N;
    g1.n_grid = n_grid;
    g1.Y = fused ? nullptr : H;
    g1.H = fused ? h : nullptr;
    g1.partial = nullptr;
    g1.err = err;
    g1.timeout_ns = g_timeout_ns;
    g1.fault_mode = 0;
    g1.num_sms = num_sms;
    if (qdq_warps) {
      g1.qdq_W = static_cast<const __nv_bfloat16*>(W_gu);
      g1.qdq_S = S;
      g1.qdq_Wt = Wt;
      g1.qdq_ready = err + 4;
      g1.qdq_K = K;
      g1.qdq_N = N;
      g1.qdq_interleave = F;
      g1.qdq_grid = n_grid;
    }
    // GEMM 2: h W_down^T; mode 0 writes the reference block output (tiled), mode 1 the
    // per-tile squared error of one candidate against it
    LossGemmArgs g2 = g1;
    g2.Xb = h;
    g2.Wt = WdT;
    g2.K = F;
    g2.N = K_out;
    g2.n_grid = 0;  // one operand slot for the tensor map
    g2.Y = Y;
    g2.H = nullptr;
    g2.slot_base = 0;
    CUtensorMap a1, b1, a2, b2, a2b, b2b;
    const char* why = "";
    // the batched second GEMM: A = the stack of intermediates [1 + h_batch][M][F]
    LossGemmArgs g2b = g2;
    g2b.qdq_W = nullptr;  // the batched second GEMM reads no candidate operand
    g2b.a_slotted = 1;
    g2b.a_slots = 1 + h_batch;
    if ((e = make_operand_maps(g1, &a1, &b1, &why, kTileN)) != cudaSuccess ||
        (e = make_operand_maps(g2, &a2, &b2, &why, kTileN)) != cudaSuccess ||
        (fused && (e = make_operand_maps(g2b, &a2b, &b2b, &why, kTileN)) != cudaSuccess)) {
      status = set_error(AWQ_ERR_CUDA, std::string("TMA descriptor: ") + why);
      break;
    }
    g2.n_grid = 1;  // one candidate per launch
    if (fused) {
      // reference block: h_0 = block intermediate with bf16(W), then Y = h_0 W_down^T
      g1.slot_base = 0;
      g1.cands = 1;
      g1.qdq_cands = g2.qdq_cands = 2;  // the QDQ warps claim candidate pieces while these run
      if ((e = launch_loss_gemm(g1, a1, b1, 3, s, &launches)) != cudaSuccess) { where = "block GEMM 1"; break; }
      g2.partial = part;
      if ((e = launch_loss_gemm(g2, a2, b2, 0, s, &launches)) != cudaSuccess) { where = "block GEMM 2"; break; }
      g1.qdq_cands = 1;   // ... and the rest during the candidates' first GEMM, which then walks
      g1.cand_inner = qdq_warps ? 1 : 0;  // every candidate of an operand tile before the next
      for (int c0 = 0; c0 < n_grid && e == cudaSuccess; c0 += h_batch) {
        const int nb = std::min(h_batch, n_grid - c0);
        g1.slot_base = 1 + c0;  // candidate c0 + i in B slot 1 + c0 + i ...
        g1.cands = nb;
        g1.H = h + h_bytes / 2;  // ... writes h slot 1 + i
        g1.h_stride = h_bytes / 2;
        if ((e = launch_loss_gemm(g1, a1, b1, 3, s, &launches)) != cudaSuccess) { where = "block GEMM 1"; break; }
        g2b.a_slot_base = 1;
        g2b.cands = nb;
        g2b.b_per_cand = 0;  // every candidate against the same W_down
        g2b.slot_base = 0;
        g2b.n_grid = nb;
        g2b.partial = part + static_cast<int64_t>(c0) * tiles2;
        if ((e = launch_loss_gemm(g2b, a2b, b2b, 1, s, &launches)) != cudaSuccess) { where = "block GEMM 2"; break; }
      }
    } else {
      for (int c = -1; c < n_grid && e == cudaSuccess; ++c) {
        g1.slot_base = c + 1;  // slot 0: bf16(W), the reference block
        if ((e = launch_loss_gemm(g1, a1, b1, 2, s, &launches)) != cudaSuccess) { where = "block GEMM 1"; break; }
        if ((e = launch_silu_mul(H, M, F, h, s, &launches)) != cudaSuccess) { where = "silu-mul kernel"; break; }
        g2.partial = part + static_cast<int64_t>(c < 0 ? 0 : c) * tiles2;
        if ((e = launch_loss_gemm(g2, a2, b2, c < 0 ? 0 : 1, s, &launches)) != cudaSuccess) {
          where = "block GEMM 2";
          break;
        }
      }
    }
    if (e != cudaSuccess) break;
    if ((e = launch_loss_reduce(part, tiles2, n_grid, M, K_out, losses, s, &launches)) != cudaSuccess) {
      where = "loss reduction kernel";
      break;
    }
    if ((e = launch_pack(W_gu, in_dtype, K, N, group, n_grid, S, losses, best, out_codes,
                         static_cast<__half*>(out_steps), static_cast<__half*>(out_zeros), out_scales, s,
                         &launches)) != cudaSuccess) {
      where = "pack kernel";
      break;
    }
    if (out_losses &&
        (e = cudaMemcpyAsync(out_losses, losses, static_cast<size_t>(n_grid) * 4, cudaMemcpyDeviceToDevice, s)) !=
            cudaSuccess) {
      where = "copy of the losses";
      break;
    }
    if (out_best && (e = cudaMemcpyAsync(out_best, best, sizeof(int32_t), cudaMemcpyDeviceToDevice, s)) != cudaSuccess) {
      where = "copy of the chosen index";
      break;
    }
  } while (false);
  int* pinned = pinned_status_word(dev);
  int* status_dst = pinned ? pinned : &h_err;
  if (status == AWQ_OK && e == cudaSuccess) {
    e = cudaMemcpyAsync(status_dst, err, sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) where = "status read-back";
  }
  if (status == AWQ_OK && e != cudaSuccess) status = cuda_error(e, where);
  cudaFreeAsync(ws, s);
  cudaError_t se = cudaStreamSynchronize(s);
  if (status == AWQ_OK && se != cudaSuccess) status = cuda_error(se, "stream synchronize");
  if (pinned) h_err = *pinned;
  if (status == AWQ_OK) {
    g_last_launches = launches;
    if (h_err & kErrTimeout)
      status = set_error(AWQ_ERR_TIMEOUT, "a bounded wait in a block GEMM ran out");
    else if (h_err & (kErrNonfiniteX | kErrNonfiniteW))
      status = set_error(AWQ_ERR_NONFINITE, (h_err & kErrNonfiniteX) ? "non-finite value in X" : "non-finite value in W");
    else if (h_err)
      status = set_error(AWQ_ERR_CUDA, "device status word " + std::to_string(h_err));
  }
  return status;
}

// ---- module-level objective: an attention block ----------------------------------------
// Phase events of the last profiled attention-block search: QDQ, the Q|K GEMM, the V^T
// GEMM, the reference attention, the candidates' attention with the fused loss, and the
// loss reduction with the artifact.
constexpr int kAttnPhases = 6;
float g_attn_ms[kAttnPhases] = {0};
cudaEvent_t* attn_events(int dev) {
  static cudaEvent_t ev[64][kAttnPhases + 1];
  static bool made[64] = {false};
  if (dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!made[dev]) {
    for (auto& e : ev[dev])
      if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    made[dev] = true;
  }
  return ev[dev];
}

int awq_search_attn(const void* X, const void* W_qkv, int in_dtype, int64_t M, int64_t K, int64_t D, int n_heads,
                    int64_t seq_len, int group, int n_grid, float* out_scales, int32_t* out_codes, void* out_steps,
                    void* out_zeros, float* out_losses, int32_t* out_best, awq_stream_t stream) {
  t_last_error.clear();
  int st = validate(X, W_qkv, in_dtype, M, K, 3 * D, group, n_grid, out_scales, out_codes, out_steps, out_zeros, true);
  if (st != AWQ_OK) return st;
  if (n_heads < 1 || D != static_cast<int64_t>(n_heads) * kAttnHeadDim)
    return set_error(AWQ_ERR_SHAPE, "D must be n_heads * 128 (heads of dimension 128)");
  if (seq_len < 128 || seq_len > kAttnMaxSeq || seq_len % 128 || M % seq_len)
    return set_error(AWQ_ERR_SHAPE, "seq_len must be 128, 256, 384 or 512 and divide M");
  if ((out_losses && (reinterpret_cast<uintptr_t>(out_losses) & 3u)) ||
      (out_best && (reinterpret_cast<uintptr_t>(out_best) & 3u)))
    return set_error(AWQ_ERR_INVALID_ARG, "out_losses / out_best misaligned");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DeviceRestore restore_device;
  bind_device(s, X);
  int dev = 0, num_sms = 0;
  if ((st = check_device(&dev, &num_sms)) != AWQ_OK) return st;
  if (!is_device_memory(X) || !is_device_memory(W_qkv) || !is_device_memory(out_scales) ||
      !is_device_memory(out_codes) || !is_device_memory(out_steps) || !is_device_memory(out_zeros) ||
      (out_losses && !is_device_memory(out_losses)) || (out_best && !is_device_memory(out_best)))
    return set_error(AWQ_ERR_INVALID_ARG, "inputs and outputs must be device memory");
  const int64_t N = 3 * D;
  const int slots = n_grid + 1;  // slot 0: bf16(W), slot 1 + i: candidate i
  const int64_t units = (M / seq_len) * n_heads * (seq_len / 128);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align_up(bytes);
    return at;
  };
  // bf16 W with group 128: the Q|K GEMM's QDQ warps make the candidate operands of
  // [W_q | W_k] (while that GEMM walks every slot of an operand tile before the next) and
  // then of W_v (which the V^T GEMM, the next launch, reads)
  const bool qdq_warps = qdq_in_loss_gemm(in_dtype, group, 1, M, K, N, n_grid);
  const size_t flag_bytes = 16 + static_cast<size_t>(ceil_div(2 * D, kTileN) + 1) * 4;  // status word, QDQ counters
  const size_t o_err = take(flag_bytes), o_a = take(static_cast<size_t>(K) * 4), o_S = take(static_cast<size_t>(n_grid) * K * 4),
               o_best = take(16), o_losses = take(static_cast<size_t>(n_grid) * 4),
               o_Xb = in_dtype == AWQ_DTYPE_F32 ? take(static_cast<size_t>(M) * K * 2) : 0,
               o_Wqk = take(static_cast<size_t>(slots) * 2 * D * K * 2),
               o_Wv = take(static_cast<size_t>(slots) * D * K * 2),
               o_QK = take(static_cast<size_t>(slots) * M * 2 * D * 2),
               o_VT = take(static_cast<size_t>(slots) * D * M * 2),
               o_O = take(static_cast<size_t>(M) * D * 4),
               o_part = take(static_cast<size_t>(n_grid) * units * 8);
  cudaMemPool_t pool;
  if ((st = get_pool(dev, &pool)) != AWQ_OK) return st;
  void* ws = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(&ws, off, pool, s);
  if (e != cudaSuccess || !ws) {
    cudaGetLastError();
    return set_error(AWQ_ERR_OOM, "work space of " + std::to_string(off) + " bytes");
  }
  uint8_t* b = static_cast<uint8_t*>(ws);
  int* err = reinterpret_cast<int*>(b + o_err);
  float* a = reinterpret_cast<float*>(b + o_a);
  float* S = reinterpret_cast<float*>(b + o_S);
  int* best = reinterpret_cast<int*>(b + o_best);
  float* losses = reinterpret_cast<float*>(b + o_losses);
  __nv_bfloat16* Wqk = reinterpret_cast<__nv_bfloat16*>(b + o_Wqk);
  __nv_bfloat16* Wv = reinterpret_cast<__nv_bfloat16*>(b + o_Wv);
  __nv_bfloat16* QK = reinterpret_cast<__nv_bfloat16*>(b + o_QK);
  __nv_bfloat16* VT = reinterpret_cast<__nv_bfloat16*>(b + o_VT);
  float* O_ref = reinterpret_cast<float*>(b + o_O);
  double* part = reinterpret_cast<double*>(b + o_part);
  const __nv_bfloat16* Xb = in_dtype == AWQ_DTYPE_F32 ? reinterpret_cast<__nv_bfloat16*>(b + o_Xb)
                                                      : static_cast<const __nv_bfloat16*>(X);
  const size_t eb = in_dtype == AWQ_DTYPE_F32 ? 4 : 2;
  const void* W_v = static_cast<const uint8_t*>(W_qkv) + 2 * D * eb;  // columns 2D .. 3D - 1 of each row
  cudaEvent_t* ev = g_profile ? attn_events(dev) : nullptr;
  auto mark = [&](int i) {
    if (ev) cudaEventRecord(ev[i], s);
  };
  int launches = 0, h_err = 0, status = AWQ_OK;
  const char* where = "";
  do {
    if ((e = cudaMemsetAsync(err, 0, flag_bytes, s)) != cudaSuccess) { where = "cudaMemsetAsync"; break; }
    mark(0);
    if ((e = launch_statistic(X, in_dtype, M, K, a, err, s, &launches)) != cudaSuccess) {
      where = "statistic kernel";
      break;
    }
    if ((e = launch_scales(a, K, n_grid, S, s, &launches)) != cudaSuccess) { where = "scales kernel"; break; }
    if (in_dtype == AWQ_DTYPE_F32 &&
        (e = launch_to_bf16(static_cast<const float*>(X), M * K, const_cast<__nv_bfloat16*>(Xb), s, &launches)) !=
            cudaSuccess) {
      where = "bf16 operand kernel";
      break;
    }
    // the query and key columns, then the value columns, each into a stack of K-major slots
    // (with the QDQ warps, the reference slot alone)
    const int qdq_slots = qdq_warps ? 0 : n_grid;
    if ((e = launch_qdq(W_qkv, in_dtype, K, 2 * D, group, qdq_slots, S, Wqk, err, s, &launches, kQuantAsym, 0, N)) !=
            cudaSuccess ||
        (e = launch_qdq(W_v, in_dtype, K, D, group, qdq_slots, S, Wv, err, s, &launches, kQuantAsym, 0, N)) !=
            cudaSuccess) {
      where = "qdq kernel";
      break;
    }
    mark(1);
    // [Q | K] of every slot: X_b [M][K] times the slot's [W_q | W_k] (mode 5, bf16 out)
    LossGemmArgs g;
    g.Xb = Xb;
    g.Wt = Wqk;
    g.M = M;
    g.K = K;
    g.N = 2 * D;
    g.n_grid = n_grid;
    g.Y = nullptr;
    g.partial = nullptr;
    g.err = err;
    g.timeout_ns = g_timeout_ns;
    g.fault_mode = 0;
    g.num_sms = num_sms;
    g.H = QK;
    g.h_stride = M * 2 * D;
    g.cands = slots;
    g.slot_base = 0;
    g.b_per_cand = 1;
    if (qdq_warps) {
      g.qdq_W = static_cast<const __nv_bfloat16*>(W_qkv);
      g.qdq_S = S;
      g.qdq_Wt = Wqk;
      g.qdq_ready = err + 4;
      g.qdq_cands = 1;
      g.qdq_K = K;
      g.qdq_N = 2 * D;
      g.qdq_ldw = N;
      g.qdq_grid = n_grid;
      g.qdq_W2 = static_cast<const __nv_bfloat16*>(W_v);
      g.qdq_Wt2 = Wv;
      g.qdq_N2 = D;
      g.cand_inner = 1;  // every slot of an operand tile before the next
    }
    // V^T of every slot: the slot's W_v^T [D][K] (a stack of A operands) times X_b
    LossGemmArgs gv = g;
    gv.qdq_W = nullptr;  // W_v's slots are complete when this launch starts
    gv.qdq_W2 = nullptr;
    gv.cand_inner = 0;
    gv.Xb = Wv;
    gv.a_slotted = 1;
    gv.a_slots = slots;
    gv.a_slot_base = 0;
    gv.M = D;
    gv.Wt = Xb;
    gv.N = M;
    gv.n_grid = 0;  // one B slot for the tensor map
    gv.H = VT;
    gv.h_stride = D * M;
    gv.b_per_cand = 0;
    CUtensorMap mA, mB, vA, vB;
    const char* why = "";
    if ((e = make_operand_maps(g, &mA, &mB, &why, kTileN)) != cudaSuccess ||
        (e = make_operand_maps(gv, &vA, &vB, &why, kTileN)) != cudaSuccess) {
      status = set_error(AWQ_ERR_CUDA, std::string("TMA descriptor: ") + why);
      break;
    }
    if ((e = launch_loss_gemm(g, mA, mB, 5, s, &launches)) != cudaSuccess) { where = "Q|K GEMM"; break; }
    mark(2);
    if ((e = launch_loss_gemm(gv, vA, vB, 5, s, &launches)) != cudaSuccess) { where = "V^T GEMM"; break; }
    mark(3);
    AttnLossArgs at;
    at.QK = QK;
    at.VT = VT;
    at.total_slots = slots;
    at.M = M;
    at.D = D;
    at.T = seq_len;
    at.n_heads = n_heads;
    at.O_ref = O_ref;
    at.partial = part;
    at.err = err;
    at.timeout_ns = g_timeout_ns;
    at.num_sms = num_sms;
    at.fault_mode = g_fault_mode;
    at.slot0 = 0;
    at.slots = 1;
    if ((e = launch_attn_loss(at, 1, s, &launches)) != cudaSuccess) { where = "reference attention"; break; }
    mark(4);
    at.slot0 = 1;
    at.slots = n_grid;
    if ((e = launch_attn_loss(at, 0, s, &launches)) != cudaSuccess) { where = "candidate attention"; break; }
    mark(5);
    if ((e = launch_loss_reduce(part, units, n_grid, M, D, losses, s, &launches)) != cudaSuccess) {
      where = "loss reduction kernel";
      break;
    }
    if ((e = launch_pack(W_qkv, in_dtype, K, N, group, n_grid, S, losses, best, out_codes,
                         static_cast<__half*>(out_steps), static_cast<__half*>(out_zeros), out_scales, s,
                         &launches)) != cudaSuccess) {
      where = "pack kernel";
      break;
    }
    mark(6);
    if (out_losses &&
        (e = cudaMemcpyAsync(out_losses, losses, static_cast<size_t>(n_grid) * 4, cudaMemcpyDeviceToDevice, s)) !=
            cudaSuccess) {
      where = "copy of the losses";
      break;
    }
    if (out_best && (e = cudaMemcpyAsync(out_best, best, sizeof(int32_t), cudaMemcpyDeviceToDevice, s)) != cudaSuccess) {
      where = "copy of the chosen index";
      break;
    }
  } while (false);
  int* pinned = pinned_status_word(dev);
  int* status_dst = pinned ? pinned : &h_err;
  if (status == AWQ_OK && e == cudaSuccess) {
    e = cudaMemcpyAsync(status_dst, err, sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) where = "status read-back";
  }
  if (status == AWQ_OK && e != cudaSuccess) status = cuda_error(e, where);
  cudaFreeAsync(ws, s);
  cudaError_t se = cudaStreamSynchronize(s);
  if (status == AWQ_OK && se != cudaSuccess) status = cuda_error(se, "stream synchronize");
  if (pinned) h_err = *pinned;
  if (status == AWQ_OK) {
    g_last_launches = launches;
    if (ev)
      for (int i = 0; i < kAttnPhases; ++i) cudaEventElapsedTime(&g_attn_ms[i], ev[i], ev[i + 1]);
    status = status_from_word(h_err);
  }
  return status;
}

int awq_attn_profile_last(float* ms, int n) {
  for (int i = 0; i < n && i < kAttnPhases; ++i) ms[i] = g_attn_ms[i];
  return kAttnPhases;
}

int awq_clip_profile_last(float* ms, int n) {
  for (int i = 0; i < n && i < 2; ++i) ms[i] = g_clip_ms[i];
  return 2;
}

int awq_fp64_mma_peak(double* tflops, awq_stream_t stream) {
  t_last_error.clear();
  if (!tflops) return set_error(AWQ_ERR_INVALID_ARG, "tflops is NULL");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DeviceRestore restore_device;
  bind_device(s, nullptr);
  int dev = 0, num_sms = 0, st;
  if ((st = check_device(&dev, &num_sms)) != AWQ_OK) return st;
  cudaMemPool_t pool;
  if ((st = get_pool(dev, &pool)) != AWQ_OK) return st;
  const int blocks = 4 * num_sms, iters = 4096;
  void* out = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(&out, static_cast<size_t>(blocks) * 256 * sizeof(double), pool, s);
  if (e != cudaSuccess || !out) {
    cudaGetLastError();
    return set_error(AWQ_ERR_OOM, "probe buffer");
  }
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  float ms = 0.0f;
  if ((e = cudaEventCreate(&e0)) == cudaSuccess && (e = cudaEventCreate(&e1)) == cudaSuccess &&
      (e = launch_fp64_mma_peak(static_cast<double*>(out), blocks, iters, s)) == cudaSuccess &&
      (e = cudaEventRecord(e0, s)) == cudaSuccess &&
      (e = launch_fp64_mma_peak(static_cast<double*>(out), blocks, iters, s)) == cudaSuccess &&
      (e = cudaEventRecord(e1, s)) == cudaSuccess && (e = cudaEventSynchronize(e1)) == cudaSuccess)
    e = cudaEventElapsedTime(&ms, e0, e1);
  cudaFreeAsync(out, s);
  cudaError_t se = cudaStreamSynchronize(s);
  if (e0) cudaEventDestroy(e0);
  if (e1) cudaEventDestroy(e1);
  if (e != cudaSuccess) return cuda_error(e, "fp64 MMA probe");
  if (se != cudaSuccess) return cuda_error(se, "stream synchronize");
  // per launch: blocks x 8 warps x iters x 8 MMAs of 8 x 8 x 4 multiply-adds
  const double flops = 2.0 * blocks * 8.0 * iters * 8.0 * 256.0;
  *tflops = ms > 0.0f ? flops / (ms * 1e-3) / 1e12 : 0.0;
  return AWQ_OK;
}

int64_t awq_clip_token_count(int64_t M, int64_t max_tokens) {
  if (M <= 0 || max_tokens <= 0) return 0;
  return clip_token_count(M, max_tokens);
}

void awq_tile_shape(int* tile_m, int* tile_n) {
  if (tile_m) *tile_m = kTileM;
  if (tile_n) *tile_n = kTileN;
}

int64_t awq_workspace_bytes(int in_dtype, int64_t M, int64_t K, int64_t N, int group, int n_grid) {
  static int dummy;
  if (validate(&dummy, &dummy, in_dtype, M, K, N, group, n_grid, &dummy, &dummy, &dummy, &dummy, false) != AWQ_OK)
    return 0;
  return static_cast<int64_t>(plan(in_dtype, M, K, N, n_grid).total);
}

int awq_release_cached(void) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return set_error(AWQ_ERR_CUDA, "cudaGetDevice");
  std::lock_guard<std::mutex> lock(g_mu);
  auto it = g_pools.find(dev);
  if (it == g_pools.end()) return AWQ_OK;
  cudaError_t e = cudaMemPoolTrimTo(it->second, 0);
  return e == cudaSuccess ? AWQ_OK : cuda_error(e, "cudaMemPoolTrimTo");
}

const char* awq_status_string(int status) {
  switch (status) {
    case AWQ_OK: return "AWQ_OK";
    case AWQ_ERR_INVALID_ARG: return "AWQ_ERR_INVALID_ARG";
    case AWQ_ERR_SHAPE: return "AWQ_ERR_SHAPE";
    case AWQ_ERR_NONFINITE: return "AWQ_ERR_NONFINITE";
    case AWQ_ERR_OOM: return "AWQ_ERR_OOM";
    case AWQ_ERR_CUDA: return "AWQ_ERR_CUDA";
    case AWQ_ERR_TIMEOUT: return "AWQ_ERR_TIMEOUT";
    case AWQ_ERR_UNSUPPORTED_DEVICE: return "AWQ_ERR_UNSUPPORTED_DEVICE";
    default: return "AWQ_ERR_UNKNOWN";
  }
}

const char* awq_last_error_message(void) { return t_last_error.c_str(); }

int awq_profile_enable(int on) {
  g_profile = on != 0;
  return AWQ_OK;
}

int awq_profile_last(float* ms, int n) {
  for (int i = 0; i < n && i < kNumPhases; ++i) ms[i] = g_phase_ms[i];
  return kNumPhases;
}

int64_t awq_profile_last_ticket(void) { return t_last_ticket; }

int awq_profile_collect(int64_t ticket, float* ms, int n) {
  if (!ms || n < 0) return -1;
  float all[kNumPhases];
  if (!Events::collect_ticket(ticket, all)) return -1;
  for (int i = 0; i < n && i < kNumPhases; ++i) ms[i] = all[i];
  return kNumPhases;
}

const char* awq_profile_phase_name(int phase) {
  return (phase >= 0 && phase < kNumPhases) ? kPhaseNames[phase] : "";
}

int awq_last_launch_count(void) { return g_last_launches; }

int awq_debug_set_fault(int mode, int64_t timeout_ns) {
  if (mode != 0 && mode != 1 && mode != 3) return set_error(AWQ_ERR_INVALID_ARG, "fault mode must be 0, 1 or 3");
  g_fault_mode = mode;
  g_timeout_ns = timeout_ns > 0 ? static_cast<uint64_t>(timeout_ns) : kDefaultTimeoutNs;
  return AWQ_OK;
}

int awq_version(void) { return kVersion; }

int awq_loss_gemm_variant(int64_t M, int64_t K, int64_t N, int n_grid) { return gemm_variant(M, K, N, n_grid); }

int awq_loss_gemm_launches(int in_dtype, int64_t M, int64_t K, int64_t N, int group, int n_grid) {
  const int variant = gemm_variant(M, K, N, n_grid);
  if (variant == 2 || qdq_in_loss_gemm(in_dtype, group, variant, M, K, N, n_grid)) return 2;
  int dev = 0, l2_bytes = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&l2_bytes, cudaDevAttrL2CacheSize, dev);
  if (e != cudaSuccess) return -cuda_error(e, "querying the L2 cache size");
  return reference_in_own_launch(M, N, l2_bytes) ? 2 : 1;
}

int awq_qdq_in_loss_gemm(int in_dtype, int64_t M, int64_t K, int64_t N, int group, int n_grid) {
  return qdq_in_loss_gemm(in_dtype, group, gemm_variant(M, K, N, n_grid), M, K, N, n_grid) ? 1 : 0;
}

}  // extern "C"
