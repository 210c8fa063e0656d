// awq_kernels.h — host-side launchers of the search kernels (internal to libawqsearch).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace awq {

// Loss GEMM tile: BM rows of X by BN columns of W per output tile.
constexpr int kTileM = 128;
constexpr int kTileN = 256;
constexpr int kTileK = 64;

// ---- statistic (AWQ-P1 §1) -------------------------------------------------------
cudaError_t launch_statistic(const void* X, int in_dtype, int64_t M, int64_t K, float* a, int* err, cudaStream_t s,
                             int* launches);

// ---- candidate scales (AWQ-P1 §3-§4) ---------------------------------------------
cudaError_t launch_scales(const float* a, int64_t K, int n_grid, float* S, cudaStream_t s,
                          int* launches);

// ---- fp32 -> bf16 operand copy (fp32 layers only) --------------------------------
cudaError_t launch_to_bf16(const float* x, int64_t n, __nv_bfloat16* out, cudaStream_t s,
                           int* launches);

// ---- scale + QDQ + fold-back of every candidate (AWQ-P1 §4, §7) -------------------
// `quantizer`: 0 the asymmetric zero-point quantizer (AWQ-P1 §7), 1 the symmetric [-7, 7]
// teaching quantizer (AWQ-P1 §2), stored as codes q + 7 with zero point 7.
// Writes Wt[0] = bf16(W)^T and Wt[1 + i] = bf16(W_hat_i)^T, each N x K (K contiguous).
// `interleave` = F > 0 (N = 2F, F % 128 == 0) writes the columns of [W_gate | W_up] in the
// order the fused MLP GEMM reads them: every 256 rows are 128 gate columns followed by the
// 128 up columns of the same outputs. `ldw` > 0: W's rows are ldw elements apart (N columns
// of a wider matrix, e.g. the key or value part of [W_q | W_k | W_v]); 0 means N.
cudaError_t launch_qdq(const void* W, int in_dtype, int64_t K, int64_t N, int group, int n_grid,
                       const float* S, __nv_bfloat16* Wt, int* err, cudaStream_t s, int* launches,
                       int quantizer = 0, int64_t interleave = 0, int64_t ldw = 0);
// The same for the groups group0 .. group0 + groups - 1 only (rows group0*group ..).
cudaError_t launch_qdq_groups(const void* W, int in_dtype, int64_t K, int64_t N, int group, int n_grid,
                              const float* S, __nv_bfloat16* Wt, int* err, int64_t group0, int64_t groups,
                              cudaStream_t s, int* launches, int quantizer = 0, int64_t interleave = 0,
                              int64_t ldw = 0);

// ---- artifact of the chosen candidate (AWQ-P1 §7; QUANT-P4 §5.3) ------------------
// The chosen candidate is the first minimum of `losses` (AWQ-P1 §3); its index is
// also written to *best.
cudaError_t launch_pack(const void* W, int in_dtype, int64_t K, int64_t N, int group, int n_grid, const float* S,
                        const float* losses, int* best, int32_t* codes, __half* steps, __half* zeros,
                        float* out_scales, cudaStream_t s, int* launches, int quantizer = 0);

// ---- loss GEMM (AWQ-P1 §4) ---------------------------------------------------------
struct LossGemmArgs {
  const __nv_bfloat16* Xb;   // [M][K]
  const __nv_bfloat16* Wt;   // [n_grid + 1][N][K]
  int64_t M, K, N;
  int n_grid;
  float* Y;                  // tiled reference output, tiles_m * tiles_n * BM * BN floats
  double* partial;           // [n_grid][tiles_m * tiles_n]
  int* err;
  uint64_t timeout_ns;
  int fault_mode;
  int num_sms;
  int f16 = 0;               // mode 2 only: fp16 operands (the tensor maps move 2-byte elements either way)
  int variant = 1;           // 1 the one-SM kernel, 2 the two-SM kernel (modes 0 and 1, slot_base 1)
  int slot_base = 1;         // B slot of candidate 0 (mode 1; the search's slot 0 is bf16(W)) or the
                             // slot multiplied (modes 2, 3); values other than 1 run on the one-SM kernel
  __nv_bfloat16* H = nullptr;  // mode 3: the MLP block's intermediate h, M x N/2 row-major bf16; mode 5: the output
  int64_t h_stride = 0;        // modes 3, 5: elements between successive candidates' outputs
  int cands = 0;               // modes 1, 3, 5: candidates this launch walks (0: n_grid for mode 1, else 1)
  int b_per_cand = 1;          // modes 1, 3, 5: candidate c reads B slot slot_base + c (1) or slot_base (0)
  int a_slotted = 0;           // A is a stack of a_slots operands [a_slots][M][K]; c reads a_slot_base + c
  int a_slot_base = 0;
  int a_slots = 1;
  int* ready = nullptr;        // mode 4: per-tile flags (tiles_m * tiles_n ints), zero at launch
  int cand_inner = 0;          // mode 1: walk raster group -> column tile -> candidate -> row tile, so
                               // that every candidate reads a tile of Y while it is still in L2
  // The one-SM kernel with bf16 W and group 128: when qdq_W is set, eight more warps per
  // CTA make candidate operand slots (the QDQ of the candidate loop; slot 0 comes from
  // launch_qdq with n_grid = 0) while the tensor cores run, claiming pieces (a 128 x 32
  // tile of W, a chunk of candidates) column-major from a counter that spans a search's
  // launches (qdq_cands 2: while this CTA's GEMM runs; 1: until none is left). A load of a
  // candidate slot's 256-row tile (mode 1, or modes 3 and 5 past slot 0; those launches read
  // qdq_Wt with the QDQ's K and N) waits (bounded) until that tile is complete for every
  // candidate. Mode 0 may host the warps for another GEMM (the MLP block's reference down
  // projection). qdq_interleave = F for the MLP block's [W_gate | W_up]. qdq_ready:
  // ceil(qdq_N / 256) + 1 ints, zero before the first launch.
  // The attention block's Q|K launch (mode 5) also makes W_v's slots: qdq_W2 (columns of
  // the same rows, pitch qdq_ldw) into qdq_Wt2, after the first operand, without counters
  // (only the next launch reads them).
  const __nv_bfloat16* qdq_W = nullptr;  // [qdq_K][qdq_N], row pitch qdq_ldw (0: qdq_N)
  const float* qdq_S = nullptr;          // [qdq_grid][qdq_K]
  __nv_bfloat16* qdq_Wt = nullptr;       // [qdq_grid + 1][qdq_N][qdq_K]
  int* qdq_ready = nullptr;
  int qdq_cands = 0;
  int qdq_quantizer = 0;
  int64_t qdq_K = 0, qdq_N = 0, qdq_interleave = 0, qdq_ldw = 0;
  int qdq_grid = 0;
  const __nv_bfloat16* qdq_W2 = nullptr;  // [qdq_K][qdq_N2], row pitch qdq_ldw
  __nv_bfloat16* qdq_Wt2 = nullptr;       // [qdq_grid + 1][qdq_N2][qdq_K]
  int64_t qdq_N2 = 0;
};
// Whether a search scores its candidates in two launches (mode 0, then mode 1 with
// cand_inner) rather than one mode-4 launch: when the reference output Y (M x N fp32) is
// larger than the L2 cache, so that a walk with the candidate outermost would read all of Y
// from DRAM once per candidate. AWQ_REFERENCE_LAUNCH=own or =fused in the environment
// selects a form at every size (both give bit-identical results).
bool reference_in_own_launch(int64_t M, int64_t N, int l2_bytes);
// Whether a search makes its candidate operands with the loss GEMM's QDQ warps (bf16 W,
// group 128, the one-SM kernel, below 100 TFLOP of candidate GEMM work) rather than with
// qdq_kernel before it. AWQ_QDQ=standalone or =warps in the environment selects a form
// at every size (both give bit-identical operands).
bool qdq_in_loss_gemm(int in_dtype, int group, int variant, int64_t M, int64_t K, int64_t N, int n_grid);
// Which loss GEMM runs for a search of this size: 1 = the one-SM kernel (every size; it
// measured as fast or faster than the pair kernel on every workload), 2 = the two-SM
// (cta_group::2) kernel, selected with AWQ_GEMM_VARIANT=2 in the environment.
int gemm_variant(int64_t M, int64_t K, int64_t N, int n_grid);
// Rows of the W_hat box one CTA loads: the full 256-column tile, or half of it when a
// CTA pair shares the tile.
inline int operand_b_box_rows(int variant) { return variant == 2 ? kTileN / 2 : kTileN; }
// Builds the TMA descriptors (driver entry point) for the two operands.
cudaError_t make_operand_maps(const LossGemmArgs& a, CUtensorMap* mapA, CUtensorMap* mapB,
                              const char** why, int b_box_rows);
// mode 0: Y = X_b W_b into the tiled buffer; mode 1: per-tile sum of (X_b W_hat_i - Y)^2
// (candidate outermost, or innermost but one with a.cand_inner);
// mode 2: Y = X_b Wt[0]^T written row-major fp32 into a.Y (M x N, pitch N), always on
// the one-SM kernel (make the maps with b_box_rows = kTileN);
// mode 4: modes 0 and 1 in one launch (reference tiles first, flags in a.ready; one-SM
// kernel only; the grid never exceeds the SMs, so every awaited flag belongs to a running CTA);
// mode 3: the MLP block's first GEMM with the silu-mul fused in its epilogue: the B slot
// holds [W_gate | W_up] interleaved by 128 columns (launch_qdq's `interleave`), and
// h = bf16(fl32(silu(g) u)) is written row-major into a.H (M x N/2), one-SM kernel only;
// mode 5: for each of a.cands candidates (B slot slot_base + c when b_per_cand, A slot
// a_slot_base + c when a_slotted) the product rounded to bf16, row-major (pitch N) at
// a.H + c * a.h_stride, one-SM kernel only.
cudaError_t launch_loss_gemm(const LossGemmArgs& a, const CUtensorMap& mapA, const CUtensorMap& mapB,
                             int mode, cudaStream_t s, int* launches);

// Sum the tile partials of each candidate in a fixed order, divide by M*N, round to fp32.
cudaError_t launch_loss_reduce(const double* partial, int64_t tiles, int n_grid, int64_t M, int64_t N,
                               float* losses, cudaStream_t s, int* launches);

// ---- clipping search after the scaling (AWQ-P1 §5) ---------------------------------
struct ClipArgs {
  const void* X;       // [M][K], in_dtype
  const void* W;       // [K][N], in_dtype
  int in_dtype;
  const float* s;      // [K] the chosen scales
  int64_t M, K, N;
  int group, n_shrink;
  int64_t max_tokens;  // sampled tokens: every clip_token_stride-th row, at most max_tokens
  int tokens;          // clip_token_count(M, max_tokens)
  double* H;           // work space: [K / group][group][group]
  float* max_val;      // [K / group][N]
  int32_t* best;       // [K / group][N] or nullptr
  double* errors;      // [n_shrink][K / group][N] or nullptr
  int32_t* codes;      // [K][N / 8]
  __half* steps;       // [K / group][N]
  __half* zeros;       // [K / group][N]
  int* err;
  cudaEvent_t* ev;     // nullptr, or 3 events recorded around the two launches
  int quantizer;       // 0 asymmetric, 1 symmetric teaching quantizer
};
int64_t clip_token_stride(int64_t M, int64_t max_tokens);
int64_t clip_token_count(int64_t M, int64_t max_tokens);
// Gram matrices of the sampled scaled activations, then the per-(group, column) search
// and the clipped artifact: two launches.
cudaError_t launch_clip(const ClipArgs& a, cudaStream_t s, int* launches);
// Register-only loop of fp64 tensor-core MMAs (8 accumulators per warp, `iters` x 8
// MMAs of 8x8x4 per warp); `out` holds blocks * 256 doubles.
cudaError_t launch_fp64_mma_peak(double* out, int blocks, int iters, cudaStream_t s);

// ---- W4A16 consumer of the artifact (AWQ-P1 §7-§8) ---------------------------------
struct W4A16Args {
  const __half* A;        // [M][K] fp16 activations (already divided by the scales)
  const int32_t* codes;   // [K][N/8]
  const __half* steps;    // [K/group][N]
  const __half* zeros;    // [K/group][N]
  int64_t M, K, N;
  int group;
  float* Y;               // [M][N] fp32
};
constexpr int kW4A16GemvMaxM = 16;
// Fused dequantization + GEMV for M <= kW4A16GemvMaxM; `part` holds
// gemv_split_floats(...) floats when that is non-zero (a second launch sums the splits).
cudaError_t launch_w4a16_gemv(const W4A16Args& a, int num_sms, float* part, cudaStream_t s, int* launches);
int64_t gemv_split_floats(int64_t M, int64_t K, int64_t N, int group, int num_sms, bool packed = false);
// The codes in the decode kernel's order (N % 64 == 0): same size as the codes.
cudaError_t launch_w4a16_repack(const int32_t* codes, int64_t K, int64_t N, uint32_t* packed, cudaStream_t s,
                                int* launches);
// The decode GEMV on repacked codes (M <= kW4A16GemvMaxM, N % 64 == 0); `part` as above.
cudaError_t launch_w4a16_gemv_packed(const W4A16Args& a, const uint32_t* packed, int num_sms, float* part,
                                     cudaStream_t s, int* launches);
// w16 transposed: Wt[n][k] = fp16((q - z) step), N x K with K contiguous.
cudaError_t launch_w4a16_dequant(const int32_t* codes, const __half* steps, const __half* zeros, int64_t K, int64_t N,
                                 int group, __half* Wt, cudaStream_t s, int* launches);

// ---- MLP-block objective (AWQ-P1 §4: the candidate scored on the module output) -----
// h[m][f] = bf16(fl32(silu(H[m][f]) * H[m][F + f])), H = [X W_gate | X W_up] in fp32 (M x 2F).
cudaError_t launch_silu_mul(const float* H, int64_t M, int64_t F, __nv_bfloat16* h, cudaStream_t s, int* launches);
// Wt[o][f] = bf16(W[f][o]): the down projection as a K-major operand (in_dtype 0 bf16, 1 fp32).
cudaError_t launch_transpose_bf16(const void* W, int in_dtype, int64_t rows, int64_t cols, __nv_bfloat16* Wt,
                                  cudaStream_t s, int* launches);

// ---- attention-block objective (AWQ-P1 §4: the candidate scored on its module's output) --
// Causal multi-head attention of Q, K, V = bf16(X_b W_hat) over sequences of T tokens
// (T a multiple of 128, at most kAttnMaxSeq), heads kAttnHeadDim wide, with the loss
// against the reference output fused into the epilogue.
constexpr int kAttnHeadDim = 128;
constexpr int kAttnMaxSeq = 512;
struct AttnLossArgs {
  const __nv_bfloat16* QK;  // [total_slots][M][2D]: Q in columns 0 .. D-1, K in D .. 2D-1
  const __nv_bfloat16* VT;  // [total_slots][D][M]: V transposed
  int total_slots;          // slots in both stacks
  int slot0, slots;         // the slots this launch walks
  int64_t M, D, T;          // tokens, model width (n_heads * kAttnHeadDim), tokens per sequence
  int n_heads;
  float* O_ref;             // [M][D] fp32: written by the reference launch, read by the others
  double* partial;          // [slots][M / T * n_heads * T / 128] squared-error partials
  int* err;
  uint64_t timeout_ns;
  int num_sms;
  int fault_mode = 0;       // 1: the producer skips its first key tile (tests the bounded waits)
};
// ref = 1: O of slot slot0 stored into O_ref; ref = 0: per-unit squared error against it.
cudaError_t launch_attn_loss(const AttnLossArgs& a, int ref, cudaStream_t s, int* launches);

__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Raise a kernel's dynamic shared-memory limit to `bytes` once per device (the first
// launch on each device pays for the attribute call, later launches skip it).
template <typename Kernel>
cudaError_t set_smem_limit_once(Kernel kernel, int bytes, unsigned long long* done_mask) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (__atomic_load_n(done_mask, __ATOMIC_ACQUIRE) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) __atomic_fetch_or(done_mask, bit, __ATOMIC_ACQ_REL);
  return e;
}

// Sets the text awq_last_error_message returns on the calling thread.
void record_error_message(const char* msg);

// Puts the calling thread's current device back when an entry point returns: the entry
// points make the device of the caller's stream (or pointer) current for their own work.
struct DeviceRestore {
  int dev = -1;
  DeviceRestore() {
    if (cudaGetDevice(&dev) != cudaSuccess) {
      cudaGetLastError();
      dev = -1;
    }
  }
  ~DeviceRestore() {
    if (dev >= 0) cudaSetDevice(dev);
  }
  DeviceRestore(const DeviceRestore&) = delete;
  DeviceRestore& operator=(const DeviceRestore&) = delete;
};

// Work space the caller of the search provides instead of the library's pool: `bytes`
// long, its device address resolved by `resolve` once the call's device is current.
// A search given one allocates nothing (no pool block, no pinned status word, no
// profiling events) and reads the status word back into pageable host memory.
struct FixedWorkspace {
  size_t bytes;
  int (*resolve)(int dev, void** base);
};
// The search of awq_search_ex (plus the chosen index) in a fixed work space.
int search_in_workspace(const void* X, const void* W, int in_dtype, int64_t M, int64_t K, int64_t N, int group,
                        int n_grid, float* out_scales, int32_t* out_codes, void* out_steps, void* out_zeros,
                        float* out_losses, int32_t* out_best, cudaStream_t s, const FixedWorkspace& fixed);

}  // namespace awq
