/*
 * awq_search.h — C ABI of libawqsearch.so: AWQ's activation-aware per-layer scale
 * search on one NVIDIA B200 (sm_100a).
 *
 * The operation (cited by page title and section):
 *   [AWQ-P1] "AWQ：为什么 4-bit 权重量化要先观察 Activation" — §1 statistic,
 *            §3-§4 scale family, 20-point grid and forward-output loss,
 *            §7 asymmetric 4-bit zero-point quantizer, orientation and packing,
 *            §8 bits-per-weight budget.
 *   [AWQ-P2] "AWQ salient weight / GGUF compilation" — §二 scale formula.
 *   [QUANT-P4] "model-quantization / 05 core modules" — §5.3 int4 codes packed
 *            eight per int32 with separate scale tensors.
 *
 * For one linear layer with calibration activations X (M x K, row-major, K
 * contiguous) and weights W (K x N, row-major, N contiguous — the paper's
 * orientation: K input channels, N output channels; AWQ-P1 §1, §7):
 *   1. a_j = mean_m |X[m,j]|                       (fp64 sum, one rounding to fp32)
 *   2. for alpha_i = i/n_grid, i = 0..n_grid-1:
 *        raw_ij = max(a_j^alpha_i, 1e-4);  s_ij = raw_ij / sqrt(max_j raw_ij * min_j raw_ij)
 *   3. W' = diag(s_i) W, group-wise along K (`group` rows of one column):
 *        step = (max - min)/15 (1 for an all-equal group); z = clamp(rint(-min/step), 0, 15);
 *        q = clamp(rint(W'/step) + z, 0, 15)       (rint = round half to even)
 *   4. W_hat_i = diag(s_i)^-1 ((q - z) * step)     (fp32, then bf16 for the GEMM)
 *   5. L_i = ||X_b W_b - X_b W_hat_i,b||_F^2 / (M N)  (bf16 operands, fp32 accumulation,
 *        fp64 cross-tile sum; the reference output X_b W_b is computed once)
 *   6. i* = first argmin of the fp32 losses; emit s_i*, the codes, steps and zeros.
 *
 * Artifact layout (AWQ-P1 §7-§8, QUANT-P4 §5.3):
 *   out_scales [K]        fp32   s_i* (the activation is divided by it, W' multiplied)
 *   out_codes  [K][N/8]   int32  nibble i (bits 4i..4i+3) of word [k][w] = code of column 8w+i
 *   out_steps  [K/group][N] fp16 step of each (group, column), in the scaled domain
 *   out_zeros  [K/group][N] fp16 zero point (an integer 0..15)
 *   out_losses [n_grid]   fp32   L_i (optional, may be NULL)
 *   out_best   [1]        int32  i*, the index the library chose (the forms that take it;
 *                                may be NULL): alpha* = i* / n_grid
 *   Dequantized weight: W[k][n] ~= step[g][n] * (q[k][n] - zero[g][n]) / s[k], g = k/group.
 *   4 bits + 32/group bits per weight: 4.25 at group 128 (AWQ-P1 §8).
 *
 * Preconditions (AWQ-P1 §7 shape contract, plus this library's): M, K, N > 0;
 * group in {32, 64, 128}, K % group == 0; N % 8 == 0; 1 <= n_grid <= 64;
 * device pointers 16-byte aligned; K, N < 2^31, M < 2^31.
 *
 * Ownership: every pointer is owned by the caller; the library neither keeps nor
 * frees it. Device work space (candidate weights, the reference output, partial
 * sums) comes from a library-owned stream-ordered memory pool on the current
 * device, is allocated on `stream` and returned to the pool before the call
 * returns (the pool keeps its memory for later calls; awq_release_cached frees it).
 *
 * Streams: all device work is enqueued on `stream` (NULL = the legacy default
 * stream); the call then synchronizes `stream`, so the status reflects errors the
 * kernels detected (non-finite input, a wait that ran out). Each call runs on the
 * device that owns `stream` (or X, for the legacy default stream) and gives the
 * calling thread's current device back unchanged when it returns. Outputs are valid only
 * when the status is AWQ_OK. The library is not reentrant across host threads
 * that share a device (one call at a time per process is the tested use).
 *
 * Errors: every entry point returns an awq_status; awq_status_string names it and
 * awq_last_error_message gives the detail of the last failure on this thread.
 */
#ifndef AWQ_SEARCH_H_
#define AWQ_SEARCH_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream. */
typedef struct CUstream_st* awq_stream_t;

typedef enum awq_status {
  AWQ_OK = 0,
  AWQ_ERR_INVALID_ARG = 1,        /* NULL or misaligned pointer, bad n_grid/group/dtype */
  AWQ_ERR_SHAPE = 2,              /* M, K, N out of range; K % group; N % 8 */
  AWQ_ERR_NONFINITE = 3,          /* NaN or Inf in X or W (AWQ-P1 §2: finite reals only) */
  AWQ_ERR_OOM = 4,                /* device work space could not be allocated */
  AWQ_ERR_CUDA = 5,               /* a CUDA runtime/driver call failed */
  AWQ_ERR_TIMEOUT = 6,            /* a bounded wait inside a kernel ran out */
  AWQ_ERR_UNSUPPORTED_DEVICE = 7  /* the current device is not sm_100 */
} awq_status;

enum { AWQ_DTYPE_BF16 = 0, AWQ_DTYPE_F32 = 1 };

/* The candidates' quantizer. AWQ_QUANT_ASYM is the search's asymmetric zero-point
 * quantizer (AWQ-P1 §7, steps 3-4 below). AWQ_QUANT_SYM is the symmetric [-7, 7] absmax
 * teaching quantizer of AWQ-P1 §2: per (group, column) step = max|W'| / 7 (1 for an
 * all-zero group or when the quotient underflows), q = clamp(rint(W'/step), -7, 7),
 * reconstruction q * step; the artifact stores it in the same layout as codes q + 7
 * with zero point 7, so step * (code - zero) decodes both. */
enum { AWQ_QUANT_ASYM = 0, AWQ_QUANT_SYM = 1 };

/* The search on bf16 X [M][K] and bf16 W [K][N] (device pointers). */
int awq_search(const void* X, const void* W, int64_t M, int64_t K, int64_t N,
               int group, int n_grid, float* out_scales, int32_t* out_codes,
               void* out_steps, void* out_zeros, float* out_losses,
               awq_stream_t stream);

/* The same search on fp32 X and W (device pointers). The statistic, scales and
 * QDQ read the fp32 values; the loss GEMM takes them rounded to bf16. */
int awq_search_f32(const float* X, const float* W, int64_t M, int64_t K, int64_t N,
                   int group, int n_grid, float* out_scales, int32_t* out_codes,
                   void* out_steps, void* out_zeros, float* out_losses,
                   awq_stream_t stream);

/* Full form: `in_dtype` is AWQ_DTYPE_BF16 or AWQ_DTYPE_F32 for both X and W.
 * `out_best` (device, one int32, may be NULL) receives i*, the candidate the library
 * chose and packed: the first minimum of the fp32 losses it computed (AWQ-P1 §3: the
 * search keeps the first of equal losses), decided on the device by the kernel that
 * emits the artifact.
 * `out_tile_sq_err` (may be NULL) receives the fp64 squared-error partial sums the
 * loss GEMM produced: [n_grid][tiles_m][tiles_n], tile (tm, tn) covering rows
 * tm*tile_m .. and columns tn*tile_n .. (awq_tile_shape); L_i equals the sum of row i
 * divided by M*N. `tile_sq_err_len` is its capacity in elements. */
int awq_search_ex(const void* X, const void* W, int in_dtype, int64_t M, int64_t K,
                  int64_t N, int group, int n_grid, float* out_scales,
                  int32_t* out_codes, void* out_steps, void* out_zeros,
                  float* out_losses, int32_t* out_best, double* out_tile_sq_err,
                  int64_t tile_sq_err_len, awq_stream_t stream);

/* The search with the candidates quantized by `quantizer` (AWQ_QUANT_ASYM gives
 * awq_search_ex without tile partials). */
int awq_search_quant(const void* X, const void* W, int in_dtype, int64_t M, int64_t K,
                     int64_t N, int group, int n_grid, int quantizer, float* out_scales,
                     int32_t* out_codes, void* out_steps, void* out_zeros, float* out_losses,
                     int32_t* out_best, awq_stream_t stream);

/* Asynchronous form of awq_search_ex (no tile partials): enqueues the whole search on
 * `stream` and returns without waiting. Argument checks happen before anything is
 * enqueued and their errors are returned at once; errors the kernels detect (non-finite
 * input, a bounded wait that ran out) are reported through `status_word`, a 4-byte word
 * of PINNED host memory (cudaHostAlloc / cudaMallocHost) that the call's last copy
 * writes. After synchronizing `stream` the caller passes the word to awq_search_status,
 * which returns the call's status (AWQ_OK or the error awq_search_ex would have
 * returned) and sets awq_last_error_message. The outputs, the status word, X and W must stay
 * allocated until the stream has passed the call. Consecutive calls on one stream run
 * back to back, with no host round trip between them. */
int awq_search_async(const void* X, const void* W, int in_dtype, int64_t M, int64_t K,
                     int64_t N, int group, int n_grid, float* out_scales, int32_t* out_codes,
                     void* out_steps, void* out_zeros, float* out_losses, int32_t* out_best,
                     int32_t* status_word, awq_stream_t stream);
int awq_search_status(int32_t status_word);

/* End-to-end form with HOST buffers: copies X and W to the device on `stream`,
 * runs awq_search_ex, copies the outputs back (out_losses and out_best may be NULL;
 * out_best receives the chosen index as one int32). Pinned host memory makes the
 * copies asynchronous; pageable memory also works. */
int awq_search_host(const void* X_host, const void* W_host, int in_dtype, int64_t M,
                    int64_t K, int64_t N, int group, int n_grid, float* out_scales_host,
                    int32_t* out_codes_host, void* out_steps_host, void* out_zeros_host,
                    float* out_losses_host, int32_t* out_best_host, awq_stream_t stream);
/* The same for n_layers layers of one shape (X_hosts[i] M x K, W_hosts[i] K x N; the
 * output arrays hold one host pointer per layer, out_losses_host and out_best_host or
 * their entries may be NULL). Layer i + 1's inputs are copied to the device while layer i is searched (two
 * device slots) and layer i's artifact is copied back while layer i + 1 runs, so with
 * pinned host memory the transfers hide behind the searches. The whole batch is enqueued
 * at once and the call returns when every output has landed. A layer whose kernels
 * report a problem (non-finite input, a bounded wait that ran out) does not stop the
 * others: the call returns the status of the first such layer, and that layer's outputs
 * are undefined; an error while enqueueing stops the batch there. */
int awq_search_host_batch(int n_layers, const void* const* X_hosts, const void* const* W_hosts,
                          int in_dtype, int64_t M, int64_t K, int64_t N, int group, int n_grid,
                          float* const* out_scales_host, int32_t* const* out_codes_host,
                          void* const* out_steps_host, void* const* out_zeros_host,
                          float* const* out_losses_host, int32_t* const* out_best_host,
                          awq_stream_t stream);

/* ---- The steps one at a time (same kernels as awq_search; device pointers) ----
 * Step 1 (AWQ-P1 §1): out_a[K] = mean_m |X[m,j]| (fp64 sum, one rounding to fp32).
 * Returns AWQ_ERR_NONFINITE if X holds NaN or Inf. */
int awq_activation_statistic(const void* X, int in_dtype, int64_t M, int64_t K,
                             float* out_a, awq_stream_t stream);
/* Step 2 (AWQ-P1 §3-§4): out_S[n_grid][K], row i the scales of alpha_i = i/n_grid. */
int awq_candidate_scales(const float* a, int64_t K, int n_grid, float* out_S,
                         awq_stream_t stream);
/* Steps 3-4 (AWQ-P1 §4, §7): from W [K][N] and S [n_grid][K], the operands the loss
 * GEMM reads: out_wt [n_grid + 1][N][K] bf16, K contiguous; slot 0 = bf16(W)^T,
 * slot 1 + i = bf16(diag(s_i)^-1 Q(diag(s_i) W))^T. */
int awq_qdq_candidates(const void* W, int in_dtype, int64_t K, int64_t N, int group,
                       int n_grid, const float* S, void* out_wt, awq_stream_t stream);

/* Output tile of the loss GEMM (rows of X, columns of W). */
void awq_tile_shape(int* tile_m, int* tile_n);

/* Work space bytes one call needs for these sizes (0 on bad arguments). */
int64_t awq_workspace_bytes(int in_dtype, int64_t M, int64_t K, int64_t N, int group,
                            int n_grid);

/* Return the memory cached by the library's pool on the current device. */
int awq_release_cached(void);

const char* awq_status_string(int status);
/* Detail of the last failure on the calling thread (empty when none). */
const char* awq_last_error_message(void);

/* Per-phase device timing of the next calls: CUDA events recorded on `stream`
 * between the kernels of each call. awq_profile_last writes up to `n` phase
 * times (ms) of the last call and returns the number of phases. */
int awq_profile_enable(int on);
int awq_profile_last(float* ms, int n);
/* Profiled calls also get a ticket: awq_profile_last_ticket returns the calling thread's
 * last one (-1 if none); awq_profile_collect writes up to `n` phase times (ms) of that
 * call once its work has completed (e.g. an awq_search_async call after the stream has
 * been synchronized) and returns the number of phases, or -1 if the call is still
 * running or 256 later profiled calls on its device have reused its events. */
int64_t awq_profile_last_ticket(void);
int awq_profile_collect(int64_t ticket, float* ms, int n);
const char* awq_profile_phase_name(int phase);
/* Kernel launches the last call made (all of them this library's own kernels). */
int awq_last_launch_count(void);

/* Testing hook for the bounded waits: mode 1 makes the loss GEMM's producer skip
 * one stage's loads and arrive, so its consumer's wait runs out and the call
 * returns AWQ_ERR_TIMEOUT; mode 3 makes the loss GEMM's QDQ warps (bf16 W, group
 * 128) withhold one finished tile's count, so the producer's wait for that column
 * tile runs out, with the same result; `timeout_ns` bounds every wait (0 = the
 * default 2 s). Mode 0 restores normal operation. */
int awq_debug_set_fault(int mode, int64_t timeout_ns);

/* ---- Clipping search after the scaling ----------------------------------------
 * [AWQ-P1] §5: after the channel scaling, a few large weights can still stretch a
 * group's range; clipping trades them for a finer step. For each input group g and
 * output column n of the scaled layer W' = fl32(s W) (the layer once the scales are
 * folded in, AWQ-P1 §6; `scales` [K] fp32, typically awq_search's out_scales):
 *   c_i = fl32(absmax_g,n * fl32(1 - i/20)),  i = 0 .. n_shrink-1  (10 in the page: 1 .. 0.55)
 *   delta_i = Q(clamp(W'_g[:, n], -c_i, c_i)) - W'_g[:, n]   (Q = `quantizer`, AWQ_QUANT_*)
 *   e_i = mean over sampled tokens t of (sum_{k in g} X'[t,k] delta_i[k])^2,  X' = fl32(X / s)
 *   i* = first argmin of e_i (fp64); the output is the clipped group's artifact.
 * Sampled tokens: rows 0, d, 2d, ... of X with d = max(1, M / max_tokens), at most
 * max_tokens of them (awq_clip_token_count). The products run in fp64 as
 * delta^T (X'_g^T X'_g) delta / T.
 * Outputs (device memory):
 *   out_max_val [K/group][N] fp32   c_i* (the clamp applied before quantizing)
 *   out_best    [K/group][N] int32  i* (may be NULL)
 *   out_errors  [n_shrink][K/group][N] fp64  e_i (may be NULL)
 *   out_codes, out_steps, out_zeros: the artifact of Q(clamp(W', c_i*)), same layout as
 *   awq_search (dequantized W ~= step * (q - zero) / s).
 * Preconditions as awq_search (group 32/64/128, K % group == 0, N % 8 == 0; X and W
 * 16-byte aligned); 1 <= n_shrink <= 20; max_tokens >= 1; scales positive and finite
 * (AWQ_ERR_INVALID_ARG otherwise). Work space: (K/group) * group^2 * 8 bytes from the
 * library's pool. Synchronizes `stream`. Skipping layers (the page leaves query/key
 * projections unclipped) is the caller's decision. */
int awq_clip_search(const void* X, const void* W, int in_dtype, const float* scales,
                    int64_t M, int64_t K, int64_t N, int group, int n_shrink,
                    int64_t max_tokens, int quantizer, float* out_max_val, int32_t* out_best,
                    double* out_errors, int32_t* out_codes, void* out_steps,
                    void* out_zeros, awq_stream_t stream);
/* Number of tokens the clipping search samples from M rows (0 on bad arguments). */
int64_t awq_clip_token_count(int64_t M, int64_t max_tokens);
/* With profiling on (awq_profile_enable), device times (ms) of the last clipping
 * search's two kernels: [0] the Gram matrices, [1] the search. Returns 2. */
int awq_clip_profile_last(float* ms, int n);

/* Measured throughput (TFLOP/s, 2 flops per multiply-add) of the fp64 tensor-core
 * MMA on the current device: a register-only loop of 8x8x4 fp64 MMAs, 4 CTAs of 8
 * warps per SM, timed with CUDA events on `stream`. The roofline denominator of the
 * clipping search's products. */
int awq_fp64_mma_peak(double* tflops, awq_stream_t stream);

/* ---- Module-level objective: an MLP block ------------------------------------------
 * [AWQ-P1] §4: a candidate may be scored on the output of the whole module. For a
 * Llama-shaped MLP block with input X (M x K), gate and up projections searched jointly
 * as W_gu = [W_gate | W_up] (K x 2F, one scale vector) and the down projection W_down
 * (F x K_out, kept as it is):
 *   Y_i = h_i W_down,b,  h_i = bf16(fl32(silu(G_i) * U_i)),  [G_i | U_i] = X_b W_hat_i,b
 *   L_i = ||Y_i - Y_ref||_F^2 / (M K_out),  Y_ref the block with bf16(W_gu)
 * silu(x) = x / (1 + exp(-x)) in fp32; the GEMMs take bf16 operands and accumulate in
 * fp32. Steps 1-4 and 6 as awq_search (statistic and scales from X; QDQ, argmin and the
 * artifact of W_gu: out_codes [K][2F/8], out_steps/out_zeros [K/group][2F]; out_best,
 * device, may be NULL: the chosen index).
 * Preconditions as awq_search with N = 2F, plus F and K_out multiples of 8; W_down has
 * the dtype of X and W_gu. When F % 128 == 0 the silu-mul runs in the first GEMM's
 * epilogue (gate and up columns interleaved by 128 in the candidate operand) and each
 * GEMM runs once for a batch of candidates; otherwise the first GEMM writes [G | U] in
 * fp32 and a separate kernel forms h, one candidate at a time. Both give the same bits;
 * AWQ_MLP_UNFUSED=1 in the environment selects the second form. Work space from the
 * library's pool: the candidates ((n_grid + 1) 2F K bf16), h for the reference and a
 * batch of candidates (up to 4 GiB; the unfused form: M 2F fp32 plus M F bf16), the
 * transposed down projection and the reference output. Synchronizes `stream`. */
int awq_search_mlp(const void* X, const void* W_gu, const void* W_down, int in_dtype,
                   int64_t M, int64_t K, int64_t F, int64_t K_out, int group, int n_grid,
                   float* out_scales, int32_t* out_codes, void* out_steps, void* out_zeros,
                   float* out_losses, int32_t* out_best, awq_stream_t stream);

/* ---- Module-level objective: an attention block ---------------------------------------
 * [AWQ-P1] §4: the inspected module may be an attention block holding several
 * projections. The query, key and value projections read the same input X (M x K) and
 * are searched jointly with one scale vector, W_qkv = [W_q | W_k | W_v] (K x 3D, row-major,
 * D = n_heads * 128); each candidate is scored on the causal multi-head attention output
 * of the calibration sequences:
 *   [Q | K | V]_i = bf16(X_b W_hat_i,b)  (fp32 accumulation, then bf16);
 *   per sequence (seq_len consecutive rows of X) and head h (columns 128 h .. 128 h + 127
 *   of each of Q, K, V), for query t and keys u <= t:
 *     s_tu = q_t . k_u;  m_t = max_u s_tu;  e_tu = exp((s_tu - m_t) / sqrt(128));
 *     o_t = (sum_u bf16(e_tu) v_u) / (sum_u e_tu)       (fp32; no position encoding,
 *                                                        no output projection)
 *   L_i = ||O_i - O_ref||_F^2 / (M D),  O_ref the module with bf16(W_qkv).
 * Steps 1-4 and 6 as awq_search (statistic and scales from X; QDQ, first argmin and the
 * artifact of W_qkv: out_codes [K][3D/8], out_steps / out_zeros [K/group][3D]; out_losses
 * [n_grid] and out_best (one int32, the chosen index) device, may be NULL).
 * Preconditions as awq_search with N = 3D, plus n_heads >= 1, D = n_heads * 128, seq_len
 * in {128, 256, 384, 512} dividing M. The Q|K and V^T products run on the tensor cores for
 * all candidates at once; the attention kernel forms each unit's weights from the exact
 * row maximum (the scores of up to 512 keys are held in tensor memory) and reduces the
 * squared error in its epilogue, so no candidate's output reaches device memory. Work
 * space from the library's pool: (n_grid + 1) (3 D K + 3 D M) bf16 values, M D fp32 of
 * reference output and n_grid (M / 128) n_heads fp64 partials. Synchronizes `stream`. */
int awq_search_attn(const void* X, const void* W_qkv, int in_dtype, int64_t M, int64_t K,
                    int64_t D, int n_heads, int64_t seq_len, int group, int n_grid,
                    float* out_scales, int32_t* out_codes, void* out_steps, void* out_zeros,
                    float* out_losses, int32_t* out_best, awq_stream_t stream);
/* With profiling on (awq_profile_enable), device times (ms) of the last attention-block
 * search's phases: [0] statistic, scales and QDQ, [1] the Q|K products, [2] the V^T
 * products, [3] the reference attention, [4] the candidates' attention with the fused
 * loss, [5] the loss reduction and the artifact. Returns 6. */
int awq_attn_profile_last(float* ms, int n);

/* ---- W4A16 consumer of the artifact ---------------------------------------------
 * [AWQ-P1] §7: the artifact feeds a W4A16 kernel, checked by decoding it and comparing
 * the kernel's output with a reference; §8: 4-bit weights, 16-bit activations; §6: the
 * scales are folded into the operation that produces the activations.
 *   Y[m][n] = sum_k A[m][k] * w16[k][n],  w16[k][n] = fp16((q[k][n] - z[g][n]) * step[g][n])
 * A [M][K] fp16 activations already divided by the scales (A = fp16(X / s)); codes
 * [K][N/8] int32, steps and zeros [K/group][N] fp16 (the artifact of awq_search or
 * awq_clip_search); Y [M][N] fp32. Every product is exact in fp32 and the sums are fp32.
 * M <= 16 runs a fused dequantize + GEMV (bound by the 4.25-bit weight stream) and is
 * asynchronous: the call returns once the work is enqueued on `stream` (launch errors
 * are reported; Y is ready when the stream reaches that point). Larger M dequantizes
 * to an N x K fp16 work space (N K 2 bytes from the library's pool), runs the
 * tensor-core GEMM and synchronizes `stream` (its waits are bounded and reported as
 * AWQ_ERR_TIMEOUT). Same preconditions as awq_search on K, N and group; all pointers
 * device memory, 16-byte aligned. NaN or Inf in A propagates to Y. */
int awq_w4a16_matmul(const void* A, const int32_t* codes, const void* steps,
                     const void* zeros, int64_t M, int64_t K, int64_t N, int group,
                     float* Y, awq_stream_t stream);
/* With profiling on (awq_profile_enable): device time (ms) of the last call's kernels,
 * waiting for them if needed; -1 when the last call was not profiled. */
float awq_w4a16_profile_last(void);
/* Decode on repacked codes. awq_w4a16_repack rewrites the artifact's codes (K x N/8
 * int32; K % 32 == 0, N % 64 == 0) once, e.g. at load time, into the order the decode
 * kernel reads them: for every 16 rows, 64 columns and MMA lane, 16 contiguous bytes in
 * the A-fragment order of 16 x 8 x 16 MMAs whose A operand is the weights (16 columns by
 * 16 rows), nibbles arranged so that one mask (plus one shift per two pairs) gives an
 * fp16 pair. Same size as the codes; synchronizes `stream`. A layout written by an older
 * build is not compatible: repack again. awq_w4a16_matmul_packed is awq_w4a16_matmul for
 * M <= 16 on that layout (same result definition, steps and zeros unchanged; fixed-order,
 * deterministic sums), asynchronous on `stream`. */
int awq_w4a16_repack(const int32_t* codes, int64_t K, int64_t N, int32_t* out_packed,
                     awq_stream_t stream);
int awq_w4a16_matmul_packed(const void* A, const int32_t* packed, const void* steps,
                            const void* zeros, int64_t M, int64_t K, int64_t N, int group,
                            float* Y, awq_stream_t stream);
/* The dequantized operand alone: out_wt [N][K] fp16 (K contiguous) = w16 transposed. */
int awq_w4a16_dequant(const int32_t* codes, const void* steps, const void* zeros,
                      int64_t K, int64_t N, int group, void* out_wt, awq_stream_t stream);

int awq_version(void);

/* The loss-GEMM kernel a search of this size runs: 1 = the one-SM kernel (the default
 * for every size), 2 = the two-SM (cta_group::2) kernel when AWQ_GEMM_VARIANT=2 is set in
 * the environment. */
int awq_loss_gemm_variant(int64_t M, int64_t K, int64_t N, int n_grid);

/* Whether a search of this form makes its candidate operands with the loss GEMM's own
 * QDQ warps (1) or with a QDQ kernel launched before it (0): 1 for bf16 inputs with
 * group 128 on the one-SM GEMM kernel below 100 TFLOP of candidate GEMM work
 * (2 M K N n_grid); AWQ_QDQ=standalone or =warps in the environment selects a form at
 * every size. Eight more warps per GEMM CTA then quantize W while the tensor cores run;
 * a load of a column tile of a candidate operand waits (bounded) for that tile. Both
 * forms give bit-identical results. */
int awq_qdq_in_loss_gemm(int in_dtype, int64_t M, int64_t K, int64_t N, int group, int n_grid);

/* How many loss-GEMM launches a search of this form runs on the current device: 2 when
 * the QDQ warps make the operands (they claim candidate pieces during the reference
 * output's launch and make the rest during the candidates'), when the reference output Y (M x N fp32) is
 * larger than the device's L2 cache, or with the two-SM kernel: the reference output in
 * its own launch, then a launch that scores every candidate of a column tile before the
 * next column tile, so each tile of Y is read from DRAM once; 1 otherwise (one launch
 * computes the reference tiles and then the candidates, each candidate tile waiting for
 * its reference tile). Without the QDQ warps, AWQ_REFERENCE_LAUNCH=own or =fused in the
 * environment selects a form at every size. All forms give bit-identical results.
 * Returns the count, or minus an AWQ_ERR_* status when the device cannot be queried. */
int awq_loss_gemm_launches(int in_dtype, int64_t M, int64_t K, int64_t N, int group, int n_grid);

/* ---- Searching without allocating -------------------------------------------
 * No counterpart in the paper or the pages: this is a deployment variant of
 * awq_search_ex for callers that cannot call cudaMalloc — e.g. a plugin whose host
 * framework owns all device memory, a process whose memory budget was fixed at
 * start-up, or a loop that must not risk an allocation's synchronisation or
 * failure. Same arguments as awq_search_ex without the tile partials; it runs the
 * same search (argument checks, kernels, launch sequence and work-space layout), so
 * its results are bit-identical to awq_search_ex's. The work space comes from one
 * array of AWQ_NOALLOC_SCRATCH_BYTES compiled into the library instead of the
 * library's pool; nothing is allocated or freed, and the call synchronizes `stream`
 * (its status word is read back into pageable host memory).
 * The array belongs to the library's code module: CUDA materialises it on a GPU at
 * the first call made there, which returns AWQ_ERR_CUDA if that GPU has no room left
 * for it; from then on that GPU holds it until the process exits.
 * Layers whose work space (awq_workspace_bytes, the same layout) exceeds the array
 * are rejected with AWQ_ERR_SHAPE and a message giving both sizes — a
 * 1024 x 1024 x 1024 bf16 layer with 20 candidates fits, the Llama-shaped layers do
 * not; an fp32 layer also needs M*K*2 bytes for its bf16 copy of X.
 * The first call on each device also looks up the array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call before
 * any stream capture. All calls share the array and it keeps the last call's
 * contents (the status word and the per-tile flags are cleared at the start of each
 * call, everything else is overwritten before it is read): calls that overlap on the
 * GPU — on different streams or from different host threads on one device — race on
 * it and must be serialised by the caller. */
#define AWQ_NOALLOC_SCRATCH_BYTES (64ll << 20)
int awq_search_noalloc(const void* X, const void* W, int in_dtype, int64_t M, int64_t K,
                       int64_t N, int group, int n_grid, float* out_scales,
                       int32_t* out_codes, void* out_steps, void* out_zeros,
                       float* out_losses, int32_t* out_best, awq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* AWQ_SEARCH_H_ */
