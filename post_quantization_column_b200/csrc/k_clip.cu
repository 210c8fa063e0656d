// k_clip.cu — the clipping search that follows the channel scaling ("AWQ：为什么 4-bit
// 权重量化要先观察 Activation" §5).
//
// For every input group g and output column n of the scaled layer (W' = fl32(s W),
// X' = fl32(X / s), the layer once the scales are folded in, same page §6), the search
// tries the thresholds c_i = fl32(absmax * fl32(1 - i/20)), i = 0 .. n_shrink-1, clamps
// the group to [-c_i, c_i], quantizes it with the asymmetric 4-bit quantizer (§7; or the
// symmetric teaching quantizer of §2), and
// scores the candidate by the mean squared error of the group's partial dot product
// over the sampled tokens:
//     e_i = (1/T) sum_t ( sum_{k in g} X'[t,k] delta_i[k] )^2 = delta_i^T H_g delta_i / T,
//     delta_i = Q(clamp(W'_g[:, n], c_i)) - W'_g[:, n],  H_g = X'_g^T X'_g.
// The first minimum wins; its threshold, codes, steps and zeros are written out.
//
// gram_kernel: H_g for every group in fp64 on the tensor cores (the products of two
// fp32 values are exact in fp64; only the token sums round). Small: T * G^2 per group.
//
// clip_kernel: one CTA per (group, 64 output columns). It stages the lower block
// triangle of H_g in shared memory once, keeps its share of W' in registers, and for
// each threshold builds the G x 64 matrix of deltas in shared memory (double-buffered,
// so building one threshold overlaps the products of the previous one), then evaluates
// every column's delta^T H_g delta from one block triangle of H_g (32-row blocks,
// G (G + 32) / 2 products per (threshold, column)) with fp64 tensor-core MMAs, 16 warps
// sharing the work evenly. The kernel is bound by the fp64 tensor pipe, not by memory
// (H_g comes from L2, W is read once).
#include "awq_device.cuh"
#include "awq_kernels.h"

namespace awq {
namespace {

constexpr int kShrinkGrid = 20;    // factor_i = 1 - i / 20
constexpr int kClipCols = 64;      // output columns per CTA
constexpr int kClipThreads = 512;  // 16 warps
constexpr int kGramThreads = 256;  // 8 warps
constexpr int kGramChunk = 32;     // tokens staged per pass

// ---- fp64 tensor-core helpers ------------------------------------------------------------
// D (8x8) += A (8x4, row-major) * B (4x8) in fp64 on the tensor cores. Lane (g, t) =
// (lane / 4, lane % 4) holds A[g][t], B[t][g] and D[g][2t], D[g][2t + 1].
__device__ __forceinline__ void mma_f64(double (&d)[2], double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
               : "+d"(d[0]), "+d"(d[1])
               : "d"(a), "d"(b));
}

// ---- Gram matrices -------------------------------------------------------------------
// CTA (g, tile): a TB x TB tile of H_g, TB = min(G, 64), rows r0.., columns c0... The
// sampled tokens are staged 32 at a time as fp64 X' values (rows part and columns part,
// row pitch TB + 4 so the fragment loads hit 32 banks); each of the 8 warps owns a
// (TB/2) x (TB/4) sub-tile and accumulates it with fp64 MMAs over 4 tokens per step.
template <typename T, int G>
__global__ void __launch_bounds__(kGramThreads) gram_kernel(const T* __restrict__ X, int64_t K, int64_t stride,
                                                            int tokens, const float* __restrict__ s,
                                                            double* __restrict__ H, int* err) {
  constexpr int TB = G < 64 ? G : 64;
  constexpr int TILES = G / TB;
  constexpr int PX = TB + 4;
  constexpr int WR = TB / 2, WC = TB / 4;  // warp sub-tile: 2 x 4 warps
  constexpr int MI = WR / 8, MJ = WC / 8;  // 8x8 MMA tiles per warp (4x2 for TB 64, 2x1 for TB 32)
  __shared__ __align__(16) double xa[kGramChunk][PX];
  __shared__ __align__(16) double xb[kGramChunk][PX];

  const int64_t g = blockIdx.x;
  const int r0 = (blockIdx.y / TILES) * TB, c0 = (blockIdx.y % TILES) * TB;
  const int64_t col0 = g * G;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int gq = lane >> 2, tq = lane & 3;
  const int wr = warp / 4, wc = warp % 4;

  double acc[MI][MJ][2];
#pragma unroll
  for (int a = 0; a < MI; ++a)
#pragma unroll
    for (int b = 0; b < MJ; ++b) acc[a][b][0] = acc[a][b][1] = 0.0;

  // the tile's scales, once
  __shared__ float ss[2][TB];
  bool bad_x = false, bad_s = false;
  for (int i = threadIdx.x; i < 2 * TB; i += kGramThreads) {
    const float sc = s[col0 + (i < TB ? r0 + i : c0 + i - TB)];
    bad_s |= !(sc > 0.0f) || !isfinite(sc);
    ss[i / TB][i % TB] = sc;
  }

  // 16-byte vectors of the sampled rows: NV per thread per chunk, prefetched into
  // registers one chunk ahead of the products
  constexpr int VEC = 16 / sizeof(T);
  constexpr int VPR = TB / VEC;  // vectors per row of one half
  constexpr int NV = 2 * kGramChunk * VPR / kGramThreads;
  static_assert(NV * kGramThreads == 2 * kGramChunk * VPR, "staging vectors must split evenly");
  uint4 pre[NV];
  auto fetch = [&](int t0) {
#pragma unroll
    for (int q = 0; q < NV; ++q) {
      const int idx = threadIdx.x + q * kGramThreads;
      const int half = idx / (kGramChunk * VPR), rem = idx % (kGramChunk * VPR);
      const int t = rem / VPR, v = rem % VPR;
      pre[q] = make_uint4(0, 0, 0, 0);  // tokens past the end contribute zero
      if (t0 + t < tokens)
        pre[q] = __ldg(reinterpret_cast<const uint4*>(X + static_cast<int64_t>(t0 + t) * stride * K + col0 +
                                                      (half ? c0 : r0) + v * VEC));
    }
  };
  fetch(0);
  __syncthreads();  // ss is visible
  for (int t0 = 0; t0 < tokens; t0 += kGramChunk) {
#pragma unroll
    for (int q = 0; q < NV; ++q) {
      const int idx = threadIdx.x + q * kGramThreads;
      const int half = idx / (kGramChunk * VPR), rem = idx % (kGramChunk * VPR);
      const int t = rem / VPR, v = rem % VPR;
      const T* e = reinterpret_cast<const T*>(&pre[q]);
      double* dst = (half ? xb[t] : xa[t]) + v * VEC;
#pragma unroll
      for (int i = 0; i < VEC; ++i) {
        const float xs = __fdiv_rn(to_f32<T>(e[i]), ss[half][v * VEC + i]);  // X' = fl32(X / s)
        bad_x |= !isfinite(xs);
        dst[i] = static_cast<double>(xs);
      }
    }
    __syncthreads();
    if (t0 + kGramChunk < tokens) fetch(t0 + kGramChunk);
#pragma unroll 2
    for (int k4 = 0; k4 < kGramChunk; k4 += 4) {
      double av[MI], bv[MJ];
#pragma unroll
      for (int a = 0; a < MI; ++a) av[a] = xa[k4 + tq][wr * WR + 8 * a + gq];  // A[k][t] = X'[t][k]
#pragma unroll
      for (int b = 0; b < MJ; ++b) bv[b] = xb[k4 + tq][wc * WC + 8 * b + gq];  // B[t][l] = X'[t][l]
#pragma unroll
      for (int a = 0; a < MI; ++a)
#pragma unroll
        for (int b = 0; b < MJ; ++b) mma_f64(acc[a][b], av[a], bv[b]);
    }
    __syncthreads();
  }
  if (bad_x) atomicOr(err, kErrNonfiniteX);
  if (bad_s) atomicOr(err, kErrBadScale);
  double* Hg = H + g * G * G;
#pragma unroll
  for (int a = 0; a < MI; ++a)
#pragma unroll
    for (int b = 0; b < MJ; ++b) {
      const int row = r0 + wr * WR + 8 * a + gq, col = c0 + wc * WC + 8 * b + 2 * tq;
      *reinterpret_cast<double2*>(Hg + row * G + col) = make_double2(acc[a][b][0], acc[a][b][1]);
    }
}

// ---- clipping search -------------------------------------------------------------------
// Shared-memory layout (G = 128: 80 KB of H, 2 x 64 KB of deltas):
//  * H_g, the lower block triangle only: the 32 x 32 blocks (c, b), c >= b, of the
//    stored H[l][k], block (c, b) at index c (c + 1) / 2 + b, row-major inside;
//  * two buffers of the G x 64 deltas (one threshold is built while the previous one
//    is multiplied).
// Both swizzle the column index with the row: column x of row y sits at x ^ f(y & 3),
// f(0..3) = 0, 8, 4, 12, so the MMA fragment loads (rows l = 4 s + t for lane t), the
// 16-byte loads of the fold (rows 8 i + g) and the delta stores touch distinct banks
// without padding.
template <int G>
struct ClipTile {
  static constexpr int EPT = G * kClipCols / kClipThreads;   // W' elements per thread (G / 8)
  static constexpr int kRowStep = kClipThreads / kClipCols;  // 8
  static constexpr int kSliceCols = 16;                      // columns of one warp's tile
  static constexpr int NB = G / 32;                          // 32-row blocks
  static constexpr int kBlocksH = NB * (NB + 1) / 2;         // stored blocks of H
  static constexpr int kSteps = 8 * kBlocksH;                // k-steps of 4 per column slice
  static constexpr int kWarps = kClipThreads / 32;
  static constexpr int kWarpsPerSlice = kWarps / (kClipCols / kSliceCols);
  static constexpr int kStepsPerWarp = kSteps / kWarpsPerSlice;
  static_assert(kSteps % kWarpsPerSlice == 0, "k-steps must split evenly over the warps of a slice");
  static_assert(kStepsPerWarp % 2 == 0, "runs start and end on even steps");
  static_assert(kSliceCols == 16, "the product is written for two 8-column MMA tiles per warp");
  static constexpr size_t kSmemH = sizeof(double) * kBlocksH * 32 * 32;
  static constexpr size_t kSmemD = sizeof(double) * G * kClipCols;  // one buffer
  static constexpr size_t kSmemRed = sizeof(double) * 2 * kWarps * kSliceCols;
  static constexpr size_t kSmem = kSmemH + 2 * kSmemD + kSmemRed;
};

__device__ __forceinline__ int swz(int row, int col) { return col ^ (((row & 1) << 3) | ((row & 2) << 1)); }

// H[l][k] (l in block c >= k's block b) in the triangular layout
__device__ __forceinline__ int h_index(int l, int k) {
  const int c = l >> 5, b = k >> 5, lr = l & 31, kr = k & 31;
  return ((c * (c + 1) / 2 + b) * 32 + lr) * 32 + swz(lr, kr);
}

__device__ __forceinline__ int d_index(int row, int col) { return row * kClipCols + swz(row, col); }

__device__ __forceinline__ float shrink_factor(int i) {
  return __double2float_rn(__dsub_rn(1.0, __ddiv_rn(static_cast<double>(i), static_cast<double>(kShrinkGrid))));
}

__device__ __forceinline__ float clamp_to(float w, float c) { return fminf(fmaxf(w, -c), c); }

__device__ __forceinline__ void cp_async_16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

constexpr float kRoundMagic = 12582912.0f;            // 1.5 * 2^23: (x + m) - m = rint(x) for |x| < 2^22
constexpr float kNearHalf = 0.5f - 1.0f / 32768.0f;   // |t - rint(t)| at or above this: exact division
constexpr float kTinyStep = 7.888609052210118e-31f;   // 2^-100
constexpr float kHugeRecip = 1.2676506002282294e30f;  // 2^100

template <typename T, int G>
__global__ void __launch_bounds__(kClipThreads, 1)
    clip_kernel(const T* __restrict__ W, int64_t N, const float* __restrict__ s, const double* __restrict__ H,
                int n_shrink, int tokens, float* __restrict__ max_val, int32_t* __restrict__ best_out,
                double* __restrict__ errors, int32_t* __restrict__ codes, __half* __restrict__ steps,
                __half* __restrict__ zeros, int* err, int quantizer) {
  using CT = ClipTile<G>;
  constexpr int MJ = CT::kSliceCols / 8;  // 8-column MMA tiles per warp
  extern __shared__ __align__(16) uint8_t smem[];
  double* sH = reinterpret_cast<double*>(smem);                                  // triangular H_g
  double* sD = reinterpret_cast<double*>(smem + CT::kSmemH);                     // [2][G][64] deltas
  double* sRed = reinterpret_cast<double*>(smem + CT::kSmemH + 2 * CT::kSmemD);  // [2][warp][kSliceCols]
  __shared__ float sAbs[CT::kRowStep][kClipCols], sMin[CT::kRowStep][kClipCols], sMax[CT::kRowStep][kClipCols];
  __shared__ int sBest[kClipCols];
  __shared__ float sF[kShrinkGrid];  // the shrink factors

  const int64_t g = blockIdx.y;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kClipCols;
  const int64_t G_total = gridDim.y;

  // the lower block triangle of H_g -> shared memory, asynchronously (it overlaps the
  // load of W below); 16-byte pieces: block q, row lr, column pair kp
  {
    const double* src = H + g * G * G;
    for (int i = threadIdx.x; i < CT::kBlocksH * 32 * 16; i += kClipThreads) {
      const int q = i / 512, rem = i % 512, lr = rem / 16, kp = rem % 16;
      int c = 0;
      while ((c + 1) * (c + 2) / 2 <= q) ++c;
      const int b = q - c * (c + 1) / 2;
      const int l = 32 * c + lr, k = 32 * b + 2 * kp;
      cp_async_16(sH + h_index(l, k), src + l * G + k);
    }
  }

  // this thread's share of W': column n, rows k = r + kRowStep j
  const int n = threadIdx.x % kClipCols, r = threadIdx.x / kClipCols;
  const bool col_ok = n0 + n < N;
  float wp[CT::EPT];
  float amax = 0.0f, mn = INFINITY, mx = -INFINITY;
  bool bad = false;
#pragma unroll
  for (int j = 0; j < CT::EPT; ++j) {
    const int64_t k = g * G + r + CT::kRowStep * j;
    float w = 0.0f;
    if (col_ok) {
      w = to_f32<T>(W[k * N + n0 + n]);
      bad |= !isfinite(w);
    }
    wp[j] = __fmul_rn(s[k], w);  // W' = fl32(s * W)
    amax = fmaxf(amax, fabsf(wp[j]));
    mn = fminf(mn, wp[j]);
    mx = fmaxf(mx, wp[j]);
  }
  if (bad) atomicOr(err, kErrNonfiniteW);
  if (threadIdx.x < n_shrink) sF[threadIdx.x] = shrink_factor(threadIdx.x);
  sAbs[r][n] = amax;
  sMin[r][n] = mn;
  sMax[r][n] = mx;
  cp_async_wait_all();
  __syncthreads();
  amax = sAbs[0][n];
  mn = sMin[0][n];
  mx = sMax[0][n];
#pragma unroll
  for (int q = 1; q < CT::kRowStep; ++q) {
    amax = fmaxf(amax, sAbs[q][n]);
    mn = fminf(mn, sMin[q][n]);
    mx = fmaxf(mx, sMax[q][n]);
  }

  // Product. H_g is symmetric, so with 32-row blocks b, c:
  //   delta^T H delta = sum_b delta_b^T (2 sum_{c > b} H_bc delta_c + H_bb delta_b),
  // the upper block triangle only, read as H[l][k] from the stored lower one. For one
  // 16-column slice these items, taken b-major (the weight-2 blocks c > b first, then
  // the diagonal one) in k-steps of 4 values of l, form kSteps steps; each of the
  // slice's warps takes an equal contiguous run of them and computes a 32 x 16 tile of
  // Q_b = sum_c H_bc Delta_c with fp64 tensor-core MMAs, doubling Q_b when it reaches
  // the diagonal block and folding Delta_b .* Q_b into its column sums when its row
  // block changes.
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int gq = lane >> 2, tq = lane & 3;
  const int slice = warp / CT::kWarpsPerSlice;
  const int colw = slice * CT::kSliceCols;  // first column of the slice
  int b_start = 0, ks_start = (warp % CT::kWarpsPerSlice) * CT::kStepsPerWarp;
  while (ks_start >= 8 * (CT::NB - b_start)) {
    ks_start -= 8 * (CT::NB - b_start);
    ++b_start;
  }
  const int j_start = ks_start / 8;
  ks_start %= 8;

  // lanes 0..3 of every warp keep the running first minimum of column 4 warp + lane
  const int my_col = warp * 4 + lane;
  double best_e = 0.0;
  int best_i = 0;
  const double tokens_d = static_cast<double>(tokens);

  // One barrier per threshold: in step it, the deltas of threshold it are built into
  // buffer it % 2 while the products of threshold it - 1 run on the other buffer and the
  // column sums of threshold it - 2 are reduced. Each warp interleaves the two: its share
  // of the build is spread over the units of its product run, so the ALU work of the
  // build issues while the warp's own tensor-core MMAs are in flight.
  struct BuildParams {
    double* dbuf;
    float c, recip, lo, hi;
    QdqParams p;
    bool col_exact;
  };
  auto build_params = [&](int it) {
    // clamp -> QDQ -> delta. Clamping is monotone, so the clamped group's min and max are
    // the clamped min and max. Codes use a correctly rounded reciprocal of the step; a
    // quotient within 2^-15 of a half-integer takes the exact division.
    BuildParams bp;
    bp.dbuf = sD + (it & 1) * G * kClipCols;
    bp.c = __fmul_rn(amax, sF[it]);
    bp.p = qdq_params_q(clamp_to(mn, bp.c), clamp_to(mx, bp.c), quantizer);
    bp.recip = __frcp_rn(bp.p.step);
    bp.col_exact = !(bp.p.step >= kTinyStep && bp.recip <= kHugeRecip);
    bp.lo = -bp.p.zero;
    bp.hi = bp.p.qmax - bp.p.zero;
    return bp;
  };
  auto build_one = [&](const BuildParams& bp, int j) {  // element j of this thread's share
    const float wc = clamp_to(wp[j], bp.c);
    const float tv = fminf(fmaxf(__fmul_rn(wc, bp.recip), bp.lo), bp.hi);
    float qz = __fsub_rn(__fadd_rn(tv, kRoundMagic), kRoundMagic);  // q - z
    if (bp.col_exact || fabsf(__fsub_rn(tv, qz)) >= kNearHalf) qz = __fsub_rn(qdq_code(wc, bp.p), bp.p.zero);
    const float rec = __fmul_rn(qz, bp.p.step);
    bp.dbuf[d_index(r + CT::kRowStep * j, n)] = __dsub_rn(static_cast<double>(rec), static_cast<double>(wp[j]));
  };
  auto build = [&](int it) {  // the whole share at once (the first threshold: no products to hide it behind)
    const BuildParams bp = build_params(it);
#pragma unroll
    for (int j = 0; j < CT::EPT; ++j) build_one(bp, j);
  };
  // products of threshold it - 1; with_build: threshold it's deltas built alongside
  auto product = [&](int it, bool with_build) {
    constexpr int kUnits = CT::kStepsPerWarp / 2;  // two k-steps per unit
    const double* dbuf = sD + ((it - 1) & 1) * G * kClipCols;
    BuildParams bp;
    if (with_build) bp = build_params(it);
    double ep[MJ][2];  // column sums of this lane: columns colw + 8 jt + 2 tq + {0, 1}
    double acc[4][MJ][2];
#pragma unroll
    for (int jt = 0; jt < MJ; ++jt) {
      ep[jt][0] = ep[jt][1] = 0.0;
#pragma unroll
      for (int i4 = 0; i4 < 4; ++i4) acc[i4][jt][0] = acc[i4][jt][1] = 0.0;
    }
    auto fold = [&](int blk) {  // ep += Delta_blk .* Q_blk, then clear Q
#pragma unroll
      for (int i4 = 0; i4 < 4; ++i4) {
        const int row = 32 * blk + 8 * i4 + gq;
#pragma unroll
        for (int jt = 0; jt < MJ; ++jt) {
          const double2 dv = *reinterpret_cast<const double2*>(dbuf + d_index(row, colw + 8 * jt + 2 * tq));
          ep[jt][0] = __fma_rn(dv.x, acc[i4][jt][0], ep[jt][0]);
          ep[jt][1] = __fma_rn(dv.y, acc[i4][jt][1], ep[jt][1]);
          acc[i4][jt][0] = acc[i4][jt][1] = 0.0;
        }
      }
    };
    auto double_q = [&]() {  // exact: the weight-2 sums
#pragma unroll
      for (int i4 = 0; i4 < 4; ++i4)
#pragma unroll
        for (int jt = 0; jt < MJ; ++jt) {
          acc[i4][jt][0] = __dadd_rn(acc[i4][jt][0], acc[i4][jt][0]);
          acc[i4][jt][1] = __dadd_rn(acc[i4][jt][1], acc[i4][jt][1]);
        }
    };
    // The run, as units of two k-steps (runs start and end on even steps, so a unit never
    // crosses a 32-row block): row block b, column block cb, steps ks, ks + 1. Every load
    // is a fixed offset from one of four per-lane pointers: with x = tq & 1 the swizzle
    // maps the fragment columns 8 m + gq of row 4 s + tq to 8 (m ^ x) + (gq ^ 4 (tq >> 1)),
    // so pointers pa0 / pa1 (pd0 / pd1) serve the even / odd MMA rows (columns).
    const int x = tq & 1;
    const int lane_off = gq ^ (4 * (tq >> 1));
    int b = b_start, j = j_start, ks = ks_start;
    bool on_diag = false;
#pragma unroll
    for (int unit = 0; unit < kUnits; ++unit) {
      const int n_off = CT::NB - 1 - b;  // weight-2 blocks right of the diagonal
      const int cb = j < n_off ? b + 1 + j : b;
      on_diag = cb == b;
      if (on_diag && ks == 0) double_q();  // entering the diagonal block
      const double* hrow = sH + ((cb * (cb + 1) / 2 + b) * 32 + 4 * ks + tq) * 32 + lane_off;
      const double* pa0 = hrow + 8 * x;
      const double* pa1 = hrow + 8 * (1 - x);
      const double* drow = dbuf + (32 * cb + 4 * ks + tq) * kClipCols + colw + lane_off;
      const double* pd0 = drow + 8 * x;
      const double* pd1 = drow + 8 * (1 - x);
#pragma unroll
      for (int v = 0; v < 2; ++v) {
        const int oa = v * 128, od = v * 4 * kClipCols;
        const double a0 = pa0[oa], a1 = pa1[oa], a2 = pa0[oa + 16], a3 = pa1[oa + 16];
        const double b0 = pd0[od], b1 = pd1[od];
        mma_f64(acc[0][0], a0, b0);
        mma_f64(acc[0][1], a0, b1);
        mma_f64(acc[1][0], a1, b0);
        mma_f64(acc[1][1], a1, b1);
        mma_f64(acc[2][0], a2, b0);
        mma_f64(acc[2][1], a2, b1);
        mma_f64(acc[3][0], a3, b0);
        mma_f64(acc[3][1], a3, b1);
      }
      if (with_build) {  // this unit's slice of the next threshold's deltas
#pragma unroll
        for (int e = unit * CT::EPT / kUnits; e < (unit + 1) * CT::EPT / kUnits; ++e) build_one(bp, e);
      }
      ks += 2;
      if (ks == 8) {
        ks = 0;
        if (++j == CT::NB - b) {
          fold(b);
          ++b;
          j = 0;
        }
      }
    }
    if (b < CT::NB) {  // the run ended inside row block b (a no-op after a clean block end)
      if (!on_diag) double_q();  // it never reached the diagonal block
      fold(b);
    }
    // combine the 8 lanes (gq) that hold partial sums of the same columns
#pragma unroll
    for (int jt = 0; jt < MJ; ++jt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        double v = ep[jt][h];
        v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, 4));
        v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, 8));
        v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, 16));
        ep[jt][h] = v;
      }
    if (gq == 0) {
      double* red = sRed + ((it - 1) & 1) * CT::kWarps * CT::kSliceCols + warp * CT::kSliceCols;
#pragma unroll
      for (int jt = 0; jt < MJ; ++jt) {
        red[8 * jt + 2 * tq] = ep[jt][0];
        red[8 * jt + 2 * tq + 1] = ep[jt][1];
      }
    }
  };
  for (int it = 0; it < n_shrink + 2; ++it) {
    if (it >= 1 && it <= n_shrink)
      product(it, it < n_shrink);
    else if (it < n_shrink)
      build(it);
    if (it >= 2 && lane < 4) {
      const int i = it - 2;
      const double* red = sRed + (i & 1) * CT::kWarps * CT::kSliceCols;
      const int w0 = (my_col / CT::kSliceCols) * CT::kWarpsPerSlice;
      double e = 0.0;
#pragma unroll
      for (int q = 0; q < CT::kWarpsPerSlice; ++q) e = __dadd_rn(e, red[(w0 + q) * CT::kSliceCols + my_col % CT::kSliceCols]);
      e = __ddiv_rn(e, tokens_d);  // the mean over the sampled tokens
      if (errors && n0 + my_col < N) errors[(static_cast<int64_t>(i) * G_total + g) * N + n0 + my_col] = e;
      if (i == 0 || e < best_e) {  // first minimum
        best_e = e;
        best_i = i;
      }
    }
    __syncthreads();
  }
  if (lane < 4) sBest[my_col] = best_i;
  __syncthreads();

  // artifact of the chosen threshold: codes through shared memory, packed eight per
  // int32 along N; steps and zeros as fp16
  const int bi = sBest[n];
  const float c = __fmul_rn(amax, sF[bi]);
  const QdqParams p = qdq_params_q(clamp_to(mn, c), clamp_to(mx, c), quantizer);
  uint8_t* sQ = reinterpret_cast<uint8_t*>(sD);  // [G][64] codes
#pragma unroll
  for (int j = 0; j < CT::EPT; ++j)
    sQ[(r + CT::kRowStep * j) * kClipCols + n] = static_cast<uint8_t>(qdq_code(clamp_to(wp[j], c), p));
  if (r == 0 && col_ok) {
    const int64_t at = g * N + n0 + n;
    max_val[at] = c;
    if (best_out) best_out[at] = bi;
    steps[at] = __float2half_rn(p.step);
    zeros[at] = __float2half_rn(p.zero);
  }
  __syncthreads();
  const int64_t words = N / 8;
  for (int idx = threadIdx.x; idx < G * (kClipCols / 8); idx += kClipThreads) {
    const int k = idx / (kClipCols / 8), w = idx % (kClipCols / 8);
    if (n0 + 8 * w >= N) continue;  // N % 8 == 0: a word lies wholly inside or outside
    uint32_t word = 0;
#pragma unroll
    for (int bb = 0; bb < 8; ++bb) word |= static_cast<uint32_t>(sQ[k * kClipCols + 8 * w + bb]) << (4 * bb);
    codes[(g * G + k) * words + n0 / 8 + w] = static_cast<int32_t>(word);
  }
}

template <typename T, int G>
cudaError_t launch_clip_t(const ClipArgs& a, cudaStream_t st, int* launches) {
  const int64_t groups = a.K / G;
  const int64_t stride = clip_token_stride(a.M, a.max_tokens);
  if (a.ev) cudaEventRecord(a.ev[0], st);
  {
    constexpr int TB = G < 64 ? G : 64;
    dim3 grid(static_cast<unsigned>(groups), (G / TB) * (G / TB));
    gram_kernel<T, G><<<grid, kGramThreads, 0, st>>>(static_cast<const T*>(a.X), a.K, stride, a.tokens, a.s, a.H,
                                                     a.err);
    *launches += 1;
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (a.ev) cudaEventRecord(a.ev[1], st);
  static unsigned long long done = 0;
  cudaError_t e = set_smem_limit_once(clip_kernel<T, G>, static_cast<int>(ClipTile<G>::kSmem), &done);
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(ceil_div(a.N, kClipCols)), static_cast<unsigned>(groups));
  clip_kernel<T, G><<<grid, kClipThreads, ClipTile<G>::kSmem, st>>>(
      static_cast<const T*>(a.W), a.N, a.s, a.H, a.n_shrink, a.tokens, a.max_val, a.best, a.errors, a.codes, a.steps,
      a.zeros, a.err, a.quantizer);
  *launches += 1;
  if (a.ev) cudaEventRecord(a.ev[2], st);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_clip_dtype(const ClipArgs& a, cudaStream_t st, int* launches) {
  switch (a.group) {
    case 32: return launch_clip_t<T, 32>(a, st, launches);
    case 64: return launch_clip_t<T, 64>(a, st, launches);
    default: return launch_clip_t<T, 128>(a, st, launches);
  }
}

// Throughput probe of the fp64 tensor-core MMA: register operands, 8 independent
// accumulators per warp, no memory traffic but one store per thread.
__global__ void __launch_bounds__(256) fp64_mma_peak_kernel(double* out, int iters) {
  const int lane = threadIdx.x & 31;
  double a[4], b[2], d[8][2];
#pragma unroll
  for (int i = 0; i < 4; ++i) a[i] = 1.0 + 1e-9 * (lane + i);
#pragma unroll
  for (int i = 0; i < 2; ++i) b[i] = 1.0 - 1e-9 * (lane + i);
#pragma unroll
  for (int i = 0; i < 8; ++i) d[i][0] = d[i][1] = 0.0;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < 8; ++i) mma_f64(d[i], a[i & 3], b[i >> 2]);
  }
  double s = 0.0;
#pragma unroll
  for (int i = 0; i < 8; ++i) s += d[i][0] + d[i][1];
  out[static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x] = s;
}

}  // namespace

int64_t clip_token_stride(int64_t M, int64_t max_tokens) { return M / max_tokens > 1 ? M / max_tokens : 1; }

int64_t clip_token_count(int64_t M, int64_t max_tokens) {
  const int64_t stride = clip_token_stride(M, max_tokens);
  const int64_t t = ceil_div(M, stride);
  return t < max_tokens ? t : max_tokens;
}

cudaError_t launch_clip(const ClipArgs& a, cudaStream_t s, int* launches) {
  return a.in_dtype == 0 ? launch_clip_dtype<__nv_bfloat16>(a, s, launches) : launch_clip_dtype<float>(a, s, launches);
}

}  // namespace awq

namespace awq {
// Blocks x 256 threads of the probe; `out` holds blocks * 256 doubles.
cudaError_t launch_fp64_mma_peak(double* out, int blocks, int iters, cudaStream_t s) {
  fp64_mma_peak_kernel<<<blocks, 256, 0, s>>>(out, iters);
  return cudaGetLastError();
}
}  // namespace awq
