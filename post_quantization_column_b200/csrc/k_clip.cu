// k_clip.cu — the clipping search that follows the channel scaling ("AWQ：为什么 4-bit
// 权重量化要先观察 Activation" §5).
//
// For every input group g and output column n of the scaled layer (W' = fl32(s W),
// X' = fl32(X / s), the layer once the scales are folded in, same page §6), the search
// tries the thresholds c_i = fl32(absmax * fl32(1 - i/20)), i = 0 .. n_shrink-1, clamps
// the group to [-c_i, c_i], quantizes it with the asymmetric 4-bit quantizer (§7), and
// scores the candidate by the mean squared error of the group's partial dot product
// over the sampled tokens:
//     e_i = (1/T) sum_t ( sum_{k in g} X'[t,k] delta_i[k] )^2 = delta_i^T H_g delta_i / T,
//     delta_i = Q(clamp(W'_g[:, n], c_i)) - W'_g[:, n],  H_g = X'_g^T X'_g.
// The first minimum wins; its threshold, codes, steps and zeros are written out.
//
// gram_kernel: H_g for every group, fp64 (products of two fp32 values are exact in
// fp64; the token sum runs in token order, so H is bit-symmetric). Small: T * G^2 per
// group.
//
// clip_kernel: one CTA per (group, 64 output columns). It stages H_g (G x G fp64) in
// shared memory once, keeps its share of W' in registers, and for each threshold builds
// the G x 64 matrix of deltas in shared memory, then forms Q = H_g Delta with a
// register-tiled fp64 product (each thread 8 rows x 4 columns for G = 128) and the
// column sums of Delta .* Q. The work is n_shrink * G^2 fp64 FMAs per (group, column):
// the kernel is bound by the fp64 pipe, not by memory (H_g comes from L2, W is read
// once).
#include "awq_device.cuh"
#include "awq_kernels.h"

namespace awq {
namespace {

constexpr int kShrinkGrid = 20;    // factor_i = 1 - i / 20
constexpr int kClipCols = 64;      // output columns per CTA
constexpr int kClipThreads = 256;  // 16 row-blocks x 16 column-lanes
constexpr int kGramThreads = 256;  // 16 x 16
constexpr int kGramChunk = 32;     // tokens staged per pass

// ---- Gram matrices -------------------------------------------------------------------
// CTA (g, tile): a TB x TB tile of H_g, TB = min(G, 64). Thread (ty, tx) owns rows
// r0 + ty + 16 a and columns c0 + tx + 16 b (a, b < TB / 16).
template <typename T, int G>
__global__ void __launch_bounds__(kGramThreads) gram_kernel(const T* __restrict__ X, int64_t K, int64_t stride,
                                                            int tokens, const float* __restrict__ s,
                                                            double* __restrict__ H, int* err) {
  constexpr int TB = G < 64 ? G : 64;
  constexpr int R = TB / 16;
  constexpr int TILES = G / TB;
  __shared__ double xa[kGramChunk][TB];
  __shared__ double xb[kGramChunk][TB];

  const int64_t g = blockIdx.x;
  const int r0 = (blockIdx.y / TILES) * TB, c0 = (blockIdx.y % TILES) * TB;
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  const int64_t col0 = g * G;

  double acc[R][R];
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int b = 0; b < R; ++b) acc[a][b] = 0.0;

  bool bad_x = false, bad_s = false;
  for (int t0 = 0; t0 < tokens; t0 += kGramChunk) {
    for (int idx = threadIdx.x; idx < 2 * kGramChunk * TB; idx += kGramThreads) {
      const int half = idx / (kGramChunk * TB);
      const int rem = idx % (kGramChunk * TB);
      const int t = rem / TB, c = rem % TB;
      const int64_t col = col0 + (half ? c0 : r0) + c;
      double v = 0.0;
      if (t0 + t < tokens) {
        const float x = to_f32<T>(X[static_cast<int64_t>(t0 + t) * stride * K + col]);
        const float sc = s[col];
        bad_s |= !(sc > 0.0f) || !isfinite(sc);
        const float xs = __fdiv_rn(x, sc);  // X' = fl32(X / s)
        bad_x |= !isfinite(xs);
        v = static_cast<double>(xs);
      }
      (half ? xb : xa)[t][c] = v;
    }
    __syncthreads();
#pragma unroll 4
    for (int t = 0; t < kGramChunk; ++t) {
      double ra[R], rb[R];
#pragma unroll
      for (int a = 0; a < R; ++a) ra[a] = xa[t][ty + 16 * a];
#pragma unroll
      for (int b = 0; b < R; ++b) rb[b] = xb[t][tx + 16 * b];
#pragma unroll
      for (int a = 0; a < R; ++a)
#pragma unroll
        for (int b = 0; b < R; ++b) acc[a][b] = __fma_rn(ra[a], rb[b], acc[a][b]);
    }
    __syncthreads();
  }
  if (bad_x) atomicOr(err, kErrNonfiniteX);
  if (bad_s) atomicOr(err, kErrBadScale);
  double* Hg = H + g * G * G;
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int b = 0; b < R; ++b) Hg[(r0 + ty + 16 * a) * G + c0 + tx + 16 * b] = acc[a][b];
}

// ---- clipping search -------------------------------------------------------------------
template <int G>
struct ClipTile {
  static constexpr int RM = G / 16;                 // rows per thread in the product
  static constexpr int EPT = G * kClipCols / kClipThreads;  // W' elements per thread (G / 4)
  static constexpr int kRowStep = kClipThreads / kClipCols; // 4
  static constexpr size_t kSmemH = sizeof(double) * G * G;
  static constexpr size_t kSmemD = sizeof(double) * G * kClipCols;
  static constexpr size_t kSmemRed = sizeof(double) * 16 * kClipCols;
  static constexpr size_t kSmem = kSmemH + kSmemD + kSmemRed;
};

__device__ __forceinline__ float shrink_factor(int i) {
  return __double2float_rn(__dsub_rn(1.0, __ddiv_rn(static_cast<double>(i), static_cast<double>(kShrinkGrid))));
}

__device__ __forceinline__ float clamp_to(float w, float c) { return fminf(fmaxf(w, -c), c); }

template <typename T, int G>
__global__ void __launch_bounds__(kClipThreads, 1)
    clip_kernel(const T* __restrict__ W, int64_t N, const float* __restrict__ s, const double* __restrict__ H,
                int n_shrink, int tokens, float* __restrict__ max_val, int32_t* __restrict__ best_out,
                double* __restrict__ errors, int32_t* __restrict__ codes, __half* __restrict__ steps,
                __half* __restrict__ zeros, int* err) {
  using CT = ClipTile<G>;
  extern __shared__ __align__(16) uint8_t smem[];
  double* sH = reinterpret_cast<double*>(smem);                           // [G][G]
  double* sD = reinterpret_cast<double*>(smem + CT::kSmemH);              // [G][64]
  double* sRed = reinterpret_cast<double*>(smem + CT::kSmemH + CT::kSmemD);  // [16][64]
  __shared__ float sAbs[4][kClipCols], sMin[4][kClipCols], sMax[4][kClipCols];
  __shared__ int sBest[kClipCols];

  const int64_t g = blockIdx.y;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kClipCols;
  const int64_t G_total = gridDim.y;

  // H_g -> shared memory (16-byte vectors; it was written by the previous launch)
  {
    const double2* src = reinterpret_cast<const double2*>(H + g * G * G);
    double2* dst = reinterpret_cast<double2*>(sH);
    for (int i = threadIdx.x; i < G * G / 2; i += kClipThreads) dst[i] = src[i];
  }

  // this thread's share of W': column n, rows k = r + 4 j
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
  sAbs[r][n] = amax;
  sMin[r][n] = mn;
  sMax[r][n] = mx;
  __syncthreads();
  amax = fmaxf(fmaxf(sAbs[0][n], sAbs[1][n]), fmaxf(sAbs[2][n], sAbs[3][n]));
  mn = fminf(fminf(sMin[0][n], sMin[1][n]), fminf(sMin[2][n], sMin[3][n]));
  mx = fmaxf(fmaxf(sMax[0][n], sMax[1][n]), fmaxf(sMax[2][n], sMax[3][n]));

  // product layout: thread (tr, tc) owns rows RM*tr .. RM*tr+RM-1, columns tc + 16 c
  const int tr = threadIdx.x / 16, tc = threadIdx.x % 16;
  double best_e = 0.0;
  int best_i = 0;
  const double tokens_d = static_cast<double>(tokens);

  for (int i = 0; i < n_shrink; ++i) {
    // clamp -> QDQ -> delta. Clamping is monotone, so the clamped group's min and max
    // are the clamped min and max.
    const float c = __fmul_rn(amax, shrink_factor(i));
    const QdqParams p = qdq_params(clamp_to(mn, c), clamp_to(mx, c));
#pragma unroll
    for (int j = 0; j < CT::EPT; ++j) {
      const float q = qdq_code(clamp_to(wp[j], c), p);
      const float rec = __fmul_rn(__fsub_rn(q, p.zero), p.step);
      sD[(r + CT::kRowStep * j) * kClipCols + n] = __dsub_rn(static_cast<double>(rec), static_cast<double>(wp[j]));
    }
    __syncthreads();

    double acc[CT::RM][4];
#pragma unroll
    for (int a = 0; a < CT::RM; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = 0.0;
#pragma unroll 2
    for (int l = 0; l < G; ++l) {
      double ha[CT::RM], db[4];
      const double2* hrow = reinterpret_cast<const double2*>(sH + l * G + CT::RM * tr);  // H symmetric: H[k][l] = H[l][k]
#pragma unroll
      for (int a = 0; a < CT::RM / 2; ++a) {
        const double2 v = hrow[a];
        ha[2 * a] = v.x;
        ha[2 * a + 1] = v.y;
      }
#pragma unroll
      for (int b = 0; b < 4; ++b) db[b] = sD[l * kClipCols + tc + 16 * b];
#pragma unroll
      for (int a = 0; a < CT::RM; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = __fma_rn(ha[a], db[b], acc[a][b]);
    }
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      double pe = 0.0;
#pragma unroll
      for (int a = 0; a < CT::RM; ++a) pe = __fma_rn(sD[(CT::RM * tr + a) * kClipCols + tc + 16 * b], acc[a][b], pe);
      sRed[tr * kClipCols + tc + 16 * b] = pe;
    }
    __syncthreads();
    if (threadIdx.x < kClipCols) {
      double e = 0.0;
#pragma unroll
      for (int q = 0; q < 16; ++q) e = __dadd_rn(e, sRed[q * kClipCols + threadIdx.x]);
      e = __ddiv_rn(e, tokens_d);  // the mean over the sampled tokens
      if (errors && col_ok) errors[(static_cast<int64_t>(i) * G_total + g) * N + n0 + threadIdx.x] = e;
      if (i == 0 || e < best_e) {  // first minimum
        best_e = e;
        best_i = i;
      }
    }
    // the next candidate overwrites sD only after this barrier-separated phase; sRed
    // is rewritten after the next candidate's first barrier
  }
  if (threadIdx.x < kClipCols) sBest[threadIdx.x] = best_i;
  __syncthreads();

  // artifact of the chosen threshold: codes through shared memory, packed eight per
  // int32 along N; steps and zeros as fp16
  const int bi = sBest[n];
  const float c = __fmul_rn(amax, shrink_factor(bi));
  const QdqParams p = qdq_params(clamp_to(mn, c), clamp_to(mx, c));
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
    for (int b = 0; b < 8; ++b) word |= static_cast<uint32_t>(sQ[k * kClipCols + 8 * w + b]) << (4 * b);
    codes[(g * G + k) * words + n0 / 8 + w] = static_cast<int32_t>(word);
  }
}

template <typename T, int G>
cudaError_t launch_clip_t(const ClipArgs& a, cudaStream_t st, int* launches) {
  const int64_t groups = a.K / G;
  const int64_t stride = clip_token_stride(a.M, a.max_tokens);
  {
    constexpr int TB = G < 64 ? G : 64;
    dim3 grid(static_cast<unsigned>(groups), (G / TB) * (G / TB));
    gram_kernel<T, G><<<grid, kGramThreads, 0, st>>>(static_cast<const T*>(a.X), a.K, stride, a.tokens, a.s, a.H,
                                                     a.err);
    *launches += 1;
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  static unsigned long long done = 0;
  cudaError_t e = set_smem_limit_once(clip_kernel<T, G>, static_cast<int>(ClipTile<G>::kSmem), &done);
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(ceil_div(a.N, kClipCols)), static_cast<unsigned>(groups));
  clip_kernel<T, G><<<grid, kClipThreads, ClipTile<G>::kSmem, st>>>(
      static_cast<const T*>(a.W), a.N, a.s, a.H, a.n_shrink, a.tokens, a.max_val, a.best, a.errors, a.codes, a.steps,
      a.zeros, a.err);
  *launches += 1;
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
