// k_qdq.cu — candidate weights and the packed artifact.
//
// qdq_kernel: for every candidate scale vector s_i, W' = diag(s_i) W is quantized and
// dequantized group-wise along K with the asymmetric 4-bit zero-point quantizer and
// folded back, W_hat_i = diag(s_i)^-1 Q(W') ("AWQ：为什么 4-bit 权重量化要先观察
// Activation" §4 candidate loop, §7 quantizer). A CTA stages one `group` x 64 tile of
// W in shared memory once, keeps it in registers, and emits all n_grid candidates
// (plus the plain bf16 copy of W used for the reference output), so W is read from
// HBM once for the whole grid. Each lane owns 8 rows of 2 columns in registers. Phase A
// finds the group range of every (candidate, column) with a shuffle butterfly over the
// row-lanes (its first step also splits the pair of columns between two lanes) and then
// computes each column's parameters once, spread over the warp's lanes, into shared
// memory; phase B streams the candidates: codes, reconstruction and fold-back, each
// lane writing its 8 rows as one 16-byte run of the K-major operand (N x K, K
// contiguous) that the loss GEMM's TMA reads. Elements travel in pairs through sm_100's
// f32x2 multiply/add/fma instructions, which round each half as the scalar ones do.
//
// Arithmetic. The definition is a chain of IEEE fp32 operations (see
// awq_device.cuh): q = clamp(rint(w'/step) + z), W_hat = bf16(((q - z) * step) / s).
// Both divisions use correctly rounded reciprocals (one per column, one per row). The
// fold-back quotient is formed correctly rounded by two fused multiply-add correction
// steps (Markstein's method, div2_rn). The code's quotient is read from the plain product
// w' * (1/step), within 2^-19 of the quotient where its rounding matters; when that
// product lies within 2^-15 of a half-integer (about 6 in 10^5 elements) the warp's run
// is redone with the corrected quotient. Columns or groups outside the range guards take
// the IEEE divisions. Rounding to an integer uses (x + 1.5*2^23) - 1.5*2^23, exact
// round-half-to-even for |x| < 2^22.
//
// pack_kernel: the same quantizer for the chosen candidate only (the first argmin of
// the fp32 losses, computed by every warp), one warp per group x 32-column strip with no
// shared memory: codes are packed eight per int32 along N in registers (QUANT-P4 §5.3)
// and stored directly, steps and zeros are written as fp16, and the chosen scales are
// copied out.
#include "awq_device.cuh"
#include "awq_kernels.h"

namespace awq {
namespace {

constexpr int kQdqCols = 64;                          // columns per CTA
constexpr int kRowsPerLane = 8;                       // one 16-byte bf16 run per column
constexpr float kRoundMagic = 12582912.0f;            // 1.5 * 2^23
constexpr float kNearHalf = 0.5f - 1.0f / 32768.0f;   // |x - rint(x)| at or above this: recheck
// Range guards of the fast arithmetic: a column whose step lies outside [2^-80, 2^80], or
// a group with a scale whose reciprocal lies outside [2^-40, 2^40], takes the definition's
// IEEE divisions instead (no realistic layer comes near these bounds).
constexpr float kTinyStep = 8.271806125530277e-25f;   // 2^-80
constexpr float kHugeStep = 1.2089258196146292e24f;   // 2^80
constexpr float kHugeRecip = 1.2089258196146292e24f;  // 2^80
constexpr float kScaleRecipMin = 9.094947017729282e-13f;  // 2^-40
constexpr float kScaleRecipMax = 1099511627776.0f;        // 2^40

// Thread layout for a group size G and a tile of COLS columns: RL row-lanes x CG
// column-lanes per warp, each lane 8 rows x 2 columns; a warp covers G rows x 2*CG
// columns.
template <int G, int COLS = kQdqCols>
struct Tile {
  static constexpr int RL = G / kRowsPerLane;       // 4, 8, 16
  static constexpr int CG = 32 / RL;                // 8, 4, 2
  static constexpr int kColsPerWarp = 2 * CG;       // 16, 8, 4
  static constexpr int kCols = COLS;
  static constexpr int kWarps = COLS / kColsPerWarp;
  static constexpr int kThreads = 32 * kWarps;      // 64 columns: 128, 256, 512 threads
  static constexpr int kPitch = G + 1;              // transposed W tile, odd pitch
  static constexpr int kSkewPitch = G + G / 16;     // candidate rows of scales, skewed
  static constexpr int kBlocksPerSm = 1024 / kThreads;  // at <= 64 registers
  static_assert(COLS % kColsPerWarp == 0, "whole warps per tile");
};

// Row r of a candidate's scales sits at r + 2 (r / 32): every lane's run of 8 rows starts
// on an even word (pair loads), and the row-lanes' pair loads hit distinct banks (for
// the qdq kernel's row order; the pack kernel reads its own unskewed copy).
__device__ __forceinline__ int skew(int r) { return r + 2 * (r >> 5); }

// Output row of column n in the candidate operand. With interleave = F > 0 (W = [W_gate |
// W_up], 2F columns, F % 128 == 0) every 256 rows hold 128 gate columns followed by the
// 128 up columns of the same outputs, so one 128 x 256 GEMM tile holds both halves of the
// MLP block's 128 intermediate columns; otherwise the identity.
__device__ __forceinline__ int64_t interleaved_column(int64_t n, int64_t interleave) {
  if (interleave <= 0) return n;
  const int64_t half = n >= interleave ? 1 : 0, f = n - half * interleave;
  return (f >> 7) * 256 + half * 128 + (f & 127);
}

__device__ __forceinline__ float round_small(float x) {
  return __fsub_rn(__fadd_rn(x, kRoundMagic), kRoundMagic);
}

// Stage a G x L::kCols tile of W (row pitch ldw elements) transposed in shared memory
// (sWT[col][row]) from coalesced 16-byte global loads; columns at or beyond N read as 0.
// Returns whether a non-finite value was seen.
template <typename T, int G, typename L>
__device__ __forceinline__ bool stage_tile(const T* __restrict__ W, int64_t N, int64_t ldw, int64_t k0, int64_t n0,
                                           float* sWT) {
  constexpr int VEC = 16 / sizeof(T);
  constexpr int VPR = L::kCols / VEC;
  bool bad = false;
  for (int idx = threadIdx.x; idx < G * VPR; idx += L::kThreads) {
    const int r = idx / VPR, v = idx % VPR;
    const int64_t col = n0 + static_cast<int64_t>(v) * VEC;
    float vals[VEC];
    if (col < N) {  // N % 8 == 0: a vector lies wholly inside or outside
      const uint4 raw = __ldcs(reinterpret_cast<const uint4*>(W + (k0 + r) * ldw + col));
      const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
      for (int i = 0; i < VEC; ++i) {
        vals[i] = to_f32<T>(e[i]);
        bad |= !isfinite(vals[i]);
      }
    } else {
#pragma unroll
      for (int i = 0; i < VEC; ++i) vals[i] = 0.0f;
    }
#pragma unroll
    for (int i = 0; i < VEC; ++i) sWT[(v * VEC + i) * L::kPitch + r] = vals[i];
  }
  return bad;
}

struct ColumnQdq {
  QdqParams p;
  float recip;  // correctly rounded 1/step
  bool exact;   // take the exact path for the whole column
};

// Finish both columns' group min/max across the RL row-lanes that share them (a
// butterfly over the low lane bits), then compute each column's parameters once per
// column-group — even row-lanes column 0, odd ones column 1 — and broadcast them.
template <int RL>
__device__ __forceinline__ void column_qdq(float (&mn)[2], float (&mx)[2], ColumnQdq (&cq)[2], int quantizer) {
#pragma unroll
  for (int o = 1; o < RL; o <<= 1) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      mn[j] = fminf(mn[j], __shfl_xor_sync(0xffffffffu, mn[j], o));
      mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], o));
    }
  }
  const int lane = threadIdx.x & 31;
  const int odd = lane & 1;
  const QdqParams p = qdq_params_q(odd ? mn[1] : mn[0], odd ? mx[1] : mx[0], quantizer);
  const float r = __frcp_rn(p.step);
  const int exact = !(p.step >= kTinyStep && r <= kHugeRecip);
  const int base = lane & ~(RL - 1);
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    cq[j].p.step = __shfl_sync(0xffffffffu, p.step, base + j);
    cq[j].p.zero = __shfl_sync(0xffffffffu, p.zero, base + j);
    cq[j].p.qmax = p.qmax;  // the same for every column of the launch
    cq[j].recip = __shfl_sync(0xffffffffu, r, base + j);
    cq[j].exact = __shfl_sync(0xffffffffu, exact, base + j) != 0;
  }
}

// ---- the candidate loop ---------------------------------------------------------------
// sm_100's f32x2 instructions round each half exactly as the scalar instruction does
// (round to nearest even, subnormals kept), so a pair of elements costs one issue per
// operation of the definition's chain; three-input min/max halve the range reductions.
__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Range of the 8 values held as four pairs.
__device__ __forceinline__ void range8(const float2 (&v)[4], float& mn, float& mx) {
  mn = fmin3(fmin3(v[0].x, v[0].y, v[1].x), fmin3(v[1].y, v[2].x, v[2].y), fminf(v[3].x, v[3].y));
  mx = fmax3(fmax3(v[0].x, v[0].y, v[1].x), fmax3(v[1].y, v[2].x, v[2].y), fmaxf(v[3].x, v[3].y));
}

__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// One column's quantizer parameters from its group range, with the step's correctly
// rounded reciprocal and whether the column takes the exact path. The step is the
// definition's division. The zero point clamp(rint(-min / step), 0, 15) is read from
// t = -min * (1/step), first clamped to [-1, 16] (which leaves the clamped zero
// unchanged): for |t| <= 16.5 that product is within 2^-19 of the quotient, so its
// rounding agrees unless t lies within 2^-15 of a half-integer, where the exact division
// decides.
__device__ __forceinline__ ColumnQdq column_params(float mn, float mx, int quantizer) {
  ColumnQdq c;
  if (quantizer == kQuantSym) {
    c.p = qdq_params_sym(mn, mx);
    c.recip = __frcp_rn(c.p.step);
  } else {
    float step = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
    if (mx == mn || step == 0.0f) step = 1.0f;  // all-equal group (or underflow): step 1
    const float r = __frcp_rn(step);
    const float t = fminf(fmaxf(__fmul_rn(-mn, r), -1.0f), 16.0f);
    float z = round_small(t);
    if (fabsf(__fsub_rn(t, z)) >= kNearHalf || !(step >= kTinyStep && r <= kHugeRecip))
      z = rintf(__fdiv_rn(-mn, step));
    z = fminf(fmaxf(z, 0.0f), 15.0f);
    c.p.step = step;
    c.p.zero = __fadd_rn(z, 0.0f);  // rint(-0.25) = -0 becomes +0
    c.p.qmax = 15.0f;
    c.recip = r;
  }
  c.exact = !(c.p.step >= kTinyStep && c.p.step <= kHugeStep && c.recip <= kHugeRecip);
  return c;
}

// Correctly rounded quotients a / b of a pair, given nb = -b and r = RN(1/b), by two
// correction steps (P. Markstein, "Computation of elementary functions on the IBM RISC
// System/6000 processor", IBM J. Res. Dev. 34(1), 1990). RN(a r) lies within 1.5 ulps
// of a / b; q + (a - b q) r, the remainder taken from one fused multiply-add, lands
// within half an ulp plus a term of order 2^-23 ulp, i.e. on a neighbour of a / b; from
// such a faithful q the remainder is exact and the same step returns RN(a / b)
// (Markstein's theorem). Valid while no intermediate underflows or overflows, which the
// callers' range guards (kTinyStep, kHugeRecip, kScaleRecipMin/Max) ensure.
__device__ __forceinline__ float2 div2_rn(float2 a, float2 nb, float2 r) {
  float2 q = __fmul2_rn(a, r);
  q = __ffma2_rn(__ffma2_rn(q, nb, a), r, q);
  return __ffma2_rn(__ffma2_rn(q, nb, a), r, q);
}

// Codes (as q - z), reconstruction and fold-back of 8 rows of one column held as four
// pairs (wp = W', ns = -s, rs = RN(1/s)), rounded to bf16 pairs. The quotient w' / step
// is read from w' * (1/step) (within 2^-19 of it for |t| <= 16.5, the range where its
// rounding matters); kExactT forms it with div2_rn instead. Returns whether any quotient
// lay within 2^-15 of a half-integer, where only the exact quotient decides the code.
template <bool kClamp, bool kExactT>
__device__ __forceinline__ bool fold_back_pairs(const float2 (&wp)[4], const float2 (&ns)[4], const float2* rs,
                                                const ColumnQdq& c, uint32_t (&out)[4]) {
  const float2 rc = make_float2(c.recip, c.recip), st = make_float2(c.p.step, c.p.step);
  const float2 nst = make_float2(-c.p.step, -c.p.step);
  const float2 magic = make_float2(kRoundMagic, kRoundMagic), nmagic = make_float2(-kRoundMagic, -kRoundMagic);
  const float2 minus1 = make_float2(-1.0f, -1.0f);
  const float lo = -c.p.zero, hi = c.p.qmax - c.p.zero;
  float dmax = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (!kClamp && !kExactT) {
      // The usual case, one operation shorter: a fused multiply-add rounds the exact
      // product w' (1/step) onto -1.5 2^23, which gives -(q - z) once 1.5 2^23 is added back
      // (the product is not rounded first, which only brings it closer to the quotient), and
      // a second one gives w' (1/step) - (q - z) for the half-integer check.
      const float2 nrc = make_float2(-c.recip, -c.recip);
      const float2 nqz = __fadd2_rn(__ffma2_rn(wp[i], nrc, nmagic), magic);  // -(q - z)
      const float2 d = __ffma2_rn(wp[i], rc, nqz);
      dmax = fmax3(dmax, fabsf(d.x), fabsf(d.y));
      const float2 v = div2_rn(__fmul2_rn(nqz, nst), ns[i], rs[i]);  // ((q - z) step) / s
      out[i] = bf16x2_bits(v.x, v.y);
      continue;
    }
    float2 t = kExactT ? div2_rn(wp[i], nst, rc) : __fmul2_rn(wp[i], rc);
    if (kClamp) {
      t.x = fminf(fmaxf(t.x, lo), hi);
      t.y = fminf(fmaxf(t.y, lo), hi);
    }
    const float2 qz = __fadd2_rn(__fadd2_rn(t, magic), nmagic);  // q - z, round half to even
    if (!kExactT) {
      const float2 d = __ffma2_rn(qz, minus1, t);  // t - (q - z), exact
      dmax = fmax3(dmax, fabsf(d.x), fabsf(d.y));
    }
    const float2 v = div2_rn(__fmul2_rn(qz, st), ns[i], rs[i]);  // ((q - z) step) / s
    out[i] = bf16x2_bits(v.x, v.y);
  }
  return dmax >= kNearHalf;
}

// The definition's chain, divisions included, for 8 rows of one column; kept out of line
// so that its division subroutines do not weigh on the candidate loop's registers.
__device__ __forceinline__ uint32_t exact_pair(float2 w, float2 s, QdqParams p) {
  const float2 wp = __fmul2_rn(s, w);
  return bf16x2_bits(qdq_fold_back(qdq_code(wp.x, p), p, s.x), qdq_fold_back(qdq_code(wp.y, p), p, s.y));
}
__device__ __noinline__ void exact_run(float2 w0, float2 w1, float2 w2, float2 w3, float2 s0, float2 s1, float2 s2,
                                       float2 s3, QdqParams p, uint4* dst) {
  *dst = make_uint4(exact_pair(w0, s0, p), exact_pair(w1, s1, p), exact_pair(w2, s2, p), exact_pair(w3, s3, p));
}

template <typename T, int G>
__global__ void __launch_bounds__(Tile<G>::kThreads, Tile<G>::kBlocksPerSm)
    qdq_kernel(const T* __restrict__ W, int64_t K, int64_t N, int n_grid, const float* __restrict__ S,
               __nv_bfloat16* __restrict__ Wt, int* err, int64_t group0, int quantizer, int64_t interleave,
               int64_t ldw) {
  using L = Tile<G>;
  extern __shared__ float smem[];
  float* sWT = smem;                                    // [64][kPitch]
  float* sS = sWT + L::kCols * L::kPitch;               // [n_grid][kSkewPitch] negated scales -s
  float* sR = sS + n_grid * L::kSkewPitch;              // [n_grid][kSkewPitch] correctly rounded 1/s
  float4* sPar = reinterpret_cast<float4*>(sR + n_grid * L::kSkewPitch);  // [n_grid][64] column parameters
  __shared__ uint32_t sRowsExact[2];                    // candidates with an extreme 1/s in this group

  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * L::kCols;
  const int64_t k0 = (group0 + static_cast<int64_t>(blockIdx.y)) * G;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float qmax = quantizer == kQuantSym ? 14.0f : 15.0f;

  if (threadIdx.x < 2) sRowsExact[threadIdx.x] = 0u;
  __syncthreads();
  if (stage_tile<T, G, L>(W, N, ldw, k0, n0, sWT)) atomicOr(err, kErrNonfiniteW);
  for (int idx = threadIdx.x; idx < n_grid * G; idx += L::kThreads) {
    const int c = idx / G, r = idx % G;
    const float s = S[static_cast<int64_t>(c) * K + k0 + r];
    const float rs = __frcp_rn(s);
    sS[c * L::kSkewPitch + skew(r)] = -s;
    sR[c * L::kSkewPitch + skew(r)] = rs;
    if (!(fabsf(rs) <= kScaleRecipMax && fabsf(rs) >= kScaleRecipMin)) atomicOr(&sRowsExact[c >> 5], 1u << (c & 31));
  }
  __syncthreads();

  // Lane (rl, cg) holds 8 rows of two adjacent columns, negated (W' = (-s)(-w) exactly,
  // and -s is what the fold-back's remainders need); w2[0] is its own column
  // (col0 + (rl & 1)), w2[1] the other one, so that the first butterfly step hands each
  // lane of a pair the other's partial range of the lane's own column. Even row-lanes
  // hold the first half of the group's rows and odd ones the second, so that each
  // store instruction writes whole 128-byte runs of both columns.
  const int rl = lane % L::RL, cg = lane / L::RL;
  const int own = rl & 1;
  const int col0 = warp * L::kColsPerWarp + cg * 2;
  const int row0 = (rl >> 1) * kRowsPerLane + own * (G / 2);
  const bool active = n0 + col0 < N;  // N is even: both columns are in or both out
  __nv_bfloat16* const dst0 = Wt + interleaved_column(n0 + col0 + own, interleave) * K + k0 + row0;
  const int64_t dst1_off = own ? -K : K;  // the lane's other column (a pair never straddles 128 columns)

  float2 w2[2][4];
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float* src = sWT + (col0 + (j ^ own)) * L::kPitch + row0 + 2 * i;
      w2[j][i] = make_float2(-src[0], -src[1]);
    }

  // reference operand: bf16(W), transposed
  if (active) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      uint4 v;
      v.x = bf16x2_bits(-w2[j][0].x, -w2[j][0].y);
      v.y = bf16x2_bits(-w2[j][1].x, -w2[j][1].y);
      v.z = bf16x2_bits(-w2[j][2].x, -w2[j][2].y);
      v.w = bf16x2_bits(-w2[j][3].x, -w2[j][3].y);
      *reinterpret_cast<uint4*>(dst0 + (j ? dst1_off : 0)) = v;
    }
  }
  const int srow = skew(row0);  // even, and the lane's 8 rows never straddle a skew pad

  // Phase A: the group range of every (candidate, column) of the warp: W' = s W per
  // lane, then a butterfly over the RL row-lanes whose first step also splits the two
  // columns between the lanes of a pair.
  for (int c = 0; c < n_grid; ++c) {
    const float2* sp = reinterpret_cast<const float2*>(sS + c * L::kSkewPitch + srow);
    float mn[2], mx[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float2 wp[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) wp[i] = __fmul2_rn(sp[i], w2[j][i]);
      range8(wp, mn[j], mx[j]);
    }
    float mo = fminf(mn[0], __shfl_xor_sync(0xffffffffu, mn[1], 1));
    float Mo = fmaxf(mx[0], __shfl_xor_sync(0xffffffffu, mx[1], 1));
#pragma unroll
    for (int o = 2; o < L::RL; o <<= 1) {
      mo = fminf(mo, __shfl_xor_sync(0xffffffffu, mo, o));
      Mo = fmaxf(Mo, __shfl_xor_sync(0xffffffffu, Mo, o));
    }
    if (rl < 2) sPar[c * L::kCols + col0 + own] = make_float4(mo, Mo, 0.0f, 0.0f);
  }
  __syncwarp();
  // ... and each (candidate, column) parameter set computed once, spread over the lanes:
  // step, zero, 1/step and flags (1: outside the range guards, 2: no element can clamp,
  // since t = w' * (1/step) is monotone in w' and kNearHalf covers the distance to the
  // quotient)
  for (int it = lane; it < n_grid * L::kColsPerWarp; it += 32) {
    float4* e = &sPar[(it / L::kColsPerWarp) * L::kCols + warp * L::kColsPerWarp + it % L::kColsPerWarp];
    const float mo = e->x, Mo = e->y;
    const ColumnQdq q = column_params(mo, Mo, quantizer);
    const bool clamp_free = !q.exact && __fmul_rn(mo, q.recip) >= -q.p.zero - kNearHalf &&
                            __fmul_rn(Mo, q.recip) <= q.p.qmax - q.p.zero + kNearHalf;
    *e = make_float4(q.p.step, q.p.zero, q.recip, __int_as_float((q.exact ? 1 : 0) | (clamp_free ? 2 : 0)));
  }
  __syncwarp();

  // Phase B: codes, reconstruction and fold-back of every candidate. A candidate for
  // which one of the lane's runs holds a code decided only by the exact quotient, lies
  // outside the range guards, or may clamp a code (a column whose zero point clips its
  // range, or whose rounded zero sits half a step from the range's end) is recorded and
  // redone after the pass (the thread rewrites its own stores), which keeps the rare
  // paths out of the streaming loop: it runs one instruction stream for every lane.
  uint64_t redo = 0;
  for (int c = 0; c < n_grid; ++c) {
    float2 s2[4];
    {
      const float2* sp = reinterpret_cast<const float2*>(sS + c * L::kSkewPitch + srow);
#pragma unroll
      for (int i = 0; i < 4; ++i) s2[i] = sp[i];
    }
    const float2* rs = reinterpret_cast<const float2*>(sR + c * L::kSkewPitch + srow);
    bool flag = (sRowsExact[c >> 5] >> (c & 31)) & 1u;
    __nv_bfloat16* const slot = dst0 + static_cast<int64_t>(c + 1) * N * K;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float4 e = sPar[c * L::kCols + col0 + (j ^ own)];
      ColumnQdq cq;
      cq.p.step = e.x;
      cq.p.zero = e.y;
      cq.p.qmax = qmax;
      cq.recip = e.z;
      const int flags = __float_as_int(e.w);
      float2 wp[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) wp[i] = __fmul2_rn(s2[i], w2[j][i]);
      uint32_t out[4];
      flag |= (flags & 3) != 2;  // outside the range guards, or a code may clamp
      flag |= fold_back_pairs<false, false>(wp, s2, rs, cq, out);
      if (active) *reinterpret_cast<uint4*>(slot + (j ? dst1_off : 0)) = make_uint4(out[0], out[1], out[2], out[3]);
    }
    redo |= static_cast<uint64_t>(flag) << c;
  }

  // the recorded candidates of this lane: codes from the corrected quotients, and the
  // IEEE divisions for columns or groups outside the range guards
  while (redo && active) {
    const int c = __ffsll(static_cast<long long>(redo)) - 1;
    redo &= redo - 1;
    float2 s2[4];
    {
      const float2* sp = reinterpret_cast<const float2*>(sS + c * L::kSkewPitch + srow);
#pragma unroll
      for (int i = 0; i < 4; ++i) s2[i] = sp[i];
    }
    const float2* rs = reinterpret_cast<const float2*>(sR + c * L::kSkewPitch + srow);
    const bool rows_x = (sRowsExact[c >> 5] >> (c & 31)) & 1u;
    __nv_bfloat16* const slot = dst0 + static_cast<int64_t>(c + 1) * N * K;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float4 e = sPar[c * L::kCols + col0 + (j ^ own)];
      ColumnQdq cq;
      cq.p.step = e.x;
      cq.p.zero = e.y;
      cq.p.qmax = qmax;
      cq.recip = e.z;
      const int flags = __float_as_int(e.w);
      uint4* const dst = reinterpret_cast<uint4*>(slot + (j ? dst1_off : 0));
      if (rows_x || (flags & 1)) {
        const float2 m1 = make_float2(-1.0f, -1.0f);
        exact_run(__fmul2_rn(w2[j][0], m1), __fmul2_rn(w2[j][1], m1), __fmul2_rn(w2[j][2], m1),
                  __fmul2_rn(w2[j][3], m1), __fmul2_rn(s2[0], m1), __fmul2_rn(s2[1], m1), __fmul2_rn(s2[2], m1),
                  __fmul2_rn(s2[3], m1), cq.p, dst);
      } else {
        float2 wp[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) wp[i] = __fmul2_rn(s2[i], w2[j][i]);
        uint32_t out[4];
        if (flags & 2)
          fold_back_pairs<false, true>(wp, s2, rs, cq, out);
        else
          fold_back_pairs<true, true>(wp, s2, rs, cq, out);
        *dst = make_uint4(out[0], out[1], out[2], out[3]);
      }
    }
  }
}

// Lane layout of the pack kernel: each warp quantizes one group x kCols strip on its
// own, with no shared memory and no block barrier. Lane (lr, lc) = (lane / LC, lane % LC)
// holds the 16-byte vector of VEC adjacent columns (lc VEC .. lc VEC + VEC - 1 of the
// strip) in rows lr, lr + LR, ..., so every load instruction reads eight 64-byte row runs.
// (Two lanes across and 16 down, at 80 registers and 24 warps per SM, ran no faster.)
template <typename T, int G>
struct PackShape {
  static constexpr int VEC = 16 / sizeof(T);  // columns per lane: 8 (bf16) or 4 (fp32)
  static constexpr int LC = 4;                // lanes across the strip
  static constexpr int LR = 32 / LC;          // lanes down the group
  static constexpr int RPL = G / LR;          // rows per lane: 16, 8, 4
  static constexpr int kCols = LC * VEC;      // columns per warp: 32 or 16
  static constexpr int kWarps = 4;
  static constexpr int kThreads = 32 * kWarps;
};

// A read-only load the compiler cannot merge with an earlier one of the same address, so
// the first pass's value need not stay live in a register (an L1 hit).
__device__ __forceinline__ float reload_f32(const float* p) {
  float v;
  asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
}

// The VEC values of a 16-byte vector times s, as pairs (bf16 widened by a shift or a mask).
template <typename T>
__device__ __forceinline__ void scaled_pairs(const uint4& raw, float s, float2 (&out)[8 / sizeof(T)]) {
  const float2 s2 = make_float2(s, s);
  const uint32_t u[4] = {raw.x, raw.y, raw.z, raw.w};
  if constexpr (sizeof(T) == 2) {
#pragma unroll
    for (int h = 0; h < 4; ++h)
      out[h] = __fmul2_rn(s2, make_float2(__uint_as_float(u[h] << 16), __uint_as_float(u[h] & 0xFFFF0000u)));
  } else {
#pragma unroll
    for (int h = 0; h < 2; ++h)
      out[h] = __fmul2_rn(s2, make_float2(__uint_as_float(u[2 * h]), __uint_as_float(u[2 * h + 1])));
  }
}

template <typename T>
__device__ __forceinline__ void unpack16(const uint4& raw, float (&w)[16 / sizeof(T)]) {
  const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
  for (int j = 0; j < static_cast<int>(16 / sizeof(T)); ++j) w[j] = to_f32<T>(e[j]);
}

// Codes of the chosen candidate with its group steps and zeros, packed eight per int32
// along N. Per lane: the group range of each of its columns over its rows, finished by a
// butterfly over the eight row-lanes; each row-lane then computes one column's parameters
// (the definition's divisions) and shares them; codes come from the correctly rounded
// reciprocal of the step with the same half-integer check as the candidate kernel, and a
// row holding a code that only the exact quotient decides is redone with the IEEE
// division after the pass. A lane's VEC codes of a row form one int32 (bf16) or its low
// or high 16 bits (fp32), stored directly.
template <typename T, int G>
__global__ void __launch_bounds__(PackShape<T, G>::kThreads, 4)
    pack_kernel(const T* __restrict__ W, int64_t K, int64_t N, int n_grid, const float* __restrict__ S,
                const float* __restrict__ losses, int* __restrict__ best_out, int32_t* __restrict__ codes,
                __half* __restrict__ steps, __half* __restrict__ zeros, float* __restrict__ out_scales,
                int quantizer) {
  using P = PackShape<T, G>;
  constexpr int VEC = P::VEC;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int lc = lane % P::LC, lr = lane / P::LC;
  const int64_t k0 = static_cast<int64_t>(blockIdx.y) * G;
  const int64_t n0 = (static_cast<int64_t>(blockIdx.x) * P::kWarps + warp) * P::kCols;
  const int64_t nl = n0 + lc * VEC;  // the lane's first column
  const bool active = nl < N;        // N % 8 == 0: a lane's columns are all in or all out
  const int64_t words = N / 8;

  uint4 raw[P::RPL];
  if (active) {
#pragma unroll
    for (int i = 0; i < P::RPL; ++i) raw[i] = __ldcs(reinterpret_cast<const uint4*>(W + (k0 + lr + P::LR * i) * N + nl));
  } else {
#pragma unroll
    for (int i = 0; i < P::RPL; ++i) raw[i] = make_uint4(0u, 0u, 0u, 0u);
  }

  // the chosen candidate: first minimum of the fp32 losses
  int best = 0;
  if (lane == 0) {
    float bv = losses[0];
    for (int c = 1; c < n_grid; ++c) {
      const float v = losses[c];
      if (v < bv) {
        bv = v;
        best = c;
      }
    }
    if (blockIdx.x == 0 && blockIdx.y == 0 && warp == 0) *best_out = best;
  }
  best = __shfl_sync(0xffffffffu, best, 0);
  const float* Sb = S + static_cast<int64_t>(best) * K + k0;
  float s[P::RPL];
#pragma unroll
  for (int i = 0; i < P::RPL; ++i) s[i] = Sb[lr + P::LR * i];
  if (n0 == 0 && lc == 0) {
#pragma unroll
    for (int i = 0; i < P::RPL; ++i) out_scales[k0 + lr + P::LR * i] = s[i];
  }

  // group range of the lane's columns over its rows (two rows per three-input min / max),
  // then across the row-lanes
  float mn[VEC], mx[VEC];
#pragma unroll
  for (int j = 0; j < VEC; ++j) {
    mn[j] = INFINITY;
    mx[j] = -INFINITY;
  }
#pragma unroll
  for (int i = 0; i < P::RPL; i += 2) {
    float2 a[VEC / 2], b[VEC / 2];
    scaled_pairs<T>(raw[i], s[i], a);
    scaled_pairs<T>(raw[i + 1], s[i + 1], b);
#pragma unroll
    for (int h = 0; h < VEC / 2; ++h) {
      mn[2 * h] = fmin3(mn[2 * h], a[h].x, b[h].x);
      mx[2 * h] = fmax3(mx[2 * h], a[h].x, b[h].x);
      mn[2 * h + 1] = fmin3(mn[2 * h + 1], a[h].y, b[h].y);
      mx[2 * h + 1] = fmax3(mx[2 * h + 1], a[h].y, b[h].y);
    }
  }
#pragma unroll
  for (int o = P::LC; o < 32; o <<= 1)
#pragma unroll
    for (int j = 0; j < VEC; ++j) {
      mn[j] = fminf(mn[j], __shfl_xor_sync(0xffffffffu, mn[j], o));
      mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xffffffffu, mx[j], o));
    }

  // row-lane lr computes the parameters of column lr % VEC of its strip, and shares them
  const int jc = lr % VEC;
  float cmn = mn[0], cmx = mx[0];
#pragma unroll
  for (int j = 1; j < VEC; ++j)
    if (jc == j) {
      cmn = mn[j];
      cmx = mx[j];
    }
  const QdqParams pc = qdq_params_q(cmn, cmx, quantizer);
  const float rc = __frcp_rn(pc.step);
  const int exact_c = !(pc.step >= kTinyStep && rc <= kHugeRecip);
  if (active && lr < VEC) {
    const int64_t o = (k0 / G) * N + nl + jc;
    steps[o] = __float2half_rn(pc.step);
    zeros[o] = __float2half_rn(pc.zero);
  }
  // per column: 1/step, the clamp bounds lo = -z and hi = qmax - z (integers, so z = -lo
  // and qmax = hi - lo exactly), -(1.5 2^23 + z), and the step for the exact path
  float rcp[VEC], lo[VEC], hi[VEC], nmz[VEC], stp[VEC];
  bool col_exact = false;
#pragma unroll
  for (int j = 0; j < VEC; ++j) {
    const int src = j * P::LC + lc;
    stp[j] = __shfl_sync(0xffffffffu, pc.step, src);
    const float z = __shfl_sync(0xffffffffu, pc.zero, src);
    rcp[j] = __shfl_sync(0xffffffffu, rc, src);
    col_exact |= __shfl_sync(0xffffffffu, exact_c, src) != 0;
    lo[j] = -z;
    hi[j] = __fsub_rn(pc.qmax, z);
    nmz[j] = -__fadd_rn(kRoundMagic, z);
  }

  // codes: t = clamp(w' (1/step), -z, qmax - z); m = RN(t + 1.5 2^23 + z) holds rint(t) + z
  // = q in its low bits (the two agree unless t is a half-integer, which the check below
  // sends to the exact path). The low bytes of a row's m values are gathered with byte
  // permutes and their low nibbles merged into the packed word. W' is formed again from
  // the raw vectors (the empty asm hides them from the compiler, which would otherwise keep
  // the first pass's VEC x RPL products live in registers).
#pragma unroll
  for (int i = 0; i < P::RPL; ++i)
    asm volatile("" : "+r"(raw[i].x), "+r"(raw[i].y), "+r"(raw[i].z), "+r"(raw[i].w));
  const float2 minus1 = make_float2(-1.0f, -1.0f);
  uint32_t redo = 0;
  int32_t* const crow = codes + k0 * words + nl / 8;
#pragma unroll
  for (int i = 0; i < P::RPL; ++i) {
    float2 wp[VEC / 2];
    scaled_pairs<T>(raw[i], reload_f32(Sb + lr + P::LR * i), wp);
    uint32_t mb[VEC];
    float dmax = 0.0f;
#pragma unroll
    for (int h = 0; h < VEC / 2; ++h) {
      float2 tc = __fmul2_rn(wp[h], make_float2(rcp[2 * h], rcp[2 * h + 1]));
      tc.x = fminf(fmaxf(tc.x, lo[2 * h]), hi[2 * h]);
      tc.y = fminf(fmaxf(tc.y, lo[2 * h + 1]), hi[2 * h + 1]);
      const float2 nm = make_float2(nmz[2 * h], nmz[2 * h + 1]);
      const float2 m = __ffma2_rn(nm, minus1, tc);         // t + 1.5 2^23 + z, rounded once
      const float2 d = __ffma2_rn(__fadd2_rn(m, nm), minus1, tc);  // t - rint(t), exact
      dmax = fmax3(dmax, fabsf(d.x), fabsf(d.y));
      mb[2 * h] = __float_as_uint(m.x);
      mb[2 * h + 1] = __float_as_uint(m.y);
    }
    redo |= static_cast<uint32_t>(dmax >= kNearHalf) << i;
    if (active) {
      if constexpr (VEC == 8) {
        const uint32_t ev = __byte_perm(__byte_perm(mb[0], mb[2], 0x0040), __byte_perm(mb[4], mb[6], 0x0040), 0x5410);
        const uint32_t od = __byte_perm(__byte_perm(mb[1], mb[3], 0x0040), __byte_perm(mb[5], mb[7], 0x0040), 0x5410);
        crow[(lr + P::LR * i) * words] = static_cast<int32_t>((ev & 0x0F0F0F0Fu) | ((od << 4) & 0xF0F0F0F0u));
      } else {
        const uint32_t ev = __byte_perm(mb[0], mb[2], 0x0040), od = __byte_perm(mb[1], mb[3], 0x0040);
        reinterpret_cast<uint16_t*>(crow + (lr + P::LR * i) * words)[lc & 1] =
            static_cast<uint16_t>((ev & 0x0F0Fu) | ((od << 4) & 0xF0F0u));
      }
    }
  }
  if (col_exact) redo = (1u << P::RPL) - 1u;
  // rows with a code decided only by the exact quotient (or columns outside the range
  // guards): the definition's division, rewriting the lane's own stores
  while (redo && active) {
    const int i = __ffs(redo) - 1;
    redo &= redo - 1;
    const int64_t r = lr + P::LR * i;
    const uint4 v = *reinterpret_cast<const uint4*>(W + (k0 + r) * N + nl);
    const float sv = Sb[r];
    float w[VEC];
    unpack16<T>(v, w);
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < VEC; ++j) {
      const QdqParams pj{stp[j], -lo[j], __fsub_rn(hi[j], lo[j])};
      word |= static_cast<uint32_t>(qdq_code(__fmul_rn(sv, w[j]), pj)) << (4 * j);
    }
    if (VEC == 8)
      crow[r * words] = static_cast<int32_t>(word);
    else
      reinterpret_cast<uint16_t*>(crow + r * words)[lc & 1] = static_cast<uint16_t>(word);
  }
}

template <typename T, int G>
cudaError_t launch_qdq_t(const T* W, int64_t K, int64_t N, int n_grid, const float* S, __nv_bfloat16* Wt,
                         int* err, int64_t group0, int64_t groups, cudaStream_t s, int quantizer,
                         int64_t interleave, int64_t ldw) {
  using L = Tile<G>;
  auto bytes = [](int grid_points) {
    return (static_cast<size_t>(L::kCols) * L::kPitch + 2 * static_cast<size_t>(grid_points) * L::kSkewPitch +
            4 * static_cast<size_t>(grid_points) * L::kCols) * sizeof(float);
  };
  // the limit is raised once, to what the largest grid (64 candidates) needs
  static unsigned long long attr_done = 0;
  cudaError_t e = set_smem_limit_once(qdq_kernel<T, G>, static_cast<int>(bytes(64)), &attr_done);
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(ceil_div(N, static_cast<int64_t>(L::kCols))), static_cast<unsigned>(groups));
  qdq_kernel<T, G><<<grid, L::kThreads, bytes(n_grid), s>>>(W, K, N, n_grid, S, Wt, err, group0, quantizer,
                                                            interleave, ldw > 0 ? ldw : N);
  return cudaGetLastError();
}

template <typename T, int G>
cudaError_t launch_pack_t(const T* W, int64_t K, int64_t N, int n_grid, const float* S, const float* losses,
                          int* best, int32_t* codes, __half* steps, __half* zeros, float* out_scales,
                          cudaStream_t s, int quantizer) {
  using P = PackShape<T, G>;
  dim3 grid(static_cast<unsigned>(ceil_div(N, static_cast<int64_t>(P::kWarps) * P::kCols)),
            static_cast<unsigned>(K / G));
  pack_kernel<T, G><<<grid, P::kThreads, 0, s>>>(W, K, N, n_grid, S, losses, best, codes, steps, zeros, out_scales,
                                                 quantizer);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_qdq_groups(const void* W, int in_dtype, int64_t K, int64_t N, int group, int n_grid,
                              const float* S, __nv_bfloat16* Wt, int* err, int64_t group0, int64_t groups,
                              cudaStream_t s, int* launches, int quantizer, int64_t interleave, int64_t ldw) {
  *launches += 1;
  if (in_dtype == 0) {
    const auto* w = static_cast<const __nv_bfloat16*>(W);
    switch (group) {
      case 32: return launch_qdq_t<__nv_bfloat16, 32>(w, K, N, n_grid, S, Wt, err, group0, groups, s, quantizer, interleave, ldw);
      case 64: return launch_qdq_t<__nv_bfloat16, 64>(w, K, N, n_grid, S, Wt, err, group0, groups, s, quantizer, interleave, ldw);
      default: return launch_qdq_t<__nv_bfloat16, 128>(w, K, N, n_grid, S, Wt, err, group0, groups, s, quantizer, interleave, ldw);
    }
  }
  const auto* w = static_cast<const float*>(W);
  switch (group) {
    case 32: return launch_qdq_t<float, 32>(w, K, N, n_grid, S, Wt, err, group0, groups, s, quantizer, interleave, ldw);
    case 64: return launch_qdq_t<float, 64>(w, K, N, n_grid, S, Wt, err, group0, groups, s, quantizer, interleave, ldw);
    default: return launch_qdq_t<float, 128>(w, K, N, n_grid, S, Wt, err, group0, groups, s, quantizer, interleave, ldw);
  }
}

cudaError_t launch_qdq(const void* W, int in_dtype, int64_t K, int64_t N, int group, int n_grid, const float* S,
                       __nv_bfloat16* Wt, int* err, cudaStream_t s, int* launches, int quantizer, int64_t interleave,
                       int64_t ldw) {
  return launch_qdq_groups(W, in_dtype, K, N, group, n_grid, S, Wt, err, 0, K / group, s, launches, quantizer,
                           interleave, ldw);
}

cudaError_t launch_pack(const void* W, int in_dtype, int64_t K, int64_t N, int group, int n_grid, const float* S,
                        const float* losses, int* best, int32_t* codes, __half* steps, __half* zeros,
                        float* out_scales, cudaStream_t s, int* launches, int quantizer) {
  *launches += 1;
  if (in_dtype == 0) {
    const auto* w = static_cast<const __nv_bfloat16*>(W);
    switch (group) {
      case 32: return launch_pack_t<__nv_bfloat16, 32>(w, K, N, n_grid, S, losses, best, codes, steps, zeros, out_scales, s, quantizer);
      case 64: return launch_pack_t<__nv_bfloat16, 64>(w, K, N, n_grid, S, losses, best, codes, steps, zeros, out_scales, s, quantizer);
      default: return launch_pack_t<__nv_bfloat16, 128>(w, K, N, n_grid, S, losses, best, codes, steps, zeros, out_scales, s, quantizer);
    }
  }
  const auto* w = static_cast<const float*>(W);
  switch (group) {
    case 32: return launch_pack_t<float, 32>(w, K, N, n_grid, S, losses, best, codes, steps, zeros, out_scales, s, quantizer);
    case 64: return launch_pack_t<float, 64>(w, K, N, n_grid, S, losses, best, codes, steps, zeros, out_scales, s, quantizer);
    default: return launch_pack_t<float, 128>(w, K, N, n_grid, S, losses, best, codes, steps, zeros, out_scales, s, quantizer);
  }
}

}  // namespace awq
