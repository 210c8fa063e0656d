// qdq_tile.cuh — the candidate-weight tile shared by the stand-alone QDQ kernel and the
// loss GEMM's QDQ warps ("AWQ：为什么 4-bit 权重量化要先观察 Activation" §4 candidate loop,
// §7 quantizer). For a G x COLS tile of W and a range of candidate scale vectors s_i:
// W' = diag(s_i) W quantized and dequantized group-wise along K with the 4-bit quantizer
// and folded back, W_hat_i = diag(s_i)^-1 Q(W'), written as the K-major bf16 operand the
// loss GEMM's TMA reads. The arithmetic and its exactness argument are described in
// k_qdq.cu.
#pragma once

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
                                           float* sWT, int tid) {
  constexpr int VEC = 16 / sizeof(T);
  constexpr int VPR = L::kCols / VEC;
  bool bad = false;
  for (int idx = tid; idx < G * VPR; idx += L::kThreads) {
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

// One G x L::kCols tile of W at rows k0 .., columns n0 .. (the tile's threads tid 0 ..
// L::kThreads - 1, `sync` a barrier over exactly those threads): with `stage` the tile is
// read into sWT (else sWT still holds it), with `reference` the plain bf16 copy of W is
// written to slot 0, and candidates c0 .. c1 - 1 (at most 64) are written to slots
// c0 + 1 .. c1. sS and sR hold (c1 - c0) rows of kSkewPitch floats, sPar (c1 - c0) x
// L::kCols parameter sets.
template <typename T, int G, typename L, typename Sync>
__device__ __forceinline__ void qdq_tile(const T* __restrict__ W, int64_t K, int64_t N, int64_t ldw, int64_t k0,
                                         int64_t n0, const float* __restrict__ S, int c0, int c1, bool stage,
                                         bool reference, __nv_bfloat16* __restrict__ Wt, int* err, int quantizer,
                                         int64_t interleave, float* sWT, float* sS, float* sR, float4* sPar,
                                         uint32_t* sRowsExact, int tid, Sync sync) {
  const int nc = c1 - c0;
  const int lane = tid & 31, warp = tid >> 5;
  const float qmax = quantizer == kQuantSym ? 14.0f : 15.0f;

  sync();  // the previous tile's readers of the shared arrays are done
  if (tid < 2) sRowsExact[tid] = 0u;
  if (stage && stage_tile<T, G, L>(W, N, ldw, k0, n0, sWT, tid)) atomicOr(err, kErrNonfiniteW);
  sync();
  for (int idx = tid; idx < nc * G; idx += L::kThreads) {
    const int c = idx / G, r = idx % G;
    const float s = S[static_cast<int64_t>(c0 + c) * K + k0 + r];
    const float rs = __frcp_rn(s);
    sS[c * L::kSkewPitch + skew(r)] = -s;
    sR[c * L::kSkewPitch + skew(r)] = rs;
    if (!(fabsf(rs) <= kScaleRecipMax && fabsf(rs) >= kScaleRecipMin)) atomicOr(&sRowsExact[c >> 5], 1u << (c & 31));
  }
  sync();

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
  if (reference && active) {
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
  if (nc <= 0) return;
  const int srow = skew(row0);  // even, and the lane's 8 rows never straddle a skew pad

  // Phase A: the group range of every (candidate, column) of the warp: W' = s W per
  // lane, then a butterfly over the RL row-lanes whose first step also splits the two
  // columns between the lanes of a pair.
  for (int c = 0; c < nc; ++c) {
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
  for (int it = lane; it < nc * L::kColsPerWarp; it += 32) {
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
  for (int c = 0; c < nc; ++c) {
    float2 s2[4];
    {
      const float2* sp = reinterpret_cast<const float2*>(sS + c * L::kSkewPitch + srow);
#pragma unroll
      for (int i = 0; i < 4; ++i) s2[i] = sp[i];
    }
    const float2* rs = reinterpret_cast<const float2*>(sR + c * L::kSkewPitch + srow);
    bool flag = (sRowsExact[c >> 5] >> (c & 31)) & 1u;
    __nv_bfloat16* const slot = dst0 + static_cast<int64_t>(c0 + c + 1) * N * K;
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
    __nv_bfloat16* const slot = dst0 + static_cast<int64_t>(c0 + c + 1) * N * K;
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

}  // namespace
}  // namespace awq
