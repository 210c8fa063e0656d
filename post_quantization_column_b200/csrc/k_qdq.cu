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
#include "qdq_tile.cuh"

namespace awq {
namespace {

struct CtaSync {
  __device__ __forceinline__ void operator()() const { __syncthreads(); }
};

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
  qdq_tile<T, G, L>(W, K, N, ldw, k0, n0, S, 0, n_grid, true, true, Wt, err, quantizer, interleave, sWT, sS, sR, sPar,
                    sRowsExact, static_cast<int>(threadIdx.x), CtaSync{});
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
