// Arithmetic of the 2-D RoPE rotation, shared by the RoPE kernels and a host
// build used by the CPU tests (plain C++; on the host it must be compiled
// with -ffp-contract=off so that nothing is fused).
//
// The rotation (UltraGen-ar §2.ب "Scaled Positional Embeddings"): a pair
// (x0, x1) of bf16 channels turns by an angle whose cosine c and sine s are
// fp32 values:
//     y0 = x0 c - x1 s,   y1 = x0 s + x1 c
// (the transposed rotation, for gradients, uses -s).  The result is defined
// as: exact products (bf16 x fp32 fits in fp64), one fp64 subtraction /
// addition, then round to nearest even into bf16.
//
// Fast path, in fp32.  Each table value is split as c = c_hi + c_lo, c_hi
// keeping the leading 16 bits of c's significand and c_lo (at most 8
// significant bits, |c_lo| < 2^-15 |c|) the rest.  A bf16 value has 8
// significant bits, so x c_hi and x c_lo are exact in fp32, and
//     v = x0 c - x1 s = (x0 c_hi - x1 s_hi) + (x0 c_lo - x1 s_lo)
// is evaluated as y = fl(hi + lo) with hi = fma(x0, c_hi, -x1 s_hi) and
// lo = fma(x0, c_lo, -x1 s_lo), each one rounding of an exact value.  Then
// |v - y| <= 2u|y| + 2^-37 M (u = 2^-24, M the largest |x| of the chunk),
// plus far less than one fp32 ulp of y from subnormal products.  When
// |y| >= 2^-13 M and |y| >= 2^-60 that is under 3 ulp(y); if y then lies at
// least 4 ulp from every bf16 rounding midpoint, v rounds to the same bf16 as
// y, and so does the fp64 value of v (its rounding cannot reach a midpoint
// that far away).  This is Ziv's rounding test ("Fast evaluation of
// elementary mathematical functions with correctly rounded last bit", ACM
// TOMS 1991): decide the rounding from a cheap estimate when its error bound
// allows, else recompute exactly.  Chunks whose inputs reach 2^100 (or are
// not finite) are not tried, so nothing here overflows.  The test fails for
// about 2^-12 of the chunks; those take the exact fp64 route of the kernels.
#pragma once

#include <cstdint>
#include <cstring>
#include <cmath>

#if defined(__CUDACC__)
#define UG_RM_FN __host__ __device__ __forceinline__
#else
#define UG_RM_FN inline
#endif

namespace ug {
namespace rope_math {

UG_RM_FN float as_f(uint32_t u) {
#if defined(__CUDA_ARCH__)
  return __uint_as_float(u);
#else
  float f;
  std::memcpy(&f, &u, 4);
  return f;
#endif
}

UG_RM_FN uint32_t as_u(float f) {
#if defined(__CUDA_ARCH__)
  return __float_as_uint(f);
#else
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return u;
#endif
}

// The split of a table value: the leading 16 significand bits, and the rest.
UG_RM_FN float split_hi(float c) { return as_f(as_u(c) & 0xFFFFFF00u); }
UG_RM_FN float split_lo(float c) { return c - split_hi(c); }

// Two finite fp32 values rounded to nearest even into bf16, packed with lo
// in the low half.
UG_RM_FN uint32_t pack_bf16_rn(float lo, float hi) {
#if defined(__CUDA_ARCH__)
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
#else
  auto rn = [](float f) {
    const uint32_t b = as_u(f);
    return (b + 0x7FFFu + ((b >> 16) & 1u)) >> 16;
  };
  return rn(lo) | (rn(hi) << 16);
#endif
}

// Bit pattern (fp32) of the lower bound on |y|: max(2^-13 M, 2^-60), M the
// largest bf16 magnitude among the chunk's words; 0xFFFFFFFF (nothing
// decided) when M reaches 2^100 or a value is not finite.
UG_RM_FN uint32_t lower_bound(const uint32_t w[4]) {
  uint32_t m = 0;
  for (int k = 0; k < 4; ++k) {
    const uint32_t a = w[k] & 0x7FFFu, b = (w[k] >> 16) & 0x7FFFu;
    m = a > m ? a : m;
    m = b > m ? b : m;
  }
  if (m >= 0x7180u) return 0xFFFFFFFFu;  // 2^100 and above, inf, NaN
  const int32_t lb = (int32_t)(m << 16) - (13 << 23);
  return (uint32_t)(lb > 0x21800000 ? lb : 0x21800000);  // 2^-60
}

// y at least 4 ulps from the bf16 midpoint of its binade (low 16 bits
// outside [0x7FFD, 0x8004]).
UG_RM_FN bool clear_of_midpoint(float y) { return ((as_u(y) + 3u) & 0xFFF8u) != 0x8000u; }

// The cos/sin of a chunk's 4 pairs, split.
struct Angles4 {
  float ch[4], sh[4], cl[4], sl[4];
};

#if defined(__CUDA_ARCH__)
// Two pairs (words wa, wb) with packed fp32x2 arithmetic.
template <bool kTranspose>
__device__ __forceinline__ void two_pairs(uint32_t wa, uint32_t wb, float2 ch, float2 sh,
                                          float2 cl, float2 sl, float2& y0, float2& y1) {
  const float2 x0 = make_float2(__uint_as_float(wa << 16), __uint_as_float(wb << 16));
  const float2 x1 = make_float2(__uint_as_float(wa & 0xFFFF0000u),
                                __uint_as_float(wb & 0xFFFF0000u));
  const float2 nx = kTranspose ? make_float2(-x0.x, -x0.y) : make_float2(-x1.x, -x1.y);
  // y0 = x0 c - x1 s (transpose: + x1 s); y1 = x0 s + x1 c (transpose: - x0 s)
  const float2 a0 = __fmul2_rn(kTranspose ? x1 : nx, sh);
  const float2 b0 = __fmul2_rn(kTranspose ? x1 : nx, sl);
  const float2 h0 = __ffma2_rn(x0, ch, a0);
  const float2 l0 = __ffma2_rn(x0, cl, b0);
  const float2 a1 = __fmul2_rn(x1, ch);
  const float2 b1 = __fmul2_rn(x1, cl);
  const float2 h1 = __ffma2_rn(kTranspose ? nx : x0, sh, a1);
  const float2 l1 = __ffma2_rn(kTranspose ? nx : x0, sl, b1);
  y0 = __fadd2_rn(h0, l0);
  y1 = __fadd2_rn(h1, l1);
}
#endif

// Fast path for one 16-byte chunk (4 pairs, x0 in the low half of each
// word): writes the 4 rotated words to out and returns whether every output
// passed the rounding test (out is unspecified otherwise).
template <bool kTranspose>
UG_RM_FN bool chunk_fast(const uint32_t w[4], const Angles4& t, uint32_t out[4]) {
  const uint32_t lb = lower_bound(w);
  float y0[4], y1[4];
#if defined(__CUDA_ARCH__)
  for (int k = 0; k < 4; k += 2) {
    float2 a, b;
    two_pairs<kTranspose>(w[k], w[k + 1], make_float2(t.ch[k], t.ch[k + 1]),
                          make_float2(t.sh[k], t.sh[k + 1]), make_float2(t.cl[k], t.cl[k + 1]),
                          make_float2(t.sl[k], t.sl[k + 1]), a, b);
    y0[k] = a.x;
    y0[k + 1] = a.y;
    y1[k] = b.x;
    y1[k + 1] = b.y;
  }
#else
  for (int k = 0; k < 4; ++k) {
    const float x0 = as_f(w[k] << 16), x1 = as_f(w[k] & 0xFFFF0000u);
    const float sgn = kTranspose ? -1.0f : 1.0f;
    // y0 = x0 c - sgn x1 s; y1 = sgn x0 s + x1 c (each product exact)
    const float h0 = std::fma(x0, t.ch[k], -sgn * x1 * t.sh[k]);
    const float l0 = std::fma(x0, t.cl[k], -sgn * x1 * t.sl[k]);
    const float h1 = std::fma(sgn * x0, t.sh[k], x1 * t.ch[k]);
    const float l1 = std::fma(sgn * x0, t.sl[k], x1 * t.cl[k]);
    y0[k] = h0 + l0;
    y1[k] = h1 + l1;
  }
#endif
  // every |y| >= lb (one comparison of the chunk's smallest |y|: no output
  // of a chunk that passed lower_bound is infinite or NaN), and every y
  // clear of its midpoint
  float amin = std::fabs(y0[0]);
  bool ok = true;
  for (int k = 0; k < 4; ++k) {
    amin = std::fmin(amin, std::fmin(std::fabs(y0[k]), std::fabs(y1[k])));
    ok = ok & clear_of_midpoint(y0[k]) & clear_of_midpoint(y1[k]);
    out[k] = pack_bf16_rn(y0[k], y1[k]);
  }
  return ok & (as_u(amin) >= lb);
}

}  // namespace rope_math
}  // namespace ug
