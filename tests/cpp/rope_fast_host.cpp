// Host build of the RoPE kernels' fp32 fast path (ug_rope_math.h), exported
// for tests/test_rope_fast_path.py.  Compile with -ffp-contract=off.
#include <cstdint>

#include "ug_rope_math.h"

// n chunks of 4 words; per word k of chunk i the fp32 cos c[4i+k] and sin
// s[4i+k], split as the plan's tables are.  ok[i]: the fast path decided.
extern "C" void rope_chunks_fast(const uint32_t* w, const float* c, const float* s, int transpose,
                                 uint32_t* out, uint8_t* ok, int64_t n) {
  using namespace ug::rope_math;
  for (int64_t i = 0; i < n; ++i) {
    Angles4 t;
    for (int k = 0; k < 4; ++k) {
      t.ch[k] = split_hi(c[4 * i + k]);
      t.cl[k] = split_lo(c[4 * i + k]);
      t.sh[k] = split_hi(s[4 * i + k]);
      t.sl[k] = split_lo(s[4 * i + k]);
    }
    ok[i] = transpose ? chunk_fast<true>(w + 4 * i, t, out + 4 * i)
                      : chunk_fast<false>(w + 4 * i, t, out + 4 * i);
  }
}

// The split itself: hi keeps the leading 16 significand bits, hi + lo == c.
extern "C" void rope_split(const float* c, float* hi, float* lo, int64_t n) {
  for (int64_t i = 0; i < n; ++i) {
    hi[i] = ug::rope_math::split_hi(c[i]);
    lo[i] = ug::rope_math::split_lo(c[i]);
  }
}
