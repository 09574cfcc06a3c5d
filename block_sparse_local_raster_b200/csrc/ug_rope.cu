// 2-D axial RoPE with rho-scaled low-res positions (UltraGen-ar §2.ب
// "Scaled Positional Embeddings"; UltraGen-fr §2.B; UltraGen-es §2), alone and
// fused into the window-first permutation (UltraGen-fr §2.A).
//
// Per token: position (row, col) from its token set -- high-res raster,
// high-res window-first, or low-res (whose table rows were built at rho*i,
// rho*j).  Channels [0, a_y) rotate with the row, [a_y, d) with the column;
// pair (2k, 2k+1) of a segment turns by pos * theta^(-2k/a).  Arithmetic is
// reproducible bit for bit: bf16 x fp32 products are exact in fp64 (the
// tables hold the fp32-rounded cos/sin as fp64), their sum is one fp64
// rounding (no contraction), and the fp64 -> bf16 conversion is correctly
// rounded (round to odd into fp32, then round to nearest even, the method of
// Boldo & Melquiond, "Emulation of FMA and correctly rounded sums: proved
// algorithms using rounding to odd", IEEE Trans. Computers 2008).
//
// The backward pass rotates gradients by the transposed rotation: the same
// c, s with s negated (exact), so it is reproducible in the same way.
//
// HBM-bound: 2 bytes moved per byte of tensor.  The rotation keeps the
// fp32 <-> fp64 conversions (the slowest part of the arithmetic) to 4 per
// channel pair.
#include <cstdint>

#include <cuda_bf16.h>

#include "ug_internal.h"

namespace ug {
namespace {

constexpr int kThreads = 256;

// fp64 -> fp32 rounded to odd: truncate, then set the last bit if anything
// was dropped.  For results in fp32's normal range the dropped part is the
// low 29 bits of the fp64 significand; elsewhere compare exactly.
__device__ __forceinline__ float to_odd_f32(double v) {
  const float f = __double2float_rz(v);
  uint32_t u = __float_as_uint(f);
  const uint64_t b = (uint64_t)__double_as_longlong(v);
  const uint32_t e = (uint32_t)(b >> 52) & 0x7FFu;
  bool inexact;
  if (e >= 1023u - 126u && e <= 1023u + 127u)
    inexact = ((uint32_t)b & 0x1FFFFFFFu) != 0u;
  else
    inexact = (double)f != v;
  if (inexact) u |= 1u;
  return __uint_as_float(u);
}

// One channel pair (x0 in the low half of xw): (x0 c - x1 s, x0 s + x1 c).
__device__ __forceinline__ uint32_t rotate_pair(uint32_t xw, double c, double s) {
  const double x0 = (double)__uint_as_float(xw << 16);
  const double x1 = (double)__uint_as_float(xw & 0xFFFF0000u);
  const double y0 = __dsub_rn(__dmul_rn(x0, c), __dmul_rn(x1, s));
  const double y1 = __dadd_rn(__dmul_rn(x0, s), __dmul_rn(x1, c));
  const __nv_bfloat162 r = __floats2bfloat162_rn(to_odd_f32(y0), to_odd_f32(y1));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// Rotates one 16-byte chunk (4 channel pairs) with the table rows of its
// position.  k: chunk index inside the head (8 channels per chunk).  sgn is
// +1 (rotation) or -1 (its transpose).
__device__ __forceinline__ uint4 rotate_chunk(uint4 v, int k, int ay_chunks, const double* cr,
                                              const double* sr, const double* cc,
                                              const double* sc, double sgn) {
  const bool ax_row = k < ay_chunks;
  const double* cp = ax_row ? cr + k * 4 : cc + (k - ay_chunks) * 4;
  const double* sp = ax_row ? sr + k * 4 : sc + (k - ay_chunks) * 4;
  const double2 c01 = __ldg(reinterpret_cast<const double2*>(cp));
  const double2 c23 = __ldg(reinterpret_cast<const double2*>(cp) + 1);
  const double2 s01 = __ldg(reinterpret_cast<const double2*>(sp));
  const double2 s23 = __ldg(reinterpret_cast<const double2*>(sp) + 1);
  uint4 o;
  o.x = rotate_pair(v.x, c01.x, sgn * s01.x);
  o.y = rotate_pair(v.y, c01.y, sgn * s01.y);
  o.z = rotate_pair(v.z, c23.x, sgn * s23.x);
  o.w = rotate_pair(v.w, c23.y, sgn * s23.y);
  return o;
}

struct RopeArgs {
  const uint4* x;
  uint4* y;
  const double* cos_r;  // row-axis table, [coord][a_y/2]
  const double* sin_r;
  const double* cos_c;  // column-axis table, [coord][a_x/2]
  const double* sin_c;
  int64_t n_rows;      // batch * tokens
  int32_t n_tok;       // tokens per batch element
  int32_t row_chunks;  // heads * head_dim / 8
  int32_t head_chunks; // head_dim / 8
  int32_t ay_chunks;   // a_y / 8
  int32_t my, mx;      // a_y / 2, a_x / 2
  int32_t set;         // ug_token_set
  int32_t grid_w, win_h, win_w, nwx, T, lr_w;
  int32_t text_len;    // UG_LR: leading text rows, copied unrotated
  double sgn;          // +1 rotation, -1 its transpose (backward)
};

// One warp per token row: lanes walk the row's 16-byte chunks (coalesced);
// the cos/sin rows come from L1.
template <int HEAD_CHUNKS>  // 8, 16, or 0 = read from args
__global__ void __launch_bounds__(kThreads) rope_kernel(const RopeArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * kThreads) >> 5;
  const int hc = HEAD_CHUNKS ? HEAD_CHUNKS : a.head_chunks;
  for (int64_t row = warp0; row < a.n_rows; row += nwarps) {
    const int32_t t = (int32_t)(row % a.n_tok);
    int32_t pr, pc;  // grid row / column of the token
    if (a.set == UG_LR) {
      if (t < a.text_len) {  // text token: no grid position, no rotation
        const uint4* __restrict__ xs = a.x + row * a.row_chunks;
        uint4* __restrict__ ys = a.y + row * a.row_chunks;
        for (int32_t c = lane; c < a.row_chunks; c += 32) ys[c] = xs[c];
        continue;
      }
      pr = (t - a.text_len) / a.lr_w;
      pc = (t - a.text_len) - pr * a.lr_w;
    } else if (a.set == UG_HR_RASTER) {
      pr = t / a.grid_w;
      pc = t - pr * a.grid_w;
    } else {
      const int32_t w = t / a.T, l = t - (t / a.T) * a.T;
      const int32_t wy = w / a.nwx, wx = w - wy * a.nwx;
      const int32_t ly = l / a.win_w, lx = l - ly * a.win_w;
      pr = wy * a.win_h + ly;
      pc = wx * a.win_w + lx;
    }
    const double* cr = a.cos_r + (int64_t)pr * a.my;
    const double* sr = a.sin_r + (int64_t)pr * a.my;
    const double* cc = a.cos_c + (int64_t)pc * a.mx;
    const double* sc = a.sin_c + (int64_t)pc * a.mx;
    const uint4* __restrict__ xs = a.x + row * a.row_chunks;
    uint4* __restrict__ ys = a.y + row * a.row_chunks;
    for (int32_t c = lane; c < a.row_chunks; c += 32)
      ys[c] = rotate_chunk(xs[c], c % hc, a.ay_chunks, cr, sr, cc, sc, a.sgn);
  }
}

// Window-first permutation with the RoPE of each token applied on the way:
// dst[b, perm[r]] = rope(src[b, r]) at the token's grid position.  Equal bit
// for bit to the permutation followed by ug_rope_2d on the window-first set
// (the rotation depends on the token's position only), in one pass over HBM.
// A CTA copies whole window-row segments (win_w tokens, contiguous in both
// orders), so the row position is fixed per segment.
struct PermuteRopeArgs {
  const uint4* src;
  uint4* dst;
  const double* cos_r;
  const double* sin_r;
  const double* cos_c;
  const double* sin_c;
  int64_t n_seg;
  int64_t n_tok;
  int32_t row_chunks, head_chunks, ay_chunks, my, mx;
  int32_t grid_h, grid_w, win_h, win_w, nwx, T;
  bool inverse;  // false: raster -> window-first, rotated; true: window-first -> raster, transposed
};

template <int HEAD_CHUNKS>
__global__ void __launch_bounds__(kThreads) permute_rope_kernel(const PermuteRopeArgs a) {
  const int hc = HEAD_CHUNKS ? HEAD_CHUNKS : a.head_chunks;
  for (int64_t seg = blockIdx.x; seg < a.n_seg; seg += gridDim.x) {
    const int64_t per_b = (int64_t)a.grid_h * a.nwx;
    const int64_t b = seg / per_b;
    const int32_t rem = (int32_t)(seg - b * per_b);
    const int32_t y = rem / a.nwx, wx = rem - (rem / a.nwx) * a.nwx;
    const int32_t wy = y / a.win_h, ly = y - wy * a.win_h;
    const int64_t r0 = (int64_t)y * a.grid_w + (int64_t)wx * a.win_w;
    const int64_t p0 = ((int64_t)wy * a.nwx + wx) * a.T + (int64_t)ly * a.win_w;
    const uint4* __restrict__ s = a.src + (b * a.n_tok + (a.inverse ? p0 : r0)) * a.row_chunks;
    uint4* __restrict__ d = a.dst + (b * a.n_tok + (a.inverse ? r0 : p0)) * a.row_chunks;
    const double sgn = a.inverse ? -1.0 : 1.0;
    const double* cr = a.cos_r + (int64_t)y * a.my;
    const double* sr = a.sin_r + (int64_t)y * a.my;
#pragma unroll 4
    for (int32_t tl = 0; tl < a.win_w; ++tl) {  // token inside the segment
      const int32_t x = wx * a.win_w + tl;      // its grid column
      const double* cc = a.cos_c + (int64_t)x * a.mx;
      const double* sc = a.sin_c + (int64_t)x * a.mx;
      for (int32_t rc = threadIdx.x; rc < a.row_chunks; rc += kThreads)
        d[tl * a.row_chunks + rc] =
            rotate_chunk(__ldcs(s + tl * a.row_chunks + rc), rc % hc, a.ay_chunks, cr, sr, cc, sc,
                         sgn);
    }
  }
}

int grid_for(const ug_plan* p, int64_t want) {
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, p->device);
  return (int)std::min<int64_t>(want, (int64_t)sms * (2048 / kThreads) * 4);
}

}  // namespace

int launch_rope(const ug_plan* p, const void* x, void* y, int set, cudaStream_t st,
                bool transpose) {
  RopeArgs a;
  a.sgn = transpose ? -1.0 : 1.0;
  a.x = static_cast<const uint4*>(x);
  a.y = static_cast<uint4*>(y);
  const bool lr = set == UG_LR;
  const double* t = p->d_rope;
  a.cos_r = t + (lr ? p->rope.lr_y_cos : p->rope.hr_y_cos);
  a.sin_r = t + (lr ? p->rope.lr_y_sin : p->rope.hr_y_sin);
  a.cos_c = t + (lr ? p->rope.lr_x_cos : p->rope.hr_x_cos);
  a.sin_c = t + (lr ? p->rope.lr_x_sin : p->rope.hr_x_sin);
  a.n_tok = (int32_t)(lr ? p->L : p->N);
  a.n_rows = (int64_t)p->g.batch * a.n_tok;
  a.head_chunks = p->g.head_dim / 8;
  a.row_chunks = p->g.heads * a.head_chunks;
  a.ay_chunks = p->g.rope_dim_y / 8;
  a.my = p->g.rope_dim_y / 2;
  a.mx = p->g.rope_dim_x / 2;
  a.set = set;
  a.grid_w = p->g.grid_w;
  a.win_h = p->g.win_h;
  a.win_w = p->g.win_w;
  a.nwx = p->nwx;
  a.T = (int32_t)p->T;
  a.lr_w = p->g.lr_w;
  a.text_len = p->g.text_len;
  if (a.n_rows == 0) return UG_OK;
  const int blocks = grid_for(p, (a.n_rows + (kThreads / 32) - 1) / (kThreads / 32));
  if (a.head_chunks == 16)
    rope_kernel<16><<<blocks, kThreads, 0, st>>>(a);
  else if (a.head_chunks == 8)
    rope_kernel<8><<<blocks, kThreads, 0, st>>>(a);
  else
    rope_kernel<0><<<blocks, kThreads, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? UG_OK : UG_ERR_CUDA;
}

int launch_permute_rope(const ug_plan* p, const void* src, void* dst, cudaStream_t st,
                        bool inverse) {
  PermuteRopeArgs a;
  a.inverse = inverse;
  a.src = static_cast<const uint4*>(src);
  a.dst = static_cast<uint4*>(dst);
  const double* t = p->d_rope;
  a.cos_r = t + p->rope.hr_y_cos;
  a.sin_r = t + p->rope.hr_y_sin;
  a.cos_c = t + p->rope.hr_x_cos;
  a.sin_c = t + p->rope.hr_x_sin;
  a.n_tok = p->N;
  a.head_chunks = p->g.head_dim / 8;
  a.row_chunks = p->g.heads * a.head_chunks;
  a.ay_chunks = p->g.rope_dim_y / 8;
  a.my = p->g.rope_dim_y / 2;
  a.mx = p->g.rope_dim_x / 2;
  a.grid_h = p->g.grid_h;
  a.grid_w = p->g.grid_w;
  a.win_h = p->g.win_h;
  a.win_w = p->g.win_w;
  a.nwx = p->nwx;
  a.T = (int32_t)p->T;
  a.n_seg = (int64_t)p->g.batch * p->g.grid_h * p->nwx;
  const int blocks = grid_for(p, a.n_seg);
  if (a.head_chunks == 16)
    permute_rope_kernel<16><<<blocks, kThreads, 0, st>>>(a);
  else if (a.head_chunks == 8)
    permute_rope_kernel<8><<<blocks, kThreads, 0, st>>>(a);
  else
    permute_rope_kernel<0><<<blocks, kThreads, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? UG_OK : UG_ERR_CUDA;
}

}  // namespace ug
