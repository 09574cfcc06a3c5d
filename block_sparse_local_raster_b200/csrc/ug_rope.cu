// 2-D axial RoPE with rho-scaled low-res positions (UltraGen-ar §2.ب
// "Scaled Positional Embeddings"; UltraGen-fr §2.B; UltraGen-es §2), alone and
// fused into the window-first permutation (UltraGen-fr §2.A).
//
// Per token: position (row, col) from its token set -- high-res raster,
// high-res window-first, or low-res (whose table rows were built at rho*i,
// rho*j).  Channels [0, a_y) rotate with the row, [a_y, d) with the column;
// pair (2k, 2k+1) of a segment turns by pos * theta^(-2k/a).  Arithmetic is
// reproducible bit for bit: the result is the bf16 (round to nearest even)
// of the fp64 value formed from exact bf16 x fp32 products by one fp64
// subtraction or addition.  It is computed by the fp32 fast path of
// ug_rope_math.h (error-free products and a rounding test), and for the rare
// chunk whose rounding that test cannot decide, by the exact fp64 route:
// exact fp64 products, one fp64 rounding (no contraction), and a correctly
// rounded fp64 -> bf16 conversion (round to odd into fp32, then round to
// nearest even: Boldo & Melquiond, "Emulation of FMA and correctly rounded
// sums: proved algorithms using rounding to odd", IEEE Trans. Computers
// 2008).
//
// The backward pass rotates gradients by the transposed rotation: the same
// c, s with s negated (exact), so it is reproducible in the same way.
//
// HBM-bound in principle: 2 bytes moved per byte of tensor.  The fast path
// keeps the arithmetic near 100 instructions per 16-byte chunk (packed fp32x2
// products of split table values, one rounding test per chunk), and each
// thread keeps several 16-byte loads in flight before it computes.
#include <cstdint>

#include <cuda_bf16.h>

#include "ug_debug.h"
#include "ug_internal.h"
#include "ug_rope_math.h"

namespace ug {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 6;  // 16-byte chunks in flight per thread (4: 153 us, 6: 149 us per 4K tensor)

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

// Exact route for one channel pair (x0 in the low half of xw):
// (x0 c - x1 s, x0 s + x1 c) from exact fp64 products.
__device__ __noinline__ uint32_t rotate_pair_exact(uint32_t xw, float cf, float sf) {
  const double c = (double)cf, s = (double)sf;
  const double x0 = (double)__uint_as_float(xw << 16);
  const double x1 = (double)__uint_as_float(xw & 0xFFFF0000u);
  const double y0 = __dsub_rn(__dmul_rn(x0, c), __dmul_rn(x1, s));
  const double y1 = __dadd_rn(__dmul_rn(x0, s), __dmul_rn(x1, c));
  const __nv_bfloat162 r = __floats2bfloat162_rn(to_odd_f32(y0), to_odd_f32(y1));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// The split cos/sin of chunk k (8 channels, 4 pairs) inside a head: row
// axis for k < ay_chunks, column axis after.  r / c point at the row's and
// the column's table rows ([pair] of each of the four tables); rows are
// 16-byte aligned.
struct AxisRow {
  const float *ch, *sh, *cl, *sl;
};

__device__ __forceinline__ AxisRow axis_row(const float* t, const AxisTables& a, int64_t coord,
                                            int m) {
  const int64_t o = coord * m;
  return AxisRow{t + a.cos_hi + o, t + a.sin_hi + o, t + a.cos_lo + o, t + a.sin_lo + o};
}

__device__ __forceinline__ rope_math::Angles4 chunk_angles(int k, int ay_chunks,
                                                           const AxisRow& r, const AxisRow& c) {
  const bool ax_row = k < ay_chunks;
  const int off = ax_row ? k * 4 : (k - ay_chunks) * 4;
  const AxisRow& x = ax_row ? r : c;
  rope_math::Angles4 t;
  *reinterpret_cast<float4*>(t.ch) = __ldg(reinterpret_cast<const float4*>(x.ch + off));
  *reinterpret_cast<float4*>(t.sh) = __ldg(reinterpret_cast<const float4*>(x.sh + off));
  *reinterpret_cast<float4*>(t.cl) = __ldg(reinterpret_cast<const float4*>(x.cl + off));
  *reinterpret_cast<float4*>(t.sl) = __ldg(reinterpret_cast<const float4*>(x.sl + off));
  return t;
}

// Rotates one 16-byte chunk (4 channel pairs): the fp32 fast path, or for
// the rare chunk it cannot decide, the exact route pair by pair.
template <bool kTranspose>
__device__ __forceinline__ uint4 rotate_chunk(uint4 v, const rope_math::Angles4& t) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[4];
  if (!rope_math::chunk_fast<kTranspose>(w, t, o)) {
    for (int k = 0; k < 4; ++k) {
      const float c = t.ch[k] + t.cl[k], s = t.sh[k] + t.sl[k];  // exact
      o[k] = rotate_pair_exact(w[k], c, kTranspose ? -s : s);
    }
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

enum RowMode { kSetRows = 0, kPermuteRows = 1, kUnpermuteRows = 2 };

struct RopeArgs {
  const uint4* x;
  uint4* y;
  const float* tables;  // the plan's table buffer
  AxisTables row, col;  // the token set's row-axis and column-axis tables
  int64_t n_rows;       // batch * tokens
  int32_t n_tok;        // tokens per batch element
  int32_t row_chunks;   // heads * head_dim / 8
  int32_t head_chunks;  // head_dim / 8
  int32_t ay_chunks;    // a_y / 8
  int32_t my, mx;       // a_y / 2, a_x / 2
  int32_t set;          // kSetRows: ug_token_set
  int32_t grid_w, win_h, win_w, nwx, T, lr_w;
  int32_t text_len;         // UG_LR: leading text rows, copied unrotated
  int32_t rows_r, rows_c;   // coordinates in the row / column tables (debug checks)
  int* err;                 // the plan's error word
};

// One warp per token row, the three uses sharing it:
//   kSetRows        y[b, t] = R x[b, t] for the tokens of one set (high-res
//                   raster or window-first, or the global set: text rows
//                   copied, low-res rows at rho-scaled positions);
//   kPermuteRows    y[b, perm(r)] = R x[b, r]: the window-first permutation
//                   with RoPE applied on the way, over raster tokens r;
//   kUnpermuteRows  y[b, r] = R^T x[b, perm(r)]: its inverse for gradients.
// A token row (heads * head_dim * 2 bytes) is contiguous in every order, so
// each warp reads and writes whole rows, lanes on consecutive 16-byte chunks
// with kUnroll in flight each; the table rows of the token's position come
// from L1.
template <int HEAD_CHUNKS, int MODE, bool kTranspose>  // HEAD_CHUNKS 8, 16, or 0 = from args
__global__ void __launch_bounds__(kThreads, 3) rope_rows_kernel(const RopeArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * kThreads) >> 5;
  const int hc = HEAD_CHUNKS ? HEAD_CHUNKS : a.head_chunks;
  for (int64_t row = warp0; row < a.n_rows; row += nwarps) {
    const int64_t b = row / a.n_tok;
    const int32_t t = (int32_t)(row - b * a.n_tok);
    int32_t pr, pc;      // grid row / column of the token
    int64_t src = row, dst = row;
    if (MODE == kSetRows) {
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
    } else {
      // t is a raster token; its window-first index
      pr = t / a.grid_w;
      pc = t - pr * a.grid_w;
      const int32_t wy = pr / a.win_h, ly = pr - wy * a.win_h;
      const int32_t wx = pc / a.win_w, lx = pc - wx * a.win_w;
      const int64_t p = ((int64_t)wy * a.nwx + wx) * a.T + (int64_t)ly * a.win_w + lx;
      if (MODE == kPermuteRows)
        dst = b * a.n_tok + p;
      else
        src = b * a.n_tok + p;
      if (!dbg_ok(p >= 0 && p < a.n_tok, a.err)) continue;
    }
    if (!dbg_ok(pr >= 0 && pr < a.rows_r && pc >= 0 && pc < a.rows_c, a.err)) continue;
    const uint4* __restrict__ xs = a.x + src * a.row_chunks;
    uint4* __restrict__ ys = a.y + dst * a.row_chunks;
    const AxisRow rr = axis_row(a.tables, a.row, pr, a.my);
    const AxisRow cc = axis_row(a.tables, a.col, pc, a.mx);
    // A lane meets chunks lane, lane + 32, ...: when the head's chunk count
    // divides 32 they all sit at the same place in their head, so the lane's
    // angles are loaded once per row.
    constexpr bool kFixed = HEAD_CHUNKS != 0 && 32 % (HEAD_CHUNKS ? HEAD_CHUNKS : 1) == 0;
    rope_math::Angles4 fixed;
    if (kFixed) fixed = chunk_angles(lane % hc, a.ay_chunks, rr, cc);
    for (int32_t c0 = lane; c0 < a.row_chunks; c0 += 32 * kUnroll) {
      uint4 v[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int32_t c = c0 + 32 * u;
        if (c < a.row_chunks) v[u] = __ldcs(xs + c);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int32_t c = c0 + 32 * u;
        if (c < a.row_chunks)
          ys[c] = rotate_chunk<kTranspose>(
              v[u], kFixed ? fixed : chunk_angles(c % hc, a.ay_chunks, rr, cc));
      }
    }
  }
}

int grid_for(const ug_plan* p, int64_t want) {
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, p->device);
  return (int)std::min<int64_t>(want, (int64_t)sms * (2048 / kThreads) * 4);
}

template <int MODE, bool kTranspose>
void launch_rows(const RopeArgs& a, int blocks, cudaStream_t st) {
  if (a.head_chunks == 16)
    rope_rows_kernel<16, MODE, kTranspose><<<blocks, kThreads, 0, st>>>(a);
  else if (a.head_chunks == 8)
    rope_rows_kernel<8, MODE, kTranspose><<<blocks, kThreads, 0, st>>>(a);
  else
    rope_rows_kernel<0, MODE, kTranspose><<<blocks, kThreads, 0, st>>>(a);
}

void common_args(const ug_plan* p, RopeArgs& a) {
  a.tables = p->d_rope;
  a.head_chunks = p->g.head_dim / 8;
  a.row_chunks = p->g.heads * a.head_chunks;
  a.ay_chunks = p->g.rope_dim_y / 8;
  a.my = p->g.rope_dim_y / 2;
  a.mx = p->g.rope_dim_x / 2;
  a.grid_w = p->g.grid_w;
  a.win_h = p->g.win_h;
  a.win_w = p->g.win_w;
  a.nwx = p->nwx;
  a.T = (int32_t)p->T;
  a.lr_w = p->g.lr_w;
  a.text_len = p->g.text_len;
  a.err = p->d_err;
}

}  // namespace

int launch_rope(const ug_plan* p, const void* x, void* y, int set, cudaStream_t st,
                bool transpose) {
  RopeArgs a;
  common_args(p, a);
  a.x = static_cast<const uint4*>(x);
  a.y = static_cast<uint4*>(y);
  const bool lr = set == UG_LR;
  a.row = lr ? p->rope.lr_y : p->rope.hr_y;
  a.col = lr ? p->rope.lr_x : p->rope.hr_x;
  a.n_tok = (int32_t)(lr ? p->L : p->N);
  a.n_rows = (int64_t)p->g.batch * a.n_tok;
  a.set = set;
  a.rows_r = lr ? p->g.lr_h : p->g.grid_h;
  a.rows_c = lr ? p->g.lr_w : p->g.grid_w;
  if (a.n_rows == 0) return UG_OK;
  const int blocks = grid_for(p, (a.n_rows + (kThreads / 32) - 1) / (kThreads / 32));
  if (transpose)
    launch_rows<kSetRows, true>(a, blocks, st);
  else
    launch_rows<kSetRows, false>(a, blocks, st);
  return cudaGetLastError() == cudaSuccess ? UG_OK : UG_ERR_CUDA;
}

int launch_permute_rope(const ug_plan* p, const void* src, void* dst, cudaStream_t st,
                        bool inverse) {
  RopeArgs a;
  common_args(p, a);
  a.x = static_cast<const uint4*>(src);
  a.y = static_cast<uint4*>(dst);
  a.row = p->rope.hr_y;
  a.col = p->rope.hr_x;
  a.n_tok = (int32_t)p->N;
  a.n_rows = (int64_t)p->g.batch * a.n_tok;
  a.set = UG_HR_RASTER;
  a.rows_r = p->g.grid_h;
  a.rows_c = p->g.grid_w;
  const int blocks = grid_for(p, (a.n_rows + (kThreads / 32) - 1) / (kThreads / 32));
  if (inverse)
    launch_rows<kUnpermuteRows, true>(a, blocks, st);
  else
    launch_rows<kPermuteRows, false>(a, blocks, st);
  return cudaGetLastError() == cudaSuccess ? UG_OK : UG_ERR_CUDA;
}

// The RoPE kernels need no per-device set-up (static shared memory only).
int prepare_rope(int) { return UG_OK; }

}  // namespace ug
