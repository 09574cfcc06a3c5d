// 2-D axial RoPE with rho-scaled low-res positions (UltraGen-ar §2.ب
// "Scaled Positional Embeddings"; UltraGen-fr §2.B; UltraGen-es §2).
//
// Per token: position (row, col) from its token set -- high-res raster,
// high-res window-first, or low-res (whose table rows were built at rho*i,
// rho*j).  Channels [0, a_y) rotate with the row, [a_y, d) with the column;
// pair (2k, 2k+1) of a segment turns by pos * theta^(-2k/a).  Arithmetic is
// reproducible bit for bit: bf16 x fp32 products are exact in fp64, their sum
// is one fp64 rounding (no contraction), and the fp64 -> bf16 conversion is
// correctly rounded (round to odd into fp32, then round to nearest even, the
// method of Boldo & Melquiond, "Emulation of FMA and correctly rounded sums:
// proved algorithms using rounding to odd", IEEE Trans. Computers 2008).
//
// One warp per token row: lanes walk the row's 16-byte chunks (8 channels =
// 4 pairs), so loads and stores are coalesced; the cos/sin rows (<= 256 B per
// axis) come from L1.  HBM-bound: 2 bytes moved per byte of tensor.
#include <cstdint>

#include <cuda_bf16.h>

#include "ug_internal.h"

namespace ug {
namespace {

constexpr int kThreads = 256;

struct RopeArgs {
  const uint4* x;
  uint4* y;
  const float* cos_r;  // row-axis table, [coord][a_y/2]
  const float* sin_r;
  const float* cos_c;  // column-axis table, [coord][a_x/2]
  const float* sin_c;
  int64_t n_rows;      // batch * tokens
  int32_t n_tok;       // tokens per batch element
  int32_t row_chunks;  // heads * head_dim / 8
  int32_t head_chunks; // head_dim / 8
  int32_t ay_chunks;   // a_y / 8
  int32_t my, mx;      // a_y / 2, a_x / 2
  int32_t set;         // ug_token_set
  int32_t grid_w, win_h, win_w, nwx, T, lr_w;
};

// fp64 -> bf16, round to nearest even, via round-to-odd into fp32.
__device__ __forceinline__ float to_odd_f32(double v) {
  const float f = __double2float_rz(v);
  uint32_t u = __float_as_uint(f);
  if ((double)f != v) u |= 1u;
  return __uint_as_float(u);
}

__device__ __forceinline__ uint32_t rotate_pair(uint32_t xw, float c, float s) {
  const double x0 = (double)__uint_as_float(xw << 16);
  const double x1 = (double)__uint_as_float(xw & 0xFFFF0000u);
  const double dc = (double)c, ds = (double)s;
  const double y0 = __dsub_rn(__dmul_rn(x0, dc), __dmul_rn(x1, ds));
  const double y1 = __dadd_rn(__dmul_rn(x0, ds), __dmul_rn(x1, dc));
  const __nv_bfloat162 r = __floats2bfloat162_rn(to_odd_f32(y0), to_odd_f32(y1));
  return *reinterpret_cast<const uint32_t*>(&r);
}

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
      pr = t / a.lr_w;
      pc = t - pr * a.lr_w;
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
    const float* cr = a.cos_r + (int64_t)pr * a.my;
    const float* sr = a.sin_r + (int64_t)pr * a.my;
    const float* cc = a.cos_c + (int64_t)pc * a.mx;
    const float* sc = a.sin_c + (int64_t)pc * a.mx;
    const uint4* __restrict__ xs = a.x + row * a.row_chunks;
    uint4* __restrict__ ys = a.y + row * a.row_chunks;
    for (int32_t c = lane; c < a.row_chunks; c += 32) {
      const int32_t k = c % hc;  // chunk inside the head
      const uint4 v = xs[c];
      const bool ax_row = k < a.ay_chunks;
      const float* cp = ax_row ? cr + k * 4 : cc + (k - a.ay_chunks) * 4;
      const float* sp = ax_row ? sr + k * 4 : sc + (k - a.ay_chunks) * 4;
      const float4 c4 = __ldg(reinterpret_cast<const float4*>(cp));
      const float4 s4 = __ldg(reinterpret_cast<const float4*>(sp));
      uint4 o;
      o.x = rotate_pair(v.x, c4.x, s4.x);
      o.y = rotate_pair(v.y, c4.y, s4.y);
      o.z = rotate_pair(v.z, c4.z, s4.z);
      o.w = rotate_pair(v.w, c4.w, s4.w);
      ys[c] = o;
    }
  }
}

}  // namespace

int launch_rope(const ug_plan* p, const void* x, void* y, int set, cudaStream_t st) {
  RopeArgs a;
  a.x = static_cast<const uint4*>(x);
  a.y = static_cast<uint4*>(y);
  const bool lr = set == UG_LR;
  const float* t = p->d_rope;
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
  if (a.n_rows == 0) return UG_OK;
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, p->device);
  const int64_t want = (a.n_rows + (kThreads / 32) - 1) / (kThreads / 32);
  const int64_t blocks = std::min<int64_t>(want, (int64_t)sms * (2048 / kThreads) * 4);
  if (a.head_chunks == 16)
    rope_kernel<16><<<(unsigned)blocks, kThreads, 0, st>>>(a);
  else if (a.head_chunks == 8)
    rope_kernel<8><<<(unsigned)blocks, kThreads, 0, st>>>(a);
  else
    rope_kernel<0><<<(unsigned)blocks, kThreads, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? UG_OK : UG_ERR_CUDA;
}

}  // namespace ug
