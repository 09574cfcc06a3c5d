// Warm-start initialisation of the high-res state (UltraGen-ar §2.د
// "Warm-Start Initialization"; UltraGen-fr §2.D): the low-res latent is
// upsampled by an integer factor, sharpened, and blended with Gaussian noise
// at timestep t:
//   u   = bilinear(x_lr) at ((y + 0.5) / s - 0.5, (x + 0.5) / s - 0.5),
//         indices clamped to the low-res image;
//   x0  = u + amount * (u - blur(u)), blur = (1/4, 1/2, 1/4) in each
//         direction with edges replicated (unsharp mask);
//   out = (1 - t) * x0 + t * noise.
//
// HBM-bound: per high-res pixel one fp32 noise read and one fp32 write; the
// low-res image (1/s^2 of that) is read through L1.  A CTA owns a 32 x 128
// output tile of one plane: it evaluates u on the tile plus a one-pixel halo
// into shared memory (rows and columns clamped at the image border, which is
// the edge replication of the blur), then each thread blurs, sharpens and
// blends 4 x 4 pixels, streaming noise in and the result out as float4.
#include <cstdint>

#include "ug_internal.h"

namespace ug {
namespace {

constexpr int kTileH = 32;
constexpr int kTileW = 128;
constexpr int kThreads = 256;  // 32 x 8: a thread owns 4 columns x 4 rows
constexpr int kUH = kTileH + 2;
constexpr int kUW = kTileW + 2;
constexpr int kUStride = kUW + 2;

struct WarmArgs {
  const float* x_lr;
  const float* noise;
  float* out;
  int32_t h, w;     // low-res size
  int32_t H, W;     // high-res size
  int32_t s;        // upsampling factor
  float amount, t;
};

// Source coordinate of high-res index d along an axis of n low-res samples:
// (d + 0.5) / s - 0.5 = (2d + 1 - s) / (2s).  The integer part and the
// fraction are taken from the exact integer numerator.
__device__ __forceinline__ void taps(int d, int s, int n, int& i0, int& i1, float& f) {
  const int num = 2 * d + 1 - s, den = 2 * s;
  const int fl = num >= 0 ? num / den : -((-num + den - 1) / den);
  f = (float)(num - fl * den) / (float)den;
  i0 = min(max(fl, 0), n - 1);
  i1 = min(max(fl + 1, 0), n - 1);
}

template <bool VEC>
__global__ void __launch_bounds__(kThreads) warm_start_kernel(const WarmArgs a) {
  __shared__ float u[kUH][kUStride];
  // The low-res samples the tile reads.  Tap indices grow with the output
  // coordinate and span at most one more sample than the tile has rows
  // (columns), which happens at s = 1.
  __shared__ float patch[(kUH + 1) * (kUW + 1)];
  __shared__ int row_a[kUH], row_b[kUH], col_a[kUW], col_b[kUW];
  __shared__ float row_f[kUH], col_f[kUW];
  const int64_t plane = blockIdx.z;
  const int y0 = blockIdx.y * kTileH, x0 = blockIdx.x * kTileW;
  const float* __restrict__ lr = a.x_lr + plane * a.h * a.w;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int cx = 4 * tx;  // first tile column of this thread
  const int x = x0 + cx;
  // The noise this thread blends, requested first so that its DRAM latency
  // overlaps the upsampling below.
  float4 nz[4];
  if (VEC) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int y = y0 + ty + 8 * k;
      nz[k] = (y < a.H && x + 3 < a.W)
                  ? __ldcs(reinterpret_cast<const float4*>(a.noise +
                                                           (plane * a.H + y) * (int64_t)a.W + x))
                  : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }

  // Source taps of the tile's rows and columns (with the halo, clamped to
  // the image), once per CTA.
  for (int i = threadIdx.x; i < kUH + kUW; i += kThreads) {
    if (i < kUH) {
      taps(min(max(y0 - 1 + i, 0), a.H - 1), a.s, a.h, row_a[i], row_b[i], row_f[i]);
    } else {
      const int c = i - kUH;
      taps(min(max(x0 - 1 + c, 0), a.W - 1), a.s, a.w, col_a[c], col_b[c], col_f[c]);
    }
  }
  __syncthreads();
  // The low-res rectangle the taps reach, staged once with coalesced loads.
  const int r0 = row_a[0], pr = row_b[kUH - 1] - r0 + 1;
  const int c0 = col_a[0], pc = col_b[kUW - 1] - c0 + 1;
  for (int i = threadIdx.x; i < pr * pc; i += kThreads) {
    const int r = i / pc, c = i - (i / pc) * pc;
    patch[i] = __ldg(lr + (int64_t)(r0 + r) * a.w + c0 + c);
  }
  __syncthreads();
  // u on the tile and its halo.
  for (int i = threadIdx.x; i < kUH * kUW; i += kThreads) {
    const int r = i / kUW, c = i - (i / kUW) * kUW;
    const float fy = row_f[r], fx = col_f[c];
    const int xa = col_a[c] - c0, xb = col_b[c] - c0;
    const float* ra = patch + (row_a[r] - r0) * pc;
    const float* rb = patch + (row_b[r] - r0) * pc;
    const float top = ra[xa] * (1.f - fx) + ra[xb] * fx;
    const float bot = rb[xa] * (1.f - fx) + rb[xb] * fx;
    u[r][c] = top * (1.f - fy) + bot * fy;
  }
  __syncthreads();

  const float keep = 1.f + a.amount, t1 = 1.f - a.t;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int ry = ty + 8 * k;  // tile row
    const int y = y0 + ry;
    if (y >= a.H) break;
    float hb[3][4];  // horizontal blur of the three rows around ry
#pragma unroll
    for (int dy = 0; dy < 3; ++dy) {
      const float* row = &u[ry + dy][cx];
      float v[6];
#pragma unroll
      for (int j = 0; j < 6; ++j) v[j] = row[j];
#pragma unroll
      for (int j = 0; j < 4; ++j) hb[dy][j] = 0.25f * v[j] + 0.5f * v[j + 1] + 0.25f * v[j + 2];
    }
    float res[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float b = 0.25f * hb[0][j] + 0.5f * hb[1][j] + 0.25f * hb[2][j];
      const float c = u[ry + 1][cx + 1 + j];
      res[j] = t1 * (keep * c - a.amount * b);
    }
    const int64_t off = (plane * a.H + y) * (int64_t)a.W + x;
    if (VEC && x + 3 < a.W) {
      const float4 n = nz[k];
      float4 o;
      o.x = fmaf(a.t, n.x, res[0]);
      o.y = fmaf(a.t, n.y, res[1]);
      o.z = fmaf(a.t, n.z, res[2]);
      o.w = fmaf(a.t, n.w, res[3]);
      __stcs(reinterpret_cast<float4*>(a.out + off), o);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (x + j < a.W) a.out[off + j] = fmaf(a.t, __ldcs(a.noise + off + j), res[j]);
    }
  }
}

}  // namespace

int launch_warm_start(const ug_warm_start_params* p, const float* x_lr, const float* noise,
                      float* out, cudaStream_t st) {
  WarmArgs a;
  a.x_lr = x_lr;
  a.noise = noise;
  a.out = out;
  a.h = p->lr_h;
  a.w = p->lr_w;
  a.s = p->scale;
  a.H = p->lr_h * p->scale;
  a.W = p->lr_w * p->scale;
  a.amount = p->sharpen;
  a.t = p->t;
  const dim3 grid((a.W + kTileW - 1) / kTileW, (a.H + kTileH - 1) / kTileH,
                  (unsigned)(p->batch * p->channels));
  if (a.W % 4 == 0)
    warm_start_kernel<true><<<grid, kThreads, 0, st>>>(a);
  else
    warm_start_kernel<false><<<grid, kThreads, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? UG_OK : UG_ERR_CUDA;
}

}  // namespace ug
