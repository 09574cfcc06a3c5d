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
// Per high-res pixel one fp32 noise read and one fp32 write; the low-res
// image (1/s^2 of that) is read through L1.
//
// Factor 4 (the benchmark's): the whole map is linear in x_lr, and the s x s
// output block of low-res pixel (Y, X) depends only on the 3 x 3 low-res
// neighbourhood around it -- its rows y-1, y, y+1 sample source rows within
// (Y - 1, Y + 1), and likewise for columns -- with weights that depend only
// on the pixel's phase (y mod s, x mod s):
//   out = sum_{r,c} W[py][px][r][c] * x_lr[Y + r - 1][X + c - 1] + t * noise,
//   W = (1 - t) ((1 + amount) e_py e_px^T - amount f_py f_px^T),
// e_p the bilinear weights of phase p over the three source rows and f_p the
// (1/4, 1/2, 1/4) combination of those of phases p - 1, p, p + 1 (the blur).
// Clamping the neighbourhood's indices to the image gives both the bilinear
// clamp and the blur's edge replication: at a border, the high-res row just
// outside the image and the first row inside sample only clamped source
// rows, so they are equal.  The host computes W once per call in fp64; one
// thread per low-res pixel reads its 9 neighbours (L1) and its 16 noise
// values, and writes its 4 x 4 block with 9 fused multiply-adds per output
// plus the noise term.
//
// Other factors: each thread streams 4 adjacent
// columns down a strip of kRows rows with everything in registers:
// the source taps of its 6 columns (the 4 plus one on each side for the
// blur), the two low-res rows it interpolates between (horizontally
// interpolated at those 6 columns), and a rolling window of three upsampled
// rows.  Its noise is requested before any arithmetic.  No shared memory and
// no barrier: every warp streams on its own.  Clamping the rows and columns
// of u at the image border is the blur's edge replication.
#include <cmath>
#include <cstdint>

#include "ug_internal.h"

namespace ug {
namespace {

constexpr int kThreads = 128;
constexpr int kRows = 8;  // output rows per thread

struct WarmArgs {
  const float* x_lr;
  const float* noise;
  float* out;
  int32_t h, w;     // low-res size
  int32_t H, W;     // high-res size
  int32_t s;        // upsampling factor
  int32_t groups;   // ceil(W / 4) column groups per row
  int32_t strips;   // ceil(H / kRows) row strips per plane
  int64_t threads;  // planes * strips * groups
  float amount, t;
};

template <bool VEC>
__global__ void __launch_bounds__(kThreads) warm_start_kernel(const WarmArgs a) {
  const int64_t tid = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (tid >= a.threads) return;
  const int g = (int)(tid % a.groups);
  const int64_t rest = tid / a.groups;
  const int strip = (int)(rest % a.strips);
  const int64_t plane = rest / a.strips;
  const int x0 = 4 * g, y0 = strip * kRows;
  const float* __restrict__ lr = a.x_lr + plane * a.h * a.w;
  const int64_t obase = plane * a.H * (int64_t)a.W;

  // noise of the strip, first
  float4 nz[kRows];
  if (VEC) {
#pragma unroll
    for (int k = 0; k < kRows; ++k)
      nz[k] = (y0 + k < a.H)
                  ? __ldcs(reinterpret_cast<const float4*>(a.noise + obase +
                                                           (int64_t)(y0 + k) * a.W + x0))
                  : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // Source coordinate of high-res index d along an axis of n low-res
  // samples: (d + 0.5) / s - 0.5 = (2d + 1 - s) / (2s), integer part and
  // fraction from the exact integer numerator.  Taps advance incrementally:
  // from index d to d+1 the numerator grows by 2 and carries into the
  // integer part at 2s, so only the first index of a run needs a division.
  const int den = 2 * a.s;
  const float inv_den = 1.0f / (float)den;
  // column taps of x0-1 .. x0+4, clamped to the image
  int ca[6], cb[6];
  float cf[6];
  {
    const int xs = max(x0 - 1, 0);
    int num = 2 * xs + 1 - a.s;
    int fl = num >= 0 ? num / den : -((-num + den - 1) / den);
    int rem = num - fl * den;
    int x = xs;
#pragma unroll
    for (int j = 0; j < 6; ++j) {
      if (x0 - 1 + j > x && x < a.W - 1) {  // advance to column x0-1+j (clamped)
        ++x;
        rem += 2;
        if (rem >= den) {
          rem -= den;
          ++fl;
        }
      }
      ca[j] = min(max(fl, 0), a.w - 1);
      cb[j] = min(max(fl + 1, 0), a.w - 1);
      cf[j] = (float)rem * inv_den;
    }
  }
  // one low-res row interpolated at the 6 columns
  auto hrow = [&](int r, float* hv) {
    const float* row = lr + (int64_t)r * a.w;
#pragma unroll
    for (int j = 0; j < 6; ++j) hv[j] = __ldg(row + ca[j]) * (1.f - cf[j]) + __ldg(row + cb[j]) * cf[j];
  };
  int ra = -1, rb = -1;  // low-res rows held in ha, hb
  float ha[6], hb[6];
  // row taps, advanced one row per call from row max(y0-1, 0) (clamped
  // at the last row)
  int ry = max(y0 - 1, 0);
  int rnum = 2 * ry + 1 - a.s;
  int rfl = rnum >= 0 ? rnum / den : -((-rnum + den - 1) / den);
  int rrem = rnum - rfl * den;
  // u at high-res row y (clamped) and the 6 columns; y never decreases
  auto urow = [&](int y, float* u) {
    const int yc = min(max(y, 0), a.H - 1);
    while (ry < yc) {
      ++ry;
      rrem += 2;
      if (rrem >= den) {
        rrem -= den;
        ++rfl;
      }
    }
    const int ya = min(max(rfl, 0), a.h - 1), yb = min(max(rfl + 1, 0), a.h - 1);
    const float fy = (float)rrem * inv_den;
    if (ya != ra) {
      if (ya == rb) {
#pragma unroll
        for (int j = 0; j < 6; ++j) ha[j] = hb[j];
      } else {
        hrow(ya, ha);
      }
      ra = ya;
    }
    if (yb != rb) {
      hrow(yb, hb);
      rb = yb;
    }
#pragma unroll
    for (int j = 0; j < 6; ++j) u[j] = ha[j] * (1.f - fy) + hb[j] * fy;
  };
  // horizontal blur of u at the 4 output columns
  auto hblur = [](const float* u, float* b) {
#pragma unroll
    for (int j = 0; j < 4; ++j) b[j] = 0.25f * u[j] + 0.5f * u[j + 1] + 0.25f * u[j + 2];
  };
  float u_cur[6], u_nxt[6], b_prev[4], b_cur[4], b_nxt[4];
  urow(y0 - 1, u_cur);
  hblur(u_cur, b_prev);
  urow(y0, u_cur);
  hblur(u_cur, b_cur);
  const float keep = 1.f + a.amount, t1 = 1.f - a.t;
#pragma unroll
  for (int k = 0; k < kRows; ++k) {
    const int y = y0 + k;
    if (y >= a.H) break;
    urow(y + 1, u_nxt);
    hblur(u_nxt, b_nxt);
    float res[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float bl = 0.25f * b_prev[j] + 0.5f * b_cur[j] + 0.25f * b_nxt[j];
      res[j] = t1 * (keep * u_cur[j + 1] - a.amount * bl);
    }
    const int64_t off = obase + (int64_t)y * a.W + x0;
    if (VEC) {
      if (x0 + 3 < a.W) {
        float4 o;
        o.x = fmaf(a.t, nz[k].x, res[0]);
        o.y = fmaf(a.t, nz[k].y, res[1]);
        o.z = fmaf(a.t, nz[k].z, res[2]);
        o.w = fmaf(a.t, nz[k].w, res[3]);
        __stcs(reinterpret_cast<float4*>(a.out + off), o);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (x0 + j < a.W) a.out[off + j] = fmaf(a.t, __ldcs(a.noise + off + j), res[j]);
    }
#pragma unroll
    for (int j = 0; j < 6; ++j) u_cur[j] = u_nxt[j];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      b_prev[j] = b_cur[j];
      b_cur[j] = b_nxt[j];
    }
  }
}

constexpr int kStencilS = 4;
constexpr int kStencilThreads = 256;

struct StencilArgs {
  const float* x_lr;
  const float* noise;
  float* out;
  int32_t h, w;  // low-res size
  int64_t n;     // low-res pixels over all planes
  float t;
  float wt[kStencilS][kStencilS][9];  // [py][px][3 r + c]
};

__global__ void __launch_bounds__(kStencilThreads) warm_start_stencil_kernel(const StencilArgs a) {
  constexpr int S = kStencilS;
  const int64_t tid = (int64_t)blockIdx.x * kStencilThreads + threadIdx.x;
  if (tid >= a.n) return;
  const int X = (int)(tid % a.w);
  const int64_t rest = tid / a.w;
  const int Y = (int)(rest % a.h);
  const int64_t plane = rest / a.h;
  const int64_t W = (int64_t)S * a.w;
  const int64_t obase = (plane * a.h * S + (int64_t)S * Y) * W + (int64_t)S * X;
  // the block's noise first (every read before any write: out may be noise)
  float4 nz[S];
#pragma unroll
  for (int py = 0; py < S; ++py)
    nz[py] = __ldcs(reinterpret_cast<const float4*>(a.noise + obase + py * W));
  const float* __restrict__ lr = a.x_lr + plane * a.h * a.w;
  const int ys[3] = {max(Y - 1, 0), Y, min(Y + 1, a.h - 1)};
  const int xs[3] = {max(X - 1, 0), X, min(X + 1, a.w - 1)};
  float nb[9];
#pragma unroll
  for (int r = 0; r < 3; ++r)
#pragma unroll
    for (int c = 0; c < 3; ++c) nb[3 * r + c] = __ldg(lr + (int64_t)ys[r] * a.w + xs[c]);
#pragma unroll
  for (int py = 0; py < S; ++py) {
    float o[S];
#pragma unroll
    for (int px = 0; px < S; ++px) {
      float acc = a.wt[py][px][0] * nb[0];
#pragma unroll
      for (int k = 1; k < 9; ++k) acc = fmaf(a.wt[py][px][k], nb[k], acc);
      o[px] = acc;
    }
    const float4 n4 = nz[py];
    __stcs(reinterpret_cast<float4*>(a.out + obase + py * W),
           make_float4(fmaf(a.t, n4.x, o[0]), fmaf(a.t, n4.y, o[1]), fmaf(a.t, n4.z, o[2]),
                       fmaf(a.t, n4.w, o[3])));
  }
}

}  // namespace

// W of the stencil for factor s = kStencilS, in fp64, rounded once to fp32,
// as [py][px][3 r + c].
void warm_start_stencil_weights(double amount, double t, float* wt) {
  constexpr int S = kStencilS;
  // bilinear weights over source rows (Y-1, Y, Y+1) of the high-res row
  // S*Y + p + a, a in {-1, 0, 1}: source coordinate Y + q, q = (p + a +
  // 0.5)/S - 0.5 in [-0.625, 0.625]
  double e[S][3] = {}, f[S][3] = {};
  const double g[3] = {0.25, 0.5, 0.25};
  for (int p = 0; p < S; ++p)
    for (int a = -1; a <= 1; ++a) {
      const double q = (p + a + 0.5) / S - 0.5;
      const double fl = std::floor(q), fr = q - fl;
      double v[3] = {0.0, 0.0, 0.0};
      v[(int)fl + 1] += 1.0 - fr;
      v[(int)fl + 2] += fr;
      for (int r = 0; r < 3; ++r) {
        if (a == 0) e[p][r] = v[r];
        f[p][r] += g[a + 1] * v[r];
      }
    }
  for (int py = 0; py < S; ++py)
    for (int px = 0; px < S; ++px)
      for (int r = 0; r < 3; ++r)
        for (int c = 0; c < 3; ++c)
          wt[(py * S + px) * 9 + 3 * r + c] =
              (float)((1.0 - t) * ((1.0 + amount) * e[py][r] * e[px][c] -
                                   amount * f[py][r] * f[px][c]));
}

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
  if (p->scale == kStencilS) {
    StencilArgs sa;
    sa.x_lr = x_lr;
    sa.noise = noise;
    sa.out = out;
    sa.h = p->lr_h;
    sa.w = p->lr_w;
    sa.n = (int64_t)p->batch * p->channels * p->lr_h * p->lr_w;
    sa.t = p->t;
    warm_start_stencil_weights(p->sharpen, p->t, &sa.wt[0][0][0]);
    const int64_t blocks = (sa.n + kStencilThreads - 1) / kStencilThreads;
    warm_start_stencil_kernel<<<(unsigned)blocks, kStencilThreads, 0, st>>>(sa);
    return cudaGetLastError() == cudaSuccess ? UG_OK : UG_ERR_CUDA;
  }
  a.groups = (a.W + 3) / 4;
  a.strips = (a.H + kRows - 1) / kRows;
  a.threads = (int64_t)p->batch * p->channels * a.strips * a.groups;
  const int64_t blocks = (a.threads + kThreads - 1) / kThreads;
  if (a.W % 4 == 0)
    warm_start_kernel<true><<<(unsigned)blocks, kThreads, 0, st>>>(a);
  else
    warm_start_kernel<false><<<(unsigned)blocks, kThreads, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? UG_OK : UG_ERR_CUDA;
}

}  // namespace ug
