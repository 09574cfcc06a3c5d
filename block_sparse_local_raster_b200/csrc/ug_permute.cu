// Window-first permutation of the high-res token grid and its inverse
// (UltraGen-fr §2.A "Ordre Window-First"; UltraGen-ar §2.أ).
//
// One row of one window -- win_w raster-consecutive tokens -- stays
// consecutive in window-first order, so the permutation moves contiguous
// segments of win_w * heads * head_dim * 2 bytes (96 KiB at 16 tokens x 24
// heads x 128 dims).  Each CTA copies whole segments with 16-byte loads and
// stores: fully coalesced on both sides, no shared memory, index arithmetic
// once per segment.  HBM-bound: 2 bytes moved per byte of tensor.
#include <cstdint>

#include "ug_debug.h"
#include "ug_internal.h"

namespace ug {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

struct PermuteArgs {
  const uint4* src;
  uint4* dst;
  int64_t n_seg;       // batch * grid_h * windows per row
  int64_t n_tok;       // high-res tokens per batch element
  int32_t row_chunks;  // 16-byte chunks per token row (heads * head_dim / 8)
  int32_t seg_chunks;  // win_w * row_chunks
  int32_t grid_h, grid_w, win_h, win_w, nwx, T;
  int32_t inverse;     // 0: raster -> window-first, 1: window-first -> raster
  int64_t batch;       // B (debug-build range checks)
  int* err;            // the plan's error word
};

__global__ void __launch_bounds__(kThreads) permute_kernel(const PermuteArgs a) {
  for (int64_t seg = blockIdx.x; seg < a.n_seg; seg += gridDim.x) {
    const int64_t per_b = (int64_t)a.grid_h * a.nwx;
    const int64_t b = seg / per_b;
    const int32_t rem = (int32_t)(seg - b * per_b);
    const int32_t y = rem / a.nwx, wx = rem - (rem / a.nwx) * a.nwx;
    const int32_t wy = y / a.win_h, ly = y - wy * a.win_h;
    const int64_t r0 = (int64_t)y * a.grid_w + (int64_t)wx * a.win_w;        // raster token
    const int64_t p0 = ((int64_t)wy * a.nwx + wx) * a.T + (int64_t)ly * a.win_w;  // window-first
    const int64_t s_tok = a.inverse ? p0 : r0;
    const int64_t d_tok = a.inverse ? r0 : p0;
    // both runs of win_w tokens lie inside their batch element's tensor
    if (!dbg_ok(b < a.batch && s_tok >= 0 && d_tok >= 0 && s_tok + a.win_w <= a.n_tok &&
                    d_tok + a.win_w <= a.n_tok,
                a.err))
      continue;
    const uint4* __restrict__ s = a.src + (b * a.n_tok + s_tok) * a.row_chunks;
    uint4* __restrict__ d = a.dst + (b * a.n_tok + d_tok) * a.row_chunks;
    int32_t c = threadIdx.x;
    for (; c + (kUnroll - 1) * kThreads < a.seg_chunks; c += kUnroll * kThreads) {
      uint4 v[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) v[u] = __ldcs(s + c + u * kThreads);
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) d[c + u * kThreads] = v[u];
    }
    for (; c < a.seg_chunks; c += kThreads) d[c] = __ldcs(s + c);
  }
}

}  // namespace

int launch_permute(const ug_plan* p, const void* src, void* dst, bool inverse, cudaStream_t st) {
  PermuteArgs a;
  a.src = static_cast<const uint4*>(src);
  a.dst = static_cast<uint4*>(dst);
  a.grid_h = p->g.grid_h;
  a.grid_w = p->g.grid_w;
  a.win_h = p->g.win_h;
  a.win_w = p->g.win_w;
  a.nwx = p->nwx;
  a.T = (int32_t)p->T;
  a.n_tok = p->N;
  a.row_chunks = p->g.heads * p->g.head_dim / 8;
  a.seg_chunks = a.win_w * a.row_chunks;
  a.n_seg = (int64_t)p->g.batch * p->g.grid_h * p->nwx;
  a.inverse = inverse ? 1 : 0;
  a.batch = p->g.batch;
  a.err = p->d_err;
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, p->device);
  const int64_t blocks = std::min<int64_t>(a.n_seg, (int64_t)sms * (2048 / kThreads));
  permute_kernel<<<(unsigned)blocks, kThreads, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? UG_OK : UG_ERR_CUDA;
}

}  // namespace ug
