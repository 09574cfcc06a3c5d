// Backward of the block-sparse joint-softmax attention on B200 (sm_100a).
//
// The gradients of O = softmax(scale * Q K^T, masked) V, with the mask of the
// forward (UltraGen-ar §2.ب "Attention Masking"), are needed to train the
// LoRA adapters of the q/k/v projections the pages describe (UltraGen-ar
// §2.ج, UltraGen-fr §2.C).  With P recomputed from the forward's
// log-sum-exp and D = rowsum(dO * O):
//   dP = dO V^T,  dS = P * (dP - D),
//   dQ = scale * dS K,  dK = scale * dS^T Q,  dV = P^T dO.
// Three kernels:
//   delta_kernel  D for every query row (HBM-bound, one pass over O and dO);
//   dq_kernel     one 128-row query tile per CTA; Q and dO stay in shared
//                 memory while K_j, V_j stream through a 5-slot TMA ring over
//                 the forward's key-block list; per block S = Q K^T and
//                 dP = dO V^T share one TMEM buffer, P (bf16) waits for dP in
//                 the TMEM quarter the layout leaves free, and dS (bf16,
//                 written over S/dP) is the TMEM A operand of dQ += dS K;
//   dkv_kernel    one 128-key block per CTA; K and V stay in shared memory
//                 while Q_i, dO_i stream over the block's list of query
//                 tiles; S^T = K Q_i^T gives P^T (bf16 in TMEM), the A
//                 operand of dV += P^T dO_i; dP^T = V dO_i^T then gives dS^T,
//                 the A operand of dK += dS^T Q_i.
// In both, two TMEM buffers take consecutive blocks (or tiles), and the two
// warpgroups of the softmax warps take one buffer each, so one block's
// exponentials overlap the other block's products.  TMEM lanes hold the
// rows of the stationary operand (queries in dq_kernel, keys in dkv_kernel),
// so every per-row quantity stays in its thread.
//
// Waits are bounded as in the forward: on expiry the kernel records
// UG_ERR_TIMEOUT, unwinds (in-flight loads and MMAs drained), frees TMEM and
// exits.
#include <cstdint>

#include <cuda.h>
#include <cuda_bf16.h>

#include "ug_debug.h"
#include "ug_internal.h"
#include "ug_per_device.h"
#include "ug_tc.cuh"

namespace ug {
namespace {

constexpr int kBwdThreads = 320;  // warps 0-7 softmax (2 warpgroups), 8 producer, 9 MMA
constexpr int kBwdProducer = 8;
constexpr int kBwdMma = 9;
constexpr int kRing = 5;

struct BwdParams {
  const QTile* qtiles;
  const uint32_t* kvlist;
  const KTile* ktiles;
  const uint32_t* qlist;
  const float* lse;    // [B, h, N + L], natural log (forward output)
  const float* delta;  // [B, h, N + L]
  __nv_bfloat16* dq_hr;
  __nv_bfloat16* dq_lr;
  __nv_bfloat16* dk_hr;
  __nv_bfloat16* dk_lr;
  __nv_bfloat16* dv_hr;
  __nv_bfloat16* dv_lr;
  int* err;
  int64_t timeout_ns;
  int32_t N, L, T, nwx, radius, heads;
  float scale;       // softmax scale
  float scale_log2;  // softmax scale * log2(e)
  int32_t kv_len, q_len;  // entries in kvlist / qlist (debug-build range checks)
  // Raster-order high-res V, O, dO and dV (V and dO read through 5-D tensor
  // maps, one 128-row tile = 128 / win_w whole rows of one window; dV rows
  // scattered to their raster positions).
  int32_t vo_raster;
  int32_t grid_w, win_h, win_w;
};

// Raster index of the high-res token at window-first position p.
__device__ __forceinline__ int raster_of(int p, int T, int nwx, int win_h, int win_w,
                                         int grid_w) {
  const int w = p / T, l = p - (p / T) * T;
  const int wy = w / nwx, wx = w - (w / nwx) * nwx;
  const int ly = l / win_w, lx = l - (l / win_w) * win_w;
  return (wy * win_h + ly) * grid_w + wx * win_w + lx;
}

// One 128-row tile (rows row0.. of the window-first order, one head) of a
// high-res tensor into shared memory: through the 4-D map of a window-first
// tensor, or the 5-D map of a raster one (the tile is 128 / win_w whole rows
// of one window, landing in window-first order).
template <int kRegions>
__device__ __forceinline__ void load_hr_tile(uint32_t dst, const CUtensorMap* map, bool raster,
                                             int row0, int head, int b, const BwdParams& P,
                                             uint32_t bar) {
  if (raster) {
    const int w = row0 / P.T, ly0 = (row0 - (row0 / P.T) * P.T) / P.win_w;
    const int wy = w / P.nwx, wx = w - (w / P.nwx) * P.nwx;
    for (int r = 0; r < kRegions; ++r)
      tma_load_5d(dst + r * kRowsPerTile * 128, map, r * 64, head, wx * P.win_w,
                  wy * P.win_h + ly0, b, bar);
  } else {
    for (int r = 0; r < kRegions; ++r)
      tma_load_4d(dst + r * kRowsPerTile * 128, map, r * 64, head, row0, b, bar);
  }
}

// Debug build: a list slice [off, off + len) inside a list of n entries, and
// every 128-row block it names inside its token set.
__device__ __forceinline__ bool list_in_range(const uint32_t* list, int off, int len, int n,
                                              int n_hr, int n_lr) {
  bool ok = off >= 0 && len >= 0 && off + len <= n;
  for (int j = 0; ok && j < len; ++j) {
    const uint32_t e = list[off + j];
    ok = (int64_t)(e & kBlockIndexMask) * kRowsPerTile < ((e & kBlockLowres) ? n_lr : n_hr);
  }
  return ok;
}

constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------------ delta

// D[b, h, r] = sum_c dO[b, r, h, c] * O[b, r, h, c] (fp32), for the high-res
// rows (window-first order r; O and dO window-first, or raster with
// `raster`) then the global rows.  One warp per token row; D/8 lanes per head.
template <int D>
__global__ void __launch_bounds__(256) delta_kernel(const __nv_bfloat16* __restrict__ o_hr,
                                                    const __nv_bfloat16* __restrict__ do_hr,
                                                    const __nv_bfloat16* __restrict__ o_lr,
                                                    const __nv_bfloat16* __restrict__ do_lr,
                                                    float* __restrict__ delta, int B, int N,
                                                    int L, int H, int raster, int T, int nwx,
                                                    int win_h, int win_w, int grid_w) {
  constexpr int kCh = D / 8;        // 16-byte chunks per head
  constexpr int kHeadsPer = 32 / kCh;
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t rows = (int64_t)B * (N + L);
  for (int64_t r = warp0; r < rows; r += nwarps) {
    const int b = (int)(r / (N + L));
    const int tok = (int)(r - (int64_t)b * (N + L));
    const bool lr = tok >= N;
    const int t = lr ? tok - N : tok;
    const int n = lr ? L : N;
    // with raster o_hr / do_hr, window-first row t sits at its raster position
    const int mt = (!lr && raster) ? raster_of(t, T, nwx, win_h, win_w, grid_w) : t;
    const int64_t base = ((int64_t)b * n + mt) * H * D;
    const uint4* o = reinterpret_cast<const uint4*>((lr ? o_lr : o_hr) + base);
    const uint4* g = reinterpret_cast<const uint4*>((lr ? do_lr : do_hr) + base);
    for (int h0 = 0; h0 < H; h0 += kHeadsPer) {
      const int h = h0 + lane / kCh;
      float acc = 0.0f;
      if (h < H) {
        const uint4 a = __ldcs(o + h * kCh + lane % kCh);
        const uint4 c = __ldcs(g + h * kCh + lane % kCh);
        const uint32_t* pa = reinterpret_cast<const uint32_t*>(&a);
        const uint32_t* pc = reinterpret_cast<const uint32_t*>(&c);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 x = unpack_bf16(pa[k]), y = unpack_bf16(pc[k]);
          acc = fmaf(x.x, y.x, acc);
          acc = fmaf(x.y, y.y, acc);
        }
      }
#pragma unroll
      for (int off = kCh / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
      if (h < H && lane % kCh == 0) delta[((int64_t)b * H + h) * (N + L) + tok] = acc;
    }
  }
}

// ------------------------------------------------------------------ shared pieces

template <int D>
struct Tiles {
  static constexpr int kTile = kRowsPerTile * D * 2;  // 128 rows x D bf16
  static constexpr int kRegions = D / 64;              // 128-byte swizzle spans 64 columns
};

// D = A B^T over D/16 K-steps: A and B are 128-row tiles, K-major, 128-byte
// swizzled in D/64 regions of 128 rows x 128 bytes.
template <int D>
__device__ __forceinline__ void mma_rows(uint32_t d, uint32_t a, uint32_t b) {
  constexpr uint32_t kId = instr_desc(128, false);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk / 4) * (kRowsPerTile * 128) + (kk % 4) * 32;
    mma_bf16(d, smem_desc(a + off, 16, 1024), smem_desc(b + off, 16, 1024), kId, kk > 0);
  }
}

// D += A B with A (128 x 128, bf16 pairs over 64 TMEM columns from a_tmem)
// and B a 128-row tile read MN-major (N = D columns, K = its 128 rows).
template <int D>
__device__ __forceinline__ void mma_tmem_rows(uint32_t d, uint32_t a_tmem, uint32_t b, bool acc) {
  constexpr uint32_t kId = instr_desc(D, true);
#pragma unroll
  for (int kk = 0; kk < kRowsPerTile / 16; ++kk)
    mma_bf16_tmem_a(d, a_tmem + kk * 8, smem_desc(b + kk * 16 * 128, kRowsPerTile * 128, 1024),
                    kId, (acc || kk > 0) ? 1u : 0u);
}

// Masks the row's scores where a high-res pair is invisible: `mine` is the
// window of this thread's row (query in dq_kernel, key in dkv_kernel), the
// COLS columns are the tokens c0 .. c0+COLS-1 of the other side.  Visibility
// changes only at window boundaries, so each window met is tested once.
template <int COLS>
__device__ __forceinline__ void mask_windows(float* s, int c0, int mine, const BwdParams& P) {
  const int my = mine / P.nwx, mx = mine - (mine / P.nwx) * P.nwx;
  int i0 = 0;
  while (i0 < COLS) {
    const int c = c0 + i0;
    const int w = c / P.T;
    const int run = min(COLS, (w + 1) * P.T - c0);
    const int wy = w / P.nwx, wx = w - (w / P.nwx) * P.nwx;
    const bool vis = abs(wy - my) <= P.radius && abs(wx - mx) <= P.radius;
    const int lim = vis ? min(run, P.N - c0) : i0;  // columns [i0, lim) stay
#pragma unroll
    for (int i = 0; i < COLS; ++i)
      if (i >= i0 && i < run && i >= lim) s[i] = kNegInf;
    i0 = run;
  }
}

// Bounded polling for an issue loop that tests several barriers: gives up
// (records UG_ERR_TIMEOUT, raises the abort flag) after timeout_ns without
// progress, or when the abort flag is up.
struct PollTimer {
  uint64_t last;
  uint32_t spins;
  __device__ PollTimer() : last(globaltimer()), spins(0) {}
  __device__ bool step(bool progressed, volatile uint32_t* abort, int* err, int64_t timeout_ns) {
    if (progressed) {
      spins = 0;
      last = globaltimer();
      return true;
    }
    if ((++spins & 15u) != 0u) return true;
    if (*abort) return false;
    if ((int64_t)(globaltimer() - last) > timeout_ns) {
      atomicCAS(err, 0, (int)UG_ERR_TIMEOUT);
      *abort = 1u;
      return false;
    }
    return true;
  }
};

// ------------------------------------------------------------------ dQ

template <int D>
struct DqLayout {
  static constexpr int kTile = Tiles<D>::kTile;
  static constexpr int kQ = 0;
  static constexpr int kDO = kQ + kTile;
  static constexpr int kKV = kDO + kTile;
  static constexpr int kBar = kKV + kRing * kTile;
  // q_full, kv_full[R], kv_empty[R], s_full[2], s_free[2], dp_full[2], ds_full[2], dq_done, drain
  static constexpr int kNumBars = 1 + 2 * kRing + 8 + 2;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
};

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    dq_kernel(const __grid_constant__ CUtensorMap tm_q_hr,
              const __grid_constant__ CUtensorMap tm_k_hr,
              const __grid_constant__ CUtensorMap tm_v_hr,
              const __grid_constant__ CUtensorMap tm_do_hr,
              const __grid_constant__ CUtensorMap tm_q_lr,
              const __grid_constant__ CUtensorMap tm_k_lr,
              const __grid_constant__ CUtensorMap tm_v_lr,
              const __grid_constant__ CUtensorMap tm_do_lr, const BwdParams P) {
  using Lay = DqLayout<D>;
  constexpr int kRegions = Tiles<D>::kRegions;
  constexpr int kTile = Lay::kTile;
  const QTile qt = P.qtiles[blockIdx.x >> 1];
  const int q0 = qt.q0 + (int)(blockIdx.x & 1) * kRowsPerTile;
  const int ntok = qt.lowres ? P.L : P.N;
  if (q0 >= ntok) return;  // the second half of a short last CTA: no rows

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + Lay::kBar;
  const uint32_t q_full = bar0;
  auto kv_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto kv_empty = [&](int s) { return bar0 + 8u * (1 + kRing + s); };
  auto s_full = [&](int t) { return bar0 + 8u * (1 + 2 * kRing + t); };
  auto s_free = [&](int t) { return bar0 + 8u * (1 + 2 * kRing + 2 + t); };
  auto dp_full = [&](int t) { return bar0 + 8u * (1 + 2 * kRing + 4 + t); };
  auto ds_full = [&](int t) { return bar0 + 8u * (1 + 2 * kRing + 6 + t); };
  const uint32_t dq_done = bar0 + 8u * (1 + 2 * kRing + 8);
  const uint32_t drain = bar0 + 8u * (1 + 2 * kRing + 9);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMisc);
  volatile uint32_t* abort = reinterpret_cast<volatile uint32_t*>(smem + Lay::kMisc + 4);
  int* const err = P.err;
  const int64_t timeout_ns = P.timeout_ns;
  auto wait1 = [&](uint32_t bar, uint32_t par) {
    return mbar_wait(bar, par, abort, err, timeout_ns, false);
  };
  auto drain_wait = [&](uint32_t bar, uint32_t par) {
    return mbar_wait(bar, par, abort, err, kDefaultWaitTimeoutNs, true);
  };
  auto wait_warp = [&](uint32_t bar, uint32_t par) {
    return __all_sync(0xFFFFFFFFu, mbar_wait(bar, par, abort, err, timeout_ns, false)) != 0;
  };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int head = blockIdx.y;
  const int b = blockIdx.z;
  const int nblk = qt.list_len;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kRing; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(s_full(t), 1);
      mbar_init(s_free(t), kRowsPerTile);
      mbar_init(dp_full(t), 1);
      mbar_init(ds_full(t), kRowsPerTile);
    }
    mbar_init(dq_done, 1);
    mbar_init(drain, 1);
    *abort = *reinterpret_cast<volatile int*>(err) != 0 ? 1u : 0u;
#if UG_DEBUG
    if (!dbg_ok(list_in_range(P.kvlist, qt.list_off, nblk, P.kv_len, P.N, P.L) && qt.q0 >= 0 &&
                    qt.q0 < (qt.lowres ? P.L : P.N),
                err))
      *abort = 1u;
#endif
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kBwdMma) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     smem_u32(tmem_slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (warp == kBwdProducer && lane == 0) {
    prefetch_map(qt.lowres ? &tm_q_lr : &tm_q_hr);
    prefetch_map(qt.lowres ? &tm_do_lr : &tm_do_hr);
    prefetch_map(&tm_k_hr);
    prefetch_map(&tm_v_hr);
    if (P.L > 0) {
      prefetch_map(&tm_k_lr);
      prefetch_map(&tm_v_lr);
    }
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool skip = *abort != 0u;
  // ring item 2j is K_j, item 2j+1 is V_j
  auto slot = [](int it) { return it % kRing; };
  auto phase = [](int it) { return (uint32_t)(it / kRing) & 1u; };

  if (skip) {
  } else if (warp == kBwdProducer) {
    if (lane == 0) {
      mbar_expect_tx(q_full, 2 * kTile);
      for (int r = 0; r < kRegions; ++r)
        tma_load_4d(sbase + Lay::kQ + r * kRowsPerTile * 128, qt.lowres ? &tm_q_lr : &tm_q_hr,
                    r * 64, head, q0, b, q_full);
      load_hr_tile<kRegions>(sbase + Lay::kDO, qt.lowres ? &tm_do_lr : &tm_do_hr,
                             !qt.lowres && P.vo_raster, q0, head, b, P, q_full);
      int it = 0;
      bool ok = true;
      for (int j = 0; j < nblk && ok; ++j) {
        const uint32_t e = P.kvlist[qt.list_off + j];
        const bool lr = (e & kBlockLowres) != 0;
        const int k0 = (int)(e & kBlockIndexMask) * kKeysPerBlock;
        for (int kv = 0; kv < 2; ++kv, ++it) {
          const CUtensorMap* m = kv == 0 ? (lr ? &tm_k_lr : &tm_k_hr) : (lr ? &tm_v_lr : &tm_v_hr);
          if (!wait1(kv_empty(slot(it)), phase(it) ^ 1u)) {
            ok = false;
            break;
          }
          mbar_expect_tx(kv_full(slot(it)), kTile);
          load_hr_tile<kRegions>(sbase + Lay::kKV + slot(it) * kTile, m,
                                 kv == 1 && !lr && P.vo_raster, k0, head, b, P,
                                 kv_full(slot(it)));
        }
      }
      for (int i = (it > kRing ? it - kRing : 0); i < it; ++i) drain_wait(kv_full(slot(i)), phase(i));
      drain_wait(q_full, 0);
    }
  } else if (warp == kBwdMma) {
    if (lane == 0) {
      const uint32_t tB[2] = {tmem + 0u, tmem + 128u};
      const uint32_t tQ = tmem + 256u;
      const uint32_t sQ = sbase + Lay::kQ, sDO = sbase + Lay::kDO;
      auto kv_addr = [&](int it) { return sbase + Lay::kKV + slot(it) * kTile; };
      // Issue each step as soon as its inputs are ready: S_j = Q K_j^T (needs
      // K_j and buffer j&1 free, i.e. dQ_{j-2} issued), dP_j = dO V_j^T over S_j
      // (needs V_j and the softmax done reading S_j), dQ += dS_j K_j (needs
      // dS_j).  Steps of one kind go in block order; no barrier is tested
      // more than one phase ahead.
      bool ok = wait1(q_full, 0);
      int ns = 0, na = 0, nb = 0;  // next S, next dP, next dQ
      PollTimer poll;
      while (ok && nb < nblk) {
        bool did = true;
        if (nb < na && mbar_test(ds_full(nb & 1), (uint32_t)(nb >> 1) & 1u)) {
          fence_after();
          mma_tmem_rows<D>(tQ, tB[nb & 1], kv_addr(2 * nb), nb > 0);  // dQ += dS_j K_j
          mma_commit(kv_empty(slot(2 * nb)));
          ++nb;
        } else if (na < ns && mbar_test(kv_full(slot(2 * na + 1)), phase(2 * na + 1)) &&
                   mbar_test(s_free(na & 1), (uint32_t)(na >> 1) & 1u)) {
          fence_after();
          mma_rows<D>(tB[na & 1], sDO, kv_addr(2 * na + 1));  // dP_j = dO V_j^T, over S_j
          mma_commit(dp_full(na & 1));
          mma_commit(kv_empty(slot(2 * na + 1)));
          ++na;
        } else if (ns < nblk && ns <= nb + 1 && mbar_test(kv_full(slot(2 * ns)), phase(2 * ns))) {
          fence_after();
          mma_rows<D>(tB[ns & 1], sQ, kv_addr(2 * ns));  // S_j = Q K_j^T
          mma_commit(s_full(ns & 1));
          ++ns;
        } else {
          did = false;
        }
        ok = poll.step(did, abort, err, timeout_ns);
      }
      if (ok) mma_commit(dq_done);
      mma_commit(drain);
      drain_wait(drain, 0);
    }
  } else {
    const int g = warp >> 2;                   // warpgroup: blocks j = g, g+2, ...
    const int row = (warp & 3) * 32 + lane;    // TMEM lane = query row of the tile
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tb = tmem + lane_base + (g ? 128u : 0u);
    const uint32_t tp = tmem + lane_base + 384u + (g ? 64u : 0u);  // parked P (bf16 pairs)
    const int tok = q0 + row;
    const bool valid = tok < ntok;
    const int64_t ridx = ((int64_t)b * P.heads + head) * (P.N + P.L) + (qt.lowres ? P.N : 0) + tok;
    // Rows past the tensor get probability 0 everywhere.
    const float lse2 = valid ? P.lse[ridx] * kLog2e : __int_as_float(0x7f800000);
    const float dlt = valid ? P.delta[ridx] : 0.0f;
    const int q_w = tok / P.T;
    bool ok = true;
    for (int j = g; j < nblk; j += 2) {
      const uint32_t e = P.kvlist[qt.list_off + j];
      const uint32_t ph = (uint32_t)(j >> 1) & 1u;
      if (!(ok = wait_warp(s_full(g), ph))) break;
      fence_after();
      // P = 2^(s * scale * log2e - lse2) as bf16 pairs, parked in this
      // warpgroup's 64 columns of the last TMEM quarter until dS needs it;
      // the scores are read in two halves of 64 keys.
      const float2 sc2 = make_float2(P.scale_log2, P.scale_log2);
      const float2 nl2 = make_float2(-lse2, -lse2);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t pk[32];
        float s[64];
        tmem_ld32(tb + 64 * hf, s);
        tmem_ld32(tb + 64 * hf + 32, s + 32);
        tmem_ld_wait();
        if (e & kBlockMasked) {
          const int k0 = (int)(e & kBlockIndexMask) * kKeysPerBlock + 64 * hf;
          if (e & kBlockLowres) {
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (k0 + i >= P.L) s[i] = kNegInf;
          } else {
            mask_windows<64>(s, k0, q_w, P);
          }
        }
#pragma unroll
        for (int i = 0; i < 64; i += 2) {
          const float2 x = __ffma2_rn(make_float2(s[i], s[i + 1]), sc2, nl2);
          pk[i / 2] = pack_bf16(fast_exp2(x.x), fast_exp2(x.y));
        }
        tmem_st32u(tp + 32 * hf, pk);
      }
      tmem_st_wait();
      fence_before();
      mbar_arrive(s_free(g));  // S read: dP may overwrite the buffer
      if (!(ok = wait_warp(dp_full(g), ph))) break;
      fence_after();
      // dS = P (dP - D) as bf16 pairs over the first 64 columns; chunk c
      // writes columns [16c, 16c+16), all already read.
#pragma unroll
      for (int c = 0; c < kKeysPerBlock / 32; ++c) {
        float dp[32];
        float pf[16];
        tmem_ld32(tb + c * 32, dp);
        tmem_ld16(tp + c * 16, pf);
        tmem_ld_wait();
        const uint32_t* pk = reinterpret_cast<const uint32_t*>(pf);
        uint32_t ds[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float2 p = unpack_bf16(pk[i / 2]);
          ds[i / 2] = pack_bf16(p.x * (dp[i] - dlt), p.y * (dp[i + 1] - dlt));
        }
        tmem_st16u(tb + c * 16, ds);
      }
      tmem_st_wait();
      fence_before();
      mbar_arrive(ds_full(g));
    }
    if (g == 0) {
      if (ok && nblk > 0) ok = wait_warp(dq_done, 0);
      if (ok) {
        fence_after();
        __nv_bfloat16* dst =
            (qt.lowres ? P.dq_lr : P.dq_hr) + (((int64_t)b * ntok + tok) * P.heads + head) * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          if (nblk > 0) {
            tmem_ld32(tmem + lane_base + 256u + c * 32, o);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = 0.0f;
          }
          if (valid) {
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              const float k = P.scale;
              *reinterpret_cast<uint4*>(dst + c * 32 + i) =
                  make_uint4(pack_bf16(o[i] * k, o[i + 1] * k), pack_bf16(o[i + 2] * k, o[i + 3] * k),
                             pack_bf16(o[i + 4] * k, o[i + 5] * k), pack_bf16(o[i + 6] * k, o[i + 7] * k));
            }
          }
        }
      }
    }
  }

  fence_before();
  __syncthreads();
  if (warp == kBwdMma) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

// ------------------------------------------------------------------ dK, dV

template <int D>
struct DkvLayout {
  static constexpr int kTile = Tiles<D>::kTile;
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTile;
  static constexpr int kRingOff = kV + kTile;
  static constexpr int kStats = kRingOff + kRing * kTile;  // lse2[2][128], delta[2][128]
  static constexpr int kBar = kStats + 4 * kRowsPerTile * 4;
  // kv_full, ring_full[R], ring_empty[R], s_full[2], p_full[2], dp_full[2], ds_full[2], acc_done,
  // drain, group[2]
  static constexpr int kNumBars = 1 + 2 * kRing + 8 + 2 + 2;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16;
  // No alignment slack at D = 128 (the layout fills the 227 KB a CTA may
  // use): the kernel checks that the dynamic shared memory starts on a
  // 1024-byte boundary and reports UG_ERR_UNSUPPORTED otherwise.
  static constexpr int kAlloc = kBytes;
};

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    dkv_kernel(const __grid_constant__ CUtensorMap tm_q_hr,
               const __grid_constant__ CUtensorMap tm_k_hr,
               const __grid_constant__ CUtensorMap tm_v_hr,
               const __grid_constant__ CUtensorMap tm_do_hr,
               const __grid_constant__ CUtensorMap tm_q_lr,
               const __grid_constant__ CUtensorMap tm_k_lr,
               const __grid_constant__ CUtensorMap tm_v_lr,
               const __grid_constant__ CUtensorMap tm_do_lr, const BwdParams P) {
  using Lay = DkvLayout<D>;
  constexpr int kRegions = Tiles<D>::kRegions;
  constexpr int kTile = Lay::kTile;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicCAS(P.err, 0, (int)UG_ERR_UNSUPPORTED);
    return;
  }
  uint8_t* smem = smem_raw;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + Lay::kBar;
  const uint32_t kv_full = bar0;
  auto ring_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto ring_empty = [&](int s) { return bar0 + 8u * (1 + kRing + s); };
  auto s_full = [&](int t) { return bar0 + 8u * (1 + 2 * kRing + t); };
  auto p_full = [&](int t) { return bar0 + 8u * (1 + 2 * kRing + 2 + t); };
  auto dp_full = [&](int t) { return bar0 + 8u * (1 + 2 * kRing + 4 + t); };
  auto ds_full = [&](int t) { return bar0 + 8u * (1 + 2 * kRing + 6 + t); };
  const uint32_t acc_done = bar0 + 8u * (1 + 2 * kRing + 8);
  const uint32_t drain = bar0 + 8u * (1 + 2 * kRing + 9);
  // a barrier of the 128 threads of one softmax warpgroup
  auto group = [&](int t) { return bar0 + 8u * (1 + 2 * kRing + 10 + t); };
  float* const stat_lse = reinterpret_cast<float*>(smem + Lay::kStats);              // [2][128]
  float* const stat_dlt = reinterpret_cast<float*>(smem + Lay::kStats) + 2 * kRowsPerTile;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMisc);
  volatile uint32_t* abort = reinterpret_cast<volatile uint32_t*>(smem + Lay::kMisc + 4);
  int* const err = P.err;
  const int64_t timeout_ns = P.timeout_ns;
  auto wait1 = [&](uint32_t bar, uint32_t par) {
    return mbar_wait(bar, par, abort, err, timeout_ns, false);
  };
  auto drain_wait = [&](uint32_t bar, uint32_t par) {
    return mbar_wait(bar, par, abort, err, kDefaultWaitTimeoutNs, true);
  };
  auto wait_warp = [&](uint32_t bar, uint32_t par) {
    return __all_sync(0xFFFFFFFFu, mbar_wait(bar, par, abort, err, timeout_ns, false)) != 0;
  };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const KTile kt = P.ktiles[blockIdx.x];
  const int head = blockIdx.y;
  const int b = blockIdx.z;
  const int nq = kt.list_len;
  const int nk = kt.lowres ? P.L : P.N;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < kRing; ++s) {
      mbar_init(ring_full(s), 1);
      mbar_init(ring_empty(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(s_full(t), 1);
      mbar_init(p_full(t), kRowsPerTile);
      mbar_init(dp_full(t), 1);
      mbar_init(ds_full(t), kRowsPerTile);
    }
    mbar_init(acc_done, 1);
    mbar_init(drain, 1);
    mbar_init(group(0), kRowsPerTile);
    mbar_init(group(1), kRowsPerTile);
    *abort = *reinterpret_cast<volatile int*>(err) != 0 ? 1u : 0u;
#if UG_DEBUG
    if (!dbg_ok(list_in_range(P.qlist, kt.list_off, nq, P.q_len, P.N, P.L) && kt.k0 >= 0 &&
                    kt.k0 < nk,
                err))
      *abort = 1u;
#endif
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kBwdMma) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     smem_u32(tmem_slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (warp == kBwdProducer && lane == 0) {
    prefetch_map(kt.lowres ? &tm_k_lr : &tm_k_hr);
    prefetch_map(kt.lowres ? &tm_v_lr : &tm_v_hr);
    prefetch_map(&tm_q_hr);
    prefetch_map(&tm_do_hr);
    if (P.L > 0) {
      prefetch_map(&tm_q_lr);
      prefetch_map(&tm_do_lr);
    }
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool skip = *abort != 0u;
  // ring item 2i is Q_i, item 2i+1 is dO_i
  auto slot = [](int it) { return it % kRing; };
  auto phase = [](int it) { return (uint32_t)(it / kRing) & 1u; };

  if (skip) {
  } else if (warp == kBwdProducer) {
    if (lane == 0) {
      mbar_expect_tx(kv_full, 2 * kTile);
      for (int r = 0; r < kRegions; ++r)
        tma_load_4d(sbase + Lay::kK + r * kKeysPerBlock * 128, kt.lowres ? &tm_k_lr : &tm_k_hr,
                    r * 64, head, kt.k0, b, kv_full);
      load_hr_tile<kRegions>(sbase + Lay::kV, kt.lowres ? &tm_v_lr : &tm_v_hr,
                             !kt.lowres && P.vo_raster, kt.k0, head, b, P, kv_full);
      int it = 0;
      bool ok = true;
      for (int i = 0; i < nq && ok; ++i) {
        const uint32_t e = P.qlist[kt.list_off + i];
        const bool lr = (e & kBlockLowres) != 0;
        const int q0 = (int)(e & kBlockIndexMask) * kRowsPerTile;
        for (int x = 0; x < 2; ++x, ++it) {
          const CUtensorMap* m = x == 0 ? (lr ? &tm_q_lr : &tm_q_hr) : (lr ? &tm_do_lr : &tm_do_hr);
          if (!wait1(ring_empty(slot(it)), phase(it) ^ 1u)) {
            ok = false;
            break;
          }
          mbar_expect_tx(ring_full(slot(it)), kTile);
          load_hr_tile<kRegions>(sbase + Lay::kRingOff + slot(it) * kTile, m,
                                 x == 1 && !lr && P.vo_raster, q0, head, b, P,
                                 ring_full(slot(it)));
        }
      }
      for (int i = (it > kRing ? it - kRing : 0); i < it; ++i)
        drain_wait(ring_full(slot(i)), phase(i));
      drain_wait(kv_full, 0);
    }
  } else if (warp == kBwdMma) {
    if (lane == 0) {
      const uint32_t tB[2] = {tmem + 0u, tmem + 128u};
      const uint32_t tdV = tmem + 256u, tdK = tmem + 384u;
      const uint32_t sK = sbase + Lay::kK, sV = sbase + Lay::kV;
      auto ring_addr = [&](int it) { return sbase + Lay::kRingOff + slot(it) * kTile; };
      // As in dq_kernel: S^T_i = K Q_i^T (needs Q_i and buffer i&1 free, i.e.
      // dK_{i-2} issued), then dV += P^T_i dO_i and dP^T_i = V dO_i^T (need
      // dO_i and P^T_i), then dK += dS^T_i Q_i (needs dS^T_i), each kind in
      // tile order, issued as soon as ready.
      bool ok = wait1(kv_full, 0);
      int ns = 0, na = 0, nb = 0;
      PollTimer poll;
      while (ok && nb < nq) {
        bool did = true;
        if (nb < na && mbar_test(ds_full(nb & 1), (uint32_t)(nb >> 1) & 1u)) {
          fence_after();
          mma_tmem_rows<D>(tdK, tB[nb & 1], ring_addr(2 * nb), nb > 0);  // dK += dS^T_i Q_i
          mma_commit(ring_empty(slot(2 * nb)));
          ++nb;
        } else if (na < ns && mbar_test(ring_full(slot(2 * na + 1)), phase(2 * na + 1)) &&
                   mbar_test(p_full(na & 1), (uint32_t)(na >> 1) & 1u)) {
          fence_after();
          mma_tmem_rows<D>(tdV, tB[na & 1], ring_addr(2 * na + 1), na > 0);  // dV += P^T_i dO_i
          mma_rows<D>(tB[na & 1], sV, ring_addr(2 * na + 1));  // dP^T_i = V dO_i^T
          mma_commit(dp_full(na & 1));
          mma_commit(ring_empty(slot(2 * na + 1)));
          ++na;
        } else if (ns < nq && ns <= nb + 1 && mbar_test(ring_full(slot(2 * ns)), phase(2 * ns))) {
          fence_after();
          mma_rows<D>(tB[ns & 1], sK, ring_addr(2 * ns));  // S^T_i = K Q_i^T
          mma_commit(s_full(ns & 1));
          ++ns;
        } else {
          did = false;
        }
        ok = poll.step(did, abort, err, timeout_ns);
      }
      if (ok) mma_commit(acc_done);
      mma_commit(drain);
      drain_wait(drain, 0);
    }
  } else {
    const int g = warp >> 2;                  // warpgroup: query tiles i = g, g+2, ...
    const int row = (warp & 3) * 32 + lane;   // TMEM lane = key of the block
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tb = tmem + lane_base + (g ? 128u : 0u);
    const int key = kt.k0 + row;
    const int k_w = key / P.T;
    float* const my_lse = stat_lse + g * kRowsPerTile;
    float* const my_dlt = stat_dlt + g * kRowsPerTile;
    const int64_t hbase = ((int64_t)b * P.heads + head) * (P.N + P.L);
    // Warpgroup barrier with a bounded wait: a thread that gives up (abort
    // or timeout) cannot strand the others, who see the abort flag.
    uint32_t gphase = 0;
    auto group_sync = [&]() {
      mbar_arrive(group(g));
      const bool r = wait_warp(group(g), gphase & 1u);
      ++gphase;
      return r;
    };
    // Per-query lse (log2 units) and D of a tile, one entry per thread;
    // queries past the tensor get probability 0 and D = 0.  Loaded one tile
    // of this warpgroup ahead, so the load latency is off the critical path.
    auto load_stats = [&](int i, float& l, float& dd) {
      l = __int_as_float(0x7f800000);
      dd = 0.0f;
      if (i < nq) {
        const uint32_t e = P.qlist[kt.list_off + i];
        const bool qlr = (e & kBlockLowres) != 0;
        const int q = (int)(e & kBlockIndexMask) * kRowsPerTile + row;
        if (q < (qlr ? P.L : P.N)) {
          const int64_t ri = hbase + (qlr ? P.N : 0) + q;
          l = P.lse[ri] * kLog2e;
          dd = P.delta[ri];
        }
      }
    };
    float nx_lse, nx_dlt;
    load_stats(g, nx_lse, nx_dlt);
    bool ok = true;
    for (int i = g; i < nq; i += 2) {
      const uint32_t e = P.qlist[kt.list_off + i];
      const uint32_t ph = (uint32_t)(i >> 1) & 1u;
      const int q0 = (int)(e & kBlockIndexMask) * kRowsPerTile;
      if (!(ok = group_sync())) break;  // the previous tile's readers are done
      my_lse[row] = nx_lse;
      my_dlt[row] = nx_dlt;
      load_stats(i + 2, nx_lse, nx_dlt);
      if (!(ok = group_sync())) break;
      if (!(ok = wait_warp(s_full(g), ph))) break;
      fence_after();
      // P^T in two halves of 64 queries (bounded register use); half h
      // writes its 32 bf16-pair columns over S^T columns it has just read.
      uint32_t pk[kRowsPerTile / 2];
      const float2 sc2 = make_float2(P.scale_log2, P.scale_log2);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        float s[64];
        tmem_ld32(tb + 64 * hf, s);
        tmem_ld32(tb + 64 * hf + 32, s + 32);
        tmem_ld_wait();
        if (e & kBlockMasked) mask_windows<64>(s, q0 + 64 * hf, k_w, P);
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const float2 l2 = *reinterpret_cast<const float2*>(my_lse + 64 * hf + c);
          const float2 x =
              __ffma2_rn(make_float2(s[c], s[c + 1]), sc2, make_float2(-l2.x, -l2.y));
          pk[32 * hf + c / 2] = pack_bf16(fast_exp2(x.x), fast_exp2(x.y));
        }
        tmem_st32u(tb + 32 * hf, pk + 32 * hf);
      }
      tmem_st_wait();
      fence_before();
      mbar_arrive(p_full(g));  // P^T in TMEM: dV += P^T dO, then dP^T over it
      if (!(ok = wait_warp(dp_full(g), ph))) break;
      fence_after();
#pragma unroll
      for (int c = 0; c < kRowsPerTile / 32; ++c) {
        float dp[32];
        tmem_ld32(tb + c * 32, dp);
        tmem_ld_wait();
        uint32_t ds[16];
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          const float2 p = unpack_bf16(pk[c * 16 + x / 2]);
          const float2 d2 = *reinterpret_cast<const float2*>(my_dlt + c * 32 + x);
          ds[x / 2] = pack_bf16(p.x * (dp[x] - d2.x), p.y * (dp[x + 1] - d2.y));
        }
        tmem_st16u(tb + c * 16, ds);
      }
      tmem_st_wait();
      fence_before();
      mbar_arrive(ds_full(g));
    }
    if (ok && nq > 0) ok = wait_warp(acc_done, 0);
    if (ok) {
      fence_after();
      // warpgroup 0 writes dV, warpgroup 1 writes dK (scaled)
      bool valid = key < nk;
      // dV of high-res keys goes to its raster row when dV is raster-ordered
      const int orow = (valid && g == 0 && !kt.lowres && P.vo_raster)
                           ? raster_of(key, P.T, P.nwx, P.win_h, P.win_w, P.grid_w)
                           : key;
      if (valid) valid = dbg_ok(orow >= 0 && orow < nk, err);
      __nv_bfloat16* dst = (g == 0 ? (kt.lowres ? P.dv_lr : P.dv_hr) : (kt.lowres ? P.dk_lr : P.dk_hr)) +
                           (((int64_t)b * nk + orow) * P.heads + head) * D;
      const float k = g == 0 ? 1.0f : P.scale;
      const uint32_t tacc = tmem + lane_base + (g == 0 ? 256u : 384u);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        if (nq > 0) {
          tmem_ld32(tacc + c * 32, o);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int x = 0; x < 32; ++x) o[x] = 0.0f;
        }
        if (valid) {
#pragma unroll
          for (int x = 0; x < 32; x += 8)
            *reinterpret_cast<uint4*>(dst + c * 32 + x) =
                make_uint4(pack_bf16(o[x] * k, o[x + 1] * k), pack_bf16(o[x + 2] * k, o[x + 3] * k),
                           pack_bf16(o[x + 4] * k, o[x + 5] * k), pack_bf16(o[x + 6] * k, o[x + 7] * k));
        }
      }
    }
  }

  fence_before();
  __syncthreads();
  if (warp == kBwdMma) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

// ------------------------------------------------------------------ host side

template <int D>
int launch_bwd_d(const ug_plan* p, const void* q_hr, const void* k_hr, const void* v_hr,
                 const void* q_lr, const void* k_lr, const void* v_lr, const void* o_hr,
                 const void* o_lr, const void* do_hr, const void* do_lr, const float* lse,
                 void* dq_hr, void* dk_hr, void* dv_hr, void* dq_lr, void* dk_lr, void* dv_lr,
                 float* delta, bool vo_raster, cudaStream_t st) {
  const int64_t B = p->g.batch;
  const int H = p->g.heads;
  const bool has_lr = p->L > 0;
  const int64_t nl = has_lr ? p->L : p->N;
  CUtensorMap m[8];  // q, k, v, do (high-res), then the same for the global set
  const void* hr[4] = {q_hr, k_hr, v_hr, do_hr};
  const void* lr[4] = {has_lr ? q_lr : q_hr, has_lr ? k_lr : k_hr, has_lr ? v_lr : v_hr,
                       has_lr ? do_lr : do_hr};
  for (int i = 0; i < 4; ++i) {
    const bool ok_hr = (vo_raster && i >= 2)
                           ? make_map_raster(&m[i], hr[i], B, p->g.grid_h, p->g.grid_w, H, D,
                                             p->g.win_w)
                           : make_map(&m[i], hr[i], B, p->N, H, D);
    if (!ok_hr || !make_map(&m[4 + i], lr[i], B, nl, H, D)) return UG_ERR_CUDA;
  }
  BwdParams P;
  P.qtiles = p->d_qtiles;
  P.kvlist = p->d_kvlist;
  P.ktiles = p->d_ktiles;
  P.qlist = p->d_qlist;
  P.lse = lse;
  P.delta = delta;
  P.dq_hr = static_cast<__nv_bfloat16*>(dq_hr);
  P.dk_hr = static_cast<__nv_bfloat16*>(dk_hr);
  P.dv_hr = static_cast<__nv_bfloat16*>(dv_hr);
  P.dq_lr = static_cast<__nv_bfloat16*>(dq_lr);
  P.dk_lr = static_cast<__nv_bfloat16*>(dk_lr);
  P.dv_lr = static_cast<__nv_bfloat16*>(dv_lr);
  P.err = p->d_err;
  P.timeout_ns = p->wait_timeout_ns;
  P.N = (int32_t)p->N;
  P.L = (int32_t)p->L;
  P.T = (int32_t)p->T;
  P.nwx = p->nwx;
  P.radius = p->g.radius;
  P.heads = H;
  P.scale = p->scale;
  P.scale_log2 = p->scale * kLog2e;
  P.kv_len = (int32_t)p->kvlist.size();
  P.q_len = (int32_t)p->qlist.size();
  P.vo_raster = vo_raster ? 1 : 0;
  P.grid_w = p->g.grid_w;
  P.win_h = p->g.win_h;
  P.win_w = p->g.win_w;
  if (const int pst = prepare_attention_bwd(p->device)) return pst;
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, p->device);
  const int64_t rows = B * (p->N + p->L);
  const int dblocks = (int)std::min<int64_t>((rows + 7) / 8, (int64_t)sms * 16);
  delta_kernel<D><<<dblocks, 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(o_hr), static_cast<const __nv_bfloat16*>(do_hr),
      static_cast<const __nv_bfloat16*>(has_lr ? o_lr : o_hr),
      static_cast<const __nv_bfloat16*>(has_lr ? do_lr : do_hr), delta, (int)B, (int)p->N,
      (int)p->L, H, vo_raster ? 1 : 0, (int)p->T, p->nwx, p->g.win_h, p->g.win_w, p->g.grid_w);
  const dim3 gq((unsigned)(2 * p->qtiles.size()), (unsigned)H, (unsigned)B);
  dq_kernel<D><<<gq, kBwdThreads, DqLayout<D>::kAlloc, st>>>(m[0], m[1], m[2], m[3], m[4], m[5],
                                                             m[6], m[7], P);
  const dim3 gk((unsigned)p->ktiles.size(), (unsigned)H, (unsigned)B);
  dkv_kernel<D><<<gk, kBwdThreads, DkvLayout<D>::kAlloc, st>>>(m[0], m[1], m[2], m[3], m[4], m[5],
                                                               m[6], m[7], P);
  return cudaGetLastError() == cudaSuccess ? UG_OK : UG_ERR_CUDA;
}

PerDevice<char> g_bwd_ready;

}  // namespace

// The dQ and dK/dV kernels need more than 48 KB of dynamic shared memory, an
// opt-in that is per device; done once per device (ug_plan_create calls this).
int prepare_attention_bwd(int device) {
  return g_bwd_ready.get(device, [](char&) {
    const bool ok =
        cudaFuncSetAttribute(dq_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DqLayout<128>::kAlloc) == cudaSuccess &&
        cudaFuncSetAttribute(dkv_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DkvLayout<128>::kAlloc) == cudaSuccess &&
        cudaFuncSetAttribute(dq_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DqLayout<64>::kAlloc) == cudaSuccess &&
        cudaFuncSetAttribute(dkv_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DkvLayout<64>::kAlloc) == cudaSuccess;
    if (!ok) cudaGetLastError();
    return ok ? UG_OK : UG_ERR_CUDA;
  });
}

int launch_attention_bwd(const ug_plan* p, const void* q_hr, const void* k_hr, const void* v_hr,
                         const void* q_lr, const void* k_lr, const void* v_lr, const void* o_hr,
                         const void* o_lr, const void* do_hr, const void* do_lr, const float* lse,
                         void* dq_hr, void* dk_hr, void* dv_hr, void* dq_lr, void* dk_lr,
                         void* dv_lr, float* delta, bool vo_raster, cudaStream_t st) {
  if (p->g.head_dim == 128)
    return launch_bwd_d<128>(p, q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, o_hr, o_lr, do_hr, do_lr, lse,
                             dq_hr, dk_hr, dv_hr, dq_lr, dk_lr, dv_lr, delta, vo_raster, st);
  if (p->g.head_dim == 64)
    return launch_bwd_d<64>(p, q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, o_hr, o_lr, do_hr, do_lr, lse,
                            dq_hr, dk_hr, dv_hr, dq_lr, dk_lr, dv_lr, delta, vo_raster, st);
  return UG_ERR_UNSUPPORTED;
}

}  // namespace ug
