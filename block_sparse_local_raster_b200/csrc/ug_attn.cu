// Block-sparse joint-softmax attention of the hierarchical local attention
// layer on B200 (sm_100a): tcgen05 MMA with TMEM accumulators, TMA loads,
// mbarrier pipeline, warp specialisation.
//
// What it computes (UltraGen-ar §2.ب "Attention Masking"; UltraGen-es §2,
// guidance item; UltraGen-it §2): a high-res query of window w attends, under
// one softmax, to the high-res keys of every window within Chebyshev distance
// `radius` of w and to every low-res key; a low-res query attends to the
// low-res keys only.  High-res tensors arrive window-first (UltraGen-fr §2.A),
// so a window is a contiguous run of keys and the mask is block structured:
// a host-built list names, per 256-row query CTA, the 128-key blocks that
// hold visible keys (every other block is never loaded), and flags the few
// blocks that need a per-pair test (ragged ends, windows that straddle a
// block).
//
// CTA layout (320 threads):
//   warps 0-3  softmax for query tile 0 (rows 0..127 of the CTA)
//   warps 4-7  softmax for query tile 1 (rows 128..255)
//   warp 8     TMA producer: Q once, then K_j, V_j into a 5-slot ring
//   warp 9     TMEM allocation and the tcgen05.mma issuer
// TMEM (512 columns x 128 lanes x 32 bit): S0 [0,128) S1 [128,256)
//   O0 [256, 256+D) O1 [384, 384+D).  One TMEM lane = one query row, so the
//   row max and row sum are in-thread.  The softmax writes the bf16
//   probabilities P_t over the first 64 columns of S_t, and O_t += P_t V_j
//   reads its A operand straight from TMEM: P never touches shared memory,
//   which leaves shared-memory bandwidth to the tensor pipe's Q, K and V reads
//   and the TMA writes.
// Pipeline: per key block j the MMA warp issues
//   O0 += P0(j) V_j, S0(j+1) = Q0 K_{j+1}^T, O1 += P1(j) V_j, S1(j+1) = ...
// so one tile's softmax runs while the tensor pipe works on the other tile;
// the tensor pipe executes in issue order, so S_t(j+1) overwrites P_t(j) only
// after O_t += P_t(j) V_j has read it, and the commit that signals S_t(j+1)
// also covers that product (the softmax never waits for O separately).
// P_t is handed over in two halves (keys 0-63, then 64-127), so the first
// half of O_t += P_t V_j runs while the softmax computes the second; each
// softmax warp arrives once per half, after its own stores are complete.
// Online softmax in the log2 domain with lazy rescaling: the running
// reference max moves (and O, l are rescaled) only when a block's max exceeds
// it by more than 8 (a factor 256), so probabilities stay <= 256 and O is
// rarely touched.
//
// Every wait is bounded (globaltimer); on expiry a thread records
// UG_ERR_TIMEOUT in the plan's error word, raises a CTA-wide abort flag and
// every role unwinds: the producer waits (bounded) for its loads in flight,
// the MMA warp for its MMAs, then TMEM is freed and the CTA exits.
#include <cstdint>
#include <cstring>

#include <cuda.h>
#include <cuda_bf16.h>

#include "ug_debug.h"
#include "ug_internal.h"
#include "ug_per_device.h"
#include "ug_tc.cuh"

namespace ug {
namespace {

constexpr int kThreads = 320;
constexpr int kStages = 5;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct Layout {
  static constexpr int kTileBytes = kRowsPerTile * D * 2;     // Q tile, K or V tile
  static constexpr int kQ = 0;
  static constexpr int kKV = kQ + kTilesPerCta * kTileBytes;
  static constexpr int kBar = kKV + kStages * kTileBytes;
  // barriers: q_full, kv_full[S], kv_empty[S], s_full[2], p_full[2], o_done[2], drain,
  // p_half[2]
  static constexpr int kNumBars = 1 + 2 * kStages + 4 * kTilesPerCta + 1;
  static constexpr int kMisc = kBar + kNumBars * 8;  // tmem base (u32), abort flag (u32)
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
};

struct AttnParams {
  const QTile* qtiles;
  const uint32_t* kvlist;
  __nv_bfloat16* o_hr;
  __nv_bfloat16* o_lr;
  float* lse;
  int* err;
  int64_t timeout_ns;
  int32_t N, L, T, nwx, radius, heads;
  float scale_log2;  // softmax scale * log2(e)
  // Raster-order high-res V (read through a 5-D tensor map, one 128-key
  // tile = 128 / win_w whole rows of one window) and raster-order o_hr.
  int32_t vo_raster;
  int32_t grid_w, win_h, win_w;
  int32_t kv_len;  // entries in kvlist (debug-build range checks)
};

// Raster index of the high-res token at window-first position p.
__device__ __forceinline__ int raster_of(int p, const AttnParams& P) {
  const int w = p / P.T, l = p - (p / P.T) * P.T;
  const int wy = w / P.nwx, wx = w - (w / P.nwx) * P.nwx;
  const int ly = l / P.win_w, lx = l - (l / P.win_w) * P.win_w;
  return (wy * P.win_h + ly) * P.grid_w + wx * P.win_w + lx;
}

// ---------------------------------------------------------------- the kernel

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    hier_attn_kernel(const __grid_constant__ CUtensorMap tm_q_hr,
                     const __grid_constant__ CUtensorMap tm_k_hr,
                     const __grid_constant__ CUtensorMap tm_v_hr,
                     const __grid_constant__ CUtensorMap tm_q_lr,
                     const __grid_constant__ CUtensorMap tm_k_lr,
                     const __grid_constant__ CUtensorMap tm_v_lr, const AttnParams P) {
  using Lay = Layout<D>;
  constexpr int kRegions = D / 64;  // 128-byte swizzle spans 64 bf16 columns
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + Lay::kBar;
  const uint32_t q_full = bar0;
  auto kv_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto kv_empty = [&](int s) { return bar0 + 8u * (1 + kStages + s); };
  auto s_full = [&](int t) { return bar0 + 8u * (1 + 2 * kStages + t); };
  auto p_full = [&](int t) { return bar0 + 8u * (1 + 2 * kStages + 2 + t); };
  auto o_done = [&](int t) { return bar0 + 8u * (1 + 2 * kStages + 4 + t); };
  const uint32_t drain = bar0 + 8u * (1 + 2 * kStages + 6);
  auto p_half = [&](int t) { return bar0 + 8u * (1 + 2 * kStages + 7 + t); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMisc);
  volatile uint32_t* abort = reinterpret_cast<volatile uint32_t*>(smem + Lay::kMisc + 4);
  int* const err = P.err;
  const int64_t timeout_ns = P.timeout_ns;
  // Single-thread roles wait alone; the softmax warps agree on the outcome so
  // that the warp-collective tcgen05 loads that follow never run diverged.
  auto wait1 = [&](uint32_t bar, uint32_t par) {
    return mbar_wait(bar, par, abort, err, timeout_ns, false);
  };
  // Draining (loads and MMAs already in flight) always gets the full bound,
  // whatever the plan's wait limit: TMEM and shared memory are released only
  // after the asynchronous units are done with them.
  auto drain_wait = [&](uint32_t bar, uint32_t par) {
    return mbar_wait(bar, par, abort, err, kDefaultWaitTimeoutNs, true);
  };
  auto wait_warp = [&](uint32_t bar, uint32_t par) {
    return __all_sync(0xFFFFFFFFu, mbar_wait(bar, par, abort, err, timeout_ns, false)) != 0;
  };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const QTile qt = P.qtiles[blockIdx.x];
  const int head = blockIdx.y;
  const int b = blockIdx.z;
  const int nblk = qt.list_len;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    for (int t = 0; t < kTilesPerCta; ++t) {
      mbar_init(s_full(t), 1);
      mbar_init(p_half(t), 4);  // one arrive per softmax warp of the tile
      mbar_init(p_full(t), 4);
      mbar_init(o_done(t), 1);
    }
    mbar_init(drain, 1);
    // A CTA that starts after another one gave up does no work.
    *abort = *reinterpret_cast<volatile int*>(err) != 0 ? 1u : 0u;
#if UG_DEBUG
    // the CTA's slice of the block list, and every block in it, in range
    bool lst = qt.list_off >= 0 && qt.list_len >= 1 && qt.list_off + qt.list_len <= P.kv_len;
    for (int j = 0; lst && j < nblk; ++j) {
      const uint32_t e = P.kvlist[qt.list_off + j];
      const int n = (e & kBlockLowres) ? P.L : P.N;
      lst = (int64_t)(e & kBlockIndexMask) * kKeysPerBlock < n;
    }
    const int ntq = qt.lowres ? P.L : P.N;
    if (!dbg_ok(lst && qt.q0 >= 0 && qt.q0 < ntq, err)) *abort = 1u;
#endif
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     smem_u32(tmem_slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_map(&tm_q_hr);
    prefetch_map(&tm_k_hr);
    prefetch_map(&tm_v_hr);
    if (P.L > 0) {
      prefetch_map(&tm_q_lr);
      prefetch_map(&tm_k_lr);
      prefetch_map(&tm_v_lr);
    }
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool skip = *abort != 0u;

  if (skip) {
    // nothing issued: fall through to the teardown
  } else if (warp == kProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const CUtensorMap* mq = qt.lowres ? &tm_q_lr : &tm_q_hr;
      mbar_expect_tx(q_full, kTilesPerCta * Lay::kTileBytes);
      for (int t = 0; t < kTilesPerCta; ++t)
        for (int r = 0; r < kRegions; ++r)
          tma_load_4d(sbase + Lay::kQ + t * Lay::kTileBytes + r * kRowsPerTile * 128, mq, r * 64,
                      head, qt.q0 + t * kRowsPerTile, b, q_full);
      // K_j then V_j, block after block: the order the MMA warp consumes them.
      int it = 0;
      bool ok = true;
      for (int j = 0; j < nblk && ok; ++j) {
        const uint32_t e = P.kvlist[qt.list_off + j];
        const bool lr = (e & kBlockLowres) != 0;
        const int k0 = (int)(e & kBlockIndexMask) * kKeysPerBlock;
        for (int kv = 0; kv < 2 && ok; ++kv, ++it) {
          const CUtensorMap* m = kv == 0 ? (lr ? &tm_k_lr : &tm_k_hr) : (lr ? &tm_v_lr : &tm_v_hr);
          const int s = it % kStages;
          const uint32_t ph = (uint32_t)(it / kStages) & 1u;
          if (!wait1(kv_empty(s), ph ^ 1u)) {
            ok = false;
            break;
          }
          mbar_expect_tx(kv_full(s), Lay::kTileBytes);
          if (kv == 1 && !lr && P.vo_raster) {
            // the block's keys are 128 / win_w whole rows of one window
            const int w = k0 / P.T, ly0 = (k0 - (k0 / P.T) * P.T) / P.win_w;
            const int wy = w / P.nwx, wx = w - (w / P.nwx) * P.nwx;
            for (int r = 0; r < kRegions; ++r)
              tma_load_5d(sbase + Lay::kKV + s * Lay::kTileBytes + r * kKeysPerBlock * 128, m,
                          r * 64, head, wx * P.win_w, wy * P.win_h + ly0, b, kv_full(s));
          } else {
            for (int r = 0; r < kRegions; ++r)
              tma_load_4d(sbase + Lay::kKV + s * Lay::kTileBytes + r * kKeysPerBlock * 128, m,
                          r * 64, head, k0, b, kv_full(s));
          }
        }
      }
      // Loads still in flight land before the CTA may exit.  The last
      // kStages loads each own a distinct slot, and no later phase of that
      // slot exists, so waiting for that phase is unambiguous.
      for (int i = (it > kStages ? it - kStages : 0); i < it; ++i)
        drain_wait(kv_full(i % kStages), (uint32_t)(i / kStages) & 1u);
      drain_wait(q_full, 0);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = instr_desc(kKeysPerBlock, false);
      constexpr uint32_t kIdO = instr_desc(D, true);
      const uint32_t tS[2] = {tmem + 0u, tmem + 128u};
      const uint32_t tO[2] = {tmem + 256u, tmem + 256u + 128u};
      auto issue_s = [&](int t, int slot) {
        const uint32_t qa = sbase + Lay::kQ + t * Lay::kTileBytes;
        const uint32_t ka = sbase + Lay::kKV + slot * Lay::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * (kRowsPerTile * 128) + (kk % 4) * 32;
          mma_bf16(tS[t], smem_desc(qa + off, 16, 1024), smem_desc(ka + off, 16, 1024), kIdS,
                   kk > 0);
        }
      };
      // O_t += P_t V over keys [16 kk0, 16 kk1): P_t (bf16, 128 x 128) sits in
      // the first 64 columns of S_t, 16 keys per 8 columns; V (keys x D, D
      // contiguous) is MN-major.
      auto issue_pv = [&](int t, int slot, bool acc, int kk0, int kk1) {
        const uint32_t va = sbase + Lay::kKV + slot * Lay::kTileBytes;
#pragma unroll
        for (int kk = kk0; kk < kk1; ++kk)
          mma_bf16_tmem_a(tO[t], tS[t] + kk * 8, smem_desc(va + kk * 16 * 128, kKeysPerBlock * 128, 1024),
                          kIdO, (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = wait1(q_full, 0);
      if (ok) ok = wait1(kv_full(0), 0);
      if (ok) {
        fence_after();
        issue_s(0, 0);
        mma_commit(s_full(0));
        issue_s(1, 0);
        mma_commit(s_full(1));
        mma_commit(kv_empty(0));
      }
      for (int j = 0; j < nblk && ok; ++j) {
        const int itv = 2 * j + 1, itk = 2 * j + 2;
        const int sv = itv % kStages, sk = itk % kStages;
        const bool more = j + 1 < nblk;
        if (!(ok = wait1(kv_full(sv), (uint32_t)(itv / kStages) & 1u))) break;
        if (!(ok = wait1(p_half(0), (uint32_t)j & 1u))) break;
        fence_after();
        issue_pv(0, sv, j > 0, 0, kKeysPerBlock / 32);
        if (!(ok = wait1(p_full(0), (uint32_t)j & 1u))) break;
        fence_after();
        issue_pv(0, sv, true, kKeysPerBlock / 32, kKeysPerBlock / 16);
        if (!more) mma_commit(o_done(0));
        if (more) {
          if (!(ok = wait1(kv_full(sk), (uint32_t)(itk / kStages) & 1u))) break;
          fence_after();
          issue_s(0, sk);
          mma_commit(s_full(0));
        }
        if (!(ok = wait1(p_half(1), (uint32_t)j & 1u))) break;
        fence_after();
        issue_pv(1, sv, j > 0, 0, kKeysPerBlock / 32);
        if (!(ok = wait1(p_full(1), (uint32_t)j & 1u))) break;
        fence_after();
        issue_pv(1, sv, true, kKeysPerBlock / 32, kKeysPerBlock / 16);
        if (!more) mma_commit(o_done(1));
        mma_commit(kv_empty(sv));
        if (more) {
          issue_s(1, sk);
          mma_commit(s_full(1));
          mma_commit(kv_empty(sk));
        }
      }
      // Every MMA issued above completes before TMEM may be freed.
      mma_commit(drain);
      drain_wait(drain, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int t = warp >> 2;               // query tile
    const int row = (warp & 3) * 32 + lane;  // TMEM lane = row in tile
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + (t ? 128u : 0u);
    const uint32_t tO = tmem + lane_base + 256u + (t ? 128u : 0u);
    const int tok = qt.q0 + t * kRowsPerTile + row;  // query token in its tensor
    const int q_w = tok / P.T;
    const int q_wy = q_w / P.nwx, q_wx = q_w - (q_w / P.nwx) * P.nwx;
    // This warp's probability stores complete and ordered before the MMA
    // warp's reads: wait for them, fence, then one arrive for the warp.
    auto hand_over = [&](uint32_t bar) {
      tmem_st_wait();
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
    };
    float m_ref = kNegInf;  // reference max (log2 units) of the O/l accumulators
    float l = 0.0f;
    bool ok = true;
    for (int j = 0; j < nblk; ++j) {
      const uint32_t e = P.kvlist[qt.list_off + j];
      // S_t(j) complete; the commit that signals it also covers every earlier
      // MMA of this CTA, in particular O_t += P_t(j-1) V_{j-1}.
      if (!(ok = wait_warp(s_full(t), (uint32_t)j & 1u))) break;
      fence_after();
      float s[kKeysPerBlock];
#pragma unroll
      for (int c = 0; c < kKeysPerBlock / 32; ++c) tmem_ld32(tS + c * 32, s + c * 32);
      tmem_ld_wait();
      if (e & kBlockMasked) {
        const int k0 = (int)(e & kBlockIndexMask) * kKeysPerBlock;
        if (e & kBlockLowres) {
#pragma unroll
          for (int i = 0; i < kKeysPerBlock; ++i)
            if (k0 + i >= P.L) s[i] = kNegInf;
        } else {
          // Visibility changes only at window boundaries: test each key
          // window met in the block once, then mask its run of keys.
          int i0 = 0;
          while (i0 < kKeysPerBlock) {
            const int k = k0 + i0;
            const int kw = k / P.T;
            const int run = min(kKeysPerBlock, (kw + 1) * P.T - k0);
            const int kwy = kw / P.nwx, kwx = kw - (kw / P.nwx) * P.nwx;
            const bool vis = abs(kwy - q_wy) <= P.radius && abs(kwx - q_wx) <= P.radius;
            const int lim = vis ? min(run, P.N - k0) : i0;  // keys [i0, lim) stay
#pragma unroll
            for (int i = 0; i < kKeysPerBlock; ++i)
              if (i >= i0 && i < run && i >= lim) s[i] = kNegInf;
            i0 = run;
          }
        }
      }
      // Row max: four independent chains of three-input maxima.
      float mc[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) mc[c] = fmaxf(s[2 * c], s[2 * c + 1]);
#pragma unroll
      for (int i = 8; i < kKeysPerBlock; i += 8) {
#pragma unroll
        for (int c = 0; c < 4; ++c) mc[c] = fmax3(mc[c], s[i + 2 * c], s[i + 2 * c + 1]);
      }
      const float mx = fmax3(fmaxf(mc[0], mc[1]), mc[2], mc[3]);
      const float m_blk = mx * P.scale_log2;
      const bool rescale = m_blk > m_ref + kRescaleThreshold;
      const float m_new = rescale ? m_blk : m_ref;
      const float alpha = rescale ? fast_exp2(m_ref - m_new) : 1.0f;
      const float m_use = m_new == kNegInf ? 0.0f : m_new;
      m_ref = m_new;
      if (j > 0 && __any_sync(0xFFFFFFFFu, rescale)) {
#pragma unroll 1
        for (int c = 0; c < D / 16; ++c) {
          float o[16];
          tmem_ld16(tO + c * 16, o);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] *= alpha;
          tmem_st16(tO + c * 16, o);
        }
      }
      // p = 2^(s*scale*log2e - m): fp32 row sum; bf16 pairs (even key in the
      // low half) over the first 64 columns of S_t, the A operand of O += P V,
      // stored 8 columns at a time so that few packed values are live next to
      // the 128 scores (no register spills).
      const float2 sc2 = make_float2(P.scale_log2, P.scale_log2);
      const float2 nm2 = make_float2(-m_use, -m_use);
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                       make_float2(0.f, 0.f)};
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        uint32_t pk[8];
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
          const int k = 16 * h + i;
          const float2 x = __ffma2_rn(make_float2(s[k], s[k + 1]), sc2, nm2);
          const float2 pp = make_float2(fast_exp2(x.x), fast_exp2(x.y));
          acc[(k / 2) & 3] = __fadd2_rn(acc[(k / 2) & 3], pp);
          pk[i / 2] = pack_bf16(pp.x, pp.y);
        }
        tmem_st8u(tS + 8 * h, pk);
        if (h == kKeysPerBlock / 32 - 1) hand_over(p_half(t));  // keys 0-63 stored
      }
      const float2 a4 = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
      l = l * alpha + (a4.x + a4.y);
      hand_over(p_full(t));
    }
    // ------------------------------------------------------------ epilogue
    if (ok) ok = wait_warp(o_done(t), 0);
    if (ok) {
      fence_after();
      const int ntok = qt.lowres ? P.L : P.N;
      bool valid = tok < ntok;
      const float inv_l = 1.0f / l;
      const int orow = (!qt.lowres && P.vo_raster && valid) ? raster_of(tok, P) : tok;
      if (valid) valid = dbg_ok(orow >= 0 && orow < ntok, err);
      __nv_bfloat16* dst = (qt.lowres ? P.o_lr : P.o_hr) +
                           (((int64_t)b * ntok + orow) * P.heads + head) * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        tmem_ld32(tO + c * 32, o);
        tmem_ld_wait();
        if (valid) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 v = make_uint4(pack_bf16(o[i] * inv_l, o[i + 1] * inv_l),
                                 pack_bf16(o[i + 2] * inv_l, o[i + 3] * inv_l),
                                 pack_bf16(o[i + 4] * inv_l, o[i + 5] * inv_l),
                                 pack_bf16(o[i + 6] * inv_l, o[i + 7] * inv_l));
            *reinterpret_cast<uint4*>(dst + c * 32 + i) = v;
          }
        }
      }
      if (valid && P.lse) {
        const float lse = (m_ref + __log2f(l)) * 0.69314718055994531f;
        P.lse[((int64_t)b * P.heads + head) * (P.N + P.L) + (qt.lowres ? P.N : 0) + tok] = lse;
      }
    }
  }

  fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

// ---------------------------------------------------------------- host side

template <int D>
int launch_d(const ug_plan* p, const void* q_hr, const void* k_hr, const void* v_hr,
             const void* q_lr, const void* k_lr, const void* v_lr, void* o_hr, void* o_lr,
             float* lse, bool vo_raster, cudaStream_t st) {
  const int64_t B = p->g.batch;
  const int H = p->g.heads;
  CUtensorMap m[6];
  const void* lrs[3] = {q_lr ? q_lr : q_hr, k_lr ? k_lr : k_hr, v_lr ? v_lr : v_hr};
  const int64_t nl = p->L > 0 ? p->L : p->N;
  const bool vmap = vo_raster ? make_map_raster(&m[2], v_hr, B, p->g.grid_h, p->g.grid_w, H, D,
                                                p->g.win_w)
                              : make_map(&m[2], v_hr, B, p->N, H, D);
  if (!make_map(&m[0], q_hr, B, p->N, H, D) || !make_map(&m[1], k_hr, B, p->N, H, D) || !vmap ||
      !make_map(&m[3], lrs[0], B, nl, H, D) || !make_map(&m[4], lrs[1], B, nl, H, D) ||
      !make_map(&m[5], lrs[2], B, nl, H, D))
    return UG_ERR_CUDA;
  AttnParams P;
  P.qtiles = p->d_qtiles;
  P.kvlist = p->d_kvlist;
  P.o_hr = static_cast<__nv_bfloat16*>(o_hr);
  P.o_lr = static_cast<__nv_bfloat16*>(o_lr);
  P.lse = lse;
  P.err = p->d_err;
  P.timeout_ns = p->wait_timeout_ns;
  P.N = (int32_t)p->N;
  P.L = (int32_t)p->L;
  P.T = (int32_t)p->T;
  P.nwx = p->nwx;
  P.radius = p->g.radius;
  P.heads = H;
  P.scale_log2 = p->scale * 1.4426950408889634f;
  P.vo_raster = vo_raster ? 1 : 0;
  P.grid_w = p->g.grid_w;
  P.win_h = p->g.win_h;
  P.win_w = p->g.win_w;
  P.kv_len = (int32_t)p->kvlist.size();
  if (const int pst = prepare_attention(p->device)) return pst;
  const dim3 grid((unsigned)p->qtiles.size(), (unsigned)H, (unsigned)B);
  hier_attn_kernel<D><<<grid, kThreads, Layout<D>::kAlloc, st>>>(m[0], m[1], m[2], m[3], m[4],
                                                                  m[5], P);
  return cudaGetLastError() == cudaSuccess ? UG_OK : UG_ERR_CUDA;
}

PerDevice<char> g_attn_ready;

}  // namespace

// The kernels need more than 48 KB of dynamic shared memory, an opt-in that
// is per device; done once per device (ug_plan_create calls this).
int prepare_attention(int device) {
  return g_attn_ready.get(device, [](char&) {
    const bool ok = cudaFuncSetAttribute(hier_attn_kernel<128>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Layout<128>::kAlloc) == cudaSuccess &&
                    cudaFuncSetAttribute(hier_attn_kernel<64>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Layout<64>::kAlloc) == cudaSuccess;
    if (!ok) cudaGetLastError();
    return ok ? UG_OK : UG_ERR_CUDA;
  });
}

int launch_attention(const ug_plan* p, const void* q_hr, const void* k_hr, const void* v_hr,
                     const void* q_lr, const void* k_lr, const void* v_lr, void* o_hr,
                     void* o_lr, float* lse, bool vo_raster, cudaStream_t st) {
  if (p->g.head_dim == 128)
    return launch_d<128>(p, q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, o_hr, o_lr, lse, vo_raster, st);
  if (p->g.head_dim == 64)
    return launch_d<64>(p, q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, o_hr, o_lr, lse, vo_raster, st);
  return UG_ERR_UNSUPPORTED;
}

bool vo_raster_supported(const ug_geom& g) {
  const int64_t T = (int64_t)g.win_h * g.win_w;
  return g.win_w <= kRowsPerTile && kRowsPerTile % g.win_w == 0 && T % kRowsPerTile == 0;
}

}  // namespace ug
