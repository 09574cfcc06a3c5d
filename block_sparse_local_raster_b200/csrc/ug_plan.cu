// Host side of the plan: geometry checks, index maps, attention work lists,
// RoPE tables.  Nothing here touches the GPU.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <set>
#include <vector>

#include "ug_internal.h"
#include "ug_rope_math.h"

namespace ug {

int validate(const ug_geom* g) {
  if (!g) return UG_ERR_INVALID_ARG;
  if (g->batch < 1 || g->grid_h < 1 || g->grid_w < 1 || g->win_h < 1 || g->win_w < 1 ||
      g->heads < 1 || g->head_dim < 2 || g->radius < 0 || g->lr_h < 0 || g->lr_w < 0 ||
      g->text_len < 0)
    return UG_ERR_INVALID_ARG;
  // Fixed non-overlapping windows that tile the grid; no padding.
  if (g->grid_h % g->win_h || g->grid_w % g->win_w) return UG_ERR_INVALID_ARG;
  if ((g->lr_h == 0) != (g->lr_w == 0)) return UG_ERR_INVALID_ARG;
  if (!(g->rho > 0.0) || !(g->rope_theta > 1.0) || !(g->softmax_scale >= 0.0f))
    return UG_ERR_INVALID_ARG;
  if (g->rope_dim_y < 0 || g->rope_dim_x < 0 || g->rope_dim_y + g->rope_dim_x != g->head_dim ||
      g->rope_dim_y % 8 || g->rope_dim_x % 8)
    return UG_ERR_INVALID_ARG;
  const int64_t row = (int64_t)g->heads * g->head_dim;
  const int64_t n = (int64_t)g->grid_h * g->grid_w;
  const int64_t l = global_tokens(*g);
  if (row * 2 % 16) return UG_ERR_UNSUPPORTED;
  if ((int64_t)g->batch * n * row >= (1ll << 31) || (int64_t)g->batch * l * row >= (1ll << 31))
    return UG_ERR_INVALID_ARG;
  if ((n + kKeysPerBlock - 1) / kKeysPerBlock > (int64_t)kBlockIndexMask) return UG_ERR_UNSUPPORTED;
  return UG_OK;
}

void build_perm(const ug_geom& g, std::vector<int32_t>& perm) {
  const int64_t W = g.grid_w, nwx = g.grid_w / g.win_w, T = (int64_t)g.win_h * g.win_w;
  perm.resize((size_t)g.grid_h * g.grid_w);
  for (int64_t y = 0; y < g.grid_h; ++y) {
    const int64_t wy = y / g.win_h, ly = y % g.win_h;
    for (int64_t x = 0; x < W; ++x) {
      const int64_t wx = x / g.win_w, lx = x % g.win_w;
      perm[(size_t)(y * W + x)] = (int32_t)((wy * nwx + wx) * T + ly * g.win_w + lx);
    }
  }
}

void build_neighbours(const ug_geom& g, std::vector<int32_t>& off, std::vector<int32_t>& idx) {
  const int nwy = g.grid_h / g.win_h, nwx = g.grid_w / g.win_w, r = g.radius;
  off.assign(1, 0);
  idx.clear();
  for (int wy = 0; wy < nwy; ++wy)
    for (int wx = 0; wx < nwx; ++wx) {
      for (int vy = std::max(0, wy - r); vy <= std::min(nwy - 1, wy + r); ++vy)
        for (int vx = std::max(0, wx - r); vx <= std::min(nwx - 1, wx + r); ++vx)
          idx.push_back(vy * nwx + vx);
      off.push_back((int32_t)idx.size());
    }
}

// Per query CTA (256 rows), the 128-key blocks holding at least one key that
// some row of the CTA may see.  The global tokens (text, then low-res) form
// one key set that every query sees.  A block is "full" when every valid row of the
// CTA sees every key of the block (then the kernel skips per-pair tests).
void build_attention_lists(const ug_geom& g, const std::vector<int32_t>& nbr_off,
                           const std::vector<int32_t>& nbr_idx, std::vector<QTile>& qtiles,
                           std::vector<uint32_t>& kvlist, int32_t* n_hr_ctas,
                           int32_t* n_lr_ctas) {
  const int64_t N = (int64_t)g.grid_h * g.grid_w, L = global_tokens(g);
  const int64_t T = (int64_t)g.win_h * g.win_w;
  const int nwx = g.grid_w / g.win_w;
  const int64_t BK = kKeysPerBlock;
  qtiles.clear();
  kvlist.clear();
  const int64_t n_lr_blocks = (L + BK - 1) / BK;
  auto near = [&](int64_t a, int64_t b) {  // window ids
    return std::llabs(a / nwx - b / nwx) <= g.radius && std::llabs(a % nwx - b % nwx) <= g.radius;
  };
  auto add_lowres_blocks = [&]() {
    for (int64_t kb = 0; kb < n_lr_blocks; ++kb)
      kvlist.push_back((uint32_t)kb | kBlockLowres | ((kb + 1) * BK > L ? kBlockMasked : 0u));
  };
  int32_t nhr = 0;
  for (int64_t q0 = 0; q0 < N; q0 += kRowsPerCta, ++nhr) {
    const int64_t q1 = std::min(N, q0 + kRowsPerCta);
    const int64_t w0 = q0 / T, w1 = (q1 - 1) / T;  // query windows [w0, w1]
    std::set<int64_t> blocks;
    for (int64_t w = w0; w <= w1; ++w)
      for (int32_t e = nbr_off[(size_t)w]; e < nbr_off[(size_t)w + 1]; ++e) {
        const int64_t v = nbr_idx[(size_t)e];
        for (int64_t kb = v * T / BK; kb <= (v * T + T - 1) / BK; ++kb) blocks.insert(kb);
      }
    QTile t;
    t.lowres = 0;
    t.q0 = (int32_t)q0;
    t.list_off = (int32_t)kvlist.size();
    for (int64_t kb : blocks) {
      const int64_t k0 = kb * BK, k1 = std::min(N, k0 + BK);
      bool full = (k0 + BK <= N);
      for (int64_t kw = k0 / T; full && kw <= (k1 - 1) / T; ++kw)
        for (int64_t w = w0; full && w <= w1; ++w) full = near(w, kw);
      kvlist.push_back((uint32_t)kb | (full ? 0u : kBlockMasked));
    }
    add_lowres_blocks();
    t.list_len = (int32_t)kvlist.size() - t.list_off;
    qtiles.push_back(t);
  }
  int32_t nlr = 0;
  for (int64_t q0 = 0; q0 < L; q0 += kRowsPerCta, ++nlr) {
    QTile t;
    t.lowres = 1;
    t.q0 = (int32_t)q0;
    t.list_off = (int32_t)kvlist.size();
    add_lowres_blocks();
    t.list_len = (int32_t)kvlist.size() - t.list_off;
    qtiles.push_back(t);
  }
  *n_hr_ctas = nhr;
  *n_lr_ctas = nlr;
}

// Per 128-key block, the 128-row query tiles that see one of its keys.
// Global key blocks come first (every query tile sees them: the longest
// lists start earliest), then the high-res blocks, whose queries are those of
// the windows neighbouring the block's windows (the neighbour relation is
// symmetric).  An entry is flagged when some in-range (query, key) pair of
// the tile and block is invisible; ranges past the end of a tensor need no
// flag (the kernel zeroes those queries' probabilities and drops those keys).
void build_backward_lists(const ug_geom& g, const std::vector<int32_t>& nbr_off,
                          const std::vector<int32_t>& nbr_idx, std::vector<KTile>& ktiles,
                          std::vector<uint32_t>& qlist) {
  const int64_t N = (int64_t)g.grid_h * g.grid_w, L = global_tokens(g);
  const int64_t T = (int64_t)g.win_h * g.win_w;
  const int nwx = g.grid_w / g.win_w;
  const int64_t BK = kKeysPerBlock, BQ = kRowsPerTile;
  const int64_t n_hr_q = (N + BQ - 1) / BQ, n_lr_q = (L + BQ - 1) / BQ;
  ktiles.clear();
  qlist.clear();
  auto near = [&](int64_t a, int64_t b) {  // window ids
    return std::llabs(a / nwx - b / nwx) <= g.radius && std::llabs(a % nwx - b % nwx) <= g.radius;
  };
  for (int64_t kb = 0; kb * BK < L; ++kb) {
    KTile t;
    t.lowres = 1;
    t.k0 = (int32_t)(kb * BK);
    t.list_off = (int32_t)qlist.size();
    for (int64_t qt = 0; qt < n_hr_q; ++qt) qlist.push_back((uint32_t)qt);
    for (int64_t qt = 0; qt < n_lr_q; ++qt) qlist.push_back((uint32_t)qt | kBlockLowres);
    t.list_len = (int32_t)qlist.size() - t.list_off;
    ktiles.push_back(t);
  }
  for (int64_t kb = 0; kb * BK < N; ++kb) {
    const int64_t k0 = kb * BK, k1 = std::min(N, k0 + BK);
    const int64_t kw0 = k0 / T, kw1 = (k1 - 1) / T;  // key windows
    std::set<int64_t> tiles;
    for (int64_t kw = kw0; kw <= kw1; ++kw)
      for (int32_t e = nbr_off[(size_t)kw]; e < nbr_off[(size_t)kw + 1]; ++e) {
        const int64_t w = nbr_idx[(size_t)e];
        for (int64_t qt = w * T / BQ; qt <= (w * T + T - 1) / BQ; ++qt) tiles.insert(qt);
      }
    KTile t;
    t.lowres = 0;
    t.k0 = (int32_t)k0;
    t.list_off = (int32_t)qlist.size();
    for (int64_t qt : tiles) {
      const int64_t q0 = qt * BQ, q1 = std::min(N, q0 + BQ);
      bool full = true;
      for (int64_t qw = q0 / T; full && qw <= (q1 - 1) / T; ++qw)
        for (int64_t kw = kw0; full && kw <= kw1; ++kw) full = near(qw, kw);
      qlist.push_back((uint32_t)qt | (full ? 0u : kBlockMasked));
    }
    t.list_len = (int32_t)qlist.size() - t.list_off;
    ktiles.push_back(t);
  }
}

// f_k = theta^(-2k/a) (one pow in fp64); angle = position * f_k (one fp64
// product); cos and sin from the C library in fp64, rounded to fp32.
// cos and sin of pos * theta^(-2k/a) for every position and pair k: the
// angle in fp64, cos/sin from the C library, rounded to fp32 once, then
// stored split into the fp32 high part (leading 16 significand bits) and the
// remainder, which add back to the fp32 value exactly.
static void axis_table(const std::vector<double>& pos, int a, double theta, float* out,
                       const AxisTables& t) {
  const int m = a / 2;
  std::vector<double> f((size_t)m);
  for (int k = 0; k < m; ++k) f[(size_t)k] = std::pow(theta, -2.0 * k / a);
  for (size_t i = 0; i < pos.size(); ++i)
    for (int k = 0; k < m; ++k) {
      const double ang = pos[i] * f[(size_t)k];
      const float c = (float)std::cos(ang), s = (float)std::sin(ang);
      const size_t at = i * m + k;
      out[t.cos_hi + at] = rope_math::split_hi(c);
      out[t.cos_lo + at] = rope_math::split_lo(c);
      out[t.sin_hi + at] = rope_math::split_hi(s);
      out[t.sin_lo + at] = rope_math::split_lo(s);
    }
}

void build_rope_tables(const ug_geom& g, RopeTables& o, std::vector<float>& data) {
  const int64_t my = g.rope_dim_y / 2, mx = g.rope_dim_x / 2;
  int64_t at = 0;
  auto take = [&](int64_t n) {
    const int64_t r = at;
    at += (n + 3) / 4 * 4;  // keep every table 16-byte aligned
    return r;
  };
  auto axis = [&](int64_t n) {
    AxisTables t;
    t.cos_hi = take(n);
    t.sin_hi = take(n);
    t.cos_lo = take(n);
    t.sin_lo = take(n);
    return t;
  };
  o.hr_y = axis(g.grid_h * my);
  o.hr_x = axis(g.grid_w * mx);
  o.lr_y = axis(g.lr_h * my);
  o.lr_x = axis(g.lr_w * mx);
  o.total = std::max<int64_t>(at, 4);
  data.assign((size_t)o.total, 0.0f);
  std::vector<double> py, px, ly, lx;
  for (int i = 0; i < g.grid_h; ++i) py.push_back((double)i);
  for (int i = 0; i < g.grid_w; ++i) px.push_back((double)i);
  for (int i = 0; i < g.lr_h; ++i) ly.push_back(g.rho * (double)i);
  for (int i = 0; i < g.lr_w; ++i) lx.push_back(g.rho * (double)i);
  axis_table(py, g.rope_dim_y, g.rope_theta, data.data(), o.hr_y);
  axis_table(px, g.rope_dim_x, g.rope_theta, data.data(), o.hr_x);
  if (g.lr_h > 0) {
    axis_table(ly, g.rope_dim_y, g.rope_theta, data.data(), o.lr_y);
    axis_table(lx, g.rope_dim_x, g.rope_theta, data.data(), o.lr_x);
  }
}

}  // namespace ug
