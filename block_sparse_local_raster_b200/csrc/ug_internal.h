// Internal declarations shared by the library's translation units.
#pragma once

#include <cstdint>
#include <vector>

#include <cuda_runtime.h>

#include "ug.h"

namespace ug {

// Attention tiling: a CTA owns 256 consecutive query rows of one token set
// (two 128-row tiles, one TMEM lane per row) and walks a list of 128-key
// blocks.
constexpr int kRowsPerTile = 128;
constexpr int kTilesPerCta = 2;
constexpr int kRowsPerCta = kRowsPerTile * kTilesPerCta;
constexpr int kKeysPerBlock = 128;

// One query CTA of the attention: which token set its rows belong to, its
// first row, and its slice of the key-block list.
struct QTile {
  int32_t lowres;    // 0: high-res rows (window-first), 1: low-res rows
  int32_t q0;        // first query token of the CTA inside its tensor
  int32_t list_off;  // first entry in the key-block list
  int32_t list_len;  // number of key blocks (>= 1)
};

// One key CTA of the attention backward (dK, dV): its 128 keys, and its slice
// of the query-tile list (the 128-row query tiles holding a query that sees
// one of the keys).
struct KTile {
  int32_t lowres;    // 0: high-res keys (window-first), 1: global keys
  int32_t k0;        // first key of the block inside its tensor
  int32_t list_off;  // first entry in the query-tile list
  int32_t list_len;  // number of query tiles (>= 1)
};

// Key-block list entry: block index (keys [128*idx, 128*idx + 128) of its
// tensor), whether it lies in the low-res tensor, and whether some
// (query, key) pair inside it is invisible or out of range so that the
// kernel must test each pair.
constexpr uint32_t kBlockIndexMask = (1u << 29) - 1;
constexpr uint32_t kBlockLowres = 1u << 29;
constexpr uint32_t kBlockMasked = 1u << 30;

// Offsets (in elements) of the RoPE tables inside the plan's table buffer,
// for one axis of one token set.  Each table is [coordinate][pair k]; the
// fp32-rounded cos and sin are each stored split, c = hi + lo with hi the
// leading 16 bits of c's significand (ug_rope_math.h), every table and row
// 16-byte aligned.
struct AxisTables {
  int64_t cos_hi, sin_hi, cos_lo, sin_lo;
};
struct RopeTables {
  AxisTables hr_y, hr_x, lr_y, lr_x;
  int64_t total;
};

// Tokens of the global set: text tokens, then the low-res grid.
inline int64_t global_tokens(const ug_geom& g) {
  return (int64_t)g.text_len + (int64_t)g.lr_h * g.lr_w;
}

// Upper bound of a device-side wait before a kernel gives up (ns).
constexpr int64_t kDefaultWaitTimeoutNs = 2000000000ll;

}  // namespace ug

struct ug_plan {
  ug_geom g;
  int64_t N, L, T;   // high-res tokens, global (text + low-res) tokens, tokens per window
  int32_t nwy, nwx;  // windows per axis
  float scale;       // softmax scale actually used
  int device;

  std::vector<int32_t> perm, nbr_off, nbr_idx;
  std::vector<ug::QTile> qtiles;
  std::vector<uint32_t> kvlist;
  std::vector<ug::KTile> ktiles;  // backward: key CTAs
  std::vector<uint32_t> qlist;    // backward: query tiles per key CTA (entry format as kvlist)
  int32_t n_hr_ctas, n_lr_ctas;
  ug::RopeTables rope;

  void* d_mem;             // one device allocation holding everything below
  float* d_rope;           // RoPE tables
  ug::QTile* d_qtiles;     // attention query CTAs
  uint32_t* d_kvlist;      // attention key-block lists
  ug::KTile* d_ktiles;     // backward key CTAs
  uint32_t* d_qlist;       // backward query-tile lists
  int* d_err;              // first device-side error status (0 = none)
  int64_t wait_timeout_ns;
};

namespace ug {

// Host plan pieces (ug_plan.cu).
int validate(const ug_geom* g);
void build_perm(const ug_geom& g, std::vector<int32_t>& perm);
void build_neighbours(const ug_geom& g, std::vector<int32_t>& off, std::vector<int32_t>& idx);
void build_attention_lists(const ug_geom& g, const std::vector<int32_t>& nbr_off,
                           const std::vector<int32_t>& nbr_idx, std::vector<QTile>& qtiles,
                           std::vector<uint32_t>& kvlist, int32_t* n_hr_ctas, int32_t* n_lr_ctas);
void build_backward_lists(const ug_geom& g, const std::vector<int32_t>& nbr_off,
                          const std::vector<int32_t>& nbr_idx, std::vector<KTile>& ktiles,
                          std::vector<uint32_t>& qlist);
void build_rope_tables(const ug_geom& g, RopeTables& off, std::vector<float>& data);

// Kernel launchers (one .cu each).  Arguments are already checked.
int launch_permute(const ug_plan* p, const void* src, void* dst, bool inverse, cudaStream_t s);
int launch_rope(const ug_plan* p, const void* x, void* y, int token_set, cudaStream_t s,
                bool transpose = false);
int launch_permute_rope(const ug_plan* p, const void* src, void* dst, cudaStream_t s,
                        bool inverse = false);
int launch_attention_bwd(const ug_plan* p, const void* q_hr, const void* k_hr, const void* v_hr,
                         const void* q_lr, const void* k_lr, const void* v_lr, const void* o_hr,
                         const void* o_lr, const void* do_hr, const void* do_lr, const float* lse,
                         void* dq_hr, void* dk_hr, void* dv_hr, void* dq_lr, void* dk_lr,
                         void* dv_lr, float* delta, bool vo_raster, cudaStream_t s);
int launch_warm_start(const ug_warm_start_params* p, const float* x_lr, const float* noise,
                      float* out, cudaStream_t s);
// The factor-4 warm start's weights, [py][px][3 r + c] (host, fp64 -> fp32).
void warm_start_stencil_weights(double amount, double t, float* wt);
int launch_attention(const ug_plan* p, const void* q_hr, const void* k_hr, const void* v_hr,
                     const void* q_lr, const void* k_lr, const void* v_lr, void* o_hr,
                     void* o_lr, float* lse, bool vo_raster, cudaStream_t s);
// Per-device set-up, done once per device and run by ug_plan_create with the
// plan's device current: the attention and RoPE kernels' shared-memory
// opt-in, and the device address of the static scratch of
// ug_layer_fwd_static_scratch.
int prepare_attention(int device);
int prepare_attention_bwd(int device);
int prepare_rope(int device);
int prepare_static_scratch(int device);
// Whether a 128-key tile is always 128 / win_w whole rows of one window, so
// that raster-order V can be read tile by tile.
bool vo_raster_supported(const ug_geom& g);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace ug
