// The C ABI: argument checks, plan lifetime, the layer sequence.
#include <cmath>
#include <cstring>
#include <new>
#include <vector>

#include "ug_internal.h"

using namespace ug;

namespace {

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

bool overlap(const void* a, int64_t na, const void* b, int64_t nb) {
  if (!a || !b || na <= 0 || nb <= 0) return false;
  const char* pa = static_cast<const char*>(a);
  const char* pb = static_cast<const char*>(b);
  return pa < pb + nb && pb < pa + na;
}

// The plan's tables live in the memory of the device that was current when
// it was created; its kernels must launch there.
int check_device(const ug_plan* p) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return UG_ERR_CUDA;
  }
  return dev == p->device ? UG_OK : UG_ERR_INVALID_ARG;
}

int64_t hr_bytes(const ug_plan* p) {
  return (int64_t)p->g.batch * p->N * p->g.heads * p->g.head_dim * 2;
}
int64_t lr_bytes(const ug_plan* p) {
  return (int64_t)p->g.batch * p->L * p->g.heads * p->g.head_dim * 2;
}

}  // namespace

extern "C" {

int ug_geom_validate(const ug_geom* g) { return validate(g); }

int ug_index_map_sizes(const ug_geom* g, int64_t* n_perm, int64_t* n_nbr_off,
                       int64_t* n_nbr_idx) {
  int st = validate(g);
  if (st != UG_OK) return st;
  const int64_t nwy = g->grid_h / g->win_h, nwx = g->grid_w / g->win_w;
  std::vector<int32_t> off, idx;
  build_neighbours(*g, off, idx);
  if (n_perm) *n_perm = (int64_t)g->grid_h * g->grid_w;
  if (n_nbr_off) *n_nbr_off = nwy * nwx + 1;
  if (n_nbr_idx) *n_nbr_idx = (int64_t)idx.size();
  return UG_OK;
}

int ug_build_index_maps(const ug_geom* g, int32_t* perm, int32_t* nbr_off, int32_t* nbr_idx) {
  int st = validate(g);
  if (st != UG_OK) return st;
  std::vector<int32_t> p, off, idx;
  build_perm(*g, p);
  build_neighbours(*g, off, idx);
  if (perm) std::memcpy(perm, p.data(), p.size() * sizeof(int32_t));
  if (nbr_off) std::memcpy(nbr_off, off.data(), off.size() * sizeof(int32_t));
  if (nbr_idx) std::memcpy(nbr_idx, idx.data(), idx.size() * sizeof(int32_t));
  return UG_OK;
}

int ug_visible_pairs(const ug_geom* g, int64_t* hr_hr, int64_t* hr_lr, int64_t* lr_lr) {
  int st = validate(g);
  if (st != UG_OK) return st;
  std::vector<int32_t> off, idx;
  build_neighbours(*g, off, idx);
  const int64_t T = (int64_t)g->win_h * g->win_w;
  const int64_t N = (int64_t)g->grid_h * g->grid_w, L = global_tokens(*g);
  if (hr_hr) *hr_hr = (int64_t)idx.size() * T * T;
  if (hr_lr) *hr_lr = N * L;
  if (lr_lr) *lr_lr = L * L;
  return UG_OK;
}

namespace {

int work_lists(const ug_geom* g, std::vector<QTile>& qt, std::vector<uint32_t>& kv,
               std::vector<KTile>& kt, std::vector<uint32_t>& ql) {
  int st = validate(g);
  if (st != UG_OK) return st;
  std::vector<int32_t> off, idx;
  build_neighbours(*g, off, idx);
  int32_t nhr, nlr;
  build_attention_lists(*g, off, idx, qt, kv, &nhr, &nlr);
  build_backward_lists(*g, off, idx, kt, ql);
  return UG_OK;
}

}  // namespace

int ug_work_list_sizes(const ug_geom* g, int64_t* n_qctas, int64_t* n_kvlist, int64_t* n_kctas,
                       int64_t* n_qlist) {
  std::vector<QTile> qt;
  std::vector<uint32_t> kv, ql;
  std::vector<KTile> kt;
  int st;
  try {
    st = work_lists(g, qt, kv, kt, ql);
  } catch (...) {
    return UG_ERR_NO_MEMORY;
  }
  if (st != UG_OK) return st;
  if (n_qctas) *n_qctas = (int64_t)qt.size();
  if (n_kvlist) *n_kvlist = (int64_t)kv.size();
  if (n_kctas) *n_kctas = (int64_t)kt.size();
  if (n_qlist) *n_qlist = (int64_t)ql.size();
  return UG_OK;
}

int ug_build_work_lists(const ug_geom* g, int32_t* qctas, uint32_t* kvlist, int32_t* kctas,
                        uint32_t* qlist) {
  std::vector<QTile> qt;
  std::vector<uint32_t> kv, ql;
  std::vector<KTile> kt;
  int st;
  try {
    st = work_lists(g, qt, kv, kt, ql);
  } catch (...) {
    return UG_ERR_NO_MEMORY;
  }
  if (st != UG_OK) return st;
  for (size_t i = 0; qctas && i < qt.size(); ++i) {
    qctas[4 * i] = qt[i].lowres;
    qctas[4 * i + 1] = qt[i].q0;
    qctas[4 * i + 2] = qt[i].list_off;
    qctas[4 * i + 3] = qt[i].list_len;
  }
  for (size_t i = 0; kctas && i < kt.size(); ++i) {
    kctas[4 * i] = kt[i].lowres;
    kctas[4 * i + 1] = kt[i].k0;
    kctas[4 * i + 2] = kt[i].list_off;
    kctas[4 * i + 3] = kt[i].list_len;
  }
  if (kvlist) std::memcpy(kvlist, kv.data(), kv.size() * sizeof(uint32_t));
  if (qlist) std::memcpy(qlist, ql.data(), ql.size() * sizeof(uint32_t));
  return UG_OK;
}

const char* ug_status_string(int s) {
  switch (s) {
    case UG_OK: return "ok";
    case UG_ERR_INVALID_ARG: return "invalid argument";
    case UG_ERR_UNSUPPORTED: return "unsupported geometry";
    case UG_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
    case UG_ERR_ALIAS: return "output overlaps an input";
    case UG_ERR_CUDA: return "CUDA error";
    case UG_ERR_TIMEOUT: return "device-side wait timed out";
    case UG_ERR_NO_MEMORY: return "out of memory";
    default: return "unknown status";
  }
}

int ug_plan_create(const ug_geom* g, ug_plan** out) {
  if (!out) return UG_ERR_INVALID_ARG;
  *out = nullptr;
  int st = validate(g);
  if (st != UG_OK) return st;
  ug_plan* p = new (std::nothrow) ug_plan();
  if (!p) return UG_ERR_NO_MEMORY;
  p->g = *g;
  p->N = (int64_t)g->grid_h * g->grid_w;
  p->L = global_tokens(*g);
  p->T = (int64_t)g->win_h * g->win_w;
  p->nwy = g->grid_h / g->win_h;
  p->nwx = g->grid_w / g->win_w;
  p->scale = g->softmax_scale > 0.0f ? g->softmax_scale : (float)(1.0 / std::sqrt((double)g->head_dim));
  p->wait_timeout_ns = kDefaultWaitTimeoutNs;
  p->d_mem = nullptr;
  try {
    build_perm(*g, p->perm);
    build_neighbours(*g, p->nbr_off, p->nbr_idx);
    build_attention_lists(*g, p->nbr_off, p->nbr_idx, p->qtiles, p->kvlist, &p->n_hr_ctas,
                          &p->n_lr_ctas);
    build_backward_lists(*g, p->nbr_off, p->nbr_idx, p->ktiles, p->qlist);
    std::vector<float> tables;
    build_rope_tables(*g, p->rope, tables);
    // One device block: [err (256 B)] [rope tables] [qtiles] [kvlist] [ktiles] [qlist]
    const size_t a_err = 0;
    const size_t a_rope = 256;
    const size_t a_qt = (a_rope + tables.size() * sizeof(float) + 255) / 256 * 256;
    const size_t a_kv = (a_qt + p->qtiles.size() * sizeof(QTile) + 255) / 256 * 256;
    const size_t a_kt = (a_kv + std::max<size_t>(1, p->kvlist.size()) * sizeof(uint32_t) + 255) /
                        256 * 256;
    const size_t a_ql = (a_kt + p->ktiles.size() * sizeof(KTile) + 255) / 256 * 256;
    const size_t total = a_ql + std::max<size_t>(1, p->qlist.size()) * sizeof(uint32_t);
    if (cudaGetDevice(&p->device) != cudaSuccess) { delete p; return UG_ERR_CUDA; }
    // once per device: kernel attributes, the static scratch's address
    if ((st = prepare_attention(p->device)) != UG_OK ||
        (st = prepare_attention_bwd(p->device)) != UG_OK ||
        (st = prepare_rope(p->device)) != UG_OK ||
        (st = prepare_static_scratch(p->device)) != UG_OK) {
      delete p;
      return st;
    }
    if (cudaMalloc(&p->d_mem, total) != cudaSuccess) {
      cudaGetLastError();
      delete p;
      return UG_ERR_NO_MEMORY;
    }
    char* base = static_cast<char*>(p->d_mem);
    p->d_err = reinterpret_cast<int*>(base + a_err);
    p->d_rope = reinterpret_cast<float*>(base + a_rope);
    p->d_qtiles = reinterpret_cast<QTile*>(base + a_qt);
    p->d_kvlist = reinterpret_cast<uint32_t*>(base + a_kv);
    p->d_ktiles = reinterpret_cast<KTile*>(base + a_kt);
    p->d_qlist = reinterpret_cast<uint32_t*>(base + a_ql);
    std::vector<char> host(total, 0);
    std::memcpy(host.data() + a_rope, tables.data(), tables.size() * sizeof(float));
    std::memcpy(host.data() + a_qt, p->qtiles.data(), p->qtiles.size() * sizeof(QTile));
    std::memcpy(host.data() + a_kv, p->kvlist.data(), p->kvlist.size() * sizeof(uint32_t));
    std::memcpy(host.data() + a_kt, p->ktiles.data(), p->ktiles.size() * sizeof(KTile));
    std::memcpy(host.data() + a_ql, p->qlist.data(), p->qlist.size() * sizeof(uint32_t));
    if (cudaMemcpy(p->d_mem, host.data(), total, cudaMemcpyHostToDevice) != cudaSuccess) {
      cudaFree(p->d_mem);
      delete p;
      return UG_ERR_CUDA;
    }
  } catch (const std::bad_alloc&) {
    if (p->d_mem) cudaFree(p->d_mem);
    delete p;
    return UG_ERR_NO_MEMORY;
  }
  *out = p;
  return UG_OK;
}

int ug_plan_destroy(ug_plan* p) {
  if (!p) return UG_OK;
  int st = UG_OK;
  if (p->d_mem) {
    // free on the plan's device, then restore the caller's current device
    int cur = -1;
    const bool have_cur = cudaGetDevice(&cur) == cudaSuccess;
    const bool other = have_cur && cur != p->device;
    if (other && cudaSetDevice(p->device) != cudaSuccess) st = UG_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) st = UG_ERR_CUDA;
    if (cudaFree(p->d_mem) != cudaSuccess) st = UG_ERR_CUDA;
    if (other && cudaSetDevice(cur) != cudaSuccess) st = UG_ERR_CUDA;
  }
  delete p;
  return st;
}

int ug_get_index_maps(const ug_plan* p, int32_t* perm, int32_t* nbr_off, int32_t* nbr_idx) {
  if (!p) return UG_ERR_INVALID_ARG;
  if (perm) std::memcpy(perm, p->perm.data(), p->perm.size() * sizeof(int32_t));
  if (nbr_off) std::memcpy(nbr_off, p->nbr_off.data(), p->nbr_off.size() * sizeof(int32_t));
  if (nbr_idx) std::memcpy(nbr_idx, p->nbr_idx.data(), p->nbr_idx.size() * sizeof(int32_t));
  return UG_OK;
}

static int permute_common(const ug_plan* p, const void* src, void* dst, bool inverse, void* s) {
  if (!p || !src || !dst) return UG_ERR_INVALID_ARG;
  if (!aligned16(src) || !aligned16(dst)) return UG_ERR_ALIGNMENT;
  const int64_t n = hr_bytes(p);
  if (overlap(src, n, dst, n)) return UG_ERR_ALIAS;
  if (const int st = check_device(p)) return st;
  return launch_permute(p, src, dst, inverse, as_stream(s));
}

int ug_permute_window_first(const ug_plan* p, const void* src_raster, void* dst_wf, void* s) {
  return permute_common(p, src_raster, dst_wf, false, s);
}

int ug_permute_rope_window_first(const ug_plan* p, const void* src_raster, void* dst_wf,
                                 void* s) {
  if (!p || !src_raster || !dst_wf) return UG_ERR_INVALID_ARG;
  if (!aligned16(src_raster) || !aligned16(dst_wf)) return UG_ERR_ALIGNMENT;
  const int64_t n = hr_bytes(p);
  if (overlap(src_raster, n, dst_wf, n)) return UG_ERR_ALIAS;
  if (const int st = check_device(p)) return st;
  return launch_permute_rope(p, src_raster, dst_wf, as_stream(s));
}

int ug_unpermute(const ug_plan* p, const void* src_wf, void* dst_raster, void* s) {
  return permute_common(p, src_wf, dst_raster, true, s);
}

int ug_rope_2d(const ug_plan* p, const void* x, void* y, int token_set, void* s) {
  if (!p || !x || !y) return UG_ERR_INVALID_ARG;
  if (token_set != UG_HR_WINDOW_FIRST && token_set != UG_HR_RASTER && token_set != UG_LR)
    return UG_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y)) return UG_ERR_ALIGNMENT;
  const int64_t n = token_set == UG_LR ? lr_bytes(p) : hr_bytes(p);
  if (n == 0) return UG_OK;
  if (x != y && overlap(x, n, y, n)) return UG_ERR_ALIAS;
  if (const int st = check_device(p)) return st;
  return launch_rope(p, x, y, token_set, as_stream(s));
}

}  // extern "C"

namespace {

// Pointers, alignment and overlaps of a forward call's tensors: inputs
// q/k/v (high-res and global), outputs o_hr, o_lr and the optional lse.
int check_fwd_tensors(const ug_plan* p, const void* q_hr, const void* k_hr, const void* v_hr,
                      const void* q_lr, const void* k_lr, const void* v_lr, const void* o_hr,
                      const void* o_lr, const float* lse) {
  if (!p || !q_hr || !k_hr || !v_hr || !o_hr) return UG_ERR_INVALID_ARG;
  if (p->L > 0 && (!q_lr || !k_lr || !v_lr || !o_lr)) return UG_ERR_INVALID_ARG;
  if (p->g.head_dim != 64 && p->g.head_dim != 128) return UG_ERR_UNSUPPORTED;
  if (p->L == 0) q_lr = k_lr = v_lr = o_lr = nullptr;
  const void* ins[6] = {q_hr, k_hr, v_hr, q_lr, k_lr, v_lr};
  for (const void* a : ins)
    if (a && !aligned16(a)) return UG_ERR_ALIGNMENT;
  if (!aligned16(o_hr) || (o_lr && !aligned16(o_lr)) || (lse && !aligned16(lse)))
    return UG_ERR_ALIGNMENT;
  const int64_t nh = hr_bytes(p), nl = lr_bytes(p);
  const int64_t nlse = lse ? (int64_t)p->g.batch * p->g.heads * (p->N + p->L) * 4 : 0;
  const int64_t sizes[6] = {nh, nh, nh, nl, nl, nl};
  for (int i = 0; i < 6; ++i) {
    if (overlap(o_hr, nh, ins[i], sizes[i]) || overlap(o_lr, nl, ins[i], sizes[i]) ||
        overlap(lse, nlse, ins[i], sizes[i]))
      return UG_ERR_ALIAS;
  }
  if (overlap(o_hr, nh, o_lr, nl) || overlap(o_hr, nh, lse, nlse) || overlap(o_lr, nl, lse, nlse))
    return UG_ERR_ALIAS;
  return UG_OK;
}

int attn_fwd_checked(const ug_plan* p, const void* q_hr, const void* k_hr, const void* v_hr,
                     const void* q_lr, const void* k_lr, const void* v_lr, void* o_hr,
                     void* o_lr, float* lse, bool vo_raster, void* s) {
  if (const int st = check_fwd_tensors(p, q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, o_hr, o_lr, lse))
    return st;
  if (const int st = check_device(p)) return st;
  return launch_attention(p, q_hr, k_hr, v_hr, p->L ? q_lr : nullptr, p->L ? k_lr : nullptr,
                          p->L ? v_lr : nullptr, o_hr, p->L ? o_lr : nullptr, lse, vo_raster,
                          as_stream(s));
}

}  // namespace

extern "C" {

int ug_hier_local_attn_fwd(const ug_plan* p, const void* q_hr, const void* k_hr,
                           const void* v_hr, const void* q_lr, const void* k_lr,
                           const void* v_lr, void* o_hr, void* o_lr, float* lse, void* s) {
  return attn_fwd_checked(p, q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, o_hr, o_lr, lse, false, s);
}

int ug_hier_local_attn_fwd_vo_raster(const ug_plan* p, const void* q_hr, const void* k_hr,
                                     const void* v_hr_raster, const void* q_lr, const void* k_lr,
                                     const void* v_lr, void* o_hr_raster, void* o_lr, float* lse,
                                     void* s) {
  if (p && !vo_raster_supported(p->g)) return UG_ERR_UNSUPPORTED;
  return attn_fwd_checked(p, q_hr, k_hr, v_hr_raster, q_lr, k_lr, v_lr, o_hr_raster, o_lr, lse,
                          true, s);
}


int64_t ug_layer_workspace_bytes(const ug_plan* p) {
  if (!p) return -1;
  auto up = [](int64_t n) { return (n + 255) / 256 * 256; };
  return 4 * up(hr_bytes(p)) + 2 * up(lr_bytes(p));
}

int ug_layer_fwd(const ug_plan* p, const void* q_hr, const void* k_hr, const void* v_hr,
                 const void* q_lr, const void* k_lr, const void* v_lr, void* o_hr, void* o_lr,
                 float* lse, void* workspace, int64_t workspace_bytes, void* s) {
  // Every argument check runs here, before the first launch is queued.
  if (!p || !workspace) return UG_ERR_INVALID_ARG;
  if (workspace_bytes < ug_layer_workspace_bytes(p)) return UG_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return UG_ERR_ALIGNMENT;
  if (const int st = check_fwd_tensors(p, q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, o_hr, o_lr, lse))
    return st;
  const int64_t ws = ug_layer_workspace_bytes(p);
  const int64_t nh = hr_bytes(p), nl = lr_bytes(p);
  const int64_t nlse = lse ? (int64_t)p->g.batch * p->g.heads * (p->N + p->L) * 4 : 0;
  const void* ts[9] = {q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, o_hr, o_lr, lse};
  const int64_t sizes[9] = {nh, nh, nh, nl, nl, nl, nh, nl, nlse};
  for (int i = 0; i < 9; ++i)
    if (overlap(workspace, ws, ts[i], sizes[i])) return UG_ERR_ALIAS;
  if (const int st = check_device(p)) return st;
  auto up = [](int64_t n) { return (n + 255) / 256 * 256; };
  char* w = static_cast<char*>(workspace);
  void* q_wf = w;
  void* k_wf = w + up(nh);
  void* v_wf = w + 2 * up(nh);
  void* o_wf = w + 3 * up(nh);
  void* q_lr_r = w + 4 * up(nh);
  void* k_lr_r = w + 4 * up(nh) + up(nl);
  int st;
  if ((st = ug_permute_rope_window_first(p, q_hr, q_wf, s)) != UG_OK) return st;
  if ((st = ug_permute_rope_window_first(p, k_hr, k_wf, s)) != UG_OK) return st;
  if (p->L > 0) {
    if ((st = ug_rope_2d(p, q_lr, q_lr_r, UG_LR, s)) != UG_OK) return st;
    if ((st = ug_rope_2d(p, k_lr, k_lr_r, UG_LR, s)) != UG_OK) return st;
  }
  // Where 128-key tiles are whole window rows, the attention reads v and
  // writes o in raster order itself: no permute of v, no unpermute of o.
  if (vo_raster_supported(p->g))
    return ug_hier_local_attn_fwd_vo_raster(p, q_wf, k_wf, v_hr, q_lr_r, k_lr_r, v_lr, o_hr,
                                            o_lr, lse, s);
  if ((st = ug_permute_window_first(p, v_hr, v_wf, s)) != UG_OK) return st;
  if ((st = ug_hier_local_attn_fwd(p, q_wf, k_wf, v_wf, q_lr_r, k_lr_r, v_lr, o_wf, o_lr, lse,
                                   s)) != UG_OK)
    return st;
  return ug_unpermute(p, o_wf, o_hr, s);
}

// ---- backward ----------------------------------------------------------------

int ug_rope_2d_bwd(const ug_plan* p, const void* dy, void* dx, int token_set, void* s) {
  if (!p || !dy || !dx) return UG_ERR_INVALID_ARG;
  if (token_set != UG_HR_WINDOW_FIRST && token_set != UG_HR_RASTER && token_set != UG_LR)
    return UG_ERR_INVALID_ARG;
  if (!aligned16(dy) || !aligned16(dx)) return UG_ERR_ALIGNMENT;
  const int64_t n = token_set == UG_LR ? lr_bytes(p) : hr_bytes(p);
  if (n == 0) return UG_OK;
  if (dy != dx && overlap(dy, n, dx, n)) return UG_ERR_ALIAS;
  if (const int st = check_device(p)) return st;
  return launch_rope(p, dy, dx, token_set, as_stream(s), true);
}

int ug_unpermute_rope_bwd(const ug_plan* p, const void* src_wf, void* dst_raster, void* s) {
  if (!p || !src_wf || !dst_raster) return UG_ERR_INVALID_ARG;
  if (!aligned16(src_wf) || !aligned16(dst_raster)) return UG_ERR_ALIGNMENT;
  const int64_t n = hr_bytes(p);
  if (overlap(src_wf, n, dst_raster, n)) return UG_ERR_ALIAS;
  if (const int st = check_device(p)) return st;
  return launch_permute_rope(p, src_wf, dst_raster, as_stream(s), true);
}

int64_t ug_attn_bwd_workspace_bytes(const ug_plan* p) {
  if (!p) return -1;
  return ((int64_t)p->g.batch * p->g.heads * (p->N + p->L) * 4 + 255) / 256 * 256;
}

}  // extern "C"

namespace {

int attn_bwd_checked(const ug_plan* p, const void* q_hr, const void* k_hr, const void* v_hr,
                     const void* q_lr, const void* k_lr, const void* v_lr, const void* o_hr,
                     const void* o_lr, const void* do_hr, const void* do_lr, const float* lse,
                     void* dq_hr, void* dk_hr, void* dv_hr, void* dq_lr, void* dk_lr, void* dv_lr,
                     void* workspace, int64_t workspace_bytes, bool vo_raster, void* s) {
  if (!p || !lse || !workspace) return UG_ERR_INVALID_ARG;
  if (workspace_bytes < ug_attn_bwd_workspace_bytes(p)) return UG_ERR_INVALID_ARG;
  const bool lr = p->L > 0;
  if (!lr) q_lr = k_lr = v_lr = o_lr = do_lr = dq_lr = dk_lr = dv_lr = nullptr;
  const void* ins[10] = {q_hr, k_hr, v_hr, o_hr, do_hr, q_lr, k_lr, v_lr, o_lr, do_lr};
  void* outs[6] = {dq_hr, dk_hr, dv_hr, dq_lr, dk_lr, dv_lr};
  for (int i = 0; i < 10; ++i)
    if (!ins[i] && (i < 5 || lr)) return UG_ERR_INVALID_ARG;
  for (int i = 0; i < 6; ++i)
    if (!outs[i] && (i < 3 || lr)) return UG_ERR_INVALID_ARG;
  if (p->g.head_dim != 64 && p->g.head_dim != 128) return UG_ERR_UNSUPPORTED;
  for (const void* a : ins)
    if (a && !aligned16(a)) return UG_ERR_ALIGNMENT;
  for (const void* a : outs)
    if (a && !aligned16(a)) return UG_ERR_ALIGNMENT;
  if (!aligned16(lse) || !aligned16(workspace)) return UG_ERR_ALIGNMENT;
  const int64_t nh = hr_bytes(p), nl = lr ? lr_bytes(p) : 0;
  const int64_t nlse = (int64_t)p->g.batch * p->g.heads * (p->N + p->L) * 4;
  const int64_t nws = ug_attn_bwd_workspace_bytes(p);
  // every output and the workspace are disjoint from each other and from every input
  const void* w[7] = {outs[0], outs[1], outs[2], outs[3], outs[4], outs[5], workspace};
  const int64_t wn[7] = {nh, nh, nh, nl, nl, nl, nws};
  for (int i = 0; i < 7; ++i) {
    for (int j = 0; j < 10; ++j)
      if (overlap(w[i], wn[i], ins[j], j < 5 ? nh : nl)) return UG_ERR_ALIAS;
    if (overlap(w[i], wn[i], lse, nlse)) return UG_ERR_ALIAS;
    for (int j = i + 1; j < 7; ++j)
      if (overlap(w[i], wn[i], w[j], wn[j])) return UG_ERR_ALIAS;
  }
  if (const int st = check_device(p)) return st;
  return launch_attention_bwd(p, q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, o_hr, o_lr, do_hr, do_lr,
                              lse, dq_hr, dk_hr, dv_hr, dq_lr, dk_lr, dv_lr,
                              static_cast<float*>(workspace), vo_raster, as_stream(s));
}

}  // namespace

extern "C" {

int ug_hier_local_attn_bwd(const ug_plan* p, const void* q_hr, const void* k_hr,
                           const void* v_hr, const void* q_lr, const void* k_lr,
                           const void* v_lr, const void* o_hr, const void* o_lr,
                           const void* do_hr, const void* do_lr, const float* lse, void* dq_hr,
                           void* dk_hr, void* dv_hr, void* dq_lr, void* dk_lr, void* dv_lr,
                           void* workspace, int64_t workspace_bytes, void* s) {
  return attn_bwd_checked(p, q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, o_hr, o_lr, do_hr, do_lr, lse,
                          dq_hr, dk_hr, dv_hr, dq_lr, dk_lr, dv_lr, workspace, workspace_bytes,
                          false, s);
}

int ug_hier_local_attn_bwd_vo_raster(const ug_plan* p, const void* q_hr, const void* k_hr,
                                     const void* v_hr_raster, const void* q_lr,
                                     const void* k_lr, const void* v_lr,
                                     const void* o_hr_raster, const void* o_lr,
                                     const void* do_hr_raster, const void* do_lr,
                                     const float* lse, void* dq_hr, void* dk_hr,
                                     void* dv_hr_raster, void* dq_lr, void* dk_lr, void* dv_lr,
                                     void* workspace, int64_t workspace_bytes, void* s) {
  if (p && !vo_raster_supported(p->g)) return UG_ERR_UNSUPPORTED;
  return attn_bwd_checked(p, q_hr, k_hr, v_hr_raster, q_lr, k_lr, v_lr, o_hr_raster, o_lr,
                          do_hr_raster, do_lr, lse, dq_hr, dk_hr, dv_hr_raster, dq_lr, dk_lr,
                          dv_lr, workspace, workspace_bytes, true, s);
}

int64_t ug_layer_bwd_workspace_bytes(const ug_plan* p) {
  if (!p) return -1;
  auto up = [](int64_t n) { return (n + 255) / 256 * 256; };
  return 8 * up(hr_bytes(p)) + 2 * up(lr_bytes(p)) + ug_attn_bwd_workspace_bytes(p);
}

int ug_layer_bwd(const ug_plan* p, const void* q_hr, const void* k_hr, const void* v_hr,
                 const void* q_lr, const void* k_lr, const void* v_lr, const void* o_hr,
                 const void* o_lr, const float* lse, const void* do_hr, const void* do_lr,
                 void* dq_hr, void* dk_hr, void* dv_hr, void* dq_lr, void* dk_lr, void* dv_lr,
                 void* workspace, int64_t workspace_bytes, void* s) {
  if (!p || !workspace) return UG_ERR_INVALID_ARG;
  const int64_t ws = ug_layer_bwd_workspace_bytes(p);
  if (workspace_bytes < ws) return UG_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return UG_ERR_ALIGNMENT;
  const bool lr = p->L > 0;
  const void* ins[10] = {q_hr, k_hr, v_hr, o_hr, do_hr, q_lr, k_lr, v_lr, o_lr, do_lr};
  void* outs[6] = {dq_hr, dk_hr, dv_hr, dq_lr, dk_lr, dv_lr};
  if (!lse) return UG_ERR_INVALID_ARG;
  for (int i = 0; i < 10; ++i)
    if (!ins[i] && (i < 5 || lr)) return UG_ERR_INVALID_ARG;
  for (int i = 0; i < 6; ++i)
    if (!outs[i] && (i < 3 || lr)) return UG_ERR_INVALID_ARG;
  if (p->g.head_dim != 64 && p->g.head_dim != 128) return UG_ERR_UNSUPPORTED;
  const int64_t nh = hr_bytes(p), nl = lr ? lr_bytes(p) : 0;
  for (int i = 0; i < 10; ++i)
    if (overlap(workspace, ws, ins[i], i < 5 ? nh : nl)) return UG_ERR_ALIAS;
  for (int i = 0; i < 6; ++i)
    if (overlap(workspace, ws, outs[i], i < 3 ? nh : nl)) return UG_ERR_ALIAS;
  // the gradients are disjoint from every input and from each other
  const int64_t nlse = (int64_t)p->g.batch * p->g.heads * (p->N + p->L) * 4;
  if (overlap(workspace, ws, lse, nlse)) return UG_ERR_ALIAS;
  for (int i = 0; i < 6; ++i) {
    const int64_t ni = i < 3 ? nh : nl;
    for (int j = 0; j < 10; ++j)
      if (overlap(outs[i], ni, ins[j], j < 5 ? nh : nl)) return UG_ERR_ALIAS;
    if (overlap(outs[i], ni, lse, nlse)) return UG_ERR_ALIAS;
    for (int j = i + 1; j < 6; ++j)
      if (overlap(outs[i], ni, outs[j], j < 3 ? nh : nl)) return UG_ERR_ALIAS;
  }
  for (int i = 0; i < 10; ++i)
    if ((i < 5 || lr) && !aligned16(ins[i])) return UG_ERR_ALIGNMENT;
  for (int i = 0; i < 6; ++i)
    if ((i < 3 || lr) && !aligned16(outs[i])) return UG_ERR_ALIGNMENT;
  if (!aligned16(lse)) return UG_ERR_ALIGNMENT;
  if (const int st = check_device(p)) return st;
  auto up = [](int64_t n) { return (n + 255) / 256 * 256; };
  char* w = static_cast<char*>(workspace);
  void* q_wf = w;
  void* k_wf = w + up(nh);
  void* v_wf = w + 2 * up(nh);
  void* o_wf = w + 3 * up(nh);
  void* do_wf = w + 4 * up(nh);
  void* dq_wf = w + 5 * up(nh);
  void* dk_wf = w + 6 * up(nh);
  void* dv_wf = w + 7 * up(nh);
  void* q_lr_r = w + 8 * up(nh);
  void* k_lr_r = w + 8 * up(nh) + up(nl);
  void* delta = w + 8 * up(nh) + 2 * up(nl);
  int st;
  if ((st = ug_permute_rope_window_first(p, q_hr, q_wf, s)) != UG_OK) return st;
  if ((st = ug_permute_rope_window_first(p, k_hr, k_wf, s)) != UG_OK) return st;
  // Where 128-row tiles are whole window rows, the attention backward reads
  // v, o, dO and writes dv in raster order itself (no permutes of v, o, dO,
  // no unpermute of dv).
  const bool raster = vo_raster_supported(p->g);
  if (!raster) {
    if ((st = ug_permute_window_first(p, v_hr, v_wf, s)) != UG_OK) return st;
    if ((st = ug_permute_window_first(p, o_hr, o_wf, s)) != UG_OK) return st;
    if ((st = ug_permute_window_first(p, do_hr, do_wf, s)) != UG_OK) return st;
  }
  if (lr) {
    if ((st = ug_rope_2d(p, q_lr, q_lr_r, UG_LR, s)) != UG_OK) return st;
    if ((st = ug_rope_2d(p, k_lr, k_lr_r, UG_LR, s)) != UG_OK) return st;
  }
  // global dq, dk land in the outputs in the rotated frame, then rotate back in place
  if (raster)
    st = ug_hier_local_attn_bwd_vo_raster(p, q_wf, k_wf, v_hr, q_lr_r, k_lr_r, v_lr, o_hr, o_lr,
                                          do_hr, do_lr, lse, dq_wf, dk_wf, dv_hr, dq_lr, dk_lr,
                                          dv_lr, delta, ug_attn_bwd_workspace_bytes(p), s);
  else
    st = ug_hier_local_attn_bwd(p, q_wf, k_wf, v_wf, q_lr_r, k_lr_r, v_lr, o_wf, o_lr, do_wf,
                                do_lr, lse, dq_wf, dk_wf, dv_wf, dq_lr, dk_lr, dv_lr, delta,
                                ug_attn_bwd_workspace_bytes(p), s);
  if (st != UG_OK) return st;
  if ((st = ug_unpermute_rope_bwd(p, dq_wf, dq_hr, s)) != UG_OK) return st;
  if ((st = ug_unpermute_rope_bwd(p, dk_wf, dk_hr, s)) != UG_OK) return st;
  if (!raster && (st = ug_unpermute(p, dv_wf, dv_hr, s)) != UG_OK) return st;
  if (lr) {
    if ((st = ug_rope_2d_bwd(p, dq_lr, dq_lr, UG_LR, s)) != UG_OK) return st;
    if ((st = ug_rope_2d_bwd(p, dk_lr, dk_lr, UG_LR, s)) != UG_OK) return st;
  }
  return UG_OK;
}

int ug_plan_set_wait_timeout(ug_plan* p, int64_t ns) {
  if (!p || ns <= 0) return UG_ERR_INVALID_ARG;
  p->wait_timeout_ns = ns;
  return UG_OK;
}

int ug_warm_start(const ug_warm_start_params* q, const float* x_lr, const float* noise,
                  float* out, void* s) {
  if (!q || !x_lr || !noise || !out) return UG_ERR_INVALID_ARG;
  if (q->batch < 1 || q->channels < 1 || q->lr_h < 1 || q->lr_w < 1 || q->scale < 1)
    return UG_ERR_INVALID_ARG;
  if ((int64_t)q->batch * q->channels > 65535) return UG_ERR_INVALID_ARG;
  if ((int64_t)q->lr_h * q->scale > (1 << 24) || (int64_t)q->lr_w * q->scale > (1 << 24))
    return UG_ERR_INVALID_ARG;
  if (!std::isfinite(q->sharpen) || !(q->t >= 0.0f && q->t <= 1.0f)) return UG_ERR_INVALID_ARG;
  if (!aligned16(x_lr) || !aligned16(noise) || !aligned16(out)) return UG_ERR_ALIGNMENT;
  const int64_t planes = (int64_t)q->batch * q->channels;
  const int64_t lo = planes * q->lr_h * q->lr_w * 4;
  const int64_t hi = planes * ((int64_t)q->lr_h * q->scale) * ((int64_t)q->lr_w * q->scale) * 4;
  if (overlap(out, hi, x_lr, lo)) return UG_ERR_ALIAS;
  if (out != noise && overlap(out, hi, noise, hi)) return UG_ERR_ALIAS;
  return launch_warm_start(q, x_lr, noise, out, as_stream(s));
}

int ug_warm_start_stencil_weights(float sharpen, float t, float* weights) {
  if (!weights || !std::isfinite(sharpen) || !(t >= 0.0f && t <= 1.0f)) return UG_ERR_INVALID_ARG;
  warm_start_stencil_weights(sharpen, t, weights);
  return UG_OK;
}

int ug_check_error(const ug_plan* p, void* s) {
  if (!p) return UG_ERR_INVALID_ARG;
  if (const int st = check_device(p)) return st;
  if (cudaStreamSynchronize(as_stream(s)) != cudaSuccess) return UG_ERR_CUDA;
  int h = 0;
  if (cudaMemcpy(&h, p->d_err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return UG_ERR_CUDA;
  if (h != 0) {
    const int zero = 0;
    if (cudaMemcpy(p->d_err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
      return UG_ERR_CUDA;
    return h;
  }
  if (cudaGetLastError() != cudaSuccess) return UG_ERR_CUDA;
  return UG_OK;
}

}  // extern "C"
