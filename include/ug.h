/*
 * ug.h -- C ABI of a B200 (sm_100a) library for one hierarchical-local-
 * attention layer of UltraGen ("UltraGen: Efficient Ultra-High-Resolution
 * Image Generation with Hierarchical Local Attention", arXiv 2510.16325).
 *
 * The layer, as the gist.science summaries of the paper state it
 * (UltraGen-it, -fr, -es, -ar, -ko; sections cited per call below):
 *   1. the high-res latent token grid is cut into fixed, non-overlapping
 *      windows and its tokens are reordered window-first, so that each window
 *      is one contiguous run of the sequence;
 *   2. 2-D RoPE is applied; the positions of the low-res guidance tokens are
 *      multiplied by rho (4 on the pages) to land on the high-res scale;
 *   3. attention is block sparse: every high-res window attends to itself,
 *      its neighbouring windows and all low-res tokens under one softmax; the
 *      low-res tokens attend to each other only;
 *   4. the high-res output is put back into raster order.
 *
 * Conventions shared by every call
 *   - Tensors are bf16, contiguous, laid out [batch, tokens, heads, head_dim]
 *     ("token-major"); the caller owns them.  Every device pointer must be
 *     16-byte aligned (UG_ERR_ALIGNMENT otherwise).
 *   - High-res tokens: N = grid_h * grid_w.  Raster order: token r sits at
 *     row r / grid_w, column r % grid_w.  Window-first order: windows in
 *     raster order (w = wy * (grid_w / win_w) + wx), each window's
 *     T = win_h * win_w tokens in raster order inside it, so window w is the
 *     range [w*T, (w+1)*T).
 *   - Global tokens: the tensors named *_lr hold L = text_len + lr_h * lr_w
 *     rows: the text tokens first (the MMDiT joint sequence concatenates
 *     text, high-res and low-res tokens: UltraGen-it §2, LoRA item;
 *     UltraGen-fr §2.C), then the low-res guidance grid in raster order.
 *     They are never permuted.  Text tokens are seen by every query and see
 *     the global tokens only, exactly like the low-res tokens; they carry no
 *     grid position, so RoPE leaves them unchanged.
 *   - Launches are asynchronous on the given stream (a cudaStream_t passed as
 *     a void*, NULL = the legacy default stream); nothing synchronises except
 *     ug_check_error.  Only ug_plan_create allocates device memory and only
 *     ug_plan_destroy frees it.
 *   - Every call returns a ug_status; no C++ exception crosses the ABI.
 *     Argument errors are reported before any work is queued.
 *   - A plan belongs to the device that was current when it was created:
 *     every call taking a plan must run with that device current
 *     (UG_ERR_INVALID_ARG otherwise), because the plan's tables live in that
 *     device's memory.  Plans on several devices of one process, and calls
 *     from several host threads, are supported.
 */
#ifndef UG_H_
#define UG_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum ug_status {
  UG_OK = 0,
  UG_ERR_INVALID_ARG = 1,  /* null pointer, bad geometry, bad token set         */
  UG_ERR_UNSUPPORTED = 2,  /* a valid geometry the library does not run        */
  UG_ERR_ALIGNMENT = 3,    /* a device pointer not 16-byte aligned              */
  UG_ERR_ALIAS = 4,        /* output overlaps an input where that is not allowed */
  UG_ERR_CUDA = 5,         /* a CUDA runtime/driver call failed                 */
  UG_ERR_TIMEOUT = 6,      /* a bounded device-side wait expired (kernel gave up) */
  UG_ERR_NO_MEMORY = 7     /* host or device allocation failed in ug_plan_create */
} ug_status;

/* Token sets for ug_rope_2d: which grid the rows of x belong to and in which
 * order, hence which RoPE positions they take. */
typedef enum ug_token_set {
  UG_HR_WINDOW_FIRST = 0, /* [B, N, h, d], high-res, window-first order */
  UG_HR_RASTER = 1,       /* [B, N, h, d], high-res, raster order       */
  UG_LR = 2               /* [B, L, h, d], low-res, raster order        */
} ug_token_set;

/* Problem statement (UltraGen-fr §2.A-B, UltraGen-ar §2.أ-ب): the token grid,
 * the fixed window, the neighbourhood radius, the low-res grid and its RoPE
 * scale rho, heads and head dim, the axial RoPE split. */
typedef struct ug_geom {
  int32_t batch;       /* B >= 1                                              */
  int32_t grid_h;      /* high-res token grid H x W                           */
  int32_t grid_w;
  int32_t win_h;       /* window in tokens; must divide the grid exactly      */
  int32_t win_w;
  int32_t radius;      /* neighbourhood in windows, Chebyshev (1 -> 3x3)      */
  int32_t lr_h;        /* low-res grid; 0 x 0 = no low-res tokens             */
  int32_t lr_w;
  double rho;          /* low-res RoPE position scale (4 on the pages), > 0   */
  int32_t heads;       /* h >= 1                                              */
  int32_t head_dim;    /* d; the attention runs d in {64, 128}                */
  int32_t rope_dim_y;  /* channels [0, a_y) rotate with the row position      */
  int32_t rope_dim_x;  /* channels [a_y, d) with the column; a_y + a_x = d,   */
                       /* each a multiple of 8                                */
  double rope_theta;   /* RoPE base, > 1 (10000)                               */
  float softmax_scale; /* 0 -> 1/sqrt(head_dim)                               */
  int32_t text_len;    /* text tokens at the head of the global tensors, >= 0 */
} ug_geom;

typedef struct ug_plan ug_plan; /* opaque: geometry, device index lists, RoPE
                                   tables, device error word */

/* ---- host-only helpers (no GPU needed) ---------------------------------- */

/* Checks a geometry.  UG_OK, UG_ERR_INVALID_ARG (null, non-positive sizes,
 * windows that do not tile the grid, a RoPE split that does not sum to d or
 * has a segment not a multiple of 8, lr_h*lr_w == 0 with one of them != 0,
 * rho <= 0, theta <= 1, negative radius or text_len, sizes whose element count passes
 * 2^31 per tensor) or UG_ERR_UNSUPPORTED. */
int ug_geom_validate(const ug_geom* g);

/* Element counts of the three index maps of ug_build_index_maps. */
int ug_index_map_sizes(const ug_geom* g, int64_t* n_perm, int64_t* n_nbr_off,
                       int64_t* n_nbr_idx);

/* Index maps, into caller-owned host arrays (sizes from ug_index_map_sizes):
 *   perm[r]  (N entries): window-first position of raster token r
 *            (UltraGen-fr §2.A "Ordre Window-First");
 *   nbr_off  (nWin + 1) / nbr_idx: CSR lists, per window w (raster window
 *            id), of the windows it attends to: Chebyshev distance <= radius,
 *            clipped at the grid border, itself included, ascending
 *            (UltraGen-ar §2.ب, attention mask, first item). */
int ug_build_index_maps(const ug_geom* g, int32_t* perm, int32_t* nbr_off, int32_t* nbr_idx);

/* Visible (query, key) pairs per (batch element, head): high-res query with
 * high-res key, high-res query with global key, global with global (global =
 * text and low-res tokens, L = text_len + lr_h * lr_w of them).  The
 * useful FLOPs of the attention are 4 * head_dim * heads * batch * (sum). */
int ug_visible_pairs(const ug_geom* g, int64_t* hr_hr, int64_t* hr_lr, int64_t* lr_lr);

/* Element counts of the attention work lists of ug_build_work_lists. */
int ug_work_list_sizes(const ug_geom* g, int64_t* n_qctas, int64_t* n_kvlist, int64_t* n_kctas,
                       int64_t* n_qlist);

/* The work lists the attention kernels walk, into caller-owned host arrays
 * (sizes from ug_work_list_sizes; any pointer may be NULL):
 *   qctas  (4 per forward query CTA): token set (0 high-res, 1 global), first
 *          query row, offset and length of its slice of kvlist.  A CTA owns
 *          256 rows (two 128-row tiles) of its token set.
 *   kvlist: one entry per 128-key block a CTA must visit: bits 0-28 the block
 *          index (keys [128 i, 128 i + 128) of its tensor), bit 29 set for
 *          the global tensor, bit 30 set when some in-range (query, key) pair
 *          of the CTA and block is invisible or the block passes the end of
 *          its tensor (the kernel then tests each pair; rows past the end of
 *          the query tensor are computed but never written).
 *   kctas  (4 per backward key CTA): token set, first key, offset and length
 *          of its slice of qlist.
 *   qlist: one entry per 128-row query tile a key CTA must visit, same bit
 *          layout; bit 30 marks an invisible in-range pair.
 * Host only, no GPU needed. */
int ug_build_work_lists(const ug_geom* g, int32_t* qctas, uint32_t* kvlist, int32_t* kctas,
                        uint32_t* qlist);

const char* ug_status_string(int status);

/* ---- plan ---------------------------------------------------------------- */

/* Validates g, builds the index maps, the attention work lists and the RoPE
 * tables on the host, allocates device memory for them and copies them once
 * (synchronously) to the current CUDA device.  *out is NULL on failure. */
int ug_plan_create(const ug_geom* g, ug_plan** out);
int ug_plan_destroy(ug_plan* plan); /* NULL is allowed; synchronises the device */

/* The plan's index maps, copied into caller-owned host arrays (as
 * ug_build_index_maps).  Any of the three pointers may be NULL. */
int ug_get_index_maps(const ug_plan* plan, int32_t* perm, int32_t* nbr_off, int32_t* nbr_idx);

/* ---- the four steps of the layer (device pointers) ----------------------- */

/* Step 1.  dst_wf[b, perm[r]] = src_raster[b, r] for every high-res token,
 * whole [h, d] rows copied bit for bit.  src/dst: [B, N, h, d] bf16.
 * UG_ERR_ALIAS if the two ranges overlap.
 * (UltraGen-fr §2.A "Ordre Window-First"; UltraGen-es §2, window-first
 * permutation bullet; UltraGen-ar §2.أ.) */
int ug_permute_window_first(const ug_plan* plan, const void* src_raster, void* dst_wf,
                            void* stream);

/* Steps 1 and 2 in one pass: dst_wf[b, perm[r]] = RoPE(src_raster[b, r]) at
 * the token's grid position, for high-res queries and keys.  Bit for bit the
 * same as ug_permute_window_first followed by ug_rope_2d(UG_HR_WINDOW_FIRST)
 * (the rotation depends only on the token's position), with one read and one
 * write of the tensor instead of two each.  src/dst: [B, N, h, d] bf16;
 * UG_ERR_ALIAS if they overlap.  (UltraGen-fr §2.A "Ordre Window-First" and
 * §2.B; UltraGen-ar §2.ب "Scaled Positional Embeddings".) */
int ug_permute_rope_window_first(const ug_plan* plan, const void* src_raster, void* dst_wf,
                                 void* stream);

/* Step 4.  dst_raster[b, r] = src_wf[b, perm[r]]; the inverse of step 1. */
int ug_unpermute(const ug_plan* plan, const void* src_wf, void* dst_raster, void* stream);

/* Step 2.  2-D axial RoPE of x into y (y == x allowed; any other overlap is
 * UG_ERR_ALIAS).  x, y: [B, N, h, d] (high-res sets) or [B, L, h, d] (UG_LR,
 * the global tokens: rows [0, text_len) are text and are copied unchanged).
 * A high-res token at grid (row, col) takes positions (row, col); the low-res
 * token (i, j) takes (rho*i, rho*j) (UltraGen-ar §2.ب "Scaled Positional
 * Embeddings": the low-res position indices are multiplied by rho; UltraGen-fr
 * §2.B).  Channels [0, a_y) rotate by pos_row * f_k, channels [a_y, d) by
 * pos_col * f_k, f_k = theta^(-2k/a) for the k-th adjacent channel pair
 * (2k, 2k+1) of the segment of a channels: (x0, x1) -> (x0 c - x1 s,
 * x0 s + x1 c), c and s the fp32-rounded fp64 cos/sin of the angle.  Each
 * output is formed from exact fp64 products, one fp64 add, and one
 * round-to-nearest-even to bf16, so results are reproducible bit for bit.
 * Applied to queries and keys, never to values. */
int ug_rope_2d(const ug_plan* plan, const void* x, void* y, int token_set, void* stream);

/* Step 3.  Block-sparse joint attention (UltraGen-ar §2.ب "Attention
 * Masking"; UltraGen-es §2, guidance item; UltraGen-it §2, one softmax over a
 * window's own tokens and the guidance).  Inputs (already rotated):
 *   q_hr, k_hr, v_hr: [B, N, h, d], high-res, WINDOW-FIRST order;
 *   q_lr, k_lr, v_lr: [B, L, h, d], global tokens, text then low-res
 *                     (ignored, may be NULL, if L = 0).
 * A high-res query of window w sees the high-res keys of every window within
 * Chebyshev distance radius of w and every global key; a global (text or
 * low-res) query sees the global keys only; scores are softmax_scale * <q, k>,
 * one softmax per
 * query over everything it sees, output = probabilities times values.
 * Outputs: o_hr [B, N, h, d] (window-first), o_lr [B, L, h, d], bf16, fp32
 * accumulation; lse (optional, NULL to skip): fp32 [B, h, N + L], natural
 * log of the softmax denominator, high-res rows first (window-first order).
 * The outputs may not overlap any input (UG_ERR_ALIAS).  Requires
 * d in {64, 128} (UG_ERR_UNSUPPORTED).  A device-side wait that exceeds its
 * bound makes the kernel give up and record UG_ERR_TIMEOUT, read by
 * ug_check_error. */
int ug_hier_local_attn_fwd(const ug_plan* plan, const void* q_hr, const void* k_hr,
                           const void* v_hr, const void* q_lr, const void* k_lr,
                           const void* v_lr, void* o_hr, void* o_lr, float* lse, void* stream);

/* Step 3 reading v and writing o in raster order, which removes the
 * permutation of v and the unpermutation of o from the layer.  The same
 * attention as ug_hier_local_attn_fwd with q_hr, k_hr window-first (rotated)
 * but v_hr_raster [B, N, h, d] in raster order and o_hr_raster written in
 * raster order; the global tensors and lse (high-res rows window-first) as
 * there.  Each 128-key tile of V is read as 128 / win_w whole rows of one
 * window, so the call needs win_w dividing 128 and 128 dividing
 * win_h * win_w (UG_ERR_UNSUPPORTED otherwise; the 2K, 4K, 8K and 4K-CFG
 * geometries qualify).  ug_layer_fwd uses it where it applies. */
int ug_hier_local_attn_fwd_vo_raster(const ug_plan* plan, const void* q_hr, const void* k_hr,
                                     const void* v_hr_raster, const void* q_lr, const void* k_lr,
                                     const void* v_lr, void* o_hr_raster, void* o_lr, float* lse,
                                     void* stream);

/* ---- the whole layer ------------------------------------------------------ */

/* Bytes of device scratch that ug_layer_fwd needs (window-first copies of the
 * high-res q, k, v and o, rotated global q and k), or -1 for a NULL plan. */
int64_t ug_layer_workspace_bytes(const ug_plan* plan);

/* Steps 1-4 in order on raster-order inputs: window-first permute of
 * q_hr, k_hr, v_hr (q and k with their RoPE applied in the same pass, as
 * ug_permute_rope_window_first); RoPE of the global q and k (rho-scaled
 * low-res positions, text rows unchanged); attention; unpermute of the
 * high-res output into o_hr (raster order).  Where
 * ug_hier_local_attn_fwd_vo_raster applies, the attention reads v_hr and
 * writes o_hr in raster order itself instead.  q/k/v are not modified.  lse as in
 * ug_hier_local_attn_fwd (its high-res rows stay in window-first order).
 * workspace: caller-owned device scratch of at least
 * ug_layer_workspace_bytes(plan) bytes, 256-byte aligned; the call uses it
 * for intermediates only. */
int ug_layer_fwd(const ug_plan* plan, const void* q_hr, const void* k_hr, const void* v_hr,
                 const void* q_lr, const void* k_lr, const void* v_lr, void* o_hr, void* o_lr,
                 float* lse, void* workspace, int64_t workspace_bytes, void* stream);

/* Capacity in bytes of the static scratch of ug_layer_fwd_static_scratch. */
#define UG_STATIC_SCRATCH_BYTES (32ll << 20)

/* The paper has no counterpart to this call; it exists for callers that must
 * not allocate device memory while they run the layer: servers that reserve
 * device memory at start-up and forbid allocation while serving (cudaMalloc
 * can synchronise the device and fragments a tuned pool), real-time
 * pipelines with a fixed latency budget, hosts where another component owns
 * all device memory.
 * Same arguments and results as ug_layer_fwd without the workspace: the
 * intermediates live in one static device array of UG_STATIC_SCRATCH_BYTES
 * (32 MiB) that every GPU which loads this library holds until the process
 * exits.  The call allocates nothing (no cudaMalloc/cudaFree, no allocating
 * library routine); the plan is created beforehand, at set-up, by
 * ug_plan_create (which does allocate).
 *   - UG_ERR_UNSUPPORTED, before any work is queued, when the plan's
 *     ug_layer_workspace_bytes exceeds UG_STATIC_SCRATCH_BYTES;
 *     UG_ERR_INVALID_ARG when the plan's device is not the current device.
 *   - ug_plan_create looks up the array's device address
 *     (cudaGetSymbolAddress) once per device, with the plan's device
 *     current; that lookup is also what loads the array onto the device, so
 *     it happens at set-up and not on this call's path.  Create the plan
 *     before any stream capture.
 *   - Every call shares the one array, which keeps the last call's contents.
 *     Nothing in it needs clearing (each call writes what it reads), but calls
 *     that overlap on the GPU race on it: issue them on one stream. */
int ug_layer_fwd_static_scratch(const ug_plan* plan, const void* q_hr, const void* k_hr,
                                const void* v_hr, const void* q_lr, const void* k_lr,
                                const void* v_lr, void* o_hr, void* o_lr, float* lse,
                                void* stream);

/* ---- backward pass ------------------------------------------------------------
 * Gradients of the layer for training (the pages train LoRA adapters on the
 * q/k/v projections of the low-res guidance: UltraGen-ar §2.ج, UltraGen-fr
 * §2.C).  With P the forward's probabilities (recomputed from its lse),
 * D = rowsum(dO * O), dP = dO V^T and dS = P * (dP - D):
 *   dQ = scale * dS K,  dK = scale * dS^T Q,  dV = P^T dO;
 * RoPE's gradient is the transposed rotation; the permutation's is its
 * inverse.  bf16 in and out, fp32 accumulation; P and dS are rounded to bf16
 * as tensor-core operands. */

/* Transposed rotation of ug_rope_2d (the same fp32 cos/sin, sine negated):
 * dx = R^T dy per channel pair, bit-reproducible like ug_rope_2d.  dy == dx
 * is allowed; text rows of UG_LR are copied. */
int ug_rope_2d_bwd(const ug_plan* plan, const void* dy, void* dx, int token_set, void* stream);

/* The inverse of ug_permute_rope_window_first for gradients:
 * dst_raster[b, r] = R^T(src_wf[b, perm[r]]) at raster token r's position,
 * in one pass.  UG_ERR_ALIAS if the ranges overlap. */
int ug_unpermute_rope_bwd(const ug_plan* plan, const void* src_wf, void* dst_raster,
                          void* stream);

/* Device scratch of ug_hier_local_attn_bwd: D, fp32 [B, h, N + L]. */
int64_t ug_attn_bwd_workspace_bytes(const ug_plan* plan);

/* Gradients of ug_hier_local_attn_fwd.  Inputs as its inputs (rotated q, k;
 * high-res window-first), plus its outputs o_hr/o_lr and lse (required), and
 * the output gradients do_hr [B, N, h, d] (window-first) and do_lr
 * [B, L, h, d].  Outputs dq/dk/dv in the layouts of q/k/v (the *_lr ones
 * ignored, may be NULL, if L = 0).  workspace: device, 16-byte aligned, at
 * least ug_attn_bwd_workspace_bytes.  Outputs and workspace may not overlap
 * each other or any input (UG_ERR_ALIAS).  d in {64, 128}.  Device waits are
 * bounded as in the forward (UG_ERR_TIMEOUT via ug_check_error); a device
 * whose dynamic shared memory is not 1024-byte aligned makes the dK/dV
 * kernel record UG_ERR_UNSUPPORTED. */
int ug_hier_local_attn_bwd(const ug_plan* plan, const void* q_hr, const void* k_hr,
                           const void* v_hr, const void* q_lr, const void* k_lr,
                           const void* v_lr, const void* o_hr, const void* o_lr,
                           const void* do_hr, const void* do_lr, const float* lse, void* dq_hr,
                           void* dk_hr, void* dv_hr, void* dq_lr, void* dk_lr, void* dv_lr,
                           void* workspace, int64_t workspace_bytes, void* stream);

/* ug_hier_local_attn_bwd with the high-res v, o, dO read and dv written in
 * raster order (q, k, dq, dk stay window-first; the global tensors as
 * before), so that the layer's backward needs no permutes of v, o and dO and
 * no unpermute of dv.  As ug_hier_local_attn_fwd_vo_raster, it needs every
 * 128-row tile to be whole rows of one window: win_w dividing 128 and 128
 * dividing win_h * win_w (UG_ERR_UNSUPPORTED otherwise).  Results equal the
 * window-first call's, permuted, bit for bit.  ug_layer_bwd uses it where it
 * applies. */
int ug_hier_local_attn_bwd_vo_raster(const ug_plan* plan, const void* q_hr, const void* k_hr,
                                     const void* v_hr_raster, const void* q_lr,
                                     const void* k_lr, const void* v_lr,
                                     const void* o_hr_raster, const void* o_lr,
                                     const void* do_hr_raster, const void* do_lr,
                                     const float* lse, void* dq_hr, void* dk_hr,
                                     void* dv_hr_raster, void* dq_lr, void* dk_lr, void* dv_lr,
                                     void* workspace, int64_t workspace_bytes, void* stream);

/* Device scratch of ug_layer_bwd. */
int64_t ug_layer_bwd_workspace_bytes(const ug_plan* plan);

/* Gradients of ug_layer_fwd with respect to its raster-order inputs: given
 * the layer's inputs q/k/v, its outputs o_hr (raster) / o_lr and lse, and
 * do_hr (raster) / do_lr, writes dq/dk/dv (same layouts as q/k/v; dq, dk
 * are gradients w.r.t. the unrotated q, k).  Recomputes the window-first,
 * rotated operands, runs ug_hier_local_attn_bwd (or its raster variant where
 * that applies: then v, o, dO are read and dv written in raster order
 * directly), then the inverse permutation with the transposed RoPE.  workspace: at least
 * ug_layer_bwd_workspace_bytes, 256-byte aligned, disjoint from every
 * argument. */
int ug_layer_bwd(const ug_plan* plan, const void* q_hr, const void* k_hr, const void* v_hr,
                 const void* q_lr, const void* k_lr, const void* v_lr, const void* o_hr,
                 const void* o_lr, const float* lse, const void* do_hr, const void* do_lr,
                 void* dq_hr, void* dk_hr, void* dv_hr, void* dq_lr, void* dk_lr, void* dv_lr,
                 void* workspace, int64_t workspace_bytes, void* stream);

/* ---- warm-start initialisation -------------------------------------------- */

/* Sizes and constants of ug_warm_start. */
typedef struct ug_warm_start_params {
  int32_t batch;     /* B >= 1                                               */
  int32_t channels;  /* C >= 1 latent channels; B * C <= 65535               */
  int32_t lr_h;      /* low-res latent h x w, >= 1                            */
  int32_t lr_w;
  int32_t scale;     /* integer factor s >= 1: the high-res latent is        */
                     /* (h*s) x (w*s), each side at most 2^24                */
  float sharpen;     /* unsharp-mask amount (finite; 0 = no sharpening)      */
  float t;           /* timestep in [0, 1]: 0 = the sharpened upsample,      */
                     /* 1 = pure noise                                        */
} ug_warm_start_params;

/* Warm-start of the high-res state (UltraGen-ar §2.د "Warm-Start
 * Initialization": the low-res guidance is upsampled, sharpened and added to
 * the high-res representation at an intermediate timestep; UltraGen-fr §2.D:
 * Gaussian noise combined with the upscaled low-res image).  Per plane of
 * x_lr [B, C, h, w] fp32:
 *   u   = bilinear upsampling by s with half-pixel centres: high-res pixel
 *         (y, x) samples ((y + 0.5)/s - 0.5, (x + 0.5)/s - 0.5), low-res
 *         indices clamped to the image;
 *   x0  = u + sharpen * (u - blur(u)), blur the 3x3 binomial filter
 *         (1/4, 1/2, 1/4) per axis with edges replicated;
 *   out = (1 - t) * x0 + t * noise           (rectified-flow interpolation).
 * noise and out: [B, C, h*s, w*s] fp32, device, 16-byte aligned; the caller
 * draws the noise.  out == noise is allowed (in place); any other overlap of
 * out with an input is UG_ERR_ALIAS.  fp32 arithmetic: within a few fp32
 * ulps of the exact value.  No plan is needed. */
int ug_warm_start(const ug_warm_start_params* params, const float* x_lr, const float* noise,
                  float* out, void* stream);

/* Host only (no GPU needed): the weights ug_warm_start applies for factor
 * s = 4.  The map above is linear in x_lr, and output pixel (4Y + py,
 * 4X + px) of a plane depends only on the 3 x 3 low-res neighbourhood of
 * (Y, X):
 *   out = sum_{r, c = 0..2} weights[(4 py + px) * 9 + 3 r + c]
 *                           * x_lr[clamp(Y + r - 1)][clamp(X + c - 1)] + t * noise,
 * indices clamped to the image (which also gives the blur's edge
 * replication: the high-res rows and columns just outside the image sample
 * only clamped source pixels, so they equal the border ones).  Writes the
 * UG_WARM_START_STENCIL_WEIGHTS fp32 weights, computed in fp64 and rounded
 * once; the caller owns the array.  UG_ERR_INVALID_ARG for a NULL pointer, a
 * non-finite sharpen or t outside [0, 1]. */
#define UG_WARM_START_STENCIL_WEIGHTS 144
int ug_warm_start_stencil_weights(float sharpen, float t, float* weights);

/* ---- errors ---------------------------------------------------------------- */

/* Bound, in ns, on each device-side wait of this plan's attention kernel
 * (default 2e9).  A wait that exceeds it makes the kernel record
 * UG_ERR_TIMEOUT, stop issuing work, let its in-flight loads and MMAs finish,
 * free its tensor memory and exit; later CTAs of the launch skip their work.
 * A very small bound makes ordinary waits expire, which exercises that path
 * without any fault.  UG_ERR_INVALID_ARG for a NULL plan or ns <= 0. */
int ug_plan_set_wait_timeout(ug_plan* plan, int64_t ns);

/* Synchronises `stream`, then returns (and clears) the first status a kernel
 * of this plan recorded on the device (UG_ERR_TIMEOUT), else UG_ERR_CUDA if
 * the stream reports an error, else UG_OK. */
int ug_check_error(const ug_plan* plan, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* UG_H_ */
