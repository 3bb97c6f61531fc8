/*
 * splat.h -- C ABI of libsplat: tile-based 3D Gaussian Splatting render followed by the analytic
 * score replay, for NVIDIA B200 (sm_100a).
 *
 * Sources (web pages, cited by title and section):
 *   [P1] "Research Proposal: Renderer Score Tokens for Recurrent Gaussian Splatting"
 *        - "Two-Stage Algorithm", Stage 1 (standard render: gsplat tile binning, contributor
 *          sorting, front-to-back compositing, residual; tile bins and sorted contributor
 *          indices stay in the renderer workspace) and Stage 2 (analytic score replay, suffix
 *          composite equation, masked per-Gaussian accumulation);
 *        - "Exact Score Operators" (o = sigmoid(a), alpha = o G, w = T alpha; rho and q; opacity
 *          logit score; SH score; projected-centre mean score; projection Jacobian J; cross-view
 *          weights gamma; covector pullback b; conditioning matrix A and its statistics);
 *        - "Final Token and Updater" (token z_g of dimension 9 + 3 d_SH).
 *   [P5] "ATSplat: Compact Feed-forward 3D Gaussian Splatting with Adaptive Token Expansion",
 *        prerequisites section (the 3DGS primitive: centre, rotation, scale, opacity, SH).
 *
 * Conventions for every call:
 *   - All array arguments are DEVICE pointers (cudaMalloc / torch CUDA tensors) on the device
 *     that was current when the workspace was created, C-contiguous fp32/int32 as stated, 4-byte
 *     aligned. The caller owns them; the library never frees or retains them past the call
 *     except where a call says so.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream). Every call
 *     only enqueues work on that stream and returns; the exception is splat_bin_sort, which
 *     waits for the per-view instance counts (a few words that kernels store into mapped
 *     pinned host memory). Nothing a call enqueues uses a copy engine: clears and these small
 *     exchanges are kernels, so a step never waits behind the caller's large host<->device
 *     copies on other streams. (When splat_bin_sort has to grow the instance lists -- the first
 *     step of a workspace, or more instances than before -- the device allocation synchronises
 *     with every stream; steady-state steps allocate nothing.)
 *   - Return value: SPLAT_OK (0) or a negative splat_status. No C++ exception crosses the ABI.
 *     On error, splat_last_error(ws) returns a NUL-terminated message owned by the workspace,
 *     valid until the next call on it. Argument errors are detected before any work is
 *     enqueued. A workspace is not thread-safe: one host thread at a time.
 *   - Call order per problem: splat_project -> splat_bin_sort -> splat_render, then any of
 *     splat_score_replay, splat_score_partials, splat_backward, splat_render_features,
 *     splat_scatter, splat_attribution (each reads the last render). A call made out of order
 *     returns SPLAT_ERR_STATE.
 */
#ifndef SPLAT_H
#define SPLAT_H

#ifdef __cplusplus
extern "C" {
#endif

typedef struct splat_ws splat_ws; /* opaque, library-owned workspace */

typedef enum splat_status {
  SPLAT_OK = 0,
  SPLAT_ERR_INVALID_ARG = -1,    /* null/misaligned/host pointer, size out of range */
  SPLAT_ERR_CAPACITY = -2,       /* sizes above the workspace maxima or 2^31 instances */
  SPLAT_ERR_STATE = -3,          /* calls out of order */
  SPLAT_ERR_CUDA = -4,           /* a CUDA runtime call or kernel launch failed */
  SPLAT_ERR_BOUNDS = -5,         /* a device-side bounds check failed (reported, access skipped) */
  SPLAT_ERR_DEVICE_TIMEOUT = -6, /* reserved: a bounded device-side wait ran out */
  SPLAT_ERR_OOM = -7             /* device allocation failed */
} splat_status;

/*
 * Create a workspace on the current device for problems with at most max_G Gaussians, max_V
 * views of at most max_H x max_W pixels and SH degree <= max_sh_degree (0..3). Allocates the
 * per-(Gaussian, view) records and accumulators up front; the instance (tile, Gaussian) lists
 * grow on demand inside splat_bin_sort. *ws is set to NULL on failure. SPLAT_ERR_CAPACITY when
 * an image has more 16x16 tiles, ceil(max_W/16) ceil(max_H/16), than the binning kernels' shared
 * memory holds per-warp counts for (7,264 tiles).
 */
int splat_ws_create(splat_ws** ws, int max_G, int max_V, int max_H, int max_W,
                    int max_sh_degree);

/* Free all device and host memory of the workspace (synchronises its device). NULL is a no-op. */
void splat_ws_destroy(splat_ws* ws);

/* Message describing the last error on this workspace ("" when none). */
const char* splat_last_error(const splat_ws* ws);

/*
 * Stage 1 preprocess ([P1] Stage 1 "original gsplat"; [P5] 3DGS primitive; [P1] "Projected-Center
 * Mean Partial Score" for G and Sigma2D): for every Gaussian g and view v, the camera-space centre,
 * the EWA 2-D covariance Sigma2D = J W Sigma3D W^T J^T + 0.3 I and its inverse (the conic), the
 * 3-sigma footprint radius and its rectangle of 16x16 tiles, the opacity o = sigmoid(a), the view
 * direction and the SH colour c = max(0, B(dir) . sh + 0.5). Culled when z <= 0.01, when an input
 * is not finite, for a zero quaternion, det(Sigma2D) <= 0 or an empty tile rectangle.
 *   means       [G,3]   world-space centres
 *   log_scales  [G,3]   per-axis log standard deviations
 *   quats       [G,4]   rotation quaternions (w, x, y, z), normalised here
 *   opac_logits [G]     opacity logits a
 *   sh          [G,d,3] SH coefficients, d = (sh_degree + 1)^2, channel-minor
 *   viewmats    [V,4,4] world-to-camera, row-major; camera x right, y down, z forward
 *   intrin      [V,4]   fx, fy, cx, cy in pixels; pixel (i, j) has centre (i + 0.5, j + 0.5)
 * G >= 0 (G = 0 renders background only), 1 <= V, 1 <= H, W. The input arrays are read by this
 * call only.
 */
int splat_project(splat_ws* ws, const float* means, const float* log_scales, const float* quats,
                  const float* opac_logits, const float* sh, int G, int sh_degree,
                  const float* viewmats, const float* intrin, int V, int H, int W, void* stream);

/*
 * Stage 1 tile binning and contributor sort ([P1] Stage 1 step 1): every visible (g, v) emits one
 * instance per tile of its rectangle; each tile's list is ordered by (camera depth z, Gaussian
 * index) -- a stable radix sort of one fp32 depth key per (view, Gaussian), less the view's
 * smallest visible key, over the width of the key range; emission of the instances in that
 * order; and one stable counting sort by tile.
 * The lists stay in the workspace ([P1] Stage 1: not exposed as a per-pixel tensor).
 * n_instances_out (HOST pointer, may be NULL) receives V counts. Synchronises with the stream
 * once (the counts size the sort).
 */
int splat_bin_sort(splat_ws* ws, long long* n_instances_out, void* stream);

/*
 * Stage 1 front-to-back compositing ([P1] Stage 1 step 2): per pixel, over its tile's list,
 * alpha = min(0.99, o G); entries with a positive exponent or alpha < 1/255 are skipped; the
 * traversal stops before an entry that would take T below 1e-4. Writes
 *   img       [V,H,W,3] C_hat = sum T alpha c + T_final bg
 *   T_final   [V,H,W]   final transmittance
 *   n_contrib [V,H,W]   number of composited Gaussians (int32)
 * bg is a device pointer to 3 floats. The replay reads img back (it is C_hat) and n_contrib (the
 * per-pixel composited counts size its work per warp), and the backward img, T_final and bg, so
 * these must stay unmodified until splat_score_replay / splat_backward have run.
 */
int splat_render(splat_ws* ws, const float* bg, float* img, float* T_final, int* n_contrib,
                 void* stream);

/*
 * Stage 2 analytic score replay and token finalisation ([P1] Stage 2, "Exact Score Operators",
 * "Final Token and Updater"). Re-traverses every pixel's list in the same order and with the same
 * decisions as splat_render, keeps prefix colour P and transmittance T, recovers
 *   C+ = (C_hat - P - T alpha c) / (T (1 - alpha) + 1e-12),
 * masks with M_alpha = (T (1 - alpha) >= 1e-4 and alpha < 0.99) and M_color (colour clamp
 * inactive), forms r = C_hat - C_obs, rho = <r, c - C+>, w = T alpha and accumulates per (g, v)
 *   q = sum w, sum w r, sum M_alpha w rho, sum M_alpha w rho (p - mu2D)
 * in fp32 (per warp either every pixel's own composited entries reduced pair by pair, or each
 * entry summed over the warp first and reduced once; the order of the additions is not fixed, so
 * the last bits vary between runs -- see splat_set_deterministic). Then, per Gaussian over the
 * views where it
 * is visible: q_gv = 1e-6 + q, q_g = 1e-6 + sum_v q_gv, gamma = q_gv / q_g, and
 *   tokens[g] = [ b_mu (3) = sum_v gamma J^T Sigma2D^-1 Sd / q_gv,
 *                 s_alpha (1) = sum_v gamma (1 - o) Sa / q_gv,
 *                 s_SH (3d) = sum_v gamma M_color (B(dir) (x) Swr) / q_gv   (index k*3 + channel),
 *                 log q_g (1),
 *                 eig(A) descending / (tr A + 1e-6) (3),  log(tr A + 1e-6) (1) ],
 *   A = lambda I + sum_v gamma J^T J,  J = d pi_v(mu) / d mu (unclamped pinhole Jacobian).
 *   obs    [V,H,W,3] observed images C_obs
 *   lambda conditioning regulariser (fixed after scene normalisation; 1.0 by default)
 *   tokens [G, 9 + 3d] fp32 output
 */
int splat_score_replay(splat_ws* ws, const float* obs, float lambda, float* tokens,
                       void* stream);

/*
 * splat_render followed by splat_score_replay in one call, with the same outputs (img, T_final,
 * n_contrib, tokens) and the same arithmetic and decisions: in the default accumulation mode the
 * render and the replay run as one kernel -- each warp renders its 8x4 pixel block and replays
 * the entries it composited at once, with the pixel state still in registers, so that across the
 * GPU the render's issue-bound work and the replay's L2 reductions overlap. (Deterministic mode:
 * the two kernels of splat_render and splat_score_replay, one after the other.) The tokens agree
 * with the two-call sequence up to the order of the fp32 reductions. Afterwards the workspace is
 * in the state splat_score_replay leaves (splat_backward, splat_render_features, splat_scatter
 * and splat_attribution may follow, with img, T_final and bg unchanged).
 */
int splat_render_score(splat_ws* ws, const float* bg, const float* obs, float lambda, float* img,
                       float* T_final, int* n_contrib, float* tokens, void* stream);

/*
 * View-sharded replay ([P1] "Exact Score Operators": every cross-view quantity of the token --
 * q_g, the covector pullback, s^alpha, s^SH and A -- is a per-Gaussian sum over views, so the sums
 * of disjoint view sets add). splat_score_partials runs the replay of splat_score_replay for this
 * workspace's views and writes, instead of tokens, the per-Gaussian sums over those views:
 *   partials [G, 11 + 3d] fp32 = [sum_v (1e-6 + q_gv), sum_v J^T Sigma2D^-1 Sd (3),
 *                                 sum_v (1 - o) Sa, sum_v q_gv J^T J (00 01 02 11 12 22),
 *                                 sum_v M_color (B (x) Swr) (3d, index k*3 + channel)].
 * Devices that replay disjoint view sets of one scene add their partials (e.g. an NCCL
 * reduce-scatter over the Gaussian axis) and call splat_finalize_partials on any slice of rows:
 * it turns summed partials [n, 11 + 3d] into tokens [n, 9 + 3d] exactly as splat_score_replay
 * would. splat_finalize_partials needs no workspace and allocates nothing; both are asynchronous
 * on `stream`. On one device, partials of all views give the tokens of splat_score_replay.
 */
int splat_score_partials(splat_ws* ws, const float* obs, float* partials, void* stream);
int splat_finalize_partials(const float* partials, int G, int sh_degree, float lambda,
                            float* tokens, void* stream);

/*
 * Renderer backward: the gradient comparators of [P1] "Relation to Gradient" (raw, detached,
 * support-normalised and parameter-scale-normalised gradients; the pages' "kill test" baseline).
 * Derivatives of L = 1/2 sum over views and pixels of |C_hat - C_obs|^2 (RGB squared loss,
 * [P1] "Exact Score Operators") with the contributor order, the skip and early-stop decisions and
 * the clamp decisions of splat_render held fixed. One back-to-front traversal of the entries
 * splat_render composited (same decisions), from T_final and the background term, forms per
 * entry d C_hat / d alpha = T c - S / (1 - alpha), S the composite behind it (summed as the
 * traversal goes), and per (Gaussian, view) the sums
 *   q = sum w, sum w r, and where alpha = o G < 0.99 with h = <r, d C_hat / d alpha> alpha:
 *   sum h, sum h (p - mu2D), sum h (dx^2, dx dy, dy^2);
 * then one pass per Gaussian chains them through the conic, the EWA covariance
 * Sigma2D = J R_v Sigma3D R_v^T J^T + 0.3 I (tangent clamp at 1.3x the half field of view
 * included), the projected centre, the SH view direction, Sigma3D = R S S^T R^T with
 * S = diag(exp(log_scale)) and R from the normalised quaternion. Output rows, fp32 [G, 11 + 3d]:
 *   [dL/dmean (3), dL/dlog_scale (3), dL/dquat (w, x, y, z), dL/dopacity_logit,
 *    dL/dsh (3d, index k*3 + channel)]
 * for the variants (each pointer may be NULL; at least one must be given when G > 0):
 *   grad_raw      the derivative itself;
 *   grad_detached the derivative with the paths the score operators stop cut (Sigma2D and the
 *                 view direction): mean through the projected centre only, zero scale and
 *                 rotation blocks, opacity and SH blocks as in grad_raw;
 *   grad_support  grad_raw / q_g, q_g = 1e-6 + sum_v (1e-6 + q_gv), the tokens' normaliser;
 *   grad_pscale   grad_raw with the mean block multiplied by exp(mean of the three log-scales)
 *                 (the derivative per unit of the Gaussian's own size).
 * log_scales, quats, sh must be the arrays given to the last splat_project, unchanged (the
 * means enter through the camera points the projection recorded).
 * Needs splat_render; obs [V,H,W,3]. Leaves the workspace stage as it was (the score replay may
 * still follow). The first call allocates the backward sums, 80 bytes per (view, Gaussian) of the
 * workspace maxima (SPLAT_ERR_OOM when that fails).
 */
int splat_backward(splat_ws* ws, const float* obs, const float* log_scales, const float* quats,
                   const float* sh, float* grad_raw, float* grad_detached, float* grad_support,
                   float* grad_pscale, void* stream);

/*
 * Attribute compositing and its transpose, over the entries the last splat_render composited
 * (same order and decisions; w = T alpha; no background term). Sources: "ReCoSplat" 2.1 (learned
 * feature channels rendered beside RGB), "ATSplat" core method (a per-Gaussian uncertainty score
 * rendered by alpha compositing), "L2D2-GS" method (a 2D gain back-projected to Gaussians through
 * the rasteriser's mask channel), [P1] "Novelty Boundary" / Block 3 (alphaT scatter, PRIMU-style
 * scalar error/coverage).
 *
 * splat_render_features: feats [G, C] per-Gaussian attributes -> out [V, H, W, C],
 *   out_p = sum over composited entries of w f_g. Channels are composited 16 per pass.
 * splat_scatter: map [V, H, W, C] per-pixel values -> out [G, C], out_g = sum over views and
 *   pixels of w m_p (the adjoint of splat_render_features; with m = dL/dF it is the gradient
 *   with respect to the attributes with the Gaussians' other parameters held, as in ATSplat's
 *   stop-gradient uncertainty loss). Sums in fp64, rounded to fp32 at the end.
 * splat_attribution: obs [V, H, W, 3] -> out [G, 3] = [sum w (alphaT coverage),
 *   sum w |C_hat - C_obs| (PRIMU-style error), error / (coverage + 1e-6)].
 * 1 <= C <= 64. Need splat_render (img, T_final, bg unchanged since). The scatter calls grow a
 * workspace buffer of 8 G C bytes when needed (cudaMalloc; SPLAT_ERR_OOM when that fails).
 */
int splat_render_features(splat_ws* ws, const float* feats, int C, float* out, void* stream);
int splat_scatter(splat_ws* ws, const float* map, int C, float* out, void* stream);
int splat_attribution(splat_ws* ws, const float* obs, float* out, void* stream);

/*
 * Deterministic accumulation (a library option; the pages have none). With enable != 0 the score
 * replay (splat_score_replay, splat_score_partials) and the renderer backward add their per-(view,
 * Gaussian) sums as 128-bit fixed-point integers (units of 2^-60; two 64-bit integer atomics with
 * an exact carry), which do not depend on the order of the adds: tokens and gradients are then
 * the same bits on every run, which exposes any race between runs. Off by default (fp32
 * reductions: results agree to rounding order). The first deterministic call allocates 16 bytes per sum of
 * the workspace maxima (SPLAT_ERR_OOM when that fails); each call then clears them and adds one
 * conversion pass. Takes effect from the next call.
 */
int splat_set_deterministic(splat_ws* ws, int enable);

/*
 * Checked build (the library compiled with -DSPLAT_CHECKED, libsplat_checked.so; a library option,
 * the pages have none): every index the kernels take from data -- tile-list entries, scatter and
 * emission positions -- is bounds-checked; a failed check skips the access and sets a device
 * error word. splat_check_status synchronises `stream`, reads and clears the words and returns
 * SPLAT_ERR_BOUNDS when any check failed since the last call (always SPLAT_OK in the release
 * build). splat_checked_build returns 1 in the checked build, 0 otherwise.
 */
int splat_check_status(splat_ws* ws, void* stream);
int splat_checked_build(void);

/* ---------------------------------------------------------------------------------------------
 * Inspection calls (tests and benchmarks; not part of the render/replay path). They copy
 * workspace state into caller-owned DEVICE buffers on `stream`, or report host-side counters.
 * ------------------------------------------------------------------------------------------- */

/* Per (v, g) record, fp32 [V,G,16]: mx, my, conic a, b, c, opacity, colour r, g, b, cut,
 * ex, ey, depth z, x_c, y_c, flags (int bits: bit 0..2 colour-clamp-inactive per channel, bit 8
 * visible). cut = log((1/255)/opacity) - 1e-3 bounds the exponent below which alpha < 1/255;
 * (ex, ey) are the conservatively widened half-extents of the ellipse where it is not.
 * rect [V,G,4] int32 tile rectangle x0, y0, x1, y1 (zeros when culled). Needs splat_project. */
int splat_copy_projection(splat_ws* ws, float* rec, int* rect, void* stream);

/* Tile lists after splat_bin_sort: tile_offsets [V, n_t + 1] int64 (global positions, view-major,
 * n_t = ceil(W/16) ceil(H/16), tiles row-major) and ids [sum of counts] int32 Gaussian indices. */
int splat_copy_tile_lists(splat_ws* ws, long long* tile_offsets, int* ids, void* stream);

/* Per-pixel list bound after splat_render: last [V,H,W] int32 = 1 + the list position of the last
 * composited entry (0 when none), i.e. the number of entries both passes traverse. */
int splat_copy_last(splat_ws* ws, int* last, void* stream);

/* Per-(v, g) sums after splat_score_replay: acc [V,G,8] fp64 = q, Swr(3), Sa, Sd(2), 0 (the sums
 * are kept in fp32 and widened by this copy). */
int splat_copy_accumulators(splat_ws* ws, double* acc, void* stream);

/* Gaussian-pixel pairs traversed by the last render (sum over pixels of `last`); synchronises. */
int splat_pair_count(splat_ws* ws, long long* pairs, void* stream);

/* Number of kernels this workspace has launched since creation (host counter). */
long long splat_launch_count(const splat_ws* ws);

/* Per-kernel device timing. When enabled, every kernel of the path is bracketed by a pair of
 * CUDA events on the launch stream; splat_profile_read synchronises on them and adds, per kernel
 * group id (0 .. SPLAT_NUM_KERNELS-1), the elapsed milliseconds and the number of timed launches
 * since the last reset (reset != 0 clears after reading). Off by default. */
enum {
  SPLAT_K_PROJECT = 0, SPLAT_K_DEPTH_HIST, SPLAT_K_DEPTH_SCATTER,
  SPLAT_K_EMIT, SPLAT_K_TILE_HIST, SPLAT_K_HIST_SCAN, SPLAT_K_TILE_SCATTER, SPLAT_K_TILE_RANGES,
  SPLAT_K_RENDER, SPLAT_K_REPLAY, SPLAT_K_FINALIZE, SPLAT_K_BACKWARD, SPLAT_K_GRAD,
  SPLAT_K_FEATURES, SPLAT_K_SCATTER, SPLAT_K_RENDER_REPLAY, SPLAT_K_OTHER, SPLAT_NUM_KERNELS
};
int splat_profile_enable(splat_ws* ws, int enable);
int splat_profile_read(splat_ws* ws, double* ms, long long* launches, int reset);
/* Static name of a kernel group id ("?" when out of range). */
const char* splat_kernel_name(int id);

/* ---------------------------------------------------------------------------------------------
 * Allocation-free depth ordering. The pages have no counterpart: this is a library addition.
 *
 * For callers that cannot allocate device memory where they need an ordering -- code running
 * under another framework's allocator hooks or memory pool, plugins handed fixed buffers, phases
 * where cudaMalloc/cudaFree would synchronise the device or fail -- this computes, without
 * allocating anything, the stable ascending order of n fp32 depths (equal values keep their
 * index order). For the positive depths the projection produces this is the binning's per-view
 * depth order, and so the order in which it lists a tile's contributors. Writes order[0..n) as
 * int32 indices into depths. Both are DEVICE pointers owned by the caller.
 *
 * Scratch: one fixed file-scope __device__ array of 4 * SPLAT_NOALLOC_MAX_N 32-bit words
 * (4 MiB), which every GPU that loads this library holds until the process exits. No cudaMalloc,
 * cudaFree or allocating library routine is called.
 *   - n > SPLAT_NOALLOC_MAX_N returns SPLAT_ERR_CAPACITY before any work; n < 0, or NULL
 *     pointers with n > 0, return SPLAT_ERR_INVALID_ARG; n == 0 returns SPLAT_OK.
 *   - Every call looks up the array's device address in the current context
 *     (cudaGetSymbolAddress, host-side); the first lookup on a device also loads the module, so
 *     make the first call on each device before any stream capture there. After
 *     cudaDeviceReset the next call finds the array again (its contents are then undefined,
 *     which no call depends on).
 *   - All calls share the array and it keeps the last call's contents (nothing in it needs to
 *     start at zero: every word read is written first by the same call). Calls whose kernels
 *     overlap on one GPU -- different streams, or host threads without ordering -- race and
 *     corrupt each other's results; serialise them on one stream.
 *   - Order of values (this entry point's own beyond the positive depths of the projection):
 *     negatives before positives, -0.0 before +0.0, NaNs by bit pattern.
 *   - Enqueued on `stream` (a cudaStream_t, NULL = legacy default); returns without waiting.
 *     Kernel-launch failures return SPLAT_ERR_CUDA.
 */
#define SPLAT_NOALLOC_MAX_N 262144
int splat_sort_depths_noalloc(const float* depths, int n, int* order, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* SPLAT_H */
