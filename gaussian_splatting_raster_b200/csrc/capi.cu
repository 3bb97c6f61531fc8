// C ABI of libsplat (declared in include/splat.h): argument validation, workspace management and
// the call order project -> bin_sort -> render -> score_replay.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>

#include "common.cuh"

using splat::Workspace;

namespace {

constexpr int kMaxViews = 1024;

int fail(Workspace& w, int code, const char* fmt, ...) __attribute__((format(printf, 3, 4)));
int fail(Workspace& w, int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  w.err = buf;
  return code;
}

int cuda_fail(Workspace& w, const char* what, cudaError_t e) {
  return fail(w, SPLAT_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// device (or managed) memory of the workspace's device, 4-byte aligned
int check_dev_ptr(Workspace& w, const void* p, const char* name, bool allow_null = false) {
  if (!p) {
    if (allow_null) return SPLAT_OK;
    return fail(w, SPLAT_ERR_INVALID_ARG, "%s is NULL", name);
  }
  if (((uintptr_t)p) & 3u) return fail(w, SPLAT_ERR_INVALID_ARG, "%s is not 4-byte aligned", name);
  cudaPointerAttributes at;
  cudaError_t e = cudaPointerGetAttributes(&at, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(w, SPLAT_ERR_INVALID_ARG, "%s is not a CUDA pointer", name);
  }
  if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged)
    return fail(w, SPLAT_ERR_INVALID_ARG, "%s must be device memory", name);
  if (at.type == cudaMemoryTypeDevice && at.device != w.device)
    return fail(w, SPLAT_ERR_INVALID_ARG, "%s lives on device %d, workspace on device %d", name,
                at.device, w.device);
  return SPLAT_OK;
}

template <typename T>
int alloc(Workspace& w, T** p, size_t n, const char* what) {
  if (n == 0) n = 1;
  cudaError_t e = cudaMalloc((void**)p, n * sizeof(T));
  if (e != cudaSuccess) {
    cudaGetLastError();
    *p = nullptr;
    return fail(w, SPLAT_ERR_OOM, "device allocation of %zu bytes failed (%s)", n * sizeof(T), what);
  }
  return SPLAT_OK;
}

// pinned host memory the kernels read and write directly (mapped): the few words a step exchanges
// with the host move without a copy engine
template <typename T>
int alloc_mapped(Workspace& w, T** h, T** d, size_t n, const char* what) {
  *h = nullptr;
  *d = nullptr;
  if (cudaHostAlloc((void**)h, n * sizeof(T), cudaHostAllocMapped) != cudaSuccess) {
    cudaGetLastError();
    *h = nullptr;
    return fail(w, SPLAT_ERR_OOM, "pinned host allocation of %zu bytes failed (%s)", n * sizeof(T), what);
  }
  if (cudaHostGetDevicePointer((void**)d, *h, 0) != cudaSuccess) {
    cudaGetLastError();
    return fail(w, SPLAT_ERR_CUDA, "no device address for mapped host memory (%s)", what);
  }
  return SPLAT_OK;
}

void free_all(Workspace& w) {
  void* dev[] = {w.rec, w.rect, w.counts, w.acc, w.views, w.last, w.part,
                 w.inst_tile, w.inst_g, w.sval, w.hist, w.tile_off, w.d_vstart, w.d_bstart,
                 w.d_scratch, w.dkey, w.kbits, w.dk1, w.dk2, w.dv0, w.dv1, w.rect_s, w.ntot, w.umask, w.lmask, w.accb, w.sacc,
                 w.acc_fix, w.accb_fix, w.tile_order};
  for (void* p : dev)
    if (p) cudaFree(p);
  if (w.h_vstart) cudaFreeHost(w.h_vstart);
  if (w.h_bstart) cudaFreeHost(w.h_bstart);
  if (w.h_scratch) cudaFreeHost(w.h_scratch);
  if (w.h_kbits) cudaFreeHost(w.h_kbits);
  if (w.h_ntot) cudaFreeHost(w.h_ntot);
  for (cudaEvent_t e : w.ev_pool) cudaEventDestroy(e);
  w.ev_pool.clear();
}

const char* const kKernelNames[SPLAT_NUM_KERNELS] = {
    "project", "depth_hist", "depth_scatter", "emit", "tile_hist", "hist_scan",
    "tile_scatter", "tile_ranges", "render", "replay", "finalize", "backward", "grad", "features", "scatter",
    "render_replay", "other"};

// fold every recorded (start, end) pair into the per-kernel sums
int fold_events(Workspace& w) {
  for (size_t k = 0; k + 1 < w.ev_open.size(); k += 2) {
    const int id = w.ev_open[k], a = w.ev_open[k + 1];
    cudaError_t e = cudaEventSynchronize(w.ev_pool[a + 1]);
    float ms = 0.0f;
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, w.ev_pool[a], w.ev_pool[a + 1]);
    if (e != cudaSuccess) return cuda_fail(w, "reading timing events", e);
    w.prof_ms[id] += ms;
    w.prof_n[id] += 1;
  }
  w.ev_open.clear();
  w.ev_used = 0;
  return SPLAT_OK;
}


}  // namespace

extern "C" {

int splat_ws_create(splat_ws** out, int max_G, int max_V, int max_H, int max_W,
                    int max_sh_degree) {
  if (!out) return SPLAT_ERR_INVALID_ARG;
  *out = nullptr;
  if (max_G < 0 || max_V < 1 || max_V > kMaxViews || max_H < 1 || max_W < 1 ||
      max_sh_degree < 0 || max_sh_degree > 3)
    return SPLAT_ERR_INVALID_ARG;
  splat_ws* ws = new (std::nothrow) splat_ws();
  if (!ws) return SPLAT_ERR_OOM;
  Workspace& w = ws->w;
  cudaGetDevice(&w.device);
  w.max_G = max_G;
  w.max_V = max_V;
  w.max_H = max_H;
  w.max_W = max_W;
  w.max_deg = max_sh_degree;
  w.max_nt = ((max_W + 15) / 16) * ((max_H + 15) / 16);
  const size_t VG = (size_t)max_V * max_G;
  int rc = 0;
  if (!rc) rc = alloc(w, &w.rec, splat::rec_f4_count(VG), "records");
  if (!rc) rc = alloc(w, &w.rect, VG, "rectangles");
  if (!rc) rc = alloc(w, &w.counts, VG, "tile counts in depth order, then their scan");
  if (!rc) rc = alloc(w, &w.acc, VG * splat::kAccN, "accumulators");
  if (!rc) rc = alloc(w, &w.views, (size_t)max_V * 20, "views");
  if (!rc) rc = alloc(w, &w.last, (size_t)max_V * max_H * max_W, "list bounds");
  if (!rc) rc = alloc(w, &w.tile_off, (size_t)max_V * (w.max_nt + 1), "tile offsets");
  if (!rc) rc = alloc(w, &w.tile_order, (size_t)max_V * w.max_nt, "tile launch order");
  if (!rc) rc = alloc(w, &w.d_vstart, (size_t)max_V + 1, "view starts");
  if (!rc) rc = alloc(w, &w.d_bstart, (size_t)max_V + 1, "block starts");
  if (!rc) rc = alloc(w, &w.d_scratch, 8, "scratch");
  if (!rc) rc = alloc(w, &w.dkey, VG, "depth keys");
  if (!rc) rc = alloc(w, &w.kbits, (size_t)2 * splat::kKeyStripes * max_V, "key statistics");
  if (!rc) rc = alloc(w, &w.ntot, (size_t)splat::kKeyStripes * max_V, "instance counts");
  if (!rc) rc = alloc_mapped(w, &w.h_ntot, &w.hd_ntot, (size_t)splat::kKeyStripes * max_V,
                             "instance counts (host)");
  if (!rc) rc = alloc(w, &w.dk1, VG, "depth keys 2");
  if (!rc) rc = alloc(w, &w.dk2, VG, "depth keys 3");
  if (!rc) rc = alloc(w, &w.dv0, VG, "depth order");
  if (!rc) rc = alloc(w, &w.dv1, VG, "depth order 2");
  if (!rc) rc = alloc(w, &w.rect_s, VG, "rectangles in depth order");
  if (!rc) rc = alloc_mapped(w, &w.h_kbits, &w.hd_kbits, (size_t)2 * splat::kKeyStripes * max_V,
                             "key statistics (host)");
  if (!rc) rc = alloc_mapped(w, &w.h_vstart, &w.hd_vstart, (size_t)max_V + 1, "view starts (host)");
  if (!rc) rc = alloc_mapped(w, &w.h_bstart, &w.hd_bstart, (size_t)max_V + 1, "block starts (host)");
  if (!rc && cudaMallocHost(&w.h_scratch, 8 * sizeof(long long)) != cudaSuccess)
    rc = SPLAT_ERR_OOM;
  if (!rc) rc = splat::binning_configure(w);
  if (!rc) w.ev_open.reserve(1024);
  if (rc) {
    cudaGetLastError();
    free_all(w);
    delete ws;
    return rc;
  }
  *out = ws;
  return SPLAT_OK;
}

void splat_ws_destroy(splat_ws* ws) {
  if (!ws) return;
  cudaDeviceSynchronize();
  free_all(ws->w);
  delete ws;
}

const char* splat_last_error(const splat_ws* ws) { return ws ? ws->w.err.c_str() : "no workspace"; }

int splat_project(splat_ws* ws, const float* means, const float* log_scales, const float* quats,
                  const float* opac_logits, const float* sh, int G, int sh_degree,
                  const float* viewmats, const float* intrin, int V, int H, int W,
                  void* stream) {
  if (!ws) return SPLAT_ERR_INVALID_ARG;
  Workspace& w = ws->w;
  w.err.clear();
  if (G < 0 || V < 1 || H < 1 || W < 1 || sh_degree < 0 || sh_degree > 3)
    return fail(w, SPLAT_ERR_INVALID_ARG, "bad sizes G=%d V=%d H=%d W=%d deg=%d", G, V, H, W,
                sh_degree);
  if (G > w.max_G || V > w.max_V || H > w.max_H || W > w.max_W || sh_degree > w.max_deg)
    return fail(w, SPLAT_ERR_CAPACITY, "sizes exceed the workspace maxima");
  int rc;
  const bool none = G == 0;
  if ((rc = check_dev_ptr(w, log_scales, "log_scales", none))) return rc;
  if ((rc = check_dev_ptr(w, quats, "quats", none))) return rc;
  if ((rc = check_dev_ptr(w, opac_logits, "opac_logits", none))) return rc;
  if ((rc = check_dev_ptr(w, sh, "sh", none))) return rc;
  if ((rc = check_dev_ptr(w, viewmats, "viewmats"))) return rc;
  if ((rc = check_dev_ptr(w, intrin, "intrin"))) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  w.G = G;
  w.V = V;
  w.H = H;
  w.W = W;
  w.deg = sh_degree;
  w.TX = (W + 15) / 16;
  w.TY = (H + 15) / 16;
  w.nt = w.TX * w.TY;
  w.stage = 0;
  cudaError_t e = cudaMemcpy2DAsync(w.views, 20 * sizeof(float), viewmats, 16 * sizeof(float),
                                    16 * sizeof(float), V, cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess)
    e = cudaMemcpy2DAsync(w.views + 16, 20 * sizeof(float), intrin, 4 * sizeof(float),
                          4 * sizeof(float), V, cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) return cuda_fail(w, "copying the cameras", e);
  if ((rc = splat::launch_project(w, means, log_scales, quats, opac_logits, sh, st))) return rc;
  w.stage = 1;
  return SPLAT_OK;
}

int splat_bin_sort(splat_ws* ws, long long* n_instances_out, void* stream) {
  if (!ws) return SPLAT_ERR_INVALID_ARG;
  Workspace& w = ws->w;
  w.err.clear();
  if (w.stage < 1) return fail(w, SPLAT_ERR_STATE, "splat_bin_sort before splat_project");
  cudaStream_t st = (cudaStream_t)stream;
  int rc;
  // the one synchronisation of the path: per-view instance counts and depth-key statistics,
  // accumulated in striped copies by the projection, folded here
  const int ns = splat::kKeyStripes;
  // (kernels store them into mapped host memory: no copy engine, so the wait is not queued
  // behind a caller's large transfers on other streams)
  if ((rc = splat::copy_words(w, w.ntot, w.hd_ntot, (size_t)ns * w.V * sizeof(unsigned long long),
                              st, "instance counts readback")) ||
      (rc = splat::copy_words(w, w.kbits, w.hd_kbits, (size_t)2 * ns * w.V * sizeof(uint32_t), st,
                              "key statistics readback")))
    return rc;
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(w, "reading the instance counts", e);
  w.h_vstart[0] = 0;
  for (int v = 0; v < w.V; ++v) {
    unsigned long long nv = 0;
    for (int k = 0; k < ns; ++k) nv += w.h_ntot[v * ns + k];
    w.h_vstart[v + 1] = w.h_vstart[v] + (long long)nv;
  }
  w.n_total = w.h_vstart[w.V];
  if (w.n_total >= (1LL << 31) - 1)
    return fail(w, SPLAT_ERR_CAPACITY, "%lld instances exceed the 2^31 limit", w.n_total);
  if ((rc = splat::launch_binning(w, st))) return rc;
  if (n_instances_out)
    for (int v = 0; v < w.V; ++v) n_instances_out[v] = w.h_vstart[v + 1] - w.h_vstart[v];
  w.stage = 2;
  return SPLAT_OK;
}

int splat_render(splat_ws* ws, const float* bg, float* img, float* T_final, int* n_contrib,
                 void* stream) {
  if (!ws) return SPLAT_ERR_INVALID_ARG;
  Workspace& w = ws->w;
  w.err.clear();
  if (w.stage < 2) return fail(w, SPLAT_ERR_STATE, "splat_render before splat_bin_sort");
  int rc;
  if ((rc = check_dev_ptr(w, bg, "bg"))) return rc;
  if ((rc = check_dev_ptr(w, img, "img"))) return rc;
  if ((rc = check_dev_ptr(w, T_final, "T_final"))) return rc;
  if ((rc = check_dev_ptr(w, n_contrib, "n_contrib"))) return rc;
  if ((rc = splat::launch_render(w, bg, img, T_final, n_contrib, (cudaStream_t)stream))) return rc;
  w.img = img;
  w.Tfin = T_final;
  w.ncon = n_contrib;
  w.bg = bg;
  w.stage = 3;
  return SPLAT_OK;
}

int splat_score_replay(splat_ws* ws, const float* obs, float lambda, float* tokens,
                       void* stream) {
  if (!ws) return SPLAT_ERR_INVALID_ARG;
  Workspace& w = ws->w;
  w.err.clear();
  if (w.stage < 3) return fail(w, SPLAT_ERR_STATE, "splat_score_replay before splat_render");
  if (!(lambda >= 0.0f) || !std::isfinite(lambda))
    return fail(w, SPLAT_ERR_INVALID_ARG, "lambda must be finite and >= 0");
  int rc;
  if ((rc = check_dev_ptr(w, obs, "obs"))) return rc;
  if ((rc = check_dev_ptr(w, tokens, "tokens", w.G == 0))) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  if ((rc = splat::launch_replay(w, obs, st))) return rc;
  if ((rc = splat::launch_finalize(w, lambda, tokens, st))) return rc;
  w.stage = 4;
  return SPLAT_OK;
}

int splat_render_score(splat_ws* ws, const float* bg, const float* obs, float lambda, float* img,
                       float* T_final, int* n_contrib, float* tokens, void* stream) {
  if (!ws) return SPLAT_ERR_INVALID_ARG;
  Workspace& w = ws->w;
  w.err.clear();
  if (w.stage < 2) return fail(w, SPLAT_ERR_STATE, "splat_render_score before splat_bin_sort");
  if (!(lambda >= 0.0f) || !std::isfinite(lambda))
    return fail(w, SPLAT_ERR_INVALID_ARG, "lambda must be finite and >= 0");
  int rc;
  if ((rc = check_dev_ptr(w, bg, "bg"))) return rc;
  if ((rc = check_dev_ptr(w, obs, "obs"))) return rc;
  if ((rc = check_dev_ptr(w, img, "img"))) return rc;
  if ((rc = check_dev_ptr(w, T_final, "T_final"))) return rc;
  if ((rc = check_dev_ptr(w, n_contrib, "n_contrib"))) return rc;
  if ((rc = check_dev_ptr(w, tokens, "tokens", w.G == 0))) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  w.img = img;
  w.Tfin = T_final;
  w.ncon = n_contrib;
  w.bg = bg;
  if (w.det) {
    if ((rc = splat::launch_render(w, bg, img, T_final, n_contrib, st))) return rc;
    if ((rc = splat::launch_replay(w, obs, st))) return rc;
  } else if ((rc = splat::launch_render_replay(w, bg, obs, img, T_final, n_contrib, st))) {
    return rc;
  }
  if ((rc = splat::launch_finalize(w, lambda, tokens, st))) return rc;
  w.stage = 4;
  return SPLAT_OK;
}

int splat_backward(splat_ws* ws, const float* obs, const float* log_scales, const float* quats,
                   const float* sh, float* grad_raw, float* grad_detached, float* grad_support,
                   float* grad_pscale, void* stream) {
  if (!ws) return SPLAT_ERR_INVALID_ARG;
  Workspace& w = ws->w;
  w.err.clear();
  if (w.stage < 3) return fail(w, SPLAT_ERR_STATE, "splat_backward before splat_render");
  if (w.G > 0 && !grad_raw && !grad_detached && !grad_support && !grad_pscale)
    return fail(w, SPLAT_ERR_INVALID_ARG, "splat_backward: no output requested");
  int rc;
  const bool none = w.G == 0;
  if ((rc = check_dev_ptr(w, obs, "obs"))) return rc;
  if ((rc = check_dev_ptr(w, log_scales, "log_scales", none))) return rc;
  if ((rc = check_dev_ptr(w, quats, "quats", none))) return rc;
  if ((rc = check_dev_ptr(w, sh, "sh", none))) return rc;
  float* outs[4] = {grad_raw, grad_detached, grad_support, grad_pscale};
  const char* names[4] = {"grad_raw", "grad_detached", "grad_support", "grad_pscale"};
  for (int k = 0; k < 4; ++k)
    if (outs[k] && (rc = check_dev_ptr(w, outs[k], names[k], none))) return rc;
  if (!w.accb && (rc = alloc(w, &w.accb, (size_t)w.max_V * w.max_G * splat::kAccBN,
                             "backward sums")))
    return rc;
  cudaStream_t st = (cudaStream_t)stream;
  if ((rc = splat::launch_backward(w, obs, st))) return rc;
  return splat::launch_grad(w, log_scales, quats, sh, grad_raw, grad_detached, grad_support,
                            grad_pscale, st);
}

constexpr int kMaxAttributeChannels = 64;

int splat_render_features(splat_ws* ws, const float* feats, int C, float* out, void* stream) {
  if (!ws) return SPLAT_ERR_INVALID_ARG;
  Workspace& w = ws->w;
  w.err.clear();
  if (w.stage < 3) return fail(w, SPLAT_ERR_STATE, "splat_render_features before splat_render");
  if (C < 1 || C > kMaxAttributeChannels)
    return fail(w, SPLAT_ERR_INVALID_ARG, "splat_render_features: C must be in [1, %d]",
                kMaxAttributeChannels);
  int rc;
  if ((rc = check_dev_ptr(w, feats, "feats", w.G == 0))) return rc;
  if ((rc = check_dev_ptr(w, out, "out"))) return rc;
  return splat::launch_features(w, feats, C, out, (cudaStream_t)stream);
}

int splat_scatter(splat_ws* ws, const float* map, int C, float* out, void* stream) {
  if (!ws) return SPLAT_ERR_INVALID_ARG;
  Workspace& w = ws->w;
  w.err.clear();
  if (w.stage < 3) return fail(w, SPLAT_ERR_STATE, "splat_scatter before splat_render");
  if (C < 1 || C > kMaxAttributeChannels)
    return fail(w, SPLAT_ERR_INVALID_ARG, "splat_scatter: C must be in [1, %d]",
                kMaxAttributeChannels);
  int rc;
  if ((rc = check_dev_ptr(w, map, "map"))) return rc;
  if ((rc = check_dev_ptr(w, out, "out", w.G == 0))) return rc;
  return splat::launch_scatter(w, map, nullptr, C, out, (cudaStream_t)stream);
}

int splat_attribution(splat_ws* ws, const float* obs, float* out, void* stream) {
  if (!ws) return SPLAT_ERR_INVALID_ARG;
  Workspace& w = ws->w;
  w.err.clear();
  if (w.stage < 3) return fail(w, SPLAT_ERR_STATE, "splat_attribution before splat_render");
  int rc;
  if ((rc = check_dev_ptr(w, obs, "obs"))) return rc;
  if ((rc = check_dev_ptr(w, out, "out", w.G == 0))) return rc;
  return splat::launch_scatter(w, nullptr, obs, 2, out, (cudaStream_t)stream);
}

int splat_score_partials(splat_ws* ws, const float* obs, float* partials, void* stream) {
  if (!ws) return SPLAT_ERR_INVALID_ARG;
  Workspace& w = ws->w;
  w.err.clear();
  if (w.stage < 3) return fail(w, SPLAT_ERR_STATE, "splat_score_partials before splat_render");
  int rc;
  if ((rc = check_dev_ptr(w, obs, "obs"))) return rc;
  if ((rc = check_dev_ptr(w, partials, "partials", w.G == 0))) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  if ((rc = splat::launch_replay(w, obs, st))) return rc;
  if ((rc = splat::launch_partials(w, partials, st))) return rc;
  w.stage = 4;
  return SPLAT_OK;
}

int splat_finalize_partials(const float* partials, int G, int sh_degree, float lambda,
                            float* tokens, void* stream) {
  if (G < 0 || sh_degree < 0 || sh_degree > 3 || !(lambda >= 0.0f) || !std::isfinite(lambda))
    return SPLAT_ERR_INVALID_ARG;
  if (G == 0) return SPLAT_OK;
  if (!partials || !tokens || (((uintptr_t)partials | (uintptr_t)tokens) & 3u))
    return SPLAT_ERR_INVALID_ARG;
  cudaError_t e = splat::launch_finalize_partials(partials, G, sh_degree, (double)lambda, tokens,
                                                  (cudaStream_t)stream);
  return e == cudaSuccess ? SPLAT_OK : SPLAT_ERR_CUDA;
}

// ----------------------------------------------------------------------------------------------
int splat_copy_projection(splat_ws* ws, float* rec, int* rect, void* stream) {
  if (!ws) return SPLAT_ERR_INVALID_ARG;
  Workspace& w = ws->w;
  if (w.stage < 1) return fail(w, SPLAT_ERR_STATE, "no projection yet");
  const size_t VG = (size_t)w.V * w.G;
  if (VG == 0) return SPLAT_OK;
  int rc;
  if ((rc = check_dev_ptr(w, rec, "rec"))) return rc;
  if ((rc = check_dev_ptr(w, rect, "rect"))) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  if ((rc = splat::launch_copy_records(w, rec, st))) return rc;
  return splat::launch_copy_rects(w, rect, st);
}

int splat_copy_tile_lists(splat_ws* ws, long long* tile_offsets, int* ids, void* stream) {
  if (!ws) return SPLAT_ERR_INVALID_ARG;
  Workspace& w = ws->w;
  if (w.stage < 2) return fail(w, SPLAT_ERR_STATE, "no tile lists yet");
  int rc;
  if ((rc = check_dev_ptr(w, tile_offsets, "tile_offsets"))) return rc;
  if ((rc = check_dev_ptr(w, ids, "ids", w.n_total == 0))) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(tile_offsets, w.tile_off, (size_t)w.V * (w.nt + 1) * 8,
                                  cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess && w.n_total > 0)
    e = cudaMemcpyAsync(ids, w.sval, (size_t)w.n_total * 4, cudaMemcpyDeviceToDevice, st);
  return e == cudaSuccess ? SPLAT_OK : cuda_fail(w, "copy tile lists", e);
}

int splat_copy_last(splat_ws* ws, int* last, void* stream) {
  if (!ws) return SPLAT_ERR_INVALID_ARG;
  Workspace& w = ws->w;
  if (w.stage < 3) return fail(w, SPLAT_ERR_STATE, "no render yet");
  int rc;
  if ((rc = check_dev_ptr(w, last, "last"))) return rc;
  cudaError_t e = cudaMemcpyAsync(last, w.last, (size_t)w.V * w.H * w.W * 4,
                                  cudaMemcpyDeviceToDevice, (cudaStream_t)stream);
  return e == cudaSuccess ? SPLAT_OK : cuda_fail(w, "copy last", e);
}

int splat_copy_accumulators(splat_ws* ws, double* acc, void* stream) {
  if (!ws) return SPLAT_ERR_INVALID_ARG;
  Workspace& w = ws->w;
  if (w.stage < 4) return fail(w, SPLAT_ERR_STATE, "no replay yet");
  const size_t VG = (size_t)w.V * w.G;
  if (VG == 0) return SPLAT_OK;
  int rc;
  if ((rc = check_dev_ptr(w, acc, "acc"))) return rc;
  return splat::launch_acc_to_double(w, acc, (cudaStream_t)stream);
}

int splat_pair_count(splat_ws* ws, long long* pairs, void* stream) {
  if (!ws || !pairs) return SPLAT_ERR_INVALID_ARG;
  Workspace& w = ws->w;
  if (w.stage < 3) return fail(w, SPLAT_ERR_STATE, "no render yet");
  cudaStream_t st = (cudaStream_t)stream;
  int rc;
  if ((rc = splat::launch_pair_count(w, st))) return rc;
  cudaError_t e = cudaMemcpyAsync(w.h_scratch, w.d_scratch, 8, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(w, "pair count", e);
  *pairs = w.h_scratch[0];
  return SPLAT_OK;
}

long long splat_launch_count(const splat_ws* ws) { return ws ? ws->w.launches : 0; }

int splat_check_status(splat_ws* ws, void* stream) {
  if (!ws) return SPLAT_ERR_INVALID_ARG;
  Workspace& w = ws->w;
  w.err.clear();
  cudaStream_t st = (cudaStream_t)stream;
  const unsigned int bad = splat::bounds_word_raster(st) | splat::bounds_word_binning(st) |
                           splat::bounds_word_attributes(st);
  if (bad & 0x80000000u) return fail(w, SPLAT_ERR_CUDA, "reading the bounds-check words failed");
  if (bad) return fail(w, SPLAT_ERR_BOUNDS, "a device-side bounds check failed (access skipped)");
  return SPLAT_OK;
}

int splat_checked_build(void) { return splat::kChecked ? 1 : 0; }

int splat_set_deterministic(splat_ws* ws, int enable) {
  if (!ws) return SPLAT_ERR_INVALID_ARG;
  ws->w.det = enable != 0;
  return SPLAT_OK;
}

int splat_profile_enable(splat_ws* ws, int enable) {
  if (!ws) return SPLAT_ERR_INVALID_ARG;
  Workspace& w = ws->w;
  if (!enable && w.prof) {
    const int rc = fold_events(w);
    if (rc) return rc;
  }
  w.prof = enable != 0;
  return SPLAT_OK;
}

int splat_profile_read(splat_ws* ws, double* ms, long long* launches, int reset) {
  if (!ws) return SPLAT_ERR_INVALID_ARG;
  Workspace& w = ws->w;
  const int rc = fold_events(w);
  if (rc) return rc;
  for (int i = 0; i < SPLAT_NUM_KERNELS; ++i) {
    if (ms) ms[i] = w.prof_ms[i];
    if (launches) launches[i] = w.prof_n[i];
    if (reset) {
      w.prof_ms[i] = 0.0;
      w.prof_n[i] = 0;
    }
  }
  return SPLAT_OK;
}

const char* splat_kernel_name(int id) {
  return (id >= 0 && id < SPLAT_NUM_KERNELS) ? kKernelNames[id] : "?";
}

}  // extern "C"
