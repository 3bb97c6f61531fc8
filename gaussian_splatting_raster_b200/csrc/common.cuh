// Internal definitions shared by the libsplat CUDA translation units.
//
// Every file of the library is compiled with -fmad=false (no implicit multiply-add
// contraction), IEEE division and square root, and denormals preserved. The preprocess, render
// and replay decisions that turn floating point into integers (tile rectangle, depth order, the
// 1/255 and 1e-4 thresholds, the 0.99 clamp) therefore depend only on the stated sequence of
// correctly rounded fp32 operations; fused multiply-adds appear only where written as fmaf() or
// __ffma2_rn(). (-fmad=false does not cover packed pairs: the compiler fuses a packed product
// into a packed add that is its only consumer, so packed products only feed scalar adds; see the
// list-walking helpers.)
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <vector>

#include "splat.h"

namespace splat {

constexpr int kTile = 16;        // 16x16 pixel tiles
constexpr int kTilePix = 256;
constexpr int kAccN = 8;         // doubles per (v, g) accumulator
constexpr int kAccBN = 10;       // doubles per (v, g) renderer-backward sums
constexpr int kFlagVisible = 256;
constexpr int kKeyStripes = 64;  // striped copies of the per-view depth-key statistics

// Record of one (view, Gaussian), 4 x float4 = 64 bytes, in two halves:
//   low  r0 = (mx, my, colour r, colour g)      r1 = (colour b, cut, ex, ey)
//   high r2 = (conic a, conic b, conic c, opacity)   r3 = (depth z, x_c, y_c, flags as int bits)
// stored in blocks of 32 entries (view-major (v, g) index i): the block's 32 low halves, then its
// 32 high halves (2 KB per block). The list-walking kernels gather r0, r1 and r2; the finaliser
// and the gradient chain need only the high halves, which lie contiguous for consecutive
// Gaussians (DRAM is read in 64-byte pieces: with whole records side by side the finaliser read
// all 64 bytes of each).
__host__ __device__ __forceinline__ size_t rec_lo(size_t i) { return (i >> 5) * 128 + (i & 31) * 2; }
__host__ __device__ __forceinline__ size_t rec_hi(size_t i) { return rec_lo(i) + 64; }
__host__ __device__ __forceinline__ size_t rec_f4_count(size_t n) { return (n + 31) / 32 * 128; }
// (splat_copy_projection hands it out in the documented order mx, my, a, b, c, o, r, g, b, cut,
// ex, ey, z, x_c, y_c, flags.)
// cut = log((1/255) / o) - 1e-3: an exponent below it gives alpha < 1/255 for certain;
// (ex, ey) = half-extents of the ellipse {exponent >= cut} widened by 1 % + 0.05 px (+inf for a
// nearly singular conic, -1 when no pixel can pass).
// flags: bits 0..2 colour clamp inactive per channel (M_color), bit 8 visible.

// ---------------------------------------------------------------------------------------------
// exp for the decision path, written from Cody & Waite (1980), "Software Manual for the
// Elementary Functions": x = k ln2 + r with k = rint(x log2 e), ln2 split into a 16-bit high
// part (k * hi exact for |k| <= 128) and a low correction, e^r by its Taylor series to degree 7
// (Horner, fused multiply-adds) on |r| <= ln2 / 2, scaled by 2^k through the exponent field.
// Zero below -87, +inf above 88.
// ---------------------------------------------------------------------------------------------
namespace cw {
constexpr double kLn2 = 0.693147180559945309417232121458;
constexpr float kLog2e = (float)(1.0 / kLn2);
constexpr float kLn2Hi = 45426.0f / 65536.0f;  // floor(ln2 * 2^16) / 2^16
constexpr float kLn2Lo = (float)(kLn2 - 45426.0 / 65536.0);
constexpr float kC2 = (float)(1.0 / 2.0);
constexpr float kC3 = (float)(1.0 / 6.0);
constexpr float kC4 = (float)(1.0 / 24.0);
constexpr float kC5 = (float)(1.0 / 120.0);
constexpr float kC6 = (float)(1.0 / 720.0);
constexpr float kC7 = (float)(1.0 / 5040.0);
}  // namespace cw

// exp of x in [-87, 88] without range checks (exp_cw below adds them), bit-identical to exp_cw
// there. k = round-half-even(x log2e) is taken by adding and subtracting 1.5 * 2^23 (exact for
// |x log2e| < 2^22; the addition itself rounds half to even), whose bits also hold k as an
// integer: no float-to-integer conversions.
__device__ __forceinline__ float exp_cw_core(float x) {
  const float kMagic = 12582912.0f;  // 1.5 * 2^23, bits 0x4B400000
  const float t = x * cw::kLog2e + kMagic;
  const float k = t - kMagic;
  const int ki = __float_as_int(t) - 0x4B400000;
  // k * ln2_hi is exact (16-bit ln2_hi, |k| < 2^8), so one fused step rounds as x - k ln2_hi does
  const float r = fmaf(-k, cw::kLn2Hi, x) - k * cw::kLn2Lo;
  float p = cw::kC7;
  p = fmaf(p, r, cw::kC6);
  p = fmaf(p, r, cw::kC5);
  p = fmaf(p, r, cw::kC4);
  p = fmaf(p, r, cw::kC3);
  p = fmaf(p, r, cw::kC2);
  p = fmaf(p, r, 1.0f);
  p = fmaf(p, r, 1.0f);
  return p * __int_as_float((ki + 127) << 23);
}

__device__ __forceinline__ float exp_cw(float x) {
  if (x != x) return x;
  if (!(x > -87.0f)) return 0.0f;
  if (x > 88.0f) return __int_as_float(0x7f800000);
  const float k = rintf(x * cw::kLog2e);
  const float r = (x - k * cw::kLn2Hi) - k * cw::kLn2Lo;
  float p = cw::kC7;
  p = fmaf(p, r, cw::kC6);
  p = fmaf(p, r, cw::kC5);
  p = fmaf(p, r, cw::kC4);
  p = fmaf(p, r, cw::kC3);
  p = fmaf(p, r, cw::kC2);
  p = fmaf(p, r, 1.0f);
  p = fmaf(p, r, 1.0f);
  return p * __int_as_float(((int)k + 127) << 23);
}

// ---------------------------------------------------------------------------------------------
// Real spherical harmonics up to degree 3 of a unit direction, Condon-Shortley phase (the 3DGS
// colour model), as Cartesian polynomials. Normalisations: Y00 = 1/(2 sqrt(pi));
// l=1: sqrt(3/(4 pi)); l=2: sqrt(15/pi)/2, sqrt(5/pi)/4, sqrt(15/pi)/4;
// l=3: sqrt(35/(2 pi))/4, sqrt(105/pi)/2, sqrt(21/(2 pi))/4, sqrt(7/pi)/4, sqrt(105/pi)/4.
// ---------------------------------------------------------------------------------------------
template <int DEG>
__device__ __forceinline__ void sh_poly(float x, float y, float z, float* B) {
  B[0] = 0.28209479177387814f;
  if (DEG >= 1) {
    const float c1 = 0.48860251190291992f;
    B[1] = -c1 * y;
    B[2] = c1 * z;
    B[3] = -c1 * x;
  }
  if (DEG >= 2) {
    const float xx = x * x, yy = y * y, zz = z * z;
    B[4] = 1.0925484305920792f * (x * y);
    B[5] = -1.0925484305920792f * (y * z);
    B[6] = 0.31539156525252005f * (2.0f * zz - xx - yy);
    B[7] = -1.0925484305920792f * (x * z);
    B[8] = 0.54627421529603959f * (xx - yy);
    if (DEG >= 3) {
      B[9] = -0.59004358992664352f * y * (3.0f * xx - yy);
      B[10] = 2.8906114426405538f * (x * y) * z;
      B[11] = -0.45704579946446572f * y * (4.0f * zz - xx - yy);
      B[12] = 0.37317633259011540f * z * (2.0f * zz - 3.0f * xx - 3.0f * yy);
      B[13] = -0.45704579946446572f * x * (4.0f * zz - xx - yy);
      B[14] = 1.4453057213202769f * z * (xx - yy);
      B[15] = -0.59004358992664352f * x * (xx - 3.0f * yy);
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Checked build (-DSPLAT_CHECKED): the kernels bounds-check every index that comes from data
// (list entries, scatter positions); a failed check sets a bit in the error word of its source
// file and the access is skipped; splat_check_status reads and clears the words. In the release
// build the checks compile to nothing.
// ---------------------------------------------------------------------------------------------
#ifdef SPLAT_CHECKED
constexpr bool kChecked = true;
#else
constexpr bool kChecked = false;
#endif

__device__ __forceinline__ bool in_bounds(unsigned long long i, unsigned long long n,
                                          unsigned int* word) {
  if (!kChecked || i < n) return true;
  atomicOr(word, 1u);
  return false;
}

// one error word per source file, with a host accessor that reads and clears it (stream-ordered)
#define SPLAT_BOUNDS_WORD(accessor)                                                         \
  static __device__ unsigned int g_bounds_word;                                             \
  unsigned int accessor(cudaStream_t st) {                                                   \
    unsigned int v = 0, z = 0;                                                               \
    if (!kChecked) return 0;                                                                 \
    if (cudaMemcpyFromSymbolAsync(&v, g_bounds_word, sizeof v, 0, cudaMemcpyDeviceToHost,   \
                                  st) != cudaSuccess ||                                      \
        cudaMemcpyToSymbolAsync(g_bounds_word, &z, sizeof z, 0, cudaMemcpyHostToDevice,     \
                                st) != cudaSuccess ||                                        \
        cudaStreamSynchronize(st) != cudaSuccess)                                           \
      return 0x80000000u;                                                                    \
    return v;                                                                                \
  }

// ---------------------------------------------------------------------------------------------
// workspace
// ---------------------------------------------------------------------------------------------
struct Workspace {
  int device = 0;
  int max_G = 0, max_V = 0, max_H = 0, max_W = 0, max_deg = 0, max_nt = 0;
  // current problem
  int G = 0, V = 0, H = 0, W = 0, deg = 0, TX = 0, TY = 0, nt = 0;
  int stage = 0;  // 0 empty, 1 projected, 2 binned, 3 rendered, 4 replayed
  bool det = false;  // fixed-point integer accumulation (bitwise reproducible sums)
  long long launches = 0;

  // per (v, g)
  float4* rec = nullptr;     // [V*G*4]
  ushort4* rect = nullptr;   // [V*G] tile rectangle x0, y0, x1, y1 (16-bit tile coordinates)
  int* counts = nullptr;     // [V*G] tile counts in depth order, then their exclusive scan
  float* acc = nullptr;      // [V*G*8] score sums: (q, w r (3)), (w rho, w rho d (2), unused)
  bool acc_clean = false;    // acc is all zero (the projection clears it; a replay uses it up)
  double* accb = nullptr;    // [max_V*max_G*10] renderer-backward sums, allocated on first use
  double* sacc = nullptr;    // [G*C] scatter sums, grown on demand
  // deterministic mode: 128-bit fixed-point (low, high) words of the replay / backward sums
  unsigned long long* acc_fix = nullptr;
  size_t acc_fix_cap = 0;
  unsigned long long* accb_fix = nullptr;
  size_t accb_fix_cap = 0;
  size_t sacc_cap = 0;
  float* views = nullptr;    // [V*20]: viewmat (16) + intrinsics (4)
  int* last = nullptr;       // [V*H*W]
  const float* img = nullptr;   // C_hat written by the last render (caller-owned)
  const float* Tfin = nullptr;  // final transmittance written by the last render (caller-owned)
  const int* ncon = nullptr;    // contributor counts written by the last render (caller-owned)
  const float* bg = nullptr;    // background colour of the last render (caller-owned)

  // scan partials (int64)
  long long* part = nullptr;
  size_t part_cap = 0;

  // per-(v, g) depth order
  uint32_t* dkey = nullptr;    // [V*G] depth sort keys (written by the projection)
  uint32_t* kbits = nullptr;   // [V][kKeyStripes][2]: max visible key, max complement of one
  unsigned long long* ntot = nullptr;  // [V][kKeyStripes] instance counts (striped)
  unsigned long long* h_ntot = nullptr;  // pinned, mapped (hd_ntot: its device address)
  unsigned long long* hd_ntot = nullptr;
  uint32_t* dk1 = nullptr;     // [V*G] radix ping-pong keys (dkey itself is never overwritten)
  uint32_t* dk2 = nullptr;     // [V*G]
  uint32_t* dv0 = nullptr;     // [V*G] radix values (Gaussian index), ping
  uint32_t* dv1 = nullptr;     // [V*G] pong
  ushort4* rect_s = nullptr;   // [V*G] tile rectangles in depth order

  // instances
  size_t inst_cap = 0;
  uint32_t* inst_tile = nullptr;  // [N] tile id within its view, emitted in depth order
  uint32_t* inst_g = nullptr;     // [N] Gaussian index
  uint32_t* sval = nullptr;       // [N] the tile lists: Gaussian indices, tile-major
  // per (tile, 32-entry chunk, warp): entries some pixel of the warp composited (render -> replay)
  uint32_t* umask = nullptr;
  size_t umask_cap = 0;
  // per (tile, pixel, 32-entry chunk): entries that pixel composited (render -> score replay),
  // four chunks of one pixel per 16-byte group, pixels side by side
  uint32_t* lmask = nullptr;
  size_t lmask_cap = 0;

  // tile histogram [sum_v nt * blocks_v] (int32, scanned in place)
  size_t hist_cap = 0;
  int* hist = nullptr;
  long long* tile_off = nullptr;  // [V*(nt+1)]
  int* tile_order = nullptr;      // [V*nt] tiles (v*nt + t) in launch order, longest list first

  // per-view tables
  long long* d_vstart = nullptr;  // [V+1] first instance of each view
  int* d_bstart = nullptr;        // [V+1] first binning block of each view
  long long* h_vstart = nullptr;  // pinned, mapped (hd_*: device addresses of the same memory)
  int* h_bstart = nullptr;        // pinned, mapped
  uint32_t* h_kbits = nullptr;    // pinned, mapped [V][kKeyStripes][2]
  long long* hd_vstart = nullptr;
  int* hd_bstart = nullptr;
  uint32_t* hd_kbits = nullptr;
  long long n_total = 0;
  int n_blocks = 0;

  long long* d_scratch = nullptr;  // small device scratch (reductions)
  long long* h_scratch = nullptr;  // pinned

  // per-kernel timing (off by default)
  bool prof = false;
  std::vector<cudaEvent_t> ev_pool;
  std::vector<int> ev_open;  // (id, start event, end event) triples of recorded launches
  int ev_used = 0;
  double prof_ms[SPLAT_NUM_KERNELS] = {0};
  long long prof_n[SPLAT_NUM_KERNELS] = {0};

  std::string err;
};

}  // namespace splat

struct splat_ws {
  splat::Workspace w;
};

// launch helpers ------------------------------------------------------------------------------
namespace splat {

inline int set_err(Workspace& w, int code, const std::string& msg) {
  w.err = msg;
  return code;
}

// Bracket a kernel with timing events when profiling is on. Returns a token for prof_end.
inline int prof_begin(Workspace& w, cudaStream_t st, int id) {
  if (!w.prof) return -1;
  while ((int)w.ev_pool.size() < w.ev_used + 2) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return -1;
    w.ev_pool.push_back(e);
  }
  const int a = w.ev_used;
  w.ev_used += 2;
  cudaEventRecord(w.ev_pool[a], st);
  w.ev_open.push_back(id);
  w.ev_open.push_back(a);
  return a;
}
inline void prof_end(Workspace& w, cudaStream_t st, int tok) {
  if (tok < 0) return;
  cudaEventRecord(w.ev_pool[tok + 1], st);
}

inline int check_launch(Workspace& w, const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return set_err(w, SPLAT_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
  w.launches += 1;
  return SPLAT_OK;
}

// host entry points implemented in the .cu files
int launch_project(Workspace& w, const float* means, const float* lsc, const float* quats,
                   const float* opac, const float* sh, cudaStream_t st);
int launch_binning(Workspace& w, cudaStream_t st);
int launch_render(Workspace& w, const float* bg, float* img, float* T_final, int* n_contrib,
                  cudaStream_t st);
int launch_replay(Workspace& w, const float* obs, cudaStream_t st);
int launch_render_replay(Workspace& w, const float* bg, const float* obs, float* img,
                         float* T_final, int* n_contrib, cudaStream_t st);
int launch_finalize(Workspace& w, float lambda, float* tokens, cudaStream_t st);
int launch_partials(Workspace& w, float* partials, cudaStream_t st);
cudaError_t launch_finalize_partials(const float* partials, int G, int deg, double lambda,
                                     float* tokens, cudaStream_t st);
int launch_backward(Workspace& w, const float* obs, cudaStream_t st);
int launch_grad(Workspace& w, const float* lsc, const float* quats, const float* sh, float* raw,
                float* det, float* sup, float* psc, cudaStream_t st);
int launch_features(Workspace& w, const float* feats, int C, float* out, cudaStream_t st);
int launch_scatter(Workspace& w, const float* map, const float* obs, int C, float* out,
                   cudaStream_t st);
int launch_pair_count(Workspace& w, cudaStream_t st);
// the score sums widened to doubles into out [V*G*8] (the inspection copy)
int launch_acc_to_double(Workspace& w, double* out, cudaStream_t st);
// the records in the documented order into out [V*G*16] (the inspection copy)
int launch_copy_records(Workspace& w, float* out, cudaStream_t st);
int launch_copy_rects(Workspace& w, int* out, cudaStream_t st);
unsigned int bounds_word_raster(cudaStream_t st);
unsigned int bounds_word_binning(cudaStream_t st);
unsigned int bounds_word_attributes(cudaStream_t st);
int binning_configure(Workspace& w);

// reduce-then-scan over n int32 values into int64 exclusive prefixes (out has n + 1 entries; the
// last is the total). Uses w.part as scratch.
// same, int32 in place (values and total < 2^31)
int scan_i32_inplace(Workspace& w, int* data, long long n, cudaStream_t st);
// Stream-ordered clear and word copy done by kernels on the SMs, never by a copy engine: inside a
// step nothing may queue behind a caller's large host<->device transfers on other streams (a
// copy engine serves its queue in order). copy_words also moves the few words the host reads or
// writes each step through mapped pinned memory (sizes in bytes, multiples of 4).
int zero_async(Workspace& w, void* p, size_t bytes, cudaStream_t st, const char* what);
int copy_words(Workspace& w, const void* src, void* dst, size_t bytes, cudaStream_t st,
               const char* what);

}  // namespace splat
