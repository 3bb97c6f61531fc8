// Device helpers shared by the kernels that traverse the per-tile contributor lists (render,
// score replay, renderer backward, attribute render and scatter): the rasteriser's per-entry alpha
// with its skip rules, the warp-block reach test, the composited-entry mask index, and the
// transpose-reduction that sums per-entry values over a warp's 32 pixels.
//
// Source: "Research Proposal: Renderer Score Tokens for Recurrent Gaussian Splatting",
// "Two-Stage Algorithm" (both passes walk the same tile bins in the same order with the same
// decisions; per-Gaussian contributions are reduced on chip -- here over each warp of a tile --
// before global atomics).
//
// Packed fp32 pairs (__fmul2_rn, __fadd2_rn, __ffma2_rn: one instruction for two lanes' worth of
// work) round each element exactly like the scalar operation, and the pair loops here are
// issue-bound, so they use them where two independent operations of one kind meet. One rule
// keeps the results bit-identical to the scalar arithmetic: the compiler fuses a packed product
// whose only consumer is a packed add into one fma (also when both are written as PTX with an
// explicit rounding mode, and -fmad=false does not stop it), so a packed product only ever feeds
// scalar adds (which -fmad=false keeps unfused), packed adds take no products, and a packed fma
// stands only where one rounding is meant (fma(a, -1, b) is b - a rounded once).
#pragma once
#include "common.cuh"

namespace splat {
namespace {

// A tile's eight warp blocks run in kCtaPerTile CTAs of kCtaWarps warps each (two of four by
// default). The warps walk the lists independently (no CTA barriers), so a CTA is only a residency
// unit: smaller CTAs let the warps of a finished block make room sooner.
#ifndef SPLAT_CTA_WARPS
#define SPLAT_CTA_WARPS 4
#endif
constexpr int kCtaWarps = SPLAT_CTA_WARPS;
static_assert(kCtaWarps == 1 || kCtaWarps == 2 || kCtaWarps == 4 || kCtaWarps == 8,
              "warps per CTA divide the tile's eight warp blocks");
constexpr int kCtaPerTile = 8 / kCtaWarps;
constexpr int kThreads = 32 * kCtaWarps;
constexpr float kAlphaMin = 1.0f / 255.0f;

struct Entry {
  bool use;
  float alpha, dx, dy;
};

// Pixel blocks of the warps. A tile has eight warps (over its CTAs); warp w covers a kWarpW x
// kWarpH block of the 16x16 tile (row-major), lane l the pixel (l % kWarpW, l / kWarpW) of its
// block. Every kernel that walks the lists uses this one mapping: the render records per warp
// which entries some pixel of the block composited, and the later passes read those masks.
#ifndef SPLAT_WARP_W
#define SPLAT_WARP_W 8
#endif
constexpr int kWarpW = SPLAT_WARP_W;
constexpr int kWarpH = 32 / kWarpW;
static_assert(kTile % kWarpW == 0 && kTile % kWarpH == 0 &&
              (kTile / kWarpW) * (kTile / kWarpH) == 8, "eight warp blocks per tile");

// this warp's block (0 .. 7) in its tile
__device__ __forceinline__ int tile_warp() {
  return (int)((blockIdx.y * gridDim.x + blockIdx.x) % kCtaPerTile) * kCtaWarps +
         (int)(threadIdx.x >> 5);
}

// pixel of this thread in tile (tx, ty), and the top-left corner of its warp's block
__device__ __forceinline__ void tile_pixel(int tx, int ty, int& i, int& j, int& bx, int& by) {
  const int warp = tile_warp(), lane = threadIdx.x & 31;
  bx = tx * kTile + (warp % (kTile / kWarpW)) * kWarpW;
  by = ty * kTile + (warp / (kTile / kWarpW)) * kWarpH;
  i = bx + lane % kWarpW;
  j = by + lane / kWarpW;
}

// Can the entry's ellipse {exponent >= cut} (centre A.xy, half-extents ex, ey precomputed by the
// projection, conservatively widened) reach a pixel centre of the warp's block: columns
// x0 + 0.5 .. x0 + kWarpW - 0.5, rows y0 + 0.5 .. y0 + kWarpH - 0.5? Entries outside would only
// be skipped, so leaving them out changes no decision.
__device__ __forceinline__ bool reaches_block(float4 A, float ex, float ey, float x0, float y0) {
  return A.x + ex >= x0 + 0.5f && A.x - ex <= x0 + ((float)kWarpW - 0.5f) &&
         A.y + ey >= y0 + 0.5f && A.y - ey <= y0 + ((float)kWarpH - 0.5f);
}

// (tile, view) of this CTA: the list-walking kernels launch a (tiles x kCtaPerTile, views) grid
// and take the tiles in the order the binning wrote (longest list first). False for an order
// entry outside [0, V nt) (checked build only; the CTA then does nothing).
__device__ __forceinline__ bool block_tile(const int* __restrict__ order, int nt,
                                           unsigned int* bounds_word, int& t, int& v) {
  const int o = order[(blockIdx.y * gridDim.x + blockIdx.x) / kCtaPerTile];
  if (!in_bounds((unsigned)o, (unsigned long long)nt * gridDim.y, bounds_word)) return false;
  v = o / nt;
  t = o - v * nt;
  return true;
}

// position of the composited-entry mask of (global tile gt, chunk starting at list position p):
// distinct for every chunk of every tile, at most N / 32 + V * nt
__device__ __forceinline__ long long chunk_index(long long p, int gt) { return (p >> 5) + gt; }

// Per-pixel composited-entry masks: the render stores, for every 32-entry chunk its warp walks,
// one word per pixel (bit q: the pixel composited list entry 32 c + q of its tile). Four
// consecutive chunks of one pixel form a 16-byte group, and the 256 pixels' groups of chunks
// 4 gr .. 4 gr + 3 lie side by side (a warp stores 512 contiguous bytes per group; a pixel loads
// one group per four chunks). The tile's region starts at word 1024 ((s >> 7) + gt) (s = the
// tile's first list position, gt = v nt + t) and holds ceil(len / 128) groups of 1024 words; the
// regions of consecutive tiles do not overlap because ceil(len / 128) <= (e >> 7) - (s >> 7) + 1,
// and all of them fit in 1024 ((N >> 7) + V nt + 1) words for N list entries in total.
__device__ __forceinline__ size_t lmask_region(long long s, int gt) {
  return (size_t)1024 * (size_t)((s >> 7) + gt);
}

// The list-walking kernels stage, per entry, the record's r0 = (mx, my, colour r, colour g) and
// r2 = (conic a, b, c, opacity) as they are, plus (colour b, cut) from r1, and form the
// evaluation operands from them (register moves only):
//   A = (mx, my, conic a, conic b), B = (conic c, opacity, colour r, colour g)
__device__ __forceinline__ void entry_operands(float4 R0, float4 R2, float4& A, float4& B) {
  A = make_float4(R0.x, R0.y, R2.x, R2.y);
  B = make_float4(R2.z, R2.w, R0.z, R0.w);
}

// alpha of one list entry at pixel centre (px, py), with the rasteriser's skip rules
__device__ __forceinline__ Entry eval_entry(const float4 A, const float4 Bq, float cut, float px,
                                            float py) {
  Entry e;
  // (px - A.x, py - A.y) in one packed op: fma(a, -1, p) rounds p - a exactly once
  const float2 d = __ffma2_rn(make_float2(A.x, A.y), make_float2(-1.0f, -1.0f), make_float2(px, py));
  e.dx = d.x;
  e.dy = d.y;
  const float t1 = A.z * e.dx * e.dx;
  const float t2 = Bq.x * e.dy * e.dy;
  const float t3 = A.w * e.dx * e.dy;
  const float pw = -0.5f * (t1 + t2) - t3;
  e.use = false;
  e.alpha = 0.0f;
  if (pw > 0.0f || pw < cut) return e;
  // here cut <= pw <= 0 and cut >= log(1/255) - 1e-3 (opacity <= 1), inside exp_cw_core's range
  const float al = fminf(0.99f, Bq.y * exp_cw_core(pw));
  if (al < kAlphaMin) return e;
  e.alpha = al;
  e.use = true;
  return e;
}

// one butterfly step of the transpose-reduction: lanes with `hi` keep the upper half of their
// values and send the lower half, the others the reverse; the received half is added
template <int HALF>
__device__ __forceinline__ void tr_step(float* x, bool hi, int off) {
  if constexpr (HALF == 1) {
    const float send = hi ? x[0] : x[1];
    const float keep = hi ? x[1] : x[0];
    x[0] = keep + __shfl_xor_sync(0xffffffffu, send, off);
  } else {
#pragma unroll
    for (int k = 0; k < HALF; k += 2) {  // two values per packed add (keep + received)
      const float s0 = hi ? x[k] : x[k + HALF], k0 = hi ? x[k + HALF] : x[k];
      const float s1 = hi ? x[k + 1] : x[k + 1 + HALF], k1 = hi ? x[k + 1 + HALF] : x[k + 1];
      const float2 rv = make_float2(__shfl_xor_sync(0xffffffffu, s0, off),
                                    __shfl_xor_sync(0xffffffffu, s1, off));
      const float2 sum = __fadd2_rn(make_float2(k0, k1), rv);
      x[k] = sum.x;
      x[k + 1] = sum.y;
    }
  }
}

// Sum NV per-lane values over the warp so that value k ends in the lanes whose `slot` is k:
// log2(NV) transpose steps (each lane keeps half of what it holds and sends the other half), then
// a plain butterfly over the remaining lane bits. After it, lane l holds the warp sum of value
// (l >> (5 - log2 NV)) & (NV - 1) in x[0] when (l & (32 / NV - 1)) == 0.
template <int NV>
__device__ __forceinline__ void slot_reduce(float* x, int lane) {
  if constexpr (NV >= 16) tr_step<8>(x, lane & 16, 16);
  if constexpr (NV >= 8) tr_step<4>(x, lane & (NV >= 16 ? 8 : 16), NV >= 16 ? 8 : 16);
  if constexpr (NV >= 4) tr_step<2>(x, lane & (32 / NV * 2), 32 / NV * 2);
  if constexpr (NV >= 2) tr_step<1>(x, lane & (32 / NV), 32 / NV);
#pragma unroll
  for (int o = 32 / NV / 2; o >= 1; o >>= 1) x[0] += __shfl_xor_sync(0xffffffffu, x[0], o);
}
template <int NV>
__device__ __forceinline__ int slot_of(int lane) {
  constexpr int sh = NV == 1 ? 5 : NV == 2 ? 4 : NV == 4 ? 3 : NV == 8 ? 2 : 1;
  return NV == 1 ? 0 : (lane >> sh) & (NV - 1);
}
template <int NV>
__device__ __forceinline__ bool slot_holder(int lane) { return (lane & (32 / NV - 1)) == 0; }

}  // namespace
}  // namespace splat
