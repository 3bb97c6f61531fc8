// Stage 1 front-to-back compositing and Stage 2 analytic score replay.
//
// Source: "Research Proposal: Renderer Score Tokens for Recurrent Gaussian Splatting" --
// "Two-Stage Algorithm" (Stage 1 step 2: compositing to C_hat, final transmittance, contributor
// count; Stage 2: second front-to-back traversal over the same tile bins and order, prefix colour
// P and transmittance T, suffix composite C+ = (C_hat - P - T alpha c) / (T (1 - alpha) + eps),
// explicit masks, per-Gaussian segmented/atomic accumulation) and "Exact Score Operators"
// (o = sigmoid(a), alpha = o G, w = T alpha, rho = <r, c - C+>, q = sum w; the opacity-logit,
// SH and projected-centre scores).
//
// One thread per pixel of the 16x16 tile in kCtaPerTile CTAs per (tile, view), the CTAs taking
// the tiles in the binning's launch order (longest list first, so that no long list starts in the
// last wave); the eight warps (an 8x4 pixel block each) walk the tile's list independently, with
// no CTA barrier: each warp stages 32-entry
// chunks of records in its own shared-memory slice, keeps by ballot the entries whose precomputed
// box reaches its block, and stops when all its pixels are saturated. Both passes evaluate alpha
// through the same device function, so the replay takes exactly the render's decisions; the
// render also leaves, per (tile, warp, chunk), the mask of entries that composited some pixel of
// the warp, and the replay visits only those.
//
// Early skip. Most (pixel, entry) pairs of a tile lie far outside the Gaussian's footprint. The
// projection stores with every record cut = log((1/255) / o) - 1e-3; an exponent below cut
// gives o exp(pw) < (1/255) exp(-1e-3), far below 1/255 even after the few-ulp errors of the
// exp and of the product, so the entry is skipped without evaluating exp -- the same decision the
// full evaluation takes, never a different one. The record also holds the half-extents of the
// ellipse {exponent >= cut}; a warp only evaluates the entries whose box reaches its block. (8x4
// blocks meet ~17 % fewer entries than 16x2 strips of the same area: a squarer block has a
// shorter perimeter for footprints to overlap.)
//
// Replay arithmetic. The suffix numerators C_hat - P - T alpha c are formed per channel exactly
// as the recovery equation writes them (their cancellation dominates the fp32 error of C+), then
// multiplied by one fast reciprocal of T (1 - alpha) + eps (T (1 - alpha) >= 1e-6 wherever the
// result is used; relative error a few 1e-8). (Rewriting rho through
// running dot products <r, P> is algebraically the same but moves that cancellation and costs
// ~4e-4 relative token error.) The seven per-pixel terms (w, w r (3), w rho, w rho (p - mu2D) (2))
// reach the (view, Gaussian) sums either pair by pair (two 16-byte fp32 vector reductions) or,
// where many pixels of a warp composite the same entry, summed over the warp first by a
// transpose-reduction (each exchange step halves the values a lane carries: 9 shuffles instead of
// 35) and reduced once per (entry, warp block) -- see k_replay. The SH block never enters the
// pixel loop: M_color w (B (x) r) factors into M_color B (x) (sum w r); the mean block
// Sigma^-1 (sum w rho d) is formed once per (Gaussian, view) in finalisation. The render and the
// replay also run as one kernel (k_render<true>, splat_render_score).
#include <algorithm>

#include "traverse.cuh"

namespace splat {

SPLAT_BOUNDS_WORD(bounds_word_raster)

namespace {

// Deterministic accumulation: each warp's partial sum x (fp32) is turned into the signed 128-bit
// fixed-point integer X = x 2^60 (exact for |x| >= 2^-37; smaller values are truncated toward
// zero, the same way every run) and added with two 64-bit integer atomics -- the low word, then
// the high word plus the carry out of this particular low-word add. Integer addition does not
// depend on order, so the sums are the same bits on every run; the total of the carries is exactly
// the number of times the low word wrapped. A last pass turns (high, low) into a double.
constexpr int kFixShift = 60;

__device__ __forceinline__ void add_fixed(unsigned long long* lohi, float x) {
  const unsigned int bits = __float_as_uint(x);
  const int ex = (int)((bits >> 23) & 0xffu);
  if (ex == 0 || ex == 0xff) return;  // zero, subnormal (below 2^-126) or not finite
  const unsigned long long m = (bits & 0x7fffffu) | 0x800000u;  // x = +-m 2^(ex - 150)
  const int sh = ex - 150 + kFixShift;                           // X = m 2^sh
  unsigned long long lo, hi;
  if (sh >= 64) {
    lo = 0ull;
    hi = sh - 64 < 40 ? m << (sh - 64) : 0ull;  // |x| >= 2^67 does not occur here
  } else if (sh > 40) {
    lo = m << sh;
    hi = m >> (64 - sh);
  } else if (sh >= 0) {
    lo = m << sh;
    hi = 0ull;
  } else {
    lo = -sh < 24 ? m >> (-sh) : 0ull;
    hi = 0ull;
  }
  if (bits >> 31) {  // two's complement of the 128-bit value
    lo = ~lo + 1ull;
    hi = ~hi + (lo == 0ull ? 1ull : 0ull);
  }
  if (lo) {
    const unsigned long long old = atomicAdd(lohi, lo);
    if (old + lo < old) hi += 1ull;  // carry out of this add
  }
  if (hi) atomicAdd(lohi + 1, hi);
}

// (high, low) pairs -> T (double or float): dst[k] = (hi 2^64 + lo) 2^-60, rounded once to T
template <typename T>
__global__ void k_fixed_to(const unsigned long long* __restrict__ src, T* __restrict__ dst,
                           long long n) {
  for (long long k = (long long)blockIdx.x * blockDim.x + threadIdx.x; k < n;
       k += (long long)gridDim.x * blockDim.x) {
    const unsigned long long lo = src[2 * k], hi = src[2 * k + 1];
    dst[k] = (T)(ldexp((double)(long long)hi, 64 - kFixShift) + ldexp((double)lo, -kFixShift));
  }
}

// Score replay in deterministic mode: each warp walks the entries that some pixel of its block
// composited, reduces the seven per-pixel terms of each entry over the warp (a fixed tree) and
// adds the warp's sums as fixed-point integers (order-independent).
__global__ void __launch_bounds__(kThreads, 5 * kCtaPerTile)  // 48 registers: 40 warps per SM
k_replay_det(const float4* __restrict__ rec, const uint32_t* __restrict__ ids,
             const long long* __restrict__ tile_off, const int* __restrict__ order,
             int G, int H, int W, int TX, int nt,
             const float* __restrict__ img, const float* __restrict__ obs,
             const int* __restrict__ last, const uint32_t* __restrict__ umask,
             unsigned long long* __restrict__ acc_fix) {
  int t, v;
  if (!block_tile(order, nt, &g_bounds_word, t, v)) return;
  const int tx = t % TX, ty = t / TX;
  int i, j, bx, by;
  tile_pixel(tx, ty, i, j, bx, by);
  const bool inside = i < W && j < H;
  const long long s = tile_off[(size_t)v * (nt + 1) + t];
  const int gt = v * nt + t;
  // Like the render, each warp walks the list on its own (no CTA barriers), in 32-entry chunks;
  // per chunk it stages and evaluates only the entries the render recorded as composited by some
  // pixel of the warp -- every other entry contributes nothing to any of its pixels. Its
  // per-entry sums go straight from the seven lanes holding them to the fixed-point words.
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;  // warp in the CTA
  const int twarp = tile_warp();                                 // block in the tile
  __shared__ float4 s_a[kThreads], s_b[kThreads];
  __shared__ float2 s_c[kThreads];
  __shared__ uint32_t s_g[kThreads];
  float4* wa = s_a + warp * 32;
  float4* wb = s_b + warp * 32;
  float2* wc = s_c + warp * 32;
  uint32_t* wg = s_g + warp * 32;
  const float px = (float)i + 0.5f, py = (float)j + 0.5f;
  float Ch0 = 0.0f, Ch1 = 0.0f, Ch2 = 0.0f, r0 = 0.0f, r1 = 0.0f, r2 = 0.0f;
  int lst = 0;
  if (inside) {
    const size_t p = ((size_t)v * H + j) * W + i;
    Ch0 = img[3 * p];
    Ch1 = img[3 * p + 1];
    Ch2 = img[3 * p + 2];
    r0 = Ch0 - obs[3 * p];
    r1 = Ch1 - obs[3 * p + 1];
    r2 = Ch2 - obs[3 * p + 2];
    lst = last[p];
  }
  const int wmax = __reduce_max_sync(0xffffffffu, lst);  // entries this warp must traverse
  const size_t vG = (size_t)v * G;
  float T = 1.0f, P2 = 0.0f;  // transmittance, prefix colour (channels 0 and 1 packed)
  float2 P01 = make_float2(0.0f, 0.0f);
  const float2 Ch01 = make_float2(Ch0, Ch1), r01 = make_float2(r0, r1);
  const float2 m1 = make_float2(-1.0f, -1.0f);
  const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
  const int slot = (lane >> 2) & 7;  // value index this lane holds after the reduction
  for (int base = 0; base < wmax; base += 32) {
    uint32_t bits = umask[chunk_index(s + base, gt) * 8 + twarp];
    if (!bits) continue;  // warp-uniform
    bool bad = false;
    if ((bits >> lane) & 1u) {
      const uint32_t g = ids[s + base + lane];
      bad = !in_bounds(g, (unsigned)G, &g_bounds_word);
      if (!bad) {
        const float4* rl = rec + rec_lo(vG + g);  // r0, r1
        const float4* rh = rec + rec_hi(vG + g);  // r2, r3
        const float2 r1 = reinterpret_cast<const float2*>(rl + 1)[0];  // (colour b, cut)
        wa[lane] = rl[0];
        wb[lane] = rh[0];
        wc[lane] = r1;
        wg[lane] = g;
      }
    }
    if (kChecked) bits &= ~__ballot_sync(0xffffffffu, bad);
    __syncwarp();
    while (bits) {  // warp-uniform: entries some pixel of this warp composited, in list order
      const int q = __ffs(bits) - 1;
      bits &= bits - 1;
      float x[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
      bool used = false;
      if (base + q < lst) {
        float4 A, Bq;
        entry_operands(wa[q], wb[q], A, Bq);
        const float2 Cq = wc[q];
        const Entry E = eval_entry(A, Bq, Cq.y, px, py);
        if (E.use) {
          used = true;
          const float al = E.alpha;
          const float den = T * (1.0f - al);
          const float w = al * T;
          const float c0 = Bq.z, c1 = Bq.w, c2 = Cq.x;
          // suffix numerators C_hat - P - w c per channel, in the recovery equation's order and
          // unfused like the render's colour sum, so that at the last entry C_hat - P - w c is
          // exactly the background term (their cancellation dominates the fp32 error of C+);
          // then one reciprocal of the denominator (T (1 - alpha) >= 1e-6 here, so the fast
          // reciprocal's relative error of a few 1e-8 is far inside the tokens' bar)
          const float2 ww = make_float2(w, w);
          const float2 c01 = make_float2(c0, c1);
          const float2 wc01 = __fmul2_rn(ww, c01);
          const float wc2 = w * c2;
          // C_hat - P for channels 0 and 1 in one op (fma(P, -1, C_hat) rounds the difference
          // once); the products w c are subtracted by scalar ops
          const float2 cp01 = __ffma2_rn(P01, m1, Ch01);
          const float n0 = cp01.x - wc01.x;
          const float n1 = cp01.y - wc01.y;
          const float n2 = (Ch2 - P2) - wc2;
          const float inv = __fdividef(1.0f, den + 1e-12f);
          const float2 a01 = __ffma2_rn(make_float2(n0, n1), make_float2(-inv, -inv), c01);
          const float rho = fmaf(r0, a01.x, fmaf(r1, a01.y, r2 * fmaf(-n2, inv, c2)));
          const bool Ma = (den >= 1e-4f) && (al < 0.99f);
          const float2 wr01 = __fmul2_rn(ww, r01);
          x[0] = w;
          x[1] = wr01.x;
          x[2] = wr01.y;
          x[3] = w * r2;
          if (Ma) {
            const float wr = w * rho;
            const float2 wd = __fmul2_rn(make_float2(wr, wr), make_float2(E.dx, E.dy));
            x[4] = wr;
            x[5] = wd.x;
            x[6] = wd.y;
          }
          P01.x = P01.x + wc01.x;
          P01.y = P01.y + wc01.y;
          P2 = P2 + wc2;
          T = den;
        }
      }
      if (__any_sync(0xffffffffu, used)) {
        tr_step<4>(x, b4, 16);
        tr_step<2>(x, b3, 8);
        tr_step<1>(x, b2, 4);
        x[0] += __shfl_xor_sync(0xffffffffu, x[0], 2);
        x[0] += __shfl_xor_sync(0xffffffffu, x[0], 1);
        if ((lane & 3) == 0 && slot < 7 && x[0] != 0.0f)
          add_fixed(acc_fix + 2 * (((size_t)v * G + wg[q]) * kAccN + slot), x[0]);
      }
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------------------------
// Score replay (the default accumulation mode): per warp, one of two traversals.
//
// Per-pixel walks: each lane walks only the list entries ITS pixel composited -- read from the
// per-pixel masks the render stored -- in list order, keeping the pixel's prefix transmittance T
// and colour P exactly as the recovery equation needs them, and adds each (pixel, entry) pair's
// terms straight into the (view, Gaussian) sums with two 16-byte vector reductions into L2
// (red.global.add.v4.f32: (w, w r) and, where M_alpha holds, (w rho, w rho (p - mu2D), 0)). The
// warp runs as many iterations as its longest walk.
//
// Union loop: the warp visits every entry that some pixel of its block composited (the render's
// per-warp masks), all 32 lanes evaluate it, the seven per-pixel terms are summed over the warp
// (the transpose-reduction) and lanes 0 and 16 issue the two reductions once per (entry, warp).
//
// The walk does a pair's arithmetic once but costs one or two L2 reductions per pair (the L2
// reduction rate bounds it); the union loop spends ~160 instructions per visited entry whatever
// the number of lanes that composited it, but reduces once. So each warp counts its union entries
// U (the render's masks) and its composited pairs P (the pixels' contributor counts) and takes
// the union loop when P >= kUnionLanes U -- entries composited by many of its pixels at once, as
// with large Gaussians -- and the walks otherwise (pixel-aligned scenes: ~7 lanes per entry).
// Either way the per-pixel terms are the same fp32 values; the sums are fp32 and the order of the
// additions is not fixed, so their last bits vary from run to run (the deterministic mode gives
// fixed bits).
#ifndef SPLAT_UNION_LANES
#define SPLAT_UNION_LANES 9
#endif
constexpr int kUnionLanes = SPLAT_UNION_LANES;

__device__ __forceinline__ void red_add4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

// one composited (pixel, entry) pair of the replay: the suffix numerators C_hat - P - w c per
// channel in the recovery equation's order, unfused like the render's colour sum (at the last
// entry C_hat - P - w c is exactly the background term), one fast reciprocal of T (1 - alpha)
// (>= 1e-6 here), rho, the seven terms x (x[4..6] zero where M_alpha is off), then P and T
struct PixelState {
  float2 Ch01, r01, P01;
  float Ch2, r2, P2, T;
};
__device__ __forceinline__ bool replay_pair(PixelState& ps, const Entry& E, float c0, float c1,
                                            float c2, float x[8]) {
  const float al = E.alpha;
  const float den = ps.T * (1.0f - al);
  const float w = al * ps.T;
  const float2 ww = make_float2(w, w);
  const float2 c01 = make_float2(c0, c1);
  const float2 wc01 = __fmul2_rn(ww, c01);
  const float wc2 = w * c2;
  const float2 cp01 = __ffma2_rn(ps.P01, make_float2(-1.0f, -1.0f), ps.Ch01);
  const float nn0 = cp01.x - wc01.x;
  const float nn1 = cp01.y - wc01.y;
  const float nn2 = (ps.Ch2 - ps.P2) - wc2;
  const float inv = __fdividef(1.0f, den + 1e-12f);
  const float2 a01 = __ffma2_rn(make_float2(nn0, nn1), make_float2(-inv, -inv), c01);
  const float rho = fmaf(ps.r01.x, a01.x, fmaf(ps.r01.y, a01.y, ps.r2 * fmaf(-nn2, inv, c2)));
  const float2 wr01 = __fmul2_rn(ww, ps.r01);
  x[0] = w;
  x[1] = wr01.x;
  x[2] = wr01.y;
  x[3] = w * ps.r2;
  const bool ma = (den >= 1e-4f) && (al < 0.99f);  // M_alpha
  if (ma) {
    const float wr = w * rho;
    const float2 wd = __fmul2_rn(make_float2(wr, wr), make_float2(E.dx, E.dy));
    x[4] = wr;
    x[5] = wd.x;
    x[6] = wd.y;
  }
  ps.P01.x = ps.P01.x + wc01.x;
  ps.P01.y = ps.P01.y + wc01.y;
  ps.P2 = ps.P2 + wc2;
  ps.T = den;
  return ma;
}

// The replay of one warp block, given its pixel's state (C_hat, r = C_hat - C_obs, T = 1, P = 0),
// list bound lst and the warp's union entries U and composited pairs P. kFresh: the composited-
// entry masks were stored by this same launch (read through the coherent path, not the
// read-only one).
template <bool kFresh>
__device__ __forceinline__ void replay_walk(const float4* __restrict__ rec,
                                            const uint32_t* __restrict__ ids, long long s, int gt,
                                            int G, size_t vG, float px, float py, PixelState ps,
                                            int lst, int U, int P, const uint32_t* umask,
                                            const uint32_t* lmask, float* __restrict__ accv,
                                            float4* wa, float4* wb, float2* wc, uint32_t* wg) {
  const int lane = threadIdx.x & 31;
  const int twarp = tile_warp();
  if (U == 0) return;  // warp-uniform: nothing composited here
  const int wmax = __reduce_max_sync(0xffffffffu, lst);

  if (P >= kUnionLanes * U) {
    // ---- union loop ----------------------------------------------------------------------
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
    for (int base = 0; base < wmax; base += 32) {
      uint32_t bits = umask[chunk_index(s + base, gt) * 8 + twarp];
      if (!bits) continue;  // warp-uniform
      bool bad = false;
      if ((bits >> lane) & 1u) {
        const uint32_t g = ids[s + base + lane];
        bad = !in_bounds(g, (unsigned)G, &g_bounds_word);
        if (!bad) {
          const float4* rl = rec + rec_lo(vG + g);  // r0, r1
          const float4* rh = rec + rec_hi(vG + g);  // r2, r3
          const float2 r1 = reinterpret_cast<const float2*>(rl + 1)[0];  // (colour b, cut)
          wa[lane] = rl[0];
          wb[lane] = rh[0];
          wc[lane] = r1;
          wg[lane] = g;
        }
      }
      if (kChecked) bits &= ~__ballot_sync(0xffffffffu, bad);
      __syncwarp();
      while (bits) {  // warp-uniform: entries some pixel of this warp composited, in list order
        const int q = __ffs(bits) - 1;
        bits &= bits - 1;
        float x[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
        bool used = false;
        if (base + q < lst) {
          float4 A, Bq;
          entry_operands(wa[q], wb[q], A, Bq);
          const float2 Cq = wc[q];
          const Entry E = eval_entry(A, Bq, Cq.y, px, py);
          if (E.use) {
            used = true;
            replay_pair(ps, E, Bq.z, Bq.w, Cq.x, x);
          }
        }
        if (__any_sync(0xffffffffu, used)) {
          tr_step<4>(x, b4, 16);
          tr_step<2>(x, b3, 8);
          tr_step<1>(x, b2, 4);
          x[0] += __shfl_xor_sync(0xffffffffu, x[0], 2);
          x[0] += __shfl_xor_sync(0xffffffffu, x[0], 1);
          // value k now sits in lanes 4k .. 4k + 3: lanes 0 and 16 collect four each
          const float s1 = __shfl_down_sync(0xffffffffu, x[0], 4);
          const float s2 = __shfl_down_sync(0xffffffffu, x[0], 8);
          const float s3 = __shfl_down_sync(0xffffffffu, x[0], 12);
          float* a = accv + (size_t)wg[q] * kAccN;
          if (lane == 0) red_add4(a, x[0], s1, s2, s3);
          if (lane == 16 && (x[0] != 0.0f || s1 != 0.0f || s2 != 0.0f))
            red_add4(a + 4, x[0], s1, s2, 0.0f);
        }
      }
      __syncwarp();
    }
    return;
  }

  // ---- per-pixel walks (no warp-wide operation below: lanes leave independently) ------------
  const int cend = (lst + 31) >> 5;  // chunks holding this pixel's composited entries
  if (cend == 0) return;
  // this pixel's mask words: chunk c's in m, the rest of its group of four in n1..n3, the next
  // group prefetched in pre
  const uint4* lm = reinterpret_cast<const uint4*>(lmask + lmask_region(s, gt)) + (twarp * 32 + lane);
  const uint4 g0 = kFresh ? lm[0] : __ldg(lm);
  uint32_t m = g0.x, n1 = g0.y, n2 = g0.z, n3 = g0.w;
  uint4 pre = make_uint4(0u, 0u, 0u, 0u);
  if (4 < cend) pre = kFresh ? lm[256] : __ldg(lm + 256);
  int c = 0;
  for (;;) {
    while (!m) {  // next chunk with an entry of this pixel
      if (++c >= cend) return;
      if ((c & 3) == 0) {
        m = pre.x;
        n1 = pre.y;
        n2 = pre.z;
        n3 = pre.w;
        if (c + 4 < cend) {
          const uint4* nx = lm + (size_t)((c >> 2) + 1) * 256;
          pre = kFresh ? nx[0] : __ldg(nx);
        }
      } else {
        m = n1;
        n1 = n2;
        n2 = n3;
      }
    }
    const int q = __ffs(m) - 1;
    m &= m - 1u;
    const uint32_t g = ids[s + 32LL * c + q];
    if (!in_bounds(g, (unsigned)G, &g_bounds_word)) continue;
    const float4* rl = rec + rec_lo(vG + g);  // r0, r1
    const float4* rh = rec + rec_hi(vG + g);  // r2, r3
    const float4 r0 = __ldg(rl), r2 = __ldg(rh);
    const float c2 = __ldg(reinterpret_cast<const float*>(rl + 1));  // colour b
    const float4 A = make_float4(r0.x, r0.y, r2.x, r2.y), Bq = make_float4(r2.z, r2.w, r0.z, r0.w);
    // the render's alpha, bit for bit (a composited entry always passes the exponent cut)
    const Entry E = eval_entry(A, Bq, -INFINITY, px, py);
    if (!E.use) continue;
    float x[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
    const bool ma = replay_pair(ps, E, Bq.z, Bq.w, c2, x);
    float* a = accv + (size_t)g * kAccN;
    red_add4(a, x[0], x[1], x[2], x[3]);
    if (ma) red_add4(a + 4, x[4], x[5], x[6], 0.0f);
  }
}

// pixel state of the replay from the rendered colour and the observation
__device__ __forceinline__ PixelState replay_state(float Ch0, float Ch1, float Ch2, float o0,
                                                   float o1, float o2) {
  PixelState ps;
  ps.T = 1.0f;
  ps.P01 = make_float2(0.0f, 0.0f);
  ps.P2 = 0.0f;
  ps.Ch01 = make_float2(Ch0, Ch1);
  ps.Ch2 = Ch2;
  ps.r01 = make_float2(Ch0 - o0, Ch1 - o1);
  ps.r2 = Ch2 - o2;
  return ps;
}

__global__ void __launch_bounds__(kThreads, 4)
k_replay(const float4* __restrict__ rec, const uint32_t* __restrict__ ids,
         const long long* __restrict__ tile_off, const int* __restrict__ order,
         int G, int H, int W, int TX, int nt, const float* __restrict__ img,
         const float* __restrict__ obs, const int* __restrict__ last,
         const int* __restrict__ ncon, const uint32_t* __restrict__ umask,
         const uint32_t* __restrict__ lmask, float* __restrict__ acc) {
  int t, v;
  if (!block_tile(order, nt, &g_bounds_word, t, v)) return;  // CTA-uniform
  const int tx = t % TX, ty = t / TX;
  int i, j, bx, by;
  tile_pixel(tx, ty, i, j, bx, by);
  const bool inside = i < W && j < H;
  const long long s = tile_off[(size_t)v * (nt + 1) + t];
  const int gt = v * nt + t;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int twarp = tile_warp();
  float Ch0 = 0.0f, Ch1 = 0.0f, Ch2 = 0.0f, o0 = 0.0f, o1 = 0.0f, o2 = 0.0f;
  int lst = 0, nc = 0;
  if (inside) {
    const size_t p = ((size_t)v * H + j) * W + i;
    Ch0 = img[3 * p];
    Ch1 = img[3 * p + 1];
    Ch2 = img[3 * p + 2];
    o0 = obs[3 * p];
    o1 = obs[3 * p + 1];
    o2 = obs[3 * p + 2];
    lst = last[p];
    nc = ncon[p];
  }
  // the warp's union entries U (the render's per-warp masks) and composited pairs P
  const int wmax = __reduce_max_sync(0xffffffffu, lst);
  const int wch = (wmax + 31) >> 5;
  int u = 0;
  for (int c = lane; c < wch; c += 32) u += __popc(umask[chunk_index(s + 32LL * c, gt) * 8 + twarp]);
  const int U = __reduce_add_sync(0xffffffffu, u);
  const int P = __reduce_add_sync(0xffffffffu, nc);
  __shared__ float4 s_a[kThreads], s_b[kThreads];
  __shared__ float2 s_c[kThreads];
  __shared__ uint32_t s_g[kThreads];
  replay_walk<false>(rec, ids, s, gt, G, (size_t)v * G, (float)i + 0.5f, (float)j + 0.5f,
                     replay_state(Ch0, Ch1, Ch2, o0, o1, o2), lst, U, P, umask, lmask,
                     acc + (size_t)v * G * kAccN, s_a + warp * 32, s_b + warp * 32,
                     s_c + warp * 32, s_g + warp * 32);
}

// The render (kReplay = false), or render and score replay in one launch (kReplay): each warp
// renders its block, stores the render's outputs and masks, and replays its composited entries
// at once with the pixel state still in registers. Across an SM the warps are in different
// phases, so the render's issue-bound work and the replay's L2 reductions overlap instead of
// following one another. The arithmetic and the decisions are those of the separate passes.
template <bool kReplay>
__global__ void __launch_bounds__(kThreads)
k_render(const float4* __restrict__ rec, const uint32_t* __restrict__ ids,
         const long long* __restrict__ tile_off, const int* __restrict__ order,
         int G, int H, int W, int TX, int nt,
         const float* __restrict__ bgp, float* __restrict__ img, float* __restrict__ Tout,
         int* __restrict__ ncout, int* __restrict__ last, uint32_t* __restrict__ umask,
         uint32_t* __restrict__ lmask, const float* __restrict__ obs, float* __restrict__ acc) {
  int t, v;
  if (!block_tile(order, nt, &g_bounds_word, t, v)) return;
  const int tx = t % TX, ty = t / TX;
  int i, j, bx, by;
  tile_pixel(tx, ty, i, j, bx, by);
  const bool inside = i < W && j < H;
  const long long s = tile_off[(size_t)v * (nt + 1) + t];
  const long long e = tile_off[(size_t)v * (nt + 1) + t + 1];
  const int gt = v * nt + t;
  // Each warp walks the whole list on its own (no CTA barriers): it stages 32 entries into its
  // slice of shared memory, ballots which of them can reach its pixel block, evaluates only
  // those, and leaves as soon as its 32 pixels are done. Per 32-entry chunk it records which
  // entries some pixel of the warp composited: the replay visits exactly those.
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;  // warp in the CTA
  const int twarp = tile_warp();                                 // block in the tile
  __shared__ float4 s_a[kThreads], s_b[kThreads];
  __shared__ float2 s_c[kThreads];  // (colour b, exponent cut)
  float4* wa = s_a + warp * 32;
  float4* wb = s_b + warp * 32;
  float2* wc = s_c + warp * 32;
  // this pixel's composited-entry mask words (read by the score replay): chunk cc at
  // lmw[1024 (cc / 4) + cc % 4]
  uint32_t* lmw = lmask + lmask_region(s, gt) + 4 * (twarp * 32 + lane);
  int cc = 0;  // chunks walked
  const float x0f = (float)bx, y0f = (float)by;
  const float px = (float)i + 0.5f, py = (float)j + 0.5f;
  float T = 1.0f, C0 = 0.0f, C1 = 0.0f, C2 = 0.0f;
  int n = 0, lst = 0;
  int U = 0;  // (kReplay) entries some pixel of the warp composited
  bool done = !inside;
  const size_t vG = (size_t)v * G;
  for (long long base = s; base < e; base += 32, ++cc) {
    if (__all_sync(0xffffffffu, done)) break;
    const long long k = base + lane;
    bool hit = false;
    if (k < e) {
      const uint32_t gi = ids[k];
      if (in_bounds(gi, (unsigned)G, &g_bounds_word)) {
        const float4* rl = rec + rec_lo(vG + gi);  // r0, r1
        const float4* rh = rec + rec_hi(vG + gi);  // r2, r3
        const float4 r0 = rl[0], r1 = rl[1], r2 = rh[0];  // r1 = (colour b, cut, ex, ey)
        wa[lane] = r0;
        wb[lane] = r2;
        wc[lane] = make_float2(r1.x, r1.y);
        hit = reaches_block(r0, r1.z, r1.w, x0f, y0f);
      }
    }
    uint32_t bits = __ballot_sync(0xffffffffu, hit);
    uint32_t lbits = 0u;  // entries of this chunk this lane composited
    __syncwarp();
    while (bits) {  // warp-uniform: entries that can reach this warp's rows, in list order
      const int q = __ffs(bits) - 1;
      bits &= bits - 1;
      if (!done) {
        float4 A, Bq;
        entry_operands(wa[q], wb[q], A, Bq);
        const float2 Cq = wc[q];
        const Entry E = eval_entry(A, Bq, Cq.y, px, py);
        if (E.use) {
          const float Tn = T * (1.0f - E.alpha);
          if (Tn < 1e-4f) {
            done = true;
          } else {
            const float wgt = E.alpha * T;
            // unfused, as the replay accumulates its prefix P: at the last entry C_hat - P is
            // then exactly the background term, and the suffix recovery sees no rounding mismatch
            const float2 wc01 = __fmul2_rn(make_float2(wgt, wgt), make_float2(Bq.z, Bq.w));
            C0 = C0 + wc01.x;
            C1 = C1 + wc01.y;
            C2 = C2 + wgt * Cq.x;
            T = Tn;
            ++n;
            lst = (int)(base - s) + q + 1;
            lbits |= 1u << q;
          }
        }
      }
    }
    const uint32_t ubits = __reduce_or_sync(0xffffffffu, lbits);
    if (kReplay) U += __popc(ubits);
    if (lane == 0) umask[chunk_index(base, gt) * 8 + twarp] = ubits;
    lmw[(size_t)(cc >> 2) * 1024 + (cc & 3)] = lbits;
    __syncwarp();
  }
  if constexpr (!kReplay) {
    if (inside) {
      const size_t p = ((size_t)v * H + j) * W + i;
      img[3 * p + 0] = C0 + T * bgp[0];
      img[3 * p + 1] = C1 + T * bgp[1];
      img[3 * p + 2] = C2 + T * bgp[2];
      Tout[p] = T;
      ncout[p] = n;
      last[p] = lst;
    }
  } else {
    float Ch0 = 0.0f, Ch1 = 0.0f, Ch2 = 0.0f, o0 = 0.0f, o1 = 0.0f, o2 = 0.0f;
    if (inside) {
      const size_t p = ((size_t)v * H + j) * W + i;
      Ch0 = C0 + T * bgp[0];
      Ch1 = C1 + T * bgp[1];
      Ch2 = C2 + T * bgp[2];
      img[3 * p + 0] = Ch0;
      img[3 * p + 1] = Ch1;
      img[3 * p + 2] = Ch2;
      Tout[p] = T;
      ncout[p] = n;
      last[p] = lst;
      o0 = obs[3 * p];
      o1 = obs[3 * p + 1];
      o2 = obs[3 * p + 2];
    }
    const int P = __reduce_add_sync(0xffffffffu, n);
    __shared__ uint32_t s_g[kThreads];
    replay_walk<true>(rec, ids, s, gt, G, vG, px, py, replay_state(Ch0, Ch1, Ch2, o0, o1, o2),
                      lst, U, P, umask, lmask, acc + vG * kAccN, wa, wb, wc, s_g + warp * 32);
  }
}


// Renderer backward of L = 1/2 sum |C_hat - C_obs|^2 with the render's decisions held fixed.
// Each warp walks its composited entries BACK TO FRONT (chunks from the last one down, entries in
// a chunk from the highest position down), starting from the final transmittance and the
// background term: per entry T_i = T_{i+1} / (1 - alpha_i), and the composite behind the entry,
// S = sum_{j>i} T_j alpha_j c_j + T_final bg, is summed as it goes (no cancellation, unlike the
// front-to-back recovery C_hat - P - T alpha c). With
//   d C_hat / d alpha = T c - S / (1 - alpha),  ga = <r, d C_hat / d alpha>,
// and, where alpha = o G is not clamped, h = ga alpha, the pixel adds to its (view, Gaussian)
//   q += w, w r (3), h, h (dx, dy), h (dx^2, dx dy, dy^2)     (w = T alpha)
// by a 16-slot transpose-reduction per entry and fp64 atomics from the ten lanes holding sums.
template <bool kDet>
__global__ void __launch_bounds__(kThreads)
k_backward(const float4* __restrict__ rec, const uint32_t* __restrict__ ids,
           const long long* __restrict__ tile_off, const int* __restrict__ order,
           int G, int H, int W, int TX, int nt,
           const float* __restrict__ img, const float* __restrict__ Tfin,
           const float* __restrict__ bgp, const float* __restrict__ obs,
           const int* __restrict__ last, const uint32_t* __restrict__ umask,
           double* __restrict__ accb, unsigned long long* __restrict__ accb_fix) {
  int t, v;
  if (!block_tile(order, nt, &g_bounds_word, t, v)) return;
  const int tx = t % TX, ty = t / TX;
  int i, j, bx, by;
  tile_pixel(tx, ty, i, j, bx, by);
  const bool inside = i < W && j < H;
  const long long s = tile_off[(size_t)v * (nt + 1) + t];
  const int gt = v * nt + t;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;  // warp in the CTA
  const int twarp = tile_warp();                                 // block in the tile
  __shared__ float4 s_a[kThreads], s_b[kThreads];
  __shared__ float2 s_c[kThreads];
  __shared__ uint32_t s_g[kThreads];
  float4* wa = s_a + warp * 32;
  float4* wb = s_b + warp * 32;
  float2* wc = s_c + warp * 32;
  uint32_t* wg = s_g + warp * 32;
  const float px = (float)i + 0.5f, py = (float)j + 0.5f;
  float r0 = 0.0f, r1 = 0.0f, r2 = 0.0f, T = 1.0f, S0 = 0.0f, S1 = 0.0f, S2 = 0.0f;
  int lst = 0;
  if (inside) {
    const size_t p = ((size_t)v * H + j) * W + i;
    r0 = img[3 * p] - obs[3 * p];
    r1 = img[3 * p + 1] - obs[3 * p + 1];
    r2 = img[3 * p + 2] - obs[3 * p + 2];
    T = Tfin[p];
    S0 = T * bgp[0];
    S1 = T * bgp[1];
    S2 = T * bgp[2];
    lst = last[p];
  }
  const int wmax = __reduce_max_sync(0xffffffffu, lst);
  const size_t vG = (size_t)v * G;
  double* accv = accb + (size_t)v * G * kAccBN;
  const int slot = (lane >> 1) & 15;  // value index this lane holds after the reduction
  for (int base = (wmax - 1) & ~31; base >= 0; base -= 32) {
    uint32_t bits = umask[chunk_index(s + base, gt) * 8 + twarp];
    if (!bits) continue;  // warp-uniform
    bool bad = false;
    if ((bits >> lane) & 1u) {
      const uint32_t g = ids[s + base + lane];
      bad = !in_bounds(g, (unsigned)G, &g_bounds_word);
      if (!bad) {
        const float4* rl = rec + rec_lo(vG + g);  // r0, r1
        const float4* rh = rec + rec_hi(vG + g);  // r2, r3
        wa[lane] = rl[0];
        wb[lane] = rh[0];
        wc[lane] = reinterpret_cast<const float2*>(rl + 1)[0];  // (colour b, cut)
        wg[lane] = g;
      }
    }
    if (kChecked) bits &= ~__ballot_sync(0xffffffffu, bad);
    __syncwarp();
    while (bits) {  // warp-uniform, from the highest list position down
      const int q = 31 - __clz(bits);
      bits &= ~(1u << q);
      float x[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) x[k] = 0.0f;
      bool used = false;
      if (base + q < lst) {
        float4 A, Bq;
        entry_operands(wa[q], wb[q], A, Bq);
        const float2 Cq = wc[q];
        const Entry E = eval_entry(A, Bq, Cq.y, px, py);
        if (E.use) {
          used = true;
          const float al = E.alpha;
          const float i1m = __frcp_rn(1.0f - al);
          T = T * i1m;  // transmittance in front of the entry
          const float w = al * T;
          const float c0 = Bq.z, c1 = Bq.w, c2 = Cq.x;
          x[0] = w;
          x[1] = w * r0;
          x[2] = w * r1;
          x[3] = w * r2;
          if (al < 0.99f) {
            const float ga = T * (r0 * c0 + r1 * c1 + r2 * c2) - (r0 * S0 + r1 * S1 + r2 * S2) * i1m;
            const float h = ga * al;
            const float hx = h * E.dx, hy = h * E.dy;
            x[4] = h;
            x[5] = hx;
            x[6] = hy;
            x[7] = hx * E.dx;
            x[8] = hx * E.dy;
            x[9] = hy * E.dy;
          }
          S0 = S0 + w * c0;
          S1 = S1 + w * c1;
          S2 = S2 + w * c2;
        }
      }
      if (__any_sync(0xffffffffu, used)) {
        tr_step<8>(x, lane & 16, 16);
        tr_step<4>(x, lane & 8, 8);
        tr_step<2>(x, lane & 4, 4);
        tr_step<1>(x, lane & 2, 2);
        x[0] += __shfl_xor_sync(0xffffffffu, x[0], 1);
        if ((lane & 1) == 0 && slot < kAccBN && x[0] != 0.0f)
        {
          if constexpr (kDet)
            add_fixed(accb_fix + 2 * (((size_t)v * G + wg[q]) * kAccBN + slot), x[0]);
          else
            atomicAdd(accv + (size_t)wg[q] * kAccBN + slot, (double)x[0]);
        }
      }
    }
    __syncwarp();
  }
}

__global__ void k_widen(const float* __restrict__ src, double* __restrict__ dst, long long n) {
  for (long long k = (long long)blockIdx.x * blockDim.x + threadIdx.x; k < n;
       k += (long long)gridDim.x * blockDim.x)
    dst[k] = (double)src[k];
}

__global__ void k_pair_sum(const int* __restrict__ last, long long n, long long* out) {
  long long sacc = 0;
  for (long long k = (long long)blockIdx.x * blockDim.x + threadIdx.x; k < n;
       k += (long long)gridDim.x * blockDim.x)
    sacc += last[k];
  for (int o = 16; o > 0; o >>= 1) sacc += __shfl_xor_sync(0xffffffffu, sacc, o);
  if ((threadIdx.x & 31) == 0) atomicAdd((unsigned long long*)out, (unsigned long long)sacc);
}

}  // namespace

int launch_render(Workspace& w, const float* bg, float* img, float* T_final, int* n_contrib,
                  cudaStream_t st) {
  dim3 grid(w.nt * kCtaPerTile, w.V);
  const int tok = prof_begin(w, st, SPLAT_K_RENDER);
  k_render<false><<<grid, kThreads, 0, st>>>(w.rec, w.sval, w.tile_off, w.tile_order, w.G, w.H,
                                             w.W, w.TX, w.nt, bg, img, T_final, n_contrib, w.last,
                                             w.umask, w.lmask, nullptr, nullptr);
  prof_end(w, st, tok);
  return check_launch(w, "render kernel");
}

// the fixed-point (high, low) words of deterministic mode: allocated on first use, sized for the
// workspace maxima, cleared before every pass
static int fix_buffer(Workspace& w, unsigned long long** buf, size_t& cap, int nslot,
                      cudaStream_t st) {
  const size_t need = (size_t)w.max_V * w.max_G * nslot * 2;
  if (cap < need) {
    if (*buf) cudaFree(*buf);
    *buf = nullptr;
    cap = 0;
    if (cudaMalloc(buf, need * sizeof(unsigned long long)) != cudaSuccess) {
      *buf = nullptr;
      cudaGetLastError();
      return set_err(w, SPLAT_ERR_OOM, "deterministic sums: device allocation failed");
    }
    cap = need;
  }
  return zero_async(w, *buf, (size_t)w.V * w.G * nslot * 2 * sizeof(unsigned long long), st,
                    "deterministic sums clear");
}

template <typename T>
static int fix_to(Workspace& w, const unsigned long long* src, T* dst, int nslot,
                  cudaStream_t st) {
  const long long n = (long long)w.V * w.G * nslot;
  k_fixed_to<T><<<(unsigned)std::min<long long>((n + 255) / 256, 8 * 148), 256, 0, st>>>(
      src, dst, n);
  return check_launch(w, "fixed-point conversion kernel");
}

int launch_replay(Workspace& w, const float* obs, cudaStream_t st) {
  const int tok = prof_begin(w, st, SPLAT_K_REPLAY);
  int rc = SPLAT_OK;
  const bool det = w.det && w.G > 0;
  if (det) {
    rc = fix_buffer(w, &w.acc_fix, w.acc_fix_cap, kAccN, st);
  } else if (w.G > 0 && !w.acc_clean) {
    rc = zero_async(w, w.acc, (size_t)w.V * w.G * kAccN * sizeof(float), st, "accumulator clear");
  }
  w.acc_clean = false;
  if (!rc) {
    dim3 grid(w.nt * kCtaPerTile, w.V);
    if (det)
      k_replay_det<<<grid, kThreads, 0, st>>>(w.rec, w.sval, w.tile_off, w.tile_order, w.G, w.H,
                                              w.W, w.TX, w.nt, w.img, obs, w.last, w.umask,
                                              w.acc_fix);
    else
      k_replay<<<grid, kThreads, 0, st>>>(w.rec, w.sval, w.tile_off, w.tile_order, w.G, w.H, w.W,
                                          w.TX, w.nt, w.img, obs, w.last, w.ncon, w.umask,
                                          w.lmask, w.acc);
    rc = check_launch(w, "replay kernel");
  }
  if (!rc && det) rc = fix_to<float>(w, w.acc_fix, w.acc, kAccN, st);
  prof_end(w, st, tok);
  return rc;
}

// render and replay in one launch (default accumulation mode only; the deterministic mode runs
// launch_render and launch_replay)
int launch_render_replay(Workspace& w, const float* bg, const float* obs, float* img,
                         float* T_final, int* n_contrib, cudaStream_t st) {
  const int tok = prof_begin(w, st, SPLAT_K_RENDER_REPLAY);
  int rc = SPLAT_OK;
  if (w.G > 0 && !w.acc_clean)
    rc = zero_async(w, w.acc, (size_t)w.V * w.G * kAccN * sizeof(float), st, "accumulator clear");
  w.acc_clean = false;
  if (rc) {
    prof_end(w, st, tok);
    return rc;
  }
  dim3 grid(w.nt * kCtaPerTile, w.V);
  k_render<true><<<grid, kThreads, 0, st>>>(w.rec, w.sval, w.tile_off, w.tile_order, w.G, w.H,
                                            w.W, w.TX, w.nt, bg, img, T_final, n_contrib, w.last,
                                            w.umask, w.lmask, obs, w.acc);
  prof_end(w, st, tok);
  return check_launch(w, "render and replay kernel");
}

int launch_backward(Workspace& w, const float* obs, cudaStream_t st) {
  const int tok = prof_begin(w, st, SPLAT_K_BACKWARD);
  int rc = SPLAT_OK;
  const bool det = w.det && w.G > 0;
  if (det) {
    rc = fix_buffer(w, &w.accb_fix, w.accb_fix_cap, kAccBN, st);
  } else if (w.G > 0) {
    rc = zero_async(w, w.accb, (size_t)w.V * w.G * kAccBN * sizeof(double), st,
                    "backward sums clear");
  }
  if (!rc) {
    dim3 grid(w.nt * kCtaPerTile, w.V);
    if (det)
      k_backward<true><<<grid, kThreads, 0, st>>>(w.rec, w.sval, w.tile_off, w.tile_order, w.G, w.H, w.W, w.TX,
                                                  w.nt, w.img, w.Tfin, w.bg, obs, w.last,
                                                  w.umask, w.accb, w.accb_fix);
    else
      k_backward<false><<<grid, kThreads, 0, st>>>(w.rec, w.sval, w.tile_off, w.tile_order, w.G, w.H, w.W,
                                                   w.TX, w.nt, w.img, w.Tfin, w.bg, obs, w.last,
                                                   w.umask, w.accb, nullptr);
    rc = check_launch(w, "backward kernel");
  }
  if (!rc && det) rc = fix_to<double>(w, w.accb_fix, w.accb, kAccBN, st);
  prof_end(w, st, tok);
  return rc;
}

int launch_acc_to_double(Workspace& w, double* out, cudaStream_t st) {
  const long long n = (long long)w.V * w.G * kAccN;
  if (n == 0) return SPLAT_OK;
  k_widen<<<(unsigned)std::min<long long>((n + 255) / 256, 8 * 148), 256, 0, st>>>(w.acc, out, n);
  return check_launch(w, "accumulator copy kernel");
}

int launch_pair_count(Workspace& w, cudaStream_t st) {
  int rc = zero_async(w, w.d_scratch, sizeof(long long), st, "pair count clear");
  if (rc) return rc;
  const long long n = (long long)w.V * w.H * w.W;
  k_pair_sum<<<296, 256, 0, st>>>(w.last, n, w.d_scratch);
  return check_launch(w, "pair count kernel");
}

}  // namespace splat
