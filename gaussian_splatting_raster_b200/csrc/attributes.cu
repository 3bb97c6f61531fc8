// Attribute compositing and its transpose, over the entries the last render composited.
//
// Sources: "ReCoSplat" section 2.1 (learned feature channels rendered beside RGB), "ATSplat",
// core method (a per-Gaussian uncertainty score rendered as a scalar attribute by alpha
// compositing), "L2D2-GS" method (a 2D gain back-projected to Gaussians through the rasteriser's
// mask channel), "Research Proposal: Renderer Score Tokens for Recurrent Gaussian Splatting",
// "Novelty Boundary" and Block 3 (alphaT scatter and PRIMU-style scalar error/coverage).
//
//   attribute render   F_p = sum_i w_i f_{g_i}            [V, H, W, C]
//   scatter            s_g = sum_v sum_p w_pgv m_p        [G, C]   (the render's adjoint)
//   attribution        [sum w, sum w |r|, sum w |r| / (sum w + 1e-6)] per Gaussian, r = C_hat - C_obs
// with w = T alpha of the composited entries (the render's decisions; no background term).
//
// Same traversal as the score replay (kCtaPerTile CTAs per (tile, view)); each warp walks the list for its
// 8x4 pixel block on its own in 32-entry chunks, staging only the entries the render marked as
// composited by some pixel of the warp. The attribute render keeps up to 16 channels per pixel in
// registers (more channels take further passes); the scatter reduces each entry's per-pixel
// values over the warp (transpose-reduction) and adds them with fp64 atomics into a workspace
// buffer that a last kernel rounds to fp32.
#include "traverse.cuh"

namespace splat {

SPLAT_BOUNDS_WORD(bounds_word_attributes)

namespace {

constexpr int kMaxPass = 16;  // channels per traversal

// F[c0 .. c0 + CB) of every pixel. Each lane walks only the entries its pixel composited (the
// render's per-pixel masks, as in the score replay), in list order, so a warp runs its longest
// walk instead of every entry some pixel of its block composited; every pixel's output is its own
// (no reduction), and the sum is the same as over the render's order.
template <int CB>
__global__ void __launch_bounds__(kThreads)
k_features(const float4* __restrict__ rec, const uint32_t* __restrict__ ids,
           const long long* __restrict__ tile_off, const int* __restrict__ order,
           int G, int H, int W, int TX, int nt,
           const int* __restrict__ last, const uint32_t* __restrict__ lmask,
           const float* __restrict__ feats, int C, int c0, float* __restrict__ out) {
  int t, v;
  if (!block_tile(order, nt, &g_bounds_word, t, v)) return;
  const int tx = t % TX, ty = t / TX;
  int i, j, bx, by;
  tile_pixel(tx, ty, i, j, bx, by);
  if (i >= W || j >= H) return;  // no warp-wide operation below
  const long long s = tile_off[(size_t)v * (nt + 1) + t];
  const int gt = v * nt + t;
  const int lane = threadIdx.x & 31, twarp = tile_warp();
  const int nc = min(CB, C - c0);
  const float px = (float)i + 0.5f, py = (float)j + 0.5f;
  const size_t p = ((size_t)v * H + j) * W + i;
  const int cend = (last[p] + 31) >> 5;  // chunks holding this pixel's composited entries
  const size_t vG = (size_t)v * G;
  float F[CB];
#pragma unroll
  for (int k = 0; k < CB; ++k) F[k] = 0.0f;
  float T = 1.0f;
  if (cend > 0) {
    const uint4* lm =
        reinterpret_cast<const uint4*>(lmask + lmask_region(s, gt)) + (twarp * 32 + lane);
    const uint4 g0 = __ldg(lm);
    uint32_t m = g0.x, n1 = g0.y, n2 = g0.z, n3 = g0.w;
    uint4 pre = make_uint4(0u, 0u, 0u, 0u);
    if (4 < cend) pre = __ldg(lm + 256);
    int c = 0;
    for (;;) {
      if (!m) {  // next chunk with an entry of this pixel
        if (++c >= cend) break;
        if ((c & 3) == 0) {
          m = pre.x;
          n1 = pre.y;
          n2 = pre.z;
          n3 = pre.w;
          if (c + 4 < cend) pre = __ldg(lm + (size_t)((c >> 2) + 1) * 256);
        } else {
          m = n1;
          n1 = n2;
          n2 = n3;
        }
        continue;
      }
      const int q = __ffs(m) - 1;
      m &= m - 1u;
      const uint32_t g = ids[s + 32LL * c + q];
      if (!in_bounds(g, (unsigned)G, &g_bounds_word)) continue;
      const float4* rl = rec + rec_lo(vG + g);  // r0, r1
      const float4* rh = rec + rec_hi(vG + g);  // r2, r3
      float4 A, Bq;
      entry_operands(__ldg(rl), __ldg(rh), A, Bq);
      const Entry E = eval_entry(A, Bq, -INFINITY, px, py);  // the render's alpha, bit for bit
      if (!E.use) continue;
      const float w = E.alpha * T;
      const float* fg = feats + (size_t)g * C + c0;
#pragma unroll
      for (int k = 0; k < CB; ++k)
        if (k < nc) F[k] = F[k] + w * __ldg(fg + k);
      T = T * (1.0f - E.alpha);
    }
  }
#pragma unroll
  for (int k = 0; k < CB; ++k)
    if (k < nc) out[p * C + c0 + k] = F[k];
}

// sum over pixels of w m[c0 .. c0 + NV) per (Gaussian), into acc [G, C] (fp64). RESID: the map is
// (1, |C_hat - C_obs|) computed here from img and obs (C = 2).
template <int NV, bool RESID>
__global__ void __launch_bounds__(kThreads)
k_scatter(const float4* __restrict__ rec, const uint32_t* __restrict__ ids,
          const long long* __restrict__ tile_off, const int* __restrict__ order,
          int G, int H, int W, int TX, int nt,
          const int* __restrict__ last, const uint32_t* __restrict__ umask,
          const float* __restrict__ map, const float* __restrict__ img,
          const float* __restrict__ obs, int C, int c0, double* __restrict__ acc) {
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
  __shared__ float s_cut[kThreads];
  __shared__ uint32_t s_g[kThreads];
  float4* wa = s_a + warp * 32;
  float4* wb = s_b + warp * 32;
  float* wc = s_cut + warp * 32;
  uint32_t* wg = s_g + warp * 32;
  const int nc = min(NV, C - c0);
  const float px = (float)i + 0.5f, py = (float)j + 0.5f;
  const size_t p = ((size_t)v * H + j) * W + i;
  int lst = 0;
  float m[NV];
#pragma unroll
  for (int k = 0; k < NV; ++k) m[k] = 0.0f;
  if (inside) {
    lst = last[p];
    if constexpr (RESID) {
      const float r0 = img[3 * p] - obs[3 * p], r1 = img[3 * p + 1] - obs[3 * p + 1],
                  r2 = img[3 * p + 2] - obs[3 * p + 2];
      m[0] = 1.0f;
      m[1] = sqrtf(r0 * r0 + r1 * r1 + r2 * r2);
    } else {
#pragma unroll
      for (int k = 0; k < NV; ++k)
        if (k < nc) m[k] = map[p * C + c0 + k];
    }
  }
  const int wmax = __reduce_max_sync(0xffffffffu, lst);
  const size_t vG = (size_t)v * G;
  const int slot = slot_of<NV>(lane);
  const bool holder = slot_holder<NV>(lane) && slot < nc;
  float T = 1.0f;
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
        wa[lane] = rl[0];
        wb[lane] = rh[0];
        wc[lane] = reinterpret_cast<const float*>(rl + 1)[1];  // cut
        wg[lane] = g;
      }
    }
    if (kChecked) bits &= ~__ballot_sync(0xffffffffu, bad);
    __syncwarp();
    while (bits) {
      const int q = __ffs(bits) - 1;
      bits &= bits - 1;
      float x[NV];
#pragma unroll
      for (int k = 0; k < NV; ++k) x[k] = 0.0f;
      bool used = false;
      if (base + q < lst) {
        float4 A, Bq;
        entry_operands(wa[q], wb[q], A, Bq);
        const Entry E = eval_entry(A, Bq, wc[q], px, py);
        if (E.use) {
          used = true;
          const float w = E.alpha * T;
#pragma unroll
          for (int k = 0; k < NV; ++k) x[k] = w * m[k];
          T = T * (1.0f - E.alpha);
        }
      }
      if (__any_sync(0xffffffffu, used)) {
        slot_reduce<NV>(x, lane);
        if (holder && x[0] != 0.0f) atomicAdd(acc + (size_t)wg[q] * C + c0 + slot, (double)x[0]);
      }
    }
    __syncwarp();
  }
}

// fp64 sums -> fp32 output; ATTR: [sum w, sum w |r|] -> [sum w, sum w |r|, sum w |r| / (sum w + 1e-6)]
template <bool ATTR>
__global__ void k_scatter_out(const double* __restrict__ acc, long long G, int C,
                              float* __restrict__ out) {
  for (long long k = (long long)blockIdx.x * blockDim.x + threadIdx.x; k < G * (ATTR ? 3 : C);
       k += (long long)gridDim.x * blockDim.x) {
    if constexpr (ATTR) {
      const long long g = k / 3;
      const int c = (int)(k - g * 3);
      const double cov = acc[2 * g], err = acc[2 * g + 1];
      out[k] = (float)(c == 0 ? cov : (c == 1 ? err : err / (cov + 1e-6)));
    } else {
      out[k] = (float)acc[k];
    }
  }
}

int grow_scratch(Workspace& w, size_t n) {
  if (n <= w.sacc_cap) return SPLAT_OK;
  if (w.sacc) cudaFree(w.sacc);
  w.sacc = nullptr;
  w.sacc_cap = 0;
  cudaError_t e = cudaMalloc(&w.sacc, n * sizeof(double));
  if (e != cudaSuccess) {
    w.sacc = nullptr;
    return set_err(w, SPLAT_ERR_OOM, "scatter sums: device allocation failed");
  }
  w.sacc_cap = n;
  return SPLAT_OK;
}

}  // namespace

int launch_features(Workspace& w, const float* feats, int C, float* out, cudaStream_t st) {
  const int tok = prof_begin(w, st, SPLAT_K_FEATURES);
  dim3 grid(w.nt * kCtaPerTile, w.V);
  for (int c0 = 0; c0 < C; c0 += kMaxPass) {
    const int nc = C - c0 < kMaxPass ? C - c0 : kMaxPass;
#define SPLAT_FEAT(CB)                                                                          \
  k_features<CB><<<grid, kThreads, 0, st>>>(w.rec, w.sval, w.tile_off, w.tile_order, w.G, w.H, w.W, w.TX,    \
                                           w.nt, w.last, w.lmask, feats, C, c0, out)
    if (nc == 1) SPLAT_FEAT(1);
    else if (nc <= 4) SPLAT_FEAT(4);
    else if (nc <= 8) SPLAT_FEAT(8);
    else SPLAT_FEAT(16);
#undef SPLAT_FEAT
    const int rc = check_launch(w, "attribute render kernel");
    if (rc) {
      prof_end(w, st, tok);
      return rc;
    }
  }
  prof_end(w, st, tok);
  return SPLAT_OK;
}

int launch_scatter(Workspace& w, const float* map, const float* obs, int C, float* out,
                   cudaStream_t st) {
  const bool attr = map == nullptr;  // attribution: map = (1, |r|) from the render and obs
  if (attr) C = 2;
  int rc;
  if ((rc = grow_scratch(w, (size_t)w.G * C))) return rc;
  if ((rc = zero_async(w, w.sacc, (size_t)w.G * C * sizeof(double), st, "scatter sums clear")))
    return rc;
  const int tok = prof_begin(w, st, SPLAT_K_SCATTER);
  struct EndTok {  // closes the timing bracket on every return path
    Workspace& w;
    cudaStream_t st;
    int tok;
    ~EndTok() { prof_end(w, st, tok); }
  } end_tok{w, st, tok};
  dim3 grid(w.nt * kCtaPerTile, w.V);
  if (attr) {
    k_scatter<2, true><<<grid, kThreads, 0, st>>>(w.rec, w.sval, w.tile_off, w.tile_order, w.G, w.H, w.W, w.TX,
                                                  w.nt, w.last, w.umask, nullptr, w.img, obs, 2,
                                                  0, w.sacc);
    if ((rc = check_launch(w, "attribution kernel"))) return rc;
  } else {
    for (int c0 = 0; c0 < C; c0 += kMaxPass) {
      const int nc = C - c0 < kMaxPass ? C - c0 : kMaxPass;
#define SPLAT_SCAT(NV)                                                                          \
  k_scatter<NV, false><<<grid, kThreads, 0, st>>>(w.rec, w.sval, w.tile_off, w.tile_order, w.G, w.H, w.W,    \
                                                  w.TX, w.nt, w.last, w.umask, map, nullptr,   \
                                                  nullptr, C, c0, w.sacc)
      if (nc == 1) SPLAT_SCAT(1);
      else if (nc == 2) SPLAT_SCAT(2);
      else if (nc <= 4) SPLAT_SCAT(4);
      else if (nc <= 8) SPLAT_SCAT(8);
      else SPLAT_SCAT(16);
#undef SPLAT_SCAT
      if ((rc = check_launch(w, "scatter kernel"))) return rc;
    }
  }
  const long long n = (long long)w.G * (attr ? 3 : C);
  const int blocks = (int)((n + 255) / 256 < 4 * 148 ? (n + 255) / 256 : 4 * 148);
  if (n > 0) {
    if (attr) k_scatter_out<true><<<blocks, 256, 0, st>>>(w.sacc, w.G, 2, out);
    else k_scatter_out<false><<<blocks, 256, 0, st>>>(w.sacc, w.G, C, out);
    if ((rc = check_launch(w, "scatter output kernel"))) return rc;
  }
  return SPLAT_OK;
}

}  // namespace splat
