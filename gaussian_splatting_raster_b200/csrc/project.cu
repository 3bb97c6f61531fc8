// Stage 1 preprocess: EWA projection of every Gaussian into every view, tile rectangle,
// opacity and SH colour.
//
// Sources: "Research Proposal: Renderer Score Tokens for Recurrent Gaussian Splatting",
// "Two-Stage Algorithm" Stage 1 (standard gsplat render) and "Projected-Center Mean Partial
// Score" (G and Sigma2D); "ATSplat: Compact Feed-forward 3D Gaussian Splatting with Adaptive Token
// Expansion", prerequisites (the 3DGS primitive). The EWA details follow the standard 3DGS tile
// rasteriser: tangent clamp at 1.3x the half field of view inside the covariance Jacobian,
// 0.3 px^2 dilation, 3-sigma square footprint, near plane z = 0.01.
//
// One thread per Gaussian reads its parameters once (SH included) and writes one record per view:
// the SH coefficients, which dominate the input bytes at degree 3, are never re-read per view.
#include <algorithm>

#include "common.cuh"

namespace splat {
namespace {

constexpr int kProjThreads = 128;

__device__ __forceinline__ int clamp_tile(float val, int hi) {
  if (!(val > 0.0f)) return 0;  // NaN -> 0
  if (val > (float)hi) return hi;
  return (int)val;
}

template <int DEG>
__global__ void __launch_bounds__(kProjThreads)
k_project(const float* __restrict__ means, const float* __restrict__ lsc,
          const float* __restrict__ quats, const float* __restrict__ opac,
          const float* __restrict__ sh, const float* __restrict__ views_in, int G, int V, int H,
          int W, int TX, int TY, float4* __restrict__ rec, ushort4* __restrict__ rect,
          uint32_t* __restrict__ dkey, uint32_t* __restrict__ kbits, float4* __restrict__ acc,
          unsigned long long* __restrict__ ntot) {
  constexpr int D = (DEG + 1) * (DEG + 1);
  constexpr int NSH = D * 3;
  // shared memory: the block's SH coefficients [kProjThreads][NSH], the views [V][20], then per
  // view the tangent-clamp limits and the camera centre [V][5] (view constants, computed once)
  extern __shared__ float s_dyn[];
  constexpr int SP = NSH | 1;  // odd per-thread stride: conflict-free shared-memory reads
  float* s_sh = s_dyn;
  float* s_views = s_dyn + kProjThreads * SP;
  float* s_vc = s_views + V * 20;
  for (int i = threadIdx.x; i < V * 20; i += blockDim.x) s_views[i] = views_in[i];
  for (int v = threadIdx.x; v < V; v += blockDim.x) {
    const float* vw = views_in + 20 * v;
    s_vc[5 * v] = 1.3f * ((0.5f * (float)W) / vw[16]);
    s_vc[5 * v + 1] = 1.3f * ((0.5f * (float)H) / vw[17]);
    // camera centre -R^T t
    s_vc[5 * v + 2] = -(vw[0] * vw[3] + vw[4] * vw[7] + vw[8] * vw[11]);
    s_vc[5 * v + 3] = -(vw[1] * vw[3] + vw[5] * vw[7] + vw[9] * vw[11]);
    s_vc[5 * v + 4] = -(vw[2] * vw[3] + vw[6] * vw[7] + vw[10] * vw[11]);
  }
  // coalesced staging of the block's contiguous SH rows (they dominate the input bytes)
  {
    const long long g0 = (long long)blockIdx.x * kProjThreads;
    const int ng = (int)min((long long)kProjThreads, (long long)G - g0);
    const int nf = ng * NSH;
    const float* src = sh + g0 * NSH;
    if ((((uintptr_t)src) & 15) == 0) {
      const float4* s4 = reinterpret_cast<const float4*>(src);
      for (int k = threadIdx.x; k < nf / 4; k += blockDim.x) {
        const float4 f = s4[k];
        const float e[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int L = 4 * k + c, t = L / NSH;
          s_sh[t * SP + (L - t * NSH)] = e[c];
        }
      }
      for (int L = (nf / 4) * 4 + threadIdx.x; L < nf; L += blockDim.x) {
        const int t = L / NSH;
        s_sh[t * SP + (L - t * NSH)] = src[L];
      }
    } else {
      for (int L = threadIdx.x; L < nf; L += blockDim.x) {
        const int t = L / NSH;
        s_sh[t * SP + (L - t * NSH)] = src[L];
      }
    }
  }
  __syncthreads();
  const int g = blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= G) return;

  const float m0 = means[3 * g], m1 = means[3 * g + 1], m2 = means[3 * g + 2];
  const float l0 = lsc[3 * g], l1 = lsc[3 * g + 1], l2 = lsc[3 * g + 2];
  const float q0 = quats[4 * g], q1 = quats[4 * g + 1], q2 = quats[4 * g + 2],
              q3 = quats[4 * g + 3];
  const float a_logit = opac[g];
  const float* shc = s_sh + threadIdx.x * SP;

  bool ok = isfinite(m0) && isfinite(m1) && isfinite(m2) && isfinite(l0) && isfinite(l1) &&
            isfinite(l2) && isfinite(q0) && isfinite(q1) && isfinite(q2) && isfinite(q3) &&
            isfinite(a_logit);

  // view-independent part: rotation, scales, Sigma3D, opacity
  float Sw[3][3];
  float o = 0.0f;
  {
    const float n2 = q0 * q0 + q1 * q1 + q2 * q2 + q3 * q3;
    if (!(n2 > 0.0f)) ok = false;
    const float inv = 1.0f / sqrtf(n2);
    const float qw = q0 * inv, qx = q1 * inv, qy = q2 * inv, qz = q3 * inv;
    float Rq[3][3];
    Rq[0][0] = 1.0f - 2.0f * (qy * qy + qz * qz);
    Rq[0][1] = 2.0f * (qx * qy - qw * qz);
    Rq[0][2] = 2.0f * (qx * qz + qw * qy);
    Rq[1][0] = 2.0f * (qx * qy + qw * qz);
    Rq[1][1] = 1.0f - 2.0f * (qx * qx + qz * qz);
    Rq[1][2] = 2.0f * (qy * qz - qw * qx);
    Rq[2][0] = 2.0f * (qx * qz - qw * qy);
    Rq[2][1] = 2.0f * (qy * qz + qw * qx);
    Rq[2][2] = 1.0f - 2.0f * (qx * qx + qy * qy);
    const float S[3] = {exp_cw(l0), exp_cw(l1), exp_cw(l2)};
    float M[3][3];
#pragma unroll
    for (int i = 0; i < 3; ++i)
#pragma unroll
      for (int j = 0; j < 3; ++j) M[i][j] = Rq[i][j] * S[j];
#pragma unroll
    for (int i = 0; i < 3; ++i)
#pragma unroll
      for (int j = 0; j < 3; ++j) Sw[i][j] = M[i][0] * M[j][0] + M[i][1] * M[j][1] + M[i][2] * M[j][2];
    o = 1.0f / (1.0f + exp_cw(-a_logit));
  }
  // the render's early-skip bound: exponents below it give alpha < 1/255 (per Gaussian)
  const float cut = logf((1.0f / 255.0f) / o) - 1e-3f;

  for (int v = 0; v < V; ++v) {
    const size_t i = (size_t)v * G + g;
    const float* vw = s_views + 20 * v;
    float4 r0 = make_float4(0, 0, 0, 0), r1 = r0, r2 = r0, r3 = r0;
    ushort4 rc = make_ushort4(0, 0, 0, 0);
    int cnt = 0;
    bool vis = ok;
    float Rv[3][3], t[3];
#pragma unroll
    for (int a = 0; a < 3; ++a) {
#pragma unroll
      for (int b = 0; b < 3; ++b) Rv[a][b] = vw[4 * a + b];
      t[a] = vw[4 * a + 3];
    }
    const float fx = vw[16], fy = vw[17], cx = vw[18], cy = vw[19];
    const float x = Rv[0][0] * m0 + Rv[0][1] * m1 + Rv[0][2] * m2 + t[0];
    const float y = Rv[1][0] * m0 + Rv[1][1] * m1 + Rv[1][2] * m2 + t[1];
    const float z = Rv[2][0] * m0 + Rv[2][1] * m1 + Rv[2][2] * m2 + t[2];
    if (!(z > 0.01f)) vis = false;
    if (vis) {
      float T1[3][3], Sc[3][3];
#pragma unroll
      for (int a = 0; a < 3; ++a)
#pragma unroll
        for (int b = 0; b < 3; ++b) T1[a][b] = Rv[a][0] * Sw[0][b] + Rv[a][1] * Sw[1][b] + Rv[a][2] * Sw[2][b];
#pragma unroll
      for (int a = 0; a < 3; ++a)
#pragma unroll
        for (int b = 0; b < 3; ++b) Sc[a][b] = T1[a][0] * Rv[b][0] + T1[a][1] * Rv[b][1] + T1[a][2] * Rv[b][2];
      const float u = x / z, vv = y / z;
      const float limx = s_vc[5 * v], limy = s_vc[5 * v + 1];
      const float uc = fminf(limx, fmaxf(-limx, u));
      const float vc = fminf(limy, fmaxf(-limy, vv));
      const float J00 = fx / z, J02 = -(fx * uc) / z;
      const float J11 = fy / z, J12 = -(fy * vc) / z;
      float T0[3], Tr1[3];
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        T0[k] = J00 * Sc[0][k] + J02 * Sc[2][k];
        Tr1[k] = J11 * Sc[1][k] + J12 * Sc[2][k];
      }
      float ca = T0[0] * J00 + T0[2] * J02;
      const float cb = T0[1] * J11 + T0[2] * J12;
      float cc = Tr1[1] * J11 + Tr1[2] * J12;
      ca = ca + 0.3f;
      cc = cc + 0.3f;
      const float det = ca * cc - cb * cb;
      if (!(det > 0.0f)) vis = false;
      const float qa = cc / det, qb = -cb / det, qc = ca / det;
      const float mid = 0.5f * (ca + cc);
      const float lam = mid + sqrtf(fmaxf(0.1f, mid * mid - det));
      const float rr = ceilf(3.0f * sqrtf(lam));
      if (!(rr > 0.0f)) vis = false;
      const float mx = fx * u + cx, my = fy * vv + cy;
      const int x0 = clamp_tile(floorf((mx - rr) / 16.0f), TX);
      const int x1 = clamp_tile(floorf((mx + rr) / 16.0f) + 1.0f, TX);
      const int y0 = clamp_tile(floorf((my - rr) / 16.0f), TY);
      const int y1 = clamp_tile(floorf((my + rr) / 16.0f) + 1.0f, TY);
      if (x1 <= x0 || y1 <= y0) vis = false;
      if (vis) {
        // view direction (world) from the camera centre; the SH colour only has to agree with
        // the oracle's to a few ulp, so one reciprocal square root instead of three divisions
        const float d0 = m0 - s_vc[5 * v + 2], d1 = m1 - s_vc[5 * v + 3], d2 = m2 - s_vc[5 * v + 4];
        const float il = rsqrtf(d0 * d0 + d1 * d1 + d2 * d2);
        const float dx = d0 * il, dy = d1 * il, dz = d2 * il;
        float B[16];
        sh_poly<DEG>(dx, dy, dz, B);
        float col[3];
        int flags = kFlagVisible;
#pragma unroll
        for (int ch = 0; ch < 3; ++ch) {
          float s = 0.0f;
#pragma unroll
          for (int k = 0; k < D; ++k) s = s + B[k] * shc[3 * k + ch];
          s = s + 0.5f;
          if (s > 0.0f) flags |= 1 << ch;
          col[ch] = fmaxf(s, 0.0f);
        }
        // the render's early-skip bound and the half-extents of the ellipse {exponent >= cut}
        // (bounding box of every pixel centre that can reach alpha >= 1/255), widened by
        // 1 % + 0.05 px -- far more than fp32 rounding of the exponent (or of det Q when
        // det Q > 1e-4 qa qc) can move its boundary; nearly singular conics get an unbounded box
        float ex = -1.0f, ey = -1.0f;
        if (cut < 0.0f) {
          const float dq = qa * qc - qb * qb;
          if (dq > 1e-4f * (qa * qc)) {
            // a cull bound, not a decision: fast reciprocal and square root (relative errors of a
            // few 1e-7, far inside the 1 % widening)
            // (the radicands are > 0 here; clamped so that an overflow to +inf stays unbounded
            // instead of turning into inf * 0)
            const float r2c = -2.0f * cut, idq = __fdividef(1.0f, dq);
            const float sx = fminf(r2c * qc * idq, 1e30f), sy = fminf(r2c * qa * idq, 1e30f);
            ex = sx * rsqrtf(sx) * 1.01f + 0.05f;
            ey = sy * rsqrtf(sy) * 1.01f + 0.05f;
          } else {
            ex = ey = __int_as_float(0x7f800000);
          }
        }
        r0 = make_float4(mx, my, col[0], col[1]);
        r1 = make_float4(col[2], cut, ex, ey);
        r2 = make_float4(qa, qb, qc, o);
        r3 = make_float4(z, x, y, __int_as_float(flags));
        rc = make_ushort4((unsigned short)x0, (unsigned short)y0, (unsigned short)x1,
                          (unsigned short)y1);
        cnt = (x1 - x0) * (y1 - y0);
      }
    }
    float4* rl = rec + rec_lo(i);
    float4* rh = rec + rec_hi(i);
    rl[0] = r0;
    rl[1] = r1;
    rh[0] = r2;
    rh[1] = r3;
    rect[i] = rc;
    // the score replay's (view, Gaussian) sums start from zero: cleared here, where every row is
    // written anyway, instead of by a separate pass over 32 B per (view, Gaussian)
    acc[2 * i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    acc[2 * i + 1] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    // depth sort key (fp32 bits of z > 0 order like the values; culled entries sort last) and,
    // per view, the largest visible key and the largest complement of one (the complement of the
    // smallest visible key): the sort orders key - smallest, over the bits of the key range
    const uint32_t key = cnt > 0 ? __float_as_uint(z) : 0xffffffffu;
    dkey[i] = key;
    const unsigned lanes = __activemask();
    const uint32_t khi = __reduce_max_sync(lanes, cnt > 0 ? key : 0u);
    const uint32_t klo = __reduce_max_sync(lanes, cnt > 0 ? ~key : 0u);
    const unsigned int ntile = __reduce_add_sync(lanes, (unsigned int)cnt);
    if ((threadIdx.x & 31) == __ffs(lanes) - 1 && khi) {
      // one of kKeyStripes copies per view, chosen by block, keeps same-address atomics rare;
      // the stripes are folded later (maxima of the key statistics, sum of the instance counts)
      const int stripe = v * kKeyStripes + (blockIdx.x & (kKeyStripes - 1));
      uint32_t* kb = kbits + 2 * stripe;
      atomicMax(kb, khi);
      atomicMax(kb + 1, klo);
      atomicAdd(ntot + stripe, (unsigned long long)ntile);
    }
  }
}

}  // namespace

int launch_project(Workspace& w, const float* means, const float* lsc, const float* quats,
                   const float* opac, const float* sh, cudaStream_t st) {
  int rc = zero_async(w, w.kbits, (size_t)2 * kKeyStripes * w.V * sizeof(uint32_t), st,
                      "key statistics clear");
  if (!rc)
    rc = zero_async(w, w.ntot, (size_t)kKeyStripes * w.V * sizeof(unsigned long long), st,
                    "instance counts clear");
  if (rc) return rc;
  if (w.G == 0) return SPLAT_OK;
  const int blocks = (w.G + kProjThreads - 1) / kProjThreads;
  const int tok = prof_begin(w, st, SPLAT_K_PROJECT);
#define SPLAT_PROJ(DEG)                                                                          \
  {                                                                                              \
    const size_t smem = ((size_t)kProjThreads * ((3 * (DEG + 1) * (DEG + 1)) | 1) + (size_t)w.V * 25) * \
                        sizeof(float);                                                           \
    if (smem > 48 * 1024 &&                                                                      \
        cudaFuncSetAttribute(k_project<DEG>, cudaFuncAttributeMaxDynamicSharedMemorySize,       \
                             (int)smem) != cudaSuccess)                                          \
      return set_err(w, SPLAT_ERR_CAPACITY, "too many views for the projection kernel");        \
    k_project<DEG><<<blocks, kProjThreads, smem, st>>>(means, lsc, quats, opac, sh, w.views,     \
                                                       w.G, w.V, w.H, w.W, w.TX, w.TY, w.rec,    \
                                                       w.rect, w.dkey, w.kbits,                  \
                                                       reinterpret_cast<float4*>(w.acc),         \
                                                       w.ntot);                                  \
  }
  switch (w.deg) {
    case 0: SPLAT_PROJ(0); break;
    case 1: SPLAT_PROJ(1); break;
    case 2: SPLAT_PROJ(2); break;
    default: SPLAT_PROJ(3); break;
  }
#undef SPLAT_PROJ
  prof_end(w, st, tok);
  const int rc2 = check_launch(w, "project kernel");
  w.acc_clean = rc2 == SPLAT_OK;
  return rc2;
}

// the records in the order splat_copy_projection documents: mx, my, a, b, c, o, colour r, g, b,
// cut, ex, ey, z, x_c, y_c, flags
__global__ void k_copy_records(const float4* __restrict__ rec, float4* __restrict__ out, long long n) {
  for (long long k = (long long)blockIdx.x * blockDim.x + threadIdx.x; k < n;
       k += (long long)gridDim.x * blockDim.x) {
    const float4 r0 = rec[rec_lo(k)], r1 = rec[rec_lo(k) + 1];
    const float4 r2 = rec[rec_hi(k)], r3 = rec[rec_hi(k) + 1];
    out[4 * k] = make_float4(r0.x, r0.y, r2.x, r2.y);
    out[4 * k + 1] = make_float4(r2.z, r2.w, r0.z, r0.w);
    out[4 * k + 2] = r1;
    out[4 * k + 3] = r3;
  }
}

// the tile rectangles widened to the documented int32 [V, G, 4]
__global__ void k_copy_rects(const ushort4* __restrict__ rect, int4* __restrict__ out, long long n) {
  for (long long k = (long long)blockIdx.x * blockDim.x + threadIdx.x; k < n;
       k += (long long)gridDim.x * blockDim.x) {
    const ushort4 r = rect[k];
    out[k] = make_int4(r.x, r.y, r.z, r.w);
  }
}

int launch_copy_records(Workspace& w, float* out, cudaStream_t st) {
  const long long n = (long long)w.V * w.G;
  if (n == 0) return SPLAT_OK;
  k_copy_records<<<(unsigned)std::min<long long>((n + 255) / 256, 8 * 148), 256, 0, st>>>(
      w.rec, reinterpret_cast<float4*>(out), n);
  return check_launch(w, "record copy kernel");
}

int launch_copy_rects(Workspace& w, int* out, cudaStream_t st) {
  const long long n = (long long)w.V * w.G;
  if (n == 0) return SPLAT_OK;
  k_copy_rects<<<(unsigned)std::min<long long>((n + 255) / 256, 8 * 148), 256, 0, st>>>(
      w.rect, reinterpret_cast<int4*>(out), n);
  return check_launch(w, "rectangle copy kernel");
}

}  // namespace splat
