// Renderer backward, per-Gaussian part: the chain from the per-(view, Gaussian) sums of the
// backward traversal (raster.cu) to the derivatives of L = 1/2 sum |C_hat - C_obs|^2 with respect
// to every parameter, and the comparator variants.
//
// Source: "Research Proposal: Renderer Score Tokens for Recurrent Gaussian Splatting",
// "Relation to Gradient" (raw, detached, support-normalised and parameter-scale-normalised
// gradients as the comparators of the score tokens) and "Exact Score Operators" (RGB squared loss;
// the stop-gradient list of the projected-centre score -- projected covariance, view direction,
// order, clamp decisions -- which defines the detached variant; q_g = eps + sum_v q_gv). The
// forward being differentiated is the 3DGS EWA projection of "original gsplat" (Stage 1).
//
// One thread per Gaussian, views in a loop. Per visible view (fp64 from the fp32 record and the
// ten sums q, w r (3), h, h d (2), h (dx^2, dx dy, dy^2)):
//   opacity logit  (1 - o) h                       colour  dL/dc = w r where the clamp is inactive
//   SH             B(dir) (x) dL/dc                view direction  sum_k <dL/dc, sh_k> grad B_k
//   centre         dL/dmu2D = Q sum h d            conic  dL/dQ = -1/2 [[Hxx, Hxy], [Hxy, Hyy]]
//   covariance     dL/dSigma2D = -Q (dL/dQ) Q      Sigma2D = J Sc J^T + 0.3 I:
//                  dL/dSc = J^T (dL/dSigma2D) J,  dL/dJ = 2 (dL/dSigma2D) J Sc
//   camera point   through mu2D(x_c) and J(x_c) (the clamped tangent's derivative is zero),
//   world          dL/dmu += R_v^T dL/dx_c,  dL/dSigma3D += R_v^T (dL/dSc) R_v,
// and after the loop Sigma3D = M M^T, M = Rq diag(exp(log_scale)), Rq from q / |q|.
// The SH coefficients are staged in shared memory (columns per thread, conflict-free) and the SH
// gradient block is accumulated in fp32 directly in the shared-memory output tile, which is
// written out with coalesced stores once per requested variant.
#include "common.cuh"

namespace splat {
namespace {

constexpr int kGradThreads = 128;
constexpr int kP = kGradThreads + 1;  // padded column stride of the shared-memory tiles

// gradient of the real SH basis function k (Cartesian polynomial form of sh_poly) at (x, y, z);
// only its component tangent to the sphere is used by the caller
__device__ __forceinline__ void sh_dB(int k, double x, double y, double z, double g[3]) {
  const double c1 = 0.48860251190291992, c2a = 1.0925484305920792, c2b = 0.31539156525252005,
               c2c = 0.54627421529603959, c3a = 0.59004358992664352, c3b = 2.8906114426405538,
               c3c = 0.45704579946446572, c3d = 0.37317633259011540, c3e = 1.4453057213202769;
  const double xx = x * x, yy = y * y, zz = z * z;
  switch (k) {
    case 1: g[0] = 0.0; g[1] = -c1; g[2] = 0.0; break;
    case 2: g[0] = 0.0; g[1] = 0.0; g[2] = c1; break;
    case 3: g[0] = -c1; g[1] = 0.0; g[2] = 0.0; break;
    case 4: g[0] = c2a * y; g[1] = c2a * x; g[2] = 0.0; break;
    case 5: g[0] = 0.0; g[1] = -c2a * z; g[2] = -c2a * y; break;
    case 6: g[0] = -2.0 * c2b * x; g[1] = -2.0 * c2b * y; g[2] = 4.0 * c2b * z; break;
    case 7: g[0] = -c2a * z; g[1] = 0.0; g[2] = -c2a * x; break;
    case 8: g[0] = 2.0 * c2c * x; g[1] = -2.0 * c2c * y; g[2] = 0.0; break;
    case 9: g[0] = -6.0 * c3a * x * y; g[1] = -3.0 * c3a * (xx - yy); g[2] = 0.0; break;
    case 10: g[0] = c3b * y * z; g[1] = c3b * x * z; g[2] = c3b * x * y; break;
    case 11:
      g[0] = 2.0 * c3c * x * y; g[1] = -c3c * (4.0 * zz - xx - 3.0 * yy); g[2] = -8.0 * c3c * y * z;
      break;
    case 12:
      g[0] = -6.0 * c3d * x * z; g[1] = -6.0 * c3d * y * z; g[2] = c3d * (6.0 * zz - 3.0 * xx - 3.0 * yy);
      break;
    case 13:
      g[0] = -c3c * (4.0 * zz - 3.0 * xx - yy); g[1] = 2.0 * c3c * x * y; g[2] = -8.0 * c3c * x * z;
      break;
    case 14: g[0] = 2.0 * c3e * x * z; g[1] = -2.0 * c3e * y * z; g[2] = c3e * (xx - yy); break;
    case 15: g[0] = -3.0 * c3a * (xx - yy); g[1] = 6.0 * c3a * x * y; g[2] = 0.0; break;
    default: g[0] = 0.0; g[1] = 0.0; g[2] = 0.0; break;
  }
}

template <int DEG>
__global__ void __launch_bounds__(kGradThreads, 3)
k_grad(const float4* __restrict__ rec, const double* __restrict__ accb,
       const float* __restrict__ views, const float* __restrict__ lsc,
       const float* __restrict__ quats, const float* __restrict__ sh, int G, int V, int H, int W,
       float* __restrict__ out_raw, float* __restrict__ out_det, float* __restrict__ out_sup,
       float* __restrict__ out_psc) {
  constexpr int D = (DEG + 1) * (DEG + 1);
  constexpr int K = 11 + 3 * D;
  extern __shared__ float smem[];
  float* s_sh = smem;                // [3D][kP] SH coefficients, column per Gaussian
  float* s_out = s_sh + 3 * D * kP;  // [K][kP] raw gradient rows
  float* s_det = s_out + K * kP;     // [3][kP] detached mean block
  float* s_fac = s_det + 3 * kP;     // [2][kP] 1 / q_g, exp(mean log-scale)
  const int g0 = blockIdx.x * kGradThreads;
  const int ng = min(kGradThreads, G - g0);
  const int g = g0 + threadIdx.x;
  {
    const float* src = sh + (size_t)g0 * 3 * D;
    for (int L = threadIdx.x; L < ng * 3 * D; L += kGradThreads) {
      const int row = L / (3 * D), c = L - row * 3 * D;
      s_sh[c * kP + row] = src[L];
    }
  }
  float* col = s_out + threadIdx.x;
  const float* shc = s_sh + threadIdx.x;
#pragma unroll
  for (int k = 0; k < 3 * D; ++k) col[(11 + k) * kP] = 0.0f;
  __syncthreads();
  if (g < G) {
    const double eps = 1e-6;
    double qg = eps, glogit = 0.0;
    double gmu[3] = {0.0, 0.0, 0.0}, gdet[3] = {0.0, 0.0, 0.0};
    double dS[6] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0};  // dL/dSigma3D, symmetric: 00 01 02 11 12 22
    // Sigma3D (double, from the fp32 parameters)
    double Sg[6];
    {
      const float4 q4 = reinterpret_cast<const float4*>(quats)[g];
      const double qn = sqrt((double)q4.x * q4.x + (double)q4.y * q4.y + (double)q4.z * q4.z +
                             (double)q4.w * q4.w);
      const double w = q4.x / qn, x = q4.y / qn, y = q4.z / qn, z = q4.w / qn;
      const double R[3][3] = {{1 - 2 * (y * y + z * z), 2 * (x * y - w * z), 2 * (x * z + w * y)},
                              {2 * (x * y + w * z), 1 - 2 * (x * x + z * z), 2 * (y * z - w * x)},
                              {2 * (x * z - w * y), 2 * (y * z + w * x), 1 - 2 * (x * x + y * y)}};
      const double s0 = exp((double)lsc[3 * g]), s1 = exp((double)lsc[3 * g + 1]),
                   s2 = exp((double)lsc[3 * g + 2]);
      const double ss[3] = {s0 * s0, s1 * s1, s2 * s2};
      int e = 0;
#pragma unroll
      for (int i = 0; i < 3; ++i)
#pragma unroll
        for (int j = i; j < 3; ++j)
          Sg[e++] = R[i][0] * R[j][0] * ss[0] + R[i][1] * R[j][1] * ss[1] + R[i][2] * R[j][2] * ss[2];
    }
    for (int v = 0; v < V; ++v) {
      const size_t iv = (size_t)v * G + g;
      // all loads of the view issued together (one memory round trip per view); the record and
      // sums of a view where g is culled are read but not used
      const float4* rh = rec + rec_hi(iv);
      const float4 r3 = rh[1];  // (z, x_c, y_c, flags)
      const float4 r2 = rh[0];  // (conic a, b, c, opacity)
      const double2* a2 = reinterpret_cast<const double2*>(accb + iv * kAccBN);
      const double2 aq = a2[0], ar = a2[1], ah = a2[2], ad = a2[3], ae = a2[4];
      const int flags = __float_as_int(r3.w);
      if (!(flags & kFlagVisible)) continue;
      // aq = (q, w r0), ar = (w r1, w r2), ah = (h, h dx), ad = (h dy, h dx dx), ae = (h dx dy, h dy dy)
      qg += eps + aq.x;
      const double o = r2.w;
      glogit += (1.0 - o) * ah.x;
      const float* vw = views + 20 * v;
      // colour: SH block and view direction
      const double gc0 = (flags & 1) ? aq.y : 0.0, gc1 = (flags & 2) ? ar.x : 0.0,
                   gc2 = (flags & 4) ? ar.y : 0.0;
      {
        const double xw = r3.y, yw = r3.z, zw = r3.x;  // camera point
        const double d0 = vw[0] * xw + vw[4] * yw + vw[8] * zw;
        const double d1 = vw[1] * xw + vw[5] * yw + vw[9] * zw;
        const double d2 = vw[2] * xw + vw[6] * yw + vw[10] * zw;
        const double len = sqrt(d0 * d0 + d1 * d1 + d2 * d2);
        const double il = 1.0 / len;
        const double u0 = d0 * il, u1 = d1 * il, u2 = d2 * il;
        float B[16];
        sh_poly<DEG>((float)u0, (float)u1, (float)u2, B);
        double gd[3] = {0.0, 0.0, 0.0};
#pragma unroll
        for (int k = 0; k < D; ++k) {
          col[(11 + 3 * k) * kP] += B[k] * (float)gc0;
          col[(12 + 3 * k) * kP] += B[k] * (float)gc1;
          col[(13 + 3 * k) * kP] += B[k] * (float)gc2;
          if (k > 0) {
            const double gB = gc0 * shc[(3 * k) * kP] + gc1 * shc[(3 * k + 1) * kP] +
                              gc2 * shc[(3 * k + 2) * kP];
            double db[3];
            sh_dB(k, u0, u1, u2, db);
            gd[0] += gB * db[0];
            gd[1] += gB * db[1];
            gd[2] += gB * db[2];
          }
        }
        const double dg = u0 * gd[0] + u1 * gd[1] + u2 * gd[2];
        gmu[0] += (gd[0] - u0 * dg) * il;
        gmu[1] += (gd[1] - u1 * dg) * il;
        gmu[2] += (gd[2] - u2 * dg) * il;
      }
      // projected centre (through the conic the render used) and conic
      const double qa = r2.x, qb = r2.y, qc = r2.z;
      const double gmx = qa * ah.y + qb * ad.x, gmy = qb * ah.y + qc * ad.x;
      const double gqa = -0.5 * ad.y, gqb2 = -0.5 * ae.x, gqc = -0.5 * ae.y;  // dL/dQ, symmetric
      // EWA Jacobian with the projection's fp32 clamp decision
      const float uf = r3.y / r3.x, vf = r3.z / r3.x;
      const float limx = 1.3f * ((0.5f * (float)W) / vw[16]);
      const float limy = 1.3f * ((0.5f * (float)H) / vw[17]);
      const bool in_u = uf >= -limx && uf <= limx, in_v = vf >= -limy && vf <= limy;
      const double fx = vw[16], fy = vw[17];
      const double x = r3.y, y = r3.z, z = r3.x;
      const double iz = 1.0 / z;
      const double uc = in_u ? x * iz : (double)fminf(limx, fmaxf(-limx, uf));
      const double vc = in_v ? y * iz : (double)fminf(limy, fmaxf(-limy, vf));
      const double j00 = fx * iz, j02 = -fx * uc * iz, j11 = fy * iz, j12 = -fy * vc * iz;
      // Sc = R_v Sigma3D R_v^T
      double Rv[3][3];
#pragma unroll
      for (int i = 0; i < 3; ++i)
#pragma unroll
        for (int j = 0; j < 3; ++j) Rv[i][j] = vw[4 * i + j];
      double Sc[3][3];
      {
        const double S3[3][3] = {{Sg[0], Sg[1], Sg[2]}, {Sg[1], Sg[3], Sg[4]}, {Sg[2], Sg[4], Sg[5]}};
        double T3[3][3];
#pragma unroll
        for (int i = 0; i < 3; ++i)
#pragma unroll
          for (int j = 0; j < 3; ++j)
            T3[i][j] = Rv[i][0] * S3[0][j] + Rv[i][1] * S3[1][j] + Rv[i][2] * S3[2][j];
#pragma unroll
        for (int i = 0; i < 3; ++i)
#pragma unroll
          for (int j = 0; j < 3; ++j)
            Sc[i][j] = T3[i][0] * Rv[j][0] + T3[i][1] * Rv[j][1] + T3[i][2] * Rv[j][2];
      }
      // rows of J Sc; Sigma2D and its inverse (double)
      const double JS0[3] = {j00 * Sc[0][0] + j02 * Sc[2][0], j00 * Sc[0][1] + j02 * Sc[2][1],
                             j00 * Sc[0][2] + j02 * Sc[2][2]};
      const double JS1[3] = {j11 * Sc[1][0] + j12 * Sc[2][0], j11 * Sc[1][1] + j12 * Sc[2][1],
                             j11 * Sc[1][2] + j12 * Sc[2][2]};
      const double sa = JS0[0] * j00 + JS0[2] * j02 + 0.3;
      const double sb = JS0[1] * j11 + JS0[2] * j12;
      const double sc = JS1[1] * j11 + JS1[2] * j12 + 0.3;
      const double idet = 1.0 / (sa * sc - sb * sb);
      const double Q00 = sc * idet, Q01 = -sb * idet, Q11 = sa * idet;
      // dL/dSigma2D = -Q (dL/dQ) Q
      const double A00 = Q00 * gqa + Q01 * gqb2, A01 = Q00 * gqb2 + Q01 * gqc;
      const double A10 = Q01 * gqa + Q11 * gqb2, A11 = Q01 * gqb2 + Q11 * gqc;
      const double e00 = -(A00 * Q00 + A01 * Q01);
      const double e01 = -(A00 * Q01 + A01 * Q11);
      const double e11 = -(A10 * Q01 + A11 * Q11);
      // dL/dJ = 2 (dL/dSigma2D) J Sc (the four non-zero entries of J)
      const double dj00 = 2.0 * (e00 * JS0[0] + e01 * JS1[0]);
      const double dj02 = 2.0 * (e00 * JS0[2] + e01 * JS1[2]);
      const double dj11 = 2.0 * (e01 * JS0[1] + e11 * JS1[1]);
      const double dj12 = 2.0 * (e01 * JS0[2] + e11 * JS1[2]);
      // camera point
      const double iz2 = iz * iz;
      const double gxd = gmx * fx * iz, gyd = gmy * fy * iz;
      const double gzd = -(gmx * fx * x + gmy * fy * y) * iz2;
      double gx = gxd, gy = gyd, gz = gzd;
      gz -= (dj00 * fx + dj11 * fy) * iz2;
      if (in_u) { gx -= dj02 * fx * iz2; gz += 2.0 * dj02 * fx * x * iz2 * iz; }
      else gz += dj02 * fx * uc * iz2;
      if (in_v) { gy -= dj12 * fy * iz2; gz += 2.0 * dj12 * fy * y * iz2 * iz; }
      else gz += dj12 * fy * vc * iz2;
#pragma unroll
      for (int i = 0; i < 3; ++i) {
        gmu[i] += Rv[0][i] * gx + Rv[1][i] * gy + Rv[2][i] * gz;
        gdet[i] += Rv[0][i] * gxd + Rv[1][i] * gyd + Rv[2][i] * gzd;
      }
      // dL/dSc = J^T (dL/dSigma2D) J, then dL/dSigma3D += R_v^T dL/dSc R_v
      {
        const double J0[3] = {j00, 0.0, j02}, J1[3] = {0.0, j11, j12};
        double dSc[3][3];
#pragma unroll
        for (int k = 0; k < 3; ++k)
#pragma unroll
          for (int l = 0; l < 3; ++l)
            dSc[k][l] = e00 * J0[k] * J0[l] + e01 * (J0[k] * J1[l] + J1[k] * J0[l]) +
                        e11 * J1[k] * J1[l];
        double U[3][3];
#pragma unroll
        for (int k = 0; k < 3; ++k)
#pragma unroll
          for (int j = 0; j < 3; ++j)
            U[k][j] = dSc[k][0] * Rv[0][j] + dSc[k][1] * Rv[1][j] + dSc[k][2] * Rv[2][j];
        int e = 0;
#pragma unroll
        for (int i = 0; i < 3; ++i)
#pragma unroll
          for (int j = i; j < 3; ++j) dS[e++] += Rv[0][i] * U[0][j] + Rv[1][i] * U[1][j] + Rv[2][i] * U[2][j];
      }
    }
    // Sigma3D = M M^T with M = Rq diag(s): dL/dM = 2 dL/dSigma3D M
    double glsc[3], gq[4];
    {
      const float4 q4 = reinterpret_cast<const float4*>(quats)[g];
      const double qn = sqrt((double)q4.x * q4.x + (double)q4.y * q4.y + (double)q4.z * q4.z +
                             (double)q4.w * q4.w);
      const double w = q4.x / qn, x = q4.y / qn, y = q4.z / qn, z = q4.w / qn;
      const double R[3][3] = {{1 - 2 * (y * y + z * z), 2 * (x * y - w * z), 2 * (x * z + w * y)},
                              {2 * (x * y + w * z), 1 - 2 * (x * x + z * z), 2 * (y * z - w * x)},
                              {2 * (x * z - w * y), 2 * (y * z + w * x), 1 - 2 * (x * x + y * y)}};
      const double s[3] = {exp((double)lsc[3 * g]), exp((double)lsc[3 * g + 1]),
                           exp((double)lsc[3 * g + 2])};
      const double dSm[3][3] = {{dS[0], dS[1], dS[2]}, {dS[1], dS[3], dS[4]}, {dS[2], dS[4], dS[5]}};
      double dR[3][3];
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        double gs = 0.0;
#pragma unroll
        for (int i = 0; i < 3; ++i) {
          // dL/dM_ik = 2 sum_j dSigma_ij M_jk, M_jk = R_jk s_k
          const double dM = 2.0 * (dSm[i][0] * R[0][k] + dSm[i][1] * R[1][k] + dSm[i][2] * R[2][k]) * s[k];
          gs += dM * R[i][k];
          dR[i][k] = dM * s[k];
        }
        glsc[k] = gs * s[k];
      }
      // rotation entries as functions of the unit quaternion (w, x, y, z)
      const double gw = 2.0 * (-z * dR[0][1] + y * dR[0][2] + z * dR[1][0] - x * dR[1][2] -
                               y * dR[2][0] + x * dR[2][1]);
      const double gx = 2.0 * (y * dR[0][1] + z * dR[0][2] + y * dR[1][0] - 2.0 * x * dR[1][1] -
                               w * dR[1][2] + z * dR[2][0] + w * dR[2][1] - 2.0 * x * dR[2][2]);
      const double gy = 2.0 * (-2.0 * y * dR[0][0] + x * dR[0][1] + w * dR[0][2] + x * dR[1][0] +
                               z * dR[1][2] - w * dR[2][0] + z * dR[2][1] - 2.0 * y * dR[2][2]);
      const double gz = 2.0 * (-2.0 * z * dR[0][0] - w * dR[0][1] + x * dR[0][2] + w * dR[1][0] -
                               2.0 * z * dR[1][1] + y * dR[1][2] + x * dR[2][0] + y * dR[2][1]);
      const double dot = w * gw + x * gx + y * gy + z * gz;
      gq[0] = (gw - w * dot) / qn;
      gq[1] = (gx - x * dot) / qn;
      gq[2] = (gy - y * dot) / qn;
      gq[3] = (gz - z * dot) / qn;
    }
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      col[i * kP] = (float)gmu[i];
      col[(3 + i) * kP] = (float)glsc[i];
      s_det[i * kP + threadIdx.x] = (float)gdet[i];
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) col[(6 + i) * kP] = (float)gq[i];
    col[10 * kP] = (float)glogit;
    s_fac[threadIdx.x] = (float)(1.0 / qg);
    s_fac[kP + threadIdx.x] =
        (float)exp(((double)lsc[3 * g] + (double)lsc[3 * g + 1] + (double)lsc[3 * g + 2]) / 3.0);
  }
  __syncthreads();
  // coalesced stores of the requested variants: the block's rows are contiguous in each output
  float* outs[4] = {out_raw, out_det, out_sup, out_psc};
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    float* dst = outs[m];
    if (!dst) continue;
    dst += (size_t)g0 * K;
    for (int L = threadIdx.x; L < ng * K; L += kGradThreads) {
      const int row = L / K, c = L - row * K;
      float val = s_out[c * kP + row];
      if (m == 1) val = c < 3 ? s_det[c * kP + row] : (c < 10 ? 0.0f : val);
      else if (m == 2) val = (float)((double)val * (double)s_fac[row]);
      else if (m == 3 && c < 3) val = (float)((double)val * (double)s_fac[kP + row]);
      dst[L] = val;
    }
  }
}

template <int DEG>
int grad_launch(Workspace& w, const float* lsc, const float* quats, const float* sh, float* raw,
                float* det, float* sup, float* psc, cudaStream_t st) {
  constexpr int D = (DEG + 1) * (DEG + 1);
  constexpr int K = 11 + 3 * D;
  const size_t smem = (size_t)(3 * D + K + 5) * kP * sizeof(float);
  static int configured_device = -1;  // the attribute is per device
  if (configured_device != w.device) {
    cudaError_t e = cudaFuncSetAttribute(k_grad<DEG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess)
      return set_err(w, SPLAT_ERR_CUDA, std::string("gradient kernel attribute: ") +
                                            cudaGetErrorString(e));
    configured_device = w.device;
  }
  const int blocks = (w.G + kGradThreads - 1) / kGradThreads;
  k_grad<DEG><<<blocks, kGradThreads, smem, st>>>(w.rec, w.accb, w.views, lsc, quats, sh, w.G,
                                                   w.V, w.H, w.W, raw, det, sup, psc);
  return SPLAT_OK;
}

}  // namespace

int launch_grad(Workspace& w, const float* lsc, const float* quats, const float* sh, float* raw,
                float* det, float* sup, float* psc, cudaStream_t st) {
  if (w.G == 0) return SPLAT_OK;
  const int tok = prof_begin(w, st, SPLAT_K_GRAD);
  int rc;
  switch (w.deg) {
    case 0: rc = grad_launch<0>(w, lsc, quats, sh, raw, det, sup, psc, st); break;
    case 1: rc = grad_launch<1>(w, lsc, quats, sh, raw, det, sup, psc, st); break;
    case 2: rc = grad_launch<2>(w, lsc, quats, sh, raw, det, sup, psc, st); break;
    default: rc = grad_launch<3>(w, lsc, quats, sh, raw, det, sup, psc, st); break;
  }
  prof_end(w, st, tok);
  if (rc) return rc;
  return check_launch(w, "gradient kernel");
}

}  // namespace splat
