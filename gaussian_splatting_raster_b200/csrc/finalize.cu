// Token finalisation: per Gaussian, over the views in which it is visible, the cross-view
// weights, the 3-D covector pullback of the projected-centre score, the conditioning statistics
// and the cross-view appearance scores.
//
// Source: "Research Proposal: Renderer Score Tokens for Recurrent Gaussian Splatting",
// "Exact Score Operators" (q_gv = eps + sum_p w; opacity-logit score; SH score; projected-centre
// score with grad G = G Sigma2D^-1 (p - mu2D); J_gv = d pi_v(mu_g) / d mu_g;
// gamma_gv = q_gv / (eps + sum_v' q_gv'); b = sum_v gamma J^T s^mu2D; A = lambda I +
// sum_v gamma J^T J; e~ = eig(A) / (tr A + eps); l = log(tr A + eps); s^alpha_g and s^SH_g as
// gamma-weighted sums) and "Final Token and Updater" (z_g = [b(3), s^alpha, s^SH(3 d_SH),
// log q_g, e~(3), l], 9 + 3 d_SH entries).
//
// Because gamma_gv / q_gv = 1 / q_g for every view, each block is a plain sum over views divided
// once by q_g (the linear rewrite; no second pass over the views). Sums and the eigenvalues are
// evaluated in double; the SH block's per-view products in fp32, accumulated in a shared-memory
// tile of the block's token rows (keeps registers, hence occupancy, low) that is then written out
// with coalesced stores.
#include "common.cuh"

namespace splat {
namespace {

constexpr int kFinThreads = 128;

// eigenvalues of a symmetric 3x3 matrix, descending, by the trigonometric solution of the
// characteristic cubic (O. K. Smith, "Eigenvalues of a symmetric 3x3 matrix", CACM 4(4), 1961)
__device__ void eig3_sym(double a00, double a01, double a02, double a11, double a12, double a22,
                         double ev[3]) {
  const double p1 = a01 * a01 + a02 * a02 + a12 * a12;
  const double q = (a00 + a11 + a22) / 3.0;
  const double d0 = a00 - q, d1 = a11 - q, d2 = a22 - q;
  const double p2 = d0 * d0 + d1 * d1 + d2 * d2 + 2.0 * p1;
  if (p2 <= 0.0) {
    ev[0] = ev[1] = ev[2] = q;
    return;
  }
  const double p = sqrt(p2 / 6.0);
  const double ip = 1.0 / p;
  const double b00 = d0 * ip, b11 = d1 * ip, b22 = d2 * ip;
  const double b01 = a01 * ip, b02 = a02 * ip, b12 = a12 * ip;
  const double detB = b00 * (b11 * b22 - b12 * b12) - b01 * (b01 * b22 - b12 * b02) +
                      b02 * (b01 * b12 - b11 * b02);
  double r = 0.5 * detB;
  r = fmin(1.0, fmax(-1.0, r));
  const double phi = acos(r) / 3.0;
  const double e1 = q + 2.0 * p * cos(phi);
  const double e3 = q + 2.0 * p * cos(phi + 2.0943951023931954923);  // + 2 pi / 3
  const double e2 = 3.0 * q - e1 - e3;
  ev[0] = e1;
  ev[1] = e2;
  ev[2] = e3;
  // e1 >= e2 >= e3 holds analytically; enforce it against rounding
  if (ev[1] > ev[0]) { const double tt = ev[0]; ev[0] = ev[1]; ev[1] = tt; }
  if (ev[2] > ev[1]) { const double tt = ev[1]; ev[1] = ev[2]; ev[2] = tt; }
  if (ev[1] > ev[0]) { const double tt = ev[0]; ev[0] = ev[1]; ev[1] = tt; }
}

template <int DEG>
__global__ void __launch_bounds__(kFinThreads, 4)
k_finalize(const float4* __restrict__ rec, const double* __restrict__ acc,
           const float* __restrict__ views, int G, int V, double lambda,
           float* __restrict__ tokens) {
  constexpr int D = (DEG + 1) * (DEG + 1);
  constexpr int DT = 9 + 3 * D;
  constexpr int P = kFinThreads + 1;  // padded column stride: conflict-free row/column access
  // the block's token rows, column-major; the SH block is accumulated here directly
  __shared__ float s_tok[DT * P];
  const int g0 = blockIdx.x * kFinThreads;
  const int g = g0 + threadIdx.x;
  float* col = s_tok + threadIdx.x;
#pragma unroll
  for (int k = 0; k < 3 * D; ++k) col[(4 + k) * P] = 0.0f;
  if (g < G) {
    const double eps = 1e-6;
    double qsum = 0.0, b0 = 0.0, b1 = 0.0, b2 = 0.0, sa = 0.0;
    double A00 = 0.0, A01 = 0.0, A02 = 0.0, A11 = 0.0, A12 = 0.0, A22 = 0.0;
    for (int v = 0; v < V; ++v) {
      const size_t i = (size_t)v * G + g;
      const float4 r3 = rec[i * kRecF4 + 3];  // (z, x_c, y_c, flags)
      const int flags = __float_as_int(r3.w);
      if (!(flags & kFlagVisible)) continue;
      const float4 r0 = rec[i * kRecF4], r1 = rec[i * kRecF4 + 1];
      const double2* a2 = reinterpret_cast<const double2*>(acc + i * kAccN);
      const double2 a01 = a2[0], a23 = a2[1], a45 = a2[2], a67 = a2[3];
      const double qgv = eps + a01.x;
      qsum += qgv;
      sa += (1.0 - (double)r1.y) * a45.x;
      const double qa = r0.z, qb = r0.w, qc = r1.x;
      const double sm0 = qa * a45.y + qb * a67.x;
      const double sm1 = qb * a45.y + qc * a67.x;
      // J = J_cam(x_c) R_v, unclamped pinhole Jacobian
      const float* vw = views + 20 * v;
      const double fx = vw[16], fy = vw[17];
      const double x = r3.y, y = r3.z, z = r3.x;
      const double j00 = fx / z, j02 = -fx * x / (z * z);
      const double j11 = fy / z, j12 = -fy * y / (z * z);
      double J0[3], J1[3];
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        J0[c] = j00 * (double)vw[c] + j02 * (double)vw[8 + c];
        J1[c] = j11 * (double)vw[4 + c] + j12 * (double)vw[8 + c];
      }
      b0 += J0[0] * sm0 + J1[0] * sm1;
      b1 += J0[1] * sm0 + J1[1] * sm1;
      b2 += J0[2] * sm0 + J1[2] * sm1;
      A00 += qgv * (J0[0] * J0[0] + J1[0] * J1[0]);
      A01 += qgv * (J0[0] * J0[1] + J1[0] * J1[1]);
      A02 += qgv * (J0[0] * J0[2] + J1[0] * J1[2]);
      A11 += qgv * (J0[1] * J0[1] + J1[1] * J1[1]);
      A12 += qgv * (J0[1] * J0[2] + J1[1] * J1[2]);
      A22 += qgv * (J0[2] * J0[2] + J1[2] * J1[2]);
      // view direction (mu - camera centre) / |.| = R_v^T x_c / |x_c|
      float B[16];
      {
        const float dw0 = vw[0] * r3.y + vw[4] * r3.z + vw[8] * r3.x;
        const float dw1 = vw[1] * r3.y + vw[5] * r3.z + vw[9] * r3.x;
        const float dw2 = vw[2] * r3.y + vw[6] * r3.z + vw[10] * r3.x;
        const float il = rsqrtf(dw0 * dw0 + dw1 * dw1 + dw2 * dw2);
        sh_poly<DEG>(dw0 * il, dw1 * il, dw2 * il, B);
      }
      const float w0 = (flags & 1) ? (float)a01.y : 0.0f;
      const float w1 = (flags & 2) ? (float)a23.x : 0.0f;
      const float w2 = (flags & 4) ? (float)a23.y : 0.0f;
#pragma unroll
      for (int k = 0; k < D; ++k) {
        col[(4 + 3 * k) * P] += B[k] * w0;
        col[(5 + 3 * k) * P] += B[k] * w1;
        col[(6 + 3 * k) * P] += B[k] * w2;
      }
    }
    const double qg = eps + qsum;
    const double inv = 1.0 / qg;
    A00 = A00 * inv + lambda;
    A11 = A11 * inv + lambda;
    A22 = A22 * inv + lambda;
    A01 *= inv;
    A02 *= inv;
    A12 *= inv;
    double ev[3];
    eig3_sym(A00, A01, A02, A11, A12, A22, ev);
    const double tr = A00 + A11 + A22;
    col[0 * P] = (float)(b0 * inv);
    col[1 * P] = (float)(b1 * inv);
    col[2 * P] = (float)(b2 * inv);
    col[3 * P] = (float)(sa * inv);
#pragma unroll
    for (int k = 0; k < 3 * D; ++k) col[(4 + k) * P] = (float)((double)col[(4 + k) * P] * inv);
    col[(4 + 3 * D) * P] = (float)log(qg);
    const double itr = 1.0 / (tr + eps);
    col[(5 + 3 * D) * P] = (float)(ev[0] * itr);
    col[(6 + 3 * D) * P] = (float)(ev[1] * itr);
    col[(7 + 3 * D) * P] = (float)(ev[2] * itr);
    col[(8 + 3 * D) * P] = (float)log(tr + eps);
  }
  __syncthreads();
  // the block's rows are contiguous in the output: coalesced stores
  const int ng = min(kFinThreads, G - g0);
  float* out = tokens + (size_t)g0 * DT;
  for (int L = threadIdx.x; L < ng * DT; L += kFinThreads) {
    const int row = L / DT, c = L - row * DT;
    out[L] = s_tok[c * P + row];
  }
}

}  // namespace

int launch_finalize(Workspace& w, float lambda, float* tokens, cudaStream_t st) {
  if (w.G == 0) return SPLAT_OK;
  const int blocks = (w.G + kFinThreads - 1) / kFinThreads;
  const int tok = prof_begin(w, st, SPLAT_K_FINALIZE);
#define SPLAT_FIN(DEG)                                                                     \
  k_finalize<DEG><<<blocks, kFinThreads, 0, st>>>(w.rec, w.acc, w.views, w.G, w.V,        \
                                                  (double)lambda, tokens)
  switch (w.deg) {
    case 0: SPLAT_FIN(0); break;
    case 1: SPLAT_FIN(1); break;
    case 2: SPLAT_FIN(2); break;
    default: SPLAT_FIN(3); break;
  }
#undef SPLAT_FIN
  prof_end(w, st, tok);
  return check_launch(w, "finalize kernel");
}

}  // namespace splat
