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
// once by q_g (the linear rewrite; no second pass over the views). The per-view terms (Jacobian,
// pullback, J^T J, SH products) are fp32 products (~6e-8 relative rounding each; fewer registers,
// so more Gaussians in flight in this latency-bound loop); the sums over views, the division by
// q_g and the eigenvalues are double. The SH block is accumulated in a shared-memory tile of the
// block's token rows (keeps registers, hence occupancy, low) that is then written out with
// coalesced stores.
#include "common.cuh"

namespace splat {
namespace {

constexpr int kFinThreads = 128;
// 7 blocks of 128 threads per SM: 72 registers a thread (the shared-memory token tile, 29 KB a
// block at degree 3, also allows 7)
constexpr int kFinMinBlocks = 7;


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

// Per-Gaussian sums over the views where g is visible, all linear in the per-view terms (so the
// sums of disjoint view sets add): qsum = sum_v q_gv, b = sum_v J^T Sigma^-1 Sd,
// sa = sum_v (1 - o) Sa, A = sum_v q_gv J^T J (6 entries) in registers (double); the SH block
// sum_v M_color (Swr (x) B) is added into the shared-memory column `col` (stride P) at 4 + k.
template <int DEG, int P>
__device__ __forceinline__ void view_sums(const float4* __restrict__ rec,
                                          const float* __restrict__ acc,
                                          const float* __restrict__ views, int G, int V, int g,
                                          double& qsum, double b[3], double& sa, double A[6],
                                          float* col) {
  constexpr int D = (DEG + 1) * (DEG + 1);
  const double eps = 1e-6;
  for (int v = 0; v < V; ++v) {
    const size_t i = (size_t)v * G + g;
    const float4* rh = rec + rec_hi(i);
    const float4 r3 = rh[1];  // (z, x_c, y_c, flags)
    const int flags = __float_as_int(r3.w);
    if (!(flags & kFlagVisible)) continue;
    const float4 r2 = rh[0];  // (conic a, b, c, opacity)
    // (q, w r (3)) and (w rho, w rho d (2), unused)
    const float4* a4 = reinterpret_cast<const float4*>(acc + i * kAccN);
    const float4 aq = a4[0], as = a4[1];
    const double qgv = eps + (double)aq.x;
    qsum += qgv;
    sa += (1.0 - (double)r2.w) * (double)as.x;
    // per-view products in fp32 (rounding ~1e-7 relative), sums over views in double
    const float sd0 = as.y, sd1 = as.z;
    const float sm0 = r2.x * sd0 + r2.y * sd1;
    const float sm1 = r2.y * sd0 + r2.z * sd1;
    // J = J_cam(x_c) R_v, unclamped pinhole Jacobian
    const float* vw = views + 20 * v;
    const float fx = vw[16], fy = vw[17];
    const float x = r3.y, y = r3.z, iz = 1.0f / r3.x;
    const float j00 = fx * iz, j02 = -fx * x * iz * iz;
    const float j11 = fy * iz, j12 = -fy * y * iz * iz;
    float J0[3], J1[3];
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      J0[c] = j00 * vw[c] + j02 * vw[8 + c];
      J1[c] = j11 * vw[4 + c] + j12 * vw[8 + c];
    }
    b[0] += (double)(J0[0] * sm0 + J1[0] * sm1);
    b[1] += (double)(J0[1] * sm0 + J1[1] * sm1);
    b[2] += (double)(J0[2] * sm0 + J1[2] * sm1);
    const float qf = (float)qgv;
    A[0] += (double)(qf * (J0[0] * J0[0] + J1[0] * J1[0]));
    A[1] += (double)(qf * (J0[0] * J0[1] + J1[0] * J1[1]));
    A[2] += (double)(qf * (J0[0] * J0[2] + J1[0] * J1[2]));
    A[3] += (double)(qf * (J0[1] * J0[1] + J1[1] * J1[1]));
    A[4] += (double)(qf * (J0[1] * J0[2] + J1[1] * J1[2]));
    A[5] += (double)(qf * (J0[2] * J0[2] + J1[2] * J1[2]));
    // view direction (mu - camera centre) / |.| = R_v^T x_c / |x_c|
    float B[16];
    {
      const float dw0 = vw[0] * r3.y + vw[4] * r3.z + vw[8] * r3.x;
      const float dw1 = vw[1] * r3.y + vw[5] * r3.z + vw[9] * r3.x;
      const float dw2 = vw[2] * r3.y + vw[6] * r3.z + vw[10] * r3.x;
      const float il = rsqrtf(dw0 * dw0 + dw1 * dw1 + dw2 * dw2);
      sh_poly<DEG>(dw0 * il, dw1 * il, dw2 * il, B);
    }
    const float w0 = (flags & 1) ? aq.y : 0.0f;
    const float w1 = (flags & 2) ? aq.z : 0.0f;
    const float w2 = (flags & 4) ? aq.w : 0.0f;
#pragma unroll
    for (int k = 0; k < D; ++k) {
      col[(4 + 3 * k) * P] += B[k] * w0;
      col[(5 + 3 * k) * P] += B[k] * w1;
      col[(6 + 3 * k) * P] += B[k] * w2;
      // (a compiler-only fence every four coefficients: without it the 3 x D shared-memory
      // loads of the block are all hoisted ahead of their adds, which holds ~48 more registers
      // and caps the kernel at 16 warps per SM)
      if ((k & 3) == 3) asm volatile("" ::: "memory");
    }
  }
}

// token from the sums: q_g = eps + qsum, everything divided once by q_g (gamma_gv / q_gv = 1/q_g),
// A = lambda I + (sum q_gv J^T J) / q_g, conditioning statistics of A. Writes columns 0..DT-1 of
// `col`; the SH block must already sit in columns 4 .. 4 + 3d - 1 (it is scaled in place).
template <int DEG, int P>
__device__ __forceinline__ void finish_token(double qsum, const double b[3], double sa,
                                             const double An[6], double lambda, float* col) {
  constexpr int D = (DEG + 1) * (DEG + 1);
  const double eps = 1e-6;
  const double qg = eps + qsum;
  const double inv = 1.0 / qg;
  const double A00 = An[0] * inv + lambda, A11 = An[3] * inv + lambda, A22 = An[5] * inv + lambda;
  const double A01 = An[1] * inv, A02 = An[2] * inv, A12 = An[4] * inv;
  double ev[3];
  eig3_sym(A00, A01, A02, A11, A12, A22, ev);
  const double tr = A00 + A11 + A22;
  col[0 * P] = (float)(b[0] * inv);
  col[1 * P] = (float)(b[1] * inv);
  col[2 * P] = (float)(b[2] * inv);
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

// the block's rows (ncols each) are contiguous in the output: coalesced stores from the tile
template <int P>
__device__ __forceinline__ void store_rows(const float* s_tile, int ncols, int g0, int G,
                                           float* out_rows) {
  const int ng = min(kFinThreads, G - g0);
  float* out = out_rows + (size_t)g0 * ncols;
  for (int L = threadIdx.x; L < ng * ncols; L += kFinThreads) {
    const int row = L / ncols, c = L - row * ncols;
    out[L] = s_tile[c * P + row];
  }
}

// fused single-device path: sums over all views, then the token
template <int DEG>
__global__ void __launch_bounds__(kFinThreads, kFinMinBlocks)
k_finalize(const float4* __restrict__ rec, const float* __restrict__ acc,
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
    double qsum = 0.0, sa = 0.0, b[3] = {0.0, 0.0, 0.0}, A[6] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
    view_sums<DEG, P>(rec, acc, views, G, V, g, qsum, b, sa, A, col);
    finish_token<DEG, P>(qsum, b, sa, A, lambda, col);
  }
  __syncthreads();
  store_rows<P>(s_tok, DT, g0, G, tokens);
}

// sharded path, part 1: this device's per-Gaussian partial sums over its views,
// [qsum, b(3), sa, A(6: 00 01 02 11 12 22), SH block (3d)] = 11 + 3d floats per Gaussian
template <int DEG>
__global__ void __launch_bounds__(kFinThreads, kFinMinBlocks)
k_partials(const float4* __restrict__ rec, const float* __restrict__ acc,
           const float* __restrict__ views, int G, int V, float* __restrict__ partials) {
  constexpr int D = (DEG + 1) * (DEG + 1);
  constexpr int K = 11 + 3 * D;
  constexpr int P = kFinThreads + 1;
  __shared__ float s_tile[K * P];
  const int g0 = blockIdx.x * kFinThreads;
  const int g = g0 + threadIdx.x;
  float* col = s_tile + threadIdx.x;
  // the SH sums are accumulated at columns 4.. (the layout view_sums writes), then moved behind
  // the eleven scalar sums
#pragma unroll
  for (int k = 0; k < 3 * D; ++k) col[(4 + k) * P] = 0.0f;
  if (g < G) {
    double qsum = 0.0, sa = 0.0, b[3] = {0.0, 0.0, 0.0}, A[6] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
    view_sums<DEG, P>(rec, acc, views, G, V, g, qsum, b, sa, A, col);
#pragma unroll
    for (int k = 3 * D - 1; k >= 0; --k) col[(11 + k) * P] = col[(4 + k) * P];
    col[0] = (float)qsum;
    col[1 * P] = (float)b[0];
    col[2 * P] = (float)b[1];
    col[3 * P] = (float)b[2];
    col[4 * P] = (float)sa;
#pragma unroll
    for (int k = 0; k < 6; ++k) col[(5 + k) * P] = (float)A[k];
  }
  __syncthreads();
  store_rows<P>(s_tile, K, g0, G, partials);
}

// sharded path, part 2: tokens from (summed) partials; needs no workspace
template <int DEG>
__global__ void __launch_bounds__(kFinThreads, 4)
k_finalize_partials(const float* __restrict__ partials, int G, double lambda,
                    float* __restrict__ tokens) {
  constexpr int D = (DEG + 1) * (DEG + 1);
  constexpr int K = 11 + 3 * D;
  constexpr int DT = 9 + 3 * D;
  constexpr int P = kFinThreads + 1;
  __shared__ float s_tile[K * P];
  const int g0 = blockIdx.x * kFinThreads;
  const int ng = min(kFinThreads, G - g0);
  const float* in = partials + (size_t)g0 * K;
  for (int L = threadIdx.x; L < ng * K; L += kFinThreads) {
    const int row = L / K, c = L - row * K;
    s_tile[c * P + row] = in[L];
  }
  __syncthreads();
  float* col = s_tile + threadIdx.x;
  double qsum = 0.0, sa = 0.0, b[3], A[6];
  if (threadIdx.x < ng) {
    qsum = col[0];
    b[0] = col[1 * P];
    b[1] = col[2 * P];
    b[2] = col[3 * P];
    sa = col[4 * P];
#pragma unroll
    for (int k = 0; k < 6; ++k) A[k] = col[(5 + k) * P];
  }
  __syncthreads();  // the token overwrites the tile's columns in place
  if (threadIdx.x < ng) {
#pragma unroll
    for (int k = 0; k < 3 * D; ++k) col[(4 + k) * P] = col[(11 + k) * P];
    finish_token<DEG, P>(qsum, b, sa, A, lambda, col);
  }
  __syncthreads();
  store_rows<P>(s_tile, DT, g0, G, tokens);
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

int launch_partials(Workspace& w, float* partials, cudaStream_t st) {
  if (w.G == 0) return SPLAT_OK;
  const int blocks = (w.G + kFinThreads - 1) / kFinThreads;
  const int tok = prof_begin(w, st, SPLAT_K_FINALIZE);
#define SPLAT_PART(DEG) \
  k_partials<DEG><<<blocks, kFinThreads, 0, st>>>(w.rec, w.acc, w.views, w.G, w.V, partials)
  switch (w.deg) {
    case 0: SPLAT_PART(0); break;
    case 1: SPLAT_PART(1); break;
    case 2: SPLAT_PART(2); break;
    default: SPLAT_PART(3); break;
  }
#undef SPLAT_PART
  prof_end(w, st, tok);
  return check_launch(w, "partial sums kernel");
}

cudaError_t launch_finalize_partials(const float* partials, int G, int deg, double lambda,
                                     float* tokens, cudaStream_t st) {
  if (G == 0) return cudaSuccess;
  const int blocks = (G + kFinThreads - 1) / kFinThreads;
  switch (deg) {
    case 0: k_finalize_partials<0><<<blocks, kFinThreads, 0, st>>>(partials, G, lambda, tokens); break;
    case 1: k_finalize_partials<1><<<blocks, kFinThreads, 0, st>>>(partials, G, lambda, tokens); break;
    case 2: k_finalize_partials<2><<<blocks, kFinThreads, 0, st>>>(partials, G, lambda, tokens); break;
    default: k_finalize_partials<3><<<blocks, kFinThreads, 0, st>>>(partials, G, lambda, tokens); break;
  }
  return cudaGetLastError();
}

}  // namespace splat
