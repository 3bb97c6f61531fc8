// CPU oracle for the tile-based Gaussian-splatting render and the analytic score replay.
//
// TEST INFRASTRUCTURE ONLY. This file is the slow, plain reference that the CUDA library is
// checked against. Only the tests, the smoke check and the bench's CPU-baseline leg load it; the
// product path never does. It shares no code, header or constant table with the CUDA library.
//
// Sources (web pages; cited by title and section):
//   [P1] "Research Proposal: Renderer Score Tokens for Recurrent Gaussian Splatting" --
//        sections "Two-Stage Algorithm" (Stage 1 standard render, Stage 2 analytic score
//        replay, suffix-composite equation) and "Exact Score Operators" (opacity/weight
//        definitions, residual-suffix contrast, opacity-logit score, SH score, projected-centre
//        mean score, projection Jacobian, cross-view weights, covector pullback, conditioning
//        matrix, final token).
//   [P5] "ATSplat: Compact Feed-forward 3D Gaussian Splatting with Adaptive Token Expansion" --
//        section on prerequisites (3DGS primitive: centre, rotation, scale, opacity, SH
//        coefficients; alpha-compositing rasterisation).
// Where the pages leave a step open (the EWA projection details, near plane, tile rule, SH sign
// convention, thresholds), the standard 3DGS tile rasteriser ("original gsplat tile binning",
// [P1] Stage 1) is the reading; every such reading is listed with the design notes.
//
// Every routine is templated on the working precision R (float or double). In float mode each
// arithmetic step is the IEEE fp32 operation in the stated order (compiled with
// -ffp-contract=off, no fast math), so that the decisions that become integers (which tiles a
// Gaussian touches, the depth order, the alpha/transmittance thresholds) are taken in the same
// precision as the GPU path. Per-Gaussian sums are always accumulated in double.
//
// Parity pins: see the oracle tests (closed forms, brute force, finite differences, eigvalsh,
// std::exp, SH quadrature).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

constexpr int TILE = 16;  // 16x16 pixel tiles ([P1] Stage 1: gsplat tile binning)

// ------------------------------------------------------------------------------------------
// exp. The alpha and transmittance thresholds and the tile footprint turn exp() results into
// integers, so both implementations must produce identical fp32 bits. fp32 mode therefore uses
// an exp written from a published method: Cody & Waite (1980), "Software Manual for the
// Elementary Functions" -- additive range reduction x = k ln2 + r with ln2 split into a short
// high part (so k * hi is exact) and a low correction, then a polynomial for e^r on
// |r| <= ln2 / 2 (here the Taylor series to degree 7 in Horner form with fused multiply-adds),
// then scaling by 2^k through the exponent field. Double mode uses std::exp.
// ------------------------------------------------------------------------------------------
struct CodyWaiteConstants {
  float log2e, ln2_hi, ln2_lo, c[8];
  CodyWaiteConstants() {
    const double ln2 = std::log(2.0);
    log2e = (float)(1.0 / ln2);
    // high part: ln 2 truncated to 16 fractional bits, so |k| <= 128 times it is exact in fp32
    ln2_hi = (float)std::ldexp(std::floor(std::ldexp(ln2, 16)), -16);
    ln2_lo = (float)(ln2 - (double)ln2_hi);
    double f = 1.0;
    for (int n = 0; n < 8; ++n) {  // c[n] = 1 / n!
      if (n > 0) f *= n;
      c[n] = (float)(1.0 / f);
    }
  }
};
const CodyWaiteConstants& cw() {
  static const CodyWaiteConstants k;
  return k;
}

float exp_cw(float x) {
  if (x != x) return x;
  if (!(x > -87.0f)) return 0.0f;
  if (x > 88.0f) return INFINITY;
  const CodyWaiteConstants& K = cw();
  float k = std::nearbyintf(x * K.log2e);  // round half to even (default rounding mode)
  float r = (x - k * K.ln2_hi) - k * K.ln2_lo;
  float p = K.c[7];
  for (int n = 6; n >= 0; --n) p = std::fmaf(p, r, K.c[n]);
  int ki = (int)k;  // in [-126, 127] for x in (-87, 88]
  uint32_t bits = (uint32_t)(ki + 127) << 23;
  float scale;
  std::memcpy(&scale, &bits, 4);
  return p * scale;
}

inline float rexp(float x) { return exp_cw(x); }
inline double rexp(double x) { return std::exp(x); }
inline float rsqrt_ieee(float x) { return std::sqrt(x); }
inline double rsqrt_ieee(double x) { return std::sqrt(x); }

// ------------------------------------------------------------------------------------------
// Real spherical harmonics B_k(dir), k = l^2 + l + m, l = 0..3, m = -l..l, with the
// Condon-Shortley phase (the convention of the 3DGS colour model, [P1] "SH Score": B(d) is the
// SH basis of the view direction). Written from the definition: associated Legendre functions by
// the standard three-term recurrence, normalisation sqrt((2l+1)/(4 pi) (l-|m|)!/(l+|m|)!),
// sqrt(2) cos(m phi) for m > 0 and sqrt(2) sin(|m| phi) for m < 0. Evaluated in double.
// ------------------------------------------------------------------------------------------
void sh_basis_def(int deg, const double dir[3], double* out) {
  const double x = dir[0], y = dir[1], z = dir[2];
  const double ct = z;
  const double st = std::sqrt(std::max(0.0, x * x + y * y));
  const double phi = std::atan2(y, x);
  double P[4][4] = {{0}};  // P[l][m], m >= 0, with Condon-Shortley phase
  for (int m = 0; m <= deg; ++m) {
    double pmm = 1.0;
    for (int i = 1; i <= m; ++i) pmm *= -(2.0 * i - 1.0) * st;  // (-1)^m (2m-1)!! sin^m
    P[m][m] = pmm;
    if (m + 1 <= deg) P[m + 1][m] = ct * (2.0 * m + 1.0) * pmm;
    for (int l = m + 2; l <= deg; ++l)
      P[l][m] = ((2.0 * l - 1.0) * ct * P[l - 1][m] - (l + m - 1.0) * P[l - 2][m]) / (l - m);
  }
  auto fact = [](int n) { double f = 1; for (int i = 2; i <= n; ++i) f *= i; return f; };
  for (int l = 0; l <= deg; ++l) {
    for (int m = -l; m <= l; ++m) {
      const int am = m < 0 ? -m : m;
      const double K = std::sqrt((2.0 * l + 1.0) / (4.0 * M_PI) * fact(l - am) / fact(l + am));
      double v;
      if (m == 0) v = K * P[l][0];
      else if (m > 0) v = std::sqrt(2.0) * K * P[l][am] * std::cos(am * phi);
      else v = std::sqrt(2.0) * K * P[l][am] * std::sin(am * phi);
      out[l * l + l + m] = v;
    }
  }
}

// ------------------------------------------------------------------------------------------
// Symmetric 3x3 eigenvalues by the cyclic Jacobi rotation method (Jacobi 1846; any numerical
// linear algebra text). Used for the conditioning statistics eig(A_g) ([P1] "Exact Score
// Operators", conditioning matrix). Returned in descending order.
// ------------------------------------------------------------------------------------------
void eig3_jacobi(const double A_in[9], double ev[3]) {
  double a[3][3];
  for (int i = 0; i < 3; ++i)
    for (int j = 0; j < 3; ++j) a[i][j] = 0.5 * (A_in[3 * i + j] + A_in[3 * j + i]);
  for (int sweep = 0; sweep < 64; ++sweep) {
    double off = a[0][1] * a[0][1] + a[0][2] * a[0][2] + a[1][2] * a[1][2];
    double diag = a[0][0] * a[0][0] + a[1][1] * a[1][1] + a[2][2] * a[2][2];
    if (off <= 1e-36 * diag || off == 0.0) break;
    for (int p = 0; p < 2; ++p) {
      for (int q = p + 1; q < 3; ++q) {
        if (a[p][q] == 0.0) continue;
        // rotation angle that zeroes a[p][q]
        const double theta = (a[q][q] - a[p][p]) / (2.0 * a[p][q]);
        const double t = (theta >= 0 ? 1.0 : -1.0) / (std::fabs(theta) + std::sqrt(theta * theta + 1.0));
        const double c = 1.0 / std::sqrt(t * t + 1.0), s = t * c;
        for (int k = 0; k < 3; ++k) {  // A <- A G (columns p, q)
          const double akp = a[k][p], akq = a[k][q];
          a[k][p] = c * akp - s * akq;
          a[k][q] = s * akp + c * akq;
        }
        for (int k = 0; k < 3; ++k) {  // A <- G^T A (rows p, q)
          const double apk = a[p][k], aqk = a[q][k];
          a[p][k] = c * apk - s * aqk;
          a[q][k] = s * apk + c * aqk;
        }
      }
    }
  }
  ev[0] = a[0][0]; ev[1] = a[1][1]; ev[2] = a[2][2];
  std::sort(ev, ev + 3, [](double u, double v) { return u > v; });
}

// per-(Gaussian, view) record layout of the double arrays handed back to Python
enum SplatField {
  F_MX = 0, F_MY, F_QA, F_QB, F_QC, F_DEPTH, F_OPAC, F_C0, F_C1, F_C2,
  F_XC, F_YC, F_ZC, F_CMASK, F_TILES, F_NFIELDS = 16
};
constexpr int ACC_N = 8;  // q, Swr(3), Sa, Sd(2), pixel count
constexpr int NB = 16;    // max SH basis size (degree 3)

// ------------------------------------------------------------------------------------------
// Projection of one Gaussian into one view (3DGS EWA splatting; [P1] Stage 1 "original gsplat";
// [P1] "Projected-Center Mean Partial Score" defines G with Sigma2D; [P5] 3DGS primitive).
// Returns false when the Gaussian is culled in this view.
// ------------------------------------------------------------------------------------------
template <typename R>
bool project_one(const float* mean, const float* lsc, const float* quat, float opac_logit,
                 const float* sh, int deg, const float* vm, const float* K, int H, int W,
                 double* rec, int* rect, double* Bout) {
  for (int i = 0; i < 3; ++i)
    if (!std::isfinite(mean[i]) || !std::isfinite(lsc[i])) return false;
  for (int i = 0; i < 4; ++i)
    if (!std::isfinite(quat[i])) return false;
  if (!std::isfinite(opac_logit)) return false;

  const R m0 = mean[0], m1 = mean[1], m2 = mean[2];
  R Rv[3][3], t[3];
  for (int i = 0; i < 3; ++i) {
    for (int j = 0; j < 3; ++j) Rv[i][j] = vm[4 * i + j];
    t[i] = vm[4 * i + 3];
  }
  const R fx = K[0], fy = K[1], cx = K[2], cy = K[3];

  // camera-space centre x_c = R_v mu + t_v
  R xc[3];
  for (int i = 0; i < 3; ++i) xc[i] = Rv[i][0] * m0 + Rv[i][1] * m1 + Rv[i][2] * m2 + t[i];
  const R x = xc[0], y = xc[1], z = xc[2];
  if (!(z > (R)0.01)) return false;  // near plane

  // rotation from the normalised quaternion (w, x, y, z)
  R qw = quat[0], qx = quat[1], qy = quat[2], qz = quat[3];
  const R n2 = qw * qw + qx * qx + qy * qy + qz * qz;
  if (!(n2 > (R)0)) return false;
  const R inv = (R)1 / rsqrt_ieee(n2);
  qw = qw * inv; qx = qx * inv; qy = qy * inv; qz = qz * inv;
  R Rq[3][3];
  Rq[0][0] = (R)1 - (R)2 * (qy * qy + qz * qz);
  Rq[0][1] = (R)2 * (qx * qy - qw * qz);
  Rq[0][2] = (R)2 * (qx * qz + qw * qy);
  Rq[1][0] = (R)2 * (qx * qy + qw * qz);
  Rq[1][1] = (R)1 - (R)2 * (qx * qx + qz * qz);
  Rq[1][2] = (R)2 * (qy * qz - qw * qx);
  Rq[2][0] = (R)2 * (qx * qz - qw * qy);
  Rq[2][1] = (R)2 * (qy * qz + qw * qx);
  Rq[2][2] = (R)1 - (R)2 * (qx * qx + qy * qy);

  // Sigma3D = (Rq S)(Rq S)^T, S = diag(exp(log_scale))
  R S[3];
  for (int i = 0; i < 3; ++i) S[i] = rexp((R)lsc[i]);
  R M[3][3];
  for (int i = 0; i < 3; ++i)
    for (int j = 0; j < 3; ++j) M[i][j] = Rq[i][j] * S[j];
  R Sw[3][3];
  for (int i = 0; i < 3; ++i)
    for (int j = 0; j < 3; ++j) Sw[i][j] = M[i][0] * M[j][0] + M[i][1] * M[j][1] + M[i][2] * M[j][2];

  // camera-frame covariance R_v Sigma3D R_v^T
  R T1[3][3], Sc[3][3];
  for (int i = 0; i < 3; ++i)
    for (int j = 0; j < 3; ++j) T1[i][j] = Rv[i][0] * Sw[0][j] + Rv[i][1] * Sw[1][j] + Rv[i][2] * Sw[2][j];
  for (int i = 0; i < 3; ++i)
    for (int j = 0; j < 3; ++j) Sc[i][j] = T1[i][0] * Rv[j][0] + T1[i][1] * Rv[j][1] + T1[i][2] * Rv[j][2];

  // EWA: local affine approximation of the perspective projection at the centre; the tangent
  // (x/z, y/z) entering the covariance Jacobian is clamped to 1.3x the half field of view
  const R u = x / z, v = y / z;
  const R limx = (R)1.3 * (((R)0.5 * (R)W) / fx);
  const R limy = (R)1.3 * (((R)0.5 * (R)H) / fy);
  const R uc = std::min(limx, std::max(-limx, u));
  const R vc = std::min(limy, std::max(-limy, v));
  const R J00 = fx / z, J02 = -(fx * uc) / z;
  const R J11 = fy / z, J12 = -(fy * vc) / z;
  // T = J Sc (rows 0 and 1), Sigma2D = T J^T + 0.3 I
  R T0[3], Tr1[3];
  for (int k = 0; k < 3; ++k) {
    T0[k] = J00 * Sc[0][k] + J02 * Sc[2][k];
    Tr1[k] = J11 * Sc[1][k] + J12 * Sc[2][k];
  }
  R a = T0[0] * J00 + T0[2] * J02;
  const R b = T0[1] * J11 + T0[2] * J12;
  R c = Tr1[1] * J11 + Tr1[2] * J12;
  a = a + (R)0.3;
  c = c + (R)0.3;
  const R det = a * c - b * b;
  if (!(det > (R)0)) return false;
  const R qa = c / det, qb = -b / det, qc = a / det;  // conic = Sigma2D^{-1}

  // footprint: 3 sigma of the major axis, in whole pixels
  const R mid = (R)0.5 * (a + c);
  const R lam = mid + rsqrt_ieee(std::max((R)0.1, mid * mid - det));
  const R rr = std::ceil((R)3 * rsqrt_ieee(lam));
  if (!(rr > (R)0)) return false;

  const R mx = fx * u + cx, my = fy * v + cy;  // projected centre in pixels

  // tile rectangle [x0, x1) x [y0, y1) of 16x16 tiles overlapped by the footprint square
  const int TX = (W + TILE - 1) / TILE, TY = (H + TILE - 1) / TILE;
  auto clampt = [](R val, int hi) -> int {
    if (!(val > (R)0)) return 0;  // also maps NaN to 0
    if (val > (R)hi) return hi;
    return (int)val;
  };
  const int x0 = clampt(std::floor((mx - rr) / (R)TILE), TX);
  const int x1 = clampt(std::floor((mx + rr) / (R)TILE) + (R)1, TX);
  const int y0 = clampt(std::floor((my - rr) / (R)TILE), TY);
  const int y1 = clampt(std::floor((my + rr) / (R)TILE) + (R)1, TY);
  if (x1 <= x0 || y1 <= y0) return false;

  // opacity o = sigmoid(a) ([P1] "Exact Score Operators")
  const R o = (R)1 / ((R)1 + rexp(-(R)opac_logit));

  // view direction (world) and SH colour c = max(0, B(d) . sh + 0.5)
  R cam[3];
  for (int i = 0; i < 3; ++i) cam[i] = -(Rv[0][i] * t[0] + Rv[1][i] * t[1] + Rv[2][i] * t[2]);
  R dv[3] = {m0 - cam[0], m1 - cam[1], m2 - cam[2]};
  const R len = rsqrt_ieee(dv[0] * dv[0] + dv[1] * dv[1] + dv[2] * dv[2]);
  double dird[3];
  for (int i = 0; i < 3; ++i) dird[i] = (double)(dv[i] / len);
  double Bd[NB];
  sh_basis_def(deg, dird, Bd);
  const int d = (deg + 1) * (deg + 1);
  R B[NB];
  for (int k = 0; k < d; ++k) B[k] = (R)Bd[k];
  R col[3];
  int cmask = 0;
  for (int ch = 0; ch < 3; ++ch) {
    R s = (R)0;
    for (int k = 0; k < d; ++k) s = s + B[k] * (R)sh[3 * k + ch];
    s = s + (R)0.5;
    if (s > (R)0) cmask |= 1 << ch;
    col[ch] = std::max(s, (R)0);
  }

  rec[F_MX] = mx; rec[F_MY] = my;
  rec[F_QA] = qa; rec[F_QB] = qb; rec[F_QC] = qc;
  rec[F_DEPTH] = z; rec[F_OPAC] = o;
  rec[F_C0] = col[0]; rec[F_C1] = col[1]; rec[F_C2] = col[2];
  rec[F_XC] = x; rec[F_YC] = y; rec[F_ZC] = z;
  rec[F_CMASK] = cmask;
  rec[F_TILES] = (double)((x1 - x0) * (y1 - y0));
  rect[0] = x0; rect[1] = y0; rect[2] = x1; rect[3] = y1;
  for (int k = 0; k < NB; ++k) Bout[k] = k < d ? (double)B[k] : 0.0;
  return true;
}

template <typename R>
int project_all(const float* means, const float* lsc, const float* quats, const float* opac,
                const float* sh, int G, int deg, const float* viewmats, const float* intrin,
                int V, int H, int W, int* valid, double* rec, int* rect, double* B) {
  const int d = (deg + 1) * (deg + 1);
  long long total = (long long)G * V;
#pragma omp parallel for schedule(static)
  for (long long i = 0; i < total; ++i) {
    const int v = (int)(i / G), g = (int)(i % G);
    double* r = rec + i * F_NFIELDS;
    int* rc = rect + i * 4;
    double* b = B + i * NB;
    std::fill(r, r + F_NFIELDS, 0.0);
    std::fill(rc, rc + 4, 0);
    std::fill(b, b + NB, 0.0);
    valid[i] = project_one<R>(means + 3 * g, lsc + 3 * g, quats + 4 * g, opac[g],
                              sh + (long long)g * d * 3, deg, viewmats + 16 * v, intrin + 4 * v,
                              H, W, r, rc, b) ? 1 : 0;
  }
  return 0;
}

// ------------------------------------------------------------------------------------------
// One pixel's front-to-back traversal of its tile list ([P1] Stage 1 step 2 and Stage 2).
// The per-entry decisions (skip when the exponent is positive or alpha < 1/255, alpha clamped
// at 0.99, stop before an entry that would take T below 1e-4) follow the 3DGS tile
// rasteriser. The same routine drives the render and the replay so that both take exactly the
// same decisions.
// ------------------------------------------------------------------------------------------
template <typename R>
struct EntryEval {
  bool use;   // passes the positive-exponent and 1/255 tests
  R alpha;    // min(0.99, o G)
  R dx, dy;   // p - mu2D
};

template <typename R>
inline EntryEval<R> eval_entry(const double* rec, R px, R py) {
  EntryEval<R> e;
  const R mx = (R)rec[F_MX], my = (R)rec[F_MY];
  const R qa = (R)rec[F_QA], qb = (R)rec[F_QB], qc = (R)rec[F_QC];
  const R o = (R)rec[F_OPAC];
  e.dx = px - mx;
  e.dy = py - my;
  // exponent of G: -1/2 d^T Sigma2D^{-1} d
  const R t1 = qa * e.dx * e.dx;
  const R t2 = qc * e.dy * e.dy;
  const R t3 = qb * e.dx * e.dy;
  const R pw = (R)(-0.5) * (t1 + t2) - t3;
  e.use = false;
  e.alpha = (R)0;
  if (pw > (R)0) return e;
  const R al = std::min((R)0.99, o * rexp(pw));
  if (al < (R)1 / (R)255) return e;
  e.alpha = al;
  e.use = true;
  return e;
}

struct Lists {
  const long long* off;  // [V, n_t + 1]
  const int* ids;
};

template <typename R>
void render_pixel(const double* rec_v, const Lists& L, long long ofs_base, int n_t, int tile,
                  int i, int j, const R bg[3], double* img, double* Tout, int* nc, int* last,
                  long long* evaluated) {
  const long long s = L.off[ofs_base + tile], e = L.off[ofs_base + tile + 1];
  const R px = (R)i + (R)0.5, py = (R)j + (R)0.5;
  R T = (R)1;
  R C[3] = {0, 0, 0};
  int n = 0, lst = 0;
  long long ev = 0;
  for (long long k = s; k < e; ++k) {
    ++ev;
    const double* rec = rec_v + (long long)L.ids[k] * F_NFIELDS;
    EntryEval<R> E = eval_entry<R>(rec, px, py);
    if (!E.use) continue;
    const R Tn = T * ((R)1 - E.alpha);
    if (Tn < (R)1e-4) break;  // stop before compositing this entry
    const R w = E.alpha * T;
    for (int ch = 0; ch < 3; ++ch) C[ch] = C[ch] + w * (R)rec[F_C0 + ch];
    T = Tn;
    ++n;
    lst = (int)(k - s) + 1;
  }
  (void)n_t;
  for (int ch = 0; ch < 3; ++ch) img[ch] = (double)(C[ch] + T * bg[ch]);
  *Tout = (double)T;
  *nc = n;
  *last = lst;
  *evaluated = ev;
}

// Stage 2 replay of one pixel ([P1] "Stage 2: Analytic Score Replay" and "Exact Score
// Operators"): prefix colour P and transmittance T, suffix composite
//   C+ = (C_hat - P - T alpha c) / (T (1 - alpha) + eps),
// masks M_alpha (denominator >= 1e-4 and alpha not clamped at 0.99) and M_color (colour clamp not
// active), rho = <r, c - C+>, w = T alpha, r = C_hat - C_obs. Per (Gaussian, view) it adds
//   q += w, Swr += w r, and where M_alpha: Sa += w rho, Sd += w rho (p - mu2D),
// from which the finaliser forms the opacity-logit score (1 - o) Sa, the SH score
// M_color (Swr (x) B) and the projected-centre score Sigma2D^{-1} Sd (o grad G = alpha Sigma^{-1} d
// when alpha = o G is not clamped). When `sh_lit` is given, it also accumulates the SH score
// literally per pixel as M_color w [B (x) r] (the form printed in "SH Score").
template <typename R>
void replay_pixel(const double* rec_v, const double* B_v, int d, const Lists& L,
                  long long ofs_base, int tile, int i, int j, const double* chat_d,
                  const float* obs, int lst, double* acc_v, double* shlit_v) {
  const long long s = L.off[ofs_base + tile];
  const R px = (R)i + (R)0.5, py = (R)j + (R)0.5;
  R Ch[3], r[3];
  for (int ch = 0; ch < 3; ++ch) {
    Ch[ch] = (R)chat_d[ch];
    r[ch] = Ch[ch] - (R)obs[ch];
  }
  R T = (R)1;
  R P[3] = {0, 0, 0};
  const R eps = (R)1e-12;
  for (long long k = s; k < s + lst; ++k) {
    const int g = L.ids[k];
    const double* rec = rec_v + (long long)g * F_NFIELDS;
    EntryEval<R> E = eval_entry<R>(rec, px, py);
    if (!E.use) continue;
    const R al = E.alpha;
    const R den = T * ((R)1 - al);
    const R w = al * T;
    R c[3], Cp[3];
    for (int ch = 0; ch < 3; ++ch) {
      c[ch] = (R)rec[F_C0 + ch];
      Cp[ch] = ((Ch[ch] - P[ch]) - w * c[ch]) / (den + eps);
    }
    const bool Ma = (den >= (R)1e-4) && (al < (R)0.99);
    R rho = (R)0;
    for (int ch = 0; ch < 3; ++ch) rho = rho + r[ch] * (c[ch] - Cp[ch]);
    double* a = acc_v + (long long)g * ACC_N;
    const double wd = (double)w;
#pragma omp atomic
    a[0] += wd;
    for (int ch = 0; ch < 3; ++ch) {
      const double v = (double)w * (double)r[ch];
#pragma omp atomic
      a[1 + ch] += v;
    }
    if (Ma) {
      const double wr = (double)w * (double)rho;
#pragma omp atomic
      a[4] += wr;
      const double sx = wr * (double)E.dx, sy = wr * (double)E.dy;
#pragma omp atomic
      a[5] += sx;
#pragma omp atomic
      a[6] += sy;
    }
#pragma omp atomic
    a[7] += 1.0;
    if (shlit_v) {
      const int cm = (int)rec[F_CMASK];
      const double* Bg = B_v + (long long)g * NB;
      double* sl = shlit_v + (long long)g * NB * 3;
      for (int k2 = 0; k2 < d; ++k2)
        for (int ch = 0; ch < 3; ++ch) {
          if (!((cm >> ch) & 1)) continue;
          const double v = (double)w * Bg[k2] * (double)r[ch];
#pragma omp atomic
          sl[3 * k2 + ch] += v;
        }
    }
    for (int ch = 0; ch < 3; ++ch) P[ch] = P[ch] + w * c[ch];
    T = den;
  }
}


// ------------------------------------------------------------------------------------------
// Gradient of the SH basis with respect to the view direction, for the renderer backward.
// On the unit sphere each real SH function is a polynomial in (x, y, z):
//   B_lm = N_lm (-1)^m [d^|m| P_l / dz^|m|](z) A_m(x, y),
//   A_m = Re (x + i y)^m (m > 0), Im (x + i y)^|m| (m < 0), 1 (m = 0),
// since (1 - z^2)^{m/2} e^{i m phi} = (x + i y)^m there (the associated Legendre function with
// the Condon-Shortley phase is (-1)^m (1 - z^2)^{m/2} d^m P_l / dz^m). N_lm is the normalisation
// of sh_basis_def (times sqrt 2 for m != 0). The Legendre polynomial coefficients come from
// Bonnet's recurrence (n + 1) P_{n+1} = (2n + 1) z P_n - n P_{n-1}. This extension off the sphere
// is differentiated by hand (product rule); the caller projects the gradient onto the tangent
// plane, which removes any dependence on how the basis is extended off the sphere.
// ------------------------------------------------------------------------------------------
void sh_poly_grad_def(int deg, const double dir[3], double* B, double (*dB)[3]) {
  const double x = dir[0], y = dir[1], z = dir[2];
  double Pc[5][5] = {{0}};  // Pc[l][k]: coefficient of z^k in P_l
  Pc[0][0] = 1.0;
  Pc[1][1] = 1.0;
  for (int n = 1; n + 1 <= 4; ++n)
    for (int k = 0; k <= n + 1; ++k)
      Pc[n + 1][k] = ((2.0 * n + 1.0) * (k > 0 ? Pc[n][k - 1] : 0.0) - n * Pc[n - 1][k]) / (n + 1.0);
  // D^m P_l evaluated at z, for m = 0..l+1
  auto dpoly = [&](int l, int m) {
    double v = 0.0;
    for (int k = m; k <= l; ++k) {
      double c = Pc[l][k];
      for (int t = 0; t < m; ++t) c *= (double)(k - t);
      v += c * std::pow(z, k - m);
    }
    return v;
  };
  auto fact = [](int n) { double f = 1; for (int i = 2; i <= n; ++i) f *= i; return f; };
  // (x + i y)^m and its x-derivative m (x + i y)^{m-1} (the y-derivative is i times that)
  double re[5], im[5];
  re[0] = 1.0; im[0] = 0.0;
  for (int m = 1; m <= 4; ++m) {
    re[m] = re[m - 1] * x - im[m - 1] * y;
    im[m] = re[m - 1] * y + im[m - 1] * x;
  }
  for (int l = 0; l <= deg; ++l) {
    for (int m = -l; m <= l; ++m) {
      const int am = m < 0 ? -m : m;
      double N = std::sqrt((2.0 * l + 1.0) / (4.0 * M_PI) * fact(l - am) / fact(l + am));
      if (am) N *= std::sqrt(2.0);
      if (am & 1) N = -N;
      double A, Ax, Ay;
      if (m == 0) { A = 1.0; Ax = 0.0; Ay = 0.0; }
      else if (m > 0) { A = re[am]; Ax = am * re[am - 1]; Ay = -am * im[am - 1]; }
      else { A = im[am]; Ax = am * im[am - 1]; Ay = am * re[am - 1]; }
      const double Dm = dpoly(l, am), Dm1 = dpoly(l, am + 1);
      const int k = l * l + l + m;
      B[k] = N * Dm * A;
      dB[k][0] = N * Dm * Ax;
      dB[k][1] = N * Dm * Ay;
      dB[k][2] = N * Dm1 * A;
    }
  }
}

// ------------------------------------------------------------------------------------------
// Renderer backward of one pixel: derivatives of L = 1/2 sum_p |C_hat_p - C_obs_p|^2 ("Relation
// to Gradient": the raw gradient the score tokens are compared with; RGB squared loss as in
// "Exact Score Operators"), with the contributor order, the skip decisions, the early stop and
// the clamp decisions held fixed. With the composited entries i = 1..n,
//   C_hat = sum_i T_i alpha_i c_i + T_{n+1} bg,   T_{i+1} = T_i (1 - alpha_i),
//   d C_hat / d c_i = T_i alpha_i,
//   d C_hat / d alpha_i = T_i c_i - S_i / (1 - alpha_i),  S_i = sum_{j>i} T_j alpha_j c_j + T_{n+1} bg,
// the suffix S_i being summed back to front (its definition; no recovery equation). With
// ga_i = <r, d C_hat / d alpha_i> and, where alpha = o G is not clamped, d alpha = alpha d(pw) +
// G d o with pw = -1/2 d^T Q d, d = p - mu2D, Q the conic, the pixel adds to its (Gaussian, view)
//   q += w, Swr += w r (w = T alpha), and with h = ga alpha:  H += h, Hd += h d (2),
//   Hdd += h (dx^2, dx dy, dy^2),
// from which the per-Gaussian chain forms every parameter's derivative. T_i are products of
// (1 - alpha) in double.
// ------------------------------------------------------------------------------------------
constexpr int ACCB_N = 10;  // q, Swr(3), H, Hdx, Hdy, Hdxdx, Hdxdy, Hdydy

template <typename R>
void backward_pixel(const double* rec_v, const Lists& L, long long ofs_base, int tile, int i,
                    int j, const double* chat, const float* obs, const float* bg, int lst,
                    double* accb_v) {
  const long long s = L.off[ofs_base + tile];
  const R px = (R)i + (R)0.5, py = (R)j + (R)0.5;
  double r[3];
  for (int ch = 0; ch < 3; ++ch) r[ch] = chat[ch] - (double)obs[ch];
  struct Hit { int g; double al, dx, dy; };
  std::vector<Hit> hits;
  for (long long k = s; k < s + lst; ++k) {
    const int g = L.ids[k];
    EntryEval<R> E = eval_entry<R>(rec_v + (long long)g * F_NFIELDS, px, py);
    if (E.use) hits.push_back({g, (double)E.alpha, (double)E.dx, (double)E.dy});
  }
  const int n = (int)hits.size();
  std::vector<double> T(n + 1);
  T[0] = 1.0;
  for (int k = 0; k < n; ++k) T[k + 1] = T[k] * (1.0 - hits[k].al);
  double S[3];
  for (int ch = 0; ch < 3; ++ch) S[ch] = T[n] * (double)bg[ch];
  for (int k = n - 1; k >= 0; --k) {
    const Hit& e = hits[k];
    const double* rec = rec_v + (long long)e.g * F_NFIELDS;
    const double w = T[k] * e.al;
    double ga = 0.0;
    for (int ch = 0; ch < 3; ++ch) ga += r[ch] * (T[k] * rec[F_C0 + ch] - S[ch] / (1.0 - e.al));
    double* a = accb_v + (long long)e.g * ACCB_N;
    double add[ACCB_N] = {w, w * r[0], w * r[1], w * r[2], 0, 0, 0, 0, 0, 0};
    if (e.al < 0.99) {
      const double h = ga * e.al;
      add[4] = h;
      add[5] = h * e.dx;
      add[6] = h * e.dy;
      add[7] = h * e.dx * e.dx;
      add[8] = h * e.dx * e.dy;
      add[9] = h * e.dy * e.dy;
    }
    for (int q = 0; q < ACCB_N; ++q) {
#pragma omp atomic
      a[q] += add[q];
    }
    for (int ch = 0; ch < 3; ++ch) S[ch] += w * rec[F_C0 + ch];
  }
}


// ------------------------------------------------------------------------------------------
// Per-Gaussian attributes composited with the render's weights -- the multi-channel /
// scalar-attribute render (learned feature channels rendered beside RGB, as in "ReCoSplat"
// section 2.1; a per-Gaussian uncertainty score rendered by alpha compositing into a map, as in
// "ATSplat", core method) -- and its transpose, the scatter of a per-pixel map back to the
// Gaussians with the same weights (the mask-channel back-projection of a 2D gain, "L2D2-GS"
// method; with a map of ones the alphaT coverage, with the residual norm the PRIMU-style error of
// "Relation to Gradient" / "Novelty Boundary"):
//   F_p = sum_i w_i f_{g_i},      s_g = sum_p sum_{i: g_i = g} w_i m_p,      w = T alpha,
// over the entries render_pixel composited (same decisions; no background term for attributes).
// ------------------------------------------------------------------------------------------
template <typename R>
void pixel_weights(const double* rec_v, const Lists& L, long long ofs_base, int tile, int i,
                   int j, int lst, std::vector<std::pair<int, R>>& out) {
  out.clear();
  const long long s = L.off[ofs_base + tile];
  const R px = (R)i + (R)0.5, py = (R)j + (R)0.5;
  R T = (R)1;
  for (long long k = s; k < s + lst; ++k) {
    const int g = L.ids[k];
    EntryEval<R> E = eval_entry<R>(rec_v + (long long)g * F_NFIELDS, px, py);
    if (!E.use) continue;
    out.push_back({g, E.alpha * T});
    T = T * ((R)1 - E.alpha);
  }
}

}  // namespace

// ==========================================================================================
// C entry points (ctypes). Arrays are C-contiguous; `_f` = fp32 working precision, `_d` = fp64.
// ==========================================================================================
extern "C" {

float orc_exp_f(float x) { return exp_cw(x); }

void orc_exp_f_vec(const float* x, float* y, long long n) {
  for (long long i = 0; i < n; ++i) y[i] = exp_cw(x[i]);
}

void orc_sh_basis(int deg, const double* dirs, long long n, double* out) {
  for (long long i = 0; i < n; ++i) {
    double tmp[NB] = {0};
    sh_basis_def(deg, dirs + 3 * i, tmp);
    for (int k = 0; k < NB; ++k) out[i * NB + k] = tmp[k];
  }
}

void orc_eig3(const double* A, long long n, double* ev) {
  for (long long i = 0; i < n; ++i) eig3_jacobi(A + 9 * i, ev + 3 * i);
}

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void orc_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

#define ORC_PROJECT(SUF, R)                                                                     \
  int orc_project_##SUF(const float* means, const float* lsc, const float* quats,             \
                        const float* opac, const float* sh, int G, int deg,                   \
                        const float* viewmats, const float* intrin, int V, int H, int W,      \
                        int* valid, double* rec, int* rect, double* B) {                      \
    if (G < 0 || V < 0 || H <= 0 || W <= 0 || deg < 0 || deg > 3) return -1;                   \
    return project_all<R>(means, lsc, quats, opac, sh, G, deg, viewmats, intrin, V, H, W,     \
                          valid, rec, rect, B);                                               \
  }
ORC_PROJECT(f, float)
ORC_PROJECT(d, double)

// Tile binning and contributor order ([P1] Stage 1 step 1): every visible Gaussian is listed in
// each tile of its rectangle; each tile's list is sorted by (depth, Gaussian index). This uses a
// comparison sort per tile (std::sort), not the GPU's algorithm. `off` must hold V * (n_t + 1)
// entries; when `ids` is null only the counts/offsets are produced.
long long orc_bin(const int* valid, const double* rec, const int* rect, int G, int V, int H,
                  int W, long long* off, int* ids) {
  const int TX = (W + TILE - 1) / TILE, TY = (H + TILE - 1) / TILE, nt = TX * TY;
  long long total = 0;
  for (int v = 0; v < V; ++v) {
    std::vector<std::vector<int>> lists(nt);
    for (int g = 0; g < G; ++g) {
      const long long i = (long long)v * G + g;
      if (!valid[i]) continue;
      const int* rc = rect + 4 * i;
      for (int ty = rc[1]; ty < rc[3]; ++ty)
        for (int tx = rc[0]; tx < rc[2]; ++tx) lists[ty * TX + tx].push_back(g);
    }
    const double* recv = rec + (long long)v * G * F_NFIELDS;
    long long* o = off + (long long)v * (nt + 1);
    for (int t = 0; t < nt; ++t) {
      auto& l = lists[t];
      std::sort(l.begin(), l.end(), [&](int a, int b) {
        const double da = recv[(long long)a * F_NFIELDS + F_DEPTH];
        const double db = recv[(long long)b * F_NFIELDS + F_DEPTH];
        if (da != db) return da < db;
        return a < b;
      });
      o[t] = total;
      if (ids) std::copy(l.begin(), l.end(), ids + total);
      total += (long long)l.size();
    }
    o[nt] = total;
  }
  return total;
}

// Render the listed (view, tile) pairs (all tiles when n_sel < 0). Outputs are [V, H, W(, 3)];
// only pixels of the selected tiles are written. Returns the number of evaluated entries.
#define ORC_RENDER(SUF, R)                                                                      \
  long long orc_render_##SUF(const double* rec, const long long* off, const int* ids, int G,   \
                             int V, int H, int W, const float* bg, const int* sel, int n_sel, \
                             double* img, double* Tf, int* nc, int* last) {                   \
    const int TX = (W + TILE - 1) / TILE, TY = (H + TILE - 1) / TILE, nt = TX * TY;            \
    const long long nsel = n_sel < 0 ? (long long)V * nt : n_sel;                               \
    Lists L{off, ids};                                                                          \
    const R bgr[3] = {(R)bg[0], (R)bg[1], (R)bg[2]};                                            \
    long long evaluated = 0;                                                                    \
    _Pragma("omp parallel for schedule(dynamic, 1) reduction(+ : evaluated)")                  \
    for (long long s = 0; s < nsel; ++s) {                                                      \
      const int v = n_sel < 0 ? (int)(s / nt) : sel[2 * s];                                     \
      const int t = n_sel < 0 ? (int)(s % nt) : sel[2 * s + 1];                                 \
      const int tx = t % TX, ty = t / TX;                                                       \
      const double* recv = rec + (long long)v * G * F_NFIELDS;                                  \
      for (int j = ty * TILE; j < std::min(H, ty * TILE + TILE); ++j)                           \
        for (int i = tx * TILE; i < std::min(W, tx * TILE + TILE); ++i) {                       \
          const long long p = ((long long)v * H + j) * W + i;                                   \
          long long ev = 0;                                                                     \
          render_pixel<R>(recv, L, (long long)v * (nt + 1), nt, t, i, j, bgr, img + 3 * p,    \
                          Tf + p, nc + p, last + p, &ev);                                       \
          evaluated += ev;                                                                      \
        }                                                                                       \
    }                                                                                           \
    return evaluated;                                                                           \
  }
ORC_RENDER(f, float)
ORC_RENDER(d, double)

// Replay the listed (view, tile) pairs, adding into acc [V, G, 8] (q, Swr[3], Sa, Sd[2], npix)
// and, when sh_lit is non-null, into sh_lit [V, G, 16, 3].
#define ORC_REPLAY(SUF, R)                                                                      \
  int orc_replay_##SUF(const double* rec, const double* B, int deg, const long long* off,      \
                       const int* ids, int G, int V, int H, int W, const double* chat,         \
                       const float* obs, const int* last, const int* sel, int n_sel,           \
                       double* acc, double* sh_lit) {                                           \
    const int TX = (W + TILE - 1) / TILE, TY = (H + TILE - 1) / TILE, nt = TX * TY;            \
    const int d = (deg + 1) * (deg + 1);                                                        \
    const long long nsel = n_sel < 0 ? (long long)V * nt : n_sel;                               \
    Lists L{off, ids};                                                                          \
    _Pragma("omp parallel for schedule(dynamic, 1)")                                           \
    for (long long s = 0; s < nsel; ++s) {                                                      \
      const int v = n_sel < 0 ? (int)(s / nt) : sel[2 * s];                                     \
      const int t = n_sel < 0 ? (int)(s % nt) : sel[2 * s + 1];                                 \
      const int tx = t % TX, ty = t / TX;                                                       \
      const double* recv = rec + (long long)v * G * F_NFIELDS;                                  \
      const double* Bv = B + (long long)v * G * NB;                                             \
      double* accv = acc + (long long)v * G * ACC_N;                                            \
      double* slv = sh_lit ? sh_lit + (long long)v * G * NB * 3 : nullptr;                      \
      for (int j = ty * TILE; j < std::min(H, ty * TILE + TILE); ++j)                           \
        for (int i = tx * TILE; i < std::min(W, tx * TILE + TILE); ++i) {                       \
          const long long p = ((long long)v * H + j) * W + i;                                   \
          replay_pixel<R>(recv, Bv, d, L, (long long)v * (nt + 1), t, i, j, chat + 3 * p,     \
                          obs + 3 * p, last[p], accv, slv);                                     \
        }                                                                                       \
    }                                                                                           \
    return 0;                                                                                   \
  }
ORC_REPLAY(f, float)
ORC_REPLAY(d, double)

// Per-pixel trace for the suffix check: for the composited entries of pixel (i, j) in view v,
// writes [g, alpha, T (before the entry), c(3), C+(3) by the suffix equation, T (1 - alpha)]
// (double, [n, 10]); returns the number of composited entries (at most cap).
#define ORC_TRACE(SUF, R)                                                                       \
  int orc_trace_##SUF(const double* rec, const long long* off, const int* ids, int G, int V,   \
                      int H, int W, const float* bg, int v, int i, int j, int cap,             \
                      double* out) {                                                            \
    (void)V;                                                                                    \
    const int TX = (W + TILE - 1) / TILE, TY = (H + TILE - 1) / TILE, nt = TX * TY;            \
    (void)TY;                                                                                   \
    const int t = (j / TILE) * TX + (i / TILE);                                                 \
    const double* recv = rec + (long long)v * G * F_NFIELDS;                                    \
    Lists L{off, ids};                                                                          \
    const R bgr[3] = {(R)bg[0], (R)bg[1], (R)bg[2]};                                            \
    double img[3], Tf;                                                                          \
    int nc, lst;                                                                                \
    long long ev;                                                                               \
    render_pixel<R>(recv, L, (long long)v * (nt + 1), nt, t, i, j, bgr, img, &Tf, &nc, &lst,  \
                    &ev);                                                                       \
    const long long s = off[(long long)v * (nt + 1) + t];                                       \
    const R px = (R)i + (R)0.5, py = (R)j + (R)0.5;                                             \
    R T = 1, P[3] = {0, 0, 0};                                                                  \
    int n = 0;                                                                                  \
    for (long long k = s; k < s + lst && n < cap; ++k) {                                        \
      const int g = ids[k];                                                                     \
      const double* rc = recv + (long long)g * F_NFIELDS;                                       \
      EntryEval<R> E = eval_entry<R>(rc, px, py);                                               \
      if (!E.use) continue;                                                                     \
      const R den = T * ((R)1 - E.alpha), w = E.alpha * T;                                      \
      double* o = out + 10 * n;                                                                 \
      o[0] = g; o[1] = E.alpha; o[2] = T; o[9] = den;                                           \
      for (int ch = 0; ch < 3; ++ch) {                                                          \
        const R c = (R)rc[F_C0 + ch];                                                           \
        o[3 + ch] = c;                                                                          \
        o[6 + ch] = (((R)img[ch] - P[ch]) - w * c) / (den + (R)1e-12);                          \
        P[ch] = P[ch] + w * c;                                                                  \
      }                                                                                         \
      T = den;                                                                                  \
      ++n;                                                                                      \
    }                                                                                           \
    return n;                                                                                   \
  }
ORC_TRACE(f, float)
ORC_TRACE(d, double)

// Token finalisation ([P1] "Exact Score Operators": projection Jacobian, cross-view weights,
// covector pullback, conditioning matrix and statistics, cross-view appearance, "Final Token and
// Updater"). Always evaluated in double from the per-(Gaussian, view) sums.
//   q_gv = eps + sum_p w,  q_g = eps + sum_v q_gv,  gamma_gv = q_gv / q_g
//   s^alpha_gv = (1 - o) Sa / q_gv;  s^SH_gv = M_color (Swr (x) B) / q_gv;
//   s^mu2D_gv = Sigma2D^{-1} Sd / q_gv;  J_gv = d pi_v(mu) / d mu (unclamped)
//   b = sum_v gamma J^T s^mu2D;  s^alpha = sum_v gamma s^alpha_gv;  s^SH likewise
//   A = lambda I + sum_v gamma J^T J;  e~ = eig(A) (descending) / (tr A + eps);
//   l = log(tr A + eps);  z = [b(3), s^alpha, s^SH (k-major, channel-minor), log q_g, e~(3), l]
// Views in which the Gaussian is culled contribute nothing.
int orc_finalize(const int* valid, const double* rec, const double* B, const double* acc,
                 const float* viewmats, const float* intrin, int G, int V, int deg,
                 double lambda, double* tokens) {
  const int d = (deg + 1) * (deg + 1);
  const int D = 9 + 3 * d;
  const double eps = 1e-6;
#pragma omp parallel for schedule(static)
  for (int g = 0; g < G; ++g) {
    double qsum = 0.0;
    for (int v = 0; v < V; ++v) {
      const long long i = (long long)v * G + g;
      if (valid[i]) qsum += eps + acc[i * ACC_N + 0];
    }
    const double qg = eps + qsum;
    double bmu[3] = {0, 0, 0}, sa = 0.0, ssh[NB * 3] = {0}, A[9] = {0};
    for (int v = 0; v < V; ++v) {
      const long long i = (long long)v * G + g;
      if (!valid[i]) continue;
      const double* a = acc + i * ACC_N;
      const double* rc = rec + i * F_NFIELDS;
      const double qgv = eps + a[0];
      const double gam = qgv / qg;
      const double o = rc[F_OPAC];
      const double s_alpha = (1.0 - o) * a[4] / qgv;
      const double smu[2] = {(rc[F_QA] * a[5] + rc[F_QB] * a[6]) / qgv,
                             (rc[F_QB] * a[5] + rc[F_QC] * a[6]) / qgv};
      const int cm = (int)rc[F_CMASK];
      const double* Bg = B + i * NB;
      for (int k = 0; k < d; ++k)
        for (int ch = 0; ch < 3; ++ch)
          if ((cm >> ch) & 1) ssh[3 * k + ch] += gam * a[1 + ch] * Bg[k] / qgv;
      // J = J_cam(x_c) R_v, J_cam = [[fx/z, 0, -fx x/z^2], [0, fy/z, -fy y/z^2]]
      const float* vm = viewmats + 16 * v;
      const double fx = intrin[4 * v], fy = intrin[4 * v + 1];
      const double x = rc[F_XC], y = rc[F_YC], z = rc[F_ZC];
      const double Jc[2][3] = {{fx / z, 0.0, -fx * x / (z * z)}, {0.0, fy / z, -fy * y / (z * z)}};
      double J[2][3];
      for (int r = 0; r < 2; ++r)
        for (int c = 0; c < 3; ++c)
          J[r][c] = Jc[r][0] * vm[0 * 4 + c] + Jc[r][1] * vm[1 * 4 + c] + Jc[r][2] * vm[2 * 4 + c];
      for (int c = 0; c < 3; ++c) bmu[c] += gam * (J[0][c] * smu[0] + J[1][c] * smu[1]);
      sa += gam * s_alpha;
      for (int r = 0; r < 3; ++r)
        for (int c = 0; c < 3; ++c) A[3 * r + c] += gam * (J[0][r] * J[0][c] + J[1][r] * J[1][c]);
    }
    for (int r = 0; r < 3; ++r) A[4 * r] += lambda;
    double ev[3];
    eig3_jacobi(A, ev);
    const double tr = A[0] + A[4] + A[8];
    double* z = tokens + (long long)g * D;
    z[0] = bmu[0]; z[1] = bmu[1]; z[2] = bmu[2];
    z[3] = sa;
    for (int k = 0; k < 3 * d; ++k) z[4 + k] = ssh[k];
    z[4 + 3 * d] = std::log(qg);
    for (int r = 0; r < 3; ++r) z[5 + 3 * d + r] = ev[r] / (tr + eps);
    z[8 + 3 * d] = std::log(tr + eps);
  }
  return 0;
}


// Per-Gaussian sums over the views in `use_view` (null = all) for view-sharded finalisation
// ([P1] "Exact Score Operators": gamma_gv / q_gv = 1 / q_g makes every block a sum over views
// divided once by q_g). out [G, 11 + 3d] = [sum (eps + q_gv), sum J^T Sigma^-1 Sd (3),
// sum (1 - o) Sa, sum q_gv J^T J (00 01 02 11 12 22), sum M_color Swr (x) B (3d)].
int orc_partials(const int* valid, const double* rec, const double* B, const double* acc,
                 const float* viewmats, const float* intrin, const int* use_view, int G, int V,
                 int deg, double* out) {
  const int d = (deg + 1) * (deg + 1);
  const int K = 11 + 3 * d;
  const double eps = 1e-6;
#pragma omp parallel for schedule(static)
  for (int g = 0; g < G; ++g) {
    double* o = out + (long long)g * K;
    for (int k = 0; k < K; ++k) o[k] = 0.0;
    for (int v = 0; v < V; ++v) {
      const long long i = (long long)v * G + g;
      if (!valid[i] || (use_view && !use_view[v])) continue;
      const double* a = acc + i * ACC_N;
      const double* rc = rec + i * F_NFIELDS;
      const double qgv = eps + a[0];
      o[0] += qgv;
      const double smu[2] = {rc[F_QA] * a[5] + rc[F_QB] * a[6], rc[F_QB] * a[5] + rc[F_QC] * a[6]};
      const float* vm = viewmats + 16 * v;
      const double fx = intrin[4 * v], fy = intrin[4 * v + 1];
      const double x = rc[F_XC], y = rc[F_YC], z = rc[F_ZC];
      const double Jc[2][3] = {{fx / z, 0.0, -fx * x / (z * z)}, {0.0, fy / z, -fy * y / (z * z)}};
      double J[2][3];
      for (int r = 0; r < 2; ++r)
        for (int c = 0; c < 3; ++c)
          J[r][c] = Jc[r][0] * vm[0 * 4 + c] + Jc[r][1] * vm[1 * 4 + c] + Jc[r][2] * vm[2 * 4 + c];
      for (int c = 0; c < 3; ++c) o[1 + c] += J[0][c] * smu[0] + J[1][c] * smu[1];
      o[4] += (1.0 - rc[F_OPAC]) * a[4];
      const int pr[6][2] = {{0, 0}, {0, 1}, {0, 2}, {1, 1}, {1, 2}, {2, 2}};
      for (int e = 0; e < 6; ++e) {
        const int r = pr[e][0], c = pr[e][1];
        o[5 + e] += qgv * (J[0][r] * J[0][c] + J[1][r] * J[1][c]);
      }
      const int cm = (int)rc[F_CMASK];
      const double* Bg = B + i * NB;
      for (int k = 0; k < d; ++k)
        for (int ch = 0; ch < 3; ++ch)
          if ((cm >> ch) & 1) o[11 + 3 * k + ch] += a[1 + ch] * Bg[k];
    }
  }
  return 0;
}

// Tokens from summed partials: q_g = eps + sum (eps + q_gv); every block divided by q_g;
// A = lambda I + (sum q_gv J^T J) / q_g; eigenvalues descending; same layout as orc_finalize.
int orc_finalize_partials(const double* P, int G, int deg, double lambda, double* tokens) {
  const int d = (deg + 1) * (deg + 1);
  const int K = 11 + 3 * d, D = 9 + 3 * d;
  const double eps = 1e-6;
#pragma omp parallel for schedule(static)
  for (int g = 0; g < G; ++g) {
    const double* p = P + (long long)g * K;
    double* z = tokens + (long long)g * D;
    const double qg = eps + p[0];
    for (int c = 0; c < 3; ++c) z[c] = p[1 + c] / qg;
    z[3] = p[4] / qg;
    for (int k = 0; k < 3 * d; ++k) z[4 + k] = p[11 + k] / qg;
    double A[9];
    const int pr[6][2] = {{0, 0}, {0, 1}, {0, 2}, {1, 1}, {1, 2}, {2, 2}};
    for (int e = 0; e < 6; ++e) {
      const int r = pr[e][0], c = pr[e][1];
      A[3 * r + c] = A[3 * c + r] = p[5 + e] / qg;
    }
    for (int r = 0; r < 3; ++r) A[4 * r] += lambda;
    double ev[3];
    eig3_jacobi(A, ev);
    const double tr = A[0] + A[4] + A[8];
    z[4 + 3 * d] = std::log(qg);
    for (int r = 0; r < 3; ++r) z[5 + 3 * d + r] = ev[r] / (tr + eps);
    z[8 + 3 * d] = std::log(tr + eps);
  }
  return 0;
}


// Renderer backward over the listed (view, tile) pairs (all when n_sel < 0), adding into
// accb [V, G, 10] (q, Swr[3], H, Hd[2], Hdd[3]; see backward_pixel). `img` is the render's
// C_hat [V, H, W, 3], `last` its list bounds.
#define ORC_BACKWARD(SUF, R)                                                                    \
  void orc_backward_##SUF(const double* rec, const long long* off, const int* ids, int G,      \
                          int V, int H, int W, const double* img, const float* obs,            \
                          const float* bg, const int* last, const int* sel, int n_sel,         \
                          double* accb) {                                                       \
    const int TX = (W + TILE - 1) / TILE, TY = (H + TILE - 1) / TILE, nt = TX * TY;            \
    const long long npairs = n_sel < 0 ? (long long)V * nt : n_sel;                             \
    Lists L{off, ids};                                                                          \
    _Pragma("omp parallel for schedule(dynamic, 4)")                                           \
    for (long long q = 0; q < npairs; ++q) {                                                    \
      const int v = n_sel < 0 ? (int)(q / nt) : sel[2 * q];                                     \
      const int t = n_sel < 0 ? (int)(q % nt) : sel[2 * q + 1];                                 \
      const int tx = t % TX, ty = t / TX;                                                       \
      for (int j = ty * TILE; j < std::min(H, (ty + 1) * TILE); ++j)                            \
        for (int i = tx * TILE; i < std::min(W, (tx + 1) * TILE); ++i) {                        \
          const long long p = ((long long)v * H + j) * W + i;                                   \
          backward_pixel<R>(rec + (long long)v * G * F_NFIELDS, L, (long long)v * (nt + 1), t, \
                            i, j, img + 3 * p, obs + 3 * p, bg, last[p],                        \
                            accb + (long long)v * G * ACCB_N);                                  \
        }                                                                                       \
    }                                                                                           \
  }
ORC_BACKWARD(f, float)
ORC_BACKWARD(d, double)

// Per-Gaussian chain of the renderer backward ("Relation to Gradient": raw, detached,
// support-normalised and parameter-scale-normalised gradients). Rows [G, 11 + 3d]:
//   [dL/dmu (3), dL/dlog_scale (3), dL/dquat (w, x, y, z), dL/dopacity_logit, dL/dsh (k-major)].
// Per visible view, from the sums of backward_pixel (Q = stored conic, o = opacity):
//   dL/da += (1 - o) H;  dL/dc_ch = Swr_ch where the colour clamp is inactive, else 0;
//   dL/dsh_k += B_k dL/dc;  dL/dB_k = <dL/dc, sh_k>;  dL/d mu2D = Q Hd;
//   dL/d(qa, qb, qc) = (-Hdxdx / 2, -Hdxdy, -Hdydy / 2);
// then through the conic (qa, qb, qc) = (c, -b, a) / (a c - b^2) of Sigma2D = [[a, b], [b, c]]
// (entry-wise partials), Sigma2D = J Sc J^T + 0.3 I (J the EWA Jacobian with the tangent clamped
// at 1.3x the half field of view, Sc = R_v Sigma3D R_v^T), J and mu2D as functions of the camera
// point x_c = R_v mu + t_v, the view direction dir = (mu - cam) / |mu - cam| of the SH colour,
// and after the view loop Sigma3D = (Rq S)(Rq S)^T, S = diag(exp(log_scale)), Rq from q / |q|.
// Variants ("Relation to Gradient" lists them; the readings are the plainest ones):
//   detached: the same derivative with the paths the score operators stop -- Sigma2D, the view
//     direction -- cut; it keeps the opacity-logit and SH blocks and the mean through mu2D only
//     (sum_v J_gv^T Q Hd with J_gv = d pi_v / d mu), and is zero for scale and rotation;
//   support: raw / q_g with q_g = eps + sum_v (eps + q_gv), the tokens' support normaliser;
//   pscale: raw with the mean block times exp(mean of the three log-scales), the derivative with
//     respect to the mean measured in units of the Gaussian's own size.
// `fp32_decisions`: take the tangent-clamp decision in fp32 exactly as the fp32 projection does.
// Any output pointer may be null.
int orc_grad_finalize(const int* valid, const double* rec, const double* accb,
                      const float* means, const float* lsc, const float* quats, const float* sh,
                      const float* viewmats, const float* intrin, int G, int V, int H, int W,
                      int deg, int fp32_decisions, double* raw, double* det, double* sup,
                      double* psc) {
  const int d = (deg + 1) * (deg + 1);
  const int K = 11 + 3 * d;
  const double eps = 1e-6;
#pragma omp parallel for schedule(static)
  for (int g = 0; g < G; ++g) {
    std::vector<double> gr(K, 0.0), gd(K, 0.0);
    double dSig[3][3] = {{0}};  // dL / dSigma3D (entry-wise)
    double qg = eps;
    const double mu[3] = {means[3 * g], means[3 * g + 1], means[3 * g + 2]};
    // Gaussian frame (double, from the fp32 parameters)
    double qv[4] = {quats[4 * g], quats[4 * g + 1], quats[4 * g + 2], quats[4 * g + 3]};
    const double qn = std::sqrt(qv[0] * qv[0] + qv[1] * qv[1] + qv[2] * qv[2] + qv[3] * qv[3]);
    const double w_ = qv[0] / qn, x_ = qv[1] / qn, y_ = qv[2] / qn, z_ = qv[3] / qn;
    const double Rq[3][3] = {
        {1 - 2 * (y_ * y_ + z_ * z_), 2 * (x_ * y_ - w_ * z_), 2 * (x_ * z_ + w_ * y_)},
        {2 * (x_ * y_ + w_ * z_), 1 - 2 * (x_ * x_ + z_ * z_), 2 * (y_ * z_ - w_ * x_)},
        {2 * (x_ * z_ - w_ * y_), 2 * (y_ * z_ + w_ * x_), 1 - 2 * (x_ * x_ + y_ * y_)}};
    double Sd[3], Mm[3][3], Sig[3][3];
    for (int k = 0; k < 3; ++k) Sd[k] = std::exp((double)lsc[3 * g + k]);
    for (int i = 0; i < 3; ++i)
      for (int k = 0; k < 3; ++k) Mm[i][k] = Rq[i][k] * Sd[k];
    for (int i = 0; i < 3; ++i)
      for (int j = 0; j < 3; ++j) {
        Sig[i][j] = 0;
        for (int k = 0; k < 3; ++k) Sig[i][j] += Mm[i][k] * Mm[j][k];
      }
    const float* shg = sh + (long long)g * d * 3;
    for (int v = 0; v < V; ++v) {
      const long long iv = (long long)v * G + g;
      if (!valid[iv]) continue;
      const double* rc = rec + iv * F_NFIELDS;
      const double* a = accb + iv * ACCB_N;
      qg += eps + a[0];
      const float* vm = viewmats + 16 * v;
      double Rv[3][3], tv[3];
      for (int i = 0; i < 3; ++i) {
        for (int j = 0; j < 3; ++j) Rv[i][j] = vm[4 * i + j];
        tv[i] = vm[4 * i + 3];
      }
      const double fx = intrin[4 * v], fy = intrin[4 * v + 1];
      const double o = rc[F_OPAC];
      const double qa = rc[F_QA], qb = rc[F_QB], qc = rc[F_QC];
      // opacity logit
      gr[10] += (1.0 - o) * a[4];
      // colour -> SH coefficients and view direction
      const int cm = (int)rc[F_CMASK];
      double gc[3];
      for (int ch = 0; ch < 3; ++ch) gc[ch] = ((cm >> ch) & 1) ? a[1 + ch] : 0.0;
      double cam[3], dv[3];
      for (int i = 0; i < 3; ++i) cam[i] = -(Rv[0][i] * tv[0] + Rv[1][i] * tv[1] + Rv[2][i] * tv[2]);
      for (int i = 0; i < 3; ++i) dv[i] = mu[i] - cam[i];
      const double len = std::sqrt(dv[0] * dv[0] + dv[1] * dv[1] + dv[2] * dv[2]);
      const double dir[3] = {dv[0] / len, dv[1] / len, dv[2] / len};
      double Bv[16], dB[16][3];
      sh_poly_grad_def(deg, dir, Bv, dB);
      double gdir[3] = {0, 0, 0};
      for (int k = 0; k < d; ++k) {
        double gB = 0.0;
        for (int ch = 0; ch < 3; ++ch) {
          gr[11 + 3 * k + ch] += Bv[k] * gc[ch];
          gB += gc[ch] * (double)shg[3 * k + ch];
        }
        for (int i = 0; i < 3; ++i) gdir[i] += gB * dB[k][i];
      }
      const double dg = dir[0] * gdir[0] + dir[1] * gdir[1] + dir[2] * gdir[2];
      for (int i = 0; i < 3; ++i) gr[i] += (gdir[i] - dir[i] * dg) / len;
      // projected centre and conic
      const double gmx = qa * a[5] + qb * a[6], gmy = qb * a[5] + qc * a[6];
      const double gqa = -0.5 * a[7], gqb = -a[8], gqc = -0.5 * a[9];
      // camera point (double) and the EWA Jacobian with its clamp decision
      double xc[3];
      for (int i = 0; i < 3; ++i)
        xc[i] = Rv[i][0] * mu[0] + Rv[i][1] * mu[1] + Rv[i][2] * mu[2] + tv[i];
      const double x = xc[0], y = xc[1], z = xc[2];
      bool in_u, in_v;
      if (fp32_decisions) {
        const float uf = (float)rc[F_XC] / (float)rc[F_ZC], vf = (float)rc[F_YC] / (float)rc[F_ZC];
        const float lxf = 1.3f * ((0.5f * (float)W) / (float)fx);
        const float lyf = 1.3f * ((0.5f * (float)H) / (float)fy);
        in_u = uf >= -lxf && uf <= lxf;
        in_v = vf >= -lyf && vf <= lyf;
      } else {
        const double ud = rc[F_XC] / rc[F_ZC], vd = rc[F_YC] / rc[F_ZC];
        const double lxd = 1.3 * ((0.5 * W) / fx), lyd = 1.3 * ((0.5 * H) / fy);
        in_u = ud >= -lxd && ud <= lxd;
        in_v = vd >= -lyd && vd <= lyd;
      }
      const double lx = 1.3 * ((0.5 * W) / fx), ly = 1.3 * ((0.5 * H) / fy);
      const double uc = in_u ? x / z : (x / z > 0 ? lx : -lx);
      const double vc = in_v ? y / z : (y / z > 0 ? ly : -ly);
      const double J[2][3] = {{fx / z, 0.0, -fx * uc / z}, {0.0, fy / z, -fy * vc / z}};
      double Sc[3][3];
      for (int i = 0; i < 3; ++i)
        for (int j = 0; j < 3; ++j) {
          double acc2 = 0.0;
          for (int k = 0; k < 3; ++k)
            for (int l = 0; l < 3; ++l) acc2 += Rv[i][k] * Sig[k][l] * Rv[j][l];
          Sc[i][j] = acc2;
        }
      double s2a = 0.3, s2b = 0.0, s2c = 0.3;
      for (int k = 0; k < 3; ++k)
        for (int l = 0; l < 3; ++l) {
          s2a += J[0][k] * Sc[k][l] * J[0][l];
          s2b += J[0][k] * Sc[k][l] * J[1][l];
          s2c += J[1][k] * Sc[k][l] * J[1][l];
        }
      const double D = s2a * s2c - s2b * s2b, D2 = D * D;
      // d(qa, qb, qc) / d(a, b, c) entry by entry
      const double ga_ = gqa * (-s2c * s2c / D2) + gqb * (s2b * s2c / D2) + gqc * (-s2b * s2b / D2);
      const double gb_ = gqa * (2 * s2b * s2c / D2) + gqb * (-1.0 / D - 2 * s2b * s2b / D2) +
                         gqc * (2 * s2a * s2b / D2);
      const double gc_ = gqa * (-s2b * s2b / D2) + gqb * (s2a * s2b / D2) + gqc * (-s2a * s2a / D2);
      // Sigma2D entries: a = J0 Sc J0^T, b = J0 Sc J1^T, c = J1 Sc J1^T
      double dSc[3][3], dJ[2][3];
      for (int k = 0; k < 3; ++k)
        for (int l = 0; l < 3; ++l)
          dSc[k][l] = ga_ * J[0][k] * J[0][l] + gb_ * J[0][k] * J[1][l] + gc_ * J[1][k] * J[1][l];
      for (int k = 0; k < 3; ++k) {
        double s00 = 0, s01 = 0, s11 = 0, s10 = 0;
        for (int l = 0; l < 3; ++l) {
          s00 += (Sc[k][l] + Sc[l][k]) * J[0][l];
          s01 += Sc[k][l] * J[1][l];
          s10 += J[0][l] * Sc[l][k];
          s11 += (Sc[k][l] + Sc[l][k]) * J[1][l];
        }
        dJ[0][k] = ga_ * s00 + gb_ * s01;
        dJ[1][k] = gb_ * s10 + gc_ * s11;
      }
      // camera-point gradient: mu2D = (fx x / z + cx, fy y / z + cy), and J(x, y, z)
      double gx = gmx * fx / z, gy = gmy * fy / z;
      double gz = -gmx * fx * x / (z * z) - gmy * fy * y / (z * z);
      gz += dJ[0][0] * (-fx / (z * z)) + dJ[1][1] * (-fy / (z * z));
      if (in_u) { gx += dJ[0][2] * (-fx / (z * z)); gz += dJ[0][2] * (2 * fx * x / (z * z * z)); }
      else gz += dJ[0][2] * (fx * uc / (z * z));
      if (in_v) { gy += dJ[1][2] * (-fy / (z * z)); gz += dJ[1][2] * (2 * fy * y / (z * z * z)); }
      else gz += dJ[1][2] * (fy * vc / (z * z));
      const double gxc[3] = {gx, gy, gz};
      for (int i = 0; i < 3; ++i)
        gr[i] += Rv[0][i] * gxc[0] + Rv[1][i] * gxc[1] + Rv[2][i] * gxc[2];
      // detached mean: through mu2D only
      const double gxd[3] = {gmx * fx / z, gmy * fy / z,
                             -gmx * fx * x / (z * z) - gmy * fy * y / (z * z)};
      for (int i = 0; i < 3; ++i)
        gd[i] += Rv[0][i] * gxd[0] + Rv[1][i] * gxd[1] + Rv[2][i] * gxd[2];
      // Sc = R_v Sigma3D R_v^T
      for (int p2 = 0; p2 < 3; ++p2)
        for (int q2 = 0; q2 < 3; ++q2) {
          double acc2 = 0.0;
          for (int i = 0; i < 3; ++i)
            for (int j = 0; j < 3; ++j) acc2 += dSc[i][j] * Rv[i][p2] * Rv[j][q2];
          dSig[p2][q2] += acc2;
        }
    }
    // Sigma3D = M M^T, M = Rq diag(S)
    double dM[3][3];
    for (int i = 0; i < 3; ++i)
      for (int k = 0; k < 3; ++k) {
        dM[i][k] = 0.0;
        for (int j = 0; j < 3; ++j) dM[i][k] += (dSig[i][j] + dSig[j][i]) * Mm[j][k];
      }
    double dR[3][3];
    for (int k = 0; k < 3; ++k) {
      double gS = 0.0;
      for (int i = 0; i < 3; ++i) {
        gS += dM[i][k] * Rq[i][k];
        dR[i][k] = dM[i][k] * Sd[k];
      }
      gr[3 + k] = gS * Sd[k];
    }
    // rotation entries as functions of the unit quaternion (w, x, y, z)
    const double gw = dR[0][1] * (-2 * z_) + dR[0][2] * (2 * y_) + dR[1][0] * (2 * z_) +
                      dR[1][2] * (-2 * x_) + dR[2][0] * (-2 * y_) + dR[2][1] * (2 * x_);
    const double gx_ = dR[0][1] * (2 * y_) + dR[0][2] * (2 * z_) + dR[1][0] * (2 * y_) +
                       dR[1][1] * (-4 * x_) + dR[1][2] * (-2 * w_) + dR[2][0] * (2 * z_) +
                       dR[2][1] * (2 * w_) + dR[2][2] * (-4 * x_);
    const double gy_ = dR[0][0] * (-4 * y_) + dR[0][1] * (2 * x_) + dR[0][2] * (2 * w_) +
                       dR[1][0] * (2 * x_) + dR[1][2] * (2 * z_) + dR[2][0] * (-2 * w_) +
                       dR[2][1] * (2 * z_) + dR[2][2] * (-4 * y_);
    const double gz_ = dR[0][0] * (-4 * z_) + dR[0][1] * (-2 * w_) + dR[0][2] * (2 * x_) +
                       dR[1][0] * (2 * w_) + dR[1][1] * (-4 * z_) + dR[1][2] * (2 * y_) +
                       dR[2][0] * (2 * x_) + dR[2][1] * (2 * y_);
    // q_hat = q / |q|
    const double qh[4] = {w_, x_, y_, z_}, gqh[4] = {gw, gx_, gy_, gz_};
    const double dotq = qh[0] * gqh[0] + qh[1] * gqh[1] + qh[2] * gqh[2] + qh[3] * gqh[3];
    for (int k = 0; k < 4; ++k) gr[6 + k] = (gqh[k] - qh[k] * dotq) / qn;
    // detached keeps opacity and SH as they are
    gd[10] = gr[10];
    for (int k = 11; k < K; ++k) gd[k] = gr[k];
    const double sig = std::exp(((double)lsc[3 * g] + (double)lsc[3 * g + 1] +
                                 (double)lsc[3 * g + 2]) / 3.0);
    for (int k = 0; k < K; ++k) {
      const long long o = (long long)g * K + k;
      if (raw) raw[o] = gr[k];
      if (det) det[o] = gd[k];
      if (sup) sup[o] = gr[k] / qg;
      if (psc) psc[o] = k < 3 ? gr[k] * sig : gr[k];
    }
  }
  return 0;
}

// SH basis and its gradient by the polynomial form (for the oracle's own checks):
// dirs [n, 3] unit vectors -> B [n, 16], dB [n, 16, 3].
void orc_sh_poly_grad(int deg, const double* dirs, long long n, double* B, double* dB) {
  for (long long i = 0; i < n; ++i) {
    double b[16] = {0}, db[16][3] = {{0}};
    sh_poly_grad_def(deg, dirs + 3 * i, b, db);
    for (int k = 0; k < 16; ++k) {
      B[16 * i + k] = b[k];
      for (int c = 0; c < 3; ++c) dB[48 * i + 3 * k + c] = db[k][c];
    }
  }
}


// Attribute render [V, H, W, C] (fp accumulation in the working precision, like the colour) and
// map scatter [G, C] (double) over the listed (view, tile) pairs (all when n_sel < 0); `last` is
// the render's list bound per pixel.
#define ORC_FEATURES(SUF, R)                                                                    \
  void orc_render_features_##SUF(const double* rec, const long long* off, const int* ids,      \
                                 int G, int V, int H, int W, const int* last,                  \
                                 const float* feats, int C, const int* sel, int n_sel,         \
                                 double* out) {                                                 \
    const int TX = (W + TILE - 1) / TILE, TY = (H + TILE - 1) / TILE, nt = TX * TY;            \
    const long long nsel = n_sel < 0 ? (long long)V * nt : n_sel;                               \
    Lists L{off, ids};                                                                          \
    _Pragma("omp parallel for schedule(dynamic, 1)")                                           \
    for (long long q = 0; q < nsel; ++q) {                                                      \
      const int v = n_sel < 0 ? (int)(q / nt) : sel[2 * q];                                     \
      const int t = n_sel < 0 ? (int)(q % nt) : sel[2 * q + 1];                                 \
      const int tx = t % TX, ty = t / TX;                                                       \
      std::vector<std::pair<int, R>> wts;                                                       \
      std::vector<R> F(C);                                                                      \
      for (int j = ty * TILE; j < std::min(H, ty * TILE + TILE); ++j)                           \
        for (int i = tx * TILE; i < std::min(W, tx * TILE + TILE); ++i) {                       \
          const long long p = ((long long)v * H + j) * W + i;                                   \
          pixel_weights<R>(rec + (long long)v * G * F_NFIELDS, L, (long long)v * (nt + 1), t,  \
                           i, j, last[p], wts);                                                 \
          for (int c = 0; c < C; ++c) F[c] = (R)0;                                              \
          for (const auto& e : wts)                                                             \
            for (int c = 0; c < C; ++c)                                                         \
              F[c] = F[c] + e.second * (R)feats[(long long)e.first * C + c];                    \
          for (int c = 0; c < C; ++c) out[p * C + c] = (double)F[c];                            \
        }                                                                                       \
    }                                                                                           \
  }                                                                                             \
  void orc_scatter_##SUF(const double* rec, const long long* off, const int* ids, int G, int V, \
                         int H, int W, const int* last, const float* map, int C,               \
                         const int* sel, int n_sel, double* out) {                              \
    const int TX = (W + TILE - 1) / TILE, TY = (H + TILE - 1) / TILE, nt = TX * TY;            \
    const long long nsel = n_sel < 0 ? (long long)V * nt : n_sel;                               \
    Lists L{off, ids};                                                                          \
    _Pragma("omp parallel for schedule(dynamic, 1)")                                           \
    for (long long q = 0; q < nsel; ++q) {                                                      \
      const int v = n_sel < 0 ? (int)(q / nt) : sel[2 * q];                                     \
      const int t = n_sel < 0 ? (int)(q % nt) : sel[2 * q + 1];                                 \
      const int tx = t % TX, ty = t / TX;                                                       \
      std::vector<std::pair<int, R>> wts;                                                       \
      for (int j = ty * TILE; j < std::min(H, ty * TILE + TILE); ++j)                           \
        for (int i = tx * TILE; i < std::min(W, tx * TILE + TILE); ++i) {                       \
          const long long p = ((long long)v * H + j) * W + i;                                   \
          pixel_weights<R>(rec + (long long)v * G * F_NFIELDS, L, (long long)v * (nt + 1), t,  \
                           i, j, last[p], wts);                                                 \
          for (const auto& e : wts)                                                             \
            for (int c = 0; c < C; ++c) {                                                       \
              const double add = (double)e.second * (double)map[p * C + c];                     \
              _Pragma("omp atomic")                                                             \
              out[(long long)e.first * C + c] += add;                                           \
            }                                                                                   \
        }                                                                                       \
    }                                                                                           \
  }
ORC_FEATURES(f, float)
ORC_FEATURES(d, double)

}  // extern "C"
