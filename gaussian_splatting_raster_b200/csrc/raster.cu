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
// One CTA per (tile, view), one thread per pixel of the 16x16 tile. The tile's list is walked in
// batches of 256 entries whose records (mean, conic, opacity, colour: 36 bytes) are staged in
// shared memory by one coalesced gather per batch. Both passes evaluate alpha through the same
// device function, so the replay takes exactly the render's decisions.
//
// Replay accumulation: per entry of a batch, each warp reduces its 32 pixels' seven
// contributions (q, w r (3), w rho, w rho (p - mu2D) (2)) with shuffles and adds them to a
// shared-memory slot of that entry; at the end of the batch one thread per entry adds the CTA's
// sums to the (view, Gaussian) accumulator with fp64 atomics -- seven global atomics per
// (Gaussian, tile) instead of per (Gaussian, pixel). The SH block never enters the pixel loop:
// its per-pixel term M_color w (B (x) r) factors into M_color B (x) (sum w r), and the mean block
// Sigma^-1 (sum w rho d) is formed once per (Gaussian, view) in finalisation.
#include "common.cuh"

namespace splat {
namespace {

constexpr int kThreads = 256;

struct Entry {
  bool use;
  float alpha, dx, dy;
};

// alpha of one list entry at pixel centre (px, py), with the rasteriser's skip rules
__device__ __forceinline__ Entry eval_entry(const float4 A, const float4 Bq, float px, float py) {
  Entry e;
  e.dx = px - A.x;
  e.dy = py - A.y;
  const float t1 = A.z * e.dx * e.dx;
  const float t2 = Bq.x * e.dy * e.dy;
  const float t3 = A.w * e.dx * e.dy;
  const float pw = -0.5f * (t1 + t2) - t3;
  e.use = false;
  e.alpha = 0.0f;
  if (pw > 0.0f) return e;
  const float al = fminf(0.99f, Bq.y * exp_cw(pw));
  if (al < 1.0f / 255.0f) return e;
  e.alpha = al;
  e.use = true;
  return e;
}

__global__ void __launch_bounds__(kThreads)
k_render(const float4* __restrict__ rec, const uint32_t* __restrict__ ids,
         const long long* __restrict__ tile_off, int G, int H, int W, int TX, int nt,
         const float* __restrict__ bgp, float* __restrict__ img, float* __restrict__ Tout,
         int* __restrict__ ncout, int* __restrict__ last) {
  const int t = blockIdx.x, v = blockIdx.y;
  const int tx = t % TX, ty = t / TX;
  const int i = tx * kTile + (threadIdx.x & 15), j = ty * kTile + (threadIdx.x >> 4);
  const bool inside = i < W && j < H;
  const long long s = tile_off[(size_t)v * (nt + 1) + t];
  const long long e = tile_off[(size_t)v * (nt + 1) + t + 1];
  __shared__ float4 s_a[kThreads], s_b[kThreads];
  __shared__ float s_c[kThreads];
  const float px = (float)i + 0.5f, py = (float)j + 0.5f;
  float T = 1.0f, C0 = 0.0f, C1 = 0.0f, C2 = 0.0f;
  int n = 0, lst = 0;
  bool done = !inside;
  const float4* recv = rec + (size_t)v * G * kRecF4;
  for (long long base = s; base < e; base += kThreads) {
    if (__syncthreads_count(done) == kThreads) break;
    const long long k = base + threadIdx.x;
    if (k < e) {
      const float4* r = recv + (size_t)ids[k] * kRecF4;
      s_a[threadIdx.x] = r[0];
      s_b[threadIdx.x] = r[1];
      s_c[threadIdx.x] = r[2].x;
    }
    __syncthreads();
    const int cnt = (int)min((long long)kThreads, e - base);
    if (!done) {
      for (int q = 0; q < cnt; ++q) {
        const float4 A = s_a[q], Bq = s_b[q];
        const Entry E = eval_entry(A, Bq, px, py);
        if (!E.use) continue;
        const float Tn = T * (1.0f - E.alpha);
        if (Tn < 1e-4f) {
          done = true;
          break;
        }
        const float wgt = E.alpha * T;
        C0 = C0 + wgt * Bq.z;
        C1 = C1 + wgt * Bq.w;
        C2 = C2 + wgt * s_c[q];
        T = Tn;
        ++n;
        lst = (int)(base - s) + q + 1;
      }
    }
  }
  if (inside) {
    const size_t p = ((size_t)v * H + j) * W + i;
    img[3 * p + 0] = C0 + T * bgp[0];
    img[3 * p + 1] = C1 + T * bgp[1];
    img[3 * p + 2] = C2 + T * bgp[2];
    Tout[p] = T;
    ncout[p] = n;
    last[p] = lst;
  }
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__global__ void __launch_bounds__(kThreads)
k_replay(const float4* __restrict__ rec, const uint32_t* __restrict__ ids,
         const long long* __restrict__ tile_off, int G, int H, int W, int TX, int nt,
         const float* __restrict__ img, const float* __restrict__ obs,
         const int* __restrict__ last, double* __restrict__ acc) {
  const int t = blockIdx.x, v = blockIdx.y;
  const int tx = t % TX, ty = t / TX;
  const int i = tx * kTile + (threadIdx.x & 15), j = ty * kTile + (threadIdx.x >> 4);
  const bool inside = i < W && j < H;
  const long long s = tile_off[(size_t)v * (nt + 1) + t];
  __shared__ float4 s_a[kThreads], s_b[kThreads];
  __shared__ float s_c[kThreads];
  __shared__ uint32_t s_g[kThreads];
  __shared__ float s_acc[7][kThreads];
  __shared__ int s_max;
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
  if (threadIdx.x == 0) s_max = 0;
  __syncthreads();
  atomicMax(&s_max, lst);
  __syncthreads();
  const int maxl = s_max;
  const float4* recv = rec + (size_t)v * G * kRecF4;
  double* accv = acc + (size_t)v * G * kAccN;
  float T = 1.0f, P0 = 0.0f, P1 = 0.0f, P2 = 0.0f;
  const int lane = threadIdx.x & 31;
  for (int base = 0; base < maxl; base += kThreads) {
    const int cnt = min(kThreads, maxl - base);
    if ((int)threadIdx.x < cnt) {
      const uint32_t g = ids[s + base + threadIdx.x];
      const float4* r = recv + (size_t)g * kRecF4;
      s_a[threadIdx.x] = r[0];
      s_b[threadIdx.x] = r[1];
      s_c[threadIdx.x] = r[2].x;
      s_g[threadIdx.x] = g;
    }
#pragma unroll
    for (int c = 0; c < 7; ++c) s_acc[c][threadIdx.x] = 0.0f;
    __syncthreads();
    for (int q = 0; q < cnt; ++q) {
      float v0 = 0.0f, v1 = 0.0f, v2 = 0.0f, v3 = 0.0f, v4 = 0.0f, v5 = 0.0f, v6 = 0.0f;
      bool used = false;
      if (base + q < lst) {
        const float4 A = s_a[q], Bq = s_b[q];
        const Entry E = eval_entry(A, Bq, px, py);
        if (E.use) {
          used = true;
          const float al = E.alpha;
          const float den = T * (1.0f - al);
          const float w = al * T;
          const float c0 = Bq.z, c1 = Bq.w, c2 = s_c[q];
          const float dd = den + 1e-12f;
          const float Cp0 = ((Ch0 - P0) - w * c0) / dd;
          const float Cp1 = ((Ch1 - P1) - w * c1) / dd;
          const float Cp2 = ((Ch2 - P2) - w * c2) / dd;
          const bool Ma = (den >= 1e-4f) && (al < 0.99f);
          const float rho = r0 * (c0 - Cp0) + r1 * (c1 - Cp1) + r2 * (c2 - Cp2);
          v0 = w;
          v1 = w * r0;
          v2 = w * r1;
          v3 = w * r2;
          if (Ma) {
            const float wr = w * rho;
            v4 = wr;
            v5 = wr * E.dx;
            v6 = wr * E.dy;
          }
          P0 = P0 + w * c0;
          P1 = P1 + w * c1;
          P2 = P2 + w * c2;
          T = den;
        }
      }
      if (__any_sync(0xffffffffu, used)) {
        v0 = warp_sum(v0);
        v1 = warp_sum(v1);
        v2 = warp_sum(v2);
        v3 = warp_sum(v3);
        v4 = warp_sum(v4);
        v5 = warp_sum(v5);
        v6 = warp_sum(v6);
        if (lane == 0) {
          atomicAdd(&s_acc[0][q], v0);
          atomicAdd(&s_acc[1][q], v1);
          atomicAdd(&s_acc[2][q], v2);
          atomicAdd(&s_acc[3][q], v3);
          atomicAdd(&s_acc[4][q], v4);
          atomicAdd(&s_acc[5][q], v5);
          atomicAdd(&s_acc[6][q], v6);
        }
      }
    }
    __syncthreads();
    if ((int)threadIdx.x < cnt && s_acc[0][threadIdx.x] != 0.0f) {
      double* a = accv + (size_t)s_g[threadIdx.x] * kAccN;
#pragma unroll
      for (int c = 0; c < 7; ++c) atomicAdd(a + c, (double)s_acc[c][threadIdx.x]);
    }
    __syncthreads();
  }
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
  dim3 grid(w.nt, w.V);
  const int tok = prof_begin(w, st, SPLAT_K_RENDER);
  k_render<<<grid, kThreads, 0, st>>>(w.rec, w.sval, w.tile_off, w.G, w.H, w.W, w.TX, w.nt, bg,
                                      img, T_final, n_contrib, w.last);
  prof_end(w, st, tok);
  return check_launch(w, "render kernel");
}

int launch_replay(Workspace& w, const float* obs, cudaStream_t st) {
  const int tok = prof_begin(w, st, SPLAT_K_REPLAY);
  if (w.G > 0) {
    cudaError_t e = cudaMemsetAsync(w.acc, 0, (size_t)w.V * w.G * kAccN * sizeof(double), st);
    if (e != cudaSuccess)
      return set_err(w, SPLAT_ERR_CUDA, std::string("accumulator clear: ") + cudaGetErrorString(e));
  }
  dim3 grid(w.nt, w.V);
  k_replay<<<grid, kThreads, 0, st>>>(w.rec, w.sval, w.tile_off, w.G, w.H, w.W, w.TX, w.nt,
                                      w.img, obs, w.last, w.acc);
  prof_end(w, st, tok);
  return check_launch(w, "replay kernel");
}

int launch_pair_count(Workspace& w, cudaStream_t st) {
  cudaMemsetAsync(w.d_scratch, 0, sizeof(long long), st);
  const long long n = (long long)w.V * w.H * w.W;
  k_pair_sum<<<296, 256, 0, st>>>(w.last, n, w.d_scratch);
  return check_launch(w, "pair count kernel");
}

}  // namespace splat
