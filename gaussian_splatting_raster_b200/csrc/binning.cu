// Stage 1 tile binning and contributor sort.
//
// Source: "Research Proposal: Renderer Score Tokens for Recurrent Gaussian Splatting",
// "Two-Stage Algorithm" Stage 1 step 1 (gsplat tile binning and contributor sorting; the bins and
// sorted indices stay in the renderer workspace). The required order inside each tile is
// (camera depth, Gaussian index).
//
// Design (differs from a single 64-bit (tile | depth) key radix sort):
//   1. scan of the per-(v, g) tile counts -> instance offsets (reduce-then-scan, no waits);
//   2. emit: each visible (v, g) writes its instances (tile id, depth bits, g) in index order;
//   3. stable counting sort by tile: per-warp tile histograms per block of 16K instances, an
//      exclusive scan of the (tile, block) counts, then a scatter that ranks equal tiles in
//      instance order with warp match -- one pass over the instances instead of one per digit;
//      the scanned histogram also yields every tile's [start, end) for free;
//   4. per tile, a stable LSD radix sort of the fp32 depth bits (only the bits that vary inside
//      the tile), in shared memory for lists of up to 8192 entries, in global memory above.
// Stability of 3 and 4 gives the index tie-break.
#include "common.cuh"

namespace splat {
namespace {

// ---------------------------------------------------------------------------------------------
// scans
constexpr int kScanThreads = 512;
constexpr int kScanIpt = 8;
constexpr int kScanTile = kScanThreads * kScanIpt;

template <typename T>
__device__ __forceinline__ T block_exclusive_scan(T v, T* s_warp, T* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
  T inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    T u = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += u;
  }
  if (lane == 31) s_warp[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    T x = lane < nw ? s_warp[lane] : (T)0;
    T xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      T u = __shfl_up_sync(0xffffffffu, xi, o);
      if (lane >= o) xi += u;
    }
    if (lane < nw) s_warp[lane] = xi - x;
    if (lane == nw - 1 && total) *total = xi;
  }
  __syncthreads();
  const T r = s_warp[warp] + inc - v;
  __syncthreads();
  return r;
}

template <typename TI>
__global__ void __launch_bounds__(kScanThreads)
k_scan_reduce(const TI* __restrict__ in, long long n, long long* __restrict__ part) {
  __shared__ long long s_warp[32];
  __shared__ long long s_tot;
  const long long base = (long long)blockIdx.x * kScanTile + (long long)threadIdx.x * kScanIpt;
  long long s = 0;
#pragma unroll
  for (int k = 0; k < kScanIpt; ++k)
    if (base + k < n) s += (long long)in[base + k];
  block_exclusive_scan<long long>(s, s_warp, &s_tot);
  if (threadIdx.x == 0) part[blockIdx.x] = s_tot;
}

// exclusive scan of the block partials in place (single block, chunked with a carry);
// part[nb] receives the grand total
__global__ void __launch_bounds__(1024) k_scan_partials(long long* part, int nb) {
  __shared__ long long s_warp[32];
  __shared__ long long s_tot;
  long long carry = 0;
  for (int base = 0; base < nb; base += 1024) {
    const int i = base + threadIdx.x;
    const long long v = i < nb ? part[i] : 0;
    const long long ex = block_exclusive_scan<long long>(v, s_warp, &s_tot);
    if (i < nb) part[i] = carry + ex;
    __syncthreads();
    carry += s_tot;
    __syncthreads();
  }
  if (threadIdx.x == 0) part[nb] = carry;
}

template <typename TI, typename TO>
__global__ void __launch_bounds__(kScanThreads)
k_scan_down(const TI* in, TO* out, long long n, const long long* __restrict__ part) {
  __shared__ long long s_warp[32];
  const long long base = (long long)blockIdx.x * kScanTile + (long long)threadIdx.x * kScanIpt;
  long long v[kScanIpt];
  long long s = 0;
#pragma unroll
  for (int k = 0; k < kScanIpt; ++k) {
    v[k] = base + k < n ? (long long)in[base + k] : 0;
    const long long t = v[k];
    v[k] = s;
    s += t;
  }
  const long long ex = block_exclusive_scan<long long>(s, s_warp, nullptr) + part[blockIdx.x];
#pragma unroll
  for (int k = 0; k < kScanIpt; ++k)
    if (base + k < n) out[base + k] = (TO)(ex + v[k]);
}

__global__ void k_store_total(const long long* part, int nb, long long* dst) { *dst = part[nb]; }

int ensure_part(Workspace& w, long long nb) {
  if ((size_t)(nb + 1) <= w.part_cap) return SPLAT_OK;
  if (w.part) cudaFree(w.part);
  w.part = nullptr;
  const size_t cap = (size_t)(nb + 1) * 2;
  if (cudaMalloc(&w.part, cap * sizeof(long long)) != cudaSuccess) {
    cudaGetLastError();
    w.part_cap = 0;
    return set_err(w, SPLAT_ERR_OOM, "scan scratch allocation failed");
  }
  w.part_cap = cap;
  return SPLAT_OK;
}

// ---------------------------------------------------------------------------------------------
// emit
__global__ void k_emit(const float4* __restrict__ rec, const int4* __restrict__ rect,
                       const long long* __restrict__ offs, long long VG, int G, int TX,
                       uint32_t* __restrict__ inst_tile, uint2* __restrict__ inst_kv) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= VG) return;
  const int4 rc = rect[i];
  if (rc.z <= rc.x || rc.w <= rc.y) return;
  const uint32_t g = (uint32_t)(i % G);
  const uint32_t depth = __float_as_uint(rec[i * kRecF4 + 2].y);
  long long pos = offs[i];
  for (int ty = rc.y; ty < rc.w; ++ty)
    for (int tx = rc.x; tx < rc.z; ++tx) {
      inst_tile[pos] = (uint32_t)(ty * TX + tx);
      inst_kv[pos] = make_uint2(depth, g);
      ++pos;
    }
}

// ---------------------------------------------------------------------------------------------
// stable counting sort by tile
constexpr int kBinWarps = 8;
constexpr int kBinThreads = kBinWarps * 32;
constexpr int kBinChunk = 16384;                 // instances per block
constexpr int kBinPerWarp = kBinChunk / kBinWarps;

__device__ __forceinline__ int find_view(const int* bstart, int V, int b) {
  int v = 0;
  while (v + 1 < V && bstart[v + 1] <= b) ++v;
  return v;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__global__ void __launch_bounds__(kBinThreads)
k_tile_hist(const uint32_t* __restrict__ inst_tile, const long long* __restrict__ vstart,
            const int* __restrict__ bstart, int V, int nt, int* __restrict__ hist) {
  extern __shared__ uint32_t s_cnt[];  // [kBinWarps][nt]
  const int b = blockIdx.x;
  const int v = find_view(bstart, V, b);
  const int lb = b - bstart[v];
  const int nbv = bstart[v + 1] - bstart[v];
  const long long beg = vstart[v] + (long long)lb * kBinChunk;
  const long long end = min(beg + (long long)kBinChunk, vstart[v + 1]);
  for (int t = threadIdx.x; t < kBinWarps * nt; t += blockDim.x) s_cnt[t] = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* cnt = s_cnt + warp * nt;
  const long long wb = beg + (long long)warp * kBinPerWarp;
  const long long we = min(wb + (long long)kBinPerWarp, end);
  for (long long base = wb; base < we; base += 32) {
    const long long i = base + lane;
    const bool ok = i < we;
    const uint32_t t = ok ? inst_tile[i] : (0x80000000u | lane);
    const uint32_t peers = __match_any_sync(0xffffffffu, t);
    if (ok && lane == __ffs(peers) - 1) cnt[t] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  int* h = hist + (size_t)nt * bstart[v];
  for (int t = threadIdx.x; t < nt; t += blockDim.x) {
    uint32_t s = 0;
#pragma unroll
    for (int ww = 0; ww < kBinWarps; ++ww) s += s_cnt[ww * nt + t];
    h[(size_t)t * nbv + lb] = (int)s;
  }
}

__global__ void __launch_bounds__(kBinThreads)
k_tile_scatter(const uint32_t* __restrict__ inst_tile, const uint2* __restrict__ inst_kv,
               const long long* __restrict__ vstart, const int* __restrict__ bstart, int V,
               int nt, const int* __restrict__ hist_scan, uint32_t* __restrict__ skey,
               uint32_t* __restrict__ sval) {
  extern __shared__ uint32_t s_cnt[];  // [kBinWarps][nt]
  const int b = blockIdx.x;
  const int v = find_view(bstart, V, b);
  const int lb = b - bstart[v];
  const int nbv = bstart[v + 1] - bstart[v];
  const long long beg = vstart[v] + (long long)lb * kBinChunk;
  const long long end = min(beg + (long long)kBinChunk, vstart[v + 1]);
  for (int t = threadIdx.x; t < kBinWarps * nt; t += blockDim.x) s_cnt[t] = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* cnt = s_cnt + warp * nt;
  const long long wb = beg + (long long)warp * kBinPerWarp;
  const long long we = min(wb + (long long)kBinPerWarp, end);
  for (long long base = wb; base < we; base += 32) {
    const long long i = base + lane;
    const bool ok = i < we;
    const uint32_t t = ok ? inst_tile[i] : (0x80000000u | lane);
    const uint32_t peers = __match_any_sync(0xffffffffu, t);
    if (ok && lane == __ffs(peers) - 1) cnt[t] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // per tile: global start of this block's run, then one sub-run per warp in warp order
  const int* h = hist_scan + (size_t)nt * bstart[v];
  for (int t = threadIdx.x; t < nt; t += blockDim.x) {
    uint32_t run = (uint32_t)h[(size_t)t * nbv + lb];
#pragma unroll
    for (int ww = 0; ww < kBinWarps; ++ww) {
      const uint32_t c = s_cnt[ww * nt + t];
      s_cnt[ww * nt + t] = run;
      run += c;
    }
  }
  __syncthreads();
  const uint32_t lt = lanemask_lt();
  for (long long base = wb; base < we; base += 32) {
    const long long i = base + lane;
    const bool ok = i < we;
    const uint32_t t = ok ? inst_tile[i] : (0x80000000u | lane);
    const uint32_t peers = __match_any_sync(0xffffffffu, t);
    if (ok) {
      const uint2 kv = inst_kv[i];
      const uint32_t pos = cnt[t] + __popc(peers & lt);
      skey[pos] = kv.x;
      sval[pos] = kv.y;
    }
    __syncwarp();
    if (ok && lane == __ffs(peers) - 1) cnt[t] += __popc(peers);
    __syncwarp();
  }
}

__global__ void k_tile_ranges(const int* __restrict__ hist_scan, const long long* __restrict__ vstart,
                              const int* __restrict__ bstart, int V, int nt,
                              long long* __restrict__ tile_off) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= V * (nt + 1)) return;
  const int v = idx / (nt + 1), t = idx % (nt + 1);
  const int nbv = bstart[v + 1] - bstart[v];
  long long o;
  if (t == nt) o = vstart[v + 1];
  else if (nbv == 0) o = vstart[v];
  else o = hist_scan[(size_t)nt * bstart[v] + (size_t)t * nbv];
  tile_off[idx] = o;
}

// ---------------------------------------------------------------------------------------------
// per-tile stable LSD radix sort of the depth bits
constexpr int kSortWarps = 16;
constexpr int kSortThreads = kSortWarps * 32;
constexpr int kSortCap = 8192;  // entries sorted in shared memory

// one stable 8-bit digit pass over n entries; cnt is [kSortWarps][256] in shared memory
__device__ void radix_pass(const uint32_t* kin, const uint32_t* vin, uint32_t* kout,
                           uint32_t* vout, int n, int shift, uint32_t* cnt, uint32_t* s_warp) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per = (((n + kSortWarps - 1) / kSortWarps) + 31) & ~31;
  const int wb = warp * per;
  const int we = min(n, wb + per);
  for (int d = lane; d < 256; d += 32) cnt[warp * 256 + d] = 0;
  __syncwarp();
  for (int base = wb; base < we; base += 32) {
    const int i = base + lane;
    const bool ok = i < we;
    const uint32_t dig = ok ? (kin[i] >> shift) & 255u : 256u + lane;
    const uint32_t peers = __match_any_sync(0xffffffffu, dig);
    if (ok && lane == __ffs(peers) - 1) cnt[warp * 256 + dig] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // exclusive scan in (digit, warp) order: thread t owns digit t/2, warps (t&1)*8 .. +8
  {
    const int d = threadIdx.x >> 1, w0 = (threadIdx.x & 1) * 8;
    uint32_t vals[8];
    uint32_t s = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint32_t c = cnt[(w0 + k) * 256 + d];
      vals[k] = s;
      s += c;
    }
    const uint32_t ex = block_exclusive_scan<uint32_t>(s, s_warp, nullptr);
#pragma unroll
    for (int k = 0; k < 8; ++k) cnt[(w0 + k) * 256 + d] = ex + vals[k];
  }
  __syncthreads();
  const uint32_t lt = lanemask_lt();
  for (int base = wb; base < we; base += 32) {
    const int i = base + lane;
    const bool ok = i < we;
    const uint32_t key = ok ? kin[i] : 0u;
    const uint32_t dig = ok ? (key >> shift) & 255u : 256u + lane;
    const uint32_t peers = __match_any_sync(0xffffffffu, dig);
    if (ok) {
      const uint32_t pos = cnt[warp * 256 + dig] + __popc(peers & lt);
      kout[pos] = key;
      vout[pos] = vin[i];
    }
    __syncwarp();
    if (ok && lane == __ffs(peers) - 1) cnt[warp * 256 + dig] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kSortThreads)
k_tile_sort(const long long* __restrict__ tile_off, int nt, uint32_t* skey, uint32_t* sval,
            uint32_t* skey2, uint32_t* sval2) {
  extern __shared__ uint32_t s_mem[];
  uint32_t* cnt = s_mem;                     // [16][256]
  uint32_t* kbuf = s_mem + kSortWarps * 256; // [2][cap]
  uint32_t* vbuf = kbuf + 2 * kSortCap;      // [2][cap]
  __shared__ uint32_t s_warp[32];
  __shared__ uint32_t s_diff;
  const int seg = blockIdx.x;
  const int v = seg / nt, t = seg % nt;
  const long long s = tile_off[(size_t)v * (nt + 1) + t];
  const long long e = tile_off[(size_t)v * (nt + 1) + t + 1];
  const int n = (int)(e - s);
  if (n <= 1) return;
  if (threadIdx.x == 0) s_diff = 0;
  __syncthreads();
  const uint32_t k0 = skey[s];
  uint32_t dl = 0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) dl |= skey[s + i] ^ k0;
  atomicOr(&s_diff, dl);
  __syncthreads();
  const uint32_t diff = s_diff;
  const int nbits = diff ? 32 - __clz(diff) : 0;
  const int passes = (nbits + 7) >> 3;
  if (passes == 0) return;  // equal depths: index order already holds
  if (n <= kSortCap) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      kbuf[i] = skey[s + i];
      vbuf[i] = sval[s + i];
    }
    __syncthreads();
    for (int p = 0; p < passes; ++p) {
      const int a = p & 1, bsel = a ^ 1;
      radix_pass(kbuf + a * kSortCap, vbuf + a * kSortCap, kbuf + bsel * kSortCap,
                 vbuf + bsel * kSortCap, n, 8 * p, cnt, s_warp);
    }
    const uint32_t* vf = vbuf + (passes & 1) * kSortCap;
    for (int i = threadIdx.x; i < n; i += blockDim.x) sval[s + i] = vf[i];
  } else {
    uint32_t* K[2] = {skey + s, skey2 + s};
    uint32_t* Vv[2] = {sval + s, sval2 + s};
    for (int p = 0; p < passes; ++p) {
      const int a = p & 1, bsel = a ^ 1;
      radix_pass(K[a], Vv[a], K[bsel], Vv[bsel], n, 8 * p, cnt, s_warp);
    }
    if (passes & 1)
      for (int i = threadIdx.x; i < n; i += blockDim.x) sval[s + i] = sval2[s + i];
  }
}

template <typename T>
int grow(Workspace& w, T** p, size_t n, const char* what) {
  if (*p) cudaFree(*p);
  *p = nullptr;
  if (cudaMalloc(p, n * sizeof(T)) != cudaSuccess) {
    cudaGetLastError();
    return set_err(w, SPLAT_ERR_OOM, std::string("allocation failed: ") + what);
  }
  return SPLAT_OK;
}

}  // namespace

// ---------------------------------------------------------------------------------------------
int scan_i32_to_i64(Workspace& w, const int* in, long long* out, long long n, cudaStream_t st) {
  const long long nb = (n + kScanTile - 1) / kScanTile;
  int rc = ensure_part(w, nb > 0 ? nb : 1);
  if (rc) return rc;
  if (nb > 0) {
    k_scan_reduce<int><<<(unsigned)nb, kScanThreads, 0, st>>>(in, n, w.part);
    if ((rc = check_launch(w, "scan reduce"))) return rc;
  }
  k_scan_partials<<<1, 1024, 0, st>>>(w.part, (int)nb);
  if ((rc = check_launch(w, "scan partials"))) return rc;
  if (nb > 0) {
    k_scan_down<int, long long><<<(unsigned)nb, kScanThreads, 0, st>>>(in, out, n, w.part);
    if ((rc = check_launch(w, "scan downsweep"))) return rc;
  }
  k_store_total<<<1, 1, 0, st>>>(w.part, (int)nb, out + n);
  return check_launch(w, "scan total");
}

int scan_i32_inplace(Workspace& w, int* data, long long n, cudaStream_t st) {
  const long long nb = (n + kScanTile - 1) / kScanTile;
  int rc = ensure_part(w, nb > 0 ? nb : 1);
  if (rc) return rc;
  if (nb == 0) return SPLAT_OK;
  k_scan_reduce<int><<<(unsigned)nb, kScanThreads, 0, st>>>(data, n, w.part);
  if ((rc = check_launch(w, "hist scan reduce"))) return rc;
  k_scan_partials<<<1, 1024, 0, st>>>(w.part, (int)nb);
  if ((rc = check_launch(w, "hist scan partials"))) return rc;
  k_scan_down<int, int><<<(unsigned)nb, kScanThreads, 0, st>>>(data, data, n, w.part);
  return check_launch(w, "hist scan downsweep");
}

int launch_scan_counts(Workspace& w, cudaStream_t st) {
  const int tok = prof_begin(w, st, SPLAT_K_SCAN_COUNTS);
  const int rc = scan_i32_to_i64(w, w.counts, w.offs, (long long)w.V * w.G, st);
  prof_end(w, st, tok);
  return rc;
}

// after the host has read the per-view instance starts into w.h_vstart
int launch_binning(Workspace& w, cudaStream_t st) {
  int rc;
  const long long N = w.n_total;
  // block table: ceil(N_v / chunk) blocks per view
  w.h_bstart[0] = 0;
  for (int v = 0; v < w.V; ++v) {
    const long long nv = w.h_vstart[v + 1] - w.h_vstart[v];
    w.h_bstart[v + 1] = w.h_bstart[v] + (int)((nv + kBinChunk - 1) / kBinChunk);
  }
  w.n_blocks = w.h_bstart[w.V];
  const size_t hist_n = (size_t)w.nt * (size_t)w.n_blocks;
  if (N > w.inst_cap) {
    const size_t cap = (size_t)(N + N / 4 + 1024);
    if ((rc = grow(w, &w.inst_tile, cap, "instance tiles"))) return rc;
    if ((rc = grow(w, &w.inst_kv, cap, "instance keys"))) return rc;
    if ((rc = grow(w, &w.skey, cap, "sort keys"))) return rc;
    if ((rc = grow(w, &w.sval, cap, "sort values"))) return rc;
    if ((rc = grow(w, &w.skey2, cap, "sort keys 2"))) return rc;
    if ((rc = grow(w, &w.sval2, cap, "sort values 2"))) return rc;
    w.inst_cap = cap;
  }
  if (hist_n + 1 > w.hist_cap) {
    const size_t cap = hist_n + hist_n / 4 + 1024;
    if ((rc = grow(w, &w.hist, cap, "tile histogram"))) return rc;
    w.hist_cap = cap;
  }
  cudaMemcpyAsync(w.d_vstart, w.h_vstart, (w.V + 1) * sizeof(long long),
                  cudaMemcpyHostToDevice, st);
  cudaMemcpyAsync(w.d_bstart, w.h_bstart, (w.V + 1) * sizeof(int), cudaMemcpyHostToDevice, st);
  const long long VG = (long long)w.V * w.G;
  if (N > 0) {
    int tok = prof_begin(w, st, SPLAT_K_EMIT);
    k_emit<<<(unsigned)((VG + 255) / 256), 256, 0, st>>>(w.rec, w.rect, w.offs, VG, w.G, w.TX,
                                                          w.inst_tile, w.inst_kv);
    prof_end(w, st, tok);
    if ((rc = check_launch(w, "emit kernel"))) return rc;
    const size_t smem = (size_t)kBinWarps * w.nt * sizeof(uint32_t);
    tok = prof_begin(w, st, SPLAT_K_TILE_HIST);
    k_tile_hist<<<w.n_blocks, kBinThreads, smem, st>>>(w.inst_tile, w.d_vstart, w.d_bstart, w.V,
                                                       w.nt, w.hist);
    prof_end(w, st, tok);
    if ((rc = check_launch(w, "tile histogram kernel"))) return rc;
    tok = prof_begin(w, st, SPLAT_K_HIST_SCAN);
    rc = scan_i32_inplace(w, w.hist, (long long)hist_n, st);
    prof_end(w, st, tok);
    if (rc) return rc;
    tok = prof_begin(w, st, SPLAT_K_TILE_SCATTER);
    k_tile_scatter<<<w.n_blocks, kBinThreads, smem, st>>>(w.inst_tile, w.inst_kv, w.d_vstart,
                                                          w.d_bstart, w.V, w.nt, w.hist, w.skey,
                                                          w.sval);
    prof_end(w, st, tok);
    if ((rc = check_launch(w, "tile scatter kernel"))) return rc;
  }
  const int nr = w.V * (w.nt + 1);
  int tok_r = prof_begin(w, st, SPLAT_K_TILE_RANGES);
  k_tile_ranges<<<(nr + 255) / 256, 256, 0, st>>>(w.hist, w.d_vstart, w.d_bstart, w.V, w.nt,
                                                  w.tile_off);
  prof_end(w, st, tok_r);
  if ((rc = check_launch(w, "tile ranges kernel"))) return rc;
  if (N > 0) {
    const size_t smem = (size_t)(kSortWarps * 256 + 4 * kSortCap) * sizeof(uint32_t);
    const int tok_s = prof_begin(w, st, SPLAT_K_TILE_SORT);
    k_tile_sort<<<w.V * w.nt, kSortThreads, smem, st>>>(w.tile_off, w.nt, w.skey, w.sval, w.skey2,
                                                         w.sval2);
    prof_end(w, st, tok_s);
    if ((rc = check_launch(w, "tile depth sort kernel"))) return rc;
  }
  return SPLAT_OK;
}

// shared-memory opt-in for the binning kernels (called once per workspace)
int binning_configure(Workspace& w) {
  const int sort_smem = (kSortWarps * 256 + 4 * kSortCap) * sizeof(uint32_t);
  const int bin_smem = kBinWarps * w.max_nt * sizeof(uint32_t);
  cudaError_t e1 = cudaFuncSetAttribute(k_tile_sort, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        sort_smem);
  cudaError_t e2 = cudaFuncSetAttribute(k_tile_hist, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        bin_smem);
  cudaError_t e3 = cudaFuncSetAttribute(k_tile_scatter,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, bin_smem);
  if (e1 != cudaSuccess || e2 != cudaSuccess || e3 != cudaSuccess) {
    cudaGetLastError();
    return set_err(w, SPLAT_ERR_CAPACITY,
                   "image has too many tiles for the binning kernels' shared memory");
  }
  return SPLAT_OK;
}

}  // namespace splat
