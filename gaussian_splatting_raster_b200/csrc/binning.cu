// Stage 1 tile binning and contributor sort.
//
// Source: "Research Proposal: Renderer Score Tokens for Recurrent Gaussian Splatting",
// "Two-Stage Algorithm" Stage 1 step 1 (gsplat tile binning and contributor sorting; the bins and
// sorted indices stay in the renderer workspace). The required order inside each tile is
// (camera depth, Gaussian index).
//
// Design (instead of one radix sort of 64-bit (tile | depth) keys over all instances):
//   1. per view, a stable LSD radix sort of the (v, g) depth keys -- one key per Gaussian, not per
//      instance -- over the width of the view's key range: the first pass orders key - kmin(view)
//      (the projection records each view's smallest and largest visible key), so depths in
//      [1, 100] take 26 bits (3 passes of 9) where the varying bits of the raw keys were 31;
//   2. the tile rectangles gathered into that depth order, their tile counts scanned, and the
//      instances (tile, g) emitted in depth order;
//   3. one stable counting sort of the instances by tile. Stability of 1 (index order of equal
//      depths) and 3 (depth order inside each tile) gives exactly (depth, index) per tile, and the
//      scanned (tile, block) histogram yields every tile's [start, end).
// Every pass -- each depth digit and the tile pass -- is a stable counting sort over blocks of 16K
// items: per-warp shared-memory histograms (shared-memory atomics), an int32 exclusive scan of the
// (bucket, block) counts, and a scatter that ranks equal buckets inside each 32-item batch with
// match.any (stable: earlier items first). The depth passes (512 buckets) lay each 4K-item round
// out in bucket order in shared memory and write whole bucket runs; the tile pass (one bucket per
// tile, ~2 items per bucket and round) writes each item straight to its place. Uniform,
// bandwidth-shaped work; no decoupled look-back, so no device-side waits.
#include "common.cuh"

namespace splat {

SPLAT_BOUNDS_WORD(bounds_word_binning)

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

// tile sums (the order of the adds does not matter: coalesced loads)
template <typename TI>
__global__ void __launch_bounds__(kScanThreads)
k_scan_reduce(const TI* __restrict__ in, long long n, long long* __restrict__ part) {
  __shared__ long long s_warp[32];
  __shared__ long long s_tot;
  const long long base = (long long)blockIdx.x * kScanTile + threadIdx.x;
  long long s = 0;
#pragma unroll
  for (int k = 0; k < kScanIpt; ++k) {
    const long long i = base + (long long)k * kScanThreads;
    if (i < n) s += (long long)in[i];
  }
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

// exclusive scan of one tile plus its partial: coalesced loads into shared memory, a sequential
// scan of kScanIpt contiguous values per thread, a block scan of the thread sums, coalesced
// stores. The whole tile is read before any of it is written, so in == out is allowed.
__device__ __forceinline__ int scan_pad(int i) { return i + (i >> 4); }  // 1 word per 16: banks

template <typename TI, typename TO>
__global__ void __launch_bounds__(kScanThreads)
k_scan_down(const TI* in, TO* out, long long n, const long long* __restrict__ part) {
  __shared__ long long s_buf[kScanTile + kScanTile / 16];
  __shared__ long long s_warp[32];
  const long long base = (long long)blockIdx.x * kScanTile;
#pragma unroll
  for (int k = 0; k < kScanIpt; ++k) {
    const int i = threadIdx.x + k * kScanThreads;
    s_buf[scan_pad(i)] = base + i < n ? (long long)in[base + i] : 0;
  }
  __syncthreads();
  long long v[kScanIpt];
  long long s = 0;
#pragma unroll
  for (int k = 0; k < kScanIpt; ++k) {
    const long long t = s_buf[scan_pad(threadIdx.x * kScanIpt + k)];
    v[k] = s;
    s += t;
  }
  const long long ex = block_exclusive_scan<long long>(s, s_warp, nullptr) + part[blockIdx.x];
#pragma unroll
  for (int k = 0; k < kScanIpt; ++k) s_buf[scan_pad(threadIdx.x * kScanIpt + k)] = ex + v[k];
  __syncthreads();
#pragma unroll
  for (int k = 0; k < kScanIpt; ++k) {
    const int i = threadIdx.x + k * kScanThreads;
    if (base + i < n) out[base + i] = (TO)s_buf[scan_pad(i)];
  }
}

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
// the stable counting-sort pass
constexpr int kBinWarps = 8;
constexpr int kBinThreads = kBinWarps * 32;
constexpr int kDepthChunk = 16384;  // items per block, depth-key passes
// widest depth digit: the key range's bits are split into ceil(bits / max) passes of equal width
#ifndef SPLAT_DEPTH_DIGIT_MAX
#define SPLAT_DEPTH_DIGIT_MAX 11
#endif
constexpr int kDepthDigitMax = SPLAT_DEPTH_DIGIT_MAX;
constexpr int kTileChunk = 16384;   // items per block, tile pass


// Items of view v are [start(v), start(v + 1)); each view is cut into blocks of `chunk` items.
// Uniform layout (every view holds `per_view` items, blocks_per_view blocks) or tables.
struct Segs {
  long long per_view;        // >= 0: uniform layout
  int blocks_per_view;
  const long long* vstart;   // tables (per_view < 0): [V + 1] item starts
  const int* bstart;         // [V + 1] block starts
  int V;
  int chunk;                 // items per block (a multiple of 32 * kBinWarps)
};

struct BlockRange {
  int v, lb, nbv, b0;  // view, block within view, blocks of the view, first block of the view
  long long beg, end, vbeg;
};

__device__ __forceinline__ BlockRange block_range(const Segs& sg, int b) {
  BlockRange r;
  if (sg.per_view >= 0) {
    r.nbv = sg.blocks_per_view;
    r.v = b / r.nbv;
    r.lb = b - r.v * r.nbv;
    r.b0 = r.v * r.nbv;
    r.vbeg = (long long)r.v * sg.per_view;
    r.beg = r.vbeg + (long long)r.lb * sg.chunk;
    r.end = min(r.beg + (long long)sg.chunk, r.vbeg + sg.per_view);
  } else {
    int v = 0;
    while (v + 1 < sg.V && sg.bstart[v + 1] <= b) ++v;
    r.v = v;
    r.b0 = sg.bstart[v];
    r.lb = b - r.b0;
    r.nbv = sg.bstart[v + 1] - r.b0;
    r.vbeg = sg.vstart[v];
    r.beg = r.vbeg + (long long)r.lb * sg.chunk;
    r.end = min(r.beg + (long long)sg.chunk, sg.vstart[v + 1]);
  }
  return r;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Digit source of a depth key. The first depth pass reads the projection's keys and orders
// key - kmin(view) (kmin = the view's smallest visible key), clamped to `top` = 2^bits - 1 where
// bits is the width of the largest view's key range; culled entries (key 0xffffffff) clamp to the
// top and sort last. The pass writes the mapped keys, so the later passes read them unchanged
// (kbits == nullptr: identity).
struct KeyMap {
  const uint32_t* kbits;  // [V][kKeyStripes][2] statistics of the projection, or nullptr
  uint32_t top;
};

// the view's smallest visible key: the complement of the largest complement over the stripes
__device__ __forceinline__ uint32_t view_kmin(const uint32_t* __restrict__ kbits, int v) {
  const int lane = threadIdx.x & 31;
  uint32_t m = 0;
  for (int s = lane; s < kKeyStripes; s += 32) m = max(m, kbits[2 * (v * kKeyStripes + s) + 1]);
  return ~__reduce_max_sync(0xffffffffu, m);
}

__device__ __forceinline__ uint32_t map_key(uint32_t k, uint32_t kmin, uint32_t top) {
  const uint32_t d = k - kmin;
  return d < top ? d : top;
}

constexpr int kUnroll = 16;      // 32-item batches whose loads are issued together (ranking)
constexpr int kCountUnroll = 32; // 32-item batches whose loads are issued together (counting)
constexpr int kHistUnroll = 32;  // the same for the histogram kernel

// per-warp bucket counts of the items [wb, we) into cnt (shared memory): the loads of UNR
// batches are issued together, then each lane adds its items with shared-memory atomics (counts
// do not depend on the order of the adds); whole groups without tail checks, then the tail
template <int UNR>
__device__ __forceinline__ void warp_counts(const uint32_t* __restrict__ keys, uint32_t kmin,
                                            uint32_t top, int shift, uint32_t mask, long long wb,
                                            long long we, uint32_t* cnt) {
  const int lane = threadIdx.x & 31;
  const uint32_t* kp = keys + wb;
  const int n = we > wb ? (int)(we - wb) : 0;
  const int nfull = n / (32 * UNR) * (32 * UNR);
  for (int b = 0; b < nfull; b += 32 * UNR) {
    uint32_t bk[UNR];
#pragma unroll
    for (int u = 0; u < UNR; ++u) bk[u] = (map_key(kp[b + 32 * u + lane], kmin, top) >> shift) & mask;
#pragma unroll
    for (int u = 0; u < UNR; ++u) atomicAdd(cnt + bk[u], 1u);
  }
  if (nfull < n) {
    uint32_t bk[UNR];
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int o = nfull + 32 * u + lane;
      bk[u] = o < n ? (map_key(kp[o], kmin, top) >> shift) & mask : 0xffffffffu;
    }
#pragma unroll
    for (int u = 0; u < UNR; ++u)
      if (bk[u] != 0xffffffffu) atomicAdd(cnt + bk[u], 1u);
  }
}

// histogram: hist[nbk * b0 + bucket * nbv + lb] = count of the block's items in the bucket
__global__ void __launch_bounds__(kBinThreads)
k_count_hist(const uint32_t* __restrict__ keys, KeyMap km, int shift, uint32_t mask, int nbk,
             Segs sg, int* __restrict__ hist) {
  extern __shared__ uint32_t s_cnt[];  // [kBinWarps][nbk]
  const BlockRange r = block_range(sg, blockIdx.x);
  for (int t = threadIdx.x; t < kBinWarps * nbk; t += blockDim.x) s_cnt[t] = 0;
  const uint32_t kmin = km.kbits ? view_kmin(km.kbits, r.v) : 0u;
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  const long long wb = r.beg + (long long)warp * (sg.chunk / kBinWarps);
  const long long we = min(wb + (long long)(sg.chunk / kBinWarps), r.end);
  warp_counts<kHistUnroll>(keys, kmin, km.top, shift, mask, wb, we, s_cnt + warp * nbk);
  __syncthreads();
  int* h = hist + (size_t)nbk * r.b0;
  for (int t = threadIdx.x; t < nbk; t += blockDim.x) {
    uint32_t s = 0;
#pragma unroll
    for (int ww = 0; ww < kBinWarps; ++ww) s += s_cnt[ww * nbk + t];
    h[(size_t)t * r.nbv + r.lb] = (int)s;
  }
}

// stable scatter of (key, value) by bucket; vals == nullptr means value = index within the view;
// kout == nullptr drops the keys
__global__ void __launch_bounds__(kBinThreads)
k_count_scatter(const uint32_t* __restrict__ keys, const uint32_t* __restrict__ vals, KeyMap km,
                int shift, uint32_t mask, int nbk, Segs sg, const int* __restrict__ hist_scan,
                uint32_t* __restrict__ kout, uint32_t* __restrict__ vout) {
  extern __shared__ uint32_t s_cnt[];  // [kBinWarps][nbk]
  const BlockRange r = block_range(sg, blockIdx.x);
  for (int t = threadIdx.x; t < kBinWarps * nbk; t += blockDim.x) s_cnt[t] = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* cnt = s_cnt + warp * nbk;
  const long long wb = r.beg + (long long)warp * (sg.chunk / kBinWarps);
  const long long we = min(wb + (long long)(sg.chunk / kBinWarps), r.end);
  const uint32_t kmin = km.kbits ? view_kmin(km.kbits, r.v) : 0u;
  warp_counts<kCountUnroll>(keys, kmin, km.top, shift, mask, wb, we, cnt);
  __syncthreads();
  // per bucket: global start of this block's run, then one sub-run per warp in warp order
  const int* h = hist_scan + (size_t)nbk * r.b0;
  for (int t = threadIdx.x; t < nbk; t += blockDim.x) {
    uint32_t run = (uint32_t)h[(size_t)t * r.nbv + r.lb];
#pragma unroll
    for (int ww = 0; ww < kBinWarps; ++ww) {
      const uint32_t c = s_cnt[ww * nbk + t];
      s_cnt[ww * nbk + t] = run;
      run += c;
    }
  }
  __syncthreads();
  const uint32_t lt = lanemask_lt();
  const unsigned long long lim =
      sg.per_view >= 0 ? (unsigned long long)sg.per_view * sg.V : (unsigned long long)sg.vstart[sg.V];
  // 32-bit offsets from the warp's first item; whole groups without tail checks, then the tail
  const uint32_t* kp = keys + wb;
  const uint32_t* vp = vals ? vals + wb : nullptr;
  const int n = we > wb ? (int)(we - wb) : 0;
  const uint32_t vbase = (uint32_t)(wb - r.vbeg);
  const int nfull = n / (32 * kUnroll) * (32 * kUnroll);
  for (int b = 0; b < nfull; b += 32 * kUnroll) {
    uint32_t key[kUnroll], val[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int o = b + 32 * u + lane;
      key[u] = map_key(kp[o], kmin, km.top);
      val[u] = vp ? vp[o] : vbase + (uint32_t)o;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const uint32_t bk = (key[u] >> shift) & mask;
      const uint32_t peers = __match_any_sync(0xffffffffu, bk);
      const uint32_t pos = cnt[bk] + __popc(peers & lt);
      if (in_bounds(pos, lim, &g_bounds_word)) {
        if (kout) kout[pos] = key[u];
        vout[pos] = val[u];
      }
      __syncwarp();
      if (lane == __ffs(peers) - 1) cnt[bk] += __popc(peers);
      __syncwarp();
    }
  }
  for (int b = nfull; b < n; b += 32) {
    const int o = b + lane;
    const bool ok = o < n;
    const uint32_t key = ok ? map_key(kp[o], kmin, km.top) : 0u;
    const uint32_t val = ok ? (vp ? vp[o] : vbase + (uint32_t)o) : 0u;
    const uint32_t bk = ok ? (key >> shift) & mask : (0x80000000u | lane);
    const uint32_t peers = __match_any_sync(0xffffffffu, bk);
    if (ok) {
      const uint32_t pos = cnt[bk] + __popc(peers & lt);
      if (in_bounds(pos, lim, &g_bounds_word)) {
        if (kout) kout[pos] = key;
        vout[pos] = val;
      }
    }
    __syncwarp();
    if (ok && lane == __ffs(peers) - 1) cnt[bk] += __popc(peers);
    __syncwarp();
  }
}

// Stable scatter of (key, value) by bucket, one round of kRound consecutive items at a time
// (vals == nullptr: value = index within the view; kout == nullptr drops the keys). In a round
// each warp ranks its kWarpRound items in order -- match.any inside each 32-item batch and a
// per-warp count per bucket -- and a block scan over (bucket, warp), bucket-major, turns the
// counts into every item's place in the round's bucket order (stable: a warp's items in order,
// the warps in order). The round is laid out in shared memory in that order and then written
// out: thread j stores place j at base(bucket) + j - start(bucket), so a warp's stores fall on a
// few bucket runs instead of 32 scattered words. base(bucket) starts at the block's entry of the
// scanned (bucket, block) histogram and advances by the bucket's count after every round.
constexpr int kRoundIpt = 16;                        // items per thread per round
constexpr int kRound = kBinThreads * kRoundIpt;      // items per round
constexpr int kWarpRound = kRound / kBinWarps;       // items per warp per round

// buckets per thread in the (bucket, warp) scan: odd, so that the threads' strided reads of the
// counts fall on distinct banks
__host__ __device__ __forceinline__ int scan_bpt(int nbk) {
  return ((nbk + 1 + kBinThreads - 1) / kBinThreads) | 1;
}

// dynamic shared memory of k_rank_scatter: counts [kBinWarps][nbk + 1], bases [nbk], the round's
// keys and values [kRound] each
__host__ __device__ __forceinline__ size_t rank_scatter_smem(int nbk) {
  return ((size_t)kBinWarps * (nbk + 1) + nbk + 2 * (size_t)kRound) * sizeof(uint32_t);
}

__device__ __forceinline__ void cp_async4(uint32_t* dst, const uint32_t* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src));
}

__global__ void __launch_bounds__(kBinThreads, 4)
k_rank_scatter(const uint32_t* __restrict__ keys, const uint32_t* __restrict__ vals, KeyMap km,
               int shift, uint32_t mask, int nbk, Segs sg, const int* __restrict__ hist_scan,
               uint32_t* __restrict__ kout, uint32_t* __restrict__ vout) {
  extern __shared__ uint32_t s_mem[];
  __shared__ uint32_t s_warp[32];
  const int ncol = nbk + 1;                       // column nbk: the items past the end
  uint32_t* s_cnt = s_mem;                        // [kBinWarps][ncol]
  uint32_t* s_base = s_cnt + kBinWarps * ncol;    // [nbk]
  uint32_t* s_key = s_base + nbk;                 // [kRound] values as read, then keys in bucket order
  uint32_t* s_val = s_key + kRound;               // [kRound] values in bucket order
  const BlockRange r = block_range(sg, blockIdx.x);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t kmin = km.kbits ? view_kmin(km.kbits, r.v) : 0u;
  const int* h = hist_scan + (size_t)nbk * r.b0;
  for (int t = threadIdx.x; t < nbk; t += kBinThreads) s_base[t] = (uint32_t)h[(size_t)t * r.nbv + r.lb];
  const uint32_t lt = lanemask_lt();
  const unsigned long long lim =
      sg.per_view >= 0 ? (unsigned long long)sg.per_view * sg.V : (unsigned long long)sg.vstart[sg.V];
  const int bpt = scan_bpt(nbk);
  const int sb0 = threadIdx.x * bpt, sb1 = min(sb0 + bpt, ncol);
  const int wo = warp * kWarpRound + lane;
  uint32_t* cnt = s_cnt + warp * ncol;
  for (long long rb = r.beg; rb < r.end; rb += kRound) {
    const int n = (int)min((long long)kRound, r.end - rb);
    for (int t = threadIdx.x; t < kBinWarps * ncol; t += kBinThreads) s_cnt[t] = 0;
    // the values go to shared memory asynchronously (read at the layout step), the keys to
    // registers
    if (vals)
      for (int j = threadIdx.x; j < n; j += kBinThreads) cp_async4(s_key + j, vals + rb + j);
    asm volatile("cp.async.commit_group;\n" ::);
    const uint32_t* kq = keys + rb + wo;
    uint32_t key[kRoundIpt], rank[kRoundIpt / 2];  // ranks: two 16-bit halves per word
    if (n == kRound) {
#pragma unroll
      for (int u = 0; u < kRoundIpt; ++u) key[u] = map_key(kq[32 * u], kmin, km.top);
    } else {
#pragma unroll
      for (int u = 0; u < kRoundIpt; ++u)
        key[u] = wo + 32 * u < n ? map_key(kq[32 * u], kmin, km.top) : 0u;
    }
    __syncthreads();
    // rank inside the warp: earlier items of the same bucket, in (batch, lane) order
#pragma unroll
    for (int u = 0; u < kRoundIpt; ++u) {
      const uint32_t bk = wo + 32 * u < n ? (key[u] >> shift) & mask : (uint32_t)nbk;
      const uint32_t peers = __match_any_sync(0xffffffffu, bk);
      const uint32_t c = cnt[bk];
      const uint32_t rk = c + __popc(peers & lt);  // < kWarpRound
      rank[u / 2] = (u & 1) ? rank[u / 2] | (rk << 16) : rk;
      __syncwarp();
      if (lane == __ffs(peers) - 1) cnt[bk] = c + __popc(peers);
      __syncwarp();
    }
    __syncthreads();
    // exclusive scan of the counts in (bucket, warp) order; row 0 then holds the bucket starts
    uint32_t sum = 0;
    for (int b = sb0; b < sb1; ++b)
#pragma unroll
      for (int ww = 0; ww < kBinWarps; ++ww) sum += s_cnt[ww * ncol + b];
    uint32_t off = block_exclusive_scan<uint32_t>(sum, s_warp, nullptr);
    for (int b = sb0; b < sb1; ++b)
#pragma unroll
      for (int ww = 0; ww < kBinWarps; ++ww) {
        const uint32_t c = s_cnt[ww * ncol + b];
        s_cnt[ww * ncol + b] = off;
        off += c;
      }
    asm volatile("cp.async.wait_group 0;\n" ::: "memory");
    __syncthreads();
    // the round in bucket order: first the values (read from where they landed in s_key), then,
    // once every value is read, the keys
    const uint32_t vbase = (uint32_t)(rb - r.vbeg) + (uint32_t)wo;
#pragma unroll
    for (int u = 0; u < kRoundIpt; ++u) {
      if (wo + 32 * u < n) {
        const uint32_t lp = cnt[(key[u] >> shift) & mask] + ((rank[u / 2] >> (16 * (u & 1))) & 0xffffu);
        s_val[lp] = vals ? s_key[wo + 32 * u] : vbase + 32 * u;
      }
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kRoundIpt; ++u) {
      if (wo + 32 * u < n) {
        const uint32_t lp = cnt[(key[u] >> shift) & mask] + ((rank[u / 2] >> (16 * (u & 1))) & 0xffffu);
        s_key[lp] = key[u];
      }
    }
    __syncthreads();
    for (int j = threadIdx.x; j < n; j += kBinThreads) {
      const uint32_t k = s_key[j];
      const uint32_t bk = (k >> shift) & mask;
      const uint32_t pos = s_base[bk] + (uint32_t)j - s_cnt[bk];
      if (in_bounds(pos, lim, &g_bounds_word)) {
        if (kout) kout[pos] = k;
        vout[pos] = s_val[j];
      }
    }
    __syncthreads();
    for (int b = threadIdx.x; b < nbk; b += kBinThreads) s_base[b] += s_cnt[b + 1] - s_cnt[b];
    __syncthreads();
  }
}

// tile rectangles and their tile counts in depth order (order == nullptr: index order)
__global__ void k_gather_rects(const ushort4* __restrict__ rect, const uint32_t* __restrict__ order,
                               long long VG, int G, ushort4* __restrict__ rect_s,
                               int* __restrict__ cnt_s) {
  const long long k = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= VG) return;
  const long long v = k / G;
  const uint32_t g = order ? order[k] : (uint32_t)(k - v * G);
  const ushort4 rc = rect[v * G + g];
  rect_s[k] = rc;
  cnt_s[k] = ((int)rc.z - (int)rc.x) * ((int)rc.w - (int)rc.y);
}

// instances (tile, g) in depth order. One warp per 32 consecutive entries: the lanes write the
// warp's output range in order, 32 consecutive positions at a time (coalesced, and balanced
// however many tiles each entry covers); each position finds its entry by a binary search over
// the 32 entry offsets, then its tile from its index inside the entry's rectangle (row-major).
__global__ void __launch_bounds__(256)
k_emit(const ushort4* __restrict__ rect_s, const uint32_t* __restrict__ order,
       const int* __restrict__ offs, long long VG, long long n_inst, int G, int TX,
       uint32_t* __restrict__ inst_tile, uint32_t* __restrict__ inst_g) {
  const int lane = threadIdx.x & 31;
  const long long k0 = (long long)blockIdx.x * blockDim.x + (threadIdx.x & ~31);
  if (k0 >= VG) return;  // warp-uniform
  const long long k = k0 + lane;
  const bool ok = k < VG;
  int x0e = 0, y0e = 0, wdt = 0;
  uint32_t g = 0;
  if (ok) {
    const ushort4 rc = rect_s[k];
    x0e = rc.x;
    y0e = rc.y;
    wdt = (int)rc.z - (int)rc.x;
    const long long v = k / G;
    g = order ? order[k] : (uint32_t)(k - v * G);
  }
  // offs: exclusive scan of the entries' tile counts (int32: the instance total is below 2^31)
  const int start = offs[k0];
  const int total = (k0 + 32 < VG ? offs[k0 + 32] : (int)n_inst) - start;
  // entry start relative to the warp's range; lanes past the end sit at the end (never chosen)
  const int rel = ok ? offs[k] - start : total;
  const unsigned long long lim = kChecked ? (unsigned long long)n_inst : 0ull;
  for (int b = 0; b < total; b += 32) {
    const int p = b + lane;
    // the last entry whose start is <= p (starts are non-decreasing; entry 0 starts at 0)
    int j = 0;
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1)
      if (__shfl_sync(0xffffffffu, rel, j + s) <= p) j += s;
    const int x0 = __shfl_sync(0xffffffffu, x0e, j);
    const int y0 = __shfl_sync(0xffffffffu, y0e, j);
    const int wj = __shfl_sync(0xffffffffu, wdt, j);
    const int rj = __shfl_sync(0xffffffffu, rel, j);
    const uint32_t gj = __shfl_sync(0xffffffffu, g, j);
    if (p < total) {
      const int li = p - rj;  // wj > 0: an entry with an empty rectangle owns no position
      const int dy = (int)((unsigned)li / (unsigned)wj);
      const long long pos = start + p;
      if (in_bounds(pos, lim, &g_bounds_word)) {
        inst_tile[pos] = (uint32_t)((y0 + dy) * TX + x0 + (li - dy * wj));
        inst_g[pos] = gj;
      }
    }
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

// Launch order of the (tile, view) CTAs of the kernels that walk the lists: longest list first.
// The CTAs of a launch start in block-index order, so the long lists start in the first waves and
// the last wave holds short ones instead of leaving SMs idle behind one long list. Length classes
// of eight per octave (the leading bit and the next three, monotone in the length); inside a class
// the tiles keep their (view, row, column) order, so neighbouring tiles, which share Gaussians,
// still run close together. One block: a stable counting sort over 32 warp segments, the same
// scheme as the binning passes (per-warp class counts, a scan over (class, warp), match.any
// ranking).
constexpr int kOrderThreads = 1024;
constexpr int kOrderWarps = kOrderThreads / 32;
constexpr int kOrderClasses = 256;

__device__ __forceinline__ int len_class(const long long* __restrict__ tile_off, int nt, int k) {
  const int v = k / nt;
  const long long* o = tile_off + (size_t)v * (nt + 1) + (k - v * nt);
  const long long len = o[1] - o[0];
  if (len <= 0) return kOrderClasses - 1;  // empty lists last
  const unsigned long long u = (unsigned long long)len;
  const int msb = 63 - __clzll(u);
  const int frac = msb >= 3 ? (int)((u >> (msb - 3)) & 7u) : (int)((u << (3 - msb)) & 7u);
  return kOrderClasses - 2 - (min(msb, 30) * 8 + frac);  // longest lists in the lowest class
}

__global__ void __launch_bounds__(kOrderThreads)
k_tile_order(const long long* __restrict__ tile_off, int V, int nt, int* __restrict__ order) {
  __shared__ int s_cnt[kOrderWarps * kOrderClasses];  // [warp][class]
  __shared__ int s_warp[32];
  const int n = V * nt;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per = (n + kOrderWarps - 1) / kOrderWarps;
  const int kb = min(n, warp * per), ke = min(n, kb + per);
  for (int c = threadIdx.x; c < kOrderWarps * kOrderClasses; c += blockDim.x) s_cnt[c] = 0;
  __syncthreads();
  for (int k = kb + lane; k < ke; k += 32) atomicAdd(&s_cnt[warp * kOrderClasses + len_class(tile_off, nt, k)], 1);
  __syncthreads();
  // exclusive scan in (class, warp) order: thread t owns entries 8t .. 8t + 7 of that order
  constexpr int kPer = kOrderWarps * kOrderClasses / kOrderThreads;
  int c[kPer], sum = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = kPer * threadIdx.x + i;
    c[i] = s_cnt[(e % kOrderWarps) * kOrderClasses + e / kOrderWarps];
    sum += c[i];
  }
  int run = block_exclusive_scan<int>(sum, s_warp, nullptr);
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = kPer * threadIdx.x + i;
    s_cnt[(e % kOrderWarps) * kOrderClasses + e / kOrderWarps] = run;
    run += c[i];
  }
  __syncthreads();
  // each warp places its segment in order; equal classes inside a batch of 32 ranked by lane
  const uint32_t lt = lanemask_lt();
  int* cnt = s_cnt + warp * kOrderClasses;
  for (int base = kb; base < ke; base += 32) {
    const int k = base + lane;
    const bool ok = k < ke;
    const int cl = ok ? len_class(tile_off, nt, k) : -1 - lane;  // unique for idle lanes
    const uint32_t peers = __match_any_sync(0xffffffffu, cl);
    if (ok) {
      const int pos = cnt[cl] + __popc(peers & lt);
      if (in_bounds(pos, (unsigned long long)n, &g_bounds_word)) order[pos] = k;
    }
    __syncwarp();
    if (ok && lane == __ffs(peers) - 1) cnt[cl] += __popc(peers);
    __syncwarp();
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

int ensure_hist(Workspace& w, size_t n) {
  if (n + 1 <= w.hist_cap) return SPLAT_OK;
  const size_t cap = n + n / 4 + 1024;
  const int rc = grow(w, &w.hist, cap, "bucket histogram");
  w.hist_cap = rc ? 0 : cap;
  return rc;
}

}  // namespace

namespace {
__global__ void k_zero(uint4* __restrict__ p16, size_t n16, uint32_t* __restrict__ p4, size_t n4) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t k = (size_t)blockIdx.x * blockDim.x + threadIdx.x; k < n16; k += stride)
    p16[k] = make_uint4(0u, 0u, 0u, 0u);
  for (size_t k = (size_t)blockIdx.x * blockDim.x + threadIdx.x; k < n4; k += stride) p4[k] = 0u;
}
__global__ void k_copy_words(const uint32_t* __restrict__ src, uint32_t* __restrict__ dst, size_t n) {
  for (size_t k = (size_t)blockIdx.x * blockDim.x + threadIdx.x; k < n;
       k += (size_t)gridDim.x * blockDim.x)
    dst[k] = src[k];
}
}  // namespace

int zero_async(Workspace& w, void* p, size_t bytes, cudaStream_t st, const char* what) {
  if (bytes == 0) return SPLAT_OK;
  if (((uintptr_t)p & 15) || (bytes & 3))
    return set_err(w, SPLAT_ERR_INVALID_ARG, std::string(what) + ": clear of an unaligned range");
  const size_t n16 = bytes / 16, n4 = (bytes - n16 * 16) / 4;
  const size_t want = (n16 + 255) / 256;
  const unsigned blocks = (unsigned)(want < 148 * 8 ? (want > 0 ? want : 1) : 148 * 8);
  k_zero<<<blocks, 256, 0, st>>>(reinterpret_cast<uint4*>(p), n16,
                                 reinterpret_cast<uint32_t*>(static_cast<char*>(p) + n16 * 16), n4);
  return check_launch(w, what);
}

int copy_words(Workspace& w, const void* src, void* dst, size_t bytes, cudaStream_t st,
               const char* what) {
  if (bytes == 0) return SPLAT_OK;
  if ((bytes & 3) || ((uintptr_t)src & 3) || ((uintptr_t)dst & 3))
    return set_err(w, SPLAT_ERR_INVALID_ARG, std::string(what) + ": copy of an unaligned range");
  const size_t n = bytes / 4;
  const unsigned blocks = (unsigned)((n + 255) / 256 < 64 ? (n + 255) / 256 : 64);
  k_copy_words<<<blocks, 256, 0, st>>>(static_cast<const uint32_t*>(src),
                                       static_cast<uint32_t*>(dst), n);
  return check_launch(w, what);
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


// one stable counting-sort pass (histogram, scan, scatter; runs: the scatter through bucket runs)
static int count_pass(Workspace& w, cudaStream_t st, const uint32_t* keys, const uint32_t* vals,
                      KeyMap km, int shift, uint32_t mask, int nbk, const Segs& sg, int nblocks,
                      uint32_t* kout, uint32_t* vout, int id_hist, int id_scatter, bool runs) {
  int rc;
  const size_t hist_n = (size_t)nbk * nblocks;
  if ((rc = ensure_hist(w, hist_n))) return rc;
  const size_t smem = (size_t)kBinWarps * nbk * sizeof(uint32_t);
  int tok = prof_begin(w, st, id_hist);
  k_count_hist<<<nblocks, kBinThreads, smem, st>>>(keys, km, shift, mask, nbk, sg, w.hist);
  prof_end(w, st, tok);
  if ((rc = check_launch(w, "histogram kernel"))) return rc;
  tok = prof_begin(w, st, SPLAT_K_HIST_SCAN);
  rc = scan_i32_inplace(w, w.hist, (long long)hist_n, st);
  prof_end(w, st, tok);
  if (rc) return rc;
  tok = prof_begin(w, st, id_scatter);
  if (runs)
    k_rank_scatter<<<nblocks, kBinThreads, rank_scatter_smem(nbk), st>>>(keys, vals, km, shift, mask,
                                                                        nbk, sg, w.hist, kout, vout);
  else
    k_count_scatter<<<nblocks, kBinThreads, smem, st>>>(keys, vals, km, shift, mask, nbk, sg, w.hist,
                                                         kout, vout);
  prof_end(w, st, tok);
  return check_launch(w, "scatter kernel");
}

// after the host has read the per-view instance starts (h_vstart) and key statistics (h_kbits)
int launch_binning(Workspace& w, cudaStream_t st) {
  int rc;
  const long long N = w.n_total;
  const long long VG = (long long)w.V * w.G;
  if (N > (long long)w.inst_cap) {
    const size_t cap = (size_t)(N + N / 4 + 1024);
    if ((rc = grow(w, &w.inst_tile, cap, "instance tiles"))) return rc;
    if ((rc = grow(w, &w.inst_g, cap, "instance indices"))) return rc;
    if ((rc = grow(w, &w.sval, cap, "tile lists"))) return rc;
    w.inst_cap = cap;
  }
  {
    const size_t need = ((size_t)N / 32 + (size_t)w.V * w.nt + 2) * 8;
    if (need > w.umask_cap) {
      const size_t cap = need + need / 4;
      if ((rc = grow(w, &w.umask, cap, "composited-entry masks"))) return rc;
      w.umask_cap = cap;
    }
  }
  {
    const size_t need = ((size_t)(N >> 7) + (size_t)w.V * w.nt + 1) * 1024;
    if (need > w.lmask_cap) {
      const size_t cap = need + need / 4;
      if ((rc = grow(w, &w.lmask, cap, "per-pixel composited-entry masks"))) return rc;
      w.lmask_cap = cap;
    }
  }
  // ---- 1. depth order of every view's Gaussians --------------------------------------------
  // width of the widest view's visible key range -> number of digit passes
  uint32_t range = 0;
  for (int v = 0; v < w.V; ++v) {
    uint32_t khi = 0, klo = 0;
    for (int sidx = 0; sidx < kKeyStripes; ++sidx) {
      khi = max(khi, w.h_kbits[2 * (v * kKeyStripes + sidx)]);
      klo = max(klo, w.h_kbits[2 * (v * kKeyStripes + sidx) + 1]);
    }
    if (khi) range = max(range, khi - ~klo);  // no visible key: both stay 0
  }
  const int bits = range ? 32 - __builtin_clz(range) : 0;
  const KeyMap map0{w.kbits, bits >= 32 ? 0xffffffffu : (1u << bits) - 1u};
  const int passes = bits == 0 ? 0 : (bits + kDepthDigitMax - 1) / kDepthDigitMax;
  const int dbits = passes ? (bits + passes - 1) / passes : 0;
  const uint32_t* order = nullptr;  // sorted Gaussian indices per view (nullptr: index order)
  if (passes > 0 && VG > 0) {
    Segs sg{w.G, (int)((w.G + kDepthChunk - 1) / kDepthChunk), nullptr, nullptr, w.V, kDepthChunk};
    const int nblocks = sg.blocks_per_view * w.V;
    const uint32_t* kin = w.dkey;
    const uint32_t* vin = nullptr;
    uint32_t* kb[2] = {w.dk1, w.dk2};
    uint32_t* vb[2] = {w.dv0, w.dv1};
    for (int p = 0; p < passes; ++p) {
      const int shift = p * dbits;
      const int width = min(dbits, 32 - shift);
      const uint32_t mask = (width >= 32) ? 0xffffffffu : ((1u << width) - 1u);
      uint32_t* kout = (p + 1 < passes) ? kb[p & 1] : nullptr;
      uint32_t* vout = vb[p & 1];
      const KeyMap km = p == 0 ? map0 : KeyMap{nullptr, 0xffffffffu};
      if ((rc = count_pass(w, st, kin, vin, km, shift, mask, (int)mask + 1, sg, nblocks, kout,
                           vout, SPLAT_K_DEPTH_HIST, SPLAT_K_DEPTH_SCATTER, true)))
        return rc;
      kin = kout;
      vin = vout;
    }
    order = vin;
  }
  // ---- 2. rectangles in depth order, their offsets, instance emission -------------------------
  if (VG > 0) {
    int tok = prof_begin(w, st, SPLAT_K_EMIT);
    const unsigned grid = (unsigned)((VG + 255) / 256);
    k_gather_rects<<<grid, 256, 0, st>>>(w.rect, order, VG, w.G, w.rect_s, w.counts);
    if ((rc = check_launch(w, "rectangle gather kernel"))) return rc;
    if ((rc = scan_i32_inplace(w, w.counts, VG, st))) return rc;
    k_emit<<<grid, 256, 0, st>>>(w.rect_s, order, w.counts, VG, N, w.G, w.TX, w.inst_tile,
                                 w.inst_g);
    prof_end(w, st, tok);
    if ((rc = check_launch(w, "emit kernel"))) return rc;
  }
  // ---- 3. stable counting sort by tile --------------------------------------------------------
  w.h_bstart[0] = 0;
  for (int v = 0; v < w.V; ++v) {
    const long long nv = w.h_vstart[v + 1] - w.h_vstart[v];
    w.h_bstart[v + 1] = w.h_bstart[v] + (int)((nv + kTileChunk - 1) / kTileChunk);
  }
  w.n_blocks = w.h_bstart[w.V];
  if ((rc = copy_words(w, w.hd_vstart, w.d_vstart, (w.V + 1) * sizeof(long long), st,
                       "view starts upload")) ||
      (rc = copy_words(w, w.hd_bstart, w.d_bstart, (w.V + 1) * sizeof(int), st,
                       "block starts upload")))
    return rc;
  if (N > 0) {
    Segs sg{-1, 0, w.d_vstart, w.d_bstart, w.V, kTileChunk};
    if ((rc = count_pass(w, st, w.inst_tile, w.inst_g, KeyMap{nullptr, 0xffffffffu}, 0,
                         0xffffffffu, w.nt, sg, w.n_blocks, nullptr, w.sval, SPLAT_K_TILE_HIST,
                         SPLAT_K_TILE_SCATTER, false)))
      return rc;
  } else if ((rc = ensure_hist(w, 1))) {
    return rc;
  }
  const int nr = w.V * (w.nt + 1);
  const int tok_r = prof_begin(w, st, SPLAT_K_TILE_RANGES);
  k_tile_ranges<<<(nr + 255) / 256, 256, 0, st>>>(w.hist, w.d_vstart, w.d_bstart, w.V, w.nt,
                                                  w.tile_off);
  if ((rc = check_launch(w, "tile ranges kernel"))) {
    prof_end(w, st, tok_r);
    return rc;
  }
  if (w.V * w.nt > 0) {
    k_tile_order<<<1, kOrderThreads, 0, st>>>(w.tile_off, w.V, w.nt, w.tile_order);
    rc = check_launch(w, "tile order kernel");
  }
  prof_end(w, st, tok_r);
  return rc;
}

// shared-memory opt-in for the counting-sort kernels (called once per workspace)
int binning_configure(Workspace& w) {
  const int nbk = max(w.max_nt, 2048);
  const size_t need_hist = (size_t)kBinWarps * nbk * sizeof(uint32_t);
  cudaError_t e2 = cudaFuncSetAttribute(k_count_hist, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)need_hist);
  // (the runs scatter serves only the depth passes: at most 2^kDepthDigitMax buckets)
  cudaError_t e3 = cudaFuncSetAttribute(k_rank_scatter, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)rank_scatter_smem(1 << kDepthDigitMax));
  cudaError_t e4 = cudaFuncSetAttribute(k_count_scatter, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)need_hist);
  if (e2 != cudaSuccess || e3 != cudaSuccess || e4 != cudaSuccess) {
    cudaGetLastError();
    return set_err(w, SPLAT_ERR_CAPACITY,
                   "image has too many tiles for the binning kernels' shared memory");
  }
  return SPLAT_OK;
}

}  // namespace splat
