// Depth ordering without any device allocation.
//
// Some callers cannot allocate device memory at the point where they need an ordering: code that
// runs inside another framework's memory pool or allocator hooks, plugins that are handed fixed
// buffers, or phases where cudaMalloc/cudaFree would synchronise the device or fail for lack of
// memory. splat_sort_depths_noalloc gives them the contributor ordering of the tile binning (the
// stable sort of fp32 depths, ties kept in index order) while allocating nothing: its ping-pong
// scratch is a file-scope __device__ array of fixed size, present on every GPU that loads this
// library until the process exits. The caller passes only its input and output buffers.
//
// For the positive depths the projection produces, the result equals the binning's per-view depth
// order (the binning sorts the raw fp32 bits of each view's visible depths, stably, and emits
// every tile's list in that order), so it is also the order of each tile's contributors. The
// order of negative values, -0.0 and NaNs is this entry point's own (an order-preserving map of
// the fp32 bits). One CTA runs a stable least-significant-digit radix sort with 8-bit digits
// over that 32-bit image of the depths, keeping per-warp digit counters in shared memory.
#include "common.cuh"

namespace splat {
namespace {

constexpr int kNaMax = SPLAT_NOALLOC_MAX_N;
constexpr int kNaWarps = 16;
constexpr int kNaThreads = kNaWarps * 32;

// ping-pong keys and values: [2][kNaMax] + [2][kNaMax] 32-bit words (4 MiB at 2^18 entries)
static __device__ __align__(256) uint32_t g_noalloc_scratch[4 * kNaMax];

__device__ __forceinline__ uint32_t na_lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// order-preserving map of an IEEE fp32 to an unsigned key (negative values reversed)
__device__ __forceinline__ uint32_t float_key(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ uint32_t na_block_exclusive_scan(uint32_t v, uint32_t* s_warp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t u = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += u;
  }
  if (lane == 31) s_warp[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const uint32_t x = lane < kNaWarps ? s_warp[lane] : 0u;
    uint32_t xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xffffffffu, xi, o);
      if (lane >= o) xi += u;
    }
    if (lane < kNaWarps) s_warp[lane] = xi - x;
  }
  __syncthreads();
  const uint32_t r = s_warp[warp] + inc - v;
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kNaThreads)
k_sort_depths_noalloc(const float* __restrict__ depths, int n, uint32_t* scratch,
                      int* __restrict__ order) {
  __shared__ uint32_t cnt[kNaWarps * 256];
  __shared__ uint32_t s_warp[32];
  uint32_t* K[2] = {scratch, scratch + kNaMax};
  uint32_t* Vv[2] = {scratch + 2 * kNaMax, scratch + 3 * kNaMax};
  // every scratch word read below is written first in this call: nothing needs clearing
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    K[0][i] = float_key(depths[i]);
    Vv[0][i] = (uint32_t)i;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per = (((n + kNaWarps - 1) / kNaWarps) + 31) & ~31;
  const int wb = warp * per, we = min(n, wb + per);
  const uint32_t lt = na_lanemask_lt();
  for (int p = 0; p < 4; ++p) {
    const uint32_t* kin = K[p & 1];
    const uint32_t* vin = Vv[p & 1];
    uint32_t* kout = K[(p & 1) ^ 1];
    uint32_t* vout = Vv[(p & 1) ^ 1];
    const int shift = 8 * p;
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
    {  // exclusive scan in (digit, warp) order; thread t owns digit t/2, warps (t&1)*8 .. +8
      const int d = threadIdx.x >> 1, w0 = (threadIdx.x & 1) * 8;
      uint32_t vals[8];
      uint32_t s = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t c = cnt[(w0 + k) * 256 + d];
        vals[k] = s;
        s += c;
      }
      const uint32_t ex = na_block_exclusive_scan(s, s_warp);
#pragma unroll
      for (int k = 0; k < 8; ++k) cnt[(w0 + k) * 256 + d] = ex + vals[k];
    }
    __syncthreads();
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
  // four passes: the result is back in buffer 0
  for (int i = threadIdx.x; i < n; i += blockDim.x) order[i] = (int)Vv[0][i];
}

}  // namespace
}  // namespace splat

extern "C" int splat_sort_depths_noalloc(const float* depths, int n, int* order, void* stream) {
  using namespace splat;
  if (n < 0 || (n > 0 && (!depths || !order))) return SPLAT_ERR_INVALID_ARG;
  if (n > kNaMax) return SPLAT_ERR_CAPACITY;
  if (n == 0) return SPLAT_OK;
  // The array's device address in the current device's context, looked up on every call: host
  // code cannot use the symbol itself (a host-side stand-in), and a cached address would go
  // stale when the module is loaded again (after cudaDeviceReset, or in another context). The
  // lookup is host-side, not a stream operation; the first one on a device also loads the module.
  void* scratch = nullptr;
  if (cudaGetSymbolAddress(&scratch, g_noalloc_scratch) != cudaSuccess || !scratch) {
    cudaGetLastError();
    return SPLAT_ERR_CUDA;
  }
  k_sort_depths_noalloc<<<1, kNaThreads, 0, (cudaStream_t)stream>>>(
      depths, n, static_cast<uint32_t*>(scratch), order);
  if (cudaGetLastError() != cudaSuccess) return SPLAT_ERR_CUDA;
  return SPLAT_OK;
}
