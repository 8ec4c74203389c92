// gsg_route.cu -- MoE routing permutation (stable counting sort of routed rows by expert).
//
// "Hardware-Native Joint Sparse-Quantization for Trillion-Scale Mixture-of-Experts"
// (paperlayer.ai summary): §2 "Execution gap" (p.3) -- the grouped GEMM runs routing-dependent
// expert problems with different token counts together; §D.1 (p.19) -- dispatch/scatter.
//
// Routed pair (t, j) has flat index f = t*k + j; rows of expert e are [off[e], off[e+1]) in
// ascending f.  Work is split into chunks of kRouteChunk flat indices, one 1024-thread block per
// chunk and 32 sub-chunks (one per warp).  Within a warp, equal ids are ranked with
// __match_any_sync; per-warp histograms live in shared memory (32 x E ints).  A single chunk
// (R <= kRouteChunk) runs as one launch; larger R uses histogram -> scan -> scatter launches
// with a [chunks x E] workspace.  The result is deterministic.
#include "gsg_internal.cuh"

namespace gsg {

constexpr int kRouteThreads = 1024;
constexpr int kRouteChunk = 8192;
constexpr int kRouteMaxE = 1024;

// A warp's sub-chunk holds at most kRouteChunk / 32 = 256 flat indices: eight per lane, loaded
// once into registers (all loads in flight together) and reused by both passes.
constexpr int kPerLane = kRouteChunk / (32 * 32);

__device__ __forceinline__ void warp_load_ids(const int32_t* __restrict__ ids, int f0, int f1, int E,
                                              int x[kPerLane], int* status) {
  const int lane = threadIdx.x & 31;
  bool bad = false;
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) {
    const int f = f0 + 32 * i + lane;
    x[i] = f < f1 ? __ldg(ids + f) : -1;
  }
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) {
    const int f = f0 + 32 * i + lane;
    if (f < f1 && (x[i] < 0 || x[i] >= E)) { bad = true; x[i] = -1; }
  }
  if (bad && status != nullptr) set_status(status, GSG_ERR_BAD_ROUTING);
}

// Per-warp histogram of the warp's ids.  hist row = this warp's E counters.
__device__ __forceinline__ void warp_histogram(const int x[kPerLane], int* hist) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) {
    const unsigned mask = __match_any_sync(0xffffffffu, x[i]);
    if (x[i] >= 0 && lane == __ffs(mask) - 1) hist[x[i]] += __popc(mask);
    __syncwarp();
  }
}

// Stable scatter of the warp's ids; base[x] = first row of id x for this warp (advanced).
__device__ __forceinline__ void warp_scatter(const int x[kPerLane], int f0, int* base, int32_t* perm_src,
                                             int32_t* inv_perm) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) {
    const int f = f0 + 32 * i + lane;
    const unsigned mask = __match_any_sync(0xffffffffu, x[i]);
    if (x[i] >= 0) {
      const int pos = base[x[i]] + __popc(mask & lt);
      perm_src[pos] = f;
      inv_perm[f] = pos;
    }
    __syncwarp();
    if (x[i] >= 0 && lane == __ffs(mask) - 1) base[x[i]] += __popc(mask);
    __syncwarp();
  }
}

// Exclusive scan of v over the block (blockDim.x == 1024); returns this thread's prefix.
__device__ int block_exclusive_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    warp_sums[lane] = wi - w;
    if (lane == 31) *total = wi;
  }
  __syncthreads();
  return warp_sums[warp] + incl - v;
}

__device__ __forceinline__ void sub_chunk(int c0, int c1, int& f0, int& f1) {
  const int per = ((c1 - c0) + 31) / 32;
  const int warp = threadIdx.x >> 5;
  f0 = c0 + warp * per;
  f1 = min(f0 + per, c1);
  if (f0 > c1) f0 = c1;
}

// One chunk holds everything: histogram, scan, scatter in one launch.
__global__ void __launch_bounds__(kRouteThreads)
route_single_kernel(const int32_t* __restrict__ ids, int R, int E, int32_t* off, int32_t* perm_src,
                    int32_t* inv_perm, int* status) {
  extern __shared__ int hist[];  // [32][E]
  __shared__ int warp_sums[32];
  __shared__ int total;
  for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  int f0, f1;
  sub_chunk(0, R, f0, f1);
  int x[kPerLane];
  warp_load_ids(ids, f0, f1, E, x, status);
  warp_histogram(x, hist + warp * E);
  __syncthreads();
  const int ex = threadIdx.x;
  int tot = 0;
  if (ex < E)
    for (int w = 0; w < 32; ++w) tot += hist[w * E + ex];
  const int start = block_exclusive_scan(tot, warp_sums, &total);
  if (ex < E) {
    off[ex] = start;
    int run = start;
    for (int w = 0; w < 32; ++w) {
      int c = hist[w * E + ex];
      hist[w * E + ex] = run;
      run += c;
    }
  }
  if (ex == 0) off[E] = total;
  __syncthreads();
  warp_scatter(x, f0, hist + warp * E, perm_src, inv_perm);
}

// Multi-chunk path, launch 1: per-chunk histograms -> ws_hist[chunk][E].
__global__ void __launch_bounds__(kRouteThreads)
route_hist_kernel(const int32_t* __restrict__ ids, int R, int E, int* ws_hist, int* status) {
  extern __shared__ int hist[];
  for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int c0 = blockIdx.x * kRouteChunk, c1 = min(c0 + kRouteChunk, R);
  int f0, f1;
  sub_chunk(c0, c1, f0, f1);
  int x[kPerLane];
  warp_load_ids(ids, f0, f1, E, x, status);
  warp_histogram(x, hist + (threadIdx.x >> 5) * E);
  __syncthreads();
  for (int x = threadIdx.x; x < E; x += blockDim.x) {
    int s = 0;
    for (int w = 0; w < 32; ++w) s += hist[w * E + x];
    ws_hist[(size_t)blockIdx.x * E + x] = s;
  }
}

// Launch 2 (one block): offsets and each chunk's first row per expert -> ws_base[chunk][E].
__global__ void __launch_bounds__(kRouteThreads)
route_scan_kernel(const int* ws_hist, int nchunks, int E, int32_t* off, int* ws_base) {
  __shared__ int warp_sums[32];
  __shared__ int total;
  const int x = threadIdx.x;
  int tot = 0;
  if (x < E)
    for (int b = 0; b < nchunks; ++b) tot += ws_hist[(size_t)b * E + x];
  const int start = block_exclusive_scan(tot, warp_sums, &total);
  if (x < E) {
    off[x] = start;
    int run = start;
    for (int b = 0; b < nchunks; ++b) {
      int c = ws_hist[(size_t)b * E + x];
      ws_base[(size_t)b * E + x] = run;
      run += c;
    }
  }
  if (x == 0) off[E] = total;
}

// Launch 3: per chunk, warp bases from the chunk base, then the stable scatter.
__global__ void __launch_bounds__(kRouteThreads)
route_scatter_kernel(const int32_t* __restrict__ ids, int R, int E, const int* ws_base,
                     int32_t* perm_src, int32_t* inv_perm) {
  extern __shared__ int hist[];
  for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int c0 = blockIdx.x * kRouteChunk, c1 = min(c0 + kRouteChunk, R);
  int f0, f1;
  sub_chunk(c0, c1, f0, f1);
  const int warp = threadIdx.x >> 5;
  int x[kPerLane];
  warp_load_ids(ids, f0, f1, E, x, nullptr);
  warp_histogram(x, hist + warp * E);
  __syncthreads();
  for (int x = threadIdx.x; x < E; x += blockDim.x) {
    int run = ws_base[(size_t)blockIdx.x * E + x];
    for (int w = 0; w < 32; ++w) {
      int c = hist[w * E + x];
      hist[w * E + x] = run;
      run += c;
    }
  }
  __syncthreads();
  warp_scatter(x, f0, hist + warp * E, perm_src, inv_perm);
}

int route_chunks(int R) { return R <= kRouteChunk ? 1 : (R + kRouteChunk - 1) / kRouteChunk; }

size_t route_workspace_bytes(int R, int E) {
  const int nc = route_chunks(R);
  return nc <= 1 ? 0 : (size_t)2 * nc * E * sizeof(int);
}

bool route_supported(int E) { return E >= 1 && E <= kRouteMaxE; }

cudaError_t route_set_smem_attrs() {
  const int bytes = 32 * kRouteMaxE * (int)sizeof(int);
  cudaError_t e1 = cudaFuncSetAttribute(route_single_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  cudaError_t e2 = cudaFuncSetAttribute(route_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  cudaError_t e3 = cudaFuncSetAttribute(route_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e1 != cudaSuccess) return e1;
  if (e2 != cudaSuccess) return e2;
  return e3;
}

cudaError_t launch_route(const int32_t* ids, int R, int E, int32_t* off, int32_t* perm_src,
                         int32_t* inv_perm, void* ws, int* status, cudaStream_t stream) {
  const size_t smem = (size_t)32 * E * sizeof(int);
  const int nc = route_chunks(R);
  if (nc <= 1) {
    route_single_kernel<<<1, kRouteThreads, smem, stream>>>(ids, R, E, off, perm_src, inv_perm, status);
    return cudaGetLastError();
  }
  int* ws_hist = static_cast<int*>(ws);
  int* ws_base = ws_hist + (size_t)nc * E;
  route_hist_kernel<<<nc, kRouteThreads, smem, stream>>>(ids, R, E, ws_hist, status);
  route_scan_kernel<<<1, kRouteThreads, 0, stream>>>(ws_hist, nc, E, off, ws_base);
  route_scatter_kernel<<<nc, kRouteThreads, smem, stream>>>(ids, R, E, ws_base, perm_src, inv_perm);
  return cudaGetLastError();
}

}  // namespace gsg
