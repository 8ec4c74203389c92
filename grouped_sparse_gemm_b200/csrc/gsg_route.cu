// gsg_route.cu -- MoE routing permutation (stable counting sort of routed rows by expert).
//
// "Hardware-Native Joint Sparse-Quantization for Trillion-Scale Mixture-of-Experts"
// (paperlayer.ai summary): §2 "Execution gap" (p.3) -- the grouped GEMM runs routing-dependent
// expert problems with different token counts together; §D.1 (p.19) -- dispatch/scatter.
//
// Routed pair (t, j) has flat index f = t*k + j; rows of expert e are [off[e], off[e+1]) in
// ascending f.  The flat indices are cut into chunks, one 1024-thread block per chunk: 1024
// indices (one per thread) while ceil(R/1024) * E <= 16384 (a workspace of at most 128 KiB),
// else 8192 (eight per thread).  Each warp owns a contiguous run of its chunk; lanes holding
// the same id are found with one ballot per id bit, which gives each index its rank among equal
// ids of its warp, and per-warp histograms live in shared memory (32 x E ints).  R <= 2048 is
// one launch of one block (up to 2 indices per thread, no workspace): at these sizes the pass is
// latency-bound and a second launch costs more than the block's extra round (measured: at
// R = 4096 four indices per thread in one block are slower than two launches).  Larger R is
// histogram -> (scan) -> scatter over a [chunks x E] workspace, the scan folded into the
// scatter for 1024-index chunks.  For gsg_moe_dispatch_nvfp4 the first of these launches also
// carries the activation quantizer's amax blocks (route_amax_kernel).  Only integer arithmetic:
// the result is deterministic.
#include "gsg_internal.cuh"

namespace gsg {

constexpr int kRouteThreads = 1024;
constexpr int kRouteMaxE = 1024;
constexpr long long kSmallChunkMaxCells = 16384;   // chunks x experts of the 1024-index path
constexpr int kSingleMaxR = 2048;                  // one block, up to 2 indices per thread
constexpr int kDispatchMaxAmaxBlocks = 256;        // amax blocks added to the first routing launch

int route_chunk_size(int R, int E) {
  return ((long long)(R + 1023) / 1024) * E <= kSmallChunkMaxCells ? 1024 : 8192;
}

// Lanes of the warp holding the same key as this lane: one ballot per key bit (key = id + 1,
// so the invalid id -1 is key 0 and needs no special case).  nbits = bit length of E.
__device__ __forceinline__ unsigned peer_mask(int x, int nbits) {
  const unsigned key = (unsigned)(x + 1);
  unsigned m = 0xffffffffu;
  for (int b = 0; b < nbits; ++b) {
    const unsigned bit = (key >> b) & 1u;
    const unsigned bal = __ballot_sync(0xffffffffu, bit);
    m &= bit ? bal : ~bal;
  }
  return m;
}

__device__ __forceinline__ int key_bits(int E) { return 32 - __clz(E); }

// The ids of this warp's run [f0, f1): kPer per lane, index f0 + 32*i + lane (-1 past the end or
// out of range; an out-of-range id also records GSG_ERR_BAD_ROUTING when status is given).
template <int kPer>
__device__ __forceinline__ void warp_load_ids(const int32_t* __restrict__ ids, int f0, int f1, int E,
                                              int x[kPer], int* status) {
  const int lane = threadIdx.x & 31;
  bool bad = false;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int f = f0 + 32 * i + lane;
    x[i] = f < f1 ? __ldg(ids + f) : -1;
  }
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int f = f0 + 32 * i + lane;
    if (f < f1 && (x[i] < 0 || x[i] >= E)) { bad = true; x[i] = -1; }
  }
  if (bad && status != nullptr) set_status(status, GSG_ERR_BAD_ROUTING);
}

// Peer masks of the warp's ids and the warp's histogram (hist = this warp's E counters).
template <int kPer>
__device__ __forceinline__ void warp_histogram(const int x[kPer], unsigned m[kPer], int f0, int f1, int* hist,
                                               int nbits) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    if (f0 + 32 * i >= f1) break;   // warp-uniform
    m[i] = peer_mask(x[i], nbits);
    if (x[i] >= 0 && lane == __ffs(m[i]) - 1) hist[x[i]] += __popc(m[i]);
    __syncwarp();
  }
}

// Stable scatter of the warp's ids; base[x] = first row of id x for this warp (advanced).
template <int kPer>
__device__ __forceinline__ void warp_scatter(const int x[kPer], const unsigned m[kPer], int f0, int f1, int* base,
                                             int32_t* perm_src, int32_t* inv_perm) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    if (f0 + 32 * i >= f1) break;   // warp-uniform
    const int f = f0 + 32 * i + lane;
    if (x[i] >= 0) {
      const int pos = base[x[i]] + __popc(m[i] & lt);
      perm_src[pos] = f;
      inv_perm[f] = pos;
    } else if (f < f1) {
      inv_perm[f] = -1;   // a pair with an out-of-range id has no row: later kernels skip it
    }
    __syncwarp();
    if (x[i] >= 0 && lane == __ffs(m[i]) - 1) base[x[i]] += __popc(m[i]);
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

// This warp's run of the chunk [c0, c1): 32*kPer indices starting at c0 + warp*32*kPer.
template <int kPer>
__device__ __forceinline__ void warp_run(int c0, int c1, int& f0, int& f1) {
  const int warp = threadIdx.x >> 5;
  f0 = min(c0 + warp * 32 * kPer, c1);
  f1 = min(f0 + 32 * kPer, c1);
}

// One block holds everything (R <= 1024 * kPer, kPer indices per thread): histogram, scan,
// scatter in one launch.  hist: 32 x E ints of shared memory.
template <int kPer>
__device__ __forceinline__ void route_single_body(const int32_t* __restrict__ ids, int R, int E, int32_t* off,
                                                  int32_t* perm_src, int32_t* inv_perm, int* status, int* hist) {
  __shared__ int warp_sums[32];
  __shared__ int total;
  for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) hist[i] = 0;
  const int warp = threadIdx.x >> 5;
  int f0, f1;
  warp_run<kPer>(0, R, f0, f1);
  pdl_wait();
  int x[kPer];
  unsigned m[kPer];
  warp_load_ids<kPer>(ids, f0, f1, E, x, status);
  __syncthreads();
  warp_histogram<kPer>(x, m, f0, f1, hist + warp * E, key_bits(E));
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
  warp_scatter<kPer>(x, m, f0, f1, hist + warp * E, perm_src, inv_perm);
}

template <int kPer>
__global__ void __launch_bounds__(kRouteThreads)
route_single_kernel(const int32_t* __restrict__ ids, int R, int E, int32_t* off, int32_t* perm_src,
                    int32_t* inv_perm, int* status) {
  extern __shared__ int hist[];  // [32][E]
  pdl_launch_dependents();
  route_single_body<kPer>(ids, R, E, off, perm_src, inv_perm, status, hist);
}

// Multi-chunk path, launch 1: the histogram of chunk `chunk` -> ws_hist[chunk][E].
template <int kPer>
__device__ __forceinline__ void route_hist_body(const int32_t* __restrict__ ids, int R, int E, int chunk,
                                                int* ws_hist, int* status, int* hist) {
  for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) hist[i] = 0;
  pdl_wait();
  const int c0 = chunk * 1024 * kPer, c1 = min(c0 + 1024 * kPer, R);
  int f0, f1;
  warp_run<kPer>(c0, c1, f0, f1);
  int x[kPer];
  unsigned m[kPer];
  warp_load_ids<kPer>(ids, f0, f1, E, x, status);
  __syncthreads();
  warp_histogram<kPer>(x, m, f0, f1, hist + (threadIdx.x >> 5) * E, key_bits(E));
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int s = 0;
    for (int w = 0; w < 32; ++w) s += hist[w * E + e];
    ws_hist[(size_t)chunk * E + e] = s;
  }
}

template <int kPer>
__global__ void __launch_bounds__(kRouteThreads)
route_hist_kernel(const int32_t* __restrict__ ids, int R, int E, int* ws_hist, int* status) {
  extern __shared__ int hist[];
  pdl_launch_dependents();
  route_hist_body<kPer>(ids, R, E, blockIdx.x, ws_hist, status, hist);
}

// The routing launch above (one-block routing when kSingle, else the chunk histograms) in
// blocks [0, nroute), and the activation quantizer's partial max|X| in blocks [nroute, grid):
// both only read their inputs, so the amax pass needs no launch of its own.
template <int kPer, bool kSingle>
__global__ void __launch_bounds__(kRouteThreads)
route_amax_kernel(const int32_t* __restrict__ ids, int R, int E, int nroute, int32_t* off, int32_t* perm_src,
                  int32_t* inv_perm, int* ws_hist, const uint16_t* __restrict__ X, long long n8, float* partial,
                  int* status) {
  extern __shared__ int hist[];
  __shared__ float red[kRouteThreads / 32];
  pdl_launch_dependents();
  if ((int)blockIdx.x >= nroute) {
    pdl_wait();
    block_amax_partial(X, n8, (int)blockIdx.x - nroute, (int)gridDim.x - nroute, partial, red, status);
    return;
  }
  if constexpr (kSingle)
    route_single_body<kPer>(ids, R, E, off, perm_src, inv_perm, status, hist);
  else
    route_hist_body<kPer>(ids, R, E, blockIdx.x, ws_hist, status, hist);
}

// Launch 2 (one block): offsets and each chunk's first row per expert -> ws_base[chunk][E].
__global__ void __launch_bounds__(kRouteThreads)
route_scan_kernel(const int* ws_hist, int nchunks, int E, int32_t* off, int* ws_base) {
  __shared__ int warp_sums[32];
  __shared__ int total;
  pdl_launch_dependents();
  pdl_wait();
  const int e = threadIdx.x;
  int tot = 0;
  if (e < E)
    for (int b = 0; b < nchunks; ++b) tot += ws_hist[(size_t)b * E + e];
  const int start = block_exclusive_scan(tot, warp_sums, &total);
  if (e < E) {
    off[e] = start;
    int run = start;
    for (int b = 0; b < nchunks; ++b) {
      int c = ws_hist[(size_t)b * E + e];
      ws_base[(size_t)b * E + e] = run;
      run += c;
    }
  }
  if (e == 0) off[E] = total;
}

// Launch 3: per chunk, warp bases from the chunk base, then the stable scatter.  With kSelfScan
// (1024-index chunks, where chunks x experts is small) there is no launch 2: every block sums the
// chunk histograms itself (ws = ws_hist), block 0 writes the offsets.  Otherwise ws = ws_base.
template <int kPer, bool kSelfScan>
__global__ void __launch_bounds__(kRouteThreads)
route_scatter_kernel(const int32_t* __restrict__ ids, int R, int E, const int* ws, int nchunks, int32_t* off,
                     int32_t* perm_src, int32_t* inv_perm) {
  extern __shared__ int hist[];
  __shared__ int warp_sums[32];
  __shared__ int total;
  pdl_launch_dependents();
  pdl_wait();
  int chunk_base = 0;
  if (kSelfScan) {
    // expert e's first row in this chunk: rows of experts < e, then of earlier chunks
    const int e = threadIdx.x;
    int tot = 0, before = 0;
    if (e < E)
      for (int b = 0; b < nchunks; ++b) {
        const int c = ws[(size_t)b * E + e];
        tot += c;
        if (b < (int)blockIdx.x) before += c;
      }
    const int start = block_exclusive_scan(tot, warp_sums, &total);
    chunk_base = start + before;
    if (blockIdx.x == 0) {
      if (e < E) off[e] = start;
      if (e == 0) off[E] = total;
    }
  }
  for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) hist[i] = 0;
  const int c0 = blockIdx.x * 1024 * kPer, c1 = min(c0 + 1024 * kPer, R);
  int f0, f1;
  warp_run<kPer>(c0, c1, f0, f1);
  const int warp = threadIdx.x >> 5;
  int x[kPer];
  unsigned m[kPer];
  warp_load_ids<kPer>(ids, f0, f1, E, x, nullptr);
  __syncthreads();
  warp_histogram<kPer>(x, m, f0, f1, hist + warp * E, key_bits(E));
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = kSelfScan ? chunk_base : ws[(size_t)blockIdx.x * E + e];
    for (int w = 0; w < 32; ++w) {
      int c = hist[w * E + e];
      hist[w * E + e] = run;
      run += c;
    }
  }
  __syncthreads();
  warp_scatter<kPer>(x, m, f0, f1, hist + warp * E, perm_src, inv_perm);
}

int route_chunks(int R, int E) {
  if (R <= kSingleMaxR) return 1;
  const int c = route_chunk_size(R, E);
  return (R + c - 1) / c;
}

size_t route_workspace_bytes(int R, int E) {
  const int nc = route_chunks(R, E);
  return nc <= 1 ? 0 : (size_t)2 * nc * E * sizeof(int);
}

bool route_supported(int E) { return E >= 1 && E <= kRouteMaxE; }

cudaError_t route_set_smem_attrs() {
  const int bytes = 32 * kRouteMaxE * (int)sizeof(int);
  const cudaError_t errs[10] = {
      cudaFuncSetAttribute(route_single_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes),
      cudaFuncSetAttribute(route_single_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes),
      cudaFuncSetAttribute(route_amax_kernel<1, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes),
      cudaFuncSetAttribute(route_amax_kernel<2, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes),
      cudaFuncSetAttribute(route_amax_kernel<1, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes),
      cudaFuncSetAttribute(route_amax_kernel<8, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes),
      cudaFuncSetAttribute(route_hist_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes),
      cudaFuncSetAttribute(route_hist_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes),
      cudaFuncSetAttribute(route_scatter_kernel<1, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes),
      cudaFuncSetAttribute(route_scatter_kernel<8, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)};
  for (cudaError_t e : errs)
    if (e != cudaSuccess) return e;
  return cudaSuccess;
}

int dispatch_amax_blocks(long long n_elems) {
  const long long n8 = n_elems / 8;
  long long b = (n8 + 4LL * kRouteThreads - 1) / (4LL * kRouteThreads);   // 4 units per thread
  if (b < 1) b = 1;
  if (b > kDispatchMaxAmaxBlocks) b = kDispatchMaxAmaxBlocks;
  return int(b);
}

// The routing launches; with X != nullptr and n_elems > 0 the first one also computes the amax
// partials of X in P extra blocks (*amax_parts = P).
static cudaError_t route_launches(const int32_t* ids, int R, int E, int32_t* off, int32_t* perm_src,
                                  int32_t* inv_perm, void* ws, const uint16_t* X, long long n_elems,
                                  float* amax_partial, int* amax_parts, int* status, cudaStream_t stream) {
  const size_t smem = (size_t)32 * E * sizeof(int);
  const int nc = route_chunks(R, E);
  const int P = (X != nullptr && n_elems > 0) ? dispatch_amax_blocks(n_elems) : 0;
  if (amax_parts != nullptr) *amax_parts = P;
  const long long n8 = n_elems / 8;
  if (nc <= 1) {
    if (P == 0) {
      auto single = R <= 1024 ? route_single_kernel<1> : route_single_kernel<2>;
      return launch_pdl(single, 1, kRouteThreads, smem, stream, ids, R, E, off, perm_src, inv_perm, status);
    }
    auto single = R <= 1024 ? route_amax_kernel<1, true> : route_amax_kernel<2, true>;
    return launch_pdl(single, 1 + P, kRouteThreads, smem, stream, ids, R, E, 1, off, perm_src, inv_perm,
                      (int*)nullptr, X, n8, amax_partial, status);
  }
  int* ws_hist = static_cast<int*>(ws);
  int* ws_base = ws_hist + (size_t)nc * E;
  cudaError_t e;
  if (route_chunk_size(R, E) == 1024) {
    e = P == 0 ? launch_pdl(route_hist_kernel<1>, nc, kRouteThreads, smem, stream, ids, R, E, ws_hist, status)
               : launch_pdl(route_amax_kernel<1, false>, nc + P, kRouteThreads, smem, stream, ids, R, E, nc, off,
                            perm_src, inv_perm, ws_hist, X, n8, amax_partial, status);
    if (e == cudaSuccess)
      e = launch_pdl(route_scatter_kernel<1, true>, nc, kRouteThreads, smem, stream, ids, R, E,
                     (const int*)ws_hist, nc, off, perm_src, inv_perm);
  } else {
    e = P == 0 ? launch_pdl(route_hist_kernel<8>, nc, kRouteThreads, smem, stream, ids, R, E, ws_hist, status)
               : launch_pdl(route_amax_kernel<8, false>, nc + P, kRouteThreads, smem, stream, ids, R, E, nc, off,
                            perm_src, inv_perm, ws_hist, X, n8, amax_partial, status);
    if (e == cudaSuccess)
      e = launch_pdl(route_scan_kernel, 1, kRouteThreads, 0, stream, (const int*)ws_hist, nc, E, off, ws_base);
    if (e == cudaSuccess)
      e = launch_pdl(route_scatter_kernel<8, false>, nc, kRouteThreads, smem, stream, ids, R, E,
                     (const int*)ws_base, nc, off, perm_src, inv_perm);
  }
  return e;
}

cudaError_t launch_route(const int32_t* ids, int R, int E, int32_t* off, int32_t* perm_src,
                         int32_t* inv_perm, void* ws, int* status, cudaStream_t stream) {
  return route_launches(ids, R, E, off, perm_src, inv_perm, ws, nullptr, 0, nullptr, nullptr, status, stream);
}

cudaError_t launch_route_amax(const int32_t* ids, int R, int E, int32_t* off, int32_t* perm_src, int32_t* inv_perm,
                              void* ws, const uint16_t* X, long long n_elems, float* amax_partial, int* amax_parts,
                              int* status, cudaStream_t stream) {
  return route_launches(ids, R, E, off, perm_src, inv_perm, ws, X, n_elems, amax_partial, amax_parts, status,
                        stream);
}

}  // namespace gsg
