// gsg_pack.cu -- weight packers: paired 4:8 NVFP4 (sparse) and NVFP4 (dense control).
//
// "Hardware-Native Joint Sparse-Quantization for Trillion-Scale Mixture-of-Experts"
// (paperlayer.ai summary): App. A "Blackwell paired 4:8 NVFP4" (p.14, Fig. 3 p.15) -- each
// aligned 8-group keeps two of its four adjacent pairs, retained values on the E2M1 grid,
// 16 retained values per 32-weight block share one UE4M3 scale; "Storage layout" (p.15) --
// four retained values + a pattern index per 8-group; §3.4 (p.5) -- E2M1 values, sparse
// metadata and UE4M3 scales are packed together.  The support is chosen by pair energy
// (fp32, ties to the lower pair); the per-expert fp32 tensor scale is amax / 2688.
//
// Two launches per call: (1) per-expert partial amax of the kept weights, (2) one thread per
// 32-block (sparse) or 16-block (dense) writes codes, metadata and the scale directly into the
// interleaved tile-major chunk blocks the grouped GEMM streams (see include/gsg.h).
#include "gsg_internal.cuh"

namespace gsg {

constexpr int kPackThreads = 256;

__device__ __forceinline__ void select_pairs(const float w[8], int& i0, int& i1) {
  float m[4];
#pragma unroll
  for (int p = 0; p < 4; ++p)
    m[p] = __fadd_rn(__fmul_rn(w[2 * p], w[2 * p]), __fmul_rn(w[2 * p + 1], w[2 * p + 1]));
  // running maxima carried by value (an index into m would put m in local memory)
  int a = 0;
  float ma = m[0];
#pragma unroll
  for (int p = 1; p < 4; ++p)
    if (m[p] > ma) { ma = m[p]; a = p; }
  int b = (a == 0) ? 1 : 0;
  float mb = (a == 0) ? m[1] : m[0];
#pragma unroll
  for (int p = 0; p < 4; ++p)
    if (p != a && m[p] > mb) { mb = m[p]; b = p; }
  i0 = a < b ? a : b;
  i1 = a < b ? b : a;
}

// Element 2*i + half of w (i = pair index 0..3) by selects, not an indexed load: a runtime index
// into w would put the array in local memory.
__device__ __forceinline__ float pair_elem(const float w[8], int i, int half) {
  const float lo = i == 0 ? w[0] : i == 1 ? w[2] : i == 2 ? w[4] : w[6];
  const float hi = i == 0 ? w[1] : i == 1 ? w[3] : i == 2 ? w[5] : w[7];
  return half ? hi : lo;
}

__device__ __forceinline__ bool all_finite8(const float w[8]) {
  bool ok = true;
#pragma unroll
  for (int i = 0; i < 8; ++i) ok &= isfinite(w[i]);
  return ok;
}

__device__ __forceinline__ void load8(const float* p, float w[8]) {
  float4 a = __ldg(reinterpret_cast<const float4*>(p));
  float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
  w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
}

// Block-wide max of non-negative floats (blockDim.x == kPackThreads).
__device__ float block_max(float v, float* red) {
  v = warp_max(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < (kPackThreads / 32) ? red[lane] : 0.0f;
    v = warp_max(v);
    if (lane == 0) red[0] = v;
  }
  __syncthreads();
  float r = red[0];
  __syncthreads();
  return r;
}

// (1) partial amax per (expert, block).  sparse: over kept weights only.
template <bool kSparse>
__global__ void __launch_bounds__(kPackThreads)
pack_amax_kernel(const float* __restrict__ W, long long groups_per_expert, float* __restrict__ partial,
                 int* status) {
  __shared__ float red[32];
  const int e = blockIdx.y;
  const float* We = W + (size_t)e * (size_t)groups_per_expert * 8;
  float mx = 0.0f;
  bool finite = true;
  for (long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x; g < groups_per_expert;
       g += (long long)gridDim.x * blockDim.x) {
    float w[8];
    load8(We + g * 8, w);
    finite &= all_finite8(w);
    if (kSparse) {
      int i0, i1;
      select_pairs(w, i0, i1);
      mx = fmaxf(mx, fmaxf(fmaxf(fabsf(pair_elem(w, i0, 0)), fabsf(pair_elem(w, i0, 1))),
                           fmaxf(fabsf(pair_elem(w, i1, 0)), fabsf(pair_elem(w, i1, 1)))));
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(w[i]));
    }
  }
  if (!finite) set_status(status, GSG_ERR_NONFINITE);
  float bm = block_max(mx, red);
  if (threadIdx.x == 0) partial[(size_t)e * gridDim.x + blockIdx.x] = bm;
}

__device__ float expert_scale_from_partials(const float* partial, int e, int nparts, float* red) {
  float v = 0.0f;
  for (int i = threadIdx.x; i < nparts; i += blockDim.x) v = fmaxf(v, partial[(size_t)e * nparts + i]);
  return tensor_scale_from_amax(block_max(v, red));
}

// (2a) sparse encode: one thread per 32-block (4 groups, 16 retained values).
__global__ void __launch_bounds__(kPackThreads)
pack_sparse_encode_kernel(const float* __restrict__ W, int N, int K, const float* __restrict__ partial,
                          int nparts, uint8_t* __restrict__ packed, float* __restrict__ w_tensor_scale) {
  __shared__ float red[32];
  const int e = blockIdx.y;
  const float s = expert_scale_from_partials(partial, e, nparts, red);
  if (blockIdx.x == 0 && threadIdx.x == 0) w_tensor_scale[e] = s;
  const float six_s = __fmul_rn(6.0f, s);
  const int blocks_per_row = K / 32;
  const long long nblk = (long long)N * blocks_per_row;
  const int NT = N / kTileN, KC = K / kChunkK;
  for (long long bi = (long long)blockIdx.x * blockDim.x + threadIdx.x; bi < nblk;
       bi += (long long)gridDim.x * blockDim.x) {
    const int n = int(bi / blocks_per_row), b = int(bi % blocks_per_row);
    const float* src = W + ((size_t)e * N + n) * K + (size_t)b * 32;
    float kept[16];
    uint32_t pat[4];
    float bmax = 0.0f;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      float w[8];
      load8(src + 8 * g, w);
      int i0, i1;
      select_pairs(w, i0, i1);
      kept[4 * g + 0] = pair_elem(w, i0, 0);
      kept[4 * g + 1] = pair_elem(w, i0, 1);
      kept[4 * g + 2] = pair_elem(w, i1, 0);
      kept[4 * g + 3] = pair_elem(w, i1, 1);
      pat[g] = uint32_t(i0) | (uint32_t(i1) << 2);
#pragma unroll
      for (int i = 0; i < 4; ++i) bmax = fmaxf(bmax, fabsf(kept[4 * g + i]));
    }
    const BlockScale bs = block_scale(bmax, six_s, s);
    uint64_t codes = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i)
      codes |= uint64_t(e2m1_encode(__fmul_rn(kept[i], bs.inv))) << (4 * i);
    const int nt = n / kTileN, r = n % kTileN;
    // chunk block of (e, nt, chunk b/8); k-block h = (b/4)%2 of the chunk, 32-block q = b%4
    const int kc = b >> 3, h = (b >> 2) & 1, q = b & 3, g8 = b & 7;
    uint8_t* cb = packed + (((size_t)e * NT + nt) * KC + kc) * kSparseChunkBytes;
    // values: stored values 16*q .. +15 of the k-block -> bytes 8*q .. +7 of the row
    *reinterpret_cast<uint64_t*>(cb + h * 4096 + (r >> 3) * 256 + (q >> 1) * 128 + (r & 7) * 16 + (q & 1) * 8) = codes;
    // metadata: groups 4*(b%8) .. +3 of the chunk -> bytes 2*(b%8), +1 of the row
    const uint32_t m16 = pat[0] | (pat[1] << 4) | (pat[2] << 8) | (pat[3] << 12);
    *reinterpret_cast<uint16_t*>(cb + 8192 + r * 16 + 2 * g8) = uint16_t(m16);
    // scale atom of k-block h
    cb[10240 + h * 512 + 16 * (r & 31) + 4 * (r >> 5) + q] = uint8_t(bs.sc);
  }
}

// (2b) dense encode: one thread per 16-block.
__global__ void __launch_bounds__(kPackThreads)
pack_dense_encode_kernel(const float* __restrict__ W, int N, int K, const float* __restrict__ partial,
                         int nparts, uint8_t* __restrict__ packed, float* __restrict__ w_tensor_scale) {
  __shared__ float red[32];
  const int e = blockIdx.y;
  const float s = expert_scale_from_partials(partial, e, nparts, red);
  if (blockIdx.x == 0 && threadIdx.x == 0) w_tensor_scale[e] = s;
  const float six_s = __fmul_rn(6.0f, s);
  const int blocks_per_row = K / 16;
  const long long nblk = (long long)N * blocks_per_row;
  const int NT = N / kTileN, KC = K / kChunkK;
  for (long long bi = (long long)blockIdx.x * blockDim.x + threadIdx.x; bi < nblk;
       bi += (long long)gridDim.x * blockDim.x) {
    const int n = int(bi / blocks_per_row), b = int(bi % blocks_per_row);
    const float* src = W + ((size_t)e * N + n) * K + (size_t)b * 16;
    float w[16];
    load8(src, w);
    load8(src + 8, w + 8);
    float bmax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) bmax = fmaxf(bmax, fabsf(w[i]));
    const BlockScale bs = block_scale(bmax, six_s, s);
    uint64_t c = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) c |= uint64_t(e2m1_encode(__fmul_rn(w[i], bs.inv))) << (4 * i);
    const int nt = n / kTileN, r = n % kTileN;
    // chunk block of (e, nt, chunk b/16); k-block h = (b/4)%4 of the chunk (64 K each), q = b%4
    const int kc = b >> 4, h = (b >> 2) & 3, q = b & 3;
    uint8_t* cb = packed + (((size_t)e * NT + nt) * KC + kc) * kDenseChunkBytes;
    *reinterpret_cast<uint64_t*>(cb + h * 4096 + (r >> 3) * 256 + (q >> 1) * 128 + (r & 7) * 16 + (q & 1) * 8) = c;
    cb[16384 + h * 512 + 16 * (r & 31) + 4 * (r >> 5) + q] = uint8_t(bs.sc);
  }
}

// Number of partial-amax blocks per expert (host and workspace sizing agree on it).
int pack_partials_per_expert(int N, int K) {
  long long groups = (long long)N * K / 8;
  long long want = (groups + kPackThreads * 16 - 1) / (kPackThreads * 16);
  if (want < 1) want = 1;
  if (want > 256) want = 256;
  return int(want);
}

cudaError_t launch_pack(bool sparse, const float* W, int E, int N, int K, uint8_t* packed, float* w_tensor_scale,
                        float* partial, int* status, cudaStream_t stream) {
  const int P = pack_partials_per_expert(N, K);
  const long long groups = (long long)N * K / 8;
  dim3 g1(P, E);
  if (sparse)
    pack_amax_kernel<true><<<g1, kPackThreads, 0, stream>>>(W, groups, partial, status);
  else
    pack_amax_kernel<false><<<g1, kPackThreads, 0, stream>>>(W, groups, partial, status);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const long long nblk = (long long)N * K / (sparse ? 32 : 16);
  long long nb = (nblk + kPackThreads - 1) / kPackThreads;
  if (nb > 1024) nb = 1024;
  dim3 g2((unsigned)nb, E);
  if (sparse)
    pack_sparse_encode_kernel<<<g2, kPackThreads, 0, stream>>>(W, N, K, partial, P, packed, w_tensor_scale);
  else
    pack_dense_encode_kernel<<<g2, kPackThreads, 0, stream>>>(W, N, K, partial, P, packed, w_tensor_scale);
  return cudaGetLastError();
}

}  // namespace gsg
