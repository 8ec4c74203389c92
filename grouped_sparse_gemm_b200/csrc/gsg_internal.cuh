// gsg_internal.cuh -- shared device helpers of libgsg (sm_100a only).
//
// Number formats (App. A of "Hardware-Native Joint Sparse-Quantization for Trillion-Scale
// Mixture-of-Experts", p.14): E2M1 values and UE4M3 block scales.  Encoders round to nearest,
// ties to even, and saturate; every fp32 step uses the _rn intrinsics so that no
// multiply-add is contracted and the results are reproducible bit for bit.
#pragma once

#include <cstdint>
#include <utility>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "gsg.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libgsg is written for sm_100a (Blackwell B200) only"
#endif

namespace gsg {

constexpr int kTileN = 128;            // weight rows per tile (MMA M)
constexpr int kChunkK = 256;           // logical K per pipeline stage / metadata chunk
constexpr int kActScalePadRows = 256;  // extra zero rows of the quad activation-scale layout
constexpr int kSparseChunkBytes = 11264;  // packed weight chunk block: values 8192 | meta 2048 | scales 1024
constexpr int kDenseChunkBytes = 18432;   // dense control chunk block: codes 16384 | scales 2048
constexpr float kTensorScaleDen = 2688.0f;  // 6 * 448

// ------------------------------------------------------------------ status word
__device__ __forceinline__ void set_status(int* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

// ------------------------------------------------------------------ codecs
// UE4M3 (E4M3 without sign): bias 7, subnormal q * 2^-9, max 448 = code 0x7E.
__device__ __forceinline__ float ue4m3_decode(uint32_t code) {
  uint32_t e = (code >> 3) & 0xF, m = code & 7;
  if (e == 0) return __uint2float_rn(m) * (1.0f / 512.0f);
  // (8 + m) * 2^(e - 10): exact in fp32.
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// x >= 0 and finite.  Round to nearest, ties to even code, saturate at 448.
__device__ __forceinline__ uint32_t ue4m3_encode(float x) {
  if (!(x > 0.0f)) return 0u;
  if (x >= 448.0f) return 0x7Eu;
  uint32_t u = __float_as_uint(x);
  int e = int(u >> 23) - 127;
  if (e < -6) {                                  // UE4M3 subnormal range: q * 2^-9, q in 0..8
    return __float2uint_rn(__fmul_rn(x, 512.0f));  // exact scaling, round half to even
  }
  uint32_t m = u & 0x7FFFFFu;
  uint32_t q = m >> 20;
  uint32_t rem = m & 0xFFFFFu;
  if (rem > 0x80000u || (rem == 0x80000u && (q & 1u))) q += 1u;
  uint32_t eb = uint32_t(e + 7);
  if (q == 8u) { q = 0u; eb += 1u; }
  uint32_t code = (eb << 3) | q;
  return code > 0x7Eu ? 0x7Eu : code;
}

// E2M1: magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}; sign bit 3 copied from the input (-0 -> 0x8).
__device__ __forceinline__ uint32_t e2m1_encode(float v) {
  const float a = fabsf(v);
  // code = number of decision thresholds below |v| (strict at the ties that round down to the
  // even code, inclusive at those that round up); NaN saturates like the largest magnitude
  uint32_t c = (uint32_t)(a > 0.25f) + (uint32_t)(a >= 0.75f) + (uint32_t)(a > 1.25f) + (uint32_t)(a >= 1.75f) +
               (uint32_t)(a > 2.5f) + (uint32_t)(a >= 3.5f) + (uint32_t)(a > 5.0f);
  if (a != a) c = 7u;
  return c | ((__float_as_uint(v) >> 28) & 8u);
}

// The same two encoders on the hardware converters (PTX cvt.rn.satfinite to e2m1x2 / e4m3x2):
// round to nearest, ties to even, saturating at the largest finite value, sign kept.  For a
// non-negative finite x the E4M3 code equals the UE4M3 code (sign bit 0).  Eight values -> eight
// E2M1 codes, v[i] in bits 4i..4i+3.
__device__ __forceinline__ uint32_t e2m1_encode8_cvt(const float v[8]) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return r;
}
__device__ __forceinline__ uint32_t ue4m3_encode_cvt(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return r & 0xFFu;
}

// Block rule shared by weights and activations (s = tensor scale, b = block amax):
//   sc = UE4M3(b / (6 s)),  d = dec(sc) * s,  inv = d == 0 ? 0 : 1/d,  code = E2M1(v * inv)
struct BlockScale {
  uint32_t sc;
  float inv;
};
__device__ __forceinline__ BlockScale block_scale(float blk_amax, float six_s, float s) {
  BlockScale r;
  r.sc = ue4m3_encode(__fdiv_rn(blk_amax, six_s));
  float d = __fmul_rn(ue4m3_decode(r.sc), s);
  r.inv = (d == 0.0f) ? 0.0f : __frcp_rn(d);
  return r;
}
__device__ __forceinline__ BlockScale block_scale_cvt(float blk_amax, float six_s, float s) {
  BlockScale r;
  r.sc = ue4m3_encode_cvt(__fdiv_rn(blk_amax, six_s));
  float d = __fmul_rn(ue4m3_decode(r.sc), s);
  r.inv = (d == 0.0f) ? 0.0f : __frcp_rn(d);
  return r;
}

__device__ __forceinline__ float tensor_scale_from_amax(float amax) {
  return amax == 0.0f ? 1.0f : __fdiv_rn(amax, kTensorScaleDen);
}

// ------------------------------------------------------------------ programmatic dependent launch
// The step's kernels are launched with programmatic stream serialization: a kernel may be
// scheduled while the previous kernel in the stream is still running, does only set-up that
// touches no global memory (shared memory, barriers, TMEM, tensor-map prefetch), then waits in
// pdl_wait() until the previous grid has completed and its writes are visible.  Every global
// read and write comes after pdl_wait(), so stream order is kept exactly; each kernel lets its
// own successor launch early with pdl_launch_dependents().  Without a programmatic predecessor
// (first kernel, other work before it) the wait returns at once.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// The same for a kernel launched as thread-block clusters of `cluster_x` CTAs along x (gridDim.x
// a multiple of it).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                      cudaStream_t stream, unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster_x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ------------------------------------------------------------------ small utilities
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__host__ __device__ inline int ceil_div_i(int a, int b) { return (a + b - 1) / b; }

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

// Partial max|X| of bf16 X (n8 128-bit units) for block `blk` of `nblk` (grid-stride over the
// units, four 128-bit loads in flight per thread and round), written to partial[blk]; a
// non-finite element sets GSG_ERR_NONFINITE.  Block-wide: every thread calls it; red holds
// blockDim.x / 32 floats of shared memory.
__device__ __forceinline__ void block_amax_partial(const uint16_t* __restrict__ X, long long n8, int blk, int nblk,
                                                   float* partial, float* red, int* status) {
  float mx = 0.0f;
  bool finite = true;
  const uint4* X4 = reinterpret_cast<const uint4*>(X);
  const long long stride = (long long)nblk * blockDim.x;
  for (long long i0 = (long long)blk * blockDim.x + threadIdx.x; i0 < n8; i0 += 4 * stride) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const long long i = i0 + u * stride;
      v[u] = i < n8 ? __ldg(X4 + i) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t lo = w[j] & 0xFFFFu, hi = w[j] >> 16;
        finite &= ((lo & 0x7F80u) != 0x7F80u) && ((hi & 0x7F80u) != 0x7F80u);
        mx = fmaxf(mx, fmaxf(fabsf(bf16_bits_to_f32(lo)), fabsf(bf16_bits_to_f32(hi))));
      }
    }
  }
  if (!finite) set_status(status, GSG_ERR_NONFINITE);
  mx = warp_max(mx);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (int)(blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
    v = warp_max(v);
    if (threadIdx.x == 0) partial[blk] = v;
  }
}

}  // namespace gsg
