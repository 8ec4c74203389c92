// gsg_unpermute.cu -- gate-weighted scatter of expert outputs back to tokens.
//
// "Hardware-Native Joint Sparse-Quantization for Trillion-Scale Mixture-of-Experts"
// (paperlayer.ai summary), §D.1 (p.19): scatter after the expert GEMM.
//   out[t][n] = bf16_rne( sum_{j<k} fp32(g[t][j] * Y[inv_perm[t*k + j]][n]) ),
// products and the running sum in fp32 (starting at 0), j ascending.  One thread owns eight
// consecutive outputs: 128-bit gathers of Y rows (a token's rows all in flight at once),
// 128-bit stores of out.
#include "gsg_internal.cuh"

namespace gsg {

constexpr int kUnpermThreads = 256;

__global__ void __launch_bounds__(kUnpermThreads)
unpermute_kernel(const uint16_t* __restrict__ Y, const int32_t* __restrict__ inv_perm,
                 const float* __restrict__ gates, int T, int k, int N, int R, uint16_t* __restrict__ out,
                 int* status) {
  pdl_launch_dependents();
  pdl_wait();
  const unsigned n8 = (unsigned)N / 8u;
  const unsigned total = (unsigned)T * n8;   // T * N / 8 < 2^31 is checked on the host
  for (unsigned i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    const int t = int(i / n8), c = int(i % n8);
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.0f;
    // up to eight routed rows at a time: every index, gate and row load is issued before the
    // first use, then the products are summed in j order
    for (int j0 = 0; j0 < k; j0 += 8) {
      int row[8];
      float g[8];
      uint4 v[8];
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const bool in = j0 + jj < k;
        row[jj] = in ? __ldg(inv_perm + (size_t)t * k + j0 + jj) : -1;
        g[jj] = in ? __ldg(gates + (size_t)t * k + j0 + jj) : 0.0f;
      }
#pragma unroll
      for (int jj = 0; jj < 8; ++jj)
        v[jj] = (row[jj] >= 0 && row[jj] < R) ? __ldg(reinterpret_cast<const uint4*>(Y + (size_t)row[jj] * N) + c)
                                              : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        if (j0 + jj >= k) break;
        if (row[jj] < 0 || row[jj] >= R) { set_status(status, GSG_ERR_BAD_ROUTING); continue; }
        const uint32_t w[4] = {v[jj].x, v[jj].y, v[jj].z, v[jj].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[2 * q] = __fadd_rn(acc[2 * q], __fmul_rn(g[jj], __uint_as_float(w[q] << 16)));
          acc[2 * q + 1] = __fadd_rn(acc[2 * q + 1], __fmul_rn(g[jj], __uint_as_float(w[q] & 0xFFFF0000u)));
        }
      }
    }
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * q]));
      const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * q + 1]));
      o[q] = lo | (hi << 16);
    }
    reinterpret_cast<uint4*>(out + (size_t)t * N)[c] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

cudaError_t launch_unpermute(const uint16_t* Y, const int32_t* inv_perm, const float* gates, int T,
                             int k, int N, uint16_t* out, int* status, int num_sms, cudaStream_t stream) {
  const long long total = (long long)T * (N / 8);
  if (total == 0) return cudaSuccess;
  long long blocks = (total + kUnpermThreads - 1) / kUnpermThreads;
  if (blocks > (long long)num_sms * 16) blocks = (long long)num_sms * 16;
  return launch_pdl(unpermute_kernel, (unsigned)blocks, kUnpermThreads, 0, stream, Y, inv_perm, gates, T, k, N,
                    T * k, out, status);
}

}  // namespace gsg
