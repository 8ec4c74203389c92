// gsg_launch.h -- host-side launchers of the individual kernels (internal to libgsg).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "gsg.h"

namespace gsg {

// gsg_api.cu: per-device set-up (first call on a device), device status word and SM count
gsg_status_t device_setup(int** status, int* num_sms);

// gsg_pack.cu
int pack_partials_per_expert(int N, int K);
cudaError_t launch_pack(bool sparse, const float* W, int E, int N, int K, uint8_t* packed, float* w_tensor_scale,
                        float* partial, int* status, cudaStream_t stream);

// gsg_quant.cu
int quant_partials(long long n_elems);
// Raw scale-word buffer of the two-phase scale path (0 when R*K is below its threshold) and its
// offset in the quantizer's workspace (after the amax partials).
size_t quant_raw_bytes(long long R, int K);
size_t quant_raw_offset(long long n_elems);
// partials_ready > 0: partial[0, partials_ready) already hold the partial maxima of X (the
// dispatch launch computed them), so no amax launch is made.
// raw: workspace of quant_raw_bytes(T*k, K) bytes for the two-phase scale path (nullptr: direct).
cudaError_t launch_quant(const uint16_t* X, int T, int K, int sf, const int32_t* inv_perm, int k, const float* s_in,
                         uint8_t* codes, uint8_t* scales, float* s_out, float* partial, int partials_ready,
                         uint32_t* raw, int* status, int num_sms, cudaStream_t stream);

// gsg_route.cu
int route_chunks(int R, int E);
size_t route_workspace_bytes(int R, int E);
bool route_supported(int E);
cudaError_t route_set_smem_attrs();
cudaError_t launch_route(const int32_t* ids, int R, int E, int32_t* off, int32_t* perm_src, int32_t* inv_perm,
                         void* ws, int* status, cudaStream_t stream);
// Routing with the activation quantizer's amax pass folded into its first launch: X bf16 of
// n_elems elements (nullptr / 0: no amax blocks); *amax_parts = number of partial maxima written
// to amax_partial (0 when none).
int dispatch_amax_blocks(long long n_elems);
cudaError_t launch_route_amax(const int32_t* ids, int R, int E, int32_t* off, int32_t* perm_src, int32_t* inv_perm,
                              void* ws, const uint16_t* X, long long n_elems, float* amax_partial, int* amax_parts,
                              int* status, cudaStream_t stream);

// gsg_unpermute.cu
cudaError_t launch_unpermute(const uint16_t* Y, const int32_t* inv_perm, const float* gates, int T, int k, int N,
                             uint16_t* out, int* status, int num_sms, cudaStream_t stream);

// gsg_gemm.cu
struct CombineArgs {          // the combine epilogue of the down-projection
  const int32_t* perm_src;    // routed row -> flat index t*k + j
  const float* gates;         // [T][k]
  int* counters;              // [T][N/32], zero on entry, left zero
  uint16_t* out;              // [T][N] bf16
  int k;
};
bool gemm_supported(int E);
// test hook: GEMM launches after this call stall their MMA warp for `ns` on a barrier nothing
// arrives on (0 = off); see GemmParams::stall_ns
void gemm_set_test_stall(unsigned long long ns);
// test hook: GEMM launches after this call keep at most `cap` tile-table entries per CTA (-1 = off)
void gemm_set_test_table_cap(int cap);
int gemm_pick_bn(int max_rows, int R, int E);
cudaError_t gemm_set_smem_attrs();
int launch_gemm(bool sparse, const uint8_t* a_codes, const uint8_t* a_scales, const float* x_scale,
                const uint8_t* w_packed, const float* w_scale, const int32_t* off, int E, int N, int K, int R,
                int max_rows, void* Y, int y_f32, int* status, int num_sms, cudaStream_t stream,
                uint8_t* h_scales = nullptr, const float* h_scale = nullptr, const CombineArgs* comb = nullptr,
                bool native = false);

}  // namespace gsg
