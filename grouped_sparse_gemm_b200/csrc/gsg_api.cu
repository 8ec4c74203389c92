// gsg_api.cu -- the exported C ABI (include/gsg.h): argument checks, per-device state,
// device status word, launches.  Every entry point returns before launching anything when
// an argument is invalid.
#include <cstdint>
#include <cstring>
#include <mutex>

#include "gsg_internal.cuh"
#include "gsg_launch.h"

namespace {

__device__ int g_device_status;  // sticky first device-side error of this device

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool ready = false;
  int* status = nullptr;
  int num_sms = 0;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

// Per-device set-up on first use (needs that device current): status word address, SM count,
// shared-memory limits of the kernels that need more than 48 KB.
gsg_status_t device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GSG_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& d = g_dev[dev];
  if (!d.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return GSG_ERR_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return GSG_ERR_CUDA;
    if (gsg::route_set_smem_attrs() != cudaSuccess) return GSG_ERR_CUDA;
    if (gsg::gemm_set_smem_attrs() != cudaSuccess) return GSG_ERR_CUDA;
    d.status = static_cast<int*>(p);
    d.num_sms = sms;
    d.ready = true;
  }
  *out = &d;
  return GSG_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }
inline gsg_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? GSG_OK : GSG_ERR_CUDA; }

size_t combine_slot_bytes(int T, int k, int N) { return ((size_t)T * k * N * 2 + 255) / 256 * 256; }

bool weight_shape_ok(int E, int N, int K) {
  return E >= 1 && N >= 128 && K >= 256 && N % 128 == 0 && K % 256 == 0;
}

}  // namespace

namespace gsg {
// The library's per-device set-up and status word, for entry points defined in other files.
gsg_status_t device_setup(int** status, int* num_sms) {
  DeviceState* d = nullptr;
  gsg_status_t st = device_state(&d);
  if (st != GSG_OK) return st;
  *status = d->status;
  *num_sms = d->num_sms;
  return GSG_OK;
}
}  // namespace gsg

extern "C" {

size_t gsg_sparse_packed_bytes(int E, int N, int K) {
  return (size_t)E * (N / gsg::kTileN) * (K / gsg::kChunkK) * gsg::kSparseChunkBytes;
}
size_t gsg_dense_packed_bytes(int E, int N, int K) {
  return (size_t)E * (N / gsg::kTileN) * (K / gsg::kChunkK) * gsg::kDenseChunkBytes;
}
size_t gsg_act_codes_bytes(int R, int K) { return (size_t)R * K / 2; }
size_t gsg_act_scales_bytes(int R, int K, int sf_block) {
  if (sf_block <= 0) return 0;
  return (size_t)(K / (4 * sf_block)) * (size_t)(R + gsg::kActScalePadRows) * 16;
}

size_t gsg_workspace_size(int op, int E, int N, int K, int T, int k) {
  switch (op) {
    case GSG_OP_PACK_SPARSE:
    case GSG_OP_PACK_DENSE:
      if (E < 1 || N < 1 || K < 8) return 0;
      return (size_t)E * gsg::pack_partials_per_expert(N, K) * sizeof(float);
    case GSG_OP_ROUTE:
      if (E < 1 || T < 0 || k < 1) return 0;
      return gsg::route_workspace_bytes(T * k, E);
    case GSG_OP_QUANTIZE: {  // amax partials, then (large R*K) the raw scale words
      if (T < 0 || K < 1 || k < 1) return 0;
      const size_t raw = gsg::quant_raw_bytes((long long)T * k, K);
      return raw > 0 ? gsg::quant_raw_offset((long long)T * K) + raw
                     : (size_t)gsg::quant_partials((long long)T * K) * sizeof(float);
    }
    case GSG_OP_DISPATCH:  // routing workspace, amax partials (each 256-byte rounded), raw scale words
      if (E < 1 || T < 0 || k < 1 || K < 1) return 0;
      return (gsg::route_workspace_bytes(T * k, E) + 255) / 256 * 256 +
             ((size_t)gsg::dispatch_amax_blocks((long long)T * K) * sizeof(float) + 255) / 256 * 256 +
             gsg::quant_raw_bytes((long long)T * k, K);
    case GSG_OP_COMBINE:   // slots bf16 [T*k][N], then counters int32 [T][N/32]
      if (T < 0 || k < 1 || N < 32) return 0;
      return combine_slot_bytes(T, k, N) + (size_t)T * (N / 32) * sizeof(int);
    default:
      return 0;
  }
}

static gsg_status_t pack_common(bool sparse, const float* W, int E, int N, int K, uint8_t* packed,
                                float* w_tensor_scale, void* ws, size_t ws_bytes, void* stream) {
  if (!W || !packed || !w_tensor_scale) return GSG_ERR_INVALID_ARG;
  if (!weight_shape_ok(E, N, K)) return GSG_ERR_UNSUPPORTED_SHAPE;
  if (E > 65535) return GSG_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(W) || !aligned16(packed)) return GSG_ERR_INVALID_ARG;
  const size_t need = gsg_workspace_size(sparse ? GSG_OP_PACK_SPARSE : GSG_OP_PACK_DENSE, E, N, K, 0, 1);
  if (ws == nullptr || ws_bytes < need) return GSG_ERR_WORKSPACE;
  DeviceState* d = nullptr;
  gsg_status_t st = device_state(&d);
  if (st != GSG_OK) return st;
  return from_cuda(gsg::launch_pack(sparse, W, E, N, K, packed, w_tensor_scale, static_cast<float*>(ws), d->status,
                                    as_stream(stream)));
}

gsg_status_t gsg_pack_sparse_nvfp4(const float* W, int E, int N, int K, uint8_t* w_packed, float* w_tensor_scale,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  return pack_common(true, W, E, N, K, w_packed, w_tensor_scale, workspace, workspace_bytes, stream);
}

gsg_status_t gsg_pack_dense_nvfp4(const float* W, int E, int N, int K, uint8_t* w_packed, float* w_tensor_scale,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  return pack_common(false, W, E, N, K, w_packed, w_tensor_scale, workspace, workspace_bytes, stream);
}

gsg_status_t gsg_moe_route_permute(const int32_t* topk_ids, int T, int k, int E, int32_t* expert_offsets,
                                   int32_t* perm_src, int32_t* inv_perm, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  if (T < 0 || k < 1) return GSG_ERR_INVALID_ARG;
  if (!gsg::route_supported(E)) return GSG_ERR_UNSUPPORTED_SHAPE;
  if ((long long)T * k > (1ll << 30)) return GSG_ERR_UNSUPPORTED_SHAPE;
  if (!expert_offsets) return GSG_ERR_INVALID_ARG;
  if (T > 0 && (!topk_ids || !perm_src || !inv_perm)) return GSG_ERR_INVALID_ARG;
  const size_t need = gsg::route_workspace_bytes(T * k, E);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return GSG_ERR_WORKSPACE;
  DeviceState* d = nullptr;
  gsg_status_t st = device_state(&d);
  if (st != GSG_OK) return st;
  return from_cuda(gsg::launch_route(topk_ids, T * k, E, expert_offsets, perm_src, inv_perm, workspace, d->status,
                                     as_stream(stream)));
}

gsg_status_t gsg_quantize_act_nvfp4(const uint16_t* X, int T, int K, int sf_block, const int32_t* inv_perm, int k,
                                    const float* x_tensor_scale_in, uint8_t* codes, uint8_t* scales,
                                    float* x_tensor_scale_out, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  if (T < 0 || k < 1 || (sf_block != 16 && sf_block != 32)) return GSG_ERR_INVALID_ARG;
  if (K < 256 || K % 256 != 0) return GSG_ERR_UNSUPPORTED_SHAPE;
  if ((long long)T * k > (1ll << 30)) return GSG_ERR_UNSUPPORTED_SHAPE;
  if ((long long)T * (K / 8) >= (1ll << 31)) return GSG_ERR_UNSUPPORTED_SHAPE;  // 32-bit unit index
  if (inv_perm == nullptr && k != 1) return GSG_ERR_INVALID_ARG;
  if (!scales || !x_tensor_scale_out) return GSG_ERR_INVALID_ARG;
  if (T > 0 && (!X || !codes)) return GSG_ERR_INVALID_ARG;
  if ((X && !aligned16(X)) || (codes && !aligned16(codes)) || !aligned16(scales)) return GSG_ERR_INVALID_ARG;
  const size_t raw_bytes = sf_block == 32 ? gsg::quant_raw_bytes((long long)T * k, K) : 0;
  if (x_tensor_scale_in == nullptr || raw_bytes > 0) {
    const size_t need = gsg_workspace_size(GSG_OP_QUANTIZE, 0, 0, K, T, k);
    if (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)) return GSG_ERR_WORKSPACE;
  }
  DeviceState* d = nullptr;
  gsg_status_t st = device_state(&d);
  if (st != GSG_OK) return st;
  uint32_t* raw = raw_bytes > 0 ? reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) +
                                                              gsg::quant_raw_offset((long long)T * K))
                                : nullptr;
  return from_cuda(gsg::launch_quant(X, T, K, sf_block, inv_perm, k, x_tensor_scale_in, codes, scales,
                                     x_tensor_scale_out, static_cast<float*>(workspace), 0, raw, d->status,
                                     d->num_sms, as_stream(stream)));
}

gsg_status_t gsg_moe_dispatch_nvfp4(const int32_t* topk_ids, const uint16_t* X, int T, int k, int E, int K,
                                    int sf_block, const float* x_tensor_scale_in, int32_t* expert_offsets,
                                    int32_t* perm_src, int32_t* inv_perm, uint8_t* codes, uint8_t* scales,
                                    float* x_tensor_scale_out, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  // the checks of gsg_moe_route_permute and gsg_quantize_act_nvfp4
  if (T < 0 || k < 1 || (sf_block != 16 && sf_block != 32)) return GSG_ERR_INVALID_ARG;
  if (!gsg::route_supported(E)) return GSG_ERR_UNSUPPORTED_SHAPE;
  if (K < 256 || K % 256 != 0) return GSG_ERR_UNSUPPORTED_SHAPE;
  if ((long long)T * k > (1ll << 30)) return GSG_ERR_UNSUPPORTED_SHAPE;
  if ((long long)T * (K / 8) >= (1ll << 31)) return GSG_ERR_UNSUPPORTED_SHAPE;
  if (!expert_offsets || !scales || !x_tensor_scale_out) return GSG_ERR_INVALID_ARG;
  if (T > 0 && (!topk_ids || !perm_src || !inv_perm || !X || !codes)) return GSG_ERR_INVALID_ARG;
  if ((X && !aligned16(X)) || (codes && !aligned16(codes)) || !aligned16(scales)) return GSG_ERR_INVALID_ARG;
  const size_t need = gsg_workspace_size(GSG_OP_DISPATCH, E, 0, K, T, k);
  if (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)) return GSG_ERR_WORKSPACE;
  DeviceState* d = nullptr;
  gsg_status_t st = device_state(&d);
  if (st != GSG_OK) return st;
  const size_t route_bytes = (gsg::route_workspace_bytes(T * k, E) + 255) / 256 * 256;
  const size_t part_bytes = ((size_t)gsg::dispatch_amax_blocks((long long)T * K) * sizeof(float) + 255) / 256 * 256;
  float* partial = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + route_bytes);
  uint32_t* raw = (sf_block == 32 && gsg::quant_raw_bytes((long long)T * k, K) > 0)
                      ? reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + route_bytes + part_bytes)
                      : nullptr;
  const bool amax = x_tensor_scale_in == nullptr;
  int parts = 0;
  cudaError_t e = gsg::launch_route_amax(topk_ids, T * k, E, expert_offsets, perm_src, inv_perm, workspace,
                                         amax ? X : nullptr, amax ? (long long)T * K : 0, partial, &parts,
                                         d->status, as_stream(stream));
  if (e == cudaSuccess)
    e = gsg::launch_quant(X, T, K, sf_block, inv_perm, k, x_tensor_scale_in, codes, scales, x_tensor_scale_out,
                          partial, parts, raw, d->status, d->num_sms, as_stream(stream));
  return from_cuda(e);
}

static gsg_status_t gemm_common(bool sparse, const uint8_t* a_codes, const uint8_t* a_scales, const float* x_scale,
                                const uint8_t* w_packed, const float* w_scale, const int32_t* off, int E, int N,
                                int K, int R, int max_rows, void* Y, int y_dtype, void* stream,
                                bool native = false) {
  if (R < 0 || (y_dtype != GSG_OUT_BF16 && y_dtype != GSG_OUT_F32)) return GSG_ERR_INVALID_ARG;
  if (!weight_shape_ok(E, N, K) || !gsg::gemm_supported(E)) return GSG_ERR_UNSUPPORTED_SHAPE;
  if ((long long)R > (1ll << 30)) return GSG_ERR_UNSUPPORTED_SHAPE;
  if (!off || !w_packed || !w_scale || !x_scale) return GSG_ERR_INVALID_ARG;
  if (R == 0) return GSG_OK;  // nothing routed: nothing to compute or write
  if (!a_codes || !a_scales || !Y) return GSG_ERR_INVALID_ARG;
  if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(w_packed) || !aligned16(Y)) return GSG_ERR_INVALID_ARG;
  DeviceState* d = nullptr;
  gsg_status_t st = device_state(&d);
  if (st != GSG_OK) return st;
  const int rc = gsg::launch_gemm(sparse, a_codes, a_scales, x_scale, w_packed, w_scale, off, E, N, K, R, max_rows,
                                  Y, y_dtype == GSG_OUT_F32 ? 1 : 0, d->status, d->num_sms, as_stream(stream),
                                  nullptr, nullptr, nullptr, native);
  return rc == 0 ? GSG_OK : GSG_ERR_CUDA;
}

gsg_status_t gsg_grouped_sparse_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const float* x_tensor_scale,
                                     const uint8_t* w_packed, const float* w_tensor_scale,
                                     const int32_t* expert_offsets, int E, int N, int K, int R,
                                     int max_rows_per_expert, void* Y, int y_dtype, void* stream) {
  return gemm_common(true, a_codes, a_scales, x_tensor_scale, w_packed, w_tensor_scale, expert_offsets, E, N, K, R,
                     max_rows_per_expert, Y, y_dtype, stream);
}

gsg_status_t gsg_grouped_dense_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const float* x_tensor_scale,
                                    const uint8_t* w_packed, const float* w_tensor_scale,
                                    const int32_t* expert_offsets, int E, int N, int K, int R,
                                    int max_rows_per_expert, void* Y, int y_dtype, void* stream) {
  return gemm_common(false, a_codes, a_scales, x_tensor_scale, w_packed, w_tensor_scale, expert_offsets, E, N, K, R,
                     max_rows_per_expert, Y, y_dtype, stream);
}

gsg_status_t gsg_grouped_dense_gemm_native(const uint8_t* a_codes, const uint8_t* a_scales,
                                           const float* x_tensor_scale, const uint8_t* w_packed,
                                           const float* w_tensor_scale, const int32_t* expert_offsets, int E, int N,
                                           int K, int R, int max_rows_per_expert, void* Y, int y_dtype,
                                           void* stream) {
  return gemm_common(false, a_codes, a_scales, x_tensor_scale, w_packed, w_tensor_scale, expert_offsets, E, N, K, R,
                     max_rows_per_expert, Y, y_dtype, stream, true);
}

gsg_status_t gsg_grouped_sparse_gemm_swiglu(const uint8_t* a_codes, const uint8_t* a_scales,
                                            const float* x_tensor_scale, const uint8_t* w_packed,
                                            const float* w_tensor_scale, const int32_t* expert_offsets, int E,
                                            int N2, int K, int R, int max_rows_per_expert,
                                            const float* h_tensor_scale, uint8_t* h_codes, uint8_t* h_scales,
                                            void* stream) {
  if (R < 0) return GSG_ERR_INVALID_ARG;
  if (!weight_shape_ok(E, N2, K) || N2 % 256 != 0 || !gsg::gemm_supported(E)) return GSG_ERR_UNSUPPORTED_SHAPE;
  if ((long long)R > (1ll << 30)) return GSG_ERR_UNSUPPORTED_SHAPE;
  if (!expert_offsets || !w_packed || !w_tensor_scale || !x_tensor_scale || !h_tensor_scale || !h_scales)
    return GSG_ERR_INVALID_ARG;
  if (!aligned16(h_scales) || !aligned16(w_packed)) return GSG_ERR_INVALID_ARG;
  DeviceState* d = nullptr;
  gsg_status_t st = device_state(&d);
  if (st != GSG_OK) return st;
  if (R == 0) {   // nothing routed: only the (all padding) scale entries to clear
    const size_t n = gsg_act_scales_bytes(0, N2 / 2, 32);
    return from_cuda(cudaMemsetAsync(h_scales, 0, n, as_stream(stream)));
  }
  if (!a_codes || !a_scales || !h_codes) return GSG_ERR_INVALID_ARG;
  if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(h_codes)) return GSG_ERR_INVALID_ARG;
  const int rc = gsg::launch_gemm(true, a_codes, a_scales, x_tensor_scale, w_packed, w_tensor_scale, expert_offsets,
                                  E, N2, K, R, max_rows_per_expert, h_codes, 0, d->status, d->num_sms,
                                  as_stream(stream), h_scales, h_tensor_scale);
  return rc == 0 ? GSG_OK : GSG_ERR_CUDA;
}

gsg_status_t gsg_grouped_sparse_gemm_combine(const uint8_t* a_codes, const uint8_t* a_scales,
                                             const float* x_tensor_scale, const uint8_t* w_packed,
                                             const float* w_tensor_scale, const int32_t* expert_offsets, int E,
                                             int N, int K, int T, int k, int max_rows_per_expert,
                                             const int32_t* perm_src, const float* gates, void* workspace,
                                             size_t workspace_bytes, uint16_t* out, void* stream) {
  if (T < 0 || k < 1) return GSG_ERR_INVALID_ARG;
  if (!weight_shape_ok(E, N, K) || !gsg::gemm_supported(E)) return GSG_ERR_UNSUPPORTED_SHAPE;
  if ((long long)T * k > (1ll << 30)) return GSG_ERR_UNSUPPORTED_SHAPE;
  if ((long long)T * (N / 8) >= (1ll << 31)) return GSG_ERR_UNSUPPORTED_SHAPE;   // token sums: 32-bit unit index
  if (T == 0) return GSG_OK;
  const int R = T * k;
  if (!a_codes || !a_scales || !x_tensor_scale || !w_packed || !w_tensor_scale || !expert_offsets || !perm_src ||
      !gates || !out)
    return GSG_ERR_INVALID_ARG;
  if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(w_packed) || !aligned16(out))
    return GSG_ERR_INVALID_ARG;
  if (workspace == nullptr || !aligned16(workspace) ||
      workspace_bytes < gsg_workspace_size(GSG_OP_COMBINE, E, N, K, T, k))
    return GSG_ERR_WORKSPACE;
  DeviceState* d = nullptr;
  gsg_status_t st = device_state(&d);
  if (st != GSG_OK) return st;
  gsg::CombineArgs ca;
  ca.perm_src = perm_src;
  ca.gates = gates;
  ca.counters = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + combine_slot_bytes(T, k, N));
  ca.out = out;
  ca.k = k;
  const int rc = gsg::launch_gemm(true, a_codes, a_scales, x_tensor_scale, w_packed, w_tensor_scale, expert_offsets,
                                  E, N, K, R, max_rows_per_expert, workspace, 0, d->status, d->num_sms,
                                  as_stream(stream), nullptr, nullptr, &ca);
  return rc == 0 ? GSG_OK : GSG_ERR_CUDA;
}

gsg_status_t gsg_unpermute_scale(const uint16_t* Y, const int32_t* inv_perm, const float* gates, int T, int k, int N,
                                 uint16_t* out, void* stream) {
  if (T < 0 || k < 1 || N < 8 || N % 8 != 0) return GSG_ERR_INVALID_ARG;
  if ((long long)T * k > (1ll << 30)) return GSG_ERR_UNSUPPORTED_SHAPE;
  if ((long long)T * (N / 8) >= (1ll << 31)) return GSG_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return GSG_OK;
  if (!Y || !inv_perm || !gates || !out) return GSG_ERR_INVALID_ARG;
  if (!aligned16(Y) || !aligned16(out)) return GSG_ERR_INVALID_ARG;
  DeviceState* d = nullptr;
  gsg_status_t st = device_state(&d);
  if (st != GSG_OK) return st;
  return from_cuda(gsg::launch_unpermute(Y, inv_perm, gates, T, k, N, out, d->status, d->num_sms, as_stream(stream)));
}

gsg_status_t gsg_get_device_status(void* stream) {
  DeviceState* d = nullptr;
  gsg_status_t st = device_state(&d);
  if (st != GSG_OK) return st;
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return GSG_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, d->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return GSG_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpy(d->status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return GSG_ERR_CUDA;
  }
  return static_cast<gsg_status_t>(v);
}

const char* gsg_status_string(gsg_status_t s) {
  switch (s) {
    case GSG_OK: return "ok";
    case GSG_ERR_INVALID_ARG: return "invalid argument";
    case GSG_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case GSG_ERR_CUDA: return "CUDA error";
    case GSG_ERR_BAD_ROUTING: return "expert id or expert offsets out of range";
    case GSG_ERR_NONFINITE: return "non-finite value in a quantized tensor";
    case GSG_ERR_DEVICE_TIMEOUT: return "a bounded wait inside a kernel timed out";
    case GSG_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

int gsg_version(void) { return 1; }

void gsg_test_set_gemm_stall_ns(unsigned long long ns) { gsg::gemm_set_test_stall(ns); }
void gsg_test_set_gemm_table_cap(int tiles) { gsg::gemm_set_test_table_cap(tiles); }

}  // extern "C"
