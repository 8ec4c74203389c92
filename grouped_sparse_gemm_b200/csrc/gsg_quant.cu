// gsg_quant.cu -- NVFP4 activation quantizer fused with MoE dispatch.
//
// "Hardware-Native Joint Sparse-Quantization for Trillion-Scale Mixture-of-Experts"
// (paperlayer.ai summary), §D.1 (p.19): activation quantization forms 32-element scale blocks
// and is fused with dispatch for the first expert GEMM; §3.4 (pp.5-6): weights and quantized
// activations are packed in corresponding scale blocks.
//
// Launch 1 (skipped when the caller supplies s_x, or made by the routing's first launch in
// gsg_moe_dispatch_nvfp4): partial max|X| per block, 128-bit loads, warp-shuffle reductions.
// Launch 2, 32-element blocks (the sparse path): one lane per block (act_quant32_kernel, below;
// from R*K = 2^27 followed by act_scales_quad_kernel).  Launch 2, 16-element blocks (the dense
// control): every block
// folds the partials into s_x = amax/2688,
// then each warp quantizes 256 consecutive elements of one token row at a time (8 per lane, one
// 128-bit load), groups of 4 lanes (2 for 16-element blocks) combine their maxima into the
// block amax, the four scales of one MMA k-block are gathered into a 32-bit word, and the
// token's codes and scale words are written to each of its k routed rows (the dispatch), the
// rows read once per warp (lane j holds row j) and the scale words spread over the lanes.  The same launch zero-fills
// the padding entries of the quad scale layout.
#include "gsg_internal.cuh"
#include "gsg_launch.h"

namespace gsg {

constexpr int kQuantThreads = 256;
constexpr int kQuantMainThreads = 128;   // the quantize launch: more, smaller blocks balance the SMs
// From R*K = 2^27 (R routed rows) the 32-element quantizer writes its scale words row-major to a
// workspace and a second launch builds the quad layout: writing the quad entries directly is
// four scattered 4-byte stores per routed row and k-block, each its own 32-byte sector, and at
// these sizes the partial sectors leave L2 before they fill (DRAM read-modify-write).
constexpr long long kQuantRawMinRK = 1ll << 27;

__global__ void __launch_bounds__(kQuantThreads)
act_amax_kernel(const uint16_t* __restrict__ X, long long n8, float* __restrict__ partial, int* status) {
  __shared__ float red[kQuantThreads / 32];
  pdl_launch_dependents();
  pdl_wait();
  block_amax_partial(X, n8, blockIdx.x, gridDim.x, partial, red, status);
}

struct QuantParams {
  const uint16_t* X;
  const int32_t* inv_perm;
  const float* s_in;
  const float* partial;
  int nparts;
  int T, K, sf, k, R, rcap;
  uint8_t* codes;
  uint8_t* scales;
  float* s_out;
  int* status;
  uint32_t* raw;   // non-null: scale words go to raw[row][K/128] (then act_scales_quad_kernel)
};

// The tensor scale: the caller's value, or max|X| folded from the partial maxima (block-wide;
// every thread of the block must call it).
__device__ __forceinline__ float quant_tensor_scale(const QuantParams& p, float* red, float* s_sh) {
  if (p.s_in != nullptr) {
    if (threadIdx.x == 0) *s_sh = __ldg(p.s_in);
  } else {
    float v = 0.0f;
    for (int i = threadIdx.x; i < p.nparts; i += blockDim.x) v = fmaxf(v, p.partial[i]);
    v = warp_max(v);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    if (threadIdx.x < 32) {
      float w = threadIdx.x < (int)(blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
      w = warp_max(w);
      if (threadIdx.x == 0) *s_sh = tensor_scale_from_amax(w);
    }
  }
  __syncthreads();
  const float s = *s_sh;
  if (blockIdx.x == 0 && threadIdx.x == 0) *p.s_out = s;
  return s;
}

// Zero the quad scale entries that refer to rows >= R (no routed row writes them).
__device__ __forceinline__ void quant_zero_padding(const QuantParams& p) {
  uint32_t* sw = reinterpret_cast<uint32_t*>(p.scales);
  const int KBa = p.K / (4 * p.sf);
  const int r_lo = p.R > 96 ? p.R - 96 : 0;
  const int span = p.rcap - r_lo;                 // at most 352 rows
  const int npad = KBa * span * 4;                // K / 64 * 352 * 4 < 2^31
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < npad; i += gridDim.x * blockDim.x) {
    const int c = i & 3;
    const int rest = i >> 2;
    const int rr = r_lo + rest % span;
    const int kb = rest / span;
    if (rr + 32 * c >= p.R) sw[((size_t)kb * p.rcap + rr) * 4 + c] = 0u;
  }
}

// 32-element blocks: one lane quantizes one whole block (four 128-bit loads, the block max, one
// scale, 16 bytes of codes), so the per-block work is not repeated across lanes.  Four
// consecutive lanes hold the four blocks of one MMA k-block (K % 128 == 0) and assemble its scale
// word; lane c of the four writes quad entry c of each routed row.  Lanes load their token's
// routed rows themselves (lanes of one token read the same addresses).
constexpr int kQ32Rows = 8;   // routed rows loaded ahead with the block (the rest on demand)

struct Quant32Unit {
  uint4 x[4];
  int rows[kQ32Rows];
  int t, b;
  bool valid;
};

__device__ __forceinline__ void quant32_fetch(const QuantParams& p, long long u, long long U, int bpr, Quant32Unit& q) {
  q.valid = u < U;
  const unsigned u32 = (unsigned)(q.valid ? u : 0);   // U = T*K/32 < 2^31 (checked on the host)
  q.t = int(u32 / (unsigned)bpr);
  q.b = int(u32 % (unsigned)bpr);
  const uint4* src = reinterpret_cast<const uint4*>(p.X + (size_t)q.t * p.K + (size_t)q.b * 32);
#pragma unroll
  for (int i = 0; i < 4; ++i) q.x[i] = q.valid ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
  for (int j = 0; j < kQ32Rows; ++j)
    q.rows[j] = (q.valid && j < p.k) ? (p.inv_perm != nullptr ? __ldg(p.inv_perm + (size_t)q.t * p.k + j) : q.t) : -1;
}

__global__ void __launch_bounds__(128)
act_quant32_kernel(QuantParams p) {
  __shared__ float red[4];
  __shared__ float s_sh;
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int bpr = p.K / 32;                                    // blocks per row
  const long long U = (long long)p.T * bpr;
  const int gwarp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  const long long wstep = (long long)nwarps * 32;
  long long base = (long long)gwarp * 32;
  Quant32Unit cur;
  quant32_fetch(p, base + lane, U, bpr, cur);                  // before the tensor scale is known
  const float s = quant_tensor_scale(p, red, &s_sh);
  const float six_s = __fmul_rn(6.0f, s);
  uint32_t* sw = reinterpret_cast<uint32_t*>(p.scales);
  for (; base < U; base += wstep) {
    const Quant32Unit q = cur;
    if (base + wstep < U) quant32_fetch(p, base + wstep + lane, U, bpr, cur);
    float x[32];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t w[4] = {q.x[i].x, q.x[i].y, q.x[i].z, q.x[i].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        x[8 * i + 2 * j] = bf16_bits_to_f32(w[j] & 0xFFFFu);
        x[8 * i + 2 * j + 1] = bf16_bits_to_f32(w[j] >> 16);
      }
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(x[i]));
    const BlockScale bs = block_scale_cvt(amax, six_s, s);
    uint32_t cw[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float xs[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) xs[j] = __fmul_rn(x[8 * i + j], bs.inv);
      cw[i] = e2m1_encode8_cvt(xs);
    }
    const int g = lane & ~3;
    const uint32_t word = __shfl_sync(0xffffffffu, bs.sc, g) | (__shfl_sync(0xffffffffu, bs.sc, g + 1) << 8) |
                          (__shfl_sync(0xffffffffu, bs.sc, g + 2) << 16) | (__shfl_sync(0xffffffffu, bs.sc, g + 3) << 24);
    if (!q.valid) continue;
    const int kb = q.b >> 2, cq = lane & 3;
    auto dispatch = [&](int row) {
      if (row < 0 || row >= p.R) { set_status(p.status, GSG_ERR_BAD_ROUTING); return; }
      *reinterpret_cast<uint4*>(p.codes + (size_t)row * (p.K / 2) + (size_t)q.b * 16) =
          make_uint4(cw[0], cw[1], cw[2], cw[3]);
      if (p.raw != nullptr) {   // one word per row and k-block (K % 1024 == 0: a warp's 32 contiguous bytes)
        if (cq == 0) p.raw[(size_t)row * (p.K / 128) + kb] = word;
        return;
      }
      const int rr = row - 32 * cq;
      if (rr >= 0) sw[((size_t)kb * p.rcap + rr) * 4 + cq] = word;
    };
#pragma unroll
    for (int j = 0; j < kQ32Rows; ++j)
      if (j < p.k) dispatch(q.rows[j]);
    for (int j = kQ32Rows; j < p.k; ++j) dispatch(__ldg(p.inv_perm + (size_t)q.t * p.k + j));
  }
  if (p.raw == nullptr) quant_zero_padding(p);
}

// Second launch of the two-phase path: raw scale words [R][KBa] -> the quad layout,
//   quad[kb][rr][c] = raw[rr + 32c][kb]  (0 where rr + 32c >= R),  rr in [0, rcap).
// A block builds 128 quad rows x 16 k-blocks from 224 raw rows staged in shared memory (row
// pitch 17 words: conflict-free column reads); reads are 64-byte row segments, writes 16-byte
// entries, 2 KB contiguous per k-block.  The padding entries are written too.
constexpr int kQuadTileRows = 128;
constexpr int kQuadTileKb = 16;

__global__ void __launch_bounds__(256)
act_scales_quad_kernel(const uint32_t* __restrict__ raw, int R, int KBa, int rcap, uint32_t* __restrict__ quad) {
  __shared__ uint32_t tile[kQuadTileRows + 96][kQuadTileKb + 1];
  pdl_launch_dependents();
  pdl_wait();
  const int r0 = blockIdx.x * kQuadTileRows, kb0 = blockIdx.y * kQuadTileKb;
  for (int i = threadIdx.x; i < (kQuadTileRows + 96) * kQuadTileKb; i += blockDim.x) {
    const int rr = i / kQuadTileKb, kk = i % kQuadTileKb;
    const int row = r0 + rr, kb = kb0 + kk;
    tile[rr][kk] = (row < R && kb < KBa) ? __ldg(raw + (size_t)row * KBa + kb) : 0u;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kQuadTileRows * kQuadTileKb; i += blockDim.x) {
    const int kk = i / kQuadTileRows, rr = i % kQuadTileRows;
    const int row = r0 + rr, kb = kb0 + kk;
    if (row >= rcap || kb >= KBa) continue;
    *reinterpret_cast<uint4*>(quad + ((size_t)kb * rcap + row) * 4) =
        make_uint4(tile[rr][kk], tile[rr + 32][kk], tile[rr + 64][kk], tile[rr + 96][kk]);
  }
}

// One warp-iteration covers 256 consecutive elements of one token row (K % 256 == 0): lane L
// holds elements 8L..8L+7 of them, and lane j < k also holds the token's j-th routed row.
struct QuantSlice {
  uint4 x;
  int myrow;
};

__device__ __forceinline__ void quant_fetch(const QuantParams& p, long long base, int units_per_row, int lane,
                                            QuantSlice& q) {
  const unsigned b32 = (unsigned)base;   // U = T*K/8 < 2^31 is checked on the host
  const int t = int(b32 / (unsigned)units_per_row);
  const int c8 = int(b32 % (unsigned)units_per_row) + lane;
  q.x = __ldg(reinterpret_cast<const uint4*>(p.X + (size_t)t * p.K + (size_t)c8 * 8));
  q.myrow = lane < p.k ? (p.inv_perm != nullptr ? __ldg(p.inv_perm + (size_t)t * p.k + lane) : t) : -1;
}

__global__ void __launch_bounds__(kQuantMainThreads)
act_quant_kernel(QuantParams p) {
  __shared__ float red[kQuantMainThreads / 32];
  __shared__ float s_sh;
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int units_per_row = p.K / 8;
  const long long U = (long long)p.T * units_per_row;   // a multiple of 32
  const int gwarp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  const long long wstep = (long long)nwarps * 32;
  // the first slice's loads go out before the tensor scale is known (they do not depend on it)
  long long base = (long long)gwarp * 32;
  QuantSlice cur;
  if (base < U) quant_fetch(p, base, units_per_row, lane, cur);

  // ---- tensor scale
  const float s = quant_tensor_scale(p, red, &s_sh);
  const float six_s = __fmul_rn(6.0f, s);

  // a 32-element block is 4 lanes (16-element block: 2 lanes); one MMA k-block's four scales
  // sit in 16 lanes (8), so a slice holds nkb = 2 (4) k-blocks
  const int step = p.sf == 32 ? 4 : 2;
  const int nkb = 8 / step;
  const int lg_ent = p.sf == 32 ? 3 : 4;   // log2(4 * nkb): scale entries per routed row and slice
  uint32_t* sw = reinterpret_cast<uint32_t*>(p.scales);
  for (; base < U; base += wstep) {
    const QuantSlice q = cur;
    if (base + wstep < U) quant_fetch(p, base + wstep, units_per_row, lane, cur);
    const unsigned b32 = (unsigned)base;
    const int t = int(b32 / (unsigned)units_per_row);
    const int c80 = int(b32 % (unsigned)units_per_row);   // first unit of the slice in its row
    float x[8];
    const uint32_t w[4] = {q.x.x, q.x.y, q.x.z, q.x.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      x[2 * j] = bf16_bits_to_f32(w[j] & 0xFFFFu);
      x[2 * j + 1] = bf16_bits_to_f32(w[j] >> 16);
    }
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(x[j]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    if (p.sf == 32) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const BlockScale bs = block_scale_cvt(amax, six_s, s);
    float xs[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) xs[j] = __fmul_rn(x[j], bs.inv);
    const uint32_t codes = e2m1_encode8_cvt(xs);
    // four scales of one MMA k-block -> one 32-bit word, held by the k-block's first lane
    const int g = lane & ~(4 * step - 1);
    const uint32_t word = __shfl_sync(0xffffffffu, bs.sc, g) | (__shfl_sync(0xffffffffu, bs.sc, g + step) << 8) |
                          (__shfl_sync(0xffffffffu, bs.sc, g + 2 * step) << 16) |
                          (__shfl_sync(0xffffffffu, bs.sc, g + 3 * step) << 24);
    // dispatch: codes of the slice to each of the token's k routed rows (row j from lane j)
    int myrow = q.myrow;
    for (int j0 = 0; j0 < p.k; j0 += 32) {
      if (j0 > 0)
        myrow = j0 + lane < p.k ? (p.inv_perm != nullptr ? __ldg(p.inv_perm + (size_t)t * p.k + j0 + lane) : t) : -1;
      const int jn = min(32, p.k - j0);
      for (int j = 0; j < jn; ++j) {
        const int row = __shfl_sync(0xffffffffu, myrow, j);
        if (row < 0 || row >= p.R) {   // warp-uniform
          if (lane == 0) set_status(p.status, GSG_ERR_BAD_ROUTING);
          continue;
        }
        *reinterpret_cast<uint32_t*>(p.codes + (size_t)row * (p.K / 2) + (size_t)(c80 + lane) * 4) = codes;
      }
      // scale words: entry (j, c, kbw) of this row group, spread over the lanes
      const int ng = jn * 4 * nkb;
      for (int e0 = 0; e0 < ng; e0 += 32) {
        const int e = e0 + lane;
        const int jj = e >> lg_ent, rem = e & (4 * nkb - 1);
        const int c = rem & 3, kbw = rem >> 2;
        const int row = __shfl_sync(0xffffffffu, myrow, jj & 31);
        const uint32_t wd = __shfl_sync(0xffffffffu, word, (kbw * 4 * step) & 31);
        const int rr = row - 32 * c;
        if (e < ng && row >= 0 && row < p.R && rr >= 0) {
          const int kb = c80 / (4 * step) + kbw;
          sw[((size_t)kb * p.rcap + rr) * 4 + c] = wd;
        }
      }
    }
  }
  quant_zero_padding(p);
}

size_t quant_raw_offset(long long n_elems) {
  return ((size_t)quant_partials(n_elems) * sizeof(float) + 255) / 256 * 256;
}

size_t quant_raw_bytes(long long R, int K) {
  return R * (long long)K >= kQuantRawMinRK ? (size_t)(R * (long long)(K / 128) * 4) : 0;
}

int quant_partials(long long n_elems) {
  long long n8 = n_elems / 8;
  long long b = (n8 + kQuantThreads * 4 - 1) / (kQuantThreads * 4);
  if (b < 1) b = 1;
  if (b > 512) b = 512;
  return int(b);
}

cudaError_t launch_quant(const uint16_t* X, int T, int K, int sf, const int32_t* inv_perm, int k,
                         const float* s_in, uint8_t* codes, uint8_t* scales, float* s_out,
                         float* partial, int partials_ready, uint32_t* raw, int* status, int num_sms,
                         cudaStream_t stream) {
  const long long n = (long long)T * K;
  int P = partials_ready > 0 ? partials_ready : quant_partials(n);
  if (s_in == nullptr && n > 0 && partials_ready <= 0) {
    cudaError_t err = launch_pdl(act_amax_kernel, P, kQuantThreads, 0, stream, X, n / 8, partial, status);
    if (err != cudaSuccess) return err;
  }
  if (n == 0) P = 0;  // no data: the quant kernel folds zero partials -> amax 0 -> s_x = 1
  QuantParams p;
  p.X = X; p.inv_perm = inv_perm; p.s_in = s_in; p.partial = partial; p.nparts = P;
  p.T = T; p.K = K; p.sf = sf; p.k = k; p.R = T * k; p.rcap = T * k + kActScalePadRows;
  p.codes = codes; p.scales = scales; p.s_out = s_out; p.status = status;
  // two-phase scales (32-element blocks, large R*K, raw buffer given): see act_scales_quad_kernel
  p.raw = (sf == 32 && raw != nullptr && quant_raw_bytes(p.R, K) > 0) ? raw : nullptr;
  const long long units = (long long)T * (K / (sf == 32 ? 32 : 8));   // lanes of work
  const long long pad = p.raw != nullptr ? 0
      : (long long)(K / (4 * sf)) * (T * k + kActScalePadRows - (T * k > 96 ? T * k - 96 : 0)) * 4;
  long long blocks = ((units > pad ? units : pad) + kQuantMainThreads - 1) / kQuantMainThreads;
  if (blocks < 1) blocks = 1;
  if (blocks > (long long)num_sms * 16) blocks = (long long)num_sms * 16;
  if (sf == 32) {
    cudaError_t e = launch_pdl(act_quant32_kernel, (unsigned)blocks, kQuantMainThreads, 0, stream, p);
    if (e != cudaSuccess || p.raw == nullptr) return e;
    const int KBa = K / 128;
    const dim3 grid((unsigned)ceil_div_i(p.rcap, kQuadTileRows), (unsigned)ceil_div_i(KBa, kQuadTileKb));
    return launch_pdl(act_scales_quad_kernel, grid, 256, 0, stream, (const uint32_t*)p.raw, p.R, KBa, p.rcap,
                      reinterpret_cast<uint32_t*>(scales));
  }
  return launch_pdl(act_quant_kernel, (unsigned)blocks, kQuantMainThreads, 0, stream, p);
}

}  // namespace gsg
