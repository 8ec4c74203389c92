// gsg_gemm.cu -- persistent grouped NVFP4 expert GEMM on the Blackwell tensor cores.
//
// "Hardware-Native Joint Sparse-Quantization for Trillion-Scale Mixture-of-Experts"
// (paperlayer.ai summary): §3.4 (pp.5-6) -- grouped execution of routing-dependent expert
// problems in one launch using Blackwell sparse MMA, the sparse weight placed as operand A;
// §2 "Hardware opportunity" (p.3) -- paired 4:8 NVFP4 runs at twice the dense NVFP4 rate;
// §D.2 (p.19) -- a dense control that differs from the sparse kernel only in sparsity.
//
// One CTA per SM, 352 threads (11 warps; 480 = 15 warps for wide pair tiles), warp-specialised
// around one shared-memory ring whose stages hold 256 to 768 logical K of one tile (weights,
// activation codes and both scales):
//   warp 0      weight producer: per stage one bulk copy per interleaved packed weight block and
//               one 3-D TMA box of the activation scale atoms, each from its own lane.
//   warp 2      activation producer: tensor-map TMA boxes (128B swizzle, 64 or 32 rows) of only the
//               token rows the tile holds, each from its own lane.
//   warps 7..10 scale/metadata loaders, one per TMEM lane quadrant: read the stage's metadata and
//               scale atoms from shared memory and tcgen05.st them into one of three TMEM sets.
//   warp 1      TMEM owner and MMA issuer: per stage only tcgen05.mma(.sp) kind::mxf4nvf4
//               block_scale (M = 128 weight rows, N = the tile's token count rounded to 16, K = 128
//               logical sparse / 64 dense) and one tcgen05.commit; up to eight TMEM accumulators.
//   warps 3..6  epilogue: tcgen05.ld accumulator lanes, multiply by s_x * s_w[e], store rows of Y.
//   warps 11..14 (wide pair tiles only) a second epilogue, for the tile's second n-tile pair.
// Every TMA and tcgen05 instruction is issued by an elected lane of a converged warp.
// 128-token tiles run on CTA pairs (cta_group::2, M = 256 weight rows).  Where N holds whole
// groups of four n-tiles, a pair tile is wide: 512 weight rows (two MMAs per k-block into two
// accumulators) against one 128-token activation tile, so the activations cross from L2 to the
// SMs once for 512 weight rows instead of once per 256.  Its two accumulators fill TMEM beside the
// metadata sets, so there is one accumulator buffer; the MMA warp waits for the epilogue between
// tiles, and the two epilogue warp groups halve that wait.
// Tiles are (expert e, 128 weight rows nt, token tile mt) in e -> nt -> mt order; CTAs take
// tiles round-robin and decode their own tile list into shared memory once, at set-up.
// Experts with no rows produce no tiles.  Every mbarrier wait is bounded:
// on expiry the kernel records GSG_ERR_DEVICE_TIMEOUT, drains its own copies and MMAs, frees
// TMEM and returns.
#include <atomic>

#include <cuda.h>

#include "gsg_internal.cuh"
#include "gsg_launch.h"

namespace gsg {

constexpr int kGemmThreads = 352;
// a wide pair tile adds four epilogue warps (11..14) that drain the tile's second n-tile while
// warps 3..6 drain the first
constexpr int kGemmThreadsWide = 480;
__host__ __device__ constexpr int gemm_threads(bool wide) { return wide ? kGemmThreadsWide : kGemmThreads; }
constexpr int kMaxE = 1024;
constexpr int kMaxAcc = 8;
constexpr int kNSets = 3;                  // TMEM sets of metadata + scales
constexpr uint32_t kSetCols = 64;
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;   // 2 s
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColAcc = kNSets * kSetCols;       // first accumulator (192)
constexpr int kOutStageBytes = 16 * 32 * 4;           // epilogue transpose buffer per warp
constexpr int kGluStageBytes = 32 * 36 * 4;           // SwiGLU epilogue: 32 tokens x 32 features (+4 pad)

struct GemmParams {
  const uint8_t* a_scales;
  const float* x_scale;
  const uint8_t* w_packed;
  const float* w_scale;
  const int32_t* off;
  void* Y;                 // Y [R][N] (bf16 or fp32); with the SwiGLU epilogue: h codes [R][N/4]
  int* status;
  int E, N, K, R, y_f32, rcap;
  int stages, nacc, tcap;
  int sched;               // tile schedule: kSchedRoundRobin or kSchedRuns (see tile_of)
  uint8_t* h_scales;       // SwiGLU epilogue: h scales, quad layout [N/256][R+256][4][4]
  const float* h_scale;    // SwiGLU epilogue: tensor scale of h
  // combine epilogue (perm_src non-null): Y is the slot buffer [T*k][N] bf16 (row = flat index
  // t*k + j of the routed pair), counters [T][N/32] (zero on entry, left zero), out [T][N] bf16
  const int32_t* perm_src;
  const float* gates;
  int* counters;
  uint16_t* out;
  int k;
  // test hook (0 = off): before its second tile (its first, if it has only one) the MMA warp waits
  // this long on a barrier that nothing arrives on, so that the bounded wait runs out and the
  // abort path -- status word, drain of copies and MMAs, TMEM release -- runs as it would after
  // a real stall
  unsigned long long stall_ns;
};

// ------------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// ---- CTA pairs (thread-block clusters of two CTAs on two SMs; see kCG below)
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// The shared::cluster address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_addr(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
// Arrive on an mbarrier given by its shared::cluster address (a barrier of this CTA or of the
// other CTA of the pair).  Default semantics (no cluster-scope release, which costs a fence per
// arrive): what the arrive hands over is already complete when it is issued -- copies that landed
// (their full barrier completed) and TMEM stores waited on with tcgen05.wait::st -- and is read
// only by the leader's tensor-core work issued after the leader observed the phase.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cl_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cl_addr) : "memory");
}
// Every thread of both CTAs of the cluster: all earlier writes (barrier initialisation included)
// are visible to the other CTA afterwards.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// The issue wrappers below are executed by a whole converged warp: elect.sync picks one lane
// and predicates the instruction on it, so the warp never diverges around a TMA or tcgen05
// instruction (issuing them from a lone lane of a diverged warp costs several times more).
#define GSG_ELECT "elect.sync _|P, 0xffffffff;\n\t"
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .pred P;\n\t" GSG_ELECT "@P mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n\t}" ::"r"(bar),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred P;\n\t" GSG_ELECT
      "@P cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n\t}" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred P;\n\t" GSG_ELECT
      "@P cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n\t}" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred P;\n\t" GSG_ELECT
      "@P cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];\n\t}" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}
// Per-lane forms: every lane of the (converged) warp executes the instruction and the lanes with
// `on` set each issue their own copy.  The TMA unit works through the copies of one issuing thread
// one after another, so the copies of a stage are spread over lanes to be in flight together.
__device__ __forceinline__ void bulk_g2s_lane(bool on, uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred P;\n\tsetp.ne.b32 P, %4, 0;\n\t"
      "@P cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n\t}" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "r"((uint32_t)on)
      : "memory");
}
__device__ __forceinline__ void tma_load_2d_lane(bool on, uint32_t dst, const CUtensorMap* map, int x, int y,
                                                 uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred P;\n\tsetp.ne.b32 P, %5, 0;\n\t"
      "@P cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n\t}" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "r"((uint32_t)on)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_lane(bool on, uint32_t dst, const CUtensorMap* map, int x, int y, int z,
                                                 uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred P;\n\tsetp.ne.b32 P, %6, 0;\n\t"
      "@P cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];\n\t}" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar), "r"((uint32_t)on)
      : "memory");
}
__device__ __forceinline__ void lds128(uint32_t saddr, uint32_t& a, uint32_t& b, uint32_t& c, uint32_t& d) {
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(a), "=r"(b), "=r"(c), "=r"(d) : "r"(saddr) : "memory");
}
// tcgen05.st of N consecutive 32-bit columns for the 32 lanes of this warp's quadrant.
__device__ __forceinline__ void tc_st_x4(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(r[0]), "r"(r[1]),
               "r"(r[2]), "r"(r[3])
               : "memory");
}
__device__ __forceinline__ void tc_st_x8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void tc_st_x16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// Writes `kCols` (a multiple of 4) columns from registers, largest pieces first.
template <int kCols>
__device__ __forceinline__ void tc_st_cols(uint32_t taddr, const uint32_t* r) {
  int c = 0;
#pragma unroll
  for (; c + 16 <= kCols; c += 16) tc_st_x16(taddr + c, r + c);
  if constexpr (kCols % 16 >= 8) {
    tc_st_x8(taddr + (kCols / 16) * 16, r + (kCols / 16) * 16);
  }
  if constexpr (kCols % 8 >= 4) {
    tc_st_x4(taddr + (kCols / 8) * 8, r + (kCols / 8) * 8);
  }
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("{\n\t.reg .pred P;\n\t" GSG_ELECT
               "@P tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
               : "memory");
}
// Pair form: once the pair's earlier tensor-core work has completed, arrive once on the barrier at
// this shared-memory offset in every CTA of `mask` (bit r = CTA rank r).
__device__ __forceinline__ void tc_commit_pair(uint32_t bar, uint16_t mask) {
  asm volatile("{\n\t.reg .pred P;\n\t" GSG_ELECT
               "@P tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
               "\n\t}" ::"r"(bar), "h"(mask)
               : "memory");
}
__device__ __forceinline__ void tc_mma_sparse(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate, uint32_t sfa, uint32_t sfb, uint32_t meta) {
  asm volatile(
      "{\n\t.reg .pred p, P;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t" GSG_ELECT
      "@P tcgen05.mma.sp.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, [%7], %3, [%5], [%6], p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb), "r"(meta)
      : "memory");
}
__device__ __forceinline__ void tc_mma_dense(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate, uint32_t sfa, uint32_t sfb) {
  asm volatile(
      "{\n\t.reg .pred p, P;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t" GSG_ELECT
      "@P tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}
// The same two MMAs issued for a CTA pair (M = 256: each CTA supplies its 128 weight rows and half
// of the tile's token columns from its own shared memory at the same offsets, and holds its rows'
// accumulator, metadata and scales -- the scales of all N token columns -- in its own TMEM at the
// same addresses).
__device__ __forceinline__ void tc_mma_sparse_pair(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                   uint32_t accumulate, uint32_t sfa, uint32_t sfb, uint32_t meta) {
  asm volatile(
      "{\n\t.reg .pred p, P;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t" GSG_ELECT
      "@P tcgen05.mma.sp.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, [%7], %3, [%5], [%6], p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb), "r"(meta)
      : "memory");
}
__device__ __forceinline__ void tc_mma_dense_pair(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                  uint32_t accumulate, uint32_t sfa, uint32_t sfb) {
  asm volatile(
      "{\n\t.reg .pred p, P;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t" GSG_ELECT
      "@P tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}
// 32 accumulator columns of this lane's TMEM row, times `scale`, rounded to bf16 and packed in
// pairs: h[i] = column 2i (low half) and column 2i + 1 (high half).
__device__ __forceinline__ void tc_ld_32_bf16(uint32_t taddr, float scale, uint32_t h[16]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(__uint_as_float(r[2 * i]), scale)));
    const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(__uint_as_float(r[2 * i + 1]), scale)));
    h[i] = lo | (hi << 16);
  }
}

__device__ __forceinline__ void tc_ld_16(uint32_t taddr, float v[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor (tcgen05 format): start, leading/stride byte offsets,
// version 1, layout type (0 = no swizzle, 2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | ((uint64_t)layout << 61);
}

// Instruction descriptor of kind::mxf4nvf4 block-scaled MMA: A/B E2M1, UE4M3 scales,
// K-major A and B, M = 128 (256 for a CTA pair), N = BN; bit 2 marks the sparse form (K = 128
// logical).
__host__ __device__ inline uint32_t make_idesc(bool sparse, int BN, int M = 128) {
  return (sparse ? (1u << 2) : 0u) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

struct Ctl {
  int abort;
  uint32_t tmem_base;
  int tile_begin, tile_end;   // this CTA's contiguous range of tiles
};

// Bounded wait: true when the phase completed; false on timeout or when another role aborted.
__device__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* status,
                             uint64_t limit_ns = kWaitTimeoutNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0u) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        *abort_flag = 1;
        set_status(status, GSG_ERR_DEVICE_TIMEOUT);
        return false;
      }
    }
  }
}

// Warp-uniform bounded wait: every lane polls, and the warp agrees on the outcome so that the
// .sync instructions that follow (elect.sync, tcgen05.ld/st) always see a converged warp.
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* status,
                                          uint64_t limit_ns = kWaitTimeoutNs) {
  const bool ok = wait_bounded(bar, parity, abort_flag, status, limit_ns);
  return __all_sync(0xffffffffu, ok);
}

// One tile of this CTA: expert, n-tile, first routed row and number of rows.
struct TileDesc {
  int e, nt, r0, valid;
};

// Largest e with pref[e] <= t (pref[0] = 0, pref[E] = total tiles), then the tile's rows.
__device__ __forceinline__ TileDesc decode_tile(int t, const int* pref, const int* offs, int E, int BN) {
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (pref[mid] <= t) lo = mid; else hi = mid;
  }
  const int local = t - pref[lo];
  const int mte = (offs[lo + 1] - offs[lo] + BN - 1) / BN;
  TileDesc d;
  d.e = lo;
  d.nt = local / mte;
  d.r0 = offs[lo] + (local % mte) * BN;
  d.valid = min(BN, offs[lo + 1] - d.r0);
  return d;
}

// Tile schedules (tiles numbered expert-major, then n-tile, then token tile):
//  kSchedRoundRobin: tile j * grid + CTA.  Neighbouring tiles run at the same time on different
//    CTAs, so the token tiles of one weight tile and the n-tiles of one activation tile are read
//    from DRAM once and shared through L2.
//  kSchedRuns: each CTA takes a contiguous run of tiles holding an equal share of the bytes (see
//    tile_at_cost) and streams its own stretch of the weight array.  Used when every expert has
//    one token tile and the CTAs hold dozens of tiles (decode batches of 32-256 tokens on 384
//    experts: 5-10 % faster); with several token tiles per expert it loses the sharing above
//    (the 30B and 1T prefill GEMMs ran 20-60 % slower), and with a handful of tiles per CTA
//    (one token on 8 experts) it measured 20 % slower.  A reversed-order (snake) round-robin,
//    tried for the load balance of heavy token tiles, measured slower than the plain one.
constexpr int kSchedRoundRobin = 0;
constexpr int kSchedRuns = 1;

// `unit` / `nunits`: this CTA's index and the number of CTAs, or for CTA pairs the pair's index
// and the number of pairs (both CTAs of a pair take the same tiles).
__device__ __forceinline__ int tile_of(int j, int sched, int tb, int unit, int nunits) {
  if (sched == kSchedRuns) return tb + j;
  return j * nunits + unit;
}

// The j-th tile of this CTA: from the shared-memory table filled at set-up, or decoded on the
// spot past its capacity.
__device__ __forceinline__ TileDesc my_tile(int j, const int4* table, int tcap, const int* pref, const int* offs,
                                            int E, int BN, int sched, int tb, int unit, int nunits) {
  if (j < tcap) {
    const int4 v = table[j];
    return TileDesc{v.x, v.y, v.z, v.w};
  }
  return decode_tile(tile_of(j, sched, tb, unit, nunits), pref, offs, E, BN);
}

// Tile schedule: every CTA takes a contiguous run of tiles (expert-major, then n-tile, then token
// tile) holding an equal share of the launch's bytes.  A tile's cost is its weight bytes wc plus
// ac per token row (activation codes and scales, output); costp[e] = cost of experts < e.  Returns
// the first tile that starts at or after `target` bytes (total_tiles when none does).
__device__ __forceinline__ int tile_at_cost(long long target, const long long* costp, const int* pref,
                                            const int* offs, int E, int BN, long long wc, long long ac) {
  if (target >= costp[E]) return pref[E];
  int lo = 0, hi = E;   // largest e with costp[e] <= target: a non-empty expert
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (costp[mid] <= target) lo = mid; else hi = mid;
  }
  const int rows = offs[lo + 1] - offs[lo];
  const int mte = (rows + BN - 1) / BN;
  const long long cn = mte * wc + rows * ac;            // one n-tile's token tiles
  const long long rel = target - costp[lo];
  long long nt = rel / cn;
  const long long rem = rel - nt * cn;
  const long long cf = wc + (long long)BN * ac;         // a full token tile (all but the last)
  long long tt = (rem + cf - 1) / cf;
  if (tt >= mte) { ++nt; tt = 0; }
  return pref[lo] + (int)(nt * mte + tt);
}

// 256-wide K chunks per ring stage: short token tiles take longer stages (fewer waits per weight
// byte); 128-token tiles keep two-chunk stages, also on CTA pairs (three-chunk stages, three of
// them in shared memory, measured slower than five two-chunk stages).  Wide pair tiles: two-chunk
// stages for the sparse weights (three 62 KB stages; six one-chunk stages measured slower), one
// chunk for the dense control's larger blocks.
__host__ __device__ constexpr int stage_chunks(bool sparse, int BN, bool glu, int cg, bool wide = false) {
  return wide ? (sparse ? 2 : 1) : glu ? 2 : sparse ? (BN <= 32 ? 3 : 2) : (BN <= 32 ? 2 : 1);
}

// Compile-time stage geometry of one (sparse/dense, token tile, SwiGLU, CTA group) instantiation.
// With the SwiGLU epilogue a tile holds two weight n-tiles (gate rows nt*128.., up rows
// N/2 + nt*128..) that share the activation tile: two MMAs per k-block into two accumulators side
// by side.  With kCG = 2 a tile is 256 weight rows (n-tiles 2*np and 2*np + 1) x kBN tokens, run
// by a pair of CTAs on two SMs: CTA r holds n-tile 2*np + r and half of the token rows, and the
// pair's MMAs (M = 256) read both CTAs' shared memory, so each SM stages its own weights but only
// half of the shared activation tile.
template <bool kSparse, int kBN, bool kGLU = false, int kCG = 1, bool kWide = false>
struct Geo {
  static_assert(kCG == 1 || (kCG == 2 && !kGLU && kBN == 128), "CTA pairs: 128-token tiles, plain epilogue");
  static_assert(!kWide || kCG == 2, "wide tiles run on CTA pairs");
  static constexpr int kNT = (kGLU || kWide) ? 2 : 1;              // weight n-tiles per tile (per CTA)
  static constexpr int kKbLogical = kSparse ? 128 : 64;            // logical K per MMA
  static constexpr int kKbPerChunk = kChunkK / kKbLogical;         // 2 sparse, 4 dense
  // 256-wide K chunks per stage: short token tiles take longer stages (fewer waits per weight byte)
  static constexpr int kCPS = stage_chunks(kSparse, kBN, kGLU, kCG, kWide);
  static constexpr int kKbps = kCPS * kKbPerChunk;                 // k-blocks per stage
  static constexpr int kCB = kSparse ? kSparseChunkBytes : kDenseChunkBytes;   // packed chunk block
  static constexpr int kCBMeta = 8192;                             // metadata offset in a chunk block
  static constexpr int kCBScale = kSparse ? 10240 : 16384;         // scale atoms offset in a chunk block
  static constexpr int kBRows = kBN / kCG;                         // token rows this CTA stages
  static constexpr int kBChunk = kBRows * 128;                     // activation codes per chunk
  static constexpr int kOffW = kCPS * kBChunk;                     // stage layout: B chunks | W blocks | SFB
  static constexpr int kOffSFB = kOffW + kNT * kCPS * kCB;
  static constexpr int kStage = (kOffSFB + kKbps * 512 + 1023) / 1024 * 1024;
  static constexpr int kMetaCols = kSparse ? 4 * kCPS * kNT : 0;   // TMEM set: meta | SFA | SFB
  static constexpr int kColSFA = kMetaCols;
  static constexpr int kColSFB = kMetaCols + 4 * kKbps * kNT;
  static constexpr int kSetUsed = kColSFB + 4 * kKbps;
  static constexpr uint32_t kBStep = kSparse ? 64 : 32;            // B bytes per row per MMA
  static constexpr int kBoxH = kBRows < 32 ? kBRows : 32;          // token rows per TMA box
  static constexpr int kAccStride = kBN < 32 ? 32 : kBN;
  static_assert(kSetUsed <= (int)kSetCols, "TMEM set too small");
};

// kCG = 2: launched as clusters of two CTAs (a CTA pair on two SMs) that run 256-row weight tiles
// together; see Geo.  CTA rank 0 of the pair (the leader) issues the pair's MMAs and owns the
// barriers the MMAs wait on (tfull, acce: arrived on by both CTAs' loader and epilogue warps);
// every MMA completion is signalled to the barriers of both CTAs (empty, accf).
// kNative: the dense control in the activation-stationary orientation -- the tile's 128 token rows
// are MMA operand A (M = 128, padded when fewer rows are routed) and the weight n-tile is operand
// B (N = 128); the accumulator then holds a token per TMEM lane and a feature per column.
// Combine epilogue, second phase: once every CTA of the launch has written its routed rows to their
// token slots (a bounded grid barrier on two counters of the workspace: every CTA is resident, one
// per SM), the CTAs sum each token's k slots in j order -- the scatter's arithmetic: fp32 products
// and running sum from 0, one bf16 rounding, eight outputs per thread (16-byte slot loads, the
// token's slots all in flight).  The last CTA to leave sets both counters back to zero.
__device__ void combine_tokens(const GemmParams& p, volatile int* abort_flag) {
  __shared__ int go;
  int* arrive = p.counters;
  int* depart = p.counters + 1;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();   // this CTA's slot stores before its arrival
    atomicAdd(arrive, 1);
    const uint64_t t0 = globaltimer_ns();
    int ok = 1;
    while (*reinterpret_cast<volatile int*>(arrive) < (int)gridDim.x) {
      if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
        set_status(p.status, GSG_ERR_DEVICE_TIMEOUT);
        ok = 0;
        break;
      }
    }
    __threadfence();   // the other CTAs' slot stores before this CTA's loads
    go = ok && !*abort_flag;
  }
  __syncthreads();
  if (go) {
    const int T = p.R / p.k;
    const unsigned n8 = (unsigned)p.N / 8u;
    const unsigned total = (unsigned)T * n8;   // T * N / 8 < 2^31 (checked on the host)
    const uint16_t* slots = static_cast<const uint16_t*>(p.Y);
    for (unsigned u = blockIdx.x * blockDim.x + threadIdx.x; u < total; u += gridDim.x * blockDim.x) {
      const int t = int(u / n8), c = int(u % n8);
      float acc[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] = 0.0f;
      for (int j0 = 0; j0 < p.k; j0 += 8) {
        float g[8];
        uint4 v[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const bool in = j0 + jj < p.k;
          g[jj] = in ? __ldg(p.gates + (size_t)t * p.k + j0 + jj) : 0.0f;
          v[jj] = in ? __ldcg(reinterpret_cast<const uint4*>(slots + ((size_t)t * p.k + j0 + jj) * p.N) + c)
                     : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          if (j0 + jj >= p.k) break;
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
      reinterpret_cast<uint4*>(p.out + (size_t)t * p.N)[c] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (atomicAdd(depart, 1) == (int)gridDim.x - 1) {   // every CTA has passed the barrier
      *reinterpret_cast<volatile int*>(arrive) = 0;
      *reinterpret_cast<volatile int*>(depart) = 0;
    }
  }
}

template <bool kSparse, int kBN, bool kGLU, int kCG, bool kNative = false, bool kWide = false>
__global__ void __launch_bounds__(gemm_threads(kWide), 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmap_b, const __grid_constant__ CUtensorMap tmap_b64,
                    const __grid_constant__ CUtensorMap tmap_sfb,
                    const GemmParams p) {
  using G = Geo<kSparse, kBN, kGLU, kCG, kWide>;
  constexpr int kThreads = gemm_threads(kWide);
  constexpr bool kPair = kCG == 2;
  static_assert(!kNative || (!kSparse && kBN == 128 && !kGLU && kCG == 1), "native orientation: dense, 128 tokens");
  extern __shared__ uint8_t smem_raw[];
  // NT: weight n-tiles; tiles run over NT / (kNT * kCG) columns (the gate n-tiles with the SwiGLU
  // epilogue, n-tile pairs for CTA pairs)
  const int E = p.E, NT = p.N / kTileN, NTt = NT / (G::kNT * kCG), KC = p.K / kChunkK;
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;         // this CTA's rank in its pair
  const int unit = kPair ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int nunits = kPair ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  const int S = p.stages, NACC = p.nacc;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + (size_t)S * G::kStage);
  // bars: full[S], empty[S], tfull[kNSets], accf[NACC], acce[NACC], drain, never (test hook)
  const int nbars = 2 * S + kNSets + 2 * NACC + 2;
  Ctl* ctl = reinterpret_cast<Ctl*>(bars + nbars);
  int* offs = reinterpret_cast<int*>(ctl + 1);   // [E+1]
  int* pref = offs + (E + 1);                    // [E+1]
  float* wsc = reinterpret_cast<float*>(pref + (E + 1));   // [E]
  long long* costp = reinterpret_cast<long long*>((reinterpret_cast<uintptr_t>(wsc + E) + 15) & ~uintptr_t(15));
  int4* ttab = reinterpret_cast<int4*>((reinterpret_cast<uintptr_t>(costp + (E + 1)) + 15) & ~uintptr_t(15));
  // per-epilogue-warp staging buffer: 16 tokens x 32 output features (fp32 worst case), or the
  // SwiGLU epilogue's 32 x 36 fp32
  uint8_t* ostage = reinterpret_cast<uint8_t*>(ttab + p.tcap);   // [4][kOutStageBytes or kGluStageBytes]
  volatile int* abort_flag = &ctl->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_u32(bars);
  const uint32_t sbase = smem_u32(base);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
  auto tfull_bar = [&](int s) { return bar0 + 8u * (2 * S + s); };
  auto accf_bar = [&](int a) { return bar0 + 8u * (2 * S + kNSets + a); };
  auto acce_bar = [&](int a) { return bar0 + 8u * (2 * S + kNSets + NACC + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * S + kNSets + 2 * NACC);
  const uint32_t never_bar = drain_bar + 8u;

  // ---- set-up: barriers, TMEM, tile schedule, tensor scales (global memory only after pdl_wait)
  pdl_launch_dependents();
  if (warp == 2 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_b)) : "memory");
    if (kBN >= 64) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_b64)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_sfb)) : "memory");
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(full_bar(s), 2); mbar_init(empty_bar(s), 1); }
    for (int s = 0; s < kNSets; ++s) mbar_init(tfull_bar(s), 4 * kCG);
    for (int a = 0; a < NACC; ++a) { mbar_init(accf_bar(a), 1); mbar_init(acce_bar(a), 4 * kCG * (kWide ? 2 : 1)); }
    mbar_init(drain_bar, 1);
    mbar_init(never_bar, 1);
    ctl->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    if constexpr (kPair) {   // the same columns in both CTAs of the pair (both warps 1 allocate)
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(&ctl->tmem_base)),
                   "r"(kTmemCols)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    } else {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(&ctl->tmem_base)),
                   "r"(kTmemCols)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
  }
  pdl_wait();
  // expert offsets, clamped to [0, R] so a corrupt array can never send a copy or a store out
  // of bounds (a decreasing pair makes that expert empty, see below)
  bool bad = false;
  for (int i = threadIdx.x; i <= E; i += blockDim.x) {
    int v = __ldg(p.off + i);
    if (v < 0 || v > p.R) { bad = true; v = v < 0 ? 0 : p.R; }
    offs[i] = v;
    if (i < E) wsc[i] = __ldg(p.w_scale + i);
  }
  if (kGLU) {
    // h scale entries that refer to rows >= R (no tile writes them): zero, shared by the CTAs
    const int r_lo = p.R > 96 ? p.R - 96 : 0, span = p.rcap - r_lo, kbh = p.N / 256;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < kbh * span * 4; i += gridDim.x * blockDim.x) {
      const int cc = i & 3, rest = i >> 2, rr = r_lo + rest % span, kb = rest / span;
      if (rr + 32 * cc >= p.R) *reinterpret_cast<uint32_t*>(p.h_scales + ((size_t)kb * p.rcap + rr) * 16 + cc * 4) = 0u;
    }
  }
  __syncthreads();
  {
    // chunked exclusive scan of tiles_e = ceil(rows_e / BN) * NTt over E experts
    const int per = (E + kThreads - 1) / kThreads;
    const int e0 = threadIdx.x * per, e1 = min(e0 + per, E);
    int local = 0;
    for (int e = e0; e < e1; ++e) {
      int rows = offs[e + 1] - offs[e];
      if (rows < 0) { bad = true; rows = 0; }
      local += ((rows + kBN - 1) / kBN) * NTt;
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    __shared__ int wsum[kThreads / 32];
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    int run = before + incl - local;
    for (int e = e0; e < e1; ++e) {
      pref[e] = run;
      int rows = offs[e + 1] - offs[e];
      if (rows < 0) rows = 0;
      run += ((rows + kBN - 1) / kBN) * NTt;
    }
    if (threadIdx.x == kThreads - 1) pref[E] = before + incl;
  }
  // bytes per tile: weights wc, plus ac per token row (codes, scales, output row segment)
  const long long wc = (long long)G::kNT * kCG * kTileN * p.K * (kSparse ? 11 : 18) / 32;
  const long long ac = p.K / 2 + p.K / (kSparse ? 32 : 16) + (long long)G::kNT * kCG * kTileN * (p.y_f32 ? 4 : 2);
  if (p.sched == kSchedRuns) {   // (only the byte-balanced schedule reads the costs; uniform branch)
    // chunked exclusive scan of cost_e = NTt * (ceil(rows_e / BN) * wc + rows_e * ac)
    const int per = (E + kThreads - 1) / kThreads;
    const int e0 = threadIdx.x * per, e1 = min(e0 + per, E);
    long long local = 0;
    for (int e = e0; e < e1; ++e) {
      const int rows = max(offs[e + 1] - offs[e], 0);
      local += (long long)NTt * (((rows + kBN - 1) / kBN) * wc + rows * ac);
    }
    long long incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    __shared__ long long csum[kThreads / 32];
    if (lane == 31) csum[warp] = incl;
    __syncthreads();
    long long run = incl - local;
    for (int w = 0; w < warp; ++w) run += csum[w];
    for (int e = e0; e < e1; ++e) {
      costp[e] = run;
      const int rows = max(offs[e + 1] - offs[e], 0);
      run += (long long)NTt * (((rows + kBN - 1) / kBN) * wc + rows * ac);
    }
    if (threadIdx.x == kThreads - 1) costp[E] = run;
  }
  if (bad) set_status(p.status, GSG_ERR_BAD_ROUTING);
  __syncthreads();
  const int total_tiles = pref[E];
  if (threadIdx.x == 0) {
    const int b = unit, G_ = nunits;
    if (p.sched == kSchedRuns) {
      const long long C = costp[E];
      const int tb = tile_at_cost(C * b / G_, costp, pref, offs, E, kBN, wc, ac);
      const int te = b == G_ - 1 ? total_tiles : tile_at_cost(C * (b + 1) / G_, costp, pref, offs, E, kBN, wc, ac);
      ctl->tile_begin = tb;
      ctl->tile_end = te;
    } else {
      ctl->tile_begin = 0;
      ctl->tile_end = b < total_tiles ? (total_tiles - b + G_ - 1) / G_ : 0;
    }
  }
  __syncthreads();
  const int tb = ctl->tile_begin;
  // this CTA's tiles, decoded once
  const int n_my = ctl->tile_end - tb;
  for (int j = threadIdx.x; j < n_my && j < p.tcap; j += blockDim.x) {
    const TileDesc d = decode_tile(tile_of(j, p.sched, tb, unit, nunits), pref, offs, E, kBN);
    ttab[j] = make_int4(d.e, d.nt, d.r0, d.valid);
  }
  tc_fence_before();
  if constexpr (kPair) {
    cluster_sync_all();   // both CTAs' barriers initialised before either arrives on the other's
  } else {
    __syncthreads();
  }
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp == 0 || warp == 2) {
    // =============================== producers: warp 0 weights, warp 2 activations.  The copies of
    // a stage are issued from separate lanes (see bulk_g2s_lane): the TMA unit works through one
    // thread's copies one after another, so one lane issuing every copy would keep a single copy
    // in flight per producer.
    const bool wprod = warp == 0;
    int s = 0, g = 0;   // ring slot and stage counter
    uint32_t ph = 0;
    for (int j = 0; j < n_my && !*abort_flag; ++j) {
      const TileDesc c = my_tile(j, ttab, p.tcap, pref, offs, E, kBN, p.sched, tb, unit, nunits);
      // this CTA's first weight n-tile: tile c.nt spans n-tiles [c.nt * kCG * kNT, +kCG * kNT) of the
      // expert (SwiGLU: the gate n-tiles only), CTA r of a pair takes every other one from r
      const uint8_t* wsrc =
          p.w_packed + ((size_t)c.e * NT + c.nt * kCG * (kWide ? 2 : 1) + rank) * KC * G::kCB;
      // its second n-tile: SwiGLU, the matching up n-tile; a wide pair tile, the next pair's
      const uint8_t* wsrc_up = wsrc + (size_t)(kWide ? kCG : NT / 2) * KC * G::kCB;
      // this CTA's token rows [r0, r0 + cnt): all of the tile's, or for a CTA pair the half of the
      // MMA's N = valid rounded up to 16 that this CTA supplies (rank 1: the upper half)
      const int nh = kPair ? ((c.valid + 15) & ~15) / 2 : kBN;
      const int r0 = c.r0 + (int)rank * nh;
      const int cnt = min(max(c.valid - (int)rank * nh, 0), nh);
      // token rows to fetch: whole 32-row boxes (BN <= 32: one box of BN rows), as few 64-row
      // boxes as possible for the larger tiles -- every TMA instruction costs the issuing warp
      const int rows = (cnt + G::kBoxH - 1) / G::kBoxH * G::kBoxH;
      const int n64 = G::kBRows >= 64 ? rows / 64 : 0;
      const int n32 = (rows - 64 * n64) / G::kBoxH;
      bool ok = true;
      for (int kc = 0; kc < KC; kc += G::kCPS) {
        const int nch = KC - kc >= G::kCPS ? G::kCPS : KC - kc;
        if (!wait_warp(empty_bar(s), ph ^ 1u, abort_flag, p.status)) { ok = false; break; }
        const uint32_t st = sbase + (uint32_t)s * G::kStage;
        const uint32_t fb = full_bar(s);
        if (wprod) {
          // weights (+ metadata + weight scales): lane t * nch + ch copies chunk block ch of weight
          // n-tile t (t = 1: the SwiGLU up n-tile); lane 31 copies the activation scale atoms of the
          // whole tile's tokens from its first row (in both CTAs of a pair: each CTA's MMA share
          // needs the scales of all N token columns)
          mbar_arrive_expect_tx(fb, (uint32_t)(G::kNT * nch * G::kCB + G::kKbps * 512));
          const int t = lane / nch, ch = lane - t * nch;
          bulk_g2s_lane(lane < G::kNT * nch, st + G::kOffW + (t * G::kCPS + ch) * G::kCB,
                        (t == 0 ? wsrc : wsrc_up) + (size_t)(kc + ch) * G::kCB, G::kCB, fb);
          tma_load_3d_lane(lane == 31, st + G::kOffSFB, &tmap_sfb, 0, c.r0, kc * G::kKbPerChunk, fb);
        } else {
          // activation codes: lane ch * nb + b copies box b (64-row boxes first) of chunk ch
          mbar_arrive_expect_tx(fb, (uint32_t)(nch * rows * 128));
          const int nb = n64 + n32;
          const int ch = nb > 0 ? lane / nb : 0, b = lane - ch * nb;
          const bool b64 = b < n64;
          const int roff = b64 ? 64 * b : 64 * n64 + (b - n64) * G::kBoxH;
          tma_load_2d_lane(lane < nch * nb, st + ch * G::kBChunk + roff * 128, b64 ? &tmap_b64 : &tmap_b,
                           (kc + ch) * 128, r0 + roff, fb);
        }
        ++g;
        if (++s == S) { s = 0; ph ^= 1u; }
      }
      if (!ok) break;
    }
    if (*abort_flag && lane == 0) {
      // wait (2 s in all) for copies still landing in the stages this warp filled: the last S
      // before stage g (the first one it did not issue)
      const uint64_t t0 = globaltimer_ns();
      for (int g2 = g > S ? g - S : 0; g2 < g; ++g2) {
        while (!mbar_try_wait(full_bar(g2 % S), (uint32_t)(g2 / S) & 1u) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
        }
      }
    }
  } else if (warp >= 7 && warp <= 10) {
    // =============================== metadata / scale loaders (TMEM quadrant q = warp % 4)
    const int q = warp & 3;
    const int row = 32 * q + lane;
    const uint32_t tlane = (uint32_t)(32 * q) << 16;
    int s = 0, set = 0, i = 0;
    uint32_t ph = 0;
    for (int j = 0; j < n_my && !*abort_flag; ++j) {
      bool ok = true;
      for (int kc = 0; kc < KC; kc += G::kCPS) {
        const int nch = KC - kc >= G::kCPS ? G::kCPS : KC - kc;
        // the TMEM set is free once the MMAs of the stage that last used it have completed
        if (i >= kNSets) {
          const int j = i - kNSets;
          if (!wait_warp(empty_bar(j % S), (uint32_t)(j / S) & 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
        }
        if (!wait_warp(full_bar(s), ph, abort_flag, p.status)) { ok = false; break; }
        const uint32_t st = sbase + (uint32_t)s * G::kStage;
        uint32_t r[G::kSetUsed];
        if (kSparse) {
#pragma unroll
          for (int t = 0; t < G::kNT; ++t)
#pragma unroll
            for (int ch = 0; ch < G::kCPS; ++ch)
              if (ch < nch) {
                const int m = 4 * (t * G::kCPS + ch);
                lds128(st + G::kOffW + (t * G::kCPS + ch) * G::kCB + G::kCBMeta + row * 16, r[m], r[m + 1], r[m + 2],
                       r[m + 3]);
              }
        }
#pragma unroll
        for (int kb = 0; kb < G::kKbps; ++kb) {
          if (kb < nch * G::kKbPerChunk) {
#pragma unroll
            for (int t = 0; t < G::kNT; ++t) {
              const uint32_t sfa = st + G::kOffW + (t * G::kCPS + kb / G::kKbPerChunk) * G::kCB + G::kCBScale +
                                   (kb % G::kKbPerChunk) * 512;
              const int m = G::kColSFA + 4 * (t * G::kKbps + kb);
              lds128(sfa + lane * 16, r[m], r[m + 1], r[m + 2], r[m + 3]);
            }
            lds128(st + G::kOffSFB + kb * 512 + lane * 16, r[G::kColSFB + 4 * kb], r[G::kColSFB + 4 * kb + 1],
                   r[G::kColSFB + 4 * kb + 2], r[G::kColSFB + 4 * kb + 3]);
          }
        }
        tc_st_cols<G::kSetUsed>(tmem + tlane + (uint32_t)set * kSetCols, r);
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {   // the set (and, for a pair, this CTA's stage) is ready for the MMA issuer
          if constexpr (kPair) mbar_arrive_cluster(cluster_addr(tfull_bar(set), 0u));
          else mbar_arrive(tfull_bar(set));
        }
        ++i;
        if (++set == kNSets) set = 0;
        if (++s == S) { s = 0; ph ^= 1u; }
      }
      if (!ok) break;
    }
  } else if (warp == 1) {
    // =============================== MMA issuer (whole warp, one elected lane issues); for a CTA
    // pair only the leader's, whose MMAs run on both SMs (the other CTA's warp 1 has no tiles)
    int s = 0, set = 0, i = 0, acc = 0;
    uint32_t ph = 0, aph = 0;   // ring phase, accumulator phase
    bool any = false;
    const int n_mma = rank == 0u ? n_my : 0;
    for (int j = 0; j < n_mma && !*abort_flag; ++j) {
      const TileDesc c = my_tile(j, ttab, p.tcap, pref, offs, E, kBN, p.sched, tb, unit, nunits);
      const uint32_t idesc = kNative ? make_idesc(false, kTileN, kBN)   // M = 128 tokens, N = 128 weight rows
                                     : make_idesc(kSparse, (c.valid + 15) & ~15, kTileN * kCG);
      if (p.stall_ns != 0ull && j == (n_mma > 1 ? 1 : 0) &&
          !wait_warp(never_bar, 0u, abort_flag, p.status, p.stall_ns))
        break;
      if (!wait_warp(acce_bar(acc), aph ^ 1u, abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem + kColAcc + (uint32_t)(acc * G::kNT * G::kAccStride);
      bool ok = true;
      for (int kc = 0; kc < KC; kc += G::kCPS) {
        const int nch = KC - kc >= G::kCPS ? G::kCPS : KC - kc;
        if (!wait_warp(full_bar(s), ph, abort_flag, p.status) ||
            !wait_warp(tfull_bar(set), (uint32_t)(i / kNSets) & 1u, abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t st = sbase + (uint32_t)s * G::kStage;
        const uint32_t tset = tmem + (uint32_t)set * kSetCols;
#pragma unroll
        for (int ch = 0; ch < G::kCPS; ++ch) {
          if (ch < nch) {
#pragma unroll
            for (int h = 0; h < G::kKbPerChunk; ++h) {
              const int kbi = ch * G::kKbPerChunk + h;
              const uint64_t bdesc = smem_desc(st + ch * G::kBChunk + G::kBStep * h, 16, 1024, 2);
              const uint32_t accum = (kc | ch | h) != 0 ? 1u : 0u;
#pragma unroll
              for (int t = 0; t < G::kNT; ++t) {
                const uint64_t adesc =
                    smem_desc(st + G::kOffW + (t * G::kCPS + ch) * G::kCB + 4096u * h, 128, 256, 0);
                const uint32_t d = d_tmem + (uint32_t)(t * G::kAccStride);
                const int kt = t * G::kKbps + kbi;
                const uint32_t sfa = tset + G::kColSFA + 4 * kt, sfb = tset + G::kColSFB + 4 * kbi;
                if constexpr (kNative)   // tokens as A, weights as B: the operands and their scales swap
                  tc_mma_dense(d, bdesc, adesc, idesc, accum, sfb, sfa);
                else if constexpr (kSparse && kPair)
                  tc_mma_sparse_pair(d, adesc, bdesc, idesc, accum, sfa, sfb, tset + 2 * kt);
                else if constexpr (kSparse)
                  tc_mma_sparse(d, adesc, bdesc, idesc, accum, sfa, sfb, tset + 2 * kt);
                else if constexpr (kPair)
                  tc_mma_dense_pair(d, adesc, bdesc, idesc, accum, sfa, sfb);
                else
                  tc_mma_dense(d, adesc, bdesc, idesc, accum, sfa, sfb);
              }
            }
          }
        }
        if constexpr (kPair) tc_commit_pair(empty_bar(s), 3);   // the stage is free in both CTAs
        else tc_commit(empty_bar(s));
        any = true;
        ++i;
        if (++set == kNSets) set = 0;
        if (++s == S) { s = 0; ph ^= 1u; }
      }
      if (!ok) break;
      if constexpr (kPair) tc_commit_pair(accf_bar(acc), 3);   // both CTAs' epilogues
      else tc_commit(accf_bar(acc));
      if (++acc == NACC) { acc = 0; aph ^= 1u; }
    }
    __syncwarp();
    if (any) {
      // all MMAs issued by this warp have completed once the drain barrier fires
      if constexpr (kPair) tc_commit_pair(drain_bar, 1);
      else tc_commit(drain_bar);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(drain_bar, 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
    }
  } else {
    // =============================== epilogue (warps 3..6, and 11..14 for wide tiles -> TMEM lane
    // quadrants 3,0,1,2)
    const int q = warp & 3;
    const float sx = __ldg(p.x_scale);
    int acc = 0;
    uint32_t aph = 0;
    for (int j = 0; j < n_my; ++j) {
      const TileDesc c = my_tile(j, ttab, p.tcap, pref, offs, E, kBN, p.sched, tb, unit, nunits);
      const int r0 = c.r0, valid = c.valid;
      if (!wait_warp(accf_bar(acc), aph, abort_flag, p.status)) break;
      tc_fence_after();
      const float scale = __fmul_rn(sx, wsc[c.e]);
      const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + kColAcc + (uint32_t)(acc * G::kNT * G::kAccStride);
      bool released = false;   // the accumulator already handed back to the MMA warp
      if constexpr (kNative) {
        // lane = token 32q + lane of the tile, columns = the n-tile's 128 features: each lane scales
        // and stores its own token's row segment (16-byte stores, 16 features at a time)
        const int tok = 32 * q + lane;
        const size_t col0 = (size_t)c.nt * kTileN;
        for (int f0 = 0; f0 < kTileN; f0 += 16) {
          float v[16];
          tc_ld_16(taddr + f0, v);
          if (tok < valid) {
            if (p.y_f32) {
              float* Yr = static_cast<float*>(p.Y) + (size_t)(r0 + tok) * p.N + col0 + f0;
#pragma unroll
              for (int w = 0; w < 4; ++w)
                *reinterpret_cast<float4*>(Yr + 4 * w) =
                    make_float4(__fmul_rn(v[4 * w], scale), __fmul_rn(v[4 * w + 1], scale),
                                __fmul_rn(v[4 * w + 2], scale), __fmul_rn(v[4 * w + 3], scale));
            } else {
              uint32_t pk[8];
#pragma unroll
              for (int w = 0; w < 8; ++w)
                pk[w] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(v[2 * w], scale))) |
                        ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(v[2 * w + 1], scale))) << 16);
              uint4* Yr = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.Y) + (size_t)(r0 + tok) * p.N + col0 + f0);
              Yr[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
              Yr[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
          }
        }
      } else if constexpr (kGLU) {
        // SwiGLU output preparation, 32 tokens at a time: lane = feature f of this warp's
        // 32-feature block (one NVFP4 block of the down-projection's K), h = silu(gate) * up in
        // fp32; the block is transposed through shared memory so that each lane then owns one
        // token's 32 values: block max, UE4M3 scale and E2M1 codes once per token, 16-byte code
        // stores, scale bytes into the quad layout (k-block nt, position q).
        const float sh = __ldg(p.h_scale);
        const float six_sh = __fmul_rn(6.0f, sh);
        const int f0 = c.nt * kTileN + 32 * q;
        const int hrow = p.N / 4;                 // bytes of h codes per row (N/2 features)
        uint8_t* hc = static_cast<uint8_t*>(p.Y);
        const uint32_t tb = smem_u32(ostage + (size_t)(warp - 3) * kGluStageBytes);   // [32][36] fp32
        for (int c0 = 0; c0 < valid; c0 += 32) {
          float g[32], u[32];
          tc_ld_16(taddr + c0, g);
          tc_ld_16(taddr + c0 + 16, g + 16);
          tc_ld_16(taddr + G::kAccStride + c0, u);
          tc_ld_16(taddr + G::kAccStride + c0 + 16, u + 16);
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            const float gs = __fmul_rn(g[t], scale), us = __fmul_rn(u[t], scale);
            const float hv = __fmul_rn(__fdividef(gs, __fadd_rn(1.0f, __expf(-gs))), us);
            asm volatile("st.shared.f32 [%0], %1;" ::"r"(tb + (uint32_t)(t * 36 + lane) * 4u), "f"(hv) : "memory");
          }
          __syncwarp();
          float v[32];
#pragma unroll
          for (int k4 = 0; k4 < 8; ++k4) {
            uint32_t a, b, cc, d;
            lds128(tb + (uint32_t)(lane * 36 + 4 * k4) * 4u, a, b, cc, d);
            v[4 * k4] = __uint_as_float(a);
            v[4 * k4 + 1] = __uint_as_float(b);
            v[4 * k4 + 2] = __uint_as_float(cc);
            v[4 * k4 + 3] = __uint_as_float(d);
          }
          __syncwarp();
          float am = 0.0f;
#pragma unroll
          for (int k = 0; k < 32; ++k) am = fmaxf(am, fabsf(v[k]));
          const BlockScale bs = block_scale_cvt(am, six_sh, sh);
          uint32_t wd[4];
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            float xs[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) xs[i] = __fmul_rn(v[8 * w + i], bs.inv);
            wd[w] = e2m1_encode8_cvt(xs);
          }
          const int row = r0 + c0 + lane;
          if (c0 + lane < valid) {
            *reinterpret_cast<uint4*>(hc + (size_t)row * hrow + f0 / 2) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              const int rr = row - 32 * cc;
              if (rr >= 0) p.h_scales[((size_t)c.nt * p.rcap + rr) * 16 + cc * 4 + q] = (uint8_t)bs.sc;
            }
          }
        }
      } else {
      // Each 16-token chunk: TMEM lane (= output feature) -> registers, scale, transpose through
      // the warp's shared buffer into [token][32 features], then 16-byte stores of whole row
      // segments (64 B bf16 / 128 B fp32 per token).
      uint8_t* obuf = ostage + (size_t)(warp >= 11 ? warp - 7 : warp - 3) * kOutStageBytes;
      const uint32_t obuf_s = smem_u32(obuf);
      // the tile's n-tiles: a wide pair tile's second one goes to warps 11..14
      const int u_begin = kWide ? (warp >= 11 ? 1 : 0) : 0, u_end = kWide ? u_begin + 1 : G::kNT;
      if constexpr (kBN == 128 && G::kNT == 1 + (kWide ? 1 : 0)) {
        if (!p.y_f32 && p.perm_src == nullptr) {
          // bf16 output of a 128-token tile (one n-tile per warp): the warp's whole accumulator
          // block in 32-column TMEM loads, held as packed bf16, and the accumulator released
          // before any store, so the MMA warp's next tile waits for the loads, not for the stores
          const uint32_t tcol = taddr + (uint32_t)(u_begin * G::kAccStride);
          const size_t col0 = ((size_t)c.nt * kCG * G::kNT + u_begin * kCG + rank) * kTileN + 32 * q;
          uint32_t hb[64];
#pragma unroll
          for (int h = 0; h < 4; ++h)
            if (32 * h < valid) tc_ld_32_bf16(tcol + 32u * h, scale, hb + 16 * h);   // warp-uniform
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if constexpr (kPair) mbar_arrive_cluster(cluster_addr(acce_bar(acc), 0u));
            else mbar_arrive(acce_bar(acc));
          }
          released = true;
          __nv_bfloat16* Y = static_cast<__nv_bfloat16*>(p.Y);
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            if (16 * g < valid) {   // warp-uniform
#pragma unroll
              for (int j = 0; j < 16; j += 2) {
                const uint32_t w = hb[8 * g + j / 2];
                asm volatile("st.shared.u16 [%0], %1;" ::"r"(obuf_s + (uint32_t)(j * 64 + lane * 2)),
                             "h"((unsigned short)(w & 0xffffu)) : "memory");
                asm volatile("st.shared.u16 [%0], %1;" ::"r"(obuf_s + (uint32_t)((j + 1) * 64 + lane * 2)),
                             "h"((unsigned short)(w >> 16)) : "memory");
              }
              __syncwarp();
#pragma unroll
              for (int k = 0; k < 2; ++k) {   // 16 tokens x 4 chunks of 16 B
                const int ci = lane + 32 * k, tok = ci >> 2, part = ci & 3;
                if (16 * g + tok < valid) {
                  uint32_t a, b, cc, d;
                  lds128(obuf_s + (uint32_t)(tok * 64 + part * 16), a, b, cc, d);
                  *reinterpret_cast<uint4*>(Y + (size_t)(r0 + 16 * g + tok) * p.N + col0 + part * 8) =
                      make_uint4(a, b, cc, d);
                }
              }
              __syncwarp();
            }
          }
        }
      }
      for (int u = u_begin; u < u_end && !released; ++u) {
      // first feature of this warp
      const size_t col0 = ((size_t)c.nt * kCG * G::kNT + u * kCG + rank) * kTileN + 32 * q;
      for (int c0 = 0; c0 < valid; c0 += 16) {
        float v[16];
        tc_ld_16(taddr + (uint32_t)(u * G::kAccStride) + c0, v);
        if (p.y_f32) {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            asm volatile("st.shared.f32 [%0], %1;" ::"r"(obuf_s + (uint32_t)(j * 128 + lane * 4)), "f"(__fmul_rn(v[j], scale)) : "memory");
          __syncwarp();
          float* Y = static_cast<float*>(p.Y);
#pragma unroll
          for (int k = 0; k < 4; ++k) {          // 16 tokens x 8 chunks of 16 B
            const int ci = lane + 32 * k, tok = ci >> 3, part = ci & 7;
            if (c0 + tok < valid) {
              uint32_t a, b, cc, d;
              lds128(obuf_s + (uint32_t)(tok * 128 + part * 16), a, b, cc, d);
              *reinterpret_cast<uint4*>(Y + (size_t)(r0 + c0 + tok) * p.N + col0 + part * 4) = make_uint4(a, b, cc, d);
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const unsigned short h = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(v[j], scale)));
            asm volatile("st.shared.u16 [%0], %1;" ::"r"(obuf_s + (uint32_t)(j * 64 + lane * 2)), "h"(h) : "memory");
          }
          __syncwarp();
          __nv_bfloat16* Y = static_cast<__nv_bfloat16*>(p.Y);
          // combine: lane j < 16 holds the flat index f = t*k + j of chunk row j; the row goes to
          // slot f instead of row r
          const bool comb = p.perm_src != nullptr;
          int myf = (comb && lane < 16 && c0 + lane < valid) ? __ldg(p.perm_src + r0 + c0 + lane) : 0;
          // a slot index outside [0, T*k) (corrupt routing) gets nothing stored
          const unsigned badf = __ballot_sync(0xffffffffu, comb && lane < 16 && c0 + lane < valid &&
                                                               (myf < 0 || myf >= p.R));
          if (badf != 0u && lane == 0) set_status(p.status, GSG_ERR_BAD_ROUTING);
          if ((badf >> lane) & 1u) myf = 0;
#pragma unroll
          for (int k = 0; k < 2; ++k) {          // 16 tokens x 4 chunks of 16 B
            const int ci = lane + 32 * k, tok = ci >> 2, part = ci & 3;
            const int f = __shfl_sync(0xffffffffu, myf, tok);
            if (c0 + tok < valid && !((badf >> tok) & 1u)) {
              uint32_t a, b, cc, d;
              lds128(obuf_s + (uint32_t)(tok * 64 + part * 16), a, b, cc, d);
              const size_t dst = comb ? (size_t)f : (size_t)(r0 + c0 + tok);
              *reinterpret_cast<uint4*>(Y + dst * p.N + col0 + part * 8) = make_uint4(a, b, cc, d);
            }
          }
        }
        __syncwarp();
      }
      }
      }
      if (!released) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {   // the accumulator may be overwritten (for a pair: once both CTAs read it)
          if constexpr (kPair) mbar_arrive_cluster(cluster_addr(acce_bar(acc), 0u));
          else mbar_arrive(acce_bar(acc));
        }
      }
      if (++acc == NACC) { acc = 0; aph ^= 1u; }
    }
  }

  // ---- teardown (a CTA of a pair leaves only once the other is done with its shared memory and
  // barriers: the leader's MMAs read both CTAs' stages, and both CTAs arrive on the leader's
  // barriers)
  tc_fence_before();
  if constexpr (kPair) {
    __syncwarp();          // the cluster barrier is executed by converged warps
    cluster_sync_all();
  } else {
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    if constexpr (kPair)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    else
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
  if (p.perm_src != nullptr) combine_tokens(p, abort_flag);
}

// ------------------------------------------------------------------ host side
struct GemmPlan {
  int BN, cps, stage, stages, nacc, tcap;
  size_t smem;
};

constexpr int kMaxStages = 12;
constexpr int kStageBudget128 = 192 * 1024;   // 128-token tiles: a deeper ring only adds L2 pressure
// opt-in dynamic shared memory per block minus room for static shared memory (set per device)
static int g_smem_limit = 232448 - 1024;

// tcap: capacity of the per-CTA tile table (tiles beyond it are decoded on the fly); an upper
// bound on a CTA's tiles is ceil((ceil(R/BN) + E) * NT / grid).  cg = 2: a CTA of a pair, which
// stages half of the tile's token rows (the geometry of Geo<..., 2>).
static GemmPlan make_plan(bool sparse, int BN, int E, int tcap, bool glu = false, int cg = 1, bool wide = false) {
  GemmPlan g;
  g.BN = BN;
  g.tcap = tcap;
  // weight n-tiles per tile and CTA: gate + up with the SwiGLU epilogue, two n-tile pairs for a
  // wide pair tile
  const int nt = glu || wide ? 2 : 1;
  g.cps = stage_chunks(sparse, BN, glu, cg, wide);
  const int kbps = g.cps * (sparse ? 2 : 4);
  const int body =
      g.cps * (BN / cg) * 128 + nt * g.cps * (sparse ? kSparseChunkBytes : kDenseChunkBytes) + kbps * 512;
  g.stage = (body + 1023) / 1024 * 1024;
  // everything but the stage ring and the tile table, at its largest
  const int ostage = (wide ? 8 : 4) * (glu ? kGluStageBytes : kOutStageBytes);
  const int fixed = 1024 + (2 * kMaxStages + kNSets + 2 * kMaxAcc + 2) * 8 + (int)sizeof(Ctl) + (3 * E + 2) * 4 +
                    16 + (E + 1) * 8 + 16 + ostage;
  int budget = g_smem_limit - fixed;
  if (BN == 128 && cg == 1 && budget > kStageBudget128) budget = kStageBudget128;
  g.stages = (budget - tcap * 16) / g.stage;
  if (g.stages > kMaxStages) g.stages = kMaxStages;
  // the ring comes before the tile table: where the table would cost a stage, it keeps only what
  // fits beside the full ring (a CTA decodes its later tiles from the expert offsets instead)
  int ring = budget / g.stage;
  if (ring > kMaxStages) ring = kMaxStages;
  if (g.stages < ring) {
    g.stages = ring;
    g.tcap = (budget - ring * g.stage) / 16;
  }
  const int acc_stride = (BN < 32 ? 32 : BN) * nt;
  g.nacc = (int)((kTmemCols - kColAcc) / acc_stride);
  if (g.nacc > kMaxAcc) g.nacc = kMaxAcc;
  const int nbars = 2 * g.stages + kNSets + 2 * g.nacc + 2;
  g.smem = 1024 + (size_t)g.stages * g.stage + nbars * 8 + sizeof(Ctl) + (size_t)(3 * E + 2) * 4 + 16 +
           (size_t)(E + 1) * 8 + 16 +
           (size_t)g.tcap * 16 + ostage;
  return g;
}

constexpr int kMaxTableTiles = 1024;

// test hook: the MMA warp's stall of GemmParams::stall_ns for the launches that follow (0 = off)
static std::atomic<unsigned long long> g_test_stall_ns{0ull};
void gemm_set_test_stall(unsigned long long ns) { g_test_stall_ns.store(ns); }
// test hook: at most this many entries of the per-CTA tile table (-1 = no limit); the tiles past
// it are decoded from the expert offsets as the roles reach them
static std::atomic<int> g_test_table_cap{-1};
void gemm_set_test_table_cap(int cap) { g_test_table_cap.store(cap); }

// Token tile: the smallest of 16/32/64 that holds the largest expert; past 64 rows, 128 only when
// experts average at least 64 rows (R / E), since a 128-row activation chunk takes shared memory
// from the weight ring that the many small experts of a skewed routing would leave unused.
int gemm_pick_bn(int max_rows, int R, int E) {
  if (max_rows > 0 && max_rows <= 16) return 16;
  if (max_rows > 0 && max_rows <= 32) return 32;
  if (max_rows > 0 && max_rows <= 64) return 64;
  return (long long)R >= 64ll * E ? 128 : 64;
}

bool gemm_supported(int E) { return E >= 1 && E <= kMaxE; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

template <bool kSparse, int kBN, bool kGLU = false, int kCG = 1, bool kNative = false, bool kWide = false>
static cudaError_t set_attr_one(int bytes) {
  return cudaFuncSetAttribute(grouped_gemm_kernel<kSparse, kBN, kGLU, kCG, kNative, kWide>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

// CTA pairs the device can hold at once at one CTA per SM (the pairs' SMs must share a GPC), per
// sparse/dense; 0 when the device cannot run them (then 128-token tiles run one CTA per tile).
static int g_pair_units[2] = {0, 0};
static int g_wide_units[2] = {0, 0};   // the same for the wide pair tiles

template <bool kSparse, bool kWide = false>
static int max_pairs(int smem) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(gemm_threads(kWide));
  cfg.dynamicSmemBytes = (size_t)smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, grouped_gemm_kernel<kSparse, 128, false, 2, false, kWide>, &cfg) !=
      cudaSuccess) {
    cudaGetLastError();   // clear the error: pairs are then simply not used
    return 0;
  }
  return n;
}

cudaError_t gemm_set_smem_attrs() {
  // every plan stays below the opt-in limit (make_plan sizes the ring from it)
  int dev = 0, maxb = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&maxb, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  maxb -= 1024;   // room for the kernels' static shared memory
  g_smem_limit = maxb;
  cudaError_t errs[16] = {set_attr_one<true, 16>(maxb),       set_attr_one<true, 32>(maxb),
                          set_attr_one<true, 64>(maxb),       set_attr_one<true, 128>(maxb),
                          set_attr_one<false, 16>(maxb),      set_attr_one<false, 32>(maxb),
                          set_attr_one<false, 64>(maxb),      set_attr_one<false, 128>(maxb),
                          set_attr_one<true, 16, true>(maxb), set_attr_one<true, 32, true>(maxb),
                          set_attr_one<true, 64, true>(maxb), set_attr_one<true, 128, false, 2>(maxb),
                          set_attr_one<false, 128, false, 2>(maxb), set_attr_one<false, 128, false, 1, true>(maxb),
                          set_attr_one<true, 128, false, 2, false, true>(maxb),
                          set_attr_one<false, 128, false, 2, false, true>(maxb)};
  for (cudaError_t x : errs)
    if (x != cudaSuccess) return x;
  g_pair_units[1] = max_pairs<true>(maxb);
  g_pair_units[0] = max_pairs<false>(maxb);
  g_wide_units[1] = max_pairs<true, true>(maxb);
  g_wide_units[0] = max_pairs<false, true>(maxb);
  return cudaSuccess;
}

template <bool kSparse, bool kGLU = false>
static cudaError_t launch_bn(int BN, int grid, size_t smem, cudaStream_t stream, const CUtensorMap& tb,
                             const CUtensorMap& tb64, const CUtensorMap& ts, const GemmParams& p) {
  switch (BN) {
    case 16: return launch_pdl(grouped_gemm_kernel<kSparse, 16, kGLU, 1>, grid, kGemmThreads, smem, stream, tb, tb64, ts, p);
    case 32: return launch_pdl(grouped_gemm_kernel<kSparse, 32, kGLU, 1>, grid, kGemmThreads, smem, stream, tb, tb64, ts, p);
    default: return launch_pdl(grouped_gemm_kernel<kSparse, 64, kGLU, 1>, grid, kGemmThreads, smem, stream, tb, tb64, ts, p);
  }
}

template <bool kSparse>
static cudaError_t launch_bn(int BN, int grid, size_t smem, cudaStream_t stream, const CUtensorMap& tb,
                             const CUtensorMap& tb64, const CUtensorMap& ts, const GemmParams& p, bool glu,
                             bool pair, bool native = false, bool wide = false) {
  if (glu) return launch_bn<true, true>(BN, grid, smem, stream, tb, tb64, ts, p);
  if (!kSparse && native)
    return launch_pdl(grouped_gemm_kernel<false, 128, false, 1, true>, grid, kGemmThreads, smem, stream, tb, tb64, ts,
                      p);
  if (BN == 128 && pair && wide)
    return launch_pdl_cluster(grouped_gemm_kernel<kSparse, 128, false, 2, false, true>, grid, kGemmThreadsWide, smem,
                              stream, 2u, tb, tb64, ts, p);
  if (BN == 128 && pair)
    return launch_pdl_cluster(grouped_gemm_kernel<kSparse, 128, false, 2>, grid, kGemmThreads, smem, stream, 2u, tb,
                              tb64, ts, p);
  if (BN == 128)
    return launch_pdl(grouped_gemm_kernel<kSparse, 128, false, 1>, grid, kGemmThreads, smem, stream, tb, tb64, ts, p);
  return launch_bn<kSparse, false>(BN, grid, smem, stream, tb, tb64, ts, p);
}

// returns 0 ok, 1 cuda error, 2 tensor map failure.  h_scales / h_scale non-null: the SwiGLU
// epilogue (sparse only; Y receives the h codes).  comb non-null: the combine epilogue (Y is the
// slot buffer, bf16 output only).
int launch_gemm(bool sparse, const uint8_t* a_codes, const uint8_t* a_scales, const float* x_scale,
                const uint8_t* w_packed, const float* w_scale, const int32_t* off, int E, int N, int K, int R,
                int max_rows, void* Y, int y_f32, int* status, int num_sms, cudaStream_t stream,
                uint8_t* h_scales, const float* h_scale, const CombineArgs* comb, bool native) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr) return 2;
  const bool glu = h_scales != nullptr;
  if (native && (sparse || glu || comb != nullptr)) return 1;
  int BN = native ? 128 : gemm_pick_bn(max_rows, R, E);   // the native orientation: 128-token tiles (MMA M)
  if (glu && BN > 64) BN = 64;   // two accumulators per tile: 64-token tiles at most
  // 128-token tiles run as CTA pairs (256 weight rows per tile) when N holds whole n-tile pairs
  // and the device can co-schedule pairs
  // a wide pair tile (no combine epilogue, N a multiple of 512) holds two n-tile pairs, 512 weight
  // rows, and reads its 128 tokens' activations once for both
  const bool wide = BN == 128 && !glu && !native && comb == nullptr && (N / kTileN) % 4 == 0 &&
                    g_wide_units[sparse ? 1 : 0] > 0;
  const int pair_units = wide ? g_wide_units[sparse ? 1 : 0] : g_pair_units[sparse ? 1 : 0];
  const bool pair = BN == 128 && !glu && !native && (N / kTileN) % 2 == 0 && pair_units > 0;
  const int cg = pair ? 2 : 1;
  const int units = pair ? (pair_units < num_sms / 2 ? pair_units : num_sms / 2) : num_sms;   // pairs or CTAs
  const int grid = units * cg;
  const int ntt = glu || (pair && wide) ? 2 : 1;   // weight n-tiles per tile and CTA
  const long long bound = (((long long)R + BN - 1) / BN + E) * (N / kTileN / ntt / cg);
  // schedule: contiguous byte-balanced runs when every expert fits one token tile (max_rows known)
  // and the CTAs can hold at least 32 tiles each (at most min(E, R) experts are touched), else
  // round-robin
  const int NTt = N / kTileN / ntt / cg;
  const long long touched_max = R < E ? R : E;
  const int sched = (!pair && max_rows > 0 && max_rows <= BN && touched_max * NTt >= 32LL * units) ? kSchedRuns
                                                                                                  : kSchedRoundRobin;
  long long tcap;
  if (sched == kSchedRuns) {
    // a CTA's share of the bytes holds at most (wc + BN ac) / (wc + ac) times the average tile count
    const long long wc = (glu ? 2LL : 1LL) * kTileN * K * (sparse ? 11 : 18) / 32;
    const long long ac = K / 2 + K / (sparse ? 32 : 16) + (glu ? 2LL : 1LL) * kTileN * (y_f32 ? 4 : 2);
    tcap = (bound * (wc + BN * ac) / (wc + ac) + units - 1) / units + 2;
  } else {
    tcap = (bound + units - 1) / units;
  }
  if (tcap > kMaxTableTiles) tcap = kMaxTableTiles;
  const int tcap_test = g_test_table_cap.load();
  if (tcap_test >= 0 && tcap > tcap_test) tcap = tcap_test;
  const GemmPlan g = make_plan(sparse, BN, E, (int)tcap, glu, cg, pair && wide);
  if (g.stages < kNSets || g.smem > (size_t)g_smem_limit) return 1;   // ring too shallow: refuse, launch nothing
  const int box_h = g.BN / cg < 32 ? g.BN / cg : 32;
  const int kbps = g.cps * (sparse ? 2 : 4);
  const int rcap = R + kActScalePadRows;
  const int KBa = K / (sparse ? 128 : 64);
  CUtensorMap tb, tb64, ts;
  // activation codes [R][K/2]: boxes of 128 bytes x box_h rows, and (token tiles >= 64) x 64 rows
  for (int m = 0; m < 2; ++m) {
    if (m == 1 && g.BN / cg < 64) { tb64 = tb; break; }
    cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)R};
    cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    cuuint32_t box[2] = {128u, (cuuint32_t)(m == 0 ? box_h : 64)};
    cuuint32_t estr[2] = {1u, 1u};
    if (enc(m == 0 ? &tb : &tb64, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(a_codes), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return 2;
  }
  {
    // activation scale quad entries as a [KBa][rcap][16 B] tensor; one box = the stage's atoms
    cuuint64_t dims[3] = {16u, (cuuint64_t)rcap, (cuuint64_t)KBa};
    cuuint64_t strides[2] = {16u, (cuuint64_t)rcap * 16u};
    cuuint32_t box[3] = {16u, 32u, (cuuint32_t)kbps};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    if (enc(&ts, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(a_scales), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return 2;
  }
  GemmParams p;
  p.a_scales = a_scales; p.x_scale = x_scale; p.w_packed = w_packed;
  p.w_scale = w_scale; p.off = off; p.Y = Y; p.status = status;
  p.E = E; p.N = N; p.K = K; p.R = R; p.y_f32 = y_f32; p.rcap = rcap;
  p.stages = g.stages; p.nacc = g.nacc; p.tcap = g.tcap; p.sched = sched;
  p.h_scales = h_scales; p.h_scale = h_scale;
  p.perm_src = comb ? comb->perm_src : nullptr;
  p.gates = comb ? comb->gates : nullptr;
  p.counters = comb ? comb->counters : nullptr;
  p.out = comb ? comb->out : nullptr;
  p.k = comb ? comb->k : 1;
  p.stall_ns = g_test_stall_ns.load();
  const cudaError_t e = sparse ? launch_bn<true>(g.BN, grid, g.smem, stream, tb, tb64, ts, p, glu, pair, false, wide)
                               : launch_bn<false>(g.BN, grid, g.smem, stream, tb, tb64, ts, p, false, pair, native, wide);
  return e == cudaSuccess ? 0 : 1;
}

}  // namespace gsg
