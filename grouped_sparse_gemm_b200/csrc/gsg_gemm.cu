// gsg_gemm.cu -- persistent grouped NVFP4 expert GEMM on the Blackwell tensor cores.
//
// "Hardware-Native Joint Sparse-Quantization for Trillion-Scale Mixture-of-Experts"
// (paperlayer.ai summary): §3.4 (pp.5-6) -- grouped execution of routing-dependent expert
// problems in one launch using Blackwell sparse MMA, the sparse weight placed as operand A;
// §2 "Hardware opportunity" (p.3) -- paired 4:8 NVFP4 runs at twice the dense NVFP4 rate;
// §D.2 (p.19) -- a dense control that differs from the sparse kernel only in sparsity.
//
// One CTA per SM, 192 threads, warp-specialised:
//   warp 0      producer: per 256-wide K chunk, bulk copies of the pre-tiled weight values,
//               metadata and scales, one tensor-map TMA box of activation codes (128B swizzle)
//               and bulk copies of the activation scale atoms, into a ring of smem stages.
//   warp 1      TMEM owner and MMA issuer: tcgen05.cp metadata/scales into TMEM, then
//               tcgen05.mma(.sp) kind::mxf4nvf4 block_scale (M = 128 weight rows, N = token
//               tile, K = 128 logical sparse / 64 dense), accumulating in one of two TMEM
//               accumulators; tcgen05.commit releases smem stages and hands tiles to the epilogue.
//   warps 2..5  epilogue: tcgen05.ld accumulator lanes, multiply by s_x * s_w[e], store rows of Y.
// Tiles are (expert e, 128 weight rows nt, token tile mt) in e -> nt -> mt order; CTAs take
// tiles round-robin.  Experts with no rows produce no tiles.  Every mbarrier wait is bounded:
// on expiry the kernel records GSG_ERR_DEVICE_TIMEOUT, drains its own copies and MMAs, frees
// TMEM and returns.
#include <cuda.h>

#include "gsg_internal.cuh"

namespace gsg {

constexpr int kGemmThreads = 192;
constexpr int kMaxE = 1024;
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;   // 2 s
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColAcc1 = 128;
constexpr uint32_t kColMeta = 256;
constexpr uint32_t kColSFA = 272;
constexpr uint32_t kColSFB = 304;

struct GemmParams {
  const uint8_t* a_scales;
  const float* x_scale;
  const uint8_t* w_vals;
  const uint8_t* w_meta;
  const uint8_t* w_scales;
  const float* w_scale;
  const int32_t* off;
  void* Y;
  int* status;
  int E, N, K, R, BN, y_f32, rcap;
  int stages, stage_bytes;
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
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_cp_128x128b(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.128x128b [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ void tc_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ void tc_mma_sparse(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate, uint32_t sfa, uint32_t sfb, uint32_t meta) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.sp.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, [%7], %3, [%5], [%6], p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb), "r"(meta)
      : "memory");
}
__device__ __forceinline__ void tc_mma_dense(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate, uint32_t sfa, uint32_t sfb) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
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
// K-major A and B, M = 128, N = BN; bit 2 marks the sparse form (K = 128 logical).
__host__ __device__ inline uint32_t make_idesc(bool sparse, int BN) {
  return (sparse ? (1u << 2) : 0u) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((128u >> 4) << 24);
}

struct Ctl {
  int abort;
  uint32_t tmem_base;
};

// Bounded wait: true when the phase completed; false on timeout or when another role aborted.
__device__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0u) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
        *abort_flag = 1;
        set_status(status, GSG_ERR_DEVICE_TIMEOUT);
        return false;
      }
    }
  }
}

struct TileCoord {
  int e, nt, mt;
};

// Largest e with pref[e] <= t (pref[0] = 0, pref[E] = total tiles).
__device__ __forceinline__ TileCoord decode_tile(int t, const int* pref, const int* offs, int E, int NT, int BN) {
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (pref[mid] <= t) lo = mid; else hi = mid;
  }
  TileCoord c;
  c.e = lo;
  const int local = t - pref[lo];
  const int mte = (offs[lo + 1] - offs[lo] + BN - 1) / BN;
  c.nt = local / mte;
  c.mt = local % mte;
  (void)NT;
  return c;
}

template <bool kSparse>
__global__ void __launch_bounds__(kGemmThreads, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmap_b, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  constexpr int kKbLogical = kSparse ? 128 : 64;       // logical K per MMA
  constexpr int kKbPerStage = kChunkK / kKbLogical;    // MMAs per stage: 2 sparse, 4 dense
  constexpr int kABytes = kSparse ? 8192 : 16384;      // weight values per stage
  constexpr int kMetaBytes = kSparse ? 2048 : 0;
  constexpr int kSfBytes = kKbPerStage * 512;
  constexpr uint32_t kBStep = kSparse ? 64 : 32;       // B bytes per row consumed by one MMA

  const int BN = p.BN, E = p.E, NT = p.N / kTileN, KC = p.K / kChunkK;
  const int KBt = p.K / kKbLogical;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = p.stages;
  uint8_t* stage0 = base;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + (size_t)S * p.stage_bytes);
  // bars: full[S], empty[S], accf[2], acce[2], drain
  Ctl* ctl = reinterpret_cast<Ctl*>(bars + 2 * S + 5);
  int* offs = reinterpret_cast<int*>(ctl + 1);   // [E+1]
  int* pref = offs + (E + 1);                    // [E+1]
  volatile int* abort_flag = &ctl->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
  auto accf_bar = [&](int a) { return bar0 + 8u * (2 * S + a); };
  auto acce_bar = [&](int a) { return bar0 + 8u * (2 * S + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * S + 4);

  // ---- set-up: barriers, TMEM, tile schedule
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(accf_bar(a), 1);
      mbar_init(acce_bar(a), 4);
    }
    mbar_init(drain_bar, 1);
    ctl->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&ctl->tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // expert offsets (clamped to [0, R] and made monotone so a corrupt array can never send a
  // copy or a store out of bounds) and the per-expert tile prefix
  bool bad = false;
  for (int i = threadIdx.x; i <= E; i += blockDim.x) {
    int v = __ldg(p.off + i);
    if (v < 0 || v > p.R) { bad = true; v = v < 0 ? 0 : p.R; }
    offs[i] = v;
  }
  __syncthreads();
  {
    // chunked exclusive scan of tiles_e = ceil(rows_e / BN) * NT over E experts
    const int per = (E + kGemmThreads - 1) / kGemmThreads;
    const int e0 = threadIdx.x * per, e1 = min(e0 + per, E);
    int local = 0;
    for (int e = e0; e < e1; ++e) {
      int rows = offs[e + 1] - offs[e];
      if (rows < 0) { bad = true; rows = 0; }
      local += ((rows + BN - 1) / BN) * NT;
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    __shared__ int wsum[kGemmThreads / 32];
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    int run = before + incl - local;
    for (int e = e0; e < e1; ++e) {
      pref[e] = run;
      int rows = offs[e + 1] - offs[e];
      if (rows < 0) rows = 0;
      run += ((rows + BN - 1) / BN) * NT;
    }
    if (threadIdx.x == kGemmThreads - 1) pref[E] = before + incl;
  }
  if (bad) set_status(p.status, GSG_ERR_BAD_ROUTING);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // a decreasing offset makes that expert empty (its count is clamped to 0 above); keep the
  // row arithmetic below consistent with that
  const int total_tiles = pref[E];
  const uint32_t tmem = ctl->tmem_base;

  if (warp == 0) {
    // =============================== producer
    if (lane == 0) {
      const uint32_t tx_bytes = (uint32_t)(BN * 128 + kABytes + kMetaBytes + 2 * kSfBytes);
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int t = blockIdx.x; t < total_tiles && !*abort_flag; t += gridDim.x) {
        const TileCoord c = decode_tile(t, pref, offs, E, NT, BN);
        const int r0 = offs[c.e] + c.mt * BN;
        const size_t tile = (size_t)c.e * NT + c.nt;
        const uint8_t* av = p.w_vals + tile * KBt * 4096;
        const uint8_t* am = kSparse ? p.w_meta + tile * KC * 2048 : nullptr;
        const uint8_t* as = p.w_scales + tile * KBt * 512;
        bool ok = true;
        for (int kc = 0; kc < KC; ++kc) {
          if (!wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, p.status)) { ok = false; break; }
          uint8_t* sb = stage0 + (size_t)stage * p.stage_bytes;
          const uint32_t sB = smem_u32(sb);
          const uint32_t sA = sB + BN * 128;
          const uint32_t sM = sA + kABytes;
          const uint32_t sSFA = sM + kMetaBytes;
          const uint32_t sSFB = sSFA + kSfBytes;
          const uint32_t fb = full_bar(stage);
          mbar_arrive_expect_tx(fb, tx_bytes);
          bulk_g2s(sA, av + (size_t)kc * kABytes, kABytes, fb);
          if (kSparse) bulk_g2s(sM, am + (size_t)kc * 2048, 2048, fb);
          bulk_g2s(sSFA, as + (size_t)kc * kSfBytes, kSfBytes, fb);
          tma_load_2d(sB, &tmap_b, kc * 128, r0, fb);
#pragma unroll
          for (int h = 0; h < kKbPerStage; ++h) {
            const size_t kb = (size_t)kc * kKbPerStage + h;
            bulk_g2s(sSFB + h * 512, p.a_scales + (kb * p.rcap + r0) * 16, 512, fb);
          }
          ++issued;
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      if (*abort_flag) {
        // drain: wait for the copies this thread issued into the last min(S, issued) stages
        int s = stage;
        uint32_t ph = phase;
        for (int i = 0; i < S && i < issued; ++i) {
          if (--s < 0) { s = S - 1; ph ^= 1u; }
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(full_bar(s), ph) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // =============================== MMA issuer
    if (lane == 0) {
      const uint32_t idesc = make_idesc(kSparse, BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool any = false;
      for (int t = blockIdx.x; t < total_tiles && !*abort_flag; t += gridDim.x) {
        if (!wait_bounded(acce_bar(acc), acc_phase ^ 1u, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (acc ? kColAcc1 : 0u);
        bool ok = true;
        for (int kc = 0; kc < KC; ++kc) {
          if (!wait_bounded(full_bar(stage), phase, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sB = smem_u32(stage0 + (size_t)stage * p.stage_bytes);
          const uint32_t sA = sB + BN * 128;
          const uint32_t sM = sA + kABytes;
          const uint32_t sSFA = sM + kMetaBytes;
          const uint32_t sSFB = sSFA + kSfBytes;
          if (kSparse) tc_cp_128x128b(tmem + kColMeta, smem_desc(sM, 128, 128, 0));
#pragma unroll
          for (int h = 0; h < kKbPerStage; ++h) {
            tc_cp_32x128b_x4(tmem + kColSFA + 4 * h, smem_desc(sSFA + 512 * h, 128, 128, 0));
            tc_cp_32x128b_x4(tmem + kColSFB + 4 * h, smem_desc(sSFB + 512 * h, 128, 128, 0));
          }
#pragma unroll
          for (int h = 0; h < kKbPerStage; ++h) {
            const uint64_t adesc = smem_desc(sA + 4096u * h, 128, 256, 0);
            const uint64_t bdesc = smem_desc(sB + kBStep * h, 16, 1024, 2);
            const uint32_t accum = (kc | h) != 0 ? 1u : 0u;
            if (kSparse)
              tc_mma_sparse(d_tmem, adesc, bdesc, idesc, accum, tmem + kColSFA + 4 * h, tmem + kColSFB + 4 * h,
                            tmem + kColMeta + 2 * h);
            else
              tc_mma_dense(d_tmem, adesc, bdesc, idesc, accum, tmem + kColSFA + 4 * h, tmem + kColSFB + 4 * h);
          }
          tc_commit(empty_bar(stage));
          any = true;
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(accf_bar(acc));
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (any) {
        // all MMAs issued by this thread have completed once the drain barrier fires
        tc_commit(drain_bar);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(drain_bar, 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
        }
      }
    }
  } else {
    // =============================== epilogue (warps 2..5 -> TMEM lane quadrants 2,3,0,1)
    const int q = warp & 3;
    const int row = 32 * q + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    const float sx = __ldg(p.x_scale);
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
      const TileCoord c = decode_tile(t, pref, offs, E, NT, BN);
      const int r0 = offs[c.e] + c.mt * BN;
      const int valid = min(BN, offs[c.e + 1] - r0);
      if (!wait_bounded(accf_bar(acc), acc_phase, abort_flag, p.status)) break;
      tc_fence_after();
      const float scale = __fmul_rn(sx, __ldg(p.w_scale + c.e));
      const int n = c.nt * kTileN + row;
      const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + (acc ? kColAcc1 : 0u);
      for (int c0 = 0; c0 < BN; c0 += 16) {
        if (c0 >= valid) break;
        float v[16];
        tc_ld_16(taddr + c0, v);
        if (p.y_f32) {
          float* Y = static_cast<float*>(p.Y);
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c0 + j < valid) Y[(size_t)(r0 + c0 + j) * p.N + n] = __fmul_rn(v[j], scale);
        } else {
          __nv_bfloat16* Y = static_cast<__nv_bfloat16*>(p.Y);
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c0 + j < valid) Y[(size_t)(r0 + c0 + j) * p.N + n] = __float2bfloat16_rn(__fmul_rn(v[j], scale));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce_bar(acc));
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// ------------------------------------------------------------------ host side
int gemm_stage_bytes(bool sparse, int BN) {
  const int a = sparse ? 8192 : 16384, m = sparse ? 2048 : 0, sf = (sparse ? 2 : 4) * 512;
  const int b = BN * 128 + a + m + 2 * sf;
  return (b + 1023) / 1024 * 1024;
}

int gemm_pick_bn(int max_rows) {
  if (max_rows <= 0) return 128;
  if (max_rows <= 16) return 16;
  if (max_rows <= 32) return 32;
  if (max_rows <= 64) return 64;
  return 128;
}

constexpr int kSmemBudget = 200 * 1024;

int gemm_stages(bool sparse, int BN) {
  int s = kSmemBudget / gemm_stage_bytes(sparse, BN);
  if (s > 16) s = 16;
  return s;
}

size_t gemm_smem_bytes(bool sparse, int BN, int E) {
  const int S = gemm_stages(sparse, BN);
  return 1024 + (size_t)S * gemm_stage_bytes(sparse, BN) + (2 * S + 5) * 8 + sizeof(Ctl) + (size_t)2 * (E + 1) * 4;
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

cudaError_t gemm_set_smem_attrs() {
  int maxb = 0;
  for (int bn = 16; bn <= 128; bn *= 2) {
    const int a = (int)gemm_smem_bytes(true, bn, kMaxE), b = (int)gemm_smem_bytes(false, bn, kMaxE);
    if (a > maxb) maxb = a;
    if (b > maxb) maxb = b;
  }
  cudaError_t e1 = cudaFuncSetAttribute(grouped_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, maxb);
  cudaError_t e2 = cudaFuncSetAttribute(grouped_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, maxb);
  return e1 != cudaSuccess ? e1 : e2;
}

// returns 0 ok, 1 cuda error, 2 tensor map failure
int launch_gemm(bool sparse, const uint8_t* a_codes, const uint8_t* a_scales, const float* x_scale,
                const uint8_t* w_vals, const uint8_t* w_meta, const uint8_t* w_scales, const float* w_scale,
                const int32_t* off, int E, int N, int K, int R, int max_rows, void* Y, int y_f32, int* status,
                int num_sms, cudaStream_t stream) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr) return 2;
  const int BN = gemm_pick_bn(max_rows);
  CUtensorMap tmap;
  cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)R};
  cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
  cuuint32_t box[2] = {128u, (cuuint32_t)BN};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult cr = enc(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(a_codes), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return 2;
  GemmParams p;
  p.a_scales = a_scales; p.x_scale = x_scale; p.w_vals = w_vals; p.w_meta = w_meta; p.w_scales = w_scales;
  p.w_scale = w_scale; p.off = off; p.Y = Y; p.status = status;
  p.E = E; p.N = N; p.K = K; p.R = R; p.BN = BN; p.y_f32 = y_f32; p.rcap = R + kActScalePadRows;
  p.stages = gemm_stages(sparse, BN);
  p.stage_bytes = gemm_stage_bytes(sparse, BN);
  const size_t smem = gemm_smem_bytes(sparse, BN, E);
  if (sparse)
    grouped_gemm_kernel<true><<<num_sms, kGemmThreads, smem, stream>>>(tmap, p);
  else
    grouped_gemm_kernel<false><<<num_sms, kGemmThreads, smem, stream>>>(tmap, p);
  return cudaGetLastError() == cudaSuccess ? 0 : 1;
}

}  // namespace gsg
