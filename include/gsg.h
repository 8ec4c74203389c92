/*
 * gsg.h -- C ABI of the grouped sparse-NVFP4 expert GEMM library (libgsg.so).
 *
 * The operation is the routed Mixture-of-Experts expert projection described in
 * "Hardware-Native Joint Sparse-Quantization for Trillion-Scale Mixture-of-Experts"
 * (paperlayer.ai summary page): for every expert e, Y_e = X_e . W_e^T over the rows
 * routed to e, with W_e stored as paired 4:8 NVFP4 (App. A "Blackwell paired 4:8 NVFP4",
 * p.14; "Storage layout", p.15), activations quantized to NVFP4 with 32-element scale
 * blocks and fused with dispatch (§D.1, p.19), all experts executed in one grouped launch
 * with the sparse weight as MMA operand A (§3.4, pp.5-6).
 *
 * Conventions for every call
 *   - Pointers are DEVICE pointers owned by the caller unless stated otherwise.  The library
 *     allocates nothing; calls that need scratch take a caller workspace (size from
 *     gsg_workspace_size).  `stream` is a cudaStream_t (NULL = legacy default stream).
 *   - Calls are asynchronous on `stream`.  Errors the host can detect (bad sizes, NULL
 *     pointers, small workspace) return at once without launching anything.  Errors found
 *     on the device (expert id out of range, non-finite input, a bounded wait that timed
 *     out) set a sticky per-device status word (first error wins); read and clear it with
 *     gsg_get_device_status.  Outputs of a call that raised a device error are unspecified.
 *   - Shapes: K % 256 == 0, N % 128 == 0, E >= 1.  bf16 tensors are passed as uint16_t bit
 *     patterns.  Multi-dimensional buffers are dense, last index fastest.
 *   - Re-entrant across streams; the only global state is the device status word (and the
 *     fixed scratch of gsg_moe_route_permute_noalloc, described there).
 *
 * Packed weight layout (one buffer, tile-major, the order the GEMM streams it): for expert e,
 * n-tile nt (128 output rows, NT = N/128) and 256-wide K chunk kc, one contiguous chunk block
 * at ((e*NT + nt)*(K/256) + kc) * CB holding, for the chunk's MMA k-blocks h (64 stored 4-bit
 * values per row each: 128 logical K sparse, 64 dense):
 *   values  h*4096 + (r/8)*256 + (c/16)*128 + (r%8)*16 + c%16 for row r (0..127) and byte
 *           c = v/2 of stored value v (0..63) of the k-block, low nibble = even v.  Sparse: the
 *           four retained E2M1 codes of each 8-group in K order; dense: every code.
 *   meta    (sparse) 8192 + r*16 + g/2 for 8-group g (0..31) of the chunk, low nibble = even g;
 *           nibble = i0 | i1 << 2 (the kept pairs, i0 < i1).
 *   scales  V + h*512 + 16*(r%32) + 4*(r/32) + j for block j (0..3) of k-block h: UE4M3 codes,
 *           one per 32 logical weights (sparse) or 16 (dense).
 * Sparse: CB = 11264, V = 10240 (2 k-blocks, 2.75 bit/weight).  Dense: CB = 18432, V = 16384
 * (4 k-blocks, 4.5 bit/weight).
 * Activation layouts (R routed rows; KBa = K/(4*sf)):
 *   codes  [R][K/2]  row-major E2M1, low nibble = even k.
 *   scales [KBa][R + 256][4][4 B]: entry (kb, r, c, j) = UE4M3 scale of block 4*kb + j of
 *          row r + 32*c (0 when r + 32*c >= R).  Each scale is stored four times so that the
 *          GEMM fetches the scale tile of ANY starting row with one contiguous copy.
 */
#ifndef GSG_H
#define GSG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GSG_OK = 0,
  GSG_ERR_INVALID_ARG = -1,       /* NULL pointer, negative size, bad enum value            */
  GSG_ERR_UNSUPPORTED_SHAPE = -2, /* K % 256, N % 128, sizes beyond the library's limits      */
  GSG_ERR_CUDA = -3,              /* a CUDA runtime call or a launch failed                   */
  GSG_ERR_BAD_ROUTING = -4,       /* device: expert id outside [0, E), or inconsistent offsets */
  GSG_ERR_NONFINITE = -5,         /* device: NaN/Inf in a tensor that is being quantized      */
  GSG_ERR_DEVICE_TIMEOUT = -6,    /* device: a bounded wait inside a kernel gave up           */
  GSG_ERR_WORKSPACE = -7          /* workspace NULL or smaller than gsg_workspace_size()      */
} gsg_status_t;

/* Operation ids for gsg_workspace_size. */
enum {
  GSG_OP_PACK_SPARSE = 1,
  GSG_OP_PACK_DENSE = 2,
  GSG_OP_ROUTE = 3,
  GSG_OP_QUANTIZE = 4,
  GSG_OP_GEMM = 5,
  GSG_OP_COMBINE = 6,   /* gsg_grouped_sparse_gemm_combine: token slots + barrier counters    */
  GSG_OP_DISPATCH = 7   /* gsg_moe_dispatch_nvfp4: routing workspace + quantizer workspace    */
};

/* Output element types of the grouped GEMMs. */
enum { GSG_OUT_BF16 = 0, GSG_OUT_F32 = 1 };

/* ----------------------------------------------------------------------------------------
 * Buffer sizes in bytes (host-only arithmetic, no GPU access).
 */
size_t gsg_sparse_packed_bytes(int E, int N, int K);          /* E*N*K*11/32 (2.75 bit)     */
size_t gsg_dense_packed_bytes(int E, int N, int K);           /* E*N*K*9/16 (4.5 bit)       */
size_t gsg_act_codes_bytes(int R, int K);                     /* R*K/2                      */
size_t gsg_act_scales_bytes(int R, int K, int sf_block);      /* K/(4 sf) * (R+256) * 16    */
/* Workspace needed by `op` (0 when none).  T = tokens, k = experts per token. */
size_t gsg_workspace_size(int op, int E, int N, int K, int T, int k);

/* ----------------------------------------------------------------------------------------
 * gsg_pack_sparse_nvfp4 -- weight packer (offline).
 * Paper: App. A "Blackwell paired 4:8 NVFP4" (p.14) and "Storage layout" (p.15); §3.4 (p.5).
 * W fp32 [E][N][K] (K contiguous).  Per 8-group of K the two adjacent pairs with the largest
 * energy w0*w0 + w1*w1 (fp32, ties -> lower pair) are kept; s_w[e] = amax(kept W_e)/2688
 * (1 if 0); per 32-block b: sc = UE4M3(b / (6 s_w)), codes = E2M1(w / (dec(sc) s_w)),
 * round-to-nearest-even with saturation.  Writes the packed layout above (w_packed, size
 * gsg_sparse_packed_bytes) and w_tensor_scale fp32 [E].  Non-finite W sets GSG_ERR_NONFINITE.
 */
gsg_status_t gsg_pack_sparse_nvfp4(const float* W, int E, int N, int K, uint8_t* w_packed,
                                   float* w_tensor_scale,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* gsg_pack_dense_nvfp4 -- dense NVFP4 packer for the in-repo control GEMM (16-element
 * blocks, the block size the dense block-scaled MMA takes; §D.2, p.19: the control differs
 * from the sparse kernel only in sparsity).  Packed layout above, size gsg_dense_packed_bytes. */
gsg_status_t gsg_pack_dense_nvfp4(const float* W, int E, int N, int K, uint8_t* w_packed,
                                  float* w_tensor_scale,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* ----------------------------------------------------------------------------------------
 * gsg_moe_route_permute -- group routed rows by expert.
 * Paper: §2 "Execution gap" (p.3): routing-dependent expert products with different token
 * counts run together; §D.1 (p.19): dispatch.  topk_ids int32 [T][k] in [0, E).
 * Routed pair (t, j) has flat index f = t*k + j.  Rows of expert e are [off[e], off[e+1]),
 * in ascending f.  Outputs: expert_offsets int32 [E+1], perm_src int32 [R] (row -> f),
 * inv_perm int32 [R] (f -> row).  Out-of-range ids set GSG_ERR_BAD_ROUTING: such a pair gets
 * no row and inv_perm[f] = -1 (the quantizer and the scatter skip it); the offsets and the rows of
 * the valid pairs are then unspecified.  Deterministic.
 */
gsg_status_t gsg_moe_route_permute(const int32_t* topk_ids, int T, int k, int E,
                                   int32_t* expert_offsets, int32_t* perm_src, int32_t* inv_perm,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* ----------------------------------------------------------------------------------------
 * gsg_quantize_act_nvfp4 -- NVFP4 activation quantizer fused with dispatch.
 * Paper: §D.1 (p.19): activation quantization forms 32-element scale blocks and is fused
 * with dispatch; §3.4 (pp.5-6): corresponding scale blocks for weights and activations.
 * X bf16 [T][K].  s_x = max|X|/2688 (1 if 0), or *x_tensor_scale_in when that is non-NULL.
 * Each token row is quantized once (per sf_block block: UE4M3 scale + E2M1 codes, same rule
 * as the weights) and written to each of its k routed rows inv_perm[t*k + j]
 * (inv_perm NULL: row t, and k must be 1).  sf_block: 32 (sparse GEMM) or 16 (dense control).
 * Outputs: codes [R][K/2], scales in the quad layout above (R = T*k), x_tensor_scale_out fp32[1].
 * Limits: T*k <= 2^30 and T*K/8 < 2^31, else GSG_ERR_UNSUPPORTED_SHAPE.
 * workspace: gsg_workspace_size(GSG_OP_QUANTIZE, 0, 0, K, T, k) bytes, 16-byte aligned, needed
 * when s_x is computed (the partial maxima) and, for sf_block 32, once R*K >= 2^27: there the
 * scale words are first written row-major to the workspace and a second launch rearranges
 * them into the quad layout (scattered 4-byte quad writes cost DRAM read-modify-writes at
 * that size).  The result is the same either way.  Otherwise it may be NULL.
 */
gsg_status_t gsg_quantize_act_nvfp4(const uint16_t* X, int T, int K, int sf_block,
                                    const int32_t* inv_perm, int k,
                                    const float* x_tensor_scale_in,
                                    uint8_t* codes, uint8_t* scales, float* x_tensor_scale_out,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* ----------------------------------------------------------------------------------------
 * gsg_moe_dispatch_nvfp4 -- routing and the activation quantizer in one call.
 * Paper: §D.1 (p.19): dispatch fused with activation quantization ahead of the first expert
 * GEMM; §2 "Execution gap" (p.3): grouped expert problems.
 * Computes exactly what gsg_moe_route_permute(topk_ids, T, k, E, ...) followed by
 * gsg_quantize_act_nvfp4(X, T, K, sf_block, inv_perm, k, x_tensor_scale_in, ...) compute, bit
 * for bit, with the same arguments, outputs, limits and errors as the two.  The difference is
 * the launches: the quantizer's max|X| pass runs inside the routing's first launch (extra
 * blocks beside the routing blocks; both only read their inputs), so the pair takes one launch
 * fewer.  workspace: gsg_workspace_size(GSG_OP_DISPATCH, E, 0, K, T, k) bytes, 16-byte aligned.
 */
gsg_status_t gsg_moe_dispatch_nvfp4(const int32_t* topk_ids, const uint16_t* X, int T, int k, int E, int K,
                                    int sf_block, const float* x_tensor_scale_in,
                                    int32_t* expert_offsets, int32_t* perm_src, int32_t* inv_perm,
                                    uint8_t* codes, uint8_t* scales, float* x_tensor_scale_out,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* ----------------------------------------------------------------------------------------
 * gsg_grouped_sparse_gemm -- the grouped paired-4:8 NVFP4 expert GEMM.
 * Paper: §3.4 (pp.5-6): Blackwell sparse MMA with grouped scheduling, one launch, the sparse
 * weight as operand A; §2 (p.3): the sparse NVFP4 path peaks at 2x dense NVFP4.
 * For each expert e and routed row r in [off[e], off[e+1]):
 *     Y[r][n] = s_x * s_w[e] * sum_k a[r][k] * w[e][n][k]      (fp32 accumulation)
 * a_codes/a_scales from gsg_quantize_act_nvfp4 (sf_block 32); w_packed and w_tensor_scale from
 * gsg_pack_sparse_nvfp4.
 * expert_offsets int32 [E+1], monotone, off[0] = 0, off[E] <= R.  max_rows_per_expert is a
 * host-side hint that picks the token tile and the tile schedule (<= 0: unknown); any value
 * gives a correct result, a wrong one only a slower launch.  Y [R][N] bf16 (y_dtype
 * GSG_OUT_BF16) or fp32 (GSG_OUT_F32); rows >= off[E] are not written.  No workspace.
 * Persistent kernel, one CTA per SM: TMA/bulk copies into a shared-memory ring, tcgen05
 * block-scaled sparse MMA into TMEM, epilogue applies s_x*s_w[e].
 */
gsg_status_t gsg_grouped_sparse_gemm(const uint8_t* a_codes, const uint8_t* a_scales,
                                     const float* x_tensor_scale,
                                     const uint8_t* w_packed, const float* w_tensor_scale,
                                     const int32_t* expert_offsets, int E, int N, int K, int R,
                                     int max_rows_per_expert, void* Y, int y_dtype, void* stream);

/* gsg_grouped_dense_gemm -- the dense-NVFP4 control on the same skeleton (non-sparse MMA,
 * 16-element blocks).  a_* from gsg_quantize_act_nvfp4 with sf_block 16; w_* from
 * gsg_pack_dense_nvfp4.  Same semantics as gsg_grouped_sparse_gemm. */
gsg_status_t gsg_grouped_dense_gemm(const uint8_t* a_codes, const uint8_t* a_scales,
                                    const float* x_tensor_scale,
                                    const uint8_t* w_packed, const float* w_tensor_scale,
                                    const int32_t* expert_offsets, int E, int N, int K, int R,
                                    int max_rows_per_expert, void* Y, int y_dtype, void* stream);

/* gsg_grouped_dense_gemm_native -- the same dense control in the activation-stationary ("native")
 * orientation of the paper's kernel benchmark (§D.2, p.19, Figure 5: CUTLASS dense NVFP4 "native"
 * and "transposed").  Each tile's 128 token rows are MMA operand A and the weight n-tile is
 * operand B; gsg_grouped_dense_gemm (and the sparse kernel) put the weights in A and the tokens in
 * B ("transposed").  Same arguments, result and errors as gsg_grouped_dense_gemm; every token tile
 * is 128 rows (MMA M), padded when an expert has fewer routed rows. */
gsg_status_t gsg_grouped_dense_gemm_native(const uint8_t* a_codes, const uint8_t* a_scales,
                                           const float* x_tensor_scale,
                                           const uint8_t* w_packed, const float* w_tensor_scale,
                                           const int32_t* expert_offsets, int E, int N, int K, int R,
                                           int max_rows_per_expert, void* Y, int y_dtype, void* stream);

/* gsg_grouped_sparse_gemm_swiglu -- the up-projection with SwiGLU output preparation fused into
 * the epilogue, producing the down-projection's NVFP4 input directly.
 * Paper: §D.1 (p.19): the serving integration fuses SwiGLU output preparation for the second
 * expert GEMM; §3.4 (pp.5-6) and App. A: the NVFP4 block rule.
 * The weights are one fused [N2][K] matrix per expert, gate rows [0, I) then up rows [I, 2I)
 * (I = N2/2), packed with gsg_pack_sparse_nvfp4 as usual (one s_w[e] for both halves).  With
 * y[r][n] = s_x * s_w[e] * sum_k a[r][k] * w[e][n][k] (fp32, never rounded to bf16):
 *     h[r][f] = silu(y[r][f]) * y[r][I + f],  silu(x) = x / (1 + exp(-x)),   f < I
 * then h is quantized like the activations (32-element blocks along f, UE4M3 scale, E2M1 codes)
 * with the caller's tensor scale *h_tensor_scale (a calibrated value; the dynamic amax of h
 * would need a pass over all of h before any block could be encoded):
 *     h_codes  [R][I/2]  (low nibble = even f)
 *     h_scales the quad layout above for K = I (gsg_act_scales_bytes(R, I, 32) bytes)
 * i.e. exactly what gsg_grouped_sparse_gemm takes as a_codes / a_scales for the down-projection
 * over the same expert_offsets (with x_tensor_scale = h_tensor_scale).  N2 % 256 == 0; rows >=
 * off[E] are not written (their scale entries are zero).  silu is evaluated in fp32 with the
 * fast exponential and division (a few ulp), so h is not reproducible bit for bit by a CPU;
 * parity is checked against the exact h within the GEMM tolerance plus one quantization step.
 * Token tiles are at most 64 rows (two accumulators per tile).  No workspace.
 */
gsg_status_t gsg_grouped_sparse_gemm_swiglu(const uint8_t* a_codes, const uint8_t* a_scales,
                                            const float* x_tensor_scale,
                                            const uint8_t* w_packed, const float* w_tensor_scale,
                                            const int32_t* expert_offsets, int E, int N2, int K, int R,
                                            int max_rows_per_expert, const float* h_tensor_scale,
                                            uint8_t* h_codes, uint8_t* h_scales, void* stream);

/* gsg_grouped_sparse_gemm_combine -- the down-projection with the gate-weighted combine fused
 * into the epilogue: gsg_grouped_sparse_gemm (bf16 Y) followed by gsg_unpermute_scale, in one
 * launch, with the same result bit for bit.
 * Paper: §D.1 (p.19): the serving integration fuses dispatch and scatter into the expert GEMMs.
 * Every routed row is written (bf16, as Y would hold it) to its token slot f = t*k + j of the
 * workspace instead of row r; once every CTA of the launch has written its rows (a bounded grid
 * barrier on two of the workspace's counters), the CTAs compute
 *     out[t][n] = bf16_rne( sum_{j<k} fp32(gates[t][j] * slot[t*k + j][n]) )   (j ascending, from 0)
 * -- the scatter's arithmetic and order.  R = T*k routed rows; perm_src int32 [R] and
 * expert_offsets from gsg_moe_route_permute; gates fp32 [T][k]; out bf16 [T][N] (T*N/8 < 2^31,
 * else GSG_ERR_UNSUPPORTED_SHAPE).  A routed row whose perm_src entry lies outside [0, T*k) is
 * skipped (nothing stored for it) and sets GSG_ERR_BAD_ROUTING.
 * workspace: gsg_workspace_size(GSG_OP_COMBINE, E, N, K, T, k) bytes, 16-byte aligned: the slots
 * bf16 [T*k][N] and then int32 counters [T][N/32] (the first two count the CTAs through the grid
 * barrier).  The counters must be zero before the first call (e.g. allocate the workspace zeroed);
 * every call that completes leaves them zero again, so a workspace can be reused call after call.
 * After a device error the outputs and the counters are unspecified: zero the workspace again.
 * Calls that share a workspace must not run concurrently.  The launch's CTAs (one per SM) wait
 * for one another at the barrier: while another kernel keeps SMs busy on a concurrent stream, the
 * CTAs already running wait for the rest, and a wait longer than 2 s ends with
 * GSG_ERR_DEVICE_TIMEOUT (outputs unspecified) instead of hanging.
 */
gsg_status_t gsg_grouped_sparse_gemm_combine(const uint8_t* a_codes, const uint8_t* a_scales,
                                             const float* x_tensor_scale,
                                             const uint8_t* w_packed, const float* w_tensor_scale,
                                             const int32_t* expert_offsets, int E, int N, int K, int T, int k,
                                             int max_rows_per_expert, const int32_t* perm_src,
                                             const float* gates, void* workspace, size_t workspace_bytes,
                                             uint16_t* out, void* stream);

/* ----------------------------------------------------------------------------------------
 * gsg_unpermute_scale -- gate-weighted scatter back to tokens.
 * Paper: §D.1 (p.19): scatter after the expert GEMM.
 *     out[t][n] = bf16_rne( sum_{j<k} fp32(gates[t][j] * Y[inv_perm[t*k+j]][n]) )
 * fp32 products and running sum (starting at 0), j ascending.  Y bf16 [R][N],
 * gates fp32 [T][k], out bf16 [T][N].  N % 8 == 0; T*k <= 2^30 and T*N/8 < 2^31, else
 * GSG_ERR_UNSUPPORTED_SHAPE.
 */
gsg_status_t gsg_unpermute_scale(const uint16_t* Y, const int32_t* inv_perm, const float* gates,
                                 int T, int k, int N, uint16_t* out, void* stream);

/* ----------------------------------------------------------------------------------------
 * gsg_moe_route_permute_noalloc -- gsg_moe_route_permute for callers that cannot allocate.
 * The paper has no counterpart: this is a library convenience, not a step of the method.
 * Who needs it: code that may not call cudaMalloc or any allocating routine when it routes
 * tokens (its device memory is owned and pre-carved by another component, or it must not grow
 * its footprint after start-up), so it cannot supply the routing workspace.  Same inputs,
 * outputs, result and errors as gsg_moe_route_permute; the workspace is replaced by a fixed
 * 256 KiB device array inside the library, which every GPU that loads the library holds until
 * the process exits.  The call allocates nothing.
 * Limit: R = T*k <= 2048 needs no scratch; above that ceil(R/8192) * E <= 32768
 * (E = 384: R <= 696,320; E = 128: R <= 2,097,152), else GSG_ERR_UNSUPPORTED_SHAPE with no
 * launch.  The first call on a device sets up that device (the library's per-device set-up and
 * the scratch's device address); make that first call before any stream capture begins.
 * All calls on a device share the one array and it keeps the last call's contents (nothing in
 * it needs to start at zero); calls whose launches overlap on the GPU (unordered streams) race
 * on it and must be serialised by the caller.
 */
gsg_status_t gsg_moe_route_permute_noalloc(const int32_t* topk_ids, int T, int k, int E,
                                           int32_t* expert_offsets, int32_t* perm_src,
                                           int32_t* inv_perm, void* stream);

/* ----------------------------------------------------------------------------------------
 * gsg_test_set_gemm_stall_ns -- fault injection for tests of the device timeout path.  Not a step
 * of the method: the paper has no counterpart.  ns > 0: every grouped GEMM launched afterwards
 * (sparse, dense control, SwiGLU and combine epilogues) makes its MMA warp wait up to `ns`
 * nanoseconds, before its second tile (its first if it has one), on an internal barrier that
 * nothing arrives on.  The wait runs out; the launch sets GSG_ERR_DEVICE_TIMEOUT, waits for its
 * own copies and tensor-core work, frees its tensor memory and returns, with its outputs
 * unspecified -- exactly what happens when a real wait exceeds its 2 s limit.  ns = 0 (the
 * default) switches the hook off.  Process-wide: set it only while no other thread launches.
 */
void gsg_test_set_gemm_stall_ns(unsigned long long ns);

/* ----------------------------------------------------------------------------------------
 * gsg_test_set_gemm_table_cap -- test hook for the grouped GEMM's tile bookkeeping.  Not a step of
 * the method.  Every CTA of a grouped GEMM decodes the list of its tiles (expert, n-tile, token
 * rows) from the expert offsets once, into a table in shared memory; a CTA with more tiles than
 * the table holds decodes the rest as it reaches them.  tiles >= 0: launches afterwards keep at
 * most `tiles` table entries, so that path runs at any size (results are bit-identical); -1 (the
 * default) switches the hook off.  Process-wide: set it only while no other thread launches.
 */
void gsg_test_set_gemm_table_cap(int tiles);

/* ----------------------------------------------------------------------------------------
 * Status.  gsg_get_device_status synchronizes `stream`, returns the device status word of the
 * current device and clears it.  gsg_status_string never returns NULL.
 */
gsg_status_t gsg_get_device_status(void* stream);
const char* gsg_status_string(gsg_status_t status);
int gsg_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GSG_H */
