/*
 * mxfp8.h -- C ABI of the B200 (sm_100a) MXFP8 quantisers and the dropless
 * grouped GEMM of a Mixture-of-Experts expert layer.
 *
 * What is computed
 *   MXFP8: every block of 32 consecutive elements shares one power-of-two
 *   scale (opensourcebeat.com, "Enabling up to 41% faster pre-training: MXFP8
 *   and DeepEP for DeepSeek-V3 on B200 with TorchTitan", FAQ "What is
 *   MXFP8?"; the same page, section "Двухсторонняя атака", says Blackwell's
 *   5th-generation tensor cores run it natively).  The block rules are OCP MX
 *   v1.0: the E8M0 scale byte is s + 127 with s = floor(log2(amax)) - 8
 *   clamped to [-127, 127] (amax = 0 gives byte 0x00); each element becomes
 *   the E4M3 code of x * 2^-s, rounded to nearest even and saturated to
 *   +-448; the sign survives on zero.  A block with a non-finite element is
 *   outside the contract and gets scale 0xFF and codes 0x7F.
 *
 *   Grouped GEMM: all experts run in one launch, each on its real token count,
 *   with no padding to a capacity and no dropped tokens (iitak.ru, "NVIDIA
 *   в 10 раз ускорила обучение моделей-«смесей экспертов» на JAX", paragraphs
 *   on dropless routing and the Transformer Engine grouped GEMM; the two
 *   all-to-alls around it are on opensourcebeat.com, section "Двухсторонняя
 *   атака").  For expert e owning rows offs[e] .. offs[e+1]-1:
 *     forward  Y_e  = X_e  W_e^T     Y  [M, N]
 *     dgrad    dX_e = dY_e W_e       dX [M, K]
 *     wgrad    dW_e = dY_e^T X_e     dW [E, N, K]  (zero when m_e = 0)
 *   Products of dequantised operands are accumulated in fp32 (tensor memory)
 *   and written as bf16 (round to nearest even).
 *
 * Conventions
 *   - Every pointer except the `stream` is a DEVICE pointer owned by the
 *     caller; the library allocates nothing and keeps no pointer after a call.
 *   - bf16 data is passed as its uint16 bit pattern.  All matrices are
 *     row-major.  Data and scale pointers must be 16-byte aligned.
 *   - `d_offs` is an int32 device array of num_groups + 1 exclusive prefix
 *     offsets: d_offs[0] = 0, non-decreasing, d_offs[num_groups] = rows.  A
 *     NULL `d_offs` means one group holding every row.  The quantisers never
 *     read or write out of bounds for any offsets (they clamp them); the GEMMs
 *     check them on the device and report MXF8_ERR_BAD_OFFSETS through the
 *     workspace status without touching the output.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls are
 *     asynchronous: a return of MXF8_OK means the launch was accepted.
 *   - Only sm_100 devices (B200/GB200) are supported.
 *
 * Layouts (shared by the quantisers' outputs and the GEMMs' inputs)
 *   Scale atoms: scales are stored in 512-byte atoms covering 128 rows x 4
 *   32-blocks; atom (rb, cb) starts at byte 512*(rb*pitch + cb) and logical
 *   scale (row, blk) sits at byte (row%32)*16 + ((row%128)/32)*4 + blk%4 inside
 *   it.  This is the scale-factor layout tcgen05 block-scaled MMA reads from
 *   tensor memory after a 32x128-bit copy; pad bytes inside a written atom
 *   are 0x00.
 *   Rowwise (blocks along the last dimension): codes keep the [rows, cols]
 *   layout; scale rows of group g start at a multiple of 128 (padded row
 *   128*RB_g + t for row d_offs[g] + t, RB_g = sum over h < g of
 *   ceil(m_h/128)); pitch = ceil(cols/128).
 *   Colwise (blocks along rows, restarting at every group offset; a short
 *   last block covers the real rows only): codes are transposed, qT[c, P_g + t]
 *   holds element (d_offs[g] + t, c) with P_g = sum over h < g of
 *   round_up(m_h, 32), and the pad columns up to round_up(m_g, 32) are 0x00;
 *   the row stride is ldT = mxfp8_colwise_ld(rows, num_groups).  The scales
 *   form the matrix S^T[c, 4*RB_g + t/32] with pitch
 *   mxfp8_colwise_pitch(rows, num_groups).  Every GEMM operand is then K-major.
 */
#ifndef MXFP8_H
#define MXFP8_H

#include <stdint.h>

/* Symbols of the shared library are exported explicitly (it is built with
 * hidden visibility). */
#if defined(__GNUC__)
#define MXF8_API __attribute__((visibility("default")))
#else
#define MXF8_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MXF8_OK = 0,
    MXF8_ERR_INVALID_ARG = 1,  /* null pointer, bad size, buffer too small, too many groups */
    MXF8_ERR_ALIGNMENT = 2,    /* a pointer is not 16-byte aligned */
    MXF8_ERR_UNSUPPORTED = 3,  /* the current device is not sm_100 */
    MXF8_ERR_CUDA = 4,         /* a CUDA call failed; see mxfp8_last_cuda_error() */
    MXF8_ERR_BAD_OFFSETS = 5,  /* device side: d_offs is not a valid prefix of `rows` */
    MXF8_ERR_TIMEOUT = 6,      /* device side: a pipeline wait ran past its limit (2 s); tests provoke it
                                  with mxfp8_testing_stall_first_stage */
    MXF8_ERR_BAD_ROUTING = 7   /* device side: an expert id outside [0, num_experts) */
} mxf8_status;

/* Largest num_groups (experts) a grouped GEMM accepts. */
#define MXF8_GEMM_MAX_GROUPS 256

/* ---------------------------------------------------------------- sizes */

/* Bytes the rowwise scale buffer needs for a [rows, cols] input split into
 * num_groups groups: (ceil(rows/128) + num_groups - 1) * ceil(cols/128) * 512
 * (0 when rows = 0).  Only the prefix used by the actual offsets is written. */
MXF8_API int64_t mxfp8_rowwise_scale_bytes(int64_t rows, int64_t cols, int32_t num_groups);

/* Atom pitch of the colwise scale matrix: ceil(rows/128) + num_groups - 1. */
MXF8_API int64_t mxfp8_colwise_pitch(int64_t rows, int32_t num_groups);

/* Bytes the colwise scale buffer needs: ceil(cols/128) * pitch * 512. */
MXF8_API int64_t mxfp8_colwise_scale_bytes(int64_t rows, int64_t cols, int32_t num_groups);

/* Row stride (bytes) of the transposed colwise codes:
 * round_up(round_up(rows, 32) + 32*(num_groups-1), 128), at least 128. */
MXF8_API int64_t mxfp8_colwise_ld(int64_t rows, int32_t num_groups);

/* Bytes of the workspace a grouped GEMM needs (a status word and reserve). */
MXF8_API int64_t mxfp8_workspace_bytes(int32_t num_groups, int64_t M, int64_t N, int64_t K);

/* ---------------------------------------------------------------- quantisers */

/* Rowwise MXFP8 quantisation (32-blocks along `cols`).
 *   x       bf16 [rows, cols], cols % 32 == 0, rows >= 0
 *   d_offs  num_groups + 1 row offsets (NULL: one group)
 *   q       uint8 [rows, cols] E4M3 codes
 *   scales  uint8 [scale_bytes] E8M0 atoms, scale_bytes >=
 *           mxfp8_rowwise_scale_bytes(rows, cols, num_groups)
 * Errors: INVALID_ARG (null x/q/scales -- x and q may be NULL when rows = 0 --,
 * cols % 32, num_groups < 1, buffer too small), ALIGNMENT, UNSUPPORTED, CUDA.
 * Nothing is launched on error. */
MXF8_API mxf8_status mxfp8_quantize_rowwise(const uint16_t* x, int64_t rows, int64_t cols,
                                   const int32_t* d_offs, int32_t num_groups,
                                   uint8_t* q, uint8_t* scales, int64_t scale_bytes,
                                   void* stream);

/* Colwise MXFP8 quantisation (32-blocks along `rows`, restarting at every
 * group offset), written transposed.
 *   x        bf16 [rows, cols], cols % 32 == 0
 *   qT       uint8 [cols, ldT], ldT == mxfp8_colwise_ld(rows, num_groups);
 *            columns past the last group's padded end are not written
 *   scalesT  uint8 [scale_bytes] >= mxfp8_colwise_scale_bytes(...)
 * Errors as mxfp8_quantize_rowwise, plus INVALID_ARG for a wrong ldT. */
MXF8_API mxf8_status mxfp8_quantize_colwise(const uint16_t* x, int64_t rows, int64_t cols,
                                   const int32_t* d_offs, int32_t num_groups,
                                   uint8_t* qT, int64_t ldT, uint8_t* scalesT,
                                   int64_t scale_bytes, void* stream);

/* Rowwise and colwise quantisation of the same input in one pass (one read
 * of x, both outputs).  Outputs, layouts and errors are exactly those of
 * mxfp8_quantize_rowwise(x, ..., q, scales) followed by
 * mxfp8_quantize_colwise(x, ..., qT, ldT, scalesT): in training X and dY need
 * both layouts (forward/dgrad read rowwise, wgrad colwise) and W needs
 * rowwise (forward) and colwise (dgrad). */
MXF8_API mxf8_status mxfp8_quantize_dual(const uint16_t* x, int64_t rows, int64_t cols,
                                         const int32_t* d_offs, int32_t num_groups,
                                         uint8_t* q, uint8_t* scales, int64_t scale_bytes,
                                         uint8_t* qT, int64_t ldT, uint8_t* scalesT,
                                         int64_t scaleT_bytes, void* stream);

/* ---------------------------------------------------------------- grouped GEMMs
 * Shared arguments: E = num_groups (1..MXF8_GEMM_MAX_GROUPS); M = total rows
 * (d_offs[E]); N % 128 == 0; K % 32 == 0; N, K > 0.  `work` is a device
 * workspace of work_bytes >= mxfp8_workspace_bytes(E, M, N, K) that one call
 * at a time may use; when M = 0 the row-indexed operand and output may be NULL
 * (wgrad still writes dW = 0).  The status word is cleared at the start of every call
 * and set by the device on BAD_OFFSETS or TIMEOUT (read it with
 * mxfp8_get_status).  Errors returned directly: INVALID_ARG, ALIGNMENT,
 * UNSUPPORTED, CUDA; nothing is launched on error. */

/* Forward: y[M, N] bf16.  xq/xs: rowwise(X [M, K], d_offs);
 * wq/ws: rowwise(W viewed as [E*N, K], one group). */
MXF8_API mxf8_status mxfp8_grouped_gemm_fwd(const uint8_t* xq, const uint8_t* xs, int64_t xs_bytes,
                                   const uint8_t* wq, const uint8_t* ws, int64_t ws_bytes,
                                   const int32_t* d_offs, int32_t E, int64_t M, int64_t N,
                                   int64_t K, uint16_t* y, void* work, int64_t work_bytes,
                                   void* stream);

/* Dgrad: dx[M, K] bf16.  dyq/dys: rowwise(dY [M, N], d_offs);
 * wqT/wsT: colwise(W viewed as [E*N, K], one group), ldT = mxfp8_colwise_ld(E*N, 1). */
MXF8_API mxf8_status mxfp8_grouped_gemm_dgrad(const uint8_t* dyq, const uint8_t* dys, int64_t dys_bytes,
                                     const uint8_t* wqT, const uint8_t* wsT, int64_t wsT_bytes,
                                     const int32_t* d_offs, int32_t E, int64_t M, int64_t N,
                                     int64_t K, uint16_t* dx, void* work, int64_t work_bytes,
                                     void* stream);

/* Wgrad: dw[E, N, K] bf16.  dyqT/dysT: colwise(dY [M, N], d_offs);
 * xqT/xsT: colwise(X [M, K], d_offs); both with ldT = mxfp8_colwise_ld(M, E).
 * Experts with no rows get dW_e = 0. */
MXF8_API mxf8_status mxfp8_grouped_gemm_wgrad(const uint8_t* dyqT, const uint8_t* dysT, int64_t dysT_bytes,
                                     const uint8_t* xqT, const uint8_t* xsT, int64_t xsT_bytes,
                                     const int32_t* d_offs, int32_t E, int64_t M, int64_t N,
                                     int64_t K, uint16_t* dw, void* work, int64_t work_bytes,
                                     void* stream);

/* Fwd and dgrad with a quantising epilogue: the GEMM's output, rounded to
 * bf16 as in mxfp8_grouped_gemm_fwd/_dgrad, is also written as MXFP8 straight
 * from the accumulator, so a following MXFP8 GEMM needs no separate
 * quantisation pass over it.  The copies are exactly (byte for byte) what
 *   mxfp8_quantize_rowwise(out, rows = M, cols = C, d_offs, E, q, scales) and
 *   mxfp8_quantize_colwise(out, rows = M, cols = C, d_offs, E, qT, ldT, scalesT)
 * would write from the bf16 output (C = N for fwd, K for dgrad): the MXFP8
 * block encoding of opensourcebeat.com, "Enabling up to 41% faster
 * pre-training: MXFP8 and DeepEP ...", FAQ (OCP MX v1.0), and the layouts at
 * the top of this header.  The pages do not describe this fusion; it
 * follows that page's section "Двухсторонняя атака: MXFP8 и DeepEP", which
 * credits the speed-up to the pipeline as a whole being reworked rather than
 * to one kernel.  The arithmetic is exactly that of the quantisers.
 *   out      bf16 [M, C] or NULL (not written)
 *   q        uint8 [M, C] rowwise codes or NULL; scales (>= scale_bytes =
 *            mxfp8_rowwise_scale_bytes(M, C, E)) must be given with q
 *   qT       uint8 [C, ldT] colwise codes or NULL, ldT = mxfp8_colwise_ld(M, E);
 *            scalesT (>= scaleT_bytes = mxfp8_colwise_scale_bytes(M, C, E))
 *            must be given with qT
 * At least one of out, q, qT must be non-NULL.  Other arguments, errors and
 * the device status are those of mxfp8_grouped_gemm_fwd / _dgrad.
 * Cost: the epilogue's work per output tile is fixed, so the fusion pays off
 * on long contractions (measured on B200: faster than the GEMM followed by
 * mxfp8_quantize_dual from about 32 K blocks of 128); over a short one
 * (16 K blocks and fewer) the two separate calls are faster and give the
 * same bytes. */
MXF8_API mxf8_status mxfp8_grouped_gemm_fwd_quant(const uint8_t* xq, const uint8_t* xs, int64_t xs_bytes,
                                                  const uint8_t* wq, const uint8_t* ws, int64_t ws_bytes,
                                                  const int32_t* d_offs, int32_t E, int64_t M, int64_t N,
                                                  int64_t K, uint16_t* y, uint8_t* q, uint8_t* scales,
                                                  int64_t scale_bytes, uint8_t* qT, int64_t ldT,
                                                  uint8_t* scalesT, int64_t scaleT_bytes, void* work,
                                                  int64_t work_bytes, void* stream);
MXF8_API mxf8_status mxfp8_grouped_gemm_dgrad_quant(const uint8_t* dyq, const uint8_t* dys, int64_t dys_bytes,
                                                    const uint8_t* wqT, const uint8_t* wsT, int64_t wsT_bytes,
                                                    const int32_t* d_offs, int32_t E, int64_t M, int64_t N,
                                                    int64_t K, uint16_t* dx, uint8_t* q, uint8_t* scales,
                                                    int64_t scale_bytes, uint8_t* qT, int64_t ldT,
                                                    uint8_t* scalesT, int64_t scaleT_bytes, void* work,
                                                    int64_t work_bytes, void* stream);

/* Forward gate/up grouped GEMM fused with SwiGLU and MXFP8 quantisation of
 * its result, for the down projection that follows.  The pages credit the
 * MXFP8 speed-up to the expert pipeline as a whole (opensourcebeat.com,
 * section "Двухсторонняя атака: MXFP8 и DeepEP"), and the DeepSeek-V3 and
 * Llama 4 experts apply SwiGLU between their two linears; the pages give no
 * formula, so the plainest reading is used:
 *   Y_e = X_e W_e^T        (W_e: [N, K], N = 2I; Y accumulated in fp32, never written)
 *   h[i, j] = silu(Y[i, j]) * Y[i, I + j],  silu(g) = g / (1 + exp(-g)),
 * evaluated in fp32 from the accumulator and rounded once to bf16 (nearest
 * even).  h is [M, I]; it is written as bf16 (`h`, nullable) and/or as
 * MXFP8 exactly as mxfp8_quantize_rowwise / _colwise(h, d_offs) would encode
 * that bf16 h (q/scales and qT/ldT/scalesT, each pair nullable; at least one
 * of the three outputs).  N % 256 == 0 (I % 128 == 0), otherwise
 * MXF8_ERR_INVALID_ARG; every other argument and error is that of
 * mxfp8_grouped_gemm_fwd_quant with C = I. */
MXF8_API mxf8_status mxfp8_grouped_gemm_fwd_swiglu(const uint8_t* xq, const uint8_t* xs, int64_t xs_bytes,
                                                   const uint8_t* wq, const uint8_t* ws, int64_t ws_bytes,
                                                   const int32_t* d_offs, int32_t E, int64_t M, int64_t N, int64_t K,
                                                   uint16_t* h, uint8_t* q, uint8_t* scales, int64_t scale_bytes,
                                                   uint8_t* qT, int64_t ldT, uint8_t* scalesT, int64_t scaleT_bytes,
                                                   void* work, int64_t work_bytes, void* stream);

/* Forward grouped GEMM that allocates nothing and takes no workspace.
 * The paper has no counterpart to this entry point; it exists for callers
 * that cannot call cudaMalloc (for example a plugin inside an engine that owns
 * the device-memory budget, or a path where an allocation's implicit device
 * synchronisation is not acceptable).  Arguments and results are those of
 * mxfp8_grouped_gemm_fwd without work/work_bytes; the scratch is a static
 * device array of MXF8_NOALLOC_SCRATCH_BYTES inside the library, held by
 * every GPU that loads the library until the process exits.
 *   - The first call on a device looks up that array's device address (with
 *     the device current); make that first call before any stream capture.
 *     The address is kept for the life of the process: after a
 *     cudaDeviceReset on that device it is stale, so do not call this entry
 *     point on a device that has been reset.
 *   - Every call on a device shares the one array; its status word is cleared
 *     at the start of each call, but calls that overlap on the GPU (other
 *     streams, other host threads) race on it.
 *   - host_status (nullable, HOST pointer): when given, the call synchronises
 *     `stream` and stores the device status (an mxf8_status) there.
 *   - Returns MXF8_ERR_INVALID_ARG if the call would need more scratch than
 *     MXF8_NOALLOC_SCRATCH_BYTES, plus every error mxfp8_grouped_gemm_fwd
 *     returns.  It calls no allocating routine. */
#define MXF8_NOALLOC_SCRATCH_BYTES 4096
MXF8_API mxf8_status mxfp8_grouped_gemm_fwd_noalloc(const uint8_t* xq, const uint8_t* xs, int64_t xs_bytes,
                                                    const uint8_t* wq, const uint8_t* ws, int64_t ws_bytes,
                                                    const int32_t* d_offs, int32_t E, int64_t M, int64_t N,
                                                    int64_t K, uint16_t* y, int32_t* host_status,
                                                    void* stream);

/* ---------------------------------------------------------------- tuning and testing switches */

/* Overrides, for the calling process, the tile configuration the grouped
 * GEMMs choose per pass.  The pages fix no tiling; these are this library's
 * own pipeline shapes.
 *   cta_pair  -1 = the library's rule, 0 = 1-CTA 128x256 tiles,
 *             1 = CTA-pair 256x256 tiles (cta_group::2; in fwd/dgrad each
 *             group's ragged last tile runs with the operand roles swapped)
 *   stage_k   -1 = the library's rule, 1 = 128-deep K stages, 2 = 256-deep
 *             (MXFP8 only; the NVFP4 GEMMs take cta_pair and always use
 *             single 128-byte K blocks per stage)
 * Every setting computes the same exact products in fp32 and meets the same
 * tolerance; the hardware's summation order inside a tile may differ between
 * shapes, so results can differ in the last bits.  Only speed is meant to
 * change.  Returns MXF8_ERR_INVALID_ARG for any other value.  Not
 * thread-safe against concurrent GEMM calls. */
MXF8_API mxf8_status mxfp8_set_gemm_tiling(int32_t cta_pair, int32_t stage_k);

/* Test switch for the bounded pipeline waits: while enabled (enable != 0),
 * every grouped GEMM launch (1-CTA tiles and CTA pairs alike) leaves its
 * first pipeline stage unfilled, so the wait on it runs out after the 2 s
 * limit; the kernel drains what it issued, frees tensor memory and returns
 * with MXF8_ERR_TIMEOUT in the workspace status.  Off by default; meant only
 * for tests of that path. */
MXF8_API void mxfp8_testing_stall_first_stage(int32_t enable);

/* ---------------------------------------------------------------- MoE dispatch / combine */
/* The steps around the grouped GEMM in a Mixture-of-Experts layer on one
 * GPU: tokens are permuted so every expert's rows are contiguous (with their
 * real counts, no capacity padding: iitak.ru, "NVIDIA в 10 раз ускорила
 * обучение моделей-«смесей экспертов» на JAX", paragraph on the Transformer
 * Engine grouped GEMM), quantised on the way, and the experts' outputs are
 * combined back per token with the router weights.  Across GPUs these are
 * the dispatch and combine all-to-alls (opensourcebeat.com, section
 * "Двухсторонняя атака: MXFP8 и DeepEP"); the pages give no formulas, so the
 * plainest reading is used: a stable grouping by expert and a weighted sum. */

/* Largest num_experts the plan accepts. */
#define MXF8_MOE_MAX_EXPERTS 256

/* Workspace of mxfp8_moe_plan in bytes (status word + per-pair ranks +
 * per-chunk histograms). */
MXF8_API int64_t mxfp8_moe_plan_workspace_bytes(int64_t num_tokens, int32_t top_k, int32_t num_experts);

/* Dispatch plan of a top-k routing.
 *   idx     int32 [T, k] expert id of slot j of token t (row-major)
 *   offs    int32 [E + 1] out: exclusive prefix of the per-expert pair counts
 *           (offs[E] = T*k when every id is valid) -- the grouped GEMM's d_offs
 *   perm    int32 [T*k] out: token of permuted row r
 *   inv     int32 [T, k] out: permuted row of slot (t, j)
 * Inside an expert the pairs keep ascending (token, slot) order, so the plan
 * is deterministic.  work/work_bytes >= mxfp8_moe_plan_workspace_bytes; the
 * device status (mxfp8_get_status(work)) is MXF8_ERR_BAD_ROUTING if an id is
 * outside [0, E): such slots get inv = -1 and no row.
 * Errors: INVALID_ARG (null pointers, T < 0, k < 1, E outside [1, 256],
 * T*k >= 2^31, small workspace), ALIGNMENT (work), UNSUPPORTED, CUDA. */
MXF8_API mxf8_status mxfp8_moe_plan(const int32_t* idx, int64_t num_tokens, int32_t top_k, int32_t num_experts,
                                    int32_t* offs, int32_t* perm, int32_t* inv, void* work, int64_t work_bytes,
                                    void* stream);

/* Token permute fused with dual MXFP8 quantisation: quantises the matrix
 * Xp[r] = x[perm[r]] (r < rows, grouped by d_offs) into both layouts, byte
 * for byte what mxfp8_quantize_dual(Xp, rows, cols, d_offs, ...) writes,
 * without materialising Xp.
 *   x       bf16 [num_tokens, cols], cols % 32 == 0
 *   perm    int32 [rows] (from mxfp8_moe_plan; rows = T*k); an entry outside
 *           [0, num_tokens) quantises a zero row
 *   d_offs  int32 [num_groups + 1] (from mxfp8_moe_plan)
 *   q, scales, qT, ldT, scalesT: as mxfp8_quantize_dual with `rows` rows.
 * Errors as mxfp8_quantize_dual, plus INVALID_ARG for null perm/x. */
MXF8_API mxf8_status mxfp8_permute_quantize_dual(const uint16_t* x, int64_t num_tokens, int64_t cols,
                                                 const int32_t* perm, int64_t rows, const int32_t* d_offs,
                                                 int32_t num_groups, uint8_t* q, uint8_t* scales,
                                                 int64_t scale_bytes, uint8_t* qT, int64_t ldT, uint8_t* scalesT,
                                                 int64_t scaleT_bytes, void* stream);

/* Combine: y[t, c] = sum over j < k of w[t, j] * yp[inv[t, j], c].  The
 * products (fp32 weight x bf16 value) are exact in fp64, the sum runs in
 * fp64 in slot order and is rounded once to bf16 (nearest even).
 *   yp      bf16 [rows, cols] expert outputs in permuted order, cols % 8 == 0
 *   inv     int32 [T, k] (from mxfp8_moe_plan); an entry outside [0, rows)
 *           contributes nothing
 *   w       fp32 [T, k] router weights
 *   y       bf16 [T, cols] out
 * Errors: INVALID_ARG (null pointers, cols % 8, T < 0, k < 1), ALIGNMENT
 * (yp, y), UNSUPPORTED, CUDA. */
MXF8_API mxf8_status mxfp8_moe_combine(const uint16_t* yp, int64_t rows, int64_t cols, const int32_t* inv,
                                       const float* w, int64_t num_tokens, int32_t top_k, uint16_t* y,
                                       void* stream);

/* ---------------------------------------------------------------- expert-parallel dispatch */
/* What an expert-parallel MoE layer sends between GPUs.  Each layer sends
 * every token to the GPUs holding its experts and brings the expert outputs
 * back (opensourcebeat.com, "Enabling up to 41% faster pre-training: MXFP8
 * and DeepEP ...", section "Двухсторонняя атака: MXFP8 и DeepEP"); a token
 * needed by several experts of one destination crosses the network once and
 * is copied there (iitak.ru, "NVIDIA в 10 раз ускорила обучение
 * моделей-«смесей экспертов» на JAX", paragraph on NCCL EP).  These calls
 * prepare and unpack what travels; the transfer itself is the caller's
 * (an NCCL all-to-all, split by the counts below).
 *
 * Readings (the pages give no format): P ranks own E/P consecutive experts
 * each (rank p: experts p*E/P .. (p+1)*E/P - 1).  A token travels to each
 * rank owning one of its experts as one record: its row in rowwise MXFP8 --
 * byte 32b + n is the E4M3 code of element 32b + n, byte C + b the E8M0 scale
 * byte of block b (the quantisers' block rule), then zeros up to
 * mxfp8_ep_record_bytes(C) -- 1 + 1/32 bytes per element instead of bf16's 2.
 * Each routed (token, slot) pair travels as a pair entry: its local expert
 * id (e - p*E/P) and its record index, counted from the first record sent to
 * that rank.  Send order: destination rank, then token, then slot, all
 * ascending; a receiver concatenates what its sources sent in rank order. */

#define MXF8_EP_MAX_RANKS 256
#define MXF8_EP_MAX_TOP_K 32

/* Bytes of one record holding a row of `cols` elements (a multiple of 16). */
MXF8_API int64_t mxfp8_ep_record_bytes(int64_t cols);

/* Workspace of mxfp8_ep_plan in bytes. */
MXF8_API int64_t mxfp8_ep_plan_workspace_bytes(int64_t num_tokens, int32_t num_ranks);

/* Send plan of a top-k routing over P ranks (no host synchronisation).
 *   idx          int32 [T, k] global expert ids
 *   counts       int32 [2P] out: records sent to rank p at [p], pairs at [P + p]
 *   rec_token    int32 [T * min(k, P)] out: token of record i (the first
 *                sum(counts[0..P-1]) entries are written)
 *   pair_expert  int32 [T * k] out: local expert id of pair s
 *   pair_rec     int32 [T * k] out: record of pair s within its rank's records
 *   ret_pos      int32 [T, k] out: pair index of slot (t, j) -- the row of
 *                the returned expert outputs that belongs to it -- or -1
 * An id outside [0, E) is not sent (ret_pos -1) and sets the device status
 * (mxfp8_get_status(work)) to MXF8_ERR_BAD_ROUTING.
 * Errors: INVALID_ARG (null pointers, T < 0, k outside [1, MXF8_EP_MAX_TOP_K],
 * P outside [1, MXF8_EP_MAX_RANKS], E < 1 or not a multiple of P, T*k >= 2^31,
 * small workspace), ALIGNMENT (work), UNSUPPORTED, CUDA. */
MXF8_API mxf8_status mxfp8_ep_plan(const int32_t* idx, int64_t num_tokens, int32_t top_k, int32_t num_experts,
                                   int32_t num_ranks, int32_t* counts, int32_t* rec_token, int32_t* pair_expert,
                                   int32_t* pair_rec, int32_t* ret_pos, void* work, int64_t work_bytes,
                                   void* stream);

/* Quantise and pack: record i = rowwise MXFP8 of x[rec_token[i]] (a token
 * index outside [0, T) packs an all-zero record).
 *   x        bf16 [T, cols], cols % 32 == 0, 16-byte aligned
 *   records  uint8 [num_records, mxfp8_ep_record_bytes(cols)] out, 16-byte aligned
 * Errors: INVALID_ARG (null pointers, sizes), ALIGNMENT, UNSUPPORTED, CUDA. */
MXF8_API mxf8_status mxfp8_ep_pack(const uint16_t* x, int64_t num_tokens, int64_t cols, const int32_t* rec_token,
                                   int64_t num_records, uint8_t* records, void* stream);

/* Receiving side.  R records and `rows` pair entries arrived from P sources,
 * each source's after those of lower ranks; src_base int32 [2(P + 1)]
 * (device) holds the first pair of each source at [q] (the total at [P]) and
 * its first record at [P + 1 + q] (the total at [2P + 1]).  Grouped row r
 * (rows grouped by local expert with d_offs, e.g. mxfp8_moe_plan of the pair
 * entries' expert ids) is pair perm[r]; its record is
 * src_base[P + 1 + q] + pair_rec[perm[r]], q the source whose pairs hold
 * perm[r].  Writes the grouped rows' rowwise MXFP8 -- codes q [rows, cols]
 * and scale atoms -- byte for byte what mxfp8_quantize_rowwise writes for
 * the bf16 rows the records were made from (rowwise blocks lie within one
 * row, so quantising before the transfer changes nothing).  A pair or record
 * index out of range gives a zero row.
 * Errors: INVALID_ARG (null pointers, cols % 32, P outside
 * [1, MXF8_EP_MAX_RANKS], num_groups < 1, small scale buffer), ALIGNMENT
 * (records, q, scales), UNSUPPORTED, CUDA. */
MXF8_API mxf8_status mxfp8_ep_unpack(const uint8_t* records, int64_t num_records, int64_t cols,
                                     const int32_t* pair_rec, const int32_t* src_base, int32_t num_sources,
                                     const int32_t* perm, int64_t rows, const int32_t* d_offs, int32_t num_groups,
                                     uint8_t* q, uint8_t* scales, int64_t scale_bytes, void* stream);

/* dst[i] = src[idx[i]] for rows of row_bytes bytes (a multiple of 16); an
 * index outside [0, src_rows) gives a zero row.  Used for the return trip:
 * each received pair's expert output row, in arrival order.
 * Errors: INVALID_ARG (null pointers, sizes), ALIGNMENT (src, dst),
 * UNSUPPORTED, CUDA. */
MXF8_API mxf8_status mxfp8_gather_rows(const void* src, int64_t src_rows, int64_t row_bytes, const int32_t* idx,
                                       int64_t n, void* dst, void* stream);

/* ---------------------------------------------------------------- NVFP4 */
/* NVFP4 quantisation: 4-bit E2M1 elements in blocks of 16 that share an E4M3
 * scale, plus one fp32 scale per tensor.  The pages name NVFP4 only as the
 * format NVIDIA's MoE training adds next (iitak.ru, "NVIDIA в 10 раз
 * ускорила обучение моделей-«смесей экспертов» на JAX", closing paragraph);
 * the rules are NVIDIA's public NVFP4 definition, read plainly, with every
 * fp32 operation rounded to nearest in this order:
 *   S  = 2688 / amax(tensor)         (2688 = 448 * 6; S = 1 when amax = 0)
 *   sf = E4M3((amax_block * S) / 6)  (nearest even, saturating at 448)
 *   q  = E2M1((x * S) / sf)          (nearest even, saturating at +-6; 0 when sf = 0)
 *   x ~ q * sf / S
 * Non-finite inputs are outside the contract.
 * Layouts (as MXFP8, with 16-element blocks and packed codes):
 *   codes hold two elements per byte, element 2i in the low nibble of byte i;
 *   a 512-byte scale atom covers 128 rows x 4 blocks = 64 elements, byte
 *   (row%32)*16 + ((row%128)/32)*4 + blk%4;
 *   rowwise: q [rows, cols/2]; scale rows of group g start at a multiple of
 *     128 (as MXFP8); pitch ceil(cols/64) atoms;
 *   colwise: qT [cols, ldT/2] bytes, ldT = mxfp8_nvfp4_colwise_ld(rows, G)
 *     elements; element (d_offs[g] + t, c) at nibble P_g + t of row c,
 *     P_g = sum over h < g of round_up(m_h, 32), pad nibbles 0; blocks of 16
 *     rows restart at every group offset; scales S^T[c, 4*Q_g + t/16] with
 *     Q_g = sum over h < g of ceil(m_h/64), pitch mxfp8_nvfp4_colwise_pitch. */
MXF8_API int64_t mxfp8_nvfp4_rowwise_scale_bytes(int64_t rows, int64_t cols, int32_t num_groups);
MXF8_API int64_t mxfp8_nvfp4_colwise_pitch(int64_t rows, int32_t num_groups);
MXF8_API int64_t mxfp8_nvfp4_colwise_scale_bytes(int64_t rows, int64_t cols, int32_t num_groups);
MXF8_API int64_t mxfp8_nvfp4_colwise_ld(int64_t rows, int32_t num_groups);

/* amax (device fp32, out) = largest |x| over n bf16 elements (x 16-byte
 * aligned; n = 0 gives 0).  Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED, CUDA. */
MXF8_API mxf8_status mxfp8_nvfp4_amax(const uint16_t* x, int64_t n, float* amax, void* stream);

/* Rowwise / colwise NVFP4 of x [rows, cols] (cols % 64 == 0) with groups
 * d_offs, the tensor scale taken from the device amax written by
 * mxfp8_nvfp4_amax.  Buffer sizes from the functions above; errors as the
 * MXFP8 quantisers. */
MXF8_API mxf8_status mxfp8_nvfp4_quantize_rowwise(const uint16_t* x, int64_t rows, int64_t cols,
                                                  const int32_t* d_offs, int32_t num_groups, const float* amax,
                                                  uint8_t* q, uint8_t* scales, int64_t scale_bytes, void* stream);
MXF8_API mxf8_status mxfp8_nvfp4_quantize_colwise(const uint16_t* x, int64_t rows, int64_t cols,
                                                  const int32_t* d_offs, int32_t num_groups, const float* amax,
                                                  uint8_t* qT, int64_t ldT, uint8_t* scalesT, int64_t scale_bytes,
                                                  void* stream);

/* NVFP4 grouped GEMMs: the MXFP8 fwd / dgrad / wgrad with NVFP4 operands
 * (E2M1 x E2M1 block-scaled MMA, kind::mxf4nvf4, 16-element E4M3 scales
 * applied in hardware, fp32 accumulation), the output multiplied by
 * 1 / (S_a * S_b) (S = 2688 / amax of each operand's tensor, as the
 * quantisers use) and written as bf16.  Operands are the NVFP4 quantisers'
 * outputs in the same roles as for MXFP8:
 *   fwd:   rowwise(X, d_offs), rowwise(W as [E*N, K], one group)
 *   dgrad: rowwise(dY, d_offs), colwise(W as [E*N, K], one group)
 *   wgrad: colwise(dY, d_offs), colwise(X, d_offs)
 * with the amax (device fp32) each was quantised with.  K % 64 == 0 and the
 * MXFP8 GEMMs' other rules apply; errors and device status as for MXFP8. */
MXF8_API mxf8_status mxfp8_nvfp4_grouped_gemm_fwd(const uint8_t* xq, const uint8_t* xs, int64_t xs_bytes,
                                                  const float* x_amax, const uint8_t* wq, const uint8_t* ws,
                                                  int64_t ws_bytes, const float* w_amax, const int32_t* d_offs,
                                                  int32_t E, int64_t M, int64_t N, int64_t K, uint16_t* y,
                                                  void* work, int64_t work_bytes, void* stream);
MXF8_API mxf8_status mxfp8_nvfp4_grouped_gemm_dgrad(const uint8_t* dyq, const uint8_t* dys, int64_t dys_bytes,
                                                    const float* dy_amax, const uint8_t* wqT, const uint8_t* wsT,
                                                    int64_t wsT_bytes, const float* w_amax, const int32_t* d_offs,
                                                    int32_t E, int64_t M, int64_t N, int64_t K, uint16_t* dx,
                                                    void* work, int64_t work_bytes, void* stream);
MXF8_API mxf8_status mxfp8_nvfp4_grouped_gemm_wgrad(const uint8_t* dyqT, const uint8_t* dysT, int64_t dysT_bytes,
                                                    const float* dy_amax, const uint8_t* xqT, const uint8_t* xsT,
                                                    int64_t xsT_bytes, const float* x_amax, const int32_t* d_offs,
                                                    int32_t E, int64_t M, int64_t N, int64_t K, uint16_t* dw,
                                                    void* work, int64_t work_bytes, void* stream);

/* ---------------------------------------------------------------- status */

/* Synchronises `stream`, then stores the device status of the last GEMM that
 * used `work` (an mxf8_status value, MXF8_OK if none) in *device_status. */
MXF8_API mxf8_status mxfp8_get_status(const void* work, void* stream, int32_t* device_status);

/* Static description of a status code. */
MXF8_API const char* mxfp8_status_string(int32_t status);

/* Text of the last CUDA error seen by this thread ("" if none). */
MXF8_API const char* mxfp8_last_cuda_error(void);

/* 1 if the current device is sm_100 (the only target), else 0. */
MXF8_API int32_t mxfp8_device_supported(void);

#ifdef __cplusplus
}
#endif
#endif /* MXFP8_H */
