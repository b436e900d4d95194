// launch.h -- internal launchers behind the C ABI (arguments already checked).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace mxf8 {

// Bytes of the workspace every grouped GEMM takes: its status word and a
// reserve (mxfp8_workspace_bytes).
constexpr int64_t kGemmWorkspaceBytes = 256;

// 2D TMA map over a row-major matrix [rows, cols] of `esize`-byte elements
// with row stride `ld` elements; box = box_cols x box_rows; zero fill
// outside the matrix.  False if the driver rejects it.
bool make_tensor_map(CUtensorMap* m, const void* base, CUtensorMapDataType dtype, int esize, int64_t rows,
                     int64_t cols, int64_t ld, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz);

cudaError_t launch_quantize_rowwise(const uint16_t* x, int64_t rows, int64_t cols,
                                    const int32_t* offs, int32_t G, uint8_t* q, uint8_t* sf,
                                    cudaStream_t stream);

cudaError_t launch_quantize_colwise(const uint16_t* x, int64_t rows, int64_t cols,
                                    const int32_t* offs, int32_t G, uint8_t* qT, int64_t ldT,
                                    uint8_t* sfT, cudaStream_t stream);

cudaError_t launch_quantize_dual(const uint16_t* x, int64_t rows, int64_t cols, const int32_t* offs,
                                 int32_t G, uint8_t* q, uint8_t* sf, uint8_t* qT, int64_t ldT, uint8_t* sfT,
                                 cudaStream_t stream);

// Dual quantisation of x[perm[r]] for r < rows (the MoE token permute);
// perm entries outside [0, src_rows) read as zero rows.
cudaError_t launch_permute_quantize_dual(const uint16_t* x, int64_t src_rows, int64_t cols, const int32_t* perm,
                                         int64_t rows, const int32_t* offs, int32_t G, uint8_t* q, uint8_t* sf,
                                         uint8_t* qT, int64_t ldT, uint8_t* sfT, cudaStream_t stream);

// MoE dispatch plan: chunks of ranked pairs (workspace sizing) and the launch.
int64_t moe_plan_chunks(int64_t pairs);
cudaError_t launch_moe_plan(const int32_t* idx, int64_t T, int32_t k, int32_t E, int32_t* offs, int32_t* perm,
                            int32_t* inv, int32_t* status, int32_t* rank, int32_t* hist, cudaStream_t stream);

// MoE combine: y[t] = sum_j w[t, j] * yp[inv[t, j]] (cols % 8 == 0).
cudaError_t launch_moe_combine(const uint16_t* yp, int64_t rows, int64_t cols, const int32_t* inv, const float* w,
                               int64_t T, int32_t k, uint16_t* y, cudaStream_t stream);

// NVFP4: tensor amax (fp32, device), rowwise and colwise quantisation.
cudaError_t launch_nvfp4_amax(const uint16_t* x, int64_t n, float* amax, cudaStream_t stream);
cudaError_t launch_nvfp4_rowwise(const uint16_t* x, int64_t rows, int64_t cols, const int32_t* offs, int32_t G,
                                 const float* amax, uint8_t* q, uint8_t* sf, cudaStream_t stream);
cudaError_t launch_nvfp4_colwise(const uint16_t* x, int64_t rows, int64_t cols, const int32_t* offs, int32_t G,
                                 const float* amax, uint8_t* qT, int64_t ldT, uint8_t* sfT, cudaStream_t stream);

enum GemmMode : int { kFwd = 0, kDgrad = 1, kWgrad = 2 };

// One grouped GEMM.  a/b: operand codes (K-major), lda/ldb their row strides
// in bytes, a_rows/b_rows their row counts; sfa/sfb: scale atoms with the
// given pitch (atoms per atom row) and total atom counts.
struct GemmArgs {
  int mode;
  int32_t E;
  int64_t M, N, K;
  const int32_t* offs;
  const uint8_t* a; int64_t lda, a_rows, a_cols;
  const uint8_t* b; int64_t ldb, b_rows, b_cols;
  const uint8_t* sfa; int64_t sfa_pitch, sfa_atoms;
  const uint8_t* sfb; int64_t sfb_pitch, sfb_atoms;
  uint16_t* out;                 // bf16 output; may be null when a quantised copy is requested
  int32_t* status;
  uint64_t timeout_ns;
  // Test hook (1-CTA launches): the producer leaves its first pipeline stage
  // unfilled, so the MMA warp's bounded wait for it runs out (MXF8_ERR_TIMEOUT).
  int32_t inject_skip_stage = 0;
  // fwd/dgrad only: MXFP8 copies of the output written by the epilogue, in
  // the quantisers' rowwise (qr, sr) and colwise (qc, sc) layouts over the
  // GEMM's groups; null = not written.
  uint8_t* qr = nullptr; uint8_t* sr = nullptr;
  uint8_t* qc = nullptr; uint8_t* sc = nullptr;
  int64_t qc_ld = 0, sc_pitch = 0;
  // NVFP4 operands (codes packed two per byte, 16-element E4M3 scales):
  // device amax of each operand tensor; lda/ldb/a_cols/b_cols are in bytes.
  bool fp4 = false;
  const float* amax_a = nullptr;
  const float* amax_b = nullptr;
  // fwd only: the epilogue applies SwiGLU to the gate/up output (gate =
  // columns 0..N/2-1, up = N/2..N-1) and writes h [M, N/2] (bf16 `out`
  // and/or the MXFP8 copies above); requires N % 256 == 0.
  bool swiglu = false;
};

// Returns cudaSuccess or the CUDA error; *detail gets a short reason for
// failures detected before the launch (tensor-map encoding).
cudaError_t launch_grouped_gemm(const GemmArgs& args, cudaStream_t stream, const char** detail);

// Process-wide tile overrides set through mxfp8_set_gemm_tiling (-1 = rule).
void gemm_tiling_override(int* cta_pair, int* stage_k);

// Records a CUDA failure for mxfp8_last_cuda_error (thread-local text).
void record_cuda_error(cudaError_t e, const char* where, const char* detail);

}  // namespace mxf8
