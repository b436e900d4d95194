// launch.h -- internal launchers behind the C ABI (arguments already checked).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace mxf8 {

cudaError_t launch_quantize_rowwise(const uint16_t* x, int64_t rows, int64_t cols,
                                    const int32_t* offs, int32_t G, uint8_t* q, uint8_t* sf,
                                    cudaStream_t stream);

cudaError_t launch_quantize_colwise(const uint16_t* x, int64_t rows, int64_t cols,
                                    const int32_t* offs, int32_t G, uint8_t* qT, int64_t ldT,
                                    uint8_t* sfT, cudaStream_t stream);

cudaError_t launch_quantize_dual(const uint16_t* x, int64_t rows, int64_t cols, const int32_t* offs,
                                 int32_t G, uint8_t* q, uint8_t* sf, uint8_t* qT, int64_t ldT, uint8_t* sfT,
                                 cudaStream_t stream);

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
  // fwd/dgrad only: MXFP8 copies of the output written by the epilogue, in
  // the quantisers' rowwise (qr, sr) and colwise (qc, sc) layouts over the
  // GEMM's groups; null = not written.
  uint8_t* qr = nullptr; uint8_t* sr = nullptr;
  uint8_t* qc = nullptr; uint8_t* sc = nullptr;
  int64_t qc_ld = 0, sc_pitch = 0;
};

// Returns cudaSuccess or the CUDA error; *detail gets a short reason for
// failures detected before the launch (tensor-map encoding).
cudaError_t launch_grouped_gemm(const GemmArgs& args, cudaStream_t stream, const char** detail);

}  // namespace mxf8
