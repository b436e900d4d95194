// api.cu -- the extern "C" entry points declared in include/mxfp8.h: argument
// checks, workspace status handling and kernel launches.  No entry point
// allocates device memory.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "ep_launch.h"
#include "launch.h"
#include "mxfp8.h"

namespace {

thread_local char g_last_error[256] = "";

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;   // a pipeline wait gives up after 2 s
constexpr int64_t kWorkspaceBytes = mxf8::kGemmWorkspaceBytes;   // status word + reserve

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
int64_t round_up(int64_t a, int64_t b) { return cdiv(a, b) * b; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t blocks128_bound(int64_t rows, int32_t G) { return rows <= 0 ? 0 : cdiv(rows, 128) + G - 1; }

// Switches set through mxfp8_testing_stall_first_stage / mxfp8_set_gemm_tiling.
std::atomic<int> g_stall_first_stage{0};
std::atomic<int> g_tiling_cta_pair{-1};
std::atomic<int> g_tiling_stage_k{-1};

mxf8_status cuda_fail(cudaError_t e, const char* where, const char* detail = nullptr) {
  mxf8::record_cuda_error(e, where, detail);
  return MXF8_ERR_CUDA;
}

// Only sm_100 parts carry the tcgen05 instructions this library is built for.
mxf8_status check_device() {
  static int cached[64];   // 0 unknown, 1 supported, 2 unsupported
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return MXF8_ERR_UNSUPPORTED;
  if (cached[dev] == 0) {
    int major = 0, minor = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    cached[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return cached[dev] == 1 ? MXF8_OK : MXF8_ERR_UNSUPPORTED;
}

mxf8_status check_quant_args(const uint16_t* x, int64_t rows, int64_t cols, int32_t G, const void* q,
                             const void* scales, int64_t scale_bytes, int64_t need) {
  if (rows < 0 || cols <= 0 || cols % 32 != 0 || G < 1) return MXF8_ERR_INVALID_ARG;
  if ((rows > 0 && (!x || !q)) || !scales) return MXF8_ERR_INVALID_ARG;   // no rows: x and q may be empty
  if (rows > (int64_t(1) << 31) - 1 || cols > int64_t(65535) * 128) return MXF8_ERR_INVALID_ARG;
  if (scale_bytes < need) return MXF8_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(q) || !aligned16(scales)) return MXF8_ERR_ALIGNMENT;
  return MXF8_OK;
}

struct GemmCheck {
  const uint8_t* a; const uint8_t* as; int64_t as_bytes;
  const uint8_t* b; const uint8_t* bs; int64_t bs_bytes;
  const int32_t* offs; int32_t E; int64_t M, N, K;
  const void* out; void* work; int64_t work_bytes;
};

mxf8_status check_gemm_args(const GemmCheck& c) {
  // With no rows the row-indexed buffers (a for fwd/dgrad, out) may be empty.
  if ((c.M > 0 && (!c.a || !c.out)) || !c.as || !c.b || !c.bs || !c.offs || !c.work) return MXF8_ERR_INVALID_ARG;
  if (c.E < 1 || c.E > MXF8_GEMM_MAX_GROUPS) return MXF8_ERR_INVALID_ARG;
  if (c.M < 0 || c.M > (int64_t(1) << 30) || c.N <= 0 || c.K <= 0) return MXF8_ERR_INVALID_ARG;
  if (c.N % 128 != 0 || c.K % 32 != 0) return MXF8_ERR_INVALID_ARG;
  if (int64_t(c.E) * c.N > (int64_t(1) << 30) || c.K > (int64_t(1) << 30)) return MXF8_ERR_INVALID_ARG;
  if (c.work_bytes < kWorkspaceBytes) return MXF8_ERR_INVALID_ARG;
  if (!aligned16(c.a) || !aligned16(c.as) || !aligned16(c.b) || !aligned16(c.bs) || !aligned16(c.out) ||
      !aligned16(c.work))
    return MXF8_ERR_ALIGNMENT;
  return MXF8_OK;
}

mxf8_status run_gemm(mxf8::GemmArgs& g, void* work, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  g.status = static_cast<int32_t*>(work);
  g.timeout_ns = kDefaultTimeoutNs;
  // Test switch for the bounded-wait path (mxfp8_testing_stall_first_stage):
  // the launch leaves its first pipeline stage unfilled and the device
  // status becomes MXF8_ERR_TIMEOUT after the wait limit.
  g.inject_skip_stage = g_stall_first_stage.load(std::memory_order_relaxed);
  cudaError_t e = cudaMemsetAsync(work, 0, sizeof(int32_t), st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(status)");
  const char* detail = nullptr;
  e = mxf8::launch_grouped_gemm(g, st, &detail);
  if (e != cudaSuccess) return cuda_fail(e, "grouped_gemm launch", detail);
  return MXF8_OK;
}

// Quantising epilogue: checks the output copies and attaches them to g.
// C = columns of the GEMM output.  `out` may be NULL when a copy is asked for.
mxf8_status attach_quant_outputs(mxf8::GemmArgs& g, int64_t C, const uint16_t* out, uint8_t* q,
                                 uint8_t* scales, int64_t scale_bytes, uint8_t* qT, int64_t ldT,
                                 uint8_t* scalesT, int64_t scaleT_bytes) {
  if (!out && !q && !qT) return MXF8_ERR_INVALID_ARG;
  if (q) {
    if (!scales || scale_bytes < mxfp8_rowwise_scale_bytes(g.M, C, g.E)) return MXF8_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(scales)) return MXF8_ERR_ALIGNMENT;
  }
  if (qT) {
    if (!scalesT || ldT != mxfp8_colwise_ld(g.M, g.E) || scaleT_bytes < mxfp8_colwise_scale_bytes(g.M, C, g.E))
      return MXF8_ERR_INVALID_ARG;
    if (!aligned16(qT) || !aligned16(scalesT)) return MXF8_ERR_ALIGNMENT;
  }
  g.qr = q; g.sr = q ? scales : nullptr;
  g.qc = qT; g.sc = qT ? scalesT : nullptr;
  g.qc_ld = ldT; g.sc_pitch = mxfp8_colwise_pitch(g.M, g.E);
  return MXF8_OK;
}

}  // namespace

namespace mxf8 {

void record_cuda_error(cudaError_t e, const char* where, const char* detail) {
  std::snprintf(g_last_error, sizeof g_last_error, "%s: %s%s%s", where, cudaGetErrorString(e),
                detail ? " -- " : "", detail ? detail : "");
}

void gemm_tiling_override(int* cta_pair, int* stage_k) {
  *cta_pair = g_tiling_cta_pair.load(std::memory_order_relaxed);
  *stage_k = g_tiling_stage_k.load(std::memory_order_relaxed);
}

}  // namespace mxf8

extern "C" {

mxf8_status mxfp8_set_gemm_tiling(int32_t cta_pair, int32_t stage_k) {
  if (cta_pair < -1 || cta_pair > 1 || stage_k < -1 || stage_k == 0 || stage_k > 2) return MXF8_ERR_INVALID_ARG;
  g_tiling_cta_pair.store(cta_pair, std::memory_order_relaxed);
  g_tiling_stage_k.store(stage_k, std::memory_order_relaxed);
  return MXF8_OK;
}

void mxfp8_testing_stall_first_stage(int32_t enable) {
  g_stall_first_stage.store(enable != 0 ? 1 : 0, std::memory_order_relaxed);
}

int64_t mxfp8_rowwise_scale_bytes(int64_t rows, int64_t cols, int32_t num_groups) {
  if (rows < 0 || cols <= 0 || num_groups < 1) return 0;
  return blocks128_bound(rows, num_groups) * cdiv(cols, 128) * 512;
}

int64_t mxfp8_colwise_pitch(int64_t rows, int32_t num_groups) {
  if (rows < 0 || num_groups < 1) return 0;
  return blocks128_bound(rows, num_groups);
}

int64_t mxfp8_colwise_scale_bytes(int64_t rows, int64_t cols, int32_t num_groups) {
  if (rows < 0 || cols <= 0 || num_groups < 1) return 0;
  return cdiv(cols, 128) * mxfp8_colwise_pitch(rows, num_groups) * 512;
}

int64_t mxfp8_colwise_ld(int64_t rows, int32_t num_groups) {
  if (rows < 0 || num_groups < 1) return 0;
  const int64_t ld = round_up(round_up(rows, 32) + 32 * int64_t(num_groups - 1), 128);
  return ld < 128 ? 128 : ld;
}

int64_t mxfp8_workspace_bytes(int32_t num_groups, int64_t M, int64_t N, int64_t K) {
  (void)num_groups; (void)M; (void)N; (void)K;
  return kWorkspaceBytes;
}

mxf8_status mxfp8_quantize_rowwise(const uint16_t* x, int64_t rows, int64_t cols, const int32_t* d_offs,
                                   int32_t num_groups, uint8_t* q, uint8_t* scales, int64_t scale_bytes,
                                   void* stream) {
  mxf8_status s = check_quant_args(x, rows, cols, num_groups, q, scales, scale_bytes,
                                   mxfp8_rowwise_scale_bytes(rows, cols, num_groups));
  if (s != MXF8_OK) return s;
  if (!d_offs && num_groups != 1) return MXF8_ERR_INVALID_ARG;
  if ((s = check_device()) != MXF8_OK) return s;
  cudaError_t e = mxf8::launch_quantize_rowwise(x, rows, cols, d_offs, num_groups, q, scales,
                                                static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MXF8_OK : cuda_fail(e, "quantize_rowwise launch");
}

mxf8_status mxfp8_quantize_colwise(const uint16_t* x, int64_t rows, int64_t cols, const int32_t* d_offs,
                                   int32_t num_groups, uint8_t* qT, int64_t ldT, uint8_t* scalesT,
                                   int64_t scale_bytes, void* stream) {
  mxf8_status s = check_quant_args(x, rows, cols, num_groups, qT, scalesT, scale_bytes,
                                   mxfp8_colwise_scale_bytes(rows, cols, num_groups));
  if (s != MXF8_OK) return s;
  if (!d_offs && num_groups != 1) return MXF8_ERR_INVALID_ARG;
  if (ldT != mxfp8_colwise_ld(rows, num_groups)) return MXF8_ERR_INVALID_ARG;
  if ((s = check_device()) != MXF8_OK) return s;
  cudaError_t e = mxf8::launch_quantize_colwise(x, rows, cols, d_offs, num_groups, qT, ldT, scalesT,
                                                static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MXF8_OK : cuda_fail(e, "quantize_colwise launch");
}

mxf8_status mxfp8_quantize_dual(const uint16_t* x, int64_t rows, int64_t cols, const int32_t* d_offs,
                                int32_t num_groups, uint8_t* q, uint8_t* scales, int64_t scale_bytes, uint8_t* qT,
                                int64_t ldT, uint8_t* scalesT, int64_t scaleT_bytes, void* stream) {
  mxf8_status s = check_quant_args(x, rows, cols, num_groups, q, scales, scale_bytes,
                                   mxfp8_rowwise_scale_bytes(rows, cols, num_groups));
  if (s != MXF8_OK) return s;
  s = check_quant_args(x, rows, cols, num_groups, qT, scalesT, scaleT_bytes,
                       mxfp8_colwise_scale_bytes(rows, cols, num_groups));
  if (s != MXF8_OK) return s;
  if (!d_offs && num_groups != 1) return MXF8_ERR_INVALID_ARG;
  if (ldT != mxfp8_colwise_ld(rows, num_groups)) return MXF8_ERR_INVALID_ARG;
  if ((s = check_device()) != MXF8_OK) return s;
  cudaError_t e = mxf8::launch_quantize_dual(x, rows, cols, d_offs, num_groups, q, scales, qT, ldT, scalesT,
                                             static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MXF8_OK : cuda_fail(e, "quantize_dual launch");
}

mxf8_status mxfp8_grouped_gemm_fwd(const uint8_t* xq, const uint8_t* xs, int64_t xs_bytes, const uint8_t* wq,
                                   const uint8_t* ws, int64_t ws_bytes, const int32_t* d_offs, int32_t E,
                                   int64_t M, int64_t N, int64_t K, uint16_t* y, void* work,
                                   int64_t work_bytes, void* stream) {
  mxf8_status s = check_gemm_args({xq, xs, xs_bytes, wq, ws, ws_bytes, d_offs, E, M, N, K, y, work, work_bytes});
  if (s != MXF8_OK) return s;
  if (xs_bytes < mxfp8_rowwise_scale_bytes(M, K, E) || ws_bytes < mxfp8_rowwise_scale_bytes(E * N, K, 1))
    return MXF8_ERR_INVALID_ARG;
  if ((s = check_device()) != MXF8_OK) return s;
  if (M == 0) return cudaMemsetAsync(work, 0, sizeof(int32_t), static_cast<cudaStream_t>(stream)) == cudaSuccess
                         ? MXF8_OK : cuda_fail(cudaGetLastError(), "cudaMemsetAsync(status)");
  mxf8::GemmArgs g{};
  g.mode = mxf8::kFwd; g.E = E; g.M = M; g.N = N; g.K = K; g.offs = d_offs;
  g.a = xq; g.lda = K; g.a_rows = M; g.a_cols = K;
  g.b = wq; g.ldb = K; g.b_rows = E * N; g.b_cols = K;
  g.sfa = xs; g.sfa_pitch = cdiv(K, 128); g.sfa_atoms = xs_bytes / 512;
  g.sfb = ws; g.sfb_pitch = cdiv(K, 128); g.sfb_atoms = ws_bytes / 512;
  g.out = y;
  return run_gemm(g, work, stream);
}

mxf8_status mxfp8_grouped_gemm_dgrad(const uint8_t* dyq, const uint8_t* dys, int64_t dys_bytes,
                                     const uint8_t* wqT, const uint8_t* wsT, int64_t wsT_bytes,
                                     const int32_t* d_offs, int32_t E, int64_t M, int64_t N, int64_t K,
                                     uint16_t* dx, void* work, int64_t work_bytes, void* stream) {
  mxf8_status s =
      check_gemm_args({dyq, dys, dys_bytes, wqT, wsT, wsT_bytes, d_offs, E, M, N, K, dx, work, work_bytes});
  if (s != MXF8_OK) return s;
  if (dys_bytes < mxfp8_rowwise_scale_bytes(M, N, E) || wsT_bytes < mxfp8_colwise_scale_bytes(E * N, K, 1))
    return MXF8_ERR_INVALID_ARG;
  if ((s = check_device()) != MXF8_OK) return s;
  if (M == 0) return cudaMemsetAsync(work, 0, sizeof(int32_t), static_cast<cudaStream_t>(stream)) == cudaSuccess
                         ? MXF8_OK : cuda_fail(cudaGetLastError(), "cudaMemsetAsync(status)");
  const int64_t ldw = mxfp8_colwise_ld(E * N, 1);
  mxf8::GemmArgs g{};
  g.mode = mxf8::kDgrad; g.E = E; g.M = M; g.N = N; g.K = K; g.offs = d_offs;
  g.a = dyq; g.lda = N; g.a_rows = M; g.a_cols = N;
  g.b = wqT; g.ldb = ldw; g.b_rows = K; g.b_cols = ldw;
  g.sfa = dys; g.sfa_pitch = cdiv(N, 128); g.sfa_atoms = dys_bytes / 512;
  g.sfb = wsT; g.sfb_pitch = mxfp8_colwise_pitch(E * N, 1); g.sfb_atoms = wsT_bytes / 512;
  g.out = dx;
  return run_gemm(g, work, stream);
}

mxf8_status mxfp8_grouped_gemm_wgrad(const uint8_t* dyqT, const uint8_t* dysT, int64_t dysT_bytes,
                                     const uint8_t* xqT, const uint8_t* xsT, int64_t xsT_bytes,
                                     const int32_t* d_offs, int32_t E, int64_t M, int64_t N, int64_t K,
                                     uint16_t* dw, void* work, int64_t work_bytes, void* stream) {
  mxf8_status s =
      check_gemm_args({dyqT, dysT, dysT_bytes, xqT, xsT, xsT_bytes, d_offs, E, M, N, K, dw, work, work_bytes});
  if (s != MXF8_OK) return s;
  if (dysT_bytes < mxfp8_colwise_scale_bytes(M, N, E) || xsT_bytes < mxfp8_colwise_scale_bytes(M, K, E))
    return MXF8_ERR_INVALID_ARG;
  if ((s = check_device()) != MXF8_OK) return s;
  const int64_t ldt = mxfp8_colwise_ld(M, E);
  mxf8::GemmArgs g{};
  g.mode = mxf8::kWgrad; g.E = E; g.M = M; g.N = N; g.K = K; g.offs = d_offs;
  g.a = dyqT; g.lda = ldt; g.a_rows = N; g.a_cols = ldt;
  g.b = xqT; g.ldb = ldt; g.b_rows = K; g.b_cols = ldt;
  const int64_t pitch = mxfp8_colwise_pitch(M, E);
  g.sfa = dysT; g.sfa_pitch = pitch; g.sfa_atoms = dysT_bytes / 512;
  g.sfb = xsT; g.sfb_pitch = pitch; g.sfb_atoms = xsT_bytes / 512;
  g.out = dw;
  if (g.sfa_atoms < 1 || g.sfb_atoms < 1) {
    // M = 0: no scale atoms exist; point at the (unread) code buffers instead.
    g.sfa = dyqT; g.sfb = xqT; g.sfa_atoms = g.sfb_atoms = 1;
  }
  return run_gemm(g, work, stream);
}

mxf8_status mxfp8_grouped_gemm_fwd_quant(const uint8_t* xq, const uint8_t* xs, int64_t xs_bytes, const uint8_t* wq,
                                         const uint8_t* ws, int64_t ws_bytes, const int32_t* d_offs, int32_t E,
                                         int64_t M, int64_t N, int64_t K, uint16_t* y, uint8_t* q, uint8_t* scales,
                                         int64_t scale_bytes, uint8_t* qT, int64_t ldT, uint8_t* scalesT,
                                         int64_t scaleT_bytes, void* work, int64_t work_bytes, void* stream) {
  // The output pointer check of the plain GEMM applies to whichever output exists.
  const void* any_out = y ? static_cast<const void*>(y) : (q ? static_cast<const void*>(q) : qT);
  mxf8_status s = check_gemm_args({xq, xs, xs_bytes, wq, ws, ws_bytes, d_offs, E, M, N, K, any_out, work, work_bytes});
  if (s != MXF8_OK) return s;
  if (xs_bytes < mxfp8_rowwise_scale_bytes(M, K, E) || ws_bytes < mxfp8_rowwise_scale_bytes(E * N, K, 1))
    return MXF8_ERR_INVALID_ARG;
  mxf8::GemmArgs g{};
  g.mode = mxf8::kFwd; g.E = E; g.M = M; g.N = N; g.K = K; g.offs = d_offs;
  if ((s = attach_quant_outputs(g, N, y, q, scales, scale_bytes, qT, ldT, scalesT, scaleT_bytes)) != MXF8_OK)
    return s;
  if ((s = check_device()) != MXF8_OK) return s;
  if (M == 0) return cudaMemsetAsync(work, 0, sizeof(int32_t), static_cast<cudaStream_t>(stream)) == cudaSuccess
                         ? MXF8_OK : cuda_fail(cudaGetLastError(), "cudaMemsetAsync(status)");
  g.a = xq; g.lda = K; g.a_rows = M; g.a_cols = K;
  g.b = wq; g.ldb = K; g.b_rows = E * N; g.b_cols = K;
  g.sfa = xs; g.sfa_pitch = cdiv(K, 128); g.sfa_atoms = xs_bytes / 512;
  g.sfb = ws; g.sfb_pitch = cdiv(K, 128); g.sfb_atoms = ws_bytes / 512;
  g.out = y;
  return run_gemm(g, work, stream);
}

mxf8_status mxfp8_grouped_gemm_fwd_swiglu(const uint8_t* xq, const uint8_t* xs, int64_t xs_bytes, const uint8_t* wq,
                                          const uint8_t* ws, int64_t ws_bytes, const int32_t* d_offs, int32_t E,
                                          int64_t M, int64_t N, int64_t K, uint16_t* h, uint8_t* q, uint8_t* scales,
                                          int64_t scale_bytes, uint8_t* qT, int64_t ldT, uint8_t* scalesT,
                                          int64_t scaleT_bytes, void* work, int64_t work_bytes, void* stream) {
  const void* any_out = h ? static_cast<const void*>(h) : (q ? static_cast<const void*>(q) : qT);
  mxf8_status s = check_gemm_args({xq, xs, xs_bytes, wq, ws, ws_bytes, d_offs, E, M, N, K, any_out, work, work_bytes});
  if (s != MXF8_OK) return s;
  if (N % 256 != 0) return MXF8_ERR_INVALID_ARG;   // gate and up halves in whole 128-column tiles
  if (xs_bytes < mxfp8_rowwise_scale_bytes(M, K, E) || ws_bytes < mxfp8_rowwise_scale_bytes(E * N, K, 1))
    return MXF8_ERR_INVALID_ARG;
  mxf8::GemmArgs g{};
  g.mode = mxf8::kFwd; g.E = E; g.M = M; g.N = N; g.K = K; g.offs = d_offs;
  g.swiglu = true;
  if ((s = attach_quant_outputs(g, N / 2, h, q, scales, scale_bytes, qT, ldT, scalesT, scaleT_bytes)) != MXF8_OK)
    return s;
  if ((s = check_device()) != MXF8_OK) return s;
  if (M == 0) return cudaMemsetAsync(work, 0, sizeof(int32_t), static_cast<cudaStream_t>(stream)) == cudaSuccess
                         ? MXF8_OK : cuda_fail(cudaGetLastError(), "cudaMemsetAsync(status)");
  g.a = xq; g.lda = K; g.a_rows = M; g.a_cols = K;
  g.b = wq; g.ldb = K; g.b_rows = E * N; g.b_cols = K;
  g.sfa = xs; g.sfa_pitch = cdiv(K, 128); g.sfa_atoms = xs_bytes / 512;
  g.sfb = ws; g.sfb_pitch = cdiv(K, 128); g.sfb_atoms = ws_bytes / 512;
  g.out = h;
  return run_gemm(g, work, stream);
}

mxf8_status mxfp8_grouped_gemm_dgrad_quant(const uint8_t* dyq, const uint8_t* dys, int64_t dys_bytes,
                                           const uint8_t* wqT, const uint8_t* wsT, int64_t wsT_bytes,
                                           const int32_t* d_offs, int32_t E, int64_t M, int64_t N, int64_t K,
                                           uint16_t* dx, uint8_t* q, uint8_t* scales, int64_t scale_bytes,
                                           uint8_t* qT, int64_t ldT, uint8_t* scalesT, int64_t scaleT_bytes,
                                           void* work, int64_t work_bytes, void* stream) {
  const void* any_out = dx ? static_cast<const void*>(dx) : (q ? static_cast<const void*>(q) : qT);
  mxf8_status s =
      check_gemm_args({dyq, dys, dys_bytes, wqT, wsT, wsT_bytes, d_offs, E, M, N, K, any_out, work, work_bytes});
  if (s != MXF8_OK) return s;
  if (dys_bytes < mxfp8_rowwise_scale_bytes(M, N, E) || wsT_bytes < mxfp8_colwise_scale_bytes(E * N, K, 1))
    return MXF8_ERR_INVALID_ARG;
  mxf8::GemmArgs g{};
  g.mode = mxf8::kDgrad; g.E = E; g.M = M; g.N = N; g.K = K; g.offs = d_offs;
  if ((s = attach_quant_outputs(g, K, dx, q, scales, scale_bytes, qT, ldT, scalesT, scaleT_bytes)) != MXF8_OK)
    return s;
  if ((s = check_device()) != MXF8_OK) return s;
  if (M == 0) return cudaMemsetAsync(work, 0, sizeof(int32_t), static_cast<cudaStream_t>(stream)) == cudaSuccess
                         ? MXF8_OK : cuda_fail(cudaGetLastError(), "cudaMemsetAsync(status)");
  const int64_t ldw = mxfp8_colwise_ld(E * N, 1);
  g.a = dyq; g.lda = N; g.a_rows = M; g.a_cols = N;
  g.b = wqT; g.ldb = ldw; g.b_rows = K; g.b_cols = ldw;
  g.sfa = dys; g.sfa_pitch = cdiv(N, 128); g.sfa_atoms = dys_bytes / 512;
  g.sfb = wsT; g.sfb_pitch = mxfp8_colwise_pitch(E * N, 1); g.sfb_atoms = wsT_bytes / 512;
  g.out = dx;
  return run_gemm(g, work, stream);
}

int64_t mxfp8_moe_plan_workspace_bytes(int64_t num_tokens, int32_t top_k, int32_t num_experts) {
  if (num_tokens < 0 || top_k < 1 || num_experts < 1) return 0;
  const int64_t pairs = num_tokens * top_k;
  return kWorkspaceBytes + round_up(pairs * 4, 256) +
         round_up(mxf8::moe_plan_chunks(pairs) * int64_t(num_experts) * 4, 256);
}

mxf8_status mxfp8_moe_plan(const int32_t* idx, int64_t num_tokens, int32_t top_k, int32_t num_experts,
                           int32_t* offs, int32_t* perm, int32_t* inv, void* work, int64_t work_bytes,
                           void* stream) {
  if (num_tokens < 0 || top_k < 1 || num_experts < 1 || num_experts > MXF8_MOE_MAX_EXPERTS)
    return MXF8_ERR_INVALID_ARG;
  const int64_t pairs = num_tokens * top_k;
  if (pairs >= (int64_t(1) << 31)) return MXF8_ERR_INVALID_ARG;
  if (!offs || !work || (pairs > 0 && (!idx || !perm || !inv))) return MXF8_ERR_INVALID_ARG;
  if (work_bytes < mxfp8_moe_plan_workspace_bytes(num_tokens, top_k, num_experts)) return MXF8_ERR_INVALID_ARG;
  if (!aligned16(work)) return MXF8_ERR_ALIGNMENT;
  mxf8_status s = check_device();
  if (s != MXF8_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(work);
  int32_t* status = reinterpret_cast<int32_t*>(w);
  int32_t* rank = reinterpret_cast<int32_t*>(w + kWorkspaceBytes);
  int32_t* hist = reinterpret_cast<int32_t*>(w + kWorkspaceBytes + round_up(pairs * 4, 256));
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int32_t), st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(status)");
  e = mxf8::launch_moe_plan(idx, num_tokens, top_k, num_experts, offs, perm, inv, status, rank, hist, st);
  return e == cudaSuccess ? MXF8_OK : cuda_fail(e, "moe_plan launch");
}

mxf8_status mxfp8_permute_quantize_dual(const uint16_t* x, int64_t num_tokens, int64_t cols, const int32_t* perm,
                                        int64_t rows, const int32_t* d_offs, int32_t num_groups, uint8_t* q,
                                        uint8_t* scales, int64_t scale_bytes, uint8_t* qT, int64_t ldT,
                                        uint8_t* scalesT, int64_t scaleT_bytes, void* stream) {
  if (num_tokens < 0 || (rows > 0 && (!x || !perm)) || !d_offs) return MXF8_ERR_INVALID_ARG;
  mxf8_status s = check_quant_args(x, rows, cols, num_groups, q, scales, scale_bytes,
                                   mxfp8_rowwise_scale_bytes(rows, cols, num_groups));
  if (s != MXF8_OK) return s;
  s = check_quant_args(x, rows, cols, num_groups, qT, scalesT, scaleT_bytes,
                       mxfp8_colwise_scale_bytes(rows, cols, num_groups));
  if (s != MXF8_OK) return s;
  if (ldT != mxfp8_colwise_ld(rows, num_groups)) return MXF8_ERR_INVALID_ARG;
  if ((s = check_device()) != MXF8_OK) return s;
  cudaError_t e = mxf8::launch_permute_quantize_dual(x, num_tokens, cols, perm, rows, d_offs, num_groups, q, scales,
                                                     qT, ldT, scalesT, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MXF8_OK : cuda_fail(e, "permute_quantize_dual launch");
}

mxf8_status mxfp8_moe_combine(const uint16_t* yp, int64_t rows, int64_t cols, const int32_t* inv, const float* w,
                              int64_t num_tokens, int32_t top_k, uint16_t* y, void* stream) {
  if (rows < 0 || cols <= 0 || cols % 8 != 0 || num_tokens < 0 || top_k < 1) return MXF8_ERR_INVALID_ARG;
  if (num_tokens > 0 && (!inv || !w || !y || (rows > 0 && !yp))) return MXF8_ERR_INVALID_ARG;
  if (!aligned16(yp) || !aligned16(y)) return MXF8_ERR_ALIGNMENT;
  mxf8_status s = check_device();
  if (s != MXF8_OK) return s;
  cudaError_t e = mxf8::launch_moe_combine(yp, rows, cols, inv, w, num_tokens, top_k, y,
                                           static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MXF8_OK : cuda_fail(e, "moe_combine launch");
}

int64_t mxfp8_ep_record_bytes(int64_t cols) {
  if (cols <= 0 || cols % 32 != 0) return 0;
  return mxf8::ep_record_stride(cols);
}

int64_t mxfp8_ep_plan_workspace_bytes(int64_t num_tokens, int32_t num_ranks) {
  if (num_tokens < 0 || num_ranks < 1 || num_ranks > MXF8_EP_MAX_RANKS) return 0;
  // status word | first record and first pair of each rank | per-chunk counts (records, pairs per rank)
  return kWorkspaceBytes + 2 * MXF8_EP_MAX_RANKS * 4 +
         round_up(mxf8::ep_plan_chunks(num_tokens) * 2 * num_ranks * 4, 256);
}

mxf8_status mxfp8_ep_plan(const int32_t* idx, int64_t num_tokens, int32_t top_k, int32_t num_experts,
                          int32_t num_ranks, int32_t* counts, int32_t* rec_token, int32_t* pair_expert,
                          int32_t* pair_rec, int32_t* ret_pos, void* work, int64_t work_bytes, void* stream) {
  if (num_tokens < 0 || top_k < 1 || top_k > MXF8_EP_MAX_TOP_K) return MXF8_ERR_INVALID_ARG;
  if (num_ranks < 1 || num_ranks > MXF8_EP_MAX_RANKS || num_experts < 1 || num_experts % num_ranks != 0)
    return MXF8_ERR_INVALID_ARG;
  if (num_tokens * top_k >= (int64_t(1) << 31)) return MXF8_ERR_INVALID_ARG;
  if (!counts || !work || (num_tokens > 0 && (!idx || !rec_token || !pair_expert || !pair_rec || !ret_pos)))
    return MXF8_ERR_INVALID_ARG;
  if (work_bytes < mxfp8_ep_plan_workspace_bytes(num_tokens, num_ranks)) return MXF8_ERR_INVALID_ARG;
  if (!aligned16(work)) return MXF8_ERR_ALIGNMENT;
  mxf8_status s = check_device();
  if (s != MXF8_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(work);
  int32_t* status = reinterpret_cast<int32_t*>(w);
  int32_t* bases = reinterpret_cast<int32_t*>(w + kWorkspaceBytes);
  int32_t* hist = reinterpret_cast<int32_t*>(w + kWorkspaceBytes + 2 * MXF8_EP_MAX_RANKS * 4);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int32_t), st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(status)");
  e = mxf8::launch_ep_plan(idx, num_tokens, top_k, num_experts, num_ranks, counts, rec_token, pair_expert, pair_rec,
                           ret_pos, status, bases, hist, st);
  return e == cudaSuccess ? MXF8_OK : cuda_fail(e, "ep_plan launch");
}

mxf8_status mxfp8_ep_pack(const uint16_t* x, int64_t num_tokens, int64_t cols, const int32_t* rec_token,
                          int64_t num_records, uint8_t* records, void* stream) {
  if (num_tokens < 0 || num_records < 0 || cols <= 0 || cols % 32 != 0) return MXF8_ERR_INVALID_ARG;
  if (num_records > (int64_t(1) << 31) - 1 || cols > (int64_t(1) << 30)) return MXF8_ERR_INVALID_ARG;
  if (num_records > 0 && (!rec_token || !records || (num_tokens > 0 && !x))) return MXF8_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(records)) return MXF8_ERR_ALIGNMENT;
  mxf8_status s = check_device();
  if (s != MXF8_OK) return s;
  cudaError_t e = mxf8::launch_ep_pack(x, num_tokens, cols, rec_token, num_records, records,
                                       static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MXF8_OK : cuda_fail(e, "ep_pack launch");
}

mxf8_status mxfp8_ep_unpack(const uint8_t* records, int64_t num_records, int64_t cols, const int32_t* pair_rec,
                            const int32_t* src_base, int32_t num_sources, const int32_t* perm, int64_t rows,
                            const int32_t* d_offs, int32_t num_groups, uint8_t* q, uint8_t* scales,
                            int64_t scale_bytes, void* stream) {
  if (num_records < 0 || num_sources < 1 || num_sources > MXF8_EP_MAX_RANKS) return MXF8_ERR_INVALID_ARG;
  if (!d_offs || !src_base || (rows > 0 && (!pair_rec || !perm || (num_records > 0 && !records))))
    return MXF8_ERR_INVALID_ARG;
  // the rows' codes and scales follow the rowwise quantiser's rules and layout
  mxf8_status s = check_quant_args(nullptr, 0, cols, num_groups, q, scales, scale_bytes,
                                   mxfp8_rowwise_scale_bytes(rows, cols, num_groups));
  if (s != MXF8_OK) return s;
  if (rows < 0 || rows > (int64_t(1) << 31) - 1 || (rows > 0 && !q)) return MXF8_ERR_INVALID_ARG;
  if (!aligned16(records)) return MXF8_ERR_ALIGNMENT;
  if ((s = check_device()) != MXF8_OK) return s;
  cudaError_t e = mxf8::launch_ep_unpack(records, num_records, cols, pair_rec, src_base, num_sources, perm, rows,
                                         d_offs, num_groups, q, scales, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MXF8_OK : cuda_fail(e, "ep_unpack launch");
}

mxf8_status mxfp8_gather_rows(const void* src, int64_t src_rows, int64_t row_bytes, const int32_t* idx, int64_t n,
                              void* dst, void* stream) {
  if (src_rows < 0 || n < 0 || row_bytes <= 0 || row_bytes % 16 != 0) return MXF8_ERR_INVALID_ARG;
  if (n > 0 && (!idx || !dst || (src_rows > 0 && !src))) return MXF8_ERR_INVALID_ARG;
  if (!aligned16(src) || !aligned16(dst)) return MXF8_ERR_ALIGNMENT;
  mxf8_status s = check_device();
  if (s != MXF8_OK) return s;
  cudaError_t e = mxf8::launch_gather_rows(src, src_rows, row_bytes, idx, n, dst, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MXF8_OK : cuda_fail(e, "gather_rows launch");
}

int64_t mxfp8_nvfp4_rowwise_scale_bytes(int64_t rows, int64_t cols, int32_t num_groups) {
  if (rows < 0 || cols <= 0 || num_groups < 1) return 0;
  return blocks128_bound(rows, num_groups) * cdiv(cols, 64) * 512;
}

int64_t mxfp8_nvfp4_colwise_pitch(int64_t rows, int32_t num_groups) {
  if (rows <= 0 || num_groups < 1) return 0;
  return cdiv(rows, 64) + num_groups - 1;
}

int64_t mxfp8_nvfp4_colwise_scale_bytes(int64_t rows, int64_t cols, int32_t num_groups) {
  if (rows < 0 || cols <= 0 || num_groups < 1) return 0;
  return cdiv(cols, 128) * mxfp8_nvfp4_colwise_pitch(rows, num_groups) * 512;
}

int64_t mxfp8_nvfp4_colwise_ld(int64_t rows, int32_t num_groups) {
  if (rows < 0 || num_groups < 1) return 0;
  const int64_t ld = round_up(round_up(rows, 32) + 32 * int64_t(num_groups - 1), 256);
  return ld < 256 ? 256 : ld;
}

mxf8_status mxfp8_nvfp4_amax(const uint16_t* x, int64_t n, float* amax, void* stream) {
  if (n < 0 || !amax || (n > 0 && !x)) return MXF8_ERR_INVALID_ARG;
  if (!aligned16(x)) return MXF8_ERR_ALIGNMENT;
  mxf8_status s = check_device();
  if (s != MXF8_OK) return s;
  cudaError_t e = mxf8::launch_nvfp4_amax(x, n, amax, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MXF8_OK : cuda_fail(e, "nvfp4_amax launch");
}

mxf8_status mxfp8_nvfp4_quantize_rowwise(const uint16_t* x, int64_t rows, int64_t cols, const int32_t* d_offs,
                                         int32_t num_groups, const float* amax, uint8_t* q, uint8_t* scales,
                                         int64_t scale_bytes, void* stream) {
  if (!amax || cols % 64 != 0) return MXF8_ERR_INVALID_ARG;
  mxf8_status s = check_quant_args(x, rows, cols, num_groups, q, scales, scale_bytes,
                                   mxfp8_nvfp4_rowwise_scale_bytes(rows, cols, num_groups));
  if (s != MXF8_OK) return s;
  if ((s = check_device()) != MXF8_OK) return s;
  cudaError_t e = mxf8::launch_nvfp4_rowwise(x, rows, cols, d_offs, num_groups, amax, q, scales,
                                             static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MXF8_OK : cuda_fail(e, "nvfp4_rowwise launch");
}

mxf8_status mxfp8_nvfp4_quantize_colwise(const uint16_t* x, int64_t rows, int64_t cols, const int32_t* d_offs,
                                         int32_t num_groups, const float* amax, uint8_t* qT, int64_t ldT,
                                         uint8_t* scalesT, int64_t scale_bytes, void* stream) {
  if (!amax || cols % 64 != 0) return MXF8_ERR_INVALID_ARG;
  mxf8_status s = check_quant_args(x, rows, cols, num_groups, qT, scalesT, scale_bytes,
                                   mxfp8_nvfp4_colwise_scale_bytes(rows, cols, num_groups));
  if (s != MXF8_OK) return s;
  if (ldT != mxfp8_nvfp4_colwise_ld(rows, num_groups)) return MXF8_ERR_INVALID_ARG;
  if ((s = check_device()) != MXF8_OK) return s;
  cudaError_t e = mxf8::launch_nvfp4_colwise(x, rows, cols, d_offs, num_groups, amax, qT, ldT, scalesT,
                                             static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MXF8_OK : cuda_fail(e, "nvfp4_colwise launch");
}

mxf8_status mxfp8_nvfp4_grouped_gemm_fwd(const uint8_t* xq, const uint8_t* xs, int64_t xs_bytes, const float* x_amax,
                                         const uint8_t* wq, const uint8_t* ws, int64_t ws_bytes, const float* w_amax,
                                         const int32_t* d_offs, int32_t E, int64_t M, int64_t N, int64_t K,
                                         uint16_t* y, void* work, int64_t work_bytes, void* stream) {
  mxf8_status s = check_gemm_args({xq, xs, xs_bytes, wq, ws, ws_bytes, d_offs, E, M, N, K, y, work, work_bytes});
  if (s != MXF8_OK) return s;
  if (!x_amax || !w_amax || K % 64 != 0) return MXF8_ERR_INVALID_ARG;
  if (xs_bytes < mxfp8_nvfp4_rowwise_scale_bytes(M, K, E) || ws_bytes < mxfp8_nvfp4_rowwise_scale_bytes(E * N, K, 1))
    return MXF8_ERR_INVALID_ARG;
  if ((s = check_device()) != MXF8_OK) return s;
  if (M == 0) return cudaMemsetAsync(work, 0, sizeof(int32_t), static_cast<cudaStream_t>(stream)) == cudaSuccess
                         ? MXF8_OK : cuda_fail(cudaGetLastError(), "cudaMemsetAsync(status)");
  mxf8::GemmArgs g{};
  g.mode = mxf8::kFwd; g.E = E; g.M = M; g.N = N; g.K = K; g.offs = d_offs;
  g.fp4 = true; g.amax_a = x_amax; g.amax_b = w_amax;
  g.a = xq; g.lda = K / 2; g.a_rows = M; g.a_cols = K / 2;
  g.b = wq; g.ldb = K / 2; g.b_rows = E * N; g.b_cols = K / 2;
  g.sfa = xs; g.sfa_pitch = cdiv(K, 64); g.sfa_atoms = xs_bytes / 512;
  g.sfb = ws; g.sfb_pitch = cdiv(K, 64); g.sfb_atoms = ws_bytes / 512;
  g.out = y;
  return run_gemm(g, work, stream);
}

mxf8_status mxfp8_nvfp4_grouped_gemm_dgrad(const uint8_t* dyq, const uint8_t* dys, int64_t dys_bytes,
                                           const float* dy_amax, const uint8_t* wqT, const uint8_t* wsT,
                                           int64_t wsT_bytes, const float* w_amax, const int32_t* d_offs, int32_t E,
                                           int64_t M, int64_t N, int64_t K, uint16_t* dx, void* work,
                                           int64_t work_bytes, void* stream) {
  mxf8_status s =
      check_gemm_args({dyq, dys, dys_bytes, wqT, wsT, wsT_bytes, d_offs, E, M, N, K, dx, work, work_bytes});
  if (s != MXF8_OK) return s;
  if (!dy_amax || !w_amax || K % 64 != 0) return MXF8_ERR_INVALID_ARG;
  if (dys_bytes < mxfp8_nvfp4_rowwise_scale_bytes(M, N, E) ||
      wsT_bytes < mxfp8_nvfp4_colwise_scale_bytes(E * N, K, 1))
    return MXF8_ERR_INVALID_ARG;
  if ((s = check_device()) != MXF8_OK) return s;
  if (M == 0) return cudaMemsetAsync(work, 0, sizeof(int32_t), static_cast<cudaStream_t>(stream)) == cudaSuccess
                         ? MXF8_OK : cuda_fail(cudaGetLastError(), "cudaMemsetAsync(status)");
  const int64_t ldw = mxfp8_nvfp4_colwise_ld(E * N, 1) / 2;   // bytes
  mxf8::GemmArgs g{};
  g.mode = mxf8::kDgrad; g.E = E; g.M = M; g.N = N; g.K = K; g.offs = d_offs;
  g.fp4 = true; g.amax_a = dy_amax; g.amax_b = w_amax;
  g.a = dyq; g.lda = N / 2; g.a_rows = M; g.a_cols = N / 2;
  g.b = wqT; g.ldb = ldw; g.b_rows = K; g.b_cols = ldw;
  g.sfa = dys; g.sfa_pitch = cdiv(N, 64); g.sfa_atoms = dys_bytes / 512;
  g.sfb = wsT; g.sfb_pitch = mxfp8_nvfp4_colwise_pitch(E * N, 1); g.sfb_atoms = wsT_bytes / 512;
  g.out = dx;
  return run_gemm(g, work, stream);
}

mxf8_status mxfp8_nvfp4_grouped_gemm_wgrad(const uint8_t* dyqT, const uint8_t* dysT, int64_t dysT_bytes,
                                           const float* dy_amax, const uint8_t* xqT, const uint8_t* xsT,
                                           int64_t xsT_bytes, const float* x_amax, const int32_t* d_offs, int32_t E,
                                           int64_t M, int64_t N, int64_t K, uint16_t* dw, void* work,
                                           int64_t work_bytes, void* stream) {
  mxf8_status s =
      check_gemm_args({dyqT, dysT, dysT_bytes, xqT, xsT, xsT_bytes, d_offs, E, M, N, K, dw, work, work_bytes});
  if (s != MXF8_OK) return s;
  if (!dy_amax || !x_amax || K % 64 != 0) return MXF8_ERR_INVALID_ARG;
  if (dysT_bytes < mxfp8_nvfp4_colwise_scale_bytes(M, N, E) || xsT_bytes < mxfp8_nvfp4_colwise_scale_bytes(M, K, E))
    return MXF8_ERR_INVALID_ARG;
  if ((s = check_device()) != MXF8_OK) return s;
  const int64_t ldt = mxfp8_nvfp4_colwise_ld(M, E) / 2;   // bytes
  mxf8::GemmArgs g{};
  g.mode = mxf8::kWgrad; g.E = E; g.M = M; g.N = N; g.K = K; g.offs = d_offs;
  g.fp4 = true; g.amax_a = dy_amax; g.amax_b = x_amax;
  g.a = dyqT; g.lda = ldt; g.a_rows = N; g.a_cols = ldt;
  g.b = xqT; g.ldb = ldt; g.b_rows = K; g.b_cols = ldt;
  const int64_t pitch = mxfp8_nvfp4_colwise_pitch(M, E);
  g.sfa = dysT; g.sfa_pitch = pitch; g.sfa_atoms = dysT_bytes / 512;
  g.sfb = xsT; g.sfb_pitch = pitch; g.sfb_atoms = xsT_bytes / 512;
  g.out = dw;
  if (g.sfa_atoms < 1 || g.sfb_atoms < 1) {
    // M = 0: no scale atoms exist; point at the (unread) code buffers instead.
    g.sfa = dyqT; g.sfb = xqT; g.sfa_atoms = g.sfb_atoms = 1;
  }
  return run_gemm(g, work, stream);
}

mxf8_status mxfp8_get_status(const void* work, void* stream, int32_t* device_status) {
  if (!work || !device_status) return MXF8_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  e = cudaMemcpy(device_status, work, sizeof(int32_t), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(status)");
  return MXF8_OK;
}

const char* mxfp8_status_string(int32_t status) {
  switch (status) {
    case MXF8_OK: return "ok";
    case MXF8_ERR_INVALID_ARG: return "invalid argument";
    case MXF8_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case MXF8_ERR_UNSUPPORTED: return "device is not sm_100";
    case MXF8_ERR_CUDA: return "CUDA error";
    case MXF8_ERR_BAD_OFFSETS: return "group offsets are not a valid prefix";
    case MXF8_ERR_TIMEOUT: return "device pipeline wait timed out";
    case MXF8_ERR_BAD_ROUTING: return "an expert id is outside [0, num_experts)";
    default: return "unknown status";
  }
}

const char* mxfp8_last_cuda_error(void) { return g_last_error; }

int32_t mxfp8_device_supported(void) { return check_device() == MXF8_OK ? 1 : 0; }

}  // extern "C"
