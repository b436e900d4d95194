// noalloc.cu -- forward grouped GEMM for callers that cannot allocate device
// memory.
//
// The ordinary entry points take a caller-allocated workspace.  Some callers
// cannot provide one: a plugin running inside a host engine that owns the
// whole device-memory budget and forbids its components to call cudaMalloc,
// or a latency-critical loop where a cudaMalloc (which may synchronise the
// device) is not acceptable.  For them this file keeps the scratch in a
// static device array that lives in the library image: every GPU that loads
// the library holds MXF8_NOALLOC_SCRATCH_BYTES of it until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "launch.h"
#include "mxfp8.h"

static_assert(MXF8_NOALLOC_SCRATCH_BYTES >= mxf8::kGemmWorkspaceBytes,
              "the static scratch must hold a grouped GEMM workspace");

namespace {

// The scratch itself.  In host code this name is only a host-side stand-in
// for the device symbol, never a device address: its device address is
// looked up once per device with cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MXF8_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device (looked up on the
// first call made with that device current).  Returns nullptr on failure.
void* scratch_for_current_device(cudaError_t* err) {
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (*err != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" mxf8_status mxfp8_grouped_gemm_fwd_noalloc(const uint8_t* xq, const uint8_t* xs, int64_t xs_bytes,
                                                      const uint8_t* wq, const uint8_t* ws, int64_t ws_bytes,
                                                      const int32_t* d_offs, int32_t E, int64_t M, int64_t N,
                                                      int64_t K, uint16_t* y, int32_t* host_status,
                                                      void* stream) {
  if (mxfp8_workspace_bytes(E, M, N, K) > MXF8_NOALLOC_SCRATCH_BYTES) return MXF8_ERR_INVALID_ARG;
  cudaError_t err = cudaSuccess;
  void* scratch = scratch_for_current_device(&err);
  if (!scratch) {
    mxf8::record_cuda_error(err, "mxfp8_grouped_gemm_fwd_noalloc: scratch address lookup", nullptr);
    return MXF8_ERR_CUDA;
  }
  // The forward entry point clears the status word in the scratch before its
  // launch, so the last call's contents never leak into this one.
  mxf8_status s = mxfp8_grouped_gemm_fwd(xq, xs, xs_bytes, wq, ws, ws_bytes, d_offs, E, M, N, K, y, scratch,
                                         MXF8_NOALLOC_SCRATCH_BYTES, stream);
  if (s != MXF8_OK || !host_status) return s;
  return mxfp8_get_status(scratch, stream, host_status);
}
