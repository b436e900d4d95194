// ep_launch.h -- host launchers of the expert-parallel dispatch kernels
// (ep.cu); the argument checks live in api.cu.
#pragma once
#include <cuda_runtime.h>

#include <cstdint>

namespace mxf8 {

int64_t ep_plan_chunks(int64_t T);
int64_t ep_record_stride(int64_t C);
cudaError_t launch_ep_plan(const int32_t* idx, int64_t T, int32_t k, int32_t E, int32_t P, int32_t* counts,
                           int32_t* rec_token, int32_t* pair_expert, int32_t* pair_rec, int32_t* ret_pos,
                           int32_t* status, int32_t* bases, int32_t* hist, cudaStream_t stream);
cudaError_t launch_ep_pack(const uint16_t* x, int64_t T, int64_t C, const int32_t* rec_token, int64_t R,
                           uint8_t* records, cudaStream_t stream);
cudaError_t launch_ep_unpack(const uint8_t* records, int64_t R, int64_t C, const int32_t* pair_rec,
                             const int32_t* src_base, int32_t P, const int32_t* perm, int64_t rows,
                             const int32_t* offs, int32_t G, uint8_t* q, uint8_t* sf, cudaStream_t stream);
cudaError_t launch_gather_rows(const void* src, int64_t src_rows, int64_t row_bytes, const int32_t* idx, int64_t n,
                               void* dst, cudaStream_t stream);

}  // namespace mxf8
