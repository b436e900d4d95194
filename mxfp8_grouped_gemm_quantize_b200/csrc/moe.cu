// moe.cu -- the steps around the grouped GEMM of a Mixture-of-Experts layer:
// the dispatch plan (which permuted row every routed (token, slot) pair
// takes) and the weighted combine of the experts' outputs back to tokens.
// The permute itself is fused with MXFP8 quantisation in quantize.cu.
//
// The grouped GEMM consumes each expert's tokens as one contiguous run of
// rows with its real count (iitak.ru, "NVIDIA в 10 раз ускорила обучение
// моделей-«смесей экспертов» на JAX", paragraph on the Transformer Engine
// grouped GEMM); tokens travel to their experts and back through the two
// all-to-alls of opensourcebeat.com, section "Двухсторонняя атака: MXFP8 и
// DeepEP".  On one GPU those exchanges reduce to this permute and combine.
//
// Plan: a stable counting sort of the (token, slot) pairs by expert, so that
// inside an expert the pairs keep ascending (token, slot) order and the
// result is deterministic.  Three launches: (1) one warp per chunk of pairs
// walks them in order and ranks each pair among the chunk's earlier pairs of
// the same expert (warp match + shared counters), writing the chunk's
// per-expert histogram; (2) one CTA turns the histograms into per-chunk
// bases and the group offsets; (3) every pair scatters its token id.
//
// Combine: y[t] = sum over slots j of w[t, j] * yp[inv[t, j]].  Products of
// an fp32 weight and a bf16 value are exact in fp64, the sum runs in fp64 in
// slot order, and the result is rounded once to bf16 (nearest even), so the
// output is exactly the rounded fp64 sum.
#include <cuda_runtime.h>

#include <cstdint>

#include "launch.h"
#include "mxfp8.h"

namespace mxf8 {
namespace {

constexpr int kPlanChunk = 1024;   // pairs ranked by one warp
constexpr int kCombineThreads = 256;

// Pass 1.  rank[i]: earlier pairs of the same expert in i's chunk.
__global__ void __launch_bounds__(32) plan_rank_kernel(const int32_t* __restrict__ idx, int64_t n, int32_t E,
                                                       int32_t* __restrict__ rank, int32_t* __restrict__ hist,
                                                       int32_t* __restrict__ status) {
  __shared__ int32_t cnt[MXF8_MOE_MAX_EXPERTS];
  const int lane = threadIdx.x;
  for (int e = lane; e < E; e += 32) cnt[e] = 0;
  __syncwarp();
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kPlanChunk;
  const int64_t end = base + kPlanChunk < n ? base + kPlanChunk : n;
  for (int64_t i0 = base; i0 < end; i0 += 32) {
    const int64_t i = i0 + lane;
    int32_t e = i < end ? __ldg(idx + i) : -1;
    const bool bad = i < end && (e < 0 || e >= E);
    if (bad) atomicCAS(status, 0, static_cast<int32_t>(MXF8_ERR_BAD_ROUTING));
    if (bad) e = -1;
    const unsigned same = __match_any_sync(0xffffffffu, e);
    const int before = __popc(same & ((1u << lane) - 1u));
    const int32_t r = e >= 0 ? cnt[e] + before : -1;
    __syncwarp();
    if (e >= 0 && before == 0) cnt[e] += __popc(same);   // the group's lowest lane
    __syncwarp();
    if (i < end) rank[i] = r;
  }
  __syncwarp();
  for (int e = lane; e < E; e += 32) hist[static_cast<int64_t>(blockIdx.x) * E + e] = cnt[e];
}

// Pass 2 (one CTA of MXF8_MOE_MAX_EXPERTS threads): hist[c][e] becomes the
// first permuted row of chunk c's pairs of expert e; offs is the exclusive
// prefix of the per-expert totals.
__global__ void __launch_bounds__(MXF8_MOE_MAX_EXPERTS) plan_offsets_kernel(int32_t* __restrict__ hist,
                                                                            int64_t chunks, int32_t E,
                                                                            int32_t* __restrict__ offs) {
  __shared__ int32_t tot[MXF8_MOE_MAX_EXPERTS];
  const int e = threadIdx.x;
  int32_t run = 0;
  if (e < E) {
    for (int64_t c = 0; c < chunks; ++c) {
      const int32_t h = hist[c * E + e];
      hist[c * E + e] = run;
      run += h;
    }
  }
  tot[e] = e < E ? run : 0;
  __syncthreads();
  // exclusive scan over experts (Hillis-Steele on shared memory)
  for (int d = 1; d < MXF8_MOE_MAX_EXPERTS; d <<= 1) {
    const int32_t v = e >= d ? tot[e - d] : 0;
    __syncthreads();
    tot[e] += v;
    __syncthreads();
  }
  const int32_t start = e > 0 ? tot[e - 1] : 0;   // tot is now inclusive
  if (e < E) {
    offs[e] = start;
    for (int64_t c = 0; c < chunks; ++c) hist[c * E + e] += start;
  }
  if (e == E - 1) offs[E] = tot[e];
}

// Pass 3: scatter.
__global__ void plan_scatter_kernel(const int32_t* __restrict__ idx, int64_t n, int32_t k, int32_t E,
                                    const int32_t* __restrict__ rank, const int32_t* __restrict__ hist,
                                    int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int32_t e = __ldg(idx + i);
    if (e < 0 || e >= E) {
      inv[i] = -1;
      continue;
    }
    const int32_t r = hist[(i / kPlanChunk) * E + e] + rank[i];
    perm[r] = static_cast<int32_t>(i / k);
    inv[i] = r;
  }
}

// Nearest-even bf16 bits of a double (one rounding: ties to even, overflow
// to Inf, bf16 subnormals kept) by the hardware conversion; a NaN becomes the
// quiet NaN 0x7FC0 with its sign, the definition's pattern.
__device__ __forceinline__ uint16_t bf16_bits_rne(double v) {
  uint16_t r;
  asm("cvt.rn.bf16.f64 %0, %1;" : "=h"(r) : "d"(v));
  if (v != v) r = static_cast<uint16_t>(((__double_as_longlong(v) >> 48) & 0x8000) | 0x7FC0);
  return r;
}

__device__ __forceinline__ double bf16_lo(uint32_t w) { return static_cast<double>(__uint_as_float(w << 16)); }
__device__ __forceinline__ double bf16_hi(uint32_t w) { return static_cast<double>(__uint_as_float(w & 0xFFFF0000u)); }

// One thread: 8 consecutive columns of one token.
// Adds slot j's contribution w_j * yp[r_j] to the fp64 accumulators.  The
// product of an fp32 weight and a bf16 value has at most 32 significant bits,
// so it is exact in fp64 and one fused multiply-add rounds exactly as the
// separate multiply and add of the definition do.
__device__ __forceinline__ void combine_add(double (&acc)[8], double wj, const uint4& v) {
  acc[0] = __fma_rn(wj, bf16_lo(v.x), acc[0]);
  acc[1] = __fma_rn(wj, bf16_hi(v.x), acc[1]);
  acc[2] = __fma_rn(wj, bf16_lo(v.y), acc[2]);
  acc[3] = __fma_rn(wj, bf16_hi(v.y), acc[3]);
  acc[4] = __fma_rn(wj, bf16_lo(v.z), acc[4]);
  acc[5] = __fma_rn(wj, bf16_hi(v.z), acc[5]);
  acc[6] = __fma_rn(wj, bf16_lo(v.w), acc[6]);
  acc[7] = __fma_rn(wj, bf16_hi(v.w), acc[7]);
}

// Slots are summed in order 0..k-1; an unrouted slot is skipped (not added
// as zero, which would turn -0 into +0).  For top-k with k <= 8 a thread
// issues all k row loads before the sums, so k independent 16-byte loads
// are in flight instead of one dependent index -> row chain per slot.
constexpr int kCombineSlots = 8;

__global__ void __launch_bounds__(kCombineThreads) combine_kernel(
    const uint16_t* __restrict__ yp, int64_t rows, int64_t cols, const int32_t* __restrict__ inv,
    const float* __restrict__ w, int64_t T, int32_t k, uint16_t* __restrict__ y) {
  const int64_t per_row = cols / 8;
  const int64_t units = T * per_row;
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; u < units;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = u / per_row, c = (u - t * per_row) * 8;
    double acc[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
    if (k <= kCombineSlots) {
      int32_t r[kCombineSlots];
      uint4 v[kCombineSlots];
#pragma unroll
      for (int j = 0; j < kCombineSlots; ++j) {
        r[j] = j < k ? __ldg(inv + t * k + j) : -1;
        if (r[j] >= rows) r[j] = -1;                // an unrouted slot contributes nothing
      }
#pragma unroll
      for (int j = 0; j < kCombineSlots; ++j)
        v[j] = r[j] >= 0 ? __ldg(reinterpret_cast<const uint4*>(yp + static_cast<int64_t>(r[j]) * cols + c))
                         : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int j = 0; j < kCombineSlots; ++j)
        if (r[j] >= 0) combine_add(acc, static_cast<double>(__ldg(w + t * k + j)), v[j]);
    } else {
      for (int32_t j = 0; j < k; ++j) {
        const int32_t r = __ldg(inv + t * k + j);
        if (r < 0 || r >= rows) continue;
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(yp + static_cast<int64_t>(r) * cols + c));
        combine_add(acc, static_cast<double>(__ldg(w + t * k + j)), v);
      }
    }
    auto pack = [](double lo, double hi) {
      return static_cast<uint32_t>(bf16_bits_rne(lo)) | (static_cast<uint32_t>(bf16_bits_rne(hi)) << 16);
    };
    *reinterpret_cast<uint4*>(y + t * cols + c) =
        make_uint4(pack(acc[0], acc[1]), pack(acc[2], acc[3]), pack(acc[4], acc[5]), pack(acc[6], acc[7]));
  }
}

int grid_for(int64_t work, int threads) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t need = (work + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(sms) * 16;
  return static_cast<int>(need < cap ? (need > 0 ? need : 1) : cap);
}

}  // namespace

int64_t moe_plan_chunks(int64_t pairs) { return (pairs + kPlanChunk - 1) / kPlanChunk; }

cudaError_t launch_moe_plan(const int32_t* idx, int64_t T, int32_t k, int32_t E, int32_t* offs, int32_t* perm,
                            int32_t* inv, int32_t* status, int32_t* rank, int32_t* hist, cudaStream_t stream) {
  const int64_t n = T * k;
  const int64_t chunks = moe_plan_chunks(n);
  if (chunks > 0) {
    plan_rank_kernel<<<static_cast<unsigned>(chunks), 32, 0, stream>>>(idx, n, E, rank, hist, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  plan_offsets_kernel<<<1, MXF8_MOE_MAX_EXPERTS, 0, stream>>>(hist, chunks, E, offs);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || n == 0) return e;
  plan_scatter_kernel<<<grid_for(n, 256), 256, 0, stream>>>(idx, n, k, E, rank, hist, perm, inv);
  return cudaGetLastError();
}

cudaError_t launch_moe_combine(const uint16_t* yp, int64_t rows, int64_t cols, const int32_t* inv, const float* w,
                               int64_t T, int32_t k, uint16_t* y, cudaStream_t stream) {
  const int64_t units = T * (cols / 8);
  if (units == 0) return cudaSuccess;
  combine_kernel<<<grid_for(units, kCombineThreads), kCombineThreads, 0, stream>>>(yp, rows, cols, inv, w, T, k,
                                                                                   y);
  return cudaGetLastError();
}

}  // namespace mxf8
