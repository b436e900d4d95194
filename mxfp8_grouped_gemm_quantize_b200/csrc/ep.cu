// ep.cu -- what an expert-parallel MoE layer sends between GPUs, prepared and
// unpacked on the device.
//
// Each MoE layer sends every token to the GPUs holding its experts and brings
// the expert outputs back (opensourcebeat.com, "Enabling up to 41% faster
// pre-training: MXFP8 and DeepEP ...", section "Двухсторонняя атака: MXFP8 и
// DeepEP"); a token needed by several experts of one destination crosses the
// network once and is copied there (iitak.ru, "NVIDIA в 10 раз ускорила
// обучение моделей-«смесей экспертов» на JAX", paragraph on NCCL EP).
// P ranks own E/P consecutive experts each.  A token travels to each rank
// owning one of its experts as one record: its row in rowwise MXFP8 (C codes,
// then C/32 scale bytes, zero padding to a multiple of 16), 1 + 1/32 bytes per
// element instead of bf16's 2; each routed (token, slot) pair travels as a
// pair entry (local expert id, record index within the records sent to that
// rank).  Send order: destination rank, token, slot, all ascending.
//
// Plan (three launches, no host round trip): (1) one warp per chunk of 32
// tokens (a lane per token) counts the chunk's records and pairs per
// destination with ballots and warp sums; (2) one CTA turns the counts into
// per-chunk start positions (warp scans over chunks, then over ranks); (3)
// every chunk warp places its records, pairs and return positions, lane
// order giving token order.
// Pack: one thread per 32-element block of a record encodes it with the same
// block rule as the rowwise quantiser.  Unpack: one CTA per 128-row x
// 128-column tile of the receiver's grouped rows, like the rowwise quantiser,
// copies codes and places the scale bytes into the 512-byte atom layout.
#include <cuda_runtime.h>

#include <cstdint>

#include "codec.cuh"
#include "ep_launch.h"
#include "groups.cuh"
#include "mxfp8.h"

namespace mxf8 {
namespace {

constexpr int kEpChunk = 32;   // tokens of one plan warp (one per lane)
constexpr int kPlanThreads = 128;
constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ int32_t owner_of(int32_t e, int32_t E, int32_t epr) {
  return (e >= 0 && e < E) ? e / epr : -1;
}

__device__ __forceinline__ int32_t warp_incl_sum(int32_t v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int32_t n = __shfl_up_sync(kFull, v, d);
    if (lane >= d) v += n;
  }
  return v;
}

// Loads a lane's token's expert ids and owners (a lane past T has none).
__device__ __forceinline__ bool load_slots(const int32_t* __restrict__ idx, int64_t t, int64_t T, int32_t k,
                                           int32_t E, int32_t epr, int32_t (&eid)[MXF8_EP_MAX_TOP_K],
                                           int32_t (&own)[MXF8_EP_MAX_TOP_K]) {
  bool bad = false;
  for (int32_t j = 0; j < k; ++j) {
    const int32_t e = t < T ? __ldg(idx + t * k + j) : -1;
    eid[j] = e;
    own[j] = t < T ? owner_of(e, E, epr) : -1;
    bad = bad || (t < T && own[j] < 0);
  }
  return bad;
}

// Pass 1 (one warp per chunk of 32 tokens).  hist[p][c]: records chunk c
// sends to rank p; hist[P + p][c]: pairs.
__global__ void __launch_bounds__(kPlanThreads) ep_count_kernel(const int32_t* __restrict__ idx, int64_t T,
                                                                 int32_t k, int32_t E, int32_t P,
                                                                 int32_t* __restrict__ hist, int64_t chunks,
                                                                 int32_t* __restrict__ status) {
  const int64_t c = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (c >= chunks) return;   // whole warps only
  int32_t eid[MXF8_EP_MAX_TOP_K], own[MXF8_EP_MAX_TOP_K];
  if (load_slots(idx, c * kEpChunk + lane, T, k, E, E / P, eid, own))
    atomicCAS(status, 0, static_cast<int32_t>(MXF8_ERR_BAD_ROUTING));
  for (int32_t p = 0; p < P; ++p) {
    int32_t n = 0;
    for (int32_t j = 0; j < k; ++j) n += own[j] == p ? 1 : 0;
    const unsigned bal = __ballot_sync(kFull, n > 0);
    const int32_t tot = bal ? __reduce_add_sync(kFull, n) : 0;
    if (lane == 0) {
      hist[static_cast<int64_t>(p) * chunks + c] = __popc(bal);
      hist[static_cast<int64_t>(P + p) * chunks + c] = tot;
    }
  }
}

// Pass 2 (one CTA): every hist row becomes its exclusive prefix over chunks
// (one warp per row); bases[p] = first record of rank p, bases[MAX + p] =
// its first pair; counts as documented.
__global__ void __launch_bounds__(1024) ep_scan_kernel(int32_t* __restrict__ hist, int64_t chunks, int32_t P,
                                                      int32_t* __restrict__ counts, int32_t* __restrict__ bases) {
  __shared__ int32_t tot[2 * MXF8_EP_MAX_RANKS];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int row = warp; row < 2 * P; row += 32) {
    int32_t* h = hist + static_cast<int64_t>(row) * chunks;
    int32_t carry = 0;
    for (int64_t c0 = 0; c0 < chunks; c0 += 32) {
      const int64_t c = c0 + lane;
      const int32_t v = c < chunks ? h[c] : 0;
      const int32_t incl = warp_incl_sum(v);
      if (c < chunks) h[c] = carry + incl - v;
      carry += __shfl_sync(kFull, incl, 31);
    }
    if (lane == 0) tot[row] = carry;
  }
  __syncthreads();
  if (warp < 2) {   // warp 0: records, warp 1: pairs -- exclusive scans over ranks
    int32_t carry = 0;
    for (int p0 = 0; p0 < P; p0 += 32) {
      const int p = p0 + lane;
      const int32_t v = p < P ? tot[warp * P + p] : 0;
      const int32_t incl = warp_incl_sum(v);
      if (p < P) {
        bases[warp * MXF8_EP_MAX_RANKS + p] = carry + incl - v;
        counts[warp * P + p] = v;
      }
      carry += __shfl_sync(kFull, incl, 31);
    }
  }
}

// Pass 3 (one warp per chunk): placement.  Lane L's record for rank p comes
// after the chunk's records of lanes < L for p; its pairs for p after theirs,
// in slot order.
__global__ void __launch_bounds__(kPlanThreads) ep_place_kernel(
    const int32_t* __restrict__ idx, int64_t T, int32_t k, int32_t E, int32_t P, const int32_t* __restrict__ hist,
    int64_t chunks, const int32_t* __restrict__ bases, int32_t* __restrict__ rec_token,
    int32_t* __restrict__ pair_expert, int32_t* __restrict__ pair_rec, int32_t* __restrict__ ret_pos) {
  const int64_t c = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (c >= chunks) return;
  const int32_t epr = E / P;
  const int64_t t = c * kEpChunk + lane;
  int32_t eid[MXF8_EP_MAX_TOP_K], own[MXF8_EP_MAX_TOP_K];
  load_slots(idx, t, T, k, E, epr, eid, own);
  if (t < T)
    for (int32_t j = 0; j < k; ++j)
      if (own[j] < 0) ret_pos[t * k + j] = -1;
  const unsigned below = (1u << lane) - 1u;
  for (int32_t p = 0; p < P; ++p) {
    int32_t n = 0;
    for (int32_t j = 0; j < k; ++j) n += own[j] == p ? 1 : 0;
    const unsigned bal = __ballot_sync(kFull, n > 0);
    if (bal == 0) continue;   // uniform across the warp
    const int32_t excl = warp_incl_sum(n) - n;
    if (n > 0) {
      const int32_t rb = __ldg(bases + p);
      const int32_t ri = rb + __ldg(hist + static_cast<int64_t>(p) * chunks + c) + __popc(bal & below);
      rec_token[ri] = static_cast<int32_t>(t);
      int32_t s = __ldg(bases + MXF8_EP_MAX_RANKS + p) + __ldg(hist + static_cast<int64_t>(P + p) * chunks + c) +
                  excl;
      for (int32_t j = 0; j < k; ++j) {
        if (own[j] != p) continue;
        pair_expert[s] = eid[j] - p * epr;
        pair_rec[s] = ri - rb;
        ret_pos[t * k + j] = s;
        ++s;
      }
    }
  }
}

__device__ __forceinline__ uint4 ld_nc16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Pack: thread g encodes block b = g % nb of record i = g / nb.
__global__ void ep_pack_kernel(const uint16_t* __restrict__ x, int64_t T, int64_t C,
                               const int32_t* __restrict__ rec_token, int64_t R, uint8_t* __restrict__ out,
                               int64_t stride) {
  const int64_t nb = C / 32, n = R * nb;
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < n;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t i = g / nb, b = g - i * nb;
    const int32_t t = __ldg(rec_token + i);
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = make_uint4(0, 0, 0, 0);
    if (t >= 0 && t < T) {
      const uint16_t* src = x + static_cast<int64_t>(t) * C + 32 * b;
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = ld_nc16(src + 8 * u);
    }
    const uint32_t a = max(max(amax_bits8(v[0]), amax_bits8(v[1])), max(amax_bits8(v[2]), amax_bits8(v[3])));
    const uint32_t sb = scale_byte(a);
    const uint2 w0 = encode8(v[0], sb), w1 = encode8(v[1], sb), w2 = encode8(v[2], sb), w3 = encode8(v[3], sb);
    uint8_t* r = out + i * stride;
    reinterpret_cast<uint4*>(r + 32 * b)[0] = make_uint4(w0.x, w0.y, w1.x, w1.y);
    reinterpret_cast<uint4*>(r + 32 * b)[1] = make_uint4(w2.x, w2.y, w3.x, w3.y);
    r[C + b] = static_cast<uint8_t>(sb);
    if (b == 0)
      for (int64_t z = C + nb; z < stride; ++z) r[z] = 0;
  }
}

// Unpack: CTA (padded 128-row block, 128-column tile) of the receiver's
// grouped rows.  Thread t < 128 resolves row t's record once.
__global__ void __launch_bounds__(256) ep_unpack_kernel(
    const uint8_t* __restrict__ rec, int64_t R, int64_t C, int64_t stride, const int32_t* __restrict__ pair_rec,
    const int32_t* __restrict__ src_base, int32_t P, const int32_t* __restrict__ perm, int64_t rows,
    const int32_t* __restrict__ offs, int32_t G, uint8_t* __restrict__ q, uint8_t* __restrict__ sf, int64_t pitch) {
  __shared__ __align__(16) uint8_t atom[512];
  __shared__ int64_t src_row[128];
  BlockRows br;
  if (!resolve_block(offs, G, rows, &br)) return;
  const int t = threadIdx.x;
  if (t < 128) {
    int64_t ri = -1;
    if (t < br.nrows) {
      const int32_t s = __ldg(perm + br.row0 + t);
      if (s >= 0 && s < rows) {
        int lo = 0, hi = P - 1;   // the last source whose first pair is <= s
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (__ldg(src_base + mid) <= s) lo = mid;
          else hi = mid - 1;
        }
        ri = static_cast<int64_t>(__ldg(src_base + P + 1 + lo)) + __ldg(pair_rec + s);
        if (ri < 0 || ri >= R) ri = -1;
      }
    }
    src_row[t] = ri;
  }
  __syncthreads();
  const int64_t col0 = static_cast<int64_t>(blockIdx.y) * 128;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int id = t + 256 * u, rr = id >> 3;
    const int64_t col = col0 + 16 * (id & 7);
    if (rr < br.nrows && col < C) {
      const int64_t ri = src_row[rr];
      const uint4 v = ri >= 0 ? ld_nc16(rec + ri * stride + col) : make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(q + (br.row0 + rr) * C + col) = v;
    }
  }
  if (t < 128) {
    uint32_t w = 0;
    const int64_t ri = src_row[t], b0 = col0 / 32, nb = C / 32;
    if (t < br.nrows && ri >= 0) {
      const uint8_t* s = rec + ri * stride + C + b0;
      if (b0 + 4 <= nb) {
        w = *reinterpret_cast<const uint32_t*>(s);   // C % 32 == 0 and b0 % 4 == 0: 4-byte aligned
      } else {
        for (int64_t j = 0; j < nb - b0; ++j) w |= static_cast<uint32_t>(s[j]) << (8 * j);
      }
    }
    *reinterpret_cast<uint32_t*>(atom + (t & 31) * 16 + (t >> 5) * 4) = w;
  }
  __syncthreads();
  if (t < 32) {
    const int64_t a = static_cast<int64_t>(blockIdx.x) * pitch + blockIdx.y;
    reinterpret_cast<uint4*>(sf + a * 512)[t] = reinterpret_cast<const uint4*>(atom)[t];
  }
}

__global__ void gather_rows_kernel(const uint8_t* __restrict__ src, int64_t src_rows, int64_t row_bytes,
                                   const int32_t* __restrict__ idx, int64_t n, uint8_t* __restrict__ dst) {
  const int64_t v = row_bytes / 16, total = n * v;
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < total;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t i = g / v, c = g - i * v;
    const int32_t r = __ldg(idx + i);
    const uint4 val = (r >= 0 && r < src_rows) ? ld_nc16(src + r * row_bytes + 16 * c) : make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4*>(dst + i * row_bytes + 16 * c) = val;
  }
}

unsigned grid_for(int64_t work, int threads) {
  const int64_t b = (work + threads - 1) / threads;
  return static_cast<unsigned>(b < 148 * 32 ? (b > 0 ? b : 1) : 148 * 32);
}

}  // namespace

int64_t ep_plan_chunks(int64_t T) { return (T + kEpChunk - 1) / kEpChunk; }

cudaError_t launch_ep_plan(const int32_t* idx, int64_t T, int32_t k, int32_t E, int32_t P, int32_t* counts,
                           int32_t* rec_token, int32_t* pair_expert, int32_t* pair_rec, int32_t* ret_pos,
                           int32_t* status, int32_t* bases, int32_t* hist, cudaStream_t stream) {
  const int64_t chunks = ep_plan_chunks(T);
  const int64_t warps_per_cta = kPlanThreads / 32;
  const unsigned blocks = static_cast<unsigned>((chunks + warps_per_cta - 1) / warps_per_cta);
  if (chunks > 0) {
    ep_count_kernel<<<blocks, kPlanThreads, 0, stream>>>(idx, T, k, E, P, hist, chunks, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  ep_scan_kernel<<<1, 1024, 0, stream>>>(hist, chunks, P, counts, bases);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || chunks == 0) return e;
  ep_place_kernel<<<blocks, kPlanThreads, 0, stream>>>(idx, T, k, E, P, hist, chunks, bases, rec_token, pair_expert,
                                                      pair_rec, ret_pos);
  return cudaGetLastError();
}

int64_t ep_record_stride(int64_t C) { return (C + C / 32 + 15) / 16 * 16; }

cudaError_t launch_ep_pack(const uint16_t* x, int64_t T, int64_t C, const int32_t* rec_token, int64_t R,
                           uint8_t* records, cudaStream_t stream) {
  if (R == 0) return cudaSuccess;
  ep_pack_kernel<<<grid_for(R * (C / 32), 256), 256, 0, stream>>>(x, T, C, rec_token, R, records,
                                                                  ep_record_stride(C));
  return cudaGetLastError();
}

cudaError_t launch_ep_unpack(const uint8_t* records, int64_t R, int64_t C, const int32_t* pair_rec,
                             const int32_t* src_base, int32_t P, const int32_t* perm, int64_t rows,
                             const int32_t* offs, int32_t G, uint8_t* q, uint8_t* sf, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const int64_t nb = (rows + 127) / 128 + G - 1;
  const dim3 grid(static_cast<unsigned>(nb), static_cast<unsigned>((C + 127) / 128));
  ep_unpack_kernel<<<grid, 256, 0, stream>>>(records, R, C, ep_record_stride(C), pair_rec, src_base, P, perm, rows,
                                            offs, G, q, sf, (C + 127) / 128);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const void* src, int64_t src_rows, int64_t row_bytes, const int32_t* idx, int64_t n,
                               void* dst, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  gather_rows_kernel<<<grid_for(n * (row_bytes / 16), 256), 256, 0, stream>>>(
      static_cast<const uint8_t*>(src), src_rows, row_bytes, idx, n, static_cast<uint8_t*>(dst));
  return cudaGetLastError();
}

}  // namespace mxf8
