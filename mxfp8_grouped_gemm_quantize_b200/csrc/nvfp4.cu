// nvfp4.cu -- NVFP4 quantisers for sm_100a: 4-bit E2M1 elements in blocks of
// 16 sharing an E4M3 scale, with one fp32 scale per tensor.
//
// The pages name NVFP4 only as the format NVIDIA's MoE training adds next
// (iitak.ru, "NVIDIA в 10 раз ускорила обучение моделей-«смесей экспертов»
// на JAX", closing paragraph); the rules are NVIDIA's public definition:
//   S  = 2688 / amax(tensor)              (448 * 6; 1 when amax = 0)
//   sf = E4M3(amax_block * S / 6)         (round to nearest even)
//   q  = E2M1((x * S) / sf)               (nearest even, saturating at 6; 0 when sf = 0)
// Every fp32 operation is rounded to nearest in exactly this order, so the
// code of each element is decided in fp32 the same way on any IEEE machine.
//
// Layouts mirror the MXFP8 ones with 16-element blocks: the 512-byte scale
// atom covers 128 rows x 4 blocks = 64 elements along the contraction; codes
// are packed two per byte, element 2i in the low nibble of byte i.
//   rowwise: q [R, C/2]; scale atom (rb, cb) at 512*(rb*ceil(C/64) + cb) with
//            rb the group-padded 128-row block (as for MXFP8).
//   colwise: qT [C, ld/2] with group g's rows from nibble P_g (32-padded);
//            scales S^T[c, 4*Q_g + t/16], Q_g = sum of ceil(m_h/64) over h < g,
//            pitch ceil(R/64) + G - 1.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "groups.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace mxf8 {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float bf_lo_f(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi_f(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// E4M3 byte of a non-negative fp32 value, nearest even, saturating at 448.
__device__ __forceinline__ uint32_t e4m3_byte(float v) { return cvt_e4m3x2(v, 0.0f) & 0xFFu; }

// Value of an E4M3 byte (exact, through the hardware f16 widening).
__device__ __forceinline__ float e4m3_value(uint32_t b) {
  uint32_t h;
  const uint16_t in = static_cast<uint16_t>(b);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(in));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h & 0xFFFFu)));
}

// Two E2M1 codes (nearest even, saturating): lo in bits 0-3, hi in bits 4-7.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint32_t out;
  asm("{\n\t.reg .b8 b;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b, %2, %1;\n\t"
      "mov.b32 %0, {b, b, b, b};\n\t}"
      : "=r"(out)
      : "f"(lo), "f"(hi));
  return out & 0xFFu;
}

__device__ __forceinline__ float tensor_scale(const float* amax) {
  const float a = __ldg(amax);
  return a == 0.0f ? 1.0f : __fdiv_rn(2688.0f, a);
}

// Block scale byte from the block amax, and the element divisor it decodes to.
__device__ __forceinline__ uint32_t block_scale(float amax, float S, float* r) {
  const uint32_t sb = e4m3_byte(__fdiv_rn(__fmul_rn(amax, S), 6.0f));
  *r = e4m3_value(sb);
  return sb;
}

// Codes of 8 bf16 (one uint4) given S and the block's divisor r: 4 bytes.
__device__ __forceinline__ uint32_t encode8_fp4(const uint4& v, float S, float r) {
  if (r == 0.0f) return 0u;
  auto e = [&](uint32_t w) {
    return e2m1x2(__fdiv_rn(__fmul_rn(bf_lo_f(w), S), r), __fdiv_rn(__fmul_rn(bf_hi_f(w), S), r));
  };
  return e(v.x) | (e(v.y) << 8) | (e(v.z) << 16) | (e(v.w) << 24);
}

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// ---------------------------------------------------------------- amax
__global__ void __launch_bounds__(kThreads) amax_kernel(const uint16_t* __restrict__ x, int64_t n,
                                                        unsigned int* __restrict__ out) {
  uint32_t m = 0;
  const int64_t n8 = n / 8;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 v = ld_stream(x + 8 * i);
    const uint32_t k = 0x7FFF7FFFu;
    m = __vmaxu2(m, __vmaxu2(__vmaxu2(v.x & k, v.y & k), __vmaxu2(v.z & k, v.w & k)));
  }
  for (int64_t i = 8 * n8 + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    m = __vmaxu2(m, x[i] & 0x7FFFu);
  m = max(m & 0xFFFFu, m >> 16);
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, d));
  // bf16 magnitude bits -> fp32 bits; non-negative floats order like their bits
  if ((threadIdx.x & 31) == 0 && m) atomicMax(out, m << 16);
}

// Group lookup for the CTA's 128-row block (blockIdx.x).
struct Rows {
  int64_t row0, dst0, qatom0;
  int nrows, padded, natoms;
};

__device__ __forceinline__ bool resolve_rows(const int32_t* offs, int32_t G, int64_t rows, Rows* out) {
  __shared__ Rows s_r;
  __shared__ int s_ok;
  if (threadIdx.x < 32) {
    const GroupBlock gb = warp_find_block(offs, G, rows, blockIdx.x);
    if (threadIdx.x == 0) {
      s_ok = gb.g >= 0;
      if (gb.g >= 0) {
        const int64_t local = static_cast<int64_t>(blockIdx.x) - gb.rb;
        const int64_t left = gb.m - 128 * local, pad_left = (gb.m + 31) / 32 * 32 - 128 * local;
        const int64_t q_left = (gb.m + 63) / 64 - 2 * local;
        s_r.row0 = gb.lo + 128 * local;
        s_r.nrows = static_cast<int>(left < 128 ? left : 128);
        s_r.dst0 = gb.p + 128 * local;
        s_r.padded = static_cast<int>(pad_left < 128 ? pad_left : 128);
        s_r.qatom0 = gb.q + 2 * local;
        s_r.natoms = static_cast<int>(q_left < 2 ? q_left : 2);
      }
    }
  }
  __syncthreads();
  *out = s_r;
  return s_ok != 0;
}

// ---------------------------------------------------------------- rowwise
// CTA: 128 rows x 128 columns (two scale atoms).  Thread (rsub = t/16,
// ch = t%16) holds 8 elements of rows rsub + 16*i; two lanes form a block.
__global__ void __launch_bounds__(kThreads) nvfp4_rowwise_kernel(
    const uint16_t* __restrict__ x, int64_t rows, int64_t cols, const int32_t* __restrict__ offs, int32_t G,
    const float* __restrict__ amax, uint8_t* __restrict__ q, uint8_t* __restrict__ sf, int64_t pitch) {
  __shared__ __align__(16) uint8_t atom[2][512];
  Rows br;
  if (!resolve_rows(offs, G, rows, &br)) return;
  const float S = tensor_scale(amax);
  const int t = threadIdx.x, ch = t & 15, rsub = t >> 4;
  const int64_t col = static_cast<int64_t>(blockIdx.y) * 128 + 8 * ch;
  const bool col_ok = col < cols;
  uint4 v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int rr = rsub + 16 * i;
    v[i] = make_uint4(0, 0, 0, 0);
    if (rr < br.nrows && col_ok) v[i] = ld_stream(x + (br.row0 + rr) * cols + col);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int rr = rsub + 16 * i;
    const uint32_t k = 0x7FFF7FFFu;
    uint32_t m = __vmaxu2(__vmaxu2(v[i].x & k, v[i].y & k), __vmaxu2(v[i].z & k, v[i].w & k));
    m = max(m & 0xFFFFu, m >> 16);
    m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
    float r;
    const uint32_t sb = block_scale(__uint_as_float(m << 16), S, &r);
    if (rr < br.nrows && col_ok)
      *reinterpret_cast<uint32_t*>(q + (br.row0 + rr) * (cols / 2) + col / 2) = encode8_fp4(v[i], S, r);
    if ((ch & 1) == 0) {
      const int blk = ch >> 1;   // 16-block within the CTA's 128 columns (0..7)
      atom[blk >> 2][(rr & 31) * 16 + (rr >> 5) * 4 + (blk & 3)] = static_cast<uint8_t>(sb);
    }
  }
  __syncthreads();
  if (t < 64) {
    const int h = t >> 5;
    const int64_t cb = static_cast<int64_t>(blockIdx.y) * 2 + h;
    if (cb < pitch) {
      const int64_t a = static_cast<int64_t>(blockIdx.x) * pitch + cb;
      reinterpret_cast<uint4*>(sf + a * 512)[t & 31] = reinterpret_cast<const uint4*>(atom[h])[t & 31];
    }
  }
}

// ---------------------------------------------------------------- colwise
// The 128x128 bf16 tile is staged in shared memory; thread (blk = t/64,
// p = t%64) takes columns 2p and 2p+1 over rows 32*blk .. +31, i.e. two
// 16-row blocks per column, and writes 16 bytes of packed codes per column
// to a swizzled stage; code rows leave as coalesced 64-byte rows of qT.
__global__ void __launch_bounds__(kThreads) nvfp4_colwise_kernel(
    const uint16_t* __restrict__ x, int64_t rows, int64_t cols, const int32_t* __restrict__ offs, int32_t G,
    const float* __restrict__ amax, uint8_t* __restrict__ qT, int64_t ldT_bytes, uint8_t* __restrict__ sfT,
    int64_t pitch) {
  __shared__ __align__(16) uint32_t tile[128 * 64];   // [row][64 words of bf16 pairs]
  __shared__ __align__(16) uint4 stage[128 * 4];      // [code row][4 chunks of 16 B]
  __shared__ __align__(16) uint8_t atom[2][512];
  Rows br;
  if (!resolve_rows(offs, G, rows, &br)) return;
  const float S = tensor_scale(amax);
  const int t = threadIdx.x;
  const int64_t col0 = static_cast<int64_t>(blockIdx.y) * 128;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int id = t + kThreads * i, r = id >> 4, c16 = id & 15;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < br.nrows && col0 + 8 * c16 < cols) v = ld_stream(x + (br.row0 + r) * cols + col0 + 8 * c16);
    reinterpret_cast<uint4*>(tile)[r * 16 + c16] = v;
  }
  __syncthreads();
  const int blk = t >> 6, p = t & 63;
  uint32_t w[32];
#pragma unroll
  for (int r = 0; r < 32; ++r) w[r] = tile[(32 * blk + r) * 64 + p];
  uint32_t olo[4], ohi[4];
#pragma unroll
  for (int hb = 0; hb < 2; ++hb) {   // 16-row block 2*blk + hb
    uint32_t m = 0;
#pragma unroll
    for (int r = 0; r < 16; ++r) m = __vmaxu2(m, w[16 * hb + r] & 0x7FFF7FFFu);
    float rlo, rhi;
    const uint32_t sb_lo = block_scale(__uint_as_float((m & 0xFFFFu) << 16), S, &rlo);
    const uint32_t sb_hi = block_scale(__uint_as_float(m & 0xFFFF0000u), S, &rhi);
#pragma unroll
    for (int j = 0; j < 2; ++j) {   // 8 rows -> 4 bytes per column
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t a = w[16 * hb + 8 * j + 2 * k], b = w[16 * hb + 8 * j + 2 * k + 1];
        if (rlo != 0.0f)
          lo |= e2m1x2(__fdiv_rn(__fmul_rn(bf_lo_f(a), S), rlo), __fdiv_rn(__fmul_rn(bf_lo_f(b), S), rlo)) << (8 * k);
        if (rhi != 0.0f)
          hi |= e2m1x2(__fdiv_rn(__fmul_rn(bf_hi_f(a), S), rhi), __fdiv_rn(__fmul_rn(bf_hi_f(b), S), rhi)) << (8 * k);
      }
      olo[2 * hb + j] = lo;
      ohi[2 * hb + j] = hi;
    }
    const int b16 = 2 * blk + hb;    // 16-row block within the CTA (0..7)
    const int r0 = 2 * p, r1 = 2 * p + 1;
    atom[b16 >> 2][(r0 & 31) * 16 + (r0 >> 5) * 4 + (b16 & 3)] = static_cast<uint8_t>(sb_lo);
    atom[b16 >> 2][(r1 & 31) * 16 + (r1 >> 5) * 4 + (b16 & 3)] = static_cast<uint8_t>(sb_hi);
  }
  // stage: code row 2p / 2p+1, 16-byte chunk blk (rows 32*blk .. +31), swizzled by code row
  stage[(2 * p) * 4 + (blk ^ (p & 3))] = make_uint4(olo[0], olo[1], olo[2], olo[3]);
  stage[(2 * p + 1) * 4 + (blk ^ (p & 3))] = make_uint4(ohi[0], ohi[1], ohi[2], ohi[3]);
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int id = t + kThreads * i, c = id >> 2, j = id & 3;
    if (col0 + c < cols && 32 * j < br.padded)
      *reinterpret_cast<uint4*>(qT + (col0 + c) * ldT_bytes + br.dst0 / 2 + 16 * j) =
          stage[c * 4 + (j ^ ((c >> 1) & 3))];
  }
  if (t < 64) {
    const int h = t >> 5;
    if (h < br.natoms) {
      const int64_t a = static_cast<int64_t>(blockIdx.y) * pitch + br.qatom0 + h;
      reinterpret_cast<uint4*>(sfT + a * 512)[t & 31] = reinterpret_cast<const uint4*>(atom[h])[t & 31];
    }
  }
}

int64_t block_bound(int64_t rows, int32_t G) { return rows == 0 ? 0 : (rows + 127) / 128 + G - 1; }

}  // namespace

cudaError_t launch_nvfp4_amax(const uint16_t* x, int64_t n, float* amax, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float), stream);
  if (e != cudaSuccess || n == 0) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t need = (n / 8 + kThreads - 1) / kThreads;
  const int grid = static_cast<int>(need < 4 * sms ? (need > 0 ? need : 1) : 4 * sms);
  amax_kernel<<<grid, kThreads, 0, stream>>>(x, n, reinterpret_cast<unsigned int*>(amax));
  return cudaGetLastError();
}

cudaError_t launch_nvfp4_rowwise(const uint16_t* x, int64_t rows, int64_t cols, const int32_t* offs, int32_t G,
                                 const float* amax, uint8_t* q, uint8_t* sf, cudaStream_t stream) {
  const int64_t nb = block_bound(rows, G);
  if (nb == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>(nb), static_cast<unsigned>((cols + 127) / 128));
  nvfp4_rowwise_kernel<<<grid, kThreads, 0, stream>>>(x, rows, cols, offs, G, amax, q, sf, (cols + 63) / 64);
  return cudaGetLastError();
}

cudaError_t launch_nvfp4_colwise(const uint16_t* x, int64_t rows, int64_t cols, const int32_t* offs, int32_t G,
                                 const float* amax, uint8_t* qT, int64_t ldT, uint8_t* sfT, cudaStream_t stream) {
  const int64_t nb = block_bound(rows, G);
  if (nb == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>(nb), static_cast<unsigned>((cols + 127) / 128));
  nvfp4_colwise_kernel<<<grid, kThreads, 0, stream>>>(x, rows, cols, offs, G, amax, qT, ldT / 2, sfT,
                                                      (rows + 63) / 64 + G - 1);
  return cudaGetLastError();
}

}  // namespace mxf8
