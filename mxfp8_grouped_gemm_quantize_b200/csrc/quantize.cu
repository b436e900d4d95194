// quantize.cu -- rowwise and colwise MXFP8 quantisers for sm_100a.
//
// MXFP8 (opensourcebeat.com, "Enabling up to 41% faster pre-training: MXFP8
// and DeepEP ...", FAQ): 32 consecutive elements share one power-of-two
// scale.  Per OCP MX v1.0 the E8M0 scale byte of a block is s + 127 with
// s = floor(log2 amax) - 8 clamped to [-127, 127], and each element is the
// E4M3 code of x * 2^-s, rounded to nearest even and saturated to +-448.
//
// The kernels are HBM-bound (2 bytes read, 1 + 1/32 written per element and
// layout; the dual kernel writes both layouts from one read, 4 + 1/16 bytes).
// A CTA owns one 128-row x 128-column tile, i.e. exactly one 512-byte scale
// atom of the tcgen05 scale-factor layout, so scales leave the CTA as 32
// coalesced 16-byte stores.  Rows are read with 16-byte loads, block amax is
// an integer max over the bf16 magnitude bits (packed, two per instruction),
// and codes come from the hardware E4M3x2 conversion.
#include <cuda_runtime.h>

#include "codec.cuh"
#include "groups.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace mxf8 {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Resolves this CTA's 128-row block (blockIdx.x) to rows of a group.
// Returns false if the block lies past the last group's blocks.
struct BlockRows {
  int64_t row0;     // first input row
  int nrows;        // real rows in the block (<= 128)
  int64_t dst0;     // colwise: first code column (P_g + 128*local)
  int padded;       // colwise: written code columns (multiple of 32, <= 128)
};

__device__ __forceinline__ bool resolve_block(const int32_t* offs, int32_t G, int64_t rows,
                                              BlockRows* out) {
  __shared__ BlockRows s_br;
  __shared__ int s_ok;
  if (threadIdx.x < 32) {
    const GroupBlock gb = warp_find_block(offs, G, rows, blockIdx.x);
    if (threadIdx.x == 0) {
      s_ok = gb.g >= 0;
      if (gb.g >= 0) {
        const int64_t local = static_cast<int64_t>(blockIdx.x) - gb.rb;
        const int64_t left = gb.m - 128 * local;
        const int64_t pad_left = (gb.m + 31) / 32 * 32 - 128 * local;
        s_br.row0 = gb.lo + 128 * local;
        s_br.nrows = static_cast<int>(left < 128 ? left : 128);
        s_br.dst0 = gb.p + 128 * local;
        s_br.padded = static_cast<int>(pad_left < 128 ? pad_left : 128);
      }
    }
  }
  __syncthreads();
  *out = s_br;
  return s_ok != 0;
}

// ---------------------------------------------------------------------------
// Rowwise: thread (rsub = t/16, ch = t%16) handles the 8 elements at columns
// 8*ch.. of rows rsub + 16*i, i = 0..7; four consecutive lanes form a 32-block.
__global__ void __launch_bounds__(kThreads) quantize_rowwise_kernel(
    const uint16_t* __restrict__ x, int64_t rows, int64_t cols, const int32_t* __restrict__ offs,
    int32_t G, uint8_t* __restrict__ q, uint8_t* __restrict__ sf, int64_t pitch) {
  __shared__ __align__(16) uint8_t atom[512];
  BlockRows br;
  if (!resolve_block(offs, G, rows, &br)) return;
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
    uint32_t a = amax_bits8(v[i]);
    a = max(a, __shfl_xor_sync(0xffffffffu, a, 1));
    a = max(a, __shfl_xor_sync(0xffffffffu, a, 2));
    const uint32_t sb = scale_byte(a);
    if (rr < br.nrows && col_ok)
      *reinterpret_cast<uint2*>(q + (br.row0 + rr) * cols + col) = encode8(v[i], sb);
    if ((ch & 3) == 0) atom[(rr & 31) * 16 + (rr >> 5) * 4 + (ch >> 2)] = static_cast<uint8_t>(sb);
  }
  __syncthreads();
  if (t < 32) {
    const int64_t a = static_cast<int64_t>(blockIdx.x) * pitch + blockIdx.y;
    reinterpret_cast<uint4*>(sf + a * 512)[t] = reinterpret_cast<const uint4*>(atom)[t];
  }
}

// ---------------------------------------------------------------------------
// Colwise: the 128x128 bf16 tile is staged in shared memory; thread
// (blk = t/64, p = t%64) reduces columns 2p and 2p+1 over rows 32*blk..+31 and
// encodes them; the 128 code rows (one per input column, 128 bytes each) are
// staged again, swizzled by 16-byte chunk, and leave as coalesced rows of qT.
__global__ void __launch_bounds__(kThreads) quantize_colwise_kernel(
    const uint16_t* __restrict__ x, int64_t rows, int64_t cols, const int32_t* __restrict__ offs,
    int32_t G, uint8_t* __restrict__ qT, int64_t ldT, uint8_t* __restrict__ sfT, int64_t pitch) {
  __shared__ __align__(16) uint32_t tile[128 * 64];   // [row][64 words]; later [code row][32 words]
  __shared__ __align__(16) uint8_t atom[512];
  BlockRows br;
  if (!resolve_block(offs, G, rows, &br)) return;
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
  uint32_t mx = 0;
#pragma unroll
  for (int r = 0; r < 32; ++r) {
    w[r] = tile[(32 * blk + r) * 64 + p];
    mx = __vmaxu2(mx, w[r] & 0x7FFF7FFFu);
  }
  const uint32_t sb_lo = scale_byte(mx & 0xFFFFu), sb_hi = scale_byte(mx >> 16);
  const int vrows = min(32, max(0, br.nrows - 32 * blk));   // real rows of this 32-block
  uint32_t olo[8], ohi[8];
  {
    const float flo = inv_scale(sb_lo == 0xFFu ? 0u : sb_lo);
    const float fhi = inv_scale(sb_hi == 0xFFu ? 0u : sb_hi);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t a0 = cvt_e4m3x2(__fmul_rn(bf_lo(w[4 * j]), flo), __fmul_rn(bf_lo(w[4 * j + 1]), flo));
      const uint32_t a1 = cvt_e4m3x2(__fmul_rn(bf_lo(w[4 * j + 2]), flo), __fmul_rn(bf_lo(w[4 * j + 3]), flo));
      const uint32_t b0 = cvt_e4m3x2(__fmul_rn(bf_hi(w[4 * j]), fhi), __fmul_rn(bf_hi(w[4 * j + 1]), fhi));
      const uint32_t b1 = cvt_e4m3x2(__fmul_rn(bf_hi(w[4 * j + 2]), fhi), __fmul_rn(bf_hi(w[4 * j + 3]), fhi));
      olo[j] = sb_lo == 0xFFu ? nan_codes4(j, vrows) : (a0 | (a1 << 16));
      ohi[j] = sb_hi == 0xFFu ? nan_codes4(j, vrows) : (b0 | (b1 << 16));
    }
  }
  __syncthreads();   // every thread has read its columns; the tile becomes the code stage

  uint4* stage = reinterpret_cast<uint4*>(tile);     // [128 code rows][8 chunks of 16 B]
  const int sw = p & 7;                               // chunk swizzle of code rows 2p and 2p+1
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int chunk = (2 * blk + h) ^ sw;
    stage[(2 * p) * 8 + chunk] = make_uint4(olo[4 * h], olo[4 * h + 1], olo[4 * h + 2], olo[4 * h + 3]);
    stage[(2 * p + 1) * 8 + chunk] = make_uint4(ohi[4 * h], ohi[4 * h + 1], ohi[4 * h + 2], ohi[4 * h + 3]);
  }
  {
    const int r0 = 2 * p, r1 = 2 * p + 1;
    atom[(r0 & 31) * 16 + (r0 >> 5) * 4 + blk] = static_cast<uint8_t>(sb_lo);
    atom[(r1 & 31) * 16 + (r1 >> 5) * 4 + blk] = static_cast<uint8_t>(sb_hi);
  }
  __syncthreads();

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int id = t + kThreads * i, c = id >> 3, j = id & 7;
    if (col0 + c < cols && 16 * j < br.padded)
      *reinterpret_cast<uint4*>(qT + (col0 + c) * ldT + br.dst0 + 16 * j) = stage[c * 8 + (j ^ ((c >> 1) & 7))];
  }
  if (t < 32) {
    const int64_t a = static_cast<int64_t>(blockIdx.y) * pitch + blockIdx.x;
    reinterpret_cast<uint4*>(sfT + a * 512)[t] = reinterpret_cast<const uint4*>(atom)[t];
  }
}

// ---------------------------------------------------------------------------
// Dual: one read of the 128x128 bf16 tile produces both layouts.  The load
// phase uses the rowwise kernel's thread mapping (four consecutive lanes hold
// one 32-element row block), so rowwise codes and scales are encoded straight
// from the loaded registers; the tile then goes to shared memory and the
// colwise pass proceeds exactly as in quantize_colwise_kernel.
// GATHER: row r of the quantised matrix is row gather[r] of x (a token
// permute fused with the quantisation); a gather index outside [0, src_rows)
// reads as a zero row.
template <bool GATHER>
__global__ void __launch_bounds__(kThreads) quantize_dual_kernel(
    const uint16_t* __restrict__ x, int64_t rows, int64_t cols, const int32_t* __restrict__ offs,
    int32_t G, uint8_t* __restrict__ q, uint8_t* __restrict__ sf, int64_t pitch_r,
    uint8_t* __restrict__ qT, int64_t ldT, uint8_t* __restrict__ sfT, int64_t pitch_c,
    const int32_t* __restrict__ gather, int64_t src_rows) {
  __shared__ __align__(16) uint32_t tile[128 * 64];
  __shared__ __align__(16) uint8_t atom_r[512];
  __shared__ __align__(16) uint8_t atom_c[512];
  BlockRows br;
  if (!resolve_block(offs, G, rows, &br)) return;
  const int t = threadIdx.x, ch = t & 15, rsub = t >> 4;
  const int64_t col0 = static_cast<int64_t>(blockIdx.y) * 128;
  const bool col_ok = col0 + 8 * ch < cols;

  uint4 v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int rr = rsub + 16 * i;
    v[i] = make_uint4(0, 0, 0, 0);
    if (rr < br.nrows && col_ok) {
      int64_t src = br.row0 + rr;
      if constexpr (GATHER) src = __ldg(gather + src);
      if (!GATHER || (src >= 0 && src < src_rows)) v[i] = ld_stream(x + src * cols + col0 + 8 * ch);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int rr = rsub + 16 * i;
    uint32_t a = amax_bits8(v[i]);
    a = max(a, __shfl_xor_sync(0xffffffffu, a, 1));
    a = max(a, __shfl_xor_sync(0xffffffffu, a, 2));
    const uint32_t sb = scale_byte(a);
    if (rr < br.nrows && col_ok)
      *reinterpret_cast<uint2*>(q + (br.row0 + rr) * cols + col0 + 8 * ch) = encode8(v[i], sb);
    if ((ch & 3) == 0) atom_r[(rr & 31) * 16 + (rr >> 5) * 4 + (ch >> 2)] = static_cast<uint8_t>(sb);
    reinterpret_cast<uint4*>(tile)[rr * 16 + ch] = v[i];
  }
  __syncthreads();
  if (t < 32) {
    const int64_t a = static_cast<int64_t>(blockIdx.x) * pitch_r + blockIdx.y;
    reinterpret_cast<uint4*>(sf + a * 512)[t] = reinterpret_cast<const uint4*>(atom_r)[t];
  }

  const int blk = t >> 6, p = t & 63;
  uint32_t w[32];
  uint32_t mx = 0;
#pragma unroll
  for (int r = 0; r < 32; ++r) {
    w[r] = tile[(32 * blk + r) * 64 + p];
    mx = __vmaxu2(mx, w[r] & 0x7FFF7FFFu);
  }
  const uint32_t sb_lo = scale_byte(mx & 0xFFFFu), sb_hi = scale_byte(mx >> 16);
  const int vrows = min(32, max(0, br.nrows - 32 * blk));   // real rows of this 32-block
  uint32_t olo[8], ohi[8];
  {
    const float flo = inv_scale(sb_lo == 0xFFu ? 0u : sb_lo);
    const float fhi = inv_scale(sb_hi == 0xFFu ? 0u : sb_hi);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t a0 = cvt_e4m3x2(__fmul_rn(bf_lo(w[4 * j]), flo), __fmul_rn(bf_lo(w[4 * j + 1]), flo));
      const uint32_t a1 = cvt_e4m3x2(__fmul_rn(bf_lo(w[4 * j + 2]), flo), __fmul_rn(bf_lo(w[4 * j + 3]), flo));
      const uint32_t b0 = cvt_e4m3x2(__fmul_rn(bf_hi(w[4 * j]), fhi), __fmul_rn(bf_hi(w[4 * j + 1]), fhi));
      const uint32_t b1 = cvt_e4m3x2(__fmul_rn(bf_hi(w[4 * j + 2]), fhi), __fmul_rn(bf_hi(w[4 * j + 3]), fhi));
      olo[j] = sb_lo == 0xFFu ? nan_codes4(j, vrows) : (a0 | (a1 << 16));
      ohi[j] = sb_hi == 0xFFu ? nan_codes4(j, vrows) : (b0 | (b1 << 16));
    }
  }
  __syncthreads();

  uint4* stage = reinterpret_cast<uint4*>(tile);
  const int sw = p & 7;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int chunk = (2 * blk + h) ^ sw;
    stage[(2 * p) * 8 + chunk] = make_uint4(olo[4 * h], olo[4 * h + 1], olo[4 * h + 2], olo[4 * h + 3]);
    stage[(2 * p + 1) * 8 + chunk] = make_uint4(ohi[4 * h], ohi[4 * h + 1], ohi[4 * h + 2], ohi[4 * h + 3]);
  }
  {
    const int r0 = 2 * p, r1 = 2 * p + 1;
    atom_c[(r0 & 31) * 16 + (r0 >> 5) * 4 + blk] = static_cast<uint8_t>(sb_lo);
    atom_c[(r1 & 31) * 16 + (r1 >> 5) * 4 + blk] = static_cast<uint8_t>(sb_hi);
  }
  __syncthreads();

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int id = t + kThreads * i, c = id >> 3, j = id & 7;
    if (col0 + c < cols && 16 * j < br.padded)
      *reinterpret_cast<uint4*>(qT + (col0 + c) * ldT + br.dst0 + 16 * j) = stage[c * 8 + (j ^ ((c >> 1) & 7))];
  }
  if (t < 32) {
    const int64_t a = static_cast<int64_t>(blockIdx.y) * pitch_c + blockIdx.x;
    reinterpret_cast<uint4*>(sfT + a * 512)[t] = reinterpret_cast<const uint4*>(atom_c)[t];
  }
}

int64_t block_bound(int64_t rows, int32_t G) { return rows == 0 ? 0 : (rows + 127) / 128 + G - 1; }

}  // namespace

cudaError_t launch_quantize_rowwise(const uint16_t* x, int64_t rows, int64_t cols,
                                    const int32_t* offs, int32_t G, uint8_t* q, uint8_t* sf,
                                    cudaStream_t stream) {
  const int64_t nb = block_bound(rows, G);
  if (nb == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>(nb), static_cast<unsigned>((cols + 127) / 128));
  quantize_rowwise_kernel<<<grid, kThreads, 0, stream>>>(x, rows, cols, offs, G, q, sf, (cols + 127) / 128);
  return cudaGetLastError();
}

cudaError_t launch_quantize_colwise(const uint16_t* x, int64_t rows, int64_t cols,
                                    const int32_t* offs, int32_t G, uint8_t* qT, int64_t ldT,
                                    uint8_t* sfT, cudaStream_t stream) {
  const int64_t nb = block_bound(rows, G);
  if (nb == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>(nb), static_cast<unsigned>((cols + 127) / 128));
  quantize_colwise_kernel<<<grid, kThreads, 0, stream>>>(x, rows, cols, offs, G, qT, ldT, sfT, nb);
  return cudaGetLastError();
}

cudaError_t launch_quantize_dual(const uint16_t* x, int64_t rows, int64_t cols, const int32_t* offs,
                                 int32_t G, uint8_t* q, uint8_t* sf, uint8_t* qT, int64_t ldT, uint8_t* sfT,
                                 cudaStream_t stream) {
  const int64_t nb = block_bound(rows, G);
  if (nb == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>(nb), static_cast<unsigned>((cols + 127) / 128));
  quantize_dual_kernel<false><<<grid, kThreads, 0, stream>>>(x, rows, cols, offs, G, q, sf, (cols + 127) / 128, qT,
                                                              ldT, sfT, nb, nullptr, rows);
  return cudaGetLastError();
}

cudaError_t launch_permute_quantize_dual(const uint16_t* x, int64_t src_rows, int64_t cols, const int32_t* perm,
                                         int64_t rows, const int32_t* offs, int32_t G, uint8_t* q, uint8_t* sf,
                                         uint8_t* qT, int64_t ldT, uint8_t* sfT, cudaStream_t stream) {
  const int64_t nb = block_bound(rows, G);
  if (nb == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>(nb), static_cast<unsigned>((cols + 127) / 128));
  quantize_dual_kernel<true><<<grid, kThreads, 0, stream>>>(x, rows, cols, offs, G, q, sf, (cols + 127) / 128, qT,
                                                             ldT, sfT, nb, perm, src_rows);
  return cudaGetLastError();
}

}  // namespace mxf8
