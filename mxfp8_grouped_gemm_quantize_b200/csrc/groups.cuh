// groups.cuh -- on-device reading of the ragged group offsets.
//
// Every kernel derives what it needs from the int32 offsets itself (no host
// round trip): offsets are clamped to [0, rows] and made non-decreasing, so
// that any input, valid or not, keeps every access in bounds.  Per group g
// (m_g = offs'[g+1] - offs'[g]):
//   RB_g = sum over h < g of ceil(m_h / 128)   (128-row blocks; scale atoms)
//   P_g  = sum over h < g of round_up(m_h, 32) (32-padded rows; colwise codes)
//   Q_g  = sum over h < g of ceil(m_h / 64)    (64-row blocks; NVFP4 colwise scale atoms)
#pragma once
#include <cstdint>

namespace mxf8 {

struct GroupBlock {
  int32_t g;       // group index, -1 if the block index is past the last block
  int64_t lo;      // first row of the group
  int64_t m;       // rows in the group
  int64_t rb;      // RB_g
  int64_t p;       // P_g
  int64_t q;       // Q_g
};

__device__ __forceinline__ int64_t clamp_off(const int32_t* offs, int32_t h, int64_t rows) {
  int64_t v = offs ? static_cast<int64_t>(__ldg(offs + h)) : (h == 0 ? 0 : rows);
  return v < 0 ? 0 : (v > rows ? rows : v);
}

// Warp-cooperative lookup of the group owning padded 128-row block `pb`
// (blocks ordered group by group).  Every lane returns the same result.
__device__ __forceinline__ GroupBlock warp_find_block(const int32_t* offs, int32_t G, int64_t rows,
                                                      int64_t pb) {
  const int lane = threadIdx.x & 31;
  int64_t o_prev = clamp_off(offs, 0, rows);
  int64_t carry_rb = 0, carry_p = 0, carry_q = 0;
  for (int32_t base = 0; base < G; base += 32) {
    const int32_t h = base + lane;
    int64_t v = (h < G) ? clamp_off(offs, h + 1, rows) : 0;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      int64_t t = __shfl_up_sync(0xffffffffu, v, d);
      if (lane >= d) v = v > t ? v : t;
    }
    const int64_t hi = v > o_prev ? v : o_prev;           // offs'[h + 1]
    int64_t lo = __shfl_up_sync(0xffffffffu, hi, 1);
    if (lane == 0) lo = o_prev;                           // offs'[h]
    const int64_t m = (h < G) ? hi - lo : 0;
    const int64_t nb = (m + 127) / 128, np = (m + 31) / 32 * 32, nq = (m + 63) / 64;
    int64_t snb = nb, snp = np, snq = nq;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      int64_t a = __shfl_up_sync(0xffffffffu, snb, d);
      int64_t b = __shfl_up_sync(0xffffffffu, snp, d);
      int64_t c = __shfl_up_sync(0xffffffffu, snq, d);
      if (lane >= d) { snb += a; snp += b; snq += c; }
    }
    const int64_t rb0 = carry_rb + snb - nb, p0 = carry_p + snp - np, q0 = carry_q + snq - nq;
    const bool found = (h < G) && nb > 0 && pb >= rb0 && pb < rb0 + nb;
    const uint32_t ball = __ballot_sync(0xffffffffu, found);
    if (ball) {
      const int src = __ffs(ball) - 1;
      GroupBlock r;
      r.g = __shfl_sync(0xffffffffu, h, src);
      r.lo = __shfl_sync(0xffffffffu, lo, src);
      r.m = __shfl_sync(0xffffffffu, m, src);
      r.rb = __shfl_sync(0xffffffffu, rb0, src);
      r.p = __shfl_sync(0xffffffffu, p0, src);
      r.q = __shfl_sync(0xffffffffu, q0, src);
      return r;
    }
    carry_rb = __shfl_sync(0xffffffffu, carry_rb + snb, 31);
    carry_p = __shfl_sync(0xffffffffu, carry_p + snp, 31);
    carry_q = __shfl_sync(0xffffffffu, carry_q + snq, 31);
    o_prev = __shfl_sync(0xffffffffu, hi, 31);
  }
  GroupBlock none;
  none.g = -1; none.lo = 0; none.m = 0; none.rb = 0; none.p = 0; none.q = 0;
  return none;
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

}  // namespace mxf8
