// grouped_gemm.cu -- persistent MXFP8 grouped GEMM for sm_100a (tcgen05).
//
// All experts run in one launch, each on its real token count (iitak.ru,
// "NVIDIA ... JAX", paragraph on the Transformer Engine grouped GEMM: no
// padding to a capacity, no dropped tokens).  The three products of a MoE
// expert layer share this kernel:
//   fwd    Y_e  = X_e  W_e^T   A = X rowwise,    B = W rowwise       (contract K)
//   dgrad  dX_e = dY_e W_e     A = dY rowwise,   B = W colwise       (contract N)
//   wgrad  dW_e = dY_e^T X_e   A = dY colwise,   B = X colwise       (contract m_e)
// Every operand is K-major E4M3 with E8M0 scales per 32 elements along K
// (MXFP8: opensourcebeat.com, "Enabling up to 41% faster pre-training ...",
// FAQ), so one block-scaled MMA instruction (kind::mxf8f6f4, K = 32) applies
// the scales in hardware and accumulates in fp32 tensor memory.  The NVFP4
// variant (FP4) takes E2M1 operands with E4M3 scales per 16 elements
// (kind::mxf4nvf4, K = 64) through the same pipeline.
//
// One kernel template, CG = CTAs per MMA:
//   CG = 2: CTA pairs (clusters of 2) issue 256x256x32 MMAs
//     (cta_group::2).  Each CTA stages its own 128 rows of A, half of B's 256
//     rows and all 256 rows of B's scales; the pair computes a 256x256 output
//     tile, 128 rows in each CTA's tensor memory.  Per CTA this moves 2/3 of
//     the operand bytes per FLOP of a 1-CTA 128x256 tile.  In fwd/dgrad a
//     group's ragged last tile (r < 256 rows) runs with the operand roles
//     swapped: 256 B rows x round_up(r, 32) tokens, so pairs pad a group to
//     32 rows rather than 256.
//   CG = 1: 128x256x32 MMAs (cta_group::1), one CTA per tile.
// Roles per CTA (192 threads): warp 0 TMA producer; warp 1 allocates the 512
// tensor-memory columns, and (in the leader CTA) one thread copies scale
// atoms to tensor memory and issues the MMAs; warps 2-5 drain the
// accumulator: tcgen05.ld -> bf16 -> 128-byte-swizzled shared stage -> TMA
// bulk-tensor store (plain masked stores only for a group's ragged slice and
// for the row segments of a swapped tile).
// Two 128x256 fp32 accumulators overlap in 64 or 128 columns (0..255 and
// 192..447, or 128..383 when more pipeline stages need more scale columns);
// the epilogue drains the shared columns first and releases the accumulator,
// so the next tile's MMAs overlap the rest of the drain.  The columns after
// accumulator 1 hold the scale-factor sets (see Cfg).
// The tile schedule is built on the device from the group offsets at kernel
// start (no host synchronisation); tiles are dealt round-robin.  Every wait is
// bounded: on timeout the kernel records MXF8_ERR_TIMEOUT, drains its
// in-flight copies and MMAs, frees tensor memory and exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdlib>
#include <cstring>
#include <type_traits>

#include "codec.cuh"
#include "launch.h"
#include "mxfp8.h"
#include "ptx.cuh"

namespace mxf8 {
namespace {

constexpr int BM = 128, BN = 256, BK = 128;
constexpr int SFA_TILE = 512, SFB_TILE = 1024;
constexpr int NUM_THREADS = 192;
constexpr int EPI_STAGE = 32 * 128;        // one epilogue buffer: 32 rows x 64 bf16, 128B-swizzled
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_STRIDE = 12;        // per stage: SFA 4 columns, then SFB 8 columns
constexpr int MAXG = MXF8_GEMM_MAX_GROUPS;
constexpr int SCHED_INTS = 6 * (MAXG + 1);

constexpr int round_up_c(int a, int b) { return (a + b - 1) / b * b; }

// Pipeline shape: CG CTAs per MMA, KS 128-wide K blocks per stage.  The ring
// takes as many stages as shared memory holds: 1 CTA: 4 x 128-deep or
// 2 x 256-deep; pair: 6 x 128-deep or 3 x 256-deep.  Deeper stages amortise
// the fixed cost of a stage hand-off (barrier round trip, copy issue) over
// twice the MMAs.
// FP4 (NVFP4 operands): a 128-byte K block holds 256 elements = four MMAs of
// K = 64, each with its own scale atom (16-element blocks), so a stage
// carries four times the scale bytes, the ring is one stage shorter, and the
// scale sets alternate between two tensor-memory sets of 48 columns.
template <int CG, int KS_, bool FP4 = false>
struct Cfg {
  static constexpr int KS = KS_;
  static constexpr int STAGES = FP4 ? (CG == 2 ? 5 : 3) : (CG == 2 ? (KS == 2 ? 3 : 6) : (KS == 2 ? 2 : 4));
  static constexpr int APK = FP4 ? 4 : 1;              // scale atoms per K block and 128 rows
  static constexpr int SFA_T = SFA_TILE * APK, SFB_T = SFB_TILE * APK;
  static constexpr int SLOTS = STAGES * KS;            // 128-wide K-block slots in the ring
  static constexpr int B_ROWS = BN / CG;               // B rows staged by each CTA
  static constexpr int A_TILE = BM * BK;               // 16 KB of E4M3 codes
  static constexpr int B_TILE = B_ROWS * BK;
  static constexpr int EPI_BUFS = 1;
  // The two 128x256 accumulators overlap in OV 64-column chunks: accumulator 1
  // starts at column ACC_STRIDE, and the scale sets follow it.  Scale sets
  // either rotate with the ring's K-block slots or, where the ring is deep
  // (NVFP4, pairs with 6 x 128-deep stages), alternate between two sets: the
  // copies and MMAs of one thread execute in issue order, so the copy into a
  // set follows the MMAs of the K block before last that read it.
  static constexpr bool SF_ALT = FP4 || SLOTS > 4;
  static constexpr int SF_SETS = SF_ALT ? 2 : SLOTS;   // scale sets in tensor memory
  static constexpr int SF_SET_COLS = SF_STRIDE * APK;  // columns of one set
  static constexpr int OV = (SF_SETS * SF_SET_COLS <= 64) ? 1 : 2;
  static constexpr uint32_t ACC_STRIDE = 256 - 64 * OV;
  static constexpr uint32_t SF_COL = ACC_STRIDE + 256;
  // Bytes one CTA pair (or CTA) receives for a stage holding `nh` K blocks:
  // the scale boxes always span all KS atoms.
  static constexpr uint32_t stage_tx(int nh) {
    return CG * (nh * (A_TILE + B_TILE) + KS * (SFA_T + SFB_T));
  }
  // Slot q = stage * KS + h.  Scale atoms of one stage are fetched as boxes of
  // KS consecutive atoms: SFA box at OFF_SFA + stage * KS * 512, the two SFB
  // boxes (B rows 0-127, 128-255) at OFF_SFB + stage * 2 * KS * 512 (+ KS * 512).
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + SLOTS * A_TILE;
  static constexpr int OFF_SFA = OFF_B + SLOTS * B_TILE;
  static constexpr int OFF_SFB = OFF_SFA + SLOTS * SFA_T;
  static constexpr int OFF_EPI = round_up_c(OFF_SFB + SLOTS * SFB_T, 1024);
  static constexpr int OFF_BAR = OFF_EPI + 4 * EPI_BUFS * EPI_STAGE;
  static constexpr int OFF_MISC = OFF_BAR + 128;
  static constexpr int OFF_SCHED = OFF_MISC + 64;
  static constexpr int SMEM_BYTES = OFF_SCHED + SCHED_INTS * 4 + 1024;   // + slack to align the base
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(OFF_B % 1024 == 0 && B_TILE % 1024 == 0 && OFF_EPI % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static_assert(SF_COL + SF_SET_COLS * SF_SETS <= TMEM_COLS, "scale columns");
  static_assert(KS >= 1 && KS <= 2 && STAGES >= 2, "pipeline shape");
  static_assert((2 * STAGES + 3) * 8 <= 128, "barrier area");
};

struct Params {
  int mode;
  int32_t E;
  int64_t M, N, K;
  const int32_t* offs;
  int64_t sfa_pitch, sfb_pitch;        // atoms per atom row of the A / B scale matrices
  uint16_t* out;                       // output (fwd [M,N], dgrad [M,K], wgrad [E*N,K]); may be
                                       // null in a quantising epilogue
  int64_t out_ld;                      // output row stride (elements)
  int32_t* status;
  uint64_t timeout_ns;
  int32_t inject_skip_stage;           // test hook: the producers leave stage 0 unfilled
  // Quantising epilogue (fwd/dgrad): MXFP8 copies of the bf16 output, in the
  // quantisers' layouts with the GEMM's groups.  Null pointers skip a layout.
  uint8_t* qr;                         // rowwise codes [M, out_ld]
  uint8_t* sr;                         // rowwise scale atoms, pitch ceil(out_ld / 128)
  uint8_t* qc;                         // colwise codes [out_ld, qc_ld] (transposed)
  uint8_t* sc;                         // colwise scale atoms, pitch sc_pitch
  int64_t qc_ld, sc_pitch;
  // NVFP4 operands: device amax of each operand's tensor (tensor scale
  // S = 2688 / amax); the output is the accumulator times 1 / (S_a * S_b).
  const float* amax_a;
  const float* amax_b;
};

// Per-CTA schedule, built from the offsets by warp 0.  Tiles are numbered
// slot by slot; slot i holds the tiles of expert slot[i] (fwd/dgrad: slot i
// is expert i; wgrad: experts by decreasing token count, so the long K loops
// run first and the short ones fill the end of the schedule).
struct Sched {
  int32_t* tile0;   // [E+1] first tile of each slot (prefix)
  int32_t* slot;    // [E]   expert of each slot
  int32_t* off;     // [E+1] row offsets
  int32_t* rb;      // [E]   RB_e: 128-row blocks before group e (rowwise scale rows,
                    //       colwise scale block-columns / 4)
  int32_t* p;       // [E]   P_e: 32-padded rows before group e (colwise code column)
  int32_t* q;       // [E]   Q_e: 64-row blocks before group e (NVFP4 colwise scale atoms)
};

// One CTA's share of a tile.
struct Tile {
  int32_t kblocks;       // 128-wide K blocks (0: nothing to accumulate)
  int32_t ksteps_last;   // 32-wide MMA steps in the last K block
  int32_t a_x, a_y, b_x, b_y;           // TMA coordinates of the first K block (this CTA's rows)
  int64_t sfa_atom, sfb_atom0, sfb_atom1;   // scale atoms of the first K block
  int64_t out_row, out_col;             // output element (row, col) of this CTA's tile corner
  int32_t rows, cols;    // valid rows (0..128) and columns (<= 256) of this CTA's tile
  int32_t q_rb;          // fwd/dgrad: RB_e + row block, the output's rowwise scale atom row
                         //            and colwise scale atom column
  int32_t q_p;           // fwd/dgrad: P_e + 128 * row block, the output's colwise code column
  bool swapped;          // CTA pairs, fwd/dgrad: a group's ragged last tile with the operand roles
                         // swapped (A = the B operand's 256 rows, B = the group's last tokens)
  int32_t ntok;          // swapped: MMA N = the tile's tokens rounded up to 32
};

__device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__device__ __forceinline__ int32_t cdiv32(int64_t a, int64_t b) { return static_cast<int32_t>((a + b - 1) / b); }

// SwiGLU of one gate/up pair from the fp32 accumulators: silu(g) * u with
// silu(g) = g / (1 + exp(-g)) (g -> -inf gives -0: the division by an
// infinite denominator returns zero).
__device__ __forceinline__ float swiglu_f32(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

template <int CG>
__device__ __forceinline__ int32_t group_m_units(const Params& p, int32_t m) {
  return cdiv32(p.mode == kWgrad ? cdiv32(p.N, BM) : cdiv32(m, BM), CG);
}

__device__ __forceinline__ int32_t n_tiles(const Params& p) {
  return p.mode == kFwd ? cdiv32(p.N, BN) : cdiv32(p.K, BN);
}

// Slot of tile t: the last slot whose first tile is <= t.  A CTA visits its
// tiles in increasing order, so the search advances from the previous answer
// `i` (start at 0) instead of bisecting every time.
__device__ __forceinline__ int32_t advance_group(const Sched& s, int32_t E, int32_t t, int32_t i) {
  while (i + 1 < E && s.tile0[i + 1] <= t) ++i;
  return i;
}

// Tile t (a pair tile when CG = 2) of slot `si` as seen by CTA `rank` of its pair.
// SG (SwiGLU, fwd only): output tile nt covers columns 128nt..128nt+127 of
// h [M, N/2]; its B rows are gate rows e*N + 128nt.. and up rows
// e*N + N/2 + 128nt.. (CTA pairs: rank 0 stages the gate rows, rank 1 the up rows).
//
// ST (CTA pairs, fwd/dgrad): a group whose row count is not a multiple of 256
// ends in a tile of r < 256 rows.  Padded to 256 rows it would cost a whole
// pair tile; instead the pair computes its transpose, Y_tail^T = W_half X_tail^T:
// A = the 256 B-operand rows of the output-column block (each CTA stages its
// 128, exactly as it would stage them as B), B = the tail's r tokens rounded
// up to 32 (MMA N, each CTA staging half), with the scale maps exchanged the
// same way.  The accumulator then holds output columns in its lanes and
// tokens in its columns, and the epilogue writes it back transposed.  The
// tensor work of the tile shrinks from 256 to round_up(r, 32) rows.
template <int CG, bool FP4 = false, bool SG = false, bool ST = false>
__device__ __forceinline__ Tile decode_tile(const Params& p, const Sched& s, int32_t t, int32_t si, uint32_t rank) {
  // K blocks are 128 bytes of codes: 128 E4M3 or 256 E2M1 elements; MMA steps
  // take 32 (E4M3) or 64 (E2M1) elements.  TMA x coordinates count bytes.
  constexpr int KE = FP4 ? 256 : 128, KSTEP = FP4 ? 64 : 32, EB = FP4 ? 2 : 1;   // EB: elements per byte
  constexpr int RPA = FP4 ? 64 : 128;   // colwise rows per scale atom column
  Tile tl;
  const int32_t e = s.slot[si];
  const int32_t row0 = s.off[e], m = s.off[e + 1] - s.off[e];
  const int32_t munits = group_m_units<CG>(p, m);
  const int32_t local = t - s.tile0[si];
  const int32_t mt = CG * (local % munits) + static_cast<int32_t>(rank);   // this CTA's 128-row block
  const int32_t nt = local / munits;
  const int32_t b_half = (CG == 2) ? BN / 2 * static_cast<int32_t>(rank) : 0;
  const int64_t L = p.mode == kFwd ? p.K : (p.mode == kDgrad ? p.N : m);
  tl.kblocks = static_cast<int32_t>((L + KE - 1) / KE);
  tl.ksteps_last = tl.kblocks > 0 ? static_cast<int32_t>((L - int64_t(KE) * (tl.kblocks - 1) + KSTEP - 1) / KSTEP) : 0;
  int64_t sfa_row, sfa_col, sfb_row, sfb_row1, sfb_col, out_cols;
  if (p.mode == kFwd) {
    tl.a_x = 0;                              tl.a_y = row0 + BM * mt;
    tl.b_x = 0;
    if constexpr (SG) {
      const int64_t I = p.N / 2;
      tl.b_y = static_cast<int32_t>(e * p.N + 128 * nt + (CG == 2 ? int64_t(rank) * I : 0));
      sfb_row = e * (p.N / 128) + nt;        sfb_row1 = sfb_row + I / 128;
      out_cols = I;
    } else {
      tl.b_y = static_cast<int32_t>(e * p.N) + BN * nt + b_half;
      sfb_row = e * (p.N / 128) + 2 * nt;    sfb_row1 = sfb_row + 1;
      out_cols = p.N;
    }
    sfa_row = s.rb[e] + mt;                  sfa_col = 0;
    sfb_col = 0;
    tl.q_rb = s.rb[e] + mt;                  tl.q_p = s.p[e] + BM * mt;
    tl.out_row = int64_t(row0) + BM * mt;
    tl.rows = static_cast<int32_t>(min64(BM, m - BM * mt));
  } else if (p.mode == kDgrad) {
    tl.a_x = 0;                              tl.a_y = row0 + BM * mt;
    tl.b_x = static_cast<int32_t>(e * p.N / EB); tl.b_y = BN * nt + b_half;
    sfa_row = s.rb[e] + mt;                  sfa_col = 0;
    sfb_row = 2 * nt;                        sfb_col = e * (p.N / RPA);
    sfb_row1 = sfb_row + 1;
    tl.q_rb = s.rb[e] + mt;                  tl.q_p = s.p[e] + BM * mt;
    tl.out_row = int64_t(row0) + BM * mt;
    tl.rows = static_cast<int32_t>(min64(BM, m - BM * mt));
    out_cols = p.K;
  } else {
    tl.a_x = s.p[e] / EB;                    tl.a_y = BM * mt;
    tl.b_x = s.p[e] / EB;                    tl.b_y = BN * nt + b_half;
    sfa_row = mt;                            sfa_col = FP4 ? s.q[e] : s.rb[e];
    sfb_row = 2 * nt;                        sfb_col = FP4 ? s.q[e] : s.rb[e];
    sfb_row1 = sfb_row + 1;
    tl.q_rb = 0;                             tl.q_p = 0;
    tl.out_row = int64_t(e) * p.N + BM * mt;
    tl.rows = static_cast<int32_t>(min64(BM, p.N - int64_t(BM) * mt));
    out_cols = p.K;
  }
  if (tl.rows < 0) tl.rows = 0;
  constexpr int OUT_W = SG ? BN / 2 : BN;   // output columns per tile
  tl.out_col = int64_t(OUT_W) * nt;
  tl.cols = static_cast<int32_t>(min64(OUT_W, out_cols - tl.out_col));
  tl.sfa_atom = sfa_row * p.sfa_pitch + sfa_col;
  tl.sfb_atom0 = sfb_row * p.sfb_pitch + sfb_col;
  tl.sfb_atom1 = sfb_row1 * p.sfb_pitch + sfb_col;
  tl.swapped = false;
  tl.ntok = 0;
  if constexpr (ST) {
    const int32_t mp = local % munits;   // the pair's 256-row block
    if (p.mode != kWgrad && mp == munits - 1 && (m & 255) != 0) {
      const int32_t r = m - 256 * mp;
      tl.swapped = true;
      tl.ntok = (r + 31) & ~31;
      // A slot <- this CTA's 128 B-operand rows (the B staging of a normal pair tile)
      tl.a_x = tl.b_x;
      tl.a_y = tl.b_y;
      // B slot <- this CTA's half of the tail tokens (rows of the A operand)
      tl.b_x = 0;
      tl.b_y = row0 + 256 * mp + static_cast<int32_t>(rank) * (tl.ntok / 2);
      // A scales: the atom of this CTA's B-operand half; B scales: the tail's two atom rows
      tl.sfa_atom = (rank == 0 ? tl.sfb_atom0 : tl.sfb_atom1);
      tl.sfb_atom0 = int64_t(s.rb[e] + 2 * mp) * p.sfa_pitch;
      tl.sfb_atom1 = tl.sfb_atom0 + p.sfa_pitch;
      tl.out_row = int64_t(row0) + 256 * mp;
      tl.q_rb = s.rb[e] + 2 * mp;            // the tail's first 128-row scale block
      tl.q_p = s.p[e] + 256 * mp;            // and its first colwise code column
      tl.rows = r;
      tl.out_col = int64_t(BN) * nt + 128 * static_cast<int32_t>(rank);
      tl.cols = static_cast<int32_t>(min64(128, out_cols - tl.out_col));
      if (tl.cols < 0) tl.cols = 0;
    }
  }
  return tl;
}

__device__ __forceinline__ void record_error(int32_t* status, int32_t code, volatile int* abort) {
  *abort = 1;
  atomicCAS(status, 0, code);
}

// Warp 0: validate the offsets and build the schedule.  Returns the total
// tile count (0 if the offsets are invalid).
template <int CG>
__device__ int32_t build_schedule(const Params& p, const Sched& s) {
  const int lane = threadIdx.x & 31;
  const int32_t ntl = n_tiles(p);
  int32_t carry_t = 0, carry_rb = 0, carry_p = 0, carry_q = 0;
  bool bad = false;
  for (int32_t base = 0; base < p.E; base += 32) {
    const int32_t h = base + lane;
    int32_t a = 0, b = 0;
    if (h < p.E) { a = __ldg(p.offs + h); b = __ldg(p.offs + h + 1); }
    bool lbad = (h < p.E) && (b < a || a < 0 || int64_t(b) > p.M);
    if (h == 0 && a != 0) lbad = true;
    if (h == p.E - 1 && int64_t(b) != p.M) lbad = true;
    bad |= __any_sync(0xffffffffu, lbad);
    const int32_t m = (h < p.E && !lbad) ? b - a : 0;
    const int32_t tiles = (h < p.E) ? group_m_units<CG>(p, m) * ntl : 0;
    const int32_t nb = (m + BM - 1) / BM, np = (m + 31) / 32 * 32, nq = (m + 63) / 64;
    int32_t st = tiles, sr = nb, sp = np, sq = nq;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int32_t x = __shfl_up_sync(0xffffffffu, st, d);
      const int32_t y = __shfl_up_sync(0xffffffffu, sr, d);
      const int32_t z = __shfl_up_sync(0xffffffffu, sp, d);
      const int32_t w = __shfl_up_sync(0xffffffffu, sq, d);
      if (lane >= d) { st += x; sr += y; sp += z; sq += w; }
    }
    if (h < p.E) {
      s.tile0[h] = carry_t + st - tiles;
      s.rb[h] = carry_rb + sr - nb;
      s.p[h] = carry_p + sp - np;
      s.q[h] = carry_q + sq - nq;
      s.off[h] = a;
      if (h == p.E - 1) { s.off[p.E] = b; s.tile0[p.E] = carry_t + st; }
    }
    carry_t = __shfl_sync(0xffffffffu, carry_t + st, 31);
    carry_rb = __shfl_sync(0xffffffffu, carry_rb + sr, 31);
    carry_p = __shfl_sync(0xffffffffu, carry_p + sp, 31);
    carry_q = __shfl_sync(0xffffffffu, carry_q + sq, 31);
  }
  if (bad) {
    if (lane == 0 && blockIdx.x == 0) atomicCAS(p.status, 0, static_cast<int32_t>(MXF8_ERR_BAD_OFFSETS));
    return 0;
  }
  if (p.mode != kWgrad) {
    for (int32_t h = lane; h < p.E; h += 32) s.slot[h] = h;
    return carry_t;
  }
  // wgrad: slot order = decreasing rows (ties by expert index), then the
  // tile prefix in slot order
  __syncwarp();
  for (int32_t h = lane; h < p.E; h += 32) {
    const int32_t mh = s.off[h + 1] - s.off[h];
    int32_t r = 0;
    for (int32_t g = 0; g < p.E; ++g) {
      const int32_t mg = s.off[g + 1] - s.off[g];
      r += (mg > mh || (mg == mh && g < h)) ? 1 : 0;
    }
    s.slot[r] = h;
  }
  __syncwarp();
  carry_t = 0;
  for (int32_t base = 0; base < p.E; base += 32) {
    const int32_t i = base + lane;
    int32_t tiles = 0;
    if (i < p.E) {
      const int32_t e = s.slot[i];
      tiles = group_m_units<CG>(p, s.off[e + 1] - s.off[e]) * ntl;
    }
    int32_t st = tiles;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int32_t x = __shfl_up_sync(0xffffffffu, st, d);
      if (lane >= d) st += x;
    }
    if (i < p.E) s.tile0[i] = carry_t + st - tiles;
    if (i == p.E - 1) s.tile0[p.E] = carry_t + st;
    carry_t = __shfl_sync(0xffffffffu, carry_t + st, 31);
  }
  return carry_t;
}

// tcgen05.wait::ld, tied to the registers the outstanding loads write so that
// no use of them can be scheduled before the wait.
__device__ __forceinline__ void tmem_wait_regs(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                 "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),
                 "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),
                 "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}

template <int CG, int KS, bool QE, bool FP4, bool SG>
__global__ void __launch_bounds__(NUM_THREADS, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                    const __grid_constant__ CUtensorMap tmOut, const Params p) {
  using C = Cfg<CG, KS, FP4>;
  constexpr int STAGES = C::STAGES;
  constexpr bool ST = CG == 2 && !SG;   // swapped ragged last tiles (see decode_tile)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = (CG == 2) ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int32_t unit0 = (CG == 2) ? static_cast<int32_t>(blockIdx.x >> 1) : static_cast<int32_t>(blockIdx.x);
  const int32_t nunits = (CG == 2) ? static_cast<int32_t>(gridDim.x >> 1) : static_cast<int32_t>(gridDim.x);

  const uint32_t bar0 = smem_addr(smem + C::OFF_BAR);
  auto full_bar = [&](uint32_t s) { return bar0 + 8 * s; };
  auto empty_bar = [&](uint32_t s) { return bar0 + 8 * (STAGES + s); };
  const uint32_t acc_full = bar0 + 8 * (2 * STAGES);
  const uint32_t acc_empty = bar0 + 8 * (2 * STAGES + 1);   // used in the leader CTA
  const uint32_t drain_bar = bar0 + 8 * (2 * STAGES + 2);
  volatile int32_t* misc = reinterpret_cast<volatile int32_t*>(smem + C::OFF_MISC);
  // misc[0]: tensor-memory base, misc[1]: abort flag, misc[2]: total tiles
  Sched sc;
  int32_t* sched = reinterpret_cast<int32_t*>(smem + C::OFF_SCHED);
  sc.tile0 = sched;
  sc.off = sched + (MAXG + 1);
  sc.rb = sched + 2 * (MAXG + 1);
  sc.p = sched + 3 * (MAXG + 1);
  sc.q = sched + 4 * (MAXG + 1);
  sc.slot = sched + 5 * (MAXG + 1);

  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < STAGES; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
      mbar_init(acc_full, 1);
      mbar_init(acc_empty, CG * 4);   // one arrival per epilogue warp
      mbar_init(drain_bar, 1);
      fence_barrier_init();
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmB);
      prefetch_tmap(&tmSFA);
      prefetch_tmap(&tmSFB);
      prefetch_tmap(&tmOut);
      misc[1] = 0;
    }
    const int32_t total = build_schedule<CG>(p, sc);
    if (lane == 0) misc[2] = total;
  } else if (warp == 1) {
    if constexpr (CG == 2) {
      tmem_alloc_pair(smem_addr(const_cast<int32_t*>(misc)), TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_addr(const_cast<int32_t*>(misc)), TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (CG == 2) cluster_sync();   // peer barriers initialised before any cross-CTA signal
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc[0]);
  const int32_t total = misc[2];
  volatile int* abort_flag = reinterpret_cast<volatile int*>(const_cast<int32_t*>(misc) + 1);
  volatile int never = 0;
  const uint64_t lim = p.timeout_ns;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer (every CTA)
      uint32_t it = 0, s = 0, ph = 0;
      int32_t eh = 0;
      bool failed = false;
      // Test hook: stage 0 gets neither its copies nor its arrival (in both
      // CTAs of a pair), so the MMA warp's bounded wait on it runs out; the
      // drain below skips it.
      const bool skip0 = p.inject_skip_stage != 0;
      for (int32_t t = unit0; t < total && !failed; t += nunits) {
        eh = advance_group(sc, p.E, t, eh);
        const Tile tl = decode_tile<CG, FP4, SG, ST>(p, sc, t, eh, rank);
        for (int32_t kb0 = 0; kb0 < tl.kblocks; kb0 += C::KS) {
          if (!mbar_wait(empty_bar(s), ph ^ 1, abort_flag, lim)) {
            record_error(p.status, MXF8_ERR_TIMEOUT, abort_flag);
            failed = true;
            break;
          }
          if (skip0 && it == 0) {
            ++it;
            if (++s == STAGES) { s = 0; ph ^= 1; }
            continue;
          }
          const int32_t nh = min(C::KS, tl.kblocks - kb0);   // K blocks in this stage
          const uint32_t fb = full_bar(s);
          const uint32_t ssa = smem_addr(smem + C::OFF_SFA + s * C::KS * C::SFA_T);
          const uint32_t ssb = smem_addr(smem + C::OFF_SFB + s * C::KS * C::SFB_T);
          // Scale atoms are 4 rows of 128 bytes in the scale maps; each box
          // takes the KS * APK consecutive atoms of the stage (those past the
          // tile's K blocks are fetched but unused; atoms past the buffer read
          // as zero).
          const int32_t ya = static_cast<int32_t>(4 * (tl.sfa_atom + C::APK * kb0));
          const int32_t yb0 = static_cast<int32_t>(4 * (tl.sfb_atom0 + C::APK * kb0));
          const int32_t yb1 = static_cast<int32_t>(4 * (tl.sfb_atom1 + C::APK * kb0));
          if constexpr (CG == 2) {
            if (leader) mbar_arrive_expect_tx(fb, C::stage_tx(nh));   // both CTAs' bytes land here
          } else {
            mbar_arrive_expect_tx(fb, C::stage_tx(nh));
          }
          for (int32_t h = 0; h < nh; ++h) {
            const uint32_t q = s * C::KS + h;
            const uint32_t sa = smem_addr(smem + C::OFF_A + q * C::A_TILE);
            const uint32_t sb = smem_addr(smem + C::OFF_B + q * C::B_TILE);
            const int32_t kx = BK * (kb0 + h);
            if constexpr (CG == 2) {
              // a swapped tile stages the B operand's rows in the A slot and its
              // tokens (a whole 128-row box, of which the MMA reads ntok / 2) in the B slot
              tma_load_2d_pair(sa, tl.swapped ? &tmB : &tmA, tl.a_x + kx, tl.a_y, fb);
              tma_load_2d_pair(sb, tl.swapped ? &tmA : &tmB, tl.b_x + kx, tl.b_y, fb);
            } else if constexpr (SG) {
              // gate rows, then the up rows N/2 further (two 128-row boxes)
              tma_load_2d(sa, &tmA, tl.a_x + kx, tl.a_y, fb);
              tma_load_2d(sb, &tmB, tl.b_x + kx, tl.b_y, fb);
              tma_load_2d(sb + 128 * BK, &tmB, tl.b_x + kx, tl.b_y + static_cast<int32_t>(p.N / 2), fb);
            } else {
              tma_load_2d(sa, &tmA, tl.a_x + kx, tl.a_y, fb);
              tma_load_2d(sb, &tmB, tl.b_x + kx, tl.b_y, fb);
            }
          }
          if constexpr (CG == 2) {
            const CUtensorMap* msa = tl.swapped ? &tmSFB : &tmSFA;
            const CUtensorMap* msb = tl.swapped ? &tmSFA : &tmSFB;
            tma_load_2d_pair(ssa, msa, 0, ya, fb);
            tma_load_2d_pair(ssb, msb, 0, yb0, fb);
            tma_load_2d_pair(ssb + C::KS * C::APK * 512, msb, 0, yb1, fb);
          } else {
            tma_load_2d(ssa, &tmSFA, 0, ya, fb);
            tma_load_2d(ssb, &tmSFB, 0, yb0, fb);
            tma_load_2d(ssb + C::KS * C::APK * 512, &tmSFB, 0, yb1, fb);
          }
          ++it;
          if (++s == STAGES) { s = 0; ph ^= 1; }
        }
      }
      if (failed || skip0) {
        // Let every copy already issued land before the CTA can exit (with the
        // test hook the MMA warp stops at stage 0 and never waits for the rest).
        if (leader) {
          for (uint32_t j = it > STAGES ? it - STAGES : 0; j < it; ++j)
            if (!(skip0 && j == 0)) mbar_wait(full_bar(j % STAGES), (j / STAGES) & 1, &never, lim);
        } else {
          for (int i = 0; i < 100; ++i) __nanosleep(1000);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------------------ MMA issuer (leader CTA)
      // Instruction descriptor: E4M3 x E4M3, E8M0 scales, K-major A and B,
      // M = 128*CG, N = 256; the scale-factor ids (bits 4-5 for B, 29-30 for
      // A) select the byte of the 32-bit scale column used by each K step.
      // FP4: E2M1 x E2M1 (format 1 in both fields), E4M3 scales (bit 23 clear),
      // K = 64 per MMA, the whole 32-bit scale column (4 blocks of 16) per MMA.
      const uint32_t idesc0 = FP4 ? ((1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) | (uint32_t((BM * CG) >> 4) << 24))
                                  : ((1u << 23) | (uint32_t(BN >> 3) << 17) | (uint32_t((BM * CG) >> 4) << 24));
      constexpr int KE = FP4 ? 256 : 128, KSTEP = FP4 ? 64 : 32;   // elements per K block / per MMA
      uint32_t kbc = 0;                                             // K blocks issued (FP4 scale set parity)
      // The tensor pipe queues only a few instructions, so scalar work between
      // MMAs stalls it: everything below is set up once, descriptors of a
      // slot are the base descriptor plus the slot's offset in 16-byte units
      // (the 14-bit start field cannot overflow below 256 KB), and the stage
      // index and phase advance incrementally.
      const uint64_t da0 = desc_kmajor_sw128(smem_addr(smem + C::OFF_A));
      const uint64_t db0 = desc_kmajor_sw128(smem_addr(smem + C::OFF_B));
      const uint64_t dsa0 = desc_sf_32x16(smem_addr(smem + C::OFF_SFA));
      const uint64_t dsb0 = desc_sf_32x16(smem_addr(smem + C::OFF_SFB));
      const uint32_t sf_t0 = tmem + C::SF_COL;
      // fwd/dgrad: every tile has the same K loop; wgrad: the group's rows.
      const int64_t L_fixed = p.mode == kFwd ? p.K : p.N;
      const int32_t kb_fixed = static_cast<int32_t>((L_fixed + KE - 1) / KE);
      const int32_t ks_fixed = static_cast<int32_t>((L_fixed - int64_t(KE) * (kb_fixed - 1) + KSTEP - 1) / KSTEP);
      uint32_t s = 0, ph = 0, j = 0;
      int32_t eh = 0;
      bool failed = false;
      for (int32_t t = unit0; t < total && !failed; t += nunits) {
        int32_t kblocks = kb_fixed, ksteps_last = ks_fixed;
        uint32_t idesc_t = idesc0;
        if constexpr (ST) {
          if (p.mode != kWgrad) {
            // a group's ragged last pair tile runs swapped with N = its tokens rounded up to 32
            eh = advance_group(sc, p.E, t, eh);
            const int32_t e = sc.slot[eh];
            const int32_t m = sc.off[e + 1] - sc.off[e];
            const int32_t munits = group_m_units<CG>(p, m);
            if ((t - sc.tile0[eh]) % munits == munits - 1 && (m & 255) != 0) {
              const uint32_t ntok = static_cast<uint32_t>((m - 256 * (munits - 1) + 31) & ~31);
              idesc_t = (idesc0 & ~(0x3Fu << 17)) | ((ntok >> 3) << 17);
            }
          }
        }
        if (p.mode == kWgrad) {
          eh = advance_group(sc, p.E, t, eh);
          const int32_t e = sc.slot[eh];
          const int32_t m = sc.off[e + 1] - sc.off[e];
          kblocks = (m + KE - 1) / KE;
          if (kblocks == 0) continue;
          ksteps_last = (m - KE * (kblocks - 1) + KSTEP - 1) / KSTEP;
        }
        const uint32_t d_tmem = tmem + (j & 1) * C::ACC_STRIDE;
        if (!mbar_wait(acc_empty, (j & 1) ^ 1, abort_flag, lim)) {
          record_error(p.status, MXF8_ERR_TIMEOUT, abort_flag);
          failed = true;
          break;
        }
        tc_fence_after();
        uint32_t acc = 0;
        // One K block of slot q (stage s, position h): its scale copies and
        // MMAs.  FULL (compile time): all four MMA steps, no predicates --
        // every K block but a tile's last; the tile's last takes nk steps.
        auto issue_kb = [&](uint32_t q, uint32_t st, int h, int32_t nk, auto full_tag) {
          constexpr bool FULL = decltype(full_tag)::value;
          const uint64_t da = da0 + (C::A_TILE >> 4) * q, db = db0 + (C::B_TILE >> 4) * q;
          if constexpr (FP4) {
            // four MMAs of K = 64, each with its own atoms: SFA atom i of the
            // stage's SFA box, SFB atoms i of its two SFB boxes
            const uint32_t set0 = sf_t0 + C::SF_SET_COLS * (kbc & 1);
            const uint64_t dsa = dsa0 + (C::SFA_T >> 4) * q;
            const uint64_t dsb = dsb0 + (C::SFB_T >> 4) * C::KS * st + (C::APK * 512 >> 4) * h;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              if (FULL || i < nk) {
                const uint32_t sfa_t = set0 + SF_STRIDE * i, sfb_t = sfa_t + 4;
                if constexpr (CG == 2) {
                  tc_cp_32x128b_x4_pair(sfa_t, dsa + (512 >> 4) * i);
                  tc_cp_32x128b_x4_pair(sfb_t, dsb + (512 >> 4) * i);
                  tc_cp_32x128b_x4_pair(sfb_t + 4, dsb + (512 >> 4) * (C::KS * C::APK + i));
                } else {
                  tc_cp_32x128b_x4(sfa_t, dsa + (512 >> 4) * i);
                  tc_cp_32x128b_x4(sfb_t, dsb + (512 >> 4) * i);
                  tc_cp_32x128b_x4(sfb_t + 4, dsb + (512 >> 4) * (C::KS * C::APK + i));
                }
              }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              if (FULL || i < nk) {
                const uint32_t sfa_t = set0 + SF_STRIDE * i, sfb_t = sfa_t + 4;
                if constexpr (CG == 2)
                  tc_mma_nvf4_pair(d_tmem, da + 2 * i, db + 2 * i, idesc_t, sfa_t, sfb_t, acc);
                else
                  tc_mma_nvf4(d_tmem, da + 2 * i, db + 2 * i, idesc_t, sfa_t, sfb_t, acc);
                acc = 1;
              }
            }
            ++kbc;
          } else {
            const uint32_t sfa_t = sf_t0 + SF_STRIDE * (C::SF_ALT ? (kbc & 1) : q), sfb_t = sfa_t + 4;
            ++kbc;
            const uint64_t dsa = dsa0 + (SFA_TILE >> 4) * q;
            const uint64_t dsb = dsb0 + (SFB_TILE >> 4) * C::KS * st + (512 >> 4) * h;
            if constexpr (CG == 2) {
              tc_cp_32x128b_x4_pair(sfa_t, dsa);
              tc_cp_32x128b_x4_pair(sfb_t, dsb);
              tc_cp_32x128b_x4_pair(sfb_t + 4, dsb + (512 >> 4) * C::KS);
            } else {
              tc_cp_32x128b_x4(sfa_t, dsa);
              tc_cp_32x128b_x4(sfb_t, dsb);
              tc_cp_32x128b_x4(sfb_t + 4, dsb + (512 >> 4) * C::KS);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              if (FULL || k < nk) {
                // +2 per step: the start-address field counts 16-byte units, one step is 32 bytes of K
                const uint32_t idesc = idesc_t | (uint32_t(k) << 4) | (uint32_t(k) << 29);
                if constexpr (CG == 2)
                  tc_mma_mxf8_pair(d_tmem, da + 2 * k, db + 2 * k, idesc, sfa_t | (uint32_t(k) << 30),
                                   sfb_t | (uint32_t(k) << 30), acc);
                else
                  tc_mma_mxf8(d_tmem, da + 2 * k, db + 2 * k, idesc, sfa_t | (uint32_t(k) << 30),
                              sfb_t | (uint32_t(k) << 30), acc);
                acc = 1;
              }
            }
          }
        };
        // Stages before the tile's last hold only full-depth K blocks.
        const int32_t last0 = ((kblocks - 1) / C::KS) * C::KS;   // first K block of the last stage
        for (int32_t kb0 = 0; kb0 <= last0; kb0 += C::KS) {
          if (!mbar_wait(full_bar(s), ph, abort_flag, lim)) {
            record_error(p.status, MXF8_ERR_TIMEOUT, abort_flag);
            failed = true;
            break;
          }
          tc_fence_after();
          if (kb0 < last0) {
#pragma unroll
            for (int h = 0; h < C::KS; ++h) issue_kb(s * C::KS + h, s, h, 4, std::true_type{});
          } else {
#pragma unroll
            for (int h = 0; h < C::KS; ++h) {
              const int32_t kb = kb0 + h;
              if (kb < kblocks) issue_kb(s * C::KS + h, s, h, kb == kblocks - 1 ? ksteps_last : 4, std::false_type{});
            }
          }
          if constexpr (CG == 2) tc_commit_pair(empty_bar(s), 0x3);
          else tc_commit(empty_bar(s));
          if (++s == STAGES) { s = 0; ph ^= 1; }
        }
        if (failed) break;
        if constexpr (CG == 2) tc_commit_pair(acc_full, 0x3);
        else tc_commit(acc_full);
        ++j;
      }
      if (failed) {
        // Wait for the MMAs and copies already issued before freeing tensor memory.
        if constexpr (CG == 2) tc_commit_pair(drain_bar, 0x1);
        else tc_commit(drain_bar);
        mbar_wait(drain_bar, 0, &never, lim);
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue (every CTA)
    const uint32_t quarter = warp & 3;   // tensor-memory lanes 32*quarter .. +31
    uint8_t* stage_base = smem + C::OFF_EPI + (warp - 2) * C::EPI_BUFS * EPI_STAGE;
    const int srow = lane >> 3, schunk = lane & 7;
    const int32_t row_base = 32 * static_cast<int32_t>(quarter);
    uint32_t j = 0, ec = 0;
    int32_t eh = 0;
    float oscale = 1.0f;   // FP4: 1 / (S_a * S_b), S = 2688 / amax (1 when amax = 0)
    if constexpr (FP4) {
      const float aa = __ldg(p.amax_a), ab = __ldg(p.amax_b);
      const float sa = aa == 0.0f ? 1.0f : __fdiv_rn(2688.0f, aa), sb = ab == 0.0f ? 1.0f : __fdiv_rn(2688.0f, ab);
      oscale = __frcp_rn(__fmul_rn(sa, sb));
    }
    for (int32_t t = unit0; t < total; t += nunits) {
      eh = advance_group(sc, p.E, t, eh);
      const Tile tl = decode_tile<CG, FP4, SG, ST>(p, sc, t, eh, rank);
      const int32_t vr = max(0, min(32, tl.rows - row_base));       // valid rows of this warp's slice
      uint16_t* out_tile = p.out + tl.out_row * p.out_ld + tl.out_col;
      if (tl.kblocks == 0) {
        // An expert without tokens: dW_e = 0.
        for (int c = 0; c < 4; ++c)
          for (int i = 0; i < 8; ++i) {
            const int rr = 4 * i + srow, col = 64 * c + 8 * schunk;
            if (rr < vr && col < tl.cols)
              *reinterpret_cast<uint4*>(out_tile + int64_t(row_base + rr) * p.out_ld + col) = make_uint4(0, 0, 0, 0);
          }
        continue;
      }
      if (!mbar_wait(acc_full, j & 1, abort_flag, lim)) {
        record_error(p.status, MXF8_ERR_TIMEOUT, abort_flag);
        break;
      }
      tc_fence_after();
      const uint32_t buf = j & 1;
      const uint32_t tbase = tmem + ((32 * quarter) << 16) + buf * C::ACC_STRIDE;
      // Every lane's tcgen05.ld has completed (wait::ld) before the warp
      // syncs; one lane then arrives for the warp.
      auto release = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (CG == 2) {
            if (leader) mbar_arrive(acc_empty); else mbar_arrive_cluster(acc_empty, 0);
          } else {
            mbar_arrive(acc_empty);
          }
        }
      };
      // Writes output chunk c (64 columns from tl.out_col + 64c, this warp's
      // 32 rows) from 64 packed bf16 values per lane: the bf16 output through
      // a swizzled stage (TMA store for a full slice, masked stores for a
      // group's ragged slice) and, in a quantising epilogue, its MXFP8 copies.
      auto emit = [&](const uint32_t (&pk)[32], int c) {
        uint32_t rs = 0, cs0 = 0, cs1 = 0;   // quantising epilogue: scale bytes (0 = pad)
        if (vr > 0 && 64 * c < tl.cols) {
          uint8_t* stg = stage_base + (ec % C::EPI_BUFS) * EPI_STAGE;
          uint4* st4 = reinterpret_cast<uint4*>(stg);
          if (lane == 0) bulk_wait_read<C::EPI_BUFS - 1>();   // the buffer's previous store has read it
          __syncwarp();
#pragma unroll
          for (int q = 0; q < 8; ++q)   // 128-byte swizzle: chunk q of row `lane` at q ^ (lane % 8)
            st4[lane * 8 + (q ^ (lane & 7))] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          if (!QE || p.out != nullptr) {
            if (vr == 32) {
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_2d(&tmOut, static_cast<int32_t>(tl.out_col + 64 * c),
                             static_cast<int32_t>(tl.out_row + row_base), smem_addr(stg));
                bulk_commit_group();
              }
            } else {
              __syncwarp();
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const int rr = 4 * i + srow, col = 64 * c + 8 * schunk;
                if (rr < vr && col < tl.cols)
                  *reinterpret_cast<uint4*>(out_tile + int64_t(row_base + rr) * p.out_ld + col) =
                      st4[rr * 8 + (schunk ^ (rr & 7))];
              }
            }
          }
          if constexpr (QE) {
            __syncwarp();
            if (p.qr != nullptr && lane < vr) {
              // Rowwise: this lane's row holds the chunk's two 32-blocks.
              uint8_t* qrow = p.qr + (tl.out_row + row_base + lane) * p.out_ld + tl.out_col + 64 * c;
#pragma unroll
              for (int b = 0; b < 2; ++b) {
                if (64 * c + 32 * b < tl.cols) {
                  const uint32_t* v = pk + 16 * b;
                  uint32_t m = 0;
#pragma unroll
                  for (int i = 0; i < 16; ++i) m = __vmaxu2(m, v[i] & 0x7FFF7FFFu);
                  const uint32_t sb = scale_byte(max(m & 0xFFFFu, m >> 16));
                  uint2 w[4];
#pragma unroll
                  for (int i = 0; i < 4; ++i) w[i] = encode8(make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]), sb);
                  *reinterpret_cast<uint4*>(qrow + 32 * b) = make_uint4(w[0].x, w[0].y, w[1].x, w[1].y);
                  *reinterpret_cast<uint4*>(qrow + 32 * b + 16) = make_uint4(w[2].x, w[2].y, w[3].x, w[3].y);
                  rs |= sb << (8 * b);
                }
              }
            }
            if (p.qc != nullptr && 64 * c + 2 * lane < tl.cols) {
              // Colwise: this lane takes columns 64c + 2*lane and +1 over the
              // warp's 32 rows, one group-relative 32-block (rows past the
              // group are pad: excluded from amax, code 0).
              const uint32_t* s32 = reinterpret_cast<const uint32_t*>(stg);
              uint32_t w[32], m = 0;
#pragma unroll
              for (int r = 0; r < 32; ++r) {
                w[r] = r < vr ? s32[r * 32 + (((lane >> 2) ^ (r & 7)) << 2) + (lane & 3)] : 0u;
                m = __vmaxu2(m, w[r] & 0x7FFF7FFFu);
              }
              cs0 = scale_byte(m & 0xFFFFu);
              cs1 = scale_byte(m >> 16);
              const float f0 = inv_scale(cs0 == 0xFFu ? 0u : cs0), f1 = inv_scale(cs1 == 0xFFu ? 0u : cs1);
              uint32_t o0[8], o1[8];
#pragma unroll
              for (int jj = 0; jj < 8; ++jj) {
                const uint32_t a0 = cvt_e4m3x2(__fmul_rn(bf_lo(w[4 * jj]), f0), __fmul_rn(bf_lo(w[4 * jj + 1]), f0));
                const uint32_t a1 = cvt_e4m3x2(__fmul_rn(bf_lo(w[4 * jj + 2]), f0), __fmul_rn(bf_lo(w[4 * jj + 3]), f0));
                const uint32_t b0 = cvt_e4m3x2(__fmul_rn(bf_hi(w[4 * jj]), f1), __fmul_rn(bf_hi(w[4 * jj + 1]), f1));
                const uint32_t b1 = cvt_e4m3x2(__fmul_rn(bf_hi(w[4 * jj + 2]), f1), __fmul_rn(bf_hi(w[4 * jj + 3]), f1));
                o0[jj] = cs0 == 0xFFu ? nan_codes4(jj, vr) : (a0 | (a1 << 16));
                o1[jj] = cs1 == 0xFFu ? nan_codes4(jj, vr) : (b0 | (b1 << 16));
              }
              uint8_t* qcol = p.qc + (tl.out_col + 64 * c + 2 * lane) * p.qc_ld + tl.q_p + row_base;
              reinterpret_cast<uint4*>(qcol)[0] = make_uint4(o0[0], o0[1], o0[2], o0[3]);
              reinterpret_cast<uint4*>(qcol)[1] = make_uint4(o0[4], o0[5], o0[6], o0[7]);
              reinterpret_cast<uint4*>(qcol + p.qc_ld)[0] = make_uint4(o1[0], o1[1], o1[2], o1[3]);
              reinterpret_cast<uint4*>(qcol + p.qc_ld)[1] = make_uint4(o1[4], o1[5], o1[6], o1[7]);
            }
          }
          __syncwarp();
          ++ec;
        }
        if constexpr (QE) {
          // Scale bytes, zeros included, for every atom this tile covers:
          // pad rows and blocks inside a written atom are 0x00.
          if (tl.rows > 0) {
            const int64_t col = tl.out_col + 64 * c;
            if (p.sr != nullptr && col / 128 < (p.out_ld + 127) / 128)
              *reinterpret_cast<uint16_t*>(p.sr + 512 * (int64_t(tl.q_rb) * ((p.out_ld + 127) / 128) + col / 128) +
                                           lane * 16 + quarter * 4 + 2 * (c & 1)) = static_cast<uint16_t>(rs);
            const int64_t n = col + 2 * lane;   // colwise: the output columns are the scale rows
            if (p.sc != nullptr && n / 128 < (p.out_ld + 127) / 128) {
              uint8_t* a = p.sc + 512 * ((n / 128) * p.sc_pitch + tl.q_rb) + ((n % 128) / 32) * 4 + quarter;
              a[(n % 32) * 16] = static_cast<uint8_t>(cs0);
              a[((n + 1) % 32) * 16] = static_cast<uint8_t>(cs1);
            }
          }
        }
      };
      if constexpr (ST) {
        if (tl.swapped) {
          // Swapped tile: lane n of this warp's quarter is output column
          // out_col + 32 * quarter + n, accumulator column i is token i.  Each
          // 32-token chunk goes through the warp's stage as a [32 tokens][32
          // columns] bf16 block (neighbouring lanes pair their columns with a
          // shuffle, so each lane stores 4-byte words; the 16-byte chunk q of
          // token row j sits at chunk q ^ (j / 2 % 4), which keeps both the
          // stores and the 16-byte row reads free of bank conflicts), then
          // leaves as 64-byte row segments (tokens past the group are not
          // written).  Chunks shared with the other accumulator are drained
          // first (buffer 0: the high ones, buffer 1: the low ones), then the
          // accumulator is released.
          // Quantising epilogue: a lane's 32 tokens of one column are that
          // column's colwise 32-block (encoded from registers; tokens past the
          // group are pad: out of the amax, code 0), and a stage row is one
          // token's rowwise 32-block (encoded by the lane that reads it back).
          // Every scale byte of the 128-token blocks the tile covers is
          // written, zero for pad tokens and blocks.
          const int nch = tl.ntok / 32;
          const int ov_lo = buf == 0 ? static_cast<int>(C::ACC_STRIDE / 32) : 0;
          const int ov_hi = buf == 0 ? 8 : static_cast<int>((256 - C::ACC_STRIDE) / 32);
          const int n_ov = max(0, min(nch, ov_hi) - ov_lo);
          if (n_ov == 0) release();
          int done_ov = 0;
          uint32_t* stg32 = reinterpret_cast<uint32_t*>(stage_base);
          const uint4* stg4 = reinterpret_cast<const uint4*>(stage_base);
          auto swz = [](int row, int q) { return row * 4 + (q ^ ((row >> 1) & 3)); };   // 16-byte chunk index
          if (lane == 0) bulk_wait_read<0>();   // an earlier tile's TMA store has read the stage
          __syncwarp();
          const bool col_ok = tl.cols > 32 * static_cast<int32_t>(quarter);
          const int64_t col_q = tl.out_col + 32 * quarter;   // this warp's first output column
          const int64_t n_col = col_q + lane;                 // this lane's output column
          const int64_t pitch_r = (p.out_ld + 127) / 128;     // rowwise atoms per atom row
          const bool atoms = tl.out_col / 128 < pitch_r;      // this CTA's columns own scale atoms
          // Scale bytes of token chunk jc: rowwise (token 32 jc + lane, block
          // `quarter` of this CTA's atom column), colwise (column n_col, 32-token
          // sub-block jc % 4).
          auto put_scales = [&](int jc, uint32_t rs, uint32_t cs) {
            if constexpr (QE) {
              if (!atoms) return;
              const int64_t rb = tl.q_rb + jc / 4;
              if (p.sr != nullptr)
                p.sr[512 * (rb * pitch_r + tl.out_col / 128) + lane * 16 + (jc & 3) * 4 + quarter] =
                    static_cast<uint8_t>(rs);
              if (p.sc != nullptr)
                p.sc[512 * ((n_col / 128) * p.sc_pitch + rb) + lane * 16 + quarter * 4 + (jc & 3)] =
                    static_cast<uint8_t>(cs);
            }
          };
#pragma unroll 1
          for (int i = 0; i < nch; ++i) {
            const int jc = buf == 0 ? nch - 1 - i : i;
            uint32_t v[32];
            tmem_ld_32x32b_x32(tbase + 32 * jc, v);
            tmem_wait_regs(v);
            if (jc >= ov_lo && jc < ov_hi && ++done_ov == n_ov) release();
            uint32_t rs = 0, cs = 0;
            if (col_ok) {
              uint32_t pk[16];   // bf16 tokens 2k (low half) and 2k + 1 of this lane's column
              const bool odd = lane & 1;
#pragma unroll
              for (int k = 0; k < 16; ++k) {
                float f0 = __uint_as_float(v[2 * k]), f1 = __uint_as_float(v[2 * k + 1]);
                if constexpr (FP4) { f0 = __fmul_rn(f0, oscale); f1 = __fmul_rn(f1, oscale); }
                pk[k] = cvt_bf16x2(f0, f1);
                // even lane: token 2k of columns (lane, lane + 1); odd lane: token 2k + 1 of (lane - 1, lane)
                const uint32_t other = __shfl_xor_sync(0xffffffffu, pk[k], 1);
                const uint32_t word = odd ? __byte_perm(other, pk[k], 0x7632) : __byte_perm(pk[k], other, 0x5410);
                const int row = 2 * k + (odd ? 1 : 0), w = lane >> 1;
                stg32[swz(row, w >> 2) * 4 + (w & 3)] = word;
              }
              if constexpr (QE) {
                if (p.qc != nullptr) {
                  const int valid = min(32, tl.rows - 32 * jc);   // real tokens of this 32-block
#pragma unroll
                  for (int k = 0; k < 16; ++k) {
                    if (2 * k >= valid) pk[k] = 0u;
                    else if (2 * k + 1 >= valid) pk[k] &= 0xFFFFu;
                  }
                  uint32_t a = 0;
#pragma unroll
                  for (int u = 0; u < 4; ++u)
                    a = max(a, amax_bits8(make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3])));
                  cs = scale_byte(a);
                  uint32_t o[8];
#pragma unroll
                  for (int u = 0; u < 4; ++u) {
                    const uint2 w = encode8(make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]), cs);
                    o[2 * u] = cs == 0xFFu ? nan_codes4(2 * u, valid) : w.x;
                    o[2 * u + 1] = cs == 0xFFu ? nan_codes4(2 * u + 1, valid) : w.y;
                  }
                  uint4* qcol = reinterpret_cast<uint4*>(p.qc + n_col * p.qc_ld + tl.q_p + 32 * jc);
                  qcol[0] = make_uint4(o[0], o[1], o[2], o[3]);
                  qcol[1] = make_uint4(o[4], o[5], o[6], o[7]);
                }
              }
              __syncwarp();
              if (p.out != nullptr) {
                uint16_t* out_q = p.out + tl.out_row * p.out_ld + col_q;
#pragma unroll
                for (int it = 0; it < 4; ++it) {
                  const int row = 8 * it + (lane >> 2), q = lane & 3;
                  const int32_t tok = 32 * jc + row;
                  if (tok < tl.rows)
                    *reinterpret_cast<uint4*>(out_q + int64_t(tok) * p.out_ld + 8 * q) = stg4[swz(row, q)];
                }
              }
              if constexpr (QE) {
                const int32_t tok = 32 * jc + lane;
                if (p.qr != nullptr && tok < tl.rows) {
                  const uint4 r0 = stg4[swz(lane, 0)], r1 = stg4[swz(lane, 1)], r2 = stg4[swz(lane, 2)],
                              r3 = stg4[swz(lane, 3)];
                  rs = scale_byte(max(max(amax_bits8(r0), amax_bits8(r1)), max(amax_bits8(r2), amax_bits8(r3))));
                  const uint2 w0 = encode8(r0, rs), w1 = encode8(r1, rs), w2 = encode8(r2, rs), w3 = encode8(r3, rs);
                  uint4* qrow = reinterpret_cast<uint4*>(p.qr + (tl.out_row + tok) * p.out_ld + col_q);
                  qrow[0] = make_uint4(w0.x, w0.y, w1.x, w1.y);
                  qrow[1] = make_uint4(w2.x, w2.y, w3.x, w3.y);
                }
              }
              __syncwarp();
            }
            put_scales(jc, rs, cs);
          }
          if constexpr (QE) {
            // the rest of the last 128-token block: pad tokens, zero scales
            for (int jc = nch; jc < (nch + 3) / 4 * 4; ++jc) put_scales(jc, 0u, 0u);
          }
          ++j;
          continue;
        }
      }
      if constexpr (SG) {
        // SwiGLU: accumulator columns 0-127 hold the gate, 128-255 the up
        // projection of the same 128 output columns; output chunk cc pairs
        // gate chunk cc with up chunk cc + 2.  The chunk shared with the other
        // accumulator goes first, so the release comes as early as it can.
        const int first = buf == 0 ? 1 : 0;
#pragma unroll 1
        for (int it = 0; it < 2; ++it) {
          const int cc = it == 0 ? first : 1 - first;
          uint32_t g0[32], g1[32], u0[32], u1[32];
          tmem_ld_32x32b_x32(tbase + 64 * cc, g0);
          tmem_ld_32x32b_x32(tbase + 64 * cc + 32, g1);
          tmem_ld_32x32b_x32(tbase + 64 * (cc + 2), u0);
          tmem_ld_32x32b_x32(tbase + 64 * (cc + 2) + 32, u1);
          tmem_wait_regs(g0);
          tmem_wait_regs(g1);
          tmem_wait_regs(u0);
          tmem_wait_regs(u1);
          if ((C::OV == 1 && it == 0) || it == 1) release();
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            pk[i] = cvt_bf16x2(swiglu_f32(__uint_as_float(g0[2 * i]), __uint_as_float(u0[2 * i])),
                               swiglu_f32(__uint_as_float(g0[2 * i + 1]), __uint_as_float(u0[2 * i + 1])));
            pk[16 + i] = cvt_bf16x2(swiglu_f32(__uint_as_float(g1[2 * i]), __uint_as_float(u1[2 * i])),
                                    swiglu_f32(__uint_as_float(g1[2 * i + 1]), __uint_as_float(u1[2 * i + 1])));
          }
          emit(pk, cc);
        }
      } else {
        // Accumulator 0's last OV chunks are accumulator 1's first OV chunks:
        // drain those first, then release the accumulator to the MMA issuer.
        auto chunk_of = [&](int ci) { return buf == 0 ? (ci + 4 - C::OV) & 3 : ci; };
        uint32_t ra0[32], ra1[32], rb0[32], rb1[32];
        tmem_ld_32x32b_x32(tbase + 64 * chunk_of(0), ra0);
        tmem_ld_32x32b_x32(tbase + 64 * chunk_of(0) + 32, ra1);
        tmem_wait_regs(ra0);
        tmem_wait_regs(ra1);
        if (C::OV == 1) release();
#pragma unroll
        for (int ci = 0; ci < 4; ++ci) {
          uint32_t(&c0)[32] = (ci & 1) ? rb0 : ra0;
          uint32_t(&c1)[32] = (ci & 1) ? rb1 : ra1;
          uint32_t(&n0)[32] = (ci & 1) ? ra0 : rb0;
          uint32_t(&n1)[32] = (ci & 1) ? ra1 : rb1;
          if (ci < 3) {   // next chunk's tensor-memory load overlaps this chunk's conversion and store
            tmem_ld_32x32b_x32(tbase + 64 * chunk_of(ci + 1), n0);
            tmem_ld_32x32b_x32(tbase + 64 * chunk_of(ci + 1) + 32, n1);
          }
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            if constexpr (FP4) {
              pk[i] = cvt_bf16x2(__fmul_rn(__uint_as_float(c0[2 * i]), oscale),
                                 __fmul_rn(__uint_as_float(c0[2 * i + 1]), oscale));
              pk[16 + i] = cvt_bf16x2(__fmul_rn(__uint_as_float(c1[2 * i]), oscale),
                                      __fmul_rn(__uint_as_float(c1[2 * i + 1]), oscale));
            } else {
              pk[i] = cvt_bf16x2(__uint_as_float(c0[2 * i]), __uint_as_float(c0[2 * i + 1]));
              pk[16 + i] = cvt_bf16x2(__uint_as_float(c1[2 * i]), __uint_as_float(c1[2 * i + 1]));
            }
          }
          emit(pk, chunk_of(ci));
          if (ci < 3) {
            tmem_wait_regs(n0);
            tmem_wait_regs(n1);
            if (ci + 2 == C::OV) release();   // chunk ci + 1 (the last shared one) is now in registers
          }
        }
      }
      ++j;
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  __syncwarp();
  tc_fence_before();
  if constexpr (CG == 2) cluster_sync();   // both CTAs are done with tensor memory
  else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (CG == 2) tmem_dealloc_pair(tmem, TMEM_COLS);
    else tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side
// Per device: SM count and, per kernel variant, whether its attributes are
// set and how many CTA pairs fit (cluster launches).
constexpr int kVariants = 32;   // CG x KS x QE x FP4 x SG
struct DeviceSetup {
  bool done[kVariants] = {};
  int num_sms = 0;
  int max_pairs[kVariants] = {};
};
DeviceSetup g_setup[64];

template <int CG, int KS, bool QE, bool FP4 = false, bool SG = false>
cudaError_t launch_cg(const Params& p, const CUtensorMap (&maps)[5], cudaStream_t stream) {
  using C = Cfg<CG, KS, FP4>;
  constexpr int V = (CG - 1) * 16 + (KS - 1) * 8 + int(QE) * 4 + int(FP4) * 2 + int(SG);
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  DeviceSetup& ds = g_setup[dev];
  auto kernel = grouped_gemm_kernel<CG, KS, QE, FP4, SG>;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  if (!ds.done[V]) {
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (err != cudaSuccess) return err;
    err = cudaDeviceGetAttribute(&ds.num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess) return err;
    if (CG == 2) {
      cudaLaunchConfig_t q = {};
      q.gridDim = dim3(2 * (ds.num_sms / 2));
      q.blockDim = dim3(NUM_THREADS);
      q.dynamicSmemBytes = C::SMEM_BYTES;
      q.attrs = attr;
      q.numAttrs = 1;
      int clusters = 0;
      err = cudaOccupancyMaxActiveClusters(&clusters, kernel, &q);
      if (err != cudaSuccess) return err;
      ds.max_pairs[V] = clusters > 0 ? clusters : 1;
    }
    ds.done[V] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  if (CG == 2) {
    cfg.gridDim = dim3(2 * ds.max_pairs[V]);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  } else {
    cfg.gridDim = dim3(ds.num_sms);
  }
  return cudaLaunchKernelEx(&cfg, kernel, maps[0], maps[1], maps[2], maps[3], maps[4], p);
}

}  // namespace

cudaError_t launch_grouped_gemm(const GemmArgs& a, cudaStream_t stream, const char** detail) {
  // Tile configuration, from sizes the host knows (the group sizes stay on
  // the device).  fwd/dgrad over long contractions (>= 32 K blocks) run CTA
  // pairs with 256-deep stages: pairs move 2/3 of the operand bytes per FLOP,
  // and each group's ragged last tile runs swapped with N = its tokens rounded
  // up to 32, so the padding stays small.  The SwiGLU epilogue has no swapped
  // tile (its pair tiles pad groups to 256 rows), so it takes pairs only where
  // groups average >= 768 rows over >= 40 K blocks.  Everything else runs
  // 1-CTA 128x256 tiles with 128-deep stages (on B200 these won every other
  // pass of the three MoE layers).  mxfp8_set_gemm_tiling overrides either choice.
  int force_cg = -1, force_ks = -1;
  gemm_tiling_override(&force_cg, &force_ks);
  int cg = 1, ks = 1;
  if (a.mode != kWgrad && !a.fp4) {
    const int64_t kblocks = ((a.mode == kFwd ? a.K : a.N) + BK - 1) / BK;
    if (a.swiglu ? (kblocks >= 40 && a.M >= int64_t(768) * a.E) : kblocks >= 32) { cg = 2; ks = 2; }
  }
  if (force_cg == 0 || force_cg == 1) cg = force_cg == 1 ? 2 : 1;
  if (force_ks == 1 || force_ks == 2) ks = force_ks;
  // NVFP4: 128-byte K blocks (256 elements) in single-block stages: 1-CTA tiles
  // (3 stages) unless mxfp8_set_gemm_tiling asks for CTA pairs (5 stages).
  // Pairs halve the operand bytes per FLOP but not the scale-factor copies
  // each SM receives (three per K = 64 MMA), which bound this kernel: on
  // B200 they measured 0.80-0.88x of the 1-CTA tiles on every pass.
  if (a.fp4) { ks = 1; cg = force_cg == 1 ? 2 : 1; }
  const uint32_t sf_box_rows = 4 * ks * (a.fp4 ? 4 : 1);
  const int64_t out_rows = a.mode == kWgrad ? int64_t(a.E) * a.N : a.M;
  const int64_t out_cols = a.mode == kFwd ? (a.swiglu ? a.N / 2 : a.N) : a.K;
  // B boxes: 128 rows when a CTA stages half of a 256-row B tile (pairs) or
  // the gate and up halves separately (SwiGLU), else the whole tile.
  const uint32_t b_box_rows = (cg == 2 || a.swiglu) ? BN / 2 : BN;
  CUtensorMap maps[5];
  const bool ok =
      make_tensor_map(&maps[0], a.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.a_rows, a.a_cols, a.lda, BK, BM,
               CU_TENSOR_MAP_SWIZZLE_128B) &&
      make_tensor_map(&maps[1], a.b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.b_rows, a.b_cols, a.ldb, BK, b_box_rows,
               CU_TENSOR_MAP_SWIZZLE_128B) &&
      make_tensor_map(&maps[2], a.sfa, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.sfa_atoms * 4, 128, 128, 128, sf_box_rows,
               CU_TENSOR_MAP_SWIZZLE_NONE) &&
      make_tensor_map(&maps[3], a.sfb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.sfb_atoms * 4, 128, 128, 128, sf_box_rows,
               CU_TENSOR_MAP_SWIZZLE_NONE) &&
      (a.out != nullptr
           ? make_tensor_map(&maps[4], a.out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, out_rows, out_cols, out_cols, 64, 32,
                      CU_TENSOR_MAP_SWIZZLE_128B)
           // no bf16 output (quantising epilogue only): a placeholder map over
           // the status word that the kernel never uses
           : make_tensor_map(&maps[4], a.status, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 1, 64, 64, 64, 32,
                      CU_TENSOR_MAP_SWIZZLE_128B));
  if (!ok) {
    if (detail) *detail = "cuTensorMapEncodeTiled failed";
    return cudaErrorInvalidValue;
  }
  Params p;
  p.mode = a.mode;
  p.E = a.E;
  p.M = a.M; p.N = a.N; p.K = a.K;
  p.offs = a.offs;
  p.sfa_pitch = a.sfa_pitch; p.sfb_pitch = a.sfb_pitch;
  p.out = a.out;
  p.out_ld = out_cols;
  p.status = a.status;
  p.timeout_ns = a.timeout_ns;
  p.inject_skip_stage = a.inject_skip_stage;
  p.qr = a.qr; p.sr = a.sr; p.qc = a.qc; p.sc = a.sc;
  p.qc_ld = a.qc_ld; p.sc_pitch = a.sc_pitch;
  p.amax_a = a.amax_a; p.amax_b = a.amax_b;
  if (a.fp4) return cg == 2 ? launch_cg<2, 1, false, true>(p, maps, stream) : launch_cg<1, 1, false, true>(p, maps, stream);
  if (a.swiglu) {
    if (cg == 2) return ks == 2 ? launch_cg<2, 2, true, false, true>(p, maps, stream)
                                : launch_cg<2, 1, true, false, true>(p, maps, stream);
    return ks == 2 ? launch_cg<1, 2, true, false, true>(p, maps, stream) : launch_cg<1, 1, true, false, true>(p, maps, stream);
  }
  const bool qe = a.qr != nullptr || a.qc != nullptr;
  if (qe) {
    if (cg == 2) return ks == 2 ? launch_cg<2, 2, true>(p, maps, stream) : launch_cg<2, 1, true>(p, maps, stream);
    return ks == 2 ? launch_cg<1, 2, true>(p, maps, stream) : launch_cg<1, 1, true>(p, maps, stream);
  }
  if (cg == 2) return ks == 2 ? launch_cg<2, 2, false>(p, maps, stream) : launch_cg<2, 1, false>(p, maps, stream);
  return ks == 2 ? launch_cg<1, 2, false>(p, maps, stream) : launch_cg<1, 1, false>(p, maps, stream);
}

}  // namespace mxf8
