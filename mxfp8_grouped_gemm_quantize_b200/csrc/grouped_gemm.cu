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
// the scales in hardware and accumulates in fp32 tensor memory.
//
// Structure (one CTA per SM, 192 threads):
//   warp 0   TMA producer: per 128-wide K block, A 128x128 and B 256x128 code
//            tiles (128-byte swizzle) and three 512-byte scale atoms into a
//            4-stage shared-memory ring.
//   warp 1   allocates 512 tensor-memory columns; one thread copies the scale
//            atoms to tensor memory (tcgen05.cp 32x128b.warpx4) and issues the
//            128x256x32 MMAs; tcgen05.commit releases ring stages and signals
//            a finished accumulator.
//   warps 2-5 epilogue: tensor memory -> registers -> bf16 -> shared (swizzled)
//            -> coalesced 16-byte global stores, masked to the group's real
//            rows and the matrix columns.
// Two 128x256 fp32 accumulators overlap in 64 columns (0..255 and 192..447),
// which leaves columns 448..511 for per-stage scale factors; the epilogue
// drains the shared 64 columns first and then releases the accumulator, so
// the next tile's MMAs overlap the rest of the epilogue.
// The tile schedule is built on the device from the group offsets at kernel
// start (no host synchronisation); tiles are dealt round-robin to the CTAs.
// Every wait is bounded: on timeout the kernel records MXF8_ERR_TIMEOUT,
// drains its in-flight copies and MMAs, frees tensor memory and exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include "launch.h"
#include "mxfp8.h"
#include "ptx.cuh"

namespace mxf8 {
namespace {

constexpr int BM = 128, BN = 256, BK = 128, STAGES = 4;
constexpr int A_TILE = BM * BK;            // 16 KB of E4M3 codes
constexpr int B_TILE = BN * BK;            // 32 KB
constexpr int SFA_TILE = 512, SFB_TILE = 1024;
constexpr uint32_t STAGE_TX = A_TILE + B_TILE + SFA_TILE + SFB_TILE;
constexpr int NUM_THREADS = 192;
constexpr int EPI_STAGE = 32 * 128;        // per epilogue warp: 32 rows x 64 bf16
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_STRIDE = 192;       // accumulator 1 starts at column 192
constexpr uint32_t SF_COL = 448;           // stage s: SFA at 448 + 16 s (4 columns), SFB at +4 (8 columns)
constexpr uint32_t SF_STRIDE = 16;
constexpr int MAXG = MXF8_GEMM_MAX_GROUPS;

// Shared-memory map (offsets from a 1024-byte aligned base).
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * A_TILE;
constexpr int OFF_SFA = OFF_B + STAGES * B_TILE;
constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_TILE;
constexpr int OFF_EPI = OFF_SFB + STAGES * SFB_TILE;
constexpr int OFF_BAR = OFF_EPI + 4 * EPI_STAGE;
constexpr int NUM_BARS = 2 * STAGES + 3;   // full[S], empty[S], acc_full, acc_empty, drain
constexpr int OFF_MISC = OFF_BAR + 128;
constexpr int OFF_SCHED = OFF_MISC + 64;
constexpr int SCHED_INTS = 4 * (MAXG + 1);
constexpr int SMEM_USED = OFF_SCHED + SCHED_INTS * 4;
constexpr int SMEM_BYTES = SMEM_USED + 1024;   // slack for aligning the base
static_assert(NUM_BARS * 8 <= 128, "barrier area");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
static_assert(OFF_B % 1024 == 0 && OFF_SFA % 1024 == 0, "swizzled tiles need 1024-byte alignment");
static_assert(SF_COL + SF_STRIDE * (STAGES - 1) + 12 <= TMEM_COLS, "scale columns");
static_assert(ACC_STRIDE + BN <= SF_COL, "accumulators must not reach the scale columns");

struct Params {
  int mode;
  int32_t E;
  int64_t M, N, K;
  const int32_t* offs;
  const uint8_t* sfa;
  const uint8_t* sfb;
  int64_t sfa_pitch, sfb_pitch, sfa_atoms, sfb_atoms;
  uint16_t* out;
  int32_t* status;
  uint64_t timeout_ns;
};

// Per-CTA schedule, built from the offsets by warp 0.
struct Sched {
  int32_t* tile0;   // [E+1] first tile of each group (prefix)
  int32_t* off;     // [E+1] row offsets
  int32_t* rb;      // [E]   RB_e: 128-row blocks before group e (rowwise scale rows,
                    //       colwise scale block-columns / 4)
  int32_t* p;       // [E]   P_e: 32-padded rows before group e (colwise code column)
};

struct Tile {
  int32_t e, mt, nt;
  int32_t kblocks;       // 128-wide K blocks (0: nothing to accumulate)
  int32_t ksteps_last;   // 32-wide MMA steps in the last K block
  int32_t a_x, a_y, b_x, b_y;           // TMA coordinates of the first K block
  int64_t sfa_row, sfa_col, sfb_row, sfb_col;   // scale atom (row, column) of the first K block
  uint16_t* out;         // output element (0, 0) of the tile
  int64_t ld;            // output row stride (elements)
  int32_t rows, cols;    // valid rows (<= 128) and columns (<= 256) of the tile
};

__device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

__device__ __forceinline__ int32_t cdiv32(int64_t a, int64_t b) { return static_cast<int32_t>((a + b - 1) / b); }

__device__ __forceinline__ int32_t group_m_tiles(const Params& p, int32_t m) {
  return p.mode == kWgrad ? cdiv32(p.N, BM) : cdiv32(m, BM);
}

__device__ __forceinline__ int32_t n_tiles(const Params& p) {
  return p.mode == kFwd ? cdiv32(p.N, BN) : cdiv32(p.K, BN);
}

__device__ __forceinline__ Tile decode_tile(const Params& p, const Sched& s, int32_t t) {
  int32_t lo = 0, hi = p.E - 1;   // last group whose first tile is <= t
  while (lo < hi) {
    const int32_t mid = (lo + hi + 1) >> 1;
    if (s.tile0[mid] <= t) lo = mid; else hi = mid - 1;
  }
  Tile tl;
  const int32_t e = lo;
  const int32_t row0 = s.off[e], m = s.off[e + 1] - s.off[e];
  const int32_t mtiles = group_m_tiles(p, m);
  const int32_t local = t - s.tile0[e];
  tl.e = e;
  tl.mt = local % mtiles;
  tl.nt = local / mtiles;
  const int64_t L = p.mode == kFwd ? p.K : (p.mode == kDgrad ? p.N : m);
  tl.kblocks = static_cast<int32_t>((L + BK - 1) / BK);
  tl.ksteps_last = tl.kblocks > 0 ? static_cast<int32_t>((L - int64_t(BK) * (tl.kblocks - 1) + 31) / 32) : 0;
  if (p.mode == kFwd) {
    tl.a_x = 0;            tl.a_y = row0 + BM * tl.mt;
    tl.b_x = 0;            tl.b_y = static_cast<int32_t>(e * p.N) + BN * tl.nt;
    tl.sfa_row = s.rb[e] + tl.mt;                 tl.sfa_col = 0;
    tl.sfb_row = e * (p.N / 128) + 2 * tl.nt;     tl.sfb_col = 0;
    tl.out = p.out + (int64_t(row0) + BM * tl.mt) * p.N + BN * tl.nt;
    tl.ld = p.N;
    tl.rows = min(BM, m - BM * tl.mt);
    tl.cols = static_cast<int32_t>(min64(BN, p.N - int64_t(BN) * tl.nt));
  } else if (p.mode == kDgrad) {
    tl.a_x = 0;                                   tl.a_y = row0 + BM * tl.mt;
    tl.b_x = static_cast<int32_t>(e * p.N);       tl.b_y = BN * tl.nt;
    tl.sfa_row = s.rb[e] + tl.mt;                 tl.sfa_col = 0;
    tl.sfb_row = 2 * tl.nt;                       tl.sfb_col = e * (p.N / 128);
    tl.out = p.out + (int64_t(row0) + BM * tl.mt) * p.K + BN * tl.nt;
    tl.ld = p.K;
    tl.rows = min(BM, m - BM * tl.mt);
    tl.cols = static_cast<int32_t>(min64(BN, p.K - int64_t(BN) * tl.nt));
  } else {
    tl.a_x = s.p[e];       tl.a_y = BM * tl.mt;
    tl.b_x = s.p[e];       tl.b_y = BN * tl.nt;
    tl.sfa_row = tl.mt;                           tl.sfa_col = s.rb[e];
    tl.sfb_row = 2 * tl.nt;                       tl.sfb_col = s.rb[e];
    tl.out = p.out + int64_t(e) * p.N * p.K + int64_t(BM) * tl.mt * p.K + BN * tl.nt;
    tl.ld = p.K;
    tl.rows = static_cast<int32_t>(min64(BM, p.N - int64_t(BM) * tl.mt));
    tl.cols = static_cast<int32_t>(min64(BN, p.K - int64_t(BN) * tl.nt));
  }
  return tl;
}

// Scale atom address, clamped into the buffer: atoms that fall outside it
// only ever feed masked output rows/columns.
__device__ __forceinline__ const uint8_t* atom_ptr(const uint8_t* base, int64_t row, int64_t col,
                                                   int64_t pitch, int64_t atoms) {
  int64_t a = row * pitch + col;
  a = a < 0 ? 0 : (a >= atoms ? atoms - 1 : a);
  return base + a * 512;
}

__device__ __forceinline__ void record_error(int32_t* status, int32_t code, volatile int* abort) {
  *abort = 1;
  atomicCAS(status, 0, code);
}

// Warp 0: validate the offsets and build the schedule.  Returns the total
// tile count (0 if the offsets are invalid).
__device__ int32_t build_schedule(const Params& p, const Sched& s) {
  const int lane = threadIdx.x & 31;
  const int32_t ntl = n_tiles(p);
  int32_t carry_t = 0, carry_rb = 0, carry_p = 0;
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
    const int32_t tiles = (h < p.E) ? group_m_tiles(p, m) * ntl : 0;
    const int32_t nb = (m + BM - 1) / BM, np = (m + 31) / 32 * 32;
    int32_t st = tiles, sr = nb, sp = np;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int32_t x = __shfl_up_sync(0xffffffffu, st, d);
      const int32_t y = __shfl_up_sync(0xffffffffu, sr, d);
      const int32_t z = __shfl_up_sync(0xffffffffu, sp, d);
      if (lane >= d) { st += x; sr += y; sp += z; }
    }
    if (h < p.E) {
      s.tile0[h] = carry_t + st - tiles;
      s.rb[h] = carry_rb + sr - nb;
      s.p[h] = carry_p + sp - np;
      s.off[h] = a;
      if (h == p.E - 1) { s.off[p.E] = b; s.tile0[p.E] = carry_t + st; }
    }
    carry_t = __shfl_sync(0xffffffffu, carry_t + st, 31);
    carry_rb = __shfl_sync(0xffffffffu, carry_rb + sr, 31);
    carry_p = __shfl_sync(0xffffffffu, carry_p + sp, 31);
  }
  if (bad) {
    if (lane == 0 && blockIdx.x == 0) atomicCAS(p.status, 0, static_cast<int32_t>(MXF8_ERR_BAD_OFFSETS));
    return 0;
  }
  return carry_t;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const uint32_t bar0 = smem_addr(smem + OFF_BAR);
  auto full_bar = [&](uint32_t s) { return bar0 + 8 * s; };
  auto empty_bar = [&](uint32_t s) { return bar0 + 8 * (STAGES + s); };
  const uint32_t acc_full = bar0 + 8 * (2 * STAGES);
  const uint32_t acc_empty = bar0 + 8 * (2 * STAGES + 1);
  const uint32_t drain_bar = bar0 + 8 * (2 * STAGES + 2);
  volatile int32_t* misc = reinterpret_cast<volatile int32_t*>(smem + OFF_MISC);
  // misc[0]: tensor-memory base, misc[1]: abort flag, misc[2]: total tiles
  Sched sc;
  int32_t* sched = reinterpret_cast<int32_t*>(smem + OFF_SCHED);
  sc.tile0 = sched;
  sc.off = sched + (MAXG + 1);
  sc.rb = sched + 2 * (MAXG + 1);
  sc.p = sched + 3 * (MAXG + 1);

  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < STAGES; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
      mbar_init(acc_full, 1);
      mbar_init(acc_empty, 4 * 32);
      mbar_init(drain_bar, 1);
      fence_barrier_init();
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmB);
      misc[1] = 0;
    }
    const int32_t total = build_schedule(p, sc);
    if (lane == 0) misc[2] = total;
  } else if (warp == 1) {
    tmem_alloc(smem_addr(const_cast<int32_t*>(misc)), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc[0]);
  const int32_t total = misc[2];
  volatile int* abort_flag = reinterpret_cast<volatile int*>(const_cast<int32_t*>(misc) + 1);
  volatile int never = 0;
  const uint64_t lim = p.timeout_ns;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      uint32_t it = 0;
      bool failed = false;
      for (int32_t t = blockIdx.x; t < total && !failed; t += gridDim.x) {
        const Tile tl = decode_tile(p, sc, t);
        for (int32_t kb = 0; kb < tl.kblocks; ++kb) {
          const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
          if (!mbar_wait(empty_bar(s), ph ^ 1, abort_flag, lim)) {
            record_error(p.status, MXF8_ERR_TIMEOUT, abort_flag);
            failed = true;
            break;
          }
          const uint32_t fb = full_bar(s);
          mbar_arrive_expect_tx(fb, STAGE_TX);
          tma_load_2d(smem_addr(smem + OFF_A + s * A_TILE), &tmA, tl.a_x + BK * kb, tl.a_y, fb);
          tma_load_2d(smem_addr(smem + OFF_B + s * B_TILE), &tmB, tl.b_x + BK * kb, tl.b_y, fb);
          bulk_load(smem_addr(smem + OFF_SFA + s * SFA_TILE),
                    atom_ptr(p.sfa, tl.sfa_row, tl.sfa_col + kb, p.sfa_pitch, p.sfa_atoms), 512, fb);
          bulk_load(smem_addr(smem + OFF_SFB + s * SFB_TILE),
                    atom_ptr(p.sfb, tl.sfb_row, tl.sfb_col + kb, p.sfb_pitch, p.sfb_atoms), 512, fb);
          bulk_load(smem_addr(smem + OFF_SFB + s * SFB_TILE + 512),
                    atom_ptr(p.sfb, tl.sfb_row + 1, tl.sfb_col + kb, p.sfb_pitch, p.sfb_atoms), 512, fb);
          ++it;
        }
      }
      if (failed) {
        // Let every copy already issued land before the CTA can exit.
        for (uint32_t j = it > STAGES ? it - STAGES : 0; j < it; ++j)
          mbar_wait(full_bar(j % STAGES), (j / STAGES) & 1, &never, lim);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      // Instruction descriptor: E4M3 x E4M3, E8M0 scales, K-major A and B,
      // M = 128, N = 256; the scale-factor ids (bits 4-5 for B, 29-30 for A)
      // select the byte of the 32-bit scale column used by each K step.
      const uint32_t idesc0 = (1u << 23) | (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);
      uint32_t it = 0, j = 0;
      bool failed = false;
      for (int32_t t = blockIdx.x; t < total && !failed; t += gridDim.x) {
        const Tile tl = decode_tile(p, sc, t);
        if (tl.kblocks == 0) continue;
        const uint32_t d_tmem = tmem + (j & 1) * ACC_STRIDE;
        if (!mbar_wait(acc_empty, (j & 1) ^ 1, abort_flag, lim)) {
          record_error(p.status, MXF8_ERR_TIMEOUT, abort_flag);
          failed = true;
          break;
        }
        tc_fence_after();
        for (int32_t kb = 0; kb < tl.kblocks; ++kb) {
          const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
          if (!mbar_wait(full_bar(s), ph, abort_flag, lim)) {
            record_error(p.status, MXF8_ERR_TIMEOUT, abort_flag);
            failed = true;
            break;
          }
          tc_fence_after();
          const uint32_t sfa_t = tmem + SF_COL + SF_STRIDE * s, sfb_t = sfa_t + 4;
          tc_cp_32x128b_x4(sfa_t, desc_sf_32x16(smem_addr(smem + OFF_SFA + s * SFA_TILE)));
          tc_cp_32x128b_x4(sfb_t, desc_sf_32x16(smem_addr(smem + OFF_SFB + s * SFB_TILE)));
          tc_cp_32x128b_x4(sfb_t + 4, desc_sf_32x16(smem_addr(smem + OFF_SFB + s * SFB_TILE + 512)));
          const uint64_t da = desc_kmajor_sw128(smem_addr(smem + OFF_A + s * A_TILE));
          const uint64_t db = desc_kmajor_sw128(smem_addr(smem + OFF_B + s * B_TILE));
          const int32_t nk = (kb == tl.kblocks - 1) ? tl.ksteps_last : BK / 32;
          for (int32_t k = 0; k < nk; ++k) {
            const uint32_t idesc = idesc0 | (uint32_t(k) << 4) | (uint32_t(k) << 29);
            // +2 per step: the start-address field counts 16-byte units, one step is 32 bytes of K
            tc_mma_mxf8(d_tmem, da + 2 * k, db + 2 * k, idesc, sfa_t | (uint32_t(k) << 30),
                        sfb_t | (uint32_t(k) << 30), (kb | k) != 0);
          }
          tc_commit(empty_bar(s));
          ++it;
        }
        if (failed) break;
        tc_commit(acc_full);
        ++j;
      }
      if (failed) {
        // Wait for the MMAs and copies already issued before freeing tensor memory.
        tc_commit(drain_bar);
        mbar_wait(drain_bar, 0, &never, lim);
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const uint32_t quarter = warp & 3;   // tensor-memory lanes 32*quarter .. +31
    uint4* stage = reinterpret_cast<uint4*>(smem + OFF_EPI + (warp - 2) * EPI_STAGE);
    const int srow = lane >> 3, schunk = lane & 7;
    uint32_t j = 0;
    for (int32_t t = blockIdx.x; t < total; t += gridDim.x) {
      const Tile tl = decode_tile(p, sc, t);
      const int32_t row_base = 32 * quarter;
      if (tl.kblocks == 0) {
        // An expert without tokens: dW_e = 0.
        for (int c = 0; c < 4; ++c)
          for (int i = 0; i < 8; ++i) {
            const int r = row_base + 4 * i + srow, col = 64 * c + 8 * schunk;
            if (r < tl.rows && col < tl.cols)
              *reinterpret_cast<uint4*>(tl.out + int64_t(r) * tl.ld + col) = make_uint4(0, 0, 0, 0);
          }
        continue;
      }
      if (!mbar_wait(acc_full, j & 1, abort_flag, lim)) {
        record_error(p.status, MXF8_ERR_TIMEOUT, abort_flag);
        break;
      }
      tc_fence_after();
      const uint32_t buf = j & 1;
      for (int ci = 0; ci < 4; ++ci) {
        // Buffer 0 shares its last 64 columns with buffer 1's first 64: drain them first.
        const int c = buf == 0 ? (ci + 3) & 3 : ci;
        const uint32_t taddr = tmem + ((32 * quarter) << 16) + buf * ACC_STRIDE + 64 * c;
        uint32_t r0[32], r1[32];
        tmem_ld_32x32b_x32(taddr, r0);
        tmem_ld_32x32b_x32(taddr + 32, r1);
        tmem_ld_wait();
        if (ci == 0) {
          tc_fence_before();
          mbar_arrive(acc_empty);
        }
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          pk[i] = cvt_bf16x2(__uint_as_float(r0[2 * i]), __uint_as_float(r0[2 * i + 1]));
          pk[16 + i] = cvt_bf16x2(__uint_as_float(r1[2 * i]), __uint_as_float(r1[2 * i + 1]));
        }
#pragma unroll
        for (int q = 0; q < 8; ++q)
          stage[lane * 8 + (q ^ (lane & 7))] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int rr = 4 * i + srow;
          const int r = row_base + rr, col = 64 * c + 8 * schunk;
          if (r < tl.rows && col < tl.cols)
            *reinterpret_cast<uint4*>(tl.out + int64_t(r) * tl.ld + col) = stage[rr * 8 + (schunk ^ (rr & 7))];
        }
        __syncwarp();
      }
      ++j;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 2D map over uint8 codes [rows, cols] with row stride ld bytes; box = box_cols x box_rows,
// 128-byte swizzle (box_cols = 128), zero fill outside the matrix.
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_grouped_gemm(const GemmArgs& a, cudaStream_t stream, const char** detail) {
  static int configured_device = -1;
  static int num_sms = 0;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (configured_device != dev) {
    err = cudaFuncSetAttribute(grouped_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (err != cudaSuccess) return err;
    err = cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess) return err;
    configured_device = dev;
  }
  CUtensorMap tmA, tmB;
  if (!make_map(&tmA, a.a, a.a_rows, a.a_cols, a.lda, BM) || !make_map(&tmB, a.b, a.b_rows, a.b_cols, a.ldb, BN)) {
    if (detail) *detail = "cuTensorMapEncodeTiled failed";
    return cudaErrorInvalidValue;
  }
  Params p;
  p.mode = a.mode;
  p.E = a.E;
  p.M = a.M; p.N = a.N; p.K = a.K;
  p.offs = a.offs;
  p.sfa = a.sfa; p.sfb = a.sfb;
  p.sfa_pitch = a.sfa_pitch; p.sfb_pitch = a.sfb_pitch;
  p.sfa_atoms = a.sfa_atoms; p.sfb_atoms = a.sfb_atoms;
  p.out = a.out;
  p.status = a.status;
  p.timeout_ns = a.timeout_ns;
  grouped_gemm_kernel<<<num_sms, NUM_THREADS, SMEM_BYTES, stream>>>(tmA, tmB, p);
  return cudaGetLastError();
}

}  // namespace mxf8
