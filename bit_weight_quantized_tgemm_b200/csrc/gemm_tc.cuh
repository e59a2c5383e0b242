// gemm_tc.cuh -- large-M path: persistent tcgen05 (5th-generation tensor core) kernel.
//
// Schedule: a tile's work is `ksteps` units (its 128-k stages, then the branch's stages),
// numbered tile-major.  The tiles are split in two regions:
//   whole-tile region, tiles [0, sk_t0): CTA c owns the units [c * dpc, (c + 1) * dpc),
//     a whole number of tiles;
//   split region, tiles [sk_t0, num_tiles): its units are cut into equal contiguous ranges
//     of `upc`, one per CTA, so a tile can be shared by consecutive CTAs ("stream-K"): each
//     writes its f32 partial sum to a slot in the workspace and the last to arrive adds the
//     slots in k order.
// A CTA works through its split-region range first, then its whole tiles, so the split
// tiles' partial sums and fix-ups overlap the whole tiles' MMAs and every CTA ends on a
// whole tile stored straight from the accumulator.  The host picks sk_t0 = 0 with upc a
// multiple of ksteps (whole tiles only), sk_t0 = 0 with dpc = 0 (all tiles shared, for
// fewer tiles than SMs), or sk_t0 = floor(tiles / SMs) * SMs (the remainder shared).
//
// Tile: 128 weight rows (MMA M, TMEM lanes) x 256 tokens (MMA N, accumulator columns),
// 128 k per stage (an M=128 MMA costs the same time for any N up to 256, so N is 256;
// a stage of eight K=16 MMAs keeps the single issuing thread's per-stage wait and commit
// small next to the tensor core's work).  The dequantized weights never touch shared memory: dequant warps write
// them straight into tensor memory (tcgen05.st) and the MMA reads its A operand from
// there (tcgen05.mma ... [a_tmem]).  Shared memory then carries only the activation
// tiles (TMA in, MMA out), which keeps its traffic at 128 bytes per MMA cycle.
//
// Tensor memory (512 columns x 128 lanes of 32 bits):
//   columns [0, 256)             the f32 accumulator
//   columns [256 + 64 s, +64)    A stage s (s < 3): 128 rows x 128 k of f16, element k of
//                                a row in column k/2 (low half for even k)
//   columns [448, 512)           the epilogue's stash: half of a finished tile's bf16
//                                output (32 columns per half of the accumulator)
// Stage s of the pipeline is the activation tile in shared memory plus A stage s; one
// mbarrier says it is full (TMA bytes + the eight dequant warps) and one says it is
// free (the MMA's commit), so the MMA thread waits once and commits once per stage.
// With one accumulator the MMA waits while a finished tile is read out; the epilogue
// releases it as soon as the tile is out of TMEM (into a shared-memory box, registers and
// the stash), before any store to y, and the stages keep filling meanwhile.
//
// Warp roles (19 warps, one CTA per SM):
//   warp 0      TMA producer: activation tile, 256 tokens x 128 k as two 64-k boxes (f16,
//               128-byte swizzle)
//   warp 1      TMEM allocator and MMA issuer (one thread): 8 x tcgen05.mma 128x256x16
//   warps 2-9   dequantizers: warp w handles TMEM lanes 32*(w%4).. (weight rows), warps
//               2-5 the first 64 k of a stage and warps 6-9 the second; codes come from
//               a shared-memory ring that warp 18 fills by TMA (one 128-row box per
//               stage), scales straight from global memory one item ahead; they are
//               unpacked and scaled in f16 and stored with one tcgen05.st of 32 columns
//   warps 10-17 epilogue: warp w reads TMEM lanes 32*(w%4).. and half of the columns
//               (tcgen05.ld) and stores y.  A whole tile's bf16 output is turned around
//               through a [32 tokens][128 rows] shared-memory box per column half, so
//               that each warp store writes 256 contiguous bytes of one token row;
//               otherwise lanes write consecutive rows n of one token row
//   warp 18     TMA producer: packed codes, one box of the tile's 128 rows per stage
//
// Operand precision: kind::f16 with both operands f16.  Q2_0 weights (q - 1) * d are
// exact in f16; 4-bit weights are computed as ((q - z) * s) in f16, exact up to the
// final rounding.  The activations arrive as an f16 copy (prep_x16_kernel) whose k order
// inside each 16-group (Q2) or 8-group (4-bit) is permuted to match the order in which a
// 32-bit word of packed codes unpacks with one shift and one mask per pair:
//   Q2:    pair i of a 16-code word = codes (i, i+8),  i < 8
//   4-bit: pair i of an 8-code word = codes (i, i+4),  i < 4
// Both operands use the same permutation, so the contraction is unchanged.
//
// The low-rank branch y += (x A^T) B^T ("mindview-t2i-turbo", section "One step") runs as
// extra pipeline stages after the main K loop: the weight-side stage holds [B | B], the
// token-side stage holds u = x A^T as a bf16 pair [hi | lo], and a bf16 MMA adds
// u_hi B^T + u_lo B^T into the same accumulator.
#pragma once

#include "common.cuh"

namespace tgemm {

#ifndef TGEMM_TC_STAGES
#define TGEMM_TC_STAGES 3
#endif
constexpr int kTcRows = 128;   // weight rows per tile (MMA M)
constexpr int kTcTok = 256;    // tokens per tile (MMA N)
constexpr int kTcBK = 128;     // k per stage
constexpr int kTcBox = 64;     // k per TMA box (one 128-byte swizzle row of f16)
// One ring of stages: stage s is an activation tile in shared memory plus an A tile in
// TMEM, filled by the TMA producer and the dequant warps and released together.
constexpr int kTcStages = TGEMM_TC_STAGES;
constexpr int kTcEpiWarps = 8;
#ifndef TGEMM_TC_DEQ_WARPS
#define TGEMM_TC_DEQ_WARPS 8
#endif
// Dequant warps: kTcDeqParts per TMEM lane quarter, each unpacking kTcDeqCodes codes of
// its row per stage.
constexpr int kTcDeqWarps = TGEMM_TC_DEQ_WARPS;
constexpr int kTcDeqParts = kTcDeqWarps / 4;
constexpr int kTcDeqCodes = 128 / kTcDeqParts;
static_assert(kTcDeqWarps == 8 || kTcDeqWarps == 16, "2 or 4 dequant warps per lane quarter");
constexpr int kTcEpiWarp0 = 2 + kTcDeqWarps;                // first epilogue warp
constexpr int kTcWProdWarp = kTcEpiWarp0 + kTcEpiWarps;     // the packed-weight TMA producer
constexpr int kTcThreads = (kTcWProdWarp + 1) * 32;
constexpr int kTcXBytes = kTcTok * kTcBK * 2;   // 64 KB: two 32 KB boxes
constexpr int kTcXBoxBytes = kTcTok * kTcBox * 2;
constexpr int kTcTmemCols = 512;
constexpr int kTcAccCols = kTcTok;              // f32 accumulator columns
constexpr int kTcACol0 = kTcAccCols;            // first A-stage column
constexpr int kTcACols = kTcBK / 2;             // columns per A stage (2 f16 per column)
// Past the A stages: where the epilogue parks half of a finished tile's bf16 output (32
// columns per column half of the accumulator) so that the accumulator is released sooner.
constexpr int kTcStashCol0 = kTcACol0 + kTcStages * kTcACols;
static_assert(kTcStashCol0 + 64 <= kTcTmemCols, "the epilogue's stash must fit in TMEM");
static_assert(kTcACol0 + kTcStages * kTcACols <= kTcTmemCols, "TMEM budget");

template <int FMT>
struct TcFmt {
  static constexpr int kWqRowBytes = FMT == 0 ? 32 : 64;  // packed bytes per row per stage
  // Packed weights reach the dequant warps through their own ring of shared-memory
  // stages (one TMA box of 128 rows per stage), filled this many stages ahead: deep
  // enough to hide a DRAM miss, small enough to fit beside the activation stages (and,
  // for Q2, the output boxes).
  static constexpr int kWStages = 4;
  static constexpr int kWBytes = kTcRows * kWqRowBytes;
  static constexpr int kXOff = 0;
  static constexpr int kWOff = kXOff + kTcStages * kTcXBytes;
  // Q2: two [32 tokens][128 rows] bf16 boxes, one per half of the accumulator's columns,
  // through which a whole tile's bf16 output is turned around for coalesced stores
  static constexpr int kYBoxBytes = 32 * kTcRows * 2;
  static constexpr int kYOff = kWOff + kWStages * kWBytes;
  static constexpr int kBarOff = kYOff + (FMT == 0 ? 2 * kYBoxBytes : 0);
  static constexpr int kNumBars = 2 * kTcStages + 3 + 2 * kWStages + 4;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemBytes = kMiscOff + 16 + 1024;  // + alignment slack
};

struct TcParams {
  int M, N, K;
  int tiles_m, num_tiles;
  int kt_main;     // main stages: ceil(K / 128), or kt1 + ceil(K2 / 128) for two inputs
  int kt1;         // stages of the first input; stages [kt1, kt_main) read the second
  int K2;          // the second input's width (0: one input)
  int kt_lora;     // extra stages for the low-rank branch (0 without it)
  int ksteps;      // kt_main + kt_lora: units of work per tile
  int upc;         // split region: CTA c owns units sk_t0 * ksteps + [c * upc, (c + 1) * upc)
  int units;       // U = num_tiles * ksteps
  int lora_mmas;   // K=16 MMAs in those stages: 2 * round_up(r, 16) / 16
  int R;           // round_up(r, 16): width of u_hi (and of u_lo) in the concatenation
  int r;
  int out_f32;
  const uint8_t* wq;       // packed codes [N][K/4] (Q2) or [N][K/2] (4-bit)
  const uint16_t* scales;  // Q2: d [N][K/128]; 4-bit: sz [N][K/64][2]
  const uint16_t* scales2; // the second input's scales (two inputs only)
  const uint16_t* lb;      // low-rank B (bf16): element (n, i) at lb[n * lb_sn + i * lb_si]
  void* y;
  float* part;             // split tiles: 2 slots of 128 x 256 f32 per CTA
  int* cnt;                // split region: 8 arrival counters per tile, zero at launch
  int sk_t0;               // first tile of the split region (tiles before it are whole per CTA)
  int dpc;                 // whole-tile region: CTA c owns units [c * dpc, (c + 1) * dpc) (0: none)
  int lb_sn, lb_si;        // B's element strides: (r, 1) for B [N][r], (1, N) for B^T [r][N]
  int y_box;               // whole tiles leave through the output boxes (Q2, bf16 y, N % 4 == 0)
};

// One tile's share of a CTA's unit range [u, u1): tile `tile`, stages [ka, kb).
struct TcSeg {
  int tile, ka, kb;
};
__device__ __forceinline__ TcSeg tc_seg_at(const TcParams& p, int u, int u1) {
  const int t = u / p.ksteps;
  const int end = min(u1, (t + 1) * p.ksteps);
  return TcSeg{t, u - t * p.ksteps, end - t * p.ksteps};
}
// A CTA's two unit ranges: [a0, a1) in the split region, then [b0, b1) of whole tiles
// (either may be empty).
struct TcRanges {
  int a0, a1, b0, b1;
};
__device__ __forceinline__ TcRanges tc_ranges(const TcParams& p, int c) {
  const int sk_u0 = p.sk_t0 * p.ksteps;
  TcRanges r;
  r.a0 = sk_u0 + c * p.upc;
  r.a1 = max(r.a0, min(p.units, r.a0 + p.upc));
  r.b0 = c * p.dpc;
  r.b1 = max(r.b0, min(sk_u0, r.b0 + p.dpc));
  return r;
}
// Slot of the partial sum that CTA c writes for its segment of split-region tile t: a
// segment that starts mid-tile (or at the tile's start) is the CTA's first, any other its
// last.
__device__ __forceinline__ int tc_slot(const TcParams& p, int c, int t) {
  return c * p.upc >= (t - p.sk_t0) * p.ksteps ? 2 * c : 2 * c + 1;
}
constexpr int kTcSlotFloats = kTcRows * kTcTok;
// The dequant warps prefetch a row's low-rank B values this many stages before the
// tile's branch stage.
constexpr int kLoraPrefetchStages = 4;

// A warp-uniform bounded wait: every lane gets the same answer, so the .sync.aligned
// tcgen05 instructions that follow never run with part of a warp.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity,
                                               volatile uint32_t* abort_flag) {
  return __all_sync(0xFFFFFFFFu, mbar_wait(bar, parity, abort_flag));
}

// Unpacking without per-pair shifts.  A field of b bits at mantissa bit position p of an
// f16 whose other mantissa bits are zero and whose exponent makes the field's lowest bit
// worth 1 reads as 2^(10-p) + q: so one lop3 (mask the field, or in the exponent) turns a
// code in place into an exact f16 integer offset by a known constant, as long as the field
// lies inside the 10-bit mantissa.  Both halves of a 32-bit word are done at once (f16x2).
//   2-bit fields at bits 0, 2, 4, 6, 8:  exponents of 1024, 256, 64, 16, 4
//   4-bit fields at bits 0, 4:           exponents of 1024, 64
// Fields at bits 10 and up are moved down by one shift first.
// Q2: 16 codes -> 8 f16x2 pairs (codes i, i+8) of (q - 1) * d.
__device__ __forceinline__ void q2_word_to_f16(uint32_t w, uint32_t d2, uint32_t* o) {
  // per field position j: the magic (2^(10-2j) as f16x2) and 2^(10-2j) + 1
  constexpr uint32_t kMagic[5] = {0x64006400u, 0x5C005C00u, 0x54005400u, 0x4C004C00u, 0x44004400u};
  constexpr uint32_t kBase1[5] = {0x64016401u, 0x5C045C04u, 0x54105410u, 0x4C404C40u, 0x45004500u};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int j = i < 5 ? i : i - 5;
    const uint32_t src = i < 5 ? w : (w >> 10);
    const uint32_t t = lop3_and_or(src, 0x00030003u << (2 * j), kMagic[j]);  // base + q
    o[i] = hmul2_u32(hsub2_u32(t, kBase1[j]), d2);                              // (q-1)*d
  }
}

// 4-bit: 8 codes -> 4 f16x2 pairs (codes i, i+4) of (q - z) * s.
__device__ __forceinline__ void q4_word_to_f16(uint32_t w, uint32_t s2, uint32_t z2,
                                               uint32_t* o) {
  constexpr uint32_t kMagic[2] = {0x64006400u, 0x54005400u};  // 1024, 64
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int j = i & 1;
    const uint32_t src = i < 2 ? w : (w >> 8);
    const uint32_t t = lop3_and_or(src, 0x000F000Fu << (4 * j), kMagic[j]);  // base + q
    o[i] = hmul2_u32(hsub2_u32(hsub2_u32(t, kMagic[j]), z2), s2);             // (q-z)*s
  }
}

// DUAL: stages [kt1, kt_main) read a second input (tm_x2, tm_w2, scales2, K2).
// HYB: the schedule has a whole-tile region as well as the split region (p.dpc > 0); without
// it every CTA runs one unit range and the loops compile to that alone.
template <int FMT, bool LORA, bool DUAL, bool HYB>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tm_x,
                   const __grid_constant__ CUtensorMap tm_u,
                   const __grid_constant__ CUtensorMap tm_w,
                   const __grid_constant__ CUtensorMap tm_x2,
                   const __grid_constant__ CUtensorMap tm_w2, const TcParams p) {
  using F = TcFmt<FMT>;
  static_assert(F::kSmemBytes <= 232448, "shared memory budget");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + F::kBarOff;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kTcStages + s); };
  const uint32_t accfull_bar = bar0 + 8u * (2 * kTcStages);
  const uint32_t accempty_bar = bar0 + 8u * (2 * kTcStages + 1);
  const uint32_t drain_bar = bar0 + 8u * (2 * kTcStages + 2);
  auto wfull_bar = [&](int w) { return bar0 + 8u * (2 * kTcStages + 3 + w); };
  auto wempty_bar = [&](int w) { return bar0 + 8u * (2 * kTcStages + 3 + F::kWStages + w); };
  // output boxes (Q2, bf16): filled / read out by the 4 warps of a column half
  auto yfull_bar = [&](int h) { return bar0 + 8u * (2 * kTcStages + 3 + 2 * F::kWStages + h); };
  auto yfree_bar = [&](int h) { return bar0 + 8u * (2 * kTcStages + 5 + 2 * F::kWStages + h); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + F::kMiscOff);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + F::kMiscOff + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(full_bar(s), 1 + kTcDeqWarps);  // producer's expect_tx + dequant warps
      mbar_init(empty_bar(s), 1);      // MMA commit
    }
    mbar_init(accfull_bar, 1);             // MMA commit
    mbar_init(accempty_bar, kTcEpiWarps);  // epilogue warps
    mbar_init(drain_bar, 1);
    for (int w = 0; w < F::kWStages; ++w) {
      mbar_init(wfull_bar(w), 1);   // weight producer's expect_tx
      mbar_init(wempty_bar(w), kTcDeqWarps);  // every dequant warp has read its codes
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(yfull_bar(h), 4);  // the column half's 4 epilogue warps have filled the box
      mbar_init(yfree_bar(h), 4);  // ... and have read it out
    }
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_x);
    if (LORA) tma_prefetch_desc(&tm_u);
    if (DUAL) tma_prefetch_desc(&tm_x2);
  }
  if (warp == kTcWProdWarp && lane == 0) {
    tma_prefetch_desc(&tm_w);
    if (DUAL) tma_prefetch_desc(&tm_w2);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTcTmemCols);
    tmem_relinquish();
  }
  __syncwarp();  // reconverge after the single-thread set-up above
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Let the next kernel be scheduled.  Only the warps that touch memory the kernels ahead
  // may write wait for them: the activation producer (x, or the branch's u, come from the
  // preparation kernel) and the epilogue (y; the split-tile counters that kernel zeroes).
  // The packed-weight producer, the dequantizers (codes, scales, the branch's B) and the
  // MMA issuer (shared and tensor memory only) start at once: the packed weights are not
  // written by the kernels ahead, so the first stages fill while those finish.
  pdl_trigger();
  if (warp == 0 || (warp >= kTcEpiWarp0 && warp < kTcWProdWarp)) pdl_wait();
  const uint32_t tmem_base = *tmem_slot;
  const int ksteps = p.ksteps;
  const int kt1 = DUAL ? p.kt1 : p.kt_main;  // stages of the first input
  const TcRanges rg = tc_ranges(p, static_cast<int>(blockIdx.x));  // this CTA's units

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int r = 0; ok && r < (HYB ? 2 : 1); ++r)
      for (int u = r ? rg.b0 : rg.a0, ue = r ? rg.b1 : rg.a1; u < ue; ++u, ++it) {
        const int tile = u / ksteps, ks = u - tile * ksteps;
        const int tm = tile % p.tiles_m;
        const uint32_t s = it % kTcStages, ph = (it / kTcStages) & 1u;
        if (!mbar_wait(empty_bar(s), ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t xdst = sbase + F::kXOff + s * kTcXBytes;
        mbar_arrive_expect_tx(full_bar(s), kTcXBytes);
        // stage ks: first input, second input, or the branch's u
        const CUtensorMap* map = ks < kt1 ? &tm_x : (ks < p.kt_main ? &tm_x2 : &tm_u);
        const int k0 = (ks < kt1 ? ks : (ks < p.kt_main ? ks - kt1 : ks - p.kt_main)) * kTcBK;
        tma_load_2d(xdst, map, full_bar(s), k0, tm * kTcTok);
        tma_load_2d(xdst + kTcXBoxBytes, map, full_bar(s), k0 + kTcBox, tm * kTcTok);
      }
      // every load issued must land before the CTA may exit
      const uint32_t n_issued = it;
      for (uint32_t j = (n_issued > kTcStages ? n_issued - kTcStages : 0); j < n_issued; ++j)
        mbar_wait_drain(full_bar(j % kTcStages), (j / kTcStages) & 1u);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescMain = make_idesc_f16(0u, kTcRows, kTcTok);  // f16 x f16
      constexpr uint32_t kIdescLora = make_idesc_f16(1u, kTcRows, kTcTok);  // bf16 x bf16
      uint32_t it = 0, scount = 0;
      bool ok = true;
      for (int r = 0; ok && r < (HYB ? 2 : 1); ++r)
      for (int u = r ? rg.b0 : rg.a0, ue = r ? rg.b1 : rg.a1; ok && u < ue; ++scount) {
        const TcSeg sg = tc_seg_at(p, u, ue);
        u += sg.kb - sg.ka;
        if (!mbar_wait(accempty_bar, (scount & 1u) ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base;
        for (int ks = sg.ka; ks < sg.kb; ++ks, ++it) {
          const uint32_t s = it % kTcStages, ph = (it / kTcStages) & 1u;
          if (!mbar_wait(full_bar(s), ph, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_tmem = tmem_base + kTcACol0 + s * kTcACols;              // weights
          const uint32_t xs = sbase + F::kXOff + s * kTcXBytes;                      // tokens
          // K=16 step kk reads columns 8kk.. of the A stage and 32-byte offset (kk % 4) in
          // the (kk / 4)-th 64-k box of the activation tile
          auto bdesc = [&](int kk) {
            return smem_desc_sw128(xs + (kk >> 2) * kTcXBoxBytes) + 2u * (kk & 3);
          };
          if (!LORA || ks < p.kt_main) {
#pragma unroll
            for (int kk = 0; kk < kTcBK / 16; ++kk)
              mma_f16_ts(d_tmem, a_tmem + 8u * kk, bdesc(kk), kIdescMain,
                         (ks > sg.ka || kk > 0) ? 1u : 0u);
          } else {
            const int done = (ks - p.kt_main) * (kTcBK / 16);
            for (int kk = 0; kk < kTcBK / 16 && done + kk < p.lora_mmas; ++kk)
              mma_f16_ts(d_tmem, a_tmem + 8u * kk, bdesc(kk), kIdescLora,
                         (ks > sg.ka || kk > 0) ? 1u : 0u);
          }
          mma_commit(empty_bar(s));
        }
        if (!ok) break;
        mma_commit(accfull_bar);
      }
      // all MMAs this thread issued must finish before TMEM is released
      mma_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0u);
    }
  } else if (warp < kTcEpiWarp0) {
    // ------------------------------------------------------------ dequantizers
    constexpr int kC = kTcDeqCodes;                       // codes per thread per stage
    constexpr int kWords = FMT == 0 ? kC / 16 : kC / 8;   // 32-bit words of packed codes
    const int q = warp & 3;                // TMEM lane quarter this warp may access
    const int rt = 32 * q + lane;          // weight row within the tile
    const int part = (warp - 2) >> 2;      // which kC codes of the stage's 128
    const int nscale = FMT == 0 ? p.K / 128 : p.K / 64;
    const int nscale2 = FMT == 0 ? p.K2 / 128 : p.K2 / 64;
    const uint32_t a_lane = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + kTcACol0 +
                            static_cast<uint32_t>(part * (kC / 2));
    // this thread's codes inside a weight stage (row rt, part `part`)
    const uint32_t w_mine =
        sbase + F::kWOff + rt * F::kWqRowBytes + part * (F::kWqRowBytes / kTcDeqParts);
    uint32_t wit = 0;   // A stages written
    uint32_t wcnt = 0;  // weight stages consumed
    bool ok = true;
    // This CTA's work is one stream of (tile, stage) items: its split-region units, then
    // its whole tiles.  The position is advanced item by item with one compare against
    // the end of the current tile's segment (its last stage, or the first range's end);
    // only there is the next tile (or the jump to the whole tiles) worked out.
    const int n_first = rg.a1 - rg.a0;
    const int n_items = HYB ? n_first + (rg.b1 - rg.b0) : n_first;
    bool in_first = !HYB || n_first > 0;
    const int u_start = in_first ? rg.a0 : rg.b0;
    int tile = u_start / ksteps, ks = u_start - tile * ksteps;
    int seg_end = HYB && in_first ? min(ksteps, rg.a1 - tile * ksteps) : ksteps;
    int row = (tile / p.tiles_m) * kTcRows + rt;
    // The scale of the item at (ks, row): Q2 block scale d, or the 4-bit group's (s, z)
    // pair (0 where the item has none: a branch stage, a row past N, codes past K).
    auto scale_at = [&](int ks_, int row_, bool in) -> uint32_t {
      if (!in || row_ >= p.N || ks_ >= p.kt_main) return 0u;
      const bool second = DUAL && ks_ >= kt1;  // the second input's stages
      if (second) ks_ -= kt1;
      const int k_first = ks_ * kTcBK + part * kC;
      if (k_first >= (second ? p.K2 : p.K)) return 0u;
      const uint16_t* srow = (second ? p.scales2 : p.scales) +
                             static_cast<int64_t>(row_) * (second ? nscale2 : nscale) * (FMT == 0 ? 1 : 2);
      return FMT == 0 ? static_cast<uint32_t>(__ldg(srow + ks_))
                      : __ldg(reinterpret_cast<const uint32_t*>(srow) + k_first / 64);
    };
    uint32_t sc_next = scale_at(ks, row, n_items > 0);  // loaded one item ahead
    for (int i = 0; ok && i < n_items; ++i) {
      const uint32_t sc = sc_next;
      const bool valid = row < p.N;
      int nks = ks + 1, ntile = tile, nrow = row;
      if (nks == seg_end) {
        nks = 0;
        if (HYB && in_first && ntile * ksteps + seg_end == rg.a1) {
          in_first = false;  // on to the whole tiles, which start on a tile boundary
          ntile = rg.b0 / ksteps;
        } else {
          ++ntile;
        }
        if (HYB) seg_end = in_first ? min(ksteps, rg.a1 - ntile * ksteps) : ksteps;
        nrow = (ntile / p.tiles_m) * kTcRows + rt;
      }
      sc_next = scale_at(nks, nrow, i + 1 < n_items);
      if (LORA && valid && ks == (p.kt_main > kLoraPrefetchStages ? p.kt_main - kLoraPrefetchStages : 0)) {
        // the row's B values for this tile's branch stage -> L1, a few stages ahead
        if (p.lb_si == 1) {
          const uint16_t* br = p.lb + static_cast<int64_t>(row) * p.lb_sn;
          prefetch_l1(br);
          if (((reinterpret_cast<uintptr_t>(br) & 127) + 2 * p.r) > 128) prefetch_l1(br + 64);
        } else {
          for (int ii = part; ii < p.r; ii += kTcDeqParts)
            prefetch_l1(p.lb + static_cast<int64_t>(ii) * p.lb_si + static_cast<int64_t>(row) * p.lb_sn);
        }
      }
      uint32_t o[kC / 2];
      if (!LORA || ks < p.kt_main) {
        // codes from the weight ring (rows past N and k past K arrive zero-filled)
        const uint32_t w = wcnt % F::kWStages, wph = (wcnt / F::kWStages) & 1u;
        if (!mbar_wait_warp(wfull_bar(w), wph, abort_flag)) {
          ok = false;
          break;
        }
        uint32_t cw[kWords];
        const uint32_t src = w_mine + w * F::kWBytes;
        if (kWords == 2) {
          const uint2 v = ld_shared_v2(src);
          cw[0] = v.x;
          cw[1] = v.y;
        } else {
#pragma unroll
          for (int j = 0; j < kWords; j += 4) {
            const uint4 v = ld_shared_v4(src + 4 * j);
            cw[j] = v.x;
            cw[j + 1] = v.y;
            cw[j + 2] = v.z;
            cw[j + 3] = v.w;
          }
        }
        // the ring slot is refilled by TMA (the async proxy) once every dequant warp has
        // released it: order these generic-proxy reads before that write
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(wempty_bar(w));
        ++wcnt;
        if (FMT == 0) {
          const uint32_t d2 = sc | (sc << 16);
#pragma unroll
          for (int j = 0; j < kWords; ++j) q2_word_to_f16(cw[j], d2, o + 8 * j);
        } else {
          const uint32_t s2 = (sc & 0xFFFFu) | (sc << 16);
          const uint32_t z2 = (sc >> 16) | (sc & 0xFFFF0000u);
#pragma unroll
          for (int j = 0; j < kWords; ++j) q4_word_to_f16(cw[j], s2, z2, o + 4 * j);
        }
      } else {
        // low-rank stage: weight-side values [j0, j0 + kC) of [B | B], zero beyond 2R and
        // in each copy's padding (columns r..R-1); a chunk of 8 columns is either all
        // padding (skipped, warp-uniform), a 16-byte load, or up to 8 element loads
        const int j0 = (ks - p.kt_main) * kTcBK + part * kC;
#pragma unroll
        for (int q = 0; q < kC / 2; ++q) o[q] = 0u;
        if (j0 < 2 * p.R) {
          const uint16_t* br = p.lb + static_cast<int64_t>(valid ? row : 0) * p.lb_sn;
          const bool vec = p.lb_si == 1 && (p.lb_sn & 7) == 0 &&
                           (reinterpret_cast<uintptr_t>(p.lb) & 15) == 0;
#pragma unroll
          for (int cq = 0; cq < kC / 8; ++cq) {
            const int jc = j0 + 8 * cq;
            if (jc >= 2 * p.R) break;
            const int ic = jc < p.R ? jc : jc - p.R;
            if (ic >= p.r || !valid) continue;
            if (vec && ic + 8 <= p.r) {
              const uint4 v = *reinterpret_cast<const uint4*>(br + ic);
              o[4 * cq] = v.x;
              o[4 * cq + 1] = v.y;
              o[4 * cq + 2] = v.z;
              o[4 * cq + 3] = v.w;
            } else {
#pragma unroll
              for (int e = 0; e < 8; ++e)
                if (ic + e < p.r)
                  o[4 * cq + e / 2] |= static_cast<uint32_t>(br[static_cast<int64_t>(ic + e) * p.lb_si])
                                       << (16 * (e & 1));
            }
          }
        }
      }
      tile = ntile;
      ks = nks;
      row = nrow;
      const uint32_t ws = wit % kTcStages, wph = (wit / kTcStages) & 1u;
      if (!mbar_wait_warp(empty_bar(ws), wph ^ 1u, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (kC == 64)
        tmem_st_32x32b_x32(a_lane + ws * kTcACols, *reinterpret_cast<uint32_t(*)[32]>(o));
      else
        tmem_st_32x32b_x16(a_lane + ws * kTcACols, *reinterpret_cast<uint32_t(*)[16]>(o));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(full_bar(ws));
      ++wit;
    }
  } else if (warp < kTcWProdWarp) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                // TMEM lane quarter this warp may access
    const int eh = (warp - kTcEpiWarp0) >> 2;  // which half of the accumulator's columns
    const int piece = warp - kTcEpiWarp0;      // this warp's 32 x 128 piece of the tile
    constexpr int kChunks = kTcTok / 32 / 2;
    constexpr int kPieceFloats = kTcSlotFloats / kTcEpiWarps;
    uint32_t scount = 0;
    uint32_t ycount = 0;  // output boxes this warp has filled
    bool ok = true;
    for (int r = 0; ok && r < (HYB ? 2 : 1); ++r)
    for (int u = r ? rg.b0 : rg.a0, ue = r ? rg.b1 : rg.a1; u < ue; ++scount) {
      const TcSeg sg = tc_seg_at(p, u, ue);
      u += sg.kb - sg.ka;
      const int tm = sg.tile % p.tiles_m, tn = sg.tile / p.tiles_m;
      if (!mbar_wait_warp(accfull_bar, scount & 1u, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int n = tn * kTcRows + q * 32 + lane;  // this thread's weight row
      const bool nv = n < p.N;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + eh * (kTcTok / 2);
      const int mbase = tm * kTcTok + eh * (kTcTok / 2);
      // y[m0 + e][n] for e < 32 (lanes write consecutive n: coalesced)
      auto put = [&](int m0, const uint32_t (&v)[32]) {
        if (!nv || m0 >= p.M) return;
        if (p.out_f32) {
          float* dst = reinterpret_cast<float*>(p.y) + static_cast<int64_t>(m0) * p.N + n;
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (m0 + e < p.M) dst[static_cast<int64_t>(e) * p.N] = __uint_as_float(v[e]);
        } else {
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.y) + static_cast<int64_t>(m0) * p.N + n;
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (m0 + e < p.M) dst[static_cast<int64_t>(e) * p.N] = __float2bfloat16_rn(__uint_as_float(v[e]));
        }
      };
      if (FMT == 0 && p.y_box && sg.ka == 0 && sg.kb == ksteps) {
        // The whole tile, bf16.  A thread holds one weight row, so its stores of y (one
        // token row per store) would land 2 bytes apart from its neighbours'; instead, each
        // 32-token chunk of this half of the accumulator is turned around in a
        // [32 tokens][128 rows] box in shared memory, and each of the half's 4 warps then
        // writes 8 token rows of 256 contiguous bytes (8 bytes a lane).  The accumulator is
        // released before any of that: chunk 0 goes into the box, chunk 1 is kept in
        // registers and chunks 2-3 in the TMEM stash, as packed bf16 pairs.  The 4 warps
        // meet twice per chunk: box filled (yfull), box read out (yfree); both waits are
        // bounded.
        uint16_t* ybox = reinterpret_cast<uint16_t*>(smem + F::kYOff + eh * F::kYBoxBytes);
        uint16_t* ymine = ybox + q * 32 + lane;  // this thread's row in the box
        const uint32_t tstash = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + kTcStashCol0 + eh * 32;
        const int n4 = tn * kTcRows + 4 * lane;  // this lane's 4 rows in the copy-out
        // chunk 0 goes into the box at once (its previous read-out ended with the last
        // tile), chunk 1 stays in registers as packed bf16 pairs, chunks 2-3 are parked in
        // the stash; then the accumulator is released
        if (!mbar_wait_warp(yfree_bar(eh), (ycount & 1u) ^ 1u, abort_flag)) {
          ok = false;
          continue;
        }
        uint32_t pk1[16];  // pk1[i]: tokens 32 + 2i (low half), 33 + 2i of this row
#pragma unroll
        for (int cc = 0; cc < kChunks; ++cc)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t v[16];
            tmem_ld_32x32b_x16(tbase + cc * 32 + hh * 16, v);
            tmem_wait_ld();
            if (cc == 0) {
#pragma unroll
              for (int e = 0; e < 16; ++e)
                ymine[(16 * hh + e) * kTcRows] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[e])));
              continue;
            }
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) w[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
            if (cc == 1) {
#pragma unroll
              for (int i = 0; i < 8; ++i) pk1[8 * hh + i] = w[i];
            } else {
              tmem_st_32x32b_x8(tstash + (cc - 2) * 16 + hh * 8, w);
            }
          }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(accempty_bar);
#pragma unroll 1
        for (int cc = 0; cc < kChunks; ++cc) {
          const uint32_t yph = (ycount + cc) & 1u;
          if (cc > 0) {
            if (!mbar_wait_warp(yfree_bar(eh), yph ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
            uint32_t w[16];
            if (cc == 1) {
#pragma unroll
              for (int i = 0; i < 16; ++i) w[i] = pk1[i];
            } else {
              tmem_ld_32x32b_x16(tstash + (cc - 2) * 16, w);
              tmem_wait_ld();
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              ymine[(2 * i) * kTcRows] = static_cast<uint16_t>(w[i] & 0xFFFFu);
              ymine[(2 * i + 1) * kTcRows] = static_cast<uint16_t>(w[i] >> 16);
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(yfull_bar(eh));
          if (!mbar_wait_warp(yfull_bar(eh), yph, abort_flag)) {
            ok = false;
            break;
          }
          {
            // this warp's 8 token rows of the chunk
            const int m0 = mbase + cc * 32 + 8 * q;
            const int rows = n4 < p.N ? min(8, p.M - m0) : 0;
            const uint2* src = reinterpret_cast<const uint2*>(ybox + 8 * q * kTcRows + 4 * lane);
            uint2* dst = reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(p.y) +
                                                  static_cast<int64_t>(m0) * p.N + n4);
#pragma unroll
            for (int e8 = 0; e8 < 8; ++e8)
              if (e8 < rows) dst[static_cast<int64_t>(e8) * (p.N / 4)] = src[e8 * (kTcRows / 4)];
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(yfree_bar(eh));
        }
        ycount += kChunks;
        continue;
      }
      if (sg.ka == 0 && sg.kb == ksteps) {
        // the whole tile: accumulator -> y
#pragma unroll 1
        for (int cc = 0; cc < kChunks; ++cc) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tbase + cc * 32, v);
          tmem_wait_ld();
          if (cc == kChunks - 1) {
            // the accumulator is read out: let the next segment's MMAs start
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(accempty_bar);
          }
          put(mbase + cc * 32, v);
        }
        continue;
      }
      // Part of a tile shared with other CTAs.
      const int t_rel = sg.tile - p.sk_t0;  // the tile's place in the split region
      // Write this piece's f32 partial sum to the CTA's slot; the warp that completes the
      // piece's arrival count adds all slots of the tile in k order (deterministic) and
      // stores y.
      float* mine = p.part + static_cast<int64_t>(tc_slot(p, blockIdx.x, sg.tile)) * kTcSlotFloats +
                    piece * kPieceFloats;
#pragma unroll 1
      for (int cc = 0; cc < kChunks; ++cc) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tbase + cc * 32, v);
        tmem_wait_ld();
        if (cc == kChunks - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(accempty_bar);
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) __stcg(mine + (cc * 32 + e) * 32 + lane, __uint_as_float(v[e]));
      }
      __threadfence();
      __syncwarp();
      int before = 0;
      if (lane == 0) before = atomicAdd(p.cnt + t_rel * kTcEpiWarps + piece, 1);
      before = __shfl_sync(0xFFFFFFFFu, before, 0);
      const int c_lo = t_rel * ksteps / p.upc;
      const int c_hi = ((t_rel + 1) * ksteps - 1) / p.upc;
      if (before != c_hi - c_lo) continue;  // another CTA's warp finishes this piece
      __threadfence();
#pragma unroll 1
      for (int cc = 0; cc < kChunks; ++cc) {
        float acc[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) acc[e] = 0.f;
#pragma unroll 1
        for (int c = c_lo; c <= c_hi; ++c) {
          const float* src = p.part + static_cast<int64_t>(tc_slot(p, c, sg.tile)) * kTcSlotFloats +
                             piece * kPieceFloats + cc * 32 * 32 + lane;
#pragma unroll
          for (int e = 0; e < 32; ++e) acc[e] += __ldcg(src + e * 32);
        }
        uint32_t v[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(acc[e]);
        put(mbase + cc * 32, v);
      }
    }
  } else {
    // ------------------------------------------------------------ packed-weight producer
    // One TMA box per main stage: the tile's 128 rows x the stage's packed bytes, into
    // the weight ring, as far ahead of the dequant warps as the ring allows.
    if (lane == 0) {
      uint32_t wit = 0;
      bool ok = true;
      for (int r = 0; ok && r < (HYB ? 2 : 1); ++r)
      for (int u = r ? rg.b0 : rg.a0, ue = r ? rg.b1 : rg.a1; u < ue; ++u) {
        const int tile = u / ksteps, ks = u - tile * ksteps;
        if (ks >= p.kt_main) continue;  // branch stages carry no codes
        const uint32_t w = wit % F::kWStages, ph = (wit / F::kWStages) & 1u;
        if (!mbar_wait(wempty_bar(w), ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(wfull_bar(w), F::kWBytes);
        const bool second = DUAL && ks >= kt1;
        tma_load_2d(sbase + F::kWOff + w * F::kWBytes, second ? &tm_w2 : &tm_w, wfull_bar(w),
                    (second ? ks - kt1 : ks) * F::kWqRowBytes, (tile / p.tiles_m) * kTcRows);
        ++wit;
      }
      // every load issued must land before the CTA may exit
      for (uint32_t j = (wit > F::kWStages ? wit - F::kWStages : 0); j < wit; ++j)
        mbar_wait_drain(wfull_bar(j % F::kWStages), (j / F::kWStages) & 1u);
    }
  }

  // ------------------------------------------------------------ teardown
  // Warps 0, 1 and the weight producer run their roles on lane 0 alone; the other lanes
  // wait here for it, so that every warp reaches the CTA barrier converged (an aligned
  // barrier must not be executed by part of a warp) and TMEM is released only after the
  // last MMA has drained.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTcTmemCols);
  }
}

}  // namespace tgemm
