// gemv_stream.cuh -- small-M path (1..16 tokens), streaming form: one persistent CTA per SM
// that streams its share of the packed weights from HBM through a ring of shared-memory
// slots while its warps run the products.
//
// Work split.  The rows of W are cut into contiguous ranges (multiples of 8 rows), one per
// CTA (one or, up to 8 tokens, two CTAs per SM), and each range into tiles of 32 rows (two m16 halves of mma.sync m16n8k16).  K is
// cut into units of 128 weights and, when the activations of all of K do not fit in
// shared memory, into passes of `kp` weights.  For each (pass, tile) item every compute
// warp takes the units u = w, w + 8, ... of the pass, so one warp's products form 2T
// independent accumulator chains (two row halves x T token tiles of 8) that share each B
// fragment; the 8 warps' partial sums are added through shared memory (in warp order, so
// the result does not depend on timing; two buffers, so one barrier per item) and, after
// the last pass, stored.
//
// Data movement.
//   * Weights: one producer thread loads each item's packed codes -- 32 rows x the pass's
//     bytes -- into a ring slot with 2-D TMA boxes of 32 rows x 128 bytes (128-byte swizzle,
//     so the warps' word reads hit distinct banks), completing on the slot's mbarrier.
//     The first slots are issued before the kernel waits for the kernels ahead of it on
//     the stream (griddepcontrol.wait): the packed weights are not an output of those
//     kernels, so their fetch overlaps the end of the previous kernel.
//   * Scales: every scale of the CTA's rows (all of K) is staged in shared memory before
//     the wait, with several loads in flight per thread.
//   * Activations (the kernels ahead may have written them): after the wait, the compute
//     warps copy each pass's x into shared memory with its k order permuted (below), two
//     (Q2) or four (4-bit) threads per (token, unit), and meanwhile form the per-(unit,
//     token) correction sums, added across those threads by warp shuffles.
//
// The unpack.  Inside a 32-bit word of packed codes, a bf16 whose exponent makes a field's
// lowest bit worth 1 reads as base + q, so one lop3 (mask the field, or in the exponent)
// turns a pair of codes 16 bits apart into an exact bf16 pair (base + q_lo, base + q_hi):
//   Q2_0 word (16 codes, code i at bits 2i): pairs (i, i+8), i < 8.  Fields at bits 0, 2,
//        4 use the exponents of 128, 32, 8; the word shifted by 6 and by 12 gives the rest:
//        bases 128, 32, 8, 128, 32, 8, 128, 32 for i = 0..7.
//   4-bit word (8 codes, code i at bits 4i): pairs (i, i+4), i < 4, from the word shifted
//        by 4i, base 128.
// The offsets are removed after the products, per unit (Q2) or group (4-bit):
//   Q2:    y += d * (sum_k (base_k + q_k) x_k - sum_k (base_k + 1) x_k)
//   4-bit: y += s * (sum_k (128 + q_k) x_k - (128 + z) sum_k x_k)
// which is sum_k (q - 1) d x and sum_k (q - z) s x up to f32 rounding (the products of the
// bf16 operands are exact in the f32 accumulators).
//
// k order.  In k16 step s of a unit, lane (g, c) of the MMA supplies the A slots
// {2c, 2c+1 | 2c+8, 2c+9} of weight rows g and g+8 (of each half); they are two code pairs
// of one word of that lane: Q2 word c + 4 (s / 4), pairs 2 (s % 4) and 2 (s % 4) + 1;
// 4-bit word c + 4 (s / 2), pairs 2 (s % 2) and 2 (s % 2) + 1.  The staged activations
// put the matching x values at those slots, so the B fragments come from ldmatrix (8
// consecutive staged values per token row).  The mapping is the same for A and B, so the
// contraction is unchanged; gs_stage_k() states it.
#pragma once

#include "common.cuh"

namespace tgemm {

constexpr int kGsWarps = 8;                      // compute warps
constexpr int kGsThreads = (kGsWarps + 1) * 32;  // + the weight producer warp
constexpr int kGsRows = 32;                      // weight rows per tile: two m16 halves
constexpr int kGsUnit = 128;                     // k per unit
constexpr int kGsMaxUW = 4;                      // units per warp per pass (kp <= 4096)
constexpr int kGsBoxBytes = kGsRows * 128;       // one TMA box: 32 rows x 128 bytes

template <int FMT>
struct GsFmt {
  static constexpr int kUnitBytes = FMT == 0 ? 32 : 64;  // packed bytes of one row-unit
  static constexpr int kWordsPerUnit = kUnitBytes / 4;
  static constexpr int kScl = FMT == 0 ? 1 : 2;          // scale entries per row-unit
  static constexpr int kCorr = FMT == 0 ? 1 : 2;         // correction sums per (unit, token)
};

// Staged position 16 s + j of a unit (s = k16 step, j = slot) holds the activation of
// unit-relative k = gs_stage_k(s, j).  Slots 2c + e (e = 0, 1) and 8 + 2c + e of lane
// column c hold the low/high halves of the lane's two code pairs for the step.
template <int FMT>
__host__ __device__ constexpr int gs_stage_k(int s, int j) {
  const int c = (j & 7) >> 1, e = j & 1, hi = j >> 3;
  if (FMT == 0) {
    const int w = c + 4 * (s >> 2), sp = s & 3;  // word of the lane, pair 2 sp + hi
    return 16 * w + 2 * sp + hi + 8 * e;          // pair i = (code i, code i + 8)
  } else {
    const int w = c + 4 * (s >> 1), h = s & 1;   // word of the lane, pair 2 h + hi
    return 8 * w + 2 * h + hi + 4 * e;            // pair i = (code i, code i + 4)
  }
}

// Q2 base of code i of a word (its pair i % 8): 128, 32, 8, 128, 32, 8, 128, 32.
__host__ __device__ constexpr int gs_q2_base(int i) {
  return (i & 7) % 3 == 0 ? 128 : ((i & 7) % 3 == 1 ? 32 : 8);
}

struct GsParams {
  const uint16_t* x;
  const uint8_t* wq;
  const uint16_t* scales;  // Q2: d [N][K/128]; 4-bit: sz [N][K/64][2]
  void* y;
  int M, N, K, out_f32;
  int U;           // units along K: ceil(K / 128)
  int kp;          // weights per pass (a multiple of 128, at most 4096)
  int passes;      // ceil(K / kp)
  int grid;        // CTAs
  int j_max;       // most tiles of any CTA's row range
  int S;           // ring slots
  int nbox;        // TMA boxes per item: ceil(kp * bits / 8 / 128)
  int xs_stride;   // bytes per token row of the staged activations (kp * 2 + 16)
  int off_x, off_corr, off_red, off_acc, off_sc, off_ring, off_bar;  // shared-memory layout
};

// Shared address of 32-bit word `w` (bytes 4w..4w+3 of the row's pass bytes) of row r in a
// ring slot whose boxes are stored with the 128-byte swizzle (16-byte chunk index XOR
// row % 8).
__device__ __forceinline__ uint32_t gs_code_addr(uint32_t slot, int r, int w) {
  const int b = w >> 5, o = (w & 31) * 4;
  return slot + b * kGsBoxBytes + r * 128 + ((((o >> 4) ^ (r & 7)) << 4) | (o & 15));
}

__device__ __forceinline__ void ldmatrix_x2(uint32_t saddr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(saddr));
}

__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t saddr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(saddr) : "memory");
  return v;
}

// Q2: the 8 code pairs (i, i+8) of a word as bf16 pairs (base_i + q_i, base_i + q_{i+8}).
__device__ __forceinline__ void gs_q2_pairs(uint32_t w, uint32_t (&p)[8]) {
  const uint32_t w6 = w >> 6, w12 = w >> 12;
  p[0] = lop3_and_or(w, 0x00030003u, 0x43004300u);    // 128
  p[1] = lop3_and_or(w, 0x000C000Cu, 0x42004200u);    // 32
  p[2] = lop3_and_or(w, 0x00300030u, 0x41004100u);    // 8
  p[3] = lop3_and_or(w6, 0x00030003u, 0x43004300u);   // 128
  p[4] = lop3_and_or(w6, 0x000C000Cu, 0x42004200u);   // 32
  p[5] = lop3_and_or(w6, 0x00300030u, 0x41004100u);   // 8
  p[6] = lop3_and_or(w12, 0x00030003u, 0x43004300u);  // 128
  p[7] = lop3_and_or(w12, 0x000C000Cu, 0x42004200u);  // 32
}

// 4-bit: the 4 code pairs (i, i+4) of a word as bf16 pairs (128 + q_i, 128 + q_{i+4}).
__device__ __forceinline__ void gs_q4_pairs(uint32_t w, uint32_t (&p)[4]) {
  p[0] = lop3_and_or(w, 0x000F000Fu, 0x43004300u);
  p[1] = lop3_and_or(w >> 4, 0x000F000Fu, 0x43004300u);
  p[2] = lop3_and_or(w >> 8, 0x000F000Fu, 0x43004300u);
  p[3] = lop3_and_or(w >> 12, 0x000F000Fu, 0x43004300u);
}

// T: token tiles of 8 (1 for up to 8 tokens, 2 for up to 16).
// Up to 8 tokens two CTAs share an SM (more warps to hide the MMA and load latencies).
template <int FMT, int T>
__global__ void __launch_bounds__(kGsThreads, T == 1 ? 2 : 1)
    gemv_stream_kernel(const __grid_constant__ CUtensorMap tm_w, const GsParams p) {
  using F = GsFmt<FMT>;
  extern __shared__ __align__(128) uint8_t gs_smem_raw[];
  // 1024-byte alignment: the swizzle pattern of the weight boxes follows address bits 7-9
  uint8_t* gs_smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(gs_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(gs_smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;

  // this CTA's rows [r0, r1), tiles of 32
  const int n8 = (p.N + 7) / 8;
  const int cta = static_cast<int>(blockIdx.x);
  const int r0 = 8 * static_cast<int>(static_cast<int64_t>(cta) * n8 / p.grid);
  const int r1 = min(p.N, 8 * static_cast<int>(static_cast<int64_t>(cta + 1) * n8 / p.grid));
  const int J = r1 > r0 ? (r1 - r0 + kGsRows - 1) / kGsRows : 0;
  const int items = J * p.passes;  // item i: pass i / J, tile i % J

  const uint32_t bar0 = sb + p.off_bar;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (p.S + s); };
  volatile uint32_t* abort_flag =
      reinterpret_cast<volatile uint32_t*>(gs_smem + p.off_bar + 16 * p.S);

  if (tid == 0) {
    for (int s = 0; s < p.S; ++s) {
      mbar_init(full_bar(s), 1);          // the producer's expect_tx
      mbar_init(empty_bar(s), kGsWarps);  // every compute warp
    }
    *abort_flag = 0u;
    fence_mbar_init();
  }
  pdl_trigger();
  __syncwarp();
  __syncthreads();

  if (warp == kGsWarps) {
    // ---------------------------------------------------------- weight producer
    // Packed weights are not written by the kernels ahead on the stream, so the loads
    // start before the dependency wait.
    if (lane == 0) {
      tma_prefetch_desc(&tm_w);
      const uint32_t ring = sb + p.off_ring;
      const uint32_t slot_bytes = static_cast<uint32_t>(p.nbox * kGsBoxBytes);
      int i = 0;
      for (; i < items; ++i) {
        const int s = i % p.S;
        const uint32_t ph = static_cast<uint32_t>(i / p.S) & 1u;
        if (!mbar_wait(empty_bar(s), ph ^ 1u, abort_flag)) break;
        const int pass = i / J, t = i - pass * J;
        mbar_arrive_expect_tx(full_bar(s), static_cast<uint32_t>(p.nbox * kGsBoxBytes));
        const int xb = pass * (p.kp / kGsUnit) * F::kUnitBytes;  // the pass's first byte
        for (int b = 0; b < p.nbox; ++b)
          tma_load_2d(ring + s * slot_bytes + b * kGsBoxBytes, &tm_w, full_bar(s), xb + 128 * b,
                      r0 + t * kGsRows);
      }
      // every load issued must land before the CTA may exit
      for (int ii = max(0, i - p.S); ii < i; ++ii)
        mbar_wait_drain(full_bar(ii % p.S), static_cast<uint32_t>(ii / p.S) & 1u);
    }
    __syncwarp();
    return;
  }

  // ------------------------------------------------------------ compute warps
  const uint32_t ring = sb + p.off_ring;
  const uint32_t slot_bytes = static_cast<uint32_t>(p.nbox * kGsBoxBytes);
  const uint32_t xs = sb + p.off_x;
  float* corr = reinterpret_cast<float*>(gs_smem + p.off_corr);  // [unit of pass][16 tokens]
  float* red = reinterpret_cast<float*>(gs_smem + p.off_red);    // 2 x [warp][8T values][32 lanes]
  float* accs = reinterpret_cast<float*>(gs_smem + p.off_acc);   // [tile][8T values][32 lanes]
  // ldmatrix row addresses: lane l -> matrix l / 8 (token block l / 16, slot half (l / 8) % 2)
  // (only the M real token rows are staged: rows of absent tokens read the last real row,
  // and the outputs they feed are never stored)
  const uint32_t lm_addr = xs + min((lane >> 4) * 8 + (lane & 7), p.M - 1) * p.xs_stride +
                           ((lane >> 3) & 1) * 16;
  const int upass = p.kp / kGsUnit;  // units of a (full) pass

  // ---- every scale of this CTA's rows -> shared memory (zero past the rows), before the
  // wait: the scales are not written by the kernels ahead
  const int nsc = FMT == 0 ? p.K / 128 : p.K / 64;  // scale entries per row
  const int sc_row = p.U * F::kScl;                  // staged entries per row (whole units)
  {
    const int total = J * kGsRows * sc_row;
    constexpr int kBatch = 8;  // loads in flight per thread before their stores
    for (int e0 = tid; e0 < total; e0 += kBatch * kGsWarps * 32) {
      uint32_t v[kBatch];
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const int e = e0 + i * kGsWarps * 32;
        const int rt = e / sc_row, si = e - rt * sc_row;
        const int n = r0 + rt;
        v[i] = 0u;
        if (e < total && n < r1 && si < nsc) {
          const int64_t idx = static_cast<int64_t>(n) * nsc + si;
          v[i] = FMT == 0 ? static_cast<uint32_t>(__ldg(p.scales + idx))
                          : __ldg(reinterpret_cast<const uint32_t*>(p.scales) + idx);
        }
      }
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const int e = e0 + i * kGsWarps * 32;
        if (e >= total) break;
        if (FMT == 0)
          reinterpret_cast<uint16_t*>(gs_smem + p.off_sc)[e] = static_cast<uint16_t>(v[i]);
        else
          reinterpret_cast<uint32_t*>(gs_smem + p.off_sc)[e] = v[i];
      }
    }
  }
  const uint16_t* sc16 = reinterpret_cast<const uint16_t*>(gs_smem + p.off_sc);
  const uint32_t* sc32 = reinterpret_cast<const uint32_t*>(gs_smem + p.off_sc);
  pdl_wait();  // the activations may come from the kernels ahead

  bool ok = true;
  for (int it = 0; it < items; ++it) {
    const int pass = it / J, t = it - pass * J;
    const int row0 = r0 + t * kGsRows;
    if (t == 0) {
      // ---- this pass's activations -> shared memory (staged order), correction sums
      if (pass > 0) named_barrier_sync(1, kGsWarps * 32);  // everyone is done with the last pass
      const int u0 = pass * upass;
      const int un = min(upass, p.U - u0);
      // thread part of an item: Q2 halves (staged steps 4 h.. 4 h + 3 take words 4 h..4 h + 3,
      // k in [64 h, 64 h + 64)), 4-bit quarters (steps 2 h, 2 h + 1 take words 4 h..4 h + 3,
      // k in [32 h, 32 h + 32)); consecutive threads of a warp share an item
      constexpr int kParts = FMT == 0 ? 2 : 4;
      constexpr int kPk = kGsUnit / kParts;  // k of one part
      // warp-uniform trip count: every lane reaches the shuffle below
      for (int qb = warp * 32; qb < p.M * un * kParts; qb += kGsWarps * 32) {
        const int q0 = qb + lane;
        const bool active = q0 < p.M * un * kParts;
        const int item = active ? q0 / kParts : 0, h = q0 % kParts;
        const int m = item / un, u = item - m * un;
        const int k0 = (u0 + u) * kGsUnit + h * kPk;
        const int kv = active ? min(kPk, p.K - k0) : 0;  // k of this part present (4-bit half units)
        const uint4* src = reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(m) * p.K + k0);
        uint32_t v[kPk / 2];
#pragma unroll
        for (int i = 0; i < kPk / 8; ++i) {
          uint4 tt = make_uint4(0u, 0u, 0u, 0u);
          if (8 * i < kv) tt = __ldg(src + i);
          v[4 * i] = tt.x;
          v[4 * i + 1] = tt.y;
          v[4 * i + 2] = tt.z;
          v[4 * i + 3] = tt.w;
        }
        // x at part-relative k
        auto xk = [&](int k) -> uint32_t { return (v[k >> 1] >> (16 * (k & 1))) & 0xFFFFu; };
        const uint32_t dst = xs + m * p.xs_stride + u * (2 * kGsUnit);
        constexpr int kSteps = 8 / kParts;  // staged 16-groups of this part
#pragma unroll
        for (int ss = 0; ss < kSteps; ++ss) {
          if (!active) break;
          const int s = h * kSteps + ss;
          uint32_t o[8];
#pragma unroll
          for (int j = 0; j < 8; ++j)
            o[j] = xk(gs_stage_k<FMT>(ss, 2 * j)) | (xk(gs_stage_k<FMT>(ss, 2 * j + 1)) << 16);
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst + 32 * s), "r"(o[0]),
                       "r"(o[1]), "r"(o[2]), "r"(o[3])
                       : "memory");
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst + 32 * s + 16), "r"(o[4]),
                       "r"(o[5]), "r"(o[6]), "r"(o[7])
                       : "memory");
        }
        float sum = 0.f;
        if (FMT == 0) {
#pragma unroll
          for (int k = 0; k < kPk; ++k)  // sum_k (base_k + 1) x_k over the part, k ascending
            sum = fmaf(static_cast<float>(gs_q2_base(k) + 1), bf16_bits_to_f32(xk(k)), sum);
        } else {
#pragma unroll
          for (int k = 0; k < kPk; ++k) sum += bf16_bits_to_f32(xk(k));  // sum_k x_k over the part
        }
        // parts of one item sit in consecutive lanes (kParts divides 32, the stride is a
        // multiple of 32): add them in part order
        const float s1 = __shfl_down_sync(0xFFFFFFFFu, sum, 1);
        if (active) {
          if (FMT == 0) {
            if (h == 0) corr[u * 16 + m] = sum + s1;
          } else {
            if ((h & 1) == 0) corr[(2 * u + (h >> 1)) * 16 + m] = sum + s1;
          }
        }
      }
      named_barrier_sync(1, kGsWarps * 32);
    }

    const int s = it % p.S;
    if (!__all_sync(0xFFFFFFFFu, mbar_wait(full_bar(s), static_cast<uint32_t>(it / p.S) & 1u, abort_flag))) {
      ok = false;
    }
    float acc[2][T][4];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf)
#pragma unroll
      for (int tt = 0; tt < T; ++tt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[hf][tt][e] = 0.f;
    const uint32_t slot = ring + s * slot_bytes;
    const int un = min(upass, p.U - pass * upass);  // units of this pass
#pragma unroll
    for (int i = 0; i < kGsMaxUW; ++i) {
      const int u = warp + kGsWarps * i;  // unit within the pass
      if (!ok || u >= un) break;
      const int uw = u * F::kWordsPerUnit;
      if (FMT == 0) {
        float pacc[2][T][4];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
          for (int tt = 0; tt < T; ++tt)
#pragma unroll
            for (int e = 0; e < 4; ++e) pacc[hf][tt][e] = 0.f;
#pragma unroll
        for (int hw = 0; hw < 2; ++hw) {  // the lane's words c and c + 4
          uint32_t wd[4][3];              // rows g, g + 8, g + 16, g + 24: the word >> 0, 6, 12
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            wd[r][0] = ld_shared_u32(gs_code_addr(slot, g + 8 * r, uw + c + 4 * hw));
            wd[r][1] = wd[r][0] >> 6;
            wd[r][2] = wd[r][0] >> 12;
          }
#pragma unroll
          for (int sp = 0; sp < 4; ++sp) {
            // pairs 2 sp and 2 sp + 1 of each row's word (see gs_q2_pairs)
            uint32_t pr[4][8];
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
              for (int q = 2 * sp; q < 2 * sp + 2; ++q) {
                constexpr uint32_t kMask[3] = {0x00030003u, 0x000C000Cu, 0x00300030u};
                constexpr uint32_t kMagic[3] = {0x43004300u, 0x42004200u, 0x41004100u};
                pr[r][q] = lop3_and_or(wd[r][q / 3], kMask[q % 3], kMagic[q % 3]);
              }
            const uint32_t baddr = lm_addr + (u * kGsUnit + 16 * (4 * hw + sp)) * 2;
            uint32_t b[4];
            if (T == 1) {
              ldmatrix_x2(baddr, b[0], b[1]);
            } else {
              ldmatrix_x4(baddr, b);
            }
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              const uint32_t a[4] = {pr[2 * hf][2 * sp], pr[2 * hf + 1][2 * sp], pr[2 * hf][2 * sp + 1],
                                     pr[2 * hf + 1][2 * sp + 1]};
              mma_bf16_16816(pacc[hf][0], a, b[0], b[1]);
              if (T == 2) mma_bf16_16816(pacc[hf][T - 1], a, b[2], b[3]);
            }
          }
        }
#pragma unroll
        for (int tt = 0; tt < T; ++tt) {
          const float c0 = corr[u * 16 + 2 * c + 8 * tt], c1 = corr[u * 16 + 2 * c + 1 + 8 * tt];
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const int srow = (t * kGsRows + 16 * hf + g) * sc_row + pass * upass + u;
            const float d0 = __half2float(__ushort_as_half(sc16[srow]));
            const float d1 = __half2float(__ushort_as_half(sc16[srow + 8 * sc_row]));
            acc[hf][tt][0] = fmaf(d0, pacc[hf][tt][0] - c0, acc[hf][tt][0]);
            acc[hf][tt][1] = fmaf(d0, pacc[hf][tt][1] - c1, acc[hf][tt][1]);
            acc[hf][tt][2] = fmaf(d1, pacc[hf][tt][2] - c0, acc[hf][tt][2]);
            acc[hf][tt][3] = fmaf(d1, pacc[hf][tt][3] - c1, acc[hf][tt][3]);
          }
        }
      } else {
        const int ng = (pass * upass + u) * kGsUnit + 64 < p.K ? 2 : 1;  // groups of the unit
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          if (h2 >= ng) break;
          float pacc[2][T][4];
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
#pragma unroll
            for (int tt = 0; tt < T; ++tt)
#pragma unroll
              for (int e = 0; e < 4; ++e) pacc[hf][tt][e] = 0.f;
#pragma unroll
          for (int hw = 0; hw < 2; ++hw) {  // words c + 4 (2 h2 + hw): steps 4 h2 + 2 hw + {0, 1}
            const int word = c + 4 * (2 * h2 + hw);
            uint32_t pr[4][4];
#pragma unroll
            for (int r = 0; r < 4; ++r) gs_q4_pairs(ld_shared_u32(gs_code_addr(slot, g + 8 * r, uw + word)), pr[r]);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const uint32_t baddr = lm_addr + (u * kGsUnit + 16 * (4 * h2 + 2 * hw + hh)) * 2;
              uint32_t b[4];
              if (T == 1) {
                ldmatrix_x2(baddr, b[0], b[1]);
              } else {
                ldmatrix_x4(baddr, b);
              }
#pragma unroll
              for (int hf = 0; hf < 2; ++hf) {
                const uint32_t a[4] = {pr[2 * hf][2 * hh], pr[2 * hf + 1][2 * hh], pr[2 * hf][2 * hh + 1],
                                       pr[2 * hf + 1][2 * hh + 1]};
                mma_bf16_16816(pacc[hf][0], a, b[0], b[1]);
                if (T == 2) mma_bf16_16816(pacc[hf][T - 1], a, b[2], b[3]);
              }
            }
          }
#pragma unroll
          for (int tt = 0; tt < T; ++tt) {
            const float S0 = corr[(2 * u + h2) * 16 + 2 * c + 8 * tt];
            const float S1 = corr[(2 * u + h2) * 16 + 2 * c + 1 + 8 * tt];
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              const int srow = (t * kGsRows + 16 * hf + g) * sc_row + 2 * (pass * upass + u) + h2;
              const uint32_t v0 = sc32[srow], v1 = sc32[srow + 8 * sc_row];
              const float s0 = __half2float(__ushort_as_half(static_cast<uint16_t>(v0 & 0xFFFFu)));
              const float z0 = 128.f + __half2float(__ushort_as_half(static_cast<uint16_t>(v0 >> 16)));
              const float s1 = __half2float(__ushort_as_half(static_cast<uint16_t>(v1 & 0xFFFFu)));
              const float z1 = 128.f + __half2float(__ushort_as_half(static_cast<uint16_t>(v1 >> 16)));
              acc[hf][tt][0] = fmaf(s0, fmaf(-z0, S0, pacc[hf][tt][0]), acc[hf][tt][0]);
              acc[hf][tt][1] = fmaf(s0, fmaf(-z0, S1, pacc[hf][tt][1]), acc[hf][tt][1]);
              acc[hf][tt][2] = fmaf(s1, fmaf(-z1, S0, pacc[hf][tt][2]), acc[hf][tt][2]);
              acc[hf][tt][3] = fmaf(s1, fmaf(-z1, S1, pacc[hf][tt][3]), acc[hf][tt][3]);
            }
          }
        }
      }
    }
    // the slot's codes are read: order those generic-proxy reads before the producer's
    // next TMA write into the slot, then release it
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar(s));

    // ---- add the 8 warps' partial sums (warp order), over the passes; store after the last.
    // Value i of lane l of warp w sits at redb[(w * 8T + i) * 32 + l]: each store and each
    // load of a warp touches 32 consecutive words (no bank conflicts).  Thread (i, l) adds
    // value i of lane l over the warps: for i = (hf T + tt) 4 + e that is row-in-tile
    // rr = 16 hf + g + 8 (e >> 1) and token m = 8 tt + 2 c + (e & 1), with (g, c) of lane l.
    float* redb = red + (it & 1) * (kGsWarps * 32 * 8 * T);  // two buffers, alternating
#pragma unroll
    for (int hf = 0; hf < 2; ++hf)
#pragma unroll
      for (int tt = 0; tt < T; ++tt)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          redb[(warp * 8 * T + (hf * T + tt) * 4 + e) * 32 + lane] = acc[hf][tt][e];
    named_barrier_sync(1, kGsWarps * 32);
    const bool last = pass == p.passes - 1;
#pragma unroll
    for (int rep = 0; rep < T; ++rep) {
      const int o = tid + rep * kGsWarps * 32;  // (value i, lane l) = (o / 32, o % 32)
      const int i = o >> 5, l = o & 31;
      float v = pass > 0 ? accs[(t * 8 * T + i) * 32 + l] : 0.f;
#pragma unroll
      for (int w = 0; w < kGsWarps; ++w) v += redb[(w * 8 * T + i) * 32 + l];
      const int hf = i / (4 * T), tt = (i >> 2) % T, e = i & 3;
      const int rr = 16 * hf + (l >> 2) + 8 * (e >> 1);
      const int m = 8 * tt + 2 * (l & 3) + (e & 1);
      const int n = row0 + rr;
      if (!last) {
        accs[(t * 8 * T + i) * 32 + l] = v;
      } else if (n < r1 && m < p.M) {
        if (p.out_f32)
          reinterpret_cast<float*>(p.y)[static_cast<int64_t>(m) * p.N + n] = v;
        else
          reinterpret_cast<__nv_bfloat16*>(p.y)[static_cast<int64_t>(m) * p.N + n] = __float2bfloat16_rn(v);
      }
    }
    // no second barrier: the next item writes the other buffer, and this one is written
    // again only after every thread has passed the next item's barrier
  }
}

}  // namespace tgemm
