// gemv.cuh -- small-M path (up to 16 tokens per tile): HBM-bound on the packed weights.
//
// Each CTA owns 16 weight rows (two 8-row n-tiles of mma.sync m16n8k16); its 8 warps split
// K in units of 128 weights.  Per pass of up to kp weights along K:
//   * every lane issues all of its packed-weight loads for the pass first: lane (g, c)
//     loads the c-th quarter of row g's packed bytes of each of its units, so the warp
//     reads each row-unit once and a whole pass costs one memory round trip;
//   * the CTA stages the pass's activation rows in shared memory, converted to the
//     fragment order of the codes (below), so one ldmatrix.x4 yields a whole A fragment;
//     tokens past the tile read a shared row of zeros;
//   * codes are unpacked in registers (the word a lane needs comes from the lane of its
//     quad that loaded it, by shuffle) into exact bf16 integers for the mma;
//   * block scales are applied to the f32 partial sums after each block:
//       Q2_0:  B = q - 1 in {-1, 0, 1}, then y += d * sum              (128-weight block)
//       4-bit: B = q in 0..15, S = sum of x over the group (an mma against ones),
//              then y += s * (sum - z * S)                              (64-weight group)
//     which equals sum_k (q - 1) d x  and  sum_k (q - z) s x  with only f32 rounding.
// The warps' partial sums are reduced through shared memory; the optional low-rank
// branch adds sum_i B[n][i] u[m][i] (u = A x in f32, from the lora kernels).
//
// Fragment order: a 32-bit word of Q2 codes unpacks with one shift and mask per pair into
// codes (i, i+8); a word of 4-bit codes into codes (i, i+4).  The staged activations hold,
// in each 16-group (Q2) or 8-group (4-bit), x[i] and x[i+8] (x[i] and x[i+4]) side by
// side, so the mma's k pair (2i, 2i+1) is the same pair of weights on both operands.
#pragma once

#include "common.cuh"

namespace tgemm {

constexpr int kGvRows = 16;   // weight rows per CTA
constexpr int kGvWarps = 8;   // warps per CTA, splitting K
constexpr int kGvUnit = 128;  // K per unit
constexpr int kGvMaxU = 6;    // units per warp per pass
constexpr int kGvKPMax = kGvMaxU * kGvWarps * kGvUnit;  // 6144
// Dynamic shared memory per CTA: the staged activations (two CTAs per SM, 16 tokens x
// 3072 in one pass); after the last pass it holds the warps' partial sums instead.
constexpr int kGvXBudget = 104960;
constexpr int kGvRedBytes = kGvWarps * 16 * (kGvRows + 1) * 4;

__host__ __device__ constexpr int gemv_row_stride_bytes(int kp) { return 2 * kp + 16; }
// K per pass: the largest multiple of 128 (at most kGvKPMax) whose staged activation rows
// (`mrows` tokens plus one row of zeros) fit kGvXBudget; never more than K needs.
__host__ __device__ inline int gemv_pass_k(int mrows, int K) {
  int kp = (K + kGvUnit - 1) / kGvUnit * kGvUnit;
  if (kp > kGvKPMax) kp = kGvKPMax;
  while (kp > kGvUnit && (mrows + 1) * gemv_row_stride_bytes(kp) > kGvXBudget) kp -= kGvUnit;
  return kp;
}
__host__ __device__ constexpr int gemv_smem_bytes(int mrows, int kp) {
  return (mrows + 1) * gemv_row_stride_bytes(kp) > kGvRedBytes
             ? (mrows + 1) * gemv_row_stride_bytes(kp)
             : kGvRedBytes;
}

// bf16x2 a - b (exact for the small integers used here)
__device__ __forceinline__ uint32_t bsub2(uint32_t a, uint32_t b) {
  __nv_bfloat162 r =
      __hsub2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

// Two 2-bit codes (bits s..s+1 and s+16..s+17 of w) -> bf16x2 (q - 1).
__device__ __forceinline__ uint32_t q2_pair_bf16(uint32_t w, int s) {
  const uint32_t t = lop3_and_or(w >> s, 0x00030003u, 0x43004300u);  // 128 + q
  return bsub2(t, 0x43014301u);                                       // - 129
}

// Two 4-bit codes (bits s..s+3 and s+16..s+19 of w) -> bf16x2 q.
__device__ __forceinline__ uint32_t q4_pair_bf16(uint32_t w, int s) {
  const uint32_t t = lop3_and_or(w >> s, 0x000F000Fu, 0x43004300u);  // 128 + q
  return bsub2(t, 0x43004300u);                                       // - 128
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

__device__ __forceinline__ void st_shared_v4(uint32_t saddr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(saddr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// 16 bf16 activations (v: pairs (0,1) .. (14,15)) -> the fragment order of format FMT.
//   Q2:    word i = (x[i], x[i+8])                         i < 8
//   4-bit: word 4h+i = (x[8h+i], x[8h+i+4])                h < 2, i < 4
template <int FMT>
__device__ __forceinline__ void x_fragment_order(const uint32_t (&v)[8], uint32_t (&o)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (FMT == 0) {
      const uint32_t sel = (i & 1) ? 0x7632u : 0x5410u;  // odd i: the high halves
      o[i] = prmt(v[i >> 1], v[4 + (i >> 1)], sel);
    } else {
      const int h = i >> 2, j = i & 3;
      const uint32_t sel = (j & 1) ? 0x7632u : 0x5410u;
      o[i] = prmt(v[4 * h + (j >> 1)], v[4 * h + 2 + (j >> 1)], sel);
    }
  }
}

// DUAL: a second input (x2, wq2, scales2, K2) whose product adds into the same sums.
template <int FMT, bool LORA, bool DUAL>
__global__ void __launch_bounds__(256) gemv_kernel(
    const uint16_t* __restrict__ x, const uint8_t* __restrict__ wq,
    const uint16_t* __restrict__ scales, void* __restrict__ y, int M, int N, int K, int out_f32,
    const float* __restrict__ u, const uint16_t* __restrict__ lb, int r, int lb_sn, int lb_si,
    int mrows, int kp,
    const uint16_t* __restrict__ x2, const uint8_t* __restrict__ wq2,
    const uint16_t* __restrict__ scales2, int K2) {
  extern __shared__ __align__(16) uint8_t gv_smem[];
  // the warps' partial sums, over the staged activations once all passes are done
  auto red = reinterpret_cast<float(*)[16][kGvRows + 1]>(gv_smem);
  // scales of this CTA's rows for one pass: Q2 d per unit, 4-bit (s, z) per group
  constexpr int kScl = FMT == 0 ? kGvKPMax / 128 : kGvKPMax / 64;
  __shared__ uint32_t scl[kGvRows][kScl];
  pdl_trigger();
  {
    // the first pass's packed rows -> L2 while the previous kernel finishes (no data
    // reaches the SM before the wait below)
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    const int64_t rb = FMT == 0 ? K / 4 : K / 2;
    const int units0 = min((K + kGvUnit - 1) / kGvUnit, kp / kGvUnit);
    const int row = blockIdx.x * kGvRows + (l & 15);
    if (row < N)
      for (int un = w + kGvWarps * (l >> 4); un < units0; un += 2 * kGvWarps)
        prefetch_l2(wq + static_cast<int64_t>(row) * rb + static_cast<int64_t>(un) * (FMT == 0 ? 32 : 64));
  }
  pdl_wait();
  const uint32_t xs = smem_u32(gv_smem);
  const int rs = gemv_row_stride_bytes(kp);
  const uint32_t zrow = xs + mrows * rs;  // zeros: the rows of tokens past the tile

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const int n0 = blockIdx.x * kGvRows;
  constexpr int kUnitBytes = FMT == 0 ? 32 : 64;  // packed bytes of one row per unit
  constexpr int kQW = FMT == 0 ? 2 : 4;           // 32-bit words a lane loads per row-unit

  // ldmatrix.x4 row address of this lane: matrices (tokens 0-7 | 8-15) x (k 0-7 | 8-15)
  const int mi = lane >> 3, arow = (mi & 1) * 8 + (lane & 7);
  const uint32_t a_col = (mi >> 1) * 16;

  for (int m0 = 0; m0 < M; m0 += 16) {
    const int mt = min(16, M - m0);  // tokens in this tile (<= mrows)
    const uint32_t a_row = (arow < mt ? xs + arow * rs : zrow) + a_col;
    // (re)zero the zero row: the previous tile's partial sums may have covered it
    for (int i = tid; i < rs / 16; i += blockDim.x) st_shared_v4(zrow + 16 * i, 0u, 0u, 0u, 0u);
    float acc[2][4];
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;

    // one input, or two (a projection split along its input axis: their products add
    // into the same partial sums)
    for (int part = 0; part < (DUAL ? 2 : 1); ++part) {
      const uint16_t* xq = part ? x2 : x;
      const uint8_t* wqq = part ? wq2 : wq;
      const uint16_t* sq = part ? scales2 : scales;
      const int Kq = part ? K2 : K;
      const int nunitsq = (Kq + kGvUnit - 1) / kGvUnit;
      const int64_t row_bytesq = FMT == 0 ? Kq / 4 : Kq / 2;
      const int nscaleq = FMT == 0 ? Kq / 128 : Kq / 64;
      for (int k0 = 0; k0 < Kq; k0 += kp) {
        const int kpass = min(kp, Kq - k0);
        const int u_base = k0 / kGvUnit;
        const int u_end = min(nunitsq, (k0 + kpass + kGvUnit - 1) / kGvUnit);
        // ---- every packed-weight load of this pass (lane (g, c): quarter c of row g)
        uint32_t wreg[kGvMaxU][2][kQW];
#pragma unroll
        for (int i = 0; i < kGvMaxU; ++i) {
          const int unit = u_base + i * kGvWarps + warp;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int row = n0 + 8 * j + g;
            const bool ok = unit < u_end && row < N;
            const uint8_t* base = wqq + static_cast<int64_t>(row) * row_bytesq +
                                  static_cast<int64_t>(unit) * kUnitBytes;
            if (FMT == 0) {
              uint2 v = make_uint2(0x55555555u, 0x55555555u);  // code 1 everywhere = weight 0
              if (ok) v = __ldg(reinterpret_cast<const uint2*>(base + 8 * c));
              wreg[i][j][0] = v.x;
              wreg[i][j][1] = v.y;
            } else {
              // a unit's second 32 bytes exist only where K reaches its second group
              uint4 v = make_uint4(0u, 0u, 0u, 0u);
              if (ok && (c < 2 || static_cast<int64_t>(unit) * kGvUnit + 64 < Kq))
                v = __ldg(reinterpret_cast<const uint4*>(base + 16 * c));
              wreg[i][j][0] = v.x;
              wreg[i][j][1] = v.y;
              wreg[i][j][2] = v.z;
              wreg[i][j][3] = v.w;
            }
          }
        }
        // ---- this pass's sq for the CTA's rows
        {
          const int s_base = FMT == 0 ? u_base : 2 * u_base;
          const int s_cnt = FMT == 0 ? (u_end - u_base) : min(nscaleq - s_base, 2 * (u_end - u_base));
          for (int it = tid; it < kGvRows * s_cnt; it += blockDim.x) {
            const int rl = it / s_cnt, si = it - rl * s_cnt;
            const int n = n0 + rl;
            uint32_t v = 0;
            if (n < N) {
              const int64_t idx = static_cast<int64_t>(n) * nscaleq + s_base + si;
              v = FMT == 0 ? static_cast<uint32_t>(sq[idx])
                           : reinterpret_cast<const uint32_t*>(sq)[idx];
            }
            scl[rl][si] = v;
          }
        }
        // ---- the pass's activations, in fragment order
        {
          const int ng = kpass / 16;  // 16-element groups per token row
          for (int gi = tid; gi < mt * ng; gi += blockDim.x) {
            const int row = gi / ng, grp = gi - row * ng;
            const uint4* src = reinterpret_cast<const uint4*>(
                xq + static_cast<int64_t>(m0 + row) * Kq + k0 + 16 * grp);
            const uint4 a = __ldg(src), b = __ldg(src + 1);
            const uint32_t v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
            uint32_t o[8];
            x_fragment_order<FMT>(v, o);
            const uint32_t dst = xs + row * rs + 32 * grp;
            st_shared_v4(dst, o[0], o[1], o[2], o[3]);
            st_shared_v4(dst + 16, o[4], o[5], o[6], o[7]);
          }
        }
        __syncthreads();
        // ---- the warp's units: A fragments by ldmatrix, B fragments from the codes
#pragma unroll
        for (int i = 0; i < kGvMaxU; ++i) {
          const int unit = u_base + i * kGvWarps + warp;
          if (unit >= u_end) break;
          const int ku = (unit - u_base) * kGvUnit;  // unit offset within the pass
          if (FMT == 0) {
            float part[2][4];
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
              for (int e = 0; e < 4; ++e) part[j][e] = 0.f;
#pragma unroll
            for (int s = 0; s < 8; ++s) {  // k16 step s: word s of the row-unit
              uint32_t af[4];
              ldmatrix_x4(a_row + 2 * (ku + 16 * s), af);
              const int src = (lane & ~3) | (s >> 1);  // the quad lane that loaded word s
#pragma unroll
              for (int j = 0; j < 2; ++j) {
                const uint32_t w = __shfl_sync(0xFFFFFFFFu, wreg[i][j][s & 1], src);
                mma_bf16_16816(part[j], af, q2_pair_bf16(w, 2 * c), q2_pair_bf16(w, 2 * c + 8));
              }
            }
            // part[j][e]: token g (+8 for e >= 2), weight row 8j + 2c + (e & 1)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const int rl = 8 * j + 2 * c, ui = unit - u_base;
              const float d0 = __half2float(__ushort_as_half(static_cast<uint16_t>(scl[rl][ui])));
              const float d1 = __half2float(__ushort_as_half(static_cast<uint16_t>(scl[rl + 1][ui])));
              acc[j][0] = fmaf(d0, part[j][0], acc[j][0]);
              acc[j][1] = fmaf(d1, part[j][1], acc[j][1]);
              acc[j][2] = fmaf(d0, part[j][2], acc[j][2]);
              acc[j][3] = fmaf(d1, part[j][3], acc[j][3]);
            }
          } else {
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int grp = 2 * unit + h2;
              if (grp * 64 >= Kq) break;
              float part[2][4], ssum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
              for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) part[j][e] = 0.f;
#pragma unroll
              for (int sq = 0; sq < 4; ++sq) {  // k16 step s: words 2s, 2s+1 of the row-unit
                const int s = 4 * h2 + sq;
                uint32_t af[4];
                ldmatrix_x4(a_row + 2 * (ku + 16 * s), af);
                mma_bf16_16816(ssum, af, 0x3F803F80u, 0x3F803F80u);  // xq against ones
                const int src = (lane & ~3) | (s >> 1);
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                  const uint32_t w0 = __shfl_sync(0xFFFFFFFFu, wreg[i][j][2 * (s & 1)], src);
                  const uint32_t w1 = __shfl_sync(0xFFFFFFFFu, wreg[i][j][2 * (s & 1) + 1], src);
                  mma_bf16_16816(part[j], af, q4_pair_bf16(w0, 4 * c), q4_pair_bf16(w1, 4 * c));
                }
              }
              // ssum[0] = S for token g, ssum[2] = S for token g + 8
#pragma unroll
              for (int j = 0; j < 2; ++j) {
                const int rl = 8 * j + 2 * c, gi = grp - 2 * u_base;
                const uint32_t v0 = scl[rl][gi], v1 = scl[rl + 1][gi];
                const float s0 = __half2float(__ushort_as_half(static_cast<uint16_t>(v0 & 0xFFFFu)));
                const float z0 = __half2float(__ushort_as_half(static_cast<uint16_t>(v0 >> 16)));
                const float s1 = __half2float(__ushort_as_half(static_cast<uint16_t>(v1 & 0xFFFFu)));
                const float z1 = __half2float(__ushort_as_half(static_cast<uint16_t>(v1 >> 16)));
                acc[j][0] = fmaf(s0, fmaf(-z0, ssum[0], part[j][0]), acc[j][0]);
                acc[j][1] = fmaf(s1, fmaf(-z1, ssum[0], part[j][1]), acc[j][1]);
                acc[j][2] = fmaf(s0, fmaf(-z0, ssum[2], part[j][2]), acc[j][2]);
                acc[j][3] = fmaf(s1, fmaf(-z1, ssum[2], part[j][3]), acc[j][3]);
              }
            }
          }
        }
        __syncthreads();  // everyone is done with this pass's activations and sq
      }
    }

    // ---- reduce the warps' partial sums and write y ---------------------------------
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      red[warp][g][8 * j + 2 * c] = acc[j][0];
      red[warp][g][8 * j + 2 * c + 1] = acc[j][1];
      red[warp][g + 8][8 * j + 2 * c] = acc[j][2];
      red[warp][g + 8][8 * j + 2 * c + 1] = acc[j][3];
    }
    __syncthreads();
    for (int o = tid; o < 16 * kGvRows; o += blockDim.x) {
      const int mm = o / kGvRows, nn = o % kGvRows;
      const int m = m0 + mm, n = n0 + nn;
      if (m >= M || n >= N) continue;
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kGvWarps; ++w) v += red[w][mm][nn];
      if (LORA) {
        float br = 0.f;
        for (int i = 0; i < r; ++i)
          br = fmaf(bf16_bits_to_f32(lb[static_cast<int64_t>(n) * lb_sn + static_cast<int64_t>(i) * lb_si]),
                    u[static_cast<int64_t>(m) * r + i], br);
        v += br;
      }
      if (out_f32)
        reinterpret_cast<float*>(y)[static_cast<int64_t>(m) * N + n] = v;
      else
        reinterpret_cast<__nv_bfloat16*>(y)[static_cast<int64_t>(m) * N + n] = __float2bfloat16_rn(v);
    }
    __syncthreads();
  }
}

}  // namespace tgemm
