// gemv.cuh -- small-M path (M <= 16 tokens per pass): HBM-bound on the packed weights.
//
// Each CTA owns 32 weight rows (four 8-row n-blocks); its 8 warps split K in units of
// 128 weights.  Per pass of up to kGvKP weights along K:
//   * one thread copies the pass's activation rows into shared memory with bulk async
//     copies (cp.async.bulk, completion on an mbarrier), while
//   * every lane issues all of its packed-weight loads for the pass (8- or 16-byte loads
//     straight from HBM into registers),
// so the pass costs one memory round trip.  Codes are unpacked in registers into bf16
// mma.sync fragments and multiplied with the activations; block scales are applied to
// the f32 partial sums after each block, so the tensor cores see small exact integers:
//   Q2_0:  B = q - 1 in {-1, 0, 1}, then y += d * sum          (one 128-weight block)
//   4-bit: B = q in 0..15, S = sum of x over the group (an extra mma against ones),
//          then y += s * (sum - z * S)                          (two 64-weight groups)
// which equals sum_k (q - 1) d x  and  sum_k (q - z) s x  with only f32 rounding.
// The warps' partial sums are reduced through shared memory; the optional low-rank
// branch adds sum_i B[n][i] u[m][i] (u = A x in f32, from the lora kernels).
//
// Fragment order: a 32-bit word of Q2 codes unpacks with one shift and mask per pair
// into codes (i, i+8); a word of 4-bit codes into codes (i, i+4).  The matching
// activation pairs are gathered from shared memory with two 16-bit loads.
#pragma once

#include "common.cuh"

namespace tgemm {

constexpr int kGvRows = 32;         // weight rows per CTA
constexpr int kGvWarps = 8;         // warps per CTA, splitting K
constexpr int kGvUnit = 128;        // K per unit
constexpr int kGvKP = 4096;         // K per pass (activations staged in shared memory)
constexpr int kGvMaxU = kGvKP / kGvUnit / kGvWarps;  // units per warp per pass (4)

__host__ __device__ constexpr int gemv_row_stride_bytes(int kp) { return 2 * kp + 16; }
__host__ __device__ constexpr int gemv_smem_bytes(int mrows, int kp) {
  return mrows * gemv_row_stride_bytes(kp) + 16;
}

// mma.sync m16n8k16, bf16 inputs, f32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
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

__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}

// (x[k_lo], x[k_hi]) of one staged row as a bf16x2 fragment register.
__device__ __forceinline__ uint32_t x_pair(uint32_t row_addr, int k_lo, int k_hi) {
  return lds_u16(row_addr + 2 * k_lo) | (lds_u16(row_addr + 2 * k_hi) << 16);
}

__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                              uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

template <int FMT, bool LORA>
__global__ void __launch_bounds__(256) gemv_kernel(
    const uint16_t* __restrict__ x, const uint8_t* __restrict__ wq,
    const uint16_t* __restrict__ scales, void* __restrict__ y, int M, int N, int K, int out_f32,
    const float* __restrict__ u, const uint16_t* __restrict__ lb, int r, int mrows, int kp) {
  extern __shared__ __align__(16) uint8_t gv_smem[];
  __shared__ float red[kGvWarps][16][kGvRows + 1];
  // scales of this CTA's rows for one pass: Q2 d per unit, 4-bit (s, z) per group
  constexpr int kScl = FMT == 0 ? kGvKP / 128 : kGvKP / 64;
  __shared__ uint32_t scl[kGvRows][kScl];
  __shared__ uint32_t abort_flag;
  const uint32_t xs = smem_u32(gv_smem);
  const int rs = gemv_row_stride_bytes(kp);
  const uint32_t bar = xs + mrows * rs;  // 8-byte aligned: rs and the base are 16-aligned

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int n0 = blockIdx.x * kGvRows;
  const int nunits = K / kGvUnit + ((K % kGvUnit) ? 1 : 0);
  constexpr int kUnitBytes = FMT == 0 ? 32 : 64;   // packed bytes of one row per unit
  constexpr int kWords = FMT == 0 ? 2 : 4;         // 32-bit words a lane loads per row per unit
  const int64_t row_bytes = FMT == 0 ? K / 4 : K / 2;
  const int nscale = FMT == 0 ? K / 128 : K / 64;  // scale entries per row

  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    abort_flag = 0u;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_trigger_and_wait();
  uint32_t phase = 0;

  for (int m0 = 0; m0 < M; m0 += 16) {
    const int mt = min(16, M - m0);  // tokens in this tile (<= mrows)
    float acc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;

    for (int k0 = 0; k0 < K; k0 += kp) {
      const int kpass = min(kp, K - k0);
      // ---- activations for this pass: one bulk copy per token row
      if (threadIdx.x == 0) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(bar, static_cast<uint32_t>(mt * kpass * 2));
        for (int i = 0; i < mt; ++i)
          bulk_copy_g2s(xs + i * rs, x + static_cast<int64_t>(m0 + i) * K + k0,
                        static_cast<uint32_t>(kpass * 2), bar);
      }
      // ---- every packed-weight load of this pass
      const int u_base = k0 / kGvUnit;
      const int u_end = min(nunits, (k0 + kpass + kGvUnit - 1) / kGvUnit);
      uint32_t wreg[kGvMaxU][4][kWords];
#pragma unroll
      for (int i = 0; i < kGvMaxU; ++i) {
        const int unit = u_base + i * kGvWarps + warp;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int row = n0 + 8 * j + g;
          const bool ok = unit < u_end && row < N;
          const uint8_t* base = wq + static_cast<int64_t>(row) * row_bytes +
                                static_cast<int64_t>(unit) * kUnitBytes;
          if (FMT == 0) {
            uint2 v = make_uint2(0x55555555u, 0x55555555u);  // code 1 everywhere = weight 0
            if (ok) v = __ldg(reinterpret_cast<const uint2*>(base + 8 * c));
            wreg[i][j][0] = v.x;
            wreg[i][j][1] = v.y;
          } else {
            uint2 v0 = make_uint2(0u, 0u), v1 = make_uint2(0u, 0u);
            if (ok) {
              v0 = __ldg(reinterpret_cast<const uint2*>(base + 8 * c));
              if (static_cast<int64_t>(unit) * kGvUnit + 64 < K)
                v1 = __ldg(reinterpret_cast<const uint2*>(base + 32 + 8 * c));
            }
            wreg[i][j][0] = v0.x;
            wreg[i][j][1] = v0.y;
            wreg[i][j][2] = v1.x;
            wreg[i][j][3] = v1.y;
          }
        }
      }
      // ---- this pass's scales for the CTA's rows, staged in shared memory
      {
        const int s_base = FMT == 0 ? u_base : 2 * u_base;
        const int s_cnt = FMT == 0 ? (u_end - u_base) : min(nscale - s_base, 2 * (u_end - u_base));
        for (int it = threadIdx.x; it < kGvRows * s_cnt; it += blockDim.x) {
          const int rl = it / s_cnt, si = it % s_cnt;
          const int n = n0 + rl;
          uint32_t v = 0;
          if (n < N) {
            const int64_t idx = static_cast<int64_t>(n) * nscale + s_base + si;
            v = FMT == 0 ? static_cast<uint32_t>(scales[idx])
                         : reinterpret_cast<const uint32_t*>(scales)[idx];
          }
          scl[rl][si] = v;
        }
      }
      // ---- wait for the activations (bounded; the CTA leaves together on a timeout)
      const bool ok = mbar_wait(bar, phase, &abort_flag);
      if (__syncthreads_or(!ok)) return;
      phase ^= 1u;
      const bool g0 = g < mt, g1 = g + 8 < mt;
      const uint32_t row0 = xs + g * rs, row1 = xs + (g + 8) * rs;
#pragma unroll
      for (int i = 0; i < kGvMaxU; ++i) {
        const int unit = u_base + i * kGvWarps + warp;
        if (unit >= u_end) break;
        const int ku = (unit - u_base) * kGvUnit;  // unit offset within the pass
        if (FMT == 0) {
          float part[4][4];
#pragma unroll
          for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) part[j][e] = 0.f;
#pragma unroll
          for (int kb = 0; kb < 8; ++kb) {
            const int jw = kb >> 2, p = kb & 3;
            const int k1 = ku + 32 * c + 16 * jw + p;  // codes (k1, k1+8) and (k1+4, k1+12)
            const uint32_t a0 = g0 ? x_pair(row0, k1, k1 + 8) : 0u;
            const uint32_t a1 = g1 ? x_pair(row1, k1, k1 + 8) : 0u;
            const uint32_t a2 = g0 ? x_pair(row0, k1 + 4, k1 + 12) : 0u;
            const uint32_t a3 = g1 ? x_pair(row1, k1 + 4, k1 + 12) : 0u;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t wv = wreg[i][j][jw];
              mma_bf16_16816(part[j], a0, a1, a2, a3, q2_pair_bf16(wv, 2 * p),
                             q2_pair_bf16(wv, 2 * p + 8));
            }
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
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
            if (grp * 64 >= K) break;
            float part[4][4], ssum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
              for (int e = 0; e < 4; ++e) part[j][e] = 0.f;
#pragma unroll
            for (int kq = 0; kq < 4; ++kq) {
              const int jj = kq >> 1, half = kq & 1;
              const int k1 = ku + 64 * h2 + 16 * c + 8 * jj + 2 * half;  // (k1, k1+4), (k1+1, k1+5)
              const uint32_t a0 = g0 ? x_pair(row0, k1, k1 + 4) : 0u;
              const uint32_t a1 = g1 ? x_pair(row1, k1, k1 + 4) : 0u;
              const uint32_t a2 = g0 ? x_pair(row0, k1 + 1, k1 + 5) : 0u;
              const uint32_t a3 = g1 ? x_pair(row1, k1 + 1, k1 + 5) : 0u;
              mma_bf16_16816(ssum, a0, a1, a2, a3, 0x3F803F80u, 0x3F803F80u);
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const uint32_t wv = wreg[i][j][2 * h2 + jj];
                mma_bf16_16816(part[j], a0, a1, a2, a3, q4_pair_bf16(wv, 8 * half),
                               q4_pair_bf16(wv, 8 * half + 4));
              }
            }
            // ssum[0] = S for token g, ssum[2] = S for token g + 8
#pragma unroll
            for (int j = 0; j < 4; ++j) {
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
      __syncthreads();  // everyone is done with this pass's activations
    }

    // ---- reduce the warps' partial sums and write y ---------------------------------
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      red[warp][g][8 * j + 2 * c] = acc[j][0];
      red[warp][g][8 * j + 2 * c + 1] = acc[j][1];
      red[warp][g + 8][8 * j + 2 * c] = acc[j][2];
      red[warp][g + 8][8 * j + 2 * c + 1] = acc[j][3];
    }
    __syncthreads();
    for (int o = threadIdx.x; o < 16 * kGvRows; o += blockDim.x) {
      const int mm = o / kGvRows, nn = o % kGvRows;
      const int m = m0 + mm, n = n0 + nn;
      if (m >= M || n >= N) continue;
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kGvWarps; ++w) v += red[w][mm][nn];
      if (LORA) {
        float br = 0.f;
        for (int i = 0; i < r; ++i)
          br = fmaf(bf16_bits_to_f32(lb[static_cast<int64_t>(n) * r + i]), u[static_cast<int64_t>(m) * r + i], br);
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
