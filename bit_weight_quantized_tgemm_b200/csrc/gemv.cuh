// gemv.cuh -- small-M path (M <= 16 tokens per pass): HBM-bound on the packed weights.
//
// Each CTA owns 32 weight rows (four 8-row n-blocks) and all K; its 8 warps split K in
// units of 128 weights.  Per unit, a lane loads its share of the packed rows straight
// from HBM with 8- or 16-byte loads (all of a pass's loads are issued before any is
// used), unpacks the codes in registers into bf16 mma.sync fragments and multiplies them
// with the activations held in shared memory.  Block scales are applied to the f32
// partial sums after each unit, so the tensor cores see small exact integers:
//   Q2_0:  B = q - 1 in {-1, 0, 1}, then y += d * sum          (one 128-weight block)
//   4-bit: B = q in 0..15, S = sum of x over the group (an extra mma against ones),
//          then y += s * (sum - z * S)                          (two 64-weight groups)
// which equals sum_k (q - 1) d x  and  sum_k (q - z) s x  with only f32 rounding.
// The warps' partial sums are reduced through shared memory; the optional low-rank
// branch adds sum_i B[n][i] u[m][i] (u = A x in f32, computed by lora_down_kernel).
#pragma once

#include "common.cuh"

namespace tgemm {

constexpr int kGvRows = 32;         // weight rows per CTA
constexpr int kGvWarps = 8;         // warps per CTA, splitting K
constexpr int kGvUnit = 128;        // K per unit
constexpr int kGvMaxU = 4;          // units per warp per pass (weights held in registers)
constexpr int kGvSub = kGvWarps;    // units per X sub-chunk (one per warp)
constexpr int kGvRowWords = kGvSub * 64 + 4;  // X words per token row in smem (+4 pad)

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

// Activation staging.  For one unit (128 k) of one token row the 64 words hold bf16
// pairs in the order the fragments want them, lane-minor so a warp's 32 loads of one
// fragment register hit 32 different banks (row stride = 516 words = 4 mod 32):
//   Q2:   word ((j*4 + p)*2 + h)*4 + c = (x[32c+16j+p+4h], x[32c+16j+p+4h+8])
//   4-bit word (kb*2 + hh)*4 + c       = (x[k1+hh], x[k1+hh+4]),
//         k1 = 64*(kb/4) + 16c + 8*((kb%4)/2) + 2*(kb%2)
// (j, p: word and pair of a Q2 lane's codes; kb: mma k-block; c = lane % 4).
template <int FMT>
__device__ __forceinline__ void stage_x_subchunk(uint32_t* xs, const uint16_t* __restrict__ x,
                                                 int M, int K, int m0, int k0) {
  // 16 rows x (kGvSub*128) k; thread handles 16 consecutive k of one row per step
  constexpr int kGroupsPerRow = kGvSub * kGvUnit / 16;
  for (int it = threadIdx.x; it < 16 * kGroupsPerRow; it += blockDim.x) {
    const int row = it / kGroupsPerRow;
    const int gi = it % kGroupsPerRow;  // 16-k group within the sub-chunk
    const int m = m0 + row;
    const int k = k0 + gi * 16;
    uint32_t v[8];
    if (m < M && k < K) {
      const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(m) * K + k);
      const uint4 a = __ldg(src), b = __ldg(src + 1);
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
      v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0u;
    }
    // element e of the group = half (e & 1) of v[e >> 1]
    auto el = [&](int e) -> uint32_t { return (v[e >> 1] >> (16 * (e & 1))) & 0xFFFFu; };
    uint32_t* rowp = xs + row * kGvRowWords + (gi / 8) * 64;  // unit base
    const int gu = gi % 8;                                     // 16-group within the unit
    if (FMT == 0) {
      const int c = gu >> 1, j = gu & 1;
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int h = 0; h < 2; ++h)
          rowp[((j * 4 + p) * 2 + h) * 4 + c] = el(p + 4 * h) | (el(p + 4 * h + 8) << 16);
    } else {
      // two 8-groups: 8-group index within the unit G8 = 2*gu + e8
#pragma unroll
      for (int e8 = 0; e8 < 2; ++e8) {
        const int G8 = 2 * gu + e8;          // = 8*h2 + 2c + jj
        const int h2 = G8 >> 3, c = (G8 >> 1) & 3, jj = G8 & 1;
#pragma unroll
        for (int half = 0; half < 2; ++half) {   // kb % 2
          const int kb = 4 * h2 + 2 * jj + half;
          const int i0 = 2 * half;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
            rowp[(kb * 2 + hh) * 4 + c] =
                el(8 * e8 + i0 + hh) | (el(8 * e8 + i0 + hh + 4) << 16);
        }
      }
    }
  }
}

template <int FMT, bool LORA>
__global__ void __launch_bounds__(256) gemv_kernel(
    const uint16_t* __restrict__ x, const uint8_t* __restrict__ wq,
    const uint16_t* __restrict__ scales, void* __restrict__ y, int M, int N, int K, int out_f32,
    const float* __restrict__ u, const uint16_t* __restrict__ lb, int r) {
  __shared__ uint32_t xs[16 * kGvRowWords];
  // the warps' partial sums reuse the activation buffer once a token tile is done
  static_assert(sizeof(float) * kGvWarps * 16 * (kGvRows + 1) <= sizeof(uint32_t) * 16 * kGvRowWords,
                "reduction buffer must fit in the staging buffer");
  auto red = reinterpret_cast<float (*)[16][kGvRows + 1]>(xs);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int n0 = blockIdx.x * kGvRows;
  const int nunits = (K + kGvUnit - 1) / kGvUnit;
  constexpr int kUnitBytes = FMT == 0 ? 32 : 64;   // packed bytes of one row per unit
  constexpr int kWords = FMT == 0 ? 2 : 4;         // 32-bit words a lane loads per row per unit
  const int64_t row_bytes = FMT == 0 ? K / 4 : K / 2;
  const int nscale = FMT == 0 ? K / 128 : K / 64;  // scale entries per row

  for (int m0 = 0; m0 < M; m0 += 16) {
    float acc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;

    for (int pass_u = 0; pass_u < nunits; pass_u += kGvSub * kGvMaxU) {
      // ---- issue every weight load of this pass --------------------------------------
      uint32_t wreg[kGvMaxU][4][kWords];
#pragma unroll
      for (int i = 0; i < kGvMaxU; ++i) {
        const int unit = pass_u + i * kGvSub + warp;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int row = n0 + 8 * j + g;
          const bool ok = unit < nunits && row < N;
          const uint8_t* base = wq + static_cast<int64_t>(row) * row_bytes + static_cast<int64_t>(unit) * kUnitBytes;
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
      // ---- consume them sub-chunk by sub-chunk ---------------------------------------
#pragma unroll
      for (int i = 0; i < kGvMaxU; ++i) {
        const int sub_u = pass_u + i * kGvSub;
        if (sub_u >= nunits) break;
        __syncthreads();  // previous readers of xs are done
        stage_x_subchunk<FMT>(xs, x, M, K, m0, sub_u * kGvUnit);
        __syncthreads();
        const int unit = sub_u + warp;
        if (unit >= nunits) continue;
        const uint32_t* xrow0 = xs + g * kGvRowWords + warp * 64;
        const uint32_t* xrow1 = xs + (g + 8) * kGvRowWords + warp * 64;
        if (FMT == 0) {
          float part[4][4];
#pragma unroll
          for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) part[j][e] = 0.f;
#pragma unroll
          for (int kb = 0; kb < 8; ++kb) {
            const int jw = kb >> 2, p = kb & 3;
            const int w0 = ((jw * 4 + p) * 2 + 0) * 4 + c, w1 = w0 + 4;
            const uint32_t a0 = xrow0[w0], a1 = xrow1[w0], a2 = xrow0[w1], a3 = xrow1[w1];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t wv = wreg[i][j][jw];
              mma_bf16_16816(part[j], a0, a1, a2, a3, q2_pair_bf16(wv, 2 * p),
                             q2_pair_bf16(wv, 2 * p + 8));
            }
          }
          // block scale d[n][unit] for columns n = n0 + 8j + 2c, +1
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int n = n0 + 8 * j + 2 * c;
            const float d0 = n < N ? __half2float(__ushort_as_half(scales[static_cast<int64_t>(n) * nscale + unit])) : 0.f;
            const float d1 = n + 1 < N ? __half2float(__ushort_as_half(scales[static_cast<int64_t>(n + 1) * nscale + unit])) : 0.f;
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
              const int kb = 4 * h2 + kq;
              const int jj = kq >> 1, half = kq & 1;
              const int w0 = (kb * 2 + 0) * 4 + c, w1 = w0 + 4;
              const uint32_t a0 = xrow0[w0], a1 = xrow1[w0], a2 = xrow0[w1], a3 = xrow1[w1];
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
              const int n = n0 + 8 * j + 2 * c;
              float s0 = 0.f, z0 = 0.f, s1 = 0.f, z1 = 0.f;
              if (n < N) {
                const uint32_t v = reinterpret_cast<const uint32_t*>(scales)[static_cast<int64_t>(n) * nscale + grp];
                s0 = __half2float(__ushort_as_half(static_cast<uint16_t>(v & 0xFFFFu)));
                z0 = __half2float(__ushort_as_half(static_cast<uint16_t>(v >> 16)));
              }
              if (n + 1 < N) {
                const uint32_t v = reinterpret_cast<const uint32_t*>(scales)[static_cast<int64_t>(n + 1) * nscale + grp];
                s1 = __half2float(__ushort_as_half(static_cast<uint16_t>(v & 0xFFFFu)));
                z1 = __half2float(__ushort_as_half(static_cast<uint16_t>(v >> 16)));
              }
              acc[j][0] = fmaf(s0, fmaf(-z0, ssum[0], part[j][0]), acc[j][0]);
              acc[j][1] = fmaf(s1, fmaf(-z1, ssum[0], part[j][1]), acc[j][1]);
              acc[j][2] = fmaf(s0, fmaf(-z0, ssum[2], part[j][2]), acc[j][2]);
              acc[j][3] = fmaf(s1, fmaf(-z1, ssum[2], part[j][3]), acc[j][3]);
            }
          }
        }
      }
    }

    // ---- reduce the warps' partial sums and write y ---------------------------------
    __syncthreads();  // every warp is done reading xs
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
