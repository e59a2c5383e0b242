// prep.cuh -- preparation kernels of the tensor-core path: the f16, pair-permuted copy of
// the activations that the tensor-core kernel reads (prep_x16_kernel), and, with the
// low-rank branch, that copy together with u = x A^T (prep_lora_kernel, its K-slice
// partial sums, then lora_finalize_kernel).  The k order of the copy is the one the
// tensor-core kernel's dequantizers produce (gemm_tc.cuh).
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"

namespace tgemm {

// ---- activation preparation ---------------------------------------------------------

// One 16-element group: bf16 -> f16 with the pair permutation of format FMT.
template <int FMT>
__device__ __forceinline__ void x16_group(const uint4& v0, const uint4& v1, uint4* dst) {
  const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
  float f[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
  uint32_t o[8];
  if (FMT == 0) {
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = pack_f16x2(f[i], f[i + 8]);
  } else {
#pragma unroll
    for (int e8 = 0; e8 < 2; ++e8)
#pragma unroll
      for (int i = 0; i < 4; ++i) o[4 * e8 + i] = pack_f16x2(f[8 * e8 + i], f[8 * e8 + i + 4]);
  }
  dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
  dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
}

// bf16 [M][K] -> f16 [M][K] with the pair permutation the dequantizers produce
// (FMT 0: within each 16-group, position 2i <- i, 2i+1 <- i+8; FMT 1: within each
// 8-group, 2i <- i, 2i+1 <- i+4).  Up to four 16-element groups per thread per round.  It also zeroes the
// matmul's `ncnt` split-tile arrival counters, which the matmul kernel that follows on
// the stream expects at zero.
template <int FMT>
__global__ void __launch_bounds__(256) prep_x16_kernel(const uint16_t* __restrict__ x,
                                                       uint16_t* __restrict__ x16,
                                                       int64_t ngroups, int* __restrict__ cnt,
                                                       int ncnt) {
  pdl_trigger_and_wait();
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t first = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (int64_t i = first; i < ncnt; i += nthreads) cnt[i] = 0;
  const uint4* src = reinterpret_cast<const uint4*>(x);
  uint4* dst = reinterpret_cast<uint4*>(x16);
  // up to four groups per thread per round, all loads issued before any conversion
  for (int64_t base = first; base < ngroups; base += 4 * nthreads) {
    uint4 v[4][2];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t g = base + j * nthreads;
      if (g < ngroups) {
        v[j][0] = __ldg(src + 2 * g);
        v[j][1] = __ldg(src + 2 * g + 1);
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t g = base + j * nthreads;
      if (g < ngroups) x16_group<FMT>(v[j][0], v[j][1], dst + 2 * g);
    }
  }
}

// Activation prep and the branch's first product in one pass over x (tensor-core path
// with the low-rank branch).  CTA (token block of kPlTok, K slice of kLoraKc):
//   - writes the f16, pair-permuted copy of its x tile (as prep_x16_kernel);
//   - keeps the bf16 tile in shared memory and multiplies it with the matching slice
//     of A, 64 columns of u at a time (ldmatrix + mma.sync, f32 accumulation);
//   - stores the slice's partial sums in part[slice][m][col] (f32, `rpad` columns).
// lora_finalize_kernel then adds the slices in order.  Also zeroes `ncnt` counters.
constexpr int kLoraKc = 512;      // K slice of the branch's partial sums
constexpr int kPlTok = 64;
constexpr int kPlPitch = kLoraKc + 8;  // bf16 elements per shared row (16-byte rows, no ldmatrix conflicts)
constexpr int kPlSmemBytes = 2 * kPlTok * kPlPitch * 2;

template <int FMT>
__global__ void __launch_bounds__(256) prep_lora_kernel(const uint16_t* __restrict__ x,
                                                        uint16_t* __restrict__ x16,
                                                        const uint16_t* __restrict__ a, int M,
                                                        int K, int r, int rpad,
                                                        float* __restrict__ part,
                                                        int* __restrict__ cnt, int ncnt,
                                                        int a_vec) {
  static_assert((kPlPitch * 2) % 16 == 0, "pitch");
  extern __shared__ __align__(16) uint16_t pl_smem[];
  uint16_t* xs = pl_smem;                     // [kPlTok][kPlPitch] bf16 x tile
  uint16_t* as = pl_smem + kPlTok * kPlPitch;  // [64][kPlPitch] bf16 rows of A
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int k0 = blockIdx.y * kLoraKc;
  // Columns [c0, c0 + 64) of A's K slice -> `as` by cp.async (A 16-byte aligned): 64 rows x
  // 32 pieces of 16 bytes, zeros past r and K.  The first chunk is a weight read and goes
  // out before the dependency wait, so its trip to memory overlaps the kernels ahead.
  auto a_async = [&](int c0) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int pi = tid + 256 * j;  // piece: row pi / 64, 8 elements at (pi % 64) * 8
      const int row = pi >> 6, e = (pi & 63) * 8;
      const int col = c0 + row, k = k0 + e;
      const bool in = col < r && k < K;  // K is a multiple of 128: a piece is all in or out
      cp_async16(smem_u32(as + row * kPlPitch + e), in ? a + static_cast<int64_t>(col) * K + k : a, in ? 16u : 0u);
    }
  };
  pdl_trigger();
  if (a_vec) a_async(0);
  pdl_wait();
  {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * gridDim.y * blockDim.x;
    for (int64_t i = (static_cast<int64_t>(blockIdx.y) * gridDim.x + blockIdx.x) * blockDim.x + tid;
         i < ncnt; i += stride)
      cnt[i] = 0;
  }
  const int m0 = blockIdx.x * kPlTok;
  // x tile: 64 rows x 32 groups of 16 (thread -> group, a warp covers one row); each
  // thread's 8 groups are loaded 4 at a time before any is stored
#pragma unroll 1
  for (int half = 0; half < 2; ++half) {
    uint4 v[4][2];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gi = tid + 256 * (4 * half + j);
      const int row = gi >> 5, g = gi & 31;
      const int m = m0 + row, k = k0 + 16 * g;
      v[j][0] = make_uint4(0, 0, 0, 0);
      v[j][1] = v[j][0];
      if (m < M && k < K) {
        const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(m) * K + k);
        v[j][0] = __ldg(src);
        v[j][1] = __ldg(src + 1);
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gi = tid + 256 * (4 * half + j);
      const int row = gi >> 5, g = gi & 31;
      const int m = m0 + row, k = k0 + 16 * g;
      uint4* sdst = reinterpret_cast<uint4*>(xs + row * kPlPitch + 16 * g);
      sdst[0] = v[j][0];
      sdst[1] = v[j][1];
      if (m < M && k < K)
        x16_group<FMT>(v[j][0], v[j][1], reinterpret_cast<uint4*>(x16 + static_cast<int64_t>(m) * K + k));
    }
  }
  const int mt = warp & 3;   // 16-token row block of the warp
  const int nh = warp >> 2;  // 32-column half of the 64-column chunk
  const int ksteps = min(kLoraKc, K - k0) / 16;
  for (int c0 = 0; c0 < rpad; c0 += 64) {
    __syncthreads();  // x tile written (first pass) / previous A chunk consumed
    if (a_vec) {
      if (c0 > 0) a_async(c0);
      cp_async_wait_all();
    }
#pragma unroll 1
    for (int half = 0; half < (a_vec ? 0 : 2); ++half) {
      uint4 v[4][2];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int gi = tid + 256 * (4 * half + j);
        const int row = gi >> 5, g = gi & 31;
        const int col = c0 + row, k = k0 + 16 * g;
        v[j][0] = make_uint4(0, 0, 0, 0);
        v[j][1] = v[j][0];
        if (col < r && k < K) {  // A only 4-byte aligned
          const uint32_t* src = reinterpret_cast<const uint32_t*>(a + static_cast<int64_t>(col) * K + k);
          v[j][0] = make_uint4(__ldg(src), __ldg(src + 1), __ldg(src + 2), __ldg(src + 3));
          v[j][1] = make_uint4(__ldg(src + 4), __ldg(src + 5), __ldg(src + 6), __ldg(src + 7));
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int gi = tid + 256 * (4 * half + j);
        const int row = gi >> 5, g = gi & 31;
        uint4* sdst = reinterpret_cast<uint4*>(as + row * kPlPitch + 16 * g);
        sdst[0] = v[j][0];
        sdst[1] = v[j][1];
      }
    }
    __syncthreads();
    float acc[4][4];
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[t][e] = 0.f;
    // ldmatrix row addresses: A (x) matrices (m 0-7 | 8-15) x (k 0-7 | 8-15);
    // B (rows of A) matrices (n 0-7, k 0-7), (n 0-7, k 8-15), (n 8-15, k 0-7), (n 8-15, k 8-15)
    const int mi = lane >> 3, rr = lane & 7;
    const uint32_t xa = smem_u32(xs + (mt * 16 + (mi & 1) * 8 + rr) * kPlPitch + (mi >> 1) * 8);
    const uint32_t ba = smem_u32(as + (nh * 32 + (mi >> 1) * 8 + rr) * kPlPitch + (mi & 1) * 8);
    for (int ks = 0; ks < ksteps; ++ks) {
      uint32_t af[4], b01[4], b23[4];
      ldmatrix_x4(xa + ks * 32, af);
      ldmatrix_x4(ba + ks * 32, b01);
      ldmatrix_x4(ba + 16 * kPlPitch * 2 + ks * 32, b23);
      mma_bf16_16816(acc[0], af, b01[0], b01[1]);
      mma_bf16_16816(acc[1], af, b01[2], b01[3]);
      mma_bf16_16816(acc[2], af, b23[0], b23[1]);
      mma_bf16_16816(acc[3], af, b23[2], b23[3]);
    }
    // fragment (t, e): token mt*16 + lane/4 (+8 for e >= 2), column nh*32 + 8t + 2(lane%4) + (e&1)
    const int g4 = lane >> 2, c4 = lane & 3;
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int m = m0 + mt * 16 + g4 + 8 * h;
        if (m >= M) continue;
        const int col = c0 + nh * 32 + 8 * t + 2 * c4;
        float2* dst = reinterpret_cast<float2*>(part + (static_cast<int64_t>(blockIdx.y) * M + m) * rpad + col);
        *dst = make_float2(acc[t][2 * h], acc[t][2 * h + 1]);
      }
  }
}

// Tensor-core path, second step of u = x A^T: sums prep_lora_kernel's K-slice partials in a
// fixed order (no atomics) and writes the concatenation ucat [M][wcat] =
// [bf16(u) pad R | bf16(u - bf16(u)) pad R | 0], the branch stages' activations.
__global__ void __launch_bounds__(256) lora_finalize_kernel(const float* __restrict__ part,
                                                            int slices, int M, int r, int rpad,
                                                            int R, int wcat,
                                                            uint16_t* __restrict__ ucat) {
  pdl_trigger_and_wait();
  const int64_t total = static_cast<int64_t>(M) * wcat;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int64_t m = i / wcat;
    const int j = static_cast<int>(i % wcat);
    uint16_t out = 0;
    if (j < 2 * R) {
      const int col = j < R ? j : j - R;
      if (col < r) {
        float v = 0.f;
        for (int sl = 0; sl < slices; ++sl) v += part[(sl * static_cast<int64_t>(M) + m) * rpad + col];
        const __nv_bfloat16 h = __float2bfloat16_rn(v);
        out = j < R ? __bfloat16_as_ushort(h)
                    : __bfloat16_as_ushort(__float2bfloat16_rn(v - __bfloat162float(h)));
      }
    }
    ucat[i] = out;
  }
}

}  // namespace tgemm
