// mma_rate.cuh -- measurement hook: the issue rate of back-to-back tcgen05 MMAs of one
// shape, and of TMEM loads, on every SM at once.  It backs two design decisions with
// numbers: how an M = 128 MMA's cost depends on N (small-M tiles of 8..16 tokens), and
// what 8-bit integer MMAs (kind::i8) and a per-stage accumulator drain (tcgen05.ld) cost.
// Operands are zero-filled shared memory (and, for the TMEM-A form, whatever TMEM holds):
// the values do not affect timing, and nothing reads the results.
#pragma once

#include "common.cuh"

namespace tgemm {

// Instruction descriptor, kind::i8, dense, s32 accumulate, signed 8-bit A and B, K-major.
__host__ __device__ constexpr uint32_t make_idesc_i8(uint32_t M, uint32_t N) {
  return (2u << 4)           // D format s32
         | (1u << 7)         // A signed 8-bit
         | (1u << 10)        // B signed 8-bit
         | ((N >> 3) << 17)  // N / 8
         | ((M >> 4) << 24); // M / 16
}

__device__ __forceinline__ void mma_i8_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

constexpr int kRateA = 128 * 128;                // A: 128 rows x 128 bytes
constexpr int kRateB = 256 * 128;                // B: up to 256 rows x 128 bytes
// large enough that only one CTA fits on an SM (each allocates all 512 TMEM columns)
constexpr int kRateSmem = 116 * 1024;

// mode 0: kind::f16 (f16 x f16), A from shared memory; 1: kind::f16, A from TMEM;
// 2: kind::i8 (s8 x s8), A from shared memory; 3: tcgen05.ld of 16 columns x 32 lanes per
// warp (4 warps), each followed by its wait.  M = 128, N = n, K = 16 (f16) or 32 (i8).
// mode 4: warp-level mma.sync m16n8k16 bf16 -> f32; 5: mma.sync m16n8k32 s8 -> s32; each
// of the 4 warps runs 8 independent accumulator chains (one warp per SM sub-partition).
// out[cta] = cycles for `iters` operations (modes 4, 5: `iters` mma per warp).
__global__ void __launch_bounds__(128, 1) mma_rate_kernel(int mode, int n, int iters,
                                                          unsigned long long* out) {
  extern __shared__ uint8_t rate_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(rate_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5;
  for (int i = tid; i < (kRateA + kRateB) / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(sm)[i] = make_uint4(0u, 0u, 0u, 0u);
  const uint32_t sa = smem_u32(sm), sbx = sa + kRateA;
  const uint32_t bar = sa + kRateA + kRateB;
  uint32_t* slot = reinterpret_cast<uint32_t*>(sm + kRateA + kRateB + 8);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(sm + kRateA + kRateB + 16);
  if (tid == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(slot), 512);
    tmem_relinquish();
  }
  fence_proxy_async_smem();  // the zero fill is read by the tensor core (async proxy)
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  if (mode <= 2) {
    if (tid == 0) {
      const uint32_t idesc = mode == 2 ? make_idesc_i8(128u, static_cast<uint32_t>(n))
                                       : make_idesc_f16(0u, 128u, static_cast<uint32_t>(n));
      const uint64_t adesc = smem_desc_sw128(sa), bdesc = smem_desc_sw128(sbx);
      const unsigned long long t0 = clock64();
      for (int i = 0; i < iters; ++i) {
        const uint32_t k = static_cast<uint32_t>(i & 3);  // 32-byte K step in the 128-byte row
        if (mode == 0)
          mma_f16_ss(tmem, adesc + 2u * k, bdesc + 2u * k, idesc, i > 0 ? 1u : 0u);
        else if (mode == 1)
          mma_f16_ts(tmem, tmem + 256u + 8u * k, bdesc + 2u * k, idesc, i > 0 ? 1u : 0u);
        else
          mma_i8_ss(tmem, adesc + 2u * k, bdesc + 2u * k, idesc, i > 0 ? 1u : 0u);
      }
      mma_commit(bar);
      mbar_wait_drain(bar, 0u);
      out[blockIdx.x] = clock64() - t0;
    }
  } else if (mode >= 4) {
    float facc[8][4];
    int iacc[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        facc[j][e] = 0.f;
        iacc[j][e] = 0;
      }
    const uint32_t a[4] = {static_cast<uint32_t>(tid), 1u, 2u, 3u};
    const unsigned long long t0 = clock64();
    if (mode == 4) {
      for (int i = 0; i < iters; i += 8) {
#pragma unroll
        for (int j = 0; j < 8; ++j) mma_bf16_16816(facc[j], a, static_cast<uint32_t>(i), static_cast<uint32_t>(j));
      }
    } else {
      for (int i = 0; i < iters; i += 8) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          asm volatile(
              "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
              "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
              : "+r"(iacc[j][0]), "+r"(iacc[j][1]), "+r"(iacc[j][2]), "+r"(iacc[j][3])
              : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(static_cast<uint32_t>(i)),
                "r"(static_cast<uint32_t>(j)));
      }
    }
    float keep = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) keep += facc[j][0] + static_cast<float>(iacc[j][0]);
    const unsigned long long t1 = clock64();
    if (keep == 12345.f) out[blockIdx.x] = 0;  // keeps the products
    if (tid == 0) out[blockIdx.x] = t1 - t0;
  } else {
    // each warp reads its TMEM lane quarter, 16 columns at a time
    const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    uint32_t acc = 0u;
    const unsigned long long t0 = clock64();
    for (int i = 0; i < iters; ++i) {
      uint32_t v[16];
      tmem_ld_32x32b_x16(taddr + 16u * static_cast<uint32_t>(i & 15), v);
      tmem_wait_ld();
      acc ^= v[i & 15];
    }
    const unsigned long long t1 = clock64();
    if ((tid & 31) == 0 && acc == 0x12345678u) out[blockIdx.x] = 0;  // keeps the loads
    if (tid == 0) out[blockIdx.x] = t1 - t0;
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Modes 6-8: the steady state of an 8-bit-activation design in which each 128-k block's
// int32 products (M = 128 weight rows x N = 256 tokens, kind::i8, four K = 32 MMAs) are
// drained from TMEM by 16 epilogue warps -- 4 per TMEM lane quarter, 64 token columns each,
// read 16 at a time -- converted to f32 and added, times a per-row scale, into running sums held in
// registers, while the next block's MMAs fill the other of two 256-column accumulators.
//   mode 6: MMAs and drains together, int -> float by cvt;
//   mode 7: the drains alone (no MMA; the same columns read each block), cvt;
//   mode 8: as mode 6, int -> float by the exponent trick (i + 0x4B400000 read as a float
//           is 12582912 + i for |i| < 2^22);
//   mode 9: as mode 8 with the subtraction and the multiply-add on packed f32x2 pairs;
//   mode 10: as mode 6 with the multiply-add on packed f32x2 pairs.
// out[cta] = cycles for `iters` blocks, from the MMA-issuing thread (modes 6, 8: the last
// block's drain included) or from epilogue warp 0 (mode 7).
constexpr int kDrainWarps = 16;
constexpr int kDrainThreads = (kDrainWarps + 1) * 32;
__global__ void __launch_bounds__(kDrainThreads, 1) drain_rate_kernel(int mode, int iters,
                                                                   unsigned long long* out) {
  extern __shared__ uint8_t rate_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(rate_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < (kRateA + kRateB) / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(sm)[i] = make_uint4(0u, 0u, 0u, 0u);
  const uint32_t sa = smem_u32(sm), sbx = sa + kRateA;
  const uint32_t full0 = sa + kRateA + kRateB, empty0 = full0 + 16;  // two barriers each, 8 bytes apart
  uint32_t* slot = reinterpret_cast<uint32_t*>(sm + kRateA + kRateB + 32);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(sm + kRateA + kRateB + 40);
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, kDrainWarps);
    }
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(slot), 512);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  const bool with_mma = mode != 7;
  if (warp == kDrainWarps) {
    if (lane == 0 && with_mma) {
      const uint32_t idesc = make_idesc_i8(128u, 256u);
      const uint64_t adesc = smem_desc_sw128(sa), bdesc = smem_desc_sw128(sbx);
      const unsigned long long t0 = clock64();
      bool ok = true;
      for (int b = 0; b < iters && ok; ++b) {
        const int p = b & 1;
        if (b >= 2) ok = mbar_wait(empty0 + 8 * p, static_cast<uint32_t>(((b >> 1) - 1) & 1), abort_flag);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_i8_ss(tmem + 256u * p, adesc + 2u * k, bdesc + 2u * k, idesc, k > 0 ? 1u : 0u);
        mma_commit(full0 + 8 * p);
      }
      if (ok) {
        const int b = iters - 1;
        ok = mbar_wait(empty0 + 8 * (b & 1), static_cast<uint32_t>((b >> 1) & 1), abort_flag);
      }
      out[blockIdx.x] = ok ? clock64() - t0 : 0ull;
    }
  } else {
    const int lq = warp & 3, cs = warp >> 2;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(lq * 32) << 16) + 64u * cs;
    const float d = 1.0f + 1e-3f * lane;
    float acc[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) acc[i] = 0.f;
    const unsigned long long t0 = clock64();
    for (int b = 0; b < iters; ++b) {
      const int p = b & 1;
      if (with_mma) {
        if (!mbar_wait(full0 + 8 * p, static_cast<uint32_t>((b >> 1) & 1), abort_flag)) break;
        tc_fence_after();
      }
#pragma unroll
      for (int h = 0; h < 4; ++h) {  // 16 columns at a time (registers: 64 sums + 16 loaded)
        uint32_t v[16];
        tmem_ld_32x32b_x16(taddr + 256u * p + 16u * h, v);
        tmem_wait_ld();
        if (h == 3 && with_mma) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(empty0 + 8 * p);
        }
        if (mode >= 9) {
          // packed f32x2 arithmetic, two columns per instruction
#pragma unroll
          for (int i = 0; i < 16; i += 2) {
            float f0, f1;
            if (mode == 9) {
              f0 = __uint_as_float(v[i] + 0x4B400000u);
              f1 = __uint_as_float(v[i + 1] + 0x4B400000u);
            } else {
              f0 = static_cast<float>(static_cast<int>(v[i]));
              f1 = static_cast<float>(static_cast<int>(v[i + 1]));
            }
            unsigned long long fv = (static_cast<unsigned long long>(__float_as_uint(f1)) << 32) | __float_as_uint(f0);
            if (mode == 9) {
              const unsigned long long mc = 0xCB400000CB400000ull;  // (-12582912, -12582912)
              asm("add.rn.f32x2 %0, %1, %2;" : "=l"(fv) : "l"(fv), "l"(mc));
            }
            const unsigned long long dd = (static_cast<unsigned long long>(__float_as_uint(d)) << 32) | __float_as_uint(d);
            unsigned long long ac = (static_cast<unsigned long long>(__float_as_uint(acc[16 * h + i + 1])) << 32) |
                                    __float_as_uint(acc[16 * h + i]);
            asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(ac) : "l"(dd), "l"(fv));
            acc[16 * h + i] = __uint_as_float(static_cast<uint32_t>(ac));
            acc[16 * h + i + 1] = __uint_as_float(static_cast<uint32_t>(ac >> 32));
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float f = mode == 8 ? __uint_as_float(v[i] + 0x4B400000u) - 12582912.f
                                      : static_cast<float>(static_cast<int>(v[i]));
            acc[16 * h + i] = fmaf(d, f, acc[16 * h + i]);
          }
        }
      }
    }
    const unsigned long long t1 = clock64();
    float keep = 0.f;
#pragma unroll
    for (int i = 0; i < 64; ++i) keep += acc[i];
    if (keep == 12345.f) out[blockIdx.x] = 1ull;  // keeps the sums
    if (mode == 7 && tid == 0) out[blockIdx.x] = t1 - t0;
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tgemm
