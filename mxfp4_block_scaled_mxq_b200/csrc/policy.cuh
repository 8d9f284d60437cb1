// policy.cuh -- the measurement behind the per-layer precision selection: the output
// SQNR of a quantised layer against its BF16 reference,
//   SQNR = 10 log10( sum ref^2 / sum (y - ref)^2 )  dB,
// whose sums are accumulated here in FP64 on the device.
// [AMD Quark adds native W4A8 mixed-precision for Wan2.2 video generation on MI350 --
//  "Block-level SQNR calibration": whole-block output SQNR against BF16 decides between
//  plain W4A4, W4A8 promotion, transform-enabled W4A4 and BF16 fallback]
#pragma once

#include <cstdint>

namespace mxq {

constexpr int kSqnrThreads = 256;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// acc[0] += sum ref^2, acc[1] += sum (y - ref)^2 over the M x N values (row strides ldy,
// ldr elements).  Each thread takes 8-column chunks (16-byte loads when the chunk is
// whole), grid-stride; per-thread FP64 sums, then warp shuffles, shared memory and one
// FP64 atomicAdd pair per CTA.  BF16 squares and differences are exact in FP64, so only
// the order of the FP64 additions varies from run to run.
__global__ void __launch_bounds__(kSqnrThreads) sqnr_sums_kernel(const uint16_t* __restrict__ y, int64_t ldy,
                                                                  const uint16_t* __restrict__ ref, int64_t ldr,
                                                                  int64_t M, int64_t N, double* __restrict__ acc) {
  const int64_t chunks_per_row = (N + 7) / 8;
  const int64_t total = M * chunks_per_row;
  double s = 0.0, e = 0.0;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / chunks_per_row;
    const int64_t c0 = (i - r * chunks_per_row) * 8;
    const uint16_t* yp = y + r * ldy + c0;
    const uint16_t* rp = ref + r * ldr + c0;
    if (c0 + 8 <= N) {
      const uint4 a = *reinterpret_cast<const uint4*>(yp);
      const uint4 b = *reinterpret_cast<const uint4*>(rp);
      const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const double r0 = bf16_lo(bw[j]), r1 = bf16_hi(bw[j]);
        const double d0 = static_cast<double>(bf16_lo(aw[j])) - r0;
        const double d1 = static_cast<double>(bf16_hi(aw[j])) - r1;
        s += r0 * r0 + r1 * r1;
        e += d0 * d0 + d1 * d1;
      }
    } else {
      for (int64_t c = 0; c < N - c0; ++c) {
        const double rv = __uint_as_float(static_cast<uint32_t>(rp[c]) << 16);
        const double d = static_cast<double>(__uint_as_float(static_cast<uint32_t>(yp[c]) << 16)) - rv;
        s += rv * rv;
        e += d * d;
      }
    }
  }
#pragma unroll
  for (int sh = 16; sh > 0; sh >>= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, sh);
    e += __shfl_xor_sync(0xffffffffu, e, sh);
  }
  __shared__ double part[2][kSqnrThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    part[0][warp] = s;
    part[1][warp] = e;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double ts = 0.0, te = 0.0;
    for (int w = 0; w < kSqnrThreads / 32; ++w) {
      ts += part[0][w];
      te += part[1][w];
    }
    atomicAdd(acc, ts);
    atomicAdd(acc + 1, te);
  }
}

}  // namespace mxq
