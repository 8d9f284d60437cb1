// quantize.cuh -- activation quantiser (MXFP4 with OCP / UOS block scales and an
// optional fixed 128-point Hadamard rotation; FP8 E4M3 with a static per-tensor
// scale) and the offline MXFP4 weight packer.
//
// MXFP4: 32 consecutive K elements share one E8M0 power-of-two scale; elements are
// E2M1.  [MXAttention: Data-Free Optimal Scaling and Pre-Normalization Quantization
// for MXFP4 Attention -- "What it actually does"; AMD Quark ... FLUX.1-dev MXFP4 --
// "MXFP4とは何か"]  The scale rule is either stock OCP (e = floor(log2 amax) - 2) or
// the UOS boundary Qmax = 7.25 (smallest e with amax / 2^e <= 7.25).  Dynamic MXFP4
// activations (W4A4) and static FP8 E4M3 activations (W4A8) follow [AMD Quark adds
// native W4A8 ... Wan2.2 -- "MXFP4 formats and precision levels"]; the rotation is
// the fixed, parameter-free Hadamard of the same page ("Fixed rotation selector").
//
// The pass is bound by HBM bandwidth (2 bytes in, 0.53 bytes out per element), so the
// design is about bytes in flight: each thread issues eight 16-byte loads before it
// computes anything, loads are fully coalesced (a warp reads 2 rows x 256 bytes per
// instruction), and the block scales of a 128 x 128 tile are assembled in shared
// memory and leave as one 512-byte atom.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace mxq {

constexpr int kQuantThreads = 256;   // 8 warps; a CTA owns 128 rows x 128 K columns
constexpr uint32_t kInvSqrt128Bits = 0x3DB504F3u;  // fl32(1 / sqrt(128))

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Two non-negative floats -> one byte of two E2M1 magnitudes (round to nearest even,
// saturating at 6): `lo` in bits 0-3, `hi` in bits 4-7.
__device__ __forceinline__ uint32_t e2m1x2_magnitude(float lo, float hi) {
  uint32_t out;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
      : "=r"(out)
      : "f"(hi), "f"(lo));
  return out;
}

// Two non-negative floats -> two E4M3 magnitudes (RNE, saturating at 448): `lo` in
// bits 0-7, `hi` in bits 8-15.
__device__ __forceinline__ uint32_t e4m3x2_magnitude(float lo, float hi) {
  uint32_t out;
  asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tcvt.u32.u16 %0, t;\n\t}"
      : "=r"(out)
      : "f"(hi), "f"(lo));
  return out;
}

__device__ __forceinline__ void bf16x8_to_float(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    f[2 * j] = __uint_as_float(w[j] << 16);
    f[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
}

// Block exponent from the block's absolute maximum (integer arithmetic on the FP32
// bit pattern, no log2).  OCP: floor(log2 amax) - 2.  UOS: one more when the
// significand exceeds 1.8125 = 7.25 / 4, i.e. amax > 7.25 * 2^(OCP exponent);
// biased exponents 0 and 1 give an OCP exponent below -127, which clamps to -127
// where amax <= 7.25 * 2^-127 always holds, so they never bump.
template <bool kUOS>
__device__ __forceinline__ int block_exponent(float amax) {
  const uint32_t bits = __float_as_uint(amax);
  const int biased = static_cast<int>(bits >> 23);  // amax >= 0
  int e = biased - 127 - 2;
  if (kUOS && biased >= 2 && (bits & 0x7FFFFFu) > 0x680000u) e += 1;
  e = e < -127 ? -127 : e;
  e = e > 126 ? 126 : e;  // only non-finite input (out of contract) reaches 126+
  return e;
}

// 128-point normalised Sylvester-Hadamard across the 16 lanes of a half-warp, each
// lane holding 8 consecutive elements (element j = 8 * (lane % 16) + i).  Butterfly
// strides 1, 2, 4 inside the thread, then 8, 16, 32, 64 across lanes (xor 1, 2, 4, 8),
// each stage (t_i, t_i+h) <- (t_i + t_i+h, t_i - t_i+h) in FP32 round-to-nearest, then
// one multiply by fl32(1/sqrt(128)) -- the exact order of the definition.
__device__ __forceinline__ void fwht128_halfwarp(float (&f)[8], int l16) {
#pragma unroll
  for (int h = 1; h < 8; h *= 2) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i & h) continue;
      const float a = f[i], b = f[i + h];
      f[i] = __fadd_rn(a, b);
      f[i + h] = __fsub_rn(a, b);
    }
  }
#pragma unroll
  for (int bit = 0; bit < 4; ++bit) {
    const bool upper = (l16 >> bit) & 1;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float p = __shfl_xor_sync(0xffffffffu, f[i], 1 << bit);
      f[i] = upper ? __fsub_rn(p, f[i]) : __fadd_rn(f[i], p);
    }
  }
  const float c = __uint_as_float(kInvSqrt128Bits);
#pragma unroll
  for (int i = 0; i < 8; ++i) f[i] = __fmul_rn(f[i], c);
}

// One CTA quantises rows [128*by, +128) x K columns [128*bx, +128) of x[rows][ld]:
// codes [rows][K/2], and the CTA's 512-byte scale atom (rows beyond `rows`, and
// blocks beyond K, are written as 0x00 padding).
template <bool kHadamard, bool kUOS>
__device__ __forceinline__ void quantize_mxfp4_tile(const uint16_t* __restrict__ x, int64_t rows, int64_t K,
                                                    int64_t ld, uint8_t* __restrict__ codes,
                                                    uint8_t* __restrict__ sf) {
  __shared__ __align__(16) uint32_t atom[128];  // u32 (r%32)*4 + r/32 holds blocks 0..3 of row r
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int half = lane >> 4, l16 = lane & 15;
  const int64_t row0 = static_cast<int64_t>(blockIdx.y) * 128;
  const int64_t k = static_cast<int64_t>(blockIdx.x) * 128 + 8 * l16;
  const bool k_ok = k < K;  // K % 32 == 0: a 32-block is entirely in or out

  if (tid < 128) atom[tid] = 0u;

  uint4 v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t row = row0 + 16 * warp + 2 * i + half;
    v[i] = (row < rows && k_ok) ? ld_stream_v4(x + row * ld + k) : make_uint4(0, 0, 0, 0);
  }
  __syncthreads();  // atom zeroed

#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = 16 * warp + 2 * i + half;  // row within the tile
    const int64_t row = row0 + r;
    float f[8];
    bf16x8_to_float(v[i], f);
    if (kHadamard) fwht128_halfwarp(f, l16);

    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(f[j]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const int e = block_exponent<kUOS>(amax);
    const float inv_scale = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);  // 2^-e, exact

    uint32_t packed = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a0 = f[2 * j], a1 = f[2 * j + 1];
      uint32_t byte = e2m1x2_magnitude(__fmul_rn(fabsf(a0), inv_scale), __fmul_rn(fabsf(a1), inv_scale));
      byte |= ((__float_as_uint(a0) >> 31) << 3) | ((__float_as_uint(a1) >> 31) << 7);
      packed |= byte << (8 * j);
    }
    if (row < rows && k_ok) *reinterpret_cast<uint32_t*>(codes + row * (K / 2) + k / 2) = packed;

    // Scale bytes of this row's four blocks sit in lanes 0, 4, 8, 12 of the half-warp.
    const uint32_t sbyte = (row < rows && k_ok) ? static_cast<uint32_t>(e + 127) : 0u;
    const int base = lane & 16;
    const uint32_t b0 = __shfl_sync(0xffffffffu, sbyte, base + 0);
    const uint32_t b1 = __shfl_sync(0xffffffffu, sbyte, base + 4);
    const uint32_t b2 = __shfl_sync(0xffffffffu, sbyte, base + 8);
    const uint32_t b3 = __shfl_sync(0xffffffffu, sbyte, base + 12);
    if (l16 == 0) atom[(r & 31) * 4 + (r >> 5)] = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
  }
  __syncthreads();
  if (tid < 32) {
    const int64_t atoms_per_row_tile = (K + 127) / 128;
    const int64_t idx = static_cast<int64_t>(blockIdx.y) * atoms_per_row_tile + blockIdx.x;
    const uint4 w = reinterpret_cast<const uint4*>(atom)[tid];
    reinterpret_cast<uint4*>(sf + idx * 512)[tid] = w;
  }
}

template <bool kHadamard, bool kUOS>
__global__ void __launch_bounds__(kQuantThreads) quantize_act_mxfp4_kernel(
    const uint16_t* __restrict__ x, int64_t M, int64_t K, int64_t ldx, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ sf) {
  quantize_mxfp4_tile<kHadamard, kUOS>(x, M, K, ldx, codes, sf);
}

// The offline weight packer: the same block arithmetic on W[N][K] rows.
template <bool kHadamard, bool kUOS>
__global__ void __launch_bounds__(kQuantThreads) pack_weight_mxfp4_kernel(
    const uint16_t* __restrict__ w, int64_t N, int64_t K, int64_t ldw, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ sf) {
  quantize_mxfp4_tile<kHadamard, kUOS>(w, N, K, ldw, codes, sf);
}

// Static FP8: q = E4M3_RNE_satfinite(fl32(x * inv_scale)), sign bit kept.  Each thread
// converts 8-element chunks (16 bytes in, 8 bytes out) in a grid-stride loop.
__global__ void __launch_bounds__(kQuantThreads) quantize_act_fp8_kernel(const uint16_t* __restrict__ x, int64_t M,
                                                                          int64_t K, int64_t ldx, float inv_scale,
                                                                          uint8_t* __restrict__ q) {
  const int64_t chunks_per_row = K / 8;
  const int64_t total = M * chunks_per_row;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c < total; c += stride) {
    const int64_t row = c / chunks_per_row;
    const int64_t k = (c - row * chunks_per_row) * 8;
    float f[8];
    bf16x8_to_float(ld_stream_v4(x + row * ldx + k), f);
    uint32_t w[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      uint32_t out = 0;
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        const float a0 = __fmul_rn(f[4 * j + 2 * p], inv_scale);
        const float a1 = __fmul_rn(f[4 * j + 2 * p + 1], inv_scale);
        uint32_t two = e4m3x2_magnitude(fabsf(a0), fabsf(a1));
        two |= ((__float_as_uint(a0) >> 31) << 7) | ((__float_as_uint(a1) >> 31) << 15);
        out |= two << (16 * p);
      }
      w[j] = out;
    }
    *reinterpret_cast<uint2*>(q + row * K + k) = make_uint2(w[0], w[1]);
  }
}

}  // namespace mxq
