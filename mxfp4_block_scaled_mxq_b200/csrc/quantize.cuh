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
// The pass is bound by HBM bandwidth (2 bytes in, 0.53 bytes out per element) as long
// as it issues few enough instructions per element, so each thread owns 16
// consecutive elements (one 32-byte load; a warp reads 1 KB per instruction), the
// non-rotated path takes the block amax on packed BF16 pairs, a 32-element block
// spans two lanes (one shuffle), and each block's scale byte goes straight into the
// CTA's 512-byte scale atom in shared memory, which leaves as one coalesced write.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "ptx.cuh"

namespace mxq {

constexpr int kQuantThreads = 256;                 // 8 warps; a CTA owns 128 rows x 128 K columns
constexpr uint32_t kInvSqrt128Bits = 0x3DB504F3u;  // fl32(1 / sqrt(128))

// 16 consecutive BF16 values (32 bytes) of a streamed input: one 32-byte load where the
// address allows it, else two 16-byte loads (rows of a 16-byte-aligned slice, or a row
// stride that is an odd multiple of 8 elements).  The test is uniform across a warp
// whenever the rows share their alignment.
__device__ __forceinline__ void ld_stream_v8(const void* p, uint32_t (&w)[8]) {
  if ((reinterpret_cast<uintptr_t>(p) & 31u) == 0) {
    asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
                 : "l"(p));
  } else {
    asm volatile(
        "ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%8];\n\t"
        "ld.global.nc.L1::no_allocate.v4.u32 {%4,%5,%6,%7}, [%8+16];"
        : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
        : "l"(p));
  }
}

// Two floats -> one byte of two E2M1 codes (round to nearest even, saturating at 6):
// `lo` in bits 0-3, `hi` in bits 4-7.  The conversion keeps the sign bit of its input
// in bit 3 of each code, also for -0 and for negative values that round to zero
// (0x8) -- the sign rule of the format as defined here; the exhaustive BF16 parity
// tests check this against the oracle.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint32_t out;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
      : "=r"(out)
      : "f"(hi), "f"(lo));
  return out;
}

// Eight floats -> eight E2M1 codes in one word, element i in bits [4i, 4i + 4): the same
// conversion as e2m1x2 four times, the four bytes joined by one vector move.
__device__ __forceinline__ uint32_t e2m1x8(float v0, float v1, float v2, float v3, float v4, float v5, float v6,
                                           float v7) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
  return out;
}

// Two floats -> two E4M3 codes (RNE, saturating at 448, sign kept): `lo` in bits 0-7,
// `hi` in bits 8-15.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint32_t out;
  asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tcvt.u32.u16 %0, t;\n\t}"
      : "=r"(out)
      : "f"(hi), "f"(lo));
  return out;
}

// One byte of two E2M1 codes -> two BF16 values code * scale (scale a power of two:
// the product is exact in FP32, or overflows to Inf; BF16 holds it exactly): `lo`
// nibble in bits 0-15.
__device__ __forceinline__ uint32_t e2m1x2_to_bf16x2(uint32_t byte, float scale) {
  uint32_t h;
  asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(h) : "r"(byte));
  const float lo = __fmul_rn(__half2float(__ushort_as_half(static_cast<unsigned short>(h & 0xFFFFu))), scale);
  const float hi = __fmul_rn(__half2float(__ushort_as_half(static_cast<unsigned short>(h >> 16))), scale);
  uint32_t out;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(out) : "f"(hi), "f"(lo));
  return out;
}

// Two E4M3 codes (bits 0-7, 8-15) -> two BF16 values bf16_rne(fl32(q * scale)).
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t two, float scale) {
  uint32_t h;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(h) : "r"(two));
  const float lo = __fmul_rn(__half2float(__ushort_as_half(static_cast<unsigned short>(h & 0xFFFFu))), scale);
  const float hi = __fmul_rn(__half2float(__ushort_as_half(static_cast<unsigned short>(h >> 16))), scale);
  uint32_t out;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(out) : "f"(hi), "f"(lo));
  return out;
}

__device__ __forceinline__ void bf16x16_to_float(const uint32_t (&w)[8], float (&f)[16]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    f[2 * j] = __uint_as_float(w[j] << 16);
    f[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
}

// Largest |x| over 16 BF16 values held as 8 packed pairs, as FP32 bits (exact).
// Magnitudes are compared by the packed BF16 max of absolute values (its result's sign,
// the XOR of the operands' signs, is cleared at the end); non-negative BF16 patterns
// order like unsigned integers, which combines the two halves.
__device__ __forceinline__ uint32_t bf16x16_absmax(const uint32_t (&w)[8]) {
  uint32_t m = w[0];
#pragma unroll
  for (int j = 1; j < 8; ++j) asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(m) : "r"(w[j]));
  m &= 0x7FFF7FFFu;
  return max(m & 0xFFFFu, m >> 16) << 16;
}

// Block exponent from the block's absolute maximum (integer arithmetic on the FP32
// bit pattern, no log2).  OCP: floor(log2 amax) - 2.  UOS: one more when the
// significand exceeds 1.8125 = 7.25 / 4, i.e. amax > 7.25 * 2^(OCP exponent);
// biased exponents 0 and 1 give an OCP exponent below -127, which clamps to -127
// where amax <= 7.25 * 2^-127 always holds, so they never bump.  A non-finite amax
// (an FP32 overflow inside the rotation of finite BF16 inputs) satisfies neither
// rule for any e, and takes the largest exponent, 127.
template <bool kUOS>
__device__ __forceinline__ int block_exponent(uint32_t amax_bits) {
  const int biased = static_cast<int>(amax_bits >> 23);  // amax >= 0
  if (biased == 255) return 127;
  int e = biased - 127 - 2;
  if (kUOS && biased >= 2 && (amax_bits & 0x7FFFFFu) > 0x680000u) e += 1;
  return e < -127 ? -127 : e;  // a finite amax gives e <= 126
}

// 2^-e for e in [-127, 127]: a normal float down to 2^-126, the subnormal 2^-127 at e = 127.
__device__ __forceinline__ float exp2_neg(int e) {
  return e < 127 ? __uint_as_float(static_cast<uint32_t>(127 - e) << 23) : __uint_as_float(0x00400000u);
}

// 2^e for e in [-127, 127].
__device__ __forceinline__ float exp2_pos(int e) { return exp2_neg(-e); }

// What a quantiser tile produces.
enum TileOut : int {
  kOutCodes = 0,   // MXFP4 codes + the tile's 512-byte scale atom
  kOutQdq = 1,     // BF16(dequant(quant(x))): the quantise-dequantise emulation
  kOutAbsmax = 2,  // per-channel max |y| over the tile's rows (calibration statistic)
};

struct TileArgs {
  uint8_t* codes = nullptr;      // kOutCodes: [rows][K/2]
  uint8_t* sf = nullptr;         // kOutCodes: swizzled scale bytes
  uint16_t* qdq = nullptr;       // kOutQdq: BF16 [rows][ldq]
  int64_t ldq = 0;
  const float* chan = nullptr;   // kSmooth: per-channel multiplier applied after the rotation
  float* chan_amax = nullptr;    // kOutAbsmax: FP32 maxima, merged with atomicMax on the bits
};

// One CTA quantises rows [128*by, +128) x K columns [128*bx, +128) of x[rows][ld]
// without rotation: codes [rows][K/2] and the tile's 512-byte scale atom (rows beyond
// `rows` and blocks beyond K stay 0x00 padding).  Thread (warp w, lane l) owns, in iteration i, row
// 16w + 4i + l/8 and elements [16 * (l%8), +16) of the tile's 128 columns.
// kOut selects what is written (TileOut); kSmooth multiplies each value by the channel's
// factor o.chan[k] (one FP32 product) before the block maximum, as SmoothQuant does.
template <bool kUOS, int kOut = kOutCodes, bool kSmooth = false>
__device__ __forceinline__ void quantize_mxfp4_tile(const uint16_t* __restrict__ x, int64_t rows, int64_t K,
                                                    int64_t ld, const TileArgs& o) {
  constexpr bool kQdq = kOut == kOutQdq;
  __shared__ __align__(16) uint8_t atom[512];  // byte (r%32)*16 + (r/32)*4 + block; column maxima
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int l8 = lane & 7;
  const int64_t row0 = static_cast<int64_t>(blockIdx.y) * 128;
  const int64_t k = static_cast<int64_t>(blockIdx.x) * 128 + 16 * l8;
  const bool k_ok = k < K;  // K % 32 == 0: a 16-element chunk is entirely in or out

  reinterpret_cast<uint32_t*>(atom)[tid & 127] = 0u;

  uint32_t w[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t row = row0 + 16 * warp + 4 * i + (lane >> 3);
    if (row < rows && k_ok) {
      ld_stream_v8(x + row * ld + k, w[i]);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) w[i][j] = 0u;
    }
  }
  __syncthreads();  // atom zeroed

  if constexpr (kOut == kOutAbsmax) {
    // lanes l, l^8, l^16, l^24 of a warp own the same 16 columns (rows beyond `rows` are 0)
    uint32_t* cmax = reinterpret_cast<uint32_t*>(atom);  // 128 columns, FP32 bits
    float cm[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) cm[j] = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float f[16];
      bf16x16_to_float(w[i], f);
#pragma unroll
      for (int j = 0; j < 16; ++j) cm[j] = fmaxf(cm[j], fabsf(f[j]));
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      cm[j] = fmaxf(cm[j], __shfl_xor_sync(0xffffffffu, cm[j], 8));
      cm[j] = fmaxf(cm[j], __shfl_xor_sync(0xffffffffu, cm[j], 16));
    }
    if (lane < 8 && k_ok)
#pragma unroll
      for (int j = 0; j < 16; ++j) atomicMax(cmax + 16 * l8 + j, __float_as_uint(cm[j]));
    __syncthreads();
    const int64_t col = static_cast<int64_t>(blockIdx.x) * 128 + tid;
    if (tid < 128 && col < K) atomicMax(reinterpret_cast<unsigned int*>(o.chan_amax) + col, cmax[tid]);
  } else {
    float cm[16];  // kSmooth: this thread's 16 channel factors (the same for all its rows)
    if constexpr (kSmooth) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 v = k_ok ? *reinterpret_cast<const float4*>(o.chan + k + 4 * q) : make_float4(0.f, 0.f, 0.f, 0.f);
        cm[4 * q] = v.x;
        cm[4 * q + 1] = v.y;
        cm[4 * q + 2] = v.z;
        cm[4 * q + 3] = v.w;
      }
    }

#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = 16 * warp + 4 * i + (lane >> 3);  // row within the tile
      const int64_t row = row0 + r;
      float f[16];
      bf16x16_to_float(w[i], f);
      uint32_t amax;
      if constexpr (kSmooth) {
        float m = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          f[j] = __fmul_rn(f[j], cm[j]);
          m = fmaxf(m, fabsf(f[j]));
        }
        amax = __float_as_uint(m);
      } else {
        amax = bf16x16_absmax(w[i]);
      }
      amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 1));  // the other half of the block
      const int e = block_exponent<kUOS>(amax);
      const float s = exp2_neg(e);  // exact power of two

      uint32_t out[2];
      const float2 s2 = make_float2(s, s);
#pragma unroll
      for (int q = 0; q < 2; ++q) {  // packed FP32x2 products (each exact, as two scalar ones)
        const float* g = f + 8 * q;
        const float2 v0 = __fmul2_rn(make_float2(g[0], g[1]), s2), v1 = __fmul2_rn(make_float2(g[2], g[3]), s2);
        const float2 v2 = __fmul2_rn(make_float2(g[4], g[5]), s2), v3 = __fmul2_rn(make_float2(g[6], g[7]), s2);
        out[q] = e2m1x8(v0.x, v0.y, v1.x, v1.y, v2.x, v2.y, v3.x, v3.y);
      }
      if (kQdq) {
        if (row < rows && k_ok) {
          const float up = exp2_pos(e);
          uint32_t b[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) b[j] = e2m1x2_to_bf16x2((out[j >> 2] >> (8 * (j & 3))) & 0xFFu, up);
          uint4* dst = reinterpret_cast<uint4*>(o.qdq + row * o.ldq + k);
          dst[0] = make_uint4(b[0], b[1], b[2], b[3]);
          dst[1] = make_uint4(b[4], b[5], b[6], b[7]);
        }
      } else if (row < rows && k_ok) {
        *reinterpret_cast<uint2*>(o.codes + row * (K / 2) + k / 2) = make_uint2(out[0], out[1]);
        if ((l8 & 1) == 0) atom[(r & 31) * 16 + (r >> 5) * 4 + (l8 >> 1)] = static_cast<uint8_t>(e + 127);
      }
    }
    if (kQdq) return;  // uniform: no scale atom to write
    __syncthreads();
    if (tid < 32) {
      const int64_t atoms_per_row_tile = (K + 127) / 128;
      const int64_t idx = static_cast<int64_t>(blockIdx.y) * atoms_per_row_tile + blockIdx.x;
      reinterpret_cast<uint4*>(o.sf + idx * 512)[tid] = reinterpret_cast<const uint4*>(atom)[tid];
    }
  }
}

// The rotated variant of the tile: four lanes per 128-element chunk, lane j holding the
// chunk's 32-block j as 16 packed pairs P[i] = (t[i], t[i + 16]).  Butterfly strides 1..8
// run on packed pairs (FP32x2 adds, the difference by a negated operand: each exactly
// rounded per half), stride 16 is the within-pair butterfly, strides 32 and 64 are
// cross-lane exchanges (lanes xor 1 and xor 2);
// the stage order and every rounding are those of the definition, so the rotated values are
// bit-identical to the element-by-element butterfly.  A lane ends with exactly one 32-block:
// its maximum, scale and 16 code bytes need no further exchange.  256 threads cover 64 rows
// per pass, two passes per 128-row tile.
template <bool kUOS, int kOut = kOutCodes, bool kSmooth = false>
__device__ __forceinline__ void quantize_mxfp4_hadamard_tile(const uint16_t* __restrict__ x, int64_t rows,
                                                             int64_t K, int64_t ld, const TileArgs& o) {
  constexpr bool kQdq = kOut == kOutQdq;
  __shared__ __align__(16) uint8_t atom[512];  // scale atom, or the 128 column maxima (kOutAbsmax)
  // the tile's 128 channel factors, paired as the values are: block b's pair i (at 18 b + i,
  // rows of 18 pairs so that the four blocks' reads fall in different banks) holds
  // channels 32 b + i and 32 b + 16 + i
  __shared__ __align__(16) float2 s_chan[kSmooth ? 72 : 1];
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int j = tid & 3;  // 32-block of the chunk
  const int64_t k = static_cast<int64_t>(blockIdx.x) * 128 + 32 * j;  // K % 128 == 0

  reinterpret_cast<uint32_t*>(atom)[tid & 127] = 0u;
  if constexpr (kSmooth) {
    if (tid < 128) {
      const float v = o.chan[static_cast<int64_t>(blockIdx.x) * 128 + tid];
      float* pairs = reinterpret_cast<float*>(s_chan);
      pairs[(tid >> 5) * 36 + (tid & 15) * 2 + ((tid >> 4) & 1)] = v;
    }
  }
  __syncthreads();  // atom zeroed, channel factors staged

  const float c = __uint_as_float(kInvSqrt128Bits);
  const float2 cc = make_float2(c, c);
  constexpr bool kFold = !kSmooth && kOut != kOutAbsmax;
  // kOutAbsmax: this lane's 32 column maxima over its rows of both passes; column k of
  // block j is cm[k] (k < 16: element k, else element k of the pairs' upper halves)
  float cm[kOut == kOutAbsmax ? 32 : 1];
  if constexpr (kOut == kOutAbsmax) {
#pragma unroll
    for (int q = 0; q < 32; ++q) cm[q] = 0.f;
  }
  // both passes' rows are loaded before either is computed: the second pass's loads are
  // in flight during the first pass's arithmetic
  uint32_t w[2][2][8];
#pragma unroll
  for (int pass = 0; pass < 2; ++pass) {
    const int64_t row = static_cast<int64_t>(blockIdx.y) * 128 + 64 * pass + (tid >> 2);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      if (row < rows) {
        ld_stream_v8(x + row * ld + k + 16 * q, w[pass][q]);
      } else {
#pragma unroll
        for (int u = 0; u < 8; ++u) w[pass][q][u] = 0u;
      }
    }
  }
#pragma unroll
  for (int pass = 0; pass < 2; ++pass) {
    const int r = 64 * pass + (tid >> 2);  // row within the tile
    const int64_t row = static_cast<int64_t>(blockIdx.y) * 128 + r;
    const bool ok = row < rows;
    float2 P[16];
    // element i of the block sits in w[pass][i / 16][(i % 16) / 2] (low / high half)
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t wl = w[pass][0][i >> 1], wh = w[pass][1][i >> 1];
      P[i].x = __uint_as_float((i & 1) ? (wl & 0xFFFF0000u) : (wl << 16));
      P[i].y = __uint_as_float((i & 1) ? (wh & 0xFFFF0000u) : (wh << 16));
    }
#pragma unroll
    for (int h = 1; h < 16; h *= 2) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if (i & h) continue;
        const float2 a = P[i], b = P[i + h];
        P[i] = __fadd2_rn(a, b);
        P[i + h] = __fadd2_rn(a, make_float2(-b.x, -b.y));  // a - b, exactly rounded
      }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {  // stride 16: the two halves of each pair
      const float a = P[i].x, b = P[i].y;
      P[i] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
    }
#pragma unroll
    for (int sh = 1; sh <= 2; sh <<= 1) {  // strides 32 (lanes xor 1) and 64 (lanes xor 2):
      // the lower block gets own + partner, the upper partner - own
      const float sgn = (j & sh) ? -1.f : 1.f;
      const float2 sg = make_float2(sgn, sgn);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 p =
            make_float2(__shfl_xor_sync(0xffffffffu, P[i].x, sh), __shfl_xor_sync(0xffffffffu, P[i].y, sh));
        P[i] = __ffma2_rn(P[i], sg, p);
      }
    }
    // The rotated values are y = fl32(t * c).  Where only their codes are needed (no
    // SmoothQuant, no channel maxima), the multiply by c is folded into the block scale
    // below (kFold) and P keeps the butterfly outputs t.
    if constexpr (!kFold) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        P[i] = __fmul2_rn(P[i], cc);
        if constexpr (kSmooth) {  // read at the point of use: the 32 factors are not held in registers
          float2 ch;
          asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(ch.x), "=f"(ch.y) : "r"(smem_u32(&s_chan[18 * j + i])));
          P[i] = __fmul2_rn(P[i], ch);
        }
      }
    }
    if constexpr (kOut == kOutAbsmax) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        cm[i] = fmaxf(cm[i], fabsf(P[i].x));
        cm[16 + i] = fmaxf(cm[16 + i], fabsf(P[i].y));
      }
      continue;
    }
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) m = fmaxf(m, fmaxf(fabsf(P[i].x), fabsf(P[i].y)));
    // Folded scaling.  max |y| = fl32(max |t| * c) since rounding is monotone, so the block
    // exponent is the definition's.  Each code is then taken from fl32(t * fl32(c 2^-e))
    // instead of fl32(fl32(t * c) 2^-e); the two agree for every t the butterfly can
    // produce from BF16 rows:
    //  - where fl32(t * c) is normal, scaling by the power of two 2^-e commutes with the
    //    rounding (both values below 2^-126 after scaling give code 0 with the sign of t);
    //  - where fl32(t * c) would be subnormal, |t| < 2^-122.5 and t is a multiple of 2^-133
    //    (BF16 values are, and so are FP32 sums of them at these magnitudes): for every such t
    //    and every block exponent the two forms give the same code (an exhaustive host test);
    //  - an infinite block maximum (e = 127, from a butterfly overflow) gives 6 for the
    //    infinite elements and 0 for the finite ones either way (|t| c 2^-127 < 1/4).
    if constexpr (kFold) m = __fmul_rn(m, c);
    const int e = block_exponent<kUOS>(__float_as_uint(m));
    const float s1 = kFold ? __fmul_rn(c, exp2_neg(e)) : exp2_neg(e);
    const float2 sc = make_float2(s1, s1);
    // Scaled as the pairs are held, V[i] = P[i] * s1 (block elements i and i + 16): pairing
    // elements of different registers for the packed multiply would cost two moves each.
    // Code word w holds elements 8w..8w+7: V[8w + u].x for w < 2, V[8(w - 2) + u].y else.
    float2 V[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) V[i] = __fmul2_rn(P[i], sc);
    uint32_t out[4];
#pragma unroll
    for (int wd = 0; wd < 4; ++wd) {
      const int b = 8 * (wd & 1);
      out[wd] = wd < 2 ? e2m1x8(V[b].x, V[b + 1].x, V[b + 2].x, V[b + 3].x, V[b + 4].x, V[b + 5].x, V[b + 6].x, V[b + 7].x)
                       : e2m1x8(V[b].y, V[b + 1].y, V[b + 2].y, V[b + 3].y, V[b + 4].y, V[b + 5].y, V[b + 6].y, V[b + 7].y);
    }
    if (kQdq) {
      if (ok) {
        const float up = exp2_pos(e);
        uint32_t b[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) b[u] = e2m1x2_to_bf16x2((out[u >> 2] >> (8 * (u & 3))) & 0xFFu, up);
        uint4* dst = reinterpret_cast<uint4*>(o.qdq + row * o.ldq + k);
#pragma unroll
        for (int q = 0; q < 4; ++q) dst[q] = make_uint4(b[4 * q], b[4 * q + 1], b[4 * q + 2], b[4 * q + 3]);
      }
    } else {
      if (ok)
        *reinterpret_cast<uint4*>(o.codes + row * (K / 2) + k / 2) = make_uint4(out[0], out[1], out[2], out[3]);
      atom[(r & 31) * 16 + (r >> 5) * 4 + j] = static_cast<uint8_t>(e + 127);
    }
  }
  if (kQdq) return;  // uniform: no scale atom to write
  if constexpr (kOut == kOutAbsmax) {
    // Column maxima over the 8 rows of this warp that share block j (lanes xor 4, 8, 16)
    // by reduce-scatter: each round keeps half of the columns and takes the partner's
    // maxima of them (28 shuffles instead of 96), leaving every lane 4 finished columns;
    // then over the warps in shared memory.
    const int b4 = (lane >> 4) & 1, b3 = (lane >> 3) & 1, b2 = (lane >> 2) & 1;
    float c16[16], c8[8], c4[4];
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const float send = b4 ? cm[q] : cm[16 + q];
      c16[q] = fmaxf(b4 ? cm[16 + q] : cm[q], __shfl_xor_sync(0xffffffffu, send, 16));
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float send = b3 ? c16[q] : c16[8 + q];
      c8[q] = fmaxf(b3 ? c16[8 + q] : c16[q], __shfl_xor_sync(0xffffffffu, send, 8));
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float send = b2 ? c8[q] : c8[4 + q];
      c4[q] = fmaxf(b2 ? c8[4 + q] : c8[q], __shfl_xor_sync(0xffffffffu, send, 4));
    }
    uint32_t* cmax = reinterpret_cast<uint32_t*>(atom);
    const int col = 32 * j + 16 * b4 + 8 * b3 + 4 * b2;
#pragma unroll
    for (int q = 0; q < 4; ++q) atomicMax(cmax + col + q, __float_as_uint(c4[q]));
  }
  __syncthreads();
  if constexpr (kOut == kOutAbsmax) {
    if (tid < 128)
      atomicMax(reinterpret_cast<unsigned int*>(o.chan_amax) + static_cast<int64_t>(blockIdx.x) * 128 + tid,
                reinterpret_cast<const uint32_t*>(atom)[tid]);
  } else if (tid < 32) {
    const int64_t idx = static_cast<int64_t>(blockIdx.y) * (K / 128) + blockIdx.x;
    reinterpret_cast<uint4*>(o.sf + idx * 512)[tid] = reinterpret_cast<const uint4*>(atom)[tid];
  }
}

template <bool kHadamard, bool kUOS, int kOut, bool kSmooth>
__device__ __forceinline__ void mxfp4_tile(const uint16_t* __restrict__ x, int64_t rows, int64_t K, int64_t ld,
                                           const TileArgs& o) {
  if constexpr (kHadamard)
    quantize_mxfp4_hadamard_tile<kUOS, kOut, kSmooth>(x, rows, K, ld, o);
  else
    quantize_mxfp4_tile<kUOS, kOut, kSmooth>(x, rows, K, ld, o);
}

// Occupancy: without rotation the tile fits 48 registers, five CTAs (40 warps) per SM to
// cover the load latency; the rotated tile is held to 64 registers, four CTAs per SM
// (three at the 76-78 it takes unconstrained; four measured 0.6 % faster per step).
template <bool kHadamard, bool kUOS>
__global__ void __launch_bounds__(kQuantThreads, kHadamard ? 4 : 5) quantize_act_mxfp4_kernel(
    const uint16_t* __restrict__ x, int64_t M, int64_t K, int64_t ldx, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ sf) {
  griddep_launch_dependents();  // a GEMM launched after this may run its prologue now
  TileArgs o;
  o.codes = codes;
  o.sf = sf;
  mxfp4_tile<kHadamard, kUOS, kOutCodes, false>(x, M, K, ldx, o);
}

// The offline weight packer: the same block arithmetic on W[N][K] rows.
template <bool kHadamard, bool kUOS>
__global__ void __launch_bounds__(kQuantThreads) pack_weight_mxfp4_kernel(
    const uint16_t* __restrict__ w, int64_t N, int64_t K, int64_t ldw, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ sf) {
  TileArgs o;
  o.codes = codes;
  o.sf = sf;
  mxfp4_tile<kHadamard, kUOS, kOutCodes, false>(w, N, K, ldw, o);
}

// Quantise-dequantise emulation of the MXFP4 activation quantiser (BF16 out).
template <bool kHadamard, bool kUOS>
__global__ void __launch_bounds__(kQuantThreads) qdq_act_mxfp4_kernel(const uint16_t* __restrict__ x, int64_t M,
                                                                       int64_t K, int64_t ldx,
                                                                       uint16_t* __restrict__ out, int64_t ldo) {
  TileArgs o;
  o.qdq = out;
  o.ldq = ldo;
  mxfp4_tile<kHadamard, kUOS, kOutQdq, false>(x, M, K, ldx, o);
}

// SmoothQuant after the (optional) rotation: codes of (x R) * chan per channel.  Serves
// activations (chan = 1/lambda) and the offline weight packer (chan = lambda).
template <bool kHadamard, bool kUOS>
__global__ void __launch_bounds__(kQuantThreads) quantize_smooth_mxfp4_kernel(
    const uint16_t* __restrict__ x, int64_t rows, int64_t K, int64_t ld, const float* __restrict__ chan,
    uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
  griddep_launch_dependents();  // a GEMM launched after this may run its prologue now
  TileArgs o;
  o.codes = codes;
  o.sf = sf;
  o.chan = chan;
  mxfp4_tile<kHadamard, kUOS, kOutCodes, true>(x, rows, K, ld, o);
}

// Calibration statistic: amax[k] = max(amax[k], max over rows of |(x R)[r][k]|).
template <bool kHadamard>
__global__ void __launch_bounds__(kQuantThreads) channel_absmax_kernel(const uint16_t* __restrict__ x,
                                                                        int64_t rows, int64_t K, int64_t ld,
                                                                        float* __restrict__ amax) {
  TileArgs o;
  o.chan_amax = amax;
  mxfp4_tile<kHadamard, false, kOutAbsmax, false>(x, rows, K, ld, o);
}

// SmoothQuant migration factors, one thread per channel:
// lambda = max(ax^a / max(aw, 1e-5)^(1-a), 1e-5), inv_lambda = 1 / lambda (IEEE division).
__global__ void smooth_factors_kernel(const float* __restrict__ ax, const float* __restrict__ aw, int64_t K,
                                      float alpha, float* __restrict__ lambda, float* __restrict__ inv_lambda) {
  const int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (k >= K) return;
  const float l = fmaxf(__fdiv_rn(powf(ax[k], alpha), powf(fmaxf(aw[k], 1e-5f), 1.0f - alpha)), 1e-5f);
  lambda[k] = l;
  inv_lambda[k] = __fdiv_rn(1.0f, l);
}

// MXFP4 -> BF16: a unit of work is 16 elements (8 code bytes + their scale byte from the
// swizzled buffer) expanded into 32 contiguous output bytes, so a warp reads 256 and writes
// 1024 contiguous bytes per unit.  Each thread takes kDequantUnroll units spaced one grid
// apart per pass, loading all of them before converting any (independent loads in flight),
// grid-stride over the [rows][K/16] units with (row, unit) advanced incrementally (no
// 64-bit division inside the loop).
constexpr int kDequantUnroll = 4;

__global__ void __launch_bounds__(kQuantThreads) dequant_mxfp4_kernel(const uint8_t* __restrict__ codes,
                                                                       const uint8_t* __restrict__ sf, int64_t rows,
                                                                       int64_t K, uint16_t* __restrict__ out,
                                                                       int64_t ldo) {
  const int64_t cpr = K / 16;  // units per row
  const int64_t atoms_per_row_tile = (K / 32 + 3) / 4;
  const int64_t S = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t start = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t dr1 = S / cpr, dc1 = S - dr1 * cpr;  // one grid of units
  const int64_t step = S * kDequantUnroll;
  const int64_t drU = step / cpr, dcU = step - drU * cpr;
  int64_t r[kDequantUnroll], c[kDequantUnroll];
  r[0] = start / cpr;
  c[0] = start - r[0] * cpr;
#pragma unroll
  for (int u = 1; u < kDequantUnroll; ++u) {
    r[u] = r[u - 1] + dr1;
    c[u] = c[u - 1] + dc1;
    if (c[u] >= cpr) {
      c[u] -= cpr;
      ++r[u];
    }
  }
  while (r[0] < rows) {  // r[0] <= r[1] <= ...: later units may already be past the end
    uint2 cw[kDequantUnroll];
    uint32_t sb[kDequantUnroll];
#pragma unroll
    for (int u = 0; u < kDequantUnroll; ++u) {
      if (r[u] < rows) {
        cw[u] = *reinterpret_cast<const uint2*>(codes + r[u] * (K / 2) + c[u] * 8);
        const int64_t blk = c[u] >> 1;
        sb[u] = sf[((r[u] >> 7) * atoms_per_row_tile + (blk >> 2)) * 512 + (r[u] & 31) * 16 +
                   ((r[u] & 127) >> 5) * 4 + (blk & 3)];
      }
    }
#pragma unroll
    for (int u = 0; u < kDequantUnroll; ++u) {
      if (r[u] < rows) {
        const float up = exp2_pos(static_cast<int>(sb[u]) - 127);
        uint32_t b[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          b[j] = e2m1x2_to_bf16x2((((j < 4) ? cw[u].x : cw[u].y) >> (8 * (j & 3))) & 0xFFu, up);
        uint4* dst = reinterpret_cast<uint4*>(out + r[u] * ldo + c[u] * 16);
        dst[0] = make_uint4(b[0], b[1], b[2], b[3]);
        dst[1] = make_uint4(b[4], b[5], b[6], b[7]);
      }
      r[u] += drU;
      c[u] += dcU;
      if (c[u] >= cpr) {
        c[u] -= cpr;
        ++r[u];
      }
    }
  }
}

// Static FP8: q = E4M3_RNE_satfinite(fl32(x * inv_scale)), sign bit kept, 16-element
// chunks (32 bytes in, 16 bytes out).  A CTA covers kFp8Rows rows x 64 chunks
// (grid.x over the chunk columns, grid.y over row groups, striding by gridDim.y groups); a
// thread takes one chunk column and kFp8Unroll rows kFp8Rows / kFp8Unroll apart, all their
// loads issued before any conversion (independent loads in flight, no index division).
constexpr int kFp8Unroll = 4;
constexpr int kFp8Rows = 4 * kFp8Unroll;  // 256 threads = 4 row slots x 64 chunk slots

__global__ void __launch_bounds__(kQuantThreads, 4) quantize_act_fp8_kernel(const uint16_t* __restrict__ x, int64_t M,
                                                                          int64_t K, int64_t ldx, float inv_scale,
                                                                          uint8_t* __restrict__ q) {
  griddep_launch_dependents();  // a GEMM launched after this may run its prologue now
  const int64_t kc = static_cast<int64_t>(blockIdx.x) * 64 + (threadIdx.x & 63);  // chunk column
  if (kc >= K / 16) return;  // no barrier below: threads past the row end leave early
  const int64_t k = kc * 16;
  for (int64_t r0 = static_cast<int64_t>(blockIdx.y) * kFp8Rows + (threadIdx.x >> 6); r0 < M;
       r0 += static_cast<int64_t>(gridDim.y) * kFp8Rows) {
    uint32_t w[kFp8Unroll][8];
#pragma unroll
    for (int u = 0; u < kFp8Unroll; ++u) {
      const int64_t row = r0 + 4 * u;
      if (row < M) ld_stream_v8(x + row * ldx + k, w[u]);
    }
#pragma unroll
    for (int u = 0; u < kFp8Unroll; ++u) {
      const int64_t row = r0 + 4 * u;
      if (row >= M) continue;
      float f[16];
      bf16x16_to_float(w[u], f);
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t lo = e4m3x2(__fmul_rn(f[4 * j], inv_scale), __fmul_rn(f[4 * j + 1], inv_scale));
        const uint32_t hi = e4m3x2(__fmul_rn(f[4 * j + 2], inv_scale), __fmul_rn(f[4 * j + 3], inv_scale));
        o[j] = lo | (hi << 16);
      }
      *reinterpret_cast<uint4*>(q + row * K + k) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

}  // namespace mxq

namespace mxq {

// Quantise-dequantise emulation of the static FP8 activations:
// out = bf16_rne(fl32(E4M3(fl32(x * inv_scale)) * scale)).
__global__ void __launch_bounds__(kQuantThreads) qdq_act_fp8_kernel(const uint16_t* __restrict__ x, int64_t M,
                                                                     int64_t K, int64_t ldx, float inv_scale,
                                                                     float scale, uint16_t* __restrict__ out,
                                                                     int64_t ldo) {
  const int64_t chunks_per_row = K / 16;
  const int64_t total = M * chunks_per_row;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c < total; c += stride) {
    const int64_t row = c / chunks_per_row;
    const int64_t k = (c - row * chunks_per_row) * 16;
    uint32_t w[8];
    ld_stream_v8(x + row * ldx + k, w);
    float f[16];
    bf16x16_to_float(w, f);
    uint32_t b[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      b[j] = e4m3x2_to_bf16x2(e4m3x2(__fmul_rn(f[2 * j], inv_scale), __fmul_rn(f[2 * j + 1], inv_scale)), scale);
    uint4* dst = reinterpret_cast<uint4*>(out + row * ldo + k);
    dst[0] = make_uint4(b[0], b[1], b[2], b[3]);
    dst[1] = make_uint4(b[4], b[5], b[6], b[7]);
  }
}

}  // namespace mxq
