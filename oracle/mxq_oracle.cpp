// mxq_oracle.cpp -- plain, slow, CPU reference of the MXFP4 quantized linear layer.
//
// TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
// this file; only the test suite, the package's smoke check and the CPU-baseline
// leg of the benchmark do.  It shares no code, header, table or constant with
// the CUDA library: every value below is derived here from the definitions.
//
// What it computes, and where each step comes from:
//
//  * MXFP4 block format -- 32 consecutive elements along K share one E8M0
//    (power-of-two, no mantissa) scale; elements are 4-bit E2M1.
//      [MXAttention: Data-Free Optimal Scaling and Pre-Normalization Quantization
//       for MXFP4 Attention -- "What it actually does", Universal Optimal Scaling]
//      [AMD Quark ... FLUX.1-dev MXFP4 -- "MXFP4とは何か": 32-element blocks share
//       one scale factor]
//    E2M1 magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6} and the E8M0 bias of 127 are the
//    OCP Microscaling (MX) v1.0 element / scale formats.
//  * OCP scale rule (stock OCP MXFP4): block exponent = floor(log2 amax) - 2, i.e.
//    the smallest e with amax / 2^e < 8 (2 = E2M1 emax), clamped to [-127, 127].
//  * UOS rule: the scaling boundary Qmax = 7.25, read as the smallest e with
//    amax / 2^e <= 7.25, clamped to [-127, 127].
//      [MXAttention -- TL;DR and "What it actually does": Qmax = 7.25]
//  * E2M1 element: round to nearest, ties to the even code index, saturating at
//    6, sign bit always kept (so -0 and small negatives encode to 0x8).
//  * Fixed 128-point block-Hadamard rotation: a deterministic, parameter-free
//    rotation.  [AMD Quark adds native W4A8 ... Wan2.2 -- "Quark quantization
//    pipeline and mixed-precision selection": fixed Hadamard rotations, no
//    learned parameters]  Normalised Sylvester H/sqrt(128) applied by an FP32
//    butterfly in a fixed order (stride 1, 2, 4, ..., 64), then one multiply by
//    fl32(1/sqrt(128)).
//  * FP8 E4M3 static activations (W4A8): q = E4M3_RNE_satfinite(fl32(x * inv_s))
//    with inv_s = fl32(1/s), s the static per-tensor scale.
//      [AMD Quark adds native W4A8 -- "MXFP4 formats and precision levels"]
//  * GEMM: the kernel consumes MX operands directly, with no dequantisation
//    phase, so its exact result is the GEMM of the dequantised operands:
//      y[m][n] = alpha * sum_k deqA[m][k] * deqB[n][k] + bias[n]   (in FP64).
//      [AMD Quark ... FLUX.1-dev MXFP4 -- "AMD Instinctプラットフォーム上の拡散
//       モデル向けMXFP4量子化": the GEMM takes MXFP4 inputs with no dequant phase]
//  * Quantise-dequantise (QDQ) emulation, the way the W4A8 results on the Wan2.2 page
//    were obtained before native execution ("Native execution paths": QDQ emulation,
//    quality only): out = BF16(dequant(quant(x))).  MXFP4: E2M1(code) * 2^e, exact in
//    FP32 and in BF16 (overflow to Inf only for e = 127); FP8: fl32(E4M3(q) * s)
//    rounded to BF16 (round to nearest even).
//  * SmoothQuant after the fixed rotation: the block-selection transform is a fixed
//    Hadamard rotation followed by SmoothQuant [AMD Quark adds native W4A8 ... Wan2.2 --
//    "Fixed rotation selector" and "Block-level SQNR calibration"].  Per channel k of
//    the (rotated) values y: activations y_k * (1/lambda_k), weight rows y_k * lambda_k,
//    so that the product is unchanged.  lambda is the SmoothQuant migration factor
//    (the pages give no formula; the published SmoothQuant definition is used):
//      lambda_k = max(ax_k^a / max(aw_k, 1e-5)^(1-a), 1e-5),
//    ax_k / aw_k = max over rows of |y_k| of the calibration activations / weights,
//    a = the migration strength.  The multiply is one FP32 product per element,
//    before the block maximum.
//  * Per-layer precision selection [AMD Quark adds native W4A8 ... Wan2.2 -- "Block-level
//    SQNR calibration"]: the output SQNR against the BF16 layer,
//      SQNR = 10 log10( sum ref^2 / sum (y - ref)^2 )  dB,
//    measured with plain MXFP4 and with the transform (rotation + SmoothQuant), then
//    tiered thresholds (values not on the pages; parameters): plain >= high -> plain W4A4;
//    else transform >= high -> transform-enabled W4A4; else the better of the two >= low
//    -> W4A8 promotion; else BF16 fallback.
//  * MXFP4 attention with UOS and PNQ [MXAttention: Data-Free Optimal Scaling and
//    Pre-Normalization Quantization for MXFP4 Attention -- TL;DR, "Architecture" and
//    "What it actually does"]: Q, K and V in MXFP4 (Q, K in 32-blocks along the head
//    dimension, V in 32-blocks along the keys), scores S = deq(Q) deq(K)^T, the
//    unnormalised exponentials quantised to MXFP4 in 32-key blocks BEFORE the row sum
//    (PNQ), the row sum l taken over the quantised values, O = (deq(P) deq(V)) / l.
//    Readings (the pages fix none of these): the numerators are taken in base 2,
//    t = fl32(fl32(S) * fl32(log2(e) / sqrt(d))) (the scores in FP32, as a tensor core
//    accumulates them), relative to an integer offset c = ceil(max_j t_j) -- a
//    power-of-two offset, under which E8M0 block scaling is exactly equivariant, so the
//    codes do not depend on it.  Each numerator is the exact exponential 2^(t - c),
//    evaluated in FP64; a 32-key block's E8M0 exponent follows the MX definition, from
//    the maximum of that block's numerators, and each numerator is rounded to E2M1 in
//    FP64 against it.  The row sum, the division and the product with V are FP64.
//  * Scale-factor memory layout (not given by the pages; a reading): rows padded
//    to a multiple of 128, scale columns to a multiple of 4, 512-byte atoms of
//    128 rows x 4 scale columns, byte
//      ((r/128)*(C/4) + c/4)*512 + (r%32)*16 + ((r%128)/32)*4 + (c%4),
//    padding bytes 0x00.  This is a separate function (oracle_sf_swizzle) applied
//    to the logical [rows][K/32] scale array.
//
// Build: g++ -O2 -std=c++17 -ffp-contract=off -fPIC -shared -pthread
// (no -ffast-math: every float operation below is a correctly rounded IEEE op).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

constexpr int kBlock = 32;        // MX block size along K
constexpr int kHadamardN = 128;   // block-Hadamard length along K
[[maybe_unused]] constexpr int kRuleOCP = 0;
constexpr int kRuleUOS = 1;

float bf16_bits_to_float(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return f;
}

// E2M1 magnitudes, index = the 3 low bits of a code.
const double kE2M1Magnitude[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

// Runs fn(row_begin, row_end) over [0, rows) on nthreads std::threads.
template <class Fn>
void parallel_rows(int64_t rows, int nthreads, Fn fn) {
  if (nthreads < 1) nthreads = 1;
  if (rows < nthreads) nthreads = static_cast<int>(std::max<int64_t>(rows, 1));
  if (nthreads == 1) {
    fn(int64_t{0}, rows);
    return;
  }
  std::vector<std::thread> pool;
  const int64_t chunk = (rows + nthreads - 1) / nthreads;
  for (int t = 0; t < nthreads; ++t) {
    const int64_t b = t * chunk;
    const int64_t e = std::min(rows, b + chunk);
    if (b >= e) break;
    pool.emplace_back([=] { fn(b, e); });
  }
  for (auto& th : pool) th.join();
}

}  // namespace

extern "C" {

// ---------------------------------------------------------------- element codecs

// E2M1 encode of a value already divided by its block scale.
// Nearest of the eight magnitudes to a = min(|v|, 6); on an exact tie the
// candidate with the even index wins.  Bit 3 = sign bit of v, always kept.
uint8_t oracle_e2m1_encode(double v) {
  const int sign = std::signbit(v) ? 1 : 0;
  double a = std::fabs(v);
  if (a > 6.0) a = 6.0;
  int best = 0;
  double best_dist = INFINITY;
  for (int i = 0; i < 8; ++i) {
    const double d = std::fabs(a - kE2M1Magnitude[i]);
    if (d < best_dist || (d == best_dist && i % 2 == 0)) {
      best = i;
      best_dist = d;
    }
  }
  return static_cast<uint8_t>((sign << 3) | best);
}

double oracle_e2m1_decode(uint8_t code) {
  const double mag = kE2M1Magnitude[code & 7];
  return (code & 8) ? -mag : mag;
}

// FP8 E4M3 (OCP "FN" variant: no infinities, S.1111.111 is NaN) decode.
double oracle_e4m3_decode(uint8_t code) {
  const int sign = code >> 7;
  const int exp_field = (code >> 3) & 0xF;
  const int man = code & 7;
  double mag;
  if (exp_field == 0xF && man == 7) {
    mag = NAN;
  } else if (exp_field == 0) {
    mag = std::ldexp(static_cast<double>(man), -9);  // subnormal: man/8 * 2^-6
  } else {
    mag = std::ldexp(1.0 + man / 8.0, exp_field - 7);
  }
  return sign ? -mag : mag;
}

// FP8 E4M3 encode: round to nearest, ties to even code (the even mantissa), with
// saturation to the largest finite magnitude 448 ("satfinite"); sign bit kept.
uint8_t oracle_e4m3_encode(double v) {
  const int sign = std::signbit(v) ? 1 : 0;
  double a = std::fabs(v);
  if (a > 448.0) a = 448.0;
  // Magnitudes of every non-negative finite code 0x00..0x7E, ascending.
  static const std::vector<double> table = [] {
    std::vector<double> t(0x7F);
    for (int c = 0; c <= 0x7E; ++c) t[c] = oracle_e4m3_decode(static_cast<uint8_t>(c));
    return t;
  }();
  int best = 0;
  double best_dist = INFINITY;
  for (int c = 0; c <= 0x7E; ++c) {
    const double d = std::fabs(a - table[c]);
    if (d < best_dist || (d == best_dist && c % 2 == 0)) {
      best = c;
      best_dist = d;
    }
  }
  return static_cast<uint8_t>((sign << 7) | best);
}

// ---------------------------------------------------------------- block scale

// Shared block exponent e (scale 2^e, stored as the E8M0 byte e + 127).
//   OCP: smallest e in [-127, 127] with amax / 2^e <  8
//   UOS: smallest e in [-127, 127] with amax / 2^e <= 7.25
// amax = 0 gives e = -127 (byte 0x00).
int oracle_block_exponent(double amax, int rule) {
  for (int e = -127; e <= 127; ++e) {
    if (rule == kRuleUOS) {
      if (amax <= std::ldexp(7.25, e)) return e;
    } else {
      if (amax < std::ldexp(8.0, e)) return e;
    }
  }
  return 127;  // only reached by non-finite amax, which is out of contract
}

// ---------------------------------------------------------------- rotation

// 128-point normalised Sylvester-Hadamard on one chunk, in FP32, fixed order.
void oracle_fwht128(const float* x, float* y) {
  float t[kHadamardN];
  for (int i = 0; i < kHadamardN; ++i) t[i] = x[i];
  for (int h = 1; h < kHadamardN; h *= 2) {
    for (int i = 0; i < kHadamardN; ++i) {
      if (i & h) continue;
      const float a = t[i];
      const float b = t[i + h];
      t[i] = a + b;
      t[i + h] = a - b;
    }
  }
  const float c = static_cast<float>(1.0 / std::sqrt(128.0));
  for (int i = 0; i < kHadamardN; ++i) y[i] = t[i] * c;
}

float oracle_hadamard_scale(void) { return static_cast<float>(1.0 / std::sqrt(128.0)); }

// ---------------------------------------------------------------- SF layout

int64_t oracle_sf_padded_rows(int64_t rows) { return (rows + 127) / 128 * 128; }
int64_t oracle_sf_padded_cols(int64_t K) { return (K / kBlock + 3) / 4 * 4; }
int64_t oracle_sf_bytes(int64_t rows, int64_t K) {
  return oracle_sf_padded_rows(rows) * oracle_sf_padded_cols(K);
}

int64_t oracle_sf_offset(int64_t r, int64_t c, int64_t K) {
  const int64_t C = oracle_sf_padded_cols(K);
  return ((r / 128) * (C / 4) + c / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);
}

// logical [rows][K/32] -> physical swizzled buffer of oracle_sf_bytes(rows, K),
// padding bytes 0x00.
void oracle_sf_swizzle(const uint8_t* logical, int64_t rows, int64_t K, uint8_t* physical) {
  const int64_t nb = K / kBlock;
  std::memset(physical, 0, static_cast<size_t>(oracle_sf_bytes(rows, K)));
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < nb; ++c) physical[oracle_sf_offset(r, c, K)] = logical[r * nb + c];
}

void oracle_sf_unswizzle(const uint8_t* physical, int64_t rows, int64_t K, uint8_t* logical) {
  const int64_t nb = K / kBlock;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < nb; ++c) logical[r * nb + c] = physical[oracle_sf_offset(r, c, K)];
}

// ---------------------------------------------------------------- quantizers

// Optional rotation of one row: y = FP32 values the quantiser sees.
static void row_to_float(const uint16_t* xrow, int64_t K, int hadamard, float* y) {
  for (int64_t k = 0; k < K; ++k) y[k] = bf16_bits_to_float(xrow[k]);
  if (hadamard) {
    float tmp[kHadamardN];
    for (int64_t c0 = 0; c0 < K; c0 += kHadamardN) {
      oracle_fwht128(y + c0, tmp);
      std::memcpy(y + c0, tmp, sizeof tmp);
    }
  }
}

// MXFP4 quantisation of rows x K BF16 values (row stride ld elements), with an optional
// per-channel multiplier applied after the rotation (chan_scale == nullptr: none).
// codes: [rows][K/2] bytes, element k in byte k/2, low nibble when k is even.
// sf_logical: [rows][K/32] E8M0 bytes.
static void quantize_rows(const uint16_t* x, int64_t rows, int64_t K, int64_t ld, int rule, int hadamard,
                          const float* chan_scale, uint8_t* codes, uint8_t* sf_logical, int nthreads) {
  parallel_rows(rows, nthreads, [&](int64_t r0, int64_t r1) {
    std::vector<float> y(static_cast<size_t>(K));
    for (int64_t r = r0; r < r1; ++r) {
      row_to_float(x + r * ld, K, hadamard, y.data());
      if (chan_scale)
        for (int64_t k = 0; k < K; ++k) y[k] = y[k] * chan_scale[k];  // fl32 product
      for (int64_t b = 0; b < K / kBlock; ++b) {
        const float* blk = y.data() + b * kBlock;
        double amax = 0.0;
        for (int i = 0; i < kBlock; ++i) amax = std::max(amax, std::fabs(static_cast<double>(blk[i])));
        const int e = oracle_block_exponent(amax, rule);
        sf_logical[r * (K / kBlock) + b] = static_cast<uint8_t>(e + 127);
        for (int i = 0; i < kBlock; ++i) {
          const int64_t k = b * kBlock + i;
          const uint8_t q = oracle_e2m1_encode(std::ldexp(static_cast<double>(blk[i]), -e));
          uint8_t& byte = codes[r * (K / 2) + k / 2];
          if (k % 2 == 0) byte = static_cast<uint8_t>((byte & 0xF0) | q);
          else            byte = static_cast<uint8_t>((byte & 0x0F) | (q << 4));
        }
      }
    }
  });
}

void oracle_quantize_mxfp4(const uint16_t* x, int64_t rows, int64_t K, int64_t ld, int rule,
                           int hadamard, uint8_t* codes, uint8_t* sf_logical, int nthreads) {
  quantize_rows(x, rows, K, ld, rule, hadamard, nullptr, codes, sf_logical, nthreads);
}

// The same with SmoothQuant's per-channel multiplier (1/lambda for activations, lambda
// for weights) applied to the rotated values.
void oracle_quantize_mxfp4_smooth(const uint16_t* x, int64_t rows, int64_t K, int64_t ld, int rule,
                                  int hadamard, const float* chan_scale, uint8_t* codes,
                                  uint8_t* sf_logical, int nthreads) {
  quantize_rows(x, rows, K, ld, rule, hadamard, chan_scale, codes, sf_logical, nthreads);
}

// Calibration statistic: amax[k] = max over rows of |y[r][k]| (y rotated or not).
void oracle_channel_absmax(const uint16_t* x, int64_t rows, int64_t K, int64_t ld, int hadamard,
                           float* amax) {
  std::vector<float> y(static_cast<size_t>(K));
  for (int64_t k = 0; k < K; ++k) amax[k] = 0.0f;
  for (int64_t r = 0; r < rows; ++r) {
    row_to_float(x + r * ld, K, hadamard, y.data());
    for (int64_t k = 0; k < K; ++k) amax[k] = std::max(amax[k], std::fabs(y[k]));
  }
}

// SmoothQuant migration factors: lambda[k] = max(ax^a / max(aw, 1e-5)^(1 - a), 1e-5),
// evaluated in FP64 and rounded once to FP32; inv_lambda[k] = fl32(1 / lambda[k]).
void oracle_smooth_factors(const float* ax, const float* aw, int64_t K, double alpha, float* lambda,
                           float* inv_lambda) {
  for (int64_t k = 0; k < K; ++k) {
    const double w = std::max(static_cast<double>(aw[k]), 1e-5);
    const double l = std::max(std::pow(static_cast<double>(ax[k]), alpha) / std::pow(w, 1.0 - alpha), 1e-5);
    lambda[k] = static_cast<float>(l);
    inv_lambda[k] = 1.0f / lambda[k];
  }
}

// Returns the rotated FP32 values the quantiser sees (for tests).
void oracle_rotate_rows(const uint16_t* x, int64_t rows, int64_t K, int64_t ld, int hadamard,
                        float* y) {
  for (int64_t r = 0; r < rows; ++r) row_to_float(x + r * ld, K, hadamard, y + r * K);
}

// Static FP8 E4M3 activation quantisation: q = E4M3(fl32(x * inv_scale)).
void oracle_quantize_fp8(const uint16_t* x, int64_t rows, int64_t K, int64_t ld, float inv_scale,
                         uint8_t* q, int nthreads) {
  parallel_rows(rows, nthreads, [&](int64_t r0, int64_t r1) {
    for (int64_t r = r0; r < r1; ++r)
      for (int64_t k = 0; k < K; ++k) {
        const float v = bf16_bits_to_float(x[r * ld + k]) * inv_scale;  // fl32 product
        q[r * K + k] = oracle_e4m3_encode(static_cast<double>(v));
      }
  });
}

// ---------------------------------------------------------------- dequantisation

// MXFP4 -> FP64: value = E2M1(code) * 2^(sf - 127), sf read from the swizzled buffer.
void oracle_dequant_mxfp4(const uint8_t* codes, const uint8_t* sf_physical, int64_t rows,
                          int64_t K, double* out) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t k = 0; k < K; ++k) {
      const uint8_t byte = codes[r * (K / 2) + k / 2];
      const uint8_t q = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
      const int sf = sf_physical[oracle_sf_offset(r, k / kBlock, K)];
      out[r * K + k] = std::ldexp(oracle_e2m1_decode(q), sf - 127);
    }
}

// ---------------------------------------------------------------- QDQ emulation

// FP32 -> BF16, round to nearest, ties to even; NaN stays a (quiet) NaN.
uint16_t oracle_bf16_rne(float f) {
  uint32_t u;
  std::memcpy(&u, &f, sizeof u);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return static_cast<uint16_t>((u >> 16) | 0x40u);
  const uint32_t lsb = (u >> 16) & 1u;
  return static_cast<uint16_t>((u + 0x7FFFu + lsb) >> 16);
}

// BF16 of the dequantised MXFP4 values (scales from the swizzled buffer).
void oracle_dequant_mxfp4_bf16(const uint8_t* codes, const uint8_t* sf_physical, int64_t rows, int64_t K,
                               uint16_t* out) {
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t k = 0; k < K; ++k) {
      const uint8_t byte = codes[r * (K / 2) + k / 2];
      const uint8_t q = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
      const int sf = sf_physical[oracle_sf_offset(r, k / kBlock, K)];
      const double v = std::ldexp(oracle_e2m1_decode(q), sf - 127);  // exact, also as FP32 (or Inf)
      out[r * K + k] = oracle_bf16_rne(static_cast<float>(v));
    }
  }
}

// out = BF16(dequant(quant(x))) for MXFP4 with the given rule / rotation.
void oracle_qdq_mxfp4(const uint16_t* x, int64_t rows, int64_t K, int64_t ld, int rule, int hadamard,
                      uint16_t* out, int nthreads) {
  std::vector<uint8_t> codes(static_cast<size_t>(rows * (K / 2)));
  std::vector<uint8_t> sf_logical(static_cast<size_t>(rows * (K / kBlock)));
  oracle_quantize_mxfp4(x, rows, K, ld, rule, hadamard, codes.data(), sf_logical.data(), nthreads);
  std::vector<uint8_t> sf(static_cast<size_t>(oracle_sf_bytes(rows, K)));
  oracle_sf_swizzle(sf_logical.data(), rows, K, sf.data());
  oracle_dequant_mxfp4_bf16(codes.data(), sf.data(), rows, K, out);
}

// out = BF16(fl32(E4M3(fl32(x * inv_scale)) * scale)).
void oracle_qdq_fp8(const uint16_t* x, int64_t rows, int64_t K, int64_t ld, float inv_scale, float scale,
                    uint16_t* out, int nthreads) {
  std::vector<uint8_t> q(static_cast<size_t>(rows * K));
  oracle_quantize_fp8(x, rows, K, ld, inv_scale, q.data(), nthreads);
  for (int64_t i = 0; i < rows * K; ++i) {
    const float v = static_cast<float>(oracle_e4m3_decode(q[i])) * scale;  // fl32 product
    out[i] = oracle_bf16_rne(v);
  }
}

// ---------------------------------------------------------------- GEMM

// y[i][n] = alpha * sum_k A(row_idx[i], k) * B(n, k) + bias[n], FP64, unrounded.
//   a_kind 0: A is MXFP4 (a_codes [M][K/2] + swizzled a_sf)
//   a_kind 1: A is FP8 E4M3 (a_codes [M][K]; a_sf unused)
//   B is MXFP4 (b_codes [N][K/2] + swizzled b_sf); bias: N BF16 values or null.
void oracle_gemm(int a_kind, const uint8_t* a_codes, const uint8_t* a_sf, int64_t M,
                 const uint8_t* b_codes, const uint8_t* b_sf, int64_t N, int64_t K, double alpha,
                 const uint16_t* bias, const int64_t* row_idx, int64_t n_rows, double* y,
                 int nthreads) {
  std::vector<double> B(static_cast<size_t>(N * K));
  oracle_dequant_mxfp4(b_codes, b_sf, N, K, B.data());
  parallel_rows(n_rows, nthreads, [&](int64_t i0, int64_t i1) {
    std::vector<double> a(static_cast<size_t>(K));
    for (int64_t i = i0; i < i1; ++i) {
      const int64_t m = row_idx[i];
      if (a_kind == 0) {
        for (int64_t k = 0; k < K; ++k) {
          const uint8_t byte = a_codes[m * (K / 2) + k / 2];
          const uint8_t q = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
          const int sf = a_sf[oracle_sf_offset(m, k / kBlock, K)];
          a[k] = std::ldexp(oracle_e2m1_decode(q), sf - 127);
        }
      } else {
        for (int64_t k = 0; k < K; ++k) a[k] = oracle_e4m3_decode(a_codes[m * K + k]);
      }
      for (int64_t n = 0; n < N; ++n) {
        const double* b = B.data() + n * K;
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k) acc += a[k] * b[k];
        double v = alpha * acc;
        if (bias) v += static_cast<double>(bf16_bits_to_float(bias[n]));
        y[i * N + n] = v;
      }
    }
  });
  (void)M;
}

// ---------------------------------------------------------------- MXFP4 attention

// Attention of the sampled query rows q_rows[0..n_rows) for every head.
//   q: [Sq][ld], k, v: [Skv][ld] BF16, head h in columns [h*d, (h+1)*d), d % 32 == 0.
//   mode 0: PNQ (quantise the numerators, then the row sum); 1: the conventional order
//   (row-normalise in FP64, quantise the probabilities, no further division); 2: no
//   quantisation of P (FP64 softmax of the quantised-operand scores).
//   out: [n_rows][H][d] FP64; wsum: [n_rows][H] sum of the implied attention weights.
void oracle_attention_mxfp4(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t Sq, int64_t Skv,
                            int64_t H, int64_t d, int64_t ld, int rule, int mode, const int64_t* q_rows,
                            int64_t n_rows, double* out, double* wsum, int nthreads) {
  const int64_t HD = H * d;
  // K codes / scales for all rows (blocks along the head dimension).
  std::vector<uint8_t> kc(static_cast<size_t>(Skv * HD / 2)), ks(static_cast<size_t>(Skv * HD / kBlock));
  oracle_quantize_mxfp4(k, Skv, HD, ld, rule, 0, kc.data(), ks.data(), nthreads);
  // V^T per head and channel, blocks along the keys, zero-padded to a whole block.
  const int64_t Sp = (Skv + kBlock - 1) / kBlock * kBlock;
  std::vector<uint16_t> vt(static_cast<size_t>(HD * Sp), 0);
  for (int64_t j = 0; j < Skv; ++j)
    for (int64_t c = 0; c < HD; ++c) vt[c * Sp + j] = v[j * ld + c];
  std::vector<uint8_t> vc(static_cast<size_t>(HD * Sp / 2)), vs(static_cast<size_t>(HD * Sp / kBlock));
  oracle_quantize_mxfp4(vt.data(), HD, Sp, Sp, rule, 0, vc.data(), vs.data(), nthreads);
  auto deq = [](const uint8_t* codes, const uint8_t* sf, int64_t rowlen, int64_t r, int64_t i) {
    const uint8_t byte = codes[r * (rowlen / 2) + i / 2];
    const uint8_t c = (i % 2 == 0) ? (byte & 0xF) : (byte >> 4);
    return std::ldexp(oracle_e2m1_decode(c), static_cast<int>(sf[r * (rowlen / kBlock) + i / kBlock]) - 127);
  };
  std::vector<double> K(static_cast<size_t>(Skv * HD)), VT(static_cast<size_t>(HD * Sp));
  for (int64_t j = 0; j < Skv; ++j)
    for (int64_t c = 0; c < HD; ++c) K[j * HD + c] = deq(kc.data(), ks.data(), HD, j, c);
  for (int64_t c = 0; c < HD; ++c)
    for (int64_t j = 0; j < Sp; ++j) VT[c * Sp + j] = deq(vc.data(), vs.data(), Sp, c, j);
  const float scale = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d)));

  parallel_rows(n_rows, nthreads, [&](int64_t i0, int64_t i1) {
    std::vector<uint8_t> qc(static_cast<size_t>(HD / 2)), qs(static_cast<size_t>(HD / kBlock));
    std::vector<double> Q(static_cast<size_t>(HD)), P(static_cast<size_t>(Sp));
    std::vector<float> t(static_cast<size_t>(Skv));
    std::vector<double> pd(static_cast<size_t>(Sp));
    for (int64_t i = i0; i < i1; ++i) {
      const int64_t row = q_rows[i];
      oracle_quantize_mxfp4(q + row * ld, 1, HD, ld, rule, 0, qc.data(), qs.data(), 1);
      for (int64_t c = 0; c < HD; ++c) Q[c] = deq(qc.data(), qs.data(), HD, 0, c);
      for (int64_t h = 0; h < H; ++h) {
        float tmax = -INFINITY;
        for (int64_t j = 0; j < Skv; ++j) {
          double s = 0.0;
          for (int64_t c = 0; c < d; ++c) s += Q[h * d + c] * K[j * HD + h * d + c];
          t[j] = static_cast<float>(s) * scale;  // fl32(fl32(S) * scale)
          tmax = std::max(tmax, t[j]);
        }
        if (mode == 2) {  // FP64 softmax, no quantisation of P
          double l = 0.0;
          for (int64_t j = 0; j < Skv; ++j) l += (P[j] = std::exp2(static_cast<double>(t[j]) - tmax));
          for (int64_t j = Skv; j < Sp; ++j) P[j] = 0.0;
          for (int64_t j = 0; j < Sp; ++j) P[j] /= l;
        } else {
          // the unnormalised exponentials relative to the integer offset c, exact in FP64
          const double c = std::ceil(static_cast<double>(tmax));
          for (int64_t j = 0; j < Sp; ++j) pd[j] = j < Skv ? std::exp2(static_cast<double>(t[j]) - c) : 0.0;
          if (mode == 1) {  // conventional: normalise, then quantise
            double l = 0.0;
            for (int64_t j = 0; j < Sp; ++j) l += pd[j];
            for (int64_t j = 0; j < Sp; ++j) pd[j] /= l;
          }
          for (int64_t b = 0; b < Sp / kBlock; ++b) {  // MXFP4 of the numerators, 32-key blocks
            double amax = 0.0;  // the MX block maximum
            for (int u = 0; u < kBlock; ++u) amax = std::max(amax, std::fabs(pd[b * kBlock + u]));
            const int e = oracle_block_exponent(amax, rule);
            for (int u = 0; u < kBlock; ++u) {
              const double x = std::ldexp(pd[b * kBlock + u], -e);
              P[b * kBlock + u] = std::ldexp(oracle_e2m1_decode(oracle_e2m1_encode(x)), e);
            }
          }
          if (mode == 0) {  // PNQ: the row sum over the quantised numerators
            double l = 0.0;
            for (int64_t j = 0; j < Sp; ++j) l += P[j];
            for (int64_t j = 0; j < Sp; ++j) P[j] /= l;
          }
        }
        double ws = 0.0;
        for (int64_t j = 0; j < Sp; ++j) ws += P[j];
        if (wsum) wsum[i * H + h] = ws;
        for (int64_t c = 0; c < d; ++c) {
          double acc = 0.0;
          const double* vrow = VT.data() + (h * d + c) * Sp;
          for (int64_t j = 0; j < Sp; ++j) acc += P[j] * vrow[j];
          out[(i * H + h) * d + c] = acc;
        }
      }
    }
  });
  (void)Sq;
}

// ---------------------------------------------------------------- precision selection

// signal_noise[0] = sum ref^2, signal_noise[1] = sum (y - ref)^2 over n values (FP64).
void oracle_sqnr_sums(const double* y, const double* ref, int64_t n, double* signal_noise) {
  double s = 0.0, e = 0.0;
  for (int64_t i = 0; i < n; ++i) {
    s += ref[i] * ref[i];
    const double d = y[i] - ref[i];
    e += d * d;
  }
  signal_noise[0] = s;
  signal_noise[1] = e;
}

double oracle_sqnr_db(double signal, double noise) {
  if (noise <= 0.0) return HUGE_VAL;
  if (signal <= 0.0) return -HUGE_VAL;
  return 10.0 * std::log10(signal / noise);
}

// 0 = plain W4A4, 1 = transform-enabled W4A4 (rotation + SmoothQuant), 2 = W4A8, 3 = BF16.
int oracle_select_precision(double sqnr_plain_db, double sqnr_transform_db, double high_db, double low_db) {
  if (sqnr_plain_db >= high_db) return 0;
  if (sqnr_transform_db >= high_db) return 1;
  if (std::max(sqnr_plain_db, sqnr_transform_db) >= low_db) return 2;
  return 3;
}

}  // extern "C"
