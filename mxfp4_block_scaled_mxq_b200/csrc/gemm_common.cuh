// gemm_common.cuh -- what the two block-scaled GEMM kernels share.
//
// Both compute D[m][n] = bf16_rne(alpha * sum_k a[m][k] b[n][k] + bias[n]) on the
// 5th-generation tensor cores (tcgen05) with the MX operands as they are, with no
// dequantisation phase in between [AMD Quark ... FLUX.1-dev MXFP4 on MI350 -- "AMD
// Instinctプラットフォーム上の拡散モデル向けMXFP4量子化": the GEMM takes MXFP4 inputs directly]:
//   W4A4: tcgen05.mma kind::mxf4 -- A and B are E2M1 packed two per byte, one E8M0
//         scale per 32 K-elements per row, K = 64 per instruction.
//   W4A8: tcgen05.mma kind::mxf8f6f4 -- A is E4M3 (unit block scales, the static
//         per-tensor scale is the epilogue's alpha), B is E2M1 which the TMA unpacks
//         into 8-bit containers (16U4_ALIGN16B), K = 32 per instruction.
//   [AMD Quark adds native W4A8 ... Wan2.2 -- "MXFP4 formats and precision levels",
//    "Native execution paths"]
//
//   gemm_pair.cuh  M > 128: a two-CTA cluster per 256 x 192 output tile.
//   gemm_swap.cuh  M <= 128: one CTA per 128 weight rows, the tokens as the MMA's N.
//
// Every wait is bounded (ptx.cuh): on a timeout a kernel records MXQ_ERR_TIMEOUT,
// drains its own copies and MMAs, releases TMEM and returns.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "ptx.cuh"

namespace mxq {

constexpr int kBM = 128;           // rows of one CTA's share of a tile (TMEM lanes)
constexpr int kBN = 192;           // output columns of a CTA-pair tile
constexpr int kGemmThreads = 320;  // CTA-pair kernel: producer, MMA and 8 epilogue warps
constexpr int kEpiWarps = 8;
constexpr uint32_t kTmemCols = 512;

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&p);
}

}  // namespace mxq
