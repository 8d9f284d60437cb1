// gemm.cuh -- block-scaled GEMM on the 5th-generation tensor cores (tcgen05) with a
// fused BF16 epilogue:  D[m][n] = bf16_rne(alpha * sum_k a[m][k] b[n][k] + bias[n]).
//
// The MX operands go to the tensor cores as they are, with no dequantisation phase
// in between [AMD Quark ... FLUX.1-dev MXFP4 on MI350 -- "AMD Instinctプラット
// フォーム上の拡散モデル向けMXFP4量子化": the GEMM takes MXFP4 inputs directly]:
//   W4A4: tcgen05.mma kind::mxf4 -- A and B are E2M1 packed two per byte, one E8M0
//         scale per 32 K-elements per row, K = 64 per instruction.
//   W4A8: tcgen05.mma kind::mxf8f6f4 -- A is E4M3 (unit block scales, the static
//         per-tensor scale is the epilogue's alpha), B is E2M1 which the TMA unpacks
//         into 8-bit containers (16U4_ALIGN16B), K = 32 per instruction.
//   [AMD Quark adds native W4A8 ... Wan2.2 -- "MXFP4 formats and precision levels",
//    "Native execution paths"]
//
// Structure (one CTA per SM, persistent over 128 x 256 output tiles, N-fastest):
//   warp 0      TMA producer: A/B code tiles (2-D tensor maps, 128-byte swizzle) and
//               the tiles' scale atoms (1-D bulk copies) into a 4-stage ring.
//   warp 1      MMA issuer: tcgen05.cp of the scale atoms into TMEM, 4 MMAs per stage
//               into one 128 x 256 FP32 TMEM accumulator, tcgen05.commit to release
//               the stage / hand the accumulator to the epilogue.  Also owns the
//               TMEM allocation.
//   warps 2..9  epilogue: each warp drains 32 lanes x 128 columns of the accumulator
//               into registers and at once releases TMEM (so the next tile's MMAs
//               start), then scales, adds the bias, rounds to BF16, stages 32 x 32
//               sub-tiles in shared memory (64-byte swizzle) and TMA-stores them.
//
// Every wait is bounded (ptx.cuh): on a timeout the kernel records MXQ_ERR_TIMEOUT,
// drains its own copies and MMAs, releases TMEM and returns.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "ptx.cuh"

namespace mxq {

constexpr int kBM = 128;          // output rows per tile (TMEM lanes)
constexpr int kBN = 256;          // output columns per tile (TMEM columns)
constexpr int kStages = 4;
constexpr int kGemmThreads = 320; // 10 warps
constexpr int kEpiWarps = 8;
constexpr int kEpiStageBytes = 32 * 64;  // one warp's 32 rows x 32 BF16 columns
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0;          // accumulator: columns [0, 256)
constexpr uint32_t kSfaCol = 256;        // A scales: 2 parities x up to 2 atoms x 4 columns
constexpr uint32_t kSfbCol = 272;        // B scales: 2 parities x up to 2 atoms x 8 columns

template <bool kW4A8>
struct GemmShape {
  static constexpr int kBK = kW4A8 ? 128 : 256;        // K elements per stage
  static constexpr int kAtoms = kBK / 128;             // scale atoms (128 K each) per stage
  static constexpr int kMmaK = kW4A8 ? 32 : 64;        // K per MMA instruction
  static constexpr int kMmaPerAtom = 128 / kMmaK;      // 4 (W4A8) or 2 (W4A4)
  static constexpr int kAStage = kBM * 128;            // bytes: 128 rows x one 128-byte swizzle row
  static constexpr int kBStage = kBN * 128;
  static constexpr uint32_t kATx = kBM * 128;          // bytes the TMA delivers for A
  static constexpr uint32_t kBTx = kW4A8 ? kBN * 64 : kBN * 128;  // unpacked FP4: packed bytes count
  static constexpr int kSfaStage = kW4A8 ? 0 : kAtoms * 512;
  static constexpr int kSfbStage = 2 * kAtoms * 512;   // [row tile j][atom a]
  static constexpr int kSfaConst = kW4A8 ? 512 : 0;    // unit scales for E4M3 A
  static constexpr int kSmemBytes = 1024 /*alignment slack*/ + kStages * (kAStage + kBStage) +
                                    kEpiWarps * kEpiStageBytes + kStages * (kSfaStage + kSfbStage) +
                                    kSfaConst + 256 /*barriers + TMEM slot*/;
  // Instruction descriptor without the scale-factor ids (kind::mxf4 / kind::mxf8f6f4,
  // block_scale, K-major A and B, UE8M0 scales, M = 128, N = 256).
  static constexpr uint32_t kIdesc = (kW4A8 ? (0u << 7) | (5u << 10)    // A E4M3, B E2M1 (mxf8f6f4 codes)
                                            : (1u << 7) | (1u << 10))   // A, B E2M1 (mxf4 codes)
                                     | (static_cast<uint32_t>(kBN >> 3) << 17) | (1u << 23) /*UE8M0*/ |
                                     (static_cast<uint32_t>(kBM >> 4) << 24);
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&p);
}

template <bool kW4A8>
__global__ void __launch_bounds__(kGemmThreads, 1)
    mx_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                   const __grid_constant__ CUtensorMap tmap_d, const uint8_t* __restrict__ sfa,
                   const uint8_t* __restrict__ sfb, const __nv_bfloat16* __restrict__ bias, int M, int N, int K,
                   float alpha) {
  using S = GemmShape<kW4A8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + kStages * S::kAStage;
  uint8_t* sEpi = sB + kStages * S::kBStage;
  uint8_t* sSfa = sEpi + kEpiWarps * kEpiStageBytes;
  uint8_t* sSfb = sSfa + kStages * S::kSfaStage + S::kSfaConst;
  uint64_t* full = reinterpret_cast<uint64_t*>(sSfb + kStages * S::kSfbStage);
  uint64_t* empty = full + kStages;
  uint64_t* tmem_full = empty + kStages;
  uint64_t* tmem_empty = tmem_full + 1;
  uint64_t* drain = tmem_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m_tiles = (M + kBM - 1) / kBM;
  const int n_tiles = (N + kBN - 1) / kBN;
  const int num_tiles = m_tiles * n_tiles;
  const int k_stages = (K + S::kBK - 1) / S::kBK;
  const int atoms_per_row_tile = K / 128;  // K % 128 == 0

  if (threadIdx.x == 0) {
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    prefetch_tmap(&tmap_d);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, kEpiWarps);
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (kW4A8 && warp >= 2 && warp < 6) {
    // Unit block scales (E8M0 127 = 1.0) for the E4M3 activations: one atom.
    reinterpret_cast<uint32_t*>(sSfa)[threadIdx.x - 64] = 0x7F7F7F7Fu;
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0;  // bit s: stage s has loads in flight (parity = bit s of issued_phase)
      uint32_t issued_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        const int mt = tile / n_tiles, nt = tile % n_tiles;
        for (int ks = 0; ks < k_stages; ++ks) {
          if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
          issued |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          const int atoms = min(S::kAtoms, K / 128 - ks * S::kAtoms);
          const bool b_hi = (2 * nt + 1) * 128 < N;  // second 128-row half of the B tile exists
          const uint32_t tx = S::kATx + S::kBTx + (kW4A8 ? 0u : atoms * 512u) + (b_hi ? 2u : 1u) * atoms * 512u;
          mbar_arrive_expect_tx(&full[stage], tx);
          const int kx = kW4A8 ? ks * S::kBK : ks * (S::kBK / 2);  // A: E4M3 bytes / FP4 code bytes
          tma_load_2d(sA + stage * S::kAStage, &tmap_a, kx, mt * kBM, &full[stage]);
          tma_load_2d(sB + stage * S::kBStage, &tmap_b, kW4A8 ? ks * S::kBK : ks * (S::kBK / 2), nt * kBN,
                      &full[stage]);
          const int64_t atom0 = static_cast<int64_t>(ks) * S::kAtoms;
          if (!kW4A8)
            bulk_load(sSfa + stage * S::kSfaStage, sfa + (static_cast<int64_t>(mt) * atoms_per_row_tile + atom0) * 512,
                      atoms * 512, &full[stage]);
          for (int j = 0; j < (b_hi ? 2 : 1); ++j)
            bulk_load(sSfb + stage * S::kSfbStage + j * S::kAtoms * 512,
                      sfb + (static_cast<int64_t>(2 * nt + j) * atoms_per_row_tile + atom0) * 512, atoms * 512,
                      &full[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        // Drain: let every load already issued land before the CTA can exit.
        for (int s = 0; s < kStages; ++s)
          if (issued & (1u << s)) mbar_wait_drain(&full[s], (issued_phase >> s) & 1u);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0, sf_par = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        if (!mbar_wait(tmem_empty, acc_phase ^ 1)) { ok = false; break; }
        tc_fence_after();
        for (int ks = 0; ks < k_stages; ++ks) {
          if (!mbar_wait(&full[stage], phase)) { ok = false; break; }
          tc_fence_after();
          const int atoms = min(S::kAtoms, K / 128 - ks * S::kAtoms);
          const uint32_t par = sf_par;
          sf_par ^= 1u;  // alternate TMEM scale buffers from one stage to the next
          const uint32_t sfa_base = kW4A8 ? kSfaCol : kSfaCol + par * (S::kAtoms * 4);
          const uint32_t sfb_base = kSfbCol + par * (S::kAtoms * 8);
          for (int a = 0; a < atoms; ++a) {
            if (!kW4A8)
              tc_cp_sf_atom(tmem + sfa_base + 4 * a, smem_desc(smem_u32(sSfa + stage * S::kSfaStage + a * 512), 0, 128, 0));
            for (int j = 0; j < 2; ++j)
              tc_cp_sf_atom(tmem + sfb_base + 8 * a + 4 * j,
                            smem_desc(smem_u32(sSfb + stage * S::kSfbStage + j * S::kAtoms * 512 + a * 512), 0, 128, 0));
          }
          if (kW4A8 && tile == static_cast<int>(blockIdx.x) && ks == 0)
            tc_cp_sf_atom(tmem + kSfaCol, smem_desc(smem_u32(sSfa), 0, 128, 0));
          const uint32_t a_base = smem_u32(sA + stage * S::kAStage);
          const uint32_t b_base = smem_u32(sB + stage * S::kBStage);
          for (int kk = 0; kk < atoms * S::kMmaPerAtom; ++kk) {
            const int a = kk / S::kMmaPerAtom;
            const uint32_t sf_id = kW4A8 ? static_cast<uint32_t>(kk % S::kMmaPerAtom)
                                         : static_cast<uint32_t>((kk % S::kMmaPerAtom) * 2);
            const uint32_t idesc = S::kIdesc | (sf_id << 29) | (sf_id << 4);
            const uint64_t adesc = smem_desc(a_base + kk * 32, 16, 1024, 2);
            const uint64_t bdesc = smem_desc(b_base + kk * 32, 16, 1024, 2);
            const uint32_t tsfa = kW4A8 ? tmem + kSfaCol : tmem + sfa_base + 4 * a;
            const uint32_t tsfb = tmem + sfb_base + 8 * a;
            if (kW4A8)
              tc_mma_mxf8f6f4(tmem + kAccCol, adesc, bdesc, idesc, tsfa, tsfb, (ks | kk) != 0);
            else
              tc_mma_mxf4(tmem + kAccCol, adesc, bdesc, idesc, tsfa, tsfb, (ks | kk) != 0);
          }
          tc_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc_commit(tmem_full);
        acc_phase ^= 1;
      }
      if (!ok) {
        // Drain: wait (bounded) for every tcgen05 operation this thread issued.
        tc_commit(drain);
        mbar_wait_drain(drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int ew = warp - 2;          // 0..7
    const int quad = warp & 3;        // TMEM lanes [32*quad, +32) are this warp's
    const int chalf = ew >> 2;        // accumulator columns [128*chalf, +128)
    uint8_t* stage_buf = sEpi + ew * kEpiStageBytes;
    const uint32_t stage_addr = smem_u32(stage_buf);
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int mt = tile / n_tiles, nt = tile % n_tiles;
      // warp-uniform wait: tcgen05.ld below is .sync.aligned
      if (!__all_sync(0xffffffffu, mbar_wait(tmem_full, acc_phase))) break;
      tc_fence_after();
      uint32_t acc[4][32];
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quad * 32) << 16) + kAccCol + chalf * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(taddr + 32 * c, acc[c]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tmem_empty);
      acc_phase ^= 1;

      const int row_base = mt * kBM + quad * 32;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int n0 = nt * kBN + chalf * 128 + 32 * c;
        // previous sub-tile's store must have finished reading the staging buffer
        if (lane == 0) bulk_wait_read0();
        __syncwarp();
        uint32_t packed[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          float b0 = 0.f, b1 = 0.f;
          if (bias != nullptr) {
            const int n = n0 + 2 * j;
            if (n < N) b0 = __bfloat162float(bias[n]);
            if (n + 1 < N) b1 = __bfloat162float(bias[n + 1]);
          }
          const float v0 = __fmaf_rn(alpha, __uint_as_float(acc[c][2 * j]), b0);
          const float v1 = __fmaf_rn(alpha, __uint_as_float(acc[c][2 * j + 1]), b1);
          packed[j] = pack_bf16x2(v0, v1);
        }
        // Row `lane` of the 32 x 32 sub-tile: four 16-byte chunks, 64-byte swizzle
        // (chunk q of row r lives at chunk q ^ ((r >> 1) & 3)).
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t off = lane * 64 + ((q ^ ((lane >> 1) & 3)) * 16);
          asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(stage_addr + off), "r"(packed[4 * q]),
                       "r"(packed[4 * q + 1]), "r"(packed[4 * q + 2]), "r"(packed[4 * q + 3])
                       : "memory");
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && n0 < N && row_base < M) {
          tma_store_2d(&tmap_d, stage_buf, n0, row_base);
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait0();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace mxq
