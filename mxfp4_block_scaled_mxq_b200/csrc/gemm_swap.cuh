// gemm_swap.cuh -- the block-scaled GEMM for few tokens (M <= 128), computed as
// D^T = W X^T: the weights are the MMA's 128-row operand and the M tokens its N
// side (16..128), so the work spreads over N / 128 CTAs (108 for N = 13824) that
// stream the weights at HBM speed -- the weight-streaming regime of the layer.
//
// One CTA per 128-row weight tile, persistent if there are more tiles than SMs:
//   warp 0      TMA producer: weight tile (128 rows x 128 B), token tile (Mt rows x
//               128 B), the weight tile's and the token tile's scale atoms (4-D
//               boxes); the ring is as deep as shared memory allows for this Mt (up
//               to 16 stages: the weights come from HBM, so depth is what hides the
//               latency).
//   warp 1      MMA issuer: tcgen05.cp of the scale atoms, 4 MMAs of M = 128,
//               N = Mt per stage into a TMEM accumulator [128 weight rows][Mt].
//   warps 2..5  epilogue: lane = weight row n, columns = tokens m; alpha * acc +
//               bias[n] -> BF16, stored so that a warp writes 32 consecutive n of
//               one output row (64 contiguous bytes) per instruction.
#pragma once

#include "gemm_common.cuh"

namespace mxq {

constexpr int kSwapMaxStages = 16;
constexpr int kSwapThreads = 192;  // 6 warps
constexpr uint32_t kSwapTmemCols = 256;
constexpr uint32_t kSwapAcc = 0;     // accumulator: columns [0, 128)
constexpr uint32_t kSwapSfw = 128;   // weight scales: 2 parities x 2 atoms x 4 columns
constexpr uint32_t kSwapSft = 144;   // token scales:  2 parities x 2 atoms x 4 columns

template <bool kW4A8>
struct SwapShape {
  static constexpr int kBK = kW4A8 ? 128 : 256;
  static constexpr int kAtoms = kBK / 128;
  static constexpr int kMmaK = kW4A8 ? 32 : 64;
  static constexpr int kMmas = kBK / kMmaK;
  static constexpr int kMmaPerAtom = 128 / kMmaK;
  static constexpr int kWStage = 128 * 128;            // weight rows (8-bit containers for W4A8)
  static constexpr int kSfwStage = kAtoms * 512;
  static constexpr int kSftStage = kW4A8 ? 0 : kAtoms * 512;
  static constexpr int kSftConst = kW4A8 ? 512 : 0;    // unit scales for E4M3 tokens
  static constexpr int kFixedBytes = 1024 /*alignment slack*/ + kSftConst + 512 /*34 barriers + TMEM slot*/;
  static constexpr uint32_t kWTx = kW4A8 ? 128 * 64 : 128 * 128;  // unpacked FP4 counts packed bytes
  // A = weights (E2M1), B = tokens (E2M1 / E4M3); M = 128, N set at run time.
  static constexpr uint32_t kIdescBase =
      (kW4A8 ? (5u << 7) | (0u << 10) : (1u << 7) | (1u << 10)) | (1u << 23) | (static_cast<uint32_t>(128 >> 4) << 24);
  // One stage for Mt token rows (Mt % 16 == 0 keeps every tile 1 KB aligned).
  static constexpr int stage_bytes(int Mt) { return kWStage + Mt * 128 + kSfwStage + kSftStage; }
};

template <bool kW4A8>
__global__ void __launch_bounds__(kSwapThreads, 1)
    mx_gemm_swap_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_t,
                        const __grid_constant__ CUtensorMap tmap_sfw, const __grid_constant__ CUtensorMap tmap_sft,
                        __nv_bfloat16* __restrict__ d, int64_t ldd, const __nv_bfloat16* __restrict__ bias, int M,
                        int N, int K, float alpha, int stages) {
  using S = SwapShape<kW4A8>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int Mt = (M + 15) / 16 * 16;  // MMA N: tokens rounded up to 16 (rows beyond M are zero-filled)
  const int kTStage = Mt * 128;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sW = smem;
  uint8_t* sT = sW + stages * S::kWStage;
  uint8_t* sSfw = sT + stages * kTStage;
  uint8_t* sSft = sSfw + stages * S::kSfwStage;  // + the unit atom for W4A8
  uint64_t* full = reinterpret_cast<uint64_t*>(sSft + stages * S::kSftStage + S::kSftConst);
  uint64_t* empty = full + kSwapMaxStages;
  uint64_t* acc_full = empty + kSwapMaxStages;
  uint64_t* acc_free = acc_full + 1;
  uint64_t* drain = acc_free + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_tiles = (N + 127) / 128;
  const int k_stages = (K + S::kBK - 1) / S::kBK;
  const uint32_t t_bytes = static_cast<uint32_t>(Mt) * 128u;

  if (threadIdx.x == 0) {
    prefetch_tmap(&tmap_w);
    prefetch_tmap(&tmap_t);
    prefetch_tmap(&tmap_sfw);
    if (!kW4A8) prefetch_tmap(&tmap_sft);
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_free, 4);
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (kW4A8 && warp >= 2) {
    reinterpret_cast<uint32_t*>(sSft)[threadIdx.x - 64] = 0x7F7F7F7Fu;  // unit E8M0 scales, 128 words
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kSwapTmemCols);
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
      uint32_t issued = 0, issued_phase = 0;
      bool ok = true;
      const uint32_t tx = S::kWTx + t_bytes + S::kSfwStage + S::kSftStage;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        for (int ks = 0; ks < k_stages; ++ks) {
          if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
          issued |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          mbar_arrive_expect_tx(&full[stage], tx);
          tma_load_2d(sW + stage * S::kWStage, &tmap_w, ks * 128, tile * 128, &full[stage]);
          tma_load_2d(sT + stage * kTStage, &tmap_t, ks * 128, 0, &full[stage]);
          tma_load_4d(sSfw + stage * S::kSfwStage, &tmap_sfw, 0, 0, ks * S::kAtoms, tile, &full[stage]);
          if (!kW4A8) tma_load_4d(sSft + stage * S::kSftStage, &tmap_sft, 0, 0, ks * S::kAtoms, 0, &full[stage]);
          if (++stage == stages) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        for (int s = 0; s < stages; ++s)
          if (issued & (1u << s)) mbar_wait_drain(&full[s], (issued_phase >> s) & 1u);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0, sf_par = 0;
      bool ok = true, first = true;
      const uint32_t idesc_n = S::kIdescBase | (static_cast<uint32_t>(Mt >> 3) << 17);
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        if (!mbar_wait(acc_free, acc_phase ^ 1)) { ok = false; break; }
        tc_fence_after();
        for (int ks = 0; ks < k_stages; ++ks) {
          if (!mbar_wait(&full[stage], phase)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sfw_base = kSwapSfw + sf_par * (S::kAtoms * 4);
          const uint32_t sft_base = kW4A8 ? kSwapSft : kSwapSft + sf_par * (S::kAtoms * 4);
          sf_par ^= 1u;
#pragma unroll
          for (int a = 0; a < S::kAtoms; ++a) {
            tc_cp_sf_atom(tmem + sfw_base + 4 * a, smem_desc(smem_u32(sSfw + stage * S::kSfwStage + a * 512), 0, 128, 0));
            if (!kW4A8)
              tc_cp_sf_atom(tmem + sft_base + 4 * a,
                            smem_desc(smem_u32(sSft + stage * S::kSftStage + a * 512), 0, 128, 0));
          }
          if (kW4A8 && first) tc_cp_sf_atom(tmem + kSwapSft, smem_desc(smem_u32(sSft), 0, 128, 0));
          first = false;
          const uint32_t w_base = smem_u32(sW + stage * S::kWStage);
          const uint32_t t_base = smem_u32(sT + stage * kTStage);
#pragma unroll
          for (int kk = 0; kk < S::kMmas; ++kk) {
            const int a = kk / S::kMmaPerAtom;
            const uint32_t sf_id = kW4A8 ? static_cast<uint32_t>(kk % S::kMmaPerAtom)
                                         : static_cast<uint32_t>((kk % S::kMmaPerAtom) * 2);
            const uint32_t idesc = idesc_n | (sf_id << 29) | (sf_id << 4);
            const uint64_t wdesc = smem_desc(w_base + kk * 32, 16, 1024, 2);
            const uint64_t tdesc = smem_desc(t_base + kk * 32, 16, 1024, 2);
            const uint32_t tsfw = tmem + sfw_base + 4 * a;
            const uint32_t tsft = kW4A8 ? tmem + kSwapSft : tmem + sft_base + 4 * a;
            if (kW4A8)
              tc_mma_mxf8f6f4(tmem + kSwapAcc, wdesc, tdesc, idesc, tsfw, tsft, (ks | kk) != 0);
            else
              tc_mma_mxf4(tmem + kSwapAcc, wdesc, tdesc, idesc, tsfw, tsft, (ks | kk) != 0);
          }
          tc_commit(&empty[stage]);
          if (++stage == stages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc_commit(acc_full);
        acc_phase ^= 1;
      }
      if (!ok) {
        tc_commit(drain);
        mbar_wait_drain(drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2..5)
    const int quad = warp & 3;  // TMEM lanes [32 quad, +32) = weight rows of this warp
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      if (!__all_sync(0xffffffffu, mbar_wait(acc_full, acc_phase))) break;
      tc_fence_after();
      const int n = tile * 128 + quad * 32 + lane;
      const float b = (bias != nullptr && n < N) ? __bfloat162float(bias[n]) : 0.f;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quad * 32) << 16) + kSwapAcc;
      uint32_t v[128];  // token columns [0, Mt) of this lane's weight row
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (32 * c < Mt) tmem_ld32(taddr + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(v + 32 * c));
      tmem_ld_wait();
      if (n < N) {
#pragma unroll
        for (int m = 0; m < 128; ++m)
          if (m < M)
            d[static_cast<int64_t>(m) * ldd + n] = __float2bfloat16_rn(__fmaf_rn(alpha, __uint_as_float(v[m]), b));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_free);
      acc_phase ^= 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kSwapTmemCols);
  }
}

}  // namespace mxq
