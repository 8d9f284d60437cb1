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
//               latency).  Mt (the tokens rounded up to 16) is a template parameter.
//   warp 1      MMA issuer: tcgen05.cp of the scale atoms, 4 MMAs of M = 128,
//               N = Mt per stage, rotating over up to 4 adjacent TMEM accumulators
//               [128 weight rows][Mt].  MMAs into one accumulator form a dependency
//               chain whose latency, not the tensor pipe, sets the pace when N is
//               this small (one accumulator at Mt = 16: ~390 ns per stage with the
//               weights in L2, more than the ~340 ns HBM needs to deliver a stage);
//               independent accumulators overlap it.  All accumulators together span
//               at most 128 columns.
//   warps 2..5  epilogue: lane = weight row n, columns = tokens m; every accumulator
//               column loaded with a single wait, summed in FP32, alpha * sum +
//               bias[n] -> BF16 into a shared-memory tile D[Mt][128], which one TMA
//               tensor store writes out (clipped at M and N).  Storing the same values
//               with one 64-byte warp store per output row took ~29 ns a row.
#pragma once

#include "gemm_common.cuh"

namespace mxq {

constexpr int kSwapMaxStages = 16;
constexpr int kSwapThreads = 192;  // 6 warps
constexpr uint32_t kSwapTmemCols = 256;
constexpr uint32_t kSwapAcc = 0;     // accumulators: columns [0, 128), Mt columns each
constexpr uint32_t kSwapSfw = 128;   // weight scales: 2 parities x 2 atoms x 4 columns
constexpr uint32_t kSwapSft = 144;   // token scales:  2 parities x 2 atoms x 4 columns
// independent accumulators for Mt token columns: 4 at Mt <= 32, 2 at Mt <= 64, else 1
__host__ __device__ constexpr int swap_accs(int Mt) { return Mt <= 32 ? 4 : Mt <= 64 ? 2 : 1; }

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
  __host__ __device__ static constexpr int out_bytes(int Mt) { return Mt * 128 * 2; }  // BF16 output tile [Mt][128]
  static constexpr uint32_t kWTx = kW4A8 ? 128 * 64 : 128 * 128;  // unpacked FP4 counts packed bytes
  // A = weights (E2M1), B = tokens (E2M1 / E4M3); M = 128, N set at run time.
  static constexpr uint32_t kIdescBase =
      (kW4A8 ? (5u << 7) | (0u << 10) : (1u << 7) | (1u << 10)) | (1u << 23) | (static_cast<uint32_t>(128 >> 4) << 24);
  // One stage for Mt token rows (Mt % 16 == 0 keeps every tile 1 KB aligned).
  static constexpr int stage_bytes(int Mt) { return kWStage + Mt * 128 + kSfwStage + kSftStage; }
};

template <bool kW4A8, int Mt>
__global__ void __launch_bounds__(kSwapThreads, 1)
    mx_gemm_swap_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_t,
                        const __grid_constant__ CUtensorMap tmap_sfw, const __grid_constant__ CUtensorMap tmap_sft,
                        const __grid_constant__ CUtensorMap tmap_d, const __nv_bfloat16* __restrict__ bias, int M,
                        int N, int K, float alpha, int stages) {
  using S = SwapShape<kW4A8>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // MMA N = Mt: the tokens rounded up to 16 (rows beyond M are zero-filled)
  static_assert(Mt % 16 == 0 && Mt >= 16 && Mt <= 128, "token tile");
  constexpr int kAccs = swap_accs(Mt);
  constexpr int kAccCols = kAccs * Mt;
  static_assert(kAccCols <= static_cast<int>(kSwapSfw), "accumulators overlap the scale columns");
  constexpr int kTStage = Mt * 128;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sD = smem;  // output tile, BF16 [Mt][128]
  uint8_t* sW = sD + S::out_bytes(Mt);
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

  // First of all, an L2 prefetch of the first weight stages (as many as the ring holds):
  // the weight stream from HBM starts while the prologue below runs.  A prefetch is only a
  // hint: the loads later read whatever memory holds.
  if (threadIdx.x == 32 && static_cast<int>(blockIdx.x) < num_tiles) {
    const int pre = stages < k_stages ? stages : k_stages;
    for (int s = 0; s < pre; ++s) {
      tma_prefetch_2d(&tmap_w, s * 128, blockIdx.x * 128);
      tma_prefetch_4d(&tmap_sfw, 0, 0, s * S::kAtoms, blockIdx.x);
    }
  }
  if (threadIdx.x == 0) {
    prefetch_tmap(&tmap_w);
    prefetch_tmap(&tmap_t);
    prefetch_tmap(&tmap_sfw);
    if (!kW4A8) prefetch_tmap(&tmap_sft);
    prefetch_tmap(&tmap_d);
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
  // Launched with programmatic stream serialisation: everything above, and the L2
  // prefetch of the first weight stages issued at entry, may overlap the kernel before this
  // one (the activation quantiser); nothing that kernel may write is read before
  // griddep_wait.
  griddep_wait();

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
      constexpr uint32_t naccs = static_cast<uint32_t>(kAccs);
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        if (!mbar_wait(acc_free, acc_phase ^ 1)) { ok = false; break; }
        tc_fence_after();
        uint32_t g = 0, acc = 0;  // MMAs issued for this tile; accumulator g % naccs
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
            const uint32_t tacc = tmem + kSwapAcc + acc * static_cast<uint32_t>(Mt);
            if (kW4A8)
              tc_mma_mxf8f6f4(tacc, wdesc, tdesc, idesc, tsfw, tsft, g >= naccs);
            else
              tc_mma_mxf4(tacc, wdesc, tdesc, idesc, tsfw, tsft, g >= naccs);
            ++g;
            if (++acc == naccs) acc = 0;
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
    const bool store_thread = warp == 2 && lane == 0;
    // the four epilogue warps only (named barrier 1)
    auto epilogue_bar_sync = [] { asm volatile("bar.sync 1, 128;" ::: "memory"); };
    // true for all 128 epilogue threads iff it is true for each of them, so that they
    // leave the loop together and none is left waiting at the barrier above
    auto epilogue_all = [](bool ok) {
      uint32_t r;
      asm volatile(
          "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
          "bar.red.and.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
          : "=r"(r)
          : "r"(static_cast<uint32_t>(ok))
          : "memory");
      return r != 0u;
    };
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      if (!epilogue_all(mbar_wait(acc_full, acc_phase))) break;
      tc_fence_after();
      const int n = tile * 128 + quad * 32 + lane;
      const float b = (bias != nullptr && n < N) ? __bfloat162float(bias[n]) : 0.f;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quad * 32) << 16) + kSwapAcc;
      uint32_t v[kAccCols];  // accumulator a, token m at v[a * Mt + m]
#pragma unroll
      for (int c = 0; c < kAccCols / 16; ++c) tmem_ld16(taddr + 16 * c, v + 16 * c);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_free);
      // the previous tile's store has finished reading the output tile
      if (store_thread) bulk_wait_read0();
      epilogue_bar_sync();
      uint16_t* out = reinterpret_cast<uint16_t*>(sD) + quad * 32 + lane;  // column n - 128 tile
#pragma unroll
      for (int m = 0; m < Mt; ++m) {
        float sum = __uint_as_float(v[m]);
#pragma unroll
        for (int a = 1; a < kAccs; ++a) sum = __fadd_rn(sum, __uint_as_float(v[a * Mt + m]));
        out[m * 128] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmaf_rn(alpha, sum, b)));
      }
      fence_proxy_async_smem();
      epilogue_bar_sync();
      if (store_thread) {
        tma_store_2d(&tmap_d, sD, tile * 128, 0);
        bulk_commit();
      }
      acc_phase ^= 1;
    }
    if (store_thread) bulk_wait0();  // the output is written before the CTA leaves
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kSwapTmemCols);
  }
}

}  // namespace mxq
