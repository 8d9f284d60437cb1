// gemm_pair.cuh -- the block-scaled GEMM of gemm.cuh with a pair of CTAs (a
// two-CTA thread-block cluster on two SMs) per 256 x 256 output tile.
//
// One tcgen05.mma.cta_group::2 of M = 256 spans both SMs: CTA r holds rows
// [128r, 128r + 128) of the A tile and of the B tile (the N half), its own A-row
// scales and all 256 B-row scales, and accumulates D[its 128 rows][256] in its own
// TMEM.  Compared with one CTA per 128 x 256 tile, each SM moves 64 instead of 96
// bytes of operands per MMA clock out of L2 and through shared memory, and a stage
// is 35 KB instead of 51 KB, so the ring is deeper.
//
// Protocol (one elected thread per role):
//   producer (warp 0, both CTAs)   waits its own `empty[s]`, loads its halves with
//                                  TMA whose completion is counted on the LEADER's
//                                  `full[s]`; the leader alone arms `full[s]` with
//                                  the bytes of both CTAs.
//   MMA (warp 1, leader CTA only)  waits `full[s]`, copies the scale atoms of both
//                                  CTAs into their TMEMs (tcgen05.cp.cta_group::2),
//                                  issues 4 MMAs, commits to `empty[s]` of both CTAs;
//                                  after the K loop commits to `tmem_full` of both.
//   epilogue (warps 2..9, both)    drain their CTA's accumulator, arrive on the
//                                  LEADER's `tmem_empty` (16 arrivals per tile), then
//                                  scale / bias / round and TMA-store their 128 rows.
// Every wait is bounded as in gemm.cuh; the CTAs leave only after a final cluster
// barrier, so neither frees TMEM or shared memory the pair's MMAs may still use.
#pragma once

#include "gemm.cuh"

namespace mxq {

constexpr int kPairStages = 5;

template <bool kW4A8>
struct PairShape {
  static constexpr int kBK = kW4A8 ? 128 : 256;        // K elements per stage: 128 bytes per row
  static constexpr int kAtoms = kBK / 128;             // scale atoms per stage
  static constexpr int kMmaK = kW4A8 ? 32 : 64;
  static constexpr int kMmas = kBK / kMmaK;            // MMAs per stage (4)
  static constexpr int kMmaPerAtom = 128 / kMmaK;
  static constexpr int kAStage = 128 * 128;            // this CTA's 128 A rows
  static constexpr int kBStage = 128 * 128;            // this CTA's 128 B rows (8-bit containers for W4A8)
  static constexpr int kSfaStage = kW4A8 ? 0 : kAtoms * 512;
  static constexpr int kSfbStage = 2 * kAtoms * 512;   // [B row tile j][atom a], both halves of N
  static constexpr int kSfaConst = kW4A8 ? 512 : 0;
  static constexpr uint32_t kTxPerCta =
      128 * 128 + (kW4A8 ? 128 * 64 : 128 * 128) + kSfaStage + kSfbStage;  // unpacked FP4 counts packed bytes
  static constexpr int kSmemBytes = 1024 + kPairStages * (kAStage + kBStage + kSfaStage + kSfbStage) + kSfaConst +
                                    kEpiWarps * kEpiStageBytes + 256;
  static constexpr uint32_t kIdesc = (kW4A8 ? (0u << 7) | (5u << 10) : (1u << 7) | (1u << 10)) |
                                     (static_cast<uint32_t>(256 >> 3) << 17) | (1u << 23) |
                                     (static_cast<uint32_t>(256 >> 4) << 24);
};

template <bool kW4A8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    mx_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                        const __grid_constant__ CUtensorMap tmap_sfa, const __grid_constant__ CUtensorMap tmap_sfb,
                        const __grid_constant__ CUtensorMap tmap_d, const __nv_bfloat16* __restrict__ bias, int M,
                        int N, int K, float alpha) {
  using S = PairShape<kW4A8>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + kPairStages * S::kAStage;
  uint8_t* sEpi = sB + kPairStages * S::kBStage;
  uint8_t* sSfa = sEpi + kEpiWarps * kEpiStageBytes;
  uint8_t* sSfb = sSfa + kPairStages * S::kSfaStage + S::kSfaConst;
  uint64_t* full = reinterpret_cast<uint64_t*>(sSfb + kPairStages * S::kSfbStage);
  uint64_t* empty = full + kPairStages;
  uint64_t* tmem_full = empty + kPairStages;
  uint64_t* tmem_empty = tmem_full + 1;
  uint64_t* drain = tmem_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int m_tiles = (M + 255) / 256;
  const int n_tiles = (N + 255) / 256;
  const int num_tiles = m_tiles * n_tiles;
  const int k_stages = (K + S::kBK - 1) / S::kBK;
  const int cluster = static_cast<int>(cluster_id_x());
  const int nclusters = static_cast<int>(num_clusters_x());

  if (threadIdx.x == 0) {
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    prefetch_tmap(&tmap_sfa);
    prefetch_tmap(&tmap_sfb);
    prefetch_tmap(&tmap_d);
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, 2 * kEpiWarps);
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (kW4A8 && warp >= 2 && warp < 6) {
    reinterpret_cast<uint32_t*>(sSfa)[threadIdx.x - 64] = 0x7F7F7F7Fu;  // unit E8M0 scales
    fence_proxy_async_smem();
  }
  cluster_sync();  // both CTAs' barriers exist before anything signals across the pair
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs hold their TMEM before the leader's first MMA
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer (both CTAs)
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = cluster; tile < num_tiles; tile += nclusters) {
        const int mt = tile / n_tiles, nt = tile % n_tiles;
        bool ok = true;
        for (int ks = 0; ks < k_stages; ++ks) {
          if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(&full[stage], 2u * S::kTxPerCta);
          const uint32_t bar = map_to_rank(&full[stage], 0);
          tma_load_2d_pair(sA + stage * S::kAStage, &tmap_a, ks * 128, mt * 256 + rank * 128, bar);
          tma_load_2d_pair(sB + stage * S::kBStage, &tmap_b, ks * 128, nt * 256 + rank * 128, bar);
          if (!kW4A8)
            tma_load_4d_pair(sSfa + stage * S::kSfaStage, &tmap_sfa, 0, 0, ks * S::kAtoms, 2 * mt + rank, bar);
          tma_load_4d_pair(sSfb + stage * S::kSfbStage, &tmap_sfb, 0, 0, ks * S::kAtoms, 2 * nt, bar);
          if (++stage == kPairStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (leader CTA)
    if (leader && elect_one()) {
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0, sf_par = 0;
      bool ok = true;
      bool first = true;
      for (int tile = cluster; ok && tile < num_tiles; tile += nclusters) {
        if (!mbar_wait(tmem_empty, acc_phase ^ 1)) { ok = false; break; }
        tc_fence_after();
        for (int ks = 0; ks < k_stages; ++ks) {
          if (!mbar_wait(&full[stage], phase)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sfa_base = kW4A8 ? kSfaCol : kSfaCol + sf_par * (S::kAtoms * 4);
          const uint32_t sfb_base = kSfbCol + sf_par * (S::kAtoms * 8);
          sf_par ^= 1u;
#pragma unroll
          for (int a = 0; a < S::kAtoms; ++a) {
            if (!kW4A8)
              tc_cp_sf_atom_pair(tmem + sfa_base + 4 * a,
                                 smem_desc(smem_u32(sSfa + stage * S::kSfaStage + a * 512), 0, 128, 0));
#pragma unroll
            for (int j = 0; j < 2; ++j)
              tc_cp_sf_atom_pair(tmem + sfb_base + 8 * a + 4 * j,
                                 smem_desc(smem_u32(sSfb + stage * S::kSfbStage + j * S::kAtoms * 512 + a * 512),
                                           0, 128, 0));
          }
          if (kW4A8 && first) tc_cp_sf_atom_pair(tmem + kSfaCol, smem_desc(smem_u32(sSfa), 0, 128, 0));
          first = false;
          const uint32_t a_base = smem_u32(sA + stage * S::kAStage);
          const uint32_t b_base = smem_u32(sB + stage * S::kBStage);
#pragma unroll
          for (int kk = 0; kk < S::kMmas; ++kk) {
            const int a = kk / S::kMmaPerAtom;
            const uint32_t sf_id = kW4A8 ? static_cast<uint32_t>(kk % S::kMmaPerAtom)
                                         : static_cast<uint32_t>((kk % S::kMmaPerAtom) * 2);
            const uint32_t idesc = S::kIdesc | (sf_id << 29) | (sf_id << 4);
            const uint64_t adesc = smem_desc(a_base + kk * 32, 16, 1024, 2);
            const uint64_t bdesc = smem_desc(b_base + kk * 32, 16, 1024, 2);
            const uint32_t tsfa = kW4A8 ? tmem + kSfaCol : tmem + sfa_base + 4 * a;
            const uint32_t tsfb = tmem + sfb_base + 8 * a;
            if (kW4A8)
              tc_mma_mxf8f6f4_pair(tmem + kAccCol, adesc, bdesc, idesc, tsfa, tsfb, (ks | kk) != 0);
            else
              tc_mma_mxf4_pair(tmem + kAccCol, adesc, bdesc, idesc, tsfa, tsfb, (ks | kk) != 0);
          }
          tc_commit_pair(&empty[stage], 0x3);
          if (++stage == kPairStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc_commit_pair(tmem_full, 0x3);
        acc_phase ^= 1;
      }
      if (!ok) {
        tc_commit_pair(drain, 0x1);
        mbar_wait_drain(drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    const int ew = warp - 2;
    const int quad = warp & 3;
    const int chalf = ew >> 2;
    uint8_t* stage_buf = sEpi + ew * kEpiStageBytes;
    const uint32_t stage_addr = smem_u32(stage_buf);
    const uint32_t tmem_empty_leader = map_to_rank(tmem_empty, 0);
    uint32_t acc_phase = 0;
    for (int tile = cluster; tile < num_tiles; tile += nclusters) {
      const int mt = tile / n_tiles, nt = tile % n_tiles;
      if (!mbar_wait(tmem_full, acc_phase)) break;
      tc_fence_after();
      uint32_t acc[4][32];
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quad * 32) << 16) + kAccCol + chalf * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(taddr + 32 * c, acc[c]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tmem_empty_leader);
      acc_phase ^= 1;

      const int row_base = mt * 256 + static_cast<int>(rank) * 128 + quad * 32;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int n0 = nt * 256 + chalf * 128 + 32 * c;
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
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace mxq
