// gemm_pair.cuh -- the block-scaled GEMM (gemm_common.cuh) for M > 128 with a pair of
// CTAs (a two-CTA thread-block cluster on two SMs) per 256 x 192 output tile.
//
// One tcgen05.mma.cta_group::2 of M = 256, N = 192 spans both SMs: CTA r holds rows
// [128r, 128r + 128) of the A tile and rows [96r, 96r + 96) of the B tile (its N
// half), its own A-row scales and the scales of all 192 B rows, and accumulates
// D[its 128 rows][192] in its own TMEM.  Compared with one CTA per 128-row tile, each
// SM moves half the B operand per MMA clock out of L2 and through shared memory.
//
// B scales of an odd weight tile: rows [192 nt, 192 nt + 192) start 64 rows into a
// 128-row scale atom.  The two covering atoms land in TMEM as 8 columns, one column per
// 32 rows, so the MMA reads that tile's scales from 2 columns further on.
//
// Protocol (one elected thread per role):
//   producer (warp 0, both CTAs)   waits its own `empty[s]`, loads its halves with
//                                  TMA whose completion is counted on the LEADER's
//                                  `full[s]`; the leader alone arms `full[s]` with
//                                  the bytes of both CTAs.
//   MMA (warp 1, leader CTA only)  waits `full[s]`, copies the scale atoms of both
//                                  CTAs into their TMEMs (tcgen05.cp.cta_group::2),
//                                  issues 4 MMAs, commits to `empty[s]` of both CTAs;
//                                  after the K loop commits to `acc_full[a]` of both.
//   epilogue (warps 2..9, both)    drain their CTA's accumulator, arrive on the
//                                  LEADER's barriers, then scale / bias / round and
//                                  store their 128 rows.
//
// Two disjoint 192-column accumulators (TMEM columns [0, 192) and [192, 384)) beside the
// scale columns: tiles alternate between them, so the next tile's MMAs wait only for the
// drain of the tile two back (`acc_free[a]`), which the epilogue finished long before,
// and the tensor pipe never idles at a tile boundary.  (256-column tiles would need two
// accumulators sharing columns and a hand-off wait that cost 10 % of the mainloop.)
// Every wait is bounded (ptx.cuh); the CTAs leave only after a final cluster
// barrier, so neither frees TMEM or shared memory the pair's MMAs may still use.
// The kernel is launched with programmatic stream serialisation (griddep_wait below).
#pragma once

#include "gemm_common.cuh"

namespace mxq {

constexpr int kPairStages = 7;
__device__ __forceinline__ constexpr uint32_t pair_acc_col(uint32_t a) { return a * kBN; }
constexpr uint32_t kPairSfa = 2 * kBN;       // A scales: 2 parities x 2 atoms x 4 columns
constexpr uint32_t kPairSfb = kPairSfa + 16; // B scales: 2 parities x 2 atoms x 8 columns (to 432)
static_assert(kPairSfb + 32 <= kTmemCols, "accumulators and scales exceed TMEM");

template <bool kW4A8>
struct PairShape {
  static constexpr int kBK = kW4A8 ? 128 : 256;        // K elements per stage: 128 bytes per row
  static constexpr int kAtoms = kBK / 128;             // scale atoms per stage
  static constexpr int kMmaK = kW4A8 ? 32 : 64;
  static constexpr int kMmas = kBK / kMmaK;            // MMAs per stage (4)
  static constexpr int kMmaPerAtom = 128 / kMmaK;
  static constexpr int kAStage = 128 * 128;            // this CTA's 128 A rows
  static constexpr int kBRows = kBN / 2;               // this CTA's B rows
  static constexpr int kBStage = kBRows * 128;         // (8-bit containers for W4A8)
  static constexpr int kSfaStage = kW4A8 ? 0 : kAtoms * 512;
  static constexpr int kSfbStage = 2 * kAtoms * 512;   // [B row tile j][atom a], both halves of N
  static constexpr int kSfaConst = kW4A8 ? 512 : 0;
  static constexpr uint32_t kTxPerCta =
      128 * 128 + (kW4A8 ? kBRows * 64 : kBRows * 128) + kSfaStage + kSfbStage;  // unpacked FP4 counts packed bytes
  static constexpr int kSmemBytes = 1024 + kPairStages * (kAStage + kBStage + kSfaStage + kSfbStage) + kSfaConst + 256;
  static constexpr uint32_t kIdesc = (kW4A8 ? (0u << 7) | (5u << 10) : (1u << 7) | (1u << 10)) |
                                     (static_cast<uint32_t>(kBN >> 3) << 17) | (1u << 23) |
                                     (static_cast<uint32_t>(256 >> 4) << 24);
};

template <bool kW4A8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    mx_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                        const __grid_constant__ CUtensorMap tmap_sfa, const __grid_constant__ CUtensorMap tmap_sfb,
                        __nv_bfloat16* __restrict__ d, int64_t ldd, int d_vec32,
                        const __nv_bfloat16* __restrict__ bias, int M, int N, int K, float alpha) {
  using S = PairShape<kW4A8>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + kPairStages * S::kAStage;
  uint8_t* sSfa = sB + kPairStages * S::kBStage;
  uint8_t* sSfb = sSfa + kPairStages * S::kSfaStage + S::kSfaConst;
  uint64_t* full = reinterpret_cast<uint64_t*>(sSfb + kPairStages * S::kSfbStage);
  uint64_t* empty = full + kPairStages;
  uint64_t* acc_full = empty + kPairStages;  // [2]
  uint64_t* acc_free = acc_full + 2;         // [2], leader's used
  uint64_t* drain = acc_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int m_tiles = (M + 255) / 256;
  const int n_tiles = (N + kBN - 1) / kBN;
  const int num_tiles = m_tiles * n_tiles;
  const int k_stages = (K + S::kBK - 1) / S::kBK;
  const int cluster = static_cast<int>(cluster_id_x());
  const int nclusters = static_cast<int>(num_clusters_x());

  if (threadIdx.x == 0) {
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    prefetch_tmap(&tmap_sfa);
    prefetch_tmap(&tmap_sfb);
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_free[a], 2 * kEpiWarps);  // every epilogue warp of both CTAs
    }
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
  // Launched with programmatic stream serialisation: everything above, and an L2
  // prefetch of the first weight stages, may overlap the kernel before this one (the
  // activation quantiser); nothing that kernel may write is read before griddep_wait.
  if (warp == 0 && lane == 0 && cluster < num_tiles) {
    const int nt = cluster % n_tiles;
    const int pre = kPairStages < k_stages ? kPairStages : k_stages;
    for (int s = 0; s < pre; ++s) {
      tma_prefetch_2d(&tmap_b, s * 128, nt * kBN + static_cast<int>(rank) * S::kBRows);
      tma_prefetch_4d(&tmap_sfb, 0, 0, s * S::kAtoms, nt * kBN / 128);
    }
  }
  griddep_wait();

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer (both CTAs)
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      const uint64_t keep = l2_policy_evict_last();  // weights: reused by every row tile
      // W4A4 activations: a row tile is read by the ~74 concurrent tiles of its row within
      // about one tile period and never again; evict-first keeps it from displacing the
      // weights (Wan FFN step +1.5 %).  The FP8 activations of the W4A8 path are loaded
      // without a policy: on the FLUX shapes (11 MB of activations, 48-64 weight tiles per
      // row tile) evict-first made the GEMMs 8 % slower, an explicit evict-normal 4 %.
      const uint64_t once = l2_policy_evict_first();
      for (int tile = cluster; tile < num_tiles; tile += nclusters) {
        const int mt = tile / n_tiles, nt = tile % n_tiles;
        bool ok = true;
        for (int ks = 0; ks < k_stages; ++ks) {
          if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(&full[stage], 2u * S::kTxPerCta);
          const uint32_t bar = map_to_rank(&full[stage], 0);
          if (kW4A8)
            tma_load_2d_pair(sA + stage * S::kAStage, &tmap_a, ks * 128, mt * 256 + rank * 128, bar);
          else
            tma_load_2d_pair_hint(sA + stage * S::kAStage, &tmap_a, ks * 128, mt * 256 + rank * 128, bar, once);
          tma_load_2d_pair_hint(sB + stage * S::kBStage, &tmap_b, ks * 128, nt * kBN + rank * S::kBRows, bar, keep);
          if (!kW4A8)
            tma_load_4d_pair(sSfa + stage * S::kSfaStage, &tmap_sfa, 0, 0, ks * S::kAtoms, 2 * mt + rank, bar);
          // the two 128-row scale atoms that cover the tile's B rows
          tma_load_4d_pair(sSfb + stage * S::kSfbStage, &tmap_sfb, 0, 0, ks * S::kAtoms, nt * kBN / 128, bar);
          if (++stage == kPairStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (leader CTA)
    if (leader && elect_one()) {
      int stage = 0;
      uint32_t phase = 0, sf_par = 0;
      bool ok = true;
      bool first = true;
      uint32_t it = 0;  // this cluster's tile count: accumulator it & 1, its use it >> 1
      for (int tile = cluster; ok && tile < num_tiles; tile += nclusters, ++it) {
        const uint32_t a_idx = it & 1u;
        if (!mbar_wait(&acc_free[a_idx], ((it >> 1) & 1u) ^ 1u)) { ok = false; break; }  // drained 2 tiles ago
        tc_fence_after();
        const uint32_t acc_col = pair_acc_col(a_idx);
        // first B row of the tile within its first scale atom, in 32-row TMEM columns (0 or 2)
        const uint32_t sfb_shift = static_cast<uint32_t>((tile % n_tiles) * kBN % 128) / 32u;
        for (int ks = 0; ks < k_stages; ++ks) {
          if (!mbar_wait(&full[stage], phase)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sfa_base = kW4A8 ? kPairSfa : kPairSfa + sf_par * (S::kAtoms * 4);
          const uint32_t sfb_base = kPairSfb + sf_par * (S::kAtoms * 8);
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
          if (kW4A8 && first) tc_cp_sf_atom_pair(tmem + kPairSfa, smem_desc(smem_u32(sSfa), 0, 128, 0));
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
            const uint32_t tsfa = kW4A8 ? tmem + kPairSfa : tmem + sfa_base + 4 * a;
            const uint32_t tsfb = tmem + sfb_base + 8 * a + sfb_shift;
            if (kW4A8)
              tc_mma_mxf8f6f4_pair(tmem + acc_col, adesc, bdesc, idesc, tsfa, tsfb, (ks | kk) != 0);
            else
              tc_mma_mxf4_pair(tmem + acc_col, adesc, bdesc, idesc, tsfa, tsfb, (ks | kk) != 0);
          }
          tc_commit_pair(&empty[stage], 0x3);
          if (++stage == kPairStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc_commit_pair(&acc_full[a_idx], 0x3);
      }
      if (!ok) {
        tc_commit_pair(drain, 0x1);
        mbar_wait_drain(drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    // Thread `lane` of warp (quad, chalf) owns output row 32*quad + lane of its CTA's
    // 128 rows and columns [96*chalf, +96) of the tile: it loads all 96 accumulator
    // columns, releases the accumulator, then scales, rounds and stores them.
    constexpr int kCols = kBN / 2;
    const int ew = warp - 2;
    const int quad = warp & 3;
    const int chalf = ew >> 2;
    const uint32_t acc_free_leader0 = map_to_rank(&acc_free[0], 0);
    const uint32_t acc_free_leader1 = map_to_rank(&acc_free[1], 0);
    const uint64_t stream_out = l2_policy_evict_first();
    uint32_t it = 0;
    for (int tile = cluster; tile < num_tiles; tile += nclusters, ++it) {
      const int mt = tile / n_tiles, nt = tile % n_tiles;
      const uint32_t a_idx = it & 1u;
      // warp-uniform wait: tcgen05.ld below is .sync.aligned
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[a_idx], (it >> 1) & 1u))) break;
      tc_fence_after();
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quad * 32) << 16) + pair_acc_col(a_idx) + chalf * kCols;
      uint32_t v[kCols];
      tmem_ld64(taddr, *reinterpret_cast<uint32_t(*)[64]>(v));
      tmem_ld32(taddr + 64, *reinterpret_cast<uint32_t(*)[32]>(v + 64));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(a_idx ? acc_free_leader1 : acc_free_leader0);
      const int row = mt * 256 + static_cast<int>(rank) * 128 + quad * 32 + lane;
      if (row >= M) continue;
      __nv_bfloat16* drow = d + static_cast<int64_t>(row) * ldd;
#pragma unroll
      for (int c = 0; c < kCols / 32; ++c) {
        const int n0 = nt * kBN + chalf * kCols + 32 * c;
        if (n0 >= N) continue;
        uint32_t packed[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          float b0 = 0.f, b1 = 0.f;
          if (bias != nullptr) {
            const int n = n0 + 2 * j;
            if (n < N) b0 = __bfloat162float(bias[n]);
            if (n + 1 < N) b1 = __bfloat162float(bias[n + 1]);
          }
          const float v0 = __fmaf_rn(alpha, __uint_as_float(v[32 * c + 2 * j]), b0);
          const float v1 = __fmaf_rn(alpha, __uint_as_float(v[32 * c + 2 * j + 1]), b1);
          packed[j] = pack_bf16x2(v0, v1);
        }
        if (d_vec32 && n0 + 32 <= N) {
          st_global_v8_hint(drow + n0, packed, stream_out);
          st_global_v8_hint(drow + n0 + 16, packed + 8, stream_out);
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = n0 + 2 * j;
            if (n + 1 < N)
              *reinterpret_cast<uint32_t*>(drow + n) = packed[j];
            else if (n < N)
              *reinterpret_cast<uint16_t*>(drow + n) = static_cast<uint16_t>(packed[j] & 0xFFFFu);
          }
        }
      }
    }
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
