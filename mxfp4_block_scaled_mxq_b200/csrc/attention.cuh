// attention.cuh -- MXFP4 attention with the data-free UOS block-scale rule and
// pre-normalisation quantisation (PNQ) of the softmax numerators, on tcgen05.
// [MXAttention: Data-Free Optimal Scaling and Pre-Normalization Quantization for MXFP4
//  Attention -- TL;DR, "Architecture", "What it actually does"]
//
//   O = (deq(P) deq(V)) / l,   P = MXFP4(2^(t - c)),   l = sum_j deq(P)_j,
//   t = fl32(S * log2(e) / sqrt(d)),   S = deq(Q) deq(K)^T,
//
// with Q, K in 32-blocks along the head dimension, V and P in 32-blocks along the keys and
// c an integer offset (a power-of-two factor, under which the E8M0 block scaling is
// exactly equivariant: the codes of P do not depend on it).  The numerators' values are
// never needed, only their MXFP4 codes, and those the kernel decides exactly as the exact
// exponential does (the code cubic below): a block's E8M0 exponent is taken from its largest
// score by integer arithmetic, and each code from a cubic in g = t - rint(t) that crosses
// the four E2M1 decision levels it can meet at the same FP32 g as 2^g does.  The row sum is
// taken over the quantised numerators (PNQ), so the implied weights sum to one by
// construction; it is computed by the tensor core itself: V^T carries one extra row of
// ones, so column d of the P V accumulator is l.
//
// One CTA per (128 queries, head), head dimension 128, 256 keys per tile:
//   warp 0      TMA producer: the Q tile (64-byte swizzle) once; per key tile the K
//               tile (256 x 64 B, 64-byte swizzle), the V^T tile (128 x 128 B, 128-byte
//               swizzle) and their scale atoms (4-D boxes, zero fill past the end).
//   warp 1      MMA issuer: S = Q K^T (M 128, N 256, K 128) into TMEM; for the previous
//               tile, O += P V^T (M 128, N 144: d columns + the ones row, K 256 keys);
//               the next tile's scores are issued before the previous tile's P V, so
//               the tensor core works while the softmax warps quantise.
//   warps 2, 3  idle (their warpgroup hands its registers to the softmax warps)
//   warps 4..19 softmax / PNQ, four threads per query row (64 keys of the tile each):
//               scores from TMEM, the row maximum through shared memory, the
//               offset c raised only when the maximum passes c + 8 (then O, l are
//               rescaled in TMEM by the exact power of two), numerators, UOS/OCP block
//               scales and E2M1 codes written to shared memory in the 128-byte-swizzled
//               operand layout, scale bytes in the 512-byte atom layout; at the end
//               O / l -> BF16.
//
// Every wait is bounded (ptx.cuh); on a timeout the kernel records MXQ_ERR_TIMEOUT,
// drains its own copies and MMAs, and returns.
#pragma once

#include "gemm_common.cuh"
#include "quantize.cuh"

namespace mxq {

constexpr int kAttnD = 128;       // head dimension
constexpr int kAttnBM = 128;      // queries per CTA
constexpr int kAttnBN = 256;      // keys per tile
constexpr int kAttnStages = 3;
constexpr int kAttnThreads = 640;  // producer, MMA, 2 idle warps, 16 softmax warps
// Registers: launched with 96 a thread (640 x 96 = 61440); the control warpgroup (warps
// 0-3) then gives up all but 32 and the four softmax warpgroups take 112: 128 x 32 +
// 512 x 112 = 61440, exactly the launch's total, so the increase always completes.
constexpr int kAttnCtrlRegs = 32;
constexpr int kAttnSoftRegs = 112;
static_assert(128 * kAttnCtrlRegs + 512 * kAttnSoftRegs <= kAttnThreads * 96, "register split");
constexpr int kAttnSoftWarps = 16;  // four per TMEM lane quadrant: keys [64 q, +64) of a tile each
constexpr int kAttnNv = kAttnD + 16;  // P V's N: the d value columns and 16 rows holding the ones row
constexpr uint32_t kAttnTmemCols = 512;
constexpr uint32_t kColS = 0;      // scores, 256 columns
constexpr uint32_t kColO = 256;    // output accumulator, 144 columns (column 128 = l)
constexpr uint32_t kColSfq = 400;  // Q scales, 4 columns
constexpr uint32_t kColSfk = 404;  // K scales: 2 parities x 8 columns (two 128-key row groups)
constexpr uint32_t kColSfp = 420;  // P scales: 2 parities x 2 atoms x 4 columns
constexpr uint32_t kColSfv = 436;  // V^T scales: 2 parities x 2 atoms x 8 columns (values, ones)

// Shared memory (offsets from a 1024-byte aligned base).
constexpr int kAttnQBytes = kAttnBM * 64;                   // 8 KB, 64-byte swizzle
constexpr int kAttnKBytes = kAttnBN * 64;                   // 16 KB, 64-byte swizzle
constexpr int kAttnVBytes = kAttnNv * 128;                  // 18 KB, 128-byte swizzle (+ ones rows)
constexpr int kAttnStageBytes = kAttnKBytes + kAttnVBytes + 1024 /*K scales*/ + 1024 /*V scales*/;
constexpr int kAttnOffSfq = kAttnQBytes;
constexpr int kAttnOffStages = kAttnQBytes + 1024;
constexpr int kAttnOffP = kAttnOffStages + kAttnStages * kAttnStageBytes;
constexpr int kAttnOffSfp = kAttnOffP + kAttnBM * 128;      // 2 atoms
constexpr int kAttnOffSfOnes = kAttnOffSfp + 1024;          // 2 atoms of unit scales
constexpr int kAttnOffRmax = kAttnOffSfOnes + 1024;         // float [2 parities][4 quarters][128]
constexpr int kAttnOffBar = kAttnOffRmax + 4096;
constexpr int kAttnSmemBytes = 1024 + kAttnOffBar + 256;

// Instruction descriptors (kind::mxf4 block_scale, E2M1 x E2M1, UE8M0 scales, K-major).
__host__ __device__ constexpr uint32_t attn_idesc(int n) {
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | (1u << 23) |
         (static_cast<uint32_t>(kAttnBM >> 4) << 24);
}

// The numerators' codes.  A key's scaled numerator is x = 2^(t - c - e) = 2^m 2^g with
// n = rint(t) (ties to even), g = t - n in [-1/2, 1/2] (exact in FP32) and m = n - c - e an
// integer; its E2M1 code is decided by x against the rounding boundaries 0.25, 0.75, 1.25,
// 1.75, 2.5, 3.5 and 5.  With 2^g in [0.707, 1.415] the boundary an octave m can meet sits at
// one of four levels of 2^g: 0.75 (m = 0), 0.875 (m = 1, 2), 1 (m = -2) and 1.25 (m = 0, 1,
// 2); octaves m <= -3 give 0 and m = 3 gives 6 whatever g is.  So a code needs 2^g only on
// the right side of those four levels.  The kernel uses the cubic
//   q(g) = 1 + a1 g + a2 g^2 + a3 g^3  (Horner, FP32 fused multiply-adds, the last step
//   rounded toward +infinity),
// monotone on [-1/2, 1/2] and within 4e-4 of 2^g, whose FP32 coefficients were chosen by
// search so that, for every FP32 g, q(g) reaches 0.75, 0.875 and 1.25 (with the E2M1 tie
// rule of the conversion: a tie at 0.75 or 0.875 goes up, at 1.25 down) exactly when 2^g
// does, i.e. when g passes log2(0.75), log2(0.875), log2(1.25); the rounded-up last step
// makes q(g) > 1 exactly when g > 0.  The codes are therefore those of the exact
// exponential for every key whose block scale lies within the E8M0 range (keys at least
// 2^-126 of the row's largest numerator); only numerators below that are flushed to 0.
constexpr float kCodeA1 = 0x1.63037cp-1f, kCodeA2 = 0x1.ee3f14p-3f, kCodeA3 = 0x1.b23daap-5f;
// log2(0.90625) = log2(7.25 / 8), rounded down to FP32: the UOS rule raises a block's
// exponent when the fraction of its largest t - c exceeds log2(1.8125), i.e. when g lies in
// (log2(0.90625), 0); g > this constant is the exact test (the logarithm is irrational).
constexpr float kUosFracThreshold = -0x1.22dadep-3f;

struct AttnParams {
  float t_scale;   // fl32(log2(e) / sqrt(d))
  int Sq;
  int Skv;
  int num_tiles;   // ceil(Skv / 256)
};

// max(a, b, c) and min(a, b, c) in one instruction each (exact, like fmaxf / fminf; the
// inputs are never NaN).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Scaled code values of a pair of keys: q(g) 2^(n - chat), n = rint(t), g = t - n, q the code
// cubic above (Horner, FP32 fused multiply-adds, the last one rounded up), 0 when n - chat <
// -126.  Everything runs on the FMA pipe: t is first raised to chat - 127 (masked keys at -inf
// and every t whose n - chat would be -127 or less give exactly 0 below); r = t + 1.5 * 2^23
// holds rint(t) in its low mantissa bits (|t| < 2^22), so n = r - 1.5 * 2^23 and g = t - n are
// exact; and the FP32 bit pattern of 2^(n - chat) is (bits(r) + 127 - chat) * 2^23 modulo 2^32
// (bits(1.5 * 2^23) * 2^23 vanishes modulo 2^32), one integer multiply-add, 0 for n - chat = -127.
__device__ __forceinline__ float2 pnq_code_pair(float2 t, float lo, uint32_t bias_bits) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  t = make_float2(fmaxf(t.x, lo), fmaxf(t.y, lo));
  const float2 r = __fadd2_rn(t, make_float2(kMagic, kMagic));
  const float2 n = __fadd2_rn(r, make_float2(-kMagic, -kMagic));
  const float2 g = __fadd2_rn(t, make_float2(-n.x, -n.y));
  float2 p = __ffma2_rn(make_float2(kCodeA3, kCodeA3), g, make_float2(kCodeA2, kCodeA2));
  p = __ffma2_rn(p, g, make_float2(kCodeA1, kCodeA1));
  p = __ffma2_ru(p, g, make_float2(1.0f, 1.0f));
  const float2 sc = make_float2(__uint_as_float(__float_as_uint(r.x) * 8388608u + bias_bits),
                                __uint_as_float(__float_as_uint(r.y) * 8388608u + bias_bits));
  return __fmul2_rn(p, sc);
}

// E8M0 exponent of a block whose largest score is tmax, relative to the offset cp: the MX
// rule applied to the exact largest numerator 2^(tmax - cp), by integer arithmetic on
// n = rint(tmax) and g = tmax - n: floor(tmax - cp) - 2 (OCP), one more under UOS when the
// fraction of tmax - cp exceeds log2(1.8125) (largest numerator above 7.25 2^(e - 2)),
// clamped to -127; -127 for a block with no key at or above cp - 127 (masked keys are -inf).
template <bool kUOS>
__device__ __forceinline__ int pnq_block_exponent(float tmax, int cp) {
  if (!(tmax >= static_cast<float>(cp - 127))) return -127;
  const float n = rintf(tmax);  // nearest, ties to even (|tmax| < 2^22)
  const float g = tmax - n;     // exact, in [-1/2, 1/2]
  int e = static_cast<int>(n) - cp - 2;
  if (g < 0.f && !(kUOS && g > kUosFracThreshold)) e -= 1;
  return e < -127 ? -127 : e;
}

// E2M1 codes of one 32-key block: code values q(g) 2^(n - c) (t raised to c - 127 first, so
// keys past the end and underflowing keys give 0) times the block's 2^-e, rounded to
// nearest even with saturation.  The general form.
__device__ __forceinline__ void pnq_block_codes(const float* t, float lo, uint32_t bias_bits, float s1,
                                                uint32_t* codes) {
  const float2 sc = make_float2(s1, s1);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    float2 v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      v[q] = __fmul2_rn(pnq_code_pair(make_float2(t[8 * w + 2 * q], t[8 * w + 2 * q + 1]), lo, bias_bits), sc);
    codes[w] = e2m1x8(v[0].x, v[0].y, v[1].x, v[1].y, v[2].x, v[2].y, v[3].x, v[3].y);
  }
}

// The same codes, two multiplies fewer per pair of keys, for a block in which every key has
// rint(t) - c >= -126 and rint(t) - c - e >= -125, with |ce| <= 100 (ce = c + e).  The
// factor 2^-(c + e) rides on the cubic's coefficients: a power of two, so every Horner step
// (the rounded-up last one too) rounds as it would unscaled and q'(g) = q(g) 2^-(c + e)
// exactly.  2^n then enters by an integer add to the exponent field (bits(r) * 2^23 = n * 2^23
// modulo 2^32, as in pnq_code_pair), which stays within [1, 254]: the value is
// q(g) 2^(n - c - e), the one the general form rounds to E2M1.
__device__ __forceinline__ void pnq_block_codes_folded(const float* t, int ce, uint32_t* codes) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  const float f = __uint_as_float(static_cast<uint32_t>(127 - ce) << 23);
  const float a0 = f, a1 = __fmul_rn(kCodeA1, f), a2 = __fmul_rn(kCodeA2, f), a3 = __fmul_rn(kCodeA3, f);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    float v[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 x = make_float2(t[8 * w + 2 * q], t[8 * w + 2 * q + 1]);
      const float2 r = __fadd2_rn(x, make_float2(kMagic, kMagic));
      const float2 n = __fadd2_rn(r, make_float2(-kMagic, -kMagic));
      const float2 g = __fadd2_rn(x, make_float2(-n.x, -n.y));
      float2 p = __ffma2_rn(make_float2(a3, a3), g, make_float2(a2, a2));
      p = __ffma2_rn(p, g, make_float2(a1, a1));
      p = __ffma2_ru(p, g, make_float2(a0, a0));
      v[2 * q] = __uint_as_float(__float_as_uint(p.x) + __float_as_uint(r.x) * 8388608u);
      v[2 * q + 1] = __uint_as_float(__float_as_uint(p.y) + __float_as_uint(r.y) * 8388608u);
    }
    codes[w] = e2m1x8(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]);
  }
}

template <bool kUOS>
__global__ void __launch_bounds__(kAttnThreads, 1)
    mx_attention_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_sfq,
                        const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_sfk,
                        const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_sfv,
                        __nv_bfloat16* __restrict__ out, int64_t ldo, const AttnParams prm) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sSfq = smem + kAttnOffSfq;
  uint8_t* sStages = smem + kAttnOffStages;
  uint8_t* sP = smem + kAttnOffP;
  uint8_t* sSfp = smem + kAttnOffSfp;
  uint8_t* sSfOnes = smem + kAttnOffSfOnes;
  float* sRmax = reinterpret_cast<float*>(smem + kAttnOffRmax);
  uint64_t* q_full = reinterpret_cast<uint64_t*>(smem + kAttnOffBar);
  uint64_t* kv_full = q_full + 1;
  uint64_t* kv_empty = kv_full + kAttnStages;
  uint64_t* s_full = kv_empty + kAttnStages;
  uint64_t* s_free = s_full + 1;
  uint64_t* p_full = s_free + 1;
  uint64_t* o_done = p_full + 1;
  uint64_t* rbar = o_done + 1;  // [2]
  uint64_t* drain = rbar + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  auto sK = [&](int s) { return sStages + s * kAttnStageBytes; };
  auto sV = [&](int s) { return sStages + s * kAttnStageBytes + kAttnKBytes; };
  auto sSfk = [&](int s) { return sStages + s * kAttnStageBytes + kAttnKBytes + kAttnVBytes; };
  auto sSfv = [&](int s) { return sStages + s * kAttnStageBytes + kAttnKBytes + kAttnVBytes + 1024; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int q_tile = blockIdx.x;
  const int head = blockIdx.y;
  const int nt = prm.num_tiles;

  if (threadIdx.x == 0) {
    prefetch_tmap(&tmap_q);
    prefetch_tmap(&tmap_sfq);
    prefetch_tmap(&tmap_k);
    prefetch_tmap(&tmap_sfk);
    prefetch_tmap(&tmap_v);
    prefetch_tmap(&tmap_sfv);
    mbar_init(q_full, 1);
    for (int s = 0; s < kAttnStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, kAttnSoftWarps);  // one arrival per softmax warp
    mbar_init(p_full, kAttnSoftWarps);
    mbar_init(o_done, 1);
    mbar_init(&rbar[0], kAttnSoftWarps);  // one arrival per softmax warp
    mbar_init(&rbar[1], kAttnSoftWarps);
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp >= 4) {
    // Constant parts of the P V operand: the row of ones (row d = 128 of each V^T stage:
    // E2M1 1.0 = code 2 in every nibble; rows 129..143 zero) and their unit scales.
    const int t = threadIdx.x - 128;  // 0..511
    for (int s = 0; s < kAttnStages; ++s) {
      uint32_t* ones = reinterpret_cast<uint32_t*>(sV(s) + kAttnD * 128);  // 16 rows x 128 B = 512 words
      ones[t] = t < 32 ? 0x22222222u : 0u;
    }
    if (t < 256) reinterpret_cast<uint32_t*>(sSfOnes)[t] = 0x7F7F7F7Fu;  // 2 atoms = 256 words
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kAttnTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp < 4) {
    setmaxnreg_dec<kAttnCtrlRegs>();  // the whole control warpgroup, one instruction
    if (warp == 0) {
      // ------------------------------------------------------------------ TMA producer
      if (elect_one()) {
        bool ok = true;
        mbar_arrive_expect_tx(q_full, kAttnQBytes + 512);
        tma_load_2d(sQ, &tmap_q, head * 64, q_tile * kAttnBM, q_full);
        tma_load_4d(sSfq, &tmap_sfq, 0, 0, head, q_tile, q_full);
        int stage = 0;
        uint32_t phase = 0, issued = 0, issued_phase = 0;
        const uint32_t tx = kAttnKBytes + kAttnD * 128 + 1024 + 1024;
        for (int j = 0; j < nt; ++j) {
          if (!mbar_wait(&kv_empty[stage], phase ^ 1)) { ok = false; break; }
          issued |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          mbar_arrive_expect_tx(&kv_full[stage], tx);
          tma_load_2d(sK(stage), &tmap_k, head * 64, j * kAttnBN, &kv_full[stage]);
          tma_load_4d(sSfk(stage), &tmap_sfk, 0, 0, head, 2 * j, &kv_full[stage]);
          tma_load_2d(sV(stage), &tmap_v, j * (kAttnBN / 2), head * kAttnD, &kv_full[stage]);
          tma_load_4d(sSfv(stage), &tmap_sfv, 0, 0, 2 * j, head, &kv_full[stage]);
          if (++stage == kAttnStages) { stage = 0; phase ^= 1; }
        }
        mbar_wait_drain(q_full, 0);
        if (!ok) {
          for (int s = 0; s < kAttnStages; ++s)
            if (issued & (1u << s)) mbar_wait_drain(&kv_full[s], (issued_phase >> s) & 1u);
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------------ MMA issuer
      if (elect_one()) {
        bool ok = mbar_wait(q_full, 0);
        if (ok) {
          tc_fence_after();
          tc_cp_sf_atom(tmem + kColSfq, smem_desc(smem_u32(sSfq), 0, 128, 0));
        }
        // O += P V^T for key tile i (P from shared memory, written by the softmax warps).
        auto issue_pv = [&](int i) -> bool {
          if (!mbar_wait(p_full, i & 1)) return false;
          tc_fence_after();
          const int st = i % kAttnStages;
          const uint32_t par = static_cast<uint32_t>(i & 1);
          const uint32_t sfp = kColSfp + par * 8, sfv = kColSfv + par * 16;
  #pragma unroll
          for (int a = 0; a < 2; ++a) {
            tc_cp_sf_atom(tmem + sfp + 4 * a, smem_desc(smem_u32(sSfp + a * 512), 0, 128, 0));
            tc_cp_sf_atom(tmem + sfv + 8 * a, smem_desc(smem_u32(sSfv(st) + a * 512), 0, 128, 0));
            tc_cp_sf_atom(tmem + sfv + 8 * a + 4, smem_desc(smem_u32(sSfOnes + a * 512), 0, 128, 0));
          }
          const uint32_t p_base = smem_u32(sP), v_base = smem_u32(sV(st));
  #pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // 4 x 64 keys
            const int a = kk >> 1;
            const uint32_t sf_id = static_cast<uint32_t>((kk & 1) * 2);
            const uint32_t idesc = attn_idesc(kAttnNv) | (sf_id << 29) | (sf_id << 4);
            tc_mma_mxf4(tmem + kColO, smem_desc(p_base + kk * 32, 16, 1024, 2), smem_desc(v_base + kk * 32, 16, 1024, 2),
                        idesc, tmem + sfp + 4 * a, tmem + sfv + 8 * a, (i | kk) != 0);
          }
          tc_commit(o_done);
          tc_commit(&kv_empty[st]);
          return true;
        };
        int stage = 0;
        uint32_t phase = 0;
        for (int j = 0; ok && j < nt; ++j) {
          if (!mbar_wait(&kv_full[stage], phase)) { ok = false; break; }
          if (j > 0 && !mbar_wait(s_free, (j - 1) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sfk = kColSfk + static_cast<uint32_t>(j & 1) * 8;
          tc_cp_sf_atom(tmem + sfk, smem_desc(smem_u32(sSfk(stage)), 0, 128, 0));
          tc_cp_sf_atom(tmem + sfk + 4, smem_desc(smem_u32(sSfk(stage) + 512), 0, 128, 0));
          const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK(stage));
  #pragma unroll
          for (int kk = 0; kk < 2; ++kk) {  // 2 x 64 of the head dimension
            const uint32_t sf_id = static_cast<uint32_t>(kk * 2);
            const uint32_t idesc = attn_idesc(kAttnBN) | (sf_id << 29) | (sf_id << 4);
            tc_mma_mxf4(tmem + kColS, smem_desc(q_base + kk * 32, 16, 512, 4), smem_desc(k_base + kk * 32, 16, 512, 4),
                        idesc, tmem + kColSfq, tmem + sfk, kk != 0);
          }
          tc_commit(s_full);
          if (j > 0 && !issue_pv(j - 1)) { ok = false; break; }
          if (++stage == kAttnStages) { stage = 0; phase ^= 1; }
        }
        if (ok) ok = issue_pv(nt - 1);
        if (!ok) {
          tc_commit(drain);
          mbar_wait_drain(drain, 0);
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tmem, kAttnTmemCols);
    }
  } else {
    setmaxnreg_inc<kAttnSoftRegs>();
    // ------------------------------------------------------------------ softmax / PNQ (warps 4..19)
    const int quad = warp & 3;          // TMEM lanes [32 quad, +32)
    const int qt = (warp - 4) >> 2;     // keys [64 qt, +64) of every tile
    const int r = quad * 32 + lane;     // query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    int chat = 0;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(s_full, j & 1))) { ok = false; break; }
      tc_fence_after();
      float t[64];
      {
        uint32_t v[64];
        tmem_ld64(tmem + lane_off + kColS + 64 * qt, v);
        tmem_ld_wait();
        const float2 ts = make_float2(prm.t_scale, prm.t_scale);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 x = __fmul2_rn(make_float2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])), ts);
          t[2 * i] = x.x;
          t[2 * i + 1] = x.y;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);
      // keys past the end do not take part (only the last tile has any)
      const int key0 = j * kAttnBN + 64 * qt;
      if (key0 + 64 > prm.Skv) {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (key0 + i >= prm.Skv) t[i] = -INFINITY;
      }
      float bmax[2], bmin[2];  // per 32-key block, three operands per instruction
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        float mb = t[32 * b], nb = t[32 * b];
#pragma unroll
        for (int i = 1; i < 31; i += 2) {
          mb = fmax3(mb, t[32 * b + i], t[32 * b + i + 1]);
          nb = fmin3(nb, t[32 * b + i], t[32 * b + i + 1]);
        }
        bmax[b] = fmaxf(mb, t[32 * b + 31]);
        bmin[b] = fminf(nb, t[32 * b + 31]);
      }
      // Publish this thread's maximum; the row's offset is settled after the codes.
      const float m_own = fmaxf(bmax[0], bmax[1]);
      float* slot = sRmax + (j & 1) * 512;
      slot[qt * 128 + r] = m_own;
      __syncwarp();  // the warp's 32 slots are written before its one (release) arrival
      if (lane == 0) mbar_arrive(&rbar[j & 1]);
      // Provisional offset cp: the lazy rule applied to this thread's own keys.  The row's
      // offset chat (settled below) is never below it, and the E8M0 block scaling is
      // equivariant under the power of two 2^(cp - chat): the codes computed against cp
      // are the row's codes, and only the scale bytes move by cp - chat.
      int cp = chat;
      if (m_own > -INFINITY) {
        const int own = static_cast<int>(ceilf(m_own));
        if (j == 0 || own > chat + 8) cp = own;
      } else if (j == 0) {
        cp = 0;  // every key of this thread is past the end: codes 0 whatever the offset
      }
      uint32_t codes[8];
      int eb[2];
      {
        const float lo = static_cast<float>(cp - 127);
        const uint32_t bias_bits = static_cast<uint32_t>(127 - cp) << 23;
        // the block exponents from the blocks' largest scores (-127 if none)
        eb[0] = pnq_block_exponent<kUOS>(bmax[0], cp);
        eb[1] = pnq_block_exponent<kUOS>(bmax[1], cp);
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          const int e = eb[b];
          const int ce = cp + e;
          if (ce >= -100 && ce <= 100 && bmin[b] >= static_cast<float>(max(cp - 126, ce - 125))) {
            pnq_block_codes_folded(t + 32 * b, ce, codes + 4 * b);  // the usual case
          } else {
            pnq_block_codes(t + 32 * b, lo, bias_bits, exp2_neg(e), codes + 4 * b);
          }
        }
      }
      // The row's offset: the maximum over its four threads, raised lazily.
      if (!__all_sync(0xffffffffu, mbar_wait(&rbar[j & 1], (j >> 1) & 1))) { ok = false; break; }
      const float m = fmaxf(fmaxf(slot[r], slot[128 + r]), fmaxf(slot[256 + r], slot[384 + r]));  // key j*256: finite
      const int cand = static_cast<int>(ceilf(m));
      float rescale = 1.f;
      if (j == 0) {
        chat = cand;
      } else if (cand > chat + 8) {
        // 2^(chat - cand), exact; 0 once it is below the normal range
        rescale = cand - chat > 126 ? 0.f : __int_as_float((127 + chat - cand) << 23);
        chat = cand;
      }
      uint32_t sf_half = 0;
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        int e = eb[b] + cp - chat;
        if (e < -127) {  // below the E8M0 range relative to the row: numerators < 2^-120 of it
          codes[4 * b] = codes[4 * b + 1] = codes[4 * b + 2] = codes[4 * b + 3] = 0u;
          e = -127;
        }
        sf_half |= static_cast<uint32_t>(min(e, 127) + 127) << (8 * b);
      }
      // the previous tile's P V must be done before P is overwritten or O rescaled
      if (j > 0) {
        if (!__all_sync(0xffffffffu, mbar_wait(o_done, (j - 1) & 1))) { ok = false; break; }
        tc_fence_after();
      }
      if (__any_sync(0xffffffffu, rescale != 1.f)) {
        uint32_t v[32];
        const uint32_t a0 = tmem + lane_off + kColO + 32 * qt;
        tmem_ld32(a0, *reinterpret_cast<uint32_t(*)[32]>(v));
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__fmul_rn(__uint_as_float(v[i]), rescale));
        tmem_st32(a0, v);
        if (qt == 0) {  // the l column block (column 128 and the zero columns after it)
          const uint32_t a1 = tmem + lane_off + kColO + kAttnD;
          tmem_ld16(a1, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = __float_as_uint(__fmul_rn(__uint_as_float(v[i]), rescale));
          tmem_st16(a1, v);
        }
        tmem_st_wait();
      }
      // codes: row r, bytes [32 qt, +32) = 16-byte chunks 2 qt + b, 128-byte swizzle
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const int chunk = (2 * qt + b) ^ (r & 7);
        *reinterpret_cast<uint4*>(sP + r * 128 + chunk * 16) =
            make_uint4(codes[4 * b], codes[4 * b + 1], codes[4 * b + 2], codes[4 * b + 3]);
      }
      *reinterpret_cast<uint16_t*>(sSfp + (qt >> 1) * 512 + (r & 31) * 16 + (r >> 5) * 4 + 2 * (qt & 1)) =
          static_cast<uint16_t>(sf_half);
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // ---------------------------------------------------------------- O / l -> BF16
    if (ok && __all_sync(0xffffffffu, mbar_wait(o_done, (nt - 1) & 1))) {
      tc_fence_after();
      uint32_t v[32], lv[16];
      tmem_ld32(tmem + lane_off + kColO + 32 * qt, *reinterpret_cast<uint32_t(*)[32]>(v));
      tmem_ld16(tmem + lane_off + kColO + kAttnD, lv);
      tmem_ld_wait();
      const float inv_l = __fdiv_rn(1.0f, __uint_as_float(lv[0]));
      const int64_t row = static_cast<int64_t>(q_tile) * kAttnBM + r;
      if (row < prm.Sq) {
        uint4* dst = reinterpret_cast<uint4*>(out + row * ldo + head * kAttnD + 32 * qt);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q)
            w[q] = pack_bf16x2(__fmul_rn(__uint_as_float(v[8 * c + 2 * q]), inv_l),
                               __fmul_rn(__uint_as_float(v[8 * c + 2 * q + 1]), inv_l));
          dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
    tc_fence_before();
    __syncthreads();
  }
}

// V [S][ldv] BF16 -> V^T in MXFP4 with 32-key blocks: codes [HD][Sp/2], scales for the
// [HD][Sp/32] grid in the 512-byte atom layout; keys in [S, Sp) are zero.  One CTA per
// 128 keys x 128 channels: the tile is staged in shared memory (BF16) and read back
// column-wise (a warp: 32 consecutive channels of one key row per step).
template <bool kUOS>
__global__ void __launch_bounds__(256) quantize_vt_kernel(const uint16_t* __restrict__ v, int64_t S, int64_t ldv,
                                                           int64_t Sp, uint8_t* __restrict__ codes,
                                                           uint8_t* __restrict__ sf) {
  constexpr int kPitch = 136;  // halfwords per staged row (272 bytes: 16-byte aligned rows)
  __shared__ __align__(16) uint16_t tile[128 * kPitch];
  const int tid = threadIdx.x;
  const int64_t key0 = static_cast<int64_t>(blockIdx.y) * 128;
  const int64_t ch0 = static_cast<int64_t>(blockIdx.x) * 128;
  {
    const int i = tid >> 1, c0 = 64 * (tid & 1);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t w[8];
      if (key0 + i < S) {
        ld_stream_v8(v + (key0 + i) * ldv + ch0 + c0 + 16 * q, w);
      } else {
#pragma unroll
        for (int u = 0; u < 8; ++u) w[u] = 0u;
      }
      uint4* dst = reinterpret_cast<uint4*>(tile + i * kPitch + c0 + 16 * q);
      dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
      dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
  }
  __syncthreads();
  const int c = tid & 127, th = tid >> 7;  // a warp: 32 consecutive channels, one key half
  const int64_t row = ch0 + c;
  auto val = [&](int k) { return __uint_as_float(static_cast<uint32_t>(tile[k * kPitch + c]) << 16); };
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    const int k0 = 64 * th + 32 * b;
    float amax = 0.f;
#pragma unroll
    for (int u = 0; u < 32; ++u) amax = fmaxf(amax, fabsf(val(k0 + u)));
    const int e = block_exponent<kUOS>(__float_as_uint(amax));
    const float s = exp2_neg(e);
    uint32_t word[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int b = k0 + 8 * w;
      word[w] = e2m1x8(__fmul_rn(val(b), s), __fmul_rn(val(b + 1), s), __fmul_rn(val(b + 2), s),
                       __fmul_rn(val(b + 3), s), __fmul_rn(val(b + 4), s), __fmul_rn(val(b + 5), s),
                       __fmul_rn(val(b + 6), s), __fmul_rn(val(b + 7), s));
    }
    const int64_t kb = key0 + k0;  // first key of the block
    *reinterpret_cast<uint4*>(codes + row * (Sp / 2) + kb / 2) = make_uint4(word[0], word[1], word[2], word[3]);
    const int64_t col = kb / 32;
    sf[((row >> 7) * (Sp / 128) + (col >> 2)) * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 + (col & 3)] =
        static_cast<uint8_t>(e + 127);
  }
}

}  // namespace mxq
