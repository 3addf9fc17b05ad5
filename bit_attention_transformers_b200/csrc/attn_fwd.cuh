// Fused NVFP4 FlashAttention forward for sm_100a (tcgen05 + TMEM + TMA).
//
// What it computes [HiFA4 summary, theflow.svmpsp.dev related-papers feed;
// EFQ-Softmax abstract, scholarbro.com page "AVQ Attention: Adaptive
// Vector-Quantized Attention"]: both QK^T and PV are 4-bit block-scaled
// contractions; the softmax keeps a running row maximum and row sum in fp32,
// rescales the accumulated output when the maximum grows, and the probability
// tile is exponentiated in fp32 and re-quantised to NVFP4 per 16 keys before
// the PV contraction (exp-then-quantize); the output is normalised at the end.
//
// Per CTA: one tile of 128 query rows of one (batch, head); key tiles of 128.
//   warp 0      TMA producer: Q once, K/V tiles (+ their scales) into a ring
//   warp 1      TMEM owner and S issuer (one thread): S = Q K^T into a
//               double-buffered TMEM tile, S_{t+2} as soon as S_t has been read
//   warp 2      PV issuer (one thread): O += P V into a TMEM accumulator once
//               P_t is written; each issuer commits only its own operations
//   warp 3      idle (it completes the first warpgroup)
//   warps 4..11 softmax: one thread per query row and two streams per
//               32-row quadrant: stream s takes the key tiles t = s mod 2
//               (S buffer s, P buffer s), so two tiles are in flight on every
//               SM sub-partition; the running maximum, the only value a tile
//               needs from the one before, passes between the two streams
//               through shared memory; P (NVFP4 codes and block scales, or
//               FP8 codes) goes to TMEM with tcgen05.st, where PV reads it as
//               its A operand
// TMEM columns: S0 [0,128) S1 [128,256) O [256,256+D) scales from 384, then
// P's codes (two buffers: 16 columns NVFP4, 32 columns FP8).
//
// EFQ variant (template flag EFQ) [EFQ-Softmax abstract]: P is generated
// without exponentials. Per 16-key block, E = floor(max z) - 2 with z = x - m
// (max z formed as fl(x_max) - m, exactly 0 in the block of the running
// maximum); codes clamp(rne(2 (z - E) + 2), 0, 7), computed as
// rne(7 * sat(s c' + o)) with c' = 2c/7 and o = (2 - 2 (m + E)) / 7: one
// saturating FMA (the clamp) and one FMA that adds 2^23 (the rounding) per
// score, the low mantissa bits being the code; scale byte 2^(E + 10) (P's
// tensor scale 2^-10). The denominator P~1 comes from the tensor cores: two
// more MMAs per tile multiply P~ by a constant all-ones FP4 tile into 16 TMEM
// columns beside O (L [256+D, 256+D+16)), so the same rescaling applies to
// it; the scale columns then start at 400.
//
// FP8 variant (PG = kPgFp8) [SageAttention2 abstract, searcharxiv.com author
// page "Pengle Zhang": P~ and V in FP8]: P~ = E4M3(256 p) per key (no block
// scales), V in E4M3 with one tensor scale, PV as four kind::f8f6f4 MMAs
// (K = 32) over 128-byte-swizzled tiles; l sums 256 p.
// BIAS (smoothed Q, same page): the per-key correction hi + lo (tf32) joins
// the S accumulator as a rank-1 product ones x [hi, lo]^T (kind::tf32) after
// the tile's FP4 MMAs; the softmax is unchanged.
// LSE (the training forward): the epilogue also writes m + log2 l per row.
//
// Causal launches order the CTAs longest first across all heads (query tile
// ntq-1 of every head, then ntq-2, ...), so the short tiles fill the last wave.
//
// Every wait is bounded (2 s of %globaltimer); on expiry the kernel sets the
// device error word, stops issuing, drains its tensor-core work and the bulk
// copies still in flight into shared memory, and returns.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "quantize.cuh"

namespace fp4 {

constexpr int kBM = 128;                    // query rows per CTA
constexpr int kBN = 128;                    // keys per tile (the method's Bc)
constexpr int kStages = 3;                  // K/V ring depth
constexpr int kAttnThreads = 384;  // 12 warps = 3 warpgroups
// Register budgets after the warpgroups re-balance: 128 x 56 + 256 x 224 equals
// the 384 x 168 registers the block is launched with.
constexpr uint32_t kRegsCtl = 56, kRegsSoftmax = 224;
constexpr uint64_t kTimeoutNs = 2000000000ull;

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity,
                                         uint64_t limit_ns = kTimeoutNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*reinterpret_cast<volatile unsigned*>(&g_fp4_err) != 0u) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      atomicOr(&g_fp4_err, kDevErrTimeout);
      return false;
    }
  }
  return true;
}

// Bounded wait that ignores the error word (used only to drain in-flight work).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > kTimeoutNs / 20) return;
}

// Test support: one thread waits, with the kernels' bounded wait and the given
// limit, on an mbarrier that nothing arrives on; the wait expires, sets the
// device error word and returns. *ok receives 0 (expired) or 1.
__global__ void wait_timeout_kernel(uint64_t limit_ns, int* ok) {
  __shared__ uint64_t b;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&b), 1);
    fence_mbar_init();
    *ok = wait_bar(smem_u32(&b), 0, limit_ns) ? 1 : 0;
  }
}

#ifdef FP4_DEBUG
// Test support of the debug build: one check that fails by construction and
// guards no access (the reporting path of FP4_CHECK, nothing else).
__global__ void dbg_selftest_kernel(unsigned site) {
  volatile unsigned never = 0u;
  if (!FP4_CHECK(never != 0u, site)) return;
}
#endif

struct AttnParams {
  const uint8_t* q_sf;
  const uint8_t* k_sf;
  const uint8_t* v_sf;
  const float* amax_q;  // absolute maxima of the source tensors
  const float* amax_k;
  const float* amax_v;
  __nv_bfloat16* out;  // [B][H][N][D]
  float* lse;          // [B*H][N]: log2 sum_j 2^(x_ij) per row for the backward, or NULL
  int B, H, Hkv, N, Npad, ntq;
  float softmax_scale;
};

// P generation: exp-then-quantize to NVFP4 (the method), EFQ-Softmax, or
// exp-then-quantize to FP8 E4M3 with V in FP8 as well.
enum : int { kPgExp = 0, kPgEfq = 1, kPgFp8 = 2 };

template <int D, bool FP8 = false, bool BIAS = false>
struct AttnSmem {
  static constexpr int kQ = kBM * D / 2;   // Q codes tile
  static constexpr int kK = kBN * D / 2;   // K codes tile
  static constexpr int kV = FP8 ? D * kBN : D * kBN / 2;    // V^T codes tile
  static constexpr int kP = FP8 ? kBM * kBN : kBM * kBN / 2;  // P codes tile (reserved; P lives in TMEM)
  static constexpr int kSfQK = (D / 64) * 512;
  static constexpr int oQ = 0;
  static constexpr int oK = oQ + kQ;
  static constexpr int oV = oK + kStages * kK;
  static constexpr int oP = oV + kStages * kV;
  static constexpr int oOnes = oP + 2 * kP;     // EFQ: 16 x 128 FP4 ones (code 2), 1 KB
  static constexpr int oOnesSf = oOnes + 1024;  // EFQ: one scale atom of 1.0 (E4M3 0x38)
  static constexpr int oQsf = oOnesSf + 512;
  static constexpr int oKsf = oQsf + 1024;
  static constexpr int oVsf = oKsf + kStages * 1024;
  static constexpr int oPsf = oVsf + kStages * 1024;  // reserved (P scales live in TMEM)
  static constexpr int oRed = oPsf + 2 * 1024;  // float [2][128] running max per stream, [2][128] l
  static constexpr int oPtab = oRed + 2048;     // float [128]
  static constexpr int oBar = oPtab + 512;      // mbarriers
  static constexpr int oTmem = oBar + 256;
  // BIAS: the rank-1 score correction, 128 keys x (hi, lo, 0, 0, 0, 0, 0, 0)
  // tf32 per K stage (32-byte swizzle), and its all-ones A operand
  static constexpr int oBiasB = (oTmem + 16 + 1023) / 1024 * 1024;
  static constexpr int oOnesT = oBiasB + kStages * 4096;
  static constexpr int kBytes = (BIAS ? oOnesT + 4096 : oTmem + 16) + 1024;  // + alignment slack
};

// Barrier indices (8 bytes each).
enum : int {
  kBarQ = 0,
  kBarKFull = 1,
  kBarKEmpty = kBarKFull + kStages,
  kBarVFull = kBarKEmpty + kStages,
  kBarVEmpty = kBarVFull + kStages,
  kBarSFull = kBarVEmpty + kStages,
  kBarSEmpty = kBarSFull + 2,
  kBarPFull = kBarSEmpty + 2,
  kBarO = kBarPFull + 2,            // [2]: PV of tile t completes O[t & 1]
  kBarMax = kBarO + 2,              // [4 quadrants][2]: running max of tile t published
  kBarDrain = kBarMax + 8,  // [2]: S issuer, PV issuer
  kNumBars = kBarDrain + 2
};

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;
// Scale-factor columns: after O (at most 128 columns) and, for EFQ, the 16
// denominator columns beside it.
template <bool EFQ>
struct TmemCols {
  static constexpr uint32_t kSf = EFQ ? 400 : 384;
  static constexpr uint32_t kQsf = kSf, kKsf = kSf + 8, kPsf = kSf + 24, kVsf = kSf + 40,
                            kOnesSf = kSf + 56,
                            kPc = kSf + 64,  // [2] x 16: P codes (NVFP4 paths), 8 per column
                            kP8 = kSf + 32;  // [2] x 32: P codes (FP8 path), 4 per column
};
constexpr float kInv7 = 1.0f / 7.0f;
constexpr float kRound = 8388608.0f;  // 2^23: x + 2^23 rounds x (0 <= x < 2^22) to an integer

// BIAS: add a per-key correction beta'_j = hi_j + lo_j (two tf32 values, in the
// contraction's units) to the S accumulator as a rank-1 tensor-core product,
// ones[128 x 8] x [hi, lo, 0, ...]^T (kind::tf32, K = 8) after the FP4 MMAs
// of the tile (the smoothed-Q path; exp-then-quantize P only). The key tile's
// corrections travel with its K tile (tmB) and the softmax is unchanged.
// LSE: also write lse = m + log2 l per row (the training forward).
template <int D, bool CAUSAL, int PG, bool BIAS = false, bool LSE = false>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmB,
                    const AttnParams p) {
  constexpr bool EFQ = PG == kPgEfq, FP8 = PG == kPgFp8;
  static_assert(!BIAS || PG == kPgExp, "the score correction is built for exp-then-quantize P");
  static_assert(!LSE || PG == kPgExp, "lse is written by the exp-then-quantize forward");
  using L = AttnSmem<D, FP8, BIAS>;
  using TC = TmemCols<EFQ>;
  constexpr uint32_t kColQsf = TC::kQsf, kColKsf = TC::kKsf, kColPsf = TC::kPsf,
                     kColVsf = TC::kVsf, kColL = kColO + D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // causal: a 1D grid, longest query tiles of every head first
  int qt, h, b;
  if (CAUSAL) {
    const int nbh = p.B * p.H;
    const int i = (int)blockIdx.x;
    qt = p.ntq - 1 - i / nbh;
    h = (i % nbh) % p.H;
    b = (i % nbh) / p.H;
  } else {
    qt = (int)blockIdx.x;
    h = (int)blockIdx.y;
    b = (int)blockIdx.z;
  }
  const int gq = b * p.H + h;
  const int gk = b * p.Hkv + h / (p.H / p.Hkv);
  const int nkv = (p.N + kBN - 1) / kBN;
  const int nt = CAUSAL ? min(qt + 1, nkv) : nkv;
  auto bar = [&](int i) -> uint32_t { return sb + L::oBar + 8 * i; };

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQ), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarKEmpty + s), 1);
      mbar_init(bar(kBarVFull + s), 1);
      mbar_init(bar(kBarVEmpty + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBarSFull + s), 1);
      mbar_init(bar(kBarSEmpty + s), 4);
      mbar_init(bar(kBarPFull + s), 4);
      mbar_init(bar(kBarO + s), 1);
    }
    for (int s = 0; s < 8; ++s) mbar_init(bar(kBarMax + s), 1);
    mbar_init(bar(kBarDrain), 1);
    mbar_init(bar(kBarDrain + 1), 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(sb + L::oTmem, kTmemCols);
    tmem_relinquish();
  }
  // r = 2688 / dec(e) for every E4M3 scale byte e of the P quantiser (0 -> 0)
  float* ptab = reinterpret_cast<float*>(sm + L::oPtab);
  if (threadIdx.x >= 64 && threadIdx.x < 192) {
    const uint32_t e = threadIdx.x - 64;
    const float de = e4m3_to_f32(e);
    ptab[e] = (e >= 127u || de == 0.0f) ? 0.0f : __fdiv_rn(kTensorRange, de);
  }
  if (BIAS && threadIdx.x >= 128 && threadIdx.x < 384) {
    // the rank-1 correction's A operand: every row [1, 1, 0, 0 | 1, 1, 0, 0]
    // (both 16-byte halves alike, so the 32-byte swizzle leaves it unchanged)
    const int i = threadIdx.x - 128;  // 256 threads x 16 bytes = 4 KB
    *reinterpret_cast<uint4*>(sm + L::oOnesT + 16 * i) =
        make_uint4(0x3F800000u, 0x3F800000u, 0u, 0u);
    fence_proxy_async_smem();
  }
  if (EFQ && threadIdx.x >= 192 && threadIdx.x < 288) {
    // the all-ones B operand of P~1 (every code 2 = 1.0) and its scales (1.0)
    const int i = threadIdx.x - 192;  // 96 threads x 16 bytes = 1536 bytes
    *reinterpret_cast<uint4*>(sm + L::oOnes + 16 * i) =
        i < 64 ? make_uint4(0x22222222u, 0x22222222u, 0x22222222u, 0x22222222u)
               : make_uint4(0x38383838u, 0x38383838u, 0x38383838u, 0x38383838u);
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + L::oTmem);

  if (warp < 4) {
  regs_dec<kRegsCtl>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      bool ok = true;
      int kissued = 0, vissued = 0;  // tiles whose K / V loads were started
      const int qrow0 = gq * p.Npad + qt * kBM;
      const int64_t Gq = (int64_t)p.B * p.H, Gk = (int64_t)p.B * p.Hkv;
      mbar_arrive_expect_tx(bar(kBarQ), L::kQ + L::kSfQK);
      if (FP4_CHECK(tma_ok(0, D / 2, D / 2, 1, qrow0, kBM, Gq * p.Npad), 201))
        tma_load_2d(sb + L::oQ, &tmQ, 0, qrow0, bar(kBarQ));
      const int64_t qsf = ((int64_t)gq * (p.Npad / kBM) + qt) * L::kSfQK;
      if (FP4_CHECK(in_range(qsf, L::kSfQK, Gq * (p.Npad / kBM) * L::kSfQK), 202))
        bulk_load(sb + L::oQsf, p.q_sf + qsf, L::kSfQK, bar(kBarQ));
      for (int j = 0; j < nt && ok; ++j) {
        const int st = j % kStages;
        const uint32_t pe = ((j / kStages) - 1) & 1;
        if (j >= kStages && !(ok = wait_bar(bar(kBarKEmpty + st), pe))) break;
        mbar_arrive_expect_tx(bar(kBarKFull + st), L::kK + L::kSfQK + (BIAS ? 4096 : 0));
        if (FP4_CHECK(tma_ok(0, D / 2, D / 2, 1, gk * p.Npad + j * kBN, kBN, Gk * p.Npad), 203))
          tma_load_2d(sb + L::oK + st * L::kK, &tmK, 0, gk * p.Npad + j * kBN, bar(kBarKFull + st));
        if (BIAS && FP4_CHECK(tma_ok(0, 32, 32, 1, gq * p.Npad + j * kBN, kBN, Gq * p.Npad), 204))
          tma_load_2d(sb + L::oBiasB + st * 4096, &tmB, 0, gq * p.Npad + j * kBN,
                      bar(kBarKFull + st));
        const int64_t ksf = ((int64_t)gk * (p.Npad / kBN) + j) * L::kSfQK;
        if (FP4_CHECK(in_range(ksf, L::kSfQK, Gk * (p.Npad / kBN) * L::kSfQK), 205))
          bulk_load(sb + L::oKsf + st * 1024, p.k_sf + ksf, L::kSfQK, bar(kBarKFull + st));
        kissued = j + 1;
        if (j >= kStages && !(ok = wait_bar(bar(kBarVEmpty + st), pe))) break;
        mbar_arrive_expect_tx(bar(kBarVFull + st), L::kV + (FP8 ? 0 : 1024));
        constexpr int kVx = FP8 ? kBN : kBN / 2;  // bytes of one tile's keys in a V^T row
        if (FP4_CHECK(tma_ok(j * kVx, kVx, (int64_t)p.Npad * kVx / kBN, 1, gk * D, D, Gk * D), 206))
          tma_load_2d(sb + L::oV + st * L::kV, &tmV, j * kVx, gk * D, bar(kBarVFull + st));
        const int64_t vsf = ((int64_t)gk * (p.Npad / 64) + 2 * j) * 512;
        if (!FP8 && FP4_CHECK(in_range(vsf, 1024, Gk * (p.Npad / 64) * 512), 207))
          bulk_load(sb + L::oVsf + st * 1024, p.v_sf + vsf, 1024, bar(kBarVFull + st));
        vissued = j + 1;
      }
      if (!ok) {
        // no bulk copy may outlive the CTA: wait (bounded) for the last load
        // started on every stage; a stage its consumer already took has
        // completed that phase, and no later phase was started
        drain_wait(bar(kBarQ), 0);
        for (int j = max(0, kissued - kStages); j < kissued; ++j)
          drain_wait(bar(kBarKFull + j % kStages), (j / kStages) & 1);
        for (int j = max(0, vissued - kStages); j < vissued; ++j)
          drain_wait(bar(kBarVFull + j % kStages), (j / kStages) & 1);
      }
    }
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ MMA issuers
    // warp 1 issues S_{t+2} as soon as the softmax has read S_t; warp 2 issues
    // PV_t once P_t is written. Each commits only its own operations.
    if (lane == 0) {
      constexpr uint32_t kSw = (D == 128) ? 4u : 6u;     // 64- or 32-byte swizzle
      constexpr uint32_t kSboQK = (D == 128) ? 512u : 256u;
      constexpr uint32_t kIdS = idesc_mxf4nvf4(kBM, kBN);
      constexpr uint32_t kIdO = idesc_mxf4nvf4(kBM, D);
      const uint32_t tO = tmem + kColO, tQsf = tmem + kColQsf;
      bool ok = true;
      if (warp == 1) {
        auto issue_s = [&](int t) -> bool {
          const int st = t % kStages;
          const uint32_t tKsf = tmem + kColKsf + 8 * (t & 1);
          if (!wait_bar(bar(kBarKFull + st), (t / kStages) & 1)) return false;
          tc_fence_after();
#pragma unroll
          for (int kc = 0; kc < D / 64; ++kc)
            tc_cp_32x128b_x4(tKsf + 4 * kc, smem_desc(sb + L::oKsf + st * 1024 + 512 * kc, 0, 128, 0));
#pragma unroll
          for (int kc = 0; kc < D / 64; ++kc)
            mma_mxf4nvf4(tmem + kColS + (t & 1) * kBN, smem_desc(sb + L::oQ + 32 * kc, 16, kSboQK, kSw),
                         smem_desc(sb + L::oK + st * L::kK + 32 * kc, 16, kSboQK, kSw), kIdS,
                         tQsf + 4 * kc, tKsf + 4 * kc, kc > 0 ? 1u : 0u);
          if constexpr (BIAS)  // S += ones x (hi + lo)^T: the correction, in the same accumulator
            mma_tf32(tmem + kColS + (t & 1) * kBN, smem_desc(sb + L::oOnesT, 16, 256, 6),
                     smem_desc(sb + L::oBiasB + st * 4096, 16, 256, 6), idesc_tf32(kBM, kBN), 1u);
          tc_commit(bar(kBarSFull + (t & 1)));
          tc_commit(bar(kBarKEmpty + st));
          return true;
        };
        ok = wait_bar(bar(kBarQ), 0);
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int kc = 0; kc < D / 64; ++kc)
            tc_cp_32x128b_x4(tQsf + 4 * kc, smem_desc(sb + L::oQsf + 512 * kc, 0, 128, 0));
          ok = issue_s(0) && (nt < 2 || issue_s(1));
        }
        for (int t = 0; ok && t + 2 < nt; ++t) {
          if (!(ok = wait_bar(bar(kBarSEmpty + (t & 1)), (t >> 1) & 1))) break;
          ok = issue_s(t + 2);
        }
      } else {
        if (EFQ) tc_cp_32x128b_x4(tmem + TC::kOnesSf, smem_desc(sb + L::oOnesSf, 0, 128, 0));
        for (int t = 0; ok && t < nt; ++t) {
          const int st = t % kStages;
          const uint32_t tPsf = tmem + kColPsf + 8 * (t & 1);
          const uint32_t tVsf = tmem + kColVsf + 8 * (t & 1);
          if (!(ok = wait_bar(bar(kBarVFull + st), (t / kStages) & 1))) break;
          if (!(ok = wait_bar(bar(kBarPFull + (t & 1)), (t >> 1) & 1))) break;
          tc_fence_after();
          if constexpr (FP8) {
            // E4M3 P (128 bytes per row) times E4M3 V^T, 128-byte swizzle, K = 32 per MMA
#pragma unroll
            for (int c = 0; c < 4; ++c)
              mma_f8e4m3_ta(tO, tmem + TC::kP8 + 32 * (t & 1) + 8 * c,
                            smem_desc(sb + L::oV + st * L::kV + 32 * c, 16, 1024, 2),
                            idesc_f8e4m3(kBM, D), (t > 0 || c > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int c = 0; c < 2; ++c)
              tc_cp_32x128b_x4(tVsf + 4 * c, smem_desc(sb + L::oVsf + st * 1024 + 512 * c, 0, 128, 0));
            // P's codes and block scales were written to TMEM by the softmax warps
#pragma unroll
            for (int c = 0; c < 2; ++c)
              mma_mxf4nvf4_ta(tO, tmem + TC::kPc + 16 * (t & 1) + 8 * c,
                              smem_desc(sb + L::oV + st * L::kV + 32 * c, 16, 512, 4), kIdO,
                              tPsf + 4 * c, tVsf + 4 * c, (t > 0 || c > 0) ? 1u : 0u);
          }
          if (EFQ) {
#pragma unroll
            for (int c = 0; c < 2; ++c)
              mma_mxf4nvf4_ta(tmem + kColL, tmem + TC::kPc + 16 * (t & 1) + 8 * c,
                              smem_desc(sb + L::oOnes + 32 * c, 16, 512, 4), idesc_mxf4nvf4(kBM, 16),
                              tPsf + 4 * c, tmem + TC::kOnesSf, (t > 0 || c > 0) ? 1u : 0u);
          }
          tc_commit(bar(kBarO + (t & 1)));
          tc_commit(bar(kBarVEmpty + st));
        }
      }
      if (!ok) {  // drain whatever this issuer issued before giving up
        tc_commit(bar(kBarDrain + (warp - 1)));
        drain_wait(bar(kBarDrain + (warp - 1)), 0);
      }
    }
    __syncwarp();
  }
  } else {
    regs_inc<kRegsSoftmax>();
    // ------------------------------------------------------------ softmax
    const int stream = (warp - 4) >> 2;   // key tiles t with t % 2 == stream
    const int quad = warp & 3;            // TMEM lanes 32*quad .. 32*quad+31
    const int row = quad * 32 + lane;     // query row within the tile
    const int qrow = qt * kBM + row;
    const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
    float* mval = reinterpret_cast<float*>(sm + L::oRed);  // [2][128]: running max after tile t, slot t & 1
    float* lval = mval + 2 * kBM;                          // [2][128]: each stream's row sum
    const float sq = tensor_senc(*p.amax_q), sk = tensor_senc(*p.amax_k),
                sv = FP8 ? fp8_senc(*p.amax_v) : tensor_senc(*p.amax_v);
    const float dq = __fdiv_rn(1.0f, sq), dk = __fdiv_rn(1.0f, sk), dv = __fdiv_rn(1.0f, sv);
    const float c = __fmul_rn(__fmul_rn(__fmul_rn(dq, dk), p.softmax_scale), kLog2e);
    // d_P d_V; with FP8 P the row sum is kept in units of 256 p, so d_V alone
    const float fpv = FP8 ? dv : __fmul_rn(__fdiv_rn(1.0f, kTensorRange), dv);
    const uint64_t c2 = pk(c, c);
    const float c27 = __fdiv_rn(__fmul_rn(2.0f, c), 7.0f);  // EFQ: slope of the affine rule / 7
    float m_own = -INFINITY;   // running max after this stream's previous tile
    float m_last = -INFINITY;  // running max after the last tile processed
    float l = 0.0f;            // this stream's row sum, relative to m_own
    bool fail = false;
    for (int t = stream; t < nt; t += 2) {
      float s[kBN];
      bool ok = __all_sync(0xFFFFFFFFu, wait_bar(bar(kBarSFull + stream), (t >> 1) & 1));
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < kBN; cc += 32) tmem_ld32(tl + kColS + stream * kBN + cc, s + cc);
        tmem_wait_ld();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarSEmpty + stream));
      // mask: keys beyond N, and (causal) keys after the query
      const int key0 = t * kBN;
      if (key0 + kBN > p.N || (CAUSAL && key0 + kBN - 1 > qrow)) {
#pragma unroll
        for (int i = 0; i < kBN; ++i)
          if (key0 + i >= p.N || (CAUSAL && key0 + i > qrow)) s[i] = -INFINITY;
      }
      float bm[8];
#pragma unroll
      for (int bk = 0; bk < 8; ++bk) {
        const float* x = s + 16 * bk;
        const float a0 = fmax3(x[0], x[1], x[2]), a1 = fmax3(x[3], x[4], x[5]),
                    a2 = fmax3(x[6], x[7], x[8]), a3 = fmax3(x[9], x[10], x[11]),
                    a4 = fmax3(x[12], x[13], x[14]);
        bm[bk] = fmaxf(fmax3(a0, a1, a2), fmax3(a3, a4, x[15]));
      }
      const float mx = fmaxf(fmax3(bm[0], bm[1], bm[2]),
                             fmaxf(fmax3(bm[3], bm[4], bm[5]), fmax3(bm[6], bm[7], -INFINITY)));
      // running max: the previous tile's (the other stream) and this tile's
      float m_prev = -INFINITY;
      if (t > 0) {
        ok = __all_sync(0xFFFFFFFFu,
                        wait_bar(bar(kBarMax + quad * 2 + (stream ^ 1)), ((t - 1) >> 1) & 1));
        m_prev = mval[(stream ^ 1) * kBM + row];
      }
      if (!ok) {
        fail = true;
        break;
      }
      const float m_new = fmaxf(m_prev, __fmul_rn(mx, c));
      mval[stream * kBM + row] = m_new;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarMax + quad * 2 + stream));
      const float alpha = (m_prev == -INFINITY) ? 0.0f : ex2_approx(m_prev - m_new);
      const float neg_m = (m_new == -INFINITY) ? 0.0f : -m_new;
      const uint64_t nm2 = pk(neg_m, neg_m);
      uint32_t pc[FP8 ? 32 : 16];
      uint32_t sfw[2] = {0u, 0u};
      float lsum = 0.0f;
      if constexpr (FP8) {
        // FP8 P: p' = 2^(x - m + 8) = 256 p, E4M3 per key (round to nearest
        // even, the 256 keeps p' inside E4M3's range); the row sum of p'
        const float nm8 = (m_new == -INFINITY) ? 0.0f : __fsub_rn(8.0f, m_new);
        const uint64_t n8 = pk(nm8, nm8);
#pragma unroll
        for (int bk = 0; bk < 8; ++bk) {
          uint64_t acc = 0;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float u0, u1;
            upk(fma2(pk(s[16 * bk + 2 * i], s[16 * bk + 2 * i + 1]), c2, n8), u0, u1);
            const float p0 = ex2_approx(u0), p1 = ex2_approx(u1);
            const uint64_t pp = pk(p0, p1);
            acc = (i == 0) ? pp : add2(acc, pp);
            const uint32_t h = cvt_e4m3x2(p0, p1);
            if (i & 1)
              pc[4 * bk + (i >> 1)] |= h << 16;
            else
              pc[4 * bk + (i >> 1)] = h;
          }
          float a0, a1;
          upk(acc, a0, a1);
          lsum += a0 + a1;
        }
      } else if constexpr (EFQ) {
        // EFQ-Softmax: per block, E = floor(max z) - 2 and scale byte 2^(E + 10);
        // per score, code = rne(7 sat((2 (z - E) + 2) / 7)) from the bits of
        // fma(sat(s c' + o), 7, 2^23); eight codes per word by shift-and-add
        // (the eight 2^23 exponents leave the constant 0xFB000000 behind)
#pragma unroll
        for (int bk = 0; bk < 8; ++bk) {
          const float bz = __fsub_rn(__fmul_rn(bm[bk], c), m_new);  // max z of the block
          uint32_t e = 0u;
          float o7 = 0.0f;
          if (bz > -INFINITY) {
            const float Ef = floorf(bz) - 2.0f;
            const int k = __float2int_rz(Ef) + 10;
            e = k >= -6 ? (uint32_t)(k + 7) << 3 : (k >= -9 ? 1u << (k + 9) : 0u);
            o7 = __fmul_rn(fmaf(-2.0f, __fadd_rn(m_new, Ef), 2.0f), kInv7);
          }
          const uint64_t r2 = pk(kRound, kRound);
#pragma unroll
          for (int h8 = 0; h8 < 2; ++h8) {
            uint32_t f[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int j = 16 * bk + 8 * h8 + 2 * i;
              const float t0 = fma_sat(s[j], c27, o7), t1 = fma_sat(s[j + 1], c27, o7);
              float f0, f1;
              upk(fma2(pk(t0, t1), pk(7.0f, 7.0f), r2), f0, f1);
              f[2 * i] = __float_as_uint(f0);
              f[2 * i + 1] = __float_as_uint(f1);
            }
            uint32_t w = f[7];
#pragma unroll
            for (int i = 6; i >= 0; --i) w = (w << 4) + f[i];
            pc[2 * bk + h8] = w - 0xFB000000u;
          }
          sfw[bk >> 2] |= e << (8 * (bk & 3));
        }
      } else {
        // P -> NVFP4 per 16 keys with the fixed tensor scale 2688 (p <= 1):
        // p = 2^(x - m) in fp32, block scale e = E4M3(448 a_b) with
        // a_b = 2^(max_b - m), codes E2M1(p r) with r = 2688 / dec(e)
#pragma unroll
        for (int bk = 0; bk < 8; ++bk) {
          const float a = ex2_approx(fmaf(bm[bk], c, neg_m));
          const uint32_t e = cvt_e4m3(__fmul_rn(a, 448.0f));
          const float r = ptab[e];
          const uint64_t r2 = pk(r, r);
          float y[16];
          uint64_t acc = 0;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float u0, u1;
            upk(fma2(pk(s[16 * bk + 2 * i], s[16 * bk + 2 * i + 1]), c2, nm2), u0, u1);
            const uint64_t pp = pk(ex2_approx(u0), ex2_approx(u1));
            acc = (i == 0) ? pp : add2(acc, pp);
            upk(mul2(pp, r2), y[2 * i], y[2 * i + 1]);
          }
          float a0, a1;
          upk(acc, a0, a1);
          lsum += a0 + a1;
          pc[2 * bk] = cvt_e2m1x8(y);
          pc[2 * bk + 1] = cvt_e2m1x8(y + 8);
          sfw[bk >> 2] |= e << (8 * (bk & 3));
        }

      }
      // this stream's sum, carried to the new running max
      l = (m_own == -INFINITY) ? lsum : fmaf(l, ex2_approx(m_own - m_new), lsum);
      m_own = m_new;
      m_last = m_new;
      // PV of the previous tile (the other stream's) must be complete before O
      // is rescaled and before P buffer `stream` (read by PV two tiles ago) is
      // overwritten
      if (t >= 1) ok = __all_sync(0xFFFFFFFFu, wait_bar(bar(kBarO + (stream ^ 1)), ((t - 1) >> 1) & 1));
      if (!ok) {
        fail = true;
        break;
      }
      if (t >= 1 && __any_sync(0xFFFFFFFFu, alpha != 1.0f)) {
        tc_fence_after();
        const uint64_t al2 = pk(alpha, alpha);
#pragma unroll
        for (int cc = 0; cc < D + (EFQ ? 16 : 0); cc += 16) {
          float o[16];
          const uint32_t ta = tl + kColO + cc;
          tmem_ld16(ta, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 8; ++i) upk(mul2(pk(o[2 * i], o[2 * i + 1]), al2), o[2 * i], o[2 * i + 1]);
          tmem_st16(ta, o);
        }
        tmem_wait_st();
      }
      if constexpr (FP8) {
        // codes to TMEM, where PV takes them as its A operand (four per column)
        tc_fence_after();
        tmem_st32u(tl + TC::kP8 + 32 * stream, pc);
        tmem_wait_st();
      } else {
        // codes to TMEM, where PV takes them as its A operand (eight codes per
        // column), and the row's scale word of each 64-key chunk into all four
        // columns of the chunk's scale group in its own lane: no shared-memory
        // store and no proxy fence on the softmax's path
        tc_fence_after();
        tmem_st16(tl + TC::kPc + 16 * stream, reinterpret_cast<const float*>(pc));
        const uint32_t sw8[8] = {sfw[0], sfw[0], sfw[0], sfw[0], sfw[1], sfw[1], sfw[1], sfw[1]};
        tmem_st8u(tl + kColPsf + 8 * stream, sw8);
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarPFull + stream));
    }
    // ------------------------------------------------------------ epilogue
    // both streams carry their sums to the final running max (the last tile's)
    const int tlast = nt - 1;
    bool ok = !fail && __all_sync(0xFFFFFFFFu, wait_bar(bar(kBarO + (tlast & 1)), (tlast >> 1) & 1));
    if (stream != (tlast & 1) && ok)
      ok = __all_sync(0xFFFFFFFFu, wait_bar(bar(kBarMax + quad * 2 + (tlast & 1)), (tlast >> 1) & 1));
    const float m_fin = ok ? mval[(tlast & 1) * kBM + row] : 0.0f;
    const float l_own = (nt > stream && m_last != -INFINITY) ? l * ex2_approx(m_last - m_fin) : 0.0f;
    lval[stream * kBM + row] = l_own;
    fail = bar_red_or(1 + quad, 64, !ok);
    if (!fail) {
      tc_fence_after();
      float inv;
      if constexpr (EFQ) {
        // P~1 accumulated beside O in the same units: out = O d_V / (P~1)
        float lq[16];
        tmem_ld16(tl + kColL, lq);
        tmem_wait_ld();
        inv = __fdiv_rn(dv, lq[0]);
      } else {
        const float lsum = lval[row] + lval[kBM + row];
        inv = __fdiv_rn(fpv, lsum);
        if (LSE && stream == 0 && qrow < p.N &&
            FP4_CHECK(in_range((int64_t)gq * p.N + qrow, 1, (int64_t)p.B * p.H * p.N), 208))
          p.lse[(int64_t)gq * p.N + qrow] = m_fin + log2f(lsum);
      }
      constexpr int DH = D / 2;             // each stream writes half the channels
      __nv_bfloat16* dst = p.out + ((int64_t)gq * p.N + qrow) * D + stream * DH;
#pragma unroll
      for (int cc = 0; cc < DH; cc += 32) {
        float o[32];
        tmem_ld32(tl + kColO + stream * DH + cc, o);
        tmem_wait_ld();
        if (qrow < p.N && FP4_CHECK(in_range(((int64_t)gq * p.N + qrow) * D + stream * DH + cc, 32,
                                             (int64_t)p.B * p.H * p.N * D), 209)) {
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            __nv_bfloat162 v2 = __floats2bfloat162_rn(o[2 * i] * inv, o[2 * i + 1] * inv);
            w[i] = *reinterpret_cast<uint32_t*>(&v2);
          }
          uint4* d4 = reinterpret_cast<uint4*>(dst + cc);
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4)
            d4[k4] = make_uint4(w[4 * k4], w[4 * k4 + 1], w[4 * k4 + 2], w[4 * k4 + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace fp4
