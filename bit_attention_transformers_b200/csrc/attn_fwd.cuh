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
//   warp 1      TMEM owner and MMA issuer (one thread): S = Q K^T into a
//               double-buffered TMEM tile, O += P V into a TMEM accumulator
//   warps 2..9  softmax: two threads per query row, 64 keys each
// TMEM columns: S0 [0,128) S1 [128,256) O [256,256+D) scales from 384.
// Every wait is bounded (2 s of %globaltimer); on expiry the kernel sets the
// device error word, stops issuing, drains its tensor-core work and returns.
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
constexpr int kAttnThreads = 320;           // 10 warps
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr float kLog2e = 1.44269504088896340736f;

enum : unsigned { kDevErrTimeout = 1u };

// Device error word (one per device); read and cleared by fp4_status().
__device__ unsigned g_fp4_err;

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*reinterpret_cast<volatile unsigned*>(&g_fp4_err) != 0u) return false;
    if (globaltimer_ns() - t0 > kTimeoutNs) {
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

// bar.sync over the softmax warps that also ORs a per-thread flag.
__device__ __forceinline__ bool softmax_bar_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, 1, 256, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

struct AttnParams {
  const uint8_t* q_sf;
  const uint8_t* k_sf;
  const uint8_t* v_sf;
  const float* amax_q;  // absolute maxima of the source tensors
  const float* amax_k;
  const float* amax_v;
  __nv_bfloat16* out;  // [B][H][N][D]
  int H, Hkv, N, Npad, ntq;
  float softmax_scale;
};

template <int D>
struct AttnSmem {
  static constexpr int kQ = kBM * D / 2;   // Q codes tile
  static constexpr int kK = kBN * D / 2;   // K codes tile
  static constexpr int kV = D * kBN / 2;   // V^T codes tile
  static constexpr int kP = kBM * kBN / 2; // P codes tile
  static constexpr int kSfQK = (D / 64) * 512;
  static constexpr int oQ = 0;
  static constexpr int oK = oQ + kQ;
  static constexpr int oV = oK + kStages * kK;
  static constexpr int oP = oV + kStages * kV;
  static constexpr int oQsf = oP + 2 * kP;
  static constexpr int oKsf = oQsf + 1024;
  static constexpr int oVsf = oKsf + kStages * 1024;
  static constexpr int oPsf = oVsf + kStages * 1024;
  static constexpr int oRed = oPsf + 2 * 1024;  // float [2][2][128]
  static constexpr int oPtab = oRed + 2048;     // float [128]
  static constexpr int oBar = oPtab + 512;      // mbarriers
  static constexpr int oTmem = oBar + 256;
  static constexpr int kBytes = oTmem + 16 + 1024;  // + alignment slack
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
  kBarO = kBarPFull + 2,
  kBarDrain = kBarO + 1,
  kNumBars = kBarDrain + 1
};

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256, kColQsf = 384, kColKsf = 392, kColPsf = 408,
                   kColVsf = 424;

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using L = AttnSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = CAUSAL ? (p.ntq - 1 - (int)blockIdx.x) : (int)blockIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
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
      mbar_init(bar(kBarSEmpty + s), 8);
      mbar_init(bar(kBarPFull + s), 8);
    }
    mbar_init(bar(kBarO), 1);
    mbar_init(bar(kBarDrain), 1);
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + L::oTmem);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      bool ok = true;
      const int qrow0 = gq * p.Npad + qt * kBM;
      mbar_arrive_expect_tx(bar(kBarQ), L::kQ + L::kSfQK);
      tma_load_2d(sb + L::oQ, &tmQ, 0, qrow0, bar(kBarQ));
      bulk_load(sb + L::oQsf, p.q_sf + ((int64_t)gq * (p.Npad / kBM) + qt) * L::kSfQK, L::kSfQK,
                bar(kBarQ));
      for (int j = 0; j < nt && ok; ++j) {
        const int st = j % kStages;
        const uint32_t pe = ((j / kStages) - 1) & 1;
        if (j >= kStages && !(ok = wait_bar(bar(kBarKEmpty + st), pe))) break;
        mbar_arrive_expect_tx(bar(kBarKFull + st), L::kK + L::kSfQK);
        tma_load_2d(sb + L::oK + st * L::kK, &tmK, 0, gk * p.Npad + j * kBN, bar(kBarKFull + st));
        bulk_load(sb + L::oKsf + st * 1024,
                  p.k_sf + ((int64_t)gk * (p.Npad / kBN) + j) * L::kSfQK, L::kSfQK,
                  bar(kBarKFull + st));
        if (j >= kStages && !(ok = wait_bar(bar(kBarVEmpty + st), pe))) break;
        mbar_arrive_expect_tx(bar(kBarVFull + st), L::kV + 1024);
        tma_load_2d(sb + L::oV + st * L::kV, &tmV, j * (kBN / 2), gk * D, bar(kBarVFull + st));
        bulk_load(sb + L::oVsf + st * 1024, p.v_sf + ((int64_t)gk * (p.Npad / 64) + 2 * j) * 512,
                  1024, bar(kBarVFull + st));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kSw = (D == 128) ? 4u : 6u;     // 64- or 32-byte swizzle
      constexpr uint32_t kSboQK = (D == 128) ? 512u : 256u;
      constexpr uint32_t kIdS = idesc_mxf4nvf4(kBM, kBN);
      constexpr uint32_t kIdO = idesc_mxf4nvf4(kBM, D);
      const uint32_t tS[2] = {tmem + kColS, tmem + kColS + kBN};
      const uint32_t tO = tmem + kColO, tQsf = tmem + kColQsf;
      bool ok = wait_bar(bar(kBarQ), 0);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int kc = 0; kc < D / 64; ++kc)
          tc_cp_32x128b_x4(tQsf + 4 * kc, smem_desc(sb + L::oQsf + 512 * kc, 0, 128, 0));
      }
      for (int j = 0; ok && j <= nt; ++j) {
        if (j < nt) {
          const int st = j % kStages;
          const uint32_t tKsf = tmem + kColKsf + 8 * (j & 1);
          if (!(ok = wait_bar(bar(kBarKFull + st), (j / kStages) & 1))) break;
          if (j >= 2 && !(ok = wait_bar(bar(kBarSEmpty + (j & 1)), ((j >> 1) - 1) & 1))) break;
          tc_fence_after();
#pragma unroll
          for (int kc = 0; kc < D / 64; ++kc)
            tc_cp_32x128b_x4(tKsf + 4 * kc,
                             smem_desc(sb + L::oKsf + st * 1024 + 512 * kc, 0, 128, 0));
#pragma unroll
          for (int kc = 0; kc < D / 64; ++kc)
            mma_mxf4nvf4(tS[j & 1], smem_desc(sb + L::oQ + 32 * kc, 16, kSboQK, kSw),
                         smem_desc(sb + L::oK + st * L::kK + 32 * kc, 16, kSboQK, kSw), kIdS,
                         tQsf + 4 * kc, tKsf + 4 * kc, kc > 0 ? 1u : 0u);
          tc_commit(bar(kBarSFull + (j & 1)));
          tc_commit(bar(kBarKEmpty + st));
        }
        if (j >= 1) {
          const int t = j - 1, st = t % kStages;
          const uint32_t tPsf = tmem + kColPsf + 8 * (t & 1);
          const uint32_t tVsf = tmem + kColVsf + 8 * (t & 1);
          if (!(ok = wait_bar(bar(kBarVFull + st), (t / kStages) & 1))) break;
          if (!(ok = wait_bar(bar(kBarPFull + (t & 1)), (t >> 1) & 1))) break;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            tc_cp_32x128b_x4(tPsf + 4 * c,
                             smem_desc(sb + L::oPsf + (t & 1) * 1024 + 512 * c, 0, 128, 0));
            tc_cp_32x128b_x4(tVsf + 4 * c,
                             smem_desc(sb + L::oVsf + st * 1024 + 512 * c, 0, 128, 0));
          }
#pragma unroll
          for (int c = 0; c < 2; ++c)
            mma_mxf4nvf4(tO, smem_desc(sb + L::oP + (t & 1) * L::kP + 32 * c, 16, 512, 4),
                         smem_desc(sb + L::oV + st * L::kV + 32 * c, 16, 512, 4), kIdO,
                         tPsf + 4 * c, tVsf + 4 * c, (t > 0 || c > 0) ? 1u : 0u);
          tc_commit(bar(kBarO));
          tc_commit(bar(kBarVEmpty + st));
        }
      }
      if (!ok) {  // drain whatever was issued before giving up
        tc_commit(bar(kBarDrain));
        drain_wait(bar(kBarDrain), 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int sw = warp - 2;
    const int half = sw >> 2;             // keys [64*half, 64*half+64) of each tile
    const int quad = warp & 3;            // TMEM lanes 32*quad .. 32*quad+31
    const int row = quad * 32 + lane;     // query row within the tile
    const int qrow = qt * kBM + row;
    const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
    float* red = reinterpret_cast<float*>(sm + L::oRed);
    const float sq = tensor_senc(*p.amax_q), sk = tensor_senc(*p.amax_k),
                sv = tensor_senc(*p.amax_v);
    const float dq = __fdiv_rn(1.0f, sq), dk = __fdiv_rn(1.0f, sk), dv = __fdiv_rn(1.0f, sv);
    const float c = __fmul_rn(__fmul_rn(__fmul_rn(dq, dk), p.softmax_scale), kLog2e);
    const float fpv = __fmul_rn(__fdiv_rn(1.0f, kTensorRange), dv);  // d_P * d_V
    float m_old = -INFINITY, l = 0.0f;
    bool fail = false;
    int j = 0;
    for (; j < nt; ++j) {
      float s[64];
      bool ok = __all_sync(0xFFFFFFFFu, wait_bar(bar(kBarSFull + (j & 1)), (j >> 1) & 1));
      if (ok) {
        tc_fence_after();
        tmem_ld32(tl + kColS + (j & 1) * kBN + half * 64, s);
        tmem_ld32(tl + kColS + (j & 1) * kBN + half * 64 + 32, s + 32);
        tmem_wait_ld();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarSEmpty + (j & 1)));
      // mask: keys beyond N, and (causal) keys after the query
      const int key0 = j * kBN + half * 64;
      if (key0 + 64 > p.N || (CAUSAL && key0 + 63 > qrow)) {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (key0 + i >= p.N || (CAUSAL && key0 + i > qrow)) s[i] = -INFINITY;
      }
      float bm[4];
#pragma unroll
      for (int bk = 0; bk < 4; ++bk) {
        float m0 = fmax3(s[16 * bk + 0], s[16 * bk + 1], s[16 * bk + 2]);
        float m1 = fmax3(s[16 * bk + 3], s[16 * bk + 4], s[16 * bk + 5]);
        float m2 = fmax3(s[16 * bk + 6], s[16 * bk + 7], s[16 * bk + 8]);
        float m3 = fmax3(s[16 * bk + 9], s[16 * bk + 10], s[16 * bk + 11]);
        float m4 = fmax3(s[16 * bk + 12], s[16 * bk + 13], s[16 * bk + 14]);
        bm[bk] = fmax3(fmax3(m0, m1, m2), fmax3(m3, m4, s[16 * bk + 15]), -INFINITY);
      }
      const float tmax = fmax3(fmaxf(bm[0], bm[1]), bm[2], bm[3]);
      red[((j & 1) * 2 + half) * kBM + row] = tmax;
      fail = softmax_bar_or(!ok || fail);
      if (fail) break;
      const float mx = fmaxf(tmax, red[((j & 1) * 2 + (half ^ 1)) * kBM + row]);
      const float m_new = fmaxf(m_old, __fmul_rn(mx, c));
      const float alpha = (m_old == -INFINITY) ? 0.0f : ex2_approx(m_old - m_new);
      const float neg_m = (m_new == -INFINITY) ? 0.0f : -m_new;
      float ls = 0.0f;
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        s[i] = ex2_approx(fmaf(s[i], c, neg_m));
        ls += s[i];
      }
      l = fmaf(l, alpha, ls);
      // P -> NVFP4 per 16 keys (fixed tensor scale 2688: p <= 1)
      uint32_t pc[8];
      uint32_t sfw = 0;
#pragma unroll
      for (int bk = 0; bk < 4; ++bk) {
        const float a = ex2_approx(fmaf(bm[bk], c, neg_m));
        const uint32_t e = cvt_e4m3(__fmul_rn(a, 448.0f));
        const float r = ptab[e];
        float y[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) y[i] = __fmul_rn(s[16 * bk + i], r);
        pc[2 * bk] = cvt_e2m1x8(y);
        pc[2 * bk + 1] = cvt_e2m1x8(y + 8);
        sfw |= e << (8 * bk);
      }
      // PV of the previous tile must be complete before O is rescaled and
      // before this tile's P buffer (last read two tiles ago) is overwritten
      if (j >= 1) ok = __all_sync(0xFFFFFFFFu, wait_bar(bar(kBarO), (j - 1) & 1));
      if (!ok) {
        fail = true;
      } else if (j >= 1 && __any_sync(0xFFFFFFFFu, alpha != 1.0f)) {
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < D / 2; cc += 16) {
          float o[16];
          const uint32_t ta = tl + kColO + half * (D / 2) + cc;
          tmem_ld16(ta, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] *= alpha;
          tmem_st16(ta, o);
        }
        tmem_wait_st();
      }
      uint8_t* pbuf = sm + L::oP + (j & 1) * L::kP;
#pragma unroll
      for (int k2 = 0; k2 < 2; ++k2) {
        const int chunk = (half * 2 + k2) ^ ((row >> 1) & 3);  // 64-byte swizzle
        *reinterpret_cast<uint4*>(pbuf + row * 64 + chunk * 16) =
            make_uint4(pc[4 * k2], pc[4 * k2 + 1], pc[4 * k2 + 2], pc[4 * k2 + 3]);
      }
      *reinterpret_cast<uint32_t*>(sm + L::oPsf + (j & 1) * 1024 + half * 512 + (row & 31) * 16 +
                                   (row >> 5) * 4) = sfw;
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarPFull + (j & 1)));
      m_old = m_new;
    }
    // ------------------------------------------------------------ epilogue
    bool ok = !fail && __all_sync(0xFFFFFFFFu, wait_bar(bar(kBarO), (nt - 1) & 1));
    red[((nt & 1) * 2 + half) * kBM + row] = l;
    fail = softmax_bar_or(!ok);
    if (!fail) {
      tc_fence_after();
      const float ltot = l + red[((nt & 1) * 2 + (half ^ 1)) * kBM + row];
      const float inv = __fdiv_rn(fpv, ltot);
      __nv_bfloat16* dst = p.out + ((int64_t)gq * p.N + qrow) * D + half * (D / 2);
#pragma unroll
      for (int cc = 0; cc < D / 2; cc += 32) {
        float o[32];
        tmem_ld32(tl + kColO + half * (D / 2) + cc, o);
        tmem_wait_ld();
        if (qrow < p.N) {
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
