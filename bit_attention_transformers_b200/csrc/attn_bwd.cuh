// FP4 attention backward on sm_100a.
//
// Reading [Attn-QAT abstract, arxiv listing "Attn-QAT: 4-Bit Attention With
// Quantization-Aware Training": the backward recomputes the scores in the
// forward's low precision, and FlashAttention's D = dO . O holds an implicit
// precision assumption]:
//   S = Q^ K^T from the forward's NVFP4 operands (Q^, K^, V^ = val(code) dec(e),
//       contraction units, exact in bf16; the tensor scales d_Q, d_K, d_V are
//       applied as fp32 factors), x = S c with the forward's c
//   P_ij = 2^(x_ij - lse_i), lse from the forward (log2 units)
//   dP = d_V dO V^T,  D_i = sum_j P_ij dP_ij  (from this P and V~, not dO . O)
//   dS = P (dP - D),  dq = scale d_K dS K^,  dk = scale d_Q dS^T Q^,  dv = P^T dO
// with straight-through quantisers (the gradients of q~, k~, v~ serve as
// those of q, k, v).
//
// Kernels (contractions on tcgen05 with fp32 accumulators in TMEM: the dk/dv
// kernel's S^T on kind::mxf4nvf4 from the forward's NVFP4 codes, every other
// one on kind::f16 with bf16 operands, K-major with the 128-byte swizzle,
// transposed copies prepared by the pre-kernels so that no MN-major operand is
// needed):
//   quant_rows_kernel  the forward's own quantiser: Q's and K's NVFP4 codes
//       and block scales, for S^T
//   fq_rows_kernel / fq_tokens_kernel  the forward's quantisers, decoded to
//       bf16 (Q^, K^ and their transposes; V^), bit-identical codes and scales
//   pad_transpose_kernel  dO padded to Npad rows, and dO^T
//   lse_pad_kernel        lse padded with +inf (padded rows get P = 0)
//   bwd_dq_kernel   one CTA per 128 query rows, one pass over the key tiles:
//       D and dQ (dQ from two sums accumulated in TMEM, see the kernel)
//   sf64_kernel     Q's block scales regrouped per 64-query tile
//   bwd_dkdv_kernel one CTA per 128 keys: over the query tiles of every query
//       head of its key/value head, S^T from the NVFP4 codes (kind::mxf4nvf4),
//       dV += P^T dO and dK += dS^T Q^ in TMEM (P^T and dS^T from TMEM)
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "attn_fwd.cuh"  // the bounded-wait limit and the device error word
#include "ptx.cuh"
#include "quantize.cuh"

namespace fp4 {

// dk/dv kernel: warps 0 and 2 load, warp 1 issues MMAs, warps 4-11 compute
// (two warps per TMEM lane quarter, each on half of a tile's 64 queries)
constexpr int kBwdThreads = 384;
constexpr int kBwdQ = 128;        // dq kernel: query rows per CTA
constexpr int kBwdKt = 64;        // dq kernel: keys per tile
constexpr int kBwdK = 128;        // dk/dv kernel: keys per CTA
constexpr int kBwdQt = 64;        // dk/dv kernel: queries per tile

// Instruction descriptor of kind::f16 with bf16 A and B (both K-major), fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16(uint32_t M, uint32_t N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 operands, K = 16 per instruction.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, bf16 operands, K = 16 per instruction; A
// (M = 128 rows, one per TMEM lane) holds two consecutive K elements per
// 32-bit column, the even one in the low half.
__device__ __forceinline__ void mma_bf16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// K-major bf16 operand with the 128-byte swizzle: `rows` rows, K split in
// 64-element atoms stored one after another (rows x 128 bytes each). The
// descriptor of K step s (16 elements) starts 32 bytes further inside an atom.
__device__ __forceinline__ uint64_t kmaj_desc(uint32_t base, int rows, int s) {
  return smem_desc(base + (s >> 2) * rows * 128 + (s & 3) * 32, 16, 1024, 2);
}

// Decoded E2M1 magnitude times the block scale: code c (sign bit 3), scale byte e.
__device__ __forceinline__ float e2m1_value(uint32_t c) {
  const uint32_t m = c & 7u;
  const float mag = m < 4 ? 0.5f * (float)m : (m == 4 ? 2.0f : (m == 5 ? 3.0f : (m == 6 ? 4.0f : 6.0f)));
  return (c & 8u) ? -mag : mag;
}

// 16 decoded values of one block from its codes (lo: elements 0..7, hi: 8..15).
__device__ __forceinline__ void decode_block16(uint32_t lo, uint32_t hi, uint32_t e, float* out) {
  const float de = e4m3_to_f32(e);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    out[i] = e2m1_value((lo >> (4 * i)) & 15u) * de;
    out[8 + i] = e2m1_value((hi >> (4 * i)) & 15u) * de;
  }
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ---------------------------------------------------------- pre-kernels ----
// Q or K [G][N][D] -> Q^ [G][Npad][D] and Q^T [G][D][Npad] (bf16, decoded
// NVFP4 with blocks of 16 along D, the forward's quantiser). One CTA per
// (group, 128-row tile); thread = row.
template <int D>
__global__ void __launch_bounds__(128) fq_rows_kernel(const __nv_bfloat16* __restrict__ x, int N,
                                                      int Npad, const float* __restrict__ amax,
                                                      __nv_bfloat16* __restrict__ xh,
                                                      __nv_bfloat16* __restrict__ xt) {
  __shared__ __align__(16) uint16_t tile[128 * (D + 8)];  // +8: no bank conflicts on the transpose
  constexpr int LD = D + 8;
  const int ntile = Npad >> 7;
  const int64_t g = blockIdx.x / ntile;
  const int t = blockIdx.x % ntile;
  const float s_enc = tensor_senc(*amax);
  const int r = threadIdx.x, n = t * 128 + r;
  __nv_bfloat16* dst = xh + (g * Npad + n) * D;
#pragma unroll 1
  for (int kb = 0; kb < D / 16; ++kb) {
    float xv[16];
    if (n < N) {
      const __nv_bfloat16* src = x + ((g * N + n) * D + kb * 16);
      bf16x8_to_f32(ld_nc_v4(src), xv);
      bf16x8_to_f32(ld_nc_v4(src + 8), xv + 8);
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) xv[i] = 0.0f;
    }
    uint32_t lo, hi;
    const uint32_t e = quant_block16(xv, s_enc, lo, hi);
    float yv[16];
    decode_block16(lo, hi, e, yv);
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = pack_bf16(yv[2 * i], yv[2 * i + 1]);
    uint4* d4 = reinterpret_cast<uint4*>(dst + kb * 16);
    d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
    d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
    uint32_t* s32 = reinterpret_cast<uint32_t*>(&tile[r * LD + kb * 16]);
#pragma unroll
    for (int i = 0; i < 8; ++i) s32[i] = w[i];
  }
  __syncthreads();
  // transpose: one channel per thread, 128 consecutive rows written as 256 bytes
  for (int d = threadIdx.x; d < D; d += 128) {
    uint32_t w[64];
#pragma unroll
    for (int i = 0; i < 64; ++i)
      w[i] = (uint32_t)tile[(2 * i) * LD + d] | ((uint32_t)tile[(2 * i + 1) * LD + d] << 16);
    if (!FP4_CHECK(in_range((g * D + d) * (int64_t)Npad + t * 128, 128,
                            (int64_t)(gridDim.x / ntile) * D * Npad), 321))
      continue;
    uint4* d4 = reinterpret_cast<uint4*>(xt + (g * D + d) * (int64_t)Npad + t * 128);
#pragma unroll
    for (int k = 0; k < 16; ++k) d4[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
  }
}

// V [G][N][D] -> V^ [G][Npad][D] (bf16, decoded NVFP4 with blocks of 16 tokens
// per channel, the forward's quantiser). One CTA per (group, 128-token tile);
// thread = channel.
template <int D>
__global__ void __launch_bounds__(128) fq_tokens_kernel(const __nv_bfloat16* __restrict__ v, int N,
                                                        int Npad, const float* __restrict__ amax,
                                                        __nv_bfloat16* __restrict__ vh) {
  __shared__ __align__(16) uint16_t tile[128 * D];
  const int ntile = Npad >> 7;
  const int64_t g = blockIdx.x / ntile;
  const int t = blockIdx.x % ntile;
  const float s_enc = tensor_senc(*amax);
  constexpr int VEC = D / 8;
  for (int idx = threadIdx.x; idx < 128 * VEC; idx += blockDim.x) {
    const int tok = idx / VEC, c = idx % VEC;
    const int n = t * 128 + tok;
    uint4 w = make_uint4(0, 0, 0, 0);
    if (n < N) w = ld_nc_v4(v + ((g * N + n) * D + c * 8));
    *reinterpret_cast<uint4*>(&tile[tok * D + c * 8]) = w;
  }
  __syncthreads();
  const int d = threadIdx.x;
  if (d < D) {
#pragma unroll 1
    for (int b = 0; b < 8; ++b) {
      float xv[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        xv[i] = __uint_as_float((uint32_t)tile[(b * 16 + i) * D + d] << 16);
      uint32_t lo, hi;
      const uint32_t e = quant_block16(xv, s_enc, lo, hi);
      float yv[16];
      decode_block16(lo, hi, e, yv);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        __nv_bfloat16 h = __float2bfloat16_rn(yv[i]);
        tile[(b * 16 + i) * D + d] = *reinterpret_cast<uint16_t*>(&h);
      }
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < 128 * VEC; idx += blockDim.x) {
    const int tok = idx / VEC, c = idx % VEC;
    *reinterpret_cast<uint4*>(vh + ((g * Npad + t * 128 + tok) * D + c * 8)) =
        *reinterpret_cast<const uint4*>(&tile[tok * D + c * 8]);
  }
}

// dO [G][N][D] -> dO [G][Npad][D] (rows >= N zero) and dO^T [G][D][Npad].
template <int D>
__global__ void __launch_bounds__(128) pad_transpose_kernel(const __nv_bfloat16* __restrict__ x,
                                                            int N, int Npad,
                                                            __nv_bfloat16* __restrict__ xp,
                                                            __nv_bfloat16* __restrict__ xt) {
  __shared__ __align__(16) uint16_t tile[128 * (D + 8)];
  constexpr int LD = D + 8, VEC = D / 8;
  const int ntile = Npad >> 7;
  const int64_t g = blockIdx.x / ntile;
  const int t = blockIdx.x % ntile;
  for (int idx = threadIdx.x; idx < 128 * VEC; idx += blockDim.x) {
    const int tok = idx / VEC, c = idx % VEC;
    const int n = t * 128 + tok;
    uint4 w = make_uint4(0, 0, 0, 0);
    if (n < N) w = ld_nc_v4(x + ((g * N + n) * D + c * 8));
    *reinterpret_cast<uint4*>(xp + ((g * Npad + n) * D + c * 8)) = w;
    uint32_t* s32 = reinterpret_cast<uint32_t*>(&tile[tok * LD + c * 8]);
    s32[0] = w.x;
    s32[1] = w.y;
    s32[2] = w.z;
    s32[3] = w.w;
  }
  __syncthreads();
  for (int d = threadIdx.x; d < D; d += 128) {
    uint32_t w[64];
#pragma unroll
    for (int i = 0; i < 64; ++i)
      w[i] = (uint32_t)tile[(2 * i) * LD + d] | ((uint32_t)tile[(2 * i + 1) * LD + d] << 16);
    if (!FP4_CHECK(in_range((g * D + d) * (int64_t)Npad + t * 128, 128,
                            (int64_t)(gridDim.x / ntile) * D * Npad), 322))
      continue;
    uint4* d4 = reinterpret_cast<uint4*>(xt + (g * D + d) * (int64_t)Npad + t * 128);
#pragma unroll
    for (int k = 0; k < 16; ++k) d4[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
  }
}

// Block scales of Q in the forward's layout (atoms of 128 rows: row r of a
// 64-element chunk at byte (r % 32) 16 + (r / 32) 4 + k) -> one atom per
// 64-row tile whose 4-byte columns 0 and 1 hold the tile's rows: the lower
// tile's atom is the same bytes, the upper tile's swaps the two 8-byte halves
// of every 16-byte lane. One thread per 16 bytes of the input.
__global__ void sf64_kernel(const uint4* __restrict__ sf, int64_t n16, int atom16,
                            uint4* __restrict__ sf64) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t tile = i / atom16, j = i % atom16;
    if (!FP4_CHECK(in_range((2 * tile + 1) * atom16 + j, 1, 2 * n16), 323)) continue;
    const uint4 w = sf[i];
    sf64[(2 * tile) * atom16 + j] = w;
    sf64[(2 * tile + 1) * atom16 + j] = make_uint4(w.z, w.w, w.x, w.y);
  }
}

// lse [G][N] -> [G][Npad], +inf beyond N.
__global__ void lse_pad_kernel(const float* __restrict__ lse, int64_t G, int N, int Npad,
                               float* __restrict__ out) {
  const int64_t total = G * Npad;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t g = i / Npad;
    const int n = (int)(i % Npad);
    out[i] = n < N ? lse[g * N + n] : INFINITY;
  }
}

struct BwdParams {
  const float* amax;   // [3]: Q, K, V maxima (the forward's tensor scales)
  const float* lse;    // [B*H][Npad], +inf on padded rows
  float* Dvec;         // [B*H][Npad]: D, written by the dq kernel
  const __nv_bfloat16* out;  // [B][H][N][D]: the forward's output O (centres dP, dq kernel)
  const uint8_t* k_sf;       // K block scales, the forward's layout (one atom set per 128 keys)
  const uint8_t* q_sf64;     // Q block scales, one atom set per 64-query tile (sf64_kernel)
  __nv_bfloat16* dq;   // [B][H][N][D]
  __nv_bfloat16* dk;   // [B][Hkv][N][D]
  __nv_bfloat16* dv;
  int H, Hkv, N, Npad;
  float softmax_scale;
};

struct BwdScales {
  float c, dv, sdq, sdk;  // score multiplier, d_V, scale d_K (for dq), scale d_Q (for dk)
};

__device__ __forceinline__ BwdScales bwd_scales(const BwdParams& p) {
  const float dq = __fdiv_rn(1.0f, tensor_senc(p.amax[0]));
  const float dk = __fdiv_rn(1.0f, tensor_senc(p.amax[1]));
  const float dv = __fdiv_rn(1.0f, tensor_senc(p.amax[2]));
  BwdScales s;
  s.c = __fmul_rn(__fmul_rn(__fmul_rn(dq, dk), p.softmax_scale), kLog2e);
  s.dv = dv;
  s.sdq = __fmul_rn(p.softmax_scale, dk);
  s.sdk = __fmul_rn(p.softmax_scale, dq);
  return s;
}

// Bounded wait (the forward's rule: a device error word and a time limit).
__device__ __forceinline__ bool bwd_wait(uint32_t bar, uint32_t parity) {
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

// ------------------------------------------------------------- dq kernel ----
constexpr int kDqThreads = 384;  // warps 0-3 control, 4-11 compute (two warpgroups)
constexpr uint32_t kDqRegsCtl = 56, kDqRegsCompute = 224;  // 128 x 56 + 256 x 224 = 384 x 168

// Key tiles pass once. D_i is not known until every key has been seen, so
// dQ_i = scale d_K sum_j P_ij (dP_ij - D_i) K^_j is split into two sums that
// are both accumulated in that one pass (dP in real units, d_V applied):
//   A_i = sum_j P_ij (dP_ij - c_i) K^_j,   B_i = sum_j P_ij K^_j,
//   dQ_i = scale d_K (A_i - (D_i - c_i) B_i),
// an identity for any per-row constant c_i, with D_i = D'_i + c_i sum_j P_ij
// and D'_i = sum_j P_ij (dP_ij - c_i) formed in the same pass, so D is still
// this P's and v~'s. c_i = dO_i . O_i with the forward's output O: O_i is
// sum_j P_ij v~_j up to the FP4 rounding of P, so c_i is close to D_i, the
// terms of A are as small as those of dS and the subtraction at the end
// cancels nothing large (with c_i = 0 a row whose P sits on one key loses
// dQ to the bf16 rounding of P dP). Only the rounding depends on O.
// Ring A (K^, V^) feeds S and dP and is released when they complete; ring B
// (K^T) feeds A and B a tile later; each ring has its own producer warp.
// Warp 1 issues S and dP, warp 3 issues A and B, so that neither kind waits
// behind the other's barriers.
constexpr int kDqRingA = 2, kDqRingB = 2;

template <int D>
struct BwdDqSmem {
  static constexpr int kQ = kBwdQ * D * 2;    // Q^ tile, bf16
  static constexpr int kK = kBwdKt * D * 2;   // K^ tile
  static constexpr int kKT = D * kBwdKt * 2;  // K^T tile (D rows x 64 keys)
  static constexpr int kPT = kBwdQ * kBwdKt * 2;  // one 128 x 64 bf16 operand tile
  static constexpr int oQ = 0;
  static constexpr int oDO = oQ + kQ;
  static constexpr int oA = oDO + kQ;                // [kDqRingA]: K^ then V^
  static constexpr int oB = oA + kDqRingA * 2 * kK;  // [kDqRingB]: K^T
  static constexpr int oP = oB + kDqRingB * kKT;     // [2 streams]: P then P (dP - c), bf16
  static constexpr int oBar = oP + 2 * 2 * kPT;
  static constexpr int oTmem = oBar + 256;
  static constexpr int kBytes = oTmem + 16 + 1024;
  static_assert(kBytes <= 232448, "shared memory of one CTA");
};

enum : int {
  kDqBarQ = 0,
  kDqBarFullA = 1,                        // [kDqRingA]
  kDqBarEmptyA = kDqBarFullA + kDqRingA,  // [kDqRingA]
  kDqBarFullB = kDqBarEmptyA + kDqRingA,  // [kDqRingB]
  kDqBarEmptyB = kDqBarFullB + kDqRingB,  // [kDqRingB]
  kDqBarSFull = kDqBarEmptyB + kDqRingB,  // [2] S/dP buffers (= compute streams)
  kDqBarSEmpty = kDqBarSFull + 2,         // [2]
  kDqBarPFull = kDqBarSEmpty + 2,         // [2] P / P (dP - c) buffers
  kDqBarPEmpty = kDqBarPFull + 2,         // [2]
  kDqBarDone = kDqBarPEmpty + 2,          // every A / B contraction complete
  kDqBarDoneS = kDqBarDone + 1,           // every S / dP contraction complete
  kDqNumBars = kDqBarDoneS + 1,
};
static_assert(kDqNumBars * 8 <= 256, "barrier area");

// One CTA per (128-query tile, head, batch). Two compute streams (warpgroups)
// take alternate key tiles, so that one forms its P while the tensor core
// works for the other. TMEM: S[b] at 128 b, dP[b] at 128 b + 64 (64 columns
// each, b = tile parity = stream), A at 256, B at 256 + D.
template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kDqThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmKT, const BwdParams p) {
  using L = BwdDqSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int gq = b * p.H + h;
  const int gk = b * p.Hkv + h / (p.H / p.Hkv);
  const int nk_all = (p.N + kBwdKt - 1) / kBwdKt;
  const int nkt = CAUSAL ? min(nk_all, (qt * kBwdQ + kBwdQ - 1) / kBwdKt + 1) : nk_all;
  auto bar = [&](int i) -> uint32_t { return sb + L::oBar + 8 * i; };
  if (threadIdx.x == 0) {
    mbar_init(bar(kDqBarQ), 1);
    for (int s = 0; s < kDqRingA; ++s) {
      mbar_init(bar(kDqBarFullA + s), 1);
      mbar_init(bar(kDqBarEmptyA + s), 1);
    }
    for (int s = 0; s < kDqRingB; ++s) {
      mbar_init(bar(kDqBarFullB + s), 1);
      mbar_init(bar(kDqBarEmptyB + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kDqBarSFull + s), 1);
      mbar_init(bar(kDqBarSEmpty + s), 4);
      mbar_init(bar(kDqBarPFull + s), 4);
      mbar_init(bar(kDqBarPEmpty + s), 1);
    }
    mbar_init(bar(kDqBarDone), 1);
    mbar_init(bar(kDqBarDoneS), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sb + L::oTmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + L::oTmem);
  constexpr int NA = D / 64;  // 64-element atoms along D

  if (warp < 4) {
    regs_dec<kDqRegsCtl>();
    if (warp == 0 && lane == 0) {
      bool ok = true;
      int issued = 0;
      const int64_t Gq = (int64_t)gridDim.z * p.H, Gk = (int64_t)gridDim.z * p.Hkv;
      mbar_arrive_expect_tx(bar(kDqBarQ), 2 * L::kQ);
      for (int a = 0; a < NA; ++a) {
        if (!FP4_CHECK(tma_ok(a * 64, 64, D, 2, gq * p.Npad + qt * kBwdQ, kBwdQ, Gq * p.Npad), 301))
          continue;
        tma_load_2d(sb + L::oQ + a * kBwdQ * 128, &tmQ, a * 64, gq * p.Npad + qt * kBwdQ, bar(kDqBarQ));
        tma_load_2d(sb + L::oDO + a * kBwdQ * 128, &tmDO, a * 64, gq * p.Npad + qt * kBwdQ,
                    bar(kDqBarQ));
      }
      for (int t = 0; t < nkt && ok; ++t) {  // ring A: K^ and V^
        const int st = t % kDqRingA;
        if (t >= kDqRingA && !(ok = bwd_wait(bar(kDqBarEmptyA + st), ((t / kDqRingA) - 1) & 1)))
          break;
        const uint32_t base = sb + L::oA + st * 2 * L::kK;
        mbar_arrive_expect_tx(bar(kDqBarFullA + st), 2 * L::kK);
        for (int a = 0; a < NA; ++a) {
          if (!FP4_CHECK(tma_ok(a * 64, 64, D, 2, gk * p.Npad + t * kBwdKt, kBwdKt, Gk * p.Npad),
                         302))
            continue;
          tma_load_2d(base + a * kBwdKt * 128, &tmK, a * 64, gk * p.Npad + t * kBwdKt,
                      bar(kDqBarFullA + st));
          tma_load_2d(base + L::kK + a * kBwdKt * 128, &tmV, a * 64, gk * p.Npad + t * kBwdKt,
                      bar(kDqBarFullA + st));
        }
        issued = t + 1;
      }
      // copies still in flight after a failed wait land before the CTA exits
      drain_wait(bar(kDqBarQ), 0);
      for (int t = max(0, issued - kDqRingA); t < issued; ++t)
        drain_wait(bar(kDqBarFullA + t % kDqRingA), (t / kDqRingA) & 1);
    } else if (warp == 2 && lane == 0) {
      bool ok = true;
      int issued = 0;
      for (int t = 0; t < nkt && ok; ++t) {  // ring B: K^T
        const int st = t % kDqRingB;
        if (t >= kDqRingB && !(ok = bwd_wait(bar(kDqBarEmptyB + st), ((t / kDqRingB) - 1) & 1)))
          break;
        mbar_arrive_expect_tx(bar(kDqBarFullB + st), L::kKT);
        if (FP4_CHECK(tma_ok(t * kBwdKt, kBwdKt, p.Npad, 2, (int64_t)gk * D, D,
                             (int64_t)gridDim.z * p.Hkv * D), 303))
          tma_load_2d(sb + L::oB + st * L::kKT, &tmKT, t * kBwdKt, gk * D, bar(kDqBarFullB + st));
        issued = t + 1;
      }
      for (int t = max(0, issued - kDqRingB); t < issued; ++t)
        drain_wait(bar(kDqBarFullB + t % kDqRingB), (t / kDqRingB) & 1);
    } else if (warp == 1 && lane == 0) {  // S = Q^ K^T and dP = dO V^T of every key tile
      bool ok = bwd_wait(bar(kDqBarQ), 0);
      const uint32_t idS = idesc_bf16(kBwdQ, kBwdKt);
      for (int t = 0; t < nkt && ok; ++t) {
        const int st = t % kDqRingA, buf = t & 1;
        if (!(ok = bwd_wait(bar(kDqBarFullA + st), (t / kDqRingA) & 1))) break;
        if (t >= 2 && !(ok = bwd_wait(bar(kDqBarSEmpty + buf), ((t >> 1) - 1) & 1))) break;
        tc_fence_after();
        const uint32_t base = sb + L::oA + st * 2 * L::kK;
#pragma unroll
        for (int s = 0; s < D / 16; ++s) {
          mma_bf16(tmem + buf * 128, kmaj_desc(sb + L::oQ, kBwdQ, s), kmaj_desc(base, kBwdKt, s),
                   idS, s > 0 ? 1u : 0u);
          mma_bf16(tmem + buf * 128 + 64, kmaj_desc(sb + L::oDO, kBwdQ, s),
                   kmaj_desc(base + L::kK, kBwdKt, s), idS, s > 0 ? 1u : 0u);
        }
        tc_commit(bar(kDqBarSFull + buf));
        tc_commit(bar(kDqBarEmptyA + st));
      }
      tc_commit(bar(kDqBarDoneS));
      drain_wait(bar(kDqBarDoneS), 0);  // every MMA complete before TMEM is freed
    } else if (warp == 3 && lane == 0) {  // A += (P (dP - c)) K^ and B += P K^, a tile behind
      bool ok = true;
      const uint32_t idQ = idesc_bf16(kBwdQ, D);
      for (int t = 0; t < nkt && ok; ++t) {
        const int buf = t & 1, st = t % kDqRingB;
        if (!(ok = bwd_wait(bar(kDqBarPFull + buf), (t >> 1) & 1))) break;
        if (!(ok = bwd_wait(bar(kDqBarFullB + st), (t / kDqRingB) & 1))) break;
        tc_fence_after();
        const uint32_t kt = sb + L::oB + st * L::kKT;
        const uint32_t pp = sb + L::oP + buf * 2 * L::kPT;
#pragma unroll
        for (int s = 0; s < kBwdKt / 16; ++s) {
          const uint32_t acc = (t > 0 || s > 0) ? 1u : 0u;
          mma_bf16(tmem + 256, kmaj_desc(pp + L::kPT, kBwdQ, s), kmaj_desc(kt, D, s), idQ, acc);
          mma_bf16(tmem + 256 + D, kmaj_desc(pp, kBwdQ, s), kmaj_desc(kt, D, s), idQ, acc);
        }
        tc_commit(bar(kDqBarEmptyB + st));
        tc_commit(bar(kDqBarPEmpty + buf));
      }
      tc_commit(bar(kDqBarDone));
      drain_wait(bar(kDqBarDone), 0);
    }
  } else {
    regs_inc<kDqRegsCompute>();
    const int stream = (warp - 4) >> 2, quad = warp & 3;
    const int row = quad * 32 + lane, qrow = qt * kBwdQ + row;
    const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
    const BwdScales sc = bwd_scales(p);
    const float lse = p.lse[(int64_t)gq * p.Npad + qrow];
    bool ok = __all_sync(0xFFFFFFFFu, bwd_wait(bar(kDqBarQ), 0));
    // c_i = dO_i . O_i: dO_i from the row's 128-byte-swizzled chunks, O_i from
    // the forward's output (0 on padded rows)
    float cv = 0.0f;
    if (ok && qrow < p.N &&
        FP4_CHECK(in_range(((int64_t)gq * p.N + qrow) * D, D, (int64_t)gridDim.z * p.H * p.N * D),
                  304)) {
      const __nv_bfloat16* orow = p.out + ((int64_t)gq * p.N + qrow) * D;
#pragma unroll
      for (int a = 0; a < NA; ++a) {
        const uint8_t* src = sm + L::oDO + a * kBwdQ * 128 + row * 128;
#pragma unroll
        for (int k2 = 0; k2 < 8; ++k2) {
          float x[8], o[8];
          bf16x8_to_f32(*reinterpret_cast<const uint4*>(src + ((k2 ^ (row & 7)) * 16)), x);
          bf16x8_to_f32(ld_nc_v4(orow + a * 64 + k2 * 8), o);
#pragma unroll
          for (int e = 0; e < 8; ++e) cv = fmaf(x[e], o[e], cv);
        }
      }
    }
    // this stream's sums: D' = sum P (dP - c), the same of the bf16-rounded
    // terms that enter A, and sum P
    float Dp = 0.0f, Dr = 0.0f, Sp = 0.0f;
    const int qrow0 = qt * kBwdQ;  // the CTA's first row: tiles below it need no causal mask
    for (int t = stream; t < nkt && ok; t += 2) {
      const int buf = stream;
      float s[64], dp[64];
      ok = __all_sync(0xFFFFFFFFu, bwd_wait(bar(kDqBarSFull + buf), (t >> 1) & 1));
      if (ok) {
        tc_fence_after();
        tmem_ld32(tl + buf * 128, s);
        tmem_ld32(tl + buf * 128 + 32, s + 32);
        tmem_ld32(tl + buf * 128 + 64, dp);
        tmem_ld32(tl + buf * 128 + 96, dp + 32);
        tmem_wait_ld();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kDqBarSEmpty + buf));
      if (!ok) break;
      const int key0 = t * kBwdKt;
      if (key0 + kBwdKt <= p.N && (!CAUSAL || key0 + kBwdKt - 1 <= qrow0)) {
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = ex2_approx(fmaf(s[c], sc.c, -lse));  // P
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const int key = key0 + c;
          const bool live = key < p.N && (!CAUSAL || key <= qrow);
          s[c] = live ? ex2_approx(fmaf(s[c], sc.c, -lse)) : 0.0f;
        }
      }
      // x = P (dP - c) and its bf16 rounding r, the operand of A; pairwise
      // sums (f32x2) of x, r and P, two chains each
      uint32_t wp[32], wd[32];
      uint64_t dx[2] = {0, 0}, dr[2] = {0, 0}, dsp[2] = {0, 0};
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float x0 = s[2 * c] * fmaf(dp[2 * c], sc.dv, -cv);
        const float x1 = s[2 * c + 1] * fmaf(dp[2 * c + 1], sc.dv, -cv);
        wp[c] = pack_bf16(s[2 * c], s[2 * c + 1]);
        wd[c] = pack_bf16(x0, x1);
        dx[c & 1] = add2(dx[c & 1], pk(x0, x1));
        dr[c & 1] = add2(dr[c & 1], pk(__uint_as_float(wd[c] << 16),
                                       __uint_as_float(wd[c] & 0xFFFF0000u)));
        dsp[c & 1] = add2(dsp[c & 1], pk(s[2 * c], s[2 * c + 1]));
      }
      {
        float a0, a1, b0, b1;
        upk(add2(dx[0], dx[1]), a0, a1);
        Dp += a0 + a1;
        upk(add2(dr[0], dr[1]), a0, a1);
        Dr += a0 + a1;
        upk(add2(dsp[0], dsp[1]), b0, b1);
        Sp += b0 + b1;
      }
      if (t >= 2)
        ok = __all_sync(0xFFFFFFFFu, bwd_wait(bar(kDqBarPEmpty + buf), ((t >> 1) - 1) & 1));
      if (!ok) break;
      uint8_t* pr = sm + L::oP + buf * 2 * L::kPT + row * 128;
#pragma unroll
      for (int k2 = 0; k2 < 8; ++k2) {
        const int off = (k2 ^ (row & 7)) * 16;
        *reinterpret_cast<uint4*>(pr + off) =
            make_uint4(wp[4 * k2], wp[4 * k2 + 1], wp[4 * k2 + 2], wp[4 * k2 + 3]);
        *reinterpret_cast<uint4*>(pr + L::kPT + off) =
            make_uint4(wd[4 * k2], wd[4 * k2 + 1], wd[4 * k2 + 2], wd[4 * k2 + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kDqBarPFull + buf));
    }
    // every A / B contraction has read its P tiles: the P area holds the two
    // streams' partial sums of the row
    ok = ok && __all_sync(0xFFFFFFFFu, bwd_wait(bar(kDqBarDone), 0));
    float* part = reinterpret_cast<float*>(sm + L::oP);  // [stream][3][kBwdQ]
    if (ok) {
      part[(stream * 3 + 0) * kBwdQ + row] = Dp;
      part[(stream * 3 + 1) * kBwdQ + row] = Dr;
      part[(stream * 3 + 2) * kBwdQ + row] = Sp;
    }
    named_bar_sync(1, 256);  // both warpgroups, on every path
    ok = __all_sync(0xFFFFFFFFu, ok && *reinterpret_cast<volatile unsigned*>(&g_fp4_err) == 0u);
    if (ok) {  // warp-uniform: tcgen05.ld is a whole-warp instruction; only the stores are per row
      const float Dq = part[row] + part[3 * kBwdQ + row];                  // D'_i
      const float Dqr = part[kBwdQ + row] + part[4 * kBwdQ + row];         // its rounded terms
      const float Sq = part[2 * kBwdQ + row] + part[5 * kBwdQ + row];      // sum_j P_ij
      // D_i - c_i for dQ, from the rounded terms that A holds: a row whose P
      // sits on one key then gets dQ = 0 exactly, as dS = 0 there
      const float E = fmaf(cv, Sq - 1.0f, Dqr);
      if (stream == 0 &&
          FP4_CHECK(in_range((int64_t)gq * p.Npad + qrow, 1, (int64_t)gridDim.z * p.H * p.Npad), 305))
        p.Dvec[(int64_t)gq * p.Npad + qrow] = fmaf(cv, Sq, Dq);  // 0 on padded rows
      tc_fence_after();
      constexpr int DH = D / 2;  // each stream writes half the channels
      __nv_bfloat16* dst = p.dq + ((int64_t)gq * p.N + qrow) * D + stream * DH;
#pragma unroll
      for (int cc = 0; cc < DH; cc += 32) {
        float oa[32], ob[32];
        __syncwarp();
        tmem_ld32(tl + 256 + stream * DH + cc, oa);
        tmem_ld32(tl + 256 + D + stream * DH + cc, ob);
        tmem_wait_ld();
        if (qrow < p.N &&
            FP4_CHECK(in_range(((int64_t)gq * p.N + qrow) * D + stream * DH + cc, 32,
                               (int64_t)gridDim.z * p.H * p.N * D), 306)) {
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = pack_bf16(fmaf(-E, ob[2 * i], oa[2 * i]) * sc.sdq,
                             fmaf(-E, ob[2 * i + 1], oa[2 * i + 1]) * sc.sdq);
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
    tmem_dealloc(tmem, 512);
  }
}

// ----------------------------------------------------------- dk/dv kernel ----
// S^T = K^ Q^T straight from the forward's NVFP4 codes and block scales
// (tcgen05 kind::mxf4nvf4, M = 128 keys, N = 64 queries, K = 64 per
// instruction), the other contractions in bf16. The block scales of a
// 64-query B operand: the forward stores one scale atom per 128 rows (row r
// of chunk k at byte (r % 32) 16 + (r / 32) 4 + k, copied to TMEM with
// tcgen05.cp 32x128b.warpx4, where row r's four scales sit in column r / 32);
// an N = 64 operand reads columns 0 and 1, so sf64_kernel stores for every
// 64-query tile an atom whose first two columns hold its rows.
template <int D>
struct BwdDkvSmem {
  static constexpr int kK = kBwdK * D * 2;      // V^ tile (128 keys), bf16
  static constexpr int kKc = kBwdK * D / 2;     // K codes (128 keys)
  static constexpr int kSf = (D / 64) * 512;    // scale atoms of one tile, one per 64-element chunk
  static constexpr int kQ = kBwdQt * D * 2;     // dO tile (64 queries), bf16
  static constexpr int kQc = kBwdQt * D / 2;    // Q codes (64 queries)
  static constexpr int kQT = D * kBwdQt * 2;    // Q^T or dO^T tile
  static constexpr int kSlotA = (kQ + kQc + kSf + 1023) / 1024 * 1024;  // dO, Q codes, Q scales
  static constexpr int oV = 0;
  static constexpr int oKc = oV + kK;
  static constexpr int oKsf = oKc + kKc;
  static constexpr int oA = oKsf + (kSf + 1023) / 1024 * 1024;  // ring A [2] (S^T, dP^T)
  static constexpr int oB = oA + 2 * kSlotA;          // ring B [2]: Q^T then dO^T (dK, dV)
  static constexpr int oLse = oB + 2 * 2 * kQT;       // ring B [2]: lse[64], D[64]
  static constexpr int oBar = oLse + 2 * 512;
  static constexpr int oTmem = oBar + 256;
  static constexpr int kBytes = oTmem + 16 + 1024;
  static_assert(kBytes <= 232448, "shared memory of one CTA");
};

// Ring A (dO, Q codes and scales) is released when S^T and dP^T complete;
// ring B (Q^T, dO^T, lse, D) when dV and dK complete; each has its own
// producer warp. One S^T/dP^T buffer: the compute warps copy it to registers
// at once, so the next tile's S^T and dP^T run while they work on this one.
// P^T and dS^T go back to TMEM (tcgen05.st) as the A operands of dV and dK:
// no shared-memory store and no proxy fence on the compute warps' path.
enum : int {
  kKvBarKV = 0,
  kKvBarFullA = 1,    // [2]
  kKvBarEmptyA = 3,   // [2]
  kKvBarFullB = 5,    // [2]
  kKvBarEmptyB = 7,   // [2]
  kKvBarSFull = 9,
  kKvBarSEmpty = 10,
  kKvBarPFull = 11,
  kKvBarPEmpty = 12,
  kKvBarDone = 13,
};

// TMEM columns of the dk/dv kernel.
template <int D>
struct DkvCols {
  static constexpr uint32_t kS = 0, kDP = 64, kDV = 128, kDK = 128 + D, kKsf = 128 + 2 * D,
                            kQsf = kKsf + 8,                 // [2] x 8
                            kPT = (kQsf + 16 + 31) / 32 * 32,  // P^T: 64 bf16 per key = 32 columns
                            kDST = kPT + 32;                   // dS^T
  static_assert(kDST + 32 <= 512, "TMEM columns");
};

// One CTA per (128-key tile, key/value head, batch); tiles of 64 queries of
// every query head of the group.
template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmKc, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmQc, const __grid_constant__ CUtensorMap tmDO,
                    const __grid_constant__ CUtensorMap tmQT,
                    const __grid_constant__ CUtensorMap tmDOT, const BwdParams p) {
  using L = BwdDkvSmem<D>;
  using TC = DkvCols<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int gk = b * p.Hkv + hk;
  const int G = p.H / p.Hkv;
  const int nq_all = (p.N + kBwdQt - 1) / kBwdQt;
  const int i0 = CAUSAL ? (kt * kBwdK) / kBwdQt : 0;  // first query tile that sees these keys
  const int nqt = max(0, nq_all - i0);
  const int T = G * nqt;
  auto bar = [&](int i) -> uint32_t { return sb + L::oBar + 8 * i; };
  if (threadIdx.x == 0) {
    mbar_init(bar(kKvBarKV), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kKvBarFullA + s), 1);
      mbar_init(bar(kKvBarEmptyA + s), 1);
      mbar_init(bar(kKvBarFullB + s), 1);
      mbar_init(bar(kKvBarEmptyB + s), 1);
    }
    mbar_init(bar(kKvBarSFull), 1);
    mbar_init(bar(kKvBarSEmpty), 8);
    mbar_init(bar(kKvBarPFull), 8);
    mbar_init(bar(kKvBarPEmpty), 1);
    mbar_init(bar(kKvBarDone), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sb + L::oTmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + L::oTmem);
  constexpr int NA = D / 64;
  const int64_t ntq128 = p.Npad / 128;

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      int issued = 0;
      const int64_t Gq = (int64_t)gridDim.z * p.H, Gk = (int64_t)gridDim.z * p.Hkv;
      mbar_arrive_expect_tx(bar(kKvBarKV), L::kK + L::kKc + L::kSf);
      if (FP4_CHECK(tma_ok(0, D / 2, D / 2, 1, gk * p.Npad + kt * kBwdK, kBwdK, Gk * p.Npad), 311)) {
        for (int a = 0; a < NA; ++a)
          tma_load_2d(sb + L::oV + a * kBwdK * 128, &tmV, a * 64, gk * p.Npad + kt * kBwdK,
                      bar(kKvBarKV));
        tma_load_2d(sb + L::oKc, &tmKc, 0, gk * p.Npad + kt * kBwdK, bar(kKvBarKV));
      }
      if (FP4_CHECK(in_range(((int64_t)gk * ntq128 + kt) * L::kSf, L::kSf, Gk * ntq128 * L::kSf),
                    312))
        bulk_load(sb + L::oKsf, p.k_sf + ((int64_t)gk * ntq128 + kt) * L::kSf, L::kSf,
                  bar(kKvBarKV));
      for (int t = 0; t < T && ok; ++t) {  // ring A: dO, Q codes and scales
        const int st = t & 1;
        const int gq = b * p.H + hk * G + t / nqt, i = i0 + t % nqt;
        if (t >= 2 && !(ok = bwd_wait(bar(kKvBarEmptyA + st), ((t >> 1) - 1) & 1))) break;
        const uint32_t base = sb + L::oA + st * L::kSlotA;
        mbar_arrive_expect_tx(bar(kKvBarFullA + st), L::kQ + L::kQc + L::kSf);
        if (FP4_CHECK(tma_ok(0, D / 2, D / 2, 1, gq * p.Npad + i * kBwdQt, kBwdQt, Gq * p.Npad),
                      313)) {
          for (int a = 0; a < NA; ++a)
            tma_load_2d(base + a * kBwdQt * 128, &tmDO, a * 64, gq * p.Npad + i * kBwdQt,
                        bar(kKvBarFullA + st));
          tma_load_2d(base + L::kQ, &tmQc, 0, gq * p.Npad + i * kBwdQt, bar(kKvBarFullA + st));
        }
        const int64_t qsf = ((int64_t)gq * (2 * ntq128) + i) * L::kSf;
        if (FP4_CHECK(in_range(qsf, L::kSf, Gq * 2 * ntq128 * L::kSf), 314))
          bulk_load(base + L::kQ + L::kQc, p.q_sf64 + qsf, L::kSf, bar(kKvBarFullA + st));
        issued = t + 1;
      }
      drain_wait(bar(kKvBarKV), 0);
      for (int t = max(0, issued - 2); t < issued; ++t)
        drain_wait(bar(kKvBarFullA + (t & 1)), (t >> 1) & 1);
    }
  } else if (warp == 2) {
    if (lane == 0) {
      bool ok = true;
      int issued = 0;
      for (int t = 0; t < T && ok; ++t) {  // ring B: Q^T, dO^T, lse, D
        const int st = t & 1;
        const int gq = b * p.H + hk * G + t / nqt, i = i0 + t % nqt;
        if (t >= 2 && !(ok = bwd_wait(bar(kKvBarEmptyB + st), ((t >> 1) - 1) & 1))) break;
        const uint32_t base = sb + L::oB + st * 2 * L::kQT;
        const int64_t Gq = (int64_t)gridDim.z * p.H;
        mbar_arrive_expect_tx(bar(kKvBarFullB + st), 2 * L::kQT + 512);
        if (FP4_CHECK(tma_ok(i * kBwdQt, kBwdQt, p.Npad, 2, (int64_t)gq * D, D, Gq * D), 315)) {
          tma_load_2d(base, &tmQT, i * kBwdQt, gq * D, bar(kKvBarFullB + st));
          tma_load_2d(base + L::kQT, &tmDOT, i * kBwdQt, gq * D, bar(kKvBarFullB + st));
        }
        if (FP4_CHECK(in_range((int64_t)gq * p.Npad + i * kBwdQt, 64, Gq * p.Npad), 316)) {
          bulk_load(sb + L::oLse + st * 512, p.lse + (int64_t)gq * p.Npad + i * kBwdQt, 256,
                    bar(kKvBarFullB + st));
          bulk_load(sb + L::oLse + st * 512 + 256, p.Dvec + (int64_t)gq * p.Npad + i * kBwdQt, 256,
                    bar(kKvBarFullB + st));
        }
        issued = t + 1;
      }
      for (int t = max(0, issued - 2); t < issued; ++t)
        drain_wait(bar(kKvBarFullB + (t & 1)), (t >> 1) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kSw = (D == 128) ? 4u : 6u;     // codes: 64- or 32-byte swizzle
      constexpr uint32_t kSbo = (D == 128) ? 512u : 256u;
      const uint32_t idS = idesc_mxf4nvf4(kBwdK, kBwdQt), idP = idesc_bf16(kBwdK, kBwdQt);
      const uint32_t idO = idesc_bf16(kBwdK, D);
      bool ok = bwd_wait(bar(kKvBarKV), 0);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int kc = 0; kc < NA; ++kc)
          tc_cp_32x128b_x4(tmem + TC::kKsf + 4 * kc, smem_desc(sb + L::oKsf + 512 * kc, 0, 128, 0));
      }
      auto issue_kv = [&](int t) {  // dV += P^T dO, dK += dS^T Q^ of tile t
        const int st = t & 1;
        ok = ok && bwd_wait(bar(kKvBarPFull), t & 1);
        ok = ok && bwd_wait(bar(kKvBarFullB + st), (t >> 1) & 1);
        if (!ok) return;
        tc_fence_after();
        const uint32_t base = sb + L::oB + st * 2 * L::kQT;
#pragma unroll
        for (int s = 0; s < kBwdQt / 16; ++s) {  // A (P^T, dS^T) from TMEM, 8 columns per K step
          const uint32_t acc = (t > 0 || s > 0) ? 1u : 0u;
          mma_bf16_ta(tmem + TC::kDV, tmem + TC::kPT + 8 * s, kmaj_desc(base + L::kQT, D, s), idO,
                      acc);
          mma_bf16_ta(tmem + TC::kDK, tmem + TC::kDST + 8 * s, kmaj_desc(base, D, s), idO, acc);
        }
        tc_commit(bar(kKvBarEmptyB + st));
        tc_commit(bar(kKvBarPEmpty));
      };
      for (int t = 0; t < T && ok; ++t) {
        const int st = t & 1;
        if (!(ok = bwd_wait(bar(kKvBarFullA + st), (t >> 1) & 1))) break;
        if (t >= 1 && !(ok = bwd_wait(bar(kKvBarSEmpty), (t - 1) & 1))) break;
        tc_fence_after();
        const uint32_t base = sb + L::oA + st * L::kSlotA;
        const uint32_t tQsf = tmem + TC::kQsf + 8 * st;
#pragma unroll
        for (int kc = 0; kc < NA; ++kc)
          tc_cp_32x128b_x4(tQsf + 4 * kc, smem_desc(base + L::kQ + L::kQc + 512 * kc, 0, 128, 0));
#pragma unroll
        for (int kc = 0; kc < NA; ++kc)
          mma_mxf4nvf4(tmem + TC::kS, smem_desc(sb + L::oKc + 32 * kc, 16, kSbo, kSw),
                       smem_desc(base + L::kQ + 32 * kc, 16, kSbo, kSw), idS,
                       tmem + TC::kKsf + 4 * kc, tQsf + 4 * kc, kc > 0 ? 1u : 0u);
#pragma unroll
        for (int s = 0; s < D / 16; ++s)
          mma_bf16(tmem + TC::kDP, kmaj_desc(sb + L::oV, kBwdK, s), kmaj_desc(base, kBwdQt, s), idP,
                   s > 0 ? 1u : 0u);
        tc_commit(bar(kKvBarSFull));
        tc_commit(bar(kKvBarEmptyA + st));
        if (t > 0) issue_kv(t - 1);
      }
      if (ok && T > 0) issue_kv(T - 1);
      tc_commit(bar(kKvBarDone));
      drain_wait(bar(kKvBarDone), 0);
    }
  } else if (warp >= 4) {
    // this warp: the rows of its lane quarter, queries half * 32 .. + 31 of each tile
    const int quad = warp & 3, half = (warp - 4) >> 2;
    const int row = quad * 32 + lane, key = kt * kBwdK + row;
    const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
    const BwdScales sc = bwd_scales(p);
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      const int st = t & 1, i = i0 + t % nqt;
      float s[32], dp[32];
      ok = ok && __all_sync(0xFFFFFFFFu, bwd_wait(bar(kKvBarSFull), t & 1));
      if (ok) {
        tc_fence_after();
        tmem_ld32(tl + TC::kS + half * 32, s);
        tmem_ld32(tl + TC::kDP + half * 32, dp);
        tmem_wait_ld();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kKvBarSEmpty));
      if (!ok) break;
      // the stage's lse and D: its full barrier has completed (S^T was issued
      // after it); the wait makes the bulk copies' data visible to this thread
      ok = __all_sync(0xFFFFFFFFu, bwd_wait(bar(kKvBarFullB + st), (t >> 1) & 1));
      if (!ok) break;
      // this half's lse and D (a predicated select per pair: a separate
      // unmasked path for full tiles measured slower)
      const float* lq = reinterpret_cast<const float*>(sm + L::oLse + st * 512) + half * 32;
      const float* dq = lq + 64;
      const int q0 = i * kBwdQt + half * 32;
      uint32_t wp[16], wd[16];
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        float pv[2], dv2[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int q = q0 + c + u;
          const bool live = key < p.N && q < p.N && (!CAUSAL || key <= q);
          pv[u] = live ? ex2_approx(fmaf(s[c + u], sc.c, -lq[c + u])) : 0.0f;
          dv2[u] = pv[u] * fmaf(dp[c + u], sc.dv, -dq[c + u]);
        }
        wp[c >> 1] = pack_bf16(pv[0], pv[1]);
        wd[c >> 1] = pack_bf16(dv2[0], dv2[1]);
      }
      if (t > 0) ok = __all_sync(0xFFFFFFFFu, bwd_wait(bar(kKvBarPEmpty), (t - 1) & 1));
      if (!ok) break;
      // P^T and dS^T of this warp's 32 queries: TMEM columns half * 16 .. + 15
      tc_fence_after();
      tmem_st16(tl + TC::kPT + half * 16, reinterpret_cast<const float*>(wp));
      tmem_st16(tl + TC::kDST + half * 16, reinterpret_cast<const float*>(wd));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kKvBarPFull));
    }
    ok = ok && __all_sync(0xFFFFFFFFu, bwd_wait(bar(kKvBarDone), 0));
    if (ok) {  // warp-uniform: tcgen05.ld is a whole-warp instruction; only the stores are per row
      tc_fence_after();
      __nv_bfloat16* dvp = p.dv + ((int64_t)gk * p.N + key) * D;
      __nv_bfloat16* dkp = p.dk + ((int64_t)gk * p.N + key) * D;
#pragma unroll
      for (int cc = half * (D / 2); cc < (half + 1) * (D / 2); cc += 32) {  // this warp's channels
        float o[32], o2[32];
        if (T > 0) {
          __syncwarp();
          tmem_ld32(tl + TC::kDV + cc, o);
          tmem_ld32(tl + TC::kDK + cc, o2);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int u = 0; u < 32; ++u) o[u] = o2[u] = 0.0f;
        }
        if (key < p.N &&
            FP4_CHECK(in_range(((int64_t)gk * p.N + key) * D + cc, 32,
                               (int64_t)gridDim.z * p.Hkv * p.N * D), 317)) {
          uint32_t wv[16], wk[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            wv[u] = pack_bf16(o[2 * u], o[2 * u + 1]);
            wk[u] = pack_bf16(o2[2 * u] * sc.sdk, o2[2 * u + 1] * sc.sdk);
          }
          uint4* v4 = reinterpret_cast<uint4*>(dvp + cc);
          uint4* k4 = reinterpret_cast<uint4*>(dkp + cc);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            v4[u] = make_uint4(wv[4 * u], wv[4 * u + 1], wv[4 * u + 2], wv[4 * u + 3]);
            k4[u] = make_uint4(wk[4 * u], wk[4 * u + 1], wk[4 * u + 2], wk[4 * u + 3]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fp4
