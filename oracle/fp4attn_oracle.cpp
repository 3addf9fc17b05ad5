// CPU oracle for the NVFP4 FlashAttention forward.
//
// TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the CPU-baseline
// leg of the benchmark load this file's library. The CUDA path shares no code,
// header, table or constant generator with it.
//
// Plain, slow and written to be checked by eye against the method:
//  * "4-bit attention" runs both QK^T and PV as 4-bit block-scaled
//    contractions while the online-softmax state stays in higher precision
//    [HiFA4 summary, theflow.svmpsp.dev related-papers feed; EFQ-Softmax
//    abstract, scholarbro.com page "AVQ Attention: Adaptive Vector-Quantized
//    Attention"].
//  * The operand format is block-scaled E2M1, named NVFP4 [TetraJet-v2
//    abstract, searcharxiv.com author page "Pengle Zhang"; Minima summary,
//    theflow feed; EFQ-Softmax abstract].
//  * The probability path is exp-then-quantize: shifted-score exponentials in
//    higher precision form a temporary probability block that is quantized
//    before the low-bit PV product; the FlashAttention row-maximum update,
//    historical rescaling, high-precision accumulation and final normalisation
//    are kept [EFQ-Softmax abstract].
//  * Flag 8 replaces that path with EFQ-Softmax: E2M1 codes generated straight
//    from the shifted scores by an exponent-only block scale and one affine
//    rule, the same operand in numerator and denominator [EFQ-Softmax
//    abstract]; the reading is at efq_block.
//  * Flags 32 and 64 smooth K and Q before quantisation (mean subtraction per
//    channel, with the score correction that keeps the softmax exact)
//    [SageAttention2 abstract, searcharxiv.com author page "Pengle Zhang"];
//    the reading is at channel_mean.
//  * The backward (ora_attn_bwd) recomputes the scores from the forward's
//    FP4 operands and takes D from its own P and V~ [Attn-QAT abstract, arxiv
//    listing "Attn-QAT: 4-Bit Attention With Quantization-Aware Training"];
//    the reading is at attn_bwd_group.
// The pages give no formula for any of these steps. Where this file fixes one
// (format constants, scale recipe, rounding, masking, GQA mapping, the
// denominator) it states the reading it takes.
//
// Precision: quantisation runs in IEEE fp32, one correctly rounded operation
// per step and never a fused multiply-add (build with -ffp-contract=off).
// Dot products of dequantised operands are exact in double: every product has
// at most 12 significant bits and a sum over <= 128 terms spans at most 50
// bits of binary exponent, below double's 53.
//
// Parity pins: every function here is pinned by the CPU tests (tests/
// test_oracle_*.py): format tables written from the format definitions, brute
// force nearest-value search, exactly representable round trips, hand-worked
// attention examples (tests/golden/), closed forms (uniform scores, one key),
// and brute-force fp64 attention within an a-posteriori FP4 error bound.
#include <algorithm>
#include <atomic>
#include <cfloat>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

// ---------------------------------------------------------------- bf16 ----
float bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x40);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

// ---------------------------------------------------------------- E2M1 ----
// E2M1: 1 sign bit (bit 3), 2 exponent bits, 1 mantissa bit. Magnitudes of
// codes 0..7 are {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
const float kE2M1Mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

// Round to nearest, ties to the even code (mantissa bit 0); magnitudes above
// 6 saturate to 6 (the "satfinite" behaviour). The sign bit is copied from the
// input, so -0 and small negatives that round to zero give code 8.
uint8_t e2m1_encode(float y) {
  uint8_t s = std::signbit(y) ? 8 : 0;
  float a = std::fabs(y);
  uint8_t c;
  if (a <= 0.25f) c = 0;        // tie 0.25 -> code 0
  else if (a < 0.75f) c = 1;
  else if (a <= 1.25f) c = 2;   // ties 0.75 and 1.25 -> code 2
  else if (a < 1.75f) c = 3;
  else if (a <= 2.5f) c = 4;    // ties 1.75 and 2.5 -> code 4
  else if (a < 3.5f) c = 5;
  else if (a <= 5.0f) c = 6;    // ties 3.5 and 5 -> code 6
  else c = 7;                   // (5, inf] -> 6
  return s | c;
}

float e2m1_decode(uint8_t c) {
  float m = kE2M1Mag[c & 7];
  return (c & 8) ? -m : m;
}

// ---------------------------------------------------------------- E4M3 ----
// E4M3 (OCP FP8 E4M3): bias 7, no infinities, 0x7F/0xFF are NaN, largest
// finite magnitude 0x7E = 448, subnormals m * 2^-9.
float e4m3_decode(uint8_t c) {
  int e = (c >> 3) & 15, m = c & 7;
  float mag;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) mag = std::ldexp((float)m, -9);
  else mag = std::ldexp(1.0f + m / 8.0f, e - 7);
  return (c & 0x80) ? -mag : mag;
}

// Round to nearest, ties to the even code; magnitudes above 448 saturate to
// 448 (satfinite). Nearest-value search over the 127 finite magnitudes.
uint8_t e4m3_encode(float y) {
  if (std::isnan(y)) return 0x7F;
  uint8_t s = std::signbit(y) ? 0x80 : 0;
  float a = std::fabs(y);
  static float mags[127];
  static bool init = false;
  if (!init) {  // benign race: every thread writes the same values
    for (int c = 0; c < 127; ++c) mags[c] = e4m3_decode((uint8_t)c);
    init = true;
  }
  if (a >= 448.0f) return s | 0x7E;
  // first code whose magnitude is >= a
  int hi = (int)(std::lower_bound(mags, mags + 127, a) - mags);
  if (hi == 0) return s;  // a == 0
  int lo = hi - 1;
  double dlo = (double)a - mags[lo], dhi = (double)mags[hi] - a;
  int c;
  if (dlo < dhi) c = lo;
  else if (dhi < dlo) c = hi;
  else c = (lo % 2 == 0) ? lo : hi;
  return s | (uint8_t)c;
}

// ------------------------------------------------------- NVFP4 recipe ----
// Reading (the pages name NVFP4 and "block-scaled E2M1" but give no recipe):
// the standard two-level NVFP4 scaling. One fp32 scale per tensor maps the
// tensor's absolute maximum onto 6 * 448 = 2688, the product of the largest
// E2M1 and E4M3 magnitudes; each block of 16 elements carries an E4M3 scale.
const float kTensorRange = 2688.0f;  // 6 * 448

// s_enc = 2688 / amax; amax == 0 gives s_enc = 1; a non-finite quotient
// saturates to FLT_MAX. The decode scale is d = 1 / s_enc.
void tensor_scale(float amax, float* s_enc, float* d) {
  float s = (amax > 0.0f) ? kTensorRange / amax : 1.0f;
  if (!std::isfinite(s)) s = FLT_MAX;
  *s_enc = s;
  *d = 1.0f / s;
}

// One block (n <= 16 values; absent values of a tail block count as zero):
//   a = max |x_i|
//   e = E4M3(fl(fl(a / 6) * s_enc))
//   r = fl(s_enc / dec(e)), or 0 when dec(e) == 0
//   code_i = E2M1(fl(x_i * r))
// Each operation is one correctly rounded fp32 operation.
void quantize_block(const float* x, int n, float s_enc, uint8_t* codes, uint8_t* scale) {
  float a = 0.0f;
  for (int i = 0; i < n; ++i) a = std::max(a, std::fabs(x[i]));
  float t = a / 6.0f;
  t = t * s_enc;
  uint8_t e = e4m3_encode(t);
  float de = e4m3_decode(e);
  float r = (de == 0.0f) ? 0.0f : s_enc / de;
  for (int i = 0; i < n; ++i) {
    float y = x[i] * r;
    codes[i] = e2m1_encode(y);
  }
  *scale = e;
}

float amax_bf16(const uint16_t* x, int64_t n) {
  float a = 0.0f;
  for (int64_t i = 0; i < n; ++i) a = std::max(a, std::fabs(bf16_to_f32(x[i])));
  return a;
}

template <class F>
void parallel_for(int64_t n, int nthreads, F&& f) {
  if (nthreads <= 0) nthreads = (int)std::max(1u, std::thread::hardware_concurrency());
  if (nthreads == 1 || n < 2) {
    for (int64_t i = 0; i < n; ++i) f(i);
    return;
  }
  std::atomic<int64_t> next(0);
  std::vector<std::thread> ts;
  for (int t = 0; t < nthreads; ++t)
    ts.emplace_back([&] {
      for (int64_t i; (i = next.fetch_add(1)) < n;) f(i);
    });
  for (auto& t : ts) t.join();
}

// Rows of `cols` values, blocks of 16 along the row (Q and K: along D).
// codes [rows][cols/2]: element 2i in the low nibble of byte i.
// scales [rows][cols/16].
// With `mean` (one fp32 per column; the smoothing of flags 32 and 64) the
// quantised values are the smoothed fl32(x - mean[col]).
void quantize_rows(const uint16_t* x, int64_t rows, int cols, float s_enc, uint8_t* codes,
                   uint8_t* scales, int nthreads, const float* mean = nullptr) {
  const int nb = cols / 16;
  parallel_for(rows, nthreads, [&](int64_t r) {
    float blk[16];
    uint8_t c[16];
    for (int b = 0; b < nb; ++b) {
      for (int i = 0; i < 16; ++i) {
        blk[i] = bf16_to_f32(x[r * cols + b * 16 + i]);
        if (mean) blk[i] = blk[i] - mean[b * 16 + i];
      }
      quantize_block(blk, 16, s_enc, c, &scales[r * nb + b]);
      for (int i = 0; i < 8; ++i)
        codes[r * (cols / 2) + b * 8 + i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
    }
  });
}

// V: blocks of 16 consecutive tokens for each channel d, stored transposed.
// x [N][D]; codes [D][npad/2], scales [D][npad/16]; tokens >= N count as 0.
void quantize_tokens_T(const uint16_t* x, int N, int D, float s_enc, uint8_t* codes,
                       uint8_t* scales, int npad) {
  const int nb = npad / 16;
  for (int d = 0; d < D; ++d)
    for (int b = 0; b < nb; ++b) {
      float blk[16];
      uint8_t c[16];
      for (int i = 0; i < 16; ++i) {
        int n = b * 16 + i;
        blk[i] = (n < N) ? bf16_to_f32(x[(int64_t)n * D + d]) : 0.0f;
      }
      quantize_block(blk, 16, s_enc, c, &scales[(int64_t)d * nb + b]);
      for (int i = 0; i < 8; ++i)
        codes[(int64_t)d * (npad / 2) + b * 8 + i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
    }
}

// Dequantised value in the contraction's own units: E2M1 value times the E4M3
// block scale. The tensor scale d is applied after the contraction.
// FP8 variant of V (flag 16) [SageAttention2 abstract, searcharxiv.com author
// page "Pengle Zhang": P~ and V quantised to FP8 for the PV product]. The page
// gives no recipe; the reading: one fp32 scale per tensor mapping its absolute
// maximum onto E4M3's largest value 448, s8 = fl(448 / amax) (1 if amax == 0,
// FLT_MAX on overflow), code = E4M3(fl(v s8)) round to nearest even,
// saturating; v~ = dec(code) / s8.
void fp8_tensor_scale(float amax, float* s8, float* d8) {
  float s = (amax > 0.0f) ? 448.0f / amax : 1.0f;
  if (!std::isfinite(s)) s = FLT_MAX;
  *s8 = s;
  *d8 = 1.0f / s;
}

// x [N][D] -> codes [D][npad] (channel-major, tokens >= N zero).
void quantize_fp8_tokens_T(const uint16_t* x, int N, int D, float s8, uint8_t* codes, int npad) {
  for (int d = 0; d < D; ++d)
    for (int n = 0; n < npad; ++n)
      codes[(int64_t)d * npad + n] =
          n < N ? e4m3_encode(bf16_to_f32(x[(int64_t)n * D + d]) * s8) : (uint8_t)0;
}

inline double deq(uint8_t code, uint8_t scale) {
  return (double)e2m1_decode(code) * (double)e4m3_decode(scale);
}

const float kLog2e = 1.44269504088896340736f;  // fl32(1 / ln 2)

// -------------------------------------------- smoothing (flags 32, 64) ----
// Outlier smoothing [SageAttention2 abstract, searcharxiv.com author page
// "Pengle Zhang": Q is smoothed to make the low-bit QK^T more accurate]. The
// page gives no formula; the reading taken here:
//   per (batch, head) and channel d, the mean over the head's N tokens,
//   x'_nd = fl32(x_nd - mean_d), quantised as usual (tensor scale from
//   max |x'| over the whole smoothed tensor).
//   K (flag 32): S_ij changes by -q_i . mean_K, the same for every key of
//   row i, which the softmax cancels: nothing is added back.
//   Q (flag 64): q_i . k_j = q'_i . k_j + mean_Q . k_j; the second term
//   depends on the key, so it is added back to the scores:
//   delta_j = mean_Q . k'_j (k' the smoothed K under flag 32, else K), the
//   dot product itself (each product exact in double, the D terms summed in
//   double), taken to the contraction's units, beta_j = delta_j s_Q s_K (the
//   encode scales of the quantised Q' and K, their product exact in double);
//   the scores are x_ij = fl32(fl32(S'_ij + beta_j) c), S'_ij + beta_j summed
//   in double and rounded once to fp32.
// The mean is made independent of summation order so that it is one value on
// any machine: every element is truncated toward zero to the fixed-point
// grid 2^-s with s = 44 - E, 2^(E-1) <= amax < 2^E (amax of the raw tensor),
// the integers are summed exactly (|x| 2^s < 2^44, so N <= 2^19 tokens fit in
// 64 bits), and mean = fl32(fl64(fl64(T) 2^-s) / N); amax == 0 gives 0.
const int kMeanGridBits = 44;

void channel_mean(const uint16_t* x, int N, int D, float amax, float* mean) {
  if (!(amax > 0.0f)) {
    for (int d = 0; d < D; ++d) mean[d] = 0.0f;
    return;
  }
  int E;
  std::frexp(amax, &E);
  const int s = kMeanGridBits - E;
  for (int d = 0; d < D; ++d) {
    int64_t T = 0;
    for (int64_t n = 0; n < N; ++n)
      T += (int64_t)std::trunc(std::ldexp((double)bf16_to_f32(x[n * D + d]), s));
    mean[d] = (float)(std::ldexp((double)T, -s) / (double)N);
  }
}

// max |fl32(x - mean)| over G slabs [N][D] with means [G][D].
float smoothed_amax(const uint16_t* x, int64_t G, int N, int D, const float* mean) {
  float a = 0.0f;
  for (int64_t g = 0; g < G; ++g)
    for (int64_t n = 0; n < N; ++n)
      for (int d = 0; d < D; ++d)
        a = std::max(a, std::fabs(bf16_to_f32(x[(g * N + n) * D + d]) - mean[g * D + d]));
  return a;
}

// delta_j for the N keys of one head: qmean [D]; k [N][D] bf16; kmean [D]
// (NULL: K not smoothed). absum_j = sum_d |qmean_d k'_jd| (may be NULL).
void score_bias(const float* qmean, const uint16_t* k, const float* kmean, int N, int D,
                double* delta, double* absum) {
  for (int64_t j = 0; j < N; ++j) {
    double acc = 0.0, mag = 0.0;
    for (int d = 0; d < D; ++d) {
      float kv = bf16_to_f32(k[j * D + d]);
      if (kmean) kv = kv - kmean[d];
      const double prod = (double)qmean[d] * (double)kv;  // exact: 24 x 24 bits
      acc += prod;
      mag += std::fabs(prod);
    }
    delta[j] = acc;
    if (absum) absum[j] = mag;
  }
}

struct Tensors {
  const uint16_t *q, *k, *v;
  int B, H, Hkv, N, D;
  float sq, dq, sk, dk, sv, dv;
  bool fp8v;                   // V in FP8 (flag 16): sv, dv are s8, d8
  const float* qmean = nullptr;  // flag 64: [B*H][D]
  const float* kmean = nullptr;  // flag 32: [B*Hkv][D]
  const double* bias = nullptr;  // flag 64: [B*H][N], beta_j (contraction units)
  // flag 64: [B*H][N], how far another correct evaluation of beta_j may lie
  // from it (contraction units; see ora_attn_fwd)
  const double* bias_unc = nullptr;
};

// K and V of one (b, kv-head), dequantised to contraction units, [N][D].
struct KVGroup {
  std::vector<double> K, V;
};

KVGroup make_group(const Tensors& T, int b, int hk) {
  const int N = T.N, D = T.D;
  const int64_t off = ((int64_t)b * T.Hkv + hk) * N * D;
  KVGroup g;
  g.K.resize((size_t)N * D);
  g.V.resize((size_t)N * D);
  std::vector<uint8_t> kc((size_t)N * D / 2), ks((size_t)N * D / 16);
  quantize_rows(T.k + off, N, D, T.sk, kc.data(), ks.data(), 1,
                T.kmean ? T.kmean + ((int64_t)b * T.Hkv + hk) * D : nullptr);
  for (int64_t n = 0; n < N; ++n)
    for (int d = 0; d < D; ++d) {
      uint8_t byte = kc[n * (D / 2) + d / 2];
      uint8_t c = (d & 1) ? (byte >> 4) : (byte & 15);
      g.K[n * D + d] = deq(c, ks[n * (D / 16) + d / 16]);
    }
  if (T.fp8v) {  // FP8 V: contraction units dec(code), d8 applied at the end
    std::vector<uint8_t> v8((size_t)D * N);
    quantize_fp8_tokens_T(T.v + off, N, D, T.sv, v8.data(), N);
    for (int d = 0; d < D; ++d)
      for (int64_t n = 0; n < N; ++n) g.V[n * D + d] = (double)e4m3_decode(v8[d * N + n]);
    return g;
  }
  const int npad = (N + 15) / 16 * 16;
  std::vector<uint8_t> vc((size_t)D * npad / 2), vs((size_t)D * npad / 16);
  quantize_tokens_T(T.v + off, N, D, T.sv, vc.data(), vs.data(), npad);
  for (int d = 0; d < D; ++d)
    for (int64_t n = 0; n < N; ++n) {
      uint8_t byte = vc[d * (npad / 2) + n / 2];
      uint8_t c = (n & 1) ? (byte >> 4) : (byte & 15);
      g.V[n * D + d] = deq(c, vs[d * (npad / 16) + n / 16]);
    }
  return g;
}

enum { FLAG_QP_DENOMINATOR = 1, FLAG_FLIP_BOUND = 2, FLAG_PERTURB_P = 4, FLAG_EFQ = 8,
       FLAG_SMOOTH_K = 32, FLAG_SMOOTH_Q = 64,
       FLAG_FP8PV = 16 };

// FP8 P (flag 16): p~ = E4M3(fl(p * 256)) / 256, round to nearest even; p <= 1
// so p * 256 <= 256 stays inside E4M3's range (largest 448) and the scaling is
// exact; d_P = 2^-8. The reading matches V's: one tensor scale, here a power
// of two.
const float kFp8PScale = 256.0f;

// EFQ-Softmax P generation for one block of n <= 16 keys of one row
// [EFQ-Softmax abstract, scholarbro.com page "AVQ Attention: Adaptive
// Vector-Quantized Attention": for each microscaling block, an exponent-only
// scale chosen from the local maximum, the shifted scores mapped to a
// normalised residual domain, nonnegative E2M1 codes from a single affine rule;
// the same operand feeds the numerator and the denominator]. The abstract gives
// no formula; the reading taken here:
//   z_u = x_u - m          shifted scores (log2 units, <= 0; -inf when masked)
//   E = floor(max_u z_u) - 2   exponent-only scale 2^E: the microscaling shared
//                          exponent, 2 being E2M1's largest exponent
//   r_u = z_u - E          residual; the block maximum has r in [2, 3)
//   c_u = min(7, max(0, rne(2 r_u + 2)))   the affine rule: two E2M1 codes per
//                          binade, code 2 = 1.0, code 4 = 2.0, code 6 = 4.0;
//                          rne = round half to even
//   p~_u = val(c_u) 2^E
// Stored as NVFP4 with P's tensor scale 2^-10 (kEfqScaleExp): the block's scale
// byte is the E4M3 value 2^(E + 10), exact for E + 10 in [-9, 8]; E <= -2 since
// z <= 0, and a block with E + 10 < -9 has no such byte and is zero.
// z is exact in double (fp32 x minus fp32 m). Returns E (INT32_MIN when every
// key is masked).
const int kEfqScaleExp = 10;

int efq_block(const double* z, int n, uint8_t* codes, uint8_t* scale) {
  double b = -INFINITY;
  for (int u = 0; u < n; ++u) b = std::max(b, z[u]);
  for (int u = 0; u < n; ++u) codes[u] = 0;
  *scale = 0;
  if (b == -INFINITY) return INT32_MIN;
  const int E = (int)std::floor(b) - 2;
  if (E + kEfqScaleExp < -9) return E;
  *scale = e4m3_encode(std::ldexp(1.0f, E + kEfqScaleExp));
  for (int u = 0; u < n; ++u) {
    if (z[u] == -INFINITY) continue;
    double t = std::nearbyint(2.0 * (z[u] - E) + 2.0);  // default rounding: ties to even
    codes[u] = (uint8_t)std::min(7.0, std::max(0.0, t));
  }
  return E;
}

// The codes of a block for a given E (to evaluate the other rounding of floor).
void efq_block_with_exp(const double* z, int n, int E, uint8_t* codes, uint8_t* scale) {
  for (int u = 0; u < n; ++u) codes[u] = 0;
  *scale = 0;
  if (E + kEfqScaleExp < -9 || E + kEfqScaleExp > 8) return;
  *scale = e4m3_encode(std::ldexp(1.0f, E + kEfqScaleExp));
  for (int u = 0; u < n; ++u) {
    if (z[u] == -INFINITY) continue;
    double t = std::nearbyint(2.0 * (z[u] - E) + 2.0);
    codes[u] = (uint8_t)std::min(7.0, std::max(0.0, t));
  }
}

// E2M1 rounding boundaries of |y| between codes c and c+1 (c = 0..6).
const float kE2M1Mid[7] = {0.25f, 0.75f, 1.25f, 1.75f, 2.5f, 3.5f, 5.0f};

// Codes of a block with a given scale byte e (the second half of the block
// recipe), used to evaluate the other rounding of a block scale.
void quantize_block_with_scale(const float* x, int n, float s_enc, uint8_t e, uint8_t* codes) {
  float de = e4m3_decode(e);
  float r = (de == 0.0f) ? 0.0f : s_enc / de;
  for (int i = 0; i < n; ++i) codes[i] = e2m1_encode(x[i] * r);
}

uint64_t mix64(uint64_t z) {
  z += 0x9E3779B97F4A7C15ULL;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

// EFQ P of one key tile: pq[jj] = val(c) dec(e) per key (units of d_P = 2^-10).
// Flip bound: t = 2 (x - m - E) + 2 decides the codes, floor(max z) decides E.
// Another correct fp32 evaluation (S accumulated in another order, t formed as
// fma(s, 2c, 2 - 2 (m + E)) with one rounding per operation) moves t by at most
//   2 c u (A_j + A_max) + 2 u |x| + 8 u |m| + 4 u |E| + 10 u,  u = 2^-22
// (A_j = sum_d |q~_d k~_d| of the key, A_max that of the row maximum); eps_t is
// four times this. A code whose t lies within eps_t of a rounding point k + 1/2
// (k = 0..6) may take the neighbouring code; a block whose max z lies within
// eps_t of an integer may take the other E, except max z = 0 exactly: that block
// holds the running maximum, and max z = fl(x_max) - m is then exactly 0 in
// every evaluation that forms it that way. FLAG_PERTURB_P moves each z < 0 by
// up to eps_t / 8 (seeded by the row) to test the bound.
void efq_tile(const std::vector<float>& x, const std::vector<double>& A, double amx, float c,
              double m_new, int Bc, int j0, int j1, int flags, uint64_t rowkey,
              std::vector<double>& pq, std::vector<double>& dlt, double& epsmax) {
  const double u = std::ldexp(1.0, -22);
  std::vector<double> z(Bc), eb(Bc, 0.0);
  for (int jj = 0; jj < Bc; ++jj) {
    const bool live = j0 + jj < j1 && x[jj] != -INFINITY;
    z[jj] = live ? (double)x[jj] - m_new : -INFINITY;
    dlt[jj] = 0.0;
    if (live) {
      eb[jj] = 4.0 * (2.0 * (double)c * u * (A[jj] + amx) + 2.0 * u * std::fabs((double)x[jj]) +
                      8.0 * u * std::fabs(m_new) + 10.0 * u);
      if ((flags & FLAG_PERTURB_P) && z[jj] < 0.0) {
        double uu = (double)(mix64(rowkey ^ mix64((uint64_t)(j0 + jj))) >> 11) *
                    std::ldexp(1.0, -53);
        z[jj] = std::min(0.0, z[jj] + (2.0 * uu - 1.0) * eb[jj] / 8.0);
      }
    }
  }
  for (int b0 = 0; b0 < Bc; b0 += 16) {
    const int n = std::min(16, Bc - b0);
    uint8_t codes[16], e;
    const int E = efq_block(&z[b0], n, codes, &e);
    for (int k = 0; k < n; ++k) pq[b0 + k] = deq(codes[k], e);
    if (E == INT32_MIN) continue;
    const double de = (double)e4m3_decode(e);
    double ebk = 0.0, b = -INFINITY;
    for (int k = 0; k < n; ++k) {
      if (z[b0 + k] == -INFINITY) continue;
      const double et = eb[b0 + k] + 16.0 * u * std::fabs((double)E);
      epsmax = std::max(epsmax, et);
      ebk = std::max(ebk, et);
      b = std::max(b, z[b0 + k]);
      if (!(flags & FLAG_FLIP_BOUND)) continue;
      const double t = 2.0 * (z[b0 + k] - E) + 2.0;
      for (int k2 = 0; k2 < 7; ++k2)
        if (std::fabs(t - (k2 + 0.5)) <= et)
          dlt[b0 + k] = std::max(dlt[b0 + k], (double)(kE2M1Mag[k2 + 1] - kE2M1Mag[k2]) * de);
    }
    if (!(flags & FLAG_FLIP_BOUND)) continue;
    // the other rounding of floor(max z)
    const double fb = std::floor(b);
    int other = INT32_MIN;
    if (b == 0.0) other = INT32_MIN;  // the running maximum's block: exact
    else if (b - fb <= ebk) other = E - 1;
    else if (fb + 1.0 - b <= ebk) other = E + 1;
    if (other != INT32_MIN) {
      uint8_t alt[16], ealt;
      efq_block_with_exp(&z[b0], n, other, alt, &ealt);
      for (int k = 0; k < n; ++k)
        dlt[b0 + k] = std::max(dlt[b0 + k], std::fabs(deq(alt[k], ealt) - pq[b0 + k]));
    }
  }
}

// One query row: the tiled forward over key tiles of Bc keys.
//   S_ij = fl32(exact dot product of dequantised q_i, k_j)
//   x_ij = fl32(S_ij * c), c = fl32(fl32(fl32(d_Q d_K) * softmax_scale) * log2 e)
//          (flag 64: S_ij + beta_j, exact, before the rounding to fp32)
//   masked (causal j > i, top-left aligned) -> -inf
// per tile: m_new = max(m, max_j x_ij); alpha = exp2(m - m_new) (0 while m is -inf)
//   p_ij = fl32(exp2(x_ij - m_new)) (double exp2, rounded once)
//   l = alpha l + sum_j p_ij         (reading: the denominator sums the fp32 p
//                                     before quantisation; flag: sum of p~)
//   p~ = NVFP4(p) per 16 keys with the fixed tensor scale 2688 (p <= 1)
//   O = alpha O + sum_j p~_ij v~_j   (exact tile product, accumulated in double)
// out = bf16(fl32(O * fl32(d_P d_V) / l)), d_P = fl32(1 / 2688).
// With FLAG_EFQ the P block comes from efq_block instead (no exponential of
// the scores), l sums those p~ (the same operand in numerator and
// denominator) and d_P = 2^-10.
//
// Flip bound (diagnostic, FLAG_FLIP_BOUND): a P code or block scale is a
// rounding decision; another correct fp32 evaluation of the same row (a
// different accumulation order of S, another exp2 within a few ulp) may land
// on the other side of a rounding boundary. For every decision whose input lies
// within eps of a boundary, the bound adds |p~ change| * |v~_jd| (propagated
// like O) to flip[d] (output units), plus eps |out_d| for the continuous
// change of the denominator. eps is four times the relative
// uncertainty of p from: S rounding (2^-22 of sum_d |q~_d k~_d|, for the key
// and for the row maximum; with flag 64 the sum includes |beta_j|, and the
// distance of another evaluation of beta_j is added), two fp32 roundings of
// the exponent argument and 2^-21 for the exponential. FLAG_PERTURB_P multiplies each p by
// (1 + u eps/4), u uniform in [-1, 1] (seeded by the row), to test the bound.
void row_forward(const Tensors& T, const KVGroup& g, int b, int h, int i, float c, int Bc,
                 int causal, int flags, double* o_out, double* ml_out, uint16_t* bf_out,
                 double* flip_out) {
  const int N = T.N, D = T.D;
  const bool want_flip = (flags & (FLAG_FLIP_BOUND | FLAG_PERTURB_P)) != 0;
  // quantise the query row
  const uint16_t* qrow = T.q + (((int64_t)b * T.H + h) * N + i) * D;
  std::vector<uint8_t> qc(D / 2), qs(D / 16);
  quantize_rows(qrow, 1, D, T.sq, qc.data(), qs.data(), 1,
                T.qmean ? T.qmean + ((int64_t)b * T.H + h) * D : nullptr);
  const double* brow = T.bias ? T.bias + ((int64_t)b * T.H + h) * N : nullptr;
  const double* burow = T.bias_unc ? T.bias_unc + ((int64_t)b * T.H + h) * N : nullptr;
  std::vector<double> qd(D);
  for (int d = 0; d < D; ++d) {
    uint8_t byte = qc[d / 2];
    qd[d] = deq((d & 1) ? (byte >> 4) : (byte & 15), qs[d / 16]);
  }
  const bool efq = (flags & FLAG_EFQ) != 0;
  const bool fp8 = (flags & FLAG_FP8PV) != 0;
  float sP, dP;
  tensor_scale(1.0f, &sP, &dP);  // P: a-priori amax 1, so s_enc = 2688
  if (efq) dP = std::ldexp(1.0f, -kEfqScaleExp);
  if (fp8) dP = 1.0f / kFp8PScale;
  std::vector<double> O(D, 0.0), F(D, 0.0);
  std::vector<float> x(Bc), p(Bc);
  std::vector<double> pq(Bc), A(Bc, 0.0), eps(Bc, 0.0), dlt(Bc, 0.0), z(Bc);
  double Fl = 0.0;  // flip bound of the p~ denominator (EFQ), in units of pq
  double m = -INFINITY, l = 0.0, epsmax = 0.0;
  const int ntiles = (N + Bc - 1) / Bc;
  const uint64_t rowkey = mix64(((uint64_t)b * 65536 + h) * 4294967296ULL + (uint64_t)i);
  for (int t = 0; t < ntiles; ++t) {
    const int j0 = t * Bc, j1 = std::min(j0 + Bc, N);
    if (causal && j0 > i) break;  // fully masked tiles contribute nothing
    float mt = -INFINITY;
    double amx = 0.0;
    for (int j = j0; j < j1; ++j) {
      float xv = -INFINITY;
      double aj = 0.0;
      if (!(causal && j > i)) {
        double s = 0.0;
        const double* kr = &g.K[(int64_t)j * D];
        for (int d = 0; d < D; ++d) s += qd[d] * kr[d];
        if (want_flip)
          for (int d = 0; d < D; ++d) aj += std::fabs(qd[d] * kr[d]);
        if (brow) {  // the correction joins the accumulated sum, one rounding
          s += brow[j];
          // flip bound: the sum's rounding covers |beta_j| too; another
          // evaluation of beta_j adds its own distance (in units of u)
          aj += std::fabs(brow[j]) + burow[j] * std::ldexp(1.0, 22);
        }
        float sf = (float)s;
        xv = sf * c;
      }
      x[j - j0] = xv;
      A[j - j0] = aj;
      if (xv > mt) {
        mt = xv;
        amx = aj;
      }
    }
    double m_new = std::max(m, (double)mt);
    double alpha = (m == -INFINITY) ? 0.0 : std::exp2(m - m_new);
    if (efq) {
      efq_tile(x, A, amx, c, m_new, Bc, j0, j1, flags, rowkey, pq, dlt, epsmax);
    } else {
      for (int jj = 0; jj < Bc; ++jj) {
        int j = j0 + jj;
        bool live = j < j1 && x[jj] != -INFINITY;
        p[jj] = live ? (float)std::exp2((double)x[jj] - m_new) : 0.0f;
        eps[jj] = 0.0;
        if (live && want_flip) {
          const double u = std::ldexp(1.0, -22);
          eps[jj] = std::log(2.0) * ((double)c * u * (A[jj] + amx) +
                                     u * (std::fabs((double)x[jj]) + std::fabs(m_new) +
                                          (fp8 ? 8.0 : 0.0))) +
                    std::ldexp(1.0, -21);
          if (flags & FLAG_PERTURB_P) {
            double uu = (double)(mix64(rowkey ^ mix64((uint64_t)j)) >> 11) * std::ldexp(1.0, -53);
            p[jj] = (float)((double)p[jj] * (1.0 + (2.0 * uu - 1.0) * eps[jj]));
          }
          eps[jj] *= 4.0;
          epsmax = std::max(epsmax, eps[jj]);
        }
      }
      // P quantisation: FP8 per key (flag 16), else NVFP4 blocks of 16 keys
      if (fp8) {
        for (int jj = 0; jj < Bc; ++jj) {
          const float y = p[jj] * kFp8PScale;
          const uint8_t code = e4m3_encode(y);
          pq[jj] = (double)e4m3_decode(code);
          dlt[jj] = 0.0;
          if (!(flags & FLAG_FLIP_BOUND) || y == 0.0f) continue;
          // a neighbouring code whose rounding midpoint lies within eps of y
          for (int nb = -1; nb <= 1; nb += 2) {
            const int c2 = (int)code + nb;
            if (c2 < 0 || c2 > 126) continue;
            const double v2 = (double)e4m3_decode((uint8_t)c2);
            if (std::fabs((double)y - 0.5 * (pq[jj] + v2)) <= eps[jj] * (double)y + 1e-30)
              dlt[jj] = std::max(dlt[jj], std::fabs(v2 - pq[jj]));
          }
        }
      }
      for (int b0 = 0; !fp8 && b0 < Bc; b0 += 16) {
        int n = std::min(16, Bc - b0);
        uint8_t codes[16], e;
        quantize_block(&p[b0], n, sP, codes, &e);
        for (int u = 0; u < n; ++u) pq[b0 + u] = deq(codes[u], e);
        if (!(flags & FLAG_FLIP_BOUND)) continue;
        const float de = e4m3_decode(e);
        const float r = (de == 0.0f) ? 0.0f : sP / de;
        double epsb = 0.0;
        for (int u = 0; u < n; ++u) {
          dlt[b0 + u] = 0.0;
          epsb = std::max(epsb, eps[b0 + u]);
          float y = std::fabs(p[b0 + u] * r);
          for (int k2 = 0; k2 < 7; ++k2)
            if (std::fabs((double)y - kE2M1Mid[k2]) <= eps[b0 + u] * (double)y + 1e-30)
              dlt[b0 + u] = std::max(dlt[b0 + u],
                                     (double)(kE2M1Mag[k2 + 1] - kE2M1Mag[k2]) * (double)de);
        }
        // the block scale's own rounding
        float a = 0.0f;
        for (int u = 0; u < n; ++u) a = std::max(a, std::fabs(p[b0 + u]));
        float tt = (a / 6.0f) * sP;
        int other = (tt >= de) ? e + 1 : e - 1;
        if (a > 0.0f && other >= 0 && other <= 126) {
          double mid = 0.5 * ((double)de + (double)e4m3_decode((uint8_t)other));
          if (std::fabs((double)tt - mid) <= epsb * (double)tt + 1e-30) {
            uint8_t alt[16];
            quantize_block_with_scale(&p[b0], n, sP, (uint8_t)other, alt);
            for (int u = 0; u < n; ++u)
              dlt[b0 + u] = std::max(dlt[b0 + u],
                                     std::fabs(deq(alt[u], (uint8_t)other) - pq[b0 + u]));
          }
        }
      }
    }  // exp-then-quantize
    double lt = 0.0, flt = 0.0;
    if (efq) {
      for (int jj = 0; jj < Bc; ++jj) lt += pq[jj] * (double)dP;
      if (flags & FLAG_FLIP_BOUND)
        for (int jj = 0; jj < Bc; ++jj) flt += dlt[jj];
    } else if (flags & FLAG_QP_DENOMINATOR)
      for (int jj = 0; jj < Bc; ++jj) lt += pq[jj] * (double)dP;
    else
      for (int jj = 0; jj < Bc; ++jj) lt += (double)p[jj];
    l = alpha * l + lt;
    Fl = alpha * Fl + flt;
    for (int d = 0; d < D; ++d) {
      double acc = 0.0, fl = 0.0;
      for (int j = j0; j < j1; ++j) acc += pq[j - j0] * g.V[(int64_t)j * D + d];
      if (flags & FLAG_FLIP_BOUND)
        for (int j = j0; j < j1; ++j) fl += dlt[j - j0] * std::fabs(g.V[(int64_t)j * D + d]);
      O[d] = alpha * O[d] + acc;
      F[d] = alpha * F[d] + fl;
    }
    m = m_new;
  }
  const float fpv = dP * T.dv;
  for (int d = 0; d < D; ++d) {
    double y = O[d] * (double)fpv / l;
    if (o_out) o_out[d] = y;
    if (bf_out) bf_out[d] = f32_to_bf16_rne((float)y);
    // decisions near a boundary, plus the change of l: continuous (|dl| <= eps l)
    // for the fp32-p denominator; for EFQ's p~ denominator the same flips move
    // l by up to Fl d_P, so y moves by at most (|dO| + |y| |dl|) / (l - |dl|)
    if (flip_out) {
      const double dl = Fl * (double)dP;
      flip_out[d] = !efq ? F[d] * (double)fpv / l + epsmax * std::fabs(y)
                    : (l > dl ? (F[d] * (double)fpv + std::fabs(y) * dl) / (l - dl) : INFINITY);
    }
  }
  if (ml_out) {
    ml_out[0] = m;
    ml_out[1] = l;
    ml_out[2] = epsmax;
  }
}

// ---------------------------------------------------------------- backward ----
// FP4 attention backward [Attn-QAT abstract, arxiv listing "Attn-QAT: 4-Bit
// Attention With Quantization-Aware Training": stable FP4 attention training
// needs (1) the backward to recompute the attention scores in the same low
// precision as the forward and (2) FlashAttention's gradient computation to be
// freed of an implicit precision assumption]. The abstract gives no formula;
// the reading taken here, for one (batch, key/value head) group:
//   q~, k~, v~   the forward's NVFP4 operands, dequantised to real values
//                (val(code) dec(e) d, d the tensor's decode scale)
//   s_ij         q~_i . k~_j, exact; masked (causal j > i) -> -inf   (1)
//   P_ij         exp(scale s_ij - lse_i), lse_i = log sum_j exp(scale s_ij):
//                the forward's probabilities before their quantisation
//   dP_ij        dO_i . v~_j
//   D_i          sum_j P_ij dP_ij                                   (2)
//                FlashAttention forms D from the forward output as dO_i . O_i,
//                which equals sum_j P_ij dP_ij only when O = P V~ exactly in
//                the backward's precision; the FP4 forward's O is P~ V~ / l with
//                quantised P~, so D is taken from this P and v~ instead
//   dS_ij        P_ij (dP_ij - D_i)
//   dq_i         scale sum_j dS_ij k~_j
//   dk_j         scale sum_{i, query heads of the group} dS_ij q~_i
//   dv_j         sum_{i, query heads of the group} P_ij dO_i
// The quantisers pass gradients straight through: dq, dk, dv are the
// gradients with respect to q~, k~, v~ and serve as those of q, k, v.
// Everything in double.
struct BwdGroup {
  int N, D, G;
  std::vector<double> K, V;       // [N][D] real values
  std::vector<double> Q, dO;      // [G][N][D]
};

BwdGroup make_bwd_group(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                        const uint16_t* dout, int B, int H, int Hkv, int N, int D, int b, int hk,
                        const float* s_enc, const float* dec) {
  (void)B;
  BwdGroup g;
  g.N = N;
  g.D = D;
  g.G = H / Hkv;
  const int64_t nd = (int64_t)N * D;
  g.K.resize(nd);
  g.V.resize(nd);
  g.Q.resize(g.G * nd);
  g.dO.resize(g.G * nd);
  std::vector<uint8_t> c((size_t)nd / 2), sc((size_t)nd / 16);
  auto deq_rows = [&](const uint16_t* x, float se, float d, double* outp) {
    quantize_rows(x, N, D, se, c.data(), sc.data(), 1);
    for (int64_t n = 0; n < N; ++n)
      for (int dd = 0; dd < D; ++dd) {
        uint8_t byte = c[n * (D / 2) + dd / 2];
        outp[n * D + dd] = deq((dd & 1) ? (byte >> 4) : (byte & 15), sc[n * (D / 16) + dd / 16]) *
                           (double)d;
      }
  };
  const int64_t kvoff = ((int64_t)b * Hkv + hk) * nd;
  deq_rows(k + kvoff, s_enc[1], dec[1], g.K.data());
  {
    const int npad = (N + 15) / 16 * 16;
    std::vector<uint8_t> vc((size_t)D * npad / 2), vs((size_t)D * npad / 16);
    quantize_tokens_T(v + kvoff, N, D, s_enc[2], vc.data(), vs.data(), npad);
    for (int dd = 0; dd < D; ++dd)
      for (int64_t n = 0; n < N; ++n) {
        uint8_t byte = vc[dd * (npad / 2) + n / 2];
        g.V[n * D + dd] = deq((n & 1) ? (byte >> 4) : (byte & 15), vs[dd * (npad / 16) + n / 16]) *
                          (double)dec[2];
      }
  }
  for (int gg = 0; gg < g.G; ++gg) {
    const int64_t qoff = ((int64_t)b * H + hk * g.G + gg) * nd;
    deq_rows(q + qoff, s_enc[0], dec[0], &g.Q[gg * nd]);
    for (int64_t e = 0; e < nd; ++e) g.dO[gg * nd + e] = (double)bf16_to_f32(dout[qoff + e]);
  }
  return g;
}

// One query row of head gg of the group: P (N), dS (N) and D; row masked to
// keys <= i when causal.
void bwd_row(const BwdGroup& g, int gg, int i, int causal, double scale, double* P, double* dS,
             double* Dout) {
  const int N = g.N, D = g.D;
  const double* qi = &g.Q[((int64_t)gg * N + i) * D];
  const double* di = &g.dO[((int64_t)gg * N + i) * D];
  const int jmax = causal ? i + 1 : N;
  double mx = -INFINITY;
  for (int j = 0; j < jmax; ++j) {
    double s = 0.0;
    for (int d = 0; d < D; ++d) s += qi[d] * g.K[(int64_t)j * D + d];
    P[j] = scale * s;
    mx = std::max(mx, P[j]);
  }
  double sum = 0.0;
  for (int j = 0; j < jmax; ++j) sum += std::exp(P[j] - mx);
  const double lse = mx + std::log(sum);
  double Dsum = 0.0;
  for (int j = 0; j < N; ++j) {
    if (j >= jmax) {
      P[j] = 0.0;
      dS[j] = 0.0;
      continue;
    }
    P[j] = std::exp(P[j] - lse);
    double dp = 0.0;
    for (int d = 0; d < D; ++d) dp += di[d] * g.V[(int64_t)j * D + d];
    dS[j] = dp;  // dP for now
    Dsum += P[j] * dp;
  }
  for (int j = 0; j < jmax; ++j) dS[j] = P[j] * (dS[j] - Dsum);
  *Dout = Dsum;
}

}  // namespace

extern "C" {

uint8_t ora_e2m1_encode(float y) { return e2m1_encode(y); }
float ora_e2m1_decode(uint8_t c) { return e2m1_decode(c); }
uint8_t ora_e4m3_encode(float y) { return e4m3_encode(y); }
float ora_e4m3_decode(uint8_t c) { return e4m3_decode(c); }

// Codes of the fp32 bit patterns start .. start+count-1, one byte each; NaN
// inputs (outside the contract) give the marker 0xFF.
void ora_e2m1_encode_range(uint32_t start, int64_t count, uint8_t* out, int nthreads) {
  const int64_t chunk = 1 << 16;
  parallel_for((count + chunk - 1) / chunk, nthreads, [&](int64_t c) {
    int64_t hi = std::min(count, (c + 1) * chunk);
    for (int64_t i = c * chunk; i < hi; ++i) {
      uint32_t u = start + (uint32_t)i;
      float f;
      std::memcpy(&f, &u, 4);
      out[i] = std::isnan(f) ? 0xFF : e2m1_encode(f);
    }
  });
}

void ora_e4m3_encode_range(uint32_t start, int64_t count, uint8_t* out, int nthreads) {
  e4m3_encode(0.0f);  // build the magnitude table before the threads start
  const int64_t chunk = 1 << 16;
  parallel_for((count + chunk - 1) / chunk, nthreads, [&](int64_t c) {
    int64_t hi = std::min(count, (c + 1) * chunk);
    for (int64_t i = c * chunk; i < hi; ++i) {
      uint32_t u = start + (uint32_t)i;
      float f;
      std::memcpy(&f, &u, 4);
      out[i] = std::isnan(f) ? 0xFF : e4m3_encode(f);
    }
  });
}

float ora_amax_bf16(const uint16_t* x, int64_t n) { return amax_bf16(x, n); }

void ora_tensor_scale(float amax, float* s_enc, float* d) { tensor_scale(amax, s_enc, d); }

// One block of n <= 16 fp32 values: n codes (one per byte) and the scale byte.
void ora_quantize_block(const float* x, int n, float s_enc, uint8_t* codes, uint8_t* scale) {
  quantize_block(x, n, s_enc, codes, scale);
}

void ora_quantize_rows(const uint16_t* x, int64_t rows, int cols, float s_enc, uint8_t* codes,
                       uint8_t* scales, int nthreads) {
  e4m3_encode(0.0f);
  quantize_rows(x, rows, cols, s_enc, codes, scales, nthreads);
}

// Smoothed rows: the values fl32(x - mean[col]) (mean: one fp32 per column).
void ora_quantize_rows_smoothed(const uint16_t* x, int64_t rows, int cols, float s_enc,
                                const float* mean, uint8_t* codes, uint8_t* scales, int nthreads) {
  e4m3_encode(0.0f);
  quantize_rows(x, rows, cols, s_enc, codes, scales, nthreads, mean);
}

// Smoothing (flags 32, 64): the channel means of one head's slab x [N][D]
// (amax: max |x| of the whole raw tensor), max |x - mean| over G slabs, and
// the score bias delta_j cs of one query head (kmean may be NULL).
void ora_channel_mean(const uint16_t* x, int N, int D, float amax, float* mean) {
  channel_mean(x, N, D, amax, mean);
}
float ora_smoothed_amax(const uint16_t* x, int64_t G, int N, int D, const float* mean) {
  return smoothed_amax(x, G, N, D, mean);
}
void ora_score_bias(const float* qmean, const uint16_t* k, const float* kmean, int N, int D,
                    double* delta, double* absum) {
  score_bias(qmean, k, kmean, N, D, delta, absum);
}

void ora_quantize_tokens_T(const uint16_t* x, int N, int D, float s_enc, uint8_t* codes,
                           uint8_t* scales, int npad) {
  quantize_tokens_T(x, N, D, s_enc, codes, scales, npad);
}

// EFQ P generation of one block (n <= 16 shifted scores z, -inf when masked):
// n codes and the scale byte (P tensor scale 2^-10); returns E (INT32_MIN when
// every key is masked).
int ora_efq_block(const double* z, int n, uint8_t* codes, uint8_t* scale) {
  e4m3_encode(0.0f);
  return efq_block(z, n, codes, scale);
}

// FP8 V (flag 16's quantiser): x [N][D] bf16 -> codes [D][npad]; the scale
// comes from ora_fp8_tensor_scale of the whole tensor's maximum.
void ora_fp8_tensor_scale(float amax, float* s8, float* d8) { fp8_tensor_scale(amax, s8, d8); }
void ora_quantize_fp8_tokens_T(const uint16_t* x, int N, int D, float s8, uint8_t* codes,
                               int npad) {
  e4m3_encode(0.0f);
  quantize_fp8_tokens_T(x, N, D, s8, codes, npad);
}

// Unscaled scores of one head: S[i][j] = fl32(exact q~_i . k~_j), contraction
// units (before d_Q d_K), no mask. S is [N][N].
int ora_scores_head(const uint16_t* q, const uint16_t* k, int B, int H, int Hkv, int N, int D,
                    int b, int h, float* S, int nthreads) {
  if (B <= 0 || H <= 0 || Hkv <= 0 || H % Hkv || N <= 0 || D % 16 || b >= B || h >= H) return -1;
  e4m3_encode(0.0f);
  Tensors T{q, k, k, B, H, Hkv, N, D, 0, 0, 0, 0, 0, 0, false};
  tensor_scale(amax_bf16(q, (int64_t)B * H * N * D), &T.sq, &T.dq);
  tensor_scale(amax_bf16(k, (int64_t)B * Hkv * N * D), &T.sk, &T.dk);
  const int hk = h / (H / Hkv);
  std::vector<uint8_t> qc((size_t)N * D / 2), qs((size_t)N * D / 16), kc(qc.size()), ks(qs.size());
  quantize_rows(q + ((int64_t)b * H + h) * N * D, N, D, T.sq, qc.data(), qs.data(), nthreads);
  quantize_rows(k + ((int64_t)b * Hkv + hk) * N * D, N, D, T.sk, kc.data(), ks.data(), nthreads);
  auto val = [&](const std::vector<uint8_t>& c, const std::vector<uint8_t>& s, int64_t n, int d) {
    uint8_t byte = c[n * (D / 2) + d / 2];
    return deq((d & 1) ? (byte >> 4) : (byte & 15), s[n * (D / 16) + d / 16]);
  };
  parallel_for(N, nthreads, [&](int64_t i) {
    for (int j = 0; j < N; ++j) {
      double s = 0.0;
      for (int d = 0; d < D; ++d) s += val(qc, qs, i, d) * val(kc, ks, j, d);
      S[i * N + j] = (float)s;
    }
  });
  return 0;
}

// The FP4 attention backward (reading at bwd_row / make_bwd_group).
//   q, dout [B][H][N][D], k, v [B][Hkv][N][D] bf16 bit patterns.
//   q_rows: nq (b, h, i) triples whose dq rows are wanted (NULL: every row);
//   kv_rows: nkv (b, hk, j) triples whose dk and dv rows are wanted (NULL:
//   every row; nkv < 0: none). dq_out [nq][D], dk_out / dv_out [nkv][D]
//   (fp64, may be NULL), D_out [B][H][N] (may be NULL; computed for every
//   row of a group that needs any).
// Returns 0, or -1 on bad arguments.
int ora_attn_bwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* dout,
                 int B, int H, int Hkv, int N, int D, int causal, float softmax_scale,
                 const int64_t* q_rows, int64_t nq, const int64_t* kv_rows, int64_t nkv,
                 double* dq_out, double* dk_out, double* dv_out, double* D_out, int nthreads) {
  if (B <= 0 || H <= 0 || Hkv <= 0 || H % Hkv || N <= 0 || D <= 0 || D % 16) return -1;
  e4m3_encode(0.0f);
  float se[3], dc[3];
  tensor_scale(amax_bf16(q, (int64_t)B * H * N * D), &se[0], &dc[0]);
  tensor_scale(amax_bf16(k, (int64_t)B * Hkv * N * D), &se[1], &dc[1]);
  tensor_scale(amax_bf16(v, (int64_t)B * Hkv * N * D), &se[2], &dc[2]);
  if (!(softmax_scale > 0.0f)) softmax_scale = 1.0f / std::sqrt((float)D);
  const double scale = (double)softmax_scale;
  const int G = H / Hkv;
  std::vector<int64_t> allq, allkv;
  if (!q_rows) {
    nq = (int64_t)B * H * N;
    allq.resize((size_t)nq * 3);
    for (int64_t r = 0; r < nq; ++r) {
      allq[r * 3] = r / ((int64_t)H * N);
      allq[r * 3 + 1] = (r / N) % H;
      allq[r * 3 + 2] = r % N;
    }
    q_rows = allq.data();
  }
  if (!kv_rows && nkv >= 0) {
    nkv = (int64_t)B * Hkv * N;
    allkv.resize((size_t)nkv * 3);
    for (int64_t r = 0; r < nkv; ++r) {
      allkv[r * 3] = r / ((int64_t)Hkv * N);
      allkv[r * 3 + 1] = (r / N) % Hkv;
      allkv[r * 3 + 2] = r % N;
    }
    kv_rows = allkv.data();
  }
  if (nkv < 0) nkv = 0;
  for (int64_t r = 0; r < nq; ++r)
    if (q_rows[r * 3] < 0 || q_rows[r * 3] >= B || q_rows[r * 3 + 1] < 0 ||
        q_rows[r * 3 + 1] >= H || q_rows[r * 3 + 2] < 0 || q_rows[r * 3 + 2] >= N)
      return -1;
  for (int64_t r = 0; r < nkv; ++r)
    if (kv_rows[r * 3] < 0 || kv_rows[r * 3] >= B || kv_rows[r * 3 + 1] < 0 ||
        kv_rows[r * 3 + 1] >= Hkv || kv_rows[r * 3 + 2] < 0 || kv_rows[r * 3 + 2] >= N)
      return -1;
  for (int b = 0; b < B; ++b)
    for (int hk = 0; hk < Hkv; ++hk) {
      std::vector<int64_t> mq, mkv;
      for (int64_t r = 0; r < nq; ++r)
        if (q_rows[r * 3] == b && q_rows[r * 3 + 1] / G == hk) mq.push_back(r);
      for (int64_t r = 0; r < nkv; ++r)
        if (kv_rows[r * 3] == b && kv_rows[r * 3 + 1] == hk) mkv.push_back(r);
      if (mq.empty() && mkv.empty() && !D_out) continue;
      const BwdGroup g = make_bwd_group(q, k, v, dout, B, H, Hkv, N, D, b, hk, se, dc);
      // dq rows: one row's P and dS each
      parallel_for((int64_t)mq.size(), nthreads, [&](int64_t u) {
        const int64_t r = mq[u];
        const int gg = (int)q_rows[r * 3 + 1] % G, i = (int)q_rows[r * 3 + 2];
        std::vector<double> P(N), dS(N);
        double Dv;
        bwd_row(g, gg, i, causal, scale, P.data(), dS.data(), &Dv);
        if (dq_out)
          for (int d = 0; d < D; ++d) {
            double acc = 0.0;
            for (int j = 0; j < N; ++j) acc += dS[j] * g.K[(int64_t)j * D + d];
            dq_out[r * D + d] = scale * acc;
          }
      });
      if (mkv.empty() && !D_out) continue;
      // dk, dv rows and D: every query row of every head of the group
      std::vector<double> dK(mkv.size() * D, 0.0), dV(mkv.size() * D, 0.0);
      std::vector<double> Dall((size_t)G * N);
      std::vector<double> Pall, dSall;
      if (!mkv.empty()) {
        Pall.resize((size_t)G * N * mkv.size());
        dSall.resize(Pall.size());
      }
      parallel_for((int64_t)G * N, nthreads, [&](int64_t rr) {
        const int gg = (int)(rr / N), i = (int)(rr % N);
        std::vector<double> P(N), dS(N);
        bwd_row(g, gg, i, causal, scale, P.data(), dS.data(), &Dall[rr]);
        for (size_t u = 0; u < mkv.size(); ++u) {
          const int j = (int)kv_rows[mkv[u] * 3 + 2];
          Pall[(size_t)rr * mkv.size() + u] = P[j];
          dSall[(size_t)rr * mkv.size() + u] = dS[j];
        }
      });
      if (D_out)
        for (int gg = 0; gg < G; ++gg)
          for (int i = 0; i < N; ++i)
            D_out[((int64_t)b * H + hk * G + gg) * N + i] = Dall[(size_t)gg * N + i];
      parallel_for((int64_t)mkv.size(), nthreads, [&](int64_t u) {
        for (int d = 0; d < D; ++d) {
          double ak = 0.0, av = 0.0;
          for (int64_t rr = 0; rr < (int64_t)G * N; ++rr) {
            const size_t at = (size_t)rr * mkv.size() + u;
            ak += dSall[at] * g.Q[rr * D + d];
            av += Pall[at] * g.dO[rr * D + d];
          }
          if (dk_out) dk_out[mkv[u] * D + d] = scale * ak;
          if (dv_out) dv_out[mkv[u] * D + d] = av;
        }
      });
    }
  return 0;
}

// The tiled NVFP4 attention forward.
//   q [B][H][N][D], k and v [B][Hkv][N][D], bf16 bit patterns.
//   rows: nrows (b, h, i) triples to compute, or NULL for every row.
//   out_bf16 / out_f64: [nrows][D] (or [B][H][N][D] when rows is NULL); either
//   may be NULL. out_ml: [nrows][3] final (m, l) and the largest relative
//   uncertainty eps of the row's p (nonzero with flags 2 or 4), may be NULL.
//   Bc: key tile (128 on the path); flags: 1 = denominator from p~,
//   2 = flip bound into out_flip ([nrows][D], may be NULL otherwise),
//   4 = perturb p within the flip bound's uncertainty (tests the bound),
//   8 = EFQ-Softmax P generation (efq_block), denominator from its p~,
//   16 = P and V in FP8 E4M3 (not with 8), 32 = smooth K, 64 = smooth Q
//   (channel_mean; N <= 2^19 with either).
// Returns 0, or -1 on bad arguments.
int ora_attn_fwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int H, int Hkv,
                 int N, int D, int causal, float softmax_scale, int Bc, int flags,
                 const int64_t* rows, int64_t nrows, uint16_t* out_bf16, double* out_f64,
                 double* out_ml, double* out_flip, int nthreads) {
  if (B <= 0 || H <= 0 || Hkv <= 0 || H % Hkv || N <= 0 || D <= 0 || D % 16 || Bc <= 0 ||
      Bc % 16)
    return -1;
  e4m3_encode(0.0f);
  if ((flags & FLAG_FP8PV) && (flags & FLAG_EFQ)) return -1;
  if ((flags & (FLAG_SMOOTH_K | FLAG_SMOOTH_Q)) && N > (1 << 19)) return -1;
  Tensors T{q, k, v, B, H, Hkv, N, D, 0, 0, 0, 0, 0, 0, (flags & FLAG_FP8PV) != 0};
  if (!(softmax_scale > 0.0f)) softmax_scale = 1.0f / std::sqrt((float)D);
  const int64_t Gq = (int64_t)B * H, Gk = (int64_t)B * Hkv;
  std::vector<float> qmean, kmean;
  std::vector<double> delta, absum, bias, bias_unc;
  float amax_q = amax_bf16(q, Gq * N * D), amax_k = amax_bf16(k, Gk * N * D);
  if (flags & FLAG_SMOOTH_K) {
    kmean.resize((size_t)(Gk * D));
    for (int64_t g = 0; g < Gk; ++g) channel_mean(k + g * N * D, N, D, amax_k, &kmean[g * D]);
    amax_k = smoothed_amax(k, Gk, N, D, kmean.data());
    T.kmean = kmean.data();
  }
  if (flags & FLAG_SMOOTH_Q) {
    qmean.resize((size_t)(Gq * D));
    for (int64_t g = 0; g < Gq; ++g) channel_mean(q + g * N * D, N, D, amax_q, &qmean[g * D]);
    amax_q = smoothed_amax(q, Gq, N, D, qmean.data());
    T.qmean = qmean.data();
    delta.resize((size_t)(Gq * N));
    absum.resize(delta.size());
    parallel_for(Gq, nthreads, [&](int64_t g) {
      const int64_t gk = (g / H) * Hkv + (g % H) / (H / Hkv);
      score_bias(&qmean[g * D], k + gk * N * D, T.kmean ? T.kmean + gk * D : nullptr, N, D,
                 &delta[g * N], &absum[g * N]);
    });
  }
  tensor_scale(amax_q, &T.sq, &T.dq);
  tensor_scale(amax_k, &T.sk, &T.dk);
  if (flags & FLAG_SMOOTH_Q) {
    // beta_j = delta_j s_Q s_K. For the flip bound only: another correct fp32
    // evaluation of the correction (a D-term fp32 dot product, one fp32
    // product with fl32(s_Q s_K), and beta carried into the fp32 score sum as
    // two parts of 11 significant bits each) lies within
    //   (D + 4) 2^-24 s_Q s_K sum_d |mean_d k'_d| + 2^-20 |beta_j|
    // of beta_j; bias_unc holds that distance.
    const double sqsk = (double)T.sq * (double)T.sk;
    bias.resize(delta.size());
    bias_unc.resize(delta.size());
    for (size_t u = 0; u < delta.size(); ++u) {
      bias[u] = delta[u] * sqsk;
      bias_unc[u] = (D + 4) * std::ldexp(1.0, -24) * sqsk * absum[u] +
                    std::ldexp(1.0, -20) * std::fabs(bias[u]);
    }
    T.bias = bias.data();
    T.bias_unc = bias_unc.data();
  }
  if (T.fp8v)
    fp8_tensor_scale(amax_bf16(v, (int64_t)B * Hkv * N * D), &T.sv, &T.dv);
  else
    tensor_scale(amax_bf16(v, (int64_t)B * Hkv * N * D), &T.sv, &T.dv);
  float c = T.dq * T.dk;
  c = c * softmax_scale;
  c = c * kLog2e;

  std::vector<int64_t> all;
  if (!rows) {
    nrows = (int64_t)B * H * N;
    all.resize((size_t)nrows * 3);
    for (int64_t r = 0; r < nrows; ++r) {
      all[r * 3 + 0] = r / ((int64_t)H * N);
      all[r * 3 + 1] = (r / N) % H;
      all[r * 3 + 2] = r % N;
    }
    rows = all.data();
  }
  for (int64_t r = 0; r < nrows; ++r)
    if (rows[r * 3] < 0 || rows[r * 3] >= B || rows[r * 3 + 1] < 0 || rows[r * 3 + 1] >= H ||
        rows[r * 3 + 2] < 0 || rows[r * 3 + 2] >= N)
      return -1;
  const int G = H / Hkv;
  for (int b = 0; b < B; ++b)
    for (int hk = 0; hk < Hkv; ++hk) {
      std::vector<int64_t> mine;
      for (int64_t r = 0; r < nrows; ++r)
        if (rows[r * 3] == b && rows[r * 3 + 1] / G == hk) mine.push_back(r);
      if (mine.empty()) continue;
      KVGroup g = make_group(T, b, hk);
      parallel_for((int64_t)mine.size(), nthreads, [&](int64_t u) {
        int64_t r = mine[u];
        row_forward(T, g, b, (int)rows[r * 3 + 1], (int)rows[r * 3 + 2], c, Bc, causal, flags,
                    out_f64 ? out_f64 + r * D : nullptr, out_ml ? out_ml + r * 3 : nullptr,
                    out_bf16 ? out_bf16 + r * D : nullptr, out_flip ? out_flip + r * D : nullptr);
      });
    }
  return 0;
}

}  // extern "C"
