/*
 * fp4attn: NVFP4 (4-bit) FlashAttention on NVIDIA B200 (sm_100a): the forward,
 * its variants (EFQ-Softmax P, FP8 P and V, Q/K smoothing) and the backward.
 *
 * C ABI. Every pointer argument is a device pointer owned by the caller unless
 * stated otherwise; the library allocates no device memory on any call path,
 * keeps no state between calls beyond a per-device error word, and launches
 * its work asynchronously on the caller's stream (a cudaStream_t passed as
 * void*; NULL is the legacy default stream). Arguments are validated before
 * anything is launched: a call that returns an error has launched nothing.
 * Kernel-side failures (a bounded wait that expired) are reported later by
 * fp4_status(). Functions are thread-safe; fp4_last_error() is per thread.
 *
 * Method. The pages this library restates describe 4-bit attention in which
 * both QK^T and PV run as 4-bit block-scaled contractions while the online-
 * softmax state stays in higher precision (HiFA4 summary, theflow.svmpsp.dev
 * related-papers feed), the probability tile is formed from exponentials in
 * higher precision and quantised before the low-bit PV product, and the
 * FlashAttention row-maximum update, historical rescaling, high-precision
 * accumulation and final normalisation are kept (EFQ-Softmax abstract,
 * scholarbro.com page "AVQ Attention: Adaptive Vector-Quantized Attention").
 * The operand format is block-scaled E2M1, NVFP4 (TetraJet-v2 abstract,
 * searcharxiv.com author page "Pengle Zhang"), run on the FP4 tensor cores of
 * Blackwell GPUs (SageAttention3 abstract, same page).
 *
 * NVFP4 as implemented (the pages name the format but give no recipe; this is
 * the standard two-level reading):
 *   element   E2M1 code, 4 bits: magnitudes {0,.5,1,1.5,2,3,4,6}, sign bit 3;
 *             two codes per byte, element 2i in the low nibble of byte i
 *   block     16 consecutive elements share one E4M3 scale byte (UE4M3)
 *   tensor    one fp32 scale s_enc = 2688 / amax (1 if amax == 0, FLT_MAX on
 *             overflow), amax = max |x| over the whole tensor
 *   block scale  e = E4M3(fl(fl(a_b / 6) * s_enc)), a_b = block max |x|
 *   codes        E2M1(fl(x * r)), r = fl(s_enc / dec(e)) or 0 if dec(e) == 0
 *   conversions  round to nearest even, saturating (E2M1 to +-6, E4M3 to 448)
 *   value        x ~= val(code) * dec(e) / s_enc
 *
 * Attention forward (fp4_attn_fwd), per query row i of head h:
 *   S_ij = (q~_i . k~_j) as a block-scaled FP4 contraction, fp32 accumulation
 *   x_ij = S_ij * d_Q * d_K * softmax_scale * log2(e), masked keys -> -inf
 *   keys in tiles of 128 (the tile is part of the method: the running maximum
 *   is updated once per tile): m_new = max(m, max_j x_ij), alpha = 2^(m-m_new)
 *   p_ij = 2^(x_ij - m_new) in fp32; l = alpha l + sum_j p_ij (fp32, before
 *   quantisation); O = alpha O + NVFP4(p) . v~ with P quantised per 16 keys
 *   with the fixed tensor scale 2688 (p <= 1); out = O d_P d_V / l, bf16.
 *   Causal masking keeps keys j <= i (query and key positions aligned at 0).
 *   Grouped heads: query head h reads key/value head h / (H / Hkv).
 *
 * Tensor layouts (row-major, contiguous, 16-byte aligned base pointers):
 *   q, out  bf16 [B][H][N][D]      k, v  bf16 [B][Hkv][N][D]
 *   D in {64, 128}; H % Hkv == 0; N >= 1; B, H <= 65535.
 */
#ifndef FP4ATTN_H_
#define FP4ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FP4_OK = 0,
  FP4_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or shape */
  FP4_ERR_UNSUPPORTED = 2, /* head dim not in {64,128}, or the device is not sm_100 */
  FP4_ERR_WORKSPACE = 3,   /* workspace smaller than the entry's *_workspace_bytes() */
  FP4_ERR_CUDA = 4,        /* a CUDA runtime call failed (message in fp4_last_error) */
  FP4_ERR_TIMEOUT = 5,     /* a kernel's bounded wait expired (from fp4_status) */
  FP4_ERR_BOUNDS = 6       /* FP4_DEBUG builds: a kernel's bounds or alignment check failed
                              (from fp4_status; the access was skipped) */
} fp4_status_t;

typedef enum {
  FP4_BLOCK_ALONG_D = 0,  /* Q, K: blocks of 16 along the head dimension */
  FP4_BLOCK_ALONG_N_T = 1 /* V: blocks of 16 along tokens, stored transposed */
} fp4_axis_t;

/*
 * A quantised tensor as fp4_quantize() writes it (device pointers).
 * Npad = N rounded up to a multiple of 128; G = B*H (Q) or B*Hkv (K, V).
 *   FP4_BLOCK_ALONG_D:   codes [G][Npad][D/2] (rows >= N are zero)
 *   FP4_BLOCK_ALONG_N_T: codes [G][D][Npad/2] (tokens >= N are zero)
 *   scales: the tensor-core block-scale layout in 512-byte atoms; an atom holds
 *   128 rows x 4 consecutive blocks, row r and block k at byte
 *   (r % 32) * 16 + (r / 32) * 4 + k.
 *     ALONG_D:   atom ((g * Npad/128 + n/128) * D/64 + block/4) for row n
 *     ALONG_N_T: rows are the D channels (padded to 128 with zero scales);
 *                atom (g * Npad/64 + token_block/4)
 *   amax: one fp32, max |x| of the whole source tensor.
 */
typedef struct {
  const uint8_t* codes;
  const uint8_t* scales;
  const float* amax;
} fp4_tensor_t;

/* Bytes of codes / scales fp4_quantize() writes for a [G][N][D] tensor. */
size_t fp4_codes_bytes(int G, int N, int D, fp4_axis_t axis);
size_t fp4_scales_bytes(int G, int N, int D, fp4_axis_t axis);

/* Workspace fp4_attn_fwd() needs (holds quantised Q, K, V and their maxima). */
size_t fp4_attn_workspace_bytes(int B, int H, int Hkv, int N, int D);

/*
 * NVFP4 quantisation of one bf16 tensor x [G][N][D] (steps: amax over the whole
 * tensor, then codes and block scales as described above).
 * Outputs codes (fp4_codes_bytes), scales (fp4_scales_bytes) and *amax (one
 * fp32) in device memory; all three must be 16-byte aligned.
 */
fp4_status_t fp4_quantize(const void* x, int G, int N, int D, fp4_axis_t axis, uint8_t* codes,
                          uint8_t* scales, float* amax, void* stream);

/*
 * The tensor maximum alone (the first step of fp4_quantize): *amax = max |x|
 * over a bf16 tensor x [G][N][D] (shape rules as fp4_quantize; x 16-byte
 * aligned, amax one fp32 in device memory, 4-byte aligned). With
 * fp4_quantize_scaled this splits fp4_quantize in two, so that a tensor held
 * in shards (by head, one shard per GPU) can be quantised exactly as the whole
 * tensor would be: each shard's maximum is computed here, the maxima are
 * combined by max across the shards (the head-sharded forward all-reduces
 * them), and every shard is then quantised with the combined value. The
 * pages' recipe has one fp32 scale per tensor (TetraJet-v2 abstract); this
 * entry point only lets that scale be formed from shards.
 */
fp4_status_t fp4_amax(const void* x, int G, int N, int D, float* amax, void* stream);

/*
 * fp4_quantize with the tensor maximum given instead of computed: the tensor
 * scale is s_enc = 2688 / *amax, read on the device when the kernel runs
 * (amax: one fp32 in device memory, 4-byte aligned; it must be >= max |x|,
 * else the largest blocks saturate to the E4M3 maximum 448). Writes codes
 * and scales as fp4_quantize (16-byte aligned); *amax is not modified.
 */
fp4_status_t fp4_quantize_scaled(const void* x, int G, int N, int D, fp4_axis_t axis,
                                 const float* amax, uint8_t* codes, uint8_t* scales,
                                 void* stream);

/*
 * The block scales fp4_quantize() wrote (tensor-core atom layout, above) in
 * their logical layout, for callers that inspect or compare them:
 *   FP4_BLOCK_ALONG_D:   canonical [G][N][D/16], byte (g, n, b) = scale of
 *                        row n, block b (16 elements along D)
 *   FP4_BLOCK_ALONG_N_T: canonical [G][D][Npad/16], byte (g, d, t) = scale of
 *                        channel d, token block t (tokens >= N have zero codes)
 * native and canonical are device pointers; canonical holds G*N*D/16 or
 * G*D*Npad/16 bytes. The pages define no layout; this is the plain one.
 */
fp4_status_t fp4_scales_to_canonical(const uint8_t* native, int G, int N, int D,
                                     fp4_axis_t axis, uint8_t* canonical, void* stream);

/*
 * The NVFP4 attention forward: quantises q and k along D and v along tokens
 * into the workspace, then runs the fused forward. softmax_scale <= 0 (or NaN)
 * selects 1/sqrt(D). out may not alias q, k, v or the workspace.
 */
fp4_status_t fp4_attn_fwd(const void* q, const void* k, const void* v, void* out, int B, int H,
                          int Hkv, int N, int D, int causal, float softmax_scale, void* stream,
                          void* workspace, size_t workspace_bytes);

/*
 * The attention forward end to end from HOST memory: q_host, k_host, v_host
 * (bf16, layouts as fp4_attn_fwd) are copied to the device, fp4_attn_fwd runs,
 * and the output is copied back into out_host; the call returns once
 * out_host holds the result (it synchronises `stream`). One cudaMemcpyAsync
 * per tensor in each direction, all on `stream`. Host buffers should be
 * pinned (cudaHostAlloc / cudaHostRegister) for the copies to run at full
 * speed; pageable memory works but copies through a staging buffer.
 * dev_workspace (device, caller-owned, 16-byte aligned) holds the device
 * copies of q, k, v and out followed by fp4_attn_fwd's workspace:
 * fp4_attn_host_workspace_bytes() bytes. Errors as fp4_attn_fwd; a failed
 * copy returns FP4_ERR_CUDA. The pages define no interface (the method is the
 * forward above); this entry exists so that a whole host-to-host call is one
 * C function.
 */
size_t fp4_attn_host_workspace_bytes(int B, int H, int Hkv, int N, int D);
fp4_status_t fp4_attn_fwd_host(const void* q_host, const void* k_host, const void* v_host,
                               void* out_host, int B, int H, int Hkv, int N, int D, int causal,
                               float softmax_scale, void* stream, void* dev_workspace,
                               size_t dev_workspace_bytes);

/*
 * The fused forward alone, on tensors fp4_quantize() produced (q with
 * FP4_BLOCK_ALONG_D and G = B*H; k with FP4_BLOCK_ALONG_D and v with
 * FP4_BLOCK_ALONG_N_T, G = B*Hkv), all for the same N and D.
 */
fp4_status_t fp4_attn_fwd_quantized(const fp4_tensor_t* q, const fp4_tensor_t* k,
                                    const fp4_tensor_t* v, void* out, int B, int H, int Hkv,
                                    int N, int D, int causal, float softmax_scale, void* stream);

/*
 * The EFQ-Softmax variant of fp4_attn_fwd / fp4_attn_fwd_quantized (same
 * arguments, layouts and errors). P is generated without exponentials
 * (EFQ-Softmax abstract, scholarbro.com page "AVQ Attention: Adaptive
 * Vector-Quantized Attention": an exponent-only scale per microscaling block
 * chosen from the local maximum, the shifted scores mapped to a residual
 * domain, nonnegative E2M1 codes from a single affine rule, and the same
 * operand in the numerator P~V and the denominator P~1). The abstract gives no
 * formula; the reading implemented, per 16-key block of a row with
 * z = x - m (log2 units) and the running maximum m updated as above:
 *   E = floor(max z) - 2            (shared exponent; 2 = E2M1's largest)
 *   code = clamp(rne(2 (z - E) + 2), 0, 7)   (rne: round half to even)
 *   p~ = val(code) * 2^E            (block scale byte 2^(E + 10), P's tensor
 *                                     scale 2^-10; a block with E < -19 is zero)
 *   l = alpha l + sum_j p~_j,  out = O / l  (O and l both from p~).
 */
fp4_status_t fp4_attn_fwd_efq(const void* q, const void* k, const void* v, void* out, int B,
                              int H, int Hkv, int N, int D, int causal, float softmax_scale,
                              void* stream, void* workspace, size_t workspace_bytes);
fp4_status_t fp4_attn_fwd_quantized_efq(const fp4_tensor_t* q, const fp4_tensor_t* k,
                                        const fp4_tensor_t* v, void* out, int B, int H, int Hkv,
                                        int N, int D, int causal, float softmax_scale,
                                        void* stream);

/*
 * FP8 V (the FP8 P/V variant below): x [G][N][D] bf16 -> E4M3 codes
 * [G][D][Npad] (one byte per element, channel-major, keys >= N zero; Npad = N
 * rounded up to 128). SageAttention2 abstract (searcharxiv.com author page
 * "Pengle Zhang": P~ and V in FP8 for the PV product) gives no recipe; the
 * reading: one fp32 scale per tensor, s8 = 448 / amax (1 if amax == 0, FLT_MAX
 * if the quotient overflows), code = E4M3(fl(v s8)), round to nearest even,
 * saturating; v~ = dec(code) / s8. Steps: *amax = max |x| (written, stream
 * order), then the codes. fp4_fp8_codes_bytes gives the size of codes (0 for a
 * bad shape). x and codes 16-byte aligned, amax 4-byte aligned, all device
 * memory, caller-owned. Errors: as fp4_quantize.
 */
size_t fp4_fp8_codes_bytes(int G, int N, int D);
fp4_status_t fp4_quantize_fp8(const void* x, int G, int N, int D, uint8_t* codes, float* amax,
                              void* stream);
/* The codes step alone, with a given tensor maximum *amax (device memory, read
 * only; e.g. combined over shards as for fp4_quantize_scaled). */
fp4_status_t fp4_quantize_fp8_scaled(const void* x, int G, int N, int D, const float* amax,
                                     uint8_t* codes, void* stream);

/*
 * The FP8 P/V variant of fp4_attn_fwd / fp4_attn_fwd_quantized (same
 * arguments, layouts and errors, except as stated). Q and K and S = QK^T as in
 * the method; V quantised by fp4_quantize_fp8; P per key in E4M3 without block
 * scales: p~ = E4M3(fl(256 p)) / 256 with p = 2^(x - m) (the 256 keeps every
 * p <= 1 inside E4M3's range and its subnormals below 2^-17); O = P~ V~ as a
 * tcgen05 kind::f8f6f4 contraction; l sums the unquantised p; out = O / l.
 * fp4_attn_fwd_fp8pv needs fp4_attn_workspace_bytes_fp8pv bytes of workspace.
 * fp4_attn_fwd_quantized_fp8pv takes v->codes from fp4_quantize_fp8 and
 * v->amax its maximum; v->scales is not read and may be NULL.
 */
/*
 * Outlier smoothing of Q and K before NVFP4 (SageAttention2 abstract,
 * searcharxiv.com author page "Pengle Zhang": Q is smoothed to make the
 * low-bit QK^T more accurate). The page gives no formula; the reading:
 *   per (batch, head) and channel d, mean_d over the head's N tokens, on a
 *   fixed-point grid so that it does not depend on summation order: each
 *   element truncated toward zero to a multiple of 2^-s, s = 44 - E with
 *   2^(E-1) <= amax < 2^E (amax: max |x| of the whole raw tensor), the
 *   integers summed exactly in 64 bits (hence N <= 2^19), and
 *   mean = fl32(fl64(fl64(T) * 2^-s) / N) (0 when amax == 0);
 *   x' = fl32(x - mean) quantised as NVFP4 with the tensor scale taken from
 *   max |x'| over the whole smoothed tensor.
 *   Smoothing K changes every score of a query row by the same amount, which
 *   the softmax cancels. Smoothing Q leaves the key-dependent term
 *   mean_Q . k'_j, added back to the scores: delta_j = a sequential fp32 fma
 *   chain over d = 0..D-1 from 0 of mean_Q[d] * k'_j[d] (k' = fl32(k - mean_K)
 *   if K is smoothed, else k). In the contraction's units beta_j = fl32(delta_j *
 *   fl32(s_Q * s_K)) (the encode scales of the quantised Q' and K), split in
 *   two tf32 parts hi = tf32_rz(beta), lo = tf32_rz(fl32(beta - hi)) (low 13
 *   mantissa bits cleared); the fused kernel adds hi + lo to the S
 *   accumulator as a rank-1 tensor-core product before the scores are scaled.
 */
#define FP4_SMOOTH_K 1
#define FP4_SMOOTH_Q 2

/*
 * The whole smoothed forward: fp4_attn_fwd with Q and/or K smoothed (smooth =
 * FP4_SMOOTH_K | FP4_SMOOTH_Q, 0 gives the plain forward) and
 * fp4_attn_workspace_bytes_smooth bytes of workspace (0 for a bad shape or
 * N > 2^19). Same layouts and errors as fp4_attn_fwd; FP4_ERR_INVALID_ARG
 * for unknown smooth bits or N > 2^19.
 */
size_t fp4_attn_workspace_bytes_smooth(int B, int H, int Hkv, int N, int D);
fp4_status_t fp4_attn_fwd_smooth(const void* q, const void* k, const void* v, void* out, int B,
                                 int H, int Hkv, int N, int D, int causal, float softmax_scale,
                                 int smooth, void* stream, void* workspace,
                                 size_t workspace_bytes);

/*
 * The steps of the smoothed forward, one by one.
 * fp4_channel_mean: x [G][N][D] bf16 -> mean [G][D] fp32 on the grid of *amax
 *   (the raw tensor's maximum, device memory); sums: G*D uint64 device scratch
 *   (overwritten). N <= 2^19.
 * fp4_amax_smoothed: *amax = max |fl32(x - mean)| over x [G][N][D].
 * fp4_quantize_smoothed: NVFP4 codes and scales (FP4_BLOCK_ALONG_D layouts) of
 *   fl32(x - mean) with the tensor scale 2688 / *amax (amax of the smoothed
 *   tensor, device memory, read only).
 * fp4_score_bias: bias [B*H][Npad][8] fp32, per key (hi, lo, 0, 0, 0, 0, 0,
 *   0) (keys >= N all 0), from qmean [B*H][D], k [B][Hkv][N][D] bf16, kmean
 *   [B*Hkv][D] (NULL when K is not smoothed) and the maxima q_amax, k_amax
 *   (one fp32 each, device) the quantised Q' and K are encoded with.
 * fp4_attn_fwd_quantized_bias: fp4_attn_fwd_quantized (exp-then-quantize P)
 *   with that correction: S_ij + hi_j + lo_j before the scores are scaled.
 * Pointers: device memory, 16-byte aligned (amax 4-byte aligned).
 */
fp4_status_t fp4_channel_mean(const void* x, int G, int N, int D, const float* amax,
                              float* mean, unsigned long long* sums, void* stream);
fp4_status_t fp4_amax_smoothed(const void* x, int G, int N, int D, const float* mean, float* amax,
                               void* stream);
fp4_status_t fp4_quantize_smoothed(const void* x, int G, int N, int D, const float* mean,
                                   const float* amax, uint8_t* codes, uint8_t* scales,
                                   void* stream);
fp4_status_t fp4_score_bias(const float* qmean, const void* k, const float* kmean, int B, int H,
                            int Hkv, int N, int D, const float* q_amax, const float* k_amax,
                            float* bias, void* stream);
fp4_status_t fp4_attn_fwd_quantized_bias(const fp4_tensor_t* q, const fp4_tensor_t* k,
                                         const fp4_tensor_t* v, const float* bias, void* out,
                                         int B, int H, int Hkv, int N, int D, int causal,
                                         float softmax_scale, void* stream);

/*
 * Training support: the forward of fp4_attn_fwd that also writes, per query
 * row, lse [B*H][N] fp32 = log2 sum_j 2^(x_ij) with x_ij = S_ij * c (the
 * scores in log2 units, the quantity the backward needs to re-form P). Same
 * arguments as fp4_attn_fwd plus lse (device memory, 4-byte aligned).
 */
fp4_status_t fp4_attn_fwd_lse(const void* q, const void* k, const void* v, void* out, float* lse,
                              int B, int H, int Hkv, int N, int D, int causal,
                              float softmax_scale, void* stream, void* workspace,
                              size_t workspace_bytes);

/*
 * The FP4 attention backward. The Attn-QAT abstract (arxiv listing "Attn-QAT:
 * 4-Bit Attention With Quantization-Aware Training") asks that (1) the
 * backward recompute the attention scores in the forward's low precision and
 * (2) FlashAttention's gradient lose an implicit precision assumption; it
 * gives no formula. The reading implemented:
 *   q~, k~, v~  the forward's NVFP4 operands (same tensor scales, codes and
 *               block scales as fp4_attn_fwd), dequantised
 *   P_ij = 2^(S_ij c - lse_i)   scores recomputed from q~, k~ (1)
 *   dP_ij = dO_i . v~_j,  D_i = sum_j P_ij dP_ij   (2): D from this P and v~,
 *               not FlashAttention's dO . O, which assumes O = P V exactly
 *   dS = P (dP - D),  dq = scale dS k~,  dk = scale dS^T q~,  dv = P^T dO
 *   (dk, dv summed over the query heads of each key/value head)
 * with straight-through quantisers. Inputs: q, k, v as fp4_attn_fwd; out
 * [B][H][N][D] bf16, the forward's output; dout [B][H][N][D] bf16; lse from
 * fp4_attn_fwd_lse. Outputs (bf16): dq [B][H][N][D], dk and dv
 * [B][Hkv][N][D]. The contractions run on the tensor cores in bf16 with fp32
 * accumulation (P and dS rounded to bf16 for theirs). dq is accumulated in
 * one pass over the keys as A - (D - c) B with A = sum_j P_ij (dP_ij - c_i)
 * k~_j, B = sum_j P_ij k~_j and c_i = dO_i . out_i: out enters only through
 * c, an identity's free constant, so it changes the rounding and not the
 * definition above (D stays this P's; out close to P v~ keeps the terms of A
 * small). All device pointers 16-byte aligned (lse 4-byte); none may be NULL
 * (FP4_ERR_INVALID_ARG). workspace: fp4_attn_bwd_workspace_bytes(B, H, Hkv,
 * N, D) bytes, else FP4_ERR_WORKSPACE. The library owns no argument.
 */
size_t fp4_attn_bwd_workspace_bytes(int B, int H, int Hkv, int N, int D);
/*
 * For tensors held in shards (by head, one shard per GPU): the backward with
 * the three tensor maxima given, amax[3] = {max|q|, max|k|, max|v|} of the
 * whole tensors (device memory, 4-byte aligned; e.g. each shard's maxima
 * from fp4_amax combined by max across the shards), so that every shard's
 * operands are quantised as the whole tensors' are; and the training forward
 * on quantised tensors (fp4_quantize_scaled with the same maxima) writing lse.
 */
fp4_status_t fp4_attn_bwd_scaled(const void* q, const void* k, const void* v, const void* out,
                                 const void* dout, const float* lse, const float* amax, void* dq,
                                 void* dk, void* dv, int B, int H, int Hkv, int N, int D,
                                 int causal, float softmax_scale, void* stream, void* workspace,
                                 size_t workspace_bytes);
fp4_status_t fp4_attn_fwd_quantized_lse(const fp4_tensor_t* q, const fp4_tensor_t* k,
                                        const fp4_tensor_t* v, void* out, float* lse, int B,
                                        int H, int Hkv, int N, int D, int causal,
                                        float softmax_scale, void* stream);
fp4_status_t fp4_attn_bwd(const void* q, const void* k, const void* v, const void* out,
                          const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                          int H, int Hkv, int N, int D, int causal, float softmax_scale,
                          void* stream, void* workspace, size_t workspace_bytes);

size_t fp4_attn_workspace_bytes_fp8pv(int B, int H, int Hkv, int N, int D);
fp4_status_t fp4_attn_fwd_fp8pv(const void* q, const void* k, const void* v, void* out, int B,
                                int H, int Hkv, int N, int D, int causal, float softmax_scale,
                                void* stream, void* workspace, size_t workspace_bytes);
fp4_status_t fp4_attn_fwd_quantized_fp8pv(const fp4_tensor_t* q, const fp4_tensor_t* k,
                                          const fp4_tensor_t* v, void* out, int B, int H, int Hkv,
                                          int N, int D, int causal, float softmax_scale,
                                          void* stream);

/*
 * fp4_attn_fwd without a caller-supplied workspace, for callers that cannot
 * allocate device memory: code whose device memory is owned by a host
 * framework that hands it no allocator, or code that must not call
 * cudaMalloc because it may synchronise the device. This entry point has no
 * counterpart on the source pages; it only changes where the scratch lives.
 *
 * The scratch is one array of FP4_NOALLOC_SCRATCH_BYTES in this library's
 * device memory, reserved on every GPU that loads the library until the
 * process exits. Problems whose workspace (fp4_attn_workspace_bytes) exceeds
 * it are rejected with FP4_ERR_WORKSPACE and launch nothing. Every call uses
 * the same array: calls whose work overlaps on the GPU (other streams, other
 * host threads, other devices' calls are fine) race on it and must be
 * ordered by the caller. The first call on a device looks up the array's
 * device address and caches it; make that first call before any stream
 * capture. No call allocates or frees memory. Arguments as fp4_attn_fwd.
 */
#define FP4_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
fp4_status_t fp4_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out, int B,
                                  int H, int Hkv, int N, int D, int causal, float softmax_scale,
                                  void* stream);

/*
 * Synchronises the stream, then returns FP4_ERR_BOUNDS if a kernel of an
 * FP4_DEBUG build failed a bounds or alignment check on the current device
 * since the last call (the message names the check's site), else
 * FP4_ERR_TIMEOUT if one reported an expired wait, and clears the report;
 * FP4_ERR_CUDA on a CUDA error; else FP4_OK.
 */
fp4_status_t fp4_status(void* stream);

/* Message of the last failing call on this thread ("" if none). */
const char* fp4_last_error(void);

/*
 * Test support: the hardware conversion applied to the fp32 bit patterns
 * start .. start+count-1, one output byte each: kind 0 = E2M1 code (as the
 * quantiser's cvt produces it), kind 1 = E4M3 byte. out: device, count bytes.
 */
fp4_status_t fp4_probe_cvt(uint32_t start, int64_t count, int kind, uint8_t* out, void* stream);

/*
 * Test support for failure detection: launches one thread that waits, with
 * the same bounded wait the attention kernel uses and a limit of limit_ns
 * (0 < limit_ns <= 5 s), on an mbarrier that nothing arrives on. The wait
 * expires and sets the device error word, so the next fp4_status() returns
 * FP4_ERR_TIMEOUT; *ok (device int) receives 0. Nothing faults or hangs, and
 * the context stays usable. The pages have no counterpart; this exists so
 * the timeout path can be exercised without breaking a real kernel.
 */
fp4_status_t fp4_test_wait_timeout(uint64_t limit_ns, int* ok, void* stream);

/*
 * The debug build. The library built with -DFP4_DEBUG (libfp4attn_debug.so
 * beside the release library, same entry points) checks the index arithmetic
 * of its kernels' guarded global accesses (bulk copies, TMA coordinates and
 * the 16-byte rule for their x, epilogue stores, quantizer writes) against
 * the extent of the buffer each addresses; a failed check records its site
 * number, skips the access and sets the device error word, and fp4_status()
 * returns FP4_ERR_BOUNDS (waits that depended on a skipped copy then expire
 * within their bound). Nothing traps. This is the bounds checker that stands
 * in for compute-sanitizer. fp4_debug_build() returns 1 in that build, else
 * 0. fp4_debug_selftest() launches one thread whose check fails by
 * construction (it addresses no memory), so that the next fp4_status()
 * returns FP4_ERR_BOUNDS with site `site` (1 .. 99); in the release build it
 * launches nothing and returns FP4_ERR_UNSUPPORTED.
 */
int fp4_debug_build(void);
fp4_status_t fp4_debug_selftest(unsigned site, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FP4ATTN_H_ */
