// Host side of the fp4attn C ABI (include/fp4attn.h): argument validation,
// workspace layout, TMA descriptors and kernel launches. No device memory is
// allocated here; every buffer belongs to the caller.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/fp4attn.h"
#include "attn_bwd.cuh"
#include "attn_fwd.cuh"
#include "quantize.cuh"

namespace {

thread_local std::string g_last_error;

fp4_status_t fail(fp4_status_t s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

#define FP4_CUDA(call)                                                                  \
  do {                                                                                  \
    cudaError_t e_ = (call);                                                            \
    if (e_ != cudaSuccess)                                                              \
      return fail(FP4_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_));        \
  } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

constexpr int kMaxDevices = 64;
std::mutex g_mu;
bool g_attr_done[kMaxDevices];
int g_num_sms[kMaxDevices];

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

using AttnKernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap,
                            const CUtensorMap, const fp4::AttnParams);

template <int PG>
AttnKernel attn_kernel_pg(int D, int causal) {
  if (D == 128)
    return causal ? fp4::attn_fwd_kernel<128, true, PG> : fp4::attn_fwd_kernel<128, false, PG>;
  return causal ? fp4::attn_fwd_kernel<64, true, PG> : fp4::attn_fwd_kernel<64, false, PG>;
}

// The fused kernel for head dim D, causal masking and P generation pg
// (fp4::kPgExp, kPgEfq, kPgFp8); bias: with the per-key score correction of
// smoothed Q (exp-then-quantize only).
AttnKernel attn_kernel(int D, int causal, int pg, bool bias = false, bool lse = false) {
  if (lse) {
    if (D == 128)
      return causal ? fp4::attn_fwd_kernel<128, true, fp4::kPgExp, false, true>
                    : fp4::attn_fwd_kernel<128, false, fp4::kPgExp, false, true>;
    return causal ? fp4::attn_fwd_kernel<64, true, fp4::kPgExp, false, true>
                  : fp4::attn_fwd_kernel<64, false, fp4::kPgExp, false, true>;
  }
  if (bias) {
    if (D == 128)
      return causal ? fp4::attn_fwd_kernel<128, true, fp4::kPgExp, true>
                    : fp4::attn_fwd_kernel<128, false, fp4::kPgExp, true>;
    return causal ? fp4::attn_fwd_kernel<64, true, fp4::kPgExp, true>
                  : fp4::attn_fwd_kernel<64, false, fp4::kPgExp, true>;
  }
  if (pg == fp4::kPgEfq) return attn_kernel_pg<fp4::kPgEfq>(D, causal);
  if (pg == fp4::kPgFp8) return attn_kernel_pg<fp4::kPgFp8>(D, causal);
  return attn_kernel_pg<fp4::kPgExp>(D, causal);
}

int attn_smem_bytes(int D, int pg, bool bias = false) {
  if (pg == fp4::kPgFp8) return D == 128 ? fp4::AttnSmem<128, true>::kBytes : fp4::AttnSmem<64, true>::kBytes;
  if (bias)
    return D == 128 ? fp4::AttnSmem<128, false, true>::kBytes : fp4::AttnSmem<64, false, true>::kBytes;
  return D == 128 ? fp4::AttnSmem<128>::kBytes : fp4::AttnSmem<64>::kBytes;
}

using BwdKernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap,
                          const CUtensorMap, const CUtensorMap, const fp4::BwdParams);
using BwdKvKernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap,
                             const CUtensorMap, const CUtensorMap, const CUtensorMap,
                             const fp4::BwdParams);

BwdKernel bwd_dq_kernel_for(int D, int causal) {
  if (D == 128) return causal ? fp4::bwd_dq_kernel<128, true> : fp4::bwd_dq_kernel<128, false>;
  return causal ? fp4::bwd_dq_kernel<64, true> : fp4::bwd_dq_kernel<64, false>;
}
BwdKvKernel bwd_dkdv_kernel_for(int D, int causal) {
  if (D == 128) return causal ? fp4::bwd_dkdv_kernel<128, true> : fp4::bwd_dkdv_kernel<128, false>;
  return causal ? fp4::bwd_dkdv_kernel<64, true> : fp4::bwd_dkdv_kernel<64, false>;
}

// sm_100 check, per-device one-time kernel attributes, SM count.
fp4_status_t device_setup(int* dev_out, int* sms_out) {
  int dev;
  FP4_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return fail(FP4_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_attr_done[dev]) {
    int major = 0, minor = 0, sms = 0;
    FP4_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
    FP4_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
    FP4_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    if (major != 10 || minor != 0)
      return fail(FP4_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a",
                  dev, major, minor);
    for (int d = 0; d < 2; ++d)
      for (int causal = 0; causal < 2; ++causal)
        for (int pg = 0; pg < 5; ++pg)  // 3: with the score correction, 4: writing lse
          FP4_CUDA(cudaFuncSetAttribute(attn_kernel(d ? 128 : 64, causal, pg % 3, pg == 3, pg == 4),
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        attn_smem_bytes(d ? 128 : 64, pg % 3, pg == 3)));
    for (int d = 0; d < 2; ++d)
      for (int causal = 0; causal < 2; ++causal) {
        FP4_CUDA(cudaFuncSetAttribute(bwd_dq_kernel_for(d ? 128 : 64, causal),
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      d ? fp4::BwdDqSmem<128>::kBytes : fp4::BwdDqSmem<64>::kBytes));
        FP4_CUDA(cudaFuncSetAttribute(bwd_dkdv_kernel_for(d ? 128 : 64, causal),
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      d ? fp4::BwdDkvSmem<128>::kBytes : fp4::BwdDkvSmem<64>::kBytes));
      }
    if (!g_encode) {
      cudaDriverEntryPointQueryResult q;
      void* fn = nullptr;
      FP4_CUDA(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
      if (q != cudaDriverEntryPointSuccess || !fn)
        return fail(FP4_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    g_num_sms[dev] = sms;
    g_attr_done[dev] = true;
  }
  *dev_out = dev;
  *sms_out = g_num_sms[dev];
  return FP4_OK;
}

// 2D uint8 tensor map: rows x inner bytes, box rows x box_inner bytes.
fp4_status_t tmap_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                     uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw) {
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FP4_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return FP4_OK;
}

// 2D bf16 tensor map: rows x inner elements, box rows x 64 elements, 128-byte swizzle.
fp4_status_t tmap_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                       uint32_t box_rows) {
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FP4_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return FP4_OK;
}

struct WsLayout {
  size_t amax, qc, qs, kc, ks, vc, vs, sums, qmean, kmean, bias, total;
};

size_t codes_bytes(int64_t G, int64_t N, int64_t D) { return (size_t)(G * round_up(N, 128) * D / 2); }
size_t scales_bytes(int64_t G, int64_t N, int64_t D, fp4_axis_t axis) {
  const int64_t Npad = round_up(N, 128);
  return axis == FP4_BLOCK_ALONG_D ? (size_t)(G * Npad * D / 16) : (size_t)(G * (Npad / 64) * 512);
}

size_t fp8_codes_bytes(int64_t G, int64_t N, int64_t D) { return (size_t)(G * D * round_up(N, 128)); }

// Workspace of the quantizing forwards; fp8v: V as E4M3 codes, no V scales;
// smooth: the smoothing sums, means and Q's score correction as well.
WsLayout ws_layout(int B, int H, int Hkv, int N, int D, bool fp8v = false, bool smooth = false) {
  WsLayout w;
  size_t off = 0;
  auto take = [&](size_t n) {
    size_t o = off;
    off += (size_t)round_up((int64_t)n, 1024);
    return o;
  };
  const int64_t Gq = (int64_t)B * H, Gk = (int64_t)B * Hkv;
  w.amax = take(256);
  w.qc = take(codes_bytes(Gq, N, D));
  w.qs = take(scales_bytes(Gq, N, D, FP4_BLOCK_ALONG_D));
  w.kc = take(codes_bytes(Gk, N, D));
  w.ks = take(scales_bytes(Gk, N, D, FP4_BLOCK_ALONG_D));
  w.vc = take(fp8v ? fp8_codes_bytes(Gk, N, D) : codes_bytes(Gk, N, D));
  w.vs = take(fp8v ? 0 : scales_bytes(Gk, N, D, FP4_BLOCK_ALONG_N_T));
  const int64_t Npad = round_up(N, 128);
  w.sums = take(smooth ? (size_t)((Gq + Gk) * D * 8) : 0);
  w.qmean = take(smooth ? (size_t)(Gq * D * 4) : 0);
  w.kmean = take(smooth ? (size_t)(Gk * D * 4) : 0);
  w.bias = take(smooth ? (size_t)(Gq * Npad * 32) : 0);  // (hi, lo, 0 x 6) per key
  w.total = off;
  return w;
}

// Workspace of the backward: the maxima, the decoded operands (Q^, Q^T, K^,
// K^T, V^), dO padded and transposed, lse padded, D.
struct BwdWs {
  size_t amax, qh, qt, kh, kt, vh, dop, dot, lse, dvec, qc, qs, qs64, kc, ks, total;
};

BwdWs bwd_ws_layout(int B, int H, int Hkv, int N, int D) {
  BwdWs w;
  size_t off = 0;
  auto take = [&](size_t n) {
    size_t o = off;
    off += (size_t)round_up((int64_t)n, 1024);
    return o;
  };
  const int64_t Npad = round_up(N, 128), Gq = (int64_t)B * H, Gk = (int64_t)B * Hkv;
  const size_t q2 = (size_t)(Gq * Npad * D * 2), k2 = (size_t)(Gk * Npad * D * 2);
  w.amax = take(256);
  w.qh = take(q2);
  w.qt = take(q2);
  w.kh = take(k2);
  w.kt = take(k2);
  w.vh = take(k2);
  w.dop = take(q2);
  w.dot = take(q2);
  w.lse = take((size_t)(Gq * Npad * 4));
  w.dvec = take((size_t)(Gq * Npad * 4));
  w.qc = take(codes_bytes(Gq, N, D));
  w.qs = take(scales_bytes(Gq, N, D, FP4_BLOCK_ALONG_D));
  w.qs64 = take(2 * scales_bytes(Gq, N, D, FP4_BLOCK_ALONG_D));
  w.kc = take(codes_bytes(Gk, N, D));
  w.ks = take(scales_bytes(Gk, N, D, FP4_BLOCK_ALONG_D));
  w.total = off;
  return w;
}

fp4_status_t check_shape(int B, int H, int Hkv, int N, int D) {
  if (B < 1 || H < 1 || Hkv < 1 || N < 1)
    return fail(FP4_ERR_INVALID_ARG, "B, H, Hkv and N must be >= 1 (got %d, %d, %d, %d)", B, H,
                Hkv, N);
  if (H % Hkv) return fail(FP4_ERR_INVALID_ARG, "H (%d) must be a multiple of Hkv (%d)", H, Hkv);
  if (D != 64 && D != 128) return fail(FP4_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", D);
  if (B > 65535 || H > 65535) return fail(FP4_ERR_INVALID_ARG, "B and H must be <= 65535");
  const int64_t Npad = round_up(N, 128);
  if ((int64_t)B * H * Npad > INT32_MAX || (int64_t)B * Hkv * D > INT32_MAX ||
      Npad / 128 > INT32_MAX)
    return fail(FP4_ERR_INVALID_ARG, "problem too large");
  return FP4_OK;
}

fp4_status_t launch_amax(const void* x0, int64_t n0, const void* x1, int64_t n1, const void* x2,
                         int64_t n2, float* a0, float* a1, float* a2, int sms,
                         cudaStream_t stream) {
  const int tensors = x2 ? 3 : (x1 ? 2 : 1);
  FP4_CUDA(cudaMemsetAsync(a0, 0, sizeof(float), stream));
  if (x1) FP4_CUDA(cudaMemsetAsync(a1, 0, sizeof(float), stream));
  if (x2) FP4_CUDA(cudaMemsetAsync(a2, 0, sizeof(float), stream));
  dim3 grid(sms * 4, tensors);
  fp4::amax3_kernel<<<grid, 256, 0, stream>>>(
      static_cast<const uint4*>(x0), n0 / 8, static_cast<const uint4*>(x1), n1 / 8,
      static_cast<const uint4*>(x2), n2 / 8, reinterpret_cast<unsigned*>(a0),
      reinterpret_cast<unsigned*>(a1), reinterpret_cast<unsigned*>(a2));
  FP4_CUDA(cudaGetLastError());
  return FP4_OK;
}

fp4_status_t launch_quant(const void* x, int64_t G, int N, int D, fp4_axis_t axis, uint8_t* codes,
                          uint8_t* scales, const float* amax, int sms, cudaStream_t stream,
                          const float* mean = nullptr) {
  const int64_t Npad = round_up(N, 128);
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  if (axis == FP4_BLOCK_ALONG_D) {
    const int64_t total = G * Npad * (D / 16);
    const int64_t blocks = std::min<int64_t>((total + 255) / 256, (int64_t)sms * 16);
    const unsigned nb = (unsigned)blocks;
    if (mean && D == 128)
      fp4::quant_rows_kernel<128, true><<<nb, 256, 0, stream>>>(xb, (int)G, N, (int)Npad, amax,
                                                                codes, scales, mean);
    else if (mean)
      fp4::quant_rows_kernel<64, true><<<nb, 256, 0, stream>>>(xb, (int)G, N, (int)Npad, amax,
                                                               codes, scales, mean);
    else if (D == 128)
      fp4::quant_rows_kernel<128><<<nb, 256, 0, stream>>>(xb, (int)G, N, (int)Npad, amax, codes,
                                                          scales);
    else
      fp4::quant_rows_kernel<64><<<nb, 256, 0, stream>>>(xb, (int)G, N, (int)Npad, amax, codes,
                                                         scales);
  } else {
    const int64_t blocks = G * (Npad / 128);
    if (blocks > INT32_MAX) return fail(FP4_ERR_INVALID_ARG, "problem too large");
    if (D == 128)
      fp4::quant_tokens_T_kernel<128><<<(unsigned)blocks, 128, 0, stream>>>(
          xb, (int)G, N, (int)Npad, amax, codes, scales);
    else
      fp4::quant_tokens_T_kernel<64><<<(unsigned)blocks, 128, 0, stream>>>(
          xb, (int)G, N, (int)Npad, amax, codes, scales);
  }
  FP4_CUDA(cudaGetLastError());
  return FP4_OK;
}

float resolve_scale(float softmax_scale, int D) {
  return (softmax_scale > 0.0f && std::isfinite(softmax_scale)) ? softmax_scale
                                                                 : 1.0f / std::sqrt((float)D);
}

// Smoothing means of x [G][N][D]: sums [G][D] (zeroed here) on the grid of
// *amax, then mean [G][D].
fp4_status_t launch_mean(const void* x, int64_t G, int N, int D, const float* amax,
                         unsigned long long* sums, float* mean, cudaStream_t stream) {
  if (G > 65535) return fail(FP4_ERR_INVALID_ARG, "more than 65535 heads");
  FP4_CUDA(cudaMemsetAsync(sums, 0, (size_t)(G * D * 8), stream));
  dim3 grid((unsigned)((N + fp4::kSumRows - 1) / fp4::kSumRows), (unsigned)G);
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  if (D == 128)
    fp4::colsum_fixed_kernel<128><<<grid, 256, 0, stream>>>(xb, N, amax, sums);
  else
    fp4::colsum_fixed_kernel<64><<<grid, 256, 0, stream>>>(xb, N, amax, sums);
  FP4_CUDA(cudaGetLastError());
  const int64_t n = G * D;
  fp4::mean_from_sums_kernel<<<(unsigned)std::min<int64_t>((n + 255) / 256, 4096), 256, 0, stream>>>(
      sums, n, N, amax, mean);
  FP4_CUDA(cudaGetLastError());
  return FP4_OK;
}

// *out = max |fl32(x - mean)| (zeroed here).
fp4_status_t launch_amax_smoothed(const void* x, int64_t G, int N, int D, const float* mean,
                                  float* out, int sms, cudaStream_t stream) {
  FP4_CUDA(cudaMemsetAsync(out, 0, sizeof(float), stream));
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  if (D == 128)
    fp4::amax_smoothed_kernel<128><<<sms * 4, 256, 0, stream>>>(xb, G, N, mean,
                                                                reinterpret_cast<unsigned*>(out));
  else
    fp4::amax_smoothed_kernel<64><<<sms * 4, 256, 0, stream>>>(xb, G, N, mean,
                                                               reinterpret_cast<unsigned*>(out));
  FP4_CUDA(cudaGetLastError());
  return FP4_OK;
}

// Q's score correction bias [B*H][Npad][8] (hi, lo, 0 ...), with the maxima
// the quantised Q' and K were encoded with.
fp4_status_t launch_score_bias(const float* qmean, const void* k, const float* kmean, int B, int H,
                               int Hkv, int N, int D, const float* amax_q, const float* amax_k,
                               float* bias, cudaStream_t stream) {
  const int64_t Npad = round_up(N, 128);
  if ((int64_t)B * Hkv > 65535) return fail(FP4_ERR_INVALID_ARG, "more than 65535 key/value heads");
  dim3 grid((unsigned)(Npad / 128), (unsigned)(B * Hkv));
  const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(k);
  if (D == 128)
    fp4::score_bias_kernel<128><<<grid, 128, 0, stream>>>(qmean, kb, kmean, H, Hkv, N, (int)Npad,
                                                          amax_q, amax_k, bias);
  else
    fp4::score_bias_kernel<64><<<grid, 128, 0, stream>>>(qmean, kb, kmean, H, Hkv, N, (int)Npad,
                                                         amax_q, amax_k, bias);
  FP4_CUDA(cudaGetLastError());
  return FP4_OK;
}

// V [G][N][D] bf16 -> E4M3 codes [G][D][Npad] with the tensor maximum *amax.
fp4_status_t launch_quant_fp8(const void* x, int64_t G, int N, int D, uint8_t* codes,
                              const float* amax, cudaStream_t stream) {
  const int64_t Npad = round_up(N, 128);
  const int64_t blocks = G * (Npad / 128);
  if (blocks > INT32_MAX) return fail(FP4_ERR_INVALID_ARG, "problem too large");
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  if (D == 128)
    fp4::quant_fp8_tokens_T_kernel<128><<<(unsigned)blocks, 128, 0, stream>>>(xb, (int)G, N,
                                                                              (int)Npad, amax, codes);
  else
    fp4::quant_fp8_tokens_T_kernel<64><<<(unsigned)blocks, 128, 0, stream>>>(xb, (int)G, N,
                                                                             (int)Npad, amax, codes);
  FP4_CUDA(cudaGetLastError());
  return FP4_OK;
}

fp4_status_t launch_attn(const uint8_t* qc, const uint8_t* qs, const float* qa, const uint8_t* kc,
                         const uint8_t* ks, const float* ka, const uint8_t* vc, const uint8_t* vs,
                         const float* va, void* out, int B, int H, int Hkv, int N, int D,
                         int causal, float softmax_scale, int pg, cudaStream_t stream,
                         const float* bias = nullptr, float* lse = nullptr) {
  const int64_t Npad = round_up(N, 128);
  const int64_t Gq = (int64_t)B * H, Gk = (int64_t)B * Hkv;
  const CUtensorMapSwizzle swQK =
      D == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  CUtensorMap tq, tk, tv, tb;
  std::memset(&tb, 0, sizeof(tb));
  fp4_status_t s;
  if ((s = tmap_2d(&tq, qc, D / 2, Gq * Npad, D / 2, 128, swQK)) != FP4_OK) return s;
  // the rank-1 correction: 128 keys x 32 bytes per K tile, 32-byte swizzle
  if (bias && (s = tmap_2d(&tb, bias, 32, Gq * Npad, 32, 128, CU_TENSOR_MAP_SWIZZLE_32B)) != FP4_OK)
    return s;
  if ((s = tmap_2d(&tk, kc, D / 2, Gk * Npad, D / 2, 128, swQK)) != FP4_OK) return s;
  if (pg == fp4::kPgFp8) {  // E4M3 V^T: 128 one-byte keys per row, 128-byte swizzle
    if ((s = tmap_2d(&tv, vc, Npad, Gk * D, 128, D, CU_TENSOR_MAP_SWIZZLE_128B)) != FP4_OK)
      return s;
  } else if ((s = tmap_2d(&tv, vc, Npad / 2, Gk * D, 64, D, CU_TENSOR_MAP_SWIZZLE_64B)) != FP4_OK) {
    return s;
  }
  fp4::AttnParams p;
  p.q_sf = qs;
  p.k_sf = ks;
  p.v_sf = vs;
  p.amax_q = qa;
  p.amax_k = ka;
  p.amax_v = va;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.N = N;
  p.Npad = (int)Npad;
  p.ntq = (int)(Npad / 128);
  p.lse = lse;
  p.softmax_scale = resolve_scale(softmax_scale, D);
  // causal: one linear grid, the longest query tiles of every head first
  if (causal && (int64_t)p.ntq * B * H > INT32_MAX)
    return fail(FP4_ERR_INVALID_ARG, "problem too large");
  const dim3 grid = causal ? dim3((unsigned)((int64_t)p.ntq * B * H)) : dim3(p.ntq, H, B);
  if ((bias || lse) && pg != fp4::kPgExp)
    return fail(FP4_ERR_UNSUPPORTED, "the score correction and lse need exp-then-quantize P");
  if (bias && lse) return fail(FP4_ERR_UNSUPPORTED, "lse with the score correction");
  attn_kernel(D, causal, pg, bias != nullptr, lse != nullptr)<<<
      grid, fp4::kAttnThreads, attn_smem_bytes(D, pg, bias != nullptr), stream>>>(tq, tk, tv, tb, p);
  FP4_CUDA(cudaGetLastError());
  return FP4_OK;
}

fp4_status_t attn_fwd_any(const void* q, const void* k, const void* v, void* out, int B, int H,
                          int Hkv, int N, int D, int causal, float softmax_scale, void* stream,
                          void* workspace, size_t workspace_bytes, int pg, float* lse = nullptr) {
  g_last_error.clear();
  fp4_status_t s;
  if ((s = check_shape(B, H, Hkv, N, D)) != FP4_OK) return s;
  if (!q || !k || !v || !out || !workspace) return fail(FP4_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(workspace))
    return fail(FP4_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const WsLayout w = ws_layout(B, H, Hkv, N, D, pg == fp4::kPgFp8);
  if (workspace_bytes < w.total)
    return fail(FP4_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", workspace_bytes, w.total);
  int dev, sms;
  if ((s = device_setup(&dev, &sms)) != FP4_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* amax = reinterpret_cast<float*>(ws + w.amax);
  const int64_t nq = (int64_t)B * H * N * D, nkv = (int64_t)B * Hkv * N * D;
  if ((s = launch_amax(q, nq, k, nkv, v, nkv, amax, amax + 1, amax + 2, sms, st)) != FP4_OK)
    return s;
  if ((s = launch_quant(q, (int64_t)B * H, N, D, FP4_BLOCK_ALONG_D, ws + w.qc, ws + w.qs, amax,
                        sms, st)) != FP4_OK)
    return s;
  if ((s = launch_quant(k, (int64_t)B * Hkv, N, D, FP4_BLOCK_ALONG_D, ws + w.kc, ws + w.ks,
                        amax + 1, sms, st)) != FP4_OK)
    return s;
  if (pg == fp4::kPgFp8)
    s = launch_quant_fp8(v, (int64_t)B * Hkv, N, D, ws + w.vc, amax + 2, st);
  else
    s = launch_quant(v, (int64_t)B * Hkv, N, D, FP4_BLOCK_ALONG_N_T, ws + w.vc, ws + w.vs,
                     amax + 2, sms, st);
  if (s != FP4_OK) return s;
  return launch_attn(ws + w.qc, ws + w.qs, amax, ws + w.kc, ws + w.ks, amax + 1, ws + w.vc,
                     ws + w.vs, amax + 2, out, B, H, Hkv, N, D, causal, softmax_scale, pg, st,
                     nullptr, lse);
}

// The smoothed forward: smooth bit 0 = K, bit 1 = Q (FP4_SMOOTH_K / _Q).
fp4_status_t attn_fwd_smooth_any(const void* q, const void* k, const void* v, void* out, int B,
                                 int H, int Hkv, int N, int D, int causal, float softmax_scale,
                                 int smooth, void* stream, void* workspace,
                                 size_t workspace_bytes) {
  g_last_error.clear();
  fp4_status_t s;
  if ((s = check_shape(B, H, Hkv, N, D)) != FP4_OK) return s;
  if (smooth & ~3) return fail(FP4_ERR_INVALID_ARG, "smooth flags %d", smooth);
  if (N > (1 << 19)) return fail(FP4_ERR_INVALID_ARG, "smoothing takes N <= 2^19 (got %d)", N);
  if (!q || !k || !v || !out || !workspace) return fail(FP4_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(workspace))
    return fail(FP4_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const WsLayout w = ws_layout(B, H, Hkv, N, D, false, true);
  if (workspace_bytes < w.total)
    return fail(FP4_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", workspace_bytes, w.total);
  int dev, sms;
  if ((s = device_setup(&dev, &sms)) != FP4_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* amax = reinterpret_cast<float*>(ws + w.amax);  // raw Q, K, V; smoothed Q, K
  const int64_t Gq = (int64_t)B * H, Gk = (int64_t)B * Hkv;
  auto* sums = reinterpret_cast<unsigned long long*>(ws + w.sums);
  float* qmean = reinterpret_cast<float*>(ws + w.qmean);
  float* kmean = reinterpret_cast<float*>(ws + w.kmean);
  float* bias = reinterpret_cast<float*>(ws + w.bias);
  if ((s = launch_amax(q, Gq * N * D, k, Gk * N * D, v, Gk * N * D, amax, amax + 1, amax + 2, sms,
                       st)) != FP4_OK)
    return s;
  const float* ak = amax + 1;
  const float* kmean_used = nullptr;
  if (smooth & 1) {
    if ((s = launch_mean(k, Gk, N, D, amax + 1, sums + Gq * D, kmean, st)) != FP4_OK) return s;
    if ((s = launch_amax_smoothed(k, Gk, N, D, kmean, amax + 4, sms, st)) != FP4_OK) return s;
    ak = amax + 4;
    kmean_used = kmean;
  }
  if ((s = launch_quant(k, Gk, N, D, FP4_BLOCK_ALONG_D, ws + w.kc, ws + w.ks, ak, sms, st,
                        kmean_used)) != FP4_OK)
    return s;
  const float* aq = amax;
  const float* qmean_used = nullptr;
  if (smooth & 2) {
    if ((s = launch_mean(q, Gq, N, D, amax, sums, qmean, st)) != FP4_OK) return s;
    if ((s = launch_amax_smoothed(q, Gq, N, D, qmean, amax + 3, sms, st)) != FP4_OK) return s;
    if ((s = launch_score_bias(qmean, k, kmean_used, B, H, Hkv, N, D, amax + 3, ak, bias, st)) !=
        FP4_OK)
      return s;
    aq = amax + 3;
    qmean_used = qmean;
  }
  if ((s = launch_quant(q, Gq, N, D, FP4_BLOCK_ALONG_D, ws + w.qc, ws + w.qs, aq, sms, st,
                        qmean_used)) != FP4_OK)
    return s;
  if ((s = launch_quant(v, Gk, N, D, FP4_BLOCK_ALONG_N_T, ws + w.vc, ws + w.vs, amax + 2, sms,
                        st)) != FP4_OK)
    return s;
  return launch_attn(ws + w.qc, ws + w.qs, aq, ws + w.kc, ws + w.ks, ak, ws + w.vc, ws + w.vs,
                     amax + 2, out, B, H, Hkv, N, D, causal, softmax_scale, fp4::kPgExp, st,
                     (smooth & 2) ? bias : nullptr);
}

// The backward (attn_bwd.cuh): pre-kernels, then the dq kernel (D and dQ),
// then the dk/dv kernel.
// amax_in: the three tensor maxima (Q, K, V) to quantise with, e.g. combined
// over shards, or NULL to compute them from q, k, v.
fp4_status_t attn_bwd_any(const void* q, const void* k, const void* v, const void* out,
                          const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                          int H, int Hkv, int N, int D, int causal, float softmax_scale, void* stream,
                          void* workspace, size_t workspace_bytes,
                          const float* amax_in = nullptr) {
  g_last_error.clear();
  fp4_status_t s;
  if ((s = check_shape(B, H, Hkv, N, D)) != FP4_OK) return s;
  if (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv || !workspace)
    return fail(FP4_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) ||
      !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || !aligned16(workspace) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return fail(FP4_ERR_INVALID_ARG, "pointers must be 16-byte aligned (lse 4-byte)");
  const BwdWs w = bwd_ws_layout(B, H, Hkv, N, D);
  if (workspace_bytes < w.total)
    return fail(FP4_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", workspace_bytes, w.total);
  if (amax_in && (reinterpret_cast<uintptr_t>(amax_in) & 3u))
    return fail(FP4_ERR_INVALID_ARG, "amax must be 4-byte aligned");
  int dev, sms;
  if ((s = device_setup(&dev, &sms)) != FP4_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* amax = reinterpret_cast<float*>(ws + w.amax);
  const int64_t Npad = round_up(N, 128), Gq = (int64_t)B * H, Gk = (int64_t)B * Hkv;
  if (amax_in) {
    FP4_CUDA(cudaMemcpyAsync(amax, amax_in, 3 * sizeof(float), cudaMemcpyDeviceToDevice, st));
  } else if ((s = launch_amax(q, Gq * N * D, k, Gk * N * D, v, Gk * N * D, amax, amax + 1,
                              amax + 2, sms, st)) != FP4_OK) {
    return s;
  }
  auto* qh = reinterpret_cast<__nv_bfloat16*>(ws + w.qh);
  auto* qt = reinterpret_cast<__nv_bfloat16*>(ws + w.qt);
  auto* kh = reinterpret_cast<__nv_bfloat16*>(ws + w.kh);
  auto* kt = reinterpret_cast<__nv_bfloat16*>(ws + w.kt);
  auto* vh = reinterpret_cast<__nv_bfloat16*>(ws + w.vh);
  auto* dop = reinterpret_cast<__nv_bfloat16*>(ws + w.dop);
  auto* dot = reinterpret_cast<__nv_bfloat16*>(ws + w.dot);
  float* lsep = reinterpret_cast<float*>(ws + w.lse);
  float* dvec = reinterpret_cast<float*>(ws + w.dvec);
  const auto* qb = static_cast<const __nv_bfloat16*>(q);
  const auto* kb = static_cast<const __nv_bfloat16*>(k);
  const auto* vb = static_cast<const __nv_bfloat16*>(v);
  const auto* ob = static_cast<const __nv_bfloat16*>(dout);
  const unsigned tq = (unsigned)(Gq * (Npad / 128)), tk = (unsigned)(Gk * (Npad / 128));
  if (D == 128) {
    fp4::fq_rows_kernel<128><<<tq, 128, 0, st>>>(qb, N, (int)Npad, amax, qh, qt);
    fp4::fq_rows_kernel<128><<<tk, 128, 0, st>>>(kb, N, (int)Npad, amax + 1, kh, kt);
    fp4::fq_tokens_kernel<128><<<tk, 128, 0, st>>>(vb, N, (int)Npad, amax + 2, vh);
    fp4::pad_transpose_kernel<128><<<tq, 128, 0, st>>>(ob, N, (int)Npad, dop, dot);
  } else {
    fp4::fq_rows_kernel<64><<<tq, 128, 0, st>>>(qb, N, (int)Npad, amax, qh, qt);
    fp4::fq_rows_kernel<64><<<tk, 128, 0, st>>>(kb, N, (int)Npad, amax + 1, kh, kt);
    fp4::fq_tokens_kernel<64><<<tk, 128, 0, st>>>(vb, N, (int)Npad, amax + 2, vh);
    fp4::pad_transpose_kernel<64><<<tq, 128, 0, st>>>(ob, N, (int)Npad, dop, dot);
  }
  FP4_CUDA(cudaGetLastError());
  // Q's and K's NVFP4 codes and block scales (the forward's quantiser) for S^T,
  // Q's scales regrouped per 64-query tile
  if ((s = launch_quant(q, Gq, N, D, FP4_BLOCK_ALONG_D, ws + w.qc, ws + w.qs, amax, sms, st)) !=
      FP4_OK)
    return s;
  if ((s = launch_quant(k, Gk, N, D, FP4_BLOCK_ALONG_D, ws + w.kc, ws + w.ks, amax + 1, sms,
                        st)) != FP4_OK)
    return s;
  {
    const int64_t n16 = (int64_t)scales_bytes(Gq, N, D, FP4_BLOCK_ALONG_D) / 16;
    fp4::sf64_kernel<<<(unsigned)std::min<int64_t>((n16 + 255) / 256, (int64_t)sms * 8), 256, 0,
                       st>>>(reinterpret_cast<const uint4*>(ws + w.qs), n16, D / 64 * 32,
                             reinterpret_cast<uint4*>(ws + w.qs64));
    FP4_CUDA(cudaGetLastError());
  }
  fp4::lse_pad_kernel<<<(unsigned)std::min<int64_t>((Gq * Npad + 255) / 256, (int64_t)sms * 8), 256,
                        0, st>>>(lse, Gq, N, (int)Npad, lsep);
  FP4_CUDA(cudaGetLastError());
  CUtensorMap mQ, mDO, mK64, mV64, mKT, mKc, mV128, mQc, mDO64, mQT, mDOT;
  const CUtensorMapSwizzle swQK = D == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  if ((s = tmap_bf16(&mQ, qh, D, Gq * Npad, fp4::kBwdQ)) != FP4_OK) return s;
  if ((s = tmap_bf16(&mDO, dop, D, Gq * Npad, fp4::kBwdQ)) != FP4_OK) return s;
  if ((s = tmap_bf16(&mK64, kh, D, Gk * Npad, fp4::kBwdKt)) != FP4_OK) return s;
  if ((s = tmap_bf16(&mV64, vh, D, Gk * Npad, fp4::kBwdKt)) != FP4_OK) return s;
  if ((s = tmap_bf16(&mKT, kt, Npad, Gk * D, D)) != FP4_OK) return s;
  if ((s = tmap_2d(&mKc, ws + w.kc, D / 2, Gk * Npad, D / 2, fp4::kBwdK, swQK)) != FP4_OK)
    return s;
  if ((s = tmap_bf16(&mV128, vh, D, Gk * Npad, fp4::kBwdK)) != FP4_OK) return s;
  if ((s = tmap_2d(&mQc, ws + w.qc, D / 2, Gq * Npad, D / 2, fp4::kBwdQt, swQK)) != FP4_OK)
    return s;
  if ((s = tmap_bf16(&mDO64, dop, D, Gq * Npad, fp4::kBwdQt)) != FP4_OK) return s;
  if ((s = tmap_bf16(&mQT, qt, Npad, Gq * D, D)) != FP4_OK) return s;
  if ((s = tmap_bf16(&mDOT, dot, Npad, Gq * D, D)) != FP4_OK) return s;
  fp4::BwdParams p;
  p.amax = amax;
  p.lse = lsep;
  p.Dvec = dvec;
  p.out = static_cast<const __nv_bfloat16*>(out);
  p.k_sf = ws + w.ks;
  p.q_sf64 = ws + w.qs64;
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.H = H;
  p.Hkv = Hkv;
  p.N = N;
  p.Npad = (int)Npad;
  p.softmax_scale = resolve_scale(softmax_scale, D);
  dim3 g1((unsigned)(Npad / fp4::kBwdQ), (unsigned)H, (unsigned)B);
  bwd_dq_kernel_for(D, causal)<<<g1, fp4::kDqThreads,
                                 D == 128 ? fp4::BwdDqSmem<128>::kBytes : fp4::BwdDqSmem<64>::kBytes,
                                 st>>>(mQ, mDO, mK64, mV64, mKT, p);
  FP4_CUDA(cudaGetLastError());
  dim3 g2((unsigned)(Npad / fp4::kBwdK), (unsigned)Hkv, (unsigned)B);
  bwd_dkdv_kernel_for(D, causal)<<<g2, fp4::kBwdThreads,
                                   D == 128 ? fp4::BwdDkvSmem<128>::kBytes
                                            : fp4::BwdDkvSmem<64>::kBytes,
                                   st>>>(mKc, mV128, mQc, mDO64, mQT, mDOT, p);
  FP4_CUDA(cudaGetLastError());
  return FP4_OK;
}

fp4_status_t attn_fwd_quantized_any(const fp4_tensor_t* q, const fp4_tensor_t* k,
                                    const fp4_tensor_t* v, void* out, int B, int H, int Hkv,
                                    int N, int D, int causal, float softmax_scale, void* stream,
                                    int pg, const float* bias = nullptr, float* lse = nullptr) {
  g_last_error.clear();
  fp4_status_t s;
  if ((s = check_shape(B, H, Hkv, N, D)) != FP4_OK) return s;
  if (!q || !k || !v || !out) return fail(FP4_ERR_INVALID_ARG, "null pointer");
  const fp4_tensor_t* t[3] = {q, k, v};
  for (int i = 0; i < 3; ++i) {
    const fp4_tensor_t* x = t[i];
    const bool no_scales = i == 2 && pg == fp4::kPgFp8;  // E4M3 V has no block scales
    if (!x->codes || (!x->scales && !no_scales) || !x->amax)
      return fail(FP4_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(x->codes) || (!no_scales && !aligned16(x->scales)) ||
        (reinterpret_cast<uintptr_t>(x->amax) & 3u))
      return fail(FP4_ERR_INVALID_ARG, "codes/scales must be 16-byte aligned");
  }
  if (!aligned16(out)) return fail(FP4_ERR_INVALID_ARG, "out must be 16-byte aligned");
  if (bias && !aligned16(bias)) return fail(FP4_ERR_INVALID_ARG, "bias must be 16-byte aligned");
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u))
    return fail(FP4_ERR_INVALID_ARG, "lse must be 4-byte aligned");
  int dev, sms;
  if ((s = device_setup(&dev, &sms)) != FP4_OK) return s;
  return launch_attn(q->codes, q->scales, q->amax, k->codes, k->scales, k->amax, v->codes,
                     v->scales, v->amax, out, B, H, Hkv, N, D, causal, softmax_scale, pg,
                     static_cast<cudaStream_t>(stream), bias, lse);
}

}  // namespace

extern "C" {

size_t fp4_codes_bytes(int G, int N, int D, fp4_axis_t) {
  if (G < 1 || N < 1 || D < 16) return 0;
  return codes_bytes(G, N, D);
}

size_t fp4_scales_bytes(int G, int N, int D, fp4_axis_t axis) {
  if (G < 1 || N < 1 || D < 16) return 0;
  return scales_bytes(G, N, D, axis);
}

size_t fp4_attn_workspace_bytes(int B, int H, int Hkv, int N, int D) {
  if (check_shape(B, H, Hkv, N, D) != FP4_OK) return 0;
  return ws_layout(B, H, Hkv, N, D).total;
}

size_t fp4_attn_bwd_workspace_bytes(int B, int H, int Hkv, int N, int D) {
  if (check_shape(B, H, Hkv, N, D) != FP4_OK) return 0;
  return bwd_ws_layout(B, H, Hkv, N, D).total;
}

fp4_status_t fp4_attn_bwd(const void* q, const void* k, const void* v, const void* out,
                          const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                          int H, int Hkv, int N, int D, int causal, float softmax_scale,
                          void* stream, void* workspace, size_t workspace_bytes) {
  return attn_bwd_any(q, k, v, out, dout, lse, dq, dk, dv, B, H, Hkv, N, D, causal,
                      softmax_scale, stream, workspace, workspace_bytes);
}

fp4_status_t fp4_attn_bwd_scaled(const void* q, const void* k, const void* v, const void* out,
                                 const void* dout, const float* lse, const float* amax, void* dq,
                                 void* dk, void* dv, int B, int H, int Hkv, int N, int D,
                                 int causal, float softmax_scale, void* stream, void* workspace,
                                 size_t workspace_bytes) {
  if (!amax) {
    g_last_error.clear();
    return fail(FP4_ERR_INVALID_ARG, "null pointer");
  }
  return attn_bwd_any(q, k, v, out, dout, lse, dq, dk, dv, B, H, Hkv, N, D, causal,
                      softmax_scale, stream, workspace, workspace_bytes, amax);
}

fp4_status_t fp4_attn_fwd_quantized_lse(const fp4_tensor_t* q, const fp4_tensor_t* k,
                                        const fp4_tensor_t* v, void* out, float* lse, int B,
                                        int H, int Hkv, int N, int D, int causal,
                                        float softmax_scale, void* stream) {
  if (!lse) {
    g_last_error.clear();
    return fail(FP4_ERR_INVALID_ARG, "null pointer");
  }
  return attn_fwd_quantized_any(q, k, v, out, B, H, Hkv, N, D, causal, softmax_scale, stream, 0,
                                nullptr, lse);
}

fp4_status_t fp4_attn_fwd_lse(const void* q, const void* k, const void* v, void* out, float* lse,
                              int B, int H, int Hkv, int N, int D, int causal,
                              float softmax_scale, void* stream, void* workspace,
                              size_t workspace_bytes) {
  if (!lse || (reinterpret_cast<uintptr_t>(lse) & 3u)) {
    g_last_error.clear();
    return fail(FP4_ERR_INVALID_ARG, "lse must be a 4-byte aligned device pointer");
  }
  return attn_fwd_any(q, k, v, out, B, H, Hkv, N, D, causal, softmax_scale, stream, workspace,
                      workspace_bytes, 0, lse);
}

size_t fp4_attn_workspace_bytes_smooth(int B, int H, int Hkv, int N, int D) {
  if (check_shape(B, H, Hkv, N, D) != FP4_OK || N > (1 << 19)) return 0;
  return ws_layout(B, H, Hkv, N, D, false, true).total;
}

fp4_status_t fp4_channel_mean(const void* x, int G, int N, int D, const float* amax,
                              float* mean, unsigned long long* sums, void* stream) {
  g_last_error.clear();
  fp4_status_t s;
  if ((s = check_shape(1, G, G, N, D)) != FP4_OK) return s;
  if (N > (1 << 19)) return fail(FP4_ERR_INVALID_ARG, "N <= 2^19 (got %d)", N);
  if (!x || !amax || !mean || !sums) return fail(FP4_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(x) || !aligned16(mean) || !aligned16(sums) ||
      (reinterpret_cast<uintptr_t>(amax) & 3u))
    return fail(FP4_ERR_INVALID_ARG, "x, mean and sums 16-byte aligned, amax 4-byte aligned");
  int dev, sms;
  if ((s = device_setup(&dev, &sms)) != FP4_OK) return s;
  return launch_mean(x, G, N, D, amax, sums, mean, static_cast<cudaStream_t>(stream));
}

fp4_status_t fp4_amax_smoothed(const void* x, int G, int N, int D, const float* mean, float* amax,
                               void* stream) {
  g_last_error.clear();
  fp4_status_t s;
  if ((s = check_shape(1, G, G, N, D)) != FP4_OK) return s;
  if (!x || !mean || !amax) return fail(FP4_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(x) || !aligned16(mean) || (reinterpret_cast<uintptr_t>(amax) & 3u))
    return fail(FP4_ERR_INVALID_ARG, "x and mean 16-byte aligned, amax 4-byte aligned");
  int dev, sms;
  if ((s = device_setup(&dev, &sms)) != FP4_OK) return s;
  return launch_amax_smoothed(x, G, N, D, mean, amax, sms, static_cast<cudaStream_t>(stream));
}

fp4_status_t fp4_quantize_smoothed(const void* x, int G, int N, int D, const float* mean,
                                   const float* amax, uint8_t* codes, uint8_t* scales,
                                   void* stream) {
  g_last_error.clear();
  fp4_status_t s;
  if ((s = check_shape(1, G, G, N, D)) != FP4_OK) return s;
  if (!x || !mean || !amax || !codes || !scales) return fail(FP4_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(x) || !aligned16(mean) || !aligned16(codes) || !aligned16(scales) ||
      (reinterpret_cast<uintptr_t>(amax) & 3u))
    return fail(FP4_ERR_INVALID_ARG,
                "x, mean, codes and scales 16-byte aligned, amax 4-byte aligned");
  int dev, sms;
  if ((s = device_setup(&dev, &sms)) != FP4_OK) return s;
  return launch_quant(x, G, N, D, FP4_BLOCK_ALONG_D, codes, scales, amax, sms,
                      static_cast<cudaStream_t>(stream), mean);
}

fp4_status_t fp4_score_bias(const float* qmean, const void* k, const float* kmean, int B, int H,
                            int Hkv, int N, int D, const float* q_amax, const float* k_amax,
                            float* bias, void* stream) {
  g_last_error.clear();
  fp4_status_t s;
  if ((s = check_shape(B, H, Hkv, N, D)) != FP4_OK) return s;
  if (!qmean || !k || !bias || !q_amax || !k_amax) return fail(FP4_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(qmean) || !aligned16(k) || !aligned16(bias) || (kmean && !aligned16(kmean)) ||
      (reinterpret_cast<uintptr_t>(q_amax) & 3u) || (reinterpret_cast<uintptr_t>(k_amax) & 3u))
    return fail(FP4_ERR_INVALID_ARG, "pointers must be 16-byte aligned (maxima 4-byte)");
  int dev, sms;
  if ((s = device_setup(&dev, &sms)) != FP4_OK) return s;
  return launch_score_bias(qmean, k, kmean, B, H, Hkv, N, D, q_amax, k_amax, bias,
                           static_cast<cudaStream_t>(stream));
}

fp4_status_t fp4_attn_fwd_smooth(const void* q, const void* k, const void* v, void* out, int B,
                                 int H, int Hkv, int N, int D, int causal, float softmax_scale,
                                 int smooth, void* stream, void* workspace,
                                 size_t workspace_bytes) {
  return attn_fwd_smooth_any(q, k, v, out, B, H, Hkv, N, D, causal, softmax_scale, smooth, stream,
                             workspace, workspace_bytes);
}

fp4_status_t fp4_attn_fwd_quantized_bias(const fp4_tensor_t* q, const fp4_tensor_t* k,
                                         const fp4_tensor_t* v, const float* bias, void* out,
                                         int B, int H, int Hkv, int N, int D, int causal,
                                         float softmax_scale, void* stream) {
  if (!bias) {
    g_last_error.clear();
    return fail(FP4_ERR_INVALID_ARG, "null pointer");
  }
  return attn_fwd_quantized_any(q, k, v, out, B, H, Hkv, N, D, causal, softmax_scale, stream, 0,
                                bias);
}

size_t fp4_attn_workspace_bytes_fp8pv(int B, int H, int Hkv, int N, int D) {
  if (check_shape(B, H, Hkv, N, D) != FP4_OK) return 0;
  return ws_layout(B, H, Hkv, N, D, true).total;
}

size_t fp4_fp8_codes_bytes(int G, int N, int D) {
  if (G < 1 || N < 1 || D < 16) return 0;
  return fp8_codes_bytes(G, N, D);
}

fp4_status_t fp4_quantize_fp8(const void* x, int G, int N, int D, uint8_t* codes, float* amax,
                              void* stream) {
  g_last_error.clear();
  fp4_status_t s;
  if ((s = check_shape(1, G, G, N, D)) != FP4_OK) return s;
  if (!x || !codes || !amax) return fail(FP4_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(x) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(amax) & 3u))
    return fail(FP4_ERR_INVALID_ARG, "x and codes must be 16-byte aligned, amax 4-byte aligned");
  int dev, sms;
  if ((s = device_setup(&dev, &sms)) != FP4_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = launch_amax(x, (int64_t)G * N * D, nullptr, 0, nullptr, 0, amax, nullptr, nullptr, sms,
                       st)) != FP4_OK)
    return s;
  return launch_quant_fp8(x, G, N, D, codes, amax, st);
}

fp4_status_t fp4_quantize_fp8_scaled(const void* x, int G, int N, int D, const float* amax,
                                     uint8_t* codes, void* stream) {
  g_last_error.clear();
  fp4_status_t s;
  if ((s = check_shape(1, G, G, N, D)) != FP4_OK) return s;
  if (!x || !codes || !amax) return fail(FP4_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(x) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(amax) & 3u))
    return fail(FP4_ERR_INVALID_ARG, "x and codes must be 16-byte aligned, amax 4-byte aligned");
  int dev, sms;
  if ((s = device_setup(&dev, &sms)) != FP4_OK) return s;
  return launch_quant_fp8(x, G, N, D, codes, amax, static_cast<cudaStream_t>(stream));
}

fp4_status_t fp4_quantize(const void* x, int G, int N, int D, fp4_axis_t axis, uint8_t* codes,
                          uint8_t* scales, float* amax, void* stream) {
  g_last_error.clear();
  fp4_status_t s;
  if ((s = check_shape(1, G, G, N, D)) != FP4_OK) return s;
  if (axis != FP4_BLOCK_ALONG_D && axis != FP4_BLOCK_ALONG_N_T)
    return fail(FP4_ERR_INVALID_ARG, "axis %d", (int)axis);
  if (!x || !codes || !scales || !amax) return fail(FP4_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || !aligned16(amax))
    return fail(FP4_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  int dev, sms;
  if ((s = device_setup(&dev, &sms)) != FP4_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t n = (int64_t)G * N * D;
  if ((s = launch_amax(x, n, nullptr, 0, nullptr, 0, amax, nullptr, nullptr, sms, st)) != FP4_OK)
    return s;
  return launch_quant(x, G, N, D, axis, codes, scales, amax, sms, st);
}

fp4_status_t fp4_amax(const void* x, int G, int N, int D, float* amax, void* stream) {
  g_last_error.clear();
  fp4_status_t s;
  if ((s = check_shape(1, G, G, N, D)) != FP4_OK) return s;
  if (!x || !amax) return fail(FP4_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(amax) & 3u))
    return fail(FP4_ERR_INVALID_ARG, "x must be 16-byte and amax 4-byte aligned");
  int dev, sms;
  if ((s = device_setup(&dev, &sms)) != FP4_OK) return s;
  return launch_amax(x, (int64_t)G * N * D, nullptr, 0, nullptr, 0, amax, nullptr, nullptr, sms,
                     static_cast<cudaStream_t>(stream));
}

fp4_status_t fp4_quantize_scaled(const void* x, int G, int N, int D, fp4_axis_t axis,
                                 const float* amax, uint8_t* codes, uint8_t* scales,
                                 void* stream) {
  g_last_error.clear();
  fp4_status_t s;
  if ((s = check_shape(1, G, G, N, D)) != FP4_OK) return s;
  if (axis != FP4_BLOCK_ALONG_D && axis != FP4_BLOCK_ALONG_N_T)
    return fail(FP4_ERR_INVALID_ARG, "axis %d", (int)axis);
  if (!x || !codes || !scales || !amax) return fail(FP4_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) ||
      (reinterpret_cast<uintptr_t>(amax) & 3u))
    return fail(FP4_ERR_INVALID_ARG,
                "x, codes and scales must be 16-byte aligned, amax 4-byte aligned");
  int dev, sms;
  if ((s = device_setup(&dev, &sms)) != FP4_OK) return s;
  return launch_quant(x, G, N, D, axis, codes, scales, amax, sms,
                      static_cast<cudaStream_t>(stream));
}

fp4_status_t fp4_attn_fwd(const void* q, const void* k, const void* v, void* out, int B, int H,
                          int Hkv, int N, int D, int causal, float softmax_scale, void* stream,
                          void* workspace, size_t workspace_bytes) {
  return attn_fwd_any(q, k, v, out, B, H, Hkv, N, D, causal, softmax_scale, stream, workspace,
                      workspace_bytes, 0);
}

size_t fp4_attn_host_workspace_bytes(int B, int H, int Hkv, int N, int D) {
  if (check_shape(B, H, Hkv, N, D) != FP4_OK) return 0;
  const size_t nq = (size_t)B * H * N * D * 2, nkv = (size_t)B * Hkv * N * D * 2;
  return 2 * (size_t)round_up((int64_t)nq, 1024) + 2 * (size_t)round_up((int64_t)nkv, 1024) +
         ws_layout(B, H, Hkv, N, D).total;
}

fp4_status_t fp4_attn_fwd_host(const void* q_host, const void* k_host, const void* v_host,
                               void* out_host, int B, int H, int Hkv, int N, int D, int causal,
                               float softmax_scale, void* stream, void* dev_workspace,
                               size_t dev_workspace_bytes) {
  g_last_error.clear();
  fp4_status_t s;
  if ((s = check_shape(B, H, Hkv, N, D)) != FP4_OK) return s;
  if (!q_host || !k_host || !v_host || !out_host || !dev_workspace)
    return fail(FP4_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(dev_workspace))
    return fail(FP4_ERR_INVALID_ARG, "the device workspace must be 16-byte aligned");
  const size_t need = fp4_attn_host_workspace_bytes(B, H, Hkv, N, D);
  if (dev_workspace_bytes < need)
    return fail(FP4_ERR_WORKSPACE, "device workspace of %zu bytes, %zu needed",
                dev_workspace_bytes, need);
  const size_t nq = (size_t)B * H * N * D * 2, nkv = (size_t)B * Hkv * N * D * 2;
  const size_t aq = (size_t)round_up((int64_t)nq, 1024), akv = (size_t)round_up((int64_t)nkv, 1024);
  uint8_t* base = static_cast<uint8_t*>(dev_workspace);
  uint8_t *dq = base, *dk = dq + aq, *dv = dk + akv, *dout = dv + akv, *ws = dout + aq;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  FP4_CUDA(cudaMemcpyAsync(dq, q_host, nq, cudaMemcpyHostToDevice, st));
  FP4_CUDA(cudaMemcpyAsync(dk, k_host, nkv, cudaMemcpyHostToDevice, st));
  FP4_CUDA(cudaMemcpyAsync(dv, v_host, nkv, cudaMemcpyHostToDevice, st));
  if ((s = fp4_attn_fwd(dq, dk, dv, dout, B, H, Hkv, N, D, causal, softmax_scale, stream, ws,
                        dev_workspace_bytes - (size_t)(ws - base))) != FP4_OK)
    return s;
  FP4_CUDA(cudaMemcpyAsync(out_host, dout, nq, cudaMemcpyDeviceToHost, st));
  FP4_CUDA(cudaStreamSynchronize(st));
  return FP4_OK;
}

fp4_status_t fp4_attn_fwd_efq(const void* q, const void* k, const void* v, void* out, int B,
                              int H, int Hkv, int N, int D, int causal, float softmax_scale,
                              void* stream, void* workspace, size_t workspace_bytes) {
  return attn_fwd_any(q, k, v, out, B, H, Hkv, N, D, causal, softmax_scale, stream, workspace,
                      workspace_bytes, 1);
}

fp4_status_t fp4_attn_fwd_quantized(const fp4_tensor_t* q, const fp4_tensor_t* k,
                                    const fp4_tensor_t* v, void* out, int B, int H, int Hkv,
                                    int N, int D, int causal, float softmax_scale, void* stream) {
  return attn_fwd_quantized_any(q, k, v, out, B, H, Hkv, N, D, causal, softmax_scale, stream, 0);
}

fp4_status_t fp4_attn_fwd_quantized_efq(const fp4_tensor_t* q, const fp4_tensor_t* k,
                                        const fp4_tensor_t* v, void* out, int B, int H, int Hkv,
                                        int N, int D, int causal, float softmax_scale,
                                        void* stream) {
  return attn_fwd_quantized_any(q, k, v, out, B, H, Hkv, N, D, causal, softmax_scale, stream, 1);
}

fp4_status_t fp4_attn_fwd_fp8pv(const void* q, const void* k, const void* v, void* out, int B,
                                int H, int Hkv, int N, int D, int causal, float softmax_scale,
                                void* stream, void* workspace, size_t workspace_bytes) {
  return attn_fwd_any(q, k, v, out, B, H, Hkv, N, D, causal, softmax_scale, stream, workspace,
                      workspace_bytes, 2);
}

fp4_status_t fp4_attn_fwd_quantized_fp8pv(const fp4_tensor_t* q, const fp4_tensor_t* k,
                                          const fp4_tensor_t* v, void* out, int B, int H, int Hkv,
                                          int N, int D, int causal, float softmax_scale,
                                          void* stream) {
  return attn_fwd_quantized_any(q, k, v, out, B, H, Hkv, N, D, causal, softmax_scale, stream, 2);
}



// Scratch for fp4_attn_fwd_noalloc: reserved in every GPU's copy of this
// module; its device address is looked up once per device.
static __device__ __align__(256) uint8_t g_fp4_noalloc_scratch[FP4_NOALLOC_SCRATCH_BYTES];
static void* g_noalloc_ptr[kMaxDevices];

fp4_status_t fp4_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out, int B,
                                  int H, int Hkv, int N, int D, int causal, float softmax_scale,
                                  void* stream) {
  g_last_error.clear();
  fp4_status_t s;
  if ((s = check_shape(B, H, Hkv, N, D)) != FP4_OK) return s;
  const size_t need = ws_layout(B, H, Hkv, N, D).total;
  if (need > FP4_NOALLOC_SCRATCH_BYTES)
    return fail(FP4_ERR_WORKSPACE,
                "this problem needs %zu bytes of scratch; the built-in scratch of "
                "fp4_attn_fwd_noalloc holds %zu (use fp4_attn_fwd with a workspace)",
                need, (size_t)FP4_NOALLOC_SCRATCH_BYTES);
  int dev, sms;
  if ((s = device_setup(&dev, &sms)) != FP4_OK) return s;
  void* scratch;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_noalloc_ptr[dev]) {
      void* ptr = nullptr;
      cudaError_t e = cudaGetSymbolAddress(&ptr, g_fp4_noalloc_scratch);
      if (e != cudaSuccess || !ptr)
        return fail(FP4_ERR_CUDA, "cudaGetSymbolAddress of the scratch failed: %s",
                    cudaGetErrorString(e));
      g_noalloc_ptr[dev] = ptr;
    }
    scratch = g_noalloc_ptr[dev];
  }
  return fp4_attn_fwd(q, k, v, out, B, H, Hkv, N, D, causal, softmax_scale, stream, scratch,
                      FP4_NOALLOC_SCRATCH_BYTES);
}

fp4_status_t fp4_status(void* stream) {
  FP4_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  FP4_CUDA(cudaGetLastError());
  unsigned err = 0;
  FP4_CUDA(cudaMemcpyFromSymbol(&err, fp4::g_fp4_err, sizeof(err)));
  if (err) {
    const unsigned zero = 0;
    unsigned site = 0;
    FP4_CUDA(cudaMemcpyFromSymbol(&site, fp4::g_fp4_dbg_site, sizeof(site)));
    FP4_CUDA(cudaMemcpyToSymbol(fp4::g_fp4_err, &zero, sizeof(zero)));
    FP4_CUDA(cudaMemcpyToSymbol(fp4::g_fp4_dbg_site, &zero, sizeof(zero)));
    if (err & fp4::kDevErrBounds)
      return fail(FP4_ERR_BOUNDS, "a bounds or alignment check failed at site %u (error word %u)",
                  site, err);
    return fail(FP4_ERR_TIMEOUT, "a kernel's bounded wait expired (device error word %u)", err);
  }
  return FP4_OK;
}

const char* fp4_last_error(void) { return g_last_error.c_str(); }

fp4_status_t fp4_probe_cvt(uint32_t start, int64_t count, int kind, uint8_t* out, void* stream) {
  g_last_error.clear();
  if (count < 0 || (kind != 0 && kind != 1) || (count > 0 && !out))
    return fail(FP4_ERR_INVALID_ARG, "bad probe arguments");
  if ((int64_t)start + count > (int64_t)1 << 32)
    return fail(FP4_ERR_INVALID_ARG, "range beyond 2^32");
  int dev, sms;
  fp4_status_t s;
  if ((s = device_setup(&dev, &sms)) != FP4_OK) return s;
  if (count == 0) return FP4_OK;
  fp4::probe_cvt_kernel<<<sms * 8, 256, 0, static_cast<cudaStream_t>(stream)>>>(start, count,
                                                                                 kind, out);
  FP4_CUDA(cudaGetLastError());
  return FP4_OK;
}

fp4_status_t fp4_scales_to_canonical(const uint8_t* native, int G, int N, int D,
                                     fp4_axis_t axis, uint8_t* canonical, void* stream) {
  g_last_error.clear();
  fp4_status_t s;
  if ((s = check_shape(1, G, G, N, D)) != FP4_OK) return s;
  if (axis != FP4_BLOCK_ALONG_D && axis != FP4_BLOCK_ALONG_N_T)
    return fail(FP4_ERR_INVALID_ARG, "axis %d", (int)axis);
  if (!native || !canonical) return fail(FP4_ERR_INVALID_ARG, "null pointer");
  int dev, sms;
  if ((s = device_setup(&dev, &sms)) != FP4_OK) return s;
  fp4::scales_canonical_kernel<<<sms * 4, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      native, G, N, D, (int)axis, canonical);
  FP4_CUDA(cudaGetLastError());
  return FP4_OK;
}

int fp4_debug_build(void) {
#ifdef FP4_DEBUG
  return 1;
#else
  return 0;
#endif
}

fp4_status_t fp4_debug_selftest(unsigned site, void* stream) {
  g_last_error.clear();
#ifdef FP4_DEBUG
  if (site < 1 || site > 99) return fail(FP4_ERR_INVALID_ARG, "site must be in 1 .. 99");
  int dev, sms;
  fp4_status_t s;
  if ((s = device_setup(&dev, &sms)) != FP4_OK) return s;
  fp4::dbg_selftest_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(site);
  FP4_CUDA(cudaGetLastError());
  return FP4_OK;
#else
  (void)site;
  (void)stream;
  return fail(FP4_ERR_UNSUPPORTED, "not a debug build (FP4_DEBUG)");
#endif
}

fp4_status_t fp4_test_wait_timeout(uint64_t limit_ns, int* ok, void* stream) {
  g_last_error.clear();
  if (limit_ns == 0 || limit_ns > 5000000000ull || !ok)
    return fail(FP4_ERR_INVALID_ARG, "limit must be in (0, 5 s] and ok non-null");
  int dev, sms;
  fp4_status_t s;
  if ((s = device_setup(&dev, &sms)) != FP4_OK) return s;
  fp4::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, ok);
  FP4_CUDA(cudaGetLastError());
  return FP4_OK;
}

}  // extern "C"
