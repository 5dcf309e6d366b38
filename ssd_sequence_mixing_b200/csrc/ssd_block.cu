// ssd_block.cu -- the steps either side of the SSD in the Mamba-2 block ("Transformers
// are SSMs", the wikillm.com card: the Mamba-2 block sketch of sec. 7.1 and "Paper vs
// code" 1, 2 and 9):
//   before: a depthwise causal convolution of kernel 4 over the concatenated x, B, C
//           channels, then SiLU;
//   after:  the gated RMSNorm, gate first: g = y * silu(z), out = g / rms(g) * weight.
// Both are bound by HBM bandwidth: every input element is read once and every output
// element written once.  What made them fast was keeping the threads light (few registers,
// many warps in flight) and the hot paths free of per-element bounds checks.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "ssd.h"
#include "ssd_common.cuh"

namespace ssd {
namespace {

// v sigmoid(v) with the hardware exponential and the approximate division (relative error
// a few ulp, far below bf16 rounding; 0 where e^-v overflows); both kernels are bound by
// instruction issue with the IEEE forms.
__device__ __forceinline__ float silu(float v) { return __fdividef(v, 1.f + __expf(-v)); }

// 8 consecutive fp32 values (the norm's weights).
struct Vec8 {
  float v[8];
};
__device__ __forceinline__ Vec8 load8(const float* p) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p)), b = __ldg(reinterpret_cast<const float4*>(p + 4));
  return Vec8{{a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w}};
}
// The raw 16 (bf16) or 32 (fp32) bytes of 8 channels, unpacked when used.
template <typename T>
struct Raw8;
template <>
struct Raw8<__nv_bfloat16> {
  uint4 q;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { q = __ldg(reinterpret_cast<const uint4*>(p)); }
  __device__ __forceinline__ float at(int i) const {
    const uint32_t word = (i >> 1) == 0 ? q.x : (i >> 1) == 1 ? q.y : (i >> 1) == 2 ? q.z : q.w;
    return __uint_as_float((i & 1) ? (word & 0xFFFF0000u) : (word << 16));
  }
};
template <>
struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = __ldg(reinterpret_cast<const float4*>(p));
    b = __ldg(reinterpret_cast<const float4*>(p + 4));
  }
  __device__ __forceinline__ float at(int i) const {
    const float4& h = i < 4 ? a : b;
    const int j = i & 3;
    return j == 0 ? h.x : j == 1 ? h.y : j == 2 ? h.z : h.w;
  }
};

__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&v)[8]) {
  uint4 q;
  uint32_t* w = reinterpret_cast<uint32_t*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  *reinterpret_cast<uint4*>(p) = q;
}
__device__ __forceinline__ void store8(float* p, const float (&v)[8]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}

// 4 consecutive channels of one token, kept packed until used: 8 bytes (bf16) or 16 (fp32).
template <typename T>
struct Raw4;
template <>
struct Raw4<__nv_bfloat16> {
  uint2 q;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { q = __ldg(reinterpret_cast<const uint2*>(p)); }
  __device__ __forceinline__ void zero() { q = make_uint2(0u, 0u); }
  __device__ __forceinline__ void get(float (&v)[4]) const {
    v[0] = __uint_as_float(q.x << 16), v[1] = __uint_as_float(q.x & 0xFFFF0000u);
    v[2] = __uint_as_float(q.y << 16), v[3] = __uint_as_float(q.y & 0xFFFF0000u);
  }
};
template <>
struct Raw4<float> {
  float4 q;
  __device__ __forceinline__ void load(const float* p) { q = __ldg(reinterpret_cast<const float4*>(p)); }
  __device__ __forceinline__ void zero() { q = make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ void get(float (&v)[4]) const { v[0] = q.x, v[1] = q.y, v[2] = q.z, v[3] = q.w; }
};
__device__ __forceinline__ void store4(__nv_bfloat16* p, const float (&v)[4]) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
  *reinterpret_cast<uint2*>(p) = make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b));
}
__device__ __forceinline__ void store4(float* p, const float (&v)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}

// ------------------------------------------------------------- causal conv1d
// A thread makes 4 channels of 16 consecutive tokens: it loads those tokens' inputs and
// the three before them (the halo; an L2 hit after the neighbouring block's loads) at
// once, then slides a 4-token window over them, unpacking each input once.  Threads are
// kept light (registers capped for 12 blocks of 64 per SM) so that enough loads are in
// flight while other warps compute.  Grid: channel blocks x token blocks (channel block
// fastest).  Inputs before the start of a token's sequence count as zero.
struct ConvArgs {
  int64_t tokens, channels, seqlen;  // seqlen: dense row length when cu == null
  int nseq;
  const void* in;
  const float* w;     // (channels, 4): out[t] = sum_k w[c][k] in[t - 3 + k]
  const float* bias;  // (channels) or null
  const int32_t* cu;  // (nseq + 1) or null
  void* out;
};
constexpr int kConvTok = 16;
constexpr int kConvThreads = 64;
constexpr int kConvMinBlocks = 12;

__device__ __forceinline__ int64_t seq_start_of(const ConvArgs& a, int64_t s) {
  return a.cu ? (int64_t)a.cu[s] : s * a.seqlen;
}

template <typename T>
__global__ void __launch_bounds__(kConvThreads, kConvMinBlocks) conv1d_silu_kernel(ConvArgs a) {
  const int64_t cblocks = (a.channels / 4 + kConvThreads - 1) / kConvThreads;
  const int64_t c0 = ((int64_t)(blockIdx.x % cblocks) * kConvThreads + threadIdx.x) * 4;
  if (c0 >= a.channels) return;
  const int64_t t0 = (int64_t)(blockIdx.x / cblocks) * kConvTok;
  const int64_t t1 = min(t0 + (int64_t)kConvTok, a.tokens);
  const T* in = static_cast<const T*>(a.in);
  T* out = static_cast<T*>(a.out);
  Raw4<T> raw[kConvTok + 3];  // tokens t0 - 3 .. t0 + 15
  if (t0 >= 3 && t0 + kConvTok <= a.tokens) {  // interior block: every row exists
    const T* p = in + (t0 - 3) * a.channels + c0;
#pragma unroll
    for (int k = 0; k < kConvTok + 3; ++k) raw[k].load(p + k * a.channels);
  } else {
#pragma unroll
    for (int k = 0; k < kConvTok + 3; ++k) {
      const int64_t t = t0 - 3 + k;
      if (t >= 0 && t < t1)
        raw[k].load(in + t * a.channels + c0);
      else
        raw[k].zero();
    }
  }
  float w[4][4], b[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 q = __ldg(reinterpret_cast<const float4*>(a.w + (c0 + i) * 4));
    w[i][0] = q.x, w[i][1] = q.y, w[i][2] = q.z, w[i][3] = q.w;
    b[i] = a.bias ? __ldg(a.bias + c0 + i) : 0.f;
  }
  // the sequence holding t0: its start, and where the next one starts
  int64_t s;
  if (a.cu) {
    int lo = 0, hi = a.nseq;  // cu[lo] <= t0 < cu[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (a.cu[mid] <= t0)
        lo = mid;
      else
        hi = mid;
    }
    s = lo;
  } else {
    s = t0 / a.seqlen;
  }
  int64_t start = seq_start_of(a, s), next = seq_start_of(a, s + 1);
  float x0[4], x1[4], x2[4], x3[4];  // inputs t - 3 .. t
  raw[0].get(x0), raw[1].get(x1), raw[2].get(x2);
  if (start <= t0 - 3 && next >= t1) {  // no sequence start in the window: every tap is live
#pragma unroll
    for (int k = 0; k < kConvTok; ++k) {
      const int64_t t = t0 + k;
      if (t >= t1) break;
      raw[k + 3].get(x3);
      float o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        o[i] = silu(fmaf(w[i][3], x3[i], fmaf(w[i][2], x2[i], fmaf(w[i][1], x1[i], fmaf(w[i][0], x0[i], b[i])))));
      store4(out + t * a.channels + c0, o);
#pragma unroll
      for (int i = 0; i < 4; ++i) x0[i] = x1[i], x1[i] = x2[i], x2[i] = x3[i];
    }
    return;
  }
#pragma unroll
  for (int k = 0; k < kConvTok; ++k) {
    const int64_t t = t0 + k;
    if (t >= t1) break;
    while (t >= next && s + 1 < a.nseq) {  // empty sequences end where the next begins
      ++s;
      start = next;
      next = seq_start_of(a, s + 1);
    }
    raw[k + 3].get(x3);
    const float l0 = t - 3 >= start, l1 = t - 2 >= start, l2 = t - 1 >= start;  // live taps (t itself is)
    float o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      o[i] = silu(fmaf(w[i][3], x3[i], fmaf(w[i][2], l2 * x2[i], fmaf(w[i][1], l1 * x1[i], fmaf(w[i][0], l0 * x0[i], b[i])))));
    store4(out + t * a.channels + c0, o);
#pragma unroll
    for (int i = 0; i < 4; ++i) x0[i] = x1[i], x1[i] = x2[i], x2[i] = x3[i];
  }
}

// ------------------------------------------------------------ gated RMSNorm
// One block of 128 threads per token; thread j holds the 8-feature vectors j, j + 128, ...
// (VECS of them, dim <= 8 x 128 x VECS) of y and z in registers: g = y silu(z), a block sum
// of g^2, then out = g rsqrt(mean(g^2) + eps) w.  Each row is read once and written once.
struct NormArgs {
  int64_t tokens, dim;
  const void* y;
  const void* z;
  const float* w;
  float eps;
  void* out;
};
constexpr int kNormThreads = 128;
constexpr int kNormMaxVecs = 8;  // dim <= 8192

template <typename T, int VECS, bool FULL>  // FULL: dim == 8 x 128 x VECS (no bounds checks)
__global__ void __launch_bounds__(kNormThreads) gated_rmsnorm_kernel(NormArgs a) {
  __shared__ float s_part[kNormThreads / 32];
  const int64_t tok = blockIdx.x;
  const T* y = static_cast<const T*>(a.y) + tok * a.dim;
  const T* z = static_cast<const T*>(a.z) + tok * a.dim;
  T* out = static_cast<T*>(a.out) + tok * a.dim;
  const int nv = (int)(a.dim / 8);
  Raw8<T> yr[VECS], zr[VECS];
#pragma unroll
  for (int k = 0; k < VECS; ++k) {
    const int v = threadIdx.x + k * kNormThreads;
    if (FULL || v < nv) yr[k].load(y + v * 8), zr[k].load(z + v * 8);
  }
  float g[VECS][8];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < VECS; ++k) {
    const bool in = FULL || threadIdx.x + k * kNormThreads < nv;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      g[k][i] = in ? yr[k].at(i) * silu(zr[k].at(i)) : 0.f;
      ss = fmaf(g[k][i], g[k][i], ss);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int i = 0; i < kNormThreads / 32; ++i) tot += s_part[i];
  const float r = rsqrtf(tot / (float)a.dim + a.eps);
#pragma unroll
  for (int k = 0; k < VECS; ++k) {
    const int v = threadIdx.x + k * kNormThreads;
    if (FULL || v < nv) {
      const Vec8 wv = load8(a.w + v * 8);
      float o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = g[k][i] * r * wv.v[i];
      store8(out + v * 8, o);
    }
  }
}

template <typename T, int VECS = 1>
cudaError_t launch_norm(int vecs, const NormArgs& a, cudaStream_t st) {
  if constexpr (VECS < kNormMaxVecs) {
    if (vecs > VECS) return launch_norm<T, VECS + 1>(vecs, a, st);
  }
  if (a.dim == 8 * kNormThreads * VECS)
    gated_rmsnorm_kernel<T, VECS, true><<<(unsigned)a.tokens, kNormThreads, 0, st>>>(a);
  else
    gated_rmsnorm_kernel<T, VECS, false><<<(unsigned)a.tokens, kNormThreads, 0, st>>>(a);
  return cudaGetLastError();
}

bool misaligned(const void* p) { return p && ((uintptr_t)p & 15u); }

}  // namespace
}  // namespace ssd

extern "C" int ssd_causal_conv1d_silu(int64_t batch, int64_t seqlen, int64_t channels, ssd_dtype io_dtype,
                                      const void* xbc, const float* weight, const float* bias,
                                      const int32_t* cu_seqlens, int64_t nseq, void* out, ssd_stream_t stream) {
  if (batch < 0 || seqlen < 0 || channels <= 0) return SSD_ERR_INVALID_ARG;
  if (io_dtype != SSD_F32 && io_dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
  if (cu_seqlens && (batch != 1 || nseq < 1)) return SSD_ERR_INVALID_ARG;
  if (channels % 8 || channels > ((int64_t)1 << 24)) return SSD_ERR_UNSUPPORTED;
  const int64_t tokens = batch * seqlen;
  if (tokens > ((int64_t)1 << 31) || nseq > ((int64_t)1 << 30)) return SSD_ERR_UNSUPPORTED;
  if (tokens == 0) return SSD_OK;
  if (!xbc || !weight || !out) return SSD_ERR_INVALID_ARG;
  if (ssd::misaligned(xbc) || ssd::misaligned(weight) || ssd::misaligned(bias) || ssd::misaligned(out) ||
      ssd::misaligned(cu_seqlens))
    return SSD_ERR_MISALIGNED;
  ssd::ConvArgs a;
  a.tokens = tokens;
  a.channels = channels;
  a.seqlen = cu_seqlens ? tokens : seqlen;
  a.nseq = (int)(cu_seqlens ? nseq : batch);
  a.in = xbc, a.w = weight, a.bias = bias, a.cu = cu_seqlens, a.out = out;
  const int64_t cblocks = (channels / 4 + ssd::kConvThreads - 1) / ssd::kConvThreads;
  const int64_t grid = cblocks * ((tokens + ssd::kConvTok - 1) / ssd::kConvTok);
  if (grid > ((int64_t)1 << 31) - 1) return SSD_ERR_UNSUPPORTED;
  cudaStream_t st = (cudaStream_t)stream;
  if (io_dtype == SSD_BF16)
    ssd::conv1d_silu_kernel<__nv_bfloat16><<<(unsigned)grid, ssd::kConvThreads, 0, st>>>(a);
  else
    ssd::conv1d_silu_kernel<float><<<(unsigned)grid, ssd::kConvThreads, 0, st>>>(a);
  ssd::count_launches(1);
  return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

extern "C" int ssd_gated_rmsnorm(int64_t tokens, int64_t dim, ssd_dtype io_dtype, const void* y, const void* z,
                                 const float* weight, float eps, void* out, ssd_stream_t stream) {
  if (tokens < 0 || dim <= 0 || !(eps >= 0.f)) return SSD_ERR_INVALID_ARG;
  if (io_dtype != SSD_F32 && io_dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
  if (dim % 8 || dim > 8 * ssd::kNormThreads * ssd::kNormMaxVecs) return SSD_ERR_UNSUPPORTED;
  if (tokens > ((int64_t)1 << 31) - 1) return SSD_ERR_UNSUPPORTED;
  if (tokens == 0) return SSD_OK;
  if (!y || !z || !weight || !out) return SSD_ERR_INVALID_ARG;
  if (ssd::misaligned(y) || ssd::misaligned(z) || ssd::misaligned(weight) || ssd::misaligned(out))
    return SSD_ERR_MISALIGNED;
  ssd::NormArgs a;
  a.tokens = tokens;
  a.dim = dim;
  a.y = y, a.z = z, a.w = weight, a.eps = eps, a.out = out;
  const int vecs = (int)((dim / 8 + ssd::kNormThreads - 1) / ssd::kNormThreads);
  cudaStream_t st = (cudaStream_t)stream;
  const cudaError_t e = io_dtype == SSD_BF16 ? ssd::launch_norm<__nv_bfloat16>(vecs, a, st)
                                             : ssd::launch_norm<float>(vecs, a, st);
  ssd::count_launches(1);
  return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
