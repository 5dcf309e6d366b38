// ssd_block.cu -- the steps either side of the SSD in the Mamba-2 block ("Transformers
// are SSMs", the wikillm.com card: the Mamba-2 block sketch of sec. 7.1 and "Paper vs
// code" 1, 2 and 9):
//   before: a depthwise causal convolution of kernel 4 over the concatenated x, B, C
//           channels, then SiLU;
//   after:  the gated RMSNorm, gate first: g = y * silu(z), out = g / rms(g) * weight.
// Both are bound by HBM bandwidth: every input element is read once and every output
// element written once.
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

// 8 consecutive channels of one token: one 16-byte (bf16) or two (fp32) loads.
struct Vec8 {
  float v[8];
};
__device__ __forceinline__ Vec8 load8(const __nv_bfloat16* p) {
  const uint4 q = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
  Vec8 r;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    r.v[2 * i] = __uint_as_float(w[i] << 16);
    r.v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
  return r;
}
__device__ __forceinline__ Vec8 load8(const float* p) {
  const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  return Vec8{{a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w}};
}
// The raw 16 (bf16) or 32 (fp32) bytes of 8 channels, unpacked when used.
template <typename T>
struct Raw8;
template <>
struct Raw8<__nv_bfloat16> {
  uint4 q;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { q = *reinterpret_cast<const uint4*>(p); }
  __device__ __forceinline__ float at(int i) const {
    const uint32_t word = (i >> 1) == 0 ? q.x : (i >> 1) == 1 ? q.y : (i >> 1) == 2 ? q.z : q.w;
    return __uint_as_float((i & 1) ? (word & 0xFFFF0000u) : (word << 16));
  }
};
template <>
struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = *reinterpret_cast<const float4*>(p);
    b = *reinterpret_cast<const float4*>(p + 4);
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

// ------------------------------------------------------------- causal conv1d
struct ConvArgs {
  int64_t tokens, channels, seqlen;  // seqlen: dense row length when cu == null
  int nseq;
  const void* in;
  const float* w;     // (channels, 4): out[t] = sum_k w[c][k] in[t - 3 + k]
  const float* bias;  // (channels) or null
  const int32_t* cu;  // (nseq + 1) or null
  void* out;
};
constexpr int kConvTok = 16;  // tokens per thread: their inputs and the 3-token halo load at once
constexpr int kConvThreads = 128;

__device__ __forceinline__ int64_t seq_start_of(const ConvArgs& a, int64_t s) {
  return a.cu ? (int64_t)a.cu[s] : s * a.seqlen;
}

// Grid: ceil(channels / 8 / 128) channel blocks x ceil(tokens / 16) token blocks, flattened
// (channel block fastest).  A thread computes 8 channels of 16
// consecutive tokens: it loads those tokens and the three before them (the halo, an L2 hit
// after the neighbouring thread block's load) in one go, then walks them in order.  Inputs
// before the start of a token's sequence count as zero.
template <typename T>
__global__ void __launch_bounds__(kConvThreads) conv1d_silu_kernel(ConvArgs a) {
  const int64_t cblocks = (a.channels / 8 + kConvThreads - 1) / kConvThreads;
  const int64_t c0 = ((int64_t)(blockIdx.x % cblocks) * kConvThreads + threadIdx.x) * 8;
  if (c0 >= a.channels) return;
  const int64_t t0 = (int64_t)(blockIdx.x / cblocks) * kConvTok;
  const int64_t t1 = min(t0 + (int64_t)kConvTok, a.tokens);
  const T* in = static_cast<const T*>(a.in);
  T* out = static_cast<T*>(a.out);
  Raw8<T> raw[kConvTok + 3];  // tokens t0 - 3 .. t0 + 7
#pragma unroll
  for (int k = 0; k < kConvTok + 3; ++k) {
    const int64_t t = t0 - 3 + k;
    if (t >= 0 && t < t1) raw[k].load(in + t * a.channels + c0);
  }
  float w[8][4], b[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 q = *reinterpret_cast<const float4*>(a.w + (c0 + i) * 4);
    w[i][0] = q.x, w[i][1] = q.y, w[i][2] = q.z, w[i][3] = q.w;
    b[i] = a.bias ? a.bias[c0 + i] : 0.f;
  }
  // the sequence holding t0: its start, and where the next one starts
  int64_t s;
  if (a.cu) {
    int lo = 0, hi = a.nseq;  // cu[lo] <= t0 < cu[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (a.cu[mid] <= t0) lo = mid;
      else hi = mid;
    }
    s = lo;
  } else {
    s = t0 / a.seqlen;
  }
  int64_t start = seq_start_of(a, s), next = seq_start_of(a, s + 1);
  if (start <= t0 - 3 && next >= t1) {  // no sequence start in the window: every tap is live
#pragma unroll
    for (int k = 0; k < kConvTok; ++k) {
      const int64_t t = t0 + k;
      if (t >= t1) break;
      float o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float acc = b[i];
#pragma unroll
        for (int j = 0; j < 4; ++j) acc = fmaf(w[i][j], raw[k + j].at(i), acc);  // input t - 3 + j
        o[i] = silu(acc);
      }
      store8(out + t * a.channels + c0, o);
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
    bool live[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) live[j] = t - 3 + j >= start;
    float o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float acc = b[i];
#pragma unroll
      for (int j = 0; j < 4; ++j)  // input t - 3 + j sits in raw[k + j]
        if (live[j]) acc = fmaf(w[i][j], raw[k + j].at(i), acc);
      o[i] = silu(acc);
    }
    store8(out + t * a.channels + c0, o);
  }
}

// ------------------------------------------------------------ gated RMSNorm
struct NormArgs {
  int64_t tokens, dim;
  const void* y;
  const void* z;
  const float* w;
  float eps;
  void* out;
};
constexpr int kNormThreads = 256;
constexpr int kNormVecs = 4;  // 8-feature vectors per thread held in registers: dim <= 8192

// One block per token: g = y silu(z) in fp32 registers (with the weights loaded alongside),
// a block sum of g^2, then out = g * rsqrt(mean(g^2) + eps) * w.
template <typename T>
__global__ void __launch_bounds__(kNormThreads) gated_rmsnorm_kernel(NormArgs a) {
  __shared__ float s_part[kNormThreads / 32];
  const int64_t tok = blockIdx.x;
  const T* y = static_cast<const T*>(a.y) + tok * a.dim;
  const T* z = static_cast<const T*>(a.z) + tok * a.dim;
  T* out = static_cast<T*>(a.out) + tok * a.dim;
  const int nv = (int)(a.dim / 8);
  float g[kNormVecs][8], wr[kNormVecs][8];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < kNormVecs; ++k) {
    const int v = threadIdx.x + k * kNormThreads;
    if (v < nv) {
      const Vec8 yv = load8(y + v * 8), zv = load8(z + v * 8), wv = load8(a.w + v * 8);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        g[k][i] = yv.v[i] * silu(zv.v[i]);
        wr[k][i] = wv.v[i];
        ss = fmaf(g[k][i], g[k][i], ss);
      }
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
  for (int k = 0; k < kNormVecs; ++k) {
    const int v = threadIdx.x + k * kNormThreads;
    if (v < nv) {
      float o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = g[k][i] * r * wr[k][i];
      store8(out + v * 8, o);
    }
  }
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
  const int64_t nblocks = (channels / 8 + ssd::kConvThreads - 1) / ssd::kConvThreads *
                          ((tokens + ssd::kConvTok - 1) / ssd::kConvTok);
  if (nblocks > ((int64_t)1 << 31) - 1) return SSD_ERR_UNSUPPORTED;
  const dim3 grid((unsigned)nblocks);
  cudaStream_t st = (cudaStream_t)stream;
  if (io_dtype == SSD_BF16)
    ssd::conv1d_silu_kernel<__nv_bfloat16><<<grid, ssd::kConvThreads, 0, st>>>(a);
  else
    ssd::conv1d_silu_kernel<float><<<grid, ssd::kConvThreads, 0, st>>>(a);
  ssd::count_launches(1);
  return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

extern "C" int ssd_gated_rmsnorm(int64_t tokens, int64_t dim, ssd_dtype io_dtype, const void* y, const void* z,
                                 const float* weight, float eps, void* out, ssd_stream_t stream) {
  if (tokens < 0 || dim <= 0 || !(eps >= 0.f)) return SSD_ERR_INVALID_ARG;
  if (io_dtype != SSD_F32 && io_dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
  if (dim % 8 || dim > 8 * ssd::kNormThreads * ssd::kNormVecs) return SSD_ERR_UNSUPPORTED;
  if (tokens > ((int64_t)1 << 31) - 1) return SSD_ERR_UNSUPPORTED;
  if (tokens == 0) return SSD_OK;
  if (!y || !z || !weight || !out) return SSD_ERR_INVALID_ARG;
  if (ssd::misaligned(y) || ssd::misaligned(z) || ssd::misaligned(weight) || ssd::misaligned(out))
    return SSD_ERR_MISALIGNED;
  ssd::NormArgs a;
  a.tokens = tokens;
  a.dim = dim;
  a.y = y, a.z = z, a.w = weight, a.eps = eps, a.out = out;
  cudaStream_t st = (cudaStream_t)stream;
  if (io_dtype == SSD_BF16)
    ssd::gated_rmsnorm_kernel<__nv_bfloat16><<<(unsigned)tokens, ssd::kNormThreads, 0, st>>>(a);
  else
    ssd::gated_rmsnorm_kernel<float><<<(unsigned)tokens, ssd::kNormThreads, 0, st>>>(a);
  ssd::count_launches(1);
  return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
