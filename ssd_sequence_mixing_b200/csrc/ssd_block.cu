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

#include <algorithm>
#include <atomic>

#include "sm100_ptx.cuh"
#include "ssd.h"
#include "ssd_common.cuh"
#include "ssd_tc.cuh"

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

// Bounded wait on an mbarrier phase; false (and the status word's timeout bit set) if it
// gave up, so a lost copy can never hang the GPU.
__device__ __forceinline__ bool bar_wait(uint64_t* bar, uint32_t parity, unsigned int* status) {
  if (sm100::mbar_wait_bounded(bar, parity, 4ll << 30)) return true;
  if (status) atomicOr(status, kStatusTimeout);
  return false;
}

// ------------------------------------------------------------- causal conv1d
// Persistent CTAs.  A work item is 32 tokens x 256 channels; CTA c keeps one channel slice
// (and its weights, in registers) for its whole life and walks every token block b with
// b = c / slices (mod CTAs per slice).  One copy thread brings each item's input rows
// t0 - 3 .. t0 + 31 (the 3-row halo before the block, zero before token 0) into a ring of
// shared-memory stages by TMA, up to kConvStages items ahead; 8 compute warps each make 4
// output tokens of the 256 channels (a lane: 8 channels) and store them straight to global
// memory (512 contiguous bytes per warp and token).  Inputs before the start of a token's
// sequence count as zero.
struct ConvArgs {
  int64_t tokens, channels, seqlen;  // seqlen: dense row length when cu == null
  int nseq;
  const float* w;     // (channels, 4): out[t] = sum_k w[c][k] in[t - 3 + k]
  const float* bias;  // (channels) or null
  const int32_t* cu;  // (nseq + 1) or null
  void* out;
  int slices, blocks, ctas_per_slice;
  unsigned int* status;
};
constexpr int kConvChannels = 256;               // channels per item (one TMA box row)
constexpr int kConvTokens = 32;                  // output tokens per item
constexpr int kConvRows = kConvTokens + 3;       // input rows per item (with the halo)
constexpr int kConvWarps = 8;                    // compute warps: kConvTokens / kConvWarps tokens each
constexpr int kConvThreads = (kConvWarps + 1) * 32;
constexpr int kConvStages = 4;

template <typename T>
__global__ void __launch_bounds__(kConvThreads) conv1d_silu_kernel(const __grid_constant__ CUtensorMap tm_in,
                                                                   ConvArgs a) {
  extern __shared__ uint8_t smem_raw[];
  // TMA tile destinations: 128-byte aligned (the launch reserves the slack)
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  __shared__ uint64_t full[kConvStages], empty[kConvStages];
  __shared__ int64_t seq_start[2][kConvTokens];
  constexpr uint32_t kStage = kConvRows * kConvChannels * sizeof(T);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slice = blockIdx.x % a.slices;
  const int first = blockIdx.x / a.slices;
  if (first >= a.ctas_per_slice) return;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kConvStages; ++s) {
      sm100::mbar_init(&full[s], 1);
      sm100::mbar_init(&empty[s], kConvWarps);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const int c_base = slice * kConvChannels;
  if (warp == kConvWarps) {  // the copy warp
    if (lane == 0) {
      int k = 0;
      for (int b = first; b < a.blocks; b += a.ctas_per_slice, ++k) {
        const int s = k % kConvStages;
        if (k >= kConvStages && !bar_wait(&empty[s], ((k / kConvStages) - 1) & 1, a.status)) break;
        sm100::mbar_expect_tx(&full[s], kStage);
        sm100::tma_load_2d(smem + s * kStage, &tm_in, c_base, b * kConvTokens - 3, &full[s]);
      }
      // every issued copy is waited for by the compute warps before the CTA ends
    }
    return;
  }
  const int64_t c0 = c_base + 8 * lane;  // this lane's 8 channels
  const bool live = c0 < a.channels;
  float w[8][4], bias[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
    if (live) q = *reinterpret_cast<const float4*>(a.w + (c0 + i) * 4);
    w[i][0] = q.x, w[i][1] = q.y, w[i][2] = q.z, w[i][3] = q.w;
    bias[i] = (live && a.bias) ? a.bias[c0 + i] : 0.f;
  }
  T* out = static_cast<T*>(a.out);
  int k = 0;
  for (int b = first; b < a.blocks; b += a.ctas_per_slice, ++k) {
    const int s = k % kConvStages;
    const int64_t t0 = (int64_t)b * kConvTokens;
    // warp 0: the first token of each output token's sequence (double-buffered by item)
    if (warp == 0) {
      const int64_t t = t0 + lane;
      int64_t st = 0;
      if (t < a.tokens) {
        if (a.cu) {
          int lo = 0, hi = a.nseq;  // cu[lo] <= t < cu[hi]; empty sequences end where the next begins
          while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (a.cu[mid] <= t) lo = mid;
            else hi = mid;
          }
          st = a.cu[lo];
        } else {
          st = t - t % a.seqlen;
        }
      }
      seq_start[k & 1][lane] = st;
    }
    asm volatile("bar.sync 1, %0;" ::"r"(kConvWarps * 32) : "memory");  // seq_start written
    if (!bar_wait(&full[s], (k / kConvStages) & 1, a.status)) return;
    const T* tile = reinterpret_cast<const T*>(smem + s * kStage) + 8 * lane;
    Raw8<T> raw[kConvTokens / kConvWarps + 3];
#pragma unroll
    for (int j = 0; j < kConvTokens / kConvWarps + 3; ++j) raw[j].load(tile + (warp * (kConvTokens / kConvWarps) + j) * kConvChannels);
    __syncwarp();
    if (lane == 0) sm100::mbar_arrive(&empty[s]);  // this warp has its rows: the stage may be refilled
#pragma unroll
    for (int r = 0; r < kConvTokens / kConvWarps; ++r) {
      const int tl = warp * (kConvTokens / kConvWarps) + r;  // token within the item
      const int64_t t = t0 + tl;
      if (t >= a.tokens || !live) continue;
      const int64_t st = seq_start[k & 1][tl];
      float o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float acc = bias[i];
#pragma unroll
        for (int j = 0; j < 4; ++j)  // input t - 3 + j sits in raw[r + j]
          if (t - 3 + j >= st) acc = fmaf(w[i][j], raw[r + j].at(i), acc);
        o[i] = silu(acc);
      }
      store8(out + t * a.channels + c0, o);
    }
  }
}

// ------------------------------------------------------------ gated RMSNorm
// Persistent CTAs; CTA c takes tokens c, c + CTAs, ...  One copy thread brings each
// token's y and z rows into a ring of shared-memory stages by bulk copies, up to
// `stages` tokens ahead; 10 compute warps form g = y silu(z) in fp32 registers (each
// thread up to 4 vectors of 8 features, with its weights in registers for the CTA's
// whole life), reduce sum(g^2) over the CTA, and store out = g * rsqrt(mean(g^2) + eps)
// * w straight to global memory.
struct NormArgs {
  int64_t tokens, dim;
  const void* y;
  const void* z;
  const float* w;
  float eps;
  void* out;
  int stages;
  unsigned int* status;
};
constexpr int kNormWarps = 10;
constexpr int kNormCompute = kNormWarps * 32;
constexpr int kNormThreads = kNormCompute + 32;  // + the copy warp
constexpr int kNormVecs = 4;                     // 8-feature vectors per thread: dim <= 8 * 320 * 4
constexpr int kNormMaxStages = 4;

template <typename T>
__global__ void __launch_bounds__(kNormThreads) gated_rmsnorm_kernel(NormArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t full[kNormMaxStages], empty[kNormMaxStages];
  __shared__ float part[2][kNormWarps];
  const uint32_t row = (uint32_t)(a.dim * sizeof(T));
  const int S = a.stages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      sm100::mbar_init(&full[s], 1);
      sm100::mbar_init(&empty[s], kNormWarps);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (warp == kNormWarps) {  // the copy warp
    if (lane == 0) {
      int k = 0;
      for (int64_t tok = blockIdx.x; tok < a.tokens; tok += gridDim.x, ++k) {
        const int s = k % S;
        if (k >= S && !bar_wait(&empty[s], ((k / S) - 1) & 1, a.status)) break;
        uint8_t* dst = smem + (size_t)s * 2 * row;
        sm100::mbar_expect_tx(&full[s], 2 * row);
        sm100::bulk_load(dst, static_cast<const uint8_t*>(a.y) + tok * row, row, &full[s]);
        sm100::bulk_load(dst + row, static_cast<const uint8_t*>(a.z) + tok * row, row, &full[s]);
      }
    }
    return;
  }
  const int tid = threadIdx.x;
  const int nv = (int)(a.dim / 8);
  float wr[kNormVecs][8];
#pragma unroll
  for (int j = 0; j < kNormVecs; ++j) {
    const int v = tid + j * kNormCompute;
    const Vec8 wv = v < nv ? load8(a.w + v * 8) : Vec8{};
#pragma unroll
    for (int i = 0; i < 8; ++i) wr[j][i] = wv.v[i];
  }
  T* out = static_cast<T*>(a.out);
  int k = 0;
  for (int64_t tok = blockIdx.x; tok < a.tokens; tok += gridDim.x, ++k) {
    const int s = k % S;
    if (!bar_wait(&full[s], (k / S) & 1, a.status)) return;
    const T* ys = reinterpret_cast<const T*>(smem + (size_t)s * 2 * row);
    const T* zs = reinterpret_cast<const T*>(smem + (size_t)s * 2 * row + row);
    float g[kNormVecs][8];
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < kNormVecs; ++j) {
      const int v = tid + j * kNormCompute;
      if (v < nv) {
        const Vec8 yv = load8(ys + v * 8), zv = load8(zs + v * 8);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          g[j][i] = yv.v[i] * silu(zv.v[i]);
          ss = fmaf(g[j][i], g[j][i], ss);
        }
      }
    }
    __syncwarp();
    if (lane == 0) sm100::mbar_arrive(&empty[s]);  // this warp has read the stage
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) part[k & 1][warp] = ss;
    asm volatile("bar.sync 1, %0;" ::"r"(kNormCompute) : "memory");
    float tot = 0.f;
#pragma unroll
    for (int i = 0; i < kNormWarps; ++i) tot += part[k & 1][i];
    const float r = rsqrtf(tot / (float)a.dim + a.eps);
#pragma unroll
    for (int j = 0; j < kNormVecs; ++j) {
      const int v = tid + j * kNormCompute;
      if (v < nv) {
        float o[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = g[j][i] * r * wr[j][i];
        store8(out + tok * a.dim + v * 8, o);
      }
    }
  }
}

int device_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                 cudaSuccess)
    return 148;
  return sms;
}

// The dynamic shared memory limit of `kernel` is raised once per device.
template <typename K>
cudaError_t allow_smem(K kernel, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
  if (bit && (done.load() & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit);
  return e;
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
  a.w = weight, a.bias = bias, a.cu = cu_seqlens, a.out = out;
  a.status = ssd::device_status_word();
  a.slices = (int)((channels + ssd::kConvChannels - 1) / ssd::kConvChannels);
  const int64_t blocks = (tokens + ssd::kConvTokens - 1) / ssd::kConvTokens;
  if (blocks > ((int64_t)1 << 30)) return SSD_ERR_UNSUPPORTED;
  a.blocks = (int)blocks;
  // about two CTAs per SM, spread over the channel slices
  const int64_t want = 2 * (int64_t)ssd::device_sms();
  a.ctas_per_slice = (int)std::max<int64_t>(1, std::min<int64_t>(blocks, (want + a.slices - 1) / a.slices));
  const int64_t grid = (int64_t)a.slices * a.ctas_per_slice;
  if (grid > ((int64_t)1 << 31) - 1) return SSD_ERR_UNSUPPORTED;
  // the input as a 2-D {channels, tokens} tensor: boxes of 256 channels x 35 rows
  auto enc = ssd::tensor_map_encoder();
  if (!enc) return SSD_ERR_CUDA;
  const bool bf = io_dtype == SSD_BF16;
  const size_t es = bf ? 2 : 4;
  CUtensorMap tm;
  cuuint64_t dims[2] = {(cuuint64_t)channels, (cuuint64_t)tokens};
  cuuint64_t strides[1] = {(cuuint64_t)channels * es};
  cuuint32_t box[2] = {(cuuint32_t)ssd::kConvChannels, (cuuint32_t)ssd::kConvRows};
  cuuint32_t estr[2] = {1, 1};
  if (enc(&tm, bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(xbc),
          dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return SSD_ERR_CUDA;
  const int smem = ssd::kConvStages * ssd::kConvRows * ssd::kConvChannels * (int)es + 128;
  cudaStream_t st = (cudaStream_t)stream;
  static std::atomic<uint64_t> done_bf{0}, done_f{0};
  cudaError_t e;
  if (bf) {
    e = ssd::allow_smem(ssd::conv1d_silu_kernel<__nv_bfloat16>, smem, done_bf);
    if (e == cudaSuccess)
      ssd::conv1d_silu_kernel<__nv_bfloat16><<<(unsigned)grid, ssd::kConvThreads, smem, st>>>(tm, a);
  } else {
    e = ssd::allow_smem(ssd::conv1d_silu_kernel<float>, smem, done_f);
    if (e == cudaSuccess) ssd::conv1d_silu_kernel<float><<<(unsigned)grid, ssd::kConvThreads, smem, st>>>(tm, a);
  }
  ssd::count_launches(1);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

extern "C" int ssd_gated_rmsnorm(int64_t tokens, int64_t dim, ssd_dtype io_dtype, const void* y, const void* z,
                                 const float* weight, float eps, void* out, ssd_stream_t stream) {
  if (tokens < 0 || dim <= 0 || !(eps >= 0.f)) return SSD_ERR_INVALID_ARG;
  if (io_dtype != SSD_F32 && io_dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
  if (dim % 8 || dim > 8192) return SSD_ERR_UNSUPPORTED;
  if (tokens > ((int64_t)1 << 31) - 1) return SSD_ERR_UNSUPPORTED;
  if (tokens == 0) return SSD_OK;
  if (!y || !z || !weight || !out) return SSD_ERR_INVALID_ARG;
  if (ssd::misaligned(y) || ssd::misaligned(z) || ssd::misaligned(weight) || ssd::misaligned(out))
    return SSD_ERR_MISALIGNED;
  ssd::NormArgs a;
  a.tokens = tokens;
  a.dim = dim;
  a.y = y, a.z = z, a.w = weight, a.eps = eps, a.out = out;
  a.status = ssd::device_status_word();
  const int row = (int)(dim * (io_dtype == SSD_BF16 ? 2 : 4));
  // up to 4 tokens in flight per CTA within about 100 KB, at least 2
  a.stages = std::max(2, std::min(ssd::kNormMaxStages, (100 << 10) / (2 * row)));
  const int smem = a.stages * 2 * row;  // at most 2 x 2 x 32 KB (dim 8192, fp32)
  const int per_sm = std::max(1, std::min(4, (220 << 10) / (smem + 2048)));
  const int64_t grid = std::min<int64_t>(tokens, (int64_t)per_sm * ssd::device_sms());
  cudaStream_t st = (cudaStream_t)stream;
  static std::atomic<uint64_t> done_bf{0}, done_f{0};
  cudaError_t e;
  // the attribute is raised once to the largest size any call of this kernel takes
  constexpr int kNormSmemMax = 2 * 2 * 8192 * 4;
  if (io_dtype == SSD_BF16) {
    e = ssd::allow_smem(ssd::gated_rmsnorm_kernel<__nv_bfloat16>, kNormSmemMax, done_bf);
    if (e == cudaSuccess)
      ssd::gated_rmsnorm_kernel<__nv_bfloat16><<<(unsigned)grid, ssd::kNormThreads, smem, st>>>(a);
  } else {
    e = ssd::allow_smem(ssd::gated_rmsnorm_kernel<float>, kNormSmemMax, done_f);
    if (e == cudaSuccess) ssd::gated_rmsnorm_kernel<float><<<(unsigned)grid, ssd::kNormThreads, smem, st>>>(a);
  }
  ssd::count_launches(1);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
