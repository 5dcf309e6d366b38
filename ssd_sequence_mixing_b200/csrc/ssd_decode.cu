// ssd_decode.cu -- one recurrent generation step of the SSD layer for a batch of
// sequences ("Transformers are SSMs", the wikillm.com card's Method step 8 and sec. 6.3:
// in generation the layer is the linear recurrence, N^2 work per token and head).
//
// For every batch row b and head h (group g = h / (H/G)), with the fp32 state S (P x N):
//   a = exp(dt A_h);   S <- a S + dt x B^T;   y = S C + D_h x
// The state is read and written once: the step is bound by HBM bandwidth on it.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ssd.h"
#include "ssd_common.cuh"

namespace ssd {
namespace {

struct DecodeArgs {
  int64_t rows;  // batch rows
  int H, P, N, G, hpg;
  const void* x;
  const float* dt;
  const float* A;
  const void* B;
  const void* C;
  const float* D;
  float* state;
  void* y;
};

constexpr int kRowsPerWarp = 8;  // state rows (p) a warp advances together (their loads in flight at once)
constexpr int kWarps = 4;
constexpr int kRowsPerCta = kRowsPerWarp * kWarps;

__device__ __forceinline__ void load4(const float* p, float (&v)[4]) {
  const float4 q = *reinterpret_cast<const float4*>(p);
  v[0] = q.x, v[1] = q.y, v[2] = q.z, v[3] = q.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16* p, float (&v)[4]) {
  const uint2 q = *reinterpret_cast<const uint2*>(p);
  v[0] = __uint_as_float(q.x << 16), v[1] = __uint_as_float(q.x & 0xFFFF0000u);
  v[2] = __uint_as_float(q.y << 16), v[3] = __uint_as_float(q.y & 0xFFFF0000u);
}

// Grid (rows * H, ceil(P / 32)); 4 warps, each advancing 8 state rows.  Lane l owns the
// state columns n = 4 l + 128 k (k < KN, N <= 128 KN, N % 4 == 0): float4 loads and stores
// of a 512-byte row segment per warp instruction.  y_p is the warp sum of C_n S[p][n].
template <typename T, int KN>
__global__ void __launch_bounds__(kWarps * 32) decode_step_kernel(DecodeArgs a) {
  const int64_t bh = blockIdx.x;
  const int64_t b = bh / a.H;
  const int h = (int)(bh % a.H);
  const int g = h / a.hpg;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float dtv = a.dt[bh];
  const float decay = expf(dtv * a.A[h]);
  const float Dh = a.D ? a.D[h] : 0.f;
  const T* Bv = static_cast<const T*>(a.B) + (b * a.G + g) * a.N;
  const T* Cv = static_cast<const T*>(a.C) + (b * a.G + g) * a.N;
  const T* xv = static_cast<const T*>(a.x) + bh * a.P;
  T* yv = static_cast<T*>(a.y) + bh * a.P;
  float* S = a.state + bh * (int64_t)a.P * a.N;

  float bq[KN][4], cq[KN][4];
#pragma unroll
  for (int k = 0; k < KN; ++k) {
    const int n0 = 4 * lane + 128 * k;
    if (n0 < a.N) {
      load4(Bv + n0, bq[k]);
      load4(Cv + n0, cq[k]);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) bq[k][j] = cq[k][j] = 0.f;
    }
  }
  const int p0 = blockIdx.y * kRowsPerCta + warp * kRowsPerWarp;
  float s[kRowsPerWarp][KN][4];
  float xp[kRowsPerWarp];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int p = p0 + r;
    xp[r] = p < a.P ? to_f(xv[p]) : 0.f;
#pragma unroll
    for (int k = 0; k < KN; ++k) {
      const int n0 = 4 * lane + 128 * k;
      if (p < a.P && n0 < a.N) load4(S + (int64_t)p * a.N + n0, s[r][k]);
    }
  }
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int p = p0 + r;
    const float dx = dtv * xp[r];
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k < KN; ++k) {
      const int n0 = 4 * lane + 128 * k;
      if (p < a.P && n0 < a.N) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          s[r][k][j] = fmaf(decay, s[r][k][j], dx * bq[k][j]);
          acc = fmaf(cq[k][j], s[r][k][j], acc);
        }
        *reinterpret_cast<float4*>(S + (int64_t)p * a.N + n0) =
            make_float4(s[r][k][0], s[r][k][1], s[r][k][2], s[r][k][3]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0 && p < a.P) yv[p] = from_f<T>(acc + Dh * xp[r]);
  }
}

}  // namespace
}  // namespace ssd

extern "C" int ssd_decode_step(const ssd_shape* s, const void* x, const float* dt, const float* A, const void* B,
                               const void* C, const float* D, float* state, void* y, ssd_stream_t stream) {
  if (!s) return SSD_ERR_INVALID_ARG;
  if (s->batch < 0 || s->seqlen != 1 || s->nheads <= 0 || s->headdim <= 0 || s->dstate <= 0 || s->ngroups <= 0)
    return SSD_ERR_INVALID_ARG;
  if (s->io_dtype != SSD_F32 && s->io_dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
  if (s->nheads % s->ngroups || s->dstate % 4 || s->dstate > 256 || s->nheads > (1 << 20) ||
      s->headdim > (1 << 16))
    return SSD_ERR_UNSUPPORTED;
  if (s->batch * s->nheads > ((int64_t)1 << 31) - 1) return SSD_ERR_UNSUPPORTED;
  if (s->batch == 0) return SSD_OK;
  if (!x || !dt || !A || !B || !C || !state || !y) return SSD_ERR_INVALID_ARG;
  const void* ptrs[] = {x, dt, A, B, C, D, state, y};
  for (const void* p : ptrs)
    if (p && ((uintptr_t)p & 15u)) return SSD_ERR_MISALIGNED;
  ssd::DecodeArgs a;
  a.rows = s->batch;
  a.H = (int)s->nheads;
  a.P = (int)s->headdim;
  a.N = (int)s->dstate;
  a.G = (int)s->ngroups;
  a.hpg = a.H / a.G;
  a.x = x, a.dt = dt, a.A = A, a.B = B, a.C = C, a.D = D, a.state = state, a.y = y;
  const dim3 grid((unsigned)(s->batch * s->nheads), (unsigned)((s->headdim + ssd::kRowsPerCta - 1) / ssd::kRowsPerCta));
  cudaStream_t st = (cudaStream_t)stream;
  const bool wide = s->dstate > 128;
  if (s->io_dtype == SSD_BF16) {
    if (wide)
      ssd::decode_step_kernel<__nv_bfloat16, 2><<<grid, ssd::kWarps * 32, 0, st>>>(a);
    else
      ssd::decode_step_kernel<__nv_bfloat16, 1><<<grid, ssd::kWarps * 32, 0, st>>>(a);
  } else {
    if (wide)
      ssd::decode_step_kernel<float, 2><<<grid, ssd::kWarps * 32, 0, st>>>(a);
    else
      ssd::decode_step_kernel<float, 1><<<grid, ssd::kWarps * 32, 0, st>>>(a);
  }
  ssd::count_launches(1);
  return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
