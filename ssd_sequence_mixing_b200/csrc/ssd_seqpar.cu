// ssd_seqpar.cu -- the two small steps of the sequence-parallel SSD ("Transformers are
// SSMs", the wikillm.com card: Method step 5, the centre factor that passes the state from
// one chunk to the next, applied here between segments of one sequence held by different
// GPUs).  A rank runs its segment from a zero state and publishes its end state s_r and
// its segment log-decay lambda_r = sum_t dt_t A_h; the start state of segment r is then
//     h_0 = init,   h_{q+1} = exp(lambda_q) h_q + s_q,
// after which the rank runs its segment again from h_r.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "ssd.h"
#include "ssd_common.cuh"

namespace ssd {
namespace {

constexpr int kHeadsPerBlock = 32, kTokLanes = 32, kSliceTokens = 512;

// The sum of dt over tokens [t0, t1) of heads blockIdx.x * 32 + (0 .. 31), into out[h]: a
// block of 32 heads x 32 token lanes reads dt rows coalesced, each lane four tokens at a
// time, and the lanes' sums are added in a fixed order (the result does not depend on
// scheduling).
__device__ void logdecay_slice(int64_t t0, int64_t t1, int H, const float* dt, float* out) {
  __shared__ float part[kTokLanes][kHeadsPerBlock];
  const int hl = threadIdx.x % kHeadsPerBlock, tl = threadIdx.x / kHeadsPerBlock;
  const int h = blockIdx.x * kHeadsPerBlock + hl;
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  if (h < H)
    for (int64_t t = t0 + tl; t < t1; t += 4 * kTokLanes) {
      a0 += __ldg(dt + t * H + h);
      if (t + kTokLanes < t1) a1 += __ldg(dt + (t + kTokLanes) * H + h);
      if (t + 2 * kTokLanes < t1) a2 += __ldg(dt + (t + 2 * kTokLanes) * H + h);
      if (t + 3 * kTokLanes < t1) a3 += __ldg(dt + (t + 3 * kTokLanes) * H + h);
    }
  part[tl][hl] = (a0 + a1) + (a2 + a3);
  __syncthreads();
  if (tl == 0 && h < H) {
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < kTokLanes; ++k) s += part[k][hl];
    out[h] = s;
  }
}

// out[h] = A[h] * sum of dt over all tokens; grid ceil(H / 32).
__global__ void __launch_bounds__(kHeadsPerBlock * kTokLanes)
    segment_logdecay_kernel(int64_t tokens, int H, const float* dt, const float* A, float* out) {
  logdecay_slice(0, tokens, H, dt, out);
  __syncthreads();
  const int h = blockIdx.x * kHeadsPerBlock + threadIdx.x;
  if (threadIdx.x < kHeadsPerBlock && h < H) out[h] *= A[h];
}

// One thread per state element (h, p, n): the recurrence over the preceding segments.
__global__ void __launch_bounds__(256) state_prefix_kernel(int rank, int64_t H, int64_t PN, const float* states,
                                                           const float* logdecay, const float* init, float* out) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= H * PN) return;
  const int64_t h = e / PN;
  float acc = init ? init[e] : 0.f;
  for (int q = 0; q < rank; ++q) acc = fmaf(expf(logdecay[q * H + h]), acc, states[q * H * PN + e]);
  out[e] = acc;
}

}  // namespace
}  // namespace ssd

extern "C" int ssd_segment_logdecay(int64_t tokens, int64_t nheads, const float* dt, const float* A, float* out,
                                    ssd_stream_t stream) {
  if (tokens < 0 || nheads <= 0 || nheads > (1 << 24)) return SSD_ERR_INVALID_ARG;
  if (!dt || !A || !out) return SSD_ERR_INVALID_ARG;
  const unsigned blocks = (unsigned)((nheads + ssd::kHeadsPerBlock - 1) / ssd::kHeadsPerBlock);
  ssd::segment_logdecay_kernel<<<blocks, ssd::kHeadsPerBlock * ssd::kTokLanes, 0, (cudaStream_t)stream>>>(
      tokens, (int)nheads, dt, A, out);
  ssd::count_launches(1);
  return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

extern "C" int ssd_state_prefix(int rank, int64_t nheads, int64_t headdim, int64_t dstate, const float* states,
                                const float* logdecay, const float* init_state, float* out, ssd_stream_t stream) {
  if (rank < 0 || nheads <= 0 || headdim <= 0 || dstate <= 0) return SSD_ERR_INVALID_ARG;
  if (!out || (rank > 0 && (!states || !logdecay))) return SSD_ERR_INVALID_ARG;
  const int64_t n = nheads * headdim * dstate;
  if (n > ((int64_t)1 << 40)) return SSD_ERR_UNSUPPORTED;
  ssd::state_prefix_kernel<<<(unsigned)((n + 255) / 256), 256, 0, (cudaStream_t)stream>>>(
      rank, nheads, headdim * dstate, states, logdecay, init_state, out);
  ssd::count_launches(1);
  return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

// ----------------------------------------------------------- long sequences in segments
// A dense batch whose units are long enough that one unit would span several CTAs of the
// tensor-core kernel is cut into segments (the chunked algorithm one level up): a
// final-state-only pass from zero gives every segment's end state s, the segments' decays
// give each segment's true start state by the same recurrence as above, and the full pass
// runs on the segments as independent packed sequences from those states.
namespace ssd {
namespace {

// cu[j] = first token of segment j: sequence s = j / k has segments [s L + i seg, ...),
// the last one of each sequence ending at the sequence's end.
__global__ void segment_offsets_kernel(int nseq, int64_t L, int k, int64_t seg, int32_t* cu) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j > nseq * k) return;
  const int s = j / k, i = j % k;
  cu[j] = (int32_t)(s == nseq ? (int64_t)nseq * L : (int64_t)s * L + (int64_t)i * seg);
}

// part[j][z][h] = sum of dt over slice z (512 tokens) of segment j (0 past its end); grid
// (ceil(H / 32), nseg, Z).
__global__ void __launch_bounds__(kHeadsPerBlock * kTokLanes)
    segments_logdecay_kernel(const int32_t* cu, int H, int Z, const float* dt, float* part) {
  const int j = blockIdx.y;
  const int64_t t0 = (int64_t)cu[j] + (int64_t)blockIdx.z * kSliceTokens, end = cu[j + 1];
  logdecay_slice(t0, t0 + kSliceTokens < end ? t0 + kSliceTokens : end, H, dt,
                 part + ((int64_t)j * Z + blockIdx.z) * H);
}

// lam[j][h] = A[h] * sum over z of part[j][z][h], in slice order.
__global__ void segments_lam_kernel(int nseg, int H, int Z, const float* part, const float* A, float* lam) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (int64_t)nseg * H) return;
  const int64_t j = e / H, h = e % H;
  float s = 0.f;
  for (int z = 0; z < Z; ++z) s += part[(j * Z + z) * H + h];
  lam[e] = s * A[h];
}

// Start state of every segment: for each sequence s (k segments) and state element e,
// h[s k] = init[s], h[s k + i + 1] = exp(lam[s k + i]) h[s k + i] + states[s k + i];
// the last step of the recurrence is the sequence's final state (written when fin != null).
__global__ void __launch_bounds__(256) segments_prefix_kernel(int nseq, int k, int64_t H, int64_t PN,
                                                              const float* states, const float* lam,
                                                              const float* init, float* out, float* fin) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int s = blockIdx.y;
  if (e >= H * PN) return;
  const int64_t h = e / PN;
  float acc = init ? init[(int64_t)s * H * PN + e] : 0.f;
  for (int i0 = 0; i0 < k; i0 += 4) {  // the states of four segments in flight at once
    float sv[4], lv[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int64_t j = (int64_t)s * k + i0 + q;
      sv[q] = i0 + q < k ? __ldg(states + j * H * PN + e) : 0.f;
      lv[q] = i0 + q < k ? __ldg(lam + j * H + h) : 0.f;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (i0 + q >= k) break;
      out[((int64_t)s * k + i0 + q) * H * PN + e] = acc;
      acc = fmaf(expf(lv[q]), acc, sv[q]);
    }
  }
  if (fin) fin[(int64_t)s * H * PN + e] = acc;
}

}  // namespace

cudaError_t launch_segment_offsets(int nseq, int64_t L, int k, int64_t seg, int32_t* cu, cudaStream_t st) {
  const int n = nseq * k + 1;
  segment_offsets_kernel<<<(n + 255) / 256, 256, 0, st>>>(nseq, L, k, seg, cu);
  count_launches(1);
  return cudaGetLastError();
}

int segments_slices(int64_t max_len) { return (int)((max_len + kSliceTokens - 1) / kSliceTokens); }

cudaError_t launch_segments_logdecay(const int32_t* cu, int nseg, int64_t max_len, int H, const float* dt,
                                     const float* A, float* part, float* lam, cudaStream_t st) {
  const int Z = segments_slices(max_len);
  if (Z < 1 || Z > 65535 || nseg > 65535) return cudaErrorInvalidValue;
  segments_logdecay_kernel<<<dim3((H + kHeadsPerBlock - 1) / kHeadsPerBlock, nseg, (unsigned)Z),
                             kHeadsPerBlock * kTokLanes, 0, st>>>(cu, H, Z, dt, part);
  const int64_t n = (int64_t)nseg * H;
  segments_lam_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(nseg, H, Z, part, A, lam);
  count_launches(2);
  return cudaGetLastError();
}

cudaError_t launch_segments_prefix(int nseq, int k, int64_t H, int64_t PN, const float* states, const float* lam,
                                   const float* init, float* out, float* fin, cudaStream_t st) {
  segments_prefix_kernel<<<dim3((unsigned)((H * PN + 255) / 256), nseq), 256, 0, st>>>(nseq, k, H, PN, states,
                                                                                       lam, init, out, fin);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace ssd
