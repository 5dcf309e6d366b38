// ssd_common.cuh -- device-side problem description shared by the kernels of libssd.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ssd.h"

namespace ssd {

// Status bits OR-ed into the per-device status word by kernels.
enum : unsigned int { kStatusBadSeqlens = 1u, kStatusTimeout = 2u };

// One chunk of one sequence: tokens [t0, t0 + len) of sequence `seq`, the
// `idx`-th chunk of that sequence.  Chunks never straddle a sequence boundary:
// each sequence is cut into ceil(len / Q) chunks, the last one possibly partial.
struct ChunkRec {
  int32_t seq, t0, len, idx;
};

// Everything a launch needs, passed by value to every kernel.
struct Problem {
  int64_t tokens;  // total tokens over all sequences
  int64_t seqlen;  // dense row length (dense batches)
  int nseq, H, P, N, G, hpg, Q;
  int bf16;  // io dtype: 1 = bf16, 0 = fp32
  const void* x;
  const float* dt;
  const float* A;
  const void* B;
  const void* C;
  const float* D;     // nullable
  const float* init;  // nullable
  const int32_t* cu;  // nullable (dense batch)
  void* y;
  float* final_state;  // nullable
  unsigned int* status;
  // scratch
  ChunkRec* chunks;    // Cmax records
  int32_t* nchunks;    // number of valid records, -1 when cu_seqlens was invalid
  int32_t* seq_first;  // nseq + 1: first chunk of each sequence
  float* cs;           // (Cmax, H, Q) in-chunk inclusive cumsum of dt * A
  float* states;       // (Cmax, H, P, N) chunk states, then chunk start states
  int Cmax;
  // tensor-core path scratch
  int32_t* seq_tiles;    // nseq + 1: prefix over sequences of ceil(len / kTcTile) (packed batches)
  int dense_tiles;       // tiles per sequence of a dense batch
  float* carry;          // (ranges, 2, P, N) states handed between CTAs
  uint64_t* carry_flag;  // (ranges, 16): `epoch` once a compute warp has published its part
  uint64_t epoch;        // unique per launch, so flags left in reused scratch never match
  uint8_t* tile_w;       // weighted work split: a weight per flat tile (then 16 bytes of slack)
  uint64_t* split_flag;  // (ranges): `epoch` once a CTA has written its share of tile_w
  int weights_ready;     // tile_w already holds this problem's weights (no barrier)
  int ranges;            // CTAs of the tensor-core launch
  long long wait_limit;  // SM cycles a device-side wait may take before it gives up
  int withhold_carry;    // test hook, bits: 1 CTAs never publish the state they hand on,
                         // 2 CTA 0 never publishes its flag of the split's weight barrier
  // tensor-core launches on a column range of a wider state: this launch's state columns
  // are [n_off, n_off + N) of rows n_stride long, and y_accum adds its y to the y in memory
  int n_off, n_stride, y_accum;
  // host-side measurement hooks (events around the dominant kernel, or null)
  cudaEvent_t prof_start, prof_stop;
  // fused dt prologue (ssd_forward_dt): dt holds the raw values, see dt_value()
  int dt_prologue, dt_softplus;
  const float* dt_bias;  // (H) or null
  float dt_min, dt_max;
};

// The step size of head h from the stored value v: v itself, or with the fused prologue
// of the pages' discretisation clamp(softplus(v + dt_bias[h]), dt_min, dt_max)
// (softplus(v) = log(1 + exp(v)), evaluated as max(v, 0) + log1p(exp(-|v|))).
__device__ __forceinline__ float dt_value(const Problem& pb, float v, int h) {
  if (!pb.dt_prologue) return v;
  if (pb.dt_bias) v += pb.dt_bias[h];
  if (pb.dt_softplus) v = fmaxf(v, 0.f) + log1pf(expf(-fabsf(v)));
  return fminf(fmaxf(v, pb.dt_min), pb.dt_max);
}

__device__ __forceinline__ int64_t seq_off(const Problem& pb, int s) {
  return pb.cu ? (int64_t)pb.cu[s] : (int64_t)s * pb.seqlen;
}

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f(float v);
template <>
__device__ __forceinline__ float from_f<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// Tile length (tokens) of the tensor-core path: the UMMA M dimension.
constexpr int kTcTile = 128;

// Upper bound on the number of chunks over all sequences: sum ceil(len_s/Q) <= ceil(T/Q) + nseq.
inline int max_chunks(int64_t tokens, int nseq, int Q) { return (int)((tokens + Q - 1) / Q) + nseq; }

// Adds n to the process-wide count of kernels launched by the library.
void count_launches(int n);

// Address of the current device's status word (looked up once per device), or null.
unsigned int* device_status_word();

// ssd_forward's shape and chunk rules (and the optional host cu_seqlens check), no launch.
int check_shape(const ssd_shape* s, bool packed, int chunk);

// Launchers implemented in the kernel files.
cudaError_t launch_chunk_table(const Problem& pb, cudaStream_t st);
cudaError_t launch_simt(const Problem& pb, cudaStream_t st);
// Long sequences in segments (ssd_seqpar.cu): segment offsets of a dense batch of nseq
// sequences of L tokens cut into k segments of `seg` tokens (the last of each shorter);
// per-segment log-decays; every segment's start state and (fin != null) each sequence's
// final state, by the recurrence over its segments' zero-start end states.
cudaError_t launch_segment_offsets(int nseq, int64_t L, int k, int64_t seg, int32_t* cu, cudaStream_t st);
// Slices of 512 tokens in a segment of max_len tokens (the partial sums launch_segments_logdecay
// keeps: nseg x slices x H floats in `part`).
int segments_slices(int64_t max_len);
cudaError_t launch_segments_logdecay(const int32_t* cu, int nseg, int64_t max_len, int H, const float* dt,
                                     const float* A, float* part, float* lam, cudaStream_t st);
cudaError_t launch_segments_prefix(int nseq, int k, int64_t H, int64_t PN, const float* states, const float* lam,
                                   const float* init, float* out, float* fin, cudaStream_t st);

}  // namespace ssd
