// ssd_simt.cu -- the general CUDA-core path of the chunked SSD forward pass.
//
// Works for every shape the API accepts (any P, N in 1..256, fp32 or bf16 I/O,
// any chunk length) and is the fp32 path, which needs full fp32 arithmetic
// (TF32 operands could not meet a 1e-4 relative error).  The four steps follow
// the chunked algorithm of "Transformers are SSMs" (wikillm.com card, Method
// step 5, sec. 6), with chunk boundaries restarted at every sequence start:
//
//   chunk_cumsum   cs = in-chunk inclusive cumsum of dt * A        (sec. 5.1, 6)
//   chunk_states   right factors: s_c = sum_t exp(cs_end - cs_t) dt_t x_t B_t^T
//   state_passing  centre factors: h_{c+1} = exp(cs_end_c) h_c + s_c, with the
//                  sequence's initial state at its first chunk; the last h is the
//                  final state
//   chunk_output   diagonal block (L o C B^T)(dt x) + left factor
//                  exp(cs_t) C_t h_c + D x_t, written in the I/O dtype
//
// Scratch: the chunk table, cs and the (Cmax, H, P, N) fp32 state buffer.
#include <algorithm>

#include "ssd_common.cuh"

namespace ssd {

// ---------------------------------------------------------------- chunk table
// One block: validates cu_seqlens (0 = c0 <= ... <= c_nseq = tokens), then lays
// out every sequence's chunks in sequence order.  On invalid input it records
// kStatusBadSeqlens and sets nchunks = -1, and every later kernel does nothing.
// The tensor-core path (seq_tiles set) needs only the prefix over 128-token tiles
// and the validity flag; the SIMT path needs the chunk prefix and chunk records.
__global__ void __launch_bounds__(1024) chunk_table_kernel(Problem pb) {
  __shared__ int s_bad;
  __shared__ int s_warp[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) s_bad = 0;
  __syncthreads();
  if (pb.cu) {
    for (int s = tid; s <= pb.nseq; s += blockDim.x) {
      const int v = pb.cu[s];
      if ((s == 0 && v != 0) || (s == pb.nseq && (int64_t)v != pb.tokens) || (s > 0 && v < pb.cu[s - 1]))
        atomicOr(&s_bad, 1);
    }
  }
  __syncthreads();
  if (s_bad) {
    if (tid == 0) {
      *pb.nchunks = -1;
      atomicOr(pb.status, kStatusBadSeqlens);
    }
    return;
  }
  const bool tc = pb.seq_tiles != nullptr;
  const int unit = tc ? kTcTile : pb.Q;
  int32_t* out = tc ? pb.seq_tiles : pb.seq_first;
  // exclusive prefix over sequences of ceil(len / unit), 1024 sequences at a time
  int carry = 0;  // the same in every thread
  for (int base = 0; base < pb.nseq; base += blockDim.x) {
    const int s = base + tid;
    int n = 0;
    if (s < pb.nseq) {
      const int64_t len = seq_off(pb, s + 1) - seq_off(pb, s);
      n = (int)((len + unit - 1) / unit);
    }
    int v = n;  // inclusive scan within the warp
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += u;
    }
    if (lane == 31) s_warp[warp] = v;
    __syncthreads();
    if (warp == 0) {
      int w = lane < (int)(blockDim.x >> 5) ? s_warp[lane] : 0;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, w, off);
        if (lane >= off) w += u;
      }
      s_warp[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    if (s < pb.nseq) out[s] = carry + (warp > 0 ? s_warp[warp - 1] : 0) + v - n;
    carry += s_warp[31];
    __syncthreads();  // s_warp is rewritten by the next round
  }
  if (tid == 0) {
    out[pb.nseq] = carry;
    *pb.nchunks = tc ? 0 : carry;  // the tensor-core path reads only the validity flag
  }
  if (tc) return;
  for (int s = tid; s < pb.nseq; s += blockDim.x) {
    const int64_t off = seq_off(pb, s), len = seq_off(pb, s + 1) - off;
    const int first = pb.seq_first[s];  // written above by this same thread
    for (int c = 0; (int64_t)c * pb.Q < len; ++c) {
      ChunkRec r;
      r.seq = s;
      r.t0 = (int32_t)(off + (int64_t)c * pb.Q);
      r.len = (int32_t)min((int64_t)pb.Q, len - (int64_t)c * pb.Q);
      r.idx = c;
      pb.chunks[first + c] = r;
    }
  }
}

cudaError_t launch_chunk_table(const Problem& pb, cudaStream_t st) {
  chunk_table_kernel<<<1, 1024, 0, st>>>(pb);
  count_launches(1);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ cumsum
// Grid (Cmax, ceil(H/8)), 8 warps; warp w scans head blockIdx.y*8 + w of one chunk.
__global__ void __launch_bounds__(256) chunk_cumsum_kernel(Problem pb) {
  const int c = blockIdx.x;
  if (c >= *pb.nchunks) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y * 8 + warp;
  if (h >= pb.H) return;
  const ChunkRec r = pb.chunks[c];
  const float Ah = pb.A[h];
  const int per = (pb.Q + 31) / 32;  // <= 8 consecutive tokens per lane
  float v[8];
  float run = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int q = lane * per + i;
    float l = 0.f;
    if (i < per && q < r.len) l = dt_value(pb, pb.dt[((int64_t)r.t0 + q) * pb.H + h], h) * Ah;
    run += l;
    v[i] = run;
  }
  // exclusive scan of the lane totals
  float incl = run;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  const float excl = incl - run;
  float* out = pb.cs + ((int64_t)c * pb.H + h) * pb.Q;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int q = lane * per + i;
    if (i < per && q < r.len) out[q] = excl + v[i];
  }
}

// ------------------------------------------------------------ chunk states
// Grid (Cmax, H, ceil(P/64) * ceil(N/64)); a 64 x 64 tile of s_c[p][n] per block,
// 4 x 4 outputs per thread, tokens staged 32 at a time.
template <typename T>
__global__ void __launch_bounds__(256) chunk_states_kernel(Problem pb) {
  const int c = blockIdx.x;
  if (c >= *pb.nchunks) return;
  const int h = blockIdx.y, g = h / pb.hpg;
  const int ntn = (pb.N + 63) / 64;
  const int p0 = (blockIdx.z / ntn) * 64, n0 = (blockIdx.z % ntn) * 64;
  const ChunkRec r = pb.chunks[c];
  const float* cs = pb.cs + ((int64_t)c * pb.H + h) * pb.Q;
  const float cs_end = cs[r.len - 1];
  const T* x = (const T*)pb.x;
  const T* Bm = (const T*)pb.B;
  __shared__ float xs[32][64 + 1];
  __shared__ float bs[32][64 + 1];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < r.len; k0 += 32) {
    for (int i = threadIdx.x; i < 32 * 64; i += 256) {
      const int k = i >> 6, col = i & 63;
      const int q = k0 + k;
      float xv = 0.f, bv = 0.f;
      if (q < r.len) {
        const int64_t t = (int64_t)r.t0 + q;
        if (p0 + col < pb.P) {
          const float w = expf(cs_end - cs[q]) * dt_value(pb, pb.dt[t * pb.H + h], h);
          xv = w * to_f(x[(t * pb.H + h) * pb.P + p0 + col]);
        }
        if (n0 + col < pb.N) bv = to_f(Bm[(t * pb.G + g) * pb.N + n0 + col]);
      }
      xs[k][col] = xv;
      bs[k][col] = bv;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < 32; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = xs[k][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = bs[k][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  float* out = pb.states + ((int64_t)c * pb.H + h) * pb.P * pb.N;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int p = p0 + ty + 16 * i, n = n0 + tx + 16 * j;
      if (p < pb.P && n < pb.N) out[(int64_t)p * pb.N + n] = acc[i][j];
    }
}

// ----------------------------------------------------------- state passing
// Grid (nseq, H, ceil(P*N/256)); one state element per thread, walking the
// sequence's chunks in order.  Replaces each chunk state by the state entering
// that chunk and writes the final state.
__global__ void __launch_bounds__(256) state_passing_kernel(Problem pb) {
  if (*pb.nchunks < 0) return;
  const int s = blockIdx.x, h = blockIdx.y;
  const int64_t PN = (int64_t)pb.P * pb.N;
  const int64_t e = (int64_t)blockIdx.z * 256 + threadIdx.x;
  if (e >= PN) return;
  float hv = pb.init ? pb.init[((int64_t)s * pb.H + h) * PN + e] : 0.f;
  const int c0 = pb.seq_first[s], c1 = pb.seq_first[s + 1];
  for (int c = c0; c < c1; ++c) {
    float* sp = pb.states + ((int64_t)c * pb.H + h) * PN + e;
    const float sc = *sp;
    *sp = hv;
    const int len = pb.chunks[c].len;
    const float ltot = pb.cs[((int64_t)c * pb.H + h) * pb.Q + len - 1];
    hv = fmaf(expf(ltot), hv, sc);
  }
  if (pb.final_state) pb.final_state[((int64_t)s * pb.H + h) * PN + e] = hv;
}

// ------------------------------------------------------------ chunk output
// Grid (Cmax * Q/64, H, ceil(P/64)): a 64-row x 64-column tile of y per block.
//   y[t] = exp(cs_t) C_t h_c^T  +  sum_{j<=t} (C_t . B_j) exp(cs_t - cs_j) dt_j x_j  +  D x_t
template <typename T>
__global__ void __launch_bounds__(256) chunk_output_kernel(Problem pb) {
  const int rtiles = pb.Q / 64;
  const int c = blockIdx.x / rtiles, rt = blockIdx.x % rtiles;
  if (c >= *pb.nchunks) return;
  const ChunkRec r = pb.chunks[c];
  const int row0 = rt * 64;
  if (row0 >= r.len) return;
  const int rows = min(64, r.len - row0);
  const int h = blockIdx.y, g = h / pb.hpg;
  const int p0 = blockIdx.z * 64;
  const T* x = (const T*)pb.x;
  const T* Bm = (const T*)pb.B;
  const T* Cm = (const T*)pb.C;
  const float* cs = pb.cs + ((int64_t)c * pb.H + h) * pb.Q;
  const float* hs = pb.states + ((int64_t)c * pb.H + h) * pb.P * pb.N;

  // As: C rows (t, n slice); Bs: B rows (j, n slice) or state rows (p, n slice);
  // Xs: x rows (j, p), aliasing As/Bs (never live at the same time); Sm: masked scores (t, j).
  __shared__ float ab_buf[2 * 64 * 33];
  __shared__ float Sm[64][65];
  float(*As)[33] = reinterpret_cast<float(*)[33]>(ab_buf);
  float(*Bs)[33] = reinterpret_cast<float(*)[33]>(ab_buf + 64 * 33);
  float(*Xs)[65] = reinterpret_cast<float(*)[65]>(ab_buf);
  __shared__ float cs_row[64], cs_col[64], dt_col[64];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  if (threadIdx.x < 64) cs_row[threadIdx.x] = threadIdx.x < rows ? cs[row0 + threadIdx.x] : 0.f;

  // left factor: acc[t][p] = sum_n C[t][n] h[p][n]
  float acc[4][4] = {};
  for (int n0 = 0; n0 < pb.N; n0 += 32) {
    for (int i = threadIdx.x; i < 64 * 32; i += 256) {
      const int rr = i >> 5, k = i & 31;
      const int n = n0 + k;
      As[rr][k] = (rr < rows && n < pb.N)
                      ? to_f(Cm[(((int64_t)r.t0 + row0 + rr) * pb.G + g) * pb.N + n])
                      : 0.f;
      Bs[rr][k] = (p0 + rr < pb.P && n < pb.N) ? hs[(int64_t)(p0 + rr) * pb.N + n] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < 32; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[ty + 16 * i][k];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[tx + 16 * j][k];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = ty + 16 * i;
    const float sc = t < rows ? expf(cs_row[t]) : 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] *= sc;
  }

  // diagonal block, column tiles 0..rt of this chunk
  for (int ct = 0; ct <= rt; ++ct) {
    const int col0 = ct * 64;
    const int cols = min(64, r.len - col0);
    __syncthreads();
    if (threadIdx.x < 64) {
      const int j = threadIdx.x;
      cs_col[j] = j < cols ? cs[col0 + j] : 0.f;
      dt_col[j] = j < cols ? dt_value(pb, pb.dt[((int64_t)r.t0 + col0 + j) * pb.H + h], h) : 0.f;
    }
    // scores S[t][j] = C_t . B_j, 4 x 4 per thread at (ty + 16 i, tx + 16 j)
    float sacc[4][4] = {};
    for (int n0 = 0; n0 < pb.N; n0 += 32) {
      __syncthreads();
      for (int i = threadIdx.x; i < 64 * 32; i += 256) {
        const int rr = i >> 5, k = i & 31;
        const int n = n0 + k;
        As[rr][k] = (rr < rows && n < pb.N)
                        ? to_f(Cm[(((int64_t)r.t0 + row0 + rr) * pb.G + g) * pb.N + n])
                        : 0.f;
        Bs[rr][k] = (rr < cols && n < pb.N)
                        ? to_f(Bm[(((int64_t)r.t0 + col0 + rr) * pb.G + g) * pb.N + n])
                        : 0.f;
      }
      __syncthreads();
#pragma unroll 8
      for (int k = 0; k < 32; ++k) {
        float a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = As[ty + 16 * i][k];
#pragma unroll
        for (int j = 0; j < 4; ++j) b[j] = Bs[tx + 16 * j][k];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) sacc[i][j] = fmaf(a[i], b[j], sacc[i][j]);
      }
    }
    // mask (before exp: only i >= j reaches the exponential) and scale by dt_j
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int tl = ty + 16 * i, jl = tx + 16 * j;
        const int tg = row0 + tl, jg = col0 + jl;
        float v = 0.f;
        if (tl < rows && jl < cols && jg <= tg) v = sacc[i][j] * expf(cs_row[tl] - cs_col[jl]) * dt_col[jl];
        Sm[tl][jl] = v;
      }
    __syncthreads();  // As/Bs reads are done before Xs overwrites them
    for (int i = threadIdx.x; i < 64 * 64; i += 256) {
      const int j = i >> 6, p = i & 63;
      Xs[j][p] = (j < cols && p0 + p < pb.P)
                     ? to_f(x[(((int64_t)r.t0 + col0 + j) * pb.H + h) * pb.P + p0 + p])
                     : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int j = 0; j < 64; ++j) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = Sm[ty + 16 * i][j];
#pragma unroll
      for (int q = 0; q < 4; ++q) b[q] = Xs[j][tx + 16 * q];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[i][q] = fmaf(a[i], b[q], acc[i][q]);
    }
  }

  // skip term and store
  T* y = (T*)pb.y;
  const float Dh = pb.D ? pb.D[h] : 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int tl = ty + 16 * i;
    if (tl >= rows) continue;
    const int64_t t = (int64_t)r.t0 + row0 + tl;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int p = p0 + tx + 16 * q;
      if (p >= pb.P) continue;
      const int64_t idx = (t * pb.H + h) * pb.P + p;
      y[idx] = from_f<T>(acc[i][q] + Dh * to_f(x[idx]));
    }
  }
}

template <typename T>
static cudaError_t launch_simt_t(const Problem& pb, cudaStream_t st) {
  int n = 0;
  if (pb.Cmax > 0) {
    chunk_cumsum_kernel<<<dim3(pb.Cmax, (pb.H + 7) / 8), 256, 0, st>>>(pb);
    const int tiles = ((pb.P + 63) / 64) * ((pb.N + 63) / 64);
    chunk_states_kernel<T><<<dim3(pb.Cmax, pb.H, tiles), 256, 0, st>>>(pb);
    n += 2;
  }
  const int64_t PN = (int64_t)pb.P * pb.N;
  state_passing_kernel<<<dim3(pb.nseq, pb.H, (unsigned)((PN + 255) / 256)), 256, 0, st>>>(pb);
  ++n;
  if (pb.Cmax > 0 && pb.y) {  // y == null: only the final states are wanted
    if (pb.prof_start) cudaEventRecord(pb.prof_start, st);
    chunk_output_kernel<T><<<dim3(pb.Cmax * (pb.Q / 64), pb.H, (pb.P + 63) / 64), 256, 0, st>>>(pb);
    if (pb.prof_stop) cudaEventRecord(pb.prof_stop, st);
    ++n;
  }
  count_launches(n);
  return cudaGetLastError();
}

cudaError_t launch_simt(const Problem& pb, cudaStream_t st) {
  return pb.bf16 ? launch_simt_t<__nv_bfloat16>(pb, st) : launch_simt_t<float>(pb, st);
}

}  // namespace ssd
