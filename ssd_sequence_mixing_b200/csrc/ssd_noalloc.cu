// ssd_noalloc.cu -- ssd_forward_noalloc: the SIMT path with its scratch in a
// file-scope device array, for callers that cannot allocate device memory (a
// caller that owns the GPU's memory through its own pool cannot let a library
// call cudaMallocAsync).  The kernels are the SIMT path's, unchanged; only where
// their scratch lives differs.
#include <cuda_runtime.h>
#include <stdint.h>

#include "ssd.h"
#include "ssd_common.cuh"

namespace {

// Scratch of every ssd_forward_noalloc call.  Each GPU that loads the library
// holds these SSD_NOALLOC_SCRATCH_BYTES until the process exits.  In host code
// this name is a host-side stand-in, not a device address: kernels get the
// address looked up by scratch_base().
static __device__ __align__(256) unsigned char g_noalloc_scratch[SSD_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device, looked up on every call
// (with that device current), so that a context recreated after a device reset is
// never handed an address from the old one.  The lookup allocates nothing.
unsigned char* scratch_base() {
  void* sym = nullptr;
  if (cudaGetSymbolAddress(&sym, g_noalloc_scratch) != cudaSuccess || !sym) return nullptr;
  return (unsigned char*)sym;
}

size_t up256(size_t v) { return (v + 255) & ~(size_t)255; }

}  // namespace

extern "C" int ssd_forward_noalloc(const ssd_shape* s, const void* x, const float* dt, const float* A,
                                   const void* B, const void* C, const float* D, const float* init_state,
                                   const int32_t* cu, int chunk, void* y, float* fin, ssd_stream_t stream) {
  // Shape and chunk rules are ssd_forward's.
  const int rc = ssd::check_shape(s, cu != nullptr, chunk);
  if (rc) return rc;
  const int64_t tokens = s->batch * s->seqlen;
  if (!A || (tokens > 0 && (!x || !dt || !B || !C || !y))) return SSD_ERR_INVALID_ARG;  // as ssd_forward
  const void* ptrs[] = {x, dt, A, B, C, D, init_state, cu, y, fin};
  for (const void* p : ptrs)
    if (p && ((uintptr_t)p & 15u)) return SSD_ERR_MISALIGNED;
  const int64_t nseq = cu ? s->nseq : s->batch;
  if (nseq == 0) return SSD_OK;

  // Scratch layout of the SIMT path, carved from the static array.
  const int H = (int)s->nheads, P = (int)s->headdim, N = (int)s->dstate;
  const int Cmax = ssd::max_chunks(tokens, (int)nseq, chunk);
  const size_t off_table = 0;
  const size_t off_first = off_table + up256(sizeof(ssd::ChunkRec) * (size_t)Cmax);
  const size_t off_count = off_first + up256(sizeof(int32_t) * (size_t)(nseq + 1));
  const size_t off_cs = off_count + up256(sizeof(int32_t));
  const size_t off_states = off_cs + up256(sizeof(float) * (size_t)Cmax * H * chunk);
  const size_t total = off_states + up256(sizeof(float) * (size_t)Cmax * H * P * N);
  if (total > (size_t)SSD_NOALLOC_SCRATCH_BYTES) return SSD_ERR_SCRATCH_LIMIT;

  unsigned char* base = scratch_base();
  unsigned int* status = ssd::device_status_word();
  if (!base || !status) return SSD_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;

  ssd::Problem pb{};
  pb.tokens = tokens;
  pb.seqlen = s->seqlen;
  pb.nseq = (int)nseq;
  pb.H = H;
  pb.P = P;
  pb.N = N;
  pb.G = (int)s->ngroups;
  pb.hpg = pb.H / pb.G;
  pb.Q = chunk;
  pb.bf16 = s->io_dtype == SSD_BF16;
  pb.x = x;
  pb.dt = dt;
  pb.A = A;
  pb.B = B;
  pb.C = C;
  pb.D = D;
  pb.init = init_state;
  pb.cu = cu;
  pb.y = y;
  pb.final_state = fin;
  pb.status = status;
  pb.Cmax = Cmax;
  pb.chunks = (ssd::ChunkRec*)(base + off_table);
  pb.seq_first = (int32_t*)(base + off_first);
  pb.nchunks = (int32_t*)(base + off_count);
  pb.cs = (float*)(base + off_cs);
  pb.states = (float*)(base + off_states);

  // The array keeps the previous call's contents.  Every scratch word a kernel reads
  // is written earlier in this call, except the chunk count, which is reset here to
  // "no valid table" (-1) so later kernels do nothing if the table is never built.
  if (cudaMemsetAsync(pb.nchunks, 0xFF, sizeof(int32_t), st) != cudaSuccess) return SSD_ERR_CUDA;
  cudaError_t e = ssd::launch_chunk_table(pb, st);
  if (e == cudaSuccess) e = ssd::launch_simt(pb, st);
  return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
