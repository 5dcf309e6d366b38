// ssd_api.cu -- the extern "C" boundary of libssd.so: argument validation,
// path selection, stream-ordered scratch, launch sequencing and the status word.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <atomic>

#include "ssd.h"
#include "ssd_common.cuh"
#include "ssd_tc.cuh"

namespace {

// Per-device status word; kernels OR ssd::kStatus* bits into it.
__device__ unsigned int g_status_word;

constexpr int kMaxDevices = 64;
std::atomic<unsigned int*> g_status_ptr[kMaxDevices];
std::atomic<int> g_path{SSD_PATH_AUTO};
std::atomic<uint64_t> g_launches{0};
std::atomic<cudaEvent_t> g_prof_start{nullptr}, g_prof_stop{nullptr};

unsigned int* status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  unsigned int* p = g_status_ptr[dev].load();
  if (!p) {
    void* sym = nullptr;
    if (cudaGetSymbolAddress(&sym, g_status_word) != cudaSuccess) return nullptr;
    p = (unsigned int*)sym;
    g_status_ptr[dev].store(p);
  }
  return p;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

int64_t nstate_rows(const ssd_shape* s, const int32_t* cu) { return cu ? s->nseq : s->batch; }

// Host-side validation shared by every entry point.  `cu` is the (device or host)
// cu_seqlens pointer as passed by the caller; only its nullness is used here.
int validate(const ssd_shape* s, const void* x, const float* dt, const float* A, const void* B, const void* C,
             const int32_t* cu, int chunk, const void* y) {
  if (!s) return SSD_ERR_INVALID_ARG;
  if (s->batch < 0 || s->seqlen < 0 || s->nheads <= 0 || s->headdim <= 0 || s->dstate <= 0 || s->ngroups <= 0)
    return SSD_ERR_INVALID_ARG;
  if (s->io_dtype != SSD_F32 && s->io_dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
  if (cu && (s->batch != 1 || s->nseq < 1)) return SSD_ERR_INVALID_ARG;
  if (chunk != 64 && chunk != 128 && chunk != 256) return SSD_ERR_UNSUPPORTED;
  if (s->nheads % s->ngroups) return SSD_ERR_UNSUPPORTED;
  if (s->headdim > 256 || s->dstate > 256 || s->nheads > 65535) return SSD_ERR_UNSUPPORTED;
  const int64_t tokens = s->batch * s->seqlen;
  if (tokens > ((int64_t)1 << 30) || tokens * s->nheads * s->headdim > ((int64_t)1 << 40))
    return SSD_ERR_UNSUPPORTED;
  if (!A || !dt) return SSD_ERR_INVALID_ARG;
  if (tokens > 0 && (!x || !B || !C || !y)) return SSD_ERR_INVALID_ARG;
  if (s->cu_seqlens_host) {
    const int32_t* c = s->cu_seqlens_host;
    if (c[0] != 0 || (int64_t)c[s->nseq] != tokens) return SSD_ERR_BAD_SEQLENS;
    for (int64_t i = 1; i <= s->nseq; ++i)
      if (c[i] < c[i - 1]) return SSD_ERR_BAD_SEQLENS;
  }
  return SSD_OK;
}

struct Scratch {
  size_t table, seq_first, nchunks, cs, states, seq_tiles, carry, carry_flag, total;
  int ranges;
};

int device_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                 cudaSuccess)
    return 148;
  return sms;
}

Scratch scratch_layout(const ssd_shape* s, const int32_t* cu, int chunk, int path) {
  auto up = [](size_t v) { return (v + 255) & ~(size_t)255; };
  const int64_t tokens = s->batch * s->seqlen;
  const int64_t nseq = nstate_rows(s, cu);
  const int Cmax = ssd::max_chunks(tokens, (int)nseq, chunk);
  Scratch w{};
  w.table = 0;
  w.seq_first = w.table + up(sizeof(ssd::ChunkRec) * (size_t)Cmax);
  w.nchunks = w.seq_first + up(sizeof(int32_t) * (size_t)(nseq + 1));
  w.cs = w.nchunks + up(sizeof(int32_t));
  size_t cs_bytes = 0, st_bytes = 0;
  if (path == SSD_PATH_SIMT) {
    cs_bytes = up(sizeof(float) * (size_t)Cmax * s->nheads * chunk);
    st_bytes = up(sizeof(float) * (size_t)Cmax * s->nheads * s->headdim * s->dstate);
  }
  w.states = w.cs + cs_bytes;
  w.seq_tiles = w.states + st_bytes;
  w.carry = w.seq_tiles;
  w.carry_flag = w.seq_tiles;
  w.total = w.seq_tiles;
  w.ranges = 0;
  if (path == SSD_PATH_TC) {
    // one CTA per SM; each may hand a (2 heads x P x N) fp32 state and two cumsums on
    w.ranges = device_sms();
    w.carry = w.seq_tiles + up(sizeof(int32_t) * (size_t)(nseq + 1));
    w.carry_flag = w.carry + up(sizeof(float) * (size_t)w.ranges * 2 * (s->headdim * s->dstate + 1));
    w.total = w.carry_flag + up(sizeof(int32_t) * (size_t)w.ranges);
  }
  return w;
}

int select_path(const ssd_shape* s, int chunk) {
  const int want = g_path.load();
  const bool tc_ok = ssd::tc_supports(s, chunk);
  if (want == SSD_PATH_SIMT) return SSD_PATH_SIMT;
  if (want == SSD_PATH_TC) return tc_ok ? SSD_PATH_TC : -SSD_ERR_UNSUPPORTED;
  return tc_ok ? SSD_PATH_TC : SSD_PATH_SIMT;
}

int forward_impl(const ssd_shape* s, const void* x, const float* dt, const float* A, const void* B, const void* C,
                 const float* D, const float* init, const int32_t* cu, int chunk, void* y, float* fin,
                 cudaStream_t st) {
  int rc = validate(s, x, dt, A, B, C, cu, chunk, y);
  if (rc) return rc;
  const void* ptrs[] = {x, dt, A, B, C, D, init, cu, y, fin};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return SSD_ERR_MISALIGNED;
  const int path = select_path(s, chunk);
  if (path < 0) return -path;
  const int64_t tokens = s->batch * s->seqlen;
  const int64_t nseq = nstate_rows(s, cu);
  if (nseq == 0) return SSD_OK;
  unsigned int* status = status_ptr();
  if (!status) return SSD_ERR_CUDA;

  ssd::Problem pb{};
  pb.tokens = tokens;
  pb.seqlen = s->seqlen;
  pb.nseq = (int)nseq;
  pb.H = (int)s->nheads;
  pb.P = (int)s->headdim;
  pb.N = (int)s->dstate;
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
  pb.init = init;
  pb.cu = cu;
  pb.y = y;
  pb.final_state = fin;
  pb.status = status;
  pb.Cmax = ssd::max_chunks(tokens, (int)nseq, chunk);
  pb.prof_start = g_prof_start.load();
  pb.prof_stop = g_prof_stop.load();
  if (!pb.prof_start || !pb.prof_stop) pb.prof_start = pb.prof_stop = nullptr;

  const Scratch w = scratch_layout(s, cu, chunk, path);
  char* ws = nullptr;
  if (cudaMallocAsync((void**)&ws, w.total, st) != cudaSuccess) return SSD_ERR_CUDA;
  pb.chunks = (ssd::ChunkRec*)(ws + w.table);
  pb.seq_first = (int32_t*)(ws + w.seq_first);
  pb.nchunks = (int32_t*)(ws + w.nchunks);
  pb.cs = (float*)(ws + w.cs);
  pb.states = (float*)(ws + w.states);
  pb.seq_tiles = path == SSD_PATH_TC ? (int32_t*)(ws + w.seq_tiles) : nullptr;
  pb.carry = (float*)(ws + w.carry);
  pb.carry_flag = (int32_t*)(ws + w.carry_flag);
  pb.ranges = w.ranges;

  cudaError_t e = ssd::launch_chunk_table(pb, st);
  if (e == cudaSuccess) e = path == SSD_PATH_TC ? ssd::launch_tc(pb, st) : ssd::launch_simt(pb, st);
  const cudaError_t e2 = cudaFreeAsync(ws, st);
  return (e != cudaSuccess || e2 != cudaSuccess) ? SSD_ERR_CUDA : SSD_OK;
}

}  // namespace

namespace ssd {
void count_launches(int n) { g_launches.fetch_add((uint64_t)n); }
unsigned int* device_status_word() { return status_ptr(); }
int check_shape(const ssd_shape* s, bool packed, int chunk) {
  const void* f = (const void*)16;  // stands for every required pointer: only shapes are checked
  return validate(s, f, (const float*)f, (const float*)f, f, f, packed ? (const int32_t*)f : nullptr, chunk, f);
}
}  // namespace ssd

extern "C" {

int ssd_forward(const ssd_shape* shape, const void* x, const float* dt, const float* A, const void* B,
                const void* C, const float* D, const float* init_state, const int32_t* cu_seqlens, int chunk,
                void* y, float* final_state, ssd_stream_t stream) {
  return forward_impl(shape, x, dt, A, B, C, D, init_state, cu_seqlens, chunk, y, final_state,
                      (cudaStream_t)stream);
}

int ssd_forward_host(const ssd_shape* s, const void* x, const float* dt, const float* A, const void* B,
                     const void* C, const float* D, const float* init_state, const int32_t* cu_seqlens, int chunk,
                     void* y, float* final_state, ssd_stream_t stream) {
  int rc = validate(s, x, dt, A, B, C, cu_seqlens, chunk, y);
  if (rc) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  const int64_t tokens = s->batch * s->seqlen;
  const int64_t nseq = nstate_rows(s, cu_seqlens);
  const size_t es = s->io_dtype == SSD_BF16 ? 2 : 4;
  const size_t H = (size_t)s->nheads, P = (size_t)s->headdim, N = (size_t)s->dstate, G = (size_t)s->ngroups;
  const size_t bytes[10] = {
      (size_t)tokens * H * P * es,                 // x
      (size_t)tokens * H * 4,                      // dt
      H * 4,                                       // A
      (size_t)tokens * G * N * es,                 // B
      (size_t)tokens * G * N * es,                 // C
      D ? H * 4 : 0,                               // D
      init_state ? (size_t)nseq * H * P * N * 4 : 0,  // init
      cu_seqlens ? (size_t)(nseq + 1) * 4 : 0,     // cu_seqlens
      (size_t)tokens * H * P * es,                 // y
      final_state ? (size_t)nseq * H * P * N * 4 : 0,  // final
  };
  const void* hin[8] = {x, dt, A, B, C, D, init_state, cu_seqlens};
  void* dev[10] = {};
  auto cleanup = [&]() {
    for (void* p : dev)
      if (p) cudaFreeAsync(p, st);
  };
  for (int i = 0; i < 10; ++i) {
    if (!bytes[i]) continue;
    if (cudaMallocAsync(&dev[i], bytes[i], st) != cudaSuccess) {
      cleanup();
      return SSD_ERR_CUDA;
    }
  }
  for (int i = 0; i < 8; ++i) {
    if (!bytes[i]) continue;
    if (cudaMemcpyAsync(dev[i], hin[i], bytes[i], cudaMemcpyHostToDevice, st) != cudaSuccess) {
      cleanup();
      return SSD_ERR_CUDA;
    }
  }
  ssd_shape sd = *s;
  sd.cu_seqlens_host = nullptr;  // validated above
  rc = forward_impl(&sd, dev[0], (const float*)dev[1], (const float*)dev[2], dev[3], dev[4],
                    (const float*)dev[5], (const float*)dev[6], (const int32_t*)dev[7], chunk, dev[8],
                    (float*)dev[9], st);
  if (rc == SSD_OK && bytes[8] && cudaMemcpyAsync(y, dev[8], bytes[8], cudaMemcpyDeviceToHost, st) != cudaSuccess)
    rc = SSD_ERR_CUDA;
  if (rc == SSD_OK && bytes[9] &&
      cudaMemcpyAsync(final_state, dev[9], bytes[9], cudaMemcpyDeviceToHost, st) != cudaSuccess)
    rc = SSD_ERR_CUDA;
  cleanup();
  if (cudaStreamSynchronize(st) != cudaSuccess) return SSD_ERR_CUDA;
  if (rc != SSD_OK) return rc;
  return ssd_query_status(stream);
}

size_t ssd_workspace_bytes(const ssd_shape* shape, int chunk) {
  if (!shape) return 0;
  const int path = select_path(shape, chunk);
  if (path < 0) return 0;
  // Upper bound over both readings of the shape (dense rows or packed sequences).
  ssd_shape s = *shape;
  s.nseq = s.nseq > s.batch ? s.nseq : s.batch;
  return scratch_layout(&s, (const int32_t*)&s, chunk, path).total;
}

int ssd_query_status(ssd_stream_t stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return SSD_ERR_CUDA;
  unsigned int* p = status_ptr();
  if (!p) return SSD_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return SSD_ERR_CUDA;
  if (v) {
    const unsigned int zero = 0;
    if (cudaMemcpy(p, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return SSD_ERR_CUDA;
  }
  if (v & ssd::kStatusBadSeqlens) return SSD_ERR_BAD_SEQLENS;
  if (v & ssd::kStatusTimeout) return SSD_ERR_DEVICE_TIMEOUT;
  return SSD_OK;
}

const char* ssd_status_string(int status) {
  switch (status) {
    case SSD_OK: return "ok";
    case SSD_ERR_INVALID_ARG: return "invalid argument";
    case SSD_ERR_UNSUPPORTED: return "unsupported shape or chunk length";
    case SSD_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case SSD_ERR_CUDA: return "CUDA runtime error";
    case SSD_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait gave up";
    case SSD_ERR_BAD_SEQLENS: return "cu_seqlens must be 0 = c0 <= c1 <= ... <= c_nseq = seqlen";
    case SSD_ERR_SCRATCH_LIMIT: return "shape needs more scratch than SSD_NOALLOC_SCRATCH_BYTES";
    default: return "unknown status";
  }
}

int ssd_set_path(int path) {
  if (path != SSD_PATH_AUTO && path != SSD_PATH_SIMT && path != SSD_PATH_TC) return -SSD_ERR_INVALID_ARG;
  return g_path.exchange(path);
}

int ssd_profile_dominant(ssd_event_t start, ssd_event_t stop) {
  g_prof_start.store((cudaEvent_t)start);
  g_prof_stop.store((cudaEvent_t)stop);
  return SSD_OK;
}

uint64_t ssd_kernel_launch_count(void) { return g_launches.load(); }

int ssd_select_path(const ssd_shape* shape, int chunk) {
  const int rc = validate(shape, (const void*)16, (const float*)16, (const float*)16, (const void*)16,
                          (const void*)16, shape && shape->cu_seqlens_host ? (const int32_t*)16 : nullptr, chunk,
                          (const void*)16);
  if (rc) return -rc;
  return select_path(shape, chunk);
}

}  // extern "C"
