// ssd_api.cu -- the extern "C" boundary of libssd.so: argument validation,
// path selection, stream-ordered scratch, launch sequencing and the status word.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <chrono>
#include <mutex>
#include <vector>

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
// Device-side waits give up after this many SM cycles (about 2 s at the B200's clock).
constexpr long long kDefaultWaitLimit = 4ll << 30;
std::atomic<long long> g_wait_limit{kDefaultWaitLimit};
std::atomic<int> g_withhold_carry{0};

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

// A value no earlier launch of this process used: the tensor-core kernel's carry flags
// are set to it, so flags left over in reused scratch never look published.  The high
// half is drawn from the address of a stack variable and the clock once per process.
uint64_t next_epoch() {
  static std::atomic<uint64_t> counter{0};
  static const uint64_t salt = [] {
    int probe = 0;
    uint64_t v = (uint64_t)(uintptr_t)&probe ^ (uint64_t)std::chrono::steady_clock::now().time_since_epoch().count();
    v ^= v >> 29;
    v *= 0xbf58476d1ce4e5b9ull;
    v ^= v >> 32;
    return v << 32;
  }();
  return salt | ((counter.fetch_add(1) + 1) & 0xffffffffull);
}

// The library's stream-ordered pool on the current device: scratch and the host entry
// point's device buffers come from it, and freed blocks stay cached for the next call
// (release threshold: never), so repeated calls do not go back to the driver.
std::atomic<cudaMemPool_t> g_pool[kMaxDevices];
cudaMemPool_t lib_pool() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  cudaMemPool_t p = g_pool[dev].load();
  if (p) return p;
  cudaMemPoolProps props{};
  props.allocType = cudaMemAllocationTypePinned;
  props.location.type = cudaMemLocationTypeDevice;
  props.location.id = dev;
  if (cudaMemPoolCreate(&p, &props) != cudaSuccess) return nullptr;
  uint64_t keep = UINT64_MAX;
  cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &keep);
  cudaMemPool_t expected = nullptr;
  if (!g_pool[dev].compare_exchange_strong(expected, p)) {
    cudaMemPoolDestroy(p);
    p = expected;
  }
  return p;
}

cudaError_t pool_alloc(void** ptr, size_t bytes, cudaStream_t st) {
  cudaMemPool_t pool = lib_pool();
  if (!pool) return cudaErrorMemoryAllocation;
  return cudaMallocFromPoolAsync(ptr, bytes, pool, st);
}

int64_t nstate_rows(const ssd_shape* s, const int32_t* cu) { return cu ? s->nseq : s->batch; }

// Host-side validation shared by every entry point.  `cu` is the (device or host)
// cu_seqlens pointer as passed by the caller; only its nullness is used here.
int validate(const ssd_shape* s, const void* x, const float* dt, const float* A, const void* B, const void* C,
             const int32_t* cu, int chunk, const void* y, bool state_only = false) {
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
  if (!A) return SSD_ERR_INVALID_ARG;
  if (tokens > 0 && (!x || !dt || !B || (!state_only && (!C || !y)))) return SSD_ERR_INVALID_ARG;  // empty inputs may be NULL
  if (s->cu_seqlens_host) {
    const int32_t* c = s->cu_seqlens_host;
    if (c[0] != 0 || (int64_t)c[s->nseq] != tokens) return SSD_ERR_BAD_SEQLENS;
    for (int64_t i = 1; i <= s->nseq; ++i)
      if (c[i] < c[i - 1]) return SSD_ERR_BAD_SEQLENS;
  }
  return SSD_OK;
}

struct Scratch {
  size_t table, seq_first, nchunks, cs, states, seq_tiles, carry, carry_flag, split_flag, tile_w, total;
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
  w.carry = w.carry_flag = w.split_flag = w.tile_w = w.seq_tiles;
  w.total = w.seq_tiles;
  w.ranges = 0;
  if (path == SSD_PATH_TC) {
    // one CTA per SM; each may hand a (2 heads x P x N) fp32 state on, with one flag per
    // compute warp (16)
    w.ranges = device_sms();
    w.carry = w.seq_tiles + up(sizeof(int32_t) * (size_t)(nseq + 1));
    w.carry_flag = w.carry + up(sizeof(float) * (size_t)w.ranges * 2 * s->headdim * s->dstate);
    // the weighted split: a byte per flat tile (at most ceil(tokens / 128) + nseq tiles
    // per head pair), with slack for 16-byte loads
    const int64_t flat = (cu ? (tokens + ssd::kTcTile - 1) / ssd::kTcTile + nseq
                             : s->batch * ((s->seqlen + ssd::kTcTile - 1) / ssd::kTcTile)) *
                         (s->nheads / 2);
    // one flag per CTA for the barrier after the split's weights
    w.split_flag = w.carry_flag + up(sizeof(uint64_t) * 16 * (size_t)w.ranges);
    w.tile_w = w.split_flag + up(sizeof(uint64_t) * (size_t)w.ranges);
    w.total = w.tile_w + up((size_t)flat + 16);
  }
  return w;
}

// ssd_forward_host's two copy streams (in, out) and its events, one set per device,
// created on first use and kept for the life of the process.
constexpr int kHostGroups = 8;
struct HostCopies {
  std::mutex mu;
  bool ready = false;
  cudaStream_t sin = nullptr, sout = nullptr;
  cudaEvent_t ev[2 * kHostGroups + 1] = {};
  bool create() {
    if (cudaStreamCreateWithFlags(&sin, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&sout, cudaStreamNonBlocking) != cudaSuccess)
      return false;
    for (auto& e : ev)
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return false;
    ready = true;
    return true;
  }
};
HostCopies g_host_copies[kMaxDevices];
HostCopies* host_copies() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  return &g_host_copies[dev];
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
                 cudaStream_t st, const ssd_dt_prologue* pro = nullptr);

// Segments per sequence for a dense batch on the tensor-core path.  Its CTAs cut the flat
// tile list into equal ranges; a unit (sequence, head pair) much longer than a range is
// processed range after range, each CTA waiting for the state of the one before (at the
// (2, 65536) length-sweep point a unit is 2.3 ranges long and the kernel takes the time of
// a whole unit).  Cutting each sequence into k segments of at most a range's length and
// passing the state between segments as the chunked algorithm passes it between chunks
// costs one final-state-only pass (x, dt and B again) and removes the wait.
int segments_for(const ssd_shape* s, int path, const int32_t* cu, const ssd_dt_prologue* pro) {
  if (path != SSD_PATH_TC || cu || pro || s->batch < 1 || s->seqlen <= 0) return 1;
  const int64_t tiles = (s->seqlen + ssd::kTcTile - 1) / ssd::kTcTile;
  const int64_t units = s->batch * (s->nheads / 2);
  // tiles per CTA (at least one: with fewer tiles than SMs every CTA takes one)
  const int64_t share = std::max<int64_t>(1, units * tiles / std::max(1, device_sms()));
  if (2 * tiles <= 3 * share) return 1;
  const int64_t k0 = (tiles + share - 1) / share;         // segments of at most one share ...
  const int64_t seg_tiles = (tiles + k0 - 1) / k0;        // ... of whole tiles
  const int64_t k = (tiles + seg_tiles - 1) / seg_tiles;
  if (k < 2 || s->batch * k > (1 << 20)) return 1;
  return (int)k;
}

int forward_segmented(const ssd_shape* s, int k, const void* x, const float* dt, const float* A, const void* B,
                      const void* C, const float* D, const float* init, int chunk, void* y, float* fin,
                      cudaStream_t st) {
  const int64_t L = s->seqlen, tiles = (L + ssd::kTcTile - 1) / ssd::kTcTile;
  const int64_t seg = (tiles + k - 1) / k * ssd::kTcTile;  // tokens per segment, whole tiles
  k = (int)((L + seg - 1) / seg);
  const int nseq = (int)s->batch, nseg = nseq * k;
  const int64_t H = s->nheads, PN = s->headdim * s->dstate, HPN = H * PN;
  auto up = [](size_t v) { return (v + 255) & ~(size_t)255; };
  const int Z = ssd::segments_slices(seg);
  const size_t o_cu = 0, o_st = up(sizeof(int32_t) * (nseg + 1)), o_lam = o_st + up(sizeof(float) * nseg * HPN),
               o_part = o_lam + up(sizeof(float) * nseg * H), o_h = o_part + up(sizeof(float) * nseg * Z * H),
               total = o_h + up(sizeof(float) * nseg * HPN);
  char* ws = nullptr;
  if (pool_alloc((void**)&ws, total, st) != cudaSuccess) return SSD_ERR_CUDA;
  int32_t* cu = (int32_t*)(ws + o_cu);
  float *states = (float*)(ws + o_st), *lam = (float*)(ws + o_lam), *h_in = (float*)(ws + o_h);
  float* part = (float*)(ws + o_part);
  ssd_shape sg = *s;
  sg.batch = 1;
  sg.seqlen = s->batch * L;
  sg.nseq = nseg;
  sg.cu_seqlens_host = nullptr;
  int rc = SSD_OK;
  if (ssd::launch_segment_offsets(nseq, L, k, seg, cu, st) != cudaSuccess) rc = SSD_ERR_CUDA;
  // 1. every segment's end state from a zero state (x, dt, B only)
  if (rc == SSD_OK) rc = forward_impl(&sg, x, dt, A, B, nullptr, nullptr, nullptr, cu, chunk, nullptr, states, st);
  // 2. the segments' decays, true start states and the sequences' final states
  if (rc == SSD_OK && (ssd::launch_segments_logdecay(cu, nseg, seg, (int)H, dt, A, part, lam, st) != cudaSuccess ||
                       ssd::launch_segments_prefix(nseq, k, H, PN, states, lam, init, h_in, fin, st) != cudaSuccess))
    rc = SSD_ERR_CUDA;
  // 3. the full pass on the segments from their start states (y only)
  if (rc == SSD_OK && y) rc = forward_impl(&sg, x, dt, A, B, C, D, h_in, cu, chunk, y, nullptr, st);
  if (cudaFreeAsync(ws, st) != cudaSuccess && rc == SSD_OK) rc = SSD_ERR_CUDA;
  return rc;
}

int forward_impl(const ssd_shape* s, const void* x, const float* dt, const float* A, const void* B, const void* C,
                 const float* D, const float* init, const int32_t* cu, int chunk, void* y, float* fin,
                 cudaStream_t st, const ssd_dt_prologue* pro) {
  // y == NULL: only the final states are computed (C and D are not read)
  const bool state_only = y == nullptr && fin != nullptr;
  int rc = validate(s, x, dt, A, B, C, cu, chunk, y, state_only);
  if (rc) return rc;
  if (state_only) C = nullptr, D = nullptr;
  if (pro && !(pro->dt_min >= 0.f && pro->dt_max >= pro->dt_min)) return SSD_ERR_INVALID_ARG;  // NaN fails too
  const void* ptrs[] = {x, dt, A, B, C, D, init, cu, y, fin, pro ? pro->dt_bias : nullptr};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return SSD_ERR_MISALIGNED;
  const int path = select_path(s, chunk);
  if (path < 0) return -path;
  const int64_t tokens = s->batch * s->seqlen;
  const int64_t nseq = nstate_rows(s, cu);
  if (nseq == 0) return SSD_OK;
  unsigned int* status = status_ptr();
  if (!status) return SSD_ERR_CUDA;
  {
    const int k = segments_for(s, path, cu, pro);
    if (k > 1) return forward_segmented(s, k, x, dt, A, B, C, D, init, chunk, y, fin, st);
  }

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
  if (pro) {
    pb.dt_prologue = 1;
    pb.dt_softplus = pro->softplus != 0;
    pb.dt_bias = pro->dt_bias;
    pb.dt_min = pro->dt_min;
    pb.dt_max = pro->dt_max;
  }
  pb.prof_start = g_prof_start.load();
  pb.prof_stop = g_prof_stop.load();
  if (!pb.prof_start || !pb.prof_stop) pb.prof_start = pb.prof_stop = nullptr;

  const Scratch w = scratch_layout(s, cu, chunk, path);
  char* ws = nullptr;
  if (pool_alloc((void**)&ws, w.total, st) != cudaSuccess) return SSD_ERR_CUDA;
  pb.chunks = (ssd::ChunkRec*)(ws + w.table);
  pb.seq_first = (int32_t*)(ws + w.seq_first);
  pb.nchunks = (int32_t*)(ws + w.nchunks);
  pb.cs = (float*)(ws + w.cs);
  pb.states = (float*)(ws + w.states);
  pb.seq_tiles = path == SSD_PATH_TC ? (int32_t*)(ws + w.seq_tiles) : nullptr;
  pb.dense_tiles = (int)((s->seqlen + ssd::kTcTile - 1) / ssd::kTcTile);
  pb.carry = (float*)(ws + w.carry);
  pb.carry_flag = (uint64_t*)(ws + w.carry_flag);
  pb.tile_w = (uint8_t*)(ws + w.tile_w);
  pb.split_flag = (uint64_t*)(ws + w.split_flag);
  pb.epoch = next_epoch();
  pb.ranges = w.ranges;
  pb.wait_limit = g_wait_limit.load();
  if (path == SSD_PATH_TC && pb.wait_limit == kDefaultWaitLimit) {
    // A CTA whose range lies inside one unit waits for the CTA before it to finish its
    // range, and every role of the CTA waits behind it; along a chain of such CTAs the
    // wait grows with the work ahead.  Allow 16K cycles (about 8 us, several times the
    // measured cost) per tile of the whole problem on top of the default.
    const int64_t tiles = (tokens / ssd::kTcTile + nseq) * ((s->nheads + 1) / 2);
    pb.wait_limit += (long long)tiles * 16384;
  }
  pb.withhold_carry = g_withhold_carry.load();

  // The chunk table: the SIMT path's chunk records, or the tensor-core path's tile
  // prefix over packed sequences (a dense batch needs none).
  cudaError_t e = cudaSuccess;
  if (path == SSD_PATH_SIMT || cu) e = ssd::launch_chunk_table(pb, st);
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

int ssd_forward_dt(const ssd_shape* shape, const ssd_dt_prologue* prologue, const void* x, const float* dt_raw,
                   const float* A, const void* B, const void* C, const float* D, const float* init_state,
                   const int32_t* cu_seqlens, int chunk, void* y, float* final_state, ssd_stream_t stream) {
  return forward_impl(shape, x, dt_raw, A, B, C, D, init_state, cu_seqlens, chunk, y, final_state,
                      (cudaStream_t)stream, prologue);
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
  const size_t tok_x = H * P * es, tok_dt = H * 4, tok_bc = G * N * es, seq_state = H * P * N * 4;
  if (cu_seqlens && s->cu_seqlens_host != cu_seqlens) {  // the host array is the one to check
    ssd_shape chk = *s;
    chk.cu_seqlens_host = cu_seqlens;
    if ((rc = validate(&chk, x, dt, A, B, C, cu_seqlens, chunk, y))) return rc;
  }
  auto seq_start = [&](int64_t q) -> int64_t { return cu_seqlens ? cu_seqlens[q] : q * s->seqlen; };

  // Whole sequences in up to kGroups groups of about equal token counts: group g's
  // inputs are copied in while group g-1 computes and group g-2's outputs go out.
  constexpr int kGroups = kHostGroups;
  std::vector<int64_t> gs{0};
  for (int g = 1; g <= kGroups && gs.back() < nseq; ++g) {
    const int64_t target = tokens * g / kGroups;
    int64_t q = gs.back() + 1;
    while (q < nseq && seq_start(q) < target) ++q;
    gs.push_back(g == kGroups ? nseq : q);
  }
  if (gs.back() < nseq) gs.back() = nseq;
  const int ng = (int)gs.size() - 1;

  // Device buffers for the whole problem.  Each group's slice of a per-token or
  // per-sequence array starts on a 256-byte boundary (the kernels need 16).
  auto up = [](size_t v) { return (v + 255) & ~(size_t)255; };
  std::vector<size_t> seq_off(ng + 1, 0), cu_off(ng + 1, 0);
  for (int g = 0; g < ng; ++g) {
    const int64_t q0 = gs[g], q1 = gs[g + 1];
    seq_off[g + 1] = seq_off[g] + up((size_t)(q1 - q0) * seq_state);
    cu_off[g + 1] = cu_off[g] + ((size_t)(q1 - q0 + 1 + 63) & ~(size_t)63);  // int32 entries
  }
  // per-token arrays: the group's first token index in a padded token space, so that
  // every slice is aligned for every per-token row size
  std::vector<int64_t> ptok(ng + 1, 0);
  for (int g = 0; g < ng; ++g) {
    const int64_t nt = (gs[g + 1] < nseq ? seq_start(gs[g + 1]) : tokens) - seq_start(gs[g]);
    ptok[g + 1] = ptok[g] + ((nt + 255) & ~(int64_t)255);
  }
  const int64_t ptokens = ptok[ng];
  const size_t bytes[11] = {
      (size_t)ptokens * tok_x,                                 // x
      (size_t)ptokens * tok_dt,                                // dt
      H * 4,                                                   // A
      (size_t)ptokens * tok_bc,                                // B
      (size_t)ptokens * tok_bc,                                // C
      D ? H * 4 : 0,                                           // D
      init_state ? seq_off[ng] : 0,                            // init
      cu_seqlens ? cu_off[ng] * 4 : 0,                         // each group's cu_seqlens from 0
      (size_t)ptokens * tok_x,                                 // y
      final_state ? seq_off[ng] : 0,                           // final
      0,
  };
  void* dev[11] = {};
  // the device's copy streams and events, created once; calls on one device take turns
  HostCopies* hc = host_copies();
  if (!hc) return SSD_ERR_CUDA;
  std::lock_guard<std::mutex> lock(hc->mu);
  if (!hc->ready && !hc->create()) return SSD_ERR_CUDA;
  cudaStream_t sin = hc->sin, sout = hc->sout;
  cudaEvent_t* ev = hc->ev;
  auto cleanup = [&]() {
    cudaStreamSynchronize(sin);
    cudaStreamSynchronize(sout);
    for (void* p : dev)
      if (p) cudaFreeAsync(p, st);
  };
  auto fail = [&](int code) {
    cleanup();
    cudaStreamSynchronize(st);
    return code;
  };
  for (int i = 0; i < 10; ++i)
    if (bytes[i] && pool_alloc(&dev[i], bytes[i], st) != cudaSuccess) return fail(SSD_ERR_CUDA);
  // the buffers were taken on `st`: the copy streams start after that
  if (cudaEventRecord(ev[2 * ng], st) != cudaSuccess || cudaStreamWaitEvent(sin, ev[2 * ng], 0) != cudaSuccess ||
      cudaStreamWaitEvent(sout, ev[2 * ng], 0) != cudaSuccess)
    return fail(SSD_ERR_CUDA);

  std::vector<int32_t> cu_groups;  // host copy of each group's cu_seqlens, rebased to 0
  if (cu_seqlens) {
    cu_groups.assign(cu_off[ng], 0);
    for (int g = 0; g < ng; ++g)
      for (int64_t q = gs[g]; q <= gs[g + 1]; ++q)
        cu_groups[cu_off[g] + (q - gs[g])] = cu_seqlens[q] - cu_seqlens[gs[g]];
  }
  auto h2d = [&](void* d, const void* h, size_t n) {
    return n == 0 || cudaMemcpyAsync(d, h, n, cudaMemcpyHostToDevice, sin) == cudaSuccess;
  };
  auto d2h = [&](void* h, const void* d, size_t n) {
    return n == 0 || cudaMemcpyAsync(h, d, n, cudaMemcpyDeviceToHost, sout) == cudaSuccess;
  };
  if (!h2d(dev[2], A, bytes[2]) || !h2d(dev[5], D, bytes[5]) ||
      (cu_seqlens && !h2d(dev[7], cu_groups.data(), bytes[7])))
    return fail(SSD_ERR_CUDA);
  if (cu_seqlens && cudaStreamSynchronize(sin) != cudaSuccess) return fail(SSD_ERR_CUDA);  // pageable source

  auto at = [](void* base, size_t off) { return base ? (void*)((char*)base + off) : nullptr; };
  auto group_tokens = [&](int g, int64_t& t0, int64_t& nt) {
    t0 = seq_start(gs[g]);
    nt = (gs[g + 1] < nseq ? seq_start(gs[g + 1]) : tokens) - t0;
  };
  // Every group's inputs are queued on the input stream first, so the copies run back to
  // back at the link's speed whatever the host takes to queue the groups' kernels.
  for (int g = 0; g < ng; ++g) {
    const int64_t q0 = gs[g], q1 = gs[g + 1];
    int64_t t0, nt;
    group_tokens(g, t0, nt);
    const size_t p0 = (size_t)ptok[g];  // first token of the group in the device buffers
    if (!h2d(at(dev[0], p0 * tok_x), (const char*)x + t0 * tok_x, nt * tok_x) ||
        !h2d(at(dev[1], p0 * tok_dt), (const char*)dt + t0 * tok_dt, nt * tok_dt) ||
        !h2d(at(dev[3], p0 * tok_bc), (const char*)B + t0 * tok_bc, nt * tok_bc) ||
        !h2d(at(dev[4], p0 * tok_bc), (const char*)C + t0 * tok_bc, nt * tok_bc) ||
        (init_state && !h2d(at(dev[6], seq_off[g]), (const char*)init_state + q0 * seq_state,
                            (q1 - q0) * seq_state)) ||
        cudaEventRecord(ev[2 * g], sin) != cudaSuccess) {
      rc = SSD_ERR_CUDA;
      break;
    }
  }
  // Then each group's compute once its inputs are in, and its outputs out once computed.
  for (int g = 0; g < ng && rc == SSD_OK; ++g) {
    const int64_t q0 = gs[g], q1 = gs[g + 1];
    int64_t t0, nt;
    group_tokens(g, t0, nt);
    const size_t p0 = (size_t)ptok[g];
    if (cudaStreamWaitEvent(st, ev[2 * g], 0) != cudaSuccess) {
      rc = SSD_ERR_CUDA;
      break;
    }
    ssd_shape sg = *s;
    if (cu_seqlens) {
      sg.batch = 1;
      sg.seqlen = nt;
      sg.nseq = q1 - q0;
      sg.cu_seqlens_host = nullptr;  // validated above
    } else {
      sg.batch = q1 - q0;
      sg.cu_seqlens_host = nullptr;
    }
    rc = forward_impl(&sg, at(dev[0], p0 * tok_x), (const float*)at(dev[1], p0 * tok_dt), (const float*)dev[2],
                      at(dev[3], p0 * tok_bc), at(dev[4], p0 * tok_bc), (const float*)dev[5],
                      (const float*)at(dev[6], seq_off[g]),
                      cu_seqlens ? (const int32_t*)dev[7] + cu_off[g] : nullptr, chunk, at(dev[8], p0 * tok_x),
                      (float*)at(dev[9], seq_off[g]), st);
    if (rc != SSD_OK) break;
    if (cudaEventRecord(ev[2 * g + 1], st) != cudaSuccess || cudaStreamWaitEvent(sout, ev[2 * g + 1], 0) != cudaSuccess ||
        !d2h((char*)y + t0 * tok_x, at(dev[8], p0 * tok_x), nt * tok_x) ||
        (final_state && !d2h((char*)final_state + q0 * seq_state, at(dev[9], seq_off[g]), (q1 - q0) * seq_state)))
      rc = SSD_ERR_CUDA;
  }
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

int ssd_set_test_hooks(int64_t wait_limit_cycles, int withhold) {
  if (wait_limit_cycles < 0 || (withhold & ~3)) return SSD_ERR_INVALID_ARG;
  g_wait_limit.store(wait_limit_cycles ? (long long)wait_limit_cycles : kDefaultWaitLimit);
  g_withhold_carry.store(withhold);
  return SSD_OK;
}

int ssd_select_path(const ssd_shape* shape, int chunk) {
  const int rc = validate(shape, (const void*)16, (const float*)16, (const float*)16, (const void*)16,
                          (const void*)16, shape && shape->cu_seqlens_host ? (const int32_t*)16 : nullptr, chunk,
                          (const void*)16);
  if (rc) return -rc;
  return select_path(shape, chunk);
}

}  // extern "C"
