// ssd_tc.cu -- the tensor-core path: one fused sm_100a kernel for the whole chunked
// SSD forward pass ("Transformers are SSMs", wikillm.com card, Method step 5, sec. 6).
//
// One persistent CTA per SM walks an equal share of the flat list of 128-token tiles
// (the tcgen05 M) of all units (sequence, pair of heads sharing a B/C group), handing
// the state on through global memory where its share starts or ends inside a unit.
// The P x N state of each head never leaves the chip: it stays in fp32 in tensor
// memory, with a bf16 copy in shared memory as an MMA operand.  Per tile:
//
//   cumsum   cs_j = running in-chunk cumsum of dt_j A_h in log2 units (restarted at
//            each chunk start, so a 256-token chunk spans two tiles)   [helper warps]
//   MMA  S   = C B^T                                   (128 x 128, K = N, once per pair)
//   MMA  Yo  = C [h0 h1]^T        left factor           (128 x 128, K = N)
//   MMA  h^T += B^T [w0 o x0 | w1 o x1]   right factor  (N x 128, K = 128),
//            w_j = exp(cs_end - cs_j) dt_j, onto the decay-scaled state
//   mask     P_ij = S_ij exp(cs_i - cs_j) dt_j for j <= i, else 0 (mask before exp),
//            written as bf16 pairs to tensor memory
//   scale    Y_i = exp(cs_i - cs_start) Yo_i
//   MMA  Y  += P_h x_h            diagonal block, A from tensor memory  (128 x 64, K = 128)
//   state    h <- exp(cs_end' - cs_start') h for the next tile (centre factor), its bf16
//            copy, or the final state / hand-on at the end of a piece
//   epilogue y_i = Y_i + D x_i    (bf16, staged over the x tile, TMA store)
//
// Roles: 16 compute warps (per head, two column halves x four lane quarters), one
// issuer warp (every TMA load of x, B, C and every tcgen05.mma) and two helper warps
// (dt loads and the per-tile descriptors: cumsums, column factors, decays, flags).
// Tensor memory: S 128 columns, P 2 x 64, Y 2 x 64, h^T 2 x 64.
// Every wait is bounded; a wait that gives up records SSD_ERR_DEVICE_TIMEOUT in the
// status word, drains what is in flight (bounded), frees tensor memory and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <stdio.h>
#include <stdlib.h>

#include "sm100_ptx.cuh"
#include "ssd_tc.cuh"

#ifndef SSD_TRACE
#define SSD_TRACE 0  // 1: record per-phase clock64 stamps of the first CTAs (profiling builds only)
#endif
#if SSD_TRACE
namespace ssd {
constexpr int kTraceCtas = 4, kTraceTiles = 64, kTraceMarks = 24;
__device__ unsigned long long g_trace[3 * kTraceCtas * kTraceTiles * kTraceMarks];
}  // namespace ssd
extern "C" int ssd_trace_dump(unsigned long long* host, int n) {
  return (int)cudaMemcpyFromSymbol(host, ssd::g_trace, sizeof(unsigned long long) * n);
}
#define TRACE_MARK(m)                                                                              \
  do {                                                                                             \
    if ((tid == 0 || tid == 96) && blockIdx.x < kTraceCtas && trace_tile < kTraceTiles)            \
      g_trace[(((tid != 0) * kTraceCtas + blockIdx.x) * kTraceTiles + trace_tile) * kTraceMarks +  \
              (m)] = clock64();                                                                    \
  } while (0)
#define TRACE_ISSUE(m)                                                                             \
  do {                                                                                             \
    if (blockIdx.x < kTraceCtas && t < kTraceTiles)                                                \
      g_trace[((2 * kTraceCtas + blockIdx.x) * kTraceTiles + t) * kTraceMarks + (m)] = clock64();  \
  } while (0)
#else
#define TRACE_ISSUE(m) \
  do {                 \
  } while (0)
#define TRACE_MARK(m) \
  do {                \
  } while (0)
#endif


namespace ssd {

namespace {

using namespace sm100;

constexpr int kTile = 128;          // tokens per tile (UMMA M)
constexpr int kHeadDim = 64;        // P supported by this path
constexpr int kWGThreads = 128;     // a warpgroup: thread i <-> TMEM lane i
constexpr int kHeads = 2;           // heads of one B/C group processed together
constexpr int kHalves = 2;          // each head's Y and state columns split over two warpgroups
constexpr int kComputeThreads = kHeads * kHalves * kWGThreads;
constexpr int kComputeWarps = kComputeThreads / 32;
constexpr int kHelperWarps = kHeads;  // one helper warp per head of the pair
constexpr int kThreads = kComputeThreads + 32 + 32 * kHelperWarps;  // + the issuer warp (TMA and UMMA), helpers
constexpr int kIssuerWarp = kComputeWarps, kHelperWarp = kComputeWarps + 1;
constexpr int kDescSlots = 2;  // tile descriptors the helper warp may run ahead
constexpr int kDtStages = 4;   // dt tiles in flight
constexpr uint32_t kTmemCols = 512;
// TMEM columns: S = C B^T (fp32, 128), P_h (bf16 pairs, 64 per head), Y_h (64 per head;
// the left factor is written first, row-scaled, then P_h x_h accumulates on top) and
// the fp32 state h^T of each head (64 per head): every tile it is scaled by the tile's
// decay in place and the right-factor MMA accumulates B^T (w o x) onto it.
constexpr uint32_t kColS = 0, kColP = 128, kColY = 256, kColSt = 384;
constexpr long long kWaitLimit = 4ll << 30;  // SM cycles (about 2 s) before a wait gives up
constexpr uint32_t kAtom = kTile * 128;      // one 128-row x 128-byte swizzled operand column

// mbarriers.  Issuer -> compute: tile loads (tx bytes) and UMMA commits.
// Compute -> issuer (one arrival per compute warp): ht, xw, p, free, x-free.
// Helper -> compute: a tile descriptor is written; compute -> helper: it was used up.
enum {
  kBarLoad0 = 0,  // x, B, C of a tile in x stage 0
  kBarLoad1,      // ... stage 1
  kBarS,          // S = C B^T done
  kBarYo,         // left factor C h^T written into Y
  kBarSt,         // right factor accumulated onto the state
  kBarY,          // P x accumulated into Y
  kBarHt,         // bf16 state for the next tile written
  kBarXw,         // w o x written and the state scaled by this tile's decay
  kBarP,          // P written and Y rows scaled
  kBarFree,       // Y read (the next left factor may overwrite it)
  kBarXfree,      // a stage's x buffer (which held that tile's y for the TMA stores) is reusable
  kBarDt0,        // kHelperWarps x kDtStages barriers: dt of a tile (4 heads x 128 tokens) in a helper's stage
  kBarDescFull0 = kBarDt0 + kHelperWarps * kDtStages,  // kDescSlots barriers: descriptor written (both helpers)
  kBarDescFree0 = kBarDescFull0 + kDescSlots,  // kDescSlots barriers: descriptor used up
  kBarPair0 = kBarDescFree0 + kDescSlots,  // 8 barriers: the column-half-1 warp of a row quarter staged its y
  kNumBars = kBarPair0 + kHeads * 4
};

// One tile as the helper warp lays it out for the compute warps: where it is, what to do
// with the state around it, and per head the in-chunk cumsum of dt A (log2 units), the
// 32-block column factors exp(cs(block end) - cs_j) dt_j, and dt.
enum {
  kDescFirst = 1,    // first tile of a piece: load the state (initial or handed on) before it
  kDescCarryIn = 2,  // ... from the carry of CTA carry_src
  kDescToFinal = 4,  // last tile of a unit: the state after it is the final state
  kDescToCarry = 8,  // last tile of a range that ends inside a unit: hand the state on
  kDescEnd = 16      // no tile: the range is done
};
struct TileDesc {
  int t0;         // token index of row 0
  int rem;        // rows of the tile inside the sequence (1..128)
  int s;          // sequence
  int h0;         // first head of the pair
  int flags;
  int carry_src;
  int pad[2];
  float cs_start[kHeads];  // cumsum before row 0
  float cs_end[kHeads];    // cumsum after the last row (rows past the end add 0)
  float decay[kHeads];     // exp2(cs_end - cs_start)
  float dskip[kHeads];     // D
  float cs[kHeads][kTile];
  float cc[kHeads][kTile];
  float dtv[kHeads][kTile];  // 0 past the end of the sequence
};
constexpr uint32_t kDescBytes = (sizeof(TileDesc) + 127) / 128 * 128;

template <int NS>
struct Layout {
  static constexpr uint32_t x = 0;                          // [stage][head] [128 tok][64 p]
  static constexpr uint32_t b = x + 2 * kHeads * kAtom;     // NS/64 atoms [128 tok][64 n]
  static constexpr uint32_t c = b + (NS / 64) * kAtom;
  static constexpr uint32_t xw = c + (NS / 64) * kAtom;     // [head] [128 tok][64 p]
  static constexpr uint32_t ht = xw + kHeads * kAtom;       // [head] [NS n][64 p]
  static constexpr uint32_t desc = ht + kHeads * NS * 128;           // TileDesc[kDescSlots]
  static constexpr uint32_t sdt = desc + kDescSlots * kDescBytes;    // float[helper][stage][128 tok][4 heads]
  static constexpr uint32_t bars = sdt + kHelperWarps * kDtStages * kTile * 16;  // uint64[kNumBars]
  static constexpr uint32_t flag = bars + kNumBars * 8;     // int: a wait gave up
  static constexpr uint32_t bytes = flag + 16;
};
template <int NS>
constexpr uint32_t kDynSmem = Layout<NS>::bytes + 1024;  // + base alignment slack
static_assert(kDynSmem<128> <= 227 * 1024, "shared memory per CTA");
static_assert(kNumBars <= 32, "phase bits of a 32-bit mask");

// Work split.  The tiles of all units (sequence, head pair), unit by unit and each
// unit's 128-token tiles in order, form one flat list; CTA r takes the contiguous
// range [W r / R, W (r + 1) / R).  A range may start inside a unit (it then needs the
// state the previous CTA reached there: "carry in") and end inside one (it then hands
// its state on: "carry out").  A CTA processes its last, truncated piece first, so the
// state it hands on is ready early; then the whole units; then the piece that needs a
// carry.  Issuer and compute threads walk the same sequence.
struct TileCursor {
  int unit, k0, len;  // k0: token offset of the tile in the sequence
  int tb;             // first token of the sequence (tokens < 2^31 on this path)
  int kend;           // token offset where this piece ends
  int piece;
  int flags;          // kCarryIn | kCarryOut | kUnitEnd
};
enum { kCarryIn = 1, kCarryOut = 2, kUnitEnd = 4 };

struct RangePlan {
  int u0, k0, u1, ke1, npieces;  // first unit/tile, last unit and its end tile (tiles)
  int carry_src;                 // the CTA whose range holds the tile before this range's first
};

__device__ __forceinline__ int unit_tiles(const Problem& pb, int u) {
  const int s = u / (pb.H / kHeads);
  return pb.seq_tiles[s + 1] - pb.seq_tiles[s];
}

__device__ __forceinline__ int64_t unit_first_tile(const Problem& pb, int u) {
  const int pairs = pb.H / kHeads;
  const int s = u / pairs;
  return (int64_t)pb.seq_tiles[s] * pairs + (int64_t)(u % pairs) * (pb.seq_tiles[s + 1] - pb.seq_tiles[s]);
}

// The unit holding flat tile w (0 <= w < W).
__device__ __forceinline__ int unit_of_tile(const Problem& pb, int64_t w) {
  const int pairs = pb.H / kHeads;
  int lo = 0, hi = pb.nseq;  // seq_tiles[lo] * pairs <= w < seq_tiles[hi] * pairs
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if ((int64_t)pb.seq_tiles[mid] * pairs <= w)
      lo = mid;
    else
      hi = mid;
  }
  const int T = pb.seq_tiles[lo + 1] - pb.seq_tiles[lo];
  return lo * pairs + (int)((w - (int64_t)pb.seq_tiles[lo] * pairs) / T);
}

__device__ __forceinline__ RangePlan plan_range(const Problem& pb) {
  RangePlan rp{};
  const int64_t W = (int64_t)pb.seq_tiles[pb.nseq] * (pb.H / kHeads);
  const int64_t w0 = W * blockIdx.x / gridDim.x, w1 = W * (blockIdx.x + 1) / gridDim.x;
  if (w0 >= w1) return rp;
  rp.u0 = unit_of_tile(pb, w0);
  rp.k0 = (int)(w0 - unit_first_tile(pb, rp.u0));
  rp.u1 = unit_of_tile(pb, w1 - 1);
  rp.ke1 = (int)(w1 - unit_first_tile(pb, rp.u1));
  rp.npieces = rp.u0 == rp.u1 ? 1 : rp.u1 - rp.u0 + 1;
  // range r holds tiles [W r / R, W (r + 1) / R): tile w lies in range ceil((w + 1) R / W) - 1
  // (empty ranges are skipped over when there are fewer tiles than CTAs)
  if (w0 > 0) rp.carry_src = (int)((w0 * gridDim.x + W - 1) / W) - 1;
  return rp;
}

// Loads piece `pi` (processing order) into c; false when it has no tiles.
__device__ __forceinline__ bool load_piece(const Problem& pb, const RangePlan& rp, int pi, TileCursor& c) {
  int u, kb, ke;
  if (rp.npieces == 1) {
    u = rp.u0, kb = rp.k0, ke = rp.ke1;
  } else if (pi == 0) {  // the truncated last piece first
    u = rp.u1, kb = 0, ke = rp.ke1;
  } else if (pi < rp.npieces - 1) {  // whole units
    u = rp.u0 + pi, kb = 0, ke = unit_tiles(pb, rp.u0 + pi);
  } else {  // the first piece last: it may need the previous CTA's state
    u = rp.u0, kb = rp.k0, ke = unit_tiles(pb, rp.u0);
  }
  if (ke <= kb) return false;
  const int pairs = pb.H / kHeads;
  const int s = u / pairs;
  c.unit = u;
  c.tb = (int)seq_off(pb, s);
  c.len = (int)(seq_off(pb, s + 1) - c.tb);
  c.k0 = kb * kTile;
  c.kend = min(ke * kTile, c.len);
  c.piece = pi;
  const bool unit_end = ke == unit_tiles(pb, u);
  c.flags = (kb > 0 ? kCarryIn : 0) | (unit_end ? kUnitEnd : kCarryOut);
  return true;
}

__device__ __forceinline__ bool cursor_from(const Problem& pb, const RangePlan& rp, int pi, TileCursor& c) {
  for (; pi < rp.npieces; ++pi)
    if (load_piece(pb, rp, pi, c)) return true;
  return false;
}

__device__ __forceinline__ bool cursor_first(const Problem& pb, const RangePlan& rp, TileCursor& c) {
  return cursor_from(pb, rp, 0, c);
}

// Advances to the next tile of this CTA's range; false when done.
__device__ __forceinline__ bool cursor_next(const Problem& pb, const RangePlan& rp, TileCursor& c) {
  c.k0 += kTile;
  if (c.k0 < c.kend) return true;
  return cursor_from(pb, rp, c.piece + 1, c);
}

// One arrival for the whole warp, after every lane's prior work (the lanes' own fences
// come before it).
__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
  __syncwarp();
}

// Bounded wait that also gives up when another thread has recorded a failure.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitLimit) {
      *abort_flag = 1;
      return false;
    }
  }
  return true;
}

// ------------------------------------------------------------------ issuer
template <int NS>
__device__ void issuer_loop(const CUtensorMap* tm_x, const CUtensorMap* tm_b, const CUtensorMap* tm_c,
                            const Problem& pb, uint8_t* smem, uint32_t tmem, uint64_t* bars,
                            volatile int* abort_flag) {
  using L = Layout<NS>;
  uint8_t* sx = smem + L::x;
  uint8_t* sb = smem + L::b;
  uint8_t* sc = smem + L::c;
  constexpr uint32_t kLoadBytes = kHeads * kAtom + 2u * (NS / 64) * kAtom;
  const uint32_t id_s = idesc_bf16(128, 128, 0, 0);
  const uint32_t id_y = idesc_bf16(128, 64, 0, 1);
  const uint32_t id_yo = idesc_bf16(128, 128, 0, 1);
  const uint32_t id_st = idesc_bf16(128, 128, 1, 1);
  const uint32_t a_sb = smem_u32(sb), a_sc = smem_u32(sc);
  const uint32_t a_sxw = smem_u32(smem + L::xw), a_sht = smem_u32(smem + L::ht);
  // For N = 64 the B^T operand has one M atom; the second (unused) half of s^T reads
  // the C tile that follows it, and those lanes are ignored.
  const uint32_t lbo_bt = kAtom;
  const int pairs = pb.H / kHeads;

  auto issue_x = [&](int stage, const TileCursor& c) {
    const int h0 = (c.unit % pairs) * kHeads;
#pragma unroll
    for (int hh = 0; hh < kHeads; ++hh)
      tma_load_3d(sx + (stage * kHeads + hh) * kAtom, tm_x, 0, h0 + hh, c.tb + c.k0, &bars[stage]);
  };
  auto issue_bc = [&](int stage, const TileCursor& c) {
    const int g = ((c.unit % pairs) * kHeads) / pb.hpg;
#pragma unroll
    for (int a = 0; a < NS / 64; ++a) {
      tma_load_3d(sb + a * kAtom, tm_b, a * 64, g, c.tb + c.k0, &bars[stage]);
      tma_load_3d(sc + a * kAtom, tm_c, a * 64, g, c.tb + c.k0, &bars[stage]);
    }
  };

  uint32_t phase = 0;    // bit k: parity of the next phase of bars[k] this thread waits for
  uint32_t pending = 0;  // bit k: async work on bars[k] issued and not waited for
  auto wait = [&](int k) -> bool {
    if (!wait_or_abort(&bars[k], (phase >> k) & 1u, abort_flag)) return false;
    phase ^= 1u << k;
    pending &= ~(1u << k);
    return true;
  };

  const RangePlan rp = plan_range(pb);
  TileCursor cur;
  bool have = cursor_first(pb, rp, cur);
  int stage = 0, t = 0;
  if (have) {
    mbar_expect_tx(&bars[kBarLoad0], kLoadBytes);
    issue_x(0, cur);
    issue_bc(0, cur);
    pending |= 1u << kBarLoad0;
  }
  bool ok = true;
  while (have) {
    TileCursor nxt = cur;
    const bool have_next = cursor_next(pb, rp, nxt);
    TRACE_ISSUE(0);
    // S = C B^T once this tile's x, B, C are in (the previous mask finished with S).
    if (!(ok = wait(stage))) break;
    TRACE_ISSUE(1);
    tc_fence_after();
#pragma unroll
    for (int kk = 0; kk < NS / 16; ++kk) {
      const uint32_t koff = (kk >> 2) * kAtom + (kk & 3) * 32;
      umma_f16(tmem + kColS, sdesc_sw128(a_sc + koff, 16, 1024), sdesc_sw128(a_sb + koff, 16, 1024), id_s, kk > 0);
    }
    umma_commit(&bars[kBarS]);
    pending |= 1u << kBarS;
    // Left factor C h^T into Y: needs the bf16 state and the previous epilogue done with Y.
    if (!(ok = wait(kBarHt))) break;
    TRACE_ISSUE(2);
    if (t > 0 && !(ok = wait(kBarFree))) break;
    TRACE_ISSUE(3);
    tc_fence_after();
#pragma unroll
    for (int kk = 0; kk < NS / 16; ++kk) {
      const uint32_t koff = (kk >> 2) * kAtom + (kk & 3) * 32;
      umma_f16(tmem + kColY, sdesc_sw128(a_sc + koff, 16, 1024), sdesc_sw128(a_sht + kk * 2048, NS * 128, 1024),
               id_yo, kk > 0);
    }
    umma_commit(&bars[kBarYo]);
    pending |= 1u << kBarYo;
    if (have_next) {  // the other x stage (tile t-1's x, then its y) is free once its y store read it
      if (t > 0 && !(ok = wait(kBarXfree))) break;
      TRACE_ISSUE(4);
      fence_proxy_async();
      mbar_expect_tx(&bars[stage ^ 1], kLoadBytes);
      issue_x(stage ^ 1, nxt);
      pending |= 1u << (stage ^ 1);
    }
    // Right factor onto the (decay-scaled) state: h^T += B^T [w0 x0 | w1 x1].
    if (!(ok = wait(kBarXw))) break;
    TRACE_ISSUE(5);
    tc_fence_after();
#pragma unroll
    for (int kk = 0; kk < kTile / 16; ++kk)
      umma_f16(tmem + kColSt, sdesc_sw128(a_sb + kk * 2048, lbo_bt, 1024),
               sdesc_sw128(a_sxw + kk * 2048, kAtom, 1024), id_st, 1);
    umma_commit(&bars[kBarSt]);
    pending |= 1u << kBarSt;
    // B and C are free once S and both factors are done: next tile's, issued now so that
    // the load runs under this tile's masked product and epilogue.
    if (have_next) {
      if (!(ok = wait(kBarS)) || !(ok = wait(kBarYo)) || !(ok = wait(kBarSt))) break;
      TRACE_ISSUE(6);
      fence_proxy_async();
      issue_bc(stage ^ 1, nxt);
    }
    // Y_h += P_h x_h (A from tensor memory).
    if (!(ok = wait(kBarP))) break;
    TRACE_ISSUE(7);
    tc_fence_after();
    {
      const uint32_t a_sx = smem_u32(sx + stage * kHeads * kAtom);
#pragma unroll
      for (int hh = 0; hh < kHeads; ++hh) {
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          umma_f16_ta(tmem + kColY + hh * 64, tmem + kColP + hh * 64 + kk * 8,
                      sdesc_sw128(a_sx + hh * kAtom + kk * 2048, kAtom, 1024), id_y, 1);
      }
    }
    umma_commit(&bars[kBarY]);
    pending |= 1u << kBarY;
    cur = nxt;
    have = have_next;
    stage ^= 1;
    ++t;
  }
  if (!ok) {
    *abort_flag = 1;
    // Drain what this thread issued (again bounded) before tensor memory is freed.
    for (int k = 0; k < kNumBars; ++k)
      if (pending & (1u << k)) mbar_wait_bounded(&bars[k], (phase >> k) & 1u, kWaitLimit);
  }
}

// --------------------------------------------------------- compute warpgroups
// Four warpgroups: two per head of the pair, one per 32-column half of that head's Y and
// state columns in tensor memory.  Warp (head hw, half ch, quarter wq) owns TMEM lanes /
// tile rows 32 wq .. 32 wq + 31 and columns 32 ch .. 32 ch + 31 of its head's Y and state;
// of the masked product it computes the 32-column blocks ch and ch + 2.  What is the same
// for every row of a tile (where it is, the cumsums and column factors) comes from the
// helper warp's tile descriptor.  The two halves of a row quarter meet once a tile, on a
// one-arrival barrier, before the half-0 warp stores their 32 rows of y by TMA.  Every
// wait is warp-uniform and bounded.
template <int NS>
__device__ void compute_loop(const CUtensorMap* tm_y32, const Problem& pb, uint8_t* smem, uint32_t tmem,
                             uint64_t* bars, volatile int* abort_flag) {
  using L = Layout<NS>;
  const int tid = threadIdx.x;
  const int wid = tid >> 5;                 // compute warp 0..15
  const int hw = wid >> 3;                  // head of the pair
  const int ch = (wid >> 2) & 1;            // column half
  const int wq = wid & 3, lane = tid & 31;  // lane quarter (a warp reaches TMEM lanes 32 (warp % 4) ..)
  const int i = wq * 32 + lane;             // row / TMEM lane
  const int pair_bar = kBarPair0 + hw * 4 + wq;
  const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
  const uint32_t col_h = hw * 64 + ch * 32;  // this warp's Y and state columns
  uint8_t* sx = smem + L::x;
  uint8_t* sxw = smem + L::xw;
  uint8_t* sht = smem + L::ht;
  const TileDesc* descs = reinterpret_cast<const TileDesc*>(smem + L::desc);
  const int pairs = pb.H / kHeads;
  const int units = pb.nseq * pairs;

  uint32_t phase = 0;
  // Warp-uniform bounded wait on a barrier.
  auto wait = [&](int k) -> bool {
    const bool mine = wait_or_abort(&bars[k], (phase >> k) & 1u, abort_flag);
    if (__any_sync(0xffffffffu, !mine)) return false;
    phase ^= 1u << k;
    return true;
  };

  // Units whose sequences are empty have no tiles: CTA r writes final = init for the
  // empty units u with u % R == r.
  if (pb.final_state && i < NS) {
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
      if (unit_tiles(pb, u) != 0) continue;
      const int s = u / pairs;
      const int h = (u % pairs) * kHeads + hw;
      const int64_t base = ((int64_t)s * pb.H + h) * kHeadDim * NS;
      for (int p = 32 * ch; p < 32 * ch + 32; ++p)
        pb.final_state[base + (int64_t)p * NS + i] = pb.init ? pb.init[base + (int64_t)p * NS + i] : 0.f;
    }
  }

  // The head state lives in tensor memory as h^T (lane n = state column n, 64 fp32
  // columns, 32 per half); its bf16 copy in shared memory is the B operand of the left factor.
  const uint32_t t_state = tmem + lane_base + kColSt + col_h;
  auto write_ht_from = [&](const uint32_t (&r)[32]) {
    if (i < NS) {
      uint8_t* hdst = sht + hw * NS * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint4 hv;
        hv.x = bf16x2_of(f2u(r[8 * c + 0], r[8 * c + 1]));
        hv.y = bf16x2_of(f2u(r[8 * c + 2], r[8 * c + 3]));
        hv.z = bf16x2_of(f2u(r[8 * c + 4], r[8 * c + 5]));
        hv.w = bf16x2_of(f2u(r[8 * c + 6], r[8 * c + 7]));
        *reinterpret_cast<uint4*>(hdst + sw128_off(i, 4 * ch + c)) = hv;
      }
    }
  };
  // The state at the start of the piece whose first tile d describes, into r: the
  // sequence's initial state (or zero), or the state the previous CTA handed on.
  // False if the wait for that hand-on gave up.
  auto load_state = [&](const TileDesc& d, uint32_t (&r)[32]) -> bool {
    const float* src_p = nullptr;
    if (d.flags & kDescCarryIn) {
      const int src = d.carry_src;
      bool mine = true;
      if (lane == 0) {
        const long long t0 = clock64();
        while (ld_acquire_gpu(&pb.carry_flag[src]) < kComputeWarps) {
          if (*abort_flag || clock64() - t0 > kWaitLimit) {
            *abort_flag = 1;
            mine = false;
            break;
          }
          __nanosleep(200);
        }
      }
      if (__any_sync(0xffffffffu, !mine)) return false;
      __threadfence();
      src_p = pb.carry + ((size_t)src * kHeads + hw) * kHeadDim * NS + i;
    } else if (pb.init) {
      src_p = pb.init + ((int64_t)d.s * pb.H + d.h0 + hw) * kHeadDim * NS + i;
    }
#pragma unroll
    for (int q = 0; q < 32; ++q)
      r[q] = __float_as_uint((src_p && i < NS) ? __ldcg(src_p + (size_t)(32 * ch + q) * NS) : 0.f);
    return true;
  };
  // r holds the state at the start of the tile d describes: its bf16 copy is the left
  // factor's operand; scaled by the tile's decay it is what the right factor accumulates onto.
  auto start_tile_state = [&](const TileDesc& d, uint32_t (&r)[32]) {
    write_ht_from(r);
    const float decay = d.decay[hw];
    const uint64_t decay2 = f2(decay, decay);
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      float lo, hi;
      unf2(mul2(decay2, f2u(r[2 * q], r[2 * q + 1])), lo, hi);
      r[2 * q] = __float_as_uint(lo);
      r[2 * q + 1] = __float_as_uint(hi);
    }
    tmem_st32(t_state, r);
    tmem_st_wait();
  };
  // P values of one 32-column block of S (fp32 bits in r) for row i.
  auto mask_block = [&](int cb, const uint32_t* r, float cs_i, const float* dcs, const float* dcc,
                        const float* ddt, uint32_t (&pk)[16]) {
    if (cb < wq) {  // strictly below the diagonal: exp(cs_i - cs_j) = rf * exp(cs_ref - cs_j)
      const float rf = ex2(cs_i - dcs[cb * 32 + 31]);
      const uint64_t rf2 = f2(rf, rf);
      const float4* cc4 = reinterpret_cast<const float4*>(dcc + cb * 32);
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        const float4 c = cc4[q4];
        const uint64_t f0 = mul2(rf2, f2(c.x, c.y)), f1 = mul2(rf2, f2(c.z, c.w));
        pk[2 * q4] = bf16x2_of(mul2(f0, f2u(r[4 * q4], r[4 * q4 + 1])));
        pk[2 * q4 + 1] = bf16x2_of(mul2(f1, f2u(r[4 * q4 + 2], r[4 * q4 + 3])));
      }
    } else {  // diagonal block: mask first (-inf), then exp
      const float4* c4 = reinterpret_cast<const float4*>(dcs + cb * 32);
      const float4* d4 = reinterpret_cast<const float4*>(ddt + cb * 32);
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        const float4 cj = c4[q4], dj = d4[q4];
        const int j0 = 4 * q4;  // column within the block; this row is `lane`
        const float e0 = ex2(j0 <= lane ? cs_i - cj.x : -INFINITY);
        const float e1 = ex2(j0 + 1 <= lane ? cs_i - cj.y : -INFINITY);
        const float e2 = ex2(j0 + 2 <= lane ? cs_i - cj.z : -INFINITY);
        const float e3 = ex2(j0 + 3 <= lane ? cs_i - cj.w : -INFINITY);
        pk[2 * q4] = bf16x2_of(mul2(mul2(f2(e0, e1), f2(dj.x, dj.y)), f2u(r[j0], r[j0 + 1])));
        pk[2 * q4 + 1] = bf16x2_of(mul2(mul2(f2(e2, e3), f2(dj.z, dj.w)), f2u(r[j0 + 2], r[j0 + 3])));
      }
    }
  };

  if (!wait(kBarDescFull0)) return;
  if (descs[0].flags & kDescEnd) return;
  {
    uint32_t r[32];
    if (!load_state(descs[0], r)) return;
    start_tile_state(descs[0], r);
  }
  fence_proxy_async();
  tc_fence_before();
  warp_arrive(&bars[kBarHt]);
  int trace_tile = 0;
  (void)trace_tile;

  for (int t = 0;; ++t) {
    const int slot = t % kDescSlots, stage = t & 1;
    const TileDesc& d = descs[slot];
    TRACE_MARK(0);
    const int h = d.h0 + hw;
    const int t0 = d.t0, rem = d.rem, flags = d.flags;
    const float* dcs = d.cs[hw];
    const float* dcc = d.cc[hw];
    const float* ddt = d.dtv[hw];
    const float cs_start = d.cs_start[hw], cs_end = d.cs_end[hw];
    const float cs_i = dcs[i];
    const float w_i = ex2(cs_end - cs_i) * ddt[i];  // right-factor weight (0 past the end)
    const float carry = ex2(cs_i - cs_start);      // decay of the carried-in state to token i
    TRACE_MARK(1);

    // ---- this tile's x: w o x, the right-factor input
    if (!wait(stage)) return;
    TRACE_MARK(2);
    const uint8_t* sxh = sx + (stage * kHeads + hw) * kAtom;
    {
      uint8_t* dst = sxw + hw * kAtom;
      const uint32_t w2 = pack_bf16(w_i, w_i);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const uint32_t o = sw128_off(i, 4 * ch + cc);
        uint4 xv = *reinterpret_cast<const uint4*>(sxh + o);
        xv.x = mul_bf16x2(xv.x, w2);
        xv.y = mul_bf16x2(xv.y, w2);
        xv.z = mul_bf16x2(xv.z, w2);
        xv.w = mul_bf16x2(xv.w, w2);
        *reinterpret_cast<uint4*>(dst + o) = xv;
      }
    }
    fence_proxy_async();
    warp_arrive(&bars[kBarXw]);
    if (t > 0) {  // this warp's y store of the previous tile has read its x stage: release it
      if (lane == 0) bulk_wait_read();
      warp_arrive(&bars[kBarXfree]);
    }
    TRACE_MARK(3);

    // ---- P_h = mask_h(S), bf16 pairs in tensor memory
    if (!wait(kBarS)) return;
    TRACE_MARK(4);
    tc_fence_after();
    {
      // blocks ch and ch + 2 (32 columns of S each) -> P columns 16 cb .. 16 cb + 15
      const uint32_t colp = kColP + hw * 64;
#pragma unroll 1
      for (int cb = ch; cb < 4; cb += 2) {
        uint32_t pk[16];
        if (cb <= wq) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_base + kColS + cb * 32, r);
          tmem_ld_wait();
          mask_block(cb, r, cs_i, dcs, dcc, ddt, pk);
        } else {  // above the diagonal: zero
#pragma unroll
          for (int q = 0; q < 16; ++q) pk[q] = 0u;
        }
        tmem_st16(tmem + lane_base + colp + cb * 16, pk);
      }
    }
    TRACE_MARK(5);

    // ---- scale the left factor's row by exp(cs_i - cs_start), in place in Y
    if (!wait(kBarYo)) return;
    tc_fence_after();
    {
      const uint64_t carry2 = f2(carry, carry);
      uint32_t r[32];
      tmem_ld32(tmem + lane_base + kColY + col_h, r);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        float lo, hi;
        unf2(mul2(carry2, f2u(r[2 * q], r[2 * q + 1])), lo, hi);
        r[2 * q] = __float_as_uint(lo);
        r[2 * q + 1] = __float_as_uint(hi);
      }
      tmem_st32(tmem + lane_base + kColY + col_h, r);
    }
    tmem_st_wait();
    tc_fence_before();
    warp_arrive(&bars[kBarP]);
    TRACE_MARK(6);

    // ---- the state after this tile: at the end of a piece the final state or the
    // hand-on to the next CTA; then the next tile's start state (this one, or the next
    // piece's) as its bf16 copy and, decay-scaled, in tensor memory
    if (!wait(kBarSt)) return;
    tc_fence_after();
    const int nslot = (t + 1) % kDescSlots;
    bool more;
    {
      uint32_t r[32];
      tmem_ld32(t_state, r);
      tmem_ld_wait();
      if ((flags & kDescToFinal) && i < NS) {
        float* fp = pb.final_state + ((int64_t)d.s * pb.H + h) * kHeadDim * NS + i;
#pragma unroll
        for (int q = 0; q < 32; ++q) fp[(size_t)(32 * ch + q) * NS] = __uint_as_float(r[q]);
      }
      if (flags & kDescToCarry) {  // hand the state on: one release increment per warp once its part is out
        if (i < NS) {
          float* cp = pb.carry + ((size_t)blockIdx.x * kHeads + hw) * kHeadDim * NS + i;
#pragma unroll
          for (int q = 0; q < 32; ++q) cp[(size_t)(32 * ch + q) * NS] = __uint_as_float(r[q]);
        }
        if (i == 0 && ch == 0)
          pb.carry[(size_t)pb.ranges * kHeads * kHeadDim * NS + blockIdx.x * kHeads + hw] = cs_end;
        __threadfence();
        __syncwarp();
        if (lane == 0) red_add_release_gpu(&pb.carry_flag[blockIdx.x], 1);
        __syncwarp();
      }
      TRACE_MARK(10);
      if (!wait(kBarDescFull0 + nslot)) return;
      TRACE_MARK(11);
      const TileDesc& dn = descs[nslot];
      more = !(dn.flags & kDescEnd);
      if (more) {
        if ((dn.flags & kDescFirst) && !load_state(dn, r)) return;
        start_tile_state(dn, r);
      }
    }
    fence_proxy_async();
    tc_fence_before();
    warp_arrive(&bars[kBarHt]);
    TRACE_MARK(7);

    // ---- epilogue: y = Y + D x, staged over this tile's x; the half-0 warp of each row
    // quarter stores the quarter's 32 rows by TMA once the half-1 warp has staged its columns
    if (!wait(kBarY)) return;
    TRACE_MARK(8);
    tc_fence_after();
    {
      const float Dh = d.dskip[hw];
      const uint64_t d2 = f2(Dh, Dh);
      const bool full = rem >= 32 * wq + 32;  // all 32 rows of this quarter are in the sequence
      uint8_t* ystage = const_cast<uint8_t*>(sxh);  // each thread overwrites the x chunks it reads
      __nv_bfloat16* yrow = static_cast<__nv_bfloat16*>(pb.y) + ((int64_t)(t0 + i) * pb.H + h) * kHeadDim;
      uint32_t ry[32];
      tmem_ld32(tmem + lane_base + kColY + col_h, ry);
      tmem_ld_wait();
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const int c = 4 * ch + cc;
        const uint32_t o = sw128_off(i, c);
        const uint4 xv = *reinterpret_cast<const uint4*>(sxh + o);
        const uint32_t xu[4] = {xv.x, xv.y, xv.z, xv.w};
        uint32_t out[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {  // bf16 pair -> fp32 pair (exact), then D x + Y as one f32x2 fma
          const uint64_t x2 = f2u(xu[q] << 16, xu[q] & 0xFFFF0000u);
          out[q] = bf16x2_of(fma2(d2, x2, f2u(ry[8 * cc + 2 * q], ry[8 * cc + 2 * q + 1])));
        }
        const uint4 ov = make_uint4(out[0], out[1], out[2], out[3]);
        if (full)
          *reinterpret_cast<uint4*>(ystage + o) = ov;
        else if (i < rem)
          *reinterpret_cast<uint4*>(yrow + 8 * c) = ov;
      }
      tc_fence_before();
      if (full) fence_proxy_async();
      __syncwarp();
      if (ch == 1) {
        if (lane == 0) mbar_arrive(&bars[pair_bar]);
      } else {
        if (!wait(pair_bar)) return;
        if (full && lane == 0) {
          tma_store_3d(tm_y32, ystage + wq * 32 * 128, 0, h, t0 + 32 * wq);
          bulk_commit();
        }
      }
      __syncwarp();
    }
    // Y is free for the next left factor; this tile's descriptor is used up
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&bars[kBarFree]);
      mbar_arrive(&bars[kBarDescFree0 + slot]);
    }
    __syncwarp();
    TRACE_MARK(9);
    ++trace_tile;
    if (!more) break;
  }
}

// ------------------------------------------------------------------ helper warps
// Helper warp hh walks the CTA's tile sequence a few tiles ahead of the compute warps,
// loads each tile's dt by TMA into a ring of its own (kDtStages tiles in flight) and
// writes head hh's part of the tile's descriptor into a ring of kDescSlots: the in-chunk
// cumsum of dt A in log2 units (restarted at every chunk boundary, and continued from the
// handing-on CTA's value at a hand-on), the column factors exp2(cs(end of 32-block) -
// cs_j) dt_j, dt (0 past the sequence end), the decay and D.  Helper 0 also writes where
// the tile is and what happens to the state around it.  The descriptor is complete when
// both helpers have arrived.
template <int NS>
__device__ void helper_loop(const CUtensorMap* tm_dt, const Problem& pb, uint8_t* smem, uint64_t* bars,
                            volatile int* abort_flag, int hh) {
  using L = Layout<NS>;
  const int lane = threadIdx.x & 31;
  uint8_t* my_dt = smem + L::sdt + hh * kDtStages * kTile * 16;
  uint64_t* my_bar = bars + kBarDt0 + hh * kDtStages;
  const int pairs = pb.H / kHeads;
  TileDesc* descs = reinterpret_cast<TileDesc*>(smem + L::desc);
  uint32_t phase = 0;
  auto wait = [&](int k) -> bool {
    const bool mine = wait_or_abort(&bars[k], (phase >> k) & 1u, abort_flag);
    if (__any_sync(0xffffffffu, !mine)) return false;
    phase ^= 1u << k;
    return true;
  };
  const RangePlan rp = plan_range(pb);

  // dt loads run up to kDtStages tiles ahead on a cursor of their own
  TileCursor ahead;
  bool have_ahead = cursor_first(pb, rp, ahead);
  int dt_issued = 0;
  auto issue_dt = [&]() {
    if (lane == 0) {
      const int st = dt_issued % kDtStages;
      const int h0 = (ahead.unit % pairs) * kHeads;
      mbar_expect_tx(&my_bar[st], kTile * 16);
      tma_load_2d(my_dt + st * kTile * 16, tm_dt, h0 & ~3, ahead.tb + ahead.k0, &my_bar[st]);
    }
    ++dt_issued;
    have_ahead = cursor_next(pb, rp, ahead);
  };
  for (int k = 0; k < kDtStages && have_ahead; ++k) issue_dt();

  TileCursor cur;
  bool have = cursor_first(pb, rp, cur);
  float cs_base = 0.f, a2 = 0.f, dsk = 0.f;
  int a_unit = -1, prev_piece = -1;
  bool ok = true;
  int t = 0;
  for (;; ++t) {
    const int slot = t % kDescSlots;
    if (t >= kDescSlots && !(ok = wait(kBarDescFree0 + slot))) break;
    TileDesc& d = descs[slot];
    if (!have) {
      if (hh == 0 && lane == 0) d.flags = kDescEnd;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarDescFull0 + slot]);
      break;
    }
    TileCursor nxt = cur;
    const bool have_next = cursor_next(pb, rp, nxt);
    const bool first = cur.piece != prev_piece;
    const bool last = !have_next || nxt.piece != cur.piece;
    prev_piece = cur.piece;
    const int h0 = (cur.unit % pairs) * kHeads;
    if (cur.unit != a_unit) {
      a_unit = cur.unit;
      a2 = pb.A[h0 + hh] * 1.4426950408889634f;  // A_h log2(e): cumsums are in log2 units
      dsk = pb.D ? pb.D[h0 + hh] : 0.f;
    }
    int flags = 0;
    if (first) {
      flags |= kDescFirst;
      cs_base = 0.f;
      if (cur.flags & kCarryIn) {  // continue from the cumsum the previous CTA reached
        flags |= kDescCarryIn;
        bool mine = true;
        if (lane == 0) {
          const long long c0 = clock64();
          while (ld_acquire_gpu(&pb.carry_flag[rp.carry_src]) < kComputeWarps) {
            if (*abort_flag || clock64() - c0 > kWaitLimit) {
              *abort_flag = 1;
              mine = false;
              break;
            }
            __nanosleep(200);
          }
        }
        if (__any_sync(0xffffffffu, !mine)) {
          ok = false;
          break;
        }
        __threadfence();
        cs_base = __ldcg(pb.carry + (size_t)pb.ranges * kHeads * kHeadDim * NS + rp.carry_src * kHeads + hh);
      }
    }
    if (last && (cur.flags & kUnitEnd) && pb.final_state) flags |= kDescToFinal;
    if (last && (cur.flags & kCarryOut)) flags |= kDescToCarry;
    if (cur.k0 % pb.Q == 0) cs_base = 0.f;

    // this tile's dt: row 4 lane + j holds the 4 heads' dt of one token; a lane reads its
    // rows in the order j = (k + rot) & 3, rot = (lane / 2) & 3, so each quarter warp's
    // 16-byte loads fall in distinct banks
    if (!(ok = wait(kBarDt0 + hh * kDtStages + t % kDtStages))) break;
    float dtt[4];
    {
      const float4* rows = reinterpret_cast<const float4*>(my_dt + (t % kDtStages) * kTile * 16) + 4 * lane;
      const int rot = (lane >> 1) & 3, c = (h0 & 3) + hh;  // this head's column in the 4-head row
      float v[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float4 q = rows[(k + rot) & 3];
        v[k] = c == 0 ? q.x : c == 1 ? q.y : c == 2 ? q.z : q.w;
      }
      const int left = cur.len - cur.k0 - 4 * lane;
#pragma unroll
      for (int j = 0; j < 4; ++j) {  // token j came in as k = (j - rot) & 3
        const int k = (j - rot) & 3;
        const float val = k == 0 ? v[0] : k == 1 ? v[1] : k == 2 ? v[2] : v[3];
        dtt[j] = j < left ? dt_value(pb, val, h0 + hh) : 0.f;
      }
    }
    {
      float c0 = dtt[0] * a2, c1 = c0 + dtt[1] * a2, c2 = c1 + dtt[2] * a2, c3 = c2 + dtt[3] * a2;
      float v = c3;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
      }
      const float base = cs_base + v - c3;  // cumsum before token 4 lane
      c0 += base, c1 += base, c2 += base, c3 += base;
      reinterpret_cast<float4*>(d.cs[hh])[lane] = make_float4(c0, c1, c2, c3);
      reinterpret_cast<float4*>(d.dtv[hh])[lane] = make_float4(dtt[0], dtt[1], dtt[2], dtt[3]);
      // block ends (tokens 31, 63, 95, 127) live in lanes 7, 15, 23, 31
      const float ref = __shfl_sync(0xffffffffu, c3, (lane & ~7) | 7);
      reinterpret_cast<float4*>(d.cc[hh])[lane] = make_float4(ex2(ref - c0) * dtt[0], ex2(ref - c1) * dtt[1],
                                                              ex2(ref - c2) * dtt[2], ex2(ref - c3) * dtt[3]);
      const float cs_end = __shfl_sync(0xffffffffu, c3, 31);  // tokens past the end add 0
      if (lane == 0) {
        d.cs_start[hh] = cs_base;
        d.cs_end[hh] = cs_end;
        d.decay[hh] = ex2(cs_end - cs_base);
        d.dskip[hh] = dsk;
      }
      cs_base = cs_end;
    }
    if (hh == 0 && lane == 0) {
      d.t0 = cur.tb + cur.k0;
      d.rem = min(kTile, cur.len - cur.k0);
      d.s = cur.unit / pairs;
      d.h0 = h0;
      d.flags = flags;
      d.carry_src = rp.carry_src;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars[kBarDescFull0 + slot]);
    // the dt stage this tile used is read: refill it
    if (have_ahead) issue_dt();
    cur = nxt;
    have = have_next;
  }
  if (!ok) {
    *abort_flag = 1;
    // dt loads still in flight land before the CTA ends (bounded)
    if (lane == 0)
      for (int n = t; n < dt_issued; ++n)
        mbar_wait_bounded(&my_bar[n % kDtStages], (n / kDtStages) & 1, kWaitLimit);
  }
}

template <int NS>
__global__ void __launch_bounds__(kThreads, 1)
    ssd_fused_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                        const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_y32,
                        const __grid_constant__ CUtensorMap tm_dt, Problem pb) {
  using L = Layout<NS>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem_base;
  const int tid = threadIdx.x, warp = tid >> 5;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::bars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::flag);

  if (*pb.nchunks < 0) return;  // cu_seqlens rejected by the table kernel

  if (warp == 0) {
    tmem_alloc(&s_tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bars[kBarLoad0], 1);
    mbar_init(&bars[kBarLoad1], 1);
    mbar_init(&bars[kBarS], 1);
    mbar_init(&bars[kBarYo], 1);
    mbar_init(&bars[kBarSt], 1);
    mbar_init(&bars[kBarY], 1);
    mbar_init(&bars[kBarHt], kComputeWarps);
    mbar_init(&bars[kBarXw], kComputeWarps);
    mbar_init(&bars[kBarP], kComputeWarps);
    mbar_init(&bars[kBarFree], kComputeWarps);
    mbar_init(&bars[kBarXfree], kComputeWarps);
    for (int k = 0; k < kHelperWarps * kDtStages; ++k) mbar_init(&bars[kBarDt0 + k], 1);
    for (int k = 0; k < kDescSlots; ++k) {
      mbar_init(&bars[kBarDescFull0 + k], kHelperWarps);
      mbar_init(&bars[kBarDescFree0 + k], kComputeWarps);
    }
    for (int k = 0; k < kHeads * 4; ++k) mbar_init(&bars[kBarPair0 + k], 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tensormap(&tm_x);
    prefetch_tensormap(&tm_b);
    prefetch_tensormap(&tm_c);
    prefetch_tensormap(&tm_y32);
    prefetch_tensormap(&tm_dt);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem_base;

  if (warp == kIssuerWarp) {
    if ((tid & 31) == 0) issuer_loop<NS>(&tm_x, &tm_b, &tm_c, pb, smem, tmem, bars, abort_flag);
    __syncwarp();  // the issuer warp reconverges before the CTA-wide barrier
  } else if (warp >= kHelperWarp) {
    helper_loop<NS>(&tm_dt, pb, smem, bars, abort_flag, warp - kHelperWarp);
    __syncwarp();
  } else {
    compute_loop<NS>(&tm_y32, pb, smem, tmem, bars, abort_flag);
    if ((tid & 31) == 0) bulk_wait_all();  // this warp's y stores complete before the CTA exits
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (tid == 0 && *abort_flag) atomicOr(pb.status, kStatusTimeout);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(s_tmem_base, kTmemCols);
  }
}

// ----------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 3-D bf16 map {inner, mid, tokens} with a {64, 1, rows} box and 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t tokens,
              uint32_t rows = kTile) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, mid, tokens};
  cuuint64_t strides[2] = {inner * 2, inner * mid * 2};
  cuuint32_t box[3] = {64, 1, rows};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D fp32 map of dt {H, tokens} with a {4 heads, 128 tokens} box (16-byte rows, no swizzle).
bool make_dt_map(CUtensorMap* m, const float* dt, uint64_t H, uint64_t tokens) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {H, tokens};
  cuuint64_t strides[1] = {H * 4};
  cuuint32_t box[2] = {4, (cuuint32_t)kTile};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(dt), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NS>
cudaError_t launch_ns(const Problem& pb, cudaStream_t st) {
  CUtensorMap mx, mb, mc, my, mdt;
  const uint64_t tokens = (uint64_t)pb.tokens;
  if (!make_map(&mx, pb.x, kHeadDim, pb.H, tokens) || !make_map(&mb, pb.B, NS, pb.G, tokens) ||
      !make_map(&mc, pb.C, NS, pb.G, tokens) || !make_map(&my, pb.y, kHeadDim, pb.H, tokens, 32) ||
      !make_dt_map(&mdt, pb.dt, pb.H, tokens))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(ssd_fused_tc_kernel<NS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kDynSmem<NS>);
  if (e != cudaSuccess) {
    if (getenv("SSD_DEBUG")) fprintf(stderr, "ssd: smem attribute failed: %s\n", cudaGetErrorString(e));
    return e;
  }
  // One CTA per SM (at most), each on an equal share of the flat tile list; a flat tile
  // count is not known on the host for packed batches, so the grid covers every SM and
  // ranges may be empty when there are fewer tiles than SMs.
  const int grid = pb.ranges;
  if (grid <= 0) return cudaSuccess;
  e = cudaMemsetAsync(pb.carry_flag, 0, sizeof(int32_t) * (size_t)grid, st);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kDynSmem<NS>;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // all CTAs resident: carry waits always end
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (pb.prof_start) cudaEventRecord(pb.prof_start, st);
  e = cudaLaunchKernelEx(&cfg, ssd_fused_tc_kernel<NS>, mx, mb, mc, my, mdt, pb);
  if (pb.prof_stop) cudaEventRecord(pb.prof_stop, st);
  count_launches(1);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess && getenv("SSD_DEBUG"))
    fprintf(stderr, "ssd: fused kernel launch failed: %s (smem %u, threads %d)\n", cudaGetErrorString(e),
            (unsigned)kDynSmem<NS>, kThreads);
  return e;
}

}  // namespace

bool tc_supports(const ssd_shape* s, int chunk) {
  if (!s || s->io_dtype != SSD_BF16 || s->headdim != kHeadDim) return false;
  if (s->dstate != 64 && s->dstate != 128) return false;
  if (s->nheads % kHeads || (s->nheads / s->ngroups) % kHeads) return false;  // head pairs share a group
  if (s->nheads % 4) return false;  // dt rows of 4 heads (16 bytes) per TMA box
  if (chunk != 128 && chunk != 256) return false;
  const int64_t tokens = s->batch * s->seqlen;
  return tokens >= 1 && tokens < ((int64_t)1 << 31) - kTile;
}

cudaError_t launch_tc(const Problem& pb, cudaStream_t st) {
  return pb.N == 128 ? launch_ns<128>(pb, st) : launch_ns<64>(pb, st);
}

}  // namespace ssd
