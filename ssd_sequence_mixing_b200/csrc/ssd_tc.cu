// ssd_tc.cu -- the tensor-core path: one fused sm_100a kernel for the whole chunked
// SSD forward pass ("Transformers are SSMs", wikillm.com card, Method step 5, sec. 6).
//
// One persistent CTA per SM walks a share of the flat list of 128-token tiles (the
// tcgen05 M) of all units (sequence, pair of heads sharing a B/C group), cut at equal
// shares of a per-tile weight, handing the state on through global memory where its
// share starts or ends inside a unit.
// The P x N state of each head never leaves the chip: it stays in fp32 in tensor
// memory, with a bf16 copy in shared memory as an MMA operand.
//
// Decay factorisation.  Inside a tile, with c_i the inclusive cumsum of dt A (log2 units,
// restarted at the tile start) of one head, the diagonal block needs the factor
// 2^(c_i - c_j) for j <= i.  Around a reference m (per tile and head) it splits into a
// row factor r_i = 2^(c_i - m) and a column factor 2^(m - c_j).  The column factor (with
// dt_j) goes onto x:  U_j = 2^(m - c_j) dt_j x_j, and the row factor into the epilogue.
// What is left of the masked matrix, P = causal(C B^T), no longer depends on the head:
// it is computed once per pair, without exponentials, and both heads' diagonal blocks
// are one N = 128 product P [U_0 | U_1].  The same U feeds the chunk state, which tensor
// memory holds scaled as H = 2^(m - c_start) h (h^, the state in the reference's scale),
// so that one accumulator holds everything a row needs before its factor r_i:
//
//   MMA  S   = C B^T                               (128 x 128, K = N, once per pair)
//   mask     P = bf16(S) on and below the diagonal, 0 above (mask before use)
//   MMA  Y   = C [h^_0 h^_1]^T     left factor     (128 x 128, K = N)
//   MMA  H  += B^T [U_0 | U_1]     right factor    (N x 128, K = 128), H holds h^
//   MMA  Y  += P [U_0 | U_1]       diagonal block  (128 x 128, K = 128, A in tensor memory)
//   state    h_end = 2^(c_end - m) H; at the end of a piece the final state or the
//            hand-on; the bf16 copy of H for the next left factor
//   epilogue y_i = r_i Y_i + D x_i  (bf16, staged over the tile's U, TMA store)
//
// The reference m carries over from tile to tile: in the next tile's cumsum (restarted
// at 0) it is m' = m - c_end, so H accumulates the next right factor as it stands and
// the state step only reads it.  The split needs 2^(m - c_j) and 2^(c_i - m) to stay
// inside the fp32 / bf16 range: while every row of a tile keeps |m - c_j| <= kRangeHalf
// (log2 units) the reference stays; otherwise the pass re-centres it (m = the midpoint
// of its rows' cumsums, H rescaled to match) and, if the tile's rows span more than
// 2 kRangeHalf, the tile is processed in several passes over the same loaded data,
// each over a run of rows whose range fits (on the pages' input distributions,
// 1 - 3 % of tiles).
//
// Roles: 16 compute warps (U, the mask, the state step, the epilogue), one MMA warp
// (every tcgen05.mma), one load warp (every TMA load of x, B, C), one helper warp (dt
// loads, the per-pass descriptors: passes, references, row factors, flags) and, with
// final states only, a scan warp that takes the helper's dt loads and cumsums.
// Tensor memory: two S/P buffers of 128 columns (P is written in place over S),
// Y 128, H 128.  Shared memory: x (two stages; U and then y are written in place),
// a ring of three B/C tiles, the bf16 state, the descriptors, the cumsums and the dt
// stages; with final states only, two U buffers in place of C and the state copy.
// Every wait is bounded; a wait that gives up records SSD_ERR_DEVICE_TIMEOUT in the
// status word, drains what is in flight (bounded), frees tensor memory and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <stdio.h>
#include <stdlib.h>

#include <atomic>

#include "sm100_ptx.cuh"
#include "ssd_tc.cuh"

namespace ssd {

namespace {

using namespace sm100;

constexpr int kTile = 128;          // tokens per tile (UMMA M)
constexpr int kHeadDim = 64;        // P supported by this path
constexpr int kHeads = 2;           // heads of one B/C group processed together
constexpr int kComputeWarps = 16;   // (head, column half, lane quarter)
constexpr int kMmaWarp = kComputeWarps, kLoadWarp = kComputeWarps + 1, kHelperWarp = kComputeWarps + 2,
              kScanWarp = kComputeWarps + 3;
constexpr int kThreads = (kComputeWarps + 4) * 32;
constexpr int kDescSlots = 3;  // pass descriptors the helper may run ahead
constexpr int kDtStages = 4;   // dt tiles in flight
constexpr int kScanSlots = 2;  // (final states only) tiles the scan warp has handed to the helper
constexpr int kRing = 3;       // B / C tiles in shared memory (C(t), B(t) and the next one)
constexpr int kXStages = 2;    // x tiles in shared memory
constexpr int kMaxRanges = 1024;  // CTAs of one launch (one per SM)
constexpr uint32_t kTmemCols = 512;
// TMEM columns: two S/P buffers (S fp32, then P as bf16 pairs in the first 16 columns
// of each 32-column block), Y (64 per head) and the fp32 state H = h^T (64 per head).
constexpr uint32_t kColSP = 0, kColY = 256, kColH = 384;
constexpr float kRangeHalf = 100.f;           // |m - c_j| bound (log2 units): 2^100 stays well inside bf16
constexpr uint32_t kAtom = kTile * 128;       // one 128-row x 128-byte swizzled operand column
// Kernel variants (a template parameter, so each instance carries only its own code):
// y and final states; y added to what y holds (the second column half of N = 256);
// final states only (no C, no y).
enum { kModeFull = 0, kModeAccum = 1, kModeState = 2 };

// mbarriers (index = bit of the 64-bit phase masks)
enum {
  kBarX0 = 0,                         // kXStages: x of a tile in stage s (tx bytes)
  kBarXfree0 = kBarX0 + kXStages,     // kXStages: stage s free again (16 compute arrivals)
  kBarRing0 = kBarXfree0 + kXStages,  // kRing: B or C tile in a ring slot (tx bytes)
  kBarRingFree0 = kBarRing0 + kRing,  // kRing: ring slot free (one UMMA commit)
  kBarS0 = kBarRingFree0 + kRing,     // 2: S = C B^T in S/P buffer b (commit)
  kBarP0 = kBarS0 + 2,                // 2: P written in buffer b (16 arrivals)
  kBarSt = kBarP0 + 2,                // right factor accumulated onto H (commit)
  kBarY,                              // P U accumulated into Y (commit)
  kBarU,                              // U written (16); with final states only, U of even passes
  kBarU1,                             // (final states only) U of odd passes written (16)
  kBarHt,                             // bf16 copy of H written for the left factor (16)
  kBarHRead,                          // H read (and rescaled if needed): the next right factor may add (16)
  kBarFree,                           // Y read by the epilogue (16)
  kBarDrain,                          // the MMA warp's last commit (after its last pass or an abort)
  kBarUFree0,                         // 2: (final states only) U buffer b read by the right factor (commit)
  kBarDt0 = kBarUFree0 + 2,           // kDtStages: dt of a tile (4 heads x 128 tokens)
  kBarDescFull0 = kBarDt0 + kDtStages,           // kDescSlots: descriptor written (helper)
  kBarDescFree0 = kBarDescFull0 + kDescSlots,    // kDescSlots: used up (16 compute + MMA)
  kBarPair0 = kBarDescFree0 + kDescSlots,        // 8: column-half-1 warp of (head, quarter) staged its y
  kBarScanFull0 = kBarPair0 + kHeads * 4,        // kScanSlots: a tile's dt and cumsum written (scan warp)
  kBarScanFree0 = kBarScanFull0 + kScanSlots,    // kScanSlots: the helper is done with the slot
  kNumBars = kBarScanFree0 + kScanSlots
};
static_assert(kNumBars <= 64, "phase bits of a 64-bit mask");
// every group of barriers has its own slots: the next group starts past its last one
static_assert(kBarXfree0 == kBarX0 + kXStages && kBarRing0 == kBarXfree0 + kXStages &&
                  kBarRingFree0 == kBarRing0 + kRing &&
                  kBarS0 == kBarRingFree0 + kRing && kBarP0 == kBarS0 + 2 && kBarSt == kBarP0 + 2 &&
                  kBarDescFull0 == kBarDt0 + kDtStages && kBarDescFree0 == kBarDescFull0 + kDescSlots &&
                  kBarPair0 == kBarDescFree0 + kDescSlots,
              "barrier slots");

// Pass descriptor flags
enum {
  kPFirst = 1,       // first pass of a tile: S / P, x into registers
  kPLast = 2,        // last pass of a tile: its B / C / x may be released
  kPPieceStart = 4,  // the state before this pass is the piece's initial state ...
  kPCarryIn = 8,     // ... handed on by CTA carry_src
  kPToFinal = 16,    // the state after this pass is the unit's final state
  kPToCarry = 32,    // ... is handed on to the next CTA
  kPEnd = 64,        // no pass: the range is done
  kPRescale0 = 128,  // (<< head) re-centred reference: H = sig_in sig_out' H before this pass
  kPRescaleAny = kPRescale0 | (kPRescale0 << 1)
};
struct PassDesc {
  int t0;         // token index of row 0 of the tile
  int rem;        // rows of the tile inside the sequence (1..128)
  int lo, hi;     // rows of this pass
  int s;          // sequence
  int h0;         // first head of the pair
  int flags;
  int carry_src;
  float sig_in[kHeads];   // piece start or re-centred: H = sig_in h before the pass, 2^(m - c_before(lo))
  float sig_out[kHeads];  // h after the pass = sig_out H: 2^(c(hi - 1) - m)
  float dskip[kHeads];    // D
  float pad[2];
  float u[kHeads][kTile];  // 2^(m - c_j) dt_j on the pass's rows, else 0
  float r[kHeads][kTile];  // 2^(c_i - m) on the pass's rows, else 0
};
constexpr uint32_t kDescBytes = (sizeof(PassDesc) + 127) / 128 * 128;
// One tile's c (inclusive cumsum of dt A in log2 units from the tile start) and dt of both
// heads, rows past the tile's end zero.  With y the helper keeps c of the current tile in
// the first slot; with final states only the scan warp hands the helper a ring of them.
struct ScanTile {
  float c[kHeads][kTile];
  float dt[kHeads][kTile];
};
constexpr uint32_t kScanBytes = sizeof(ScanTile);

// Shared memory.  The final-state-only variant (no C, no y, no state copy) spends what
// those take on two U buffers of its own: x is read into registers and its stage released
// at once, and U of the next pass is written while the right factor still reads this one.
template <int NS, int MODE>
struct Layout {
  static constexpr bool kStateOnly = MODE == kModeState;
  static constexpr int kUBufs = kStateOnly ? 2 : 0;                 // U buffers (else U is written over x)
  static constexpr int kRingSlots = kStateOnly ? 2 : kRing;         // B (and C) tiles
  static constexpr uint32_t kSlot = (NS / 64) * kAtom;             // one B or C tile
  static constexpr uint32_t x = 0;                                 // [stage][head] [128 tok][64 p]
  static constexpr uint32_t ub = x + kXStages * kHeads * kAtom;    // [buffer][head] [128 tok][64 p]
  static constexpr uint32_t ring = ub + kUBufs * kHeads * kAtom;   // ring slots [NS/64 atoms][128 tok][64 n]
  static constexpr uint32_t ht = ring + kRingSlots * kSlot;        // [head] [NS n][64 p]
  // For N = 64 the right factor's B^T operand (M = 128) also reads the atom after its ring
  // slot (rows never used); after the last slot that is the state copy, or in the
  // final-state-only variant a pad of one atom, so the read stays inside the CTA's memory.
  static constexpr uint32_t kHtBytes = kStateOnly ? (NS == 64 ? kAtom : 0) : kHeads * NS * 128;
  static constexpr uint32_t desc = ht + kHtBytes;                   // PassDesc[kDescSlots]
  static constexpr uint32_t scan = desc + kDescSlots * kDescBytes; // ScanTile[kScanSlots]
  static constexpr uint32_t sdt = scan + kScanSlots * kScanBytes;  // float[stage][128 tok][4 heads]
  static constexpr uint32_t bars = sdt + kDtStages * kTile * 16;   // uint64[kNumBars]
  static constexpr uint32_t flag = bars + kNumBars * 8;            // int: a wait gave up
  static constexpr uint32_t bytes = flag + 16;
};
template <int NS, int MODE>
constexpr uint32_t kDynSmem = Layout<NS, MODE>::bytes + 1024;  // + base alignment slack
template <int NS, int MODE>
constexpr bool kBtInside = NS != 64 || Layout<NS, MODE>::ring + Layout<NS, MODE>::kRingSlots * Layout<NS, MODE>::kSlot +
                                               kAtom <= Layout<NS, MODE>::desc;
static_assert(kBtInside<64, kModeFull> && kBtInside<64, kModeState> && kBtInside<128, kModeFull> &&
                  kBtInside<128, kModeAccum> && kBtInside<128, kModeState>,
              "the N = 64 B^T operand's second atom lies inside the CTA's shared memory");
static_assert(kDynSmem<128, kModeFull> <= 227 * 1024 && kDynSmem<128, kModeState> <= 227 * 1024,
              "shared memory per CTA");

// Work split.  The tiles of all units (sequence, head pair), unit by unit and each
// unit's 128-token tiles in order, form one flat list; CTA r takes the contiguous
// range that holds share r of R of the tiles' weights (below).  A range may start
// inside a unit (it then needs the state the previous CTA reached there: "carry in")
// and end inside one (it then hands its state on: "carry out").  A CTA processes its
// last, truncated piece first, so the state it hands on is ready early; then the whole
// units; then the piece that needs a carry.  The load, helper and compute roles walk
// the same sequence.
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

// First tile of sequence s in the per-sequence tile prefix (dense batches: every
// sequence has dense_tiles tiles; packed ones: the table kernel's prefix).
__device__ __forceinline__ int64_t seq_tile0(const Problem& pb, int s) {
  return pb.cu ? (int64_t)pb.seq_tiles[s] : (int64_t)s * pb.dense_tiles;
}

__device__ __forceinline__ int unit_tiles(const Problem& pb, int u) {
  const int s = u / (pb.H / kHeads);
  return (int)(seq_tile0(pb, s + 1) - seq_tile0(pb, s));
}

__device__ __noinline__ int64_t unit_first_tile(const Problem& pb, int u) {
  const int pairs = pb.H / kHeads;
  const int s = u / pairs;
  const int64_t a = seq_tile0(pb, s), b = seq_tile0(pb, s + 1);
  return a * pairs + (int64_t)(u % pairs) * (b - a);
}

// The unit holding flat tile w (0 <= w < W).
__device__ __noinline__ int unit_of_tile(const Problem& pb, int64_t w) {
  const int pairs = pb.H / kHeads;
  if (!pb.cu) return (int)(w / pb.dense_tiles);
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

// dt of head h from the stored value; the prologue's softplus is out of line.
__device__ __noinline__ float dt_prologue(const Problem& pb, float v, int h) { return dt_value(pb, v, h); }
__device__ __forceinline__ float dt_of(const Problem& pb, float v, int h) { return pb.dt_prologue ? dt_prologue(pb, v, h) : v; }

// The plan of flat tiles [w0, w1) whose first tile's predecessor is in CTA carry_src's range.
__device__ __noinline__ RangePlan plan_of(const Problem& pb, int64_t w0, int64_t w1, int carry_src) {
  RangePlan rp{};
  if (w0 >= w1) return rp;
  rp.u0 = unit_of_tile(pb, w0);
  rp.k0 = (int)(w0 - unit_first_tile(pb, rp.u0));
  rp.u1 = unit_of_tile(pb, w1 - 1);
  rp.ke1 = (int)(w1 - unit_first_tile(pb, rp.u1));
  rp.npieces = rp.u0 == rp.u1 ? 1 : rp.u1 - rp.u0 + 1;
  rp.carry_src = carry_src;
  return rp;
}

// The cursor at the first tile of the first piece pi' >= pi (processing order) that has
// tiles, or one with piece = -1 when there is none.  Everything is passed and returned by
// value, so the callers' cursors stay in registers.
__device__ __noinline__ TileCursor cursor_from(const Problem& pb, RangePlan rp, int pi) {
  TileCursor c{};
  c.piece = -1;
  for (; pi < rp.npieces; ++pi) {
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
    if (ke <= kb) continue;
    const int s = u / (pb.H / kHeads);
    c.unit = u;
    c.tb = (int)seq_off(pb, s);
    c.len = (int)(seq_off(pb, s + 1) - c.tb);
    c.k0 = kb * kTile;
    c.kend = min(ke * kTile, c.len);
    c.piece = pi;
    const bool unit_end = ke == unit_tiles(pb, u);
    c.flags = (kb > 0 ? kCarryIn : 0) | (unit_end ? kUnitEnd : kCarryOut);
    return c;
  }
  return c;
}

__device__ __forceinline__ bool cursor_first(const Problem& pb, const RangePlan& rp, TileCursor& c) {
  c = cursor_from(pb, rp, 0);
  return c.piece >= 0;
}

// Advances to the next tile of this CTA's range; false when done.
__device__ __forceinline__ bool cursor_next(const Problem& pb, const RangePlan& rp, TileCursor& c) {
  c.k0 += kTile;
  if (c.k0 < c.kend) return true;
  c = cursor_from(pb, rp, c.piece + 1);
  return c.piece >= 0;
}

// One arrival for the whole warp, after every lane's prior work (the lanes' own fences
// come before it).
__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
  __syncwarp();
}

// Bounded wait (at most `limit` SM cycles) that also gives up when another thread has
// recorded a failure.  The spin is out of line: the hot loops stay small enough for the
// instruction cache.
__device__ __noinline__ bool wait_spin(uint64_t* bar, uint32_t parity, volatile int* abort_flag, long long limit) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > limit) {
      *abort_flag = 1;
      return false;
    }
  }
  return true;
}
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                              long long limit) {
  return mbar_try_wait(bar, parity) || wait_spin(bar, parity, abort_flag, limit);
}
// The same for a whole warp (every lane waits; warp-uniform result).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          long long limit) {
  const bool mine = wait_or_abort(bar, parity, abort_flag, limit);
  return !__any_sync(0xffffffffu, !mine);
}

// Phase bookkeeping of one thread (or one warp, waiting uniformly) over all barriers.
struct Phases {
  uint64_t bits = 0;  // bit k: parity of the next phase of bars[k] to wait for
  __device__ __forceinline__ uint32_t parity(int k) const { return (uint32_t)(bits >> k) & 1u; }
  __device__ __forceinline__ void flip(int k) { bits ^= 1ull << k; }
};

// ------------------------------------------------------------------ work split
// The flat tile list is cut at equal shares of a per-tile weight that follows the tile's
// passes, so that CTAs whose units decay strongly (tiles of several passes) or that start
// many short units do not finish last.  A head whose decay across a tile spans more than
// 2 kRangeHalf (log2 units) cuts the tile into passes; such passes write y row by row and
// weigh a little more than a single-pass tile (4 per single-pass tile, 5 per pass of a
// multi-pass tile), and the first tile of a unit adds the cost of starting a piece (6).
// Each CTA first writes the weight bytes of its share of the sequence tiles; the CTAs meet
// once at a flag barrier (all of them are resident: the launch is cooperative); then every
// CTA forms the same prefix sums and takes its own cut points.
constexpr int kSplitVec = 16;     // weights per 16-byte load
struct SplitScratch {             // in the x stages, which the split runs before
  int64_t pre[kThreads + 1];      // weight of the flat tiles before thread t's run
};
static_assert(sizeof(SplitScratch) <= 2 * kHeads * kAtom, "the split's scratch fits in the x stages");
static_assert(sizeof(float4) * kThreads <= 2 * kHeads * kAtom, "the weights' scratch fits in the x stages");

// The (byte) weights of tiles [a, a + 16) into qs, those at or past `end` zeroed; returns
// their sum.
__device__ __forceinline__ int load16(const uint8_t* tw, int64_t a, int64_t end, uint32_t (&qs)[4]) {
  qs[0] = qs[1] = qs[2] = qs[3] = 0u;
  if (a >= end) return 0;
  const uint4 q = __ldcg(reinterpret_cast<const uint4*>(tw + a));
  const uint32_t raw[4] = {q.x, q.y, q.z, q.w};
  const int64_t n = end - a;  // valid weights in this group (> 0)
  uint32_t s = 0;             // (unsigned bytes: weights reach 251)
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int64_t left = n - 4 * k;
    const uint32_t m = left >= 4 ? 0xFFFFFFFFu : left <= 0 ? 0u : (0xFFFFFFFFu >> (8 * (4 - left)));
    qs[k] = raw[k] & m;
    s = __dp4a(qs[k], 0x01010101u, s);
  }
  return (int)s;
}
__device__ __forceinline__ int weights16(const uint8_t* tw, int64_t a, int64_t end) {
  uint32_t qs[4];
  return load16(tw, a, end, qs);
}

// The first tile w of [a, b) whose preceding weight P(w) reaches t (P(a) = before < t), or
// b; *pw = P(w) and *pprev = P(w - 1) (-1 if no tile reaches t).  Whole warp: each lane
// loads 16 weights, a scan over the lanes finds the lane of the cut, and that lane walks
// its weights in registers.  a is a multiple of 16.
__device__ __noinline__ int64_t cut_in(const uint8_t* tw, int64_t a, int64_t b, int64_t before, int64_t t,
                                       int64_t* pw, int64_t* pprev) {
  const int lane = threadIdx.x & 31;
  int64_t acc = before;
  for (int64_t base = a; base < b; base += 32 * kSplitVec) {
    const int64_t lo = base + kSplitVec * lane;
    uint32_t qs[4];
    const int sum = load16(tw, lo, b, qs);
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += x;
    }
    const int64_t mine = acc + incl - sum;  // P(lo)
    // the cut lies in the first lane whose run ends at or past t (P(lo) + sum >= t)
    const uint32_t hit = __ballot_sync(0xffffffffu, lo < b && mine + sum >= t);
    if (hit) {
      const int L = __ffs(hit) - 1;
      // that lane's P(lo) is below t and every weight is positive, so the walk takes at
      // least one tile and stops inside the valid ones
      int64_t w = lo, p = mine, prev = mine;
#pragma unroll
      for (int k = 0; k < kSplitVec; ++k) {
        const int64_t wt = (qs[k >> 2] >> (8 * (k & 3))) & 0xffu;
        if (p < t) prev = p, p += wt, ++w;
      }
      *pw = __shfl_sync(0xffffffffu, p, L);
      *pprev = __shfl_sync(0xffffffffu, prev, L);
      return __shfl_sync(0xffffffffu, w, L);
    }
    acc += __shfl_sync(0xffffffffu, incl, 31);
  }
  *pw = acc;
  *pprev = -1;
  return b;
}

// This CTA's range, cut at equal weight shares (all threads of the CTA).  Thread t sums
// the weights of its run [t per, (t + 1) per) of the flat list, a block scan gives each
// run's preceding weight and the total T, and CTA c's range starts at the first tile
// whose preceding weight reaches ceil(T c / R).  The tile before a CTA's first lies in
// the range of the largest c' with ceil(T c' / R) <= that tile's preceding weight.
__device__ __noinline__ RangePlan split_work(const Problem& pb, SplitScratch* sc) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int R = gridDim.x, r = blockIdx.x;
  const int64_t W = seq_tile0(pb, pb.nseq) * (pb.H / kHeads);
  if (W == 0) return RangePlan{};
  const uint8_t* tw = pb.tile_w;
  const int64_t per = (W + (int64_t)kThreads * kSplitVec - 1) / ((int64_t)kThreads * kSplitVec) * kSplitVec;
  {
    const int64_t a = tid * per, b = a + per < W ? a + per : W;
    int sum = 0;
    for (int64_t v = a; v < b; v += 4 * kSplitVec) {  // four loads in flight
      int s4[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) s4[k] = weights16(tw, v + k * kSplitVec, b);
      sum += s4[0] + s4[1] + s4[2] + s4[3];
    }
    // block scan of the runs' sums: within the warp, then over the warps' totals
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += x;
    }
    if (lane == 31) sc->pre[warp] = incl;  // warp total, scanned below
    __syncthreads();
    if (warp == 0) {
      const int64_t wt = lane < kThreads / 32 ? sc->pre[lane] : 0;
      int64_t wi = wt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int64_t x = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += x;
      }
      __syncwarp();
      if (lane < kThreads / 32) sc->pre[lane] = wi - wt;  // weight before warp `lane`
      if (lane == kThreads / 32 - 1) sc->pre[kThreads] = wi;
    }
    __syncthreads();
    const int64_t before_warp = sc->pre[warp];
    __syncthreads();
    sc->pre[tid] = before_warp + incl - sum;
  }
  __syncthreads();
  __shared__ int64_t s_cut[2], s_at, s_prev;
  const int64_t T = sc->pre[kThreads];
  if (warp < 2) {  // warp 0: this CTA's first tile, warp 1: the next CTA's
    const int c = r + warp;
    int64_t w = W, at = T, prev = -1;
    if (c < R) {
      const int64_t fl = T * c / R;
      const int64_t t = fl + (fl * R < T * c);  // ceil(T c / R)
      int lo = 0, hi = kThreads - 1;  // the last run with pre < t (pre[0] = 0)
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (sc->pre[mid] < t)
          lo = mid;
        else
          hi = mid - 1;
      }
      if (t <= 0) {
        w = 0, at = 0;
      } else {
        const int64_t a = lo * per, b = a + per < W ? a + per : W;
        w = cut_in(tw, a, b, sc->pre[lo], t, &at, &prev);
      }
    }
    if (lane == 0) {
      s_cut[warp] = w;
      if (warp == 0) s_at = at, s_prev = prev;
    }
  }
  __syncthreads();
  __shared__ RangePlan s_rp;
  if (tid == 0) {
    const int64_t w0 = s_cut[0], w1 = s_cut[1];
    int src = 0;
    if (w0 > 0 && w0 < w1) {  // P(w0 - 1) R / T, rounded down
      const int64_t pp = s_prev >= 0 ? s_prev : s_at - (int64_t)__ldcg(tw + (w0 - 1));
      src = (int)(pp * R / T);
    }
    s_rp = plan_of(pb, w0, w1, src);
  }
  __syncthreads();
  return s_rp;
}

// The weight bytes of sequence tile st: one per head pair, from the tile's dt summed per
// head over its tokens (all NTHR threads of the block).  Thread t owns the four heads
// 4 g .. 4 g + 3 (g = t % gn) and the token rows t / gn + k RP (RP = rows covered at
// once), so the tile's rows are read as contiguous 16-byte runs, four in flight, and
// summed in registers; `part` (NTHR float4 of shared memory) combines the row phases.
template <int NTHR>
__device__ __noinline__ void weigh_tile(const Problem& pb, int64_t st, float4* part) {
  const int tid = threadIdx.x;
  const int pairs = pb.H / kHeads, G4 = pb.H / 4;
  int s;
  if (!pb.cu) {
    s = (int)(st / pb.dense_tiles);
  } else {
    int lo = 0, hi = pb.nseq;  // seq_tiles[lo] <= st < seq_tiles[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pb.seq_tiles[mid] <= st)
        lo = mid;
      else
        hi = mid;
    }
    s = lo;
  }
  const int kt = (int)(st - seq_tile0(pb, s));
  const int64_t tb = seq_off(pb, s), len = seq_off(pb, s + 1) - tb;
  const int64_t tok0 = tb + (int64_t)kt * kTile;
  const int ntok = (int)(len - (int64_t)kt * kTile < kTile ? len - (int64_t)kt * kTile : kTile);
  const float4* rows = reinterpret_cast<const float4*>(pb.dt + tok0 * pb.H);  // 16-byte aligned (H % 4 == 0)
  for (int g0 = 0; g0 < G4; g0 += NTHR) {  // (one round unless H > 4 NTHR)
    const int gn = G4 - g0 < NTHR ? G4 - g0 : NTHR, RP = NTHR / gn;
    const int g = g0 + tid % gn, ph = tid / gn;
    if (ph < RP) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int r0 = ph; r0 < ntok; r0 += 4 * RP) {  // four rows in flight
        float4 v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int rr = r0 + k * RP;
          v[k] = rr < ntok ? __ldg(rows + (int64_t)rr * G4 + g) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (r0 + k * RP < ntok) {
            acc.x += dt_of(pb, v[k].x, 4 * g);
            acc.y += dt_of(pb, v[k].y, 4 * g + 1);
            acc.z += dt_of(pb, v[k].z, 4 * g + 2);
            acc.w += dt_of(pb, v[k].w, 4 * g + 3);
          }
        }
      }
      part[ph * gn + tid % gn] = acc;
    }
    __syncthreads();
    if (tid < gn) {  // heads 4 g .. 4 g + 3 (g = g0 + tid): pairs 2 g and 2 g + 1
      float hs[4] = {0.f, 0.f, 0.f, 0.f};
      for (int q = 0; q < RP; ++q) {
        const float4 v = part[q * gn + tid];
        hs[0] += v.x, hs[1] += v.y, hs[2] += v.z, hs[3] += v.w;
      }
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int pr = 2 * g + k, h0 = 2 * pr;
        const float q = fmaxf(fabsf(pb.A[h0] * hs[2 * k]), fabsf(pb.A[h0 + 1] * hs[2 * k + 1])) *
                        (1.4426950408889634f / (2.f * kRangeHalf));
        const int passes = q >= 1.f ? (q < 49.f ? 1 + (int)q : 49) : 1;  // (NaN: 1)
        pb.tile_w[unit_first_tile(pb, s * pairs + pr) + kt] =
            (uint8_t)((passes == 1 ? 4 : 5 * passes) + (kt == 0 ? 6 : 0));
      }
    }
    __syncthreads();
  }
}

// The weights of problems with many sequence tiles per SM, ahead of the fused kernel: one
// block per sequence tile, several resident per SM, so the dt loads of many tiles overlap.
constexpr int kWeightThreads = 512;
__global__ void __launch_bounds__(kWeightThreads) tile_weight_kernel(const __grid_constant__ Problem pb) {
  __shared__ float4 part[kWeightThreads];
  if (pb.cu && *pb.nchunks < 0) return;  // cu_seqlens rejected by the table kernel
  const int64_t seqtiles = seq_tile0(pb, pb.nseq);
  for (int64_t st = blockIdx.x; st < seqtiles; st += gridDim.x) weigh_tile<kWeightThreads>(pb, st, part);
}

// Every CTA's weights are written before any CTA reads them: CTA r sets split_flag[r] to
// this launch's epoch (release) and waits, bounded, until every flag holds it.  The result
// is the same for all threads of the CTA; false if a wait gave up.
__device__ __noinline__ bool weights_barrier(const Problem& pb, volatile int* abort_flag) {
  __syncthreads();  // this CTA's weight bytes are written
  if (threadIdx.x == 0 && !(blockIdx.x == 0 && (pb.withhold_carry & 2))) {
    __threadfence();
    st_release_gpu_u64(&pb.split_flag[blockIdx.x], pb.epoch);
  }
  bool ok = true;
  for (int k = threadIdx.x; k < (int)gridDim.x && ok; k += kThreads) {
    const long long t0 = clock64();
    while (ld_acquire_gpu_u64(&pb.split_flag[k]) != pb.epoch) {
      if (clock64() - t0 > pb.wait_limit) {
        ok = false;
        break;
      }
      __nanosleep(32);
    }
  }
  if (!ok) *abort_flag = 1;
  __threadfence();
  __syncthreads();
  return !*abort_flag;
}

// ------------------------------------------------------------------ load warp
template <int NS, int MODE>
__device__ void load_loop(const CUtensorMap* tm_x, const CUtensorMap* tm_b, const CUtensorMap* tm_c,
                          const Problem& pb, const RangePlan& rp, uint8_t* smem, uint64_t* bars,
                          volatile int* abort_flag) {
  using L = Layout<NS, MODE>;
  Phases ph;
  auto wait = [&](int k) -> bool {
    if (!wait_or_abort(&bars[k], ph.parity(k), abort_flag, pb.wait_limit)) return false;
    ph.flip(k);
    return true;
  };
  const int pairs = pb.H / kHeads;
  TileCursor cur;
  bool have = cursor_first(pb, rp, cur);
  uint32_t nring = 0;  // ring loads issued
  int t = 0;
  bool ok = true;
  // last issued load per barrier (parity of its phase), for the drain after an abort
  uint64_t issued = 0, issued_par = 0;
  auto note = [&](int k, uint32_t par) {
    issued |= 1ull << k;
    issued_par = (issued_par & ~(1ull << k)) | ((uint64_t)par << k);
  };
  auto ring_load = [&](const CUtensorMap* tm, int g, int tok) -> bool {
    const int slot = nring % L::kRingSlots;
    if (nring >= (uint32_t)L::kRingSlots && !wait(kBarRingFree0 + slot)) return false;
    uint8_t* dst = smem + L::ring + slot * L::kSlot;
    mbar_expect_tx(&bars[kBarRing0 + slot], L::kSlot);
#pragma unroll
    for (int a = 0; a < NS / 64; ++a) tma_load_3d(dst + a * kAtom, tm, a * 64, g, tok, &bars[kBarRing0 + slot]);
    note(kBarRing0 + slot, (nring / L::kRingSlots) & 1u);
    ++nring;
    return true;
  };
  constexpr bool state_only = MODE == kModeState;  // no y: C is not needed
  while (have) {
    const int h0 = (cur.unit % pairs) * kHeads, g = h0 / pb.hpg, tok = cur.tb + cur.k0;
    // C(t) goes into the slot B(t-2) held, x(t) into stage t & 1 once tile t-2's y is
    // out of it, B(t) into the slot C(t-1) held (free once the left factor of t-1 is done)
    if (!state_only && !(ok = ring_load(tm_c, g, tok))) break;
    const int st = t % kXStages;
    if (t >= kXStages && !(ok = wait(kBarXfree0 + st))) break;
    mbar_expect_tx(&bars[kBarX0 + st], kHeads * kAtom);
#pragma unroll
    for (int hh = 0; hh < kHeads; ++hh)
      tma_load_3d(smem + L::x + (st * kHeads + hh) * kAtom, tm_x, 0, h0 + hh, tok, &bars[kBarX0 + st]);
    note(kBarX0 + st, (uint32_t)(t / kXStages) & 1u);
    if (!(ok = ring_load(tm_b, g, tok))) break;
    ++t;
    have = cursor_next(pb, rp, cur);
  }
  if (!ok) {
    *abort_flag = 1;
    // loads still in flight land before the CTA ends (bounded)
    for (int k = 0; k < kNumBars; ++k)
      if (issued & (1ull << k)) mbar_wait_bounded(&bars[k], (uint32_t)(issued_par >> k) & 1u, pb.wait_limit);
  }
}

// ------------------------------------------------------------------ MMA warp
// The whole warp walks the passes (so every operand is warp-uniform); one elected lane
// issues each tcgen05.mma and commit.
template <int NS, int MODE>
__device__ void mma_loop(const Problem& pb, uint8_t* smem, uint32_t tmem, uint64_t* bars,
                         volatile int* abort_flag) {
  using L = Layout<NS, MODE>;
  const uint32_t id_s = idesc_bf16(128, 128, 0, 0);   // C (K-major) x B (K-major)
  const uint32_t id_y = idesc_bf16(128, 128, 0, 1);   // C or P x (N-major h^ / U)
  const uint32_t id_h = idesc_bf16(128, 128, 1, 1);   // B^T (M-major) x U (N-major)
  // Descriptors differ only in the start address field (address / 16, low bits), so a
  // K step adds its byte offset / 16 to the operand's base descriptor.
  const uint64_t k_major = sdesc_sw128(0, 16, 1024), mn_major = sdesc_sw128(0, kAtom, 1024);
  const uint64_t ht_major = sdesc_sw128(0, NS * 128, 1024);
  auto at = [](uint64_t tmpl, uint32_t addr) { return tmpl | (uint64_t)(addr >> 4); };
  const uint32_t a_ht = smem_u32(smem + L::ht);
  const PassDesc* descs = reinterpret_cast<const PassDesc*>(smem + L::desc);
  const bool leader = elect_one();
  // For N = 64 the B^T operand has one M atom; the second (unused) half of H^T reads
  // the next ring slot or the state copy after it, and those lanes are never read.
  Phases ph;
  auto wait = [&](int k) -> bool {
    if (!warp_wait(&bars[k], ph.parity(k), abort_flag, pb.wait_limit)) return false;
    ph.flip(k);
    return true;
  };
  auto commit = [&](int k) {
    if (leader) umma_commit(&bars[k]);
  };
  // H += B^T [U_0 | U_1] (K = 128 tokens, 8 steps of 16 rows = 2048 bytes)
  auto right_factor = [&](uint64_t db, uint64_t dx) {
    if (leader) {
#pragma unroll 1
      for (int kk = 0; kk < kTile / 16; ++kk) umma_f16(tmem + kColH, db + kk * 128, dx + kk * 128, id_h, 1);
    }
  };
  constexpr bool state_only = MODE == kModeState;  // only the right factor: no S, P, Y
  bool ok = true, issued_any = false;
  int prev_flags = 0;  // (final states only) the previous pass's flags
  int t = -1;
  uint32_t c_slot = 0, b_slot = 0;
  uint64_t dc = 0, db = 0, dbm = 0, dx = 0;
  for (int p = 0;; ++p) {
    const int ds = p % kDescSlots;
    if (!(ok = wait(kBarDescFull0 + ds))) break;
    const PassDesc& d = descs[ds];
    const int flags = d.flags;
    if (flags & kPEnd) break;
    if (flags & kPFirst) {
      ++t;
      c_slot = (2 * t) % kRing;
      b_slot = state_only ? t % L::kRingSlots : (2 * t + 1) % kRing;
      const uint32_t a_c = smem_u32(smem + L::ring + c_slot * L::kSlot);
      const uint32_t a_b = smem_u32(smem + L::ring + b_slot * L::kSlot);
      dc = at(k_major, a_c);
      db = at(k_major, a_b);
      dbm = at(mn_major, a_b);
      dx = at(mn_major, smem_u32(smem + L::x + (t % kXStages) * kHeads * kAtom));
      if (!state_only && !(ok = wait(kBarRing0 + c_slot))) break;
      if (!(ok = wait(kBarRing0 + b_slot))) break;
    }
    if (state_only) {  // H += B^T [U_0 | U_1] onto h^, U from buffer p & 1
      // the compute warps touch H only after a pass that ends a piece or before one that
      // starts or re-centres a state; only then does the product wait for them
      const bool touched = (prev_flags & (kPToFinal | kPToCarry)) || (flags & (kPPieceStart | kPRescaleAny));
      prev_flags = flags;
      if (touched && !(ok = wait(kBarHRead))) break;
      if (!(ok = wait(kBarU + (p & 1)))) break;
      tc_fence_after();
      right_factor(dbm, at(mn_major, smem_u32(smem + L::ub + (p & 1) * kHeads * kAtom)));
      commit(kBarUFree0 + (p & 1));  // U buffer free, and H holds this pass
      if (flags & kPLast) commit(kBarRingFree0 + b_slot);
      issued_any = true;
      if (leader) mbar_arrive(&bars[kBarDescFree0 + ds]);
      continue;
    }
    if (flags & kPFirst) {
      tc_fence_after();
      // S = C B^T into buffer t & 1 (the diagonal product that read P(t - 2) from it was
      // issued earlier by this warp, and tcgen05.mma executes in issue order); K step kk
      // (16 state columns) is 32 bytes into 64-column atom kk / 4
      const uint32_t d_s = tmem + kColSP + (t & 1) * 128;
      if (leader) {
#pragma unroll 1
        for (int kk = 0; kk < NS / 16; ++kk) {
          const uint32_t koff = ((kk >> 2) * kAtom + (kk & 3) * 32) >> 4;
          umma_f16(d_s, dc + koff, db + koff, id_s, kk > 0);
        }
      }
      commit(kBarS0 + (t & 1));
      issued_any = true;
    }
    // left factor Y = C [h^_0 h^_1]^T: needs the bf16 copy of H and the previous
    // epilogue done with Y
    if (!(ok = wait(kBarHt))) break;
    if (p > 0 && !(ok = wait(kBarFree))) break;
    tc_fence_after();
    if (leader) {
      const uint64_t dh = at(ht_major, a_ht);
#pragma unroll 1
      for (int kk = 0; kk < NS / 16; ++kk) {
        const uint32_t koff = ((kk >> 2) * kAtom + (kk & 3) * 32) >> 4;
        umma_f16(tmem + kColY, dc + koff, dh + kk * 128, id_y, kk > 0);
      }
    }
    if (flags & kPLast) commit(kBarRingFree0 + c_slot);  // C(t) read for the last time
    // right factor H += B^T [U_0 | U_1]: needs U and the state step done reading H
    if (!(ok = wait(kBarU)) || !(ok = wait(kBarHRead))) break;
    tc_fence_after();
    right_factor(dbm, dx);
    commit(kBarSt);
    if (flags & kPLast) commit(kBarRingFree0 + b_slot);  // B(t) read for the last time
    // diagonal block Y += P [U_0 | U_1], P from tensor memory: K step kk (16 tokens) is
    // 8 columns at 32 (kk / 2) + 8 (kk % 2) of the buffer
    if ((flags & kPFirst) && !(ok = wait(kBarP0 + (t & 1)))) break;
    tc_fence_after();
    if (leader) {
      const uint32_t a_p = tmem + kColSP + (t & 1) * 128;
#pragma unroll 1
      for (int kk = 0; kk < kTile / 16; ++kk)
        umma_f16_ta(tmem + kColY, a_p + 32 * (kk >> 1) + 8 * (kk & 1), dx + kk * 128, id_y, 1);
    }
    commit(kBarY);
    if (leader) mbar_arrive(&bars[kBarDescFree0 + ds]);
  }
  if (!ok) *abort_flag = 1;
  // every tcgen05.mma this warp issued completes before tensor memory is freed
  if (issued_any) {
    commit(kBarDrain);
    if (!mbar_wait_bounded(&bars[kBarDrain], 0, pb.wait_limit)) *abort_flag = 1;
  }
}

// --------------------------------------------------------- compute warps
// Warp w: lane quarter q = w % 4 (TMEM lanes / tile rows 32 q .. 32 q + 31, or state
// rows n), head hw = w / 8 and column half ch = (w / 4) % 2 of that head's Y, U and
// state columns; of the mask it converts the 32 x 32 block (q, 2 hw + ch) of S.
// What is the same for every row of a pass (where it is, the factors, the flags)
// comes from the helper warp's descriptor.  The two halves of a row quarter meet
// once a pass, on a one-arrival barrier, before the half-0 warp stores their 32 rows
// of y by TMA.  Every wait is warp-uniform and bounded.  The rare paths (initial
// states, hand-ons, final states, empty units) are out-of-line functions, so the
// per-pass loop stays small enough for the instruction cache.

// Where this warp's part of the state (row n = i, columns 32 ch .. 32 ch + 31 of head hw)
// lives in memory: state row (s, h, p) is n_stride long and this launch owns its columns
// [n_off, n_off + N); hand-ons are N long per row, one block per CTA.
__device__ __forceinline__ int64_t state_index(const Problem& pb, int s, int h, int ch, int i) {
  return ((int64_t)s * pb.H + h) * kHeadDim * pb.n_stride + pb.n_off + (int64_t)(32 * ch) * pb.n_stride + i;
}
__device__ __forceinline__ int64_t carry_index(const Problem& pb, int cta, int hw, int ch, int i) {
  return ((int64_t)cta * kHeads + hw) * kHeadDim * pb.N + (int64_t)(32 * ch) * pb.N + i;
}

// Units whose sequences are empty have no tiles: CTA r writes final = init (or 0) for
// the empty units u with u % R == r.
__device__ __noinline__ void empty_unit_states(const Problem& pb, int hw, int ch, int i) {
  if (!pb.final_state || i >= pb.N) return;
  const int pairs = pb.H / kHeads, units = pb.nseq * pairs;
  for (int u = blockIdx.x; u < units; u += gridDim.x) {
    if (unit_tiles(pb, u) != 0) continue;
    const int64_t at = state_index(pb, u / pairs, (u % pairs) * kHeads + hw, ch, i);
    float v[32];  // every load in flight before the first store
#pragma unroll
    for (int k = 0; k < 32; ++k) v[k] = pb.init ? __ldg(pb.init + at + (int64_t)k * pb.n_stride) : 0.f;
#pragma unroll
    for (int k = 0; k < 32; ++k) pb.final_state[at + (int64_t)k * pb.n_stride] = v[k];
  }
}

// The state at the start of the piece whose first pass d describes, times `scale`, into
// tensor memory at t_state: the sequence's initial state (or zero), or the state CTA
// d.carry_src handed on (each warp waits for the matching warp of that CTA).  Whole warp;
// the values stay in registers, all 32 loads in flight at once.  False if the wait gave up.
__device__ __noinline__ bool fetch_state(const Problem& pb, const PassDesc& d, int hw, int ch, int i, int wid,
                                         volatile int* abort_flag, uint32_t t_state, float scale) {
  const float* src = nullptr;
  int stride = pb.n_stride;
  if (d.flags & kPCarryIn) {
    bool mine = true;
    if ((threadIdx.x & 31) == 0) {
      const long long t0 = clock64();
      while (ld_acquire_gpu_u64(&pb.carry_flag[d.carry_src * kComputeWarps + wid]) != pb.epoch) {
        if (*abort_flag || clock64() - t0 > pb.wait_limit) {
          *abort_flag = 1;
          mine = false;
          break;
        }
        __nanosleep(100);
      }
    }
    if (__any_sync(0xffffffffu, !mine)) return false;
    __threadfence();
    src = pb.carry + carry_index(pb, d.carry_src, hw, ch, i);
    stride = pb.N;
  } else if (pb.init) {
    src = pb.init + state_index(pb, d.s, d.h0 + hw, ch, i);
  }
  if (!src || i >= pb.N) src = nullptr;
  float v[32];
#pragma unroll
  for (int k = 0; k < 32; ++k) v[k] = src ? __ldcg(src + (int64_t)k * stride) : 0.f;
  uint32_t r[32];
#pragma unroll
  for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(v[k] * scale);
  tmem_st32(t_state, r);
  tmem_st_wait();
  return true;
}

// The state after the pass d describes, h = scale H (H from tensor memory at t_state), as
// the unit's final state or as the hand-on to the next CTA (then released to it, one flag
// per warp).  Whole warp; the values stay in registers.
__device__ __noinline__ void put_state(const Problem& pb, const PassDesc& d, int hw, int ch, int i, int wid,
                                       uint32_t t_state, float scale) {
  uint32_t r[32];
  tmem_ld32(t_state, r);
  tmem_ld_wait();
  const bool to_final = d.flags & kPToFinal;
  if (i < pb.N) {
    float* dst = to_final ? pb.final_state + state_index(pb, d.s, d.h0 + hw, ch, i)
                          : pb.carry + carry_index(pb, blockIdx.x, hw, ch, i);
    const int64_t stride = to_final ? pb.n_stride : pb.N;
#pragma unroll
    for (int k = 0; k < 32; ++k) dst[k * stride] = __uint_as_float(r[k]) * scale;
  }
  if (!to_final) {
    __threadfence();
    __syncwarp();
    if ((threadIdx.x & 31) == 0 && !(pb.withhold_carry & 1))
      st_release_gpu_u64(&pb.carry_flag[blockIdx.x * kComputeWarps + wid], pb.epoch);
    __syncwarp();
  }
}

__device__ __forceinline__ void scale32(uint32_t (&r)[32], float f) {
#pragma unroll
  for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * f);
}

template <int NS, int MODE>
__device__ void compute_loop(const CUtensorMap* tm_y32, const Problem& pb, uint8_t* smem, uint32_t tmem,
                             uint64_t* bars, volatile int* abort_flag) {
  using L = Layout<NS, MODE>;
  const int tid = threadIdx.x;
  const int wid = tid >> 5;
  const int hw = wid >> 3;                   // head of the pair
  const int ch = (wid >> 2) & 1;             // column half
  const int q = wid & 3, lane = tid & 31;    // lane quarter
  const int kb = wid >> 2;                   // S block column of the mask
  const int i = q * 32 + lane;               // row / TMEM lane
  const int pair_bar = kBarPair0 + hw * 4 + q;
  const uint32_t lane_base = (uint32_t)(q * 32) << 16;
  const uint32_t col_h = hw * 64 + ch * 32;  // this warp's Y and state columns
  uint8_t* sx = smem + L::x;
  uint8_t* sht = smem + L::ht + hw * NS * 128;  // this head's bf16 copy of H
  const PassDesc* descs = reinterpret_cast<const PassDesc*>(smem + L::desc);

  Phases ph;
  auto wait = [&](int k) -> bool {
    if (!warp_wait(&bars[k], ph.parity(k), abort_flag, pb.wait_limit)) return false;
    ph.flip(k);
    return true;
  };
  // Final states only: the right factor of pass q completes phase q / 2 of U-free barrier
  // q & 1.  Each phase is waited for once, in order: before U(q + 2) is written into the
  // buffer, or earlier, where pass q ends a piece or precedes a re-centred / new state and
  // H is read.  Either wait comes after this warp's wait for phase q / 2 - 1 and before it
  // hands U(q + 2) to the MMA warp, so the barrier is never a phase behind or two past it.
  int uf_waited[2] = {0, 0};  // phases of U-free barrier b this warp has waited for
  auto wait_uf = [&](int q) -> bool {
    const int b = q & 1, k = q >> 1;
    if (uf_waited[b] > k) return true;
    if (!warp_wait(&bars[kBarUFree0 + b], (uint32_t)k & 1u, abort_flag, pb.wait_limit)) return false;
    uf_waited[b] = k + 1;
    return true;
  };

  empty_unit_states(pb, hw, ch, i);

  // The head state lives in tensor memory as H = h^T (lane n = state column n, 64 fp32
  // columns per head, 32 per half) in the scale of the pass reference; its bf16 copy in
  // shared memory is the B operand of the left factor.
  const uint32_t t_state = tmem + lane_base + kColH + col_h;
  constexpr bool state_only = MODE == kModeState;  // only the final states: no mask, no epilogue
  auto write_copy = [&](const uint32_t (&r)[32]) {
    if constexpr (state_only) return;
    if (i >= NS) return;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float* v = reinterpret_cast<const float*>(r) + 8 * c;
      const uint4 hv = make_uint4(bf16x2(v[0], v[1]), bf16x2(v[2], v[3]), bf16x2(v[4], v[5]), bf16x2(v[6], v[7]));
      *reinterpret_cast<uint4*>(sht + sw128_off(i, 4 * ch + c)) = hv;
    }
  };
  // Installs the state before the pass d describes: the piece's initial state (a new
  // piece) or H rescaled to d's reference (sig_out of the pass before, then sig_in), into
  // tensor memory and r.  False if fetching the initial state gave up.
  auto install = [&](const PassDesc& d, float sig_prev, uint32_t (&r)[32]) -> bool {
    if (d.flags & kPPieceStart) {
      if (!fetch_state(pb, d, hw, ch, i, wid, abort_flag, t_state, d.sig_in[hw])) return false;
      if (!state_only) {  // r: the installed H, for its bf16 copy
        tmem_ld32(t_state, r);
        tmem_ld_wait();
      }
      return true;
    }
    scale32(r, sig_prev);
    scale32(r, d.sig_in[hw]);
    tmem_st32(t_state, r);
    tmem_st_wait();
    return true;
  };

  if (!wait(kBarDescFull0)) return;
  if (descs[0].flags & kPEnd) return;
  {
    uint32_t r[32];
    if (!install(descs[0], 1.f, r)) return;
    tc_fence_before();
    warp_arrive(&bars[kBarHRead]);
    write_copy(r);
  }
  fence_proxy_async();
  if (!state_only) warp_arrive(&bars[kBarHt]);

  uint32_t xr[16];  // this thread's x of the current tile: row i, columns 32 ch .. 32 ch + 31 of head hw
  int t = -1;
  bool staged_prev = false;  // the previous tile's y went out by TMA from its x stage
  for (int p = 0;; ++p) {
    const int ds = p % kDescSlots;
    const PassDesc& d = descs[ds];
    const int flags = d.flags;
    if (flags & kPFirst) ++t;
    const int st = t % kXStages;
    uint8_t* sxh = sx + (st * kHeads + hw) * kAtom;

    // ---- U = u_i x_i over the tile's x, in place (x itself stays in registers); with
    // final states only, into U buffer p & 1 once the right factor of pass p - 2 has read it
    if (flags & kPFirst) {
      if (!wait(kBarX0 + st)) return;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 v = *reinterpret_cast<const uint4*>(sxh + sw128_off(i, 4 * ch + c));
        xr[4 * c] = v.x, xr[4 * c + 1] = v.y, xr[4 * c + 2] = v.z, xr[4 * c + 3] = v.w;
      }
      if (state_only) warp_arrive(&bars[kBarXfree0 + st]);  // x is in registers: the stage may refill
    }
    uint8_t* suh = sxh;
    if constexpr (state_only) {
      suh = smem + L::ub + ((p & 1) * kHeads + hw) * kAtom;
      if (p >= 2 && !wait_uf(p - 2)) return;
    }
    {
      const float u = d.u[hw][i];
      const uint32_t u2 = pack_bf16(u, u);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint4 v;
        v.x = mul_bf16x2(xr[4 * c], u2);
        v.y = mul_bf16x2(xr[4 * c + 1], u2);
        v.z = mul_bf16x2(xr[4 * c + 2], u2);
        v.w = mul_bf16x2(xr[4 * c + 3], u2);
        *reinterpret_cast<uint4*>(suh + sw128_off(i, 4 * ch + c)) = v;
      }
    }
    // (final states only: one barrier per buffer, so an arrival for pass p + 1 never counts
    // toward pass p; one for pass p + 2 comes after the right factor of pass p)
    fence_proxy_async();
    warp_arrive(&bars[kBarU + (state_only ? (p & 1) : 0)]);

    if ((flags & kPFirst) && t > 0 && !state_only) {
      // the previous tile's x stage: its y store has read it, so it may take tile t + 1's x
      if (staged_prev && ch == 0 && lane == 0) bulk_wait_read();
      warp_arrive(&bars[kBarXfree0 + (st + kXStages - 1) % kXStages]);
    }
    // ---- P = bf16(S) on and below the diagonal, written in place over S: block (q, kb)
    // is kept whole below the diagonal (kb < q), lower-triangular on it, zero above
    if ((flags & kPFirst) && !state_only) {
      if (!wait(kBarS0 + (t & 1))) return;
      tc_fence_after();
      const uint32_t t_blk = tmem + lane_base + kColSP + (t & 1) * 128 + kb * 32;
      uint32_t pk[16];
      if (kb > q) {
#pragma unroll
        for (int k = 0; k < 16; ++k) pk[k] = 0u;
      } else {
        uint32_t sv[32];
        tmem_ld32(t_blk, sv);
        tmem_ld_wait();
        if (kb == q) {  // on the diagonal: column j of row lane kept for j <= lane
#pragma unroll
          for (int k = 0; k < 32; ++k) sv[k] = k <= lane ? sv[k] : 0u;
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) pk[k] = bf16x2(__uint_as_float(sv[2 * k]), __uint_as_float(sv[2 * k + 1]));
      }
      tmem_st16(t_blk, pk);
      tmem_st_wait();
      tc_fence_before();
      warp_arrive(&bars[kBarP0 + (t & 1)]);
    }

    // ---- the state after this pass: at the end of a piece the final state or the
    // hand-on; then the next pass's H (as it stands, or re-centred, or the next piece's
    // initial state) and its bf16 copy
    const int nds = (p + 1) % kDescSlots;
    if constexpr (state_only) {  // H is read only where a piece ends or the next pass resets it
      if (!wait(kBarDescFull0 + nds)) return;
      const PassDesc& dn = descs[nds];
      const bool more = !(dn.flags & kPEnd);
      const bool out = flags & (kPToFinal | kPToCarry);
      const bool reset = more && (dn.flags & (kPPieceStart | (kPRescale0 << hw)));
      const bool touched = out || (more && (dn.flags & (kPPieceStart | kPRescaleAny)));  // same for all warps
      // On such a pass every warp waits for the pass's right factor before it arrives on
      // "H read": then no warp can arrive for the next such pass while another has not yet
      // arrived for this one, and the MMA warp waits for it on exactly these passes.
      if (touched) {
        if (!wait_uf(p)) return;
        tc_fence_after();
        if (out) put_state(pb, d, hw, ch, i, wid, t_state, d.sig_out[hw]);
        if (reset) {
          uint32_t r[32];
          tmem_ld32(t_state, r);
          tmem_ld_wait();
          if (!install(dn, d.sig_out[hw], r)) return;
        }
        tc_fence_before();
        warp_arrive(&bars[kBarHRead]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarDescFree0 + ds]);
      __syncwarp();
      if (!more) break;
      continue;
    }
    if (!wait(kBarSt)) return;
    tc_fence_after();
    bool more;
    {
      if (flags & (kPToFinal | kPToCarry)) put_state(pb, d, hw, ch, i, wid, t_state, d.sig_out[hw]);
      uint32_t r[32];
      tmem_ld32(t_state, r);
      tmem_ld_wait();
      if (!wait(kBarDescFull0 + nds)) return;
      const PassDesc& dn = descs[nds];
      more = !(dn.flags & kPEnd);
      if (more && (dn.flags & (kPPieceStart | (kPRescale0 << hw))) && !install(dn, d.sig_out[hw], r)) return;
      tc_fence_before();
      warp_arrive(&bars[kBarHRead]);
      if (more) write_copy(r);
    }
    fence_proxy_async();
    warp_arrive(&bars[kBarHt]);

    // ---- epilogue: y = r_i Y + D x; a single-pass tile stages y over its U and the
    // half-0 warp of each row quarter stores the quarter's 32 rows by TMA once the
    // half-1 warp has staged its columns; other rows go out as row stores
    if (!wait(kBarY)) return;
    tc_fence_after();
    const bool single = (flags & (kPFirst | kPLast)) == (kPFirst | kPLast);
    const bool staged = single && d.rem >= 32 * q + 32;  // all 32 rows of this quarter are in the sequence
    {
      uint32_t ry[32];
      tmem_ld32(tmem + lane_base + kColY + col_h, ry);
      const float rr = d.r[hw][i];
      const float Dh = d.dskip[hw];
      const int h = d.h0 + hw;
      const bool in_pass = i >= d.lo && i < d.hi && i < d.rem;
      const bool row_out = !staged && in_pass;
      const bool add_prev = MODE == kModeAccum && in_pass;  // y of the other state columns
      __nv_bfloat16* yrow = static_cast<__nv_bfloat16*>(pb.y) + ((int64_t)(d.t0 + i) * pb.H + h) * kHeadDim + 32 * ch;
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t out[4];
        uint4 prev = make_uint4(0u, 0u, 0u, 0u);
        if (add_prev) prev = *reinterpret_cast<const uint4*>(yrow + 8 * c);
        const uint32_t pv[4] = {prev.x, prev.y, prev.z, prev.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {  // r Y + D x (+ y so far), x from its bf16 pair (exact)
          const uint32_t xu = xr[4 * c + k];
          float lo = fmaf(rr, __uint_as_float(ry[8 * c + 2 * k]), Dh * bf16_lo(xu));
          float hi = fmaf(rr, __uint_as_float(ry[8 * c + 2 * k + 1]), Dh * bf16_hi(xu));
          if (MODE == kModeAccum) lo += bf16_lo(pv[k]), hi += bf16_hi(pv[k]);
          out[k] = bf16x2(lo, hi);
        }
        const uint4 ov = make_uint4(out[0], out[1], out[2], out[3]);
        if (staged)
          *reinterpret_cast<uint4*>(sxh + sw128_off(i, 4 * ch + c)) = ov;
        else if (row_out)
          *reinterpret_cast<uint4*>(yrow + 8 * c) = ov;
      }
      tc_fence_before();
      if (staged) fence_proxy_async();
      __syncwarp();
      if (ch == 1) {
        if (lane == 0) mbar_arrive(&bars[pair_bar]);
      } else {
        if (!wait(pair_bar)) return;
        if (staged && lane == 0) {
          tma_store_3d(tm_y32, sxh + q * 32 * 128, 0, h, d.t0 + 32 * q);
          bulk_commit();
        }
      }
      __syncwarp();
    }
    if (flags & kPLast) staged_prev = staged;
    // Y is free for the next left factor; this pass's descriptor is used up
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&bars[kBarFree]);
      mbar_arrive(&bars[kBarDescFree0 + ds]);
    }
    __syncwarp();
    if (!more) break;
  }
}

// ------------------------------------------------------------------ scan warp
// With final states only, a warp of its own loads each tile's dt by TMA into a ring
// (kDtStages tiles in flight) and hands the helper both heads' dt and c, the inclusive
// cumsum of dt A in log2 units from the tile start, through a ring of kScanSlots.
struct ScanState {
  TileCursor ahead, cur;  // dt loads run up to kDtStages tiles ahead on a cursor of their own
  bool have_ahead, have;
  int dt_issued, t, a_unit;
  float a2[kHeads];  // A log2(e) of the current unit's heads
  Phases ph;         // dt barriers (and, in the scan warp, the slots' barriers)
};

template <int NS, int MODE>
__device__ __forceinline__ void scan_issue_dt(ScanState& S, const CUtensorMap* tm_dt, const Problem& pb,
                                              const RangePlan& rp, uint8_t* smem, uint64_t* bars) {
  using L = Layout<NS, MODE>;
  if ((threadIdx.x & 31) == 0) {
    const int st = S.dt_issued % kDtStages;
    const int h0 = (S.ahead.unit % (pb.H / kHeads)) * kHeads;
    mbar_expect_tx(&bars[kBarDt0 + st], kTile * 16);
    tma_load_2d(smem + L::sdt + st * kTile * 16, tm_dt, h0 & ~3, S.ahead.tb + S.ahead.k0, &bars[kBarDt0 + st]);
  }
  ++S.dt_issued;
  S.have_ahead = cursor_next(pb, rp, S.ahead);
}

template <int NS, int MODE>
__device__ void scan_init(ScanState& S, const CUtensorMap* tm_dt, const Problem& pb, const RangePlan& rp,
                          uint8_t* smem, uint64_t* bars) {
  S.have_ahead = cursor_first(pb, rp, S.ahead);
  S.have = cursor_first(pb, rp, S.cur);
  S.dt_issued = S.t = 0;
  S.a_unit = -1;
  S.a2[0] = S.a2[1] = 0.f;
  for (int k = 0; k < kDtStages && S.have_ahead; ++k) scan_issue_dt<NS, MODE>(S, tm_dt, pb, rp, smem, bars);
}

// The scan step of tile S.t (S.have): lane's rows 4 lane .. 4 lane + 3 of c and dt into
// cth and dtt, c also into o.c and, if `with_dt`, dt into o.dt; then on to the next tile.
// Whole warp; false if the dt wait gave up.
template <int NS, int MODE>
__device__ __forceinline__ bool scan_tile(ScanState& S, float (&cth)[kHeads][4], float (&dtt)[kHeads][4],
                                          ScanTile& o, bool with_dt, const CUtensorMap* tm_dt, const Problem& pb,
                                          const RangePlan& rp, uint8_t* smem, uint64_t* bars,
                                          volatile int* abort_flag) {
  using L = Layout<NS, MODE>;
  const int lane = threadIdx.x & 31;
  const TileCursor& cur = S.cur;
  const int h0 = (cur.unit % (pb.H / kHeads)) * kHeads;
  if (cur.unit != S.a_unit) {
    S.a_unit = cur.unit;
#pragma unroll
    for (int hh = 0; hh < kHeads; ++hh) S.a2[hh] = pb.A[h0 + hh] * 1.4426950408889634f;  // log2 units
  }
  const int rem = min(kTile, cur.len - cur.k0);
  const int dst = S.t % kDtStages;
  if (!warp_wait(&bars[kBarDt0 + dst], S.ph.parity(kBarDt0 + dst), abort_flag, pb.wait_limit)) return false;
  S.ph.flip(kBarDt0 + dst);
  // row 4 lane + j holds the 4 heads' dt of one token; a lane reads its rows in the order
  // j = (k + rot) & 3, rot = (lane / 2) & 3, so each quarter warp's 16-byte loads fall in
  // distinct banks
  {
    const float4* rows = reinterpret_cast<const float4*>(smem + L::sdt + dst * kTile * 16) + 4 * lane;
    const int rot = (lane >> 1) & 3, c0 = h0 & 3;  // the pair's first column in the 4-head row
    float v0[4], v1[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float4 qv = rows[(k + rot) & 3];
      v0[k] = c0 == 0 ? qv.x : qv.z;
      v1[k] = c0 == 0 ? qv.y : qv.w;
    }
    const int left = rem - 4 * lane;
#pragma unroll
    for (int j = 0; j < 4; ++j) {  // token j came in as k = (j - rot) & 3
      const int k = (j - rot) & 3;
      const float x0 = k == 0 ? v0[0] : k == 1 ? v0[1] : k == 2 ? v0[2] : v0[3];
      const float x1 = k == 0 ? v1[0] : k == 1 ? v1[1] : k == 2 ? v1[2] : v1[3];
      dtt[0][j] = j < left ? dt_of(pb, x0, h0) : 0.f;
      dtt[1][j] = j < left ? dt_of(pb, x1, h0 + 1) : 0.f;
    }
  }
  // the dt stage is read: refill it
  __syncwarp();
  if (S.have_ahead) scan_issue_dt<NS, MODE>(S, tm_dt, pb, rp, smem, bars);
#pragma unroll
  for (int hh = 0; hh < kHeads; ++hh) {
    const float a2 = S.a2[hh];
    float c0 = dtt[hh][0] * a2, c1 = c0 + dtt[hh][1] * a2, c2 = c1 + dtt[hh][2] * a2, c3 = c2 + dtt[hh][3] * a2;
    float v = c3;
#pragma unroll
    for (int k = 1; k < 32; k <<= 1) {
      const float u = __shfl_up_sync(0xffffffffu, v, k);
      if (lane >= k) v += u;
    }
    const float base = v - c3;  // cumsum before token 4 lane
    cth[hh][0] = c0 + base, cth[hh][1] = c1 + base, cth[hh][2] = c2 + base, cth[hh][3] = c3 + base;
    reinterpret_cast<float4*>(o.c[hh])[lane] = make_float4(cth[hh][0], cth[hh][1], cth[hh][2], cth[hh][3]);
    if (with_dt)
      reinterpret_cast<float4*>(o.dt[hh])[lane] = make_float4(dtt[hh][0], dtt[hh][1], dtt[hh][2], dtt[hh][3]);
  }
  __syncwarp();
  ++S.t;
  S.have = cursor_next(pb, rp, S.cur);
  return true;
}

// After a failure: the dt loads still in flight land before the CTA ends (bounded).
__device__ __forceinline__ void scan_drain(const ScanState& S, const Problem& pb, uint64_t* bars) {
  if ((threadIdx.x & 31) == 0)
    for (int n = S.t; n < S.dt_issued; ++n)
      mbar_wait_bounded(&bars[kBarDt0 + n % kDtStages], (n / kDtStages) & 1, pb.wait_limit);
}

// The scan warp (final states only, whose compute warps wait for the helper): the scan
// step, kScanSlots tiles ahead of the helper.
template <int NS, int MODE>
__device__ void scan_loop(const CUtensorMap* tm_dt, const Problem& pb, const RangePlan& rp, uint8_t* smem,
                          uint64_t* bars, volatile int* abort_flag) {
  using L = Layout<NS, MODE>;
  ScanTile* ring = reinterpret_cast<ScanTile*>(smem + L::scan);
  ScanState S;
  scan_init<NS, MODE>(S, tm_dt, pb, rp, smem, bars);
  bool ok = true;
  while (S.have) {
    const int slot = S.t % kScanSlots, k = kBarScanFree0 + slot;
    if (S.t >= kScanSlots) {
      if (!(ok = warp_wait(&bars[k], S.ph.parity(k), abort_flag, pb.wait_limit))) break;
      S.ph.flip(k);
    }
    float cth[kHeads][4], dtt[kHeads][4];
    if (!(ok = scan_tile<NS, MODE>(S, cth, dtt, ring[slot], true, tm_dt, pb, rp, smem, bars, abort_flag))) break;
    if ((threadIdx.x & 31) == 0) mbar_arrive(&bars[kBarScanFull0 + slot]);
  }
  if (!ok) {
    *abort_flag = 1;
    scan_drain(S, pb, bars);
  }
}

// ------------------------------------------------------------------ helper warp
// The helper walks the CTA's tile sequence ahead of the compute warps, loads each
// tile's dt by TMA into a ring of its own (kDtStages tiles in flight), and writes one
// descriptor per pass into a ring of kDescSlots: where the pass is, its rows, the
// factors u and r of both heads, the state scalings and the piece flags.  Per tile it
// forms c (the inclusive cumsum of dt A in log2 units from the tile start, both heads),
// keeps or re-centres each head's reference and cuts the valid rows into passes: one
// pass unless a head decays by more than 2^-(2 kRangeHalf) across the tile.  With final
// states only, dt and c come from the scan warp instead.
template <int NS, int MODE>
__device__ void helper_loop(const CUtensorMap* tm_dt, const Problem& pb, const RangePlan& rp, uint8_t* smem,
                            uint64_t* bars, volatile int* abort_flag) {
  using L = Layout<NS, MODE>;
  const int lane = threadIdx.x & 31;
  uint8_t* sdt = smem + L::sdt;
  uint64_t* dt_bar = bars + kBarDt0;
  float* sc = reinterpret_cast<float*>(smem + L::scan);  // c[head][128]
  const int pairs = pb.H / kHeads;
  PassDesc* descs = reinterpret_cast<PassDesc*>(smem + L::desc);
  Phases ph;
  auto wait = [&](int k) -> bool {
    if (!warp_wait(&bars[k], ph.parity(k), abort_flag, pb.wait_limit)) return false;
    ph.flip(k);
    return true;
  };
  // dt loads run up to kDtStages tiles ahead on a cursor of their own
  TileCursor ahead;
  bool have_ahead = cursor_first(pb, rp, ahead);
  int dt_issued = 0;
  auto issue_dt = [&]() {
    if (lane == 0) {
      const int st = dt_issued % kDtStages;
      const int h0 = (ahead.unit % pairs) * kHeads;
      mbar_expect_tx(&dt_bar[st], kTile * 16);
      tma_load_2d(sdt + st * kTile * 16, tm_dt, h0 & ~3, ahead.tb + ahead.k0, &dt_bar[st]);
    }
    ++dt_issued;
    have_ahead = cursor_next(pb, rp, ahead);
  };
  constexpr bool from_scan = MODE == kModeState;  // dt and c from the scan warp
  if (from_scan) have_ahead = false;
  for (int k = 0; k < kDtStages && have_ahead; ++k) issue_dt();
  const ScanTile* ring = reinterpret_cast<const ScanTile*>(smem + L::scan);

  TileCursor cur;
  bool have = cursor_first(pb, rp, cur);
  float a2[kHeads] = {0.f, 0.f}, dsk[kHeads] = {0.f, 0.f};
  float sg[kHeads] = {0.f, 0.f};  // per head: the pass reference m relative to the state before the next row
  int a_unit = -1, prev_piece = -1;
  bool ok = true;
  int t = 0, p = 0;
  auto take_slot = [&]() -> PassDesc* {
    const int slot = p % kDescSlots;
    if (p >= kDescSlots && !wait(kBarDescFree0 + slot)) return nullptr;
    return &descs[slot];
  };
  auto publish = [&]() {
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars[kBarDescFull0 + p % kDescSlots]);
    ++p;
  };
  for (;; ++t) {
    if (!have) {
      PassDesc* d = take_slot();
      if (!d) {
        ok = false;
        break;
      }
      if (lane == 0) d->flags = kPEnd;
      publish();
      break;
    }
    TileCursor nxt = cur;
    const bool have_next = cursor_next(pb, rp, nxt);
    const bool first_tile = cur.piece != prev_piece;
    const bool last_tile = !have_next || nxt.piece != cur.piece;
    prev_piece = cur.piece;
    const int h0 = (cur.unit % pairs) * kHeads;
    if (cur.unit != a_unit) {
      a_unit = cur.unit;
#pragma unroll
      for (int hh = 0; hh < kHeads; ++hh) {
        a2[hh] = pb.A[h0 + hh] * 1.4426950408889634f;  // A_h log2(e): cumsums are in log2 units
        dsk[hh] = pb.D ? pb.D[h0 + hh] : 0.f;
      }
    }
    const int rem = min(kTile, cur.len - cur.k0);

    float dtt[kHeads][4], cth[kHeads][4];
    const float* sct = sc;  // c[head][128] of this tile
    const int sslot = t % kScanSlots;
    if constexpr (from_scan) {  // lane: rows 4 lane .. 4 lane + 3
      if (!(ok = wait(kBarScanFull0 + sslot))) break;
      sct = ring[sslot].c[0];
#pragma unroll
      for (int hh = 0; hh < kHeads; ++hh) {
        const float4 cv = reinterpret_cast<const float4*>(ring[sslot].c[hh])[lane];
        const float4 dv = reinterpret_cast<const float4*>(ring[sslot].dt[hh])[lane];
        cth[hh][0] = cv.x, cth[hh][1] = cv.y, cth[hh][2] = cv.z, cth[hh][3] = cv.w;
        dtt[hh][0] = dv.x, dtt[hh][1] = dv.y, dtt[hh][2] = dv.z, dtt[hh][3] = dv.w;
      }
    } else {
      // this tile's dt: row 4 lane + j holds the 4 heads' dt of one token; a lane reads its
      // rows in the order j = (k + rot) & 3, rot = (lane / 2) & 3, so each quarter warp's
      // 16-byte loads fall in distinct banks
      if (!(ok = wait(kBarDt0 + t % kDtStages))) break;
      {
        const float4* rows = reinterpret_cast<const float4*>(sdt + (t % kDtStages) * kTile * 16) + 4 * lane;
        const int rot = (lane >> 1) & 3, c0 = h0 & 3;  // the pair's first column in the 4-head row
        float v0[4], v1[4];
  #pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float4 qv = rows[(k + rot) & 3];
          v0[k] = c0 == 0 ? qv.x : qv.z;
          v1[k] = c0 == 0 ? qv.y : qv.w;
        }
        const int left = rem - 4 * lane;
  #pragma unroll
        for (int j = 0; j < 4; ++j) {  // token j came in as k = (j - rot) & 3
          const int k = (j - rot) & 3;
          const float x0 = k == 0 ? v0[0] : k == 1 ? v0[1] : k == 2 ? v0[2] : v0[3];
          const float x1 = k == 0 ? v1[0] : k == 1 ? v1[1] : k == 2 ? v1[2] : v1[3];
          dtt[0][j] = j < left ? dt_of(pb, x0, h0) : 0.f;
          dtt[1][j] = j < left ? dt_of(pb, x1, h0 + 1) : 0.f;
        }
      }
      // the dt stage is read: refill it
      __syncwarp();
      if (have_ahead) issue_dt();
      // inclusive cumsum c of dt A (log2 units) from the tile start, both heads
  #pragma unroll
      for (int hh = 0; hh < kHeads; ++hh) {
        float c0 = dtt[hh][0] * a2[hh], c1 = c0 + dtt[hh][1] * a2[hh], c2 = c1 + dtt[hh][2] * a2[hh],
              c3 = c2 + dtt[hh][3] * a2[hh];
        float v = c3;
  #pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float u = __shfl_up_sync(0xffffffffu, v, o);
          if (lane >= o) v += u;
        }
        const float base = v - c3;  // cumsum before token 4 lane
        cth[hh][0] = c0 + base, cth[hh][1] = c1 + base, cth[hh][2] = c2 + base, cth[hh][3] = c3 + base;
        reinterpret_cast<float4*>(sc + hh * kTile)[lane] = make_float4(cth[hh][0], cth[hh][1], cth[hh][2], cth[hh][3]);
      }
      __syncwarp();
    }

    // passes over rows [0, rem).  A head keeps its reference m (sg[hh] = m - c_before(lo),
    // carried over from the pass before) while every remaining row stays within
    // kRangeHalf of it; otherwise the pass re-centres it on its rows, which then span at
    // most 2 kRangeHalf (the pass ends where a re-centred head's range would be wider).
    for (int lo = 0; lo < rem;) {
      const bool piece_start = first_tile && lo == 0;
      float c0[kHeads], clo[kHeads];
      bool keep[kHeads];
#pragma unroll
      for (int hh = 0; hh < kHeads; ++hh) {
        c0[hh] = lo > 0 ? sct[hh * kTile + lo - 1] : 0.f;
        clo[hh] = sct[hh * kTile + lo];
        bool out = piece_start;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int row = 4 * lane + j;
          out |= row >= lo && row < rem && fabsf(sg[hh] + c0[hh] - cth[hh][j]) > kRangeHalf;
        }
        keep[hh] = !__any_sync(0xffffffffu, out);
      }
      int bad = kTile;  // first row j > lo whose range from lo is too wide for a re-centred head
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int row = 4 * lane + j;
        bool over = false;
#pragma unroll
        for (int hh = 0; hh < kHeads; ++hh) over |= !keep[hh] && fabsf(clo[hh] - cth[hh][j]) > 2.f * kRangeHalf;
        if (row > lo && row < rem && bad == kTile && over) bad = row;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) bad = min(bad, __shfl_xor_sync(0xffffffffu, bad, o));
      const int hi = min(bad, rem);

      PassDesc* d = take_slot();
      if (!d) {
        ok = false;
        break;
      }
      int rescale = 0;
#pragma unroll
      for (int hh = 0; hh < kHeads; ++hh) {
        const float* ch_ = sct + hh * kTile;
        const float m = keep[hh] ? c0[hh] + sg[hh] : 0.5f * (clo[hh] + ch_[hi - 1]);
        float u[4], r[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int row = 4 * lane + j;
          const bool in = row >= lo && row < hi;
          u[j] = in ? ex2(m - cth[hh][j]) * dtt[hh][j] : 0.f;
          r[j] = in ? ex2(cth[hh][j] - m) : 0.f;
        }
        reinterpret_cast<float4*>(d->u[hh])[lane] = make_float4(u[0], u[1], u[2], u[3]);
        reinterpret_cast<float4*>(d->r[hh])[lane] = make_float4(r[0], r[1], r[2], r[3]);
        if (lane == 0) {
          d->sig_in[hh] = ex2(m - c0[hh]);
          d->sig_out[hh] = ex2(ch_[hi - 1] - m);
          d->dskip[hh] = dsk[hh];
        }
        if (!keep[hh] && !piece_start) rescale |= kPRescale0 << hh;
        sg[hh] = m - ch_[hi - 1];  // the reference relative to the state after this pass
      }
      if (lane == 0) {
        int flags = rescale;
        if (lo == 0) flags |= kPFirst;
        if (hi == rem) flags |= kPLast;
        if (piece_start) flags |= kPPieceStart | ((cur.flags & kCarryIn) ? kPCarryIn : 0);
        if (last_tile && hi == rem) {
          if ((cur.flags & kUnitEnd) && pb.final_state) flags |= kPToFinal;
          if (cur.flags & kCarryOut) flags |= kPToCarry;
        }
        d->t0 = cur.tb + cur.k0;
        d->rem = rem;
        d->lo = lo;
        d->hi = hi;
        d->s = cur.unit / pairs;
        d->h0 = h0;
        d->flags = flags;
        d->carry_src = rp.carry_src;
      }
      publish();
      lo = hi;
    }
    if (!ok) break;
    if constexpr (from_scan) {  // the slot is used up: the scan warp may refill it
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarScanFree0 + sslot]);
    }
    cur = nxt;
    have = have_next;
  }
  if (!ok) {
    *abort_flag = 1;
    // dt loads still in flight land before the CTA ends (bounded)
    if (lane == 0)
      for (int n = t; n < dt_issued; ++n) mbar_wait_bounded(&dt_bar[n % kDtStages], (n / kDtStages) & 1, pb.wait_limit);
  }
}

template <int NS, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    ssd_fused_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                        const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_y32,
                        const __grid_constant__ CUtensorMap tm_dt, const __grid_constant__ Problem pb) {
  using L = Layout<NS, MODE>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem_base;
  const int tid = threadIdx.x, warp = tid >> 5;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::bars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::flag);

  if (pb.cu && *pb.nchunks < 0) return;  // cu_seqlens rejected by the table kernel

  if (warp == 0) {
    tmem_alloc(&s_tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int k = 0; k < kXStages; ++k) {
      mbar_init(&bars[kBarX0 + k], 1);
      mbar_init(&bars[kBarXfree0 + k], kComputeWarps);
    }
    for (int k = 0; k < 2; ++k) mbar_init(&bars[kBarUFree0 + k], 1);
    for (int k = 0; k < 2; ++k) {
      mbar_init(&bars[kBarS0 + k], 1);
      mbar_init(&bars[kBarP0 + k], kComputeWarps);
    }
    for (int k = 0; k < L::kRingSlots; ++k) {
      mbar_init(&bars[kBarRing0 + k], 1);
      mbar_init(&bars[kBarRingFree0 + k], 1);
    }
    mbar_init(&bars[kBarSt], 1);
    mbar_init(&bars[kBarY], 1);
    mbar_init(&bars[kBarU], kComputeWarps);
    mbar_init(&bars[kBarU1], kComputeWarps);
    mbar_init(&bars[kBarHt], kComputeWarps);
    mbar_init(&bars[kBarHRead], kComputeWarps);
    mbar_init(&bars[kBarFree], kComputeWarps);
    mbar_init(&bars[kBarDrain], 1);
    for (int k = 0; k < kDtStages; ++k) mbar_init(&bars[kBarDt0 + k], 1);
    for (int k = 0; k < kDescSlots; ++k) {
      mbar_init(&bars[kBarDescFull0 + k], 1);
      mbar_init(&bars[kBarDescFree0 + k], kComputeWarps + 1);
    }
    for (int k = 0; k < kHeads * 4; ++k) mbar_init(&bars[kBarPair0 + k], 1);
    for (int k = 0; k < kScanSlots; ++k) {
      mbar_init(&bars[kBarScanFull0 + k], 1);
      mbar_init(&bars[kBarScanFree0 + k], 1);
    }
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
  // the split's weights (the second column half of N = 256 reuses the first launch's)
  // the split's weights: from tile_weight_kernel or the first column half of N = 256, or
  // here (CTA r weighs sequence tiles r, r + R, ...; few per CTA) and a barrier
  bool weights_ok = true;
  if (!pb.weights_ready) {
    const int64_t seqtiles = seq_tile0(pb, pb.nseq);
    for (int64_t st = blockIdx.x; st < seqtiles; st += gridDim.x)
      weigh_tile<kThreads>(pb, st, reinterpret_cast<float4*>(smem + L::x));
    weights_ok = weights_barrier(pb, abort_flag);
  }
  const RangePlan rp = weights_ok ? split_work(pb, reinterpret_cast<SplitScratch*>(smem + L::x)) : RangePlan{};

  if (warp == kMmaWarp) {
    mma_loop<NS, MODE>(pb, smem, tmem, bars, abort_flag);
    __syncwarp();  // the warp reconverges before the CTA-wide barrier
  } else if (warp == kLoadWarp) {
    if ((tid & 31) == 0) load_loop<NS, MODE>(&tm_x, &tm_b, &tm_c, pb, rp, smem, bars, abort_flag);
    __syncwarp();
  } else if (warp == kHelperWarp) {
    helper_loop<NS, MODE>(&tm_dt, pb, rp, smem, bars, abort_flag);
    __syncwarp();
  } else if (warp == kScanWarp) {
    if (MODE == kModeState) scan_loop<NS, MODE>(&tm_dt, pb, rp, smem, bars, abort_flag);
    __syncwarp();
  } else {
    compute_loop<NS, MODE>(&tm_y32, pb, smem, tmem, bars, abort_flag);
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
}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() { return tensor_map_encoder(); }

// 3-D bf16 map {inner, mid, tokens} with a {64, 1, rows} box and 128-byte swizzle; rows of
// the innermost dimension are `pitch` elements apart (default: inner).
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t tokens,
              uint32_t rows = kTile, uint64_t pitch = 0) {
  auto fn = encode_fn();
  if (!fn) return false;
  if (!pitch) pitch = inner;
  cuuint64_t dims[3] = {inner, mid, tokens};
  cuuint64_t strides[2] = {pitch * 2, pitch * mid * 2};
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

// The kernel's shared-memory size is set once per device and kernel instance.
template <int NS, int MODE>
cudaError_t set_smem_attribute() {
  static std::atomic<uint64_t> done{0};  // bit d: set on device d
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
  if (bit && (done.load() & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(ssd_fused_tc_kernel<NS, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kDynSmem<NS, MODE>);
  if (e == cudaSuccess && bit) done.fetch_or(bit);
  return e;
}

template <int NS, int MODE>
cudaError_t launch_mode(const Problem& pb, cudaStream_t st) {
  CUtensorMap mx, mb, mc, my, mdt;
  const uint64_t tokens = (uint64_t)pb.tokens;
  // B and C: boxes of 64 state columns; past N the box reads zeros (N < NS).  Without y
  // (final states only) C and y are not read and their maps stand in as copies.
  constexpr bool state_only = MODE == kModeState;
  const __nv_bfloat16* b0 = static_cast<const __nv_bfloat16*>(pb.B) + pb.n_off;
  const __nv_bfloat16* c0 = static_cast<const __nv_bfloat16*>(pb.C) + pb.n_off;
  if (!make_map(&mx, pb.x, kHeadDim, pb.H, tokens) || !make_map(&mb, b0, pb.N, pb.G, tokens, kTile, pb.n_stride) ||
      (!state_only && (!make_map(&mc, c0, pb.N, pb.G, tokens, kTile, pb.n_stride) ||
                       !make_map(&my, pb.y, kHeadDim, pb.H, tokens, 32))) ||
      !make_dt_map(&mdt, pb.dt, pb.H, tokens))
    return cudaErrorInvalidValue;
  if (state_only) mc = mb, my = mx;
  cudaError_t e = set_smem_attribute<NS, MODE>();
  if (e != cudaSuccess) {
    if (getenv("SSD_DEBUG")) fprintf(stderr, "ssd: smem attribute failed: %s\n", cudaGetErrorString(e));
    return e;
  }
  // One CTA per SM (at most), each on a weighted share of the flat tile list; a flat tile
  // count is not known on the host for packed batches, so the grid covers every SM and
  // ranges may be empty when there are fewer tiles than SMs.
  const int grid = pb.ranges;
  if (grid <= 0) return cudaSuccess;
  if (grid > kMaxRanges) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kDynSmem<NS, MODE>;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // all CTAs resident: carry waits always end
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (pb.prof_start) cudaEventRecord(pb.prof_start, st);
  e = cudaLaunchKernelEx(&cfg, ssd_fused_tc_kernel<NS, MODE>, mx, mb, mc, my, mdt, pb);
  if (pb.prof_stop) cudaEventRecord(pb.prof_stop, st);
  count_launches(1);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess && getenv("SSD_DEBUG"))
    fprintf(stderr, "ssd: fused kernel launch failed: %s (smem %u, threads %d)\n", cudaGetErrorString(e),
            (unsigned)kDynSmem<NS, MODE>, kThreads);
  return e;
}

template <int NS>
cudaError_t launch_ns(const Problem& pb, cudaStream_t st) {
  if (!pb.y) return launch_mode<NS, kModeState>(pb, st);
  return launch_mode<NS, kModeFull>(pb, st);
}

}  // namespace

bool tc_supports(const ssd_shape* s, int chunk) {
  (void)chunk;  // the tiles are 128 tokens whatever the chunk length; results do not depend on it
  if (!s || s->io_dtype != SSD_BF16 || s->headdim != kHeadDim) return false;
  // N up to 128 in steps of 8 (16-byte rows of B and C), run as 64 or 128 with zero columns;
  // N = 256 as two launches on its column halves
  if ((s->dstate > 128 && s->dstate != 256) || s->dstate % 8) return false;
  if (s->nheads % kHeads || (s->nheads / s->ngroups) % kHeads) return false;  // head pairs share a group
  if (s->nheads % 4) return false;  // dt rows of 4 heads (16 bytes) per TMA box
  const int64_t tokens = s->batch * s->seqlen;
  return tokens >= 1 && tokens < ((int64_t)1 << 31) - kTile;
}

cudaError_t launch_tc(const Problem& pb_in, cudaStream_t st) {
  // The split's weights: each CTA weighs its share of the sequence tiles before the split,
  // unless there are more than two per CTA; then a kernel of their own, with many tiles in
  // flight per SM, weighs them first.
  Problem pb = pb_in;
  const int64_t seqtiles = pb.cu ? (pb.tokens + kTile - 1) / kTile + pb.nseq : (int64_t)pb.nseq * pb.dense_tiles;
  if (seqtiles > 2 * (int64_t)pb.ranges) {
    const int grid = (int)(seqtiles < 32 * kMaxRanges ? seqtiles : 32 * kMaxRanges);
    // the fused kernel's shared-memory carve-out, so the SMs need not switch between the launches
    static std::atomic<uint64_t> carve{0};
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && dev < 64 && !(carve.load() & (1ull << dev))) {
      cudaFuncSetAttribute(tile_weight_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
      carve.fetch_or(1ull << dev);
    }
    tile_weight_kernel<<<grid, kWeightThreads, 0, st>>>(pb);
    count_launches(1);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    pb.weights_ready = 1;
  }
  if (pb.N <= 128) {
    Problem q = pb;
    q.n_off = 0, q.n_stride = pb.N, q.y_accum = 0;
    return pb.N > 64 ? launch_ns<128>(q, st) : launch_ns<64>(q, st);
  }
  // N = 256: the state's columns are independent and y is linear in them, so the call is
  // two launches on the column halves of B, C and the states; the second adds its y to the
  // first's (and D x only once).  The measurement events span both.
  Problem a = pb, b = pb;
  a.N = b.N = 128;
  a.n_stride = b.n_stride = pb.N;
  a.n_off = 0, b.n_off = 128;
  a.y_accum = 0, b.y_accum = pb.y != nullptr;
  b.weights_ready = 1;  // the first launch wrote the split's weights
  b.D = nullptr;
  a.prof_stop = nullptr, b.prof_start = nullptr;
  b.epoch = pb.epoch ^ 0x8000000000000000ull;  // a value no other launch's flags hold
  cudaError_t e = launch_ns<128>(a, st);
  if (e != cudaSuccess) return e;
  return b.y_accum ? launch_mode<128, kModeAccum>(b, st) : launch_ns<128>(b, st);
}

}  // namespace ssd
