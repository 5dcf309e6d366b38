// ssd_tc.cu -- the tensor-core path: one fused sm_100a kernel for the whole chunked
// SSD forward pass ("Transformers are SSMs", wikillm.com card, Method step 5, sec. 6).
//
// A CTA owns one (sequence, head) at a time and walks the sequence in 128-token
// tiles (the tcgen05 M).  The P x N state never leaves the chip: each of the 128
// threads keeps one column n of the fp32 state in registers.  Per tile:
//
//   cumsum   cs_j = running in-chunk cumsum of dt_j A_h (restarted at each chunk
//            start, so a 256-token chunk spans two tiles)
//   MMA  S   = C B^T                                   (128 x 128, K = N)
//   mask     P_ij = S_ij exp(cs_i - cs_j) dt_j for j <= i, else 0 (mask before exp),
//            written as bf16 to shared memory
//   MMA  Y   = P X                 diagonal block      (128 x 64, K = 128)
//   MMA  Yo  = C h^T               left factor         (128 x 64, K = N)
//   MMA  s^T = B^T (w o X)         right factor        (N x 64, K = 128), w_j = exp(cs_end - cs_j) dt_j
//   epilogue y_i = Y_i + exp(cs_i - cs_start) Yo_i + D x_i  (bf16 store)
//            h  <- exp(cs_end - cs_start) h + s          (centre factor, in registers)
//
// Operands come from shared memory: x, B, C by TMA with 128-byte swizzle; P, w o X
// and the bf16 copy of h are written by the threads in the same swizzled layouts.
// Accumulators live in tensor memory (S 128 cols, Y 64, Yo 64, s^T 64).
// Every wait is bounded; a wait that gives up records SSD_ERR_DEVICE_TIMEOUT in the
// status word, drains what is in flight (bounded), frees tensor memory and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "sm100_ptx.cuh"
#include "ssd_tc.cuh"

namespace ssd {

namespace {

using namespace sm100;

constexpr int kTile = 128;         // tokens per tile (UMMA M)
constexpr int kHeadDim = 64;       // P supported by this path
constexpr int kWGThreads = 128;    // one warpgroup per head: thread i <-> TMEM lane i
constexpr int kHeads = 2;          // heads of one B/C group processed together
constexpr int kThreads = kHeads * kWGThreads;
constexpr uint32_t kTmemCols = 512;
// TMEM columns.  S (fp32, 128 cols) is reused for the right-factor accumulator s^T of
// both heads once the masks have read it; P_h are bf16 pairs (64 cols per head).
constexpr uint32_t kColS = 0, kColSt = 0, kColP = 128, kColY = 256, kColYo = 384;
constexpr long long kWaitLimit = 4ll << 30;  // SM cycles (about 2 s) before a wait gives up
constexpr uint32_t kAtom = kTile * 128;      // one 128-row x 128-byte swizzled operand column

template <int NS>
struct Layout {
  static constexpr uint32_t x = 0;                          // [stage][head] [128 tok][64 p]
  static constexpr uint32_t b = x + 2 * kHeads * kAtom;     // NS/64 atoms [128 tok][64 n]
  static constexpr uint32_t c = b + (NS / 64) * kAtom;
  static constexpr uint32_t xw = c + (NS / 64) * kAtom;     // [head] [128 tok][64 p]  (N = 128 operand)
  static constexpr uint32_t ht = xw + kHeads * kAtom;       // [head] [NS n][64 p]     (N = 128 operand)
  static constexpr uint32_t cs = ht + kHeads * NS * 128;    // float[head][128] in-chunk cumsum
  static constexpr uint32_t dt = cs + kHeads * kTile * 4;   // float[head][128]
  static constexpr uint32_t cc = dt + kHeads * kTile * 4;   // float[head][128] column factors
  static constexpr uint32_t red = cc + kHeads * kTile * 4;  // float[head][4]
  static constexpr uint32_t bars = red + kHeads * 16;       // load[2], s, mma
  static constexpr uint32_t bytes = bars + 4 * 8;
};
template <int NS>
constexpr uint32_t kDynSmem = Layout<NS>::bytes + 1024;  // + base alignment slack

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// The tiles one CTA walks: units (sequence, head pair) in a strided order, each
// unit's 128-token tiles in sequence order.
struct TileCursor {
  int unit, k0, len;
  int64_t tb;
};

__device__ __forceinline__ bool cursor_load(const Problem& pb, int unit, TileCursor& c) {
  const int units = pb.nseq * (pb.H / kHeads);
  if (unit >= units) return false;
  const int s = unit / (pb.H / kHeads);
  c.unit = unit;
  c.k0 = 0;
  c.tb = seq_off(pb, s);
  c.len = (int)(seq_off(pb, s + 1) - c.tb);
  return true;
}

// Advances to the next tile (skipping empty sequences' tile loops); false when done.
__device__ __forceinline__ bool cursor_next(const Problem& pb, TileCursor& c) {
  c.k0 += kTile;
  while (c.k0 >= c.len) {
    if (!cursor_load(pb, c.unit + gridDim.x, c)) return false;
    if (c.len > 0) return true;
  }
  return true;
}

template <int NS>
__device__ __forceinline__ void issue_x(const CUtensorMap* tm_x, uint8_t* sx_stage, uint64_t* bar,
                                        const Problem& pb, const TileCursor& c) {
  const int h0 = (c.unit % (pb.H / kHeads)) * kHeads;
#pragma unroll
  for (int hh = 0; hh < kHeads; ++hh)
    tma_load_3d(sx_stage + hh * kAtom, tm_x, 0, h0 + hh, (int)(c.tb + c.k0), bar);
}

template <int NS>
__device__ __forceinline__ void issue_bc(const CUtensorMap* tm_b, const CUtensorMap* tm_c, uint8_t* sb,
                                         uint8_t* sc, uint64_t* bar, const Problem& pb, const TileCursor& c) {
  const int g = ((c.unit % (pb.H / kHeads)) * kHeads) / pb.hpg;
#pragma unroll
  for (int a = 0; a < NS / 64; ++a) {
    tma_load_3d(sb + a * kAtom, tm_b, a * 64, g, (int)(c.tb + c.k0), bar);
    tma_load_3d(sc + a * kAtom, tm_c, a * 64, g, (int)(c.tb + c.k0), bar);
  }
}

template <int NS>
__global__ void __launch_bounds__(kThreads, 1)
    ssd_fused_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                        const __grid_constant__ CUtensorMap tm_c, Problem pb) {
  using L = Layout<NS>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem_base;
  const int tid = threadIdx.x;
  const int hw = tid / kWGThreads;     // which head of the pair this warpgroup handles
  const int i = tid % kWGThreads;      // row / TMEM lane
  const int wq = i >> 5, lane = i & 31;  // lane quarter of this warp
  const bool issuer = tid == 0;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sx = smem + L::x;
  uint8_t* sb = smem + L::b;
  uint8_t* sc = smem + L::c;
  uint8_t* sxw = smem + L::xw;
  uint8_t* sht = smem + L::ht;
  float* s_cs = reinterpret_cast<float*>(smem + L::cs) + hw * kTile;
  float* s_dt = reinterpret_cast<float*>(smem + L::dt) + hw * kTile;
  float* s_cc = reinterpret_cast<float*>(smem + L::cc) + hw * kTile;
  float* s_red = reinterpret_cast<float*>(smem + L::red) + hw * 4;
  uint64_t* bar_load = reinterpret_cast<uint64_t*>(smem + L::bars);  // [2], one per x stage
  uint64_t* bar_s = bar_load + 2;
  uint64_t* bar_mma = bar_load + 3;

  if (*pb.nchunks < 0) return;  // cu_seqlens rejected by the table kernel

  if (tid < 32) {
    tmem_alloc(&s_tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (issuer) {
    mbar_init(&bar_load[0], 1);
    mbar_init(&bar_load[1], 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_mma, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tensormap(&tm_x);
    prefetch_tensormap(&tm_b);
    prefetch_tensormap(&tm_c);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem_base;
  const uint32_t lane_base = (uint32_t)(wq * 32) << 16;

  constexpr uint32_t kLoadBytes = kHeads * kAtom + 2u * (NS / 64) * kAtom;
  const uint32_t id_s = idesc_bf16(128, 128, 0, 0);
  const uint32_t id_y = idesc_bf16(128, 64, 0, 1);
  const uint32_t id_yo = idesc_bf16(128, 128, 0, 1);
  const uint32_t id_st = idesc_bf16(128, 128, 1, 1);
  const uint32_t a_sb = smem_u32(sb), a_sc = smem_u32(sc), a_sxw = smem_u32(sxw), a_sht = smem_u32(sht);
  // For N = 64 the B^T operand has one M atom; the second (unused) half of s^T reads
  // the C tile that follows it, and those lanes are ignored.
  const uint32_t lbo_bt = kAtom;

  uint32_t ph_load[2] = {0, 0}, ph_s = 0, ph_mma = 0;
  bool ok = true;
  int pend_load = 0;  // bit k: a load on bar_load[k] issued and not yet waited for
  bool pend_s = false, pend_mma = false;

  TileCursor cur;
  bool have = cursor_load(pb, blockIdx.x, cur);
  while (have && cur.len == 0) have = cursor_next(pb, cur);  // nothing to do for empty sequences

  // Empty sequences still need final = init: handled by the units loop below on the fly.
  float hst[kHeadDim];
  int stage = 0;
  int cur_unit = -1;
  float cs_base = 0.f, dt_next = 0.f;

  if (have && issuer) {
    mbar_expect_tx(&bar_load[0], kLoadBytes);
    issue_x<NS>(&tm_x, sx, &bar_load[0], pb, cur);
    issue_bc<NS>(&tm_b, &tm_c, sb, sc, &bar_load[0], pb, cur);
  }
  if (have) pend_load = 1;

  // Units of this CTA whose sequences are empty get their final state here.
  auto finish_empty_units = [&](int from_unit, int to_unit) {
    for (int u = from_unit; u < to_unit; u += gridDim.x) {
      const int s = u / (pb.H / kHeads);
      const int h = (u % (pb.H / kHeads)) * kHeads + hw;
      if (seq_off(pb, s + 1) - seq_off(pb, s) != 0) continue;
      if (pb.final_state && i < NS) {
        const int64_t base = ((int64_t)s * pb.H + h) * kHeadDim * NS;
        for (int p = 0; p < kHeadDim; ++p)
          pb.final_state[base + (int64_t)p * NS + i] = pb.init ? pb.init[base + (int64_t)p * NS + i] : 0.f;
      }
    }
  };
  finish_empty_units(blockIdx.x, have ? cur.unit : pb.nseq * (pb.H / kHeads));

  while (have && ok) {
    const int pair = cur.unit % (pb.H / kHeads);
    const int s = cur.unit / (pb.H / kHeads);
    const int h = pair * kHeads + hw;
    const float Ah = pb.A[h];
    const float Dh = pb.D ? pb.D[h] : 0.f;
    const int64_t st_base = ((int64_t)s * pb.H + h) * kHeadDim * NS;
    const int64_t t0 = cur.tb + cur.k0;
    const int rem = min(kTile, cur.len - cur.k0);

    if (cur.unit != cur_unit) {  // first tile of a unit: initial state, first dt
      cur_unit = cur.unit;
#pragma unroll
      for (int p = 0; p < kHeadDim; ++p) hst[p] = 0.f;
      if (pb.init && i < NS) {
#pragma unroll
        for (int p = 0; p < kHeadDim; ++p) hst[p] = pb.init[st_base + (int64_t)p * NS + i];
      }
      dt_next = (i < cur.len) ? pb.dt[(cur.tb + i) * pb.H + h] : 0.f;
    }
    if (cur.k0 % pb.Q == 0) cs_base = 0.f;

    // ---- look ahead: the next tile's x goes to the other stage now
    TileCursor nxt = cur;
    const bool have_next = cursor_next(pb, nxt);
    if (have_next && issuer) {
      fence_proxy_async();
      mbar_expect_tx(&bar_load[stage ^ 1], kLoadBytes);
      issue_x<NS>(&tm_x, sx + (stage ^ 1) * kHeads * kAtom, &bar_load[stage ^ 1], pb, nxt);
    }
    if (have_next) pend_load |= 1 << (stage ^ 1);

    // ---- in-chunk cumsum of dt*A; the next tile's dt is fetched meanwhile
    const float dtj = dt_next;
    dt_next = (cur.k0 + kTile + i < cur.len) ? pb.dt[(t0 + kTile + i) * pb.H + h] : 0.f;
    float v = dtj * Ah;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    if (lane == 31) s_red[wq] = v;
    __syncthreads();
    float off = cs_base;
    for (int w = 0; w < wq; ++w) off += s_red[w];
    const float cs_i = off + v;
    s_cs[i] = cs_i;
    __syncthreads();
    const float cs_start = cs_base;
    const float cs_end = s_cs[kTile - 1];  // tokens past the end add 0
    cs_base = cs_end;
    // column factor for blocks below the diagonal: exp(cs_ref - cs_i) dt_i, with cs_ref
    // the cumsum at the end of i's 32-token block
    s_cc[i] = __expf(s_cs[wq * 32 + 31] - cs_i) * dtj;
    s_dt[i] = dtj;
    const float w_i = __expf(cs_end - cs_i) * dtj;  // right-factor weight (0 past the end)

    // ---- wait for x, B, C of this tile, then S = C B^T (shared by both heads)
    ok = mbar_wait_bounded(&bar_load[stage], ph_load[stage], kWaitLimit);
    if (__syncthreads_or(!ok)) {
      ok = false;
      break;
    }
    ph_load[stage] ^= 1;
    pend_load &= ~(1 << stage);
    pend_s = true;
    if (issuer) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < NS / 16; ++kk) {
        const uint32_t koff = (kk >> 2) * kAtom + (kk & 3) * 32;
        umma_f16(tmem + kColS, sdesc_sw128(a_sc + koff, 16, 1024), sdesc_sw128(a_sb + koff, 16, 1024), id_s,
                 kk > 0);
      }
      umma_commit(bar_s);
    }

    // ---- w o x (right-factor input) and the bf16 state copy, while S runs
    const uint8_t* sxh = sx + (stage * kHeads + hw) * kAtom;
    {
      uint8_t* dst = sxw + hw * kAtom;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t o = sw128_off(i, c);
        uint4 xv = *reinterpret_cast<const uint4*>(sxh + o);
        uint32_t* u = reinterpret_cast<uint32_t*>(&xv);
#pragma unroll
        for (int q = 0; q < 4; ++q) u[q] = pack_bf16(bf16_lo(u[q]) * w_i, bf16_hi(u[q]) * w_i);
        *reinterpret_cast<uint4*>(dst + o) = xv;
      }
      if (i < NS) {
        uint8_t* hdst = sht + hw * NS * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4 hv;
          hv.x = pack_bf16(hst[8 * c + 0], hst[8 * c + 1]);
          hv.y = pack_bf16(hst[8 * c + 2], hst[8 * c + 3]);
          hv.z = pack_bf16(hst[8 * c + 4], hst[8 * c + 5]);
          hv.w = pack_bf16(hst[8 * c + 6], hst[8 * c + 7]);
          *reinterpret_cast<uint4*>(hdst + sw128_off(i, c)) = hv;
        }
      }
    }
    fence_proxy_async();

    // ---- P_h = mask_h(S), bf16 pairs in tensor memory
    ok = mbar_wait_bounded(bar_s, ph_s, kWaitLimit);
    if (__syncthreads_or(!ok)) {
      ok = false;
      break;
    }
    ph_s ^= 1;
    pend_s = false;
    tc_fence_after();
    {
      const uint32_t colp = kColP + hw * 64;
#pragma unroll 1
      for (int cb = 0; cb < 4; ++cb) {  // 32-column blocks of S -> P columns 16cb..16cb+15
        uint32_t pk[16];
        if (cb < wq) {  // strictly below the diagonal: exp(cs_i - cs_j) = rf * exp(cs_ref - cs_j)
          uint32_t r[32];
          tmem_ld32(tmem + lane_base + kColS + cb * 32, r);
          const float rf = __expf(cs_i - s_cs[cb * 32 + 31]);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const float e0 = __uint_as_float(r[2 * q]) * rf * s_cc[cb * 32 + 2 * q];
            const float e1 = __uint_as_float(r[2 * q + 1]) * rf * s_cc[cb * 32 + 2 * q + 1];
            pk[q] = pack_bf16(e0, e1);
          }
        } else if (cb == wq) {  // diagonal block: mask first, then exp
          uint32_t r[32];
          tmem_ld32(tmem + lane_base + kColS + cb * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            float e[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int jj = 2 * q + u;  // column within the block; this row is `lane`
              e[u] = 0.f;
              if (jj <= lane)
                e[u] = __uint_as_float(r[jj]) * __expf(cs_i - s_cs[cb * 32 + jj]) * s_dt[cb * 32 + jj];
            }
            pk[q] = pack_bf16(e[0], e[1]);
          }
        } else {  // above the diagonal: zero
#pragma unroll
          for (int q = 0; q < 16; ++q) pk[q] = 0u;
        }
        tmem_st16(tmem + lane_base + colp + cb * 16, pk);
      }
    }
    tmem_st_wait();
    tc_fence_before();
    __syncthreads();

    // ---- Y_h = P_h x_h, Yo = C [h0 h1]^T, s^T = B^T [w0 x0 | w1 x1]
    pend_mma = true;
    if (issuer) {
      tc_fence_after();
      const uint32_t a_sx = smem_u32(sx + stage * kHeads * kAtom);
#pragma unroll
      for (int hh = 0; hh < kHeads; ++hh) {
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          umma_f16_ta(tmem + kColY + hh * 64, tmem + kColP + hh * 64 + kk * 8,
                      sdesc_sw128(a_sx + hh * kAtom + kk * 2048, kAtom, 1024), id_y, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < NS / 16; ++kk) {
        const uint32_t koff = (kk >> 2) * kAtom + (kk & 3) * 32;
        umma_f16(tmem + kColYo, sdesc_sw128(a_sc + koff, 16, 1024),
                 sdesc_sw128(a_sht + kk * 2048, NS * 128, 1024), id_yo, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < kTile / 16; ++kk)
        umma_f16(tmem + kColSt, sdesc_sw128(a_sb + kk * 2048, lbo_bt, 1024),
                 sdesc_sw128(a_sxw + kk * 2048, kAtom, 1024), id_st, kk > 0);
      umma_commit(bar_mma);
    }
    ok = mbar_wait_bounded(bar_mma, ph_mma, kWaitLimit);
    if (__syncthreads_or(!ok)) {
      ok = false;
      break;
    }
    ph_mma ^= 1;
    pend_mma = false;
    tc_fence_after();

    // ---- B and C are free: fetch the next tile's (its x is already on the way)
    if (have_next && issuer) {
      fence_proxy_async();
      issue_bc<NS>(&tm_b, &tm_c, sb, sc, &bar_load[stage ^ 1], pb, nxt);
    }

    // ---- epilogue: y rows and the state update
    {
      const float carry = __expf(cs_i - cs_start);
      __nv_bfloat16* yrow = static_cast<__nv_bfloat16*>(pb.y) + ((t0 + i) * pb.H + h) * kHeadDim;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t ry[32], ro[32];
        tmem_ld32(tmem + lane_base + kColY + hw * 64 + half * 32, ry);
        tmem_ld32(tmem + lane_base + kColYo + hw * 64 + half * 32, ro);
        tmem_ld_wait();
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const int c = half * 4 + c4;  // 16-byte chunk of the 64-wide row: p = 8c..8c+7
          const uint4 xv = *reinterpret_cast<const uint4*>(sxh + sw128_off(i, c));
          const uint32_t* xu = reinterpret_cast<const uint32_t*>(&xv);
          uint32_t out[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int e0 = c4 * 8 + 2 * q;
            const float y0 = __uint_as_float(ry[e0]) + carry * __uint_as_float(ro[e0]) + Dh * bf16_lo(xu[q]);
            const float y1 = __uint_as_float(ry[e0 + 1]) + carry * __uint_as_float(ro[e0 + 1]) + Dh * bf16_hi(xu[q]);
            out[q] = pack_bf16(y0, y1);
          }
          if (i < rem) *reinterpret_cast<uint4*>(yrow + 8 * c) = make_uint4(out[0], out[1], out[2], out[3]);
        }
      }
      const float decay = __expf(cs_end - cs_start);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t rs[32];
        tmem_ld32(tmem + lane_base + kColSt + hw * 64 + half * 32, rs);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 32; ++q) hst[half * 32 + q] = fmaf(decay, hst[half * 32 + q], __uint_as_float(rs[q]));
      }
    }

    const bool unit_done = !have_next || nxt.unit != cur.unit;
    if (unit_done && pb.final_state && i < NS) {
#pragma unroll
      for (int p = 0; p < kHeadDim; ++p) pb.final_state[st_base + (int64_t)p * NS + i] = hst[p];
    }
    if (unit_done) finish_empty_units(cur.unit + gridDim.x, have_next ? nxt.unit : pb.nseq * (pb.H / kHeads));
    tc_fence_before();
    __syncthreads();  // this stage's x and tensor memory are free again
    cur = nxt;
    have = have_next;
    stage ^= 1;
  }

  if (!ok) {
    // A wait gave up: drain what is still in flight (again bounded), record the failure.
    for (int k = 0; k < 2; ++k)
      if (pend_load & (1 << k)) mbar_wait_bounded(&bar_load[k], ph_load[k], kWaitLimit);
    if (pend_s) mbar_wait_bounded(bar_s, ph_s, kWaitLimit);
    if (pend_mma) mbar_wait_bounded(bar_mma, ph_mma, kWaitLimit);
    if (tid == 0) atomicOr(pb.status, kStatusTimeout);
  }
  tc_fence_before();
  __syncthreads();
  if (tid < 32) {
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

// 3-D bf16 map {inner, mid, tokens} with a {64, 1, 128} box and 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t tokens) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, mid, tokens};
  cuuint64_t strides[2] = {inner * 2, inner * mid * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)kTile};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NS>
cudaError_t launch_ns(const Problem& pb, cudaStream_t st) {
  CUtensorMap mx, mb, mc;
  const uint64_t tokens = (uint64_t)pb.tokens;
  if (!make_map(&mx, pb.x, kHeadDim, pb.H, tokens) || !make_map(&mb, pb.B, NS, pb.G, tokens) ||
      !make_map(&mc, pb.C, NS, pb.G, tokens))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(ssd_fused_tc_kernel<NS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kDynSmem<NS>);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int units = pb.nseq * (pb.H / kHeads);
  const int grid = units < sms ? units : sms;
  if (grid <= 0) return cudaSuccess;
  if (pb.prof_start) cudaEventRecord(pb.prof_start, st);
  ssd_fused_tc_kernel<NS><<<grid, kThreads, kDynSmem<NS>, st>>>(mx, mb, mc, pb);
  if (pb.prof_stop) cudaEventRecord(pb.prof_stop, st);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

bool tc_supports(const ssd_shape* s, int chunk) {
  if (!s || s->io_dtype != SSD_BF16 || s->headdim != kHeadDim) return false;
  if (s->dstate != 64 && s->dstate != 128) return false;
  if (s->nheads % kHeads || (s->nheads / s->ngroups) % kHeads) return false;  // head pairs share a group
  if (chunk != 128 && chunk != 256) return false;
  const int64_t tokens = s->batch * s->seqlen;
  return tokens >= 1 && tokens < ((int64_t)1 << 31) - kTile;
}

cudaError_t launch_tc(const Problem& pb, cudaStream_t st) {
  return pb.N == 128 ? launch_ns<128>(pb, st) : launch_ns<64>(pb, st);
}

}  // namespace ssd
