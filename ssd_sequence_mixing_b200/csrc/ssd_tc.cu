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

constexpr int kTile = 128;     // tokens per tile (UMMA M)
constexpr int kHeadDim = 64;   // P supported by this path
constexpr int kThreads = 128;  // one warpgroup: thread i <-> TMEM lane i
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColY = 128, kColYo = 192, kColSt = 256;
constexpr long long kWaitLimit = 4ll << 30;  // SM cycles (about 2 s) before a wait gives up

template <int NS>
struct Layout {
  static constexpr uint32_t x = 0;                       // [128 tok][64 p]      16 KB
  static constexpr uint32_t b = x + kTile * 128;          // NS/64 atoms [128 tok][64 n]
  static constexpr uint32_t c = b + (NS / 64) * kTile * 128;
  static constexpr uint32_t p = c + (NS / 64) * kTile * 128;  // 2 K-atoms [128 i][64 j]  32 KB
  static constexpr uint32_t xw = p + 2 * kTile * 128;    // [128 tok][64 p]      16 KB
  static constexpr uint32_t ht = xw + kTile * 128;       // [NS n][64 p]
  static constexpr uint32_t cs = ht + NS * 128;          // float[128]
  static constexpr uint32_t dt = cs + kTile * 4;         // float[128]
  static constexpr uint32_t red = dt + kTile * 4;        // float[4]
  static constexpr uint32_t bars = red + 64;             // 2 x uint64
  static constexpr uint32_t tmem = bars + 16;            // uint32
  static constexpr uint32_t flags = tmem + 16;           // int
  static constexpr uint32_t bytes = flags + 16;
  static constexpr uint32_t dyn_bytes = bytes + 1024;    // + alignment slack
};

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

template <int NS>
__global__ void __launch_bounds__(kThreads, 1)
    ssd_fused_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                        const __grid_constant__ CUtensorMap tm_c, Problem pb) {
  using L = Layout<NS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sx = smem + L::x;
  uint8_t* sb = smem + L::b;
  uint8_t* sc = smem + L::c;
  uint8_t* sp = smem + L::p;
  uint8_t* sxw = smem + L::xw;
  uint8_t* sht = smem + L::ht;
  float* s_cs = reinterpret_cast<float*>(smem + L::cs);
  float* s_dt = reinterpret_cast<float*>(smem + L::dt);
  float* s_red = reinterpret_cast<float*>(smem + L::red);
  uint64_t* bar_load = reinterpret_cast<uint64_t*>(smem + L::bars);
  uint64_t* bar_mma = bar_load + 1;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + L::tmem);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (*pb.nchunks < 0) return;  // cu_seqlens rejected by the table kernel

  if (warp == 0) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar_load, 1);
    mbar_init(bar_mma, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tensormap(&tm_x);
    prefetch_tensormap(&tm_b);
    prefetch_tensormap(&tm_c);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  uint32_t ph_load = 0, ph_mma = 0;
  bool ok = true;
  bool load_pending = false, mma_pending = false;  // async work issued and not yet waited for

  constexpr uint32_t kAtom = kTile * 128;  // bytes of one 128-row, 128-byte-wide swizzle column
  const uint32_t id_s = idesc_bf16(128, 128, 0, 0);
  const uint32_t id_y = idesc_bf16(128, 64, 0, 1);
  const uint32_t id_st = idesc_bf16(128, 64, 1, 1);
  const uint32_t a_sx = smem_u32(sx), a_sb = smem_u32(sb), a_sc = smem_u32(sc), a_sp = smem_u32(sp);
  const uint32_t a_sxw = smem_u32(sxw), a_sht = smem_u32(sht);
  // For N = 64 the B^T operand has one M atom; the second (unused) half of s^T reads
  // the C tile that follows it, and those lanes are ignored.
  const uint32_t lbo_bt = kAtom;

  const int units = pb.nseq * pb.H;
  for (int unit = blockIdx.x; unit < units && ok; unit += gridDim.x) {
    const int s = unit / pb.H, h = unit % pb.H, g = h / pb.hpg;
    const int64_t tb = seq_off(pb, s);
    const int len = (int)(seq_off(pb, s + 1) - tb);
    const float Ah = pb.A[h];
    const float Dh = pb.D ? pb.D[h] : 0.f;
    const int64_t st_base = ((int64_t)s * pb.H + h) * kHeadDim * NS;

    // thread n keeps column n of the state: hst[p] = h[p][n]
    float hst[kHeadDim];
#pragma unroll
    for (int p = 0; p < kHeadDim; ++p) hst[p] = 0.f;
    if (pb.init && tid < NS) {
#pragma unroll
      for (int p = 0; p < kHeadDim; ++p) hst[p] = pb.init[st_base + (int64_t)p * NS + tid];
    }

    float cs_base = 0.f;
    for (int k0 = 0; k0 < len && ok; k0 += kTile) {
      const int64_t t0 = tb + k0;
      const int rem = min(kTile, len - k0);
      if (k0 % pb.Q == 0) cs_base = 0.f;

      // ---- TMA: x, B, C tiles
      load_pending = true;
      if (tid == 0) {
        fence_proxy_async();
        mbar_expect_tx(bar_load, kAtom + 2u * (NS / 64) * kAtom);
        tma_load_3d(sx, &tm_x, 0, h, (int)t0, bar_load);
#pragma unroll
        for (int a = 0; a < NS / 64; ++a) {
          tma_load_3d(sb + a * kAtom, &tm_b, a * 64, g, (int)t0, bar_load);
          tma_load_3d(sc + a * kAtom, &tm_c, a * 64, g, (int)t0, bar_load);
        }
      }

      // ---- in-chunk cumsum of dt*A (overlaps the loads)
      float dtj = 0.f, l = 0.f;
      if (tid < rem) {
        dtj = pb.dt[(t0 + tid) * pb.H + h];
        l = dtj * Ah;
      }
      float v = l;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
      }
      if (lane == 31) s_red[warp] = v;
      __syncthreads();
      float off = cs_base;
      for (int w = 0; w < warp; ++w) off += s_red[w];
      const float cs_i = off + v;
      s_cs[tid] = cs_i;
      s_dt[tid] = dtj;
      __syncthreads();
      const float cs_start = cs_base;
      const float cs_end = s_cs[kTile - 1];  // rows past the end add 0
      cs_base = cs_end;
      const float w_i = __expf(cs_end - cs_i) * dtj;  // right-factor weight of token i (0 past the end)

      // ---- wait for the tiles, then S = C B^T
      ok = mbar_wait_bounded(bar_load, ph_load, kWaitLimit);
      if (__syncthreads_or(!ok)) {
        ok = false;
        break;
      }
      ph_load ^= 1;
      load_pending = false;
      mma_pending = true;
      if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < NS / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * kAtom + (kk & 3) * 32;
          umma_f16(tmem + kColS, sdesc_sw128(a_sc + koff, 16, 1024), sdesc_sw128(a_sb + koff, 16, 1024), id_s,
                   kk > 0);
        }
        umma_commit(bar_mma);
      }

      // ---- w o X (right-factor input) and the bf16 state copy, while S runs
      {
        const int j = tid;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t o = sw128_off(j, c);
          uint4 xv = *reinterpret_cast<const uint4*>(sx + o);
          uint32_t* u = reinterpret_cast<uint32_t*>(&xv);
#pragma unroll
          for (int q = 0; q < 4; ++q) u[q] = pack_bf16(bf16_lo(u[q]) * w_i, bf16_hi(u[q]) * w_i);
          *reinterpret_cast<uint4*>(sxw + o) = xv;
        }
        if (tid < NS) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint4 hv;
            hv.x = pack_bf16(hst[8 * c + 0], hst[8 * c + 1]);
            hv.y = pack_bf16(hst[8 * c + 2], hst[8 * c + 3]);
            hv.z = pack_bf16(hst[8 * c + 4], hst[8 * c + 5]);
            hv.w = pack_bf16(hst[8 * c + 6], hst[8 * c + 7]);
            *reinterpret_cast<uint4*>(sht + sw128_off(tid, c)) = hv;
          }
        }
      }

      // ---- P = mask(S), written K-major (two 64-column K atoms)
      ok = mbar_wait_bounded(bar_mma, ph_mma, kWaitLimit);
      if (__syncthreads_or(!ok)) {
        ok = false;
        break;
      }
      ph_mma ^= 1;
      mma_pending = false;
      tc_fence_after();
      {
        const int i = tid;
#pragma unroll 1
        for (int cb = 0; cb < 4; ++cb) {  // 32-column blocks of S
          uint32_t pk[16];
          if (cb <= warp) {  // blocks right of this warp's rows are all zero
            uint32_t r[32];
            tmem_ld32(tmem + lane_base + kColS + cb * 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              float e[2];
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const int j = cb * 32 + 2 * q + u;
                e[u] = 0.f;
                if (j <= i && j < rem) e[u] = __uint_as_float(r[2 * q + u]) * __expf(cs_i - s_cs[j]) * s_dt[j];
              }
              pk[q] = pack_bf16(e[0], e[1]);
            }
          } else {
#pragma unroll
            for (int q = 0; q < 16; ++q) pk[q] = 0u;
          }
          const int katom = cb >> 1;
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const int c = (cb & 1) * 4 + c4;
            *reinterpret_cast<uint4*>(sp + katom * kAtom + sw128_off(i, c)) =
                make_uint4(pk[4 * c4], pk[4 * c4 + 1], pk[4 * c4 + 2], pk[4 * c4 + 3]);
          }
        }
      }
      fence_proxy_async();
      tc_fence_before();
      __syncthreads();

      // ---- Y = P X, Yo = C h^T, s^T = B^T (w o X)
      mma_pending = true;
      if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * kAtom + (kk & 3) * 32;
          umma_f16(tmem + kColY, sdesc_sw128(a_sp + koff, 16, 1024), sdesc_sw128(a_sx + kk * 2048, kAtom, 1024),
                   id_y, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < NS / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * kAtom + (kk & 3) * 32;
          umma_f16(tmem + kColYo, sdesc_sw128(a_sc + koff, 16, 1024), sdesc_sw128(a_sht + kk * 2048, kAtom, 1024),
                   id_y, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          umma_f16(tmem + kColSt, sdesc_sw128(a_sb + kk * 2048, lbo_bt, 1024),
                   sdesc_sw128(a_sxw + kk * 2048, kAtom, 1024), id_st, kk > 0);
        }
        umma_commit(bar_mma);
      }
      ok = mbar_wait_bounded(bar_mma, ph_mma, kWaitLimit);
      if (__syncthreads_or(!ok)) {
        ok = false;
        break;
      }
      ph_mma ^= 1;
      mma_pending = false;
      tc_fence_after();

      // ---- epilogue: y rows and the state update
      {
        const int i = tid;
        const float carry = __expf(cs_i - cs_start);
        __nv_bfloat16* yrow = static_cast<__nv_bfloat16*>(pb.y) + ((t0 + i) * pb.H + h) * kHeadDim;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t ry[32], ro[32];
          tmem_ld32(tmem + lane_base + kColY + half * 32, ry);
          tmem_ld32(tmem + lane_base + kColYo + half * 32, ro);
          tmem_ld_wait();
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const int c = half * 4 + c4;  // 16-byte chunk of the 64-wide row: p = 8c..8c+7
            const uint4 xv = *reinterpret_cast<const uint4*>(sx + sw128_off(i, c));
            const uint32_t* xu = reinterpret_cast<const uint32_t*>(&xv);
            uint32_t out[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int e0 = c4 * 8 + 2 * q;
              const float y0 = __uint_as_float(ry[e0]) + carry * __uint_as_float(ro[e0]) + Dh * bf16_lo(xu[q]);
              const float y1 =
                  __uint_as_float(ry[e0 + 1]) + carry * __uint_as_float(ro[e0 + 1]) + Dh * bf16_hi(xu[q]);
              out[q] = pack_bf16(y0, y1);
            }
            if (i < rem) *reinterpret_cast<uint4*>(yrow + 8 * c) = make_uint4(out[0], out[1], out[2], out[3]);
          }
        }
        const float decay = __expf(cs_end - cs_start);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t rs[32];
          tmem_ld32(tmem + lane_base + kColSt + half * 32, rs);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 32; ++q) hst[half * 32 + q] = fmaf(decay, hst[half * 32 + q], __uint_as_float(rs[q]));
        }
      }
      tc_fence_before();
      __syncthreads();  // x tile and TMEM are free for the next tile
    }

    if (ok && pb.final_state && tid < NS) {
#pragma unroll
      for (int p = 0; p < kHeadDim; ++p) pb.final_state[st_base + (int64_t)p * NS + tid] = hst[p];
    }
  }

  if (!ok) {
    // A wait gave up: drain what is still in flight (again bounded), record the failure.
    if (load_pending) mbar_wait_bounded(bar_load, ph_load, kWaitLimit);
    if (mma_pending) mbar_wait_bounded(bar_mma, ph_mma, kWaitLimit);
    if (tid == 0) atomicOr(pb.status, kStatusTimeout);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
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
  using L = Layout<NS>;
  cudaError_t e = cudaFuncSetAttribute(ssd_fused_tc_kernel<NS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)L::dyn_bytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int units = pb.nseq * pb.H;
  const int grid = units < sms ? units : sms;
  if (grid <= 0) return cudaSuccess;
  if (pb.prof_start) cudaEventRecord(pb.prof_start, st);
  ssd_fused_tc_kernel<NS><<<grid, kThreads, L::dyn_bytes, st>>>(mx, mb, mc, pb);
  if (pb.prof_stop) cudaEventRecord(pb.prof_stop, st);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

bool tc_supports(const ssd_shape* s, int chunk) {
  if (!s || s->io_dtype != SSD_BF16 || s->headdim != kHeadDim) return false;
  if (s->dstate != 64 && s->dstate != 128) return false;
  if (chunk != 128 && chunk != 256) return false;
  const int64_t tokens = s->batch * s->seqlen;
  return tokens >= 1 && tokens < ((int64_t)1 << 31) - kTile;
}

cudaError_t launch_tc(const Problem& pb, cudaStream_t st) {
  return pb.N == 128 ? launch_ns<128>(pb, st) : launch_ns<64>(pb, st);
}

}  // namespace ssd
