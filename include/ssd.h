/*
 * ssd.h -- C ABI of the B200 (sm_100a) chunked SSD forward library, libssd.so.
 *
 * SSD ("structured state space duality") is the sequence-mixing core of the
 * Mamba-2 layer ("Transformers are SSMs", Dao & Gu, ICML 2024).  For every
 * sequence and head h (group g = h / (H/G)), with a P x N fp32 state S:
 *
 *     a_t = exp(dt_t * A_h)                          (scalar decay per head)
 *     S_t = a_t * S_{t-1} + (dt_t * x_t) B_t^T       (x_t in R^P, B_t in R^N)
 *     y_t = S_t C_t + D_h * x_t
 *
 * which equals multiplication by the 1-semiseparable-masked matrix
 * M = L o (C B^T) (wikillm.com card, Method steps 1-3; sec. 2, 3, 5.1), computed
 * by the chunked algorithm (Method step 5, sec. 6: diagonal blocks, right,
 * centre and left factors) with chunk length `chunk`.  Discretisation follows
 * the card's Method step 7 / "Paper vs code" item 7: dt scales the input and the
 * decay; the D skip uses the unscaled x (item 3).
 *
 * Conventions for every entry point:
 *  - All tensors are dense, row-major and contiguous.  Unless an entry point
 *    says "host", every pointer is a DEVICE pointer of the current device and
 *    must be 16-byte aligned.  The caller owns every buffer; the library keeps
 *    no pointer after the call returns.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) unless stated otherwise.  Scratch memory, when needed, comes from a
 *    stream-ordered pool the library creates per device (cudaMallocFromPoolAsync
 *    / cudaFreeAsync on `stream`); freed blocks stay in that pool for later calls
 *    and are returned to the driver when the process exits.
 *  - The return value is an ssd_status.  On any host-detected error nothing is
 *    launched and no output is written.  Errors found on the device (bad
 *    cu_seqlens values, a bounded wait that ran out) are recorded in a per-device
 *    status word, read with ssd_query_status().  With SSD_DEBUG set in the
 *    environment, a failed tensor-core launch also prints its CUDA error to stderr.
 */
#ifndef SSD_H_
#define SSD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream, declared here so this header needs no CUDA header. */
typedef struct CUstream_st* ssd_stream_t;

typedef enum { SSD_F32 = 0, SSD_BF16 = 1 } ssd_dtype;

typedef enum {
  SSD_OK = 0,
  SSD_ERR_INVALID_ARG = 1,    /* null required pointer, negative size, bad dtype           */
  SSD_ERR_UNSUPPORTED = 2,    /* chunk not in {64,128,256}, H % G != 0, P or N outside 1..256 */
  SSD_ERR_MISALIGNED = 3,     /* a pointer is not 16-byte aligned                            */
  SSD_ERR_CUDA = 4,           /* a CUDA runtime call or kernel launch failed                 */
  SSD_ERR_DEVICE_TIMEOUT = 5, /* a bounded device-side wait gave up (kernel returned early)  */
  SSD_ERR_BAD_SEQLENS = 6,    /* cu_seqlens not 0 = c0 <= c1 <= ... <= c_nseq = seqlen        */
  SSD_ERR_SCRATCH_LIMIT = 7   /* ssd_forward_noalloc: the shape needs more scratch than
                                 SSD_NOALLOC_SCRATCH_BYTES                                   */
} ssd_status;

/*
 * Problem shape.  Raw pointers carry no shapes, so every call takes one.
 *   batch    dense batch rows (must be 1 when cu_seqlens is given)
 *   seqlen   tokens per row; for a packed batch, the total number of tokens T
 *   nheads   H;  headdim P;  dstate N;  ngroups G (H % G == 0, heads h*G/H share B, C)
 *   nseq     number of packed sequences when cu_seqlens is given (ignored otherwise)
 *   io_dtype dtype of x, B, C and y (dt, A, D and the states are always fp32)
 *   cu_seqlens_host  optional HOST copy of cu_seqlens; when given it is validated on
 *            the host (SSD_ERR_BAD_SEQLENS) before anything is launched.
 */
typedef struct {
  int64_t batch, seqlen, nheads, headdim, dstate, ngroups, nseq;
  ssd_dtype io_dtype;
  const int32_t* cu_seqlens_host;
} ssd_shape;

/*
 * ssd_forward -- the chunked SSD forward pass (wikillm.com card, Method step 5, sec. 6,
 * Theorem 6.1; varlen per the GVA / variable-length note of the Chinese wiki page).
 *
 *   x           (batch, seqlen, H, P)  io_dtype   input
 *   dt          (batch, seqlen, H)     fp32       step sizes, > 0 (already softplus'ed)
 *   A           (H)                    fp32       decay rates, < 0 (A = -exp(A_log))
 *   B, C        (batch, seqlen, G, N)  io_dtype   SSM input / output matrices
 *   D           (H)                    fp32       skip weights, or NULL (= 0)
 *   init_state  (nseq_or_batch, H, P, N) fp32     state before each sequence, or NULL (= 0)
 *   cu_seqlens  (nseq + 1)             int32      packed-sequence offsets (device), or NULL
 *                                                 for a dense batch; the state resets at each
 *                                                 sequence start
 *   chunk       Q in {64, 128, 256}: length of the chunks of the block decomposition
 *   y           (batch, seqlen, H, P)  io_dtype   output (may not alias an input)
 *   final_state (nseq_or_batch, H, P, N) fp32     state after each sequence, or NULL
 * When the shape has no tokens (every sequence empty), x, dt, B, C and y may be NULL and
 * final_state gets init_state (or zeros).  With y == NULL and final_state given, only the
 * final states are computed: C and D are not read (either may be NULL), and the
 * tensor-core kernel loads only x, dt and B (the first pass of sequence parallelism).
 * Returns SSD_OK or an error code (see ssd_status).  Asynchronous on `stream`.
 */
int ssd_forward(const ssd_shape* shape, const void* x, const float* dt, const float* A, const void* B,
                const void* C, const float* D, const float* init_state, const int32_t* cu_seqlens, int chunk,
                void* y, float* final_state, ssd_stream_t stream);

/*
 * ssd_forward_dt -- ssd_forward with the step size made inside the kernels from the raw
 * per-head projection, as the pages' discretisation does it (the wikillm.com card: the
 * Mamba-2 block sketch of sec. 7.1, Method note 7 "Discretisation", "Paper vs code" 7:
 * dt = softplus(dt_raw + dt_bias)).  Every kernel that reads dt applies, per token t
 * and head h,
 *     v  = dt_raw[t,h] + (dt_bias ? dt_bias[h] : 0)
 *     dt = softplus ? log(1 + exp(v)) : v,   then clamped to [dt_min, dt_max]
 * so no separate pass over dt precedes the call.  `dt_raw` has dt's layout (batch,
 * seqlen, H) fp32; dt_bias is (H) fp32 on the device or NULL; use dt_min = 0 and
 * dt_max = INFINITY for no clamp.  prologue == NULL is ssd_forward.  Errors as
 * ssd_forward, plus SSD_ERR_INVALID_ARG for dt_min < 0, dt_max < dt_min or a NaN bound
 * and SSD_ERR_MISALIGNED for a dt_bias not 16-byte aligned.
 */
typedef struct {
  const float* dt_bias;  /* (H) fp32 device pointer, or NULL (= 0) */
  int softplus;          /* 1: dt = softplus(dt_raw + dt_bias); 0: dt = dt_raw + dt_bias */
  float dt_min, dt_max;  /* clamp after softplus */
} ssd_dt_prologue;
int ssd_forward_dt(const ssd_shape* shape, const ssd_dt_prologue* prologue, const void* x, const float* dt_raw,
                   const float* A, const void* B, const void* C, const float* D, const float* init_state,
                   const int32_t* cu_seqlens, int chunk, void* y, float* final_state, ssd_stream_t stream);

/*
 * ssd_forward_host -- the same computation on HOST buffers (pinned memory gives full
 * copy bandwidth; pageable memory works but its copies do not overlap).  The
 * sequences are split into up to 8 groups of whole sequences with about equal token
 * counts; device buffers come from the library's pool; group g's inputs are copied in
 * on one library stream while group g-1 runs ssd_forward on `stream` and group g-2's
 * outputs are copied back on another, and the call synchronises all of them before
 * returning.  Every sequence's outputs are the ones a single ssd_forward call gives.
 * Same layouts and errors as ssd_forward; cu_seqlens is a host pointer here and is
 * checked on the host (SSD_ERR_BAD_SEQLENS).  Returns SSD_ERR_DEVICE_TIMEOUT when the
 * device reported one during this call.  The two copy streams and their events are
 * created on a device's first call and kept; calls on one device from several host
 * threads take turns (a per-device lock).
 */
int ssd_forward_host(const ssd_shape* shape, const void* x, const float* dt, const float* A, const void* B,
                     const void* C, const float* D, const float* init_state, const int32_t* cu_seqlens, int chunk,
                     void* y, float* final_state, ssd_stream_t stream);

/*
 * ssd_forward_noalloc -- ssd_forward for callers that cannot allocate device memory.
 * The paper has no counterpart to this entry point; it exists for integration.
 *
 * Who needs it: a caller that reserves the GPU's memory up front and hands it out
 * itself (an inference server that gives nearly all HBM to weights and KV caches, or
 * a runtime that accounts for every byte through its own pool) cannot let a library
 * allocate device memory (cudaMallocAsync or a pool of its own): the allocation can
 * fail once the memory is spent, and it can stall a latency-critical loop while the
 * driver grows or trims a pool.
 *
 * Same arguments, layouts and results as ssd_forward.  It always runs the SIMT
 * kernels, and their scratch (chunk table, cumsums, chunk states) lives in one
 * file-scope device array of SSD_NOALLOC_SCRATCH_BYTES that every GPU loading this
 * library holds until the process exits.  No call allocates: no cudaMalloc,
 * cudaMallocAsync, cudaFree or allocating library routine.
 *  - Shapes whose scratch exceeds SSD_NOALLOC_SCRATCH_BYTES (ssd_workspace_bytes with
 *    ssd_set_path(SSD_PATH_SIMT) gives the need) return SSD_ERR_SCRATCH_LIMIT and
 *    launch nothing.
 *  - Every call looks up the array's device address on the current device
 *    (cudaGetSymbolAddress, which allocates nothing), so a context recreated after a
 *    device reset gets its own copy of the array.  The first call on a device loads
 *    the module there; make that first call before any stream capture.
 *  - All calls share the one array and it keeps the last call's contents; each call
 *    first resets the word that marks the chunk table as not yet built.  Calls whose
 *    work overlaps on the GPU (different streams, or different host threads, without
 *    ordering between them) race on the array: serialise them.
 */
#define SSD_NOALLOC_SCRATCH_BYTES (32u << 20)
int ssd_forward_noalloc(const ssd_shape* shape, const void* x, const float* dt, const float* A, const void* B,
                        const void* C, const float* D, const float* init_state, const int32_t* cu_seqlens,
                        int chunk, void* y, float* final_state, ssd_stream_t stream);

/*
 * ssd_decode_step -- one recurrent generation step for a batch of sequences (the
 * wikillm.com card, Method step 8 and sec. 6.3: in generation the layer runs as its
 * linear recurrence, N^2 work per token and head).  For every row b and head h, with
 * g = h / (H/G) and the fp32 state S = state[b,h] (P x N, N contiguous), in place:
 *   a = exp(dt[b,h] A[h]);  S <- a S + dt[b,h] x[b,h,:] B[b,g,:]^T;
 *   y[b,h,:] = S C[b,g,:] + D[h] x[b,h,:]
 * This is the same recurrence ssd_forward evaluates in chunks, one token at a time:
 * T steps from init_state give ssd_forward's y rows and final_state.
 *
 *   shape       batch = rows, seqlen = 1, nheads H, headdim P, dstate N (N % 4 == 0,
 *               N <= 256), ngroups G; io_dtype for x, B, C, y; nseq and
 *               cu_seqlens_host unused
 *   x, y        (batch, H, P)       io_dtype
 *   dt          (batch, H)          fp32, > 0
 *   A, D        (H)                 fp32 (D may be NULL = 0)
 *   B, C        (batch, G, N)       io_dtype
 *   state       (batch, H, P, N)    fp32, read and overwritten
 * Device pointers, 16-byte aligned; no scratch; asynchronous on `stream`.  Errors:
 * SSD_ERR_INVALID_ARG (null pointer, seqlen != 1), SSD_ERR_UNSUPPORTED (N % 4, N > 256,
 * H % G), SSD_ERR_MISALIGNED, SSD_ERR_CUDA; nothing is launched on an error.
 */
int ssd_decode_step(const ssd_shape* shape, const void* x, const float* dt, const float* A, const void* B,
                    const void* C, const float* D, float* state, void* y, ssd_stream_t stream);

/*
 * ssd_causal_conv1d_silu -- the step before the SSD in the Mamba-2 block (the wikillm.com
 * card: the Mamba-2 block sketch of sec. 7.1, "Paper vs code" 1 and 2): a depthwise causal
 * convolution of kernel 4 over the concatenated x, B, C channels, then SiLU,
 *     out[t,c] = silu(bias[c] + sum_{k=0..3} weight[c,k] in[t-3+k, c]),  silu(v) = v / (1 + e^-v)
 * with in[] = 0 before each sequence's first token (the window restarts at every sequence).
 *   xbc, out    (batch, seqlen, channels)  io_dtype (out may not alias xbc)
 *   weight      (channels, 4)              fp32;  bias (channels) fp32 or NULL (= 0)
 *   cu_seqlens  (nseq + 1) int32 on the device, or NULL for a dense batch; it must be a
 *               valid offset list (0 = c_0 <= ... <= c_nseq = seqlen, batch = 1): this
 *               call does not check its values.
 * channels % 8 == 0 (SSD_ERR_UNSUPPORTED otherwise).  Device pointers, 16-byte aligned;
 * no scratch; asynchronous on `stream`.
 */
int ssd_causal_conv1d_silu(int64_t batch, int64_t seqlen, int64_t channels, ssd_dtype io_dtype, const void* xbc,
                           const float* weight, const float* bias, const int32_t* cu_seqlens, int64_t nseq,
                           void* out, ssd_stream_t stream);

/*
 * ssd_gated_rmsnorm -- the step after the SSD in the Mamba-2 block (the wikillm.com card:
 * the Mamba-2 block sketch of sec. 7.1 and "Paper vs code" 9: gated RMSNorm, gate before
 * the norm, eps 1e-5 there), per token over its `dim` features:
 *     g = y * silu(z);   out = g / sqrt(mean(g^2) + eps) * weight
 *   y, z, out   (tokens, dim)  io_dtype;   weight (dim) fp32
 * dim % 8 == 0 and dim <= 8192.  Device pointers, 16-byte aligned; asynchronous on `stream`.
 */
int ssd_gated_rmsnorm(int64_t tokens, int64_t dim, ssd_dtype io_dtype, const void* y, const void* z,
                      const float* weight, float eps, void* out, ssd_stream_t stream);

/*
 * Sequence-parallel SSD (one sequence split into contiguous segments, one per GPU): the
 * state passes from segment to segment exactly as from chunk to chunk (the wikillm.com
 * card, Method step 5, the centre factor).  Each rank r runs ssd_forward on its segment
 * from a zero state, giving its end state s_r, and ssd_segment_logdecay gives
 * lambda_r[h] = A[h] * sum_t dt[t,h] over the segment.  After an all-gather of (s, lambda),
 * ssd_state_prefix gives the segment's true start state
 *     h_0 = init,  h_{q+1} = exp(lambda_q) h_q + s_q   (q < rank),
 * and the rank runs ssd_forward again from it.  See sequence_parallel.py in the package.
 *
 * ssd_segment_logdecay: dt (tokens, H) fp32, A (H) fp32 -> out (H) fp32.
 * ssd_state_prefix: states (>= rank, H, P, N) and logdecay (>= rank, H) of the
 *   preceding segments, init_state (H, P, N) or NULL (= 0) -> out (H, P, N); all fp32.
 * Device pointers; asynchronous on `stream`; SSD_ERR_INVALID_ARG for bad sizes or nulls.
 */
int ssd_segment_logdecay(int64_t tokens, int64_t nheads, const float* dt, const float* A, float* out,
                         ssd_stream_t stream);
int ssd_state_prefix(int rank, int64_t nheads, int64_t headdim, int64_t dstate, const float* states,
                     const float* logdecay, const float* init_state, float* out, ssd_stream_t stream);

/* Bytes of stream-ordered scratch ssd_forward takes for this shape (informational). */
size_t ssd_workspace_bytes(const ssd_shape* shape, int chunk);

/*
 * Synchronises `stream`, then returns and clears the current device's status word:
 * SSD_OK, SSD_ERR_BAD_SEQLENS or SSD_ERR_DEVICE_TIMEOUT (SSD_ERR_CUDA if the
 * synchronisation itself failed).
 */
int ssd_query_status(ssd_stream_t stream);

/* Static, human-readable text for a status code. */
const char* ssd_status_string(int status);

/*
 * Kernel path selection, process-wide (not thread-safe; meant for tests and benches):
 *   SSD_PATH_AUTO  the tensor-core (tcgen05) path where the shape supports it, else SIMT
 *   SSD_PATH_SIMT  the general CUDA-core path for every shape and dtype
 *   SSD_PATH_TC    the tensor-core path; shapes it cannot take return SSD_ERR_UNSUPPORTED
 * Returns the previous setting.
 */
enum { SSD_PATH_AUTO = 0, SSD_PATH_SIMT = 1, SSD_PATH_TC = 2 };
int ssd_set_path(int path);

/* Which path ssd_forward would take for this shape and chunk under the current setting
 * (SSD_PATH_SIMT or SSD_PATH_TC), or a negative ssd_status when it would fail. */
int ssd_select_path(const ssd_shape* shape, int chunk);

/* Same type as cudaEvent_t / CUevent. */
typedef struct CUevent_st* ssd_event_t;

/*
 * Measurement hooks (process-wide, not thread-safe; meant for benches).
 * ssd_profile_dominant: when both events are non-NULL, every later ssd_forward records
 * `start` on its stream just before its dominant kernel (the one that moves the bulk
 * of the bytes: the fused tensor-core kernel, or the SIMT output kernel) and `stop`
 * just after it; NULL, NULL turns this off.  The events are the caller's.
 * ssd_kernel_launch_count: kernels launched by this library so far in this process.
 */
int ssd_profile_dominant(ssd_event_t start, ssd_event_t stop);
uint64_t ssd_kernel_launch_count(void);

/*
 * Test hooks for the failure path of the tensor-core kernel (process-wide, not
 * thread-safe; meant for tests).  Every device-side wait of that kernel is bounded:
 * after `wait_limit_cycles` SM clock cycles (0 = the default, 2^32, about 2 s) it gives
 * up, the kernel drains its in-flight copies and tensor-core work, frees tensor memory
 * and returns, and ssd_query_status() reports SSD_ERR_DEVICE_TIMEOUT; the outputs of
 * that call are then undefined.  `withhold` is a bit mask of flags to keep back, the only
 * way a test makes a wait fail:
 *   bit 0 (1): every CTA keeps back the flag that hands its state on to the next CTA (the
 *              state itself is still written), so the CTAs that wait for it run out of time;
 *   bit 1 (2): CTA 0 keeps back its flag of the barrier after the work split's tile weights
 *              (launches that weigh their tiles in the kernel), so every CTA's wait there
 *              runs out of time and no CTA takes any work.
 * Returns SSD_OK, or SSD_ERR_INVALID_ARG for a negative limit or other bits.
 */
int ssd_set_test_hooks(int64_t wait_limit_cycles, int withhold);

#ifdef __cplusplus
}
#endif
#endif /* SSD_H_ */
