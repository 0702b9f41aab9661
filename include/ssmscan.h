/*
 * ssmscan.h -- C ABI of libssmscan, a CUDA (sm_100a) implementation of the
 * Mamba selective-scan forward pass, its single-token decode step and the
 * Mamba-2 scalar-decay (SSD) chunked scan.
 *
 * Definitions (page titles as printed on the source pages):
 *  - "Mamba状态空间模型的硬件感知推理优化" (ybb.press), section 1:
 *      h_t = A h_{t-1} + B x_t,   y_t = C h_t;
 *    section 3.1 (fused scan kernel): y = C h + D x, with the decay
 *    A_t = exp(A * softplus(dt)) applied per step.
 *  - "Mamba ... 并行扫描" (mhpq.cn), sections 2.2-2.3 and 3.1: A_d =
 *    exp(A dt) with A diagonal, so the decay is an elementwise exp; the
 *    recurrence is evaluated with the combine operator
 *    (A1, B1) (+) (A2, B2) = (A2 A1, A2 B1 + B2).
 *  - "从硬件感知到算法革命：Mamba如何重塑序列建模的计算效率"
 *    (tencentcloud), section 2: dt = softplus(.), B and C depend on the
 *    input; section 3: the SiLU gate fused after the SSM.
 *  - "Mamba与选择性SSM" (mlqm.cn), section 5.4: incremental decoding keeps
 *    only the fixed-size state.
 *  - "Mamba状态空间模型的硬件感知推理优化" (ybb.press), section 4: the
 *    Mamba-2 scalar decay h_t = a_t h_{t-1} + b_t x_t, evaluated as a
 *    parallel/serial hybrid over chunks.
 *
 * Per channel (b, d) and state n the selective scan computes
 *   dt'     = softplus(delta[b,d,t] + delta_bias[d])   (or the sum itself
 *             when delta_softplus == 0)
 *   dA      = exp(dt' * A[d,n])
 *   h[n]    = dA * h[n] + dt' * B[b,n,t] * u[b,d,t]
 *   y[b,d,t]= (sum_n C[b,n,t] h[n] + D[d] u[b,d,t]) * silu(z[b,d,t])
 * and returns the final state h_L.  The skip term sits inside the gate.
 *
 * Conventions shared by every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller, except
 *    those of ssm_scan_fwd_host, which are host pointers.  The library
 *    allocates no device memory; scratch is passed as `workspace` (or
 *    `staging`) of the size the matching *_size call reports, or, for
 *    ssm_scan_fwd_noalloc, comes from a static array.
 *  - Calls are asynchronous on `stream` (0 = legacy default stream).
 *    Argument checks run on the host before any launch and return
 *    synchronously; a failed launch returns SSM_ERR_CUDA.
 *  - Kernels launch on the calling thread's current CUDA device: `stream`
 *    must belong to it, and every device pointer (workspace and staging
 *    included) must be memory that device can address, normally its own.
 *    The library cannot check this.
 *  - Outputs must not alias inputs, except `state` of ssm_scan_step.
 *  - Floating-point work is done in fp32; bf16 tensors are widened on load
 *    and y is rounded to nearest-even on store.  The state and h0 / h_last
 *    are always fp32.
 */
#ifndef SSMSCAN_H
#define SSMSCAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* ssm_stream_t; /* the same type as cudaStream_t */

typedef enum { SSM_F32 = 0, SSM_BF16 = 1 } ssm_dtype_t;

typedef enum {
  SSM_OK = 0,
  SSM_ERR_INVALID_ARG = 1,  /* null required pointer, negative size, bad flag */
  SSM_ERR_UNSUPPORTED = 2,  /* size or option outside what is implemented  */
  SSM_ERR_ALIGNMENT = 3,    /* a pointer or stride breaks a required alignment */
  SSM_ERR_CUDA = 4,         /* a CUDA launch or runtime call failed          */
  SSM_ERR_WORKSPACE = 5     /* workspace missing or smaller than required    */
} ssm_status_t;

/* ------------------------------------------------------------------------
 * Mamba-1 selective scan over a whole sequence.
 *
 * Layout (element strides; a stride of 0 selects the contiguous default):
 *   u, delta, z, y : (batch, dim, seqlen), unit stride along seqlen;
 *                    *_stride[0] = batch stride, *_stride[1] = dim stride
 *                    (defaults dim*seqlen and seqlen).
 *   B, C           : (batch, dstate, seqlen), unit stride along seqlen;
 *                    *_stride[0] = batch stride, *_stride[1] = state stride
 *                    (defaults dstate*seqlen and seqlen).
 *   A              : (dim, dstate) fp32, contiguous.
 *   D, delta_bias  : (dim) fp32, or NULL (no skip term / zero bias).
 *   z              : or NULL (no gate).
 *   h0, h_last     : (batch, dim, dstate) fp32, contiguous; h0 NULL means a
 *                    zero initial state, h_last NULL means it is not written.
 * Sizes: batch, dim >= 0; 1 <= dstate <= 16; seqlen >= 0.  seqlen == 0 only
 * writes h_last (= h0, or zeros).
 * Element type: `dtype` applies to u, delta, z, B, C and y.
 * Alignment: every pointer must be aligned to its element size.  Rows that
 * start on 16-byte boundaries (pointers and strides) take the vectorised
 * load path; others take a scalar-load path with the same results.
 * Split-and-resume: scanning [0, m) with h_last = h_m and then [m, L) with
 * h0 = h_m gives the same y and h_L as one scan (strides allow passing the
 * two halves of one tensor in place).
 */
typedef struct {
  int64_t batch, dim, dstate, seqlen;
  ssm_dtype_t dtype;
  const void* u;
  const void* delta;
  const float* A;
  const void* B;
  const void* C;
  const float* D;
  const void* z;
  const float* delta_bias;
  int delta_softplus;
  const float* h0;
  void* y;
  float* h_last;
  int64_t u_stride[2], delta_stride[2], z_stride[2], y_stride[2];
  int64_t B_stride[2], C_stride[2];
  /* Grouped B and C: with ngroups > 1, B and C are (batch, ngroups, dstate,
   * seqlen) and channel d reads group d / (dim / ngroups); dim / ngroups must
   * be a multiple of 32 (SSM_ERR_UNSUPPORTED otherwise).  *_group_stride is
   * the element stride between groups (0: the default dstate*seqlen); the
   * default batch stride becomes ngroups*dstate*seqlen.  0 or 1: one group
   * (the layout above).  Negative: SSM_ERR_INVALID_ARG. */
  int64_t ngroups;
  int64_t B_group_stride, C_group_stride;
} ssm_scan_args_t;

/* Bytes of scratch ssm_scan_fwd needs for these arguments (0 when the whole
 * sequence runs as one segment).  Only sizes, dtype, strides and pointer
 * alignment are looked at; null pointers are accepted.  Returns (size_t)-1
 * for invalid arguments. */
size_t ssm_scan_fwd_workspace_size(const ssm_scan_args_t* args);

/* Runs the selective scan.  `workspace` (device memory, 16-byte aligned,
 * at least ssm_scan_fwd_workspace_size bytes, contents ignored and
 * overwritten) holds the per-segment carries when the sequence is split
 * across thread blocks; it may be NULL when the size is 0.  The workspace
 * must not be shared by calls that may overlap on the GPU. */
ssm_status_t ssm_scan_fwd(const ssm_scan_args_t* args, void* workspace, size_t workspace_bytes,
                          ssm_stream_t stream);

/* The selective scan with the block's convolution stage in front, fused
 * into the same kernel so that the stage's input is read from HBM once.
 * Page "从硬件感知到算法革命：Mamba如何重塑序列建模的计算效率", section 3 (a
 * local convolution over time before the selective SSM, kernel size 4;
 * SiLU as the block's activation).  `args` is that of ssm_scan_fwd except
 * that args->u holds the stage's input x; the scan then runs on
 *   u[b,d,t] = silu(bias_d + sum_{k<width} weight[d,k] x[b,d,t-(width-1)+k]),
 * which also feeds the skip term D*u.  Inputs before step 0 come from x_prev
 * (entry j is the input at step j-(width-1)), or are zero when it is NULL.
 *   width  : 1..4 taps (others: SSM_ERR_UNSUPPORTED);
 *   weight : (dim, width) fp32, required;  bias : (dim) fp32 or NULL;
 *   x_prev : (batch, dim, width-1) fp32, contiguous, or NULL.
 * Workspace: as for ssm_scan_fwd (ssm_scan_fwd_workspace_size of `args`).
 * Split-and-resume: pass the last width-1 inputs of the first part as x_prev
 * of the second (together with h0 = h_last). */
typedef struct {
  int64_t width;
  const float* weight;
  const float* bias;
  const float* x_prev;
} ssm_conv_args_t;

ssm_status_t ssm_scan_fwd_conv(const ssm_scan_args_t* args, const ssm_conv_args_t* conv,
                               void* workspace, size_t workspace_bytes, ssm_stream_t stream);

/* The selective scan over a packed variable-length batch: nseq sequences
 * laid end to end along seqlen in one batch row (args->batch must be 1),
 * sequence i covering steps [cu_seqlens[i], cu_seqlens[i+1]).  The state
 * restarts from zero at every sequence start, and h_last (if not NULL) is
 * (nseq, dim, dstate) fp32: the state after each sequence's last step.
 *   cu_seqlens : device int32 (nseq + 1), cu_seqlens[0] = 0, strictly
 *                increasing (every sequence non-empty), cu_seqlens[nseq] =
 *                seqlen; other contents give undefined results (no
 *                out-of-bounds access).
 * args->h0 must be NULL (SSM_ERR_UNSUPPORTED otherwise); the rest of `args`
 * as for ssm_scan_fwd.  Workspace: ssm_scan_fwd_workspace_size(args).
 * Page "Mamba状态空间模型的硬件感知推理优化" section 1 and page
 * "从硬件感知到算法革命" (dynamic batching): each sequence is an independent
 * recurrence; packing only shares the launch. */
ssm_status_t ssm_scan_fwd_varlen(const ssm_scan_args_t* args, const int32_t* cu_seqlens,
                                 int64_t nseq, void* workspace, size_t workspace_bytes,
                                 ssm_stream_t stream);

/* Gradients of the selective scan (reverse mode) for a loss whose gradient
 * with respect to y is dy (batch, dim, seqlen) fp32: the states are
 * recomputed (page "从硬件感知到算法革命" section 1, "recomputation") and the
 * adjoint lambda[t] = ds_t C[t] + exp(dt'_{t+1} A) lambda[t+1], ds_t = dy_t
 * silu(z_t), is swept backwards.  `args` as for ssm_scan_fwd (y and h_last
 * are not used), default contiguous layouts only, one B/C group
 * (SSM_ERR_UNSUPPORTED otherwise).  Every gradient is fp32, laid out like its
 * input: du, ddelta, dz (batch, dim, seqlen); dA (dim, dstate); dB, dC
 * (batch, dstate, seqlen); dD, ddelta_bias (dim); dh0 (batch, dim, dstate).
 * dA, dB and dC are required; the others may be NULL, and those whose input
 * is NULL are not written.  Workspace: ssm_scan_bwd_workspace_size bytes
 * (16-byte aligned) for the state checkpoints. */
typedef struct {
  float* du;
  float* ddelta;
  float* dz;
  float* dA;
  float* dB;
  float* dC;
  float* dD;
  float* ddelta_bias;
  float* dh0;
} ssm_scan_grads_t;

size_t ssm_scan_bwd_workspace_size(const ssm_scan_args_t* args);
ssm_status_t ssm_scan_bwd(const ssm_scan_args_t* args, const float* dy,
                          const ssm_scan_grads_t* grads, void* workspace, size_t workspace_bytes,
                          ssm_stream_t stream);

/* Bytes of the library's static device scratch used by ssm_scan_fwd_noalloc. */
#define SSM_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)

/* The selective scan for callers that cannot allocate device memory: code
 * running inside a host framework that owns every device buffer and forbids
 * allocation while it executes (an inference-engine plugin, for instance),
 * or code on a latency-critical path that cannot afford cudaMalloc's implicit
 * synchronisation.  The pages have no counterpart to this entry point: it is
 * a packaging of ssm_scan_fwd.
 *
 * Arguments, layouts and results are those of ssm_scan_fwd; the caller still
 * passes every input and output.  The scratch that ssm_scan_fwd takes as
 * `workspace` comes instead from one array of SSM_NOALLOC_SCRATCH_BYTES
 * (4 MiB) in the library's device memory, which every GPU that loads the
 * library holds until the process exits.  The call allocates nothing.
 *  - The first call on a device looks up that array's device address (once
 *    per device, with that device current); make the first call on each
 *    device before any stream capture.
 *  - A call that would need more scratch than the array holds returns
 *    SSM_ERR_WORKSPACE, and ssm_last_error_string() says how much it needed.
 *  - All calls share the one array and it keeps the last call's contents
 *    (every call overwrites the part it reads before reading it).  Calls that
 *    may overlap on the GPU (other streams, other host threads) race on it
 *    and must be serialised by the caller. */
ssm_status_t ssm_scan_fwd_noalloc(const ssm_scan_args_t* args, ssm_stream_t stream);

/* The selective scan on inputs and outputs in HOST memory, for callers whose
 * data live on the host.  The pages have no counterpart to this entry point:
 * it is a packaging of ssm_scan_fwd that hides the PCIe transfers behind one
 * another.  The batch is cut into slices of `slice_batch` sequences that move
 * through two slots of device staging: while slice s is scanned on `stream`,
 * slice s + 1 is copied in and slice s - 1 copied out, on two copy streams
 * that the library creates on the first call on each device and keeps.
 *
 * Arguments: those of ssm_scan_fwd, except that every pointer in `args` is a
 * HOST pointer and only the default contiguous layouts are accepted (every
 * stride 0; others return SSM_ERR_UNSUPPORTED).  Page-locked host memory
 * (cudaHostAlloc or cudaHostRegister) lets the copies overlap; pageable
 * memory gives the same results without the overlap.  slice_batch >= 1.
 * `staging`: device memory, 256-byte aligned, at least
 * ssm_scan_fwd_host_staging_size(args, slice_batch) bytes, contents ignored
 * (SSM_ERR_WORKSPACE if missing or smaller).
 * Ordering: the copies start after the work queued on `stream` before the
 * call, and `stream` waits for the last copy back, so y and h_last on the
 * host are complete once `stream` has finished; until then the host buffers
 * and the staging must not be touched.  The call only queues work.  Calls
 * that share a staging buffer must not overlap.  On an error return part of
 * the work may already be queued and the outputs are undefined. */
size_t ssm_scan_fwd_host_staging_size(const ssm_scan_args_t* args, int64_t slice_batch);
ssm_status_t ssm_scan_fwd_host(const ssm_scan_args_t* args, int64_t slice_batch, void* staging,
                               size_t staging_bytes, ssm_stream_t stream);

/* ------------------------------------------------------------------------
 * One decode step ("Mamba与选择性SSM", section 5.4): the scan above for a
 * single time step, with the state read and overwritten in place.
 *   u, delta, z, y : (batch, dim) contiguous, `dtype`;
 *   B, C           : (batch, dstate) contiguous, `dtype`;
 *   A              : (dim, dstate) fp32;  D, delta_bias : (dim) fp32 or NULL;
 *   state          : (batch, dim, dstate) fp32, read then written.
 * Applying it L times reproduces ssm_scan_fwd on the same L steps.
 * Sizes: 1 <= dstate <= 16.  Needs no workspace. */
typedef struct {
  int64_t batch, dim, dstate;
  ssm_dtype_t dtype;
  const void* u;
  const void* delta;
  const void* z;
  const void* B;
  const void* C;
  const float* A;
  const float* D;
  const float* delta_bias;
  int delta_softplus;
  float* state;
  void* y;
} ssm_step_args_t;

ssm_status_t ssm_scan_step(const ssm_step_args_t* args, ssm_stream_t stream);

/* ------------------------------------------------------------------------
 * Mamba-2 scalar-decay scan, chunked ("Mamba状态空间模型的硬件感知推理优化",
 * section 4; chunked hybrid scan, section 4 end and section 5).  Per batch
 * b and head h with state S (headdim x dstate):
 *   dt'  = softplus(delta[b,t,h] + delta_bias[h]),  a_t = exp(dt' A[h])
 *   S    = a_t S + dt' x[b,t,h,:]^T B[b,t,:]
 *   y[b,t,h,:] = (S C[b,t,:] + D[h] x[b,t,h,:]) * silu(z[b,t,h,:])
 * Layout (contiguous):
 *   x, z, y     : (batch, seqlen, nheads, headdim)   `dtype`
 *   delta       : (batch, seqlen, nheads)            `dtype`
 *   B, C        : (batch, seqlen, dstate)            `dtype` (shared by all heads)
 *   A, D, delta_bias : (nheads) fp32 (D, delta_bias may be NULL)
 *   h0, h_last  : (batch, nheads, headdim, dstate) fp32 or NULL.
 * chunk is the length of the intra-chunk quadratic block; the result does
 * not depend on it beyond rounding.
 * Implemented: dtype SSM_BF16, dstate 128, headdim 64, chunk 128 or 256
 * (others return SSM_ERR_UNSUPPORTED); x, B, C, z and y 16-byte aligned.
 * The intra-chunk contractions run on the tensor cores with bf16 operands
 * and fp32 accumulation; the state carried between chunks enters them in
 * bf16 and is accumulated in fp32.
 * Workspace (ssm_scan_fwd_chunked_workspace_size bytes, 256-byte aligned):
 * its first int is a status word, zeroed by the call and set non-zero by the
 * GPU if a bounded wait for a tensor-core result gave up (the outputs are
 * then invalid); read it after the stream has finished.  The rest holds the
 * chunk-local states, the log-decay of every chunk, the state entering
 * every chunk and the discretised step and cumulative log-decay of every
 * step.  Calls sharing a workspace must not overlap. */
typedef struct {
  int64_t batch, seqlen, nheads, headdim, dstate, chunk;
  ssm_dtype_t dtype;
  const void* x;
  const void* delta;
  const float* A;
  const void* B;
  const void* C;
  const float* D;
  const float* delta_bias;
  int delta_softplus;
  const void* z;
  const float* h0;
  void* y;
  float* h_last;
} ssm_ssd_args_t;

size_t ssm_scan_fwd_chunked_workspace_size(const ssm_ssd_args_t* args);
ssm_status_t ssm_scan_fwd_chunked(const ssm_ssd_args_t* args, void* workspace,
                                  size_t workspace_bytes, ssm_stream_t stream);

/* ------------------------------------------------------------------------ */
const char* ssm_status_string(ssm_status_t status);
int ssm_version(void); /* major * 10000 + minor * 100 + patch */

/* Description of the CUDA error behind the last SSM_ERR_CUDA returned on the
 * calling host thread ("" if none).  The string stays valid until the next
 * failing call on that thread. */
const char* ssm_last_error_string(void);

#ifdef __cplusplus
}
#endif
#endif /* SSMSCAN_H */
