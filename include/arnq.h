/*
 * arnq.h -- C ABI of a B200 (sm_100a) library for the fused residual add +
 * RMSNorm + per-row symmetric dynamic quantization operator.
 *
 * The operator is the one defined on the CANN page
 * "aclnnAddRmsNormDynamicQuantV2", section "Formula":
 *
 *     x        = x1 + x2                                (written out as xOut)
 *     Rms(x)   = sqrt( (1/n) * sum_i x_i^2 + epsilon )  (over the last dim, n)
 *     y        = x / Rms(x) * gamma + beta
 *     input_k  = y * smoothScale_k   if smoothScale_k is given, else y
 *     scale_k  = row_max(|input_k|) / Q                 (Q = 127 INT8, 7 INT4)
 *     y_k      = round(input_k / scale_k)
 *
 * with one or two quantized outputs selected by outputMask and the smooth
 * scales as that page states (see arnq_selected_outputs), and the argument
 * rules of its "Constraints" section.  The no-add form is the page
 * "aclnnRmsNormDynamicQuant", formula section.
 *
 * Numerical conventions (the pages leave these open; the library fixes them):
 *   - x1 + x2 is a binary32 add rounded once more, to nearest even, to the
 *     input dtype; that rounded x is written as xOut AND is the x that is
 *     normalised.
 *   - y and input_k are kept in binary32 and never rounded to 16 bits.
 *   - scale_k is a binary32 value; the codes are the quotient input_k/scale_k
 *     rounded half-to-even and clamped to [-Q, Q].  A row whose scale is 0
 *     (all inputs 0) gets scale 0 and all codes 0.
 *   - INT4 codes are two's-complement nibbles packed two per byte, the even
 *     column in the low nibble; an INT4 row of n codes occupies n/2 bytes
 *     (or n/8 int32 words of eight codes: see arnq_qdtype).
 *   - Results are deterministic: the same inputs and the same plan give the
 *     same bits on every run ("Deterministic compute" in the Constraints
 *     section).  Sums are fixed-order trees; there are no float atomics.
 *
 * Layout: every tensor is dense row-major ("ND" in the Constraints section).
 *   x1, x2, xOut : [rows, n] of dtype (bf16 or fp16)
 *   gamma, beta, smooth1, smooth2 : [n] of dtype
 *   y1, y2 : [rows, n] int8, [rows, n/2] bytes of packed INT4, or
 *            [rows, n/8] int32 words of eight INT4 codes
 *   scale1, scale2 : [rows] binary32
 *
 * Ownership: the caller owns every buffer.  All tensor pointers are DEVICE
 * pointers on the current CUDA device.  The library allocates nothing, never
 * synchronizes, and launches only on the given stream (a cudaStream_t passed
 * as void *; NULL is the legacy default stream).  Outputs that are not
 * selected are never written and may be NULL.  xOut may be the same pointer
 * as x1 or x2 (in-place residual update); any other overlap between an
 * output and an input is undefined.
 *
 * Launches: one kernel per call, whether a row is handled by one CTA or by a
 * thread-block cluster.  It is launched as a programmatic dependent launch
 * (cudaLaunchAttributeProgrammaticStreamSerialization): its CTAs may become
 * resident while the preceding kernel on the stream finishes, but they read
 * and write no memory before that kernel has completed and its writes are
 * visible, so stream order holds as for a plain launch.
 *
 * Errors: every argument check happens on the host before anything is
 * launched; a failing call writes nothing and returns the status.  A launch
 * failure returns ARNQ_ERR_CUDA (cudaGetLastError() holds the CUDA error).
 * Kernels that wait on asynchronous copies do so with a time limit (1 s
 * unless a plan sets wait_limit_us); if a wait expires the kernel stops early
 * and records ARNQ_ERR_DEVICE_TIMEOUT in the workspace's status block (see
 * arnq_workspace_status).
 */
#ifndef ARNQ_H
#define ARNQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ARNQ_API __attribute__((visibility("default")))
#else
#define ARNQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum arnq_status {
  ARNQ_OK = 0,
  ARNQ_ERR_NULL_PTR = 1,        /* a required input, or a selected output, is NULL        */
  ARNQ_ERR_EMPTY = 2,           /* rows == 0 or n == 0: empty tensors are not supported    */
  ARNQ_ERR_SHAPE = 3,           /* n not a multiple of 2 (INT4) or 8 (INT4_INT32); n above
                                   ARNQ_MAX_N; negative sizes                              */
  ARNQ_ERR_DTYPE = 4,           /* unknown dtype or qdtype                                 */
  ARNQ_ERR_MASK = 5,            /* outputMask / smooth-scale combination the page forbids  */
  ARNQ_ERR_EPS = 6,             /* epsilon negative or not finite                          */
  ARNQ_ERR_ALIGN = 7,           /* a 16-bit tensor not 2-byte aligned, a scale (or an
                                   INT4_INT32 output) not 4-byte aligned                   */
  ARNQ_ERR_WORKSPACE = 8,       /* workspace NULL or smaller than arnq_workspace_size()    */
  ARNQ_ERR_CUDA = 9,            /* a CUDA call failed (launch, attribute, device query)    */
  ARNQ_ERR_PLAN = 10,           /* an explicit plan that cannot run this problem           */
  ARNQ_ERR_DEVICE_TIMEOUT = 11  /* reported through the workspace status block only        */
} arnq_status;

typedef enum arnq_dtype { ARNQ_BF16 = 0, ARNQ_FP16 = 1 } arnq_dtype;
/* Code types of y1 and y2 ("aclnnAddRmsNormDynamicQuantV2", Formula: y1Out is
 * INT8 or INT4; the page fixes no INT4 container):
 *   ARNQ_INT8        int8 [rows, n]
 *   ARNQ_INT4        bytes [rows, n/2], two codes a byte, even column in the
 *                    low nibble (n even)
 *   ARNQ_INT4_INT32  int32 [rows, n/8], eight codes a 32-bit word, column
 *                    8w + k of a row in bits 4k .. 4k+3 of its word w (n a
 *                    multiple of 8; y 4-byte aligned).  On a little-endian
 *                    device its bytes are those of ARNQ_INT4.
 * INT4 codes are two's-complement nibbles in [-7, 7]. */
typedef enum arnq_qdtype { ARNQ_INT8 = 0, ARNQ_INT4 = 1, ARNQ_INT4_INT32 = 2 } arnq_qdtype;

/* outputMask encoding: ARNQ_MASK_ABSENT means "outputMaskOptional not given";
 * otherwise bit 0 is outputMask[0] (y1) and bit 1 is outputMask[1] (y2). */
#define ARNQ_MASK_ABSENT (-1)
#define ARNQ_MASK_Y1 1
#define ARNQ_MASK_Y2 2

/* Largest supported row length n (elements). */
#define ARNQ_MAX_N 131072

/* Human-readable name of a status code (static storage; never NULL). */
ARNQ_API const char *arnq_status_string(arnq_status s);

/* Which outputs a call produces ("aclnnAddRmsNormDynamicQuantV2", Formula:
 * the valid / invalid cases of scale1Out, y1Out, scale2Out, y2Out) and
 * whether the combination is allowed (Constraints section):
 *   y1/scale1 are produced  iff  mask absent, or mask[0];
 *   y2/scale2 are produced  iff  mask[1], or (mask absent and both smooth
 *                                 scales given);
 *   ARNQ_ERR_MASK if the mask is given with smooth1 and !mask[0], or with
 *   smooth2 and !mask[1], or with both entries false; or if the mask is absent
 *   and smooth2 is given without smooth1.
 * y1_on / y2_on may be NULL.  Host only; touches no device. */
ARNQ_API arnq_status arnq_selected_outputs(int out_mask, int has_smooth1, int has_smooth2, int *y1_on,
                                  int *y2_on);

/* Workspace bytes arnq_run needs for this problem (first phase of the pages'
 * two-phase call, "aclnnAddRmsNormDynamicQuantV2GetWorkspaceSize"): 256 for
 * every valid problem.  The workspace holds the status block (bytes 0-15, see
 * arnq_workspace_status), which the kernels write only on error; the rest is
 * reserved.  The per-row bookkeeping of the exact scales stays in on-chip
 * shared memory.  The caller allocates it on the device (8-byte aligned) and
 * zero-fills its status block once; it may then be reused for any number of
 * calls on one stream (not by calls that overlap).  Validates the same
 * arguments as arnq_run (except pointers).  Host only. */
ARNQ_API arnq_status arnq_workspace_size(int64_t rows, int64_t n, arnq_dtype dt, arnq_qdtype qdt,
                                int out_mask, int has_smooth1, int has_smooth2, size_t *bytes);

/* The fused operator ("aclnnAddRmsNormDynamicQuantV2", Formula).
 *   x1, x2         [rows, n] dtype   required
 *   gamma          [n] dtype         required
 *   beta           [n] dtype         optional (NULL = no beta)
 *   smooth1/2      [n] dtype         optional (NULL = not given)
 *   eps            epsilon, finite and >= 0
 *   out_mask       ARNQ_MASK_ABSENT or ARNQ_MASK_Y1 | ARNQ_MASK_Y2 bits
 *   qdt            code type of y1 and y2
 *   y1, scale1     written iff selected (see arnq_selected_outputs)
 *   y2, scale2     written iff selected
 *   x_out          [rows, n] dtype, optional (NULL = not written)
 *   workspace      device buffer of at least arnq_workspace_size() bytes
 *   stream         cudaStream_t (as void *) to launch on
 * Returns ARNQ_OK once the work is enqueued; see the file header for errors. */
ARNQ_API arnq_status arnq_run(const void *x1, const void *x2, const void *gamma, const void *beta,
                     const void *smooth1, const void *smooth2, int64_t rows, int64_t n,
                     arnq_dtype dt, float eps, int out_mask, arnq_qdtype qdt, void *y1,
                     float *scale1, void *y2, float *scale2, void *x_out, void *workspace,
                     size_t workspace_bytes, void *stream);

/* The earlier interface "aclnnAddRmsNormDynamicQuant" (the V2 page: V2 adds
 * betaOptional and outputMaskOptional to it): arnq_run with beta = NULL and
 * the mask absent. */
ARNQ_API arnq_status arnq_run_v1(const void *x1, const void *x2, const void *gamma, const void *smooth1,
                        const void *smooth2, int64_t rows, int64_t n, arnq_dtype dt, float eps,
                        arnq_qdtype qdt, void *y1, float *scale1, void *y2, float *scale2,
                        void *x_out, void *workspace, size_t workspace_bytes, void *stream);

/* The no-add operator ("aclnnRmsNormDynamicQuant", formula section): x is
 * normalised as given, one optional smooth scale, one output.
 *   x [rows, n] dtype; gamma [n]; beta, smooth [n] optional;
 *   y [rows, n] int8 or [rows, n/2] packed INT4; scale [rows] binary32. */
ARNQ_API arnq_status arnq_rms_norm_dynamic_quant(const void *x, const void *gamma, const void *beta,
                                        const void *smooth, int64_t rows, int64_t n,
                                        arnq_dtype dt, float eps, arnq_qdtype qdt, void *y,
                                        float *scale, void *workspace, size_t workspace_bytes,
                                        void *stream);

/* Status block at the start of the workspace.  code is 0 (ARNQ_OK) until a
 * kernel records an error (ARNQ_ERR_DEVICE_TIMEOUT);
 * the library never clears it.  row is the first row the failing kernel did
 * not finish (-1 when no row applies).  Read it with a device-to-host copy
 * after synchronizing the stream; zero it to re-arm. */
typedef struct arnq_workspace_status {
  int32_t code;
  int32_t reserved;
  int64_t row;
} arnq_workspace_status;

/* ---- launch plans (tuning and testing) --------------------------------- */

typedef enum arnq_kernel {
  ARNQ_KERNEL_AUTO = 0,    /* let the library choose                                   */
  ARNQ_KERNEL_DIRECT = 1,  /* rows loaded straight into registers (any alignment)      */
  ARNQ_KERNEL_STAGED = 2   /* rows staged in shared memory by bulk async copies        */
} arnq_kernel;

/* How a call is launched.  Zero fields mean "choose".  Every plan computes
 * the same operator; plans may differ in the last bits of the scales and, at
 * rare rounding ties, by one in a code, because the fp32 reduction tree
 * follows the plan.  One plan always gives the same bits. */
typedef struct arnq_plan {
  int32_t kernel;        /* arnq_kernel                                        */
  int32_t cluster;       /* CTAs sharing one row: 1, 2, 4, 8 or 16             */
  int32_t threads;       /* threads per CTA (multiple of 32)                   */
  int32_t units;         /* units per thread: 1, 2, 4 (16-byte) or 1, 4, 8 (pairs) */
  int32_t stages;        /* staged kernel: rows in flight per CTA (1..8)        */
  int32_t ctas_per_sm;   /* resident CTAs per SM the grid is sized for         */
  int32_t grid;          /* CTAs launched (multiple of cluster); 0 = as many
                            clusters as cover the rows with equal row counts */
  int32_t vector;        /* output: 1 if 16-byte vector loads are used         */
  int32_t wait_limit_us; /* bounded device waits give up after this many us;
                            0 = 1 s                                          */
  int32_t test_hold_bytes; /* testing only (staged kernel): the first copy's
                            barrier of every CTA expects this many bytes more
                            than its copies bring, so that wait runs out and
                            the call records ARNQ_ERR_DEVICE_TIMEOUT; at most
                            65536; 0 in normal use                           */
  int32_t early_params;  /* 1: the kernel loads gamma, beta and the smooth
                            scales before it waits for the preceding work on
                            the stream (it is launched as a programmatic
                            dependent), so those loads overlap that work's
                            end.  Only correct when the preceding work does
                            not write them (weights that stay constant, as in
                            inference); 0 (the default): it waits first.     */
} arnq_plan;

/* Fills *plan with the plan arnq_run would use for these arguments (pointers
 * are only inspected for alignment).  Fields of *plan that are nonzero on
 * entry are kept as requested.  Queries the current device.  A requested grid
 * larger than the resident clusters runs in waves; one with more clusters
 * than rows leaves the extra clusters idle. */
ARNQ_API arnq_status arnq_make_plan(const void *x1, const void *x2, const void *gamma, const void *beta,
                           const void *smooth1, const void *smooth2, int64_t rows, int64_t n,
                           arnq_dtype dt, int out_mask, arnq_qdtype qdt, const void *y1,
                           const void *y2, const void *x_out, arnq_plan *plan);

/* arnq_run with an explicit plan (from arnq_make_plan, possibly edited).
 * ARNQ_ERR_PLAN if the plan cannot run this problem. */
ARNQ_API arnq_status arnq_run_planned(const void *x1, const void *x2, const void *gamma,
                             const void *beta, const void *smooth1, const void *smooth2,
                             int64_t rows, int64_t n, arnq_dtype dt, float eps, int out_mask,
                             arnq_qdtype qdt, void *y1, float *scale1, void *y2, float *scale2,
                             void *x_out, void *workspace, size_t workspace_bytes, void *stream,
                             const arnq_plan *plan);

/* ---- no-allocation variant ----------------------------------------------
 *
 * The paper has no counterpart: the pages' two-phase call always takes a
 * caller-allocated workspace.  Some callers cannot allocate device memory at
 * the point of the call: code running under a fixed memory budget, a caller
 * with no allocator at hand (a plain C host program that owns no CUDA
 * allocator, or one whose framework's caching allocator must not be bypassed),
 * or a caller that would otherwise have to allocate and free around every
 * call.  This entry point is arnq_run with the workspace replaced by a
 * file-scope device array inside the library, ARNQ_STATIC_SCRATCH_BYTES per
 * device, held by every GPU that loads the library until the process exits.
 * It allocates nothing: no cudaMalloc / cudaFree and no allocating library
 * routine.  Arguments and results are those of arnq_run; in addition
 *   - ARNQ_ERR_WORKSPACE if the problem needs more scratch than
 *     ARNQ_STATIC_SCRATCH_BYTES (arnq_workspace_size larger than the array;
 *     no valid problem does today: it needs 256 bytes);
 *   - ARNQ_ERR_CUDA if the array's device address cannot be obtained
 *     (cudaGetSymbolAddress fails).
 * Every call looks up the array's address for the current device (so a device
 * reset between calls does no harm) and clears the status block at its start
 * with an async memset on `stream` before the kernel.  The first call on a
 * device may load the library's device code: make it before any stream
 * capture.  The array is shared by every call on a device and keeps the last
 * call's contents: calls that overlap on the GPU (other streams, other host
 * threads) race on it; serialise them.  A device-side timeout status lands in
 * the array and is not readable from the host: use arnq_run with a workspace
 * where that status matters. */
#define ARNQ_STATIC_SCRATCH_BYTES 4096
ARNQ_API arnq_status arnq_run_static_scratch(const void *x1, const void *x2, const void *gamma,
                                    const void *beta, const void *smooth1, const void *smooth2,
                                    int64_t rows, int64_t n, arnq_dtype dt, float eps,
                                    int out_mask, arnq_qdtype qdt, void *y1, float *scale1,
                                    void *y2, float *scale2, void *x_out, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* ARNQ_H */
