/*
 * selective_scan.h -- C ABI of the B200 (sm_100a) selective scan (S6) forward library.
 *
 * The library computes, on one GPU and entirely in its own CUDA kernels, the selective state
 * space scan that the pages describe:
 *
 *   u_t      = u at the position of step t, or, with a    "Understanding Mamba from zero"
 *              convolution given (ss_launch_opts),          sec. 6.2 Step 2 (a small depthwise
 *              silu(conv_bias + sum_j conv_weight[j] *      causal 1D conv before the SSM,
 *                   u at step t - (width-1) + j)            width 4 in sec. 8); one conv per
 *              along this direction's scan order, zero      scanned sequence as in "Vision
 *              before step 0                                Mamba" sec. 2.2
 *   Delta_t  = softplus(delta_raw_t + delta_bias)          "Understanding Mamba from zero",
 *                                                           sec. 4.1 Algorithm 2 and sec. 6.2
 *                                                           Step 3 (tau_Delta(Parameter+s_Delta));
 *              delta_raw may arrive as int8 codes times     int8 Delta at inference, "S4 ->
 *              one scale per channel (SS_FLAG_DELTA_INT8)   Mamba" sec. 2.3
 *   Abar_t   = exp(Delta_t * A)                            same page, sec. 6.2 Step 4, eq. (4)
 *   Bbar_t u = Delta_t * B_t * u_t                         first-order form of eq. (4), as
 *                                                           "Mamba-UNet" sec. 4 writes it
 *   h_t      = Abar_t * h_{t-1} + Bbar_t u_t               eq. (2a); per (channel, state) a
 *                                                           scalar affine recurrence (sec. 5)
 *   y_t      = C_t . h_t + Dskip * u_t                     eq. (2b) with the D(t)x(t) skip of
 *                                                           "Mamba-UNet" sec. 4
 *   out      = (sum over directions of y) * silu(z)        Step 6 (phi = SiLU); the Vim block's
 *                                                           gate over y_fwd + y_bwd ("Vision
 *                                                           Mamba" sec. 2.2) and the SS2D merge of
 *                                                           four scan orders ("S4 -> Mamba" sec. 3)
 *
 * with A diagonal (one scalar per channel and state) and the state starting at zero (or at a
 * given initial state).
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library never frees or
 *     keeps them.  Tensors are dense, row-major (C-contiguous), with the shapes stated below.
 *   - The library allocates no memory.  Scratch, when a launch needs it, is the caller's
 *     `workspace` buffer, sized by selective_scan_workspace_size().
 *   - Work is enqueued on `stream` (a cudaStream_t, passed as void*; NULL = legacy default
 *     stream).  No call synchronises the stream except selective_scan_device_status().
 *   - Arguments are validated, tensor maps encoded and kernel attributes set before anything is
 *     launched: on any error status other than SS_ERR_CUDA nothing has been launched and no
 *     memory has been read or written.  SS_ERR_CUDA means the runtime failed; when it failed
 *     at a later launch of a call (the scan after the segment aggregates, or the direction
 *     merge), the earlier launches of that call have been enqueued.
 *   - `stream` must belong to the current device (SS_ERR_DEVICE otherwise): the library's
 *     device-side words are looked up on the current device.
 *   - Base pointers of u, delta, B, C, z, out and workspace must be 16-byte aligned, and
 *     dim * sizeof(io element) must be a multiple of 16 (SS_ERR_ALIGN otherwise).
 *   - N (dstate) is at most SS_MAX_DSTATE; at most SS_MAX_DIRS directions.
 *   - There is no CPU fallback: without a CUDA device every launch returns SS_ERR_CUDA.
 *   - The first selective_scan_fwd call on each device looks up the address of the library's
 *     device error word (cudaGetSymbolAddress, once); make that first call before capturing a
 *     stream into a CUDA graph.  The cached address (and the no-allocation scratch address of
 *     selective_scan_fwd_noalloc, and the streams and events of selective_scan_fwd_host)
 *     belongs to the device's current context: after a cudaDeviceReset the library must not be
 *     called again in the same process.
 */
#ifndef SELECTIVE_SCAN_H
#define SELECTIVE_SCAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SS_ABI_VERSION 5
#define SS_MAX_DSTATE 16
#define SS_MAX_DIRS 4
#define SS_MAX_CONV_WIDTH 4

typedef enum {
    SS_OK = 0,
    SS_ERR_NULL = 1,          /* a required pointer is NULL                                   */
    SS_ERR_SHAPE = 2,         /* a size is negative, inconsistent or too large                 */
    SS_ERR_DTYPE = 3,         /* io_dtype is not SS_F32 or SS_BF16                             */
    SS_ERR_ALIGN = 4,         /* a base pointer or the row pitch breaks the 16-byte rule       */
    SS_ERR_DIRMAP = 5,        /* bad direction code, count, or H*W != seqlen for column orders */
    SS_ERR_UNSUPPORTED = 6,   /* dstate > SS_MAX_DSTATE or an unsupported option               */
    SS_ERR_CUDA = 7,          /* the CUDA runtime reported an error at launch                  */
    SS_ERR_WORKSPACE = 8,     /* workspace NULL or smaller than selective_scan_workspace_size  */
    SS_ERR_DEVICE_TIMEOUT = 9, /* a kernel gave up a bounded wait (reported by device_status)  */
    SS_ERR_SCRATCH_LIMIT = 10, /* selective_scan_fwd_noalloc: the problem needs more scratch than
                                  SS_NOALLOC_SCRATCH_BYTES                                      */
    SS_ERR_DEVICE = 11         /* `stream` belongs to another device than the current one       */
} ss_status;

typedef enum { SS_F32 = 0, SS_BF16 = 1 } ss_dtype;

/* Scan orders over a sequence of length L that is an H x W image flattened row by row
 * (raster order, "Understanding Mamba from zero" sec. 7.2).  Step t of a scan visits the
 * spatial position p:
 *   SS_DIR_FWD      p = t
 *   SS_DIR_REV      p = L-1-t                          (Vim backward scan)
 *   SS_DIR_COL      p = (t mod H) * W + t div H         (column-major order, SS2D)
 *   SS_DIR_COL_REV  the column-major order walked from its end                             */
typedef enum { SS_DIR_FWD = 0, SS_DIR_REV = 1, SS_DIR_COL = 2, SS_DIR_COL_REV = 3 } ss_dir;

typedef struct {
    int64_t batch;    /* b  >= 0                                                   */
    int64_t seqlen;   /* L  >= 0; batch*L*4 < 2^31 and L*dim < 2^31               */
    int64_t dim;      /* D  >= 0 channels                                          */
    int64_t dstate;   /* N  in 1..SS_MAX_DSTATE                                    */
    int32_t io_dtype; /* ss_dtype of u, delta, z, B, C and out                     */
    int32_t reserved; /* must be 0                                                 */
} ss_shape;

typedef struct {
    int32_t num_dirs;            /* K in 1..SS_MAX_DIRS                                     */
    int32_t dir[SS_MAX_DIRS];    /* ss_dir of direction k (entries >= num_dirs ignored)     */
    int32_t H, W;                /* image size; H*W == seqlen when a column order is used  */
} ss_direction_map;

/* Options and optional inputs; NULL or all-zero means "defaults, choose automatically". */
typedef struct {
    int32_t segments;        /* split each sequence into this many segments (0 = auto)      */
    int32_t flags;           /* SS_FLAG_* bits                                               */
    void* scan_begin_event;  /* cudaEvent_t recorded on `stream` right before the scan
                                pipeline (the segment-aggregate launch, if any, and the scan
                                launch that writes out or the per-direction partials), or NULL */
    void* scan_end_event;    /* cudaEvent_t recorded right after that pipeline (before the
                                direction merge), or NULL                                    */
    const float* initial_state; /* [K, batch, D, N] fp32 device array: the state h before
                                   step 0 of each direction (eq. 2a's h_{-1}), or NULL for
                                   zero; read only; must not overlap last_state             */
    const float* conv_weight; /* [K, D, conv_width] fp32 device array: the causal depthwise
                                 convolution that direction k applies to u along its own scan
                                 order before the scan, followed by SiLU; tap conv_width-1
                                 multiplies the current step.  The convolved value replaces u
                                 in both Bbar*u and the D skip.  NULL: no convolution       */
    const float* conv_bias;  /* [K, D] fp32 device array, or NULL for zero (needs
                                conv_weight)                                                 */
    int32_t conv_width;      /* taps, 1..SS_MAX_CONV_WIDTH with conv_weight; 0 without      */
    int32_t reserved;        /* must be 0                                                    */
    const float* delta_scale; /* [D] fp32 device array with SS_FLAG_DELTA_INT8 (delta_raw =
                                 code * delta_scale[d]); NULL otherwise                      */
} ss_launch_opts;

#define SS_FLAG_GENERIC_A 1 /* never use the exp-power shortcut for A[d,n] = (n+1)*A[d,0]   */
#define SS_FLAG_ZOH_EXACT 2 /* Bbar = (exp(Delta*A) - 1) / A * B, eq. (4) exactly (A != 0;
                               Delta*B where A == 0), instead of the first-order Delta*B;
                               computed with the precise arithmetic for any io type        */
#define SS_FLAG_U_PER_DIRECTION 16 /* u is [K, batch, L, D]: direction k scans its own input
                                      u[k] (spatial order), in the convolution too; z stays
                                      [batch, L, D].  Sigma's cross-modal scan (CroMB, "S4 ->
                                      Mamba" sec. 4.1) is two forward directions over the two
                                      modalities' inputs with the C tensors stacked in swapped
                                      order, so that each modality reads the other's C      */
#define SS_FLAG_DELTA_INT8 32 /* delta holds int8 codes [K, batch, L, D] (one byte each); the
                                 raw value is code * delta_scale[d] (ss_launch_opts).  Needs
                                 io_dtype SS_BF16 and dim a multiple of 16 (the code rows are
                                 dim bytes; SS_ERR_ALIGN otherwise); the base pointer follows
                                 the 16-byte rule                                        */
#define SS_FLAG_PARAMS_PER_DIRECTION 64 /* A is [K, D, N], Dskip and delta_bias [K, D]:
                                           direction k uses its own parameters (VMamba's
                                           cross-scan and Vim's two directions are separate
                                           S6 modules); delta_scale stays [D]               */
#define SS_FLAG_TEST_WAIT_TIMEOUT 8 /* test hook for failure detection: every CTA waits (20 ms
                                       at most) on a barrier that nothing completes, gives up,
                                       records SS_ERR_DEVICE_TIMEOUT for
                                       selective_scan_device_status and returns without
                                       touching its outputs                                 */

/* Bytes of workspace that selective_scan_fwd needs for this problem and these options
 * (0 when it needs none).  Writes *bytes; validates shape, direction map and options the same
 * way as selective_scan_fwd.  Host-only; touches no device. */
ss_status selective_scan_workspace_size(const ss_shape* shape, const ss_direction_map* dmap,
                                        const ss_launch_opts* opts, size_t* bytes);

/*
 * The selective scan forward (see the top of this file for what it computes).
 *
 *   shape       problem sizes and io dtype (host pointer)
 *   u           [batch, L, D]      io dtype, spatial order ([K, batch, L, D] with
 *                                  SS_FLAG_U_PER_DIRECTION)
 *   delta       [K, batch, L, D]   io dtype (int8 codes with SS_FLAG_DELTA_INT8), raw Delta of
 *                                  direction k in its scan order
 *   A           [D, N]             fp32, shared by all directions ([K, D, N] with
 *                                  SS_FLAG_PARAMS_PER_DIRECTION)
 *   B, C        [K, batch, L, N]   io dtype, scan order of direction k
 *   Dskip       [D] fp32 ([K, D] with SS_FLAG_PARAMS_PER_DIRECTION), or NULL for zero
 *   z           [batch, L, D]      io dtype, spatial order, or NULL for no gate
 *   delta_bias  [D] fp32 ([K, D] with SS_FLAG_PARAMS_PER_DIRECTION), or NULL for zero
 *   softplus    nonzero: Delta = softplus(delta + bias); zero: Delta = delta + bias
 *   dmap        direction map (host pointer), or NULL for a single forward scan
 *   out         [batch, L, D]      io dtype, spatial order; every element written once
 *   last_state  [K, batch, D, N]   fp32 state h after each direction's last step, or NULL
 *   workspace   device scratch of at least selective_scan_workspace_size() bytes (may be
 *               NULL when that size is 0); its contents on entry do not matter
 *   stream      cudaStream_t to enqueue on
 *   opts        launch options (host pointer) or NULL
 *
 * Each direction is a full S6 scan with its own Dskip*u term, so with K directions the skip
 * contributes K*Dskip*u.  Inputs must not overlap out, last_state or workspace.  Returns SS_OK
 * once the kernels are enqueued.
 */
ss_status selective_scan_fwd(const ss_shape* shape, const void* u, const void* delta,
                             const float* A, const void* B, const void* C, const float* Dskip,
                             const void* z, const float* delta_bias, int32_t softplus,
                             const ss_direction_map* dmap, void* out, float* last_state,
                             void* workspace, size_t workspace_bytes, void* stream,
                             const ss_launch_opts* opts);

/* Spatial position visited at step t of direction k of dmap (NULL = forward) for sequence
 * length L, or -1 if the map or t is invalid.  Host-side entry to the same index function the
 * kernels use, so that tests can compare it with an independent implementation. */
int64_t ss_direction_position(const ss_direction_map* dmap, int32_t k, int64_t L, int64_t t);

/* Synchronises `stream`, then reports SS_ERR_DEVICE_TIMEOUT if any kernel of this library on
 * the current device gave up a bounded wait since the last call with clear != 0 (SS_OK
 * otherwise, SS_ERR_CUDA if the runtime failed).  With clear != 0 the flag is reset. */
ss_status selective_scan_device_status(void* stream, int32_t clear);

/* Bytes of the fixed scratch array that selective_scan_fwd_noalloc uses (16 MiB). */
#define SS_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * selective_scan_fwd_noalloc -- the same scan as selective_scan_fwd, for callers that cannot
 * allocate device memory.  (The pages have no counterpart to this entry point; it exists for
 * deployments, not for the method.)
 *
 * Who needs it: callers whose device memory is fixed when they start -- a plugin inside a host
 * application that owns the allocator, an inference server that sizes one arena up front, or a
 * latency-critical loop that must not call cudaMalloc (which can synchronise the device) -- and
 * that therefore cannot provide the workspace selective_scan_fwd asks for.
 *
 * Arguments are those of selective_scan_fwd without `workspace` / `workspace_bytes`; the caller
 * still passes every input and output.  The scratch comes from one array of this library's
 * device memory of SS_NOALLOC_SCRATCH_BYTES bytes, which every GPU that loads the library holds
 * until the process exits.  The call allocates nothing (no cudaMalloc, no cudaFree, no
 * allocating library routine).
 *   - A problem whose selective_scan_workspace_size() exceeds SS_NOALLOC_SCRATCH_BYTES is
 *     rejected with SS_ERR_SCRATCH_LIMIT before anything runs (at the default options: m130
 *     and the 131072-step sequence fit; the Vim and SS2D workloads, whose per-direction
 *     outputs need far more, do not).
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress,
 *     with that device current); make that first call before any stream capture.
 *   - All calls share the one array, which keeps the last call's contents.  Nothing in it has to
 *     start at zero: every value a call reads from it was written earlier by the same call.
 *     Calls whose work overlaps on the GPU (other streams, other host threads) race on the
 *     array; order them, for example on one stream.
 */
ss_status selective_scan_fwd_noalloc(const ss_shape* shape, const void* u, const void* delta,
                                     const float* A, const void* B, const void* C,
                                     const float* Dskip, const void* z, const float* delta_bias,
                                     int32_t softplus, const ss_direction_map* dmap, void* out,
                                     float* last_state, void* stream, const ss_launch_opts* opts);

/* Pieces at most that selective_scan_fwd_host cuts a call into. */
#define SS_HOST_MAX_PIECES 64

/* Bytes of device workspace selective_scan_fwd_host needs for this problem, these options and
 * this number of pieces (0 when the problem is empty): two staging slots of the largest piece
 * (its u, delta, B, C, z, out, final state and, with an initial state, a copy of its slice)
 * and the workspace of that piece's scan.  Validates like selective_scan_workspace_size;
 * SS_ERR_UNSUPPORTED for pieces outside 1..SS_HOST_MAX_PIECES.  Host-only. */
ss_status selective_scan_host_workspace_size(const ss_shape* shape, const ss_direction_map* dmap,
                                             const ss_launch_opts* opts, int32_t pieces,
                                             size_t* bytes);

/*
 * selective_scan_fwd_host -- the scan of selective_scan_fwd for activations held in HOST
 * memory, with the results written back to host memory: one call from host buffers to host
 * buffers, as a serving process that receives requests on the host makes it.
 *
 *   u, delta, B, C, z     HOST pointers, shapes and dtypes of selective_scan_fwd (z may be NULL);
 *                         page-locked memory (cudaHostAlloc / cudaHostRegister) lets the copies
 *                         run asynchronously; pageable memory works, but each copy then blocks
 *                         the calling thread
 *   out, last_state       HOST pointers (last_state may be NULL)
 *   A, Dskip, delta_bias  DEVICE pointers: the parameters stay resident on the GPU, as do
 *                         every device pointer of `opts` (initial_state, conv_weight,
 *                         conv_bias, delta_scale)
 *   workspace             DEVICE memory of selective_scan_host_workspace_size() bytes, 256-byte
 *                         aligned; its contents on entry do not matter
 *   pieces                1..SS_HOST_MAX_PIECES: the call is cut into this many pieces (groups
 *                         of batch rows; for one forward direction without convolution and with
 *                         fewer batch rows than pieces, stretches of each row's sequence of whole
 *                         16-step tiles, each continuing from the previous one's final state)
 *   stream                the caller's stream (of the current device)
 *
 * The call enqueues, on three streams of the library (created on the first call on a device and
 * kept until exit), the host->device copies of each piece (one cudaMemcpyAsync per contiguous
 * block), its scan (one selective_scan_fwd call on the piece) and the device->host copies of its
 * results, pipelined so that the copies in of piece i, the scan of piece i-1 and the copies out
 * of piece i-2 overlap.  All of it is ordered after the work already enqueued on `stream`, and
 * `stream` continues only after all of it: synchronise `stream` before reading out and
 * last_state.  Calls on one device are serialised on the library's streams; calls from several
 * host threads are safe.  Errors as selective_scan_fwd; SS_ERR_CUDA or a scan error from a later
 * piece leaves the earlier pieces enqueued.  The pages have no counterpart to this entry point:
 * it moves data; every step of the scan is selective_scan_fwd's.
 */
ss_status selective_scan_fwd_host(const ss_shape* shape, const void* u, const void* delta,
                                  const float* A, const void* B, const void* C, const float* Dskip,
                                  const void* z, const float* delta_bias, int32_t softplus,
                                  const ss_direction_map* dmap, void* out, float* last_state,
                                  void* workspace, size_t workspace_bytes, int32_t pieces,
                                  void* stream, const ss_launch_opts* opts);

/* Human-readable name of a status code (static storage). */
const char* ss_status_str(ss_status status);

/* SS_ABI_VERSION of the built library. */
int32_t ss_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SELECTIVE_SCAN_H */
