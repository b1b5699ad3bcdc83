/*
 * gspn.h -- C ABI of the B200 (sm_100a) Prop2D library, libgspn.so.
 *
 * Prop2D is the four-direction line-scan spatial propagation of GSPN, run in
 * the compressed latent channel space of C-GSPN ("Scaling Parallel Sequence
 * Models to Foundation-Scale Vision Encoders": Sec. 3 "Line-scan recurrence",
 * Sec. 5.1 "Latent-space 2D propagation" and "Fused CUDA normalization";
 * papernotes.org summary, "背景算子" paragraph and the operator
 * y_c = Prop2D(x_c; u, lambda, w)).  For every batch b, latent channel c and
 * enabled direction d, the grid is swept one line at a time and every
 * position q of line l is updated in parallel from three neighbours of the
 * previous line:
 *
 *     h_l(q) = sum_{k=0..2} w_l(q,k) h_{l-1}(q+k-1) + lambda_l(q) x_l(q),  h_{-1} = 0
 *     y      = sum_d u_d * h_d
 *
 * with row-stochastic weights made from logits by sigmoid, a sum over the
 * on-grid neighbours, a clamp of that sum at 1e-6 and a divide (Sec. 5.1
 * "Fused CUDA normalization"; papernotes.org normalisation formula).  Slot k
 * names the absolute orthogonal offset k-1 (-1 = left for row lines, up for
 * column lines); off-grid slots carry no weight.  With per-channel logits
 * the normalisation is fused into the scan and the weights are never
 * written anywhere.  In the compact mode (share_w = 1, one logit field shared
 * by all channels), gspn_prop2d_fwd_ws normalises each shared field once
 * into a caller-provided workspace and every channel's scan reads it.
 *
 * Layouts (element offsets, contiguous, row-major):
 *   x      [B][Cc][H][W]
 *   lambda [B][4][Cc][H][W]
 *   u      [B][4][Cc][H][W]
 *   wlogit [B][4][Cw][3][H][W]      Cw = share_w ? 1 : Cc
 *   out    [B][Cc][H][W]
 * Direction slots: 0 top->bottom, 1 bottom->top, 2 left->right,
 * 3 right->left.  All four slots are always present in lambda, u and wlogit;
 * slots not enabled by `dirs` are never read.
 *
 * Dtypes: inputs and output share one dtype (fp32 or bf16); the recurrence
 * state, the weight arithmetic and the direction sum are fp32 (the bf16
 * compact mode's workspace stores its normalised weights as fp16).
 *
 * Ownership: the caller owns every buffer, the workspace included.  The
 * library allocates no memory when it is called and keeps no state between
 * calls, except the scratch array that gspn_prop2d_fwd_noalloc uses in place
 * of a caller workspace (a static device array, described there).
 *
 * Errors: every entry point returns a gspn_status and never aborts or traps.
 * Argument errors are detected on the host before anything is launched;
 * a launch failure is reported as GSPN_ERR_CUDA (cudaGetLastError).
 */
#ifndef GSPN_H_
#define GSPN_H_

#include <stddef.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GSPN_F32 = 0,   /* float32 inputs and output */
    GSPN_BF16 = 1   /* bfloat16 inputs and output (fp32 state) */
} gspn_dtype;

typedef enum {
    GSPN_OK = 0,
    GSPN_ERR_NULL = 1,     /* a required pointer is NULL */
    GSPN_ERR_SHAPE = 2,    /* B, Cc, H or W negative, or a size the library cannot index */
    GSPN_ERR_DIRS = 3,     /* dirs outside 1..15, or share_w not 0/1 */
    GSPN_ERR_DTYPE = 4,    /* unknown gspn_dtype */
    GSPN_ERR_ALIGN = 5,    /* a device pointer is not 16-byte aligned */
    GSPN_ERR_CUDA = 6,     /* the CUDA runtime reported an error */
    GSPN_ERR_DEVICE = 7,   /* the current device is not sm_100 (B200) */
    GSPN_ERR_WORKSPACE = 8, /* workspace smaller than gspn_prop2d_workspace_bytes */
    GSPN_ERR_NOALLOC_LIMIT = 9, /* gspn_prop2d_fwd_noalloc: the sizes need more than
                                   GSPN_NOALLOC_WORKSPACE_BYTES of scratch */
    GSPN_ERR_SHARING = 10, /* gspn_prop2d_fwd_ex: gate_dirs not 1 or 4, or w_groups not a
                              divisor of Cc */
    GSPN_ERR_ALGO = 11     /* gspn_prop2d_fwd_algo: unknown algorithm, or one that cannot
                              run these sizes */
} gspn_status;

/* Kernel choice of gspn_prop2d_fwd_algo.  Every algorithm computes the same
 * Prop2D; they differ in how the work is spread over the GPU. */
typedef enum {
    GSPN_ALGO_AUTO = 0,       /* the library's choice, the one every other entry point makes */
    GSPN_ALGO_DIRECTION = 1,  /* one CTA per plane, one warp per direction (lines <= 256;
                                 bf16 rows of even width) */
    GSPN_ALGO_SWEEP_PAIR = 2, /* both sweeps of an orientation in the two halves of a warp
                                 (lines 2..128; bf16 rows of even width) */
    GSPN_ALGO_SPLIT = 3,      /* one cluster of four CTAs per plane, one CTA per direction,
                                 planes staged whole in shared memory (lines 2..128; the six
                                 planes a direction reads must fit one CTA; bf16 needs H*W even) */
    GSPN_ALGO_GENERIC = 4     /* the general kernel (lines <= 4096) */
} gspn_algo;

enum {
    GSPN_DIR_TB = 1,    /* top -> bottom: rows i = 0..H-1, previous row i-1 */
    GSPN_DIR_BT = 2,    /* bottom -> top: rows i = H-1..0, previous row i+1 */
    GSPN_DIR_LR = 4,    /* left -> right: columns j = 0..W-1, previous column j-1 */
    GSPN_DIR_RL = 8,    /* right -> left: columns j = W-1..0, previous column j+1 */
    GSPN_DIR_ALL = 15
};

/*
 * gspn_prop2d_fwd -- y = Prop2D(x; u, lambda, w), forward.
 *
 * x, lambda, wlogit, u : device pointers, layouts above, dtype `dtype`,
 *                        16-byte aligned.  Read only.
 * B, Cc, H, W          : sizes, >= 0.  Any size is zero -> nothing to do, GSPN_OK.
 * dirs                 : bitmask of GSPN_DIR_*, 1..15.
 * share_w              : 0 -> one logit field per channel;
 *                        1 -> one logit field per (batch, direction), used by
 *                             every channel (the compact multi-channel mode of
 *                             Sec. 4.2 "Channel-shared weights").
 * dtype                : GSPN_F32 or GSPN_BF16.
 * out                  : device pointer [B][Cc][H][W], dtype `dtype`, 16-byte
 *                        aligned; fully overwritten.  Must not alias an input.
 * stream               : CUDA stream; the call is asynchronous on it and does
 *                        not synchronise.
 *
 * Returns GSPN_OK or the first error found; on an argument error nothing is
 * launched and `out` is untouched.
 */
gspn_status gspn_prop2d_fwd(const void *x, const void *lambda, const void *wlogit,
                            const void *u, int B, int Cc, int H, int W, int dirs,
                            int share_w, gspn_dtype dtype, void *out,
                            cudaStream_t stream);

/*
 * gspn_prop2d_fwd_ex -- gspn_prop2d_fwd with the gates and the logits shared
 * more widely (Sec. 4.2 "Channel-shared weights and the attention view";
 * Sec. 6.2 "Image classification", which shares w_i across channels in all
 * modules).
 *
 * gate_dirs : 4 -> lambda and u hold one plane per direction, [B][4][Cc][H][W]
 *                  (as gspn_prop2d_fwd);
 *             1 -> one lambda plane and one u plane serve all four
 *                  directions: lambda, u are [B][1][Cc][H][W].
 * w_groups  : G, a divisor of Cc: wlogit is [B][4][G][3][H][W] and channel c
 *             uses logit field c / (Cc / G).  G = Cc is gspn_prop2d_fwd's
 *             share_w = 0, G = 1 its share_w = 1.
 * Other arguments as gspn_prop2d_fwd.  Returns GSPN_ERR_SHARING for a
 * gate_dirs other than 1 or 4 or a w_groups that does not divide Cc (w_groups
 * < 1 included), before anything is launched.
 */
gspn_status gspn_prop2d_fwd_ex(const void *x, const void *lambda, const void *wlogit,
                               const void *u, int B, int Cc, int H, int W, int dirs,
                               int gate_dirs, int w_groups, gspn_dtype dtype, void *out,
                               cudaStream_t stream);

/*
 * gspn_prop2d_fwd_algo -- gspn_prop2d_fwd_ex with the kernel named by `algo`
 * instead of the library's choice (for reproducible benchmarks, and for tests
 * that must reach one kernel).  GSPN_ALGO_AUTO is gspn_prop2d_fwd_ex.
 * Returns GSPN_ERR_ALGO, before anything is launched, for an unknown `algo`
 * or one whose limits (above) the sizes exceed; otherwise arguments and
 * errors as gspn_prop2d_fwd_ex.
 */
gspn_status gspn_prop2d_fwd_algo(const void *x, const void *lambda, const void *wlogit,
                                 const void *u, int B, int Cc, int H, int W, int dirs,
                                 int gate_dirs, int w_groups, gspn_dtype dtype, gspn_algo algo,
                                 void *out, cudaStream_t stream);

/*
 * gspn_prop2d_workspace_bytes -- size of the workspace gspn_prop2d_fwd_ws
 * needs for these arguments: B*4*3*H*W elements (fp32 for GSPN_F32, fp16 for
 * GSPN_BF16) when share_w = 1, else 0.  Returns 0 for invalid arguments.
 */
size_t gspn_prop2d_workspace_bytes(int B, int Cc, int H, int W, int dirs, int share_w,
                                   gspn_dtype dtype);

/*
 * gspn_prop2d_fwd_ws -- gspn_prop2d_fwd with a workspace for the compact mode
 * (Sec. 4.2 "Channel-shared weights": one weight field per position, shared
 * across channels).
 *
 * With share_w = 1, a first kernel normalises the shared logits of every
 * (batch, enabled direction, position) once into `workspace`, layout
 * [B][4][3][H][W]: slot 0 = w0, slot 1 = w0 + w1 + w2 (1 unless the clamp
 * binds), slot 2 = w2, in fp32 (GSPN_F32) or fp16 (GSPN_BF16); the scans of
 * all Cc channels then read those weights instead of normalising per
 * channel.  fp16 weights carry a relative rounding error of at most 2^-11
 * each; w1 is formed as the difference, so a position's weights keep their
 * exact sum.  With share_w = 0 the workspace is not used (may be NULL) and
 * the call equals gspn_prop2d_fwd.
 *
 * workspace      : device pointer, 16-byte aligned, at least
 *                  gspn_prop2d_workspace_bytes(...) bytes; overwritten; must
 *                  not alias any other argument.  Stream-ordered: it may be
 *                  reused by the next call on the same stream.
 * workspace_size : its size in bytes.
 * Other arguments and errors as gspn_prop2d_fwd, plus GSPN_ERR_NULL for a
 * NULL workspace and GSPN_ERR_WORKSPACE for one that is too small (share_w = 1).
 * gspn_last_launch_info then counts two launches.
 */
gspn_status gspn_prop2d_fwd_ws(const void *x, const void *lambda, const void *wlogit,
                               const void *u, int B, int Cc, int H, int W, int dirs,
                               int share_w, gspn_dtype dtype, void *out, void *workspace,
                               size_t workspace_size, cudaStream_t stream);

/*
 * gspn_prop2d_fwd_host -- the same operation on HOST buffers.
 *
 * Copies the four host inputs (h_x, h_lambda, h_wlogit, h_u) into the
 * caller's device buffers (d_x, d_lambda, d_wlogit, d_u), runs
 * gspn_prop2d_fwd into d_out and copies d_out back into h_out, in up to four
 * batch chunks whose uploads, kernels and downloads overlap (chunk k+1 is
 * uploaded while chunk k runs and chunk k-1 comes back).  A chunk starts at
 * a batch index whose byte offset is a multiple of 16 in every tensor, so
 * that the kernels' alignment rule holds for every chunk (one chunk when no
 * such split exists).  The chunks run on
 * three streams and a few events that the library creates once per device
 * (no device memory); they start after the work already queued on `stream`.
 * Returns after everything has finished, so h_out is valid on return.
 * Calls from several host threads on one device are serialised.  Host
 * buffers should be pinned (page-locked) for the copies to run at full
 * speed and to overlap; pageable memory works but is slower.  Device
 * buffers follow the rules of gspn_prop2d_fwd.  Nothing is allocated.
 */
gspn_status gspn_prop2d_fwd_host(const void *h_x, const void *h_lambda, const void *h_wlogit,
                                 const void *h_u, void *h_out,
                                 void *d_x, void *d_lambda, void *d_wlogit, void *d_u,
                                 void *d_out,
                                 int B, int Cc, int H, int W, int dirs, int share_w,
                                 gspn_dtype dtype, cudaStream_t stream);

/*
 * Size in bytes of the scratch array built into the library for
 * gspn_prop2d_fwd_noalloc (8 MiB).
 */
#define GSPN_NOALLOC_WORKSPACE_BYTES (8u * 1024u * 1024u)

/*
 * gspn_prop2d_fwd_noalloc -- gspn_prop2d_fwd_ws for callers that cannot
 * allocate device memory.  The paper has no counterpart: this is a
 * deployment variant of the compact mode.
 *
 * Some callers run where device allocation is not allowed: inside a host
 * framework that owns all device memory and forbids allocating while it
 * executes (an inference engine's per-request callback, a real-time loop
 * with a fixed memory budget), where cudaMalloc would implicitly synchronise
 * the device or escape the framework's accounting.  They still own x,
 * lambda, wlogit, u and out, but cannot hand over a workspace.  This entry
 * point takes the same arguments as gspn_prop2d_fwd and, with share_w = 1,
 * normalises the shared weights into a scratch array compiled into the
 * library instead of a caller workspace: a file-scope __device__ array of
 * GSPN_NOALLOC_WORKSPACE_BYTES bytes that every GPU which loads the library
 * holds until the process exits.  It calls no cudaMalloc, cudaFree or other
 * allocating routine.
 *
 * Limits and behaviour:
 *   - share_w = 1 needs gspn_prop2d_workspace_bytes(...) bytes of scratch;
 *     more than GSPN_NOALLOC_WORKSPACE_BYTES returns GSPN_ERR_NOALLOC_LIMIT
 *     and launches nothing (8 MiB holds, for example, B = 8 batches of
 *     148 x 148 bf16 grids).  With share_w = 0 no scratch is used and the
 *     call equals gspn_prop2d_fwd.
 *   - The first call on a device (with that device current) looks up the
 *     array's device address once (cudaGetSymbolAddress) and caches it; make
 *     that first call before any stream capture.
 *   - Every call on a device shares the one array, and the array keeps the
 *     last call's contents.  Each call overwrites every weight it later
 *     reads, so nothing has to start at zero.  Calls whose kernels overlap on
 *     the GPU (on different streams, or from several host threads) race on
 *     the array: order them on one stream or serialise them.
 * Other arguments, layouts and errors as gspn_prop2d_fwd_ws.
 */
gspn_status gspn_prop2d_fwd_noalloc(const void *x, const void *lambda, const void *wlogit,
                                    const void *u, int B, int Cc, int H, int W, int dirs,
                                    int share_w, gspn_dtype dtype, void *out,
                                    cudaStream_t stream);

/*
 * gspn_prop2d_bwd -- gradients of y = Prop2D(x; u, lambda, w) (the pages
 * report the backward kernel's speed-ups, Sec. 6.1 "Scaling with input size,
 * batch, and channels", Fig. 8; the gradients are the chain rule of the
 * forward recurrence and normalisation).
 *
 * Given gy = dL/dy ([B][Cc][H][W], dtype `dtype`), writes fp32 gradients in
 * the input layouts:
 *   dx       [B][Cc][H][W]          sum over the enabled directions
 *   dlambda  [B][4][Cc][H][W]       0 in slots of directions not enabled
 *   dwlogit  [B][4][Cw][3][H][W]    through sigmoid, local sum, clamp and
 *                                   divide; 0 in off-grid slots; with
 *                                   share_w = 1 summed over the channels
 *   du       [B][4][Cc][H][W]
 * The clamp of the local sum is differentiated on the branch the forward
 * takes (sum above 1e-6: the sum; else the constant 1e-6).
 *
 * x, lambda, wlogit, u, gy : device pointers, dtype `dtype`, read only.
 * dx, dlambda, dwlogit, du : device fp32 buffers; zeroed on `stream` by the
 *                            call and then written.
 * Lines (H, W) up to 256.  All pointers 16-byte aligned.  Asynchronous on
 * `stream`; one kernel launch after four cudaMemsetAsync.  Other arguments
 * and errors as gspn_prop2d_fwd.
 */
gspn_status gspn_prop2d_bwd(const void *x, const void *lambda, const void *wlogit,
                            const void *u, const void *gy, int B, int Cc, int H, int W, int dirs,
                            int share_w, gspn_dtype dtype, float *dx, float *dlambda,
                            float *dwlogit, float *du, cudaStream_t stream);

/*
 * gspn_prop2d_bwd_ex -- gspn_prop2d_bwd for the sharing variants of
 * gspn_prop2d_fwd_ex (gate_dirs, w_groups as there).  A shared input's
 * gradient is the sum of the gradients of its uses:
 *   dlambda, du  [B][gate_dirs][Cc][H][W]  (gate_dirs = 1: summed over the
 *                                           enabled directions)
 *   dwlogit      [B][4][G][3][H][W]        (summed over the Cc / G channels
 *                                           of each field)
 *   dx           [B][Cc][H][W]
 * Returns GSPN_ERR_SHARING for a gate_dirs other than 1 or 4 or a w_groups
 * that does not divide Cc, before anything runs.  Other arguments and errors
 * as gspn_prop2d_bwd; gate_dirs = 4, w_groups = Cc (or 1) is gspn_prop2d_bwd
 * with share_w = 0 (or 1).
 */
gspn_status gspn_prop2d_bwd_ex(const void *x, const void *lambda, const void *wlogit,
                               const void *u, const void *gy, int B, int Cc, int H, int W,
                               int dirs, int gate_dirs, int w_groups, gspn_dtype dtype, float *dx,
                               float *dlambda, float *dwlogit, float *du, cudaStream_t stream);

/* Human-readable name of a status code (static string, never NULL). */
const char *gspn_status_str(gspn_status status);

/*
 * gspn_last_launch_info -- describes the kernel launches made by the last
 * successful gspn_prop2d_fwd on the calling host thread: number of kernel
 * launches, grid size, threads per block and dynamic shared memory bytes of
 * the main kernel, and a short name of the path taken.  For diagnostics and
 * benchmarks; any pointer may be NULL.
 */
void gspn_last_launch_info(int *launches, int *grid, int *block, int *smem_bytes,
                           const char **path);

#ifdef __cplusplus
}
#endif

#endif /* GSPN_H_ */
