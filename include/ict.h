/*
 * ict.h -- C ABI of libict.so: the integer-only (C,e) training hot path on B200 (sm_100a).
 *
 * Method: "Memory-Efficient Integer-Only Training of Deep Neural Networks" (Shalby,
 * Pittorino, Roveri).  Every training tensor is a pair (C,e): INT8 signed mantissas C
 * with an explicit power-of-two exponent e per tensor or per group (Abstract; Figure 1
 * caption).  Layers are built from integer primitives (Abstract: products, sums,
 * divide-by-constant, nonlinear functions, weight updates; Table 6 maps convolution and
 * linear layers onto the Product primitive).  The page prints neither the equations nor
 * a rounding rule; the readings this library implements are:
 *
 *   value(C, e)   = C * 2^e,  C in [-127, 127],  e an int8 in [-127, 127];
 *                   e = ICT_E_ZERO (-128) marks a group whose mantissas are all zero.
 *   need(x, r)    = the smallest exponent e at which RNE(x * 2^(r - e)) lies in
 *                   [-127, 127] (x an exact integer at exponent r; RNE = round half
 *                   to even).
 *   FIT(group)    = requantisation after every product: the group exponent is the
 *                   largest need() of its nonzero members (ICT_E_ZERO when all are
 *                   zero), raised to at least -127; each mantissa is
 *                   RNE(x * 2^(r - e)).
 *   ALIGN_MAX     = before a contraction, an operand whose exponent varies along the
 *                   contracted index is brought, per non-contracted index, to the
 *                   largest group exponent it meets (ICT_E_ZERO groups ignored), each
 *                   mantissa shifted right with RNE (reading of the Sum primitive,
 *                   Table 6 Eq. 6).
 *   Product       = exact integer dot product of aligned mantissas (int32, int64 where a
 *                   long contraction needs it), exponents added, then FIT into the
 *                   caller's output groups.  No int32 result is ever visible to the
 *                   caller.
 *
 * Conventions for every entry point:
 *   - Device pointers are allocated and owned by the caller.  The library allocates no
 *     memory; scratch space is the caller's `ws` buffer, sized by the matching
 *     *_workspace() query.  ws must be 256-byte aligned.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void *; NULL is
 *     the legacy default stream) and never synchronises, except
 *     ict_get_device_status().
 *   - Argument errors are returned before anything is launched.  Conditions found on the
 *     device (an exponent above 127, a bounded wait that ran out) are OR-ed into a sticky
 *     device status word read by ict_get_device_status().
 *   - Unsupported geometry returns ICT_ERR_LAYOUT; there is no fallback path.
 *   - Mantissa matrices are row-major with a leading dimension `ld` (elements = bytes);
 *     outputs never alias inputs, except that the SGD step updates W and V in place.
 *   - Inputs must satisfy |C| <= 127 and have all-zero mantissas in ICT_E_ZERO groups
 *     (every output of this library does).  Other inputs give unspecified (but
 *     memory-safe) results.
 */
#ifndef ICT_H
#define ICT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ICT_E_ZERO (-128)
#define ICT_QMAX 127

typedef enum {
    ICT_OK = 0,
    ICT_ERR_INVALID_ARG = 1,    /* null pointer, bad size, inconsistent shapes */
    ICT_ERR_LAYOUT = 2,         /* group geometry or shape the library does not support */
    ICT_ERR_ALIGNMENT = 3,      /* pointer or leading dimension not 16-byte aligned */
    ICT_ERR_WORKSPACE = 4,      /* ws too small or not 256-byte aligned */
    ICT_ERR_UNSUPPORTED_ARCH = 5, /* current device is not sm_100 */
    ICT_ERR_CUDA = 6,           /* a CUDA runtime or driver call failed */
    ICT_ERR_DEVICE_TIMEOUT = 7, /* (device word) a bounded wait inside a kernel ran out */
    ICT_ERR_EXP_RANGE = 8       /* (device word) a result needed an exponent above 127 */
} ict_status;

/* One (C,e) matrix view.
 *   mant   [rows][ld] int8, |C| <= 127
 *   exp    [ceil(rows/g_rows)][ceil(cols/g_cols)] int8, row-major, contiguous;
 *          group (i, j) covers rows [i*g_rows, ...) and columns [j*g_cols, ...);
 *          edge groups may be short.  g_rows >= rows means one group row (uniform over
 *          rows), g_cols >= cols one group column.
 *   For outputs the caller chooses g_rows/g_cols and the library writes mant and exp. */
typedef struct {
    int8_t *mant;
    int8_t *exp;
    int64_t rows, cols, ld;
    int32_t g_rows, g_cols;
} ict_tensor;

/* SGD with momentum as integer multiply-shifts: beta = mom_mul * 2^-mom_shift,
 * lr = lr_mul * 2^-lr_shift (Table 10: momentum 0.9 -> 230, 8). */
typedef struct {
    int32_t mom_mul, mom_shift, lr_mul, lr_shift;
} ict_sgd_params;

/* NHWC activations, KRSC weights.  Activations are ict_tensor views
 * [n*h*w][c] (or [n*p*q][k]); weights are [k][r*s*c]. */
typedef struct {
    int32_t n, h, w, c, k, r, s, stride, pad;
} ict_conv_desc;

typedef enum { ICT_CONV_FWD = 0, ICT_CONV_BWD_DATA = 1, ICT_CONV_BWD_WEIGHT = 2 } ict_conv_dir;

typedef enum { ICT_OP_LINEAR_FWD = 0, ICT_OP_LINEAR_BWD_DATA = 1, ICT_OP_LINEAR_BWD_WEIGHT = 2 } ict_linear_op;

/* Human-readable name of a status code (static string). */
const char *ict_status_string(int32_t status);

/* Reads the sticky device status word into *host_out and clears it.  Synchronises
 * `stream`.  ICT_OK means no device-side condition was raised since the last call. */
int32_t ict_get_device_status(int32_t *host_out, void *stream);

/* Library build identification: returns a static string. */
const char *ict_version(void);

/* Number of kernels this process has launched through the library so far (all devices,
 * all threads).  Lets a caller count the device work a sequence of calls issues. */
uint64_t ict_launch_count(void);

/* Device timing by kernel class, for measurement.  While enabled, every launch the
 * library makes is bracketed by a pair of CUDA events recorded on its stream (events are
 * created on first use and reused; no device memory is allocated).  ict_timing_read()
 * synchronises the recorded events, adds their durations into per-class totals and
 * returns, for one class, the summed device time (ms), the number of timed launches and
 * their algorithmic work: multiply-add operations (2 M N K) for ICT_KC_GEMM, bytes read
 * plus written for the memory-bound classes.  reset = 1 clears every class afterwards. */
typedef enum {
    ICT_KC_GEMM = 0,    /* tensor-core Product kernels (linear, conv) */
    ICT_KC_SGD = 1,     /* integer SGD-with-momentum update */
    ICT_KC_ALIGN = 2,   /* ALIGN_MAX mantissa shifts (and transposes) */
    ICT_KC_REQUANT = 3, /* FIT of int32 / int64 values (split-K combine) */
    ICT_KC_GELU = 4,    /* GELU forward / backward */
    ICT_KC_ESTAR = 5,   /* target exponents e* of ALIGN_MAX (maxima of group exponents) */
    ICT_KC_OTHER = 6,   /* fills, weight re-layout and exponent tables */
    ICT_KC_POINTWISE = 7 /* ReLU / ReLU6 and Sum (residual add) */
} ict_kernel_class;
int32_t ict_timing_enable(int32_t on);
int32_t ict_timing_read(int32_t kernel_class, double *ms_total, int64_t *launches, double *work,
                        int32_t reset);

/* Bound, in nanoseconds, of every wait inside a kernel (0 restores the default, 2 s).
 * A wait that runs out raises ICT_ERR_DEVICE_TIMEOUT in the device status word; the
 * kernel then lets its in-flight copies and tensor-core operations finish (again with a
 * bound), releases its tensor memory and exits, leaving the context usable and the
 * outputs unspecified.  Process-wide; meant for tests of that path. */
int32_t ict_set_wait_limit_ns(uint64_t ns);

/* Self-test of the bounded-wait path: launches one block that waits on an mbarrier no
 * one ever arrives on, bounded by limit_ns (nanoseconds, > 0).  When the bound runs out
 * the block raises ICT_ERR_DEVICE_TIMEOUT in the device status word and exits; nothing
 * faults, traps or hangs, and the context stays usable.  Asynchronous on `stream`. */
int32_t ict_selftest_wait_timeout(uint64_t limit_ns, void *stream);

/* --------------------------------------------------------------------------------- */
/* Requantisation (FIT) of integer values, the step that closes every Product         */
/* (Table 6, Eqs. 5 and 3; Figure 1a).                                                 */
/*   vals      device [rows][ld_vals] of int32 (val_bits = 32) or int64 (64)            */
/*   element (i, j) has exponent base_exp + row_exp[i] + col_exp[j]                      */
/*   (row_exp / col_exp: device int8 vectors, either may be NULL = 0; an ICT_E_ZERO      */
/*   entry requires the value to be 0)                                                  */
/*   out       groups chosen by the caller; rows/cols must match                        */
int32_t ict_requant(const void *vals, int32_t val_bits, int64_t rows, int64_t cols,
                    int64_t ld_vals, int32_t base_exp, const int8_t *row_exp,
                    const int8_t *col_exp, ict_tensor *out, void *stream);

/* ALIGN_MAX of one operand (reading of the Sum primitive, Table 6 Eq. 6).
 *   axis = 1: the contracted index runs along columns -> e_star[rows]
 *   axis = 0: the contracted index runs along rows    -> e_star[cols]
 *   out_mant  device, [rows][ld_out] (or [cols][ld_out] when transpose = 1)
 *   e_star    device int8 vector of the aligned exponents                           */
int32_t ict_align(const ict_tensor *in, int32_t axis, int32_t transpose, int8_t *out_mant,
                  int64_t ld_out, int8_t *e_star, void *stream);

/* --------------------------------------------------------------------------------- */
/* Linear layer Product in the three training directions (Figure 1a; Table 6          */
/* "Linear / fully-connected").  Operands whose exponent varies along the contracted   */
/* index are aligned (ALIGN_MAX) into `ws` first; the int8 x int8 -> int32 contraction */
/* runs on the tensor cores and the FIT requant is fused into its epilogue where the   */
/* output groups lie inside one tile.                                                 */
/*   fwd          Y[M][N]  = X[M][K] * W[N][K]^T                                       */
/*   bwd_data     dX[M][K] = dY[M][N] * W[N][K]                                        */
/*   bwd_weight   dW[N][K] = dY[M][N]^T * X[M][K]                                      */
/* Output groups must be row-local (g_rows = 1).  Leading dimensions and pointers must */
/* be 16-byte aligned.                                                                 */
size_t ict_linear_workspace(int32_t op, const ict_tensor *a, const ict_tensor *b,
                            const ict_tensor *out);
int32_t ict_linear_fwd(const ict_tensor *X, const ict_tensor *W, ict_tensor *Y, void *ws,
                       size_t ws_bytes, void *stream);
int32_t ict_linear_bwd_data(const ict_tensor *dY, const ict_tensor *W, ict_tensor *dX,
                            void *ws, size_t ws_bytes, void *stream);
int32_t ict_linear_bwd_weight(const ict_tensor *dY, const ict_tensor *X, ict_tensor *dW,
                              void *ws, size_t ws_bytes, void *stream);

/* Backward-weight Product of a batch split across devices (data-parallel training, one
 * process per GPU; Abstract: the method trains ResNet and ViT models on ImageNet, whose
 * batches are split this way).  dW = dY^T X contracts over the batch, so its only
 * exchange is there; the steps are, on every device with its shard dY_r [K_r][M],
 * X_r [K_r][N] (K_r may differ, and may be 0):
 *   1. ict_linear_bwd_weight_targets(dY_r, X_r, e_dy, e_x): the ALIGN_MAX targets of the
 *      shard, the largest group exponent of each column (ICT_E_ZERO: all groups zero);
 *   2. element-wise MAX of e_dy and e_x over the devices (an all-reduce on int8; the
 *      ordering of int8 puts ICT_E_ZERO = -128 below every real exponent);
 *   3. ict_linear_bwd_weight_partial(dY_r, X_r, e_dy, e_x, acc): the shard aligned to
 *      those targets and contracted exactly,
 *        acc[m][n] = sum_k A(dY_r)[k][m] * A(X_r)[k][n],  exponent e_dy[m] + e_x[n];
 *   4. element-wise SUM of acc over the devices (an all-reduce on int32 / int64; integer
 *      addition is exact in any order);
 *   5. ict_requant(acc, bits, M, N, ld_acc, 0, e_dy, e_x, dW).
 * The result equals ict_linear_bwd_weight on the whole batch bit for bit, whatever the
 * split.  With one device, steps 2 and 4 are identities.
 *   e_dy [M], e_x [N]   device int8 target vectors; outputs of step 1, inputs of step 3.
 *                       Each target must be at least every group exponent of the shard's
 *                       column, and equal across the columns of one group column, as the
 *                       maxima of step 2 are when every device uses the same group
 *                       widths; other values give unspecified, memory-safe results.
 *   acc                 device, [M][ld_acc] row-major, int64 (acc_bits = 64) or int32
 *                       (32: allowed only when K_r * 127^2 < 2^31, and the caller must
 *                       keep the SUM of step 4 below 2^31 in magnitude, e.g. with
 *                       (sum of all K_r) * 127^2 < 2^31).  16-byte aligned, ld_acc a
 *                       multiple of 4 (ICT_ERR_ALIGNMENT otherwise).  Fully written.
 *   ws                  both calls need ict_linear_bwd_weight_partial_workspace() bytes
 *                       (256-byte aligned); returns 0 for invalid operands.
 * Operands follow ict_linear_bwd_weight's rules (16-byte aligned, cols multiples of 16,
 * row-local or uniform groups).  Asynchronous on `stream`. */
size_t ict_linear_bwd_weight_partial_workspace(const ict_tensor *dY, const ict_tensor *X);
int32_t ict_linear_bwd_weight_targets(const ict_tensor *dY, const ict_tensor *X, int8_t *e_dy,
                                      int8_t *e_x, void *ws, size_t ws_bytes, void *stream);
int32_t ict_linear_bwd_weight_partial(const ict_tensor *dY, const ict_tensor *X,
                                      const int8_t *e_dy, const int8_t *e_x, void *acc,
                                      int32_t acc_bits, int64_t ld_acc, void *ws,
                                      size_t ws_bytes, void *stream);

/* Mantissa width of the B-bit variants (Table 4 trains the same method with INT8 down to
 * INT4 mantissas; Table 7's clip bound is q_max = 2^(B-1) - 1).  Process-wide, 2 <= B <= 8,
 * default 8; read when an entry point is called.  With B < 8 every FIT of the linear
 * Products (all three directions, the split-batch forms and ict_linear_fwd_noalloc),
 * ict_requant and the SGD updates picks the smallest exponent at which the group fits
 * [-q_max, q_max]; alignment, contraction and the two-term sums are unchanged (their
 * results stay within the inputs' width).  Mantissas stay one per byte.  Entry points
 * whose FIT is INT8-only (convolution, depthwise convolution, Sum, average pool, GELU
 * backward, the output head, ReLU6) return ICT_ERR_LAYOUT while B < 8; ReLU, GELU
 * forward and patch extraction never widen a mantissa and accept any B.
 * ict_set_mantissa_bits returns ICT_ERR_INVALID_ARG outside [2, 8]. */
int32_t ict_set_mantissa_bits(int32_t bits);
int32_t ict_get_mantissa_bits(void);

/* Allocation-free forward Product.  The paper has no counterpart to this entry point;
 * it exists for callers that cannot hand the library a device workspace: integrations
 * whose device memory is reserved up front by a host framework that exposes no
 * allocator, statically budgeted deployments, and code paths that must not call
 * cudaMalloc/cudaFree because those calls can block or synchronise the device.
 * Same arguments and result as ict_linear_fwd, without ws: the scratch it needs (the
 * aligned copies of X and/or W and, when the output groups span several tiles, int32
 * partial sums) lives in one fixed array of ICT_NOALLOC_SCRATCH_BYTES bytes inside the
 * library, which every GPU that loads the library holds until the process exits.
 *   - Problems whose scratch need (ict_linear_workspace for the same arguments) exceeds
 *     ICT_NOALLOC_SCRATCH_BYTES are rejected with ICT_ERR_WORKSPACE before any launch.
 *   - It never calls cudaMalloc, cudaFree or any allocating routine.
 *   - The first call on a device looks up that device's copy of the array (with the
 *     device current); make that first call before any stream capture.  The address is
 *     kept with the CUDA context it belongs to: after a device reset (cudaDeviceReset,
 *     or a framework that resets the device) the next call looks it up again, and is
 *     then again a first call.
 *   - All calls share the one array and it keeps the last call's contents: calls that
 *     can overlap on the GPU (other streams, other threads) race on it and must be
 *     serialised by the caller. */
#define ICT_NOALLOC_SCRATCH_BYTES (16u << 20)
int32_t ict_linear_fwd_noalloc(const ict_tensor *X, const ict_tensor *W, ict_tensor *Y, void *stream);

/* --------------------------------------------------------------------------------- */
/* Convolution as implicit GEMM (Table 6: "Convolution ... Product").                  */
/*   dir FWD         a = X  [n*h*w][c], b = W [k][r*s*c] -> out = Y  [n*p*q][k]        */
/*   dir BWD_DATA    a = dY [n*p*q][k], b = W [k][r*s*c] -> out = dX [n*h*w][c]        */
/*   dir BWD_WEIGHT  a = dY [n*p*q][k], b = X [n*h*w][c] -> out = dW [k][r*s*c]        */
/* Activation exponents must be uniform over pixels (g_rows >= rows).  Output groups   */
/* of FWD / BWD_DATA are pixel-local (g_rows = 1) or span all pixels (g_rows >= rows);  */
/* their width g_cols is a multiple of 32 that divides the output tile width (64, 128,  */
/* 192 or 256 channels, the smallest that holds out_c, else 256), or covers all out_c <= */
/* 256 channels.  dW groups are per row.  The library supports square odd filters with   */
/* "same" padding and stride 1 (r = s, pad = (r - 1) / 2: 1x1, 3x3, 5x5, 7x7, ...), c    */
/* and k multiples of 64 up to 2048, w <= 128.  ict_conv_workspace() is an upper bound  */
/* for the direction.  For FWD and BWD_DATA it includes, for output groups spanning all */
/* pixels, int16 sums of the whole output (2 bytes per element) and one int32 need per  */
/* output tile and group column: the Product pass rounds each exact sum to odd at an    */
/* exponent 7 below its tile's largest need() (the int16 fits by construction) and      */
/* raises every group's largest need; a streaming pass rounds to nearest even at the    */
/* group exponent, a shift of at least 7 bits, which equals RNE of the exact sum.       */
size_t ict_conv_workspace(int32_t dir, const ict_conv_desc *d);
int32_t ict_conv_implicit_gemm(int32_t dir, const ict_conv_desc *d, const ict_tensor *a,
                               const ict_tensor *b, ict_tensor *out, void *ws,
                               size_t ws_bytes, void *stream);

/* Convolution over a batch split across devices (images split between the ranks of a
 * data-parallel run).  Every rank's activation operands must carry the exponents of the
 * whole batch's tensor (true of outputs made by this split form); then:
 *  - output groups local to each pixel (g_rows = 1): no exchange, each rank calls
 *    ict_conv_implicit_gemm on its shard;
 *  - FWD / BWD_DATA with output groups spanning all pixels: the group exponent depends
 *    on every shard.  ict_conv_split_begin writes the shard's largest need() per output
 *    group column into need[ceil(out_c / g_cols)] (int32; below -2^30 when the shard's
 *    group is all zero) and keeps the int32 sums in ws; after an element-wise MAX of need
 *    over the ranks, ict_conv_split_end writes the shard's rows of `out`.  Same
 *    arguments and the same, untouched ws (ict_conv_workspace(dir, d) bytes, d the
 *    shard's descriptor) in both calls;
 *  - BWD_WEIGHT: ict_conv_bwd_weight_partial writes the shard's exact int64 sums
 *    acc[k][(r,s,c)] (row stride ld_acc >= r*s*c) and the exponent vectors
 *    e_k[k] (dY's channel exponents) and e_rsc[(r,s,c)] (X's, per filter tap); after an
 *    element-wise SUM of acc over the ranks, ict_requant(acc, 64, k, r*s*c, ld_acc, 0,
 *    e_k, e_rsc, dW) gives dW.
 * The results equal ict_conv_implicit_gemm on the whole batch bit for bit. */
int32_t ict_conv_split_begin(int32_t dir, const ict_conv_desc *d, const ict_tensor *a,
                             const ict_tensor *b, ict_tensor *out, int32_t *need, void *ws,
                             size_t ws_bytes, void *stream);
int32_t ict_conv_split_end(int32_t dir, const ict_conv_desc *d, const ict_tensor *a,
                           const ict_tensor *b, ict_tensor *out, const int32_t *need, void *ws,
                           size_t ws_bytes, void *stream);
int32_t ict_conv_bwd_weight_partial(const ict_conv_desc *d, const ict_tensor *dY,
                                    const ict_tensor *X, int64_t *acc, int64_t ld_acc,
                                    int8_t *e_k, int8_t *e_rsc, void *ws, size_t ws_bytes,
                                    void *stream);

/* Depthwise convolution, one R x S filter per channel (Table 6: "Convolution (incl.    */
/* 1 x 1, depthwise)" -> Product; MobileNetV2).  d->k must equal d->c; any stride and    */
/* padding, R * S <= 49.  The contraction of channel ch runs over its own taps, so the    */
/* sums keep the activation's per-channel exponent: element exponent e_act[ch] + e_w[ch].*/
/*   dir FWD         a = X  [n*h*w][c], b = W [c][r*s] -> out = Y  [n*P*Q][c]          */
/*   dir BWD_DATA    a = dY [n*P*Q][c], b = W [c][r*s] -> out = dX [n*h*w][c]          */
/*   dir BWD_WEIGHT  a = dY [n*P*Q][c], b = X [n*h*w][c] -> out = dW [c][r*s]          */
/* Activation exponents uniform over pixels (g_rows >= rows); W and dW one group per row */
/* (g_rows = 1, g_cols >= r*s).  FWD / BWD_DATA outputs: any group geometry, rounded in  */
/* two passes with an int32 per output group of workspace (ict_depthwise_workspace).     */
/* Byte accesses on CUDA cores (the contraction has 9-49 terms per output).              */
size_t ict_depthwise_workspace(int32_t dir, const ict_conv_desc *d, const ict_tensor *out);
int32_t ict_depthwise(int32_t dir, const ict_conv_desc *d, const ict_tensor *a, const ict_tensor *b,
                      ict_tensor *out, void *ws, size_t ws_bytes, void *stream);

/* Patch embedding (a P x P convolution with stride P, as a ViT's first layer): the     */
/* non-overlapping patches of NHWC X [n*h*w][c] gathered into the rows of             */
/* out [n*(h/P)*(w/P)][P*P*c] in (dy, dx, channel) order, ALIGN_MAX-ed to one exponent */
/* (the largest of X's channel-group exponents, which are uniform over pixels; out has */
/* one group: g_rows >= rows, g_cols >= cols).  ict_linear_fwd(out, W [k][P*P*c]) is   */
/* then the patch-embedding forward, equal to the convolution's (stride P, pad 0)      */
/* result; ict_linear_bwd_weight(dY, out) its weight gradient.  h and w multiples of P,  */
/* P*c a multiple of 16; X's groups either one per tensor (then c may be narrow, e.g.  */
/* 3 RGB channels, with pixels packed: ld = c) or 16-aligned channel groups with c a   */
/* multiple of 16.                                                                      */
int32_t ict_patchify(const ict_tensor *X, int32_t n, int32_t h, int32_t w, int32_t P,
                     ict_tensor *out, void *stream);

/* --------------------------------------------------------------------------------- */
/* Integer SGD with momentum and per-group velocity (Figure 1b; Abstract: "per-group   */
/* velocity mechanism with independent exponent tracking").  Per group:                */
/*   v <- FIT(beta * v + g)      w <- FIT(w - lr * v)                                  */
/* each right-hand side an exact two-term Sum.  W, V, G share one shape and one        */
/* row-local group partition (g_rows = 1); W and V are updated in place.               */
int32_t ict_sgd_momentum_step(ict_tensor *W, ict_tensor *V, const ict_tensor *G,
                              const ict_sgd_params *p, void *stream);
/* The same update over n_tensors independent (W, V, G) triples in one launch
 * (n_tensors <= 128). */
int32_t ict_sgd_momentum_step_multi(int32_t n_tensors, ict_tensor *const *W,
                                    ict_tensor *const *V, const ict_tensor *const *G,
                                    const ict_sgd_params *p, void *stream);

/* --------------------------------------------------------------------------------- */
/* Integer GELU stand-in h(x) = x * clip((x + 2) / 4, 0, 1) (the page's GELU is a      */
/* lookup table, Table 7 / Eq. 19, whose contents are not printed).                    */
/*   fwd: exponent carried through unchanged (Table 7 caption); out has H's groups.    */
/*   bwd: dH = FIT(dG * h'(H)) into dH's groups; H, dG, dH share one row-local group   */
/*        partition.                                                                    */
int32_t ict_gelu_fwd(const ict_tensor *H, ict_tensor *out, void *stream);
int32_t ict_gelu_bwd(const ict_tensor *H, const ict_tensor *dG, ict_tensor *dH, void *stream);

/* --------------------------------------------------------------------------------- */
/* The nonlinear-function primitive through lookup tables.                             */
/*   Table 7 (GELU): forward LUT_fwd[e, C], backward (dY * LUT_bwd[e, C]) >> B_G, INT8  */
/*   [30, 256], the exponent carried unchanged.  Table 8 (output head): LUT_exp[e][k] = */
/*   round(exp(k 2^e) 2^7), k in [-255, 0], [30, 256]; LUT_log[p] = round(-log(p / 2^8)*/
/*   2^5), p in [1, 254], [256]; built once at initialization.                         */
/* Readings (the page prints the entry formulas only): the 30 table exponents are       */
/* e = -26 .. 3 and a lookup clamps e to them (the formulas give the end rows' values   */
/* for every exponent beyond); "round" is half to even; GELU(x) = x Phi(x) with Phi the */
/* standard normal CDF, LUT_fwd[e][C] = round(C Phi(C 2^e)), LUT_bwd[e][C] =            */
/* round(GELU'(C 2^e) 2^6) (B_G = 6: the slope lies in about [-0.129, 1.129]).          */
/* The library builds its tables once per process on the host.                          */
/*                                                                                      */
/* ict_lut_tables: host copies of the library's tables (any pointer may be NULL):        */
/*   lut_exp [30][256] uint8 at [e + 26][k + 255];  lut_log [256] uint8 at [p] (entries  */
/*   0 and 255 repeat 1 and 254);  gelu_fwd / gelu_bwd [30][256] int8 at [e + 26][C+128].*/
/*   Host memory only; launches nothing.                                                */
/* ict_gelu_lut_fwd: out mantissa = LUT_fwd[e][C]; out has H's shape and groups and      */
/*   receives H's exponents.  cols, ld and g_cols multiples of 16 (or g_cols >= cols).  */
/* ict_gelu_lut_bwd: dH = FIT(dY * LUT_bwd[e_H][C_H] * 2^-6), the exact product at       */
/*   exponent e_dY - 6 requantised into dH's groups like every product; H, dY and dH     */
/*   share one row-local group partition (g_rows = 1, g_cols a multiple of 16).          */
/* ict_softmax_ce: the output head on logits Z [rows][classes] with one target class per */
/*   row (target[rows], int32 in [0, classes), device memory).  Per row: the logits to  */
/*   one exponent e (ALIGN_MAX along the row); k = C - max C; E = LUT_exp[e][k];        */
/*   S = sum E; p = round(E 2^8 / S) (exact quotient, half to even); loss[row] =        */
/*   LUT_log[clamp(p_target, 1, 254)] (int32, device memory, the cross-entropy at scale  */
/*   2^-5); dZ = FIT(p - 2^8 [class = target]) at exponent -8 into dZ's row-local groups */
/*   (the gradient of the summed loss).  Argument errors return before any launch.      */
int32_t ict_lut_tables(uint8_t *lut_exp, uint8_t *lut_log, int8_t *gelu_fwd, int8_t *gelu_bwd);
int32_t ict_gelu_lut_fwd(const ict_tensor *H, ict_tensor *out, void *stream);
int32_t ict_gelu_lut_bwd(const ict_tensor *H, const ict_tensor *dY, ict_tensor *dH, void *stream);
int32_t ict_softmax_ce(const ict_tensor *Z, const int32_t *target, int32_t *loss, ict_tensor *dZ,
                       void *stream);

/* --------------------------------------------------------------------------------- */
/* ReLU / ReLU6, the Clip primitive (Table 6: "ReLU / ReLU6 -> Clip"; Table 7): integer  */
/* operations on the mantissas C, the exponent carried through unchanged.              */
/*   six = 0: ReLU    forward  Z = max(C, 0)          backward dX = dY * 1[C > 0]       */
/*   six = 1: ReLU6   forward  Z = clip(C, 0, c)      backward dX = dY * 1[0 < C < c]   */
/*   c = min(6 >> e, 127) for the group exponent e of C: 6 shifted right by e (left for  */
/*   e < 0), truncating, so e = 2 gives 1 and e >= 3 gives 0; taken literally, the     */
/*   backward mask also drops C = 127 where c = 127 (e <= -5).                          */
/* Forward: Z has X's shape and group geometry and receives a copy of X's exponents.    */
/* Backward: X is the forward input; dX has dY's shape and groups and receives a copy   */
/* of dY's exponents.  Tensors: cols multiple of 16, mantissas and ld 16-byte aligned,  */
/* group widths multiples of 16 (or one group per row).                                 */
int32_t ict_relu_fwd(const ict_tensor *X, int32_t six, ict_tensor *Z, void *stream);
int32_t ict_relu_bwd(const ict_tensor *X, const ict_tensor *dY, int32_t six, ict_tensor *dX,
                     void *stream);

/* --------------------------------------------------------------------------------- */
/* Sum (Table 6: "Residual add, gradient merge -> Sum", Eq. 6): Z = FIT(X + Y), every   */
/* element's two terms x * 2^ex + y * 2^ey added exactly, then requantised into Z's     */
/* groups.  X, Y, Z share one shape and one group partition: row-local groups (g_rows  */
/* = 1, as the linear layers produce) or groups spanning all rows (g_rows >= rows, the  */
/* pixel-uniform channel groups of convolution activations; at most 8192 group        */
/* columns).  Group widths are multiples of 16 or span the row; cols a multiple of 16;  */
/* mantissas and ld 16-byte aligned.  Groups spanning all rows need an int32 per group  */
/* column of workspace (ict_sum_workspace; 0 for row-local groups, where ws may be     */
/* NULL); the result is written in two streaming passes.                              */
/* Z must not alias X or Y. */
size_t ict_sum_workspace(const ict_tensor *X, const ict_tensor *Y, const ict_tensor *Z);
int32_t ict_sum(const ict_tensor *X, const ict_tensor *Y, ict_tensor *Z, void *ws,
                size_t ws_bytes, void *stream);
/* The weighted Sum Z = FIT(x_mul 2^-x_shift X + y_mul 2^-y_shift Y), weights as integer
 * multiply-shifts like the SGD step's (|mul| <= 512, 0 <= shift <= 64; others
 * ICT_ERR_INVALID_ARG).  Weights (1, 0), (1, 0) are ict_sum.  SGD's weight decay
 * (Table 10: 1e-4) is G' = FIT(G + lambda W), lambda = y_mul 2^-y_shift (105 2^-20 for
 * 1e-4), into G's groups, before ict_sgd_momentum_step.  Same rules as ict_sum. */
int32_t ict_sum_scaled(const ict_tensor *X, int32_t x_mul, int32_t x_shift, const ict_tensor *Y,
                       int32_t y_mul, int32_t y_shift, ict_tensor *Z, void *ws, size_t ws_bytes,
                       void *stream);
/* Activations fused into a rounding pass (Table 7: integer operations on C, exponents
 * unchanged): act 0 none, 1 ReLU, 2 ReLU6 (bound from the output group's exponent).
 * ict_sum_act: Z = act(FIT(X + Y)), the residual add and the ReLU after it in one pass;
 *   the ReLU backward mask can be taken from Z (Z > 0 exactly where FIT(X + Y) > 0,
 *   and Z < c where it is below the ReLU6 bound c).
 * ict_conv_fwd_act: Y = act(conv forward), fused into the streaming rounding pass when
 *   Y's groups span all pixels, else a clip pass over Y in place.  Same arguments and
 *   workspace as ict_conv_implicit_gemm with ICT_CONV_FWD. */
int32_t ict_sum_act(const ict_tensor *X, const ict_tensor *Y, ict_tensor *Z, int32_t act, void *ws,
                    size_t ws_bytes, void *stream);
int32_t ict_conv_fwd_act(const ict_conv_desc *d, const ict_tensor *X, const ict_tensor *W,
                         ict_tensor *Y, int32_t act, void *ws, size_t ws_bytes, void *stream);

/* --------------------------------------------------------------------------------- */
/* Average pool K x K, stride K (Table 6: "Average pool (K x K) -> Divide-by-constant",   */
/* Eqs. 7-8, whose text the page does not print).  Reading: every output element is an   */
/* exact integer S at exponent e divided by the constant D = K*K, rounded once by FIT    */
/* into the output's groups: mantissa RNE(S 2^(e - E) / D), E the smallest exponent at   */
/* which every member of the group fits (raised to -127; ICT_E_ZERO for all zero).       */
/*   forward   X [n*h*w][c] NHWC, exponents uniform over pixels (g_rows >= rows);        */
/*             S = the window's mantissa sum.  Y [n*(h/K)*(w/K)][c].                     */
/*   backward  dY [n*(h/K)*(w/K)][c], any group geometry; every pixel of a window takes  */
/*             S = the window's dY mantissa at dY's exponent.  dX [n*h*w][c].            */
/* h and w multiples of K, 1 <= K <= 16.  Output groups: any geometry.  Two passes (the   */
/* groups' needs into ws, int32 per output group: ict_avgpool_workspace, dir 0 = forward, */
/* 1 = backward, then the rounding).  No alignment requirements.                         */
size_t ict_avgpool_workspace(int32_t dir, const ict_tensor *in, int32_t n, int32_t h, int32_t w,
                             int32_t K, const ict_tensor *out);
int32_t ict_avgpool_fwd(const ict_tensor *X, int32_t n, int32_t h, int32_t w, int32_t K,
                        ict_tensor *Y, void *ws, size_t ws_bytes, void *stream);
int32_t ict_avgpool_bwd(const ict_tensor *dY, int32_t n, int32_t h, int32_t w, int32_t K,
                        ict_tensor *dX, void *ws, size_t ws_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* ICT_H */
