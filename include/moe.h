/*
 * moe.h - C ABI of the B200 (sm_100a) LongCat-Flash Mixture-of-Experts layer forward.
 *
 * The layer (LongCat-Flash Technical Report digest, Key claims, report §2.1 / §2.4):
 * a router scores every token against a pool of n_ffn SwiGLU FFN experts and n_zero
 * zero-computation (identity) experts and picks K of them per token. Selection uses the
 * bias-adjusted score p + b, the gate is the unbiased softmax probability p (report
 * §2.1.1). FFN picks are permuted into expert-contiguous groups and run through a grouped
 * GEMM; a zero-computation pick adds g * x and costs no GEMM. The per-batch expert
 * histogram drives a PID update of the FFN experts' biases (report §2.1.1, Fig. 3; the
 * zero experts are excluded from it, report §2.1.2).
 *
 * Conventions for every call
 *  - Expert indices: FFN experts are [0, n_ffn), zero-computation experts are
 *    [n_ffn, n_ffn + n_zero). E = n_ffn + n_zero.
 *  - Pointers marked "device" are CUDA device pointers on the current device; the caller
 *    owns every buffer. The library never allocates, frees or synchronises, except
 *    moe_read_device_status, which synchronises the given stream, and the host pipeline
 *    (its own streams and events).
 *  - Every call is asynchronous on `stream` (a cudaStream_t passed as void*; NULL is the
 *    legacy default stream). Stream order is the only requirement on inputs: any input
 *    may be written by earlier work on the same stream, including this library's own
 *    previous call (one layer's `out` passed as the next layer's `x`). The kernels start
 *    early as programmatic dependents of their predecessors, but they read nothing a
 *    predecessor may write until it has completed.
 *  - Layouts are row-major and contiguous. Device pointers must be 16-byte aligned.
 *  - x, x_perm, h, y_perm and out hold `dtype` elements (bf16 or fp32); logits, gates,
 *    biases and out_acc are fp32; indices and counts are int32.
 *  - Return value: MOE_OK (0) or a negative MOE_ERR_* code. Argument checks happen on the
 *    host before anything is launched, so a call that returns an error has launched
 *    nothing. Inconsistencies only the device can see (an expert index out of range, a
 *    bounded wait that ran out) are written to a status word inside the workspace and
 *    read back with moe_read_device_status; kernels never trap.
 *  - T = 0 is valid: the call checks its arguments and launches nothing.
 *  - Limits: 1 <= E <= 1024, 1 <= K <= min(32, E), n_ffn >= 1, n_zero >= 0, T < 2^24,
 *    T * K < 2^31, H % 16 == 0 (rows move 16 bytes at a time), I >= 1. bf16 also needs
 *    H % 128 == 0 and I % 128 == 0. Other shapes give MOE_ERR_UNSUPPORTED.
 */
#ifndef MOE_B200_H_
#define MOE_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------------------- */
#define MOE_OK                  0
#define MOE_ERR_INVALID_ARG    -1   /* null pointer, bad size, K > E, ...               */
#define MOE_ERR_UNSUPPORTED    -2   /* shape outside the limits above                   */
#define MOE_ERR_ALIGNMENT      -3   /* a device pointer is not 16-byte aligned          */
#define MOE_ERR_CUDA           -4   /* a CUDA runtime or driver call failed             */
#define MOE_ERR_WORKSPACE      -5   /* workspace missing or smaller than required       */
#define MOE_ERR_DEVICE_CHECK   -6   /* device-side consistency check failed (status)    */
#define MOE_ERR_TIMEOUT        -7   /* a bounded device-side wait ran out (status)      */
#define MOE_ERR_NO_DEVICE      -8   /* no CUDA device, or not an sm_100 device          */

typedef enum { MOE_BF16 = 0, MOE_FP32 = 1 } moe_dtype_t;

/* MOE_COMBINE_FUSED: the down-projection epilogue adds s * g * y into an fp32 out_acc with
 * atomic adds (fast; the fp32 summation order, hence the last bits, vary run to run).
 * MOE_COMBINE_DETERMINISTIC: the down projection stores y per permuted row (y_perm) and
 * moe_combine sums the K slots of each token in slot order: bit-reproducible. */
typedef enum { MOE_COMBINE_FUSED = 0, MOE_COMBINE_DETERMINISTIC = 1 } moe_combine_t;

typedef struct {
  int32_t T;              /* tokens                                                    */
  int32_t H;              /* hidden width                                              */
  int32_t I;              /* per-expert FFN intermediate width                         */
  int32_t n_ffn;          /* SwiGLU FFN experts                                        */
  int32_t n_zero;         /* zero-computation experts                                  */
  int32_t K;              /* experts chosen per token                                  */
  int32_t dtype;          /* moe_dtype_t                                               */
  int32_t combine;        /* moe_combine_t                                             */
  float ffn_out_scale;    /* s: factor on the FFN experts' outputs (report §2.3.2,
                             Eq. 8, "m*n" variance compensation; value not printed;
                             1.0 leaves the outputs unscaled)                          */
} moe_shape_t;

/* PID gains and target (report §2.1.1; the equation is not printed). target_ratio is the
 * wanted mean number of FFN picks per token divided by K. */
typedef struct {
  float kp, ki, kd, target_ratio;
} moe_pid_t;

/* ---- sizes and status ---------------------------------------------------------------- */

/* Bytes of scratch the step calls (moe_route, moe_permute, moe_grouped_ffn) need in `ws`.
 * Returns MOE_OK and writes *bytes, or an error for an invalid shape. No device access. */
int moe_scratch_size(const moe_shape_t* shape, size_t* bytes);

/* Bytes moe_forward needs in `ws`: the scratch plus every intermediate of the layer
 * (logits, zgate, offsets, the permutation, x_perm, h and y_perm or out_acc), sized for
 * the worst case of T * K FFN rows so that no call ever waits for the device. */
int moe_workspace_size(const moe_shape_t* shape, size_t* bytes);

/* Synchronises `stream`, writes the device status word of `ws` (0 when no device-side
 * check failed since the last read, else a MOE_ERR_* code) to *status and clears it. */
int moe_read_device_status(void* ws, size_t ws_bytes, void* stream, int32_t* status);

/* Static text for a MOE_* code. Never NULL. */
const char* moe_status_string(int code);

/* Number of kernels this library has launched in this process (all devices, all
 * threads). A benchmark reads it before and after a timed region. */
uint64_t moe_launch_count(void);

/* ---- tuning switches (measurements and tests) -------------------------------------------
 * The pages have no counterpart: these switches select between kernel variants that give
 * the same results, so that a measurement can compare them, plus one testing hook. Every
 * switch starts at its default. The library reads no environment variable. A switch is
 * process-wide: it applies to every device, and to every call made after it is set.
 * Changing one while another host thread is queuing calls gives that thread either
 * setting.
 *   MOE_TUNE_PDL              1 (default): kernels launch as programmatic dependents of
 *                             their predecessors on the stream; 0: plain stream order.
 *   MOE_TUNE_GEMM_PAIR        -1 (default): the bf16 expert GEMMs use CTA pairs
 *                             (tcgen05 cta_group::2, 256-row tiles) for T >= 1024, one CTA
 *                             per tile otherwise; 0: always one CTA; 1: always pairs.
 *   MOE_TUNE_PAIR_HALF        1 (default): in the CTA-pair GEMMs, an expert's last tile of
 *                             at most 128 rows runs as an M = 128 tile; 0: as M = 256.
 *   MOE_TUNE_ROUTER_N         0 (default): the bf16 router GEMM's tile width (128, 192 or
 *                             256 logits) follows from the shape; 192 or 256: that width
 *                             wherever 256-wide tiles fill a wave of SMs.
 *   MOE_TUNE_ROUTER_MIN_SPLIT 12 (default): fewest k-blocks of 64 in one split-K slice of
 *                             the bf16 router GEMM; 1 to 1024.
 *   MOE_TUNE_BWD_PAIR         1 (default): moe_backward's dgrad GEMMs run on CTA pairs
 *                             wherever the forward does, its weight-gradient GEMMs always;
 *                             2: only the dgrad GEMMs; 0: one CTA per tile everywhere.
 *   MOE_TUNE_BWD_DY_ROWS      4 (default): y rows each thread of the backward's dy kernel
 *                             loads before using them; 1: one at a time.
 *   MOE_TUNE_TEST_STALL       testing hook, 0 (default). Set to 1, the next gate/up GEMM
 *                             of moe_grouped_ffn (or moe_forward) leaves the first
 *                             k-block of its first tile unloaded. The waits on that stage
 *                             run out after their limit (2 s) and write MOE_ERR_TIMEOUT to
 *                             the status word; that call's outputs are undefined. The
 *                             switch returns to 0 when that launch is queued.
 *   MOE_TUNE_GATE_UP_BAND     0 (default): the library's choice; 1 to 64: the CTA-pair
 *   MOE_TUNE_DOWN_BAND        gate/up (down) GEMM visits an expert's 256-row M tiles in
 *                             bands of this many, each band N tile by N tile with its M
 *                             tiles fastest (1: M tile by M tile, N tiles fastest).
 *   MOE_TUNE_PAIR_INTERLEAVE  0 (default): plain expert order; 1: the CTA-pair GEMMs
 *                             spread the tiles of experts with at most 256 rows (one M
 *                             tile) evenly among the other experts' tiles.
 *   MOE_TUNE_PAIR_A_TRIM      1 (default): in the CTA-pair GEMMs each CTA loads only the A
 *                             rows of the expert's group that its MMA rows cover (boxes of
 *                             16, 64 or 128 rows, or none); 0: always 128-row boxes.
 *   MOE_TUNE_PAIR_SWAP_AB     1 (default): in the forward's CTA-pair GEMMs a tile of at
 *                             most 128 rows (a small expert, an expert's tail) runs with
 *                             the operands swapped: the expert's weights as the M = 256
 *                             side, the tile's rows (rounded up to 16, 32, 64 or 128) as
 *                             N; 0: such tiles run as M = 128 tiles.
 *   MOE_TUNE_PAIR_STREAM_HINT 1 (default): the CTA-pair GEMMs load the weights of experts
 *                             with at most 256 rows (read once) with an evict-first L2
 *                             policy; 0: plain loads.
 *   MOE_TUNE_PAIR_TAILS       0 (default): the pair kernel takes every row; 1: where the
 *                             forward's expert GEMMs use CTA pairs, each runs as two
 *                             launches: the pair kernel takes every expert's whole 256-row
 *                             tiles (and a last tile of more than 128 rows), the one-CTA
 *                             kernel the rest (at most 128 rows per expert).
 *   MOE_TUNE_PAIR_PREFETCH    0 (default): no prefetch; 1 to 64: for the tiles of experts with
 *                             at most 256 rows, the CTA-pair GEMMs' producer prefetches into
 *                             L2 the weight boxes it will load this many k-blocks later
 *                             (crossing into its next tile).
 *   MOE_TUNE_BWD_WGRAD_GROUP  tile order of the backward's weight-gradient GEMMs within an
 *                             expert: 16 (default), or 1 to 64: groups of this many M tiles,
 *                             N tiles outer within a group (a wave of tiles then spans fewer
 *                             operand columns); 0: M tiles outer, N tiles inner.
 *   MOE_TUNE_BWD_WGRAD_MIX    0 (default), or 1 to 65536: on CTA pairs, the weight-gradient
 *                             tiles of experts with at most this many rows alternate with
 *                             those of the larger experts (measured slower).
 *   MOE_TUNE_BWD_WGRAD_BK     64 (default) or 128: K rows (expert rows) per pipeline stage of
 *                             the CTA-pair weight-gradient GEMMs: six stages of 64-row
 *                             operand boxes, or three of 128-row ones.
 * moe_set_tuning returns MOE_ERR_INVALID_ARG for an unknown switch or a value outside its
 * range. moe_get_tuning writes the current value. */
typedef enum {
  MOE_TUNE_PDL = 0,
  MOE_TUNE_GEMM_PAIR = 1,
  MOE_TUNE_PAIR_HALF = 2,
  MOE_TUNE_ROUTER_N = 3,
  MOE_TUNE_ROUTER_MIN_SPLIT = 4,
  MOE_TUNE_BWD_PAIR = 5,
  MOE_TUNE_BWD_DY_ROWS = 6,
  MOE_TUNE_TEST_STALL = 7,
  MOE_TUNE_GATE_UP_BAND = 8,
  MOE_TUNE_DOWN_BAND = 9,
  MOE_TUNE_PAIR_INTERLEAVE = 10,
  MOE_TUNE_PAIR_A_TRIM = 11,
  MOE_TUNE_PAIR_SWAP_AB = 12,
  MOE_TUNE_PAIR_STREAM_HINT = 13,
  MOE_TUNE_PAIR_TAILS = 14,
  MOE_TUNE_PAIR_PREFETCH = 15,
  MOE_TUNE_BWD_WGRAD_GROUP = 16,
  MOE_TUNE_BWD_WGRAD_MIX = 17,
  MOE_TUNE_BWD_WGRAD_BK = 18
} moe_tune_t;

int moe_set_tuning(int knob, int64_t value);
int moe_get_tuning(int knob, int64_t* value);

/* ---- the steps of the layer ------------------------------------------------------------ */

/* Router: logits, softmax over all E experts, bias-adjusted top-K, gates and histograms
 * (report §2.1, §2.1.1).
 *   x          device [T, H] dtype            token activations (unused if logits_in)
 *   w_router   device [E, H] fp32             router weight (unused if logits_in)
 *   logits_in  device [T, E] fp32 or NULL     given logits; NULL: computed as x . w_r^T
 *   bias       device [E] fp32                selection bias
 *   logits_out device [T, E] fp32             receives the logits; may be NULL only when
 *                                             logits_in is given
 *   topk_idx   device [T, K] int32            chosen experts, by (p + b) descending,
 *                                             ties to the lower index
 *   topk_gate  device [T, K] fp32             gates = softmax probabilities p (not
 *                                             renormalised; the bias is not in them)
 *   counts     device [E] int32               tokens per expert (zeroed by the call)
 *   nffn_hist  device [K + 1] int32           tokens with n FFN picks (zeroed by the call)
 *   zgate      device [T] fp32                sum of each token's zero-expert gates
 *   ws         device scratch, >= moe_scratch_size bytes
 * p is computed in double and rounded once to fp32; p + b is one fp32 add. */
int moe_route(const moe_shape_t* shape, const void* x, const float* w_router,
              const float* logits_in, const float* bias, float* logits_out,
              int32_t* topk_idx, float* topk_gate, int32_t* counts, int32_t* nffn_hist,
              float* zgate, void* ws, size_t ws_bytes, void* stream);

/* The router weight in the tensor cores' format, once, at load time (bf16 layers):
 * w_packed = [hi | mid | lo] per expert row, three bf16 parts with hi + mid + lo == w
 * exactly (hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid)). moe_route splits
 * w_router like this on every call; moe_route_packed takes the packed weight instead.
 *   w_router   device [E, H] fp32
 *   w_packed   device [E, 3H] bf16, written
 * MOE_ERR_UNSUPPORTED for fp32 layers (their router runs on the CUDA cores). */
int moe_router_pack(const moe_shape_t* shape, const float* w_router, void* w_packed,
                    void* stream);

/* moe_route with the router weight from moe_router_pack (bf16 layers; the logits are
 * computed, there is no logits_in). Same outputs, bit for bit. */
int moe_route_packed(const moe_shape_t* shape, const void* x, const void* w_packed,
                     const float* bias, float* logits_out, int32_t* topk_idx, float* topk_gate,
                     int32_t* counts, int32_t* nffn_hist, float* zgate, void* ws, size_t ws_bytes,
                     void* stream);

/* Permutation of the FFN picks into expert-contiguous groups. Group e holds, in ascending
 * token order, the rows of the tokens that picked e; groups follow in expert order.
 *   topk_idx   device [T, K] int32            from moe_route
 *   topk_gate  device [T, K] fp32
 *   zgate      device [T] fp32                used only when out_acc != NULL
 *   x          device [T, H] dtype
 *   offsets    device [n_ffn + 1] int32       exclusive scan of the FFN experts' counts;
 *                                             offsets[n_ffn] = R, the number of FFN rows
 *   perm_token device [T * K] int32           token of each row; entries >= R unwritten
 *   row_of     device [T, K] int32            row of each pick, -1 for zero experts
 *   row_gate   device [T * K] fp32            gate of each row
 *   x_perm     device [T * K + 128, H] dtype  x[perm_token[r]] in row r, or NULL: no copy
 *              or NULL                        (bf16 layers can let moe_grouped_ffn gather
 *                                             the rows from x instead, which saves this
 *                                             buffer but makes the gate/up GEMM slower);
 *                                             the 128 extra rows are read (never written)
 *                                             by the GEMM
 *   out_acc    device [T, H] fp32 or NULL     if given, set to zgate[t] * x[t]: the
 *                                             zero-computation experts' term, ready for
 *                                             the fused combine
 * Every expert index is checked on the device; one outside [0, E) sets the status word to
 * MOE_ERR_DEVICE_CHECK and that pick is dropped. Bit-reproducible. */
int moe_permute(const moe_shape_t* shape, const int32_t* topk_idx, const float* topk_gate,
                const float* zgate, const void* x, int32_t* offsets, int32_t* perm_token,
                int32_t* row_of, float* row_gate, void* x_perm, float* out_acc, void* ws,
                size_t ws_bytes, void* stream);

/* Grouped SwiGLU FFN over the expert groups (report §2.4: intermediate I per expert).
 *   x          device [T, H] dtype            token activations; read when x_perm is NULL
 *   x_perm     device [T * K + 128, H] dtype  from moe_permute, or NULL (bf16 only): the
 *              or NULL                        gate/up GEMM then gathers row r from
 *                                             x[perm_token[r]] with TMA four-row gathers
 *                                             (no x_perm buffer, but about 3x slower gate/up
 *                                             GEMM on B200: 32 gathers per k-block)
 *   offsets    device [n_ffn + 1] int32
 *   w_gate_up  device [n_ffn, 2I, H] dtype    rows [0, I) gate, rows [I, 2I) up
 *   w_down     device [n_ffn, H, I] dtype
 *   perm_token device [T * K] int32           (fused combine, or x_perm NULL)
 *   row_gate   device [T * K] fp32            (fused combine only)
 *   h          device [T * K + 128, I] dtype  receives silu(x W_g^T) * (x W_u^T)
 *   y_perm     device [T * K + 128, H] dtype  deterministic combine: receives y = h W_d^T
 *   out_acc    device [T, H] fp32             fused combine: out_acc[perm_token[r]] +=
 *                                             s * row_gate[r] * y[r] (atomic fp32 adds)
 *   gu_out     device [T * K + 128, 2I] bf16  or NULL (bf16 layers only): also receives
 *              or NULL                        G = x W_g^T (columns [0, I)) and U = x W_u^T
 *                                             (columns [I, 2I)) of every row, rounded to
 *                                             bf16, for moe_backward (a training forward)
 * bf16 runs on the tensor cores (tcgen05, fp32 accumulate, h rounded to bf16); fp32 runs
 * a plain fp32 kernel. The call reads the row counts on the device: it never waits. */
int moe_grouped_ffn(const moe_shape_t* shape, const void* x, const void* x_perm,
                    const int32_t* offsets, const void* w_gate_up, const void* w_down,
                    const int32_t* perm_token, const float* row_gate, void* h, void* y_perm,
                    float* out_acc, void* gu_out, void* ws, size_t ws_bytes, void* stream);

/* Combine (report §2.1: zero-computation experts contribute g * x).
 * Fused: out = out_acc rounded to dtype. Deterministic: out[t] = sum over the FFN slots k
 * in slot order of s * g_k * y_perm[row_of[t, k]], then + zgate[t] * x[t], in fp32,
 * rounded once to dtype. Unused pointers of the other mode may be NULL.
 *   out        device [T, H] dtype */
int moe_combine(const moe_shape_t* shape, const void* x, const void* y_perm,
                const float* out_acc, const float* topk_gate, const int32_t* row_of,
                const float* zgate, void* out, void* stream);

/* Sets pid_state for a controller that starts from `bias`: b0 = bias[0, n_ffn),
 * integral = 0, prev_err = 0.
 *   bias       device [E] fp32
 *   pid_state  device [3 * n_ffn] fp32: b0, then integral, then prev_err */
int moe_pid_init(const moe_shape_t* shape, const float* bias, float* pid_state, void* stream);

/* One PID step on the FFN experts' biases from the batch histogram (report §2.1.1,
 * Fig. 3; zero experts excluded, report §2.1.2). In fp32, in this order, without fused
 * multiply-add, for i < n_ffn:
 *   f = counts[i] / T;  tau = (target_ratio * K) / n_ffn;  e = tau - f;
 *   I += e;  D = e - prev;  b = ((b0 + kp*e) + ki*I) + kd*D;  prev = e;  bias[i] = b.
 * bias[n_ffn, E) is never written.
 *   counts     device [E] int32,  nffn_hist device [K + 1] int32
 *   bias       device [E] fp32, updated in place
 *   pid_state  device [3 * n_ffn] fp32, updated
 *   stats_out  device [8] fp32 or NULL: FFN activation ratio, mean and std of FFN picks
 *              per token, max/mean FFN-expert load, FFN experts hit, zero-expert share of
 *              all picks, mean |e|, max |e|. */
int moe_pid_bias_update(const moe_pid_t* pid, const moe_shape_t* shape, const int32_t* counts,
                        const int32_t* nffn_hist, float* bias, float* pid_state,
                        float* stats_out, void* stream);

/* ---- backward ---------------------------------------------------------------------------- */

/* Bytes of workspace moe_backward needs: G|U of the FFN rows, dy, dG|dU (bf16,
 * [T * K + 128, ...] each), dx_perm (fp32 [T * K + 128, H]), the picks' gate gradients,
 * the logit gradient in three bf16 parts and W_r in bf16. */
int moe_backward_workspace_size(const moe_shape_t* shape, size_t* bytes);

/* Backward of the layer (LongCat-Flash Technical Report digest, Key claims, report §2.1
 * and §2.4: the combined pool and its SwiGLU experts), differentiated with the expert
 * selection held fixed (it is piecewise constant) and no gradient to the selection bias
 * (it only steers selection and is set by the PID, report §2.1.1):
 *   dy = s g_k dout_t (FFN rows),  d_gate = s <dout_t, y> (FFN) or <dout_t, x_t> (zero),
 *   dh = dy W_d[e], dG = dh U silu'(G), dU = dh silu(G),
 *   d_down[e] = sum dy h^T, d_gate_up[e] = sum [dG; dU] x^T, dx_t = sum W_gu[e]^T [dG; dU]
 *   + zgate_t dout_t + dL_t W_r with dL = p (dp - <p, dp>), d_router = dL^T x.
 * bf16 layers only (MOE_ERR_UNSUPPORTED otherwise). The inputs are those of a forward in
 * the deterministic combine mode on the same batch (moe_route, moe_permute with x_perm,
 * moe_grouped_ffn keeping h and y_perm):
 *   dout       device [T, H] bf16             gradient of the layer output
 *   x          device [T, H] bf16
 *   w_router   device [E, H] fp32;  w_gate_up [n_ffn, 2I, H], w_down [n_ffn, H, I] bf16
 *   logits     device [T, E] fp32             the logits the batch was routed with
 *   topk_idx, topk_gate, offsets, row_of      moe_route / moe_permute outputs
 *   x_perm, h, y_perm   device [T * K + 128, H | I | H] bf16
 *   gu         device [T * K + 128, 2I] bf16  G | U saved by moe_grouped_ffn's gu_out, or
 *              or NULL                        NULL: the call recomputes them (x_perm W_gu^T,
 *                                             the same kernels and rounding, so the results
 *                                             are the same bits either way)
 *   dx         device [T, H] fp32             receives d out / d x
 *   d_router   device [E, H] fp32             receives d / d W_r
 *   d_gate_up  device [n_ffn, 2I, H] fp32     receives d / d W_gu of every expert with
 *   d_down     device [n_ffn, H, I] fp32      rows; experts without rows are not written
 *   ws         device, >= moe_backward_workspace_size bytes, zeroed before first use
 * Every GEMM runs on the tensor cores (bf16 in, fp32 accumulate): the expert GEMMs with
 * dy, G, U, dG, dU rounded to bf16; d_router from the logit gradient split exactly into
 * three bf16 parts (exact products with the bf16 x); the router's share of dx from
 * bf16(dL) and bf16(W_r). bf16 layers with E a multiple of 8 (MOE_ERR_UNSUPPORTED
 * otherwise). Other errors as for the other calls; device-side timeouts go to the status
 * word at the start of ws. */
int moe_backward(const moe_shape_t* shape, const void* dout, const void* x,
                 const float* w_router, const void* w_gate_up, const void* w_down,
                 const float* logits, const int32_t* topk_idx, const float* topk_gate,
                 const int32_t* offsets, const int32_t* row_of, const void* x_perm,
                 const void* h, const void* y_perm, const void* gu, float* dx, float* d_router,
                 float* d_gate_up, float* d_down, void* ws, size_t ws_bytes, void* stream);

/* Device-level load-balance loss of one batch, forward value (LongCat-Flash Technical
 * Report digest, Key claims, report §2.1.1 / §2.1.2 Eqs. 3-5: DeepSeek-V3's balance loss
 * with every zero-computation expert in one virtual group; the equations are not
 * printed, so this is the form read from that description):
 *   f_i = E * counts[i] / (K * T),   P_i = (1/T) * sum_t softmax(logits[t])[i]
 *   loss = sum_{i < n_ffn} f_i * P_i + mean_{i >= n_ffn}(f_i) * sum_{i >= n_ffn} P_i
 * A balanced batch gives 1; the loss weight is the caller's. Sums in double, fixed
 * order (deterministic); T == 0 gives loss 0.
 *   logits     device [T, E] fp32             the router logits (moe_route's logits_out
 *                                             or the logits_in it was given)
 *   counts     device [E] int32               moe_route's counts for the same batch
 *   prob_mean  device [E] fp32 or NULL        receives P
 *   loss       device [1] fp32                receives the loss
 *   ws         device scratch, >= moe_scratch_size bytes
 * Errors: MOE_ERR_INVALID_ARG for a NULL pointer, MOE_ERR_ALIGNMENT for a device pointer
 * that is not 16-byte aligned (loss needs none), MOE_ERR_WORKSPACE for a short workspace,
 * MOE_ERR_CUDA for a failed launch. */
int moe_lb_loss(const moe_shape_t* shape, const float* logits, const int32_t* counts,
                float* prob_mean, float* loss, void* ws, size_t ws_bytes, void* stream);

/* The whole layer: moe_route, moe_permute, moe_grouped_ffn and moe_combine on `stream`,
 * with every intermediate in `ws` (>= moe_workspace_size bytes). topk_idx, topk_gate,
 * counts and nffn_hist are returned so the caller can chain moe_pid_bias_update.
 * logits_in may be NULL (then w_router is used) as in moe_route. */
int moe_forward(const moe_shape_t* shape, const void* x, const float* w_router,
                const float* logits_in, const float* bias, const void* w_gate_up,
                const void* w_down, void* out, int32_t* topk_idx, float* topk_gate,
                int32_t* counts, int32_t* nffn_hist, void* ws, size_t ws_bytes, void* stream);

/* ---- end-to-end runs from host memory ------------------------------------------------------
 * The pages have no counterpart to these calls: they serve a caller whose batches live in
 * host memory (a serving loop), and overlap each batch's PCIe copies with the previous and
 * next batches' layer kernels. A pipeline owns two copy streams and a few events (created
 * by moe_host_pipeline_create, the one place besides moe_read_device_status where the
 * library touches device state outside a stream) and uses the caller's device staging
 * buffers: two slots of x [T, H] dtype, out [T, H] dtype and, optionally, logits [T, E]
 * fp32. Slots alternate per batch, so a buffer is never overwritten while a copy or a
 * kernel still reads it.
 *
 * moe_host_pipeline_create(shape, x_dev, logits_dev, out_dev, stream, &pipe)
 *   x_dev, out_dev  two device pointers each (16-byte aligned), as above
 *   logits_dev      two device pointers, or NULL when no batch passes logits
 *   stream          the stream the layer's kernels run on (the caller's compute stream)
 *   Errors: MOE_ERR_INVALID_ARG (NULL pipe / buffers), MOE_ERR_ALIGNMENT, the shape's
 *   errors, MOE_ERR_NO_DEVICE, MOE_ERR_CUDA (stream or event creation; nothing is kept).
 *
 * moe_host_pipeline_submit(pipe, x_host, logits_in_host, out_host, weights..., ws, ws_bytes)
 *   x_host          host [T, H] dtype, the batch's tokens
 *   logits_in_host  host [T, E] fp32 or NULL: given router logits, as logits_in of moe_route
 *   out_host        host [T, H] dtype, receives the layer's output
 *   w_router ... ws_bytes: as in moe_forward; topk_idx, topk_gate, counts and nffn_hist
 *   are overwritten by every batch (read them on `stream` before the next batch's kernels).
 *   Queues: the copy of x (and logits) into slot n mod 2 on the input copy stream; the
 *   layer (moe_forward) on `stream` after that copy; the copy of out back on the output
 *   copy stream after the layer. The first submit after create or join orders the copy
 *   streams after the work already on `stream`. Host buffers must be page-locked (for
 *   example cudaHostAlloc) for the copies to run asynchronously and overlap; a host
 *   buffer must stay untouched until the batch's output copy has completed (join, then
 *   synchronise `stream`). Every check happens before anything is queued.
 *
 * moe_host_pipeline_join(pipe): makes `stream` wait for every copy queued so far, so that
 *   work or an event recorded on `stream` afterwards follows the last output copy.
 *   Asynchronous.
 * moe_host_pipeline_destroy(pipe): waits for the pipeline's copy streams, releases its
 *   streams and events and frees it. NULL is a no-op. */
typedef struct moe_host_pipeline moe_host_pipeline;

int moe_host_pipeline_create(const moe_shape_t* shape, void* const x_dev[2],
                             float* const logits_dev[2], void* const out_dev[2], void* stream,
                             moe_host_pipeline** pipe);
int moe_host_pipeline_submit(moe_host_pipeline* pipe, const void* x_host,
                             const float* logits_in_host, void* out_host, const float* w_router,
                             const float* bias, const void* w_gate_up, const void* w_down,
                             int32_t* topk_idx, float* topk_gate, int32_t* counts,
                             int32_t* nffn_hist, void* ws, size_t ws_bytes);
int moe_host_pipeline_join(moe_host_pipeline* pipe);
int moe_host_pipeline_destroy(moe_host_pipeline* pipe);

/* ---- allocation-free variant ------------------------------------------------------------
 * The pages have no counterpart to this call: it is moe_permute for callers that cannot
 * give the library a device workspace. Such callers include code running while its
 * stream is captured into a CUDA graph in a capture mode where cudaMalloc is an error,
 * plugins inside a host framework that owns all device memory and only passes tensors
 * in and out, and latency-bound paths that cannot afford a cudaMalloc, which may
 * synchronise the whole device.
 *
 * Arguments and results are exactly those of moe_permute without ws and ws_bytes;
 * x_perm may be NULL as there (the indices and gates only, for the gathered-rows FFN).
 * The scratch is a fixed 4 MiB array in the library's own device memory; each GPU that
 * loads the library keeps it until the process exits. A call needs
 * 1024 + 2 * round_up_1024(n_ffn * ceil(T / 32) * 4) + 4 * n_ffn bytes of it and returns
 * MOE_ERR_WORKSPACE, launching nothing, when the shape needs more (with n_ffn = 512:
 * T <= 32736). The call never calls cudaMalloc, cudaFree or any allocating routine.
 * The first call in a device's context looks up the array's device address there and
 * caches it with that context's unique id: make that first call before any stream
 * capture on that device. A new context on the device (after cudaDeviceReset, say)
 * gets its own lookup on its first call.
 * Every call uses the same array, which keeps what the last call left there. Calls whose
 * GPU work can overlap (unordered streams, several host threads) race on it and give
 * wrong results: order them on one stream. Each call clears the array's status word;
 * that word cannot be read back, so an invalid expert index is dropped (row_of = -1)
 * as in moe_permute but not reported: use moe_permute to get the report. */
int moe_permute_static_scratch(const moe_shape_t* shape, const int32_t* topk_idx,
                               const float* topk_gate, const float* zgate, const void* x,
                               int32_t* offsets, int32_t* perm_token, int32_t* row_of,
                               float* row_gate, void* x_perm, float* out_acc, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H_ */
