/*
 * wina.h -- C ABI of the weight-informed, activation-sparse linear layer for LLM decode
 * (CUDA, sm_100a / B200).
 *
 * The method (WINA gate):
 *   offline:   c_j = || W[:, j] ||_2, the l2 norm of each input column of W [out][in];
 *   per token: score_i = | x_i * c_i |, keep the K largest (ties -> lower index), or,
 *              in the Spark variant, keep { i : v_i > mu + sigma * Phi^-1(1 - s) };
 *              y = W[:, S] x[S], reading only the kept columns of W.
 * Sources, cited by page title and section:
 *   - "WINA: Weight Informed Neuron Activation" article (lsdiaocha.cn, 2025-05-29),
 *     section 一 (the gate: top-K of |x (.) c| with c the column l2 norms of W; K may be
 *     shared or per layer), section 二 (error bound for column-orthogonal W);
 *   - "Spark Transformer: 高效稀疏化大语言模型架构设计", section 2.2 (statistical top-k:
 *     mean, population variance, Gaussian quantile threshold, strict comparison) and
 *     section 3.1 (SVMM: accumulate x_j * W[j] over the active indices only, with W
 *     stored input-major so that W[j] is one contiguous run);
 *   - "哈工大EMNLP 2025论文开源 ... WAS", section on the core innovations (the gate is
 *     applied per component: Q, K, V, O, gate, up and down projections).
 *
 * Conventions (every call):
 *   - Returns wina_status_t; WINA_OK is 0. Arguments are checked on the host before any
 *     launch; a bad argument returns an error code and launches nothing.
 *   - Every pointer argument except those documented as host pointers is a DEVICE
 *     pointer, allocated and owned by the caller. The library allocates no device or
 *     host memory and keeps no state between calls (see wina_workspace_size for the
 *     scratch a call needs). Device pointers must be 16-byte aligned.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).
 *     Launch errors are returned at once (WINA_ERR_CUDA). Errors found on the device
 *     (capacity overflow, a grid-barrier timeout) are written into the optional
 *     caller-owned int32 word `status_dev` (first error wins; 0 = none) and are seen by
 *     the caller after it synchronises. Pass NULL to ignore them.
 *   - Weights are stored input-channel-major: Wt[n][m] = W[m][n]^T, so input channel j
 *     is the contiguous run Wt[j][0..m). wina_pack_in_major produces this layout.
 *   - dtype: WINA_BF16 (bfloat16) or WINA_F32. Products accumulate in float32; outputs y
 *     are float32.
 *   - Inputs must be finite; NaN/Inf inputs are not supported (results unspecified).
 */
#ifndef WINA_H
#define WINA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define WINA_ABI_VERSION 1

/* A cudaStream_t, declared opaquely so this header does not need the CUDA headers. */
typedef struct CUstream_st* wina_stream_t;

typedef enum {
  WINA_OK = 0,
  WINA_ERR_INVALID_ARG = 1,       /* bad size, null or misaligned pointer, k > n, s outside (0,1) */
  WINA_ERR_UNSUPPORTED_DTYPE = 2, /* dtype not in {WINA_F32, WINA_BF16} */
  WINA_ERR_WORKSPACE = 3,         /* workspace smaller than wina_workspace_size() */
  WINA_ERR_CAPACITY = 4,          /* device: more channels passed the threshold than `cap` */
  WINA_ERR_CUDA = 5,              /* a CUDA runtime call failed (no device, launch error) */
  WINA_ERR_TIMEOUT = 6            /* device: a grid-barrier wait gave up after its time limit */
} wina_status_t;

typedef enum { WINA_F32 = 0, WINA_BF16 = 1 } wina_dtype_t;

/* Memory layout of a weight passed to wina_col_norms. */
typedef enum {
  WINA_LAYOUT_OUT_IN = 0, /* W[m][n]: row i is output i (the matrix that multiplies x)   */
  WINA_LAYOUT_IN_MAJOR = 1 /* Wt[n][m]: row j is input channel j (the packed layout)     */
} wina_layout_t;

/* How sparse_ffn_swiglu chooses the kept channels of each projection's input. */
typedef enum {
  WINA_GATE_TOPK = 0,  /* WINA: top-K of |v_i * c_i| with the projection's own c and K */
  WINA_GATE_STAT = 1,  /* Spark: { i : v_i > mu + sigma * Phi^-1(1 - s) } on the signed v */
  WINA_GATE_DENSE = 2  /* no gate: every channel is kept (the dense comparator)          */
} wina_gate_mode_t;

typedef enum {
  WINA_OP_SELECT_TOPK = 0,
  WINA_OP_STAT_THRESHOLD = 1,
  WINA_OP_SPARSE_MATVEC = 2,
  WINA_OP_FFN_SWIGLU = 3,
  WINA_OP_SPARK_FFN = 4,
  WINA_OP_DENSE_FFN = 5
} wina_op_t;

/* The three projections of a SwiGLU FFN, already packed input-major:
 *   wt_gate, wt_up: [d][ffn];  wt_down: [ffn][d];  all of dtype wdt.
 *   c_gate, c_up: float32 [d];  c_down: float32 [ffn]  (column norms of W_gate, W_up,
 *   W_down, as written by wina_col_norms). Only WINA_GATE_TOPK reads the c's. */
typedef struct {
  const void* wt_gate;
  const void* wt_up;
  const void* wt_down;
  wina_dtype_t wdt;
  const float* c_gate;
  const float* c_up;
  const float* c_down;
  int64_t d;
  int64_t ffn;
} wina_ffn_t;

/* Byte offsets, inside the workspace of a sparse_ffn_swiglu call, of the intermediate
 * results it leaves behind (valid after the call completes; read-only diagnostics):
 *   h         float32 [batch][ffn]  h = silu(g) * u, the down projection's input
 *   keep_gate uint8   [batch][d]    1 where the gate projection's input channel was kept
 *   keep_up   uint8   [batch][d]    1 where the up projection's input channel was kept
 *   keep_down uint8   [batch][ffn]  1 where the down projection's input channel was kept
 *   stamps    int64   [16]          single-token kernel only: SM clock (clock64) of CTA 0
 *                                   at its phase boundaries: 0 start, 1 gate/up scores
 *                                   made, 2 kept set found, 3 rows listed, 4 gate/up rows
 *                                   streamed, 5 partial rows stored, 6 first grid barrier
 *                                   passed, 7 its slice of h and the down scores written,
 *                                   8 second barrier passed, 9 down scores loaded, 10 down
 *                                   kept set found, 11 rows listed, 12 down rows streamed,
 *                                   13 partial rows stored, 14 third barrier passed,
 *                                   15 its slice of y written
 *   cta_t     uint64  [CTAs][4]     single-token kernel only: global timer (ns) at which
 *                                   each CTA finished listing its gate/up rows, streaming
 *                                   them, listing its down rows and streaming them       */
typedef struct {
  size_t h;
  size_t keep_gate;
  size_t keep_up;
  size_t keep_down;
  size_t stamps;
  size_t cta_t;
} wina_ffn_ws_view_t;

/* ABI version of the loaded library (WINA_ABI_VERSION at build time). */
int32_t wina_abi_version(void);

/* Test and diagnosis hook (host function): the time limit of each grid-barrier wait of
 * the single-token sparse_ffn_swiglu kernel, for launches made after the call, process-
 * wide; 0 restores the default of 1 s. A wait that exceeds it records WINA_ERR_TIMEOUT in
 * the call's status word and the kernel returns (the workspace must then be zero-filled
 * again before its next use). */
void wina_set_wait_limit_ns(uint64_t ns);

/* Static description of a status code (host pointer to a constant string). */
const char* wina_status_string(wina_status_t status);

/* Standard normal quantile Phi^-1(p) for 0 < p < 1, in double precision (host function;
 * no device needed). The Spark threshold uses z = Phi^-1(1 - s) ("Spark Transformer",
 * section 2.2: Phi is the standard normal CDF). Computed by Newton iteration on
 * Phi(z) = erfc(-z / sqrt 2) / 2 from a bracketing start; |error| ~ 1e-15.
 * Returns NaN for p outside (0, 1). */
double wina_normal_quantile(double p);

/* Bytes of device scratch that `op` needs for the given sizes (0 if none). The
 * workspace is owned by the caller, must be zero-filled before its first use, and may
 * be reused by later calls of the same op with the same sizes, on the same device and
 * stream; the library leaves it in
 * a reusable state unless a call ended in WINA_ERR_TIMEOUT, after which it must be
 * zero-filled again. Concurrent calls need distinct workspaces.
 *   WINA_OP_SPARSE_MATVEC: n = in-features, m = out-features, k = max kept per token,
 *                          batch = tokens.
 *   WINA_OP_FFN_SWIGLU:    n = d, m = ffn, k ignored, batch = tokens.
 *   WINA_OP_SPARK_FFN:     n = d, m = ffn, k ignored, batch = 1.
 *   WINA_OP_DENSE_FFN:     n = d, m = ffn, k ignored, batch = 1.
 *   WINA_OP_SELECT_TOPK, WINA_OP_STAT_THRESHOLD: 0.                                  */
size_t wina_workspace_size(wina_op_t op, int64_t n, int64_t m, int64_t k, int64_t batch);

/* Offsets of the diagnostic views inside a sparse_ffn_swiglu workspace (host function).
 * Returns WINA_ERR_INVALID_ARG for non-positive sizes or a null `out`. */
wina_status_t wina_ffn_ws_view(int64_t d, int64_t ffn, int64_t batch, wina_ffn_ws_view_t* out);

/* Offline: transpose W[m][n] (output-major, the matrix that multiplies x) into the
 * input-channel-major Wt[n][m] used by every product below ("Spark Transformer",
 * section 3.1: SVMM reads W[j] as a whole for each active j). Bit-exact copy.
 *   W:  device, m*n elements of dt, row-major [m][n];  Wt: device, [n][m], same dtype.
 *   m, n >= 1. W and Wt must not overlap. */
wina_status_t wina_pack_in_major(const void* W, wina_dtype_t dt, int64_t m, int64_t n, void* Wt,
                                 wina_stream_t stream);

/* Offline: column l2 norms c_j = sqrt(sum_i W[i][j]^2) for j < n ("WINA" article,
 * section 一: c holds the l2 norm of each column of W). Squares are summed in float64,
 * the square root is taken in float64 and rounded once to float32.
 *   W: device; layout WINA_LAYOUT_OUT_IN means W[m][n]; WINA_LAYOUT_IN_MAJOR means the
 *      packed Wt[n][m] (the norm of row j of Wt). m = out-features, n = in-features.
 *   c: device float32 [n] (written). */
wina_status_t wina_col_norms(const void* W, wina_dtype_t dt, int64_t m, int64_t n, wina_layout_t layout,
                             float* c, wina_stream_t stream);

/* Per-token top-K gate ("WINA" article, section 一): for each of `batch` tokens,
 * score_i = |x_i * c_i| (one float32 multiply; c == NULL gives the magnitude-only gate
 * |x_i| of TEAL/CATS), keep the k largest scores, ties at the k-th value to the lower
 * index.
 *   x:      device [batch][n] of xdt;  c: device float32 [n] or NULL.
 *   idx:    device int32 [batch][k]: kept indices of each token, ascending.
 *   xs:     device float32 [batch][k] or NULL: x at the kept indices (the stored value,
 *           widened to float32), in the order of idx.
 *   scores: device float32 [batch][n] or NULL: the score vector.
 *   1 <= n <= 32768, 0 <= k <= n, batch >= 1. */
wina_status_t wina_select_topk(const void* x, wina_dtype_t xdt, const float* c, int64_t n, int64_t k,
                               int64_t batch, int32_t* idx, float* xs, float* scores, wina_stream_t stream);

/* Spark statistical top-k ("Spark Transformer", section 2.2) for each of `batch`
 * vectors v_b of length n: mu = mean(v), sigma^2 = mean((v - mu)^2) (divisor n),
 * t = mu + sigma * Phi^-1(1 - s), keep { i : v_i > t } (strict, signed). The mean and
 * variance are accumulated in float64 in one pass (per-thread Welford, Chan's pairwise
 * merge across threads); the comparison is made in float64.
 *   v:     device [batch][n] of vdt.   s: keep fraction, 0 < s < 1.
 *   idx:   device int32 [batch][cap]: kept indices ascending (the first min(count, cap)).
 *   xs:    device float32 [batch][cap] or NULL: v at the kept indices.
 *   count: device int32 [batch]: the true number of kept channels (may exceed cap).
 *   t:     device float32 [batch] or NULL: the threshold, rounded to float32.
 *   cap >= 0. If a count exceeds cap only cap indices are written and WINA_ERR_CAPACITY
 *   is recorded in *status_dev. 1 <= n <= 32768. */
wina_status_t stat_topk_threshold(const void* v, wina_dtype_t vdt, int64_t n, double s, int64_t batch,
                                  int32_t* idx, float* xs, int32_t* count, float* t, int64_t cap,
                                  int32_t* status_dev, wina_stream_t stream);

/* Sparse product over the kept channels ("Spark Transformer", section 3.1, SVMM):
 *   y[b][:] = sum over r < k_b of xs[b][r] * Wt[idx[b][r]][:]      for b < batch,
 * reading only the kept rows of the input-major weight.
 *   One token: the grid is split into column groups x row groups; a CTA streams its
 *   column group's slice of every kept row of its row group (rank = row group modulo
 *   the number of row groups), and the last CTA of a column group adds the group's few
 *   partial rows in a fixed order. No grid barrier; bit-reproducible.
 *   Two or three tokens, or f32 weights: the co-resident grid is shared among the
 *   tokens; token b gets P = grid / batch CTAs (at least one), which split its kept rows
 *   and, when P > 1, sum their partial rows in a fixed order after a grid barrier
 *   (bit-reproducible). Each token reads its own kept rows.
 *   Four or more tokens with bf16 weights: per block of up to 256 tokens, the union U
 *   of their kept rows is read once, whatever the number of tokens that keep each row,
 *   and Y = X~ . Wt[U,:] runs on the tcgen05 tensor cores (X~: each token's value at
 *   each union row or 0, split into bf16 parts that reproduce it to float32 precision);
 *   the split of U over CTAs adds into y with float atomics, so the last bits of y may
 *   differ from call to call.
 *   Wt:    device [n][m] of wdt (m % 8 == 0 and m <= 32768 for bf16; m % 4 == 0 and
 *          m <= 16384 for f32).
 *   idx:   device int32 [batch][ld_idx]: kept input channels of each token (any order;
 *          distinct within a token; each < n).
 *   xs:    device float32 [batch][ld_idx]: the input values at those channels.
 *   k:     kept count of every token (0 <= k <= ld_idx), or -1 to read each token's
 *          count from the device array `count` [batch] (as written by
 *          stat_topk_threshold; counts above ld_idx are clamped to ld_idx).
 *   y:     device float32 [batch][m] (written; does not alias the inputs).
 *   ws:    device scratch of at least wina_workspace_size(WINA_OP_SPARSE_MATVEC, n, m,
 *          ld_idx, batch) bytes (see that function for its lifetime rules).
 *   status_dev: optional device int32 word for WINA_ERR_TIMEOUT. */
wina_status_t sparse_matvec(const void* Wt, wina_dtype_t wdt, int64_t n, int64_t m, const int32_t* idx,
                            const float* xs, int64_t k, const int32_t* count, int64_t ld_idx, int64_t batch,
                            float* y, void* ws, size_t ws_bytes, int32_t* status_dev, wina_stream_t stream);

/* sparse_matvec for callers that cannot supply a workspace. The pages describe no
 * such entry point; it exists for code that runs where device allocation is not an
 * option (a framework that owns a fixed device memory pool, a latency-critical loop in
 * which cudaMalloc could synchronise the device, a plugin that is only handed input and
 * output buffers). Same arguments and results as sparse_matvec, minus ws / ws_bytes,
 * always computed by the split-K product (every token on its own CTAs, no union): the
 * scratch (a barrier word pair and the split-K partial rows) lives in a fixed
 * 8 MiB + 256 B array of device memory declared by the library, which every GPU that
 * loads the library holds until the process exits. It allocates nothing.
 *   Limit: when batch is smaller than the co-resident grid (148 CTAs on a B200), a
 *   token is split over several CTAs whose partial rows live in the 2^21-float array,
 *   so batch * m <= 1,048,576 is required (at least two partial rows per token);
 *   larger calls return WINA_ERR_INVALID_ARG. With batch at least the grid, each
 *   token has its own CTA, the array is not used and any size is accepted.
 *   Every call looks up the array's device address in the current device's context
 *   (cudaGetSymbolAddress, a cheap query), so the entry point stays valid across
 *   cudaDeviceReset; the first call on a device may also load the library's device
 *   code, so make it before any stream capture.
 *   Every call clears the barrier words on `stream` and then reuses the same array:
 *   calls that overlap on the GPU (other streams, other threads) race and must not
 *   be issued. */
wina_status_t sparse_matvec_noalloc(const void* Wt, wina_dtype_t wdt, int64_t n, int64_t m, const int32_t* idx,
                                    const float* xs, int64_t k, const int32_t* count, int64_t ld_idx,
                                    int64_t batch, float* y, int32_t* status_dev, wina_stream_t stream);

/* SwiGLU FFN decode with the gate on every projection ("WAS" article: the gate is
 * applied per component, gate/up/down among them; "WINA" article, section 一: each
 * projection uses the column norms of its own weight and its own K):
 *   S_g = gate(x, c_gate, k_gate);  g = W_gate[:, S_g] x[S_g]
 *   S_u = gate(x, c_up,   k_up);    u = W_up[:, S_u]   x[S_u]
 *   h   = silu(g) * u                (float32; silu(g) = g / (1 + e^-g))
 *   S_d = gate(h, c_down, k_down);  y = W_down[:, S_d] h[S_d]
 * With WINA_GATE_STAT every gate is the Spark threshold with keep fraction s on the
 * projection's signed input (k_* ignored; gate and up then share one kept set); with
 * WINA_GATE_DENSE every channel is kept.
 * One token (d, ffn <= 16384) runs as one persistent cooperative kernel with one CTA of
 * 1024 threads per SM. The SMs form column groups of the ffn outputs, each with four row
 * groups split between gate and up: every SM selects its projection's kept channels
 * itself (the keys in registers, a radix select on their bits), takes the kept rows of
 * its row group (every fourth, or so, in ascending order) and streams its column group's
 * slice of them with 16-byte loads into a partial row; the last SM of a column group adds
 * the group's partials in a fixed order and writes h and the down scores for the slice.
 * After the one grid barrier every SM selects the down kept set and streams its slice of
 * its row group's down rows the same way; the last SM of each column group adds those
 * partials into y. The barrier wait is bounded in time. Kept sets are exact and every
 * sum is taken in a fixed order, so repeated calls give identical bits. Several tokens
 * (or wider shapes) run as a sequence of the batched calls above, the up projection on a
 * side stream of the library beside the gate projection (one stream and two events per
 * device, created on the first such call outside stream capture and joined back to
 * `stream` by events, so graph capture of `stream` includes them).
 *   f:   host pointer to the weight descriptor (read during the call only).
 *   x:   device [batch][d] of xdt.   y: device float32 [batch][d] (written).
 *   k_gate, k_up in [0, d]; k_down in [0, ffn] (WINA_GATE_TOPK).  0 < s < 1 (STAT).
 *   ws:  device scratch of at least wina_workspace_size(WINA_OP_FFN_SWIGLU, d, ffn, 0,
 *        batch) bytes; after the call it holds the views of wina_ffn_ws_view.
 *   d % 8 == 0 and ffn % 8 == 0 (bf16) or % 4 (f32); d, ffn <= 32768 (bf16) or
 *   <= 16384 (f32). */
wina_status_t sparse_ffn_swiglu(const wina_ffn_t* f, const void* x, wina_dtype_t xdt, int64_t batch,
                                wina_gate_mode_t mode, int64_t k_gate, int64_t k_up, int64_t k_down, double s,
                                float* y, void* ws, size_t ws_bytes, int32_t* status_dev, wina_stream_t stream);

/* The Spark FFN as a key-value lookup ("Spark Transformer", section 2.1: y = sum_i
 * f(q . k_i) v_i, with the statistical top-k of section 2.2 choosing the neurons), for a
 * SwiGLU FFN and one token:
 *   g   = W_gate x                 (every neuron's score: dense, all of W_gate is read)
 *   S   = { i : g_i > mu + sigma * Phi^-1(1 - s) }    (mean, population variance of g)
 *   h_i = silu(g_i) * (W_up[i] . x)           for i in S   (only the selected rows)
 *   y   = sum over i in S of h_i * W_down[:, i]            (only the selected columns)
 *   W_gate, W_up: device [ffn][d] OUTPUT-major (row i is neuron i's key / up row);
 *   Wt_down: device [ffn][d] input-major (wina_pack_in_major of W_down [d][ffn]);
 *   x: device [d] of xdt;  y: device float32 [d] (written);
 *   g_out: device float32 [ffn] or NULL: the scores g (float32);
 *   idx: device int32 [ffn]: the selected neurons ascending (the first *count valid);
 *   count: device int32 [1]: |S|;  0 < s < 1;
 *   ws: device scratch of wina_workspace_size(WINA_OP_SPARK_FFN, d, ffn, 0, 1) bytes.
 *   d % 8 == 0 (bf16) or % 4 (f32); d, ffn <= 32768. */
wina_status_t spark_ffn_swiglu(const void* W_gate, const void* W_up, const void* Wt_down, wina_dtype_t wdt,
                               int64_t d, int64_t ffn, const void* x, wina_dtype_t xdt, double s, float* y,
                               float* g_out, int32_t* idx, int32_t* count, void* ws, size_t ws_bytes,
                               int32_t* status_dev, wina_stream_t stream);

/* The dense comparator: the unsparsified layer y = W x (every channel kept), on the
 * OUTPUT-major weight W[m][n] (the matrix that multiplies x, unpacked). The weights are
 * streamed as one flat sequence of 512-byte slabs split evenly over all warps, x staged in
 * shared memory; a row split between two warps is completed by two atomic adds onto a
 * zeroed y, which gives the same bits in either order. Batch 1. Rows that are not a whole
 * number of slabs (n not a multiple of 256 for bf16, 128 for f32), or whose x does not fit
 * in 96 KB of shared memory, take a warp-per-row kernel that reads x through L1.
 *   W:    device [m][n] of wdt (n % 8 == 0 for bf16, % 4 for f32), 16-byte aligned.
 *   x:    device [n] of xdt.   y: device float32 [m] (written).
 *   xbuf: device float32 [n] scratch (x widened; used by the long-row kernel only),
 *         16-byte aligned. */
wina_status_t wina_dense_matvec(const void* W, wina_dtype_t wdt, int64_t m, int64_t n, const void* x,
                                wina_dtype_t xdt, float* y, float* xbuf, wina_stream_t stream);

/* The dense comparator of sparse_ffn_swiglu: y = W_down (silu(W_gate x) * (W_up x)) with
 * every channel kept, on the output-major weights W_gate, W_up [ffn][d] and W_down
 * [d][ffn]. One cooperative launch of two 512-thread CTAs per SM: W_gate streamed into g
 * by half of the warps and W_up into u by the other half, each as equal flat ranges of
 * 512-byte slabs (by atomic adds, at most two per element, so the bits do not depend on
 * timing), y zeroed on the way; a grid barrier, with the first down loads already in
 * flight; h = silu(g) * u staged by every CTA in shared memory; W_down streamed into y.
 * g and u live in one of two workspace copies used by alternate calls: each call zeroes
 * the copy the next call adds into.
 * Rows that are not a whole number of slabs (d or ffn not a multiple of 256 for bf16, 128
 * for f32), or whose x or h does not fit in 96 KB of shared memory, take three
 * warp-per-row launches instead. Batch 1.
 *   x: device [d] of xdt;  y: device float32 [d] (written);
 *   ws: device scratch of at least wina_workspace_size(WINA_OP_DENSE_FFN, d, ffn, 0, 1)
 *       bytes, zero-filled before first use (it holds the grid barrier), 16-byte aligned;
 *   status_dev: optional device int32; WINA_ERR_TIMEOUT is recorded there if a grid
 *       barrier wait runs out (y is then incomplete and ws must be zero-filled again). */
wina_status_t wina_dense_ffn_swiglu(const void* W_gate, const void* W_up, const void* W_down, wina_dtype_t wdt,
                                    int64_t d, int64_t ffn, const void* x, wina_dtype_t xdt, float* y, void* ws,
                                    size_t ws_bytes, int32_t* status_dev, wina_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Double Sparsity decode attention ("大模型DoubleSparse稀疏化技术原理", section 技术原理:
 * 离线校准 and 在线前向计算). Caches are [B][Hkv][Tmax][dh] (keys, values) and
 * [B][Hkv][Tmax][r] (labels), in the key cache's dtype (bf16 or f32), token t of sequence
 * b valid for t < seq_len[b]; channels is [Hkv][r] int32 (the important channels of each
 * key/value head, ascending). All pointers are device pointers owned by the caller.
 * --------------------------------------------------------------------------------- */

/* Offline calibration, K-outlier strategy: absmean[g][c] = mean over every sequence's
 * valid tokens of |K[b][g][t][c]| (float64 sums, rounded once to float32). The r
 * channels of largest mean are then picked per head with wina_select_topk(absmean, NULL
 * c, n = dh, k = r, batch = Hkv), which lists them ascending, ties to the lower channel.
 *   seq_len: device int32 [B];  absmean: device float32 [Hkv][dh] (written). */
wina_status_t ds_channel_absmean(const void* K, wina_dtype_t kdt, int64_t B, int64_t Hkv, int64_t Tmax, int64_t dh,
                                 const int32_t* seq_len, float* absmean, wina_stream_t stream);

/* The label cache: label[b][g][t][j] = K[b][g][t][channels[g][j]] for t0 <= t < t1 and
 * t < seq_len[b] (a prefill passes [0, T), a decode step the new token [T-1, T)); other
 * entries are left as they are. 0 <= t0 <= t1 <= Tmax, 1 <= r <= dh. */
wina_status_t ds_label_build(const void* K, wina_dtype_t kdt, int64_t B, int64_t Hkv, int64_t Tmax, int64_t dh,
                             const int32_t* seq_len, const int32_t* channels, int64_t r, int64_t t0, int64_t t1,
                             void* label, wina_stream_t stream);

/* Bytes of dynamic shared memory ds_decode_attention needs per CTA (host function): the
 * call is refused (WINA_ERR_INVALID_ARG) above 225 KB, i.e. for Tmax + 2 min(k, Tmax)
 * beyond about 51 K entries. */
size_t ds_decode_smem_bytes(int64_t Tmax, int64_t dh, int64_t k);

/* One decode step of Double Sparsity attention for B sequences and Hq query heads (query
 * head h reads key/value head h / (Hq / Hkv)); one CTA per (sequence, query head):
 *   1. q[C]: the query's important channels (C = channels[g]);
 *   2. s_t = sum over j of q[C_j] * label[t][j] for every valid token t, in float32, each
 *      product rounded and added in the order j = 0..r-1;
 *   3. S = the min(k, seq_len) tokens of largest s (signed, ties to the lower token),
 *      ascending; out = sum over t in S of p_t V[t] with p = softmax over S of
 *      (q . K[t]) * scale (float32; scale <= 0 means 1 / sqrt(dh)).
 *   q: device [B][Hq][dh] of qdt;  out: device float32 [B][Hq][dh] (written; zeros when
 *   min(k, seq_len) = 0);  idx_out: optional device int32 [B][Hq][k], the first
 *   min(k, seq_len[b]) entries written;  scores_out: optional device float32
 *   [B][Hq][Tmax], the first seq_len[b] written.
 *   dh in {32, 64, 128, 256}; r a multiple of 8 (bf16) or 4 (f32), r <= dh; K, V, label
 *   16-byte aligned. A seq_len outside [0, Tmax] records WINA_ERR_INVALID_ARG in
 *   status_dev (optional) and is clamped. Deterministic: fixed-order sums throughout. */
wina_status_t ds_decode_attention(const void* q, wina_dtype_t qdt, const void* K, const void* V, const void* label,
                                  wina_dtype_t kvdt, const int32_t* channels, int64_t B, int64_t Hq, int64_t Hkv,
                                  int64_t Tmax, int64_t dh, int64_t r, const int32_t* seq_len, int64_t k,
                                  float scale, float* out, int32_t* idx_out, float* scores_out,
                                  int32_t* status_dev, wina_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* WINA_H */
