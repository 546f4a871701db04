/*
 * int8mm.h — C ABI of libint8mm.so, the B200 (sm_100a) LLM.int8()
 * mixed-precision decomposed matmul
 *
 *     Y = X W,   X fp16 [M,K] (activations),  W fp16 [K,N] (weights)
 *
 * computed as in "LLM.int8(): 8-bit Matrix Multiplication for Transformers at
 * Scale" (Dettmers et al., 2022), following these web pages about it:
 *   "LLM.int8() — 大模型激活值里藏着几个超大异常通道" (estelledc.github.io),
 *       方法1 (vector-wise quantisation) and 方法2 (mixed-precision decomposition);
 *   "AI 十大核心论文解读: LLM.int8()" (developer.aliyun.com), §2.2 and the
 *       Fig. 2 caption;
 *   "LLM.int8()" (brain.gartu.xyz), "La solution", "Seuil de détection α",
 *       "Vector-wise INT8 Quantization".
 *
 *  1. O = { j : max_i |X[i,j]| > alpha }   (outlier feature columns; strict >)
 *  2. c_x[i] = 127 / max_{j not in O} |X[i,j]|,  Xq[i,j] = rne(X[i,j] c_x[i])
 *     for j not in O and 0 for j in O;  c_w[j] = 127 / max_k |W[k,j]| over all
 *     K rows,  Wq[k,j] = rne(W[k,j] c_w[j]).  Codes are clamped to [-127, 127],
 *     rne rounds an fp32 product to the nearest integer, ties to even; an
 *     all-zero vector gets scale 0 and codes 0.
 *  3. Acc = Xq Wq  (int8 x int8 -> int32, exact)
 *  4. Y[i,j] = fp16( Acc[i,j] / (c_x[i] c_w[j]) + sum_{k in O} X[i,k] W[k,j] )
 *     with the fp16 outlier product accumulated in fp32.
 *
 * Every pointer argument named *_dev is a device pointer on the current CUDA
 * device; `stream` is a cudaStream_t (NULL = the legacy default stream).
 * All work is enqueued on `stream`; no call below synchronises the host
 * unless its comment says so.  The library never frees caller memory.
 * A handle is not safe for concurrent use from several host threads.
 *
 * Errors: argument errors are detected on the host before anything is
 * enqueued; they return a non-zero status and set int8mm_last_error().
 * A CUDA launch or allocation error returns INT8MM_ERR_CUDA (or
 * INT8MM_ERR_OOM).  A device-side wait that exceeded its time limit is
 * reported later through int8mm_get_status().  NaN or Inf in X or W gives an
 * unspecified Y (the pages assume finite activations); it is not checked.
 */
#ifndef INT8MM_H
#define INT8MM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct int8mm_weight* int8mm_weight_t; /* opaque, owned by the library */

typedef enum {
  INT8MM_OK = 0,
  INT8MM_ERR_INVALID_ARG = 1,       /* null pointer, bad size, NaN alpha, freed handle */
  INT8MM_ERR_UNSUPPORTED_SHAPE = 2, /* K or N not a multiple of 16, K > 65536, ... */
  INT8MM_ERR_ALIGNMENT = 3,         /* a pointer not 16-byte aligned */
  INT8MM_ERR_OOM = 4,               /* device allocation failed */
  INT8MM_ERR_CUDA = 5,              /* a CUDA runtime/driver call failed */
  INT8MM_ERR_TIMEOUT = 6,           /* a device wait ran out of time (see get_status) */
  INT8MM_ERR_OUTLIER_CAP = 7        /* a forward found more outlier columns than a static
                                       weight holds (see get_status) */
} int8mm_status;

/* Shape limits: 16 <= K <= 65536 with K % 16 == 0 (K <= 133144 keeps the
 * int32 accumulator exact; the row kernel holds a row in registers up to
 * 65536); 16 <= N < 2^31 with N % 16 == 0; 0 <= M < 2^31. */
#define INT8MM_MAX_K 65536

/*
 * Prepare a weight (step 2 for W; "LLM.int8() — 大模型激活值里藏着几个超大异常通道",
 * 方法1: one normalisation constant per column of the weight matrix).
 *
 * W_fp16_dev: [K, N] fp16, row-major, 16-byte aligned.  BORROWED for the
 *   life of the handle: forward calls read its rows W[O,:] for the fp16
 *   outlier product, so it must stay valid and unchanged until int8mm_free.
 * On success *out receives a handle that owns the int8 codes Wq^T [N, K]
 * (K-major), c_w [N], the TMA descriptors and a workspace that grows with M.
 * Enqueued on `stream`; the handle may be used on any stream ordered after it.
 */
int8mm_status int8mm_prepare_weight(const void* W_fp16_dev, int64_t K, int64_t N, void* stream,
                                    int8mm_weight_t* out);

/*
 * Memory-saving variant of int8mm_prepare_weight.  The outlier dimensions are
 * systematic, a few fixed input dimensions in every layer, and only they need
 * the fp16 path ("LLM.int8() — 大模型激活值里藏着几个超大异常通道": the
 * outliers sit in fixed feature dimensions; 方法2: those dimensions go
 * through fp16, a small fraction of the weight).
 *
 * Prepares the int8 codes and scales from W exactly as int8mm_prepare_weight
 * does, and copies the fp16 rows W[rows[i], :], i < n_rows, into the handle.
 * `rows` is a host array of distinct input dimensions in [0, K); n_rows may
 * be 0.  W is NOT borrowed: the call synchronises `stream` before it returns,
 * after which W may be freed.
 *
 * Each forward gathers the weight rows of the outlier columns it found
 * (one more kernel per forward).  A stored dimension uses its fp16 row.  For
 * any other outlier column the row is rebuilt from its int8 codes as
 * fp16(q * (1/c_w)) in fp32; the pages leave this case open.  The fp16
 * outlier product then uses that quantised row.
 *
 * At most `max_outliers` (1..K) outlier columns per forward.  The handle
 * holds max_outliers x N fp16 for their rows.  A forward that finds more
 * leaves the product of the columns past that count out of Y, and
 * int8mm_get_status returns INT8MM_ERR_OUTLIER_CAP.
 *
 * Errors: as int8mm_prepare_weight, plus INT8MM_ERR_INVALID_ARG for bad
 * rows, n_rows or max_outliers.
 */
int8mm_status int8mm_prepare_weight_static(const void* W_fp16_dev, int64_t K, int64_t N, const int32_t* rows,
                                           int64_t n_rows, int max_outliers, void* stream, int8mm_weight_t* out);

/*
 * Pre-size the per-forward workspace for up to M_max rows, so that later
 * forward calls with M <= M_max allocate nothing (needed before CUDA graph
 * capture of a forward): the activation workspace, the decode GEMM's scratch
 * and the split-K workspace of the largest split any M <= M_max uses with
 * the int8mm_set_split_k setting in effect (call it again after changing
 * that setting).  Stream-ordered allocation on `stream`.
 */
int8mm_status int8mm_reserve(int8mm_weight_t h, int64_t M_max, void* stream);

/*
 * Forward (steps 1-4; "LLM.int8() — 大模型激活值里藏着几个超大异常通道", 方法2:
 * Y = X_int8 W_int8 / scales + X_fp16 W_fp16; the Fig. 2 caption of the
 * AI 十大核心论文解读 article).
 *
 * X_fp16_dev: [M, K] fp16 row-major, 16-byte aligned, read-only.
 * Y_fp16_dev: [M, N] fp16 row-major, 16-byte aligned, written.
 * alpha: outlier threshold (6.0 in the pages); INFINITY disables the fp16
 *   path (pure vector-wise int8); any value below every |x| makes every
 *   column an outlier.  NaN is an argument error.
 * M == 0 is a no-op.  Decode shapes (M <= 128, K <= 16384) run as ONE
 * kernel on `stream`: the decode GEMM (a cooperative launch) does the
 * activation pass itself, each CTA on a slice of X's columns, with two grid
 * barriers, while its first weight tiles already stream.  Otherwise two or
 * three kernels run: the activation pass (outlier detection, row
 * quantisation and the outlier gather) and the fused int8 GEMM, a
 * programmatic dependent launch that starts while the activation pass
 * finishes.  That activation pass is one kernel for up to 256 rows per SM
 * (37888 on a 148-SM B200), else two (detection, then quantisation); a
 * static weight adds the gather of the outlier rows (and always takes the
 * separate activation pass); see int8mm_launches_per_forward.  The outlier count never leaves the device,
 * so the call does not synchronise.  Grows the workspace when M exceeds every
 * earlier M (stream-ordered allocation).
 */
int8mm_status int8mm_forward(int8mm_weight_t h, const void* X_fp16_dev, int64_t M, float alpha,
                             void* Y_fp16_dev, void* stream);

/*
 * Forward of a linear layer with bias: as int8mm_forward, plus the layer's
 * bias b[j] added to each output before the single rounding to fp16,
 * Y = fp16(X_int8 W_int8 / scales + X_fp16 W_fp16 + b) ("LLM.int8()",
 * brain.gartu.xyz, "Exemple pratique": the int8 layer that replaces
 * nn.Linear keeps its bias).
 *
 * bias_fp16_dev: [N] fp16, 16-byte aligned, read-only; NULL means no bias
 *   (the same as int8mm_forward).  A misaligned bias is an alignment error.
 */
int8mm_status int8mm_forward_bias(int8mm_weight_t h, const void* X_fp16_dev, int64_t M, float alpha,
                                  const void* bias_fp16_dev, void* Y_fp16_dev, void* stream);

/*
 * Same as int8mm_forward for host-resident X and Y: copies X_fp16_host
 * [M, K] into a handle-owned device buffer, runs the forward, and copies Y
 * back into Y_fp16_host [M, N], all enqueued on `stream`.  Y_fp16_host is
 * valid once `stream` has been synchronised.  Use page-locked host memory
 * for the copies to be asynchronous.  For prefills of at least 512 rows the
 * GEMM runs in up to four row chunks and each chunk of Y is copied back on a
 * handle-owned stream while the next chunk computes; `stream` waits for
 * those copies.
 */
int8mm_status int8mm_forward_host(int8mm_weight_t h, const void* X_fp16_host, int64_t M, float alpha,
                                  void* Y_fp16_host, void* stream);

/*
 * Same as int8mm_forward, and records three caller-created CUDA events
 * (cudaEvent_t, passed as void*; NULL entries are skipped) on `stream`:
 * before the activation pass, between it and the GEMM, and after the
 * GEMM, so that the GEMM can be timed on the stream it runs on.  A middle
 * event makes the GEMM an ordinary launch instead of a programmatic
 * dependent of the activation pass (its prologue then no longer overlaps it),
 * and makes decode shapes take the separate activation pass too (the same
 * results as the single decode kernel, which has no point between the two).
 */
int8mm_status int8mm_forward_events(int8mm_weight_t h, const void* X_fp16_dev, int64_t M, float alpha,
                                    void* Y_fp16_dev, void* stream, void* const events[3]);

/* Intermediate values of one forward, for verification.  Every field is a
 * device pointer or NULL (not written). */
typedef struct int8mm_debug_bufs {
  float* colmax;          /* [K]    max_i |X[i,j]| (fp32, exact) */
  int32_t* outlier_idx;   /* [K]    ascending outlier columns; first *count valid */
  int32_t* outlier_count; /* [1]    |O| */
  int8_t* x_codes;        /* [M, K] int8 codes of X, outlier columns 0 */
  float* c_x;             /* [M]    row scales */
  int8_t* w_codes_t;      /* [N, K] int8 codes of W, transposed (K-major) */
  float* c_w;             /* [N]    column scales */
  int32_t* acc;           /* [M, N] int32 accumulators Xq Wq */
} int8mm_debug_bufs;

/* Forward that also copies the intermediates into `dbg` (stream-ordered).
 * Filling `acc` makes the GEMM epilogue write the raw accumulators too. */
int8mm_status int8mm_forward_debug(int8mm_weight_t h, const void* X_fp16_dev, int64_t M, float alpha,
                                   void* Y_fp16_dev, void* stream, const int8mm_debug_bufs* dbg);

/*
 * Device status word of the handle: INT8MM_OK, INT8MM_ERR_TIMEOUT if a
 * kernel of an earlier forward gave up on a wait, or INT8MM_ERR_OUTLIER_CAP
 * if a forward with a static weight found more outlier columns than it
 * holds.  SYNCHRONISES the device, then clears the word.  Also returns
 * INT8MM_ERR_CUDA if the device reports an error.
 *
 * After a timeout, the forward that timed out AND every later forward on the
 * handle are invalid until this call has returned INT8MM_ERR_TIMEOUT: an
 * aborted kernel can leave counters (split-K and decode tickets, the
 * activation pass's grid barriers and row maxima) that a later forward would misread, and
 * this call is what resets them.
 */
int8mm_status int8mm_get_status(int8mm_weight_t h);

/*
 * Failure-detection self-test: enqueues on `stream` one single-thread kernel
 * that waits, bounded by the handle's wait limit (int8mm_set_wait_limit), on
 * a device flag that nothing sets, as the forward's kernels wait on tickets
 * and barriers.  The wait runs out; the kernel records it in the handle's
 * status word and returns, so int8mm_get_status then reports
 * INT8MM_ERR_TIMEOUT and the handle and the CUDA context stay usable.
 */
int8mm_status int8mm_wait_selftest(int8mm_weight_t h, void* stream);

/*
 * Time limit, in nanoseconds, for each device-side wait of later forwards
 * (default 2e9, i.e. two seconds), at least 1e6 (one millisecond).  A
 * kernel whose wait gives up reports INT8MM_ERR_TIMEOUT through
 * int8mm_get_status; before its blocks exit they wait, within the same
 * limit, for the copies and tensor-core operations they have already issued,
 * which take microseconds: the floor keeps that drain complete.
 * INT8MM_ERR_INVALID_ARG below the floor.
 */
int8mm_status int8mm_set_wait_limit(int8mm_weight_t h, uint64_t timeout_ns);

/*
 * Failure-detection tests of the forward's own waits (test use only).  Each
 * bit makes later forwards on the handle leave out one kind of arrival that
 * another part of the GPU waits for, and changes nothing else (no address,
 * load or store): the bounded wait then runs out as it would if that
 * arrival were lost, the kernels drain what they have in flight and exit,
 * and int8mm_get_status reports INT8MM_ERR_TIMEOUT and resets the counters.
 * The outputs of such forwards are invalid.  0 (the default) turns them off.
 *   INT8MM_TEST_SKIP_SPLITK_TICKET    split-K pieces of the prefill GEMM do
 *                                     not count themselves on the ticket the
 *                                     tile's owner waits for;
 *   INT8MM_TEST_SKIP_DECODE_TICKET    split n blocks of the decode GEMM (M <=
 *                                     64) likewise;
 *   INT8MM_TEST_SKIP_BARRIER_ARRIVAL  block 0 of the single-launch activation
 *                                     pass does not arrive at its grid barrier,
 *                                     nor CTA 0 of the decode GEMM at the first
 *                                     barrier of its own activation pass.
 * INT8MM_ERR_INVALID_ARG for other bits.
 */
#define INT8MM_TEST_SKIP_SPLITK_TICKET 1
#define INT8MM_TEST_SKIP_DECODE_TICKET 2
#define INT8MM_TEST_SKIP_BARRIER_ARRIVAL 4
int8mm_status int8mm_set_test_skip(int8mm_weight_t h, int bits);

/*
 * Split of the prefill GEMM along K (forwards with M > 128, whose 256 x 256
 * output tiles are computed by pairs of SMs).  0 (the default) lets the
 * library choose the plan that best fills the pairs' rounds of work: no
 * split; every tile cut into S in 2..4 pieces; or, when the tiles leave a
 * last round part-filled (such as an FFN contraction's 160 tiles for 74
 * pairs), only the tiles past the last full round cut into up to 8 pieces
 * spread over all pairs.  1..4 forces every tile into S pieces (capped at
 * the number of 128-deep k-blocks).  Piece sums are exact int32, so every
 * plan gives the same results.  A split tile needs (S-1) x 256 KB of
 * handle workspace.  INT8MM_ERR_INVALID_ARG for a value outside 0..4.
 */
int8mm_status int8mm_set_split_k(int8mm_weight_t h, int split);

/* Device bytes held by the handle (codes, scales, workspace). */
int8mm_status int8mm_weight_bytes(int8mm_weight_t h, size_t* bytes);

/* Number of kernels a forward of M rows launches with this handle (0 for
 * M == 0; 1 for decode shapes that run as one kernel; else 2 or 3, one more
 * for a static weight).  Host-side only; nothing is enqueued. */
int8mm_status int8mm_launches_per_forward(int8mm_weight_t h, int64_t M, int* count);

/*
 * Outlier-column detection (step 1 above) that allocates no device memory.
 * The paper has no counterpart of this entry point; it exists for callers
 * that cannot allocate when they need the outlier set: an engine plugin whose
 * enqueue step may not allocate, a serving loop that forbids allocation after
 * warm-up, or a process whose caching allocator already holds nearly all of
 * the device memory.
 *
 * X_fp16_dev: [M, K] fp16 row-major, 16-byte aligned (0 <= M < 2^31; may
 *             be NULL when M == 0).
 * idx_dev:    [K] int32, written with the ascending outlier columns; the
 *             first *count_dev entries are valid.
 * count_dev:  [1] int32, written with |O|.
 * colmax_dev: [K] fp32 max_i |X[i,j]| (all 0 when M == 0), or NULL to skip
 *             it.
 * All three outputs are device memory owned by the caller.  Same results as
 * the outlier_idx / outlier_count / colmax of int8mm_forward_debug.
 *
 * Scratch lives in one static device array of INT8MM_NOALLOC_SCRATCH_BYTES
 * (1 MiB), which every GPU that loads the library holds until the process
 * exits; the call itself makes no cudaMalloc, cudaFree or other allocation.
 * Limit: 16 <= K <= INT8MM_MAX_K, K % 16 == 0 (larger K is rejected with
 * INT8MM_ERR_UNSUPPORTED_SHAPE).  The first call on a device looks up the
 * array's device address in the current context (again after the context
 * is re-created, e.g. by cudaDeviceReset); make that first call before any
 * CUDA stream capture.  All calls share the array and each call clears what
 * must start at zero; calls whose kernels overlap on the GPU (unordered
 * streams) race.
 */
#define INT8MM_NOALLOC_SCRATCH_BYTES (1u << 20)
int8mm_status int8mm_outlier_columns_noalloc(const void* X_fp16_dev, int64_t M, int64_t K, float alpha,
                                             int32_t* idx_dev, int32_t* count_dev, float* colmax_dev,
                                             void* stream);

/* Release the handle and everything it owns.  SYNCHRONISES the device
 * first, so no enqueued forward still uses the memory.  NULL or an already
 * freed handle is a no-op. */
void int8mm_free(int8mm_weight_t h);

/* Message of the last error returned on this host thread ("" if none). */
const char* int8mm_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* INT8MM_H */
