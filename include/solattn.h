/*
 * solattn.h -- C ABI of libsolattn, a B200 (sm_100a) implementation of the
 * Sol-Attn forward attention operator.
 *
 * Sol-Attn ("Sol-Attn: Accelerating Video Generation Inference via On-the-Fly
 * Attention Sparsification", abstract and paperlayer summary §3 Methodology)
 * runs one online-softmax pass over key/value blocks. For every query block it
 * scores each key block with a proxy taken from the mean-pooled Q and K blocks,
 * keeps the block for exact attention only if the proxy clears a threshold set
 * relative to the running maximum, and folds every dropped block back in as one
 * pseudo-key that carries the block's mean V ("approximate correction" by
 * proxy-score reuse). The proxy map is never written to memory.
 *
 * Definitions used here (the pages leave these open; this library fixes them):
 *   q_i, k_j, v_j  means of Q, K, V over the VALID rows of query block i /
 *                  key block j (a ragged last block divides by its row count n_j)
 *   s_ij           = q_i . k_j / sqrt(d)                          (block proxy)
 *   visit order    query block i visits key blocks (j0 + t) mod nKB,
 *                  t = 0..nKB-1, with j0 = min(floor(i*Bq/Bk), nKB-1)
 *   threshold      M = max of the proxies visited so far (current included);
 *                  the visited block is kept iff s_ij >= M - tau
 *   output row r   keep_correct: [sum_kept sum_c e^{s_rc} v_c + sum_dropped n_j e^{s_ij} v_j]
 *                               / [sum_kept sum_c e^{s_rc} + sum_dropped n_j e^{s_ij}]
 *                  keep_drop:    the same without the dropped terms
 *                  dense:        every block kept (plain softmax attention)
 *   with s_rc = q_r . k_c / sqrt(d).
 * These are the definitions of solattn_forward. solattn_forward_gaussian and
 * solattn_forward_ex add the pages' query-dependent Gaussian threshold, sink tokens and
 * the token-to-block correction; each is defined where it is declared below.
 *
 * Data layout: q, k, v and out are contiguous row-major bf16 [B][H][N][d]
 * (token index n = (t*Y + y)*X + x for a (t, y, x) patch grid, t-major).
 * Pooled buffers are contiguous fp32 [B][H][nB][d].
 *
 * Threading: every entry point that takes a stream enqueues work on that
 * CUDA stream (cudaStream_t passed as void*, NULL = legacy default stream)
 * and returns without waiting, except solattn_get_status and
 * solattn_forward_host, which synchronise the stream.
 *
 * Ownership: the caller allocates and owns every buffer (inputs, output,
 * statistics, workspace). The library allocates no memory at run time. Its one
 * device-memory holding is the static scratch of solattn_forward_noalloc
 * (SOLATTN_NOALLOC_SCRATCH_BYTES), a module-scope device array that exists on
 * every GPU where the library's module is loaded, for the life of the process.
 * solattn_forward_host also keeps, per device, two non-blocking copy streams and
 * a few events, created at its first call there and kept for the process.
 */
#ifndef SOLATTN_H
#define SOLATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Routing / correction mode. */
typedef enum {
  SOLATTN_DENSE = 0,        /* every key block kept: plain softmax attention        */
  SOLATTN_KEEP_DROP = 1,    /* dropped blocks discarded ("keep-or-drop")             */
  SOLATTN_KEEP_CORRECT = 2  /* dropped blocks re-enter as proxy-weighted pseudo-keys */
} solattn_mode;

/* Status codes. Argument errors are returned before any device work is queued. */
typedef enum {
  SOLATTN_OK = 0,
  SOLATTN_EINVAL = -1,       /* null, misaligned or other-GPU pointer, N/B/H < 1, bad mode, tau < 0 or NaN */
  SOLATTN_EUNSUPPORTED = -2, /* d or Bq/Bk not in {64,128}, nKB > 1024, B*H > 65535, no sm_100 device */
  SOLATTN_ECUDA = -3,        /* a CUDA runtime or driver call failed                          */
  SOLATTN_ETIMEOUT = -4,     /* a device-side wait ran past its limit (reported by get_status) */
  SOLATTN_EWORKSPACE = -5,   /* workspace pointer null/misaligned or smaller than required     */
  SOLATTN_EBOUNDS = -6       /* a device-side bounds check failed (libsolattn_debug.so only:
                                the build with -DSOLATTN_DEBUG; reported by get_status)        */
} solattn_status;

/* Per-call statistics (device pointers). */
typedef struct {
  /* [B*H] int64: sum over query blocks i of |K_i| (kept key blocks) for each
   * (b, h). Required. Overwritten by every solattn_forward call; in dense mode
   * it is nQB*nKB. */
  int64_t *kept_per_head;
  /* Optional (NULL to skip): [B*H][nQB][ceil(nKB/32)] uint32 keep bit-mask,
   * bit (j & 31) of word (j >> 5) set iff query block i keeps key block j.
   * Overwritten for every valid query block. For tests; off the timed path. */
  uint32_t *keep_mask;
} solattn_stats;

/* Largest number of key blocks per head (nKB = ceil(N/Bk)) a call accepts. */
#define SOLATTN_MAX_KEY_BLOCKS 1024

/*
 * Bytes of device workspace solattn_forward needs for this shape: a small
 * header (work counter, device status word), the pooled q, k, v blocks in fp32,
 * an fp16 copy of v, the work schedule, the keep bits and correction records of
 * the routing pass, and what the Gaussian threshold and the token-to-block
 * correction need. Returns 0 for an unsupported or invalid shape.
 */
size_t solattn_workspace_size(int B, int H, int N, int d, int Bq, int Bk);

/*
 * Mean-pool one bf16 tensor x [B][H][N][d] over blocks of `blk` rows into
 * xbar [B][H][ceil(N/blk)][d] fp32 (ragged last block: mean over its valid
 * rows). Step "mean pooling of each query and key block" (paperlayer summary
 * §2 Preliminaries; §3 Methodology, "pooled keys and summed values").
 * x must be 16-byte aligned, xbar 16-byte aligned. blk in {64,128}, d in {64,128}.
 * Returns SOLATTN_OK or an error code; asynchronous on `stream`.
 */
int solattn_pool(const void *x, float *xbar, int B, int H, int N, int d, int blk,
                 void *stream);

/*
 * The Sol-Attn forward operator (one fused pass per query tile: routing,
 * exact attention on kept blocks, correction for dropped blocks; abstract and
 * paperlayer summary §3 Methodology, "Unified execution").
 *
 *   q, k, v    device, bf16 [B][H][N][d], 16-byte aligned. The P.V product runs in
 *              fp16 (on an fp16 copy of v made by the pooling pass), so entries of v
 *              must lie in the fp16 range, |v| <= 65504; larger ones become inf.
 *   out        device, bf16 [B][H][N][d], 16-byte aligned (written)
 *   B, H, N    batch, heads, tokens (>= 1); nKB = ceil(N/Bk) <= SOLATTN_MAX_KEY_BLOCKS
 *   d          head dim, 64 or 128
 *   Bq, Bk     query / key block sizes, each 64 or 128
 *   tau        threshold offset in logit units, >= 0; +INFINITY keeps every block;
 *              ignored in dense mode
 *   mode       a solattn_mode
 *   stats      required; stats->kept_per_head device [B*H] int64
 *   workspace  device, 256-byte aligned, >= solattn_workspace_size(...) bytes;
 *              must not be used by another call that runs at the same time
 *   stream     cudaStream_t (as void*)
 *
 * Every device pointer must belong to the current device (cudaGetDevice): one that
 * belongs to another GPU is rejected with SOLATTN_EINVAL. The buffers' sizes cannot be
 * checked here; the caller guarantees the sizes stated above.
 *
 * Returns SOLATTN_OK once the work is queued (errors inside the kernels are
 * reported by solattn_get_status), or an error code with nothing queued.
 */
int solattn_forward(const void *q, const void *k, const void *v, void *out,
                    int B, int H, int N, int d, int Bq, int Bk, float tau, int mode,
                    const solattn_stats *stats, void *workspace, size_t ws_bytes,
                    void *stream);

/*
 * solattn_forward plus two CUDA events (cudaEvent_t as void*, either may be NULL)
 * recorded on `stream` immediately before and after the attention kernel, so a
 * caller can time that kernel alone inside a timed region. Same arguments,
 * results and errors as solattn_forward.
 */
int solattn_forward_events(const void *q, const void *k, const void *v, void *out,
                           int B, int H, int N, int d, int Bq, int Bk, float tau, int mode,
                           const solattn_stats *stats, void *workspace, size_t ws_bytes,
                           void *stream, void *ev_attn_begin, void *ev_attn_end);

/*
 * Size of the library's static device scratch used by solattn_forward_noalloc
 * (64 MiB, held on every GPU that loads the library until the process exits).
 */
#define SOLATTN_NOALLOC_SCRATCH_BYTES (64u << 20)

/*
 * solattn_forward for callers that cannot allocate device memory. The paper has no
 * counterpart to this entry point; it is an interface convenience of this library.
 *
 * Who needs it: code that receives only its input and output buffers and a stream
 * (plugin interfaces of inference runtimes, callbacks that run while the host
 * framework's allocator is locked, processes with a fixed device-memory budget where
 * a late cudaMalloc fails or synchronises the whole device) cannot provide the
 * workspace solattn_forward asks for. This entry point takes the same arguments minus
 * the workspace and calls no allocating routine (no cudaMalloc, cudaFree or library
 * allocator); its scratch is a static device array of SOLATTN_NOALLOC_SCRATCH_BYTES.
 *
 *   - The first call on a device looks up that array's device address
 *     (cudaGetSymbolAddress) with the device current, and later calls on that device
 *     reuse it; make this first call before any stream capture. cudaDeviceReset
 *     unloads the module and may move the array: do not call this entry point on a
 *     device after resetting it in the same process.
 *   - Shapes whose solattn_workspace_size(...) exceeds SOLATTN_NOALLOC_SCRATCH_BYTES
 *     are rejected with SOLATTN_EWORKSPACE before any device work.
 *   - Every call on a device uses the same scratch, which keeps the previous call's
 *     contents; the call clears what must start at zero (work counter, status word)
 *     on its stream. Calls that overlap on the GPU (on different streams, or from
 *     different threads) race on the scratch and give wrong results: serialise them.
 *   - Device-side wait timeouts are recorded in the static scratch and are not
 *     reported to the caller; use solattn_forward and solattn_get_status when that
 *     status is needed.
 * Arguments, results and the other errors are those of solattn_forward.
 */
int solattn_forward_noalloc(const void *q, const void *k, const void *v, void *out,
                            int B, int H, int N, int d, int Bq, int Bk, float tau, int mode,
                            const solattn_stats *stats, void *stream);

/* Variant of the Gaussian threshold's variance estimate. */
typedef enum {
  SOLATTN_GAUSS_EXACT = 0,  /* full pooled-key covariance: sigma_i^2 = q_i^T Cov[K] q_i / d      */
  SOLATTN_GAUSS_DIAG = 1    /* its diagonal only: sigma_i^2 = sum_e q_ie^2 Cov[K]_ee / d          */
} solattn_gauss_variant;

/*
 * solattn_forward with the pages' query-dependent Gaussian threshold in place of the
 * running-maximum rule ("Sol-Attn: Accelerating Video Generation Inference via
 * On-the-Fly Attention Sparsification", paperlayer summary §2, Figure 2: a threshold from
 * the proxy-logit mean, standard deviation and a standardized offset beta; §3
 * "Dynamic threshold routing": mean and variance from the pooled keys' first and second
 * moments, one shared cutoff; appendix "Diagonal threshold estimator").
 *
 *   theta_i  = q_i . E[K] / sqrt(d) + beta * sigma_i, with E and Cov taken over the key
 *              blocks' pooled rows k_j (equal weight, 1/nKB), sigma_i as in `variant`
 *   keep     iff s_ij >= theta_i; the block with query block i's largest proxy (lowest
 *              index on ties) is always kept, so no exact set is empty
 *   output   as solattn_forward for `mode` (dense ignores beta)
 *
 * beta may be +-infinity (-inf keeps every block, +inf only each row's top block).
 * Errors: beta NaN or an unknown variant -> SOLATTN_EINVAL; otherwise as
 * solattn_forward. The workspace is the same (solattn_workspace_size).
 */
int solattn_forward_gaussian(const void *q, const void *k, const void *v, void *out,
                             int B, int H, int N, int d, int Bq, int Bk, float beta, int variant,
                             int mode, const solattn_stats *stats, void *workspace, size_t ws_bytes,
                             void *stream);

/* Routing rule of solattn_forward_ex. */
typedef enum {
  SOLATTN_RULE_RUNNING_MAX = 0,  /* keep iff s_ij >= M - tau (solattn_forward)                 */
  SOLATTN_RULE_GAUSS_EXACT = 1,  /* keep iff s_ij >= theta_i, exact covariance (solattn_forward_gaussian) */
  SOLATTN_RULE_GAUSS_DIAG = 2    /* the same with the diagonal covariance                       */
} solattn_rule;

/* Routing options of solattn_forward_ex. */
typedef struct {
  int rule;    /* solattn_rule                                                          */
  float tau;   /* running-max rule: tau >= 0 (+infinity keeps every block)              */
  float beta;  /* Gaussian rules: standardized offset (not NaN; +-infinity allowed)     */
  int n_sink;  /* leading key tokens kept as sinks: 0 <= n_sink <= N                    */
  int correction; /* keep_correct only: SOLATTN_CORR_BLOCK (0) or SOLATTN_CORR_TOKEN (1)   */
} solattn_route;

/* Correction of solattn_forward_ex in keep_correct mode. */
typedef enum {
  SOLATTN_CORR_BLOCK = 0,  /* dropped block j enters query block i with the block proxy s_ij     */
  SOLATTN_CORR_TOKEN = 1   /* it enters row r with the token-to-block logit q_r . k_j / sqrt(d)   */
} solattn_correction;

/*
 * The forward operator with every routing option. Sinks: the text key-value tokens that
 * the pages keep in the exact branch for every query ("Sol-Attn: Accelerating Video
 * Generation Inference via On-the-Fly Attention Sparsification", paperlayer summary,
 * App. A Additional Experimental Details). This library takes them to be the first
 * n_sink key tokens (a prefix of the [B][H][N][d] layout): every key block that holds
 * one of them, ceil(n_sink / Bk) blocks, is kept by every query block under either rule
 * and is never folded into the correction. The proxies of sink blocks still enter the
 * running maximum, so the other keep decisions do not change; under a Gaussian rule the
 * top-block guard applies only to a query block that would otherwise keep nothing.
 * Token-to-block correction (keep_correct, correction = SOLATTN_CORR_TOKEN): the pages
 * fuse routing and correction through a token-to-block score tile ("Unified execution",
 * paperlayer summary §3). Each row r then meets every block j its query block dropped as
 * one pseudo-key: logit q_r . k_j / sqrt(d) (pooled key k_j), weight n_j, value v_j,
 * inside the same online softmax as the exact blocks (computed on the tensor cores over
 * the head's pooled keys, with the kept blocks masked out).
 * With n_sink = 0 and the block correction, rule RUNNING_MAX equals solattn_forward and
 * the Gaussian rules equal solattn_forward_gaussian.
 * Errors: route NULL, an unknown rule, tau < 0 or NaN (running max), beta NaN (Gaussian),
 * n_sink outside [0, N] or an unknown correction -> SOLATTN_EINVAL; otherwise as
 * solattn_forward.
 */
int solattn_forward_ex(const void *q, const void *k, const void *v, void *out,
                       int B, int H, int N, int d, int Bq, int Bk, const solattn_route *route,
                       int mode, const solattn_stats *stats, void *workspace, size_t ws_bytes,
                       void *stream);

/*
 * The routing stage on its own, for the routing-overhead measurement ("Sol-Attn:
 * Accelerating Video Generation Inference via On-the-Fly Attention Sparsification",
 * paperlayer summary §4 Experiments, "Efficient On-the-Fly Sparsification": routing that
 * consumes proxy scores on chip, against top-k and top-p routing, which materialise the
 * proxy map and traverse its rows; §2 Block-Sparse Attention). The three routers read the
 * same pooled blocks and write keep bits in the layout of solattn_stats.keep_mask:
 *
 *   qbar, kbar  device fp32 [B][H][nQB][d] and [B][H][nKB][d] (block means, as written by
 *               solattn_pool with blk = Bq and Bk), 16-byte aligned
 *   keep_mask   device u32 [B][H][nQB][ceil(nKB/32)], written
 *   proxy_map   device fp32 scratch of solattn_proxy_map_bytes(...) bytes (map_bytes), which
 *               the top-k and top-p routers fill with s_ij = q_i . k_j / sqrt(d)
 *
 * solattn_route_keep: the running-maximum rule of solattn_forward (same visit order, same
 *   tau), computed as the forward kernel's router does, with no proxy leaving the chip.
 * solattn_route_topk: keeps the min(k, nKB) key blocks with the largest proxies of every
 *   query block (ties: lower block index). k >= 1.
 * solattn_route_topp: ranks the key blocks of a query block by mass n_j e^{s_ij} (n_j valid
 *   keys of block j; ties: lower index) and keeps the shortest prefix whose share of the
 *   row's total mass reaches p (a block is kept iff the mass ranked before it is below
 *   p times the total). 0 < p <= 1.
 * The readings of top-k and top-p are this library's (the pages name the rules only).
 * Errors: null or misaligned pointers, tau < 0 or NaN, k < 1, p outside (0, 1] ->
 * SOLATTN_EINVAL; a short proxy_map -> SOLATTN_EWORKSPACE; otherwise as solattn_forward.
 * Asynchronous on `stream`.
 */
int solattn_route_keep(const float *qbar, const float *kbar, int B, int H, int N, int d, int Bq, int Bk,
                       float tau, uint32_t *keep_mask, void *stream);
size_t solattn_proxy_map_bytes(int B, int H, int N, int Bq, int Bk);
int solattn_route_topk(const float *qbar, const float *kbar, int B, int H, int N, int d, int Bq, int Bk,
                       int k, float *proxy_map, size_t map_bytes, uint32_t *keep_mask, void *stream);
int solattn_route_topp(const float *qbar, const float *kbar, int B, int H, int N, int d, int Bq, int Bk,
                       float p, float *proxy_map, size_t map_bytes, uint32_t *keep_mask, void *stream);

/*
 * Synchronise `stream` and read the device status word of `workspace`
 * (SOLATTN_OK, or SOLATTN_ETIMEOUT if a bounded device-side wait gave up).
 */
int solattn_get_status(const void *workspace, void *stream);

/* Bytes of device scratch solattn_forward_host needs (device copies of q, k,
 * v, out, the per-head counts, per-chunk status words and the forward
 * workspace). 0 if invalid. */
size_t solattn_host_workspace_size(int B, int H, int N, int d, int Bq, int Bk);

/*
 * End-to-end call on HOST buffers: copies q, k, v (bf16 [B][H][N][d], host) to
 * the device scratch, runs the forward operator (running-max rule, `tau`,
 * `mode` as in solattn_forward), copies the bf16 output to `out` and the
 * per-head kept counts to `kept_per_head` (host int64 [B*H], may be NULL),
 * synchronises `stream` and returns the first non-zero device status, else
 * SOLATTN_OK.
 * The (b, h) heads are independent, so the call is a pipeline over up to 16
 * chunks of consecutive heads: the upload of one chunk and the download of the
 * one before overlap the forward of the chunk between them. Uploads and
 * downloads run on the library's copy streams for this device, the forward on
 * `stream`; the result equals that of one solattn_forward over all heads.
 * Copies overlap only from page-locked (pinned) host memory.
 * dev_scratch: device, 256-byte aligned, >= solattn_host_workspace_size(...).
 * Calls on one device are serialised (they share the copy streams). On an error
 * the call waits for the copies it issued before returning.
 */
int solattn_forward_host(const void *q, const void *k, const void *v, void *out,
                         int B, int H, int N, int d, int Bq, int Bk, float tau, int mode,
                         int64_t *kept_per_head, void *dev_scratch, size_t scratch_bytes,
                         void *stream);

/*
 * Self-test of the device watchdog: launches one block that waits on a
 * barrier nobody completes, with a limit of `limit_ns` nanoseconds, and
 * stores the resulting status (SOLATTN_ETIMEOUT when the watchdog works) in
 * the workspace status word. Read it with solattn_get_status.
 */
int solattn_watchdog_selftest(void *workspace, size_t ws_bytes, uint64_t limit_ns,
                              void *stream);

/*
 * Self-test of the software exp2 the softmax evaluates on the FMA pipe for part of
 * its exponentials: y[i] = 2^x[i] for n device floats (x, y device pointers).
 * Lets a test compare it with exp2 within its stated bound (relative error 7.5e-5
 * for x >= -125; smaller inputs are clamped to -125).
 */
int solattn_selftest_exp2(const float *x, float *y, int n, void *stream);

/* Static description of a status code. */
const char *solattn_strerror(int status);

#ifdef __cplusplus
}
#endif

#endif /* SOLATTN_H */
