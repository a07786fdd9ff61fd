/*
 * lola.h -- C ABI of the B200 (sm_100a) LoLA hybrid-attention inference engine.
 *
 * LoLA (Low-Rank Linear Attention with Sparse Caching, arXiv 2505.23666) splits
 * the past key/value pairs of each (batch, kv-head) stream over three memories
 * (gist.science technical summary, section "Methodologie"):
 *   - a sliding window of the `window` most recent pairs, attended by softmax;
 *   - a sparse global cache of at most `lambda_` pairs, attended by softmax;
 *   - the linear-attention state H (feat_dim x head_dim) and s (feat_dim),
 *     holding every other pair folded in as H += phi(k) v^T, s += phi(k).
 * At each update interval ("Inferentiestrategie" section) the pairs leaving the
 * window and the pairs already cached are scored by the Self-Recall Error
 * SRE(k,v|H,s) = || phi(k)^T H / (phi(k)^T s + eps) - v ||^2 (section
 * "Het Self-Recall Error (SRE) Mechanisme"), the lambda_ highest stay cached
 * (ties: the lower token index stays), the rest are folded, and each query's
 * output combines softmax over window and cache with the linear readout of the
 * state under one shared normaliser. The feature map is
 * phi(x) = [softmax(x W), softmax(-x W)] with W of shape head_dim x feat_dim/2.
 *
 * Conventions for every entry point:
 *   - Tensors are caller-owned DEVICE pointers, contiguous, 16-byte aligned,
 *     in the state's dtype (float32 or bfloat16), token-major per batch:
 *       q, out: [batch][n_tokens][n_q_heads][head_dim]
 *       k, v:   [batch][n_tokens][n_kv_heads][head_dim]
 *     Query head h reads kv-head h / (n_q_heads / n_kv_heads) (grouped queries).
 *   - The library allocates no device memory. The caller allocates
 *     lola_state_bytes() bytes of device memory (the "workspace") and passes it
 *     to lola_init_state(); it holds the persistent state and all scratch.
 *   - Work is enqueued on the caller's CUDA stream (`cuda_stream` is a
 *     cudaStream_t; NULL = the legacy default stream). Calls return once the
 *     work is enqueued; results are ready when the stream reaches them.
 *   - Host-side argument checks return a status synchronously and enqueue
 *     nothing. Errors raised on the device (bounds checks) are recorded in an
 *     error word inside the workspace and reported by lola_sync().
 *   - A state handle is not thread-safe: one host thread at a time per handle.
 */
#ifndef LOLA_H
#define LOLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LOLA_OK = 0,
    LOLA_ERR_INVALID_ARG = 1, /* null pointer, unsupported size, bad config value */
    LOLA_ERR_SHAPE = 2,       /* n_tokens not a positive multiple of chunk */
    LOLA_ERR_DTYPE = 3,       /* dtype not LOLA_F32 / LOLA_BF16 */
    LOLA_ERR_STATE = 4,       /* call not allowed in the state's current position */
    LOLA_ERR_WORKSPACE = 5,   /* workspace too small, misaligned, or n_tokens > max_prefill_tokens */
    LOLA_ERR_CUDA = 6,        /* a CUDA launch or query failed */
    LOLA_ERR_TIMEOUT = 7,     /* a bounded device wait gave up */
    LOLA_ERR_DEVICE = 8       /* a device-side bounds check fired (see lola_sync) */
} lola_status;

typedef enum { LOLA_F32 = 0, LOLA_BF16 = 1 } lola_dtype;

/* How the sparse cache ranks its candidates (the cache pairs and the pairs
 * leaving the window) at each update interval; the highest scores stay.
 * LOLA_SCORE_SRE is the method (section "Het Self-Recall Error (SRE)
 * Mechanisme"). The others are the alternatives the paper's ablations compare
 * it against (sections "Belangrijkste bijdragen" and "Ablaties") and the FIFO
 * structure the "Inferentiestrategie" section mentions; the pages do not define
 * them, this engine's readings are, for the interval's first query q and summed
 * over the query heads of the kv-head's group:
 *   LOLA_SCORE_ATTN_WEIGHT    the softmax weight of the pair among the candidates,
 *                             softmax over candidates c of q.k_c / sqrt(head_dim);
 *   LOLA_SCORE_SOFTMAX_ERROR  (that weight - phi(q).phi(k) / sum over candidates of
 *                             phi(q).phi(k_c))^2, how badly the linear attention
 *                             approximates the pair's softmax weight;
 *   LOLA_SCORE_RECENCY        the token index: the most recent pairs stay (FIFO). */
typedef enum {
    LOLA_SCORE_SRE = 0,
    LOLA_SCORE_ATTN_WEIGHT = 1,
    LOLA_SCORE_SOFTMAX_ERROR = 2,
    LOLA_SCORE_RECENCY = 3
} lola_scorer;

typedef struct {
    int32_t batch;              /* B >= 1 */
    int32_t n_q_heads;          /* multiple of n_kv_heads, at most 8 per kv-head */
    int32_t n_kv_heads;         /* >= 1 */
    int32_t head_dim;           /* d: 32, 64 or 128 */
    int32_t feat_dim;           /* D: multiple of 32 in [32, 256] */
    int32_t window;             /* eta >= 0 (0 = no softmax window) */
    int32_t lambda_;            /* sparse-cache capacity, 0..4096 (0 = no cache) */
    int32_t chunk;              /* prefill update interval C, 1..256 */
    int32_t decode_interval;    /* decode update interval, 1..min(256, window + 1) */
    int32_t max_prefill_tokens; /* largest n_tokens of one prefill call (multiple of chunk) */
    float eps;                  /* >= 0, added to every denominator (SRE and output) */
    int32_t dtype;              /* lola_dtype of q, k, v, out and W */
    int32_t scorer;             /* lola_scorer (0 = the Self-Recall Error) */
    int32_t w_per_kv_head;      /* 0: one feature-map matrix W shared by every head;
                                   1: one per kv-head (its query heads use it too) */
} lola_config;

typedef struct lola_state lola_state; /* opaque host handle */

/* Bytes of device workspace a state with this config needs (persistent state
 * plus per-call scratch sized by max_prefill_tokens). Pure host computation. */
lola_status lola_state_bytes(const lola_config *cfg, size_t *device_bytes);

/* Creates a state in `workspace` (device, >= lola_state_bytes, 256-byte
 * aligned, owned by the caller and kept alive until lola_free_state) and
 * resets it to the empty state at position 0: H = 0, s = 0, empty cache and
 * window. W: device [head_dim][feat_dim/2] in cfg->dtype, or with
 * cfg->w_per_kv_head [n_kv_heads][head_dim][feat_dim/2] (kv-head h's keys and
 * its query heads use W[h]); copied in (the caller may free it after the stream
 * has passed this call). On success *out receives a host handle. */
lola_status lola_init_state(const lola_config *cfg, const void *W, void *workspace,
                            size_t workspace_bytes, void *cuda_stream, lola_state **out);

/* Returns the state to position 0 (empty memories); W is kept. */
lola_status lola_reset_state(lola_state *st, void *cuda_stream);

/* Chunkwise prefill of n_tokens new tokens per sequence (all sequences at the
 * same position). n_tokens must be a positive multiple of cfg.chunk and at most
 * max_prefill_tokens (else LOLA_ERR_SHAPE / LOLA_ERR_WORKSPACE). The call runs
 * n_tokens / chunk update intervals of length chunk starting at the current
 * position and writes every query's output. Not allowed while a decode
 * interval is open (position not at an interval boundary): LOLA_ERR_STATE. */
lola_status lola_prefill_chunk(lola_state *st, const void *q, const void *k, const void *v,
                               int64_t n_tokens, void *out, void *cuda_stream);

/* Chunkwise prefill from host memory: the same computation as lola_prefill_chunk
 * over n_tokens tokens, with q, k, v and out in HOST memory ([B][n_tokens][heads]
 * [head_dim], as for lola_prefill_chunk; pinned memory lets the copies run
 * asynchronously). The call cuts the tokens into pieces of piece_tokens (a positive
 * multiple of cfg.chunk, at most max_prefill_tokens; the last piece may be shorter
 * but is a multiple of cfg.chunk) and runs lola_prefill_chunk on each piece in
 * turn, while the next piece's inputs go to the device and the previous piece's
 * outputs come back on two copy streams of the library. staging: device memory
 * owned by the caller, at least lola_prefill_host_staging_bytes(cfg, piece_tokens)
 * bytes, 256-byte aligned (two slots of q, k, v and out pieces); the call
 * allocates nothing. The call returns once the work is queued; when cuda_stream
 * has passed it, every output row is in `out` on the host. Errors as for
 * lola_prefill_chunk, and LOLA_ERR_WORKSPACE for a staging buffer that is too
 * small. An error from a piece after the first ends the call: the pieces before
 * it are done and their outputs copied back, the state after the failing piece is
 * undefined (reset it), and the copies already queued finish before cuda_stream
 * passes the call. */
lola_status lola_prefill_host(lola_state *st, const void *q, const void *k, const void *v, int64_t n_tokens,
                              void *out, void *staging, size_t staging_bytes, int64_t piece_tokens,
                              void *cuda_stream);
lola_status lola_prefill_host_staging_bytes(const lola_config *cfg, int64_t piece_tokens, size_t *bytes);

/* How a prefill call overlaps its two parts (no counterpart in the paper, which
 * describes no kernel; it changes when work runs, not what is computed). The
 * call's update intervals run as a sequential per-stream chain (score, select,
 * fold: the Self-Recall Error and sparse-caching steps of the "SRE" and
 * "Inferentiestrategie" sections) on a few SMs per stream, and a parallel
 * attention over all intervals on the other SMs, in segments of consecutive
 * intervals: the attention of a segment starts once every stream's chain has
 * finished that segment.
 *   mode LOLA_SCHEDULE_AUTO      the default: LOLA_SCHEDULE_SEGMENTS where the chain
 *        occupies more than a third of the device's SMs (many streams), else
 *        LOLA_SCHEDULE_ONE_CHAIN
 *   mode LOLA_SCHEDULE_ONE_CHAIN one chain launch per call; it counts finished
 *        segments in device memory and each attention segment waits for its count
 *        (a stream memory operation, no kernel waits on another). Falls back to
 *        LOLA_SCHEDULE_SEGMENTS where the driver has no stream memory operations.
 *   mode LOLA_SCHEDULE_SEGMENTS  one chain launch per segment, each attention
 *        segment gated by an event; between two chain launches the chain's SMs
 *        also take waiting attention work.
 * intervals_per_segment: 0 for the library's length, with m = max_prefill_tokens /
 * chunk intervals per call at most: max(16, m / 32) for one chain launch and
 * max(16, m / 16) for launches per segment, lowered for a call of n intervals to
 * max(8, ceil(n / 4)) where that is shorter; else >= 1. A length that would give
 * more than 64 segments per call is raised to ceil(m / 64). The setting applies
 * to the following calls of the state. Both modes and every length give the same outputs bit for bit.
 * It takes effect only for bfloat16 configs on the tensor-core chain and
 * attention with more than one interval per call; elsewhere it is stored and
 * ignored. LOLA_ERR_INVALID_ARG for a null state, an unknown mode or a negative
 * length. Host call; nothing is enqueued. */
typedef enum {
    LOLA_SCHEDULE_AUTO = 0,
    LOLA_SCHEDULE_ONE_CHAIN = 1,
    LOLA_SCHEDULE_SEGMENTS = 2
} lola_schedule;
lola_status lola_set_prefill_schedule(lola_state *st, int32_t mode, int32_t intervals_per_segment);

/* The schedule a prefill call of n_tokens tokens gets on a state with this config
 * whose schedule was set to (mode, intervals_per_segment), on a device of `sms`
 * SMs (148 on a B200): *mode_out LOLA_SCHEDULE_ONE_CHAIN or LOLA_SCHEDULE_SEGMENTS,
 * *len_out the intervals per segment and *segments_out the segments of the call. A
 * call of one segment (every call of a config that does not run the tensor-core
 * chain and attention, or of one interval) runs its chain and then its attention
 * on the caller's stream and reports LOLA_SCHEDULE_SEGMENTS with len = its
 * intervals. At run time LOLA_SCHEDULE_ONE_CHAIN becomes LOLA_SCHEDULE_SEGMENTS
 * where the driver has no stream memory operations. Pure host computation. Errors:
 * LOLA_ERR_INVALID_ARG (null output, sms < 1, bad mode or length, bad config),
 * LOLA_ERR_SHAPE / LOLA_ERR_WORKSPACE for n_tokens as in lola_prefill_chunk. */
lola_status lola_prefill_plan(const lola_config *cfg, int32_t mode, int32_t intervals_per_segment, int32_t sms,
                              int64_t n_tokens, int32_t *mode_out, int32_t *len_out, int32_t *segments_out);

/* One token per sequence: q [B][n_q_heads][head_dim], k, v [B][n_kv_heads][head_dim],
 * out [B][n_q_heads][head_dim]. When the position is at an interval boundary,
 * an update interval of length decode_interval opens here (score, select, fold);
 * the next decode_interval steps belong to it. */
lola_status lola_decode_step(lola_state *st, const void *q, const void *k, const void *v,
                             void *out, void *cuda_stream);

/* The same decode step as lola_decode_step, for callers that cannot obtain
 * device memory on demand -- for example a plugin whose host framework owns
 * all device memory and passes it only inputs, outputs and persistent state,
 * or code running while a CUDA graph is being captured, where cudaMalloc is
 * not allowed. The paper has no counterpart to this call; it only changes
 * where temporaries live. The per-step scratch of the decode attention (the
 * partial sums of the warps or CTAs that share a stream, and for bfloat16 the
 * fp32 query features) is taken from an 8 MiB array inside the library (a
 * static device array: every GPU that loads the library holds it until the
 * process exits) instead of the workspace. The call allocates nothing.
 * Configs whose decode scratch,
 * streams*parts*(n_q_heads/n_kv_heads)*(2*head_dim+4)*4 bytes (parts = partial
 * records per stream, chosen by the library) plus, for bfloat16,
 * batch*n_q_heads*feat_dim*4 bytes (each rounded up to 256), exceed 8 MiB get
 * LOLA_ERR_WORKSPACE.
 * The first call on a device looks up the array's device address (once per
 * device, with the device current); make that first call before any stream
 * capture. All calls share the one array and leave their contents in it, so
 * calls whose work overlaps on the GPU (other states, other streams) race:
 * order them on one stream or synchronise between them. */
lola_status lola_decode_step_static(lola_state *st, const void *q, const void *k, const void *v,
                                    void *out, void *cuda_stream);

/* Current position (tokens processed per sequence). */
int64_t lola_position(const lola_state *st);

/* Copies the cached token indices: dev_idx [B][n_kv_heads][lambda_] int32
 * (slot order, -1 for empty slots) and, if dev_count is not NULL,
 * dev_count [B][n_kv_heads] int32. Device pointers, enqueued on the stream. */
lola_status lola_get_cache_indices(const lola_state *st, int32_t *dev_idx, int32_t *dev_count,
                                   void *cuda_stream);

/* Bytes of persistent state + cache per stream (excludes scratch): constant
 * in the sequence length. */
lola_status lola_state_stream_bytes(const lola_config *cfg, size_t *bytes);

/* Test hook: log every update interval's kept set. dev_buf is a device int32
 * buffer of capacity * B * n_kv_heads * (lambda_ + 1) entries; interval i
 * (counted from the last init/reset) of stream s writes
 * [count, kept token ids in no particular order, -1 padding] at
 * ((i * streams) + s) * (lambda_ + 1).
 * Intervals >= capacity are not logged. NULL disables the log. */
lola_status lola_set_selection_log(lola_state *st, int32_t *dev_buf, int64_t capacity);

/* Test hook: force the kept set of each interval instead of the one the
 * selection kernel computes (the kernel still runs and still logs its own
 * choice). dev_kept has the selection-log layout with ASCENDING token ids and
 * must hold n_intervals * B * n_kv_heads * (lambda_ + 1) entries; an entry whose
 * count is negative leaves that (interval, stream) unforced, and intervals
 * >= n_intervals are not forced. NULL disables forcing. Used to keep
 * a GPU run on the reference trajectory where the top-lambda choice is
 * numerically ambiguous. */
lola_status lola_set_selection_override(lola_state *st, const int32_t *dev_kept,
                                        int64_t n_intervals);

/* Test hook: log the Self-Recall Error the engine computed for every candidate
 * of every update interval (in the precision of the state's tensor-core or SIMT
 * path) and the candidate's token. dev_sre (float) and dev_tok (int32) are
 * device buffers of capacity * B * n_kv_heads * (lambda_ + max(chunk,
 * decode_interval)) entries; candidate c of interval i (counted from the last
 * init/reset) of stream s goes to ((i * streams) + s) * (lambda_ + max(chunk,
 * decode_interval)) + c, cache slots first, then the pairs leaving the window;
 * entries past the interval's candidates are not written. Intervals >= capacity
 * are not logged. NULL pointers (both) disable the log. Used to compare the
 * engine's scores with the reference scores candidate by candidate. */
lola_status lola_set_score_log(lola_state *st, float *dev_sre, int32_t *dev_tok, int64_t capacity);

/* Test hook for failure detection. Arms one bounded device wait that nothing
 * satisfies: where = 1, the tensor-core chain of the next prefill call (or decode
 * interval) waits at its first interval; where = 2 (bfloat16), one warp of the
 * next decode step's streaming kernel waits before its first work item. The wait
 * gives up after wait_limit_ns (1 .. 2e9) nanoseconds, exactly like a real wait
 * that runs out: the kernel records LOLA_ERR_TIMEOUT in the error word, lets its
 * copies and tensor-core work in flight finish, and leaves its work; later kernels
 * of the state that read the chain's per-interval logs skip theirs, and
 * lola_sync() returns LOLA_ERR_TIMEOUT and clears the word. The state's contents
 * are then undefined (reset it). One shot: the hook disarms itself when used;
 * where = 0 disarms it. LOLA_ERR_INVALID_ARG for a target the config does not run
 * (no tensor-core chain, or not bfloat16). */
lola_status lola_set_fault_injection(lola_state *st, int32_t where, int64_t wait_limit_ns);

/* Timing hook: when enabled (enable != 0), every entry point brackets each of
 * its kernel phases with CUDA events recorded on the caller's stream. Phases:
 * 0 feature map, 1 chain (score/select/fold), 2 attention (prefill), 3 call
 * finalisation, 4 decode append, 5 decode interval update, 6 decode attention,
 * 7 state reset. lola_timing_read() waits for the recorded events, adds their
 * elapsed milliseconds to ms[8] and their count to n[8] (caller-zeroed), and
 * forgets them. Host memory; NULL pointers skip the output. */
lola_status lola_set_timing(lola_state *st, int enable);
lola_status lola_timing_read(lola_state *st, double *ms, int64_t *n);

/* Test hook for the tensor-core layer: one CTA computes, on the tcgen05 tensor
 * cores, C[128][N] (fp32, row-major) = A[128][K] * op(B), where A is bf16
 * row-major, and B is bf16 [N][K] with C = A B^T (layout 0, K-major operand)
 * or [K][N] with C = A B (layout 1, N-contiguous operand, N % 64 == 0);
 * layouts 2 and 3 take A as [K][128] (M-contiguous operand) with B as in
 * layouts 1 and 0 respectively.
 * 16 <= N, K <= 256, multiples of 16. Device pointers; dev_err is a device
 * int that receives LOLA's timeout bit if the MMA completion wait gives up.
 * Not part of the method (the paper has no counterpart); it checks the shared
 * memory layouts and descriptors the attention and scoring kernels use. */
lola_status lola_selftest_umma(int layout, const void *A, const void *B, float *C, int N, int K,
                               int *dev_err, void *cuda_stream);

/* Number of kernels this library has launched in the process so far. */
int64_t lola_launch_count(void);

/* Waits for the stream work of this state to finish and reports device-side
 * errors recorded since the last lola_sync (LOLA_ERR_DEVICE / LOLA_ERR_TIMEOUT),
 * clearing them. Once an error is recorded, the kernels that read the chain's
 * per-interval logs (prefill attention, cache finalisation) skip their work until
 * this call clears it; the state must then be reset (lola_reset_state) before its
 * results mean anything again. */
lola_status lola_sync(lola_state *st, void *cuda_stream);

/* Frees the host handle only; the workspace stays the caller's. */
lola_status lola_free_state(lola_state *st);

const char *lola_status_string(lola_status s);

#ifdef __cplusplus
}
#endif
#endif /* LOLA_H */
