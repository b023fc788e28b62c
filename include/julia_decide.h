/*
 * julia_decide.h -- C ABI of the B200 (sm_100a) Julia-1 decision-model library.
 *
 * The library computes the Julia-1 forward pass on pre-tokenized requests:
 * (state, question, 2..20 options, type) rows in; raw option logits,
 * per-question softmax probabilities and the choice / score / noul read-outs
 * out.  Sources (page title, section):
 *   "Julia-1: one score per mask token" -- "From a state to one decision"
 *       (marker layout, budgets, strict mode), "The decision head" (forward
 *       steps), "Three modes through one head" (read-outs);
 *   "Julia-1 MLX" -- "API" (predict / logits / encoding_info over rows),
 *       "Performance" (alternating attention, FP32 residual stream);
 *   "julia1 -- Rust runtime for Julia-1" -- "Use" (validation errors match the
 *       Python ValueError cases), "Why it is faster" (varlen packing, fused
 *       epilogues, marker-only last head layer).
 *
 * Conventions
 *   - Every call returns a jd_status; JD_OK is 0.  On failure a message for
 *     the calling thread is available from jd_last_error().
 *   - Host pointers are read during the call only.  Device pointers must stay
 *     valid until the work queued on the caller's stream has completed.
 *   - "stream" is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Device work is asynchronous on that stream; a kernel-side
 *     check failure (bounded wait expired, id out of range) is recorded in a
 *     device status word and reported by jd_check_status().
 *   - One jd_model serves one stream at a time: its workspace is shared by
 *     all calls on it.
 *   - Nothing in the library falls back to the CPU: without a CUDA device
 *     jd_model_create fails with JD_ERR_CUDA.
 */
#ifndef JULIA_DECIDE_H
#define JULIA_DECIDE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    JD_OK = 0,
    JD_ERR_INVALID_ARG = 1,    /* null pointer, bad option value, mismatched sizes */
    JD_ERR_OPTION_COUNT = 2,   /* K outside [2, 20], or a noul row with K != 2 */
    JD_ERR_OVERFLOW = 3,       /* strict budget violated, or nothing fits when truncating */
    JD_ERR_TOKEN_RANGE = 4,    /* a token id outside [0, vocab) */
    JD_ERR_CAPACITY = 5,       /* batch larger than the capacity given at jd_model_create */
    JD_ERR_CUDA = 6,           /* a CUDA runtime / driver call failed */
    JD_ERR_DEVICE_STATUS = 7,  /* a kernel reported a failed check (see jd_check_status) */
    JD_ERR_IO = 8              /* weights file missing or malformed */
} jd_status;

/* Decision type = row index of the 3x384 type table ("The decision head", step 1). */
typedef enum { JD_CHOICE = 0, JD_SCORE = 1, JD_NOUL = 2 } jd_type;

/* Per-row truncation bits (non-strict encoding only; "Julia-1 MLX", "API":
 * encoding_info reports whether anything was truncated). */
enum {
    JD_TRUNC_OPTION_48 = 1,   /* an option was clipped to 48 ids */
    JD_TRUNC_OPTION_CAP = 2,  /* options were capped to fit the head budget */
    JD_TRUNC_QUESTION = 4,    /* the question was clipped from its end */
    JD_TRUNC_STATE = 8        /* the state was clipped to fit max_length */
};

/* One pre-tokenized request row (host memory).  The type prefix in words
 * ("choice question: ...") is part of the caller's question ids.  For a noul
 * row the options are [false, true] in that order. */
typedef struct {
    const int32_t *state;          /* [n_state] */
    int32_t n_state;
    const int32_t *question;       /* [n_question] */
    int32_t n_question;
    const int32_t *const *options; /* [k] pointers to each option's ids */
    const int32_t *n_option_ids;   /* [k] */
    int32_t k;                     /* number of options, 2..20 */
    int32_t type;                  /* jd_type */
} jd_row;

/* Encoding options ("From a state to one decision": options <= 48 tokens,
 * head budget 256 by default / 512 in the card's example, 8192 in all). */
typedef struct {
    int32_t max_length;   /* 1..8192 */
    int32_t head_budget;  /* >= 1; tokens before the state */
    int32_t strict;       /* nonzero: raise JD_ERR_OVERFLOW instead of truncating */
    int32_t bos, eos, mask;  /* special ids, in [0, vocab) like every other id */
    int32_t vocab;        /* ids must lie in [0, vocab) */
} jd_encode_opts;

/* A packed (unpadded, row after row) batch.  jd_serialize fills one in host
 * memory that the library owns until jd_batch_free.  The same struct with
 * DEVICE pointers (caller-owned) is the input of jd_forward / jd_decide. */
typedef struct {
    int32_t n_rows;         /* B */
    int32_t n_tokens;       /* T = cu_seqlens[B] */
    int32_t n_markers;      /* M = opt_off[B] */
    int32_t max_row_len;    /* longest row, <= 8192 */
    int32_t *tokens;        /* [T]   serialized ids, rows back to back */
    int32_t *cu_seqlens;    /* [B+1] row r spans tokens [cu_seqlens[r], cu_seqlens[r+1]) */
    int32_t *mask_pos;      /* [M]   absolute token index of each <mask> marker, row order */
    int32_t *opt_off;       /* [B+1] row r's markers are mask_pos[opt_off[r] .. opt_off[r+1]) */
    int32_t *row_type;      /* [B]   jd_type of each row */
    int32_t *head_len;      /* [B]   tokens before the state (host batches only; may be NULL) */
    uint8_t *trunc;         /* [B]   JD_TRUNC_* bits (host batches only; may be NULL) */
} jd_batch;

/* Device outputs (caller-owned device memory). */
typedef struct {
    float *logits;     /* [M] raw option logits, row order */
    float *probs;      /* [M] softmax over each row's options (temperature 1) */
    int32_t *choice;   /* [B] argmax option index (lowest index on ties) */
    float *score;      /* [B] expected index sum_i i * p_i */
    float *noul;       /* [B] p(true) = probs of option 1 for noul rows, NaN otherwise */
    float *max_p;      /* [B] largest probability */
} jd_outputs;

/* Optional intermediate taps for validation (device memory, any may be NULL). */
typedef struct {
    float *encoder_out;   /* [T, 384] encoder output after the final norm (before the type row) */
    float *marker_state;  /* [M, 384] marker states after both head layers (scorer input) */
} jd_taps;

/* Precision of jd_model_config.precision.
 *   JD_PREC_BF16  BF16 tensor-core projections and attention, FP32 accumulation, FP32 residual
 *                 stream, norms, embedding, scorer and read-outs ("Julia-1 MLX", "Performance":
 *                 the projections may run at lower precision, the residual stream stays FP32).
 *   JD_PREC_FP32  FP32 everywhere (validation mode).
 *   JD_PREC_FP8   JD_PREC_BF16 with the QKV projections of the 22 encoder layers on FP8 E4M3
 *                 operands (tensor-core kind::f8f6f4, FP32 accumulation): each weight row has
 *                 its own scale (max |row| / 448), and each layer's normalized input one static
 *                 scale, sqrt(384) * max |gain| / 448, the bound of a LayerNorm output, so it
 *                 never saturates.  Every other projection stays BF16: E4M3 inputs of the GEGLU
 *                 up-projection carry their 3-bit mantissa error into residual channels that a
 *                 later projection scales to the thousands the page describes. */
enum { JD_PREC_BF16 = 0, JD_PREC_FP32 = 1, JD_PREC_FP8 = 2 };
enum { JD_SCORER_MLP = 0, JD_SCORER_LINEAR = 1 };
enum { JD_ACT_RELU = 0, JD_ACT_GELU = 1 };

typedef struct {
    int32_t max_tokens;    /* capacity: packed tokens per call */
    int32_t max_rows;      /* capacity: rows per call */
    int32_t max_markers;   /* capacity: markers per call */
    int32_t precision;     /* JD_PREC_BF16, JD_PREC_FP32 (validation mode) or JD_PREC_FP8
                              (E4M3 encoder QKV projections); see the enum above */
    int32_t scorer;        /* JD_SCORER_MLP: LayerNorm -> Linear(384,384) -> GELU -> Linear(384,1)
                              ("The decision head", step 4); JD_SCORER_LINEAR: LayerNorm -> Linear(384,1) */
    int32_t head_act;      /* feed-forward activation of the two head layers (default ReLU) */
} jd_model_config;

typedef struct jd_model jd_model;

/* Thread-local message of the last failed call on this thread ("" if none). */
const char *jd_last_error(void);

/* Library version string. */
const char *jd_version(void);

/* Serialize rows into a packed host batch ("From a state to one decision").
 * Layout per row: <bos> question <eos> (<mask> option)_k <eos> state <eos>.
 * Always errors: K outside [2,20] or noul with K != 2 (JD_ERR_OPTION_COUNT),
 * an id outside [0, vocab), the special ids included (JD_ERR_TOKEN_RANGE).
 * Invalid opts (max_length, head_budget, vocab) -> JD_ERR_INVALID_ARG; opts
 * errors leave *bad_row at -1.  Strict: an option over 48
 * ids, head over budget or total over max_length -> JD_ERR_OVERFLOW.
 * Non-strict: clip options to 48 ids; if the head is over budget cap every
 * option at the largest common length that fits (clip the question from its
 * end if even one id per option does not fit); clip the state to fit
 * max_length; report the JD_TRUNC_* bits per row.  On error *out is NULL and
 * *bad_row (if non-NULL) receives the failing row index. */
jd_status jd_serialize(const jd_row *rows, int32_t n_rows, const jd_encode_opts *opts,
                       jd_batch **out, int32_t *bad_row);
void jd_batch_free(jd_batch *batch);

/* Per-row encoding report ("Julia-1 MLX", "API": encoding_info(rows) gives the
 * lengths a request encodes to and whether anything was truncated). */
typedef struct {
    int32_t length;       /* serialized tokens of the row (head + state + final eos) */
    int32_t head_length;  /* tokens before the state: bos, question, eos, markers, options, eos */
    int32_t state_length; /* state ids kept */
    int32_t n_options;    /* k */
    int32_t truncated;    /* JD_TRUNC_* bits; 0 when nothing was clipped (always 0 in strict mode) */
} jd_encoding_info;

/* The report of a host batch from jd_serialize: per_row[n_rows] (caller-owned
 * host memory).  Errors: JD_ERR_INVALID_ARG for a NULL argument or a batch
 * without its host-side head_len / trunc arrays (a device batch). */
jd_status jd_batch_info(const jd_batch *batch, jd_encoding_info *per_row);

/* The same report straight from rows, with jd_serialize's rules and errors
 * (*bad_row as there); nothing is kept. */
jd_status jd_rows_encoding_info(const jd_row *rows, int32_t n_rows, const jd_encode_opts *opts,
                                jd_encoding_info *per_row, int32_t *bad_row);

/* Load the .jdw weights file and allocate the device workspace for the given
 * capacity on `device` (the architecture of "The decision head" and "Julia-1
 * MLX", "Performance": 22 encoder layers of width 384, a 3 x 384 type table,
 * two head layers, the scorer).  BF16 copies of the projection weights are
 * made here; the embedding table, norms, biases and head stay FP32.  On
 * success *out is a handle the caller owns and releases with
 * jd_model_destroy (NULL is accepted there); on failure *out is NULL.
 * Errors: JD_ERR_INVALID_ARG (NULL argument, a capacity < 1, unknown
 * precision, device index out of range), JD_ERR_CUDA (no CUDA device, a
 * device other than sm_100, an allocation or copy failed), JD_ERR_IO (the
 * weights file is missing, truncated, or lacks a tensor of the expected
 * shape). */
jd_status jd_model_create(const jd_model_config *cfg, const char *weights_path, int device,
                          jd_model **out);
void jd_model_destroy(jd_model *model);

/* A second handle on the weights of `base` with a workspace, staging buffers and
 * CUDA-graph cache of its own, sized by cfg (precision must equal base's; scorer
 * and head_act are this handle's).  "Julia-1 MLX", "Performance": a server taking
 * single requests scores them from several threads, each on its own stream; one
 * handle per thread / stream gives that on one copy of the weights.  Calls on one
 * handle must not overlap (they share its workspace); calls on different handles
 * may run concurrently on different streams.  `base` owns the weights' device
 * memory and must outlive every shared handle; jd_model_destroy(shared) frees only
 * the handle's own memory.  Errors: JD_ERR_INVALID_ARG (NULL, capacities < 1,
 * precision differs), JD_ERR_CUDA (allocation). */
jd_status jd_model_create_shared(const jd_model *base, const jd_model_config *cfg, jd_model **out);

/* Device bytes held by the model (weights + workspace; a shared handle counts its own memory only). */
size_t jd_model_device_bytes(const jd_model *model);

/* Full forward pass and read-outs on a packed batch in device memory ("The
 * decision head", steps 1-4: encoder, type row, two head layers, one scorer
 * logit per <mask> marker; "Three modes through one head": the per-question
 * softmax and the choice / score / noul read-outs).  `batch` is a host struct
 * whose array pointers are device pointers (tokens, cu_seqlens, mask_pos,
 * opt_off, row_type; head_len / trunc are ignored), laid out as jd_serialize
 * writes them.  All outputs of `out` are written; `taps` may be NULL.
 * Errors: JD_ERR_INVALID_ARG (NULL model / batch / output, an empty batch, a
 * row longer than 8192 tokens), JD_ERR_CAPACITY (n_tokens, n_rows or
 * n_markers above the model's capacity), JD_ERR_CUDA (a launch or graph call
 * failed).  Failed device-side checks (an id outside the vocabulary, a marker
 * index outside the batch, a bounded wait that expired) are recorded in the
 * model's status word and reported by jd_check_status. */
jd_status jd_decide(jd_model *model, const jd_batch *batch, const jd_outputs *out,
                    const jd_taps *taps, void *stream);

/* Raw logits only ("Julia-1 MLX", "API": the logits(rows) call): writes
 * logits[M] on the device; probabilities and read-outs go to the model's
 * internal buffers.  Errors as jd_decide. */
jd_status jd_forward(jd_model *model, const jd_batch *batch, float *logits, void *stream);

/* Host outputs of jd_decide_host (caller-owned host memory, sizes as jd_outputs). */
typedef struct {
    float *logits; float *probs; int32_t *choice; float *score; float *noul; float *max_p;
    int32_t n_rows, n_markers;    /* written by the call */
} jd_host_outputs;

/* End-to-end call ("Julia-1 MLX", "API": predict(rows)): serialize `rows`,
 * copy the packed batch to the device through the model's pinned staging
 * buffers, run jd_decide, copy the outputs back and synchronize `stream`.
 * Output arrays must hold the total number of options (logits/probs) and
 * n_rows entries; any of them may be NULL to skip it.  Errors: those of
 * jd_serialize and jd_decide, and JD_ERR_DEVICE_STATUS when a device-side
 * check failed during this call (the outputs are then not written). */
jd_status jd_decide_host(jd_model *model, const jd_row *rows, int32_t n_rows,
                         const jd_encode_opts *opts, jd_host_outputs *out, void *stream);

/* Same as jd_decide_host, starting from an already serialized host batch.
 * JD_ERR_INVALID_ARG while calls of jd_decide_host_submit are uncollected. */
jd_status jd_decide_packed_host(jd_model *model, const jd_batch *host_batch,
                                jd_host_outputs *out, void *stream);

/* jd_decide_host in two halves, so that the host prepares one call while the
 * device runs the previous one (the serving loop of a stream of batches):
 * submit serialises the rows, queues the copies in, the forward pass and the
 * copies back on `stream` through one of two pinned staging slots (the second
 * is allocated on first use), and returns at once with a ticket (0, 1, 2 ...
 * per handle); collect waits for the oldest call in flight and copies its
 * outputs into `out` (host memory; the same outputs as jd_decide_host, and
 * JD_ERR_DEVICE_STATUS if that call's kernels recorded a failure).  At most
 * two calls are in flight (a third submit gives JD_ERR_INVALID_ARG), tickets
 * are collected in order, and the synchronous host calls refuse to run while
 * any is in flight.  The rows need not outlive submit.  Both calls of a
 * handle come from one host thread at a time. */
jd_status jd_decide_host_submit(jd_model *model, const jd_row *rows, int32_t n_rows,
                                const jd_encode_opts *opts, void *stream, int64_t *ticket);
jd_status jd_decide_host_collect(jd_model *model, int64_t ticket, jd_host_outputs *out);

/* A choice question over up to 4096 candidate labels (host memory). */
typedef struct {
    const int32_t *state;
    int32_t n_state;
    const int32_t *question;
    int32_t n_question;
    const int32_t *const *labels;  /* [n_labels] pointers to each label's ids */
    const int32_t *n_label_ids;    /* [n_labels] */
    int32_t n_labels;              /* 1..4096 */
} jd_route_request;

/* Router outputs (host memory, caller-owned; optional arrays may be NULL). */
typedef struct {
    int32_t *winner;            /* required [n_requests] index of the chosen label (NULL: JD_ERR_INVALID_ARG) */
    float *winner_p;            /* optional [n_requests] its probability in the final call (1 if unscored) */
    int32_t *final_candidates;  /* optional [n_requests * 20] label indices of the final call, -1 padded */
    float *final_probs;         /* optional [n_requests * 20] their probabilities (1 for a lone, unscored candidate) */
    int32_t *rows_per_round;    /* optional [max_rounds] rows scored per round, all requests together */
    int32_t max_rounds;         /* >= 0 when rows_per_round is set; rounds beyond it are not recorded */
    int32_t n_rounds;           /* written: rounds including the final call */
} jd_route_outputs;

/* Router ("Julia-1: one score per mask token", "More than 20 options: the
 * Router"): per round, each request with more than 20 candidates is split in
 * order into consecutive groups of at most 20; all groups of all requests are
 * scored together (one batch per round, chunked to max_tokens / max_rows /
 * max_markers, which must not exceed the model's capacity); a group keeps its
 * winner alone if its probability is above 0.95 and every other is below 0.045,
 * else its two most probable candidates, in their original order; a group of
 * one passes through unscored.  With 20 or fewer left, one final call per
 * request picks the winner.  Rows are encoded with `opts` as choice rows. */
jd_status jd_route_host(jd_model *model, const jd_route_request *requests, int32_t n_requests,
                        const jd_encode_opts *opts, int32_t max_tokens, int32_t max_rows, int32_t max_markers,
                        jd_route_outputs *out, void *stream);

/* jd_route_host with the tournament on the device ("Julia-1: one score per
 * mask token", "More than 20 options: the Router"; no counterpart API on the
 * pages): the requests are copied to the device once; every round's rows are
 * then formed, encoded with `opts` (the serializer's layout and budget rules,
 * strict or not) and packed by kernels, scored by the forward pass, and
 * narrowed by the same survivor rule, with no host serialisation between
 * rounds.  Per round the host reads back only the round's row, token and
 * marker counts and longest row (four ints) to size the next launches; the
 * outputs come back once at the end.  Outputs equal jd_route_host's on the
 * same model (no row's result depends on the rest of its batch).
 * Differences: every id of every request is checked against opts->vocab up
 * front (JD_ERR_TOKEN_RANGE), and a round must fit the model's capacity in
 * one batch (JD_ERR_CAPACITY; jd_route_host splits rounds into chunks).
 * Strict overflow in a round gives JD_ERR_OVERFLOW.  The device workspace
 * grows on first use (one allocation, kept by the model).  `stream` may be
 * NULL; the call synchronizes it once per round. */
jd_status jd_route_device(jd_model *model, const jd_route_request *requests, int32_t n_requests,
                          const jd_encode_opts *opts, jd_route_outputs *out, void *stream);

/* Scoring callback of jd_route_scored: score n_rows choice rows (host memory,
 * valid during the call) and write the probabilities of every option of every
 * row, in row order, into probs (host memory, one entry per option of the
 * rows).  Any status other than JD_OK ends the route with that status. */
typedef jd_status (*jd_route_scorer)(void *user, const jd_row *rows, int32_t n_rows, float *probs);

/* The same tournament as jd_route_host with the scoring left to `scorer`
 * (jd_route_host is this with the model's forward pass as the scorer): the
 * grouping, the survivor rule, the final call and the outputs are identical.
 * Needs no device.  Errors: JD_ERR_INVALID_ARG (NULL scorer / out / winner, a
 * request without labels or with more than 4096), or the scorer's status. */
jd_status jd_route_scored(const jd_route_request *requests, int32_t n_requests, jd_route_scorer scorer,
                          void *user, jd_route_outputs *out);

/* Synchronize the model's last stream and read the device status word;
 * JD_ERR_DEVICE_STATUS with a message if a kernel recorded a failure. */
jd_status jd_check_status(jd_model *model);

/* CUDA-graph mode ("Julia-1 MLX", "Performance": batch-1 requests, where the
 * fixed cost of each call decides the latency).  enable = 0 turns it off (the
 * default: every call launches its kernels).  In graph mode a call runs its
 * batch padded to a bucket: n_tokens rounded up from n_tokens + 8 to a
 * multiple of 128, n_rows + 1 rows and n_markers rounded up from n_markers + 1
 * to a multiple of 8; the added last row holds the extra tokens (id 0) and
 * markers.  Each bucket's launch sequence is captured once, into a graph that
 * reads the padded batch from the model's own staging arrays; every later
 * call of that bucket, whatever its exact shape and pointers, copies its
 * batch there (jd_decide: one small kernel; jd_decide_packed_host /
 * jd_decide_host: the host-to-device copies it makes anyway), replays the
 * graph and copies its rows' outputs out.  No row's result depends on the
 * rest of its batch, so the outputs equal those of eager launches bit for bit
 * (the marker attention's key split, which depends on the longest row, is kept
 * by bucketing that length too).  At most 64 buckets are kept, the least
 * recently used dropped first.  Calls whose padded batch exceeds the model's
 * capacity, and jd_decide calls with taps, use one graph keyed on their exact
 * shape and pointers instead, captured again whenever those change. */
jd_status jd_set_graph_mode(jd_model *model, int enable);

/* Graph-mode counters of this handle since it was created: graphs captured,
 * calls served by replaying a graph captured earlier, buckets held now.  Any
 * pointer may be NULL. */
jd_status jd_graph_stats(const jd_model *model, int64_t *captures, int64_t *replays, int32_t *buckets);

/* Number of kernels the last jd_decide / jd_forward call launched (the same
 * sequence whether replayed from a graph or launched eagerly). */
int32_t jd_last_launch_count(const jd_model *model);

/* Per-kernel timing for measurement: when enabled, every launch of the
 * sequence is bracketed by CUDA events on the caller's stream, each call
 * synchronizes that stream before returning, and the elapsed times are summed
 * per kernel name.  Enabling (or disabling) clears the sums.  Graph replay is
 * not used while profiling. */
jd_status jd_set_profiling(jd_model *model, int enable);

/* Write the sums as text lines "name launches total_ms" into buf (size n).
 * JD_ERR_INVALID_ARG if buf is too small. */
jd_status jd_profile_report(jd_model *model, char *buf, size_t n);

/* jd_forward without any device allocation (no counterpart on the pages; it
 * serves callers that may not call the CUDA allocator once they are running,
 * e.g. a serving loop held to the memory budget it reserved at start-up, or a
 * host application that owns all device allocation).  Same inputs and output
 * as jd_forward: `batch` with device arrays, raw logits[M] on the device.
 * Every intermediate lives in one file-scope __device__ array of about 9.7 MB
 * that each GPU loading the library holds until the process exits.
 *   - Limits: at most 1024 packed tokens, 32 rows and 128 markers per call
 *     (JD_ERR_CAPACITY beyond them); BF16 models only (JD_ERR_INVALID_ARG).
 *   - jd_model_create (BF16) loads the module holding the array, resolves its
 *     device address and describes its buffers for TMA, so that this entry
 *     point allocates nothing from its first call on.  The model (weights)
 *     must therefore come from jd_model_create, called at start-up.
 *   - All calls share the array, and each call leaves its intermediates there:
 *     calls whose work overlaps on the GPU (different streams, or models on
 *     the same device used concurrently) race and must be serialized by the
 *     caller.
 *   - The kernels' device status word (an id outside the vocabulary, a marker
 *     index outside the batch, a bounded wait that expired) lives in the array
 *     too and is cleared at the start of every call: read it with
 *     jd_noalloc_check_status after the call and before the next one.
 *     jd_check_status does not cover these calls. */
jd_status jd_forward_noalloc(jd_model *model, const jd_batch *batch, float *logits, void *stream);

/* Status of the last jd_forward_noalloc call on the model's device (no
 * counterpart on the pages): synchronizes `stream` (the call's stream), reads
 * the array's device status word (a copy into host memory; nothing is
 * allocated) and returns JD_ERR_DEVICE_STATUS with a message when a kernel
 * recorded a failed check, JD_OK otherwise.  The logits of a call that
 * reports a failure are not meaningful.  Errors: JD_ERR_INVALID_ARG (NULL
 * model, FP32 model), JD_ERR_CUDA (the synchronization or copy failed). */
jd_status jd_noalloc_check_status(jd_model *model, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* JULIA_DECIDE_H */
