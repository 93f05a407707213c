/*
 * focus.h -- C ABI of one FOCUS focused denoising step on an NVIDIA B200 (sm_100a).
 *
 * FOCUS ("FOCUS: DLLMs Know How to Tame Their Compute Bound", project page,
 * Overview) speeds up block-diffusion LLM decoding: every denoising step runs the
 * model over a whole block of B tokens on top of an exactly cached prefix
 * (Overview -- Motivation), but only a few block positions become decodable per
 * step.  One focused step therefore
 *   1. runs layers 0 and 1 on the full block and scores every position by its
 *      attention-derived importance at both layers (Overview -- Design: importance
 *      "after the early Q/K projections"),
 *   2. turns the layer-0-to-1 importance delta (Overview -- Decodability Signal)
 *      into an adaptive per-request budget and keeps the top positions
 *      (Overview -- Runtime Action: dynamic budgeting, token eviction),
 *   3. compacts the kept rows into a ragged batch and runs layers 2..L-1 on them
 *      only, with ragged paged attention over the prefix pages plus an
 *      intra-block KV cache that holds the evicted positions' last K/V
 *      (Overview -- Runtime Action: ragged execution, intra-block KV caching;
 *      the news article's "Arquitetura do FOCUS": state compaction and ragged
 *      paged attention),
 *   4. scores the kept rows with the LM head and decodes those whose max-softmax
 *      confidence clears a threshold (project page, Quality table, "Conf.").
 *
 * Exact rules (all of them readings of pages that print no formula):
 *   importance I_l[b][j] = sum over query heads h and block query rows i of
 *       softmax_i(q_i . K^T / sqrt(d))[P_b + j], the softmax over the P_b prefix
 *       keys and the B block keys;
 *   delta = I_1 - I_0;  c_b = #{masked j : delta_j > tau};
 *   k_b = min(clamp(ceil(alpha * c_b), k_min, k_max), #masked)  (float32 product);
 *   kept = first k_b masked positions by (delta desc, j asc), listed ascending;
 *   forced_keep_frac f >= 0 instead keeps min(B, ceil(f * B)) of all positions by
 *       (masked first, delta desc, j asc); f = 1 is the dense full-block step;
 *   conf = max softmax of the logits, top id = lowest id among the maxima;
 *   a kept masked position decodes when conf > conf_threshold; if none does but
 *       the request kept a masked position, the one with the highest conf decodes
 *       (lowest j on ties).
 *
 * Conventions
 *   - All pointers inside the structs below are DEVICE pointers on the device
 *     that was current at focus_init, except focus_weights' per-layer pointer
 *     arrays themselves, which are HOST arrays (of device pointers) read during
 *     focus_init only.
 *   - Every tensor is dense row-major with the shape given (last index fastest).
 *   - Element type "T" is float32 when cfg.dtype == FOCUS_DTYPE_F32 and bfloat16
 *     when cfg.dtype == FOCUS_DTYPE_BF16.  Residual streams, importance and
 *     confidences are float32 in both cases.
 *   - Ownership: weights and batch/output buffers are borrowed from the caller and
 *     must stay valid while any call that uses them is in flight; the context owns
 *     only its workspace.
 *   - Errors: every entry point returns FOCUS_OK (0) or a negative FOCUS_ERR_*.
 *     Nothing throws across the ABI.  focus_step is asynchronous: argument errors
 *     visible on the host are returned at once; problems found on the device
 *     (bad page ids, prefix beyond the page table, token ids out of range, a
 *     bounded wait that expired) set the context's device error word instead of
 *     faulting, and focus_get_device_error reports them after a sync.
 */
#ifndef FOCUS_H_
#define FOCUS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------- */
#define FOCUS_OK                 0
#define FOCUS_ERR_INVALID_ARG   -1  /* null pointer, bad shape or parameter */
#define FOCUS_ERR_LIMITS        -2  /* request exceeds the limits given at init */
#define FOCUS_ERR_CUDA          -3  /* a CUDA runtime call failed */
#define FOCUS_ERR_TIMEOUT       -4  /* a device-side bounded wait expired */
#define FOCUS_ERR_DEVICE_BOUNDS -5  /* device-side index check failed (page id, prefix, token id, forced set) */
#define FOCUS_ERR_UNSUPPORTED   -6  /* shape the kernels do not handle (see focus_init) */
#define FOCUS_ERR_NO_MEMORY     -7  /* workspace allocation failed */

/* device error word bits (focus_get_device_error) */
#define FOCUS_DEVERR_TOKEN_ID    0x1   /* block token id outside [0, V) -- read as 0 */
#define FOCUS_DEVERR_PAGE_ID     0x2   /* page id outside [0, n_pages) -- that page skipped */
#define FOCUS_DEVERR_PREFIX      0x4   /* prefix_len < 0 or beyond the page table -- clamped */
#define FOCUS_DEVERR_TIMEOUT     0x8   /* a pipeline wait gave up -- outputs are invalid */
#define FOCUS_DEVERR_FORCED_SET  0x10  /* forced keep set not ascending / out of range -- request keeps nothing */

typedef enum { FOCUS_DTYPE_F32 = 0, FOCUS_DTYPE_BF16 = 1 } focus_dtype;

/* ---- model ---------------------------------------------------------------- */
/* A pre-norm decoder: RMSNorm, grouped-query attention with rotate-half RoPE,
 * residual, RMSNorm, SwiGLU MLP, residual; final RMSNorm and an untied LM head. */
typedef struct {
    int32_t n_layers;    /* L >= 2 (the delta needs layers 0 and 1) */
    int32_t hidden;      /* D */
    int32_t n_q_heads;   /* Hq, a multiple of n_kv_heads */
    int32_t n_kv_heads;  /* Hkv */
    int32_t head_dim;    /* d: 64 or 128 (bf16 needs 128) */
    int32_t ffn;         /* F */
    int32_t vocab;       /* V */
    float   rms_eps;     /* RMSNorm epsilon */
    float   rope_theta;  /* RoPE base: pair i turns by pos * theta^(-2i/d) */
    int32_t dtype;       /* focus_dtype */
} focus_model_cfg;

/* Weights, row-major [out_features, in_features] (y = x W^T), element type T. */
typedef struct {
    const void* embed;               /* [V, D] */
    const void* final_norm;          /* [D] */
    const void* lm_head;             /* [V, D] */
    const void* const* wqkv;         /* host array of L: [(Hq + 2 Hkv) d, D]; rows = q heads, k heads, v heads */
    const void* const* wo;           /* host array of L: [D, Hq d] */
    const void* const* wgate;        /* host array of L: [F, D] */
    const void* const* wup;          /* host array of L: [F, D] */
    const void* const* wdown;        /* host array of L: [D, F] */
    const void* const* attn_norm;    /* host array of L: [D] */
    const void* const* mlp_norm;     /* host array of L: [D] */
} focus_weights;

/* Upper bounds that size the context's workspace. */
typedef struct {
    int32_t max_requests;       /* N bound */
    int32_t max_block;          /* B bound, <= 64 */
    int32_t max_keep;           /* bound on kept positions per request (k_max, or ceil(f B) when forced) */
    int32_t max_pages_per_req;  /* row length of page_table; prefix_len <= this * page_size */
} focus_limits;

/* ---- one step --------------------------------------------------------------- */
typedef struct {
    int32_t n_requests;          /* N */
    int32_t block_size;          /* B */
    int32_t page_size;           /* S: tokens per KV page (bf16 models: 16, 32 or 64) */
    int32_t n_pages;             /* number of pages in kv_pool */
    int32_t* block_tokens;       /* [N, B] int32, updated in place: decoded positions get their id */
    uint8_t* mask;               /* [N, B] uint8, nonzero = still masked; updated in place (decoded -> 0) */
    const int32_t* prefix_len;   /* [N] int32: P_b, exact-cached prefix tokens of request b */
    const int32_t* page_table;   /* [N, max_pages_per_req] int32: page ids of request b's prefix, in order */
    const void* kv_pool;         /* [n_pages, L, 2, Hkv, S, d] T: post-RoPE prefix K (index 0) and V (1) */
    void* ibc;                   /* [N, L, 2, Hkv, B, d] T: intra-block KV cache, read and written */
} focus_batch;

typedef struct {
    float   tau;                 /* delta threshold of the budget count */
    float   alpha;               /* budget multiplier on the count (1.0 = the count itself) */
    float   conf_threshold;      /* decode when conf > this */
    float   forced_keep_frac;    /* < 0: adaptive budget; in [0, 1]: keep ceil(f B) of all positions */
    int32_t k_min;               /* budget floor */
    int32_t k_max;               /* budget ceiling, <= B and <= limits.max_keep */
    /* optional: a caller-chosen kept set replaces the selection (NULL = off).
     * [N, max_keep] int32 ascending positions, count in forced_keep_count [N]. */
    const int32_t* forced_keep_idx;
    const int32_t* forced_keep_count;
} focus_params;

typedef struct {
    int32_t* keep_count;     /* [N]          k_b */
    int32_t* retained_idx;   /* [N, max_keep] kept positions ascending, -1 padded */
    int32_t* row_offsets;    /* [N + 1]      exclusive scan of keep_count (compacted row ranges) */
    int32_t* decoded_ids;    /* [N, B]       id decoded at (b, j) this step, -1 elsewhere */
    float*   conf;           /* [N, max_keep] confidence of each kept slot (0 where unused) */
    int32_t* top_id;         /* [N, max_keep] top id of each kept slot (-1 where unused) */
    float*   importance;     /* optional [2, N, B] float32: I_0, I_1 (NULL = not written) */
    float*   hidden;         /* optional [N * max_keep, D] float32: residual after layer L-1 of the
                                compacted rows, rows 0 .. R-1 in row_offsets order (NULL = not written) */
} focus_step_out;

typedef struct focus_ctx focus_ctx;

/* Validate the model and limits, record the (borrowed) weight pointers, allocate
 * the workspace and build the TMA descriptors of every weight matrix.  Uses the
 * current CUDA device.  Supported: L >= 2, Hq % Hkv == 0, d in {64, 128} (128 for
 * bf16), D % 128 == 0 and D <= 4096, F % 64 == 0, B <= 64, max_keep <= max_block.
 * Returns FOCUS_OK and *out, or an error with *out = NULL: FOCUS_ERR_INVALID_ARG (null
 * pointers, a missing weight, an inconsistent model), FOCUS_ERR_UNSUPPORTED (a shape outside
 * the list above), FOCUS_ERR_NO_MEMORY (workspace) or FOCUS_ERR_CUDA. */
int focus_init(const focus_model_cfg* cfg, const focus_weights* w, const focus_limits* lim, focus_ctx** out);

/* Enqueue one focused denoising step on `stream` (a cudaStream_t; NULL = legacy
 * default stream).  No host synchronisation inside; the launch sequence depends
 * only on the host-visible sizes (N, B, parameters), so it can be captured in a
 * CUDA graph.  Outputs are valid once the stream has completed.  Two steps on
 * the same context must not overlap in time (the workspace is shared).  The
 * device current at the call must be the context's.  N == 0 returns FOCUS_OK and
 * launches nothing.  Returns FOCUS_ERR_INVALID_ARG (null handle or buffer, N < 0,
 * B <= 0, k_min > k_max, k_max > B, a NaN tau / threshold, alpha < 0, a forced
 * fraction above 1, forced_keep_idx without forced_keep_count or the reverse,
 * another device current), FOCUS_ERR_LIMITS (N, B or the kept bound beyond the
 * limits), FOCUS_ERR_UNSUPPORTED (a bf16 model with a page size other than 16, 32
 * or 64) or FOCUS_ERR_CUDA (a launch failed); device-side problems go to the
 * device error word (see Conventions). */
int focus_step(focus_ctx* ctx, const focus_batch* in, const focus_params* p, focus_step_out* out, void* stream);

/* ---- around the step: one block to completion --------------------------------
 * The loop a block-diffusion decoder runs around the focused step (project page, Overview --
 * Motivation: every denoising step computes the block on top of an exactly cached prefix; a decoded
 * block becomes part of that prefix).  Readings: the block's first step is dense (forced keep
 * fraction 1, filling the intra-block cache); focused steps follow until no position is masked (the
 * decode rule's fallback decodes at least one masked position of every request that has one, so at
 * most B steps); the decoded block is computed once more densely so that its cache holds the final
 * tokens' K/V; that cache is committed to the prefix pages.
 *
 * focus_commit_block copies in->ibc [N, L, 2, Hkv, B, d] into in->kv_pool at positions
 * P_b .. P_b + B - 1 of every request (pages from in->page_table, which must already map those
 * positions; the last prefix page may be shared) and then adds B to in->prefix_len[b].  It is the one
 * call that WRITES kv_pool and prefix_len (the pointers are declared const for the step, which only
 * reads them).  Asynchronous, two kernel launches.  Positions without a valid page set
 * FOCUS_DEVERR_PAGE_ID and are skipped; a prefix length outside [0, max_pages_per_req * page_size] sets
 * FOCUS_DEVERR_PREFIX and leaves that request untouched.  Returns FOCUS_OK, FOCUS_ERR_INVALID_ARG,
 * FOCUS_ERR_LIMITS or FOCUS_ERR_CUDA. */
int focus_commit_block(focus_ctx* ctx, const focus_batch* in, void* stream);

/* Run the loop above on `in` with `p` (p->forced_keep_frac is ignored: the loop's own steps are dense
 * or adaptive; p->forced_keep_idx must be NULL) and commit the block.  `out` receives each step's
 * outputs in turn (the last one is the dense refresh, which decodes nothing).  Synchronises `stream`
 * after every step to read how many positions are still masked, so it cannot be captured in a CUDA
 * graph.  Needs limits.max_keep >= B.  *steps_taken (if not NULL) receives the number of decoding
 * steps.  If positions are still masked after max_steps decoding steps, nothing is committed and
 * FOCUS_ERR_LIMITS is returned.  Other returns as for focus_step / focus_commit_block. */
int focus_decode_block(focus_ctx* ctx, const focus_batch* in, const focus_params* p, int32_t max_steps,
                       focus_step_out* out, int32_t* steps_taken, void* stream);

/* Free the workspace.  Synchronises the device first.  NULL is accepted. */
int focus_destroy(focus_ctx* ctx);

/* Static description of a status code; never NULL. */
const char* focus_status_string(int status);

/* Synchronise the device, read and clear the device error word.  Returns
 * FOCUS_OK if it was clear, FOCUS_ERR_TIMEOUT if a wait expired, else
 * FOCUS_ERR_DEVICE_BOUNDS; *bits (if not NULL) receives the raw FOCUS_DEVERR_* bits. */
int focus_get_device_error(focus_ctx* ctx, int32_t* bits);

/* Failure-path probe (no counterpart in the paper): enqueue one CTA whose pipeline wait -- the same
 * bounded mbarrier wait the GEMM and attention kernels use -- is never satisfied.  After about a second
 * the wait gives up, sets FOCUS_DEVERR_TIMEOUT in the context's device error word and the kernel
 * returns, so focus_get_device_error then reports FOCUS_ERR_TIMEOUT and the context stays usable (no
 * trap, no fault).  For health checks of the failure path.  The device current at the call must be
 * the context's.  Returns FOCUS_OK, FOCUS_ERR_INVALID_ARG or FOCUS_ERR_CUDA. */
int focus_probe_wait_timeout(focus_ctx* ctx, void* stream);

/* Size in bytes of the workspace a context with these limits allocates (0 on bad arguments). */
size_t focus_workspace_bytes(const focus_model_cfg* cfg, const focus_limits* lim);

/* ---- launch accounting and per-kernel timing ---------------------------------- */
/* Kernel classes of one step (the GEMMs of layers 0-1 on all N*B rows are separate from the
 * same GEMMs of layers 2..L-1 on the kept rows). */
typedef enum {
    FOCUS_K_EMBED_NORM = 0,      /* embedding gather + RMSNorm */
    FOCUS_K_QKV_FINALIZE = 1,    /* split-K sum, RoPE, q rows, intra-block KV-cache write */
    FOCUS_K_ATTN_SCORE = 2,      /* layers 0-1 attention with fused importance column sums */
    FOCUS_K_ATTN_RAGGED = 3,     /* layers 2..L-1 ragged paged attention of the kept rows */
    FOCUS_K_ROW_NORM = 4,        /* residual reduction + RMSNorm (and the kept-row gather) */
    FOCUS_K_SELECT = 5,          /* delta, budget, top-k, row map */
    FOCUS_K_DECODE = 6,          /* LM-head combine + threshold decode */
    FOCUS_K_GEMM_FULL_QKV = 7,   /* layers 0-1 GEMMs, all rows */
    FOCUS_K_GEMM_FULL_O = 8,
    FOCUS_K_GEMM_FULL_GATEUP = 9,
    FOCUS_K_GEMM_FULL_DOWN = 10,
    FOCUS_K_GEMM_QKV = 11,       /* layers 2..L-1 GEMMs, kept rows */
    FOCUS_K_GEMM_O = 12,
    FOCUS_K_GEMM_GATEUP = 13,
    FOCUS_K_GEMM_DOWN = 14,
    FOCUS_K_GEMM_LMHEAD = 15,    /* LM head with the fused max / sum-exp / argmax epilogue */
    FOCUS_K_COUNT = 16
} focus_kernel_class;

/* Number of kernels the most recent focus_step on this context enqueued (-1 if none ran). */
int focus_last_step_launches(const focus_ctx* ctx);

/* From now on, record a CUDA event pair (on the step's stream) around every launch of
 * `kernel_class` in later focus_step calls, for at most `max_launches` launches.  Host-side only;
 * costs two event records per timed launch.  A step captured into a CUDA graph while recording keeps
 * the pairs as event nodes: focus_profile_end then reports the most recent replay.  Returns
 * FOCUS_ERR_INVALID_ARG on a bad class. */
int focus_profile_begin(focus_ctx* ctx, int kernel_class, int max_launches);

/* Stop recording, synchronise the device, and return the summed device time of the recorded
 * launches in milliseconds and how many were recorded. */
int focus_profile_end(focus_ctx* ctx, float* total_ms, int32_t* launches);

/* ---- allocation-free LM-head confidence ---------------------------------------
 * No counterpart in the paper: this entry point exists for callers that may not call the CUDA
 * allocator (a thread recording a CUDA graph, a serving loop with a fixed memory budget, a plug-in
 * whose host framework owns all device memory).  It runs the step's last stage -- final RMSNorm,
 * LM head, max-softmax confidence, top id (lowest id among equal maxima) -- on hidden rows the
 * caller holds, and allocates nothing: its intermediate data lives in one fixed array of about
 * 5.75 MiB inside the library, which every GPU that loads the library keeps until the process exits.
 * It uses focus_step's norm routine and LM-head GEMM kernel; top ids equal focus_step's, confidences
 * equal them up to the float summation order in which the vocabulary tiles are merged.
 *
 *   hidden      [rows, hidden_dim] float32, device, 16-byte aligned: residual-stream rows (e.g.
 *               focus_step_out.hidden)
 *   final_norm  [hidden_dim] bf16, device, 8-byte aligned;  lm_head [vocab, hidden_dim] bf16, device,
 *               16-byte aligned
 *   conf        [rows] float32, device (out); top_id [rows] int32, device (out); both 4-byte aligned
 *   stream      cudaStream_t (NULL = legacy default stream); the call is asynchronous
 *
 * Limits: rows <= 256, hidden_dim <= 4096 and a multiple of 128, vocab <= 163840; larger sizes return
 * FOCUS_ERR_LIMITS (FOCUS_ERR_UNSUPPORTED for a hidden_dim that is not a multiple of 128) and launch
 * nothing; a misaligned pointer returns FOCUS_ERR_INVALID_ARG before any device call.  rows == 0
 * returns FOCUS_OK at once.  The first call on a device looks up the array's
 * device address (with that device current) and must therefore come before any stream capture on
 * that device.  All calls on a device share the array: calls that may overlap on the GPU race on it
 * and must be serialised by the caller.  If a bounded wait inside the GEMM expires, conf is NaN and
 * top_id is -1 for every row.  Returns FOCUS_OK, FOCUS_ERR_INVALID_ARG, FOCUS_ERR_LIMITS,
 * FOCUS_ERR_UNSUPPORTED or FOCUS_ERR_CUDA. */
int focus_lm_head_conf_noalloc(const float* hidden, int32_t rows, int32_t hidden_dim, const void* final_norm,
                               const void* lm_head, int32_t vocab, float rms_eps, float* conf, int32_t* top_id,
                               void* stream);

#ifdef __cplusplus
}
#endif
#endif /* FOCUS_H_ */
