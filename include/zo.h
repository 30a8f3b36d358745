/*
 * zo.h -- C ABI of the B200 two-point zeroth-order (ZO) probe step.
 *
 * The method ("Zeroth-Order Fine-Tuning Was an Inference Workload All Along",
 * sections "Why ZO Fine-Tuning Is Really Scoring" and "The System
 * Reorganization"): for a direction z = U V^T (LoZO, rank r) score every
 * prompt under theta + eps z and theta - eps z as token log-probability
 * objectives L+ and L-, form c = (L+ - L-) / (2 eps) with no 1/r factor, and
 * apply theta <- theta - eta c z.  V is held for a window of nu steps and the
 * update accumulates on the U side (U_{t+1} = U_t - eta c_t G_t,
 * Delta W = U_{t+1} V^T), so theta is never materialised: the library keeps
 * a persistent bank of factored slots (A_k, V_k), one per window, and the
 * frozen base weights are only read ("Inference-Native Zeroth-Order
 * Optimization", abstract: candidate states as factorised side states,
 * lazy updates and banks over frozen base weights; the probes of one step
 * form a ProbePlan of logical queries whose physical realisation the backend
 * chooses).
 *
 * Conventions for every call:
 *  - Return value: ZO_OK or a ZO_ERR_* code; zo_last_error(h) gives a
 *    static message for the last failure on that handle (NULL handle: the
 *    last failure of zo_create).
 *  - "dev" pointers are CUDA device pointers, "host" pointers host memory.
 *    The library never frees or writes caller memory other than the output
 *    arguments named below.
 *  - All device work is queued on the handle's stream (zo_options.stream)
 *    and is asynchronous; only calls that return host data (zo_step with a
 *    non-NULL c_out, zo_read_*, zo_stats, zo_save_state) synchronise it.
 *  - Rows: each prompt is a sequence of token ids whose LAST target_lens[i]
 *    tokens are the scored span; the objective of a row is the mean of
 *    -log p(token | prefix) over its span.  seq_len >= target_len + 1.
 */
#ifndef ZO_H
#define ZO_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes -------------------------------------------------------------------- */
enum {
    ZO_OK = 0,
    ZO_ERR_ARG = 1,          /* invalid argument (sizes, NULL, out of range, mismatch)     */
    ZO_ERR_STATE = 2,        /* wrong call order (no score before step, wrong step index) */
    ZO_ERR_CUDA = 3,         /* a CUDA runtime call failed                                 */
    ZO_ERR_OOM = 4,          /* device or pinned allocation failed                         */
    ZO_ERR_NONFINITE = 5,    /* L+ or L- not finite: update refused, bank unchanged        */
    ZO_ERR_TIMEOUT = 6,      /* a bounded device wait expired                              */
    ZO_ERR_UNSUPPORTED = 7   /* shape or option outside what the kernels implement          */
};

enum { ZO_ARCH_OPT = 0, ZO_ARCH_QWEN3 = 1 };
enum { ZO_DTYPE_FP32 = 0, ZO_DTYPE_BF16 = 1 };
/* Matrix ids (also the bit positions of zo_targets.matrix_mask).  OPT uses
 * UP for fc1 and DOWN for fc2 and has no GATE. */
enum { ZO_MAT_Q = 0, ZO_MAT_K = 1, ZO_MAT_V = 2, ZO_MAT_O = 3,
       ZO_MAT_GATE = 4, ZO_MAT_UP = 5, ZO_MAT_DOWN = 6 };
/* LOZO: factors as drawn.  MEZO: both factors scaled by fp32(1/sqrt(r)), the
 * high-rank factorised variant that tracks MeZO ("Zeroth-Order Fine-Tuning
 * Was an Inference Workload All Along", section "The System Reorganization",
 * last paragraph). */
enum { ZO_SCALE_LOZO = 0, ZO_SCALE_MEZO = 1 };

/* ---- model ------------------------------------------------------------------------- */
typedef struct zo_model_desc {
    int32_t arch;            /* ZO_ARCH_*                                                  */
    int32_t n_layers;
    int32_t d_model;
    int32_t n_heads;
    int32_t n_kv_heads;      /* == n_heads for OPT                                         */
    int32_t head_dim;        /* 128 for the shapes the library is tuned for; <= 256         */
    int32_t d_ffn;
    int32_t vocab;
    int32_t max_pos;         /* longest row: OPT rows of pos_embed, Qwen3 rotary table size */
    float   norm_eps;        /* LayerNorm (OPT) / RMSNorm (Qwen3) epsilon                   */
    float   rope_theta;      /* Qwen3 rotary base                                           */
    int32_t dtype;           /* ZO_DTYPE_*: matrices and embeddings                         */
    int32_t tie_lm_head;     /* 1: lm_head is tok_embed                                     */
} zo_model_desc;

/* One decoder layer.  Matrices are [d_out, d_in] row-major (K contiguous: y =
 * x W^T) in the model dtype; biases and norm parameters are fp32.  Unused
 * entries (OPT gate, Qwen3 biases/LN shifts, OPT q/k norms) are NULL. */
typedef struct zo_layer_weights {
    const void*  w[7];       /* indexed by ZO_MAT_*                                        */
    const float* b[7];
    const float* ln1_w;      /* pre-attention norm scale [d]                               */
    const float* ln1_b;      /* pre-attention LayerNorm shift [d] (OPT)                    */
    const float* ln2_w;      /* pre-FFN norm scale [d]                                     */
    const float* ln2_b;
    const float* q_norm;     /* Qwen3 per-head RMSNorm scales [head_dim]                   */
    const float* k_norm;
} zo_layer_weights;

/* Frozen base weights: DEVICE pointers, borrowed read-only for the lifetime
 * of the handle (the caller owns and frees them; the library never writes
 * them).  layers is a HOST array of n_layers entries, copied at create. */
typedef struct zo_weights {
    const void*  tok_embed;  /* [vocab, d] model dtype                                     */
    const void*  pos_embed;  /* [max_pos, d] model dtype (OPT), NULL for Qwen3             */
    const float* final_w;    /* final norm scale [d]                                       */
    const float* final_b;    /* final LayerNorm shift [d] (OPT)                            */
    const void*  lm_head;    /* [vocab, d]; ignored when tie_lm_head                        */
    const zo_layer_weights* layers;
} zo_weights;

/* Which matrices carry the direction: layers in layer_mask (bit l of
 * lo for l < 64, of hi for 64 <= l < 128), matrices in matrix_mask. */
typedef struct zo_targets {
    uint64_t layer_mask_lo;
    uint64_t layer_mask_hi;
    uint32_t matrix_mask;
    int32_t  scale_mode;     /* ZO_SCALE_*                                                 */
} zo_targets;

typedef struct zo_options {
    uint64_t   run_seed;     /* seeds the direction stream                                 */
    int32_t    lazy_interval;/* nu: V held for nu steps (>= 1)                              */
    int32_t    rank;         /* r                                                          */
    zo_targets targets;
    int32_t    max_tokens;   /* physical tokens per score call (probe rows count twice)     */
    int32_t    max_rows;     /* physical rows per score call                               */
    int32_t    max_scored;   /* scored positions per score call                            */
    int32_t    max_slots;    /* bank windows kept (>= 1); more windows -> ZO_ERR_UNSUPPORTED */
    uint64_t   start_step;   /* first step index (0 for a fresh run)                        */
    void*      stream;       /* cudaStream_t; NULL = legacy default stream                  */
    int32_t    impl;         /* 0: tensor cores wherever they apply (bf16), 1: CUDA cores only */
    int32_t    profile;      /* 1: time every GEMM launch with CUDA events (zo_stats gemm_*) */
    int32_t    fp8;          /* 1: the base products fed by a norm (q|k|v and the FFN input
                                projections) run in E4M3 on the tensor cores ("Inference-Native
                                Zeroth-Order Optimization", abstract: the queries inherit the
                                runtime's quantisation): weights quantised once per output
                                channel at zo_create, activations per token by the norm kernel
                                (scale = amax / 448, round to nearest even, saturated).  The
                                direction, bank and every other GEMM stay in the model dtype.
                                bf16 models with impl 0 only, else ZO_ERR_UNSUPPORTED.  0: off */
    int32_t    max_new;      /* most tokens zo_generate decodes per row (0: no generation);
                                sizes the KV cache: n_layers x (max_tokens + max_rows * max_new)
                                rows of 2 * n_kv_heads * head_dim elements                   */
} zo_options;

typedef struct zo_handle zo_handle;
typedef struct zo_plan zo_plan;

typedef struct zo_stats_t {
    uint64_t steps;                 /* completed zo_step calls                              */
    uint64_t score_calls;
    uint64_t tokens_scored;         /* physical prefill tokens processed                   */
    uint64_t positions_scored;      /* target tokens whose log-prob was produced            */
    double   ms_plan, ms_score, ms_step;   /* device time per phase, summed (CUDA events)  */
    uint64_t state_transition_bytes;/* bytes written/read to change the learning state:
                                       direction draws, bank update, window opening        */
    uint64_t dense_ref_bytes;       /* 2*|theta| bytes per step of dense mutation, summed   */
    uint64_t dense_ref_bytes_targets;/* same, counting only the targeted matrices          */
    int32_t  bank_slots;            /* windows currently in the bank                        */
    int32_t  last_error_code;
    uint64_t kernel_launches;       /* CUDA kernels this handle launched                    */
    uint64_t gemm_launches;         /* GEMM launches timed (options.profile)                */
    double   gemm_ms;               /* their summed device time                              */
    double   gemm_flops;            /* their algorithmic FLOPs (base GEMM + live extension)  */
    uint64_t tc_gemm_launches;      /* of which on tensor cores                              */
    double   tc_gemm_ms;
    double   tc_gemm_flops;
    uint64_t cuda_core_gemm_launches;/* GEMMs that ran on CUDA cores (always counted): 0 for
                                       bf16 models unless options.impl asks for CUDA cores  */
    uint64_t graph_captures;        /* zo_step_graph: step graphs captured                  */
    uint64_t graph_replays;         /* zo_step_graph: step graph launches                   */
} zo_stats_t;

/* ---- lifecycle -------------------------------------------------------------------- */

/* Validate desc, borrow the weights, allocate the bank, activations and
 * scratch for the given maxima (all device memory the library uses is
 * allocated here), and repack the attention projections into one fused
 * [q|k|v] matrix (a copy; the caller's tensors stay untouched).
 * On any failure everything allocated so far is freed, *out stays NULL and
 * zo_last_error(NULL) says why; an allocation that fails gives ZO_ERR_OOM.
 * Failure injection for tests: with the environment variable
 * ZO_FAIL_ALLOC_AT=n set when zo_create is called, the handle's n-th device
 * allocation (counted from 1) fails as if the device were out of memory. */
int zo_create(const zo_model_desc* desc, const zo_weights* weights,
              const zo_options* options, zo_handle** out);
void zo_destroy(zo_handle* h);
const char* zo_last_error(const zo_handle* h);

/* ---- the probe step ---------------------------------------------------------------- */

/* ProbePlan for step `step` ("Inference-Native Zeroth-Order Optimization",
 * abstract): draws U_t for every target on the device and, when step is the
 * first of a window (step % nu == 0), V of the window and a new bank slot
 * with A = 0.  rank and *targets must equal the handle's options (they shape
 * the bank).  step must equal the handle's step counter (ZO_ERR_STATE
 * otherwise); planning the same step again replaces the plan.  The plan is
 * owned by the handle and valid until the next zo_step. */
int zo_probe_plan(zo_handle* h, uint64_t step, int32_t rank, float eps,
                  const zo_targets* targets, zo_plan** out);

/* Score n_prompts prompts under theta + eps z and theta - eps z ("Why ZO
 * Fine-Tuning Is Really Scoring": the pair of forward objective
 * evaluations).  Each prompt becomes a + row and a - row of one packed
 * variable-length batch (all + rows, then all - rows; no padding).
 *   packed_tokens  dev  int32 [sum(seq_lens)]   prompts back to back; ids
 *                  outside [0, vocab) are checked on the device and never used
 *                  as an index: the row's objective becomes NaN and zo_step
 *                  returns ZO_ERR_ARG with the bank unchanged
 *   seq_lens       host int32 [n_prompts]
 *   target_lens    host int32 [n_prompts]       1 <= t < seq_len
 *   target_ids     dev  int32 [sum(target_lens)] or NULL; when given it must
 *                  equal each prompt's last target_lens tokens (checked on the
 *                  device; a mismatch surfaces as ZO_ERR_ARG from zo_step)
 *   L_plus, L_minus dev float [n_prompts]       per-prompt objectives
 *   tok_logprob    dev float [2*sum(target_lens)] or NULL: + spans, then - spans */
int zo_score(zo_plan* plan, const int32_t* packed_tokens, int32_t n_prompts,
             const int32_t* seq_lens, const int32_t* target_lens, const int32_t* target_ids,
             float* L_plus, float* L_minus, float* tok_logprob);

/* Generation queries ("Inference-Native Zeroth-Order Optimization", abstract:
 * the same ProbePlan covers autoregressive generation as well as token
 * scoring).  Each prompt becomes a + row and a - row (all +, then all -, as in
 * zo_score); each row decodes n_new tokens greedily under its own candidate
 * state theta +- eps z: the prompt runs once as a packed prefill whose keys and
 * values are kept in a per-layer cache, then one decode step per further token
 * appends to it.  Greedy = the largest logit, ties to the lowest token id.  The
 * row's objective is the mean of -log p(token | prefix) over its generated
 * tokens; L+/L- go to L_plus/L_minus as in zo_score, and zo_step then applies
 * the update.
 *   packed_tokens dev int32 [sum(seq_lens)], seq_lens host int32 [n_prompts], each >= 2
 *     and seq_len + n_new <= max_pos
 *   gen_tokens  dev int32 [2 n_prompts x n_new] or NULL: row r's tokens at r * n_new
 *   gen_logprob dev float [2 n_prompts x n_new] or NULL: their log-probabilities
 *   L_plus, L_minus dev float [n_prompts] or NULL
 * ZO_ERR_UNSUPPORTED when options.max_new is 0; ZO_ERR_ARG when n_new is outside
 * 1..max_new or the batch exceeds max_tokens (prompt tokens of both candidates),
 * max_rows (2 n_prompts) or max_scored (2 n_prompts). */
int zo_generate(zo_plan* plan, const int32_t* packed_tokens, int32_t n_prompts,
                const int32_t* seq_lens, int32_t n_new, int32_t* gen_tokens,
                float* gen_logprob, float* L_plus, float* L_minus);

/* zo_score with n_fg unperturbed foreground rows appended to the same
 * physical batch (co-batching: "Inference-Native Zeroth-Order Optimization",
 * abstract, foreground inference and probes in the same physical batches).
 * Foreground rows score the current state theta_t = base + bank; their
 * per-token log-probs (dev float [sum(fg_target_lens)]) are bit-identical to
 * zo_score_foreground on the same rows. */
int zo_score_cobatch(zo_plan* plan, const int32_t* packed_tokens, int32_t n_prompts,
                     const int32_t* seq_lens, const int32_t* target_lens,
                     const int32_t* target_ids, float* L_plus, float* L_minus,
                     float* tok_logprob, const int32_t* fg_tokens, int32_t n_fg,
                     const int32_t* fg_seq_lens, const int32_t* fg_target_lens,
                     float* fg_tok_logprob);

/* Foreground rows alone under theta_t (the "scored alone" counterpart).  It
 * may run between a plan's scoring and its zo_step: the plan's objectives,
 * and so the step's c, are left as they were. */
int zo_score_foreground(zo_handle* h, const int32_t* fg_tokens, int32_t n_fg,
                        const int32_t* fg_seq_lens, const int32_t* fg_target_lens,
                        float* fg_tok_logprob);

/* c = mean_i (L+_i - L-_i) / (2 eps), no 1/r, reduced on the device in a
 * fixed order in fp64; then A_k <- A_k - lr * c * U_t for every target in one
 * launch, and the step counter advances.  If c is not finite the update is
 * refused on the device and the bank is unchanged; with c_out != NULL the
 * call synchronises, writes c (host double) and returns ZO_ERR_NONFINITE
 * (and the step counter does not advance). */
int zo_step(zo_handle* h, float lr, double* c_out);

/* One whole probe step -- zo_probe_plan at the handle's step counter, zo_score
 * of n_prompts prompts (no target_ids check, no per-token output) and
 * zo_step(lr, NULL) -- as a single CUDA graph launch on the handle's stream:
 * the step's ~10 kernels per layer leave the host as one launch ("Zeroth-Order
 * Fine-Tuning Was an Inference Workload All Along", section "Why ZO
 * Fine-Tuning Is Really Scoring": the step is the pair of forward evaluations
 * plus an update that is cheap, so nothing else should cost time).
 *   packed_tokens  dev  int32 [sum(seq_lens)]; seq_lens, target_lens host int32
 *   [n_prompts]; L_plus, L_minus dev float [n_prompts] or NULL.
 * The graph is captured on first use and again whenever the batch layout
 * (n_prompts, seq_lens, target_lens), eps, lr, the token or output pointers,
 * or the bank's slot count changes; otherwise it is replayed, reading the
 * current contents of packed_tokens.  A step that opens a lazy window does the
 * window's host-side set-up eagerly first.  The direction draws and results
 * are bit-identical to the eager calls.  Never synchronises: a non-finite c
 * refuses the update on the device (bank unchanged) and the step counter
 * advances, as zo_step with c_out == NULL.  ZO_ERR_STATE if a plan from
 * zo_probe_plan is still open. */
int zo_step_graph(zo_handle* h, const int32_t* packed_tokens, int32_t n_prompts,
                  const int32_t* seq_lens, const int32_t* target_lens, float eps, float lr,
                  float* L_plus, float* L_minus);

/* Data-parallel split of zo_step: write {sum_i (L+_i - L-_i), n_prompts}
 * (dev double[2]) for this replica's prompts; after the caller has summed
 * them over replicas (one all-reduce), apply c = s[0] / s[1] / (2 eps). */
int zo_objective_sums(zo_handle* h, double* dev_sums);
int zo_step_from_sums(zo_handle* h, float lr, const double* dev_sums, double* c_out);

/* ---- state, statistics and test hooks ------------------------------------------------ */
int zo_stats(zo_handle* h, zo_stats_t* out);

/* Serialise (run seed, step, nu, rank, targets, bank slots A_k) into buf
 * (host).  With buf == NULL only *n is set.  V factors are re-drawn from the
 * counter stream on load, so a resumed run reproduces the trajectory bit for
 * bit.  Layout (little endian): an 88-byte header
 *   uint64 magic 0x5A4F42414E4B3031, version 1, run_seed, step, start_window;
 *   int32 nu, rank, n_slots, scale_mode; uint32 matrix_mask, 0;
 *   uint64 layer_mask_lo, layer_mask_hi, payload_floats
 * then, for each layer, for each fused group in the order [q|k|v], o,
 * FFN-in (OPT up; Qwen3 gate, up), FFN-out (down), for each slot j, for each
 * targeted matrix of the group in id order: A_j^T as fp32 [r x d_in].
 * zo_load_state accepts any buffer in this layout written under the same
 * options (seed, nu, rank, targets), e.g. a bank trained elsewhere. */
int zo_save_state(zo_handle* h, void* buf, size_t* n);
int zo_load_state(zo_handle* h, const void* buf, size_t n);

/* Copy the current plan's U_t [d_in x r] and the window's V [d_out x r]
 * (row-major, host float) of one target; either pointer may be NULL. */
int zo_read_factors(zo_plan* plan, int32_t layer, int32_t matrix, float* U_host,
                    float* V_host);
/* Copy bank slot `slot`'s A [d_in x r] (host float) of one target. */
int zo_read_bank(zo_handle* h, int32_t layer, int32_t matrix, int32_t slot, float* A_host);

/* Fill a device tensor with the counter stream's initial weights:
 * fp32(z * std) (+ mean when mean != 0), z the N(0,1) stream keyed by
 * (weight_seed, layer, tensor); dtype ZO_DTYPE_BF16 rounds to nearest even.
 * Queued on stream (cudaStream_t, may be NULL). */
int zo_init_tensor(void* dev, uint64_t n, uint64_t weight_seed, uint32_t layer,
                   uint32_t tensor, float std, float mean, int32_t dtype, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* ZO_H */
