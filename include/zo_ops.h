/*
 * zo_ops.h -- kernel-level entry points of the B200 ZO library.
 *
 * The single operations the probe step is built from, exposed so that each
 * can be checked and timed on its own.  None of them allocates: every
 * buffer, including scratch ("workspace"), is the caller's device memory.
 * All are queued on `stream` (cudaStream_t, NULL = legacy default stream)
 * and return ZO_OK or a ZO_ERR_* code from zo.h.  After ZO_ERR_CUDA,
 * zo_op_last_error() names what failed and the CUDA error.
 */
#ifndef ZO_OPS_H
#define ZO_OPS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ZO_ACT_NONE = 0, ZO_ACT_RELU = 1 };
enum { ZO_IMPL_AUTO = 0, ZO_IMPL_CUDA_CORES = 1, ZO_IMPL_TENSOR_CORES = 2 };

/* E4M3 quantisation of the rows of x, the format zo_options.fp8 runs the
 * norm-fed base GEMMs in ("Inference-Native Zeroth-Order Optimization",
 * abstract: the queries inherit the runtime's quantisation):
 * scale[r] = amax_r / 448 and q[r, :] = E4M3(x[r, :] * (448 / amax_r)),
 * both quotients and the product rounded to nearest in fp32, the cast
 * round-to-nearest-even and saturated at +-448; an all-zero row has scale 1.
 *   x     dev [rows x cols] dtype (fp32 or bf16), row-major
 *   q     dev uint8 [rows x cols] E4M3 codes;  scale dev float [rows]
 * ZO_ERR_ARG on NULL pointers or negative sizes.  Asynchronous on stream. */
int zo_op_quantize_rows_e4m3(const void* x, int32_t dtype, int32_t rows, int32_t cols,
                             uint8_t* q, float* scale, void* stream);

/* The E4M3 base GEMM: y = act((q_x * s_x) (q_W * s_W)^T + b) on the SM-pair
 * tcgen05 kernel (kind::f8f6f4, fp32 accumulate, dequantised in the
 * epilogue), the form zo_options.fp8 uses for q|k|v and the FFN input.
 *   xq dev uint8 [M x K], sx dev float [M]; wq dev uint8 [N x K], sw dev float [N]
 *   bias dev float [N] or NULL;  y dev bf16 [M x N];  act ZO_ACT_*
 * Needs K % 16 == 0 and N > 128 (the SM-pair tile), else ZO_ERR_UNSUPPORTED. */
int zo_op_linear_fp8(const uint8_t* xq, const float* sx, const uint8_t* wq, const float* sw,
                     const float* bias, void* y, int32_t M, int32_t N, int32_t K, int32_t act,
                     void* stream);

/* One decoder linear layer, y = act(x W^T + b) (the frozen base weights W of
 * "Inference-Native Zeroth-Order Optimization", abstract; the GEMM is the
 * batched forward that dominates the step, "Zeroth-Order Fine-Tuning Was an
 * Inference Workload All Along", section "Why ZO Fine-Tuning Is Really
 * Scoring").
 *   x    dev [M x K] dtype, row-major          W  dev [N x K] dtype, row-major
 *   bias dev float [N] or NULL
 *   y    accumulate == 0: dev [M x N] dtype; accumulate == 1: dev float [M x N],
 *        y += x W^T + b (the residual-add form)
 *   impl ZO_IMPL_TENSOR_CORES needs dtype bf16 and K % 8 == 0 (else
 *        ZO_ERR_UNSUPPORTED); AUTO picks tensor cores whenever they apply. */
int zo_op_linear(const void* x, const void* W, const float* bias, void* y, int32_t M,
                 int32_t N, int32_t K, int32_t dtype, int32_t act, int32_t accumulate,
                 int32_t impl, void* stream);

/* The decode-step form of zo_op_linear (bf16 only): the few token rows of one
 * generation step ("Inference-Native Zeroth-Order Optimization", abstract:
 * ProbePlan queries may be autoregressive generation) against a whole weight
 * matrix, which makes the GEMM a stream of the weights.  With M <= 128 the
 * weights take the 128-row side of a single-SM tcgen05 GEMM and the tokens the
 * narrow N side (32, 64 or 128 columns); K is split over the SMs, each split
 * stores its fp32 slice in ws, and a reduction adds the slices in split order
 * and applies bias, ReLU or the residual add, so the result does not depend on
 * scheduling.  Larger M splits K on the SM-pair kernel instead.
 *   x, W, bias, y, M, N, K, act, accumulate: as zo_op_linear (dtype bf16)
 *   ws   dev float [ws_floats], caller-owned scratch; at least M x N floats
 *        (room for up to 16 slices lets more splits run)
 * M = 0 is a no-op.  ZO_ERR_ARG on NULL pointers, negative sizes or ws_floats < M x N;
 * ZO_ERR_UNSUPPORTED when K % 8 is not 0, or N % 8 (N % 4 with accumulate), or a
 * pointer is not 16-byte aligned.  Asynchronous on stream. */
int zo_op_linear_decode(const void* x, const void* W, const float* bias, void* y, int32_t M,
                        int32_t N, int32_t K, int32_t act, int32_t accumulate, float* ws,
                        size_t ws_floats, void* stream);

/* Epilogues of zo_op_linear_ext. */
enum { ZO_EPI_STORE = 0, ZO_EPI_RELU = 1, ZO_EPI_RESID = 2, ZO_EPI_SWIGLU = 5,
       ZO_EPI_QK_NORM_ROPE = 6 };

/* Qwen3's per-head q/k RMSNorm and rotary positions, applied by the q|k|v GEMM's
 * epilogue (ZO_EPI_QK_NORM_ROPE). */
typedef struct zo_qk_norm_rope_args {
    const int32_t* tok_pos;   /* dev int32 [M]: each row's position within its sequence      */
    const float* q_norm;      /* dev float [128]: RMSNorm scales of the query heads, 16-B aligned */
    const float* k_norm;      /* dev float [128]: the key heads'                              */
    const float* rope_cos;    /* dev float [max_pos x 64]: cos(pos * theta^(-2i/128)), i < 64  */
    const float* rope_sin;    /* dev float [max_pos x 64]: the matching sines                 */
    float eps;                /* RMSNorm epsilon                                               */
    int32_t n_q_heads;        /* query heads (columns [0, 128 n_q_heads) of y)                */
    int32_t n_kv_heads;       /* key heads follow, then as many value heads (passed through)  */
} zo_qk_norm_rope_args;

/* The perturbed linear layer as the probe step runs it, on the tensor cores (bf16 only):
 *   acc = x W^T + x2 W2^T + b
 * where x2 W2^T is the extension that carries the candidate perturbation and the banked
 * slots (x2 = the shrink output s eps (x U) | x A_j, W2 = the expand factors V | V_j), run
 * as extra K blocks of the same tcgen05 GEMM so that no dense W + eps U V^T is formed
 * ("Zeroth-Order Fine-Tuning Was an Inference Workload All Along", section "The System
 * Reorganization"; "Inference-Native Zeroth-Order Optimization", abstract: factorised side
 * states over frozen base weights).  Then the epilogue:
 *   ZO_EPI_STORE  y = bf16(acc)                 ZO_EPI_RELU  y = bf16(max(acc, 0))
 *   ZO_EPI_RESID  y (fp32) += acc               (the residual stream)
 *   ZO_EPI_SWIGLU the rows of W (and W2, bias) hold gate and up features interleaved in
 *                 blocks of 128: rows 256 b .. 256 b + 127 are gate features 128 b .., the
 *                 next 128 rows the up features of the same indices; y [M x N/2] bf16 =
 *                 silu(gate) * up.  N % 256 == 0.
 *   ZO_EPI_QK_NORM_ROPE  acc rounded to bf16; each 128-column query and key head then gets
 *                 RMSNorm over the head (scale q_norm / k_norm) and the rotate-half rotary
 *                 rotation of the pairs (i, i + 64) at tok_pos[m]; value heads are stored as
 *                 they are.  N == 128 (n_q_heads + 2 n_kv_heads); no bias.
 *   x  dev bf16 [M x K], W dev bf16 [N x K]; x2 dev bf16 [M x K2], W2 dev bf16 [N x K2] (or
 *   K2 = 0 and both NULL); bias dev float [N] or NULL; y dev, row stride ldy elements.
 * Rows never interact: the result of a row does not depend on M or on the other rows.
 * ZO_ERR_ARG on NULL pointers, negative sizes, ldy too small or an unknown epilogue;
 * ZO_ERR_UNSUPPORTED when K, K2 or ldy is not a multiple of 8 (ldy: 4 for ZO_EPI_RESID),
 * a pointer is not 16-byte aligned, or the epilogue needs N > 128 (SwiGLU, q/k norm) and
 * does not get it.
 * Asynchronous on stream. */
int zo_op_linear_ext(const void* x, const void* W, const float* bias, const void* x2,
                     const void* W2, int32_t K2, void* y, int32_t ldy, int32_t M, int32_t N,
                     int32_t K, int32_t epi, const zo_qk_norm_rope_args* qk, void* stream);

/* The rotary tables zo_create builds for Qwen3 models: cos_t[pos * hd/2 + i] =
 * cos(pos * theta^(-2 i / head_dim)) and sin_t likewise, evaluated in double and rounded
 * to float.  cos_t, sin_t dev float [max_pos x head_dim / 2].  Asynchronous on stream. */
int zo_op_rope_table(float* cos_t, float* sin_t, int32_t max_pos, int32_t head_dim,
                     double theta, void* stream);

/* Test hook for the failure path of the tensor-core GEMM kernels.  Every mbarrier wait in
 * them gives up after `cycles` SM clock cycles: the kernel then sets bit 0 of the error
 * word (zo_op_error_word), stops issuing work, waits (again with a bound) for the copies
 * and MMAs it has already issued, frees its tensor memory and returns; its output is
 * invalid.  The default bound, about 2 s, is far beyond any wait of a healthy launch; a
 * bound of a few hundred cycles makes an ordinary launch give up at its first wait for
 * data, without any barrier being broken.  cycles <= 0 restores the default.  Applies to
 * launches queued after the call, process-wide (not synchronised with other threads).
 * Returns the previous bound. */
int64_t zo_op_set_wait_limit(int64_t cycles);

/* Bytes of workspace zo_op_lm_head_logprob needs for n_rows rows and vocab. */
size_t zo_op_lm_head_workspace(int32_t n_rows, int32_t vocab, int32_t impl);

/* Token log-probabilities through the lm_head without writing vocab-sized
 * logits to memory (the objective is the log-probability of the label
 * tokens: "Zeroth-Order Fine-Tuning Was an Inference Workload All Along",
 * sections "Why ZO Fine-Tuning Is Really Scoring" and "The System
 * Reorganization"):  logprob[i] = (h_i E^T)[target_i] - logsumexp(h_i E^T).
 *   h        dev [n_rows x d] dtype (final-norm hidden states)
 *   E        dev [vocab x d] dtype
 *   targets  dev int32 [n_rows], each in [0, vocab)
 *   logprob  dev float [n_rows]
 *   workspace dev, >= zo_op_lm_head_workspace(n_rows, vocab, impl) bytes,
 *            256-byte aligned; contents are scratch. */
int zo_op_lm_head_logprob(const void* h, const void* E, const int32_t* targets, int32_t n_rows,
                          int32_t vocab, int32_t d, int32_t dtype, float* logprob,
                          void* workspace, size_t workspace_bytes, int32_t impl, void* stream);

/* Packed variable-length causal attention, no padding ("Inference-Native
 * Zeroth-Order Optimization", abstract: padding elimination and
 * variable-length packing).
 *   qkv      dev [T x (H + 2*Hkv)*hd] dtype: q | k | v per token
 *   out      dev [T x H*hd] dtype
 *   seq_lens host int32 [n_rows], rows back to back in qkv
 *   workspace dev >= 4*(n_rows + 1 + T/64 + n_rows + 1) bytes (row offsets and tiles)
 *   impl     ZO_IMPL_TENSOR_CORES needs bf16 and head_dim 64 or 128; AUTO picks them then.
 * The tensor-core form also needs qkv and out 16-byte aligned; when out is 32-byte
 * aligned its rows are written with 32-byte stores (same values either way).
 * The call copies the row offsets from the host and synchronises the stream. */
int zo_op_attention(const void* qkv, void* out, const int32_t* seq_lens, int32_t n_rows,
                    int32_t n_heads, int32_t n_kv_heads, int32_t head_dim, int32_t dtype,
                    void* workspace, size_t workspace_bytes, int32_t impl, void* stream);

/* zo_op_lm_head_logprob without a workspace argument: the same result (same
 * kernels, same order), with the scratch taken from a 4 MiB array that the
 * library keeps in device memory (one per GPU, resident until the process
 * exits; zo_op_lm_head_noalloc_capacity() gives its size in floats).  This
 * entry point is an addition of this library, not a step of the method, so
 * no page describes it.  It is for callers that may not allocate device
 * memory when they call -- e.g. a process whose device memory belongs to
 * another runtime's pool, or a loop that must not touch the allocator after
 * start-up -- and that have no spare buffer to pass as workspace.  It never
 * allocates or frees (no cudaMalloc, no library allocator).
 *   Limit: 2 * n_rows * tiles + n_rows <= capacity, with tiles = ceil(vocab/256)
 *   on tensor cores and ceil(vocab/64) on CUDA cores; larger requests return
 *   ZO_ERR_UNSUPPORTED (nothing is launched).
 *   The first call on a device looks up the array's device address (once per
 *   device, with that device current); make that first call before any stream
 *   capture begins.
 *   All calls share the array: calls whose kernels may overlap on a GPU (other
 *   streams, no ordering between them) race and give wrong results.  Rows
 *   whose target is outside [0, vocab) get NaN. */
size_t zo_op_lm_head_noalloc_capacity(void);
int zo_op_lm_head_logprob_noalloc(const void* h, const void* E, const int32_t* targets,
                                  int32_t n_rows, int32_t vocab, int32_t d, int32_t dtype,
                                  float* logprob, int32_t impl, void* stream);

/* Synchronise the device and return the tensor-core kernels' error word:
 * 0 when clean, bit 0 set when a bounded wait inside a kernel expired (the
 * kernel then stopped early and its output is invalid), -1 when the device
 * reported an error. */
int zo_op_error_word(void);

/* The debug build (libzo_b200_debug.so, compiled with ZO_DEBUG) checks, on the
 * device, the indices its kernels derive from the host-built row metadata:
 * the attention work tiles (row and query tile), the key/value cache rows
 * of generation, and each row's scored span.  A failed check sets a bit of
 * a device word (1: attention tile, 2: cache row, 4: scored span) and the
 * access is skipped (an empty attention item, no cache copy, a NaN
 * objective); nothing traps.  The release build compiles the checks away.
 * zo_debug_build() is 1 in the debug build, else 0.  zo_debug_word(clear)
 * returns the bits set since the last clear (always 0 in the release build)
 * and clears them when clear != 0.  Synchronous (reads device memory).
 * In the debug build only, ZO_DEBUG_PLANT=attention_tile in the environment
 * makes zo_op_attention point its last work tile at a row past the batch,
 * so that a test can see the check fire. */
int zo_debug_build(void);
uint32_t zo_debug_word(int32_t clear);

/* What the calling thread's last zo_op_* call that returned ZO_ERR_CUDA ran
 * into: the step that failed and the CUDA error's name and text ("" before
 * any failure).  The string is the library's, valid until that thread's next
 * failing call. */
const char* zo_op_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* ZO_OPS_H */
