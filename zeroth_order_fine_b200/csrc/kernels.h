// Internal launch interface between the engine (engine.cpp) and the kernels.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace zo {

enum ElemType : int { E_F32 = 0, E_BF16 = 1, E_FP8 = 2 };   // E_FP8: E4M3 bytes

// ---- generator -------------------------------------------------------------------------
struct GenJob {
    float* dst;                 // fp32 factor, or null
    void* dst_bf;               // optional bf16 mirror written at the same positions
    int layer, matrix, which;   // which: 0 = U, 1 = V
    int dim, r;                 // factor is [dim x r]
    int transposed, ld;         // transposed: write element (i, c) at dst[c*ld + i]
};

struct WindowJob {
    const float* V;             // [d_out x r] row-major
    void* EB;                   // extension operand [N x ldb] (model dtype)
    float* A;                   // new slot's A_k^T rows, r*d_in floats to zero
    void* A_bf;                 // optional bf16 mirror of those rows
    int eb_type, ldb, row0, d_out, d_in, r, col_dir, col_slot;
    int interleave;             // 1: row i sits at (i / 128) * 256 + row0 + i % 128
    const float* row_div;       // optional: E_B row fr holds V / row_div[fr] (the fused
                                // matrix's FP8 weight scales), so one accumulator serves both
};

void launch_init_tensor(void* dst, uint64_t n, uint64_t key, float std_, float mean, int dtype,
                        cudaStream_t st);
// step_dev (may be null): read the step from device memory instead of `step`
void launch_gen_factors(const GenJob* d_jobs, int n_jobs, int max_pairs, uint64_t run_seed,
                        uint64_t step, const uint64_t* step_dev, uint64_t nu, float scale,
                        int apply_scale, cudaStream_t st);
void launch_set_step(uint64_t* step_dev, uint64_t v, cudaStream_t st);   // *step_dev = v
void launch_advance_step(uint64_t* step_dev, cudaStream_t st);           // *step_dev += 1
void launch_open_window(const WindowJob* d_jobs, int n_jobs, cudaStream_t st);

// ---- token metadata / embeddings / norms -----------------------------------------------
struct RowMeta {          // device arrays built from the host plan of one score call
    const int* cu_seqlens;    // [R+1] physical token offsets
    const int* row_src;       // [R] offset of the row's tokens in its source array
    const int* row_is_fg;     // [R]
    const int* row_sign;      // [R] +1 / -1 / 0
    const int* score_off;     // [R+1] offsets of each row's scored span
};

// Token ids outside [0, vocab) become -1 (a NaN embedding row; an out-of-range target gets
// a NaN logit) and set bit 1 of err_word; target_ids that differ set bit 0.
void launch_build_tokens(RowMeta m, int R, const int* probe_src, const int* fg_src, int vocab,
                         int* tok_id, int* tok_pos, int* tok_sign, int* tok_row, int* sc_tok,
                         int* sc_tgt, float* tgt_logit, const int* tgt_check_probe,
                         const int* tgt_check_fg, const int* tgt_check_off, int* err_word,
                         cudaStream_t st);
void launch_embed(const int* tok_id, const int* tok_pos, const void* tok_embed,
                  const void* pos_embed, int dtype, float* resid, int T, int d, cudaStream_t st);
// kind 0: LayerNorm(w, b), 1: RMSNorm(w).  rows: optional gather list (else 0..T-1).
// E4M3 per-row quantisation: scale[r] = amax / 448, q = E4M3(x * (448 / amax)), RN, saturated;
// an all-zero row has scale 1.  x is fp32 or bf16 [rows x ldx], q [rows x ldq] bytes.
void launch_quant_rows_e4m3(const void* x, int x_type, int rows, int cols, size_t ldx,
                            uint8_t* q, size_t ldq, float* scale, cudaStream_t st);
// q8/s8 (optional, vectorised path only): also the E4M3 quantisation of the bf16 output rows;
// pdl: the vectorised form is launched as a programmatic dependent of the kernel before it
void launch_norm(const float* x, const int* rows, int T, int d, int kind, const float* w,
                 const float* b, float eps, void* out, int out_type, cudaStream_t st,
                 uint8_t* q8 = nullptr, float* s8 = nullptr, bool pdl = false);
bool norm_fp8_supported(int d);
void launch_swiglu(const void* gu, int T, int f, void* out, int dtype, cudaStream_t st);
void launch_rope_table(float* cos_t, float* sin_t, int max_pos, int hd, double theta,
                       cudaStream_t st);
// Qwen3: per-head RMSNorm of q and k, then rotary positions, in place in the q|k|v rows
void launch_qk_norm_rope(void* qkv, int ld, int dtype, const int* tok_pos, int T, int H, int Hkv,
                         int hd, const float* qn, const float* kn, float eps, const float* cos_t,
                         const float* sin_t, cudaStream_t st);

// ---- GEMM ----------------------------------------------------------------------------
enum Epi : int {
    EPI_STORE = 0,       // C = acc + bias (out_type)
    EPI_STORE_RELU = 1,  // C = relu(acc + bias)
    EPI_RESID = 2,       // C(fp32) += acc + bias
    EPI_SHRINK = 3,      // C = acc * (col < scale_cols ? sign[row] * eps : 1)
    EPI_LSE = 4,         // per (row, 64-col tile): max, sum exp(x - max); target logit
    EPI_SWIGLU = 5,      // fused [gate|up] rows interleaved in 128-row blocks:
                         // C[m, f] = silu(gate_f) * up_f, f = n_blk * 128 + j (tensor cores)
    EPI_QKNR = 6         // Qwen3 q|k|v (bf16, head_dim 128, SM-pair tensor-core kernel only):
                         // the q and k heads (head < n_qk_heads) get per-head RMSNorm and
                         // rotary positions from the tables; v heads are stored as they are
};

// The norm that follows a residual GEMM (decode steps): fused into its split-K reduction.
struct NormNext {
    const float* w; const float* b;         // norm weight, bias (LayerNorm) or NULL
    int kind; float eps;                    // 0 LayerNorm, 1 RMSNorm
    void* out; int out_type;                // normalised rows [M x N]
    uint8_t* q8; float* s8;                 // optional E4M3 rows and scales of the output
};

// Decode steps: the q|k|v split reduction also writes each row's k|v columns into the key/value
// cache (row r's new token at cache row cu[r] + r * G + lens[r] + g, kv2 elements wide).
struct KvAppend {
    void* cache; size_t cache_rows;
    const int* cu; const int* lens; int g, G;
    int q_dim, kv2;
};

struct GemmArgs {
    const void* A; int lda; int a_type;     // [M x K], K contiguous
    const void* B; int ldb; int b_type;     // [N x K], K contiguous
    const void* A2; int lda2;               // optional extension [M x K2] (type a2_type)
    const void* B2; int ldb2;               // [N x K2] (type b2_type)
    int a2_type, b2_type, K2;
    int M, N, K;
    const float* bias;
    int epi;
    void* C; int ldc; int c_type;
    // EPI_SHRINK
    const int* row_sign; float eps; int scale_cols;
    // EPI_LSE (part_arg optional: per (row, column tile) the lowest column of the tile max)
    const int* targets; float* part_max; float* part_sum; float* tgt_logit; int n_col_tiles;
    int* part_arg;
    // E_FP8 operands: dequantisation scales per row of A [M] and of B [N]; the epilogue
    // multiplies the accumulator by a_scale[m] * b_scale[n] (the extension operands must
    // be pre-divided accordingly).  EPI_SHRINK with a_scale divides its output rows by it.
    const float* a_scale; const float* b_scale;
    // EPI_QKNR: token positions [M], norm weights [128] of q and k, rotary tables
    // [max_pos x 64]; heads below n_q_heads use qn, the next ones up to n_qk_heads kn
    const int* tok_pos; const float* qn; const float* kn;
    const float* rope_cos; const float* rope_sin; float norm_eps;
    int n_q_heads, n_qk_heads;
    // optional fp32 workspace (ws_floats floats) for decode steps: the bf16 store / ReLU /
    // residual / SwiGLU / q-k-norm GEMMs split K, over single SMs with the operands swapped
    // (M <= 128 token rows as the narrow N side) or over the SM pairs (larger M), and a
    // reduction sums the slices in order and applies the epilogue.  Callers give at least
    // M x N floats (one slice); more room allows more splits.
    float* ws; size_t ws_floats;
    // EPI_RESID with a split reduction: the reduction may also apply norm_next to each updated
    // row of C (the fp32 residual); it then sets *norm_done = 1 (else the caller runs the norm)
    const NormNext* norm_next; int* norm_done;
    // EPI_STORE / EPI_QKNR with a split reduction: the reduction may also append the k|v
    // columns to the cache (sets *kv_done = 1; else the caller copies them)
    const KvAppend* kv_append; int* kv_done;
};
// Split-K residual reduction with the next norm fused (see NormNext); false when the shape or
// alignment is outside the vectorised form (nothing launched).
bool launch_splitk_resid_norm(const float* ws, int ks, int M, int N, const float* bias, float* C,
                              int ldc, const NormNext& nn, cudaStream_t st, bool pdl);

void gemm_simt(const GemmArgs& g, cudaStream_t st);
// tcgen05 / TMEM / TMA path; returns false when the shape is outside its limits.
bool gemm_tc_supported(const GemmArgs& g);
int gemm_tc(const GemmArgs& g, cudaStream_t st);   // 0 ok, else 1
int gemm_lse_col_tiles(int N);                      // LSE column tiles, CUDA-core path (the most)
int gemm_tc_col_tiles(int N);                       // LSE column tiles, tensor-core path
int gemm_tc_error_word();                           // bit 0: a bounded wait expired
// Bound of every mbarrier wait in the tensor-core GEMM kernels launched from now on, in
// clock64 cycles (<= 0: the default, about 2 s); returns the previous bound.
long long gemm_tc_set_wait_cycles(long long cycles);

// ---- attention -----------------------------------------------------------------------
struct AttnArgs {
    const void* qkv; int ld_qkv;    // [T x ld_qkv]: q at col 0, k at q_dim, v at q_dim+kv_dim
    void* out; int ld_out;          // [T x H*hd]
    int dtype;
    const int* cu_seqlens;          // [R+1]
    const int* tiles;               // [n_tiles] packed (row << 16 | q_tile)
    int n_tiles;
    int H, Hkv, hd;
    float scale;
    int n_tokens;                   // T: rows of qkv (the tensor-core kernel's TMA extent)
    int n_rows;                     // R: entries of cu_seqlens minus one (debug bounds checks)
};
// (Qwen3's q/k RMSNorm and rotary positions are applied to the q|k|v rows before
// attention by launch_qk_norm_rope; the attention kernels take q and k as they are.)
void launch_attention(const AttnArgs& a, cudaStream_t st);          // CUDA cores, 64-query tiles
bool attention_tc_supported(const AttnArgs& a);                     // bf16, head_dim 128
bool launch_attention_tc(const AttnArgs& a, cudaStream_t st);       // tensor cores, 128-query tiles;
                                                                    // false if the tensor map fails
int attention_tc_error_word();

// ---- objective, estimator, update ------------------------------------------------------
void launch_lse_merge(const float* part_max, const float* part_sum, const float* tgt_logit,
                      int S, int n_tiles, float* logprob, cudaStream_t st);
// Greedy choice per row from the LSE partials: token = the lowest column holding the
// largest logit, logprob = that logit - logsumexp; written at row * stride.
void launch_lse_argmax_merge(const float* part_max, const float* part_sum, const int* part_arg,
                             int S, int n_tiles, int* token, float* logprob, int stride,
                             cudaStream_t st);

// ---- generation queries (KV cache) --------------------------------------------------------
// Cache layout per layer: [rows of (k | v)], row r's tokens at cu[r] + r * G + p, where cu
// are the prompt offsets and G the new tokens per row; a cache row is 2 * kv_dim wide.
// Prefill: copy each token's k|v columns of the packed q|k|v rows into the cache.
// cache_rows: rows of one layer's cache (the debug build checks every row index against it).
void launch_kv_scatter(const void* qkv, int ld_qkv, int q_dim, int kv2, const int* tok_row,
                       int T, int G, void* cache, size_t cache_rows, int dtype, cudaStream_t st);
// Decode step g (g >= 0): row r's new token sits at prompt length + g.
void launch_decode_prep(const int* gen_tok, int G, int g, const int* lens, int R, int B,
                        int* tok_id, int* tok_pos, int* tok_sign, int* tok_row, cudaStream_t st);
void launch_kv_append(const void* qkv, int ld_qkv, int q_dim, int kv2, const int* cu,
                      const int* lens, int R, int g, int G, void* cache, size_t cache_rows,
                      int dtype, cudaStream_t st);
// One query per row (its q heads in qkv row r) against the row's n = lens[r] + g + 1 cached
// keys; softmax(q k^T * scale) v into out [R x H*hd].  CUDA cores (memory-bound).  false
// when H / Hkv > 8 or hd is not 32, 64, 128 or 256.
// max_n: the most keys any row has at this step; ws (ws_floats floats) holds the partials
// when the keys split over several CTAs.
bool launch_decode_attention(const void* qkv, int ld_qkv, const void* cache, int kv2,
                             const int* cu, const int* lens, int R, int g, int G, int H, int Hkv,
                             int hd, float scale, void* out, int ld_out, int dtype, int max_n,
                             float* ws, size_t ws_floats, cudaStream_t st);
// Bank shrink for a few rows (decode steps), on CUDA cores: C[m, j] = (x[m] . FT[j]) *
// (j < scale_cols ? row_sign[m] * eps : 1) / (a_scale ? a_scale[m] : 1); x [M x K] in
// x_type, FT [N x K] in ft_type, C [M x ldc] in c_type.
// ws (optional, ws_floats floats): lets K split over more CTAs, the parts summed in order.
// The ordered sum of ks fp32 slices part[z][M][N] with the bank-shrink epilogue (columns below
// scale_cols times row_sign[m] * eps, then / a_scale[m] when given), stored to C (c_type);
// pdl: launched as a programmatic dependent of the kernel that wrote part.
void launch_shrink_rows_sum(const float* part, int ks, int M, int N, void* C, int ldc, int c_type,
                            const int* row_sign, float eps, int scale_cols, const float* a_scale,
                            cudaStream_t st, bool pdl);
void launch_shrink_rows(const void* x, int x_type, const void* FT, int ft_type, int M, int N,
                        int K, void* C, int ldc, int c_type, const int* row_sign, float eps,
                        int scale_cols, const float* a_scale, float* ws, size_t ws_floats,
                        cudaStream_t st);
// Last prompt token of each row (the hidden state that predicts the first new token) and
// the rows' prompt lengths.
void launch_last_tokens(const int* cu, int R, int* out, int* lens, cudaStream_t st);
// Generation objective: L_row[r] = -mean_g logprob[r * G + g] (fp64, fixed order); L+/L-.
void launch_gen_objective(const float* logprob, int R, int B, int G, double* L_row,
                          float* L_plus, float* L_minus, cudaStream_t st);
// per row L = -mean(logprob over its span) (fp64); L+/L- copies for the probe rows.
// S: scored positions in logprob (the debug build checks each span against it).
void launch_row_objective(const float* logprob, const int* score_off, int R, int B, long long S,
                          double* L_row, float* L_plus, float* L_minus, cudaStream_t st);
// sums[0] = sum_i (L_row[i] - L_row[B+i]) in a fixed order, sums[1] = B.
void launch_objective_sums(const double* L_row, int B, double* sums, cudaStream_t st);
// c = sums[0] / sums[1] / (2 eps); flag = 1 if not finite (update refused).
void launch_estimate(const double* sums, float eps, double* c, int* flag, cudaStream_t st);

// Bank update of every target's current slot, A <- A - coef_t U_t with coef_t = (float)(lr c)
// (0 when flag is set: a refused update leaves A as it was).  U_t is regenerated from the
// counter stream (key (run_seed, t, layer, matrix, U)), never read.  A is [r x ld] fp32, the
// transposed rows of the [dim x r] factor (element (i, c) at A[c * ld + i]), with an optional
// bf16 mirror at the same positions.
//   replay_from < 0: read-modify-write of A.
//   replay_from >= 0: A is not read.  It is rebuilt from zero by the slot's coefficients
//     coef_s, s = replay_from .. t, kept in coef_hist[s - replay_from] (this step's written
//     there): the same fused multiply-adds in the same order as the read-modify-write steps
//     since the slot opened, so both give the same bits.
// step_dev (may be null): read t from device memory instead of `step`.
struct UpdateJob { float* A; void* A_bf; int layer, matrix, dim, r, ld; };
void launch_to_bf16(const float* src, void* dst, size_t n, cudaStream_t st);
void launch_bank_update(const UpdateJob* jobs, int n_jobs, int max_pairs, const double* c,
                        const int* flag, float lr, uint64_t run_seed, uint64_t step,
                        const uint64_t* step_dev, uint64_t nu, float scale, int apply_scale,
                        long long replay_from, float* coef_hist, cudaStream_t st);

// Debug build (ZO_DEBUG): the device bounds-check words of the translation units that check
// (bits ZO_DBG_*), read and optionally cleared; always 0 in the release build.
enum : unsigned {
    ZO_DBG_ATTN_TILE = 1u,      // an attention work item names a row or query tile that is not there
    ZO_DBG_KV_SLOT = 2u,        // a key/value cache row index past the cache
    ZO_DBG_SCORE_SPAN = 4u,     // a row's scored span outside the scored positions
};
unsigned debug_word_attention_tc(bool clear);
unsigned debug_word_attention(bool clear);
unsigned debug_word_decode(bool clear);
unsigned debug_word_reduce(bool clear);
unsigned debug_word_gemm(bool clear);

}  // namespace zo
