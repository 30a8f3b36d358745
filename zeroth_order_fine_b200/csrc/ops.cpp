// Kernel-level entry points (include/zo_ops.h): argument checks and launches.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <algorithm>
#include <string>
#include <vector>

#include "../../include/zo.h"
#include "../../include/zo_ops.h"
#include "kernels.h"

using namespace zo;

namespace {
thread_local std::string t_op_err;

// ZO_OK, or ZO_ERR_CUDA with the CUDA error (a failed launch, or an earlier asynchronous
// error the launch ran into) kept for zo_op_last_error
int op_status() {
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) return ZO_OK;
    t_op_err = std::string(cudaGetErrorName(e)) + ": " + cudaGetErrorString(e);
    return ZO_ERR_CUDA;
}
int op_fail(const char* what) {
    const cudaError_t e = cudaGetLastError();
    t_op_err = what;
    if (e != cudaSuccess) t_op_err += std::string(" (") + cudaGetErrorName(e) + ")";
    return ZO_ERR_CUDA;
}

bool use_tc(int32_t impl, int dtype) {
    if (impl == ZO_IMPL_CUDA_CORES) return false;
    return dtype == ZO_DTYPE_BF16;
}
}  // namespace

extern "C" {

int zo_op_quantize_rows_e4m3(const void* x, int32_t dtype, int32_t rows, int32_t cols,
                             uint8_t* q, float* scale, void* stream) {
    if (!x || !q || !scale || rows < 0 || cols <= 0) return ZO_ERR_ARG;
    if (dtype != ZO_DTYPE_FP32 && dtype != ZO_DTYPE_BF16) return ZO_ERR_ARG;
    launch_quant_rows_e4m3(x, dtype == ZO_DTYPE_BF16 ? E_BF16 : E_F32, rows, cols, (size_t)cols, q,
                           (size_t)cols, scale, static_cast<cudaStream_t>(stream));
    return op_status();
}

int zo_op_linear_fp8(const uint8_t* xq, const float* sx, const uint8_t* wq, const float* sw,
                     const float* bias, void* y, int32_t M, int32_t N, int32_t K, int32_t act,
                     void* stream) {
    if (!xq || !sx || !wq || !sw || !y || M < 0 || N <= 0 || K <= 0) return ZO_ERR_ARG;
    if (act != ZO_ACT_NONE && act != ZO_ACT_RELU) return ZO_ERR_ARG;
    GemmArgs g;
    memset(&g, 0, sizeof(g));
    g.A = xq; g.lda = K; g.a_type = E_FP8;
    g.B = wq; g.ldb = K; g.b_type = E_FP8;
    g.a_scale = sx; g.b_scale = sw;
    g.M = M; g.N = N; g.K = K;
    g.bias = bias;
    g.epi = act == ZO_ACT_RELU ? EPI_STORE_RELU : EPI_STORE;
    g.C = y; g.ldc = N; g.c_type = E_BF16;
    if (M == 0) return ZO_OK;
    if (!gemm_tc_supported(g)) return ZO_ERR_UNSUPPORTED;
    if (gemm_tc(g, static_cast<cudaStream_t>(stream))) return op_fail("tensor-core GEMM launch failed");
    return op_status();
}

int zo_op_linear(const void* x, const void* W, const float* bias, void* y, int32_t M, int32_t N,
                 int32_t K, int32_t dtype, int32_t act, int32_t accumulate, int32_t impl,
                 void* stream) {
    if (!x || !W || !y || M < 0 || N <= 0 || K <= 0) return ZO_ERR_ARG;
    if (dtype != ZO_DTYPE_FP32 && dtype != ZO_DTYPE_BF16) return ZO_ERR_ARG;
    if (act != ZO_ACT_NONE && act != ZO_ACT_RELU) return ZO_ERR_ARG;
    if (accumulate && act != ZO_ACT_NONE) return ZO_ERR_ARG;
    GemmArgs g;
    memset(&g, 0, sizeof(g));
    const int t = dtype == ZO_DTYPE_BF16 ? E_BF16 : E_F32;
    g.A = x; g.lda = K; g.a_type = t;
    g.B = W; g.ldb = K; g.b_type = t;
    g.M = M; g.N = N; g.K = K;
    g.bias = bias;
    g.epi = accumulate ? EPI_RESID : (act == ZO_ACT_RELU ? EPI_STORE_RELU : EPI_STORE);
    g.C = y; g.ldc = N; g.c_type = accumulate ? E_F32 : t;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (M == 0) return ZO_OK;
    if (use_tc(impl, dtype)) {
        if (gemm_tc_supported(g)) {
            if (gemm_tc(g, st)) return op_fail("tensor-core GEMM launch failed");
            return op_status();
        }
        if (impl == ZO_IMPL_TENSOR_CORES) return ZO_ERR_UNSUPPORTED;
    } else if (impl == ZO_IMPL_TENSOR_CORES) {
        return ZO_ERR_UNSUPPORTED;
    }
    gemm_simt(g, st);
    return op_status();
}

int zo_op_linear_decode(const void* x, const void* W, const float* bias, void* y, int32_t M,
                        int32_t N, int32_t K, int32_t act, int32_t accumulate, float* ws,
                        size_t ws_floats, void* stream) {
    if (M < 0 || N <= 0 || K <= 0) return ZO_ERR_ARG;
    if (act != ZO_ACT_NONE && act != ZO_ACT_RELU) return ZO_ERR_ARG;
    if (accumulate && act != ZO_ACT_NONE) return ZO_ERR_ARG;
    if (M == 0) return ZO_OK;
    if (!x || !W || !y || !ws || ws_floats < (size_t)M * N) return ZO_ERR_ARG;
    if (K % 8 || N % 4) return ZO_ERR_UNSUPPORTED;
    GemmArgs g;
    memset(&g, 0, sizeof(g));
    g.A = x; g.lda = K; g.a_type = E_BF16;
    g.B = W; g.ldb = K; g.b_type = E_BF16;
    g.M = M; g.N = N; g.K = K;
    g.bias = bias;
    g.epi = accumulate ? EPI_RESID : (act == ZO_ACT_RELU ? EPI_STORE_RELU : EPI_STORE);
    g.C = y; g.ldc = N; g.c_type = accumulate ? E_F32 : E_BF16;
    g.ws = ws; g.ws_floats = ws_floats;
    if (!gemm_tc_supported(g)) return ZO_ERR_UNSUPPORTED;
    if (gemm_tc(g, static_cast<cudaStream_t>(stream))) return op_fail("tensor-core GEMM launch failed");
    return op_status();
}

size_t zo_op_lm_head_workspace(int32_t n_rows, int32_t vocab, int32_t impl) {
    (void)impl;
    const size_t tiles = (size_t)gemm_lse_col_tiles(vocab);
    const size_t part = ((size_t)n_rows * tiles * 4 + 255) / 256 * 256;
    const size_t tg = ((size_t)n_rows * 4 + 255) / 256 * 256;
    return 2 * part + tg;
}

int zo_op_lm_head_logprob(const void* h, const void* E, const int32_t* targets, int32_t n_rows,
                          int32_t vocab, int32_t d, int32_t dtype, float* logprob,
                          void* workspace, size_t workspace_bytes, int32_t impl, void* stream) {
    if (!h || !E || !targets || !logprob || n_rows < 0 || vocab <= 0 || d <= 0) return ZO_ERR_ARG;
    if (dtype != ZO_DTYPE_FP32 && dtype != ZO_DTYPE_BF16) return ZO_ERR_ARG;
    if (n_rows == 0) return ZO_OK;
    const size_t need = zo_op_lm_head_workspace(n_rows, vocab, impl);
    if (!workspace || workspace_bytes < need) return ZO_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) % 256) return ZO_ERR_ARG;
    const int tiles = gemm_lse_col_tiles(vocab);   // the larger count: both paths fit
    const size_t part = ((size_t)n_rows * tiles * 4 + 255) / 256 * 256;
    char* ws = static_cast<char*>(workspace);
    float* pmax = reinterpret_cast<float*>(ws);
    float* psum = reinterpret_cast<float*>(ws + part);
    float* tgt = reinterpret_cast<float*>(ws + 2 * part);
    const int t = dtype == ZO_DTYPE_BF16 ? E_BF16 : E_F32;
    GemmArgs g;
    memset(&g, 0, sizeof(g));
    g.A = h; g.lda = d; g.a_type = t;
    g.B = E; g.ldb = d; g.b_type = t;
    g.M = n_rows; g.N = vocab; g.K = d;
    g.epi = EPI_LSE;
    g.targets = targets; g.part_max = pmax; g.part_sum = psum; g.tgt_logit = tgt;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool tc = use_tc(impl, dtype) && gemm_tc_supported(g);
    if (impl == ZO_IMPL_TENSOR_CORES && !tc) return ZO_ERR_UNSUPPORTED;
    g.n_col_tiles = tc ? gemm_tc_col_tiles(vocab) : tiles;
    if (tc) {
        if (gemm_tc(g, st)) return op_fail("tensor-core GEMM launch failed");
    } else {
        gemm_simt(g, st);
    }
    launch_lse_merge(pmax, psum, tgt, n_rows, g.n_col_tiles, logprob, st);
    return op_status();
}

int zo_op_attention(const void* qkv, void* out, const int32_t* seq_lens, int32_t n_rows,
                    int32_t n_heads, int32_t n_kv_heads, int32_t head_dim, int32_t dtype,
                    void* workspace, size_t workspace_bytes, int32_t impl, void* stream) {
    if (!qkv || !out || !seq_lens || n_rows < 0 || n_heads <= 0 || n_kv_heads <= 0) return ZO_ERR_ARG;
    if (n_heads % n_kv_heads) return ZO_ERR_ARG;
    if (head_dim != 32 && head_dim != 64 && head_dim != 128 && head_dim != 256)
        return ZO_ERR_UNSUPPORTED;
    if (dtype != ZO_DTYPE_FP32 && dtype != ZO_DTYPE_BF16) return ZO_ERR_ARG;
    if (n_rows == 0) return ZO_OK;
    if (n_rows >= 32768) return ZO_ERR_ARG;
    std::vector<int> meta(n_rows + 1);
    meta[0] = 0;
    const bool tc = use_tc(impl, dtype) && (head_dim == 64 || head_dim == 128);
    if (impl == ZO_IMPL_TENSOR_CORES && !tc) return ZO_ERR_UNSUPPORTED;
    const int qtile = tc ? 128 : 64;
    std::vector<int> tiles;
    for (int r = 0; r < n_rows; ++r) {
        if (seq_lens[r] < 1 || seq_lens[r] > 65535 * 64) return ZO_ERR_ARG;
        meta[r + 1] = meta[r] + seq_lens[r];
        for (int q = 0; q < (seq_lens[r] + qtile - 1) / qtile; ++q) tiles.push_back((r << 16) | q);
    }
    // attention CTAs are issued in item order: longest (most key chunks) first
    if (tc)
        std::stable_sort(tiles.begin(), tiles.end(),
                         [](int x, int y) { return (x & 0xFFFF) > (y & 0xFFFF); });
#ifdef ZO_DEBUG
    // test hook of the debug build: ZO_DEBUG_PLANT=attention_tile makes the last work tile
    // name a row past the batch; the kernels' bounds checks must report it and skip it
    if (const char* plant = std::getenv("ZO_DEBUG_PLANT"))
        if (!std::strcmp(plant, "attention_tile") && !tiles.empty())
            tiles.back() = (n_rows << 16) | (tiles.back() & 0xFFFF);
#endif
    const size_t need = (meta.size() + tiles.size()) * 4;
    if (!workspace || workspace_bytes < need) return ZO_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int* w = static_cast<int*>(workspace);
    meta.insert(meta.end(), tiles.begin(), tiles.end());
    if (cudaMemcpyAsync(w, meta.data(), meta.size() * 4, cudaMemcpyHostToDevice, st) != cudaSuccess)
        return op_fail("copy of the row metadata failed");
    // the host vector must outlive the copy
    if (cudaStreamSynchronize(st) != cudaSuccess) return op_fail("stream synchronisation failed");
    AttnArgs a;
    memset(&a, 0, sizeof(a));
    a.qkv = qkv; a.ld_qkv = (n_heads + 2 * n_kv_heads) * head_dim;
    a.out = out; a.ld_out = n_heads * head_dim;
    a.dtype = dtype == ZO_DTYPE_BF16 ? E_BF16 : E_F32;
    a.cu_seqlens = w;
    a.tiles = w + n_rows + 1;
    a.n_tiles = (int)tiles.size();
    a.H = n_heads; a.Hkv = n_kv_heads; a.hd = head_dim;
    a.scale = (float)(1.0 / std::sqrt((double)head_dim));
    a.n_tokens = meta[n_rows];
    a.n_rows = n_rows;
    if (tc && attention_tc_supported(a)) {
        if (!launch_attention_tc(a, st)) return op_fail("tensor-core attention setup failed");
    } else if (impl == ZO_IMPL_TENSOR_CORES) {
        return ZO_ERR_UNSUPPORTED;
    } else {
        launch_attention(a, st);
    }
    return op_status();
}

int zo_op_linear_ext(const void* x, const void* W, const float* bias, const void* x2,
                     const void* W2, int32_t K2, void* y, int32_t ldy, int32_t M, int32_t N,
                     int32_t K, int32_t epi, const zo_qk_norm_rope_args* qk, void* stream) {
    if (!x || !W || !y || M < 0 || N <= 0 || K <= 0 || K2 < 0 || ldy <= 0) return ZO_ERR_ARG;
    if (K2 > 0 && (!x2 || !W2)) return ZO_ERR_ARG;
    GemmArgs g;
    memset(&g, 0, sizeof(g));
    switch (epi) {
        case ZO_EPI_STORE: g.epi = EPI_STORE; g.c_type = E_BF16; break;
        case ZO_EPI_RELU: g.epi = EPI_STORE_RELU; g.c_type = E_BF16; break;
        case ZO_EPI_RESID: g.epi = EPI_RESID; g.c_type = E_F32; break;
        case ZO_EPI_SWIGLU:
            if (N % 256) return ZO_ERR_UNSUPPORTED;
            g.epi = EPI_SWIGLU; g.c_type = E_BF16;
            if (ldy < N / 2) return ZO_ERR_ARG;
            break;
        case ZO_EPI_QK_NORM_ROPE:
            if (!qk || !qk->tok_pos || !qk->q_norm || !qk->k_norm || !qk->rope_cos ||
                !qk->rope_sin || qk->n_q_heads <= 0 || qk->n_kv_heads <= 0)
                return ZO_ERR_ARG;
            if (bias) return ZO_ERR_UNSUPPORTED;
            g.epi = EPI_QKNR; g.c_type = E_BF16;
            g.tok_pos = qk->tok_pos; g.qn = qk->q_norm; g.kn = qk->k_norm;
            g.rope_cos = qk->rope_cos; g.rope_sin = qk->rope_sin; g.norm_eps = qk->eps;
            g.n_q_heads = qk->n_q_heads; g.n_qk_heads = qk->n_q_heads + qk->n_kv_heads;
            if ((int64_t)(g.n_qk_heads + qk->n_kv_heads) * 128 != N) return ZO_ERR_ARG;
            break;
        default: return ZO_ERR_ARG;
    }
    if (epi != ZO_EPI_SWIGLU && ldy < N) return ZO_ERR_ARG;
    g.A = x; g.lda = K; g.a_type = E_BF16;
    g.B = W; g.ldb = K; g.b_type = E_BF16;
    if (K2 > 0) {
        g.A2 = x2; g.lda2 = K2; g.a2_type = E_BF16;
        g.B2 = W2; g.ldb2 = K2; g.b2_type = E_BF16;
        g.K2 = K2;
    }
    g.M = M; g.N = N; g.K = K;
    g.bias = bias;
    g.C = y; g.ldc = ldy;
    if (M == 0) return ZO_OK;
    if (!gemm_tc_supported(g)) return ZO_ERR_UNSUPPORTED;
    if (gemm_tc(g, static_cast<cudaStream_t>(stream))) return op_fail("tensor-core GEMM launch failed");
    return op_status();
}

int zo_op_rope_table(float* cos_t, float* sin_t, int32_t max_pos, int32_t head_dim, double theta,
                     void* stream) {
    if (!cos_t || !sin_t || max_pos <= 0 || head_dim <= 0 || head_dim % 2 || !(theta > 0.0))
        return ZO_ERR_ARG;
    launch_rope_table(cos_t, sin_t, max_pos, head_dim, theta, static_cast<cudaStream_t>(stream));
    return op_status();
}

int64_t zo_op_set_wait_limit(int64_t cycles) {
    return (int64_t)gemm_tc_set_wait_cycles((long long)cycles);
}

/* Error word of the tensor-core kernels (bit 0: a bounded wait expired);
 * synchronises the device and clears the word. */
int zo_op_error_word(void) {
    if (cudaDeviceSynchronize() != cudaSuccess) return -1;
    const int v = gemm_tc_error_word();
    const int w = attention_tc_error_word();
    if (v < 0 || w < 0) return -1;
    return v | w;
}

int zo_debug_build(void) {
#ifdef ZO_DEBUG
    return 1;
#else
    return 0;
#endif
}

uint32_t zo_debug_word(int32_t clear) {
    return debug_word_attention_tc(clear != 0) | debug_word_attention(clear != 0) |
           debug_word_decode(clear != 0) | debug_word_reduce(clear != 0) |
           debug_word_gemm(clear != 0);
}

const char* zo_op_last_error(void) { return t_op_err.c_str(); }

}  // extern "C"
