// Generation queries: the KV cache, the one-token decode attention and the greedy choice.
//
// "Inference-Native Zeroth-Order Optimization" (abstract) states that the same ProbePlan
// formulation covers autoregressive generation as well as token scoring.  A generation
// query here decodes G tokens greedily per candidate row with a KV cache: the prompt runs
// once as a packed prefill whose k|v rows are kept per layer, then every new token is one
// row of a decode step that attends over its own row's cache.  Everything is memory-bound
// (a decode step reads every weight once for all rows and each row's cache once), so these
// kernels are plain 16-byte copies and CUDA-core reductions; the GEMMs stay on tcgen05.
#include <float.h>

#include "common.cuh"
#include "kernels.h"

namespace zo {

namespace {

// 16-byte copies when both rows allow it, else element by element
__device__ __forceinline__ void copy_row(const void* src, void* dst, int n_elem, int es) {
    const size_t bytes = (size_t)n_elem * es;
    if ((bytes & 15) == 0 && ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15) == 0) {
        const uint4* s = static_cast<const uint4*>(src);
        uint4* d = static_cast<uint4*>(dst);
        for (size_t i = threadIdx.x; i < bytes / 16; i += blockDim.x) d[i] = s[i];
    } else {
        const char* s = static_cast<const char*>(src);
        char* d = static_cast<char*>(dst);
        for (size_t i = threadIdx.x; i < bytes; i += blockDim.x) d[i] = s[i];
    }
}

__global__ void kv_scatter_kernel(const char* __restrict__ qkv, int ld_qkv, int q_dim, int kv2,
                                  const int* __restrict__ tok_row, int G, char* __restrict__ cache,
                                  int es) {
    const int t = blockIdx.x;
    const size_t crow = (size_t)t + (size_t)tok_row[t] * G;
    copy_row(qkv + ((size_t)t * ld_qkv + q_dim) * es, cache + crow * kv2 * es, kv2, es);
}

__global__ void decode_prep_kernel(const int* __restrict__ gen_tok, int G, int g,
                                   const int* __restrict__ lens, int R, int B, int* tok_id,
                                   int* tok_pos, int* tok_sign, int* tok_row) {
    const int r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= R) return;
    tok_id[r] = gen_tok[(size_t)r * G + g];
    tok_pos[r] = lens[r] + g;
    tok_sign[r] = r < B ? 1 : (r < 2 * B ? -1 : 0);
    tok_row[r] = r;
}

__global__ void kv_append_kernel(const char* __restrict__ qkv, int ld_qkv, int q_dim, int kv2,
                                 const int* __restrict__ cu, const int* __restrict__ lens, int g,
                                 int G, char* __restrict__ cache, int es) {
    const int r = blockIdx.x;
    const size_t crow = (size_t)cu[r] + (size_t)r * G + lens[r] + g;
    copy_row(qkv + ((size_t)r * ld_qkv + q_dim) * es, cache + crow * kv2 * es, kv2, es);
}

// One CTA per (row, kv head): the n_rep query heads that share the kv head, keys streamed in
// chunks of 128 (one key per thread for the scores, one dimension per thread for P V), with
// an online softmax across chunks in fp32.
constexpr int DEC_THREADS = 128, DEC_CHUNK = 128, DEC_MAX_REP = 8, DEC_MAX_HD = 256;

__global__ void __launch_bounds__(DEC_THREADS) decode_attention_kernel(
    const void* __restrict__ qkv, int ld_qkv, const void* __restrict__ cache, int kv2,
    const int* __restrict__ cu, const int* __restrict__ lens, int g, int G, int H, int Hkv, int hd,
    float scale, void* __restrict__ out, int ld_out, int dtype) {
    __shared__ float qs[DEC_MAX_REP][DEC_MAX_HD];
    __shared__ float ps[DEC_MAX_REP][DEC_CHUNK];
    __shared__ float red[32];
    __shared__ float m_sh[DEC_MAX_REP], l_sh[DEC_MAX_REP], a_sh[DEC_MAX_REP];
    const int r = blockIdx.x, kvh = blockIdx.y;
    const int n_rep = H / Hkv;
    const int tid = threadIdx.x;
    const size_t base = (size_t)cu[r] + (size_t)r * G;
    const int n = lens[r] + g + 1;
    const int kv_dim = kv2 / 2;
    for (int i = tid; i < n_rep * hd; i += DEC_THREADS) {
        const int hh = i / hd, dd = i % hd;
        qs[hh][dd] = ld_elem(qkv, (size_t)r * ld_qkv + (size_t)(kvh * n_rep + hh) * hd + dd, dtype);
    }
    if (tid < n_rep) {
        m_sh[tid] = -FLT_MAX;
        l_sh[tid] = 0.f;
    }
    float acc[DEC_MAX_REP][2];
#pragma unroll
    for (int hh = 0; hh < DEC_MAX_REP; ++hh) acc[hh][0] = acc[hh][1] = 0.f;
    __syncthreads();
    for (int c0 = 0; c0 < n; c0 += DEC_CHUNK) {
        const int j = c0 + tid;
        // scores of this thread's key for every query head of the group
        float sc[DEC_MAX_REP];
#pragma unroll
        for (int hh = 0; hh < DEC_MAX_REP; ++hh) sc[hh] = -FLT_MAX;
        if (j < n) {
            const size_t kb = (base + j) * kv2 + (size_t)kvh * hd;
            for (int hh = 0; hh < n_rep; ++hh) sc[hh] = 0.f;
            for (int dd = 0; dd < hd; ++dd) {
                const float kv = ld_elem(cache, kb + dd, dtype);
#pragma unroll
                for (int hh = 0; hh < DEC_MAX_REP; ++hh)
                    if (hh < n_rep) sc[hh] = fmaf(qs[hh][dd], kv, sc[hh]);
            }
#pragma unroll
            for (int hh = 0; hh < DEC_MAX_REP; ++hh)
                if (hh < n_rep) sc[hh] *= scale;
        }
        for (int hh = 0; hh < n_rep; ++hh) {
            const float cmax = block_max(sc[hh], red);
            const float m_old = m_sh[hh];
            const float m_new = fmaxf(m_old, cmax);
            const float p = j < n ? expf(sc[hh] - m_new) : 0.f;
            ps[hh][tid] = p;
            const float csum = block_sum(p, red);
            if (tid == 0) {
                const float alpha = m_old > -FLT_MAX ? expf(m_old - m_new) : 0.f;
                a_sh[hh] = alpha;
                l_sh[hh] = l_sh[hh] * alpha + csum;
                m_sh[hh] = m_new;
            }
        }
        __syncthreads();
        const int nk = min(DEC_CHUNK, n - c0);
        for (int dd0 = 0; dd0 < 2; ++dd0) {
            const int dd = tid + dd0 * DEC_THREADS;
            if (dd >= hd) continue;
            float part[DEC_MAX_REP];
#pragma unroll
            for (int hh = 0; hh < DEC_MAX_REP; ++hh) part[hh] = 0.f;
            for (int jj = 0; jj < nk; ++jj) {
                const float v = ld_elem(cache, (base + c0 + jj) * kv2 + kv_dim + (size_t)kvh * hd + dd,
                                        dtype);
#pragma unroll
                for (int hh = 0; hh < DEC_MAX_REP; ++hh)
                    if (hh < n_rep) part[hh] = fmaf(ps[hh][jj], v, part[hh]);
            }
#pragma unroll
            for (int hh = 0; hh < DEC_MAX_REP; ++hh)
                if (hh < n_rep) acc[hh][dd0] = acc[hh][dd0] * a_sh[hh] + part[hh];
        }
        __syncthreads();                       // ps and a_sh are rewritten by the next chunk
    }
    for (int dd0 = 0; dd0 < 2; ++dd0) {
        const int dd = tid + dd0 * DEC_THREADS;
        if (dd >= hd) continue;
        for (int hh = 0; hh < n_rep; ++hh) {
            const float inv = l_sh[hh] > 0.f ? 1.f / l_sh[hh] : 0.f;
            st_elem(out, (size_t)r * ld_out + (size_t)(kvh * n_rep + hh) * hd + dd, dtype,
                    acc[hh][dd0] * inv);
        }
    }
}

__global__ void last_tokens_kernel(const int* __restrict__ cu, int R, int* out, int* lens) {
    const int r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= R) return;
    out[r] = cu[r + 1] - 1;
    lens[r] = cu[r + 1] - cu[r];
}

__global__ void gen_objective_kernel(const float* __restrict__ logprob, int R, int B, int G,
                                     double* __restrict__ L_row, float* L_plus, float* L_minus) {
    const int r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= R) return;
    double s = 0.0;
    for (int i = 0; i < G; ++i) s += (double)logprob[(size_t)r * G + i];
    const double L = -s / (double)G;
    L_row[r] = L;
    if (r < B && L_plus) L_plus[r] = (float)L;
    else if (r >= B && r < 2 * B && L_minus) L_minus[r - B] = (float)L;
}

}  // namespace

void launch_kv_scatter(const void* qkv, int ld_qkv, int q_dim, int kv2, const int* tok_row,
                       int T, int G, void* cache, int dtype, cudaStream_t st) {
    if (T == 0) return;
    kv_scatter_kernel<<<T, 128, 0, st>>>(static_cast<const char*>(qkv), ld_qkv, q_dim, kv2,
                                         tok_row, G, static_cast<char*>(cache),
                                         dtype == E_F32 ? 4 : 2);
}

void launch_decode_prep(const int* gen_tok, int G, int g, const int* lens, int R, int B,
                        int* tok_id, int* tok_pos, int* tok_sign, int* tok_row, cudaStream_t st) {
    if (R == 0) return;
    decode_prep_kernel<<<cdiv(R, 128), 128, 0, st>>>(gen_tok, G, g, lens, R, B, tok_id, tok_pos,
                                                     tok_sign, tok_row);
}

void launch_kv_append(const void* qkv, int ld_qkv, int q_dim, int kv2, const int* cu,
                      const int* lens, int R, int g, int G, void* cache, int dtype,
                      cudaStream_t st) {
    if (R == 0) return;
    kv_append_kernel<<<R, 128, 0, st>>>(static_cast<const char*>(qkv), ld_qkv, q_dim, kv2, cu,
                                        lens, g, G, static_cast<char*>(cache),
                                        dtype == E_F32 ? 4 : 2);
}

void launch_decode_attention(const void* qkv, int ld_qkv, const void* cache, int kv2,
                             const int* cu, const int* lens, int R, int g, int G, int H, int Hkv,
                             int hd, float scale, void* out, int ld_out, int dtype,
                             cudaStream_t st) {
    if (R == 0 || H / Hkv > DEC_MAX_REP || hd > DEC_MAX_HD) return;
    dim3 grid(R, Hkv);
    decode_attention_kernel<<<grid, DEC_THREADS, 0, st>>>(qkv, ld_qkv, cache, kv2, cu, lens, g, G,
                                                          H, Hkv, hd, scale, out, ld_out, dtype);
}

void launch_last_tokens(const int* cu, int R, int* out, int* lens, cudaStream_t st) {
    if (R == 0) return;
    last_tokens_kernel<<<cdiv(R, 128), 128, 0, st>>>(cu, R, out, lens);
}

void launch_gen_objective(const float* logprob, int R, int B, int G, double* L_row,
                          float* L_plus, float* L_minus, cudaStream_t st) {
    if (R == 0) return;
    gen_objective_kernel<<<cdiv(R, 128), 128, 0, st>>>(logprob, R, B, G, L_row, L_plus, L_minus);
}

}  // namespace zo
