// Generation queries: the KV cache, the one-token decode attention and the greedy choice.
//
// "Inference-Native Zeroth-Order Optimization" (abstract) states that the same ProbePlan
// formulation covers autoregressive generation as well as token scoring.  A generation
// query here decodes G tokens greedily per candidate row with a KV cache: the prompt runs
// once as a packed prefill whose k|v rows are kept per layer, then every new token is one
// row of a decode step that attends over its own row's cache.  Everything is memory-bound
// (a decode step reads every weight once for all rows and each row's cache once), so these
// kernels are plain 16-byte copies and coalesced CUDA-core reductions; the GEMMs stay on
// tcgen05.
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

// One CTA per (row, kv head): the n_rep query heads that share the kv head.  Each warp takes
// every 4th key; its 32 lanes split the head dimension (hd / 32 consecutive elements each), so
// a key's k and v rows are read as one coalesced warp access.  Per warp an online softmax
// (fp32) over its keys, then the four warps' partial results are merged.
constexpr int DEC_WARPS = 4, DEC_MAX_REP = 8, DEC_MAX_DPL = 8;      // hd <= 256

template <int DPL>
__device__ __forceinline__ void load_dims(const void* base, size_t off, int dtype, float* v) {
    if (dtype == E_F32) {
        const float* p = static_cast<const float*>(base) + off;
#pragma unroll
        for (int i = 0; i < DPL; ++i) v[i] = p[i];
    } else {
        const __nv_bfloat16* p = static_cast<const __nv_bfloat16*>(base) + off;
#pragma unroll
        for (int i = 0; i < DPL; ++i) v[i] = __bfloat162float(p[i]);
    }
}

template <int DPL>
__global__ void __launch_bounds__(DEC_WARPS * 32) decode_attention_kernel(
    const void* __restrict__ qkv, int ld_qkv, const void* __restrict__ cache, int kv2,
    const int* __restrict__ cu, const int* __restrict__ lens, int g, int G, int H, int Hkv,
    float scale, void* __restrict__ out, int ld_out, int dtype) {
    constexpr int HD = DPL * 32;
    __shared__ float sm_m[DEC_WARPS][DEC_MAX_REP], sm_l[DEC_WARPS][DEC_MAX_REP];
    __shared__ float sm_o[DEC_WARPS][DEC_MAX_REP][HD];
    const int r = blockIdx.x, kvh = blockIdx.y;
    const int n_rep = H / Hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t base = (size_t)cu[r] + (size_t)r * G;
    const int n = lens[r] + g + 1;
    const int kv_dim = kv2 / 2;
    const int d0 = lane * DPL;
    float q[DEC_MAX_REP][DPL], o[DEC_MAX_REP][DPL], m[DEC_MAX_REP], l[DEC_MAX_REP];
#pragma unroll
    for (int hh = 0; hh < DEC_MAX_REP; ++hh) {
        m[hh] = -FLT_MAX;
        l[hh] = 0.f;
#pragma unroll
        for (int i = 0; i < DPL; ++i) o[hh][i] = q[hh][i] = 0.f;
        if (hh < n_rep)
            load_dims<DPL>(qkv, (size_t)r * ld_qkv + (size_t)(kvh * n_rep + hh) * HD + d0, dtype,
                           q[hh]);
    }
    for (int j = warp; j < n; j += DEC_WARPS) {
        const size_t kr = (base + j) * kv2 + (size_t)kvh * HD + d0;
        float k[DPL], v[DPL];
        load_dims<DPL>(cache, kr, dtype, k);
        load_dims<DPL>(cache, kr + kv_dim, dtype, v);
#pragma unroll
        for (int hh = 0; hh < DEC_MAX_REP; ++hh) {
            if (hh >= n_rep) break;
            float s = 0.f;
#pragma unroll
            for (int i = 0; i < DPL; ++i) s = fmaf(q[hh][i], k[i], s);
            s = warp_sum(s) * scale;
            const float m_new = fmaxf(m[hh], s);
            const float alpha = m[hh] > -FLT_MAX ? expf(m[hh] - m_new) : 0.f;
            const float p = expf(s - m_new);
            l[hh] = l[hh] * alpha + p;
#pragma unroll
            for (int i = 0; i < DPL; ++i) o[hh][i] = fmaf(p, v[i], o[hh][i] * alpha);
            m[hh] = m_new;
        }
    }
#pragma unroll
    for (int hh = 0; hh < DEC_MAX_REP; ++hh) {
        if (hh >= n_rep) break;
        if (lane == 0) {
            sm_m[warp][hh] = m[hh];
            sm_l[warp][hh] = l[hh];
        }
#pragma unroll
        for (int i = 0; i < DPL; ++i) sm_o[warp][hh][d0 + i] = o[hh][i];
    }
    __syncthreads();
    // merge the warps' partial softmaxes in a fixed order
    for (int idx = threadIdx.x; idx < n_rep * HD; idx += DEC_WARPS * 32) {
        const int hh = idx / HD, dd = idx % HD;
        float mm = -FLT_MAX;
        for (int w = 0; w < DEC_WARPS; ++w) mm = fmaxf(mm, sm_m[w][hh]);
        float ll = 0.f, acc = 0.f;
        for (int w = 0; w < DEC_WARPS; ++w) {
            const float f = sm_m[w][hh] > -FLT_MAX ? expf(sm_m[w][hh] - mm) : 0.f;
            ll += sm_l[w][hh] * f;
            acc += sm_o[w][hh][dd] * f;
        }
        st_elem(out, (size_t)r * ld_out + (size_t)(kvh * n_rep + hh) * HD + dd, dtype,
                ll > 0.f ? acc / ll : 0.f);
    }
}

// grid (ceil(N / 8), M): one row against 8 factor rows, K split over the block (512
// threads, four K steps in flight per thread)
__global__ void __launch_bounds__(512) shrink_rows_kernel(
    const void* __restrict__ x, int x_type, const void* __restrict__ FT, int ft_type, int N, int K,
    void* __restrict__ C, int ldc, int c_type, const int* __restrict__ row_sign, float eps,
    int scale_cols, const float* __restrict__ a_scale) {
    __shared__ float red[32];
    const int m = blockIdx.y, j0 = blockIdx.x * 8;
    float acc[8];
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) acc[jj] = 0.f;
#pragma unroll 4
    for (int k = threadIdx.x; k < K; k += blockDim.x) {
        const float xv = ld_elem(x, (size_t)m * K + k, x_type);
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
            if (j0 + jj < N) acc[jj] = fmaf(xv, ld_elem(FT, (size_t)(j0 + jj) * K + k, ft_type), acc[jj]);
    }
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
        const float v = block_sum(acc[jj], red);
        const int j = j0 + jj;
        if (threadIdx.x == 0 && j < N) {
            float y = j < scale_cols ? v * ((float)row_sign[m] * eps) : v;
            if (a_scale) y = y / a_scale[m];
            st_elem(C, (size_t)m * ldc + j, c_type, y);
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

bool launch_decode_attention(const void* qkv, int ld_qkv, const void* cache, int kv2,
                             const int* cu, const int* lens, int R, int g, int G, int H, int Hkv,
                             int hd, float scale, void* out, int ld_out, int dtype,
                             cudaStream_t st) {
    if (H / Hkv > DEC_MAX_REP || hd % 32 || hd / 32 > DEC_MAX_DPL) return false;
    if (R == 0) return true;
    dim3 grid(R, Hkv);
    switch (hd / 32) {
        case 1: decode_attention_kernel<1><<<grid, DEC_WARPS * 32, 0, st>>>(qkv, ld_qkv, cache, kv2, cu, lens, g, G, H, Hkv, scale, out, ld_out, dtype); break;
        case 2: decode_attention_kernel<2><<<grid, DEC_WARPS * 32, 0, st>>>(qkv, ld_qkv, cache, kv2, cu, lens, g, G, H, Hkv, scale, out, ld_out, dtype); break;
        case 4: decode_attention_kernel<4><<<grid, DEC_WARPS * 32, 0, st>>>(qkv, ld_qkv, cache, kv2, cu, lens, g, G, H, Hkv, scale, out, ld_out, dtype); break;
        case 8: decode_attention_kernel<8><<<grid, DEC_WARPS * 32, 0, st>>>(qkv, ld_qkv, cache, kv2, cu, lens, g, G, H, Hkv, scale, out, ld_out, dtype); break;
        default: return false;
    }
    return true;
}

void launch_shrink_rows(const void* x, int x_type, const void* FT, int ft_type, int M, int N,
                        int K, void* C, int ldc, int c_type, const int* row_sign, float eps,
                        int scale_cols, const float* a_scale, cudaStream_t st) {
    if (M == 0 || N == 0) return;
    dim3 grid(cdiv(N, 8), M);
    shrink_rows_kernel<<<grid, 512, 0, st>>>(x, x_type, FT, ft_type, N, K, C, ldc, c_type,
                                             row_sign, eps, scale_cols, a_scale);
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
