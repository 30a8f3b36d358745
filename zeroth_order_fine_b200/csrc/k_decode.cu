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

#include <algorithm>

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

// One CTA per (row, kv head): the n_rep query heads that share the kv head.  The 4 warps
// take rounds of 4 consecutive keys in turn; a warp's 32 lanes split the head dimension
// (hd / 32 consecutive elements each), so a key's k and v rows are read as one coalesced warp
// access.  Per warp an online softmax (fp32) over its keys, then the four warps' partial
// results are merged.
constexpr int DEC_WARPS = 4, DEC_MAX_REP = 8, DEC_MAX_DPL = 8;      // hd <= 256

// DPL consecutive elements at off (a multiple of DPL): 8/16-byte loads when DPL % 4 == 0
template <int DPL>
__device__ __forceinline__ void load_dims(const void* base, size_t off, int dtype, float* v) {
    if (dtype == E_F32) {
        const float* p = static_cast<const float*>(base) + off;
        if (DPL % 4 == 0) {
#pragma unroll
            for (int i = 0; i < DPL; i += 4) {
                const float4 t = *reinterpret_cast<const float4*>(p + i);
                v[i] = t.x; v[i + 1] = t.y; v[i + 2] = t.z; v[i + 3] = t.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < DPL; ++i) v[i] = p[i];
        }
    } else {
        const __nv_bfloat16* p = static_cast<const __nv_bfloat16*>(base) + off;
        if (DPL % 4 == 0) {
#pragma unroll
            for (int i = 0; i < DPL; i += 4) {
                const uint2 t = *reinterpret_cast<const uint2*>(p + i);
                const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&t.x));
                const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&t.y));
                v[i] = a.x; v[i + 1] = a.y; v[i + 2] = b.x; v[i + 3] = b.y;
            }
        } else {
#pragma unroll
            for (int i = 0; i < DPL; ++i) v[i] = __bfloat162float(p[i]);
        }
    }
}

// blockIdx.z takes keys [z * kps, (z + 1) * kps) of the row.  With part == nullptr (one
// split) the CTA writes the output; else it writes its (max, sum, unnormalised output) per
// query head to part, and decode_merge_kernel combines the splits in order.
template <int DPL>
__global__ void __launch_bounds__(DEC_WARPS * 32) decode_attention_kernel(
    const void* __restrict__ qkv, int ld_qkv, const void* __restrict__ cache, int kv2,
    const int* __restrict__ cu, const int* __restrict__ lens, int g, int G, int H, int Hkv,
    float scale, void* __restrict__ out, int ld_out, int dtype, int kps, float* __restrict__ part) {
    constexpr int HD = DPL * 32;
    __shared__ float sm_m[DEC_WARPS][DEC_MAX_REP], sm_l[DEC_WARPS][DEC_MAX_REP];
    __shared__ float sm_o[DEC_WARPS][DEC_MAX_REP][HD];
    const int r = blockIdx.x, kvh = blockIdx.y;
    const int n_rep = H / Hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t base = (size_t)cu[r] + (size_t)r * G;
    const int n = lens[r] + g + 1;
    const int kbeg = blockIdx.z * kps, kend = min(n, kbeg + kps);
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
    for (int j = kbeg + warp; j < kend; j += DEC_WARPS) {
        const size_t kr = (base + j) * kv2 + (size_t)kvh * HD + d0;
        float k[DPL], v[DPL];
        load_dims<DPL>(cache, kr, dtype, k);
        load_dims<DPL>(cache, kr + kv_dim, dtype, v);
#pragma unroll
        for (int hh = 0; hh < DEC_MAX_REP; ++hh) {
            if (hh >= n_rep) break;
            float s_ = 0.f;
#pragma unroll
            for (int i = 0; i < DPL; ++i) s_ = fmaf(q[hh][i], k[i], s_);
            s_ = warp_sum(s_) * scale;
            const float m_new = fmaxf(m[hh], s_);
            const float alpha = m[hh] > -FLT_MAX ? expf(m[hh] - m_new) : 0.f;
            const float p = expf(s_ - m_new);
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
    const int S = gridDim.z;
    float* pr = part ? part + ((size_t)(r * Hkv + kvh) * S + blockIdx.z) * n_rep * (HD + 2) : nullptr;
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
        if (pr) {
            pr[hh * (HD + 2) + dd] = acc;
            if (dd == 0) {
                pr[hh * (HD + 2) + HD] = mm;
                pr[hh * (HD + 2) + HD + 1] = ll;
            }
        } else {
            st_elem(out, (size_t)r * ld_out + (size_t)(kvh * n_rep + hh) * HD + dd, dtype,
                    ll > 0.f ? acc / ll : 0.f);
        }
    }
}

// Combine the key splits of one (row, kv head) in split order.
template <int HD>
__global__ void decode_merge_kernel(const float* __restrict__ part, int S, int n_rep, int Hkv,
                                    void* __restrict__ out, int ld_out, int dtype) {
    const int r = blockIdx.x, kvh = blockIdx.y;
    const float* pr = part + (size_t)(r * Hkv + kvh) * S * n_rep * (HD + 2);
    for (int idx = threadIdx.x; idx < n_rep * HD; idx += blockDim.x) {
        const int hh = idx / HD, dd = idx % HD;
        float mm = -FLT_MAX;
        for (int z = 0; z < S; ++z) mm = fmaxf(mm, pr[((size_t)z * n_rep + hh) * (HD + 2) + HD]);
        float ll = 0.f, acc = 0.f;
        for (int z = 0; z < S; ++z) {
            const float* e = pr + ((size_t)z * n_rep + hh) * (HD + 2);
            const float f = e[HD] > -FLT_MAX ? expf(e[HD] - mm) : 0.f;
            ll += e[HD + 1] * f;
            acc += e[dd] * f;
        }
        st_elem(out, (size_t)r * ld_out + (size_t)(kvh * n_rep + hh) * HD + dd, dtype,
                ll > 0.f ? acc / ll : 0.f);
    }
}

// One CTA per (32 rows, 8 factor columns): K is walked in chunks of 128 staged in shared
// memory (fp32), each of the 256 threads owning one (row, column) dot product, so every
// factor row is read once per 32 rows and every x row once per 8 columns.
constexpr int SR_ROWS = 32, SR_COLS = 8, SR_KC = 128;

__device__ __forceinline__ void bf16x8(const uint4& u, float* f) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 t = __bfloat1622float2(h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

// With part != nullptr, blockIdx.z takes K range [z * kspan, (z + 1) * kspan) and writes its
// raw partial to part[z][m][j]; shrink_rows_sum then adds the parts in z order.
__global__ void __launch_bounds__(SR_ROWS * SR_COLS) shrink_rows_kernel(
    const void* __restrict__ x, int x_type, const void* __restrict__ FT, int ft_type, int M, int N,
    int K, void* __restrict__ C, int ldc, int c_type, const int* __restrict__ row_sign, float eps,
    int scale_cols, const float* __restrict__ a_scale, float* __restrict__ part, int kspan) {
    __shared__ float xs[SR_ROWS][SR_KC + 1];
    __shared__ float fs[SR_COLS][SR_KC + 1];
    const int tid = threadIdx.x;
    const int ml = tid / SR_COLS, jl = tid % SR_COLS;
    const int m0 = blockIdx.y * SR_ROWS, j0 = blockIdx.x * SR_COLS;
    float acc = 0.f;
    const bool vec = x_type == E_BF16 && ft_type == E_BF16 && (K & 7) == 0;
    const int kbeg = part ? blockIdx.z * kspan : 0;
    const int kend = part ? min(K, kbeg + kspan) : K;
    for (int k0 = kbeg; k0 < kend; k0 += SR_KC) {
        const int kc = min(SR_KC, kend - k0);
        if (vec && kc == SR_KC) {
            // 16-byte loads, all issued before any is used
            constexpr int XV = SR_ROWS * SR_KC / 8 / (SR_ROWS * SR_COLS);   // 2 per thread
            uint4 xv[XV], fv;
#pragma unroll
            for (int it = 0; it < XV; ++it) {
                const int i = tid + it * SR_ROWS * SR_COLS, r = i / (SR_KC / 8), k8 = i % (SR_KC / 8);
                xv[it] = m0 + r < M ? __ldg(reinterpret_cast<const uint4*>(
                                          static_cast<const __nv_bfloat16*>(x) + (size_t)(m0 + r) * K + k0) + k8)
                                    : make_uint4(0, 0, 0, 0);
            }
            const bool has_f = tid < SR_COLS * SR_KC / 8;
            const int fr = tid / (SR_KC / 8), fk8 = tid % (SR_KC / 8);
            fv = has_f && j0 + fr < N ? __ldg(reinterpret_cast<const uint4*>(
                                            static_cast<const __nv_bfloat16*>(FT) + (size_t)(j0 + fr) * K + k0) + fk8)
                                      : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int it = 0; it < XV; ++it) {
                const int i = tid + it * SR_ROWS * SR_COLS, r = i / (SR_KC / 8), k8 = i % (SR_KC / 8);
                float f[8];
                bf16x8(xv[it], f);
#pragma unroll
                for (int e = 0; e < 8; ++e) xs[r][k8 * 8 + e] = f[e];
            }
            if (has_f) {
                float f[8];
                bf16x8(fv, f);
#pragma unroll
                for (int e = 0; e < 8; ++e) fs[fr][fk8 * 8 + e] = f[e];
            }
        } else {
#pragma unroll 4
            for (int i = tid; i < SR_ROWS * SR_KC; i += SR_ROWS * SR_COLS) {
                const int r = i / SR_KC, k = i % SR_KC;
                xs[r][k] = (m0 + r < M && k < kc) ? ld_elem(x, (size_t)(m0 + r) * K + k0 + k, x_type) : 0.f;
            }
#pragma unroll 4
            for (int i = tid; i < SR_COLS * SR_KC; i += SR_ROWS * SR_COLS) {
                const int r = i / SR_KC, k = i % SR_KC;
                fs[r][k] = (j0 + r < N && k < kc) ? ld_elem(FT, (size_t)(j0 + r) * K + k0 + k, ft_type) : 0.f;
            }
        }
        __syncthreads();
        float a0 = 0.f, a1 = 0.f;
#pragma unroll 16
        for (int k = 0; k < SR_KC; k += 2) {
            a0 = fmaf(xs[ml][k], fs[jl][k], a0);
            a1 = fmaf(xs[ml][k + 1], fs[jl][k + 1], a1);
        }
        acc += a0 + a1;
        __syncthreads();
    }
    const int m = m0 + ml, j = j0 + jl;
    if (m < M && j < N) {
        if (part) {
            part[((size_t)blockIdx.z * M + m) * N + j] = acc;
            return;
        }
        float y = j < scale_cols ? acc * ((float)row_sign[m] * eps) : acc;
        if (a_scale) y = y / a_scale[m];
        st_elem(C, (size_t)m * ldc + j, c_type, y);
    }
}

__global__ void shrink_rows_sum_kernel(const float* __restrict__ part, int ks, int M, int N,
                                       void* __restrict__ C, int ldc, int c_type,
                                       const int* __restrict__ row_sign, float eps, int scale_cols,
                                       const float* __restrict__ a_scale) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= M * N) return;
    const int m = i / N, j = i % N;
    float acc = 0.f;
    for (int z = 0; z < ks; ++z) acc += part[((size_t)z * M + m) * N + j];
    float y = j < scale_cols ? acc * ((float)row_sign[m] * eps) : acc;
    if (a_scale) y = y / a_scale[m];
    st_elem(C, (size_t)m * ldc + j, c_type, y);
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
                             int hd, float scale, void* out, int ld_out, int dtype, int max_n,
                             float* ws, size_t ws_floats, cudaStream_t st) {
    if (H / Hkv > DEC_MAX_REP || hd % 32 || hd / 32 > DEC_MAX_DPL) return false;
    if (R == 0) return true;
    const int n_rep = H / Hkv;
    // with fewer than ~4 (row, kv head) CTAs per SM, split the keys into chunks of 64 so
    // enough warps stay in flight; the splits' partial softmaxes are combined in order by the
    // merge kernel
    constexpr int KPS = 64;
    int S = (long long)R * Hkv >= 4 * 148 ? 1 : (max_n + KPS - 1) / KPS;
    if (S < 1) S = 1;
    if ((size_t)R * Hkv * S * n_rep * (hd + 2) > ws_floats) S = 1;
    const int kps = S == 1 ? max_n : KPS;
    float* part = S > 1 ? ws : nullptr;
    dim3 grid(R, Hkv, S);
#define ZO_DEC(DPL)                                                                              \
    decode_attention_kernel<DPL><<<grid, DEC_WARPS * 32, 0, st>>>(qkv, ld_qkv, cache, kv2, cu,    \
                                                                 lens, g, G, H, Hkv, scale, out, \
                                                                 ld_out, dtype, kps, part)
    switch (hd / 32) {
        case 1: ZO_DEC(1); break;
        case 2: ZO_DEC(2); break;
        case 4: ZO_DEC(4); break;
        case 8: ZO_DEC(8); break;
        default: return false;
    }
#undef ZO_DEC
    if (S > 1) {
        dim3 mg(R, Hkv);
        switch (hd) {
            case 32: decode_merge_kernel<32><<<mg, 128, 0, st>>>(part, S, n_rep, Hkv, out, ld_out, dtype); break;
            case 64: decode_merge_kernel<64><<<mg, 128, 0, st>>>(part, S, n_rep, Hkv, out, ld_out, dtype); break;
            case 128: decode_merge_kernel<128><<<mg, 128, 0, st>>>(part, S, n_rep, Hkv, out, ld_out, dtype); break;
            default: decode_merge_kernel<256><<<mg, 128, 0, st>>>(part, S, n_rep, Hkv, out, ld_out, dtype); break;
        }
    }
    return true;
}

void launch_shrink_rows(const void* x, int x_type, const void* FT, int ft_type, int M, int N,
                        int K, void* C, int ldc, int c_type, const int* row_sign, float eps,
                        int scale_cols, const float* a_scale, float* ws, size_t ws_floats,
                        cudaStream_t st) {
    if (M == 0 || N == 0) return;
    dim3 grid(cdiv(N, SR_COLS), cdiv(M, SR_ROWS));
    // split K when the (rows, columns) tiles alone leave most SMs idle
    int ks = 1;
    const long long tiles = (long long)grid.x * grid.y;
    if (ws && tiles < 148) {
        ks = (int)std::min<long long>(16, (148 + tiles - 1) / tiles);
        ks = std::min(ks, std::max(1, K / (2 * SR_KC)));
        while (ks > 1 && (size_t)ks * M * N > ws_floats) --ks;
    }
    if (ks > 1) {
        const int kspan = ((K + ks - 1) / ks + SR_KC - 1) / SR_KC * SR_KC;
        grid.z = ks;
        shrink_rows_kernel<<<grid, SR_ROWS * SR_COLS, 0, st>>>(x, x_type, FT, ft_type, M, N, K, C,
                                                               ldc, c_type, row_sign, eps,
                                                               scale_cols, a_scale, ws, kspan);
        shrink_rows_sum_kernel<<<cdiv((long long)M * N, 256), 256, 0, st>>>(
            ws, ks, M, N, C, ldc, c_type, row_sign, eps, scale_cols, a_scale);
        return;
    }
    shrink_rows_kernel<<<grid, SR_ROWS * SR_COLS, 0, st>>>(x, x_type, FT, ft_type, M, N, K, C, ldc,
                                                           c_type, row_sign, eps, scale_cols,
                                                           a_scale, nullptr, 0);
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
