// Token metadata, embeddings, LayerNorm / RMSNorm (optionally gathering the
// scored rows first) and the SwiGLU activation.  All HBM-bound, one CTA per
// token row, each row read once.
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace zo {

// One CTA per physical row: token ids / positions / signs of the packed batch
// and, per scored position, the index of the hidden state that predicts it
// (the position before the target token) and the target id.
__global__ void build_tokens_kernel(RowMeta m, const int* __restrict__ probe_src,
                                    const int* __restrict__ fg_src, int vocab, int* tok_id,
                                    int* tok_pos, int* tok_sign, int* tok_row, int* sc_tok,
                                    int* sc_tgt, float* tgt_logit, const int* tgt_check_probe,
                                    const int* tgt_check_fg, const int* tgt_check_off,
                                    int* err_word) {
    const int r = blockIdx.x;
    const int start = m.cu_seqlens[r];
    const int len = m.cu_seqlens[r + 1] - start;
    const int* src = (m.row_is_fg[r] ? fg_src : probe_src) + m.row_src[r];
    const int sign = m.row_sign[r];
    for (int p = threadIdx.x; p < len; p += blockDim.x) {
        const int t = start + p;
        int id = src[p];
        // an id outside the vocabulary is never used as an index: -1 makes the embedding
        // row NaN, and bit 1 of the error word reports it
        if ((unsigned)id >= (unsigned)vocab) {
            id = -1;
            atomicOr(err_word, 2);
        }
        tok_id[t] = id;
        tok_pos[t] = p;
        tok_sign[t] = sign;
        tok_row[t] = r;
    }
    const int s0 = m.score_off[r];
    const int tl = m.score_off[r + 1] - s0;
    const int* chk = m.row_is_fg[r] ? tgt_check_fg : tgt_check_probe;
    for (int j = threadIdx.x; j < tl; j += blockDim.x) {
        const int tgt = src[len - tl + j];
        sc_tok[s0 + j] = start + len - tl + j - 1;
        // the lm_head epilogue writes the logit of an in-range target only; an out-of-range
        // one keeps this NaN, so its log-prob is NaN
        sc_tgt[s0 + j] = tgt;
        if ((unsigned)tgt >= (unsigned)vocab) tgt_logit[s0 + j] = __int_as_float(0x7fc00000);
        if (chk != nullptr && tgt_check_off[r] >= 0 && chk[tgt_check_off[r] + j] != tgt)
            atomicOr(err_word, 1);
    }
}

void launch_build_tokens(RowMeta m, int R, const int* probe_src, const int* fg_src, int vocab,
                         int* tok_id, int* tok_pos, int* tok_sign, int* tok_row, int* sc_tok,
                         int* sc_tgt, float* tgt_logit, const int* tgt_check_probe,
                         const int* tgt_check_fg, const int* tgt_check_off, int* err_word,
                         cudaStream_t st) {
    if (R == 0) return;
    build_tokens_kernel<<<R, 128, 0, st>>>(m, probe_src, fg_src, vocab, tok_id, tok_pos, tok_sign,
                                           tok_row, sc_tok, sc_tgt, tgt_logit, tgt_check_probe,
                                           tgt_check_fg, tgt_check_off, err_word);
}

// resid[t] = tok_embed[id] (+ pos_embed[pos]) in fp32; NaN for a rejected id (-1).
__global__ void embed_kernel(const int* __restrict__ tok_id, const int* __restrict__ tok_pos,
                             const void* __restrict__ tok_embed,
                             const void* __restrict__ pos_embed, int dtype,
                             float* __restrict__ resid, int d) {
    const int t = blockIdx.x;
    float* out = resid + (size_t)t * d;
    if (tok_id[t] < 0) {                         // rejected id: the row is NaN throughout
        for (int i = threadIdx.x; i < d; i += blockDim.x) out[i] = __int_as_float(0x7fc00000);
        return;
    }
    const size_t te = (size_t)tok_id[t] * d;
    const size_t pe = (size_t)tok_pos[t] * d;
    for (int i = threadIdx.x; i < d; i += blockDim.x) {
        float v = ld_elem(tok_embed, te + i, dtype);
        if (pos_embed) v += ld_elem(pos_embed, pe + i, dtype);
        out[i] = v;
    }
}

void launch_embed(const int* tok_id, const int* tok_pos, const void* tok_embed,
                  const void* pos_embed, int dtype, float* resid, int T, int d, cudaStream_t st) {
    if (T == 0) return;
    embed_kernel<<<T, 256, 0, st>>>(tok_id, tok_pos, tok_embed, pos_embed, dtype, resid, d);
}

// LayerNorm: (x - mean) / sqrt(var + eps) * w + b; RMSNorm: x / sqrt(mean(x^2) + eps) * w.
// Statistics in fp32 with a two-pass variance over the staged row.
__global__ void __launch_bounds__(256) norm_kernel(const float* __restrict__ x,
                                                   const int* __restrict__ rows, int d, int kind,
                                                   const float* __restrict__ w,
                                                   const float* __restrict__ b, float eps,
                                                   void* __restrict__ out, int out_type) {
    extern __shared__ float srow[];
    __shared__ float red[32];
    const int t = blockIdx.x;
    const int src = rows ? rows[t] : t;
    const float* xr = x + (size_t)src * d;
    float s = 0.f;
    for (int i = threadIdx.x; i < d; i += blockDim.x) {
        const float v = xr[i];
        srow[i] = v;
        s += (kind == 0) ? v : v * v;
    }
    s = block_sum(s, red);
    float mean = 0.f, rstd;
    if (kind == 0) {
        mean = s / (float)d;
        float q = 0.f;
        for (int i = threadIdx.x; i < d; i += blockDim.x) {
            const float c = srow[i] - mean;
            q += c * c;
        }
        q = block_sum(q, red);
        rstd = 1.0f / sqrtf(q / (float)d + eps);
    } else {
        rstd = 1.0f / sqrtf(s / (float)d + eps);
    }
    const size_t o = (size_t)t * d;
    for (int i = threadIdx.x; i < d; i += blockDim.x) {
        float y = (srow[i] - mean) * rstd * w[i];
        if (kind == 0) y += b[i];
        st_elem(out, o + i, out_type, y);
    }
}

// Vectorised form for d % 4 == 0, d <= 1024 * VPT: the row stays in registers
// (VPT float4 per thread), 16-byte loads, 8-byte bf16 stores.
// With q8: the bf16 output row is also quantised to E4M3 with one scale per row
// (amax / 448), from the bf16-rounded values, for the FP8 base GEMMs.
// Normalise one row held by the CTA's 256 threads as float4s (v[i] = elements 4j..4j+3, j =
// threadIdx.x + 256 i; s = their per-thread partial sum, or sum of squares for RMSNorm) and
// write output row t: LayerNorm (x - mean) / sqrt(var + eps) * w + b (kind 0) or RMSNorm
// x / sqrt(mean(x^2) + eps) * w (kind 1), statistics in fp32 with a two-pass variance, then
// (q8) the E4M3 codes and scale of the bf16-rounded row.  Shared by the norm kernel and the
// residual reduction that fuses the next norm, so both give the same bits.
template <int VPT>
__device__ __forceinline__ void norm_row_finish(float4 (&v)[VPT], float s, int t, int d, int kind,
                                                const float* __restrict__ w,
                                                const float* __restrict__ b, float eps,
                                                void* __restrict__ out, int out_type,
                                                uint8_t* __restrict__ q8, float* __restrict__ s8,
                                                float* red) {
    const int n4 = d >> 2;
    s = block_sum(s, red);
    float mean = 0.f, rstd;
    if (kind == 0) {
        mean = s / (float)d;
        float q = 0.f;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int j = threadIdx.x + i * 256;
            if (j < n4) {
                const float a = v[i].x - mean, bb = v[i].y - mean, c = v[i].z - mean,
                            e = v[i].w - mean;
                q += (a * a + bb * bb) + (c * c + e * e);
            }
        }
        q = block_sum(q, red);
        rstd = 1.0f / sqrtf(q / (float)d + eps);
    } else {
        rstd = 1.0f / sqrtf(s / (float)d + eps);
    }
    const float4* w4 = reinterpret_cast<const float4*>(w);
    const float4* b4 = reinterpret_cast<const float4*>(b);
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int j = threadIdx.x + i * 256;
        if (j >= n4) continue;
        const float4 ww = w4[j];
        float4 y;
        y.x = (v[i].x - mean) * rstd * ww.x;
        y.y = (v[i].y - mean) * rstd * ww.y;
        y.z = (v[i].z - mean) * rstd * ww.z;
        y.w = (v[i].w - mean) * rstd * ww.w;
        if (kind == 0) {
            const float4 bb = b4[j];
            y.x += bb.x; y.y += bb.y; y.z += bb.z; y.w += bb.w;
        }
        if (out_type == E_F32) {
            reinterpret_cast<float4*>(out)[(size_t)t * n4 + j] = y;
        } else {
            uint2 pk;
            __nv_bfloat162 h0 = __floats2bfloat162_rn(y.x, y.y), h1 = __floats2bfloat162_rn(y.z, y.w);
            pk.x = *reinterpret_cast<uint32_t*>(&h0);
            pk.y = *reinterpret_cast<uint32_t*>(&h1);
            reinterpret_cast<uint2*>(out)[(size_t)t * n4 + j] = pk;
            v[i] = make_float4(__low2float(h0), __high2float(h0), __low2float(h1), __high2float(h1));
        }
    }
    if (q8 == nullptr) return;
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int j = threadIdx.x + i * 256;
        if (j < n4)
            amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)),
                                     fmaxf(fabsf(v[i].z), fabsf(v[i].w))));
    }
    amax = block_max(amax, red);
    const float inv = amax > 0.f ? 448.0f / amax : 1.0f;
    if (threadIdx.x == 0) s8[t] = amax > 0.f ? amax / 448.0f : 1.0f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int j = threadIdx.x + i * 256;
        if (j >= n4) continue;
        const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(v[i].x * inv, v[i].y * inv),
                                                     __NV_SATFINITE, __NV_E4M3);
        const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(v[i].z * inv, v[i].w * inv),
                                                     __NV_SATFINITE, __NV_E4M3);
        reinterpret_cast<uint32_t*>(q8)[(size_t)t * n4 + j] = lo | (hi << 16);
    }
}

template <int VPT>
__global__ void __launch_bounds__(256) norm_vec_kernel(const float* __restrict__ x,
                                                       const int* __restrict__ rows, int d,
                                                       int kind, const float* __restrict__ w,
                                                       const float* __restrict__ b, float eps,
                                                       void* __restrict__ out, int out_type,
                                                       uint8_t* __restrict__ q8,
                                                       float* __restrict__ s8) {
    grid_dep_wait();                    // a no-op unless launched as a programmatic dependent
    grid_dep_launch();
    __shared__ float red[32];
    const int t = blockIdx.x;
    const int src = rows ? rows[t] : t;
    const float4* xr = reinterpret_cast<const float4*>(x + (size_t)src * d);
    const int n4 = d >> 2;
    float4 v[VPT];
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int j = threadIdx.x + i * 256;
        v[i] = j < n4 ? xr[j] : make_float4(0.f, 0.f, 0.f, 0.f);
        s += kind == 0 ? (v[i].x + v[i].y) + (v[i].z + v[i].w)
                       : (v[i].x * v[i].x + v[i].y * v[i].y) + (v[i].z * v[i].z + v[i].w * v[i].w);
    }
    norm_row_finish<VPT>(v, s, t, d, kind, w, b, eps, out, out_type, q8, s8, red);
}

// Residual reduction of a split-K GEMM with the next norm fused: row m of C (the fp32
// residual) gains sum_s slice_s[m] + bias, added slice by slice in split order exactly as the
// plain reduction adds them, and the updated row, still in registers, is normalised into the
// norm's output row m.  One CTA per row, 256 threads.
template <int VPT>
__global__ void __launch_bounds__(256) splitk_resid_norm_kernel(
    const float* __restrict__ ws, int ks, int M, int N, const float* __restrict__ bias,
    float* __restrict__ C, int ldc, const float* __restrict__ w, const float* __restrict__ b,
    int kind, float eps, void* __restrict__ out, int out_type, uint8_t* __restrict__ q8,
    float* __restrict__ s8) {
    grid_dep_wait();                    // a no-op unless launched as a programmatic dependent
    grid_dep_launch();
    __shared__ float red[32];
    const int m = blockIdx.x;
    const int n4 = N >> 2;
    float4* crow = reinterpret_cast<float4*>(C + (size_t)m * ldc);
    const float4* b4 = reinterpret_cast<const float4*>(bias);
    float4 v[VPT];
#pragma unroll
    for (int i = 0; i < VPT; ++i) v[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    // slices in split order; each slice's VPT loads per thread are independent, so they (and,
    // unrolled, those of the next slices) are in flight together
#pragma unroll 2
    for (int sl = 0; sl < ks; ++sl) {
        const float4* p4 = reinterpret_cast<const float4*>(ws + ((size_t)sl * M + m) * N);
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int j = threadIdx.x + i * 256;
            if (j < n4) {
                const float4 p = p4[j];
                v[i].x += p.x; v[i].y += p.y; v[i].z += p.z; v[i].w += p.w;
            }
        }
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int j = threadIdx.x + i * 256;
        if (j < n4) {
            const float4 bb = bias ? b4[j] : make_float4(0.f, 0.f, 0.f, 0.f);
            float4 c = crow[j];
            c.x += v[i].x + bb.x; c.y += v[i].y + bb.y; c.z += v[i].z + bb.z; c.w += v[i].w + bb.w;
            crow[j] = c;
            v[i] = c;
        }
        s += kind == 0 ? (v[i].x + v[i].y) + (v[i].z + v[i].w)
                       : (v[i].x * v[i].x + v[i].y * v[i].y) + (v[i].z * v[i].z + v[i].w * v[i].w);
    }
    norm_row_finish<VPT>(v, s, m, N, kind, w, b, eps, out, out_type, q8, s8, red);
}

// One CTA per row: amax, then the codes (used for the frozen weights at set-up).
__global__ void __launch_bounds__(256) quant_rows_e4m3_kernel(const void* __restrict__ x,
                                                              int x_type, int cols, size_t ldx,
                                                              uint8_t* __restrict__ q, size_t ldq,
                                                              float* __restrict__ scale) {
    __shared__ float red[32];
    const size_t r = blockIdx.x;
    float amax = 0.f;
    for (int i = threadIdx.x; i < cols; i += blockDim.x)
        amax = fmaxf(amax, fabsf(ld_elem(x, r * ldx + i, x_type)));
    amax = block_max(amax, red);
    const float inv = amax > 0.f ? 448.0f / amax : 1.0f;
    if (threadIdx.x == 0) scale[r] = amax > 0.f ? amax / 448.0f : 1.0f;
    for (int i = 2 * threadIdx.x; i < cols; i += 2 * blockDim.x) {
        const float a = ld_elem(x, r * ldx + i, x_type) * inv;
        const float b = i + 1 < cols ? ld_elem(x, r * ldx + i + 1, x_type) * inv : 0.f;
        const uint32_t c = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
        q[r * ldq + i] = (uint8_t)(c & 0xFFu);
        if (i + 1 < cols) q[r * ldq + i + 1] = (uint8_t)(c >> 8);
    }
}

void launch_quant_rows_e4m3(const void* x, int x_type, int rows, int cols, size_t ldx,
                            uint8_t* q, size_t ldq, float* scale, cudaStream_t st) {
    if (rows == 0) return;
    quant_rows_e4m3_kernel<<<rows, 256, 0, st>>>(x, x_type, cols, ldx, q, ldq, scale);
}

bool norm_fp8_supported(int d) { return d % 4 == 0 && (d / 4 + 255) / 256 <= 8; }

template <int VPT>
void norm_vec_go(bool pdl, int T, cudaStream_t st, const float* x, const int* rows, int d, int kind,
                 const float* w, const float* b, float eps, void* out, int out_type, uint8_t* q8,
                 float* s8) {
    if (pdl)
        launch_pdl(norm_vec_kernel<VPT>, dim3(T), dim3(256), 0, st, x, rows, d, kind, w, b, eps,
                   out, out_type, q8, s8);
    else
        norm_vec_kernel<VPT><<<T, 256, 0, st>>>(x, rows, d, kind, w, b, eps, out, out_type, q8, s8);
}

template <int VPT>
void resid_norm_go(bool pdl, const float* ws, int ks, int M, int N, const float* bias, float* C,
                   int ldc, const NormNext& nn, cudaStream_t st) {
    if (pdl)
        launch_pdl(splitk_resid_norm_kernel<VPT>, dim3(M), dim3(256), 0, st, ws, ks, M, N, bias, C,
                   ldc, nn.w, nn.b, nn.kind, nn.eps, nn.out, nn.out_type, nn.q8, nn.s8);
    else
        splitk_resid_norm_kernel<VPT><<<M, 256, 0, st>>>(ws, ks, M, N, bias, C, ldc, nn.w, nn.b,
                                                         nn.kind, nn.eps, nn.out, nn.out_type,
                                                         nn.q8, nn.s8);
}

bool launch_splitk_resid_norm(const float* ws, int ks, int M, int N, const float* bias, float* C,
                              int ldc, const NormNext& nn, cudaStream_t st, bool pdl) {
    if (M == 0) return true;
    const int vpt = (N / 4 + 255) / 256;
    auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (N % 4 || ldc % 4 || vpt > 8 || !al16(ws) || !al16(C) || !al16(nn.w) ||
        (nn.b && !al16(nn.b)) || (bias && !al16(bias)) || !al16(nn.out))
        return false;
    switch (vpt) {
        case 1: resid_norm_go<1>(pdl, ws, ks, M, N, bias, C, ldc, nn, st); break;
        case 2: resid_norm_go<2>(pdl, ws, ks, M, N, bias, C, ldc, nn, st); break;
        case 3: resid_norm_go<3>(pdl, ws, ks, M, N, bias, C, ldc, nn, st); break;
        case 4: resid_norm_go<4>(pdl, ws, ks, M, N, bias, C, ldc, nn, st); break;
        case 5: resid_norm_go<5>(pdl, ws, ks, M, N, bias, C, ldc, nn, st); break;
        case 6: resid_norm_go<6>(pdl, ws, ks, M, N, bias, C, ldc, nn, st); break;
        case 7: resid_norm_go<7>(pdl, ws, ks, M, N, bias, C, ldc, nn, st); break;
        default: resid_norm_go<8>(pdl, ws, ks, M, N, bias, C, ldc, nn, st); break;
    }
    return true;
}

void launch_norm(const float* x, const int* rows, int T, int d, int kind, const float* w,
                 const float* b, float eps, void* out, int out_type, cudaStream_t st,
                 uint8_t* q8, float* s8, bool pdl) {
    if (T == 0) return;
    const int vpt = (d / 4 + 255) / 256;
    auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    const bool aligned = al16(x) && al16(w) && (b == nullptr || al16(b)) && al16(out);
    if (d % 4 == 0 && vpt <= 8 && aligned) {
        switch (vpt) {
            case 1: norm_vec_go<1>(pdl, T, st, x, rows, d, kind, w, b, eps, out, out_type, q8, s8); return;
            case 2: norm_vec_go<2>(pdl, T, st, x, rows, d, kind, w, b, eps, out, out_type, q8, s8); return;
            case 3: norm_vec_go<3>(pdl, T, st, x, rows, d, kind, w, b, eps, out, out_type, q8, s8); return;
            case 4: norm_vec_go<4>(pdl, T, st, x, rows, d, kind, w, b, eps, out, out_type, q8, s8); return;
            case 5: norm_vec_go<5>(pdl, T, st, x, rows, d, kind, w, b, eps, out, out_type, q8, s8); return;
            case 6: norm_vec_go<6>(pdl, T, st, x, rows, d, kind, w, b, eps, out, out_type, q8, s8); return;
            case 7: norm_vec_go<7>(pdl, T, st, x, rows, d, kind, w, b, eps, out, out_type, q8, s8); return;
            default: norm_vec_go<8>(pdl, T, st, x, rows, d, kind, w, b, eps, out, out_type, q8, s8); return;
        }
    }
    norm_kernel<<<T, 256, d * sizeof(float), st>>>(x, rows, d, kind, w, b, eps, out, out_type);
    // the E4M3 rows of the bf16 output, when the vectorised form could not write them
    if (q8) launch_quant_rows_e4m3(out, out_type, T, d, (size_t)d, q8, (size_t)d, s8, st);
}

// out[t, j] = silu(gu[t, j]) * gu[t, f + j]; gu = [gate | up] per row.
__global__ void swiglu_kernel(const void* __restrict__ gu, int f, void* __restrict__ out,
                              int dtype) {
    const int t = blockIdx.x;
    const size_t gi = (size_t)t * 2 * f, oi = (size_t)t * f;
    for (int j = threadIdx.x; j < f; j += blockDim.x) {
        const float g = ld_elem(gu, gi + j, dtype);
        const float u = ld_elem(gu, gi + f + j, dtype);
        const float si = g / (1.0f + expf(-g));
        st_elem(out, oi + j, dtype, si * u);
    }
}

// Rotary table: cos / sin of pos * theta^(-2i/hd) for i < hd/2, angles in double.
__global__ void rope_table_kernel(float* cos_t, float* sin_t, int max_pos, int half, int hd,
                                  double theta) {
    const int n = max_pos * half;
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n; e += gridDim.x * blockDim.x) {
        const int pos = e / half, i = e % half;
        const double ang = (double)pos * pow(theta, -2.0 * i / hd);
        double sn, cs;
        sincos(ang, &sn, &cs);
        cos_t[e] = (float)cs;
        sin_t[e] = (float)sn;
    }
}

void launch_rope_table(float* cos_t, float* sin_t, int max_pos, int hd, double theta,
                       cudaStream_t st) {
    const int n = max_pos * (hd / 2);
    unsigned b = cdiv(n, 256);
    if (b > 148 * 8) b = 148 * 8;
    rope_table_kernel<<<b, 256, 0, st>>>(cos_t, sin_t, max_pos, hd / 2, hd, theta);
}

// Qwen3 q/k per-head RMSNorm then rotary positions (rotate-half pairs (i, i + hd/2)),
// in place on the q and k columns of the packed [T x ld] q|k|v rows.  One warp per
// (token, head); the position is the token's index within its row.
template <int HD>
__global__ void qk_norm_rope_kernel(void* qkv, int ld, int dtype, const int* __restrict__ tok_pos,
                                    int H, int Hkv, const float* __restrict__ qn,
                                    const float* __restrict__ kn, float eps,
                                    const float* __restrict__ cos_t,
                                    const float* __restrict__ sin_t, int T) {
    constexpr int PER = HD / 32, HALF = HD / 2;
    const int warps = blockDim.x >> 5;
    const int gw = blockIdx.x * warps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const int heads = H + Hkv;
    if (gw >= T * heads) return;
    const int t = gw / heads, hh = gw % heads;
    const float* nw = hh < H ? qn : kn;
    const size_t base = (size_t)t * ld + (size_t)hh * HD;
    // lane holds elements lane + 32 j: pairs (i, i + HD/2) sit in the same lane
    float x[PER];
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
        x[j] = ld_elem(qkv, base + lane + 32 * j, dtype);
        ss += x[j] * x[j];
    }
    ss = warp_sum(ss);
    const float rs = 1.0f / sqrtf(ss / (float)HD + eps);
#pragma unroll
    for (int j = 0; j < PER; ++j) x[j] = x[j] * rs * nw[lane + 32 * j];
    const size_t rb = (size_t)tok_pos[t] * HALF;
#pragma unroll
    for (int j = 0; j < PER / 2; ++j) {
        const int i = lane + 32 * j;                 // i < HD/2, partner at i + HD/2 = j + PER/2
        const float c = cos_t[rb + i], sn = sin_t[rb + i];
        const float a = x[j], b = x[j + PER / 2];
        x[j] = a * c - b * sn;
        x[j + PER / 2] = b * c + a * sn;
    }
#pragma unroll
    for (int j = 0; j < PER; ++j) st_elem(qkv, base + lane + 32 * j, dtype, x[j]);
}

void launch_qk_norm_rope(void* qkv, int ld, int dtype, const int* tok_pos, int T, int H, int Hkv,
                         int hd, const float* qn, const float* kn, float eps, const float* cos_t,
                         const float* sin_t, cudaStream_t st) {
    if (T == 0) return;
    const unsigned blocks = cdiv((long long)T * (H + Hkv), 8);
    switch (hd) {
        case 64: qk_norm_rope_kernel<64><<<blocks, 256, 0, st>>>(qkv, ld, dtype, tok_pos, H, Hkv, qn, kn, eps, cos_t, sin_t, T); break;
        case 128: qk_norm_rope_kernel<128><<<blocks, 256, 0, st>>>(qkv, ld, dtype, tok_pos, H, Hkv, qn, kn, eps, cos_t, sin_t, T); break;
        case 256: qk_norm_rope_kernel<256><<<blocks, 256, 0, st>>>(qkv, ld, dtype, tok_pos, H, Hkv, qn, kn, eps, cos_t, sin_t, T); break;
        default: break;
    }
}

void launch_swiglu(const void* gu, int T, int f, void* out, int dtype, cudaStream_t st) {
    if (T == 0) return;
    swiglu_kernel<<<T, 256, 0, st>>>(gu, f, out, dtype);
}

}  // namespace zo
