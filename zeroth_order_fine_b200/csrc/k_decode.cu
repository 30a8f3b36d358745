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

ZO_DEBUG_WORD(debug_word_decode)

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
                                  size_t cache_rows, int es) {
    const int t = blockIdx.x;
    const size_t crow = (size_t)t + (size_t)tok_row[t] * G;
    if (!ZO_DCHECK(crow < cache_rows, ZO_DBG_KV_SLOT)) return;     // (debug build)
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
                                 int G, char* __restrict__ cache, size_t cache_rows, int es) {
    grid_dep_wait();                    // launched as a programmatic dependent
    grid_dep_launch();
    const int r = blockIdx.x;
    const size_t crow = (size_t)cu[r] + (size_t)r * G + lens[r] + g;
    if (!ZO_DCHECK(crow < cache_rows, ZO_DBG_KV_SLOT)) return;     // (debug build)
    copy_row(qkv + ((size_t)r * ld_qkv + q_dim) * es, cache + crow * kv2 * es, kv2, es);
}

__device__ __forceinline__ void bf16x8(const uint4& u, float* f) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 t = __bfloat1622float2(h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

// 8 consecutive elements at off (a multiple of 8): one 16-byte load (bf16) or two (fp32)
__device__ __forceinline__ void load8(const void* base, size_t off, int dtype, float* v) {
    if (dtype == E_F32) {
        const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + off);
        const float4 a = p[0], b = p[1];
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
        bf16x8(*reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + off), v);
    }
}

// One CTA per (row, kv head, key split): the n_rep query heads that share the kv head (NREP =
// n_rep rounded up to a power of two; the padding heads have q = 0 and are not written), over
// the keys [kbeg, kend) of the row, in tiles of kt keys.  Per tile:
//   0. the tile's k and v rows of this head go to shared memory by asynchronous 16-byte
//      copies, all issued at once, so the whole tile is in flight together;
//   1. scores s[h][j] = scale * q_h . k_j: a key row is read by LPK = HD/8 adjacent lanes (8
//      elements each), the dot finished by xor shuffles over those lanes;
//   2. one warp per head: tile max, running max m, p = exp(s - m), running sum l, and the
//      rescale factor of the older keys;
//   3. o[h] += sum_j p[h][j] v_j, each lane accumulating its 8 dims over its key slot's keys.
// The key slots' partial outputs are added in slot order at the end.  With part == nullptr
// (one split) the CTA writes o / l; else (m, l, unnormalised o) per head for
// decode_merge_kernel, which combines the splits in split order.
constexpr int DEC_THREADS = 128, DEC_WARPS = DEC_THREADS / 32, DEC_KT_MAX = 128;
constexpr int DEC_MAX_REP = 8;

// keys per tile: the tile's k and v rows fill 64 KB of shared memory, at most DEC_KT_MAX
inline int dec_tile_keys(int hd, int es) { return std::min(DEC_KT_MAX, 65536 / (2 * hd * es)); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
// wait until at most N of this thread's committed copy groups are still in flight
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// 8 consecutive elements of a shared-memory row (bf16 or fp32)
__device__ __forceinline__ void smem8(const uint8_t* p, int es, float* v) {
    if (es == 4) {
        const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
        bf16x8(*reinterpret_cast<const uint4*>(p), v);
    }
}

template <int HD, int NREP>
__global__ void __launch_bounds__(DEC_THREADS) decode_attention_kernel(
    const void* __restrict__ qkv, int ld_qkv, const void* __restrict__ cache, int kv2,
    const int* __restrict__ cu, const int* __restrict__ lens, int g, int G, int Hkv, int n_rep,
    float scale, void* __restrict__ out, int ld_out, int dtype, int kps, int kt,
    float* __restrict__ part) {
    constexpr int LPK = HD / 8;                        // lanes per key
    constexpr int KPW = 32 / LPK;                      // keys per warp-wide access
    constexpr int SLOTS = DEC_WARPS * KPW;             // keys per CTA-wide access
    constexpr int U = NREP >= 8 ? 2 : 4;               // keys per lane per round
    grid_dep_wait();                                   // launched as a programmatic dependent
    grid_dep_launch();
    extern __shared__ __align__(16) uint8_t dsm[];
    const int es = dtype == E_F32 ? 4 : 2;
    const int row_bytes = HD * es;
    uint8_t* Ks = dsm;                                 // [kt][HD] elements
    uint8_t* Vs = dsm + (size_t)kt * row_bytes;        // [kt][HD]
    float* so = reinterpret_cast<float*>(dsm);         // [SLOTS][NREP][HD], after the last tile
    const size_t kv_bytes = (size_t)2 * kt * row_bytes, so_bytes = (size_t)SLOTS * NREP * HD * 4;
    const size_t tiles_bytes = kv_bytes > so_bytes ? kv_bytes : so_bytes;
    float* sp = reinterpret_cast<float*>(dsm + tiles_bytes);   // [NREP][kt]
    __shared__ float s_alpha[NREP], s_m[NREP], s_l[NREP];
    const int r = blockIdx.x, kvh = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / LPK, slot = warp * KPW + sub, d0 = (lane % LPK) * 8;
    const size_t base = (size_t)cu[r] + (size_t)r * G;
    const int n = lens[r] + g + 1;
    const int kbeg = blockIdx.z * kps, kend = min(n, kbeg + kps);
    const int kv_dim = kv2 / 2;
    float q[NREP][8], o[NREP][8];
#pragma unroll
    for (int h = 0; h < NREP; ++h) {
#pragma unroll
        for (int e = 0; e < 8; ++e) o[h][e] = q[h][e] = 0.f;
        if (h < n_rep)
            load8(qkv, (size_t)r * ld_qkv + (size_t)(kvh * n_rep + h) * HD + d0, dtype, q[h]);
    }
    if (threadIdx.x < NREP) {
        s_m[threadIdx.x] = -FLT_MAX;
        s_l[threadIdx.x] = 0.f;
    }
    const char* cbase = static_cast<const char*>(cache);
    const int chunks = row_bytes / 16;                 // 16-byte pieces per row
    const uint32_t ks_addr = static_cast<uint32_t>(__cvta_generic_to_shared(Ks));
    const uint32_t vs_addr = static_cast<uint32_t>(__cvta_generic_to_shared(Vs));
    for (int t0 = kbeg; t0 < kend; t0 += kt) {
        const int nt = min(kt, kend - t0);
        // 0. the tile's k rows, then its v rows, of this head: two copy groups, so that the
        //    scores and the softmax run while the v rows are still landing
        for (int c = threadIdx.x; c < nt * chunks; c += DEC_THREADS) {
            const int row = c / chunks, pc = c - row * chunks;
            cp_async16(ks_addr + row * row_bytes + pc * 16,
                       cbase + ((base + t0 + row) * kv2 + (size_t)kvh * HD) * es + pc * 16);
        }
        cp_async_commit();
        for (int c = threadIdx.x; c < nt * chunks; c += DEC_THREADS) {
            const int row = c / chunks, pc = c - row * chunks;
            cp_async16(vs_addr + row * row_bytes + pc * 16,
                       cbase + ((base + t0 + row) * kv2 + (size_t)kv_dim + (size_t)kvh * HD) * es +
                           pc * 16);
        }
        cp_async_commit();
        cp_async_wait<1>();                            // this thread's k copies have landed
        __syncthreads();
        // 1. scores; the loop bounds are uniform over the warp (the shuffles need every lane)
        for (int i0 = warp * KPW; i0 < nt; i0 += U * SLOTS) {
            float k[U][8];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int j = i0 + sub + u * SLOTS;
                if (j < nt) {
                    smem8(Ks + j * row_bytes + d0 * es, es, k[u]);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) k[u][e] = 0.f;
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int j = i0 + sub + u * SLOTS;
#pragma unroll
                for (int h = 0; h < NREP; ++h) {
                    float s_ = 0.f;
#pragma unroll
                    for (int e = 0; e < 8; ++e) s_ = fmaf(q[h][e], k[u][e], s_);
#pragma unroll
                    for (int x = LPK / 2; x > 0; x >>= 1) s_ += __shfl_xor_sync(0xffffffffu, s_, x);
                    if (d0 == 0 && j < nt) sp[h * kt + j] = s_ * scale;
                }
            }
        }
        __syncthreads();
        // 2. softmax statistics, one warp per head
        for (int h = warp; h < NREP; h += DEC_WARPS) {
            float mx = -FLT_MAX;
            for (int j = lane; j < nt; j += 32) mx = fmaxf(mx, sp[h * kt + j]);
            mx = warp_max(mx);
            const float m_old = s_m[h];
            const float m_new = fmaxf(m_old, mx);
            float sum = 0.f;
            for (int j = lane; j < nt; j += 32) {
                const float pj = expf(sp[h * kt + j] - m_new);
                sp[h * kt + j] = pj;
                sum += pj;
            }
            sum = warp_sum(sum);
            if (lane == 0) {
                const float alpha = m_old > -FLT_MAX ? expf(m_old - m_new) : 0.f;
                s_alpha[h] = alpha;
                s_m[h] = m_new;
                s_l[h] = s_l[h] * alpha + sum;
            }
        }
        cp_async_wait<0>();                            // and its v copies
        __syncthreads();
        // 3. o = alpha * o + P V
#pragma unroll
        for (int h = 0; h < NREP; ++h) {
            const float a = s_alpha[h];
#pragma unroll
            for (int e = 0; e < 8; ++e) o[h][e] *= a;
        }
        for (int j = slot; j < nt; j += SLOTS) {
            float v[8];
            smem8(Vs + j * row_bytes + d0 * es, es, v);
#pragma unroll
            for (int h = 0; h < NREP; ++h) {
                const float pj = sp[h * kt + j];
#pragma unroll
                for (int e = 0; e < 8; ++e) o[h][e] = fmaf(pj, v[e], o[h][e]);
            }
        }
        __syncthreads();                               // the tile buffers are refilled next
    }
    // add the key slots' partial outputs in slot order (so reuses the tile buffers)
#pragma unroll
    for (int h = 0; h < NREP; ++h)
#pragma unroll
        for (int e = 0; e < 8; ++e) so[(slot * NREP + h) * HD + d0 + e] = o[h][e];
    __syncthreads();
    const int S = gridDim.z;
    float* pr = part ? part + ((size_t)(r * Hkv + kvh) * S + blockIdx.z) * n_rep * (HD + 2) : nullptr;
    for (int idx = threadIdx.x; idx < n_rep * HD; idx += DEC_THREADS) {
        const int h = idx / HD, dd = idx % HD;
        float acc = 0.f;
#pragma unroll 4
        for (int sl = 0; sl < SLOTS; ++sl) acc += so[(sl * NREP + h) * HD + dd];
        const float ll = s_l[h];
        if (pr) {
            pr[h * (HD + 2) + dd] = acc;
            if (dd == 0) {
                pr[h * (HD + 2) + HD] = s_m[h];
                pr[h * (HD + 2) + HD + 1] = ll;
            }
        } else {
            st_elem(out, (size_t)r * ld_out + (size_t)(kvh * n_rep + h) * HD + dd, dtype,
                    ll > 0.f ? acc / ll : 0.f);
        }
    }
}

// Combine the key splits of one (row, kv head) in split order.
template <int HD>
__global__ void decode_merge_kernel(const float* __restrict__ part, int S, int n_rep, int Hkv,
                                    void* __restrict__ out, int ld_out, int dtype) {
    grid_dep_wait();                    // launched as a programmatic dependent
    grid_dep_launch();
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
    grid_dep_wait();
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
                       int T, int G, void* cache, size_t cache_rows, int dtype, cudaStream_t st) {
    if (T == 0) return;
    kv_scatter_kernel<<<T, 128, 0, st>>>(static_cast<const char*>(qkv), ld_qkv, q_dim, kv2,
                                         tok_row, G, static_cast<char*>(cache), cache_rows,
                                         dtype == E_F32 ? 4 : 2);
}

void launch_decode_prep(const int* gen_tok, int G, int g, const int* lens, int R, int B,
                        int* tok_id, int* tok_pos, int* tok_sign, int* tok_row, cudaStream_t st) {
    if (R == 0) return;
    decode_prep_kernel<<<cdiv(R, 128), 128, 0, st>>>(gen_tok, G, g, lens, R, B, tok_id, tok_pos,
                                                     tok_sign, tok_row);
}

void launch_kv_append(const void* qkv, int ld_qkv, int q_dim, int kv2, const int* cu,
                      const int* lens, int R, int g, int G, void* cache, size_t cache_rows,
                      int dtype, cudaStream_t st) {
    if (R == 0) return;
    launch_pdl(kv_append_kernel, dim3(R), dim3(128), 0, st, static_cast<const char*>(qkv), ld_qkv,
               q_dim, kv2, cu, lens, g, G, static_cast<char*>(cache), cache_rows,
               dtype == E_F32 ? 4 : 2);
}

template <int HD, int NR>
bool launch_dec(dim3 grid, size_t smem, cudaStream_t st, const void* qkv, int ld_qkv,
                const void* cache, int kv2, const int* cu, const int* lens, int g, int G, int Hkv,
                int n_rep, float scale, void* out, int ld_out, int dtype, int kps, int kt,
                float* part) {
    static size_t attr = 48 * 1024;
    if (smem > attr) {
        if (cudaFuncSetAttribute(decode_attention_kernel<HD, NR>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return false;
        attr = smem;
    }
    return launch_pdl(decode_attention_kernel<HD, NR>, grid, dim3(DEC_THREADS), smem, st, qkv,
                      ld_qkv, cache, kv2, cu, lens, g, G, Hkv, n_rep, scale, out, ld_out, dtype, kps,
                      kt, part) == cudaSuccess;
}

template <int HD>
bool launch_dec_hd(int nrep_p, dim3 grid, size_t smem, cudaStream_t st, const void* qkv,
                   int ld_qkv, const void* cache, int kv2, const int* cu, const int* lens, int g,
                   int G, int Hkv, int n_rep, float scale, void* out, int ld_out, int dtype,
                   int kps, int kt, float* part) {
    switch (nrep_p) {
        case 1: return launch_dec<HD, 1>(grid, smem, st, qkv, ld_qkv, cache, kv2, cu, lens, g, G, Hkv, n_rep, scale, out, ld_out, dtype, kps, kt, part);
        case 2: return launch_dec<HD, 2>(grid, smem, st, qkv, ld_qkv, cache, kv2, cu, lens, g, G, Hkv, n_rep, scale, out, ld_out, dtype, kps, kt, part);
        case 4: return launch_dec<HD, 4>(grid, smem, st, qkv, ld_qkv, cache, kv2, cu, lens, g, G, Hkv, n_rep, scale, out, ld_out, dtype, kps, kt, part);
        default: return launch_dec<HD, 8>(grid, smem, st, qkv, ld_qkv, cache, kv2, cu, lens, g, G, Hkv, n_rep, scale, out, ld_out, dtype, kps, kt, part);
    }
}

bool launch_decode_attention(const void* qkv, int ld_qkv, const void* cache, int kv2,
                             const int* cu, const int* lens, int R, int g, int G, int H, int Hkv,
                             int hd, float scale, void* out, int ld_out, int dtype, int max_n,
                             float* ws, size_t ws_floats, cudaStream_t st) {
    if (Hkv <= 0 || H % Hkv || H / Hkv > DEC_MAX_REP) return false;
    if (hd != 32 && hd != 64 && hd != 128 && hd != 256) return false;
    if (R == 0) return true;
    const int n_rep = H / Hkv;
    const int es = dtype == E_F32 ? 4 : 2;
    int kt = dec_tile_keys(hd, es);
    // with fewer than ~4 (row, kv head) CTAs per SM, split the keys into tiles so enough
    // copies stay in flight; the splits' partial softmaxes are combined in order by the merge
    // kernel.  Without a split a CTA walks its keys in half-size tiles: twice the CTAs fit on
    // an SM (2.7% faster OPT-13B b16 generation steps; with splits the full tile was faster).
    const bool many = (long long)R * Hkv >= 4 * 148;
    int S = many ? 1 : (max_n + kt - 1) / kt;
    if (S < 1) S = 1;
    if ((size_t)R * Hkv * S * n_rep * (hd + 2) > ws_floats) S = 1;
    if (S == 1) kt = std::max(16, kt / 2);
    const int kps = S == 1 ? max_n : kt;
    float* part = S > 1 ? ws : nullptr;
    const int nrep_p = n_rep == 1 ? 1 : n_rep == 2 ? 2 : n_rep <= 4 ? 4 : 8;
    const size_t slots_bytes = (size_t)(1024 / hd) * nrep_p * hd * 4;
    const size_t smem = std::max((size_t)2 * kt * hd * es, slots_bytes) + (size_t)nrep_p * kt * 4;
    dim3 grid(R, Hkv, S);
    bool ok;
    switch (hd) {
        case 32: ok = launch_dec_hd<32>(nrep_p, grid, smem, st, qkv, ld_qkv, cache, kv2, cu, lens, g, G, Hkv, n_rep, scale, out, ld_out, dtype, kps, kt, part); break;
        case 64: ok = launch_dec_hd<64>(nrep_p, grid, smem, st, qkv, ld_qkv, cache, kv2, cu, lens, g, G, Hkv, n_rep, scale, out, ld_out, dtype, kps, kt, part); break;
        case 128: ok = launch_dec_hd<128>(nrep_p, grid, smem, st, qkv, ld_qkv, cache, kv2, cu, lens, g, G, Hkv, n_rep, scale, out, ld_out, dtype, kps, kt, part); break;
        default: ok = launch_dec_hd<256>(nrep_p, grid, smem, st, qkv, ld_qkv, cache, kv2, cu, lens, g, G, Hkv, n_rep, scale, out, ld_out, dtype, kps, kt, part); break;
    }
    if (!ok) return false;
    if (S > 1) {
        dim3 mg(R, Hkv);
        switch (hd) {
            case 32: launch_pdl(decode_merge_kernel<32>, mg, dim3(128), 0, st, (const float*)part, S, n_rep, Hkv, out, ld_out, dtype); break;
            case 64: launch_pdl(decode_merge_kernel<64>, mg, dim3(128), 0, st, (const float*)part, S, n_rep, Hkv, out, ld_out, dtype); break;
            case 128: launch_pdl(decode_merge_kernel<128>, mg, dim3(128), 0, st, (const float*)part, S, n_rep, Hkv, out, ld_out, dtype); break;
            default: launch_pdl(decode_merge_kernel<256>, mg, dim3(128), 0, st, (const float*)part, S, n_rep, Hkv, out, ld_out, dtype); break;
        }
    }
    return cudaGetLastError() == cudaSuccess;
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

void launch_shrink_rows_sum(const float* part, int ks, int M, int N, void* C, int ldc, int c_type,
                            const int* row_sign, float eps, int scale_cols, const float* a_scale,
                            cudaStream_t st, bool pdl) {
    if (M == 0 || N == 0) return;
    const dim3 grid(cdiv((long long)M * N, 256));
    if (pdl) {
        launch_pdl(shrink_rows_sum_kernel, grid, dim3(256), 0, st, part, ks, M, N, C, ldc, c_type,
                   row_sign, eps, scale_cols, a_scale);
        return;
    }
    shrink_rows_sum_kernel<<<grid, 256, 0, st>>>(part, ks, M, N, C, ldc, c_type, row_sign, eps,
                                                 scale_cols, a_scale);
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
