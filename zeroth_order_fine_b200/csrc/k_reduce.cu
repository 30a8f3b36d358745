// Objective, estimator and factored bank update.
//
//  * log-sum-exp merge of the lm_head tiles' partials, in fixed tile order;
//  * per-row objective L = -mean(log p) over the row's target span (fp64);
//  * c = mean_i (L+_i - L-_i) / (2 eps), no 1/r ("Zeroth-Order Fine-Tuning
//    Was an Inference Workload All Along", sections "Why ZO Fine-Tuning Is
//    Really Scoring" and "The System Reorganization"), reduced in a fixed
//    order in fp64 with warp shuffles;
//  * A_k <- A_k - lr c U_t for every target in one launch (the U-side
//    accumulator of the lazy window, same page, "Memory-write reduction"),
//    refused on the device when c is not finite.  U_t is regenerated from the
//    counter stream rather than read, and while the slot's coefficients since
//    it opened are known the slot is rebuilt from them rather than read, so a
//    step writes the accumulator without reading it.
#include <float.h>

#include "common.cuh"
#include "kernels.h"
#include "rng.cuh"

namespace zo {

ZO_DEBUG_WORD(debug_word_reduce)

// One warp per scored position; lanes take tiles lane, lane+32, ... and the
// lane results are combined by a fixed xor tree.
__global__ void lse_merge_kernel(const float* __restrict__ pmax, const float* __restrict__ psum,
                                 const float* __restrict__ tgt, int S, int n_tiles,
                                 float* __restrict__ logprob) {
    const int s = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (s >= S) return;
    const float* pm = pmax + (size_t)s * n_tiles;
    const float* ps = psum + (size_t)s * n_tiles;
    float m = -FLT_MAX;
    for (int i = lane; i < n_tiles; i += 32) m = fmaxf(m, pm[i]);
    m = warp_max(m);
    float z = 0.f;
    for (int i = lane; i < n_tiles; i += 32) z += ps[i] * expf(pm[i] - m);
    z = warp_sum(z);
    if (lane == 0) logprob[s] = tgt[s] - (m + logf(z));
}

void launch_lse_merge(const float* part_max, const float* part_sum, const float* tgt_logit,
                      int S, int n_tiles, float* logprob, cudaStream_t st) {
    if (S == 0) return;
    lse_merge_kernel<<<cdiv(S, 8), 256, 0, st>>>(part_max, part_sum, tgt_logit, S, n_tiles,
                                                 logprob);
}

__global__ void lse_argmax_merge_kernel(const float* __restrict__ pmax, const float* __restrict__ psum,
                                        const int* __restrict__ parg, int S, int n_tiles,
                                        int* __restrict__ token, float* __restrict__ logprob,
                                        int stride) {
    const int s = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (s >= S) return;
    const float* pm = pmax + (size_t)s * n_tiles;
    const float* ps = psum + (size_t)s * n_tiles;
    float m = -FLT_MAX;
    for (int i = lane; i < n_tiles; i += 32) m = fmaxf(m, pm[i]);
    m = warp_max(m);
    int first = 0x7fffffff;                  // the lowest tile holding the maximum
    for (int i = lane; i < n_tiles; i += 32)
        if (pm[i] == m) first = min(first, i);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) first = min(first, __shfl_xor_sync(0xffffffffu, first, o));
    float z = 0.f;
    for (int i = lane; i < n_tiles; i += 32) z += ps[i] * expf(pm[i] - m);
    z = warp_sum(z);
    if (lane == 0) {
        token[(size_t)s * stride] = parg[(size_t)s * n_tiles + first];
        logprob[(size_t)s * stride] = m - (m + logf(z));
    }
}

void launch_lse_argmax_merge(const float* part_max, const float* part_sum, const int* part_arg,
                             int S, int n_tiles, int* token, float* logprob, int stride,
                             cudaStream_t st) {
    if (S == 0) return;
    lse_argmax_merge_kernel<<<cdiv(S, 8), 256, 0, st>>>(part_max, part_sum, part_arg, S, n_tiles,
                                                        token, logprob, stride);
}

__global__ void row_objective_kernel(const float* __restrict__ logprob,
                                     const int* __restrict__ score_off, int R, int B,
                                     long long S, double* __restrict__ L_row, float* L_plus,
                                     float* L_minus) {
    const int r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= R) return;
    int a = score_off[r], b = score_off[r + 1];
    // (debug build) a span outside [0, S) is not read: an empty span gives L = NaN
    if (!ZO_DCHECK(a >= 0 && a <= b && b <= S, ZO_DBG_SCORE_SPAN)) a = b = 0;
    double s = 0.0;
    for (int i = a; i < b; ++i) s += (double)logprob[i];
    const double L = -s / (double)(b - a);
    L_row[r] = L;
    if (r < B && L_plus) L_plus[r] = (float)L;
    else if (r >= B && r < 2 * B && L_minus) L_minus[r - B] = (float)L;
}

void launch_row_objective(const float* logprob, const int* score_off, int R, int B, long long S,
                          double* L_row, float* L_plus, float* L_minus, cudaStream_t st) {
    if (R == 0) return;
    row_objective_kernel<<<cdiv(R, 128), 128, 0, st>>>(logprob, score_off, R, B, S, L_row, L_plus,
                                                       L_minus);
}

// sums[0] = sum_i (L+_i - L-_i), sums[1] = B; one CTA, fixed order.
__global__ void objective_sums_kernel(const double* __restrict__ L_row, int B, double* sums) {
    __shared__ double red[32];
    double s = 0.0;
    for (int i = threadIdx.x; i < B; i += blockDim.x) s += L_row[i] - L_row[B + i];
    s = warp_sum_d(s);
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    if (lane == 0) red[w] = s;
    __syncthreads();
    if (w == 0) {
        double v = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.0;
        v = warp_sum_d(v);
        if (lane == 0) {
            sums[0] = v;
            sums[1] = (double)B;
        }
    }
}

void launch_objective_sums(const double* L_row, int B, double* sums, cudaStream_t st) {
    objective_sums_kernel<<<1, 256, 0, st>>>(L_row, B, sums);
}

__global__ void estimate_kernel(const double* sums, float eps, double* c, int* flag) {
    const double v = sums[0] / sums[1] / (2.0 * (double)eps);
    *c = v;
    *flag = isfinite(v) ? 0 : 1;
}

void launch_estimate(const double* sums, float eps, double* c, int* flag, cudaStream_t st) {
    estimate_kernel<<<1, 1, 0, st>>>(sums, eps, c, flag);
}

// One launch over every target: blockIdx.y = target, one thread per N(0,1) pair of U_t.
__global__ void __launch_bounds__(256) bank_update_kernel(
    const UpdateJob* __restrict__ jobs, const double* __restrict__ c, const int* __restrict__ flag,
    float lr, uint64_t run_seed, uint64_t step, const uint64_t* __restrict__ step_dev, uint64_t nu,
    float scale, int apply_scale, long long replay_from, float* __restrict__ coef_hist) {
    const UpdateJob jb = jobs[blockIdx.y];
    const uint64_t t = step_dev ? *step_dev : step;
    const float coef_t = *flag ? 0.0f : (float)((double)lr * *c);   // non-finite c: refused
    const bool replay = replay_from >= 0;
    const uint64_t s0 = replay ? (uint64_t)replay_from : t;
    if (replay && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0)
        coef_hist[t - s0] = coef_t;                 // later steps replay it; read below only for s < t
    const uint64_t n = (uint64_t)jb.dim * jb.r;
    const uint64_t npairs = (n + 1) / 2;
    for (uint64_t j = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; j < npairs;
         j += (uint64_t)gridDim.x * blockDim.x) {
        const uint64_t e0 = 2 * j, e1 = 2 * j + 1;
        const bool has1 = e1 < n;
        const uint64_t o0 = (e0 % jb.r) * (uint64_t)jb.ld + e0 / jb.r;
        const uint64_t o1 = has1 ? (e1 % jb.r) * (uint64_t)jb.ld + e1 / jb.r : o0;
        float a0 = replay ? 0.0f : jb.A[o0];
        float a1 = (replay || !has1) ? 0.0f : jb.A[o1];
        for (uint64_t s = s0; s <= t; ++s) {
            const float cf = s < t ? coef_hist[s - s0] : coef_t;
            float z0, z1;
            normal_pair(factor_key(run_seed, s, nu, (uint32_t)jb.layer, (uint32_t)jb.matrix, 0), j,
                        &z0, &z1);
            if (apply_scale) {
                z0 = __fmul_rn(z0, scale);
                z1 = __fmul_rn(z1, scale);
            }
            a0 = __fmaf_rn(-cf, z0, a0);
            a1 = __fmaf_rn(-cf, z1, a1);
        }
        jb.A[o0] = a0;
        if (jb.A_bf) static_cast<__nv_bfloat16*>(jb.A_bf)[o0] = __float2bfloat16_rn(a0);
        if (has1) {
            jb.A[o1] = a1;
            if (jb.A_bf) static_cast<__nv_bfloat16*>(jb.A_bf)[o1] = __float2bfloat16_rn(a1);
        }
    }
}

void launch_bank_update(const UpdateJob* jobs, int n_jobs, int max_pairs, const double* c,
                        const int* flag, float lr, uint64_t run_seed, uint64_t step,
                        const uint64_t* step_dev, uint64_t nu, float scale, int apply_scale,
                        long long replay_from, float* coef_hist, cudaStream_t st) {
    if (n_jobs == 0) return;
    unsigned bx = cdiv(max_pairs, 256);
    if (bx > 64) bx = 64;
    if (bx == 0) bx = 1;
    dim3 grid(bx, n_jobs);
    bank_update_kernel<<<grid, 256, 0, st>>>(jobs, c, flag, lr, run_seed, step, step_dev, nu, scale,
                                             apply_scale, replay_from, coef_hist);
}

}  // namespace zo
