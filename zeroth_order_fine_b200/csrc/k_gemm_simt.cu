// CUDA-core GEMM C = A B^T (+ A2 B2^T) with the step's epilogues.
//
// The fp32 path of the library (exact-precision parity against the oracle)
// and the fallback for shapes the tensor-core kernel does not take.  64x64
// tiles, 16-deep K slices staged in shared memory, 4x4 outputs per thread,
// fp32 accumulation in a fixed K order, so every output element is a
// function of its own row of A and column of B only (row position in the
// packed batch never changes a bit).
#include <float.h>

#include "common.cuh"
#include "kernels.h"

namespace zo {

namespace {
constexpr int BM = 64, BN = 64, BK = 16;

template <int EPI>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmArgs g) {
    __shared__ __align__(16) float As[BK][BM + 4];
    __shared__ __align__(16) float Bs[BK][BN + 4];
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    const int lr = tid >> 2, lk = (tid & 3) * 4;   // loader: row lr, k lk..lk+3
    for (int part = 0; part < 2; ++part) {
        const void* A = part ? g.A2 : g.A;
        const void* B = part ? g.B2 : g.B;
        const int K = part ? g.K2 : g.K;
        const int lda = part ? g.lda2 : g.lda, ldb = part ? g.ldb2 : g.ldb;
        const int at = part ? g.a2_type : g.a_type, bt = part ? g.b2_type : g.b_type;
        if (A == nullptr || B == nullptr || K <= 0) continue;
        for (int k0 = 0; k0 < K; k0 += BK) {
            const int m = m0 + lr, n = n0 + lr;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int k = k0 + lk + i;
                As[lk + i][lr] = (m < g.M && k < K) ? ld_elem(A, (size_t)m * lda + k, at) : 0.f;
                Bs[lk + i][lr] = (n < g.N && k < K) ? ld_elem(B, (size_t)n * ldb + k, bt) : 0.f;
            }
            __syncthreads();
#pragma unroll
            for (int kk = 0; kk < BK; ++kk) {
                const float4 a = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
                const float4 b = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
                const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
            }
            __syncthreads();
        }
    }

    if constexpr (EPI == EPI_LSE) {
        // per row: max and sum of exp over this tile's valid columns; the 16
        // threads of a row sit in one half-warp
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int m = m0 + ty * 4 + i;
            float v[4], mx = -FLT_MAX;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int n = n0 + tx * 4 + j;
                v[j] = n < g.N ? acc[i][j] : -FLT_MAX;
                mx = fmaxf(mx, v[j]);
            }
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            float s = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (n0 + tx * 4 + j < g.N) s += expf(v[j] - mx);
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            int arg = 0x7fffffff;                  // lowest column holding the tile max
            if (g.part_arg) {
#pragma unroll
                for (int j = 3; j >= 0; --j)
                    if (n0 + tx * 4 + j < g.N && v[j] == mx) arg = n0 + tx * 4 + j;
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) arg = min(arg, __shfl_xor_sync(0xffffffffu, arg, o));
            }
            if (m < g.M) {
                if (tx == 0) {
                    g.part_max[(size_t)m * g.n_col_tiles + blockIdx.x] = mx;
                    g.part_sum[(size_t)m * g.n_col_tiles + blockIdx.x] = s;
                    if (g.part_arg) g.part_arg[(size_t)m * g.n_col_tiles + blockIdx.x] = arg;
                }
                const int tgt = g.targets[m] - (n0 + tx * 4);
                if (tgt >= 0 && tgt < 4 && g.targets[m] < g.N) g.tgt_logit[m] = v[tgt];
            }
        }
        return;
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int m = m0 + ty * 4 + i;
            if (m >= g.M) continue;
            float rs = 1.f;
            if (EPI == EPI_SHRINK) rs = (float)g.row_sign[m] * g.eps;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int n = n0 + tx * 4 + j;
                if (n >= g.N) continue;
                float v = acc[i][j];
                const size_t ci = (size_t)m * g.ldc + n;
                if (EPI == EPI_SHRINK) {
                    if (n < g.scale_cols) v *= rs;
                    st_elem(g.C, ci, g.c_type, v);
                } else if (EPI == EPI_RESID) {
                    if (g.bias) v += g.bias[n];
                    float* C = static_cast<float*>(g.C);
                    C[ci] += v;
                } else {
                    if (g.bias) v += g.bias[n];
                    if (EPI == EPI_STORE_RELU) v = fmaxf(v, 0.f);
                    st_elem(g.C, ci, g.c_type, v);
                }
            }
        }
    }
}
}  // namespace

int gemm_lse_col_tiles(int N) { return (N + BN - 1) / BN; }

void gemm_simt(const GemmArgs& g, cudaStream_t st) {
    if (g.M <= 0 || g.N <= 0) return;
    dim3 grid(cdiv(g.N, BN), cdiv(g.M, BM));
    switch (g.epi) {
        case EPI_STORE: gemm_simt_kernel<EPI_STORE><<<grid, 256, 0, st>>>(g); break;
        case EPI_STORE_RELU: gemm_simt_kernel<EPI_STORE_RELU><<<grid, 256, 0, st>>>(g); break;
        case EPI_RESID: gemm_simt_kernel<EPI_RESID><<<grid, 256, 0, st>>>(g); break;
        case EPI_SHRINK: gemm_simt_kernel<EPI_SHRINK><<<grid, 256, 0, st>>>(g); break;
        case EPI_LSE: gemm_simt_kernel<EPI_LSE><<<grid, 256, 0, st>>>(g); break;
        default: break;
    }
}

}  // namespace zo
