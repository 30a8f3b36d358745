// Direction generator (U_t every step, V at each lazy-window start) and the
// counter-stream weight initialiser.  HBM-bound writers: one thread per
// N(0,1) pair, 8-byte stores, grids sized in multiples of the SM count.
#include "common.cuh"
#include "kernels.h"
#include "rng.cuh"

namespace zo {

// ---- weights ------------------------------------------------------------------------
__global__ void __launch_bounds__(256) init_tensor_kernel(void* dst, uint64_t n, uint64_t key,
                                                          float std_, float mean, int dtype) {
    const uint64_t npairs = (n + 1) / 2;
    for (uint64_t j = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; j < npairs;
         j += (uint64_t)gridDim.x * blockDim.x) {
        float z0, z1;
        normal_pair(key, j, &z0, &z1);
        float w0 = __fmul_rn(z0, std_), w1 = __fmul_rn(z1, std_);
        if (mean != 0.0f) { w0 = __fadd_rn(w0, mean); w1 = __fadd_rn(w1, mean); }
        const uint64_t e = 2 * j;
        if (dtype == E_F32) {
            float* d = static_cast<float*>(dst);
            if (e + 1 < n && (n % 2 == 0)) {
                reinterpret_cast<float2*>(d)[j] = make_float2(w0, w1);
            } else {
                d[e] = w0;
                if (e + 1 < n) d[e + 1] = w1;
            }
        } else {
            __nv_bfloat16* d = static_cast<__nv_bfloat16*>(dst);
            if (e + 1 < n && (n % 2 == 0)) {
                reinterpret_cast<__nv_bfloat162*>(d)[j] =
                    __halves2bfloat162(__float2bfloat16_rn(w0), __float2bfloat16_rn(w1));
            } else {
                d[e] = __float2bfloat16_rn(w0);
                if (e + 1 < n) d[e + 1] = __float2bfloat16_rn(w1);
            }
        }
    }
}

void launch_init_tensor(void* dst, uint64_t n, uint64_t key, float std_, float mean, int dtype,
                        cudaStream_t st) {
    if (n == 0) return;
    const uint64_t npairs = (n + 1) / 2;
    uint64_t blocks = (npairs + 255) / 256;
    const uint64_t cap = 148ull * 16;
    if (blocks > cap) blocks = cap;
    init_tensor_kernel<<<(unsigned)blocks, 256, 0, st>>>(dst, n, key, std_, mean, dtype);
}

// ---- directions ---------------------------------------------------------------------
// One job per (target, factor).  Element e = i*r + c of the row-major [dim x r]
// factor is written to dst[c * ld + i] (U: the transposed rows the shrink GEMM
// reads) or dst[e] (V: row-major, kept for the window); dst or its bf16 mirror
// dst_bf may be null (bf16 models keep U in bf16 only).
__global__ void __launch_bounds__(256) gen_factors_kernel(const GenJob* jobs, int n_jobs,
                                                          uint64_t run_seed, uint64_t step,
                                                          const uint64_t* step_dev,
                                                          uint64_t nu, float scale,
                                                          int apply_scale) {
    const GenJob jb = jobs[blockIdx.y];
    // a captured step graph reads the step from device memory, an eager launch takes it by value
    const uint64_t t = step_dev ? *step_dev : step;
    const uint64_t key = factor_key(run_seed, t, nu, jb.layer, jb.matrix, jb.which);
    const uint64_t n = (uint64_t)jb.dim * jb.r;
    const uint64_t npairs = (n + 1) / 2;
    for (uint64_t j = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; j < npairs;
         j += (uint64_t)gridDim.x * blockDim.x) {
        float z[2];
        normal_pair(key, j, &z[0], &z[1]);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint64_t e = 2 * j + h;
            if (e >= n) break;
            float v = z[h];
            if (apply_scale) v = __fmul_rn(v, scale);
            const uint64_t o = jb.transposed ? (e % jb.r) * (uint64_t)jb.ld + e / jb.r : e;
            if (jb.dst) jb.dst[o] = v;
            if (jb.dst_bf) static_cast<__nv_bfloat16*>(jb.dst_bf)[o] = __float2bfloat16_rn(v);
        }
    }
}

void launch_gen_factors(const GenJob* d_jobs, int n_jobs, int max_pairs, uint64_t run_seed,
                        uint64_t step, const uint64_t* step_dev, uint64_t nu, float scale,
                        int apply_scale, cudaStream_t st) {
    if (n_jobs == 0) return;
    unsigned bx = cdiv(max_pairs, 256);
    if (bx > 64) bx = 64;
    if (bx == 0) bx = 1;
    dim3 grid(bx, n_jobs);
    gen_factors_kernel<<<grid, 256, 0, st>>>(d_jobs, n_jobs, run_seed, step, step_dev, nu, scale,
                                             apply_scale);
}

__global__ void set_step_kernel(uint64_t* step_dev, uint64_t v, int add) {
    *step_dev = add ? *step_dev + v : v;
}

void launch_set_step(uint64_t* step_dev, uint64_t v, cudaStream_t st) {
    set_step_kernel<<<1, 1, 0, st>>>(step_dev, v, 0);
}

void launch_advance_step(uint64_t* step_dev, cudaStream_t st) {
    set_step_kernel<<<1, 1, 0, st>>>(step_dev, 1, 1);
}

// Window opening: write the new window's V (row-major [d_out x r], fp32) into
// the extension operand E_B (rows row0.., in the model dtype) at two column
// blocks -- the direction block (cols col_dir..) and the new slot's block
// (cols col_slot..) -- and zero the slot's accumulator rows A_k^T [r x d_in].
__global__ void open_window_kernel(const WindowJob* jobs) {
    const WindowJob jb = jobs[blockIdx.y];
    const int n = jb.d_out * jb.r;
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n; e += gridDim.x * blockDim.x) {
        const int i = e / jb.r, c = e % jb.r;
        const int fr = jb.interleave ? (i / 128) * 256 + jb.row0 + i % 128 : jb.row0 + i;
        const float v = jb.row_div ? jb.V[e] / jb.row_div[fr] : jb.V[e];
        const size_t row = (size_t)fr * jb.ldb;
        st_elem(jb.EB, row + jb.col_dir + c, jb.eb_type, v);
        st_elem(jb.EB, row + jb.col_slot + c, jb.eb_type, v);
    }
    const int na = jb.d_in * jb.r;
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < na; e += gridDim.x * blockDim.x) {
        jb.A[e] = 0.0f;
        if (jb.A_bf) static_cast<__nv_bfloat16*>(jb.A_bf)[e] = __float2bfloat16_rn(0.0f);
    }
}

__global__ void to_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                               size_t n) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
         i += (size_t)gridDim.x * blockDim.x)
        dst[i] = __float2bfloat16_rn(src[i]);
}

void launch_to_bf16(const float* src, void* dst, size_t n, cudaStream_t st) {
    if (n == 0) return;
    unsigned b = cdiv((long long)n, 256);
    if (b > 148 * 8) b = 148 * 8;
    to_bf16_kernel<<<b, 256, 0, st>>>(src, static_cast<__nv_bfloat16*>(dst), n);
}

void launch_open_window(const WindowJob* d_jobs, int n_jobs, cudaStream_t st) {
    if (n_jobs == 0) return;
    dim3 grid(64, n_jobs);
    open_window_kernel<<<grid, 256, 0, st>>>(d_jobs);
}

}  // namespace zo
