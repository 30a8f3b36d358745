// Tensor-core GEMM for sm_100a: C = A B^T (+ A2 B2^T), bf16 in, fp32 accumulate.
//
// The batched forward of both candidates is the dominant cost of the probe
// step ("Zeroth-Order Fine-Tuning Was an Inference Workload All Along",
// section "Why ZO Fine-Tuning Is Really Scoring": the pair of forward
// objective evaluations is the expensive operation), so every decoder linear
// layer -- with the candidate perturbation and the banked updates appended as
// extra K blocks (A2 = the shrink output S, B2 = the expand factors) -- runs
// here, and the lm_head runs here with a log-sum-exp epilogue so logits never
// reach memory.
//
// Design (one CTA per SM, persistent):
//   warp 0      TMA producer: 128x64 A and Nx64 B boxes, 128-byte swizzle,
//               into a 192 KB shared-memory ring (mbarrier complete_tx)
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer
//               (M=128, N=64/128/256, K=16 per instruction, kind::f16, fp32 accumulate)
//   warps 2..5  epilogue: tcgen05.ld 32x32b from a double-buffered TMEM
//               accumulator, fused bias / ReLU / residual add / SwiGLU / LSE;
//               the SM-pair kernel hands its tiles to TMA stores (reduce-add for
//               the residual stream) through swizzled shared-memory staging
// Tiles are walked in M-groups (8 blocks single-SM, 12 for SM pairs) so concurrent CTAs
// share B strips in L2.
// Every mbarrier wait is bounded: on expiry the kernel records
// ZO_TC_TIMEOUT in the error word, drains what it issued and returns.
#include <cuda.h>
#include <float.h>

#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "kernels.h"

namespace zo {

ZO_DEBUG_WORD(debug_word_gemm)

namespace {

constexpr int BM = 128, BK = 64, BN = 256;
// lm_head log-sum-exp tiles: 128 vocabulary columns, so that the ~400 tiles of a 50k-151k
// vocabulary fill the SMs' waves evenly (256-column tiles left OPT's second wave a third full)
constexpr int BN_LSE = 128;
constexpr int BK8 = 128;                    // E4M3 K block: the same 128-byte rows
constexpr int A_BYTES = BM * BK * 2;        // 16 KB
constexpr int TMEM_COLS = 512;              // two BN-wide fp32 accumulators
constexpr int GROUP_M = 8;
constexpr int NUM_THREADS = 192;
constexpr uint32_t WAIT_LIMIT = 1u << 24;   // drain polls (with back-off) after an abort
constexpr long long WAIT_CYCLES = 4000000000ll;   // ~2 s at 2 GHz: a stage that never arrives
long long g_wait_cycles = WAIT_CYCLES;             // host copy handed to every launch

// Single-SM kernel geometry for an N tile of BNT columns (64, 128 or 256): the
// ring holds 192 KB whatever the width, so narrow GEMMs (the bank shrink, whose
// N is the handful of factor columns) keep as many bytes in flight per SM as the
// wide ones and do not spend tensor-core time on columns that do not exist.
template <int BNT>
struct Tile1 {
    static_assert(BNT == 32 || BNT == 64 || BNT == 128 || BNT == 256, "N tile");
    static constexpr int B_BYTES = BNT * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;        // multiple of 1024
    static constexpr int STAGES = (192 * 1024) / STAGE_BYTES;    // 9, 8, 6, 4
    static constexpr int TMEM_COLS = 2 * BNT;                    // double-buffered accumulator
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
    // bf16 x bf16 -> fp32, both K-major, M = 128, N = BNT
    static constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) |
                                      ((uint32_t)(BNT >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
    // kind::f8f6f4, A and B both E4M3 (format code 0), fp32 accumulate, M = 128, N = BNT
    static constexpr uint32_t IDESC_F8 = (1u << 4) | ((uint32_t)(BNT >> 3) << 17) |
                                         ((uint32_t)(BM >> 4) << 24);
    // barriers (8 B each: full, empty per stage; tfull, tempty per accumulator; drain)
    // then the TMEM base and the abort flag, all inside the 256-byte tail
    static constexpr int SLOT_OFF = 240, ABORT_OFF = 248;
    static_assert(8 * (2 * STAGES + 5) <= SLOT_OFF, "barrier region");
};

// Decode steps (a few dozen token rows): the operands are swapped, so the weight rows fill
// the 128-row MMA side and the tokens are the narrow N side, and each (128 weight rows, K
// split) item stores its raw fp32 accumulator transposed, as rows of tokens, into its slice
// of a [ks][tokens][features] workspace; the split reduction applies bias and the epilogue.
constexpr int EPI_SPLIT_T = 16;

__device__ int g_tc_error = 0;              // bit 0: a bounded wait expired
constexpr bool g_use_pairs = true;          // SM-pair kernel for large decoder GEMMs

struct TcParams {
    int M, N, kb_main, kb_ext;
    int n_m_blk, n_n_blk, n_tiles;
    int group_m;                            // M blocks per raster group
    int epi;
    const float* bias;
    void* C; int ldc; int c_type;
    const int* targets; float* part_max; float* part_sum; float* tgt_logit; int n_col_tiles;
    int* part_arg;
    const int* row_sign; float eps; int scale_cols;
    const int* tok_pos; const float* qn; const float* kn;
    const float* rope_cos; const float* rope_sin; float norm_eps;
    int n_q_heads, n_qk_heads;
    const float* a_scale; const float* b_scale;   // E4M3 dequantisation (F8 kernels)
    int ksplit, kbs;                        // split-K (SPLIT kernels): splits, main blocks each
    int* err;
    long long wait_cycles;                  // bound of every mbarrier wait (clock64 cycles)
};

// ---- PTX wrappers ------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// try_wait that suspends the thread for at most ~1 us (suspendTimeHint, in ns) when the
// phase is not complete, so a waiting thread looks at its clock regularly.
__device__ __forceinline__ bool mbar_try_bounded(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(1000u)
        : "memory");
    return ok != 0;
}
// Bounded wait; false when the limit expired or another role aborted.  No
// sleep between polls: try_wait already suspends the thread in hardware (until
// the phase completes, or ~1 us at most), and a software back-off would delay
// the hand-off of every stage.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_f,
                                          int* err, long long limit) {
    if (mbar_try(bar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try_bounded(bar, parity)) return true;
        if (*abort_f) return false;
        if (clock64() - t0 > limit) {
            *abort_f = 1;
            atomicOr(err, 1);
            return false;
        }
    }
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accum) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
        : "memory");
}
__device__ __forceinline__ void tc_mma_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accum) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
        : "memory");
}
// 32 lanes x 32 consecutive fp32 columns per warp.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 bytes in 8-row groups 1024 bytes apart (stride byte offset), version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);          // start address
    d |= (uint64_t)1u << 16;                           // leading byte offset (unused, 16 B)
    d |= (uint64_t)(1024u >> 4) << 32;                 // stride byte offset
    d |= (uint64_t)1u << 46;                           // descriptor version (sm_100)
    d |= (uint64_t)2u << 61;                           // SWIZZLE_128B
    return d;
}


__device__ __forceinline__ void tile_coords(int t, const TcParams& p, int* mb, int* nb) {
    const int per_group = GROUP_M * p.n_n_blk;
    const int g = t / per_group;
    const int first_m = g * GROUP_M;
    const int gm = min(p.n_m_blk - first_m, GROUP_M);
    const int in = t - g * per_group;
    *mb = first_m + in % gm;
    *nb = in / gm;
}

template <int EPI>
__device__ __forceinline__ void epilogue_chunk(const TcParams& p, int m, int n, float* v,
                                               float* run_max, float* run_sum, int* run_arg) {
    const bool row_ok = m < p.M;
    if (EPI == EPI_LSE) {
        float mx = -FLT_MAX;
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (n + j < p.N) mx = fmaxf(mx, v[j]);
        if (p.part_arg && mx > *run_max) {
            // the lowest column of this chunk that holds its maximum
            int a = n;
#pragma unroll
            for (int j = 31; j >= 0; --j)
                if (n + j < p.N && v[j] == mx) a = n + j;
            *run_arg = a;
        }
        const float nm = fmaxf(*run_max, mx);
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (n + j < p.N) s += expf(v[j] - nm);
        *run_sum = *run_sum * expf(*run_max - nm) + s;
        *run_max = nm;
        if (row_ok) {
            const int tg = p.targets[m] - n;
            if (tg >= 0 && tg < 32 && n + tg < p.N) {     // padding columns are no target
                float tv = 0.f;
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (j == tg) tv = v[j];
                p.tgt_logit[m] = tv;
            }
        }
        return;
    }
    if (!row_ok) return;
    if (p.bias) {
        if (n + 32 <= p.N) {
            const float4* b4 = reinterpret_cast<const float4*>(p.bias + n);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 b = __ldg(b4 + q);
                v[4 * q] += b.x; v[4 * q + 1] += b.y; v[4 * q + 2] += b.z; v[4 * q + 3] += b.w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (n + j < p.N) v[j] += p.bias[n + j];
        }
    }
    if (EPI == EPI_RESID) {
        float* C = static_cast<float*>(p.C) + (size_t)m * p.ldc + n;
        if (n + 32 <= p.N) {
            float4* c4 = reinterpret_cast<float4*>(C);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                float4 c = c4[q];
                c.x += v[4 * q]; c.y += v[4 * q + 1]; c.z += v[4 * q + 2]; c.w += v[4 * q + 3];
                c4[q] = c;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (n + j < p.N) C[j] += v[j];
        }
        return;
    }
    if (EPI == EPI_STORE_RELU) {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = fmaxf(v[j], 0.f);
    }
    if (EPI == EPI_SHRINK && n < p.scale_cols) {
        // direction columns carry the row's candidate sign times eps
        const float rs = (float)p.row_sign[m] * p.eps;
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (n + j < p.scale_cols) v[j] *= rs;
    }
    if (EPI == EPI_SHRINK && p.a_scale) {
        // the group's base GEMM runs in E4M3: its accumulator is in units of 1 / a_scale[m]
        const float sa = __ldg(p.a_scale + m);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = v[j] / sa;
    }
    if (p.c_type == E_BF16) {
        __nv_bfloat16* C = static_cast<__nv_bfloat16*>(p.C) + (size_t)m * p.ldc + n;
        if (n + 32 <= p.N) {
            uint4* c4 = reinterpret_cast<uint4*>(C);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint4 w;
                __nv_bfloat162 h0 = __floats2bfloat162_rn(v[8 * q], v[8 * q + 1]);
                __nv_bfloat162 h1 = __floats2bfloat162_rn(v[8 * q + 2], v[8 * q + 3]);
                __nv_bfloat162 h2 = __floats2bfloat162_rn(v[8 * q + 4], v[8 * q + 5]);
                __nv_bfloat162 h3 = __floats2bfloat162_rn(v[8 * q + 6], v[8 * q + 7]);
                w.x = *reinterpret_cast<uint32_t*>(&h0);
                w.y = *reinterpret_cast<uint32_t*>(&h1);
                w.z = *reinterpret_cast<uint32_t*>(&h2);
                w.w = *reinterpret_cast<uint32_t*>(&h3);
                c4[q] = w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (n + j < p.N) C[j] = __float2bfloat16_rn(v[j]);
        }
    } else {
        float* C = static_cast<float*>(p.C) + (size_t)m * p.ldc + n;
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (n + j < p.N) C[j] = v[j];
    }
}

// SwiGLU epilogue: the tile's columns 0..127 are gate features nb*128 + j and
// columns 128..255 the matching up features; out[m, f] = silu(gate) * up.
__device__ __forceinline__ void epilogue_swiglu(const TcParams& p, int m, int nb, uint32_t taddr) {
    const int F = p.N >> 1;
    for (int c = 0; c < 4; ++c) {
        const int f0 = nb * 128 + c * 32;
        if (f0 >= F) break;                         // warp-uniform
        float gv[32], uv[32];
        tmem_ld32(taddr + (uint32_t)(c * 32), gv);
        tmem_ld32(taddr + (uint32_t)(128 + c * 32), uv);
        if (m >= p.M) continue;
        if (p.bias) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                if (f0 + j < F) {
                    gv[j] += p.bias[nb * 256 + c * 32 + j];
                    uv[j] += p.bias[nb * 256 + 128 + c * 32 + j];
                }
            }
        }
        __nv_bfloat16* C = static_cast<__nv_bfloat16*>(p.C) + (size_t)m * p.ldc + f0;
        float y[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) y[j] = gv[j] / (1.0f + expf(-gv[j])) * uv[j];
        if (f0 + 32 <= F) {
            uint4* c4 = reinterpret_cast<uint4*>(C);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                __nv_bfloat162 h0 = __floats2bfloat162_rn(y[8 * q], y[8 * q + 1]);
                __nv_bfloat162 h1 = __floats2bfloat162_rn(y[8 * q + 2], y[8 * q + 3]);
                __nv_bfloat162 h2 = __floats2bfloat162_rn(y[8 * q + 4], y[8 * q + 5]);
                __nv_bfloat162 h3 = __floats2bfloat162_rn(y[8 * q + 6], y[8 * q + 7]);
                uint4 w;
                w.x = *reinterpret_cast<uint32_t*>(&h0);
                w.y = *reinterpret_cast<uint32_t*>(&h1);
                w.z = *reinterpret_cast<uint32_t*>(&h2);
                w.w = *reinterpret_cast<uint32_t*>(&h3);
                c4[q] = w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (f0 + j < F) C[j] = __float2bfloat16_rn(y[j]);
        }
    }
}

// F8 (EPI_SPLIT_T only): the main K blocks are E4M3 (kind::f8f6f4, 128 elements per block),
// the extension blocks bf16, into the same accumulator; the epilogue dequantises.
template <int EPI, int BNT, bool F8 = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                   const TcParams p) {
    using T1 = Tile1<BNT>;
    constexpr int STAGES = T1::STAGES;
    constexpr int STAGE_BYTES = T1::STAGE_BYTES;
    if (EPI == EPI_SPLIT_T) {
        // launched as a dependent of the kernel that wrote its operands; its split reduction
        // is launched as a dependent of this one
        grid_dep_wait();
        grid_dep_launch();
    }
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;           // 1024-aligned for SW128
    uint8_t* gbase = smem_raw + (base - raw);
    const uint32_t bar0 = base + STAGES * STAGE_BYTES;
    // barriers: full[S] empty[S] tfull[2] tempty[2] drain
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (STAGES + s); };
    auto tfull = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
    auto tempty = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 + b); };
    const uint32_t drain = bar0 + 8u * (2 * STAGES + 4);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + STAGES * STAGE_BYTES + T1::SLOT_OFF);
    volatile int* abort_f = reinterpret_cast<volatile int*>(gbase + STAGES * STAGE_BYTES + T1::ABORT_OFF);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull(b), 1);
            mbar_init(tempty(b), 4);
        }
        mbar_init(drain, 1);
        *abort_f = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(T1::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // work items: tiles, or (tile, K split) pairs for EPI_SPLIT_T; a split takes kbs main K
    // blocks and the last split also the extension blocks
    constexpr bool SPLIT = EPI == EPI_SPLIT_T;
    const int ks = SPLIT ? p.ksplit : 1;
    const int n_items = p.n_tiles * ks;
    auto item_blocks = [&](int sp, int* kb0, int* n_main, int* n_kb) {
        if (!SPLIT) {
            *kb0 = 0;
            *n_main = p.kb_main;
            *n_kb = p.kb_main + p.kb_ext;
            return;
        }
        *kb0 = sp * p.kbs;
        *n_main = max(0, min(p.kbs, p.kb_main - *kb0));
        *n_kb = *n_main + (sp == ks - 1 ? p.kb_ext : 0);
    };

    int n_armed = 0;                        // producer: loads issued; the i-th used stage i % S,
                                            // phase (i / S) & 1
    bool issued = false;                    // MMA issuer: any MMA issued
    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < n_items && ok; t += gridDim.x) {
                int mb, nb;
                tile_coords(t / ks, p, &mb, &nb);
                int kb0, n_main, n_kb;
                item_blocks(t % ks, &kb0, &n_main, &n_kb);
                for (int i = 0; i < n_kb; ++i) {
                    const int kb = i < n_main ? kb0 + i : p.kb_main + (i - n_main);
                    if (!mbar_wait(empty(s), ph ^ 1u, abort_f, p.err, p.wait_cycles)) { ok = false; break; }
                    const uint32_t sa = base + s * STAGE_BYTES;
                    const uint32_t sb = sa + A_BYTES;
                    mbar_expect_tx(full(s), STAGE_BYTES);
                    if (kb < p.kb_main) {
                        tma_load_2d(sa, &tmA, full(s), kb * (F8 ? BK8 : BK), mb * BM);
                        tma_load_2d(sb, &tmB, full(s), kb * (F8 ? BK8 : BK), nb * BNT);
                    } else {
                        const int k = (kb - p.kb_main) * BK;
                        tma_load_2d(sa, &tmA2, full(s), k, mb * BM);
                        tma_load_2d(sb, &tmB2, full(s), k, nb * BNT);
                    }
                    ++n_armed;
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            int acc = 0;
            uint32_t aph = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < n_items && ok; t += gridDim.x) {
                if (!mbar_wait(tempty(acc), aph ^ 1u, abort_f, p.err, p.wait_cycles)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(acc * BNT);
                int kb0, n_main, n_kb;
                item_blocks(t % ks, &kb0, &n_main, &n_kb);
                for (int i = 0; i < n_kb; ++i) {
                    if (!mbar_wait(full(s), ph, abort_f, p.err, p.wait_cycles)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = base + s * STAGE_BYTES;
                    const uint32_t sb = sa + A_BYTES;
                    if (F8 && i < n_main) {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)   // K = 32 E4M3 elements = 32 bytes each
                            tc_mma_f8(d, sw128_desc(sa + kk * 32), sw128_desc(sb + kk * 32),
                                      T1::IDESC_F8, (i > 0 || kk > 0) ? 1u : 0u);
                    } else {
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk) {
                            tc_mma(d, sw128_desc(sa + kk * 32), sw128_desc(sb + kk * 32), T1::IDESC,
                                   (i > 0 || kk > 0) ? 1u : 0u);
                        }
                    }
                    issued = true;
                    tc_commit(empty(s));            // stage free once these MMAs retire
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
                tc_commit(tfull(acc));              // accumulator ready for the epilogue
                if (++acc == 2) { acc = 0; aph ^= 1u; }
            }
        }
    } else {
        // ---------------- epilogue (warps 2..5) ----------------
        const int lane_base = 32 * (warp & 3);
        int acc = 0;
        uint32_t aph = 0;
        for (int t = blockIdx.x; t < n_items; t += gridDim.x) {
            int mb, nb;
            tile_coords(t / ks, p, &mb, &nb);
            if (!mbar_wait(tfull(acc), aph, abort_f, p.err, p.wait_cycles)) break;
            tc_fence_after();
            const int m = mb * BM + lane_base + lane;
            float run_max = -FLT_MAX, run_sum = 0.f;
            int run_arg = nb * BNT;
            if (EPI == EPI_SPLIT_T) {
                // lane = feature m, columns = tokens: for each token the warp's 32 lanes
                // write 32 consecutive features
                float* slice = static_cast<float*>(p.C) + (size_t)(t % ks) * p.N * p.M;
                for (int c = 0; c < BNT / 32; ++c) {
                    const int n = nb * BNT + c * 32;
                    if (n >= p.N) break;            // warp-uniform
                    float v[32];
                    tmem_ld32(tmem + ((uint32_t)lane_base << 16) + (uint32_t)(acc * BNT + c * 32), v);
                    if (m < p.M) {
                        if (F8) {
                            // E4M3 units back to real ones: times the token's scale (N side),
                            // then the weight row's (M side), the order the SM-pair kernel uses
                            const float sw = __ldg(p.a_scale + m);
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                if (n + j < p.N) v[j] = v[j] * __ldg(p.b_scale + n + j) * sw;
                        }
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (n + j < p.N) slice[(size_t)(n + j) * p.M + m] = v[j];
                    }
                }
            } else if (EPI == EPI_SWIGLU)
                epilogue_swiglu(p, m, nb, tmem + ((uint32_t)lane_base << 16) + (uint32_t)(acc * BNT));
            else
            for (int c = 0; c < BNT / 32; ++c) {
                const int n = nb * BNT + c * 32;
                if (n >= p.N) break;                // whole chunk past N (warp-uniform)
                float v[32];
                tmem_ld32(tmem + ((uint32_t)lane_base << 16) + (uint32_t)(acc * BNT + c * 32), v);
                epilogue_chunk<EPI>(p, m, n, v, &run_max, &run_sum, &run_arg);
            }
            if (EPI == EPI_LSE && m < p.M) {
                p.part_max[(size_t)m * p.n_col_tiles + nb] = run_max;
                p.part_sum[(size_t)m * p.n_col_tiles + nb] = run_sum;
                if (p.part_arg) p.part_arg[(size_t)m * p.n_col_tiles + nb] = run_arg;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty(acc));
            if (++acc == 2) { acc = 0; aph ^= 1u; }
        }
    }

    tc_fence_before();
    __syncthreads();                        // every role has left its loop
    if (*abort_f && lane == 0) {
        // an aborted CTA lets what it issued finish before its shared and tensor memory go
        // away, whichever role gave up: the newest copies (older ones were consumed, so had
        // landed), then every MMA
        if (warp == 0) {
            const int n = n_armed < STAGES ? n_armed : STAGES;
            for (int i = 0; i < n; ++i) {
                const int a = n_armed - 1 - i;
                const uint32_t aph = (uint32_t)(a / STAGES) & 1u;
                for (uint32_t it = 0; it < WAIT_LIMIT && !mbar_try(full(a % STAGES), aph); ++it)
                    __nanosleep(128);
            }
        } else if (warp == 1 && issued) {
            tc_commit(drain);
            for (uint32_t it = 0; it < WAIT_LIMIT && !mbar_try(drain, 0); ++it) __nanosleep(128);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(T1::TMEM_COLS)
                     : "memory");
    }
}

// ---- 2-SM variant ----------------------------------------------------------------
// A CTA pair (cluster of 2) computes one 256 x 256 tile: each CTA loads its
// own 128 rows of A and its own 128 rows (half the N extent) of B, the even
// CTA issues tcgen05.mma.cta_group::2 (M = 256) over both CTAs' shared
// memory, and each CTA's TMEM receives its own 128 accumulator rows.  Per SM
// this moves a third less operand data per FLOP than the 1-SM tile, so six
// stages fit and the ring hides longer L2 latencies.  Loads carry no
// multicast: every CTA fetches its own tiles.
constexpr int BM2 = 256, STAGES2 = 6;
constexpr int A2B = 128 * BK * 2;                // 16 KB of A per CTA per stage
constexpr int B2B = 128 * BK * 2;                // 16 KB of B per CTA per stage
constexpr int STAGE2_BYTES = A2B + B2B;
// epilogue staging: 4 warps x 2 buffers x 4 KB (32 rows x 128 bytes, 128-byte swizzle)
constexpr int STG_BYTES = 4 * 2 * 4096;
constexpr int SMEM2_BYTES = STAGES2 * STAGE2_BYTES + STG_BYTES + 1024 + 256;
constexpr uint32_t kIdesc2 = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                             ((uint32_t)(BM2 >> 4) << 24);
// kind::f8f6f4, A and B both E4M3 (format code 0), fp32 accumulate, M = 256, N = 256.  A
// stage holds the same 128-byte rows, so 128 K elements instead of 64 and each of the
// four MMAs per stage covers K = 32.
constexpr uint32_t kIdesc2F8 = (1u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM2 >> 4) << 24);

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// shared::cluster address of the same offset in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_rank(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t leader_bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(leader_bar), "r"(x), "r"(y)
        : "memory");
}
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
    // arrive on the barrier at this offset in both CTAs of the pair
    asm volatile(
        "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], m;\n\t}" ::"r"(bar)
        : "memory");
}
__device__ __forceinline__ void tc_mma_pair_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accum) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
        : "memory");
}
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accum) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
        : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar)
                 : "memory");
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(src), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int x, int y,
                                             int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(src), "r"(x), "r"(y), "r"(z)
        : "memory");
}
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
    asm volatile(
        "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(src), "r"(x), "r"(y)
        : "memory");
}
__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read1() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read0() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// 16-byte chunk k (0..7) of staging row r (0..31): 128-byte rows, 128-byte swizzle
__device__ __forceinline__ uint32_t stg_off(int r, int k) {
    return (uint32_t)(r * 128 + ((k ^ (r & 7)) << 4));
}
__device__ __forceinline__ uint32_t pack2_bf16(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

// E4M3 accumulators back to real units: v[j] *= a_scale[m] * b_scale[n + j].
template <int W>
__device__ __forceinline__ void dequant_chunk(const TcParams& p, int m, int n, float* v) {
    const float sa = m < p.M ? __ldg(p.a_scale + m) : 0.f;
    if (n + W <= p.N) {                     // n is a multiple of 32: 16-byte aligned scales
        const float4* b4 = reinterpret_cast<const float4*>(p.b_scale + n);
#pragma unroll
        for (int q = 0; q < W / 4; ++q) {
            const float4 sb = __ldg(b4 + q);
            v[4 * q] = v[4 * q] * sa * sb.x;
            v[4 * q + 1] = v[4 * q + 1] * sa * sb.y;
            v[4 * q + 2] = v[4 * q + 2] * sa * sb.z;
            v[4 * q + 3] = v[4 * q + 3] * sa * sb.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < W; ++j)
            v[j] = v[j] * sa * ((n + j < p.N) ? __ldg(p.b_scale + n + j) : 0.f);
    }
}

// Pair-kernel epilogue: each warp stages its 32 rows x (32 fp32 | 64 bf16) columns in
// shared memory and one lane hands them to the TMA unit -- a store, or for the
// residual stream an fp32 reduce-add, so the SM never reads the residual.  Two
// staging buffers per warp alternate; a buffer is rewritten only after the TMA
// has read it.
template <int EPI, bool F8, bool SPLIT>
__device__ __forceinline__ void epilogue_tma(const TcParams& p, const CUtensorMap* tmC,
                                             uint32_t stg, uint8_t* stg_ptr, int& buf, int m_base,
                                             int nb, uint32_t taddr, int lane, int split) {
    const int r = lane;
    auto stage_begin = [&]() {
        if (lane == 0) bulk_wait_read1();
        __syncwarp();
    };
    auto stage_end_store = [&](int x, bool reduce) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
            if (reduce) tma_reduce_add_2d(tmC, stg + buf * 4096, x, m_base);
            else tma_store_2d(tmC, stg + buf * 4096, x, m_base);
            bulk_commit();
        }
        buf ^= 1;
    };
    if (SPLIT) {
        // one K split's raw fp32 accumulator into its slice of the workspace; the split
        // reduction applies bias and the epilogue afterwards, summing the slices in order
        for (int c = 0; c < BN / 32; ++c) {
            const int n = nb * BN + c * 32;
            if (n >= p.N) break;
            float v[32];
            tmem_ld32(taddr + (uint32_t)(c * 32), v);
            stage_begin();
            uint8_t* b = stg_ptr + buf * 4096;
#pragma unroll
            for (int k = 0; k < 8; ++k)
                *reinterpret_cast<float4*>(b + stg_off(r, k)) =
                    make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) {
                tma_store_3d(tmC, stg + buf * 4096, n, m_base, split);
                bulk_commit();
            }
            buf ^= 1;
        }
    } else if (EPI == EPI_RESID) {
        for (int c = 0; c < BN / 32; ++c) {
            const int n = nb * BN + c * 32;
            if (n >= p.N) break;
            float v[32];
            tmem_ld32(taddr + (uint32_t)(c * 32), v);
            if (p.bias) {
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] += (n + j < p.N) ? __ldg(p.bias + n + j) : 0.f;
            }
            stage_begin();
            uint8_t* b = stg_ptr + buf * 4096;
#pragma unroll
            for (int k = 0; k < 8; ++k)
                *reinterpret_cast<float4*>(b + stg_off(r, k)) =
                    make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
            stage_end_store(n, true);
        }
    } else if (EPI == EPI_SWIGLU) {
        const int F = p.N >> 1;
        for (int c = 0; c < 4; c += 2) {
            const int f0 = nb * 128 + c * 32;
            if (f0 >= F) break;
            float y[64];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float gv[32], uv[32];
                tmem_ld32(taddr + (uint32_t)((c + h) * 32), gv);
                tmem_ld32(taddr + (uint32_t)(128 + (c + h) * 32), uv);
                if (F8) {
                    dequant_chunk<32>(p, m_base + r, nb * 256 + (c + h) * 32, gv);
                    dequant_chunk<32>(p, m_base + r, nb * 256 + 128 + (c + h) * 32, uv);
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    float g = gv[j], u = uv[j];
                    if (p.bias) {
                        g += __ldg(p.bias + nb * 256 + (c + h) * 32 + j);
                        u += __ldg(p.bias + nb * 256 + 128 + (c + h) * 32 + j);
                    }
                    y[h * 32 + j] = g / (1.0f + expf(-g)) * u;
                }
            }
            stage_begin();
            uint8_t* b = stg_ptr + buf * 4096;
#pragma unroll
            for (int k = 0; k < 8; ++k)
                *reinterpret_cast<uint4*>(b + stg_off(r, k)) =
                    make_uint4(pack2_bf16(y[8 * k], y[8 * k + 1]), pack2_bf16(y[8 * k + 2], y[8 * k + 3]),
                               pack2_bf16(y[8 * k + 4], y[8 * k + 5]), pack2_bf16(y[8 * k + 6], y[8 * k + 7]));
            stage_end_store(f0, false);
        }
    } else if (EPI == EPI_QKNR) {
        // one 128-column head at a time.  The accumulator is rounded to bf16 (the value the
        // unfused path stores); q and k heads then get RMSNorm over the head and the rotary
        // rotation of the pairs (i, i + 64) at the token's position.  Columns 32c.. and
        // 64 + 32c.. are handled together, so a head goes out through both staging buffers.
        const int m = m_base + r;
        const int pos = m < p.M ? __ldg(p.tok_pos + m) : 0;
        for (int hb = 0; hb < 2; ++hb) {
            const int n0 = nb * BN + hb * 128;
            if (n0 >= p.N) break;                  // warp-uniform
            const int head = n0 >> 7;
            const bool qk = head < p.n_qk_heads;
            const uint32_t th = taddr + (uint32_t)(hb * 128);
            float rs = 1.f;
            if (qk) {
                float ss = 0.f;
                for (int c = 0; c < 4; ++c) {
                    float v[32];
                    tmem_ld32(th + (uint32_t)(c * 32), v);
                    if (F8) dequant_chunk<32>(p, m, n0 + c * 32, v);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float x = __bfloat162float(__float2bfloat16_rn(v[j]));
                        ss += x * x;
                    }
                }
                rs = 1.0f / sqrtf(ss / 128.0f + p.norm_eps);
            }
            const float* w = head < p.n_q_heads ? p.qn : p.kn;
            if (lane == 0) bulk_wait_read0();      // both staging buffers free
            __syncwarp();
            for (int c = 0; c < 2; ++c) {
                float lo[32], hi[32];
                tmem_ld32(th + (uint32_t)(c * 32), lo);
                tmem_ld32(th + (uint32_t)(64 + c * 32), hi);
                if (F8) {
                    dequant_chunk<32>(p, m, n0 + c * 32, lo);
                    dequant_chunk<32>(p, m, n0 + 64 + c * 32, hi);
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    lo[j] = __bfloat162float(__float2bfloat16_rn(lo[j]));
                    hi[j] = __bfloat162float(__float2bfloat16_rn(hi[j]));
                }
                if (qk) {
                    const float4* wl = reinterpret_cast<const float4*>(w + 32 * c);
                    const float4* wh = reinterpret_cast<const float4*>(w + 64 + 32 * c);
                    const float4* c4 = reinterpret_cast<const float4*>(p.rope_cos + (size_t)pos * 64 + 32 * c);
                    const float4* s4 = reinterpret_cast<const float4*>(p.rope_sin + (size_t)pos * 64 + 32 * c);
#pragma unroll
                    for (int j4 = 0; j4 < 8; ++j4) {
                        const float4 a4 = __ldg(wl + j4), b4 = __ldg(wh + j4);
                        const float4 cv = __ldg(c4 + j4), sv = __ldg(s4 + j4);
                        const float wa[4] = {a4.x, a4.y, a4.z, a4.w};
                        const float wb[4] = {b4.x, b4.y, b4.z, b4.w};
                        const float cs[4] = {cv.x, cv.y, cv.z, cv.w};
                        const float sn[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int j = 4 * j4 + e;
                            const float a = lo[j] * rs * wa[e], b = hi[j] * rs * wb[e];
                            lo[j] = a * cs[e] - b * sn[e];
                            hi[j] = b * cs[e] + a * sn[e];
                        }
                    }
                }
                uint8_t* b0 = stg_ptr;
                uint8_t* b1 = stg_ptr + 4096;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    *reinterpret_cast<uint4*>(b0 + stg_off(r, 4 * c + k)) =
                        make_uint4(pack2_bf16(lo[8 * k], lo[8 * k + 1]), pack2_bf16(lo[8 * k + 2], lo[8 * k + 3]),
                                   pack2_bf16(lo[8 * k + 4], lo[8 * k + 5]), pack2_bf16(lo[8 * k + 6], lo[8 * k + 7]));
                    *reinterpret_cast<uint4*>(b1 + stg_off(r, 4 * c + k)) =
                        make_uint4(pack2_bf16(hi[8 * k], hi[8 * k + 1]), pack2_bf16(hi[8 * k + 2], hi[8 * k + 3]),
                                   pack2_bf16(hi[8 * k + 4], hi[8 * k + 5]), pack2_bf16(hi[8 * k + 6], hi[8 * k + 7]));
                }
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) {
                tma_store_2d(tmC, stg, n0, m_base);
                tma_store_2d(tmC, stg + 4096, n0 + 64, m_base);
                bulk_commit();
            }
        }
    } else {   // EPI_STORE, EPI_STORE_RELU: bf16, 64 columns per store
        for (int c = 0; c < BN / 32; c += 2) {
            const int n = nb * BN + c * 32;
            if (n >= p.N) break;
            float y[64];
            tmem_ld32(taddr + (uint32_t)(c * 32), y);
            tmem_ld32(taddr + (uint32_t)((c + 1) * 32), y + 32);
            if (F8) dequant_chunk<64>(p, m_base + r, n, y);
#pragma unroll
            for (int j = 0; j < 64; ++j) {
                float v = y[j];
                if (p.bias) v += (n + j < p.N) ? __ldg(p.bias + n + j) : 0.f;
                if (EPI == EPI_STORE_RELU) v = fmaxf(v, 0.f);
                y[j] = v;
            }
            stage_begin();
            uint8_t* b = stg_ptr + buf * 4096;
#pragma unroll
            for (int k = 0; k < 8; ++k)
                *reinterpret_cast<uint4*>(b + stg_off(r, k)) =
                    make_uint4(pack2_bf16(y[8 * k], y[8 * k + 1]), pack2_bf16(y[8 * k + 2], y[8 * k + 3]),
                               pack2_bf16(y[8 * k + 4], y[8 * k + 5]), pack2_bf16(y[8 * k + 6], y[8 * k + 7]));
            stage_end_store(n, false);
        }
    }
}

__device__ __forceinline__ void tile_coords2(int t, const TcParams& p, int* mb, int* nb) {
    const int per_group = p.group_m * p.n_n_blk;
    const int g = t / per_group;
    const int first_m = g * p.group_m;
    const int gm = min(p.n_m_blk - first_m, p.group_m);
    const int in = t - g * per_group;
    *mb = first_m + in % gm;
    *nb = in / gm;
}

// F8: the main K blocks are E4M3 (kind::f8f6f4) and the epilogue dequantises; a separate
// instantiation, so the bf16 kernels carry none of it.
template <int EPI, bool F8, bool SPLIT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmA2,
                    const __grid_constant__ CUtensorMap tmB2,
                    const __grid_constant__ CUtensorMap tmC, const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;     // same offset in both CTAs
    uint8_t* gbase = smem_raw + (base - raw);
    const uint32_t stg0 = base + STAGES2 * STAGE2_BYTES;          // epilogue staging (1024-aligned)
    const uint32_t bar0 = stg0 + STG_BYTES;
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (STAGES2 + s); };
    auto tfull = [&](int b) { return bar0 + 8u * (2 * STAGES2 + b); };
    auto tempty = [&](int b) { return bar0 + 8u * (2 * STAGES2 + 2 + b); };
    const uint32_t drain = bar0 + 8u * (2 * STAGES2 + 4);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + STAGES2 * STAGE2_BYTES + STG_BYTES + 160);
    volatile int* abort_f =
        reinterpret_cast<volatile int*>(gbase + STAGES2 * STAGE2_BYTES + STG_BYTES + 168);

    const uint32_t rank = cluster_rank();
    const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES2; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull(b), 1);
            mbar_init(tempty(b), 8);        // 4 epilogue warps in each CTA of the pair
        }
        mbar_init(drain, 1);
        *abort_f = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();                         // both CTAs' barriers exist before any remote use
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // work items: tiles, or (tile, K split) pairs; a split takes kbs main K blocks and the
    // last split also the extension blocks
    const int n_items = SPLIT ? p.n_tiles * p.ksplit : p.n_tiles;
    auto item_blocks = [&](int sp, int* kb0, int* n_main, int* n_kb) {
        if (!SPLIT) {
            *kb0 = 0;
            *n_main = p.kb_main;
            *n_kb = p.kb_main + p.kb_ext;
            return;
        }
        *kb0 = sp * p.kbs;
        *n_main = max(0, min(p.kbs, p.kb_main - *kb0));
        *n_kb = *n_main + (sp == p.ksplit - 1 ? p.kb_ext : 0);
    };

    int n_armed = 0;                        // producer: loads issued; the i-th used stage i % S,
                                            // phase (i / S) & 1
    bool issued = false;                    // MMA issuer (even CTA): any MMA issued
    if (warp == 0) {
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int t = pair; t < n_items && ok; t += n_pairs) {
                int mb, nb;
                tile_coords2(SPLIT ? t / p.ksplit : t, p, &mb, &nb);
                const int row_a = mb * BM2 + (int)rank * 128;
                const int row_b = nb * BN + (int)rank * 128;
                int kb0, n_main, n_kb;
                item_blocks(SPLIT ? t % p.ksplit : 0, &kb0, &n_main, &n_kb);
                for (int i = 0; i < n_kb; ++i) {
                    const int kb = i < n_main ? kb0 + i : p.kb_main + (i - n_main);
                    if (!mbar_wait(empty(s), ph ^ 1u, abort_f, p.err, p.wait_cycles)) { ok = false; break; }
                    const uint32_t sa = base + s * STAGE2_BYTES;
                    const uint32_t sb = sa + A2B;
                    // the even CTA expects both CTAs' bytes on its barrier
                    if (rank == 0) mbar_expect_tx(full(s), 2 * STAGE2_BYTES);
                    const uint32_t lb = map_rank(full(s), 0);
                    if (kb < p.kb_main) {
                        const int k = kb * (F8 ? BK8 : BK);
                        tma_load_2d_pair(sa, &tmA, lb, k, row_a);
                        tma_load_2d_pair(sb, &tmB, lb, k, row_b);
                    } else {
                        const int k = (kb - p.kb_main) * BK;
                        tma_load_2d_pair(sa, &tmA2, lb, k, row_a);
                        tma_load_2d_pair(sb, &tmB2, lb, k, row_b);
                    }
                    ++n_armed;
                    if (++s == STAGES2) { s = 0; ph ^= 1u; }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            int s = 0;
            uint32_t ph = 0;
            int acc = 0;
            uint32_t aph = 0;
            bool ok = true;
            for (int t = pair; t < n_items && ok; t += n_pairs) {
                if (!mbar_wait(tempty(acc), aph ^ 1u, abort_f, p.err, p.wait_cycles)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(acc * BN);
                int kb0, n_main, n_kb;
                item_blocks(SPLIT ? t % p.ksplit : 0, &kb0, &n_main, &n_kb);
                for (int i = 0; i < n_kb; ++i) {
                    const int kb = i < n_main ? kb0 + i : p.kb_main + (i - n_main);
                    if (!mbar_wait(full(s), ph, abort_f, p.err, p.wait_cycles)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = base + s * STAGE2_BYTES;
                    const uint32_t sb = sa + A2B;
                    if (F8 && kb < p.kb_main) {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            tc_mma_pair_f8(d, sw128_desc(sa + kk * 32), sw128_desc(sb + kk * 32),
                                           kIdesc2F8, (i > 0 || kk > 0) ? 1u : 0u);
                    } else {
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            tc_mma_pair(d, sw128_desc(sa + kk * 32), sw128_desc(sb + kk * 32),
                                        kIdesc2, (i > 0 || kk > 0) ? 1u : 0u);
                    }
                    issued = true;
                    tc_commit_pair(empty(s));       // stage free in both CTAs
                    if (++s == STAGES2) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
                tc_commit_pair(tfull(acc));         // both halves of the accumulator ready
                if (++acc == 2) { acc = 0; aph ^= 1u; }
            }
        }
    } else {
        const int lane_base = 32 * (warp & 3);
        const uint32_t leader_tempty0 = map_rank(tempty(0), 0);
        const uint32_t leader_tempty1 = map_rank(tempty(1), 0);
        const int ew = warp & 3;
        const uint32_t stg = stg0 + (uint32_t)ew * 8192u;
        uint8_t* stg_ptr = gbase + STAGES2 * STAGE2_BYTES + ew * 8192;
        int buf = 0;
        int acc = 0;
        uint32_t aph = 0;
        for (int t = pair; t < n_items; t += n_pairs) {
            int mb, nb;
            tile_coords2(SPLIT ? t / p.ksplit : t, p, &mb, &nb);
            if (!mbar_wait(tfull(acc), aph, abort_f, p.err, p.wait_cycles)) break;
            tc_fence_after();
            const int m_base = mb * BM2 + (int)rank * 128 + lane_base;
            epilogue_tma<EPI, F8, SPLIT>(p, &tmC, stg, stg_ptr, buf, m_base, nb,
                                         tmem + ((uint32_t)lane_base << 16) + (uint32_t)(acc * BN),
                                         lane, SPLIT ? t % p.ksplit : 0);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc ? leader_tempty1 : leader_tempty0);
            if (++acc == 2) { acc = 0; aph ^= 1u; }
        }
        if (lane == 0) bulk_wait_all();    // every store of this warp has landed
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();                        // every role of this CTA has left its loop
    if (*abort_f && lane == 0 && rank == 0) {
        // an aborted pair lets what it issued finish first, whichever role gave up: both
        // CTAs' copies complete on the even CTA's barriers, and its thread issued the MMAs
        if (warp == 0) {
            const int n = n_armed < STAGES2 ? n_armed : STAGES2;
            for (int i = 0; i < n; ++i) {
                const int a = n_armed - 1 - i;
                const uint32_t aph = (uint32_t)(a / STAGES2) & 1u;
                for (uint32_t it = 0; it < WAIT_LIMIT && !mbar_try(full(a % STAGES2), aph); ++it)
                    __nanosleep(128);
            }
        } else if (warp == 1 && issued) {
            asm volatile(
                "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                    drain)
                : "memory");
            for (uint32_t it = 0; it < WAIT_LIMIT && !mbar_try(drain, 0); ++it) __nanosleep(128);
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();                         // neither CTA leaves while the pair may touch it
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(TMEM_COLS)
                     : "memory");
    }
}

// ---- bank shrink with K split over a CTA pair ---------------------------------------
// The shrink S = x FT^T has M = the batch's token rows and N = the bank's few columns, so it
// has one 128-row tile per 128 tokens (72 for 9196 rows: half the SMs) and is bound by
// reading x once.  A cluster of two CTAs computes each tile: each streams its half of K
// into its own TMEM accumulator, the odd CTA hands its fp32 half to the even CTA through
// distributed shared memory, and the even CTA adds the halves and applies the shrink
// epilogue.  The split is the same for every M, so a row's bits never depend on the batch.
template <int BNT>
struct TileS {
    static_assert(BNT == 32 || BNT == 64 || BNT == 128, "shrink N tile");
    static constexpr int B_BYTES = BNT * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;        // multiple of 1024
    // as many stages as fit beside the partial-sum buffer: each CTA's streaming rate is set
    // by the bytes of x it keeps in flight
    static constexpr int STAGES = BNT == 32 ? 10 : BNT == 64 ? 7 : 4;
    static constexpr int PART_LD = BNT + 4;                      // padded rows: no bank clash
    static constexpr int PART_BYTES = BM * PART_LD * 4;          // the odd CTA's accumulator
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + PART_BYTES + 1024 + 256;
    static constexpr uint32_t IDESC = Tile1<BNT>::IDESC;
    // barriers: full, empty per stage; tfull, tempty, part_full, part_free, drain
    static constexpr int SLOT_OFF = 200, ABORT_OFF = 208;
    static_assert(8 * (2 * STAGES + 5) <= SLOT_OFF, "barrier region");
};

__device__ __forceinline__ bool mbar_try_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(1000u)
        : "memory");
    return ok != 0;
}
// Bounded wait for an arrival from the other CTA of the pair (acquire at cluster scope,
// so the stores it released are visible).
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity,
                                                  volatile int* abort_f, int* err,
                                                  long long limit) {
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try_cluster(bar, parity)) return true;
        if (*abort_f) return false;
        if (clock64() - t0 > limit) {
            *abort_f = 1;
            atomicOr(err, 1);
            return false;
        }
    }
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, float a, float b, float c, float d) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b),
                 "f"(c), "f"(d)
                 : "memory");
}

template <int BNT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    shrink_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB, const TcParams p) {
    using TS = TileS<BNT>;
    constexpr int STAGES = TS::STAGES;
    constexpr int STAGE_BYTES = TS::STAGE_BYTES;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;           // same offset in both CTAs
    uint8_t* gbase = smem_raw + (base - raw);
    const uint32_t part0 = base + STAGES * STAGE_BYTES;
    float* part = reinterpret_cast<float*>(gbase + STAGES * STAGE_BYTES);
    const uint32_t bar0 = part0 + TS::PART_BYTES;
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (STAGES + s); };
    const uint32_t tfull = bar0 + 8u * (2 * STAGES);
    const uint32_t tempty = bar0 + 8u * (2 * STAGES + 1);
    const uint32_t part_full = bar0 + 8u * (2 * STAGES + 2);   // even CTA: the odd half landed
    const uint32_t part_free = bar0 + 8u * (2 * STAGES + 3);   // odd CTA: the even one read it
    const uint32_t drain = bar0 + 8u * (2 * STAGES + 4);
    uint8_t* tail = gbase + STAGES * STAGE_BYTES + TS::PART_BYTES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tail + TS::SLOT_OFF);
    volatile int* abort_f = reinterpret_cast<volatile int*>(tail + TS::ABORT_OFF);

    const uint32_t rank = cluster_rank();
    const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // K blocks of this CTA: the even CTA the first half, the odd one the rest
    const int half = (p.kb_main + 1) / 2;
    const int kb0 = rank == 0 ? 0 : half;
    const int n_kb = rank == 0 ? half : p.kb_main - half;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        mbar_init(tfull, 1);
        mbar_init(tempty, 4);
        mbar_init(part_full, 4);            // one arrival per epilogue warp of the odd CTA
        mbar_init(part_free, 4);            // one per epilogue warp of the even CTA
        mbar_init(drain, 1);
        *abort_f = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(BNT)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();                          // both CTAs' barriers exist before any remote arrive
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    int n_armed = 0;                         // producer: loads issued
    bool issued = false;                     // MMA issuer: any MMA issued
    if (warp == 0) {
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int t = pair; t < p.n_tiles && ok; t += n_pairs) {
                for (int i = 0; i < n_kb; ++i) {
                    if (!mbar_wait(empty(s), ph ^ 1u, abort_f, p.err, p.wait_cycles)) { ok = false; break; }
                    const uint32_t sa = base + s * STAGE_BYTES;
                    mbar_expect_tx(full(s), STAGE_BYTES);
                    tma_load_2d(sa, &tmA, full(s), (kb0 + i) * BK, t * BM);
                    tma_load_2d(sa + A_BYTES, &tmB, full(s), (kb0 + i) * BK, 0);
                    ++n_armed;
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0, tph = 0;
            bool ok = true;
            for (int t = pair; t < p.n_tiles && ok; t += n_pairs) {
                if (!mbar_wait(tempty, tph ^ 1u, abort_f, p.err, p.wait_cycles)) break;
                tc_fence_after();
                for (int i = 0; i < n_kb; ++i) {
                    if (!mbar_wait(full(s), ph, abort_f, p.err, p.wait_cycles)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = base + s * STAGE_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        tc_mma(tmem, sw128_desc(sa + kk * 32), sw128_desc(sa + A_BYTES + kk * 32),
                               TS::IDESC, (i > 0 || kk > 0) ? 1u : 0u);
                    issued = true;
                    tc_commit(empty(s));
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
                tc_commit(tfull);
                tph ^= 1u;
            }
        }
    } else {
        // epilogue: thread = accumulator row (TMEM lane), 32-column chunks
        const int lane_base = 32 * (warp & 3);
        const int r = lane_base + lane;
        const uint32_t t_row = tmem + ((uint32_t)lane_base << 16);
        const uint32_t part_row = map_rank(part0 + (uint32_t)(r * TS::PART_LD * 4), 0);
        const uint32_t peer_full = map_rank(part_full, 0);
        const uint32_t peer_free = map_rank(part_free, 1);
        uint32_t tph = 0;
        int i = 0;
        for (int t = pair; t < p.n_tiles; t += n_pairs, ++i) {
            if (!mbar_wait(tfull, tph, abort_f, p.err, p.wait_cycles)) break;
            tc_fence_after();
            const int m = t * BM + r;
            bool ok = true;
            if (rank == 1) {
                // the previous tile's half has been read before this one overwrites it
                if (i > 0 && !mbar_wait_cluster(part_free, (uint32_t)((i - 1) & 1), abort_f, p.err,
                                                p.wait_cycles))
                    ok = false;
                if (ok) {
                    for (int c = 0; c < BNT / 32; ++c) {
                        float v[32];
                        tmem_ld32(t_row + (uint32_t)(c * 32), v);
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            st_cluster_v4(part_row + (uint32_t)((c * 32 + 4 * q) * 4), v[4 * q],
                                          v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                    }
                    asm volatile("fence.acq_rel.cluster;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(peer_full);
                }
            } else {
                if (!mbar_wait_cluster(part_full, (uint32_t)(i & 1), abort_f, p.err, p.wait_cycles))
                    ok = false;
                if (ok) {
                    const float* pr = part + (size_t)r * TS::PART_LD;
                    float dummy_max = 0.f, dummy_sum = 0.f;
                    int dummy_arg = 0;
                    for (int c = 0; c < BNT / 32; ++c) {
                        const int n = c * 32;
                        if (n >= p.N) break;                 // warp-uniform
                        float v[32];
                        tmem_ld32(t_row + (uint32_t)n, v);
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float4 o = *reinterpret_cast<const float4*>(pr + n + 4 * q);
                            v[4 * q] += o.x; v[4 * q + 1] += o.y; v[4 * q + 2] += o.z; v[4 * q + 3] += o.w;
                        }
                        epilogue_chunk<EPI_SHRINK>(p, m, n, v, &dummy_max, &dummy_sum, &dummy_arg);
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(peer_free);
                }
            }
            if (!ok) break;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty);
            tph ^= 1u;
        }
    }

    tc_fence_before();
    __syncthreads();                         // every role of this CTA has left its loop
    if (*abort_f && lane == 0) {
        if (warp == 0) {
            const int n = n_armed < STAGES ? n_armed : STAGES;
            for (int k = 0; k < n; ++k) {
                const int a = n_armed - 1 - k;
                const uint32_t aph = (uint32_t)(a / STAGES) & 1u;
                for (uint32_t it = 0; it < WAIT_LIMIT && !mbar_try(full(a % STAGES), aph); ++it)
                    __nanosleep(128);
            }
        } else if (warp == 1 && issued) {
            tc_commit(drain);
            for (uint32_t it = 0; it < WAIT_LIMIT && !mbar_try(drain, 0); ++it) __nanosleep(128);
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();                          // neither CTA leaves while the other may write to it
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(BNT)
                     : "memory");
    }
}

// ---- host side ---------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2-D bf16 map over a row-major [rows x cols] matrix with leading dimension ld,
// box = 64 columns x box_rows rows, 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint64_t ld,
              uint32_t box_rows, bool fp8 = false) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    // 128-byte box rows either way: 64 bf16 or 128 E4M3 elements
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {ld * (fp8 ? 1 : 2)};
    const cuuint32_t box[2] = {fp8 ? (cuuint32_t)BK8 : (cuuint32_t)BK, box_rows};
    const cuuint32_t es[2] = {1, 1};
    return fn(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
              const_cast<void*>(ptr), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output map for the TMA-store epilogue: [rows x cols] with leading dimension ld,
// bf16 boxes of 64 columns x 32 rows or fp32 boxes of 32 columns x 32 rows (128-byte
// inner extent, 128-byte swizzle); boxes past the edges are clipped.
bool make_map_out(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint64_t ld,
                  bool f32) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t esz = f32 ? 4 : 2;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {ld * esz};
    const cuuint32_t box[2] = {f32 ? 32u : 64u, 32u};
    const cuuint32_t es[2] = {1, 1};
    return fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
              const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int num_sms() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

template <int EPI, int BNT, bool F8 = false>
int launch_epi(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& a2,
               const CUtensorMap& b2, const TcParams& p, cudaStream_t st) {
    constexpr int smem = Tile1<BNT>::SMEM_BYTES;
    static bool attr = false;
    if (!attr) {
        if (cudaFuncSetAttribute(gemm_tc_kernel<EPI, BNT, F8>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return 1;
        attr = true;
    }
    const int items = EPI == EPI_SPLIT_T ? p.n_tiles * p.ksplit : p.n_tiles;
    const int grid = items < num_sms() ? items : num_sms();
    if (EPI == EPI_SPLIT_T)
        return launch_pdl(gemm_tc_kernel<EPI, BNT, F8>, dim3(grid), dim3(NUM_THREADS), smem, st, a, b,
                          a2, b2, p) == cudaSuccess ? 0 : 1;
    gemm_tc_kernel<EPI, BNT, F8><<<grid, NUM_THREADS, smem, st>>>(a, b, a2, b2, p);
    return cudaGetLastError() == cudaSuccess ? 0 : 1;
}

// N tile of the single-SM kernel: the narrowest of 64/128/256 that covers N, for
// the epilogues that work column chunk by column chunk; the LSE partials are laid out in
// BN_LSE-column tiles and the SwiGLU gate/up interleave in 256-column tiles.
int tile1_width(const GemmArgs& g) {
    if (g.epi == EPI_LSE) return BN_LSE;
    if (g.epi == EPI_SWIGLU) return BN;
    return g.N <= 64 ? 64 : (g.N <= 128 ? 128 : 256);
}

template <int EPI>
int launch_epi_w(int bnt, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& a2,
                 const CUtensorMap& b2, const TcParams& p, cudaStream_t st) {
    switch (bnt) {
        case 64: return launch_epi<EPI, 64>(a, b, a2, b2, p, st);
        case 128: return launch_epi<EPI, 128>(a, b, a2, b2, p, st);
        default: return launch_epi<EPI, 256>(a, b, a2, b2, p, st);
    }
}

template <int BNT>
int launch_shrink_pair(const CUtensorMap& a, const CUtensorMap& b, const TcParams& p,
                       cudaStream_t st) {
    constexpr int smem = TileS<BNT>::SMEM_BYTES;
    static bool attr = false;
    if (!attr) {
        if (cudaFuncSetAttribute(shrink_pair_kernel<BNT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smem) != cudaSuccess)
            return 1;
        attr = true;
    }
    int pairs = num_sms() / 2;
    if (p.n_tiles < pairs) pairs = p.n_tiles;
    shrink_pair_kernel<BNT><<<2 * pairs, NUM_THREADS, smem, st>>>(a, b, p);
    return cudaGetLastError() == cudaSuccess ? 0 : 1;
}

template <int EPI, bool F8, bool SPLIT = false>
int launch_epi2(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& a2,
                const CUtensorMap& b2, const CUtensorMap& c, const TcParams& p, cudaStream_t st) {
    static bool attr = false;
    if (!attr) {
        if (cudaFuncSetAttribute(gemm_tc2_kernel<EPI, F8, SPLIT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 SMEM2_BYTES) != cudaSuccess)
            return 1;
        attr = true;
    }
    static int max_pairs = 0;
    if (!max_pairs) {
        // SM pairs that can be resident at once (clusters of 2 stay inside a GPC)
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = 2; at[0].val.clusterDim.y = 1; at[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(2 * (num_sms() / 2), 1, 1);
        cfg.blockDim = dim3(NUM_THREADS, 1, 1);
        cfg.dynamicSmemBytes = SMEM2_BYTES;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, gemm_tc2_kernel<EPI, F8, SPLIT>, &cfg) != cudaSuccess || n <= 0)
            n = num_sms() / 2;
        max_pairs = n;
    }
    int pairs = max_pairs;
    const int items = SPLIT ? p.n_tiles * p.ksplit : p.n_tiles;
    if (items < pairs) pairs = items;
    gemm_tc2_kernel<EPI, F8, SPLIT><<<2 * pairs, NUM_THREADS, SMEM2_BYTES, st>>>(a, b, a2, b2, c, p);
    return cudaGetLastError() == cudaSuccess ? 0 : 1;
}

}  // namespace

namespace {

// y[m, n] = sum_s ws[s, m, n] (in s order) + bias[n], then the epilogue: bf16 store / ReLU,
// or the fp32 residual add.  One thread per 4 columns.
// (kv.cache: the k|v columns of each row also go to its key/value cache row.)  Four
// consecutive bf16 outputs n..n+3 of row m (n a multiple of 4, as q_dim and kv2 are), one
// 8-byte store when they are k|v columns.
__device__ __forceinline__ uint32_t bf16_pair_bits(__nv_bfloat16 a, __nv_bfloat16 b) {
    return (uint32_t)__bfloat16_as_ushort(a) | ((uint32_t)__bfloat16_as_ushort(b) << 16);
}
__device__ __forceinline__ void kv_put4(const KvAppend& kv, int m, int n, uint2 v4) {
    const int c = n - kv.q_dim;
    if (c < 0 || c >= kv.kv2) return;
    const size_t crow = (size_t)kv.cu[m] + (size_t)m * kv.G + kv.lens[m] + kv.g;
    if (!ZO_DCHECK(crow < kv.cache_rows, ZO_DBG_KV_SLOT)) return;     // (debug build)
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(kv.cache) + crow * kv.kv2 + c) = v4;
}

__global__ void splitk_epilogue_kernel(const float* __restrict__ ws, int ks, int M, int N,
                                       const float* __restrict__ bias, int epi, void* C, int ldc,
                                       KvAppend kv) {
    grid_dep_wait();
    const int m = blockIdx.y;
    const int n = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
    if (n >= N) return;
    float y[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) y[j] = 0.f;
    for (int s = 0; s < ks; ++s) {
        const float* w = ws + ((size_t)s * M + m) * N + n;
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (n + j < N) y[j] += w[j];
    }
    __nv_bfloat16 hv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (n + j >= N) break;
        float v = y[j] + (bias ? bias[n + j] : 0.f);
        if (epi == EPI_RESID) {
            static_cast<float*>(C)[(size_t)m * ldc + n + j] += v;
        } else {
            if (epi == EPI_STORE_RELU) v = fmaxf(v, 0.f);
            hv[j] = __float2bfloat16_rn(v);
            static_cast<__nv_bfloat16*>(C)[(size_t)m * ldc + n + j] = hv[j];
        }
    }
    if (kv.cache && n + 4 <= N)
        kv_put4(kv, m, n, make_uint2(bf16_pair_bits(hv[0], hv[1]), bf16_pair_bits(hv[2], hv[3])));
}

// SwiGLU from the split slices: gate/up rows interleaved in 128-row blocks, so output f
// reads column (f / 128) * 256 + f % 128 (gate) and the one 128 after it (up).
__global__ void splitk_swiglu_kernel(const float* __restrict__ ws, int ks, int M, int N,
                                     const float* __restrict__ bias, __nv_bfloat16* C, int ldc) {
    grid_dep_wait();
    const int m = blockIdx.y;
    const int f = blockIdx.x * blockDim.x + threadIdx.x;
    const int F = N / 2;
    if (f >= F) return;
    const int gc = (f / 128) * 256 + f % 128, uc = gc + 128;
    float g = 0.f, u = 0.f;
    for (int s = 0; s < ks; ++s) {
        const float* w = ws + ((size_t)s * M + m) * N;
        g += w[gc];
        u += w[uc];
    }
    if (bias) {
        g += bias[gc];
        u += bias[uc];
    }
    C[(size_t)m * ldc + f] = __float2bfloat16_rn(g / (1.0f + expf(-g)) * u);
}

// Qwen3 q|k|v from the split slices, one warp per (row, head): the summed head is rounded
// to bf16, then q and k heads get RMSNorm over the head and the rotary rotation of the
// pairs (i, i + 64) at the token's position; lane l holds columns 4l..4l+3, its partner
// columns sit in lane l ^ 16.
__global__ void splitk_qknr_kernel(const float* __restrict__ ws, int ks, int M, int N, TcParams p,
                                   __nv_bfloat16* C, int ldc, KvAppend kv) {
    grid_dep_wait();
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    const int heads = N / 128;
    if (warp >= M * heads) return;
    const int m = warp / heads, head = warp % heads;
    const int c0 = head * 128 + 4 * lane;
    float x[4] = {0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < ks; ++s) {
        const float4 w = *reinterpret_cast<const float4*>(ws + ((size_t)s * M + m) * N + c0);
        x[0] += w.x; x[1] += w.y; x[2] += w.z; x[3] += w.w;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] = __bfloat162float(__float2bfloat16_rn(x[e]));
    if (head < p.n_qk_heads) {
        float ss = x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3];
        ss = warp_sum(ss);
        const float rs = 1.0f / sqrtf(ss / 128.0f + p.norm_eps);
        const float* w = head < p.n_q_heads ? p.qn : p.kn;
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = x[e] * rs * w[4 * lane + e];
        const int pos = p.tok_pos[m];
        const int i0 = (4 * lane) & 63;
        float partner[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) partner[e] = __shfl_xor_sync(0xffffffffu, x[e], 16);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float cs = p.rope_cos[(size_t)pos * 64 + i0 + e];
            const float sn = p.rope_sin[(size_t)pos * 64 + i0 + e];
            // lanes 0..15 hold a = x[i], lanes 16..31 hold b = x[i + 64]
            x[e] = lane < 16 ? x[e] * cs - partner[e] * sn : x[e] * cs + partner[e] * sn;
        }
    }
    __nv_bfloat16 hv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        hv[e] = __float2bfloat16_rn(x[e]);
        C[(size_t)m * ldc + c0 + e] = hv[e];
    }
    if (kv.cache)
        kv_put4(kv, m, c0, make_uint2(bf16_pair_bits(hv[0], hv[1]), bf16_pair_bits(hv[2], hv[3])));
}

// [ks][M][N] fp32 workspace, 32 x 32 boxes (128-byte rows, 128-byte swizzle)
bool make_map_ws(CUtensorMap* m, const float* ws, int ks, int M, int N) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)N, (cuuint64_t)M, (cuuint64_t)ks};
    const cuuint64_t strides[2] = {(cuuint64_t)N * 4, (cuuint64_t)M * N * 4};
    const cuuint32_t box[3] = {32u, 32u, 1u};
    const cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(ws), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The split reduction of a [ks][M][N] workspace into g.C with g's epilogue; with pdl it is
// launched as a programmatic dependent of the GEMM that wrote the slices.
int launch_split_reduce(const GemmArgs& g, const TcParams& p, int ks, cudaStream_t st, bool pdl) {
    cudaError_t e = cudaSuccess;
    // k|v to the cache from the bf16 store or q/k-norm reduction (bf16 models only)
    KvAppend kv;
    memset(&kv, 0, sizeof(kv));
    if (g.kv_append && (g.epi == EPI_STORE || g.epi == EPI_QKNR) && g.c_type == E_BF16)
        kv = *g.kv_append;
    auto go = [&](auto kernel, dim3 grid, auto... args) {
        if (pdl) {
            e = launch_pdl(kernel, grid, dim3(128), 0, st, args...);
        } else {
            kernel<<<grid, 128, 0, st>>>(args...);
            e = cudaGetLastError();
        }
    };
    if (g.epi == EPI_SHRINK) {
        launch_shrink_rows_sum(g.ws, ks, g.M, g.N, g.C, g.ldc, g.c_type, g.row_sign, g.eps,
                               g.scale_cols, g.a_scale, st, pdl);
        e = cudaGetLastError();
    } else if (g.epi == EPI_SWIGLU) {
        go(splitk_swiglu_kernel, dim3((unsigned)((g.N / 2 + 127) / 128), (unsigned)g.M),
           (const float*)g.ws, ks, g.M, g.N, g.bias, static_cast<__nv_bfloat16*>(g.C), g.ldc);
    } else if (g.epi == EPI_QKNR) {
        const long long warps = (long long)g.M * (g.N / 128);
        go(splitk_qknr_kernel, dim3((unsigned)((warps + 3) / 4)), (const float*)g.ws, ks, g.M, g.N,
           p, static_cast<__nv_bfloat16*>(g.C), g.ldc, kv);
        if (kv.cache && g.kv_done) *g.kv_done = 1;
    } else if (g.epi == EPI_RESID && g.norm_next &&
               launch_splitk_resid_norm(g.ws, ks, g.M, g.N, g.bias, static_cast<float*>(g.C),
                                        g.ldc, *g.norm_next, st, pdl)) {
        // the residual rows and the next norm in one pass
        e = cudaGetLastError();
        if (g.norm_done) *g.norm_done = 1;
    } else {
        go(splitk_epilogue_kernel, dim3((unsigned)((g.N / 4 + 127) / 128), (unsigned)g.M),
           (const float*)g.ws, ks, g.M, g.N, g.bias, g.epi, g.C, g.ldc, kv);
        if (kv.cache && g.kv_done) *g.kv_done = 1;
    }
    return e == cudaSuccess ? 0 : 1;
}

// Splits of kb_main K blocks into ks parts of kbs blocks: the number of non-empty parts.
int effective_splits(int kb_main, int ks, int* kbs) {
    *kbs = (kb_main + ks - 1) / ks;
    return (kb_main + *kbs - 1) / *kbs;
}

// Decode-step GEMM on single SMs with the operands swapped: A = the weights [N x K] (128-row
// tiles), B = the M <= 128 token rows (one N tile of 32, 64 or 128), likewise for the
// extension blocks.  Each (weight tile, K split) item writes its fp32 slice transposed into
// the workspace, then the split reduction applies g's epilogue.
int gemm_tc_swapped(const GemmArgs& g, cudaStream_t st) {
    const int bnt = g.M <= 32 ? 32 : (g.M <= 64 ? 64 : 128);
    const bool f8 = g.a_type == E_FP8;                // E4M3 main blocks (both operands)
    CUtensorMap a, b, a2, b2;
    if (!make_map(&a, g.B, g.N, g.K, g.ldb, BM, f8)) return 1;
    if (!make_map(&b, g.A, g.M, g.K, g.lda, bnt, f8)) return 1;
    if (g.K2 > 0) {
        if (!make_map(&a2, g.B2, g.N, g.K2, g.ldb2, BM)) return 1;
        if (!make_map(&b2, g.A2, g.M, g.K2, g.lda2, bnt)) return 1;
    } else {
        a2 = a;
        b2 = b;
    }
    TcParams p;
    memset(&p, 0, sizeof(p));
    p.M = g.N; p.N = g.M;
    p.kb_main = f8 ? (g.K + BK8 - 1) / BK8 : (g.K + BK - 1) / BK;
    p.kb_ext = g.K2 > 0 ? (g.K2 + BK - 1) / BK : 0;
    // swapped sides: the weight rows' scales are the kernel's M side, the tokens' its N side
    p.a_scale = g.b_scale; p.b_scale = g.a_scale;
    p.n_m_blk = (g.N + BM - 1) / BM;
    p.n_n_blk = 1;
    p.n_tiles = p.n_m_blk;
    p.group_m = GROUP_M;
    p.epi = EPI_SPLIT_T;
    p.C = g.ws; p.ldc = g.N; p.c_type = E_F32;
    p.tok_pos = g.tok_pos; p.qn = g.qn; p.kn = g.kn;
    p.rope_cos = g.rope_cos; p.rope_sin = g.rope_sin; p.norm_eps = g.norm_eps;
    p.n_q_heads = g.n_q_heads; p.n_qk_heads = g.n_qk_heads;
    int* err = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&err), g_tc_error) != cudaSuccess) return 1;
    p.err = err;
    p.wait_cycles = g_wait_cycles;
    // K splits: the weight stream is the cost.  In units of one 128 x 64 weight block, the
    // busiest SM streams rounds x (kbs + slice) blocks at up to SM_BW_REL times its fair share
    // of HBM, and all SMs together stream the weights plus the slices written and read back;
    // take the split count with the smaller bound, every split keeping at least 2 blocks.
    const int sms = num_sms();
    constexpr double SM_BW_REL = 1.25;
    const double slice = g.M / 32.0;                 // 128 x M fp32 = M / 32 weight blocks
    int ks = 1;
    double best = 1e300;
    for (int k = 1; k <= 16 && k <= std::max(1, p.kb_main / 2); ++k) {
        int kbs;
        if (effective_splits(p.kb_main, k, &kbs) != k) continue;
        if ((size_t)k * g.M * g.N > g.ws_floats) break;
        const long long items = (long long)p.n_tiles * k;
        const long long rounds = (items + sms - 1) / sms;
        const double t_sm = (double)rounds * (kbs + slice) / SM_BW_REL;
        const double t_hbm = ((double)p.n_tiles * p.kb_main + 2.0 * items * slice) / sms;
        const double cost = std::max(t_sm, t_hbm);
        if (cost < best * 0.98) {                    // a clear gain for each extra split
            best = cost;
            ks = k;
        }
    }
    ks = effective_splits(p.kb_main, ks, &p.kbs);
    p.ksplit = ks;
    int rc;
    switch (bnt + (f8 ? 1 : 0)) {
        case 32: rc = launch_epi<EPI_SPLIT_T, 32>(a, b, a2, b2, p, st); break;
        case 64: rc = launch_epi<EPI_SPLIT_T, 64>(a, b, a2, b2, p, st); break;
        case 128: rc = launch_epi<EPI_SPLIT_T, 128>(a, b, a2, b2, p, st); break;
        case 33: rc = launch_epi<EPI_SPLIT_T, 32, true>(a, b, a2, b2, p, st); break;
        case 65: rc = launch_epi<EPI_SPLIT_T, 64, true>(a, b, a2, b2, p, st); break;
        default: rc = launch_epi<EPI_SPLIT_T, 128, true>(a, b, a2, b2, p, st); break;
    }
    if (rc) return rc;
    return launch_split_reduce(g, p, ks, st, true);
}

}  // namespace

bool gemm_tc_supported(const GemmArgs& g) {
    if (g.a_type == E_FP8 || g.b_type == E_FP8) {
        // E4M3 main operands: SM-pair kernel, 16-byte rows, scales for both sides
        if (g.a_type != E_FP8 || g.b_type != E_FP8 || !g_use_pairs || g.N <= 128) return false;
        if (g.K % 16 || g.lda % 16 || g.ldb % 16 || g.K <= 0 || g.M <= 0) return false;
        if (!g.a_scale || !g.b_scale) return false;
        if (g.epi != EPI_STORE && g.epi != EPI_STORE_RELU && g.epi != EPI_QKNR &&
            g.epi != EPI_SWIGLU)
            return false;
    } else {
        if (g.a_type != E_BF16 || g.b_type != E_BF16) return false;
        if (g.K % 8 || g.lda % 8 || g.ldb % 8 || g.K <= 0 || g.M <= 0 || g.N <= 0) return false;
    }
    if (!aligned16(g.A) || !aligned16(g.B)) return false;
    if (g.K2 > 0) {
        if (g.a2_type != E_BF16 || g.b2_type != E_BF16 || g.lda2 % 8 || g.ldb2 % 8 || g.K2 % 8)
            return false;
        if (!aligned16(g.A2) || !aligned16(g.B2)) return false;
    }
    switch (g.epi) {
        case EPI_STORE:
        case EPI_STORE_RELU:
            if (g.c_type != E_BF16 || g.ldc % 8 || !aligned16(g.C)) return false;
            if (g.bias && !aligned16(g.bias)) return false;
            return true;
        case EPI_RESID:
            if (g.c_type != E_F32 || g.ldc % 4 || !aligned16(g.C)) return false;
            if (g.bias && !aligned16(g.bias)) return false;
            return true;
        case EPI_LSE:
            return true;
        case EPI_SHRINK:
            if (g.c_type != E_BF16 || g.ldc % 8 || !aligned16(g.C)) return false;
            return true;
        case EPI_SWIGLU:
            if (g.c_type != E_BF16 || g.ldc % 8 || !aligned16(g.C) || g.N % 256) return false;
            return true;
        case EPI_QKNR:
            // SM-pair kernel only; head_dim 128, whole heads per 256-column tile
            if (!g_use_pairs || g.N <= 128 || g.N % 128) return false;
            if (g.c_type != E_BF16 || g.ldc % 8 || !aligned16(g.C) || g.bias) return false;
            if (!g.tok_pos || !g.qn || !g.kn || !g.rope_cos || !g.rope_sin) return false;
            if (!aligned16(g.qn) || !aligned16(g.kn) || !aligned16(g.rope_cos) ||
                !aligned16(g.rope_sin))
                return false;
            return g.n_qk_heads * 128 <= g.N && g.n_q_heads <= g.n_qk_heads;
        default:
            return false;
    }
}

int gemm_tc_col_tiles(int N) { return (N + BN_LSE - 1) / BN_LSE; }

int gemm_tc(const GemmArgs& g, cudaStream_t st) {
    // Decoder GEMMs run on SM pairs, the LSE and shrink forms on single SMs.  The
    // choice never depends on M (the batch): a row's bits must not change with
    // the company it is scored in.  Decode steps (a workspace given) are the exception:
    // their few token rows take the swapped single-SM form.
    const bool bf16_ops = g.a_type == E_BF16 && g.b_type == E_BF16;
    const bool e4m3_ops = g.a_type == E_FP8 && g.b_type == E_FP8 && g.a_scale && g.b_scale;
    if (g.ws && g.M <= 128 && (bf16_ops || e4m3_ops) && g.N % 4 == 0 &&
        (g.epi == EPI_STORE || g.epi == EPI_STORE_RELU || g.epi == EPI_RESID ||
         g.epi == EPI_SWIGLU || g.epi == EPI_QKNR || g.epi == EPI_SHRINK))
        return gemm_tc_swapped(g, st);
    const bool pair = g_use_pairs && g.N > 128 &&
                      (g.epi == EPI_STORE || g.epi == EPI_STORE_RELU || g.epi == EPI_RESID ||
                       g.epi == EPI_SWIGLU || g.epi == EPI_QKNR);
    if (g.epi == EPI_QKNR && !pair) return 1;
    const int bnt = pair ? BN : tile1_width(g);
    const uint32_t b_rows = pair ? 128u : (uint32_t)bnt;
    CUtensorMap a, b, a2, b2;
    const bool f8 = g.a_type == E_FP8;
    if (f8 && !pair) return 1;
    if (!make_map(&a, g.A, g.M, g.K, g.lda, BM, f8)) return 1;
    if (!make_map(&b, g.B, g.N, g.K, g.ldb, b_rows, f8)) return 1;
    if (g.K2 > 0) {
        if (!make_map(&a2, g.A2, g.M, g.K2, g.lda2, BM)) return 1;
        if (!make_map(&b2, g.B2, g.N, g.K2, g.ldb2, b_rows)) return 1;
    } else {
        a2 = a;
        b2 = b;
    }
    TcParams p;
    memset(&p, 0, sizeof(p));
    p.M = g.M; p.N = g.N;
    p.kb_main = f8 ? (g.K + BK8 - 1) / BK8 : (g.K + BK - 1) / BK;
    p.a_scale = g.a_scale; p.b_scale = g.b_scale;
    p.kb_ext = g.K2 > 0 ? (g.K2 + BK - 1) / BK : 0;
    p.n_m_blk = pair ? (g.M + BM2 - 1) / BM2 : (g.M + BM - 1) / BM;
    // Raster: the SM pairs walk M groups of 12 blocks of 256 rows, each sweeping every N
    // block, so a weight strip is fetched once per group while the group's A strips stay in
    // L2.  12 was the fastest of 4..24 for both the fc1 (K = 5120) and fc2 (K = 20480) shapes
    // of the OPT-13B step, timed on B200 under the power cap.
    p.group_m = pair ? 12 : GROUP_M;
    p.n_n_blk = (g.N + bnt - 1) / bnt;
    p.n_tiles = p.n_m_blk * p.n_n_blk;
    p.epi = g.epi;
    p.bias = g.bias;
    p.C = g.C; p.ldc = g.ldc; p.c_type = g.c_type;
    p.targets = g.targets; p.part_max = g.part_max; p.part_sum = g.part_sum;
    p.tgt_logit = g.tgt_logit; p.n_col_tiles = g.n_col_tiles;
    p.part_arg = g.part_arg;
    p.row_sign = g.row_sign; p.eps = g.eps; p.scale_cols = g.scale_cols;
    p.tok_pos = g.tok_pos; p.qn = g.qn; p.kn = g.kn;
    p.rope_cos = g.rope_cos; p.rope_sin = g.rope_sin; p.norm_eps = g.norm_eps;
    p.n_q_heads = g.n_q_heads; p.n_qk_heads = g.n_qk_heads;
    int* err = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&err), g_tc_error) != cudaSuccess) return 1;
    p.err = err;
    p.wait_cycles = g_wait_cycles;
    if (g.epi == EPI_SHRINK && !g.ws && !f8 && g.K2 == 0 && bnt <= 128 && p.kb_main >= 2) {
        // the bank shrink of a scoring batch: K split over a CTA pair so that every SM streams
        // rows of x (chosen by N and K only, never by M); up to 32 bank columns take a
        // 32-wide N tile, whose smaller stages leave room for more of them in flight
        if (g.N <= 32) {
            if (!make_map(&b, g.B, g.N, g.K, g.ldb, 32u)) return 1;
            p.n_n_blk = 1;
            p.n_tiles = p.n_m_blk;
            return launch_shrink_pair<32>(a, b, p, st);
        }
        return bnt == 64 ? launch_shrink_pair<64>(a, b, p, st) : launch_shrink_pair<128>(a, b, p, st);
    }
    if (pair && g.ws && !f8 && g.N % 4 == 0 &&
        (g.epi == EPI_STORE || g.epi == EPI_STORE_RELU || g.epi == EPI_RESID ||
         g.epi == EPI_SWIGLU || g.epi == EPI_QKNR)) {
        // too few output tiles to keep the SM pairs streaming the weights: split K so that
        // about two items per pair exist, each split keeping at least 4 main K blocks
        const int pairs = num_sms() / 2;
        int ks = (2 * pairs + p.n_tiles - 1) / p.n_tiles;
        ks = std::min(ks, std::min(8, p.kb_main / 4));
        while (ks > 1 && (size_t)ks * g.M * g.N > g.ws_floats) --ks;
        if (ks > 1) ks = effective_splits(p.kb_main, ks, &p.kbs);   // no split without K blocks
        if (ks > 1) {
            p.ksplit = ks;
            CUtensorMap c;
            if (!make_map_ws(&c, g.ws, ks, g.M, g.N)) return 1;
            // the split kernels' epilogue only stores fp32 slices: one instantiation serves all
            const int rc = launch_epi2<EPI_STORE, false, true>(a, b, a2, b2, c, p, st);
            if (rc) return rc;
            return launch_split_reduce(g, p, ks, st, false);
        }
    }
    if (pair) {
        // output map for the TMA-store epilogue: 32-row boxes, 128-byte inner extent
        CUtensorMap c;
        const bool f32 = g.epi == EPI_RESID;
        const uint64_t cols = g.epi == EPI_SWIGLU ? (uint64_t)(g.N / 2) : (uint64_t)g.N;
        if (!make_map_out(&c, g.C, (uint64_t)g.M, cols, (uint64_t)g.ldc, f32)) return 1;
        switch (g.epi) {
            case EPI_STORE:
                return f8 ? launch_epi2<EPI_STORE, true>(a, b, a2, b2, c, p, st)
                          : launch_epi2<EPI_STORE, false>(a, b, a2, b2, c, p, st);
            case EPI_STORE_RELU:
                return f8 ? launch_epi2<EPI_STORE_RELU, true>(a, b, a2, b2, c, p, st)
                          : launch_epi2<EPI_STORE_RELU, false>(a, b, a2, b2, c, p, st);
            case EPI_RESID: return f8 ? 1 : launch_epi2<EPI_RESID, false>(a, b, a2, b2, c, p, st);
            case EPI_SWIGLU:
                return f8 ? launch_epi2<EPI_SWIGLU, true>(a, b, a2, b2, c, p, st)
                          : launch_epi2<EPI_SWIGLU, false>(a, b, a2, b2, c, p, st);
            case EPI_QKNR:
                return f8 ? launch_epi2<EPI_QKNR, true>(a, b, a2, b2, c, p, st)
                          : launch_epi2<EPI_QKNR, false>(a, b, a2, b2, c, p, st);
            default: return 1;
        }
    }
    switch (g.epi) {
        case EPI_STORE: return launch_epi_w<EPI_STORE>(bnt, a, b, a2, b2, p, st);
        case EPI_STORE_RELU: return launch_epi_w<EPI_STORE_RELU>(bnt, a, b, a2, b2, p, st);
        case EPI_RESID: return launch_epi_w<EPI_RESID>(bnt, a, b, a2, b2, p, st);
        case EPI_LSE: return launch_epi<EPI_LSE, BN_LSE>(a, b, a2, b2, p, st);
        case EPI_SHRINK: return launch_epi_w<EPI_SHRINK>(bnt, a, b, a2, b2, p, st);
        case EPI_SWIGLU: return launch_epi<EPI_SWIGLU, BN>(a, b, a2, b2, p, st);
        default: return 1;
    }
}


long long gemm_tc_set_wait_cycles(long long cycles) {
    const long long old = g_wait_cycles;
    g_wait_cycles = cycles > 0 ? cycles : WAIT_CYCLES;
    return old;
}

int gemm_tc_error_word() {
    int v = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_tc_error, sizeof(int)) != cudaSuccess) return -1;
    cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(int));
    return v;
}

}  // namespace zo
