// Packed variable-length causal attention on the 5th-generation tensor cores.
//
// Work items are (128-query tile of one row, head) pairs, one CTA (4 warps,
// 128 threads) each; thread i owns query row i of the tile, which is also TMEM
// lane i.  Per 128-key chunk of the row:
//   S  = Q K^T        tcgen05.mma M=128 N=128 K=128, fp32 accumulator in TMEM
//   P  = exp(S*scale - m)  (causal and length masks) written as bf16 into the
//                     K buffer, in the 128-byte-swizzled K-major layout
//   O += P V          tcgen05.mma M=128 N=128 K=128, V read as an MN-major operand
// Across chunks the softmax is online: the running maximum and sum live in the
// thread's registers, the output row in TMEM, rescaled by exp(m_old - m_new)
// before each chunk's P V accumulates onto it.  Queries, keys and
// values arrive by TMA straight into the 128-byte-swizzled layout (Qwen3's
// q/k norm and rotary positions were applied to the q|k|v rows beforehand).
// Keys past the row's end are masked to zero probability, so a query's result
// depends only on its own row: packing never changes a bit.
#include <cuda.h>
#include <float.h>

#include "common.cuh"
#include "kernels.h"

namespace zo {

namespace {

constexpr int TQ = 128, TK = 128, HD = 128;
constexpr int ATOM = TQ * 128;                  // bytes of one 64-column swizzle atom block
constexpr int BUF = 2 * ATOM;                   // one [128 x 128] bf16 operand
constexpr int SMEM = 3 * BUF + 1024 + 64;
constexpr long long WAIT_CYCLES = 4000000000ll;
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(TK >> 3) << 17) |
                            ((uint32_t)(TQ >> 4) << 24);

__device__ int g_attn_error = 0;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}
// byte offset of 16-byte chunk c (0..15) of row r in a [128 x 128] bf16 K-major SW128 operand
__device__ __forceinline__ uint32_t sw_off(int r, int c) {
    return (uint32_t)((c >> 3) * ATOM + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}
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

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
        "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
        "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
        "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
        "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}

__device__ __forceinline__ uint32_t pack_bf2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, int* err) {
    const long long t0 = clock64();
    for (uint32_t i = 0;; ++i) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
        if (ok) return true;
        if ((i & 63u) == 63u && clock64() - t0 > WAIT_CYCLES) {   // ~2 s: never arrives
            atomicOr(err, 1);
            return false;
        }
    }
}

// 8 MMAs (K = 128 = 2 atoms x 4 steps of 16) into TMEM column d_col, then commit.
__device__ __forceinline__ void mma_128(uint32_t d_tmem, uint32_t a, uint32_t b, bool accum_first,
                                        uint32_t bar) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = (kk >> 2) * ATOM + (kk & 3) * 32;
        const uint32_t acc = (kk > 0 || accum_first) ? 1u : 0u;
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(sw128_desc(a + off)), "l"(sw128_desc(b + off)), "r"(kIdesc), "r"(acc)
            : "memory");
    }
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}

__device__ __forceinline__ uint64_t sw128_desc_mn(uint32_t saddr) {
    // MN-major operand (V as the B operand of P.V): 64-element MN blocks 16 KB
    // apart (leading byte offset), 8-row K groups 1024 bytes apart (stride byte offset)
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((uint32_t)ATOM >> 4) << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}
// P.V: A = P (K-major, keys contiguous), B = V as loaded ([keys x dims], MN-major)
constexpr uint32_t kIdescPV = kIdesc | (1u << 16);

__device__ __forceinline__ void tma_box(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x,
                                        int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

// One (query tile, head) work item.
struct Item {
    int start, len, q0, nq, kend, n_chunks, h, kvh;
};
__device__ __forceinline__ Item get_item(const AttnArgs& a, int i) {
    Item it;
    const int tile = a.tiles[i / a.H];
    const int row = tile >> 16, qt = tile & 0xFFFF;
    it.h = i % a.H;
    it.kvh = it.h / (a.H / a.Hkv);
    it.start = a.cu_seqlens[row];
    it.len = a.cu_seqlens[row + 1] - it.start;
    it.q0 = qt * TQ;
    it.nq = min(TQ, it.len - it.q0);
    it.kend = min(it.len, it.q0 + TQ);
    it.n_chunks = (it.kend + TK - 1) / TK;
    return it;
}

__device__ __forceinline__ float ex2_ftz(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// One CTA per item, two CTAs per SM: while one CTA waits on its TMA loads or
// its MMAs, the other runs its softmax.  Items are dealt longest first.
__global__ void __launch_bounds__(128, 2)
    attention_tc_kernel(const __grid_constant__ CUtensorMap tm, AttnArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* g = smem_raw + (base - raw);
    uint8_t* Qb = g;
    uint8_t* KPb = g + BUF;
    uint8_t* Vb = g + 2 * BUF;
    const uint32_t bar_mma = base + 3 * BUF;
    const uint32_t bar_ld = bar_mma + 8;               // Q and K of a chunk
    const uint32_t bar_v = bar_mma + 16;               // V of a chunk: lands under QK^T + softmax
    uint32_t* tslot = reinterpret_cast<uint32_t*>(g + 3 * BUF + 32);

    const Item it = get_item(a, blockIdx.x);
    const int q_dim = a.H * HD, kv_dim = a.Hkv * HD;
    const int tid = threadIdx.x, warp = tid >> 5;
    int* err = &g_attn_error;

    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_mma));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_ld));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_v));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 256;" ::"r"(
                         smem_u32(tslot))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tslot;
    const uint32_t t_s = tmem, t_o = tmem + 128;
    const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
    uint32_t ph_mma = 0, ph_ld = 0, ph_v = 0;
    bool ok = true, v_pending = false;
    const int q = it.q0 + tid;                         // this thread's query
    const float sl2 = a.scale * 1.4426950408889634f;
    const int kcol = q_dim + it.kvh * HD, vcol = q_dim + kv_dim + it.kvh * HD;

    float m = -FLT_MAX, l = 0.f;
    for (int c = 0; c < it.n_chunks && ok; ++c) {
        const int c0 = c * TK;
        // K and V of chunk c (and Q with the first): rows past the tensor read as zero
        if (tid == 0) {
            const uint32_t bytes = (uint32_t)BUF * (c == 0 ? 2u : 1u);
            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar_ld),
                         "r"(bytes)
                         : "memory");
            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar_v),
                         "r"((uint32_t)BUF)
                         : "memory");
            const int r0 = it.start + c0;
            for (int half = 0; half < 2; ++half) {
                if (c == 0)
                    tma_box(smem_u32(Qb) + half * ATOM, &tm, bar_ld, it.h * HD + half * 64,
                            it.start + it.q0);
                tma_box(smem_u32(KPb) + half * ATOM, &tm, bar_ld, kcol + half * 64, r0);
            }
            for (int half = 0; half < 2; ++half)
                tma_box(smem_u32(Vb) + half * ATOM, &tm, bar_v, vcol + half * 64, r0);
        }
        v_pending = true;
        ok = __syncthreads_and(wait_bar(bar_ld, ph_ld, err));
        ph_ld ^= 1u;
        if (!ok) break;

        // S = Q K^T
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncthreads();
        if (tid == 0) mma_128(t_s, smem_u32(Qb), smem_u32(KPb), false, bar_mma);
        ok = __syncthreads_and(wait_bar(bar_mma, ph_mma, err));
        ph_mma ^= 1u;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        if (!ok) break;

        // keys c0 + j with j < lim are visible to this query (causal and row end); column
        // groups of 32 keys that no query of the warp sees are skipped, and so are warps
        // whose queries all lie past the row's end (warp-uniform; their P rows are zero)
        const int lim = min(q + 1, it.kend) - c0;
        const int wlim = min(it.q0 + warp * 32 + 32, it.kend) - c0;
        const bool warp_live = it.q0 + warp * 32 < it.len;
        const int ncc = (!warp_live || wlim <= 0) ? 0 : min(4, (wlim + 31) >> 5);
        float sv[4][32];
        float cmax = -FLT_MAX;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            if (cc < ncc) {
                tmem_ld32(t_s + lane_addr + cc * 32, sv[cc]);
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    sv[cc][j] = (cc * 32 + j < lim) ? sv[cc][j] : -FLT_MAX;
                    cmax = fmaxf(cmax, sv[cc][j]);
                }
            }
        }
        const float m_new = fmaxf(m, cmax);
        // rows whose every key so far is masked keep m = -FLT_MAX and contribute nothing
        const float alpha = (m > -FLT_MAX) ? exp2f((m - m_new) * sl2) : 0.f;
        // masked scores are -FLT_MAX, so exp2(s*sl2 - ms) underflows to exactly 0 for them
        const float ms = (m_new > -FLT_MAX) ? m_new * sl2 : 0.f;
        float cs0 = 0.f, cs1 = 0.f;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            uint32_t w[16];
            if (cc < ncc) {
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const float p0 = ex2_ftz(fmaf(sv[cc][j], sl2, -ms));
                    const float p1 = ex2_ftz(fmaf(sv[cc][j + 1], sl2, -ms));
                    cs0 += p0;
                    cs1 += p1;
                    w[j / 2] = pack_bf2(p0, p1);
                }
            } else {
#pragma unroll
                for (int j = 0; j < 16; ++j) w[j] = 0u;
            }
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4)
                *reinterpret_cast<uint4*>(KPb + sw_off(tid, cc * 4 + k4)) =
                    make_uint4(w[4 * k4], w[4 * k4 + 1], w[4 * k4 + 2], w[4 * k4 + 3]);
        }
        l = l * alpha + (cs0 + cs1);
        m = m_new;
        if (c > 0) {
            // the running output stays in TMEM: rescale it by exp(m_old - m_new), then P V
            // accumulates on top of it
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
                float v[32];
                tmem_ld32(t_o + lane_addr + cc * 32, v);
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] *= alpha;
                tmem_st32(t_o + lane_addr + cc * 32, v);
            }
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        }

        // O (+)= P V, once V has landed
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        ok = __syncthreads_and(wait_bar(bar_v, ph_v, err));
        if (!ok) break;
        ph_v ^= 1u;
        v_pending = false;
        if (tid == 0) {
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t acc = (kk > 0 || c > 0) ? 1u : 0u;
                const uint64_t ad = sw128_desc(smem_u32(KPb) + (kk >> 2) * ATOM + (kk & 3) * 32);
                const uint64_t bd = sw128_desc_mn(smem_u32(Vb) + kk * 2048);
                asm volatile(
                    "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                    "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(t_o),
                    "l"(ad), "l"(bd), "r"(kIdescPV), "r"(acc)
                    : "memory");
            }
            asm volatile(
                "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                    bar_mma)
                : "memory");
        }
        ok = __syncthreads_and(wait_bar(bar_mma, ph_mma, err));
        ph_mma ^= 1u;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        // the K/P and V buffers and the S columns are free again
    }
    if (ok) {
        const float inv = l > 0.f ? 1.f / l : 0.f;
        uint4* o4 = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) +
                                             (size_t)(it.start + q) * a.ld_out +
                                             (size_t)it.h * HD);
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
            float v[32];
            tmem_ld32(t_o + lane_addr + cc * 32, v);          // warp-collective: every lane
            if (tid < it.nq) {
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4)
                    o4[cc * 4 + k4] = make_uint4(pack_bf2(v[8 * k4] * inv, v[8 * k4 + 1] * inv),
                                                 pack_bf2(v[8 * k4 + 2] * inv, v[8 * k4 + 3] * inv),
                                                 pack_bf2(v[8 * k4 + 4] * inv, v[8 * k4 + 5] * inv),
                                                 pack_bf2(v[8 * k4 + 6] * inv, v[8 * k4 + 7] * inv));
            }
        }
    }
    if (v_pending && tid == 0) {
        // an aborted CTA lets its V copy land before its shared memory goes away
        const long long t0 = clock64();
        for (;;) {
            uint32_t done;
            asm volatile(
                "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                "selp.u32 %0, 1, 0, p;\n\t}"
                : "=r"(done)
                : "r"(bar_v), "r"(ph_v)
                : "memory");
            if (done || clock64() - t0 > WAIT_CYCLES) break;
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 256;" ::"r"(tmem)
                     : "memory");
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn attn_encode_fn() {
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

}  // namespace

bool attention_tc_supported(const AttnArgs& a) {
    return a.dtype == E_BF16 && a.hd == HD && a.ld_qkv % 8 == 0 && a.ld_out % 8 == 0 &&
           a.n_tokens > 0 && attn_encode_fn() != nullptr &&
           (reinterpret_cast<uintptr_t>(a.qkv) & 15) == 0 &&
           (reinterpret_cast<uintptr_t>(a.out) & 15) == 0;
}

bool launch_attention_tc(const AttnArgs& a, cudaStream_t st) {
    if (a.n_tiles == 0 || a.n_tokens <= 0) return true;
    static bool attr = false;
    if (!attr) {
        cudaFuncSetAttribute(attention_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
        attr = true;
    }
    // one map over the packed [T x ld_qkv] q|k|v rows: 64-column x 128-row boxes,
    // 128-byte swizzle, rows past T read as zero
    CUtensorMap tm;
    EncodeTiledFn fn = attn_encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)a.ld_qkv, (cuuint64_t)a.n_tokens};
    const cuuint64_t strides[1] = {(cuuint64_t)a.ld_qkv * 2};
    const cuuint32_t box[2] = {64, 128};
    const cuuint32_t es[2] = {1, 1};
    if (fn(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.qkv), dims, strides, box,
           es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    const long long items = (long long)a.n_tiles * a.H;
    if (items > 0x7fffffffLL) return false;
    attention_tc_kernel<<<(unsigned)items, 128, SMEM, st>>>(tm, a);
    return true;
}

int attention_tc_error_word() {
    int v = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_attn_error, sizeof(int)) != cudaSuccess) return -1;
    cudaMemcpyToSymbol(g_attn_error, &zero, sizeof(int));
    return v;
}

}  // namespace zo
