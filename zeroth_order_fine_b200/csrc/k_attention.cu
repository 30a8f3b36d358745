// Packed variable-length causal attention (no padding).
//
// Each CTA takes one 64-query tile of one row for one head; keys of that row
// are streamed in 64-key chunks from key 0 up to the tile's causal limit with
// an online softmax, so a query's result depends only on its own row (the
// ragged batch is a layout, never a change of results).  Scores and the
// softmax are fp32; q/k/v may be fp32 or bf16.
#include <float.h>

#include "common.cuh"
#include "kernels.h"

namespace zo {

ZO_DEBUG_WORD(debug_word_attention)

namespace {
constexpr int QT = 64;   // queries per CTA
constexpr int KC = 64;   // keys per chunk

// Stage one q or k row of head h into dst (fp32), times mul; executed by one warp.
template <int HD>
__device__ __forceinline__ void stage_row(const void* src, size_t base, int dtype, float* dst,
                                          float mul) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int i = 0; i < HD / 32; ++i) dst[lane + 32 * i] = ld_elem(src, base + lane + 32 * i, dtype) * mul;
    __syncwarp();
}

template <int HD>
__global__ void __launch_bounds__(256) attention_kernel(AttnArgs a) {
    extern __shared__ float sm[];
    float* Qs = sm;                        // [QT][HD]
    float* Ks = Qs + QT * HD;              // [KC][HD + 1]
    float* Vs = Ks + KC * (HD + 1);        // [KC][HD]
    const int tile = a.tiles[blockIdx.x];
    const int row = tile >> 16, qt = tile & 0xFFFF;
    // (debug build) a tile naming a row or query tile that is not there is skipped whole
    if (!ZO_DCHECK((unsigned)row < (unsigned)a.n_rows, ZO_DBG_ATTN_TILE)) return;
    const int h = blockIdx.y;
    const int kvh = h / (a.H / a.Hkv);
    const int start = a.cu_seqlens[row];
    const int len = a.cu_seqlens[row + 1] - start;
    const int q0 = qt * QT;
    if (!ZO_DCHECK(q0 < len, ZO_DBG_ATTN_TILE)) return;
    const int nq = min(QT, len - q0);
    const int kend = min(len, q0 + QT);    // keys needed by this tile
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q_dim = a.H * a.hd, kv_dim = a.Hkv * a.hd;

    for (int i = warp; i < nq; i += 8)
        stage_row<HD>(a.qkv, (size_t)(start + q0 + i) * a.ld_qkv + (size_t)h * HD, a.dtype,
                      Qs + i * HD, a.scale);

    constexpr int DPL = HD / 32;           // dims per lane in the PV product
    float m_i[8], l_i[8], o[8][DPL];
#pragma unroll
    for (int qi = 0; qi < 8; ++qi) {
        m_i[qi] = -FLT_MAX;
        l_i[qi] = 0.f;
#pragma unroll
        for (int d = 0; d < DPL; ++d) o[qi][d] = 0.f;
    }

    for (int c0 = 0; c0 < kend; c0 += KC) {
        __syncthreads();
        const int nk = min(KC, kend - c0);
        for (int j = warp; j < nk; j += 8) {
            const size_t tb = (size_t)(start + c0 + j) * a.ld_qkv;
            stage_row<HD>(a.qkv, tb + q_dim + (size_t)kvh * HD, a.dtype, Ks + j * (HD + 1), 1.f);
#pragma unroll
            for (int i = 0; i < HD / 32; ++i)
                Vs[j * HD + lane + 32 * i] =
                    ld_elem(a.qkv, tb + q_dim + kv_dim + (size_t)kvh * HD + lane + 32 * i, a.dtype);
        }
        __syncthreads();
#pragma unroll
        for (int qi = 0; qi < 8; ++qi) {
            const int ql = warp * 8 + qi;          // query within the tile
            if (ql >= nq) continue;
            const int qpos = q0 + ql;
            const float* qv = Qs + ql * HD;
            float s[2];
#pragma unroll
            for (int hk = 0; hk < 2; ++hk) {
                const int j = lane + 32 * hk;
                float acc = 0.f;
                const float* kv = Ks + j * (HD + 1);
#pragma unroll 8
                for (int d = 0; d < HD; ++d) acc = fmaf(qv[d], kv[d], acc);
                s[hk] = (j < nk && c0 + j <= qpos) ? acc : -FLT_MAX;
            }
            const float cmax = warp_max(fmaxf(s[0], s[1]));
            const float mnew = fmaxf(m_i[qi], cmax);
            const float p0 = s[0] > -FLT_MAX ? expf(s[0] - mnew) : 0.f;
            const float p1 = s[1] > -FLT_MAX ? expf(s[1] - mnew) : 0.f;
            const float corr = m_i[qi] > -FLT_MAX ? expf(m_i[qi] - mnew) : 0.f;
            l_i[qi] = l_i[qi] * corr + warp_sum(p0 + p1);
            m_i[qi] = mnew;
#pragma unroll
            for (int d = 0; d < DPL; ++d) o[qi][d] *= corr;
            for (int j = 0; j < nk; ++j) {
                const float p = __shfl_sync(0xffffffffu, j < 32 ? p0 : p1, j & 31);
#pragma unroll
                for (int d = 0; d < DPL; ++d) o[qi][d] = fmaf(p, Vs[j * HD + lane * DPL + d], o[qi][d]);
            }
        }
    }
#pragma unroll
    for (int qi = 0; qi < 8; ++qi) {
        const int ql = warp * 8 + qi;
        if (ql >= nq) continue;
        const float inv = 1.f / l_i[qi];
        const size_t ob = (size_t)(start + q0 + ql) * a.ld_out + (size_t)h * HD + lane * DPL;
#pragma unroll
        for (int d = 0; d < DPL; ++d) st_elem(a.out, ob + d, a.dtype, o[qi][d] * inv);
    }
}

template <int HD>
void launch_hd(const AttnArgs& a, cudaStream_t st) {
    const size_t smem = sizeof(float) * (QT * HD + KC * (HD + 1) + KC * HD);
    static bool attr_set = false;
    if (!attr_set) {
        cudaFuncSetAttribute(attention_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
        attr_set = true;
    }
    dim3 grid(a.n_tiles, a.H);
    attention_kernel<HD><<<grid, 256, smem, st>>>(a);
}
}  // namespace

void launch_attention(const AttnArgs& a, cudaStream_t st) {
    if (a.n_tiles == 0) return;
    switch (a.hd) {
        case 32: launch_hd<32>(a, st); break;
        case 64: launch_hd<64>(a, st); break;
        case 128: launch_hd<128>(a, st); break;
        case 256: launch_hd<256>(a, st); break;
        default: break;
    }
}

}  // namespace zo
