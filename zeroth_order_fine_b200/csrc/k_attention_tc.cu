// Packed variable-length causal attention on the 5th-generation tensor cores (head_dim 64
// or 128).
//
// Work items are (128-query tile of one row, head) pairs.  One persistent CTA per
// SM walks its items in turn with its warps specialised:
//   warp 0      TMA producer of Q (three buffers, one per item in flight) and of K
//               (two stages, one per 128-key chunk), 128-byte-swizzled
//   warp 6      TMA producer of V (two stages)
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer:
//                 S = Q K^T      M=128 N=128 K=HD into one of two TMEM S buffers
//                 O (+)= P V     N=HD into one of two TMEM O buffers (one per item in flight)
//               S of the next chunk is issued while the softmax works on this one
//   warps 2..5  softmax and epilogue, one query row per thread (= its TMEM lane):
//               P = exp(S*scale - m) with the causal and row-end masks, written as
//               bf16 in the swizzled K-major layout over the chunk's K buffer, or over
//               the item's Q buffer for its last chunk (so that K buffer frees once S
//               retires); across chunks the softmax is online (running max and sum in
//               registers, the output rescaled in TMEM); an item's O / l goes to memory
//               after the next item's softmax (the item's own P V runs meanwhile)
// So the next items' loads and Q K^T overlap this item's softmax and the last item's store.
// A CTA's items (up to 40) are decoded once into a shared-memory table at the start, so
// no role walks the item order and the row offsets in global memory per item.
// Queries, keys and values arrive by TMA straight from the packed q|k|v rows, each tile
// with the shortest box (32, 64, 96 or 128 rows) that covers it (Qwen3's q/k norm and
// rotary positions were applied beforehand).  Keys past the row's end get zero
// probability (the value rows they meet are finite: other rows' values, or zeros), so a
// query's result depends only on its own row: packing never changes a bit.  Every wait is
// bounded; on expiry the kernel records the error word, drains what it issued, frees its
// tensor memory and returns.
#include <cuda.h>
#include <float.h>

#include "common.cuh"
#include "kernels.h"

namespace zo {

ZO_DEBUG_WORD(debug_word_attention_tc)

namespace {

constexpr int TQ = 128, TK = 128;              // head_dim HD = 64 or 128 (template)
constexpr int ATOM = TQ * 128;                  // bytes of one 64-column swizzle atom block
constexpr int BUF = 2 * ATOM;                   // one [128 x 128] bf16 operand (P is always
                                                // 128 keys wide; Q, K, V fill HD / 64 atoms)
// Q[3] K[2] V[2] buffers, then 23 mbarriers, the TMEM base, the abort flag and the CTA's
// decoded work items (when they fit)
constexpr int ITEM_CACHE = 40;                  // items of a CTA decoded into shared memory
constexpr int SMEM = 7 * BUF + 1024 + 256 + ITEM_CACHE * 32;
constexpr int NTHREADS = 224;                   // Q/K producer, MMA issuer, 4 softmax warps,
                                                // V producer
constexpr long long WAIT_CYCLES = 4000000000ll;
constexpr uint32_t DRAIN_POLLS = 1u << 24;      // drain polls (with back-off) after an abort
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

// 32 contiguous bytes to global memory in one instruction (the address is 32-byte aligned)
__device__ __forceinline__ void st_global_32b(void* p, uint32_t w0, uint32_t w1, uint32_t w2,
                                              uint32_t w3, uint32_t w4, uint32_t w5, uint32_t w6,
                                              uint32_t w7) {
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(w0), "r"(w1),
                 "r"(w2), "r"(w3), "r"(w4), "r"(w5), "r"(w6), "r"(w7)
                 : "memory");
}

__device__ __forceinline__ bool bar_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// try_wait suspending at most ~1 us, so a waiting thread looks at its clock regularly
__device__ __forceinline__ bool bar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(1000u)
        : "memory");
    return ok != 0;
}
// Bounded wait; false when the bound expired (recorded in the error word) or another role
// of the CTA aborted.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_f,
                                         int* err) {
    if (bar_test(bar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (bar_try(bar, parity)) return true;
        if (*abort_f) return false;
        if (clock64() - t0 > WAIT_CYCLES) {   // ~2 s: never arrives
            *abort_f = 1;
            atomicOr(err, 1);
            return false;
        }
    }
}
// Drain after an abort: let an issued copy or MMA land before shared memory goes away.
__device__ __forceinline__ void drain_bar(uint32_t bar, uint32_t parity) {
    for (uint32_t i = 0; i < DRAIN_POLLS && !bar_test(bar, parity); ++i) __nanosleep(128);
}
__device__ __forceinline__ void bar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void bar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}

// S = Q K^T: HD / 16 MMAs (K = HD = HD / 64 swizzle atoms x 4 steps of 16) into TMEM at d_tmem.
template <int HD>
__device__ __forceinline__ void mma_qk(uint32_t d_tmem, uint32_t q, uint32_t k) {
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
        const uint32_t off = (kk >> 2) * ATOM + (kk & 3) * 32;
        const uint32_t acc = kk > 0 ? 1u : 0u;
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(sw128_desc(q + off)), "l"(sw128_desc(k + off)), "r"(kIdesc), "r"(acc)
            : "memory");
    }
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
// P.V: A = P (K-major, keys contiguous), B = V as loaded ([keys x dims], MN-major); N = HD
template <int HD>
constexpr uint32_t idesc_pv() {
    return (kIdesc & ~(0x3Fu << 17)) | ((uint32_t)(HD >> 3) << 17) | (1u << 16);
}

__device__ __forceinline__ void tma_box(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x,
                                        int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

// Maps over the packed q|k|v rows with boxes of 64 columns and 32, 64, 96 or 128 rows: a
// tile is fetched with the shortest box that holds its rows (queries of the tile, keys of
// the chunk), so a short row does not pull its neighbours' rows through L2.  Rows of a
// buffer past the box keep older contents: query rows there are never stored, key columns
// there are masked before the exponential, and the value rows there meet probability 0
// (the value buffers start zeroed and only ever hold value rows, so they stay finite).
struct AttnMaps {
    CUtensorMap box[4];
};
__device__ __forceinline__ int box_of(int rows) {   // rows 1..128 -> box 0..3
    return rows <= 32 ? 0 : rows <= 64 ? 1 : rows <= 96 ? 2 : 3;
}

// One (query tile, head) work item.
struct Item {
    int start, len, q0, nq, kend, n_chunks, h, kvh;
};
static_assert(sizeof(Item) == 32, "item cache slots are 32 bytes");
__device__ __forceinline__ Item make_item(const AttnArgs& a, int i, int tile, int start, int end) {
    Item it;
    const int qt = tile & 0xFFFF;
    it.h = i % a.H;
    it.kvh = it.h / (a.H / a.Hkv);
    it.start = start;
    it.len = end - start;
    it.q0 = qt * TQ;
    it.nq = min(TQ, it.len - it.q0);
    it.kend = min(it.len, it.q0 + TQ);
    it.n_chunks = (it.kend + TK - 1) / TK;
    // (debug build) a query tile past its row's end, an empty span included, becomes an empty
    // item: one fully masked key chunk at token 0 and nothing stored
    if (!ZO_DCHECK(it.q0 < it.len, ZO_DBG_ATTN_TILE)) {
        it.start = it.len = it.q0 = it.nq = it.kend = 0;
        it.n_chunks = 1;
    }
    return it;
}
// Token offsets of the row a tile names; (debug build) a row that is not there is not read
// and gives an empty span
__device__ __forceinline__ void row_span(const int* cu, int n_rows, int tile, int& s, int& e) {
    const int row = tile >> 16;
    if (ZO_DCHECK((unsigned)row < (unsigned)n_rows, ZO_DBG_ATTN_TILE)) {
        s = cu[row];
        e = cu[row + 1];
    } else {
        s = e = 0;
    }
}
__device__ __forceinline__ Item get_item(const AttnArgs& a, int i) {
    const int tile = a.tiles[i / a.H];
    int s, e;
    row_span(a.cu_seqlens, a.n_rows, tile, s, e);
    return make_item(a, i, tile, s, e);
}

// The items of this CTA in order (k-th: blockIdx.x + k * gridDim.x), with their metadata
// fetched two items ahead: the tile of item k + 2 and the row offsets of item k + 1 are
// loaded while item k is being worked on, so no role waits on the dependent loads
// (tile, then the row's offsets) when it moves to its next item.
struct ItemFeed {
    const Item* cache;          // the CTA's items decoded in shared memory, or NULL
    int n_mine;                 // this CTA's item count
    const int* tiles;
    const int* cu;
    AttnArgs shape;             // only H, Hkv and n_rows are read
    int n_items;
    int k;                      // index of cur among this CTA's items
    bool has;                   // cur exists
    Item cur;
    int tile1, s1, e1;          // item k + 1: tile and row offsets (valid when k + 1 exists)
    int tile2;                  // item k + 2: tile
    __device__ __forceinline__ int idx(int kk) const { return blockIdx.x + kk * gridDim.x; }
    __device__ __forceinline__ void init(const AttnArgs& args, int n, const Item* decoded) {
        n_mine = (int)blockIdx.x < n ? (n - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
        cache = n_mine <= ITEM_CACHE ? decoded : nullptr;
        if (cache) {
            k = 0;
            has = n_mine > 0;
            if (has) cur = cache[0];
            return;
        }
        tiles = args.tiles;
        cu = args.cu_seqlens;
        shape.H = args.H;
        shape.Hkv = args.Hkv;
        shape.n_rows = args.n_rows;
        n_items = n;
        k = 0;
        has = idx(0) < n;
        if (has) cur = get_item(args, idx(0));
        tile1 = s1 = e1 = tile2 = 0;
        if (idx(1) < n) {
            tile1 = tiles[idx(1) / shape.H];
            row_span(cu, shape.n_rows, tile1, s1, e1);
        }
        if (idx(2) < n) tile2 = tiles[idx(2) / shape.H];
    }
    __device__ __forceinline__ void advance() {
        if (cache) {
            ++k;
            has = k < n_mine;
            if (has) cur = cache[k];
            return;
        }
        ++k;
        has = idx(k) < n_items;
        if (has) cur = make_item(shape, idx(k), tile1, s1, e1);   // loaded an item ago
        if (idx(k + 1) < n_items) {
            tile1 = tile2;
            row_span(cu, shape.n_rows, tile1, s1, e1);             // used at the next advance
        }
        if (idx(k + 2) < n_items) tile2 = tiles[idx(k + 2) / shape.H];
    }
};

__device__ __forceinline__ float ex2_ftz(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// O (+)= P V: A = P (K-major, keys contiguous) over the chunk's K buffer, B = V as loaded
// ([keys x dims], MN-major); 8 MMAs of K = 16 keys, N = HD.
template <int HD>
__device__ __forceinline__ void mma_pv(uint32_t d_tmem, uint32_t pb, uint32_t vb, bool accum) {
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        const uint32_t acc = (kk > 0 || accum) ? 1u : 0u;
        const uint64_t ad = sw128_desc(pb + (kk >> 2) * ATOM + (kk & 3) * 32);
        const uint64_t bd = sw128_desc_mn(vb + kk * 2048);
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(ad), "l"(bd), "r"(idesc_pv<HD>()), "r"(acc)
            : "memory");
    }
}

// Persistent: CTA b takes items b, b + gridDim.x, ... (dealt longest first by the host).
// Chunks are numbered g = 0, 1, ... across the CTA's items: chunk g uses K/V stage g & 1
// and S buffer g & 1; item k uses Q buffer k % 3 and O buffer k & 1.  Phases follow from the
// counters: the n-th use of a two-slot resource waits parity (n >> 1) & 1.
template <int HD>
__global__ void __launch_bounds__(NTHREADS, 1)
    attention_tc_kernel(const __grid_constant__ AttnMaps tm, AttnArgs a) {
    static_assert(HD == 64 || HD == 128, "head_dim");
    constexpr int NATOM = HD / 64;              // swizzle atoms of a Q, K or V tile
    constexpr uint32_t BOX_BYTES = 32 * HD * 2;   // bytes of 32 rows of a Q, K or V tile
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* g = smem_raw + (base - raw);
    auto Qb = [&](int i) { return base + (uint32_t)(i * BUF); };          // i < 3
    auto Kb = [&](int i) { return base + (uint32_t)((3 + i) * BUF); };
    auto Vb = [&](int i) { return base + (uint32_t)((5 + i) * BUF); };
    const uint32_t bar0 = base + 7 * BUF;
    auto q_full = [&](int i) { return bar0 + 8u * (0 + i); };
    auto q_empty = [&](int i) { return bar0 + 8u * (3 + i); };
    auto k_full = [&](int i) { return bar0 + 8u * (6 + i); };
    auto v_full = [&](int i) { return bar0 + 8u * (8 + i); };
    auto k_empty = [&](int i) { return bar0 + 8u * (10 + i); };
    auto v_empty = [&](int i) { return bar0 + 8u * (12 + i); };
    auto s_full = [&](int i) { return bar0 + 8u * (14 + i); };
    auto p_full = [&](int i) { return bar0 + 8u * (16 + i); };
    auto o_full = [&](int i) { return bar0 + 8u * (18 + i); };
    auto o_free = [&](int i) { return bar0 + 8u * (20 + i); };
    const uint32_t drain = bar0 + 8u * 22;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(g + 7 * BUF + 192);
    volatile int* abort_f = reinterpret_cast<volatile int*>(g + 7 * BUF + 200);
    Item* items = reinterpret_cast<Item*>(g + 7 * BUF + 256);   // ITEM_CACHE decoded items
    // P of a chunk goes over its K buffer, except for an item's last chunk: over the item's
    // Q buffer, whose last reader (that chunk's S) has retired by then.  So the K buffer of an
    // item's last chunk is free as soon as its S retires, and the next K load overlaps the
    // softmax instead of waiting for P V.

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_items = a.n_tiles * a.H;
    const int q_dim = a.H * HD, kv_dim = a.Hkv * HD;
    int* err = &g_attn_error;

    if (tid == 0) {
        for (int i = 0; i < 3; ++i) {
            bar_init(q_full(i), 1);
            bar_init(q_empty(i), 1);
        }
        for (int i = 0; i < 2; ++i) {
            bar_init(k_full(i), 1);
            bar_init(v_full(i), 1);
            bar_init(k_empty(i), 1);
            bar_init(v_empty(i), 1);
            bar_init(s_full(i), 1);
            bar_init(p_full(i), 4);            // one arrival per softmax warp
            bar_init(o_full(i), 1);
            bar_init(o_free(i), 4);
        }
        bar_init(drain, 1);
        *abort_f = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    {
        // the CTA's work items (blockIdx.x + k * gridDim.x) decoded once, when they all fit:
        // each role then reads an item from shared memory instead of the tile -> row-offset
        // loads and the divisions by the head counts
        const int mine = (int)blockIdx.x < n_items
                             ? (n_items - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
        if (mine <= ITEM_CACHE)
            for (int kk = tid; kk < mine; kk += NTHREADS)
                items[kk] = get_item(a, (int)blockIdx.x + kk * (int)gridDim.x);
        // value buffers start at zero: rows a short box leaves untouched are finite
        uint4* vz = reinterpret_cast<uint4*>(g + 5 * BUF);
        for (int i = tid; i < 2 * BUF / 16; i += NTHREADS) vz[i] = make_uint4(0u, 0u, 0u, 0u);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // before the TMA writes
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                         smem_u32(tslot))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tslot;
    auto t_s = [&](int i) { return tmem + (uint32_t)(i * 128); };         // S buffers: cols 0, 128
    auto t_o = [&](int i) { return tmem + (uint32_t)(256 + i * 128); };   // O buffers: 256, 384

    int gq = 0, gcl = 0;                         // producers: Q loads, K (warp 0) or V (warp 6)
                                                 // chunk loads issued
    if (warp == 0 || warp == 6) {
        // ---------------- TMA producers: Q and K (warp 0), V (warp 6) ----------------
        if (lane == 0) {
            const bool vk = warp == 6;
            int& gc = gcl;
            bool ok = true;
            ItemFeed feed;
            feed.init(a, n_items, items);
            for (int k = 0; ok && feed.has; ++k, feed.advance()) {
                const Item it = feed.cur;
                if (!vk) {
                    const int qs = k % 3;
                    if (!wait_bar(q_empty(qs), ((k / 3) & 1) ^ 1u, abort_f, err)) { ok = false; break; }
                    const int qb = box_of(it.nq);
                    bar_expect_tx(q_full(qs), (uint32_t)(qb + 1) * BOX_BYTES);
                    for (int half = 0; half < NATOM; ++half)
                        tma_box(Qb(qs) + half * ATOM, &tm.box[qb], q_full(qs),
                                it.h * HD + half * 64, it.start + it.q0);
                    ++gq;
                }
                const int col = vk ? q_dim + kv_dim + it.kvh * HD : q_dim + it.kvh * HD;
                for (int c = 0; c < it.n_chunks; ++c) {
                    const int st = gc & 1;
                    const uint32_t e = vk ? v_empty(st) : k_empty(st);
                    const uint32_t f = vk ? v_full(st) : k_full(st);
                    if (!wait_bar(e, ((gc >> 1) & 1) ^ 1u, abort_f, err)) { ok = false; break; }
                    const int kb = box_of(min(TK, it.kend - c * TK));
                    bar_expect_tx(f, (uint32_t)(kb + 1) * BOX_BYTES);
                    for (int half = 0; half < NATOM; ++half)
                        tma_box((vk ? Vb(st) : Kb(st)) + half * ATOM, &tm.box[kb], f,
                                col + half * 64, it.start + c * TK);
                    ++gc;
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            // S may run one chunk ahead of P V: chunk gs's S reuses the S buffer of chunk
            // gs - 2, whose P (so its S was read) arrived before P V of gs - 2 was issued
            int sk = 0, sc = 0, gs = 0;          // next S: item counter, chunk, global chunk
            int pk = 0, pc = 0, gp = 0;          // next P V
            ItemFeed s_feed, p_feed;             // the items of the next S and the next P V
            s_feed.init(a, n_items, items);
            p_feed.init(a, n_items, items);
            bool s_more = s_feed.has, p_more = p_feed.has;
            bool ok = true, issued = false;
            long long t0 = clock64();
            while (p_more && ok) {
                bool progress = false;
                if (s_more && gs <= gp + 1 && (sc > 0 || bar_test(q_full(sk % 3), (sk / 3) & 1)) &&
                    bar_test(k_full(gs & 1), (gs >> 1) & 1)) {
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    mma_qk<HD>(t_s(gs & 1), Qb(sk % 3), Kb(gs & 1));
                    tc_commit(s_full(gs & 1));
                    // the item's last chunk keeps its P in the Q buffer: its K is free now
                    if (sc == s_feed.cur.n_chunks - 1) tc_commit(k_empty(gs & 1));
                    issued = progress = true;
                    ++gs;
                    if (++sc == s_feed.cur.n_chunks) {
                        sc = 0;
                        ++sk;
                        s_feed.advance();
                        s_more = s_feed.has;
                    }
                }
                if (gp < gs && bar_test(p_full(gp & 1), (gp >> 1) & 1) &&
                    bar_test(v_full(gp & 1), (gp >> 1) & 1) &&
                    (pc > 0 || bar_test(o_free(pk & 1), ((pk >> 1) & 1) ^ 1u))) {
                    const bool last = pc == p_feed.cur.n_chunks - 1;
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    mma_pv<HD>(t_o(pk & 1), last ? Qb(pk % 3) : Kb(gp & 1), Vb(gp & 1), pc > 0);
                    tc_commit(v_empty(gp & 1));          // V of the chunk is free
                    if (!last) tc_commit(k_empty(gp & 1));   // and its K buffer (held P)
                    issued = progress = true;
                    ++gp;
                    if (++pc == p_feed.cur.n_chunks) {
                        tc_commit(o_full(pk & 1));       // the item's output is complete
                        tc_commit(q_empty(pk % 3));      // and its Q buffer (P) free
                        pc = 0;
                        ++pk;
                        p_feed.advance();
                        p_more = p_feed.has;
                    }
                }
                if (progress) {
                    t0 = clock64();
                } else {
                    __nanosleep(32);                     // leave the issue slots to the softmax
                    if (*abort_f) {
                        ok = false;
                    } else if (clock64() - t0 > WAIT_CYCLES) {
                        *abort_f = 1;
                        atomicOr(err, 1);
                        ok = false;
                    }
                }
            }
            if (issued) {
                // every MMA retired before the CTA moves on (and before TMEM is freed)
                tc_commit(drain);
                drain_bar(drain, 0);
            }
        }
    } else {
        // ---------------- softmax and epilogue (warps 2..5) ----------------
        const int wq = warp & 3;                 // TMEM lane quarter this warp may access
        const int row = wq * 32 + lane;          // query row of the tile = TMEM lane
        const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
        const float sl2 = a.scale * 1.4426950408889634f;
        // output rows start on 32-byte boundaries: 32-byte stores (one sector each)
        const bool st32 = (reinterpret_cast<uintptr_t>(a.out) & 31) == 0 && a.ld_out % 16 == 0;
        // epilogue of item ke: O / l of this thread's query row, once its last P V retired
        auto store_item = [&](int ke, const Item& it, float l) -> bool {
            const int os = ke & 1;
            if (!wait_bar(o_full(os), (ke >> 1) & 1, abort_f, err)) return false;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const float inv = l > 0.f ? 1.f / l : 0.f;
            uint4* o4 = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) +
                                                 (size_t)(it.start + it.q0 + row) * a.ld_out +
                                                 (size_t)it.h * HD);
            const bool store = row < it.nq;
#pragma unroll 1
            for (int cc = 0; cc < HD / 32; ++cc) {
                float v[32];
                tmem_ld32(t_o(os) + lane_addr + cc * 32, v);     // warp-collective: every lane
                auto w = [&](int j) { return pack_bf2(v[2 * j] * inv, v[2 * j + 1] * inv); };
                if (store && st32) {
#pragma unroll
                    for (int k8 = 0; k8 < 2; ++k8)
                        st_global_32b(o4 + cc * 4 + k8 * 2, w(8 * k8), w(8 * k8 + 1), w(8 * k8 + 2),
                                      w(8 * k8 + 3), w(8 * k8 + 4), w(8 * k8 + 5), w(8 * k8 + 6),
                                      w(8 * k8 + 7));
                } else if (store) {
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4)
                        o4[cc * 4 + k4] = make_uint4(w(4 * k4), w(4 * k4 + 1), w(4 * k4 + 2),
                                                     w(4 * k4 + 3));
                }
            }
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            __syncwarp();
            if (lane == 0) bar_arrive(o_free(os));
            return true;
        };
        int pk = -1;                             // item whose output is still to be stored
        Item pit;
        float pl = 0.f;
        int gc = 0;
        bool ok = true;
        ItemFeed feed;
        feed.init(a, n_items, items);
        for (int k = 0; ok && feed.has; ++k, feed.advance()) {
            const Item it = feed.cur;
            const int q = it.q0 + row;
            const int os = k & 1;
            float m = -FLT_MAX, l = 0.f;
            for (int c = 0; c < it.n_chunks; ++c, ++gc) {
                const int st = gc & 1;
                // P over the chunk's K buffer, or over the item's Q buffer for its last chunk
                uint8_t* pbuf = c == it.n_chunks - 1 ? g + (k % 3) * BUF : g + (3 + st) * BUF;
                if (!wait_bar(s_full(st), (gc >> 1) & 1, abort_f, err)) { ok = false; break; }
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const int c0 = c * TK;
                // keys c0 + j with j < lim are visible to this query (causal and row end);
                // column groups of 32 keys that no query of the warp sees are skipped, and so
                // are warps whose queries all lie past the row's end (their P rows are zero)
                const int lim = min(q + 1, it.kend) - c0;
                const int wlim = min(it.q0 + wq * 32 + 32, it.kend) - c0;
                const bool warp_live = it.q0 + wq * 32 < it.len;
                const int ncc = (!warp_live || wlim <= 0) ? 0 : min(4, (wlim + 31) >> 5);
                float sv[4][32];
                // four running maxima: short dependency chains
                float cm[4] = {-FLT_MAX, -FLT_MAX, -FLT_MAX, -FLT_MAX};
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    if (cc < ncc) {
                        tmem_ld32(t_s(st) + lane_addr + cc * 32, sv[cc]);
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            sv[cc][j] = (cc * 32 + j < lim) ? sv[cc][j] : -FLT_MAX;
                            cm[j & 3] = fmaxf(cm[j & 3], sv[cc][j]);
                        }
                    }
                }
                const float cmax = fmaxf(fmaxf(cm[0], cm[1]), fmaxf(cm[2], cm[3]));
                const float m_new = fmaxf(m, cmax);
                // rows whose every key so far is masked keep m = -FLT_MAX and add nothing
                const float alpha = (m > -FLT_MAX) ? exp2f((m - m_new) * sl2) : 0.f;
                // masked scores are -FLT_MAX, so exp2(s*sl2 - ms) underflows to exactly 0
                const float ms = (m_new > -FLT_MAX) ? m_new * sl2 : 0.f;
                // eight running sums, added in a fixed tree: short dependency chains
                float cs[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint32_t w[16];
                    if (cc < ncc) {
#pragma unroll
                        for (int j = 0; j < 32; j += 2) {
                            const float p0 = ex2_ftz(fmaf(sv[cc][j], sl2, -ms));
                            const float p1 = ex2_ftz(fmaf(sv[cc][j + 1], sl2, -ms));
                            cs[j & 7] += p0;
                            cs[(j + 1) & 7] += p1;
                            w[j / 2] = pack_bf2(p0, p1);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j) w[j] = 0u;
                    }
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4)
                        *reinterpret_cast<uint4*>(pbuf + sw_off(row, cc * 4 + k4)) =
                            make_uint4(w[4 * k4], w[4 * k4 + 1], w[4 * k4 + 2], w[4 * k4 + 3]);
                }
                l = l * alpha + (((cs[0] + cs[1]) + (cs[2] + cs[3])) + ((cs[4] + cs[5]) + (cs[6] + cs[7])));
                m = m_new;
                if (c > 0) {
                    // the running output stays in TMEM: once the previous chunk's P V has
                    // retired, rescale it by exp(m_old - m_new); this chunk's P V adds on top
                    const int pv = gc - 1;
                    if (!wait_bar(v_empty(pv & 1), (pv >> 1) & 1, abort_f, err)) { ok = false; break; }
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll 1
                    for (int cc = 0; cc < HD / 32; ++cc) {
                        float v[32];
                        tmem_ld32(t_o(os) + lane_addr + cc * 32, v);
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] *= alpha;
                        tmem_st32(t_o(os) + lane_addr + cc * 32, v);
                    }
                    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                }
                // P is in shared memory (generic proxy -> the tensor core's async proxy)
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
                __syncwarp();
                if (lane == 0) bar_arrive(p_full(st));
            }
            if (!ok) break;
            // the previous item's output goes out now, after this item's softmax: its P V ran
            // meanwhile, so the wait below rarely stalls
            if (pk >= 0 && !store_item(pk, pit, pl)) { ok = false; break; }
            pk = k;
            pit = it;
            pl = l;
        }
        if (ok && pk >= 0) store_item(pk, pit, pl);
    }
    __syncthreads();                             // every role has left its loop
    if (*abort_f && (warp == 0 || warp == 6) && lane == 0) {
        // an aborted CTA lets every copy still in flight land before its shared memory goes
        // away: the newest loads of each kind (older ones were consumed, so had landed)
        if (warp == 0)
            for (int i = gq - 1; i >= 0 && i >= gq - 3; --i) drain_bar(q_full(i % 3), (i / 3) & 1);
        for (int i = gcl - 1; i >= 0 && i >= gcl - 2; --i)
            drain_bar(warp == 0 ? k_full(i & 1) : v_full(i & 1), (i >> 1) & 1);
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem)
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
    return a.dtype == E_BF16 && (a.hd == 64 || a.hd == 128) && a.ld_qkv % 8 == 0 &&
           a.ld_out % 8 == 0 &&
           a.n_tokens > 0 && attn_encode_fn() != nullptr &&
           (reinterpret_cast<uintptr_t>(a.qkv) & 15) == 0 &&
           (reinterpret_cast<uintptr_t>(a.out) & 15) == 0;
}

bool launch_attention_tc(const AttnArgs& a, cudaStream_t st) {
    if (a.n_tiles == 0 || a.n_tokens <= 0) return true;
    if (a.hd != 64 && a.hd != 128) return false;
    static cudaError_t attr[2] = {cudaErrorNotReady, cudaErrorNotReady};
    cudaError_t& at = attr[a.hd == 128];
    if (at == cudaErrorNotReady)
        at = a.hd == 128 ? cudaFuncSetAttribute(attention_tc_kernel<128>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM)
                         : cudaFuncSetAttribute(attention_tc_kernel<64>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (at != cudaSuccess) return false;
    // maps over the packed [T x ld_qkv] q|k|v rows: 64-column boxes of 32, 64, 96 and 128
    // rows, 128-byte swizzle, rows past T read as zero
    AttnMaps tm;
    EncodeTiledFn fn = attn_encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)a.ld_qkv, (cuuint64_t)a.n_tokens};
    const cuuint64_t strides[1] = {(cuuint64_t)a.ld_qkv * 2};
    const cuuint32_t es[2] = {1, 1};
    for (int b = 0; b < 4; ++b) {
        const cuuint32_t box[2] = {64, (cuuint32_t)(32 * (b + 1))};
        if (fn(&tm.box[b], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.qkv), dims,
               strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    const long long items = (long long)a.n_tiles * a.H;
    if (items > 0x7fffffffLL) return false;
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
            sms = 148;
    }
    const unsigned grid = (unsigned)(items < sms ? items : sms);
    if (a.hd == 128)
        attention_tc_kernel<128><<<grid, NTHREADS, SMEM, st>>>(tm, a);
    else
        attention_tc_kernel<64><<<grid, NTHREADS, SMEM, st>>>(tm, a);
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
