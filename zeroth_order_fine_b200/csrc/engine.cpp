// Engine behind the C ABI (include/zo.h): the handle, the persistent
// factored bank, the probe plan, the packed-batch scoring schedule and the
// estimator / update launches.  Host work is limited to building the small
// per-call metadata (row offsets, signs, scored spans) and queueing kernels
// on the handle's stream.
//
// Bank layout.  Per layer the decoder runs four fused GEMMs ("groups"):
// [q|k|v], o, FFN-in (OPT fc1; Qwen3 [gate|up]) and FFN-out.  For a group
// with n targeted matrices the shrink factors live in one fp32 buffer
// FT [(n*r*(1+max_slots)) x d_in]:
//     rows [m*r, m*r+r)                      U_t^T of target m (drawn each step)
//     rows [n*r*(1+j) + m*r, ... + r)        A_j^T of target m, bank slot j
// and the expand factors in one extension operand EB [N x kcap] (model dtype):
//     cols [m*r, m*r+r)                      V of the current window (rows of m)
//     cols [n*r*(1+j) + m*r, ... + r)        V_j of slot j
// zero elsewhere.  Scoring a group is then
//     S  = x FT^T,  with the U columns scaled by (row sign * eps)     (shrink)
//     y  = x W^T + S EB^T + b                                         (one GEMM)
// = x (W^T + sum_j A_j V_j^T + s eps U_t V_k^T) + b: the candidate states
// theta +/- eps U V^T and the banked updates are never formed densely
// ("Zeroth-Order Fine-Tuning Was an Inference Workload All Along", section
// "The System Reorganization"; "Inference-Native Zeroth-Order Optimization",
// abstract: factorised side states, persistent banks, frozen base weights).
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>   // header-only: ranges cost nothing unless a profiler is attached

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <functional>
#include <string>
#include <vector>

#include "../../include/zo.h"
#include "../../include/zo_ops.h"
#include "kernels.h"
#include "rng.cuh"

using namespace zo;

namespace {

enum GroupKind { G_QKV = 0, G_O = 1, G_IN = 2, G_OUT = 3 };
constexpr int kMaxTargetsPerGroup = 3;

struct Group {
    int N = 0, K = 0;
    const void* W = nullptr;     // [N x K]
    const float* bias = nullptr;
    int n_t = 0;                 // targeted matrices in this group
    int interleave = 0;          // [gate|up] rows interleaved in 128-row blocks (SwiGLU epilogue)
    int mats[kMaxTargetsPerGroup] = {0, 0, 0};
    int row_off[kMaxTargetsPerGroup] = {0, 0, 0};
    int d_out[kMaxTargetsPerGroup] = {0, 0, 0};
    float* FT = nullptr;         // shrink factors (fp32)
    void* FTb = nullptr;         // bf16 mirror of FT (bf16 models): the shrink GEMM operand
    void* EB = nullptr;          // expand factors (model dtype)
    float* Vcur[kMaxTargetsPerGroup] = {nullptr, nullptr, nullptr};
    uint8_t* Wq = nullptr;       // E4M3 copy of W (fp8 option, norm-fed groups)
    float* sw = nullptr;         // its per-row (output channel) scales
};

struct Layer {
    Group g[4];
    zo_layer_weights w;
};

struct PhaseTimer {
    static constexpr int kRing = 64;
    cudaEvent_t a[kRing], b[kRing];
    int head = 0, tail = 0;   // [tail, head) pending
    double total_ms = 0.0;
    bool init = false;
    nvtxRangeId_t range = 0;  // the phase's open NVTX range
};

// Per-launch GEMM timing (options.profile): event pairs in a ring, harvested
// without blocking where possible.
struct GemmProfiler {
    static constexpr int kRing = 8192;
    std::vector<cudaEvent_t> a, b;
    std::vector<double> flops;
    std::vector<char> tc;
    long long head = 0, tail = 0;
    uint64_t launches = 0, tc_launches = 0;
    double ms = 0.0, fl = 0.0, tc_ms = 0.0, tc_fl = 0.0;
    bool on = false;
};

const char* kNoErr = "no error";

}  // namespace

struct zo_plan {
    zo_handle* h;
    uint64_t step;
    float eps;
    bool scored;
    int B;          // prompts of the last score
};

struct zo_handle {
    zo_model_desc desc;
    zo_options opt;
    zo_weights wts;
    std::vector<zo_layer_weights> lw;
    cudaStream_t st = nullptr;
    int dt = E_F32;               // element type of matrices / activations
    int q_dim = 0, kv_dim = 0, n_qkv = 0;
    std::vector<Layer> layers;
    // fused weights owned by the handle
    std::vector<void*> owned;
    // activations
    float* resid = nullptr;
    float *rope_cos = nullptr, *rope_sin = nullptr;   // Qwen3 rotary tables [max_pos x hd/2]
    void *xn = nullptr, *qkv = nullptr, *att = nullptr, *act = nullptr, *gu = nullptr;
    void* ext = nullptr;          // shrink output S (model dtype) [max_tokens x kcap]
    int kcap = 0;                 // columns of FT rows / EB / ext allocated
    void* hs = nullptr;           // scored hidden states
    // generation queries (options.max_new > 0)
    void* kv_cache = nullptr;     // per layer [kv_rows x 2 kv_dim] in the model dtype
    size_t kv_rows = 0;
    int* part_arg = nullptr;      // LSE partials: argmax column per (row, tile)
    float* splitk_ws = nullptr;   // decode GEMMs' split-K slices
    size_t splitk_floats = 0;
    int *gen_tok = nullptr, *gen_last = nullptr, *gen_lens = nullptr;
    float* gen_lp = nullptr;
    float *pmax = nullptr, *psum = nullptr, *tgt = nullptr, *logprob = nullptr;
    int lse_tiles = 0;
    double* L_row = nullptr;
    int *tok_id = nullptr, *tok_pos = nullptr, *tok_sign = nullptr, *tok_row = nullptr;
    int *sc_tok = nullptr, *sc_tgt = nullptr;
    int* meta = nullptr;          // device metadata
    int* meta_h = nullptr;        // pinned staging
    size_t meta_ints = 0;
    cudaEvent_t meta_ev = nullptr;
    int max_tiles = 0;
    // estimator
    double* sums = nullptr;
    double* c_dev = nullptr;
    int* flag_dev = nullptr;
    int* err_dev = nullptr;
    // generator / window / update job tables
    GenJob* genU_d = nullptr; int n_genU = 0; int maxU_pairs = 0;
    GenJob* genU32_d = nullptr;   // bf16 models: fp32 U jobs, run only by zo_read_factors
    // bank update: coefficients of the current slot since replay_from (its opening step), or
    // replay_from = -1 when the slot must be read-modify-written (loaded state, or replay
    // too costly for the factor sizes: replay_enabled)
    float* coef_hist = nullptr;
    long long replay_from = -1;
    bool replay_enabled = false;
    GenJob* genV_d = nullptr; int n_genV = 0; int maxV_pairs = 0;
    WindowJob* win_d = nullptr; int n_win = 0;
    UpdateJob* upd_d = nullptr; int n_upd = 0; int max_upd = 0;
    void* jobs_h = nullptr;       // pinned staging for window / update jobs
    size_t jobs_bytes = 0;
    cudaEvent_t jobs_ev = nullptr;
    // run state
    uint64_t step = 0;
    int n_slots = 0;
    std::vector<int64_t> slot_window;
    zo_plan plan;
    bool have_plan = false;
    float mezo_scale = 1.f;
    bool use_tc = false;
    bool swiglu_fused = false;    // Qwen3 FFN-in GEMM writes silu(gate) * up directly
    bool qknr_fused = false;      // Qwen3 q|k|v GEMM applies q/k RMSNorm and RoPE itself
    bool fp8 = false;             // norm-fed base GEMMs in E4M3 (zo_options.fp8)
    uint8_t* xq = nullptr;        // E4M3 rows of the norm output
    float* sx = nullptr;          // their per-token scales
    // whole-step CUDA graph (zo_step_graph): captured for one batch layout, eps, lr,
    // set of buffers and bank slot count; replayed while those stay the same
    struct StepGraph {
        cudaStream_t cap = nullptr;           // capture stream (the handle's may be the legacy one)
        cudaGraphExec_t exec = nullptr;
        int* meta = nullptr;                  // device metadata of the captured layout
        uint64_t* step_dev = nullptr;         // the step the next replay generates U for
        uint64_t step_next = ~0ull;           // value *step_dev holds once queued work has run
        std::vector<int> lens, tls;
        const void* tok = nullptr;
        float *Lp = nullptr, *Lm = nullptr;
        float eps = 0.f, lr = 0.f;
        int slots = -1;
        long long replay_from = -2;           // the bank update's mode baked into the graph
        long long T = 0, S = 0;
        uint64_t launches = 0;                // kernels per replay
        uint64_t captures = 0, replays = 0;
    } graph;
    bool capturing = false;       // launches are being recorded into a graph
    // stats
    zo_stats_t stats;
    PhaseTimer tm[3];
    GemmProfiler prof;
    uint64_t bytes_per_U = 0, bytes_per_window = 0;
    uint64_t a_elems = 0;         // accumulator elements updated per step (all targets)
    uint64_t dense_bytes = 0, dense_bytes_targets = 0;
    std::string err;
    int err_code = 0;
    // allocation failure injection (ZO_FAIL_ALLOC_AT): device allocations made so far and
    // the 1-based index of the one to fail (0: none)
    long long n_allocs = 0, fail_alloc_at = 0;
};

static std::string g_create_err = kNoErr;

#define FAIL(h, code, msg)                         \
    do {                                           \
        if (h) { (h)->err = (msg); (h)->err_code = (code); } \
        return (code);                             \
    } while (0)

#define CK(h, call)                                                            \
    do {                                                                       \
        cudaError_t e_ = (call);                                               \
        if (e_ != cudaSuccess) {                                               \
            if (h) { (h)->err = std::string(#call ": ") + cudaGetErrorString(e_); \
                     (h)->err_code = ZO_ERR_CUDA; }                            \
            return e_ == cudaErrorMemoryAllocation ? ZO_ERR_OOM : ZO_ERR_CUDA; \
        }                                                                      \
    } while (0)

namespace {

size_t esize(int t) { return t == E_F32 ? 4 : 2; }

bool layer_targeted(const zo_targets& t, int l) {
    if (l < 64) return (t.layer_mask_lo >> l) & 1ull;
    if (l < 128) return (t.layer_mask_hi >> (l - 64)) & 1ull;
    return false;
}

int dev_alloc(zo_handle* h, void** p, size_t bytes) {
    if (bytes == 0) bytes = 16;
    if (++h->n_allocs == h->fail_alloc_at) {
        *p = nullptr;
        h->err = "device allocation " + std::to_string(h->n_allocs) +
                 " refused by ZO_FAIL_ALLOC_AT (injected out-of-memory)";
        h->err_code = ZO_ERR_OOM;
        return ZO_ERR_OOM;
    }
    cudaError_t e = cudaMalloc(p, bytes);
    if (e != cudaSuccess) {
        h->err = std::string("cudaMalloc: ") + cudaGetErrorString(e);
        h->err_code = ZO_ERR_OOM;
        return ZO_ERR_OOM;
    }
    h->owned.push_back(*p);
    return ZO_OK;
}

#define ALLOC(h, ptr, bytes)                                            \
    do {                                                                \
        void* p_ = nullptr;                                             \
        int rc_ = dev_alloc(h, &p_, (bytes));                           \
        if (rc_) return rc_;                                            \
        (ptr) = reinterpret_cast<decltype(ptr)>(p_);                    \
    } while (0)

void matrix_dims(const zo_model_desc& d, int m, int* di, int* dout) {
    const int q = d.n_heads * d.head_dim, kv = d.n_kv_heads * d.head_dim;
    switch (m) {
        case ZO_MAT_Q: *di = d.d_model; *dout = q; break;
        case ZO_MAT_K: case ZO_MAT_V: *di = d.d_model; *dout = kv; break;
        case ZO_MAT_O: *di = q; *dout = d.d_model; break;
        case ZO_MAT_GATE: case ZO_MAT_UP: *di = d.d_model; *dout = d.d_ffn; break;
        default: *di = d.d_ffn; *dout = d.d_model; break;
    }
}

void timer_harvest(PhaseTimer& t, bool wait) {
    while (t.tail != t.head) {
        const int i = t.tail % PhaseTimer::kRing;
        if (wait) cudaEventSynchronize(t.b[i]);
        else if (cudaEventQuery(t.b[i]) != cudaSuccess) break;
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, t.a[i], t.b[i]) == cudaSuccess) t.total_ms += ms;
        t.tail++;
    }
}

void prof_harvest(GemmProfiler& p, bool wait) {
    while (p.tail != p.head) {
        const int i = (int)(p.tail % GemmProfiler::kRing);
        if (wait) cudaEventSynchronize(p.b[i]);
        else if (cudaEventQuery(p.b[i]) != cudaSuccess) break;
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, p.a[i], p.b[i]) == cudaSuccess) {
            p.ms += ms;
            p.fl += p.flops[i];
            p.launches++;
            if (p.tc[i]) {
                p.tc_ms += ms;
                p.tc_fl += p.flops[i];
                p.tc_launches++;
            }
        }
        p.tail++;
    }
}

int prof_begin(zo_handle* h);
void prof_end(zo_handle* h, int slot, double flops, bool tc);

// Each phase (plan, score, step) is also an NVTX range, so a timeline profiler shows the
// step's structure on the host thread.
void timer_begin(zo_handle* h, int ph) {
    static const char* const kPhase[3] = {"zo_probe_plan", "zo_score", "zo_step"};
    PhaseTimer& t = h->tm[ph];
    t.range = nvtxRangeStartA(kPhase[ph]);   // start/end pairs: an error return leaves no stack
    if (!t.init) {
        for (int i = 0; i < PhaseTimer::kRing; ++i) {
            cudaEventCreate(&t.a[i]);
            cudaEventCreate(&t.b[i]);
        }
        t.init = true;
    }
    timer_harvest(t, false);
    if (t.head - t.tail >= PhaseTimer::kRing) timer_harvest(t, true);
    cudaEventRecord(t.a[t.head % PhaseTimer::kRing], h->st);
}

void timer_end(zo_handle* h, int ph) {
    PhaseTimer& t = h->tm[ph];
    cudaEventRecord(t.b[t.head % PhaseTimer::kRing], h->st);
    t.head++;
    nvtxRangeEnd(t.range);
}

int prof_begin(zo_handle* h) {
    GemmProfiler& p = h->prof;
    if (!p.on || h->capturing) return -1;
    if (p.head - p.tail >= GemmProfiler::kRing) prof_harvest(p, true);
    const int i = (int)(p.head % GemmProfiler::kRing);
    cudaEventRecord(p.a[i], h->st);
    return i;
}

void prof_end(zo_handle* h, int slot, double flops, bool tc) {
    if (slot < 0) return;
    GemmProfiler& p = h->prof;
    cudaEventRecord(p.b[slot], h->st);
    p.flops[slot] = flops;
    p.tc[slot] = tc ? 1 : 0;
    p.head++;
}

// GEMM dispatch: the tcgen05 kernel for bf16 shapes it takes, else CUDA cores.
// algo_flops: the launch's algorithmic FLOPs (for the live roofline).
int run_gemm(zo_handle* h, const GemmArgs& g, double algo_flops) {
    const bool tc = h->use_tc && gemm_tc_supported(g);
    if (g.epi == EPI_SWIGLU && !tc) FAIL(h, ZO_ERR_UNSUPPORTED, "fused SwiGLU needs tensor cores");
    if (g.epi == EPI_QKNR && !tc)
        FAIL(h, ZO_ERR_UNSUPPORTED, "fused q/k norm and rotary positions need the SM-pair kernel");
    const int slot = prof_begin(h);
    if (tc) {
        int e = gemm_tc(g, h->st);
        if (e) FAIL(h, ZO_ERR_CUDA, "tcgen05 GEMM launch failed");
    } else {
        gemm_simt(g, h->st);
        h->stats.cuda_core_gemm_launches++;
    }
    prof_end(h, slot, algo_flops, tc);
    h->stats.kernel_launches++;
    return ZO_OK;
}

// State-transition bytes of the bank update at step t: the accumulator written in fp32 (and
// its bf16 mirror); read as well unless it is rebuilt from the slot's coefficients, whose
// history is then read and this step's written.
uint64_t update_bytes(const zo_handle* h, uint64_t t) {
    const uint64_t mirror = h->dt == E_BF16 ? 2 : 0;
    if (h->replay_from >= 0)
        return h->a_elems * (4 + mirror) + 4 * (t - (uint64_t)h->replay_from + 1);
    return h->a_elems * (8 + mirror);
}

// ---- window opening: V of the window into EB, slot accumulator zeroed ------------------
int open_window(zo_handle* h, uint64_t step) {
    const int k = h->n_slots;
    if (k >= h->opt.max_slots)
        FAIL(h, ZO_ERR_UNSUPPORTED, "bank full: more lazy windows than max_slots");
    const int r = h->opt.rank;
    // V of the window for every target
    launch_gen_factors(h->genV_d, h->n_genV, h->maxV_pairs, h->opt.run_seed, step, nullptr,
                       (uint64_t)h->opt.lazy_interval, h->mezo_scale,
                       h->opt.targets.scale_mode == ZO_SCALE_MEZO, h->st);
    // staging: window jobs then update jobs
    CK(h, cudaEventSynchronize(h->jobs_ev));
    WindowJob* wj = static_cast<WindowJob*>(h->jobs_h);
    UpdateJob* uj = reinterpret_cast<UpdateJob*>(wj + h->n_win);
    int nw = 0, nu = 0, max_n = 0;
    for (int l = 0; l < (int)h->layers.size(); ++l)
        for (auto& G : h->layers[l].g)
            for (int t = 0; t < G.n_t; ++t) {
                WindowJob w;
                w.V = G.Vcur[t];
                w.EB = G.EB;
                const size_t a_off = (size_t)(G.n_t * r * (1 + k) + t * r) * G.K;
                w.A = G.FT + a_off;
                w.A_bf = G.FTb ? static_cast<char*>(G.FTb) + a_off * 2 : nullptr;
                w.eb_type = h->dt;
                w.ldb = h->kcap;
                w.row0 = G.row_off[t];
                w.d_out = G.d_out[t];
                w.d_in = G.K;
                w.r = r;
                w.col_dir = t * r;
                w.col_slot = G.n_t * r * (1 + k) + t * r;
                w.interleave = G.interleave;
                w.row_div = G.sw;               // E4M3 groups: V / s_w per expand row
                wj[nw++] = w;
                UpdateJob u;
                u.A = w.A;
                u.A_bf = w.A_bf;
                u.layer = l;
                u.matrix = G.mats[t];
                u.dim = G.K;
                u.r = r;
                u.ld = G.K;
                max_n = std::max(max_n, (r * G.K + 1) / 2);
                uj[nu++] = u;
            }
    CK(h, cudaMemcpyAsync(h->win_d, wj, sizeof(WindowJob) * nw, cudaMemcpyHostToDevice, h->st));
    CK(h, cudaMemcpyAsync(h->upd_d, uj, sizeof(UpdateJob) * nu, cudaMemcpyHostToDevice, h->st));
    CK(h, cudaEventRecord(h->jobs_ev, h->st));
    h->max_upd = max_n;
    launch_open_window(h->win_d, nw, h->st);
    h->stats.kernel_launches += 2;
    h->n_slots = k + 1;
    h->slot_window.push_back((int64_t)(step / (uint64_t)h->opt.lazy_interval));
    // the new slot starts at zero: from here its updates can be replayed from coefficients
    h->replay_from = h->replay_enabled ? (long long)step : -1;
    h->stats.state_transition_bytes += h->bytes_per_window;
    return ZO_OK;
}

// The four fused GEMM groups of a layer, with its targets.
void build_groups(zo_handle* h, int l, Layer& L) {
    const zo_model_desc& d = h->desc;
    const zo_layer_weights& w = L.w;
    const bool tl = layer_targeted(h->opt.targets, l);
    const uint32_t mm = h->opt.targets.matrix_mask;
    auto add = [&](Group& G, int m, int off) {
        if (!tl || !((mm >> m) & 1u)) return;
        int di, dout;
        matrix_dims(d, m, &di, &dout);
        G.mats[G.n_t] = m;
        G.row_off[G.n_t] = off;
        G.d_out[G.n_t] = dout;
        G.n_t++;
    };
    Group& q = L.g[G_QKV];
    q.N = h->n_qkv; q.K = d.d_model;
    add(q, ZO_MAT_Q, 0); add(q, ZO_MAT_K, h->q_dim); add(q, ZO_MAT_V, h->q_dim + h->kv_dim);
    Group& o = L.g[G_O];
    o.N = d.d_model; o.K = h->q_dim; o.W = w.w[ZO_MAT_O]; o.bias = w.b[ZO_MAT_O];
    add(o, ZO_MAT_O, 0);
    Group& in = L.g[G_IN];
    in.K = d.d_model;
    if (d.arch == ZO_ARCH_OPT) {
        in.N = d.d_ffn; in.W = w.w[ZO_MAT_UP]; in.bias = w.b[ZO_MAT_UP];
        add(in, ZO_MAT_UP, 0);
    } else {
        in.N = 2 * d.d_ffn;
        if (h->swiglu_fused) {
            // rows interleaved: gate block b at rows 256 b .. + 128, up block b right after
            in.interleave = 1;
            add(in, ZO_MAT_GATE, 0); add(in, ZO_MAT_UP, 128);
        } else {
            add(in, ZO_MAT_GATE, 0); add(in, ZO_MAT_UP, d.d_ffn);
        }
    }
    Group& out = L.g[G_OUT];
    out.N = d.d_model; out.K = d.d_ffn; out.W = w.w[ZO_MAT_DOWN]; out.bias = w.b[ZO_MAT_DOWN];
    add(out, ZO_MAT_DOWN, 0);
}

int check_desc(const zo_model_desc* d, const zo_weights* w, const zo_options* o) {
    if (!d || !w || !o) return 1;
    if (d->arch != ZO_ARCH_OPT && d->arch != ZO_ARCH_QWEN3) return 1;
    if (d->n_layers <= 0 || d->n_layers > 128 || d->d_model <= 0 || d->n_heads <= 0) return 1;
    if (d->n_kv_heads <= 0 || d->n_heads % d->n_kv_heads) return 1;
    if (d->head_dim != 32 && d->head_dim != 64 && d->head_dim != 128 && d->head_dim != 256)
        return 2;
    if (d->d_model % 8 || d->d_ffn % 8 || (d->n_heads * d->head_dim) % 8) return 2;
    if (d->arch == ZO_ARCH_QWEN3 && d->head_dim < 64) return 2;     // q/k norm + rotary kernel
    if (d->d_model > 12288) return 2;
    if (d->vocab <= 0 || d->d_ffn <= 0) return 1;
    if (d->dtype != ZO_DTYPE_FP32 && d->dtype != ZO_DTYPE_BF16) return 1;
    if (d->max_pos <= 0 || (d->arch == ZO_ARCH_OPT && !w->pos_embed)) return 1;
    if (!w->tok_embed || !w->final_w || !w->layers) return 1;
    if (!d->tie_lm_head && !w->lm_head) return 1;
    if (o->lazy_interval < 1 || o->rank < 1 || o->rank > 256 || o->max_slots < 1) return 1;
    if (o->max_tokens < 1 || o->max_rows < 1 || o->max_scored < 1) return 1;
    if (o->targets.scale_mode != ZO_SCALE_LOZO && o->targets.scale_mode != ZO_SCALE_MEZO) return 1;
    if (o->targets.matrix_mask & ~0x7Fu) return 1;
    if (o->impl != 0 && o->impl != 1) return 1;
    if (o->profile != 0 && o->profile != 1) return 1;
    if (o->fp8 != 0 && o->fp8 != 1) return 1;
    if (o->max_new < 0 || o->max_new > 4096) return 1;
    if (o->max_new > 0 && d->n_heads / d->n_kv_heads > 8) return 2;   // decode attention groups
    if (o->fp8 && (d->dtype != ZO_DTYPE_BF16 || o->impl != 0 || !norm_fp8_supported(d->d_model) ||
                   d->d_model % 16 || (d->n_heads + 2 * d->n_kv_heads) * d->head_dim <= 128 ||
                   d->d_ffn <= 64))
        return 2;
    if (d->arch == ZO_ARCH_OPT && (o->targets.matrix_mask & (1u << ZO_MAT_GATE))) return 1;
    return 0;
}

}  // namespace

// =====================================================================================
extern "C" {

const char* zo_last_error(const zo_handle* h) {
    if (!h) return g_create_err.c_str();
    return h->err.empty() ? kNoErr : h->err.c_str();
}

int zo_create(const zo_model_desc* desc, const zo_weights* weights, const zo_options* options,
              zo_handle** out) {
    if (!out) return ZO_ERR_ARG;
    *out = nullptr;
    const int chk = check_desc(desc, weights, options);
    if (chk) {
        g_create_err = chk == 2 ? "model shape outside the supported set" : "invalid model/options";
        return chk == 2 ? ZO_ERR_UNSUPPORTED : ZO_ERR_ARG;
    }
    zo_handle* h = new zo_handle();
    if (const char* fa = std::getenv("ZO_FAIL_ALLOC_AT")) h->fail_alloc_at = std::atoll(fa);
    h->desc = *desc;
    h->opt = *options;
    h->wts = *weights;
    h->lw.assign(weights->layers, weights->layers + desc->n_layers);
    h->wts.layers = h->lw.data();
    h->st = static_cast<cudaStream_t>(options->stream);
    h->dt = desc->dtype == ZO_DTYPE_BF16 ? E_BF16 : E_F32;
    h->step = options->start_step;
    h->mezo_scale = (float)(1.0 / std::sqrt((double)options->rank));
    memset(&h->stats, 0, sizeof(h->stats));
    const zo_model_desc& d = *desc;
    h->q_dim = d.n_heads * d.head_dim;
    h->kv_dim = d.n_kv_heads * d.head_dim;
    h->n_qkv = h->q_dim + 2 * h->kv_dim;
    const int r = options->rank;
    const size_t es = esize(h->dt);
    const int maxT = options->max_tokens, maxR = options->max_rows, maxS = options->max_scored;

    auto fail = [&](int rc) {
        g_create_err = h->err;
        zo_destroy(h);
        return rc;
    };
#define CRC(x)                          \
    do {                                \
        int rc__ = (x);                 \
        if (rc__) return fail(rc__);    \
    } while (0)

    h->use_tc = h->dt == E_BF16 && options->impl == 0;
    h->fp8 = options->fp8 == 1;
    h->swiglu_fused = h->use_tc && d.arch == ZO_ARCH_QWEN3 && d.d_ffn % 128 == 0;
    // the q|k|v GEMM epilogue applies the q/k norm and rotary positions when it can read
    // the norm weights as 16-byte vectors (head_dim 128, more than one head)
    h->qknr_fused = h->use_tc && d.arch == ZO_ARCH_QWEN3 && d.head_dim == 128 &&
                    h->n_qkv > 128;
    for (int l = 0; l < d.n_layers && h->qknr_fused; ++l) {
        const zo_layer_weights& lw = weights->layers[l];
        if ((reinterpret_cast<uintptr_t>(lw.q_norm) & 15) || (reinterpret_cast<uintptr_t>(lw.k_norm) & 15))
            h->qknr_fused = false;
    }
    // layers, fused weights and bank buffers
    h->layers.resize(d.n_layers);
    int max_nt = 0;
    for (int l = 0; l < d.n_layers; ++l) {
        Layer& L = h->layers[l];
        L.w = h->lw[l];
        build_groups(h, l, L);
        for (auto& G : L.g) max_nt = std::max(max_nt, G.n_t);
    }
    // extension width: U block + one block per slot, rounded to the 64-column K tile
    h->kcap = ((max_nt * r * (1 + options->max_slots) + 63) / 64) * 64;
    if (max_nt == 0) h->kcap = 0;

    auto fused_copy = [&](Layer& L, Group& G, const int* mats, int nm) -> int {
        void* W = nullptr;
        int rc = dev_alloc(h, &W, (size_t)G.N * G.K * es);
        if (rc) return rc;
        size_t off = 0;
        for (int i = 0; i < nm; ++i) {
            int di, dout;
            matrix_dims(d, mats[i], &di, &dout);
            if (!L.w.w[mats[i]]) { h->err = "missing weight matrix"; return ZO_ERR_ARG; }
            cudaError_t e = cudaMemcpyAsync(static_cast<char*>(W) + off * es, L.w.w[mats[i]],
                                            (size_t)dout * di * es, cudaMemcpyDeviceToDevice, h->st);
            if (e != cudaSuccess) { h->err = cudaGetErrorString(e); return ZO_ERR_CUDA; }
            off += (size_t)dout * di;
        }
        G.W = W;
        if (d.arch == ZO_ARCH_OPT && G.N && L.w.b[mats[0]]) {
            float* b = nullptr;
            rc = dev_alloc(h, reinterpret_cast<void**>(&b), (size_t)G.N * 4);
            if (rc) return rc;
            size_t bo = 0;
            for (int i = 0; i < nm; ++i) {
                int di, dout;
                matrix_dims(d, mats[i], &di, &dout);
                cudaMemcpyAsync(b + bo, L.w.b[mats[i]], (size_t)dout * 4, cudaMemcpyDeviceToDevice,
                                h->st);
                bo += dout;
            }
            G.bias = b;
        }
        return ZO_OK;
    };

    for (int l = 0; l < d.n_layers; ++l) {
        Layer& L = h->layers[l];
        const int qkv[3] = {ZO_MAT_Q, ZO_MAT_K, ZO_MAT_V};
        CRC(fused_copy(L, L.g[G_QKV], qkv, 3));
        if (d.arch == ZO_ARCH_QWEN3 && h->swiglu_fused) {
            Group& G = L.g[G_IN];
            void* W = nullptr;
            CRC(dev_alloc(h, &W, (size_t)G.N * G.K * es));
            const size_t blk = (size_t)128 * G.K * es;          // 128 rows of one matrix
            for (int half = 0; half < 2; ++half) {
                const void* src = L.w.w[half == 0 ? ZO_MAT_GATE : ZO_MAT_UP];
                if (!src) { h->err = "missing gate/up weights"; return fail(ZO_ERR_ARG); }
                CK(h, cudaMemcpy2DAsync(static_cast<char*>(W) + half * blk, 2 * blk, src, blk, blk,
                                        d.d_ffn / 128, cudaMemcpyDeviceToDevice, h->st));
            }
            G.W = W;
        } else if (d.arch == ZO_ARCH_QWEN3) {
            const int gu[2] = {ZO_MAT_GATE, ZO_MAT_UP};
            CRC(fused_copy(L, L.g[G_IN], gu, 2));
        }
        if (!L.g[G_O].W || !L.g[G_OUT].W || !L.g[G_IN].W || !L.w.ln1_w || !L.w.ln2_w) {
            h->err = "missing layer weights";
            return fail(ZO_ERR_ARG);
        }
        if (d.arch == ZO_ARCH_OPT && (!L.w.ln1_b || !L.w.ln2_b)) {
            h->err = "missing LayerNorm shift";
            return fail(ZO_ERR_ARG);
        }
        if (h->fp8) {
            // E4M3 copies of the norm-fed matrices, one scale per output channel
            for (int gi : {(int)G_QKV, (int)G_IN}) {
                Group& G = L.g[gi];
                void* p = nullptr;
                CRC(dev_alloc(h, &p, (size_t)G.N * G.K));
                G.Wq = static_cast<uint8_t*>(p);
                CRC(dev_alloc(h, &p, (size_t)G.N * 4));
                G.sw = static_cast<float*>(p);
                launch_quant_rows_e4m3(G.W, E_BF16, G.N, G.K, (size_t)G.K, G.Wq, (size_t)G.K, G.sw,
                                       h->st);
            }
        }
        for (auto& G : L.g) {
            if (G.n_t == 0) continue;
            if (G.K % 4) { h->err = "d_in must be a multiple of 4"; return fail(ZO_ERR_UNSUPPORTED); }
            // rows padded to the 64-row K tile: the shrink may read up to the next
            // multiple of 8 past the live rows, which stay zero
            const size_t ft_rows = ((size_t)G.n_t * r * (1 + options->max_slots) + 63) / 64 * 64;
            void* p = nullptr;
            CRC(dev_alloc(h, &p, ft_rows * G.K * 4));
            G.FT = static_cast<float*>(p);
            CK(h, cudaMemsetAsync(G.FT, 0, ft_rows * G.K * 4, h->st));
            if (h->dt == E_BF16) {
                CRC(dev_alloc(h, &p, ft_rows * G.K * 2));
                G.FTb = p;
                CK(h, cudaMemsetAsync(G.FTb, 0, ft_rows * G.K * 2, h->st));
            }
            CRC(dev_alloc(h, &p, (size_t)G.N * h->kcap * es));
            G.EB = p;
            CK(h, cudaMemsetAsync(G.EB, 0, (size_t)G.N * h->kcap * es, h->st));
            for (int t = 0; t < G.n_t; ++t) {
                CRC(dev_alloc(h, &p, (size_t)G.d_out[t] * r * 4));
                G.Vcur[t] = static_cast<float*>(p);
            }
        }
    }

    // activations and per-call buffers
    const int ffn_cols = d.arch == ZO_ARCH_QWEN3 ? 2 * d.d_ffn : d.d_ffn;
    CRC(dev_alloc(h, reinterpret_cast<void**>(&h->resid), (size_t)maxT * d.d_model * 4));
    CRC(dev_alloc(h, &h->xn, (size_t)maxT * d.d_model * es));
    if (h->fp8) {
        CRC(dev_alloc(h, reinterpret_cast<void**>(&h->xq), (size_t)maxT * d.d_model));
        CRC(dev_alloc(h, reinterpret_cast<void**>(&h->sx), (size_t)maxT * 4));
    }
    CRC(dev_alloc(h, &h->qkv, (size_t)maxT * h->n_qkv * es));
    CRC(dev_alloc(h, &h->att, (size_t)maxT * h->q_dim * es));
    CRC(dev_alloc(h, &h->act, (size_t)maxT * d.d_ffn * es));
    if (d.arch == ZO_ARCH_QWEN3 && !h->swiglu_fused)
        CRC(dev_alloc(h, &h->gu, (size_t)maxT * ffn_cols * es));
    if (h->kcap) CRC(dev_alloc(h, &h->ext, (size_t)maxT * h->kcap * es));
    // scored rows: the target positions of a score, or one row per candidate of a generation
    const int maxSR = options->max_new > 0 ? std::max(maxS, maxR) : maxS;
    CRC(dev_alloc(h, &h->hs, (size_t)maxSR * d.d_model * es));
    if (options->max_new > 0) {
        h->kv_rows = (size_t)maxT + (size_t)maxR * options->max_new;
        CRC(dev_alloc(h, &h->kv_cache,
                      (size_t)d.n_layers * h->kv_rows * 2 * h->kv_dim * es));
        CRC(dev_alloc(h, reinterpret_cast<void**>(&h->gen_tok), (size_t)maxR * options->max_new * 4));
        CRC(dev_alloc(h, reinterpret_cast<void**>(&h->gen_lp), (size_t)maxR * options->max_new * 4));
        CRC(dev_alloc(h, reinterpret_cast<void**>(&h->gen_last), (size_t)maxR * 4));
        CRC(dev_alloc(h, reinterpret_cast<void**>(&h->gen_lens), (size_t)maxR * 4));
        // up to 8 K splits of the widest decode GEMM over a decode step's rows
        const size_t ffn_in = (size_t)d.d_ffn * (d.arch == ZO_ARCH_QWEN3 ? 2 : 1);
        const size_t widest = std::max<size_t>({(size_t)h->n_qkv, ffn_in, (size_t)d.d_model});
        h->splitk_floats = 8 * (size_t)maxR * widest;
        CRC(dev_alloc(h, reinterpret_cast<void**>(&h->splitk_ws), h->splitk_floats * 4));
    }
    if (d.arch == ZO_ARCH_QWEN3) {
        const size_t n = (size_t)d.max_pos * (d.head_dim / 2);
        CRC(dev_alloc(h, reinterpret_cast<void**>(&h->rope_cos), n * 4));
        CRC(dev_alloc(h, reinterpret_cast<void**>(&h->rope_sin), n * 4));
        launch_rope_table(h->rope_cos, h->rope_sin, d.max_pos, d.head_dim, (double)d.rope_theta,
                          h->st);
    }
    h->lse_tiles = gemm_lse_col_tiles(d.vocab);
    CRC(dev_alloc(h, reinterpret_cast<void**>(&h->pmax), (size_t)maxSR * h->lse_tiles * 4));
    CRC(dev_alloc(h, reinterpret_cast<void**>(&h->psum), (size_t)maxSR * h->lse_tiles * 4));
    CRC(dev_alloc(h, reinterpret_cast<void**>(&h->tgt), (size_t)maxSR * 4));
    if (options->max_new > 0)
        CRC(dev_alloc(h, reinterpret_cast<void**>(&h->part_arg), (size_t)maxSR * h->lse_tiles * 4));
    CRC(dev_alloc(h, reinterpret_cast<void**>(&h->logprob), (size_t)maxS * 4));
    CRC(dev_alloc(h, reinterpret_cast<void**>(&h->L_row), (size_t)maxR * 8));
    for (int** p : {&h->tok_id, &h->tok_pos, &h->tok_sign, &h->tok_row})
        CRC(dev_alloc(h, reinterpret_cast<void**>(p), (size_t)maxT * 4));
    CRC(dev_alloc(h, reinterpret_cast<void**>(&h->sc_tok), (size_t)maxS * 4));
    CRC(dev_alloc(h, reinterpret_cast<void**>(&h->sc_tgt), (size_t)maxS * 4));
    h->max_tiles = maxT / 64 + maxR + 1;
    // metadata: cu[R+1] src[R] fg[R] sign[R] soff[R+1] chk[R] tiles[max_tiles]
    h->meta_ints = (size_t)6 * (maxR + 1) + h->max_tiles;
    CRC(dev_alloc(h, reinterpret_cast<void**>(&h->meta), h->meta_ints * 4));
    {
        cudaError_t e = cudaHostAlloc(reinterpret_cast<void**>(&h->meta_h), h->meta_ints * 4,
                                      cudaHostAllocDefault);
        if (e != cudaSuccess) { h->err = "pinned staging allocation failed"; return fail(ZO_ERR_OOM); }
    }
    CK(h, cudaEventCreateWithFlags(&h->meta_ev, cudaEventDisableTiming));
    CK(h, cudaEventCreateWithFlags(&h->jobs_ev, cudaEventDisableTiming));
    CRC(dev_alloc(h, reinterpret_cast<void**>(&h->sums), 16));
    CRC(dev_alloc(h, reinterpret_cast<void**>(&h->c_dev), 8));
    CRC(dev_alloc(h, reinterpret_cast<void**>(&h->flag_dev), 4));
    CRC(dev_alloc(h, reinterpret_cast<void**>(&h->err_dev), 4));
    CK(h, cudaMemsetAsync(h->err_dev, 0, 4, h->st));
    CK(h, cudaMemsetAsync(h->flag_dev, 0, 4, h->st));

    // generator job tables (constant for the run) and the job staging area
    std::vector<GenJob> gu, gv, gu32;
    uint64_t u_elems = 0, v_elems = 0, a_elems = 0;
    for (int l = 0; l < d.n_layers; ++l)
        for (auto& G : h->layers[l].g)
            for (int t = 0; t < G.n_t; ++t) {
                int di, dout;
                matrix_dims(d, G.mats[t], &di, &dout);
                // bf16 models keep U in bf16 only: the shrink reads the bf16 rows and the
                // bank update regenerates U in fp32 from the counter stream
                GenJob ju{G.FTb ? nullptr : G.FT + (size_t)t * r * G.K,
                          G.FTb ? static_cast<char*>(G.FTb) + (size_t)t * r * G.K * 2 : nullptr,
                          l, G.mats[t], 0, di, r, 1, G.K};
                GenJob ju32{G.FT + (size_t)t * r * G.K, nullptr, l, G.mats[t], 0, di, r, 1, G.K};
                GenJob jv{G.Vcur[t], nullptr, l, G.mats[t], 1, dout, r, 0, 0};
                gu.push_back(ju);
                gu32.push_back(ju32);
                gv.push_back(jv);
                h->maxU_pairs = std::max(h->maxU_pairs, (di * r + 1) / 2);
                h->maxV_pairs = std::max(h->maxV_pairs, (dout * r + 1) / 2);
                u_elems += (uint64_t)di * r;
                v_elems += (uint64_t)dout * r;
                a_elems += (uint64_t)di * r;
            }
    h->n_genU = (int)gu.size();
    h->n_genV = (int)gv.size();
    h->n_win = h->n_genU;
    if (h->n_genU) {
        CRC(dev_alloc(h, reinterpret_cast<void**>(&h->genU_d), sizeof(GenJob) * gu.size()));
        CRC(dev_alloc(h, reinterpret_cast<void**>(&h->genV_d), sizeof(GenJob) * gv.size()));
        CK(h, cudaMemcpyAsync(h->genU_d, gu.data(), sizeof(GenJob) * gu.size(),
                              cudaMemcpyHostToDevice, h->st));
        CK(h, cudaMemcpyAsync(h->genV_d, gv.data(), sizeof(GenJob) * gv.size(),
                              cudaMemcpyHostToDevice, h->st));
        if (h->dt == E_BF16) {
            CRC(dev_alloc(h, reinterpret_cast<void**>(&h->genU32_d), sizeof(GenJob) * gu32.size()));
            CK(h, cudaMemcpyAsync(h->genU32_d, gu32.data(), sizeof(GenJob) * gu32.size(),
                                  cudaMemcpyHostToDevice, h->st));
        }
        CRC(dev_alloc(h, reinterpret_cast<void**>(&h->coef_hist),
                      (size_t)options->lazy_interval * 4));
        CRC(dev_alloc(h, reinterpret_cast<void**>(&h->win_d), sizeof(WindowJob) * gu.size()));
        CRC(dev_alloc(h, reinterpret_cast<void**>(&h->upd_d), sizeof(UpdateJob) * gu.size()));
        h->jobs_bytes = (sizeof(WindowJob) + sizeof(UpdateJob)) * gu.size();
        cudaError_t e = cudaHostAlloc(&h->jobs_h, h->jobs_bytes, cudaHostAllocDefault);
        if (e != cudaSuccess) { h->err = "pinned staging allocation failed"; return fail(ZO_ERR_OOM); }
    }
    // state-transition byte model: U written each step (fp32, or bf16 only for bf16 models);
    // the update writes A (and its bf16 mirror) and reads it unless it replays the slot's
    // coefficients (update_bytes); at a window start V written (fp32), EB written twice
    // (model dtype), A and its mirror zeroed
    const uint64_t mirror = h->dt == E_BF16 ? 2 : 0;
    h->bytes_per_U = u_elems * (h->dt == E_BF16 ? 2 : 4);
    h->a_elems = a_elems;
    h->bytes_per_window = v_elems * 4 + v_elems * 2 * es + a_elems * (4 + mirror);
    // Rebuilding the slot from its coefficients regenerates one normal per element for every
    // step of the window so far: worth it while that stays small next to the step (low-rank
    // factors); high-rank factorised directions read-modify-write instead.  ZO_BANK_REPLAY=0|1
    // forces the choice (both give the same bits).
    h->replay_enabled = u_elems * (uint64_t)options->lazy_interval <= (1ull << 26);
    if (const char* rp = std::getenv("ZO_BANK_REPLAY")) {
        if (rp[0] == '0') h->replay_enabled = false;
        if (rp[0] == '1') h->replay_enabled = true;
    }
    // dense mutation reference: 2 * |theta| bytes (model dtype) per step
    uint64_t body = 0, tgt = 0;
    for (int l = 0; l < d.n_layers; ++l)
        for (int m = 0; m < 7; ++m) {
            if (d.arch == ZO_ARCH_OPT && m == ZO_MAT_GATE) continue;
            int di, dout;
            matrix_dims(d, m, &di, &dout);
            body += (uint64_t)di * dout;
            if (layer_targeted(options->targets, l) && ((options->targets.matrix_mask >> m) & 1u))
                tgt += (uint64_t)di * dout;
        }
    h->dense_bytes = 2 * body * es;
    h->dense_bytes_targets = 2 * tgt * es;
    if (options->profile) {
        GemmProfiler& p = h->prof;
        p.a.resize(GemmProfiler::kRing);
        p.b.resize(GemmProfiler::kRing);
        p.flops.assign(GemmProfiler::kRing, 0.0);
        p.tc.assign(GemmProfiler::kRing, 0);
        for (int i = 0; i < GemmProfiler::kRing; ++i) {
            CK(h, cudaEventCreate(&p.a[i]));
            CK(h, cudaEventCreate(&p.b[i]));
        }
        p.on = true;
    }
    CK(h, cudaStreamSynchronize(h->st));
    *out = h;
    return ZO_OK;
#undef CRC
}

void zo_destroy(zo_handle* h) {
    if (!h) return;
    cudaStreamSynchronize(h->st);
    if (h->graph.exec) cudaGraphExecDestroy(h->graph.exec);
    if (h->graph.cap) cudaStreamDestroy(h->graph.cap);
    for (void* p : h->owned) cudaFree(p);
    if (h->meta_h) cudaFreeHost(h->meta_h);
    if (h->jobs_h) cudaFreeHost(h->jobs_h);
    if (h->meta_ev) cudaEventDestroy(h->meta_ev);
    if (h->jobs_ev) cudaEventDestroy(h->jobs_ev);
    for (size_t i = 0; i < h->prof.a.size(); ++i) {
        if (h->prof.a[i]) cudaEventDestroy(h->prof.a[i]);
        if (h->prof.b[i]) cudaEventDestroy(h->prof.b[i]);
    }
    for (auto& t : h->tm)
        if (t.init)
            for (int i = 0; i < PhaseTimer::kRing; ++i) {
                cudaEventDestroy(t.a[i]);
                cudaEventDestroy(t.b[i]);
            }
    delete h;
}

int zo_probe_plan(zo_handle* h, uint64_t step, int32_t rank, float eps, const zo_targets* tg,
                  zo_plan** out) {
    if (!h || !out || !tg) return ZO_ERR_ARG;
    if (rank != h->opt.rank || tg->matrix_mask != h->opt.targets.matrix_mask ||
        tg->layer_mask_lo != h->opt.targets.layer_mask_lo ||
        tg->layer_mask_hi != h->opt.targets.layer_mask_hi ||
        tg->scale_mode != h->opt.targets.scale_mode)
        FAIL(h, ZO_ERR_ARG, "rank/targets differ from the handle's bank layout");
    if (!std::isfinite(eps)) FAIL(h, ZO_ERR_ARG, "eps must be finite");
    if (step != h->step) FAIL(h, ZO_ERR_STATE, "plan step differs from the handle's step counter");
    timer_begin(h, 0);
    const uint64_t nu = (uint64_t)h->opt.lazy_interval;
    const int64_t window = (int64_t)(step / nu);
    if (h->n_genU && (h->n_slots == 0 || h->slot_window.back() != window)) {
        int rc = open_window(h, step);
        if (rc) { timer_end(h, 0); return rc; }
    }
    launch_gen_factors(h->genU_d, h->n_genU, h->maxU_pairs, h->opt.run_seed, step, nullptr, nu,
                       h->mezo_scale, h->opt.targets.scale_mode == ZO_SCALE_MEZO, h->st);
    if (h->n_genU) h->stats.kernel_launches++;
    timer_end(h, 0);
    if (!h->have_plan || h->plan.step != step) h->stats.state_transition_bytes += h->bytes_per_U;
    h->plan.h = h;
    h->plan.step = step;
    h->plan.eps = eps;
    h->plan.scored = false;
    h->plan.B = 0;
    h->have_plan = true;
    *out = &h->plan;
    CK(h, cudaGetLastError());
    return ZO_OK;
}

namespace {

// Host layout of one packed physical batch (+ rows, - rows, then foreground rows):
// the metadata ints cu[R+1] src[R] fg[R] sign[R] soff[R+1] chk[R] tiles[nt] are
// written to `host`; the kernels of a score read the same layout from device memory.
struct BatchPlan {
    int R = 0, B = 0, F = 0, nt = 0;
    long long T = 0, S = 0;
    size_t nints = 0;
};

int prepare_batch(zo_handle* h, int B, const int32_t* lens, const int32_t* tls,
                  const int32_t* tgt_ids, int F, const int32_t* flens, const int32_t* ftls,
                  int* host, BatchPlan* bp) {
    const zo_model_desc& d = h->desc;
    const int R = 2 * B + F;
    int* cu = host;
    int* src = cu + (R + 1);
    int* isfg = src + R;
    int* sign = isfg + R;
    int* soff = sign + R;
    int* chk = soff + (R + 1);
    int* tiles = chk + R;
    long long T = 0, S = 0;
    int po = 0, to = 0;
    cu[0] = 0;
    soff[0] = 0;
    auto row_ok = [&](int L, int tl) {
        if (tl < 1 || L < tl + 1) return false;
        if (L > d.max_pos) return false;        // OPT positions / Qwen3 rotary table
        return L <= 65535 * 64;
    };
    std::vector<int> poff(B), toff(B);
    for (int i = 0; i < B; ++i) {
        if (!row_ok(lens[i], tls[i])) FAIL(h, ZO_ERR_ARG, "bad seq_len/target_len");
        poff[i] = po;
        toff[i] = to;
        po += lens[i];
        to += tls[i];
    }
    int fo = 0;
    int r = 0, nt = 0;
    // attention tiles: 128 queries for the tensor-core kernel, 64 for the CUDA-core one
    const bool tc_attn = h->use_tc && h->dt == E_BF16 && (d.head_dim == 64 || d.head_dim == 128);
    const int qtile = tc_attn ? 128 : 64;
    for (int pass = 0; pass < 3; ++pass) {
        const int n = pass < 2 ? B : F;
        for (int i = 0; i < n; ++i, ++r) {
            const int L = pass < 2 ? lens[i] : flens[i];
            const int tl = pass < 2 ? tls[i] : ftls[i];
            if (pass == 2 && !row_ok(L, tl)) FAIL(h, ZO_ERR_ARG, "bad fg seq_len/target_len");
            src[r] = pass < 2 ? poff[i] : fo;
            if (pass == 2) fo += L;
            isfg[r] = pass == 2;
            sign[r] = pass == 0 ? 1 : (pass == 1 ? -1 : 0);
            chk[r] = (pass < 2 && tgt_ids) ? toff[i] : -1;
            T += L;
            S += tl;
            cu[r + 1] = (int)std::min<long long>(T, 0x7fffffff);
            soff[r + 1] = (int)std::min<long long>(S, 0x7fffffff);
            for (int q = 0; q < (L + qtile - 1) / qtile; ++q) {
                if (nt >= h->max_tiles) FAIL(h, ZO_ERR_ARG, "too many attention tiles");
                tiles[nt++] = (r << 16) | q;
            }
        }
    }
    // attention CTAs are issued in item order: longest (most key chunks) first
    if (tc_attn)
        std::stable_sort(tiles, tiles + nt, [](int x, int y) { return (x & 0xFFFF) > (y & 0xFFFF); });
    if (T > h->opt.max_tokens) FAIL(h, ZO_ERR_ARG, "more tokens than max_tokens");
    if (S > h->opt.max_scored) FAIL(h, ZO_ERR_ARG, "more scored positions than max_scored");
    if (R >= 32768) FAIL(h, ZO_ERR_ARG, "too many rows");
    bp->R = R; bp->B = B; bp->F = F; bp->nt = nt; bp->T = T; bp->S = S;
    bp->nints = (size_t)(tiles - cu) + nt;
    return ZO_OK;
}

// Every kernel of one score over a batch laid out by prepare_batch, whose metadata
// is already in device memory at md.  Enqueues only (no host synchronisation), so
// it can be captured into a CUDA graph.
// One fused GEMM group of a layer over Ti token rows: the bank shrink (when the group
// carries targets) and the base GEMM with the extension K blocks, epilogue epi.
// nn (decode steps, EPI_RESID): the norm of the updated residual rows that comes next; it runs
// fused into the split reduction when that path is taken, else right after the GEMM.
// kv (decode steps, the q|k|v group): the reduction also appends k|v to the cache when it can;
// *kv_done reports whether it did.
int group_gemm(zo_handle* h, Group& G, const void* X, int epi, void* C, int ldc, int ctype,
               int Ti, float eps, const Layer* Lq = nullptr, bool decode = false,
               const NormNext* nn = nullptr, const KvAppend* kv = nullptr,
               int* kv_done = nullptr) {
    const zo_model_desc& d = h->desc;
    const int r_ = h->opt.rank;
    GemmArgs g;
    memset(&g, 0, sizeof(g));
    int norm_done = 0;
    g.norm_next = nn;
    g.norm_done = &norm_done;
    g.kv_append = kv;
    g.kv_done = kv_done;
    if (epi == EPI_QKNR) {
        g.tok_pos = h->tok_pos; g.qn = Lq->w.q_norm; g.kn = Lq->w.k_norm;
        g.rope_cos = h->rope_cos; g.rope_sin = h->rope_sin; g.norm_eps = d.norm_eps;
        g.n_q_heads = d.n_heads; g.n_qk_heads = d.n_heads + d.n_kv_heads;
    }
    g.M = Ti;
    if (G.n_t > 0) {
        // live extension columns, padded to a multiple of 8 (16-byte TMA rows); the
        // padding columns of S and E_B are zero
        const int kext = (G.n_t * r_ * (1 + h->n_slots) + 7) / 8 * 8;
        GemmArgs s;
        memset(&s, 0, sizeof(s));
        s.A = X; s.lda = G.K; s.a_type = h->dt;
        if (G.FTb) { s.B = G.FTb; s.b_type = E_BF16; }
        else { s.B = G.FT; s.b_type = E_F32; }
        s.ldb = G.K;
        s.M = Ti; s.N = kext; s.K = G.K;
        s.epi = EPI_SHRINK;
        s.C = h->ext; s.ldc = h->kcap; s.c_type = h->dt;
        s.row_sign = h->tok_sign; s.eps = eps; s.scale_cols = G.n_t * r_;
        if (G.Wq) s.a_scale = h->sx;      // S / s_x: the base GEMM accumulates in E4M3 units
        if (decode) {
            // a decode step's handful of rows: the factor rows take the 128-row side of the
            // swapped tensor-core GEMM with K split over the SMs (bf16 factors), else a tiled
            // CUDA-core dot per (row, factor column)
            s.ws = h->splitk_ws;
            s.ws_floats = h->splitk_floats;
            if (h->use_tc && Ti <= 128 && gemm_tc_supported(s)) {
                int rc = run_gemm(h, s, 2.0 * Ti * (double)G.K * kext);
                if (rc) return rc;
            } else {
                launch_shrink_rows(s.A, s.a_type, s.B, s.b_type, Ti, kext, G.K, s.C, s.ldc,
                                   s.c_type, s.row_sign, eps, s.scale_cols, s.a_scale,
                                   h->splitk_ws, h->splitk_floats, h->st);
                h->stats.kernel_launches++;
            }
        } else {
            int rc = run_gemm(h, s, 2.0 * Ti * (double)G.K * kext);
            if (rc) return rc;
        }
        g.A2 = h->ext; g.lda2 = h->kcap; g.a2_type = h->dt;
        g.B2 = G.EB; g.ldb2 = h->kcap; g.b2_type = h->dt;
        g.K2 = kext;
    }
    g.A = X; g.lda = G.K; g.a_type = h->dt;
    g.B = G.W; g.ldb = G.K; g.b_type = h->dt;
    if (G.Wq) {
        // E4M3 rows of the same norm output and of W; dequantised in the epilogue
        g.A = h->xq; g.a_type = E_FP8;
        g.B = G.Wq; g.b_type = E_FP8;
        g.a_scale = h->sx; g.b_scale = G.sw;
    }
    g.N = G.N; g.K = G.K;
    g.bias = G.bias;
    g.epi = epi;
    g.C = C; g.ldc = ldc; g.c_type = ctype;
    if (decode) {                         // few rows: the GEMM splits K (swapped operands)
        g.ws = h->splitk_ws;
        g.ws_floats = h->splitk_floats;
    }
    // algorithmic work: the base GEMM plus, per target, its own expand columns
    double fl = 2.0 * Ti * (double)G.N * G.K;
    for (int t = 0; t < G.n_t; ++t) fl += 2.0 * Ti * (double)G.d_out[t] * r_ * (1 + h->n_slots);
    const int rc = run_gemm(h, g, fl);
    if (rc || !nn || norm_done) return rc;
    launch_norm(static_cast<const float*>(C), nullptr, Ti, G.N, nn->kind, nn->w, nn->b, nn->eps,
                nn->out, nn->out_type, h->st, nn->q8, nn->s8, decode);
    h->stats.kernel_launches++;
    return ZO_OK;
}

// Every decoder layer over the Ti token rows whose ids, positions, signs and embeddings are
// in place (h->tok_*, h->resid).  attn(l) enqueues layer l's attention: it reads the q|k|v
// rows in h->qkv (q/k normalised and rotated for Qwen3) and writes h->att.
int decoder_layers(zo_handle* h, int Ti, float eps, const std::function<int(int, bool)>& attn,
                   bool decode = false,
                   const std::function<const KvAppend*(int)>& kv_of = nullptr) {
    const zo_model_desc& d = h->desc;
    const int nk = d.arch == ZO_ARCH_OPT ? 0 : 1;   // norm kind
    // decode steps: each residual GEMM also applies the norm that follows it (ln2 after o, the
    // next layer's ln1 or the final norm after the FFN), fused into its split reduction
    for (int l = 0; l < d.n_layers; ++l) {
        Layer& L = h->layers[l];
        if (!decode || l == 0)
            launch_norm(h->resid, nullptr, Ti, d.d_model, nk, L.w.ln1_w, L.w.ln1_b, d.norm_eps,
                        h->xn, h->dt, h->st, h->xq, h->sx, decode);
        // decode steps: k|v go to the cache from the q|k|v reduction when the rows it stores
        // are final (OPT, or Qwen3 with the q/k norm fused into that reduction)
        int kv_done = 0;
        const KvAppend* kv = kv_of && (d.arch == ZO_ARCH_OPT || h->qknr_fused) ? kv_of(l) : nullptr;
        int rc = group_gemm(h, L.g[G_QKV], h->xn, h->qknr_fused ? EPI_QKNR : EPI_STORE, h->qkv,
                            h->n_qkv, h->dt, Ti, eps, &L, decode, nullptr, kv, &kv_done);
        if (rc) return rc;
        if (d.arch == ZO_ARCH_QWEN3 && !h->qknr_fused)
            launch_qk_norm_rope(h->qkv, h->n_qkv, h->dt, h->tok_pos, Ti, d.n_heads, d.n_kv_heads,
                                d.head_dim, L.w.q_norm, L.w.k_norm, d.norm_eps, h->rope_cos,
                                h->rope_sin, h->st);
        rc = attn(l, kv_done != 0);
        if (rc) return rc;
        const NormNext ln2 = {L.w.ln2_w, L.w.ln2_b, nk, d.norm_eps, h->xn, h->dt, h->xq, h->sx};
        rc = group_gemm(h, L.g[G_O], h->att, EPI_RESID, h->resid, d.d_model, E_F32, Ti, eps, nullptr,
                        decode, decode ? &ln2 : nullptr);
        if (rc) return rc;
        if (!decode)
            launch_norm(h->resid, nullptr, Ti, d.d_model, nk, L.w.ln2_w, L.w.ln2_b, d.norm_eps,
                        h->xn, h->dt, h->st, h->xq, h->sx);
        if (d.arch == ZO_ARCH_OPT) {
            rc = group_gemm(h, L.g[G_IN], h->xn, EPI_STORE_RELU, h->act, d.d_ffn, h->dt, Ti, eps, nullptr, decode);
        } else if (h->swiglu_fused) {
            rc = group_gemm(h, L.g[G_IN], h->xn, EPI_SWIGLU, h->act, d.d_ffn, h->dt, Ti, eps, nullptr, decode);
        } else {
            rc = group_gemm(h, L.g[G_IN], h->xn, EPI_STORE, h->gu, 2 * d.d_ffn, h->dt, Ti, eps, nullptr, decode);
            if (!rc) launch_swiglu(h->gu, Ti, d.d_ffn, h->act, h->dt, h->st);
        }
        if (rc) return rc;
        NormNext next;
        if (l + 1 < d.n_layers) {
            const Layer& N1 = h->layers[l + 1];
            next = {N1.w.ln1_w, N1.w.ln1_b, nk, d.norm_eps, h->xn, h->dt, h->xq, h->sx};
        } else {
            next = {h->wts.final_w, h->wts.final_b, nk, d.norm_eps, h->hs, h->dt, nullptr, nullptr};
        }
        rc = group_gemm(h, L.g[G_OUT], h->act, EPI_RESID, h->resid, d.d_model, E_F32, Ti, eps, nullptr,
                        decode, decode ? &next : nullptr);
        if (rc) return rc;
    }
    return ZO_OK;
}

int launch_batch(zo_handle* h, float eps, const int* md, const BatchPlan& bp,
                 const int32_t* ptok, const int32_t* ftok, const int32_t* tgt_ids) {
    const zo_model_desc& d = h->desc;
    const int R = bp.R, nt = bp.nt;
    const long long T = bp.T, S = bp.S;
    const bool tc_attn = h->use_tc && h->dt == E_BF16 && (d.head_dim == 64 || d.head_dim == 128);
    RowMeta m;
    m.cu_seqlens = md;
    m.row_src = md + (R + 1);
    m.row_is_fg = m.row_src + R;
    m.row_sign = m.row_is_fg + R;
    m.score_off = m.row_sign + R;
    const int* chk_d = m.score_off + (R + 1);
    const int* tiles_d = chk_d + R;
    const int Ti = (int)T, Si = (int)S;

    launch_build_tokens(m, R, ptok, ftok, d.vocab, h->tok_id, h->tok_pos, h->tok_sign,
                        h->tok_row, h->sc_tok, h->sc_tgt, h->tgt, tgt_ids, nullptr, chk_d,
                        h->err_dev, h->st);
    // build_tokens, embed, per layer 2 norms + attention (+ SwiGLU), final norm, LSE merge
    h->stats.kernel_launches +=
        2 + (uint64_t)d.n_layers * (3 + (d.arch == ZO_ARCH_QWEN3 && !h->qknr_fused) +
                                    (d.arch == ZO_ARCH_QWEN3 && !h->swiglu_fused)) + 2;
    launch_embed(h->tok_id, h->tok_pos, h->wts.tok_embed,
                 d.arch == ZO_ARCH_OPT ? h->wts.pos_embed : nullptr, h->dt, h->resid, Ti,
                 d.d_model, h->st);

    const int nk = d.arch == ZO_ARCH_OPT ? 0 : 1;   // norm kind
    int rc = decoder_layers(h, Ti, eps, [&](int, bool) -> int {
            AttnArgs a;
            memset(&a, 0, sizeof(a));
            a.qkv = h->qkv; a.ld_qkv = h->n_qkv;
            a.out = h->att; a.ld_out = h->q_dim;
            a.dtype = h->dt;
            a.cu_seqlens = m.cu_seqlens;
            a.tiles = tiles_d; a.n_tiles = nt;
            a.H = d.n_heads; a.Hkv = d.n_kv_heads; a.hd = d.head_dim;
            a.scale = (float)(1.0 / std::sqrt((double)d.head_dim));
            a.n_tokens = Ti;
            a.n_rows = R;
            if (tc_attn && attention_tc_supported(a)) {
                if (!launch_attention_tc(a, h->st)) FAIL(h, ZO_ERR_CUDA, "attention tensor map failed");
            } else {
                launch_attention(a, h->st);
            }
            return ZO_OK;
        });
    if (rc) return rc;
    // scored positions: gather + final norm, then lm_head with log-sum-exp
    launch_norm(h->resid, h->sc_tok, Si, d.d_model, nk, h->wts.final_w, h->wts.final_b,
                d.norm_eps, h->hs, h->dt, h->st);
    GemmArgs g;
    memset(&g, 0, sizeof(g));
    g.A = h->hs; g.lda = d.d_model; g.a_type = h->dt;
    g.B = d.tie_lm_head ? h->wts.tok_embed : h->wts.lm_head; g.ldb = d.d_model; g.b_type = h->dt;
    g.M = Si; g.N = d.vocab; g.K = d.d_model;
    g.epi = EPI_LSE;
    g.targets = h->sc_tgt; g.part_max = h->pmax; g.part_sum = h->psum; g.tgt_logit = h->tgt;
    const bool tc = h->use_tc && gemm_tc_supported(g);
    g.n_col_tiles = tc ? gemm_tc_col_tiles(d.vocab) : h->lse_tiles;
    {
        const int slot = prof_begin(h);
        if (tc) {
            if (gemm_tc(g, h->st)) FAIL(h, ZO_ERR_CUDA, "tcgen05 lm_head launch failed");
        } else {
            gemm_simt(g, h->st);
        }
        prof_end(h, slot, 2.0 * Si * (double)d.vocab * d.d_model, tc);
        h->stats.kernel_launches++;
        if (!tc) h->stats.cuda_core_gemm_launches++;
    }
    launch_lse_merge(h->pmax, h->psum, h->tgt, Si, g.n_col_tiles, h->logprob, h->st);
    h->stats.tokens_scored += (uint64_t)T;
    h->stats.positions_scored += (uint64_t)S;
    h->stats.score_calls++;
    CK(h, cudaGetLastError());
    return ZO_OK;
}

// lm_head over M rows of h->hs with the LSE epilogue recording each tile's argmax, then
// the greedy choice per row into tok[r * stride], lp[r * stride].
int lm_head_greedy(zo_handle* h, int M, int* tok, float* lp, int stride) {
    const zo_model_desc& d = h->desc;
    GemmArgs g;
    memset(&g, 0, sizeof(g));
    g.A = h->hs; g.lda = d.d_model; g.a_type = h->dt;
    g.B = d.tie_lm_head ? h->wts.tok_embed : h->wts.lm_head; g.ldb = d.d_model; g.b_type = h->dt;
    g.M = M; g.N = d.vocab; g.K = d.d_model;
    g.epi = EPI_LSE;
    g.targets = h->gen_last;            // any valid ids: the target logit is not used here
    g.part_max = h->pmax; g.part_sum = h->psum; g.tgt_logit = h->tgt; g.part_arg = h->part_arg;
    const bool tc = h->use_tc && gemm_tc_supported(g);
    g.n_col_tiles = tc ? gemm_tc_col_tiles(d.vocab) : h->lse_tiles;
    if (tc) {
        if (gemm_tc(g, h->st)) FAIL(h, ZO_ERR_CUDA, "tcgen05 lm_head launch failed");
    } else {
        gemm_simt(g, h->st);
        h->stats.cuda_core_gemm_launches++;
    }
    launch_lse_argmax_merge(h->pmax, h->psum, h->part_arg, M, g.n_col_tiles, tok, lp, stride,
                            h->st);
    h->stats.kernel_launches += 2;
    return ZO_OK;
}

// Generation queries: packed prefill into the KV cache, then greedy decode steps.
int generate_impl(zo_handle* h, float eps, const int32_t* ptok, int B, const int32_t* lens,
                  int G) {
    const zo_model_desc& d = h->desc;
    const int R = 2 * B;
    std::vector<int> tls(B, 1);
    CK(h, cudaEventSynchronize(h->meta_ev));
    BatchPlan bp;
    int rc = prepare_batch(h, B, lens, tls.data(), nullptr, 0, nullptr, nullptr, h->meta_h, &bp);
    if (rc) return rc;
    if ((size_t)bp.T + (size_t)R * G > h->kv_rows) FAIL(h, ZO_ERR_ARG, "generation exceeds the KV cache");
    CK(h, cudaMemcpyAsync(h->meta, h->meta_h, bp.nints * 4, cudaMemcpyHostToDevice, h->st));
    CK(h, cudaEventRecord(h->meta_ev, h->st));
    const int* md = h->meta;
    RowMeta m;
    m.cu_seqlens = md;
    m.row_src = md + (R + 1);
    m.row_is_fg = m.row_src + R;
    m.row_sign = m.row_is_fg + R;
    m.score_off = m.row_sign + R;
    const int* chk_d = m.score_off + (R + 1);
    const int* tiles_d = chk_d + R;
    const int Ti = (int)bp.T, nt = bp.nt;
    const int kv2 = 2 * h->kv_dim;
    const size_t layer_elems = h->kv_rows * (size_t)kv2;
    const size_t es = esize(h->dt);
    auto cache = [&](int l) { return static_cast<char*>(h->kv_cache) + (size_t)l * layer_elems * es; };
    const bool tc_attn = h->use_tc && h->dt == E_BF16 && (d.head_dim == 64 || d.head_dim == 128);
    const int nk = d.arch == ZO_ARCH_OPT ? 0 : 1;
    const float scale = (float)(1.0 / std::sqrt((double)d.head_dim));

    // prefill: the prompts of both candidates as one packed batch, k|v kept per layer
    launch_build_tokens(m, R, ptok, nullptr, d.vocab, h->tok_id, h->tok_pos, h->tok_sign,
                        h->tok_row, h->sc_tok, h->sc_tgt, h->tgt, nullptr, nullptr, chk_d,
                        h->err_dev, h->st);
    launch_embed(h->tok_id, h->tok_pos, h->wts.tok_embed,
                 d.arch == ZO_ARCH_OPT ? h->wts.pos_embed : nullptr, h->dt, h->resid, Ti,
                 d.d_model, h->st);
    rc = decoder_layers(h, Ti, eps, [&](int l, bool) -> int {
        launch_kv_scatter(h->qkv, h->n_qkv, h->q_dim, kv2, h->tok_row, Ti, G, cache(l),
                          h->kv_rows, h->dt, h->st);
        AttnArgs a;
        memset(&a, 0, sizeof(a));
        a.qkv = h->qkv; a.ld_qkv = h->n_qkv;
        a.out = h->att; a.ld_out = h->q_dim;
        a.dtype = h->dt;
        a.cu_seqlens = m.cu_seqlens;
        a.tiles = tiles_d; a.n_tiles = nt;
        a.H = d.n_heads; a.Hkv = d.n_kv_heads; a.hd = d.head_dim;
        a.scale = scale;
        a.n_tokens = Ti;
        a.n_rows = R;
        if (tc_attn && attention_tc_supported(a)) {
            if (!launch_attention_tc(a, h->st)) FAIL(h, ZO_ERR_CUDA, "attention tensor map failed");
        } else {
            launch_attention(a, h->st);
        }
        h->stats.kernel_launches += 2;
        return ZO_OK;
    });
    if (rc) return rc;
    launch_last_tokens(md, R, h->gen_last, h->gen_lens, h->st);
    launch_norm(h->resid, h->gen_last, R, d.d_model, nk, h->wts.final_w, h->wts.final_b,
                d.norm_eps, h->hs, h->dt, h->st);
    rc = lm_head_greedy(h, R, h->gen_tok, h->gen_lp, G);
    if (rc) return rc;
    h->stats.kernel_launches += 4 + (uint64_t)d.n_layers * (2 + (d.arch == ZO_ARCH_QWEN3 && !h->qknr_fused) +
                                                             (d.arch == ZO_ARCH_QWEN3 && !h->swiglu_fused));
    h->stats.tokens_scored += (uint64_t)Ti;

    // decode: token g of every row at position len + g, attending over its row's cache
    int max_len = 0;
    for (int i = 0; i < B; ++i) max_len = std::max(max_len, (int)lens[i]);
    for (int g = 0; g + 1 < G; ++g) {
        launch_decode_prep(h->gen_tok, G, g, h->gen_lens, R, B, h->tok_id, h->tok_pos,
                           h->tok_sign, h->tok_row, h->st);
        launch_embed(h->tok_id, h->tok_pos, h->wts.tok_embed,
                     d.arch == ZO_ARCH_OPT ? h->wts.pos_embed : nullptr, h->dt, h->resid, R,
                     d.d_model, h->st);
        KvAppend kva;
        rc = decoder_layers(h, R, eps, [&](int l, bool kv_in_cache) -> int {
            if (!kv_in_cache)
                launch_kv_append(h->qkv, h->n_qkv, h->q_dim, kv2, md, h->gen_lens, R, g, G,
                                 cache(l), h->kv_rows, h->dt, h->st);
            if (!launch_decode_attention(h->qkv, h->n_qkv, cache(l), kv2, md, h->gen_lens, R, g, G,
                                         d.n_heads, d.n_kv_heads, d.head_dim, scale, h->att,
                                         h->q_dim, h->dt, max_len + g + 1, h->splitk_ws,
                                         h->splitk_floats, h->st))
                FAIL(h, ZO_ERR_UNSUPPORTED, "decode attention: more than 8 query heads per kv head");
            h->stats.kernel_launches += 2;
            return ZO_OK;
        }, true, [&](int l) -> const KvAppend* {
            kva = {cache(l), h->kv_rows, md, h->gen_lens, g, G, h->q_dim, kv2};
            return h->dt == E_BF16 ? &kva : nullptr;
        });
        if (rc) return rc;
        // (the final norm of the R rows into hs ran with the last layer's FFN reduction)
        rc = lm_head_greedy(h, R, h->gen_tok + g + 1, h->gen_lp + g + 1, G);
        if (rc) return rc;
        h->stats.kernel_launches += 3 + (uint64_t)d.n_layers * (2 + (d.arch == ZO_ARCH_QWEN3 && !h->qknr_fused) +
                                                                 (d.arch == ZO_ARCH_QWEN3 && !h->swiglu_fused));
        h->stats.tokens_scored += (uint64_t)R;
    }
    CK(h, cudaGetLastError());
    return ZO_OK;
}

int score_impl(zo_handle* h, float eps, const int32_t* ptok, int B, const int32_t* lens,
               const int32_t* tls, const int32_t* tgt_ids, const int32_t* ftok, int F,
               const int32_t* flens, const int32_t* ftls) {
    if (B < 0 || F < 0 || (B > 0 && (!ptok || !lens || !tls)) || (F > 0 && (!ftok || !flens || !ftls)))
        FAIL(h, ZO_ERR_ARG, "missing score arguments");
    const int R = 2 * B + F;
    if (R == 0) FAIL(h, ZO_ERR_ARG, "empty batch");
    if (R > h->opt.max_rows) FAIL(h, ZO_ERR_ARG, "more rows than max_rows");
    // the pinned staging buffer is reused once the previous score's copy has left it
    CK(h, cudaEventSynchronize(h->meta_ev));
    BatchPlan bp;
    int rc = prepare_batch(h, B, lens, tls, tgt_ids, F, flens, ftls, h->meta_h, &bp);
    if (rc) return rc;
    CK(h, cudaMemcpyAsync(h->meta, h->meta_h, bp.nints * 4, cudaMemcpyHostToDevice, h->st));
    CK(h, cudaEventRecord(h->meta_ev, h->st));
    return launch_batch(h, eps, h->meta, bp, ptok, ftok, tgt_ids);
}

}  // namespace

static int score_common(zo_plan* plan, zo_handle* h, const int32_t* ptok, int32_t B,
                        const int32_t* lens, const int32_t* tls, const int32_t* tgt_ids,
                        float* Lp, float* Lm, float* tok_lp, const int32_t* ftok, int32_t F,
                        const int32_t* flens, const int32_t* ftls, float* fg_lp) {
    const float eps = plan ? plan->eps : 0.f;
    timer_begin(h, 1);
    int rc = score_impl(h, eps, ptok, B, lens, tls, tgt_ids, ftok, F, flens, ftls);
    if (rc) { timer_end(h, 1); return rc; }
    const int R = 2 * B + F;
    // score_off sits after cu[R+1], src[R], fg[R], sign[R] in the device metadata
    const int* soff_d = h->meta + (R + 1) + 3 * R;
    long long Sp = 0, Sf = 0;
    for (int i = 0; i < B; ++i) Sp += tls[i];
    for (int i = 0; i < F; ++i) Sf += ftls[i];
    // the row objectives feed the estimate of a scored plan; a foreground-only call has none,
    // and must leave those of a plan scored earlier for its zo_step
    if (B > 0) {
        launch_row_objective(h->logprob, soff_d, R, B, 2 * Sp + Sf, h->L_row, Lp, Lm, h->st);
        h->stats.kernel_launches++;
    }
    if (tok_lp && Sp)
        CK(h, cudaMemcpyAsync(tok_lp, h->logprob, 2 * Sp * 4, cudaMemcpyDeviceToDevice, h->st));
    if (fg_lp && Sf)
        CK(h, cudaMemcpyAsync(fg_lp, h->logprob + 2 * Sp, Sf * 4, cudaMemcpyDeviceToDevice, h->st));
    timer_end(h, 1);
    if (plan) {
        plan->scored = B > 0;
        plan->B = B;
    }
    CK(h, cudaGetLastError());
    return ZO_OK;
}

int zo_score(zo_plan* plan, const int32_t* packed_tokens, int32_t n_prompts,
             const int32_t* seq_lens, const int32_t* target_lens, const int32_t* target_ids,
             float* L_plus, float* L_minus, float* tok_logprob) {
    if (!plan || !plan->h) return ZO_ERR_ARG;
    zo_handle* h = plan->h;
    if (!h->have_plan || plan != &h->plan) FAIL(h, ZO_ERR_STATE, "stale plan");
    if (n_prompts < 1) FAIL(h, ZO_ERR_ARG, "n_prompts must be >= 1");
    return score_common(plan, h, packed_tokens, n_prompts, seq_lens, target_lens, target_ids,
                        L_plus, L_minus, tok_logprob, nullptr, 0, nullptr, nullptr, nullptr);
}

int zo_score_cobatch(zo_plan* plan, const int32_t* packed_tokens, int32_t n_prompts,
                     const int32_t* seq_lens, const int32_t* target_lens,
                     const int32_t* target_ids, float* L_plus, float* L_minus,
                     float* tok_logprob, const int32_t* fg_tokens, int32_t n_fg,
                     const int32_t* fg_seq_lens, const int32_t* fg_target_lens,
                     float* fg_tok_logprob) {
    if (!plan || !plan->h) return ZO_ERR_ARG;
    zo_handle* h = plan->h;
    if (!h->have_plan || plan != &h->plan) FAIL(h, ZO_ERR_STATE, "stale plan");
    if (n_prompts < 1) FAIL(h, ZO_ERR_ARG, "n_prompts must be >= 1");
    return score_common(plan, h, packed_tokens, n_prompts, seq_lens, target_lens, target_ids,
                        L_plus, L_minus, tok_logprob, fg_tokens, n_fg, fg_seq_lens,
                        fg_target_lens, fg_tok_logprob);
}

int zo_generate(zo_plan* plan, const int32_t* packed_tokens, int32_t n_prompts,
                const int32_t* seq_lens, int32_t n_new, int32_t* gen_tokens,
                float* gen_logprob, float* L_plus, float* L_minus) {
    if (!plan || !plan->h) return ZO_ERR_ARG;
    zo_handle* h = plan->h;
    if (!h->have_plan || plan != &h->plan) FAIL(h, ZO_ERR_STATE, "stale plan");
    if (h->opt.max_new < 1) FAIL(h, ZO_ERR_UNSUPPORTED, "generation needs options.max_new >= 1");
    if (n_prompts < 1 || !packed_tokens || !seq_lens) FAIL(h, ZO_ERR_ARG, "missing generation arguments");
    if (n_new < 1 || n_new > h->opt.max_new) FAIL(h, ZO_ERR_ARG, "n_new outside 1..max_new");
    if (2 * n_prompts > h->opt.max_rows) FAIL(h, ZO_ERR_ARG, "more rows than max_rows");
    for (int i = 0; i < n_prompts; ++i)
        if (seq_lens[i] < 2 || (long long)seq_lens[i] + n_new > h->desc.max_pos)
            FAIL(h, ZO_ERR_ARG, "seq_len must be >= 2 and seq_len + n_new <= max_pos");
    timer_begin(h, 1);
    int rc = generate_impl(h, plan->eps, packed_tokens, n_prompts, seq_lens, n_new);
    if (rc) { timer_end(h, 1); return rc; }
    const int R = 2 * n_prompts;
    launch_gen_objective(h->gen_lp, R, n_prompts, n_new, h->L_row, L_plus, L_minus, h->st);
    if (gen_tokens)
        CK(h, cudaMemcpyAsync(gen_tokens, h->gen_tok, (size_t)R * n_new * 4,
                              cudaMemcpyDeviceToDevice, h->st));
    if (gen_logprob)
        CK(h, cudaMemcpyAsync(gen_logprob, h->gen_lp, (size_t)R * n_new * 4,
                              cudaMemcpyDeviceToDevice, h->st));
    timer_end(h, 1);
    h->stats.kernel_launches++;
    h->stats.positions_scored += (uint64_t)R * n_new;
    h->stats.score_calls++;
    plan->scored = true;
    plan->B = n_prompts;
    CK(h, cudaGetLastError());
    return ZO_OK;
}

int zo_score_foreground(zo_handle* h, const int32_t* fg_tokens, int32_t n_fg,
                        const int32_t* fg_seq_lens, const int32_t* fg_target_lens,
                        float* fg_tok_logprob) {
    if (!h) return ZO_ERR_ARG;
    if (n_fg < 1) FAIL(h, ZO_ERR_ARG, "n_fg must be >= 1");
    return score_common(nullptr, h, nullptr, 0, nullptr, nullptr, nullptr, nullptr, nullptr,
                        nullptr, fg_tokens, n_fg, fg_seq_lens, fg_target_lens, fg_tok_logprob);
}

int zo_objective_sums(zo_handle* h, double* dev_sums) {
    if (!h || !dev_sums) return ZO_ERR_ARG;
    if (!h->have_plan || !h->plan.scored) FAIL(h, ZO_ERR_STATE, "no scored plan");
    launch_objective_sums(h->L_row, h->plan.B, dev_sums, h->st);
    h->stats.kernel_launches++;
    CK(h, cudaGetLastError());
    return ZO_OK;
}

int zo_step_from_sums(zo_handle* h, float lr, const double* dev_sums, double* c_out) {
    if (!h || !dev_sums) return ZO_ERR_ARG;
    if (!h->have_plan || !h->plan.scored) FAIL(h, ZO_ERR_STATE, "zo_step needs a scored plan");
    if (!std::isfinite(lr)) FAIL(h, ZO_ERR_ARG, "lr must be finite");
    timer_begin(h, 2);
    launch_estimate(dev_sums, h->plan.eps, h->c_dev, h->flag_dev, h->st);
    launch_bank_update(h->upd_d, h->n_genU, h->max_upd, h->c_dev, h->flag_dev, lr,
                       h->opt.run_seed, h->step, nullptr, (uint64_t)h->opt.lazy_interval,
                       h->mezo_scale, h->opt.targets.scale_mode == ZO_SCALE_MEZO,
                       h->replay_from, h->coef_hist, h->st);
    h->stats.kernel_launches += 1 + (h->n_genU > 0);
    timer_end(h, 2);
    CK(h, cudaGetLastError());
    if (c_out) {
        int flag = 0, err = 0;
        CK(h, cudaMemcpyAsync(c_out, h->c_dev, 8, cudaMemcpyDeviceToHost, h->st));
        CK(h, cudaMemcpyAsync(&flag, h->flag_dev, 4, cudaMemcpyDeviceToHost, h->st));
        CK(h, cudaMemcpyAsync(&err, h->err_dev, 4, cudaMemcpyDeviceToHost, h->st));
        CK(h, cudaStreamSynchronize(h->st));
        if (err) {
            CK(h, cudaMemsetAsync(h->err_dev, 0, 4, h->st));
            if (err & 2) FAIL(h, ZO_ERR_ARG, "a token id lies outside [0, vocab): update refused");
            FAIL(h, ZO_ERR_ARG, "target_ids differ from the rows' last tokens");
        }
        if (flag) FAIL(h, ZO_ERR_NONFINITE, "non-finite objective: update refused");
    }
    h->stats.state_transition_bytes += update_bytes(h, h->step);
    h->stats.dense_ref_bytes += h->dense_bytes;
    h->stats.dense_ref_bytes_targets += h->dense_bytes_targets;
    h->stats.steps++;
    h->step++;
    h->plan.scored = false;
    h->have_plan = false;
    return ZO_OK;
}

int zo_step(zo_handle* h, float lr, double* c_out) {
    if (!h) return ZO_ERR_ARG;
    if (!h->have_plan || !h->plan.scored) FAIL(h, ZO_ERR_STATE, "zo_step needs a scored plan");
    launch_objective_sums(h->L_row, h->plan.B, h->sums, h->st);
    h->stats.kernel_launches++;
    return zo_step_from_sums(h, lr, h->sums, c_out);
}

int zo_step_graph(zo_handle* h, const int32_t* packed_tokens, int32_t n_prompts,
                  const int32_t* seq_lens, const int32_t* target_lens, float eps, float lr,
                  float* L_plus, float* L_minus) {
    if (!h) return ZO_ERR_ARG;
    if (!packed_tokens || !seq_lens || !target_lens || n_prompts < 1)
        FAIL(h, ZO_ERR_ARG, "missing step arguments");
    if (!std::isfinite(eps) || !std::isfinite(lr)) FAIL(h, ZO_ERR_ARG, "eps and lr must be finite");
    if (h->have_plan) FAIL(h, ZO_ERR_STATE, "a plan is open: finish it with zo_step first");
    const int B = n_prompts, R = 2 * B;
    if (R > h->opt.max_rows) FAIL(h, ZO_ERR_ARG, "more rows than max_rows");
    auto& G = h->graph;
    const uint64_t step = h->step;
    // a window boundary changes the bank's layout on the host: it runs eagerly, and the
    // graph is captured again below for the new slot count
    const uint64_t nu = (uint64_t)h->opt.lazy_interval;
    const int64_t window = (int64_t)(step / nu);
    if (h->n_genU && (h->n_slots == 0 || h->slot_window.back() != window)) {
        int rc = open_window(h, step);
        if (rc) return rc;
    }
    const bool same = G.exec && G.tok == packed_tokens && G.Lp == L_plus && G.Lm == L_minus &&
                      G.eps == eps && G.lr == lr && G.slots == h->n_slots &&
                      G.replay_from == h->replay_from &&
                      (int)G.lens.size() == B &&
                      std::equal(G.lens.begin(), G.lens.end(), seq_lens) &&
                      std::equal(G.tls.begin(), G.tls.end(), target_lens);
    if (!same) {
        if (G.exec) {
            CK(h, cudaStreamSynchronize(h->st));
            cudaGraphExecDestroy(G.exec);
            G.exec = nullptr;
        }
        if (!G.cap) CK(h, cudaStreamCreateWithFlags(&G.cap, cudaStreamNonBlocking));
        if (!G.meta) {
            const int rc = dev_alloc(h, reinterpret_cast<void**>(&G.meta), h->meta_ints * 4);
            if (rc) return rc;
        }
        if (!G.step_dev) {
            const int rc = dev_alloc(h, reinterpret_cast<void**>(&G.step_dev), 8);
            if (rc) return rc;
        }
        // the layout is fixed for the graph's life: its metadata goes to the device once
        std::vector<int> host(h->meta_ints);
        BatchPlan bp;
        int rc = prepare_batch(h, B, seq_lens, target_lens, nullptr, 0, nullptr, nullptr,
                               host.data(), &bp);
        if (rc) return rc;
        CK(h, cudaMemcpyAsync(G.meta, host.data(), bp.nints * 4, cudaMemcpyHostToDevice, h->st));
        CK(h, cudaStreamSynchronize(h->st));
        const zo_stats_t saved = h->stats;
        cudaStream_t user_st = h->st;
        cudaGraph_t graph = nullptr;
        CK(h, cudaStreamBeginCapture(G.cap, cudaStreamCaptureModeRelaxed));
        h->st = G.cap;
        h->capturing = true;
        const uint64_t k0 = h->stats.kernel_launches;
        launch_gen_factors(h->genU_d, h->n_genU, h->maxU_pairs, h->opt.run_seed, 0, G.step_dev,
                           nu, h->mezo_scale, h->opt.targets.scale_mode == ZO_SCALE_MEZO, h->st);
        rc = launch_batch(h, eps, G.meta, bp, packed_tokens, nullptr, nullptr);
        if (!rc) {
            const int* soff_d = G.meta + (R + 1) + 3 * R;
            launch_row_objective(h->logprob, soff_d, R, B, bp.S, h->L_row, L_plus, L_minus,
                                 h->st);
            launch_objective_sums(h->L_row, B, h->sums, h->st);
            launch_estimate(h->sums, eps, h->c_dev, h->flag_dev, h->st);
            launch_bank_update(h->upd_d, h->n_genU, h->max_upd, h->c_dev, h->flag_dev, lr,
                               h->opt.run_seed, 0, G.step_dev, nu, h->mezo_scale,
                               h->opt.targets.scale_mode == ZO_SCALE_MEZO, h->replay_from,
                               h->coef_hist, h->st);
            launch_advance_step(G.step_dev, h->st);
        }
        const uint64_t launched = h->stats.kernel_launches - k0;
        h->capturing = false;
        h->st = user_st;
        const cudaError_t ce = cudaStreamEndCapture(G.cap, &graph);
        h->stats = saved;
        if (rc) {
            if (graph) cudaGraphDestroy(graph);
            return rc;
        }
        if (ce != cudaSuccess || !graph) FAIL(h, ZO_ERR_CUDA, "step graph capture failed");
        const cudaError_t ie = cudaGraphInstantiate(&G.exec, graph, 0);
        cudaGraphDestroy(graph);
        if (ie != cudaSuccess) {
            G.exec = nullptr;
            FAIL(h, ZO_ERR_CUDA, "step graph instantiation failed");
        }
        G.tok = packed_tokens; G.Lp = L_plus; G.Lm = L_minus; G.eps = eps; G.lr = lr;
        G.slots = h->n_slots;
        G.replay_from = h->replay_from;
        G.lens.assign(seq_lens, seq_lens + B);
        G.tls.assign(target_lens, target_lens + B);
        G.T = bp.T; G.S = bp.S;
        // gen_factors, the score's kernels, objective, sums, estimate, update, step counter
        G.launches = launched + (h->n_genU ? 1 : 0) + 4 + (h->n_genU > 0);
        G.step_next = ~0ull;
        G.captures++;
    }
    // the device step counter is re-seeded when eager steps or a reload moved the host's
    if (G.step_next != step) {
        launch_set_step(G.step_dev, step, h->st);
        h->stats.kernel_launches++;
    }
    CK(h, cudaGraphLaunch(G.exec, h->st));
    G.step_next = step + 1;
    G.replays++;
    h->stats.kernel_launches += G.launches;
    h->stats.tokens_scored += (uint64_t)G.T;
    h->stats.positions_scored += (uint64_t)G.S;
    h->stats.score_calls++;
    h->stats.state_transition_bytes += h->bytes_per_U + update_bytes(h, step);
    h->stats.dense_ref_bytes += h->dense_bytes;
    h->stats.dense_ref_bytes_targets += h->dense_bytes_targets;
    h->stats.steps++;
    h->step++;
    CK(h, cudaGetLastError());
    return ZO_OK;
}

int zo_stats(zo_handle* h, zo_stats_t* out) {
    if (!h || !out) return ZO_ERR_ARG;
    CK(h, cudaStreamSynchronize(h->st));
    for (auto& t : h->tm) timer_harvest(t, true);
    prof_harvest(h->prof, true);
    int flag = 0;
    CK(h, cudaMemcpy(&flag, h->flag_dev, 4, cudaMemcpyDeviceToHost));
    *out = h->stats;
    out->ms_plan = h->tm[0].total_ms;
    out->ms_score = h->tm[1].total_ms;
    out->ms_step = h->tm[2].total_ms;
    out->bank_slots = h->n_slots;
    out->last_error_code = flag ? ZO_ERR_NONFINITE : h->err_code;
    const int ew = gemm_tc_error_word();
    if (ew > 0 && (ew & 1)) out->last_error_code = ZO_ERR_TIMEOUT;
    const int aw = attention_tc_error_word();
    if (aw > 0 && (aw & 1)) out->last_error_code = ZO_ERR_TIMEOUT;
    out->gemm_launches = h->prof.launches;
    out->gemm_ms = h->prof.ms;
    out->gemm_flops = h->prof.fl;
    out->tc_gemm_launches = h->prof.tc_launches;
    out->tc_gemm_ms = h->prof.tc_ms;
    out->tc_gemm_flops = h->prof.tc_fl;
    out->graph_captures = h->graph.captures;
    out->graph_replays = h->graph.replays;
    return ZO_OK;
}

// ---- state ---------------------------------------------------------------------------
namespace {
struct StateHeader {
    uint64_t magic, version, run_seed, step, start_window;
    int32_t nu, rank, n_slots, scale_mode;
    uint32_t matrix_mask, pad;
    uint64_t layer_lo, layer_hi, payload_floats;
};
constexpr uint64_t kMagic = 0x5A4F42414E4B3031ull;   // "ZOBANK01"
}

int zo_save_state(zo_handle* h, void* buf, size_t* n) {
    if (!h || !n) return ZO_ERR_ARG;
    const int r = h->opt.rank;
    uint64_t floats = 0;
    for (auto& L : h->layers)
        for (auto& G : L.g) floats += (uint64_t)G.n_t * r * G.K * h->n_slots;
    const size_t need = sizeof(StateHeader) + floats * 4;
    if (!buf) { *n = need; return ZO_OK; }
    if (*n < need) { *n = need; FAIL(h, ZO_ERR_ARG, "state buffer too small"); }
    StateHeader hd;
    memset(&hd, 0, sizeof(hd));
    hd.magic = kMagic; hd.version = 1; hd.run_seed = h->opt.run_seed; hd.step = h->step;
    hd.start_window = h->n_slots ? (uint64_t)h->slot_window[0] : 0;
    hd.nu = h->opt.lazy_interval; hd.rank = r; hd.n_slots = h->n_slots;
    hd.scale_mode = h->opt.targets.scale_mode; hd.matrix_mask = h->opt.targets.matrix_mask;
    hd.layer_lo = h->opt.targets.layer_mask_lo; hd.layer_hi = h->opt.targets.layer_mask_hi;
    hd.payload_floats = floats;
    memcpy(buf, &hd, sizeof(hd));
    char* p = static_cast<char*>(buf) + sizeof(hd);
    for (auto& L : h->layers)
        for (auto& G : L.g)
            for (int j = 0; j < h->n_slots; ++j) {
                const size_t bytes = (size_t)G.n_t * r * G.K * 4;
                if (!bytes) continue;
                CK(h, cudaMemcpyAsync(p, G.FT + (size_t)G.n_t * r * (1 + j) * G.K, bytes,
                                      cudaMemcpyDeviceToHost, h->st));
                p += bytes;
            }
    CK(h, cudaStreamSynchronize(h->st));
    *n = need;
    return ZO_OK;
}

int zo_load_state(zo_handle* h, const void* buf, size_t n) {
    if (!h || !buf || n < sizeof(StateHeader)) return ZO_ERR_ARG;
    StateHeader hd;
    memcpy(&hd, buf, sizeof(hd));
    if (hd.magic != kMagic || hd.version != 1) FAIL(h, ZO_ERR_ARG, "not a zo state buffer");
    if (hd.run_seed != h->opt.run_seed || hd.nu != h->opt.lazy_interval || hd.rank != h->opt.rank ||
        hd.scale_mode != h->opt.targets.scale_mode || hd.matrix_mask != h->opt.targets.matrix_mask ||
        hd.layer_lo != h->opt.targets.layer_mask_lo || hd.layer_hi != h->opt.targets.layer_mask_hi)
        FAIL(h, ZO_ERR_ARG, "state was saved under different options");
    if (hd.n_slots > h->opt.max_slots) FAIL(h, ZO_ERR_UNSUPPORTED, "state has more slots than max_slots");
    if (n < sizeof(StateHeader) + hd.payload_floats * 4) FAIL(h, ZO_ERR_ARG, "truncated state");
    // clear the bank (rows past the loaded slots must read as zero), re-open every
    // window in order (V re-drawn from the counter stream), then restore A
    const int rr = h->opt.rank;
    for (auto& L : h->layers)
        for (auto& G : L.g) {
            if (G.n_t == 0) continue;
            const size_t ft_rows = ((size_t)G.n_t * rr * (1 + h->opt.max_slots) + 63) / 64 * 64;
            CK(h, cudaMemsetAsync(G.FT, 0, ft_rows * G.K * 4, h->st));
            if (G.FTb) CK(h, cudaMemsetAsync(G.FTb, 0, ft_rows * G.K * 2, h->st));
            CK(h, cudaMemsetAsync(G.EB, 0, (size_t)G.N * h->kcap * esize(h->dt), h->st));
        }
    h->n_slots = 0;
    h->slot_window.clear();
    h->have_plan = false;
    const uint64_t saved_bytes = h->stats.state_transition_bytes;
    for (int j = 0; j < hd.n_slots; ++j) {
        int rc = open_window(h, (hd.start_window + j) * (uint64_t)hd.nu);
        if (rc) return rc;
    }
    h->stats.state_transition_bytes = saved_bytes;
    const int r = h->opt.rank;
    const char* p = static_cast<const char*>(buf) + sizeof(hd);
    for (auto& L : h->layers)
        for (auto& G : L.g)
            for (int j = 0; j < hd.n_slots; ++j) {
                const size_t bytes = (size_t)G.n_t * r * G.K * 4;
                if (!bytes) continue;
                float* dst = G.FT + (size_t)G.n_t * r * (1 + j) * G.K;
                CK(h, cudaMemcpyAsync(dst, p, bytes, cudaMemcpyHostToDevice, h->st));
                if (G.FTb)
                    launch_to_bf16(dst, static_cast<char*>(G.FTb) + (size_t)G.n_t * r * (1 + j) * G.K * 2,
                                   bytes / 4, h->st);
                p += bytes;
            }
    CK(h, cudaStreamSynchronize(h->st));
    h->step = hd.step;
    h->replay_from = -1;     // the loaded accumulator has no coefficient history here
    return ZO_OK;
}

namespace {
Group* find_target(zo_handle* h, int layer, int matrix, int* t) {
    if (layer < 0 || layer >= (int)h->layers.size()) return nullptr;
    for (auto& G : h->layers[layer].g)
        for (int i = 0; i < G.n_t; ++i)
            if (G.mats[i] == matrix) { *t = i; return &G; }
    return nullptr;
}
}  // namespace

int zo_read_factors(zo_plan* plan, int32_t layer, int32_t matrix, float* U_host, float* V_host) {
    if (!plan || !plan->h) return ZO_ERR_ARG;
    zo_handle* h = plan->h;
    int t = 0;
    Group* G = find_target(h, layer, matrix, &t);
    if (!G) FAIL(h, ZO_ERR_ARG, "not a target matrix");
    const int r = h->opt.rank;
    if (U_host) {
        if (h->genU32_d)      // bf16 models keep U in bf16: draw the fp32 rows for the copy
            launch_gen_factors(h->genU32_d, h->n_genU, h->maxU_pairs, h->opt.run_seed,
                               plan->step, nullptr, (uint64_t)h->opt.lazy_interval,
                               h->mezo_scale, h->opt.targets.scale_mode == ZO_SCALE_MEZO, h->st);
        std::vector<float> ut((size_t)r * G->K);
        CK(h, cudaMemcpyAsync(ut.data(), G->FT + (size_t)t * r * G->K, ut.size() * 4,
                              cudaMemcpyDeviceToHost, h->st));
        CK(h, cudaStreamSynchronize(h->st));
        for (int c = 0; c < r; ++c)
            for (int i = 0; i < G->K; ++i) U_host[(size_t)i * r + c] = ut[(size_t)c * G->K + i];
    }
    if (V_host) {
        CK(h, cudaMemcpyAsync(V_host, G->Vcur[t], (size_t)G->d_out[t] * r * 4,
                              cudaMemcpyDeviceToHost, h->st));
        CK(h, cudaStreamSynchronize(h->st));
    }
    return ZO_OK;
}

int zo_read_bank(zo_handle* h, int32_t layer, int32_t matrix, int32_t slot, float* A_host) {
    if (!h || !A_host) return ZO_ERR_ARG;
    int t = 0;
    Group* G = find_target(h, layer, matrix, &t);
    if (!G) FAIL(h, ZO_ERR_ARG, "not a target matrix");
    if (slot < 0 || slot >= h->n_slots) FAIL(h, ZO_ERR_ARG, "no such bank slot");
    const int r = h->opt.rank;
    std::vector<float> at((size_t)r * G->K);
    CK(h, cudaMemcpyAsync(at.data(), G->FT + (size_t)(G->n_t * r * (1 + slot) + t * r) * G->K,
                          at.size() * 4, cudaMemcpyDeviceToHost, h->st));
    CK(h, cudaStreamSynchronize(h->st));
    for (int c = 0; c < r; ++c)
        for (int i = 0; i < G->K; ++i) A_host[(size_t)i * r + c] = at[(size_t)c * G->K + i];
    return ZO_OK;
}

int zo_init_tensor(void* dev, uint64_t n, uint64_t weight_seed, uint32_t layer, uint32_t tensor,
                   float std_, float mean, int32_t dtype, void* stream) {
    if (!dev || (dtype != ZO_DTYPE_FP32 && dtype != ZO_DTYPE_BF16)) return ZO_ERR_ARG;
    launch_init_tensor(dev, n, zo::weight_key(weight_seed, layer, tensor), std_, mean,
                       dtype == ZO_DTYPE_BF16 ? E_BF16 : E_F32, static_cast<cudaStream_t>(stream));
    return cudaGetLastError() == cudaSuccess ? ZO_OK : ZO_ERR_CUDA;
}

}  // extern "C"
