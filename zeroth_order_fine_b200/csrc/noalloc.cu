// zo_op_lm_head_logprob_noalloc: the lm_head log-probability op with its
// scratch in a fixed, library-owned device array instead of a caller
// workspace.
//
// Who needs it: code that must not allocate device memory at call time and
// has no workspace of its own to lend -- for instance a serving process whose
// device memory is wholly owned by another runtime's pool (a stray
// cudaMalloc there fails or fragments the pool), or a latency-critical loop
// that is forbidden to touch the allocator after start-up.  Such a caller
// still passes its inputs and outputs; only the scratch moves here.
//
// The array below is loaded with the library on every GPU that uses it and
// stays resident until the process exits.  Calls share it: two calls whose
// kernels overlap on a GPU (different streams without ordering) race on it
// and give wrong results, so order them on one stream.
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "../../include/zo.h"
#include "../../include/zo_ops.h"
#include "kernels.h"

namespace zo {
namespace {

// 4 MiB of scratch: per-(row, vocab tile) running max and exp-sum, then one
// target logit per row.  The limit is on 2 * n_rows * tiles + n_rows floats.
constexpr size_t kNoAllocFloats = (size_t)1 << 20;
static __device__ __align__(256) float g_lse_scratch[kNoAllocFloats];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_addr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device, looked up once
// per device (host code only sees a host-side stand-in under the array's
// name, which a kernel must never be given).
int scratch_on_current_device(float** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ZO_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_lse_scratch) != cudaSuccess || !p) return ZO_ERR_CUDA;
        g_addr[dev] = static_cast<float*>(p);
    }
    *out = g_addr[dev];
    return ZO_OK;
}

}  // namespace
}  // namespace zo

using namespace zo;

extern "C" {

size_t zo_op_lm_head_noalloc_capacity(void) { return kNoAllocFloats; }

int zo_op_lm_head_logprob_noalloc(const void* h, const void* E, const int32_t* targets,
                                  int32_t n_rows, int32_t vocab, int32_t d, int32_t dtype,
                                  float* logprob, int32_t impl, void* stream) {
    if (!h || !E || !targets || !logprob || n_rows < 0 || vocab <= 0 || d <= 0) return ZO_ERR_ARG;
    if (dtype != ZO_DTYPE_FP32 && dtype != ZO_DTYPE_BF16) return ZO_ERR_ARG;
    if (impl != ZO_IMPL_AUTO && impl != ZO_IMPL_CUDA_CORES && impl != ZO_IMPL_TENSOR_CORES)
        return ZO_ERR_ARG;
    if (n_rows == 0) return ZO_OK;
    const int t = dtype == ZO_DTYPE_BF16 ? E_BF16 : E_F32;
    GemmArgs g;
    memset(&g, 0, sizeof(g));
    g.A = h; g.lda = d; g.a_type = t;
    g.B = E; g.ldb = d; g.b_type = t;
    g.M = n_rows; g.N = vocab; g.K = d;
    g.epi = EPI_LSE;
    const bool tc = impl != ZO_IMPL_CUDA_CORES && dtype == ZO_DTYPE_BF16 && gemm_tc_supported(g);
    if (impl == ZO_IMPL_TENSOR_CORES && !tc) return ZO_ERR_UNSUPPORTED;
    const int tiles = tc ? gemm_tc_col_tiles(vocab) : gemm_lse_col_tiles(vocab);
    // the whole request must fit the fixed array: reject, never fall back to allocating
    const size_t need = 2 * (size_t)n_rows * tiles + (size_t)n_rows;
    if (need > kNoAllocFloats) return ZO_ERR_UNSUPPORTED;
    float* base = nullptr;
    const int rc = scratch_on_current_device(&base);
    if (rc) return rc;
    float* pmax = base;
    float* psum = base + (size_t)n_rows * tiles;
    float* tgt = psum + (size_t)n_rows * tiles;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // The array keeps the previous call's values.  Every partial is rewritten
    // below; the target logits are set to NaN first so a row whose target is
    // outside [0, vocab) reads NaN, never a stale value.
    if (cudaMemsetAsync(tgt, 0xFF, (size_t)n_rows * sizeof(float), st) != cudaSuccess)
        return ZO_ERR_CUDA;
    g.targets = targets; g.part_max = pmax; g.part_sum = psum; g.tgt_logit = tgt;
    g.n_col_tiles = tiles;
    if (tc) {
        if (gemm_tc(g, st)) return ZO_ERR_CUDA;
    } else {
        gemm_simt(g, st);
    }
    launch_lse_merge(pmax, psum, tgt, n_rows, tiles, logprob, st);
    return cudaGetLastError() == cudaSuccess ? ZO_OK : ZO_ERR_CUDA;
}

}  // extern "C"
