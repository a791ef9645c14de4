// echo_noalloc.cu -- echo_allreduce_noalloc: the same call as
// echo_allreduce (fix-up inside the exit kernel), for callers that cannot
// allocate device memory.  The scratch the three kernels pass between each
// other (entry codes and scales, the requantized codes and scales, e_req)
// lives in one file-scope device array instead of a plan's workspace, and
// the caller owns the compensator state.  Nothing here calls cudaMalloc,
// cudaFree or a host allocator.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "echo.h"
#include "echo_entry.cuh"
#include "echo_exit.cuh"
#include "echo_reduce.cuh"

using namespace echo;

// One array per device that loads this code, held until the process exits.
static __device__ __align__(256) unsigned char echo_noalloc_scratch[ECHO_NOALLOC_MAX_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxDevices];  // device address of the array, per device

size_t round256(size_t b) { return (b + 255) / 256 * 256; }

struct ScratchLayout {
    size_t codes, scales, rcodes, rscales, e_req, total;
};

ScratchLayout scratch_layout(int P, int64_t N, int G, bool comp) {
    ScratchLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t at = off;
        off += round256(bytes);
        return at;
    };
    L.codes = take((size_t)P * N / 2);
    L.scales = take((size_t)P * (N / G) * 4);
    L.rcodes = take((size_t)N / 2);
    L.rscales = take((size_t)(N / G) * 4);
    L.e_req = comp ? take((size_t)N * 4) : 0;
    L.total = off;
    return L;
}

// Looks up the array's device address once per device, with that device
// current, and caches it.
cudaError_t scratch_address(int dev, unsigned char **out) {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, echo_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = (unsigned char *)g_scratch_addr[dev];
    return cudaSuccess;
}

bool is_aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

template <int G, int P>
void launch_all(const InPtrs &x, const OutPtrs &y, float *mf, float *ms, unsigned char *s,
                const ScratchLayout &L, int64_t N, bool comp, const Consts &k, cudaStream_t st) {
    const int64_t n_vec = N / kVec, chunk_vec = n_vec / P;
    uint32_t *codes = (uint32_t *)(s + L.codes);
    float *scales = (float *)(s + L.scales);
    uint32_t *rcodes = (uint32_t *)(s + L.rcodes);
    float *rscales = (float *)(s + L.rscales);
    float *e_req = comp ? (float *)(s + L.e_req) : nullptr;
    const Slab sl{0, chunk_vec};
    dim3 g_entry_c(entry_blocks<true>(chunk_vec), (unsigned)(P * P));
    dim3 g_entry_o(entry_blocks<false>(chunk_vec), (unsigned)(P * P));
    dim3 g_chunk((unsigned)((chunk_vec + kThreads - 1) / kThreads), (unsigned)P);
    dim3 g_red(reduce_blocks(chunk_vec), (unsigned)P);
    if (comp) {
        echo_entry_kernel<G, true, false, 4><<<g_entry_c, kThreads, 0, st>>>(
            x, mf, ms, codes, scales, e_req, n_vec, chunk_vec, sl, P, k);
        echo_reduce_kernel<G, P, true, 4><<<g_red, kThreads, 0, st>>>(
            codes, scales, rcodes, rscales, e_req, n_vec, chunk_vec, sl, k.neg_zero);
        echo_exit_kernel<G, true, 4><<<g_chunk, kThreads, 0, st>>>(
            rcodes, rscales, y, P, mf, ms, e_req, n_vec, chunk_vec, sl, k);
    } else {
        echo_entry_kernel<G, false, false, 4><<<g_entry_o, kThreads, 0, st>>>(
            x, nullptr, nullptr, codes, scales, nullptr, n_vec, chunk_vec, sl, P, k);
        echo_reduce_kernel<G, P, false, 4><<<g_red, kThreads, 0, st>>>(
            codes, scales, rcodes, rscales, nullptr, n_vec, chunk_vec, sl, k.neg_zero);
        echo_exit_kernel<G, false, 4><<<g_chunk, kThreads, 0, st>>>(
            rcodes, rscales, y, P, nullptr, nullptr, nullptr, n_vec, chunk_vec, sl, k);
    }
}

template <int G>
void launch_g(int P, const InPtrs &x, const OutPtrs &y, float *mf, float *ms, unsigned char *s,
              const ScratchLayout &L, int64_t N, bool comp, const Consts &k, cudaStream_t st) {
    switch (P) {
        case 1: launch_all<G, 1>(x, y, mf, ms, s, L, N, comp, k, st); break;
        case 2: launch_all<G, 2>(x, y, mf, ms, s, L, N, comp, k, st); break;
        case 3: launch_all<G, 3>(x, y, mf, ms, s, L, N, comp, k, st); break;
        case 4: launch_all<G, 4>(x, y, mf, ms, s, L, N, comp, k, st); break;
        case 5: launch_all<G, 5>(x, y, mf, ms, s, L, N, comp, k, st); break;
        case 6: launch_all<G, 6>(x, y, mf, ms, s, L, N, comp, k, st); break;
        case 7: launch_all<G, 7>(x, y, mf, ms, s, L, N, comp, k, st); break;
        default: launch_all<G, 8>(x, y, mf, ms, s, L, N, comp, k, st); break;
    }
}

}  // namespace

extern "C" echo_status echo_allreduce_noalloc(const echo_config *cfg, const void *const *in_device,
                                              void *const *out_device, float *m_fast_device,
                                              float *m_slow_device, void *stream) {
    if (!cfg || !in_device || !out_device) return ECHO_ERR_INVALID_ARG;
    const int P = cfg->P, G = cfg->G;
    const int64_t N = cfg->N;
    if (P < 1 || P > ECHO_MAX_RANKS) return ECHO_ERR_UNSUPPORTED;
    if (G != 32 && G != 64 && G != 128) return ECHO_ERR_UNSUPPORTED;
    if (N <= 0 || N % ((int64_t)P * G) != 0) return ECHO_ERR_SHAPE;
    auto unit = [](float v) { return std::isfinite(v) && v >= 0.0f && v <= 1.0f; };
    if (!unit(cfg->alpha) || !unit(cfg->beta_fast) || !unit(cfg->beta_slow))
        return ECHO_ERR_INVALID_ARG;
    if (cfg->compensate != 0 && cfg->compensate != 1) return ECHO_ERR_INVALID_ARG;
    if (cfg->device < 0 || cfg->device >= kMaxDevices) return ECHO_ERR_INVALID_ARG;
    if (cfg->bits != 4) return ECHO_ERR_UNSUPPORTED;   // 4-bit codes only
    const bool comp = cfg->compensate != 0;

    // the size limit of the shared array, checked before anything else runs
    const ScratchLayout L = scratch_layout(P, N, G, comp);
    if (L.total > (size_t)ECHO_NOALLOC_MAX_SCRATCH_BYTES) return ECHO_ERR_UNSUPPORTED;

    if (comp && (!m_fast_device || !m_slow_device)) return ECHO_ERR_INVALID_ARG;
    if (comp && (!is_aligned16(m_fast_device) || !is_aligned16(m_slow_device)))
        return ECHO_ERR_ALIGNMENT;
    InPtrs x{};
    OutPtrs y{};
    const size_t bytes = (size_t)N * 2;
    for (int r = 0; r < P; ++r) {
        if (!in_device[r] || !out_device[r]) return ECHO_ERR_INVALID_ARG;
        if (!is_aligned16(in_device[r]) || !is_aligned16(out_device[r])) return ECHO_ERR_ALIGNMENT;
        x.p[r] = (const uint4 *)in_device[r];
        y.p[r] = (uint4 *)out_device[r];
    }
    for (int r = 0; r < P; ++r)
        for (int s = r + 1; s < P; ++s) {
            const char *a = (const char *)out_device[r], *b = (const char *)out_device[s];
            if (a < b + bytes && b < a + bytes) return ECHO_ERR_INVALID_ARG;
        }

    int prev = -1;
    if (cudaGetDevice(&prev) != cudaSuccess) return ECHO_ERR_CUDA;
    if (prev != cfg->device && cudaSetDevice(cfg->device) != cudaSuccess) return ECHO_ERR_CUDA;
    unsigned char *scratch = nullptr;
    cudaError_t e = scratch_address(cfg->device, &scratch);
    if (e == cudaSuccess) {
        Consts k;
        k.alpha = cfg->alpha;
        k.one_m_alpha = 1.0f - cfg->alpha;
        k.beta_fast = cfg->beta_fast;
        k.one_m_beta_fast = 1.0f - cfg->beta_fast;
        k.beta_slow = cfg->beta_slow;
        k.one_m_beta_slow = 1.0f - cfg->beta_slow;
        k.neg_zero = -0.0f;
        cudaStream_t st = (cudaStream_t)stream;
        switch (G) {
            case 32: launch_g<32>(P, x, y, m_fast_device, m_slow_device, scratch, L, N, comp, k, st); break;
            case 64: launch_g<64>(P, x, y, m_fast_device, m_slow_device, scratch, L, N, comp, k, st); break;
            default: launch_g<128>(P, x, y, m_fast_device, m_slow_device, scratch, L, N, comp, k, st); break;
        }
        e = cudaGetLastError();
    }
    if (prev != cfg->device) cudaSetDevice(prev);
    return e == cudaSuccess ? ECHO_OK : ECHO_ERR_CUDA;
}
