// echo_noalloc.cu -- echo_allreduce_noalloc: the same call as
// echo_allreduce (owner fix-up inside the reduce kernel), for callers that
// cannot allocate device memory.  The scratch the kernels pass between each
// other (entry codes and scales, the requantized codes and scales, e_req)
// lives in one file-scope device array instead of a plan's workspace, and
// the caller owns the compensator state.  Nothing here calls cudaMalloc,
// cudaFree or a host allocator.
#include <cuda.h>   // CUcontext and CUresult only; the two driver calls are fetched at run time
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "echo.h"
#include "echo_host.h"
#include "echo_launch.h"

using namespace echo;

// One array per device that loads this code, held until the process exits.
static __device__ __align__(256) unsigned char echo_noalloc_scratch[ECHO_NOALLOC_MAX_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;

// The array's device address belongs to the CUDA context it was looked up
// in.  A device reset, or a caller that makes another context current on
// the device (driver-API users), loads the module anew, at an address the
// old lookup does not know.  So the cache of each device slot is keyed by
// the unique id of the context that was current at the lookup (cuCtxGetId:
// the driver never gives two contexts of one process the same id), and a
// call in any other context looks the address up again.
struct ScratchSlot {
    bool valid = false;
    unsigned long long ctx_id = 0;
    void *addr = nullptr;
};
std::mutex g_scratch_mu;
ScratchSlot g_scratch[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;
bool g_ctx_fns_tried = false;

// The id of the calling thread's current context; false if there is none
// yet or the driver cannot say.  Called with g_scratch_mu held.
bool current_context_id(unsigned long long *id) {
    if (!g_ctx_fns_tried) {
        g_ctx_fns_tried = true;
        void *f = nullptr, *g = nullptr;
        cudaDriverEntryPointQueryResult qf{}, qg{};
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault,
                                             &qf) == cudaSuccess &&
            cudaGetDriverEntryPointByVersion("cuCtxGetId", &g, 12000, cudaEnableDefault, &qg) ==
                cudaSuccess &&
            qf == cudaDriverEntryPointSuccess && qg == cudaDriverEntryPointSuccess) {
            g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(f);
            g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(g);
        }
        cudaGetLastError();
    }
    if (!g_ctx_get_current || !g_ctx_get_id) return false;
    CUcontext ctx = nullptr;
    if (g_ctx_get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return g_ctx_get_id(ctx, id) == CUDA_SUCCESS;
}

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

// The array's device address in the current context of device dev (which
// is current): cached per device and context; the set-up (the lookup with
// cudaGetSymbolAddress, which may load the module into the context) runs
// on the first call in a context, and is refused on a capturing stream,
// where loading a module could break the capture.  Without a context id
// (a driver that cannot give one) every call looks the address up.
echo_status scratch_address(int dev, cudaStream_t st, unsigned char **out) {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    const bool cap = capturing(st);
    if (cap && !g_ctx_fns_tried) return ECHO_ERR_UNSUPPORTED;   // no set-up has run yet
    ScratchSlot &slot = g_scratch[dev];
    unsigned long long id = 0;
    bool have_id = current_context_id(&id);
    if (have_id && slot.valid && slot.ctx_id == id) {
        *out = (unsigned char *)slot.addr;
        return ECHO_OK;
    }
    if (cap) return ECHO_ERR_UNSUPPORTED;
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, echo_noalloc_scratch);
    if (e != cudaSuccess) return from_cuda(e);
    if (!have_id) have_id = current_context_id(&id);   // the lookup bound a context
    slot.valid = have_id;
    slot.ctx_id = id;
    slot.addr = p;
    *out = (unsigned char *)p;
    return ECHO_OK;
}

// The launches of one call, on the array's carved sub-buffers.
void launch_all(const InPtrs &x, const OutPtrs &y, float *mf, float *ms, unsigned char *s,
                const ScratchLayout &L, const echo_config &c, cudaStream_t st) {
    Bufs b;
    b.comp = c.compensate != 0;
    b.m_fast = b.comp ? mf : nullptr;
    b.m_slow = b.comp ? ms : nullptr;
    b.codes = (uint32_t *)(s + L.codes);
    b.scales = (float *)(s + L.scales);
    b.rcodes = (uint32_t *)(s + L.rcodes);
    b.rscales = (float *)(s + L.rscales);
    b.e_req = b.comp ? (float *)(s + L.e_req) : nullptr;
    b.n_vec = c.N / kVec;
    b.chunk_vec = b.n_vec / c.P;
    b.P = c.P;
    b.G = c.G;
    b.bits = 4;
    b.k = make_consts(c);
    const Slab sl{0, b.chunk_vec};
    launch_entry(b, x, c.P, 0, b.chunk_vec, sl, false, st);
    // the reduce writes the outputs and, compensating, applies the owner
    // fix-up (as a plan's calls on one GPU do)
    launch_reduce(b, c.P, sl, st, &y, c.P, b.comp);
}

}  // namespace

extern "C" echo_status echo_allreduce_noalloc(const echo_config *cfg, const void *const *in_device,
                                              void *const *out_device, float *m_fast_device,
                                              float *m_slow_device, void *stream) {
    if (!cfg || !in_device || !out_device) return ECHO_ERR_INVALID_ARG;
    echo_config c = *cfg;
    c.fixup = ECHO_FIXUP_EXIT;   // the fix-up always runs before the call returns here
    const echo_status v = validate_config(&c);
    if (v != ECHO_OK) return v;
    if (cfg->device >= kMaxDevices) return ECHO_ERR_INVALID_ARG;
    if (cfg->bits != 4) return ECHO_ERR_UNSUPPORTED;   // 4-bit codes only
    const int P = cfg->P, G = cfg->G;
    const int64_t N = cfg->N;
    const bool comp = cfg->compensate != 0;

    // the size limit of the shared array, checked before anything else runs
    const ScratchLayout L = scratch_layout(P, N, G, comp);
    if (L.total > (size_t)ECHO_NOALLOC_MAX_SCRATCH_BYTES) return ECHO_ERR_UNSUPPORTED;

    if (comp && (!m_fast_device || !m_slow_device)) return ECHO_ERR_INVALID_ARG;
    if (comp && (!aligned16(m_fast_device) || !aligned16(m_slow_device)))
        return ECHO_ERR_ALIGNMENT;
    InPtrs x{};
    OutPtrs y{};
    const size_t bytes = (size_t)N * 2;
    for (int r = 0; r < P; ++r) {
        if (!in_device[r] || !out_device[r]) return ECHO_ERR_INVALID_ARG;
        if (!aligned16(in_device[r]) || !aligned16(out_device[r])) return ECHO_ERR_ALIGNMENT;
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
    echo_status st = scratch_address(cfg->device, (cudaStream_t)stream, &scratch);
    if (st == ECHO_OK) {
        launch_all(x, y, m_fast_device, m_slow_device, scratch, L, *cfg, (cudaStream_t)stream);
        if (cudaGetLastError() != cudaSuccess) st = ECHO_ERR_CUDA;
    }
    if (prev != cfg->device) cudaSetDevice(prev);
    return st;
}
