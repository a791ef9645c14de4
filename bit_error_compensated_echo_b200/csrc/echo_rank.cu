// echo_rank.cu -- the rank plan and the C ABI declared in include/echo_rank.h.
//
// A rank plan owns this rank's EMA states ([N] fp32 each) and e_req of its
// own chunk ([C] fp32).  The stage calls launch the same kernels as the
// plan of P virtual ranks, on the caller's exchange buffers, which keep the
// virtual plan's layouts:
//   entry  : one input row (rows = 1), grid y = the P chunks, the row's
//            rank index for the deferred fix-up, e_req of one chunk
//   reduce : the P received chunks are the P rows of a "message" of C
//            elements with a single owner chunk
//   exit   : the gathered reduced chunks are the virtual plan's reduced
//            transport; one output instead of P
// The owner fix-up of the EXIT mode runs in the reduce kernel, and that of
// the SIDE mode in its own kernel; both work on this rank's chunk of the
// state through pointers offset by rank*C.
//
// The fused transport replaces both exchanges by the kernels' own accesses
// to peer memory: entry_peers stores chunk o into rank o's receive buffer,
// exit_peers loads owner o's reduced chunk from owner o's buffer.  The
// buffers peers reach live in the plan's window, one cudaMalloc (so that one
// IPC handle maps all of it), created on first use.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <new>

#include "echo.h"
#include "echo_host.h"
#include "echo_launch.h"
#include "echo_rank.h"

using namespace echo;

struct echo_rank_plan {
    echo_config cfg;
    int bits = 4;                     // code width of the calls
    int rank = 0;
    int64_t C = 0;                    // elements per chunk
    int64_t n_vec = 0, chunk_vec = 0; // vectors per row and per chunk
    Consts k{};
    char *ws = nullptr;
    float *m_fast = nullptr, *m_slow = nullptr, *e_req = nullptr;
    bool entered = false;        // an entry ran since the last reduce
    char *win = nullptr;         // the window: recv codes, recv scales, red codes, red scales
    echo_rank_window_layout wl{};
    bool side_inflight = false;  // a side-stream fix-up may still run
    cudaEvent_t ev_reduced = nullptr, ev_side_done = nullptr;
};

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

// The window ends in a guard zone of this many kWindowGuardByte bytes.
constexpr size_t kWindowGuardBytes = 4096;
constexpr int kWindowGuardByte = 0xA5;

size_t rank_ws_bytes(const echo_config &c) {
    if (!c.compensate) return 0;
    return 2 * align_up((size_t)c.N * 4) + align_up((size_t)(c.N / c.P) * 4);
}

Bufs base_bufs(const echo_rank_plan *p) {
    Bufs b;
    b.P = p->cfg.P;
    b.G = p->cfg.G;
    b.bits = p->bits;
    b.comp = p->cfg.compensate != 0;
    b.k = p->k;
    b.e_req = p->e_req;
    return b;
}

Slab chunk_slab(const echo_rank_plan *p) { return Slab{0, p->chunk_vec}; }

cudaError_t order_after_side(echo_rank_plan *p, cudaStream_t st) {
    if (!p->side_inflight) return cudaSuccess;
    return cudaStreamWaitEvent(st, p->ev_side_done, 0);
}

// The owner fix-up (state += (1-beta)*e_req) on this rank's chunk of src,
// written to dst (src == dst: in place).
void own_chunk_fixup(echo_rank_plan *p, const float *src_f, const float *src_s, float *dst_f,
                     float *dst_s, cudaStream_t st) {
    Bufs b = base_bufs(p);
    b.n_vec = p->chunk_vec;
    b.chunk_vec = p->chunk_vec;
    const int64_t off = (int64_t)p->rank * p->C;
    launch_fixup(b, src_f + off, src_s + off, dst_f + off, dst_s + off, 1, 1, true, true,
                 chunk_slab(p), st);
}

// Step 7 after a reduce or reduce-scatter, by the plan's mode.  in_kernel:
// the launch just made already applied it (EXIT mode).
echo_status after_reduce(echo_rank_plan *p, cudaStream_t st, cudaStream_t side, bool in_kernel) {
    if (!p->cfg.compensate) return ECHO_OK;
    switch (p->cfg.fixup) {
        case ECHO_FIXUP_DEFERRED:   // e_req now holds it; the next entry applies it
            return ECHO_OK;
        case ECHO_FIXUP_EXIT:
            if (!in_kernel) {
                own_chunk_fixup(p, p->m_fast, p->m_slow, p->m_fast, p->m_slow, st);
                ECHO_TRY(cudaGetLastError());
            }
            return ECHO_OK;
        default: {  // SIDE
            cudaStream_t fs = side ? side : st;
            if (side) {
                ECHO_TRY(cudaEventRecord(p->ev_reduced, st));
                ECHO_TRY(cudaStreamWaitEvent(side, p->ev_reduced, 0));
            }
            own_chunk_fixup(p, p->m_fast, p->m_slow, p->m_fast, p->m_slow, fs);
            ECHO_TRY(cudaGetLastError());
            if (side) {
                ECHO_TRY(cudaEventRecord(p->ev_side_done, side));
                p->side_inflight = true;
            }
            return ECHO_OK;
        }
    }
}

}  // namespace

extern "C" {

echo_status echo_rank_exchange_bytes(const echo_config *cfg, size_t *chunk_code_bytes,
                                     size_t *chunk_scale_bytes) {
    const echo_status v = validate_config(cfg);
    if (v != ECHO_OK) return v;
    if (!chunk_code_bytes || !chunk_scale_bytes) return ECHO_ERR_INVALID_ARG;
    const size_t C = (size_t)(cfg->N / cfg->P);
    *chunk_code_bytes = C * (size_t)cfg->bits / 8;
    *chunk_scale_bytes = C / (size_t)cfg->G * 4;
    return ECHO_OK;
}

size_t echo_rank_workspace_bytes(const echo_config *cfg) {
    if (validate_config(cfg) != ECHO_OK) return 0;
    return rank_ws_bytes(*cfg);
}

echo_status echo_rank_plan_create(echo_rank_plan **out, const echo_config *cfg, int32_t rank) {
    if (!out) return ECHO_ERR_INVALID_ARG;
    *out = nullptr;
    const echo_status v = validate_config(cfg);
    if (v != ECHO_OK) return v;
    if (rank < 0 || rank >= cfg->P) return ECHO_ERR_INVALID_ARG;
    DeviceGuard guard(cfg->device);
    if (guard.err != cudaSuccess) return ECHO_ERR_CUDA;

    echo_rank_plan *p = new (std::nothrow) echo_rank_plan();
    if (!p) return ECHO_ERR_OOM;
    p->cfg = *cfg;
    p->rank = rank;
    p->bits = cfg->bits;
    p->C = cfg->N / cfg->P;
    p->n_vec = cfg->N / kVec;
    p->chunk_vec = p->n_vec / cfg->P;
    p->k = make_consts(*cfg);
    cudaError_t e = cudaSuccess;
    const size_t bytes = rank_ws_bytes(*cfg);
    if (bytes) {
        e = cudaMalloc((void **)&p->ws, bytes);
        if (e != cudaSuccess) {
            cudaGetLastError();
            delete p;
            return from_cuda(e);
        }
        p->m_fast = (float *)p->ws;
        p->m_slow = (float *)(p->ws + align_up((size_t)cfg->N * 4));
        p->e_req = (float *)(p->ws + 2 * align_up((size_t)cfg->N * 4));
        e = cudaMemset(p->ws, 0, bytes);
        if (e == cudaSuccess && p->cfg.compensate) {
            launch_fill(p->e_req, p->C, kNoFixup, nullptr);
            e = cudaGetLastError();
        }
    }
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->ev_reduced, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->ev_side_done, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        echo_rank_plan_destroy(p);
        return from_cuda(e);
    }
    *out = p;
    return ECHO_OK;
}

echo_status echo_rank_plan_destroy(echo_rank_plan *p) {
    if (!p) return ECHO_OK;
    DeviceGuard guard(p->cfg.device);
    cudaError_t e = cudaDeviceSynchronize();
    if (p->ev_reduced) cudaEventDestroy(p->ev_reduced);
    if (p->win) cudaFree(p->win);
    if (p->ev_side_done) cudaEventDestroy(p->ev_side_done);
    if (p->ws) cudaFree(p->ws);
    delete p;
    return from_cuda(e);
}

echo_status echo_rank_entry(echo_rank_plan *p, const void *x, void *send_codes,
                            float *send_scales, void *stream) {
    if (!p || !x || !send_codes || !send_scales) return ECHO_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(send_codes) || !aligned4(send_scales))
        return ECHO_ERR_ALIGNMENT;
    DeviceGuard guard(p->cfg.device);
    if (guard.err != cudaSuccess) return ECHO_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    ECHO_TRY(order_after_side(p, st));
    // e_req is -0 (a no-op) when no fix-up is pending
    const bool defer = p->cfg.compensate && p->cfg.fixup == ECHO_FIXUP_DEFERRED;

    Bufs b = base_bufs(p);
    b.m_fast = p->m_fast;
    b.m_slow = p->m_slow;
    b.codes = (uint32_t *)send_codes;
    b.scales = send_scales;
    b.n_vec = p->n_vec;
    b.chunk_vec = p->chunk_vec;
    InPtrs xi{};
    xi.p[0] = (const uint4 *)x;
    launch_entry(b, xi, 1, p->rank, 0, chunk_slab(p), defer, st);
    ECHO_TRY(cudaGetLastError());
    p->entered = true;
    return ECHO_OK;
}

echo_status echo_rank_reduce(echo_rank_plan *p, const void *recv_codes, const float *recv_scales,
                             void *red_codes, float *red_scales, void *stream, void *side_stream) {
    if (!p || !recv_codes || !recv_scales || !red_codes || !red_scales)
        return ECHO_ERR_INVALID_ARG;
    if (!p->entered) return ECHO_ERR_INVALID_ARG;
    if (!aligned16(recv_codes) || !aligned16(red_codes) || !aligned4(recv_scales) ||
        !aligned4(red_scales))
        return ECHO_ERR_ALIGNMENT;
    DeviceGuard guard(p->cfg.device);
    if (guard.err != cudaSuccess) return ECHO_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    // a side-stream fix-up under capture leaves in the graph an event that the
    // plan's next call would wait on
    if (side_stream && p->cfg.compensate && p->cfg.fixup == ECHO_FIXUP_SIDE && capturing(st))
        return ECHO_ERR_UNSUPPORTED;

    Bufs b = base_bufs(p);
    b.codes = (uint32_t *)recv_codes;
    b.scales = (float *)recv_scales;
    b.rcodes = (uint32_t *)red_codes;
    b.rscales = red_scales;
    b.n_vec = p->chunk_vec;       // a received row is one chunk
    b.chunk_vec = p->chunk_vec;
    const bool fix = p->cfg.compensate && p->cfg.fixup == ECHO_FIXUP_EXIT;
    if (fix) {                    // the fix-up in the reduce: this rank's chunk of its state
        const int64_t off = (int64_t)p->rank * p->C;
        b.m_fast = p->m_fast + off;
        b.m_slow = p->m_slow + off;
    }
    launch_reduce(b, 1, chunk_slab(p), st, nullptr, 0, fix);
    ECHO_TRY(cudaGetLastError());
    p->entered = false;
    return after_reduce(p, st, (cudaStream_t)side_stream, fix);
}

echo_status echo_rank_exit(echo_rank_plan *p, const void *all_codes, const float *all_scales,
                           void *out, void *stream) {
    if (!p || !all_codes || !all_scales || !out) return ECHO_ERR_INVALID_ARG;
    if (!aligned16(all_codes) || !aligned16(out) || !aligned4(all_scales))
        return ECHO_ERR_ALIGNMENT;
    DeviceGuard guard(p->cfg.device);
    if (guard.err != cudaSuccess) return ECHO_ERR_CUDA;
    Bufs b = base_bufs(p);
    b.rcodes = (uint32_t *)all_codes;
    b.rscales = (float *)all_scales;
    b.n_vec = p->n_vec;
    b.chunk_vec = p->chunk_vec;
    OutPtrs yo{};
    yo.p[0] = (uint4 *)out;
    launch_exit(b, yo, 1, p->cfg.P, chunk_slab(p), (cudaStream_t)stream);
    ECHO_TRY(cudaGetLastError());
    return ECHO_OK;
}

echo_status echo_rank_reduce_scatter(echo_rank_plan *p, const void *recv_codes,
                                     const float *recv_scales, void *out, void *stream,
                                     void *side_stream) {
    if (!p || !recv_codes || !recv_scales || !out) return ECHO_ERR_INVALID_ARG;
    if (!p->entered) return ECHO_ERR_INVALID_ARG;
    if (!aligned16(recv_codes) || !aligned16(out) || !aligned4(recv_scales))
        return ECHO_ERR_ALIGNMENT;
    DeviceGuard guard(p->cfg.device);
    if (guard.err != cudaSuccess) return ECHO_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    // a side-stream fix-up under capture leaves in the graph an event that the
    // plan's next call would wait on
    if (side_stream && p->cfg.compensate && p->cfg.fixup == ECHO_FIXUP_SIDE && capturing(st))
        return ECHO_ERR_UNSUPPORTED;
    const bool fix = p->cfg.compensate && p->cfg.fixup == ECHO_FIXUP_EXIT;

    Bufs b = base_bufs(p);
    b.codes = (uint32_t *)recv_codes;
    b.scales = (float *)recv_scales;
    if (p->cfg.compensate) {
        const int64_t off = (int64_t)p->rank * p->C;   // this rank's chunk of its state
        b.m_fast = p->m_fast + off;
        b.m_slow = p->m_slow + off;
    }
    b.n_vec = p->chunk_vec;
    b.chunk_vec = p->chunk_vec;
    OutPtrs yo{};
    yo.p[0] = (uint4 *)out;
    launch_rs(b, yo, 1, chunk_slab(p), fix, st);
    ECHO_TRY(cudaGetLastError());
    p->entered = false;
    return after_reduce(p, st, (cudaStream_t)side_stream, fix);
}

echo_status echo_rank_reset_state(echo_rank_plan *p, void *stream) {
    if (!p) return ECHO_ERR_INVALID_ARG;
    p->entered = false;
    if (!p->cfg.compensate) return ECHO_OK;
    DeviceGuard guard(p->cfg.device);
    if (guard.err != cudaSuccess) return ECHO_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    ECHO_TRY(order_after_side(p, st));
    const size_t bytes = (size_t)p->cfg.N * 4;
    ECHO_TRY(cudaMemsetAsync(p->m_fast, 0, bytes, st));
    ECHO_TRY(cudaMemsetAsync(p->m_slow, 0, bytes, st));
    launch_fill(p->e_req, p->C, kNoFixup, st);
    ECHO_TRY(cudaGetLastError());
    return ECHO_OK;
}

echo_status echo_rank_get_state(echo_rank_plan *p, float *m_fast, float *m_slow, void *stream) {
    if (!p || !m_fast || !m_slow || !p->cfg.compensate) return ECHO_ERR_INVALID_ARG;
    if (!aligned16(m_fast) || !aligned16(m_slow)) return ECHO_ERR_ALIGNMENT;
    DeviceGuard guard(p->cfg.device);
    if (guard.err != cudaSuccess) return ECHO_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    ECHO_TRY(order_after_side(p, st));
    const size_t bytes = (size_t)p->cfg.N * 4;
    ECHO_TRY(cudaMemcpyAsync(m_fast, p->m_fast, bytes, cudaMemcpyDeviceToDevice, st));
    ECHO_TRY(cudaMemcpyAsync(m_slow, p->m_slow, bytes, cudaMemcpyDeviceToDevice, st));
    if (p->cfg.fixup == ECHO_FIXUP_DEFERRED) {   // -0 in e_req when none is pending
        own_chunk_fixup(p, m_fast, m_slow, m_fast, m_slow, st);
        ECHO_TRY(cudaGetLastError());
    }
    return ECHO_OK;
}

echo_status echo_rank_set_state(echo_rank_plan *p, const float *m_fast, const float *m_slow,
                                void *stream) {
    if (!p || !m_fast || !m_slow || !p->cfg.compensate) return ECHO_ERR_INVALID_ARG;
    if (!aligned16(m_fast) || !aligned16(m_slow)) return ECHO_ERR_ALIGNMENT;
    DeviceGuard guard(p->cfg.device);
    if (guard.err != cudaSuccess) return ECHO_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    ECHO_TRY(order_after_side(p, st));
    const size_t bytes = (size_t)p->cfg.N * 4;
    ECHO_TRY(cudaMemcpyAsync(p->m_fast, m_fast, bytes, cudaMemcpyDeviceToDevice, st));
    ECHO_TRY(cudaMemcpyAsync(p->m_slow, m_slow, bytes, cudaMemcpyDeviceToDevice, st));
    launch_fill(p->e_req, p->C, kNoFixup, st);
    ECHO_TRY(cudaGetLastError());
    p->entered = false;
    return ECHO_OK;
}

echo_status echo_rank_plan_set_bits(echo_rank_plan *p, int32_t bits) {
    if (!p) return ECHO_ERR_INVALID_ARG;
    if ((bits != 4 && bits != 8) || bits > p->cfg.bits) return ECHO_ERR_UNSUPPORTED;
    p->bits = bits;
    return ECHO_OK;
}

int32_t echo_rank_launches_per_call(const echo_rank_plan *p) {
    if (!p) return 0;
    const bool own_kernel = p->cfg.compensate && p->cfg.fixup == ECHO_FIXUP_SIDE;
    return own_kernel ? 4 : 3;
}

// ------------------------------------------------------------ fused transport

echo_status echo_rank_window(echo_rank_plan *p, echo_rank_window_layout *out) {
    if (!p || !out) return ECHO_ERR_INVALID_ARG;
    if (!p->win) {
        const size_t P = (size_t)p->cfg.P, C = (size_t)p->C;
        const size_t cb = C * (size_t)p->cfg.bits / 8, cs = C / (size_t)p->cfg.G * 4;
        echo_rank_window_layout L{};
        size_t off = 0;
        auto take = [&](size_t bytes) {
            const size_t at = off;
            off += align_up(bytes);
            return at;
        };
        L.recv_codes = take(P * cb);
        L.recv_scales = take(P * cs);
        L.red_codes = take(cb);
        L.red_scales = take(cs);
        L.guard = off;                       // written by no kernel: overrun checks
        L.guard_bytes = kWindowGuardBytes;
        L.bytes = off + kWindowGuardBytes;
        DeviceGuard guard(p->cfg.device);
        if (guard.err != cudaSuccess) return ECHO_ERR_CUDA;
        cudaError_t e = cudaMalloc((void **)&p->win, L.bytes);
        if (e == cudaSuccess) e = cudaMemset(p->win, 0, L.guard);
        if (e == cudaSuccess) e = cudaMemset(p->win + L.guard, kWindowGuardByte, L.guard_bytes);
        if (e != cudaSuccess) {
            if (p->win) cudaFree(p->win);
            p->win = nullptr;
            cudaGetLastError();
            return from_cuda(e);
        }
        L.base = p->win;
        p->wl = L;
    }
    *out = p->wl;
    return ECHO_OK;
}

echo_status echo_rank_entry_peers(echo_rank_plan *p, const void *x, void *const *recv_codes_peers,
                                  float *const *recv_scales_peers, void *stream) {
    if (!p || !x || !recv_codes_peers || !recv_scales_peers) return ECHO_ERR_INVALID_ARG;
    const int P = p->cfg.P;
    for (int o = 0; o < P; ++o) {
        if (!recv_codes_peers[o] || !recv_scales_peers[o]) return ECHO_ERR_INVALID_ARG;
        if (!aligned16(recv_codes_peers[o]) || !aligned4(recv_scales_peers[o]))
            return ECHO_ERR_ALIGNMENT;
    }
    if (!aligned16(x)) return ECHO_ERR_ALIGNMENT;
    DeviceGuard guard(p->cfg.device);
    if (guard.err != cudaSuccess) return ECHO_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    ECHO_TRY(order_after_side(p, st));
    // e_req is -0 (a no-op) when no fix-up is pending
    const bool defer = p->cfg.compensate && p->cfg.fixup == ECHO_FIXUP_DEFERRED;

    Bufs b = base_bufs(p);
    b.m_fast = p->m_fast;
    b.m_slow = p->m_slow;
    b.n_vec = p->n_vec;
    b.chunk_vec = p->chunk_vec;
    // this rank's slot in rank o's receive buffer: part `rank` of [P][cb]
    const int64_t cb = p->C * p->bits / 8, cs = p->C / p->cfg.G;
    ChunkDst d{};
    for (int o = 0; o < P; ++o) {
        d.codes[o] = static_cast<uint8_t *>(recv_codes_peers[o]) + (int64_t)p->rank * cb;
        d.scales[o] = recv_scales_peers[o] + (int64_t)p->rank * cs;
    }
    InPtrs xi{};
    xi.p[0] = (const uint4 *)x;
    launch_entry(b, xi, 1, p->rank, 0, chunk_slab(p), defer, st, &d);
    ECHO_TRY(cudaGetLastError());
    p->entered = true;
    return ECHO_OK;
}

echo_status echo_rank_exit_peers(echo_rank_plan *p, const void *const *red_codes_peers,
                                 const float *const *red_scales_peers, void *out, void *stream) {
    if (!p || !red_codes_peers || !red_scales_peers || !out) return ECHO_ERR_INVALID_ARG;
    const int P = p->cfg.P;
    ChunkSrc s{};
    for (int o = 0; o < P; ++o) {
        if (!red_codes_peers[o] || !red_scales_peers[o]) return ECHO_ERR_INVALID_ARG;
        if (!aligned16(red_codes_peers[o]) || !aligned4(red_scales_peers[o]))
            return ECHO_ERR_ALIGNMENT;
        s.codes[o] = static_cast<const uint8_t *>(red_codes_peers[o]);
        s.scales[o] = red_scales_peers[o];
    }
    if (!aligned16(out)) return ECHO_ERR_ALIGNMENT;
    DeviceGuard guard(p->cfg.device);
    if (guard.err != cudaSuccess) return ECHO_ERR_CUDA;
    Bufs b = base_bufs(p);
    b.n_vec = p->n_vec;
    b.chunk_vec = p->chunk_vec;
    OutPtrs yo{};
    yo.p[0] = (uint4 *)out;
    launch_exit(b, yo, 1, P, chunk_slab(p), (cudaStream_t)stream, &s);
    ECHO_TRY(cudaGetLastError());
    return ECHO_OK;
}

echo_status echo_ipc_handle_get(const void *device_ptr, echo_ipc_handle *out) {
    if (!device_ptr || !out) return ECHO_ERR_INVALID_ARG;
    static_assert(sizeof(cudaIpcMemHandle_t) == sizeof(out->bytes), "IPC handle size");
    cudaIpcMemHandle_t h;
    const cudaError_t e = cudaIpcGetMemHandle(&h, const_cast<void *>(device_ptr));
    if (e != cudaSuccess) {
        cudaGetLastError();
        return from_cuda(e);
    }
    std::memcpy(out->bytes, &h, sizeof(h));
    return ECHO_OK;
}

echo_status echo_ipc_open(const echo_ipc_handle *handle, int32_t device, void **out) {
    if (!handle || !out || device < 0) return ECHO_ERR_INVALID_ARG;
    *out = nullptr;
    DeviceGuard guard(device);
    if (guard.err != cudaSuccess) return ECHO_ERR_CUDA;
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handle->bytes, sizeof(h));
    const cudaError_t e = cudaIpcOpenMemHandle(out, h, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess) {
        cudaGetLastError();
        *out = nullptr;
        return from_cuda(e);
    }
    return ECHO_OK;
}

echo_status echo_ipc_close(void *ptr, int32_t device) {
    if (!ptr || device < 0) return ECHO_ERR_INVALID_ARG;
    DeviceGuard guard(device);
    if (guard.err != cudaSuccess) return ECHO_ERR_CUDA;
    const cudaError_t e = cudaIpcCloseMemHandle(ptr);
    if (e != cudaSuccess) cudaGetLastError();
    return from_cuda(e);
}

}  // extern "C"
