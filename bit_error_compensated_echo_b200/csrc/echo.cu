// echo.cu -- the plan and the C ABI declared in include/echo.h.
//
// A plan owns one device allocation carved into the EMA states, the entry
// transport (packed codes + scales of all P ranks: the 4-bit "wire" of the
// reduce-scatter), the reduced transport (the wire of the all-gather) and
// e_req.  A call launches the entry and the reduce on the caller's stream
// (the reduce writes every rank's output itself: there is no exit pass on
// one GPU), plus, in side-stream mode, the owner fix-up on the side stream.
// Host code here only validates, carves memory, orders streams and
// launches: every step of the arithmetic runs in the kernels of echo_*.cuh.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <new>
#include <vector>

#include "echo.h"
#include "echo_host.h"
#include "echo_launch.h"

using namespace echo;

namespace {

constexpr size_t kAlign = 256;
// After the workspace's sub-buffers: a guard zone of this many bytes filled
// with kGuardByte at plan creation, which no kernel writes (tests read it
// through echo_debug_view_get to catch an overrun of the last sub-buffer).
constexpr size_t kGuardBytes = 4096;
constexpr int kGuardByte = 0xA5;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

struct Layout {
    size_t m_fast, m_slow, codes, scales, rcodes, rscales, e_req, total;
};

Layout layout_of(const echo_config &c) {
    Layout L{};
    const size_t N = (size_t)c.N, P = (size_t)c.P, G = (size_t)c.G;
    const bool comp = c.compensate != 0;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t at = off;
        off += align_up(bytes);
        return at;
    };
    L.m_fast = comp ? take(P * N * 4) : 0;
    L.m_slow = comp ? take(P * N * 4) : 0;
    const size_t B = (size_t)c.bits;
    L.codes = take(P * N * B / 8);
    L.scales = take(P * (N / G) * 4);
    L.rcodes = take(N * B / 8);
    L.rscales = take((N / G) * 4);
    L.e_req = comp ? take(N * 4) : 0;
    L.total = off;
    return L;
}

// Slabs of the pipelined host call: copies in, kernels and copies out of
// successive slabs overlap, and only the first slab's copy in and the last
// one's copy out are not hidden.
constexpr int kHostSlabs = 32;

struct ProfRecord {
    cudaEvent_t ev[6];   // entry start, entry end, reduce end, call end (no exit pass on one
                         // GPU: exit_ms stays ~0), fixup start, fixup end
    bool side;
    int kernels;         // kernels on the main stream
};

}  // namespace

echo_status echo::validate_config(const echo_config *c) {
    if (!c) return ECHO_ERR_INVALID_ARG;
    if (c->P < 1 || c->P > ECHO_MAX_RANKS) return ECHO_ERR_UNSUPPORTED;
    if (c->G != 32 && c->G != 64 && c->G != 128) return ECHO_ERR_UNSUPPORTED;
    if (c->N <= 0 || c->N % ((int64_t)c->P * c->G) != 0) return ECHO_ERR_SHAPE;
    auto unit = [](float v) { return std::isfinite(v) && v >= 0.0f && v <= 1.0f; };
    if (!unit(c->alpha) || !unit(c->beta_fast) || !unit(c->beta_slow))
        return ECHO_ERR_INVALID_ARG;
    if (c->compensate != 0 && c->compensate != 1) return ECHO_ERR_INVALID_ARG;
    if (c->fixup < ECHO_FIXUP_EXIT || c->fixup > ECHO_FIXUP_DEFERRED)
        return ECHO_ERR_INVALID_ARG;
    if (c->device < 0) return ECHO_ERR_INVALID_ARG;
    if (c->bits != 4 && c->bits != 8) return ECHO_ERR_UNSUPPORTED;
    return ECHO_OK;
}

struct echo_plan {
    echo_config cfg;
    Layout L;
    int64_t n_vec = 0, chunk_vec = 0;
    Bufs b;                          // the workspace as the launchers see it
    char *ws = nullptr;
    float *m_fast = nullptr, *m_slow = nullptr, *scales = nullptr, *rscales = nullptr,
          *e_req = nullptr;
    uint32_t *codes = nullptr, *rcodes = nullptr;
    bool pending = false;            // a deferred-mode call ran since the last reset (host view)
    bool side_inflight = false;      // a side-stream fix-up may still run
    cudaEvent_t ev_reduced = nullptr, ev_side_done = nullptr;
    void *stage = nullptr;           // host-call staging: [P][N] in, [P][N] out
    cudaStream_t hstream[3] = {nullptr, nullptr, nullptr};  // host call: copy in, compute, copy out
    cudaEvent_t hev[2 * kHostSlabs + 2] = {};               // host call: per-slab and boundary events
    bool profiling = false;
    std::vector<ProfRecord> records;
    std::vector<cudaEvent_t> pool;
    echo_profile totals{};
};

namespace {

cudaEvent_t take_event(echo_plan *p) {
    if (!p->pool.empty()) {
        cudaEvent_t e = p->pool.back();
        p->pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

// The plan's launches: all P virtual ranks in one grid, e_req over every
// owner chunk, the state rows in rank order.
void plan_entry(echo_plan *p, const InPtrs &x, Slab sl, cudaStream_t st, bool defer) {
    launch_entry(p->b, x, p->cfg.P, 0, p->chunk_vec, sl, defer, st);
}

// The reduce; fix applies the owner fix-up in it.  On one GPU the reduce
// also writes every rank's output: the owner that requantizes a value
// computes y = bf16(k2*scale2) from the requantized codes anyway, and
// writing it to the P outputs there replaces the exit pass (re-reading the
// reduced codes and a launch).  A/B at P = 8, G = 128, bit-identical:
// uncompensated call at 1 GiB per rank 5.10 -> 4.80 ms when this was
// introduced; compensated calls, once the reduce stored 32 bytes at a time,
// 14.03 -> 13.77 ms at 1 GiB per rank, 0.883 -> 0.863 ms at 64 MiB,
// 67.7 -> 63.5 us at 4 MiB (with 16-byte stores the separate exit pass had
// been faster from 2 MiB per rank up).  The exit kernel remains the rank
// path's all-gather.
void plan_reduce(echo_plan *p, const OutPtrs &out, Slab sl, cudaStream_t st, bool fix) {
    launch_reduce(p->b, p->cfg.P, sl, st, &out, p->cfg.P, fix);
}

void plan_rs(echo_plan *p, const OutPtrs &out, Slab sl, cudaStream_t st, bool fix) {
    launch_rs(p->b, out, p->cfg.P, sl, fix, st);
}

void plan_fixup(echo_plan *p, const float *sf, const float *ss, float *df, float *ds, bool apply,
                bool only_owner, Slab sl, cudaStream_t st) {
    launch_fixup(p->b, sf, ss, df, ds, p->cfg.P, p->cfg.P, apply, only_owner, sl, st);
}

Slab whole(const echo_plan *p) { return Slab{0, p->chunk_vec}; }

// Wait (on st) for a side-stream fix-up that may still be writing the state.
cudaError_t order_after_side(echo_plan *p, cudaStream_t st) {
    if (!p->side_inflight) return cudaSuccess;
    return cudaStreamWaitEvent(st, p->ev_side_done, 0);
}

}  // namespace

extern "C" {

void echo_config_default(echo_config *cfg) {
    if (!cfg) return;
    std::memset(cfg, 0, sizeof *cfg);
    cfg->compensate = 1;
    cfg->alpha = 0.5f;
    cfg->beta_fast = 0.5f;
    cfg->beta_slow = 0.95f;
    cfg->device = 0;
    cfg->fixup = ECHO_FIXUP_EXIT;
    cfg->bits = 4;
}

size_t echo_workspace_bytes(const echo_config *cfg) {
    if (validate_config(cfg) != ECHO_OK) return 0;
    return layout_of(*cfg).total + kGuardBytes;
}

echo_status echo_plan_create(echo_plan **out, const echo_config *cfg) {
    if (!out) return ECHO_ERR_INVALID_ARG;
    *out = nullptr;
    echo_status v = validate_config(cfg);
    if (v != ECHO_OK) return v;

    DeviceGuard guard(cfg->device);
    if (guard.err != cudaSuccess) return ECHO_ERR_CUDA;

    echo_plan *p = new (std::nothrow) echo_plan();
    if (!p) return ECHO_ERR_OOM;
    p->cfg = *cfg;
    p->L = layout_of(*cfg);
    p->n_vec = cfg->N / kVec;
    p->chunk_vec = p->n_vec / cfg->P;
    p->b.k = make_consts(*cfg);

    cudaError_t e = cudaMalloc((void **)&p->ws, p->L.total + kGuardBytes);
    if (e != cudaSuccess) {
        cudaGetLastError();
        delete p;
        return from_cuda(e);
    }
    e = cudaMemset(p->ws + p->L.total, kGuardByte, kGuardBytes);
    if (e != cudaSuccess) {
        cudaGetLastError();
        cudaFree(p->ws);
        delete p;
        return from_cuda(e);
    }
    const bool comp = cfg->compensate != 0;
    p->m_fast = comp ? (float *)(p->ws + p->L.m_fast) : nullptr;
    p->m_slow = comp ? (float *)(p->ws + p->L.m_slow) : nullptr;
    p->codes = (uint32_t *)(p->ws + p->L.codes);
    p->scales = (float *)(p->ws + p->L.scales);
    p->rcodes = (uint32_t *)(p->ws + p->L.rcodes);
    p->rscales = (float *)(p->ws + p->L.rscales);
    p->e_req = comp ? (float *)(p->ws + p->L.e_req) : nullptr;
    p->b.m_fast = p->m_fast;
    p->b.m_slow = p->m_slow;
    p->b.codes = p->codes;
    p->b.scales = p->scales;
    p->b.rcodes = p->rcodes;
    p->b.rscales = p->rscales;
    p->b.e_req = p->e_req;
    p->b.n_vec = p->n_vec;
    p->b.chunk_vec = p->chunk_vec;
    p->b.P = cfg->P;
    p->b.G = cfg->G;
    p->b.bits = cfg->bits;
    p->b.comp = comp;

    e = cudaEventCreateWithFlags(&p->ev_reduced, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->ev_side_done, cudaEventDisableTiming);
    if (e == cudaSuccess && comp) {
        e = cudaMemset(p->m_fast, 0, (size_t)cfg->P * cfg->N * 4);
        if (e == cudaSuccess) e = cudaMemset(p->m_slow, 0, (size_t)cfg->P * cfg->N * 4);
        if (e == cudaSuccess) {
            launch_fill(p->e_req, cfg->N, kNoFixup, nullptr);
            e = cudaGetLastError();
        }
    }
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        echo_plan_destroy(p);
        return from_cuda(e);
    }
    *out = p;
    return ECHO_OK;
}

echo_status echo_plan_destroy(echo_plan *p) {
    if (!p) return ECHO_OK;
    DeviceGuard guard(p->cfg.device);
    cudaError_t e = cudaDeviceSynchronize();
    for (auto &r : p->records)
        for (auto ev : r.ev)
            if (ev) cudaEventDestroy(ev);
    for (auto ev : p->pool) cudaEventDestroy(ev);
    for (auto ev : p->hev)
        if (ev) cudaEventDestroy(ev);
    for (auto hs : p->hstream)
        if (hs) cudaStreamDestroy(hs);
    if (p->ev_reduced) cudaEventDestroy(p->ev_reduced);
    if (p->ev_side_done) cudaEventDestroy(p->ev_side_done);
    if (p->stage) cudaFree(p->stage);
    if (p->ws) cudaFree(p->ws);
    delete p;
    return from_cuda(e);
}

int32_t echo_launches_per_call(const echo_plan *p) {
    if (!p) return 0;
    const int side = (p->cfg.compensate && p->cfg.fixup == ECHO_FIXUP_SIDE) ? 1 : 0;
    return 2 + side;
}

echo_status echo_allreduce(echo_plan *p, const void *const *in, void *const *out, void *stream,
                           void *side_stream) {
    if (!p || !in || !out) return ECHO_ERR_INVALID_ARG;
    const int P = p->cfg.P;
    const size_t bytes = (size_t)p->cfg.N * 2;
    InPtrs xi{};
    OutPtrs yo{};
    for (int r = 0; r < P; ++r) {
        if (!in[r] || !out[r]) return ECHO_ERR_INVALID_ARG;
        if (!aligned16(in[r]) || !aligned16(out[r])) return ECHO_ERR_ALIGNMENT;
        xi.p[r] = (const uint4 *)in[r];
        yo.p[r] = (uint4 *)out[r];
    }
    // outputs receive the same values at the same offsets: they must not
    // overlap one another (inputs are only read, before any output write)
    for (int r = 0; r < P; ++r)
        for (int s = r + 1; s < P; ++s) {
            const char *a = (const char *)out[r], *b = (const char *)out[s];
            if (a < b + bytes && b < a + bytes) return ECHO_ERR_INVALID_ARG;
        }

    DeviceGuard guard(p->cfg.device);
    if (guard.err != cudaSuccess) return ECHO_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    cudaStream_t side = (cudaStream_t)side_stream;
    const bool comp = p->cfg.compensate != 0;
    const int mode = p->cfg.fixup;
    // Under stream capture: a side-stream fix-up leaves in the graph an event
    // that the plan's next call would wait on, and profiling keeps per-call
    // events on the host; replays would honour neither.
    if (capturing(st) && (p->profiling || (comp && mode == ECHO_FIXUP_SIDE && side)))
        return ECHO_ERR_UNSUPPORTED;

    ProfRecord rec{};
    rec.kernels = 2;
    if (p->profiling) {
        for (int i = 0; i < 6; ++i) rec.ev[i] = nullptr;
        for (int i = 0; i < 4; ++i) {
            rec.ev[i] = take_event(p);
            if (!rec.ev[i]) return ECHO_ERR_CUDA;
        }
    }

    ECHO_TRY(order_after_side(p, st));
    const bool defer = comp && mode == ECHO_FIXUP_DEFERRED;   // e_req is -0 if none pending

    if (p->profiling) ECHO_TRY(cudaEventRecord(rec.ev[0], st));
    plan_entry(p, xi, whole(p), st, defer);
    ECHO_TRY(cudaGetLastError());
    if (p->profiling) ECHO_TRY(cudaEventRecord(rec.ev[1], st));
    const bool fix_in_reduce = comp && mode == ECHO_FIXUP_EXIT;
    const bool fix_on_side = comp && mode == ECHO_FIXUP_SIDE;
    plan_reduce(p, yo, whole(p), st, fix_in_reduce);
    ECHO_TRY(cudaGetLastError());
    if (p->profiling) ECHO_TRY(cudaEventRecord(rec.ev[2], st));
    if (fix_on_side && side) ECHO_TRY(cudaEventRecord(p->ev_reduced, st));
    if (p->profiling) ECHO_TRY(cudaEventRecord(rec.ev[3], st));   // no exit pass on one GPU

    if (fix_on_side) {
        cudaStream_t fs = side ? side : st;
        if (side) ECHO_TRY(cudaStreamWaitEvent(side, p->ev_reduced, 0));
        if (p->profiling) {
            rec.ev[4] = take_event(p);
            rec.ev[5] = take_event(p);
            if (!rec.ev[4] || !rec.ev[5]) return ECHO_ERR_CUDA;
            rec.side = true;
            ECHO_TRY(cudaEventRecord(rec.ev[4], fs));
        }
        plan_fixup(p, p->m_fast, p->m_slow, p->m_fast, p->m_slow, true, true, whole(p), fs);
        ECHO_TRY(cudaGetLastError());
        if (p->profiling) ECHO_TRY(cudaEventRecord(rec.ev[5], fs));
        if (side) {
            ECHO_TRY(cudaEventRecord(p->ev_side_done, side));
            p->side_inflight = true;
        } else {
            p->side_inflight = false;
        }
    }
    if (comp && mode == ECHO_FIXUP_DEFERRED) p->pending = true;
    if (p->profiling) p->records.push_back(rec);
    return ECHO_OK;
}

echo_status echo_reduce_scatter(echo_plan *p, const void *const *in, void *const *out,
                                void *stream, void *side_stream) {
    if (!p || !in || !out) return ECHO_ERR_INVALID_ARG;
    const int P = p->cfg.P;
    const size_t out_bytes = (size_t)p->cfg.N / P * 2;
    InPtrs xi{};
    OutPtrs yo{};
    for (int r = 0; r < P; ++r) {
        if (!in[r] || !out[r]) return ECHO_ERR_INVALID_ARG;
        if (!aligned16(in[r]) || !aligned16(out[r])) return ECHO_ERR_ALIGNMENT;
        xi.p[r] = (const uint4 *)in[r];
        yo.p[r] = (uint4 *)out[r];
    }
    for (int r = 0; r < P; ++r)
        for (int s2 = r + 1; s2 < P; ++s2) {
            const char *a = (const char *)out[r], *b = (const char *)out[s2];
            if (a < b + out_bytes && b < a + out_bytes) return ECHO_ERR_INVALID_ARG;
        }
    DeviceGuard guard(p->cfg.device);
    if (guard.err != cudaSuccess) return ECHO_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    cudaStream_t side = (cudaStream_t)side_stream;
    const bool comp = p->cfg.compensate != 0;
    const int mode = p->cfg.fixup;
    // Under stream capture: a side-stream fix-up leaves in the graph an event
    // that the plan's next call would wait on, and profiling keeps per-call
    // events on the host; replays would honour neither.
    if (capturing(st) && (p->profiling || (comp && mode == ECHO_FIXUP_SIDE && side)))
        return ECHO_ERR_UNSUPPORTED;

    ProfRecord rec{};
    rec.kernels = 2;
    if (p->profiling) {
        for (int i = 0; i < 4; ++i) {
            rec.ev[i] = take_event(p);
            if (!rec.ev[i]) return ECHO_ERR_CUDA;
        }
    }
    ECHO_TRY(order_after_side(p, st));
    const bool defer = comp && mode == ECHO_FIXUP_DEFERRED;   // e_req is -0 if none pending
    if (p->profiling) ECHO_TRY(cudaEventRecord(rec.ev[0], st));
    plan_entry(p, xi, whole(p), st, defer);
    ECHO_TRY(cudaGetLastError());
    if (p->profiling) ECHO_TRY(cudaEventRecord(rec.ev[1], st));
    plan_rs(p, yo, whole(p), st, comp && mode == ECHO_FIXUP_EXIT);
    ECHO_TRY(cudaGetLastError());
    if (p->profiling) {
        ECHO_TRY(cudaEventRecord(rec.ev[2], st));
        ECHO_TRY(cudaEventRecord(rec.ev[3], st));
    }
    if (comp && mode == ECHO_FIXUP_SIDE) {
        cudaStream_t fs = side ? side : st;
        if (side) {
            ECHO_TRY(cudaEventRecord(p->ev_reduced, st));
            ECHO_TRY(cudaStreamWaitEvent(side, p->ev_reduced, 0));
        }
        if (p->profiling) {
            rec.ev[4] = take_event(p);
            rec.ev[5] = take_event(p);
            if (!rec.ev[4] || !rec.ev[5]) return ECHO_ERR_CUDA;
            rec.side = true;
            ECHO_TRY(cudaEventRecord(rec.ev[4], fs));
        }
        plan_fixup(p, p->m_fast, p->m_slow, p->m_fast, p->m_slow, true, true, whole(p), fs);
        ECHO_TRY(cudaGetLastError());
        if (p->profiling) ECHO_TRY(cudaEventRecord(rec.ev[5], fs));
        if (side) {
            ECHO_TRY(cudaEventRecord(p->ev_side_done, side));
            p->side_inflight = true;
        }
    }
    if (comp && mode == ECHO_FIXUP_DEFERRED) p->pending = true;
    if (p->profiling) p->records.push_back(rec);
    return ECHO_OK;
}

echo_status echo_allreduce_host(echo_plan *p, const void *const *in_host, void *const *out_host,
                                void *stream) {
    if (!p || !in_host || !out_host) return ECHO_ERR_INVALID_ARG;
    const int P = p->cfg.P;
    for (int r = 0; r < P; ++r)
        if (!in_host[r] || !out_host[r]) return ECHO_ERR_INVALID_ARG;
    DeviceGuard guard(p->cfg.device);
    if (guard.err != cudaSuccess) return ECHO_ERR_CUDA;
    // host copies on internal streams, allocated on first use: not for capture
    if (capturing((cudaStream_t)stream)) return ECHO_ERR_UNSUPPORTED;
    const size_t bytes = (size_t)p->cfg.N * 2;
    if (!p->stage) {
        cudaError_t e = cudaMalloc(&p->stage, 2 * (size_t)P * bytes);
        if (e != cudaSuccess) {
            cudaGetLastError();
            p->stage = nullptr;
            return from_cuda(e);
        }
    }
    if (!p->hstream[0]) {
        for (auto &hs : p->hstream) ECHO_TRY(cudaStreamCreateWithFlags(&hs, cudaStreamNonBlocking));
        for (auto &ev : p->hev) ECHO_TRY(cudaEventCreateWithFlags(&ev, cudaEventDisableTiming));
    }
    cudaStream_t st = (cudaStream_t)stream;
    cudaStream_t s_in = p->hstream[0], s_comp = p->hstream[1], s_out = p->hstream[2];
    cudaEvent_t ev_start = p->hev[2 * kHostSlabs], ev_done = p->hev[2 * kHostSlabs + 1];

    InPtrs xi{};
    OutPtrs yo{};
    char *din[ECHO_MAX_RANKS];
    char *dout[ECHO_MAX_RANKS];
    for (int r = 0; r < P; ++r) {
        din[r] = (char *)p->stage + (size_t)r * bytes;
        dout[r] = (char *)p->stage + (size_t)(P + r) * bytes;
        xi.p[r] = (const uint4 *)din[r];
        yo.p[r] = (uint4 *)dout[r];
    }

    // Slab k is vectors [k*sv, (k+1)*sv) of every owner chunk: one strided
    // copy per rank moves it (P rows of sv*16 bytes, pitch chunk_vec*16).
    const int64_t align = p->cfg.G / kVec;  // slab edges on group edges (and even)
    int64_t nslab = kHostSlabs;
    if (p->chunk_vec / align < nslab) nslab = p->chunk_vec / align;
    int64_t sv = (p->chunk_vec + nslab - 1) / nslab;
    sv = (sv + align - 1) / align * align;
    const size_t pitch = (size_t)p->chunk_vec * 16;

    ECHO_TRY(cudaEventRecord(ev_start, st));
    for (auto hs : p->hstream) ECHO_TRY(cudaStreamWaitEvent(hs, ev_start, 0));
    ECHO_TRY(order_after_side(p, s_comp));
    p->side_inflight = false;
    const bool comp = p->cfg.compensate != 0;
    const bool deferred = comp && p->cfg.fixup == ECHO_FIXUP_DEFERRED;
    const bool defer = deferred;   // e_req is -0 if none pending
    for (int64_t k = 0; k < nslab; ++k) {
        const int64_t vb = k * sv;
        if (vb >= p->chunk_vec) break;
        const int64_t vc = vb + sv <= p->chunk_vec ? sv : p->chunk_vec - vb;
        const Slab sl{vb, vc};
        const size_t off = (size_t)vb * 16, width = (size_t)vc * 16;
        for (int r = 0; r < P; ++r)
            ECHO_TRY(cudaMemcpy2DAsync(din[r] + off, pitch, (const char *)in_host[r] + off, pitch,
                                       width, (size_t)P, cudaMemcpyHostToDevice, s_in));
        ECHO_TRY(cudaEventRecord(p->hev[2 * k], s_in));
        ECHO_TRY(cudaStreamWaitEvent(s_comp, p->hev[2 * k], 0));
        plan_entry(p, xi, sl, s_comp, defer);
        plan_reduce(p, yo, sl, s_comp, comp && !deferred);
        ECHO_TRY(cudaGetLastError());
        ECHO_TRY(cudaEventRecord(p->hev[2 * k + 1], s_comp));
        ECHO_TRY(cudaStreamWaitEvent(s_out, p->hev[2 * k + 1], 0));
        for (int r = 0; r < P; ++r)
            ECHO_TRY(cudaMemcpy2DAsync((char *)out_host[r] + off, pitch, dout[r] + off, pitch,
                                       width, (size_t)P, cudaMemcpyDeviceToHost, s_out));
    }
    ECHO_TRY(cudaEventRecord(ev_done, s_out));
    ECHO_TRY(cudaStreamWaitEvent(st, ev_done, 0));
    if (deferred) p->pending = true;
    return ECHO_OK;
}

echo_status echo_reset_state(echo_plan *p, void *stream) {
    if (!p) return ECHO_ERR_INVALID_ARG;
    if (!p->cfg.compensate) return ECHO_OK;
    DeviceGuard guard(p->cfg.device);
    if (guard.err != cudaSuccess) return ECHO_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    ECHO_TRY(order_after_side(p, st));
    const size_t bytes = (size_t)p->cfg.P * p->cfg.N * 4;
    ECHO_TRY(cudaMemsetAsync(p->m_fast, 0, bytes, st));
    ECHO_TRY(cudaMemsetAsync(p->m_slow, 0, bytes, st));
    launch_fill(p->e_req, p->cfg.N, kNoFixup, st);
    ECHO_TRY(cudaGetLastError());
    p->pending = false;
    return ECHO_OK;
}

echo_status echo_get_state(echo_plan *p, float *m_fast, float *m_slow, void *stream) {
    if (!p || !m_fast || !m_slow || !p->cfg.compensate) return ECHO_ERR_INVALID_ARG;
    if (!aligned16(m_fast) || !aligned16(m_slow)) return ECHO_ERR_ALIGNMENT;
    DeviceGuard guard(p->cfg.device);
    if (guard.err != cudaSuccess) return ECHO_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    ECHO_TRY(order_after_side(p, st));
    // deferred mode: e_req holds the pending fix-up, or -0 (a no-op) if none is
    // pending; applying it unconditionally is right after graph replays too
    const bool apply = p->cfg.fixup == ECHO_FIXUP_DEFERRED;
    plan_fixup(p, p->m_fast, p->m_slow, m_fast, m_slow, apply, false, whole(p), st);
    ECHO_TRY(cudaGetLastError());
    return ECHO_OK;
}

echo_status echo_set_state(echo_plan *p, const float *m_fast, const float *m_slow, void *stream) {
    if (!p || !m_fast || !m_slow || !p->cfg.compensate) return ECHO_ERR_INVALID_ARG;
    DeviceGuard guard(p->cfg.device);
    if (guard.err != cudaSuccess) return ECHO_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    ECHO_TRY(order_after_side(p, st));
    const size_t bytes = (size_t)p->cfg.P * p->cfg.N * 4;
    ECHO_TRY(cudaMemcpyAsync(p->m_fast, m_fast, bytes, cudaMemcpyDeviceToDevice, st));
    ECHO_TRY(cudaMemcpyAsync(p->m_slow, m_slow, bytes, cudaMemcpyDeviceToDevice, st));
    launch_fill(p->e_req, p->cfg.N, kNoFixup, st);
    ECHO_TRY(cudaGetLastError());
    p->pending = false;
    return ECHO_OK;
}

echo_status echo_debug_view_get(echo_plan *p, echo_debug_view *v) {
    if (!p || !v) return ECHO_ERR_INVALID_ARG;
    v->m_fast = p->m_fast;
    v->m_slow = p->m_slow;
    v->codes = (uint8_t *)p->codes;
    v->scales = p->scales;
    v->rcodes = (uint8_t *)p->rcodes;
    v->rscales = p->rscales;
    v->e_req = p->e_req;
    v->fixup_pending = p->pending ? 1 : 0;
    v->bits = p->b.bits;
    v->guard = (uint8_t *)(p->ws + p->L.total);
    v->guard_bytes = (int64_t)kGuardBytes;
    return ECHO_OK;
}

echo_status echo_plan_set_bits(echo_plan *p, int32_t bits) {
    if (!p) return ECHO_ERR_INVALID_ARG;
    if ((bits != 4 && bits != 8) || bits > p->cfg.bits) return ECHO_ERR_UNSUPPORTED;
    p->b.bits = bits;
    return ECHO_OK;
}

echo_status echo_profile_enable(echo_plan *p, int32_t on) {
    if (!p) return ECHO_ERR_INVALID_ARG;
    p->profiling = on != 0;
    return ECHO_OK;
}

echo_status echo_profile_read(echo_plan *p, echo_profile *out, int32_t reset) {
    if (!p) return ECHO_ERR_INVALID_ARG;
    DeviceGuard guard(p->cfg.device);
    if (guard.err != cudaSuccess) return ECHO_ERR_CUDA;
    for (auto &r : p->records) {
        float ms = 0.0f;
        ECHO_TRY(cudaEventSynchronize(r.ev[3]));
        ECHO_TRY(cudaEventElapsedTime(&ms, r.ev[0], r.ev[1]));
        p->totals.entry_ms += ms;
        ECHO_TRY(cudaEventElapsedTime(&ms, r.ev[1], r.ev[2]));
        p->totals.reduce_ms += ms;
        ECHO_TRY(cudaEventElapsedTime(&ms, r.ev[2], r.ev[3]));
        p->totals.exit_ms += ms;
        p->totals.launches += r.kernels;
        if (r.side) {
            ECHO_TRY(cudaEventSynchronize(r.ev[5]));
            ECHO_TRY(cudaEventElapsedTime(&ms, r.ev[4], r.ev[5]));
            p->totals.fixup_ms += ms;
            p->totals.launches += 1;
        }
        p->totals.calls += 1;
        for (auto ev : r.ev)
            if (ev) p->pool.push_back(ev);
    }
    p->records.clear();
    if (out) *out = p->totals;
    if (reset) p->totals = echo_profile{};
    return ECHO_OK;
}

const char *echo_status_string(echo_status s) {
    switch (s) {
        case ECHO_OK: return "ECHO_OK";
        case ECHO_ERR_INVALID_ARG: return "ECHO_ERR_INVALID_ARG";
        case ECHO_ERR_SHAPE: return "ECHO_ERR_SHAPE";
        case ECHO_ERR_ALIGNMENT: return "ECHO_ERR_ALIGNMENT";
        case ECHO_ERR_UNSUPPORTED: return "ECHO_ERR_UNSUPPORTED";
        case ECHO_ERR_OOM: return "ECHO_ERR_OOM";
        case ECHO_ERR_CUDA: return "ECHO_ERR_CUDA";
        case ECHO_ERR_TIMEOUT: return "ECHO_ERR_TIMEOUT";
    }
    return "ECHO_ERR_UNKNOWN";
}

echo_status echo_device_error_get(int32_t device, int32_t *flags, int32_t clear) {
    if (!flags || device < 0) return ECHO_ERR_INVALID_ARG;
    DeviceGuard guard(device);
    if (guard.err != cudaSuccess) return ECHO_ERR_CUDA;
    ECHO_TRY(device_error_read(flags, clear != 0));
    return (*flags & ECHO_DEVERR_WAIT_TIMEOUT) ? ECHO_ERR_TIMEOUT : ECHO_OK;
}

echo_status echo_selftest_wait_limit(int32_t device) {
    if (device < 0) return ECHO_ERR_INVALID_ARG;
    DeviceGuard guard(device);
    if (guard.err != cudaSuccess) return ECHO_ERR_CUDA;
    cudaStream_t st = nullptr;
    ECHO_TRY(cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking));
    launch_wait_selftest(st);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    cudaStreamDestroy(st);
    return from_cuda(e);
}

int32_t echo_abi_version(void) { return ECHO_ABI_VERSION; }

}  // extern "C"
