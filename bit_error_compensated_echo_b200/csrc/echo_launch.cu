// echo_launch.cu -- the one translation unit that instantiates the kernels
// of echo_*.cuh, behind the launchers declared in echo_launch.h.
#include "echo_entry.cuh"
#include "echo_entry_raw.cuh"
#include "echo_exit.cuh"
#include "echo_fixup.cuh"
#include "echo_launch.h"
#include "echo_reduce.cuh"

namespace echo {
namespace {

// ---- entry
template <int G, bool COMP, bool DEFER, int BITS>
void entry_t(const Bufs &b, const InPtrs &x, int rows, int rank0, int64_t er_chunk_vec, Slab sl,
             cudaStream_t st) {
    dim3 grid(entry_blocks<COMP>(sl.v_count), (unsigned)(rows * b.P));
    echo_entry_kernel<G, COMP, DEFER, BITS><<<grid, kThreads, 0, st>>>(
        x, b.m_fast, b.m_slow, b.codes, b.scales, b.e_req, b.n_vec, b.chunk_vec, sl, b.P, b.k,
        rank0, er_chunk_vec);
}

template <int G, int BITS>
void entry_raw_t(const Bufs &b, const InPtrs &x, int rows, Slab sl, cudaStream_t st) {
    dim3 grid(entry_raw_blocks(sl.v_count), (unsigned)(rows * b.P));
    echo_entry_raw_kernel<G, BITS><<<grid, kThreads, 0, st>>>(x, b.codes, b.scales, b.n_vec,
                                                               b.chunk_vec, sl, b.P, b.k);
}

template <int G, int BITS>
void entry_g(const Bufs &b, const InPtrs &x, int rows, int rank0, int64_t er, Slab sl, bool defer,
             cudaStream_t st) {
    if (!b.comp) entry_raw_t<G, BITS>(b, x, rows, sl, st);
    else if (defer) entry_t<G, true, true, BITS>(b, x, rows, rank0, er, sl, st);
    else entry_t<G, true, false, BITS>(b, x, rows, rank0, er, sl, st);
}

template <int BITS>
void entry_b(const Bufs &b, const InPtrs &x, int rows, int rank0, int64_t er, Slab sl, bool defer,
             cudaStream_t st) {
    switch (b.G) {
        case 32: entry_g<32, BITS>(b, x, rows, rank0, er, sl, defer, st); break;
        case 64: entry_g<64, BITS>(b, x, rows, rank0, er, sl, defer, st); break;
        default: entry_g<128, BITS>(b, x, rows, rank0, er, sl, defer, st); break;
    }
}

// ---- reduce
// the run-time part of a reduce launch: outputs and in-kernel fix-up
struct ReduceOut {
    OutPtrs out;
    int n_out;
    int fix;
};

template <int G, int P, int BITS>
void reduce_t(const Bufs &b, int owners, Slab sl, cudaStream_t st, const ReduceOut &ro) {
    dim3 grid(reduce_blocks(sl.v_count), (unsigned)owners);
    if (b.comp && ro.n_out > 0)
        echo_reduce_kernel<G, P, true, true, BITS><<<grid, kThreads, 0, st>>>(
            b.codes, b.scales, b.rcodes, b.rscales, b.e_req, b.n_vec, b.chunk_vec, sl, b.k,
            ro.out, ro.n_out, b.m_fast, b.m_slow, ro.fix);
    else if (b.comp)
        echo_reduce_kernel<G, P, true, false, BITS><<<grid, kThreads, 0, st>>>(
            b.codes, b.scales, b.rcodes, b.rscales, b.e_req, b.n_vec, b.chunk_vec, sl, b.k,
            ro.out, 0, b.m_fast, b.m_slow, ro.fix);
    else if (ro.n_out > 0)
        echo_reduce_kernel<G, P, false, true, BITS><<<grid, kThreads, 0, st>>>(
            b.codes, b.scales, b.rcodes, b.rscales, b.e_req, b.n_vec, b.chunk_vec, sl, b.k,
            ro.out, ro.n_out, nullptr, nullptr, 0);
    else
        echo_reduce_kernel<G, P, false, false, BITS><<<grid, kThreads, 0, st>>>(
            b.codes, b.scales, b.rcodes, b.rscales, b.e_req, b.n_vec, b.chunk_vec, sl, b.k,
            ro.out, 0, nullptr, nullptr, 0);
}

template <int G, int BITS>
void reduce_g(const Bufs &b, int owners, Slab sl, cudaStream_t st, const ReduceOut &ro) {
    switch (b.P) {
        case 1: reduce_t<G, 1, BITS>(b, owners, sl, st, ro); break;
        case 2: reduce_t<G, 2, BITS>(b, owners, sl, st, ro); break;
        case 3: reduce_t<G, 3, BITS>(b, owners, sl, st, ro); break;
        case 4: reduce_t<G, 4, BITS>(b, owners, sl, st, ro); break;
        case 5: reduce_t<G, 5, BITS>(b, owners, sl, st, ro); break;
        case 6: reduce_t<G, 6, BITS>(b, owners, sl, st, ro); break;
        case 7: reduce_t<G, 7, BITS>(b, owners, sl, st, ro); break;
        default: reduce_t<G, 8, BITS>(b, owners, sl, st, ro); break;
    }
}

template <int BITS>
void reduce_b(const Bufs &b, int owners, Slab sl, cudaStream_t st, const ReduceOut &ro) {
    switch (b.G) {
        case 32: reduce_g<32, BITS>(b, owners, sl, st, ro); break;
        case 64: reduce_g<64, BITS>(b, owners, sl, st, ro); break;
        default: reduce_g<128, BITS>(b, owners, sl, st, ro); break;
    }
}

// ---- exit
template <int G, int BITS>
void exit_g(const Bufs &b, const OutPtrs &out, int n_out, int owners, Slab sl, cudaStream_t st) {
    dim3 grid((unsigned)((sl.v_count + kThreads - 1) / kThreads), (unsigned)owners);
    echo_exit_kernel<G, BITS><<<grid, kThreads, 0, st>>>(b.rcodes, b.rscales, out, n_out,
                                                          b.chunk_vec, sl);
}

template <int BITS>
void exit_b(const Bufs &b, const OutPtrs &out, int n_out, int owners, Slab sl, cudaStream_t st) {
    switch (b.G) {
        case 32: exit_g<32, BITS>(b, out, n_out, owners, sl, st); break;
        case 64: exit_g<64, BITS>(b, out, n_out, owners, sl, st); break;
        default: exit_g<128, BITS>(b, out, n_out, owners, sl, st); break;
    }
}

// ---- reduce-scatter
template <int G, int P, int BITS>
void rs_t(const Bufs &b, const OutPtrs &out, int owners, Slab sl, bool fix, cudaStream_t st) {
    dim3 grid(reduce_blocks(sl.v_count), (unsigned)owners);
    if (!b.comp)
        echo_rs_kernel<G, P, false, false, BITS><<<grid, kThreads, 0, st>>>(
            b.codes, b.scales, out, b.m_fast, b.m_slow, b.e_req, b.n_vec, b.chunk_vec, sl, b.k);
    else if (fix)
        echo_rs_kernel<G, P, true, true, BITS><<<grid, kThreads, 0, st>>>(
            b.codes, b.scales, out, b.m_fast, b.m_slow, b.e_req, b.n_vec, b.chunk_vec, sl, b.k);
    else
        echo_rs_kernel<G, P, true, false, BITS><<<grid, kThreads, 0, st>>>(
            b.codes, b.scales, out, b.m_fast, b.m_slow, b.e_req, b.n_vec, b.chunk_vec, sl, b.k);
}

template <int G, int BITS>
void rs_g(const Bufs &b, const OutPtrs &out, int owners, Slab sl, bool fix, cudaStream_t st) {
    switch (b.P) {
        case 1: rs_t<G, 1, BITS>(b, out, owners, sl, fix, st); break;
        case 2: rs_t<G, 2, BITS>(b, out, owners, sl, fix, st); break;
        case 3: rs_t<G, 3, BITS>(b, out, owners, sl, fix, st); break;
        case 4: rs_t<G, 4, BITS>(b, out, owners, sl, fix, st); break;
        case 5: rs_t<G, 5, BITS>(b, out, owners, sl, fix, st); break;
        case 6: rs_t<G, 6, BITS>(b, out, owners, sl, fix, st); break;
        case 7: rs_t<G, 7, BITS>(b, out, owners, sl, fix, st); break;
        default: rs_t<G, 8, BITS>(b, out, owners, sl, fix, st); break;
    }
}

template <int BITS>
void rs_b(const Bufs &b, const OutPtrs &out, int owners, Slab sl, bool fix, cudaStream_t st) {
    switch (b.G) {
        case 32: rs_g<32, BITS>(b, out, owners, sl, fix, st); break;
        case 64: rs_g<64, BITS>(b, out, owners, sl, fix, st); break;
        default: rs_g<128, BITS>(b, out, owners, sl, fix, st); break;
    }
}

}  // namespace

void launch_entry(const Bufs &b, const InPtrs &x, int rows, int rank0, int64_t er_chunk_vec,
                  Slab sl, bool defer, cudaStream_t st) {
    if (b.bits == 8) entry_b<8>(b, x, rows, rank0, er_chunk_vec, sl, defer, st);
    else entry_b<4>(b, x, rows, rank0, er_chunk_vec, sl, defer, st);
}

void launch_reduce(const Bufs &b, int owners, Slab sl, cudaStream_t st, const OutPtrs *out,
                   int n_out, bool fix) {
    ReduceOut ro{};
    if (out && n_out > 0) {
        ro.out = *out;
        ro.n_out = n_out;
    }
    ro.fix = (fix && b.comp) ? 1 : 0;
    if (b.bits == 8) reduce_b<8>(b, owners, sl, st, ro);
    else reduce_b<4>(b, owners, sl, st, ro);
}

void launch_exit(const Bufs &b, const OutPtrs &out, int n_out, int owners, Slab sl,
                 cudaStream_t st) {
    if (b.bits == 8) exit_b<8>(b, out, n_out, owners, sl, st);
    else exit_b<4>(b, out, n_out, owners, sl, st);
}

void launch_rs(const Bufs &b, const OutPtrs &out, int owners, Slab sl, bool fix,
               cudaStream_t st) {
    if (b.bits == 8) rs_b<8>(b, out, owners, sl, fix, st);
    else rs_b<4>(b, out, owners, sl, fix, st);
}

void launch_fill(float *p, int64_t n, float v, cudaStream_t st) {
    int64_t blocks = (n + kThreads - 1) / kThreads;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    echo_fill_kernel<<<(unsigned)blocks, kThreads, 0, st>>>(p, n, v);
}

void launch_fixup(const Bufs &b, const float *src_fast, const float *src_slow, float *dst_fast,
                  float *dst_slow, int ranks, int owners, bool apply, bool only_owner, Slab sl,
                  cudaStream_t st) {
    dim3 grid((unsigned)((sl.v_count + kThreads - 1) / kThreads), (unsigned)owners);
    echo_fixup_kernel<<<grid, kThreads, 0, st>>>(src_fast, src_slow, dst_fast, dst_slow, b.e_req,
                                                 b.n_vec, b.chunk_vec, sl, ranks, apply ? 1 : 0,
                                                 only_owner ? 1 : 0, b.k);
}

}  // namespace echo
