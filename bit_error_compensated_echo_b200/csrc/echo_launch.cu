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

// the bounded wait on a barrier that nothing completes (see
// launch_wait_selftest): its limit must run out
__global__ void echo_wait_selftest_kernel() {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        mbar_init_fence();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_bounded(b, 0);
}

// ---- entry
template <int G, bool COMP, bool DEFER, int BITS>
void entry_t(const Bufs &b, const InPtrs &x, int rows, int rank0, int64_t er_chunk_vec, Slab sl,
             cudaStream_t st, const ChunkDst &dst) {
    dim3 grid(entry_blocks<COMP>(sl.v_count), (unsigned)(rows * b.P));
    echo_entry_kernel<G, COMP, DEFER, BITS><<<grid, kThreads, 0, st>>>(
        x, b.m_fast, b.m_slow, dst, b.e_req, b.n_vec, b.chunk_vec, sl, b.P, b.k, rank0,
        er_chunk_vec);
}

template <int G, int BITS>
void entry_raw_t(const Bufs &b, const InPtrs &x, int rows, Slab sl, cudaStream_t st,
                 const ChunkDst &dst) {
    dim3 grid(entry_raw_blocks(sl.v_count), (unsigned)(rows * b.P));
    echo_entry_raw_kernel<G, BITS><<<grid, kThreads, 0, st>>>(x, dst, b.n_vec, b.chunk_vec, sl,
                                                               b.P, b.k);
}

template <int G, int BITS>
void entry_g(const Bufs &b, const InPtrs &x, int rows, int rank0, int64_t er, Slab sl, bool defer,
             cudaStream_t st, const ChunkDst &dst) {
    if (!b.comp) entry_raw_t<G, BITS>(b, x, rows, sl, st, dst);
    else if (defer) entry_t<G, true, true, BITS>(b, x, rows, rank0, er, sl, st, dst);
    else entry_t<G, true, false, BITS>(b, x, rows, rank0, er, sl, st, dst);
}

template <int BITS>
void entry_b(const Bufs &b, const InPtrs &x, int rows, int rank0, int64_t er, Slab sl, bool defer,
             cudaStream_t st, const ChunkDst &dst) {
    switch (b.G) {
        case 32: entry_g<32, BITS>(b, x, rows, rank0, er, sl, defer, st, dst); break;
        case 64: entry_g<64, BITS>(b, x, rows, rank0, er, sl, defer, st, dst); break;
        default: entry_g<128, BITS>(b, x, rows, rank0, er, sl, defer, st, dst); break;
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
    constexpr bool stage_ok = ReduceShape<G, P, false, true, BITS>::STAGE_OK;
    if (b.comp && ro.n_out > 0)
        echo_reduce_kernel<G, P, true, true, BITS, false><<<grid, kThreads, 0, st>>>(
            b.codes, b.scales, b.rcodes, b.rscales, b.e_req, b.n_vec, b.chunk_vec, sl, b.k,
            ro.out, ro.n_out, b.m_fast, b.m_slow, ro.fix);
    else if (b.comp)
        echo_reduce_kernel<G, P, true, false, BITS, false><<<grid, kThreads, 0, st>>>(
            b.codes, b.scales, b.rcodes, b.rscales, b.e_req, b.n_vec, b.chunk_vec, sl, b.k,
            ro.out, 0, b.m_fast, b.m_slow, ro.fix);
    else if (ro.n_out > 0 && stage_ok && sl.v_count / 2 >= kStageMinRuns)
        echo_reduce_kernel<G, P, false, true, BITS, stage_ok><<<grid, kThreads, 0, st>>>(
            b.codes, b.scales, b.rcodes, b.rscales, b.e_req, b.n_vec, b.chunk_vec, sl, b.k,
            ro.out, ro.n_out, nullptr, nullptr, 0);
    else if (ro.n_out > 0)
        echo_reduce_kernel<G, P, false, true, BITS, false><<<grid, kThreads, 0, st>>>(
            b.codes, b.scales, b.rcodes, b.rscales, b.e_req, b.n_vec, b.chunk_vec, sl, b.k,
            ro.out, ro.n_out, nullptr, nullptr, 0);
    else
        echo_reduce_kernel<G, P, false, false, BITS, false><<<grid, kThreads, 0, st>>>(
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
void exit_g(const ChunkSrc &src, int64_t chunk_vec, const OutPtrs &out, int n_out, int owners,
            Slab sl, cudaStream_t st) {
    if (sl.v_count / 2 >= kExitRunMinRuns) {   // a thread per 16-element run
        dim3 grid((unsigned)((sl.v_count / 2 + kThreads - 1) / kThreads), (unsigned)owners);
        echo_exit_run_kernel<G, BITS><<<grid, kThreads, 0, st>>>(src, out, n_out, chunk_vec, sl);
        return;
    }
    dim3 grid((unsigned)((sl.v_count + kThreads - 1) / kThreads), (unsigned)owners);
    echo_exit_kernel<G, BITS><<<grid, kThreads, 0, st>>>(src, out, n_out, chunk_vec, sl);
}

template <int BITS>
void exit_b(const Bufs &b, const ChunkSrc &src, const OutPtrs &out, int n_out, int owners,
            Slab sl, cudaStream_t st) {
    switch (b.G) {
        case 32: exit_g<32, BITS>(src, b.chunk_vec, out, n_out, owners, sl, st); break;
        case 64: exit_g<64, BITS>(src, b.chunk_vec, out, n_out, owners, sl, st); break;
        default: exit_g<128, BITS>(src, b.chunk_vec, out, n_out, owners, sl, st); break;
    }
}

// ---- reduce-scatter
template <int G, int P, int BITS, bool STAGE>
void rs_s(const Bufs &b, const OutPtrs &out, int owners, Slab sl, bool fix, cudaStream_t st) {
    dim3 grid(reduce_blocks(sl.v_count), (unsigned)owners);
    if (!b.comp)
        echo_rs_kernel<G, P, false, false, BITS, STAGE><<<grid, kThreads, 0, st>>>(
            b.codes, b.scales, out, b.m_fast, b.m_slow, b.e_req, b.n_vec, b.chunk_vec, sl, b.k);
    else if (fix)
        echo_rs_kernel<G, P, true, true, BITS, STAGE><<<grid, kThreads, 0, st>>>(
            b.codes, b.scales, out, b.m_fast, b.m_slow, b.e_req, b.n_vec, b.chunk_vec, sl, b.k);
    else
        echo_rs_kernel<G, P, true, false, BITS, STAGE><<<grid, kThreads, 0, st>>>(
            b.codes, b.scales, out, b.m_fast, b.m_slow, b.e_req, b.n_vec, b.chunk_vec, sl, b.k);
}

template <int G, int P, int BITS>
void rs_t(const Bufs &b, const OutPtrs &out, int owners, Slab sl, bool fix, cudaStream_t st) {
    constexpr bool stage_ok = RsShape<G, P, BITS>::STAGE_OK;
    if (stage_ok && sl.v_count / 2 >= kStageMinRuns)
        rs_s<G, P, BITS, stage_ok>(b, out, owners, sl, fix, st);
    else
        rs_s<G, P, BITS, false>(b, out, owners, sl, fix, st);
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

ChunkDst chunks_of(const Bufs &b) {
    ChunkDst d{};
    const int64_t cbytes = b.chunk_vec * b.bits;          // 8 codes of bits/8 bytes per vector
    const int64_t cgroups = b.chunk_vec * kVec / b.G;
    for (int o = 0; o < b.P; ++o) {
        d.codes[o] = reinterpret_cast<uint8_t *>(b.codes) + o * cbytes;
        d.scales[o] = b.scales + o * cgroups;
    }
    return d;
}

ChunkSrc reduced_chunks_of(const Bufs &b) {
    ChunkSrc s{};
    const int64_t cbytes = b.chunk_vec * b.bits;
    const int64_t cgroups = b.chunk_vec * kVec / b.G;
    for (int o = 0; o < b.P; ++o) {
        s.codes[o] = reinterpret_cast<const uint8_t *>(b.rcodes) + o * cbytes;
        s.scales[o] = b.rscales + o * cgroups;
    }
    return s;
}

void launch_entry(const Bufs &b, const InPtrs &x, int rows, int rank0, int64_t er_chunk_vec,
                  Slab sl, bool defer, cudaStream_t st, const ChunkDst *dst) {
    const ChunkDst d = dst ? *dst : chunks_of(b);
    if (b.bits == 8) entry_b<8>(b, x, rows, rank0, er_chunk_vec, sl, defer, st, d);
    else entry_b<4>(b, x, rows, rank0, er_chunk_vec, sl, defer, st, d);
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
                 cudaStream_t st, const ChunkSrc *src) {
    const ChunkSrc s = src ? *src : reduced_chunks_of(b);
    if (b.bits == 8) exit_b<8>(b, s, out, n_out, owners, sl, st);
    else exit_b<4>(b, s, out, n_out, owners, sl, st);
}

void launch_rs(const Bufs &b, const OutPtrs &out, int owners, Slab sl, bool fix,
               cudaStream_t st) {
    if (b.bits == 8) rs_b<8>(b, out, owners, sl, fix, st);
    else rs_b<4>(b, out, owners, sl, fix, st);
}

cudaError_t device_error_read(int32_t *flags, bool clear) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, echo_device_error, sizeof v);
    if (e == cudaSuccess && clear && v != 0) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(echo_device_error, &zero, sizeof zero);
    }
    *flags = v;
    return e;
}

void launch_wait_selftest(cudaStream_t st) { echo_wait_selftest_kernel<<<1, 32, 0, st>>>(); }

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
