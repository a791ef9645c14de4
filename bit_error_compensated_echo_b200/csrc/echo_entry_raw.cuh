// echo_entry_raw.cuh -- the entry pass without the compensator: quantize and pack
// (operation: include/echo.h; conventions: echo_common.cuh)
#pragma once

#include "echo_common.cuh"

namespace echo {

// ------------------------------------------------------------ echo_entry, uncompensated
//
// The uncompensated entry quantizes the raw inputs: no states, 2.5 bytes
// per element, and a per-group cost (absmax exchange, the scale's division
// and reciprocal, index arithmetic) that is large next to the per-element
// work.  Here each thread owns 4 consecutive vectors (32 elements) of one
// group, so that cost is paid once per 32 elements: a group of G is G/32
// threads (G = 32: one thread, no exchange), and the thread's 4 code words
// (8 for 8-bit codes) leave in one (two) 16-byte store.  The 4 loads of a
// warp are 64 bytes apart per lane; together they read whole lines.
// Chunk o's codes and scales go to dst.codes[o] / dst.scales[o], as in the
// compensated entry.
// Grid: x over the slab's vectors / (4 * kThreads), y = rank * P + chunk.
constexpr int kRawVPT = 4;
// Resident blocks per SM the register allocation must allow.  The kernel's
// loads are all issued before its arithmetic, so the bytes in flight grow
// with the resident warps: 6 blocks (40 registers, a few spilled to local
// memory) measured 1.83 ms per 1 GiB-per-rank launch against 1.95 ms at 4
// blocks (56 registers, no spill) and 1.90 ms at 5.
constexpr int kRawMinBlocks = 6;

inline unsigned entry_raw_blocks(int64_t v_count) {
    constexpr int64_t per = (int64_t)kThreads * kRawVPT;
    return (unsigned)((v_count + per - 1) / per);
}

template <int G, int BITS>
__global__ void __launch_bounds__(kThreads, kRawMinBlocks)
echo_entry_raw_kernel(const __grid_constant__ InPtrs x, const __grid_constant__ ChunkDst dst,
                      int64_t n_vec, int64_t chunk_vec, Slab sl, int P, Consts k) {
    constexpr int VPG = G / kVec;            // vectors per group: 4, 8 or 16
    constexpr int TPG = VPG / kRawVPT;       // threads per group: 1, 2 or 4
    const int r = blockIdx.y / P, o = blockIdx.y % P;
    const int64_t t = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const bool valid = t < sl.v_count / kRawVPT;
    const int64_t vc = sl.v_begin + t * kRawVPT;          // first vector, in chunk o
    const int64_t j0 = (int64_t)o * chunk_vec + vc;         // first vector, in rank r
    const float2 z = splat2(k.neg_zero);

    float v[kRawVPT][8];
#pragma unroll
    for (int q = 0; q < kRawVPT; ++q) {
        if (valid) {
            bf16x8_to_f32(x.p[r][j0 + q], v[q]);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) v[q][i] = 0.0f;
        }
    }
    float a = 0.0f;
#pragma unroll
    for (int q = 0; q < kRawVPT; ++q)
#pragma unroll
        for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[q][i]));
    a = group_absmax<TPG>(a);                // every lane takes part
    const GroupScale gs = make_group_scale<BITS>(a);
    Packed8<BITS> w[kRawVPT];
    float kf[8];
#pragma unroll
    for (int q = 0; q < kRawVPT; ++q) w[q] = quantize8_q<BITS>(v[q], gs, kf, z);
    if (!valid) return;

    uint4 *cd = reinterpret_cast<uint4 *>(reinterpret_cast<uint32_t *>(dst.codes[o]) +
                                          ((int64_t)r * n_vec + vc) * (BITS / 4));
    if (BITS == 4) {
        cd[0] = make_uint4(w[0].w[0], w[1].w[0], w[2].w[0], w[3].w[0]);
    } else {
        cd[0] = make_uint4(w[0].w[0], w[0].w[BITS / 4 - 1], w[1].w[0], w[1].w[BITS / 4 - 1]);
        cd[1] = make_uint4(w[2].w[0], w[2].w[BITS / 4 - 1], w[3].w[0], w[3].w[BITS / 4 - 1]);
    }
    if ((threadIdx.x & (TPG - 1)) == 0)
        dst.scales[o][(int64_t)r * (n_vec / VPG) + vc / VPG] = gs.scale;
}

}  // namespace echo
