// echo_entry.cuh -- the entry pass: correction add, quantize, pack, partial EMA update
// (operation: include/echo.h; conventions: echo_common.cuh)
#pragma once

#include "echo_common.cuh"

namespace echo {

// ------------------------------------------------------------ echo_entry
//
// Correction add + group quantize + pack + partial EMA update, for every
// rank.  Grid: x over the slab's vectors, y = rank * P + owner chunk.
//   COMP  : compensator on (read/write the states)
//   DEFER : apply the previous call's pending owner fix-up first
//           (state += (1-beta)*e_req on this rank's own chunk), which is the
//           same fp32 operation the reduce kernel would have done in the
//           "exit" fix-up mode.
// The kernel serves the P virtual ranks of one plan (grid y = P*P, rank0 = 0,
// e_req holding every owner chunk: er_chunk_vec = chunk_vec) and one rank of
// a group spread over processes (grid y = P, rank0 = that rank's index, e_req
// holding its own chunk only: er_chunk_vec = 0).  Chunk o's codes and scales
// go to dst.codes[o] / dst.scales[o] (ChunkDst): one local buffer, or, on the
// rank path, rank o's receive buffer on its GPU, so that the quantized chunk
// crosses NVLink as the kernel writes it.
//   VPT   : vectors per thread.  A block covers kThreads*VPT vectors; thread t
//           takes vectors t, t + kThreads, ... so each load instruction of a
//           warp is contiguous, and all of a thread's input and state loads
//           are issued before any arithmetic.  One vector per thread (62
//           registers, 4 blocks per SM) measured faster than two (80
//           registers, 3 blocks) at every size from 1 MiB to 1 GiB per rank:
//           2.4 % per call at 1 GiB, 3-4 % at 4-16 MiB (finer blocks also
//           leave a smaller last wave).
// x is a __grid_constant__ parameter: the block's rank selects its pointer
// straight from the parameter bank.  Indexing a by-value array parameter
// with a run-time index otherwise copies the whole array to every thread's
// local memory first (64 bytes per thread, 2^28 threads per 1 GiB-per-rank
// launch), which measured 7% of the entry's time.
template <bool COMP>
struct EntryShape {
    static constexpr int VPT = COMP ? 1 : 4;
    static constexpr int MIN_BLOCKS = 4;  // resident blocks per SM (register cap)
};

template <bool COMP>
inline unsigned entry_blocks(int64_t v_count) {
    constexpr int64_t per = (int64_t)kThreads * EntryShape<COMP>::VPT;
    return (unsigned)((v_count + per - 1) / per);
}

template <int G, bool COMP, bool DEFER, int BITS>
__global__ void __launch_bounds__(kThreads, EntryShape<COMP>::MIN_BLOCKS)
echo_entry_kernel(const __grid_constant__ InPtrs x, float *__restrict__ m_fast, float *__restrict__ m_slow,
                  const __grid_constant__ ChunkDst dst,
                  const float *__restrict__ e_req, int64_t n_vec, int64_t chunk_vec,
                  Slab sl, int P, Consts k, int rank0, int64_t er_chunk_vec) {
    constexpr int LANES = G / kVec;
    constexpr int VPT = EntryShape<COMP>::VPT;
    const int r = blockIdx.y / P, o = blockIdx.y % P;  // rank (row), owner chunk
    const bool own = (o == r + rank0);                  // this rank owns chunk o
    const int64_t base = (int64_t)blockIdx.x * (kThreads * VPT) + threadIdx.x;
    const float2 z = splat2(k.neg_zero);

    float xt[VPT][8], mf[COMP ? VPT : 1][8], ms[COMP ? VPT : 1][8];
    int64_t j[VPT];
    bool valid[VPT];

    // ---- all loads first
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
        const int64_t l = base + (int64_t)v * kThreads;
        valid[v] = l < sl.v_count;
        j[v] = (int64_t)o * chunk_vec + sl.v_begin + l;   // vector index in rank r
        if (valid[v]) {
            bf16x8_to_f32(x.p[r][j[v]], xt[v]);
            if (COMP) {
                const int64_t e0 = ((int64_t)r * n_vec + j[v]) * kVec;
                ld8(m_fast + e0, mf[v]);
                ld8(m_slow + e0, ms[v]);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) xt[v][i] = 0.0f;
        }
    }

#pragma unroll
    for (int v = 0; v < VPT; ++v) {
        if (COMP && valid[v]) {
            if (DEFER && own) {
                // e_req is loaded here, not with the other operands: only the
                // owner's blocks (1/P of them) read it, and keeping its 8
                // values live across the loads would cost every block registers
                float er[8];
                const int64_t l = base + (int64_t)v * kThreads;
                ld8(e_req + ((int64_t)o * er_chunk_vec + sl.v_begin + l) * kVec, er);
                const float2 obf = splat2(k.one_m_beta_fast), obs = splat2(k.one_m_beta_slow);
#pragma unroll
                for (int i = 0; i < 8; i += 2) {
                    const float2 e2 = make_float2(er[i], er[i + 1]);
                    const float2 f = add2(make_float2(mf[v][i], mf[v][i + 1]), prod2(obf, e2, z));
                    const float2 g = add2(make_float2(ms[v][i], ms[v][i + 1]), prod2(obs, e2, z));
                    mf[v][i] = f.x; mf[v][i + 1] = f.y;
                    ms[v][i] = g.x; ms[v][i + 1] = g.y;
                }
            }
            const float2 a2 = splat2(k.alpha), oma2 = splat2(k.one_m_alpha);
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                const float2 c = add2(prod2(a2, make_float2(mf[v][i], mf[v][i + 1]), z),
                                      prod2(oma2, make_float2(ms[v][i], ms[v][i + 1]), z));
                const float2 s = add2(make_float2(xt[v][i], xt[v][i + 1]), c);
                xt[v][i] = s.x;
                xt[v][i + 1] = s.y;
            }
        }

        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(xt[v][i]));
        a = group_absmax<LANES>(a);        // every lane of the warp takes part
        float kf[8];
        float scale;
        Packed8<BITS> w;
        {
            const GroupScale gs = make_group_scale<BITS>(a);
            scale = gs.scale;
            if (COMP)   // corrected inputs carry full fp32 mantissas: ties are rare
                w = quantize8<BITS>(xt[v], gs, kf, z);
            else        // raw bf16 inputs sit on ties often: the exact quotient
                w = quantize8_q<BITS>(xt[v], gs, kf, z);
        }
        if (!valid[v]) continue;

        const int64_t vc = sl.v_begin + base + (int64_t)v * kThreads;   // vector in chunk o
        store_packed8<BITS>(reinterpret_cast<uint32_t *>(dst.codes[o]), (int64_t)r * n_vec + vc, w);
        if ((threadIdx.x & (LANES - 1)) == 0)
            dst.scales[o][(int64_t)r * (n_vec / LANES) + vc / LANES] = scale;

        if (COMP) {
            const float2 s2 = splat2(scale);
            const float2 bf2 = splat2(k.beta_fast), obf2 = splat2(k.one_m_beta_fast);
            const float2 bs2 = splat2(k.beta_slow), obs2 = splat2(k.one_m_beta_slow);
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                const float2 e = sub2(make_float2(xt[v][i], xt[v][i + 1]),
                                      prod2(make_float2(kf[i], kf[i + 1]), s2, z));
                const float2 f =
                    add2(prod2(bf2, make_float2(mf[v][i], mf[v][i + 1]), z), prod2(obf2, e, z));
                const float2 g =
                    add2(prod2(bs2, make_float2(ms[v][i], ms[v][i + 1]), z), prod2(obs2, e, z));
                mf[v][i] = f.x;
                mf[v][i + 1] = f.y;
                ms[v][i] = g.x;
                ms[v][i + 1] = g.y;
            }
            const int64_t e0 = ((int64_t)r * n_vec + j[v]) * kVec;
            st8(m_fast + e0, mf[v]);
            st8(m_slow + e0, ms[v]);
        }
    }
}

}  // namespace echo
