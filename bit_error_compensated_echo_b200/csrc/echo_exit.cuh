// echo_exit.cuh -- the all-gather half: dequantize to bf16, owner fix-up
// (operation: include/echo.h; conventions: echo_common.cuh)
#pragma once

#include "echo_common.cuh"

namespace echo {

// ------------------------------------------------------------ echo_exit
//
// All-gather half: dequantize the reduced codes once to bf16 and write them
// to all P outputs.  FIX: also apply the owner's fix-up of both EMAs
// (state += (1-beta)*e_req) for the owner's chunk.
// Grid: x over the vectors of the slab, y = owner.
template <int G, bool FIX, int BITS>
__global__ void __launch_bounds__(kThreads)
echo_exit_kernel(const uint32_t *__restrict__ rcodes, const float *__restrict__ rscales,
                 OutPtrs out, int P, float *__restrict__ m_fast, float *__restrict__ m_slow,
                 const float *__restrict__ e_req, int64_t n_vec, int64_t chunk_vec, Slab sl,
                 Consts k) {
    constexpr int LANES = G / kVec;
    const int o = blockIdx.y;
    const int64_t local = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (local >= sl.v_count) return;
    const int64_t j = (int64_t)o * chunk_vec + sl.v_begin + local;

    uint32_t w[BITS / 4];
    load_packed8<BITS>(rcodes, j, w);
    const float2 sc2 = splat2(__ldg(rscales + j / LANES));
    float2 kp[4];
    decode_pairs<BITS, 4>(w, kp);
    uint32_t yw[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) yw[p] = bf16x2_bits_rn(mul2(kp[p], sc2));
    const uint4 y = make_uint4(yw[0], yw[1], yw[2], yw[3]);
#pragma unroll
    for (int r = 0; r < kMaxRanks; ++r)
        if (r < P) __stcs(out.p[r] + j, y);

    if (FIX) {
        const int64_t e0 = ((int64_t)o * n_vec + j) * kVec;
        float er[8], mf[8], ms[8];
        ld8(e_req + j * kVec, er);
        ld8(m_fast + e0, mf);
        ld8(m_slow + e0, ms);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            mf[i] = __fadd_rn(mf[i], __fmul_rn(k.one_m_beta_fast, er[i]));
            ms[i] = __fadd_rn(ms[i], __fmul_rn(k.one_m_beta_slow, er[i]));
        }
        st8(m_fast + e0, mf);
        st8(m_slow + e0, ms);
    }
}

}  // namespace echo
