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
//           same fp32 operation the exit kernel would have done.
template <int G, bool COMP, bool DEFER>
__global__ void __launch_bounds__(kThreads, COMP ? 5 : 8)
echo_entry_kernel(InPtrs x, float *__restrict__ m_fast, float *__restrict__ m_slow,
                  uint32_t *__restrict__ codes, float *__restrict__ scales,
                  const float *__restrict__ e_req, int64_t n_vec, int64_t chunk_vec,
                  Slab sl, int P, Consts k) {
    constexpr int LANES = G / kVec;
    const int r = blockIdx.y / P, o = blockIdx.y % P;  // rank, owner chunk
    const int64_t l = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const bool valid = l < sl.v_count;
    const int64_t j = (int64_t)o * chunk_vec + sl.v_begin + l;  // vector in rank r

    float xt[8], mf[8], ms[8];
    if (valid) {
        bf16x8_to_f32(x.p[r][j], xt);
        if (COMP) {
            const int64_t e0 = ((int64_t)r * n_vec + j) * kVec;
            ld8(m_fast + e0, mf);
            ld8(m_slow + e0, ms);
            if (DEFER && o == r) {
                float er[8];
                ld8(e_req + j * kVec, er);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    mf[i] = __fadd_rn(mf[i], __fmul_rn(k.one_m_beta_fast, er[i]));
                    ms[i] = __fadd_rn(ms[i], __fmul_rn(k.one_m_beta_slow, er[i]));
                }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float c = __fadd_rn(__fmul_rn(k.alpha, mf[i]),
                                          __fmul_rn(k.one_m_alpha, ms[i]));
                xt[i] = __fadd_rn(xt[i], c);
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) xt[i] = 0.0f;
    }

    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(xt[i]));
    a = group_absmax<LANES>(a);        // every lane of the warp takes part
    const float scale = group_scale(a);
    float kf[8];
    const uint32_t w = quantize8_div(xt, scale, kf);
    if (!valid) return;

    codes[(int64_t)r * n_vec + j] = w;
    if ((threadIdx.x & (LANES - 1)) == 0)
        scales[(int64_t)r * (n_vec / LANES) + j / LANES] = scale;

    if (COMP) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float e = __fsub_rn(xt[i], __fmul_rn(kf[i], scale));
            mf[i] = __fadd_rn(__fmul_rn(k.beta_fast, mf[i]), __fmul_rn(k.one_m_beta_fast, e));
            ms[i] = __fadd_rn(__fmul_rn(k.beta_slow, ms[i]), __fmul_rn(k.one_m_beta_slow, e));
        }
        const int64_t e0 = ((int64_t)r * n_vec + j) * kVec;
        st8(m_fast + e0, mf);
        st8(m_slow + e0, ms);
    }
}

}  // namespace echo
