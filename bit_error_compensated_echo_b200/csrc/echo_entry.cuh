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

    const float2 z = splat2(k.neg_zero);
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
                const float2 obf = splat2(k.one_m_beta_fast), obs = splat2(k.one_m_beta_slow);
#pragma unroll
                for (int i = 0; i < 8; i += 2) {
                    const float2 e2 = make_float2(er[i], er[i + 1]);
                    const float2 f = add2(make_float2(mf[i], mf[i + 1]), prod2(obf, e2, z));
                    const float2 g = add2(make_float2(ms[i], ms[i + 1]), prod2(obs, e2, z));
                    mf[i] = f.x; mf[i + 1] = f.y;
                    ms[i] = g.x; ms[i + 1] = g.y;
                }
            }
            const float2 a2 = splat2(k.alpha), oma2 = splat2(k.one_m_alpha);
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                const float2 c = add2(prod2(a2, make_float2(mf[i], mf[i + 1]), z),
                                      prod2(oma2, make_float2(ms[i], ms[i + 1]), z));
                const float2 v = add2(make_float2(xt[i], xt[i + 1]), c);
                xt[i] = v.x;
                xt[i + 1] = v.y;
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
    float kf[8];
    float scale;
    uint32_t w;
    if (COMP) {   // corrected inputs carry full fp32 mantissas: ties are rare
        const GroupScale gs = make_group_scale(a);
        scale = gs.scale;
        w = quantize8(xt, gs, kf, z);
    } else {      // raw bf16 inputs often divide to exact half-integers
        scale = group_scale(a);
        w = quantize8_div(xt, scale, kf);
    }
    if (!valid) return;

    codes[(int64_t)r * n_vec + j] = w;
    if ((threadIdx.x & (LANES - 1)) == 0)
        scales[(int64_t)r * (n_vec / LANES) + j / LANES] = scale;

    if (COMP) {
        const float2 s2 = splat2(scale);
        const float2 bf2 = splat2(k.beta_fast), obf2 = splat2(k.one_m_beta_fast);
        const float2 bs2 = splat2(k.beta_slow), obs2 = splat2(k.one_m_beta_slow);
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            const float2 e = sub2(make_float2(xt[i], xt[i + 1]),
                                  prod2(make_float2(kf[i], kf[i + 1]), s2, z));
            const float2 f = add2(prod2(bf2, make_float2(mf[i], mf[i + 1]), z), prod2(obf2, e, z));
            const float2 g = add2(prod2(bs2, make_float2(ms[i], ms[i + 1]), z), prod2(obs2, e, z));
            mf[i] = f.x;
            mf[i + 1] = f.y;
            ms[i] = g.x;
            ms[i + 1] = g.y;
        }
        const int64_t e0 = ((int64_t)r * n_vec + j) * kVec;
        st8(m_fast + e0, mf);
        st8(m_slow + e0, ms);
    }
}

}  // namespace echo
