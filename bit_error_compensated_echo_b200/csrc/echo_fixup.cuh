// echo_fixup.cuh -- the owner fix-up as its own launch, and state reads
// (operation: include/echo.h; conventions: echo_common.cuh)
#pragma once

#include "echo_common.cuh"

namespace echo {

// ------------------------------------------------------------ owner fix-up
//
// The owner fix-up alone, as its own launch (side-stream mode), or, with
// dst != src, a copy of the states that applies a pending fix-up on the way
// (reading the state of a plan in deferred mode).  Grid: x over the vectors
// of the slab, y = owner chunk; only rank == owner adds the fix-up.
__global__ void __launch_bounds__(kThreads)
echo_fixup_kernel(const float *__restrict__ src_fast, const float *__restrict__ src_slow,
                  float *__restrict__ dst_fast, float *__restrict__ dst_slow,
                  const float *__restrict__ e_req, int64_t n_vec, int64_t chunk_vec,
                  Slab sl, int P, int apply, int only_owner, Consts k) {
    const int64_t local = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (local >= sl.v_count) return;
    const int o = blockIdx.y;
    // 32-byte accesses where every buffer allows (offsets are multiples of 32 bytes)
    const bool wide = aligned32(src_fast) && aligned32(src_slow) && aligned32(dst_fast) &&
                      aligned32(dst_slow) && aligned32(e_req);
    for (int r = 0; r < P; ++r) {
        const bool own = (r == o);
        if (only_owner && !own) continue;
        const int64_t j = (int64_t)o * chunk_vec + sl.v_begin + local;
        const int64_t e0 = ((int64_t)r * n_vec + j) * kVec;
        float mf[8], ms[8];
        ld8w(src_fast + e0, mf, wide);
        ld8w(src_slow + e0, ms, wide);
        if (own && apply) {
            float er[8];
            ld8w(e_req + j * kVec, er, wide);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                mf[i] = __fadd_rn(mf[i], __fmul_rn(k.one_m_beta_fast, er[i]));
                ms[i] = __fadd_rn(ms[i], __fmul_rn(k.one_m_beta_slow, er[i]));
            }
        }
        st8w(dst_fast + e0, mf, wide);
        st8w(dst_slow + e0, ms, wide);
    }
}

// ------------------------------------------------------------ e_req fill
//
// Fills n floats with v.  e_req is kept at -0.0f whenever no deferred fix-up
// is pending (plan creation, state reset and restore): the fix-up it then
// applies is m + (1-beta)*(-0) = m + (-0) = m, exactly, for every finite m
// (-0 included), so the deferred-mode entry applies e_req on every call and
// no host-side flag decides which kernel a call (or a captured graph) runs.
__global__ void __launch_bounds__(kThreads)
echo_fill_kernel(float *__restrict__ p, int64_t n, float v) {
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n; i += stride) p[i] = v;
}

}  // namespace echo
