// echo_reduce.cuh -- the reduce-scatter half: dequantize, fp32 sum, requantize
// (operation: include/echo.h; conventions: echo_common.cuh)
#pragma once

#include "echo_common.cuh"
#include "echo_stage.cuh"

namespace echo {

// ------------------------------------------------------------ echo_reduce
//
// Reduce-scatter half: for every element, dequantize the P ranks' codes,
// sum them in fp32 in ascending rank order from +0, requantize the sum and
// pack it (the reduced transport).  The dequantized sum y = bf16(k2*scale2)
// is what every rank receives, so on one GPU the kernel also writes it to
// the n_out outputs itself (OUT), with no second pass over the reduced
// codes; without OUT (the rank path) that is the exit kernel's job.
// Compensating, the
// output residual e_req = s - float(y) is either
// written out (for a side-stream or deferred fix-up) or, with fix, folded
// into the owner's states here (state row o, the owner's own chunk).
// Each thread owns 16 consecutive elements (a run): one 8-byte word pair of
// codes per rank (16 bytes at 8 bits), all P loads issued before any
// arithmetic (sum_run), or, for the configuration where that measured
// faster, the block's 256 runs of every rank staged in shared memory by bulk
// copies (stage_sum; STAGE, see ReduceShape).  Its 32 bytes of each output
// and 64 bytes of e_req leave as 32-byte stores where the buffer allows.
// Grid: x over the slab's runs in blocks of 256, y = owner.
constexpr int kRedVec = 16;

// blocks along x for a slab of v_count 8-element vectors
inline unsigned reduce_blocks(int64_t v_count) {
    return (unsigned)((v_count / 2 + kThreads - 1) / kThreads);
}

// The reduce-scatter sum of one 16-element run j (run index within a rank)
// of the P ranks: dequantize each rank's codes and add them in fp32 in
// ascending rank order from +0.  All P code and scale loads are issued
// before any arithmetic.  Lanes with valid == false produce zeros.
template <int G, int P, int BITS>
__device__ __forceinline__ void sum_run(const uint32_t *__restrict__ codes,
                                        const float *__restrict__ scales, int64_t n_vec,
                                        int64_t j, bool valid, float2 z, float s[16]) {
    constexpr int LANES = G / kRedVec;
    constexpr int WORDS = BITS / 2;                 // words holding 16 codes
    const int64_t n_run = n_vec / 2;
    const int64_t n_groups = n_run / LANES;
    uint32_t w[P][WORDS];
    float sc[P];
#pragma unroll
    for (int r = 0; r < P; ++r) {
        const int64_t run = (int64_t)r * n_run + j;
        if (BITS == 4) {
            const uint2 t = valid ? __ldcs(reinterpret_cast<const uint2 *>(codes) + run)
                                  : make_uint2(0u, 0u);
            w[r][0] = t.x;
            w[r][WORDS - 1] = t.y;
        } else {
            const uint4 t = valid ? __ldcs(reinterpret_cast<const uint4 *>(codes) + run)
                                  : make_uint4(0u, 0u, 0u, 0u);
            w[r][0] = t.x;
            w[r][1 % WORDS] = t.y;
            w[r][2 % WORDS] = t.z;
            w[r][WORDS - 1] = t.w;
        }
        sc[r] = valid ? __ldg(scales + (int64_t)r * n_groups + j / LANES) : 0.0f;
    }
    float2 s2[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) s2[i] = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int r = 0; r < P; ++r) {
        const float2 sc2 = splat2(sc[r]);
        float2 k[8];
        decode_pairs<BITS, 8>(w[r], k);
#pragma unroll
        for (int p = 0; p < 8; ++p) s2[p] = add2(s2[p], prod2(k[p], sc2, z));
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        s[2 * i] = s2[i].x;
        s[2 * i + 1] = s2[i].y;
    }
}

// The sums of a block's runs: the P ranks' codes of the
// block's runs [run0, run0 + nrun) (run indices within a rank row) arrive in
// shared memory by one bulk copy per rank, issued by thread 0 and completing
// on one mbarrier, and the block's scales by plain loads of all threads (a
// rank's row of scales need not start on 16 bytes).  Each thread then reads
// its run's P code words and P scales at fixed offsets from one shared
// address -- no per-rank address arithmetic -- dequantizes them and adds
// them in fp32 in ascending rank order from +0.  Threads past the slab
// (threadIdx.x >= nrun: whole groups, since nrun is a multiple of the lanes
// of a group) read run 0's codes; their results are not stored.  Returns
// false in every thread if the copies did not complete within the wait
// limit (the device error word is then set).
//
// Bulk-copy alignment (16 bytes for both addresses and the size): a run is
// 2*BITS bytes of codes; a rank row is N*BITS/8 bytes and N is a multiple
// of P*G >= 32; run0 = owner*C/16 + v_begin/2 + 256*blockIdx.x with C = N/P
// a multiple of G and v_begin a multiple of G/8 >= 4; nrun is even (the
// slab's run count is a multiple of G/16 >= 2); the code buffer itself is
// 16-byte aligned (every caller checks or allocates so).
template <int G, int P, int BITS>
__device__ __forceinline__ bool stage_sum(const uint32_t *__restrict__ codes,
                                          const float *__restrict__ scales, int64_t n_vec,
                                          int64_t run0, int nrun, float2 z, float s[16]) {
    constexpr int LANES = G / kRedVec;
    constexpr int WB = 2 * BITS;                    // code bytes of one run
    constexpr int WORDS = BITS / 2;                 // words holding 16 codes
    constexpr int GPB = kThreads / LANES;           // groups per block
    __shared__ __align__(128) uint8_t s_codes[P][kThreads * WB];
    __shared__ float s_scales[P][GPB];
    __shared__ __align__(8) uint64_t s_bar;
    const int t = threadIdx.x;
    const int64_t n_run = n_vec / 2;
    const int64_t n_groups = n_run / LANES;
    const uint32_t bar = smem_u32(&s_bar);
    if (t == 0) {
        mbar_init(bar, 1);
        mbar_init_fence();
    }
    __syncthreads();
    if (t == 0) {
        const uint32_t bytes = (uint32_t)nrun * WB;
        mbar_arrive_expect_tx(bar, (uint32_t)P * bytes);
#pragma unroll
        for (int r = 0; r < P; ++r)
            bulk_copy_g2s(smem_u32(s_codes[r]),
                          reinterpret_cast<const uint8_t *>(codes) + (r * n_run + run0) * WB,
                          bytes, bar);
    }
    const int ngrp = nrun / LANES;
    const int64_t g0 = run0 / LANES;
    for (int i = t; i < P * GPB; i += kThreads) {
        const int r = i / GPB, g = i - r * GPB;
        if (g < ngrp) s_scales[r][g] = __ldg(scales + r * n_groups + g0 + g);
    }
    const bool arrived = mbar_wait_bounded(bar, 0);
    if (!__syncthreads_and(arrived)) {
        // the copies may still be writing this block's shared memory: wait
        // for them once more (bounded) before the block ends
        if (t == 0) mbar_wait_bounded(bar, 0);
        return false;
    }
    const int tt = t < nrun ? t : 0;
    float2 s2[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) s2[i] = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int r = 0; r < P; ++r) {
        uint32_t w[WORDS];
        if (BITS == 4) {
            const uint2 v = reinterpret_cast<const uint2 *>(s_codes[r])[tt];
            w[0] = v.x;
            w[WORDS - 1] = v.y;
        } else {
            const uint4 v = reinterpret_cast<const uint4 *>(s_codes[r])[tt];
            w[0] = v.x;
            w[1 % WORDS] = v.y;
            w[2 % WORDS] = v.z;
            w[WORDS - 1] = v.w;
        }
        const float2 sc2 = splat2(s_scales[r][tt / LANES]);
        float2 k[8];
        decode_pairs<BITS, 8>(w, k);
#pragma unroll
        for (int p = 0; p < 8; ++p) s2[p] = add2(s2[p], prod2(k[p], sc2, z));
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        s[2 * i] = s2[i].x;
        s[2 * i + 1] = s2[i].y;
    }
    return true;
}

// Which way the reduce reads the transport.  Staging the block's tiles in
// shared memory (stage_sum) measured faster only for the uncompensated
// reduce that also writes the P outputs, at P = 8, G = 128 and owner
// chunks of at least 2^20 elements (16 MiB of bf16 per rank; 1 GiB per
// rank, 4-bit codes: 1.87 -> 1.76 ms, call 0.89 -> 0.93 of its roofline in
// the sweep; 8-bit codes: 2.29 -> 2.10 ms; its loads then leave the
// load/store queues to the stores).
// Elsewhere the direct loads of sum_run are faster: compensated (1 GiB per
// rank: 1.00 ms direct, 1.07 ms staged; 8-bit 1.21 against 1.24 ms),
// uncompensated at G = 32 or 64 (1.9
// against 2.3 ms), at P = 2 and 4 (the call 1-3 points of its roofline
// lower), and below 16 MiB per rank (4 MiB, P = 8: 29.7 against 31.7 us).
// The block-wide wait for the tiles exposes latency that the direct form
// hides warp by warp, and the address arithmetic that staging removes
// reappears as uniform instructions.  STAGE_OK says which instances may
// stage; the launcher picks the staged one only at or above kStageMinRuns
// runs per owner chunk in the slab.
template <int G, int P, bool COMP, bool OUT, int BITS>
struct ReduceShape {
    static constexpr bool STAGE_OK = !COMP && OUT && G == 128 && P == 8;
};
constexpr int64_t kStageMinRuns = int64_t(1) << 16;   // 2^20 elements

// The reduce-scatter's kernel (echo_rs) is bound by the wait for its loads
// (ncu: long scoreboard the top stall, issue 37% busy), and staging its
// tiles measured faster at P = 8, G = 128 (1 GiB per rank, compensated,
// 4-bit codes: 1.23 -> 0.98 ms, the call 13.02 -> 12.82 ms; 8-bit codes:
// 1.38 -> 1.10 ms; uncompensated 0.77 -> 0.70 and 0.82 -> 0.78 ms; 16 MiB
// per rank: 29 -> 24 us) and at P = 8, G = 64 (1.18 -> 1.07 ms); slower at
// G = 32 (1.25 -> 1.39 ms), at P = 2 (0.82 -> 0.85 ms) and at P = 4 (even at
// G = 128, worse at G = 64: 0.88 -> 0.90 ms).  The same size threshold
// applies.
template <int G, int P, int BITS>
struct RsShape {
    static constexpr bool STAGE_OK = P == 8 && G >= 64;
};

template <int G, int P, bool COMP, bool OUT, int BITS, bool STAGE>
__global__ void __launch_bounds__(kThreads)
echo_reduce_kernel(const uint32_t *__restrict__ codes, const float *__restrict__ scales,
                   uint32_t *__restrict__ rcodes, float *__restrict__ rscales,
                   float *__restrict__ e_req, int64_t n_vec, int64_t chunk_vec, Slab sl,
                   Consts k, const __grid_constant__ OutPtrs out, int n_out,
                   float *__restrict__ m_fast, float *__restrict__ m_slow, int fix) {
    constexpr int LANES = G / kRedVec;              // lanes per group
    const int o = blockIdx.y;
    const int64_t chunk_run = chunk_vec / 2;        // runs per owner chunk
    const int64_t local = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const bool valid = local < sl.v_count / 2;
    const int64_t j = (int64_t)o * chunk_run + sl.v_begin / 2 + local;  // run index in a rank
    const float2 z = splat2(k.neg_zero);
    float s[16];
    if (STAGE) {
        const int64_t left = sl.v_count / 2 - (local - threadIdx.x);   // runs from the block's first
        const int nrun = (int)(left < kThreads ? left : kThreads);
        if (!stage_sum<G, P, BITS>(codes, scales, n_vec, j - threadIdx.x, nrun, z, s)) return;
    } else {
        sum_run<G, P, BITS>(codes, scales, n_vec, j, valid, z, s);
    }

    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(s[i]));
    a = group_absmax<LANES>(a);
    const GroupScale gs = make_group_scale<BITS>(a);
    const float scale2 = gs.scale;
    float k2[16];
    const Packed8<BITS> w0 = quantize8_q<BITS>(s, gs, k2, z);
    const Packed8<BITS> w1 = quantize8_q<BITS>(s + 8, gs, k2 + 8, z);
    if (!valid) return;

    if (BITS == 4)
        reinterpret_cast<uint2 *>(rcodes)[j] = make_uint2(w0.w[0], w1.w[0]);
    else
        reinterpret_cast<uint4 *>(rcodes)[j] =
            make_uint4(w0.w[0], w0.w[BITS / 4 - 1], w1.w[0], w1.w[BITS / 4 - 1]);
    if ((threadIdx.x & (LANES - 1)) == 0) rscales[j / LANES] = scale2;
    uint32_t yw[8];                                 // y = bf16(k2*scale2), pairs
    const float2 sc2 = splat2(scale2);
#pragma unroll
    for (int i = 0; i < 8; ++i)
        yw[i] = bf16x2_bits_rn(mul2(make_float2(k2[2 * i], k2[2 * i + 1]), sc2));
    if (OUT) store_run_outputs(out, n_out, j, yw);
    if (COMP) {
        float e[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float2 d = sub2(make_float2(s[2 * i], s[2 * i + 1]), bf16x2_to_f32(yw[i]));
            e[2 * i] = d.x;
            e[2 * i + 1] = d.y;
        }
        if (fix) {   // the owner's own states, this run's 16 elements
            const int64_t e0 = ((int64_t)o * n_vec + j * 2) * kVec;
            const float2 obf = splat2(k.one_m_beta_fast), obs = splat2(k.one_m_beta_slow);
            const bool wide = aligned32(m_fast) && aligned32(m_slow);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float mf[8], ms[8];
                ld8w(m_fast + e0 + 8 * h, mf, wide);
                ld8w(m_slow + e0 + 8 * h, ms, wide);
#pragma unroll
                for (int i = 0; i < 8; i += 2) {
                    const float2 e2 = make_float2(e[8 * h + i], e[8 * h + i + 1]);
                    const float2 f = add2(make_float2(mf[i], mf[i + 1]), prod2(obf, e2, z));
                    const float2 g = add2(make_float2(ms[i], ms[i + 1]), prod2(obs, e2, z));
                    mf[i] = f.x; mf[i + 1] = f.y;
                    ms[i] = g.x; ms[i + 1] = g.y;
                }
                st8w(m_fast + e0 + 8 * h, mf, wide);
                st8w(m_slow + e0 + 8 * h, ms, wide);
            }
        } else {
            store_run16(e_req, j, e);
        }
    }
}

// ------------------------------------------------------------ echo_reduce_scatter
//
// The reduce-scatter call's second kernel: the same sum, delivered to the
// owner as bf16 without a second quantization: out[o] (N/P elements) gets
// bf16(s) of chunk o.  The owner's output residual e = s - float(bf16(s))
// is folded into its own EMAs here (FIX) or written to e_req for a
// side-stream or deferred fix-up (COMP && !FIX).
// Grid: x over the 16-element runs of the slab, y = owner (out is a
// __grid_constant__ parameter, indexed by the owner without a local copy).
// STAGE: the P code tiles staged in shared memory (stage_sum, see RsShape).
template <int G, int P, bool COMP, bool FIX, int BITS, bool STAGE>
__global__ void __launch_bounds__(kThreads)
echo_rs_kernel(const uint32_t *__restrict__ codes, const float *__restrict__ scales,
               const __grid_constant__ OutPtrs out,
               float *__restrict__ m_fast, float *__restrict__ m_slow, float *__restrict__ e_req,
               int64_t n_vec, int64_t chunk_vec, Slab sl, Consts k) {
    const int o = blockIdx.y;
    const int64_t chunk_run = chunk_vec / 2;
    const int64_t local = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const int64_t lr = sl.v_begin / 2 + local;          // run index within chunk o
    const int64_t j = (int64_t)o * chunk_run + lr;       // run index within a rank
    const float2 z = splat2(k.neg_zero);
    float s[16];
    if (STAGE) {   // every thread takes part in the staging's barriers
        const int64_t left = sl.v_count / 2 - (local - threadIdx.x);   // runs from the block's first
        const int nrun = (int)(left < kThreads ? left : kThreads);
        if (!stage_sum<G, P, BITS>(codes, scales, n_vec, j - threadIdx.x, nrun, z, s)) return;
        if ((int)threadIdx.x >= nrun) return;   // no shuffles below: lanes may leave
    } else {
        if (local >= sl.v_count / 2) return;    // no shuffles below: lanes may leave
        sum_run<G, P, BITS>(codes, scales, n_vec, j, true, z, s);
    }

    uint32_t yw[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) yw[i] = bf16x2_bits_rn(make_float2(s[2 * i], s[2 * i + 1]));
    uint4 *dst = out.p[o] + lr * 2;
    if (aligned32(out.p[o])) {
        st32_words(dst, yw);
    } else {
        dst[0] = make_uint4(yw[0], yw[1], yw[2], yw[3]);
        dst[1] = make_uint4(yw[4], yw[5], yw[6], yw[7]);
    }
    if (COMP) {
        float e[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float2 d = sub2(make_float2(s[2 * i], s[2 * i + 1]), bf16x2_to_f32(yw[i]));
            e[2 * i] = d.x;
            e[2 * i + 1] = d.y;
        }
        if (FIX) {
            const int64_t e0 = ((int64_t)o * n_vec + j * 2) * kVec;   // rank o's own state
            const float2 obf = splat2(k.one_m_beta_fast), obs = splat2(k.one_m_beta_slow);
            const bool wide = aligned32(m_fast) && aligned32(m_slow);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float mf[8], ms[8];
                ld8w(m_fast + e0 + 8 * h, mf, wide);
                ld8w(m_slow + e0 + 8 * h, ms, wide);
#pragma unroll
                for (int i = 0; i < 8; i += 2) {
                    const float2 e2 = make_float2(e[8 * h + i], e[8 * h + i + 1]);
                    const float2 f = add2(make_float2(mf[i], mf[i + 1]), prod2(obf, e2, z));
                    const float2 g = add2(make_float2(ms[i], ms[i + 1]), prod2(obs, e2, z));
                    mf[i] = f.x; mf[i + 1] = f.y;
                    ms[i] = g.x; ms[i + 1] = g.y;
                }
                st8w(m_fast + e0 + 8 * h, mf, wide);
                st8w(m_slow + e0 + 8 * h, ms, wide);
            }
        } else {
            store_run16(e_req, j, e);
        }
    }
}

}  // namespace echo
