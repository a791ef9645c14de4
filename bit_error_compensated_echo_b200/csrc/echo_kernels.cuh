// echo_kernels.cuh -- sm_100a kernels of Echo's error-compensated 4-bit
// all-reduce ("Echo: Error-Compensated 4-Bit Tensor-Parallel Communication",
// ai4snews news summary "Interpretation" and the arXiv abstract on the
// fugumt mirror).  The operation each kernel computes is written out in
// include/echo.h; here is how it maps onto the B200.
//
// The path is elementwise codec work bound by HBM bandwidth, not a
// contraction, so there are no tensor cores.  Every thread owns 8
// consecutive elements of one rank (one 16-byte bf16 vector, two float4 of
// each EMA state, one 32-bit word of packed codes).  A group of G elements
// is G/8 adjacent lanes of one warp; its absmax is a butterfly of
// __shfl_xor_sync (max is order-free, so it is exact).  All fp32 arithmetic
// uses the explicitly rounded intrinsics (__fadd_rn, __fmul_rn, __fdiv_rn),
// which the compiler never contracts into FMA, so every value is the same
// IEEE-754 single-precision result as a plain scalar evaluation of the
// definition.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace echo {

constexpr int kVec = 8;          // elements per thread
constexpr int kThreads = 256;    // threads per block of every kernel
constexpr int kMaxRanks = 8;

struct InPtrs {
    const uint4 *p[kMaxRanks];   // rank r's bf16 input, 8 elements per uint4
};
struct OutPtrs {
    uint4 *p[kMaxRanks];
};

struct Consts {
    float alpha, one_m_alpha;
    float beta_fast, one_m_beta_fast;
    float beta_slow, one_m_beta_slow;
};

// ------------------------------------------------------------ helpers

__device__ __forceinline__ void bf16x8_to_f32(const uint4 v, float f[8]) {
    f[0] = __uint_as_float(v.x << 16);
    f[1] = __uint_as_float(v.x & 0xffff0000u);
    f[2] = __uint_as_float(v.y << 16);
    f[3] = __uint_as_float(v.y & 0xffff0000u);
    f[4] = __uint_as_float(v.z << 16);
    f[5] = __uint_as_float(v.z & 0xffff0000u);
    f[6] = __uint_as_float(v.w << 16);
    f[7] = __uint_as_float(v.w & 0xffff0000u);
}

__device__ __forceinline__ uint32_t bf16_bits_rn(float f) {
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// max over the LANES adjacent lanes that hold one group
template <int LANES>
__device__ __forceinline__ float group_absmax(float a) {
#pragma unroll
    for (int off = 1; off < LANES; off <<= 1)
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
    return a;
}

// scale = a / 7, or 0 for an all-zero group
__device__ __forceinline__ float group_scale(float a) {
    return a != 0.0f ? __fdiv_rn(a, 7.0f) : 0.0f;
}

// k = clamp(rint(v / scale), -7, 7) with ties to even; 0 when scale == 0.
// Codes are packed into one word: element i in bits 4i..4i+3, so byte j
// holds element 2j in its low nibble and 2j+1 in its high nibble.
__device__ __forceinline__ uint32_t quantize8(const float v[8], float scale, int k[8]) {
    uint32_t w = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        int c = 0;
        if (scale != 0.0f) {
            c = __float2int_rn(__fdiv_rn(v[i], scale));
            c = min(max(c, -7), 7);
        }
        k[i] = c;
        w |= ((uint32_t)c & 0xfu) << (4 * i);
    }
    return w;
}

// signed nibble i of a packed word
__device__ __forceinline__ int code_at(uint32_t w, int i) {
    return ((int)(w << (28 - 4 * i))) >> 28;
}

__device__ __forceinline__ void ld8(const float *p, float v[8]) {
    const float4 a = __ldcs(reinterpret_cast<const float4 *>(p));
    const float4 b = __ldcs(reinterpret_cast<const float4 *>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void st8(float *p, const float v[8]) {
    __stcs(reinterpret_cast<float4 *>(p), make_float4(v[0], v[1], v[2], v[3]));
    __stcs(reinterpret_cast<float4 *>(p) + 1, make_float4(v[4], v[5], v[6], v[7]));
}

// ------------------------------------------------------------ echo_entry
//
// Correction add + group quantize + pack + partial EMA update, for every
// rank.  Grid: x over the N/8 vectors of a rank, y = rank.
//   COMP  : compensator on (read/write the states)
//   DEFER : apply the previous call's pending owner fix-up first
//           (state += (1-beta)*e_req on this rank's own chunk), which is the
//           same fp32 operation the exit kernel would have done.
template <int G, bool COMP, bool DEFER>
__global__ void __launch_bounds__(kThreads)
echo_entry_kernel(InPtrs x, float *__restrict__ m_fast, float *__restrict__ m_slow,
                  uint32_t *__restrict__ codes, float *__restrict__ scales,
                  const float *__restrict__ e_req, int64_t n_vec, int64_t chunk_vec,
                  Consts k) {
    constexpr int LANES = G / kVec;
    const int r = blockIdx.y;
    const int64_t j = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const bool valid = j < n_vec;

    float xt[8], mf[8], ms[8];
    if (valid) {
        bf16x8_to_f32(__ldcs(x.p[r] + j), xt);
        if (COMP) {
            const int64_t e0 = ((int64_t)r * n_vec + j) * kVec;
            ld8(m_fast + e0, mf);
            ld8(m_slow + e0, ms);
            if (DEFER && j >= r * chunk_vec && j < (r + 1) * chunk_vec) {
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
    int kc[8];
    const uint32_t w = quantize8(xt, scale, kc);
    if (!valid) return;

    codes[(int64_t)r * n_vec + j] = w;
    if ((threadIdx.x & (LANES - 1)) == 0)
        scales[(int64_t)r * (n_vec / LANES) + j / LANES] = scale;

    if (COMP) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float e = __fsub_rn(xt[i], __fmul_rn((float)kc[i], scale));
            mf[i] = __fadd_rn(__fmul_rn(k.beta_fast, mf[i]), __fmul_rn(k.one_m_beta_fast, e));
            ms[i] = __fadd_rn(__fmul_rn(k.beta_slow, ms[i]), __fmul_rn(k.one_m_beta_slow, e));
        }
        const int64_t e0 = ((int64_t)r * n_vec + j) * kVec;
        st8(m_fast + e0, mf);
        st8(m_slow + e0, ms);
    }
}

// ------------------------------------------------------------ echo_reduce
//
// Reduce-scatter half: for every element, dequantize the P ranks' codes,
// sum them in fp32 in ascending rank order from +0, requantize the sum,
// pack it, and (compensating) write e_req = s - float(bf16(k2*scale2)).
// Grid: x over the N/(8P) vectors of one owner chunk, y = owner.
template <int G, int P, bool COMP>
__global__ void __launch_bounds__(kThreads)
echo_reduce_kernel(const uint32_t *__restrict__ codes, const float *__restrict__ scales,
                   uint32_t *__restrict__ rcodes, float *__restrict__ rscales,
                   float *__restrict__ e_req, int64_t n_vec, int64_t chunk_vec) {
    constexpr int LANES = G / kVec;
    const int o = blockIdx.y;
    const int64_t local = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const bool valid = local < chunk_vec;
    const int64_t j = (int64_t)o * chunk_vec + local;
    const int64_t n_groups = n_vec / LANES;

    uint32_t w[P];
    float sc[P];
#pragma unroll
    for (int r = 0; r < P; ++r) {
        w[r] = valid ? __ldcs(codes + (int64_t)r * n_vec + j) : 0u;
        sc[r] = valid ? __ldg(scales + (int64_t)r * n_groups + j / LANES) : 0.0f;
    }
    float s[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i] = 0.0f;
#pragma unroll
    for (int r = 0; r < P; ++r) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            s[i] = __fadd_rn(s[i], __fmul_rn((float)code_at(w[r], i), sc[r]));
    }

    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(s[i]));
    a = group_absmax<LANES>(a);
    const float scale2 = group_scale(a);
    int k2[8];
    const uint32_t w2 = quantize8(s, scale2, k2);
    if (!valid) return;

    rcodes[j] = w2;
    if ((threadIdx.x & (LANES - 1)) == 0) rscales[j / LANES] = scale2;
    if (COMP) {
        float e[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t yb = bf16_bits_rn(__fmul_rn((float)k2[i], scale2));
            e[i] = __fsub_rn(s[i], __uint_as_float(yb << 16));
        }
        st8(e_req + j * kVec, e);
    }
}

// ------------------------------------------------------------ echo_exit
//
// All-gather half: dequantize the reduced codes once to bf16 and write them
// to all P outputs.  FIX: also apply the owner's fix-up of both EMAs
// (state += (1-beta)*e_req) for the owner's chunk.
// Grid: x over the vectors of one owner chunk, y = owner.
template <int G, bool FIX>
__global__ void __launch_bounds__(kThreads)
echo_exit_kernel(const uint32_t *__restrict__ rcodes, const float *__restrict__ rscales,
                 OutPtrs out, int P, float *__restrict__ m_fast, float *__restrict__ m_slow,
                 const float *__restrict__ e_req, int64_t n_vec, int64_t chunk_vec, Consts k) {
    constexpr int LANES = G / kVec;
    const int o = blockIdx.y;
    const int64_t local = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (local >= chunk_vec) return;
    const int64_t j = (int64_t)o * chunk_vec + local;

    const uint32_t w = __ldg(rcodes + j);
    const float sc = __ldg(rscales + j / LANES);
    uint32_t yb[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) yb[i] = bf16_bits_rn(__fmul_rn((float)code_at(w, i), sc));
    const uint4 y = make_uint4(yb[0] | (yb[1] << 16), yb[2] | (yb[3] << 16),
                               yb[4] | (yb[5] << 16), yb[6] | (yb[7] << 16));
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

// ------------------------------------------------------------ owner fix-up
//
// The owner fix-up alone, as its own launch (side-stream mode), or, with
// dst != src, a copy of the states that applies a pending fix-up on the way
// (reading the state of a plan in deferred mode).  Grid: x over the vectors
// of one owner chunk, y = rank; only rank == owner adds the fix-up.
__global__ void __launch_bounds__(kThreads)
echo_fixup_kernel(const float *__restrict__ src_fast, const float *__restrict__ src_slow,
                  float *__restrict__ dst_fast, float *__restrict__ dst_slow,
                  const float *__restrict__ e_req, int64_t n_vec, int64_t chunk_vec,
                  int P, int apply, int only_owner, Consts k) {
    const int64_t local = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (local >= chunk_vec) return;
    const int o = blockIdx.y;
    for (int r = 0; r < P; ++r) {
        const bool own = (r == o);
        if (only_owner && !own) continue;
        const int64_t j = (int64_t)o * chunk_vec + local;
        const int64_t e0 = ((int64_t)r * n_vec + j) * kVec;
        float mf[8], ms[8];
        ld8(src_fast + e0, mf);
        ld8(src_slow + e0, ms);
        if (own && apply) {
            float er[8];
            ld8(e_req + j * kVec, er);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                mf[i] = __fadd_rn(mf[i], __fmul_rn(k.one_m_beta_fast, er[i]));
                ms[i] = __fadd_rn(ms[i], __fmul_rn(k.one_m_beta_slow, er[i]));
            }
        }
        st8(dst_fast + e0, mf);
        st8(dst_slow + e0, ms);
    }
}

}  // namespace echo
