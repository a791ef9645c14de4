// echo_common.cuh -- shared definitions of the sm_100a kernels of Echo's error-compensated
// 4-bit all-reduce ("Echo: Error-Compensated 4-Bit Tensor-Parallel Communication",
// ai4snews news summary "Interpretation" and the arXiv abstract on the
// fugumt mirror).  The operation each kernel computes is written out in
// include/echo.h; here is how it maps onto the B200.
//
// The path is elementwise codec work bound by HBM bandwidth, not a
// contraction, so there are no tensor cores.  A thread owns runs of
// consecutive elements of one rank: vectors of 8 in the entry and exit
// passes (one 16-byte bf16 vector, two float4 of each EMA state, one word of
// 4-bit or two words of 8-bit codes), runs of 16 in the reduce pass.  A
// group of G elements is G/8 (or G/16) adjacent lanes of one warp; its
// absmax is a butterfly of __shfl_xor_sync (max is order-free, so it is
// exact).  Every fp32 operation rounds once, to nearest even, exactly as a
// plain scalar evaluation of the definition: scalar work uses the explicitly
// rounded intrinsics (__fadd_rn, __fmul_rn, __fdiv_rn, never contracted),
// paired work the sm_100 f32x2 instructions below.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace echo {

constexpr int kVec = 8;          // elements per thread (entry, exit)
constexpr int kThreads = 256;    // threads per block of every kernel
constexpr int kMaxRanks = 8;

struct InPtrs {
    const uint4 *p[kMaxRanks];   // rank r's bf16 input, 8 elements per uint4
};
struct OutPtrs {
    uint4 *p[kMaxRanks];
};

// Where the entry puts owner chunk o's packed codes and scales: codes[o]
// and scales[o] hold the chunk's first vector and first group of row 0
// (row r follows at r rows of n_vec vectors).  One buffer of every chunk
// back to back is the case codes[o] = base + o chunk sizes; the rank path
// may instead point codes[o] into rank o's receive buffer, in another
// GPU's memory.
struct ChunkDst {
    uint8_t *codes[kMaxRanks];
    float *scales[kMaxRanks];
};

// Where the exit reads owner o's reduced chunk (codes[o], scales[o]: its
// first vector and group), in this GPU's memory or in owner o's.
struct ChunkSrc {
    const uint8_t *codes[kMaxRanks];
    const float *scales[kMaxRanks];
};

// A slab: the vectors [v_begin, v_begin + v_count) of every owner chunk
// (a vector is 8 elements; owner chunk o is vectors [o*chunk_vec,
// (o+1)*chunk_vec) of every rank).  A whole call is the slab (0, chunk_vec);
// the host-buffer call pipelines copies and kernels slab by slab.  Both
// bounds are multiples of G/8 and even, so groups and 16-element runs never
// straddle a slab edge.
struct Slab {
    int64_t v_begin, v_count;
};

struct Consts {
    float alpha, one_m_alpha;
    float beta_fast, one_m_beta_fast;
    float beta_slow, one_m_beta_slow;
    float neg_zero;   // -0.0f, passed at run time (see prod2)
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

// max over the LANES adjacent lanes that hold one group
template <int LANES>
__device__ __forceinline__ float group_absmax(float a) {
#pragma unroll
    for (int off = 1; off < LANES; off <<= 1)
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
    return a;
}

// ---- packed fp32 pairs (sm_100 add/sub/mul .rn.f32x2)
//
// Each lane of a pair is an ordinary IEEE-754 fp32 operation rounded to
// nearest even (subnormals kept), so a pair op gives exactly the two scalar
// results; it issues once for both.  ptxas contracts a packed multiply whose
// result feeds a packed add or subtract into one fused multiply-add (single
// rounding) even with explicit .rn, so a product that feeds an add is
// written as prod2: a packed fma whose addend is -0 held in a register that
// is only known at run time.  a*b + (-0) rounds exactly like a*b (also for
// signed zeros), and ptxas cannot fold an addend it does not know, so the
// product stays separately rounded.
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 splat2(float v) { return make_float2(v, v); }

__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c);

// the separately rounded products a.x*b.x, a.y*b.y; z must hold the run-time
// value (-0.0f, -0.0f)
__device__ __forceinline__ float2 prod2(float2 a, float2 b, float2 z) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rz, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rz, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rz;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(z.x), "f"(z.y));
    return d;
}

// a*b + c rounded once, for a pair
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return prod2(a, b, c); }

// ---- exact integer <-> float steps without conversion instructions
//
// In [2^23, 2^24) consecutive floats are consecutive integers, so adding
// 1.5*2^23 to a float q with |q| <= 127 rounds q to an integer under the
// current rounding (nearest, ties to even -- the same result as rint(q)),
// and the low 4 (or 8) bits of the sum's bit pattern are that integer in
// two's complement (the bits of 1.5*2^23 end in 0x00).  Going back, 2^23 + u
// with u = k + 8 (k + 128 for 8-bit codes) has bit pattern 0x4B000000 | u,
// and subtracting 2^23 + 8 (2^23 + 128) gives k exactly.  Both replace the
// int<->float conversion instructions, which issue at a fraction of the
// fp32 add rate.
constexpr float kRoundMagic = 12582912.0f;   // 1.5 * 2^23

// ---- code widths
//
// BITS = 4: levels -7..7, two codes per byte (element 2j in the low nibble
// of byte j), 8 codes per 32-bit word.  BITS = 8: levels -127..127, one code
// per byte, 4 per word.  A thread's 8 (16) codes are BITS/4 (BITS/2) words.
template <int BITS>
struct CodeWidth;
template <>
struct CodeWidth<4> {
    static constexpr float levels = 7.0f;
    static constexpr float offset = 8388616.0f;     // 2^23 + 8
    static constexpr uint32_t bias = 0x88888888u;   // two's complement -> k + 8
    static constexpr float tie_window = 0x1p-18f;   // see quantize8
};
template <>
struct CodeWidth<8> {
    static constexpr float levels = 127.0f;
    static constexpr float offset = 8388736.0f;     // 2^23 + 128
    static constexpr uint32_t bias = 0x80808080u;
    static constexpr float tie_window = 0x1p-13f;
};

// The codes of 8 elements, packed (BITS/4 words).
template <int BITS>
struct Packed8 {
    uint32_t w[BITS / 4];
};

// Pack the codes of 8 elements from their magic sums t (the low bits of each
// sum's bit pattern are its code): byte permutes gather the low bytes, four
// to a word; for 4-bit codes one bitwise select then merges the odd
// elements' nibbles (shifted up by 4) into the even elements' bytes.
template <int BITS>
__device__ __forceinline__ Packed8<BITS> pack_codes(const float t[8]) {
    Packed8<BITS> p;
    uint32_t u[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) u[i] = __float_as_uint(t[i]);
    if (BITS == 4) {
        // even elements: {u0, u2, u4, u6}.b0; odd elements: {u1, u3, u5, u7}.b0
        const uint32_t e = __byte_perm(__byte_perm(u[0], u[2], 0x0040),
                                       __byte_perm(u[4], u[6], 0x0040), 0x5410);
        const uint32_t o = __byte_perm(__byte_perm(u[1], u[3], 0x0040),
                                       __byte_perm(u[5], u[7], 0x0040), 0x5410);
        p.w[0] = (e & 0x0F0F0F0Fu) | ((o << 4) & 0xF0F0F0F0u);
    } else {
        p.w[0] = __byte_perm(__byte_perm(u[0], u[1], 0x0040),
                             __byte_perm(u[2], u[3], 0x0040), 0x5410);
        p.w[BITS / 4 - 1] = __byte_perm(__byte_perm(u[4], u[5], 0x0040),
                                        __byte_perm(u[6], u[7], 0x0040), 0x5410);
    }
    return p;
}

// 2^23 + (byte b of word u), as a float
__device__ __forceinline__ float byte_as_magic(uint32_t u, int b) {
    return __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540 + b));
}

// Decode 2n codes from n*BITS/16 words (n = 4: 8 codes, n = 8: 16 codes)
// into n float pairs: pair p holds elements 2p and 2p+1.
template <int BITS, int NPAIR>
__device__ __forceinline__ void decode_pairs(const uint32_t *w, float2 k[NPAIR]) {
    const float2 off = splat2(CodeWidth<BITS>::offset);
    if (BITS == 4) {
        // byte j of lo (hi) holds k + 8 of element 2j (2j+1) of that word
#pragma unroll
        for (int q = 0; q < NPAIR / 4; ++q) {
            const uint32_t u = w[q] ^ CodeWidth<4>::bias;
            const uint32_t lo = u & 0x0F0F0F0Fu, hi = (u >> 4) & 0x0F0F0F0Fu;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                k[4 * q + j] = sub2(make_float2(byte_as_magic(lo, j), byte_as_magic(hi, j)), off);
        }
    } else {
        // byte b of a word holds k + 128 of element 4q + b
#pragma unroll
        for (int q = 0; q < NPAIR / 2; ++q) {
            const uint32_t u = w[q] ^ CodeWidth<8>::bias;
            k[2 * q] = sub2(make_float2(byte_as_magic(u, 0), byte_as_magic(u, 1)), off);
            k[2 * q + 1] = sub2(make_float2(byte_as_magic(u, 2), byte_as_magic(u, 3)), off);
        }
    }
}

// store / load the packed codes of 8-element vector v (BITS/4 words each)
template <int BITS>
__device__ __forceinline__ void store_packed8(uint32_t *base, int64_t v, const Packed8<BITS> &p) {
    if (BITS == 4) base[v] = p.w[0];
    else reinterpret_cast<uint2 *>(base)[v] = make_uint2(p.w[0], p.w[BITS / 4 - 1]);
}
template <int BITS>
__device__ __forceinline__ void load_packed8(const uint32_t *base, int64_t v, uint32_t w[BITS / 4]) {
    if (BITS == 4) {
        w[0] = __ldg(base + v);
    } else {
        const uint2 t = __ldg(reinterpret_cast<const uint2 *>(base) + v);
        w[0] = t.x;
        w[BITS / 4 - 1] = t.y;
    }
}

// bf16 round-to-nearest-even of a pair, returned as one word (first value in
// the low half), and the pair's exact fp32 values
__device__ __forceinline__ uint32_t bf16x2_bits_rn(float2 v) {
    const __nv_bfloat162 b = __float22bfloat162_rn(v);
    return *reinterpret_cast<const uint32_t *>(&b);
}
__device__ __forceinline__ float2 bf16x2_to_f32(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// Quantize 8 values of a group: k = clamp(rint(v / scale), -L, L), ties to
// even, all 0 when scale == 0; the packed codes and k as floats in kf.
//
// inv is 1/scale rounded (0 when scale == 0, which makes every code 0).
// For a normal scale, q~ = v*inv differs from the rounded quotient
// fl(v/scale) by less than |q|*2^-22 (2^-20 for |q| <= 7, 2^-15 for
// |q| <= 127), so the two round to the same integer unless the exact
// quotient lies that close to a half-integer.  The fast path rounds q~ and
// flags any element whose q~ lies within twice that (the tie window) of a
// half-integer; then (rarely), and for every group whose scale lies outside
// [2^-100, 2^100], all 8 codes are taken from the IEEE division itself.
// Either way the codes are exactly those of rint(v/scale).  For a normal
// scale |q~| <= L*(1 + 2^-22) < L + 1/2, so the fast path needs no clamp.
struct GroupScale {
    float scale;  // a / L (0 for an all-zero group)
    float inv;    // 1 / scale rounded, 0 when scale == 0
    bool exact;   // scale outside [2^-100, 2^100]: always use the division
};

template <int BITS>
__device__ __forceinline__ GroupScale make_group_scale(float a) {
    GroupScale g;
    g.scale = a != 0.0f ? __fdiv_rn(a, CodeWidth<BITS>::levels) : 0.0f;
    g.exact = g.scale != 0.0f && (g.scale < 0x1p-100f || g.scale > 0x1p100f);
    g.inv = (g.scale != 0.0f && !g.exact) ? __frcp_rn(g.scale) : 0.0f;
    return g;
}

template <int BITS>
__device__ __forceinline__ Packed8<BITS> quantize8_exact(const float v[8], float scale, float kf[8]) {
    constexpr float L = CodeWidth<BITS>::levels;
    float t[8];
    for (int i = 0; i < 8; ++i) {
        t[i] = kRoundMagic;
        if (scale != 0.0f)
            t[i] = __fadd_rn(fminf(fmaxf(__fdiv_rn(v[i], scale), -L), L), kRoundMagic);
        kf[i] = __fsub_rn(t[i], kRoundMagic);
    }
    return pack_codes<BITS>(t);
}

template <int BITS>
__device__ __forceinline__ Packed8<BITS> quantize8(const float v[8], const GroupScale &g,
                                                   float kf[8], float2 z) {
    float tt[8];
    const float2 inv2 = splat2(g.inv), magic2 = splat2(kRoundMagic);
    float dmax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        const float2 q = prod2(make_float2(v[i], v[i + 1]), inv2, z);
        const float2 t = add2(q, magic2);
        const float2 k = sub2(t, magic2);
        const float2 d = sub2(q, k);
        kf[i] = k.x;
        kf[i + 1] = k.y;
        dmax = fmaxf(dmax, fmaxf(fabsf(d.x), fabsf(d.y)));
        tt[i] = t.x;
        tt[i + 1] = t.y;
    }
    if (g.exact || dmax > 0.5f - CodeWidth<BITS>::tie_window)
        return quantize8_exact<BITS>(v, g.scale, kf);
    return pack_codes<BITS>(tt);
}

// Quantize 8 values of a group through the correctly rounded quotient,
// computed without a division by Markstein's method (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990; the theorem as stated in
// Muller et al., "Handbook of Floating-Point Arithmetic", 2nd ed.):
// with y = RN(1/s) and q within one ulp of v/s, the remainder v - q*s is
// exact in one fma and RN(q + (v - q*s)*y) = RN(v/s).  q0 = RN(v*y) is
// within 1.5 ulp of v/s, one correction brings it within one ulp (its error
// shrinks by the factor |1 - s*y| <= 2^-24, plus half an ulp of rounding),
// and a second correction yields RN(v/s).  For s in [2^-100, 2^100] no
// intermediate overflows, and the remainders of the elements that can
// round to a nonzero code (|v| >= s/2) are normal numbers.  Then
// k = rint(RN(v/s)) exactly as the definition's division, and
// |RN(v/s)| <= L + ulp(L) rounds to at most L: no clamp.  A zero scale
// (inv = 0) gives q = 0 and all codes 0.  Other scales use the division.
template <int BITS>
__device__ __forceinline__ Packed8<BITS> quantize8_q(const float v[8], const GroupScale &g,
                                                     float kf[8], float2 z) {
    if (g.exact) return quantize8_exact<BITS>(v, g.scale, kf);
    float tt[8];
    const float2 y = splat2(g.inv), ns = splat2(-g.scale), magic2 = splat2(kRoundMagic);
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        const float2 x = make_float2(v[i], v[i + 1]);
        float2 q = prod2(x, y, z);     // RN(v*y)
        float2 r = fma2(q, ns, x);     // v - q*s, exact
        q = fma2(r, y, q);
        r = fma2(q, ns, x);
        q = fma2(r, y, q);             // RN(v/s)
        const float2 t = add2(q, magic2);
        const float2 k = sub2(t, magic2);
        kf[i] = k.x;
        kf[i + 1] = k.y;
        tt[i] = t.x;
        tt[i + 1] = t.y;
    }
    return pack_codes<BITS>(tt);
}

__device__ __forceinline__ void ld8(const float *p, float v[8]) {
    const float4 a = reinterpret_cast<const float4 *>(p)[0];
    const float4 b = reinterpret_cast<const float4 *>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void st8(float *p, const float v[8]) {
    reinterpret_cast<float4 *>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4 *>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

// ---- 32-byte stores (sm_100 st.global.v8)
//
// A thread of the reduce writes 32 contiguous bytes of each output and 64
// bytes of e_req per run.  One 32-byte store for each 32 bytes, in place of
// two 16-byte ones, halves the store instructions and writes whole 32-byte
// sectors per instruction (measured: the uncompensated call at 16 MiB per
// rank 74.4 -> 64.6 us, at 1 GiB 3.67 -> 3.49 ms; the compensated reduce
// 0.92 -> 0.89 ms).  The address must be 32-byte aligned.  Offsets inside a
// buffer are multiples of 32 bytes, so the callers test the buffer's base
// (the same for every thread) and otherwise take the 16-byte form: callers'
// outputs need only 16-byte alignment.
__device__ __forceinline__ bool aligned32(const void *p) {
    return (reinterpret_cast<uintptr_t>(p) & 31) == 0;
}
__device__ __forceinline__ void st32(float *p, const float v[8]) {
    asm volatile("st.global.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "f"(v[0]),
                 "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7])
                 : "memory");
}
__device__ __forceinline__ void st32_words(void *p, const uint32_t w[8]) {
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]),
                 "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                 : "memory");
}
// the streaming form (.cs: evict first), for outputs nothing reads back
__device__ __forceinline__ void st32_words_cs(void *p, const uint32_t w[8]) {
    asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]),
                 "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                 : "memory");
}

__device__ __forceinline__ void ld32(const float *p, float v[8]) {
    asm volatile("ld.global.v8.f32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]),
                   "=f"(v[6]), "=f"(v[7])
                 : "l"(p));
}

// 8 floats at p (32 bytes): one 32-byte access when wide (p 32-byte aligned),
// else two 16-byte ones
__device__ __forceinline__ void ld8w(const float *p, float v[8], bool wide) {
    if (wide) ld32(p, v);
    else ld8(p, v);
}
__device__ __forceinline__ void st8w(float *p, const float v[8], bool wide) {
    if (wide) st32(p, v);
    else st8(p, v);
}

// 16 bf16 values (8 words) to the same 32 bytes of each of the n_out
// outputs, streamed: out.p[r] + run * 2 in 16-byte units
__device__ __forceinline__ void store_run_outputs(const OutPtrs &out, int n_out, int64_t run,
                                                  const uint32_t yw[8]) {
#pragma unroll
    for (int r = 0; r < kMaxRanks; ++r) {
        if (r < n_out) {
            uint4 *dst = out.p[r] + run * 2;
            if (aligned32(out.p[r])) {
                st32_words_cs(dst, yw);
            } else {
                __stcs(dst, make_uint4(yw[0], yw[1], yw[2], yw[3]));
                __stcs(dst + 1, make_uint4(yw[4], yw[5], yw[6], yw[7]));
            }
        }
    }
}

// the 16 floats of run `run` of a buffer of 16-float runs
__device__ __forceinline__ void store_run16(float *base, int64_t run, const float v[16]) {
    float *p = base + run * 16;
    if (aligned32(base)) {
        st32(p, v);
        st32(p + 8, v + 8);
    } else {
        st8(p, v);
        st8(p + 8, v + 8);
    }
}

}  // namespace echo
