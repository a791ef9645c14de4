// echo_exit.cuh -- the all-gather half: dequantize the reduced chunks to bf16
// (operation: include/echo.h; conventions: echo_common.cuh)
#pragma once

#include "echo_common.cuh"

namespace echo {

// ------------------------------------------------------------ echo_exit
//
// All-gather half: dequantize the reduced codes once to bf16 and write them
// to n_out outputs (all P ranks' on one GPU, this process's one across
// GPUs).  Owner o's reduced chunk is read from src.codes[o] / src.scales[o]
// (ChunkSrc): one local buffer, or, on the rank path, owner o's own buffer
// on its GPU, so that the all-gather is these loads.  Calls on one GPU
// skip the kernel: their reduce writes the outputs itself; the rank path
// launches it.
// Grid: x over the vectors of the slab, y = owner.
template <int G, int BITS>
__global__ void __launch_bounds__(kThreads)
echo_exit_kernel(const __grid_constant__ ChunkSrc src, const __grid_constant__ OutPtrs out,
                 int n_out, int64_t chunk_vec, Slab sl) {
    constexpr int LANES = G / kVec;
    const int o = blockIdx.y;
    const int64_t local = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (local >= sl.v_count) return;
    const int64_t vc = sl.v_begin + local;                  // vector in chunk o
    const int64_t j = (int64_t)o * chunk_vec + vc;          // vector in the output

    uint32_t w[BITS / 4];
    load_packed8<BITS>(reinterpret_cast<const uint32_t *>(src.codes[o]), vc, w);
    const float2 sc2 = splat2(__ldg(src.scales[o] + vc / LANES));
    float2 kp[4];
    decode_pairs<BITS, 4>(w, kp);
    uint32_t yw[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) yw[p] = bf16x2_bits_rn(mul2(kp[p], sc2));
    const uint4 y = make_uint4(yw[0], yw[1], yw[2], yw[3]);
#pragma unroll
    for (int r = 0; r < kMaxRanks; ++r)
        if (r < n_out) __stcs(out.p[r] + j, y);
}

// The same pass with a thread per 16-element run: 8 (16) bytes of codes, 16
// bf16 values, and one 32-byte store per output (store_run_outputs).  Half
// as many threads as the kernel above, so it pays only on large slabs.
// With P = 8 outputs per thread (measured while one GPU's compensated calls
// still ran this pass, G = 128): 1.377 -> 1.330 ms at 1 GiB per rank; the
// call within 0.2 % at 64 MiB per rank, 1 % slower at 16 MiB, 7 % slower at
// the Llama shape (1 Mi elements per owner).  With one output (a rank of
// the rank path, P = 8): 0.283 -> 0.209 ms at 2^29 elements per rank, 0.074
// -> 0.056 ms at 2^27, 16.8 -> 14.7 us at 2^25; at 2^23 and below both take
// 4-6 us, bound by the launch.  The launcher takes it from kExitRunMinRuns
// runs per owner chunk in the slab.
// Grid: x over the 16-element runs of the slab, y = owner.
constexpr int64_t kExitRunMinRuns = int64_t(1) << 18;   // 2^22 elements per owner

template <int G, int BITS>
__global__ void __launch_bounds__(kThreads)
echo_exit_run_kernel(const __grid_constant__ ChunkSrc src, const __grid_constant__ OutPtrs out,
                     int n_out, int64_t chunk_vec, Slab sl) {
    constexpr int LANES = G / 16;                           // runs per group
    constexpr int WORDS = BITS / 2;                         // words holding 16 codes
    const int o = blockIdx.y;
    const int64_t local = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (local >= sl.v_count / 2) return;
    const int64_t rc = sl.v_begin / 2 + local;              // run in chunk o
    const int64_t j = (int64_t)o * (chunk_vec / 2) + rc;    // run in the output

    uint32_t w[WORDS];
    if (BITS == 4) {
        const uint2 t = __ldg(reinterpret_cast<const uint2 *>(src.codes[o]) + rc);
        w[0] = t.x;
        w[WORDS - 1] = t.y;
    } else {
        const uint4 t = __ldg(reinterpret_cast<const uint4 *>(src.codes[o]) + rc);
        w[0] = t.x;
        w[1 % WORDS] = t.y;
        w[2 % WORDS] = t.z;
        w[WORDS - 1] = t.w;
    }
    const float2 sc2 = splat2(__ldg(src.scales[o] + rc / LANES));
    float2 kp[8];
    decode_pairs<BITS, 8>(w, kp);
    uint32_t yw[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) yw[p] = bf16x2_bits_rn(mul2(kp[p], sc2));
    store_run_outputs(out, n_out, j, yw);
}

}  // namespace echo
