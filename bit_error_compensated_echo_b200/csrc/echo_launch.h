// echo_launch.h -- host-side launchers of the entry, reduce, exit,
// reduce-scatter and fix-up kernels, shared by the plan of P virtual ranks
// on one GPU (echo.cu) and the plan of one rank of a group spread over
// processes (echo_rank.cu).  The kernels are instantiated once, in
// echo_launch.cu; these functions pick the instance for the run-time code
// width, group size and rank count and launch it on the given stream.  They
// do not check errors: the caller reads cudaGetLastError().
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "echo.h"
#include "echo_common.cuh"

namespace echo {

// The buffers and sizes one launch works on.
//   n_vec     : 8-element vectors in one row of the codes / state arrays
//   chunk_vec : vectors in one owner chunk of such a row
//   P         : ranks summed by the reduce (and chunks per row at entry)
struct Bufs {
    float *m_fast = nullptr, *m_slow = nullptr;    // [rows][n_vec*8] fp32
    uint32_t *codes = nullptr;                     // [rows][n_vec*8*bits/8] bytes
    float *scales = nullptr;                       // [rows][n_vec*8/G]
    uint32_t *rcodes = nullptr;                    // reduced codes
    float *rscales = nullptr;                      // reduced scales
    float *e_req = nullptr;                        // requantization / output residual
    int64_t n_vec = 0, chunk_vec = 0;
    int P = 1, G = 128, bits = 4;
    bool comp = true;
    Consts k{};
};

// The fp32 constants of the definition for *cfg; 1 - beta and 1 - alpha are
// rounded once, as the oracle rounds them.
inline Consts make_consts(const echo_config &c) {
    Consts k{};
    k.alpha = c.alpha;
    k.one_m_alpha = 1.0f - c.alpha;
    k.beta_fast = c.beta_fast;
    k.one_m_beta_fast = 1.0f - c.beta_fast;
    k.beta_slow = c.beta_slow;
    k.one_m_beta_slow = 1.0f - c.beta_slow;
    k.neg_zero = -0.0f;   // the run-time -0 addend of the packed products
    return k;
}

// The e_req value of "no fix-up pending" (see echo_fill_kernel).
constexpr float kNoFixup = -0.0f;

// p[0..n) = v on st.
void launch_fill(float *p, int64_t n, float v, cudaStream_t st);

// Entry over `rows` input rows (grid y = rows * P chunks).  rank0: index of
// row 0 in the group (the owner test for the deferred fix-up);
// er_chunk_vec: vectors between consecutive owners' e_req chunks (0 when
// e_req holds one chunk).  dst: where each chunk's codes and scales go;
// nullptr: b.codes / b.scales, chunk after chunk.
void launch_entry(const Bufs &b, const InPtrs &x, int rows, int rank0, int64_t er_chunk_vec,
                  Slab sl, bool defer, cudaStream_t st, const ChunkDst *dst = nullptr);

// b.codes / b.scales seen as consecutive chunks of b.chunk_vec vectors, and
// b.rcodes / b.rscales the same way.
ChunkDst chunks_of(const Bufs &b);
ChunkSrc reduced_chunks_of(const Bufs &b);

// Reduce of `owners` chunks (grid y): sum the P rows, requantize; with
// n_out > 0 also write the dequantized sum to the n_out outputs (else that
// is launch_exit's job); compensating, either write e_req or, with fix,
// apply the owner fix-up to state row o of each chunk o.
void launch_reduce(const Bufs &b, int owners, Slab sl, cudaStream_t st,
                   const OutPtrs *out = nullptr, int n_out = 0, bool fix = false);

// Exit over `owners` chunks (grid y): dequantize the reduced transport into
// n_out outputs.  src: where each owner's reduced chunk is read; nullptr:
// b.rcodes / b.rscales, chunk after chunk.
void launch_exit(const Bufs &b, const OutPtrs &out, int n_out, int owners, Slab sl,
                 cudaStream_t st, const ChunkSrc *src = nullptr);

// Reduce-scatter second kernel over `owners` chunks (grid y): out.p[o]
// receives bf16(s) of chunk o; fix: owner residual folded into state row o.
void launch_rs(const Bufs &b, const OutPtrs &out, int owners, Slab sl, bool fix,
               cudaStream_t st);

// Owner fix-up (src == dst) or state copy with the fix-up applied on the
// way, over `owners` chunks of `ranks` state rows.
void launch_fixup(const Bufs &b, const float *src_fast, const float *src_slow, float *dst_fast,
                  float *dst_slow, int ranks, int owners, bool apply, bool only_owner, Slab sl,
                  cudaStream_t st);

// The library's device error word on the current device (kernels set the
// kDevErr* bits of echo_stage.cuh in it): *flags = its value, then cleared
// if clear.  A synchronous copy.
cudaError_t device_error_read(int32_t *flags, bool clear);

// One block of 32 threads that waits, bounded, on a barrier nothing
// completes, so that the wait runs out and sets kDevErrWaitTimeout.
void launch_wait_selftest(cudaStream_t st);

}  // namespace echo
