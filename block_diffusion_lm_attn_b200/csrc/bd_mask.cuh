// The block-diffusion attention mask as per-row key intervals.
//
// Every query row's visible key set is two intervals [a0,a1) U [a2,a3):
//   training/prefill, noisy row of block k : [k b, k b + b) U [L, L + k b)
//   training/prefill, clean row of block k : {}             U [L, L + (k+1) b)
//   decode row j of a block after n cached : [0, n + b)   (bidirectional)
//                                            [0, n + j + 1) (causal)
//                                            [0, n)       (cross-attention only)
// which is the three-part mask M_BD / M_OBC / M_BC of "Nemotron-Labs-
// Diffusion-8B-Base 3x decoding speed-up", section 1 "Block Diffusion
// Attention", and the draft/verify attention of its section 2.
#pragma once

#include "bd_common.cuh"

namespace bd {

typedef __nv_bfloat16 bf16;

struct Span {
    int a0, a1, a2, a3;
};

__device__ __forceinline__ bool span_has(const Span &s, int c)
{
    return (c >= s.a0 && c < s.a1) || (c >= s.a2 && c < s.a3);
}

// The visible keys of training/prefill row r of [x_t ; x_0] (2L rows).
__device__ __forceinline__ Span fwd_span(int L, int b, int r)
{
    Span s;
    if (r < L) {
        int kb = r / b;
        s.a0 = kb * b; s.a1 = kb * b + b; s.a2 = L; s.a3 = L + kb * b;
    } else {
        int kb = (r - L) / b;
        s.a0 = 0; s.a1 = 0; s.a2 = L; s.a3 = L + (kb + 1) * b;
    }
    return s;
}

} // namespace bd
