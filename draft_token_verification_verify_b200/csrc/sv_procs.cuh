// The further logits processors that act on raw logits before top-k,
// temperature and the softmax: the vocabulary mask and the repetition penalty
// (speculative decoding entry "推测解码", section "提议与核验的基本步骤",
// paragraph 4: every processing rule in effect applies to the target and the
// draft distributions alike).
//
// K0 turns each sequence's inputs into two bitmaps in the workspace, padded
// to a multiple of four words per row so that every 128-element run of them
// is a 16-byte aligned span a bulk copy can move next to the logits:
//   allow[s][w]  bit v % 32 of word v / 32: token v is allowed (the caller's
//                mask, all ones without one),
//   pen[s][w]    token v is listed for the penalty and theta_s != 1.
// A processed logit is then
//   -inf                                    if v is not allowed,
//   z / theta rounded (z > 0), z * theta    if v is penalised,
//   z                                       otherwise.
#pragma once

#include "sv_common.cuh"

namespace sv {

constexpr int PROCS_NT = 256;

struct ProcsParams {
    const uint32_t* mask;     // [S][words] or null
    const int32_t* rep_ids;   // [S][n_rep] or null
    int n_rep;
    const float* rep_penalty; // [S] or null
    int V;
    int words;                // ceil(V / 32)
    int W4;                   // words per bitmap row (multiple of 4)
    uint32_t* allow;          // [S][W4]
    uint32_t* pen;            // [S][W4]
};

// What the streaming, per-sequence and residual kernels need to process a
// logit: the two bitmap rows and theta of one sequence.
struct ProcView {
    const uint32_t* allow;  // row of the sequence, or null (no processors)
    const uint32_t* pen;
    float theta;
};

__device__ __forceinline__ float penalise(float z, float theta) {
    return z > 0.f ? __fdiv_rn(z, theta) : __fmul_rn(z, theta);
}

// Processed logit of token v with raw logit z.
__device__ __forceinline__ float proc_logit(float z, long long v, const ProcView& pv) {
    if (!pv.allow) return z;
    const uint32_t bit = 1u << (v & 31);
    if (!(__ldg(pv.allow + (v >> 5)) & bit)) return NEG_INF;
    if (__ldg(pv.pen + (v >> 5)) & bit) z = penalise(z, pv.theta);
    return z;
}

__device__ __forceinline__ ProcView proc_view(const uint32_t* allow, const uint32_t* pen, const float* theta,
                                              int W4, long long s) {
    ProcView pv;
    pv.allow = allow ? allow + s * W4 : nullptr;
    pv.pen = pen ? pen + s * W4 : nullptr;
    pv.theta = theta ? theta[s] : 1.f;
    return pv;
}

// K0: one CTA per sequence builds its two bitmap rows.  Launched in plain
// stream order (not as a programmatic dependent), so the previous call's
// kernels, which may still read the bitmaps, have completed.
__global__ void __launch_bounds__(PROCS_NT) sv_procs_kernel(const ProcsParams P) {
    const long long s = blockIdx.x;
    uint32_t* allow = P.allow + s * P.W4;
    uint32_t* pen = P.pen + s * P.W4;
    for (int w = threadIdx.x; w < P.W4; w += PROCS_NT) {
        allow[w] = P.mask ? (w < P.words ? __ldg(P.mask + s * P.words + w) : 0u) : 0xffffffffu;
        pen[w] = 0u;
    }
    __syncthreads();
    const float theta = P.rep_penalty ? P.rep_penalty[s] : 1.f;
    if (P.rep_ids && theta != 1.f) {
        for (int i = threadIdx.x; i < P.n_rep; i += PROCS_NT) {
            const int v = __ldg(P.rep_ids + s * P.n_rep + i);
            if (v >= 0 && v < P.V) atomicOr(pen + (v >> 5), 1u << (v & 31));
        }
    }
    pdl_launch_dependents();
}

}  // namespace sv
