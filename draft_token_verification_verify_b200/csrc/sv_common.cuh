// Shared device definitions of the verification kernels: workspace records,
// element unpacking, order-preserving keys and warp reductions.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "sv_ptx.cuh"

namespace sv {

constexpr float NEG_INF = -__builtin_huge_valf();
constexpr float POS_INF = __builtin_huge_valf();
constexpr float LOG2E = 1.4426950408889634f;

// K1 modes
constexpr int MODE_GREEDY = 0;   // per-segment raw max and lowest-index argmax
constexpr int MODE_SOFTMAX = 1;  // per-segment online (max, sum of 2^(z*c - max))
constexpr int MODE_TOPK = 2;     // per-segment raw max + exact per-chunk kept list
constexpr int MODE_MAXONLY = 3;  // per-segment raw max (top-k resolved by radix select)

constexpr int REC_TIMEOUT = 1;   // a bulk-copy wait ran out
constexpr int REC_OVERFLOW = 2;  // the kept list did not fit

// Per-segment partial of one row (16 bytes).
struct SegRec {
    float m;    // raw max (greedy/top-k) or max of z*c (softmax); NaN-propagating
    float s;    // softmax: sum over the segment of 2^(z*c - m)
    int arg;    // greedy: lowest index holding the segment max (-1: none)
    int flags;  // REC_*
};

// Per-chunk kept list header of one row (32 bytes).  A list flagged
// REC_OVERFLOW is incomplete and the row's threshold is resolved exactly by
// the per-sequence kernel.
struct ChunkRec {
    float tau;   // K-th largest raw logit of the chunk (-inf if it has fewer than K)
    float last;  // smallest stored value
    int n;       // stored entries (sorted by index)
    int flags;   // REC_*
    float m;     // chunk maximum (NaN-propagating)
    float s;     // sum over the stored entries of 2^((z - m) * log2(e) / T)
    float zd;    // logit at the row's draft token if stored, else -inf
    int pad;
};

struct Cand {
    float v;
    int i;
};


// A final draw handed from the per-sequence kernel to the segment kernel
// (64 bytes): weights w(v) = max(0, p(v) - q(v)) over the row pair of position
// j, or p(v) alone, with p(v) = [z_t(v) >= t_tau] 2^(z_t(v)*c - t_msc) * t_invS
// and q(v) likewise from the draft row.
struct DrawReq {
    int need;        // 1: this sequence's draw is done by the segment kernel
    int j;           // position of the draw (= accepted draft tokens)
    int use_q;       // 1: residual weights, 0: p alone
    int pad0;
    long long rowt;  // row index of the target row in the target tensor
    long long rowd;  // row index of the draft row in the draft tensor
    float t_msc, t_invS, t_tau;
    float d_msc, d_invS, d_tau;
    float u;         // the sequence's final uniform u_k
    float c;         // log2(e) / T
};

template <int DT>
struct VT;
template <>
struct VT<0> {  // bf16
    static constexpr int ELT = 2, VEC = 8;
};
template <>
struct VT<1> {  // fp32
    static constexpr int ELT = 4, VEC = 4;
};

__device__ __forceinline__ uint32_t bf16x2_max_nan(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

template <int DT>
__device__ __forceinline__ void unpack(const uint4& r, float* v) {
    if constexpr (DT == 0) {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            v[2 * t] = __uint_as_float(w[t] << 16);
            v[2 * t + 1] = __uint_as_float(w[t] & 0xffff0000u);
        }
    } else {
        v[0] = __uint_as_float(r.x);
        v[1] = __uint_as_float(r.y);
        v[2] = __uint_as_float(r.z);
        v[3] = __uint_as_float(r.w);
    }
}

// NaN-propagating maximum of a full 16-byte vector.
template <int DT>
__device__ __forceinline__ float vmax_nan(const uint4& r) {
    if constexpr (DT == 0) {
        const uint32_t m = bf16x2_max_nan(bf16x2_max_nan(r.x, r.y), bf16x2_max_nan(r.z, r.w));
        return fmax_nan(__uint_as_float(m << 16), __uint_as_float(m & 0xffff0000u));
    } else {
        return fmax_nan(fmax_nan(__uint_as_float(r.x), __uint_as_float(r.y)),
                        fmax_nan(__uint_as_float(r.z), __uint_as_float(r.w)));
    }
}

template <int DT>
__device__ __forceinline__ float load_elem(const void* base, long long e) {
    if constexpr (DT == 0) {
        return __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t*>(base)[e]) << 16);
    } else {
        return static_cast<const float*>(base)[e];
    }
}

// Order-preserving unsigned key of a non-NaN float; -0.0 maps to +0.0.
__device__ __forceinline__ uint32_t okey(float x) {
    uint32_t b = __float_as_uint(x);
    if (b == 0x80000000u) b = 0u;
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float okey_inv(uint32_t key) {
    const uint32_t b = (key & 0x80000000u) ? (key & 0x7fffffffu) : ~key;
    return __uint_as_float(b);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}
__device__ __forceinline__ float warp_max_nan(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmax_nan(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}
__device__ __forceinline__ float warp_incl_scan(float x, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    return x;
}

// Combine two (max, sum of 2^(y - max)) partials.
__device__ __forceinline__ void ms_combine(float& m, float& s, float m2, float s2) {
    const float M = fmax_nan(m, m2);
    if (M == NEG_INF) {
        s = 0.f;
    } else {
        s = s * ex2(m - M) + s2 * ex2(m2 - M);
    }
    m = M;
}

// (value, index) pair order for an argmax: larger value first, then the
// lower index (unsigned, so that -1 = "none" loses every tie).
__device__ __forceinline__ bool arg_better(float v1, int i1, float v2, int i2) {
    return v1 > v2 || (v1 == v2 && static_cast<unsigned>(i1) < static_cast<unsigned>(i2));
}

__host__ __device__ constexpr int pow2_ceil(int n) {
    int p = 1;
    while (p < n) p <<= 1;
    return p;
}

}  // namespace sv
