// The nucleus (top-p) cut of a full row, for verification and sampling
// without a kept list (speculative decoding entry "推测解码", section
// "提议与核验的基本步骤", paragraph 4: nucleus sampling is one of the
// processing rules that act on the target and the draft distributions alike).
//
// With the tokens ordered by probability, the cut is the first token at which
// the running sum reaches top_p, and every token whose probability is at least
// that token's is kept and renormalised.  Probability is monotone in the
// processed logit z, so the kept set is {z >= z_cut}: the largest logit value
// whose tail mass (the weights of the values >= it) reaches top_p times the
// row's mass.  K2 and K3 already read a per-row logit threshold with its
// normaliser, so the cut enters them as that threshold.
//
// Masses are sums of fixed-point weights W = round(2^(z*c - m) * 2^40) (the
// row maximum has weight 2^40): integer sums are exact and independent of the
// order of the atomics, so every run takes the same decision.  The search
// takes two steps over the row:
//   1. a histogram of the weights by their binary exponent in steps of 1/8
//      (bin = floor(8 * (m - z*c)), monotone in z, so a bin is a range of z);
//      the bins are spread over the distribution's slope, which keeps the
//      shared-memory atomics of a row from piling onto one address;
//   2. inside the bin that holds the cut, an exact radix select over the
//      order-preserving keys of z (8 bits per pass; two passes for bf16
//      logits, whose keys have 16 significant bits, four otherwise), each
//      pass choosing the digit whose tail mass reaches what is left of the
//      target.
// With few rows the nucleus kernel splits each row over a thread-block
// cluster: every CTA histograms its share of the row in its own shared
// memory, CTA 0 sums the cluster's histograms through distributed shared
// memory and takes each decision, the others read it back from CTA 0.
#pragma once

#include <cooperative_groups.h>

#include "sv_common.cuh"
#include "sv_procs.cuh"

namespace sv {

constexpr int NUC_NT = 256;

struct NucRec {
    float cut;   // kept iff z >= cut
    float invS;  // 1 / the kept mass (weights 2^(z*c - m))
};

struct __align__(16) NucCtl {
    unsigned long long hist[256];
    unsigned long long trem;   // target mass still to be covered
    unsigned long long above;  // mass of the values above the current bin or digit
    unsigned long long last;   // mass of the chosen digit
    uint32_t prefix;           // key digits chosen so far
    int bin;                   // weight bin of the cut (histogram index)
    float m, s;                // merged row statistics (the kernel below)
};

// vector q of a row: elements [q*VEC, q*VEC + VEC) clipped to [0, V)
template <int DT>
__device__ __forceinline__ void load_vec(const void* row, bool aligned, int q, int V, float* v) {
    constexpr int VEC = VT<DT>::VEC;
    const long long e = static_cast<long long>(q) * VEC;
    if (aligned && e + VEC <= V) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(row) + q);
        unpack<DT>(raw, v);
    } else {
#pragma unroll
        for (int t = 0; t < VEC; ++t) v[t] = (e + t < V) ? load_elem<DT>(row, e + t) : NEG_INF;
    }
}

// Warp 0: the highest histogram index h whose tail mass (indices >= h)
// reaches `trem`; `before` is the mass of the indices above h, `at` that of h.
__device__ __forceinline__ void nuc_pick(const unsigned long long* hist, unsigned long long trem, int lane,
                                         int& digit, unsigned long long& before, unsigned long long& at) {
    unsigned long long s = 0ull;
#pragma unroll
    for (int i = 0; i < 8; ++i) s += hist[255 - 8 * lane - i];
    unsigned long long incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    const unsigned hit = __ballot_sync(0xffffffffu, incl >= trem);
    const int L = hit ? __ffs(hit) - 1 : 31;
    int dg = 0;
    unsigned long long bf = 0ull, a = 0ull;
    if (lane == L) {
        unsigned long long cum = incl - s;
        for (int i = 0; i < 8; ++i) {
            const int h = 255 - 8 * lane - i;
            const unsigned long long hv = hist[h];
            if (cum + hv >= trem || i == 7) {
                dg = h;
                bf = cum;
                a = hv;
                break;
            }
            cum += hv;
        }
    }
    digit = __shfl_sync(0xffffffffu, dg, L);
    before = __shfl_sync(0xffffffffu, bf, L);
    at = __shfl_sync(0xffffffffu, a, L);
}

// Nucleus cut of one row by one CTA (CL = false) or by the CTAs of a cluster
// (CL = true, each taking every ncl-th group of vectors).  Elements below
// tau0 (a top-k threshold, or -inf) weigh nothing; msc is the row maximum
// times c (over the elements >= tau0), 0 < tp < 1.  Every thread calls it;
// the results are returned to all of them.
template <int DT, int NT, bool CL = false>
__device__ void nucleus_block(const void* row, int V, float tau0, float msc, float c, float tp, const ProcView& pv,
                              NucCtl& N, float& cut, float& invS) {
    constexpr int VEC = VT<DT>::VEC;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int crank = 0, ncl = 1;
    if constexpr (CL) {
        crank = static_cast<int>(cooperative_groups::this_cluster().block_rank());
        ncl = static_cast<int>(cooperative_groups::this_cluster().num_blocks());
    }
    const bool lead = crank == 0;  // takes the decisions
    // CL: sum the cluster's histograms into CTA 0's
    auto gather = [&]() {
        if constexpr (CL) {
            auto cl = cooperative_groups::this_cluster();
            cl.sync();
            if (lead) {
                for (int h = tid; h < 256; h += NT) {
                    unsigned long long sum = N.hist[h];
                    for (int rk = 1; rk < ncl; ++rk) sum += *cl.map_shared_rank(&N.hist[h], rk);
                    N.hist[h] = sum;
                }
            }
        }
        __syncthreads();
    };
    // CL: every CTA takes CTA 0's decision
    auto share = [&]() {
        if constexpr (CL) {
            auto cl = cooperative_groups::this_cluster();
            cl.sync();
            if (!lead && tid == 0) {
                const NucCtl* D = cl.map_shared_rank(&N, 0);
                N.bin = D->bin;
                N.above = D->above;
                N.trem = D->trem;
                N.prefix = D->prefix;
                N.last = D->last;
            }
        }
        __syncthreads();
    };
    const bool al = (reinterpret_cast<uintptr_t>(row) & 15u) == 0;
    const int nvec = (V + VEC - 1) / VEC;
    const int KROUNDS = (DT == 0 && !pv.allow) ? 2 : 4;
    // f(z, x, h) for every element >= tau0 of positive weight: x = z*c - m,
    // h = 255 - weight bin (higher h: heavier)
    auto visit = [&](auto&& f) {
        constexpr int U = 4;  // vector loads in flight per thread
        const int step = NT * ncl;
        for (int q0 = crank * NT + tid; q0 < nvec; q0 += step * U) {
            uint4 raw[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int q = q0 + u * step;
                if (al && q < nvec && static_cast<long long>(q + 1) * VEC <= V)
                    raw[u] = __ldg(reinterpret_cast<const uint4*>(row) + q);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int q = q0 + u * step;
                if (q >= nvec) continue;
                const long long e0 = static_cast<long long>(q) * VEC;
                float v[VEC];
                if (al && e0 + VEC <= V) {
                    unpack<DT>(raw[u], v);
                } else {
#pragma unroll
                    for (int t = 0; t < VEC; ++t) v[t] = (e0 + t < V) ? load_elem<DT>(row, e0 + t) : NEG_INF;
                }
#pragma unroll
                for (int t = 0; t < VEC; ++t) {
                    const long long e = e0 + t;
                    float z = v[t];
                    if (pv.allow && e < V) z = proc_logit(z, e, pv);
                    if (!(z >= tau0) || !(z > NEG_INF)) continue;  // also clips the vector past V (-inf)
                    const float x = fmaf(z, c, -msc);
                    const int bin = min(max(static_cast<int>(floorf(-8.f * x)), 0), 255);
                    f(z, x, 255 - bin);
                }
            }
        }
    };
    auto weight = [](float x) { return __float2ull_rn(ex2(x) * 0x1p40f); };

    // 1. weight bins
    for (int h = tid; h < 256; h += NT) N.hist[h] = 0ull;
    __syncthreads();
    unsigned long long tail = 0ull;  // the last bin (weights below 2^-32) holds most of a
                                     // peaked row: summed in a register, added once
    visit([&](float, float x, int h) {
        const unsigned long long W = weight(x);
        if (h == 0)
            tail += W;
        else if (W)
            atomicAdd(&N.hist[h], W);
    });
    if (tail) atomicAdd(&N.hist[0], tail);
    gather();
    if (lead && warp == 0) {
        unsigned long long tot = 0ull;
#pragma unroll
        for (int i = 0; i < 8; ++i) tot += N.hist[8 * lane + i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
        // the running sum reaches top_p: mass >= tp * total, in integers
        const unsigned long long target =
            static_cast<unsigned long long>(ceil(static_cast<double>(tp) * static_cast<double>(tot)));
        int dg;
        unsigned long long bf, at;
        nuc_pick(N.hist, target, lane, dg, bf, at);
        if (lane == 0) {
            N.bin = dg;
            N.above = bf;
            N.trem = target - bf;
            N.prefix = 0u;
            N.last = at;
        }
    }
    share();
    // 2. exact key digits inside that bin
    const int hb = N.bin;
    for (int round = 0; round < KROUNDS; ++round) {
        const int shift = 24 - 8 * round;
        for (int h = tid; h < 256; h += NT) N.hist[h] = 0ull;
        __syncthreads();
        const uint32_t pre = N.prefix;
        visit([&](float z, float x, int h) {
            if (h != hb) return;
            const uint32_t key = okey(z);
            if (round != 0 && (key >> (shift + 8)) != pre) return;
            const unsigned long long W = weight(x);
            if (W) atomicAdd(&N.hist[(key >> shift) & 255u], W);
        });
        gather();
        if (lead && warp == 0) {
            int dg;
            unsigned long long bf, at;
            nuc_pick(N.hist, N.trem, lane, dg, bf, at);
            if (lane == 0) {
                N.prefix = (pre << 8) | static_cast<uint32_t>(dg);
                N.above += bf;
                N.trem -= bf;
                N.last = at;
            }
        }
        share();
    }
    const uint32_t p = N.prefix;
    cut = okey_inv(KROUNDS == 2 ? (p << 16 | ((p & 0x8000u) ? 0u : 0xffffu)) : p);
    const unsigned long long kept = N.above + N.last;
    invS = kept ? static_cast<float>(0x1p40 / static_cast<double>(kept)) : __int_as_float(0x7fc00000);
    if constexpr (CL)
        cooperative_groups::this_cluster().sync();  // no CTA leaves while CTA 0's decision is read
    else
        __syncthreads();  // N is reused by the caller
}

struct NucParams {
    const void* target;        // [B][k+1][V] (sampler: [rows][V])
    const void* draft;         // [B][k][V] or null
    long long B;
    int k;
    int V;
    const float* temperature;  // [B] or null
    const SegRec* segs;        // [R][nseg] softmax partials of the streaming pass
    int nseg;
    const float* top_p;        // [S]
    int procs_div;             // the processors' (and top_p's) sequence of b: b / procs_div
    const uint32_t* allow;     // [S][W4] or null
    const uint32_t* pen;
    const float* theta;
    int W4;
    NucRec* out;               // [R]
};

// One cluster of CTAs per row (launched with cluster size 1 to 16): the row's
// cut and kept normaliser.  Rows whose sequence has no nucleus (top_p = 1),
// an invalid setting or an invalid row get {-inf, 1/S}: K2 validates the
// settings and the row itself.
template <int DT>
__global__ void __launch_bounds__(NUC_NT) sv_nucleus_kernel(const NucParams P) {
    constexpr int ELT = VT<DT>::ELT;
    __shared__ NucCtl N;
    const long long r = blockIdx.x / cooperative_groups::this_cluster().num_blocks();
    const long long Rt = P.B * (P.k + 1);
    const char* row;
    long long b;
    if (r < Rt) {
        row = static_cast<const char*>(P.target) + static_cast<size_t>(r) * P.V * ELT;
        b = r / (P.k + 1);
    } else {
        row = static_cast<const char*>(P.draft) + static_cast<size_t>(r - Rt) * P.V * ELT;
        b = (r - Rt) / P.k;
    }
    const long long s = b / P.procs_div;
    pdl_wait_primary();  // the streaming pass's partials are complete
    pdl_launch_dependents();
    const int tid = threadIdx.x, lane = tid & 31;
    if (tid < 32) {
        float m = NEG_INF, sm = 0.f;
        for (int q = lane; q < P.nseg; q += 32) {
            const SegRec g = P.segs[r * P.nseg + q];
            ms_combine(m, sm, g.m, g.s);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            ms_combine(m, sm, __shfl_xor_sync(0xffffffffu, m, o), __shfl_xor_sync(0xffffffffu, sm, o));
        if (lane == 0) {
            N.m = m;
            N.s = sm;
        }
    }
    __syncthreads();
    const float m = N.m, sm = N.s;
    const float tp = P.top_p[s];
    const float T = P.temperature ? P.temperature[b] : 1.f;
    NucRec rec;
    rec.cut = NEG_INF;
    rec.invS = 1.f / sm;
    const bool ok = tp > 0.f && tp < 1.f && T > 0.f && T != POS_INF && m > NEG_INF && m < POS_INF && sm > 0.f;
    if (ok) {  // uniform over the block
        const float c = LOG2E / T;
        const ProcView pv = proc_view(P.allow, P.pen, P.theta, P.W4, s);
        nucleus_block<DT, NUC_NT, true>(row, P.V, NEG_INF, m, c, tp, pv, N, rec.cut, rec.invS);
    }
    if (tid == 0 && cooperative_groups::this_cluster().block_rank() == 0) P.out[r] = rec;
}

}  // namespace sv
