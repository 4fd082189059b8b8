// Speculative-sampling verification kernels for sm_100a.
//
// Method (speculative decoding entry "推测解码", section "提议与核验的基本步骤"):
// position i accepts the draft token d with probability min(1, p(d)/q(d)),
// p and q being the target and draft distributions after the same
// temperature / top-k processing; the first rejected position is redrawn from
// the normalised residual max(0, p - q); after k acceptances one bonus token is
// drawn from the target; greedy mode compares d with the target argmax.
//
// Work decomposition.  One UNIT is one position of one sequence: the pair
// (target row i, draft row i) for i < k, or the single target row k (bonus
// row; every row in greedy mode and in the proposer sampler).  A unit is owned
// by one thread-block cluster of C CTAs; CTA r holds elements
// [r*L, (r+1)*L) of each of the unit's rows in shared memory, brought in by
// bulk copies (cp.async.bulk, no multicast) completing on mbarriers whose
// waits are bounded in time.  The rows are read from HBM exactly once.
// Per-row statistics are combined across the cluster by pushing partial
// results into every peer's shared memory (st.shared::cluster) followed by a
// release/acquire cluster barrier, so that every CTA holds the same inputs and
// takes the same branch.
//
// Because the first rejected position j of a sequence is not known inside a
// unit, a unit that rejects locally draws its replacement speculatively (it is
// only used if i turns out to be the first rejection).  The unit writes one
// code into out_tokens[b][i]: CODE_ACCEPT, the speculative token, or an error
// code; a small second kernel (programmatic dependent launch) turns the codes
// of each sequence into the final tokens and the accepted count.
//
// Top-k.  tau is the K-th largest raw logit with multiplicity.  Candidate
// path: every group of g lanes computes the maximum of its elements; the K-th
// largest group maximum over the cluster is a lower bound beta <= tau (K
// distinct elements are >= it), so every kept element is among the elements
// >= beta; these candidates (about K of them) are gathered in the leader CTA,
// which selects tau exactly, normalises over the kept entries and performs the
// accept / residual / bonus steps on the candidate lists alone.  Radix path
// (K too large, candidate overflow, or forced): a cluster-wide MSB-first radix
// select over order-preserving integer keys of the resident slices.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "sv_ptx.cuh"

namespace sv {

constexpr int MAX_CLUSTER = 16;
constexpr int MAX_WARPS = 16;      // up to 512 threads per CTA
constexpr int MAX_PIECES = 16;     // bulk-copy pieces per row slice
constexpr int GMAX = 256;          // group maxima per row over the cluster
constexpr int CAND_CAP = 256;      // top-k candidates per row gathered in the leader
constexpr int MAX_TILES = 64;      // residual-scan tiles per slice

constexpr int CODE_ACCEPT = -2;
constexpr int CODE_ROW_ERR = -3;
constexpr int CODE_TIMEOUT = -4;

constexpr float NEG_INF = -__builtin_huge_valf();
constexpr float POS_INF = __builtin_huge_valf();

struct Params {
    const void* target;          // [B][k+1][V] (sampler: [rows][V])
    const void* draft;           // [B][k][V] or null
    const int32_t* draft_tokens; // [B][k]
    const float* uniforms;       // [B][k+1] (sampler: [rows])
    const float* temperature;    // [B] (sampler: [rows]) or null
    int32_t* out_codes;          // [B][k+1] codes (sampler: [rows] final tokens)
    float* out_p;                // [B][k] or null
    float* out_q;                // [B][k] or null
    int32_t* out_status;         // 1 or null
    long long B;                 // sequences (sampler: rows)
    int k;
    int V;
    int top_k;                   // 0 = disabled (already normalised on the host)
    int greedy;
    int sample_only;             // proposer sampler: every unit is one row
    int C;                       // cluster size
    int L;                       // elements per CTA slice
    int piece_bytes;             // bulk-copy piece size (multiple of 16)
    int buf_bytes;               // shared bytes per row slice buffer
    int group_lanes;             // lanes per group for the top-k lower bound
    int use_cand;                // candidate path for top-k
    unsigned long long timeout_ns;
    unsigned int test_extra_tx;
};

struct __align__(16) Ctl {
    uint64_t mbar[2][MAX_PIECES];
    float g_recv[2][GMAX];               // group maxima of the whole cluster
    float ms_recv[MAX_CLUSTER][2][2];    // per CTA, per row: online (max, sum)
    float s_recv[MAX_CLUSTER][2];        // per CTA, per row: masked exp-sum (radix path)
    float w_recv[2][MAX_CLUSTER];        // per attempt, per CTA: residual mass
    float arg_v[MAX_CLUSTER];            // greedy: CTA best value
    int arg_i[MAX_CLUSTER];              // greedy: CTA best index
    float arg_m[MAX_CLUSTER];            // greedy: CTA NaN-propagating max
    int flags_recv[MAX_CLUSTER];         // per CTA: 1 = a wait ran out
    int cnt_recv[MAX_CLUSTER][2];        // per CTA: local candidate counts
    float z_recv[2];                     // logits at the draft token (target, draft)
    int cand_n[2];                       // leader: reserved candidate slots
    int cnt_local[2];
    int nk[2];
    float row_max[2];                    // raw maximum per row
    float beta[2];
    float tau[2];
    float ssum[2];
    uint32_t rprefix[2];
    int rk[2];
    float red_f[MAX_WARPS][2];
    float red4[MAX_WARPS][4];
    int red_i[MAX_WARPS];
    float red_m[MAX_WARPS];
    int sh_i[4];
    float sh_f[4];
    union {
        float gm_local[2][GMAX];         // phase 1: this CTA's group maxima
        struct {
            float v[2][CAND_CAP];        // leader: candidates
            int i[2][CAND_CAP];
            int sidx[2][CAND_CAP];       // leader: kept entries sorted by index
            float sval[2][CAND_CAP];
            float se[2][CAND_CAP];
        } cand;
        struct {
            int hist[2][256];
            int tot[2][256];
        } radix;
        struct {
            float part[MAX_TILES][MAX_WARPS];
            float sum[MAX_TILES];
        } tiles;
    } u;
};

constexpr int CTL_BYTES = (int)((sizeof(Ctl) + 127) / 128 * 128);

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
__device__ __forceinline__ float load_elem(const unsigned char* buf, int pos) {
    if constexpr (DT == 0) {
        return __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(buf)[pos]) << 16);
    } else {
        return reinterpret_cast<const float*>(buf)[pos];
    }
}

template <int DT>
__device__ __forceinline__ float load_global_elem(const char* row, long long e) {
    if constexpr (DT == 0) {
        return __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(row)[e]) << 16);
    } else {
        return reinterpret_cast<const float*>(row)[e];
    }
}

// Order-preserving unsigned key of a (non-NaN) float; -0.0 maps to +0.0.
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

__device__ __forceinline__ float warp_incl_scan(float x, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    return x;
}

// Combine two (max, sum-of-2^(y-max)) partials.
__device__ __forceinline__ void ms_combine(float& m, float& s, float m2, float s2) {
    const float M = fmax_nan(m, m2);
    if (M == NEG_INF) {
        s = 0.f;
    } else {
        s = s * ex2(m - M) + s2 * ex2(m2 - M);
    }
    m = M;
}

// Geometry of one row slice held in shared memory.  The buffer mirrors the
// 16-byte-aligned global span [A0, A0 + 16*nvec) that covers elements
// [lo, hi); element e sits at buffer position e - e0.
struct Geom {
    uintptr_t A0, ga, gb, ga16, gb16;
    int e0, nvec, npieces;
};

template <int ELT>
__device__ __forceinline__ Geom make_geom(const char* row, int lo, int hi, int piece_bytes) {
    Geom g;
    g.ga = reinterpret_cast<uintptr_t>(row) + static_cast<uintptr_t>(lo) * ELT;
    g.gb = reinterpret_cast<uintptr_t>(row) + static_cast<uintptr_t>(hi) * ELT;
    g.A0 = g.ga & ~static_cast<uintptr_t>(15);
    const uintptr_t A1 = (g.gb + 15) & ~static_cast<uintptr_t>(15);
    g.ga16 = (g.ga + 15) & ~static_cast<uintptr_t>(15);
    g.gb16 = g.gb & ~static_cast<uintptr_t>(15);
    g.e0 = lo - static_cast<int>((g.ga - g.A0) / ELT);
    g.nvec = (hi > lo) ? static_cast<int>((A1 - g.A0) / 16) : 0;
    g.npieces = (g.nvec * 16 + piece_bytes - 1) / piece_bytes;
    return g;
}

// ---------------------------------------------------------------------------
// The unit kernel
// ---------------------------------------------------------------------------

template <int DT, int NT>
__global__ void __launch_bounds__(NT, 1024 / NT) sv_unit_kernel(const Params P) {
    constexpr int ELT = VT<DT>::ELT;
    constexpr int VEC = VT<DT>::VEC;
    constexpr int NW = NT / 32;
    extern __shared__ __align__(128) unsigned char smem[];
    Ctl& S = *reinterpret_cast<Ctl*>(smem);
    unsigned char* const buf0 = smem + CTL_BYTES;
    unsigned char* const buf1 = smem + CTL_BYTES + P.buf_bytes;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int C = P.C;
    const uint32_t rank = cluster_ctarank();
    const long long unit = blockIdx.x / C;

    // Cluster start barrier: peers may only be written after every CTA of the
    // cluster has started; the wait comes right before the first push.
    cluster_arrive_relaxed();
    // Let the finalising kernel get scheduled while this grid drains.
    pdl_launch_dependents();

    // ---- decode the unit -----------------------------------------------------
    const int V = P.V, k = P.k;
    const bool sample = P.sample_only != 0;
    const bool greedy = P.greedy != 0;
    long long b;
    int i;
    if (sample) {
        b = unit;
        i = k;
    } else {
        b = unit / (k + 1);
        i = static_cast<int>(unit - b * (k + 1));
    }
    const bool pair = !sample && !greedy && i < k;
    const char* row0;
    const char* row1 = nullptr;
    if (sample)
        row0 = static_cast<const char*>(P.target) + static_cast<size_t>(unit) * V * ELT;
    else
        row0 = static_cast<const char*>(P.target) +
               (static_cast<size_t>(b) * (k + 1) + i) * static_cast<size_t>(V) * ELT;
    if (pair)
        row1 = static_cast<const char*>(P.draft) +
               (static_cast<size_t>(b) * k + i) * static_cast<size_t>(V) * ELT;
    int d = -1;
    if (!sample && i < k) d = P.draft_tokens[b * k + i];
    float T = 1.f, u_acc = 0.f, u_fin = 0.f;
    if (!greedy) {
        if (P.temperature) T = P.temperature[sample ? unit : b];
        if (sample) {
            u_fin = P.uniforms[unit];
        } else {
            u_fin = P.uniforms[b * (k + 1) + k];
            if (pair) u_acc = P.uniforms[b * (k + 1) + i];
        }
    }
    bool bad = false;
    if (!sample && i < k && (d < 0 || d >= V)) bad = true;
    if (!greedy) {
        if (!(T > 0.f) || T == POS_INF) bad = true;
        if (!(u_fin >= 0.f && u_fin < 1.f)) bad = true;
        if (pair && !(u_acc >= 0.f && u_acc < 1.f)) bad = true;
    }
    // log2(e) / T: the softmax is evaluated as 2^(z*c - m)
    const float c = (T > 0.f && T != POS_INF) ? (1.4426950408889634f / T) : 1.f;
    if (sample == false && unit == 0 && rank == 0 && tid == 0 && P.out_status) *P.out_status = 0;

    // ---- slice geometry and loads ------------------------------------------------
    const long long lo_ll = static_cast<long long>(rank) * P.L;
    const int lo = static_cast<int>(lo_ll < V ? lo_ll : V);
    const int hi = static_cast<int>(lo_ll + P.L < V ? lo_ll + P.L : V);
    const int nrows = pair ? 2 : 1;
    const Geom g0 = make_geom<ELT>(row0, lo, hi, P.piece_bytes);
    const Geom g1 = pair ? make_geom<ELT>(row1, lo, hi, P.piece_bytes) : Geom{0, 0, 0, 0, 0, 0, 0, 0};

    if (tid == 0) {
        for (int p = 0; p < g0.npieces; ++p) mbar_init(&S.mbar[0][p], 1);
        for (int p = 0; p < g1.npieces; ++p) mbar_init(&S.mbar[1][p], 1);
        fence_mbar_init();
    }
    if (tid < 2) {
        S.cand_n[tid] = 0;
        S.cnt_local[tid] = 0;
        S.nk[tid] = 0;
        S.beta[tid] = NEG_INF;
        S.tau[tid] = NEG_INF;
        S.rprefix[tid] = 0u;
        S.rk[tid] = P.top_k;
    }
    __syncthreads();
    if (tid == 0) {
        for (int p = 0; p < MAX_PIECES; ++p) {
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const Geom& g = r ? g1 : g0;
                unsigned char* buf = r ? buf1 : buf0;
                if (p >= g.npieces) continue;
                const uintptr_t s0 = g.A0 + static_cast<uintptr_t>(p) * P.piece_bytes;
                uintptr_t s1 = s0 + P.piece_bytes;
                const uintptr_t send = g.A0 + static_cast<uintptr_t>(g.nvec) * 16;
                if (s1 > send) s1 = send;
                const uintptr_t b0 = s0 > g.ga16 ? s0 : g.ga16;
                const uintptr_t b1 = s1 < g.gb16 ? s1 : g.gb16;
                const uint32_t bytes = (b1 > b0) ? static_cast<uint32_t>(b1 - b0) : 0u;
                mbar_arrive_expect_tx(&S.mbar[r][p], bytes + P.test_extra_tx);
                if (bytes) bulk_g2s(buf + (b0 - g.A0), reinterpret_cast<const void*>(b0), bytes, &S.mbar[r][p]);
            }
        }
    }
    // elements outside the 16-byte-aligned interior: plain loads
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        if (r >= nrows) break;
        const Geom& g = r ? g1 : g0;
        const char* row = r ? row1 : row0;
        unsigned char* buf = r ? buf1 : buf0;
        int nh, ntl;
        if (hi <= lo) {
            nh = 0;
            ntl = 0;
        } else if (g.ga16 >= g.gb16) {
            nh = hi - lo;
            ntl = 0;
        } else {
            nh = static_cast<int>((g.ga16 - g.ga) / ELT);
            ntl = static_cast<int>((g.gb - g.gb16) / ELT);
        }
        for (int t = tid; t < nh + ntl; t += NT) {
            const int e = t < nh ? lo + t : hi - ntl + (t - nh);
            if constexpr (DT == 0)
                reinterpret_cast<uint16_t*>(buf)[e - g.e0] = reinterpret_cast<const uint16_t*>(row)[e];
            else
                reinterpret_cast<float*>(buf)[e - g.e0] = reinterpret_cast<const float*>(row)[e];
        }
    }
    __syncthreads();

    // Scan the vectors of row r in arrival order.  f(raw, e, full): e is the
    // element index of the vector's first element; full = all VEC valid.
    bool ok = true;
    auto scan = [&](int r, auto&& f) {
        const Geom& g = r ? g1 : g0;
        const unsigned char* buf = r ? buf1 : buf0;
        const int vpp = P.piece_bytes / 16;
        for (int p = 0; p < g.npieces; ++p) {
            if (!mbar_wait_bounded(&S.mbar[r][p], 0u, P.timeout_ns)) {
                ok = false;
                return;
            }
            const int jend = min(g.nvec, (p + 1) * vpp);
            for (int j = p * vpp + tid; j < jend; j += NT) {
                const uint4 raw = *reinterpret_cast<const uint4*>(buf + 16 * j);
                const int e = g.e0 + j * VEC;
                f(raw, e, e >= lo && e + VEC <= hi);
            }
        }
    };
    auto valid = [&](int e) { return e >= lo && e < hi; };

    // =====================================================================
    // Greedy: lowest-index argmax of the target row.
    // =====================================================================
    if (greedy) {
        float best = NEG_INF, macc = NEG_INF;
        int bidx = -1;
        scan(0, [&](const uint4& raw, int e, bool full) {
            float vm;
            if (full) {
                vm = vmax_nan<DT>(raw);
            } else {
                float v[VEC];
                unpack<DT>(raw, v);
                vm = NEG_INF;
#pragma unroll
                for (int t = 0; t < VEC; ++t)
                    if (valid(e + t)) vm = fmax_nan(vm, v[t]);
            }
            macc = fmax_nan(macc, vm);
            if (vm > best) {
                float v[VEC];
                unpack<DT>(raw, v);
#pragma unroll
                for (int t = 0; t < VEC; ++t) {
                    if (valid(e + t) && v[t] == vm) {
                        bidx = e + t;
                        best = vm;
                        break;
                    }
                }
            }
        });
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ob = __shfl_xor_sync(0xffffffffu, best, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bidx, o);
            const float om = __shfl_xor_sync(0xffffffffu, macc, o);
            if (ob > best || (ob == best && static_cast<unsigned>(oi) < static_cast<unsigned>(bidx))) {
                best = ob;
                bidx = oi;
            }
            macc = fmax_nan(macc, om);
        }
        if (lane == 0) {
            S.red_f[warp][0] = best;
            S.red_i[warp] = bidx;
            S.red_m[warp] = macc;
        }
        const int tmo = __syncthreads_or(!ok);
        cluster_wait_acquire();  // completes the start barrier
        if (tid == 0) {
            float cb = S.red_f[0][0], cm = S.red_m[0];
            int ci = S.red_i[0];
            for (int w = 1; w < NW; ++w) {
                const float ob = S.red_f[w][0];
                const int oi = S.red_i[w];
                if (ob > cb || (ob == cb && static_cast<unsigned>(oi) < static_cast<unsigned>(ci))) {
                    cb = ob;
                    ci = oi;
                }
                cm = fmax_nan(cm, S.red_m[w]);
            }
            st_cluster_f32(mapa(&S.arg_v[rank], 0), cb);
            st_cluster_s32(mapa(&S.arg_i[rank], 0), ci);
            st_cluster_f32(mapa(&S.arg_m[rank], 0), cm);
            st_cluster_s32(mapa(&S.flags_recv[rank], 0), tmo ? 1 : 0);
        }
        cluster_sync_all();
        if (rank == 0 && tid == 0) {
            float cb = NEG_INF, cm = NEG_INF;
            int ci = -1, anytmo = 0;
            for (int r = 0; r < C; ++r) {
                const float ob = S.arg_v[r];
                const int oi = S.arg_i[r];
                if (ob > cb || (ob == cb && static_cast<unsigned>(oi) < static_cast<unsigned>(ci))) {
                    cb = ob;
                    ci = oi;
                }
                cm = fmax_nan(cm, S.arg_m[r]);
                anytmo |= S.flags_recv[r];
            }
            const bool err = bad || (cm != cm) || cm == POS_INF || ci < 0;
            int code;
            if (sample) {
                code = (anytmo || err) ? -1 : ci;
            } else if (anytmo) {
                code = CODE_TIMEOUT;
            } else if (err) {
                code = CODE_ROW_ERR;
            } else if (i < k) {
                code = (d == ci) ? CODE_ACCEPT : ci;
            } else {
                code = ci;
            }
            P.out_codes[unit] = code;
        }
        if (tmo && tid == 0) {
            for (int p = 0; p < g0.npieces; ++p) mbar_wait_bounded(&S.mbar[0][p], 0u, P.timeout_ns);
        }
        return;
    }

    // =====================================================================
    // Stochastic: pass 1 over the resident slices.
    // =====================================================================
    const bool topk = P.top_k > 0;
    float tmax0 = NEG_INF, tmax1 = NEG_INF;  // raw maxima (top-k)
    float om0 = NEG_INF, os0 = 0.f, om1 = NEG_INF, os1 = 0.f;  // online (max, sum) in log2 units
    if (topk) {
        auto fmx0 = [&](const uint4& raw, int e, bool full) {
            if (full) {
                tmax0 = fmax_nan(tmax0, vmax_nan<DT>(raw));
            } else {
                float v[VEC];
                unpack<DT>(raw, v);
#pragma unroll
                for (int t = 0; t < VEC; ++t)
                    if (valid(e + t)) tmax0 = fmax_nan(tmax0, v[t]);
            }
        };
        auto fmx1 = [&](const uint4& raw, int e, bool full) {
            if (full) {
                tmax1 = fmax_nan(tmax1, vmax_nan<DT>(raw));
            } else {
                float v[VEC];
                unpack<DT>(raw, v);
#pragma unroll
                for (int t = 0; t < VEC; ++t)
                    if (valid(e + t)) tmax1 = fmax_nan(tmax1, v[t]);
            }
        };
        scan(0, fmx0);
        if (pair) scan(1, fmx1);
    } else {
        auto online = [&](float& m, float& s, const uint4& raw, int e, bool full) {
            float v[VEC];
            unpack<DT>(raw, v);
            if (!full) {
#pragma unroll
                for (int t = 0; t < VEC; ++t)
                    if (!valid(e + t)) v[t] = NEG_INF;
            }
            float vm = v[0];
#pragma unroll
            for (int t = 1; t < VEC; ++t) vm = fmax_nan(vm, v[t]);
            const float ym = vm * c;
            if (!(ym <= m)) {  // new maximum, or NaN
                if (ym != ym) {
                    m = ym;
                } else {
                    s = (m == NEG_INF) ? 0.f : s * ex2(m - ym);
                    m = ym;
                }
            }
            if (vm != NEG_INF && m == m) {
#pragma unroll
                for (int t = 0; t < VEC; ++t) s += ex2(fmaf(v[t], c, -m));
            }
        };
        scan(0, [&](const uint4& raw, int e, bool full) { online(om0, os0, raw, e, full); });
        if (pair) scan(1, [&](const uint4& raw, int e, bool full) { online(om1, os1, raw, e, full); });
    }

    // ---- reduce this CTA's partials ----------------------------------------------
    const int G = P.group_lanes;            // lanes per group (top-k)
    const int Gc = NT / G;                  // groups per CTA
    const int Gt = C * Gc;                  // groups per cluster
    if (topk) {
        for (int o = 1; o < G; o <<= 1) {
            tmax0 = fmax_nan(tmax0, __shfl_xor_sync(0xffffffffu, tmax0, o));
            tmax1 = fmax_nan(tmax1, __shfl_xor_sync(0xffffffffu, tmax1, o));
        }
        if ((lane & (G - 1)) == 0) {
            S.u.gm_local[0][tid / G] = tmax0;
            S.u.gm_local[1][tid / G] = tmax1;
        }
    } else {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            ms_combine(om0, os0, __shfl_xor_sync(0xffffffffu, om0, o), __shfl_xor_sync(0xffffffffu, os0, o));
            ms_combine(om1, os1, __shfl_xor_sync(0xffffffffu, om1, o), __shfl_xor_sync(0xffffffffu, os1, o));
        }
        if (lane == 0) {
            S.red4[warp][0] = om0;
            S.red4[warp][1] = os0;
            S.red4[warp][2] = om1;
            S.red4[warp][3] = os1;
        }
    }
    const int tmo = __syncthreads_or(!ok);
    cluster_wait_acquire();  // completes the start barrier: peers may now be written

    // ---- phase 1 pushes ------------------------------------------------------------
    if (topk) {
        const int total = nrows * Gc * C;
        for (int t = tid; t < total; t += NT) {
            const int r = t / (Gc * C);
            const int rem = t - r * (Gc * C);
            const int grp = rem / C;
            const int peer = rem - grp * C;
            st_cluster_f32(mapa(&S.g_recv[r][rank * Gc + grp], peer), S.u.gm_local[r][grp]);
        }
    } else if (tid == 0) {
        float m0 = S.red4[0][0], s0 = S.red4[0][1], m1 = S.red4[0][2], s1 = S.red4[0][3];
        for (int w = 1; w < NW; ++w) {
            ms_combine(m0, s0, S.red4[w][0], S.red4[w][1]);
            ms_combine(m1, s1, S.red4[w][2], S.red4[w][3]);
        }
        for (int peer = 0; peer < C; ++peer) {
            st_cluster_f32(mapa(&S.ms_recv[rank][0][0], peer), m0);
            st_cluster_f32(mapa(&S.ms_recv[rank][0][1], peer), s0);
            st_cluster_f32(mapa(&S.ms_recv[rank][1][0], peer), m1);
            st_cluster_f32(mapa(&S.ms_recv[rank][1][1], peer), s1);
        }
    }
    if (tid == 32 % NT) {
        for (int peer = 0; peer < C; ++peer) st_cluster_s32(mapa(&S.flags_recv[rank], peer), tmo ? 1 : 0);
    }
    if (tid == 64 % NT && pair && d >= lo && d < hi && !tmo) {
        const float zt = load_elem<DT>(buf0, d - g0.e0);
        const float zd = load_elem<DT>(buf1, d - g1.e0);
        for (int peer = 0; peer < C; ++peer) {
            st_cluster_f32(mapa(&S.z_recv[0], peer), zt);
            st_cluster_f32(mapa(&S.z_recv[1], peer), zd);
        }
    }
    cluster_sync_all();  // sync #1

    // ---- every CTA: identical view of the cluster ---------------------------------
    int anytmo = 0;
    for (int r = 0; r < C; ++r) anytmo |= S.flags_recv[r];
    float M0 = NEG_INF, M1 = NEG_INF;     // raw maxima (top-k) / scaled maxima (no top-k)
    float Ssum0 = 0.f, Ssum1 = 0.f;
    if (topk) {
        for (int j = 0; j < Gt; ++j) {
            M0 = fmax_nan(M0, S.g_recv[0][j]);
            if (pair) M1 = fmax_nan(M1, S.g_recv[1][j]);
        }
    } else {
        for (int r = 0; r < C; ++r) {
            ms_combine(M0, Ssum0, S.ms_recv[r][0][0], S.ms_recv[r][0][1]);
            if (pair) ms_combine(M1, Ssum1, S.ms_recv[r][1][0], S.ms_recv[r][1][1]);
        }
    }
    bool err = bad;
    if (M0 != M0 || M0 == POS_INF || M0 == NEG_INF) err = true;
    if (pair && (M1 != M1 || M1 == POS_INF || M1 == NEG_INF)) err = true;
    if (!topk && (Ssum0 != Ssum0 || (pair && Ssum1 != Ssum1))) err = true;

    auto write_code = [&](int code) {
        if (sample) {
            P.out_codes[unit] = code < 0 ? -1 : code;
        } else {
            P.out_codes[unit] = code;
        }
    };
    auto write_pq = [&](float p, float q) {
        if (!pair) return;
        if (P.out_p) P.out_p[b * k + i] = p;
        if (P.out_q) P.out_q[b * k + i] = q;
    };

    if (anytmo || err) {
        if (rank == 0 && tid == 0) {
            write_code(anytmo ? CODE_TIMEOUT : CODE_ROW_ERR);
            write_pq(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
        }
        if (tmo && tid == 0) {
            for (int p = 0; p < g0.npieces; ++p) mbar_wait_bounded(&S.mbar[0][p], 0u, P.timeout_ns);
            for (int p = 0; p < g1.npieces; ++p) mbar_wait_bounded(&S.mbar[1][p], 0u, P.timeout_ns);
        }
        return;
    }

    const int K = P.top_k;
    float tau0 = NEG_INF, tau1 = NEG_INF;
    bool need_radix = topk && !P.use_cand;

    // =====================================================================
    // Top-k, candidate path.
    // =====================================================================
    if (topk && P.use_cand) {
        // beta = K-th largest group maximum (with multiplicity) of each row
        for (int t = tid; t < nrows * Gt; t += NT) {
            const int r = t / Gt;
            const int j = t - r * Gt;
            const float x = S.g_recv[r][j];
            int gt = 0, ge = 0;
            for (int q = 0; q < Gt; ++q) {
                const float y = S.g_recv[r][q];
                gt += (y > x);
                ge += (y >= x);
            }
            if (gt < K && K <= ge) S.beta[r] = x;
        }
        __syncthreads();
        // pass 2: every element >= beta goes to the leader
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            if (r >= nrows) break;
            const Geom& g = r ? g1 : g0;
            const unsigned char* buf = r ? buf1 : buf0;
            const float beta = S.beta[r];
            for (int j = tid; j < g.nvec; j += NT) {
                const uint4 raw = *reinterpret_cast<const uint4*>(buf + 16 * j);
                const int e = g.e0 + j * VEC;
                // a ragged vector holds bytes outside the slice: test it element by element
                const bool full = e >= lo && e + VEC <= hi;
                if (!full || vmax_nan<DT>(raw) >= beta) {
                    float v[VEC];
                    unpack<DT>(raw, v);
#pragma unroll
                    for (int t = 0; t < VEC; ++t) {
                        if (valid(e + t) && v[t] >= beta) {
                            atomicAdd(&S.cnt_local[r], 1);
                            const int slot = atom_add_cluster_s32(mapa(&S.cand_n[r], 0), 1);
                            if (slot < CAND_CAP) {
                                st_cluster_f32(mapa(&S.u.cand.v[r][slot], 0), v[t]);
                                st_cluster_s32(mapa(&S.u.cand.i[r][slot], 0), e + t);
                            }
                        }
                    }
                }
            }
        }
        __syncthreads();
        if (tid == 0) {
            for (int peer = 0; peer < C; ++peer) {
                st_cluster_s32(mapa(&S.cnt_recv[rank][0], peer), S.cnt_local[0]);
                st_cluster_s32(mapa(&S.cnt_recv[rank][1], peer), S.cnt_local[1]);
            }
        }
        cluster_sync_all();  // sync #2
        int n0 = 0, n1 = 0;
        for (int r = 0; r < C; ++r) {
            n0 += S.cnt_recv[r][0];
            n1 += S.cnt_recv[r][1];
        }
        if (!pair) n1 = 0;
        if (n0 <= CAND_CAP && n1 <= CAND_CAP) {
            if (rank != 0) return;
            // ---------------- leader: exact tau, softmax, decision, draw ----------------
            for (int t = tid; t < nrows * CAND_CAP; t += NT) {
                const int r = t / CAND_CAP;
                const int j = t - r * CAND_CAP;
                const int n = r ? n1 : n0;
                if (j >= n) continue;
                const float x = S.u.cand.v[r][j];
                int gt = 0, ge = 0;
                for (int q = 0; q < n; ++q) {
                    const float y = S.u.cand.v[r][q];
                    gt += (y > x);
                    ge += (y >= x);
                }
                if (gt < K && K <= ge) S.tau[r] = x;
            }
            __syncthreads();
            for (int t = tid; t < nrows * CAND_CAP; t += NT) {
                const int r = t / CAND_CAP;
                const int j = t - r * CAND_CAP;
                const int n = r ? n1 : n0;
                if (j >= n) continue;
                const float tau = S.tau[r];
                const float x = S.u.cand.v[r][j];
                if (!(x >= tau)) continue;
                const int my = S.u.cand.i[r][j];
                int pos = 0;
                for (int q = 0; q < n; ++q) pos += (S.u.cand.v[r][q] >= tau && S.u.cand.i[r][q] < my);
                S.u.cand.sidx[r][pos] = my;
                S.u.cand.sval[r][pos] = x;
                atomicAdd(&S.nk[r], 1);
            }
            __syncthreads();
            if (warp < nrows) {
                const int r = warp;
                const float m = (r ? M1 : M0) * c;
                float acc = 0.f;
                for (int j = lane; j < S.nk[r]; j += 32) {
                    const float e = ex2(fmaf(S.u.cand.sval[r][j], c, -m));
                    S.u.cand.se[r][j] = e;
                    acc += e;
                }
                acc = warp_sum(acc);
                if (lane == 0) S.ssum[r] = acc;
            }
            __syncthreads();
            if (warp != 0) return;
            const int nk0 = S.nk[0], nk1 = pair ? S.nk[1] : 0;
            const float invS0 = 1.f / S.ssum[0];
            const float invS1 = pair ? 1.f / S.ssum[1] : 0.f;
            auto find = [&](int r, int nk, int v) {  // position of index v in row r's kept list, or -1
                int a = 0, z = nk - 1;
                while (a <= z) {
                    const int mid = (a + z) >> 1;
                    const int x = S.u.cand.sidx[r][mid];
                    if (x == v) return mid;
                    if (x < v) a = mid + 1; else z = mid - 1;
                }
                return -1;
            };
            bool accept = false;
            if (pair) {
                const int pt = find(0, nk0, d), pd = find(1, nk1, d);
                const float p = pt >= 0 ? S.u.cand.se[0][pt] * invS0 : 0.f;
                const float q = pd >= 0 ? S.u.cand.se[1][pd] * invS1 : 0.f;
                accept = u_acc * q < p;
                if (lane == 0) write_pq(p, q);
            }
            if (pair && accept) {
                if (lane == 0) write_code(CODE_ACCEPT);
                return;
            }
            // residual max(0, p - q) over the target's kept entries (bonus: p)
            bool use_q = pair;
            auto weight = [&](int j) {
                const float pt = S.u.cand.se[0][j] * invS0;
                if (!use_q) return pt;
                const int pd = find(1, nk1, S.u.cand.sidx[0][j]);
                const float q = pd >= 0 ? S.u.cand.se[1][pd] * invS1 : 0.f;
                return fmaxf(pt - q, 0.f);
            };
            float W = 0.f;
            for (int attempt = 0; attempt < 2; ++attempt) {
                W = 0.f;
                for (int base = 0; base < nk0; base += 32) {
                    const float w = (base + lane < nk0) ? weight(base + lane) : 0.f;
                    const float incl = warp_incl_scan(w, lane);
                    W += __shfl_sync(0xffffffffu, incl, 31);
                }
                if (W > 0.f || !use_q) break;
                use_q = false;  // zero residual mass: redraw from p
            }
            const float x = u_fin * W;
            float carry = 0.f;
            int token = -1;
            for (int base = 0; base < nk0; base += 32) {
                const float w = (base + lane < nk0) ? weight(base + lane) : 0.f;
                const float incl = warp_incl_scan(w, lane);
                const unsigned hit = __ballot_sync(0xffffffffu, base + lane < nk0 && carry + incl > x);
                if (hit) {
                    token = S.u.cand.sidx[0][base + __ffs(hit) - 1];
                    break;
                }
                carry += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (token < 0) {  // rounding: the last entry with positive weight
                int last = -1;
                for (int base = 0; base < nk0; base += 32) {
                    const float w = (base + lane < nk0) ? weight(base + lane) : 0.f;
                    const unsigned pos = __ballot_sync(0xffffffffu, w > 0.f);
                    if (pos) last = base + 31 - __clz(pos);
                }
                token = last >= 0 ? S.u.cand.sidx[0][last] : -1;
            }
            if (lane == 0) write_code(token >= 0 ? token : CODE_ROW_ERR);
            return;
        }
        need_radix = true;  // too many candidates (ties): exact radix select
    }

    // =====================================================================
    // Top-k, radix select over the resident slices.
    // =====================================================================
    if (need_radix) {
        constexpr int ROUNDS = (DT == 0) ? 2 : 4;
        for (int round = 0; round < ROUNDS; ++round) {
            const int shift = 24 - 8 * round;
            for (int t = tid; t < 2 * 256; t += NT) S.u.radix.hist[t >> 8][t & 255] = 0;
            __syncthreads();
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                if (r >= nrows) break;
                const Geom& g = r ? g1 : g0;
                const unsigned char* buf = r ? buf1 : buf0;
                const uint32_t pre = S.rprefix[r];
                for (int j = tid; j < g.nvec; j += NT) {
                    const uint4 raw = *reinterpret_cast<const uint4*>(buf + 16 * j);
                    float v[VEC];
                    unpack<DT>(raw, v);
                    const int e = g.e0 + j * VEC;
#pragma unroll
                    for (int t = 0; t < VEC; ++t) {
                        if (!valid(e + t)) continue;
                        const uint32_t key = okey(v[t]);
                        if (round == 0 || (key >> (shift + 8)) == pre)
                            atomicAdd(&S.u.radix.hist[r][(key >> shift) & 255u], 1);
                    }
                }
            }
            __syncthreads();
            cluster_sync_all();  // every CTA's histogram is complete
            for (int t = tid; t < nrows * 256; t += NT) {
                const int r = t >> 8, bin = t & 255;
                int sum = 0;
                for (int peer = 0; peer < C; ++peer) sum += ld_cluster_s32(mapa(&S.u.radix.hist[r][bin], peer));
                S.u.radix.tot[r][bin] = sum;
            }
            __syncthreads();
            if (tid < nrows) {
                const int r = tid;
                int kr = S.rk[r], cum = 0, digit = 0;
                for (int bin = 255; bin >= 0; --bin) {
                    const int cnt = S.u.radix.tot[r][bin];
                    if (cum + cnt >= kr) {
                        digit = bin;
                        kr -= cum;
                        break;
                    }
                    cum += cnt;
                }
                S.rprefix[r] = (S.rprefix[r] << 8) | static_cast<uint32_t>(digit);
                S.rk[r] = kr;
            }
            __syncthreads();
            cluster_sync_all();  // nobody reads a peer's histogram any more
        }
        if constexpr (DT == 0) {
            tau0 = okey_inv(S.rprefix[0] << 16 | ((S.rprefix[0] & 0x8000u) ? 0u : 0xffffu));
            tau1 = okey_inv(S.rprefix[1] << 16 | ((S.rprefix[1] & 0x8000u) ? 0u : 0xffffu));
        } else {
            tau0 = okey_inv(S.rprefix[0]);
            tau1 = okey_inv(S.rprefix[1]);
        }
        // masked exp-sums
        const float m0 = M0 * c, m1 = M1 * c;
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            if (r >= nrows) break;
            const Geom& g = r ? g1 : g0;
            const unsigned char* buf = r ? buf1 : buf0;
            const float tau = r ? tau1 : tau0;
            const float m = r ? m1 : m0;
            float acc = 0.f;
            for (int j = tid; j < g.nvec; j += NT) {
                const uint4 raw = *reinterpret_cast<const uint4*>(buf + 16 * j);
                float v[VEC];
                unpack<DT>(raw, v);
                const int e = g.e0 + j * VEC;
#pragma unroll
                for (int t = 0; t < VEC; ++t)
                    if (valid(e + t) && v[t] >= tau) acc += ex2(fmaf(v[t], c, -m));
            }
            if (r) a1 = acc; else a0 = acc;
        }
        a0 = warp_sum(a0);
        a1 = warp_sum(a1);
        if (lane == 0) {
            S.red_f[warp][0] = a0;
            S.red_f[warp][1] = a1;
        }
        __syncthreads();
        if (tid == 0) {
            float s0 = 0.f, s1 = 0.f;
            for (int w = 0; w < NW; ++w) {
                s0 += S.red_f[w][0];
                s1 += S.red_f[w][1];
            }
            for (int peer = 0; peer < C; ++peer) {
                st_cluster_f32(mapa(&S.s_recv[rank][0], peer), s0);
                st_cluster_f32(mapa(&S.s_recv[rank][1], peer), s1);
            }
        }
        cluster_sync_all();
        for (int r = 0; r < C; ++r) {
            Ssum0 += S.s_recv[r][0];
            Ssum1 += S.s_recv[r][1];
        }
        M0 = m0;  // from here on M holds the scaled maximum, as without top-k
        M1 = m1;
    }

    // =====================================================================
    // General path (no top-k, or radix-selected tau): decision and draw.
    // M0/M1 are scaled maxima, Ssum0/Ssum1 the (masked) sums.
    // =====================================================================
    const float invS0 = 1.f / Ssum0;
    const float invS1 = pair ? 1.f / Ssum1 : 0.f;
    bool accept = false;
    if (pair) {
        const float zt = S.z_recv[0], zd = S.z_recv[1];
        const float p = (zt >= tau0) ? ex2(fmaf(zt, c, -M0)) * invS0 : 0.f;
        const float q = (zd >= tau1) ? ex2(fmaf(zd, c, -M1)) * invS1 : 0.f;
        accept = u_acc * q < p;
        if (rank == 0 && tid == 0) write_pq(p, q);
    }
    if (pair && accept) {
        if (rank == 0 && tid == 0) write_code(CODE_ACCEPT);
        return;
    }

    // ---- residual (pair) or target (bonus / sampler) draw over the slices ------
    const bool same_grid = !pair || (g0.e0 == g1.e0);
    bool use_q = pair;
    auto wt = [&](float zt, float zd) {
        const float pt = (zt >= tau0) ? ex2(fmaf(zt, c, -M0)) * invS0 : 0.f;
        if (!use_q) return pt;
        const float qd = (zd >= tau1) ? ex2(fmaf(zd, c, -M1)) * invS1 : 0.f;
        return fmaxf(pt - qd, 0.f);
    };
    // weights of vector j of the target buffer (elements e0 + j*VEC + t)
    auto vec_weights = [&](int j, float* w) {
        const uint4 rt = *reinterpret_cast<const uint4*>(buf0 + 16 * j);
        float vt[VEC], vd[VEC];
        unpack<DT>(rt, vt);
        const int e = g0.e0 + j * VEC;
        if (use_q) {
            if (same_grid) {
                const uint4 rd = *reinterpret_cast<const uint4*>(buf1 + 16 * j);
                unpack<DT>(rd, vd);
            } else {
#pragma unroll
                for (int t = 0; t < VEC; ++t) vd[t] = valid(e + t) ? load_elem<DT>(buf1, e + t - g1.e0) : 0.f;
            }
        } else {
#pragma unroll
            for (int t = 0; t < VEC; ++t) vd[t] = 0.f;
        }
#pragma unroll
        for (int t = 0; t < VEC; ++t) w[t] = valid(e + t) ? wt(vt[t], vd[t]) : 0.f;
    };
    const int nvec = g0.nvec;
    const int ntiles = (nvec + NT - 1) / NT;
    float Wtot = 0.f;
    int attempt = 0;
    for (; attempt < 2; ++attempt) {
        for (int tile = 0; tile < ntiles; ++tile) {
            const int j = tile * NT + tid;
            float s = 0.f;
            if (j < nvec) {
                float w[VEC];
                vec_weights(j, w);
#pragma unroll
                for (int t = 0; t < VEC; ++t) s += w[t];
            }
            s = warp_sum(s);
            if (lane == 0) S.u.tiles.part[tile][warp] = s;
        }
        __syncthreads();
        if (tid < ntiles) {
            float a = 0.f;
            for (int w = 0; w < NW; ++w) a += S.u.tiles.part[tid][w];
            S.u.tiles.sum[tid] = a;
        }
        __syncthreads();
        if (tid == 0) {
            float a = 0.f;
            for (int t = 0; t < ntiles; ++t) a += S.u.tiles.sum[t];
            for (int peer = 0; peer < C; ++peer) st_cluster_f32(mapa(&S.w_recv[attempt][rank], peer), a);
        }
        cluster_sync_all();
        Wtot = 0.f;
        for (int r = 0; r < C; ++r) Wtot += S.w_recv[attempt][r];
        if (Wtot > 0.f || !use_q) break;
        use_q = false;  // zero residual mass: redraw from p at this position
    }
    // locate the CTA whose mass interval holds x = u * W
    const float x = u_fin * Wtot;
    int owner = -1;
    bool last_mode = false;
    {
        float O = 0.f;
        for (int r = 0; r < C; ++r) {
            const float nxt = O + S.w_recv[attempt][r];
            if (O <= x && x < nxt) {
                owner = r;
                break;
            }
            O = nxt;
        }
        if (owner < 0) {  // rounding put x at or past the total: last positive entry
            last_mode = true;
            for (int r = C - 1; r >= 0; --r)
                if (S.w_recv[attempt][r] > 0.f) {
                    owner = r;
                    break;
                }
        }
    }
    if (owner < 0) {  // no mass anywhere (cannot happen for a finite row): report the row
        if (rank == 0 && tid == 0) write_code(CODE_ROW_ERR);
        return;
    }
    if (owner != static_cast<int>(rank)) return;
    float base = 0.f;
    for (int r = 0; r < static_cast<int>(rank); ++r) base += S.w_recv[attempt][r];
    int tile = -1;
    if (!last_mode) {
        float a = base;
        for (int t = 0; t < ntiles; ++t) {
            const float nxt = a + S.u.tiles.sum[t];
            if (nxt > x) {
                tile = t;
                base = a;
                break;
            }
            a = nxt;
        }
    }
    if (tile < 0) {
        last_mode = true;
        for (int t = ntiles - 1; t >= 0; --t)
            if (S.u.tiles.sum[t] > 0.f) {
                tile = t;
                break;
            }
    }
    if (tid == 0) {
        S.sh_i[0] = -1;
        S.sh_i[1] = -1;
    }
    __syncthreads();
    {
        const int j = tile * NT + tid;
        float w[VEC];
        float vs = 0.f;
        if (tile >= 0 && j < nvec) {
            vec_weights(j, w);
#pragma unroll
            for (int t = 0; t < VEC; ++t) vs += w[t];
        } else {
#pragma unroll
            for (int t = 0; t < VEC; ++t) w[t] = 0.f;
        }
        // last positive element of this thread's vector
        int lastpos = -1;
#pragma unroll
        for (int t = 0; t < VEC; ++t)
            if (w[t] > 0.f) lastpos = g0.e0 + j * VEC + t;
        if (lastpos >= 0) atomicMax(&S.sh_i[1], lastpos);
        const float inw = warp_incl_scan(vs, lane);
        float exw = __shfl_up_sync(0xffffffffu, inw, 1);
        if (lane == 0) exw = 0.f;
        if (lane == 31) S.red_f[warp][0] = inw;
        __syncthreads();
        if (tid == 0) {
            float a = 0.f;
            for (int w2 = 0; w2 < NW; ++w2) {
                S.red_f[w2][1] = a;
                a += S.red_f[w2][0];
            }
        }
        __syncthreads();
        if (!last_mode) {
            const float wp = S.red_f[warp][1];
            const float incl = base + (wp + inw);
            const float excl = base + (wp + exw);
            if (excl <= x && x < incl) {
                float acc = excl;
                int tok = -1;
#pragma unroll
                for (int t = 0; t < VEC; ++t) {
                    if (tok < 0 && w[t] > 0.f) {
                        const float nacc = acc + w[t];
                        if (nacc > x) tok = g0.e0 + j * VEC + t;
                        acc = nacc;
                    }
                }
                if (tok < 0) tok = lastpos;
                S.sh_i[0] = tok;
            }
        }
        __syncthreads();
        if (tid == 0) {
            const int tok = S.sh_i[0] >= 0 ? S.sh_i[0] : S.sh_i[1];
            write_code(tok >= 0 ? tok : CODE_ROW_ERR);
        }
    }
}

// ---------------------------------------------------------------------------
// Finalise: turn the per-position codes of each sequence into the result.
// ---------------------------------------------------------------------------
__global__ void sv_finalize_kernel(int32_t* __restrict__ tokens, const int32_t* __restrict__ draft_tokens,
                                   int32_t* __restrict__ n_accepted, int32_t* __restrict__ status,
                                   long long B, int k) {
    pdl_wait_primary();
    const long long b = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
    if (b >= B) return;
    int32_t* c = tokens + b * (k + 1);
    bool err = false, tmo = false;
    for (int t = 0; t <= k; ++t) {
        const int v = c[t];
        if (v == CODE_TIMEOUT) tmo = true;
        if (v <= CODE_ROW_ERR) err = true;
    }
    int j = k;
    if (!err) {
        for (int t = 0; t < k; ++t) {
            if (c[t] != CODE_ACCEPT) {
                j = t;
                break;
            }
        }
        if (c[j] < 0) err = true;
    }
    if (err) {
        for (int t = 0; t <= k; ++t) c[t] = -1;
        n_accepted[b] = -1;
    } else {
        const int y = c[j];
        for (int t = 0; t < j; ++t) c[t] = draft_tokens[b * k + t];
        c[j] = y;
        for (int t = j + 1; t <= k; ++t) c[t] = -1;
        n_accepted[b] = j;
    }
    if (tmo && status) atomicExch(status, -4);
}

}  // namespace sv
