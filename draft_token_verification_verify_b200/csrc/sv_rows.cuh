// K1 — the streaming pass over every logit row of a verification batch.
//
// One CTA per task = one chunk (a run of consecutive segments) of one row.
// The chunk streams through a ring of shared-memory stages filled by bulk
// copies (cp.async.bulk, no multicast) that complete on mbarriers; every
// wait is bounded in time.  The refill of a stage is issued as soon as every
// thread has finished reading it; nothing else sits between a stage's
// consumption and its refill.  Each segment (one stage) leaves a 16-byte
// partial in the workspace, written at the end of the chunk:
//   greedy   raw maximum and its lowest index,
//   softmax  online (max, sum of 2^(z*c - max)) with c = log2(e)/T,
//   top-k    raw maximum.
// With top-k the chunk also keeps, in the same single pass, every element
// that can belong to the top-k set: a running lower bound theta on the
// chunk's K-th largest logit (the K-th largest of the groups' running maxima:
// K distinct elements are >= it) filters the stream into a shared candidate
// list.  At the end the exact K-th largest tau_c of the chunk and every
// element >= tau_c are stored sorted by index, with the chunk maximum, the
// sum of 2^(z*c - max*c) over the stored entries and the logit at the row's
// draft token when it is among them.
// Rows are read from HBM exactly once; no CTA waits for another.
#pragma once

#include <climits>

#include "sv_common.cuh"

namespace sv {

constexpr int MAX_STAGES = 8;
constexpr int MAX_TILES_K1 = 64; // segments per chunk
constexpr int RANK_MAX = 256;    // lists up to this size are ranked, larger ones sorted
constexpr int TILE_BYTES = 16384; // bytes per segment (one ring stage)

struct RowsParams {
    const void* target;          // [B][k+1][V] (sampler: [rows][V])
    const void* draft;           // [B][k][V] or null
    const int32_t* draft_tokens; // [B][k] or null
    long long B;                 // sequences (sampler: rows)
    int k;                       // draft length (sampler: 0)
    int V;
    int mode;                    // MODE_*
    int top_k;                   // effective K (MODE_TOPK)
    const float* temperature;    // [B] or null
    int seg;                     // elements per segment (TILE_BYTES / element size)
    int nseg;                    // segments per row
    int spc;                     // segments per chunk (<= MAX_TILES_K1)
    int nch;                     // chunks per row
    int stages;                  // ring stages (<= MAX_STAGES)
    int stage_bytes;             // shared bytes per stage
    int lcap;                    // shared candidate list capacity (power of two)
    int kcap;                    // stored kept entries per chunk
    SegRec* segs;                // [R][nseg]
    ChunkRec* chunks;            // [R][nch]
    Cand* cands;                 // [R][nch][kcap]
    int32_t* out_status;         // reset to 0 by CTA 0 (or null)
    unsigned long long timeout_ns;
    unsigned int test_extra_tx;
};

struct __align__(16) RowsCtl {
    uint64_t mbar[MAX_STAGES];
    float theta;
    float theta_new;
    int cnt;
    int cnt2;
    int overflow;
    int nkept;
    float tau;
    float wsum[16];
    float wzd[16];
    float wsel[3][16];  // per-warp bound candidates: two tile slots and the final
};

constexpr int ROWS_CTL_BYTES = (int)((sizeof(RowsCtl) + 127) / 128 * 128);

// Geometry of one segment in the ring: the stage mirrors the 16-byte aligned
// global span [A0, A0 + 16*nvec) covering elements [lo, hi).
struct TileGeom {
    uintptr_t A0, ga, gb, ga16, gb16;
    int lo, hi, e0, nvec;
};

template <int ELT>
__device__ __forceinline__ TileGeom tile_geom(const char* row, int lo, int hi) {
    TileGeom g;
    g.lo = lo;
    g.hi = hi;
    g.ga = reinterpret_cast<uintptr_t>(row) + static_cast<uintptr_t>(lo) * ELT;
    g.gb = reinterpret_cast<uintptr_t>(row) + static_cast<uintptr_t>(hi) * ELT;
    g.A0 = g.ga & ~static_cast<uintptr_t>(15);
    const uintptr_t A1 = (g.gb + 15) & ~static_cast<uintptr_t>(15);
    g.ga16 = (g.ga + 15) & ~static_cast<uintptr_t>(15);
    g.gb16 = g.gb & ~static_cast<uintptr_t>(15);
    g.e0 = lo - static_cast<int>((g.ga - g.A0) / ELT);
    g.nvec = (hi > lo) ? static_cast<int>((A1 - g.A0) / 16) : 0;
    return g;
}

template <int DT, int NT, int MODE>
__global__ void __launch_bounds__(NT, 1024 / NT) sv_rows_kernel(const RowsParams P) {
    constexpr int ELT = VT<DT>::ELT;
    constexpr int VEC = VT<DT>::VEC;
    constexpr int NW = NT / 32;
    constexpr int TV = TILE_BYTES / 16;  // vectors per tile
    constexpr int VPT = TV / NT;         // vectors per thread per tile
    static_assert(VPT * NT == TV, "tile must split evenly over the threads");
    extern __shared__ __align__(128) unsigned char smem[];
    RowsCtl& S = *reinterpret_cast<RowsCtl*>(smem);
    unsigned char* const ring = smem + ROWS_CTL_BYTES;
    float* const red_m = reinterpret_cast<float*>(ring + static_cast<size_t>(P.stages) * P.stage_bytes);
    float* const red_s = red_m + MAX_TILES_K1 * NW;
    int* const red_i = reinterpret_cast<int*>(red_s + MAX_TILES_K1 * NW);
    float* const lkey = reinterpret_cast<float*>(red_i + MAX_TILES_K1 * NW);
    int* const lidx = reinterpret_cast<int*>(lkey + P.lcap);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long task = blockIdx.x;
    const long long r = task / P.nch;
    const int c = static_cast<int>(task - r * P.nch);
    const long long Rt = P.B * (P.k + 1);
    const char* row;
    long long b;
    int pos;  // position of the row within its sequence
    if (r < Rt) {
        row = static_cast<const char*>(P.target) + static_cast<size_t>(r) * P.V * ELT;
        b = r / (P.k + 1);
        pos = static_cast<int>(r - b * (P.k + 1));
    } else {
        row = static_cast<const char*>(P.draft) + static_cast<size_t>(r - Rt) * P.V * ELT;
        b = (r - Rt) / P.k;
        pos = static_cast<int>((r - Rt) - b * P.k);
    }
    if (task == 0 && tid == 0 && P.out_status) *P.out_status = 0;
    pdl_launch_dependents();

    float cscale = 1.f;  // log2(e) / T
    if constexpr (MODE == MODE_SOFTMAX || MODE == MODE_TOPK) {
        const float T = P.temperature ? P.temperature[b] : 1.f;
        if (T > 0.f && T != POS_INF) cscale = LOG2E / T;
    }
    constexpr int SEG = TILE_BYTES / ELT;  // elements per segment
    const int s0 = c * P.spc;
    const int ntiles = min(P.spc, P.nseg - s0);
    const int K = P.top_k;

    auto geom = [&](int t) {
        const int lo = (s0 + t) * SEG;
        const int hi = min(P.V, lo + SEG);
        return tile_geom<ELT>(row, lo, hi);
    };
    // producer: fill stage (t % stages) with tile t
    auto issue = [&](int t) {
        const int st = t % P.stages;
        const TileGeom g = geom(t);
        unsigned char* buf = ring + static_cast<size_t>(st) * P.stage_bytes;
        uint32_t bytes = 0;
        if (g.hi > g.lo) {
            int nh, ntl;
            if (g.ga16 >= g.gb16) {
                nh = g.hi - g.lo;
                ntl = 0;
            } else {
                nh = static_cast<int>((g.ga16 - g.ga) / ELT);
                ntl = static_cast<int>((g.gb - g.gb16) / ELT);
                bytes = static_cast<uint32_t>(g.gb16 - g.ga16);
            }
            // elements outside the aligned interior: plain loads before the arrive
            for (int q = 0; q < nh + ntl; ++q) {
                const int e = q < nh ? g.lo + q : g.hi - ntl + (q - nh);
                if constexpr (DT == 0)
                    reinterpret_cast<uint16_t*>(buf)[e - g.e0] = reinterpret_cast<const uint16_t*>(row)[e];
                else
                    reinterpret_cast<float*>(buf)[e - g.e0] = reinterpret_cast<const float*>(row)[e];
            }
        }
        mbar_arrive_expect_tx(&S.mbar[st], bytes + P.test_extra_tx);
        if (bytes) bulk_g2s(buf + (g.ga16 - g.A0), reinterpret_cast<const void*>(g.ga16), bytes, &S.mbar[st]);
    };

    if (tid == 0) {
        for (int st = 0; st < P.stages; ++st) mbar_init(&S.mbar[st], 1);
        fence_mbar_init();
        S.theta = NEG_INF;
        S.cnt = 0;
        S.overflow = 0;
    }
    __syncthreads();
    if (tid == 0) {
        for (int t = 0; t < min(P.stages, ntiles); ++t) issue(t);
    }

    float run = NEG_INF;     // running NaN-propagating maximum of this thread's elements
    float wbest = NEG_INF;   // greedy: best value of this warp and its lowest index
    int widx = -1;
    // top-k bound.  Each warp sorts its lanes' running maxima (bitonic network
    // in registers) and takes the rsel-th largest, rsel = ceil(K / warps): that
    // warp holds rsel distinct elements at or above it, so the minimum over the
    // warps has at least K elements at or above it and is <= the chunk's K-th
    // largest logit.
    const int rsel = (K + NW - 1) / NW;  // <= 32 (K <= threads on this path)
    auto warp_bound = [&]() -> float {
        float x = run == run ? run : NEG_INF;
#pragma unroll
        for (int k2 = 2; k2 <= 32; k2 <<= 1) {
#pragma unroll
            for (int j2 = k2 >> 1; j2 > 0; j2 >>= 1) {
                const float y = __shfl_xor_sync(0xffffffffu, x, j2);
                const bool desc = (lane & k2) == 0;
                const bool lower = (lane & j2) == 0;
                x = (lower == desc) ? fmaxf(x, y) : fminf(x, y);
            }
        }
        return __shfl_sync(0xffffffffu, x, rsel - 1);
    };
    auto min_bound = [&](int slot) {
        float mn = S.wsel[slot][0];
        for (int w = 1; w < NW; ++w) mn = fminf(mn, S.wsel[slot][w]);
        return mn;
    };
    float theta = NEG_INF;  // this thread's copy of the running bound

    int tmo = 0;
    int t = 0;
    for (; t < ntiles; ++t) {
        const int st = t % P.stages;
        const uint32_t parity = static_cast<uint32_t>((t / P.stages) & 1);
        const TileGeom g = geom(t);
        const unsigned char* buf = ring + static_cast<size_t>(st) * P.stage_bytes;
        const bool ok = mbar_wait_bounded(&S.mbar[st], parity, P.timeout_ns);
        auto valid = [&](int e) { return e >= g.lo && e < g.hi; };
        auto vec_at = [&](int j) { return *reinterpret_cast<const uint4*>(buf + 16 * j); };
        // NaN-propagating maximum of the valid elements of vector j
        auto vmax_masked = [&](int j) -> float {
            const uint4 raw = vec_at(j);
            const int e = g.e0 + j * VEC;
            if (e >= g.lo && e + VEC <= g.hi) return vmax_nan<DT>(raw);
            float v[VEC];
            unpack<DT>(raw, v);
            float vm = NEG_INF;
#pragma unroll
            for (int q = 0; q < VEC; ++q)
                if (valid(e + q)) vm = fmax_nan(vm, v[q]);
            return vm;
        };
        // valid elements of vector j (others -inf)
        auto load_masked = [&](int j, float* v) {
            unpack<DT>(vec_at(j), v);
            const int e = g.e0 + j * VEC;
            if (!(e >= g.lo && e + VEC <= g.hi)) {
#pragma unroll
                for (int q = 0; q < VEC; ++q)
                    if (!valid(e + q)) v[q] = NEG_INF;
            }
        };

        // pass A (no stores): every vector maximum of this thread's share of the
        // tile.  Slot VPT is the one vector past TV that a segment starting off
        // a 16-byte boundary spans (vector TV + tid, present for tid == 0 only).
        auto jof = [&](int i) { return i < VPT ? tid + i * NT : TV + tid; };
        float vm[VPT + 1];
        const bool tile_full = ok && g.e0 == g.lo && g.nvec == TV && g.hi - g.lo == TV * VEC;
        if (tile_full) {
#pragma unroll
            for (int i = 0; i < VPT; ++i) vm[i] = vmax_nan<DT>(vec_at(tid + i * NT));
            vm[VPT] = NEG_INF;
        } else {
#pragma unroll
            for (int i = 0; i <= VPT; ++i) {
                const int j = jof(i);
                vm[i] = (ok && j < g.nvec) ? vmax_masked(j) : NEG_INF;
            }
        }
        float tm = vm[0];
#pragma unroll
        for (int i = 1; i <= VPT; ++i) tm = fmax_nan(tm, vm[i]);

        if constexpr (MODE == MODE_GREEDY) {
            run = fmax_nan(run, tm);
            float wtm = tm != tm ? NEG_INF : tm;  // NaN is reported through run
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) wtm = fmaxf(wtm, __shfl_xor_sync(0xffffffffu, wtm, o));
            if (wtm > wbest) {  // warp-uniform, rare after the first tiles
                int my = INT_MAX;
#pragma unroll
                for (int i = 0; i <= VPT; ++i) {
                    const int j = jof(i);
                    if (my == INT_MAX && vm[i] == wtm) {
                        float v[VEC];
                        load_masked(j, v);
                        const int e = g.e0 + j * VEC;
#pragma unroll
                        for (int q = VEC - 1; q >= 0; --q)
                            if (v[q] == wtm) my = e + q;
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) my = min(my, __shfl_xor_sync(0xffffffffu, my, o));
                wbest = wtm;
                widx = my;
            }
        } else if constexpr (MODE == MODE_SOFTMAX) {
            // one maximum per warp; pass B sums 2^(z*c - m) with two accumulators
            float wtm = tm;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) wtm = fmax_nan(wtm, __shfl_xor_sync(0xffffffffu, wtm, o));
            const float m = wtm * cscale;
            float s0 = 0.f, s1 = 0.f;
            if (ok && m > NEG_INF && m < POS_INF) {
#pragma unroll
                for (int i = 0; i <= VPT; ++i) {
                    const int j = jof(i);
                    if (j < g.nvec) {
                        float v[VEC];
                        load_masked(j, v);
#pragma unroll
                        for (int q = 0; q < VEC; q += 2) {
                            s0 += ex2(fmaf(v[q], cscale, -m));
                            s1 += ex2(fmaf(v[q + 1], cscale, -m));
                        }
                    }
                }
            }
            const float ws = warp_sum(s0 + s1);
            if (lane == 0) {
                red_m[t * NW + warp] = m;
                red_s[t * NW + warp] = ws;
            }
        } else if constexpr (MODE == MODE_TOPK) {
            run = fmax_nan(run, tm);
            if (t == 0) {
                // first tile: a bound from the tile itself before any append
                const float wb = warp_bound();
                if (lane == 0) S.wsel[2][warp] = wb;
                __syncthreads();
                theta = fmaxf(theta, min_bound(2));
            }
            const float th = theta;
            // pass B: the elements >= th, appended warp by warp (rare)
#pragma unroll
            for (int i = 0; i <= VPT; ++i) {
                const bool cand = ok && vm[i] >= th;
                if (__any_sync(0xffffffffu, cand)) {
                    const int j = jof(i);
                    const int e = g.e0 + j * VEC;
                    float v[VEC];
                    unsigned mask = 0u;
                    if (cand) {
                        load_masked(j, v);
#pragma unroll
                        for (int q = 0; q < VEC; ++q)
                            if (v[q] >= th) mask |= 1u << q;
                    }
                    const int cnt = __popc(mask);
                    int incl = cnt;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const int y = __shfl_up_sync(0xffffffffu, incl, o);
                        if (lane >= o) incl += y;
                    }
                    const int total = __shfl_sync(0xffffffffu, incl, 31);
                    int base = 0;
                    if (lane == 0) base = atomicAdd(&S.cnt, total);
                    base = __shfl_sync(0xffffffffu, base, 0);
                    int p = base + incl - cnt;
#pragma unroll
                    for (int q = 0; q < VEC; ++q) {
                        if ((mask >> q) & 1u) {
                            if (p < P.lcap) {
                                lkey[p] = v[q];
                                lidx[p] = e + q;
                            } else {
                                S.overflow = 1;
                            }
                            ++p;
                        }
                    }
                }
            }
            // publish this tile's warp bounds; read after the tile barrier
            const float wb = warp_bound();
            if (lane == 0) S.wsel[t & 1][warp] = wb;
        } else {
            run = fmax_nan(run, tm);  // MODE_MAXONLY
        }

        tmo = __syncthreads_or(!ok);  // every thread is done with the stage
        if (tid == 0 && !tmo && t + P.stages < ntiles) issue(t + P.stages);
        if (tmo) break;
        if constexpr (MODE == MODE_TOPK) theta = fmaxf(theta, min_bound(t & 1));

        if constexpr (MODE == MODE_TOPK) {
            // Compact the candidate list when it is half full (rare).  The
            // decision is taken from a snapshot that every thread reads
            // between two barriers: without the second one a fast warp could
            // append the next tile's candidates before a slow warp reads the
            // count, and the warps would disagree about entering the
            // compaction (and its barriers).
            const int cnt_now = S.cnt;
            const int ovf_now = S.overflow;
            __syncthreads();
            if (cnt_now > (P.lcap >> 1) && !ovf_now) {
                const int n = cnt_now;
                const int N = pow2_ceil(n);
                for (int q = n + tid; q < N; q += NT) {
                    lkey[q] = NEG_INF;
                    lidx[q] = INT_MAX;
                }
                __syncthreads();
                block_sort<true>(lkey, lidx, N);
                const float th2 = fmaxf(theta, lkey[K - 1]);
                __syncthreads();
                if (tid == 0) {
                    int m = K;
                    while (m < n && lkey[m] >= th2) ++m;
                    S.cnt = m;
                }
                theta = th2;
                __syncthreads();
            }
        }
    }

    // ---- partial records ------------------------------------------------------------
    if constexpr (MODE == MODE_SOFTMAX) {
        // one per segment
        for (int q = tid; q < ntiles; q += NT) {
            SegRec rec;
            rec.arg = -1;
            rec.flags = 0;
            if (tmo && q >= t) {  // the tile whose wait ran out, and every later one
                rec.m = __int_as_float(0x7fc00000);
                rec.s = 0.f;
                rec.flags = REC_TIMEOUT;
            } else {
                float m = red_m[q * NW], sm = red_s[q * NW];
                for (int w = 1; w < NW; ++w) ms_combine(m, sm, red_m[q * NW + w], red_s[q * NW + w]);
                rec.m = m;
                rec.s = sm;
            }
            P.segs[r * P.nseg + s0 + q] = rec;
        }
    } else if constexpr (MODE == MODE_GREEDY || MODE == MODE_MAXONLY) {
        // one per chunk, stored in slot c of the row
        run = warp_max_nan(run);
        if (lane == 0) {
            red_m[warp] = run;
            red_s[warp] = wbest;
            red_i[warp] = widx;
        }
        __syncthreads();
        if (tid == 0) {
            SegRec rec;
            rec.m = red_m[0];
            rec.s = 0.f;
            float bv = red_s[0];
            int bi = red_i[0];
            for (int w = 1; w < NW; ++w) {
                rec.m = fmax_nan(rec.m, red_m[w]);
                if (arg_better(red_s[w], red_i[w], bv, bi)) {
                    bv = red_s[w];
                    bi = red_i[w];
                }
            }
            rec.arg = MODE == MODE_GREEDY ? bi : -1;
            rec.flags = tmo ? REC_TIMEOUT : 0;
            if (tmo) rec.m = __int_as_float(0x7fc00000);
            P.segs[r * P.nseg + c] = rec;
        }
    }

    if (tmo) {
        if (tid == 0) {
            if constexpr (MODE == MODE_TOPK) {
                ChunkRec ch;
                ch.tau = NEG_INF;
                ch.last = NEG_INF;
                ch.n = 0;
                ch.flags = REC_TIMEOUT;
                ch.m = __int_as_float(0x7fc00000);
                ch.s = 0.f;
                ch.zd = NEG_INF;
                ch.pad = 0;
                P.chunks[r * P.nch + c] = ch;
            }
            // wait (bounded) for copies still in flight before the CTA exits
            for (int q = t; q < min(ntiles, t + P.stages); ++q)
                mbar_wait_bounded(&S.mbar[q % P.stages], static_cast<uint32_t>((q / P.stages) & 1), P.timeout_ns);
        }
        return;
    }
    if constexpr (MODE != MODE_TOPK) {
        return;
    } else {

    // ---- top-k: exact K-th largest of the chunk and its kept entries ----------
    const float mrow = warp_max_nan(run);  // chunk maximum (NaN-propagating)
    const float wbf = warp_bound();        // final bound from every element
    if (lane == 0) {
        S.wzd[warp] = mrow;
        S.wsel[2][warp] = wbf;
    }
    __syncthreads();
    const float thf = fmaxf(theta, min_bound(2));
    float cmax = S.wzd[0];
    for (int w = 1; w < NW; ++w) cmax = fmax_nan(cmax, S.wzd[w]);
    const int n0 = min(S.cnt, P.lcap);
    const int ovf = S.overflow;
    const int d = (pos < P.k && P.draft_tokens) ? P.draft_tokens[b * P.k + pos] : -1;
    // filtered copy of the list (entries >= the final bound) in the free ring
    Cand* fl = reinterpret_cast<Cand*>(ring);
    const int fcap = (P.stages * P.stage_bytes) / static_cast<int>(sizeof(Cand));
    if (tid == 0) S.cnt2 = 0;
    __syncthreads();
    for (int q = tid; q < n0; q += NT) {
        if (lkey[q] >= thf) {
            const int p = atomicAdd(&S.cnt2, 1);
            if (p < fcap) fl[p] = Cand{lkey[q], lidx[q]};
        }
    }
    if (tid == 0) {
        S.nkept = 0;
        S.tau = NEG_INF;
    }
    __syncthreads();
    const int n2 = S.cnt2;
    Cand* out = P.cands + (r * P.nch + c) * static_cast<long long>(P.kcap);
    float lastv = NEG_INF;
    int nk;
    if (n2 <= RANK_MAX && n2 <= fcap) {
        // rank by (value desc, index asc): tau is the value at rank K-1
        for (int q = tid; q < n2; q += NT) {
            const Cand e = fl[q];
            int rk = 0;
            for (int f = 0; f < n2; ++f) {
                const Cand o = fl[f];
                rk += (o.v > e.v) || (o.v == e.v && o.i < e.i);
            }
            if (rk == K - 1) S.tau = e.v;
        }
        __syncthreads();
        const float tau = n2 >= K ? S.tau : NEG_INF;
        for (int q = tid; q < n2; q += NT) {
            const Cand e = fl[q];
            if (!(e.v >= tau)) continue;
            int ri = 0;
            for (int f = 0; f < n2; ++f) ri += (fl[f].v >= tau && fl[f].i < e.i);
            atomicAdd(&S.nkept, 1);
            if (ri < P.kcap) out[ri] = e;
        }
        __syncthreads();
        nk = S.nkept;
        if (tid == 0) S.tau = tau;
        lastv = tau;  // every kept entry is >= tau
    } else {
        // large lists: sort the unfiltered list by value
        const int N = pow2_ceil(n0 < 2 ? 2 : n0);
        for (int q = n0 + tid; q < N; q += NT) {
            lkey[q] = NEG_INF;
            lidx[q] = INT_MAX;
        }
        __syncthreads();
        block_sort<true>(lkey, lidx, N);
        const float tau = (n0 >= K) ? lkey[K - 1] : NEG_INF;
        for (int q = tid; q < n0; q += NT)
            if (lkey[q] >= tau && (q + 1 == n0 || !(lkey[q + 1] >= tau))) S.nkept = q + 1;
        __syncthreads();
        nk = S.nkept;
        const int m = min(nk, P.kcap);
        lastv = m > 0 ? lkey[m - 1] : NEG_INF;
        const int M2 = pow2_ceil(m < 2 ? 2 : m);
        for (int q = m + tid; q < M2; q += NT) {
            lkey[q] = NEG_INF;
            lidx[q] = INT_MAX;
        }
        __syncthreads();
        block_sort<false>(lkey, lidx, M2);
        for (int q = tid; q < m; q += NT) out[q] = Cand{lkey[q], lidx[q]};
        if (tid == 0) S.tau = tau;
        __syncthreads();
    }
    // maximum, exp-sum and draft-token logit over the stored (index-sorted) entries
    const int m = min(nk, P.kcap);
    __syncthreads();
    const float msc = cmax * cscale;
    float acc = 0.f, zd = NEG_INF;
    for (int q = tid; q < m; q += NT) {
        const Cand e = out[q];
        acc += ex2(fmaf(e.v, cscale, -msc));
        if (e.i == d) zd = e.v;
    }
    acc = warp_sum(acc);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) zd = fmaxf(zd, __shfl_xor_sync(0xffffffffu, zd, o));
    if (lane == 0) {
        S.wsum[warp] = acc;
        S.wzd[warp] = zd;
    }
    __syncthreads();
    if (tid == 0) {
        float s = 0.f, z = NEG_INF;
        for (int w = 0; w < NW; ++w) {
            s += S.wsum[w];
            z = fmaxf(z, S.wzd[w]);
        }
        ChunkRec ch;
        ch.tau = S.tau;
        ch.last = lastv;
        ch.n = m;
        ch.flags = (ovf || nk > P.kcap || n2 > fcap) ? REC_OVERFLOW : 0;
        ch.m = cmax;
        ch.s = s;
        ch.zd = z;
        ch.pad = 0;
        P.chunks[r * P.nch + c] = ch;
    }
    }  // MODE_TOPK
}

}  // namespace sv
