// K1 — the streaming pass over every logit row of a verification batch.
//
// One CTA per task = one chunk (a run of consecutive 16 KB segments) of one
// row, warp-specialised.  Warp NW (the producer) streams the chunk into a
// ring of shared-memory stages with bulk copies (cp.async.bulk, no
// multicast); every stage has a "full" mbarrier (one arrival plus the copy's
// bytes) and an "empty" mbarrier (one arrival per consumer warp).  Warps
// 0..NW-1 (the consumers) work through the tiles independently of each other
// and hand each stage back as soon as they are done with it: no block-wide
// barrier runs per tile.  Every wait is bounded in time.
//
// Partials written to the workspace:
//   greedy   per chunk: raw maximum and its lowest index,
//   softmax  per segment: (max of z*c, sum of 2^(z*c - max)), c = log2(e)/T,
//   max-only per chunk: raw maximum,
//   top-k    per chunk: the exact K-th largest logit tau_c and every element
//            >= tau_c, sorted by index, with the chunk maximum, the sum of
//            2^(z*c - max*c) over them and the logit at the row's draft token.
//            The pass works on 16-byte vectors and their maxima (each maximum
//            is one element, so distinct vectors give distinct elements).
//            Warp w publishes a value b_w such that at least rsel =
//            ceil(K / NW) distinct vectors it has seen have a maximum >= b_w
//            (the rsel-th largest of its lanes' running maxima, or the
//            rsel-th largest key of its own candidate list).  Then at least
//            NW * rsel >= K vector maxima are >= min_w b_w, so that minimum
//            never exceeds the K-th largest vector maximum — whatever mix of
//            older and newer published values a warp reads — and vectors
//            whose maximum reaches it are copied, whole, into the warp's
//            private list in shared memory (one ballot per vector slot, no
//            per-element work).  A consumer hands its stage back as soon as
//            the maxima are taken and the candidates copied; publishing the
//            bounds works on registers only and overlaps the next copy.  At
//            the end the listed vectors are expanded to their elements >= the
//            final bound (the chunk's K-th largest logit is >= it, and every
//            element >= that lies in a listed vector), and the exact
//            threshold and kept entries are taken from those few elements.
// Rows are read from HBM exactly once; no CTA waits for another.
#pragma once

#include <climits>

#include "sv_common.cuh"
#include "sv_procs.cuh"

namespace sv {

constexpr int MAX_STAGES = 8;
constexpr int MAX_TILES_K1 = 64;   // segments per chunk
constexpr int TILE_BYTES = 16384;  // bytes per segment (one ring stage)
constexpr int REC_DIAG = 4;        // a device-side consistency check failed
constexpr int RANK_MAX = 256;      // expanded top-k elements ranked per chunk (more: exact fallback)
constexpr int MAX_CONSUMER_WARPS = 16;
constexpr int TOPK_WCAP = 256;     // candidate vectors per consumer warp (top-k)

struct RowsParams {
    const void* target;          // [B][k+1][V] (sampler: [rows][V])
    const void* draft;           // [B][k][V] or null
    const int32_t* draft_tokens; // [B][k] or null
    long long B;                 // sequences (sampler: rows)
    int k;                       // draft length (sampler: 0)
    int V;
    int top_k;                   // effective K (MODE_TOPK)
    const float* temperature;    // [B] or null
    int nseg;                    // segments per row
    int spc;                     // segments per chunk (<= MAX_TILES_K1)
    int nch;                     // chunks per row
    int stages;                  // ring stages (2..MAX_STAGES)
    int lcap;                    // top-k candidate vectors per CTA (NW segments of TOPK_WCAP)
    int kcap;                    // stored kept entries per chunk (top-k)
    SegRec* segs;                // [R][nseg]
    ChunkRec* chunks;            // [R][nch] (top-k)
    Cand* cands;                 // [R][nch][kcap] (top-k)
    int32_t* out_status;         // reset to 0 by CTA 0 (or null)
    unsigned long long timeout_ns;
    unsigned int test_extra_tx;
    // processors (the PROC variants): per-sequence bitmaps built by K0
    const uint32_t* allow;       // [S][W4]
    const uint32_t* pen;         // [S][W4]
    const float* theta;          // [S] or null
    int W4;
    int procs_div;               // the processors' sequence of row-owner b is b / procs_div
};

struct __align__(16) RowsCtl {
    uint64_t full[MAX_STAGES];
    uint64_t empty[MAX_STAGES];
    int issued;   // tiles the producer issued
    int copied;   // bit q: the last issue into stage q carried a bulk copy
    int tmo;      // a wait ran out
    int rawbad;   // a raw logit is NaN or +inf (processors: the row is an error even if masked)
    int diag;     // a copy failed its self-check (skipped)
    int cnt2;
    int nkept;
    float tau;
    int ne;     // expanded elements (top-k)
    float thf;  // K-th largest candidate-vector maximum (top-k finish)
    float wbound[MAX_CONSUMER_WARPS];  // published per-warp bounds (top-k)
    float wmax[MAX_CONSUMER_WARPS];
    float wbest[MAX_CONSUMER_WARPS];
    int widx[MAX_CONSUMER_WARPS];
    int wcnt[MAX_CONSUMER_WARPS];
    int wovf[MAX_CONSUMER_WARPS];
    float wsum[MAX_CONSUMER_WARPS + 1];
    float wzd[MAX_CONSUMER_WARPS + 1];
};

constexpr int ROWS_CTL_BYTES = (int)((sizeof(RowsCtl) + 127) / 128 * 128);
constexpr int STAGE_BYTES = (TILE_BYTES + 32 + 127) / 128 * 128;  // one segment plus one spare vector
// processors: each stage also holds the segment's allow and penalty bitmap words
constexpr int MASK_STAGE_BYTES = (TILE_BYTES / 2 / 32 * 4 + 32 + 127) / 128 * 128;
constexpr int STAGE_BYTES_PROC = STAGE_BYTES + 2 * MASK_STAGE_BYTES;

// Dynamic shared memory of one streaming CTA.
__host__ __device__ constexpr int rows_tail_bytes(int mode, int nt, int lcap) {
    return (mode == MODE_SOFTMAX ? 2 * MAX_TILES_K1 * (nt / 32) * 4 : 0) + (mode == MODE_TOPK ? lcap * (4 + 4) : 0);
}
__host__ __device__ constexpr int rows_smem_bytes(int mode, int nt, int stages, int lcap, bool proc) {
    // processors: each consumer thread parks its vector maxima of a tile
    return ROWS_CTL_BYTES + stages * (proc ? STAGE_BYTES_PROC : STAGE_BYTES) + rows_tail_bytes(mode, nt, lcap) +
           (proc ? (TILE_BYTES / 16 / nt + 1) * nt * 4 : 0);
}

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

// Element `el` of a ring stage (raw logit as fp32).
template <int DT>
__device__ __forceinline__ float smem_elem(const unsigned char* buf, int el) {
    if constexpr (DT == 0)
        return __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(buf)[el]) << 16);
    else
        return reinterpret_cast<const float*>(buf)[el];
}

// Named barrier 1 over the NT consumer threads only.
template <int NT>
__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory");
}

// Elements of a packed vector whose bit in `keep` is clear become -inf.
template <int DT>
__device__ __forceinline__ uint4 mask_neg_inf(uint4 r, uint32_t keep) {
    uint32_t* w = reinterpret_cast<uint32_t*>(&r);
    if constexpr (DT == 0) {  // two bf16 per word
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t k = (((keep >> (2 * i)) & 1u) ? 0x0000ffffu : 0u) |
                               (((keep >> (2 * i + 1)) & 1u) ? 0xffff0000u : 0u);
            w[i] = (w[i] & k) | (0xff80ff80u & ~k);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) w[i] = ((keep >> i) & 1u) ? w[i] : 0xff800000u;
    }
    return r;
}

template <int NT, int MODE>
struct RowsOcc {  // CTAs per SM the register budget is sized for
    // top-k CTAs hold their candidate lists in shared memory, which caps them
    // at 4 / 3 / 2 per SM; the other modes fit 6 / 4 / 2
    static constexpr int value = MODE == MODE_TOPK ? (NT <= 128 ? 4 : (NT <= 256 ? 3 : 2))
                                                   : (NT <= 128 ? 6 : (NT <= 256 ? 4 : 2));
};

template <int DT, int NT, int MODE, bool PROC>
__global__ void __launch_bounds__(NT + 32, RowsOcc<NT, MODE>::value) sv_rows_kernel(const RowsParams P) {
    constexpr int ELT = VT<DT>::ELT;
    constexpr int VEC = VT<DT>::VEC;
    constexpr int NW = NT / 32;             // consumer warps; warp NW is the producer
    constexpr int NTH = NT + 32;            // threads of the CTA
    constexpr int TV = TILE_BYTES / 16;     // vectors per tile
    constexpr int VPT = TV / NT;            // vectors per consumer thread per tile
    constexpr int SEG = TILE_BYTES / ELT;   // elements per segment
    constexpr int SSTRIDE = PROC ? STAGE_BYTES_PROC : STAGE_BYTES;  // bytes per ring stage
    constexpr uint32_t VMASK = (1u << VEC) - 1u;
    static_assert(VPT * NT == TV, "tile must split evenly over the consumer threads");
    static_assert(!PROC || MODE != MODE_GREEDY, "greedy verification takes no processors");
    static_assert(NW <= MAX_CONSUMER_WARPS, "too many consumer warps");
    extern __shared__ __align__(128) unsigned char smem[];
    RowsCtl& S = *reinterpret_cast<RowsCtl*>(smem);
    unsigned char* const ring = smem + ROWS_CTL_BYTES;
    unsigned char* const tail = ring + static_cast<size_t>(P.stages) * SSTRIDE;
    float* const red_m = reinterpret_cast<float*>(tail);          // softmax: [MAX_TILES_K1][NW]
    float* const red_s = red_m + MAX_TILES_K1 * NW;
    float* const lkey = reinterpret_cast<float*>(tail);           // top-k: [lcap] candidate-vector maxima
    int* const lidx = reinterpret_cast<int*>(lkey + P.lcap);      //        [lcap] their place: t*(TV+1) + j
    float* const vmsh = reinterpret_cast<float*>(tail + rows_tail_bytes(MODE, NT, P.lcap));  // PROC: [VPT+1][NT]

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
    // Launched as a programmatic dependent of whatever precedes it on the
    // stream (typically the previous call's per-sequence kernel, which lets its
    // dependents start early): nothing is read or written before the
    // preceding grid has completed.  A no-op when it did not start early.
    pdl_wait_primary();
    if (task == 0 && tid == 0 && P.out_status) *P.out_status = 0;
    pdl_launch_dependents();

    // processors of the row's sequence (PROC only)
    const long long pseq = PROC ? b / P.procs_div : 0;
    const float pen_theta = (PROC && P.theta) ? P.theta[pseq] : 1.f;  // repetition penalty
    const uint32_t* const gallow = PROC ? P.allow + pseq * P.W4 : nullptr;
    const uint32_t* const gpen = PROC ? P.pen + pseq * P.W4 : nullptr;
    (void)pen_theta;
    (void)gallow;
    (void)gpen;
    float cscale = 1.f;  // log2(e) / T
    if constexpr (MODE == MODE_SOFTMAX || MODE == MODE_TOPK) {
        const float T = P.temperature ? P.temperature[b] : 1.f;
        if (T > 0.f && T != POS_INF) cscale = LOG2E / T;
    }
    const int s0 = c * P.spc;
    const int ntiles = min(P.spc, P.nseg - s0);
    const int K = P.top_k;
    const int wcap = P.lcap / NW;  // top-k candidate vectors per warp segment
    auto geom = [&](int t) {
        const int lo = (s0 + t) * SEG;
        const int hi = min(P.V, lo + SEG);
        return tile_geom<ELT>(row, lo, hi);
    };

    if (tid == 0) {
        for (int st = 0; st < P.stages; ++st) {
            mbar_init(&S.full[st], 1);
            mbar_init(&S.empty[st], NW);
        }
        fence_mbar_init();
        S.issued = 0;
        S.copied = 0;
        S.tmo = 0;
        S.rawbad = 0;
        S.diag = 0;
    }
    if (tid < MAX_CONSUMER_WARPS) S.wbound[tid] = NEG_INF;
    __syncthreads();

    if (warp == NW) {
        // ================= producer: lane 0 fills the ring =================
        if (lane == 0) {
            int t = 0, copied = 0;
            for (; t < ntiles; ++t) {
                const int st = t % P.stages;
                if (*reinterpret_cast<volatile int*>(&S.tmo)) break;
                if (t >= P.stages &&
                    !mbar_wait_bounded(&S.empty[st], static_cast<uint32_t>((t / P.stages - 1) & 1), P.timeout_ns)) {
                    atomicOr(&S.tmo, 1);
                    break;
                }
                const TileGeom g = geom(t);
                unsigned char* buf = ring + static_cast<size_t>(st) * SSTRIDE;
                uint32_t bytes = 0;
                int nh = 0, ntl = 0;
                if (g.hi > g.lo) {
                    if (g.ga16 >= g.gb16) {
                        nh = g.hi - g.lo;
                    } else {
                        nh = static_cast<int>((g.ga16 - g.ga) / ELT);
                        ntl = static_cast<int>((g.gb - g.gb16) / ELT);
                        bytes = static_cast<uint32_t>(g.gb16 - g.ga16);
                    }
                }
                // self-check: a 16-byte aligned copy that stays inside its stage
                const uintptr_t doff = g.ga16 - g.A0;
                if (bytes != 0 &&
                    ((((reinterpret_cast<uintptr_t>(buf) + doff) | g.ga16 | bytes) & 15u) != 0 ||
                     doff + bytes > static_cast<uintptr_t>(STAGE_BYTES))) {
                    atomicOr(&S.diag, 1);
                    bytes = 0;
                    nh = ntl = 0;
                }
                // processors: the segment's bitmap words, a 16-byte aligned span
                // (rows padded to a multiple of 4 words, segments start at a
                // multiple of 128 elements) of whole words covering [lo, hi)
                uint32_t mbytes = 0;
                const uint32_t* asrc = nullptr;
                const uint32_t* psrc = nullptr;
                if constexpr (PROC) {
                    if (g.hi > g.lo) {
                        mbytes = static_cast<uint32_t>(((g.hi - g.lo + 127) / 128) * 16);
                        asrc = gallow + g.lo / 32;
                        psrc = gpen + g.lo / 32;
                        if (((reinterpret_cast<uintptr_t>(asrc) | reinterpret_cast<uintptr_t>(psrc) | mbytes) & 15u) != 0 ||
                            mbytes > static_cast<uint32_t>(MASK_STAGE_BYTES - 32) || g.lo % 128 != 0 ||
                            g.lo / 32 + static_cast<int>(mbytes / 4) > P.W4) {
                            atomicOr(&S.diag, 1);
                            mbytes = 0;
                        }
                    }
                }
                // Test hook: the stage expects test_extra_tx bytes that no copy
                // delivers (no bulk copy is issued), so its wait runs out.
                if (P.test_extra_tx) bytes = mbytes = 0;
                // elements outside the aligned interior: plain loads, published by the arrive
                for (int q = 0; q < nh + ntl; ++q) {
                    const int e = q < nh ? g.lo + q : g.hi - ntl + (q - nh);
                    if constexpr (DT == 0)
                        reinterpret_cast<uint16_t*>(buf)[e - g.e0] = reinterpret_cast<const uint16_t*>(row)[e];
                    else
                        reinterpret_cast<float*>(buf)[e - g.e0] = reinterpret_cast<const float*>(row)[e];
                }
                mbar_arrive_expect_tx(&S.full[st], bytes + 2 * mbytes + P.test_extra_tx);
                if (bytes) bulk_g2s(buf + doff, reinterpret_cast<const void*>(g.ga16), bytes, &S.full[st]);
                if (mbytes) {
                    bulk_g2s(buf + STAGE_BYTES, asrc, mbytes, &S.full[st]);
                    bulk_g2s(buf + STAGE_BYTES + MASK_STAGE_BYTES, psrc, mbytes, &S.full[st]);
                }
                copied = (bytes | mbytes) ? (copied | (1 << st)) : (copied & ~(1 << st));
            }
            S.issued = t;
            S.copied = copied;
        }
        __syncwarp();
    } else {
        // ================= consumers =================
        float run = NEG_INF;    // running NaN-propagating maximum of this thread's (processed) elements
        bool rawbad = false;    // processors: a raw NaN or +inf was seen
        float wbest = NEG_INF;  // greedy: best value of this warp and its lowest index
        int widx = -1;
        const int rsel = (K + NW - 1) / NW;  // <= 32 on the top-k path (K <= NT)
        float* const wkey = lkey + warp * wcap;
        int* const widxs = lidx + warp * wcap;
        int wcnt = 0;       // vectors in this warp's segment (warp-uniform)
        bool wovf = false;  // the segment lost vectors (massive ties at the bound)
        float theta = NEG_INF;
        float pub = NEG_INF;  // this warp's last published bound

        // rsel-th largest of the lanes' running maxima
        auto lane_bound = [&]() -> float {
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
        auto publish = [&](float v) {
            if (v > pub) {
                pub = v;
                if (lane == 0) *reinterpret_cast<volatile float*>(&S.wbound[warp]) = v;
            }
        };
        auto read_bound = [&]() {
            float mn = *reinterpret_cast<volatile float*>(&S.wbound[0]);
#pragma unroll
            for (int w = 1; w < NW; ++w) mn = fminf(mn, *reinterpret_cast<volatile float*>(&S.wbound[w]));
            return mn;
        };
        // Segment full: publish its rsel-th largest key (rank counting), raise
        // theta to the freshest bound and keep, in order, the vectors >= theta.
        auto compact = [&]() {
            float sel = NEG_INF;
            for (int q0 = 0; q0 < wcnt; q0 += 32) {
                const int q = q0 + lane;
                if (q < wcnt) {
                    const float x = wkey[q];
                    int gt = 0, ge = 0;
                    for (int f = 0; f < wcnt; ++f) {
                        const float y = wkey[f];
                        gt += y > x;
                        ge += y >= x;
                    }
                    if (gt < rsel && rsel <= ge) sel = x;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sel = fmaxf(sel, __shfl_xor_sync(0xffffffffu, sel, o));
            if (wcnt >= rsel) publish(sel);
            theta = fmaxf(theta, read_bound());
            int keep = 0;
            for (int q0 = 0; q0 < wcnt; q0 += 32) {
                const int q = q0 + lane;
                const bool in = q < wcnt;
                float x = NEG_INF;
                int ix = 0;
                if (in) {
                    x = wkey[q];
                    ix = widxs[q];
                }
                const bool ge = in && x >= theta;
                const unsigned m = __ballot_sync(0xffffffffu, ge);
                __syncwarp();
                if (ge) {
                    const int d = keep + __popc(m & ((1u << lane) - 1u));
                    wkey[d] = x;
                    widxs[d] = ix;
                }
                keep += __popc(m);
                __syncwarp();
            }
            wcnt = keep;
        };

        for (int t = 0; t < ntiles; ++t) {
            const int st = t % P.stages;
            const TileGeom g = geom(t);
            const unsigned char* buf = ring + static_cast<size_t>(st) * SSTRIDE;
            const uint32_t* const sallow = reinterpret_cast<const uint32_t*>(buf + STAGE_BYTES);
            const uint32_t* const spen = reinterpret_cast<const uint32_t*>(buf + STAGE_BYTES + MASK_STAGE_BYTES);
            const bool ok = mbar_wait_bounded(&S.full[st], static_cast<uint32_t>((t / P.stages) & 1), P.timeout_ns);
            if (!ok && lane == 0) atomicOr(&S.tmo, 1);
            auto valid = [&](int e) { return e >= g.lo && e < g.hi; };
            auto vec_at = [&](int j) { return *reinterpret_cast<const uint4*>(buf + 16 * j); };
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
            auto load_masked = [&](int j, float* v) {
                unpack<DT>(vec_at(j), v);
                const int e = g.e0 + j * VEC;
                if (!(e >= g.lo && e + VEC <= g.hi)) {
#pragma unroll
                    for (int q = 0; q < VEC; ++q)
                        if (!valid(e + q)) v[q] = NEG_INF;
                }
            };
            // PROC: the VEC allow or penalty bits of elements e .. e+VEC-1;
            // positions before the segment read as `ones` (validity masks them)
            auto bits_at = [&](const uint32_t* M, int e, bool ones) -> uint32_t {
                const int rr = e - g.lo;
                uint32_t x;
                if (rr >= 0)
                    x = __funnelshift_r(M[rr >> 5], M[(rr >> 5) + 1], rr & 31);
                else
                    x = (M[0] << (-rr)) | (ones ? ((1u << (-rr)) - 1u) : 0u);
                return x & VMASK;
            };
            // PROC: processed values of the vector at `raw` (first element e),
            // -inf outside the segment
            auto proc_vals = [&](const uint4& raw, int e, float* v) {
                unpack<DT>(raw, v);
                const uint32_t ab = bits_at(sallow, e, true), pb = bits_at(spen, e, false);
                if (pb) {  // a listed token in this vector (rare): the rounded quotient or product
#pragma unroll
                    for (int q = 0; q < VEC; ++q)
                        if ((pb >> q) & 1u) v[q] = penalise(v[q], pen_theta);
                }
#pragma unroll
                for (int q = 0; q < VEC; ++q)
                    if (!valid(e + q) || !((ab >> q) & 1u)) v[q] = NEG_INF;
            };
            // PROC: processed maximum of vector j (raw errors noted on the way).
            // Without a penalised element the disallowed (or out-of-segment)
            // elements are replaced by -inf in the packed vector with bit
            // operations and the plain maximum is taken; a vector holding a
            // listed id takes the per-element path.
            // Top-k with theta >= 1: no processed value exceeds its raw one, so
            // a vector whose raw maximum is below the running bound cannot be
            // a candidate and counts as -inf (the bounds stay lower bounds).
            auto proc_vmax = [&](int j, float skip_below) -> float {
                const uint4 raw = vec_at(j);
                const int e = g.e0 + j * VEC;
                const bool full = e >= g.lo && e + VEC <= g.hi;
                const float rm = full ? vmax_nan<DT>(raw) : vmax_masked(j);
                if (!(rm == rm) || rm == POS_INF) rawbad = true;
                if (rm < skip_below) return NEG_INF;
                uint32_t ab = bits_at(sallow, e, true);
                const uint32_t pb = bits_at(spen, e, false);
                if (pb == 0u) {
                    if (!full) {
#pragma unroll
                        for (int q = 0; q < VEC; ++q)
                            if (!valid(e + q)) ab &= ~(1u << q);
                    }
                    return vmax_nan<DT>(mask_neg_inf<DT>(raw, ab));
                }
                float v[VEC];
                proc_vals(raw, e, v);
                float m = NEG_INF;
#pragma unroll
                for (int q = 0; q < VEC; ++q) m = fmax_nan(m, v[q]);
                return m;
            };
            // this thread's vectors: slot i < VPT is vector tid + i*NT; slot VPT
            // is the one vector past TV that a segment starting off a 16-byte
            // boundary spans (vector TV + tid, tid == 0 only)
            auto jof = [&](int i) { return i < VPT ? tid + i * NT : TV + tid; };
            float vm[VPT + 1];
            const bool tile_full = ok && g.e0 == g.lo && g.nvec == TV && g.hi - g.lo == TV * VEC;
            // softmax with processors: this thread's running maximum of z*c and
            // sum of 2^(z*c - maximum) over its processed elements, one pass
            float pm = NEG_INF, ps = 0.f;
            (void)pm;
            (void)ps;
            if constexpr (PROC && MODE == MODE_SOFTMAX) {
#pragma unroll 1
                for (int i = 0; i <= VPT; ++i) {
                    const int j = jof(i);
                    if (!(ok && j < g.nvec)) continue;
                    const uint4 raw = vec_at(j);
                    const int e = g.e0 + j * VEC;
                    const bool full = e >= g.lo && e + VEC <= g.hi;
                    const float rm = full ? vmax_nan<DT>(raw) : vmax_masked(j);
                    if (!(rm == rm) || rm == POS_INF) rawbad = true;
                    float v[VEC];
                    if (bits_at(spen, e, false) == 0u) {
                        uint32_t ab = bits_at(sallow, e, true);
#pragma unroll
                        for (int q = 0; q < VEC; ++q)
                            if (!valid(e + q)) ab &= ~(1u << q);
                        unpack<DT>(mask_neg_inf<DT>(raw, ab), v);
                    } else {
                        proc_vals(raw, e, v);
                    }
                    float vmx = NEG_INF;
#pragma unroll
                    for (int q = 0; q < VEC; ++q) vmx = fmaxf(vmx, v[q]);
                    const float mc = vmx * cscale;
                    if (mc > pm) {
                        ps = pm > NEG_INF ? ps * ex2(pm - mc) : 0.f;
                        pm = mc;
                    }
                    if (pm > NEG_INF) {
#pragma unroll
                        for (int q = 0; q < VEC; ++q) ps += ex2(fmaf(v[q], cscale, -pm));
                    }
                }
#pragma unroll
                for (int i = 0; i <= VPT; ++i) vm[i] = NEG_INF;
            } else if constexpr (PROC) {
                // raw maxima first (the plain path's cost); then one copy of the
                // processing code (a rolled loop) over the vectors that need it,
                // whose maxima come back through this thread's own slots
                const float skip_below = (MODE == MODE_TOPK && pen_theta >= 1.f) ? theta : NEG_INF;
                unsigned need = 0u;
#pragma unroll
                for (int i = 0; i <= VPT; ++i) {
                    const int j = jof(i);
                    float rm = NEG_INF;
                    if (ok && j < g.nvec) {
                        rm = tile_full ? vmax_nan<DT>(vec_at(j)) : vmax_masked(j);
                        if (!(rm < skip_below)) need |= 1u << i;
                    }
                    if (!(rm == rm) || rm == POS_INF) rawbad = true;
                }
                for (unsigned mm = need; mm; mm &= mm - 1u) {
                    const int i = __ffs(mm) - 1;
                    vmsh[i * NT + tid] = proc_vmax(jof(i), NEG_INF);
                }
#pragma unroll
                for (int i = 0; i <= VPT; ++i) vm[i] = ((need >> i) & 1u) ? vmsh[i * NT + tid] : NEG_INF;
            } else if (tile_full) {
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
            bool held = true;  // this warp still holds the stage

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
            } else if constexpr (MODE == MODE_SOFTMAX && PROC) {
                // the lanes' running (maximum, sum) pairs, combined
                float m = pm, sm = ps;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
                    ms_combine(m, sm, __shfl_xor_sync(0xffffffffu, m, o), __shfl_xor_sync(0xffffffffu, sm, o));
                if (lane == 0) {
                    red_m[t * NW + warp] = m;
                    red_s[t * NW + warp] = sm;
                }
            } else if constexpr (MODE == MODE_SOFTMAX) {
                // one maximum per warp; pass B sums 2^(z*c - m) with two accumulators
                float wtm = tm;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) wtm = fmax_nan(wtm, __shfl_xor_sync(0xffffffffu, wtm, o));
                const float m = wtm * cscale;
                float sa = 0.f, sb = 0.f;
                if (ok && m > NEG_INF && m < POS_INF) {
                    auto acc_vec = [&](int j) {
                        float v[VEC];
                        if constexpr (PROC) {
                            const int e = g.e0 + j * VEC;
                            if (bits_at(spen, e, false) == 0u) {
                                uint32_t ab = bits_at(sallow, e, true);
#pragma unroll
                                for (int q = 0; q < VEC; ++q)
                                    if (!valid(e + q)) ab &= ~(1u << q);
                                unpack<DT>(mask_neg_inf<DT>(vec_at(j), ab), v);
                            } else {
                                proc_vals(vec_at(j), e, v);
                            }
                        } else {
                            load_masked(j, v);
                        }
#pragma unroll
                        for (int q = 0; q < VEC; q += 2) {
                            sa += ex2(fmaf(v[q], cscale, -m));
                            sb += ex2(fmaf(v[q + 1], cscale, -m));
                        }
                    };
                    if constexpr (PROC) {  // one copy of the processing code
#pragma unroll 1
                        for (int i = 0; i <= VPT; ++i)
                            if (jof(i) < g.nvec) acc_vec(jof(i));
                    } else {
#pragma unroll
                        for (int i = 0; i <= VPT; ++i)
                            if (jof(i) < g.nvec) acc_vec(jof(i));
                    }
                }
                const float ws = warp_sum(sa + sb);
                if (lane == 0) {
                    red_m[t * NW + warp] = m;
                    red_s[t * NW + warp] = ws;
                }
            } else if constexpr (MODE == MODE_TOPK) {
                run = fmax_nan(run, tm);
                // hand the stage back at once: the bookkeeping below reads the
                // maxima in registers and the warp's list only
                __syncwarp();
                if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&S.empty[st])) : "memory");
                held = false;
                if (t == 0) {
                    // every warp publishes a bound from the first tile before any append
                    publish(lane_bound());
                    consumer_sync<NT>();
                } else if (t & 1) {
                    publish(lane_bound());
                }
                theta = fmaxf(theta, read_bound());
                // Candidate vectors (finite maximum at or above the bound) go
                // to the warp's list as (maximum, place in the chunk).
                unsigned cm = 0u;  // bit i: slot i holds a candidate
                if (!wovf) {
#pragma unroll
                    for (int i = 0; i <= VPT; ++i)
                        if (ok && vm[i] > NEG_INF && vm[i] >= theta) cm |= 1u << i;
                    // each lane's candidates go to consecutive list entries: an
                    // exclusive prefix sum of the lanes' counts gives the offsets
                    int cnt = __popc(cm), incl = cnt;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const int y = __shfl_up_sync(0xffffffffu, incl, o);
                        if (lane >= o) incl += y;
                    }
                    int total = __shfl_sync(0xffffffffu, incl, 31);
                    if (total && wcnt + total > wcap) {
                        compact();  // raises theta
#pragma unroll
                        for (int i = 0; i <= VPT; ++i)
                            if (!(vm[i] >= theta)) cm &= ~(1u << i);
                        cnt = __popc(cm);
                        incl = cnt;
#pragma unroll
                        for (int o = 1; o < 32; o <<= 1) {
                            const int y = __shfl_up_sync(0xffffffffu, incl, o);
                            if (lane >= o) incl += y;
                        }
                        total = __shfl_sync(0xffffffffu, incl, 31);
                        if (wcnt + total > wcap) wovf = true;  // massive ties: exact fallback downstream
                    }
                    if (total && !wovf) {
                        int p = wcnt + incl - cnt;
#pragma unroll
                        for (int i = 0; i <= VPT; ++i) {
                            if ((cm >> i) & 1u) {
                                wkey[p] = vm[i];
                                widxs[p] = t * (TV + 1) + jof(i);
                                ++p;
                            }
                        }
                        wcnt += total;
                    }
                }
            } else {
                run = fmax_nan(run, tm);  // MODE_MAXONLY
            }

            if (held) {
                // hand the stage back to the producer
                __syncwarp();
                if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&S.empty[st])) : "memory");
            }
            if (!ok) break;
        }

        // ---- per-warp results ------------------------------------------------------
        if constexpr (PROC) {
            if (__any_sync(0xffffffffu, rawbad) && lane == 0) atomicOr(&S.rawbad, 1);
        }
        if constexpr (MODE != MODE_SOFTMAX) {
            const float wm = warp_max_nan(run);
            if (lane == 0) {
                S.wmax[warp] = wm;
                S.wbest[warp] = wbest;
                S.widx[warp] = widx;
            }
        }
        if constexpr (MODE == MODE_TOPK) {
            publish(lane_bound());  // from every element of the chunk
            if (lane == 0) {
                S.wcnt[warp] = wcnt;
                S.wovf[warp] = wovf ? 1 : 0;
            }
        }
    }
    __syncthreads();  // every tile is consumed (or a wait ran out)

    const int tmo = S.tmo;
    const int diag = S.diag;
    const bool rawerr = PROC && S.rawbad;  // the row is an error: its records carry NaN
    const int bad = tmo | diag;
    const int flag = (tmo ? REC_TIMEOUT : 0) | (diag ? REC_DIAG : 0);

    // ---- partial records ------------------------------------------------------------
    if constexpr (MODE == MODE_SOFTMAX) {
        for (int q = tid; q < ntiles; q += NTH) {
            SegRec rec;
            rec.arg = -1;
            rec.flags = flag;
            if (bad) {
                rec.m = __int_as_float(0x7fc00000);
                rec.s = 0.f;
            } else {
                float m = red_m[q * NW], sm = red_s[q * NW];
                for (int w = 1; w < NW; ++w) ms_combine(m, sm, red_m[q * NW + w], red_s[q * NW + w]);
                rec.m = rawerr ? __int_as_float(0x7fc00000) : m;
                rec.s = sm;
            }
            P.segs[r * P.nseg + s0 + q] = rec;
        }
    } else if constexpr (MODE == MODE_GREEDY || MODE == MODE_MAXONLY) {
        if (tid == 0) {
            SegRec rec;
            rec.m = S.wmax[0];
            rec.s = 0.f;
            float bv = S.wbest[0];
            int bi = S.widx[0];
            for (int w = 1; w < NW; ++w) {
                rec.m = fmax_nan(rec.m, S.wmax[w]);
                if (arg_better(S.wbest[w], S.widx[w], bv, bi)) {
                    bv = S.wbest[w];
                    bi = S.widx[w];
                }
            }
            rec.arg = MODE == MODE_GREEDY ? bi : -1;
            rec.flags = flag;
            if (bad || rawerr) rec.m = __int_as_float(0x7fc00000);
            P.segs[r * P.nseg + c] = rec;
        }
    }

    if (bad) {
        if (tid == 0) {
            if constexpr (MODE == MODE_TOPK) {
                ChunkRec ch;
                ch.tau = NEG_INF;
                ch.last = NEG_INF;
                ch.n = 0;
                ch.flags = flag;
                ch.m = __int_as_float(0x7fc00000);
                ch.s = 0.f;
                ch.zd = NEG_INF;
                ch.pad = 0;
                P.chunks[r * P.nch + c] = ch;
            }
            // wait (bounded) for the last bulk copy issued into each stage, so
            // that no copy is still writing this CTA's shared memory at exit
            const int issued = S.issued, copied = S.copied;
            for (int q = 0; q < min(issued, P.stages); ++q) {
                if (!((copied >> q) & 1)) continue;
                const int last = q + ((issued - 1 - q) / P.stages) * P.stages;
                mbar_wait_bounded(&S.full[q], static_cast<uint32_t>((last / P.stages) & 1), P.timeout_ns);
            }
        }
        return;
    }
    if constexpr (MODE == MODE_TOPK) {
        // ---- exact K-th largest of the chunk and its kept entries -----------------
        float cmax = S.wmax[0];
        float thf = S.wbound[0];
        int ovf = S.wovf[0];
        for (int w = 1; w < NW; ++w) {
            cmax = fmax_nan(cmax, S.wmax[w]);
            thf = fminf(thf, S.wbound[w]);
            ovf |= S.wovf[w];
        }
        if (rawerr) cmax = __int_as_float(0x7fc00000);
        const int d = (pos < P.k && P.draft_tokens) ? P.draft_tokens[b * P.k + pos] : -1;
        Cand* fl = reinterpret_cast<Cand*>(ring);  // candidate vectors (the ring is free now)
        const int fcap = (P.stages * STAGE_BYTES) / static_cast<int>(sizeof(Cand));
        Cand* E = reinterpret_cast<Cand*>(lkey);  // expanded elements (after step 1)
        const int ecap = P.lcap;
        if (tid == 0) {
            S.cnt2 = 0;
            S.ne = 0;
            S.nkept = 0;
            S.tau = NEG_INF;
            S.thf = NEG_INF;
        }
        __syncthreads();
        // 1. candidate vectors whose maximum reaches the final bound
        if (warp < NW) {
            const int n = S.wcnt[warp];
            const float* wk = lkey + warp * wcap;
            const int* wi = lidx + warp * wcap;
            for (int q0 = 0; q0 < n; q0 += 32) {
                const int q = q0 + lane;
                const bool ge = q < n && wk[q] >= thf;
                const unsigned m = __ballot_sync(0xffffffffu, ge);
                int base = 0;
                if (lane == 0 && m) base = atomicAdd(&S.cnt2, __popc(m));
                base = __shfl_sync(0xffffffffu, base, 0);
                const int p = base + __popc(m & ((1u << lane) - 1u));
                if (ge && p < fcap) fl[p] = Cand{wk[q], wi[q]};
            }
        }
        __syncthreads();
        const int nv = min(S.cnt2, fcap);
        // 2. tau_v = K-th largest vector maximum (with multiplicity); at least
        //    K distinct elements are >= tau_v, so the chunk's K-th largest
        //    logit is >= tau_v and lies in a vector whose maximum is >= tau_v.
        for (int q = tid; q < nv; q += NTH) {
            const float x = fl[q].v;
            int gt = 0, ge = 0;
#pragma unroll 8
            for (int f = 0; f < nv; ++f) {
                const float y = fl[f].v;
                gt += y > x;
                ge += y >= x;
            }
            if (gt < K && K <= ge) S.thf = x;
        }
        __syncthreads();
        const float tauv = S.thf;  // -inf: fewer than K candidate vectors (all are expanded)
        // 3. the elements >= tau_v of those vectors, read again from the row
        for (int q = tid; q < nv; q += NTH) {
            const Cand cv = fl[q];
            if (!(cv.v >= tauv)) continue;
            const int tt = cv.i / (TV + 1), j = cv.i - tt * (TV + 1);
            const TileGeom g = geom(tt);
            const int e = g.e0 + j * VEC;
            float v[VEC];
            if (e >= g.lo && e + VEC <= g.hi) {
                unpack<DT>(__ldg(reinterpret_cast<const uint4*>(g.A0 + 16u * static_cast<uintptr_t>(j))), v);
            } else {
#pragma unroll
                for (int u = 0; u < VEC; ++u) v[u] = (e + u >= g.lo && e + u < g.hi) ? load_elem<DT>(row, e + u) : NEG_INF;
            }
            if constexpr (PROC) {
                ProcView pv;
                pv.allow = gallow;
                pv.pen = gpen;
                pv.theta = pen_theta;
#pragma unroll
                for (int u = 0; u < VEC; ++u)
                    if (e + u >= g.lo && e + u < g.hi) v[u] = proc_logit(v[u], e + u, pv);
            }
#pragma unroll
            for (int u = 0; u < VEC; ++u) {
                if (v[u] >= tauv && e + u >= g.lo && e + u < g.hi) {
                    const int p = atomicAdd(&S.ne, 1);
                    if (p < ecap) E[p] = Cand{v[u], e + u};
                }
            }
        }
        __syncthreads();
        const int ne_all = S.ne;
        const int ne = min(ne_all, ecap);
        if (ne_all > ecap || ne > RANK_MAX) ovf = 1;  // massive ties: exact fallback downstream
        // 4. tau = K-th largest element (with multiplicity)
        if (!ovf) {
            for (int q = tid; q < ne; q += NTH) {
                const float x = E[q].v;
                int gt = 0, ge = 0;
#pragma unroll 8
                for (int f = 0; f < ne; ++f) {
                    const float y = E[f].v;
                    gt += y > x;
                    ge += y >= x;
                }
                if (gt < K && K <= ge) S.tau = x;
            }
        }
        __syncthreads();
        const float tau = S.tau;  // -inf: fewer than K elements, every one is kept
        // 5. kept entries (>= tau) in index order, staged in the ring
        Cand* ks = fl;  // fl is no longer read after step 3
        const int kscap = fcap;
        Cand* out = P.cands + (r * P.nch + c) * static_cast<long long>(P.kcap);
        if (!ovf) {
            for (int q = tid; q < ne; q += NTH) {
                const Cand x = E[q];
                if (!(x.v >= tau)) continue;
                int ri = 0;
#pragma unroll 8
                for (int f = 0; f < ne; ++f) ri += (E[f].v >= tau && E[f].i < x.i);
                atomicAdd(&S.nkept, 1);
                if (ri < kscap) ks[ri] = x;
            }
        }
        __syncthreads();
        const int nk = S.nkept;
        const float lastv = tau;  // every kept entry is >= tau
        // exp-sum and draft-token logit over the stored (index-sorted) entries
        const int m = min(nk, P.kcap);
        const float msc = cmax * cscale;
        float acc = 0.f, zd = NEG_INF;
        for (int q = tid; q < m; q += NTH) {
            const Cand e = ks[q];
            out[q] = e;
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
            for (int w = 0; w <= NW; ++w) {
                s += S.wsum[w];
                z = fmaxf(z, S.wzd[w]);
            }
            ChunkRec ch;
            ch.tau = S.tau;
            ch.last = lastv;
            ch.n = m;
            ch.flags = (ovf || nk > P.kcap) ? REC_OVERFLOW : 0;
            if (ovf) ch.n = 0;
            ch.m = cmax;
            ch.s = s;
            ch.zd = z;
            ch.pad = 0;
            P.chunks[r * P.nch + c] = ch;
        }
    }
}

}  // namespace sv
