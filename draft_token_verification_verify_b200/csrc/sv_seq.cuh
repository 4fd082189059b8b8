// K2 — one CTA per sequence: merge the streaming partials of the sequence's
// rows, take the acceptance decisions and draw the final token.
//
// Method (speculative decoding entry "推测解码", section "提议与核验的基本步骤"):
// with p and q the processed target and draft distributions, position i
// accepts d_i iff u_i * q_i(d_i) < p_i(d_i) (probability min(1, p/q)); the
// first rejected position j is redrawn from max(0, p_j - q_j), normalised;
// after k acceptances the bonus token is drawn from p_k; both draws take u_k
// through the inverse CDF in index order.  Greedy mode compares d_i with the
// lowest-index argmax of the target row.
//
// Paths: with top-k and one chunk per row, every row's chunk record and kept
// list arrive in one round of loads, and a sequence whose rows are all clean
// is finished by warp 0 alone (lane r holds row r; decisions by ballot; the
// draw over the kept lists in shared memory).  Otherwise the block path
// merges the partials with one warp per row.  Draws without top-k: a bonus
// draw locates its segment from the streaming partials and rescans that
// segment; a residual draw is handed to the segment kernel (one CTA per
// segment of the rejected (target, draft) pair).  Rows whose kept list did
// not fit (massive ties), or top-k resolved by radix select, get an exact
// radix select over the row in global memory and a draw that streams the
// row (pair) in this CTA.  A nucleus (top_p < 1) is taken over the kept lists
// on the top-k path, over the kept set of a radix-selected row here, and, with
// no top-k, by the nucleus kernel, whose per-row cut and normaliser become
// the row's threshold; every later read of a probability applies it.
#pragma once

#include <climits>

#include "sv_common.cuh"
#include "sv_nucleus.cuh"
#include "sv_procs.cuh"

namespace sv {

constexpr int SEQ_NT = 256;
constexpr int SEQ_NW = SEQ_NT / 32;

struct SeqParams {
    const void* target;          // [B][k+1][V]
    const void* draft;           // [B][k][V] or null
    const int32_t* draft_tokens; // [B][k] or null (sampler)
    const float* uniforms;       // [B][k+1] or null (greedy)
    const float* temperature;    // [B] or null
    long long B;
    int k;
    int V;
    int mode;                    // MODE_* used by the streaming pass
    int top_k;
    int sample_only;             // proposer sampler: write one token per row
    int seg, nseg, spc, nch, kcap;
    int mg;                      // gather capacity per warp (power of two)
    const SegRec* segs;
    const ChunkRec* chunks;      // [R][nch] top-k: per-chunk record
    const Cand* cands;           // [R][nch][kcap] top-k: per-chunk kept list, index order
    int32_t* out_tokens;         // [B][k+1] (sampler: [B])
    int32_t* out_n;              // [B] or null (sampler)
    float* out_p;                // [B][k] or null
    float* out_q;                // [B][k] or null
    int32_t* out_status;         // or null
    int pre;                     // top-k with one chunk per row: every row's record and kept
                                 // list is loaded into shared memory at offset pre_off
    int pre_off;
    int defer;                   // residual draws go to the segment kernel (softmax, verify)
    const float* top_p;          // [S] nucleus thresholds or null
    const NucRec* nuc;           // [R] nucleus cuts of the rows (softmax mode with top_p) or null
    DrawReq* req;                // [B] when defer
    int* counter;                // [B] when defer: zeroed here for the segment kernel
    // processors (mask, repetition penalty): bitmaps built by K0, or null
    const uint32_t* allow;       // [S][W4]
    const uint32_t* pen;         // [S][W4]
    const float* theta;          // [S] or null
    int W4;
    int procs_div;               // sequence of the processors (and top_p) of b: b / procs_div
};

struct RowStat {
    float msc;   // maximum in log2 units (z*c)
    float invS;  // 1 / normaliser
    float tau;   // kept threshold (-inf: every finite logit)
    float zd;    // logit at the draft token of the row's position (NaN if none)
    int arg;     // greedy argmax
    int err;     // 1 data error, 2 timeout
    int slow;    // top-k threshold must be resolved by radix select
    int pad;
};

struct __align__(16) SeqCtl {
    float red_f[SEQ_NW][2];
    int red_i[SEQ_NW];
    int hist[256];
    int j;
    int err;
    int token;
    int tok_cross;
    int tok_last;
    int seg_sel;
    int last_mode;
    int retry;
    int radix_digit;
    int radix_k;
    uint32_t radix_prefix;
    float x;
    float base;
    float W;
    float c;
    NucCtl nuc;  // nucleus cut of a row resolved here (radix top-k rows)
    float ftau[32];  // one-warp path with a nucleus: each row's cut and 1 / kept mass
    float finv[32];
};

constexpr int SEQ_CTL_BYTES = (int)((sizeof(SeqCtl) + 127) / 128 * 128);

template <int DT>
__global__ void __launch_bounds__(SEQ_NT, 3) sv_seq_kernel(const SeqParams P) {
    constexpr int VEC = VT<DT>::VEC;
    constexpr int ELT = VT<DT>::ELT;
    constexpr int NT = SEQ_NT, NW = SEQ_NW;
    extern __shared__ __align__(128) unsigned char smem[];
    SeqCtl& S = *reinterpret_cast<SeqCtl*>(smem);
    const int k = P.k, V = P.V;
    const bool greedy = P.mode == MODE_GREEDY;
    const int nrows = greedy || P.sample_only ? k + 1 : 2 * k + 1;
    RowStat* rs = reinterpret_cast<RowStat*>(smem + SEQ_CTL_BYTES);
    int* dtok = reinterpret_cast<int*>(rs + nrows);
    float* uu = reinterpret_cast<float*>(dtok + (k > 0 ? k : 1));
    Cand* gbuf = reinterpret_cast<Cand*>(
        smem + SEQ_CTL_BYTES +
        (((static_cast<size_t>(nrows) * sizeof(RowStat) + (k + 1) * 8 + 8) + 127) / 128 * 128));
    float* part = reinterpret_cast<float*>(gbuf + static_cast<size_t>(NW) * P.mg);  // [nseg][NW]
    float* mass = part + static_cast<size_t>(P.nseg) * NW;                            // [nseg]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long b = blockIdx.x;
    const long long Rt = P.B * (k + 1);
    const int K = P.top_k;

    // ---- inputs that do not depend on the streaming pass -----------------------
    float T = 1.f;
    if (!greedy && P.temperature) T = P.temperature[b];
    const long long pseq = b / P.procs_div;  // the processors' sequence (the sampler groups rows)
    const float tp = (!greedy && P.top_p) ? P.top_p[pseq] : 1.f;  // nucleus threshold
    const ProcView pv = proc_view(P.allow, P.pen, P.theta, P.W4, pseq);
    const float th = pv.theta;  // repetition penalty theta
    const float c = (T > 0.f && T != POS_INF) ? LOG2E / T : 1.f;
    for (int i = tid; i < k; i += NT) dtok[i] = P.draft_tokens[b * k + i];
    if (!greedy)
        for (int i = tid; i <= k; i += NT) uu[i] = P.uniforms[b * (k + 1) + i];
    if (tid == 0) {
        S.err = 0;
        S.c = c;
    }
    __syncthreads();
    if (tid == 0) {
        int bad = 0;
        for (int i = 0; i < k; ++i)
            if (dtok[i] < 0 || dtok[i] >= V) bad = 1;
        if (!greedy) {
            if (!(T > 0.f) || T == POS_INF) bad = 1;
            if (!(tp > 0.f && tp <= 1.f)) bad = 1;
            if (pv.allow && !(th > 0.f && th != POS_INF)) bad = 1;
            for (int i = 0; i <= k; ++i)
                if (!(uu[i] >= 0.f && uu[i] < 1.f)) bad = 1;
        }
        S.err = bad;
    }
    pdl_launch_dependents();  // the segment kernel may be placed early; it waits for this grid
    pdl_wait_primary();       // the streaming pass is complete from here on

    auto row_ptr = [&](int rr) -> const void* {
        if (rr <= k)
            return static_cast<const char*>(P.target) + (static_cast<size_t>(b) * (k + 1) + rr) * static_cast<size_t>(V) * ELT;
        return static_cast<const char*>(P.draft) + (static_cast<size_t>(b) * k + (rr - k - 1)) * static_cast<size_t>(V) * ELT;
    };
    auto row_index = [&](int rr) -> long long { return rr <= k ? b * (k + 1) + rr : Rt + b * k + (rr - k - 1); };
    auto row_dtok = [&](int rr) -> int {
        const int pos = rr <= k ? rr : rr - k - 1;
        return pos < k ? dtok[pos] : -1;
    };

    // top-k, one chunk per row: all of the sequence's chunk records and kept
    // lists in one cooperative round of independent loads
    Cand* const plist = P.pre ? reinterpret_cast<Cand*>(smem + P.pre_off) : nullptr;  // [nrows][kcap]
    ChunkRec* const prec = P.pre ? reinterpret_cast<ChunkRec*>(plist + static_cast<size_t>(nrows) * P.kcap) : nullptr;
    if (P.pre) {
        const int per = 2 + P.kcap / 2;  // 16-byte vectors per row: record, then list
        constexpr int PF = 4;            // loads in flight per thread before their stores
        auto src = [&](int x) {
            const int rr = x / per, o = x - (x / per) * per;
            const long long r = rr <= k ? b * (k + 1) + rr : Rt + b * k + (rr - k - 1);
            return o < 2 ? reinterpret_cast<const uint4*>(P.chunks + r) + o
                         : reinterpret_cast<const uint4*>(P.cands + r * P.kcap) + (o - 2);
        };
        auto dst = [&](int x) {
            const int rr = x / per, o = x - (x / per) * per;
            return o < 2 ? reinterpret_cast<uint4*>(prec + rr) + o
                         : reinterpret_cast<uint4*>(plist + static_cast<size_t>(rr) * P.kcap) + (o - 2);
        };
        for (int x0 = tid; x0 < nrows * per; x0 += NT * PF) {
            uint4 tmp[PF];
#pragma unroll
            for (int u = 0; u < PF; ++u)
                if (x0 + u * NT < nrows * per) tmp[u] = *src(x0 + u * NT);
#pragma unroll
            for (int u = 0; u < PF; ++u)
                if (x0 + u * NT < nrows * per) *dst(x0 + u * NT) = tmp[u];
        }
        __syncthreads();
    }

    // gather the entries >= thr of the row's chunk lists into dst (index order)
    auto gather = [&](long long r, float thr, Cand* dst, int cap) -> int {
        int base = 0;
        for (int ch = 0; ch < P.nch; ++ch) {
            const ChunkRec cr = P.chunks[r * P.nch + ch];
            const Cand* src = P.cands + (r * P.nch + ch) * static_cast<long long>(P.kcap);
            for (int e0 = 0; e0 < cr.n; e0 += 32) {
                const int e = e0 + lane;
                Cand cd = {NEG_INF, -1};
                if (e < cr.n) cd = src[e];
                const bool pred = e < cr.n && cd.v >= thr;
                const unsigned m = __ballot_sync(0xffffffffu, pred);
                const int pos = base + __popc(m & ((1u << lane) - 1u));
                if (pred && pos < cap) dst[pos] = cd;
                base += __popc(m);
            }
        }
        return base;
    };

    // ---- fast path: top-k, one chunk per row, every row clean ---------------------------
    // Warp 0 alone finishes the sequence: lane r holds row r's statistics, the
    // decisions come from shuffles and a ballot, and the draw reads the kept
    // lists already in shared memory.  Same arithmetic as the block path below.
    if (P.pre && nrows <= 32) {
        const bool clean = tid >= nrows || (prec[tid].flags == 0 && prec[tid].m == prec[tid].m &&
                                            prec[tid].m != POS_INF && prec[tid].m != NEG_INF);
        if (__syncthreads_and(clean) && !S.err) {
            const bool nucleus = tp < 1.f;
            if (nucleus) {
                // every warp: the nucleus over its rows' kept lists (the cut is the
                // largest kept value whose tail mass reaches top_p), as the block path
                for (int rr = warp; rr < nrows; rr += NW) {
                    const Cand* L = plist + static_cast<size_t>(rr) * P.kcap;
                    const int n = prec[rr].n;
                    const float rm = prec[rr].m * c, ri = 1.f / prec[rr].s, rt = prec[rr].tau;
                    float cand = NEG_INF;
                    for (int e = lane; e < n; e += 32) {
                        const float x = L[e].v;
                        if (!(x >= rt)) continue;
                        float mass = 0.f;
                        for (int f = 0; f < n; ++f) {
                            const float y = L[f].v;
                            if (y >= x && y >= rt) mass += ex2(fmaf(y, c, -rm)) * ri;
                        }
                        if (mass >= tp) cand = fmaxf(cand, x);
                    }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) cand = fmaxf(cand, __shfl_xor_sync(0xffffffffu, cand, o));
                    const float cut = fmaxf(cand, rt);
                    float acc = 0.f;
                    for (int e = lane; e < n; e += 32)
                        if (L[e].v >= cut) acc += ex2(fmaf(L[e].v, c, -rm));
                    acc = warp_sum(acc);
                    if (lane == 0) {
                        S.ftau[rr] = cut;
                        S.finv[rr] = 1.f / acc;
                    }
                }
                __syncthreads();
            }
            if (warp != 0) return;
            const ChunkRec rec = prec[lane < nrows ? lane : 0];
            const float msc = rec.m * c, zd = rec.zd;
            const float invS = nucleus ? S.finv[lane < nrows ? lane : 0] : 1.f / rec.s;
            const float tau = nucleus ? S.ftau[lane < nrows ? lane : 0] : rec.tau;
            // decisions: lane i < k holds target row i; draft row i is lane k+1+i
            int j = k;
            for (int i0 = 0; i0 < k; i0 += 32) {
                const int i = i0 + lane;
                const int src_t = i < k ? i : 0, src_d = i < k ? k + 1 + i : 0;
                const float t_msc = __shfl_sync(0xffffffffu, msc, src_t & 31), t_inv = __shfl_sync(0xffffffffu, invS, src_t & 31);
                const float t_tau = __shfl_sync(0xffffffffu, tau, src_t & 31), t_zd = __shfl_sync(0xffffffffu, zd, src_t & 31);
                const float d_msc = __shfl_sync(0xffffffffu, msc, src_d & 31), d_inv = __shfl_sync(0xffffffffu, invS, src_d & 31);
                const float d_tau = __shfl_sync(0xffffffffu, tau, src_d & 31), d_zd = __shfl_sync(0xffffffffu, zd, src_d & 31);
                bool rej = false;
                if (i < k) {
                    const float p = (t_zd >= t_tau) ? ex2(fmaf(t_zd, c, -t_msc)) * t_inv : 0.f;
                    const float q = (d_zd >= d_tau) ? ex2(fmaf(d_zd, c, -d_msc)) * d_inv : 0.f;
                    if (P.out_p) P.out_p[b * k + i] = p;
                    if (P.out_q) P.out_q[b * k + i] = q;
                    rej = !(uu[i] * q < p);
                }
                const unsigned m = __ballot_sync(0xffffffffu, rej);
                if (m && j == k) j = i0 + __ffs(m) - 1;  // the first rejection
            }
            // draw from the kept lists of position j
            const bool use_q0 = j < k;
            const float t_msc = __shfl_sync(0xffffffffu, msc, j), t_inv = __shfl_sync(0xffffffffu, invS, j);
            const float t_cut = __shfl_sync(0xffffffffu, tau, j);
            const int nt = __shfl_sync(0xffffffffu, rec.n, j);
            const int jd = use_q0 ? k + 1 + j : 0;
            const float d_msc = __shfl_sync(0xffffffffu, msc, jd), d_inv = __shfl_sync(0xffffffffu, invS, jd);
            const float d_cut = __shfl_sync(0xffffffffu, tau, jd);
            const int nd = use_q0 ? __shfl_sync(0xffffffffu, rec.n, jd) : 0;
            const Cand* lt = plist + static_cast<size_t>(j) * P.kcap;
            const Cand* ld = plist + static_cast<size_t>(jd) * P.kcap;
            float* wv = reinterpret_cast<float*>(gbuf);
            const float u = uu[k];
            auto find = [&](int v) {
                int a = 0, z = nd - 1;
                while (a <= z) {
                    const int mid = (a + z) >> 1;
                    const int x = ld[mid].i;
                    if (x == v) return mid;
                    if (x < v) a = mid + 1; else z = mid - 1;
                }
                return -1;
            };
            bool use_q = use_q0;
            float W = 0.f;
            for (int attempt = 0; attempt < 2; ++attempt) {
                for (int e = lane; e < nt; e += 32) {
                    // entries below a row's threshold (a nucleus cut) weigh nothing
                    const float pt = lt[e].v >= t_cut ? ex2(fmaf(lt[e].v, c, -t_msc)) * t_inv : 0.f;
                    float w = pt;
                    if (use_q) {
                        const int pd = find(lt[e].i);
                        const float q = (pd >= 0 && ld[pd].v >= d_cut) ? ex2(fmaf(ld[pd].v, c, -d_msc)) * d_inv : 0.f;
                        w = fmaxf(pt - q, 0.f);
                    }
                    wv[e] = w;
                }
                __syncwarp();
                W = 0.f;
                for (int base = 0; base < nt; base += 32) {
                    const float w = (base + lane < nt) ? wv[base + lane] : 0.f;
                    const float incl = warp_incl_scan(w, lane);
                    W += __shfl_sync(0xffffffffu, incl, 31);
                }
                if (W > 0.f || !use_q) break;
                use_q = false;  // zero residual mass: redraw from p at this position
                __syncwarp();
            }
            const float x = u * W;
            float carry = 0.f;
            int token = -1;
            for (int base = 0; base < nt; base += 32) {
                const float w = (base + lane < nt) ? wv[base + lane] : 0.f;
                const float incl = warp_incl_scan(w, lane);
                const unsigned hit = __ballot_sync(0xffffffffu, base + lane < nt && carry + incl > x);
                if (hit) {
                    token = lt[base + __ffs(hit) - 1].i;
                    break;
                }
                carry += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (token < 0) {  // rounding: the last entry with positive weight
                int lastp = -1;
                for (int base = 0; base < nt; base += 32) {
                    const float w = (base + lane < nt) ? wv[base + lane] : 0.f;
                    const unsigned pos = __ballot_sync(0xffffffffu, w > 0.f);
                    if (pos) lastp = base + 31 - __clz(pos);
                }
                token = lastp >= 0 ? lt[lastp].i : -1;
            }
            // outputs
            const bool err = token < 0;
            if (P.sample_only) {
                if (lane == 0) P.out_tokens[b] = err ? -1 : token;
            } else {
                int32_t* out = P.out_tokens + b * (k + 1);
                for (int i = lane; i <= k; i += 32) out[i] = err ? -1 : (i < j ? dtok[i] : (i == j ? token : -1));
                if (lane == 0) P.out_n[b] = err ? -1 : j;
            }
            return;
        }
    }

    // ---- phase 1: per-row statistics (one warp per row) ----------------------------
    for (int rr = warp; rr < nrows; rr += NW) {
        const long long r = row_index(rr);
        const int d = row_dtok(rr);
        RowStat st;
        st.tau = NEG_INF;
        st.zd = __int_as_float(0x7fc00000);
        st.arg = -1;
        st.err = 0;
        st.slow = 0;
        st.pad = 0;
        st.invS = 0.f;
        int tmo = 0;
        if (greedy) {
            float best = NEG_INF, mx = NEG_INF;
            int bi = -1;
            for (int s = lane; s < P.nch; s += 32) {  // one record per chunk
                const SegRec g = P.segs[r * P.nseg + s];
                tmo |= g.flags & REC_TIMEOUT;
                mx = fmax_nan(mx, g.m);
                if (arg_better(g.m, g.arg, best, bi)) {
                    best = g.m;
                    bi = g.arg;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ob = __shfl_xor_sync(0xffffffffu, best, o);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                if (arg_better(ob, oi, best, bi)) {
                    best = ob;
                    bi = oi;
                }
                mx = fmax_nan(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            }
            st.msc = mx;
            st.arg = bi;
            if (mx != mx || mx == POS_INF || bi < 0) st.err = 1;
        } else if (P.mode == MODE_SOFTMAX) {
            // the draft-token logit load is issued before the partials are combined
            if (d >= 0 && d < V) st.zd = proc_logit(load_elem<DT>(row_ptr(rr), d), d, pv);
            float m = NEG_INF, s = 0.f;
            for (int q = lane; q < P.nseg; q += 32) {
                const SegRec g = P.segs[r * P.nseg + q];
                tmo |= g.flags & REC_TIMEOUT;
                ms_combine(m, s, g.m, g.s);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                ms_combine(m, s, __shfl_xor_sync(0xffffffffu, m, o), __shfl_xor_sync(0xffffffffu, s, o));
            st.msc = m;
            st.invS = 1.f / s;
            if (m != m || m == POS_INF || m == NEG_INF || s != s) st.err = 1;
            if (tp < 1.f && P.nuc && !st.err) {
                // the nucleus kernel's cut: kept iff z >= cut, renormalised
                const NucRec nr = P.nuc[r];
                st.tau = nr.cut;
                st.invS = nr.invS;
                if (!(nr.invS > 0.f && nr.invS < POS_INF)) st.err = 1;
            }
        } else {
            // top-k: raw maximum over the chunks, then the kept set
            float mx = NEG_INF;
            if (P.pre) {
                const ChunkRec& g = prec[rr];
                tmo |= g.flags & REC_TIMEOUT;
                mx = g.m;
            } else for (int q = lane; q < P.nch; q += 32) {
                if (P.mode == MODE_TOPK) {
                    const ChunkRec g = P.chunks[r * P.nch + q];
                    tmo |= g.flags & REC_TIMEOUT;
                    mx = fmax_nan(mx, g.m);
                } else {
                    const SegRec g = P.segs[r * P.nseg + q];
                    tmo |= g.flags & REC_TIMEOUT;
                    mx = fmax_nan(mx, g.m);
                }
            }
            mx = warp_max_nan(mx);
            st.msc = mx * c;
            if (mx != mx || mx == POS_INF || mx == NEG_INF) st.err = 1;
            if (P.mode == MODE_MAXONLY) {
                st.slow = 1;
            } else if (!st.err) {
                float G = NEG_INF;
                int ovf = 0;
                for (int ch = lane; ch < P.nch; ch += 32) {
                    const ChunkRec cr = P.pre ? prec[rr] : P.chunks[r * P.nch + ch];
                    G = fmaxf(G, cr.tau);
                    tmo |= cr.flags & REC_TIMEOUT;
                    ovf |= cr.flags & REC_OVERFLOW;
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) G = fmaxf(G, __shfl_xor_sync(0xffffffffu, G, o));
                ovf = __any_sync(0xffffffffu, ovf);
                Cand* buf = gbuf + static_cast<size_t>(warp) * P.mg;
                int ng = 0;
                if (P.nch == 1 && !ovf) {
                    // one chunk: its header already holds tau, the sum and the draft logit
                    const ChunkRec cr = P.pre ? prec[rr] : P.chunks[r];
                    st.tau = cr.tau;
                    st.invS = 1.f / cr.s;
                    st.zd = cr.zd;
                } else if (!ovf) {
                    ng = gather(r, G, buf, P.mg);
                }
                if (P.nch == 1 && !ovf) {
                    // done
                } else if (ovf || ng > P.mg) {
                    st.slow = 1;
                } else {
                    __syncwarp();
                    float tau = G;
                    if (P.nch > 1) {
                        float cand = NEG_INF;
                        for (int e = lane; e < ng; e += 32) {
                            const float x = buf[e].v;
                            int gt = 0, ge = 0;
                            for (int q = 0; q < ng; ++q) {
                                const float y = buf[q].v;
                                gt += (y > x);
                                ge += (y >= x);
                            }
                            if (gt < K && K <= ge) cand = x;
                        }
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) cand = fmaxf(cand, __shfl_xor_sync(0xffffffffu, cand, o));
                        tau = cand;
                    }
                    float acc = 0.f, zd = NEG_INF;
                    for (int e = lane; e < ng; e += 32) {
                        const Cand cd = buf[e];
                        if (cd.v >= tau) {
                            acc += ex2(fmaf(cd.v, c, -st.msc));
                            if (cd.i == d) zd = cd.v;
                        }
                    }
                    acc = warp_sum(acc);
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) zd = fmaxf(zd, __shfl_xor_sync(0xffffffffu, zd, o));
                    st.tau = tau;
                    st.invS = 1.f / acc;
                    st.zd = zd;  // -inf: the draft token is not kept (probability 0)
                }
                if (tp < 1.f && !st.err && !st.slow) {  // slow rows: after their radix select
                    {
                        // Nucleus over the kept set: the cut is the largest kept value
                        // x whose tail mass (probabilities of the values >= x) reaches
                        // top_p; every value >= x is kept and renormalised.
                        const Cand* L = buf;
                        int n = ng;
                        if (P.pre) {
                            L = plist + static_cast<size_t>(rr) * P.kcap;
                            n = prec[rr].n;
                        } else if (P.nch == 1) {
                            n = min(gather(r, st.tau, buf, P.mg), P.mg);
                            __syncwarp();
                        }
                        float cand = NEG_INF;
                        for (int e = lane; e < n; e += 32) {
                            const float x = L[e].v;
                            if (!(x >= st.tau)) continue;
                            float mass = 0.f;
                            for (int f = 0; f < n; ++f) {
                                const float y = L[f].v;
                                if (y >= x && y >= st.tau) mass += ex2(fmaf(y, c, -st.msc)) * st.invS;
                            }
                            if (mass >= tp) cand = fmaxf(cand, x);
                        }
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) cand = fmaxf(cand, __shfl_xor_sync(0xffffffffu, cand, o));
                        const float cut = fmaxf(cand, st.tau);
                        float acc = 0.f;
                        for (int e = lane; e < n; e += 32)
                            if (L[e].v >= cut) acc += ex2(fmaf(L[e].v, c, -st.msc));
                        acc = warp_sum(acc);
                        st.tau = cut;
                        st.invS = 1.f / acc;
                    }
                }
            }
        }
        tmo = __any_sync(0xffffffffu, tmo);
        if (tmo) st.err = 2;
        if (lane == 0) rs[rr] = st;
    }
    __syncthreads();

    // ---- phase 1b: exact top-k threshold of rows that need it (rare) --------------
    if (!greedy && P.mode != MODE_SOFTMAX) {
        for (int rr = 0; rr < nrows; ++rr) {
            if (!rs[rr].slow || rs[rr].err) continue;  // uniform: read after a barrier
            const void* row = row_ptr(rr);
            // bf16 logits have 16-bit keys; penalised ones are fp32 values
            const int ROUNDS = (DT == 0 && !pv.allow) ? 2 : 4;
            if (tid == 0) {
                S.radix_prefix = 0u;
                S.radix_k = K;
            }
            for (int round = 0; round < ROUNDS; ++round) {
                const int shift = 24 - 8 * round;
                for (int q = tid; q < 256; q += NT) S.hist[q] = 0;
                __syncthreads();
                const uint32_t pre = S.radix_prefix;
                for (int e = tid; e < V; e += NT) {
                    const uint32_t key = okey(proc_logit(load_elem<DT>(row, e), e, pv));
                    if (round == 0 || (key >> (shift + 8)) == pre) atomicAdd(&S.hist[(key >> shift) & 255u], 1);
                }
                __syncthreads();
                if (tid == 0) {
                    int kr = S.radix_k, cum = 0, digit = 0;
                    for (int bin = 255; bin >= 0; --bin) {
                        const int cnt = S.hist[bin];
                        if (cum + cnt >= kr) {
                            digit = bin;
                            kr -= cum;
                            break;
                        }
                        cum += cnt;
                    }
                    S.radix_prefix = (S.radix_prefix << 8) | static_cast<uint32_t>(digit);
                    S.radix_k = kr;
                }
                __syncthreads();
            }
            float tau;
            if (ROUNDS == 2)
                tau = okey_inv(S.radix_prefix << 16 | ((S.radix_prefix & 0x8000u) ? 0u : 0xffffu));
            else
                tau = okey_inv(S.radix_prefix);
            const float msc = rs[rr].msc;
            float acc = 0.f;
            for (int e = tid; e < V; e += NT) {
                const float z = proc_logit(load_elem<DT>(row, e), e, pv);
                if (z >= tau) acc += ex2(fmaf(z, c, -msc));
            }
            acc = warp_sum(acc);
            if (lane == 0) S.red_f[warp][0] = acc;
            __syncthreads();
            if (tid == 0) {
                float s = 0.f;
                for (int w = 0; w < NW; ++w) s += S.red_f[w][0];
                rs[rr].tau = tau;
                rs[rr].invS = 1.f / s;
                const int d = row_dtok(rr);
                rs[rr].zd = (d >= 0 && d < V) ? proc_logit(load_elem<DT>(row, d), d, pv) : __int_as_float(0x7fc00000);
            }
            __syncthreads();
            if (tp > 0.f && tp < 1.f) {
                // the nucleus over the row's kept set {z >= tau}
                float cut, inv;
                nucleus_block<DT, NT>(row, V, rs[rr].tau, rs[rr].msc, c, tp, pv, S.nuc, cut, inv);
                if (tid == 0) {
                    rs[rr].tau = fmaxf(cut, rs[rr].tau);
                    rs[rr].invS = inv;
                    if (!(inv > 0.f && inv < POS_INF)) rs[rr].err = 1;
                }
                __syncthreads();
            }
        }
    }

    // ---- phase 2: decisions (warp 0, one lane per position) ----------------------------
    if (warp == 0) {
        int err = S.err, tmo = 0;
        for (int rr = lane; rr < nrows; rr += 32) {
            if (rs[rr].err) err = 1;
            if (rs[rr].err == 2) tmo = 1;
        }
        err = __any_sync(0xffffffffu, err);
        tmo = __any_sync(0xffffffffu, tmo);
        int j = k;
        for (int i0 = 0; i0 < k; i0 += 32) {
            const int i = i0 + lane;
            bool rej = false;
            if (i < k) {
                if (greedy) {
                    rej = !err && dtok[i] != rs[i].arg;
                } else if (!err) {
                    const RowStat& t = rs[i];
                    const RowStat& dd = rs[k + 1 + i];
                    const float p = (t.zd >= t.tau) ? ex2(fmaf(t.zd, c, -t.msc)) * t.invS : 0.f;
                    const float q = (dd.zd >= dd.tau) ? ex2(fmaf(dd.zd, c, -dd.msc)) * dd.invS : 0.f;
                    if (P.out_p) P.out_p[b * k + i] = p;
                    if (P.out_q) P.out_q[b * k + i] = q;
                    rej = !(uu[i] * q < p);
                } else {
                    if (P.out_p) P.out_p[b * k + i] = __int_as_float(0x7fc00000);
                    if (P.out_q) P.out_q[b * k + i] = __int_as_float(0x7fc00000);
                }
            }
            const unsigned m = __ballot_sync(0xffffffffu, rej);
            if (m && j == k) j = i0 + __ffs(m) - 1;  // the first rejection
        }
        if (lane == 0) {
            if (!err && greedy) S.token = rs[j].arg;
            if (tmo && P.out_status) atomicExch(P.out_status, -4);
            S.err = err;
            S.j = j;
        }
    }
    __syncthreads();

    // ---- phase 3: the draw -------------------------------------------------------------
    if (!greedy && !S.err) {
        const int j = S.j;
        const RowStat tst = rs[j];
        const bool use_q0 = j < k;
        const RowStat dst = use_q0 ? rs[k + 1 + j] : tst;
        const float u = uu[k];
        const bool list_draw = P.mode == MODE_TOPK && !tst.slow && !(use_q0 && dst.slow);
        if (list_draw) {
            Cand* lt = gbuf;
            Cand* ld = gbuf + P.mg;
            int nt = 0, nd = 0;
            if (P.pre) {
                // one chunk per row: the kept lists are complete, index-sorted and in shared memory
                lt = plist + static_cast<size_t>(j) * P.kcap;
                nt = prec[j].n;
                if (use_q0) {
                    ld = plist + static_cast<size_t>(k + 1 + j) * P.kcap;
                    nd = prec[k + 1 + j].n;
                }
            } else {
                if (warp == 0) nt = gather(row_index(j), tst.tau, lt, P.mg);
                if (warp == 1 && use_q0) nd = gather(row_index(k + 1 + j), dst.tau, ld, P.mg);
                if (warp == 0 && lane == 0) S.red_i[0] = nt;
                if (warp == 1 && lane == 0) S.red_i[1] = nd;
                __syncthreads();
                nt = S.red_i[0];  // every thread takes part in the weights below
                nd = S.red_i[1];
            }
            // weights of the target entries, computed once by all threads
            float* wv = reinterpret_cast<float*>(P.pre ? gbuf : gbuf + 2 * P.mg);
            auto find = [&](int v) {
                int a = 0, z = nd - 1;
                while (a <= z) {
                    const int mid = (a + z) >> 1;
                    const int x = ld[mid].i;
                    if (x == v) return mid;
                    if (x < v) a = mid + 1; else z = mid - 1;
                }
                return -1;
            };
            bool use_q = use_q0;
            for (int attempt = 0; attempt < 2; ++attempt) {
                for (int e = tid; e < nt; e += NT) {
                    // entries below a row's threshold (a nucleus cut) weigh nothing
                    const float pt = lt[e].v >= tst.tau ? ex2(fmaf(lt[e].v, c, -tst.msc)) * tst.invS : 0.f;
                    float w = pt;
                    if (use_q) {
                        const int pd = find(lt[e].i);
                        const float q = (pd >= 0 && ld[pd].v >= dst.tau) ? ex2(fmaf(ld[pd].v, c, -dst.msc)) * dst.invS
                                                                          : 0.f;
                        w = fmaxf(pt - q, 0.f);
                    }
                    wv[e] = w;
                }
                __syncthreads();
                if (warp == 0) {
                    float W = 0.f;
                    for (int base = 0; base < nt; base += 32) {
                        const float w = (base + lane < nt) ? wv[base + lane] : 0.f;
                        const float incl = warp_incl_scan(w, lane);
                        W += __shfl_sync(0xffffffffu, incl, 31);
                    }
                    if (lane == 0) S.W = W;
                }
                __syncthreads();
                if (S.W > 0.f || !use_q) break;
                use_q = false;  // zero residual mass: redraw from p at this position
                __syncthreads();
            }
            if (warp == 0) {
                const float x = u * S.W;
                float carry = 0.f;
                int token = -1;
                for (int base = 0; base < nt; base += 32) {
                    const float w = (base + lane < nt) ? wv[base + lane] : 0.f;
                    const float incl = warp_incl_scan(w, lane);
                    const unsigned hit = __ballot_sync(0xffffffffu, base + lane < nt && carry + incl > x);
                    if (hit) {
                        token = lt[base + __ffs(hit) - 1].i;
                        break;
                    }
                    carry += __shfl_sync(0xffffffffu, incl, 31);
                }
                if (token < 0) {  // rounding: the last entry with positive weight
                    int lastp = -1;
                    for (int base = 0; base < nt; base += 32) {
                        const float w = (base + lane < nt) ? wv[base + lane] : 0.f;
                        const unsigned pos = __ballot_sync(0xffffffffu, w > 0.f);
                        if (pos) lastp = base + 31 - __clz(pos);
                    }
                    token = lastp >= 0 ? lt[lastp].i : -1;
                }
                if (lane == 0) S.token = token;
            }
            __syncthreads();
        } else if (P.defer && use_q0) {
            // residual draw: handed to the segment kernel (one CTA per segment)
            if (tid == 0) {
                DrawReq q;
                q.need = 1;
                q.j = j;
                q.use_q = 1;
                q.pad0 = 0;
                q.rowt = b * (k + 1) + j;
                q.rowd = b * k + j;
                q.t_msc = tst.msc;
                q.t_invS = tst.invS;
                q.t_tau = tst.tau;
                q.d_msc = dst.msc;
                q.d_invS = dst.invS;
                q.d_tau = dst.tau;
                q.u = u;
                q.c = c;
                P.req[b] = q;
                P.counter[b] = 0;
                S.token = INT_MAX;  // written by the segment kernel
            }
            __syncthreads();
        } else {
            // streaming draw over the row(s): per-segment masses, then one segment
            const void* rowt = row_ptr(j);
            const void* rowd = use_q0 ? row_ptr(k + 1 + j) : nullptr;
            const bool alt = (reinterpret_cast<uintptr_t>(rowt) & 15u) == 0;
            const bool ald = rowd && (reinterpret_cast<uintptr_t>(rowd) & 15u) == 0;
            const int vps = P.seg / VEC;                      // vectors per segment
            const int nvec = (V + VEC - 1) / VEC;
            bool use_q = use_q0;
            auto wt = [&](float zt, float zdv) {
                const float pt = (zt >= tst.tau) ? ex2(fmaf(zt, c, -tst.msc)) * tst.invS : 0.f;
                if (!use_q) return pt;
                const float qd = (zdv >= dst.tau) ? ex2(fmaf(zdv, c, -dst.msc)) * dst.invS : 0.f;
                return fmaxf(pt - qd, 0.f);
            };
            auto vec_w = [&](int q, float* w) {
                float vt[VEC], vd[VEC];
                load_vec<DT>(rowt, alt, q, V, vt);
                if (use_q) load_vec<DT>(rowd, ald, q, V, vd);
                if (pv.allow) {
#pragma unroll
                    for (int t = 0; t < VEC; ++t) {
                        const long long v = static_cast<long long>(q) * VEC + t;
                        if (v < V) {
                            vt[t] = proc_logit(vt[t], v, pv);
                            if (use_q) vd[t] = proc_logit(vd[t], v, pv);
                        }
                    }
                }
#pragma unroll
                for (int t = 0; t < VEC; ++t) w[t] = wt(vt[t], use_q ? vd[t] : NEG_INF);
            };
            // masses known from the streaming pass: a plain (unmasked) bonus draw
            const bool known = P.mode == MODE_SOFTMAX && !use_q0 && !(tp < 1.f);
            for (int attempt = 0; attempt < 2; ++attempt) {
                if (known) {
                    for (int s = tid; s < P.nseg; s += NT) {
                        const SegRec g = P.segs[row_index(j) * P.nseg + s];
                        mass[s] = g.s * ex2(g.m - tst.msc) * tst.invS;
                    }
                } else {
                    for (int s = 0; s < P.nseg; ++s) {
                        float acc = 0.f;
                        for (int q = s * vps + tid; q < min(nvec, (s + 1) * vps); q += NT) {
                            float w[VEC];
                            vec_w(q, w);
#pragma unroll
                            for (int t = 0; t < VEC; ++t) acc += w[t];
                        }
                        acc = warp_sum(acc);
                        if (lane == 0) part[s * NW + warp] = acc;
                    }
                    __syncthreads();
                    for (int s = tid; s < P.nseg; s += NT) {
                        float a = 0.f;
                        for (int w = 0; w < NW; ++w) a += part[s * NW + w];
                        mass[s] = a;
                    }
                }
                __syncthreads();
                if (tid == 0) {
                    float W = 0.f;
                    for (int s = 0; s < P.nseg; ++s) W += mass[s];
                    S.retry = (!(W > 0.f) && use_q) ? 1 : 0;
                    const float x = u * W;
                    int sel = -1, lastm = 0;
                    float a = 0.f, base = 0.f;
                    for (int s = 0; s < P.nseg; ++s) {
                        const float nxt = a + mass[s];
                        if (nxt > x) {
                            sel = s;
                            base = a;
                            break;
                        }
                        a = nxt;
                    }
                    if (sel < 0) {
                        lastm = 1;
                        for (int s = P.nseg - 1; s >= 0; --s)
                            if (mass[s] > 0.f) {
                                sel = s;
                                break;
                            }
                    }
                    S.W = W;
                    S.x = x;
                    S.base = base;
                    S.seg_sel = sel;
                    S.last_mode = lastm;
                    S.tok_cross = -1;
                    S.tok_last = -1;
                }
                __syncthreads();
                if (!S.retry) break;
                use_q = false;  // zero residual mass: redraw from p at this position
                __syncthreads();
            }
            const int sel = S.seg_sel;
            if (sel >= 0) {
                const float x = S.x;
                float base = S.base;
                const bool lastm = S.last_mode != 0;
                const int q0 = sel * vps, q1 = min(nvec, (sel + 1) * vps);
                for (int tq = q0; tq < q1; tq += NT) {  // tiles of NT vectors, in index order
                    const int q = tq + tid;
                    float w[VEC];
                    float vs = 0.f;
                    if (q < q1) {
                        vec_w(q, w);
#pragma unroll
                        for (int t = 0; t < VEC; ++t) vs += w[t];
                    } else {
#pragma unroll
                        for (int t = 0; t < VEC; ++t) w[t] = 0.f;
                    }
                    int lastpos = -1;
#pragma unroll
                    for (int t = 0; t < VEC; ++t)
                        if (w[t] > 0.f) lastpos = q * VEC + t;
                    if (lastpos >= 0) atomicMax(&S.tok_last, lastpos);
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
                    const float wp = S.red_f[warp][1];
                    const float tile_tot = S.red_f[NW - 1][1] + S.red_f[NW - 1][0];
                    if (!lastm && S.tok_cross < 0) {
                        const float incl = base + (wp + inw);
                        const float excl = base + (wp + exw);
                        if (excl <= x && x < incl) {
                            float acc = excl;
                            int tok = -1;
#pragma unroll
                            for (int t = 0; t < VEC; ++t) {
                                if (tok < 0 && w[t] > 0.f) {
                                    const float nacc = acc + w[t];
                                    if (nacc > x) tok = q * VEC + t;
                                    acc = nacc;
                                }
                            }
                            if (tok < 0) tok = lastpos;
                            S.tok_cross = tok;
                        }
                    }
                    base = base + tile_tot;
                    __syncthreads();
                }
                if (tid == 0) S.token = S.tok_cross >= 0 ? S.tok_cross : S.tok_last;
            } else if (tid == 0) {
                S.token = -1;
            }
            __syncthreads();
        }
    }

    // ---- phase 4: outputs --------------------------------------------------------------
    if (tid == 0) {
        int err = S.err;
        const int j = S.j;
        const bool deferred = !err && !greedy && S.token == INT_MAX;
        if (P.defer && !deferred) P.req[b].need = 0;
        if (deferred) {
            int32_t* out = P.out_tokens + b * (k + 1);
            for (int i = 0; i <= k; ++i) out[i] = i < j ? dtok[i] : -1;
            P.out_n[b] = j;
            return;
        }
        const int y = err ? -1 : S.token;
        if (y < 0) err = 1;
        if (P.sample_only) {
            P.out_tokens[b] = err ? -1 : y;
        } else {
            int32_t* out = P.out_tokens + b * (k + 1);
            for (int i = 0; i <= k; ++i) out[i] = (!err && i < j) ? dtok[i] : -1;
            if (!err) out[j] = y;
            P.out_n[b] = err ? -1 : j;
        }
    }
}

}  // namespace sv
