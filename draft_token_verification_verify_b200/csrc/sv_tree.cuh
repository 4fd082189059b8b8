// KT — tree verification: one CTA per sequence walks its candidate tree.
//
// Candidate trees are named in section "提议方式与实现形态", paragraph 3, of
// the speculative decoding entry "推测解码"; the pages give no acceptance rule
// for them.  The rule taken is the one that reduces to section
// "提议与核验的基本步骤", paragraph 2, on a chain: at the current node the
// children are tried in index order against the current distribution R (the
// node's processed target row p, then, after each rejection, the normalised
// residual max(0, R - q) with q the node's processed draft row; a residual of
// no mass leaves R as it is); child c is accepted iff u_c * q(t_c) < R(t_c)
// and the walk continues from it; when no child is accepted the final token
// is drawn from R by the inverse CDF with the last uniform.  Greedy: the first
// child whose token is the node's lowest-index argmax, else that argmax.
//
// Two paths.  With top-k (or greedy) and a workspace, the streaming pass (K1)
// first runs over every target and draft row of the trees, and the list walk
// (sv_tree_list_kernel) takes each visited node's statistics and kept list
// from its records: the probabilities, every residual and the final draw live
// on the kept lists, so the walk reads no logits.  A sequence whose records
// are incomplete (a list that overflowed, a wait that ran out) and every
// sequence of the other cases go through the row walk (sv_tree_kernel).
//
// Row walk: only the rows of visited nodes are read.  Per visited node the CTA streams
// the target and draft rows: their maxima (and raw NaN / +inf), the exact
// top-k threshold by a radix select over order-preserving keys when top-k is
// on, and the normalisers; one more pass over the pair per rejection (the
// residual's mass); the final draw sums the weights per segment and rescans
// one segment.  The residual after m rejections is evaluated element by
// element from p, q and the m masses.  No workspace: everything is in shared
// memory.
#pragma once

#include "sv_common.cuh"
#include "sv_nucleus.cuh"  // load_vec
#include "sv_rows.cuh"     // record flags

namespace sv {

constexpr int TREE_NT = 256;
constexpr int TREE_NW = TREE_NT / 32;
constexpr int TREE_MAX_NODES = 256;  // N, nodes besides the root
constexpr int TREE_SEG = 4096;       // elements per segment of the final draw
constexpr int TREE_MAX_SEG = 64;     // segments (V <= 262,144)

struct TreeParams {
    const void* target;        // [B][N+1][V]
    const void* draft;         // [B][N+1][V] or null (greedy)
    const int32_t* tokens;     // [B][N] token of node n at n - 1
    const int32_t* parents;    // [B][N] parent of node n at n - 1 (in [0, n))
    const float* uniforms;     // [B][N+1] or null (greedy)
    const float* temperature;  // [B] or null
    long long B;
    int N;
    int V;
    int top_k;                 // effective K (0: none)
    int greedy;
    int32_t* out_tokens;       // [B][N+1]
    int32_t* out_n;            // [B]
    int32_t* out_nodes;        // [B][N+1] or null
    float* out_p;              // [B][N] or null: R(t_c) of each tested child, NaN if untested
    float* out_q;              // [B][N] or null: q(t_c), NaN if untested
    const int* done;           // [B] or null: sequences the list walk has finished (skipped here)
};

struct TreeRow {
    float msc;   // maximum of z*c over the row (the maximum is always kept)
    float tau;   // kept iff z >= tau
    float invS;  // 1 / sum of 2^(z*c - msc) over the kept entries
    int err;
};

struct __align__(16) TreeCtl {
    int tok[TREE_MAX_NODES];
    int par[TREE_MAX_NODES];
    float W[TREE_MAX_NODES];     // masses of the residual levels of the current node
    float mass[TREE_MAX_SEG];
    int hist[256];
    float red[TREE_NW];
    float red2[TREE_NW];
    int redi[TREE_NW];
    TreeRow rt, rd;
    uint32_t prefix;
    int krem;
    int err;
    int token;
    int seg;
    float x;
};

template <int DT>
__global__ void __launch_bounds__(TREE_NT, 1) sv_tree_kernel(const TreeParams P) {
    constexpr int VEC = VT<DT>::VEC;
    constexpr int ELT = VT<DT>::ELT;
    constexpr int NT = TREE_NT, NW = TREE_NW;
    __shared__ TreeCtl S;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long b = blockIdx.x;
    if (P.done && P.done[b]) return;  // uniform over the CTA
    const int N = P.N, V = P.V, K = P.top_k;
    const int nvec = (V + VEC - 1) / VEC;
    const bool greedy = P.greedy != 0;
    const float* u = greedy ? nullptr : P.uniforms + b * (N + 1);
    float T = 1.f;
    if (!greedy && P.temperature) T = P.temperature[b];
    const float c = (T > 0.f && T != POS_INF) ? LOG2E / T : 1.f;
    auto row_of = [&](const void* base, int node) {
        return static_cast<const char*>(base) + (static_cast<size_t>(b) * (N + 1) + node) * static_cast<size_t>(V) * ELT;
    };

    // ---- inputs of the whole tree ----------------------------------------------------
    if (tid == 0) S.err = 0;
    __syncthreads();
    for (int i = tid; i < N; i += NT) {
        const int t = P.tokens[b * N + i], p = P.parents[b * N + i];
        S.tok[i] = t;
        S.par[i] = p;
        if (t < 0 || t >= V || p < 0 || p > i) S.err = 1;
        if (P.out_p) P.out_p[b * N + i] = __int_as_float(0x7fc00000);  // NaN: not tested
        if (P.out_q) P.out_q[b * N + i] = __int_as_float(0x7fc00000);
    }
    if (!greedy) {
        if (tid == 0 && !(T > 0.f && T != POS_INF)) S.err = 1;
        for (int i = tid; i <= N; i += NT)
            if (!(u[i] >= 0.f && u[i] < 1.f)) S.err = 1;
    }
    __syncthreads();

    // block-wide sum of one float per thread, in a fixed order
    auto block_sum = [&](float v) -> float {
        v = warp_sum(v);
        if (lane == 0) S.red[warp] = v;
        __syncthreads();
        float s = 0.f;
        for (int w = 0; w < NW; ++w) s += S.red[w];
        __syncthreads();
        return s;
    };
    // f(e0, zt[VEC], zd[VEC]) over every vector of the pair of rows (zd unused
    // when rd is null), four vector loads per row in flight per thread;
    // elements past V read as -inf
    auto for_pair = [&](const void* rt, const void* rd, auto&& f) {
        constexpr int U = 4;
        const bool at = (reinterpret_cast<uintptr_t>(rt) & 15u) == 0;
        const bool ad = rd && (reinterpret_cast<uintptr_t>(rd) & 15u) == 0;
        for (int q0 = tid; q0 < nvec; q0 += NT * U) {
            uint4 wt[U], wd[U];
#pragma unroll
            for (int k2 = 0; k2 < U; ++k2) {
                const int q = q0 + k2 * NT;
                const bool whole = q < nvec && static_cast<long long>(q + 1) * VEC <= V;
                if (at && whole) wt[k2] = __ldg(reinterpret_cast<const uint4*>(rt) + q);
                if (rd && ad && whole) wd[k2] = __ldg(reinterpret_cast<const uint4*>(rd) + q);
            }
#pragma unroll
            for (int k2 = 0; k2 < U; ++k2) {
                const int q = q0 + k2 * NT;
                if (q >= nvec) continue;
                const bool whole = static_cast<long long>(q + 1) * VEC <= V;
                float zt[VEC], zd[VEC];
                if (at && whole)
                    unpack<DT>(wt[k2], zt);
                else
                    load_vec<DT>(rt, false, q, V, zt);
                if (rd) {
                    if (ad && whole)
                        unpack<DT>(wd[k2], zd);
                    else
                        load_vec<DT>(rd, false, q, V, zd);
                }
                f(q * VEC, zt, zd);
            }
        }
    };
    // statistics of one processed row (stochastic)
    auto row_stats = [&](const void* row, TreeRow& out) {
        float mx = NEG_INF;
        int bad = 0;
        for_pair(row, nullptr, [&](int, const float* z, const float*) {
#pragma unroll
            for (int t = 0; t < VEC; ++t) {
                mx = fmax_nan(mx, z[t]);
                if (!(z[t] == z[t]) || z[t] == POS_INF) bad = 1;
            }
        });
        mx = warp_max_nan(mx);
        bad = __any_sync(0xffffffffu, bad);
        if (lane == 0) {
            S.red[warp] = mx;
            S.redi[warp] = bad;
        }
        __syncthreads();
        if (tid == 0) {
            float m = NEG_INF;
            int e = 0;
            for (int w = 0; w < NW; ++w) {
                m = fmax_nan(m, S.red[w]);
                e |= S.redi[w];
            }
            out.msc = m * c;
            out.tau = NEG_INF;
            out.err = e || !(m > NEG_INF);
        }
        __syncthreads();
        if (out.err) return;
        if (K > 0 && K < V) {
            // tau = K-th largest raw logit with multiplicity (radix select, 8 bits a pass)
            const int rounds = DT == 0 ? 2 : 4;
            if (tid == 0) {
                S.prefix = 0u;
                S.krem = K;
            }
            for (int round = 0; round < rounds; ++round) {
                const int shift = 24 - 8 * round;
                for (int h = tid; h < 256; h += NT) S.hist[h] = 0;
                __syncthreads();
                const uint32_t pre = S.prefix;
                for_pair(row, nullptr, [&](int, const float* z, const float*) {
#pragma unroll
                    for (int t = 0; t < VEC; ++t) {
                        const uint32_t key = okey(z[t]);
                        const bool in = z[t] == z[t] && (round == 0 || (key >> (shift + 8)) == pre);
                        const int bin = in ? static_cast<int>((key >> shift) & 255u) : -1;
                        // one atomic per distinct bin of the warp
                        const unsigned peers = __match_any_sync(__activemask(), bin);
                        if (in && lane == __ffs(peers) - 1) atomicAdd(&S.hist[bin], __popc(peers));
                    }
                });
                __syncthreads();
                if (tid == 0) {
                    int cum = 0, kr = S.krem, digit = 0;
                    for (int h = 255; h >= 0; --h) {
                        if (cum + S.hist[h] >= kr) {
                            digit = h;
                            kr -= cum;
                            break;
                        }
                        cum += S.hist[h];
                    }
                    S.prefix = (S.prefix << 8) | static_cast<uint32_t>(digit);
                    S.krem = kr;
                }
                __syncthreads();
            }
            if (tid == 0) {
                const uint32_t p = S.prefix;
                out.tau = okey_inv(rounds == 2 ? (p << 16 | ((p & 0x8000u) ? 0u : 0xffffu)) : p);
            }
            __syncthreads();
        }
        const float msc = out.msc, tau = out.tau;
        float acc = 0.f;
        for_pair(row, nullptr, [&](int, const float* z, const float*) {
#pragma unroll
            for (int t = 0; t < VEC; ++t)
                if (z[t] >= tau) acc += ex2(fmaf(z[t], c, -msc));
        });
        const float s = block_sum(acc);
        if (tid == 0) out.invS = 1.f / s;
        __syncthreads();
    };
    auto prob = [&](float z, const TreeRow& r) { return z >= r.tau ? ex2(fmaf(z, c, -r.msc)) * r.invS : 0.f; };

    int a = 0, depth = 0, y = -1;
    int err = S.err;
    while (!err) {
        const char* rt = row_of(P.target, a);
        int next = 0;
        if (greedy) {
            // lowest-index argmax of the target row (NaN or +inf: an error)
            float best = NEG_INF;
            int bi = INT_MAX, bad = 0;
            for_pair(rt, nullptr, [&](int e0, const float* z, const float*) {
#pragma unroll
                for (int t = 0; t < VEC; ++t) {
                    if (!(z[t] == z[t]) || z[t] == POS_INF) bad = 1;
                    if (e0 + t < V && (z[t] > best || (z[t] == best && e0 + t < bi))) {
                        best = z[t];
                        bi = e0 + t;
                    }
                }
            });
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ob = __shfl_xor_sync(0xffffffffu, best, o);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                if (ob > best || (ob == best && oi < bi)) {
                    best = ob;
                    bi = oi;
                }
            }
            bad = __any_sync(0xffffffffu, bad);
            if (lane == 0) {
                S.red[warp] = best;
                S.redi[warp] = bi;
                S.red2[warp] = bad ? 1.f : 0.f;
            }
            __syncthreads();
            if (tid == 0) {
                float bv = S.red[0];
                int bx = S.redi[0], e = S.red2[0] != 0.f;
                for (int w = 1; w < NW; ++w) {
                    e |= S.red2[w] != 0.f;
                    if (S.red[w] > bv || (S.red[w] == bv && S.redi[w] < bx)) {
                        bv = S.red[w];
                        bx = S.redi[w];
                    }
                }
                S.err = e || bx == INT_MAX || !(bv > NEG_INF);
                S.token = bx;
            }
            __syncthreads();
            if (S.err) {
                err = 1;
                break;
            }
            const int g = S.token;
            for (int ch = a + 1; ch <= N && !next; ++ch)
                if (S.par[ch - 1] == a && S.tok[ch - 1] == g) next = ch;
            if (!next) {
                y = g;
                break;
            }
        } else {
            const char* rd = row_of(P.draft, a);
            row_stats(rt, S.rt);
            if (!S.rt.err) row_stats(rd, S.rd);
            if (S.rt.err || S.rd.err) {
                err = 1;
                break;
            }
            const TreeRow tr = S.rt, dr = S.rd;
            int levels = 0;  // residual levels of the current distribution
            // current distribution at element z_t / z_d
            auto cur = [&](float zt, float zd) {
                float r = prob(zt, tr);
                const float qv = prob(zd, dr);
                for (int l = 0; l < levels; ++l) r = fmaxf(r - qv, 0.f) / S.W[l];
                return r;
            };
            for (int ch = a + 1; ch <= N; ++ch) {
                if (S.par[ch - 1] != a) continue;
                const int x = S.tok[ch - 1];
                const float zt = load_elem<DT>(rt, x), zd = load_elem<DT>(rd, x);
                const float r = cur(zt, zd), qv = prob(zd, dr);
                if (tid == 0) {
                    if (P.out_p) P.out_p[b * N + ch - 1] = r;
                    if (P.out_q) P.out_q[b * N + ch - 1] = qv;
                }
                if (u[ch - 1] * qv < r) {
                    next = ch;
                    break;
                }
                // rejected: the residual's mass (one pass over the pair)
                float acc = 0.f;
                for_pair(rt, rd, [&](int e0, const float* vt, const float* vd) {
#pragma unroll
                    for (int t = 0; t < VEC; ++t)
                        if (e0 + t < V) acc += fmaxf(cur(vt[t], vd[t]) - prob(vd[t], dr), 0.f);
                });
                const float W = block_sum(acc);
                if (W > 0.f) {
                    if (tid == 0) S.W[levels] = W;
                    __syncthreads();
                    ++levels;
                }
            }
            if (!next) {
                // final draw from the current distribution: segment masses, then one segment
                const int nseg = (V + TREE_SEG - 1) / TREE_SEG;
                const bool at = (reinterpret_cast<uintptr_t>(rt) & 15u) == 0;
                const bool ad = (reinterpret_cast<uintptr_t>(rd) & 15u) == 0;
                constexpr int SV = TREE_SEG / VEC;  // vectors per segment
                // weights of vector q (elements past V weigh nothing)
                auto vec_w = [&](int q, float* w) {
                    float zt[VEC], zd[VEC];
                    load_vec<DT>(rt, at, q, V, zt);
                    load_vec<DT>(rd, ad, q, V, zd);
#pragma unroll
                    for (int t = 0; t < VEC; ++t) w[t] = q * VEC + t < V ? cur(zt[t], zd[t]) : 0.f;
                };
                for (int s = warp; s < nseg; s += NW) {
                    float acc = 0.f;
                    for (int q = s * SV + lane; q < min(nvec, (s + 1) * SV); q += 32) {
                        float w[VEC];
                        vec_w(q, w);
#pragma unroll
                        for (int t = 0; t < VEC; ++t) acc += w[t];
                    }
                    acc = warp_sum(acc);
                    if (lane == 0) S.mass[s] = acc;
                }
                __syncthreads();
                if (tid == 0) {
                    float Wt = 0.f;
                    int lastp = -1;
                    for (int s = 0; s < nseg; ++s) {
                        Wt += S.mass[s];
                        if (S.mass[s] > 0.f) lastp = s;
                    }
                    const float xx = u[N] * Wt;
                    float cum = 0.f;
                    int sel = -1;
                    for (int s = 0; s < nseg; ++s) {
                        if (cum + S.mass[s] > xx) {
                            sel = s;
                            break;
                        }
                        cum += S.mass[s];
                    }
                    if (sel < 0) {  // rounding: the last segment with mass, from its end
                        sel = lastp;
                        cum = 0.f;
                        for (int s = 0; s < sel; ++s) cum += S.mass[s];
                    }
                    S.seg = sel;
                    S.x = xx - cum;
                    S.token = -1;
                }
                __syncthreads();
                if (warp == 0 && S.seg >= 0) {
                    // 32 vectors at a time: a scan over the lanes' sums finds the
                    // lane, that lane walks its elements in index order
                    const int s = S.seg;
                    const float xx = S.x;
                    float carry = 0.f;
                    int token = -1, lastw = -1;
                    for (int q0 = s * SV; q0 < min(nvec, (s + 1) * SV); q0 += 32) {
                        const int q = q0 + lane;
                        float w[VEC];
                        if (q < nvec) {
                            vec_w(q, w);
                        } else {
#pragma unroll
                            for (int t = 0; t < VEC; ++t) w[t] = 0.f;
                        }
                        float ls = 0.f;
                        int lpos = -1;
#pragma unroll
                        for (int t = 0; t < VEC; ++t) {
                            ls += w[t];
                            if (w[t] > 0.f) lpos = q * VEC + t;
                        }
                        const float incl = warp_incl_scan(ls, lane);
                        const unsigned hit = __ballot_sync(0xffffffffu, carry + incl > xx);
                        const unsigned pos = __ballot_sync(0xffffffffu, lpos >= 0);
                        if (pos) lastw = __shfl_sync(0xffffffffu, lpos, 31 - __clz(pos));
                        if (hit) {
                            const int L = __ffs(hit) - 1;
                            int tk = -1;
                            if (lane == L) {
                                float run = carry + incl - ls;  // before this lane's first element
                                int lastp = -1;
#pragma unroll
                                for (int t = 0; t < VEC; ++t) {
                                    if (tk >= 0) continue;
                                    run += w[t];
                                    if (w[t] > 0.f) lastp = q * VEC + t;
                                    if (run > xx) tk = q * VEC + t;
                                }
                                if (tk < 0) tk = lastp;  // rounding inside the lane
                            }
                            token = __shfl_sync(0xffffffffu, tk, L);
                            break;
                        }
                        carry += __shfl_sync(0xffffffffu, incl, 31);
                    }
                    if (lane == 0) S.token = token >= 0 ? token : lastw;
                }
                __syncthreads();
                y = S.token;
                if (y < 0) err = 1;
                break;
            }
        }
        if (tid == 0 && P.out_nodes) P.out_nodes[b * (N + 1) + depth] = next;
        if (tid == 0) P.out_tokens[b * (N + 1) + depth] = S.tok[next - 1];
        ++depth;
        a = next;
    }

    // ---- outputs ------------------------------------------------------------------------
    __syncthreads();
    for (int i = tid; i <= N; i += NT) {
        if (err) {
            P.out_tokens[b * (N + 1) + i] = -1;
            if (P.out_nodes) P.out_nodes[b * (N + 1) + i] = -1;
        } else if (i > depth) {
            P.out_tokens[b * (N + 1) + i] = -1;
            if (P.out_nodes) P.out_nodes[b * (N + 1) + i] = -1;
        } else if (i == depth) {
            P.out_tokens[b * (N + 1) + i] = y;
            if (P.out_nodes) P.out_nodes[b * (N + 1) + i] = -1;
        }
    }
    if (tid == 0) P.out_n[b] = err ? -1 : depth;
}

constexpr int TREE_LIST_NT = 128;
constexpr int TREE_LIST_CAP = 1024;  // kept entries per row (the planner's largest kcap)

struct TreeListParams {
    const ChunkRec* ct;        // [B*(N+1)] target rows' records (one chunk per row)
    const Cand* lt;            // [B*(N+1)][kcap] their kept lists, by index
    const ChunkRec* cd;        // draft rows
    const Cand* ld;
    const SegRec* gt;          // greedy: [B*(N+1)][nseg], chunk 0 of each row
    int nseg;
    int kcap;
    const int32_t* tokens;
    const int32_t* parents;
    const float* uniforms;
    const float* temperature;
    long long B;
    int N;
    int V;
    int greedy;
    int32_t* out_tokens;
    int32_t* out_n;
    int32_t* out_nodes;
    float* out_p;
    float* out_q;
    int* done;                 // [B]: 1 = finished here, 0 = left to the row walk
};

struct __align__(16) TreeListCtl {
    Cand lt[TREE_LIST_CAP];
    Cand ld[TREE_LIST_CAP];
    float pw[TREE_LIST_CAP];   // p of the target list's entries
    float qw[TREE_LIST_CAP];   // q of the same tokens
    int tok[TREE_MAX_NODES];
    int par[TREE_MAX_NODES];
    float W[TREE_MAX_NODES];
    float red[TREE_LIST_NT / 32];
    int err;
    int slow;
    int token;
};

// One CTA per sequence: the tree walk on the kept lists of the streaming
// pass (top-k) or on its per-row argmax (greedy).  Same rule and outputs as
// sv_tree_kernel.
__global__ void __launch_bounds__(TREE_LIST_NT) sv_tree_list_kernel(const TreeListParams P) {
    constexpr int NT = TREE_LIST_NT, NW = NT / 32;
    __shared__ TreeListCtl S;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long b = blockIdx.x;
    const int N = P.N, V = P.V;
    const bool greedy = P.greedy != 0;
    const float* u = greedy ? nullptr : P.uniforms + b * (N + 1);
    float T = 1.f;
    if (!greedy && P.temperature) T = P.temperature[b];
    const float c = (T > 0.f && T != POS_INF) ? LOG2E / T : 1.f;
    if (tid == 0) {
        S.err = 0;
        S.slow = 0;
    }
    __syncthreads();
    for (int i = tid; i < N; i += NT) {
        const int t = P.tokens[b * N + i], p = P.parents[b * N + i];
        S.tok[i] = t;
        S.par[i] = p;
        if (t < 0 || t >= V || p < 0 || p > i) S.err = 1;
        if (P.out_p) P.out_p[b * N + i] = __int_as_float(0x7fc00000);
        if (P.out_q) P.out_q[b * N + i] = __int_as_float(0x7fc00000);
    }
    if (!greedy) {
        if (tid == 0 && !(T > 0.f && T != POS_INF)) S.err = 1;
        for (int i = tid; i <= N; i += NT)
            if (!(u[i] >= 0.f && u[i] < 1.f)) S.err = 1;
    }
    __syncthreads();
    auto block_sum = [&](float v) -> float {
        v = warp_sum(v);
        if (lane == 0) S.red[warp] = v;
        __syncthreads();
        float s = 0.f;
        for (int w = 0; w < NW; ++w) s += S.red[w];
        __syncthreads();
        return s;
    };
    // entry of token x in a list sorted by index, or -1
    auto find = [](const Cand* L, int n, int x) {
        int lo = 0, hi = n - 1;
        while (lo <= hi) {
            const int mid = (lo + hi) >> 1;
            const int y = L[mid].i;
            if (y == x) return mid;
            if (y < x) lo = mid + 1; else hi = mid - 1;
        }
        return -1;
    };

    int a = 0, depth = 0, y = -1;
    int err = S.err, slow = 0;
    while (!err) {
        const long long r = b * (N + 1) + a;
        int next = 0;
        if (greedy) {
            const SegRec g = P.gt[r * P.nseg];
            if (g.flags & (REC_TIMEOUT | REC_DIAG)) {
                slow = 1;
                break;
            }
            if (!(g.m == g.m) || g.m == POS_INF || !(g.m > NEG_INF) || g.arg < 0) {
                err = 1;
                break;
            }
            for (int ch = a + 1; ch <= N && !next; ++ch)
                if (S.par[ch - 1] == a && S.tok[ch - 1] == g.arg) next = ch;
            if (!next) {
                y = g.arg;
                break;
            }
        } else {
            const ChunkRec ct = P.ct[r], cd = P.cd[r];
            if ((ct.flags | cd.flags) & (REC_TIMEOUT | REC_OVERFLOW | REC_DIAG)) {
                slow = 1;
                break;
            }
            if (!(ct.m == ct.m) || ct.m == POS_INF || !(ct.m > NEG_INF) || !(cd.m == cd.m) || cd.m == POS_INF ||
                !(cd.m > NEG_INF) || !(ct.s > 0.f) || !(cd.s > 0.f)) {
                err = 1;
                break;
            }
            const int nt = min(ct.n, TREE_LIST_CAP), nd = min(cd.n, TREE_LIST_CAP);
            const float mt = ct.m * c, md = cd.m * c, it = 1.f / ct.s, id = 1.f / cd.s;
            for (int i = tid; i < nt; i += NT) S.lt[i] = P.lt[r * P.kcap + i];
            for (int i = tid; i < nd; i += NT) S.ld[i] = P.ld[r * P.kcap + i];
            __syncthreads();
            for (int i = tid; i < nt; i += NT) {
                S.pw[i] = ex2(fmaf(S.lt[i].v, c, -mt)) * it;
                const int j = find(S.ld, nd, S.lt[i].i);
                S.qw[i] = j >= 0 ? ex2(fmaf(S.ld[j].v, c, -md)) * id : 0.f;
            }
            __syncthreads();
            int levels = 0;
            auto cur = [&](int i) {  // current distribution at target-list entry i
                float rr = S.pw[i];
                for (int l = 0; l < levels; ++l) rr = fmaxf(rr - S.qw[i], 0.f) / S.W[l];
                return rr;
            };
            for (int ch = a + 1; ch <= N; ++ch) {
                if (S.par[ch - 1] != a) continue;
                const int x = S.tok[ch - 1];
                const int ip = find(S.lt, nt, x), iq = find(S.ld, nd, x);
                const float rr = ip >= 0 ? cur(ip) : 0.f;
                const float qv = iq >= 0 ? ex2(fmaf(S.ld[iq].v, c, -md)) * id : 0.f;
                if (tid == 0) {
                    if (P.out_p) P.out_p[b * N + ch - 1] = rr;
                    if (P.out_q) P.out_q[b * N + ch - 1] = qv;
                }
                if (u[ch - 1] * qv < rr) {
                    next = ch;
                    break;
                }
                float acc = 0.f;
                for (int i = tid; i < nt; i += NT) acc += fmaxf(cur(i) - S.qw[i], 0.f);
                const float W = block_sum(acc);
                if (W > 0.f) {
                    if (tid == 0) S.W[levels] = W;
                    __syncthreads();
                    ++levels;
                }
            }
            if (!next) {
                // inverse CDF over the target list in index order (warp 0)
                if (warp == 0) {
                    float Wt = 0.f;
                    for (int i0 = 0; i0 < nt; i0 += 32) {
                        const float w = i0 + lane < nt ? cur(i0 + lane) : 0.f;
                        Wt += __shfl_sync(0xffffffffu, warp_incl_scan(w, lane), 31);
                    }
                    const float xx = u[N] * Wt;
                    float carry = 0.f;
                    int token = -1, lastp = -1;
                    for (int i0 = 0; i0 < nt; i0 += 32) {
                        const float w = i0 + lane < nt ? cur(i0 + lane) : 0.f;
                        const float incl = warp_incl_scan(w, lane);
                        const unsigned hit = __ballot_sync(0xffffffffu, i0 + lane < nt && carry + incl > xx);
                        const unsigned pos = __ballot_sync(0xffffffffu, w > 0.f);
                        if (pos) lastp = i0 + 31 - __clz(pos);
                        if (hit) {
                            token = S.lt[i0 + __ffs(hit) - 1].i;
                            break;
                        }
                        carry += __shfl_sync(0xffffffffu, incl, 31);
                    }
                    if (lane == 0) S.token = token >= 0 ? token : (lastp >= 0 ? S.lt[lastp].i : -1);
                }
                __syncthreads();
                y = S.token;
                if (y < 0) err = 1;
                break;
            }
            __syncthreads();  // the lists are reloaded for the next node
        }
        if (tid == 0) {
            if (P.out_nodes) P.out_nodes[b * (N + 1) + depth] = next;
            P.out_tokens[b * (N + 1) + depth] = S.tok[next - 1];
        }
        ++depth;
        a = next;
    }
    __syncthreads();
    if (slow) {  // the row walk takes the whole sequence
        if (tid == 0) P.done[b] = 0;
        return;
    }
    for (int i = tid; i <= N; i += NT) {
        if (err || i > depth) {
            P.out_tokens[b * (N + 1) + i] = -1;
            if (P.out_nodes) P.out_nodes[b * (N + 1) + i] = -1;
        } else if (i == depth) {
            P.out_tokens[b * (N + 1) + i] = y;
            if (P.out_nodes) P.out_nodes[b * (N + 1) + i] = -1;
        }
    }
    if (tid == 0) {
        P.out_n[b] = err ? -1 : depth;
        P.done[b] = 1;
    }
}

}  // namespace sv
