// K3 — the final draw of sequences whose draw needs a full pass over a
// (target, draft) row pair: the residual max(0, p_j - q_j) at a rejected
// position without top-k (speculative decoding entry "推测解码", section
// "提议与核验的基本步骤": the first rejected position is redrawn from the
// normalised positive part of p - q).
//
// One CTA per (sequence, segment).  Each CTA sums the weights of its segment
// twice — residual and p alone (the fallback when the residual mass is zero) —
// and writes both; the last CTA of a sequence to finish (a counter that the
// per-sequence kernel zeroes on every call) takes the inverse CDF with u_k
// over the segment masses in index order, rescans the one segment that holds
// u_k * W and writes the token.  Sequences without such a draw leave at once.
#pragma once

#include "sv_common.cuh"
#include "sv_procs.cuh"

namespace sv {

constexpr int RES_NT = 256;
constexpr int RES_NW = RES_NT / 32;

struct ResidParams {
    const void* target;   // [B][k+1][V]
    const void* draft;    // [B][k][V]
    int V;
    int k;
    int seg;              // elements per segment
    int nseg;
    const DrawReq* req;   // [B]
    float2* mass;         // [B][nseg]: (residual mass, p mass)
    int* counter;         // [B], zeroed by the per-sequence kernel
    int32_t* out_tokens;  // [B][k+1]
    int32_t* out_n;       // [B]
    // processors (mask, repetition penalty) or null
    const uint32_t* allow;
    const uint32_t* pen;
    const float* theta;
    int W4;
};

template <int DT>
__device__ __forceinline__ void res_load_vec(const void* row, bool aligned, int q, int V, float* v,
                                             const ProcView& pv) {
    constexpr int VEC = VT<DT>::VEC;
    const long long e = static_cast<long long>(q) * VEC;
    if (aligned && e + VEC <= V) {
        unpack<DT>(__ldg(reinterpret_cast<const uint4*>(row) + q), v);
    } else {
#pragma unroll
        for (int t = 0; t < VEC; ++t) v[t] = (e + t < V) ? load_elem<DT>(row, e + t) : NEG_INF;
    }
    if (pv.allow) {
#pragma unroll
        for (int t = 0; t < VEC; ++t)
            if (e + t < V) v[t] = proc_logit(v[t], e + t, pv);
    }
}

template <int DT>
__global__ void __launch_bounds__(RES_NT) sv_resid_kernel(const ResidParams P) {
    constexpr int VEC = VT<DT>::VEC;
    constexpr int ELT = VT<DT>::ELT;
    __shared__ float red[RES_NW][2];
    __shared__ float pre[RES_NW];
    __shared__ int last, tok_cross, tok_last, sel, lastm, use_q_s;
    __shared__ float x_s, base_s;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long b = blockIdx.x / P.nseg;
    const int s = static_cast<int>(blockIdx.x - b * P.nseg);
    pdl_wait_primary();  // the per-sequence kernel's requests are visible from here
    const DrawReq R = P.req[b];
    if (!R.need) return;

    const int V = P.V;
    const ProcView pv = proc_view(P.allow, P.pen, P.theta, P.W4, b);
    const void* rowt = static_cast<const char*>(P.target) + static_cast<size_t>(R.rowt) * V * ELT;
    const void* rowd = static_cast<const char*>(P.draft) + static_cast<size_t>(R.rowd) * V * ELT;
    const bool alt = (reinterpret_cast<uintptr_t>(rowt) & 15u) == 0;
    const bool ald = (reinterpret_cast<uintptr_t>(rowd) & 15u) == 0;
    const int vps = P.seg / VEC;
    const int nvec = (V + VEC - 1) / VEC;
    auto weights = [&](int q, bool use_q, float* w) {
        float vt[VEC], vd[VEC];
        res_load_vec<DT>(rowt, alt, q, V, vt, pv);
        if (use_q) res_load_vec<DT>(rowd, ald, q, V, vd, pv);
#pragma unroll
        for (int t = 0; t < VEC; ++t) {
            const float pt = (vt[t] >= R.t_tau) ? ex2(fmaf(vt[t], R.c, -R.t_msc)) * R.t_invS : 0.f;
            if (use_q) {
                const float qd = (vd[t] >= R.d_tau) ? ex2(fmaf(vd[t], R.c, -R.d_msc)) * R.d_invS : 0.f;
                w[t] = fmaxf(pt - qd, 0.f);
            } else {
                w[t] = pt;
            }
        }
    };

    // ---- this segment's masses --------------------------------------------------------
    {
        float ar = 0.f, ap = 0.f;
        for (int q = s * vps + tid; q < min(nvec, (s + 1) * vps); q += RES_NT) {
            float vt[VEC], vd[VEC];
            res_load_vec<DT>(rowt, alt, q, V, vt, pv);
            if (R.use_q) res_load_vec<DT>(rowd, ald, q, V, vd, pv);
#pragma unroll
            for (int t = 0; t < VEC; ++t) {
                const float pt = (vt[t] >= R.t_tau) ? ex2(fmaf(vt[t], R.c, -R.t_msc)) * R.t_invS : 0.f;
                ap += pt;
                if (R.use_q) {
                    const float qd = (vd[t] >= R.d_tau) ? ex2(fmaf(vd[t], R.c, -R.d_msc)) * R.d_invS : 0.f;
                    ar += fmaxf(pt - qd, 0.f);
                }
            }
        }
        ar = warp_sum(ar);
        ap = warp_sum(ap);
        if (lane == 0) {
            red[warp][0] = ar;
            red[warp][1] = ap;
        }
        __syncthreads();
        if (tid == 0) {
            float mr = 0.f, mp = 0.f;
            for (int w = 0; w < RES_NW; ++w) {
                mr += red[w][0];
                mp += red[w][1];
            }
            P.mass[b * P.nseg + s] = make_float2(mr, mp);
            __threadfence();
            last = atomicAdd(&P.counter[b], 1) == P.nseg - 1;
        }
        __syncthreads();
        if (!last) return;
    }

    // ---- last CTA of the sequence: inverse CDF over the segments, then one segment -----
    __threadfence();
    if (tid == 0) {
        const volatile float2* m = P.mass + b * P.nseg;
        float Wr = 0.f, Wp = 0.f;
        for (int q = 0; q < P.nseg; ++q) {
            Wr += m[q].x;
            Wp += m[q].y;
        }
        const bool uq = R.use_q && Wr > 0.f;  // zero residual mass: redraw from p at this position
        const float W = uq ? Wr : Wp;
        const float x = R.u * W;
        int sl = -1, lm = 0;
        float a = 0.f, base = 0.f;
        for (int q = 0; q < P.nseg; ++q) {
            const float mq = uq ? m[q].x : m[q].y;
            const float nxt = a + mq;
            if (nxt > x) {
                sl = q;
                base = a;
                break;
            }
            a = nxt;
        }
        if (sl < 0) {
            lm = 1;
            for (int q = P.nseg - 1; q >= 0; --q)
                if ((uq ? m[q].x : m[q].y) > 0.f) {
                    sl = q;
                    break;
                }
        }
        use_q_s = uq ? 1 : 0;
        x_s = x;
        base_s = base;
        sel = sl;
        lastm = lm;
        tok_cross = -1;
        tok_last = -1;
    }
    __syncthreads();
    const bool uq = use_q_s != 0;
    const int sl = sel;
    int token = -1;
    if (sl >= 0) {
        const float x = x_s;
        float base = base_s;
        const bool lm = lastm != 0;
        const int q0 = sl * vps, q1 = min(nvec, (sl + 1) * vps);
        for (int tq = q0; tq < q1; tq += RES_NT) {  // tiles of RES_NT vectors, in index order
            const int q = tq + tid;
            float w[VEC];
            float vs = 0.f;
            if (q < q1) {
                weights(q, uq, w);
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
            if (lastpos >= 0) atomicMax(&tok_last, lastpos);
            const float inw = warp_incl_scan(vs, lane);
            float exw = __shfl_up_sync(0xffffffffu, inw, 1);
            if (lane == 0) exw = 0.f;
            if (lane == 31) red[warp][0] = inw;
            __syncthreads();
            if (tid == 0) {
                float a = 0.f;
                for (int w2 = 0; w2 < RES_NW; ++w2) {
                    pre[w2] = a;
                    a += red[w2][0];
                }
            }
            __syncthreads();
            const float wp = pre[warp];
            const float tile_tot = pre[RES_NW - 1] + red[RES_NW - 1][0];
            if (!lm && tok_cross < 0) {
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
                    tok_cross = tok;
                }
            }
            base = base + tile_tot;
            __syncthreads();
        }
        token = tok_cross >= 0 ? tok_cross : tok_last;
    }
    if (tid == 0) {
        int32_t* out = P.out_tokens + b * (P.k + 1);
        if (token >= 0) {
            out[R.j] = token;
        } else {  // no positive weight anywhere: the sequence is an error
            for (int i = 0; i <= P.k; ++i) out[i] = -1;
            P.out_n[b] = -1;
        }
    }
}

}  // namespace sv
