// Host side of the spec_verify C ABI: argument checks, launch planning,
// workspace handling and the launches, each a programmatic dependent launch
// of the one before it: the streaming pass (except for a single wave that
// fills more than half the device), the per-sequence kernel, and for softmax
// verification the segment kernel of the residual draws.  Nothing here
// synchronises the caller's stream.
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <climits>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>

#include "../../include/spec_verify.h"
#include "sv_rows.cuh"
#include "sv_resid.cuh"
#include "sv_seq.cuh"
#include "sv_tree.cuh"
#include "sv_head.cuh"

namespace {

constexpr int kVersion = 20000;  // 2.0.0
constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultTimeoutNs = 1000000000ull;
constexpr int kSegBytes = sv::TILE_BYTES;  // bytes per segment (one ring stage)
constexpr int kStages = 2;                 // ring stages of the streaming kernel
constexpr int kTopkMax = 256;         // largest K on the kept-list path (<= threads)

struct DeviceInfo {
    int ok = 0;
    int id = 0;
    int sms = 0;
    int smem_optin = 0;
    int smem_per_sm = 0;
    cudaMemPool_t pool = nullptr;
};

DeviceInfo g_dev[kMaxDevices];
std::once_flag g_dev_once[kMaxDevices];
std::once_flag g_pool_once[kMaxDevices];
// streaming-kernel instantiations: 24 plain (dtype x threads x mode) and 12 with
// processors (dtype x 128/256 threads x softmax/top-k/max-only); then the two
// per-sequence kernels
constexpr int kRowsSlots = 36;
std::once_flag g_attr_once[kMaxDevices][kRowsSlots + 2];
cudaError_t g_attr_err[kMaxDevices][kRowsSlots + 2];  // result of each one-time attribute call
std::once_flag g_occ_once[kMaxDevices][kRowsSlots];
int g_occ[kMaxDevices][kRowsSlots];

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

const DeviceInfo* device_info(int* dev_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return nullptr;
    }
    std::call_once(g_dev_once[dev], [dev] {
        DeviceInfo& d = g_dev[dev];
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) !=
                cudaSuccess) {
            cudaGetLastError();
            d.ok = 0;
            return;
        }
        // sm_100a code runs on compute capability 10.0 only (not on other 10.x parts)
        d.ok = (major == 10 && minor == 0) ? 1 : 0;
        d.id = dev;
    });
    *dev_out = dev;
    return g_dev[dev].ok ? &g_dev[dev] : nullptr;
}

// The library's own stream-ordered pool of one device: memory released with
// cudaFreeAsync is kept for the next call instead of being unmapped.
cudaMemPool_t device_pool(int dev) {
    std::call_once(g_pool_once[dev], [dev] {
        cudaMemPoolProps props;
        std::memset(&props, 0, sizeof props);
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t pool = nullptr;
        if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) {
            cudaGetLastError();
            return;
        }
        uint64_t keep = UINT64_MAX;
        cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
        cudaGetLastError();
        g_dev[dev].pool = pool;
    });
    return g_dev[dev].pool;
}

long long ceil_div(long long a, long long b) { return (a + b - 1) / b; }
long long round_up(long long a, long long b) { return ceil_div(a, b) * b; }

struct Plan {
    bool proc = false;  // processors: K0 builds the bitmaps, K1 runs its PROC variant
    int W4 = 0;         // words per bitmap row
    long long nprocs = 0;  // processor rows (sequences)
    size_t off_allow = 0, off_pen = 0;
    int mode = 0, elt = 2, seg = 0, nseg = 0, nch = 1, spc = 1, nt1 = 128, stages = kStages;
    int lcap = 0, kcap = 0, mg = 0;
    long long R = 0, tasks = 0, slots = 0;
    size_t smem1 = 0, smem2 = 0;
    size_t off_chunks = 0, off_cands = 0, ws_bytes = 0;
    bool defer = false;  // residual draws by the segment kernel
    bool pre = false;    // per-sequence kernel loads every row's kept list at once
    size_t pre_off = 0;
    size_t off_req = 0, off_mass = 0, off_counter = 0;
    bool nuc = false;  // nucleus without top-k: the nucleus kernel cuts every row
    size_t off_nuc = 0;
};

int rows_occupancy(int dev, int dt, int nt, int mode, bool proc, size_t smem);

// Plan the launches for `seqs` sequences of draft length k (rows = k+1 target
// rows per sequence, plus k draft rows when stochastic); `nprocs` > 0 when the
// processors are in use (their rows: one per sequence).
sv_status_t make_plan(const DeviceInfo& dev, long long seqs, int k, int V, int dt, bool greedy, int top_k,
                      const sv_options_t* opts, long long nprocs, Plan* out) {
    Plan p;
    p.proc = nprocs > 0;
    p.nprocs = nprocs;
    p.elt = dt ? 4 : 2;
    const int vec = 16 / p.elt;
    p.nt1 = (opts && opts->threads) ? opts->threads : 128;
    p.seg = kSegBytes / p.elt;
    p.nseg = static_cast<int>(ceil_div(V, p.seg));
    p.R = seqs * (k + 1) + (greedy ? 0 : seqs * k);
    const bool radix = opts && opts->topk_path == 2;
    if (greedy)
        p.mode = sv::MODE_GREEDY;
    else if (top_k == 0)
        p.mode = sv::MODE_SOFTMAX;
    else if (top_k <= kTopkMax && !radix)
        p.mode = sv::MODE_TOPK;
    else
        p.mode = sv::MODE_MAXONLY;
    if (opts && opts->topk_path == 1 && top_k > 0 && p.mode != sv::MODE_TOPK) return SV_ERR_UNSUPPORTED;
    if (p.proc && (greedy || p.nt1 == 512)) return SV_ERR_UNSUPPORTED;
    if (p.mode == sv::MODE_TOPK) {
        // the running bound needs K <= threads (each warp contributes <= 32 ranks)
        if (top_k > p.nt1) {
            if (opts && opts->threads) {
                if (opts->topk_path == 1) return SV_ERR_UNSUPPORTED;
                p.mode = sv::MODE_MAXONLY;
            } else {
                p.nt1 = 256;
            }
        }
        if (p.mode == sv::MODE_TOPK) p.lcap = (p.nt1 / 32) * sv::TOPK_WCAP;
    }
    if (p.proc && p.nt1 == 512) return SV_ERR_UNSUPPORTED;
    p.smem1 = static_cast<size_t>(sv::rows_smem_bytes(p.mode, p.nt1, p.stages, p.lcap, p.proc));
    if (p.smem1 > static_cast<size_t>(dev.smem_optin)) return SV_ERR_UNSUPPORTED;
    // chunks per row: one when there are enough rows to fill the device
    long long occ = rows_occupancy(dev.id, dt, p.nt1, p.mode, p.proc, p.smem1);
    if (occ < 1) return SV_ERR_CUDA;
    const long long slots = occ * dev.sms;
    p.slots = slots;
    int nch;
    if (opts && opts->chunks_per_row) {
        nch = opts->chunks_per_row;
    } else if (p.R * 2 >= slots) {
        nch = 1;
    } else {
        nch = static_cast<int>(ceil_div(slots, p.R));
    }
    if (nch > p.nseg) nch = p.nseg;
    if (nch < ceil_div(p.nseg, sv::MAX_TILES_K1)) nch = static_cast<int>(ceil_div(p.nseg, sv::MAX_TILES_K1));
    if (nch < 1) nch = 1;
    p.spc = static_cast<int>(ceil_div(p.nseg, nch));
    p.nch = static_cast<int>(ceil_div(p.nseg, p.spc));
    p.tasks = p.R * p.nch;
    if (p.tasks > INT_MAX || seqs > INT_MAX) return SV_ERR_INVALID_ARG;
    if (p.mode == sv::MODE_TOPK) {
        int kc = 64;
        while (kc < 2 * top_k) kc <<= 1;
        p.kcap = kc > 1024 ? 1024 : kc;
        p.mg = p.nch == 1 ? p.kcap : (4 * p.kcap > 1024 ? 1024 : 4 * p.kcap);
    } else {
        p.kcap = 0;
        p.mg = 64;  // also holds the two draw lists of the top-k path
    }
    // workspace: segment partials (not in top-k mode), chunk headers, kept lists
    const size_t segs = p.mode == sv::MODE_TOPK ? 0 : static_cast<size_t>(p.R) * p.nseg * sizeof(sv::SegRec);
    size_t chunks = 0, cands = 0;
    if (p.mode == sv::MODE_TOPK) {
        chunks = static_cast<size_t>(p.R) * p.nch * sizeof(sv::ChunkRec);
        cands = static_cast<size_t>(p.R) * p.nch * p.kcap * sizeof(sv::Cand);
    }
    p.off_chunks = round_up(segs, 256);
    p.off_cands = round_up(p.off_chunks + chunks, 256);
    p.ws_bytes = round_up(p.off_cands + cands, 256);
    // processors: allow and penalty bitmaps, rows of W4 words (a multiple of 4)
    if (p.proc) {
        p.W4 = static_cast<int>(4 * ceil_div(V, 128));
        const size_t bm = static_cast<size_t>(nprocs) * p.W4 * sizeof(uint32_t);
        p.off_allow = p.ws_bytes;
        p.off_pen = round_up(p.off_allow + bm, 256);
        p.ws_bytes = round_up(p.off_pen + bm, 256);
    }
    // softmax verification: residual draws by the segment kernel
    p.defer = p.mode == sv::MODE_SOFTMAX && k > 0;
    if (p.defer) {
        if (seqs * static_cast<long long>(p.nseg) > INT_MAX) return SV_ERR_INVALID_ARG;
        p.off_req = p.ws_bytes;
        p.off_mass = round_up(p.off_req + static_cast<size_t>(seqs) * sizeof(sv::DrawReq), 256);
        p.off_counter = round_up(p.off_mass + static_cast<size_t>(seqs) * p.nseg * sizeof(float2), 256);
        p.ws_bytes = round_up(p.off_counter + static_cast<size_t>(seqs) * sizeof(int), 256);
    }
    // nucleus without top-k: one cut per row
    if (opts && opts->top_p && p.mode == sv::MODE_SOFTMAX) {
        p.nuc = true;
        p.off_nuc = p.ws_bytes;
        p.ws_bytes = round_up(p.off_nuc + static_cast<size_t>(p.R) * sizeof(sv::NucRec), 256);
    }
    // per-sequence kernel: control, row stats, gather buffers, segment masses
    const int nrows = greedy ? k + 1 : 2 * k + 1;
    size_t head = static_cast<size_t>(nrows) * sizeof(sv::RowStat) + static_cast<size_t>(k + 1) * 8 + 8;
    head = round_up(head, 128);
    p.smem2 = sv::SEQ_CTL_BYTES + head + static_cast<size_t>(sv::SEQ_NW) * p.mg * sizeof(sv::Cand) +
              static_cast<size_t>(p.nseg) * (sv::SEQ_NW + 1) * sizeof(float);
    // top-k with one chunk per row: every row's record and kept list in shared memory
    const size_t pre_bytes = static_cast<size_t>(nrows) * (static_cast<size_t>(p.kcap) * sizeof(sv::Cand) + sizeof(sv::ChunkRec));
    if (p.mode == sv::MODE_TOPK && p.nch == 1 && pre_bytes <= 64 * 1024) {
        p.pre = true;
        p.pre_off = round_up(p.smem2, 16);
        p.smem2 = p.pre_off + pre_bytes;
    }
    if (p.smem1 > static_cast<size_t>(dev.smem_optin) || p.smem2 > static_cast<size_t>(dev.smem_optin))
        return SV_ERR_UNSUPPORTED;
    (void)vec;
    *out = p;
    return SV_OK;
}

using RowsFn = void (*)(sv::RowsParams);
using SeqFn = void (*)(sv::SeqParams);
using ResFn = void (*)(sv::ResidParams);
using ProcsFn = void (*)(sv::ProcsParams);
using NucFn = void (*)(sv::NucParams);
using TreeFn = void (*)(sv::TreeParams);
using TreeListFn = void (*)(sv::TreeListParams);

template <int DT, int NT, bool PROC>
RowsFn rows_for_mode(int mode) {
    if constexpr (PROC) {  // the processors have no greedy variant (rejected by the plan)
        switch (mode) {
            case sv::MODE_SOFTMAX: return sv::sv_rows_kernel<DT, NT, sv::MODE_SOFTMAX, true>;
            case sv::MODE_TOPK: return sv::sv_rows_kernel<DT, NT, sv::MODE_TOPK, true>;
            default: return sv::sv_rows_kernel<DT, NT, sv::MODE_MAXONLY, true>;
        }
    } else {
        switch (mode) {
            case sv::MODE_GREEDY: return sv::sv_rows_kernel<DT, NT, sv::MODE_GREEDY, false>;
            case sv::MODE_SOFTMAX: return sv::sv_rows_kernel<DT, NT, sv::MODE_SOFTMAX, false>;
            case sv::MODE_TOPK: return sv::sv_rows_kernel<DT, NT, sv::MODE_TOPK, false>;
            default: return sv::sv_rows_kernel<DT, NT, sv::MODE_MAXONLY, false>;
        }
    }
}

// slot = dtype * 12 + threads-class * 4 + mode (24 plain instantiations), then
// 24 + dtype * 6 + threads-class * 3 + (mode - 1) with processors (12 more)
RowsFn pick_rows(int dt, int nt, int mode, bool proc, int* slot) {
    const int ntc = nt == 128 ? 0 : (nt == 512 ? 2 : 1);
    *slot = proc ? 24 + dt * 6 + ntc * 3 + (mode - 1) : dt * 12 + ntc * 4 + mode;
    if (proc) {
        if (dt == 0) return nt == 128 ? rows_for_mode<0, 128, true>(mode) : rows_for_mode<0, 256, true>(mode);
        return nt == 128 ? rows_for_mode<1, 128, true>(mode) : rows_for_mode<1, 256, true>(mode);
    }
    if (dt == 0) {
        if (nt == 128) return rows_for_mode<0, 128, false>(mode);
        if (nt == 512) return rows_for_mode<0, 512, false>(mode);
        return rows_for_mode<0, 256, false>(mode);
    }
    if (nt == 128) return rows_for_mode<1, 128, false>(mode);
    if (nt == 512) return rows_for_mode<1, 512, false>(mode);
    return rows_for_mode<1, 256, false>(mode);
}

sv_status_t set_attrs(int dev, int dt, int nt, int mode, bool proc) {
    int slot = 0;
    RowsFn f1 = pick_rows(dt, nt, mode, proc, &slot);
    SeqFn f2 = dt ? sv::sv_seq_kernel<1> : sv::sv_seq_kernel<0>;
    std::call_once(g_attr_once[dev][slot], [&] {
        g_attr_err[dev][slot] =
            cudaFuncSetAttribute(f1, cudaFuncAttributeMaxDynamicSharedMemorySize, g_dev[dev].smem_optin);
        if (g_attr_err[dev][slot] != cudaSuccess) cudaGetLastError();
    });
    const int s2 = kRowsSlots + dt;
    std::call_once(g_attr_once[dev][s2], [&] {
        g_attr_err[dev][s2] =
            cudaFuncSetAttribute(f2, cudaFuncAttributeMaxDynamicSharedMemorySize, g_dev[dev].smem_optin);
        if (g_attr_err[dev][s2] != cudaSuccess) cudaGetLastError();
    });
    // a failed attribute call fails every later call for that kernel too
    if (g_attr_err[dev][slot] != cudaSuccess || g_attr_err[dev][s2] != cudaSuccess) return SV_ERR_CUDA;
    return SV_OK;
}

// Resident streaming CTAs per SM for one instantiation (its shared memory
// depends only on the slot), from the occupancy calculator; 0 on failure.
int rows_occupancy(int dev, int dt, int nt, int mode, bool proc, size_t smem) {
    if (set_attrs(dev, dt, nt, mode, proc) != SV_OK) return 0;
    int slot = 0;
    RowsFn f1 = pick_rows(dt, nt, mode, proc, &slot);
    std::call_once(g_occ_once[dev][slot], [&] {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, f1, nt + 32, smem) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
        g_occ[dev][slot] = n;
    });
    return g_occ[dev][slot];
}

struct Call {
    // processors (options): mask [S][ceil(V/32)], rep_ids [S][n_rep], rep_penalty [S]
    const uint32_t* mask = nullptr;
    const int32_t* rep_ids = nullptr;
    int n_rep = 0;
    const float* rep_penalty = nullptr;
    long long rows_per_seq = 1;  // sampler: rows per processor sequence
    long long nprocs = 0;        // processor rows (0: no processors)
    const void* target = nullptr;
    const void* draft = nullptr;
    const int32_t* draft_tokens = nullptr;
    const float* uniforms = nullptr;
    const float* temperature = nullptr;
    long long seqs = 0;
    int k = 0, V = 0, top_k = 0, dt = 0;
    bool greedy = false, sample = false;
    int32_t* out_tokens = nullptr;
    int32_t* out_n = nullptr;
    float* out_p = nullptr;
    float* out_q = nullptr;
    int32_t* out_status = nullptr;
};

// workspaces taken from the library pool by this process (the calls without one)
std::atomic<unsigned long long> g_pool_allocs{0};

sv_status_t run(const Call& cl, void* workspace, size_t workspace_bytes, const sv_options_t* opts,
                cudaStream_t st) {
    int dev = 0;
    const DeviceInfo* info = device_info(&dev);
    if (!info) return SV_ERR_UNSUPPORTED;
    Plan p;
    sv_status_t s = make_plan(*info, cl.seqs, cl.k, cl.V, cl.dt, cl.greedy, cl.top_k, opts, cl.nprocs, &p);
    if (s != SV_OK) return s;
    if (workspace && (workspace_bytes < p.ws_bytes || !aligned(workspace, 16))) return SV_ERR_INVALID_ARG;
    if (opts && opts->top_p && p.mode == sv::MODE_GREEDY) return SV_ERR_UNSUPPORTED;  // greedy takes no nucleus
    if ((s = set_attrs(dev, cl.dt, p.nt1, p.mode, p.proc)) != SV_OK) return s;

    void* ws = workspace;
    bool owned = false;
    if (!ws) {
        cudaMemPool_t pool = device_pool(dev);
        if (!pool || cudaMallocFromPoolAsync(&ws, p.ws_bytes, pool, st) != cudaSuccess) {
            cudaGetLastError();
            return SV_ERR_CUDA;
        }
        g_pool_allocs.fetch_add(1, std::memory_order_relaxed);
        owned = true;
    }
    auto* base = static_cast<unsigned char*>(ws);

    sv::RowsParams r;
    std::memset(&r, 0, sizeof r);
    r.target = cl.target;
    r.draft = cl.draft;
    r.draft_tokens = cl.draft_tokens;
    r.B = cl.seqs;
    r.k = cl.k;
    r.V = cl.V;
    r.top_k = cl.top_k;
    r.temperature = cl.temperature;
    r.nseg = p.nseg;
    r.spc = p.spc;
    r.nch = p.nch;
    r.stages = p.stages;
    r.lcap = p.lcap;
    r.kcap = p.kcap;
    r.segs = reinterpret_cast<sv::SegRec*>(base);
    r.chunks = reinterpret_cast<sv::ChunkRec*>(base + p.off_chunks);
    r.cands = reinterpret_cast<sv::Cand*>(base + p.off_cands);
    r.out_status = cl.sample ? nullptr : cl.out_status;
    r.timeout_ns = (opts && opts->wait_timeout_ns) ? opts->wait_timeout_ns : kDefaultTimeoutNs;
    r.test_extra_tx = opts ? opts->test_extra_tx : 0u;
    sv::ProcsParams pp;
    std::memset(&pp, 0, sizeof pp);
    if (p.proc) {
        pp.mask = cl.mask;
        pp.rep_ids = cl.rep_ids;
        pp.n_rep = cl.n_rep;
        pp.rep_penalty = cl.rep_penalty;
        pp.V = cl.V;
        pp.words = static_cast<int>(ceil_div(cl.V, 32));
        pp.W4 = p.W4;
        pp.allow = reinterpret_cast<uint32_t*>(base + p.off_allow);
        pp.pen = reinterpret_cast<uint32_t*>(base + p.off_pen);
        r.allow = pp.allow;
        r.pen = pp.pen;
        r.theta = cl.rep_penalty;
        r.W4 = p.W4;
    }
    r.procs_div = static_cast<int>(cl.rows_per_seq);

    sv::SeqParams q;
    std::memset(&q, 0, sizeof q);
    q.target = cl.target;
    q.draft = cl.draft;
    q.draft_tokens = cl.draft_tokens;
    q.uniforms = cl.uniforms;
    q.temperature = cl.temperature;
    q.B = cl.seqs;
    q.k = cl.k;
    q.V = cl.V;
    q.mode = p.mode;
    q.top_k = cl.top_k;
    q.sample_only = cl.sample ? 1 : 0;
    q.seg = p.seg;
    q.nseg = p.nseg;
    q.spc = p.spc;
    q.nch = p.nch;
    q.kcap = p.kcap;
    q.mg = p.mg;
    q.segs = r.segs;
    q.chunks = r.chunks;
    q.cands = r.cands;

    q.out_tokens = cl.out_tokens;
    q.out_n = cl.out_n;
    q.out_p = cl.out_p;
    q.out_q = cl.out_q;
    q.out_status = cl.sample ? nullptr : cl.out_status;
    q.defer = p.defer ? 1 : 0;
    q.top_p = opts ? opts->top_p : nullptr;
    q.nuc = p.nuc ? reinterpret_cast<sv::NucRec*>(base + p.off_nuc) : nullptr;
    q.pre = p.pre ? 1 : 0;
    q.pre_off = static_cast<int>(p.pre_off);
    q.req = p.defer ? reinterpret_cast<sv::DrawReq*>(base + p.off_req) : nullptr;
    q.counter = p.defer ? reinterpret_cast<int*>(base + p.off_counter) : nullptr;
    q.allow = r.allow;
    q.pen = r.pen;
    q.theta = r.theta;
    q.W4 = r.W4;
    q.procs_div = r.procs_div;

    sv::ResidParams rp;
    std::memset(&rp, 0, sizeof rp);
    rp.target = cl.target;
    rp.draft = cl.draft;
    rp.V = cl.V;
    rp.k = cl.k;
    rp.seg = p.seg;
    rp.nseg = p.nseg;
    rp.req = q.req;
    rp.mass = p.defer ? reinterpret_cast<float2*>(base + p.off_mass) : nullptr;
    rp.counter = q.counter;
    rp.out_tokens = cl.out_tokens;
    rp.out_n = cl.out_n;
    rp.allow = r.allow;
    rp.pen = r.pen;
    rp.theta = r.theta;
    rp.W4 = r.W4;

    sv_status_t result = SV_OK;
    do {
        if (opts && opts->event_start &&
            cudaEventRecord(static_cast<cudaEvent_t>(opts->event_start), st) != cudaSuccess) {
            result = SV_ERR_CUDA;
            break;
        }
        if (p.proc) {
            // K0: the processors' bitmaps, in plain stream order after the
            // previous call's kernels (which may still read them)
            cudaLaunchConfig_t c0;
            std::memset(&c0, 0, sizeof c0);
            c0.gridDim = dim3(static_cast<unsigned>(p.nprocs), 1, 1);
            c0.blockDim = dim3(sv::PROCS_NT, 1, 1);
            c0.stream = st;
            ProcsFn f0 = sv::sv_procs_kernel;
            if (cudaLaunchKernelEx(&c0, f0, pp) != cudaSuccess) {
                result = SV_ERR_CUDA;
                break;
            }
        }
        int slot = 0;
        RowsFn f1 = pick_rows(cl.dt, p.nt1, p.mode, p.proc, &slot);
        cudaLaunchConfig_t c1;
        std::memset(&c1, 0, sizeof c1);
        c1.gridDim = dim3(static_cast<unsigned>(p.tasks), 1, 1);
        c1.blockDim = dim3(p.nt1 + 32, 1, 1);  // consumer warps + the producer warp
        c1.dynamicSmemBytes = p.smem1;
        c1.stream = st;
        // programmatic dependent launch: the streaming pass may be placed while
        // the preceding kernel finishes (it waits for that grid before any
        // access), which hides the launch behind it.  Not for a single wave
        // that fills more than half the device when an SM can take more than
        // its even share of the wave: CTAs placed early, as slots free up (the
        // preceding kernels are themselves placed early), would pile onto the
        // SMs that free up first, and a few could miss the wave and run after
        // it (measured: +20 us per step).
        cudaLaunchAttribute a1[1];
        a1[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        a1[0].val.programmaticStreamSerializationAllowed = 1;
        const long long per_sm = p.slots / info->sms;  // CTAs an SM can hold
        const bool uneven = p.tasks > p.slots / 2 && p.tasks <= p.slots &&
                            per_sm > ceil_div(p.tasks, info->sms);
        c1.attrs = uneven ? nullptr : a1;
        c1.numAttrs = uneven ? 0 : 1;
        if (cudaLaunchKernelEx(&c1, f1, r) != cudaSuccess) {
            result = SV_ERR_CUDA;
            break;
        }
        if (opts && opts->event_stop &&
            cudaEventRecord(static_cast<cudaEvent_t>(opts->event_stop), st) != cudaSuccess) {
            result = SV_ERR_CUDA;
            break;
        }
        if (p.nuc) {
            // the nucleus cut of every row (programmatic dependent of the
            // streaming pass; it waits for that grid before reading)
            sv::NucParams np;
            std::memset(&np, 0, sizeof np);
            np.target = cl.target;
            np.draft = cl.draft;
            np.B = cl.seqs;
            np.k = cl.k;
            np.V = cl.V;
            np.temperature = cl.temperature;
            np.segs = r.segs;
            np.nseg = p.nseg;
            np.top_p = opts->top_p;
            np.procs_div = static_cast<int>(cl.rows_per_seq);
            np.allow = r.allow;
            np.pen = r.pen;
            np.theta = r.theta;
            np.W4 = r.W4;
            np.out = reinterpret_cast<sv::NucRec*>(base + p.off_nuc);
            // few rows: a cluster of up to 16 CTAs shares each row (16 is a
            // non-portable size: the kernel opts in, and 8 is used if refused)
            NucFn fn = cl.dt ? sv::sv_nucleus_kernel<1> : sv::sv_nucleus_kernel<0>;
            static std::once_flag nuc_once[2];
            static bool nuc16[2] = {false, false};
            std::call_once(nuc_once[cl.dt], [&] {
                nuc16[cl.dt] = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
                cudaGetLastError();
            });
            int ncl = 1;
            while (ncl < (nuc16[cl.dt] ? 16 : 8) && p.R * ncl < 2 * info->sms) ncl *= 2;
            cudaLaunchAttribute an[2];
            an[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            an[0].val.programmaticStreamSerializationAllowed = 1;
            an[1].id = cudaLaunchAttributeClusterDimension;
            an[1].val.clusterDim.x = static_cast<unsigned>(ncl);
            an[1].val.clusterDim.y = 1;
            an[1].val.clusterDim.z = 1;
            cudaLaunchConfig_t cn;
            std::memset(&cn, 0, sizeof cn);
            cn.gridDim = dim3(static_cast<unsigned>(p.R * ncl), 1, 1);
            cn.blockDim = dim3(sv::NUC_NT, 1, 1);
            cn.stream = st;
            cn.attrs = an;
            cn.numAttrs = 2;
            cudaError_t le = cudaLaunchKernelEx(&cn, fn, np);
            if (le != cudaSuccess && ncl > 8) {  // the larger cluster cannot be placed: 8
                cudaGetLastError();
                an[1].val.clusterDim.x = 8;
                cn.gridDim = dim3(static_cast<unsigned>(p.R * 8), 1, 1);
                le = cudaLaunchKernelEx(&cn, fn, np);
            }
            if (le != cudaSuccess) {
                result = SV_ERR_CUDA;
                break;
            }
        }
        cudaLaunchAttribute a2[1];
        a2[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        a2[0].val.programmaticStreamSerializationAllowed = 1;
        cudaLaunchConfig_t c2;
        std::memset(&c2, 0, sizeof c2);
        c2.gridDim = dim3(static_cast<unsigned>(cl.seqs), 1, 1);
        c2.blockDim = dim3(sv::SEQ_NT, 1, 1);
        c2.dynamicSmemBytes = p.smem2;
        c2.stream = st;
        c2.attrs = a2;
        c2.numAttrs = 1;
        SeqFn f2 = cl.dt ? sv::sv_seq_kernel<1> : sv::sv_seq_kernel<0>;
        if (cudaLaunchKernelEx(&c2, f2, q) != cudaSuccess) {
            result = SV_ERR_CUDA;
            break;
        }
        if (p.defer) {
            cudaLaunchConfig_t c3;
            std::memset(&c3, 0, sizeof c3);
            c3.gridDim = dim3(static_cast<unsigned>(cl.seqs * p.nseg), 1, 1);
            c3.blockDim = dim3(sv::RES_NT, 1, 1);
            c3.dynamicSmemBytes = 0;
            c3.stream = st;
            c3.attrs = a2;  // programmatic dependent launch, like the per-sequence kernel
            c3.numAttrs = 1;
            ResFn f3 = cl.dt ? sv::sv_resid_kernel<1> : sv::sv_resid_kernel<0>;
            if (cudaLaunchKernelEx(&c3, f3, rp) != cudaSuccess) {
                result = SV_ERR_CUDA;
                break;
            }
        }
    } while (false);
    if (result != SV_OK) cudaGetLastError();
    if (owned && cudaFreeAsync(ws, st) != cudaSuccess) {
        cudaGetLastError();
        if (result == SV_OK) result = SV_ERR_CUDA;
    }
    return result;
}

sv_status_t check_options(const sv_options_t* o) {
    if (!o) return SV_OK;
    if (o->chunks_per_row < 0) return SV_ERR_INVALID_ARG;
    if (!(o->threads == 0 || o->threads == 128 || o->threads == 256 || o->threads == 512))
        return SV_ERR_INVALID_ARG;
    if (o->topk_path < 0 || o->topk_path > 2) return SV_ERR_INVALID_ARG;
    if (o->top_p && !aligned(o->top_p, 4)) return SV_ERR_INVALID_ARG;
    if (o->n_rep < 0 || o->rows_per_sequence < 0) return SV_ERR_INVALID_ARG;
    if ((o->vocab_mask && !aligned(o->vocab_mask, 4)) || (o->rep_ids && !aligned(o->rep_ids, 4)) ||
        (o->rep_penalty && !aligned(o->rep_penalty, 4)))
        return SV_ERR_INVALID_ARG;
    return SV_OK;
}

// The processor inputs of the options, for `nseq` processor rows; greedy
// verification takes none.
sv_status_t take_procs(const sv_options_t* o, bool greedy, long long nseq, long long rows_per_seq, Call* cl) {
    cl->rows_per_seq = rows_per_seq;
    if (!o || !(o->vocab_mask || (o->rep_ids && o->n_rep > 0) || o->rep_penalty)) return SV_OK;
    if (greedy) return SV_ERR_UNSUPPORTED;
    cl->mask = o->vocab_mask;
    cl->rep_ids = o->n_rep > 0 ? o->rep_ids : nullptr;
    cl->n_rep = o->n_rep > 0 && o->rep_ids ? o->n_rep : 0;
    cl->rep_penalty = o->rep_penalty;
    cl->nprocs = nseq;
    return SV_OK;
}

bool decode_mode(int mode, bool* greedy, int* dt) {
    if (mode & ~0x1ff) return false;
    const int m = mode & 0xff, d = (mode >> 8) & 0x1;
    if (m > 1) return false;
    *greedy = m == 1;
    *dt = d;
    return true;
}

// Argument checks shared by the verify entry points; fills `cl`.
sv_status_t verify_args(const void* target_logits, const void* draft_logits, const int32_t* draft_tokens,
                        const float* uniforms, int B, int k, int V, const float* temperature, int top_k,
                        int mode, int32_t* out_tokens, int32_t* out_n_accepted, float* out_p, float* out_q,
                        int32_t* out_status, const sv_options_t* opts, bool check_ptrs, Call* cl) {
    bool greedy = false;
    int dt = 0;
    if (B <= 0 || k < 1 || V < 1 || top_k < 0) return SV_ERR_INVALID_ARG;
    if (!decode_mode(mode, &greedy, &dt)) return SV_ERR_INVALID_ARG;
    if (check_options(opts) != SV_OK) return SV_ERR_INVALID_ARG;
    const int elt = dt ? 4 : 2;
    if (static_cast<unsigned long long>(B) * static_cast<unsigned long long>(2 * k + 1) >
        (1ULL << 62) / (static_cast<unsigned long long>(V) * 4ULL))
        return SV_ERR_INVALID_ARG;
    if (check_ptrs) {
        if (!target_logits || !draft_tokens || !out_tokens || !out_n_accepted) return SV_ERR_INVALID_ARG;
        if (!greedy && (!draft_logits || !uniforms)) return SV_ERR_INVALID_ARG;
        if (!aligned(target_logits, elt) || (draft_logits && !aligned(draft_logits, elt))) return SV_ERR_INVALID_ARG;
        if (!aligned(draft_tokens, 4) || !aligned(out_tokens, 4) || !aligned(out_n_accepted, 4) ||
            (uniforms && !aligned(uniforms, 4)) || (temperature && !aligned(temperature, 4)) ||
            (out_p && !aligned(out_p, 4)) || (out_q && !aligned(out_q, 4)) ||
            (out_status && !aligned(out_status, 4)))
            return SV_ERR_INVALID_ARG;
    }
    cl->target = target_logits;
    cl->draft = greedy ? nullptr : draft_logits;
    cl->draft_tokens = draft_tokens;
    cl->uniforms = greedy ? nullptr : uniforms;
    cl->temperature = greedy ? nullptr : temperature;
    cl->seqs = B;
    cl->k = k;
    cl->V = V;
    cl->top_k = (top_k > 0 && top_k < V && !greedy) ? top_k : 0;
    cl->dt = dt;
    cl->greedy = greedy;
    cl->sample = false;
    cl->out_tokens = out_tokens;
    cl->out_n = out_n_accepted;
    cl->out_p = greedy ? nullptr : out_p;
    cl->out_q = greedy ? nullptr : out_q;
    cl->out_status = out_status;
    return take_procs(opts, greedy, B, 1, cl);
}

sv_status_t sample_args(const void* logits, const float* uniforms, int rows, int V, const float* temperature,
                        int top_k, int mode, int32_t* out_tokens, const sv_options_t* opts, bool check_ptrs,
                        Call* cl) {
    bool greedy = false;
    int dt = 0;
    if (rows <= 0 || V < 1 || top_k < 0) return SV_ERR_INVALID_ARG;
    if (!decode_mode(mode, &greedy, &dt)) return SV_ERR_INVALID_ARG;
    if (check_options(opts) != SV_OK) return SV_ERR_INVALID_ARG;
    const int elt = dt ? 4 : 2;
    if (static_cast<unsigned long long>(rows) > (1ULL << 62) / (static_cast<unsigned long long>(V) * 4ULL))
        return SV_ERR_INVALID_ARG;
    if (check_ptrs) {
        if (!logits || !out_tokens) return SV_ERR_INVALID_ARG;
        if (!greedy && !uniforms) return SV_ERR_INVALID_ARG;
        if (!aligned(logits, elt) || !aligned(out_tokens, 4) || (uniforms && !aligned(uniforms, 4)) ||
            (temperature && !aligned(temperature, 4)))
            return SV_ERR_INVALID_ARG;
    }
    cl->target = logits;
    cl->uniforms = greedy ? nullptr : uniforms;
    cl->temperature = greedy ? nullptr : temperature;
    cl->seqs = rows;
    cl->k = 0;
    cl->V = V;
    cl->top_k = (top_k > 0 && top_k < V && !greedy) ? top_k : 0;
    cl->dt = dt;
    cl->greedy = greedy;
    cl->sample = true;
    cl->out_tokens = out_tokens;
    const long long rps = (opts && opts->rows_per_sequence > 0) ? opts->rows_per_sequence : 1;
    return take_procs(opts, greedy, ceil_div(rows, rps), rps, cl);
}

size_t workspace_for(const Call& cl, const sv_options_t* opts) {
    int dev = 0;
    const DeviceInfo* info = device_info(&dev);
    if (!info) return 0;
    Plan p;
    if (make_plan(*info, cl.seqs, cl.k, cl.V, cl.dt, cl.greedy, cl.top_k, opts, cl.nprocs, &p) != SV_OK) return 0;
    return p.ws_bytes;
}

// ---- static scratch for spec_verify_static ----------------------------------------

// One fixed buffer per device, part of the library's device image: calls that
// must not allocate take their scratch from here.
std::mutex g_static_mu[kMaxDevices];
void* g_static_ptr[kMaxDevices];

}  // namespace

static __device__ __align__(256) unsigned char g_sv_static_scratch[SV_STATIC_WORKSPACE_BYTES];

namespace {

// Device address of the static buffer on `dev`, which must be the current
// device.  Only a successful lookup is cached, so a lookup that failed (for
// example one made during a stream capture) is tried again by the next call.
// NULL if the lookup failed.
void* static_scratch(int dev) {
    std::lock_guard<std::mutex> lock(g_static_mu[dev]);
    if (!g_static_ptr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_sv_static_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        g_static_ptr[dev] = ptr;
    }
    return g_static_ptr[dev];
}

}  // namespace

// The list walk of tree verification: the streaming pass over the trees'
// rows must produce one chunk per row and (stochastic) kept lists, or
// (greedy) per-row argmax records.  Workspace: target and draft records and
// lists, or the greedy records, and one flag per sequence.
struct TreePlan {
    bool fast = false;
    Plan k1;
    size_t off_ct = 0, off_lt = 0, off_cd = 0, off_ld = 0, off_gt = 0, off_done = 0, ws_bytes = 0;
};

void tree_plan(const DeviceInfo& dev, int B, int N, int V, int dt, bool greedy, int K, TreePlan* out) {
    TreePlan t;
    if (greedy || K > 0) {
        Plan p;
        if (make_plan(dev, B, N, V, dt, greedy, K, nullptr, 0, &p) == SV_OK && p.nch == 1 &&
            p.mode == (greedy ? sv::MODE_GREEDY : sv::MODE_TOPK) && p.kcap <= sv::TREE_LIST_CAP) {
            const size_t rows = static_cast<size_t>(B) * (N + 1);
            t.fast = true;
            t.k1 = p;
            size_t o = 0;
            if (greedy) {
                t.off_gt = o;
                o = round_up(o + rows * p.nseg * sizeof(sv::SegRec), 256);
            } else {
                t.off_ct = o;
                o = round_up(o + rows * sizeof(sv::ChunkRec), 256);
                t.off_lt = o;
                o = round_up(o + rows * p.kcap * sizeof(sv::Cand), 256);
                t.off_cd = o;
                o = round_up(o + rows * sizeof(sv::ChunkRec), 256);
                t.off_ld = o;
                o = round_up(o + rows * p.kcap * sizeof(sv::Cand), 256);
            }
            t.off_done = o;
            t.ws_bytes = round_up(o + static_cast<size_t>(B) * sizeof(int), 256);
        }
    }
    *out = t;
}

namespace {

// ---- the output projection with greedy verification ------------------------

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
std::once_flag g_head_attr_once[kMaxDevices];
cudaError_t g_head_attr_err[kMaxDevices];

// The driver's tensor-map encoder, looked up through the runtime (no link
// against the driver library).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        else
            cudaGetLastError();
    });
    return g_encode;
}

// Row-major bf16 matrix [outer][inner] as 2D tiles of box_outer rows x 64
// elements, 128-byte swizzled (the K-major operand layout of the MMA), zeros
// outside the matrix.
bool encode_bf16_rows(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_outer) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(sv::HEAD_BK), box_outer};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr int kHeadMaxVTiles = 65535;  // grid y of the first design; kept as the size bound

// Vocabulary entries per tile of the persistent projection kernel: the
// multiple of 16 in [64, 256] that minimises (rounds of tiles over the SMs) x
// (entries per tile + a fixed per-tile cost), so the last round is as full as
// the shape allows (151,936 entries, 3 row tiles, 148 SMs: 240, 12.9 rounds).
int head_plan_bn(int mtiles, int V, int sms) {
    int best = sv::HEAD_BN;
    long long best_cost = LLONG_MAX;
    for (int bn = sv::HEAD_BN; bn >= 64; bn -= 16) {
        const long long tiles = static_cast<long long>(mtiles) * ceil_div(V, bn);
        const long long cost = ceil_div(tiles, sms) * (bn + 16);
        if (cost < best_cost) {
            best_cost = cost;
            best = bn;
        }
    }
    return best;
}

// Workspace of the fused path: each row's running best (8 bytes) and the
// timeout flag, zeroed by one memset per call.  0 on invalid sizes.
size_t head_ws_bytes(int B, int k, int V) {
    if (B <= 0 || k < 1 || V < 1) return 0;
    const long long rows = static_cast<long long>(B) * (k + 1);
    const long long vt = ceil_div(V, sv::HEAD_BN);
    if (rows > INT_MAX / 2 || vt > kHeadMaxVTiles) return 0;
    return static_cast<size_t>(round_up(rows * 8, 16) + 16);
}

}  // namespace

extern "C" {

sv_status_t spec_verify_tree_ex(const void* target_logits, const void* draft_logits, const int32_t* tokens,
                                const int32_t* parents, const float* uniforms, int B, int N, int V,
                                const float* temperature, int top_k, int mode, int32_t* out_tokens,
                                int32_t* out_n_accepted, int32_t* out_nodes, float* out_p, float* out_q,
                                void* workspace, size_t workspace_bytes, void* stream) {
    bool greedy = false;
    int dt = 0;
    if (B <= 0 || N < 1 || N > sv::TREE_MAX_NODES || V < 1 || top_k < 0) return SV_ERR_INVALID_ARG;
    if (!decode_mode(mode, &greedy, &dt)) return SV_ERR_INVALID_ARG;
    const int elt = dt ? 4 : 2;
    if (static_cast<unsigned long long>(B) * (N + 1) > (1ULL << 62) / (static_cast<unsigned long long>(V) * 4ULL))
        return SV_ERR_INVALID_ARG;
    if (!target_logits || !tokens || !parents || !out_tokens || !out_n_accepted) return SV_ERR_INVALID_ARG;
    if (!greedy && (!draft_logits || !uniforms)) return SV_ERR_INVALID_ARG;
    if (!aligned(target_logits, elt) || (draft_logits && !aligned(draft_logits, elt)) || !aligned(tokens, 4) ||
        !aligned(parents, 4) || (uniforms && !aligned(uniforms, 4)) || (temperature && !aligned(temperature, 4)) ||
        !aligned(out_tokens, 4) || !aligned(out_n_accepted, 4) || (out_nodes && !aligned(out_nodes, 4)) ||
        (out_p && !aligned(out_p, 4)) || (out_q && !aligned(out_q, 4)))
        return SV_ERR_INVALID_ARG;
    if (workspace && !aligned(workspace, 16)) return SV_ERR_INVALID_ARG;
    if (V > sv::TREE_SEG * sv::TREE_MAX_SEG) return SV_ERR_UNSUPPORTED;
    int dev = 0;
    const DeviceInfo* info = device_info(&dev);
    if (!info) return SV_ERR_UNSUPPORTED;
    const int K = (!greedy && top_k > 0 && top_k < V) ? top_k : 0;
    TreePlan tp;
    tree_plan(*info, B, N, V, dt, greedy, K, &tp);
    const bool fast = workspace && tp.fast && workspace_bytes >= tp.ws_bytes;
    if (workspace && tp.fast && workspace_bytes < tp.ws_bytes) return SV_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int* done = nullptr;
    if (fast) {
        const Plan& p = tp.k1;
        sv_status_t s = set_attrs(dev, dt, p.nt1, p.mode, false);
        if (s != SV_OK) return s;
        auto* base = static_cast<unsigned char*>(workspace);
        done = reinterpret_cast<int*>(base + tp.off_done);
        sv::RowsParams r;
        std::memset(&r, 0, sizeof r);
        r.B = B;
        r.k = N;  // rows b*(N+1) + n: the sequence of a row is row / (N+1)
        r.V = V;
        r.top_k = K;
        r.temperature = greedy ? nullptr : temperature;
        r.nseg = p.nseg;
        r.spc = p.spc;
        r.nch = p.nch;
        r.stages = p.stages;
        r.lcap = p.lcap;
        r.kcap = p.kcap;
        r.timeout_ns = kDefaultTimeoutNs;
        r.procs_div = 1;
        int slot = 0;
        RowsFn f1 = pick_rows(dt, p.nt1, p.mode, false, &slot);
        cudaLaunchConfig_t c1;
        std::memset(&c1, 0, sizeof c1);
        c1.gridDim = dim3(static_cast<unsigned>(static_cast<long long>(B) * (N + 1)), 1, 1);
        c1.blockDim = dim3(p.nt1 + 32, 1, 1);
        c1.dynamicSmemBytes = p.smem1;
        c1.stream = st;
        // the streaming pass over the target rows, then over the draft rows
        for (int side = 0; side < (greedy ? 1 : 2); ++side) {
            r.target = side ? draft_logits : target_logits;
            r.segs = reinterpret_cast<sv::SegRec*>(base + tp.off_gt);
            r.chunks = reinterpret_cast<sv::ChunkRec*>(base + (side ? tp.off_cd : tp.off_ct));
            r.cands = reinterpret_cast<sv::Cand*>(base + (side ? tp.off_ld : tp.off_lt));
            if (cudaLaunchKernelEx(&c1, f1, r) != cudaSuccess) {
                cudaGetLastError();
                return SV_ERR_CUDA;
            }
        }
        sv::TreeListParams lp;
        std::memset(&lp, 0, sizeof lp);
        lp.ct = reinterpret_cast<sv::ChunkRec*>(base + tp.off_ct);
        lp.lt = reinterpret_cast<sv::Cand*>(base + tp.off_lt);
        lp.cd = reinterpret_cast<sv::ChunkRec*>(base + tp.off_cd);
        lp.ld = reinterpret_cast<sv::Cand*>(base + tp.off_ld);
        lp.gt = reinterpret_cast<sv::SegRec*>(base + tp.off_gt);
        lp.nseg = p.nseg;
        lp.kcap = p.kcap;
        lp.tokens = tokens;
        lp.parents = parents;
        lp.uniforms = greedy ? nullptr : uniforms;
        lp.temperature = greedy ? nullptr : temperature;
        lp.B = B;
        lp.N = N;
        lp.V = V;
        lp.greedy = greedy ? 1 : 0;
        lp.out_tokens = out_tokens;
        lp.out_n = out_n_accepted;
        lp.out_nodes = out_nodes;
        lp.out_p = greedy ? nullptr : out_p;
        lp.out_q = greedy ? nullptr : out_q;
        lp.done = done;
        cudaLaunchConfig_t cl2;
        std::memset(&cl2, 0, sizeof cl2);
        cl2.gridDim = dim3(static_cast<unsigned>(B), 1, 1);
        cl2.blockDim = dim3(sv::TREE_LIST_NT, 1, 1);
        cl2.stream = st;
        TreeListFn fl = sv::sv_tree_list_kernel;
        if (cudaLaunchKernelEx(&cl2, fl, lp) != cudaSuccess) {
            cudaGetLastError();
            return SV_ERR_CUDA;
        }
    }
    // the row walk: every sequence, or those the list walk left
    sv::TreeParams t;
    std::memset(&t, 0, sizeof t);
    t.target = target_logits;
    t.draft = greedy ? nullptr : draft_logits;
    t.tokens = tokens;
    t.parents = parents;
    t.uniforms = greedy ? nullptr : uniforms;
    t.temperature = greedy ? nullptr : temperature;
    t.B = B;
    t.N = N;
    t.V = V;
    t.top_k = K;
    t.greedy = greedy ? 1 : 0;
    t.out_tokens = out_tokens;
    t.out_n = out_n_accepted;
    t.out_nodes = out_nodes;
    t.out_p = greedy ? nullptr : out_p;
    t.out_q = greedy ? nullptr : out_q;
    t.done = done;
    cudaLaunchConfig_t ct;
    std::memset(&ct, 0, sizeof ct);
    ct.gridDim = dim3(static_cast<unsigned>(B), 1, 1);
    ct.blockDim = dim3(sv::TREE_NT, 1, 1);
    ct.stream = st;
    TreeFn ft = dt ? sv::sv_tree_kernel<1> : sv::sv_tree_kernel<0>;
    if (cudaLaunchKernelEx(&ct, ft, t) != cudaSuccess) {
        cudaGetLastError();
        return SV_ERR_CUDA;
    }
    return SV_OK;
}

sv_status_t spec_verify_tree(const void* target_logits, const void* draft_logits, const int32_t* tokens,
                             const int32_t* parents, const float* uniforms, int B, int N, int V,
                             const float* temperature, int top_k, int mode, int32_t* out_tokens,
                             int32_t* out_n_accepted, int32_t* out_nodes, float* out_p, float* out_q,
                             void* stream) {
    return spec_verify_tree_ex(target_logits, draft_logits, tokens, parents, uniforms, B, N, V, temperature, top_k,
                               mode, out_tokens, out_n_accepted, out_nodes, out_p, out_q, nullptr, 0, stream);
}

size_t spec_verify_tree_workspace_size(int B, int N, int V, int top_k, int mode) {
    bool greedy = false;
    int dt = 0;
    if (B <= 0 || N < 1 || N > sv::TREE_MAX_NODES || V < 1 || top_k < 0) return 0;
    if (!decode_mode(mode, &greedy, &dt)) return 0;
    int dev = 0;
    const DeviceInfo* info = device_info(&dev);
    if (!info) return 0;
    const int K = (!greedy && top_k > 0 && top_k < V) ? top_k : 0;
    TreePlan tp;
    tree_plan(*info, B, N, V, dt, greedy, K, &tp);
    return tp.fast ? tp.ws_bytes : 0;
}

sv_status_t spec_verify_ex(const void* target_logits, const void* draft_logits, const int32_t* draft_tokens,
                           const float* uniforms, int B, int k, int V, const float* temperature, int top_k,
                           int mode, int32_t* out_tokens, int32_t* out_n_accepted, float* out_p, float* out_q,
                           int32_t* out_status, void* workspace, size_t workspace_bytes,
                           const sv_options_t* opts, void* stream) {
    Call cl;
    const sv_status_t s = verify_args(target_logits, draft_logits, draft_tokens, uniforms, B, k, V, temperature,
                                      top_k, mode, out_tokens, out_n_accepted, out_p, out_q, out_status, opts,
                                      true, &cl);
    if (s != SV_OK) return s;
    return run(cl, workspace, workspace_bytes, opts, static_cast<cudaStream_t>(stream));
}

sv_status_t spec_verify_static(const void* target_logits, const void* draft_logits, const int32_t* draft_tokens,
                               const float* uniforms, int B, int k, int V, const float* temperature, int top_k,
                               int mode, int32_t* out_tokens, int32_t* out_n_accepted, float* out_p, float* out_q,
                               int32_t* out_status, const sv_options_t* opts, void* stream) {
    Call cl;
    sv_status_t s = verify_args(target_logits, draft_logits, draft_tokens, uniforms, B, k, V, temperature, top_k,
                                mode, out_tokens, out_n_accepted, out_p, out_q, out_status, opts, true, &cl);
    if (s != SV_OK) return s;
    int dev = 0;
    const DeviceInfo* info = device_info(&dev);
    if (!info) return SV_ERR_UNSUPPORTED;
    Plan p;
    if ((s = make_plan(*info, cl.seqs, cl.k, cl.V, cl.dt, cl.greedy, cl.top_k, opts, cl.nprocs, &p)) != SV_OK) return s;
    if (p.ws_bytes > SV_STATIC_WORKSPACE_BYTES) return SV_ERR_UNSUPPORTED;  // beyond the static buffer
    void* ws = static_scratch(dev);
    if (!ws) return SV_ERR_CUDA;
    return run(cl, ws, SV_STATIC_WORKSPACE_BYTES, opts, static_cast<cudaStream_t>(stream));
}

sv_status_t spec_verify(const void* target_logits, const void* draft_logits, const int32_t* draft_tokens,
                        const float* uniforms, int B, int k, int V, const float* temperature, int top_k,
                        int mode, int32_t* out_tokens, int32_t* out_n_accepted, void* stream) {
    return spec_verify_ex(target_logits, draft_logits, draft_tokens, uniforms, B, k, V, temperature, top_k,
                          mode, out_tokens, out_n_accepted, nullptr, nullptr, nullptr, nullptr, 0, nullptr,
                          stream);
}

size_t spec_verify_workspace_size(int B, int k, int V, int top_k, int mode, const sv_options_t* opts) {
    Call cl;
    if (verify_args(nullptr, nullptr, nullptr, nullptr, B, k, V, nullptr, top_k, mode, nullptr, nullptr,
                    nullptr, nullptr, nullptr, opts, false, &cl) != SV_OK)
        return 0;
    return workspace_for(cl, opts);
}

sv_status_t spec_sample_ex(const void* logits, const float* uniforms, int rows, int V, const float* temperature,
                           int top_k, int mode, int32_t* out_tokens, void* workspace, size_t workspace_bytes,
                           const sv_options_t* opts, void* stream) {
    Call cl;
    const sv_status_t s =
        sample_args(logits, uniforms, rows, V, temperature, top_k, mode, out_tokens, opts, true, &cl);
    if (s != SV_OK) return s;
    return run(cl, workspace, workspace_bytes, opts, static_cast<cudaStream_t>(stream));
}

sv_status_t spec_sample(const void* logits, const float* uniforms, int rows, int V, const float* temperature,
                        int top_k, int mode, int32_t* out_tokens, void* stream) {
    return spec_sample_ex(logits, uniforms, rows, V, temperature, top_k, mode, out_tokens, nullptr, 0, nullptr,
                          stream);
}

size_t spec_sample_workspace_size(int rows, int V, int top_k, int mode, const sv_options_t* opts) {
    Call cl;
    if (sample_args(nullptr, nullptr, rows, V, nullptr, top_k, mode, nullptr, opts, false, &cl) != SV_OK) return 0;
    return workspace_for(cl, opts);
}

sv_status_t spec_verify_head_greedy(const void* hidden, const void* weight, const int32_t* draft_tokens, int B,
                                    int k, int V, int H, int32_t* out_tokens, int32_t* out_n_accepted,
                                    int32_t* out_argmax, void* workspace, size_t workspace_bytes,
                                    const sv_options_t* opts, int32_t* out_status, void* stream) {
    if (B <= 0 || k < 1 || V < 1 || H < 1 || H % 8 != 0) return SV_ERR_INVALID_ARG;
    if (!hidden || !weight || !draft_tokens || !out_tokens || !out_n_accepted) return SV_ERR_INVALID_ARG;
    if (!aligned(hidden, 16) || !aligned(weight, 16) || !aligned(draft_tokens, 4) || !aligned(out_tokens, 4) ||
        !aligned(out_n_accepted, 4) || (out_argmax && !aligned(out_argmax, 4)) ||
        (out_status && !aligned(out_status, 4)))
        return SV_ERR_INVALID_ARG;
    const size_t need = head_ws_bytes(B, k, V);
    if (need == 0) return ceil_div(V, sv::HEAD_BN) > kHeadMaxVTiles ? SV_ERR_UNSUPPORTED : SV_ERR_INVALID_ARG;
    if (workspace && (!aligned(workspace, 16) || workspace_bytes < need)) return SV_ERR_INVALID_ARG;
    if (opts && check_options(opts) != SV_OK) return SV_ERR_INVALID_ARG;
    if (opts && (opts->top_p || opts->vocab_mask || opts->rep_ids)) return SV_ERR_UNSUPPORTED;  // greedy only
    int dev = 0;
    const DeviceInfo* info = device_info(&dev);
    if (!info) return SV_ERR_UNSUPPORTED;
    const int rows = B * (k + 1);
    const int mtiles = static_cast<int>(ceil_div(rows, sv::HEAD_BM));
    const int bn = head_plan_bn(mtiles, V, info->sms);
    const int vtiles = static_cast<int>(ceil_div(V, bn));
    CUtensorMap tm_h, tm_w;
    if (!tensor_map_encoder()) return SV_ERR_UNSUPPORTED;
    if (!encode_bf16_rows(&tm_h, hidden, static_cast<uint64_t>(H), static_cast<uint64_t>(rows), sv::HEAD_BM) ||
        !encode_bf16_rows(&tm_w, weight, static_cast<uint64_t>(H), static_cast<uint64_t>(V), static_cast<uint32_t>(bn)))
        return SV_ERR_INVALID_ARG;
    std::call_once(g_head_attr_once[dev], [dev] {
        g_head_attr_err[dev] =
            cudaFuncSetAttribute(sv::sv_head_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, sv::HEAD_SMEM);
        if (g_head_attr_err[dev] != cudaSuccess) cudaGetLastError();
    });
    if (g_head_attr_err[dev] != cudaSuccess) return SV_ERR_CUDA;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    void* ws = workspace;
    bool owned = false;
    if (!ws) {
        cudaMemPool_t pool = device_pool(dev);
        if (!pool || cudaMallocFromPoolAsync(&ws, need, pool, st) != cudaSuccess) {
            cudaGetLastError();
            return SV_ERR_CUDA;
        }
        g_pool_allocs.fetch_add(1, std::memory_order_relaxed);
        owned = true;
    }
    auto* base = static_cast<unsigned char*>(ws);
    int* err = reinterpret_cast<int*>(base + need - 16);
    sv::HeadParams P;
    P.rows = rows;
    P.V = V;
    P.H = H;
    P.bn = bn;
    P.mtiles = mtiles;
    P.tiles = mtiles * vtiles;
    P.best = reinterpret_cast<unsigned long long*>(base);
    P.err = err;
    P.timeout_ns = (opts && opts->wait_timeout_ns) ? opts->wait_timeout_ns : kDefaultTimeoutNs;
    P.test_hook = (opts && opts->test_extra_tx) ? 1 : 0;
    sv::HeadDecideParams D;
    D.best = P.best;
    D.err = err;
    D.draft_tokens = draft_tokens;
    D.B = B;
    D.k = k;
    D.V = V;
    D.out_tokens = out_tokens;
    D.out_n_accepted = out_n_accepted;
    D.out_argmax = out_argmax;
    D.out_status = out_status;

    sv_status_t result = SV_OK;
    do {
        if (cudaMemsetAsync(base, 0, need, st) != cudaSuccess) {  // the running bests and the flag
            result = SV_ERR_CUDA;
            break;
        }
        if (opts && opts->event_start &&
            cudaEventRecord(static_cast<cudaEvent_t>(opts->event_start), st) != cudaSuccess) {
            result = SV_ERR_CUDA;
            break;
        }
        // persistent: one CTA per SM (its shared memory admits no second)
        const int grid = P.tiles < info->sms ? P.tiles : info->sms;
        sv::sv_head_kernel<<<grid, sv::HEAD_NT, sv::HEAD_SMEM, st>>>(tm_h, tm_w, P);
        if (cudaGetLastError() != cudaSuccess) {
            result = SV_ERR_CUDA;
            break;
        }
        if (opts && opts->event_stop &&
            cudaEventRecord(static_cast<cudaEvent_t>(opts->event_stop), st) != cudaSuccess) {
            result = SV_ERR_CUDA;
            break;
        }
        cudaLaunchAttribute a[1];
        a[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        a[0].val.programmaticStreamSerializationAllowed = 1;
        cudaLaunchConfig_t c;
        std::memset(&c, 0, sizeof c);
        c.gridDim = dim3(static_cast<unsigned>(ceil_div(B, sv::HEAD_DECIDE_NT / 32)), 1, 1);
        c.blockDim = dim3(sv::HEAD_DECIDE_NT, 1, 1);
        c.stream = st;
        c.attrs = a;
        c.numAttrs = 1;
        if (cudaLaunchKernelEx(&c, sv::sv_head_decide_kernel, D) != cudaSuccess) {
            result = SV_ERR_CUDA;
            break;
        }
    } while (false);
    if (result != SV_OK) cudaGetLastError();
    if (owned && cudaFreeAsync(ws, st) != cudaSuccess) {
        cudaGetLastError();
        if (result == SV_OK) result = SV_ERR_CUDA;
    }
    return result;
}

size_t spec_verify_head_workspace_size(int B, int k, int V, int H) {
    if (H < 1 || H % 8 != 0) return 0;
    return head_ws_bytes(B, k, V);
}

const char* spec_verify_status_string(sv_status_t status) {
    switch (status) {
        case SV_OK: return "ok";
        case SV_ERR_INVALID_ARG: return "invalid argument";
        case SV_ERR_UNSUPPORTED: return "unsupported device or size";
        case SV_ERR_CUDA: return "CUDA launch failure";
        case SV_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    }
    return "unknown status";
}

int spec_verify_version(void) { return kVersion; }

unsigned long long spec_verify_pool_allocations(void) { return g_pool_allocs.load(std::memory_order_relaxed); }

}  // extern "C"
