// Host side of the spec_verify C ABI: argument checks, launch planning and
// the launches themselves.  Nothing here allocates device memory or
// synchronises the caller's stream.
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/spec_verify.h"
#include "sv_kernels.cuh"

namespace {

constexpr int kVersion = 10000;  // 1.0.0
constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultTimeoutNs = 1000000000ull;

struct DeviceInfo {
    int ok = 0;
    int sms = 0;
    int smem_optin = 0;
};

DeviceInfo g_dev[kMaxDevices];
std::once_flag g_dev_once[kMaxDevices];
std::once_flag g_attr_once[kMaxDevices][6];

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

const DeviceInfo* device_info(int* dev_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return nullptr;
    }
    std::call_once(g_dev_once[dev], [dev] {
        DeviceInfo& d = g_dev[dev];
        int major = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
                cudaSuccess) {
            cudaGetLastError();
            d.ok = 0;
            return;
        }
        d.ok = major >= 9 ? 1 : 0;
    });
    *dev_out = dev;
    return g_dev[dev].ok ? &g_dev[dev] : nullptr;
}

using KernelFn = void (*)(sv::Params);

KernelFn pick_kernel(int dt, int nt, int* slot) {
    if (dt == 0) {
        if (nt == 128) { *slot = 0; return sv::sv_unit_kernel<0, 128>; }
        if (nt == 512) { *slot = 2; return sv::sv_unit_kernel<0, 512>; }
        *slot = 1;
        return sv::sv_unit_kernel<0, 256>;
    }
    if (nt == 128) { *slot = 3; return sv::sv_unit_kernel<1, 128>; }
    if (nt == 512) { *slot = 5; return sv::sv_unit_kernel<1, 512>; }
    *slot = 4;
    return sv::sv_unit_kernel<1, 256>;
}

struct Plan {
    int C = 1, NT = 256, L = 0, piece_bytes = 0, buf_bytes = 0, group_lanes = 32, use_cand = 0;
    size_t smem = 0;
};

int ceil_div(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }
int round_up(long long a, long long b) { return static_cast<int>((a + b - 1) / b * b); }

// Choose cluster size, slice length and shared-memory layout for a launch of
// `units` units of `rows_per_unit` rows of V elements.
sv_status_t make_plan(const DeviceInfo& dev, long long units, int rows_per_unit, int V, int elt,
                      int top_k, const sv_options_t* opts, Plan* out) {
    Plan p;
    const int vec = 16 / elt;
    p.NT = (opts && opts->threads) ? opts->threads : 256;
    const long long unit_bytes = static_cast<long long>(rows_per_unit) * V * elt;
    const int smem_budget = dev.smem_optin - sv::CTL_BYTES - 256;
    int C;
    if (opts && opts->cluster_size) {
        C = opts->cluster_size;
    } else {
        // about 40 KB of logits per CTA, more CTAs for small batches
        C = 1;
        while (C < 16 && unit_bytes > static_cast<long long>(C) * 40 * 1024) C *= 2;
        while (C < 16 && units * C < 2LL * dev.sms) C *= 2;
        // no CTA should get an empty slice
        while (C > 1 && static_cast<long long>(C - 1) * round_up(ceil_div(V, C), vec) >= V) C /= 2;
    }
    for (;;) {
        p.C = C;
        p.L = round_up(ceil_div(V, C), vec);
        p.buf_bytes = round_up(static_cast<long long>(p.L) * elt + 32, 128);
        if (static_cast<long long>(p.buf_bytes) * rows_per_unit <= smem_budget) break;
        if (opts && opts->cluster_size) return SV_ERR_UNSUPPORTED;
        if (C >= 16) return SV_ERR_UNSUPPORTED;
        C *= 2;
    }
    p.piece_bytes = round_up(ceil_div(p.buf_bytes, sv::MAX_PIECES), 16);
    if (p.piece_bytes < 8192) p.piece_bytes = 8192;
    p.smem = static_cast<size_t>(sv::CTL_BYTES) + static_cast<size_t>(p.buf_bytes) * rows_per_unit;
    // top-k lower bound groups: enough groups for a tight bound, within GMAX
    p.use_cand = 0;
    p.group_lanes = 32;
    if (top_k > 0 && !(opts && opts->topk_path == 2)) {
        int best = 0;
        for (int g = 32; g >= 1; g >>= 1) {
            const long long Gt = static_cast<long long>(C) * (p.NT / g);
            if (Gt > sv::GMAX) break;
            if (Gt >= top_k) {
                best = g;
                if (Gt >= 2LL * top_k) break;
            }
        }
        if (best && top_k <= sv::CAND_CAP / 2) {
            p.group_lanes = best;
            p.use_cand = 1;
        }
    }
    if (opts && opts->topk_path == 1 && top_k > 0 && !p.use_cand) return SV_ERR_UNSUPPORTED;
    if (static_cast<long long>(p.buf_bytes) / 16 > static_cast<long long>(sv::MAX_TILES) * p.NT)
        return SV_ERR_UNSUPPORTED;
    if (units > INT_MAX / C) return SV_ERR_INVALID_ARG;
    *out = p;
    return SV_OK;
}

sv_status_t launch_units(const sv::Params& prm, const Plan& plan, int dt, int dev, cudaStream_t stream) {
    int slot = 0;
    KernelFn fn = pick_kernel(dt, plan.NT, &slot);
    cudaError_t aerr = cudaSuccess;
    std::call_once(g_attr_once[dev][slot], [&] {
        aerr = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, g_dev[dev].smem_optin);
        if (aerr == cudaSuccess)
            aerr = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    });
    if (aerr != cudaSuccess) {
        cudaGetLastError();
        return SV_ERR_CUDA;
    }
    const long long grid = (prm.sample_only ? prm.B : prm.B * (prm.k + 1)) * plan.C;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(plan.NT, 1, 1);
    cfg.dynamicSmemBytes = plan.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = plan.C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, fn, prm) != cudaSuccess) {
        cudaGetLastError();
        return SV_ERR_CUDA;
    }
    return SV_OK;
}

sv_status_t launch_finalize(int32_t* tokens, const int32_t* draft_tokens, int32_t* n_accepted,
                            int32_t* status, long long B, int k, cudaStream_t stream) {
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3(static_cast<unsigned>((B + 255) / 256), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, sv::sv_finalize_kernel, tokens, draft_tokens, n_accepted, status, B, k) !=
        cudaSuccess) {
        cudaGetLastError();
        return SV_ERR_CUDA;
    }
    return SV_OK;
}

sv_status_t check_options(const sv_options_t* o) {
    if (!o) return SV_OK;
    const int c = o->cluster_size;
    if (!(c == 0 || c == 1 || c == 2 || c == 4 || c == 8 || c == 16)) return SV_ERR_INVALID_ARG;
    if (!(o->threads == 0 || o->threads == 128 || o->threads == 256 || o->threads == 512))
        return SV_ERR_INVALID_ARG;
    if (o->topk_path < 0 || o->topk_path > 2) return SV_ERR_INVALID_ARG;
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

}  // namespace

extern "C" {

sv_status_t spec_verify_ex(const void* target_logits, const void* draft_logits, const int32_t* draft_tokens,
                           const float* uniforms, int B, int k, int V, const float* temperature, int top_k,
                           int mode, int32_t* out_tokens, int32_t* out_n_accepted, float* out_p, float* out_q,
                           int32_t* out_status, const sv_options_t* opts, void* stream) {
    bool greedy = false;
    int dt = 0;
    if (B <= 0 || k < 1 || V < 1 || top_k < 0) return SV_ERR_INVALID_ARG;
    if (!decode_mode(mode, &greedy, &dt)) return SV_ERR_INVALID_ARG;
    if (check_options(opts) != SV_OK) return SV_ERR_INVALID_ARG;
    const int elt = dt ? 4 : 2;
    if (!target_logits || !draft_tokens || !out_tokens || !out_n_accepted) return SV_ERR_INVALID_ARG;
    if (!greedy && (!draft_logits || !uniforms)) return SV_ERR_INVALID_ARG;
    if (!aligned(target_logits, elt) || (draft_logits && !aligned(draft_logits, elt))) return SV_ERR_INVALID_ARG;
    if (!aligned(draft_tokens, 4) || !aligned(out_tokens, 4) || !aligned(out_n_accepted, 4) ||
        (uniforms && !aligned(uniforms, 4)) || (temperature && !aligned(temperature, 4)) ||
        (out_p && !aligned(out_p, 4)) || (out_q && !aligned(out_q, 4)) ||
        (out_status && !aligned(out_status, 4)))
        return SV_ERR_INVALID_ARG;
    // element counts must fit in 64-bit byte offsets
    if (static_cast<unsigned long long>(B) * static_cast<unsigned long long>(k + 1) >
        (1ULL << 62) / (static_cast<unsigned long long>(V) * 4ULL))
        return SV_ERR_INVALID_ARG;
    const int eff_topk = (top_k > 0 && top_k < V && !greedy) ? top_k : 0;

    int dev = 0;
    const DeviceInfo* info = device_info(&dev);
    if (!info) return SV_ERR_UNSUPPORTED;
    const long long units = static_cast<long long>(B) * (k + 1);
    Plan plan;
    const sv_status_t ps = make_plan(*info, units, greedy ? 1 : 2, V, elt, eff_topk, opts, &plan);
    if (ps != SV_OK) return ps;

    sv::Params prm;
    std::memset(&prm, 0, sizeof prm);
    prm.target = target_logits;
    prm.draft = draft_logits;
    prm.draft_tokens = draft_tokens;
    prm.uniforms = uniforms;
    prm.temperature = temperature;
    prm.out_codes = out_tokens;
    prm.out_p = greedy ? nullptr : out_p;
    prm.out_q = greedy ? nullptr : out_q;
    prm.out_status = out_status;
    prm.B = B;
    prm.k = k;
    prm.V = V;
    prm.top_k = eff_topk;
    prm.greedy = greedy ? 1 : 0;
    prm.sample_only = 0;
    prm.C = plan.C;
    prm.L = plan.L;
    prm.piece_bytes = plan.piece_bytes;
    prm.buf_bytes = plan.buf_bytes;
    prm.group_lanes = plan.group_lanes;
    prm.use_cand = plan.use_cand;
    prm.timeout_ns = (opts && opts->wait_timeout_ns) ? opts->wait_timeout_ns : kDefaultTimeoutNs;
    prm.test_extra_tx = opts ? opts->test_extra_tx : 0u;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (opts && opts->event_start &&
        cudaEventRecord(static_cast<cudaEvent_t>(opts->event_start), st) != cudaSuccess) {
        cudaGetLastError();
        return SV_ERR_CUDA;
    }
    sv_status_t s = launch_units(prm, plan, dt, dev, st);
    if (s != SV_OK) return s;
    if (opts && opts->event_stop &&
        cudaEventRecord(static_cast<cudaEvent_t>(opts->event_stop), st) != cudaSuccess) {
        cudaGetLastError();
        return SV_ERR_CUDA;
    }
    return launch_finalize(out_tokens, draft_tokens, out_n_accepted, out_status, B, k, st);
}

sv_status_t spec_verify(const void* target_logits, const void* draft_logits, const int32_t* draft_tokens,
                        const float* uniforms, int B, int k, int V, const float* temperature, int top_k,
                        int mode, int32_t* out_tokens, int32_t* out_n_accepted, void* stream) {
    return spec_verify_ex(target_logits, draft_logits, draft_tokens, uniforms, B, k, V, temperature, top_k,
                          mode, out_tokens, out_n_accepted, nullptr, nullptr, nullptr, nullptr, stream);
}

sv_status_t spec_sample_ex(const void* logits, const float* uniforms, int rows, int V, const float* temperature,
                           int top_k, int mode, int32_t* out_tokens, const sv_options_t* opts, void* stream) {
    bool greedy = false;
    int dt = 0;
    if (rows <= 0 || V < 1 || top_k < 0) return SV_ERR_INVALID_ARG;
    if (!decode_mode(mode, &greedy, &dt)) return SV_ERR_INVALID_ARG;
    if (check_options(opts) != SV_OK) return SV_ERR_INVALID_ARG;
    const int elt = dt ? 4 : 2;
    if (!logits || !out_tokens) return SV_ERR_INVALID_ARG;
    if (!greedy && !uniforms) return SV_ERR_INVALID_ARG;
    if (!aligned(logits, elt) || !aligned(out_tokens, 4) || (uniforms && !aligned(uniforms, 4)) ||
        (temperature && !aligned(temperature, 4)))
        return SV_ERR_INVALID_ARG;
    if (static_cast<unsigned long long>(rows) > (1ULL << 62) / (static_cast<unsigned long long>(V) * 4ULL))
        return SV_ERR_INVALID_ARG;
    const int eff_topk = (top_k > 0 && top_k < V && !greedy) ? top_k : 0;

    int dev = 0;
    const DeviceInfo* info = device_info(&dev);
    if (!info) return SV_ERR_UNSUPPORTED;
    Plan plan;
    const sv_status_t ps = make_plan(*info, rows, 1, V, elt, eff_topk, opts, &plan);
    if (ps != SV_OK) return ps;

    sv::Params prm;
    std::memset(&prm, 0, sizeof prm);
    prm.target = logits;
    prm.uniforms = uniforms;
    prm.temperature = temperature;
    prm.out_codes = out_tokens;
    prm.B = rows;
    prm.k = 0;
    prm.V = V;
    prm.top_k = eff_topk;
    prm.greedy = greedy ? 1 : 0;
    prm.sample_only = 1;
    prm.C = plan.C;
    prm.L = plan.L;
    prm.piece_bytes = plan.piece_bytes;
    prm.buf_bytes = plan.buf_bytes;
    prm.group_lanes = plan.group_lanes;
    prm.use_cand = plan.use_cand;
    prm.timeout_ns = (opts && opts->wait_timeout_ns) ? opts->wait_timeout_ns : kDefaultTimeoutNs;
    prm.test_extra_tx = opts ? opts->test_extra_tx : 0u;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (opts && opts->event_start &&
        cudaEventRecord(static_cast<cudaEvent_t>(opts->event_start), st) != cudaSuccess) {
        cudaGetLastError();
        return SV_ERR_CUDA;
    }
    sv_status_t s = launch_units(prm, plan, dt, dev, st);
    if (s != SV_OK) return s;
    if (opts && opts->event_stop &&
        cudaEventRecord(static_cast<cudaEvent_t>(opts->event_stop), st) != cudaSuccess) {
        cudaGetLastError();
        return SV_ERR_CUDA;
    }
    return SV_OK;
}

sv_status_t spec_sample(const void* logits, const float* uniforms, int rows, int V, const float* temperature,
                        int top_k, int mode, int32_t* out_tokens, void* stream) {
    return spec_sample_ex(logits, uniforms, rows, V, temperature, top_k, mode, out_tokens, nullptr, stream);
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

}  // extern "C"
