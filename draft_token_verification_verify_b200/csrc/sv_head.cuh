// Greedy verification fused into the target's output projection.
//
// The target scores the k+1 positions of every sequence in one forward pass
// (entry "推测解码", section "提议与核验的基本步骤", paragraph 1); greedy
// verification needs only each position's lowest-index argmax (paragraph 4).
// K_head computes the logits z = h . W[v] in tiles of 128 rows x up to 256
// vocabulary entries on the tensor cores (tcgen05.mma, bf16 operands staged by
// 2D tensor-map copies in the 128-byte-swizzled K-major layout, fp32
// accumulators in tensor memory; one persistent CTA per SM works through the
// tiles) and its epilogue reduces each tile to each row's (maximum, lowest
// index) straight out of tensor memory and folds it into the row's running
// best with one 64-bit atomic maximum: the logits are never written.
// K_decide walks the chain on the rows' results.
#pragma once

#include <cuda.h>  // CUtensorMap (the type only; the map is encoded on the host)

#include <cstdint>

#include "sv_ptx.cuh"

namespace sv {

constexpr int HEAD_BM = 128;  // hidden-state rows per tile: the tensor-memory lanes
constexpr int HEAD_BN = 256;  // vocabulary entries per tile at most: fp32 tensor-memory columns
constexpr int HEAD_BK = 64;   // K per stage: one 128-byte swizzle row of bf16
constexpr int HEAD_STAGES = 4;
// six warps: 0 issues the copies, 1 the MMAs, 2-5 read tensor memory (warp w
// reaches the 32-lane quarter w % 4, so the four cover all 128 lanes)
constexpr int HEAD_NT = 192;
constexpr int HEAD_ACCS = 2;  // accumulators in tensor memory: the epilogue of one tile overlaps the next's MMAs
constexpr int HEAD_TMEM_COLS = HEAD_ACCS * HEAD_BN;
constexpr int HEAD_A_BYTES = HEAD_BM * HEAD_BK * 2;
constexpr int HEAD_B_BYTES = HEAD_BN * HEAD_BK * 2;
constexpr int HEAD_STAGE_BYTES = HEAD_A_BYTES + HEAD_B_BYTES;
// stages, 1 KB of slack to align them to the 1,024-byte swizzle period, barriers
constexpr int HEAD_SMEM = HEAD_STAGES * HEAD_STAGE_BYTES + 1024 + 256;
// each CTA allocates all 512 tensor-memory columns of its SM, so no second CTA
// may ever be resident beside it: its shared memory alone rules that out
// (228 KB per SM, 1 KB of it reserved per CTA)
static_assert(2 * (HEAD_SMEM + 1024) > 228 * 1024, "two projection CTAs must not fit on one SM");
constexpr int HEAD_DECIDE_NT = 128;  // one warp per sequence

// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulator (bits 4-5),
// bf16 A and B (bits 7-9, 10-12), both K-major (bits 15, 16 clear), N / 8 at
// bit 17, M / 16 at bit 24; N = bn, the tile's vocabulary entries.
__host__ __device__ constexpr uint32_t head_idesc(int bn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(bn >> 3) << 17) |
           (static_cast<uint32_t>(HEAD_BM >> 4) << 24);
}

// A row's running best as one orderable 64-bit word: the order-preserving
// bits of the largest logit (-0.0 taken as +0.0) above the complement of its
// index, so the unsigned maximum picks the largest value and, among equal
// values, the lowest index.  0: no finite logit seen; all ones: a NaN or +inf.
constexpr unsigned long long HEAD_BAD = ~0ull;

__device__ __forceinline__ unsigned long long head_key(float z, int v) {
    const uint32_t b = __float_as_uint(z == 0.f ? 0.f : z);
    const uint32_t o = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    return (static_cast<unsigned long long>(o) << 32) | static_cast<uint32_t>(0xFFFFFFFFu - static_cast<uint32_t>(v));
}

struct HeadParams {
    int rows;  // B * (k + 1)
    int V;
    int H;
    int bn;      // vocabulary entries per tile: a multiple of 16 in [64, HEAD_BN]
    int mtiles;  // ceil(rows / HEAD_BM)
    int tiles;   // mtiles * ceil(V / bn)
    unsigned long long* best;  // [rows], zeroed before the launch
    int* err;                  // set to non-zero by a wait that ran out
    unsigned long long timeout_ns;
    int test_hook;  // non-zero: the epilogue also waits for an accumulator phase that never comes
};

struct HeadDecideParams {
    const unsigned long long* best;
    const int* err;
    const int32_t* draft_tokens;  // [B][k]
    int B, k, V;
    int32_t* out_tokens;      // [B][k+1]
    int32_t* out_n_accepted;  // [B]
    int32_t* out_argmax;      // [B][k+1] or null
    int32_t* out_status;      // or null
};

// ---- tensor-core, tensor-memory and tensor-map wrappers ----------------------

// Shared-memory matrix descriptor of a K-major operand in the 128-byte
// swizzled layout: 8-row x 128-byte atoms, 1,024 bytes apart (stride byte
// offset); the leading byte offset is unused for this layout; version 1 for
// sm_100; swizzle mode 2 (128 B) in bits 61-63.  The atom base must be
// 1,024-byte aligned; advancing the start address by 32 bytes selects the
// next 16 elements of K inside the swizzled row.
__device__ __forceinline__ uint64_t head_desc(uint32_t saddr) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
           (static_cast<uint64_t>(2) << 61);
}

__device__ __forceinline__ void tmap_prefetch(const CUtensorMap* m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 2D tiled copy global -> shared of box (x .. x+box0, y .. y+box1); elements
// outside the tensor read as zero.  x * 2 bytes is a multiple of 16 here.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* m, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D (tensor memory) = A . B^T (+ D when `acc`), K = 16, bf16; M and N from `idesc`.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}

// Arrive once on `bar` when every tcgen05.mma this thread issued so far is done.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// 32 consecutive fp32 columns of this warp's 32 lanes (one row per thread).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
          "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
          "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---- K_head: logits tiles on the tensor cores, (max, argmax) per row -----------
//
// Persistent: one CTA per SM takes the tiles blockIdx.x, blockIdx.x + grid, ...
// of the order (row tile fastest, then vocabulary tile), so the CTAs running
// at one time cover whole groups of row tiles of the same vocabulary tile and
// a weight tile comes from HBM once and from L2 for the others.  Warp 0's lane
// 0 streams the copies of every tile through one ring of HEAD_STAGES stages;
// warp 1's lane 0 issues each tile's MMAs into one of two accumulators; warps
// 2-5 reduce a finished accumulator while the next tile's MMAs run in the
// other.  Every wait is bounded; a wait that runs out sets *err, the roles
// stop, and the CTA drains its copies and MMAs before it frees tensor memory.
__global__ void __launch_bounds__(HEAD_NT, 1)
    sv_head_kernel(const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_w,
                   HeadParams P) {
    extern __shared__ __align__(1024) unsigned char head_raw[];
    const uint32_t raw_s = smem_u32(head_raw);
    unsigned char* base = head_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    uint64_t* full = reinterpret_cast<uint64_t*>(base + HEAD_STAGES * HEAD_STAGE_BYTES);
    uint64_t* empty = full + HEAD_STAGES;
    uint64_t* tfull = empty + HEAD_STAGES;  // an accumulator holds a finished tile
    uint64_t* tempty = tfull + HEAD_ACCS;   // the epilogue has read it
    uint64_t* done = tempty + HEAD_ACCS;    // every MMA of this CTA is complete
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nk = (P.H + HEAD_BK - 1) / HEAD_BK;
    const int bn = P.bn;
    const uint32_t stage_tx = static_cast<uint32_t>(HEAD_A_BYTES + bn * HEAD_BK * 2);  // the two boxes

    if (tid == 0) {
        for (int s = 0; s < HEAD_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < HEAD_ACCS; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 4);  // one arrival per epilogue warp
        }
        mbar_init(done, 1);
        fence_mbar_init();
        tmap_prefetch(&tm_h);
        tmap_prefetch(&tm_w);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, HEAD_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    int failed = 0;

    if (warp == 0 && lane == 0) {
        int it = 0;  // stage uses so far, across tiles
        for (int t = blockIdx.x; t < P.tiles && !failed; t += gridDim.x) {
            const int m0 = (t % P.mtiles) * HEAD_BM, n0 = (t / P.mtiles) * bn;
            for (int kb = 0; kb < nk; ++kb, ++it) {
                const int s = it % HEAD_STAGES;
                if (it >= HEAD_STAGES &&
                    !mbar_wait_bounded(&empty[s], ((it / HEAD_STAGES) - 1) & 1, P.timeout_ns)) {
                    failed = 1;
                    break;
                }
                unsigned char* st = base + s * HEAD_STAGE_BYTES;
                mbar_arrive_expect_tx(&full[s], stage_tx);
                tma_load_2d(st, &tm_h, kb * HEAD_BK, m0, &full[s]);
                tma_load_2d(st + HEAD_A_BYTES, &tm_w, kb * HEAD_BK, n0, &full[s]);
            }
        }
        // no copy may land after the CTA is gone: wait for the last ones issued
        for (int j = it > HEAD_STAGES ? it - HEAD_STAGES : 0; j < it; ++j)
            if (!mbar_wait_bounded(&full[j % HEAD_STAGES], (j / HEAD_STAGES) & 1, P.timeout_ns)) failed = 1;
    } else if (warp == 1 && lane == 0) {
        int it = 0, lt = 0;
        const uint32_t idesc = head_idesc(bn);
        for (int t = blockIdx.x; t < P.tiles && !failed; t += gridDim.x, ++lt) {
            const int acc = lt & 1;
            if (lt >= HEAD_ACCS && !mbar_wait_bounded(&tempty[acc], ((lt >> 1) - 1) & 1, P.timeout_ns)) {
                failed = 1;
                break;
            }
            tc_fence_after();
            const uint32_t d = tmem + static_cast<uint32_t>(acc * HEAD_BN);
            for (int kb = 0; kb < nk; ++kb, ++it) {
                const int s = it % HEAD_STAGES;
                if (!mbar_wait_bounded(&full[s], (it / HEAD_STAGES) & 1, P.timeout_ns)) {
                    failed = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t a = smem_u32(base + s * HEAD_STAGE_BYTES);
                const uint32_t b = a + HEAD_A_BYTES;
#pragma unroll
                for (int kk = 0; kk < HEAD_BK / 16; ++kk)
                    umma_bf16(d, head_desc(a + kk * 32), head_desc(b + kk * 32), idesc, (kb | kk) != 0 ? 1u : 0u);
                umma_commit(&empty[s]);  // frees the stage once these MMAs have read it
            }
            if (!failed) umma_commit(&tfull[acc]);
        }
        umma_commit(done);  // completes when every MMA issued above is complete
    } else if (warp >= 2) {
        const int q = warp & 3;  // the tensor-memory quarter this warp may read
        int lt = 0;
        for (int t = blockIdx.x; t < P.tiles; t += gridDim.x, ++lt) {
            const int acc = lt & 1;
            bool got = mbar_wait_bounded(&tfull[acc], (lt >> 1) & 1, P.timeout_ns);
            if (got && P.test_hook) got = mbar_wait_bounded(&tfull[acc], ((lt >> 1) & 1) ^ 1, P.timeout_ns);
            if (!__all_sync(0xffffffffu, got)) {
                failed = 1;
                break;
            }
            tc_fence_after();
            const int m = (t % P.mtiles) * HEAD_BM + q * 32 + lane;
            const int n0 = (t / P.mtiles) * bn;
            const int n1 = n0 + bn < P.V ? n0 + bn : P.V;  // the tile's columns: n0 .. n1
            float best = -__int_as_float(0x7f800000);
            int arg = -1;
            bool bad = false;
            for (int c = 0; c < HEAD_BN / 32; ++c) {  // 32-column loads within the 256 allocated
                const int col0 = n0 + c * 32;
                if (col0 >= n1) break;  // the same for the whole warp
                uint32_t r[32];
                tmem_ld32(tmem + (static_cast<uint32_t>(q * 32) << 16) +
                              static_cast<uint32_t>(acc * HEAD_BN + c * 32),
                          r);
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float z = __uint_as_float(r[j]);
                    if (col0 + j < n1) {
                        bad |= !(z == z) || z == __int_as_float(0x7f800000);
                        if (z > best) {  // ascending index: the first of equal maxima stays
                            best = z;
                            arg = col0 + j;
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);  // the accumulator may take the tile after next
            if (m < P.rows && (bad || arg >= 0)) atomicMax(P.best + m, bad ? HEAD_BAD : head_key(best, arg));
        }
    }
    __syncwarp();
    if (__any_sync(0xffffffffu, failed) && lane == 0) atomicOr(P.err, 1);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        // the MMAs of a CTA that stopped early may still be running: free tensor memory after them
        if (lane == 0 && !mbar_wait_bounded(done, 0, P.timeout_ns)) atomicOr(P.err, 1);
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, HEAD_TMEM_COLS);
    }
}

// ---- K_decide: one warp per sequence, one lane per position ---------------------

__global__ void __launch_bounds__(HEAD_DECIDE_NT) sv_head_decide_kernel(HeadDecideParams D) {
    pdl_wait_primary();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int timed_out = *D.err != 0;
    if (blockIdx.x == 0 && threadIdx.x == 0 && D.out_status) *D.out_status = timed_out ? -4 : 0;
    const int b = blockIdx.x * (HEAD_DECIDE_NT / 32) + warp;
    if (b >= D.B) return;
    const int k = D.k;
    const int32_t* d = D.draft_tokens + static_cast<size_t>(b) * k;
    int err = timed_out;
    int j = k;  // first mismatch
    for (int i0 = 0; i0 <= k; i0 += 32) {
        const int i = i0 + lane;
        int g = -1, mismatch = 0;
        if (i <= k) {
            const unsigned long long w = D.best[static_cast<size_t>(b) * (k + 1) + i];
            if (w == 0ull || w == HEAD_BAD || timed_out) {
                err = 1;
            } else {
                g = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(w));
            }
            if (i < k) {
                const int di = d[i];
                if (di < 0 || di >= D.V) err = 1;
                mismatch = di != g;
            }
            if (D.out_argmax) D.out_argmax[static_cast<size_t>(b) * (k + 1) + i] = timed_out ? -1 : g;
        }
        const unsigned mm = __ballot_sync(0xffffffffu, mismatch);
        if (j == k && mm) j = i0 + __ffs(mm) - 1;
    }
    err = __any_sync(0xffffffffu, err);
    // the token at j: the argmax of row j (the correction, or the bonus when j = k)
    const int y = err ? -1 : static_cast<int>(0xFFFFFFFFu -
                                              static_cast<uint32_t>(D.best[static_cast<size_t>(b) * (k + 1) + j]));
    int32_t* tok = D.out_tokens + static_cast<size_t>(b) * (k + 1);
    for (int i = lane; i <= k; i += 32) tok[i] = err ? -1 : (i < j ? d[i] : (i == j ? y : -1));
    if (lane == 0) D.out_n_accepted[b] = err ? -1 : j;
}

}  // namespace sv
