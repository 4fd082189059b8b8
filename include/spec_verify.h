/*
 * spec_verify — batched speculative-sampling verification on NVIDIA B200
 * (sm_100a).  C ABI; every entry point is asynchronous on the caller's
 * CUDA stream.
 *
 * What is computed (speculative decoding entry "推测解码", glopedia.cn/401080,
 * section "提议与核验的基本步骤"):
 *   For each sequence b the caller supplies target logits at k+1 positions,
 *   draft logits at k positions, the k draft tokens d_0..d_{k-1} and k+1
 *   uniforms.  Both sides are processed identically (temperature, top-k,
 *   full-vocabulary softmax; paragraph 4).  Position i accepts d_i iff
 *   u_i * q_i(d_i) < p_i(d_i), i.e. with probability min(1, p/q)
 *   (paragraph 2); acceptance stops at the first rejection j, whose token is
 *   redrawn from the normalised residual max(0, p_j - q_j); if all k pass,
 *   a bonus token is drawn from p_k.  Both draws use u_k and the inverse
 *   CDF in index order (smallest v with C_v > u_k * W).  Greedy mode instead
 *   compares d_i with the lowest-index argmax of the target row
 *   (paragraph 4) and emits the target token at the first mismatch, or the
 *   argmax of row k after a full match.
 *
 * Conventions fixed by this library where the method leaves them open:
 *   - top-k keeps every logit >= tau, tau = the K-th largest raw logit
 *     counted with multiplicity, so ties at tau are all kept;
 *   - temperature divides the logits before the softmax; top-k is chosen on
 *     the raw logits; -inf logits have probability 0;
 *   - q(d) = 0 accepts iff p(d) > 0; a zero residual mass (only possible
 *     through rounding or when p(d) = q(d) = 0) redraws from p_j;
 *   - argmax ties go to the lowest index; -0.0 equals +0.0.
 *
 * Memory: every pointer is DEVICE memory owned by the caller and must stay
 * valid until the stream work completes.  Logits are contiguous row-major;
 * bf16 rows need 2-byte and fp32 rows 4-byte alignment (16-byte-aligned rows
 * take the fastest path).  Integer and float arrays need 4-byte alignment.
 * The kernels exchange per-row partial results through a device WORKSPACE
 * (spec_verify_workspace_size bytes, 16-byte aligned): the _ex entry points
 * take it from the caller; with workspace = NULL, and always for
 * spec_verify / spec_sample, the library takes it from its own
 * stream-ordered memory pool on the call's stream and releases it on the
 * same stream (memory the pool keeps for reuse).  Nothing else is allocated
 * and no state is kept between calls.
 *
 * Errors:
 *   - argument problems found on the host return SV_ERR_INVALID_ARG with no
 *     launch (B <= 0, k < 1, V < 1, top_k < 0, unknown mode or dtype bits,
 *     a required pointer NULL or misaligned, sizes that overflow, a
 *     workspace that is too small or misaligned);
 *   - SV_ERR_UNSUPPORTED: the current device is not of compute capability 10.0
 *     (the kernels are built for sm_100a),
 *     or sizes whose per-sequence shared-memory needs exceed the device
 *     (about k > 1000);
 *   - SV_ERR_CUDA: a CUDA call failed while launching;
 *   - per-sequence data errors do not fail the call: out_n_accepted[b] = -1
 *     and out_tokens[b, :] = -1.  They are a draft token outside [0, V), a
 *     temperature that is not finite and > 0, a uniform outside [0, 1), a
 *     NaN or +inf logit, or a row with no finite kept logit.  In greedy mode
 *     temperature, top-k and uniforms are ignored;
 *   - a device-side wait that runs out (bounded at about one second) marks
 *     its sequence as an error and writes SV_ERR_DEVICE_TIMEOUT to
 *     *out_status (spec_verify_ex).
 */
#ifndef SPEC_VERIFY_H
#define SPEC_VERIFY_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SV_API __attribute__((visibility("default")))
#else
#define SV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sv_status {
    SV_OK = 0,
    SV_ERR_INVALID_ARG = -1,
    SV_ERR_UNSUPPORTED = -2,
    SV_ERR_CUDA = -3,
    SV_ERR_DEVICE_TIMEOUT = -4
} sv_status_t;

/* mode = one SV_MODE_* (low byte) OR-ed with one SV_DTYPE_* */
enum {
    SV_MODE_STOCHASTIC = 0,
    SV_MODE_GREEDY = 1,
    SV_DTYPE_BF16 = 0 << 8,
    SV_DTYPE_F32 = 1 << 8
};

/* Tuning and instrumentation for the _ex entry points.  Zero every field for
 * the library's own choices. */
typedef struct sv_options {
    int chunks_per_row;        /* streaming tasks per logit row: 0 = auto, else >= 1 */
    int threads;               /* consumer threads per streaming CTA: 0 = auto, else 128, 256 or 512 */
    int topk_path;             /* 0 = auto, 1 = kept lists, 2 = radix select */
    void* event_start;         /* cudaEvent_t or NULL, recorded before the streaming kernel */
    void* event_stop;          /* cudaEvent_t or NULL, recorded right after it */
    uint64_t wait_timeout_ns;  /* bound of every device-side wait: 0 = 1e9 ns */
    uint32_t test_extra_tx;    /* test hook (0 in normal use): each ring stage expects this
                                  many bytes and no bulk copy is issued, so the bounded
                                  wait runs out with nothing in flight */
    const float* top_p;        /* [B] fp32 or NULL: nucleus threshold per sequence, applied
                                  to p and q alike after top-k and temperature: the most
                                  probable kept tokens whose probabilities first sum to
                                  >= top_p are kept, every token as probable as the last one
                                  included, then renormalised (1 keeps all).  Values outside
                                  (0, 1] make the sequence a row error.  With top-k the cut
                                  is taken over each row's kept set; without top-k over the
                                  whole row (one more kernel: an exact cut found by a mass
                                  histogram and a radix select over the row, two to five
                                  reads of it).  SV_MODE_GREEDY with top_p returns
                                  SV_ERR_UNSUPPORTED.  In spec_sample_ex, top_p[s] applies
                                  to the rows of sequence s (see rows_per_sequence). */
    /* Further processors (section "提议与核验的基本步骤", paragraph 4: applied
     * to the target and draft distributions alike).  They act on the raw
     * logits, before top-k, temperature, softmax and nucleus, the same way for
     * every target and draft row of a sequence.  Stochastic mode only: with
     * SV_MODE_GREEDY a non-NULL vocab_mask or rep_ids returns
     * SV_ERR_UNSUPPORTED.  S is the number of sequences (B for verification,
     * ceil(rows / rows_per_sequence) for spec_sample_ex). */
    const uint32_t* vocab_mask;  /* [S][ceil(V/32)] uint32 or NULL: token v of sequence s is
                                    allowed iff bit v % 32 of word v / 32 of row s is set; a
                                    disallowed token gets the logit -inf (probability 0); a
                                    sequence with no allowed finite logit is a row error */
    const int32_t* rep_ids;      /* [S][n_rep] int32 or NULL: token ids the repetition penalty
                                    applies to; ids outside [0, V) are ignored and a repeated
                                    id is penalised once */
    int n_rep;                   /* ids per sequence in rep_ids, >= 0 */
    const float* rep_penalty;    /* [S] fp32 or NULL (all 1): theta > 0; a listed token's logit
                                    z becomes z / theta if z > 0, else z * theta, rounded to
                                    fp32; theta not > 0 makes the sequence a row error */
    int rows_per_sequence;       /* spec_sample_ex only: row r takes the processors and top_p
                                    of sequence r / rows_per_sequence (0 = 1) */
} sv_options_t;

/*
 * spec_verify — verify one speculative round for B sequences.
 *   target_logits  [B][k+1][V]  bf16 or fp32 (per `mode`)
 *   draft_logits   [B][k][V]    same dtype; may be NULL in greedy mode
 *   draft_tokens   [B][k]       int32
 *   uniforms       [B][k+1]     fp32: u_0..u_{k-1} decide acceptance, u_k
 *                               drives the correction or bonus draw; may be
 *                               NULL in greedy mode
 *   B, k, V        sequences, draft length (>= 1), vocabulary size
 *   temperature    [B] fp32 per-sequence temperature, or NULL for 1.0
 *   top_k          0 or >= V disables top-k; else applied to p and q alike
 *   mode           SV_MODE_* | SV_DTYPE_*
 *   out_tokens     [B][k+1] int32: d_0..d_{j-1}, the corrected/bonus token at
 *                  j, then -1 (also used as scratch during the call)
 *   out_n_accepted [B] int32: j, the number of accepted draft tokens
 *   stream         cudaStream_t (NULL = legacy default stream)
 */
SV_API sv_status_t spec_verify(const void* target_logits, const void* draft_logits,
                        const int32_t* draft_tokens, const float* uniforms, int B, int k,
                        int V, const float* temperature, int top_k, int mode,
                        int32_t* out_tokens, int32_t* out_n_accepted, void* stream);

/*
 * spec_verify_workspace_size — device workspace bytes spec_verify_ex needs
 * for these arguments on the current device (0 on invalid arguments).
 */
SV_API size_t spec_verify_workspace_size(int B, int k, int V, int top_k, int mode,
                                         const sv_options_t* opts);

/*
 * spec_verify_ex — spec_verify plus optional outputs, workspace and options.
 *   out_p, out_q     [B][k] fp32 or NULL: p_i(d_i) and q_i(d_i) at EVERY
 *                    position (also past the first rejection); stochastic mode
 *   out_status       1 int32 or NULL: SV_OK, or SV_ERR_DEVICE_TIMEOUT if a
 *                    device wait ran out (written by the call's kernels)
 *   workspace        NULL (library pool) or >= spec_verify_workspace_size
 *                    bytes, 16-byte aligned; calls that share a workspace must
 *                    be ordered on one stream
 *   workspace_bytes  its size
 *   opts             NULL or options (see sv_options_t)
 */
SV_API sv_status_t spec_verify_ex(const void* target_logits, const void* draft_logits,
                                  const int32_t* draft_tokens, const float* uniforms, int B, int k,
                                  int V, const float* temperature, int top_k, int mode,
                                  int32_t* out_tokens, int32_t* out_n_accepted, float* out_p,
                                  float* out_q, int32_t* out_status, void* workspace,
                                  size_t workspace_bytes, const sv_options_t* opts, void* stream);

/* Bytes of the library's static scratch buffer used by spec_verify_static. */
#define SV_STATIC_WORKSPACE_BYTES (4u << 20)

/*
 * spec_verify_static — spec_verify_ex that allocates nothing.
 *
 * The method's description has no counterpart to this call: it is a
 * library convenience for callers that must not allocate device memory
 * while they run.  Examples are a serving loop that has given every free byte
 * to its own cache allocator, and code that holds a lock that a
 * stream-ordered pool may re-enter.  spec_verify_ex with a NULL workspace
 * draws scratch from a library pool, and with a caller workspace it needs
 * that buffer sized and kept alive.  This call instead uses a fixed
 * SV_STATIC_WORKSPACE_BYTES buffer compiled into the library for each device
 * (a __device__ array), so it performs no cudaMalloc, cudaFree or pool
 * allocation of any kind.
 *
 * Arguments and outputs are those of spec_verify_ex without the workspace.
 *
 * Set-up: the first call on a device, with that device current, looks up the
 * buffer's device address and caches it; a lookup that fails is not cached
 * and the next call tries again.  Make that first call before any stream
 * capture on that device.
 *
 * Limit: a problem whose scratch need (spec_verify_workspace_size with the
 * same arguments and options) exceeds SV_STATIC_WORKSPACE_BYTES is rejected
 * with SV_ERR_UNSUPPORTED before anything is launched.
 *
 * Contents: nothing in the buffer has to start at zero; each call writes
 * every scratch record it reads, and writes *out_status itself.
 *
 * Concurrency: there is ONE buffer per device.  Calls on one stream run one
 * after the other and are safe.  Calls whose execution can overlap, on
 * different streams or from different host threads without ordering
 * between them, use the same bytes at the same time and give wrong results.
 */
SV_API sv_status_t spec_verify_static(const void* target_logits, const void* draft_logits,
                                      const int32_t* draft_tokens, const float* uniforms, int B,
                                      int k, int V, const float* temperature, int top_k, int mode,
                                      int32_t* out_tokens, int32_t* out_n_accepted, float* out_p,
                                      float* out_q, int32_t* out_status, const sv_options_t* opts,
                                      void* stream);

/*
 * spec_sample — the proposer's sampling step (section "提议与核验的基本步骤",
 * paragraph 1: the proposer draws each candidate from its own
 * distribution): one token per logit row, drawn with the same processing
 * and inverse-CDF rule as the verification's bonus draw (stochastic), or
 * the lowest-index argmax (greedy).
 *   logits       [rows][V] bf16 or fp32
 *   uniforms     [rows] fp32 in [0, 1); NULL in greedy mode
 *   temperature  [rows] fp32 or NULL for 1.0
 *   top_k, mode  as for spec_verify
 *   out_tokens   [rows] int32; -1 for a row with a data error
 */
SV_API sv_status_t spec_sample(const void* logits, const float* uniforms, int rows, int V,
                        const float* temperature, int top_k, int mode, int32_t* out_tokens,
                        void* stream);

/* Workspace bytes of spec_sample_ex on the current device (0 on invalid arguments). */
SV_API size_t spec_sample_workspace_size(int rows, int V, int top_k, int mode,
                                         const sv_options_t* opts);

/* spec_sample with a workspace (NULL: library pool) and options (may be NULL). */
SV_API sv_status_t spec_sample_ex(const void* logits, const float* uniforms, int rows, int V,
                                  const float* temperature, int top_k, int mode,
                                  int32_t* out_tokens, void* workspace, size_t workspace_bytes,
                                  const sv_options_t* opts, void* stream);

/*
 * spec_verify_tree — verify one round of tree-shaped candidates for B
 * sequences (candidate trees: section "提议方式与实现形态", paragraph 3; the
 * pages give no acceptance rule for them, the one taken reduces to the chain
 * rule of "提议与核验的基本步骤", paragraph 2, on a chain).
 *   Node 0 of each sequence is the verified context; node n in [1, N] carries
 *   tokens[b][n-1] and has the parent parents[b][n-1] in [0, n).  Row n of
 *   target_logits / draft_logits [B][N+1][V] (bf16 or fp32, per `mode`) is
 *   the target / draft distribution of the token after node n's prefix (the
 *   children of node n were drawn from draft row n).
 *   Stochastic: the walk starts at node 0 with R = p (the node's processed
 *   target row, temperature and top-k as in spec_verify) and tries the node's
 *   children in index order; child c is accepted iff
 *   uniforms[b][c-1] * q(t_c) < R(t_c) (q the node's processed draft row),
 *   and the walk continues from it; a rejection replaces R by the normalised
 *   residual max(0, R - q) (kept as it is when that has no mass); when no
 *   child is accepted the final token is drawn from R by the inverse CDF
 *   with uniforms[b][N].  Greedy: the first child whose token is the node's
 *   lowest-index argmax is accepted, else that argmax is emitted (draft
 *   logits, uniforms and temperature unused, may be NULL).
 *   Outputs: out_tokens [B][N+1] (the accepted tokens, the final token, then
 *   -1), out_n_accepted [B] (-1: the sequence is an error); optional (NULL to
 *   skip): out_nodes [B][N+1] (the accepted nodes, then -1), out_p / out_q
 *   [B][N] (R(t_c) and q(t_c) of every tested child, NaN otherwise).
 *   Only the rows of visited nodes are read.  Row errors: a NaN or +inf
 *   logit or no finite kept logit in a row read, a token outside [0, V), a
 *   parent outside [0, n), and (stochastic) a uniform outside [0, 1) or a
 *   temperature not finite and > 0.  N <= 256, V <= 262,144
 *   (SV_ERR_UNSUPPORTED above).  Allocates nothing; all work is enqueued on
 *   `stream`.  Argument errors return SV_ERR_INVALID_ARG before any launch.
 */
SV_API sv_status_t spec_verify_tree(const void* target_logits, const void* draft_logits,
                                    const int32_t* tokens, const int32_t* parents,
                                    const float* uniforms, int B, int N, int V,
                                    const float* temperature, int top_k, int mode,
                                    int32_t* out_tokens, int32_t* out_n_accepted,
                                    int32_t* out_nodes, float* out_p, float* out_q, void* stream);

/*
 * spec_verify_tree with a caller workspace (device memory, 16-byte aligned,
 * at least spec_verify_tree_workspace_size bytes; NULL: as spec_verify_tree).
 * With top-k (0 < top_k < V, up to 256) or greedy, and a workspace, the
 * streaming pass first reads every target and draft row of the trees once and
 * the walk then works on the kept lists (or the per-row argmax) alone; rows
 * whose kept list overflowed fall back to the walk over the rows.  Same
 * results.  The workspace is not read before it is written.
 */
SV_API sv_status_t spec_verify_tree_ex(const void* target_logits, const void* draft_logits,
                                       const int32_t* tokens, const int32_t* parents,
                                       const float* uniforms, int B, int N, int V,
                                       const float* temperature, int top_k, int mode,
                                       int32_t* out_tokens, int32_t* out_n_accepted,
                                       int32_t* out_nodes, float* out_p, float* out_q,
                                       void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes for spec_verify_tree_ex's list walk; 0 when the call has no
 * list walk (no top-k) or on invalid arguments / no usable device. */
SV_API size_t spec_verify_tree_workspace_size(int B, int N, int V, int top_k, int mode);

/*
 * spec_verify_head_greedy — greedy verification fused into the target's
 * output projection.  The target scores the k+1 positions of a sequence in
 * one forward pass (section "提议与核验的基本步骤", paragraph 1); here its
 * last step, the logits z_v = h . W[v], is computed on the tensor cores and
 * reduced on chip to each position's lowest-index argmax, so the logits are
 * never written to memory; the greedy rule of paragraph 4 then runs as in
 * spec_verify with SV_MODE_GREEDY.
 *   hidden        [B][k+1][H] bf16, 16-byte aligned: the target's final
 *                 hidden state at each position
 *   weight        [V][H] bf16, 16-byte aligned: the output projection
 *   draft_tokens  [B][k] int32
 *   H             > 0 and a multiple of 8 (16-byte rows)
 *   out_tokens, out_n_accepted   as spec_verify (greedy)
 *   out_argmax    [B][k+1] int32 or NULL: each position's argmax, -1 for a
 *                 row with a NaN or +inf logit or none finite
 *   workspace     spec_verify_head_workspace_size(B, k, V, H) bytes of device
 *                 memory, 16-byte aligned, or NULL (taken from the library's
 *                 pool on `stream` and released there); written before read
 *   opts          NULL or options: wait_timeout_ns, event_start / event_stop
 *                 (around the projection kernel) and test_extra_tx (non-zero:
 *                 the projection kernel also waits for an accumulator phase
 *                 that never completes, so its bounded wait runs out with no
 *                 copy or MMA in flight); top_p, vocab_mask and rep_ids give
 *                 SV_ERR_UNSUPPORTED
 *   out_status    1 int32 or NULL: SV_OK, or SV_ERR_DEVICE_TIMEOUT when a
 *                 device-side wait ran out (then every sequence is an error)
 * The products of bf16 values are exact and are summed in fp32 on the tensor
 * cores, so a logit differs from its exact value by rounding of that sum
 * only.  Row errors as spec_verify: a draft token outside [0, V), a NaN or
 * +inf logit, or a row with no finite logit, anywhere in the sequence.
 * V up to 16,776,960 (SV_ERR_UNSUPPORTED above).
 */
SV_API sv_status_t spec_verify_head_greedy(const void* hidden, const void* weight,
                                           const int32_t* draft_tokens, int B, int k, int V, int H,
                                           int32_t* out_tokens, int32_t* out_n_accepted,
                                           int32_t* out_argmax, void* workspace,
                                           size_t workspace_bytes, const sv_options_t* opts,
                                           int32_t* out_status, void* stream);

/* Workspace bytes for spec_verify_head_greedy; 0 on invalid sizes. */
SV_API size_t spec_verify_head_workspace_size(int B, int k, int V, int H);

/* Static description of a status code. */
SV_API const char* spec_verify_status_string(sv_status_t status);

/* Library version as MAJOR * 10000 + MINOR * 100 + PATCH. */
SV_API int spec_verify_version(void);

/* Workspaces this process has taken from the library's pool: one per call of
 * spec_verify, spec_sample, or an _ex entry point given a NULL workspace.
 * Calls given a workspace (and spec_verify_static, the size queries and
 * calls refused before launch) allocate nothing and leave it unchanged. */
SV_API unsigned long long spec_verify_pool_allocations(void);

#ifdef __cplusplus
}
#endif

#endif /* SPEC_VERIFY_H */
