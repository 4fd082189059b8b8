"""CUDA path vs the fp64 oracle on identical seeded inputs (B200).

Covers the five workload value models (reduced and full sizes), the pages'
worked example, ragged and unaligned vocabularies, every top-k regime,
mixed temperatures, forced launch shapes and top-k paths, row errors, the
proposer sampler, and the emitted-token law of the GPU output itself.
"""
import math

import numpy as np
import pytest
from scipy import stats

import draft_token_verification_verify_b200 as sv
import oracle
import workloads
from paritylib import check_case, compare, compare_samples, run_gpu, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device(cuda_device):
    import __graft_entry__

    __graft_entry__.build()
    return cuda_device


def stack_cases(cases):
    """Concatenate single-sequence cases into one batch."""
    c0 = cases[0]
    cat = lambda name: None if getattr(c0, name) is None else np.concatenate([getattr(c, name) for c in cases])
    out = workloads.Case(name=c0.name, seed=c0.seed, B=sum(c.B for c in cases), k=c0.k, V=c0.V,
                         dtype=c0.dtype, mode=c0.mode, top_k=c0.top_k, target=cat("target"),
                         draft=cat("draft"), draft_proxy=cat("draft_proxy"), uniforms=cat("uniforms"),
                         draft_uniforms=cat("draft_uniforms"), temperature=cat("temperature"))
    return out


# --------------------------------------------------------------------------
# the pages' worked example on the GPU
# --------------------------------------------------------------------------

def test_worked_example_gpu():
    p = np.array([0.6, 0.3, 0.1])
    q = np.array([0.5, 0.4, 0.1])
    G = 1024
    target = np.repeat(np.log(np.stack([p, p])).astype(np.float32)[None], G, 0)
    draft = np.repeat(np.log(q).astype(np.float32)[None, None], G, 0)
    mid = ((np.arange(G) + 0.5) / G).astype(np.float32)
    u = np.stack([mid, mid[::-1].copy()], 1)
    d = np.ones((G, 1), np.int32)
    ref = oracle.verify(target, draft, d, u)
    gpu = run_gpu(target, draft, d, u, None, 0)
    rep = compare(ref, gpu, u)
    assert rep.exact + rep.flagged == G
    assert abs(np.mean(gpu.n_accepted == 1) - 0.75) < 1.0 / G
    assert np.all(gpu.tokens[gpu.n_accepted == 0, 0] == 0)    # residual lives on A only
    assert np.allclose(gpu.p, 0.3, atol=1e-6) and np.allclose(gpu.q, 0.4, atol=1e-6)


# --------------------------------------------------------------------------
# the five workload value models
# --------------------------------------------------------------------------

def test_tiny_thousand_seeds():
    case = stack_cases([workloads.make_case("tiny", seed=s) for s in range(1000)])
    rep = check_case(case)
    assert rep.exact >= 990


@pytest.mark.parametrize("seed", range(3))
def test_tiny_single_sequence_launch(seed):
    check_case(workloads.make_case("tiny", seed=seed))


@pytest.mark.parametrize("seed", range(4))
def test_single_sequence_full_size(seed):
    check_case(workloads.make_case("single", seed=seed))


def test_batched_full_size():
    rep = check_case(workloads.make_case("batched", seed=0))
    assert rep.sequences == 64


@pytest.mark.parametrize("path", [1, 2])
@pytest.mark.parametrize("seed", [1, 2])
def test_batched_topk_paths(seed, path):
    case = workloads.make_case("batched", seed=seed, B=8)
    check_case(case, opts=sv.make_options(topk_path=path))


def test_greedy_reduced_with_ties():
    case = workloads.make_case("greedy", seed=3, B=48)
    rows = workloads.bf16_bits_to_f32(case.target).reshape(-1, case.V)
    assert np.any((rows == workloads.TIE_VALUE).sum(1) == 2), "no tie rows drawn"
    check_case(case)


def test_greedy_full_size_sampled():
    """Full launch shape of the greedy workload (B=256, k=8, V=151936 bf16, ties
    in 1 % of target rows); the oracle checks a sample, bit-exact."""
    case = workloads.make_case("greedy", seed=6)
    drafts = oracle.draft_tokens_for(case)
    gpu = run_gpu(case.target, None, drafts, None, None, 0, greedy=True)
    pick = np.unique(np.linspace(0, case.B - 1, 32).astype(int))
    ref = oracle.verify(case.target[pick], None, drafts[pick], None, case.temperature[pick], 0, True)
    assert np.array_equal(gpu.n_accepted[pick], ref.n_accepted)
    assert np.array_equal(gpu.tokens[pick], ref.tokens)
    # properties at any size: accepted prefix equals the drafts, one target token, then -1
    for b in range(case.B):
        n = gpu.n_accepted[b]
        assert 0 <= n <= case.k
        assert np.array_equal(gpu.tokens[b, :n], drafts[b, :n])
        assert 0 <= gpu.tokens[b, n] < case.V and np.all(gpu.tokens[b, n + 1:] == -1)
        if n < case.k:
            assert gpu.tokens[b, n] != drafts[b, n]  # the first mismatch is replaced


def test_large_reduced_mixed_temperature():
    case = workloads.make_case("large", seed=4, B=24)
    assert len(set(case.temperature.tolist())) > 1
    check_case(case)


def test_large_full_size_sampled():
    """Full launch shape of the large workload; the oracle checks a sample."""
    case = workloads.make_case("large", seed=5)
    temp = np.repeat(case.temperature, case.k)
    drafts, _, _ = oracle.sample_rows(case.draft, case.draft_uniforms, temp, case.top_k)
    gpu = run_gpu(case.target, case.draft, drafts, case.uniforms, case.temperature, case.top_k)
    pick = np.unique(np.linspace(0, case.B - 1, 24).astype(int))
    ref = oracle.verify(case.target[pick], case.draft[pick], drafts[pick], case.uniforms[pick],
                        case.temperature[pick], case.top_k)
    sub = type(gpu)(gpu.tokens[pick], gpu.n_accepted[pick], gpu.p[pick], gpu.q[pick], gpu.status)
    rep = compare(ref, sub, case.uniforms[pick],
                  inputs=(case.target[pick], case.draft[pick], drafts[pick], case.temperature[pick], 0))
    assert rep.flagged_accept <= 1
    # properties at any size: accepted prefix equals the drafts, -1 after the draw
    for b in range(case.B):
        n = gpu.n_accepted[b]
        assert 0 <= n <= case.k
        assert np.array_equal(gpu.tokens[b, :n], drafts[b, :n])
        assert 0 <= gpu.tokens[b, n] < case.V and np.all(gpu.tokens[b, n + 1:] == -1)


# --------------------------------------------------------------------------
# shapes: ragged and unaligned vocabularies, small k / B, every top-k regime
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("V", [1, 2, 3, 7, 33, 1000, 1001, 1003, 4099, 65537])
def test_ragged_vocabularies(dtype, V):
    case = workloads.make_case("tiny", seed=V, B=5, k=3, V=V, dtype=dtype, temperature=(0.8,))
    check_case(case)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("K", [1, 2, 7, 50, 999, 1000, 1001, 1010])
def test_top_k_regimes(dtype, K):
    case = workloads.make_case("tiny", seed=K, B=6, k=2, V=1000, dtype=dtype, top_k=K, temperature=(1.3,))
    check_case(case)


@pytest.mark.parametrize("K", [1, 50, 129, 300])
def test_top_k_large_vocabulary(K):
    case = workloads.make_case("batched", seed=K, B=3, k=2, top_k=K)
    check_case(case)


def test_top_k_ties_at_threshold():
    case = workloads.make_case("batched", seed=9, B=4, k=2)
    # quantise to a coarse grid: dozens of entries share each value near tau
    t = workloads.bf16_bits_to_f32(case.target)
    d = workloads.bf16_bits_to_f32(case.draft)
    case.target = workloads.f64_to_bf16_bits(np.round(t.astype(np.float64)))
    case.draft = workloads.f64_to_bf16_bits(np.round(d.astype(np.float64)))
    for path in (0, 2):
        check_case(case, opts=sv.make_options(topk_path=path))


@pytest.mark.parametrize("k", [1, 2, 7])
def test_k_values(k):
    check_case(workloads.make_case("tiny", seed=100 + k, B=40, k=k, V=2048, dtype="bf16"))


@pytest.mark.parametrize("k", [15, 16])
def test_top_k_many_positions(k):
    """2k+1 = 31 rows take the single-warp path of the per-sequence kernel,
    33 rows the block path."""
    check_case(workloads.make_case("batched", seed=200 + k, B=3, k=k, V=30011, top_k=20))


@pytest.mark.parametrize("k", [12, 20])
def test_softmax_many_positions(k):
    check_case(workloads.make_case("single", seed=300 + k, B=2, k=k, V=20000, dtype="f32"))


def test_top_k_fp32_full_vocabulary():
    check_case(workloads.make_case("large", seed=31, B=4, top_k=50))


@pytest.mark.parametrize("K", [0, 7])
def test_many_sequences_tiny_vocabulary(K):
    check_case(workloads.make_case("tiny", seed=41 + K, B=3000, k=2, V=40, top_k=K))


@pytest.mark.parametrize("T", [0.5, 1.5])
def test_temperatures(T):
    check_case(workloads.make_case("single", seed=7, B=2, k=3, temperature=(T,)))


def test_draft_token_outside_draft_top_k():
    """q(d) = 0 (d outside the draft's kept set) accepts iff p(d) > 0."""
    case = workloads.make_case("tiny", seed=21, B=8, k=2, V=64, top_k=3)
    rng = np.random.default_rng(0)
    drafts = rng.integers(0, 64, size=(8, 2)).astype(np.int32)
    ref = oracle.verify(case.target, case.draft, drafts, case.uniforms, case.temperature, 3)
    assert np.any(ref.q == 0.0)
    gpu = run_gpu(case.target, case.draft, drafts, case.uniforms, case.temperature, 3)
    compare(ref, gpu, case.uniforms)


@pytest.mark.parametrize("chunks", [1, 2, 3, 5, 16])
@pytest.mark.parametrize("threads", [128, 256, 512])
@pytest.mark.parametrize("K", [0, 40])
def test_launch_shapes(chunks, threads, K):
    case = workloads.make_case("tiny", seed=chunks * threads + K, B=6, k=3, V=20000, dtype="bf16", top_k=K)
    check_case(case, opts=sv.make_options(chunks_per_row=chunks, threads=threads))


@pytest.mark.parametrize("chunks", [1, 4, 19])
@pytest.mark.parametrize("K", [0, 50])
def test_full_vocab_chunking(chunks, K):
    case = workloads.make_case("batched", seed=chunks, B=4, k=2, top_k=K)
    check_case(case, opts=sv.make_options(chunks_per_row=chunks))


# --------------------------------------------------------------------------
# greedy details
# --------------------------------------------------------------------------

def test_greedy_ties_signed_zero_and_bonus():
    V = 40
    target = np.full((4, 3, V), -5.0, np.float32)
    target[0, 0, [7, 3]] = 2.0                 # tie: lowest index 3
    target[0, 1, [5]] = -0.0
    target[0, 1, [2]] = 0.0                    # -0 == +0: lowest index 2
    target[0, 2, 30] = 1.0
    target[1, :, 0] = 9.0
    target[2, 1, :] = -np.inf                  # no finite logit: row error
    target[3, 0, 11] = np.nan                  # NaN: row error
    drafts = np.array([[3, 2], [0, 1], [0, 0], [0, 0]], np.int32)
    ref = oracle.verify(target, None, drafts, None, greedy=True)
    gpu = run_gpu(target, None, drafts, None, None, 0, greedy=True)
    compare(ref, gpu, None, greedy=True)
    assert gpu.tokens[0].tolist() == [3, 2, 30] and gpu.tokens[1].tolist() == [0, 0, -1]
    assert gpu.n_accepted[2] == -1 and gpu.n_accepted[3] == -1


@pytest.mark.parametrize("V", [5, 1000, 151936])
def test_greedy_bf16_ties_everywhere(V):
    rng = np.random.default_rng(V)
    t = np.round(rng.normal(0, 1, (6, 4, V)))            # many exact ties at the max
    target = workloads.f64_to_bf16_bits(t)
    drafts = rng.integers(0, V, size=(6, 3)).astype(np.int32)
    ref = oracle.verify(target, None, drafts, None, greedy=True)
    gpu = run_gpu(target, None, drafts, None, None, 0, greedy=True)
    compare(ref, gpu, None, greedy=True)


# --------------------------------------------------------------------------
# row errors
# --------------------------------------------------------------------------

@pytest.mark.parametrize("what", ["token_low", "token_high", "temp_zero", "temp_nan", "u_one",
                                  "u_neg", "nan_logit", "inf_logit", "all_neg_inf"])
def test_row_errors_gpu(what):
    V, k = 300, 2
    case = workloads.make_case("tiny", seed=3, B=3, k=k, V=V)
    target, draft = case.target.copy(), case.draft.copy()
    d = oracle.draft_tokens_for(case)
    u = case.uniforms.copy()
    T = case.temperature.copy()
    if what == "token_low": d[0, 1] = -1
    if what == "token_high": d[0, 0] = V
    if what == "temp_zero": T[0] = 0.0
    if what == "temp_nan": T[0] = np.nan
    if what == "u_one": u[0, k] = 1.0
    if what == "u_neg": u[0, 0] = -0.1
    if what == "nan_logit": draft[0, 1, 3] = np.nan
    if what == "inf_logit": target[0, 2, 0] = np.inf
    if what == "all_neg_inf": target[0, 1, :] = -np.inf
    ref = oracle.verify(target, draft, d, u, T)
    gpu = run_gpu(target, draft, d, u, T, 0)
    assert ref.n_accepted[0] == -1 and gpu.n_accepted[0] == -1
    compare(ref, gpu, u)


# --------------------------------------------------------------------------
# the proposer sampler (spec_sample)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,V,K,greedy", [("f32", 32, 0, False), ("bf16", 151936, 0, False),
                                              ("bf16", 151936, 50, False), ("f32", 128256, 0, False),
                                              ("f32", 128256, 50, False), ("bf16", 1003, 5, False),
                                              ("bf16", 151936, 0, True), ("f32", 77, 0, True)])
def test_sampler_parity(dtype, V, K, greedy):
    """spec_sample vs the oracle's sampler at T in {0.5, 1.0, 1.5}; rows whose
    uniform sits within 1e-5 of a CDF point are window-checked and counted."""
    import torch

    rows = 48
    case = workloads.make_case("tiny", seed=V + K, B=rows, k=1, V=V, dtype=dtype, top_k=K,
                               temperature=(0.5, 1.0, 1.5))
    assert set(np.unique(case.temperature)) == {0.5, 1.0, 1.5}
    logits = case.target[:, 0]
    u = case.draft_uniforms[:, 0].copy()
    ref, lo, hi = oracle.sample_rows(logits, None if greedy else u, case.temperature, K, greedy)
    out = sv.sample(to_dev(logits), None if greedy else to_dev(u), to_dev(case.temperature), K, greedy)
    torch.cuda.synchronize()
    rep = compare_samples(logits, u, case.temperature, K, out.cpu().numpy(), ref, lo, hi, greedy)
    print(rep)
    assert rep.exact + rep.flagged + rep.errors == rows


# --------------------------------------------------------------------------
# properties of the GPU output alone
# --------------------------------------------------------------------------

def test_gpu_emitted_law_chi_square():
    """Accepted drafts plus corrections reproduce the target law (GPU)."""
    import torch

    base = workloads.make_case("tiny", seed=11)
    k, V, B = base.k, base.V, 200_000
    p = [oracle.process_row(base.target[0, i]) for i in range(k + 1)]
    target = to_dev(np.ascontiguousarray(np.broadcast_to(base.target, (B, k + 1, V))))
    draft = to_dev(np.ascontiguousarray(np.broadcast_to(base.draft, (B, k, V))))
    du = to_dev(workloads.uniform_f32(77, workloads.TAG_DRAFT_UNIFORMS, B, k))
    uu = workloads.uniform_f32(77, workloads.TAG_UNIFORMS, B, k + 1)
    d = sv.sample(draft, du)                                   # drafts drawn on the GPU
    tok, n = sv.verify(target, draft, d, to_dev(uu))
    torch.cuda.synchronize()
    tok, n = tok.cpu().numpy(), n.cpu().numpy()
    for m in range(k + 1):
        sel = n >= m
        cnt = np.bincount(tok[sel, m], minlength=V)
        exp = sel.sum() * p[m]
        big = exp >= 5
        obs = np.append(cnt[big], cnt[~big].sum())
        ex = np.append(exp[big], exp[~big].sum())
        if ex[-1] == 0:
            obs, ex = obs[:-1], ex[:-1]
        assert stats.chisquare(obs, ex).pvalue > 1e-3, m


def test_repeatable():
    case = workloads.make_case("batched", seed=12, B=6)
    drafts = oracle.draft_tokens_for(case)
    a = run_gpu(case.target, case.draft, drafts, case.uniforms, case.temperature, case.top_k)
    b = run_gpu(case.target, case.draft, drafts, case.uniforms, case.temperature, case.top_k)
    assert np.array_equal(a.tokens, b.tokens) and np.array_equal(a.p, b.p) and np.array_equal(a.q, b.q)


def test_device_wait_timeout_reports_status():
    """A bulk-copy wait that can never complete (expected bytes inflated by the
    test hook) gives up after its bound and reports SV_ERR_DEVICE_TIMEOUT;
    the context stays usable."""
    case = workloads.make_case("tiny", seed=5, B=2, k=2, V=4096, dtype="bf16")
    drafts = oracle.draft_tokens_for(case)
    opts = sv.make_options(wait_timeout_ns=2_000_000, test_extra_tx=16)
    gpu = run_gpu(case.target, case.draft, drafts, case.uniforms, case.temperature, 0, opts=opts)
    assert gpu.status == sv.SV_ERR_DEVICE_TIMEOUT
    assert np.all(gpu.n_accepted == -1) and np.all(gpu.tokens == -1)
    check_case(case, drafts=drafts)      # the next call works normally
