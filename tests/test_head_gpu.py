"""Greedy verification fused into the output projection
(``spec_verify_head_greedy``) against the oracle's fp64 logits
(``oracle.verify_head_greedy``).

Rule.  The GPU forms each logit from exact bf16 products summed in fp32 on the
tensor cores: K/16 accumulations of 16-product blocks, so its logit differs
from the exact one by at most tol_v = (H/16 + 8) * 2^-23 * A_v, A_v the sum of
the products' magnitudes (the oracle's ``abs``; 2^-23 allows truncating as
well as rounding adders).  For every row the oracle checks:
* the GPU's argmax g is a valid argmax: z(g) >= z(g*) - tol_g - tol_g*, with
  g* the oracle's lowest-index argmax;
* when no other entry is that close to z(g*) (the row is unambiguous), g = g*
  exactly;
and for every sequence whose rows are all unambiguous, tokens and accepted
count equal the oracle's bit for bit.  Sequences with an ambiguous row are
counted (and printed); for them, and for every sequence at any size, the
tokens must be the greedy chain of the GPU's own per-row argmax.  Error
sequences match exactly.
"""
import numpy as np
import pytest

import oracle
import workloads
from paritylib import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device(cuda_device):
    import __graft_entry__

    __graft_entry__.build()
    return cuda_device


def _drafts(rng, ref_arg, B, k, V, seqs, p_match=0.8):
    """Draft tokens: the oracle's argmax with probability p_match, else a
    random token, for the checked sequences; random for the rest."""
    d = rng.integers(0, V, (B, k)).astype(np.int32)
    for si, b in enumerate(seqs):
        hit = rng.random(k) < p_match
        d[b, hit] = ref_arg[si, :k][hit]
    return d


def _run(case, drafts, opts=None, workspace=None):
    import torch

    import draft_token_verification_verify_b200 as sv

    dev = torch.device("cuda:0")
    arg = torch.full((case.B, case.k + 1), -7, dtype=torch.int32, device=dev)
    status = torch.full((1,), 12345, dtype=torch.int32, device=dev)
    tok, n = sv.verify_head_greedy(to_dev(case.hidden), to_dev(case.weight), torch.from_numpy(drafts).to(dev),
                                   out_argmax=arg, out_status=status, opts=opts, workspace=workspace)
    torch.cuda.synchronize()
    return tok.cpu().numpy(), n.cpu().numpy(), arg.cpu().numpy(), int(status.item())


def _chain(arg_row, d):
    """The greedy chain of per-row argmaxes (for the validity check)."""
    k = len(d)
    if np.any(arg_row < 0):
        return None
    for i in range(k):
        if d[i] != arg_row[i]:
            return i, list(d[:i]) + [int(arg_row[i])] + [-1] * (k - i)
    return k, list(d) + [int(arg_row[k])]


def _check(case, drafts, ref, tok, n, arg, max_amb_frac=0.05):
    H = case.H
    gam = (H / 16 + 8) * 2.0 ** -23
    amb_seqs = amb_rows = exact = 0
    for si, b in enumerate(ref.seqs):
        r = ref.result
        if r.n_accepted[si] < 0:
            assert n[b] == -1 and np.all(tok[b] == -1), (b, n[b], tok[b])
            continue
        seq_amb = False
        for i in range(case.k + 1):
            z, tol = ref.z[si, i], gam * ref.abs[si, i]
            g_ref = int(np.argmax(z))
            g = int(arg[b, i])
            assert 0 <= g < case.V, (b, i, g)
            assert z[g] >= z[g_ref] - tol[g] - tol[g_ref], (b, i, g, g_ref, z[g], z[g_ref])
            near = np.flatnonzero(z >= z[g_ref] - tol - tol[g_ref])
            if near.size > 1:
                amb_rows += 1
                seq_amb = True
            else:
                assert g == g_ref, (b, i, g, g_ref)
        if seq_amb:
            amb_seqs += 1
            continue
        assert n[b] == r.n_accepted[si], (b, n[b], r.n_accepted[si])
        assert np.array_equal(tok[b], r.tokens[si]), (b, tok[b], r.tokens[si])
        exact += 1
    # every sequence: the tokens are the greedy chain of the GPU's own argmaxes
    for b in range(case.B):
        ch = _chain(arg[b], drafts[b])
        if ch is None or np.any((drafts[b] < 0) | (drafts[b] >= case.V)):
            assert n[b] == -1 and np.all(tok[b] == -1), b
        else:
            assert n[b] == ch[0] and list(tok[b]) == ch[1], (b, n[b], tok[b], ch)
    print(f"checked {len(ref.seqs)} of {case.B} sequences: exact {exact}, ambiguous {amb_seqs} "
          f"({amb_rows} rows)")
    assert amb_seqs <= max(1, int(max_amb_frac * len(ref.seqs))), amb_seqs
    return exact


def _case_and_ref(seed, B, k, V, H, seqs=None, threads=4):
    case = workloads.make_head_case(seed, B, k, V, H)
    seqs = np.arange(B) if seqs is None else np.asarray(seqs)
    rng = np.random.default_rng(seed)
    # the oracle's logits first, for the drafts; then the verification on the final drafts
    pre = oracle.verify_head_greedy(case.hidden, case.weight, np.zeros((B, k), np.int32), seqs=seqs,
                                    threads=threads)
    ref_arg = pre.z.argmax(axis=-1)
    drafts = _drafts(rng, ref_arg, B, k, V, seqs)
    ref = oracle.verify_head_greedy(case.hidden, case.weight, drafts, seqs=seqs, threads=threads)
    return case, drafts, ref


@pytest.mark.parametrize("B,k,V,H", [
    (3, 2, 1000, 200),    # ragged vocabulary tile, ragged K block, one partial row tile
    (32, 3, 512, 128),    # whole tiles: 128 rows, 2 x 256 entries, 2 K blocks
    (50, 4, 4099, 512),   # 250 rows: a full and a ragged row tile
    (4, 40, 300, 8),      # long drafts, H below one K block
    (5, 2, 1, 64),        # a vocabulary of one
    (100, 7, 5003, 320),  # 800 rows: seven row tiles, the last one of 32 rows
])
def test_parity_small(B, k, V, H):
    case, drafts, ref = _case_and_ref(10 + B + k, B, k, V, H)
    tok, n, arg, status = _run(case, drafts)
    assert status == 0
    _check(case, drafts, ref, tok, n, arg)


def test_parity_wide_hidden():
    case, drafts, ref = _case_and_ref(21, 16, 4, 30011, 2048)
    tok, n, arg, _ = _run(case, drafts)
    assert _check(case, drafts, ref, tok, n, arg) >= 12


def test_full_size_sampled_sequences():
    """B = 64, k = 4, V = 151,936, H = 4,096 (the batched shape with a
    4,096-wide hidden state): the whole batch on the GPU, the oracle on 4
    sampled sequences, the chain property on all 64."""
    case, drafts, ref = _case_and_ref(22, 64, 4, 151936, 4096, seqs=[0, 21, 42, 63], threads=4)
    tok, n, arg, status = _run(case, drafts)
    assert status == 0
    _check(case, drafts, ref, tok, n, arg, max_amb_frac=0.25)


def test_exact_ties_go_to_the_lowest_index():
    """Weight rows 3 and 700 are equal and dominate every row: their logits are
    the same fp32 sums, and the lower index must win."""
    B, k, V, H = 6, 3, 1024, 256
    case = workloads.make_head_case(23, B, k, V, H)
    c = np.where(np.arange(H) % 3 == 0, 1.0, -1.0)
    hid = workloads.bf16_bits_to_f32(case.hidden).astype(np.float64) + 2.0 * c
    case.hidden[:] = workloads.f64_to_bf16_bits(hid)
    case.weight[3] = case.weight[700] = workloads.f64_to_bf16_bits(0.05 * c)
    drafts = np.full((B, k), 3, np.int32)
    drafts[1, 2] = 700
    ref = oracle.verify_head_greedy(case.hidden, case.weight, drafts)
    assert np.all(ref.z.argmax(axis=-1) == 3)
    tok, n, arg, _ = _run(case, drafts)
    assert np.all(arg == 3)
    assert np.array_equal(tok, ref.result.tokens) and np.array_equal(n, ref.result.n_accepted)


def test_row_errors():
    B, k, V, H = 5, 3, 2000, 128
    case = workloads.make_head_case(24, B, k, V, H)
    case.hidden[1, 2, 5] = 0x7FC0  # NaN: every logit of that row is NaN
    drafts = np.random.default_rng(24).integers(0, V, (B, k)).astype(np.int32)
    drafts[3, 1] = V                 # token outside [0, V)
    ref = oracle.verify_head_greedy(case.hidden, case.weight, drafts)
    tok, n, arg, _ = _run(case, drafts)
    assert list(ref.result.n_accepted[[1, 3]]) == [-1, -1]
    assert np.array_equal(n, ref.result.n_accepted) and np.array_equal(tok, ref.result.tokens)
    assert arg[1, 2] == -1 and np.all(arg[1, [0, 1, 3]] >= 0)


def test_device_wait_timeout_reports_status():
    """The test hook makes the projection kernel wait for an accumulator phase
    that never completes: the bounded wait runs out with nothing in flight,
    the call reports SV_ERR_DEVICE_TIMEOUT and every sequence as an error,
    and the next call works."""
    import draft_token_verification_verify_b200 as sv

    case, drafts, ref = _case_and_ref(25, 4, 2, 700, 64)
    opts = sv.make_options(wait_timeout_ns=2_000_000, test_extra_tx=1)
    tok, n, arg, status = _run(case, drafts, opts=opts)
    assert status == sv.SV_ERR_DEVICE_TIMEOUT
    assert np.all(n == -1) and np.all(tok == -1) and np.all(arg == -1)
    tok, n, arg, status = _run(case, drafts)
    assert status == 0
    _check(case, drafts, ref, tok, n, arg)


def test_caller_workspace_is_written_before_read():
    import torch

    import draft_token_verification_verify_b200 as sv

    case, drafts, ref = _case_and_ref(26, 9, 4, 3001, 256)
    need = sv.spec_verify_head_workspace_size(case.B, case.k, case.V, case.H)
    ws = torch.full((need,), 0xA5, dtype=torch.uint8, device="cuda:0")  # stale bytes
    a = _run(case, drafts, workspace=ws)
    b = _run(case, drafts, workspace=ws)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    _check(case, drafts, ref, *a[:3])


def test_single_sequence_full_vocabulary():
    """B = 1, k = 1 at V = 151,936, H = 4,096: one row tile, many narrow vocabulary tiles."""
    case, drafts, ref = _case_and_ref(27, 1, 1, 151936, 4096)
    tok, n, arg, status = _run(case, drafts)
    assert status == 0
    _check(case, drafts, ref, tok, n, arg)


def test_graph_capture_and_replay():
    """The call (a memset and two launches on the caller's stream) captures
    into a CUDA graph; replays give the eager result."""
    import torch

    import draft_token_verification_verify_b200 as sv

    case, drafts, ref = _case_and_ref(28, 12, 4, 20011, 512)
    dev = torch.device("cuda:0")
    h, w, d = to_dev(case.hidden), to_dev(case.weight), torch.from_numpy(drafts).to(dev)
    ws = torch.empty((sv.spec_verify_head_workspace_size(12, 4, 20011, 512),), dtype=torch.uint8, device=dev)
    tok = torch.empty((12, 5), dtype=torch.int32, device=dev)
    n = torch.empty((12,), dtype=torch.int32, device=dev)
    arg = torch.empty((12, 5), dtype=torch.int32, device=dev)
    s = torch.cuda.Stream()

    def call():
        st = sv.spec_verify_head_greedy(h, w, d, 12, 4, 20011, 512, tok, n, arg, ws, ws.numel(), None, None, s)
        assert st == sv.SV_OK

    with torch.cuda.stream(s):
        call()  # first call outside capture (one-time attribute and driver lookups)
    torch.cuda.synchronize()
    eager = [t.cpu().numpy().copy() for t in (tok, n, arg)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        call()
    for t in (tok, n, arg):
        t.fill_(-9)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    for t, e in zip((tok, n, arg), eager):
        assert np.array_equal(t.cpu().numpy(), e)
    _check(case, drafts, ref, *eager)
