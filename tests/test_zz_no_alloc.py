"""spec_verify_static (the entry point that allocates nothing) against
spec_verify_ex on the same inputs.

Every output tensor is allocated before the checked region; the checked
region makes two spec_verify_static calls in a row and must leave the
device's free memory unchanged.  The file stands alone: it runs in a fresh
process as well as after the rest of the suite.
"""
import numpy as np
import pytest

import oracle
import workloads

pytestmark = pytest.mark.gpu

PROB_TOL = 1e-6  # same kernels, same inputs: only rounding order may differ


def _inputs(name, **over):
    import torch

    from paritylib import to_dev

    case = workloads.make_case(name, seed=11, **over)
    drafts = oracle.draft_tokens_for(case)
    greedy = case.mode == "greedy"
    dev = torch.device("cuda:0")
    t = {
        "target": to_dev(case.target, dev),
        "draft": None if greedy else to_dev(case.draft, dev),
        "drafts": torch.from_numpy(np.ascontiguousarray(drafts)).to(dev),
        "uniforms": None if greedy else to_dev(case.uniforms, dev),
        "temperature": None if greedy else to_dev(case.temperature, dev),
    }
    return case, greedy, t


def _outputs(B, k):
    import torch

    dev = torch.device("cuda:0")
    return {
        "tok": torch.full((B, k + 1), -7, dtype=torch.int32, device=dev),
        "n": torch.full((B,), -7, dtype=torch.int32, device=dev),
        "p": torch.full((B, k), float("nan"), dtype=torch.float32, device=dev),
        "q": torch.full((B, k), float("nan"), dtype=torch.float32, device=dev),
        "st": torch.full((1,), 12345, dtype=torch.int32, device=dev),
    }


def _mode(case, greedy):
    import draft_token_verification_verify_b200 as sv

    return (sv.SV_MODE_GREEDY if greedy else sv.SV_MODE_STOCHASTIC) | (
        sv.SV_DTYPE_BF16 if case.dtype == "bf16" else sv.SV_DTYPE_F32)


def _call(fn, case, greedy, t, o, **extra):
    return fn(t["target"], t["draft"], t["drafts"], t["uniforms"], case.B, case.k, case.V,
              t["temperature"], case.top_k, _mode(case, greedy), o["tok"], o["n"], o["p"], o["q"], o["st"],
              **extra)


CASES = [
    ("batched", dict(B=8)),                       # bf16, T=0.7, top-k 50
    ("batched", dict(B=4, top_k=0)),              # bf16, full softmax
    ("large", dict(B=6, dtype="f32")),            # fp32, mixed temperatures
    ("greedy", dict(B=16)),                       # greedy argmax
    ("single", dict(V=4099, top_k=7)),            # ragged vocabulary
]


@pytest.mark.parametrize("name,over", CASES, ids=[f"{n}-{'-'.join(f'{a}{b}' for a, b in o.items())}"
                                                  for n, o in CASES])
def test_static_matches_workspace_entry_point_twice(name, over):
    import torch

    import draft_token_verification_verify_b200 as sv

    case, greedy, t = _inputs(name, **over)
    ref = _outputs(case.B, case.k)
    assert _call(sv.spec_verify_ex, case, greedy, t, ref) == sv.SV_OK
    need = sv.spec_verify_workspace_size(case.B, case.k, case.V, case.top_k, _mode(case, greedy))
    assert 0 < need <= sv.SV_STATIC_WORKSPACE_BYTES
    outs = [_outputs(case.B, case.k) for _ in range(2)]
    torch.cuda.synchronize()
    # first call on the device performs the one-time set-up
    assert _call(sv.spec_verify_static, case, greedy, t, _outputs(case.B, case.k)) == sv.SV_OK
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for o in outs:  # two calls in a row
        assert _call(sv.spec_verify_static, case, greedy, t, o) == sv.SV_OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, "spec_verify_static changed the device's free memory"
    for o in outs:
        assert int(o["st"].item()) == sv.SV_OK
        assert torch.equal(o["tok"], ref["tok"])
        assert torch.equal(o["n"], ref["n"])
        assert (o["n"] >= 0).all()
        if not greedy:
            torch.testing.assert_close(o["p"], ref["p"], atol=PROB_TOL, rtol=0)
            torch.testing.assert_close(o["q"], ref["q"], atol=PROB_TOL, rtol=0)


def test_static_rejects_problems_beyond_its_buffer():
    import torch

    import draft_token_verification_verify_b200 as sv

    # top-k 256 keeps 512 entries (4 KB) per row: 1536 rows need ~6.4 MB of scratch
    B, k, V, K = 512, 1, 1024, 256
    dev = torch.device("cuda:0")
    target = torch.zeros((B, k + 1, V), dtype=torch.bfloat16, device=dev)
    draft = torch.zeros((B, k, V), dtype=torch.bfloat16, device=dev)
    drafts = torch.zeros((B, k), dtype=torch.int32, device=dev)
    uni = torch.full((B, k + 1), 0.5, dtype=torch.float32, device=dev)
    tok = torch.full((B, k + 1), -7, dtype=torch.int32, device=dev)
    n = torch.full((B,), -7, dtype=torch.int32, device=dev)
    mode = sv.SV_MODE_STOCHASTIC | sv.SV_DTYPE_BF16
    assert sv.spec_verify_workspace_size(B, k, V, K, mode) > sv.SV_STATIC_WORKSPACE_BYTES
    st = sv.spec_verify_static(target, draft, drafts, uni, B, k, V, None, K, mode, tok, n)
    assert st == sv.SV_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert (tok == -7).all() and (n == -7).all()  # nothing was launched
    # the same problem runs through the workspace entry point
    assert sv.spec_verify_ex(target, draft, drafts, uni, B, k, V, None, K, mode, tok, n) == sv.SV_OK
    torch.cuda.synchronize()
    assert (n >= 0).all()


@pytest.mark.parametrize("name,over", CASES[:3], ids=["batched-topk", "batched-softmax", "large-f32"])
def test_caller_workspace_takes_nothing_from_the_pool(name, over):
    """spec_verify_ex given a workspace allocates nothing: the pool counter and
    the device's free memory stay put; without one it takes one workspace
    from the pool per call."""
    import torch

    import draft_token_verification_verify_b200 as sv

    case, greedy, t = _inputs(name, **over)
    need = sv.spec_verify_workspace_size(case.B, case.k, case.V, case.top_k, _mode(case, greedy))
    ws = torch.empty(need, dtype=torch.uint8, device=torch.device("cuda:0"))
    outs = [_outputs(case.B, case.k) for _ in range(3)]
    assert _call(sv.spec_verify_ex, case, greedy, t, outs[0], workspace=ws, workspace_bytes=need) == sv.SV_OK
    torch.cuda.synchronize()
    a0 = sv.spec_verify_pool_allocations()
    free0, _ = torch.cuda.mem_get_info()
    for o in outs[1:]:
        assert _call(sv.spec_verify_ex, case, greedy, t, o, workspace=ws, workspace_bytes=need) == sv.SV_OK
    torch.cuda.synchronize()
    assert sv.spec_verify_pool_allocations() == a0
    assert torch.cuda.mem_get_info()[0] == free0
    for o in outs[1:]:
        assert torch.equal(o["tok"], outs[0]["tok"]) and torch.equal(o["n"], outs[0]["n"])
    assert _call(sv.spec_verify_ex, case, greedy, t, _outputs(case.B, case.k)) == sv.SV_OK  # pool
    torch.cuda.synchronize()
    assert sv.spec_verify_pool_allocations() == a0 + 1
