"""C-ABI checks that need no GPU: the library loads, exports every function
``include/spec_verify.h`` declares, rejects bad arguments before touching
CUDA, and the Python mirror of ``sv_options_t`` matches the C layout."""
import ctypes
import os
import re
import subprocess

import pytest

import draft_token_verification_verify_b200 as sv
from draft_token_verification_verify_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "spec_verify.h")


@pytest.fixture(scope="module")
def L():
    _build.build()
    return sv.lib()


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"SV_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)))


def test_header_declares_entry_points():
    assert declared_functions() == sorted([
        "spec_sample", "spec_sample_ex", "spec_sample_workspace_size", "spec_verify", "spec_verify_ex",
        "spec_verify_pool_allocations", "spec_verify_static", "spec_verify_status_string", "spec_verify_tree",
        "spec_verify_tree_ex", "spec_verify_tree_workspace_size", "spec_verify_version", "spec_verify_workspace_size",
        "spec_verify_head_greedy", "spec_verify_head_workspace_size"])



def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", _build.LIB], check=True,
                         capture_output=True, text=True).stdout
    exported = set(re.findall(r"\sT\s+(\w+)$", out, flags=re.M))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(L, name)
    # nothing else leaks out of the C ABI
    assert exported == set(declared_functions())


def _no_gpu():
    """Calls below pass placeholder device pointers that get past the argument
    checks: they may only run where no GPU can launch anything."""
    import torch

    if torch.cuda.is_available():
        pytest.skip("placeholder device pointers: runs only without a GPU")


def test_no_pool_allocation_without_a_launch(L):
    """Size queries, refused calls and calls given a workspace never take a
    workspace from the library's pool (here, without a GPU, none launches)."""
    _no_gpu()
    a0 = sv.spec_verify_pool_allocations()
    sv.spec_verify_workspace_size(64, 4, 151936, 50, 0)
    sv.spec_sample_workspace_size(8, 1000, 0, 0)
    st = sv.spec_verify_ex(P, P, P, P, 2, 3, 100, None, 0, 0, P, P, None, None, None, P, 1 << 20, None, 0)
    assert st != sv.SV_OK
    st = sv.spec_verify_ex(P, P, P, P, 0, 3, 100, None, 0, 0, P, P, stream=0)  # invalid: B = 0
    assert st == sv.SV_ERR_INVALID_ARG
    assert sv.spec_verify(P, P, P, P, 2, 0, 100, None, 0, 0, P, P, stream=0) == sv.SV_ERR_INVALID_ARG  # k = 0
    assert sv.spec_verify_pool_allocations() == a0


def test_version_and_status_strings(L):
    assert sv.spec_verify_version() == 20000
    assert sv.spec_verify_status_string(sv.SV_OK) == "ok"
    assert sv.spec_verify_status_string(sv.SV_ERR_DEVICE_TIMEOUT) == "device-side wait timed out"
    assert sv.spec_verify_status_string(123) == "unknown status"


def test_options_struct_layout_matches_c(tmp_path):
    prog = tmp_path / "layout.c"
    prog.write_text(r"""
#include <stddef.h>
#include <stdio.h>
#include "spec_verify.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu\n", sizeof(sv_options_t),
         offsetof(sv_options_t, chunks_per_row), offsetof(sv_options_t, threads),
         offsetof(sv_options_t, topk_path), offsetof(sv_options_t, event_start),
         offsetof(sv_options_t, event_stop), offsetof(sv_options_t, wait_timeout_ns),
         offsetof(sv_options_t, test_extra_tx), offsetof(sv_options_t, top_p),
         offsetof(sv_options_t, vocab_mask), offsetof(sv_options_t, rep_ids),
         offsetof(sv_options_t, n_rep), offsetof(sv_options_t, rep_penalty),
         offsetof(sv_options_t, rows_per_sequence));
  return 0;
}
""")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(prog)],
                   check=True)
    c = [int(x) for x in subprocess.run([str(exe)], check=True, capture_output=True,
                                         text=True).stdout.split()]
    O = sv.SvOptions
    py = [ctypes.sizeof(O)] + [getattr(O, f).offset for f, _ in O._fields_]
    assert c == py


def test_header_compiles_as_c_and_cpp(tmp_path):
    for lang, compiler in (("c", "gcc"), ("c++", "g++")):
        src = tmp_path / f"h.{'c' if lang == 'c' else 'cpp'}"
        src.write_text('#include "spec_verify.h"\nint f(void){return SV_OK + SV_MODE_GREEDY;}\n')
        subprocess.run([compiler, "-x", lang, "-c", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        "-o", str(tmp_path / "h.o"), str(src)], check=True)


def test_c_program_links_and_calls_the_library(tmp_path, L):
    """A plain C consumer: compiled with gcc against the header, linked against the
    in-tree library, calling only what is safe on any machine (version, status
    strings, calls rejected before any CUDA work)."""
    src = tmp_path / "consumer.c"
    src.write_text(r"""
#include <stdio.h>
#include "spec_verify.h"
int main(void) {
    sv_options_t o = {0};
    sv_status_t bad_b = spec_verify(NULL, NULL, NULL, NULL, 0, 1, 10, NULL, 0,
                                    SV_MODE_STOCHASTIC | SV_DTYPE_BF16, NULL, NULL, NULL);
    sv_status_t bad_mode = spec_verify_ex(NULL, NULL, NULL, NULL, 1, 1, 10, NULL, 0, 7, NULL, NULL,
                                          NULL, NULL, NULL, NULL, 0, &o, NULL);
    size_t ws = spec_verify_workspace_size(0, 1, 10, 0, 0, NULL);
    sv_status_t bad_rows = spec_sample(NULL, NULL, 0, 10, NULL, 0, SV_MODE_GREEDY, NULL, NULL);
    printf("%d %d %d %zu %d %s\n", spec_verify_version(), (int)bad_b, (int)bad_mode, ws, (int)bad_rows,
           spec_verify_status_string(SV_ERR_UNSUPPORTED));
    return 0;
}
""")
    libdir = os.path.dirname(sv.LIB_PATH)
    exe = tmp_path / "consumer"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                    "-L", libdir, "-lspec_verify", f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split(maxsplit=5)
    assert int(out[0]) == sv.spec_verify_version()
    assert [int(x) for x in out[1:5]] == [sv.SV_ERR_INVALID_ARG, sv.SV_ERR_INVALID_ARG, 0, sv.SV_ERR_INVALID_ARG]
    assert out[5].strip() == sv.spec_verify_status_string(sv.SV_ERR_UNSUPPORTED)


# fake but aligned device pointers: argument checks run before any CUDA call
P = 0x7f0000000000


def _verify(**kw):
    a = dict(target_logits=P, draft_logits=P, draft_tokens=P, uniforms=P, B=2, k=3, V=100,
             temperature=None, top_k=0, mode=0, out_tokens=P, out_n_accepted=P, stream=0)
    a.update(kw)
    return sv.spec_verify(**a)


@pytest.mark.parametrize("kw", [
    dict(B=0), dict(B=-1), dict(k=0), dict(V=0), dict(top_k=-1),
    dict(mode=2), dict(mode=3 << 8), dict(mode=1 << 9),
    dict(target_logits=None), dict(draft_tokens=None), dict(out_tokens=None),
    dict(out_n_accepted=None), dict(draft_logits=None), dict(uniforms=None),
    dict(target_logits=P + 1), dict(draft_logits=P + 1), dict(mode=sv.SV_DTYPE_F32, target_logits=P + 2),
    dict(draft_tokens=P + 2), dict(uniforms=P + 1), dict(temperature=P + 3), dict(out_tokens=P + 1),
    dict(B=2 ** 31 - 1, k=2 ** 20, V=2 ** 31 - 1),
])
def test_invalid_arguments_rejected_before_launch(L, kw):
    assert _verify(**kw) == sv.SV_ERR_INVALID_ARG


def test_greedy_allows_null_draft_and_uniforms(L):
    st = _verify(mode=sv.SV_MODE_GREEDY, draft_logits=None, uniforms=None)
    assert st != sv.SV_ERR_INVALID_ARG


@pytest.mark.parametrize("field,val", [("chunks_per_row", -1), ("threads", 64),
                                       ("threads", 1024), ("topk_path", 3), ("topk_path", -1)])
def test_invalid_options_rejected(L, field, val):
    o = sv.make_options(**{field: val})
    st = sv.spec_verify_ex(P, P, P, P, 2, 3, 100, None, 0, 0, P, P, None, None, None, None, 0, o, 0)
    assert st == sv.SV_ERR_INVALID_ARG
    assert sv.spec_verify_workspace_size(2, 3, 100, 0, 0, o) == 0


def test_misaligned_top_p_rejected(L):
    o = sv.make_options()
    o.top_p = 0x1002  # not 4-byte aligned
    st = sv.spec_verify_ex(P, P, P, P, 2, 3, 100, None, 50, 0, P, P, None, None, None, None, 0, o, 0)
    assert st == sv.SV_ERR_INVALID_ARG


@pytest.mark.parametrize("kw", [dict(B=0), dict(k=0), dict(V=0), dict(top_k=-1), dict(mode=7)])
def test_workspace_size_invalid_arguments(L, kw):
    a = dict(B=2, k=3, V=100, top_k=0, mode=0)
    a.update(kw)
    assert sv.spec_verify_workspace_size(**a) == 0


@pytest.mark.parametrize("kw", [dict(rows=0), dict(V=0), dict(top_k=-1), dict(mode=5),
                                dict(logits=None), dict(uniforms=None), dict(out_tokens=None),
                                dict(logits=P + 1)])
def test_sample_invalid_arguments(L, kw):
    a = dict(logits=P, uniforms=P, rows=4, V=50, temperature=None, top_k=0, mode=0, out_tokens=P,
             stream=0)
    a.update(kw)
    assert sv.spec_sample(**a) == sv.SV_ERR_INVALID_ARG


def test_no_device_is_reported_as_unsupported(L):
    import torch

    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    assert _verify() == sv.SV_ERR_UNSUPPORTED


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    # monkeypatch puts the loaded library back afterwards; a module reload here
    # would leave the options class out of step with the loaded signatures
    monkeypatch.setattr(sv, "_lib", None)
    monkeypatch.setattr(sv, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        sv.lib()


# --------------------------------------------------------------------------
# tensor wrappers: layout checks before the call (CPU tensors, no GPU needed)
# --------------------------------------------------------------------------

def _verify_args(B=3, k=2, V=17):
    import torch

    return dict(target=torch.zeros(B, k + 1, V, dtype=torch.bfloat16),
                draft=torch.zeros(B, k, V, dtype=torch.bfloat16),
                draft_tokens=torch.zeros(B, k, dtype=torch.int32),
                uniforms=torch.zeros(B, k + 1, dtype=torch.float32),
                temperature=torch.ones(B, dtype=torch.float32))


def _bad_verify_cases():
    import torch

    def t(**kw):
        a = _verify_args()
        a.update(kw)
        return a

    return [
        (t(draft_tokens=torch.zeros(3, 2, dtype=torch.int64)), TypeError, "draft_tokens"),
        (t(uniforms=torch.zeros(3, 3, dtype=torch.float64)), TypeError, "uniforms"),
        (t(draft=torch.zeros(3, 2, 17, dtype=torch.float32)), TypeError, "draft"),
        (t(target=torch.zeros(3, 3, 17, dtype=torch.float16)), TypeError, "bfloat16 or float32"),
        (t(draft_tokens=torch.zeros(3, 3, dtype=torch.int32)), ValueError, "draft_tokens"),
        (t(temperature=torch.ones(4, dtype=torch.float32)), ValueError, "temperature"),
        (t(uniforms=torch.zeros(3, 3, dtype=torch.float32).t()), ValueError, "contiguous"),
        (t(draft=torch.zeros(3, 17, 2, dtype=torch.bfloat16).transpose(1, 2)), ValueError, "contiguous"),
        (t(uniforms=None), ValueError, "uniforms is required"),
        (t(target=torch.zeros(3, 17, dtype=torch.bfloat16)), ValueError, "target must be"),
        (t(draft_tokens=[[0, 0]] * 3), TypeError, "torch tensor"),
        (t(), ValueError, "CUDA device"),
    ]


@pytest.mark.parametrize("i", range(12))
def test_verify_wrapper_checks_layout(i):
    import draft_token_verification_verify_b200 as sv

    args, exc, msg = _bad_verify_cases()[i]
    with pytest.raises(exc, match=msg):
        sv.verify(args["target"], args["draft"], args["draft_tokens"], args["uniforms"], args["temperature"], 5)


def test_verify_wrapper_greedy_ignores_stochastic_inputs():
    import torch

    import draft_token_verification_verify_b200 as sv

    a = _verify_args()
    # draft, uniforms and temperature of the wrong kind are not read in greedy mode
    with pytest.raises(ValueError, match="CUDA device"):
        sv.verify(a["target"], None, a["draft_tokens"], torch.zeros(1, dtype=torch.float64), None, greedy=True)


def test_verify_wrapper_checks_outputs():
    import torch

    import draft_token_verification_verify_b200 as sv

    a = _verify_args()
    with pytest.raises(ValueError, match="out_tokens"):
        sv.verify(**a, out_tokens=torch.zeros(3, 2, dtype=torch.int32))
    with pytest.raises(TypeError, match="out_p"):
        sv.verify(**a, out_p=torch.zeros(3, 2, dtype=torch.float64))
    with pytest.raises(ValueError, match="out_status"):
        sv.verify(**a, out_status=torch.zeros(2, dtype=torch.int32))


def test_sample_wrapper_checks_layout():
    import torch

    import draft_token_verification_verify_b200 as sv

    logits = torch.zeros(4, 3, 11, dtype=torch.float32)
    u = torch.zeros(4, 3, dtype=torch.float32)
    with pytest.raises(TypeError, match="uniforms"):
        sv.sample(logits, u.double())
    with pytest.raises(ValueError, match="uniforms"):
        sv.sample(logits, torch.zeros(4, dtype=torch.float32))
    with pytest.raises(ValueError, match="temperature"):
        sv.sample(logits, u, torch.ones(4, dtype=torch.float32))
    with pytest.raises(ValueError, match="contiguous"):
        sv.sample(torch.zeros(4, 11, 3).transpose(1, 2), u)
    with pytest.raises(ValueError, match="CUDA device"):
        sv.sample(logits, u, torch.ones(12, dtype=torch.float32))   # one temperature per row: valid
    with pytest.raises(ValueError, match="CUDA device"):
        sv.sample(logits, greedy=True)


@pytest.mark.parametrize("kw", [dict(B=0), dict(N=0), dict(N=257), dict(V=0), dict(top_k=-1), dict(mode=7),
                                dict(target=None), dict(tokens=None), dict(parents=None), dict(draft=None),
                                dict(uniforms=None), dict(target=P + 1), dict(tokens=P + 2), dict(out_p=P + 2)])
def test_tree_invalid_arguments(L, kw):
    a = dict(target=P, draft=P, tokens=P, parents=P, uniforms=P, B=2, N=3, V=100, temperature=None, top_k=0,
             mode=0, out_tokens=P, out_n=P, out_nodes=None, out_p=None, out_q=None)
    a.update(kw)
    st = sv.spec_verify_tree(a["target"], a["draft"], a["tokens"], a["parents"], a["uniforms"], a["B"], a["N"],
                             a["V"], a["temperature"], a["top_k"], a["mode"], a["out_tokens"], a["out_n"],
                             a["out_nodes"], a["out_p"], a["out_q"], stream=0)
    assert st == sv.SV_ERR_INVALID_ARG


def test_tree_greedy_needs_no_draft(L):
    _no_gpu()
    # greedy reads neither the draft logits nor the uniforms: NULL passes the checks
    # (on a machine without a GPU the call then stops at the device: unsupported)
    st = sv.spec_verify_tree(P, None, P, P, None, 2, 3, 100, None, 0, sv.SV_MODE_GREEDY, P, P, stream=0)
    assert st in (sv.SV_OK, sv.SV_ERR_UNSUPPORTED)


def test_tree_ex_checks_the_workspace(L):
    st = sv.spec_verify_tree_ex(P, P, P, P, P, 2, 3, 100, None, 5, 0, P, P, workspace=P + 8, workspace_bytes=1 << 20,
                                stream=0)
    assert st == sv.SV_ERR_INVALID_ARG  # not 16-byte aligned
    assert sv.spec_verify_tree_workspace_size(0, 3, 100, 5, 0) == 0
    assert sv.spec_verify_tree_workspace_size(2, 0, 100, 5, 0) == 0


@pytest.mark.parametrize("kw", [dict(B=0), dict(k=0), dict(V=0), dict(H=0), dict(H=100), dict(hidden=None),
                                dict(weight=None), dict(drafts=None), dict(out_tokens=None), dict(out_n=None),
                                dict(hidden=P + 8), dict(weight=P + 2), dict(drafts=P + 2), dict(out_argmax=P + 1),
                                dict(out_status=P + 2), dict(workspace=P + 8), dict(workspace_bytes=16),
                                dict(V=1 << 30)])
def test_head_invalid_arguments(L, kw):
    a = dict(hidden=P, weight=P, drafts=P, B=4, k=3, V=1000, H=256, out_tokens=P, out_n=P, out_argmax=None,
             workspace=P, workspace_bytes=1 << 20, out_status=None)
    a.update(kw)
    st = sv.spec_verify_head_greedy(a["hidden"], a["weight"], a["drafts"], a["B"], a["k"], a["V"], a["H"],
                                    a["out_tokens"], a["out_n"], a["out_argmax"], a["workspace"],
                                    a["workspace_bytes"], None, a["out_status"], stream=0)
    expect = sv.SV_ERR_UNSUPPORTED if kw.get("V") == 1 << 30 else sv.SV_ERR_INVALID_ARG
    assert st == expect, kw


def test_head_processors_unsupported(L):
    import torch

    tp = torch.ones(4, dtype=torch.float32)
    st = sv.spec_verify_head_greedy(P, P, P, 4, 3, 1000, 256, P, P, None, P, 1 << 20,
                                    sv.make_options(top_p=tp), None, stream=0)
    assert st == sv.SV_ERR_UNSUPPORTED


def test_head_workspace_size(L):
    # one 8-byte running best per row, and a flag
    assert sv.spec_verify_head_workspace_size(64, 4, 151936, 4096) == 320 * 8 + 16
    assert sv.spec_verify_head_workspace_size(3, 2, 1000, 200) == ((9 * 8 + 15) // 16) * 16 + 16
    assert sv.spec_verify_head_workspace_size(0, 4, 100, 64) == 0
    assert sv.spec_verify_head_workspace_size(2, 4, 100, 60) == 0   # H not a multiple of 8
    assert sv.spec_verify_head_workspace_size(2, 4, 1 << 30, 64) == 0


def test_head_no_device_is_unsupported(L):
    _no_gpu()
    st = sv.spec_verify_head_greedy(P, P, P, 4, 3, 1000, 256, P, P, None, P, 1 << 20, None, None, stream=0)
    assert st == sv.SV_ERR_UNSUPPORTED
