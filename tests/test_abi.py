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
        "spec_verify_static", "spec_verify_status_string", "spec_verify_version", "spec_verify_workspace_size"])


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", _build.LIB], check=True,
                         capture_output=True, text=True).stdout
    exported = set(re.findall(r"\sT\s+(\w+)$", out, flags=re.M))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(L, name)
    # nothing else leaks out of the C ABI
    assert exported == set(declared_functions())


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
  printf("%zu %zu %zu %zu %zu %zu %zu %zu %zu\n", sizeof(sv_options_t),
         offsetof(sv_options_t, chunks_per_row), offsetof(sv_options_t, threads),
         offsetof(sv_options_t, topk_path), offsetof(sv_options_t, event_start),
         offsetof(sv_options_t, event_stop), offsetof(sv_options_t, wait_timeout_ns),
         offsetof(sv_options_t, test_extra_tx), offsetof(sv_options_t, top_p));
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


def test_sampler_refuses_top_p(L):
    o = sv.make_options()
    o.top_p = 0x1000
    st = sv.spec_sample_ex(P, P, 4, 50, None, 5, 0, P, None, 0, o, 0)
    assert st == sv.SV_ERR_UNSUPPORTED


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
    import importlib

    monkeypatch.setattr(sv, "_lib", None)
    monkeypatch.setattr(sv, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        sv.lib()
    importlib.reload(sv)
