"""Batched speculative-sampling verification on B200: Python binding.

Argument marshalling only.  Every entry point forwards to the C ABI of
``libspec_verify.so`` (declared in ``include/spec_verify.h``), whose CUDA
kernels do all of the work; there is no Python or CPU fallback, and a
missing library raises ``ImportError``-style errors on first use.

Pointers may be given as torch tensors (their ``data_ptr()`` is passed), as
integers, or as ``None`` (NULL).  Streams may be a ``torch.cuda.Stream``, a
raw ``cudaStream_t`` integer, or ``None`` for torch's current stream.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

from . import _build

SV_OK = 0
SV_ERR_INVALID_ARG = -1
SV_ERR_UNSUPPORTED = -2
SV_ERR_CUDA = -3
SV_ERR_DEVICE_TIMEOUT = -4

SV_MODE_STOCHASTIC = 0
SV_MODE_GREEDY = 1
SV_DTYPE_BF16 = 0 << 8
SV_DTYPE_F32 = 1 << 8
SV_STATIC_WORKSPACE_BYTES = 4 << 20  # scratch bytes available to spec_verify_static

LIB_PATH = _build.LIB

__all__ = [
    "SV_OK", "SV_ERR_INVALID_ARG", "SV_ERR_UNSUPPORTED", "SV_ERR_CUDA", "SV_ERR_DEVICE_TIMEOUT",
    "SV_MODE_STOCHASTIC", "SV_MODE_GREEDY", "SV_DTYPE_BF16", "SV_DTYPE_F32", "SvOptions",
    "SpecVerifyError", "lib", "spec_verify", "spec_verify_ex", "spec_verify_workspace_size",
    "spec_verify_static", "SV_STATIC_WORKSPACE_BYTES",
    "spec_sample", "spec_sample_ex", "spec_sample_workspace_size", "make_options",
    "spec_verify_status_string", "spec_verify_version", "spec_verify_pool_allocations", "verify", "sample",
    "spec_verify_tree", "spec_verify_tree_ex", "spec_verify_tree_workspace_size", "verify_tree",
    "spec_verify_head_greedy", "spec_verify_head_workspace_size", "verify_head_greedy",
]


class SvOptions(ctypes.Structure):
    """Mirror of ``sv_options_t``."""
    _fields_ = [
        ("chunks_per_row", ctypes.c_int),
        ("threads", ctypes.c_int),
        ("topk_path", ctypes.c_int),
        ("event_start", ctypes.c_void_p),
        ("event_stop", ctypes.c_void_p),
        ("wait_timeout_ns", ctypes.c_uint64),
        ("test_extra_tx", ctypes.c_uint32),
        ("top_p", ctypes.c_void_p),
        ("vocab_mask", ctypes.c_void_p),
        ("rep_ids", ctypes.c_void_p),
        ("n_rep", ctypes.c_int),
        ("rep_penalty", ctypes.c_void_p),
        ("rows_per_sequence", ctypes.c_int),
    ]


class SpecVerifyError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what} failed: {spec_verify_status_string(status)} ({status})")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load the C-ABI library (built in-tree by ``__graft_entry__.build()``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run __graft_entry__.build() first")
        L = ctypes.CDLL(LIB_PATH)
        P, I = ctypes.c_void_p, ctypes.c_int
        L.spec_verify.argtypes = [P, P, P, P, I, I, I, P, I, I, P, P, P]
        L.spec_verify.restype = I
        Z = ctypes.c_size_t
        OP = ctypes.POINTER(SvOptions)
        L.spec_verify_ex.argtypes = [P, P, P, P, I, I, I, P, I, I, P, P, P, P, P, P, Z, OP, P]
        L.spec_verify_ex.restype = I
        L.spec_verify_static.argtypes = [P, P, P, P, I, I, I, P, I, I, P, P, P, P, P, OP, P]
        L.spec_verify_static.restype = I
        L.spec_verify_tree.argtypes = [P, P, P, P, P, I, I, I, P, I, I, P, P, P, P, P, P]
        L.spec_verify_tree.restype = I
        L.spec_verify_tree_ex.argtypes = [P, P, P, P, P, I, I, I, P, I, I, P, P, P, P, P, P, Z, P]
        L.spec_verify_tree_ex.restype = I
        L.spec_verify_tree_workspace_size.argtypes = [I, I, I, I, I]
        L.spec_verify_tree_workspace_size.restype = Z
        L.spec_verify_head_greedy.argtypes = [P, P, P, I, I, I, I, P, P, P, P, Z, OP, P, P]
        L.spec_verify_head_greedy.restype = I
        L.spec_verify_head_workspace_size.argtypes = [I, I, I, I]
        L.spec_verify_head_workspace_size.restype = Z
        L.spec_verify_workspace_size.argtypes = [I, I, I, I, I, OP]
        L.spec_verify_workspace_size.restype = Z
        L.spec_sample.argtypes = [P, P, I, I, P, I, I, P, P]
        L.spec_sample.restype = I
        L.spec_sample_ex.argtypes = [P, P, I, I, P, I, I, P, P, Z, OP, P]
        L.spec_sample_ex.restype = I
        L.spec_sample_workspace_size.argtypes = [I, I, I, I, OP]
        L.spec_sample_workspace_size.restype = Z
        L.spec_verify_status_string.argtypes = [I]
        L.spec_verify_status_string.restype = ctypes.c_char_p
        L.spec_verify_version.argtypes = []
        L.spec_verify_version.restype = I
        L.spec_verify_pool_allocations.argtypes = []
        L.spec_verify_pool_allocations.restype = ctypes.c_ulonglong
        _lib = L
    return _lib


def _p(x):
    if x is None:
        return None
    if hasattr(x, "data_ptr"):
        return ctypes.c_void_p(x.data_ptr())
    return ctypes.c_void_p(int(x))


def _stream(s):
    if s is None:
        import torch

        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if hasattr(s, "cuda_stream"):
        return ctypes.c_void_p(s.cuda_stream)
    return ctypes.c_void_p(int(s))


def _event(e):
    if e is None:
        return None
    if hasattr(e, "cuda_event"):
        return e.cuda_event
    return int(e)


def _opts(opts: Optional[SvOptions]):
    return None if opts is None else ctypes.byref(opts)


def spec_verify_status_string(status: int) -> str:
    return lib().spec_verify_status_string(int(status)).decode()


def spec_verify_version() -> int:
    return lib().spec_verify_version()


def spec_verify_pool_allocations() -> int:
    """Workspaces taken from the library's pool so far (calls without one)."""
    return int(lib().spec_verify_pool_allocations())


def spec_verify(target_logits, draft_logits, draft_tokens, uniforms, B, k, V, temperature, top_k,
                mode, out_tokens, out_n_accepted, stream=None) -> int:
    return lib().spec_verify(_p(target_logits), _p(draft_logits), _p(draft_tokens), _p(uniforms),
                             int(B), int(k), int(V), _p(temperature), int(top_k), int(mode),
                             _p(out_tokens), _p(out_n_accepted), _stream(stream))


def spec_verify_ex(target_logits, draft_logits, draft_tokens, uniforms, B, k, V, temperature, top_k,
                   mode, out_tokens, out_n_accepted, out_p=None, out_q=None, out_status=None,
                   workspace=None, workspace_bytes=0, opts: Optional[SvOptions] = None,
                   stream=None) -> int:
    return lib().spec_verify_ex(_p(target_logits), _p(draft_logits), _p(draft_tokens), _p(uniforms),
                                int(B), int(k), int(V), _p(temperature), int(top_k), int(mode),
                                _p(out_tokens), _p(out_n_accepted), _p(out_p), _p(out_q),
                                _p(out_status), _p(workspace), int(workspace_bytes), _opts(opts),
                                _stream(stream))


def spec_verify_static(target_logits, draft_logits, draft_tokens, uniforms, B, k, V, temperature, top_k,
                       mode, out_tokens, out_n_accepted, out_p=None, out_q=None, out_status=None,
                       opts: Optional[SvOptions] = None, stream=None) -> int:
    """``spec_verify_ex`` without a workspace argument and without any device
    allocation: scratch comes from the library's fixed per-device buffer of
    ``SV_STATIC_WORKSPACE_BYTES``.  For callers that cannot allocate during
    the call.  Overlapping calls on different streams share that buffer and
    must not run at the same time."""
    return lib().spec_verify_static(_p(target_logits), _p(draft_logits), _p(draft_tokens), _p(uniforms),
                                    int(B), int(k), int(V), _p(temperature), int(top_k), int(mode),
                                    _p(out_tokens), _p(out_n_accepted), _p(out_p), _p(out_q),
                                    _p(out_status), _opts(opts), _stream(stream))


def spec_verify_workspace_size(B, k, V, top_k, mode, opts: Optional[SvOptions] = None) -> int:
    return lib().spec_verify_workspace_size(int(B), int(k), int(V), int(top_k), int(mode), _opts(opts))


def spec_sample_workspace_size(rows, V, top_k, mode, opts: Optional[SvOptions] = None) -> int:
    return lib().spec_sample_workspace_size(int(rows), int(V), int(top_k), int(mode), _opts(opts))


def spec_sample(logits, uniforms, rows, V, temperature, top_k, mode, out_tokens, stream=None) -> int:
    return lib().spec_sample(_p(logits), _p(uniforms), int(rows), int(V), _p(temperature), int(top_k),
                             int(mode), _p(out_tokens), _stream(stream))


def spec_sample_ex(logits, uniforms, rows, V, temperature, top_k, mode, out_tokens, workspace=None,
                   workspace_bytes=0, opts: Optional[SvOptions] = None, stream=None) -> int:
    return lib().spec_sample_ex(_p(logits), _p(uniforms), int(rows), int(V), _p(temperature),
                                int(top_k), int(mode), _p(out_tokens), _p(workspace),
                                int(workspace_bytes), _opts(opts), _stream(stream))


def make_options(chunks_per_row=0, threads=0, topk_path=0, event_start=None, event_stop=None,
                 wait_timeout_ns=0, test_extra_tx=0, top_p=None, vocab_mask=None, rep_ids=None,
                 rep_penalty=None, rows_per_sequence=0) -> SvOptions:
    """``sv_options_t``.  Per-sequence processor inputs are device tensors or
    None: ``top_p`` [S] fp32 (nucleus), ``vocab_mask`` [S, ceil(V/32)] uint32
    bit words (passed as int32), ``rep_ids`` [S, n_rep] int32 and
    ``rep_penalty`` [S] fp32.  Keep them alive until the call completes."""
    n_rep = 0
    if rep_ids is not None:
        n_rep = rep_ids.shape[-1] if rep_ids.dim() > 1 else rep_ids.numel()
    ptr = lambda t: None if t is None else _p(t).value
    return SvOptions(chunks_per_row, threads, topk_path, _event(event_start), _event(event_stop),
                     wait_timeout_ns, test_extra_tx, ptr(top_p), ptr(vocab_mask), ptr(rep_ids), n_rep,
                     ptr(rep_penalty), rows_per_sequence)


def _dtype_code(t) -> int:
    import torch

    if t.dtype == torch.bfloat16:
        return SV_DTYPE_BF16
    if t.dtype == torch.float32:
        return SV_DTYPE_F32
    raise TypeError(f"logits must be bfloat16 or float32, got {t.dtype}")


def _check(t, name, dtypes, numel, device):
    """Raise unless tensor ``t`` has the layout the C ABI reads: one of
    ``dtypes``, ``numel`` elements, contiguous, on ``device``."""
    if t is None:
        raise ValueError(f"{name} is required")
    if not hasattr(t, "data_ptr"):
        raise TypeError(f"{name} must be a torch tensor (use the spec_* functions for raw pointers)")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} must be {' or '.join(str(d) for d in dtypes)}, got {t.dtype}")
    if t.numel() != numel:
        raise ValueError(f"{name} must have {numel} elements, got {t.numel()} (shape {tuple(t.shape)})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, the logits on {device}")


def _check_cuda(device):
    if device.type != "cuda":
        raise ValueError(f"tensors must be on a CUDA device, got {device}")


def spec_verify_tree(target_logits, draft_logits, tokens, parents, uniforms, B, N, V, temperature, top_k, mode,
                     out_tokens, out_n_accepted, out_nodes=None, out_p=None, out_q=None, stream=None) -> int:
    return lib().spec_verify_tree(_p(target_logits), _p(draft_logits), _p(tokens), _p(parents), _p(uniforms),
                                  int(B), int(N), int(V), _p(temperature), int(top_k), int(mode),
                                  _p(out_tokens), _p(out_n_accepted), _p(out_nodes), _p(out_p), _p(out_q),
                                  _stream(stream))


def spec_verify_tree_ex(target_logits, draft_logits, tokens, parents, uniforms, B, N, V, temperature, top_k, mode,
                        out_tokens, out_n_accepted, out_nodes=None, out_p=None, out_q=None, workspace=None,
                        workspace_bytes=0, stream=None) -> int:
    return lib().spec_verify_tree_ex(_p(target_logits), _p(draft_logits), _p(tokens), _p(parents), _p(uniforms),
                                     int(B), int(N), int(V), _p(temperature), int(top_k), int(mode),
                                     _p(out_tokens), _p(out_n_accepted), _p(out_nodes), _p(out_p), _p(out_q),
                                     _p(workspace), int(workspace_bytes), _stream(stream))


def spec_verify_tree_workspace_size(B, N, V, top_k, mode) -> int:
    return int(lib().spec_verify_tree_workspace_size(int(B), int(N), int(V), int(top_k), int(mode)))


def verify_tree(target, draft, tokens, parents, uniforms=None, temperature=None, top_k: int = 0,
                greedy: bool = False, out_nodes=None, out_p=None, out_q=None, workspace=None, stream=None):
    """Tensor convenience wrapper around ``spec_verify_tree_ex``.  ``workspace``:
    None allocates (with torch) the bytes the list walk needs, if any; False
    runs the walk over the rows; a uint8 tensor is used as given.  Target and draft
    [B, N+1, V] (one row per node, node 0 the verified context), tokens and
    parents [B, N] int32 (node n at index n - 1), uniforms [B, N+1] fp32,
    temperature [B] fp32 or None; optional outputs out_nodes [B, N+1] int32,
    out_p / out_q [B, N] fp32.  Checked like ``verify``.  Returns
    (out_tokens [B, N+1], out_n_accepted [B])."""
    import torch

    if target.dim() != 3:
        raise ValueError(f"target must be [B, N+1, V], got shape {tuple(target.shape)}")
    B, n1, V = target.shape
    N = n1 - 1
    dev = target.device
    f32, i32 = (torch.float32,), (torch.int32,)
    mode = (SV_MODE_GREEDY if greedy else SV_MODE_STOCHASTIC) | _dtype_code(target)
    _check(target, "target", (target.dtype,), B * n1 * V, dev)
    _check(tokens, "tokens", i32, B * N, dev)
    _check(parents, "parents", i32, B * N, dev)
    if not greedy:
        _check(draft, "draft", (target.dtype,), B * n1 * V, dev)
        _check(uniforms, "uniforms", f32, B * n1, dev)
        if temperature is not None:
            _check(temperature, "temperature", f32, B, dev)
        for t, name in ((out_p, "out_p"), (out_q, "out_q")):
            if t is not None:
                _check(t, name, f32, B * N, dev)
    if out_nodes is not None:
        _check(out_nodes, "out_nodes", i32, B * n1, dev)
    _check_cuda(dev)
    out_tokens = torch.empty((B, n1), dtype=torch.int32, device=dev)
    out_n = torch.empty((B,), dtype=torch.int32, device=dev)
    if workspace is None:
        need = spec_verify_tree_workspace_size(B, N, V, top_k, mode)
        workspace = torch.empty((need,), dtype=torch.uint8, device=dev) if need else False
    if workspace is False:
        workspace = None
    elif workspace is not None:
        _check(workspace, "workspace", (workspace.dtype,), workspace.numel(), dev)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = spec_verify_tree_ex(target, None if greedy else draft, tokens, parents, None if greedy else uniforms, B, N, V,
                             None if greedy else temperature, top_k, mode, out_tokens, out_n, out_nodes,
                             None if greedy else out_p, None if greedy else out_q, workspace, wbytes, stream)
    if st != SV_OK:
        raise SpecVerifyError(st, "spec_verify_tree_ex")
    return out_tokens, out_n


def spec_verify_head_greedy(hidden, weight, draft_tokens, B, k, V, H, out_tokens, out_n_accepted,
                            out_argmax=None, workspace=None, workspace_bytes=0,
                            opts: Optional[SvOptions] = None, out_status=None, stream=None) -> int:
    return lib().spec_verify_head_greedy(_p(hidden), _p(weight), _p(draft_tokens), int(B), int(k), int(V), int(H),
                                         _p(out_tokens), _p(out_n_accepted), _p(out_argmax), _p(workspace),
                                         int(workspace_bytes), _opts(opts), _p(out_status), _stream(stream))


def spec_verify_head_workspace_size(B, k, V, H) -> int:
    return int(lib().spec_verify_head_workspace_size(int(B), int(k), int(V), int(H)))


def verify_head_greedy(hidden, weight, draft_tokens, out_argmax=None, out_status=None, workspace=None,
                       opts: Optional[SvOptions] = None, stream=None):
    """Tensor convenience wrapper around ``spec_verify_head_greedy``: hidden
    [B, k+1, H] and weight [V, H] bf16 (contiguous, on the GPU), draft_tokens
    [B, k] int32; optional out_argmax [B, k+1] and out_status [1] int32; the
    workspace (uint8) is allocated with torch when None.  Returns
    (out_tokens [B, k+1], out_n_accepted [B])."""
    import torch

    if hidden.dim() != 3 or weight.dim() != 2:
        raise ValueError(f"hidden must be [B, k+1, H] and weight [V, H], got {tuple(hidden.shape)}, "
                         f"{tuple(weight.shape)}")
    B, n1, H = hidden.shape
    V = weight.shape[0]
    k = n1 - 1
    dev = hidden.device
    bf, i32 = (torch.bfloat16,), (torch.int32,)
    _check(hidden, "hidden", bf, B * n1 * H, dev)
    _check(weight, "weight", bf, V * H, dev)
    _check(draft_tokens, "draft_tokens", i32, B * k, dev)
    if out_argmax is not None:
        _check(out_argmax, "out_argmax", i32, B * n1, dev)
    if out_status is not None:
        _check(out_status, "out_status", i32, 1, dev)
    _check_cuda(dev)
    out_tokens = torch.empty((B, n1), dtype=torch.int32, device=dev)
    out_n = torch.empty((B,), dtype=torch.int32, device=dev)
    if workspace is None:
        need = spec_verify_head_workspace_size(B, k, V, H)
        if need == 0:
            raise SpecVerifyError(SV_ERR_INVALID_ARG, "spec_verify_head_workspace_size")
        workspace = torch.empty((need,), dtype=torch.uint8, device=dev)
    _check(workspace, "workspace", (workspace.dtype,), workspace.numel(), dev)
    wbytes = workspace.numel() * workspace.element_size()
    st = spec_verify_head_greedy(hidden, weight, draft_tokens, B, k, V, H, out_tokens, out_n, out_argmax, workspace,
                                 wbytes, opts, out_status, stream)
    if st != SV_OK:
        raise SpecVerifyError(st, "spec_verify_head_greedy")
    return out_tokens, out_n


def verify(target, draft, draft_tokens, uniforms=None, temperature=None, top_k: int = 0,
           greedy: bool = False, out_tokens=None, out_n_accepted=None, out_p=None, out_q=None,
           out_status=None, workspace=None, opts: Optional[SvOptions] = None, stream=None):
    """Tensor convenience wrapper around ``spec_verify_ex``.

    target [B, k+1, V], draft [B, k, V] (bf16 or fp32, contiguous, on the
    GPU), draft_tokens [B, k] int32, uniforms [B, k+1] fp32, temperature [B]
    fp32 or None.  Output tensors are allocated with torch when not given; the
    workspace (a uint8 tensor) is taken from the library pool when None.
    Every tensor is checked for dtype, element count, contiguity and device
    before the call (TypeError / ValueError); greedy mode ignores draft,
    uniforms and temperature.  Returns (out_tokens [B, k+1], out_n_accepted [B]).
    """
    import torch

    if target.dim() != 3:
        raise ValueError(f"target must be [B, k+1, V], got shape {tuple(target.shape)}")
    B, k1, V = target.shape
    k = k1 - 1
    dev = target.device
    f32, i32 = (torch.float32,), (torch.int32,)
    mode = (SV_MODE_GREEDY if greedy else SV_MODE_STOCHASTIC) | _dtype_code(target)
    _check(target, "target", (target.dtype,), B * k1 * V, dev)
    _check(draft_tokens, "draft_tokens", i32, B * k, dev)
    if not greedy:  # greedy reads neither the draft logits, the uniforms nor the temperature
        _check(draft, "draft", (target.dtype,), B * k * V, dev)
        _check(uniforms, "uniforms", f32, B * k1, dev)
        if temperature is not None:
            _check(temperature, "temperature", f32, B, dev)
        for t, name in ((out_p, "out_p"), (out_q, "out_q")):
            if t is not None:
                _check(t, name, f32, B * k, dev)
    if out_tokens is not None:
        _check(out_tokens, "out_tokens", i32, B * k1, dev)
    if out_n_accepted is not None:
        _check(out_n_accepted, "out_n_accepted", i32, B, dev)
    if out_status is not None:
        _check(out_status, "out_status", i32, 1, dev)
    if workspace is not None:
        _check(workspace, "workspace", (workspace.dtype,), workspace.numel(), dev)
    _check_cuda(dev)
    if out_tokens is None:
        out_tokens = torch.empty((B, k + 1), dtype=torch.int32, device=dev)
    if out_n_accepted is None:
        out_n_accepted = torch.empty((B,), dtype=torch.int32, device=dev)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = spec_verify_ex(target, draft, draft_tokens, uniforms, B, k, V, temperature, top_k, mode,
                        out_tokens, out_n_accepted, out_p, out_q, out_status, workspace, wbytes, opts,
                        stream)
    if st != SV_OK:
        raise SpecVerifyError(st, "spec_verify_ex")
    return out_tokens, out_n_accepted


def sample(logits, uniforms=None, temperature=None, top_k: int = 0, greedy: bool = False,
           out_tokens=None, opts: Optional[SvOptions] = None, stream=None):
    """Tensor convenience wrapper around ``spec_sample_ex``: logits [..., V]
    (bf16 or fp32), uniforms and temperature fp32 with one entry per row,
    checked like the arguments of ``verify``."""
    import torch

    V = logits.shape[-1]
    rows = logits.numel() // V
    dev = logits.device
    mode = (SV_MODE_GREEDY if greedy else SV_MODE_STOCHASTIC) | _dtype_code(logits)
    _check(logits, "logits", (logits.dtype,), rows * V, dev)
    if not greedy:
        _check(uniforms, "uniforms", (torch.float32,), rows, dev)
        if temperature is not None:
            _check(temperature, "temperature", (torch.float32,), rows, dev)
    if out_tokens is not None:
        _check(out_tokens, "out_tokens", (torch.int32,), rows, dev)
    _check_cuda(dev)
    if out_tokens is None:
        out_tokens = torch.empty(logits.shape[:-1], dtype=torch.int32, device=dev)
    st = spec_sample_ex(logits, uniforms, rows, V, temperature, top_k, mode, out_tokens, None, 0, opts,
                        stream)
    if st != SV_OK:
        raise SpecVerifyError(st, "spec_sample_ex")
    return out_tokens
