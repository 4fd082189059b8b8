"""Python access to the fp64 CPU oracle (``spec_verify_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by tests/, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py``.  The CUDA library never imports it and
it never imports the CUDA library.  Arguments are numpy arrays; bf16 logits
are passed as their uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import dataclasses
from typing import Optional

import numpy as np

from . import build as _build

DTYPE_BF16 = 0
DTYPE_F32 = 1
DTYPE_F64 = 2  # logits the oracle formed itself (the output projection)

_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(_build.build())
        P, I, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        _lib.oracle_process_row.argtypes = [P, I, I, D, I, P, P]
        _lib.oracle_process_row.restype = I
        _lib.oracle_argmax_row.argtypes = [P, I, I]
        _lib.oracle_argmax_row.restype = I
        _lib.oracle_inverse_cdf.argtypes = [P, I, D, P, P, P]
        _lib.oracle_inverse_cdf.restype = I
        _lib.oracle_verify.argtypes = [P, P, P, P, I, I, I, P, I, I, I, P, P, P, P, P, P, P]
        _lib.oracle_verify.restype = I
        _lib.oracle_sample_rows.argtypes = [P, I, I, I, P, I, I, P, P, P, P]
        _lib.oracle_sample_rows.restype = I
        _lib.oracle_process_row_procs.argtypes = [P, I, I, D, I, P, P, P, P]
        _lib.oracle_process_row_procs.restype = I
        _lib.oracle_verify_procs.argtypes = [P, P, P, P, I, I, I, P, I, I, P, P, P, I, P,
                                             P, P, P, P, P, P, P]
        _lib.oracle_verify_procs.restype = I
        _lib.oracle_sample_rows_procs.argtypes = [P, I, I, I, I, P, I, P, P, P, I, P, P, P]
        _lib.oracle_sample_rows_procs.restype = I
        _lib.oracle_verify_tree.argtypes = [P, P, P, P, P, I, I, I, P, I, I, I, P, P, P, P, P, P, P, P]
        _lib.oracle_verify_tree.restype = I
        L = ctypes.c_long
        _lib.oracle_head_logits.argtypes = [P, P, L, L, I, I, P, P]
        _lib.oracle_head_logits.restype = None
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return DTYPE_BF16
    if a.dtype == np.float32:
        return DTYPE_F32
    if a.dtype == np.float64:
        return DTYPE_F64
    raise TypeError(f"logits must be uint16 (bf16 bits), float32 or float64, got {a.dtype}")


def process_row(row: np.ndarray, temperature: float = 1.0, top_k: int = 0):
    """Processed probabilities of one logit row (fp64), or None on a row error."""
    row = np.ascontiguousarray(row)
    V = row.shape[-1]
    prob = np.zeros(V, dtype=np.float64)
    work = np.zeros(V, dtype=np.float64)
    rc = lib().oracle_process_row(_ptr(row), _dtype_code(row), V, float(temperature), int(top_k),
                                  _ptr(prob), _ptr(work))
    return None if rc else prob


def argmax_row(row: np.ndarray) -> int:
    row = np.ascontiguousarray(row)
    return lib().oracle_argmax_row(_ptr(row), _dtype_code(row), row.shape[-1])


def inverse_cdf(w: np.ndarray, u: float):
    """(token, cdf_lo, cdf_hi) of the inverse-CDF draw, or None if the mass is 0."""
    w = np.ascontiguousarray(w, dtype=np.float64)
    tok = ctypes.c_int(-1)
    lo = ctypes.c_double(0)
    hi = ctypes.c_double(0)
    rc = lib().oracle_inverse_cdf(_ptr(w), w.size, float(u), ctypes.byref(tok), ctypes.byref(lo),
                                  ctypes.byref(hi))
    return None if rc else (tok.value, lo.value, hi.value)


@dataclasses.dataclass
class VerifyResult:
    tokens: np.ndarray      # [B, k+1] int32
    n_accepted: np.ndarray  # [B] int32
    p: np.ndarray           # [B, k] fp64 (NaN for greedy / error rows)
    q: np.ndarray           # [B, k] fp64
    ratio: np.ndarray       # [B, k] acceptance thresholds min(1, p/q)
    cdf_lo: np.ndarray      # [B] CDF point below the final token
    cdf_hi: np.ndarray      # [B] CDF point at the final token
    errors: int


def verify(target: np.ndarray, draft: Optional[np.ndarray], draft_tokens: np.ndarray,
           uniforms: Optional[np.ndarray], temperature: Optional[np.ndarray] = None,
           top_k: int = 0, greedy: bool = False) -> VerifyResult:
    """Verify a batch: target [B,k+1,V], draft [B,k,V], draft_tokens [B,k],
    uniforms [B,k+1], temperature [B]."""
    target = np.ascontiguousarray(target)
    B, k1, V = target.shape
    k = k1 - 1
    dt = _dtype_code(target)
    if draft is not None:
        draft = np.ascontiguousarray(draft)
        assert draft.dtype == target.dtype and draft.shape == (B, k, V)
    elif not greedy:
        raise ValueError("stochastic verification needs draft logits")
    draft_tokens = np.ascontiguousarray(draft_tokens, dtype=np.int32).reshape(B, k)
    if uniforms is not None:
        uniforms = np.ascontiguousarray(uniforms, dtype=np.float32).reshape(B, k + 1)
    elif not greedy:
        raise ValueError("stochastic verification needs uniforms")
    if temperature is not None:
        temperature = np.ascontiguousarray(temperature, dtype=np.float32).reshape(B)
    tokens = np.empty((B, k + 1), dtype=np.int32)
    n = np.empty(B, dtype=np.int32)
    p = np.empty((B, max(k, 0)), dtype=np.float64)
    q = np.empty_like(p)
    ratio = np.empty_like(p)
    lo = np.empty(B, dtype=np.float64)
    hi = np.empty(B, dtype=np.float64)
    errs = lib().oracle_verify(_ptr(target), _ptr(draft), _ptr(draft_tokens), _ptr(uniforms), B, k,
                               V, _ptr(temperature), int(top_k), int(bool(greedy)), dt,
                               _ptr(tokens), _ptr(n), _ptr(p), _ptr(q), _ptr(ratio), _ptr(lo),
                               _ptr(hi))
    if errs < 0:
        raise MemoryError("oracle_verify could not allocate its work arrays")
    return VerifyResult(tokens, n, p, q, ratio, lo, hi, errs)


def sample_rows(logits: np.ndarray, u: Optional[np.ndarray], temperature: Optional[np.ndarray] = None,
                top_k: int = 0, greedy: bool = False):
    """One token per row of ``logits`` [..., V]; returns (tokens, cdf_lo, cdf_hi)."""
    logits = np.ascontiguousarray(logits)
    shape = logits.shape[:-1]
    V = logits.shape[-1]
    rows = int(np.prod(shape)) if shape else 1
    if u is not None:
        u = np.ascontiguousarray(u, dtype=np.float32).reshape(rows)
    elif not greedy:
        raise ValueError("stochastic sampling needs uniforms")
    if temperature is not None:
        temperature = np.ascontiguousarray(temperature, dtype=np.float32).reshape(rows)
    out = np.empty(rows, dtype=np.int32)
    lo = np.empty(rows, dtype=np.float64)
    hi = np.empty(rows, dtype=np.float64)
    errs = lib().oracle_sample_rows(_ptr(logits), _dtype_code(logits), rows, V, _ptr(temperature),
                                    int(top_k), int(bool(greedy)), _ptr(u), _ptr(out), _ptr(lo),
                                    _ptr(hi))
    if errs < 0:
        raise MemoryError("oracle_sample_rows could not allocate its work arrays")
    return out.reshape(shape), lo.reshape(shape), hi.reshape(shape)


def draft_tokens_for(case) -> np.ndarray:
    """The proposer's tokens for a ``workloads.Case``: d_i ~ q_i processed with
    the case's temperature and top-k (stochastic), or the argmax of the noisy
    proxy (greedy)."""
    if case.mode == "greedy":
        tok, _, _ = sample_rows(case.draft_proxy, None, greedy=True)
        return tok.astype(np.int32)
    temp = np.repeat(case.temperature, case.k)
    tok, _, _ = sample_rows(case.draft, case.draft_uniforms, temp, case.top_k)
    return tok.astype(np.int32)


# ---- further logits processors (readings R12..R15 in spec_verify_oracle.c) -----------

class _Procs(ctypes.Structure):
    """Mirror of the oracle's ``or_procs_t``."""
    _fields_ = [("top_p", ctypes.c_double), ("rep_penalty", ctypes.c_double),
                ("rep_ids", ctypes.c_void_p), ("n_rep", ctypes.c_int), ("mask", ctypes.c_void_p)]


def allow_mask(V: int, allowed) -> np.ndarray:
    """Bitmask words (uint32, ceil(V/32)) allowing exactly the token ids in ``allowed``."""
    words = np.zeros((V + 31) // 32, dtype=np.uint32)
    for v in np.asarray(allowed, dtype=np.int64).ravel():
        words[v // 32] |= np.uint32(1) << np.uint32(v % 32)
    return words


def process_row_procs(row: np.ndarray, temperature: float = 1.0, top_k: int = 0, top_p: float = 1.0,
                      rep_penalty: float = 1.0, rep_ids=None, mask: Optional[np.ndarray] = None):
    """Processed probabilities of one row with the further processors, or None on a row error."""
    row = np.ascontiguousarray(row)
    V = row.shape[-1]
    ids = None if rep_ids is None else np.ascontiguousarray(rep_ids, dtype=np.int32).ravel()
    msk = None if mask is None else np.ascontiguousarray(mask, dtype=np.uint32).ravel()
    pr = _Procs(float(top_p), float(rep_penalty), None if ids is None else ids.ctypes.data,
                0 if ids is None else ids.size, None if msk is None else msk.ctypes.data)
    prob = np.zeros(V, dtype=np.float64)
    work = np.zeros(V, dtype=np.float64)
    pv = np.zeros(2 * V, dtype=np.float64)  # V (double, long) pairs
    rc = lib().oracle_process_row_procs(_ptr(row), _dtype_code(row), V, float(temperature), int(top_k),
                                        ctypes.byref(pr), _ptr(prob), _ptr(work), _ptr(pv))
    return None if rc else prob


def _seq_arrays(B, V, top_p, rep_penalty, rep_ids, mask):
    tp = None if top_p is None else np.ascontiguousarray(np.broadcast_to(np.asarray(top_p, np.float32), (B,)))
    rp = None if rep_penalty is None else np.ascontiguousarray(
        np.broadcast_to(np.asarray(rep_penalty, np.float32), (B,)))
    ids, n_rep = None, 0
    if rep_ids is not None:
        ids = np.ascontiguousarray(rep_ids, dtype=np.int32).reshape(B, -1)
        n_rep = ids.shape[1]
    msk = None if mask is None else np.ascontiguousarray(mask, dtype=np.uint32).reshape(B, (V + 31) // 32)
    return tp, rp, ids, n_rep, msk


def verify_procs(target, draft, draft_tokens, uniforms, temperature=None, top_k: int = 0, top_p=None,
                 rep_penalty=None, rep_ids=None, mask=None) -> VerifyResult:
    """``verify`` (stochastic) with per-sequence processors: top_p [B] or scalar,
    rep_penalty [B] or scalar, rep_ids [B, n] (-1 = unused), mask [B, ceil(V/32)]."""
    target = np.ascontiguousarray(target)
    B, k1, V = target.shape
    k = k1 - 1
    draft = np.ascontiguousarray(draft)
    assert draft.dtype == target.dtype and draft.shape == (B, k, V)
    draft_tokens = np.ascontiguousarray(draft_tokens, dtype=np.int32).reshape(B, k)
    uniforms = np.ascontiguousarray(uniforms, dtype=np.float32).reshape(B, k + 1)
    if temperature is not None:
        temperature = np.ascontiguousarray(temperature, dtype=np.float32).reshape(B)
    tp, rp, ids, n_rep, msk = _seq_arrays(B, V, top_p, rep_penalty, rep_ids, mask)
    tokens = np.empty((B, k + 1), dtype=np.int32)
    n = np.empty(B, dtype=np.int32)
    p = np.empty((B, k), dtype=np.float64)
    q = np.empty_like(p)
    ratio = np.empty_like(p)
    lo = np.empty(B, dtype=np.float64)
    hi = np.empty(B, dtype=np.float64)
    errs = lib().oracle_verify_procs(_ptr(target), _ptr(draft), _ptr(draft_tokens), _ptr(uniforms), B, k,
                                     V, _ptr(temperature), int(top_k), _dtype_code(target), _ptr(tp),
                                     _ptr(rp), _ptr(ids), n_rep, _ptr(msk), _ptr(tokens), _ptr(n),
                                     _ptr(p), _ptr(q), _ptr(ratio), _ptr(lo), _ptr(hi))
    if errs < 0:
        raise MemoryError("oracle_verify_procs could not allocate its work arrays")
    return VerifyResult(tokens, n, p, q, ratio, lo, hi, errs)


def sample_rows_procs(logits, u, temperature=None, top_k: int = 0, top_p=None, rep_penalty=None,
                      rep_ids=None, mask=None) -> np.ndarray:
    """The proposer's draw with processors: logits [B, rows_per_seq, V], u [B, rows_per_seq];
    processors per sequence as in ``verify_procs``."""
    logits = np.ascontiguousarray(logits)
    B, rps, V = logits.shape
    u = np.ascontiguousarray(u, dtype=np.float32).reshape(B * rps)
    if temperature is not None:
        temperature = np.ascontiguousarray(temperature, dtype=np.float32).reshape(B * rps)
    tp, rp, ids, n_rep, msk = _seq_arrays(B, V, top_p, rep_penalty, rep_ids, mask)
    out = np.empty(B * rps, dtype=np.int32)
    errs = lib().oracle_sample_rows_procs(_ptr(logits), _dtype_code(logits), B * rps, rps, V,
                                          _ptr(temperature), int(top_k), _ptr(tp), _ptr(rp), _ptr(ids),
                                          n_rep, _ptr(msk), _ptr(u), _ptr(out))
    if errs < 0:
        raise MemoryError("oracle_sample_rows_procs could not allocate its work arrays")
    return out.reshape(B, rps)


@dataclasses.dataclass
class TreeResult:
    tokens: np.ndarray      # [B, N+1] int32: accepted tokens, the final token, then -1
    n_accepted: np.ndarray  # [B] int32 (-1: error)
    nodes: np.ndarray       # [B, N+1] int32: the accepted nodes, then -1
    p: np.ndarray           # [B, N] current-distribution probability of each tested child's token
    q: np.ndarray           # [B, N] draft probability of it (NaN: not tested)
    ratio: np.ndarray       # [B, N] acceptance threshold min(1, p/q)
    cdf_lo: np.ndarray      # [B]
    cdf_hi: np.ndarray      # [B]
    errors: int


def verify_tree(target, draft, tokens, parents, uniforms=None, temperature=None, top_k: int = 0,
                greedy: bool = False) -> TreeResult:
    """Tree verification (reading R18 of the C source): target and draft
    [B, N+1, V] (one row per node, node 0 the verified context), tokens and
    parents [B, N] (node n at index n - 1, parent < n), uniforms [B, N+1]."""
    target = np.ascontiguousarray(target)
    B, n1, V = target.shape
    N = n1 - 1
    dt = _dtype_code(target)
    if draft is not None:
        draft = np.ascontiguousarray(draft)
        assert draft.dtype == target.dtype and draft.shape == (B, N + 1, V)
    elif not greedy:
        raise ValueError("stochastic verification needs draft logits")
    tokens = np.ascontiguousarray(tokens, dtype=np.int32).reshape(B, N)
    parents = np.ascontiguousarray(parents, dtype=np.int32).reshape(B, N)
    if uniforms is not None:
        uniforms = np.ascontiguousarray(uniforms, dtype=np.float32).reshape(B, N + 1)
    elif not greedy:
        raise ValueError("stochastic verification needs uniforms")
    if temperature is not None:
        temperature = np.ascontiguousarray(temperature, dtype=np.float32).reshape(B)
    out = np.empty((B, N + 1), dtype=np.int32)
    n = np.empty(B, dtype=np.int32)
    nodes = np.empty((B, N + 1), dtype=np.int32)
    p = np.empty((B, max(N, 1)), dtype=np.float64)
    q = np.empty_like(p)
    ratio = np.empty_like(p)
    lo = np.empty(B, dtype=np.float64)
    hi = np.empty(B, dtype=np.float64)
    errs = lib().oracle_verify_tree(_ptr(target), _ptr(draft), _ptr(tokens), _ptr(parents), _ptr(uniforms),
                                    B, N, V, _ptr(temperature), int(top_k), int(bool(greedy)), dt, _ptr(out),
                                    _ptr(n), _ptr(nodes), _ptr(p), _ptr(q), _ptr(ratio), _ptr(lo), _ptr(hi))
    if errs < 0:
        raise MemoryError("oracle_verify_tree could not allocate its work arrays")
    return TreeResult(out, n, nodes, p[:, :N], q[:, :N], ratio[:, :N], lo, hi, errs)


def head_logits(hidden: np.ndarray, weight: np.ndarray, row0: int = 0, n: Optional[int] = None):
    """The output projection in fp64 (``oracle_head_logits``): hidden [rows, H]
    (any leading shape) and weight [V, H] as bf16 bit patterns (uint16).
    Returns (z, abs) for rows row0 .. row0+n, each [n, V]: z the logits summed
    in index order, abs the sums of the products' magnitudes."""
    H = hidden.shape[-1]
    h = np.ascontiguousarray(hidden, dtype=np.uint16).reshape(-1, H)
    w = np.ascontiguousarray(weight, dtype=np.uint16)
    V = w.shape[0]
    assert w.shape == (V, H)
    n = h.shape[0] - row0 if n is None else n
    z = np.empty((n, V), dtype=np.float64)
    a = np.empty((n, V), dtype=np.float64)
    lib().oracle_head_logits(_ptr(h), _ptr(w), int(row0), int(n), int(V), int(H), _ptr(z), _ptr(a))
    return z, a


@dataclasses.dataclass
class HeadResult:
    seqs: np.ndarray        # [S] the sequences verified
    result: VerifyResult    # greedy verification of those sequences
    z: np.ndarray           # [S, k+1, V] fp64 logits
    abs: np.ndarray         # [S, k+1, V] fp64 sums of |h_j * W[v][j]|


def verify_head_greedy(hidden: np.ndarray, weight: np.ndarray, draft_tokens: np.ndarray, seqs=None,
                       threads: int = 1) -> HeadResult:
    """Greedy verification on the logits of the output projection: hidden
    [B, k+1, H] and weight [V, H] (bf16 bits), draft_tokens [B, k].  ``seqs``
    picks the sequences to verify (all when None); ``threads`` > 1 forms the
    logits of several sequences at once (the C routine runs without the GIL)."""
    B, k1, H = hidden.shape
    seqs = np.arange(B) if seqs is None else np.asarray(seqs, dtype=np.int64)
    draft_tokens = np.asarray(draft_tokens, dtype=np.int32).reshape(B, k1 - 1)
    V = weight.shape[0]
    z = np.empty((len(seqs), k1, V), dtype=np.float64)
    a = np.empty_like(z)

    def one(i):
        z[i], a[i] = head_logits(hidden, weight, int(seqs[i]) * k1, k1)

    if threads > 1:
        from concurrent.futures import ThreadPoolExecutor

        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(one, range(len(seqs))))
    else:
        for i in range(len(seqs)):
            one(i)
    res = verify(z, None, draft_tokens[seqs], None, greedy=True)
    return HeadResult(seqs, res, z, a)
