"""Seeded synthetic inputs for speculative-sampling verification.

This module is the only code shared by the oracle side (``oracle/``, the
tests) and the CUDA side (``bench.py``, the GPU tests).  It holds random
number generation, value recipes and dtype rounding, and none of the
verification arithmetic: no softmax, no top-k, no acceptance rule, no
sampling.  Draft tokens are therefore not produced here; the consumer draws
them from the draft logits with the draft uniforms this module supplies
(the oracle's sampler in tests, the library's ``spec_sample`` in the bench).

Random numbers
--------------
splitmix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014): the state advances by the golden-ratio gamma and
each output is the state passed through the 64-bit finaliser ``mix64``.
It is counter based: output ``n`` of a stream whose state is ``s`` is
``mix64(s + (n + 1) * GAMMA)``, so every element of every tensor is a pure
function of ``(seed, tag, row, column)`` and nothing depends on how the work
is split.

* fp32 uniforms in [0, 1): ``(x >> 40) * 2**-24`` (exact in fp32).
* normals: Box-Muller on the output pair ``(2j, 2j+1)`` of a row stream,
  ``u1 = ((x0 >> 11) + 1) * 2**-53`` in (0, 1], ``u2 = (x1 >> 11) * 2**-53``;
  element ``2j`` takes the cosine branch, ``2j+1`` the sine branch.
* bf16: the fp64 value is rounded to fp32, then to bf16, each round to
  nearest even.

Workloads
---------
The five shapes of the verification benchmark (speculative decoding
entry "推测解码", section "提议与核验的基本步骤": target distributions at
k+1 positions, draft distributions at k positions, k draft tokens):

==========  ====  ==  =======  =====  ===================================
name        B     k   V        dtype  value model
==========  ====  ==  =======  =====  ===================================
tiny        1     4   32       f32    target N(0,2^2), draft = target +
                                      N(0,1^2), T = 1, no top-k
single      1     8   151936   bf16   target N(0,3^2) + 5 spikes of +12 per
                                      row, draft = target + N(0,1.5^2), T=1
batched     64    4   151936   bf16   as "single", draft noise N(0,0.7^2),
                                      T = 0.7, top-k 50 on both sides
greedy      256   8   151936   bf16   target N(0,3^2); 1 % of target rows
                                      get a tie at the top (value 30.0 at
                                      two ids); draft proxy = target +
                                      N(0,2^2), draft token = its argmax
large       512   3   128256   f32    target N(0,4^2), draft = target +
                                      N(0,1^2), T per sequence uniform on
                                      {0.5, 1.0, 1.5}
==========  ====  ==  =======  =====  ===================================
"""
from __future__ import annotations

import dataclasses
import os
from typing import Optional

import numpy as np

__all__ = [
    "GAMMA", "mix64", "splitmix64_stream", "stream_state", "uniform_f32",
    "normals_f64", "f64_to_bf16_bits", "bf16_bits_to_f32", "f64_to_f32",
    "WORKLOADS", "Case", "make_case", "workload_bytes", "Processors", "make_processors",
    "HeadCase", "make_head_case",
]

M64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
_C1 = 0xBF58476D1CE4E5B9
_C2 = 0x94D049BB133111EB
_TAG_MUL = 0xD1B54A32D192ED03

# stream tags: one independent stream family per tensor of a case
TAG_TARGET = 1
TAG_DRAFT_NOISE = 2
TAG_SPIKES = 3
TAG_UNIFORMS = 4
TAG_DRAFT_UNIFORMS = 5
TAG_TEMPERATURE = 6
TAG_TIES = 7
TAG_PROXY_NOISE = 8
TAG_TOP_P = 9
TAG_REP_IDS = 10
TAG_MASK = 11
TAG_HEAD_HIDDEN = 12
TAG_HEAD_WEIGHT = 13

_U = np.uint64


def mix64(z):
    """splitmix64 output finaliser on a uint64 numpy array (wrapping)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> _U(30))) * _U(_C1)
        z = (z ^ (z >> _U(27))) * _U(_C2)
    return z ^ (z >> _U(31))


def splitmix64_stream(state: int, n: int) -> np.ndarray:
    """First ``n`` outputs of splitmix64 started from ``state``."""
    idx = np.arange(1, n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return mix64(_U(state & M64) + idx * _U(GAMMA))


def stream_state(seed: int, tag: int, rows) -> np.ndarray:
    """Per-row stream states for ``(seed, tag)``: mix64(base + (row+1)*GAMMA)."""
    with np.errstate(over="ignore"):
        base = mix64(_U((seed ^ (tag * _TAG_MUL)) & M64))
        r = np.asarray(rows, dtype=np.uint64)
        return mix64(base + (r + _U(1)) * _U(GAMMA))


def _outputs(states: np.ndarray, n: int, offset: int = 0) -> np.ndarray:
    """Outputs ``offset .. offset+n-1`` of each row stream -> [rows, n] uint64."""
    idx = np.arange(offset + 1, offset + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return mix64(states[:, None] + idx[None, :] * _U(GAMMA))


def uniform_f32(seed: int, tag: int, rows: int, n: int) -> np.ndarray:
    """[rows, n] fp32 uniforms in [0, 1), each ``(x >> 40) * 2**-24``."""
    x = _outputs(stream_state(seed, tag, np.arange(rows)), n)
    return ((x >> _U(40)).astype(np.float64) * 2.0 ** -24).astype(np.float32)


def normals_f64(seed: int, tag: int, rows, n: int) -> np.ndarray:
    """[len(rows), n] standard normals by Box-Muller (fp64)."""
    rows = np.atleast_1d(np.asarray(rows))
    npair = (n + 1) // 2
    x = _outputs(stream_state(seed, tag, rows), 2 * npair)
    u1 = ((x[:, 0::2] >> _U(11)).astype(np.float64) + 1.0) * 2.0 ** -53
    u2 = (x[:, 1::2] >> _U(11)).astype(np.float64) * 2.0 ** -53
    r = np.sqrt(-2.0 * np.log(u1))
    out = np.empty((rows.size, 2 * npair), dtype=np.float64)
    out[:, 0::2] = r * np.cos(2.0 * np.pi * u2)
    out[:, 1::2] = r * np.sin(2.0 * np.pi * u2)
    return out[:, :n]


def f64_to_f32(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp64 -> fp32 -> bf16 (each to nearest even); returns uint16 bits."""
    f = f64_to_f32(x)
    b = f.view(np.uint32).astype(np.uint64)
    nan = np.isnan(f)
    b = (b + _U(0x7FFF) + ((b >> _U(16)) & _U(1))) >> _U(16)
    out = b.astype(np.uint16)
    out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bits to fp32 (exact)."""
    return (np.asarray(bits, dtype=np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    k: int
    V: int
    dtype: str            # "bf16" | "f32"
    mode: str             # "stochastic" | "greedy"
    target_sigma: float
    draft_sigma: float    # noise added to the target to make the draft
    spikes: int           # +12 spikes per target row
    temperature: tuple    # one value, or the set drawn per sequence
    top_k: int            # 0 = disabled
    tie_fraction: float = 0.0


WORKLOADS = {
    "tiny": Workload("tiny", 1, 4, 32, "f32", "stochastic", 2.0, 1.0, 0, (1.0,), 0),
    "single": Workload("single", 1, 8, 151936, "bf16", "stochastic", 3.0, 1.5, 5, (1.0,), 0),
    "batched": Workload("batched", 64, 4, 151936, "bf16", "stochastic", 3.0, 0.7, 5, (0.7,), 50),
    "greedy": Workload("greedy", 256, 8, 151936, "bf16", "greedy", 3.0, 2.0, 0, (1.0,), 0, 0.01),
    "large": Workload("large", 512, 3, 128256, "f32", "stochastic", 4.0, 1.0, 0, (0.5, 1.0, 1.5), 0),
}

SPIKE = 12.0
TIE_VALUE = 30.0


@dataclasses.dataclass
class Case:
    """One batch of verification inputs (host numpy arrays).

    ``target`` is [B, k+1, V] and ``draft`` [B, k, V] in the storage dtype
    (uint16 bf16 bits or float32).  ``draft_proxy`` (greedy workloads) is the
    noisy copy of the target whose argmax the proposer emits.  Draft tokens
    are drawn by the consumer from ``draft`` (stochastic) or ``draft_proxy``
    (greedy) with ``draft_uniforms`` [B, k].
    """
    name: str
    seed: int
    B: int
    k: int
    V: int
    dtype: str
    mode: str
    top_k: int
    target: np.ndarray
    draft: Optional[np.ndarray]
    draft_proxy: Optional[np.ndarray]
    uniforms: np.ndarray          # [B, k+1] fp32
    draft_uniforms: np.ndarray    # [B, k]   fp32
    temperature: np.ndarray       # [B]      fp32

    @property
    def elt(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    def logit_bytes(self) -> int:
        return workload_bytes(self.B, self.k, self.V, self.elt, self.mode)


def workload_bytes(B: int, k: int, V: int, elt: int, mode: str) -> int:
    """Logit bytes one verification call reads: (2k+1) rows per sequence
    (stochastic) or k+1 target rows (greedy)."""
    rows = (k + 1) if mode == "greedy" else (2 * k + 1)
    return B * rows * V * elt


def _round(x: np.ndarray, dtype: str) -> np.ndarray:
    return f64_to_bf16_bits(x) if dtype == "bf16" else f64_to_f32(x)


def _distinct_ids(seed: int, tag: int, row: int, count: int, V: int) -> np.ndarray:
    """``count`` distinct ids in [0, V) from the row's stream (first hits)."""
    st = stream_state(seed, tag, np.array([row]))[0]
    out = []
    n = 0
    while len(out) < min(count, V):
        x = int(splitmix64_stream(int(st) + n * GAMMA, 1)[0])
        n += 1
        v = (x >> 11) % V
        if v not in out:
            out.append(v)
    return np.array(out, dtype=np.int64)


def _rows_f64(w: Workload, seed: int, B: int, k: int, V: int, chunk_rows: int = 32):
    """Target values [B, k+1, V] and draft values [B, k, V] in fp64, rounded
    to the storage dtype row block by row block."""
    nt = B * (k + 1)
    target = np.empty((nt, V), dtype=np.uint16 if w.dtype == "bf16" else np.float32)
    draft = np.empty((B * k, V), dtype=target.dtype)
    proxy = np.empty((B * k, V), dtype=target.dtype) if w.mode == "greedy" else None
    tie_u = uniform_f32(seed, TAG_TIES, nt, 4) if w.tie_fraction > 0 else None
    for r0 in range(0, nt, chunk_rows):
        rows = np.arange(r0, min(nt, r0 + chunk_rows))
        t = w.target_sigma * normals_f64(seed, TAG_TARGET, rows, V)
        for j, r in enumerate(rows):
            if w.spikes:
                t[j, _distinct_ids(seed, TAG_SPIKES, int(r), w.spikes, V)] += SPIKE
            if tie_u is not None and tie_u[r, 0] < w.tie_fraction:
                a = int(tie_u[r, 1] * V) % V
                below = tie_u[r, 2] < 0.5
                if below and a == 0:
                    below = False
                if not below and a == V - 1:
                    below = True
                if below:
                    b = int(tie_u[r, 3] * a) % a
                else:
                    b = a + 1 + int(tie_u[r, 3] * (V - 1 - a)) % (V - 1 - a)
                t[j, a] = TIE_VALUE
                t[j, b] = TIE_VALUE
        target[rows] = _round(t, w.dtype)
        # draft rows exist for positions 0..k-1 of each sequence
        seq, pos = np.divmod(rows, k + 1)
        sel = pos < k
        if np.any(sel):
            drows = seq[sel] * k + pos[sel]
            noise = normals_f64(seed, TAG_DRAFT_NOISE if w.mode != "greedy" else TAG_PROXY_NOISE,
                                drows, V)
            d = t[sel] + w.draft_sigma * noise
            if w.mode == "greedy":
                proxy[drows] = _round(d, w.dtype)
            else:
                draft[drows] = _round(d, w.dtype)
    target = target.reshape(B, k + 1, V)
    if w.mode == "greedy":
        return target, None, proxy.reshape(B, k, V)
    return target, draft.reshape(B, k, V), None


def make_case(name: str, seed: int = 0, B: Optional[int] = None, k: Optional[int] = None,
              V: Optional[int] = None, top_k: Optional[int] = None,
              temperature: Optional[tuple] = None, dtype: Optional[str] = None) -> Case:
    """Build the inputs of workload ``name``; ``B``/``k``/``V``/``top_k`` /
    ``temperature`` / ``dtype`` override the workload's own settings (for
    reduced or edge-shape test cases of the same value model)."""
    w = WORKLOADS[name]
    if dtype is not None:
        w = dataclasses.replace(w, dtype=dtype)
    B = w.B if B is None else B
    k = w.k if k is None else k
    V = w.V if V is None else V
    tk = w.top_k if top_k is None else top_k
    temps = w.temperature if temperature is None else tuple(temperature)
    target, draft, proxy = _rows_f64(w, seed, B, k, V)
    uniforms = uniform_f32(seed, TAG_UNIFORMS, B, k + 1)
    duni = uniform_f32(seed, TAG_DRAFT_UNIFORMS, B, k)
    if len(temps) == 1:
        temp = np.full(B, temps[0], dtype=np.float32)
    else:
        pick = uniform_f32(seed, TAG_TEMPERATURE, B, 1)[:, 0]
        temp = np.asarray(temps, dtype=np.float32)[(pick * len(temps)).astype(np.int64) % len(temps)]
    return Case(name=name, seed=seed, B=B, k=k, V=V, dtype=w.dtype, mode=w.mode, top_k=tk,
                target=target, draft=draft, draft_proxy=proxy, uniforms=uniforms,
                draft_uniforms=duni, temperature=temp)


@dataclasses.dataclass
class Processors:
    """Per-sequence inputs of the further logits processors (repetition
    penalty, vocabulary mask, nucleus): arrays only, no processing here."""
    top_p: np.ndarray        # [B] fp32 in (0, 1]
    rep_penalty: np.ndarray  # [B] fp32 > 0
    rep_ids: np.ndarray      # [B, n_rep] int32 token ids (the sequence's history)
    mask: np.ndarray         # [B, ceil(V/32)] uint32, bit v % 32 of word v // 32 = allowed


def make_processors(seed: int, B: int, V: int, top_p=(0.7, 0.95), rep_penalty: float = 1.2,
                    n_rep: int = 32, allowed_fraction: float = 0.5) -> Processors:
    """Seeded processor inputs for B sequences: top_p uniform on the given
    interval (or a fixed value), one penalty for every sequence, n_rep distinct
    history ids per sequence, and a mask allowing each token with probability
    ``allowed_fraction`` (always at least the sequence's first history id)."""
    if isinstance(top_p, tuple):
        lo, hi = top_p
        tp = (lo + (hi - lo) * uniform_f32(seed, TAG_TOP_P, B, 1)[:, 0].astype(np.float64)).astype(np.float32)
    else:
        tp = np.full(B, top_p, dtype=np.float32)
    rp = np.full(B, rep_penalty, dtype=np.float32)
    n_rep = min(n_rep, V)
    ids = np.stack([_distinct_ids(seed, TAG_REP_IDS, b, n_rep, V) for b in range(B)]).astype(np.int32)
    allow = uniform_f32(seed, TAG_MASK, B, V) < np.float32(allowed_fraction)
    if n_rep > 0:
        allow[np.arange(B), ids[:, 0]] = True
    else:
        allow[:, 0] = True
    words = (V + 31) // 32
    bits = np.zeros((B, words * 32), dtype=np.uint64)
    bits[:, :V] = allow
    weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))
    mask = (bits.reshape(B, words, 32) * weights).sum(axis=2).astype(np.uint32)
    return Processors(tp, rp, ids, mask)


@dataclasses.dataclass
class HeadCase:
    """Inputs of the target's output projection: the final hidden state at
    each of the k+1 positions and the projection weight, as bf16 bits."""
    hidden: np.ndarray  # [B, k+1, H] uint16
    weight: np.ndarray  # [V, H] uint16
    B: int
    k: int
    V: int
    H: int


def make_head_case(seed: int, B: int, k: int, V: int, H: int, chunk_rows: int = 2048) -> HeadCase:
    """Hidden states N(0, 1) per element; weight entries uniform on
    [-sqrt(3/H), sqrt(3/H)) (variance 1/H, so each logit has variance about
    the squared norm of the hidden state over H, about 1); both rounded to
    bf16.  The weight is generated in blocks of ``chunk_rows`` rows."""
    hidden = f64_to_bf16_bits(normals_f64(seed, TAG_HEAD_HIDDEN, np.arange(B * (k + 1)), H)).reshape(B, k + 1, H)
    a = np.sqrt(3.0 / H)
    weight = np.empty((V, H), dtype=np.uint16)

    def block(r0):
        rows = np.arange(r0, min(V, r0 + chunk_rows))
        x = _outputs(stream_state(seed, TAG_HEAD_WEIGHT, rows), H)
        u = (x >> _U(40)).astype(np.float64) * 2.0 ** -24
        weight[r0:r0 + rows.size] = f64_to_bf16_bits((2.0 * u - 1.0) * a)

    starts = range(0, V, chunk_rows)
    if len(starts) > 1:
        from concurrent.futures import ThreadPoolExecutor

        with ThreadPoolExecutor(min(16, os.cpu_count() or 1)) as ex:  # the blocks are independent
            list(ex.map(block, starts))
    else:
        for r0 in starts:
            block(r0)
    return HeadCase(hidden, weight, B, k, V, H)
