"""Seeded processor inputs (``workloads.make_processors``) and the parity
helper for near-tie nucleus cuts; CPU only."""
import numpy as np

import oracle
import workloads
from paritylib import nucleus_near_cut


def test_processor_inputs_are_seeded_and_well_formed():
    a = workloads.make_processors(5, 6, 1000)
    b = workloads.make_processors(5, 6, 1000)
    c = workloads.make_processors(6, 6, 1000)
    for f in ("top_p", "rep_penalty", "rep_ids", "mask"):
        assert np.array_equal(getattr(a, f), getattr(b, f))
    assert not np.array_equal(a.mask, c.mask)
    assert a.top_p.dtype == np.float32 and np.all((a.top_p >= 0.7) & (a.top_p <= 0.95))
    assert a.rep_ids.shape == (6, 32) and a.rep_ids.dtype == np.int32
    for row in a.rep_ids:
        assert len(set(row.tolist())) == row.size and row.min() >= 0 and row.max() < 1000
    assert a.mask.shape == (6, (1000 + 31) // 32) and a.mask.dtype == np.uint32


def test_mask_words_match_the_allow_rule():
    B, V = 3, 77
    pr = workloads.make_processors(9, B, V, allowed_fraction=0.4)
    allow = workloads.uniform_f32(9, workloads.TAG_MASK, B, V) < np.float32(0.4)
    allow[np.arange(B), pr.rep_ids[:, 0]] = True
    for b in range(B):
        bits = [(int(pr.mask[b, v // 32]) >> (v % 32)) & 1 for v in range(V)]
        assert bits == allow[b].astype(int).tolist()
        tail = [(int(pr.mask[b, v // 32]) >> (v % 32)) & 1 for v in range(V, 32 * pr.mask.shape[1])]
        assert not any(tail)  # padding bits past V stay clear
        # the oracle's allow_mask builds the same words from the allowed ids
        assert np.array_equal(oracle.allow_mask(V, np.flatnonzero(allow[b])), pr.mask[b])


def test_nucleus_near_cut_flags_ties_only():
    p = np.array([0.5, 0.25, 0.125, 0.125])
    assert nucleus_near_cut(p, 0.75)          # the running sum hits top_p exactly
    assert nucleus_near_cut(p, 0.750004)      # within 1e-5 of a step
    assert not nucleus_near_cut(p, 0.7)
    assert not nucleus_near_cut(p, 1.0)
    assert nucleus_near_cut(p, 0.5 + 5e-6)    # just past the first step
