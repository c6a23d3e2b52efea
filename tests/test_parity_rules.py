"""The comparison rules of the GPU parity tests, exercised on the CPU with
oracle-made stand-ins for the GPU's results (no GPU, no CUDA library).

A near-tie row (two candidate tiles whose oracle scores differ by less than
1e-4 at the selection boundary) may legitimately be selected either way; such
a row is accepted only if it differs at the boundary, keeps the top-k length,
and its output equals the oracle run on the list the GPU chose."""

import numpy as np
import pytest

from block_sparse_video_geometry_b200 import workloads as W
from oracle import vsa_oracle as O

import vsa_cases as C


def _head():
    wl = W.WORKLOADS["tiny"]
    lay = C.oracle_layout(wl)
    bits = C.inputs(wl, lay)
    ho = C.HeadOracle(wl, lay, bits, 0, 0, C.params_of(wl))
    return wl, lay, bits, ho


def _lists(ho, kmax):
    nt = len(ho.sel)
    idx = np.full((nt, kmax), -1, dtype=np.int32)
    cnt = np.zeros(nt, dtype=np.int32)
    for qt, s in enumerate(ho.sel):
        idx[qt, : s.size] = s
        cnt[qt] = s.size
    return idx, cnt


def _plant_near_tie(ho, qt):
    """Moves the first unselected tile of row qt to 5e-5 below the k-th score
    and returns the GPU-style list that takes it instead of the k-th tile."""
    row = ho.scores[qt]
    want = ho.sel[qt]
    kth = want[np.argmin(row[want])]
    out = np.setdiff1d(np.arange(row.size), want)[0]
    row[out] = row[kth] - 5e-5
    return np.sort(np.append(np.setdiff1d(want, [kth]), out)).astype(np.int32)


def test_near_tie_row_is_checked_on_the_gpu_list():
    wl, lay, bits, ho = _head()
    kmax = max(s.size for s in ho.sel)
    idx, cnt = _lists(ho, kmax)
    qt = lay.n_cond_tiles + 2
    alt = _plant_near_tie(ho, qt)
    idx[qt, : alt.size] = alt
    near = C.compare_selection(ho, idx, cnt)
    assert set(near) == {qt} and np.array_equal(near[qt], alt)
    # stand-in GPU output: the oracle on the GPU's lists
    out = np.zeros((1, lay.seq_len, wl.H, O.HEAD_DIM))
    for t in range(lay.n_tiles):
        toks, _, o = ho.tile_out(t, near.get(t))
        out[0, toks, 0] = o
    res = {"out": out}
    C.compare_outputs(ho, res, 0, 0, range(lay.n_tiles), near_tie=near)
    # the row's output on the GPU list differs from the oracle's own row
    toks, _, own = ho.tile_out(qt)
    assert np.abs(out[0, toks, 0] - own).max() > 0


def test_difference_away_from_the_boundary_fails():
    wl, lay, bits, ho = _head()
    kmax = max(s.size for s in ho.sel)
    idx, cnt = _lists(ho, kmax)
    qt = lay.n_cond_tiles + 1
    row, want = ho.scores[qt], ho.sel[qt]
    best = want[np.argmax(row[want])]                  # the row's top tile, far from the boundary
    out = np.setdiff1d(np.arange(row.size), want)[0]
    idx[qt, : want.size] = np.sort(np.append(np.setdiff1d(want, [best]), out))
    with pytest.raises(AssertionError):
        C.compare_selection(ho, idx, cnt)


def test_topk_list_of_wrong_length_fails_even_at_a_near_tie():
    wl, lay, bits, ho = _head()
    kmax = max(s.size for s in ho.sel) + 1
    idx, cnt = _lists(ho, kmax)
    qt = lay.n_cond_tiles + 3
    alt = _plant_near_tie(ho, qt)
    extra = np.setdiff1d(np.arange(ho.scores.shape[1]), alt)[0]
    longer = np.sort(np.append(alt, extra)).astype(np.int32)
    idx[qt, : longer.size] = longer
    cnt[qt] = longer.size
    with pytest.raises(AssertionError):
        C.compare_selection(ho, idx, cnt)


def test_list_validity_check_catches_bad_lists():
    wl, lay, bits, ho = _head()
    kmax = max(s.size for s in ho.sel)
    idx, cnt = _lists(ho, kmax)
    res = {"idx": idx[None, None], "cnt": cnt[None, None], "kmax": kmax}
    C.check_lists_valid(res, lay)
    bad = idx.copy()
    bad[4, :2] = bad[4, 1::-1]                         # descending pair
    with pytest.raises(AssertionError):
        C.check_lists_valid({"idx": bad[None, None], "cnt": cnt[None, None], "kmax": kmax}, lay)
    bad = idx.copy()
    bad[5, 0] = lay.n_video_tiles                      # out of range
    with pytest.raises(AssertionError):
        C.check_lists_valid({"idx": bad[None, None], "cnt": cnt[None, None], "kmax": kmax}, lay)
