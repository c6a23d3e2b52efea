"""GPU parity of extra_tokens (vsa_extra_tokens_select + the extra key step of
vsa_sparse_attn_fwd) against the fp64 oracle: the chosen token sets equal the
oracle's except at near-ties of their scores (then they are checked on the
GPU's set), and the outputs match with the GPU's sets."""

import numpy as np
import pytest

from block_sparse_video_geometry_b200 import vsa, workloads as W
from oracle import vsa_oracle as O

import vsa_cases as C
from test_gpu_parity import EDGE_WORKLOADS

pytestmark = pytest.mark.gpu


def extra_check(wl, E, heads=None, out_tiles=None, **prm_over):
    lay = C.oracle_layout(wl)
    bits = C.inputs(wl, lay)
    prm = C.params_of(wl, extra_tokens=E, **prm_over)
    res = C.gpu_forward(wl, bits, prm)
    assert res["status"] == vsa.OK and res["extra_status"] == vsa.OK
    C.check_lists_valid(res, lay, prm["sink"])
    assert res["extra_cnt"].min() >= 0 and res["extra_cnt"].max() <= E
    counts = []
    for b in range(wl.B):
        for h in (range(wl.H) if heads is None else heads):
            ho = C.HeadOracle(wl, lay, bits, b, h, prm)
            near = C.compare_selection(ho, res["idx"][b, h], res["cnt"][b, h])
            tiles = sorted(set(range(lay.n_tiles) if out_tiles is None else out_tiles(lay)) | set(near))
            near_x = C.compare_extra(ho, res["extra_idx"][b, h], res["extra_cnt"][b, h], tiles, near)
            C.note_near_ties(len(near) + len(near_x))
            gpu_extra = {qt: res["extra_idx"][b, h, qt, : res["extra_cnt"][b, h, qt]] for qt in tiles}
            C.compare_outputs(ho, res, b, h, tiles, near_tie=near, extra=gpu_extra)
            counts.append(res["extra_cnt"][b, h])
    return res, np.concatenate(counts)


@pytest.mark.parametrize("E", [1, 5, 64])
def test_tiny_extra_tokens(cuda_ok, E):
    res, counts = extra_check(W.WORKLOADS["tiny"], E)
    assert np.all(counts == E)            # 4 unselected tiles: 256 candidates per query tile


def test_tiny_extra_tokens_take_every_candidate(cuda_ok):
    """keep 7/8: one unselected video tile of 64 tokens, E = 64 takes them all,
    so every video tile is attended exactly."""
    res, counts = extra_check(W.WORKLOADS["tiny"], 64, keep=0.875)
    assert np.all(counts == 64)


@pytest.mark.parametrize("sink", [O.SINK_EXACT_KV_AND_ROWS, O.SINK_OFF])
def test_tiny_extra_tokens_sink_modes(cuda_ok, sink):
    res, counts = extra_check(W.WORKLOADS["tiny"], 8, sink=sink)
    if sink == O.SINK_EXACT_KV_AND_ROWS:      # dense conditioning rows take no extra tokens
        assert np.all(res["extra_cnt"][:, :, :3] == 0)


def test_tiny_extra_tokens_adaptive(cuda_ok):
    extra_check(W.WORKLOADS["tiny"].with_(mode=O.MODE_ADAPTIVE, tau=1.0), 8)


@pytest.mark.parametrize("wl,E", [(EDGE_WORKLOADS[0], 16), (EDGE_WORKLOADS[1], 8), (EDGE_WORKLOADS[3], 3)],
                         ids=["ragged_b2", "video_only", "one_tile_no_candidates"])
def test_edge_extra_tokens(cuda_ok, wl, E):
    res, counts = extra_check(wl, E)
    if wl.name == "one_tile":                 # keep 100% of one video tile: nothing left to add
        assert np.all(counts == 0)


def test_mid_extra_tokens_two_heads(cuda_ok):
    wl = W.WORKLOADS["mid"].with_(H=4)
    extra_check(wl, 32, heads=(0, 3), out_tiles=lambda lay: range(2, lay.n_tiles, 13))
