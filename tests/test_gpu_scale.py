"""GPU parity at the full 1344x768 shapes, in the launch configuration the
benchmark times (fp32 output, one call of each entry point). The oracle checks
whole selection matrices of sampled heads and the outputs of sampled query
tiles (conditioning tiles, first/last video tiles, ragged tiles, random ones)."""

import numpy as np
import pytest

from block_sparse_video_geometry_b200 import vsa, workloads as W
from oracle import vsa_oracle as O

import vsa_cases as C

pytestmark = pytest.mark.gpu


def sample_tiles(lay, rng, n_random=6):
    nc, nt = lay.n_cond_tiles, lay.n_tiles
    fixed = {0, nc - 1, nc, nc + 1, nt - 2, nt - 1} if nc else {0, 1, nt - 2, nt - 1}
    partial = [t for t in range(nc, nt) if (lay.perm[t] >= 0).sum() < O.TILE]
    if partial:
        fixed |= {partial[0], partial[-1]}
    return sorted(fixed | set(rng.choice(nt, n_random, replace=False).tolist()))


def run_case(wl, heads, n_random=6, g_zero=False, channel_gate=False, **prm_over):
    lay = C.oracle_layout(wl)
    q, k, v, g = C.inputs(wl, lay, channel_gate)
    if g_zero:
        g = np.zeros_like(g)
    prm = C.params_of(wl, **prm_over)
    res = C.gpu_forward(wl, (q, k, v, g), prm)
    assert res["status"] == vsa.OK
    rng = np.random.default_rng(1234)
    kept = []
    for h in heads:
        ho = C.HeadOracle(wl, lay, (q, k, v, g), 0, h, prm)
        assert np.abs(res["pooled"][1, 0, h] - ho.kbar).max() <= 1e-4
        assert np.abs(res["o_coarse"][0, h] - ho.o_coarse).max() <= 1e-3
        near = C.compare_selection(ho, res["idx"][0, h], res["cnt"][0, h])
        assert len(near) <= lay.n_tiles // 20
        C.note_near_ties(len(near))
        tiles = sorted(set(sample_tiles(lay, rng, n_random)) | set(near))
        C.compare_outputs(ho, res, 0, h, tiles, near_tie=near)
        kept.append(res["cnt"][0, h].mean() / lay.n_video_tiles)
    # every list of every head is valid (ascending, in range, 1 <= cnt <= kmax)
    C.check_lists_valid(res, lay, prm["sink"])
    return lay, res, kept


def test_5s_topk_10pct(cuda_ok):
    lay, res, kept = run_case(W.WORKLOADS["5s"], heads=(0, 11, 23))
    assert lay.n_video_tiles == 2016 and res["kmax"] == 202


def test_10s_ragged_rows_dense(cuda_ok):
    lay, res, kept = run_case(W.WORKLOADS["10s"], heads=(0, 23), n_random=4)
    assert lay.n_video_tiles == 4032 and res["kmax"] == 404


def test_5s_sink_off(cuda_ok):
    """sink_conditioning off at full size: every tile is a candidate."""
    lay, res, kept = run_case(W.WORKLOADS["5s"], heads=(5,), n_random=4, sink=O.SINK_OFF)
    assert res["kmax"] == O.topk_count(0.1, lay.n_tiles) == 209


def test_5s_spark_reweight_channel_gate(cuda_ok):
    """Spark-Reweight compressed branch and a per-channel gate at full size."""
    run_case(W.WORKLOADS["5s"], heads=(7,), n_random=4, channel_gate=True, coarse=O.COARSE_REWEIGHT)


@pytest.mark.parametrize("tau", [1.0, 1.5, 2.0])
def test_5s_adaptive_tau(cuda_ok, tau):
    lay, res, kept = run_case(W.WORKLOADS["5s_adaptive"].with_(tau=tau), heads=(0, 13), n_random=4)
    # kept fraction near the Gaussian tail above mean + tau * std
    import math
    tail = 0.5 * math.erfc(tau / math.sqrt(2))
    assert abs(float(np.mean(kept)) - tail) < 0.05


def test_5s_keep_all_equals_dense(cuda_ok):
    wl = W.WORKLOADS["5s"].with_(keep=1.0)
    lay = C.oracle_layout(wl)
    q, k, v, g = C.inputs(wl, lay)
    res = C.gpu_forward(wl, (q, k, v, np.zeros_like(g)), C.params_of(wl, keep=1.0))
    f = O.bf16_bits_to_f64
    rng = np.random.default_rng(7)
    for h in (0, 19):
        kk, vv = f(k[0, :, h]), f(v[0, :, h])
        for qt in rng.choice(lay.n_tiles, 3, replace=False):
            toks = lay.tile_tokens(int(qt))
            dense = O.softmax_attention(f(q[0, toks, h]), kk, vv, O.default_scale())
            err = np.abs(res["out"][0, toks, h] - dense)
            assert err.max() <= C.OUT_MAX_ABS and err.mean() <= C.OUT_MEAN_ABS


def test_5s_extra_tokens(cuda_ok):
    """extra_tokens at full size: the chosen sets of sampled query tiles against
    the oracle's ranking over their ~116k candidate tokens, and their outputs."""
    wl = W.WORKLOADS["5s"]
    E = 16
    lay = C.oracle_layout(wl)
    q, k, v, g = C.inputs(wl, lay)
    prm = C.params_of(wl, extra_tokens=E)
    res = C.gpu_forward(wl, (q, k, v, g), prm)
    assert res["status"] == vsa.OK and res["extra_status"] == vsa.OK
    assert res["extra_cnt"].min() == E and res["extra_cnt"].max() == E
    rng = np.random.default_rng(99)
    for h in (2, 21):
        ho = C.HeadOracle(wl, lay, (q, k, v, g), 0, h, prm)
        near = C.compare_selection(ho, res["idx"][0, h], res["cnt"][0, h])
        tiles = sorted(set(sample_tiles(lay, rng, 4)) | set(list(near)[:4]))
        near_x = C.compare_extra(ho, res["extra_idx"][0, h], res["extra_cnt"][0, h], tiles, near)
        C.note_near_ties(len(near_x))
        gpu_extra = {qt: res["extra_idx"][0, h, qt, :E] for qt in tiles}
        C.compare_outputs(ho, res, 0, h, tiles, near_tie=near, extra=gpu_extra)


def test_10s_extra_tokens_e64(cuda_ok):
    """extra_tokens on the 10 s clip with E = 64: the bitmap of ~3.8k candidate
    tiles and two 64-entry top-E lists leave shared memory for a single key
    tile pair stage, the smallest pipeline the kernel runs."""
    wl = W.WORKLOADS["10s"]
    E = 64
    lay = C.oracle_layout(wl)
    q, k, v, g = C.inputs(wl, lay)
    prm = C.params_of(wl, extra_tokens=E)
    assert prm["sink"] == O.SINK_EXACT_KV_AND_ROWS   # dense conditioning rows take no extra tokens
    res = C.gpu_forward(wl, (q, k, v, g), prm)
    assert res["status"] == vsa.OK and res["extra_status"] == vsa.OK
    nc = lay.n_cond_tiles
    assert np.all(res["extra_cnt"][:, :, :nc] == 0)
    assert res["extra_cnt"][:, :, nc:].min() == E and res["extra_cnt"][:, :, nc:].max() == E
    rng = np.random.default_rng(5)
    h = 11
    ho = C.HeadOracle(wl, lay, (q, k, v, g), 0, h, prm)
    near = C.compare_selection(ho, res["idx"][0, h], res["cnt"][0, h])
    tiles = sorted(set(sample_tiles(lay, rng, 3)) | set(list(near)[:2]))
    near_x = C.compare_extra(ho, res["extra_idx"][0, h], res["extra_cnt"][0, h], tiles, near)
    C.note_near_ties(len(near_x))
    gpu_extra = {qt: res["extra_idx"][0, h, qt, :E] for qt in tiles}
    C.compare_outputs(ho, res, 0, h, tiles, near_tie=near, extra=gpu_extra)
