"""GPU checks of the tensor-core selection (vsa_coarse_select with the mean
coarse branch) beyond the random-input parity tests: query tiles whose scores
tie exactly (the boundary ranking, the exact fallback passes and the
lower-ordinal rule, compared with the oracle without any near-tie allowance),
the failure path of its bounded waits, and bit-identical reruns."""

import numpy as np
import pytest

from block_sparse_video_geometry_b200 import vsa, workloads as W
from oracle import vsa_oracle as O

import vsa_cases as C

pytestmark = pytest.mark.gpu


def tied_inputs(wl, lay, n_distinct, seed=7):
    """The seeded inputs with the K of every token of video tile t replaced by
    seeded vector (t - n_cond) % n_distinct of its (batch, head): the video
    tiles' mean-pooled K takes n_distinct values, so every query tile's scores
    against the video tiles tie in n_distinct groups (exactly, in any
    precision)."""
    q, k, v, g = C.inputs(wl, lay)
    k = k.copy()
    tile = lay.inv // O.TILE
    video = np.nonzero(tile >= lay.n_cond_tiles)[0]
    grp = (tile[video] - lay.n_cond_tiles) % n_distinct
    rng = np.random.default_rng(seed)
    vecs = W.f32_to_bf16_bits(rng.standard_normal((n_distinct, wl.B, wl.H, 128)).astype(np.float32))
    k[:, video] = np.moveaxis(vecs[grp], 0, 1)
    return q, k, v, g


def select_only(wl, bits, prm):
    import torch
    dev = torch.device("cuda:0")
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).to(dev)
    q, k, v, _ = (t(x) for x in bits)
    lay = vsa.Layout(wl.segments(), wl.seq_len)
    p = vsa.make_params(**prm)
    fwd = vsa.Forward(lay, p, wl.B, wl.H, device=dev)
    vsa.coarse_select(lay, p, q, k, v, fwd.idx, fwd.cnt, fwd.o_coarse, fwd.ws_select)
    assert vsa.coarse_select_status(fwd.ws_select) == vsa.OK
    return fwd.idx.cpu().numpy(), fwd.cnt.cpu().numpy(), fwd.o_coarse.cpu().numpy()


@pytest.mark.parametrize("n_distinct", [1, 3, 8], ids=["all_equal", "3_groups_fallback", "8_groups_ranked"])
def test_exact_ties_take_the_lower_ordinals(cuda_ok, n_distinct):
    """mid: 256 candidate tiles, k = 26. One group: every score of a row is
    equal, the list is 0..25. Three groups of ~85: the boundary bin holds more
    members than the kernel ranks directly, so the exact radix fallback runs.
    Eight groups of 32: ranked directly. Lists must equal the oracle's exactly."""
    wl = W.WORKLOADS["mid"].with_(keep=0.1)
    lay = C.oracle_layout(wl)
    bits = tied_inputs(wl, lay, n_distinct)
    prm = C.params_of(wl)
    idx, cnt, oc = select_only(wl, bits, prm)
    for h in (0, 11, 23):
        ho = C.HeadOracle(wl, lay, bits, 0, h, prm)
        for qt, want in enumerate(ho.sel):
            got = idx[0, h, qt, : cnt[0, h, qt]]
            assert np.array_equal(got, want), "head %d query tile %d: %s vs %s" % (h, qt, got[:8], want[:8])
        assert np.abs(oc[0, h] - ho.o_coarse).max() <= 1e-3
        if n_distinct == 1:
            assert all(np.array_equal(s, np.arange(len(s))) for s in ho.sel)


def test_exact_ties_sink_off(cuda_ok):
    """Sink off: the conditioning tiles are candidates too and keep their
    own scores; the video tiles tie in 3 groups."""
    wl = W.WORKLOADS["mid"].with_(keep=0.2)
    lay = C.oracle_layout(wl)
    bits = tied_inputs(wl, lay, 3, seed=9)
    prm = C.params_of(wl, sink=O.SINK_OFF)
    idx, cnt, oc = select_only(wl, bits, prm)
    for h in (2, 17):
        ho = C.HeadOracle(wl, lay, bits, 0, h, prm)
        near = C.compare_selection(ho, idx[0, h], cnt[0, h])   # conditioning scores are generic: near-ties allowed
        for qt, want in enumerate(ho.sel):
            got = idx[0, h, qt, : cnt[0, h, qt]]
            assert qt in near or np.array_equal(got, want)


def _tiny_inputs():
    import torch
    wl = W.WORKLOADS["tiny"]
    lay = vsa.Layout(wl.segments(), wl.seq_len)
    perm, inv, counts, kinds = lay.tables()
    bits = W.make_inputs(wl, inv // vsa.TILE)
    dev = torch.device("cuda:0")
    q, k, v, g = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev) for x in bits)
    return wl, lay, q, k, v


@pytest.mark.parametrize("mode", [vsa.SELECT_TOPK, vsa.SELECT_ADAPTIVE], ids=["topk", "adaptive"])
def test_select_wait_timeout_is_reported_and_recoverable(cuda_ok, mode):
    import torch
    wl, lay, q, k, v = _tiny_inputs()
    p = vsa.make_params(mode=mode, keep=wl.keep, tau=1.0, sink=wl.sink)
    fwd = vsa.Forward(lay, p, wl.B, wl.H, device=q.device)
    vsa.coarse_select(lay, p, q, k, v, fwd.idx, fwd.cnt, fwd.o_coarse, fwd.ws_select)
    assert vsa.coarse_select_status(fwd.ws_select) == vsa.OK
    idx0, cnt0, oc0 = fwd.idx.clone(), fwd.cnt.clone(), fwd.o_coarse.clone()
    vsa.debug_inject_select_wait_timeout(20_000_000)      # 20 ms
    try:
        vsa.coarse_select(lay, p, q, k, v, fwd.idx, fwd.cnt, fwd.o_coarse, fwd.ws_select)
        st = vsa.coarse_select_status(fwd.ws_select)
    finally:
        vsa.debug_inject_select_wait_timeout(0)
    assert st == vsa.ERR_TIMEOUT
    assert vsa.coarse_select_failed_calls(fwd.ws_select) == 1
    # the context is still usable and the next call is correct; the failure stays counted
    vsa.coarse_select(lay, p, q, k, v, fwd.idx, fwd.cnt, fwd.o_coarse, fwd.ws_select)
    assert vsa.coarse_select_status(fwd.ws_select) == vsa.OK
    assert vsa.coarse_select_failed_calls(fwd.ws_select) == 1
    assert torch.equal(cnt0, fwd.cnt) and torch.equal(oc0.view(torch.int32), fwd.o_coarse.view(torch.int32))
    n = cnt0.cpu().numpy()
    a, b = idx0.cpu().numpy(), fwd.idx.cpu().numpy()
    live = np.arange(a.shape[-1])[None, None, None, :] < n[..., None]
    assert np.array_equal(np.where(live, a, 0), np.where(live, b, 0))


@pytest.mark.parametrize("mode", [vsa.SELECT_TOPK, vsa.SELECT_ADAPTIVE], ids=["topk", "adaptive"])
def test_select_reruns_are_bit_identical(cuda_ok, mode):
    import torch
    wl = W.WORKLOADS["mid"]
    lay = vsa.Layout(wl.segments(), wl.seq_len)
    perm, inv, counts, kinds = lay.tables()
    dev = torch.device("cuda:0")
    q, k, v, g = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
                  for x in W.make_inputs(wl, inv // vsa.TILE))
    p = vsa.make_params(mode=mode, keep=wl.keep, tau=1.0, sink=wl.sink)
    fwd = vsa.Forward(lay, p, wl.B, wl.H, device=dev)
    runs = []
    for _ in range(2):
        fwd.idx.fill_(-7)
        vsa.coarse_select(lay, p, q, k, v, fwd.idx, fwd.cnt, fwd.o_coarse, fwd.ws_select)
        assert vsa.coarse_select_status(fwd.ws_select) == vsa.OK
        runs.append((fwd.idx.clone(), fwd.cnt.clone(), fwd.o_coarse.clone()))
    (i1, c1, o1), (i2, c2, o2) = runs
    assert torch.equal(c1, c2) and torch.equal(i1, i2)
    assert torch.equal(o1.view(torch.int32), o2.view(torch.int32))
