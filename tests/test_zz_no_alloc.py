"""The allocation-free selection call, vsa_coarse_select_noalloc.

It serves callers that cannot hand the library a workspace (a host framework
whose memory planner owns every device allocation, or a step that must not pay
for cudaMalloc); its scratch is a fixed buffer inside the library. This file
is collected last so that a run stopping at the first failure has already run
every other test. It checks, through the C ABI, that two calls in a row on
different shapes give the same lists and coarse output as vsa_coarse_select
with a caller workspace, and that a shape too large for the buffer is refused.
"""

import numpy as np
import pytest

from block_sparse_video_geometry_b200 import vsa, workloads as W

pytestmark = pytest.mark.gpu


def _run_both(wl):
    import torch
    dev = torch.device("cuda:0")
    lay = vsa.Layout(wl.segments(), wl.seq_len)
    perm, inv, counts, kinds = lay.tables()
    q, k, v, g = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
                  for x in W.make_inputs(wl, inv // vsa.TILE))
    params = vsa.make_params(mode=wl.mode, keep=wl.keep, tau=wl.tau, sink=wl.sink)
    fwd = vsa.Forward(lay, params, wl.B, wl.H, device=dev)        # uploads the layout tables
    nt = lay.info.n_tiles
    # reference: the workspace-taking entry point
    vsa.coarse_select(lay, params, q, k, v, fwd.idx, fwd.cnt, fwd.o_coarse, fwd.ws_select)
    # allocation-free entry point into separate output buffers
    idx = torch.full_like(fwd.idx, -7)
    cnt = torch.full_like(fwd.cnt, -7)
    oc = torch.full_like(fwd.o_coarse, float("nan"))
    vsa.coarse_select_noalloc(lay, params, q, k, v, idx, cnt, oc)
    assert vsa.coarse_select_noalloc_status() == vsa.OK
    want_cnt, got_cnt = fwd.cnt.cpu().numpy(), cnt.cpu().numpy()
    assert np.array_equal(got_cnt, want_cnt)
    wi, gi = fwd.idx.cpu().numpy(), idx.cpu().numpy()
    for b in range(wl.B):
        for h in range(wl.H):
            for t in range(nt):
                n = want_cnt[b, h, t]
                assert np.array_equal(gi[b, h, t, :n], wi[b, h, t, :n])
    assert np.abs(oc.cpu().numpy() - fwd.o_coarse.cpu().numpy()).max() <= 1e-3


def test_noalloc_matches_workspace_call_on_two_calls_in_a_row(cuda_ok):
    # first call: the 17k-token mid workload (top-k 20%); second call: the tiny
    # workload with the adaptive threshold, reusing the buffer the first left dirty
    _run_both(W.WORKLOADS["mid"])
    _run_both(W.WORKLOADS["tiny"].with_(mode=W.MODE_ADAPTIVE, tau=1.0, seed=5))


def test_noalloc_refuses_shapes_beyond_its_buffer(cuda_ok):
    import torch
    # full-size buffers, so that even a wrong size check could not read out of bounds
    wl = W.WORKLOADS["5s"]
    lay = vsa.Layout(wl.segments(), wl.seq_len)
    lay.upload(torch.empty(lay.info.device_bytes, dtype=torch.uint8, device="cuda"))
    params = vsa.make_params(keep=wl.keep)
    q = torch.zeros((wl.B, wl.seq_len, wl.H, 128), dtype=torch.bfloat16, device="cuda")
    nt = lay.info.n_tiles
    idx = torch.empty((wl.B, wl.H, nt, lay.kmax(params)), dtype=torch.int32, device="cuda")
    cnt = torch.empty((wl.B, wl.H, nt), dtype=torch.int32, device="cuda")
    oc = torch.empty((wl.B, wl.H, nt, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(vsa.VSAError) as e:
        vsa.coarse_select_noalloc(lay, params, q, q, q, idx, cnt, oc)
    assert e.value.status == vsa.ERR_UNSUPPORTED
    assert b"33554432" in vsa.lib().vsa_last_error_detail()
