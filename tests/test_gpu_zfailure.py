"""Failure handling on the GPU without a GPU fault: a bounded kernel wait that
runs out is reported as a status and leaves the CUDA context usable, and reruns
are bit-identical."""
import time

import numpy as np
import pytest

from block_sparse_video_geometry_b200 import vsa, workloads as W

pytestmark = pytest.mark.gpu


def _inputs(wl):
    import torch
    lay = vsa.Layout(wl.segments(), wl.seq_len)
    perm, inv, cnt, kind = lay.tables()
    bits = W.make_inputs(wl, inv // vsa.TILE)
    dev = torch.device("cuda:0")
    q, k, v, g = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev) for x in bits)
    return lay, (q, k, v, g), bits


def test_injected_wait_timeout_is_reported_and_recoverable(cuda_ok):
    import torch
    wl = W.WORKLOADS["tiny"]
    lay, (q, k, v, g), bits = _inputs(wl)
    p = vsa.make_params(keep=wl.keep, sink=wl.sink)
    fwd = vsa.Forward(lay, p, wl.B, wl.H, device=q.device)
    vsa.debug_inject_wait_timeout(20_000_000)      # 20 ms
    try:
        t0 = time.time()
        fwd(q, k, v, g)
        st = vsa.sparse_attn_status(fwd.ws_attn)
        elapsed = time.time() - t0
    finally:
        vsa.debug_inject_wait_timeout(0)
    assert st == vsa.ERR_TIMEOUT
    assert elapsed < 5.0
    assert vsa.sparse_attn_failed_calls(fwd.ws_attn) == 1
    # the context is still usable and the next call is correct; the failure
    # stays counted after a good call overwrote the per-call status
    out = fwd(q, k, v, g)
    assert vsa.sparse_attn_status(fwd.ws_attn) == vsa.OK
    assert vsa.sparse_attn_failed_calls(fwd.ws_attn) == 1
    assert torch.isfinite(out).all()


def test_reruns_are_bit_identical(cuda_ok):
    import torch
    wl = W.WORKLOADS["mid"]
    lay, (q, k, v, g), bits = _inputs(wl)
    p = vsa.make_params(keep=wl.keep, sink=wl.sink)
    fwd = vsa.Forward(lay, p, wl.B, wl.H, device=q.device)
    out1 = fwd(q, k, v, g).clone()
    idx1, cnt1 = fwd.idx.clone(), fwd.cnt.clone()
    out2 = fwd(q, k, v, g)
    assert vsa.sparse_attn_status(fwd.ws_attn) == vsa.OK
    assert torch.equal(cnt1, fwd.cnt) and torch.equal(idx1, fwd.idx)
    assert torch.equal(out1.view(torch.int32), out2.view(torch.int32))
