"""GPU parity of the backward pass (vsa_sparse_attn_bwd) against the fp64
oracle's gradients (autograd through the oracle's torch restatement of the
forward) with the same block selection.

Tolerance: the fine branch's tensor-core products take P and dS in bf16 (as
the forward takes P), a relative rounding of 2^-9 per term, so each gradient
is held to max-abs error <= 1e-2 * max|ref| + 1e-3 and mean-abs error <=
1e-3 * max|ref| + 1e-4 (its own scale; dg and the coarse branch run in fp32).
"""

import numpy as np
import pytest

from block_sparse_video_geometry_b200 import vsa, workloads as W
from oracle import vsa_oracle as O

import vsa_cases as C
from test_gpu_parity import EDGE_WORKLOADS

pytestmark = pytest.mark.gpu

SMALL = W.Workload("small", B=1, H=3, cond=((W.SEG_TEXT, 96), (W.SEG_REF_IMAGE, 64)), grid=(8, 16, 16),
                   keep=0.25, seed=21)
# eleven conditioning tiles (one partial): the shared key tiles of dq_pair_kernel
# and dkv_pair_kernel run past their four copy stages, with an odd last pair
PREFIX_HEAVY = W.Workload("prefix_heavy", B=1, H=2, cond=((W.SEG_TEXT, 500), (W.SEG_REF_IMAGE, 192)),
                          grid=(8, 16, 16), keep=0.25, seed=23)


def oracle_grads(q, k, v, g, dout, lay, p, sel):
    import torch
    from oracle import vsa_backward_oracle as BO
    t = [torch.tensor(np.asarray(x, dtype=np.float64), requires_grad=True) for x in (q, k, v, g)]
    out = BO.forward_torch(*t, lay, p, sel)
    (out * torch.as_tensor(np.asarray(dout, dtype=np.float64))).sum().backward()
    return [x.grad.numpy() for x in t]


def check_grad(got, want, name):
    scale = float(np.abs(want).max())
    err = np.abs(got - want)
    assert err.max() <= 1e-2 * scale + 1e-3, "%s: max-abs %.3g (scale %.3g)" % (name, err.max(), scale)
    assert err.mean() <= 1e-3 * scale + 1e-4, "%s: mean-abs %.3g (scale %.3g)" % (name, err.mean(), scale)


def bwd_check(wl, channel_gate=False, **prm_over):
    import torch
    lay = C.oracle_layout(wl)
    bits = C.inputs(wl, lay, channel_gate)
    q, k, v, g = bits
    prm = C.params_of(wl, **prm_over)
    dev = torch.device("cuda:0")
    t = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
    tq, tk, tv, tg = t(q), t(k), t(v), t(g)
    rng = np.random.default_rng(1000 + wl.seed)
    dout = W.f32_to_bf16_bits(rng.standard_normal(q.shape).astype(np.float32))
    tdo = t(dout)
    layout = vsa.Layout(wl.segments(), wl.seq_len)
    p = vsa.make_params(**prm)
    fwd = vsa.Forward(layout, p, wl.B, wl.H, device=dev)
    vsa.coarse_select(layout, p, tq, tk, tv, fwd.idx, fwd.cnt, fwd.o_coarse, fwd.ws_select)
    grads = [torch.full(q.shape, float("nan"), dtype=torch.float32, device=dev) for _ in range(3)]
    dg = torch.full(g.shape, float("nan"), dtype=torch.float32, device=dev)
    ws = torch.empty(layout.sparse_attn_bwd_workspace_size(wl.B, wl.H, p), dtype=torch.uint8, device=dev)
    vsa.sparse_attn_bwd(layout, p, tq, tk, tv, tg, fwd.idx, fwd.cnt, fwd.kmax, fwd.o_coarse, tdo, *grads, dg, ws)
    assert vsa.sparse_attn_bwd_status(ws) == vsa.OK
    got = [x.cpu().numpy() for x in grads] + [dg.cpu().numpy()]
    idx, cnt = fwd.idx.cpu().numpy(), fwd.cnt.cpu().numpy()
    f = O.bf16_bits_to_f64
    for b in range(wl.B):
        for h in range(wl.H):
            ho = C.HeadOracle(wl, lay, bits, b, h, prm)
            near = C.compare_selection(ho, idx[b, h], cnt[b, h])
            C.note_near_ties(len(near))
            sel = [near.get(qt, s) for qt, s in enumerate(ho.sel)]
            want = oracle_grads(f(q[b, :, h]), f(k[b, :, h]), f(v[b, :, h]), f(g[b, :, h]), f(dout[b, :, h]),
                                lay, ho.p, sel)
            for name, gg, ww in zip(("dq", "dk", "dv", "dg"), got, want):
                check_grad(gg[b, :, h], ww, "%s b%d h%d" % (name, b, h))


@pytest.mark.parametrize("sink", [O.SINK_EXACT_KV, O.SINK_EXACT_KV_AND_ROWS, O.SINK_OFF])
def test_tiny_backward(cuda_ok, sink):
    bwd_check(W.WORKLOADS["tiny"], sink=sink)


def test_tiny_backward_channel_gate(cuda_ok):
    bwd_check(W.WORKLOADS["tiny"], channel_gate=True)


def test_tiny_backward_adaptive(cuda_ok):
    bwd_check(W.WORKLOADS["tiny"].with_(mode=O.MODE_ADAPTIVE, tau=1.0))


@pytest.mark.parametrize("wl", [EDGE_WORKLOADS[0], EDGE_WORKLOADS[1]], ids=["ragged_b2", "video_only"])
def test_edge_backward(cuda_ok, wl):
    bwd_check(wl)


@pytest.mark.parametrize("sink", [O.SINK_EXACT_KV, O.SINK_EXACT_KV_AND_ROWS])
def test_small_multitile_backward(cuda_ok, sink):
    bwd_check(SMALL, sink=sink)


@pytest.mark.parametrize("sink", [O.SINK_EXACT_KV, O.SINK_EXACT_KV_AND_ROWS])
def test_prefix_heavy_backward(cuda_ok, sink):
    bwd_check(PREFIX_HEAVY, sink=sink)


def test_backward_refuses_what_it_does_not_differentiate(cuda_ok):
    import torch
    wl = W.WORKLOADS["tiny"]
    layout = vsa.Layout(wl.segments(), wl.seq_len)
    x = torch.zeros((1, wl.seq_len, wl.H, 128), dtype=torch.bfloat16, device="cuda")
    f = torch.zeros((1, wl.seq_len, wl.H, 128), dtype=torch.float32, device="cuda")
    gate = torch.zeros((1, wl.seq_len, wl.H), dtype=torch.bfloat16, device="cuda")
    dg = torch.zeros((1, wl.seq_len, wl.H), dtype=torch.float32, device="cuda")
    for p in (vsa.make_params(keep=0.5, coarse=vsa.COARSE_REWEIGHT), vsa.make_params(keep=0.5, extra_tokens=4)):
        fwd = vsa.Forward(layout, p, 1, wl.H, device="cuda")
        ws = torch.empty(layout.sparse_attn_bwd_workspace_size(1, wl.H, p), dtype=torch.uint8, device="cuda")
        with pytest.raises(vsa.VSAError) as e:
            vsa.sparse_attn_bwd(layout, p, x, x, x, gate, fwd.idx, fwd.cnt, fwd.kmax, fwd.o_coarse, x, f, f.clone(),
                                f.clone(), dg, ws)
        assert e.value.status == vsa.ERR_UNSUPPORTED
