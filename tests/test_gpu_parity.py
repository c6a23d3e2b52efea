"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs. Tolerances are defined in vsa_cases."""

import ctypes
import os

import numpy as np
import pytest

from block_sparse_video_geometry_b200 import vsa, workloads as W
from oracle import vsa_oracle as O

import vsa_cases as C

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


# --------------------------------------------- tcgen05 building blocks ----
def swizzled_tile(x):
    """bf16 bits [64, 128] -> the 16 KB tile-major block the kernels copy:
    d-half j, row r, 16-byte chunk c stored at j * 8 KB + r * 128 B + 16 (c ^ (r & 7))."""
    x = np.ascontiguousarray(x).reshape(64, 2, 8, 8)          # (row, d half, chunk, element)
    out = np.empty((2, 64, 8, 8), dtype=np.uint16)
    for r in range(64):
        out[:, r, np.arange(8) ^ (r & 7), :] = x[r]
    return out.reshape(-1)


def test_tcgen05_building_blocks(cuda_ok):
    """S = Q K^T at M = 64 into both TMEM lane halves and at M = 128 on a query
    pair (bulk-copied swizzled tiles), and O = P V with P written into TMEM
    (M = 64 in lane half 1, and M = 128), against fp32 matmuls."""
    import torch
    lib = ctypes.CDLL(os.path.join(ROOT, "tests", "native", "libmma_check.so"))
    lib.mma_check_run.restype = ctypes.c_int
    rng = np.random.default_rng(0)
    bf = lambda *s: W.f32_to_bf16_bits(rng.standard_normal(s).astype(np.float32))
    q, qa, qb, k, v = bf(64, 128), bf(64, 128), bf(64, 128), bf(64, 128), bf(64, 128)
    p64, p128 = W.f32_to_bf16_bits(rng.random((64, 64)).astype(np.float32)), \
        W.f32_to_bf16_bits(rng.random((128, 64)).astype(np.float32))
    dev = lambda x: torch.from_numpy(x.view(np.int16)).cuda()
    tq, tqa, tqb, tk, tv = (dev(swizzled_tile(x)) for x in (q, qa, qb, k, v))
    tp64, tp128 = dev(p64), dev(p128)
    outs = [torch.full(sh, float("nan"), device="cuda") for sh in ((64, 64), (64, 64), (128, 64), (64, 128),
                                                                     (128, 128))]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = lib.mma_check_run(*(ptr(t) for t in (tq, tqa, tqb, tk, tv, tp64, tp128)), *(ptr(t) for t in outs), ptr(err))
    assert rc == 0 and int(err.item()) == 0
    f = lambda x: torch.from_numpy(O.bf16_bits_to_f64(x)).float()
    s64_0, s64_1, s128, o64, o128 = (t.cpu() for t in outs)
    ok = lambda got, want: torch.allclose(got, want, atol=1e-2, rtol=1e-3)
    assert ok(s64_0, f(q) @ f(k).T) and ok(s64_1, f(q) @ f(k).T)
    assert ok(s128, torch.cat([f(qa), f(qb)]) @ f(k).T)
    assert ok(o64, f(p64) @ f(v)) and ok(o128, f(p128) @ f(v))


# --------------------------------------------------------- full checks ----
def full_check(wl, out_dtype="f32", heads=None, out_tiles=None, channel_gate=False, **prm_over):
    lay = C.oracle_layout(wl)
    bits = C.inputs(wl, lay, channel_gate)
    prm = C.params_of(wl, **prm_over)
    res = C.gpu_forward(wl, bits, prm, out_dtype)
    assert res["status"] == vsa.OK
    C.check_lists_valid(res, lay, prm["sink"])
    worst = 0.0
    for b in range(wl.B):
        for h in (range(wl.H) if heads is None else heads):
            ho = C.HeadOracle(wl, lay, bits, b, h, prm)
            for t, x in enumerate((ho.qbar, ho.kbar, ho.vbar)):
                assert np.abs(res["pooled"][t, b, h] - x).max() <= 1e-4
            assert np.abs(res["o_coarse"][b, h] - ho.o_coarse).max() <= 1e-3
            near = C.compare_selection(ho, res["idx"][b, h], res["cnt"][b, h])
            assert len(near) <= max(2, lay.n_tiles // 20)
            C.note_near_ties(len(near))
            tiles = set(range(lay.n_tiles) if out_tiles is None else out_tiles(lay)) | set(near)
            mx, _ = C.compare_outputs(ho, res, b, h, sorted(tiles), bf16=(out_dtype == "bf16"), near_tie=near)
            worst = max(worst, mx)
    return res, worst


def test_tiny_full(cuda_ok):
    full_check(W.WORKLOADS["tiny"])


def test_tiny_bf16_output(cuda_ok):
    full_check(W.WORKLOADS["tiny"], out_dtype="bf16")


@pytest.mark.parametrize("sink", [O.SINK_EXACT_KV, O.SINK_EXACT_KV_AND_ROWS, O.SINK_OFF])
@pytest.mark.parametrize("keep", [0.125, 0.5, 1.0])
def test_tiny_keep_and_sink(cuda_ok, keep, sink):
    full_check(W.WORKLOADS["tiny"], keep=keep, sink=sink)


@pytest.mark.parametrize("tau", [0.0, 1.0, 1.5, 2.0])
def test_tiny_adaptive(cuda_ok, tau):
    full_check(W.WORKLOADS["tiny"].with_(mode=O.MODE_ADAPTIVE, tau=tau))


EDGE_WORKLOADS = [
    # ragged in every dimension, two batches, one conditioning segment
    W.Workload("ragged_b2", B=2, H=3, cond=((W.SEG_TEXT, 70),), grid=(5, 6, 7), keep=0.3, seed=11),
    # no conditioning prefix at all
    W.Workload("video_only", B=1, H=2, cond=(), grid=(8, 8, 12), keep=0.25, seed=12),
    # conditioning after the video, odd number of tiles, thin grid
    W.Workload("cond_after", B=1, H=2, cond=((W.SEG_TEXT, 5),), grid=(9, 4, 13), keep=0.2, seed=13,
               cond_after=((W.SEG_REF_AUDIO, 100),)),
    # one video tile only, partial
    W.Workload("one_tile", B=1, H=1, cond=((W.SEG_TEXT, 1), (W.SEG_REF_IMAGE, 64), (W.SEG_REF_AUDIO, 65)),
               grid=(1, 1, 1), keep=1.0, seed=14),
    # single-frame, single-row grid
    W.Workload("thin", B=1, H=2, cond=((W.SEG_TEXT, 40),), grid=(3, 1, 9), keep=0.5, seed=15),
]


@pytest.mark.parametrize("wl", EDGE_WORKLOADS, ids=lambda w: w.name)
@pytest.mark.parametrize("sink", [O.SINK_EXACT_KV, O.SINK_EXACT_KV_AND_ROWS, O.SINK_OFF])
def test_edge_layouts(cuda_ok, wl, sink):
    full_check(wl, sink=sink)


@pytest.mark.parametrize("tau", [0.0, 1.5])
def test_tiny_adaptive_sink_off(cuda_ok, tau):
    full_check(W.WORKLOADS["tiny"].with_(mode=O.MODE_ADAPTIVE, tau=tau), sink=O.SINK_OFF)


@pytest.mark.parametrize("wl", [W.WORKLOADS["tiny"], EDGE_WORKLOADS[0]], ids=lambda w: w.name)
@pytest.mark.parametrize("out_dtype", ["f32", "bf16"])
def test_channel_gate(cuda_ok, wl, out_dtype):
    """g [B, S, H, 128]: one gate per channel."""
    full_check(wl, out_dtype=out_dtype, channel_gate=True)


@pytest.mark.parametrize("wl,prm", [
    (W.WORKLOADS["tiny"], {}),
    (EDGE_WORKLOADS[0], {}),                                   # partial tiles, two batches
    (W.WORKLOADS["tiny"], {"sink": O.SINK_OFF}),
    (W.WORKLOADS["tiny"].with_(mode=O.MODE_ADAPTIVE, tau=1.0), {}),
], ids=["tiny", "ragged_b2", "tiny_sink_off", "tiny_adaptive"])
def test_spark_reweight(cuda_ok, wl, prm):
    """Spark-Reweight compressed branch (weighted summaries + log-mass bias)."""
    full_check(wl, coarse=O.COARSE_REWEIGHT, **prm)


def test_mid_spark_reweight_two_heads(cuda_ok):
    wl = W.WORKLOADS["mid"].with_(H=4)
    full_check(wl, heads=(1, 2), out_tiles=lambda lay: range(3, lay.n_tiles, 11), coarse=O.COARSE_REWEIGHT)


def test_mid_sink_off_two_heads(cuda_ok):
    wl = W.WORKLOADS["mid"].with_(H=4)
    full_check(wl, heads=(0, 3), out_tiles=lambda lay: range(0, lay.n_tiles, 9), sink=O.SINK_OFF,
               channel_gate=True)


def test_k_equals_one(cuda_ok):
    full_check(W.WORKLOADS["tiny"], keep=1e-6)


def test_gate_zero_gives_fine_branch_and_keep_all_gives_dense(cuda_ok):
    """keep=100% and g=0: the output is plain dense softmax attention."""
    wl = W.WORKLOADS["tiny"]
    lay = C.oracle_layout(wl)
    q, k, v, g = C.inputs(wl, lay)
    g0 = np.zeros_like(g)
    res = C.gpu_forward(wl, (q, k, v, g0), C.params_of(wl, keep=1.0))
    f = O.bf16_bits_to_f64
    for h in range(wl.H):
        dense = O.softmax_attention(f(q[0, :, h]), f(k[0, :, h]), f(v[0, :, h]), O.default_scale())
        err = np.abs(res["out"][0, :, h] - dense)
        assert err.max() <= C.OUT_MAX_ABS and err.mean() <= C.OUT_MEAN_ABS


def test_deterministic_rerun(cuda_ok):
    wl = W.WORKLOADS["tiny"]
    lay = C.oracle_layout(wl)
    bits = C.inputs(wl, lay)
    a = C.gpu_forward(wl, bits, C.params_of(wl))
    b = C.gpu_forward(wl, bits, C.params_of(wl))
    for key in ("idx", "cnt", "o_coarse", "out"):
        if key == "idx":
            for x, y, n in zip(a["idx"].reshape(-1, a["kmax"]), b["idx"].reshape(-1, b["kmax"]), a["cnt"].ravel()):
                assert np.array_equal(x[:n], y[:n])
        else:
            assert np.array_equal(a[key], b[key])


def test_mid_all_heads_selection_two_heads_outputs(cuda_ok):
    wl = W.WORKLOADS["mid"]
    lay = C.oracle_layout(wl)
    bits = C.inputs(wl, lay)
    prm = C.params_of(wl)
    res = C.gpu_forward(wl, bits, prm)
    C.check_lists_valid(res, lay)
    rng = np.random.default_rng(0)
    for h in range(wl.H):
        ho = C.HeadOracle(wl, lay, bits, 0, h, prm)
        near = C.compare_selection(ho, res["idx"][0, h], res["cnt"][0, h])
        C.note_near_ties(len(near))
        assert np.abs(res["o_coarse"][0, h] - ho.o_coarse).max() <= 1e-3
        tiles = range(lay.n_tiles) if h in (0, 17) else rng.choice(lay.n_tiles, 6, replace=False)
        C.compare_outputs(ho, res, 0, h, sorted(set(int(t) for t in tiles) | set(near)), near_tie=near)
