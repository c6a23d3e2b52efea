"""Host-side tests of libvsa (no GPU needed): the library loads and exports
every function include/vsa.h declares; the C++ geometry map equals the
oracle's bit for bit; k rounding matches; malformed arguments are rejected
with a status before any GPU work."""

import ctypes
import os
import re

import numpy as np
import pytest

from block_sparse_video_geometry_b200 import vsa, workloads as W
from oracle import vsa_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for hdr in os.listdir(os.path.join(ROOT, "include")):
        if hdr.endswith(".h"):
            text = open(os.path.join(ROOT, "include", hdr)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(vsa_\w+)\s*\(", text))
    return sorted(names)


def test_library_exports_every_declared_function():
    names = declared_functions()
    assert "vsa_layout_build" in names and "vsa_coarse_select" in names and "vsa_sparse_attn_fwd" in names
    L = vsa.lib()
    for n in names:
        assert hasattr(L, n), n
    assert vsa.version() >> 16 == 1
    assert vsa.status_string(vsa.ERR_UNSUPPORTED).startswith("unsupported")


def _segments(cond, grid, after=()):
    segs, pos = [], 0
    for kind, n in cond:
        segs.append((kind, pos, n, None))
        pos += n
    nv = grid[0] * grid[1] * grid[2]
    segs.append((vsa.SEG_VIDEO, pos, nv, grid))
    pos += nv
    for kind, n in after:
        segs.append((kind, pos, n, None))
        pos += n
    return segs, pos


CASES = [
    (((0, 32), (1, 16), (2, 16)), (8, 8, 8), ()),
    (((0, 512), (1, 448), (2, 64)), (16, 32, 32), ()),
    (((0, 70),), (5, 6, 7), ()),
    ((), (3, 1, 9), ()),
    (((0, 1), (1, 64), (2, 65)), (1, 1, 1), ()),
    (((0, 5),), (9, 4, 13), ((2, 100),)),           # conditioning after the video
    (((0, 512), (1, 4032), (2, 128)), (61, 48, 84), ()),
]


@pytest.mark.parametrize("cond,grid,after", CASES)
def test_layout_matches_oracle_bit_exact(cond, grid, after):
    segs, S = _segments(cond, grid, after)
    lay = vsa.Layout(segs, S)
    ref = O.build_layout([O.Segment(k, s, n, g) for (k, s, n, g) in segs], S)
    perm, inv, cnt, kind = lay.tables()
    assert lay.info.n_cond_tiles == ref.n_cond_tiles
    assert lay.info.n_video_tiles == ref.n_video_tiles
    assert np.array_equal(perm, ref.perm)
    assert np.array_equal(inv, ref.inv)
    assert np.array_equal(cnt, (ref.perm >= 0).sum(1))
    assert np.array_equal(kind, ref.tile_kind)
    assert lay.info.device_bytes >= perm.nbytes + inv.nbytes


def test_sink_off_candidates_are_all_tiles():
    segs, S = _segments(((0, 32), (1, 16), (2, 16)), (8, 8, 8))
    lay = vsa.Layout(segs, S)
    ref = O.build_layout([O.Segment(k, s, n, g) for (k, s, n, g) in segs], S)
    nt = lay.info.n_tiles
    for keep in (0.25, 0.5, 0.1, 1.0):
        assert lay.kmax(vsa.make_params(keep=keep, sink=vsa.SINK_OFF)) == O.topk_count(keep, nt)
        assert lay.kmax(vsa.make_params(keep=keep, sink=vsa.SINK_OFF)) == \
            O.topk_count(keep, O.candidate_tiles(ref, O.SINK_OFF)[1])
    assert lay.kmax(vsa.make_params(mode=vsa.SELECT_ADAPTIVE, sink=vsa.SINK_OFF)) == nt
    # both workspaces: a 256-byte header, then the pooled means [3, B, H, n_tiles, 128];
    # Spark-Reweight adds its score matrix and summaries, the mean branch its
    # split Kbar / Vbar chunks (32 KB per 64 candidates and head) and marks
    nv, pooled = lay.info.n_video_tiles, 256 + 3 * 2 * nt * 128 * 4
    rw = lay.coarse_select_workspace_size(1, 2, vsa.make_params(keep=0.5, coarse=vsa.COARSE_REWEIGHT))
    on = lay.coarse_select_workspace_size(1, 2, vsa.make_params(keep=0.5))
    assert rw >= pooled + 2 * nt * 64 * 4 + 2 * 2 * nv * 128 * 4
    assert on >= pooled + 2 * 2 * ((nv + 63) // 64) * 32768 + 2 * nt * 2 * ((nv + 63) // 64) * 4
    # the score matrix spans every tile: the selection workspace grows accordingly
    on = lay.coarse_select_workspace_size(1, 2, vsa.make_params(keep=0.5))
    off = lay.coarse_select_workspace_size(1, 2, vsa.make_params(keep=0.5, sink=vsa.SINK_OFF))
    assert off >= on


def test_topk_count_matches_oracle():
    segs, S = _segments(((0, 64),), (8, 8, 8))
    rng = np.random.default_rng(0)
    for nv_grid in [(8, 8, 8), (16, 32, 32), (32, 48, 84), (61, 48, 84), (7, 5, 3)]:
        segs, S = _segments(((0, 64),), nv_grid)
        lay = vsa.Layout(segs, S)
        nv = lay.info.n_video_tiles
        for keep in list(rng.uniform(0, 1, 40)) + [0.1, 0.2, 0.5, 1.0, 1e-7, 0.25]:
            keep = float(np.float32(keep))
            if keep <= 0:
                continue
            p = vsa.make_params(keep=keep)
            assert lay.kmax(p) == O.topk_count(keep, nv), (keep, nv)
        assert lay.kmax(vsa.make_params(mode=vsa.SELECT_ADAPTIVE, tau=1.0)) == nv


@pytest.mark.parametrize("segs,S,status", [
    ([(0, 0, 10, None)], 10, vsa.ERR_UNSUPPORTED),                                   # no video
    ([(4, 0, 8, (2, 2, 2)), (4, 8, 8, (2, 2, 2))], 16, vsa.ERR_UNSUPPORTED),          # two videos
    ([(0, 0, 4, None), (4, 5, 8, (2, 2, 2))], 13, vsa.ERR_INVALID_ARG),               # gap
    ([(4, 0, 9, (2, 2, 2))], 9, vsa.ERR_INVALID_ARG),                                 # grid mismatch
    ([(0, 0, 4, None), (4, 4, 8, (2, 2, 2))], 20, vsa.ERR_INVALID_ARG),               # not covering
    ([(7, 0, 4, None), (4, 4, 8, (2, 2, 2))], 12, vsa.ERR_INVALID_ARG),               # bad kind
    ([(0, 0, 0, None), (4, 0, 8, (2, 2, 2))], 8, vsa.ERR_INVALID_ARG),                # empty segment
])
def test_layout_rejects_bad_descriptors(segs, S, status):
    with pytest.raises(vsa.VSAError) as e:
        vsa.Layout(segs, S)
    assert e.value.status == status


def test_calls_validate_before_any_gpu_work():
    segs, S = _segments(((0, 64),), (8, 8, 8))
    lay = vsa.Layout(segs, S)
    L = vsa.lib()
    good = vsa.make_params(keep=0.5)
    n = ctypes.c_size_t()
    for bad in [vsa.make_params(keep=0.0), vsa.make_params(keep=1.5), vsa.make_params(mode=3),
                vsa.make_params(sink=5), vsa.make_params(sink=3), vsa.make_params(coarse=2), vsa.make_params(mode=vsa.SELECT_ADAPTIVE, tau=-1.0),
                vsa.make_params(scale=float("nan")), vsa.make_params(extra_tokens=-1),
                vsa.make_params(extra_tokens=vsa.MAX_EXTRA_TOKENS + 1)]:
        assert L.vsa_coarse_select_workspace_size(lay.handle, 1, 2, ctypes.byref(bad), ctypes.byref(n)) == \
            vsa.ERR_INVALID_ARG
    assert L.vsa_coarse_select_workspace_size(lay.handle, 1, 2, ctypes.byref(good), ctypes.byref(n)) == vsa.OK
    assert n.value > 0
    fake = 1 << 20   # aligned non-null fake pointer: validation must stop before it is touched
    args = dict(q=fake, k=fake, v=fake, sb=S * 2 * 128, ss=2 * 128, sh=128)
    # layout not uploaded
    st = L.vsa_coarse_select(lay.handle, ctypes.byref(good), 1, 2, args["q"], args["k"], args["v"], args["sb"],
                             args["ss"], args["sh"], fake, fake, fake, fake, n.value, None)
    assert st == vsa.ERR_NOT_UPLOADED
    # misaligned q, bad strides, null outputs, small workspace
    assert L.vsa_coarse_select(lay.handle, ctypes.byref(good), 1, 2, fake + 2, fake, fake, args["sb"], args["ss"],
                               args["sh"], fake, fake, fake, fake, n.value, None) == vsa.ERR_INVALID_ARG
    assert L.vsa_coarse_select(lay.handle, ctypes.byref(good), 1, 2, fake, fake, fake, args["sb"], 3,
                               args["sh"], fake, fake, fake, fake, n.value, None) == vsa.ERR_INVALID_ARG
    assert L.vsa_coarse_select(lay.handle, ctypes.byref(good), 1, 2, fake, fake, fake, args["sb"], args["ss"],
                               args["sh"], None, fake, fake, fake, n.value, None) == vsa.ERR_INVALID_ARG
    assert L.vsa_coarse_select(lay.handle, ctypes.byref(good), 0, 2, fake, fake, fake, args["sb"], args["ss"],
                               args["sh"], fake, fake, fake, fake, n.value, None) == vsa.ERR_INVALID_ARG
    kmax = lay.kmax(good)
    common = (lay.handle, ctypes.byref(good), 1, 2, fake, fake, fake, args["sb"], args["ss"], args["sh"],
              fake, 2, 2 * S, 2, 0)
    # wrong kmax, bad out dtype, unaligned out stride, not uploaded
    assert L.vsa_sparse_attn_fwd(*common, fake, fake, kmax, fake, None, None, fake, 7, S * 256, 256, 128, fake, 256,
                                 None) == vsa.ERR_INVALID_ARG
    assert L.vsa_sparse_attn_fwd(*common, fake, fake, kmax, fake, None, None, fake, vsa.OUT_BF16, S * 256, 256, 129, fake,
                                 256, None) == vsa.ERR_INVALID_ARG
    # negative channel stride of the gate
    assert L.vsa_sparse_attn_fwd(*common[:-1], -1, fake, fake, kmax, fake, None, None, fake, vsa.OUT_F32, S * 256, 256, 128,
                                 fake, 1 << 30, None) == vsa.ERR_INVALID_ARG
    ws = lay.sparse_attn_workspace_size(1, 2, good)
    assert ws >= 256 + 2 * lay.info.n_tiles * 32768          # error word + tile-major K/V
    assert L.vsa_sparse_attn_fwd(*common, fake, fake, kmax, fake, None, None, fake, vsa.OUT_F32, S * 256, 256, 128, fake,
                                 ws - 16, None) == vsa.ERR_WORKSPACE_TOO_SMALL
    assert L.vsa_sparse_attn_fwd(*common, fake, fake, kmax, fake, None, None, fake, vsa.OUT_F32, S * 256, 256, 128, fake,
                                 ws, None) == vsa.ERR_NOT_UPLOADED
    # extra_tokens: the lists are required when E > 0; the selection needs E > 0
    ex = vsa.make_params(keep=0.5, extra_tokens=8)
    ex_common = (lay.handle, ctypes.byref(ex)) + common[2:]
    ws_x = lay.sparse_attn_workspace_size(1, 2, ex)
    assert ws_x >= ws + 2 * lay.info.n_tiles * 32768           # one gathered K/V tile per (head, query tile)
    assert L.vsa_sparse_attn_fwd(*ex_common, fake, fake, kmax, fake, None, None, fake, vsa.OUT_F32, S * 256, 256,
                                 128, fake, ws_x, None) == vsa.ERR_INVALID_ARG
    assert L.vsa_sparse_attn_fwd(*ex_common, fake, fake, kmax, fake, fake, fake, fake, vsa.OUT_F32, S * 256, 256,
                                 128, fake, ws_x, None) == vsa.ERR_NOT_UPLOADED
    xs = lay.extra_tokens_workspace_size(1, 2, ex)
    assert L.vsa_extra_tokens_select(lay.handle, ctypes.byref(good), 1, 2, fake, fake, args["sb"], args["ss"],
                                     args["sh"], fake, fake, kmax, fake, fake, fake, xs, None) == vsa.ERR_INVALID_ARG
    assert L.vsa_extra_tokens_select(lay.handle, ctypes.byref(ex), 1, 2, fake, fake, args["sb"], args["ss"],
                                     args["sh"], fake, fake, kmax, fake, fake, fake, xs - 16, None) == \
        vsa.ERR_WORKSPACE_TOO_SMALL
    assert L.vsa_extra_tokens_select(lay.handle, ctypes.byref(ex), 1, 2, fake, fake, args["sb"], args["ss"],
                                     args["sh"], fake, fake, kmax, fake, fake, fake, xs, None) == vsa.ERR_NOT_UPLOADED


def test_layout_matches_oracle_on_random_descriptors():
    """Random segment layouts (conditioning before and after the video, ragged
    grids, one-token segments): the library's tables equal the oracle's."""
    rng = np.random.default_rng(2024)
    for _ in range(60):
        before = [(int(rng.integers(0, 4)), int(rng.integers(1, 200))) for _ in range(int(rng.integers(0, 4)))]
        after = [(int(rng.integers(0, 4)), int(rng.integers(1, 150))) for _ in range(int(rng.integers(0, 2)))]
        grid = tuple(int(x) for x in rng.integers(1, 14, size=3))
        segs, S = _segments(before, grid, after)
        lay = vsa.Layout(segs, S)
        ref = O.build_layout([O.Segment(k, s, n, g) for (k, s, n, g) in segs], S)
        perm, inv, cnt, kind = lay.tables()
        assert np.array_equal(perm, ref.perm) and np.array_equal(inv, ref.inv)
        assert np.array_equal(cnt, (ref.perm >= 0).sum(1)) and np.array_equal(kind, ref.tile_kind)
        # every token sits in exactly one slot
        flat = perm[perm >= 0]
        assert np.array_equal(np.sort(flat), np.arange(S))
