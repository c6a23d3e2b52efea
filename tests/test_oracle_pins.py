"""Pins of the fp64 oracle to facts that do not come from the oracle itself:
hand-worked layouts, closed forms, textbook attention, brute force on tiny
inputs, invariants, and the kept-fraction table printed for the adaptive
threshold. CPU only."""

import math
import os

import numpy as np
import pytest

from oracle import vsa_oracle as O
from block_sparse_video_geometry_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def segs_of(wl):
    return [O.Segment(k, s, n, g) for (k, s, n, g) in wl.segments()]


def layout_of(wl):
    return O.build_layout(segs_of(wl), wl.seq_len)


def read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def inputs_f64(wl, lay):
    q, k, v, g = W.make_inputs(wl, lay.inv // O.TILE)
    f = O.bf16_bits_to_f64
    return f(q), f(k), f(v), f(g)


# ----------------------------------------------------------------- layout --
def test_layout_tiny_hand_worked():
    lay = layout_of(W.WORKLOADS["tiny"])
    rows = read_golden("layout_tiny_tokens.txt")
    meta = {r[0]: int(r[1]) for r in rows if len(r) == 2}
    assert lay.n_cond_tiles == meta["n_cond_tiles"]
    assert lay.n_video_tiles == meta["n_video_tiles"]
    for r in rows:
        if len(r) == 3:
            tile, slot, tok = map(int, r)
            assert lay.perm[tile, slot] == tok, (tile, slot)


def test_layout_ragged_hand_worked():
    segs = [O.Segment(O.SEG_VIDEO, 0, 150, (5, 5, 6))]
    lay = O.build_layout(segs, 150)
    rows = read_golden("layout_ragged_tokens.txt")
    for r in rows:
        if r[0] == "valid":
            assert len(lay.tile_tokens(int(r[1]))) == int(r[2])
        elif r[0] == "n_cond_tiles":
            assert lay.n_cond_tiles == int(r[1])
        elif r[0] == "n_video_tiles":
            assert lay.n_video_tiles == int(r[1])
        else:
            tile, slot, tok = map(int, r)
            assert lay.perm[tile, slot] == tok


@pytest.mark.parametrize("name", ["tiny", "mid", "5s", "10s"])
def test_workload_tile_counts(name):
    want = {r[0]: list(map(int, r[1:])) for r in read_golden("workload_tile_counts.txt")}[name]
    lay = layout_of(W.WORKLOADS[name])
    n_valid = (lay.perm[lay.n_cond_tiles:] >= 0).sum(axis=1)
    partial = n_valid[n_valid < O.TILE]
    assert [lay.n_cond_tiles, lay.n_video_tiles, partial.size] == want[:3]
    if partial.size:
        assert set(partial.tolist()) == {want[3]}


@pytest.mark.parametrize("grid,cond", [((8, 8, 8), (32, 16, 16)), ((5, 6, 7), (70,)),
                                       ((3, 1, 9), ()), ((1, 1, 1), (1, 64, 65)), ((9, 4, 13), (5,))])
def test_layout_bijection_and_purity(grid, cond):
    segs, pos = [], 0
    for i, n in enumerate(cond):
        segs.append(O.Segment(i % 3, pos, n))
        pos += n
    nvid = grid[0] * grid[1] * grid[2]
    segs.append(O.Segment(O.SEG_VIDEO, pos, nvid, grid))
    S = pos + nvid
    lay = O.build_layout(segs, S)
    valid = lay.perm[lay.perm >= 0]
    assert np.array_equal(np.sort(valid), np.arange(S))          # every token exactly once
    flat = lay.perm.reshape(-1)
    assert np.array_equal(flat[lay.inv], np.arange(S))           # inv is the inverse
    seg_of_token = np.empty(S, dtype=np.int64)
    for si, s in enumerate(segs):
        seg_of_token[s.start:s.start + s.length] = si
    for t in range(lay.n_tiles):
        toks = lay.tile_tokens(t)
        assert toks.size > 0
        assert np.all(seg_of_token[toks] == lay.tile_segment[t])  # segment-pure
    # video tiles are 4x4x4 cubes: coordinates of a tile's tokens span < 4 per axis
    T, H, Wd = grid
    for t in range(lay.n_cond_tiles, lay.n_tiles):
        rel = lay.tile_tokens(t) - pos
        tt, hh, ww = rel // (H * Wd), (rel // Wd) % H, rel % Wd
        for axis in (tt, hh, ww):
            assert axis.max() - axis.min() < 4 and axis.min() % 4 == 0


def test_layout_rejects_bad_descriptors():
    with pytest.raises(ValueError):
        O.build_layout([O.Segment(O.SEG_TEXT, 0, 10)], 10)                       # no video
    with pytest.raises(ValueError):
        O.build_layout([O.Segment(O.SEG_VIDEO, 0, 8, (2, 2, 2)),
                        O.Segment(O.SEG_VIDEO, 8, 8, (2, 2, 2))], 16)            # two videos
    with pytest.raises(ValueError):
        O.build_layout([O.Segment(O.SEG_TEXT, 0, 4), O.Segment(O.SEG_VIDEO, 5, 8, (2, 2, 2))], 13)
    with pytest.raises(ValueError):
        O.build_layout([O.Segment(O.SEG_VIDEO, 0, 9, (2, 2, 2))], 9)             # grid mismatch


# ------------------------------------------------------- pooling, scores --
def test_pool_tile_constant_closed_form():
    wl = W.WORKLOADS["tiny"]
    lay = layout_of(wl)
    rng = np.random.default_rng(5)
    const = rng.standard_normal((lay.n_tiles, 128))
    x = const[lay.inv // O.TILE]
    assert np.allclose(O.pool_tiles(x, lay), const, rtol=0, atol=1e-14)


def test_pool_and_scores_brute_force_from_coordinates():
    # Recompute pooled means and scores with explicit loops over (t,h,w) cubes,
    # independent of the layout's perm table.
    segs = [O.Segment(O.SEG_TEXT, 0, 70), O.Segment(O.SEG_VIDEO, 70, 5 * 6 * 7, (5, 6, 7))]
    S = 70 + 210
    lay = O.build_layout(segs, S)
    rng = np.random.default_rng(7)
    D = 8
    q = rng.standard_normal((S, D))
    k = rng.standard_normal((S, D))
    qbar, kbar = O.pool_tiles(q, lay), O.pool_tiles(k, lay)
    # conditioning runs: [0,64) and [64,70)
    assert np.allclose(qbar[0], q[0:64].mean(0)) and np.allclose(qbar[1], q[64:70].mean(0))
    tid = 2
    for a in range(2):
        for b in range(2):
            for c in range(2):
                acc, n = np.zeros(D), 0
                for t in range(4 * a, min(5, 4 * a + 4)):
                    for h in range(4 * b, min(6, 4 * b + 4)):
                        for w in range(4 * c, min(7, 4 * c + 4)):
                            acc += k[70 + (t * 6 + h) * 7 + w]
                            n += 1
                assert np.allclose(kbar[tid], acc / n, atol=1e-13)
                tid += 1
    scale = 0.3
    s = O.tile_scores(qbar, kbar, lay, scale)
    assert s.shape == (lay.n_tiles, lay.n_video_tiles)
    for qt in range(lay.n_tiles):
        for v in range(lay.n_video_tiles):
            ref = sum(qbar[qt, d] * kbar[lay.n_cond_tiles + v, d] for d in range(D)) * scale
            assert abs(s[qt, v] - ref) < 1e-12


# -------------------------------------------------------------- selection --
@pytest.mark.parametrize("keep,nv,k", [(0.5, 8, 4), (0.2, 256, 52), (0.1, 2016, 202),
                                       (0.1, 4032, 404), (1.0, 2016, 2016), (1e-6, 100, 1),
                                       (0.25, 2016, 504), (0.1, 4030, 403)])
def test_topk_count(keep, nv, k):
    assert O.topk_count(keep, nv) == k


def test_topk_definition_by_rank_counting():
    rng = np.random.default_rng(11)
    scores = np.round(rng.standard_normal((40, 30)), 1)     # many exact ties
    for k in (1, 3, 7, 30):
        sel = O.select_topk(scores, k)
        for row, chosen in zip(scores, sel):
            # v is kept iff fewer than k entries beat it (higher score, or equal
            # score with a lower ordinal)
            want = [v for v in range(row.size)
                    if sum(1 for u in range(row.size)
                           if row[u] > row[v] or (row[u] == row[v] and u < v)) < k]
            assert chosen.tolist() == want


def test_topk_keep_all_and_argmax():
    rng = np.random.default_rng(2)
    s = rng.standard_normal((9, 17))
    assert all(x.tolist() == list(range(17)) for x in O.select_topk(s, 17))
    assert [int(x[0]) for x in O.select_topk(s, 1)] == s.argmax(1).tolist()


def test_adaptive_threshold_closed_form():
    s = np.array([[0.0, 2.0], [0.0, 2.0]])               # mean 1, population std 1
    assert O.adaptive_threshold(s, 1.0) == pytest.approx(2.0)
    assert O.adaptive_threshold(s, 0.5) == pytest.approx(1.5)
    sel, thr = O.select_adaptive(np.array([[0.0, 2.0], [1.0, 1.5]]), 1.0)
    # second row: nothing reaches the threshold -> it keeps its argmax
    assert sel[0].tolist() == [1] and sel[1].tolist() == [1]


def test_adaptive_kept_fraction_gaussian_tail_and_page_table():
    rng = np.random.default_rng(3)
    s = rng.standard_normal((2000, 2000))
    table = read_golden("sol_attn_tau_kept_fraction.txt")
    for tau_s, page_pct in table:
        tau, page_pct = float(tau_s), float(page_pct)
        sel, _ = O.select_adaptive(s, tau)
        frac = sum(x.size for x in sel) / s.size
        tail = 0.5 * math.erfc(tau / math.sqrt(2))           # Gaussian tail above mu+tau*sigma
        assert abs(frac - tail) < 6 * math.sqrt(tail * (1 - tail) / s.size) + 1e-4
        # the pages' rounded figures sit within half a percentage point of the tail
        assert abs(100 * frac - page_pct) < 0.5


# ----------------------------------------------------------------- coarse --
def test_coarse_tile_constant_equals_tile_resolution_attention():
    wl = W.WORKLOADS["tiny"]
    lay = layout_of(wl)
    rng = np.random.default_rng(4)
    qc, kc, vc = (rng.standard_normal((lay.n_tiles, 128)) for _ in range(3))
    tile = lay.inv // O.TILE
    q, k, v = qc[tile], kc[tile], vc[tile]
    scale = O.default_scale()
    s = O.tile_scores(O.pool_tiles(q, lay), O.pool_tiles(k, lay), lay, scale)
    oc = O.coarse_branch(s, O.pool_tiles(v, lay), lay)
    nc = lay.n_cond_tiles
    ref = O.softmax_attention(qc, kc[nc:], vc[nc:], scale)   # each key tile once
    assert np.allclose(oc, ref, atol=1e-12)


def test_coarse_is_convex_combination():
    rng = np.random.default_rng(8)
    s = rng.standard_normal((5, 6)) * 3
    segs = [O.Segment(O.SEG_VIDEO, 0, 6 * 64, (4, 4, 24))]
    lay = O.build_layout(segs, 6 * 64)
    vbar = rng.standard_normal((6, 4))
    oc = O.coarse_branch(s[:, :6], vbar, lay)
    assert np.all(oc <= vbar.max(0) + 1e-12) and np.all(oc >= vbar.min(0) - 1e-12)


# ------------------------------------------------------------------- fine --
def _tiny_case(**kw):
    wl = W.WORKLOADS["tiny"].with_(**kw)
    lay = layout_of(wl)
    q, k, v, g = inputs_f64(wl, lay)
    return wl, lay, q[0, :, 0], k[0, :, 0], v[0, :, 0], g[0, :, 0]


def test_keep_all_equals_dense_attention():
    wl, lay, q, k, v, g = _tiny_case(keep=1.0)
    res = O.vsa_forward_head(q, k, v, g, lay, O.Params(keep=1.0))
    dense = O.softmax_attention(q, k, v, O.default_scale())
    assert np.allclose(res.o_fine, dense, atol=1e-12)
    g0 = O.vsa_forward_head(q, k, v, np.zeros_like(g), lay, O.Params(keep=1.0))
    assert np.allclose(g0.out, dense, atol=1e-12)


@pytest.mark.parametrize("sink", [O.SINK_EXACT_KV, O.SINK_EXACT_KV_AND_ROWS])
def test_fine_equals_masked_dense_brute_force(sink):
    wl, lay, q, k, v, g = _tiny_case()
    p = O.Params(keep=wl.keep, sink=sink)
    res = O.vsa_forward_head(q, k, v, g, lay, p)
    S = lay.seq_len
    tile = lay.inv // O.TILE
    cond_tok = np.zeros(S, bool)
    cond_tok[lay.cond_tokens()] = True
    mask = np.zeros((S, S), bool)
    for i in range(S):
        qt = tile[i]
        if sink == O.SINK_EXACT_KV_AND_ROWS and qt < lay.n_cond_tiles:
            mask[i, :] = True
            continue
        mask[i, cond_tok] = True                       # conditioning keys never pruned
        for vsel in res.selected[qt]:
            mask[i, tile == lay.n_cond_tiles + vsel] = True
    ref = O.dense_attention_masked(q, k, v, mask, O.default_scale())
    assert np.allclose(res.o_fine, ref, atol=1e-12)


def test_prefix_keys_always_attended_and_video_only_pruning():
    wl, lay, q, k, v, g = _tiny_case()
    res = O.vsa_forward_head(q, k, v, g, lay, O.Params(keep=0.25))
    cond = set(lay.cond_tokens().tolist())
    assert len(cond) == 64
    for qt in range(lay.n_tiles):
        assert all(0 <= x < lay.n_video_tiles for x in res.selected[qt])
        keys = set(O.key_tokens_for_tile(lay, qt, res.selected[qt], O.SINK_EXACT_KV).tolist())
        assert cond <= keys
        assert len(keys) == 64 + 64 * len(res.selected[qt])


def test_no_prefix_all_tiles_is_textbook_attention():
    segs = [O.Segment(O.SEG_VIDEO, 0, 6 * 8 * 8, (6, 8, 8))]
    lay = O.build_layout(segs, 384)
    rng = np.random.default_rng(9)
    q, k, v = (rng.standard_normal((384, 128)) for _ in range(3))
    res = O.vsa_forward_head(q, k, v, np.zeros(384), lay, O.Params(keep=1.0))
    assert np.allclose(res.out, O.softmax_attention(q, k, v, O.default_scale()), atol=1e-12)


def test_rows_dense_conditioning_rows():
    wl, lay, q, k, v, g = _tiny_case(sink=O.SINK_EXACT_KV_AND_ROWS)
    res = O.vsa_forward_head(q, k, v, g, lay, O.Params(keep=0.5, sink=O.SINK_EXACT_KV_AND_ROWS))
    ct = lay.cond_tokens()
    dense = O.softmax_attention(q[ct], k, v, O.default_scale())
    assert np.allclose(res.out[ct], dense, atol=1e-12)            # no coarse term on those rows


def test_gate_zero_and_one():
    wl, lay, q, k, v, g = _tiny_case()
    p = O.Params(keep=0.5)
    r0 = O.vsa_forward_head(q, k, v, np.zeros_like(g), lay, p)
    r1 = O.vsa_forward_head(q, k, v, np.ones_like(g), lay, p)
    assert np.array_equal(r0.out, r0.o_fine)
    tile = lay.inv // O.TILE
    assert np.allclose(r1.out, r1.o_fine + r1.o_coarse[tile], atol=1e-13)


# ------------------------------------------------- sink off, channel gate --
def test_sink_off_fine_equals_masked_dense_brute_force():
    """sink off: a query attends exactly the tokens of its selected tiles and
    nothing else; the mask is built from the token -> tile map alone."""
    wl, lay, q, k, v, g = _tiny_case()
    p = O.Params(keep=0.25, sink=O.SINK_OFF)
    res = O.vsa_forward_head(q, k, v, g, lay, p)
    S = lay.seq_len
    tile = lay.inv // O.TILE
    mask = np.zeros((S, S), bool)
    for i in range(S):
        for c in res.selected[tile[i]]:
            mask[i, tile == c] = True                  # candidate ordinal = tile id
    ref = O.dense_attention_masked(q, k, v, mask, O.default_scale())
    assert np.allclose(res.o_fine, ref, atol=1e-12)


def test_sink_off_selects_over_every_tile():
    wl, lay, q, k, v, g = _tiny_case()
    nt = lay.n_tiles
    assert nt == 11
    res = O.vsa_forward_head(q, k, v, g, lay, O.Params(keep=0.25, sink=O.SINK_OFF))
    assert res.scores.shape == (nt, nt)
    for qt in range(nt):
        assert len(res.selected[qt]) == math.ceil(0.25 * nt) == 3
        assert all(0 <= c < nt for c in res.selected[qt])
    # brute force: the three highest scores of each row, ties to the lower tile
    for qt in range(nt):
        row = [(-res.scores[qt, c], c) for c in range(nt)]
        assert sorted(c for _, c in sorted(row)[:3]) == list(res.selected[qt])
    # a conditioning tile is selected somewhere (the tiny inputs give it the chance)
    assert any(c < lay.n_cond_tiles for sel in res.selected for c in sel)


def test_sink_off_keep_all_is_dense_attention():
    wl, lay, q, k, v, g = _tiny_case()
    res = O.vsa_forward_head(q, k, v, np.zeros_like(g), lay, O.Params(keep=1.0, sink=O.SINK_OFF))
    assert np.allclose(res.out, O.softmax_attention(q, k, v, O.default_scale()), atol=1e-12)


def test_sink_off_coarse_is_tile_resolution_attention_over_all_tiles():
    wl = W.WORKLOADS["tiny"]
    lay = layout_of(wl)
    rng = np.random.default_rng(11)
    qc, kc, vc = (rng.standard_normal((lay.n_tiles, 128)) for _ in range(3))
    tile = lay.inv // O.TILE
    q, k, v = qc[tile], kc[tile], vc[tile]
    scale = O.default_scale()
    s = O.tile_scores(O.pool_tiles(q, lay), O.pool_tiles(k, lay), lay, scale, O.SINK_OFF)
    oc = O.coarse_branch(s, O.pool_tiles(v, lay), lay, O.SINK_OFF)
    assert np.allclose(oc, O.softmax_attention(qc, kc, vc, scale), atol=1e-12)


def test_channel_gate():
    """g [S, D]: constant over channels equals the per-token gate; a one-hot
    channel gate adds the coarse term to that channel only."""
    wl, lay, q, k, v, g = _tiny_case()
    p = O.Params(keep=0.5)
    r_tok = O.vsa_forward_head(q, k, v, g, lay, p)
    r_ch = O.vsa_forward_head(q, k, v, np.repeat(g[:, None], 128, axis=1), lay, p)
    assert np.array_equal(r_tok.out, r_ch.out)
    onehot = np.zeros((lay.seq_len, 128))
    onehot[:, 37] = 2.0
    r1 = O.vsa_forward_head(q, k, v, onehot, lay, p)
    tile = lay.inv // O.TILE
    d = r1.out - r1.o_fine
    assert np.array_equal(np.delete(d, 37, axis=1), np.zeros((lay.seq_len, 127)))
    assert np.allclose(d[:, 37], 2.0 * r1.o_coarse[tile][:, 37], atol=1e-14)


# ------------------------------------------------------- Spark-Reweight --
def test_reweight_anchor_query_is_exact_attention_over_full_tiles():
    """With every candidate tile full, the anchor's reweighted compressed
    branch equals exact token-level softmax attention of the anchor over all
    candidate keys (the bias restores each tile's mass, the weights its
    within-tile distribution); checked against textbook attention."""
    wl, lay, q, k, v, g = _tiny_case(cond=((W.SEG_TEXT, 64), (W.SEG_REF_IMAGE, 128)))
    assert all(len(lay.tile_tokens(t)) == 64 for t in range(lay.n_tiles))
    scale = O.default_scale()
    a = O.video_query_anchor(q, lay)
    vid = np.concatenate([lay.tile_tokens(t) for t in range(lay.n_cond_tiles, lay.n_tiles)])
    assert np.allclose(a, q[vid].mean(0), atol=1e-15)
    for sink, keys in ((O.SINK_EXACT_KV, vid), (O.SINK_OFF, np.arange(lay.seq_len))):
        kt, vt, b = O.reweighted_summaries(k, v, a, lay, scale, sink)
        oc = O.coarse_branch_reweighted(a[None], kt, vt, b, scale)
        ref = O.softmax_attention(a[None], k[keys], v[keys], scale)
        assert np.allclose(oc, ref, atol=1e-12)


def test_reweight_two_token_closed_form():
    """Hand-worked tile: anchor logits 0 and ln 3 -> weights 1/4, 3/4 and an
    effective pooled logit ln((1 + 3) / 2) = ln 2."""
    segs = [O.Segment(O.SEG_VIDEO, 0, 2, (1, 1, 2))]
    lay = O.build_layout(segs, 2)
    a = np.zeros(128)
    a[0] = 1.0
    k = np.zeros((2, 128))
    k[1, 0] = math.log(3.0)                 # scale 1: x = (0, ln 3)
    v = np.zeros((2, 128))
    v[0, 5], v[1, 5] = 8.0, 4.0
    kt, vt, b = O.reweighted_summaries(k, v, a, lay, 1.0)
    assert np.isclose(kt[0, 0], 0.75 * math.log(3.0), atol=1e-15)
    assert np.isclose(vt[0, 5], 0.25 * 8.0 + 0.75 * 4.0, atol=1e-15)
    assert np.isclose(float(a @ kt[0]) + b[0], math.log(2.0), atol=1e-15)


def test_reweight_tile_constant_equals_mean_pooling():
    """Tokens of a tile all equal: the weights are uniform, the bias zero, and
    the reweighted branch is the mean-pooled one."""
    wl = W.WORKLOADS["tiny"]
    lay = layout_of(wl)
    rng = np.random.default_rng(21)
    qc, kc, vc = (rng.standard_normal((lay.n_tiles, 128)) for _ in range(3))
    tile = lay.inv // O.TILE
    q, k, v = qc[tile] + 0.3 * rng.standard_normal((lay.seq_len, 128)), kc[tile], vc[tile]
    scale = O.default_scale()
    p_mean = O.Params(keep=0.5)
    p_rw = O.Params(keep=0.5, coarse=O.COARSE_REWEIGHT)
    r0 = O.selection_for_head(q, k, v, lay, p_mean)
    r1 = O.selection_for_head(q, k, v, lay, p_rw)
    assert np.allclose(r0[6], r1[6], atol=1e-12)          # o_coarse
    for x, y in zip(r0[4], r1[4]):                        # the selection is unchanged
        assert np.array_equal(x, y)
    kt, vt, b = O.reweighted_summaries(k, v, O.video_query_anchor(q, lay), lay, scale)
    assert np.allclose(b, 0.0, atol=1e-12)


def test_reweight_changes_only_the_compressed_branch():
    wl, lay, q, k, v, g = _tiny_case()
    r0 = O.vsa_forward_head(q, k, v, g, lay, O.Params(keep=0.5))
    r1 = O.vsa_forward_head(q, k, v, g, lay, O.Params(keep=0.5, coarse=O.COARSE_REWEIGHT))
    assert np.array_equal(r0.o_fine, r1.o_fine)
    assert not np.allclose(r0.o_coarse, r1.o_coarse, atol=1e-6)
    w = O.reweighted_summaries(k, v, O.video_query_anchor(q, lay), lay, O.default_scale())[1]
    vid_v = v[np.concatenate([lay.tile_tokens(t) for t in range(lay.n_cond_tiles, lay.n_tiles)])]
    # convex combinations of the candidate values
    assert np.all(r1.o_coarse <= vid_v.max(0) + 1e-12) and np.all(r1.o_coarse >= vid_v.min(0) - 1e-12)
    assert np.all(w <= vid_v.max(0) + 1e-12) and np.all(w >= vid_v.min(0) - 1e-12)


# --------------------------------------------------------- extra tokens --
def test_extra_tokens_brute_force():
    """The added tokens are the E best by pooled-query score among the tokens
    of the unselected video tiles, found here by a plain sort over tokens."""
    wl, lay, q, k, v, g = _tiny_case()
    E = 7
    res = O.vsa_forward_head(q, k, v, g, lay, O.Params(keep=0.25, extra_tokens=E))
    tile = lay.inv // O.TILE
    scale = O.default_scale()
    S = lay.seq_len
    cond = np.zeros(S, bool)
    cond[lay.cond_tokens()] = True
    mask = np.zeros((S, S), bool)
    for qt in range(lay.n_tiles):
        rows = np.nonzero(tile == qt)[0]
        qbar = q[rows].mean(0)
        sel_tiles = {lay.n_cond_tiles + int(c) for c in res.selected[qt]}
        cands = [i for i in range(S) if tile[i] >= lay.n_cond_tiles and tile[i] not in sel_tiles]
        best = sorted(cands, key=lambda i: (-scale * float(k[i] @ qbar), i))[:E]
        for r in rows:
            mask[r, cond] = True
            mask[r, [i for i in range(S) if tile[i] in sel_tiles]] = True
            mask[r, best] = True
    ref = O.dense_attention_masked(q, k, v, mask, scale)
    assert np.allclose(res.o_fine, ref, atol=1e-12)
    # E = 0 is the method without extra tokens
    r0 = O.vsa_forward_head(q, k, v, g, lay, O.Params(keep=0.25))
    r00 = O.vsa_forward_head(q, k, v, g, lay, O.Params(keep=0.25, extra_tokens=0))
    assert np.array_equal(r0.out, r00.out)


def test_extra_tokens_covering_everything_is_dense():
    """With E at least the number of unselected video tokens every key is
    attended: the fine branch is textbook dense attention."""
    wl, lay, q, k, v, g = _tiny_case()
    res = O.vsa_forward_head(q, k, v, g, lay, O.Params(keep=0.25, extra_tokens=lay.seq_len))
    assert np.allclose(res.o_fine, O.softmax_attention(q, k, v, O.default_scale()), atol=1e-12)


# ------------------------------------------------------------- generator --
def test_generator_is_seeded_and_bf16_rounded():
    import torch
    wl = W.WORKLOADS["tiny"]
    lay = layout_of(wl)
    a = W.make_inputs(wl, lay.inv // O.TILE)
    b = W.make_inputs(wl, lay.inv // O.TILE, threads=1)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    x = np.random.default_rng(0).standard_normal(10000).astype(np.float32) * 7
    ours = W.f32_to_bf16_bits(x)
    theirs = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, theirs)
    g = O.bf16_bits_to_f64(a[3])
    assert g.min() >= 0 and g.max() <= 1


# ------------------------------------------- planted mistakes must be caught --
def test_planted_mistakes_fail_a_pin(monkeypatch):
    """A transposed score, a dropped scale or a coarse branch over the wrong key
    set each break the tile-constant coarse pin or the dense pin."""
    wl = W.WORKLOADS["tiny"]
    lay = layout_of(wl)
    rng = np.random.default_rng(4)
    qc, kc, vc = (rng.standard_normal((lay.n_tiles, 128)) for _ in range(3))
    tile = lay.inv // O.TILE
    q, k, v = qc[tile], kc[tile], vc[tile]
    scale = O.default_scale()
    nc = lay.n_cond_tiles
    ref = O.softmax_attention(qc, kc[nc:], vc[nc:], scale)

    def coarse_with(score_fn, coarse_fn):
        s = score_fn(O.pool_tiles(q, lay), O.pool_tiles(k, lay), lay, scale)
        return coarse_fn(s, O.pool_tiles(v, lay), lay)

    no_scale = lambda qb, kb, l, sc: qb @ kb[l.n_cond_tiles:].T

    def wrong_offset(s, vb, l):          # pooled V of tiles 0..Nv-1 instead of the video tiles
        p = np.exp(s - s.max(1, keepdims=True))
        p /= p.sum(1, keepdims=True)
        return p @ vb[:s.shape[1]]

    assert not np.allclose(coarse_with(no_scale, O.coarse_branch), ref, atol=1e-6)
    assert not np.allclose(coarse_with(O.tile_scores, wrong_offset), ref, atol=1e-6)

    # fine branch that forgets the conditioning keys fails keep=100% == dense
    wl2, lay2, q2, k2, v2, g2 = _tiny_case(keep=1.0)
    orig = O.key_tokens_for_tile
    monkeypatch.setattr(O, "key_tokens_for_tile",
                        lambda l, qt, sel, sink: orig(l, qt, sel, sink)[len(l.cond_tokens()):])
    bad = O.vsa_forward_head(q2, k2, v2, g2, lay2, O.Params(keep=1.0))
    dense = O.softmax_attention(q2, k2, v2, O.default_scale())
    assert not np.allclose(bad.o_fine, dense, atol=1e-6)


# ------------------------------------------------------------- backward --
def _bwd_case(seed=3, **kw):
    wl, lay, q, k, v, g = _tiny_case(**kw)
    rng = np.random.default_rng(seed)
    dout = rng.standard_normal(q.shape)
    return wl, lay, q, k, v, g, dout


def test_backward_forward_restatement_matches_oracle():
    """The torch restatement used for the gradients computes the oracle's forward."""
    import torch
    from oracle import vsa_backward_oracle as BO
    wl, lay, q, k, v, g, dout = _bwd_case()
    for p in (O.Params(keep=0.25), O.Params(keep=0.25, sink=O.SINK_OFF, coarse=O.COARSE_REWEIGHT),
              O.Params(keep=0.5, sink=O.SINK_EXACT_KV_AND_ROWS, extra_tokens=5)):
        ref = O.vsa_forward_head(q, k, v, g, lay, p).out
        sel = O.selection_for_head(q, k, v, lay, p)[4]
        got = BO.forward_torch(*(torch.tensor(x) for x in (q, k, v, g)), lay, p, sel).numpy()
        assert np.allclose(got, ref, atol=1e-12)


@pytest.mark.parametrize("params", [
    O.Params(keep=0.25),
    O.Params(keep=0.5, sink=O.SINK_EXACT_KV_AND_ROWS),
    O.Params(keep=0.25, sink=O.SINK_OFF, coarse=O.COARSE_REWEIGHT, extra_tokens=3),
], ids=["exact_kv", "rows_dense", "off_reweight_extra"])
def test_backward_matches_finite_differences(params):
    """Directional derivatives of the numpy forward (central differences, the
    selection unchanged at both points) equal <grad, direction>."""
    from oracle import vsa_backward_oracle as BO
    wl, lay, q, k, v, g, dout = _bwd_case()
    grads = BO.vsa_backward_head(q, k, v, g, dout, lay, params)
    rng = np.random.default_rng(5)
    base = (q, k, v, g)
    sel0 = O.selection_for_head(q, k, v, lay, params)[4]
    eps = 1e-5
    for which in range(4):
        u = rng.standard_normal(base[which].shape)
        xs_p = list(base)
        xs_m = list(base)
        xs_p[which] = base[which] + eps * u
        xs_m[which] = base[which] - eps * u
        for xs in (xs_p, xs_m):
            sel = O.selection_for_head(xs[0], xs[1], xs[2], lay, params)[4]
            assert all(np.array_equal(a, b) for a, b in zip(sel, sel0))
        lp = float((O.vsa_forward_head(*xs_p, lay, params).out * dout).sum())
        lm = float((O.vsa_forward_head(*xs_m, lay, params).out * dout).sum())
        fd = (lp - lm) / (2 * eps)
        an = float((grads[which] * u).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (which, fd, an)


def test_backward_keep_all_gate_zero_is_textbook_attention_backward():
    """keep = 100% and g = 0: the gradients of dense attention in closed form
    (dV = P^T dO, dS = P * (dP - rowsum(dP * P)), dQ = c dS K, dK = c dS^T Q)."""
    from oracle import vsa_backward_oracle as BO
    wl, lay, q, k, v, g, dout = _bwd_case(keep=1.0)
    dq, dk, dv, dg = BO.vsa_backward_head(q, k, v, np.zeros_like(g), dout, lay, O.Params(keep=1.0))
    c = O.default_scale()
    s = c * q @ k.T
    P = np.exp(s - s.max(1, keepdims=True))
    P /= P.sum(1, keepdims=True)
    dP = dout @ v.T
    dS = P * (dP - (dP * P).sum(1, keepdims=True))
    assert np.allclose(dv, P.T @ dout, atol=1e-10)
    assert np.allclose(dq, c * dS @ k, atol=1e-10)
    assert np.allclose(dk, c * dS.T @ q, atol=1e-10)
    # dg = <dout, o_coarse[tile]> row by row
    res = O.vsa_forward_head(q, k, v, np.zeros_like(g), lay, O.Params(keep=1.0))
    assert np.allclose(dg, (dout * res.o_coarse[lay.inv // O.TILE]).sum(1), atol=1e-10)
