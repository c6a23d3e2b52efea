"""Shared helpers of the parity tests: seeded inputs, one GPU forward through
the C ABI, the oracle on chosen (batch, head, query tile) samples, and the
comparison rules.

Tolerances (stated here once, used by every parity test):
* layout and selected tile indices: bit-exact, except rows whose oracle
  scores have a near-tie (gap < 1e-4) at the selection boundary; in such a
  row the two sets may differ only by tiles within 1e-4 of the boundary (and
  top-k lists keep their length). Both sets are then valid results of the
  method, so the row's outputs are compared with the oracle's fine branch
  evaluated on the GPU's own list: no query tile is left out;
* fp32 output: max-abs <= 2e-2 and mean-abs <= 2e-3 against the fp64 oracle;
* bf16 output: the same bounds plus the bf16 rounding of the output itself
  (half an ulp of the reference value per element, a quarter ulp on average);
* o_coarse (fp32 path vs fp64): max-abs <= 1e-3; pooled means: max-abs <= 1e-4.
"""

from __future__ import annotations

import numpy as np

from block_sparse_video_geometry_b200 import workloads as W
from oracle import vsa_oracle as O

GAP = 1e-4
OUT_MAX_ABS, OUT_MEAN_ABS = 2e-2, 2e-3

# rows whose GPU list differed from the oracle's at a near-tie (and were
# checked on the GPU's list); the session summary prints the total
NEAR_TIE_ROWS = [0]


def note_near_ties(n: int) -> None:
    NEAR_TIE_ROWS[0] += int(n)


def oracle_layout(wl):
    return O.build_layout([O.Segment(k, s, n, g) for (k, s, n, g) in wl.segments()], wl.seq_len)


def inputs(wl, lay, channel_gate=False):
    """Seeded (q, k, v, g) bf16 bits; with channel_gate, g is [B, S, H, 128]
    (seeded U(0, 1) per channel) instead of [B, S, H]."""
    q, k, v, g = W.make_inputs(wl, lay.inv // O.TILE)
    if channel_gate:
        g = W.make_channel_gate(wl)
    return q, k, v, g


def params_of(wl, **kw):
    d = dict(mode=wl.mode, keep=wl.keep, tau=wl.tau, sink=wl.sink, coarse=O.COARSE_MEAN, extra_tokens=0)
    d.update(kw)
    return d


def gpu_forward(wl, bits, prm: dict, out_dtype="f32", layout=None):
    """Runs vsa_coarse_select + vsa_sparse_attn_fwd on cuda:0; returns numpy arrays."""
    import torch
    from block_sparse_video_geometry_b200 import vsa
    q, k, v, g = bits
    dev = torch.device("cuda:0")
    t = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
    tq, tk, tv, tg = t(q), t(k), t(v), t(g)
    lay = layout or vsa.Layout(wl.segments(), wl.seq_len)
    p = vsa.make_params(**prm)
    fwd = vsa.Forward(lay, p, wl.B, wl.H, device=dev,
                      out_dtype=torch.float32 if out_dtype == "f32" else torch.bfloat16)
    out = fwd(tq, tk, tv, tg)
    assert vsa.coarse_select_status(fwd.ws_select) == vsa.OK
    st = vsa.sparse_attn_status(fwd.ws_attn)
    torch.cuda.synchronize()
    res = dict(status=st, idx=fwd.idx.cpu().numpy(), cnt=fwd.cnt.cpu().numpy(),
               o_coarse=fwd.o_coarse.cpu().numpy(), pooled=fwd.pooled().cpu().numpy(),
               out=out.float().cpu().numpy(), kmax=fwd.kmax)
    if prm.get("extra_tokens", 0) > 0:
        res["extra_status"] = vsa.extra_tokens_status(fwd.ws_extra)
        res["extra_idx"] = fwd.extra_idx.cpu().numpy()
        res["extra_cnt"] = fwd.extra_cnt.cpu().numpy()
    del fwd, tq, tk, tv, tg, out
    torch.cuda.empty_cache()
    return res


class HeadOracle:
    """Oracle state of one (batch, head): pooled means, scores, lists, coarse."""

    def __init__(self, wl, lay, bits, b, h, prm: dict):
        f = O.bf16_bits_to_f64
        q, k, v, g = bits
        self.q, self.k, self.v = f(q[b, :, h]), f(k[b, :, h]), f(v[b, :, h])
        self.g = f(g[b, :, h])
        self.lay = lay
        self.p = O.Params(mode=prm["mode"], keep=prm["keep"], tau=prm["tau"], sink=prm["sink"],
                          coarse=prm.get("coarse", O.COARSE_MEAN), extra_tokens=prm.get("extra_tokens", 0))
        (self.qbar, self.kbar, self.vbar, self.scores, self.sel, self.thr, self.o_coarse,
         self.scale) = O.selection_for_head(self.q, self.k, self.v, lay, self.p)

    def tile_out(self, qt, selected=None, extra=None):
        """Oracle rows of query tile qt; `selected` / `extra` replace the
        oracle's own list / extra tokens (a near-tie row is checked on the
        choice the GPU made)."""
        sel = self.sel[qt] if selected is None else np.asarray(selected, dtype=np.int64)
        return O.output_rows_for_tile(self.q, self.k, self.v, self.g, self.lay, self.p, qt,
                                      sel, self.o_coarse, self.scale, extra=extra)

    def extra_scores(self, qt, selected):
        """(candidate tokens, oracle scores) of query tile qt's extra-token
        ranking given its selected tiles."""
        first, count = O.candidate_tiles(self.lay, self.p.sink)
        chosen = set(int(c) for c in selected)
        toks = [self.lay.tile_tokens(first + c) for c in range(count) if c not in chosen]
        toks = np.concatenate(toks) if toks else np.zeros(0, dtype=np.int64)
        qbar = self.q[self.lay.tile_tokens(qt)].mean(axis=0)
        return toks, self.scale * (self.k[toks] @ qbar)


def check_lists_valid(res, lay, sink=O.SINK_EXACT_KV):
    """Every list of every (batch, head, query tile) is strictly ascending, in
    range (candidate ordinals) and 1 <= cnt <= kmax."""
    idx, cnt = res["idx"], res["cnt"]
    nv = O.candidate_tiles(lay, sink)[1]
    assert cnt.min() >= 1 and cnt.max() <= res["kmax"]
    live = np.arange(idx.shape[-1])[None, None, None, :] < cnt[..., None]
    assert np.all(np.where(live, idx, 0) >= 0) and np.all(np.where(live, idx, 0) < nv)
    both = live[..., 1:]
    assert np.all(np.where(both, idx[..., 1:] > idx[..., :-1], True))


def compare_selection(ho: HeadOracle, gpu_idx, gpu_cnt):
    """Checks the GPU's lists of one (batch, head) against the oracle's.

    Returns {query tile: GPU list} for the rows that differ at a near-tie;
    asserts that every other row is identical. A near-tie row may differ only
    by tiles whose oracle score lies within GAP of the selection boundary, and
    under top-k it must keep the oracle's length k."""
    near_tie = {}
    for qt, want in enumerate(ho.sel):
        got = gpu_idx[qt, : gpu_cnt[qt]]
        if got.size == want.size and np.array_equal(got, want):
            continue
        row = ho.scores[qt]
        if ho.p.mode == O.MODE_TOPK:
            assert got.size == want.size, "query tile %d: top-k list of length %d, want %d" % (
                qt, got.size, want.size)
            srt = np.sort(row)[::-1]
            kk = want.size
            edge = srt[kk - 1]
            nxt = srt[kk] if kk < srt.size else -np.inf
            assert edge - nxt < GAP, "query tile %d: selection differs without a near-tie" % qt
        else:
            edge = ho.thr
        diff = np.setxor1d(got, want)
        assert np.all(np.abs(row[diff] - edge) < GAP), "query tile %d: differs away from the boundary" % qt
        near_tie[qt] = got.copy()
    return near_tie


def compare_extra(ho: HeadOracle, gpu_idx, gpu_cnt, tiles, near_sel=None):
    """Checks the GPU's extra-token sets of the given query tiles against the
    oracle's (ranked given the selection the GPU used). Returns {query tile: GPU
    set} for sets that differ at a near-tie: same size, and every differing
    token's oracle score within GAP of the E-th best score."""
    near_sel = near_sel or {}
    E = ho.p.extra_tokens
    rows_dense = ho.p.sink == O.SINK_EXACT_KV_AND_ROWS
    near = {}
    for qt in tiles:
        got = np.sort(gpu_idx[qt, : gpu_cnt[qt]])
        if rows_dense and qt < ho.lay.n_cond_tiles:
            assert gpu_cnt[qt] == 0
            continue
        sel = near_sel.get(qt, ho.sel[qt])
        toks, sc = ho.extra_scores(qt, sel)
        order = np.lexsort((toks, -sc))
        want = np.sort(toks[order[:E]])
        assert got.size == want.size, "query tile %d: %d extra tokens, want %d" % (qt, got.size, want.size)
        if np.array_equal(got, want):
            continue
        edge = sc[order[want.size - 1]]
        diff = np.setxor1d(got, want)
        pos = {int(t): i for i, t in enumerate(toks)}
        assert all(int(t) in pos for t in diff), "query tile %d: extra token outside the candidates" % qt
        gaps = np.abs(sc[[pos[int(t)] for t in diff]] - edge)
        assert np.all(gaps < GAP), "query tile %d: extra tokens differ away from the boundary" % qt
        near[qt] = got
    return near


def out_error(got, want, bf16: bool):
    """(max excess over the bound, mean-abs error, mean bound) for one block of rows."""
    err = np.abs(got - want)
    if not bf16:
        return float(err.max()), float(err.mean()), OUT_MEAN_ABS
    half_ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(want), 1e-30))) - 8)
    return float((err - half_ulp).max()), float(err.mean()), OUT_MEAN_ABS + float((half_ulp / 2).mean())


def compare_outputs(ho: HeadOracle, res, b, h, tiles, bf16=False, near_tie=None, extra=None):
    """Compares the GPU output rows of the given query tiles with the oracle.
    Rows in `near_tie` (from compare_selection) are compared with the oracle
    evaluated on the GPU's list for that tile; with extra tokens, every row is
    evaluated on the GPU's extra set (`extra`: {query tile: tokens}), which
    compare_extra has checked against the oracle's."""
    near_tie = near_tie or {}
    extra = extra or {}
    errs, means, bounds = [], [], []
    for qt in tiles:
        toks, of, want = ho.tile_out(qt, near_tie.get(qt), extra.get(qt))
        got = res["out"][b, toks, h]
        mx, mean, bound = out_error(got, want, bf16)
        errs.append(mx)
        means.append(mean)
        bounds.append(bound)
    assert max(errs) <= OUT_MAX_ABS, "max-abs %.3g" % max(errs)
    assert float(np.mean(means)) <= float(np.mean(bounds)), "mean-abs %.3g" % np.mean(means)
    return max(errs), float(np.mean(means))
