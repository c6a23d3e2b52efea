"""Plain, slow fp64 CPU oracle for VSA-style block-sparse video attention (forward).

TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module. The
product path (the CUDA library and its Python binding) never calls it, and this
module imports nothing from the product package.

What it computes, step by step, in the order the pages describe it:

1. Geometry map. Conditioning segments (text, reference image, reference audio)
   are cut into segment-pure tiles; the generated video is cut into 4x4x4
   spatio-temporal cubes of 64 tokens.
   ("Ref2VA VSA : noeud d'attention sparse pour le Ref2VA H3", section
   "Le correctif d'attention a deux niveaux", item 1; "ComfyUI-Ref2VA-VSA",
   sections "Technical Architecture" and "The Solution: Ref2VAVSAGatePatch".)
2. Coarse branch: Q, K, V are mean-pooled per tile, query tiles are scored
   against every video key tile, and the scores are softmaxed against the pooled
   V. ("ComfyUI Agrega Nodo Central de Atencion Dispersa ...", section
   "Atencion dispersa por bloques", VSA bullet: cubic tiling with a coarse
   compression branch; "Spark-H3 ...", section "Que cambia Spark-Attn": the
   compressed branch uses mean-pooled key/value summaries.)
3. Selection of the video key tiles each query tile attends exactly: a fixed
   keep fraction (top-k), or a per-head adaptive threshold mean + tau*std.
   ("BSAI FastH3 Native VSA (recipe)", sections "The mechanism, briefly" and
   "The inputs that matter"; "ComfyUI Agrega Nodo Central ...", Sol-Attn and
   top-k bullets.) Only video key tiles are pruned; conditioning keys are never
   pruned ("ComfyUI-Ref2VA-VSA", "Video-Only Sparse Attention").
4. Fine branch: exact softmax attention of each query token over every
   conditioning key token plus the tokens of the selected video tiles
   (sink_conditioning = exact_kv). With exact_kv_and_rows the conditioning query
   rows attend to the whole sequence. With sink_conditioning = off no key tile
   is protected: conditioning tiles are scored, selected and summarised like
   video tiles. ("BSAI FastH3 Native VSA (recipe)", "The inputs that matter",
   sink_conditioning.)
5. Output: o = o_fine + g * o_coarse, g a per-token, per-head gate given as an
   input (the to_gate_compress output), either one value per (token, head) or
   one per (token, head, channel).

Where the pages leave a step open this module takes the plainest reading and
says so in the docstring of the function concerned. Every floating-point step
is carried out in float64; bf16 inputs are decoded exactly.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

TILE = 64          # tokens per tile ("The mechanism, briefly": 64-token blocks)
CUBE = 4           # 4 frames x 4 rows x 4 columns per video tile
HEAD_DIM = 128     # head_dim of the native kernel ("BSAI FastH3 Native VSA", backends)

SEG_TEXT, SEG_REF_IMAGE, SEG_REF_AUDIO, SEG_OTHER_COND, SEG_VIDEO = 0, 1, 2, 3, 4

MODE_TOPK, MODE_ADAPTIVE = 0, 1
SINK_EXACT_KV, SINK_EXACT_KV_AND_ROWS, SINK_OFF = 0, 1, 2
COARSE_MEAN, COARSE_REWEIGHT = 0, 1


# --------------------------------------------------------------------------- #
# bf16 decoding
# --------------------------------------------------------------------------- #
def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact decode of bf16 bit patterns (uint16) to float64."""
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------- #
# 1. Geometry map
# --------------------------------------------------------------------------- #
@dataclass
class Segment:
    kind: int
    start: int
    length: int
    grid: tuple[int, int, int] | None = None   # (T, H, W) for the video segment only


@dataclass
class Layout:
    seq_len: int
    n_cond_tiles: int
    n_video_tiles: int
    grid: tuple[int, int, int]
    video_start: int
    # perm[tile, slot] = token index, or -1 for a padding slot
    perm: np.ndarray = field(repr=False)
    # inv[token] = tile * 64 + slot
    inv: np.ndarray = field(repr=False)
    # per tile: segment index in the descriptor, and the segment kind
    tile_segment: np.ndarray = field(repr=False)
    tile_kind: np.ndarray = field(repr=False)

    @property
    def n_tiles(self) -> int:
        return self.n_cond_tiles + self.n_video_tiles

    def valid_slots(self, tile: int) -> np.ndarray:
        return np.nonzero(self.perm[tile] >= 0)[0]

    def tile_tokens(self, tile: int) -> np.ndarray:
        row = self.perm[tile]
        return row[row >= 0]

    def cond_tokens(self) -> np.ndarray:
        """All tokens of all conditioning tiles, in tile/slot order."""
        row = self.perm[: self.n_cond_tiles].reshape(-1)
        return row[row >= 0]


def build_layout(segments: list[Segment], seq_len: int) -> Layout:
    """Token -> tile geometry map.

    Reading of the pages (the pages name the tiles, not their exact slot order):
    * segments are given in sequence order and cover [0, seq_len) without gaps;
      exactly one of them is the generated video, the others are conditioning;
    * a conditioning segment is cut into contiguous runs of 64 tokens in
      sequence order, the last run possibly partial; no tile crosses a segment
      boundary (segment-pure tiles, "Le correctif d'attention a deux niveaux",
      item 1);
    * the video segment holds a T x H x W latent grid in raster order (t slowest,
      then h, then w). Tile (a, b, c) holds the tokens with t in [4a, 4a+4),
      h in [4b, 4b+4), w in [4c, 4c+4) clipped to the grid; tiles are numbered
      in raster order over (a, b, c); slots inside a tile are raster order over
      (t, h, w) and slots outside the grid are padding;
    * tile ids: conditioning tiles first, in segment order, then video tiles.
    """
    if seq_len <= 0:
        raise ValueError("seq_len must be positive")
    pos = 0
    n_video = 0
    for s in segments:
        if s.start != pos or s.length <= 0:
            raise ValueError("segments must be contiguous, in order, non-empty")
        if s.kind == SEG_VIDEO:
            n_video += 1
            t, h, w = s.grid
            if t * h * w != s.length:
                raise ValueError("video grid does not match the segment length")
        pos += s.length
    if pos != seq_len:
        raise ValueError("segments do not cover the sequence")
    if n_video != 1:
        raise ValueError("exactly one video segment is required")

    tiles: list[list[int]] = []
    tile_seg: list[int] = []
    tile_kind: list[int] = []
    for si, s in enumerate(segments):
        if s.kind == SEG_VIDEO:
            continue
        for run0 in range(0, s.length, TILE):
            toks = [s.start + run0 + i for i in range(min(TILE, s.length - run0))]
            tiles.append(toks + [-1] * (TILE - len(toks)))
            tile_seg.append(si)
            tile_kind.append(s.kind)
    n_cond = len(tiles)

    vi = next(i for i, s in enumerate(segments) if s.kind == SEG_VIDEO)
    vs = segments[vi]
    T, H, W = vs.grid
    for a in range(-(-T // CUBE)):
        for b in range(-(-H // CUBE)):
            for c in range(-(-W // CUBE)):
                slots = []
                for dt in range(CUBE):
                    for dh in range(CUBE):
                        for dw in range(CUBE):
                            t, h, w = CUBE * a + dt, CUBE * b + dh, CUBE * c + dw
                            if t < T and h < H and w < W:
                                slots.append(vs.start + (t * H + h) * W + w)
                            else:
                                slots.append(-1)
                tiles.append(slots)
                tile_seg.append(vi)
                tile_kind.append(SEG_VIDEO)
    perm = np.array(tiles, dtype=np.int64).reshape(-1, TILE)
    inv = np.full(seq_len, -1, dtype=np.int64)
    for tile in range(perm.shape[0]):
        for slot in range(TILE):
            tok = perm[tile, slot]
            if tok >= 0:
                inv[tok] = tile * TILE + slot
    return Layout(seq_len=seq_len, n_cond_tiles=n_cond,
                  n_video_tiles=perm.shape[0] - n_cond, grid=(T, H, W),
                  video_start=vs.start, perm=perm, inv=inv,
                  tile_segment=np.array(tile_seg, dtype=np.int64),
                  tile_kind=np.array(tile_kind, dtype=np.int64))


# --------------------------------------------------------------------------- #
# 2. Coarse branch: pooling, tile scores, softmax over pooled V
# --------------------------------------------------------------------------- #
def pool_tiles(x: np.ndarray, layout: Layout) -> np.ndarray:
    """Mean of x[token, :] over the valid tokens of each tile -> [n_tiles, D].

    x is one (batch, head) slice [seq_len, D]. Padding slots do not count
    (reading: a partial tile is the mean of the tokens it holds).
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.empty((layout.n_tiles, x.shape[1]), dtype=np.float64)
    for tile in range(layout.n_tiles):
        out[tile] = x[layout.tile_tokens(tile)].mean(axis=0)
    return out


def default_scale(head_dim: int = HEAD_DIM) -> float:
    """Softmax scale 1/sqrt(head_dim), used by both branches (reading)."""
    return 1.0 / math.sqrt(head_dim)


def candidate_tiles(layout: Layout, sink: int) -> tuple[int, int]:
    """(first tile id, count) of the key tiles that are scored, selected and
    summarised by the coarse branch.

    exact_kv and exact_kv_and_rows protect the conditioning keys, so only the
    video tiles are candidates ("Video-Only Sparse Attention"). Reading of
    sink_conditioning = off ("cheapest", "The inputs that matter"): nothing is
    protected, so every tile, conditioning or video, is a candidate on equal
    terms and no key is attended exactly unless its tile is selected.
    """
    if sink == SINK_OFF:
        return 0, layout.n_tiles
    return layout.n_cond_tiles, layout.n_video_tiles


def tile_scores(qbar: np.ndarray, kbar: np.ndarray, layout: Layout, scale: float,
                sink: int = SINK_EXACT_KV) -> np.ndarray:
    """s[qt, c] = scale * <qbar[qt], kbar[first + c]> for every query tile qt and
    every candidate key tile c (see candidate_tiles; with the conditioning
    protected, column c is video tile ordinal c, tile id n_cond + c).

    Reading: the score is the scaled logit of the pooled query against the
    pooled key; only candidate key tiles are scored because only they are pruned.
    """
    first, count = candidate_tiles(layout, sink)
    kv = kbar[first:first + count]
    return scale * (qbar @ kv.T)


def topk_count(keep: float, n_video_tiles: int) -> int:
    """k = max(1, ceil(keep * Nv)), keep given as a float32 fraction.

    Reading: the knob is a percentage of video key tiles (keep 10% / 20% /
    100%, "The inputs that matter"); a relative guard of 2^-20 absorbs the
    float32 rounding of keep so that, e.g., 0.5 * 8 = 4 and 0.1 * 4030 = 403.
    """
    kf = float(np.float32(keep))
    k = math.ceil(kf * n_video_tiles * (1.0 - 2.0 ** -20))
    return max(1, min(n_video_tiles, k))


def select_topk(scores: np.ndarray, k: int) -> list[np.ndarray]:
    """Per query tile: the k video tiles with the highest score.

    Reading: a tie in score goes to the lower tile ordinal; each list is
    returned in ascending tile order.
    """
    out = []
    ids = np.arange(scores.shape[1])
    for row in scores:
        order = np.lexsort((ids, -row))          # by score descending, then ordinal
        out.append(np.sort(order[:k]).astype(np.int64))
    return out


def adaptive_threshold(scores: np.ndarray, tau: float) -> float:
    """mean + tau * std of one head's tile-score matrix.

    Reading of the per-head threshold "in sigmas of the score distribution"
    (Sol-Attn bullet): the distribution is every (query tile, video key tile)
    score of this (batch, head), std is the population std (ddof = 0).
    """
    mu = float(np.mean(scores))
    sd = float(np.sqrt(np.mean((scores - mu) ** 2)))
    return mu + float(np.float32(tau)) * sd


def select_adaptive(scores: np.ndarray, tau: float) -> tuple[list[np.ndarray], float]:
    """Keep every video tile whose score is >= mean + tau * std; a row that keeps
    nothing keeps its argmax (lowest ordinal among equal maxima). Reading: a
    query tile always attends at least one video tile."""
    thr = adaptive_threshold(scores, tau)
    out = []
    for row in scores:
        sel = np.nonzero(row >= thr)[0]
        if sel.size == 0:
            sel = np.array([int(np.argmax(row))])
        out.append(sel.astype(np.int64))
    return out, thr


def coarse_branch(scores: np.ndarray, vbar: np.ndarray, layout: Layout,
                  sink: int = SINK_EXACT_KV) -> np.ndarray:
    """o_coarse[qt] = sum_c softmax_c(s[qt, :]) * vbar[first + c].

    Reading: the compressed branch attends, at tile resolution, to every
    candidate key tile (the video tiles, or every tile with sink off) with the
    same scores used for selection; its query is the pooled query of the tile,
    broadcast to the tile's tokens.
    """
    first, count = candidate_tiles(layout, sink)
    vv = vbar[first:first + count]
    m = scores.max(axis=1, keepdims=True)
    p = np.exp(scores - m)
    p /= p.sum(axis=1, keepdims=True)
    return p @ vv


def video_query_anchor(q: np.ndarray, layout: Layout) -> np.ndarray:
    """Mean query of every valid video token of one (batch, head): the per-head
    anchor of Spark-Reweight ("Spark-H3: atencion dispersa por bloques ...",
    "Que cambia Spark-Attn": the scoring uses the mean of the video queries as
    a per-head anchor, which keeps the extra cost linear)."""
    toks = np.concatenate([layout.tile_tokens(t) for t in range(layout.n_cond_tiles, layout.n_tiles)])
    return np.asarray(q, dtype=np.float64)[toks].mean(axis=0)


def reweighted_summaries(k: np.ndarray, v: np.ndarray, anchor: np.ndarray, layout: Layout,
                         scale: float, sink: int = SINK_EXACT_KV):
    """Spark-Reweight summaries of the candidate key tiles (same section).

    Mean pooling scores a tile with exp(E[x]) where attention weighs it with
    E[exp(x)]; Spark-Reweight uses weighted summaries plus a log-mass bias.
    Reading, per candidate tile t with valid tokens i and anchor logits
    x_i = scale * <anchor, k_i>:
      weights  w_i = exp(x_i) / sum_j exp(x_j)          (the anchor's softmax inside t)
      K~_t = sum_i w_i k_i,  V~_t = sum_i w_i v_i
      b_t  = log(mean_i exp(x_i)) - scale * <anchor, K~_t>
    so that the anchor's effective pooled logit scale * <anchor, K~_t> + b_t has
    an exponential equal to the tile's expected exponential mean_i exp(x_i).
    Returns (K~ [n_cand, D], V~ [n_cand, D], b [n_cand]).
    """
    first, count = candidate_tiles(layout, sink)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    D = k.shape[1]
    kt, vt, b = np.empty((count, D)), np.empty((count, D)), np.empty(count)
    for c in range(count):
        toks = layout.tile_tokens(first + c)
        x = scale * (k[toks] @ anchor)
        m = x.max()
        e = np.exp(x - m)
        w = e / e.sum()
        kt[c] = w @ k[toks]
        vt[c] = w @ v[toks]
        b[c] = m + math.log(e.mean()) - scale * float(anchor @ kt[c])
    return kt, vt, b


def coarse_branch_reweighted(qbar: np.ndarray, kt: np.ndarray, vt: np.ndarray, bias: np.ndarray,
                             scale: float) -> np.ndarray:
    """Compressed branch with Spark-Reweight summaries:
    o_coarse[qt] = sum_c softmax_c(scale * <qbar[qt], K~_c> + b_c) V~_c.
    Reading: the query side stays the pooled query of the tile, and only the
    compressed branch changes; the selection keeps the mean-pooled scores."""
    s = scale * (qbar @ kt.T) + bias[None, :]
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    p /= p.sum(axis=1, keepdims=True)
    return p @ vt


# --------------------------------------------------------------------------- #
# 3/4. Fine branch
# --------------------------------------------------------------------------- #
def key_tokens_for_tile(layout: Layout, qt: int, selected: np.ndarray, sink: int) -> np.ndarray:
    """Key tokens that query tile qt attends exactly.

    exact_kv: every conditioning token plus the tokens of the selected video
    tiles. exact_kv_and_rows: a conditioning query tile attends every token.
    off: the tokens of the selected tiles only (candidate ordinals, see
    candidate_tiles). Reading: under exact_kv and off the conditioning query
    tiles are treated like video query tiles (the pages only say that video
    queries see the conditioning rows exactly).
    """
    if sink == SINK_EXACT_KV_AND_ROWS and qt < layout.n_cond_tiles:
        return np.arange(layout.seq_len, dtype=np.int64)
    first, _ = candidate_tiles(layout, sink)
    parts = [] if sink == SINK_OFF else [layout.cond_tokens()]
    for c in selected:
        parts.append(layout.tile_tokens(first + int(c)))
    return np.concatenate(parts)


def extra_tokens_for_tile(qbar_qt: np.ndarray, k: np.ndarray, layout: Layout, selected: np.ndarray,
                          n_extra: int, scale: float, sink: int = SINK_EXACT_KV) -> np.ndarray:
    """extra_tokens ("ComfyUI Agrega Nodo Central de Atencion Dispersa y
    Compilador Comfy", "Atencion dispersa por bloques": the highest-scoring
    tokens beyond the selected blocks are added, to stay closer to dense).

    Reading: the candidates are the valid tokens of the candidate key tiles
    that query tile qt did not select (tokens it attends anyway are not
    candidates); a token's score is scale * <qbar[qt], k_token>, the tile
    score taken at token resolution; the n_extra highest are added to the
    exact key set of every query of the tile (ties: lower token index).
    Returns the added tokens in ascending order.
    """
    if n_extra <= 0:
        return np.zeros(0, dtype=np.int64)
    first, count = candidate_tiles(layout, sink)
    chosen = set(int(c) for c in selected)
    cand = [layout.tile_tokens(first + c) for c in range(count) if c not in chosen]
    if not cand:
        return np.zeros(0, dtype=np.int64)
    toks = np.concatenate(cand)
    sc = scale * (np.asarray(k, dtype=np.float64)[toks] @ qbar_qt)
    order = np.lexsort((toks, -sc))             # score descending, then token index
    return np.sort(toks[order[:n_extra]])


def softmax_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """Textbook softmax(q k^T * scale) v, row by row, in float64."""
    s = scale * (q @ k.T)
    s -= s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return p @ v


def fine_branch_tile(q: np.ndarray, k: np.ndarray, v: np.ndarray, layout: Layout, qt: int,
                     keys: np.ndarray, scale: float) -> np.ndarray:
    """Exact attention of the valid query tokens of tile qt over `keys`.
    Returns [n_valid_queries, D] in the tile's slot order."""
    qtok = layout.tile_tokens(qt)
    return softmax_attention(q[qtok], k[keys], v[keys], scale)


# --------------------------------------------------------------------------- #
# 5. Whole forward pass for one (batch, head) slice
# --------------------------------------------------------------------------- #
@dataclass
class Params:
    mode: int = MODE_TOPK
    keep: float = 0.1
    tau: float = 1.0
    sink: int = SINK_EXACT_KV
    scale: float = 0.0        # 0 -> 1/sqrt(D)
    coarse: int = COARSE_MEAN
    extra_tokens: int = 0     # extra key tokens per query tile (0: none)


@dataclass
class HeadResult:
    qbar: np.ndarray
    kbar: np.ndarray
    vbar: np.ndarray
    scores: np.ndarray
    selected: list
    threshold: float | None
    o_coarse: np.ndarray
    o_fine: np.ndarray | None      # [S, D] (None when only some tiles are computed)
    out: np.ndarray | None         # [S, D]


def selection_for_head(q, k, v, layout: Layout, params: Params):
    """Steps 2-3 for one (batch, head): pooled Q/K/V, scores, selection, coarse."""
    scale = params.scale if params.scale > 0 else default_scale(q.shape[1])
    qbar, kbar, vbar = pool_tiles(q, layout), pool_tiles(k, layout), pool_tiles(v, layout)
    scores = tile_scores(qbar, kbar, layout, scale, params.sink)
    if params.mode == MODE_TOPK:
        sel = select_topk(scores, topk_count(params.keep, candidate_tiles(layout, params.sink)[1]))
        thr = None
    else:
        sel, thr = select_adaptive(scores, params.tau)
    if params.coarse == COARSE_REWEIGHT:
        anchor = video_query_anchor(q, layout)
        kt, vt, bias = reweighted_summaries(k, v, anchor, layout, scale, params.sink)
        o_coarse = coarse_branch_reweighted(qbar, kt, vt, bias, scale)
    else:
        o_coarse = coarse_branch(scores, vbar, layout, params.sink)
    return qbar, kbar, vbar, scores, sel, thr, o_coarse, scale


def output_rows_for_tile(q, k, v, g, layout: Layout, params: Params, qt: int,
                         selected: np.ndarray, o_coarse: np.ndarray, scale: float, extra=None):
    """o_fine and out for the valid query tokens of tile qt.

    out = o_fine + g * o_coarse[qt], g [S] (one gate per token, broadcast over
    the head dimension) or [S, D] (one per channel); under exact_kv_and_rows
    the conditioning query rows get the dense result only (no coarse term;
    reading: they are run dense, and dense attention has no compressed branch).
    `extra`, if given, is the tile's set of extra tokens (instead of the one
    extra_tokens_for_tile chooses). Returns (tokens, o_fine, out).
    """
    keys = key_tokens_for_tile(layout, qt, selected, params.sink)
    if params.extra_tokens > 0 and not (params.sink == SINK_EXACT_KV_AND_ROWS and qt < layout.n_cond_tiles):
        if extra is None:
            qbar_qt = np.asarray(q, dtype=np.float64)[layout.tile_tokens(qt)].mean(axis=0)
            extra = extra_tokens_for_tile(qbar_qt, k, layout, selected, params.extra_tokens, scale, params.sink)
        keys = np.concatenate([keys, np.asarray(extra, dtype=np.int64)])
    of = fine_branch_tile(q, k, v, layout, qt, keys, scale)
    toks = layout.tile_tokens(qt)
    if params.sink == SINK_EXACT_KV_AND_ROWS and qt < layout.n_cond_tiles:
        out = of.copy()
    else:
        gt = np.asarray(g, dtype=np.float64)[toks]
        out = of + (gt if gt.ndim == 2 else gt[:, None]) * o_coarse[qt][None, :]
    return toks, of, out


def vsa_forward_head(q, k, v, g, layout: Layout, params: Params, tiles=None) -> HeadResult:
    """The whole forward pass for one (batch, head) slice.

    q, k, v: [S, D] float64; g: [S] or [S, D] float64. If `tiles` is given, the fine
    branch and output are computed for those query tiles only (rows of other
    tiles are left as NaN).
    """
    qbar, kbar, vbar, scores, sel, thr, o_coarse, scale = selection_for_head(q, k, v, layout, params)
    S, D = q.shape
    o_fine = np.full((S, D), np.nan)
    out = np.full((S, D), np.nan)
    for qt in (range(layout.n_tiles) if tiles is None else tiles):
        toks, of, o = output_rows_for_tile(q, k, v, g, layout, params, qt, sel[qt], o_coarse, scale)
        o_fine[toks] = of
        out[toks] = o
    return HeadResult(qbar, kbar, vbar, scores, sel, thr, o_coarse, o_fine, out)


def dense_attention_masked(q, k, v, mask: np.ndarray, scale: float) -> np.ndarray:
    """Brute-force dense attention over all S keys with a boolean [S, S] mask
    (True = attend), masked logits set to -inf. Independent of the tile
    machinery above; used to check the fine branch."""
    s = scale * (np.asarray(q) @ np.asarray(k).T)
    s = np.where(mask, s, -np.inf)
    s -= s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return p @ np.asarray(v)
