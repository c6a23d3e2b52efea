"""Plain fp64 CPU oracle of the VSA forward's gradients (backward pass).

TEST INFRASTRUCTURE, like vsa_oracle: only the test suite, smoke() and the
benchmark's CPU legs may use it; the product path never does.

What it computes: for one (batch, head) slice and an upstream gradient dout,
the gradients of sum(out * dout) with respect to q, k, v and the gate g. The
block selection (and any extra tokens) is a piecewise-constant function of
the inputs and is held fixed: its derivative is zero wherever it is defined
(reading; the pages train and distil against these modes, "BSAI FastH3
Native VSA (recipe)" and "ComfyUI Agrega Nodo Central ...", without
differentiating the choice of blocks). Everything else (pooling, the coarse
softmax, the exact attention of the fine branch, the gate) is differentiated
exactly.

The forward is restated in PyTorch fp64 CPU ops with the selection taken from
vsa_oracle, and differentiated by autograd (a library primitive); the tests
pin it to central finite differences of vsa_oracle's numpy forward and, for
keep = 100%, to the closed-form attention backward.
"""

from __future__ import annotations

import numpy as np

from oracle import vsa_oracle as O


def _key_mask(layout, params, selected, q, k, scale):
    """Boolean [S, S]: query token i attends key token j (the fine branch's sets)."""
    S = layout.seq_len
    mask = np.zeros((S, S), dtype=bool)
    qn = np.asarray(q, dtype=np.float64)
    for qt in range(layout.n_tiles):
        rows = layout.tile_tokens(qt)
        keys = O.key_tokens_for_tile(layout, qt, selected[qt], params.sink)
        if params.extra_tokens > 0 and not (params.sink == O.SINK_EXACT_KV_AND_ROWS and qt < layout.n_cond_tiles):
            keys = np.concatenate([keys, O.extra_tokens_for_tile(qn[rows].mean(axis=0), k, layout, selected[qt],
                                                                 params.extra_tokens, scale, params.sink)])
        mask[np.ix_(rows, keys)] = True
    return mask


def forward_torch(q, k, v, g, layout, params, selected):
    """The forward of one (batch, head) in torch fp64 with a fixed selection.
    q, k, v: [S, D] tensors; g: [S] or [S, D]. Returns out [S, D]."""
    import torch
    scale = params.scale if params.scale > 0 else O.default_scale(q.shape[1])
    S = layout.seq_len
    tile_of = torch.as_tensor(layout.inv // O.TILE)
    # pooling matrix: row t holds 1 / n_t at the valid tokens of tile t
    pool = torch.zeros(layout.n_tiles, S, dtype=torch.float64)
    for t in range(layout.n_tiles):
        toks = torch.as_tensor(layout.tile_tokens(t))
        pool[t, toks] = 1.0 / len(toks)
    qbar, kbar, vbar = pool @ q, pool @ k, pool @ v
    first, count = O.candidate_tiles(layout, params.sink)
    if params.coarse == O.COARSE_REWEIGHT:
        vid = torch.cat([torch.as_tensor(layout.tile_tokens(t)) for t in range(layout.n_cond_tiles, layout.n_tiles)])
        anchor = q[vid].mean(0)
        kt, vt, b = [], [], []
        for c in range(count):
            toks = torch.as_tensor(layout.tile_tokens(first + c))
            x = scale * (k[toks] @ anchor)
            w = torch.softmax(x, 0)
            kt.append(w @ k[toks])
            vt.append(w @ v[toks])
            b.append(torch.logsumexp(x, 0) - np.log(len(toks)) - scale * (anchor @ kt[-1]))
        kt, vt, b = torch.stack(kt), torch.stack(vt), torch.stack(b)
        o_coarse = torch.softmax(scale * qbar @ kt.T + b[None, :], 1) @ vt
    else:
        o_coarse = torch.softmax(scale * qbar @ kbar[first:first + count].T, 1) @ vbar[first:first + count]
    mask = torch.as_tensor(_key_mask(layout, params, selected, q.detach().numpy(), k.detach().numpy(), scale))
    s = (scale * q @ k.T).masked_fill(~mask, float("-inf"))
    o_fine = torch.softmax(s, 1) @ v
    gate = g if g.dim() == 2 else g[:, None]
    coarse_rows = torch.ones(S, 1, dtype=torch.float64)
    if params.sink == O.SINK_EXACT_KV_AND_ROWS:
        coarse_rows[torch.as_tensor(layout.cond_tokens())] = 0.0
    return o_fine + coarse_rows * gate * o_coarse[tile_of]


def vsa_backward_head(q, k, v, g, dout, layout, params):
    """(dq, dk, dv, dg) of sum(out * dout) for one (batch, head) slice, the
    selection held fixed; numpy float64 in and out (g and dg: [S] or [S, D])."""
    import torch
    sel = O.selection_for_head(q, k, v, layout, params)[4]
    t = [torch.tensor(np.asarray(x, dtype=np.float64), requires_grad=True) for x in (q, k, v, g)]
    out = forward_torch(*t, layout, params, sel)
    (out * torch.as_tensor(np.asarray(dout, dtype=np.float64))).sum().backward()
    return tuple(x.grad.numpy() for x in t)
