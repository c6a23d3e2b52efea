"""Seeded synthetic workloads: shapes, segment descriptors and input tensors.

This module holds no step of the attention method. It describes the packed
[conditioning prefix | video] sequences the pages run on (text, reference image
and reference audio segments in front of a generated video latent grid) and
draws seeded random inputs of those shapes. Both the CUDA path and the CPU
oracle read the same bf16 bytes from here.

Value model (one per tensor X in Q, K, V): for every (batch, cluster, head) a
vector c ~ N(0, I_D) is drawn once, and every token gets
    X[b, token, h, :] = z + amp * c[b, cluster(token), h, :],   z ~ N(0, I_D),
rounded once from float32 to bf16 (round to nearest even). The cluster of a
token is supplied by the caller (the tests and the benchmark pass the token's
tile), which gives tile-level structure in the scores. The gate is
g ~ U(0, 1) on [B, S, H]. Draws are made per chunk of tokens from PCG64
streams keyed by (seed, tensor, batch, chunk), so generation can run on
several threads and every chunk is reproducible on its own.
"""

from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

SEG_TEXT, SEG_REF_IMAGE, SEG_REF_AUDIO, SEG_OTHER_COND, SEG_VIDEO = 0, 1, 2, 3, 4
MODE_TOPK, MODE_ADAPTIVE = 0, 1
SINK_EXACT_KV, SINK_EXACT_KV_AND_ROWS = 0, 1

CHUNK_TOKENS = 2048


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    cond: tuple            # ((kind, length), ...) in sequence order, before the video
    grid: tuple            # (T, H, W) of the video latent grid
    mode: int = MODE_TOPK
    keep: float = 0.1
    tau: float = 1.0
    sink: int = SINK_EXACT_KV
    amp: float = 1.5
    seed: int = 0
    D: int = 128
    cond_after: tuple = field(default=())   # conditioning segments after the video

    @property
    def n_video(self) -> int:
        t, h, w = self.grid
        return t * h * w

    @property
    def seq_len(self) -> int:
        return (sum(n for _, n in self.cond) + self.n_video
                + sum(n for _, n in self.cond_after))

    def segments(self):
        """[(kind, start, length, (t, h, w) or None), ...] in sequence order."""
        segs, pos = [], 0
        for kind, n in self.cond:
            segs.append((kind, pos, n, None))
            pos += n
        segs.append((SEG_VIDEO, pos, self.n_video, tuple(self.grid)))
        pos += self.n_video
        for kind, n in self.cond_after:
            segs.append((kind, pos, n, None))
            pos += n
        return segs

    def with_(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


_PREFIX_5S = ((SEG_TEXT, 512), (SEG_REF_IMAGE, 48 * 84), (SEG_REF_AUDIO, 128))

WORKLOADS = {
    # B=1, H=2; prefix 32 text + 16 ref-image + 16 ref-audio; 8x8x8 video; keep 50%.
    "tiny": Workload("tiny", B=1, H=2, cond=((SEG_TEXT, 32), (SEG_REF_IMAGE, 16), (SEG_REF_AUDIO, 16)),
                     grid=(8, 8, 8), keep=0.5, amp=1.5, seed=0),
    # B=1, H=24; prefix 512 + 448 + 64; 16x32x32 video; keep 20%.
    "mid": Workload("mid", B=1, H=24, cond=((SEG_TEXT, 512), (SEG_REF_IMAGE, 448), (SEG_REF_AUDIO, 64)),
                    grid=(16, 32, 32), keep=0.2, amp=1.5, seed=1),
    # 1344x768, 5 s: prefix 512 text + 48x84 ref-image + 128 audio; 32x48x84 video; keep 10%.
    "5s": Workload("5s", B=1, H=24, cond=_PREFIX_5S, grid=(32, 48, 84), keep=0.1, amp=2.0, seed=2),
    # 1344x768, 10 s: 61x48x84 video (last temporal tile partial); conditioning rows dense.
    "10s": Workload("10s", B=1, H=24, cond=_PREFIX_5S, grid=(61, 48, 84), keep=0.1,
                    sink=SINK_EXACT_KV_AND_ROWS, amp=2.0, seed=3),
    # 5 s shape with the adaptive per-head threshold (tau in {1.0, 1.5, 2.0}).
    "5s_adaptive": Workload("5s_adaptive", B=1, H=24, cond=_PREFIX_5S, grid=(32, 48, 84),
                            mode=MODE_ADAPTIVE, tau=1.0, amp=2.0, seed=4),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even); returns the uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((u + (((u >> 16) & 1) + np.uint32(0x7FFF))) >> 16).astype(np.uint16)


def _rng(*key) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(list(key)))


def make_inputs(wl: Workload, cluster_of_token: np.ndarray, threads: int = 8):
    """Draw (q, k, v, g) as bf16 bit arrays: q/k/v [B, S, H, D] uint16, g [B, S, H] uint16.

    cluster_of_token: int array [S] with values in [0, n_clusters).
    """
    S, H, D, B = wl.seq_len, wl.H, wl.D, wl.B
    cl = np.asarray(cluster_of_token, dtype=np.int64)
    if cl.shape != (S,) or cl.min() < 0:
        raise ValueError("cluster_of_token must be a non-negative int array of length S")
    n_cl = int(cl.max()) + 1
    n_chunks = -(-S // CHUNK_TOKENS)
    qkv = [np.empty((B, S, H, D), dtype=np.uint16) for _ in range(3)]
    g = np.empty((B, S, H), dtype=np.uint16)
    amp = np.float32(wl.amp)

    centers = {}
    for t in range(3):
        for b in range(B):
            centers[t, b] = _rng(wl.seed, t, b, 1 << 30).standard_normal((n_cl, H, D), dtype=np.float32)

    def fill(job):
        t, b, ch = job
        s0, s1 = ch * CHUNK_TOKENS, min(S, (ch + 1) * CHUNK_TOKENS)
        if t < 3:
            z = _rng(wl.seed, t, b, ch).standard_normal((s1 - s0, H, D), dtype=np.float32)
            z += amp * centers[t, b][cl[s0:s1]]
            qkv[t][b, s0:s1] = f32_to_bf16_bits(z)
        else:
            u = _rng(wl.seed, t, b, ch).random((s1 - s0, H), dtype=np.float32)
            g[b, s0:s1] = f32_to_bf16_bits(u)

    jobs = [(t, b, ch) for t in range(4) for b in range(B) for ch in range(n_chunks)]
    with ThreadPoolExecutor(max(1, threads)) as ex:
        list(ex.map(fill, jobs))
    return qkv[0], qkv[1], qkv[2], g


def make_channel_gate(wl: Workload, threads: int = 8) -> np.ndarray:
    """A per-channel gate g ~ U(0, 1) on [B, S, H, D] as bf16 bits, drawn per
    chunk of tokens from PCG64 streams keyed (seed, 5, batch, chunk)."""
    S, H, D, B = wl.seq_len, wl.H, wl.D, wl.B
    g = np.empty((B, S, H, D), dtype=np.uint16)
    n_chunks = -(-S // CHUNK_TOKENS)

    def fill(job):
        b, ch = job
        s0, s1 = ch * CHUNK_TOKENS, min(S, (ch + 1) * CHUNK_TOKENS)
        g[b, s0:s1] = f32_to_bf16_bits(_rng(wl.seed, 5, b, ch).random((s1 - s0, H, D), dtype=np.float32))

    with ThreadPoolExecutor(max(1, threads)) as ex:
        list(ex.map(fill, [(b, ch) for b in range(B) for ch in range(n_chunks)]))
    return g
