"""Benchmark of the VSA block-sparse attention forward on B200.

One step = one VSA attention call on the 1344x768 5 s shape (133,696 tokens:
4,672 conditioning + 32x48x84 video, H=24, d=128, keep 10%, exact_kv), i.e.
vsa_coarse_select + vsa_sparse_attn_fwd on inputs resident in HBM; the
geometry map is built and uploaded once per shape, outside the timed region.

Metric: effective TFLOP/s of the fine branch's valid work (4 * 128 FLOP per
attended (query, key) pair, x heads), and ms per call. Inputs (2.5 GB) are
larger than L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun), every rank runs its own copy of the workload (weak
scaling, no collective on the data path); timing is the max over ranks.
--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload on the host cores (rank 0 only).
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ms per VSA attention call and effective TFLOP/s (% bf16 peak) at 129k tokens"
WORKLOAD = "5s"
SINKS = {"exact_kv": 0, "exact_kv_and_rows": 1, "off": 2}
COARSES = {"mean": 0, "reweight": 1}


def captured_traffic(workload: str):
    """DRAM bytes per attention call (the sum over the kernels the committed
    counter capture of this workload lists, profiles/vsa_attn_kernel_<workload>_dram.json),
    or None when there is none or the kernel code changed since the counters
    were taken (the capture records the code hash of kernel_code_hash())."""
    path = os.path.join(ROOT, "profiles", "vsa_attn_kernel_%s_dram.json" % workload)
    try:
        with open(path) as f:
            cap = json.load(f)
    except (OSError, ValueError):
        return None
    if cap.get("kernel_code_sha256_16") != kernel_code_hash():
        return None
    return sum(int(k["dram_bytes_read"]) + int(k["dram_bytes_write"]) for k in cap["kernels"].values())


def kernel_code_hash() -> str:
    """sha256 prefix of the attention kernel's code (vsa_attn.cu + sm100.cuh)
    with comments and whitespace removed, so that comment edits keep a capture."""
    import hashlib
    import re
    code = ""
    for f in ("vsa_attn.cu", "sm100.cuh"):
        text = open(os.path.join(ROOT, "block_sparse_video_geometry_b200", "csrc", f)).read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        code += " ".join(text.split()) + "\n"
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def valid_flop_fast(counts, n_cond, idx, cnt, sink_rows, sink_off=False):
    """Valid fine-branch FLOP of one call: 4 * 128 per attended (valid query,
    valid key) pair; keys of a query tile = conditioning tokens + tokens of its
    selected video tiles (all tokens for dense conditioning rows; with the sink
    off, the tokens of its selected tiles only, any tile being a candidate)."""
    counts = counts.astype(np.float64)
    cand = counts if sink_off else counts[n_cond:]
    fixed = 0.0 if sink_off else counts[:n_cond].sum()
    B, H, Nt, kmax = idx.shape
    mask = np.arange(kmax)[None, None, None, :] < cnt[..., None]
    keys = np.where(mask, cand[np.clip(idx, 0, len(cand) - 1)], 0.0).sum(-1) + fixed
    if sink_rows:
        keys[:, :, :n_cond] = counts.sum()
    return 4.0 * 128.0 * float((keys * counts[None, None, :]).sum())


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def describe(wl) -> str:
    names = {0: "text", 1: "ref image", 2: "ref audio", 3: "other"}
    cond = " + ".join("%d %s" % (n, names.get(k, "cond")) for k, n in wl.cond)
    sel = ("keep %g%%" % (100 * wl.keep)) if wl.mode == 0 else ("adaptive tau %g" % wl.tau)
    sink = {0: "exact_kv", 1: "exact_kv_and_rows", 2: "sink off"}[wl.sink]
    return "%s: %s conditioning + %dx%dx%d video tokens (S=%d), B=%d, H=%d, d=%d, %s, %s" % (
        wl.name, cond or "no", *wl.grid, wl.seq_len, wl.B, wl.H, wl.D, sel, sink)


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# --------------------------------------------------------------- CPU oracle
def oracle_sample(wl, bits, lay, head, n_tiles, rng_seed=0, coarse=0):
    """Times the oracle on one head: its whole selection and the fine branch of
    n_tiles query tiles. Returns (seconds, valid FLOP of the sampled fine work,
    seconds extrapolated to one whole call)."""
    from oracle import vsa_oracle as O
    f = O.bf16_bits_to_f64
    q, k, v, g = bits
    t0 = time.perf_counter()
    qh, kh, vh, gh = f(q[0, :, head]), f(k[0, :, head]), f(v[0, :, head]), f(g[0, :, head])
    p = O.Params(mode=wl.mode, keep=wl.keep, tau=wl.tau, sink=wl.sink, coarse=coarse)
    qb, kb, vb, sc, sel, thr, oc, scale = O.selection_for_head(qh, kh, vh, lay, p)
    t_sel = time.perf_counter() - t0
    tiles = np.random.default_rng(rng_seed).choice(lay.n_tiles, n_tiles, replace=False)
    flop = 0.0
    counts = (lay.perm >= 0).sum(1)
    t1 = time.perf_counter()
    for qt in tiles:
        keys = O.key_tokens_for_tile(lay, int(qt), sel[qt], p.sink)
        O.output_rows_for_tile(qh, kh, vh, gh, lay, p, int(qt), sel[qt], oc, scale)
        flop += 4.0 * 128 * counts[qt] * keys.size
    t_fine = time.perf_counter() - t1
    secs = t_sel * n_tiles / lay.n_tiles + t_fine
    per_call = (t_sel + t_fine * lay.n_tiles / n_tiles) * wl.H
    return secs, flop, per_call


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(n[0]) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from block_sparse_video_geometry_b200 import workloads as W
    from oracle import vsa_oracle as O
    wl = W.WORKLOADS[args.workload]
    if args.sink is not None:
        wl = wl.with_(sink=SINKS[args.sink])
    lay = O.build_layout([O.Segment(k, s, n, gr) for (k, s, n, gr) in wl.segments()], wl.seq_len)
    bits = W.make_inputs(wl, lay.inv // O.TILE)
    if args.gate == "channel":
        bits = bits[:3] + (W.make_channel_gate(wl),)
    n_tiles = args.ref_tiles
    for i in range(args.warmup):
        oracle_sample(wl, bits, lay, head=i % wl.H, n_tiles=max(2, n_tiles // 4), rng_seed=i,
                      coarse=COARSES[args.coarse])
    secs, flops = 0.0, 0.0
    per_call = []
    for i in range(args.steps):
        s, fl, pc = oracle_sample(wl, bits, lay, head=(i * 7) % wl.H, n_tiles=n_tiles, rng_seed=100 + i,
                                  coarse=COARSES[args.coarse])
        secs += s
        flops += fl
        per_call.append(pc)
    tflops = flops / secs / 1e12
    ms_call = 1e3 * statistics.mean(per_call)
    sample = ("one head per step: its whole selection (pool, scores, top-k, coarse) pro rata plus the fine "
              "branch of %d random query tiles; ms_per_step extrapolated to a whole call (24 heads)" % n_tiles)
    line = {"impl": "reference", "metric": METRIC, "value": tflops, "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_call, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": describe(wl) + ", %s coarse, %s gate, %s output" % (args.coarse, args.gate, args.out_dtype), "B": wl.B,
                       "seq_len": wl.seq_len, "parallelism": "host cores",
                       "l2": "inputs (2.5 GB) larger than L2; no flush"},
            "cpu_baseline": {"value": tflops, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": tflops, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


# -------------------------------------------------------------- GPU arm
def time_calls(stream, select_fn, attn_fn, n):
    """Median ms of the selection call and of the attention call over n calls
    (CUDA events on the launching stream), plus the sorted whole-call times."""
    import torch
    sel, att = [], []
    for _ in range(n):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record(stream)
        select_fn()
        e[1].record(stream)
        attn_fn()
        e[2].record(stream)
        torch.cuda.synchronize()
        sel.append(e[0].elapsed_time(e[1]))
        att.append(e[1].elapsed_time(e[2]))
    calls = sorted(a + b for a, b in zip(sel, att))
    return statistics.median(sel), statistics.median(att), calls


def dense_sdpa_ms(stream, q, k, v, n=3):
    """torch scaled_dot_product_attention on the same Q, K, V (a library kernel,
    timed for context: the method replaces it); None if it cannot run."""
    import torch
    try:
        qd, kd, vd = (x.transpose(1, 2) for x in (q, k, v))      # [B, H, S, 128] views
        with torch.cuda.stream(stream):
            for _ in range(2):
                torch.nn.functional.scaled_dot_product_attention(qd, kd, vd)
            d_ms = []
            for _ in range(n):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                torch.nn.functional.scaled_dot_product_attention(qd, kd, vd)
                e1.record(stream)
                torch.cuda.synchronize()
                d_ms.append(e0.elapsed_time(e1))
        return statistics.median(d_ms)
    except RuntimeError as ex:   # e.g. out of memory on a smaller GPU
        print("dense comparator skipped: %s" % ex, file=sys.stderr)
        return None
    finally:
        torch.cuda.empty_cache()


def check_failures(fwd, stream, where):
    from block_sparse_video_geometry_b200 import vsa
    n = vsa.sparse_attn_failed_calls(fwd.ws_attn, stream)
    if n:
        raise RuntimeError("%s: %d attention call(s) reported a kernel error" % (where, n))


def measure_config(name, wl, params, q, k, v, g, dev, stream, out_dtype, peak, n_calls, dense=None,
                   inputs_note=None):
    """One extra workload of the same run: ms per call (selection + attention),
    valid TFLOP/s, the attention kernel's fraction of the burst bf16 peak, the
    kept fraction of candidate tiles, and the dense comparator where given."""
    import torch
    from block_sparse_video_geometry_b200 import vsa
    lay = vsa.Layout(wl.segments(), wl.seq_len)
    perm, inv, counts, kinds = lay.tables()
    with torch.cuda.stream(stream):
        fwd = vsa.Forward(lay, params, wl.B, wl.H, device=dev, out_dtype=out_dtype, stream=stream)
        out = torch.empty(q.shape, dtype=out_dtype, device=dev)
    sel_fn, att_fn = call_fns(vsa, lay, params, fwd, q, k, v, g, out, stream)
    for _ in range(3):
        sel_fn()
        att_fn()
    torch.cuda.synchronize()
    idx, cnt = fwd.idx.cpu().numpy(), fwd.cnt.cpu().numpy()
    flop = valid_flop_fast(counts, lay.info.n_cond_tiles, idx, cnt, wl.sink == vsa.SINK_EXACT_KV_AND_ROWS,
                           wl.sink == vsa.SINK_OFF)
    if params.extra_tokens > 0:
        flop += valid_flop_extra(counts, fwd.extra_cnt.cpu().numpy(), wl.sink == vsa.SINK_EXACT_KV_AND_ROWS,
                                 lay.info.n_cond_tiles)
    sel_ms, att_ms, calls = time_calls(stream, sel_fn, att_fn, n_calls)
    check_failures(fwd, stream, name)
    call_ms = statistics.median(calls)
    n_cand = lay.info.n_tiles if wl.sink == vsa.SINK_OFF else lay.info.n_video_tiles
    res = {"workload": describe(wl), "ms_per_call": call_ms, "select_ms": sel_ms, "attn_ms": att_ms,
           "valid_tflop": flop / 1e12, "tflops_per_call": flop / (call_ms * 1e-3) / 1e12,
           "attn_tflops": flop / (att_ms * 1e-3) / 1e12, "attn_frac_of_burst": flop / (att_ms * 1e-3) / 1e12 / peak,
           "kept_fraction": float(cnt.mean()) / n_cand, "calls": n_calls}
    if inputs_note:
        res["inputs"] = inputs_note
    if dense is not None:
        res["dense_sdpa_ms"] = dense
        res["speedup_vs_dense"] = dense / call_ms
    del fwd, out
    torch.cuda.empty_cache()
    return res


def call_fns(vsa, lay, params, fwd, q, k, v, g, out, stream):
    """The two timed halves of one call: selection (plus the extra-token
    choice when params.extra_tokens > 0) and attention."""
    def select():
        vsa.coarse_select(lay, params, q, k, v, fwd.idx, fwd.cnt, fwd.o_coarse, fwd.ws_select, stream)
        if params.extra_tokens > 0:
            vsa.extra_tokens_select(lay, params, q, k, fwd.idx, fwd.cnt, fwd.kmax, fwd.extra_idx, fwd.extra_cnt,
                                    fwd.ws_extra, stream)

    def attend():
        vsa.sparse_attn_fwd(lay, params, q, k, v, g, fwd.idx, fwd.cnt, fwd.kmax, fwd.o_coarse, out, fwd.ws_attn,
                            stream, fwd.extra_idx, fwd.extra_cnt)
    return select, attend


def valid_flop_extra(counts, extra_cnt, rows_dense, n_cond):
    """FLOP of the extra-token key step: 4 * 128 per (valid query, extra token)."""
    e = extra_cnt.astype(np.float64)
    if rows_dense:
        e[:, :, :n_cond] = 0
    return 4.0 * 128.0 * float((e * counts[None, None, :].astype(np.float64)).sum())


def measure_backward(wl, params, q, k, v, g, dev, stream, n_calls, fwd_flop):
    """vsa_sparse_attn_bwd on the inputs of this run (a seeded dO): ms per call.
    Its tensor work is 7 products of 64 x 64 x 128 per (query tile, key tile)
    pair (S, dP and dQ per query tile; S^T, dP^T, dK and dV per key tile)
    against the forward's 2, so the executed-work rate counts 3.5 x the
    forward's valid FLOP."""
    import torch
    from block_sparse_video_geometry_b200 import vsa
    lay = vsa.Layout(wl.segments(), wl.seq_len)
    with torch.cuda.stream(stream):
        fwd = vsa.Forward(lay, params, wl.B, wl.H, device=dev, stream=stream)
        gen = torch.Generator(device=dev).manual_seed(77)
        dout = torch.randn(q.shape, generator=gen, device=dev).to(torch.bfloat16)
        grads = [torch.empty(q.shape, dtype=torch.float32, device=dev) for _ in range(3)]
        dg = torch.empty(g.shape, dtype=torch.float32, device=dev)
        ws = torch.empty(lay.sparse_attn_bwd_workspace_size(wl.B, wl.H, params), dtype=torch.uint8, device=dev)
    vsa.coarse_select(lay, params, q, k, v, fwd.idx, fwd.cnt, fwd.o_coarse, fwd.ws_select, stream)
    bwd = lambda: vsa.sparse_attn_bwd(lay, params, q, k, v, g, fwd.idx, fwd.cnt, fwd.kmax, fwd.o_coarse, dout,
                                      *grads, dg, ws, stream)
    for _ in range(2):
        bwd()
    ms = []
    for _ in range(n_calls):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        bwd()
        e1.record(stream)
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    if vsa.sparse_attn_bwd_status(ws, stream) != vsa.OK:
        raise RuntimeError("backward: a kernel wait ran out")
    t = statistics.median(ms)
    res = {"workload": describe(wl) + ", backward", "ms_per_call": t,
           "tflops_executed": 3.5 * fwd_flop / (t * 1e-3) / 1e12, "calls": n_calls,
           "flop_accounting": "3.5 x the forward's valid FLOP (7 tile products per attended pair vs 2)",
           "dout": "seeded N(0, 1) in bf16"}
    del fwd, dout, grads, dg, ws
    torch.cuda.empty_cache()
    return res


def run_ours(args):
    import torch
    from block_sparse_video_geometry_b200 import vsa, workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    from block_sparse_video_geometry_b200 import sharding
    wl = W.WORKLOADS[args.workload].with_(seed=sharding.replica_seed(W.WORKLOADS[args.workload].seed, rank))
    if args.sink is not None:
        wl = wl.with_(sink=SINKS[args.sink])
    if args.heads is not None:                   # --profile-call runs only (checked in main)
        wl = wl.with_(H=args.heads)
    lay = vsa.Layout(wl.segments(), wl.seq_len)
    perm, inv, counts, kinds = lay.tables()
    bits = W.make_inputs(wl, inv // vsa.TILE)
    if args.gate == "channel":
        bits = bits[:3] + (W.make_channel_gate(wl),)
    to_dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
    q, k, v, g = (to_dev(x) for x in bits)
    stream = torch.cuda.Stream(device=dev)
    out_dtype = torch.float32 if args.out_dtype == "f32" else torch.bfloat16
    params = vsa.make_params(mode=wl.mode, keep=wl.keep, tau=wl.tau, sink=wl.sink, coarse=COARSES[args.coarse],
                             extra_tokens=args.extra_tokens)
    with torch.cuda.stream(stream):
        fwd = vsa.Forward(lay, params, wl.B, wl.H, device=dev, out_dtype=out_dtype, stream=stream)
        out = torch.empty(q.shape, dtype=out_dtype, device=dev)
    torch.cuda.synchronize()
    peaks, src = measured_peaks()
    peak = peaks["bf16_tflops"]
    select, attend = call_fns(vsa, lay, params, fwd, q, k, v, g, out, stream)

    def step():
        select()
        attend()

    if args.profile_call is not None:
        # warmup + steps calls of one entry point and nothing timed: the run a
        # kernel profiler captures (the backward and the token ranking are not
        # in the headline step)
        if args.profile_call == "backward":
            gen = torch.Generator(device=dev).manual_seed(77)
            dout = torch.randn(q.shape, generator=gen, device=dev).to(torch.bfloat16)
            grads = [torch.empty(q.shape, dtype=torch.float32, device=dev) for _ in range(3)]
            dg = torch.empty(g.shape, dtype=torch.float32, device=dev)
            ws = torch.empty(lay.sparse_attn_bwd_workspace_size(wl.B, wl.H, params), dtype=torch.uint8, device=dev)
            select()
            call = lambda: vsa.sparse_attn_bwd(lay, params, q, k, v, g, fwd.idx, fwd.cnt, fwd.kmax, fwd.o_coarse,
                                               dout, *grads, dg, ws, stream)

            def check():
                if vsa.sparse_attn_bwd_status(ws, stream) != vsa.OK:
                    raise RuntimeError("backward: a kernel wait ran out")
        else:
            call = select if args.profile_call == "select" else step

            def check():
                check_failures(fwd, stream, "profiled calls")
                if vsa.coarse_select_status(fwd.ws_select, stream) != vsa.OK or (
                        args.extra_tokens > 0 and vsa.extra_tokens_status(fwd.ws_extra, stream) != vsa.OK):
                    raise RuntimeError("profiled calls: a selection kernel wait ran out")
        for _ in range(args.warmup + args.steps):
            call()
        torch.cuda.synchronize()
        check()
        print(json.dumps({"profile_call": args.profile_call, "workload": args.workload,
                          "extra_tokens": args.extra_tokens, "calls": args.warmup + args.steps}), flush=True)
        return

    for _ in range(args.warmup):
        step()
    check_failures(fwd, stream, "warm-up")
    flop = valid_flop_fast(counts, lay.info.n_cond_tiles, fwd.idx.cpu().numpy(), fwd.cnt.cpu().numpy(),
                           wl.sink == vsa.SINK_EXACT_KV_AND_ROWS, wl.sink == vsa.SINK_OFF)
    if args.extra_tokens > 0:
        flop += valid_flop_extra(counts, fwd.extra_cnt.cpu().numpy(), wl.sink == vsa.SINK_EXACT_KV_AND_ROWS,
                                 lay.info.n_cond_tiles)

    def barrier():
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()

    # ---- headline: K whole steps, device-timed on the launching stream
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        barrier()
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        barrier()
    ms_step = ev0.elapsed_time(ev1) / args.steps
    check_failures(fwd, stream, "timed steps")

    # ---- per-kernel split: selection call vs attention call, events on the same stream
    sel_ms, att_ms, call_ms = time_calls(stream, select, attend, max(3, min(args.steps, 10)))
    check_failures(fwd, stream, "per-call timing")
    call_p50 = statistics.median(call_ms)
    call_p90 = call_ms[min(len(call_ms) - 1, int(round(0.9 * (len(call_ms) - 1))))]

    dense_ms = None if args.no_dense else dense_sdpa_ms(stream, q, k, v)

    # ---- end to end through the public API with host buffers. Every step copies its inputs host ->
    # device and reads its output back inside the timed region; the copies overlap the neighbouring
    # steps' compute (step i's inputs travel while step i - 1 computes, its output comes back while
    # step i + 1 computes), with two device input and two device output buffers.
    host_in = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in bits]
    host_out = torch.empty(out.shape, dtype=out_dtype).pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in host_in)
    d2h = host_out.numel() * host_out.element_size()
    e2e_steps = max(3, min(args.steps, 10))
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    dev_in = [(q, k, v, g), tuple(torch.empty_like(x) for x in (q, k, v, g))]
    dev_out = [out, torch.empty_like(out)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    e2e_start, e2e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    e2e_start.record(s_in)
    for i in range(e2e_steps):
        bsel = i & 1
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_done[bsel])          # step i - 2 is done with these inputs
            for hsrc, ddst in zip(host_in, dev_in[bsel]):
                ddst.copy_(hsrc, non_blocking=True)
            ev_in[bsel].record(s_in)
        stream.wait_event(ev_in[bsel])
        if i >= 2:
            stream.wait_event(ev_out[bsel])              # the output of step i - 2 has been read back
        qq, kk, vv, gg = dev_in[bsel]
        s_fn, a_fn = call_fns(vsa, lay, params, fwd, qq, kk, vv, gg, dev_out[bsel], stream)
        s_fn()
        a_fn()
        ev_done[bsel].record(stream)
        s_out.wait_event(ev_done[bsel])
        with torch.cuda.stream(s_out):
            host_out.copy_(dev_out[bsel], non_blocking=True)
            ev_out[bsel].record(s_out)
    e2e_end.record(s_out)
    barrier()
    ms_e2e = e2e_start.elapsed_time(e2e_end) / e2e_steps
    check_failures(fwd, stream, "end-to-end steps")
    del dev_in, dev_out, host_in, host_out

    # ---- the other configurations of the same shapes, measured in the same run (rank 0, one GPU)
    configs = None
    if world == 1 and not args.no_configs and args.workload == "5s" and args.sink is None \
            and args.coarse == "mean" and args.gate == "token" and args.extra_tokens == 0:
        configs = {}
        n = args.config_calls
        mk = lambda **kw: vsa.make_params(**dict(dict(mode=0, keep=0.1, tau=1.0, sink=0, coarse=0, extra_tokens=0),
                                                 **kw))
        note = "the 5 s inputs of this run (seed %d)" % wl.seed
        for tau in (1.0, 1.5, 2.0):
            configs["5s_adaptive_tau%g" % tau] = measure_config(
                "adaptive tau %g" % tau, wl.with_(mode=vsa.SELECT_ADAPTIVE, tau=tau),
                mk(mode=vsa.SELECT_ADAPTIVE, tau=tau), q, k, v, g, dev, stream, out_dtype, peak, n,
                inputs_note=note)
        configs["5s_extra_tokens16"] = measure_config(
            "extra tokens 16", wl, mk(extra_tokens=16), q, k, v, g, dev, stream, out_dtype, peak, max(3, n // 2),
            inputs_note=note)
        configs["5s_backward"] = measure_backward(wl, mk(), q, k, v, g, dev, stream, max(3, n // 2), flop)
        configs["5s_keep100"] = measure_config("keep 100%", wl.with_(keep=1.0), mk(keep=1.0), q, k, v, g, dev,
                                               stream, out_dtype, peak, max(3, n // 2), dense=dense_ms,
                                               inputs_note=note)
        del q, k, v, g, out
        fwd = None
        torch.cuda.empty_cache()
        w10 = W.WORKLOADS["10s"]
        lay10 = vsa.Layout(w10.segments(), w10.seq_len)
        b10 = W.make_inputs(w10, lay10.tables()[1] // vsa.TILE)
        q10, k10, v10, g10 = (to_dev(x) for x in b10)
        del b10
        d10 = None if args.no_dense else dense_sdpa_ms(stream, q10, k10, v10, n=2)
        configs["10s_ragged_rows_dense"] = measure_config(
            "10 s", w10, mk(sink=vsa.SINK_EXACT_KV_AND_ROWS), q10, k10, v10, g10, dev, stream, out_dtype, peak,
            max(3, n // 2), dense=d10)
        del q10, k10, v10, g10
        torch.cuda.empty_cache()

    ms_step, ms_e2e, att_ms, sel_ms = sharding.max_over_ranks([ms_step, ms_e2e, att_ms, sel_ms], dist, dev)
    job_flop, = sharding.sum_over_ranks([flop], dist, dev)   # the work of every replica

    if rank == 0:
        achieved = flop / (att_ms * 1e-3) / 1e12
        info = lay.info
        # algorithmic bytes of the selection call: Q, K, V read once, idx, cnt and o_coarse written
        sel_bytes = 3 * wl.B * wl.seq_len * wl.H * 128 * 2 + 4 * wl.B * wl.H * info.n_tiles * (
            lay.kmax(params) + 1 + 128)
        value = job_flop / (ms_step * 1e-3) / 1e12
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": describe(wl) + ", %s coarse, %s gate, %s output%s" % (
                args.coarse, args.gate, args.out_dtype,
                ", %d extra tokens" % args.extra_tokens if args.extra_tokens else ""),
                       "B": wl.B, "seq_len": wl.seq_len, "parallelism": "replica per GPU" if world > 1 else "1 GPU",
                       "l2": "inputs (2.5 GB) larger than L2; no flush"},
            "roofline": {"bound": "tensor", "kernel": "vsa_sparse_attn_fwd (pair_attn_kernel + vsa_attn_kernel)",
                         "achieved": achieved, "peak": peak,
                         "unit": "TFLOP/s", "frac": achieved / peak,
                         "traffic": (captured_traffic(args.workload) if args.sink is None and args.coarse == "mean"
                                     and args.gate == "token" and args.out_dtype == "f32" else None),
                         "traffic_unit": "bytes per call (ncu dram read + write of the two attention kernels)",
                         "peak_source": "%s bf16_tflops (burst: the kernel is timed alone, once per call)" % src,
                         "frac_of_sustained": achieved / peaks.get("bf16_tflops_sustained", peak),
                         "flop_per_launch": flop, "ms_per_launch": att_ms},
            "selection": {"bound": "hbm", "achieved": sel_bytes / (sel_ms * 1e-3) / 1e9,
                          "peak": peaks["hbm_gbs"], "unit": "GB/s",
                          "frac": sel_bytes / (sel_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                          "bytes_per_call": sel_bytes, "ms_per_call": sel_ms},
            "e2e": {"value": job_flop / (ms_e2e * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e,
                    "steps": e2e_steps, "copies": "overlap the neighbouring steps' compute"},
            "gpu_launches": launches_per_call(wl.B, args.coarse, wl.sink != vsa.SINK_OFF and lay.info.n_cond_tiles > 0,
                                              args.extra_tokens > 0) * args.steps * world,
            "clocks": clocks.summary(),
            "call_ms": {"p50": call_p50, "p90": call_p90, "samples": len(call_ms)},
            "dense_sdpa": None if dense_ms is None else {
                "ms": dense_ms, "call_speedup": dense_ms / call_p50,
                "what": "torch scaled_dot_product_attention, bf16, same Q, K, V, no mask"},
        }
        if configs:
            line["configs"] = configs
        if world == 1 and not args.no_cpu_baseline:
            from oracle import vsa_oracle as O
            olay = O.build_layout([O.Segment(k_, s_, n_, g_) for (k_, s_, n_, g_) in wl.segments()], wl.seq_len)
            secs, fl, per_call = oracle_sample(wl, bits, olay, head=0, n_tiles=args.ref_tiles,
                                               coarse=COARSES[args.coarse])
            line["cpu_baseline"] = {"value": fl / secs / 1e12, "unit": "TFLOP/s", "cores": cpu_threads(),
                                    "kind": "oracle", "ms_per_call_extrapolated": per_call * 1e3,
                                    "sample": "head 0: whole selection pro rata + fine branch of %d random "
                                              "query tiles" % args.ref_tiles}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def launches_per_call(B: int, coarse: str, pair_pass: bool, extra: bool) -> int:
    """Kernels this library launches per call: selection (pool, coarse, select;
    anchor and reweight with Spark-Reweight; permute K, pool Q and the token
    ranking with extra tokens) and attention (permute, schedule, the pair pass
    and the sparse pass per batch, plus the extra-token gather)."""
    sel = 3 + (2 if coarse == "reweight" else 0) + (3 if extra else 0)
    return sel + 2 + (1 if extra else 0) + B * (2 if pair_pass else 1)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--out-dtype", choices=["f32", "bf16"], default="f32")
    ap.add_argument("--sink", choices=sorted(SINKS), default=None,
                    help="override the workload's sink_conditioning mode")
    ap.add_argument("--gate", choices=["token", "channel"], default="token",
                    help="gate g[B,S,H] (one per token and head) or g[B,S,H,128] (one per channel)")
    ap.add_argument("--coarse", choices=sorted(COARSES), default="mean",
                    help="compressed-branch summaries: mean pooling or Spark-Reweight")
    ap.add_argument("--extra-tokens", type=int, default=0,
                    help="extra_tokens E (0..64): the E best tokens beyond each query tile's selected tiles")
    ap.add_argument("--ref-tiles", type=int, default=48)
    ap.add_argument("--heads", type=int, default=None,
                    help="with --profile-call: the workload with this many heads (a smaller launch to capture)")
    ap.add_argument("--profile-call", choices=["step", "select", "backward"], default=None,
                    help="only run warmup + steps calls of one entry point (selection incl. the token ranking, "
                         "the whole step, or the backward) for a kernel profiler; prints no bench line")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true", help="skip the torch SDPA comparator")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other configurations (5 s adaptive tau, keep 100%%, 10 s ragged)")
    ap.add_argument("--config-calls", type=int, default=10, help="timed calls per extra configuration")
    args = ap.parse_args()
    if args.heads is not None and args.profile_call is None:
        ap.error("--heads only sizes --profile-call runs; the bench line keeps the workload's heads")
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
