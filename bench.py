"""Benchmark of the QSA hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl qsa|reference] [--no-decode] [--no-e2e]

One step = the whole hot path over one batch of synthetic input:
  prefill (the headline, 131072 tokens, 16 q / 2 KV heads, D 128, 4x64 indexer, k 512 + own block):
    pool indexer keys -> score + top-k (chunked scores in a workspace) -> gather-sparse attention;
  decode (second leg, 32 sequences x 262144-token caches, k 512): pool the newest block ->
    score + top-k over the pooled-key cache -> split-KV sparse attention + merge.
Inputs are resident in HBM when the timed region starts and are larger than L2 (126 MB), so no L2
flush is done between steps.  Times are CUDA events on the launching stream, max over ranks.
With N > 1 the ranks share one job (strong scaling): the prefill's query rows are sharded in
zig-zag chunks with one all-gather of K, V and the pooled keys per step (shard.py), and the decode
batch is split by sequence.  ``--impl reference`` times the CPU oracle on a bounded sample of the
same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from hybrid_sparse_attention_qsa_b200 import inputs as I  # noqa: E402

METRIC = "QSA prefill tokens/s @128K and decode tokens/s @256K ctx; % of roofline"
PREFILL = "prefill_128k"
DECODE = "decode_256k"
# Committed ncu summaries that carry the DRAM bytes of one attention launch: the summary records
# `traffic_bytes_per_launch` (dram__bytes_read.sum + dram__bytes_write.sum of one capture) and the
# sha256 of the kernel source it was taken on (`source_sha256`); once the source differs, the bench
# line reports traffic as null until the kernel is captured again.
TRAFFIC_PROFILES = {"prefill_128k": ("profiles/sparse_attn_prefill_128k.md",
                                     "hybrid_sparse_attention_qsa_b200/csrc/sparse_attn.cu")}
# The attention's gather: K and V interleaved by block, every selected 4-token block is one chunk of
# 2 * blk * Hkv * D * 2 bytes (its K then its V), fetched by 8 issuing warps into a 3-stage ring of
# 16 slots: 48 chunks of 4 KB in flight.
GATHER_PROBE = dict(issuer_warps=8, stages=3, slots_per_warp=2)


# ------------------------------------------------------------------------------------------- helpers
def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=p["hbm_gbs"], bf16_tflops=p["bf16_tflops"],
                    bf16_tflops_sustained=p.get("bf16_tflops_sustained", p["bf16_tflops"]), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def tokens_attended(T: int, k: int, blk: int = 4) -> np.ndarray:
    """|S(t)| = blk * min(t // blk, k) + t % blk + 1 for t = 0 .. T-1."""
    t = np.arange(T, dtype=np.int64)
    return blk * np.minimum(t // blk, k) + t % blk + 1


def prefill_work(w) -> dict:
    """Algorithmic work of one prefill step (per batch element times B)."""
    S = tokens_attended(w.T, w.k, w.blk)
    gathered = int(S.sum()) * w.Hkv * w.D * 2 * 2            # K and V bytes gathered
    qo = w.T * w.Hq * w.D * 2 * 2                             # q read + o written
    attn_bytes = (gathered + qo) * w.B
    attn_flops = int(S.sum()) * w.Hq * 4 * w.D * w.B
    pairs = int((np.arange(w.T) // w.blk).sum())             # causally visible (t, block) pairs
    idx_flops = pairs * 2 * w.Hi * w.Di * w.B
    return dict(attn_bytes=attn_bytes, attn_flops=attn_flops, index_flops=idx_flops, pairs=pairs * w.B)


def profile_traffic(workload: str):
    """DRAM bytes per attention launch from the committed ncu summary, or None when there is none or
    the kernel source has changed since it was taken."""
    import hashlib
    ent = TRAFFIC_PROFILES.get(workload)
    if ent is None:
        return None, None
    prof, src = (os.path.join(ROOT, p) for p in ent)
    try:
        text = open(prof).read()
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    except OSError:
        return None, None
    vals = dict(line.strip("`* ").split(":", 1) for line in text.splitlines()
                if line.strip("`* ").startswith(("traffic_bytes_per_launch:", "source_sha256:")))
    if vals.get("source_sha256", "").strip() != sha or "traffic_bytes_per_launch" not in vals:
        return None, ent[0]
    return float(vals["traffic_bytes_per_launch"]), ent[0]


def unique_kv_bytes(w) -> int:
    """Compulsory bytes of the attention: every K/V row that some query attends (here every row
    but none twice), q read once, o written once."""
    return w.B * w.T * (w.Hkv * w.D * 2 * 2 + w.Hq * w.D * 2 * 2)


def gather_ceiling(dev, stream, w, sweep: bool = False) -> dict:
    """The measured ceiling of the attention's gather: 1-D bulk copies of one block of K and V (4 KB,
    the interleaved layout the kernel reads) from random offsets of an L2-resident 32 MiB buffer into
    the same ring the attention kernel keeps in flight, and of a 4 GiB buffer (HBM); for comparison
    the same ring in 2 KB chunks (K and V of a block fetched separately, 8 and 4 warps) and with
    plain loads.  GB/s of delivered bytes, best of 3 timed launches."""
    import hybrid_sparse_attention_qsa_b200 as Q
    if kv_interleaved(w):
        chunk, cfg0 = 2 * w.blk * w.Hkv * w.D * 2, dict(GATHER_PROBE)
        half = dict(issuer_warps=8, stages=3, slots_per_warp=4, chunk_bytes=chunk // 2)
        half4 = dict(issuer_warps=4, stages=3, slots_per_warp=8, chunk_bytes=chunk // 2)
        extra = [("l2_bulk_half", 32 << 20, 0, half), ("l2_bulk_half_w4", 32 << 20, 0, half4)]
    else:   # the wide kernel: K and V blocks fetched separately by 4 warps, 8 slots a stage
        chunk, cfg0 = w.blk * w.Hkv * w.D * 2, dict(issuer_warps=4, stages=3, slots_per_warp=4)
        extra = []
    res = {"chunk_bytes": chunk, "config": dict(cfg0)}
    cases = [("l2_bulk", 32 << 20, 0, cfg0)] + extra + [("hbm_bulk", 4 << 30, 0, cfg0),
                                                        ("l2_lsu", 32 << 20, 1, cfg0)]
    if sweep:
        for iw, sl in ((1, 32), (2, 16), (8, 4), (8, 3), (12, 2), (16, 2)):
            cfg = dict(issuer_warps=iw, stages=3, slots_per_warp=sl)
            cases.append((f"l2_bulk_w{iw}_s{sl}", 32 << 20, 0, cfg))
        # smaller pieces: bulk copies of 512 B and tiled tensor boxes of 512 B / 1 KB
        for iw, sl in ((1, 32), (4, 32), (8, 16), (16, 8)):   # 192 KB rings at most
            cfg = dict(issuer_warps=iw, stages=3, slots_per_warp=sl)
            cases.append((f"l2_bulk512_w{iw}_s{sl}", 32 << 20, 0, dict(cfg, chunk_bytes=512)))
            cases.append((f"l2_tma512_w{iw}_s{sl}", 32 << 20, 3, dict(cfg, chunk_bytes=512)))
            cfg = dict(issuer_warps=iw, stages=3, slots_per_warp=max(1, sl // 2))
            cases.append((f"l2_tma1k_w{iw}_s{sl // 2}", 32 << 20, 4, dict(cfg, chunk_bytes=1024)))
    bufs = {}
    for name, nbytes, method, cfg in cases:
        if nbytes not in bufs:
            bufs[nbytes] = torch.ones(nbytes // 2, dtype=torch.bfloat16, device=dev)
        src = bufs[nbytes]
        cfg = dict(cfg)
        cb = cfg.pop("chunk_bytes", chunk)
        iters = max(1, int(2e9 // (148 * cfg["issuer_warps"] * cfg["slots_per_warp"] * cb)))
        Q.qsa.qsa_probe_gather(src, chunk_bytes=cb, method=method, iterations=max(1, iters // 10), **cfg)
        best = None
        for _ in range(3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            nb = Q.qsa.qsa_probe_gather(src, chunk_bytes=cb, method=method, iterations=iters, **cfg)
            e1.record(stream)
            torch.cuda.synchronize()
            gbs = nb / (e0.elapsed_time(e1) / 1000) / 1e9
            best = gbs if best is None else max(best, gbs)
        res[name + "_gbs"] = best
    res["ceiling_gbs"] = max(v for k, v in res.items()
                             if k.startswith("l2_bulk") and "512" not in k and k.endswith("_gbs"))
    assert Q.qsa_get_device_status() == 0
    del bufs
    torch.cuda.empty_cache()
    return res


def workload_config(name: str, w, world: int) -> dict:
    """The `config` object of both arms' JSON lines (the same workload, the same keys)."""
    return {"workload": name, "B": w.B, "T": w.T, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D, "Hi": w.Hi, "Di": w.Di,
            "blk": w.blk, "k": w.k, "boost": f"{w.boost_frac:g} of keys x{w.boost:g}",
            "l2": "inputs larger than L2, no flush",
            "parallelism": "single GPU" if world == 1 else
            f"zig-zag query-row shards x{world}, one all-gather of K/V/kp per step; decode batch split"}


def kv_interleaved(w) -> bool:
    """Whether the automatic attention path reads K and V interleaved by block for this shape."""
    return w.D == 128 and w.Hkv in (1, 2) and w.Hq // w.Hkv <= 8


def attn_kernel_name(w) -> str:
    """The attention kernel the library launches for this shape."""
    group = w.Hq // w.Hkv
    if kv_interleaved(w):
        return f"interleave_kv_kernel + sparse_attn_kernel<{w.Hkv}, false, true>"
    if w.D == 128 and group <= 8:
        return f"sparse_attn_kernel<{w.Hkv}>"
    return f"sparse_attn_wide_kernel<{w.Hkv},{w.D},{1 if group <= 8 else 2}>"


def decode_work(w) -> dict:
    nb = (w.T - 1) // w.blk
    S = w.blk * min(nb, w.k) + (w.T - 1) % w.blk + 1
    kp_bytes = nb * w.Di * 2
    gathered = S * w.Hkv * w.D * 2 * 2
    qo = w.Hq * w.D * 2 * 2 + w.Hi * w.Di * 2
    return dict(bytes=(kp_bytes + gathered + qo) * w.B, kp_bytes=kp_bytes * w.B, gathered=gathered * w.B)


class Clocks:
    """nvidia-smi sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200", "-f", self.path],
                                         stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return None
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        torch.distributed.barrier()


# ------------------------------------------------------------------------------------------- CPU oracle
def oracle_sample(w, n_rows: int, host: dict | None = None, seed: int = 0):
    """Time the oracle (as it stands) on n_rows query rows spread over the workload.  Returns
    (seconds, rows, threads)."""
    import oracle as O
    if host is None:
        x = I.make_prefill(w, "cpu")
        host = {n: I.bits(x[n]) for n in x}
    t0 = time.perf_counter()
    kp = O.pool_block_keys(host["ki"], blk=w.blk)
    rows = np.unique(np.linspace(0, w.T - 1, n_rows).astype(np.int64))
    O.prefill_rows(host["q"], host["k"], host["v"], host["qi"], kp, [(0, int(t)) for t in rows], topk=w.k, blk=w.blk)
    dt = time.perf_counter() - t0
    return dt, len(rows), O.hardware_threads()


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = I.WORKLOADS[PREFILL]
    x = I.make_prefill(w, "cpu")
    host = {n: I.bits(x[n]) for n in x}
    del x
    n_rows = args.ref_rows
    for _ in range(args.warmup):
        oracle_sample(w, n_rows, host)
    times = []
    for _ in range(args.steps):
        dt, rows, cores = oracle_sample(w, n_rows, host)
        times.append(dt)
    total = sum(times)
    value = rows * args.steps / total
    sample = f"{rows} query rows spread evenly over the {w.T}-token prefill (pooling of all keys included)"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * total / args.steps,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(PREFILL, w, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------------------- GPU arm
def select_launches(w, ws_bytes: int) -> int:
    """Kernels qsa_select_topk launches for a prefill with a workspace of ws_bytes (the library's
    own choice between the filtered and the materialised selection, restated)."""
    nbk = w.T // w.blk
    rank = max(64, (2 * w.k + 15) // 16)
    ns = (nbk - 9) // 16 + 1 if nbk > 8 else 0
    per_row = ((max(ns, 1) + 3) // 4 * 4) * 4 + 12 + 32 * rank * 8
    fit = max(0, (ws_bytes - (12 * 256 + 4 + 128 * max(nbk, 1) * 4)) // per_row)
    n = 0
    if w.Hi in (4, 8) and w.k <= 1024 and 32 * rank <= 5120 and w.T >= 16384 and fit >= min(w.T, 4096):
        R = min(w.T, fit)
        if R < w.T and R >= 64:
            R -= R % 64
        for r0 in range(0, w.T, R):
            rows = min(R, w.T - r0)
            nb_last = min(nbk, (r0 + rows - 1) // w.blk)
            # sampled scores (when a sampled block is visible), thresholds, score + filter,
            # select over the lists, exact redo of failed rows
            n += (1 if nb_last > 8 else 0) + 4
        return n * w.B
    R = max(1, ws_bytes // (nbk * 4))
    for r0 in range(0, w.T, R):
        rows = min(R, w.T - r0)
        if min(nbk, (r0 + rows - 1) // w.blk) > 0:
            n += 1          # score kernel
        n += 1              # top-k kernel
    return n * w.B


def run_qsa(args):
    import hybrid_sparse_attention_qsa_b200 as Q

    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    pk = peaks()
    stream = torch.cuda.current_stream(dev)

    # ---------------------------------------------------------------- prefill (headline)
    # One job: every rank draws the same seeded inputs.  With N > 1 the query rows are sharded in
    # zig-zag chunks (shard.py): each rank keeps its rows' inputs, pools its indexer keys, takes part
    # in one all-gather of K, V and the pooled keys per step, then selects and attends for its rows.
    w = I.WORKLOADS[args.workload]
    x = I.make_prefill(w, dev)
    nbk = w.T // w.blk
    sp = None
    if world > 1:
        from hybrid_sparse_attention_qsa_b200 import shard as SH
        sp = SH.ShardedPrefill(w.B, w.T, w.Hq, w.Hkv, w.D, w.Hi, w.Di, w.k, world, rank, dev)
        x = {n: [x[n][:, a:b].contiguous() for a, b in sp.ranges] for n in x}
        ws = sp.ws
        ws_bytes = ws.numel()
        my_ranges = sp.ranges
    else:
        ws_bytes = Q.qsa_workspace_size(Q.qsa.QSA_OP_SELECT_TOPK, w.B, w.T, nbk, w.k, w.Hq, w.D)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        kp = torch.empty(w.B, nbk, w.Di, dtype=torch.bfloat16, device=dev)
        idx = torch.empty(w.B, w.T, w.k, dtype=torch.int32, device=dev)
        out = torch.empty_like(x["q"])
        lse = torch.empty(w.B, w.T, w.Hq, dtype=torch.float32, device=dev)
        my_ranges = [(0, w.T)]

    def step(ev=None):
        """One step; with `ev` = [(label, event), ...] the events mark where each part ends."""
        mark = (lambda i: ev[i][1].record(stream)) if ev else (lambda i: None)
        if sp is None:
            Q.qsa_pool_block_keys(x["ki"], kp)
            mark(0)
            Q.qsa_select_topk(w.k, qi=x["qi"], kp=kp, idx=idx, workspace=ws)
            mark(1)
            Q.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], idx, out=out, lse=lse)
            mark(2)
        else:
            sp.pool_local(x["ki"])
            sp.exchange(x["k"], x["v"])
            mark(0)
            sp.compute(x["q"], x["qi"], events=[e for _, e in ev[1:]] if ev else None)

    labels = ["pool", "score_topk", "attention"] if sp is None else \
        ["pool_allgather"] + ["score_topk", "attention"] * len(my_ranges)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert Q.qsa_get_device_status() == 0
    evs = [[(lab, torch.cuda.Event(enable_timing=True)) for lab in labels] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    with Clocks(local) as clk:
        t0.record(stream)
        for s in range(args.steps):
            starts[s].record(stream)
            step(evs[s])
        t1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    clocks = clk.summary()
    ms_total = max_over_ranks(t0.elapsed_time(t1), world, dev)
    ms_step = ms_total / args.steps
    parts = {lab: 0.0 for lab in labels}
    for s in range(args.steps):
        prev = starts[s]
        for lab, e in evs[s]:
            parts[lab] += prev.elapsed_time(e) / args.steps
            prev = e
    ms_select = parts["score_topk"]
    ms_attn = parts["attention"]
    value = w.B * w.T / (ms_step / 1000)    # the whole job's tokens (every rank's rows)
    work = prefill_work(w)
    if sp is not None:   # this rank's share of the work
        from hybrid_sparse_attention_qsa_b200 import shard as SH
        mine = SH.causal_cost(my_ranges, w.k, w.blk)
        work = dict(attn_bytes=mine["attended_tokens"] * w.Hkv * w.D * 4 * w.B
                    + sum(b - a for a, b in my_ranges) * w.Hq * w.D * 4 * w.B,
                    attn_flops=mine["attended_tokens"] * w.Hq * 4 * w.D * w.B,
                    index_flops=mine["index_pairs"] * 2 * w.Hi * w.Di * w.B, pairs=mine["index_pairs"] * w.B)
    attn_gbs = work["attn_bytes"] / (ms_attn / 1000) / 1e9
    attn_tflops = work["attn_flops"] / (ms_attn / 1000) / 1e12
    compulsory = unique_kv_bytes(w)
    traffic, traffic_src = profile_traffic(args.workload)
    ceiling = gather_ceiling(dev, stream, w)
    if sp is None:
        attn_launches = 2 if kv_interleaved(w) else 1   # the K/V interleave pass and the kernel
        launches = (1 + select_launches(w, ws_bytes) + attn_launches) * args.steps
    else:   # per chunk: pooling, the selection's kernels, attention (NCCL's own kernels not counted)
        attn_launches = 2 if kv_interleaved(w) else 1
        launches = sum(1 + attn_launches + select_launches(w.with_(T=b - a), ws_bytes) for a, b in my_ranges) * \
            args.steps

    # the query-tile attention (tcgen05 over the union of 16 rows' blocks) on the same lists, beside
    # the row-by-row kernel the step uses (both are the library's own kernels)
    tiles = None
    if sp is None and not args.no_tiles:
        try:
            aws = torch.empty(Q.qsa_workspace_size(Q.qsa.QSA_OP_SPARSE_ATTN_PREFILL, w.B, w.T, 0, w.k, w.Hq, w.D),
                              dtype=torch.uint8, device=dev)
            Q.qsa.qsa_set_attn_options(Q.qsa.QSA_ATTN_TILES)
            otile = torch.empty_like(out)
            ltile = torch.empty_like(lse)
            Q.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], idx, out=otile, lse=ltile, workspace=aws)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(3):
                Q.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], idx, out=otile, lse=ltile, workspace=aws)
            e1.record(stream)
            torch.cuda.synchronize()
            Q.qsa.qsa_set_attn_options(Q.qsa.QSA_ATTN_AUTO)
            assert Q.qsa_get_device_status() == 0
            t_ms = e0.elapsed_time(e1) / 3
            ntiles = w.B * ((w.T + 15) // 16)
            held = min(ntiles, 4096)
            cnt = aws[:held * 4].view(torch.int32).double()   # union sizes of the last range of tiles
            ublk = float(cnt.mean())
            gath = ublk * ntiles * w.Hkv * w.blk * w.D * 2 * 2          # K/V of every union block, per tile
            # dense over the union: 128 rows x blk tokens x D, times 2 flop, for S and for PV
            tflop = ublk * ntiles * w.Hkv * (128 * w.blk * w.D * 2 * 2) / 1e12
            diff = (otile.float() - out.float()).abs()
            tiles = {"kernel": "tile_union_kernel + sparse_attn_tc_kernel<%d>" % w.Hkv, "ms": t_ms,
                     "rows_kernel_ms": ms_attn, "speedup_vs_rows": ms_attn / t_ms,
                     "union_blocks_per_tile_mean": ublk, "union_over_sum_of_lists": ublk / (16 * (w.k + 1)),
                     "union_blocks_per_tile_quantiles": {f"p{int(100 * qq)}": float(torch.quantile(cnt, qq))
                                                          for qq in (0.0, 0.1, 0.5, 0.9, 1.0)},
                     "union_tiles_sampled": f"the last {held} tiles of the call (the ones the workspace held last)",
                     "gathered_bytes": gath, "gathered_bytes_rows_kernel": work["attn_bytes"],
                     "tensor_tflops_dense_union": tflop / (t_ms / 1000),
                     "frac_of_bf16_peak": tflop / (t_ms / 1000) / pk["bf16_tflops"],
                     "max_abs_diff_vs_rows": float(diff.max()), "mean_abs_diff_vs_rows": float(diff.mean())}
            del aws, otile, ltile
        except Exception as exc:
            Q.qsa.qsa_set_attn_options(Q.qsa.QSA_ATTN_AUTO)
            tiles = {"unavailable": f"{type(exc).__name__}: {exc}"[:200]}

    # indexer alone (scores for all rows materialised once; untimed in the step above)
    idx_ms = None
    try:
        if args.no_indexer or sp is not None:
            raise torch.OutOfMemoryError("skipped")
        scores = torch.empty(w.B, w.T, nbk, dtype=torch.float32, device=dev)
        Q.qsa_index_score(x["qi"], kp, scores=scores)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 3
        e0.record(stream)
        for _ in range(reps):
            Q.qsa_index_score(x["qi"], kp, scores=scores)
        e1.record(stream)
        torch.cuda.synchronize()
        idx_ms = e0.elapsed_time(e1) / reps
        del scores
    except torch.OutOfMemoryError:
        pass

    # dense causal attention on the same q/k/v (library SDPA, GQA), the comparison the vendor's
    # kernel-level speedups are stated against; QSA's step (selection included) over it
    dense = None
    if not args.no_dense and sp is None:
        try:
            g = w.Hq // w.Hkv   # K/V expanded to every query head so the flash backend takes the call
            qd = x["q"].transpose(1, 2)
            kd = x["k"].repeat_interleave(g, dim=2).transpose(1, 2)
            vd = x["v"].repeat_interleave(g, dim=2).transpose(1, 2)
            sdpa = torch.nn.functional.scaled_dot_product_attention
            with torch.cuda.stream(stream):
                sdpa(qd, kd, vd, is_causal=True)
                f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                f0.record(stream)
                for _ in range(2):
                    sdpa(qd, kd, vd, is_causal=True)
                f1.record(stream)
            torch.cuda.synchronize()
            dense_ms = f0.elapsed_time(f1) / 2
            del qd, kd, vd
            dense = {"impl": "torch scaled_dot_product_attention (causal, bf16, K/V expanded to Hq)", "ms": dense_ms,
                     "qsa_step_ms": ms_step, "qsa_attention_ms": ms_attn,
                     "speedup_step": dense_ms / ms_step, "speedup_attention_only": dense_ms / ms_attn}
        except Exception as exc:   # library without a kernel for this shape
            dense = {"unavailable": f"{type(exc).__name__}: {exc}"[:200]}

    # end to end through the public API from pinned host buffers
    e2e = None
    if not args.no_e2e and sp is not None:
        # each rank's own rows from pinned host buffers: H2D of its input chunks, the sharded step,
        # D2H of its output rows
        hin = {n: [t.cpu().pin_memory() for t in x[n]] for n in x}
        hout = [torch.empty_like(o, device="cpu").pin_memory() for o in sp.out]
        h2d = sum(t.numel() * t.element_size() for ts in hin.values() for t in ts)
        d2h = sum(t.numel() * t.element_size() for t in hout)

        def e2e_step():
            for n in x:
                for dst, src in zip(x[n], hin[n]):
                    dst.copy_(src, non_blocking=True)
            step()
            for dst, src in zip(hout, sp.out):
                dst.copy_(src, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        a0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        a1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(a0.elapsed_time(a1), world, dev) / args.e2e_steps
        e2e = {"value": w.B * w.T / (e2e_ms / 1000), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "per_rank": True}
        del hin, hout
    elif not args.no_e2e:
        host = {n: torch.empty_like(x[n], device="cpu").pin_memory() for n in ("q", "k", "v", "qi", "ki")}
        for n in host:
            host[n].copy_(x[n])
        hout = torch.empty_like(out, device="cpu").pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = hout.numel() * hout.element_size()
        dbufs = {}

        def e2e_step():
            Q.qsa.prefill_host(host["q"], host["k"], host["v"], host["qi"], host["ki"], topk=w.k, device=dev, out=hout,
                               device_buffers=dbufs)

        e2e_step()
        torch.cuda.synchronize()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        a0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        a1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(a0.elapsed_time(a1), world, dev) / args.e2e_steps
        e2e = {"value": w.B * w.T / (e2e_ms / 1000), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}
        del host, hout, dbufs
    if sp is None:
        del idx, out, lse, kp
    del x, ws, sp
    torch.cuda.empty_cache()

    # ---------------------------------------------------------------- decode leg
    decode = None
    if not args.no_decode:
        # the decode batch is split across the ranks (no collective): each keeps its sequences
        wd = I.WORKLOADS[args.decode_workload]
        xd = I.make_decode(wd, dev)
        if world > 1:
            from hybrid_sparse_attention_qsa_b200 import shard as SH
            b0, b1 = SH.batch_range(wd.B, world, rank)
            xd = {n: t[b0:b1].contiguous() for n, t in xd.items()}
            wd = wd.with_(B=b1 - b0)
            torch.cuda.empty_cache()
        nbd = wd.T // wd.blk
        kpd = Q.qsa_pool_block_keys(xd["ki"])
        wsd = torch.empty(Q.qsa_workspace_size(Q.qsa.QSA_OP_SELECT_TOPK, wd.B, 1, nbd, wd.k, wd.Hq, wd.D),
                          dtype=torch.uint8, device=dev)
        splits = Q.qsa.lib().qsa_decode_default_splits(wd.B, wd.k)
        wsa = torch.empty(max(16, Q.qsa_workspace_size(Q.qsa.QSA_OP_SPARSE_ATTN_DECODE, wd.B, 1, 0, wd.k, wd.Hq, wd.D,
                                                       splits)), dtype=torch.uint8, device=dev)
        idxd = torch.empty(wd.B, wd.k, dtype=torch.int32, device=dev)
        outd = torch.empty_like(xd["q"])
        lsed = torch.empty(wd.B, wd.Hq, dtype=torch.float32, device=dev)

        def dsel():
            # pool the block the new token completes (when it completes one) inside the score
            # kernel, then score and select
            Q.qsa_decode_select(wd.k, qi=xd["qi"], kp=kpd, ki=xd["ki"], seqlens=xd["seqlens"], idx=idxd,
                                workspace=wsd)

        def datt():
            Q.qsa_sparse_attn_decode(xd["q"], xd["k"], xd["v"], xd["seqlens"], idxd, num_splits=splits, out=outd,
                                     lse=lsed, workspace=wsa)

        for _ in range(max(args.warmup, 3)):
            dsel()
            datt()
        torch.cuda.synchronize()
        assert Q.qsa_get_device_status() == 0
        # A decode step is replayed from a CUDA graph (the launches of one step, captured once), as a
        # serving loop does: the device time is then not bounded by the host's launch rate.
        g_step, g_sel, g_att = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_step):
            dsel()
            datt()
        with torch.cuda.graph(g_sel):
            dsel()
        with torch.cuda.graph(g_att):
            datt()
        for _ in range(3):
            g_step.replay()
        torch.cuda.synchronize()
        assert Q.qsa_get_device_status() == 0
        dsteps = args.decode_steps
        gs = torch.cuda.current_stream(dev)
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        d0.record(gs)
        for _ in range(dsteps):
            g_step.replay()
        d1.record(gs)
        torch.cuda.synchronize()
        dms = max_over_ranks(d0.elapsed_time(d1), world, dev) / dsteps
        # breakdown: each part's graph replayed 10 times back to back between two events
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record(gs)
        for _ in range(10):
            g_sel.replay()
        ev[1].record(gs)
        for _ in range(10):
            g_att.replay()
        ev[2].record(gs)
        torch.cuda.synchronize()
        d_sel = ev[0].elapsed_time(ev[1]) / 10
        d_att = ev[1].elapsed_time(ev[2]) / 10
        del g_step, g_sel, g_att
        dw = decode_work(wd)
        dgbs = dw["bytes"] / (dms / 1000) / 1e9
        decode = {"workload": args.decode_workload, "value": I.WORKLOADS[args.decode_workload].B / (dms / 1000),
                  "unit": "tokens/s",
                  "ms_per_step": dms, "launch": "CUDA graph of one step, replayed",
                  "steps": dsteps, "num_splits": splits,
                  "step_breakdown_ms": {"score_topk": d_sel, "attention_and_merge": d_att},
                  "gpu_launches_per_step": 2 + 1 + (1 if Q.qsa.lib().qsa_decode_split_merge(
                      wd.B, wd.Hq, wd.Hkv, wd.D, splits) == 2 else 0),
                  "roofline": {"bound": "hbm", "achieved": dgbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                               "frac": dgbs / pk["hbm_gbs"], "bytes_per_step": dw["bytes"],
                               "basis": "pooled-key cache read + gathered K/V of the selected tokens + q/o"}}
        # dense attention of the same new tokens over the whole caches (library SDPA, GQA): the
        # decode side of the kernel-level comparison
        if not args.no_dense:
            try:
                qd = xd["q"].view(wd.B, wd.Hq, 1, wd.D)
                kd = xd["k"].transpose(1, 2)   # [B, Hkv, L, D] views of the caches
                vd = xd["v"].transpose(1, 2)
                sdpa = torch.nn.functional.scaled_dot_product_attention
                with torch.cuda.stream(stream):
                    sdpa(qd, kd, vd, enable_gqa=True)
                    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    f0.record(stream)
                    for _ in range(5):
                        sdpa(qd, kd, vd, enable_gqa=True)
                    f1.record(stream)
                torch.cuda.synchronize()
                dd_ms = f0.elapsed_time(f1) / 5
                decode["dense_compare"] = {"impl": "torch scaled_dot_product_attention (all cache positions, GQA, bf16)",
                                           "ms": dd_ms, "qsa_step_ms": dms, "qsa_attention_ms": d_att,
                                           "speedup_step": dd_ms / dms, "speedup_attention_only": dd_ms / d_att}
            except Exception as exc:   # library without a kernel for this shape
                decode["dense_compare"] = {"unavailable": f"{type(exc).__name__}: {exc}"[:200]}
        del xd, kpd, wsd, wsa, idxd, outd, lsed

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(args.workload, w, world),
            # The attention's compulsory work is its tensor-core flops (the unique K/V bytes take a
            # tenth of that time at HBM peak), so the roofline is stated on the tensor basis; the
            # gathered-bytes rate is compared with the measured gather ceiling, not with HBM.
            "roofline": {"bound": "tensor", "kernel": attn_kernel_name(w), "achieved": attn_tflops,
                         "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": attn_tflops / pk["bf16_tflops"],
                         "traffic": traffic, "traffic_source": traffic_src, "peak_source": pk["source"],
                         "peak_kind": "bf16 dense burst (cuBLAS), of " + pk["source"],
                         "basis": "attention flops: Hq * |S(t)| * 4 * D per query row (QK^T and PV)",
                         "flops_per_launch": work["attn_flops"], "ms_per_launch": ms_attn,
                         "compulsory_hbm": {"bytes": compulsory, "achieved_gbs": compulsory / (ms_attn / 1000) / 1e9,
                                            "peak_gbs": pk["hbm_gbs"],
                                            "frac": compulsory / (ms_attn / 1000) / 1e9 / pk["hbm_gbs"],
                                            "basis": "every K/V row once + q read + o write"},
                         "gathered_bytes_rate": {
                             "bytes_per_launch": work["attn_bytes"], "achieved_gbs": attn_gbs,
                             "ceiling_gbs": ceiling["ceiling_gbs"],
                             "frac_of_ceiling": attn_gbs / ceiling["ceiling_gbs"],
                             "basis": "K/V rows of every selected token as gathered (a block once per query "
                                      "that selects it) + q read + o write, over the attention call (the "
                                      "K/V interleave pass and the kernel); ceiling = the best bulk-copy "
                                      "gather of the same 4 KB blocks (K then V) from an L2-resident "
                                      "buffer into the kernel's ring, measured in this run (gather_probe)"},
                         "gather_probe": ceiling},
            "step_breakdown_ms": parts,
            "indexer": {
                "flops": work["index_flops"],
                "selection": {"ms": ms_select, "tflops": work["index_flops"] / ms_select / 1e9,
                              "frac_of_bf16_peak": work["index_flops"] / ms_select / 1e9 / pk["bf16_tflops"],
                              "note": "the whole selection as timed in the step (filtered: sampled scores, "
                                      "thresholds, tensor-core score + filter, select, redo)"},
                "materialised_scores": None if idx_ms is None else {
                    "ms": idx_ms, "tflops": work["index_flops"] / idx_ms / 1e9,
                    "frac_of_bf16_peak": work["index_flops"] / idx_ms / 1e9 / pk["bf16_tflops"],
                    "note": "qsa_index_score alone: scores of every row written to HBM (fp32)"}},
            "gpu_launches": launches,
            "clocks": clocks,
            "e2e": e2e,
            "decode": decode,
            "dense_compare": dense,
            "attention_query_tiles": tiles,
        }
        if not args.no_cpu_baseline and world == 1:
            dt, rows, cores = oracle_sample(I.WORKLOADS[args.workload], args.ref_rows)
            line["cpu_baseline"] = {"value": rows / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                    "sample": f"{rows} query rows spread evenly over the {w.T}-token prefill, "
                                              f"pooling of all keys included"}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="qsa", choices=["qsa", "reference"])
    ap.add_argument("--decode-steps", type=int, default=50)
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--ref-rows", type=int, default=96)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-indexer", action="store_true", help="skip the stand-alone indexer timing (17 GB of scores)")
    ap.add_argument("--no-dense", action="store_true", help="skip timing dense causal attention on the same inputs")
    ap.add_argument("--no-tiles", action="store_true", help="skip timing the query-tile attention beside the rows")
    ap.add_argument("--probe-l2-gather", action="store_true",
                    help="only measure the gather ceiling (bulk-copy and cp.async gathers of the attention's "
                         "chunks from L2 and HBM, with a sweep of issuing warps) and print it as one JSON line")
    ap.add_argument("--decode-workload", default=DECODE,
                    choices=[n for n, w in I.WORKLOADS.items() if w.kind == "decode"],
                    help="decode workload of the second leg (default: 32 sequences of 256K tokens)")
    ap.add_argument("--workload", default=PREFILL, choices=[n for n, w in I.WORKLOADS.items() if w.kind == "prefill"],
                    help="prefill workload of the headline leg (default: the 128K configuration)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.probe_l2_gather:
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        w = I.WORKLOADS[args.workload]
        print(json.dumps({"probe": "gather", "workload": args.workload,
                          **gather_ceiling(dev, torch.cuda.current_stream(dev), w, sweep=True)}), flush=True)
        return 0
    return run_qsa(args)


if __name__ == "__main__":
    sys.exit(main())
