#!/usr/bin/env python
"""Benchmark of one absorbed-MLA decode step on B200.

A step = one mla_decode call (split plan + decode kernel + log-sum-exp combine) over the
whole batch of the chosen workload (default: the DeepSeek-V3-shaped decode, B=64,
H=128, r=512, d_r=64, 32768-token context, bf16 paged cache). Inputs are seeded
synthetic data (workloads.py) resident in HBM before timing; the 2.4 GB cache is far
larger than L2, and workloads whose cache is not are flushed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Prints one JSON line on rank 0. `value` is the latent-cache read rate (TB/s of
attended cache bytes, summed over ranks, over the max-over-ranks device time); TFLOP/s
and steps/s ride along. With N > 1 (torchrun) every rank runs an independent replica
(the decode has no cross-GPU exchange). `--impl reference` times the fp64 CPU oracle on
the host instead, on one sequence per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "MLA decode latent-cache TB/s, TFLOP/s, steps/s; % of roofline at 1 B200"
FLOP_PER_PAIR = None   # set from the workload: 2 (r + d_r) + 2 r per (query row, head, token)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="deepseek_v3", choices=list(W.BY_NAME))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--kernel", default="auto", choices=["auto", "simt", "tcgen05", "tc_pair"])
    ap.add_argument("--num-workers", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--extra-cpu-seconds", type=float, default=6.0,
                    help="oracle sample per extra workload (the headline one gets --cpu-seconds)")
    ap.add_argument("--only", action="store_true",
                    help="time the chosen workload alone (by default one-GPU runs also time the other four)")
    ap.add_argument("--op", default="decode", choices=["decode", "append", "absorb", "project", "dsa"],
                    help="decode: the decode step (default); append: the paged cache append of the step's new "
                         "tokens; absorb / project: the per-head W^UK / W^UV products around the decode; dsa: "
                         "the sparse decode step (indexer, top-k, decode over the selected tokens)")
    ap.add_argument("--dsa-workload", default="dsa_v32", choices=list(W.DSA_BY_NAME))
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (smaller profiling captures only)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained"), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum, one ncu capture of the decode
# kernel the workload runs on a smaller batch of the same workload; profiles/) per cached token. A figure
# only holds for the sources the kernel was built from, keyed here by kernel and the SHA-256 prefix of
# those files; for any other source the bench reports traffic as null.
MEASURED_TRAFFIC = {
    ("tc_pair", "c34dd76ad94899ec"): {"deepseek_v3": (304.350976e6 + 4.457728e6) / 262144},
}
KERNEL_SOURCES = {
    "tc_pair": ("mla_pair.cu", "ptx_sm100.cuh", "mla_device.cuh", "mla_internal.h", "mla_tc.h"),
    "tcgen05": ("mla_tc.cu", "ptx_sm100.cuh", "mla_device.cuh", "mla_internal.h", "mla_tc.h"),
}
# The same for the sparse step's indexer (dram bytes per context token, batch 8 of the
# 128K workload), keyed by the sources of mla_dsa.cu and its headers.
DSA_TRAFFIC = {
    "9f69c58ab496e496": {"dsa_v32": (138.620416e6 + 4.136448e6) / (8 * 131072)},
}
DSA_SOURCES = ("mla_dsa.cu", "ptx_sm100.cuh", "mla_device.cuh", "mla_internal.h")


def kernel_source_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "head_latent_attention_split_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(wl, model, kernel):
    """Per-launch DRAM bytes of the decode kernel scaled from the ncu capture, or None."""
    if kernel not in ("tcgen05", "tc_pair"):
        return None
    per_tok = MEASURED_TRAFFIC.get((kernel, kernel_source_hash(KERNEL_SOURCES[kernel])), {}).get(wl.name)
    return None if per_tok is None else per_tok * model["tokens"]


def reduce_max(x: float, world: int, device=None) -> float:
    """Max of x over the ranks of the default process group (x itself when world == 1)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate_tbs(world: int, steps: int, bytes_per_step: float, max_ms: float) -> float:
    """Whole-job rate in TB/s: each of `world` replicas moves bytes_per_step per step, and the job
    lasts as long as its slowest rank (max_ms for `steps` steps)."""
    return world * steps * bytes_per_step / (max_ms / 1e3) / 1e12


def work_model(inp):
    """Algorithmic bytes and FLOPs of one step: each attended cache token read once (1152 B bf16,
    644 B e4m3 + bf16 RoPE key + fp32 scale), the queries read and the outputs written once;
    2 (r + d_r) + 2 r FLOP per attended (query row, head, token)."""
    w = inp["workload"]
    lens = inp["seq_lens"].astype(np.int64)
    tok = int(lens.sum())
    per_tok = W.cache_bytes_per_token(w.r, w.d_r, w.cache_dtype)
    qsz = 4 if w.q_dtype == W.F32 else 2
    osz = 4 if w.out_dtype == W.F32 else 2
    rows = w.B * w.Sq * w.H
    cache_bytes = tok * per_tok
    io_bytes = rows * (w.r + w.d_r) * qsz + rows * w.r * osz + rows * 4
    pairs = W.attended_pairs(w, lens)
    flops = pairs * (2 * (w.r + w.d_r) + 2 * w.r)
    return dict(tokens=tok, cache_bytes=cache_bytes, io_bytes=io_bytes, bytes=cache_bytes + io_bytes,
                flops=flops, pairs=pairs)


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms in the background."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.proc = None
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_id), f"--query-gpu=timestamp,{self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.file, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None
        self.t0 = self.t1 = None

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        rows = []
        for line in open(self.file.name):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                rows.append((ts, float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.file.name)
        if not rows:
            return None
        inside = [r for r in rows if self.t0 - 1 <= r[0] <= self.t1 + 1] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i, v in enumerate(r[3]) if v.lower() == "active"})
        return dict(sm_mhz=statistics.median(r[1] for r in inside), sm_max_mhz=max(r[2] for r in inside),
                    reasons=reasons, samples=len(inside))


def cpu_oracle_rate(inp, seconds, seqs_per_step=None):
    """Time the fp64 oracle on whole sequences (all heads) until `seconds` elapse."""
    import oracle
    w = inp["workload"]
    per_tok = W.cache_bytes_per_token(w.r, w.d_r, w.cache_dtype)
    cores = os.cpu_count() or 1
    done_bytes, elapsed, nseq = 0, 0.0, 0
    b = 0
    while (seqs_per_step is None and elapsed < seconds and nseq < w.B) or (seqs_per_step and nseq < seqs_per_step):
        sl = slice(b, b + 1)
        t0 = time.perf_counter()
        oracle.decode(inp["q_lat"][sl], inp["q_rope"][sl], inp["kv_cache"], inp["block_table"][sl],
                      inp["seq_lens"][sl], w.scale, w.causal, inp.get("k_rope_cache"), inp.get("kv_scale"),
                      w.block_size, nthreads=cores)
        elapsed += time.perf_counter() - t0
        done_bytes += int(inp["seq_lens"][b]) * per_tok
        nseq += 1
        b = (b + 1) % w.B
    return dict(value=done_bytes / elapsed / 1e12, unit="TB/s", cores=cores, kind="oracle",
                sample=f"{nseq} of {w.B} sequences (all {w.Sq * w.H} query rows each, full context), "
                       f"{elapsed:.1f} s of fp64 CPU work"), elapsed


def reference_arm(args, rank):
    if rank != 0:
        return
    wl = W.BY_NAME[args.workload]
    inp = W.make_inputs(wl)
    per_tok = W.cache_bytes_per_token(wl.r, wl.d_r, wl.cache_dtype)
    for i in range(args.warmup):
        cpu_oracle_rate(inp, 0, seqs_per_step=1)
    tot_t, tot_bytes, tot_flops = 0.0, 0, 0
    for i in range(args.steps):
        b = i % wl.B
        sub = dict(inp, q_lat=inp["q_lat"][b:b + 1], q_rope=inp["q_rope"][b:b + 1],
                   block_table=inp["block_table"][b:b + 1], seq_lens=inp["seq_lens"][b:b + 1])
        import oracle
        t0 = time.perf_counter()
        oracle.decode_inputs(sub, nthreads=os.cpu_count() or 1)
        tot_t += time.perf_counter() - t0
        L = int(inp["seq_lens"][b])
        tot_bytes += L * per_tok
        tot_flops += W.attended_pairs(wl.with_(B=1, seq_lens=(L,)), np.array([L])) * (4 * wl.r + 2 * wl.d_r)
    value = tot_bytes / tot_t / 1e12
    cores = os.cpu_count() or 1
    line = dict(metric=METRIC, value=value, unit="TB/s", impl="reference", n_gpus=args.gpus, steps=args.steps,
                warmup=args.warmup, ms_per_step=1e3 * tot_t / args.steps, higher_is_better=True, scaling="weak",
                vs_baseline=None, dtype="f64", data="synthetic",
                config=dict(workload=wl.name, B=wl.B, Sq=wl.Sq, H=wl.H, r=wl.r, d_r=wl.d_r,
                            cache=W.DTYPE_NAMES[wl.cache_dtype], seq_lens=str(wl.seq_lens)[:40],
                            step="one sequence (all heads) of the workload per step"),
                tflops=tot_flops / tot_t / 1e12,
                cpu_baseline=dict(value=value, unit="TB/s", cores=cores, kind="oracle",
                                  sample=f"one of {wl.B} sequences per step, all {wl.Sq * wl.H} query rows"),
                e2e=dict(value=value, unit="TB/s", h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)


def append_arm(args, rank, local):
    """Time mla_cache_append for the workload's B x Sq new tokens (rotated RoPE keys)."""
    import torch
    import head_latent_attention_split_b200 as mla
    wl = W.BY_NAME[args.workload]
    if args.batch:
        wl = wl.with_(B=args.batch)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    lens = np.asarray(W.resolve_seq_lens(wl), np.int32)
    bs = wl.block_size
    mb = int((lens.max() + bs - 1) // bs)
    nb = wl.B * mb
    bt = torch.randperm(nb, dtype=torch.int32, device=dev).reshape(wl.B, mb)
    sl = torch.from_numpy(lens).to(dev)
    g = torch.Generator(device=dev).manual_seed(1000 + W.WORKLOADS.index(W.BY_NAME[args.workload]))
    c = torch.randn((wl.B, wl.Sq, wl.r), generator=g, device=dev).to(torch.bfloat16)
    k = torch.randn((wl.B, wl.Sq, wl.d_r), generator=g, device=dev).to(torch.bfloat16)
    fp8 = wl.cache_dtype == W.E4M3
    if fp8:
        cache = torch.zeros((nb, bs, wl.r), dtype=torch.uint8, device=dev)
        kr = torch.zeros((nb, bs, wl.d_r), dtype=torch.bfloat16, device=dev)
        sc = torch.zeros((nb, bs), dtype=torch.float32, device=dev)
    else:
        cache = torch.zeros((nb, bs, wl.r + wl.d_r), dtype=torch.bfloat16, device=dev)
        kr = sc = None
    run = lambda: mla.cache_append(c, k, cache, bt, sl, k_rope_cache=kr, kv_scale=sc, rope=True)  # noqa: E731
    for _ in range(max(args.warmup, 3)):
        run()
    torch.cuda.synchronize()
    assert mla.device_status() == 0
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record()
    for _ in range(args.steps):
        run()
    ev[1].record()
    torch.cuda.synchronize()
    us = 1e3 * ev[0].elapsed_time(ev[1]) / args.steps
    ntok = wl.B * wl.Sq
    bytes_ = ntok * ((wl.r + wl.d_r) * 2 + W.cache_bytes_per_token(wl.r, wl.d_r, wl.cache_dtype))
    peaks = load_peaks()
    gbs = bytes_ / (us * 1e-6) / 1e9
    if rank == 0:
        print(json.dumps(dict(
            metric="paged cache append GB/s (new tokens read + cache slots written)", value=gbs, unit="GB/s",
            n_gpus=1, steps=args.steps, warmup=max(args.warmup, 3), us_per_call=us, higher_is_better=True,
            dtype="bf16->" + W.DTYPE_NAMES[wl.cache_dtype], data="synthetic",
            config=dict(workload=wl.name, op="append", B=wl.B, Sq=wl.Sq, r=wl.r, d_r=wl.d_r, rope=True,
                        new_tokens=ntok, bytes_per_call=bytes_),
            roofline=dict(bound="hbm", achieved=gbs, peak=peaks["hbm_gbs"], unit="GB/s", frac=gbs / peaks["hbm_gbs"],
                          traffic=None, note="launch-latency bound: one call moves only bytes_per_call"),
            gpu_launches=args.steps)), flush=True)


def head_gemm_arm(args, rank, local):
    """Time the per-head GEMM of the workload's query rows: absorb (d_h = 128 -> r) or project (r -> d_v = 128)."""
    import torch
    import head_latent_attention_split_b200 as mla
    wl = W.BY_NAME[args.workload]
    if args.batch:
        wl = wl.with_(B=args.batch)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    rows, H = wl.B * wl.Sq, wl.H
    k, n = (128, wl.r) if args.op == "absorb" else (wl.r, 128)
    g = torch.Generator(device=dev).manual_seed(7)
    x = torch.randn((rows, H, k), generator=g, device=dev).to(torch.bfloat16)
    w = (torch.randn((H, k, n), generator=g, device=dev) / math.sqrt(k)).to(torch.bfloat16)
    y = torch.empty((rows, H, n), dtype=torch.bfloat16, device=dev)
    for _ in range(max(args.warmup, 3)):
        mla.head_gemm(x, w, y)
    torch.cuda.synchronize()
    assert mla.device_status() == 0
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record()
    for _ in range(args.steps):
        mla.head_gemm(x, w, y)
    ev[1].record()
    torch.cuda.synchronize()
    us = 1e3 * ev[0].elapsed_time(ev[1]) / args.steps
    flops = 2.0 * rows * H * k * n
    bytes_ = 2 * (rows * H * (k + n) + H * k * n)
    peaks = load_peaks()
    t_roof = max(bytes_ / (peaks["hbm_gbs"] * 1e9), flops / (peaks["bf16_tflops"] * 1e12))
    bound = "hbm" if bytes_ / (peaks["hbm_gbs"] * 1e9) >= flops / (peaks["bf16_tflops"] * 1e12) else "tensor"
    achieved = bytes_ / (us * 1e-6) / 1e9 if bound == "hbm" else flops / (us * 1e-6) / 1e12
    if rank == 0:
        print(json.dumps(dict(
            metric=f"per-head {'query absorption' if args.op == 'absorb' else 'output projection'} TFLOP/s",
            value=flops / (us * 1e-6) / 1e12, unit="TFLOP/s", n_gpus=1, steps=args.steps,
            warmup=max(args.warmup, 3), us_per_call=us, higher_is_better=True, dtype="bf16", data="synthetic",
            config=dict(workload=wl.name, op=args.op, rows=rows, H=H, k=k, n=n),
            roofline=dict(bound=bound, achieved=achieved, peak=peaks["hbm_gbs"] if bound == "hbm" else
                          peaks["bf16_tflops"], unit="GB/s" if bound == "hbm" else "TFLOP/s",
                          frac=t_roof / (us * 1e-6), traffic=None),
            gpu_launches=args.steps)), flush=True)


def dsa_work_model(inp):
    """Algorithmic bytes / FLOPs of one sparse decode step, per kernel."""
    dw = inp["dsa"]
    w = inp["workload"]
    n = np.asarray(inp["seq_lens"], np.int64)            # q_len 1: each row sees its whole sequence
    cnt = np.minimum(n, dw.top_k)
    rows = w.B * w.Sq
    idx_bytes = int(n.sum()) * (dw.dI + 4 + 4) + rows * dw.HI * (dw.dI + 8)     # key codes + scale, score out; query
    idx_flops = int(n.sum()) * dw.HI * dw.dI * 2
    topk_bytes = int(n.sum()) * 4 + rows * dw.top_k * 4                         # scores in, positions out
    dec_bytes = int(cnt.sum()) * (w.r + w.d_r) * 2 + rows * w.H * ((w.r + w.d_r) * 2 + w.r * 2 + 4)
    dec_flops = int(cnt.sum()) * w.H * (2 * (w.r + w.d_r) + 2 * w.r)
    return dict(index=dict(bytes=idx_bytes, flops=idx_flops), topk=dict(bytes=topk_bytes, flops=0),
                decode=dict(bytes=dec_bytes, flops=dec_flops), tokens=int(n.sum()), selected=int(cnt.sum()))


def dsa_cpu_baseline(inp, seconds):
    """The oracle's three steps on whole query rows until `seconds` elapse."""
    import oracle
    w = inp["workload"]
    cores = os.cpu_count() or 1
    elapsed, nrow, b = 0.0, 0, 0
    while elapsed < seconds and nrow < w.B:
        sl = slice(b, b + 1)
        L = int(inp["seq_lens"][b])
        t0 = time.perf_counter()
        sc = oracle.dsa_index(inp["iq_codes"][sl], inp["iq_scale"][sl], inp["iw"][sl], inp["ik_codes"],
                              inp["ik_scale"], inp["block_table"][sl], inp["seq_lens"][sl], max_seq_len=L,
                              nthreads=cores)
        idx, cnt = oracle.dsa_topk(sc, np.array([[L]]), inp["top_k"])
        oracle.decode_sparse(inp["q_lat"][sl], inp["q_rope"][sl], inp["kv_cache"], inp["block_table"][sl],
                             inp["seq_lens"][sl], w.scale, idx, cnt, nthreads=cores)
        elapsed += time.perf_counter() - t0
        nrow += 1
        b += 1
    return dict(value=nrow / w.B / elapsed, unit="steps/s", cores=cores, kind="oracle",
                sample=f"{nrow} of {w.B} sequences (indexer over the full context, top-k, sparse decode of all "
                       f"{w.H} heads), {elapsed:.1f} s of fp64 CPU work")


def dsa_arm(args, rank, local):
    """Time one sparse decode step: mla_dsa_index + mla_dsa_topk + mla_sparse_decode."""
    import torch
    import head_latent_attention_split_b200 as mla
    dw = W.DSA_BY_NAME[args.dsa_workload]
    if args.batch:
        m = dw.mla
        dw = W.DsaWorkload(f"{dw.name}_b{args.batch}", m.with_(B=args.batch, seq_lens=tuple(m.seq_lens[:1]) * args.batch),
                           dw.HI, dw.dI, dw.top_k, dw.w_std)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    inp = W.make_dsa_inputs(dw)
    w = inp["workload"]
    t = W.to_torch(inp, dev)
    g = {k: torch.from_numpy(np.ascontiguousarray(inp[k])).to(dev) for k in ("iq_codes", "iq_scale", "iw", "ik_codes",
                                                                              "ik_scale")}
    L, k = inp["max_seq_len"], dw.top_k
    scores = torch.empty((w.B, 1, L), dtype=torch.float32, device=dev)
    idx = torch.empty((w.B, 1, k), dtype=torch.int32, device=dev)
    cnt = torch.empty((w.B, 1), dtype=torch.int32, device=dev)
    dp = mla.dsa_params_for(g["iq_codes"], g["ik_codes"], t["block_table"], L, k)
    p = mla.params_for(t["q_lat"], t["q_rope"], t["kv_cache"], t["block_table"], w.scale, False, kernel="auto")
    ws = torch.empty(max(1, mla.workspace_size(p)), dtype=torch.uint8, device=dev)
    out = torch.empty(t["q_lat"].shape, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(t["q_lat"].shape[:3], dtype=torch.float32, device=dev)

    def step(ev):
        ev[0].record()
        mla.mla_dsa_index(dp, g["iq_codes"], g["iq_scale"], g["iw"], g["ik_codes"], g["ik_scale"], t["block_table"],
                          t["seq_lens"], scores)
        ev[1].record()
        mla.mla_dsa_topk(dp, scores, t["seq_lens"], idx, cnt)
        ev[2].record()
        mla.mla_sparse_decode(p, k, t["q_lat"], t["q_rope"], t["kv_cache"], t["block_table"], idx, cnt, out, lse, ws)
        ev[3].record()

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K + max(3, args.warmup))]
    for e in evs:
        for x in e:
            x.record()
    for i in range(max(3, args.warmup)):
        step(evs[K + i])
    torch.cuda.synchronize()
    st = mla.device_status()
    if st != 0:
        raise RuntimeError(f"device status {mla.status_string(st)}")
    props = torch.cuda.get_device_properties(local)
    gpu_id = getattr(props, "uuid", None)
    sampler = ClockSampler(f"GPU-{gpu_id}" if gpu_id is not None else local)
    time.sleep(0.3)
    torch.cuda.synchronize()
    sampler.mark_start()
    for i in range(K):
        step(evs[i])
    torch.cuda.synchronize()
    sampler.mark_end()
    clocks = sampler.stop()
    st = mla.device_status()
    if st != 0:
        raise RuntimeError(f"device status {mla.status_string(st)}")
    ms = {name: [e[i].elapsed_time(e[i + 1]) for e in evs[:K]] for i, name in enumerate(("index", "topk", "decode"))}
    total_ms = sum(evs[i][0].elapsed_time(evs[i][3]) for i in range(K))
    model = dsa_work_model(inp)
    peaks = load_peaks()
    detail = {}
    for name in ("index", "topk", "decode"):
        sec = statistics.mean(ms[name]) / 1e3
        d = model[name]
        t_hbm, t_tc = d["bytes"] / (peaks["hbm_gbs"] * 1e9), d["flops"] / (peaks["bf16_tflops"] * 1e12)
        if name == "index":
            t_tc /= 2.0    # e4m3 MMA: twice the bf16 dense rate (nominal ratio)
        detail[name] = dict(ms=1e3 * sec, algorithmic_bytes=d["bytes"], algorithmic_flops=d["flops"],
                            gbs=d["bytes"] / sec / 1e9, tflops=d["flops"] / sec / 1e12,
                            roofline_us=1e6 * max(t_hbm, t_tc), frac=max(t_hbm, t_tc) / sec,
                            bound="hbm" if t_hbm >= t_tc else "tensor")
    top = max(detail, key=lambda n: detail[n]["ms"])
    td = detail[top]
    if td["bound"] == "hbm":
        roof = dict(bound="hbm", achieved=td["gbs"], peak=peaks["hbm_gbs"], unit="GB/s", frac=td["gbs"] / peaks["hbm_gbs"])
    else:
        pk = peaks["bf16_tflops"] * (2.0 if top == "index" else 1.0)
        roof = dict(bound="tensor", achieved=td["tflops"], peak=pk, unit="TFLOP/s", frac=td["tflops"] / pk)
    per_tok = DSA_TRAFFIC.get(kernel_source_hash(DSA_SOURCES), {}).get(W.DSA_BY_NAME[args.dsa_workload].name)
    roof["traffic"] = per_tok * model["tokens"] if (per_tok is not None and top == "index") else None
    roof["kernel"] = top
    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        cpu = dsa_cpu_baseline(inp, args.cpu_seconds)
    sec = total_ms / 1e3
    if rank == 0:
        print(json.dumps(dict(
            metric="sparse (DSA) decode steps/s: FP8 indexer + top-k + MLA decode over the selected tokens",
            value=K / sec, unit="steps/s", n_gpus=1, steps=K, warmup=max(3, args.warmup), ms_per_step=total_ms / K,
            higher_is_better=True, scaling="weak", vs_baseline=None, dtype="e4m3 indexer, bf16 decode",
            data="synthetic",
            config=dict(workload=dw.name, B=w.B, H=w.H, r=w.r, d_r=w.d_r, context=int(L), index_heads=dw.HI,
                        index_dim=dw.dI, top_k=k, l2="inputs larger than L2: each step streams "
                        f"{model['index']['bytes'] / 1e9:.2f} GB of indexer keys before the decode"),
            tokens_per_s=K * w.B / sec, selected_tokens=model["selected"], context_tokens=model["tokens"],
            roofline=roof, roofline_detail=dict(kernels=detail, peaks=peaks,
                                                step_roofline_us=sum(d["roofline_us"] for d in detail.values())),
            cpu_baseline=cpu, e2e=None, gpu_launches=4 * K, clocks=clocks)), flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        reference_arm(args, rank)
        return
    if args.op == "append":
        append_arm(args, rank, local)
        return
    if args.op in ("absorb", "project"):
        head_gemm_arm(args, rank, local)
        return
    if args.op == "dsa":
        dsa_arm(args, rank, local)
        return

    import torch
    import torch.distributed as dist
    import datetime
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))

    wl = W.BY_NAME[args.workload]
    if args.batch is not None and args.batch != wl.B:
        lens = wl.seq_lens if isinstance(wl.seq_lens, str) else tuple(wl.seq_lens[:1]) * args.batch
        wl = wl.with_(B=args.batch, seq_lens=lens, name=f"{wl.name}_b{args.batch}")
    E = args.e2e_steps if args.e2e_steps is not None else max(1, min(args.steps, 50))
    head = decode_workload(args, wl, world, rank, local, E, args.cpu_seconds)
    # the other workloads of the pages (one GPU only: the scaling runs time the headline alone)
    extra = {}
    if world == 1 and not args.only and args.batch is None:
        for other in W.WORKLOADS[1:]:
            if other.name != wl.name:
                extra[other.name] = decode_workload(args, other, world, rank, local, 0, args.extra_cpu_seconds)

    if rank == 0:
        r = head
        line = dict(
            metric=METRIC, value=r["value"], unit="TB/s", n_gpus=world, steps=args.steps, warmup=args.warmup,
            ms_per_step=r["ms_per_step"], higher_is_better=True, scaling="weak", vs_baseline=None,
            dtype=r["dtype"], data="synthetic", config=r["config"], tflops=r["tflops"], steps_per_s=r["steps_per_s"],
            tokens_per_s=r["tokens_per_s"], step_ms_stats=r["step_ms_stats"], roofline=r["roofline"],
            roofline_detail=r["roofline_detail"], cpu_baseline=r["cpu_baseline"], e2e=r["e2e"],
            gpu_launches=2 * args.steps, clocks=r["clocks"])
        if extra:
            line["workloads"] = {name: {k: v for k, v in x.items() if k not in ("e2e", "value")} | {"tb_s": x["value"]}
                                 for name, x in extra.items()}
            line["gpu_launches"] += 2 * args.steps * len(extra)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def decode_workload(args, wl, world, rank, local, E, cpu_seconds):
    """Time K decode steps of workload `wl` (CUDA events from mla_decode_timed on the launching
    stream, max over ranks), then E end-to-end steps through mla_decode_host_io, then the oracle
    on a bounded sample. Returns the figures of the JSON line for this workload."""
    import torch
    import torch.distributed as dist
    import head_latent_attention_split_b200 as mla
    inp = W.make_inputs(wl, threads=max(1, (os.cpu_count() or 1) // world))
    t = W.to_torch(inp, f"cuda:{local}")
    p = mla.params_for(t["q_lat"], t["q_rope"], t["kv_cache"], t["block_table"], wl.scale, wl.causal,
                       num_workers=args.num_workers, kernel=args.kernel)
    kernel, workers = mla.resolve(p)
    ws = torch.empty(max(1, mla.workspace_size(p)), dtype=torch.uint8, device=t["q_lat"].device)
    out = torch.empty(t["q_lat"].shape, dtype=torch.bfloat16 if wl.out_dtype == W.BF16 else torch.float32,
                      device=t["q_lat"].device)
    lse = torch.empty(t["q_lat"].shape[:3], dtype=torch.float32, device=t["q_lat"].device)
    model = work_model(inp)
    props = torch.cuda.get_device_properties(local)
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20)
    resident = sum(x.numel() * x.element_size() for k, x in t.items() if k != "workload" and x is not None)
    flush = model["cache_bytes"] < 8 * l2
    flush_buf = torch.empty(2 * l2 // 4 + 1, dtype=torch.float32, device=out.device) if flush else None

    def step(ev=None):
        if ev is None:
            mla.mla_decode(p, t["q_lat"], t["q_rope"], t["kv_cache"], t["k_rope_cache"], t["kv_scale"],
                           t["block_table"], t["seq_lens"], out, lse, ws)
        else:
            mla.mla_decode_timed(p, t["q_lat"], t["q_rope"], t["kv_cache"], t["k_rope_cache"], t["kv_scale"],
                                 t["block_table"], t["seq_lens"], out, lse, ws, ev)

    for _ in range(max(3, args.warmup)):
        if flush:
            flush_buf.fill_(1.0)
        step()
    torch.cuda.synchronize()
    st = mla.device_status()
    if st != 0:
        raise RuntimeError(f"{wl.name}: device status {mla.status_string(st)}")

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    for e in evs:          # create the underlying CUDA events
        for x in e:
            x.record()
    torch.cuda.synchronize()
    gpu_id = getattr(props, "uuid", None)
    sampler = ClockSampler(f"GPU-{gpu_id}" if gpu_id is not None else local)
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.mark_start()
    for i in range(K):
        if flush:
            flush_buf.fill_(1.0)
        step(evs[i])
    torch.cuda.synchronize()
    sampler.mark_end()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    step_ms = [e[0].elapsed_time(e[2]) for e in evs]
    dec_ms = [e[0].elapsed_time(e[1]) for e in evs]
    comb_ms = [e[1].elapsed_time(e[2]) for e in evs]
    total_ms = reduce_max(sum(step_ms), world, out.device)
    st = mla.device_status()
    if st != 0:
        raise RuntimeError(f"{wl.name}: device status {mla.status_string(st)}")

    # end-to-end through the host-buffer entry point: per-step inputs copied from pinned
    # host memory, result copied back, all inside the timed region
    e2e = None
    if E > 0:
        pin = lambda x: x.cpu().pin_memory()  # noqa: E731
        hq, hqr, hbt, hsl = pin(t["q_lat"]), pin(t["q_rope"]), pin(t["block_table"]), pin(t["seq_lens"])
        hout = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        hlse = torch.empty(lse.shape, dtype=torch.float32, pin_memory=True)
        hws = torch.empty(mla.host_io_workspace_size(p), dtype=torch.uint8, device=out.device)
        h2d = sum(x.numel() * x.element_size() for x in (hq, hqr, hbt, hsl))
        d2h = hout.numel() * hout.element_size() + hlse.numel() * 4
        e2e_ms = 0.0
        for i in range(E + 2):
            if flush:
                flush_buf.fill_(1.0)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            mla.mla_decode_host_io(p, hq, hqr, t["kv_cache"], t["k_rope_cache"], t["kv_scale"], hbt, hsl, hout, hlse,
                                   hws)
            b.record()
            b.synchronize()
            if i >= 2:
                e2e_ms += a.elapsed_time(b)
        e2e_ms = reduce_max(e2e_ms, world, out.device)
        e2e = dict(value=job_rate_tbs(world, E, model["cache_bytes"], e2e_ms), unit="TB/s", h2d_bytes_per_step=h2d,
                   d2h_bytes_per_step=d2h, ms_per_step=e2e_ms / E)
        del hws

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu, _ = cpu_oracle_rate(inp, cpu_seconds)
    del t, ws, out, lse, flush_buf
    torch.cuda.empty_cache()

    peaks = load_peaks()
    sec = total_ms / 1e3
    dec_s = statistics.mean(dec_ms) / 1e3
    t_hbm = model["bytes"] / (peaks["hbm_gbs"] * 1e9)
    t_tc = model["flops"] / (peaks["bf16_tflops"] * 1e12)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    if bound == "hbm":
        achieved, peak, unit = model["bytes"] / dec_s / 1e9, peaks["hbm_gbs"], "GB/s"
    else:
        achieved, peak, unit = model["flops"] / dec_s / 1e12, peaks["bf16_tflops"], "TFLOP/s"
    stats = lambda xs: dict(mean=statistics.mean(xs), median=statistics.median(xs), min=min(xs))  # noqa: E731
    return dict(
        value=job_rate_tbs(world, K, model["cache_bytes"], total_ms), ms_per_step=total_ms / K,
        dtype=W.DTYPE_NAMES[wl.cache_dtype] if wl.cache_dtype != W.E4M3 else "e4m3+bf16",
        config=dict(workload=wl.name, B=wl.B, Sq=wl.Sq, H=wl.H, r=wl.r, d_r=wl.d_r, block_size=wl.block_size,
                    context=str(wl.seq_lens) if isinstance(wl.seq_lens, str) else int(max(wl.seq_lens)),
                    cache=W.DTYPE_NAMES[wl.cache_dtype], kernel=kernel, workers=workers,
                    parallelism=f"replicas x{world}" if world > 1 else "single GPU",
                    l2=("flushed between steps (2x L2 buffer write)" if flush else
                        f"inputs larger than L2 ({model['cache_bytes'] / 1e9:.2f} GB cache per step)"),
                    resident_bytes=resident),
        tflops=world * K * model["flops"] / sec / 1e12, steps_per_s=K / sec, tokens_per_s=world * K * wl.B * wl.Sq / sec,
        step_ms_stats=dict(step=stats(step_ms), decode=stats(dec_ms), combine=stats(comb_ms)),
        roofline=dict(bound=bound, achieved=achieved, peak=peak, unit=unit, frac=achieved / peak,
                      traffic=measured_traffic(wl, model, kernel)),
        roofline_detail=dict(
            kernel=f"decode ({kernel})", decode_ms=1e3 * dec_s, combine_ms=statistics.mean(comb_ms),
            algorithmic_bytes=model["bytes"], algorithmic_flops=model["flops"],
            hbm_gbs_achieved=model["bytes"] / dec_s / 1e9, tflops_achieved=model["flops"] / dec_s / 1e12,
            hbm_frac=model["bytes"] / dec_s / 1e9 / peaks["hbm_gbs"],
            tensor_frac=model["flops"] / dec_s / 1e12 / peaks["bf16_tflops"],
            roofline_us=1e6 * max(t_hbm, t_tc), step_frac=max(t_hbm, t_tc) / (total_ms / K / 1e3),
            peaks=peaks),
        cpu_baseline=cpu, e2e=e2e, clocks=clocks)


if __name__ == "__main__":
    main()
