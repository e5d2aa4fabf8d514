"""Benchmark of the MSA forward hot path on B200.

One step = the whole prefill forward (Index Branch kernel + inverse index +
KV-outer attention + merge) over one 131072-token sequence shaped like the
pages' setting (H_q=32, H_kv=4, d_h=128, d_idx=64, B_k=128, k=16; seeded
synthetic inputs with a sink block and retrieval blocks).  Inputs (Q alone is
1.07 GB) are larger than the 126 MB L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl msa|reference]
                    [--workload 128k|32k|1m|varlen|decode|decode_fp8] [--no-also]

On one GPU the 128K line also carries, under "also", the other parts of the
metric and the path's other workloads, each measured the same way: the
1M-token prefill ("1m", 3 steps after 2 warm-up steps), a packed batch of 32
prefill sequences of mixed lengths, 131072 tokens in all ("varlen"), the
64-sequence decode workload ("decode", 1000 steps after 10 warm-up steps, us
per token) and the same decode on a paged FP8 (E4M3) cache ("decode_fp8").
For N > 1 each rank runs an
independent replica (its own sequence): the path has no exchange step, so
there is no collective on the data path; timing is the max over ranks and
``value`` is the tokens of all ranks per second.  ``--impl reference`` times
the CPU oracle on a bounded sample instead (query rows of the prefill, or a
few sequences of the decode workload).  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import re
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of a kernel from
# one ncu capture, per unit of work, with the SHA-256 of the kernel's
# definition (comments and blank lines removed) at capture time: the figure is
# reported only while that code is unchanged.
# kernel -> (source, kernel function, sha256, bytes per unit, unit)
NCU_TRAFFIC = {
    "attn_phase1": ("sparse_attn.cu", "attn_phase1_kernel",
                    "f1b0fc93e3f2bf85ed14c4b8f528f468a9d3856cb1a9f7aeea45eaeb627e8f25",
                    (3576701184 + 4184357120) / 32768, "query"),
}


def kernel_code_hash(text: str, name: str) -> str:
    """SHA-256 of a kernel's definition in a CUDA source: from its name to the
    brace that closes its body, comments and blank lines removed."""
    import hashlib

    code = re.sub(r"//[^\n]*", "", text)
    i = code.index(name + "(")
    j = code.index("{", i)
    depth, k = 0, j
    for k in range(j, len(code)):
        if code[k] == "{":
            depth += 1
        elif code[k] == "}":
            depth -= 1
            if depth == 0:
                break
    body = "\n".join(line.rstrip() for line in code[i:k + 1].splitlines() if line.strip())
    return hashlib.sha256(body.encode()).hexdigest()


def ncu_traffic(kernel: str, units: float):
    """Bytes per launch from NCU_TRAFFIC and a note on where the figure comes
    from, or (None, None): no capture, or the kernel changed since."""
    ent = NCU_TRAFFIC.get(kernel)
    if ent is None:
        return None, None
    src, fn, sha, per_unit, unit = ent
    path = os.path.join(ROOT, "block_sparse_gqa_idx_b200", "csrc", src)
    with open(path, encoding="utf-8") as f:
        if kernel_code_hash(f.read(), fn) != sha:
            return None, None
    return per_unit * units, f"one ncu capture of {fn}, scaled by {unit}s"


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def dist_init():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


class Clocks:
    """nvidia-smi sampling during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, interval_ms: int = 20):
        self.dev = device_index
        self.interval = interval_ms
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", str(self.interval)], stdout=open(self.path, "w"),
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        # wait (up to 3 s) for the first sample, so a short timed region is
        # not over before the sampler has started
        t0 = time.time()
        while time.time() - t0 < 3.0 and os.path.getsize(self.path) == 0:
            time.sleep(0.01)
        self.skip = sum(1 for _ in open(self.path))

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for n, line in enumerate(f):
                p = [x.strip() for x in line.split(",")]
                if n >= getattr(self, "skip", 0) and len(p) >= 9:
                    rows.append(p)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[j] for r in rows for j in range(4) if r[5 + j].lower() == "active"})
        hi = [x for x in sm if mx and x > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(hi) if hi else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def max_over_ranks(value: float, device, world: int) -> float:
    """The step time every rank saw, reduced with MAX (timing is the slowest
    replica's).  device: where the collective's tensor lives (cuda for NCCL,
    cpu for gloo)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tokens_per_s(world: int, tokens_per_rank: int, ms_max: float) -> float:
    """Whole-job throughput of independent replicas: all ranks' tokens over the
    slowest rank's time."""
    return world * tokens_per_rank / (ms_max * 1e-3)


def workload(name: str):
    from block_sparse_gqa_idx_b200 import inputs

    return inputs.CONFIGS[name]


def flops_of(cfg):
    """Eq. 12 (xllm-io review): index term H_kv*d_idx*N^2, main term 4*N*H_q*k*B_k*d_h,
    summed over the sequences of a packed batch."""
    lengths = cfg.lengths() if hasattr(cfg, "lengths") else [cfg.N]
    f_idx = cfg.H_kv * cfg.d_idx * float(sum(float(n) ** 2 for n in lengths))
    f_main = 4.0 * cfg.N * cfg.H_q * cfg.k * cfg.B_k * cfg.d_h
    return f_idx, f_main


def selected_key_flops(cfg) -> float:
    """The main term without Eq. 12's k full blocks per query: 4*H_q*d_h per
    visible selected key, where query i (position within its sequence) sees
    min(k-1, i // B_k) earlier full blocks and the i % B_k + 1 keys of its
    own block.  Below Eq. 12 for the first k blocks of every sequence, so it
    is the count a batch of short sequences is measured against."""
    lengths = cfg.lengths() if hasattr(cfg, "lengths") else [cfg.N]
    keys = 0
    for n in lengths:
        i = np.arange(int(n), dtype=np.int64)
        keys += int((np.minimum(cfg.k - 1, i // cfg.B_k) * cfg.B_k + i % cfg.B_k + 1).sum())
    return 4.0 * cfg.H_q * cfg.d_h * float(keys)


# ------------------------------------------------------------ reference arm --
def run_reference(args, cfg, rank, world):
    """The CPU oracle on a bounded row sample of the prefill workload."""
    if rank != 0:
        return 0
    import oracle
    from block_sparse_gqa_idx_b200 import inputs

    varlen = isinstance(cfg, inputs.VarlenConfig)
    if varlen:
        inp, cu = inputs.varlen_inputs(cfg.prefill, cfg.lengths())
    else:
        inp = inputs.prefill_inputs(cfg)
    rng = np.random.default_rng(7)
    n_rows = args.ref_rows
    times = []
    for it in range(args.warmup + args.steps):
        rows = np.sort(rng.choice(cfg.N, size=n_rows, replace=False))
        t0 = time.perf_counter()
        if varlen:
            oracle.forward_varlen(inp, cu, cfg.B_k, cfg.k, rows=rows)
        else:
            oracle.forward(inp, cfg.B_k, cfg.k, rows=rows)
        dt = time.perf_counter() - t0
        if it >= args.warmup:
            times.append(dt)
    tps = n_rows / statistics.mean(times)
    line = {
        "impl": "reference", "metric": METRIC, "value": tps, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.mean(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "N": cfg.N, "H_q": cfg.H_q, "H_kv": cfg.H_kv,
                   "d_h": cfg.d_h, "d_idx": cfg.d_idx, "B_k": cfg.B_k, "k": cfg.k,
                   "parallelism": f"replicas x{world}", "rows_per_step": n_rows},
        "cpu_baseline": {"value": tps, "unit": "tokens/s", "cores": oracle.max_threads(),
                         "kind": "oracle",
                         "sample": f"{n_rows} uniformly drawn query rows per step of the {cfg.name} "
                                   f"workload (full causal prefix each)"},
        "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def is_fp8(cfg) -> bool:
    return cfg.name.startswith("decode_fp8")


def decode_state_of(cfg, seed=None):
    from block_sparse_gqa_idx_b200 import inputs

    return (inputs.decode_fp8_state(cfg, seed=seed) if is_fp8(cfg)
            else inputs.decode_state(cfg, seed=seed))


def decode_oracle_sample(st, cfg, n_seq: int, step: int = 0):
    """Time the oracle's decode step (append + Eq. 6-8 for the new token) on
    the first n_seq sequences of a decode state, bf16 or paged FP8:
    (us per token, seconds, cores)."""
    import oracle
    from block_sparse_gqa_idx_b200 import inputs

    si = inputs.decode_step_inputs(cfg, step, st["sink"])
    seqs = list(range(min(n_seq, cfg.S)))
    t0 = time.perf_counter()
    if is_fp8(cfg):
        oracle.paged_decode_fp8(st, si, st["seq_len"], cfg.B_k, cfg.k, seqs=seqs)
        cores = 1  # the paged FP8 oracle runs on one thread
    else:
        oracle.decode_reference(st, si, cfg.B_k, cfg.k, seqs=seqs)
        cores = oracle.max_threads()
    dt = time.perf_counter() - t0
    return 1e6 * dt / len(seqs), dt, cores


def run_reference_decode(args, cfg, rank, world):
    """The CPU oracle's decode step on a few sequences of the decode workload."""
    if rank != 0:
        return 0
    from block_sparse_gqa_idx_b200 import inputs

    st = decode_state_of(cfg)
    n_seq = args.ref_seqs
    times = []
    for it in range(args.warmup + args.steps):
        us, dt, cores = decode_oracle_sample(st, cfg, n_seq, step=it)
        if it >= args.warmup:
            times.append(us)
    us = statistics.mean(times)
    line = {
        "impl": "reference", "metric": METRIC, "value": us, "unit": "us/token",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": us * n_seq * 1e-3, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "S": cfg.S, "L0": cfg.L0, "H_q": cfg.H_q,
                   "H_kv": cfg.H_kv, "d_h": cfg.d_h, "d_idx": cfg.d_idx, "B_k": cfg.B_k,
                   "k": cfg.k, "parallelism": f"replicas x{world}", "seqs_per_step": n_seq},
        "cpu_baseline": {"value": us, "unit": "us/token", "cores": cores, "kind": "oracle",
                         "sample": f"{n_seq} of the {cfg.S} sequences per step (one token each, "
                                   f"full cache scan)"},
        "e2e": {"value": us, "unit": "us/token", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


METRIC = "MSA fwd prefill tokens/s @128K & 1M, % bf16 TC peak; decode µs/token, % HBM BW"


def tensor_roofline(work_flop: float, per_launch_ms: float, pk: dict, pk_kind: str) -> dict:
    """Achieved TFLOP/s of one launch against the measured burst bf16 peak
    (the headline fraction) and, as a second figure, the sustained one."""
    achieved = work_flop / (per_launch_ms * 1e-3) / 1e12
    return {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"],
            "unit": "TFLOP/s", "frac": achieved / pk["bf16_tflops"],
            "peak_kind": f"{pk_kind} burst",
            "frac_of_sustained": achieved / pk["bf16_tflops_sustained"]}


# ----------------------------------------------------------------- msa arm --
def run_msa(args, cfg, rank, world, local, steps, warmup, e2e_steps, cpu_rows):
    """Time `steps` prefill forwards of one sequence per rank; returns the JSON
    line on rank 0 (None elsewhere)."""
    import torch
    import torch.distributed as dist

    import block_sparse_gqa_idx_b200 as msa
    from block_sparse_gqa_idx_b200 import inputs

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)

    # every replica gets its own seeded sequence (or packed batch)
    varlen = isinstance(cfg, inputs.VarlenConfig)
    t_gen = time.time()
    if varlen:
        inp, cu = inputs.varlen_inputs(cfg.prefill, cfg.lengths(), seed=cfg.seed + 1000 * rank)
    else:
        inp = inputs.prefill_inputs(cfg, seed=cfg.seed + 1000 * rank)
    gen_s = time.time() - t_gen
    host = {k: torch.from_numpy(np.ascontiguousarray(v).view(np.int16)).view(torch.bfloat16)
            for k, v in inp.items()}
    d = {k: v.to(dev) for k, v in host.items()}
    N, H_q, H_kv, d_h, d_idx, B_k, kk = cfg.N, cfg.H_q, cfg.H_kv, cfg.d_h, cfg.d_idx, cfg.B_k, cfg.k
    idx = torch.empty((N, H_kv, kk), dtype=torch.int32, device=dev)
    o = torch.empty((N, H_q, d_h), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((N, H_q), dtype=torch.float32, device=dev)
    dims = msa.dims(N, H_q, H_kv, d_h, d_idx, B_k, kk)
    if varlen:
        if args.kl_lse:
            raise SystemExit("--kl-lse runs on one sequence per replica, not a packed batch")
        ws_bytes = msa.varlen_workspace_size(cu, N, H_q, H_kv, d_h, d_idx, B_k, kk)
    else:
        ws_bytes = max(msa.sparse_attn_fwd_workspace_size(dims), msa.index_topk_workspace_size(dims),
                       msa.index_lse_workspace_size(dims))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    lse_idx = torch.empty((N, H_kv), dtype=torch.float32, device=dev) if args.kl_lse else None

    def step(src, o_, idx_, lse_):
        if varlen:
            msa.index_topk_varlen(src["q_idx"], src["k_idx"], cu, B_k, kk, idx_out=idx_,
                                  workspace=ws, stream=stream)
            msa.sparse_attn_fwd_varlen(src["q"], src["k"], src["v"], idx_, cu, B_k, o=o_,
                                       lse=lse_, workspace=ws, stream=stream)
            return
        msa.index_topk(src["q_idx"], src["k_idx"], B_k, kk, idx_out=idx_, workspace=ws,
                       stream=stream)
        msa.sparse_attn_fwd(src["q"], src["k"], src["v"], idx_, B_k, o=o_, lse=lse_,
                            workspace=ws, stream=stream)
        if args.kl_lse:  # the KL-loss fusion's Index Branch normaliser (training forward)
            msa.index_lse(src["q_idx"], src["k_idx"], idx_, B_k, lse_idx=lse_idx, workspace=ws,
                          stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(warmup):
        step(d, o, idx, lse)
    torch.cuda.synchronize()
    code, where = msa.device_status(ws)
    if code != 0:
        raise RuntimeError(f"device status {code} at {where} after warm-up")

    clocks = Clocks(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step(d, o, idx, lse)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, dev, world)
    # the per-kernel split from a second pass with an event pair around
    # every launch (kept out of the timed pass: events between the kernels
    # would stand in the way of overlapped launches)
    msa.profile_enable(True)
    for _ in range(steps):
        step(d, o, idx, lse)
    torch.cuda.synchronize()
    msa.profile_enable(False)
    prof = msa.profile_read()
    value = aggregate_tokens_per_s(world, N, ms)
    code, where = msa.device_status(ws)
    if code != 0:
        raise RuntimeError(f"device status {code} at {where} after the timed steps")

    # ---- end to end: pinned host inputs -> device -> forward -> host result.
    # Every step uploads its inputs from pinned host memory and downloads its
    # outputs (O and the selection); uploads run on one copy stream, downloads
    # on another, so step n+1's upload and step n-1's download overlap step
    # n's compute (device inputs and outputs are double-buffered).
    pinned = {k: v.pin_memory() for k, v in host.items()}
    bufs = [d, {k: torch.empty_like(v) for k, v in d.items()}]
    outs = [(o, idx, lse), (torch.empty_like(o), torch.empty_like(idx), torch.empty_like(lse))]
    o_host = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]
    idx_host = [torch.empty(idx.shape, dtype=idx.dtype).pin_memory() for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = o.numel() * o.element_size() + idx.numel() * idx.element_size()
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]      # inputs uploaded
    ev_used = [torch.cuda.Event() for _ in range(2)]    # inputs consumed
    ev_out = [torch.cuda.Event() for _ in range(2)]     # outputs computed
    ev_read = [torch.cuda.Event() for _ in range(2)]    # outputs downloaded

    def e2e_run(n):
        for j in range(2):
            ev_used[j].record(stream)
            ev_read[j].record(stream)
        for j in range(n):
            b = j & 1
            with torch.cuda.stream(up):
                up.wait_event(ev_used[b])
                for k, v in pinned.items():
                    bufs[b][k].copy_(v, non_blocking=True)
                ev_in[b].record(up)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_read[b])
            ob, ib, lb = outs[b]
            step(bufs[b], ob, ib, lb)
            ev_used[b].record(stream)
            ev_out[b].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(ev_out[b])
                o_host[b].copy_(ob, non_blocking=True)
                idx_host[b].copy_(ib, non_blocking=True)
                ev_read[b].record(down)
        stream.wait_stream(up)
        stream.wait_stream(down)

    e2e_run(2)
    torch.cuda.synchronize()
    barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    e2e_run(e2e_steps)
    f1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1) / e2e_steps, dev, world)
    barrier()
    del pinned, bufs, outs, o_host, idx_host
    if rank != 0:
        return None

    # ---- roofline of the dominant kernel (live CUDA-event durations)
    pk, pk_kind = peaks()
    f_idx, f_main = flops_of(cfg)
    if varlen:
        # short sequences select fewer than k blocks: count the keys selected
        f_main = selected_key_flops(cfg)
    total_ms = sum(v[1] for v in prof.values())
    dom = max(prof, key=lambda n: prof[n][1])
    launches, dom_ms = prof[dom]
    per_launch_ms = dom_ms / launches
    if dom == "index_topk":
        roofline = tensor_roofline(f_idx, per_launch_ms, pk, pk_kind)
    elif dom == "attn_phase1":
        # one launch per query chunk and step: the Main Branch FLOPs of a chunk
        roofline = tensor_roofline(f_main / (launches / steps), per_launch_ms, pk, pk_kind)
    else:
        roofline = {"bound": "hbm", "achieved": None, "peak": pk["hbm_gbs"], "unit": "GB/s",
                    "frac": None, "peak_kind": pk_kind}
    # the captured bytes scale with N k; a packed batch of short sequences
    # selects fewer blocks per query, so it gets no figure
    traffic, traffic_src = (None, None) if varlen else ncu_traffic(dom, N / (launches / steps))
    roofline = {"kernel": dom, **roofline, "traffic": traffic, "traffic_source": traffic_src,
                "share": dom_ms / total_ms if total_ms else None}
    # each tensor-bound kernel against the same peak
    per_kernel = {}
    for name, work in (("index_topk", f_idx), ("attn_phase1", f_main)):
        if name in prof:
            nl, tms = prof[name]
            per_kernel[name] = tensor_roofline(work / (nl / steps), tms / nl, pk, pk_kind)

    # ---- CPU oracle on a bounded sample (rank 0, N=1 only)
    cpu = None
    if world == 1 and cpu_rows > 0:
        import oracle

        rng = np.random.default_rng(11)
        rows = np.sort(rng.choice(N, size=cpu_rows, replace=False))
        t0 = time.perf_counter()
        if varlen:
            oracle.forward_varlen(inp, cu, B_k, kk, rows=rows)
        else:
            oracle.forward(inp, B_k, kk, rows=rows)
        dt = time.perf_counter() - t0
        cpu = {"value": cpu_rows / dt, "unit": "tokens/s", "cores": oracle.max_threads(),
               "kind": "oracle",
               "sample": f"{cpu_rows} uniformly drawn query rows of the {cfg.name} workload "
                         f"(index + attention, full causal prefix), {dt:.1f} s"}

    kernels = {n: {"launches": v[0], "ms_per_step": v[1] / steps,
                   "share": v[1] / total_ms if total_ms else None} for n, v in prof.items()}
    backward = None
    if world == 1 and not varlen and getattr(args, "backward", False) and cfg.name == args.workload:
        backward = time_backward(msa, d, idx, o, lse, cfg, stream, f_main, pk, pk_kind)
    # time between kernels: the timed step minus the kernels' summed event
    # times from the profiled pass
    idle = max(0.0, ms - total_ms / steps)
    return {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": steps, "warmup": warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": cfg.name, "N": N, "H_q": H_q, "H_kv": H_kv, "d_h": d_h,
                   "d_idx": d_idx, "B_k": B_k, "k": kk, "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (Q alone %.2f GB); no flush"
                         % (N * H_q * d_h * 2 / 1e9),
                   "kl_lse": bool(args.kl_lse),
                   **({"n_seqs": cfg.n_seqs, "lengths": f"log-uniform in [{cfg.len_lo}, "
                       f"{cfg.len_hi}], min {int(np.min(np.diff(cu)))}, max "
                       f"{int(np.max(np.diff(cu)))}"} if varlen else {})},
        "tc_frac_eq12": (f_idx + f_main) / (ms * 1e-3) / 1e12 / pk["bf16_tflops"],
        "main_flops": ("selected visible keys, 4*H_q*d_h each" if varlen
                       else "Eq. 12 main term, 4*N*H_q*k*B_k*d_h"),
        "roofline": roofline,
        "roofline_per_kernel": per_kernel,
        "cpu_baseline": cpu,
        "e2e": {"value": aggregate_tokens_per_s(world, N, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "steps": e2e_steps,
                "note": "pinned host -> device -> forward -> host every step; copies of "
                        "neighbouring steps overlap compute on two copy streams"},
        "gpu_launches": sum(v[0] for v in prof.values()),
        "kernels": kernels,
        "idle_ms_per_step": idle, "idle_frac": idle / ms if ms else None,
        "clocks": clk,
        "input_generation_s": gen_s,
        **({"backward": backward} if backward is not None else {}),
    }


def time_backward(msa, d, idx, o, lse, cfg, stream, f_main, pk, pk_kind, steps=3, warmup=1):
    """The backward of the Main Branch (dQ, dK, dV with the selection fixed)
    after the timed forward steps: seeded dO, the last forward's O, LSE and
    selection; CUDA events on the stream.  Its work is the five GEMMs per
    selected key (S recomputed, dP, dQ, dK, dV): 2.5x the forward's main term."""
    import torch

    gen = torch.Generator(device=o.device).manual_seed(1234)
    d_o = torch.randn(o.shape, generator=gen, device=o.device, dtype=torch.float32).to(o.dtype)
    ws = torch.empty(msa.sparse_attn_bwd_workspace_size(
        msa.dims(cfg.N, cfg.H_q, cfg.H_kv, cfg.d_h, cfg.d_idx, cfg.B_k, cfg.k)),
        dtype=torch.uint8, device=o.device)

    def run():
        return msa.sparse_attn_bwd(d["q"], d["k"], d["v"], idx, o, lse, d_o, cfg.B_k,
                                   workspace=ws, stream=stream)

    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    msa.profile_enable(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        run()
    e1.record(stream)
    torch.cuda.synchronize()
    msa.profile_enable(False)
    prof = msa.profile_read()
    code, where = msa.device_status(ws)
    if code != 0:
        raise RuntimeError(f"device status {code} at {where} in the backward")
    ms = e0.elapsed_time(e1) / steps
    flops = 2.5 * f_main
    return {"ms_per_step": ms, "value": cfg.N / (ms * 1e-3), "unit": "tokens/s",
            "steps": steps, "warmup": warmup,
            "achieved_tflops": flops / (ms * 1e-3) / 1e12,
            "frac": flops / (ms * 1e-3) / 1e12 / pk["bf16_tflops"], "peak_kind": pk_kind,
            "flops": "2.5x the Eq. 12 main term (S, dP, dQ, dK, dV per selected key)",
            "kernels": {n: {"launches": v[0], "ms_per_step": v[1] / steps}
                        for n, v in prof.items()}}


# -------------------------------------------------------------- decode arm --
def run_decode(args, cfg, rank, world, local, steps, warmup, e2e_steps, cpu_seqs):
    """Decode workload: S sequences, one new token each per step (append +
    index scan + Top-k + gathered attention).  Reports us per token (the step
    time divided by the sequences of all ranks), us per step, and the HBM
    roofline of the step from its algorithmic bytes; returns the line on rank 0."""
    import torch

    import block_sparse_gqa_idx_b200 as msa
    from block_sparse_gqa_idx_b200 import inputs

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    fp8 = is_fp8(cfg)
    t0 = time.time()
    st = decode_state_of(cfg, seed=cfg.seed + 1000 * rank)
    gen_s = time.time() - t0

    def dv(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    if fp8:
        caches = {k: torch.from_numpy(np.ascontiguousarray(st[k])).to(dev)
                  for k in ("k_pages", "v_pages", "kidx_pages", "k_scale", "v_scale", "kidx_scale",
                            "page_table")}
    else:
        caches = {k: dv(st[k]) for k in ("k_cache", "v_cache", "k_idx_cache")}
    seq_len = torch.from_numpy(st["seq_len"]).to(dev)
    prof_steps = max(1, min(steps, 100))
    n_steps = warmup + steps + prof_steps + e2e_steps
    assert n_steps <= cfg.steps, "more steps than the cache has room for"
    host_in = [inputs.decode_step_inputs(cfg, j, st["sink"]) for j in range(n_steps)]
    steps_in = [{k: dv(v) for k, v in h.items()} for h in host_in[:warmup + steps + prof_steps]]
    S, H_q, H_kv, d_h, d_idx, B_k, kk = cfg.S, cfg.H_q, cfg.H_kv, cfg.d_h, cfg.d_idx, cfg.B_k, cfg.k
    o = torch.empty((S, H_q, d_h), dtype=torch.bfloat16, device=dev)
    idx = torch.empty((S, H_kv, kk), dtype=torch.int32, device=dev)
    if fp8:
        dd = msa.paged_dims(S, st["page_table"].shape[1], st["k_pages"].shape[0], H_q, H_kv, d_h,
                            d_idx, B_k, kk)
        ws = torch.empty(msa.paged_decode_fp8_workspace_size(dd), dtype=torch.uint8, device=dev)
    else:
        dd = msa.decode_dims(S, cfg.L_max, H_q, H_kv, d_h, d_idx, B_k, kk)
        ws = torch.empty(msa.sparse_decode_workspace_size(dd), dtype=torch.uint8, device=dev)

    def step(x):
        if fp8:
            c = caches
            msa.paged_decode_fp8(x["q"], x["q_idx"], x["k_new"], x["v_new"], x["k_idx_new"],
                                 c["k_pages"], c["k_scale"], c["v_pages"], c["v_scale"],
                                 c["kidx_pages"], c["kidx_scale"], c["page_table"], seq_len, B_k,
                                 kk, o=o, idx_out=idx, workspace=ws, stream=stream)
        else:
            msa.sparse_decode(x["q"], x["q_idx"], x["k_new"], x["v_new"], x["k_idx_new"],
                              caches["k_cache"], caches["v_cache"], caches["k_idx_cache"], seq_len,
                              B_k, kk, o=o, idx_out=idx, workspace=ws, stream=stream)

    def barrier():
        if world > 1:
            import torch.distributed as dist

            dist.barrier()

    for j in range(warmup):
        step(steps_in[j])
    torch.cuda.synchronize()
    L_before = seq_len.clone()
    clocks = Clocks(local, interval_ms=10)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for j in range(warmup, warmup + steps):
        step(steps_in[j])
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    # the slowest replica's step time; every rank's S sequences got a token
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, dev, world)
    code, where = msa.device_status(ws)
    if code != 0:
        raise RuntimeError(f"device status {code} at {where}")
    # algorithmic bytes per step: the K_idx scan of every cached token, the
    # selected K and V rows (causal part of each block), the new rows and q/o
    L = L_before.double().mean().item() + (steps - 1) / 2.0
    sel_rows = 0.0
    sel = idx.cpu().numpy()
    Lend = seq_len.cpu().numpy()
    for s_ in range(S):
        Li = int(Lend[s_])  # length after the last timed step (query at Li-1)
        for r in range(H_kv):
            for b in sel[s_, r]:
                if b >= 0:
                    sel_rows += min(B_k, Li - int(b) * B_k)
    # the per-kernel split from a second, shorter pass with an event pair
    # around every launch (kept out of the timed pass)
    msa.profile_enable(True)
    for j in range(warmup + steps, warmup + steps + prof_steps):
        step(steps_in[j])
    torch.cuda.synchronize()
    msa.profile_enable(False)
    prof = msa.profile_read()
    if fp8:
        # one byte per code plus a 4-byte scale per token (and head); the new
        # rows arrive in bf16 and are written as codes and scales
        bytes_step = (S * L * (d_idx + 4) + sel_rows * 2 * (d_h + 4)
                      + S * (H_q * d_h * 2 * 2 + H_kv * d_idx * 2 + H_kv * d_h * 2 * 2
                             + d_idx * 2 + 2 * H_kv * (d_h + 4) + d_idx + 4))
    else:
        bytes_step = (S * L * d_idx * 2 + sel_rows * d_h * 2 * 2
                      + S * (H_q * d_h * 2 * 2 + H_kv * d_idx * 2 + H_kv * d_h * 2 * 2 * 2
                             + d_idx * 2 * 2))

    # ---- end to end: each step's new rows from pinned host memory, the
    # step, and O and the selection back to pinned host memory
    pinned = [{k: torch.from_numpy(np.ascontiguousarray(v).view(np.int16)).view(torch.bfloat16)
               .pin_memory() for k, v in h.items()} for h in host_in[warmup + steps + prof_steps:]]
    dev_in = {k: torch.empty_like(v, device=dev) for k, v in pinned[0].items()}
    o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    idx_host = torch.empty(idx.shape, dtype=idx.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in pinned[0].values())
    d2h = o.numel() * o.element_size() + idx.numel() * idx.element_size()
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for x in pinned:
        for k, v in x.items():
            dev_in[k].copy_(v, non_blocking=True)
        step(dev_in)
        o_host.copy_(o, non_blocking=True)
        idx_host.copy_(idx, non_blocking=True)
    f1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1) / max(1, len(pinned)), dev, world)
    if rank != 0:
        return None
    pk, pk_kind = peaks()
    gbs = bytes_step / (ms * 1e-3) / 1e9
    cache_gb = (S * cfg.L_max * (2 * H_kv * (d_h + 4) + d_idx + 4) / 1e9 if fp8
                else S * cfg.L_max * (2 * H_kv * d_h + d_idx) * 2 / 1e9)
    total_ms = sum(v[1] for v in prof.values())
    kernels = {n: {"launches": v[0], "ms_per_step": v[1] / prof_steps,
                   "share": v[1] / total_ms if total_ms else None} for n, v in prof.items()}
    scan_ms = prof.get("dec8_scan" if fp8 else "dec_scan", (1, 0.0))[1] / prof_steps
    scan_bytes = S * L * (d_idx + 4) if fp8 else S * L * d_idx * 2
    cpu = None
    if world == 1 and cpu_seqs > 0:
        us_cpu, dt_cpu, cores = decode_oracle_sample(st, cfg, cpu_seqs)
        cpu = {"value": us_cpu, "unit": "us/token", "cores": cores, "kind": "oracle",
               "sample": f"{cpu_seqs} of the {S} sequences, one {'paged FP8 ' if fp8 else ''}"
                         f"decode step each (append, full K_idx scan, Top-k, attention), "
                         f"{dt_cpu:.1f} s"}
    idle = max(0.0, ms - total_ms / prof_steps)
    return {
        "metric": METRIC, "value": 1e3 * ms / (S * world),
        "unit": "us/token", "n_gpus": world, "steps": steps, "warmup": warmup,
        "ms_per_step": ms, "us_per_step": 1e3 * ms, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 cache, bf16 math" if fp8 else "bf16",
        "data": "synthetic",
        "config": {"workload": cfg.name, "S": S, "L": L, "H_q": H_q, "H_kv": H_kv, "d_h": d_h,
                   "d_idx": d_idx, "B_k": B_k, "k": kk,
                   "l2": f"caches {cache_gb:.1f} GB (K, V, K_idx{' codes and scales' if fp8 else ''}), "
                         f"larger than L2; no flush",
                   **({"pages": int(st["k_pages"].shape[0]), "page_tokens": B_k} if fp8 else {})},
        "roofline": {"kernel": "decode step", "bound": "hbm", "achieved": gbs,
                     "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": gbs / pk["hbm_gbs"],
                     "traffic": None, "bytes_per_step": bytes_step, "peak_kind": pk_kind,
                     "scan_kernel_gbs": scan_bytes / (scan_ms * 1e-3) / 1e9 if scan_ms else None},
        "cpu_baseline": cpu,
        "e2e": {"value": 1e3 * e2e_ms / (S * world), "unit": "us/token",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "us_per_step": 1e3 * e2e_ms, "steps": len(pinned),
                "note": "each step's new rows from pinned host memory, the step, and O and "
                        "the selection back to pinned host memory, in stream order"},
        "gpu_launches": sum(v[0] for v in prof.values()) * steps // prof_steps,
        "kernels": kernels, "kernel_split_steps": prof_steps,
        "idle_ms_per_step": idle, "clocks": clk, "input_generation_s": gen_s,
    }


def free_device_memory():
    import gc

    import torch

    gc.collect()
    torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="msa", choices=["msa", "reference"])
    ap.add_argument("--workload", default="128k")
    ap.add_argument("--cpu-rows", type=int, default=0, help="0: 256, or 32 at 1M tokens")
    ap.add_argument("--ref-rows", type=int, default=32)
    ap.add_argument("--ref-seqs", type=int, default=2,
                    help="sequences per step of the decode reference arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-also", action="store_true",
                    help="time only --workload (by default the 128K line also carries the "
                         "1M prefill and the decode workload)")
    ap.add_argument("--backward", action="store_true",
                    help="also time the backward of the Main Branch on the 128K/32K line "
                         "(on by default for the 128K workload)")
    ap.add_argument("--kl-lse", action="store_true",
                    help="add the KL-loss fusion's LSE_idx to every step (a training forward)")
    args = ap.parse_args()
    if args.workload == "128k" and not args.kl_lse:
        args.backward = True
    world, rank, local = dist_init()
    cfg = workload(args.workload)
    is_decode = args.workload.startswith("decode")
    if args.cpu_rows == 0:
        args.cpu_rows = 32 if getattr(cfg, "N", 0) >= (1 << 20) else 256
    if args.no_cpu_baseline:
        args.cpu_rows = 0
    if args.impl == "reference":
        if is_decode:
            return run_reference_decode(args, cfg, rank, world)
        return run_reference(args, cfg, rank, world)
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if is_decode:
            line = run_decode(args, cfg, rank, world, local, args.steps, args.warmup, 8,
                              0 if args.no_cpu_baseline else 4)
        else:
            e2e_steps = 2 if cfg.N >= (1 << 20) else max(2, min(args.steps, 6))
            line = run_msa(args, cfg, rank, world, local, args.steps, args.warmup, e2e_steps,
                           args.cpu_rows)
        # the other two parts of the metric, on one GPU: the 1M-token prefill
        # and the decode workload, each a nested line of its own
        if world == 1 and args.workload == "128k" and not args.no_also and not args.kl_lse:
            also = {}
            free_device_memory()
            c1m = workload("1m")
            also["1m"] = run_msa(args, c1m, rank, world, local, steps=3, warmup=2, e2e_steps=2,
                                 cpu_rows=0 if args.no_cpu_baseline else 32)
            free_device_memory()
            also["varlen"] = run_msa(args, workload("varlen"), rank, world, local, steps=10,
                                     warmup=3, e2e_steps=4,
                                     cpu_rows=0 if args.no_cpu_baseline else 128)
            free_device_memory()
            also["decode"] = run_decode(args, workload("decode"), rank, world, local, steps=1000, warmup=10,
                                        e2e_steps=8, cpu_seqs=0 if args.no_cpu_baseline else 4)
            free_device_memory()
            also["decode_fp8"] = run_decode(args, workload("decode_fp8"), rank, world, local,
                                            steps=1000, warmup=10, e2e_steps=8,
                                            cpu_seqs=0 if args.no_cpu_baseline else 4)
            line["also"] = also
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
        return 0
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
