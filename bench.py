#!/usr/bin/env python
"""Benchmark of the CSA2 decode hot path at a 1M-token context on B200.

Workload (default): 1 Full + 1 Reindex layer, batch 4, 1,048,576-token
context compressed 4:1 to N = 262,144 global entries per sequence, entry dim
128 (FP4 E2M1 + fp32 per-16 scales), int8 indexer 4 heads x 64, top-k 2048,
16 query heads, bf16 window 128.  Synthetic seeded inputs, resident in HBM.

A step = one decode token per sequence through both layers: index scan,
top-k, gather/dequant + attention.  L2 (126 MB) is flushed before every
layer (a 256 MiB write then a 256 MiB read, kept outside the timed events, so
L2 holds clean unrelated lines), because the 64 MiB of
index keys would otherwise stay L2-resident between the two layers that
share them and between steps.

Prints ONE JSON line (rank 0).  `value` = tokens/s/layer over all ranks
(each rank is an independent replica: weak scaling).  `--impl reference`
times the CPU oracle (test infrastructure) on the host cores instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from compressed_sparse_attention_topk_b200 import workloads as wl  # noqa: E402

METRIC = "CSA2 decode tokens/s per layer at 1M ctx; achieved HBM GB/s vs B200 peak"
UNIT = "tokens/s/layer"
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="csa2", choices=["csa2", "reference"])
    ap.add_argument("--workload", default=wl.LONG.name, choices=sorted(wl.ALL))
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU-baseline budget (oracle on the host cores)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--keys", default="int8", choices=["int8", "fp4"],
                    help="index key format of the entry stores (fp4: E2M1 with a power-of-two "
                         "scale per 32 elements; a supplementary line)")
    ap.add_argument("--decode-kernel", default="scan_cluster", choices=["scan_cluster", "fused"],
                    help="which kernels serve the decode rows: the index scan + per-row cluster "
                         "kernel (default) or the fused single-launch kernel")
    ap.add_argument("--pool", action="store_true",
                    help="hierarchical indexer: the Full layer keeps a pool of 2,048 blocks of 8 "
                         "positions from its scan and the second layer selects within that pool "
                         "(a supplementary line)")
    ap.add_argument("--append", action="store_true",
                    help="every step first appends one completed entry per sequence (FP4 "
                         "entry + int8 key, at the store's last row) in the Full layer")
    ap.add_argument("--profile", action="store_true",
                    help="device-resident steps only (no trace pass, e2e, clocks or CPU "
                         "baseline): the command ncu captures")
    return ap.parse_args()


def algorithmic_bytes(w0, key_format: str = "int8") -> dict:
    """Per (sequence, layer, token): index keys scanned + selected FP4 entries
    gathered (codes + scales) + bf16 window K and V.  FP4 index keys take
    d_I/2 code bytes + d_I/32 exponent bytes per entry."""
    keys = w0.N * (w0.d_I if key_format == "int8" else w0.d_I // 2 + w0.d_I // 32)
    gather = w0.topk * (w0.D // 2 + w0.D // 4)
    window = 2 * w0.W * w0.D * 2
    return {"keys": keys, "gather": gather, "window": window, "total": keys + gather + window}


# Algorithmic bytes of one launch of each library kernel of the decode step
# (per launch the kernel serves all B rows of one layer).
KERNEL_BYTES = {
    "index_scan": lambda w0, ab: w0.B * ab["keys"],
    "topk_attend": lambda w0, ab: w0.B * (ab["gather"] + ab["window"]),
    "attend_handoff": lambda w0, ab: w0.B * (ab["gather"] + ab["window"]),
    "decode_fused": lambda w0, ab: w0.B * ab["total"],
}


def step_traffic(kernels):
    """DRAM bytes of a step from the committed ncu summaries, when every
    kernel of the step has one (else None)."""
    tot = 0
    for k, v in kernels.items():
        t = v.get("traffic")
        if t is None:
            return None
        tot += t * v["launches_per_step"]
    return tot


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def dist_env():
    """(world size, rank, local rank) of a torchrun launch; (1, 0, 0) alone."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(dist, values, device):
    """Element-wise maximum over all ranks of per-rank device times (ms).
    Every rank calls it with the same number of values, in the same order."""
    if dist is None:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_tokens_per_s(world, steps, B, T, L, total_ms):
    """Whole-job throughput: the tokens x layers of every rank (independent
    replicas) over the slowest rank's device time."""
    return world * steps * B * T * L / (total_ms * 1e-3)


def pack_into_one_buffer(layers, keys, dev):
    """Move layers[l][k] (k in keys) into one uint8 device buffer, each tensor
    at a 256-byte aligned offset, and replace them by views of it (same dtype
    and shape).  Returns the buffer and the bytes it holds."""
    import torch
    plan, off = [], 0
    for l, d in enumerate(layers):
        for k in keys:
            if k not in d:  # a tensor only some layers hold
                continue
            nb = d[k].numel() * d[k].element_size()
            plan.append((l, k, off, nb))
            off += (nb + 255) // 256 * 256
    buf = torch.zeros(off, dtype=torch.uint8, device=dev)
    for l, k, o, nb in plan:
        t = layers[l][k]
        v = buf[o:o + nb].view(t.dtype).view(t.shape)
        v.copy_(t)
        layers[l][k] = v
    return buf, off


KERNEL_SOURCES = {
    "index_scan": ("index_scan.cuh", "pack.cuh", "common.cuh"),
    "topk_attend": ("row_cluster.cuh", "attn_rows.cuh", "pack.cuh", "common.cuh"),
    "attend_handoff": ("attn_handoff.cuh", "attn_rows.cuh", "common.cuh"),
    "decode_fused": ("decode_fused.cuh", "attn_rows.cuh", "pack.cuh", "common.cuh"),
}


def kernel_source_sha(kernel: str) -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(ROOT, "compressed_sparse_attention_topk_b200", "csrc", f),
                      "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from a committed ncu summary
    (profiles/<kernel>_traffic.json), only while the kernel's source is
    unchanged since the capture."""
    p = os.path.join(ROOT, "profiles", f"{kernel}_traffic.json")
    if kernel not in KERNEL_SOURCES or not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("source_sha") != kernel_source_sha(kernel):
        return None
    return d.get("dram_bytes_per_launch_full_size")


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.3)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "samples": len(sm), "reasons": sorted(reasons)}


# --------------------------------------------------------------------------- oracle timing

def oracle_sample(w0, seconds: float, min_runs: int = 1):
    """Time the CPU oracle on whole sequences (all layers of the workload),
    one sequence at a time, until `seconds` have passed."""
    import oracle
    layers = wl.all_layer_inputs(w0, B=1)
    for lay in layers:
        if "entries" in lay:
            B, N, D = lay["entries"].shape
            c, s = oracle.pack_fp4(lay["entries"].reshape(B * N, D))
            lay["codes"], lay["scales"] = c.reshape(B, N, D // 2), s.reshape(B, N, D // 16)
    runs, t0 = 0, time.perf_counter()
    while runs < min_runs or time.perf_counter() - t0 < seconds:
        oracle.layer_group(list(w0.modes), layers, w0.topk, w0.n_prior, w0.ratio)
        runs += 1
    dt = time.perf_counter() - t0
    return runs, dt


def oracle_rows_sample(w0, lay, seconds: float) -> dict:
    """Time the CPU oracle on query rows of a one-layer workload with several
    query tokens per sequence (index + top-k over the row's visible entries,
    then attention), eight rows per call, spread evenly over the chunk, until
    `seconds` have passed."""
    import oracle
    B, N, D = lay["entries"].shape
    c, s = oracle.pack_fp4(lay["entries"].reshape(B * N, D))
    layer = dict(lay, codes=c.reshape(B, N, D // 2), scales=s.reshape(B, N, D // 16))
    nrows = w0.B * w0.T
    order = np.arange(nrows).reshape(-1, 8).T.reshape(-1) if nrows % 8 == 0 else np.arange(nrows)
    done, t0 = 0, time.perf_counter()
    while done == 0 or time.perf_counter() - t0 < seconds:
        rows = order[done % nrows: done % nrows + 8]
        oracle.layer_group([(0, 0, 0)], [layer], w0.topk, w0.n_prior, w0.ratio, rows=rows)
        done += len(rows)
    dt = time.perf_counter() - t0
    return {"value": done / dt, "unit": "tokens/s/layer", "cores": 1, "kind": "oracle",
            "sample": f"{done} query rows, cycling over the {nrows} of one layer call in an "
                      f"order spread over the chunk, plain C oracle, single thread, {dt:.1f} s",
            **host_cpu()}


def host_cpu() -> dict:
    """The host's CPU model and logical core count (for the oracle timings);
    "unknown" where the system does not say."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "nproc": os.cpu_count() or 0}


def run_reference(args, w0):
    _, rank, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    layers = wl.all_layer_inputs(w0, B=1)
    for lay in layers:
        if "entries" in lay:
            B, N, D = lay["entries"].shape
            c, s = oracle.pack_fp4(lay["entries"].reshape(B * N, D))
            lay["codes"], lay["scales"] = c.reshape(B, N, D // 2), s.reshape(B, N, D // 16)

    def step():
        oracle.layer_group(list(w0.modes), layers, w0.topk, w0.n_prior, w0.ratio)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    tokens_layers = args.steps * 1 * w0.T * w0.L
    value = tokens_layers / dt
    sample = (f"1 of {w0.B} sequences per step ({w0.L} layers, N={w0.N}), "
              f"plain C oracle, single thread")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8/f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": w0.name, "B": w0.B, "N": w0.N, "layers": w0.L,
                   "topk": w0.topk, "parallelism": "host cores, rank 0 only"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample, **host_cpu()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- GPU arm

POOL_BLOCK, POOL_BLOCKS = 8, 2048   # the pages' example: 2,048 blocks x 8 = 16,384 candidates


def layer_bytes(w0, args, l) -> int:
    """Algorithmic bytes of layer l for one sequence and token: keys scanned
    (the whole store, or the Full layer's pool for a pool layer) + gathered
    entries + window."""
    ab = algorithmic_bytes(w0, args.keys)
    if args.pool and w0.modes[l][0] == 3:
        return POOL_BLOCK * POOL_BLOCKS * w0.d_I + ab["gather"] + ab["window"]
    return ab["total"]


def run_gpu(args, w0):
    import torch
    import compressed_sparse_attention_topk_b200 as csa2

    world, rank, local = dist_env()
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    csa2.lib()
    csa2.set_decode_kernel(csa2.DECODE_FUSED if args.decode_kernel == "fused"
                           else csa2.DECODE_SCAN_CLUSTER)
    stream = torch.cuda.current_stream()

    def to_dev(a):
        a = np.ascontiguousarray(a)
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(a).to(dev)

    # ---- inputs resident in HBM (replica per rank, same seeded data) ----
    host_layers = wl.all_layer_inputs(w0)
    tens = []
    for lay in host_layers:
        d = {}
        for k in ("q", "q_idx", "w", "win_k", "win_v"):
            d[k] = to_dev(lay[k])
        d["q"] = d["q"][:, 0].contiguous()              # decode: [B, H, D]
        if "entries" in lay:
            src = to_dev(lay["entries"])
            d["codes"], d["scales"] = csa2.pack_fp4(src)
            del src
            if args.keys == "fp4":
                ksrc = to_dev(wl.index_key_sources(w0, len(tens)))
                d["k_idx"], d["k_exps"] = csa2.pack_index_keys_fp4(ksrc)
                del ksrc
            else:
                d["k_idx"] = to_dev(lay["k_idx"])
            if args.append:
                app = wl.append_inputs(w0, 0)
                d["app_src"], d["app_key"] = to_dev(app["src"]), to_dev(app["key"])
                d["app_pos"] = torch.full((w0.B,), w0.N - 1, dtype=torch.int64, device=dev)
        d["idx"] = torch.empty((w0.B, 1, w0.topk), dtype=torch.int32, device=dev)
        d["out"] = torch.empty((w0.B, w0.H, w0.D), dtype=torch.float32, device=dev)
        d["lse"] = torch.empty((w0.B, w0.H), dtype=torch.float32, device=dev)
        tens.append(d)
    torch.cuda.synchronize()
    # Per-token inputs and per-step results of all layers live as views of one
    # device buffer each (256-byte aligned slots), so a step moves them with
    # one host->device and one device->host copy, as a serving loop would.
    # The per-token inputs are the queries, index queries, head weights and
    # the new token's window row (K and V of every sequence); the step writes
    # that row into the window's last slot on the device, and the older
    # window rows stay resident (a decode loop keeps its window on the GPU).
    # The layers' windows (K and V) are views of one tensor [2L, B, rows, D],
    # so the new rows of every layer (one block [2L, B, D] among the per-token
    # inputs) go into their slots with one copy.
    win_all = torch.stack([t for d in tens for t in (d["win_k"], d["win_v"])])
    for l, d in enumerate(tens):
        d["win_k"], d["win_v"] = win_all[2 * l], win_all[2 * l + 1]
    tens[0]["new_rows"] = win_all[:, :, -1].clone()
    in_keys = ("q", "q_idx", "w", "new_rows") + (("app_src", "app_key") if args.append else ())
    out_keys = ("out", "lse", "idx")
    dev_in, _ = pack_into_one_buffer(tens, in_keys, dev)
    dev_out, _ = pack_into_one_buffer(tens, out_keys, dev)
    pool_kw = {"pool_block": POOL_BLOCK, "pool_blocks": POOL_BLOCKS} if args.pool else {}
    if args.pool:
        tens[0]["pool"] = torch.empty((w0.B, POOL_BLOCK * POOL_BLOCKS), dtype=torch.int32,
                                      device=dev)
    dims = csa2.make_dims(w0.B, w0.T, w0.H, w0.D, w0.N, w0.H_I, w0.d_I, w0.topk, w0.W,
                          w0.n_prior, w0.ratio, w0.sm_scale, **pool_kw)
    group = csa2.LayerGroup(list(w0.modes), tens, dims)
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_src = torch.ones(256 << 20, dtype=torch.uint8, device=dev)
    flush_sink = torch.empty((), dtype=torch.int64, device=dev)

    def flush():
        # write a buffer larger than L2, then read another one: L2 ends up
        # holding clean lines, so the flush's own write-backs are not charged
        # to the timed kernels
        flush_buf.fill_(1)
        torch.sum(flush_src.view(torch.int64), dim=0, out=flush_sink)

    def layer(l):
        group.run_layer(l)   # one C-ABI call: scan + per-row select/attend cluster kernel

    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    # ~1 ms of GPU sleep ahead of each eager step so the host has enqueued the
    # whole step before its first kernel starts (no host gaps inside events)
    sleep_cycles = int(2.0e6)

    # Eager warm-up (sets kernel attributes, sizes the workspace), then one
    # CUDA graph per layer: replaying a layer costs the host a few us, so the
    # device timeline has no host-side launch gaps.
    for _ in range(2):
        for l in range(w0.L):
            layer(l)
    torch.cuda.synchronize()
    graphs = []
    for l in range(w0.L):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            layer(l)
        graphs.append(g)
    torch.cuda.synchronize()

    def timed_steps(K, eager=False):
        """K steps; returns per-step device ms (sum of per-layer events)."""
        pairs = []
        for _ in range(K):
            torch.cuda._sleep(sleep_cycles)
            step_pairs = []
            for l in range(w0.L):
                flush()
                a, b = ev(), ev()
                a.record(stream)
                if eager:
                    layer(l)
                else:
                    graphs[l].replay()
                b.record(stream)
                step_pairs.append((a, b))
            pairs.append(step_pairs)
        torch.cuda.synchronize()
        return [sum(a.elapsed_time(b) for a, b in sp) for sp in pairs]

    # ---- warm-up ----
    timed_steps(max(args.warmup, 3))
    if args.profile:
        timed_steps(args.steps)
        torch.cuda.synchronize()
        if rank == 0:
            print(json.dumps({"profile_steps": args.steps, "workload": w0.name}), flush=True)
        if dist:
            dist.barrier()
            dist.destroy_process_group()
        return 0

    gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
    gpu_id = gpu_uuid if gpu_uuid.startswith("GPU-") else f"GPU-{gpu_uuid}"
    clocks = ClockSampler(gpu_id)
    clocks.start()
    time.sleep(0.4)

    # ---- timed region: K steps ----
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    w_t0 = time.perf_counter()
    step_ms = timed_steps(args.steps)
    torch.cuda.synchronize()
    wall_s = time.perf_counter() - w_t0
    total_ms = max_over_ranks(dist, [float(sum(step_ms))], dev)[0]
    if dist:
        dist.barrier()

    # ---- per-kernel device times: a second pass of K steps over copies of
    # the layer graphs captured with the library's kernel trace on (an event
    # pair around each kernel, recorded as graph nodes on the launching
    # stream), so each kernel is timed as it runs in the timed region ----
    def graph_trace_pass(K):
        csa2.trace_enable(True)
        tgraphs = []
        try:
            for l in range(w0.L):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    layer(l)
                tgraphs.append(g)
            torch.cuda.synchronize()
            recs = []
            for _ in range(K):
                torch.cuda._sleep(sleep_cycles)
                for l in range(w0.L):
                    flush()
                    tgraphs[l].replay()
                torch.cuda.synchronize()
                recs += csa2.trace_records()
            return recs, "in-graph event pairs"
        finally:
            del tgraphs
            torch.cuda.synchronize()
            csa2.trace_enable(False)

    try:
        recs, trace_kind = graph_trace_pass(args.steps)
    except Exception:  # event timing inside graphs unavailable: eager launches
        csa2.trace_enable(True)
        timed_steps(args.steps, eager=True)
        recs, trace_kind = csa2.trace_records(), "eager event pairs"
        csa2.trace_enable(False)
    per_kernel = {}
    for name, ms in recs:
        c, s = per_kernel.get(name, (0, 0.0))
        per_kernel[name] = (c + 1, s + ms)
    launches_per_step = len(recs) / args.steps

    # ---- e2e: pinned host inputs -> device, hot path, results -> host ----
    host_in = dev_in.cpu().pin_memory()
    host_out = torch.empty_like(dev_out, device="cpu").pin_memory()
    h2d = host_in.numel() + tens[0]["new_rows"].numel() * tens[0]["new_rows"].element_size()
    d2h = host_out.numel()
    # A step's input staging (the pinned host buffer into the device inputs,
    # each layer's new window row from it straight into its slot) and its
    # result copy: one csa2_stage_copies launch each, replayed as a CUDA graph
    # as a serving loop would launch them.
    nr = tens[0]["new_rows"]
    off = nr.data_ptr() - dev_in.data_ptr()
    host_rows = host_in[off:off + nr.numel() * nr.element_size()].view(nr.dtype).view(nr.shape)
    in_graph, out_graph = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(in_graph):
        csa2.stage_copies([(host_in, dev_in), (host_rows, win_all[:, :, -1])])
    with torch.cuda.graph(out_graph):
        csa2.stage_copies([(dev_out, host_out)])
    torch.cuda.synchronize()

    def e2e_steps(K):
        """K end-to-end steps; per step the device ms of (inputs in + window
        append, the layers, results out)."""
        res = []
        for _ in range(K):
            torch.cuda._sleep(sleep_cycles)
            flush()
            a, b = ev(), ev()
            a.record(stream)
            in_graph.replay()
            b.record(stream)
            segs = [("h2d", a, b)]
            for l in range(w0.L):
                if l > 0:
                    flush()
                a, b = ev(), ev()
                a.record(stream)
                graphs[l].replay()
                b.record(stream)
                segs.append(("layers", a, b))
            a, b = ev(), ev()
            a.record(stream)
            out_graph.replay()
            b.record(stream)
            segs.append(("d2h", a, b))
            res.append(segs)
        torch.cuda.synchronize()
        out = []
        for segs in res:
            d = {"h2d": 0.0, "layers": 0.0, "d2h": 0.0}
            for name, a, b in segs:
                d[name] += a.elapsed_time(b)
            out.append(d)
        return out

    e2e_steps(3)
    e2e_recs = e2e_steps(args.steps)
    e2e_seg = {k: sum(r[k] for r in e2e_recs) for k in ("h2d", "layers", "d2h")}
    e2e_ms = max_over_ranks(dist, [float(sum(e2e_seg.values()))], dev)[0]
    clk = clocks.stop()

    status = csa2.get_device_status()
    if status:
        raise RuntimeError(f"device status word set: {status}")

    value = job_tokens_per_s(world, args.steps, w0.B, w0.T, w0.L, total_ms)
    e2e_value = job_tokens_per_s(world, args.steps, w0.B, w0.T, w0.L, e2e_ms)

    ab = algorithmic_bytes(w0, args.keys)
    peak, peak_kind = measured_peaks()
    step_bytes = w0.B * sum(layer_bytes(w0, args, l) for l in range(w0.L))
    ms_step = total_ms / args.steps
    step_gbs = step_bytes / (ms_step * 1e-3) / 1e9
    # Per kernel: launches and device time per step.  The trace's event pairs
    # add a fixed cost to each launch, so their sum exceeds the untraced step;
    # each kernel's share of the traced time, applied to the untraced step,
    # gives per-kernel times that add up to ms_per_step.
    traced_ms_per_step = sum(v[1] for v in per_kernel.values()) / args.steps
    kernels = {}
    for k, (c, s_) in sorted(per_kernel.items()):
        share = s_ / args.steps / traced_ms_per_step if traced_ms_per_step else 0.0
        per_launch = share * ms_step / (c / args.steps)
        b = KERNEL_BYTES.get(k, lambda w0_, ab_: None)(w0, ab)
        kernels[k] = {"launches_per_step": c / args.steps, "share_of_step": share,
                      "ms_per_launch": per_launch, "traced_ms_per_launch": s_ / c,
                      "bytes_per_launch": b}
        if b:
            kernels[k].update({"achieved_gbs": b / (per_launch * 1e-3) / 1e9,
                               "frac": b / (per_launch * 1e-3) / 1e9 / peak,
                               "traffic": ncu_traffic(k)})

    line = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            runs, dt = oracle_sample(w0, args.cpu_seconds)
            cpu = {"value": runs * w0.T * w0.L / dt, "unit": UNIT, "cores": 1, "kind": "oracle",
                   "sample": f"{runs} sequence(s) x {w0.L} layers of the same workload "
                             f"(N={w0.N}), plain C oracle, single thread, {dt:.1f} s",
                   **host_cpu()}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": {"workload": w0.name, "B": w0.B, "N": w0.N, "context_tokens": w0.N * 4,
                       "layers": "Full+Reindex" if w0.L == 2 else w0.L, "topk": w0.topk,
                       "H": w0.H, "D": w0.D, "H_I": w0.H_I, "d_I": w0.d_I, "W": w0.W,
                       "decode_kernel": args.decode_kernel,
                       "index_keys": args.keys, "entry_append_per_step": bool(args.append),
                       "pool": ({"block": POOL_BLOCK, "blocks": POOL_BLOCKS,
                                 "second_layer": "Reindex within the Full layer's pool"}
                                if args.pool else None),
                       "parallelism": f"replicas x{world}",
                       "l2": "flushed before every layer (256 MiB write, then 256 MiB read), flush not timed",
                       "step_algorithmic_bytes": step_bytes,
                       "step_hbm_gbs": step_gbs, "step_hbm_frac": step_gbs / peak,
                       "wall_s_timed_region": wall_s},
            "roofline": {"bound": "hbm", "scope": "decode step (both layers, every launch)",
                         "achieved": step_gbs, "peak": peak,
                         "peak_kind": f"{peak_kind} (copy bandwidth)", "unit": "GB/s",
                         "frac": step_gbs / peak, "frac_of_8tbs_nominal": step_gbs / 8000.0,
                         "bytes_per_step": step_bytes, "ms_per_step": ms_step,
                         "traffic": step_traffic(kernels),
                         "kernels": {k: {kk: v[kk] for kk in ("bytes_per_launch",
                                                               "ms_per_launch", "achieved_gbs",
                                                               "frac", "traffic") if kk in v}
                                     for k, v in kernels.items() if v.get("bytes_per_launch")}},
            "kernels": kernels, "kernel_timing": trace_kind + ", scaled to the untraced step",
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / args.steps,
                    "segments_ms_per_step": {k: v / args.steps for k, v in e2e_seg.items()}},
            "gpu_launches": int(round(launches_per_step * args.steps)),
            "clocks": clk,
            "cpu_baseline": cpu,
        }
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


def run_prefill(args, w0):
    """Supplementary measurement of one layer with several query tokens per
    sequence (a chunked prefill, or multi-token decode): index + top-k over
    the visible entries of every query, then attention; one GPU."""
    import torch
    import compressed_sparse_attention_topk_b200 as csa2
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    csa2.lib()
    lay = wl.layer_inputs(w0, 0)

    def to_dev(a):
        a = np.ascontiguousarray(a)
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(a).to(dev)

    t = {k: to_dev(lay[k]) for k in ("q", "q_idx", "w", "win_k", "win_v", "k_idx")}
    src = to_dev(lay["entries"])
    t["codes"], t["scales"] = csa2.pack_fp4(src)
    del src
    t["idx"] = torch.empty((w0.B, w0.T, w0.topk), dtype=torch.int32, device=dev)
    t["out"] = torch.empty((w0.B, w0.T, w0.H, w0.D), dtype=torch.float32, device=dev)
    t["lse"] = torch.empty((w0.B, w0.T, w0.H), dtype=torch.float32, device=dev)
    dims = csa2.make_dims(w0.B, w0.T, w0.H, w0.D, w0.N, w0.H_I, w0.d_I, w0.topk, w0.W,
                          w0.n_prior, w0.ratio, w0.sm_scale)
    group = csa2.LayerGroup([(0, 0, 0)], [t], dims)
    for _ in range(max(args.warmup, 1)):
        group.run_layer(0)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        group.run_layer(0)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / args.steps
    csa2.trace_enable(True)
    torch.cuda._sleep(int(2e6))  # the host enqueues the whole layer while the GPU waits
    group.run_layer(0)
    torch.cuda.synchronize()
    recs = csa2.trace_records()
    csa2.trace_enable(False)
    per = {}
    for name, m in recs:
        c, s_ = per.get(name, (0, 0.0))
        per[name] = (c + 1, s_ + m)
    cpu = None
    if not args.no_cpu_baseline:
        cpu = oracle_rows_sample(w0, lay, args.cpu_seconds)
    print(json.dumps({
        "metric": ("CSA2 chunked-prefill tokens/s per layer (supplementary)" if w0.n_prior >= 0
                   else "CSA2 multi-token decode tokens/s per layer (supplementary)"),
        "value": w0.B * w0.T / (ms * 1e-3), "unit": "tokens/s/layer", "ms_per_layer": ms,
        "steps": args.steps, "config": {"workload": w0.name, "T": w0.T, "N": w0.N,
                                          "n_prior": w0.n_prior, "topk": w0.topk},
        "kernels": {k: {"launches": c, "total_ms": s_} for k, (c, s_) in per.items()},
        "cpu_baseline": cpu,
    }), flush=True)
    return 0


def main():
    args = parse_args()
    w0 = wl.ALL[args.workload]
    if args.pool:
        if w0.modes != ((0, 0, 0), (1, 0, 1)):
            raise SystemExit("--pool runs the Full + Reindex decode workloads")
        w0 = wl.with_sizes(w0, modes=((0, 0, 0), (3, 0, 1)))
    if args.impl == "reference":
        if w0.T != 1:
            raise SystemExit("the reference leg times decode workloads")
        return run_reference(args, w0)
    if w0.T != 1 or w0.n_prior >= 0:
        return run_prefill(args, w0)
    return run_gpu(args, w0)


if __name__ == "__main__":
    sys.exit(main())
