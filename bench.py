"""Throughput of the attention forward on B200: one JSON line on rank 0.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload C] [--impl reference]

A step is one forward over the workload's whole batch (every step of the hot
path runs in one kernel launch).  The default workload is the dense BNSD fp16
forward B=2, N=24, S=4096, D=128.  Under torchrun each rank runs its own shard
of a batch N times as large (independent sequences, no data-path collective:
weak scaling); the time is the max over ranks of the summed per-step CUDA-event
times, and L2 is flushed (256 MiB write) before every step.

--impl reference times the float64 CPU oracle (rank 0 only) on a bounded
sample of the same workload with the same metric.
"""
import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from workloads import build, normal, cumulative  # noqa: E402

METRIC = "FA forward TFLOP/s and % of B200 dense BF16/FP16 peak (1 GPU)"
UNIT = "TFLOP/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
KERNEL_SOURCES = ["attention_forward_20_b200/csrc/fa_sm100.cu", "attention_forward_20_b200/csrc/sm100_ptx.cuh"]
L2_FLUSH_BYTES = 256 << 20


def workload_desc(w):
    lens = {"BNSD": (w.q.shape[0], w.q.shape[2]), "BSND": (w.q.shape[0], w.q.shape[1]),
            "BSH": (w.q.shape[0], w.q.shape[1]), "SBH": (w.q.shape[1], w.q.shape[0])}
    d, dv = head_dims(w)
    cfg = {"workload": f"{w.name} {w.layout} {w.dtype}", "layout": w.layout, "dtype": w.dtype,
           "heads": w.head_num, "head_dim": d}
    if dv != d:
        cfg["value_head_dim"] = dv
    if w.layout == "TND":
        cfg.update(tokens=w.q.shape[0], lengths=w.extra.get("lengths"))
    else:
        b, s = lens[w.layout]
        cfg.update(batch=b, seq_len=s)
    if w.next_tokens == 0:
        cfg["mask"] = "causal" + (f" band preTokens={w.pre_tokens}" if w.pre_tokens < 2**62 else "")
    if w.pse_type == 2:
        cfg["pse"] = "ALiBi slopes in-kernel"
    if w.sink is not None:
        cfg["sink"] = "per-head fp32"
    return cfg


def head_dims(w):
    """(query/key head dim, value head dim) of workload w."""
    if w.layout in ("BSH", "SBH"):
        d = w.q.shape[-1] // w.head_num
        return d, w.v.shape[-1] // (w.k.shape[-1] // d)
    return w.q.shape[-1], w.v.shape[-1]


def tile_flops(w):
    """(2*D + 2*Dv) * (query-row x key pairs), counted over every 128x128 tile
    that holds at least one kept pair (the headline rule), and the exact
    kept-pair FLOPs beside it (4*D per pair when Dv = D)."""
    d, dv = head_dims(w)
    if w.layout == "TND":
        lens_q = np.diff([0] + list(w.actual_seq_q))
        lens_k = np.diff([0] + list(w.actual_seq_kv))
        seqs = list(zip(lens_q, lens_k))
    else:
        b = w.q.shape[1] if w.layout == "SBH" else w.q.shape[0]
        sq = {"BNSD": w.q.shape[2], "BSND": w.q.shape[1], "BSH": w.q.shape[1], "SBH": w.q.shape[0]}[w.layout]
        skv = {"BNSD": w.k.shape[2], "BSND": w.k.shape[1], "BSH": w.k.shape[1], "SBH": w.k.shape[0]}[w.layout]
        seqs = [(sq, skv)] * b
    pre, nxt = w.pre_tokens, w.next_tokens
    tiles = exact = 0
    for sq, skv in seqs:
        for i0 in range(0, sq, 128):
            i1 = min(sq, i0 + 128) - 1
            for j0 in range(0, skv, 128):
                j1 = min(skv, j0 + 128) - 1
                # kept pairs of this tile: j in [max(j0, i-pre), min(j1, i+next)] per row i
                rows = np.arange(i0, i1 + 1)
                lo = np.maximum(j0, rows - min(pre, 2**40))
                hi = np.minimum(j1, rows + min(nxt, 2**40))
                kept = np.clip(hi - lo + 1, 0, None).sum()
                if kept:
                    tiles += 128 * 128
                    exact += int(kept)
    heads = w.head_num
    per_pair = 2.0 * d + 2.0 * dv
    return per_pair * tiles * heads, per_pair * exact * heads


def sources_sha():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_peak():
    try:
        with open(PEAKS_FILE) as f:
            peaks = json.load(f)
        return float(peaks["bf16_tflops"]), "measured (MEASURED_PEAKS.json bf16_tflops, burst; fp16 nominal ratio 1)"
    except (OSError, KeyError, ValueError):
        return 1590.0, "fallback 1.59 PFLOP/s"


def load_traffic(workload_name):
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    entry = t.get(workload_name)
    if not entry or entry.get("kernel_sources_sha") != sources_sha():
        return None
    return entry.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and throttle reasons with NVML in a thread."""

    REASONS = {
        0x0000000000000008: "hw_slowdown",
        0x0000000000000040: "hw_thermal_slowdown",
        0x0000000000000020: "sw_thermal_slowdown",
        0x0000000000000004: "sw_power_cap",
    }

    def __init__(self, device_index, interval=0.002, delay=0.0):
        self.samples, self.reasons, self.ok = [], set(), False
        self.interval = interval
        self.delay = delay  # seconds before the first sample (the GPU is still in its pre-queue wait)
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        nv = self.nvml
        self._stop.wait(self.delay)
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.interval)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def kernels_per_call(fa, q, k, v, kw):
    """Kernels one fa_fwd call launches: the attention kernel, plus the merge
    kernel when the plan splits the last wave into key pieces."""
    plan_kw = {key: kw[key] for key in ("input_layout", "head_num", "scale", "actual_seq_qlen",
                                        "actual_seq_kvlen", "pre_tokens", "next_tokens") if key in kw}
    text = fa.plan(q, k, v, **plan_kw)[2]
    pieces = int(text.split("pieces=")[1].split()[0]) if "pieces=" in text else 0
    return 1 + (1 if pieces > 0 else 0)


def alibi_bias_on_device(slopes, seq, first_row, dtype, dev):
    """Materialised ALiBi bias -slope_n * |i - j| as a dense [1, N, seq - first_row, seq]
    tensor (rows first_row .. seq-1), built on the device 1024 rows at a time."""
    n = slopes.shape[0]
    bias = torch.empty(1, n, seq - first_row, seq, dtype=dtype, device=dev)
    j = torch.arange(seq, device=dev, dtype=torch.float32)[None, :]
    for h in range(n):
        for r0 in range(first_row, seq, 1024):
            i = torch.arange(r0, min(seq, r0 + 1024), device=dev, dtype=torch.float32)[:, None]
            bias[0, h, r0 - first_row:r0 - first_row + i.shape[0]] = (-float(slopes[h]) * (i - j).abs()).to(dtype)
    return bias


def with_head_dims(w, d, dv):
    """Workload w with query/key head dim d and value head dim dv: same layout,
    sizes, masks and seeds, inputs redrawn N(0,1), scale d^-0.5."""
    def shaped(t, heads, hd):
        if w.layout in ("BSH", "SBH"):
            return tuple(t.shape[:2]) + (heads * hd,)
        return tuple(t.shape[:-1]) + (hd,)
    d0 = w.q.shape[-1] // w.head_num if w.layout in ("BSH", "SBH") else w.q.shape[-1]
    n_kv = w.k.shape[-1] // d0 if w.layout in ("BSH", "SBH") else None
    seed = 7000 + 17 * w.number
    w.q = normal(shaped(w.q, w.head_num, d), w.dtype, seed)
    w.k = normal(shaped(w.k, n_kv, d), w.dtype, seed + 1)
    w.v = normal(shaped(w.v, n_kv, dv), w.dtype, seed + 2)
    w.scale = d ** -0.5
    w.name = f"{w.name}_d{d}" + (f"_dv{dv}" if dv != d else "")
    return w


def rope_tensors(w, dr, seed):
    """queryRope / keyRope for workload w: the query's / key's layout and sizes, head dim dr."""
    def shaped(t, heads):
        if w.layout in ("BSH", "SBH"):
            return tuple(t.shape[:2]) + (heads * dr,)
        return tuple(t.shape[:-1]) + (dr,)
    n_kv = w.k.shape[-1] // (w.q.shape[-1] // w.head_num) if w.layout in ("BSH", "SBH") else None
    return (normal(shaped(w.q, w.head_num), "bf16", seed), normal(shaped(w.k, n_kv), "bf16", seed + 1))


def fa_kwargs(w, dev):
    c = lambda t: None if t is None else t.to(dev)  # noqa: E731
    pse = c(w.pse)
    return dict(input_layout=w.layout, head_num=w.head_num, scale=w.scale, real_shift=pse,
                pse_type=w.pse_type if pse is not None else None, atten_mask=c(w.atten_mask),
                mask_mode=w.mask_mode, sink=c(w.sink), actual_seq_qlen=w.actual_seq_q,
                actual_seq_kvlen=w.actual_seq_kv, pre_tokens=w.pre_tokens, next_tokens=w.next_tokens,
                softmax_out_layout=w.softmax_out_layout)


def time_oracle(w, budget_s, max_heads=None, rope=None):
    """Float64 oracle on whole (batch, head) pairs of the workload until
    `budget_s` seconds have passed; returns (flops done, seconds, heads done).
    rope: (queryRope, keyRope) host tensors or None."""
    from oracle import ref
    d, dv = head_dims(w)
    dr = 0
    if rope is not None:
        dr = rope[0].shape[-1] if w.layout not in ("BSH", "SBH") else rope[0].shape[-1] // w.head_num
        qrh = ref.heads_view(rope[0].double().numpy(), w.layout, dr)
        krh = ref.heads_view(rope[1].double().numpy(), w.layout, dr)
    qh = ref.heads_view(w.q.double().numpy(), w.layout, d)
    kh = ref.heads_view(w.k.double().numpy(), w.layout, d)
    vh = ref.heads_view(w.v.double().numpy(), w.layout, dv)
    n_kv = kh.shape[1]
    group = w.head_num // n_kv
    sink = None if w.sink is None else w.sink.double().numpy()
    pse = None if w.pse is None else w.pse.double().numpy()
    if w.layout == "TND":
        cq = [0] + list(w.actual_seq_q)
        ck = [0] + list(w.actual_seq_kv)
        pairs = [(b, n) for b in range(len(cq) - 1) for n in range(w.head_num)]
    else:
        pairs = [(b, n) for b in range(qh.shape[0]) for n in range(w.head_num)]
    flops = secs = 0.0
    heads = 0
    for (b, n) in pairs[:max_heads]:
        qr = kr = None
        if w.layout == "TND":
            q, k, v = (qh[cq[b]:cq[b + 1], n], kh[ck[b]:ck[b + 1], n // group], vh[ck[b]:ck[b + 1], n // group])
            if dr:
                qr, kr = qrh[cq[b]:cq[b + 1], n], krh[ck[b]:ck[b + 1], n // group]
        else:
            q, k, v = qh[b, n], kh[b, n // group], vh[b, n // group]
            if dr:
                qr, kr = qrh[b, n], krh[b, n // group]
        rows = np.arange(q.shape[0])
        t0 = time.perf_counter()
        ref.head_forward(q, k, v, w.scale, rows=rows,
                         pse=ref._pse_rows(pse, w.pse_type, b, n, rows, k.shape[0]),
                         pre_tokens=w.pre_tokens, next_tokens=w.next_tokens,
                         sink=None if sink is None else sink[n], q_rope=qr, k_rope=kr)
        secs += time.perf_counter() - t0
        flops += (2.0 * d + 2.0 * dv + 2.0 * dr) * q.shape[0] * k.shape[0]
        heads += 1
        if secs >= budget_s:
            break
    return flops, secs, heads


def shard_workload(w, rank):
    """Rank `rank`'s shard of an N-times larger batch: the workload's shapes,
    inputs redrawn from a rank-specific seed (rank 0 keeps the workload's own)."""
    if rank:
        g = torch.Generator().manual_seed(1000003 * rank)
        for name in ("q", "k", "v"):
            t = getattr(w, name)
            setattr(w, name, torch.randn(t.shape, generator=g, dtype=torch.float32).to(t.dtype))
    return w


def max_over_ranks(values, dist, device):
    """Element-wise max of a list of floats over all ranks (identity without dist)."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def hbm_line(bias_bytes, q, k, v, out, ms_per_step, bytes_override=None):
    """The materialised-bias band is HBM-heavy: algorithmic bytes (Q, K, V read,
    O written, and the bias blocks inside the band) per step time, against the
    measured copy bandwidth."""
    try:
        with open(PEAKS_FILE) as f:
            hbm_peak, src = float(json.load(f)["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    except (OSError, KeyError, ValueError):
        hbm_peak, src = 6650.0, "fallback 6.65 TB/s"
    algo = bias_bytes + sum(t.numel() * t.element_size() for t in (q, k, v, out))
    if bytes_override is not None:
        algo = bytes_override
    gbs = algo / (ms_per_step * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
            "algorithmic_bytes": algo, "peak_source": src}


def whole_job_tflops(flops_per_rank, world, ms_per_step):
    """Units all ranks processed per step over the slowest rank's step time."""
    return flops_per_rank * world / (ms_per_step * 1e-3) / 1e12


def step_stats(times_ms):
    """Median, min, p90 and mean of per-step times (ms)."""
    t = np.asarray(times_ms, dtype=np.float64)
    return {"median": float(np.median(t)), "min": float(t.min()), "p90": float(np.percentile(t, 90)),
            "mean": float(t.mean())}


def time_oracle_single_thread(w, rope=None):
    """The oracle on one whole (batch, head) of w with one BLAS thread: (TFLOP/s, seconds)."""
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):
        fl, secs, _ = time_oracle(w, 0.0, max_heads=1, rope=rope)
    return fl / secs / 1e12, secs


def with_lengths(w, lengths):
    """Varlen (TND) workload w with other sequence lengths: inputs redrawn with
    the same seeds at T = sum(lengths), q and kv lengths equal."""
    if w.layout != "TND":
        raise SystemExit("--lengths applies to the TND workload")
    lens = [int(x) for x in lengths]
    t = sum(lens)
    seed = 1000 * w.number
    w.q = normal((t,) + tuple(w.q.shape[1:]), w.dtype, seed + 1)
    w.k = normal((t,) + tuple(w.k.shape[1:]), w.dtype, seed + 2)
    w.v = normal((t,) + tuple(w.v.shape[1:]), w.dtype, seed + 3)
    w.actual_seq_q = cumulative(lens, False)
    w.actual_seq_kv = cumulative(lens, False)
    w.extra["lengths"] = lens
    w.extra["cu_seqlens"] = cumulative(lens, True)
    w.name = w.name + "_" + "_".join(str(x) for x in lens)
    return w


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count()


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1,
                    help="GPUs (ranks) on this node: under torchrun WORLD_SIZE ranks are already running; "
                         "without it this script starts one process per GPU itself")
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", type=int, default=2)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--kv-chunks", type=int, default=1,
                    help="split the keys into this many chunks: one forward per chunk at its kvStartIdx, "
                         "then fa_lse_merge (dense layouts)")
    ap.add_argument("--pse", default="slopes", choices=["slopes", "dense", "compressed"],
                    help="ALiBi workloads: slopes in-kernel, a materialised [1,N,S,S] bias, or its last 1024 rows")
    ap.add_argument("--head-dim", type=int, default=0,
                    help="the workload with this query/key head dim (fresh N(0,1) inputs, scale D^-0.5)")
    ap.add_argument("--value-head-dim", type=int, default=0, help="with --head-dim: the value head dim (default D)")
    ap.add_argument("--lengths", default="",
                    help="TND workload: comma-separated sequence lengths instead of the seeded ones")
    ap.add_argument("--rope", type=int, default=0,
                    help="bf16 workloads: add queryRope/keyRope of this head dim (N(0,1), seeded)")
    ap.add_argument("--seq-scale", type=int, default=1,
                    help="divide the workload's sequence lengths (and the band's preTokens) by this factor: "
                         "a smaller case of the same structure, for profiler captures")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)
    return args


def rank_env():
    """(rank, world size, local rank) from the launcher's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def free_port():
    import socket
    with socket.socket() as sock:
        sock.bind(("127.0.0.1", 0))
        return sock.getsockname()[1]


def spawn_ranks(n, argv, script=None, timeout_s=3600.0):
    """One process per rank, as torchrun would start them: each runs `script`
    (this file) with RANK, LOCAL_RANK = rank, WORLD_SIZE = n and a rendezvous
    on 127.0.0.1 in its environment.  If a rank fails the others are stopped.
    Returns 0 when every rank exits 0, else the first failing exit code."""
    import signal
    import subprocess
    port = free_port()
    procs = []
    for r in range(n):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE=str(n), MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, script or os.path.abspath(__file__)] + list(argv), env=env,
                                      start_new_session=True))
    deadline = time.monotonic() + timeout_s
    rc = 0
    while True:
        codes = [p.poll() for p in procs]
        failed = [c for c in codes if c not in (None, 0)]
        if failed or time.monotonic() > deadline:
            rc = failed[0] if failed else 124
            for p in procs:
                if p.poll() is None:
                    os.killpg(p.pid, signal.SIGTERM)
            for p in procs:
                try:
                    p.wait(timeout=30)
                except subprocess.TimeoutExpired:
                    os.killpg(p.pid, signal.SIGKILL)
                    p.wait()
            return rc
        if all(c == 0 for c in codes):
            return 0
        time.sleep(0.05)


def init_dist(world, backend, device=None):
    """The process group of a multi-rank run (None for one rank), with a short
    timeout so that ranks waiting on a failed peer end with an error."""
    if world <= 1:
        return None
    import datetime
    import torch.distributed as dist
    kw = {"device_id": device} if device is not None else {}
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return dist


def prepare_workload(args, rank):
    """This rank's workload: the configured one, with the flags' variations
    applied, and its inputs redrawn per rank (rank 0 keeps the workload's own)."""
    w = build(args.workload, seq_scale=args.seq_scale)
    if args.seq_scale > 1:
        w.name = f"{w.name}_seq_div{args.seq_scale}"
    if args.lengths:
        w = with_lengths(w, args.lengths.split(","))
    if args.head_dim:
        w = with_head_dims(w, args.head_dim, args.value_head_dim or args.head_dim)
    return shard_workload(w, rank)


def workload_flops(w, rope_dim=0):
    """(tile-counted, exact) FLOPs of one forward over w; with rope the QK
    contraction is D + Dr long: 2*(D + Dr) + 2*Dv per counted pair."""
    flops_tiles, flops_exact = tile_flops(w)
    if rope_dim:
        d, dv = head_dims(w)
        f = (2.0 * d + 2.0 * dv + 2.0 * rope_dim) / (2.0 * d + 2.0 * dv)
        flops_tiles, flops_exact = flops_tiles * f, flops_exact * f
    return flops_tiles, flops_exact


def qkvo_bytes(w):
    """Bytes of Q, K, V read and O written by one forward over w."""
    d, dv = head_dims(w)
    out_elems = w.q.numel() // d * dv
    es = w.q.element_size()
    return sum(t.numel() * t.element_size() for t in (w.q, w.k, w.v)) + out_elems * es


def workload_config(w, world, args):
    """The `config` object of the JSON line: the same for both arms."""
    desc = workload_desc(w)
    flops_tiles, flops_exact = workload_flops(w, args.rope)
    if args.kv_chunks > 1:
        desc["kv_chunks"] = f"{args.kv_chunks} key chunks at their kvStartIdx, then fa_lse_merge (sink added there)"
    if args.rope:
        desc["rope"] = f"queryRope/keyRope head dim {args.rope} (bf16, N(0,1)): S = scale*(Q K^T + Qr Kr^T)"
    if args.pse != "slopes" and w.pse_type == 2:
        desc["pse"] = ("materialised fp16 bias [1,N,S,S], resident" if args.pse == "dense"
                       else "compressed bias: last 1024 rows [1,N,1024,S], resident")
    return dict(desc, parallelism=f"dp{world} (independent shards)",
                l2=f"flushed before every step (256 MiB write); Q/K/V/O {qkvo_bytes(w) / 1e6:.0f} MB",
                flops_tile_counted=flops_tiles, flops_exact=flops_exact)


def run_reference(args, rank):
    if rank != 0:
        return
    w = prepare_workload(args, 0)
    rope = rope_tensors(w, args.rope, seed=9100) if args.rope else None
    for _ in range(args.warmup):
        time_oracle(w, 0.0, max_heads=1, rope=rope)
    flops = secs = 0.0
    heads = 0
    for _ in range(args.steps):
        f, s_, h = time_oracle(w, 0.0, max_heads=1, rope=rope)
        flops, secs, heads = flops + f, secs + s_, heads + h
    value = flops / secs / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, args.gpus, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                         "sample": f"one whole (batch, head) of the workload per step, {heads} heads"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    args = parse_args(argv)
    rank, world, local_rank = rank_env()
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # not started by torchrun: one process per GPU, started here
        sys.exit(spawn_ranks(args.gpus, sys.argv[1:] if argv is None else argv))
    if world > 1 and args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")

    import attention_forward_20_b200 as fa
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = init_dist(world, "nccl", dev)

    # each rank: its own shard (seed offset by rank) of the workload's batch
    w = prepare_workload(args, rank)
    flops_tiles, flops_exact = workload_flops(w, args.rope)
    q, k, v = w.q.to(dev), w.k.to(dev), w.v.to(dev)
    kw = fa_kwargs(w, dev)
    rope = None
    if args.rope:
        if w.dtype != "bf16":
            raise SystemExit("--rope needs a bf16 workload (queryRope/keyRope are BFLOAT16 only)")
        rope = rope_tensors(w, args.rope, seed=9100 + rank)
        kw["query_rope"], kw["key_rope"] = rope[0].to(dev), rope[1].to(dev)
    bias_bytes = 0
    if args.pse != "slopes" and w.pse_type == 2:
        # the same ALiBi bias, materialised in the query dtype and resident in HBM
        # (a fixed positional table, not a per-step input)
        seq = w.q.shape[1] if w.layout in ("BSH", "BSND") else w.q.shape[2]
        first = 0 if args.pse == "dense" else seq - 1024
        kw["real_shift"] = alibi_bias_on_device(w.pse.double().numpy(), seq, first, q.dtype, dev)
        kw["pse_type"] = 1
        # bias bytes the kernel reads: one 128x128 block per counted tile-block
        d, dv = head_dims(w)
        bias_bytes = flops_tiles / (2.0 * d + 2.0 * dv) * q.element_size()
    out, smax, ssum = fa.fa_fwd(q, k, v, **kw)
    if not (bool(torch.isfinite(out).all()) and not bool(torch.isnan(smax).any())):
        raise SystemExit("first forward gave non-finite outputs")
    launches_per_step = kernels_per_call(fa, q, k, v, kw)
    if args.kv_chunks > 1:
        launches_per_step = args.kv_chunks * launches_per_step + 1  # chunk forwards + the merge (upper bound)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        fa.fa_fwd(q, k, v, out=out, softmax_max=smax, softmax_sum=ssum, **kw)

    merge_events = []
    if args.kv_chunks > 1:
        # a forward split along the keys (as context parallelism would place the
        # chunks on different GPUs), each chunk at its global start, then the merge
        seq_axis = {"BNSD": 2, "BSND": 1, "BSH": 1, "SBH": 0}[w.layout]
        skv = k.shape[seq_axis]
        bounds = [(c * skv // args.kv_chunks, (c + 1) * skv // args.kv_chunks) for c in range(args.kv_chunks)]
        kcs = [k.narrow(seq_axis, a, b - a).contiguous() for a, b in bounds]
        vcs = [v.narrow(seq_axis, a, b - a).contiguous() for a, b in bounds]
        kw_base = {key_: val for key_, val in kw.items() if key_ != "sink"}
        mask = kw_base.get("atten_mask")
        # a chunk's mask is its columns of the mask (masks are indexed by in-chunk positions)
        kw_parts = [dict(kw_base, atten_mask=None if mask is None else mask[..., a:b].contiguous(), kv_start_idx=a)
                    for a, b in bounds]
        parts = [fa.fa_fwd(q, kc, vc, **kp) for kc, vc, kp in zip(kcs, vcs, kw_parts)]

        def step():  # noqa: F811
            for kc, vc, kp, (po, pm, ps) in zip(kcs, vcs, kw_parts, parts):
                fa.fa_fwd(q, kc, vc, out=po, softmax_max=pm, softmax_sum=ps, **kp)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fa.lse_merge([p_[0] for p_ in parts], [p_[1] for p_ in parts], [p_[2] for p_ in parts],
                         input_layout=w.layout, head_num=w.head_num, sink=kw.get("sink"),
                         softmax_out_layout=w.softmax_out_layout or "", out=out, softmax_max=smax,
                         softmax_sum=ssum)
            e1.record(stream)
            merge_events.append((e0, e1))

    torch.cuda.synchronize(dev)
    host_times = []
    for _ in range(args.warmup):
        t_host = time.perf_counter()
        flush.zero_()
        step()
        host_times.append(time.perf_counter() - t_host)
    host_s = statistics.median(host_times)  # host enqueue time per step (first-call costs excluded)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    # The GPU first spins long enough for the host to enqueue every timed step,
    # so that each step's events bracket device work only, never a wait for the
    # host (which matters when a step is shorter than its Python/launch cost).
    pre_s = min(2.0, max(1e-3, 1.25 * host_s * args.steps))
    torch.cuda._sleep(int(pre_s * 2.0e9))
    with ClockSampler(dev.index, delay=pre_s) as clocks:
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
    if dist:
        dist.barrier()
    step_times = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    kernel_ms = sum(step_times)
    status, word = fa.device_error()
    if status != 0:
        raise SystemExit(f"kernel error word {word:#x}")

    # End to end through fa_fwd with host buffers: every step copies its inputs
    # from pinned host memory and its results (output and statistics) back to
    # pinned host memory.  Consecutive steps overlap on three streams (copy in,
    # compute, copy out) with two sets of device buffers, as a serving loop
    # would: step i+1's inputs travel while step i computes and step i-1's
    # results return.
    host = [t.pin_memory() for t in (w.q, w.k, w.v) + (tuple(rope) if rope is not None else ())]
    n_slots = 2
    dev_in = [[torch.empty_like(t, device=dev) for t in host] for _ in range(n_slots)]
    dev_res = [tuple(torch.empty_like(t) for t in (out, smax, ssum)) for _ in range(n_slots)]
    host_res = [tuple(torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (out, smax, ssum))
                for _ in range(n_slots)]
    s_in, s_comp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_ready = [torch.cuda.Event() for _ in range(n_slots)]
    comp_done = [torch.cuda.Event() for _ in range(n_slots)]
    out_done = [torch.cuda.Event() for _ in range(n_slots)]
    used = [False] * n_slots
    e2e_steps = max(4, min(args.steps, 20))

    def e2e_step(i):
        k_ = i % n_slots
        if used[k_]:
            s_in.wait_event(comp_done[k_])     # the forward that read these input buffers is done
        with torch.cuda.stream(s_in):
            for d_, h_ in zip(dev_in[k_], host):
                d_.copy_(h_, non_blocking=True)
        in_ready[k_].record(s_in)
        s_comp.wait_event(in_ready[k_])
        if used[k_]:
            s_comp.wait_event(out_done[k_])    # these result buffers have been copied out
        with torch.cuda.stream(s_comp):
            kw_i = dict(kw, **({"query_rope": dev_in[k_][3], "key_rope": dev_in[k_][4]} if rope is not None else {}))
            o_, m_, l_ = dev_res[k_]
            fa.fa_fwd(dev_in[k_][0], dev_in[k_][1], dev_in[k_][2], out=o_, softmax_max=m_, softmax_sum=l_, **kw_i)
        comp_done[k_].record(s_comp)
        s_out.wait_event(comp_done[k_])
        with torch.cuda.stream(s_out):
            for h_, d_ in zip(host_res[k_], dev_res[k_]):
                h_.copy_(d_, non_blocking=True)
        out_done[k_].record(s_out)
        used[k_] = True

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(e2e_steps):
        e2e_step(i)
    e1.record(s_out)                           # after the last step's results reached the host
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    # the last step's results equal the device-timed run's (same inputs, same call)
    if args.kv_chunks == 1 and not torch.equal(host_res[(e2e_steps - 1) % n_slots][0], out.cpu()):
        raise SystemExit("end-to-end result differs from the device-timed result")
    h2d = sum(t.numel() * t.element_size() for t in host)
    d2h = sum(t.numel() * t.element_size() for t in host_res[0])

    kernel_ms, e2e_ms = max_over_ranks([kernel_ms, e2e_ms], dist, dev)
    if dist:
        dist.destroy_process_group()
    if rank != 0:
        return

    ms_per_step = kernel_ms / args.steps
    value = whole_job_tflops(flops_tiles, world, ms_per_step)
    per_gpu = flops_tiles / (ms_per_step * 1e-3) / 1e12
    peak, peak_src = load_peak()
    traffic = load_traffic(w.name) if args.pse == "slopes" and not args.rope else None
    fl, secs, heads = time_oracle(w, args.cpu_budget, rope=rope)
    st_value, st_secs = time_oracle_single_thread(w, rope=rope)
    cpu_value = fl / secs / 1e12
    merge_line = None
    if args.kv_chunks > 1:
        timed = merge_events[-args.steps:]
        merge_ms = sum(a.elapsed_time(b) for a, b in timed) / max(1, len(timed))
        part_bytes = out.numel() * out.element_size() + 2 * smax.numel() * smax.element_size()
        merge_line = hbm_line(0, q, k, v, out, merge_ms, bytes_override=(args.kv_chunks + 1) * part_bytes)
        merge_line["ms"] = merge_ms
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": workload_config(w, world, args),
        "roofline": {"bound": "tensor", "achieved": per_gpu, "peak": peak, "unit": UNIT,
                     "frac": per_gpu / peak, "traffic": traffic, "peak_source": peak_src,
                     "pct_of_nominal_2250": 100.0 * per_gpu / 2250.0},
        **({"hbm": hbm_line(bias_bytes, q, k, v, out, ms_per_step)} if args.pse == "dense" else {}),
        **({"merge": merge_line} if merge_line else {}),
        "cpu_baseline": {"value": cpu_value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                         "sample": f"{heads} whole (batch, head) pairs of the workload, float64 NumPy, "
                                   f"{secs:.1f} s" + ("" if args.pse == "slopes" else
                                                      " (bias from the slopes, the same values in float64)"),
                         "single_thread": {"value": st_value, "unit": UNIT,
                                           "sample": f"one whole (batch, head), one BLAS thread, {st_secs:.1f} s"}},
        "e2e": {"value": whole_job_tflops(flops_tiles, world, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "pipeline": "copy in / compute / copy out on three streams, two buffer sets"},
        "step_ms": step_stats(step_times),
        "gpu_launches": args.steps * launches_per_step,
        "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
