"""Benchmark of the gzip-guided sparse attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one pass of the whole path over one synthetic batch of the 8K-byte
workload (8 samples x 8192 bytes, 64-byte blocks -> 128 blocks, window 2,
12 heads split 6 local / 3 literal / 3 hybrid, head dim 64, bf16):
    gsa_mask_pipeline (block lengths -> literal flags -> block lists, one launch)
    -> gsa_attn_fwd -> gsa_attn_bwd
all through the C ABI (libgsa.so); the mask sweep times the three separate
calls (gsa_block_lengths, gsa_literal_flags, gsa_build_block_csr) beside it.  The headline value is live-block
attention TFLOP/s (forward 4*d and backward 8*d FLOPs per live
(query token, key token) pair, the S recompute not counted) of the whole
step, inputs resident in HBM.  The L2 is flushed between steps (a 256 MiB
write, outside the timed events).  Rank 0 prints one JSON line.

Under torchrun each rank runs its own batch (data-parallel, no collective on
the data path); the timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "live-block attn TFLOP/s fwd+bwd @8K bytes; gzip-mask GB/s of input bytes"
UNIT = "TFLOP/s"
WORKLOAD = "b8_8k"
MASK_POINT = (64, 0.3)


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "sm_max_mhz": p.get("sm_max_mhz", 1965.0), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "sm_max_mhz": 1965.0, "source": "fallback"}


def workload_desc(wl):
    hc = [int(c) for c in wl.head_classes()]
    split = "/".join(str(hc.count(c)) for c in (0, 1, 2))
    return (f"{wl.name}: batch {wl.S} x {wl.L} bytes, b={wl.b} ({wl.N} blocks), w={wl.w}, "
            f"{wl.H} heads ({split} local/literal/hybrid), d={wl.d}, {wl.dtype}, "
            f"{'fwd+bwd' if wl.backward else 'fwd'}")


def csr_nnz(csr):
    """Live block pairs per (sample, class) [S][3] from the lists' pointers;
    an implicit local class (not stored) counts its window, min(i, w) + 1
    key blocks for query block i."""
    nnz = csr.row_ptr[:, :, -1].cpu().numpy().copy()
    if not csr.stored(0):
        nnz[:, 0] = sum(min(i, csr.w) + 1 for i in range(csr.nblk))
    return nnz


def live_token_pairs_from_counts(nnz_sc, n, b, head_classes):
    """Live (query token, key token) pairs summed over heads of one sample,
    from the per-class live block-pair counts (diagonal blocks are causal)."""
    total = 0
    for c in head_classes:
        nnz = int(nnz_sc[int(c)])
        total += (nnz - n) * b * b + n * b * (b + 1) // 2
    return total


# ------------------------------------------------------------------ clocks

def _nvml_poll(uuid, period_s, conn):
    """Child process of NvmlClockSampler: read the SM clock and the clock-event
    reasons every period_s until told to stop, then send the rows back.  A
    process of its own, so the parent's kernel launches (which hold the GIL)
    cannot hold the sampling back."""
    import pynvml as nv
    try:
        nv.nvmlInit()
        handle = nv.nvmlDeviceGetHandleByUUID(uuid)
        max_mhz = nv.nvmlDeviceGetMaxClockInfo(handle, nv.NVML_CLOCK_SM)
    except Exception as e:  # pragma: no cover - reported to the parent
        conn.send(("error", repr(e)))
        return
    conn.send(("ready", max_mhz))
    rows = []
    while not conn.poll(0):
        try:
            rows.append((nv.nvmlDeviceGetClockInfo(handle, nv.NVML_CLOCK_SM),
                         nv.nvmlDeviceGetCurrentClocksEventReasons(handle)))
        except Exception:
            pass
        time.sleep(period_s)
    conn.recv()
    conn.send(rows)
    try:
        nv.nvmlShutdown()
    except Exception:
        pass


class NvmlClockSampler:
    """SM clock and clock-event (throttle) reasons read through NVML every 1 ms
    by a child process (started with spawn) while the timed loop runs: read-only
    queries, and many samples even inside a timed region of a few tens of
    milliseconds.  Same summary as ClockSampler; start() raises when NVML or
    the device is not available."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, device_index: int, period_s: float = 0.001, spawn: bool = True):
        self.device = device_index
        self.period = period_s
        self.spawn = spawn   # False: the same poller on a thread (tests with a fake NVML module)
        self.rows = []
        self.proc = None
        self.conn = None

    def start(self):
        import multiprocessing as mp
        import pynvml as nv
        import torch
        u = str(torch.cuda.get_device_properties(self.device).uuid)
        uuid = u if u.startswith("GPU-") else "GPU-" + u
        self.masks = [(name, getattr(nv, const)) for name, const in self.REASONS]
        ctx = mp.get_context("spawn")
        self.conn, child = ctx.Pipe()
        if self.spawn:
            self.proc = ctx.Process(target=_nvml_poll, args=(uuid, self.period, child), daemon=True)
        else:
            import threading
            self.proc = threading.Thread(target=_nvml_poll, args=(uuid, self.period, child), daemon=True)
        self.proc.start()
        if not self.conn.poll(60):
            if self.spawn:
                self.proc.kill()
            raise RuntimeError("clock sampler did not start")
        kind, val = self.conn.recv()
        if kind != "ready":
            self.proc.join(timeout=5)
            raise RuntimeError(f"NVML unavailable: {val}")
        self.max_mhz = val

    def stop(self):
        if self.proc is None:
            return None
        self.conn.send("stop")
        self.rows = self.conn.recv() if self.conn.poll(30) else []
        self.proc.join(timeout=5)
        if not self.rows:
            return None
        sm = [float(r[0]) for r in self.rows]
        reasons = sorted({name for _, why in self.rows for name, m in self.masks if why & m})
        loaded = [x for x in sm if x > 0.5 * self.max_mhz] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": float(self.max_mhz), "reasons": reasons,
                "samples": len(self.rows), "source": "nvml, 1 ms, own process"}


class ClockSampler:
    """nvidia-smi sampling of the SM clock and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        self.device = device_index

    def _select(self):
        """nvidia-smi -i argument for the CUDA device (its UUID), if known."""
        try:
            import torch
            u = getattr(torch.cuda.get_device_properties(self.device), "uuid", None)
            if u is not None:
                u = str(u)
                return u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            pass
        return None

    def start(self):
        sel = self._select()
        fd, self.path = tempfile.mkstemp(prefix="gsa_clocks_", suffix=".csv")
        os.close(fd)
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if sel is not None:
            probe = subprocess.run(["nvidia-smi", "-i", sel, "--query-gpu=index", "--format=csv,noheader"],
                                   capture_output=True, text=True)
            if probe.returncode == 0 and probe.stdout.strip():
                cmd += ["-i", sel]
        try:
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        reasons = set()
        for r in rows:
            for name, val in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"),
                                 r[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        loaded = [x for x in sm if x > 0.5 * (max(mx) if mx else 1)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons), "samples": len(rows)}


# ------------------------------------------------------------------ oracle (CPU baseline)

def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_sample_step(wl, x, q, k, v, do, hc, head):
    """One bounded sample of the workload on the oracle: the mask stage of
    sample 0 and the forward + backward of one head of it.  Returns the
    algorithmic FLOPs of that head."""
    from oracle import attention as oatt, deflate1, flags as oflags, mask as omask
    ln = deflate1.block_lengths(x[:1], wl.b, nthreads=1)
    fl = oflags.literal_flags(ln, wl.b)
    m = omask.block_mask(fl[0], wl.w, int(hc[head]))
    oatt.forward(q[0, head], k[0, head], v[0, head], m, wl.b)
    oatt.backward(q[0, head], k[0, head], v[0, head], do[0, head], m, wl.b)
    return 12 * wl.d * omask.live_token_pairs(m, wl.b)


def oracle_inputs(wl, seed):
    import torch
    x = W.batch_bytes(wl, seed=seed)
    g = torch.Generator().manual_seed(seed)
    shape = (1, wl.H, wl.L, wl.d)
    q, k, v, do = (torch.randn(shape, generator=g).to(torch.bfloat16).to(torch.float64).numpy() for _ in range(4))
    return x, q, k, v, do


def cpu_baseline(wl, budget_s=12.0, seed=0):
    """The oracle on the host cores over a bounded sample of the workload:
    (sample, head) units, one head of each class first, until budget_s."""
    x, q, k, v, do = oracle_inputs(wl, seed)
    hc = wl.head_classes()
    order = [0, wl.H // 2, 3 * wl.H // 4]
    order += [h for h in range(wl.H) if h not in order]
    flops, t0, units = 0, time.perf_counter(), 0
    while units < 3 or time.perf_counter() - t0 < budget_s:
        flops += oracle_sample_step(wl, x, q, k, v, do, hc, order[units % len(order)])
        units += 1
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{units} (sample, head) units of the {wl.S}x{wl.H} workload: each the gzip lengths, "
                      f"flags and mask of a sample and the forward + backward of one head (classes in "
                      f"turn), float64 numpy; {dt:.1f} s"}


# ------------------------------------------------------------ ranks
# Data-parallel with no exchange on the data path: every rank runs the whole
# path on its own batch; the only collectives are a barrier around the timed
# region and the max-over-ranks of the timed milliseconds.

def rank_inputs(wl, rank):
    """This rank's byte batch: the workload's generator seeded by the rank."""
    return W.batch_bytes(wl, seed=rank)


def max_over_ranks(ms, world, device):
    """The largest of the ranks' timed milliseconds (a MAX all-reduce)."""
    if world == 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world, work_per_rank, ms_per_step):
    """Work of all ranks per second at the slowest rank's step time (weak scaling)."""
    return world * work_per_rank / (ms_per_step * 1e-3)


def run_reference(args, rank, world):
    wl = W.WORKLOADS[WORKLOAD]
    if rank != 0:
        return 0
    x, q, k, v, do = oracle_inputs(wl, 0)
    hc = wl.head_classes()
    order = [0, wl.H // 2, 3 * wl.H // 4]
    for i in range(args.warmup):
        oracle_sample_step(wl, x, q, k, v, do, hc, order[i % 3])
    times, flops = [], 0
    for i in range(args.steps):
        t0 = time.perf_counter()
        flops += oracle_sample_step(wl, x, q, k, v, do, hc, order[i % 3])
        times.append(time.perf_counter() - t0)
    total = sum(times)
    val = flops / total / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": workload_desc(wl)},
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
                             "sample": "each step: gzip lengths, flags and mask of sample 0 and forward + "
                                       "backward of one head (classes in turn), float64 numpy"},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ------------------------------------------------------------------ ours

# The kernels behind each timed call, and the sources whose hash ties a
# recorded traffic figure to the code that produced it.
_TRAFFIC_CALLS = {
    "gsa_attn_fwd": (["attn_fwd_persist_kernel<64, 0>"],
                     ["content_adaptive_block_b200/csrc/attn_fwd_bf16.cuh",
                      "content_adaptive_block_b200/csrc/attn_fwd_persist.cuh"]),
    "gsa_attn_bwd": (["dot_kernel<64>", "dq_persist_kernel<0>", "dkdv_persist_kernel<0>"],
                     ["content_adaptive_block_b200/csrc/attn_bwd_bf16.cuh",
                      "content_adaptive_block_b200/csrc/attn_bwd_persist.cuh",
                      "content_adaptive_block_b200/csrc/attn_bwd_dq_persist.cuh"]),
}
_TRAFFIC_COMMON = ["content_adaptive_block_b200/csrc/common.cuh", "content_adaptive_block_b200/csrc/tiles.cuh",
                   "content_adaptive_block_b200/csrc/gsa.cu"]


def record_traffic(csv_path, capture):
    """Write profiles/traffic.json from an ncu raw-page CSV export (one
    launch per kernel): dram read + write bytes per call, summed over the
    call's kernels, with the hash of the sources they were built from."""
    import csv
    import hashlib
    rows = list(csv.reader(open(csv_path)))
    hdr, units, data = rows[0], rows[1], rows[2:]
    col = {h: i for i, h in enumerate(hdr)}
    scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}

    def dram(row):
        tot = 0.0
        for m in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            tot += float(row[col[m]].replace(",", "")) * scale[units[col[m]]]
        return tot

    out = {}
    for call, (kernels, srcs) in _TRAFFIC_CALLS.items():
        found = {}
        for row in data:
            name = row[col["Kernel Name"]]
            for k in kernels:
                if k in name and k not in found:
                    found[k] = dram(row)
        if len(found) != len(kernels):
            continue
        sources = srcs + _TRAFFIC_COMMON
        h = hashlib.sha256()
        for s in sources:
            with open(os.path.join(ROOT, s), "rb") as fh:
                h.update(fh.read())
        out[call] = {"bytes_per_launch": int(sum(found.values())), "per_kernel": {k: int(v) for k, v in found.items()},
                     "sources": sources, "sha256": h.hexdigest(), "capture": capture}
    with open(os.path.join(ROOT, "profiles", "traffic.json"), "w") as fh:
        json.dump(out, fh, indent=1)
    print(json.dumps(out))


_MASK_INST_SOURCES = ["content_adaptive_block_b200/csrc/deflate_lane.cuh", "content_adaptive_block_b200/csrc/common.cuh",
                      "content_adaptive_block_b200/csrc/gsa.cu"]


def _sources_hash(sources):
    import hashlib
    h = hashlib.sha256()
    for s in sources:
        with open(os.path.join(ROOT, s), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def record_mask_inst(csv_path, capture):
    """Write profiles/mask_inst.json from an ncu raw-page CSV export of one
    launch of the lengths kernel on the headline mask point: warp instructions
    executed per input byte, with the hash of the sources it was built from."""
    import csv
    rows = list(csv.reader(open(csv_path)))
    hdr, data = rows[0], rows[2:]
    col = {h: i for i, h in enumerate(hdr)}
    row = next(r for r in data if "block_lengths" in r[col["Kernel Name"]])
    inst = float(row[col["smsp__inst_executed.sum"]].replace(",", ""))
    wl = W.mask_sweep(*MASK_POINT)
    nbytes = wl.S * wl.L
    rec = {"kernel": row[col["Kernel Name"]].split("(")[0], "workload": f"b{MASK_POINT[0]}_f{MASK_POINT[1]}: {wl.S} x {wl.L} bytes",
           "warp_inst": inst, "bytes": nbytes, "inst_per_byte": inst / nbytes,
           "issue_active_pct": float(row[col["smsp__issue_active.avg.pct_of_peak_sustained_active"]]),
           "warps_active_pct": float(row[col["sm__warps_active.avg.pct_of_peak_sustained_active"]]),
           "sources": _MASK_INST_SOURCES, "sha256": _sources_hash(_MASK_INST_SOURCES), "capture": capture}
    with open(os.path.join(ROOT, "profiles", "mask_inst.json"), "w") as fh:
        json.dump(rec, fh, indent=1)
    return rec


def _mask_inst_record():
    """Warp instructions per input byte of the lengths kernel, if its sources are unchanged since the capture."""
    try:
        with open(os.path.join(ROOT, "profiles", "mask_inst.json")) as fh:
            rec = json.load(fh)
        return rec if _sources_hash(rec["sources"]) == rec["sha256"] else None
    except Exception:
        return None


def _traffic_record(kernel):
    """dram bytes per launch from a committed ncu capture, if the kernel's
    source is unchanged since (else None)."""
    try:
        import hashlib
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f).get(kernel)
        if not rec:
            return None
        h = hashlib.sha256()
        for src in rec["sources"]:
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
        return rec["bytes_per_launch"] if h.hexdigest() == rec["sha256"] else None
    except Exception:
        return None


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import content_adaptive_block_b200 as gsa
    from content_adaptive_block_b200 import build

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    build.build()
    wl = W.WORKLOADS[WORKLOAD]
    peaks = _peaks()
    hc = [int(c) for c in wl.head_classes()]

    # ---- inputs (per-rank seed), resident in HBM
    x_host = rank_inputs(wl, rank)
    x = torch.from_numpy(x_host).to(dev)
    q, k, v, do = W.qkv(wl, seed=rank, device=dev, grad=True)
    lengths = torch.empty((wl.S, wl.N), dtype=torch.int32, device=dev)
    flags = torch.empty((wl.S, wl.N), dtype=torch.uint8, device=dev)
    csr = gsa.BlockCsr(wl.S, wl.N, dev)
    o = torch.empty_like(q)
    lse = torch.empty((wl.S, wl.H, wl.L), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(gsa.gsa_attn_bwd_workspace(q, wl.b, hc), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    counters = torch.zeros(1, dtype=torch.int32, device=dev)
    names = ("gsa_mask_pipeline", "gsa_attn_fwd", "gsa_attn_bwd")
    launches_per_step = 1 + 1 + 3

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        gsa.gsa_mask_pipeline(x, wl.b, wl.w, csr, lengths=lengths, flags=flags, counters=counters,
                              head_classes=hc)
        if ev:
            ev[1].record(stream)
        gsa.gsa_attn_fwd(q, k, v, csr, hc, wl.b, o=o, lse=lse)
        if ev:
            ev[2].record(stream)
        gsa.gsa_attn_bwd(q, k, v, o, lse, do, csr, hc, wl.b, dq=dq, dk=dk, dv=dv, workspace=ws)
        if ev:
            ev[3].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert gsa.gsa_device_error() == 0, "a kernel gave up a bounded wait"

    # algorithmic work of this rank's batch
    nnz = csr_nnz(csr)
    pairs = sum(live_token_pairs_from_counts(nnz[s], wl.N, wl.b, hc) for s in range(wl.S))
    fwd_flops, bwd_flops = 4 * wl.d * pairs, 8 * wl.d * pairs
    step_flops = fwd_flops + bwd_flops
    dense_pairs = wl.S * wl.H * wl.L * (wl.L + 1) // 2

    sampler = None
    if rank == 0:
        # NVML in a child process (many samples inside a short timed region); nvidia-smi when NVML is absent
        try:
            sampler = NvmlClockSampler(local_rank)
            sampler.start()
        except Exception:
            sampler = ClockSampler(local_rank)
            sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()
        step(evs[i])
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None

    per_call = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(len(names))]
                         for i in range(args.steps)])
    step_ms = per_call.sum(axis=1)
    total_ms = max_over_ranks(float(step_ms.sum()), world, dev)
    ms_per_step = total_ms / args.steps
    value = whole_job_rate(world, step_flops, ms_per_step) / 1e12

    # ---- end to end through the API with host buffers
    e2e = None if args.no_e2e else e2e_timing(args, gsa, wl, hc, x_host, q, k, v, do, stream, world, dev,
                                                 step_flops)

    # ---- mask-stage sweep (secondary metric), rank 0
    mask = mask_stage(gsa, dev) if (rank == 0 and not args.no_mask_sweep) else None
    sweep = seq_sweep(gsa, dev) if (rank == 0 and not args.no_seq_sweep) else None
    cfgs = config_lines(gsa, dev) if (rank == 0 and not args.no_configs) else None
    variants = mask_variants(gsa, dev) if (rank == 0 and not args.no_mask_variants) else None
    block = lm_block(gsa, dev) if (rank == 0 and not args.no_lm_block) else None

    if rank != 0:
        return 0
    return report(args, wl, world, peaks, per_call, names, ms_per_step, value, fwd_flops, bwd_flops, step_flops,
                  pairs, dense_pairs, launches_per_step, e2e, clocks, mask, sweep, variants, block, cfgs)


def e2e_timing(args, gsa, wl, hc, x_host, q, k, v, do, stream, world, dev, step_flops):
    """Whole-job throughput through the public API with the data in pinned
    host memory: every step uploads its inputs (bytes, Q, K, V, dO), runs
    lengths -> flags -> lists -> forward -> backward, and downloads dQ, dK,
    dV.  Uploads, compute and downloads of consecutive steps run on separate
    streams over two sets of device tensors, as a training input pipeline
    would; the timed region opens before the first upload and closes after
    the last download."""
    import torch
    import torch.distributed as dist
    x_pin = torch.from_numpy(x_host).pin_memory()
    q_pin, k_pin, v_pin, do_pin = (t.cpu().pin_memory() for t in (q, k, v, do))

    def make_set():
        st = {"x": torch.empty(x_pin.shape, dtype=x_pin.dtype, device=dev)}
        for name, t in (("q", q), ("k", k), ("v", v), ("do", do)):
            st[name] = torch.empty_like(t)
        st["lengths"] = torch.empty((wl.S, wl.N), dtype=torch.int32, device=dev)
        st["flags"] = torch.empty((wl.S, wl.N), dtype=torch.uint8, device=dev)
        st["csr"] = gsa.BlockCsr(wl.S, wl.N, dev)
        st["counters"] = torch.zeros(1, dtype=torch.int32, device=dev)
        st["o"] = torch.empty_like(q)
        st["lse"] = torch.empty((wl.S, wl.H, wl.L), dtype=torch.float32, device=dev)
        for name in ("dq", "dk", "dv"):
            st[name] = torch.empty_like(q)
        st["ws"] = torch.empty(gsa.gsa_attn_bwd_workspace(q, wl.b, hc), dtype=torch.uint8, device=dev)
        st["host_out"] = [torch.empty_like(q, device="cpu").pin_memory() for _ in range(3)]
        return st

    sets = [make_set(), make_set()]
    h2d = x_pin.numel() + sum(t.numel() * t.element_size() for t in (q_pin, k_pin, v_pin, do_pin))
    d2h = sum(t.numel() * t.element_size() for t in sets[0]["host_out"])
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = {key: [torch.cuda.Event() for _ in range(2)] for key in ("up", "comp", "down")}

    def e2e_step(i):
        j = i % 2
        st = sets[j]
        with torch.cuda.stream(up):
            if i >= 2:
                up.wait_event(ev["comp"][j])            # step i - 2 consumed this set's inputs
            st["x"].copy_(x_pin, non_blocking=True)
            for name, src in (("q", q_pin), ("k", k_pin), ("v", v_pin), ("do", do_pin)):
                st[name].copy_(src, non_blocking=True)
            ev["up"][j].record(up)
        stream.wait_event(ev["up"][j])
        if i >= 2:
            stream.wait_event(ev["down"][j])            # step i - 2's outputs left this set
        gsa.gsa_mask_pipeline(st["x"], wl.b, wl.w, st["csr"], lengths=st["lengths"], flags=st["flags"],
                              counters=st["counters"], head_classes=hc)
        gsa.gsa_attn_fwd(st["q"], st["k"], st["v"], st["csr"], hc, wl.b, o=st["o"], lse=st["lse"])
        gsa.gsa_attn_bwd(st["q"], st["k"], st["v"], st["o"], st["lse"], st["do"], st["csr"], hc, wl.b,
                         dq=st["dq"], dk=st["dk"], dv=st["dv"], workspace=st["ws"])
        ev["comp"][j].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(ev["comp"][j])
            for dst, name in zip(st["host_out"], ("dq", "dk", "dv")):
                dst.copy_(st[name], non_blocking=True)
            ev["down"][j].record(down)

    e2e_steps = max(4, min(args.steps, 48))   # steady state: one upload and one download of fill/drain
    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    up.wait_event(e0)
    for i in range(e2e_steps):
        e2e_step(i)
    stream.wait_event(ev["down"][(e2e_steps - 1) % 2])
    e1.record(stream)
    torch.cuda.synchronize()
    assert gsa.gsa_device_error() == 0, "a kernel gave up a bounded wait"
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world, dev)
    e2e_value = whole_job_rate(world, step_flops, e2e_ms) / 1e12
    return {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": e2e_ms,
            "overlap": "uploads, compute and downloads of consecutive steps on three streams, "
                       "two sets of device tensors"}


def report(args, wl, world, peaks, per_call, names, ms_per_step, value, fwd_flops, bwd_flops, step_flops, pairs,
           dense_pairs, launches_per_step, e2e, clocks, mask, sweep=None, variants=None, block=None, cfgs=None):
    call_ms = {n: float(per_call[:, j].mean()) for j, n in enumerate(names)}
    bwd_ms, fwd_ms = call_ms["gsa_attn_bwd"], call_ms["gsa_attn_fwd"]
    # the calls are event-timed one by one inside a short region: the burst peak is their denominator
    peak_t = peaks["bf16_tflops"]
    bwd_ach = bwd_flops / (bwd_ms * 1e-3) / 1e12
    fwd_ach = fwd_flops / (fwd_ms * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload_desc(wl),
                   "l2": "flushed between steps (256 MiB write outside the timed events); "
                         "q/k/v/dO alone are 403 MB",
                   "live_token_pairs": pairs, "dense_causal_pairs": dense_pairs,
                   "live_fraction": pairs / dense_pairs, "step_gflop": step_flops / 1e9},
        "roofline": {"kernel": "gsa_attn_bwd (dot + dq + dk/dv launches)", "bound": "tensor",
                     "achieved": bwd_ach, "peak": peak_t, "unit": "TFLOP/s", "frac": bwd_ach / peak_t,
                     "peak_kind": f"bf16 burst, {peaks['source']}",
                     "frac_of_sustained": bwd_ach / peaks["bf16_tflops_sustained"],
                     "traffic": _traffic_record("gsa_attn_bwd")},
        "roofline_fwd": {"kernel": "gsa_attn_fwd", "bound": "tensor", "achieved": fwd_ach, "peak": peak_t,
                         "unit": "TFLOP/s", "frac": fwd_ach / peak_t, "traffic": _traffic_record("gsa_attn_fwd")},
        "call_ms": call_ms,
        "gpu_launches": launches_per_step * args.steps,
        "e2e": e2e,
        "clocks": clocks,
    }
    if mask:
        line["mask_stage"] = mask
    if cfgs:
        line["configs"] = cfgs
    if sweep:
        line["seq_sweep"] = sweep
    if variants:
        line["mask_variants"] = variants
    if block:
        line["lm_block"] = block
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    print(json.dumps(line))
    return 0


def mask_stage(gsa, dev):
    """gzip-mask GB/s of input bytes: lengths + flags + block lists over 256
    samples x 8192 bytes, by the three calls and by the one-launch
    gsa_mask_pipeline ("gbs" is the faster of the two).  Input batches rotate
    over > 320 MiB so the bytes come from HBM, not L2."""
    import torch
    out = {"metric": "gzip-mask GB/s of input bytes", "unit": "GB/s", "points": {}}
    n_rot = 160
    for b, f in W.MASK_SWEEP:
        wl = W.mask_sweep(b, f)
        base = torch.from_numpy(W.batch_bytes(wl, seed=0)).to(dev)
        # distinct copies: rotated rows keep the statistics, change the addresses
        batches = [torch.roll(base, shifts=i, dims=0).contiguous() for i in range(n_rot)]
        lengths = torch.empty((wl.S, wl.N), dtype=torch.int32, device=dev)
        flags = torch.empty((wl.S, wl.N), dtype=torch.uint8, device=dev)
        csr = gsa.BlockCsr(wl.S, wl.N, dev)
        counters = torch.zeros(1, dtype=torch.int32, device=dev)

        def one(xb):
            gsa.gsa_block_lengths(xb, wl.b, out=lengths)
            gsa.gsa_literal_flags(lengths, out=flags)
            gsa.gsa_build_block_csr(flags, wl.w, csr)

        def fused(xb):
            gsa.gsa_mask_pipeline(xb, wl.b, wl.w, csr, lengths=lengths, flags=flags, counters=counters)

        for i in range(3):
            one(batches[i])
            fused(batches[i])
        torch.cuda.synchronize()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        e[0].record()
        for i in range(n_rot):
            gsa.gsa_block_lengths(batches[i], wl.b, out=lengths)
        e[1].record()
        for i in range(n_rot):
            one(batches[i])
        e[2].record()
        for i in range(n_rot):
            fused(batches[i])
        e[3].record()
        torch.cuda.synchronize()
        len_ms = e[0].elapsed_time(e[1]) / n_rot
        sep_ms = e[1].elapsed_time(e[2]) / n_rot
        all_ms = e[2].elapsed_time(e[3]) / n_rot
        nbytes = wl.S * wl.L
        one(batches[0])
        nnz_sc = csr_nnz(csr)
        nnz = int(nnz_sc.sum())
        # what the stage writes: lengths (int32) and flags (uint8) per block;
        # CSR and CSC pointers, entries and pairing orders (int32) per (sample,
        # class) — the three calls for every class, the pipeline for the
        # literal and hybrid classes (the local class's lists are implicit)
        out_bytes = (wl.S * wl.N * (4 + 1)
                     + 4 * (2 * wl.S * 3 * (wl.N + 1) + 2 * nnz + 2 * wl.S * 3 * wl.N))
        nnz_pipe = int(nnz_sc[:, 1:].sum())
        out_bytes_pipe = (wl.S * wl.N * (4 + 1)
                          + 4 * (2 * (2 * wl.S) * (wl.N + 1) + 2 * nnz_pipe + 2 * (2 * wl.S) * wl.N))
        best_ms = min(sep_ms, all_ms)
        out["points"][f"b{b}_f{f}"] = {
            "gbs": nbytes / (best_ms * 1e-3) / 1e9, "lengths_gbs": nbytes / (len_ms * 1e-3) / 1e9,
            "three_calls_gbs": nbytes / (sep_ms * 1e-3) / 1e9, "pipeline_gbs": nbytes / (all_ms * 1e-3) / 1e9,
            "ms": best_ms, "lengths_ms": len_ms, "three_calls_ms": sep_ms, "pipeline_ms": all_ms,
            "bytes_in": nbytes, "bytes_out": out_bytes if sep_ms <= all_ms else out_bytes_pipe,
            "bytes_out_three_calls": out_bytes, "bytes_out_pipeline": out_bytes_pipe,
            "hbm_frac": (nbytes + (out_bytes if sep_ms <= all_ms else out_bytes_pipe)) / (best_ms * 1e-3) / 1e9
                        / _peaks()["hbm_gbs"]}
    key = f"b{MASK_POINT[0]}_f{MASK_POINT[1]}"
    out["value"] = out["points"][key]["gbs"]
    # graded against HBM: bytes in (input) and out (lengths, flags, lists) over
    # the stage's time.  The lengths kernel is latency-bound integer code far
    # below that; its issue-rate use (warp instructions per byte from an ncu
    # capture, 4 per cycle per SM at the maximum clock) is reported beside it.
    rec = _mask_inst_record()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    peak_issue = 4.0 * sms * _peaks()["sm_max_mhz"] * 1e6
    pt = out["points"][key]
    issue = rec["inst_per_byte"] * pt["lengths_gbs"] * 1e9 if rec else None
    out["roofline"] = {"kernel": "lengths + flags + lists", "bound": "hbm", "unit": "GB/s",
                       "achieved": (pt["bytes_in"] + pt["bytes_out"]) / (pt["ms"] * 1e-3) / 1e9,
                       "peak": _peaks()["hbm_gbs"], "frac": pt["hbm_frac"],
                       "inst_per_byte": rec["inst_per_byte"] if rec else None,
                       "issue_frac": issue / peak_issue if rec else None,
                       "note": "instructions per byte from profiles/mask_inst.json (null when the sources changed)"}
    out["workload"] = f"{key}: 256 x 8192 bytes, w=2"
    return out


def config_lines(gsa, dev, steps=20, warmup=3):
    """The attention calls on the other workloads: tiny fp32 (forward), 8 x 4K
    (forward) and 1 x 64K (d = 128, forward and backward), each call timed
    alone with CUDA events, L2 flushed before every call.  Per call the
    algorithmic work (live token pairs P: forward 4 d P FLOPs, backward 8 d P)
    and bytes (forward Q, K, V, O and LSE; backward Q, K, V, O, dO, LSE in and
    dQ, dK, dV out, once each), reported as FLOP/s against the bf16 burst peak
    and GB/s against the measured HBM copy bandwidth: the 4K and 64K calls
    sit near or below the ridge point, so their HBM fraction is the bar."""
    import torch
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    peaks = _peaks()
    out = {"unit_flops": "TFLOP/s", "unit_bytes": "GB/s", "peak_tflops": peaks["bf16_tflops"],
           "peak_gbs": peaks["hbm_gbs"], "workloads": {}}
    for name in ("tiny_fp32", "b8_4k", "b1_64k"):
        wl = W.WORKLOADS[name]
        hc = [int(c) for c in wl.head_classes()]
        x = torch.from_numpy(W.batch_bytes(wl, seed=0)).to(dev)
        flags = gsa.gsa_literal_flags(gsa.gsa_block_lengths(x, wl.b))
        csr = gsa.gsa_build_block_csr(flags, wl.w)
        f32 = wl.dtype == "f32"
        q, k, v, do = W.qkv(wl, seed=0, device=dev, grad=True)
        o = torch.empty_like(q)
        lse = torch.empty((wl.S, wl.H, wl.L), dtype=torch.float32, device=dev)
        calls = [("fwd", lambda: gsa.gsa_attn_fwd(q, k, v, csr, hc, wl.b, o=o, lse=lse))]
        if wl.backward:
            dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
            ws = torch.empty(gsa.gsa_attn_bwd_workspace(q, wl.b, hc), dtype=torch.uint8, device=dev)
            calls.append(("bwd", lambda: gsa.gsa_attn_bwd(q, k, v, o, lse, do, csr, hc, wl.b, dq=dq, dk=dk, dv=dv,
                                                          workspace=ws)))
        nnz = csr_nnz(csr)
        pairs = sum(live_token_pairs_from_counts(nnz[s], wl.N, wl.b, hc) for s in range(wl.S))
        esz = 4 if f32 else 2
        tensor = wl.S * wl.H * wl.L * wl.d * esz
        vec = wl.S * wl.H * wl.L * 4
        rec = {"config": workload_desc(wl), "live_token_pairs": pairs,
               "literal_blocks": float(flags.float().sum(dim=1).mean().item()),
               "live_fraction": pairs / (wl.S * wl.H * wl.L * (wl.L + 1) // 2)}
        for label, fn in calls:
            for _ in range(warmup):
                flush.zero_()
                fn()
            torch.cuda.synchronize()
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
            for e0, e1 in evs:
                flush.zero_()
                e0.record()
                fn()
                e1.record()
            torch.cuda.synchronize()
            assert gsa.gsa_device_error() == 0, "a kernel gave up a bounded wait"
            ms = float(np.mean([e0.elapsed_time(e1) for e0, e1 in evs]))
            flops = (4 if label == "fwd" else 8) * wl.d * pairs
            nbytes = 4 * tensor + vec if label == "fwd" else 8 * tensor + vec
            tf = flops / (ms * 1e-3) / 1e12
            gbs = nbytes / (ms * 1e-3) / 1e9
            rec[label] = {"ms": ms, "gflop": flops / 1e9, "mbytes": nbytes / 1e6, "tflops": tf,
                          "frac_of_burst": tf / peaks["bf16_tflops"], "gbs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"],
                          "bound": "hbm" if flops / nbytes < peaks["bf16_tflops"] * 1e3 / peaks["hbm_gbs"] else "tensor"}
            if f32:
                rec[label]["note"] = "float32 CUDA-core path (parity configuration); launch-bound at this size"
        out["workloads"][name] = rec
        del q, k, v, do, o
    return out


def seq_sweep(gsa, dev, steps=10, warmup=3):
    """The path (lengths -> flags -> lists -> forward -> backward) on the
    8x8K configuration's shape at L = 4K .. 64K bytes per sample, the batch
    shrunk so that S * L = 64 KiB per step: algorithmic fwd+bwd TFLOP/s per
    length, L2 flushed between steps, CUDA events per step."""
    import torch
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    out = {"metric": "live-block attn TFLOP/s fwd+bwd", "unit": "TFLOP/s",
           "shape": "b=64, w=2, 12 heads (6 local/3 literal/3 hybrid), d=64, bf16, S*L = 65536", "points": {}}
    for L in W.SEQ_SWEEP:
        wl = W.seq_sweep(L)
        hc = [int(c) for c in wl.head_classes()]
        x = torch.from_numpy(W.batch_bytes(wl, seed=0)).to(dev)
        q, k, v, do = W.qkv(wl, seed=0, device=dev, grad=True)
        lengths = torch.empty((wl.S, wl.N), dtype=torch.int32, device=dev)
        flags = torch.empty((wl.S, wl.N), dtype=torch.uint8, device=dev)
        csr = gsa.BlockCsr(wl.S, wl.N, dev)
        o = torch.empty_like(q)
        lse = torch.empty((wl.S, wl.H, wl.L), dtype=torch.float32, device=dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(gsa.gsa_attn_bwd_workspace(q, wl.b, hc), dtype=torch.uint8, device=dev)

        def one(ev=None):
            if ev:
                ev[0].record()
            gsa.gsa_block_lengths(x, wl.b, out=lengths)
            gsa.gsa_literal_flags(lengths, out=flags)
            gsa.gsa_build_block_csr(flags, wl.w, csr)
            if ev:
                ev[1].record()
            gsa.gsa_attn_fwd(q, k, v, csr, hc, wl.b, o=o, lse=lse)
            if ev:
                ev[2].record()
            gsa.gsa_attn_bwd(q, k, v, o, lse, do, csr, hc, wl.b, dq=dq, dk=dk, dv=dv, workspace=ws)
            if ev:
                ev[3].record()

        for _ in range(warmup):
            flush.zero_()
            one()
        torch.cuda.synchronize()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
        for i in range(steps):
            flush.zero_()
            one(evs[i])
        torch.cuda.synchronize()
        assert gsa.gsa_device_error() == 0, "a kernel gave up a bounded wait"
        t = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(3)] for i in range(steps)]).mean(axis=0)
        nnz = csr_nnz(csr)
        pairs = sum(live_token_pairs_from_counts(nnz[s], wl.N, wl.b, hc) for s in range(wl.S))
        flops = 12 * wl.d * pairs
        ms = float(t.sum())
        out["points"][f"{L // 1024}k"] = {
            "L": L, "S": wl.S, "ms": ms, "mask_ms": float(t[0]), "fwd_ms": float(t[1]), "bwd_ms": float(t[2]),
            "tflops": flops / (ms * 1e-3) / 1e12, "attn_tflops": flops / ((t[1] + t[2]) * 1e-3) / 1e12,
            "live_fraction": pairs / (wl.S * wl.H * wl.L * (wl.L + 1) // 2),
            "literal_fraction": float(flags.float().mean().item())}
        del q, k, v, do, o, dq, dk, dv, ws
    return out


def mask_variants(gsa, dev, steps=10, warmup=3):
    """The attention (forward + backward) on the 8x8K configuration's inputs
    under the adaptive gzip mask and under the fixed BigBird and Longformer
    block masks built by gsa_build_fixed_csr: per mask its list-building
    time, live fraction and fwd+bwd time and algorithmic TFLOP/s, L2 flushed
    between steps, CUDA events per step."""
    import torch
    wl = W.WORKLOADS["b8_8k"]
    hc = [int(c) for c in wl.head_classes()]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    x = torch.from_numpy(W.batch_bytes(wl, seed=0)).to(dev)
    q, k, v, do = W.qkv(wl, seed=0, device=dev, grad=True)
    o = torch.empty_like(q)
    lse = torch.empty((wl.S, wl.H, wl.L), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(gsa.gsa_attn_bwd_workspace(q, wl.b, hc), dtype=torch.uint8, device=dev)
    out = {"metric": "live-block attn TFLOP/s fwd+bwd", "unit": "TFLOP/s",
           "shape": "8 x 8192 bytes, b=64, 12 heads, d=64, bf16", "masks": {}}
    lengths = torch.empty((wl.S, wl.N), dtype=torch.int32, device=dev)
    flags = torch.empty((wl.S, wl.N), dtype=torch.uint8, device=dev)
    variants = [("gzip", None)] + [(name, cfg) for name, cfg in W.FIXED_MASKS.items()]
    for name, cfg in variants:
        csr = gsa.BlockCsr(wl.S, wl.N, dev)
        if cfg is None:
            build = (lambda csr=csr: (gsa.gsa_block_lengths(x, wl.b, out=lengths),
                                      gsa.gsa_literal_flags(lengths, out=flags),
                                      gsa.gsa_build_block_csr(flags, wl.w, csr)))
        else:
            rnd = None
            if cfg["r"] > 0:
                rnd = torch.from_numpy(W.random_words(wl.S, wl.N, cfg["r"], seed=0).view(np.int32)).to(dev)
            build = (lambda cfg=cfg, rnd=rnd, csr=csr:
                     gsa.gsa_build_fixed_csr(cfg["kind"], wl.S, wl.N, cfg["w"], cfg["g"], rnd, device=dev, csr=csr))

        def one(ev=None):
            if ev:
                ev[0].record()
            build()
            if ev:
                ev[1].record()
            gsa.gsa_attn_fwd(q, k, v, csr, hc, wl.b, o=o, lse=lse)
            gsa.gsa_attn_bwd(q, k, v, o, lse, do, csr, hc, wl.b, dq=dq, dk=dk, dv=dv, workspace=ws)
            if ev:
                ev[2].record()

        for _ in range(warmup):
            flush.zero_()
            one()
        torch.cuda.synchronize()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        for i in range(steps):
            flush.zero_()
            one(evs[i])
        torch.cuda.synchronize()
        assert gsa.gsa_device_error() == 0, "a kernel gave up a bounded wait"
        t = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(2)] for i in range(steps)]).mean(axis=0)
        nnz = csr_nnz(csr)
        pairs = sum(live_token_pairs_from_counts(nnz[s], wl.N, wl.b, hc) for s in range(wl.S))
        flops = 12 * wl.d * pairs
        out["masks"][name] = {
            "params": None if cfg is None else {kk: cfg[kk] for kk in ("w", "g", "r")},
            "build_ms": float(t[0]), "attn_ms": float(t[1]), "attn_tflops": flops / (t[1] * 1e-3) / 1e12,
            "live_fraction": pairs / (wl.S * wl.H * wl.L * (wl.L + 1) // 2)}
    return out


def lm_block(gsa, dev, steps=10, warmup=3):
    """One ByteLM block (D = 768, 12 heads, MLP 3072) forward + backward on
    the 8x8K bench batch under its gzip mask: per step the mask pipeline, the
    block forward and the block backward, L2 flushed between steps, CUDA
    events.  FLOPs: the projections' 2 T D (3D + D + 2F) forward and twice
    that backward, plus the attention's algorithmic 12 d P."""
    import torch
    wl = W.WORKLOADS["b8_8k"]
    c = W.LM_BLOCK
    D, H, F = c["D"], c["H"], c["F"]
    hc = [int(v) for v in wl.head_classes()]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    x = torch.from_numpy(W.batch_bytes(wl, seed=0)).to(dev)
    wt = W.lm_weights(D, F, seed=0, device=dev)
    g = torch.Generator(device="cpu")
    g.manual_seed(77)
    dy = torch.randn((wl.S, wl.L, D), generator=g).bfloat16().to(dev)
    lengths = torch.empty((wl.S, wl.N), dtype=torch.int32, device=dev)
    flags = torch.empty((wl.S, wl.N), dtype=torch.uint8, device=dev)
    counters = torch.zeros(1, dtype=torch.int32, device=dev)
    csr = gsa.BlockCsr(wl.S, wl.N, dev)
    y = torch.empty((wl.S, wl.L, D), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(gsa.gsa_lm_block_workspace(wl.S, wl.L, D, H, F, hc), dtype=torch.uint8, device=dev)
    grads = {n: torch.empty(wt[n].shape, dtype=torch.float32, device=dev) for n in gsa.LM_WEIGHTS}

    def one(ev=None):
        if ev:
            ev[0].record()
        gsa.gsa_mask_pipeline(x, wl.b, wl.w, csr=csr, lengths=lengths, flags=flags, counters=counters)
        if ev:
            ev[1].record()
        gsa.gsa_lm_block_fwd(x, wt, csr, hc, y=y, workspace=ws)
        if ev:
            ev[2].record()
        gsa.gsa_lm_block_bwd(x, wt, csr, hc, dy, ws, grads=grads)
        if ev:
            ev[3].record()

    for _ in range(warmup):
        flush.zero_()
        one()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        one(evs[i])
    torch.cuda.synchronize()
    assert gsa.gsa_device_error() == 0, "a kernel gave up a bounded wait"
    t = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(3)] for i in range(steps)]).mean(axis=0)
    T = wl.S * wl.L
    gemm_fwd = 2.0 * T * D * (3 * D + D + 2 * F)
    nnz = csr_nnz(csr)
    pairs = sum(live_token_pairs_from_counts(nnz[s], wl.N, wl.b, hc) for s in range(wl.S))
    attn = 12.0 * 64 * pairs
    ms = float(t.sum())
    return {"metric": "ByteLM block TFLOP/s fwd+bwd (projections + live-block attention)", "unit": "TFLOP/s",
            "shape": f"8 x 8192 bytes, D={D}, H={H} x 64, F={F}, gzip mask b=64 w=2, bf16",
            "ms": ms, "mask_ms": float(t[0]), "fwd_ms": float(t[1]), "bwd_ms": float(t[2]),
            "tflops": (3 * gemm_fwd + attn) / (ms * 1e-3) / 1e12, "gemm_gflop": 3 * gemm_fwd / 1e9,
            "attn_gflop": attn / 1e9, "projections": "this library's tcgen05 GEMM (bf16, fp32 accumulate in TMEM)"}


def profile_lengths():
    """gsa_block_lengths three times on the headline mask point (256 x 8192
    bytes, b = 64, high-entropy fraction 0.3): a short program for an ncu
    capture of the lengths kernel."""
    import torch
    import content_adaptive_block_b200 as gsa
    from content_adaptive_block_b200 import build
    build.build()
    wl = W.mask_sweep(*MASK_POINT)
    x = torch.from_numpy(W.batch_bytes(wl)).cuda()
    for _ in range(3):
        gsa.gsa_block_lengths(x, wl.b)
    torch.cuda.synchronize()
    print("lengths ok")
    return 0


def profile_pipeline():
    """gsa_mask_pipeline three times on the headline mask point (256 x 8192
    bytes, b = 64, high-entropy fraction 0.3, all three head classes): a
    short program for an ncu capture of the one-launch mask stage."""
    import torch
    import content_adaptive_block_b200 as gsa
    from content_adaptive_block_b200 import build
    build.build()
    wl = W.mask_sweep(*MASK_POINT)
    x = torch.from_numpy(W.batch_bytes(wl)).cuda()
    counters = torch.zeros(1, dtype=torch.int32, device="cuda")
    csr = gsa.BlockCsr(wl.S, wl.N, x.device)
    for _ in range(3):
        gsa.gsa_mask_pipeline(x, wl.b, wl.w, csr, counters=counters)
    torch.cuda.synchronize()
    assert gsa.gsa_device_error() == 0
    print("pipeline ok")
    return 0


def profile_lm():
    """One ByteLM block forward + backward on the 8x8K batch, twice: a short
    program for an ncu launch list of the block's kernels."""
    import torch
    import content_adaptive_block_b200 as gsa
    from content_adaptive_block_b200 import build
    build.build()
    lm_block(gsa, torch.device("cuda", 0), steps=1, warmup=1)
    print("lm ok")
    return 0


def profile_attn(name):
    """The mask and the attention calls of one workload, three times (a short
    program for an ncu capture of one attention kernel)."""
    import torch
    import content_adaptive_block_b200 as gsa
    from content_adaptive_block_b200 import build
    build.build()
    wl = W.WORKLOADS[name]
    hc = [int(c) for c in wl.head_classes()]
    x = torch.from_numpy(W.batch_bytes(wl)).cuda()
    csr = gsa.gsa_build_block_csr(gsa.gsa_literal_flags(gsa.gsa_block_lengths(x, wl.b)), wl.w)
    q, k, v, do = W.qkv(wl, seed=0, device="cuda", grad=True)
    for _ in range(3):
        o, lse = gsa.gsa_attn_fwd(q, k, v, csr, hc, wl.b)
        if wl.backward:
            gsa.gsa_attn_bwd(q, k, v, o, lse, do, csr, hc, wl.b)
    torch.cuda.synchronize()
    assert gsa.gsa_device_error() == 0
    print("attn ok")
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-mask-sweep", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-seq-sweep", action="store_true", help="skip the 4K..64K sequence-length sweep")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the tiny / 8x4K / 1x64K attention call timings")
    ap.add_argument("--no-lm-block", action="store_true", help="skip the ByteLM block timing")
    ap.add_argument("--record-mask-inst", metavar="CSV",
                    help="write profiles/mask_inst.json from an ncu raw-page CSV export and exit")
    ap.add_argument("--no-mask-variants", action="store_true",
                    help="skip the gzip / BigBird / Longformer mask comparison")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end timing")
    ap.add_argument("--record-traffic", metavar="NCU_RAW_CSV",
                    help="write profiles/traffic.json from an ncu raw-page CSV export and exit")
    ap.add_argument("--capture", default="", help="the ncu command recorded with --record-traffic")
    ap.add_argument("--profile-pipeline", action="store_true",
                    help="run gsa_mask_pipeline three times on the headline mask point and exit (for ncu)")
    ap.add_argument("--profile-lm", action="store_true",
                    help="run the ByteLM block forward + backward twice and exit (for ncu)")
    ap.add_argument("--profile-lengths", action="store_true",
                    help="run gsa_block_lengths three times on the headline mask point and exit (for ncu)")
    ap.add_argument("--profile-attn", metavar="WORKLOAD", choices=sorted(W.WORKLOADS),
                    help="run the workload's attention calls three times and exit (for ncu)")
    args = ap.parse_args()
    if args.profile_lengths:
        return profile_lengths()
    if args.profile_pipeline:
        return profile_pipeline()
    if args.profile_lm:
        return profile_lm()
    if args.profile_attn:
        return profile_attn(args.profile_attn)
    if args.record_traffic:
        record_traffic(args.record_traffic, args.capture)
        return 0
    if args.record_mask_inst:
        print(json.dumps(record_mask_inst(args.record_mask_inst, args.capture)))
        return 0
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        return run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
