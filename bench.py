#!/usr/bin/env python
"""Throughput of the STCA forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python -m torch.distributed.run --nproc-per-node N --master-addr 127.0.0.1 ... bench.py --gpus N

One step is one STCA forward over one batch of the 10K-history workload: 256 users with
L = 10,000 history items each (Zipf(1.1) over a 4M x 512 bf16 table, 16-bin time
feature), M = 3 layers, d = 512, H = 8, SwiGLU hidden 1024, 32 targets per user sharing
the user's K/V.  Inputs are synthetic and seeded; weights are random-init.  With N > 1
every rank is an independent replica serving its own users (weak scaling; the path has
no exchange step between users).  Rank 0 prints one JSON line.

Timing: W warm-up steps, then K steps between CUDA events on the launching stream with a
barrier and a synchronize on both sides, max over ranks.  Inside that region only the
dominant stage's launches are bracketed by events (its per-launch time gives the roofline);
the per-stage table comes from a second pass of K steps with every stage bracketed.

--workload 2 | 4 | 5 times the other forms on their own workloads (Beta-ragged STCA, the
pointwise ReLU target attention, the multi-sequence decode); the default is the 10K-history
STCA step above.  --impl reference times the fp64 CPU oracle on the same workload (rank 0
only), a bounded sample per step, on the host cores.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "history tokens/s through STCA layer at L=10K"
UNIT = "history tokens/s"
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal (context beside the measured copy rate)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, choices=[2, 3, 4, 5], default=3,
                    help="3 (default): the 10K-history STCA step; 2: STCA M=2 Beta-ragged; "
                         "4: pointwise ReLU TA; 5: multi-sequence decode")
    ap.add_argument("--users", type=int, default=None, help="override the batch (testing only)")
    ap.add_argument("--length", type=int, default=None, help="override L (testing only)")
    ap.add_argument("--n-items", type=int, default=None, help="override the table rows (testing only)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-dedup", action="store_true", help="run the history GEMMs once per token")
    ap.add_argument("--uniform-ids", action="store_true",
                    help="control run: history ids uniform over the table instead of Zipf")
    ap.add_argument("--kv-fold", action="store_true",
                    help="fold W_K / W_V into the queries (d = 256 STCA workloads only)")
    ap.add_argument("--probe", choices=["attention", "history-backward", "train-step"], default=None,
                    help="instead of the step: time kernels alone on the workload's shapes and print one "
                         "JSON line per kernel or input form (attention: contiguous keys and the compacted "
                         "per-user key lists of the workload's ids; history-backward: every step of one "
                         "layer's history-side backward at the workload's d, h and history tokens; "
                         "train-step: the whole training step by phase)")
    ap.add_argument("--graph", action="store_true",
                    help="train-step probe: time replays of the whole step captured as one CUDA graph")
    return ap.parse_args()


def dist_info():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def rank_data_seed(workload, rank):
    """Seed of rank ``rank``'s requests: every rank serves its own users (same shapes)."""
    return 1000 + workload + 7919 * rank


def reduce_over_ranks(v, world, op="max", device="cuda"):
    """max (timings) or sum (work) of a per-rank number over all ranks (every rank gets it)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return dict(hbm_gbs=j["hbm_gbs"], bf16_tflops=j["bf16_tflops"],
                    bf16_tflops_sustained=j.get("bf16_tflops_sustained", j["bf16_tflops"]), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def workload_config(args):
    from workloads import STCA_CONFIGS
    c = dict(STCA_CONFIGS[args.workload])
    users = args.users or c["users"]
    n_items = args.n_items or c["n_items"]
    L = args.length or c.get("L", c.get("L_feed"))
    return c, users, L, n_items


def make_workload(args, data_seed):
    """The seeded workload dict for --workload (sizes overridable for small runs)."""
    from workloads import make_hyformer, make_pointwise, make_stca
    c, users, L, n_items = workload_config(args)
    over = {"id_dist": "uniform"} if getattr(args, "uniform_ids", False) else {}
    if c["kind"] == "stca":
        return make_stca(args.workload, users=users, L=L, n_items=n_items, data_seed=data_seed, **over)
    if c["kind"] == "pointwise":
        return make_pointwise(args.workload, users=users, L=L, n_items=n_items, seed=data_seed, **over)
    return make_hyformer(args.workload, users=users, L_feed=L, n_items=n_items, seed=data_seed)


def history_tokens(wl):
    if wl["cfg"]["kind"] == "hyformer":
        return int(wl["lengths"][0].sum() + wl["lengths"][1].sum())
    return int(wl["lengths"].sum())


def config_block(wl, world, total_tokens=None):
    c = wl["cfg"]
    users = len(wl["lengths"][0]) if c["kind"] == "hyformer" else len(wl["lengths"])
    n_tok = history_tokens(wl)
    common = {"users_per_gpu": users, "global_batch_users": users * world, "n_items": c["n_items"], "d": c["d"],
              "history_tokens_per_step": int(total_tokens if total_tokens is not None else n_tok * world),
              "parallelism": f"replicas x{world} (users sharded, no collective on the data path)"}
    if c["dtype"] == "bf16" and c["kind"] != "pointwise":
        common["weights"] = "random-init, converted to the tensor-core operand layout once before timing " \
                            "(stca_pin_weights, as at model load)"
    if c["kind"] == "stca":
        L = int(wl["lengths"].max())
        lengths = f"L={L}" if int(wl["lengths"].min()) == L else f"ragged L (mean {n_tok / users:.0f})"
        common.update({
            "workload": f"STCA forward, {users} users x {lengths} history items, M={c['M']} layers, d={c['d']}, "
                        f"H={c['H']}, SwiGLU hidden {c['hidden']}, {c['m']} targets/user (RLB), "
                        f"{'Zipf(%s)' % c['zipf_s'] if c['id_dist'] == 'zipf' else 'uniform'} ids over "
                        f"{c['n_items']}x{c['d']} {c['dtype']} table"
                        + (", 16-bin time feature" if c["time_buckets"] else ""),
            "history_len": L, "layers": c["M"], "heads": c["H"], "hidden": c["hidden"],
            "targets_per_user": c["m"],
            "l2": "inputs larger than L2 (table, and K/V plus hidden activations of several GB per layer)"})
    elif c["kind"] == "pointwise":
        ids = f"Zipf({c['zipf_s']})" if c["id_dist"] == "zipf" else "uniform"
        common.update({
            "workload": f"pointwise ReLU target attention with fused lookup, {users} samples x L~U[{c['L_lo']},"
                        f"{c['L']}], D={c['d']}, {ids} ids over {c['n_items']}x{c['d']} bf16 table",
            "l2": "inputs larger than L2 (0.5 GB table, 22 MB ids; Zipf ids are partly L2-resident)"})
    else:
        common.update({
            "workload": f"multi-sequence decode, {users} users x (feed L={c['L_feed']} + search "
                        f"L={c['L_search']}), {c['n_query']} queries/sequence, {c['blocks']} blocks, d={c['d']}, "
                        f"H={c['H']}, hidden {c['hidden']}, Zipf({c['zipf_s']}) ids over {c['n_items']}x{c['d']}",
            "l2": "inputs larger than L2 (2 GB table, 2.4 GB K/V per sequence pass)"})
    return common


# ------------------------------------------------------------------------------ clocks


class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU, sampled while the timed region
    runs.  NVML is read from a host thread every 5 ms (a read of the GPU's state; nothing
    is set), so even a timed region of a fraction of a second carries dozens of samples;
    where NVML is missing, nvidia-smi samples every 20 ms.  ``start`` returns once the first
    sample has landed; ``begin``/``end`` mark the timed window on the host clock (it covers
    the GPU's work: the window closes after a synchronize), and only samples inside it are
    summarised."""

    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    SMI_FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
                  "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
                  "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_uuid, period_s=0.005):
        self.uuid, self.period = gpu_uuid, period_s
        self.samples = []      # (t, sm_mhz, sm_max_mhz, power_w, set of reasons)
        self.window = None
        self.source = None
        self._stop = None
        self._thread = None
        self._proc = None
        self._path = None

    # -- NVML
    def _start_nvml(self):
        import threading
        import pynvml as nv
        nv.nvmlInit()
        h = nv.nvmlDeviceGetHandleByUUID(self.uuid)
        bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
        sm_max = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        self._stop = threading.Event()

        def loop():
            while not self._stop.is_set():
                try:
                    sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                    pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((time.monotonic(), sm, sm_max, pw, {n for n, b in bits.items() if r & b}))
                except nv.NVMLError:
                    pass
                self._stop.wait(self.period)

        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()
        self.source = f"NVML every {self.period * 1e3:.0f} ms"

    # -- nvidia-smi fallback
    def _start_smi(self):
        fd, self._path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        self._t0 = time.monotonic()
        self._proc = subprocess.Popen(
            ["nvidia-smi", "-i", self.uuid, "--query-gpu=" + ",".join(self.SMI_FIELDS),
             "--format=csv,noheader,nounits", "-lms", "20"],
            stdout=open(self._path, "w"), stderr=subprocess.DEVNULL)
        self.source = "nvidia-smi every 20 ms"

    def _smi_rows(self):
        rows = []
        with open(self._path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) == len(self.SMI_FIELDS):
                    rows.append(parts)
        return rows

    def start(self):
        try:
            self._start_nvml()
        except Exception:
            self.source = None
            try:
                self._start_smi()
            except (OSError, FileNotFoundError):
                return
        deadline = time.monotonic() + 5.0
        while time.monotonic() < deadline:
            if (self._thread is not None and self.samples) or (self._proc is not None and self._smi_rows()):
                break
            time.sleep(0.01)

    def begin(self):
        self.window = [time.monotonic(), None]

    def end(self):
        if self.window:
            self.window[1] = time.monotonic()

    def stop(self):
        if self.source is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "no NVML and no nvidia-smi"}
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)
            rows = list(self.samples)
        else:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
            raw = self._smi_rows()
            os.unlink(self._path)
            # nvidia-smi lines carry no time stamp: spread them over the sampling span
            t1 = time.monotonic()
            rows = []
            for i, r in enumerate(raw):
                num = lambda v: float(v) if v.replace(".", "", 1).isdigit() else None
                rows.append((self._t0 + (t1 - self._t0) * (i + 0.5) / max(len(raw), 1), num(r[0]), num(r[1]),
                             num(r[2]), {n for n, v in zip(self.REASONS, r[3:]) if v == "Active"}))
        if self.window and self.window[1] is not None:
            rows = [r for r in rows if self.window[0] <= r[0] <= self.window[1]]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": self.source}
        sm = [r[1] for r in rows if r[1]]
        mx = [r[2] for r in rows if r[2]]
        pw = [r[3] for r in rows if r[3]]
        counts = {n: sum(n in r[4] for r in rows) for n in self.REASONS}
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_mhz_min": min(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "power_w_max": max(pw) if pw else None,
                "samples": len(rows), "reasons": [n for n in self.REASONS if counts[n]],
                "reason_samples": {n: c for n, c in counts.items() if c}, "source": self.source}


def clocks_rejected(clk):
    bad = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}
    if bad & set(clk.get("reasons", [])):
        return True
    sm, mx = clk.get("sm_mhz"), clk.get("sm_max_mhz")
    return bool(sm and mx and sm < 0.5 * mx and not clk.get("reasons"))


# ------------------------------------------------------------------------------ roofline


def _row_keys(ids, dt):
    import numpy as np
    key = ids.astype(np.int64) * 16
    if dt is not None:
        v = dt.astype(np.int64) + 1
        key += np.minimum(15, np.floor(np.log2(v)).astype(np.int64))
    return key


def distinct_rows(ids, dt):
    """Distinct (item id, time bucket) keys among a pass's history tokens."""
    import numpy as np
    return int(len(np.unique(_row_keys(ids, dt))))


def user_distinct_rows(ids, dt, lengths):
    """Sum over users of each user's distinct keys (the keys compacted attention reads);
    a user of 16384 or more tokens keeps every token."""
    import numpy as np
    lengths = np.asarray(lengths, np.int64)
    user = np.repeat(np.arange(len(lengths), dtype=np.int64), lengths)
    long_user = np.repeat(lengths >= 16384, lengths)
    key = np.where(long_user, np.arange(len(user), dtype=np.int64), _row_keys(ids, dt))
    return int(len(np.unique(user * (1 << 40) + key)))


_PASSES = {}


def gemm_passes(wl, dedup):
    """(rows computed by the history GEMMs, history tokens, users, targets, keys attention
    reads) per pass."""
    key = (id(wl), int(dedup))
    if key not in _PASSES:
        _PASSES[key] = _gemm_passes(wl, dedup)
    return _PASSES[key]


def _gemm_passes(wl, dedup):
    c = wl["cfg"]
    if c["kind"] == "stca":
        n = int(wl["lengths"].sum())
        rows = distinct_rows(wl["ids"], wl["dt"]) if dedup else n
        keys = user_distinct_rows(wl["ids"], wl["dt"], wl["lengths"]) if dedup == 2 else n
        return [(rows, n, len(wl["lengths"]), int(wl["targets_per_user"].sum()), keys)] * c["M"]
    nq, Bu = c["n_query"], len(wl["lengths"][0])
    out = []
    for s in (0, 1):
        n = int(wl["lengths"][s].sum())
        keys = user_distinct_rows(wl["ids"][s], None, wl["lengths"][s]) if dedup == 2 else n
        out.append((distinct_rows(wl["ids"][s], None) if dedup else n, n, Bu, Bu * nq, keys))
    return out * c["blocks"]


def stage_work(stage, wl, dedup=False, fused_ffn=False, kv_fold=False):
    """Algorithmic work of one step of a stage: (bound, amount, unit).  The history GEMMs
    count the rows they compute (distinct keys when dedup is on).  With the fused FFN
    (d = 256: one kernel runs gather, SwiGLU and W2 of every layer) the gather stage also
    carries the W2 GEMM's flops."""
    c = wl["cfg"]
    d = c["d"]
    if c["kind"] == "pointwise":
        if stage == "pointwise":
            B = len(wl["lengths"])
            n_tok = history_tokens(wl)
            # each looked-up row (2D bytes) and its id read once; q read, out written
            return "hbm", n_tok * (2 * d + 4) + B * d * 2 + B * d * 4, "byte"
        return None, None, None
    h, H = c["hidden"], c["H"]
    passes = gemm_passes(wl, dedup)
    if stage == "gather_ffn":
        w2 = sum(2.0 * p[0] * h * d for p in passes) if fused_ffn else 0.0
        return "tensor", sum(2.0 * p[0] * d * 2 * h for p in passes) + w2, "flop"
    if stage == "ffn_out":
        return "tensor", sum(2.0 * p[0] * h * d for p in passes), "flop"
    if stage == "kv":
        return "tensor", sum(2.0 * p[0] * d * 2 * d for p in passes), "flop"
    if stage == "attention" and kv_fold:
        # one d-wide bf16 history row and its two LayerNorm moments per attended key, the
        # folded queries read and the weighted rows written (fp32, d per target and head)
        return "hbm", sum(keys * (2 * d + 8) + 2 * T * c["H"] * d * 4 for _, _, _, T, keys in passes), "byte"
    if stage == "attention":
        tot = 0.0
        for _, _, _, T, keys in passes:
            # one K and one V row (bf16) read per key attended (each token, or each distinct
            # key of a user when compacted), the fp32 queries read and outputs written
            # (partial states of L-slices are overhead, not counted)
            tot += keys * 2 * d * 2 + 2 * T * d * 4
        return "hbm", tot, "byte"
    return None, None, None


def traffic_from_profiles(stage, workload):
    """Per-launch DRAM bytes of a stage's kernel at this workload's full size, from the
    committed ncu summary, or None when the kernel source changed since the counters
    were taken (the summary records a digest of the source file)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    for line in open(path):
        parts = line.split()
        if len(parts) >= 3 and not line.startswith("#") and parts[0] == f"{stage}@{workload}":
            src, digest = parts[2].split(":")
            cur = hashlib.sha256(open(os.path.join(ROOT, src), "rb").read()).hexdigest()[:16]
            if cur == digest:
                return float(parts[1])
    return None


# ------------------------------------------------------------------------------ ours


def run_ours(args):
    import torch
    import torch.distributed as dist

    from target_attention_b200 import binding as B
    from target_attention_b200.device import HyformerModel, PointwiseModel, StcaModel

    rank, world, local = dist_info()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    wl = make_workload(args, data_seed=rank_data_seed(args.workload, rank))
    kind = wl["cfg"]["kind"]
    n_tok = history_tokens(wl)
    stream = torch.cuda.current_stream()
    dedup = 2 if (kind != "pointwise" and wl["cfg"]["dtype"] == "bf16" and not args.no_dedup) else 0
    if kind == "stca":
        model = StcaModel(wl, dedup=dedup, kv_fold=int(args.kv_fold))
        x = model.inputs(wl)
        out = torch.empty((x["t_tot"], wl["cfg"]["d"]), device="cuda")
    elif kind == "pointwise":
        model = PointwiseModel(wl)
        x = model.inputs(wl)
        out = torch.empty((x["B"], wl["cfg"]["d"]), device="cuda")
    else:
        model = HyformerModel(wl, dedup=dedup)
        x = model.inputs(wl)
        out = torch.empty((x["B"], 2 * x["n_query"], wl["cfg"]["d"]), device="cuda")

    if kind != "pointwise" and wl["cfg"]["dtype"] == "bf16":
        model.pin()  # weights converted to the tensor-core layout once, as at model load

    def step(handle=None):
        if handle is None:
            B.check(model.forward(x, out, stream=stream), "forward")
        else:
            B.check(model.forward(x, out, stream=stream, handle=handle), "forward")

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(v):
        return reduce_over_ranks(v, world, "max")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = B.stca_sync_status(model.handle)
    if st != B.OK:
        raise RuntimeError(f"device status {st} ({B.strerror(st)}) after warm-up")

    uuid = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)

    # Which stage dominates: one short pass with every stage bracketed by events.
    def profiled_steps(n, names=None):
        if names is None:
            B.check(B.stca_profile_enable(model.handle, True))
        else:
            B.check(B.stca_profile_stages(model.handle, names))
        for _ in range(n):
            step()
        torch.cuda.synchronize()
        prof = B.stca_profile_read(model.handle)
        B.check(B.stca_profile_enable(model.handle, False))
        return prof

    probe = profiled_steps(2)
    # the fused history FFN (d = 256) shows no separate W2 stage
    fused = kind == "stca" and wl["cfg"]["dtype"] == "bf16" and not probe.get("ffn_out", (0, 0))[1]
    work = lambda stage: stage_work(stage, wl, dedup, fused, bool(args.kv_fold))
    dom = max((s for s in probe if probe[s][1] and work(s)[0]), key=lambda s: probe[s][0])

    # The timed region: events bracket only the dominant stage (each recorded stage adds two
    # event records per call to the stream, which at small configs is a visible share).
    def timed_region():
        B.check(B.stca_profile_stages(model.handle, [dom]))
        sampler = ClockSampler(uuid)
        sampler.start()  # returns once the first sample is in
        n0 = B.stca_launch_count()
        barrier()
        torch.cuda.synchronize()
        sampler.begin()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        sampler.end()
        barrier()
        clk = sampler.stop()
        launches = B.stca_launch_count() - n0
        prof = B.stca_profile_read(model.handle)
        B.check(B.stca_profile_enable(model.handle, False))
        return e0.elapsed_time(e1), clk, launches, prof

    ms, clk, launches, prof_dom = timed_region()
    if clocks_rejected(clk):
        ms, clk, launches, prof_dom = timed_region()
        clk["remeasured"] = True
    st = B.stca_sync_status(model.handle)
    if st != B.OK:
        raise RuntimeError(f"device status {st} ({B.strerror(st)}) in the timed region")
    ms_max = max_over_ranks(ms)
    ms_step = ms_max / args.steps
    total_tokens = reduce_over_ranks(n_tok, world, "sum")  # ranks draw their own lengths
    value = total_tokens * args.steps / (ms_max / 1e3)

    # per-stage timings from a second pass of the same steps with every stage bracketed
    # (CUDA events around each stage's launches on this stream), and the roofline of the
    # dominant kernel from the timed region itself
    prof = profiled_steps(args.steps)
    ms_prof = sum(t for t, _ in prof.values())
    peaks = load_peaks()
    stages = {}
    for name, (tot, calls) in prof.items():
        if calls == 0:
            continue
        entry = {"ms_per_step": round(tot / args.steps, 4), "share": round(tot / ms_prof, 4),
                 "launches_per_step": calls // args.steps, "launch_ms": round(tot / calls, 4)}
        bound, amount, unit = work(name)
        if bound == "tensor":
            ach = amount * args.steps / (tot / 1e3) / 1e12
            entry.update(bound="tensor", achieved_tflops=round(ach, 1),
                         frac=round(ach / peaks["bf16_tflops_sustained"], 4))
        elif bound == "hbm":
            ach = amount * args.steps / (tot / 1e3) / 1e9
            entry.update(bound="hbm", achieved_gbs=round(ach, 1), frac=round(ach / peaks["hbm_gbs"], 4),
                         frac_of_nominal=round(ach / NOMINAL_HBM_GBS, 4))
        stages[name] = entry
    bound, amount, unit = work(dom)
    tot, calls = prof_dom[dom]
    per_launch = amount * args.steps / calls
    if bound == "tensor":
        achieved, peak, runit = per_launch / (tot / calls / 1e3) / 1e12, peaks["bf16_tflops_sustained"], "TFLOP/s"
    else:
        achieved, peak, runit = per_launch / (tot / calls / 1e3) / 1e9, peaks["hbm_gbs"], "GB/s"
    roofline = {"bound": bound, "kernel": dom, "achieved": round(achieved, 2), "peak": peak, "unit": runit,
                "frac": round(achieved / peak, 4),
                "traffic": traffic_from_profiles(dom + ("+dedup" if dedup else ""), args.workload),
                "work_per_launch": per_launch, "work_unit": unit, "launch_ms": round(tot / calls, 4),
                "peak_source": f"{peaks['source']} ({'sustained bf16' if bound == 'tensor' else 'HBM copy'})",
                "timing": "CUDA events around this kernel's launches inside the timed region"}
    if bound == "tensor":  # the same against the burst figure (a GEMM timed alone at full clocks)
        roofline["frac_of_burst_peak"] = round(achieved / peaks["bf16_tflops"], 4)
    else:
        roofline["frac_of_nominal"] = round(achieved / NOMINAL_HBM_GBS, 4)
        roofline["nominal_peak"] = NOMINAL_HBM_GBS
    if clk.get("sm_mhz") and clk.get("sm_max_mhz"):
        # the step time scaled to what it would be in SM cycles at the maximum clock: compares
        # runs on boxes whose power cap held the clock at different levels
        clk["ms_per_step_x_clock_over_max"] = round(ms_step * clk["sm_mhz"] / clk["sm_max_mhz"], 4)

    # the same step with the history GEMMs run per token (dedup off), for reference
    per_token = None
    if dedup:
        h0 = model.other_handle(dedup=0)
        for _ in range(args.warmup):
            step(h0)
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step(h0)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        ms0 = max_over_ranks(e0.elapsed_time(e1))
        B.stca_destroy(h0)
        passes = gemm_passes(wl, dedup)
        per_token = {"value": round(total_tokens * args.steps / (ms0 / 1e3), 1), "unit": UNIT,
                     "ms_per_step": round(ms0 / args.steps, 3),
                     "distinct_rows_fraction": round(sum(p[0] for p in passes) / sum(p[1] for p in passes), 4),
                     "attended_keys_fraction": round(sum(p[4] for p in passes) / sum(p[1] for p in passes), 4),
                     "note": "same step with the history GEMMs and the attention run once per token instead of "
                             "once per distinct (id, time bucket) key of the call (GEMMs) and of each user "
                             "(attention, weighted by token counts); the same function up to summation order"}

    # end to end through the host-buffer entry point: pinned inputs in, z out, per step
    e2e = None
    if kind == "stca" and not args.no_e2e:
        xh = {k: (v.cpu().pin_memory() if torch.is_tensor(v) else v) for k, v in x.items()}
        zh = torch.empty(tuple(out.shape), pin_memory=True)
        h2d = sum(v.numel() * v.element_size() for k, v in xh.items() if torch.is_tensor(v))
        d2h = zh.numel() * zh.element_size()
        B.check(model.forward_host(xh, zh, stream=stream))
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            B.check(model.forward_host(xh, zh, stream=stream))
        B.check(model.host_fence(stream))  # the last step's z has landed in host memory
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        ms_e2e = max_over_ranks(e0.elapsed_time(e1))
        e2e = {"value": round(total_tokens * args.steps / (ms_e2e / 1e3), 1), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": round(ms_e2e / args.steps, 3),
               "path": "stca_forward_host: pinned host inputs -> device, forward, z -> pinned host"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl)

    model.close()
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    layers = wl["cfg"].get("M", wl["cfg"].get("blocks", 1))
    cfg_line = config_block(wl, world, total_tokens)
    if args.kv_fold:
        cfg_line["kv_fold"] = "W_K / W_V folded into the queries (no K/V rows)"
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if wl["cfg"]["dtype"] == "bf16" else "f32",
        "data": "synthetic (seeded Zipf ids, random-init weights)", "config": cfg_line,
        "token_layers_per_s": round(value * layers, 1),
        "roofline": roofline, "stages": stages,
        "stages_timing": "a second pass of the same steps with every stage bracketed by CUDA events",
        "e2e": e2e, "cpu_baseline": cpu,
        "history_gemm_rows": "distinct (id, time bucket) keys per call" if dedup else "every history token",
        "attention_keys": "distinct keys per user, weighted by token count" if dedup == 2 else "every history token",
        "per_token_path": per_token,
        "gpu_launches": int(launches), "gpu_launches_per_step": round(launches / args.steps, 1), "clocks": clk,
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------ oracle


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def oracle_sample(wl, users):
    """Runs the oracle on the given users; returns the history tokens it processed."""
    from oracle import stca_ref as R
    kind = wl["cfg"]["kind"]
    if kind == "stca":
        R.stca_forward(wl, users=users)
        return int(sum(wl["lengths"][u] for u in users))
    if kind == "pointwise":
        R.pointwise_relu_ta(wl, users=users)
        return int(sum(wl["lengths"][u] for u in users))
    R.hyformer_forward(wl, users=users)
    return int(sum(wl["lengths"][0][u] + wl["lengths"][1][u] for u in users))


def sample_users(wl):
    """Users per oracle sample, sized to a few seconds of host work."""
    kind = wl["cfg"]["kind"]
    return {"stca": 1, "pointwise": 64, "hyformer": 1}[kind]


def cpu_baseline(wl):
    """The fp64 oracle, as it stands, on a bounded sample of the same workload."""
    n_users = len(wl["lengths"][0]) if wl["cfg"]["kind"] == "hyformer" else len(wl["lengths"])
    per = sample_users(wl)
    users, toks, t0 = [], 0, time.perf_counter()
    while time.perf_counter() - t0 < 10.0 and len(users) < n_users:
        batch = list(range(len(users), min(n_users, len(users) + per)))
        toks += oracle_sample(wl, batch)
        users += batch
    dt = time.perf_counter() - t0
    return {"value": round(toks / dt, 1), "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
            "sample": f"the first {len(users)} users ({toks} history tokens, all their targets) of the same "
                      f"workload, {dt:.1f} s on the host"}


def run_reference(args):
    rank, world, _ = dist_info()
    if rank != 0:
        return
    wl = make_workload(args, data_seed=rank_data_seed(args.workload, 0))
    n_users = len(wl["lengths"][0]) if wl["cfg"]["kind"] == "hyformer" else len(wl["lengths"])
    per = sample_users(wl)
    batches = [list(range(i * per % n_users, min(n_users, i * per % n_users + per)))
               for i in range(args.warmup + args.steps)]
    for b in batches[:args.warmup]:
        oracle_sample(wl, b)
    t0 = time.perf_counter()
    toks = sum(oracle_sample(wl, b) for b in batches[args.warmup:])
    dt = time.perf_counter() - t0
    value = toks / dt
    cfg = config_block(wl, 1)
    cfg.pop("weights", None)  # the oracle reads the weights as stored
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded Zipf ids, random-init weights)", "config": cfg,
        "cpu_baseline": {"value": round(value, 1), "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
                         "sample": f"{per} user(s) of the workload per step, fp64 oracle on the host"},
        "e2e": {"value": round(value, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def compacted_keys(ids, dt, lengths):
    """Each user's distinct (item id, time bucket) keys, numbered over the whole call, in
    order of first token with their token counts: the key lists the library's per-user
    compaction gives the attention.  Returns (rows, counts, per-user count, distinct keys)."""
    import numpy as np
    keys = _row_keys(ids, dt)
    uniq, inv = np.unique(keys, return_inverse=True)
    rows, mult, lens = [], [], []
    off = 0
    for L in np.asarray(lengths, np.int64):
        seg = inv[off:off + L]
        off += L
        vals, first, cnt = np.unique(seg, return_index=True, return_counts=True)
        order = np.argsort(first)
        rows.append(vals[order]), mult.append(cnt[order]), lens.append(len(vals))
    cat = lambda xs: np.concatenate(xs).astype(np.int32) if xs else np.zeros(0, np.int32)
    return cat(rows), cat(mult), np.asarray(lens, np.int32), len(uniq)


def run_probe_attention(args):
    """The split-L attention kernel alone on config 3's shapes (d = 512, H = 8, m = 32):
    one layer's keys, K/V and queries random (the kernel's time does not depend on their
    values beyond the rare rescales), timed with CUDA events around each launch after
    warm-up; the median of 3 x steps launches.  "contiguous": every user's keys are its own
    consecutive K/V rows; "compacted": the per-user distinct keys of the workload's ids,
    gathered by row from the call's distinct-key K/V matrix and weighted by their counts.
    "backward": the training backward (stca_attention_backward, bf16 K/V gradients) over the
    contiguous keys, from the training forward's output and log-sum-exp; its bytes are the
    K/V read and the K/V gradients written (8 d per key) plus the query-side rows."""
    import statistics
    import numpy as np
    import torch
    from target_attention_b200 import binding as B
    from workloads import STCA_CONFIGS, make_stca_history
    c = STCA_CONFIGS[3]
    over = {"id_dist": "uniform"} if args.uniform_ids else {}
    hist = make_stca_history(3, users=args.users, L=args.length, n_items=args.n_items, data_seed=rank_data_seed(3, 0),
                             **over)
    d, H, m = c["d"], c["H"], c["m"]
    lengths = hist["lengths"]
    Bu = len(lengths)
    rows, mult, lens, U = compacted_keys(hist["ids"], hist["dt"], lengths)
    hoff = np.zeros(Bu + 1, np.int64)
    hoff[1:] = np.cumsum(lengths)
    # the compacted lists sit at each user's token offset, as the library lays them out
    slot_rows = np.zeros(int(hoff[-1]), np.int32)
    slot_mult = np.ones(int(hoff[-1]), np.int32)
    o = 0
    for u in range(Bu):
        slot_rows[hoff[u]:hoff[u] + lens[u]] = rows[o:o + lens[u]]
        slot_mult[hoff[u]:hoff[u] + lens[u]] = mult[o:o + lens[u]]
        o += lens[u]
    n_att = int(lens.sum())
    T = Bu * m
    dev = "cuda"
    g = torch.Generator(device=dev)
    g.manual_seed(5)
    i32 = lambda x: torch.from_numpy(np.ascontiguousarray(x, np.int32)).to(dev)
    KVu = (torch.randn((U, 2 * d), device=dev, generator=g) * 0.5).to(torch.bfloat16)
    KVc = (torch.randn((n_att, 2 * d), device=dev, generator=g) * 0.5).to(torch.bfloat16)
    Q = torch.randn((T, d), device=dev, generator=g)
    hoff_t, toff_t = i32(hoff), i32(np.arange(0, T + 1, m))
    hoff_c = i32(np.concatenate([[0], np.cumsum(lens)]))
    rows_t, mult_t, lens_t = i32(slot_rows), i32(slot_mult), i32(lens)
    pa = torch.empty((1, T, d), device=dev)
    pm = torch.empty((1, T, H, 2), device=dev)
    out = torch.empty((T, d), device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    # the training backward over the contiguous keys: the forward's output and lse first
    out_t = torch.empty((T, d), device=dev)
    lse_t = torch.empty((T, H), device=dev)
    B.check(B.stca_attention_train_forward(Q, KVc, hoff_c, toff_t, Bu, T, d, H, 1, 0, pa, pm, out_t, lse_t, err))
    dO = torch.randn((T, d), device=dev, generator=g)
    dQ = torch.empty((T, d), device=dev)
    dKV = torch.empty((n_att, 2 * d), device=dev)
    dKV16 = torch.empty((n_att, 2 * d), dtype=torch.bfloat16, device=dev)
    modes = {
        "contiguous": lambda: B.stca_k_attention(1, Q, KVc, hoff_c, toff_t, Bu, T, d, H, 1, 0, pa, pm, out, err),
        "compacted": lambda: B.stca_k_attention_rows(1, Q, KVu, hoff_t, toff_t, rows_t, lens_t, mult_t, Bu, T, d, H,
                                                     1, 0, pa, pm, out, err),
        "backward": lambda: B.stca_attention_backward(Q, KVc, hoff_c, toff_t, Bu, T, d, H, 1, 0, out_t, lse_t, dO, dQ,
                                                      dKV, None, dKV16=dKV16),
    }
    peaks = load_peaks()
    times = {k: [] for k in modes}
    for _ in range(3):
        for k, f in modes.items():
            for _ in range(max(args.warmup, 1)):
                B.check(f())
            torch.cuda.synchronize()
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
            for e0, e1 in ev:
                e0.record()
                B.check(f())
                e1.record()
            torch.cuda.synchronize()
            times[k] += [e0.elapsed_time(e1) for e0, e1 in ev]
    assert int(err.item()) == 0
    work = n_att * H * 4 * (d // H) + 2 * T * d * 4  # attended K/V segments + queries and outputs
    # backward: K/V read and their gradients written (bf16), Q, O, dO read and dQ written
    work_bwd = n_att * 8 * d + 4 * T * d * 4
    for k in modes:
        ms = statistics.median(times[k])
        w_k = work_bwd if k == "backward" else work
        gbs = w_k / ms / 1e6
        print(json.dumps({"probe": "attention", "mode": k, "users": Bu, "attended_keys": n_att,
                          "distinct_keys": int(U), "ids": "uniform" if args.uniform_ids else "zipf",
                          "median_ms": round(ms, 4), "launches": len(times[k]), "work_bytes": w_k,
                          "achieved_gbs": round(gbs, 1), "peak_gbs": peaks["hbm_gbs"],
                          "frac": round(gbs / peaks["hbm_gbs"], 4)}), flush=True)


def run_probe_history_backward(args):
    """One layer's history-side backward (target_attention_b200.training) on the workload's
    shapes (--workload 2 or 3; every history token, no distinct-key compaction): the forward
    recompute and the backward, each step bracketed by CUDA events, median over 3 x steps
    runs after warm-up.  GEMMs are charged 2 M K N flop against the measured sustained bf16
    rate; the LayerNorm / SwiGLU backward and the lookup scatter their bytes against the
    measured HBM rate."""
    import statistics
    import numpy as np
    import torch
    from target_attention_b200.training import HistoryLayerBackward
    wl = make_workload(args, data_seed=rank_data_seed(args.workload, 0))
    assert wl["cfg"]["kind"] == "stca", "history-backward probes an STCA workload (2 or 3)"
    cfg, w = wl["cfg"], wl["weights"]
    d, h = cfg["d"], cfg["hidden"]
    ids, dt = wl["ids"], wl["dt"]
    M, n_items = len(ids), int(wl["table"].shape[0])
    dev = "cuda"
    up16 = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).to(dev)
    f32 = lambda a: torch.from_numpy(np.asarray(a, np.float32)).to(dev)
    ffn = w["hist"][0]  # LayerNorm parameters are stored as float32
    layer = HistoryLayerBackward(M, d, h, up16(ffn["W1"]), up16(ffn["W3"]), up16(ffn["W2"]), up16(w["WK"][0]),
                                 up16(w["WV"][0]), f32(ffn["gamma"]), f32(ffn["beta"]))
    ids_t = torch.from_numpy(ids.astype(np.int32)).to(dev)
    dt_t = torch.from_numpy(dt.astype(np.int32)).to(dev) if dt is not None else None
    table = up16(wl["table"])
    dtab = up16(wl["dt_table"]) if dt is not None else None
    g = torch.Generator(device=dev)
    g.manual_seed(3)
    dKV = torch.randn((M, 2 * d), device=dev, generator=g).to(torch.bfloat16)
    dtable = torch.zeros((n_items, d), device=dev)
    ddt = torch.zeros((16, d), device=dev) if dt is not None else None

    times = {}
    def run(record):
        marks = []
        on_step = (lambda name: (marks.append((name, torch.cuda.Event(enable_timing=True))), marks[-1][1].record())) \
            if record else None
        start = torch.cuda.Event(enable_timing=True)
        start.record()
        layer.recompute(ids_t, dt_t, table, dtab, n_items, on_step=on_step)
        layer.backward(dKV, ids_t, dt_t, n_items, dtable, ddt, on_step=on_step)
        return start, marks

    for _ in range(max(args.warmup, 1)):
        run(False)
    torch.cuda.synchronize()
    for _ in range(3 * args.steps):
        start, marks = run(True)
        torch.cuda.synchronize()
        prev = start
        for name, ev in marks:
            times.setdefault(name, []).append(prev.elapsed_time(ev))
            prev = ev
        times.setdefault("layer", []).append(start.elapsed_time(marks[-1][1]))
    assert int(layer.err.item()) == 0
    peaks = load_peaks()
    flops = layer.flops()
    bytes_ = {"LN backward": M * d * 2 * 4, "SwiGLU backward": M * h * 2 * 5, "table rows": M * d * (2 + 2 * 4)}
    total_flop = sum(flops.values())
    for name, ts in times.items():
        ms = statistics.median(ts)
        line = {"probe": "history-backward", "step": name, "workload": args.workload, "history_tokens": M, "d": d,
                "hidden": h, "median_ms": round(ms, 4), "runs": len(ts)}
        if name in flops or name == "layer":
            f = total_flop if name == "layer" else flops[name]
            tf = f / ms / 1e9
            line.update(flop=f, achieved_tflops=round(tf, 1), peak_tflops=peaks["bf16_tflops_sustained"],
                        frac=round(tf / peaks["bf16_tflops_sustained"], 4))
        elif name in bytes_:
            gbs = bytes_[name] / ms / 1e6
            line.update(bytes=bytes_[name], achieved_gbs=round(gbs, 1), peak_gbs=peaks["hbm_gbs"],
                        frac=round(gbs / peaks["hbm_gbs"], 4))
        print(json.dumps(line), flush=True)


def run_probe_train_step(args):
    """The whole training step (target_attention_b200.training.StcaTrainingStep: every
    layer's history side recomputed, the target side, then the backward into every weight,
    the table rows and x_t) on the workload's batch (--workload 2 or 3), three phases
    bracketed by CUDA events, median over 3 x steps runs after warm-up.  The flop rate
    counts the history GEMMs and the attention products against the measured sustained
    bf16 rate."""
    import statistics
    import numpy as np
    import torch
    from target_attention_b200 import binding as B
    from target_attention_b200.training import StcaTrainingStep, device_weights
    wl = make_workload(args, data_seed=rank_data_seed(args.workload, 0))
    assert wl["cfg"]["kind"] == "stca", "train-step probes an STCA workload (2 or 3)"
    cfg = wl["cfg"]
    d = cfg["d"]
    dev = "cuda"
    lengths, tpu = wl["lengths"], wl["targets_per_user"]
    Bu, N, T = len(lengths), int(lengths.sum()), int(tpu.sum())
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.int32)).to(dev)
    up16 = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    hoff = torch.empty(Bu + 1, dtype=torch.int32, device=dev)
    toff = torch.empty(Bu + 1, dtype=torch.int32, device=dev)
    B.check(B.stca_k_offsets(i32(lengths), Bu, hoff, N, err))
    B.check(B.stca_k_offsets(i32(tpu), Bu, toff, T, err))
    step = StcaTrainingStep(cfg, device_weights(wl["weights"]), Bu, N, T)
    step.x_t_slot().copy_(up16(wl["x_t"]).float())
    ids = i32(wl["ids"])
    dt = i32(wl["dt"]) if wl["dt"] is not None else None
    table = up16(wl["table"])
    dt_table = up16(wl["dt_table"]) if wl["dt"] is not None else None
    n_items = int(wl["table"].shape[0])
    g = torch.Generator(device=dev)
    g.manual_seed(3)
    dZ = torch.randn((T, d), device=dev, generator=g)
    dtable = torch.zeros((n_items, d), device=dev)
    ddt = torch.zeros((16, d), device=dev) if dt is not None else None

    def once():
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        ev[0].record()
        step.forward_history(ids, dt, table, dt_table, n_items)
        ev[1].record()
        step.forward_target(hoff, toff)
        ev[2].record()
        step.backward(ids, dt, hoff, toff, n_items, dZ, dtable, ddt)
        ev[3].record()
        return ev

    for _ in range(max(args.warmup, 1)):
        once()
    torch.cuda.synchronize()
    times = {k: [] for k in ("history forward", "target forward", "backward", "step")}
    if args.graph:  # the whole step as one CUDA graph: only the step's time
        graph, _ = step.capture(ids, dt, hoff, toff, table, dt_table, n_items, dZ, dtable, ddt)
        times = {"step (graph)": []}
        for _ in range(max(args.warmup, 1)):
            graph.replay()
        torch.cuda.synchronize()
        for _ in range(3 * args.steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            graph.replay()
            e1.record()
            torch.cuda.synchronize()
            times["step (graph)"].append(e0.elapsed_time(e1))
    for _ in range(0 if args.graph else 3 * args.steps):
        ev = once()
        torch.cuda.synchronize()
        for k, (a, b) in zip(times, ((0, 1), (1, 2), (2, 3), (0, 3))):
            times[k].append(ev[a].elapsed_time(ev[b]))
    assert int(err.item()) == 0 and int(step.err.item()) == 0
    flops = step.flops(lengths, tpu)
    peak = load_peaks()["bf16_tflops_sustained"]
    for name, ts in times.items():
        ms = statistics.median(ts)
        line = {"probe": "train-step", "phase": name, "workload": args.workload, "users": Bu, "history_tokens": N,
                "targets": T, "d": d, "layers": cfg["M"], "score": cfg["score"], "median_ms": round(ms, 4),
                "runs": len(ts)}
        if name.startswith("step"):
            f = sum(flops.values())
            tf = f / ms / 1e9
            line.update(flop=f, flop_attention=flops["attention"], achieved_tflops=round(tf, 1), peak_tflops=peak,
                        frac=round(tf / peak, 4), history_tokens_per_s=round(N / ms * 1e3),
                        targets_per_s=round(T / ms * 1e3))
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    a = parse()
    if a.probe == "attention":
        run_probe_attention(a)
    elif a.probe == "history-backward":
        run_probe_history_backward(a)
    elif a.probe == "train-step":
        run_probe_train_step(a)
    elif a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)
