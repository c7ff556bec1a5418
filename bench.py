"""Benchmark of the chunked causal linear-attention prefill on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one whole prefill (K1 -> K2 -> K3) of the workload through the C ABI.  The
default workload is the 128K-token retention prefill (B1 H32 T131072 d128 C64, bf16
inputs, identity feature map, per-head decay, unnormalised).  With N GPUs (torchrun,
one rank per GPU) every rank runs its own independent copy (weak scaling); the value is
the tokens*heads of all ranks over the slowest rank's device time.  Rank 0 prints one
JSON line.

Extra fields: per-kernel device times from an event-instrumented pass, the roofline of
the dominant kernel against the measured HBM bandwidth, the end-to-end rate through the
host-buffer entry point, the oracle's rate on the host cores, and the SM clocks sampled
during the timed region.

`--impl reference` times the fp64 CPU oracle (the only reference implementation there
is) on a bounded sample of the same workload.
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
from pathlib import Path

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import numpy as np  # noqa: E402
import torch  # noqa: E402

from chunked_causal_linear_b200 import binding as B  # noqa: E402
from chunked_causal_linear_b200 import ranks  # noqa: E402
from chunked_causal_linear_b200.workloads import WORKLOADS, make_inputs  # noqa: E402

METRIC = "causal linear-attn prefill tokens·heads/s at H=32,d=128; % of roofline"
METRIC_BWD = "causal linear-attn backward tokens·heads/s at H=32,d=128; % of roofline"
UNIT = "tokens*heads/s"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0
BAD_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")

K2_NAMES = {"logdepth": ["k2_reduce", "k2_block_scan", "k2_downsweep"],
            "sequential": ["k2_sequential"]}
SCAN_BLOCK_ELEMS = 2048  # the log-depth scan's one-level limit (lin_attn_scan_plan)
SCAN_WARP_ELEMS = 32     # up to this many elements the block level runs as k2_warp_scan
KERNEL_SOURCES = {"k1_tc": "tc_kernels.cu", "k3_tc": "tc_kernels.cu", "k1_fma": "fma_kernels.cu",
                  "k3_fma": "fma_kernels.cu", "k2_reduce": "scan.cu",
                  "k2_block_scan": "scan.cu", "k2_warp_scan": "scan.cu", "k2_downsweep": "scan.cu",
                  "k2_sequential": "scan.cu", "k1_seg": "seg_kernels.cu",
                  "k3_seg": "seg_kernels.cu"}


def kernel_path_for(w) -> str:
    """The kernels a workload runs on: the tensor cores for bf16 inputs, the CUDA-core FMA
    kernels for float32 inputs (the small float32 workload)."""
    return "fma" if w.dtype == "f32" else "tensor_core"


def effective_algorithm(w, requested: str) -> str:
    """The algorithm the library runs for this workload (the FMA kernels are chunked)."""
    if kernel_path_for(w) == "fma":
        return "chunked"
    seg_ok = (w.dtype == "bf16" and w.C == 64 and w.dk in (64, 128) and w.dv in (64, 128)
              and not (w.feature_map == "elu1" and w.decay))
    if requested == "segmented" or (requested == "auto" and seg_ok):
        return "segmented"
    return "chunked"


def kernel_names(w, algo: str, scan: str, lseg: int = 0) -> list[str]:
    k1, k3 = ("k1_seg", "k3_seg") if algo == "segmented" else ("k1_tc", "k3_tc")
    if kernel_path_for(w) == "fma":
        k1, k3 = "k1_fma", "k3_fma"
    n, G, _ = layout(w, algo, lseg)
    k2 = ["k2_block_scan"] if scan == "logdepth" and n <= SCAN_BLOCK_ELEMS else list(K2_NAMES[scan])
    if scan == "logdepth":
        # The block level over at most 32 elements (n one level, G two) is the warp scan.
        m = n if n <= SCAN_BLOCK_ELEMS else G
        if m <= SCAN_WARP_ELEMS:
            k2 = ["k2_warp_scan" if x == "k2_block_scan" else x for x in k2]
    return [k1, *k2, k3]


# ---------------------------------------------------------------------------------------
# Algorithmic bytes


def segment_length(w, lseg: int = 0) -> int:
    """Chunks per segment of the segmented algorithm: the requested count, else the
    library's automatic choice (about four segments per SM, at most 64 chunks, unless the
    model waves x (4 + chunks per segment) predicts at least 25 % less time for a longer
    segment)."""
    NC = -(-w.T // w.C)
    if lseg > 0:
        return min(lseg, NC)
    BH = w.B * w.H
    cap = min(64, max(1, NC))
    l0 = max(1, min(cap, (BH * NC) // (4 * 148)))

    def cost(l):
        return -(-BH * -(-NC // l) // 148) * (4.0 + l)

    best = min(range(1, cap + 1), key=lambda l: (cost(l), l != l0, l))
    return best if cost(best) <= 0.75 * cost(l0) else l0


def layout(w, algo: str = "chunked", lseg: int = 0):
    """(scan elements per (b, h), scan segments G, floats per record) as the library lays
    them out: chunks for the chunked algorithm, segments of chunks for the segmented one."""
    NC = -(-w.T // w.C)
    n = NC
    if algo == "segmented":
        n = -(-NC // segment_length(w, lseg))
    Ls = max(16, -(-n // SCAN_BLOCK_ELEMS)) if n > SCAN_BLOCK_ELEMS else n
    G = -(-n // Ls)
    R = w.dk * w.dv + (w.dk if w.normalize else 0)
    return n, G, R


def kernel_bytes(w, name: str, out_elem: int, algo: str = "chunked", lseg: int = 0) -> int:
    """Bytes each kernel must move for its own role (one launch)."""
    BH = w.B * w.H
    n, G, R = layout(w, algo, lseg)
    e_in = 2 if w.dtype == "bf16" else 4
    rec = BH * n * R * 4
    if name.startswith("k1"):
        return BH * w.T * (w.dk + w.dv) * e_in + rec
    if name == "k2_reduce":
        return rec + BH * G * R * 4
    if name in ("k2_block_scan", "k2_warp_scan"):
        # One level: the records read once (the second read of a CTA's slab comes from L2)
        # and written once; two levels: the same over the segment folds.  Plus the final
        # states.
        return 2 * (rec if n <= SCAN_BLOCK_ELEMS else BH * G * R * 4) + BH * R * 4
    if name == "k2_downsweep":
        return 2 * rec + BH * G * R * 4
    if name == "k2_sequential":
        return 2 * rec + BH * R * 4
    if name in ("k3_tc", "k3_fma"):
        return BH * w.T * (2 * w.dk + w.dv) * e_in + BH * (n - 1) * R * 4 + BH * w.T * w.dv * out_elem
    if name == "k3_seg":
        return BH * w.T * (2 * w.dk + w.dv) * e_in + rec + BH * w.T * w.dv * out_elem
    raise KeyError(name)


def algo_bytes(w, out_elem: int, algo: str, lseg: int = 0) -> int:
    """Whole-step algorithmic bytes of an algorithm: its input reads (the segmented one
    reads k and v in K1 and again in K3), the output, the final states, and four passes of
    its records (K1 write, K2 read and write, K3 read)."""
    BH = w.B * w.H
    n, G, R = layout(w, algo, lseg)
    e_in = 2 if w.dtype == "bf16" else 4
    kv_again = BH * w.T * (w.dk + w.dv) * e_in if algo == "segmented" else 0
    return (BH * w.T * (2 * w.dk + w.dv) * e_in + kv_again + BH * w.T * w.dv * out_elem
            + BH * R * 4 + 4 * BH * n * R * 4)


def min_bytes(w, out_elem: int) -> int:
    """Bytes any exact method must move: q, k, v read once, output and final states written."""
    BH = w.B * w.H
    e_in = 2 if w.dtype == "bf16" else 4
    return (BH * w.T * (2 * w.dk + w.dv) * e_in + BH * w.T * w.dv * out_elem
            + BH * (w.dk * w.dv + (w.dk if w.normalize else 0)) * 4)


def method_bytes(w, out_elem: int) -> int:
    """Whole-step algorithmic bytes of the three-kernel method: inputs read once, output
    written once, final states written once, and four passes of the chunk records (K1
    write, K2 read and write, K3 read)."""
    BH = w.B * w.H
    NC, G, R = layout(w)
    e_in = 2 if w.dtype == "bf16" else 4
    return (BH * w.T * (2 * w.dk + w.dv) * e_in + BH * w.T * w.dv * out_elem
            + BH * (w.dk * w.dv + (w.dk if w.normalize else 0)) * 4 + 4 * BH * NC * R * 4)


def measured_peaks() -> tuple[float, str]:
    p = ROOT / "MEASURED_PEAKS.json"
    try:
        d = json.loads(p.read_text())
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def copy_bound_ms(h2d_pairs, d2h_pairs, reps=2):
    """Device time of the end-to-end step's copies alone: every (device, pinned host) pair of
    h2d_pairs copied in on one stream while every (pinned host, device) pair of d2h_pairs is
    copied out on another, from one event to the join of both (best of reps, after one
    warm-up).  The host-buffer prefill cannot finish faster than this."""
    dev = h2d_pairs[0][0].device
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    cur = torch.cuda.current_stream(dev)
    best = float("inf")
    for r in range(reps + 1):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(cur)
        for st, pairs in ((s_in, h2d_pairs), (s_out, d2h_pairs)):
            st.wait_event(e0)
            with torch.cuda.stream(st):
                for dst, src in pairs:
                    dst.copy_(src, non_blocking=True)
            cur.wait_stream(st)
        e1.record(cur)
        torch.cuda.synchronize(dev)
        if r > 0:
            best = min(best, e0.elapsed_time(e1))
    return best


def source_hash(fname: str) -> str:
    csrc = ROOT / "chunked_causal_linear_b200" / "csrc"
    h = hashlib.sha256()
    for f in sorted({fname, "ptx.cuh", "common.cuh", "tile_util.cuh"}):
        h.update((csrc / f).read_bytes())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if the kernel's source is the
    one those counters were taken on; otherwise None."""
    f = ROOT / "profiles" / "traffic.txt"
    if not f.exists():
        return None
    want = source_hash(KERNEL_SOURCES.get(kernel, "tc_kernels.cu"))
    for line in f.read_text().splitlines():
        parts = line.split()
        if len(parts) >= 4 and not line.startswith("#") and parts[0] == kernel \
                and parts[1] == workload and parts[2] == want:
            return int(float(parts[3]))
    return None


# ---------------------------------------------------------------------------------------
# Clocks


class ClockSampler:
    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int, interval_ms: int = 100):
        self.uuid = None
        try:
            self.uuid = str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            pass
        self.interval_ms = interval_ms
        self.proc = None
        self.tmp = None

    def start(self):
        try:
            self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(self.interval_ms)], stdout=self.tmp, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.tmp.flush()
        rows = []
        for line in Path(self.tmp.name).read_text().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            if self.uuid and self.uuid.replace("GPU-", "") not in parts[0]:
                continue
            rows.append(parts)
        os.unlink(self.tmp.name)
        if not rows:
            return None

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        pw = [num(r[3]) for r in rows if num(r[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None,
                "samples": len(rows), "reasons": reasons}


def clocks_bad(c) -> bool:
    if not c:
        return False
    if any(r in c["reasons"] for r in BAD_REASONS):
        return True
    return bool(c["sm_mhz"] and c["sm_max_mhz"] and c["sm_mhz"] < 0.6 * c["sm_max_mhz"]
                and not c["reasons"])


# ---------------------------------------------------------------------------------------
# CPU side (oracle): the reported baseline and the reference arm


class OracleTimer:
    """Times the oracle on the first T' tokens of every (b, h) of the workload `w`, T' sized
    for about `target_s` seconds of host work.  q, k, v may hold fewer tokens than the
    workload (a sample drawn with its recipe); T' never exceeds what they hold."""

    def __init__(self, w, q, k, v, target_s: float):
        from oracle.oracle import default_oracle
        self.orc = default_oracle()
        self.w = w
        self.avail = int(q.shape[2])
        self.threads = max(1, min(len(os.sched_getaffinity(0)), w.B * w.H))
        probe_t = min(self.avail, 512)
        self.inputs = (q, k, v)
        dt = self._run(probe_t)
        self.tp = min(self.avail, max(probe_t, int(probe_t * target_s / max(dt, 1e-6))))
        self.host = [t[:, :, :self.tp].to("cpu", torch.float32).numpy() for t in (q, k, v)]
        self.last_s = dt

    def _run(self, tp, host=None):
        w = self.w
        qs, ks, vs = host if host is not None else (
            t[:, :, :tp].to("cpu", torch.float32).numpy() for t in self.inputs)
        t0 = time.perf_counter()
        self.orc.forward(qs, ks, vs, feature_map=w.feature_map, gamma=w.gammas(),
                         normalize=w.normalize, nthreads=self.threads)
        return time.perf_counter() - t0

    def rate(self):
        dt = self._run(self.tp, self.host)
        self.last_s = dt
        return self.w.B * self.w.H * self.tp / dt

    @property
    def sample_tokens_heads(self) -> int:
        return self.w.B * self.w.H * self.tp

    def sample(self):
        return (f"first {self.tp} of {self.w.T} tokens of all {self.w.B * self.w.H} (b,h) "
                f"pairs, full fp64 token loop, {self.last_s:.2f} s per run on "
                f"{self.threads} threads")


def reference_arm(args, w, info):
    """The oracle as the reference arm: every step is one oracle run over a bounded sample
    of the workload (its first T' tokens of every (b, h)), sized so that warm-up plus timed
    steps take about --reference-total-s seconds.  `value` is the sample's tokens*heads
    over its measured time (the token loop's cost is the same for every token), and
    `ms_per_step` is the measured time of one sample step; the time a whole-workload step
    would take at that rate is reported beside it, labelled as extrapolated."""
    if not info.is_root:
        return
    n_runs = args.warmup + args.steps
    per_step_s = max(0.05, min(args.reference_step_s, args.reference_total_s / n_runs))
    # The oracle's cost per token does not depend on the values; draw the sample's inputs
    # on the CPU with the workload's recipe, never more tokens than a step can use.
    probe = w.with_(T=min(w.T, 1 << 15))
    q, k, v = make_inputs(probe, seed=0, device="cpu")
    timer = OracleTimer(w, q, k, v, target_s=per_step_s)
    per_step, secs = [], []
    for i in range(n_runs):
        r = timer.rate()
        if i >= args.warmup:
            per_step.append(r)
            secs.append(timer.last_s)
    value = statistics.median(per_step)
    step_s = statistics.median(secs)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": info.world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * step_s,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(w, args),
        "sample": {"tokens_heads_per_step": timer.sample_tokens_heads, "tokens": timer.tp,
                   "of_tokens": w.T, "seconds_per_step": step_s,
                   "extrapolated": timer.tp < w.T,
                   "extrapolated_full_workload_ms": 1000.0 * w.tokens_heads / value},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": timer.threads, "kind": "oracle",
                         "sample": timer.sample()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def sweep_scan(args, dev):
    """K2 device time, log-depth scan vs sequential carry, on the chunked algorithm (every
    chunk is a scan element): B1 H8 d64 C64 with 256 .. 16384 chunks, then the two
    long-sequence workloads at full size."""
    cases = [WORKLOADS["scan_depth_1m"].with_(T=nc * 64, name=f"b1h8d64_nc{nc}")
             for nc in (256, 512, 1024, 2048, 4096, 8192, 16384)]
    cases += [WORKLOADS["retention_128k"], WORKLOADS["scan_depth_1m"]]
    for w in cases:
        q, k, v = make_inputs(w, seed=0, device=dev)
        ws = torch.empty(B.lin_attn_prefill_workspace_bytes(w.B, w.H, w.T, w.dk, w.dv, w.C,
                                                            w.normalize),
                         dtype=torch.uint8, device=dev)
        out = torch.empty((w.B, w.H, w.T, w.dv), dtype=torch.float32, device=dev)
        nc = -(-w.T // w.C)
        row = {"sweep": "k2_scan", "workload": w.name, "chunks": nc,
               "columns": w.B * w.H * (w.dk * w.dv + (w.dk if w.normalize else 0)),
               "depth_logdepth": B.lin_attn_scan_plan(nc)["depth"],
               "depth_sequential": nc, "ceil_log2_chunks": math.ceil(math.log2(nc))}
        for scan in ("logdepth", "sequential"):
            kw = dict(chunk=w.C, feature_map=w.feature_map, gamma=w.gammas(),
                      normalize=w.normalize, scan=scan, kernel_path="tensor_core",
                      workspace=ws, out_dtype="f32", algorithm="chunked")
            for _ in range(3):
                B.lin_attn_prefill_timed(q, k, v, out, **kw)
            t = [B.lin_attn_prefill_timed(q, k, v, out, **kw) for _ in range(5)]
            k2 = [sum(x[1:-1]) for x in t]
            row[f"k2_ms_{scan}"] = statistics.median(k2)
        row["logdepth_speedup"] = row["k2_ms_sequential"] / row["k2_ms_logdepth"]
        print(json.dumps(row), flush=True)
        del q, k, v, ws, out


def seq_shard_bench(args, w, info, dev):
    """One sequence of the workload split across the ranks (seqshard.prefill_sequence_sharded):
    every rank holds one contiguous token range.  Timed like the main benchmark (device
    events, barriers, max over ranks); the phases of one step are timed separately."""
    from chunked_causal_linear_b200.seqshard import part_ranges, prefill_sequence_sharded
    rng = part_ranges(w.T, info.world, w.C)
    toks = [n for _, n in rng]
    s0, n = rng[info.rank]
    wr = w.with_(T=max(n, 1), name=f"{w.name}_part{info.rank}")
    q, k, v = make_inputs(wr, seed=info.rank, device=dev)
    out = torch.empty((w.B, w.H, wr.T, w.dv), dtype=torch.float32, device=dev)
    ws = torch.empty(B.lin_attn_prefill_workspace_bytes(w.B, w.H, wr.T, w.dk, w.dv, w.C,
                                                        w.normalize), dtype=torch.uint8, device=dev)
    gam = w.gammas()
    algo = effective_algorithm(wr, args.algorithm)
    kw = dict(chunk=w.C, feature_map=w.feature_map, scan=args.scan, kernel_path="tensor_core",
              workspace=ws, out_dtype="f32", algorithm=algo, segment_chunks=args.segment_chunks)

    def step():
        return prefill_sequence_sharded(q, k, v, out, info=info, part_tokens=toks, gamma=gam,
                                        normalize=w.normalize, **kw)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ranks.barrier(info)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    ranks.barrier(info)
    ms_max = ranks.max_over_ranks(e0.elapsed_time(e1) / args.steps, info, dev)

    # Phases of one step, each timed on its own.
    def timed(fn, reps=5):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        fn()
        torch.cuda.synchronize()
        a.record()
        for _ in range(reps):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps
    _, S_loc, Z_loc = B.lin_attn_prefill(q, k, v, None, gamma=gam, normalize=w.normalize,
                                         states_only=True, **kw)
    from chunked_causal_linear_b200.seqshard import _gather
    S_parts = _gather(S_loc, info)
    Z_parts = _gather(Z_loc, info) if w.normalize else None
    S_in, Z_in = B.lin_attn_combine_states(S_parts, Z_parts, info.rank, toks, gamma=gam)
    phases = {
        "states_pass": timed(lambda: B.lin_attn_prefill(q, k, v, None, gamma=gam,
                                                        normalize=w.normalize, states_only=True,
                                                        **kw)),
        "all_gather": timed(lambda: _gather(S_loc, info)),
        "combine": timed(lambda: B.lin_attn_combine_states(S_parts, Z_parts, info.rank, toks,
                                                           gamma=gam)),
        "prefill": timed(lambda: B.lin_attn_prefill(q, k, v, out, gamma=gam,
                                                    normalize=w.normalize, S_init=S_in,
                                                    Z_init=Z_in, **kw)),
    }
    phases = {key: ranks.max_over_ranks(val, info, dev) for key, val in phases.items()}
    err = B.lin_attn_device_error()
    if info.is_root:
        cfg = config_of(w, args)
        cfg["parallelism"] = (f"sequence-sharded over {info.world} rank(s): ranges of "
                              f"{toks} tokens, all_gather of B*H*(dk*dv+dk) floats per rank")
        e_in = 2
        extra = w.B * w.H * w.T * (w.dk + w.dv) * e_in  # the states pass reads k, v again
        peak, _ = measured_peaks()
        ab = algo_bytes(w, 4, algo, args.segment_chunks) + extra
        line = {
            "metric": METRIC, "value": w.tokens_heads / (ms_max / 1000.0), "unit": UNIT,
            "n_gpus": info.world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_max, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
            "mode": "seq_shard", "phases_ms": phases,
            "step_roofline": {"bytes": ab, "achieved_gbs": ab / (ms_max / 1000.0) / 1e9 / info.world,
                              "frac_of_measured": ab / (ms_max / 1000.0) / 1e9 / info.world / peak,
                              "note": "per GPU; the bytes include the states pass's second read "
                                      "of k and v"},
            "device_error": err,
        }
        print(json.dumps(line), flush=True)


class BackwardOracleTimer(OracleTimer):
    """OracleTimer for the oracle's backward (gradients of the unnormalised form)."""

    def __init__(self, w, q, k, v, do, target_s: float):
        self.do = do
        super().__init__(w, q, k, v, target_s)
        self.host_do = do[:, :, :self.tp].to("cpu", torch.float64).numpy()

    def _run(self, tp, host=None):
        w = self.w
        qs, ks, vs = host if host is not None else (
            t[:, :, :tp].to("cpu", torch.float32).numpy() for t in self.inputs)
        dos = self.host_do if host is not None else self.do[:, :, :tp].to("cpu", torch.float64).numpy()
        t0 = time.perf_counter()
        self.orc.backward(qs, ks, vs, dos, feature_map=w.feature_map, gamma=w.gammas(),
                          normalize=w.normalize,
                          nthreads=self.threads)
        return time.perf_counter() - t0

    def sample(self):
        return (f"first {self.tp} of {self.w.T} tokens of all {self.w.B * self.w.H} (b,h) "
                f"pairs, fp64 forward sweep and reverse state-gradient sweep, "
                f"{self.last_s:.1f} s per run on {self.threads} threads")


def backward_native(w, algorithm: str) -> bool:
    """Whether the library runs the backward's two reversed passes as reverse-mode
    prefills (bf16, C = 64, dk = dv = 128, not the chunked algorithm, not ELU+1 with decay)
    rather than on reversed copies."""
    return (w.dtype == "bf16" and w.C == 64 and w.dk == 128 and w.dv == 128
            and algorithm != "chunked" and not (w.feature_map == "elu1" and w.decay))


def backward_bytes(w, out_elem: int, algorithm: str, lseg: int = 0):
    """Algorithmic bytes per launch of every kernel of the backward, in launch order, for
    the bench's call (no initial or final state).  The element-wise input preparation
    (reversed copies where the reversed passes cannot run natively, psi(k) and psi(q) as
    bf16 hi / lo pairs under ELU+1); the prefill (do, v, psi(k)); for the normalised form
    the forward scan of Z (d_t, dd_t, dn_t as hi / lo, grad_q) and psi(q) / d_t; the
    prefills reversed (k, q, do or dn) and reversed (v, do, psi(q) [/ d]); each prefill
    once per bf16 half of its split operand; the reverse scan of the normaliser gradient;
    the output finish."""
    BH = w.B * w.H
    e = 2 if w.dtype == "bf16" else 4
    elu = w.feature_map == "elu1"
    split = elu and w.dtype == "bf16"
    norm = w.normalize
    native = backward_native(w, algorithm)
    halves = 2 if split else 1
    wk, wv = (not native) or elu, (not native) or norm
    w_f32 = native or out_elem == 4 or elu
    ew = 4 if w_f32 else 2
    nk, nv, nt = BH * w.T * w.dk, BH * w.T * w.dv, BH * w.T
    ops = []
    pre = 0 if native else 2 * (2 * nk + 2 * nv) * e  # reversed copies: read and write
    if elu:  # psi(k) (and psi(q) unnormalised): one read, hi (and lo) written
        pre += (1 if norm else 2) * (nk * e + halves * nk * e)
    if pre:
        ops.append(("bwd_reverse_inputs", pre))
    wa = w.with_(dk=w.dv, dv=w.dk, feature_map="identity", normalize=False)
    wb = w.with_(normalize=False)

    def prefills(pw, oe, n):
        algo = effective_algorithm(pw, algorithm)
        for _ in range(n):
            for name in kernel_names(pw, algo, "logdepth", lseg):
                ops.append((name, kernel_bytes(pw, name, oe, algo, lseg)))
    prefills(wa, 4 if elu else out_elem, halves)
    if norm:
        # totals read k; the walk reads k, q, do, S do (hi and lo passes), writes dn (hi /
        # lo), dd, 1 / d, grad_q
        ops.append(("bwd_z_scan", nk * e + 2 * nk * e + nv * e + halves * nk * 4
                    + halves * nv * e + 2 * nt * 4 + nk * out_elem))
        ops.append(("bwd_scaled_psi_q", nk * e + nt * 4 + halves * nk * e))
    prefills(wb, ew if wv else out_elem, halves if norm else 1)
    prefills(wa, ew if wk else out_elem, halves)
    if norm:  # g scan: totals and walk read q and dd; the walk writes g
        ops.append(("bwd_g_scan", 2 * (nk * e + nt * 4) + nk * 4))
    post = 0
    if wv:
        post += nv * ew * (halves if norm else 1) + nv * out_elem
    if wk:
        post += nk * ew + nk * out_elem + (nk * 4 if split else 0) + (nk * e if elu else 0)
    if elu and not norm:
        post += nk * 4 * halves + nk * e + nk * out_elem
    if norm:
        post += nk * 4  # the g term
    if post:
        ops.append(("bwd_reverse_outputs", post))
    return ops


def backward_bench(args, w, info, dev):
    """One backward (lin_attn_backward: grad_q, grad_k, grad_v for a given grad_out) per
    step, timed like the prefill."""
    q, k, v = make_inputs(w, seed=info.rank, device=dev)
    g = torch.Generator(device=dev).manual_seed(1000 + info.rank)
    do = torch.randn((w.B, w.H, w.T, w.dv), generator=g, device=dev).to(q.dtype)
    odt = torch.float32 if args.out_dtype == "f32" else q.dtype
    out_elem = 4 if args.out_dtype == "f32" else 2
    gq = torch.empty(q.shape, dtype=odt, device=dev)
    gk = torch.empty(k.shape, dtype=odt, device=dev)
    gv = torch.empty(v.shape, dtype=odt, device=dev)
    gam = w.gammas()
    ws = torch.empty(B.lin_attn_backward_workspace_bytes(q, v, chunk=w.C, feature_map=w.feature_map,
                                                        out_dtype=args.out_dtype, gamma=gam,
                                                        normalize=w.normalize,
                                                        algorithm=args.algorithm),
                     dtype=torch.uint8, device=dev)
    kw = dict(chunk=w.C, feature_map=w.feature_map, gamma=gam, out_dtype=args.out_dtype,
              kernel_path="tensor_core", algorithm=args.algorithm, workspace=ws,
              segment_chunks=args.segment_chunks)
    if w.normalize:
        kw.update(normalize=True)

    def step():
        B.lin_attn_backward(q, k, v, do, gq, gk, gv, **kw)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    def timed_region():
        sampler = None if args.no_clocks else ClockSampler(info.local_rank)
        if sampler:
            sampler.start()
        ranks.barrier(info)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            step()
        e1.record()
        torch.cuda.synchronize()
        ranks.barrier(info)
        return e0.elapsed_time(e1) / args.steps, (sampler.stop() if sampler else None)

    ms, clocks = timed_region()
    remeasured = False
    if ranks.any_over_ranks(clocks_bad(clocks), info, dev):
        ms, clocks = timed_region()
        remeasured = True
    ms_max = ranks.max_over_ranks(ms, info, dev)
    value = info.world * w.tokens_heads / (ms_max / 1000.0)

    # Per-kernel device times; kernels of the same name (the three passes) are pooled.
    tot, cnt, launches = {}, {}, 0
    reps = max(1, args.kernel_timing_steps)
    for _ in range(reps):
        t = B.lin_attn_backward_timed(q, k, v, do, gq, gk, gv, **kw)
        launches = len(t)
        for name, x in t:
            tot[name] = tot.get(name, 0.0) + x / reps
            cnt[name] = cnt.get(name, 0) + 1
    per_launch = {n: tot[n] / (cnt[n] / reps) for n in tot}
    ops = backward_bytes(w, out_elem, args.algorithm, args.segment_chunks)
    bytes_of = {}
    for name, nb in ops:
        bytes_of.setdefault(name, []).append(nb)
    dom = max(tot, key=tot.get)
    peak, peak_kind = measured_peaks()
    dom_bytes = statistics.mean(bytes_of[dom]) if dom in bytes_of else None
    achieved = dom_bytes / (per_launch[dom] / 1000.0) / 1e9 if dom_bytes else None
    roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak,
                "unit": "GB/s", "frac": achieved / peak if achieved else None,
                "traffic": None, "algorithmic_bytes": dom_bytes,
                "launches_per_step": cnt[dom] // reps,
                "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
                if peak_kind == "measured" else "fallback 6.65 TB/s"}
    step_bytes = sum(nb for _, nb in ops)
    BH = w.B * w.H
    e_in = 2 if w.dtype == "bf16" else 4
    min_b = BH * w.T * (2 * w.dk + 2 * w.dv) * e_in + BH * w.T * (2 * w.dk + w.dv) * out_elem
    gbs = lambda nb: nb / (ms_max / 1000.0) / 1e9
    step_roof = {"bytes": step_bytes, "achieved_gbs": gbs(step_bytes),
                 "frac_of_measured": gbs(step_bytes) / peak, "bytes_min": min_b,
                 "frac_min_of_measured": gbs(min_b) / peak,
                 "reversed_passes": "reverse-mode prefills" if backward_native(w, args.algorithm)
                 else "prefills on reversed copies",
                 "note": "bytes = the sum of every kernel's algorithmic bytes (three prefills "
                         "and the element-wise kernels); bytes_min = q, k, v, grad_out read once "
                         "and the three gradients written once"}

    # End to end: pinned host inputs copied in, the backward, the gradients copied out.
    e2e = None
    if not args.no_e2e:
        hin = [t.cpu().pin_memory() for t in (q, k, v, do)]
        hout = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (gq, gk, gv)]
        din = [torch.empty_like(t) for t in (q, k, v, do)]

        def e2e_step():
            for d_, h_ in zip(din, hin):
                d_.copy_(h_, non_blocking=True)
            B.lin_attn_backward(*din, gq, gk, gv, **kw)
            for h_, d_ in zip(hout, (gq, gk, gv)):
                h_.copy_(d_, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        ranks.barrier(info)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record()
        torch.cuda.synchronize()
        e_ms = ranks.max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, info, dev)
        e2e = {"value": info.world * w.tokens_heads / (e_ms / 1000.0), "unit": UNIT,
               "ms_per_step": e_ms,
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in hin),
               "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in hout),
               "api": "lin_attn_backward between pinned-host copies on the same stream"}
        del hin, hout, din

    cpu = None
    if info.is_root and info.world == 1 and not args.no_cpu_baseline:
        timer = BackwardOracleTimer(w, q, k, v, do, target_s=args.cpu_baseline_s)
        cpu = {"value": timer.rate(), "unit": UNIT, "cores": timer.threads, "kind": "oracle",
               "sample": timer.sample()}
    err = B.lin_attn_device_error()
    if info.is_root:
        cfg = config_of(w, args)
        cfg["algorithm"] = args.algorithm
        cfg.pop("segment_chunks", None)
        line = {
            "metric": METRIC_BWD, "value": value, "unit": UNIT, "n_gpus": info.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": cfg, "mode": "backward", "roofline": roofline,
            "step_roofline": step_roof, "kernels_ms": tot, "cpu_baseline": cpu, "e2e": e2e,
            "clocks": clocks, "remeasured": remeasured,
            "gpu_launches": launches * args.steps, "device_error": err,
        }
        print(json.dumps(line), flush=True)


# CUDA-core fp32 rate of one B200 from its unit counts: 148 SMs x 128 FMA lanes x 2 FLOP per
# clock x the 1965 MHz maximum SM clock (74.4 TFLOP/s).
NOMINAL_FP32_FLOPS = 148 * 128 * 2 * 1965e6
METRIC_GLA = "gated linear-attn prefill tokens·heads/s at H=32,d=128; % of roofline"


def gla_bench(args, info, dev):
    """Gated linear attention (lin_attn_gla_prefill) on the 128k-token gated workload, one
    prefill per step, timed like the main benchmark."""
    from chunked_causal_linear_b200.workloads import GLA_WORKLOADS, make_gates
    w = GLA_WORKLOADS["gla_128k"]
    if args.heads:
        w = w.with_(H=args.heads, name=f"{w.name}_h{args.heads}")
    q, k, v = make_inputs(w, seed=info.rank, device=dev)
    alpha = make_gates(w, seed=info.rank, device=dev)
    out = torch.empty((w.B, w.H, w.T, w.dv), dtype=torch.float32, device=dev)
    S = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
    ws = torch.empty(B.lin_attn_gla_workspace_bytes(w.B, w.H, w.T, w.dk, w.dv, w.C),
                     dtype=torch.uint8, device=dev)
    kw = dict(chunk=w.C, out_dtype="f32", workspace=ws, kernel_path=args.gla_path)

    def step():
        B.lin_attn_gla_prefill(q, k, v, alpha, out, S, **kw)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    sampler = None if args.no_clocks else ClockSampler(info.local_rank)
    if sampler:
        sampler.start()
    ranks.barrier(info)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    ranks.barrier(info)
    clocks = sampler.stop() if sampler else None
    ms_max = ranks.max_over_ranks(e0.elapsed_time(e1) / args.steps, info, dev)
    per = [B.lin_attn_gla_prefill_timed(q, k, v, alpha, out, S, **kw)
           for _ in range(max(1, args.kernel_timing_steps))]
    tc = args.gla_path in ("tensor_core", "auto")  # auto: the tensor cores at this shape
    names = (["gla_k1_seg", "gla_scan", "gla_k3_seg", "gla_fixup"] if tc
             else ["gla_k1", "gla_k2", "gla_k3"])
    kern_ms = {n: statistics.mean(x[i] for x in per) for i, n in enumerate(names)}
    BH, NC, C = w.B * w.H, -(-w.T // w.C), w.C
    R = w.dk * w.dv + w.dk
    pairs = C * (C + 1) // 2
    # K3's fp32 work per chunk: the prefix product C dk dv, the scores over the lower triangle
    # pairs dk, the intra product pairs dv (2 FLOP per multiply-add); with gates whose chunk
    # logs stay above -100 (all of this workload's) the scores need no exponential per pair
    k3_flop = 2 * BH * NC * (C * w.dk * w.dv + pairs * w.dk + pairs * w.dv)
    e_in = 2
    NS = -(-NC // segment_length(w))  # the tensor-core path's segments (automatic length)
    bytes_ = {"gla_k1": BH * w.T * (w.dk * (e_in + 4) + w.dv * e_in) + BH * NC * R * 4,
              "gla_k2": 2 * BH * NC * R * 4,
              "gla_k3": BH * w.T * (w.dk * (2 * e_in + 4) + w.dv * e_in + w.dv * 4) + BH * NC * R * 4,
              # tensor cores, per token*head: K1 reads k, v, gates; K3 reads q, k, v, gates and
              # writes the float32 output; per segment a record of R floats (K1 writes it,
              # the scan reads and writes it, K3 reads its state part); one flag per chunk
              "gla_k1_seg": BH * w.T * (w.dk * (e_in + 4) + w.dv * e_in) + BH * NS * R * 4,
              "gla_scan": 2 * BH * NS * R * 4 + BH * w.dk * w.dv * 4,
              "gla_k3_seg": BH * w.T * (w.dk * (2 * e_in + 4) + w.dv * e_in + w.dv * 4)
              + BH * NS * w.dk * w.dv * 4 + BH * NC,
              "gla_fixup": BH * NC}
    peak, peak_kind = measured_peaks()
    hbm = {n: bytes_[n] / (kern_ms[n] / 1e3) / 1e9 / peak for n in names}
    if tc:
        dom = max(kern_ms, key=kern_ms.get)
        roofline = {"bound": "hbm", "kernel": dom,
                    "achieved": bytes_[dom] / (kern_ms[dom] / 1e3) / 1e9, "peak": peak,
                    "unit": "GB/s", "frac": hbm[dom], "traffic": None,
                    "algorithmic_bytes": bytes_[dom],
                    "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)",
                    "hbm_frac_of_measured": hbm}
    else:
        roofline = {"bound": "alu", "kernel": "gla_k3",
                    "achieved": k3_flop / (kern_ms["gla_k3"] / 1e3) / 1e12,
                    "peak": NOMINAL_FP32_FLOPS / 1e12, "unit": "TFLOP/s (fp32, CUDA cores)",
                    "frac": k3_flop / (kern_ms["gla_k3"] / 1e3) / NOMINAL_FP32_FLOPS,
                    "traffic": None,
                    "peak_source": "unit counts: 148 SMs x 128 FMA lanes x 2 x 1965 MHz",
                    "hbm_frac_of_measured": hbm}
    if info.is_root:
        cfg = {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "dk": w.dk, "dv": w.dv, "C": w.C,
               "inputs": "bf16", "gates": "float32 sigmoid(N(4, 1))", "out_dtype": "f32",
               "kernel_path": "tensor_core (segmented, factored hi/lo operands)" if tc
               else "fma (CUDA cores)", "segments": NS if tc else None,
               "l2": "inputs larger than L2, no flush",
               "parallelism": "replicas (one independent problem per GPU)"}
        line = {"metric": METRIC_GLA, "value": info.world * w.tokens_heads / (ms_max / 1e3),
                "unit": UNIT, "n_gpus": info.world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": cfg,
                "mode": "gla", "roofline": roofline, "kernels_ms": kern_ms, "clocks": clocks,
                "gpu_launches": len(names) * args.steps, "device_error": B.lin_attn_device_error()}
        print(json.dumps(line), flush=True)


def scan_depth(w, args) -> dict:
    """The implemented K2 depth (dependent combine steps per column) of this run."""
    algo = effective_algorithm(w, args.algorithm)
    n, _, _ = layout(w, algo, getattr(args, "segment_chunks", 0))
    try:
        d = B.lin_attn_scan_plan(n, args.scan)["depth"]
    except Exception:  # library not built (CPU-only tooling)
        d = None
    return {"elements": n, "depth": d, "ceil_log2_elements": math.ceil(math.log2(max(n, 2)))}


METRIC_DEC = "causal linear-attn decode steps: state bytes/s; % of roofline"
DECODE_CASES = ((8, 32), (64, 32), (1, 32))  # (B, H) at dk = dv = 128


def decode_bytes(Bn, H, dk, dv, e_in, e_out, with_z):
    """Bytes one decode step must move: the state read and written once, q, k, v read, the
    output written (and Z read and written when it is kept)."""
    per = 2 * dk * dv * 4 + (2 * dk + dv) * e_in + dv * e_out + (2 * dk * 4 if with_z else 0)
    return Bn * H * per


def decode_bench(args, dev):
    """One decode step for every (b, h) at dk = dv = 128, bf16 q, k, v and output, float32
    state: the retention form (identity map, per-head decay) and the normalised ELU+1 form.
    The steps are captured in a CUDA graph (64 steps) and the graph replayed, so the time is
    the kernels' own; each case is first checked against the oracle (one step from the
    same state)."""
    from oracle.oracle import default_oracle
    peak, peak_kind = measured_peaks()
    dk = dv = 128
    nsteps = 64
    for Bn, H in DECODE_CASES:
        for form in ("retention", "normalised"):
            norm = form == "normalised"
            fm = "elu1" if norm else "identity"
            gam = None if norm else [float(1 - 2.0 ** (-5 - 3 * h / 31)) for h in range(H)]
            g = torch.Generator(device=dev).manual_seed(0)
            scale = 0.5 if norm else 128 ** -0.5
            q, k, v = (torch.randn((Bn, H, d), generator=g, device=dev).mul_(scale)
                       .to(torch.bfloat16) for d in (dk, dk, dv))
            S = torch.randn((Bn, H, dk, dv), generator=g, device=dev).mul_(0.1)
            Z = torch.rand((Bn, H, dk), generator=g, device=dev).add_(1.0) if norm else None
            out = torch.empty((Bn, H, dv), dtype=torch.bfloat16, device=dev)
            kw = dict(feature_map=fm, gamma=gam, normalize=norm)
            # Parity: one step against the oracle from the same state (a sample of heads).
            S0 = S.cpu().numpy()
            Z0 = Z.cpu().numpy() if Z is not None else None
            B.lin_attn_decode_step(q, k, v, S, Z, out=out, **kw)
            torch.cuda.synchronize()
            f = lambda t: t.float().cpu().numpy()[:, :, None]
            o_ref, S_ref, _ = default_oracle().forward(
                f(q), f(k), f(v), feature_map=fm, normalize=norm,
                gamma=None if gam is None else np.asarray(gam, dtype=np.float64),
                S_init=S0, Z_init=Z0)
            got = out.float().cpu().numpy()
            err_o = float(np.max(np.abs(got - o_ref[:, :, 0])) / np.sqrt(np.mean(o_ref ** 2)))
            err_S = float(np.max(np.abs(S.cpu().numpy() - S_ref)) / np.sqrt(np.mean(S_ref ** 2)))
            # Time: a graph of nsteps steps, replayed.
            stream = torch.cuda.Stream(device=dev)
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.stream(stream):
                B.lin_attn_decode_step(q, k, v, S, Z, out=out, stream=stream, **kw)
                stream.synchronize()
                with torch.cuda.graph(graph, stream=stream):
                    for _ in range(nsteps):
                        B.lin_attn_decode_step(q, k, v, S, Z, out=out, stream=stream, **kw)
            for _ in range(max(3, args.warmup)):
                graph.replay()
            torch.cuda.synchronize()
            reps = max(5, args.steps // 4)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                graph.replay()
            e1.record()
            torch.cuda.synchronize()
            us = e0.elapsed_time(e1) * 1000.0 / (reps * nsteps)
            nb = decode_bytes(Bn, H, dk, dv, 2, 2, norm)
            gbs = nb / (us * 1e-6) / 1e9
            line = {
                "metric": METRIC_DEC, "workload": f"decode_b{Bn}h{H}_d128_{form}",
                "B": Bn, "H": H, "dk": dk, "dv": dv, "heads": Bn * H,
                "us_per_step": us, "steps_per_s": 1e6 / us,
                "tokens_heads_per_s": Bn * H * 1e6 / us, "bytes_per_step": nb,
                "roofline": {"bound": "hbm", "kernel": "decode_tiles", "achieved": gbs,
                             "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                             "peak_source": peak_kind},
                "parity_vs_oracle": {"out_max_err_over_rms": err_o, "S_max_err_over_rms": err_S,
                                     "bound": 2e-2},
                "timing": f"CUDA graph of {nsteps} steps replayed {reps} times, CUDA events",
                "state_bytes": Bn * H * dk * dv * 4,
                "l2": "state larger than L2" if Bn * H * dk * dv * 4 > 126e6 else
                      "state fits in L2 (a step re-reads it from L2)",
            }
            print(json.dumps(line), flush=True)
            del graph


def config_of(w, args):
    return {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "dk": w.dk, "dv": w.dv,
            "C": w.C, "inputs": w.dtype, "feature_map": w.feature_map,
            "gamma": "1 - 2^(-5-3h/31) per head" if w.decay else None,
            "normalize": w.normalize, "scan": args.scan, "out_dtype": args.out_dtype,
            "algorithm": effective_algorithm(w, args.algorithm),
            **({"segment_chunks": segment_length(w, getattr(args, "segment_chunks", 0))}
               if effective_algorithm(w, args.algorithm) == "segmented" else {}),
            "kernel_path": kernel_path_for(w),
            "l2": "inputs larger than L2, no flush" if w.B * w.H * w.T * (2 * w.dk + w.dv)
            * (2 if w.dtype == "bf16" else 4) > 126e6 else "inputs fit in L2 (latency case)",
            "scan_depth": scan_depth(w, args),
            "parallelism": "replicas (one independent problem per GPU)"}


# ---------------------------------------------------------------------------------------
# GPU side


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="retention_128k", choices=sorted(WORKLOADS))
    ap.add_argument("--scan", default="logdepth", choices=["logdepth", "sequential"])
    ap.add_argument("--algorithm", default="auto", choices=["auto", "chunked", "segmented"])
    ap.add_argument("--out-dtype", default="f32", choices=["f32", "as_input"])
    ap.add_argument("--kernel-timing-steps", type=int, default=10)
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-baseline-s", type=float, default=15.0)
    ap.add_argument("--reference-step-s", type=float, default=10.0,
                    help="reference arm: upper bound on the seconds of one sample step")
    ap.add_argument("--reference-total-s", type=float, default=120.0,
                    help="reference arm: warm-up plus timed steps take about this long")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--sweep-scan", action="store_true",
                    help="instead of the benchmark line: time K2 (log-depth vs sequential "
                         "carry) over a range of chunk counts, one JSON line per point")
    ap.add_argument("--segment-chunks", type=int, default=0,
                    help="chunks per segment of the segmented algorithm (0: automatic)")
    ap.add_argument("--seq-shard", action="store_true",
                    help="instead of independent replicas: one sequence split across the ranks "
                         "(each rank a contiguous token range; states-only pass, all_gather of "
                         "the range states, fold, prefill from the incoming state); strong "
                         "scaling")
    ap.add_argument("--backward", action="store_true",
                    help="instead of the prefill: the backward of the unnormalised form "
                         "(grad_q, grad_k, grad_v for a random grad_out)")
    ap.add_argument("--gla", action="store_true",
                    help="instead of the prefill: gated linear attention (data-dependent decay) "
                         "on the 128k-token gated workload")
    ap.add_argument("--gla-path", default="auto", choices=["auto", "fma", "tensor_core"],
                    help="GLA kernels: the library's choice (tensor cores at this shape), the "
                         "CUDA-core ones, or the tensor-core ones")
    ap.add_argument("--decode", action="store_true",
                    help="instead of the prefill: the decode step (state in place) at B.H = "
                         "256, 2048 and 32, dk = dv = 128, one JSON line per case")
    ap.add_argument("--heads", type=int, default=None,
                    help="run the workload with this many heads instead (smaller cases for "
                         "profiler captures; every other size unchanged)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    w = WORKLOADS[args.workload]
    if args.heads:
        w = w.with_(H=args.heads, name=f"{w.name}_h{args.heads}")
    if args.impl == "reference":
        info = ranks.rank_info()
        reference_arm(args, w, info)
        return

    info = ranks.init("nccl")
    dev = torch.device("cuda", info.local_rank)
    torch.cuda.set_device(dev)
    B.load_library()
    if args.sweep_scan:
        sweep_scan(args, dev)
        ranks.finish(info)
        return
    if args.seq_shard:
        seq_shard_bench(args, w, info, dev)
        ranks.finish(info)
        return
    if args.backward:
        backward_bench(args, w, info, dev)
        ranks.finish(info)
        return
    if args.gla:
        gla_bench(args, info, dev)
        ranks.finish(info)
        return
    if args.decode:
        decode_bench(args, dev)
        ranks.finish(info)
        return

    q, k, v = make_inputs(w, seed=info.rank, device=dev)
    out_dtype = torch.float32 if args.out_dtype == "f32" else q.dtype
    out_elem = 4 if args.out_dtype == "f32" else 2
    out = torch.empty((w.B, w.H, w.T, w.dv), dtype=out_dtype, device=dev)
    S = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
    Z = torch.empty((w.B, w.H, w.dk), dtype=torch.float32, device=dev) if w.normalize else None
    ws = torch.empty(B.lin_attn_prefill_workspace_bytes(w.B, w.H, w.T, w.dk, w.dv, w.C,
                                                        w.normalize),
                     dtype=torch.uint8, device=dev)
    gam = w.gammas()
    algo = effective_algorithm(w, args.algorithm)
    kw = dict(chunk=w.C, feature_map=w.feature_map, gamma=gam, normalize=w.normalize,
              scan=args.scan, kernel_path=kernel_path_for(w), workspace=ws, out_dtype=args.out_dtype,
              algorithm=algo, segment_chunks=args.segment_chunks)

    def step():
        B.lin_attn_prefill(q, k, v, out, S, Z, **kw)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    def timed_region():
        sampler = None if args.no_clocks else ClockSampler(info.local_rank)
        if sampler:
            sampler.start()
        ranks.barrier(info)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            step()
        e1.record()
        torch.cuda.synchronize()
        ranks.barrier(info)
        clocks = sampler.stop() if sampler else None
        return e0.elapsed_time(e1) / args.steps, clocks

    ms, clocks = timed_region()
    remeasured = False
    if ranks.any_over_ranks(clocks_bad(clocks), info, dev):
        ms, clocks = timed_region()
        remeasured = True
    ms_max = ranks.max_over_ranks(ms, info, dev)
    names = kernel_names(w, algo, args.scan, args.segment_chunks)
    n_kern = len(names)
    value = info.world * w.tokens_heads / (ms_max / 1000.0)

    # Per-kernel device times (events between the library's own launches, same stream).
    per = [[] for _ in names]
    for _ in range(max(1, args.kernel_timing_steps)):
        t = B.lin_attn_prefill_timed(q, k, v, out, S, Z, **kw)
        for i, x in enumerate(t[:len(names)]):
            per[i].append(x)
    kern_ms = {n: statistics.mean(x) for n, x in zip(names, per)}
    dom = max(kern_ms, key=kern_ms.get)
    peak, peak_kind = measured_peaks()
    dom_bytes = kernel_bytes(w, dom, out_elem, algo, args.segment_chunks)
    achieved = dom_bytes / (kern_ms[dom] / 1000.0) / 1e9
    roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak,
                "unit": "GB/s", "frac": achieved / peak,
                "traffic": recorded_traffic(dom, w.name),
                "algorithmic_bytes": dom_bytes, "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
                if peak_kind == "measured" else "fallback 6.65 TB/s"}
    ab = algo_bytes(w, out_elem, algo, args.segment_chunks)
    gbs = lambda nbytes: nbytes / (ms_max / 1000.0) / 1e9
    step_roof = {"algorithm": algo, "bytes": ab, "achieved_gbs": gbs(ab),
                 "frac_of_measured": gbs(ab) / peak,
                 "frac_of_nominal_8tbs": gbs(ab) / NOMINAL_HBM_GBS,
                 "bytes_min": min_bytes(w, out_elem),
                 "frac_min_of_measured": gbs(min_bytes(w, out_elem)) / peak,
                 "bytes_chunked_method": method_bytes(w, out_elem),
                 "time_at_measured_bw_ms": ab / (peak * 1e9) * 1e3}

    # End to end through the host-buffer entry point (pinned host memory).
    e2e = None
    if not args.no_e2e:
        qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
        oh = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        Sh = torch.empty(S.shape, dtype=torch.float32).pin_memory()
        Zh = torch.empty(Z.shape, dtype=torch.float32).pin_memory() if Z is not None else None
        hkw = dict(chunk=w.C, feature_map=w.feature_map, gamma=gam, normalize=w.normalize,
                   scan=args.scan, kernel_path=kernel_path_for(w), out_dtype=args.out_dtype,
                   algorithm=algo)
        dbuf = torch.empty(B.lin_attn_prefill_host_buffer_bytes(qh, vh, chunk=w.C,
                                                                normalize=w.normalize,
                                                                out_dtype=args.out_dtype),
                           dtype=torch.uint8, device=dev)
        B.lin_attn_prefill_host(qh, kh, vh, oh, Sh, Zh, device_buffer=dbuf, **hkw)
        ranks.barrier(info)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.e2e_steps):
            B.lin_attn_prefill_host(qh, kh, vh, oh, Sh, Zh, device_buffer=dbuf, **hkw)
        e1.record()
        torch.cuda.synchronize()
        e_ms = ranks.max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, info, dev)
        h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
        d2h = oh.numel() * oh.element_size() + Sh.numel() * 4 + (Zh.numel() * 4 if Zh is not None else 0)
        copy_ms = copy_bound_ms([(q, qh), (k, kh), (v, vh)],
                                [(oh, out), (Sh, S)] + ([(Zh, Z)] if Zh is not None else []))
        e2e = {"value": info.world * w.tokens_heads / (e_ms / 1000.0), "unit": UNIT,
               "ms_per_step": e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "api": "lin_attn_prefill_host (pinned host buffers; copies in, kernels and copies out overlapped across groups of heads; synchronous)",
               "copy_bound_ms": copy_ms, "frac_of_copy_bound": copy_ms / e_ms,
               "copy_bound": "the same bytes as plain copies between the same pinned buffers and "
                             "device memory, both directions at once on two streams, no kernels"}
        del qh, kh, vh, oh, Sh, Zh, dbuf

    cpu = None
    if info.is_root and info.world == 1 and not args.no_cpu_baseline:
        timer = OracleTimer(w, q, k, v, target_s=args.cpu_baseline_s)
        rate = timer.rate()
        cpu = {"value": rate, "unit": UNIT, "cores": timer.threads, "kind": "oracle",
               "sample": timer.sample()}

    err = B.lin_attn_device_error()
    if info.is_root:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": info.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32",
            "data": "synthetic", "config": config_of(w, args), "roofline": roofline,
            "step_roofline": step_roof, "kernels_ms": kern_ms, "cpu_baseline": cpu,
            "e2e": e2e, "clocks": clocks, "remeasured": remeasured,
            "gpu_launches": n_kern * args.steps, "device_error": err,
        }
        print(json.dumps(line), flush=True)
    ranks.finish(info)


if __name__ == "__main__":
    main()
