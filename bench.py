#!/usr/bin/env python
"""Benchmark: OrbitQuant online quantized-linear path on B200.

One step = the whole hot path on one batch: by default one oq_quantized_linear call (fused
RPBH rotate + norm + Lloyd-Max quantize of the activations, whose fp16 centroids go straight to
the codebook GEMM against weight codes quantized offline, before timing); with --api calls,
oq_quantize_act followed by oq_linear.  Default workload: the FLUX-like attention projection
(T = 4608 tokens, d = 3072 -> 3072, bf16 inputs, h = 128, W4A4).  The JSON line carries the
step rate (CUDA-graph replays), the end-to-end rate from pinned host memory (e2e), the
rooflines of the GEMM (roofline) and of the quantize kernel (roofline_quantize, plus the
codes-only launch as context), the oracle's CPU rate (cpu_baseline), clocks and launches.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun, one rank per GPU): every rank runs its own batch of T tokens (weak
scaling; the path has no exchange step, so no collective touches the data); the timed region
is bracketed by a barrier + synchronize, and the max over ranks is reported.
``--impl reference`` times the fp64 CPU oracle on the host cores instead (rank 0 only).
Rank 0 prints one JSON line on stdout; everything else goes to stderr.
"""
import argparse
import csv
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from calibration_free_bit_b200 import synth  # noqa: E402

METRIC = ("quantized-linear tokens/s at d=3072; % of HBM (quantize) / BF16 tensor (GEMM) "
          "peak")
NSETS = 4            # rotating buffer sets: working set > L2 between reuses
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="flux_attn_w4a4")
    ap.add_argument("--proj", type=int, default=0, help="projection index within the workload")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--api", choices=("forward", "calls"), default="forward",
                    help="forward: oq_quantized_linear (one call, codes stay on chip); "
                         "calls: oq_quantize_act then oq_linear")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true",
                    help="time K1 (oq_quantize_act, codes output) over the activation sweep "
                         "(d x h x bits x T) and print one JSON line per point, then a summary")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_sha(rels):
    """First 16 hex digits of the SHA-256 of the concatenated source files."""
    h = hashlib.sha256()
    for rel in rels:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


GEMM_SOURCES = ("calibration_free_bit_b200/csrc/k2_linear.cu",
                "calibration_free_bit_b200/csrc/sm100_common.cuh",
                "calibration_free_bit_b200/csrc/decode4.cuh")
K1_SOURCES = ("calibration_free_bit_b200/csrc/k1_rotquant.cu",
              "calibration_free_bit_b200/csrc/k1_ops.cuh",
              "calibration_free_bit_b200/csrc/decode4.cuh")


def profile_traffic(profile_name, kernel_src):
    """DRAM bytes per launch of a kernel from a committed ncu export, or None if absent or
    stale.  The file is `ncu --csv --page raw` output (one row per captured launch, columns
    dram__bytes_read.sum and dram__bytes_write.sum in bytes) after comment lines written by the
    capture command, one of which records the SHA-256 (first 16 hex digits) of the kernel's
    sources at capture time: a capture of other sources is not used."""
    path = os.path.join(ROOT, "profiles", profile_name)
    if not os.path.exists(path):
        return None, "no profile"
    lines = open(path).read().splitlines()
    sha = None
    for ln in lines:
        m = re.match(r"#\s*sources_sha256_16:\s*([0-9a-f]{16})", ln)
        if m:
            sha = m.group(1)
    if sha is None:
        return None, "profile lacks the sources hash"
    if sha != source_sha(kernel_src):
        return None, "kernel changed since capture"
    rows = list(csv.reader([ln for ln in lines if ln and not ln.startswith("#")]))
    if len(rows) < 2:
        return None, "profile has no launch rows"
    head = rows[0]
    try:
        ir, iw = head.index("dram__bytes_read.sum"), head.index("dram__bytes_write.sum")
    except ValueError:
        return None, "profile lacks DRAM byte counters"
    vals = []
    for r_ in rows[1:]:
        try:
            vals.append(float(r_[ir]) + float(r_[iw]))
        except (ValueError, IndexError):
            continue                               # the units row of the raw page
    if not vals:
        return None, "profile has no numeric rows"
    return statistics.mean(vals), "ncu (profiles/" + profile_name + ")"


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.target = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.target = str(device_index)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", self.target], stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.06)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.flush()
        self.out.seek(0)
        sm, smax, power, reasons = [], [], [], set()
        for line in self.out.read().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
                power.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        os.unlink(self.out.name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "power_w_max": max(power), "samples": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------------------------------------------
# oracle (CPU) arm: used for --impl reference and for the cpu_baseline field
# ------------------------------------------------------------------------------------------

class OracleStep:
    """The oracle's version of one step on S tokens: fp64 RPBH + Lloyd-Max codes of the
    activations, then the naive triple-loop linear against all output features."""

    def __init__(self, p):
        import oracle as O
        self.O, self.p = O, p
        self.perm, self.sign = (O.build_rpbh if p.rotation == "rpbh" else O.build_block_rht)(
            p.d, 0)
        self.marginal = "sphere" if p.marginal == "exact" else "gauss"
        W = synth.weight(p).double().numpy()
        self.wc, self.rn = O.quantize_weight(W, p.h, self.perm, self.sign, p.bits_w,
                                             marginal=self.marginal)
        self.x = synth.activations(p, rows=np.arange(min(p.T, 2048))).double().numpy()
        self.cursor = 0

    def _rows(self, xr):
        xc, s = self.O.quantize_act(xr, self.p.h, self.perm, self.sign, self.p.bits_a,
                                    marginal=self.marginal, gelu_input=self.p.fused_gelu)
        self.O.linear(xc, s, self.wc, self.rn, self.p.d, self.p.bits_a, self.p.bits_w,
                      marginal=self.marginal)

    def run(self, S, threads=1):
        """Seconds for S tokens; threads > 1 splits the tokens into one chunk per host thread
        (the oracle's C calls release the GIL, so the chunks run in parallel)."""
        rows = (self.cursor + np.arange(S)) % len(self.x)
        self.cursor = int(rows[-1] + 1)
        xr = self.x[rows]
        self.O.codebook(self.p.bits_a, self.marginal, self.p.d)   # cached before timing
        self.O.codebook(self.p.bits_w, self.marginal, self.p.d)
        t0 = time.perf_counter()
        if threads <= 1:
            self._rows(xr)
        else:
            import concurrent.futures as cf
            parts = np.array_split(np.arange(S), threads)
            with cf.ThreadPoolExecutor(threads) as ex:
                list(ex.map(lambda ix: self._rows(xr[ix]), [q for q in parts if len(q)]))
        return time.perf_counter() - t0


def cores_used():
    return 1   # the oracle is single-threaded C


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def run_reference(args, p):
    step = OracleStep(p)
    probe = step.run(4) / 4                          # seconds per token, calibration
    budget = 120.0                                   # seconds for warmup + timed steps
    S = int(max(1, min(512, budget / max(1, args.steps + args.warmup) / max(probe, 1e-9))))
    for _ in range(args.warmup):
        step.run(S)
    total = 0.0
    for _ in range(args.steps):
        total += step.run(S)
    value = S * args.steps / total
    sample = (f"{S} tokens per step of the {p.name} workload (d={p.d} -> {p.out}): fp64 "
              f"rotate+quantize of the S rows, then all {p.out} outputs by the naive loop")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(p, 1),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores_used(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def cpu_baseline(p):
    step = OracleStep(p)
    per_tok = step.run(8) / 8
    S = int(max(8, min(1024, 15.0 / max(per_tok, 1e-9))))
    t = step.run(S)
    out = {"value": S / t, "unit": "tokens/s", "cores": cores_used(), "kind": "oracle",
           "sample": f"{S} tokens of {p.name}: fp64 rotate+quantize then all {p.out} outputs "
                     f"(naive loop), {t:.1f} s on one host core"}
    # the same oracle over token chunks on every host core, reported separately
    n = host_cores()
    if n > 1:
        Sn = int(max(8 * n, min(8192, 10.0 * n / max(per_tok, 1e-9))))
        tn = step.run(Sn, threads=n)
        out["threads"] = {"value": Sn / tn, "unit": "tokens/s", "cores": n,
                          "sample": f"{Sn} tokens in {n} chunks on {n} host threads, "
                                    f"{tn:.1f} s"}
    return out


def max_over_ranks(x: float, world: int, device) -> float:
    """Max of a per-rank scalar over all ranks (the only collective: timing, not data)."""
    if world <= 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, units_per_rank_step: int, steps: int, ms_max: float) -> float:
    """Units all ranks processed, divided by the slowest rank's time (weak scaling)."""
    return world * units_per_rank_step * steps / (ms_max / 1e3)


def workload_config(p, world):
    return {"workload": f"{p.name}: FLUX-like attention projection" if p.name.startswith(
                "flux_attn") else p.name,
            "T_per_gpu": p.T, "d": p.d, "out": p.out, "h": p.h, "bits_w": p.bits_w,
            "bits_a": p.bits_a, "input": "bf16" if p.dtype == torch.bfloat16 else "fp32",
            "l2": f"{NSETS} rotating buffer sets (x, codes, s, y, W codes) > 126 MB L2",
            "rotation": p.rotation, "codebook_marginal": p.marginal,
            "fused_gelu": p.fused_gelu,
            "parallelism": f"dp{world}: independent token batches, no collective"}


# ------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------

def run_ours(args, p, rank, world, dev):
    from calibration_free_bit_b200 import build as B
    B.build()
    from calibration_free_bit_b200 import oq

    r = (oq.oq_build_rpbh if p.rotation == "rpbh" else oq.oq_build_block_rht)(p.d, p.h, 0)
    ca = oq.oq_lloyd_max(p.d, p.bits_a, p.marginal)
    cw = oq.oq_lloyd_max(p.d, p.bits_w, p.marginal)
    x_cpu = synth.activations(p)
    W = synth.weight(p).to(dev)
    wc0, rn = oq.oq_quantize_weight(r, cw, W)                # offline, untimed
    del W
    sets = []
    for _ in range(NSETS):
        x = x_cpu.to(dev)
        sets.append({
            "x": x,
            "xc": torch.empty((p.T, p.d * p.bits_a // 8), dtype=torch.uint8, device=dev),
            "s": torch.empty(p.T, dtype=torch.float32, device=dev),
            "y": torch.empty((p.T, p.out), dtype=torch.float32, device=dev),
            "wc": wc0.clone(),
        })
    torch.cuda.synchronize()

    def run_path(b):
        if args.api == "forward":
            oq.oq_quantized_linear(r, ca, cw, b["x"], b["wc"], rn, y=b["y"], s=b["s"],
                                   gelu=p.fused_gelu)
        else:
            oq.oq_quantize_act(r, ca, b["x"], b["xc"], b["s"], gelu=p.fused_gelu)
            oq.oq_linear(ca, cw, b["xc"], b["s"], b["wc"], rn, b["y"])

    def step(i):
        run_path(sets[i % NSETS])

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    for i in range(args.warmup):
        step(i)
    oq.oq_check()
    oq.oq_timing_collect()

    # (1) eager region: the per-call path (host launch cost included)
    barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    h0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    host_ms = (time.perf_counter() - h0) * 1e3
    ev1.record()
    barrier()
    oq.oq_check()
    eager_ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)

    # (2) per-kernel region: the same eager steps, each kernel bracketed by CUDA events on its
    #     stream, queued behind a GPU spin so the host has enqueued everything before the
    #     device reaches it; the event pairs then bracket device execution, not host gaps.
    n_k = max(1, min(args.steps, 400))
    spin_s = 1.5 * (host_ms / args.steps) * n_k / 1e3 + 0.02
    barrier()
    torch.cuda._sleep(int(spin_s * 2.0e9))
    oq.oq_timing_enable(True)
    for i in range(n_k):
        step(i)
    oq.oq_timing_enable(False)
    torch.cuda.synchronize()
    oq.oq_check()
    per_kernel = {}
    for name, t in oq.oq_timing_collect():
        per_kernel.setdefault(name, []).append(t)
    # liboq kernel launches per step, counted from the timing records of the n_k eager steps
    launches_per_step = round(sum(len(v) for v in per_kernel.values()) / n_k)

    # (3) headline region: the step captured once per buffer set in a CUDA graph and replayed,
    #     so host launch cost does not pace the device
    graphs = []
    try:
        for b in range(NSETS):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step(b)
            graphs.append(g)
        replay = lambda i: graphs[i % NSETS].replay()         # noqa: E731
        timing_mode = "cuda-graph replay"
    except Exception as exc:                                  # capture unsupported: stay eager
        log(f"graph capture failed ({exc}); timing eager calls")
        graphs = []
        torch.cuda.synchronize()
        replay = step
        timing_mode = "eager calls (graph capture failed)"
    for i in range(max(3, args.warmup)):
        replay(i)
    oq.oq_check()
    clocks = ClockSampler(dev.index) if rank == 0 else None
    barrier()
    if clocks:
        clocks.start()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record()
    for i in range(args.steps):
        replay(i)
    g1.record()
    barrier()
    clock_info = clocks.stop() if clocks else None
    oq.oq_check()
    ms_max = max_over_ranks(g0.elapsed_time(g1), world, dev)
    # the quantizer writes the fp16 operand itself on the forward path with 2/4/8-bit
    # activations, bf16 x and h <= 256 (and, for 4-bit weights, decodes the weights too)
    # with OQ_LINEAR_PATH=fused and 4-bit activations the quantizer writes packed codes and the
    # GEMM decodes them in shared memory
    acodes = (os.environ.get("OQ_LINEAR_PATH") == "fused" and p.bits_a == 4
              and p.dtype == torch.bfloat16)
    # with OQ_LINEAR_PATH=wcodes and 4-bit weights the GEMM decodes the weight codes itself
    wcodes = (os.environ.get("OQ_LINEAR_PATH") == "wcodes" and p.bits_w == 4
              and os.environ.get("OQ_GEMM_PAIR") != "0")
    direct = (args.api == "forward" and not acodes and p.bits_a in (2, 4, 8)
              and p.dtype == torch.bfloat16 and 32 <= p.h <= 256)
    launches = launches_per_step * args.steps
    del graphs

    # context for the quantize roofline, outside every timed region of the step: the same K1
    # on the same rows with packed-code output (oq_quantize_act, the two-call form), which does
    # only the method's work (no fp16 operand, no weight decode)
    codes_q_ms = None
    if args.api == "forward":
        for i in range(3):
            b = sets[i % NSETS]
            oq.oq_quantize_act(r, ca, b["x"], b["xc"], b["s"], gelu=p.fused_gelu)
        n_q = 50
        torch.cuda.synchronize()
        q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        # behind a GPU spin, so that all launches are queued before the device reaches them
        torch.cuda._sleep(int(0.02 * 2.0e9))
        q0.record()
        for i in range(n_q):
            b = sets[i % NSETS]
            oq.oq_quantize_act(r, ca, b["x"], b["xc"], b["s"], gelu=p.fused_gelu)
        q1.record()
        torch.cuda.synchronize()
        oq.oq_check()
        codes_q_ms = q0.elapsed_time(q1) / n_q

    # end-to-end through the public calls with host buffers (pinned), copies inside timing
    e2e = None
    if not args.no_e2e:
        # End to end through the public API from pinned host memory, pipelined over three
        # buffer sets on three streams: the host->device copy of step i+1 and the
        # device->host copy of step i-1 run while step i computes (copies in both directions
        # overlap on the full-duplex link).  Every step still moves its whole input in and
        # its whole output out.
        NB = 3
        xh = x_cpu.pin_memory()
        yhs = [torch.empty((p.T, p.out), dtype=torch.float32).pin_memory() for _ in range(NB)]
        s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
        ev = {k: [torch.cuda.Event() for _ in range(NB)] for k in ("in", "comp", "out")}
        used = [False] * NB

        def e2e_step(i):
            k = i % NB
            b = sets[k]
            with torch.cuda.stream(s_in):
                if used[k]:
                    s_in.wait_event(ev["comp"][k])         # x[k] consumed by step i - NB
                b["x"].copy_(xh, non_blocking=True)
                ev["in"][k].record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev["in"][k])
                if used[k]:
                    s_comp.wait_event(ev["out"][k])        # y[k] read out by step i - NB
                run_path(b)
                ev["comp"][k].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev["comp"][k])
                yhs[k].copy_(b["y"], non_blocking=True)
                ev["out"][k].record(s_out)
            used[k] = True

        for i in range(max(3, min(args.warmup, 20))):
            e2e_step(i)
        n_e2e = max(1, min(args.steps, 500))
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        for st in (s_comp, s_out):
            st.wait_event(e0)
        for i in range(n_e2e):
            e2e_step(i)
        for st in (s_in, s_comp):
            s_out.wait_stream(st)
        e1.record(s_out)
        barrier()
        e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        e2e = {"value": whole_job_rate(world, p.T, n_e2e, e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": xh.numel() * xh.element_size(),
               "d2h_bytes_per_step": yhs[0].numel() * yhs[0].element_size(), "steps": n_e2e,
               "ms_per_step": e_ms / n_e2e,
               "pipeline": f"{NB} buffer sets; copy-in, compute and copy-out on three streams"}

    if rank != 0:
        return None

    pk, pk_kind = peaks()
    # the fused step (OQ_FUSED_STEP=1) runs quantize and GEMM in one kernel: its time stands
    # for both
    fused_step = "fused" in per_kernel
    if fused_step:
        per_kernel.setdefault("gemm", per_kernel["fused"])
        per_kernel.setdefault("quantize", per_kernel["fused"])
    gemm_ms = statistics.mean(per_kernel.get("gemm", [float("nan")]))
    quant_ms = statistics.mean(per_kernel.get("quantize", [float("nan")]))
    dec_ms = statistics.mean(per_kernel["decode"]) if "decode" in per_kernel else None
    flops = 2.0 * p.T * p.d * p.out
    gemm_tf = flops / (gemm_ms * 1e-3) / 1e12
    traffic, traffic_src = profile_traffic(
        f"k2_gemm_{'acodes_' if acodes else 'wcodes_' if wcodes else ''}{p.name}.ncu.csv",
        GEMM_SOURCES)
    in_bytes = 2 if p.dtype == torch.bfloat16 else 4
    # K1's algorithmic bytes are the method's: x in, the packed codes and s out, T (in*d +
    # d*ba/8 + 4).  What this design moves besides (the fp16 centroids K1 writes for the GEMM
    # instead of the codes on the one-call path, and the weight decode it may take on) is
    # reported separately as design bytes, not counted as algorithmic.
    q_bytes = p.T * (in_bytes * p.d + p.d * p.bits_a // 8 + 4)
    design_bytes = p.T * (in_bytes * p.d + (2 * p.d if direct else p.d * p.bits_a // 8) + 4)
    # with 2/4-bit weights the one-call path's K1 also decodes the weight codes (no decode
    # launch)
    fused_dec = args.api == "forward" and (direct or acodes) and dec_ms is None and not wcodes
    if fused_dec:
        design_bytes += p.out * p.d * (p.bits_w / 8 + 2)
    q_gbs = q_bytes / (quant_ms * 1e-3) / 1e9
    q_traffic, q_traffic_src = profile_traffic(
        f"k1_rotquant_{'codes_' if acodes else ''}{p.name}.ncu.csv", K1_SOURCES)
    out = {
        "metric": METRIC,
        "value": whole_job_rate(world, p.T, args.steps, ms_max),
        "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_max / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16xf16->f32 (gemm), f32 (quantize)",
        "data": "synthetic",
        "config": workload_config(p, world),
        "api": ("oq_quantized_linear (one call; x_codes stay on chip)" if args.api == "forward"
                else "oq_quantize_act + oq_linear"),
        "kernels_ms_mean": ({"fused_step": gemm_ms, "decode": dec_ms,
                             "counter_reset": (statistics.mean(per_kernel["aux"])
                                               if "aux" in per_kernel else None)}
                            if fused_step else
                            {"quantize": quant_ms, "decode": dec_ms, "gemm": gemm_ms}),
        "gemm_a_operand": ("4-bit codes, decoded in the GEMM's shared memory" if acodes else
                           "fp16 centroids written by the quantizer" if direct else
                           "fp16 centroids from the decode prepass"),
        "gemm_b_operand": ("4-bit codes, decoded in the GEMM's shared memory" if wcodes else
                           "fp16 centroids from the weight decode"),
        "roofline": {
            "kernel": ("k3_fused (rotate+quantize stage and tcgen05 cta_group::2 GEMM in one "
                       "persistent kernel; its time covers both)" if fused_step else
                       "k2_gemm_pair (tcgen05 cta_group::2 kind::f16, 256x256x64 tiles per "
                       "CTA pair" + (", 4-bit A codes decoded in shared memory)" if acodes
                                    else ", 4-bit B codes decoded in shared memory)" if wcodes
                                    else ")")),
            "bound": "tensor", "achieved": gemm_tf,
            "peak": pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]),
            "peak_note": f"{pk_kind} dense bf16 burst (fp16 kind::f16 runs at the bf16 rate)",
            "unit": "TFLOP/s",
            "frac": gemm_tf / pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]),
            # the per-kernel events come from 400 back-to-back steps, long enough for the
            # power cap to act: the measured sustained peak is the other fair denominator
            "frac_of_sustained": gemm_tf / pk.get("bf16_tflops_sustained",
                                                  FALLBACK_PEAKS["bf16_tflops_sustained"]),
            "traffic": traffic, "traffic_source": traffic_src,
            "algorithmic_per_launch": flops,
        },
        "roofline_quantize": {
            "kernel": "k1_rotquant (" + ("fp16-operand output" if direct else "codes output")
                      + (" + fused weight decode)" if fused_dec else ")"),
            "bound": "hbm", "achieved": q_gbs,
            "peak": pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]), "unit": "GB/s",
            "frac": q_gbs / pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]),
            "frac_of_8TBps_nominal": q_gbs / 8000.0,
            "algorithmic_bytes_per_launch": q_bytes,
            "algorithmic_bytes_rule": "T * (in_bytes*d + d*bits_a/8 + 4): x in, codes and s out",
            "design_bytes_per_launch": design_bytes,
            "design_gbs": design_bytes / (quant_ms * 1e-3) / 1e9,
            "traffic": q_traffic, "traffic_source": q_traffic_src,
        },
        "quantize_codes_output": (None if codes_q_ms is None else {
            "kernel": "k1_rotquant (packed-code output, oq_quantize_act)",
            "note": "context only, not part of the step: the same K1 on the same rows doing "
                    "only the method's work; CUDA events over 50 launches queued behind a GPU "
                    "spin",
            "ms": codes_q_ms,
            "achieved_gbs": q_bytes / (codes_q_ms * 1e-3) / 1e9,
            "frac": q_bytes / (codes_q_ms * 1e-3) / 1e9 / pk.get("hbm_gbs",
                                                                  FALLBACK_PEAKS["hbm_gbs"]),
        }),
        "gpu_launches": launches,
        "timing": f"value/ms_per_step: {timing_mode} of the step; kernels_ms_mean and the "
                  f"rooflines: CUDA events around each kernel of {n_k} eager steps queued "
                  "behind a GPU spin (device time, not host gaps); on the one-call path "
                  + ("K1 also decodes the 4-bit weights (no decode launch)" if fused_dec else
                     "the decode (weights) runs on a side stream beside K1, so its event "
                     "time includes that overlap"),
        "eager_ms_per_step": eager_ms / args.steps,
        "host_ms_per_step_eager": host_ms / args.steps,
        "clocks": clock_info,
    }
    if fused_step:
        out["roofline_quantize"] = {
            "kernel": "the rotate+quantize stage inside k3_fused",
            "note": "no separate time: the stage runs beside the GEMM in the same kernel",
            "algorithmic_bytes_per_launch": q_bytes}
    if e2e:
        out["e2e"] = e2e
    return out


def run_sweep(args, dev):
    """K1 over the activation sweep: d x h x activation bits x T, bf16 N(0,1) rows with 1 %
    channels x50.  Rows are a 4096-row synthetic block tiled to T (K1's cost does not depend
    on the values), rotated over buffer sets larger than the L2 when they fit in 8 GB; the
    time per launch is the CUDA-event mean over `steps` launches after `warmup`."""
    from calibration_free_bit_b200 import build as B
    B.build()
    from calibration_free_bit_b200 import oq

    pk, pk_kind = peaks()
    hbm = pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    rows_out = []
    blocks = {}
    for sp in synth.sweep_points():
        d, h, bits, T = sp.d, sp.h, sp.bits_a, sp.T
        if d not in blocks:
            blocks[d] = synth.activations(synth.sweep_projection(d, 128, 4, 4096)).to(dev)
        blk = blocks[d]
        x = blk.repeat((T + blk.shape[0] - 1) // blk.shape[0], 1)[:T].contiguous()
        one = T * d * 2
        nb = 1 if one > 2e9 else max(1, min(8, int(400e6 // max(one, 1)) + 1))
        xs = [x] + [x.clone() for _ in range(nb - 1)]
        r = oq.oq_build_rpbh(d, h, 0)
        ca = oq.oq_lloyd_max(d, bits)
        codes = torch.empty((T, d * bits // 8), dtype=torch.uint8, device=dev)
        s = torch.empty(T, device=dev)
        n = max(3, min(args.steps, 50 if T >= 4096 else 200))
        for i in range(max(3, min(args.warmup, 5))):
            oq.oq_quantize_act(r, ca, xs[i % nb], codes, s)
        torch.cuda.synchronize()
        # the n launches are captured once in a CUDA graph and replayed, so the time is the
        # device's (back-to-back launches), not the host's call rate
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(n):
                oq.oq_quantize_act(r, ca, xs[i % nb], codes, s)
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        oq.oq_check()
        del g
        us = e0.elapsed_time(e1) / n * 1e3
        byts = T * (2 * d + d * bits // 8 + 4)
        gbs = byts / (us * 1e-6) / 1e9
        row = {"d": d, "h": h, "bits_a": bits, "T": T, "k1_us": round(us, 3),
               "timing": f"CUDA-graph replay of {n} back-to-back launches",
               "gbs": round(gbs, 1), "frac": round(gbs / hbm, 4), "tokens_per_s": T / (us * 1e-6)}
        rows_out.append(row)
        print(json.dumps(row), flush=True)
        del xs, x, codes, s
    big = [r_ for r_ in rows_out if r_["T"] == 65536]
    print(json.dumps({"sweep": "k1 codes output", "points": len(rows_out), "peak_gbs": hbm,
                      "peak_kind": pk_kind,
                      "T65536_frac_min": min(r_["frac"] for r_ in big) if big else None,
                      "T65536_frac_max": max(r_["frac"] for r_ in big) if big else None}),
          flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    p = synth.get(args.workload)[args.proj]

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, p)), flush=True)
        return

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if args.sweep:
        if rank == 0:
            run_sweep(args, dev)
        return
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    try:
        out = run_ours(args, p, rank, world, dev)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                out["cpu_baseline"] = cpu_baseline(p)
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
