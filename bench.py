#!/usr/bin/env python3
"""Throughput of the fused quantized gated Delta-rule decode step on B200.

One step = one decode token for every (sequence, head) tile of the workload: unpack and
dequantise the packed recurrent state, gated Delta update, readout, refit of the dual-axis
scales and repack -- one launch of the fused kernel. The default workload is the largest
single-GPU decode configuration: the high-concurrency 4-bit layer (B=1024 sequences, H=16 heads,
d_k=d_v=128, per-key-row widths from {2, 4, 8} averaging 4 bits, lifetime-aware Lagrangian
allocation), on seeded synthetic data. The FP32-state and uniform rowwise-INT8 comparison kernels
are timed in the same run on identical inputs; the long-rollout workload also reports the output
drift of the quantized state against the FP32 state over its T steps.

Timing: R state replicas (independent layers of the same shape) are stepped round-robin so
that more than the 126 MB L2 is touched between two uses of a replica; one round of R
launches is captured in a CUDA graph and replayed; CUDA events on the launching stream bracket
the K timed steps, after W untimed warm-up steps, with a barrier + synchronize on both sides;
the K steps are timed five times and the median is reported. Under torchrun every rank runs its
own replicas (weak scaling, no collective on the data path) and the time is the maximum over
ranks; ``--gpus N`` without torchrun's environment starts N ranks itself.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import json
import os
import shutil
import statistics
import subprocess
import sys
import tempfile
import time
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "quantized delta-rule decode: state updates/s and HBM GB/s vs ~8 TB/s peak"
UNIT = "state-updates/s"
L2_BYTES = 126 * 2 ** 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=16)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=3,
                    help="synthetic workload index (0 tiny, 1 GDN 64x32, 2 KDA 256x32, 3 GDN 4-bit 1024x16, "
                         "4 long rollout 128x32)")
    ap.add_argument("--repeats", type=int, default=5, help="timed repetitions of the K steps (median reported)")
    ap.add_argument("--no-comparisons", action="store_true",
                    help="leave out the FP32-state and INT8 comparison kernels")
    ap.add_argument("--drift-steps", type=int, default=0,
                    help="rollout steps of the drift figure (0: the workload's T; long-rollout workload only)")
    ap.add_argument("--replicas", type=int, default=0, help="state replicas cycled (0 = enough to exceed L2)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--cpu-threads", type=int, default=0, help="oracle threads for cpu_baseline (0 = all cores)")
    ap.add_argument("--kernel", choices=["quant", "split", "prefill", "fp32", "int8", "leap"], default="quant",
                    help="quant: the fused step; split: the split-form ablation; prefill: a chunk of --chunk "
                         "tokens per launch; fp32 / int8: comparison states")
    ap.add_argument("--chunk", type=int, default=64, help="tokens per prefill chunk (--kernel prefill)")
    ap.add_argument("--window", type=int, default=16, help="tokens per window of the per-window 8-bit state "
                                                            "(--kernel leap)")
    ap.add_argument("--prefill-form", choices=["auto", "seq", "wy"], default="auto",
                    help="prefill chunk form: the library's choice, the sequential register-tile form, "
                         "or the chunked WY form on the tensor cores")
    ap.add_argument("--e2e-steps", type=int, default=400)
    return ap.parse_args()


def kernel_revision() -> str:
    """First 16 hex digits of the sha256 of the fused decode kernel's sources."""
    import hashlib
    csrc = ROOT / "recurrent_state_quantization_gated_b200" / "csrc"
    data = b"".join((csrc / f).read_bytes() for f in ("stepq_decode.cu", "stepq_device.cuh", "stepq_tile.cuh"))
    return hashlib.sha256(data).hexdigest()[:16]


def _profile(workload_name: str):
    """Figures of the committed ncu summary of the fused kernel on this workload
    (profiles/decode_kernel_<workload>.md): {"traffic": DRAM bytes read + written per launch,
    "instr_per_element": lane instructions per state element}, each None when absent or when
    the kernel's source has changed since the capture (its revision line no longer matches)."""
    out = {"traffic": None, "instr_per_element": None}
    p = ROOT / "profiles" / f"decode_kernel_{workload_name}.md"
    if not p.exists():
        return out
    rev = read = write = per_elem = None
    for line in p.read_text().splitlines():
        if "Kernel source revision" in line:
            rev = line.rsplit(":", 1)[-1].strip()
        cells = [c.strip() for c in line.split("|")]
        if len(cells) < 3:
            continue
        if cells[1].startswith("dram__bytes_read.sum per launch"):
            read = float(cells[2].split()[0].replace(",", ""))
        if cells[1].startswith("dram__bytes_write.sum per launch"):
            write = float(cells[2].split()[0].replace(",", ""))
        if cells[1].startswith("lane instructions per element"):
            per_elem = float(cells[2].split()[0])
    if rev != kernel_revision():
        return out
    if read is not None and write is not None:
        out["traffic"] = read + write
    out["instr_per_element"] = per_elem
    return out


def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def alu_roofline(elements_per_s, clocks, per_elem):
    """The issue-rate roofline beside the HBM one: lane instructions per second against
    148 SMs x 4 schedulers x 32 lanes x the SM clock seen during the timed region."""
    mhz = (clocks or {}).get("sm_mhz") or 1965.0
    peak = 148 * 4 * 32 * mhz * 1e6
    if per_elem is None:
        return {"bound": "alu", "achieved": None, "peak": peak, "unit": "lane-instr/s", "frac": None,
                "instr_per_element": None}
    achieved = per_elem * elements_per_s
    return {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "lane-instr/s", "frac": achieved / peak,
            "instr_per_element": per_elem}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.tmp = None

    def __enter__(self):
        if shutil.which("nvidia-smi") is None:
            return self
        self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                      "--format=csv,noheader,nounits", "-lms", "20"],
                                     stdout=self.tmp, stderr=subprocess.DEVNULL)
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if getattr(self, "_summary", None) is not None:
            return self._summary
        self._summary = self._read()
        return self._summary

    def _read(self):
        if self.tmp is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in Path(self.tmp.name).read_text().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smmax=float(parts[2]), power=float(parts[3]),
                                 hw=parts[5], hwth=parts[6], swth=parts[7], swpc=parts[8]))
            except ValueError:
                continue
        os.unlink(self.tmp.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [r for r in rows if r["power"] > 200.0] or rows
        reasons = set()
        for r in loaded:
            for key, name in (("hw", "hw_slowdown"), ("hwth", "hw_thermal_slowdown"),
                              ("swth", "sw_thermal_slowdown"), ("swpc", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded), "sm_max_mhz": max(r["smmax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(loaded)}


def algorithmic_bytes(layout_bps: int, B: int, H: int, d: int, gate_per_channel: bool, kernel: str) -> int:
    """Bytes a launch must move: state read + write, scales read + write, q/k/v, beta, gate, o.
    The per-head bit map, row-impact vector and head offsets (L2-resident) are not counted."""
    tiles = B * H
    qkv = 3 * 2 * d
    gate = 4 * d if gate_per_channel else 4
    small = tiles * (qkv + 4 + gate + 4 * d)
    if kernel == "quant":
        return 2 * B * layout_bps + tiles * 2 * (2 * d + 2 * d) + small
    if kernel.startswith("prefill"):   # the state once per chunk; every token's inputs and readout
        C = int(kernel.split(":")[1])
        return 2 * B * layout_bps + tiles * 2 * (2 * d + 2 * d) + C * small
    if kernel == "split":   # the fused step's bytes + X written, read by the fit, read by the pack + r, c re-read
        return 2 * B * layout_bps + tiles * 2 * (2 * d + 2 * d) + small + tiles * (3 * 4 * d * d + 4 * d)
    if kernel == "int8":
        return tiles * 2 * (d * d + 2 * d) + small
    if kernel.startswith("leap"):   # one token on the per-window 8-bit state, averaged over a window
        W = int(kernel.split(":")[1])
        entry = 2 * d + 4 * d + 4                       # a buffered key (bf16), u (fp32) and log gate
        per_tile = (d * d + 2 * d) + entry + (W - 1) / 2 * entry + (d * d + 2 * d + W * entry) / W
        return int(tiles * per_tile) + small
    return tiles * 2 * (4 * d * d) + small


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time: every rank takes part (same collective in the same order)."""
    if world == 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, tiles_per_rank: int, steps: int, ms: float) -> float:
    """Tile updates per second of the whole job: every rank steps its own replica of the
    workload (no data-path exchange), timed by the slowest rank."""
    return world * tiles_per_rank * steps / (ms * 1e-3)


def workload_config(wl, bits, kernel: str, world: int, chunk: int = 1, prefill_form: str = "auto") -> dict:
    extra = {"chunk": chunk, "prefill_form": prefill_form} if kernel == "prefill" else {}
    if kernel == "leap":
        extra = {"window": chunk, "format": "rowwise-absmax INT8 between windows"}
    return {"workload": wl.name, "kernel": kernel, **extra, "B": wl.B, "H": wl.H, "d_k": wl.d, "d_v": wl.d,
            "bits_mean": float(np.asarray(bits, dtype=np.float64).mean()), "allocation": wl.alloc,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


def run_reference(args, wl, budget_s: float = 90.0):
    """The oracle (plain C, host cores) on a bounded sample of the same workload: every step
    decodes B' sequences x H heads, B' chosen so the whole run stays within ``budget_s``."""
    import oracle
    from recurrent_state_quantization_gated_b200 import synth
    cores = len(os.sched_getaffinity(0))
    # The oracle's own offline calibration of the workload (row impact, distortions on the
    # initial states, allocation), as the GPU arm does with the CUDA library.
    bits, w = oracle.calibrate(wl.alloc, wl.candidates, wl.nominal_bits, synth.initial_state(wl),
                               synth.calib_tokens(wl), n_pivots=wl.n_pivots)
    if bits is None:
        bits = synth.half_bits(wl)

    def state(seqs):
        S0 = synth.initial_state(wl, seqs)
        r, c = oracle.fit_scales(S0, w, bits, nthreads=cores)
        return oracle.pack_state(S0, bits, r, c, nthreads=cores), r, c

    probe = list(range(min(wl.B, 2)))
    packed, r, c = state(probe)
    t0 = time.perf_counter()
    oracle.decode_step(synth.tokens(wl, 0, seqs=probe), bits, w, packed, r, c, nthreads=cores)
    rate = len(probe) * wl.H / (time.perf_counter() - t0)            # tiles per second
    nseq = int(budget_s * rate / ((args.steps + args.warmup) * wl.H))
    seqs = list(range(max(1, min(wl.B, nseq))))
    packed, r, c = state(seqs)
    tiles = len(seqs) * wl.H
    # The workload's inputs repeat with period T: each distinct step is drawn once, before the
    # loop (a draw generates the whole batch and keeps the sample, about 0.3 s on the largest
    # workload, which per step would dominate the run).
    toks = {}
    times = []
    for step in range(args.warmup + args.steps):
        ts = step % wl.T
        if ts not in toks:
            toks[ts] = synth.tokens(wl, ts, seqs=seqs)
        tok = toks[ts]
        t0 = time.perf_counter()
        packed, r, c, _ = oracle.decode_step(tok, bits, w, packed, r, c, nthreads=cores)
        dt = time.perf_counter() - t0
        if step >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = tiles * len(times) / total
    sample = f"{len(seqs)} of {wl.B} sequences x {wl.H} heads ({tiles} tiles) per step, {len(times)} timed steps"
    return dict(value=value, ms_per_step=1e3 * total / len(times), cores=cores, sample=sample, bits=bits)


def cpu_baseline(wl, bits, w, seconds, threads=0):
    """The oracle as it stands, timed on the host cores over a bounded sample of the workload:
    16 sequences x all heads per step, the calibrated bit map and row weights, inputs drawn
    before the timed loop."""
    import oracle
    from recurrent_state_quantization_gated_b200 import synth
    cores = threads if threads > 0 else len(os.sched_getaffinity(0))
    seqs = list(range(min(wl.B, 16)))
    S0 = synth.initial_state(wl, seqs)
    w = np.ascontiguousarray(w, dtype=np.float32)
    r, c = oracle.fit_scales(S0, w, bits, nthreads=cores)
    packed = oracle.pack_state(S0, bits, r, c, nthreads=cores)
    toks = [synth.tokens(wl, t, seqs=seqs) for t in range(8)]
    tiles = len(seqs) * wl.H
    steps, t0 = 0, time.perf_counter()
    while True:
        packed, r, c, _ = oracle.decode_step(toks[steps % len(toks)], bits, w, packed, r, c, nthreads=cores)
        steps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return {"value": tiles * steps / el, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{steps} decode steps of {len(seqs)} sequences x {wl.H} heads ({tiles} tiles), "
                      f"{'OpenMP over tiles' if cores > 1 else 'one thread'}, {el:.1f} s"}


def relaunch(args) -> int:
    """``--gpus N`` (N > 1) outside torchrun: start N ranks of this script on this node (one
    process per GPU), with the same arguments; rank 0 prints the line."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), str(Path(__file__).resolve()), *sys.argv[1:]]
    return subprocess.call(cmd)


def _drift_tokens(index_t):
    """Packed inputs of step t of workload `index` (process-pool worker of the drift rollout)."""
    from recurrent_state_quantization_gated_b200 import runtime, synth
    index, t = index_t
    return runtime.pack_tokens(synth.tokens(synth.workload(index), t))


def timed_rounds(launch_round, round_len, warmup, steps, repeats, stream, world, barrier, clock=None):
    """Captures one round of launches (`launch_round()`, `round_len` steps) in a CUDA graph,
    replays ceil(warmup / round_len) rounds untimed, then times ceil(steps / round_len) rounds
    `repeats` times with CUDA events on the stream (barrier + synchronize around each), the
    slowest rank's time each. Returns (K steps per repetition, warm-up steps, [ms per repetition])."""
    import torch
    with torch.cuda.stream(stream):
        launch_round()                       # outside capture first (kernel attributes, occupancy)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        launch_round()
    rounds_warm = max(1, -(-warmup // round_len))
    rounds = max(1, -(-steps // round_len))
    with torch.cuda.stream(stream):
        for _ in range(rounds_warm):
            graph.replay()
    stream.synchronize()
    times = []
    if clock is not None:          # clocks sampled over every timed repetition
        clock.__enter__()
    try:
        for _ in range(repeats):
            ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            barrier()
            with torch.cuda.stream(stream):
                ev0.record(stream)
                for _ in range(rounds):
                    graph.replay()
                ev1.record(stream)
            stream.synchronize()
            barrier()
            times.append(max_over_ranks(ev0.elapsed_time(ev1), world, "cuda"))
    finally:
        if clock is not None:
            clock.__exit__(None, None, None)
    del graph
    return rounds * round_len, rounds_warm * round_len, times


def main():
    args = parse()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return relaunch(args)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    from recurrent_state_quantization_gated_b200 import synth
    wl = synth.workload(args.workload)

    if args.impl == "reference":
        if rank != 0:
            return 0
        ref = run_reference(args, wl)
        line = {"metric": METRIC, "value": ref["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ref["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
                "config": workload_config(wl, ref["bits"], "quant", world),
                "cpu_baseline": {"value": ref["value"], "unit": UNIT, "cores": ref["cores"], "kind": "oracle",
                                 "sample": ref["sample"]},
                "e2e": {"value": ref["value"], "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    import torch
    import torch.distributed as dist
    from recurrent_state_quantization_gated_b200 import api, runtime

    torch.cuda.set_device(local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local_rank))

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # ---- offline calibration and initial quantisation (untimed) -------------------------
    S0_host = synth.initial_state(wl)
    S0 = torch.from_numpy(S0_host).cuda()
    del S0_host
    cal = synth.calib_tokens(wl)
    cal_dev = {k: (torch.from_numpy(np.ascontiguousarray(v).view(np.int16)).cuda().view(torch.bfloat16)
                   if v.dtype == np.uint16 else torch.from_numpy(np.ascontiguousarray(v)).cuda())
               for k, v in cal.items()}
    if wl.alloc == "half48":
        bits = synth.half_bits(wl)
        w = api.stepq_row_impact(cal_dev["q"], cal_dev["k"], cal_dev["beta"], cal_dev["gate"])
    else:
        bits, w = runtime.calibrate(wl.alloc, wl.candidates, wl.nominal_bits, S0, cal_dev,
                                    n_pivots=wl.n_pivots)
    layout = runtime.Layout.build(bits, wl.d)
    base = runtime.QuantizedState.from_fp32(S0, layout, w)
    tiles = wl.B * wl.H
    kname = {"prefill": f"prefill:{args.chunk}", "leap": f"leap:{args.window}"}.get(args.kernel, args.kernel)
    bytes_launch = algorithmic_bytes(layout.bytes_per_seq, wl.B, wl.H, wl.d, wl.gate_per_channel, kname)
    LW = args.window if args.kernel == "leap" else 1   # launches per replica per round (one window)
    if args.kernel == "leap" and wl.gate_per_channel:
        raise SystemExit("--kernel leap takes scalar gates (workloads 0, 1, 3, 4)")

    # Replicas: enough independent states that > 2x L2 is touched between reuses.
    def replicas_for(per_launch):
        return min(64, args.replicas or max(2, int(np.ceil(2 * L2_BYTES / per_launch))))

    per_rep = bytes_launch
    R = replicas_for(per_rep)
    reps, toks, outs, tok_bufs = [], [], [], []
    side = torch.cuda.Stream() if args.kernel == "split" else None
    x_ws = torch.empty((wl.B, wl.H, wl.d, wl.d), dtype=torch.float32, device="cuda") if side is not None else None
    for i in range(R):
        if args.kernel in ("quant", "split", "prefill"):
            reps.append(dict(packed=base.packed.clone(), r=base.r.clone(), c=base.c.clone()))
        elif args.kernel == "fp32":
            reps.append(dict(S=S0.clone()))
        elif args.kernel == "leap":
            reps.append(dict(win=runtime.WindowState.from_fp32(S0, args.window)))
        else:
            cds, s = api.stepq_int8_quantize_state(S0)
            reps.append(dict(codes=cds, s=s))
        # Each replica's token inputs live in one packed device buffer (q | k | v | beta | gate),
        # filled end to end by one host-to-device copy per step (per window position for leap).
        if args.kernel == "prefill":
            steps = [synth.tokens(wl, (i * args.chunk + t) % wl.T) for t in range(args.chunk)]
            host = {n: np.ascontiguousarray(np.stack([x[n] for x in steps])) for n in steps[0]}
        else:
            host = synth.tokens(wl, i % wl.T)
        if args.kernel == "leap":
            hosts = [synth.tokens(wl, (i * LW + t) % wl.T) for t in range(LW)]
            tok_bufs.append([torch.from_numpy(runtime.pack_tokens(hh)).cuda() for hh in hosts])
            toks.append([runtime.token_views(b_, hh) for b_, hh in zip(tok_bufs[-1], hosts)])
        else:
            tok_bufs.append(torch.from_numpy(runtime.pack_tokens(host)).cuda())
            toks.append(runtime.token_views(tok_bufs[-1], host))
        oshape = (args.chunk, wl.B, wl.H, wl.d) if args.kernel == "prefill" else (wl.B, wl.H, wl.d)
        outs.append(torch.empty(oshape, dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()

    def launch(i, refit=True):
        st, tk, o = reps[i], toks[i], outs[i]
        if args.kernel == "split":
            api.stepq_decode_step_split(tk["q"], tk["k"], tk["v"], tk["beta"], tk["gate"], layout.bits_dev, w,
                                        layout.head_off_dev, layout.bytes_per_seq, st["packed"], st["r"], st["c"],
                                        st["packed"], st["r"], st["c"], o, x_ws, side_stream=side, refit=refit,
                                        pivots=layout.pivots)
            if refit:
                torch.cuda.current_stream().wait_stream(side)   # writeback done before the next step
        elif args.kernel == "prefill":
            api.stepq_prefill_chunk(tk["q"], tk["k"], tk["v"], tk["beta"], tk["gate"], layout.bits_dev, w,
                                    layout.head_off_dev, layout.bytes_per_seq, st["packed"], st["r"], st["c"],
                                    st["packed"], st["r"], st["c"], o, pivots=layout.pivots, mixed=layout.mixed,
                                    form=None if args.prefill_form == "auto" else args.prefill_form)
        elif args.kernel == "quant":
            api.stepq_decode_step(tk["q"], tk["k"], tk["v"], tk["beta"], tk["gate"], layout.bits_dev, w,
                                  layout.head_off_dev, layout.bytes_per_seq, st["packed"], st["r"], st["c"],
                                  st["packed"], st["r"], st["c"], o, pivots=layout.pivots, mixed=layout.mixed,
                                  widths=layout.widths)
        elif args.kernel == "fp32":
            api.stepq_decode_step_fp32(tk["q"], tk["k"], tk["v"], tk["beta"], tk["gate"], st["S"], st["S"], o)
        elif args.kernel == "leap":
            win = st["win"]
            t_ = tk[win.t]
            win.step(t_["q"], t_["k"], t_["v"], t_["beta"], t_["gate"], o)
        else:
            api.stepq_decode_step_int8(tk["q"], tk["k"], tk["v"], tk["beta"], tk["gate"], st["codes"], st["s"],
                                       st["codes"], st["s"], o)

    def one_round():
        for _ in range(LW):
            for i in range(R):
                launch(i)

    stream = torch.cuda.Stream()
    clk = ClockSampler(local_rank)
    K, warm, times = timed_rounds(one_round, R * LW, args.warmup, args.steps, args.repeats, stream, world, barrier,
                                  clock=clk)
    flags = api.stepq_read_device_flags()
    elapsed_ms = statistics.median(times)
    ms_per_step = elapsed_ms / K
    upd = tiles * (args.chunk if args.kernel == "prefill" else 1)   # tile updates per launch
    value = job_throughput(world, upd, K, elapsed_ms)
    achieved_gbs = bytes_launch / (ms_per_step * 1e-3) / 1e9
    peak, peak_kind = peaks()

    # ---- comparison state formats on identical inputs (same initial state, same tokens) ---
    comparisons = None
    if args.kernel == "quant" and not args.no_comparisons:
        comparisons = {}
        quant_bytes = bytes_launch
        for kind in ("fp32", "int8"):
            b_k = algorithmic_bytes(layout.bytes_per_seq, wl.B, wl.H, wl.d, wl.gate_per_channel, kind)
            Rk = replicas_for(b_k)
            sts = []
            for i in range(Rk):
                if kind == "fp32":
                    sts.append(dict(S=S0.clone()))
                else:
                    cds, s_ = api.stepq_int8_quantize_state(S0)
                    sts.append(dict(codes=cds, s=s_))
            o_k = torch.empty((wl.B, wl.H, wl.d), dtype=torch.float32, device="cuda")

            def round_k(kind=kind, sts=sts, o_k=o_k, Rk=Rk):
                for i in range(Rk):
                    tk = toks[i % R]
                    if kind == "fp32":
                        api.stepq_decode_step_fp32(tk["q"], tk["k"], tk["v"], tk["beta"], tk["gate"], sts[i]["S"],
                                                   sts[i]["S"], o_k)
                    else:
                        api.stepq_decode_step_int8(tk["q"], tk["k"], tk["v"], tk["beta"], tk["gate"],
                                                   sts[i]["codes"], sts[i]["s"], sts[i]["codes"], sts[i]["s"], o_k)

            Kk, _, tk_times = timed_rounds(round_k, Rk, args.warmup, max(Rk, args.steps // 4), args.repeats, stream,
                                           world, barrier)
            ms_k = statistics.median(tk_times) / Kk
            gbs_k = b_k / (ms_k * 1e-3) / 1e9
            comparisons[kind] = {
                "value": job_throughput(world, tiles, Kk, statistics.median(tk_times)), "unit": UNIT,
                "ms_per_step": ms_k, "achieved_gbs": gbs_k, "frac": gbs_k / peak, "bytes_per_launch": b_k,
                "replicas": Rk, "steps": Kk,
                "quant_speedup": ms_k / ms_per_step, "quant_bytes_ratio": b_k / quant_bytes,
                "format": "FP32 state" if kind == "fp32" else "rowwise-absmax INT8 codes + FP16 row scales"}
            del sts
        torch.cuda.synchronize()

    split_info = None
    if args.kernel == "split":
        # The first kernel alone (o available, X written): the split form's critical path when
        # the refit and pack are hidden behind other work.
        n1 = 10 * R
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            f0.record(stream)
            for s_ in range(n1):
                launch(s_ % R, refit=False)
            f1.record(stream)
        stream.synchronize()
        ms1 = f0.elapsed_time(f1) / n1
        bytes1 = (wl.B * layout.bytes_per_seq + tiles * 4 * wl.d + tiles * 4 * wl.d * wl.d
                  + tiles * (3 * 2 * wl.d + 4 + (4 * wl.d if wl.gate_per_channel else 4) + 4 * wl.d))
        split_info = {"first_kernel_ms": ms1, "first_kernel_gbs": bytes1 / (ms1 * 1e-3) / 1e9,
                      "first_kernel_bytes": bytes1,
                      "fused_bytes_per_step": algorithmic_bytes(layout.bytes_per_seq, wl.B, wl.H, wl.d,
                                                                wl.gate_per_channel, "quant")}

    # ---- output drift of the quantized state against the FP32 state (long rollout) ---------
    drift = None
    if args.kernel == "quant" and wl.name.startswith("drift"):
        T = args.drift_steps or wl.T
        import multiprocessing as mp
        st_q = dict(packed=base.packed.clone(), r=base.r.clone(), c=base.c.clone())
        S_f = S0.clone()
        o_q = torch.empty((wl.B, wl.H, wl.d), dtype=torch.float32, device="cuda")
        o_f = torch.empty_like(o_q)
        num = torch.empty(T, dtype=torch.float64, device="cuda")
        den = torch.empty(T, dtype=torch.float64, device="cuda")
        tb = torch.empty_like(tok_bufs[0])
        host0 = synth.tokens(wl, 0)
        tv = runtime.token_views(tb, host0)
        cores = len(os.sched_getaffinity(0))
        with mp.get_context("spawn").Pool(max(1, min(16, cores))) as pool:
            for t, packed_tok in enumerate(pool.imap(_drift_tokens, [(wl.index, t) for t in range(T)], chunksize=8)):
                tb.copy_(torch.from_numpy(packed_tok))
                api.stepq_decode_step(tv["q"], tv["k"], tv["v"], tv["beta"], tv["gate"], layout.bits_dev, w,
                                      layout.head_off_dev, layout.bytes_per_seq, st_q["packed"], st_q["r"],
                                      st_q["c"], st_q["packed"], st_q["r"], st_q["c"], o_q, pivots=layout.pivots,
                                      mixed=layout.mixed, widths=layout.widths)
                api.stepq_decode_step_fp32(tv["q"], tv["k"], tv["v"], tv["beta"], tv["gate"], S_f, S_f, o_f)
                num[t] = torch.linalg.vector_norm((o_q - o_f).double())
                den[t] = torch.linalg.vector_norm(o_f.double())
        d_t = (num / den).cpu().numpy()
        drift = {"steps": T, "tiles": tiles, "mean": float(d_t.mean()), "final": float(d_t[-1]),
                 "mean_first_256": float(d_t[:256].mean()),
                 "definition": "||O_q(t) - O_fp32(t)||_F / ||O_fp32(t)||_F over every tile, averaged over "
                               "t = 1..T; both states stepped on the GPU from the same initial state and tokens"}
        del st_q, S_f
        torch.cuda.synchronize()
    del S0

    # ---- end to end through the public API with host buffers (H2D inputs, D2H output) ----
    if args.kernel == "prefill":
        host_tok = []
        for e in range(2):
            steps = [synth.tokens(wl, (e * args.chunk + t) % wl.T) for t in range(args.chunk)]
            host_tok.append({n: np.ascontiguousarray(np.stack([x[n] for x in steps])) for n in steps[0]})
    else:
        host_tok = [synth.tokens(wl, t % wl.T) for t in range(8)]
    pinned = [torch.from_numpy(runtime.pack_tokens(tk)).pin_memory() for tk in host_tok]
    o_host = [torch.empty(tuple(outs[0].shape), dtype=torch.float32).pin_memory() for _ in range(2)]
    h2d = pinned[0].numel()
    d2h = o_host[0].numel() * o_host[0].element_size()
    # The host link alone: the step's input copy and readout copy, each timed by itself.
    link = {}
    for name, (dst, src) in (("h2d_gbs", (tok_bufs[0] if args.kernel != "leap" else tok_bufs[0][0], pinned[0])),
                             ("d2h_gbs", (o_host[0], outs[0]))):
        l0, l1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            for _ in range(3):
                dst.copy_(src, non_blocking=True)
            l0.record(stream)
            for _ in range(20):
                dst.copy_(src, non_blocking=True)
            l1.record(stream)
        stream.synchronize()
        link[name] = dst.numel() * dst.element_size() * 20 / (l0.elapsed_time(l1) * 1e-3) / 1e9
    link["bound_ms_per_step"] = max(h2d / (link["h2d_gbs"] * 1e9), d2h / (link["d2h_gbs"] * 1e9)) * 1e3
    # Three streams: inputs in, step, readout out; step s's copies overlap step s-1's work, and
    # buffers are reused R steps later, ordered by events. n_g such steps (each: one H2D copy of
    # the step's inputs, the library call, one D2H copy of its readout) are captured in a CUDA
    # graph, replayed back to back, so that the host's per-call overhead does not pace the loop.
    n_g = R * LW * max(1, -(-16 // (R * LW)))
    reps_e2e = max(1, -(-args.e2e_steps // n_g))
    n_e2e = reps_e2e * n_g
    cs, ds = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_steps(n):
        ev_h = [torch.cuda.Event() for _ in range(R)]
        ev_k = [torch.cuda.Event() for _ in range(R)]
        ev_d = [torch.cuda.Event() for _ in range(R)]
        fork = torch.cuda.Event()
        fork.record(stream)
        cs.wait_event(fork)
        ds.wait_event(fork)
        for s_ in range(n):
            i = s_ % R
            src = pinned[s_ % len(pinned)]
            with torch.cuda.stream(cs):
                if s_ >= R:
                    cs.wait_event(ev_k[i])          # the step that last read toks[i] is done
                dst = tok_bufs[i][reps[i]["win"].t] if args.kernel == "leap" else tok_bufs[i]
                dst.copy_(src, non_blocking=True)   # q, k, v, beta, gate in one copy
                ev_h[i].record(cs)
            with torch.cuda.stream(stream):
                stream.wait_event(ev_h[i])
                if s_ >= R:
                    stream.wait_event(ev_d[i])      # outs[i] has been read back
                launch(i)
                ev_k[i].record(stream)
            with torch.cuda.stream(ds):
                ds.wait_event(ev_k[i])
                o_host[s_ % 2].copy_(outs[i], non_blocking=True)
                ev_d[i].record(ds)
        stream.wait_stream(cs)
        stream.wait_stream(ds)

    with torch.cuda.stream(stream):
        e2e_steps(n_g)                              # once outside capture
    stream.synchronize()
    g_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_e2e, stream=stream):
        e2e_steps(n_g)
    with torch.cuda.stream(stream):
        g_e2e.replay()                              # uploads the graph; untimed
    stream.synchronize()
    e2e_runs = []
    for _ in range(args.repeats):                   # the same count of timed runs as the device number
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps_e2e):
                g_e2e.replay()
            e1.record(stream)
        stream.synchronize()
        barrier()
        e2e_runs.append(max_over_ranks(e0.elapsed_time(e1), world, "cuda"))
    e2e_ms = statistics.median(e2e_runs)
    e2e_value = job_throughput(world, upd, n_e2e, e2e_ms)
    del g_e2e

    line = None
    if rank == 0:
        clocks = clk.summary()
        prof = _profile(wl.name) if args.kernel == "quant" else {"traffic": None, "instr_per_element": None}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": warm,
            "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": {**workload_config(wl, bits, args.kernel, world,
                                         args.window if args.kernel == "leap" else args.chunk, args.prefill_form),
                       "l2": (f"inputs larger than L2: {R} state replicas stepped round-robin, "
                              f"{R * per_rep / 2**20:.0f} MiB touched per round") if R * per_rep > L2_BYTES else
                             (f"inputs in L2 (latency case): {R} state replicas, "
                              f"{R * per_rep / 2**20:.1f} MiB touched per round"),
                       "timing": f"CUDA graph of one round of launches, CUDA events on the launching stream; "
                                 f"K steps timed {args.repeats} times, median"},
            "timing_runs_ms_per_step": [t / K for t in times],
            "elements_per_s": value * wl.d * wl.d,
            "achieved_gbs": achieved_gbs,
            "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": peak, "unit": "GB/s",
                         "frac": achieved_gbs / peak, "peak_kind": peak_kind,
                         "traffic": prof["traffic"],
                         "bytes_per_launch": bytes_launch,
                         "bytes_per_launch_formula": "2*B*bytes_per_seq + B*H*(2*(2d+2d) + 6d + 4 + gate + 4d)"},
            "alu_roofline": alu_roofline(value * wl.d * wl.d, clocks, prof["instr_per_element"])
            if args.kernel == "quant" else None,
            "comparisons": comparisons,
            "drift": drift,
            "gpu_launches": K * (3 if args.kernel == "split" else 1),   # split: first kernel, fit, pack
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": n_e2e, "link": link,
                    "method": f"CUDA graphs of {n_g} steps (each: one H2D copy of the step's inputs from pinned "
                              f"host memory, the library call, one D2H copy of its readout), replayed back to back; "
                              f"{len(e2e_runs)} timed runs, median",
                    "timing_runs_ms_per_step": [t / n_e2e for t in e2e_runs]},
            "device_flags": flags,
            "split": split_info,
            "clocks": clocks,
        }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        if not args.no_cpu_baseline and world == 1 and args.kernel == "quant":
            w_host = w.detach().cpu().numpy() if hasattr(w, "detach") else np.asarray(w)
            half = max(1.0, args.cpu_seconds / 2)
            cb = cpu_baseline(wl, bits, w_host, half, args.cpu_threads)
            cb["single_thread"] = cpu_baseline(wl, bits, w_host, half, 1)
            line["cpu_baseline"] = cb
        else:
            line["cpu_baseline"] = None
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
