"""Throughput of the GPTQ hot path: weights quantized per second.

One step = one pass of the whole path over every problem of the workload:
  for every Hessian: zero H, gptq_hessian_accumulate (K1), gptq_prepare (K2),
  gptq_quantize (ingest, K3/K4 per block, K5).
A problem is one Hessian with every row that shares it: in a decoder layer the
q/k/v/o/gate/up projections read the layer input (one stack on one H) and
down_proj reads SiLU(gate)·up (its own H).  The decoder workloads quantize
every layer of the stack per step.  Default workload: the TinyLlama-1.1B-shaped
stack, 22 layers × (15872×2048 on one H + 2048×5632), 2048 cone-structured
calibration tokens, 4-bit, group 128, block 128, damp 0.01.  The problems run
on --lanes streams (each lane its share one after the other); the step is
captured once as a CUDA graph and replayed.

    python bench.py --gpus N --steps K --warmup W [--config C] [--bits B]
                    [--layers L] [--lanes S] [--impl reference]

Multi-GPU: one process per GPU (torchrun); every rank quantizes its own,
independent stack (no collective on the data path: weak scaling); timing is
the max over ranks of the device time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from workloads import CONFIGS, normal_matrix, problems_for  # noqa: E402

METRIC = "GPTQ weights quantized/sec (params/s incl. Hessian) & % of roofline, 1 B200"
L2_BYTES = 126 * 1024 * 1024


# ---------------------------------------------------------------- host helpers

def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def layer_for_rank(rank: int) -> int:
    """Each rank quantizes its own, independent layer (seed block = rank)."""
    return rank


def max_over_ranks(value: float, world: int, device=None) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, world: int, device=None) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def workload_name(cid: int, bits: int, order: str | None = None,
                  static_groups: bool = False, layers: int = 1) -> str:
    c = CONFIGS[cid]
    tail = ("" if order is None else f", {order} order") + (", static groups" if static_groups
                                                            else "")
    if c["kind"] == "decoder":
        h, kv, it = c["hidden"], c["kv"], c["inter"]
        rows = 2 * h + 2 * kv + 2 * it
        scope = "per layer" if layers == 1 else f"{layers} layers per step"
        return (f"{c['name']}: q/k/v/o/gate/up {rows}x{h} on one H + down {h}x{it}, "
                f"T={c['T']} cone tokens, {bits}-bit g128 b128 damp0.01, {scope}{tail}")
    return f"{c['name']}: W {c['m']}x{c['n']}, T={c['T']}, {bits}-bit g128 b128 damp0.01{tail}"


def stack_layers(args) -> int:
    """Layers quantized per step: every layer of a decoder stack (--layers
    limits it), one for the single and stress layers."""
    c = CONFIGS[args.config]
    if c["kind"] != "decoder":
        return 1
    return max(1, min(int(args.layers or c["layers"]), c["layers"]))


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of the GPU's clocks during the timed region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            sel = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", sel, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------- roofline

def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "sm_max_mhz": 1965.0}, "fallback"


def fp64_peak_tflops(sm_mhz: float) -> float:
    """B200 float64 from the data sheet's unit counts: 148 SMs × 64 FP64 FMA
    lanes × 2 flops × clock (context beside the probed figure)."""
    return 148 * 64 * 2 * sm_mhz * 1e6 / 1e12


PROBE_ITERS = {"fp64": (0, 32768), "tf32": (1, 65536), "bf16": (2, 65536),
               "fp64_8warps_per_sm": (3, 32768)}


def probe_peaks(device) -> dict:
    """Measured pipe rates (TFLOP/s) from the library's peak probes: float64
    tensor-core products, tcgen05 TF32 and tcgen05 bf16 (a check of the
    probe against the cuBLAS bf16 figure).  Each probe runs ~20 ms; best of 3
    launches after one warm-up, CUDA events on the launching stream."""
    from post_weight_quantization_08_b200 import _binding as b
    info = torch.zeros(2, dtype=torch.int32, device=device)
    sink = torch.zeros(1, dtype=torch.float64, device=device)
    s = torch.cuda.current_stream(device)
    out = {}
    for name, (kind, iters) in PROBE_ITERS.items():
        best = None
        for rep in range(4):
            a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(s)
            flops = b.gptq_peak_probe(kind, iters, info, sink, s)
            e.record(s)
            e.synchronize()
            if rep > 0:
                t = flops / (a.elapsed_time(e) / 1e3) / 1e12
                best = t if best is None else max(best, t)
        st, _ = b.gptq_check(info, s)
        if st != 0:
            raise RuntimeError(f"peak probe {name}: device status {st}")
        out[name] = round(best, 1)
    return out


def chol_tile_flops(n: int) -> float:
    """Floating-point operations the factorisation executes: its 64×64 tile
    products (padded to whole tiles) and the diagonal tiles' Cholesky and
    inverse (2·64³/3 each)."""
    N = -(-n // 64)
    f = 0.0
    for k in range(N):
        r = N - k - 1
        f += (r * (r + 1) // 2 + r * (k + 1) + r + k) * 2 * 64 ** 3
        f += 2 * 64 ** 3 / 3
    return f


def kernel_work(probs, block: int):
    """Algorithmic work per kernel kind for one step: {kind: (unit, amount)}.

    hessian   flops T·n(n+1) (the upper triangle with the diagonal)
    cholesky  flops 2n³/3 (Cholesky of the reversed matrix and its triangular
              inverse; the executed, tile-padded figure is reported beside it)
    sweep     bytes per block: strip read + Err write (4 + 4 B) + codes (1 B)
              per element, the U panel 4·bw², scale + zero 5 B per (row,
              group); on the tensor-core path (n % 4 == 0) also the trailing
              update's bytes (W read + write 8 B per trailing element, Err
              4·m·bw, the U panel 4·bw·N2), since its near columns run in the
              sweep's prologue and its far columns in CTAs of the sweep's launch
    trailing  bytes: the transposed TF32 split of U (12 B per element) on the
              tensor-core path, else the SIMT trailing update's bytes
    pack      bytes: codes 1 B + packed bits/8 B per element, scale/zero
    ingest    bytes: W in (2 or 4 B) + float32 out per element
    prep_order  the min-pivot order only: flops n³/3 (the pivoted float64
              elimination that produces it)
    """
    w = {k: 0.0 for k in ("hessian", "cholesky", "sweep", "trailing", "pack", "ingest",
                          "prep_order")}
    for p in probs:
        m, n, T = p.m, p.n, p.T
        w["hessian"] += T * n * (n + 1)
        w["cholesky"] += 2.0 * n ** 3 / 3.0
        if p.order == "minpivot":
            w["prep_order"] += n ** 3 / 3.0
        ng = -(-n // p.group)
        fused = n % 4 == 0 and n > block
        if fused:
            w["trailing"] += 12 * n * n
        for c0, c1, kw in far_updates(n, block, fused):
            w["sweep" if fused else "trailing"] += 8 * m * (c1 - c0) + 4 * m * kw + 4 * kw * (c1 - c0)
        for j0 in range(0, n, block):
            bw = min(block, n - j0)
            w["sweep"] += 9 * m * bw + 4 * bw * bw + 5 * m * (-(-bw // p.group))
        w["pack"] += m * n + m * n * p.bits / 8 + 5 * m * ng
        w["ingest"] += m * n * (p.W.element_size() + 4)
    units = {"hessian": "TFLOP/s", "cholesky": "TFLOP/s", "prep_order": "TFLOP/s",
             "sweep": "GB/s", "trailing": "GB/s", "pack": "GB/s", "ingest": "GB/s"}
    return {k: (units[k], v) for k, v in w.items()}


SUPER_BLOCKS = 4


def far_updates(n: int, block: int, fused: bool):
    """The trailing-update applications of one quantize call, as (first
    column, end column, K): block b's errors reach block b+1 in its sweep's
    prologue and the rest as listed.  On the tensor-core path with 128-column
    blocks, super-blocks of SUPER_BLOCKS blocks: inside one, block b−1's errors
    reach the rest of the super-block and the block after it; the first block
    of the next super-block's launch applies the whole previous super-block to
    every column past that block."""
    S = SUPER_BLOCKS if (fused and block == 128) else 1
    out = []
    nb = -(-n // block)
    for b in range(1, nb):
        j0 = b * block
        c0 = j0 + min(block, n - j0)
        if b % S != 0:
            c1, kw = min(n, (b // S + 1) * S * block + block), block
        else:
            c1, kw = n, S * block
        if c0 < c1:
            out.append((c0, c1, kw))
    if not fused:
        # off the tensor-core path block b's errors go to the rest in one update
        out = [(b * block + block, n, block) for b in range(nb - 1) if b * block + block < n]
    return out


def trailing_flops(probs, block: int) -> float:
    """Flops of the lazy-batch trailing update, 2·m·bw·N2 per block (the
    sweep launches carry it on the tensor-core path)."""
    f = 0.0
    for p in probs:
        for j0 in range(0, p.n, block):
            bw = min(block, p.n - j0)
            f += 2.0 * p.m * bw * (p.n - j0 - bw)
    return f


def kernel_figures(work, kprof, steps, peaks, src, probed):
    """Per kernel kind: device time per step (the library's event profiler),
    achieved = algorithmic work ÷ time, and the fraction of its peak: HBM copy
    bandwidth and bf16 from MEASURED_PEAKS.json, float64 from the library's
    probe (the data-sheet unit count otherwise).  Returns (kernels, roofline
    of the kind with the largest time)."""
    fp64 = probed.get("fp64") if isinstance(probed, dict) else None
    fp64_src = "fp64 DMMA probe, measured" if fp64 else "fp64 148 SMs x 64 FMA x 2 x max clock"
    fp64 = fp64 or fp64_peak_tflops(peaks.get("sm_max_mhz", 1965.0))
    kernels = {}
    for k, (unit, amount) in work.items():
        if k not in kprof or kprof[k][1] <= 0 or amount <= 0:
            continue
        ms = kprof[k][0] / steps
        if unit == "TFLOP/s":
            ach = amount / (ms / 1e3) / 1e12
            if k == "hessian":
                bound, peak, note = "tensor", peaks["bf16_tflops"], f"bf16 burst, {src}"
            else:
                bound, peak, note = "tensor", fp64, fp64_src
        else:
            ach = amount / (ms / 1e3) / 1e9
            bound, peak, note = "hbm", peaks["hbm_gbs"], f"copy bandwidth, {src}"
        kernels[k] = {"ms_per_step": round(ms, 4), "launches_per_step": kprof[k][1] / steps,
                      "bound": bound, "achieved": round(ach, 2), "unit": unit,
                      "peak": round(peak, 1), "frac": round(ach / peak, 4),
                      "peak_source": note}
    roof = None
    if kernels:
        tot = sum(v["ms_per_step"] for v in kernels.values())
        dom = max(kernels, key=lambda k: kernels[k]["ms_per_step"])
        d = kernels[dom]
        roof = {"kernel": dom, "bound": d["bound"], "achieved": d["achieved"],
                "peak": d["peak"], "unit": d["unit"], "frac": d["frac"],
                "peak_source": d["peak_source"], "launches_per_step": d["launches_per_step"],
                "share": round(d["ms_per_step"] / max(1e-9, tot), 4)}
    return kernels, roof


def source_sha(files) -> str:
    """First 16 hex digits of the SHA-256 of the named csrc files, in order."""
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "post_weight_quantization_08_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, workload: str):
    """DRAM bytes per launch of a kernel kind on a workload, from the committed
    ncu summary (profiles/traffic.json), if its sources are unchanged since
    the capture; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            d = json.load(f)
        for e in d.get("entries", []):
            if e.get("kernel") == kernel and e.get("workload") == workload:
                if source_sha(e["sources"]) == e.get("source_sha"):
                    return e["bytes_per_launch"]
        return None
    except Exception:
        return None


# ---------------------------------------------------------------- the GPU arm

def est_cost(p) -> float:
    """Relative device time of one problem, for spreading problems over lanes:
    the float64 factorisation (2n³/3 at ≈ 30 TFLOP/s) plus the 3×TF32 trailing
    update (3·m·n² at ≈ 1 PFLOP/s)."""
    return (2.0 / 3.0) * p.n ** 3 / 30e12 + 3.0 * p.m * p.n * p.n / 1e15


def lane_plans(probs, lanes):
    """Problems per lane for the Hessians and factorisations: most expensive
    first (est_cost), each to the lane with the least work so far."""
    nl = max(1, min(int(lanes), len(probs)))
    plans, load = [[] for _ in range(nl)], [0.0] * nl
    for k in sorted(range(len(probs)), key=lambda k: -est_cost(probs[k])):
        ln = min(range(nl), key=lambda i: load[i])
        plans[ln].append(k)
        load[ln] += est_cost(probs[k])
    return plans


def quantize_order(probs):
    """Order of the quantize calls: the longest sweep chain (most blocks)
    first, then the most rows."""
    return sorted(range(len(probs)), key=lambda k: ((-probs[k].n) // probs[k].block, -probs[k].m))


def factor_workers(arg, nprobs, device):
    """Most worker CTAs a factorisation may use: ``arg`` when given (0: every
    SM but one); by default (-1) three fifths of the SMs when the step has
    eight or more problems, so that sweeps of factorised problems run beside
    the next factorisation, and every SM but one otherwise."""
    if arg >= 0:
        return int(arg)
    if nprobs < 8:
        return 0
    return int(0.6 * torch.cuda.get_device_properties(device).multi_processor_count)


class Job:
    """Device buffers of a list of problems (every layer of a stack), allocated
    once, and the step's schedule.  Hessians and factorisations run on
    ``lanes`` streams: each lane takes its share one after the other, the lanes
    side by side; problems go, most expensive first, to the lane with the least
    work so far.  Each problem's quantize then runs on one of ``qstreams``
    streams as soon as its factorisation is done, the longest column sweeps
    first: a quantize is a chain of dependent sweep launches that may hold
    only a few CTAs (a down projection of 2048 rows: 16), so several of them
    side by side fill the GPU where one alone would leave it mostly idle.
    With ``static_groups`` the quantize call fixes every group's parameters
    from the original weights (gptq_quantize_static)."""

    OUTS = ("qweight", "scale", "zero", "g_idx", "loss")

    def __init__(self, probs, device, lanes, static_groups=False, qstreams=8):
        import post_weight_quantization_08_b200 as g
        self.g = g
        self.probs = probs
        self.dev = device
        self.static_groups = bool(static_groups)
        self.items = []
        for p in probs:
            m, n = p.m, p.n
            ng = -(-n // p.group)
            nw = -(-n * p.bits // 32)
            self.items.append({
                "p": p,
                "X": p.X.to(device).contiguous(),
                "W": p.W.to(device).contiguous(),
                "H": torch.zeros(n, n, dtype=torch.float32, device=device),
                "perm": torch.empty(n, dtype=torch.int32, device=device),
                "U": torch.empty(n, n, dtype=torch.float32, device=device),
                "dead": torch.empty(n, dtype=torch.uint8, device=device),
                "info_h": torch.zeros(2, dtype=torch.int32, device=device),
                "info_p": torch.zeros(2, dtype=torch.int32, device=device),
                "info_q": torch.zeros(2, dtype=torch.int32, device=device),
                "ws_p": g.workspace(g.gptq_prepare_workspace_bytes(n), device),
                "ws_q": g.workspace(g.gptq_quantize_workspace_bytes(m, n, p.block), device),
                "qweight": torch.empty(m, nw, dtype=torch.int32, device=device),
                "scale": torch.empty(m, ng, dtype=torch.float32, device=device),
                "zero": torch.empty(m, ng, dtype=torch.uint8, device=device),
                "g_idx": torch.empty(n, dtype=torch.int32, device=device),
                "loss": torch.empty(m, dtype=torch.float32, device=device),
            })
        self.lanes = [{"s": torch.cuda.Stream(device=device), "plan": plan}
                      for plan in lane_plans(probs, lanes)]
        self.cs = torch.cuda.Stream(device=device)            # host copies
        nq = max(1, min(int(qstreams), len(probs)))
        self.qs = [torch.cuda.Stream(device=device) for _ in range(nq)]
        self.qorder = quantize_order(probs)

    def prepare_problem(self, it, s, x_ready=None):
        """Hessian and factorisation of one problem on stream ``s``; ``x_ready``:
        the event after which X is in place."""
        g, p = self.g, it["p"]
        if x_ready is not None:
            s.wait_event(x_ready)
        with torch.cuda.stream(s):
            it["H"].zero_()
        g.gptq_hessian_accumulate(it["X"], it["H"], it["info_h"], s)
        g.gptq_prepare(it["H"], p.damp, p.order, it["perm"], it["U"], it["dead"],
                       it["info_p"], it["ws_p"], s)

    def quantize_problem(self, it, s, w_ready=None, host=None):
        """Quantize of one problem on stream ``s`` (its factorisation done);
        ``w_ready``: the event after which W is in place; ``host``: pinned
        buffers for the results."""
        g, p = self.g, it["p"]
        if w_ready is not None:
            s.wait_event(w_ready)
        g.gptq_quantize(it["W"], it["U"], it["perm"], it["dead"], p.bits, p.group, p.block,
                        it["qweight"], it["scale"], it["zero"], it["g_idx"], it["loss"],
                        None, it["info_q"], it["ws_q"], s, self.static_groups)
        if host is not None:
            with torch.cuda.stream(s):
                for k in self.OUTS:
                    host[k].copy_(it[k], non_blocking=True)

    def run_problem(self, it, s):
        self.prepare_problem(it, s)
        self.quantize_problem(it, s)

    def step(self, main, hosts=None):
        """Fork the lanes and quantize streams off ``main`` and join them back.

        ``hosts``: per problem pinned input/output buffers (the end-to-end
        step).  The host→device copies then run on one copy stream: every
        problem's activations in the order the lanes need them (round r: each
        lane's r-th problem), then the weights in quantize order.  A problem's
        Hessian waits for its activations and its quantize for its weights;
        its results go back to the host on its quantize stream."""
        fork = torch.cuda.Event()
        fork.record(main)
        xr, wr = {}, {}
        if hosts is not None:
            self.cs.wait_event(fork)
            rounds = max(len(lane["plan"]) for lane in self.lanes)
            xorder = [lane["plan"][r] for r in range(rounds) for lane in self.lanes
                      if r < len(lane["plan"])]
            with torch.cuda.stream(self.cs):
                for key, order, dst in (("X", xorder, xr), ("W", self.qorder, wr)):
                    for k in order:
                        self.items[k][key].copy_(hosts[k][key], non_blocking=True)
                        e = torch.cuda.Event()
                        e.record(self.cs)
                        dst[k] = e
        prepared = {}
        joins = []
        for lane in self.lanes:
            s = lane["s"]
            s.wait_event(fork)
            for k in lane["plan"]:
                self.prepare_problem(self.items[k], s, xr.get(k))
                e = torch.cuda.Event()
                e.record(s)
                prepared[k] = e
            e = torch.cuda.Event()
            e.record(s)
            joins.append(e)
        for q, k in enumerate(self.qorder):
            s = self.qs[q % len(self.qs)]
            if q < len(self.qs):
                s.wait_event(fork)
            s.wait_event(prepared[k])
            self.quantize_problem(self.items[k], s, wr.get(k),
                                  hosts[k] if hosts is not None else None)
        for s in self.qs:
            e = torch.cuda.Event()
            e.record(s)
            joins.append(e)
        for e in joins:
            main.wait_event(e)

    def step_serial(self, main):
        """Every problem on ``main``, one after the other (for kernel timing)."""
        for it in self.items:
            self.run_problem(it, main)

    def check(self):
        s = self.lanes[0]["s"]
        for it in self.items:
            for key in ("info_h", "info_p", "info_q"):
                st, idx = self.g.gptq_check(it[key], s)
                if st != 0:
                    raise RuntimeError(f"device reported status {st} at {idx}")


def run_ours(args, rank, world, local):
    import post_weight_quantization_08_b200 as g
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    cfg = CONFIGS[args.config]
    bits = args.bits or cfg["bits"][0]
    nl = stack_layers(args)
    probs = [p for l in range(nl)
             for p in problems_for(args.config, layer=layer_for_rank(rank) * nl + l, bits=bits,
                                   order=args.order)]
    layer = Job(probs, device, args.lanes, args.static_groups, args.qstreams)
    params = sum(p.params for p in probs)
    workers = factor_workers(args.factor_workers, len(probs), device)
    g.lib().gptq_set_factor_workers(workers)
    main = torch.cuda.Stream(device=device)     # non-default: graphs capture here
    torch.cuda.set_stream(main)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)

    for _ in range(args.warmup):
        layer.step(main)
    torch.cuda.synchronize(device)
    layer.check()

    # ---- one step captured as a CUDA graph (every problem, forked lanes)
    graph = None
    launches_per_step = 0
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        c0 = g.gptq_launch_count()
        with torch.cuda.graph(graph, stream=main):
            layer.step(main)
        launches_per_step = g.gptq_launch_count() - c0
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize(device)
        layer.check()

    def run_step():
        if graph is not None:
            graph.replay()
        else:
            layer.step(main)

    # ---- device-resident timed region
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    clocks = ClockSampler(local)
    clocks.start()
    launches0 = g.gptq_launch_count()
    evs = []
    for _ in range(args.steps):
        flush.fill_(1.0)                       # evict L2 between steps
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(main)
        run_step()
        b.record(main)
        evs.append((a, b))
    torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    launches = (g.gptq_launch_count() - launches0) if graph is None else launches_per_step * args.steps
    clk = clocks.stop()
    layer.check()
    dev_ms = sum(a.elapsed_time(b) for a, b in evs)
    dev_ms = max_over_ranks(dev_ms, world, device)
    total_params = sum_over_ranks(params * args.steps, world, device)
    value = total_params / (dev_ms / 1e3)

    # ---- per-kernel durations: the same K steps launched eagerly, every
    # launch bracketed by CUDA events on its own stream
    # (problems one after the other on one stream, so that no kernel's
    # interval includes time spent waiting for the other problem's kernels)
    # (nothing else runs beside a serialised kernel, so the factorisation gets
    # every SM here, as it would alone)
    prof_steps = max(1, min(args.steps, args.profile_steps))
    g.lib().gptq_set_factor_workers(0)
    g.gptq_profile_start(1 << 17)
    for _ in range(prof_steps):
        flush.fill_(1.0)
        layer.step_serial(main)
    torch.cuda.synchronize(device)
    kprof = g.gptq_profile_stop()
    g.lib().gptq_set_factor_workers(workers)

    # ---- end to end: pinned host inputs in, packed results out, every step.
    # The copies are part of the captured step: one copy stream brings in the
    # problems' activations and weights in the order the lanes need them, a
    # problem starts once its activations are in and quantizes once its
    # weights are, and its results go back on its lane's stream.
    hosts = [{"X": it["X"].cpu().pin_memory(), "W": it["W"].cpu().pin_memory(),
              **{k: torch.empty(it[k].shape, dtype=it[k].dtype).pin_memory()
                 for k in Job.OUTS}} for it in layer.items]
    h2d = sum(h["X"].numel() * h["X"].element_size() + h["W"].numel() * h["W"].element_size()
              for h in hosts)
    d2h = sum(h[k].numel() * h[k].element_size() for h in hosts for k in Job.OUTS)
    e2e_graph = None
    if not args.no_graph:
        e2e_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(e2e_graph, stream=main):
            layer.step(main, hosts)

    def e2e_step():
        if e2e_graph is not None:
            e2e_graph.replay()
        else:
            layer.step(main, hosts)

    for _ in range(max(1, args.warmup)):
        e2e_step()
    torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    e2e_ms = 0.0
    for _ in range(args.steps):
        flush.fill_(1.0)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(main)
        e2e_step()
        b.record(main)
        torch.cuda.synchronize(device)
        e2e_ms += a.elapsed_time(b)
    e2e_ms = max_over_ranks(e2e_ms, world, device)
    layer.check()

    # ---- per-kernel figures and the roofline of the dominant kernel
    peaks, src = _peaks()
    try:
        probed = probe_peaks(device)
    except Exception as e:                     # the probes are a measurement aid
        probed = {"error": str(e)[:200]}
    work = kernel_work(probs, probs[0].block)
    kernels, roof = kernel_figures(work, kprof, prof_steps, peaks, src, probed)
    if "cholesky" in kernels:
        # the executed float64 work (whole 64-wide tiles), beside the 2n³/3 of the figures
        tiles = sum(chol_tile_flops(p.n) for p in probs)
        ex = round(tiles / (kernels["cholesky"]["ms_per_step"] / 1e3) / 1e12, 2)
        kernels["cholesky"]["executed_tile_tflops"] = ex
        if roof is not None and roof["kernel"] == "cholesky":
            roof["executed_tile_tflops"] = ex
    wl = workload_name(args.config, bits, args.order, args.static_groups, nl)
    for k, v in kernels.items():
        v["traffic"] = traffic_for(k, wl)
    if roof is not None:
        roof["traffic"] = kernels[roof["kernel"]]["traffic"]

    tot = {k: v[0] for k, v in kprof.items()}
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "params/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dev_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16->f32 Hessian, f64 prepare, f32 sweep",
        "data": "synthetic (seeded cone activations, N(0,0.02^2) weights)",
        "config": {"workload": wl, "params_per_step_per_gpu": params,
                   "global_batch": len(probs) * world, "seq_len": probs[0].T,
                   "parallelism": f"independent layers x{world}",
                   "lanes": len(layer.lanes), "qstreams": len(layer.qs),
                   "factor_workers": workers or "every SM but one",
                   "l2": "flushed between timed steps (256 MB write)",
                   "kernel_figures": "serialised eager pass, the factorisation on every SM",
                   "launch": "CUDA graph replay per step" if graph is not None else "eager launches"},
        "e2e": {"value": round(total_params / (e2e_ms / 1e3), 1), "unit": "params/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": int(launches),
        "roofline": roof,
        "kernels": kernels,
        "kernels_ms_per_step": {k: round(v / prof_steps, 4) for k, v in tot.items() if v > 0},
        "peaks_probed_tflops": probed,
        "clocks": clk,
    }
    return out, probs, params


# ---------------------------------------------------------------- the CHMC frontend

CHMC_METRIC = ("CHMC weights compressed/sec (params/s incl. Hessian, low-rank part and "
               "residual GPTQ) & % of roofline, 1 B200")
CHMC_NITER, CHMC_LAM, CHMC_DAMP, CHMC_BPW, CHMC_GS = 5, 0.05, 0.05, 4.2875, 128


class ChmcLayer:
    """Device buffers of one layer under the CHMC frontend ("Warum Geometrie
    Gewichte nicht komprimiert", Methodik): per weight matrix its rank from the
    bit budget, its test matrix Ω, its factors and residual, and the residual's
    codes with output-channel scales; per Hessian its inverse-Cholesky factor."""

    def __init__(self, probs, device):
        import post_weight_quantization_08_b200 as g
        self.g = g
        self.items = []
        for pi, p in enumerate(probs):
            n = p.n
            it = {"p": p, "X": p.X.to(device).contiguous(),
                  "H": torch.zeros(n, n, dtype=torch.float32, device=device),
                  "perm": torch.empty(n, dtype=torch.int32, device=device),
                  "U": torch.empty(n, n, dtype=torch.float32, device=device),
                  "dead": torch.empty(n, dtype=torch.uint8, device=device),
                  "info_h": torch.zeros(2, dtype=torch.int32, device=device),
                  "info_p": torch.zeros(2, dtype=torch.int32, device=device),
                  "ws_p": g.workspace(g.gptq_prepare_workspace_bytes(n), device),
                  "stream": torch.cuda.Stream(device=device), "parts": []}
            row0 = 0
            for k, (name, rows) in enumerate(p.parts):
                W = p.W[row0:row0 + rows].to(device).contiguous()
                row0 += rows
                r = g.gptq_chmc_rank(rows, n, p.bits, CHMC_GS, CHMC_BPW)
                nw = -(-n * p.bits // 32)
                it["parts"].append({
                    "name": name, "W": W, "r": r,
                    "Om": normal_matrix(n, max(r, 1), 9000 + 100 * pi + k)[:, :r].contiguous().to(device),
                    "Q": torch.empty(rows, max(r, 1), dtype=torch.float32, device=device)[:, :r],
                    "P": torch.empty(max(r, 1), n, dtype=torch.float32, device=device)[:r],
                    "R": torch.empty(rows, n, dtype=torch.float32, device=device),
                    "info_l": torch.zeros(2, dtype=torch.int32, device=device),
                    "ws_l": g.workspace(g.gptq_chmc_workspace_bytes(rows, n, r), device),
                    "qweight": torch.empty(rows, nw, dtype=torch.int32, device=device),
                    "scale": torch.empty(-(-rows // CHMC_GS), n, dtype=torch.float32, device=device),
                    "zero": torch.empty(-(-rows // CHMC_GS), n, dtype=torch.uint8, device=device),
                    "loss": torch.empty(rows, dtype=torch.float32, device=device),
                    "info_q": torch.zeros(2, dtype=torch.int32, device=device),
                    "ws_q": g.workspace(g.gptq_quantize_workspace_bytes(rows, n, p.block), device),
                    "stream": torch.cuda.Stream(device=device),
                })
            self.items.append(it)

    def run_problem(self, it, serial=False):
        """The matrices sharing one H run on streams of their own: each low-rank
        part beside the factorisation (both read only H), each residual's
        quantization once the factor is there (``serial``: all on one stream)."""
        g, p, s = self.g, it["p"], it["stream"]
        with torch.cuda.stream(s):
            it["H"].zero_()
        g.gptq_hessian_accumulate(it["X"], it["H"], it["info_h"], s)
        h_ready = torch.cuda.Event()
        h_ready.record(s)
        for q in it["parts"]:
            qs = s if serial else q["stream"]
            if not serial:
                qs.wait_event(h_ready)
            g.gptq_chmc_lowrank(q["W"], it["H"], p.T, CHMC_LAM, q["Om"], q["r"], CHMC_NITER,
                                q["Q"] if q["r"] > 0 else None, q["P"] if q["r"] > 0 else None,
                                q["R"], q["info_l"], q["ws_l"], qs)
        g.gptq_prepare(it["H"], CHMC_DAMP, "act", it["perm"], it["U"], it["dead"],
                       it["info_p"], it["ws_p"], s)
        prep_done = torch.cuda.Event()
        prep_done.record(s)
        for q in it["parts"]:
            qs = s if serial else q["stream"]
            if not serial:
                qs.wait_event(prep_done)
            g.gptq_quantize_rowgroups(q["R"], it["U"], it["perm"], it["dead"], p.bits, CHMC_GS,
                                      p.block, q["qweight"], q["scale"], q["zero"], q["loss"],
                                      None, q["info_q"], q["ws_q"], qs)
            if not serial:
                e = torch.cuda.Event()
                e.record(qs)
                s.wait_event(e)

    def step(self, main):
        fork = torch.cuda.Event()
        fork.record(main)
        joins = []
        for it in self.items:
            it["stream"].wait_event(fork)
            self.run_problem(it)
            e = torch.cuda.Event()
            e.record(it["stream"])
            joins.append(e)
        for e in joins:
            main.wait_event(e)

    def step_serial(self, main):
        for it in self.items:
            s = it["stream"]
            it["stream"] = main
            try:
                self.run_problem(it, serial=True)
            finally:
                it["stream"] = s

    def check(self):
        for it in self.items:
            for key in ("info_h", "info_p"):
                st, idx = self.g.gptq_check(it[key], it["stream"])
                if st != 0:
                    raise RuntimeError(f"device reported status {st} at {idx}")
            for q in it["parts"]:
                for key in ("info_l", "info_q"):
                    st, idx = self.g.gptq_check(q[key], it["stream"])
                    if st != 0:
                        raise RuntimeError(f"{q['name']}: device reported status {st} at {idx}")


def chmc_work(layer):
    """Algorithmic work per kernel kind for one CHMC step.

    hessian, cholesky as for GPTQ; chmc bytes: W read 2·niter + 3 times (the
    sketch, niter power iterations of two products each, Qᵀ·W, the residual)
    plus the float32 residual written; sweep/ingest/pack as for GPTQ on the
    float32 residual (scale and zero per row group and column)."""
    w = {k: 0.0 for k in ("hessian", "cholesky", "chmc", "sweep", "pack", "ingest")}
    for it in layer.items:
        p = it["p"]
        n, T = p.n, p.T
        w["hessian"] += T * n * (n + 1)
        N = -(-n // 64)
        for k in range(N):
            r = N - k - 1
            w["cholesky"] += (r * (r + 1) // 2 + r * (k + 1) + r + k) * 2 * 64 ** 3
            w["cholesky"] += 2 * 64 ** 3 / 3
        for q in it["parts"]:
            m = q["W"].shape[0]
            sw = q["W"].element_size()
            w["chmc"] += (2 * CHMC_NITER + 3) * m * n * sw + 4 * m * n
            fused = n % 4 == 0 and n > p.block
            for j0 in range(0, n, p.block):
                bw = min(p.block, n - j0)
                n2 = n - j0 - bw
                w["sweep"] += 9 * m * bw + 4 * bw * bw + 5 * (-(-m // CHMC_GS)) * bw
                if n2 > 0 and fused:
                    w["sweep"] += 8 * m * n2 + 4 * m * bw + 4 * bw * n2
            w["pack"] += m * n + m * n * p.bits / 8 + 5 * (-(-m // CHMC_GS)) * n
            w["ingest"] += m * n * 8
    units = {"hessian": "TFLOP/s", "cholesky": "TFLOP/s", "chmc": "GB/s", "sweep": "GB/s",
             "pack": "GB/s", "ingest": "GB/s"}
    return {k: (units[k], v) for k, v in w.items()}


def run_chmc(args, rank, world, local):
    """The CHMC frontend over the layer: device-timed graph replay and the
    per-kernel event profile, as for the GPTQ path (no host-copy leg)."""
    import post_weight_quantization_08_b200 as g
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    cfg = CONFIGS[args.config]
    bits = args.bits or cfg["bits"][0]
    probs = problems_for(args.config, layer=layer_for_rank(rank), bits=bits, order="act")
    layer = ChmcLayer(probs, device)
    params = sum(p.params for p in probs)
    main = torch.cuda.Stream(device=device)
    torch.cuda.set_stream(main)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)
    for _ in range(args.warmup):
        layer.step(main)
    torch.cuda.synchronize(device)
    layer.check()
    graph = torch.cuda.CUDAGraph()
    c0 = g.gptq_launch_count()
    with torch.cuda.graph(graph, stream=main):
        layer.step(main)
    launches_per_step = g.gptq_launch_count() - c0
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize(device)
    layer.check()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    clocks = ClockSampler(local)
    clocks.start()
    evs = []
    for _ in range(args.steps):
        flush.fill_(1.0)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(main)
        graph.replay()
        b.record(main)
        evs.append((a, b))
    torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    layer.check()
    dev_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), world, device)
    total_params = sum_over_ranks(params * args.steps, world, device)
    g.gptq_profile_start(1 << 16)
    for _ in range(args.steps):
        flush.fill_(1.0)
        layer.step_serial(main)
    torch.cuda.synchronize(device)
    kprof = g.gptq_profile_stop()
    work = chmc_work(layer)
    peaks, src = _peaks()
    kernels = {}
    for k, (unit, amount) in work.items():
        if k not in kprof or kprof[k][1] <= 0 or amount <= 0:
            continue
        per_step_ms = kprof[k][0] / args.steps
        if unit == "TFLOP/s":
            ach = amount / (per_step_ms / 1e3) / 1e12
            bound, peak = (("tensor", peaks["bf16_tflops"]) if k == "hessian" else
                           ("alu", fp64_peak_tflops(peaks.get("sm_max_mhz", 1965.0))))
        else:
            ach = amount / (per_step_ms / 1e3) / 1e9
            bound, peak = "hbm", peaks["hbm_gbs"]
        kernels[k] = {"ms_per_step": round(per_step_ms, 4),
                      "launches_per_step": kprof[k][1] / args.steps, "bound": bound,
                      "achieved": round(ach, 2), "unit": unit, "peak": round(peak, 1),
                      "frac": round(ach / peak, 4)}
    ranks = {q["name"]: q["r"] for it in layer.items for q in it["parts"]}
    return {
        "metric": CHMC_METRIC, "value": round(total_params / (dev_ms / 1e3), 1),
        "unit": "params/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dev_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16->f32 Hessian, f64 prepare and low-rank part, f32 sweep",
        "data": "synthetic (seeded cone activations, N(0,0.02^2) weights)",
        "config": {"workload": frontend_workload("chmc", cfg, bits, probs[0].group,
                                                 probs[0].block),
                   "params_per_step_per_gpu": params, "ranks": ranks,
                   "l2": "flushed between timed steps (256 MB write)",
                   "launch": "CUDA graph replay per step"},
        "gpu_launches": int(launches_per_step * args.steps),
        "roofline": _frontend_roofline(kernels, {k: round(v[0] / args.steps, 4)
                                                 for k, v in kprof.items() if v[0] > 0}),
        "kernels": kernels,
        "kernels_ms_per_step": {k: round(v[0] / args.steps, 4) for k, v in kprof.items()
                                if v[0] > 0},
        "clocks": clk,
    }, probs


def chmc_cpu_baseline(probs):
    """The CHMC oracle over the whole layer (every matrix, each Hessian from X
    inside the timed region), params/s."""
    from oracle import chmc as oc
    from oracle import gptq as og
    t0 = time.perf_counter()
    total = 0
    for pi, p in enumerate(probs):
        X = p.X.to(torch.float64).numpy()
        H = og.hessian(X)
        row0 = 0
        for k, (name, rows) in enumerate(p.parts):
            W = p.W[row0:row0 + rows].to(torch.float64).numpy()
            row0 += rows
            r = oc.chmc_rank(rows, p.n, p.bits, CHMC_GS, CHMC_BPW)
            Om = normal_matrix(p.n, max(r, 1), 9000 + 100 * pi + k)[:, :r].to(torch.float64).numpy()
            oc.chmc_layer(W, H, p.T, Om, rank=r, bits=p.bits, gs=CHMC_GS, damp=CHMC_DAMP,
                          niter=CHMC_NITER, block=p.block)
            total += rows * p.n
    dt = time.perf_counter() - t0
    return {"value": round(total / dt, 1), "unit": "params/s", "cores": blas_threads(),
            "kind": "oracle", "sample": "one full pass over the layer's seven matrices, "
                                        "both Hessians from X included"}


# ---------------------------------------------------------------- SSQR

SSQR_METRIC = ("SSQR weights compressed/sec (params/s incl. Hessian, the binary search's "
               "sweeps and the CSR outliers) & % of roofline, 1 B200")
SSQR_BITS, SSQR_TARGET, SSQR_ITERS, SSQR_LO, SSQR_HI = 3, 0.01, 12, 1.0 / 16, 1.0


class SsqrLayer:
    """Device buffers of one layer under SSQR ("The Geometry of LLM
    Quantization: GPTQ as Babai's Nearest Plane Algorithm", §3): per Hessian
    its factor, per weight matrix its codes, scales, CSR outliers and the
    search's trace (each matrix meets the outlier target on its own)."""

    def __init__(self, probs, device):
        import post_weight_quantization_08_b200 as g
        self.g = g
        self.items = []
        for p in probs:
            n = p.n
            it = {"p": p, "X": p.X.to(device).contiguous(),
                  "H": torch.zeros(n, n, dtype=torch.float32, device=device),
                  "perm": torch.empty(n, dtype=torch.int32, device=device),
                  "U": torch.empty(n, n, dtype=torch.float32, device=device),
                  "dead": torch.empty(n, dtype=torch.uint8, device=device),
                  "info_h": torch.zeros(2, dtype=torch.int32, device=device),
                  "info_p": torch.zeros(2, dtype=torch.int32, device=device),
                  "ws_p": g.workspace(g.gptq_prepare_workspace_bytes(n), device),
                  "stream": torch.cuda.Stream(device=device), "parts": []}
            row0 = 0
            for name, rows in p.parts:
                W = p.W[row0:row0 + rows].to(device).contiguous()
                row0 += rows
                ng = -(-n // p.group)
                cap = max(int(SSQR_TARGET * rows * n), 1)
                it["parts"].append({
                    "name": name, "W": W,
                    "qweight": torch.empty(rows, -(-n * SSQR_BITS // 32), dtype=torch.int32,
                                           device=device),
                    "scale": torch.empty(rows, ng, dtype=torch.float32, device=device),
                    "zero": torch.empty(rows, ng, dtype=torch.uint8, device=device),
                    "g_idx": torch.empty(n, dtype=torch.int32, device=device),
                    "row_ptr": torch.empty(rows + 1, dtype=torch.int64, device=device),
                    "col_idx": torch.empty(cap, dtype=torch.int32, device=device),
                    "val": torch.empty(cap, dtype=torch.float32, device=device),
                    "alpha": torch.empty(1, dtype=torch.float32, device=device),
                    "loss": torch.empty(rows, dtype=torch.float32, device=device),
                    "info_q": torch.zeros(2, dtype=torch.int32, device=device),
                    "ws_q": g.workspace(g.gptq_ssqr_workspace_bytes(rows, n, p.block), device),
                    "stream": torch.cuda.Stream(device=device),
                })
            self.items.append(it)
        # the matrices with the most blocks per pass set the step's critical
        # path: their searches look ahead (three passes side by side), the
        # others take one pass a step and leave the SMs to them
        most = max(-(-it["p"].n // it["p"].block) for it in self.items)
        for it in self.items:
            for q in it["parts"]:
                q["lookahead"] = -(-it["p"].n // it["p"].block) == most

    def run_problem(self, it, serial=False):
        """Hessian and factor on the problem's stream, then each matrix's
        search on a stream of its own (``serial``: all on one stream)."""
        g, p, s = self.g, it["p"], it["stream"]
        with torch.cuda.stream(s):
            it["H"].zero_()
        g.gptq_hessian_accumulate(it["X"], it["H"], it["info_h"], s)
        g.gptq_prepare(it["H"], p.damp, "act", it["perm"], it["U"], it["dead"],
                       it["info_p"], it["ws_p"], s)
        prep_done = torch.cuda.Event()
        prep_done.record(s)
        for q in it["parts"]:
            qs = s if serial else q["stream"]
            if not serial:
                qs.wait_event(prep_done)
            g.gptq_ssqr_quantize(q["W"], it["U"], it["perm"], it["dead"], SSQR_BITS, p.group,
                                 p.block, SSQR_TARGET, SSQR_ITERS, SSQR_LO, SSQR_HI,
                                 q["qweight"], q["scale"], q["zero"], q["g_idx"], q["row_ptr"],
                                 q["col_idx"], q["val"], q["alpha"], None, None, q["loss"],
                                 None, q["info_q"], q["ws_q"], qs, q["lookahead"])
            if not serial:
                e = torch.cuda.Event()
                e.record(qs)
                s.wait_event(e)

    step = ChmcLayer.step
    step_serial = ChmcLayer.step_serial

    def check(self):
        for it in self.items:
            for key in ("info_h", "info_p"):
                st, idx = self.g.gptq_check(it[key], it["stream"])
                if st != 0:
                    raise RuntimeError(f"device reported status {st} at {idx}")
            for q in it["parts"]:
                st, idx = self.g.gptq_check(q["info_q"], it["stream"])
                if st != 0:
                    raise RuntimeError(f"{q['name']}: device reported status {st} at {idx}")


def ssqr_work(layer):
    """Algorithmic work per kernel kind for one SSQR step: the hot path's
    per-kind figures (kernel_work) with the sweep and ingest counted once per
    pass (iters + 2 passes per matrix), the TF32 split of U and the packing
    once per matrix, and the ssqr kind's CSR fill (codes read, 1 B per
    weight)."""
    w = {k: 0.0 for k in ("hessian", "cholesky", "sweep", "trailing", "pack", "ingest", "ssqr")}
    passes = SSQR_ITERS + 2
    for it in layer.items:
        p = it["p"]
        n, T, block = p.n, p.T, p.block
        w["hessian"] += T * n * (n + 1)
        N = -(-n // 64)
        for k in range(N):
            r = N - k - 1
            w["cholesky"] += (r * (r + 1) // 2 + r * (k + 1) + r + k) * 2 * 64 ** 3
            w["cholesky"] += 2 * 64 ** 3 / 3
        fused = n % 4 == 0 and n > block
        for q in it["parts"]:
            m = q["W"].shape[0]
            if fused:
                w["trailing"] += 12 * n * n
            for j0 in range(0, n, block):
                bw = min(block, n - j0)
                n2 = n - j0 - bw
                w["sweep"] += passes * (9 * m * bw + 4 * bw * bw + 5 * m * (-(-bw // p.group)))
                if n2 > 0:
                    w["sweep" if fused else "trailing"] += passes * (8 * m * n2 + 4 * m * bw
                                                                     + 4 * bw * n2)
            w["pack"] += m * n + m * n * SSQR_BITS / 8 + 5 * m * (-(-n // p.group))
            w["ingest"] += passes * m * n * (q["W"].element_size() + 4)
            w["ssqr"] += m * n
    units = {"hessian": "TFLOP/s", "cholesky": "TFLOP/s", "sweep": "GB/s", "trailing": "GB/s",
             "pack": "GB/s", "ingest": "GB/s", "ssqr": "GB/s"}
    return {k: (units[k], v) for k, v in w.items()}


def ssqr_cpu_baseline(probs, budget_s: float = 20.0):
    """The SSQR oracle on the layer's matrices in order (Hessian from X, the
    whole binary search), until the time budget is spent; params/s over the
    matrices completed."""
    from oracle import gptq as og
    from oracle import ssqr as osq
    t0 = time.perf_counter()
    total, done = 0, []
    for p in probs:
        H = og.hessian(p.X.to(torch.float64).numpy())
        prep = og.prepare(H, p.damp, "act")
        row0 = 0
        for name, rows in p.parts:
            W = p.W[row0:row0 + rows].to(torch.float64).numpy()
            row0 += rows
            osq.ssqr_layer(W, H, bits=SSQR_BITS, group=p.group, block=p.block, damp=p.damp,
                           target=SSQR_TARGET, iters=SSQR_ITERS, alpha_lo=SSQR_LO,
                           alpha_hi=SSQR_HI, prep=prep)
            total += rows * p.n
            done.append(name)
            if time.perf_counter() - t0 >= budget_s:
                break
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": round(total / dt, 1), "unit": "params/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"the layer's matrices in order until {budget_s:.0f} s: {', '.join(done)} "
                      f"({dt:.1f} s, Hessians and factors included)"}


def run_ssqr(args, rank, world, local):
    """SSQR over the layer: device-timed graph replay and the per-kernel
    event profile, as for the CHMC frontend."""
    import post_weight_quantization_08_b200 as g
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    cfg = CONFIGS[args.config]
    probs = problems_for(args.config, layer=layer_for_rank(rank), bits=SSQR_BITS, order="act")
    layer = SsqrLayer(probs, device)
    params = sum(p.params for p in probs)
    out = _time_frontend(args, layer, device, world, local, ssqr_work(layer))
    alphas = {q["name"]: float(q["alpha"].cpu()[0]) for it in layer.items for q in it["parts"]}
    nnz = {q["name"]: int(q["row_ptr"][-1]) for it in layer.items for q in it["parts"]}
    dev_ms, launches, kernels, kms, clk = out
    total_params = sum_over_ranks(params * args.steps, world, device)
    return {
        "metric": SSQR_METRIC, "value": round(total_params / (dev_ms / 1e3), 1),
        "unit": "params/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dev_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16->f32 Hessian, f64 prepare, f32 sweep",
        "data": "synthetic (seeded cone activations, N(0,0.02^2) weights)",
        "config": {"workload": frontend_workload("ssqr", cfg, SSQR_BITS, probs[0].group,
                                                 probs[0].block),
                   "params_per_step_per_gpu": params, "alpha": alphas, "outliers": nnz,
                   "l2": "flushed between timed steps (256 MB write)",
                   "launch": "CUDA graph replay per step"},
        "gpu_launches": int(launches * args.steps),
        "roofline": _frontend_roofline(kernels, kms),
        "kernels": kernels, "kernels_ms_per_step": kms, "clocks": clk,
    }, probs


# ---------------------------------------------------------------- HPTQ

HPTQ_METRIC = ("HPTQ weights compressed/sec (params/s incl. Hessian, the binary search's "
               "sweeps and the Huffman coding) & % of roofline, 1 B200")
HPTQ_BITS, HPTQ_BUDGET, HPTQ_ITERS, HPTQ_LO, HPTQ_HI = 4, 3.125, 12, 1.0 / 16, 16.0


class HptqLayer:
    """Device buffers of one layer under HPTQ ("The Geometry of LLM
    Quantization: GPTQ as Babai's Nearest Plane Algorithm", §3): per Hessian
    its factor, per weight matrix its lattice coordinates, scales, Huffman
    table, row offsets and bit stream (each matrix meets the budget on its
    own)."""

    def __init__(self, probs, device):
        import post_weight_quantization_08_b200 as g
        self.g = g
        self.items = []
        for p in probs:
            n = p.n
            it = {"p": p, "X": p.X.to(device).contiguous(),
                  "H": torch.zeros(n, n, dtype=torch.float32, device=device),
                  "perm": torch.empty(n, dtype=torch.int32, device=device),
                  "U": torch.empty(n, n, dtype=torch.float32, device=device),
                  "dead": torch.empty(n, dtype=torch.uint8, device=device),
                  "info_h": torch.zeros(2, dtype=torch.int32, device=device),
                  "info_p": torch.zeros(2, dtype=torch.int32, device=device),
                  "ws_p": g.workspace(g.gptq_prepare_workspace_bytes(n), device),
                  "stream": torch.cuda.Stream(device=device), "parts": []}
            row0 = 0
            for name, rows in p.parts:
                W = p.W[row0:row0 + rows].to(device).contiguous()
                row0 += rows
                ng = -(-n // p.group)
                cap = int(HPTQ_BUDGET * rows * n) // 32 + rows + 1
                it["parts"].append({
                    "name": name, "W": W,
                    "codes": torch.empty(rows, n, dtype=torch.int16, device=device),
                    "scale": torch.empty(rows, ng, dtype=torch.float32, device=device),
                    "g_idx": torch.empty(n, dtype=torch.int32, device=device),
                    "code_len": torch.empty(g.HPTQ_SYMBOLS, dtype=torch.uint8, device=device),
                    "code_word": torch.empty(g.HPTQ_SYMBOLS, dtype=torch.int64, device=device),
                    "row_off": torch.empty(rows + 1, dtype=torch.int64, device=device),
                    "bitstream": torch.empty(cap, dtype=torch.int32, device=device),
                    "alpha": torch.empty(1, dtype=torch.float32, device=device),
                    "loss": torch.empty(rows, dtype=torch.float32, device=device),
                    "info_q": torch.zeros(2, dtype=torch.int32, device=device),
                    "ws_q": g.workspace(g.gptq_hptq_workspace_bytes(rows, n, p.block), device),
                    "stream": torch.cuda.Stream(device=device),
                })
            self.items.append(it)
        # the matrices with the most blocks per pass set the step's critical
        # path: their searches look ahead (three passes side by side), the
        # others take one pass a step and leave the SMs to them
        most = max(-(-it["p"].n // it["p"].block) for it in self.items)
        for it in self.items:
            for q in it["parts"]:
                q["lookahead"] = -(-it["p"].n // it["p"].block) == most

    def run_problem(self, it, serial=False):
        g, p, s = self.g, it["p"], it["stream"]
        with torch.cuda.stream(s):
            it["H"].zero_()
        g.gptq_hessian_accumulate(it["X"], it["H"], it["info_h"], s)
        g.gptq_prepare(it["H"], p.damp, "act", it["perm"], it["U"], it["dead"],
                       it["info_p"], it["ws_p"], s)
        prep_done = torch.cuda.Event()
        prep_done.record(s)
        for q in it["parts"]:
            qs = s if serial else q["stream"]
            if not serial:
                qs.wait_event(prep_done)
            g.gptq_hptq_quantize(q["W"], it["U"], it["perm"], it["dead"], HPTQ_BITS, p.group,
                                 p.block, HPTQ_BUDGET, HPTQ_ITERS, HPTQ_LO, HPTQ_HI, q["codes"],
                                 q["scale"], q["g_idx"], q["code_len"], q["code_word"],
                                 q["row_off"], q["bitstream"], q["alpha"], None, None, q["loss"],
                                 None, q["info_q"], q["ws_q"], qs, q["lookahead"])
            if not serial:
                e = torch.cuda.Event()
                e.record(qs)
                s.wait_event(e)

    step = ChmcLayer.step
    step_serial = ChmcLayer.step_serial
    check = SsqrLayer.check


def hptq_work(layer):
    """Algorithmic work per kernel kind for one HPTQ step: as SSQR's, with the
    sweep writing 2-byte coordinates, and the hptq kind's bytes: per pass the
    histogram (2 B per weight), at the end the row bit counts and the encoder
    (2 B per weight each, plus the stream written) and the original-order
    coordinates (2 B in, 2 B out per weight)."""
    w = {k: 0.0 for k in ("hessian", "cholesky", "sweep", "trailing", "ingest", "hptq")}
    passes = HPTQ_ITERS + 2
    for it in layer.items:
        p = it["p"]
        n, T, block = p.n, p.T, p.block
        w["hessian"] += T * n * (n + 1)
        N = -(-n // 64)
        for k in range(N):
            r = N - k - 1
            w["cholesky"] += (r * (r + 1) // 2 + r * (k + 1) + r + k) * 2 * 64 ** 3
            w["cholesky"] += 2 * 64 ** 3 / 3
        fused = n % 4 == 0 and n > block
        for q in it["parts"]:
            m = q["W"].shape[0]
            if fused:
                w["trailing"] += 12 * n * n
            for j0 in range(0, n, block):
                bw = min(block, n - j0)
                n2 = n - j0 - bw
                w["sweep"] += passes * (10 * m * bw + 4 * bw * bw + 5 * m * (-(-bw // p.group)))
                if n2 > 0:
                    w["sweep" if fused else "trailing"] += passes * (8 * m * n2 + 4 * m * bw
                                                                     + 4 * bw * n2)
            w["ingest"] += passes * m * n * (q["W"].element_size() + 4)
            w["hptq"] += passes * 2 * m * n + 8 * m * n + HPTQ_BUDGET * m * n / 8
    units = {"hessian": "TFLOP/s", "cholesky": "TFLOP/s", "sweep": "GB/s", "trailing": "GB/s",
             "ingest": "GB/s", "hptq": "GB/s"}
    return {k: (units[k], v) for k, v in w.items()}


def hptq_cpu_baseline(probs, budget_s: float = 20.0):
    """The HPTQ oracle on the layer's matrices in order (Hessian from X, the
    whole binary search with a Huffman code per pass, the encoding), until the
    time budget is spent; params/s over the matrices completed."""
    from oracle import gptq as og
    from oracle import hptq as oh
    t0 = time.perf_counter()
    total, done = 0, []
    for p in probs:
        H = og.hessian(p.X.to(torch.float64).numpy())
        prep = og.prepare(H, p.damp, "act")
        row0 = 0
        for name, rows in p.parts:
            W = p.W[row0:row0 + rows].to(torch.float64).numpy()
            row0 += rows
            out = oh.hptq_layer(W, H, bits=HPTQ_BITS, group=p.group, block=p.block,
                                damp=p.damp, budget=HPTQ_BUDGET, iters=HPTQ_ITERS,
                                alpha_lo=HPTQ_LO, alpha_hi=HPTQ_HI, prep=prep)
            oh.encode(out["codes"][:8], out["lengths"])      # the codec, on a row sample
            total += rows * p.n
            done.append(name)
            if time.perf_counter() - t0 >= budget_s:
                break
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": round(total / dt, 1), "unit": "params/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"the layer's matrices in order until {budget_s:.0f} s: {', '.join(done)} "
                      f"({dt:.1f} s, Hessians and factors included; the bit stream of 8 rows "
                      f"per matrix)"}


def run_hptq(args, rank, world, local):
    """HPTQ over the layer: device-timed graph replay and the per-kernel event
    profile, as for SSQR."""
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    cfg = CONFIGS[args.config]
    probs = problems_for(args.config, layer=layer_for_rank(rank), bits=HPTQ_BITS, order="act")
    layer = HptqLayer(probs, device)
    params = sum(p.params for p in probs)
    dev_ms, launches, kernels, kms, clk = _time_frontend(args, layer, device, world, local,
                                                         hptq_work(layer))
    parts = [q for it in layer.items for q in it["parts"]]
    alphas = {q["name"]: float(q["alpha"].cpu()[0]) for q in parts}
    bpw = {q["name"]: round(int(q["row_off"][-1]) / q["W"].numel(), 4) for q in parts}
    total_params = sum_over_ranks(params * args.steps, world, device)
    return {
        "metric": HPTQ_METRIC, "value": round(total_params / (dev_ms / 1e3), 1),
        "unit": "params/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dev_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16->f32 Hessian, f64 prepare, f32 sweep, int16 codes",
        "data": "synthetic (seeded cone activations, N(0,0.02^2) weights)",
        "config": {"workload": frontend_workload("hptq", cfg, HPTQ_BITS, probs[0].group,
                                                 probs[0].block),
                   "params_per_step_per_gpu": params, "alpha": alphas, "bits_per_weight": bpw,
                   "l2": "flushed between timed steps (256 MB write)",
                   "launch": "CUDA graph replay per step"},
        "gpu_launches": int(launches * args.steps),
        "roofline": _frontend_roofline(kernels, kms),
        "kernels": kernels, "kernels_ms_per_step": kms, "clocks": clk,
    }, probs


def _frontend_roofline(kernels, kms):
    """The roofline object of a frontend line: its dominant kernel kind (the
    most device time in the serialised event profile) with the same figures
    as its entry in ``kernels``; no ncu DRAM capture is kept for these
    workloads, so traffic is null."""
    if not kernels:
        return None
    dom = max(kernels, key=lambda k: kernels[k]["ms_per_step"])
    e = kernels[dom]
    _, src = _peaks()
    note = ("fp64 148 SMs x 64 FMA x 2 x max clock" if e["bound"] == "alu"
            else (f"bf16 {src}" if e["bound"] == "tensor" else f"copy bandwidth, {src}"))
    return {"kernel": dom, "bound": e["bound"], "achieved": e["achieved"], "peak": e["peak"],
            "unit": e["unit"], "frac": e["frac"], "peak_source": note, "traffic": None,
            "launches_per_step": e["launches_per_step"],
            "share": round(e["ms_per_step"] / max(1e-9, sum(kms.values())), 4)}


def _time_frontend(args, layer, device, world, local, work):
    """Warm up, capture one step in a CUDA graph, time K replays with the L2
    flushed between them (max over ranks), then time every kernel kind with
    the library's event profiler on a serialised step."""
    import post_weight_quantization_08_b200 as g
    main = torch.cuda.Stream(device=device)
    torch.cuda.set_stream(main)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)
    for _ in range(args.warmup):
        layer.step(main)
    torch.cuda.synchronize(device)
    layer.check()
    graph = torch.cuda.CUDAGraph()
    c0 = g.gptq_launch_count()
    with torch.cuda.graph(graph, stream=main):
        layer.step(main)
    launches_per_step = g.gptq_launch_count() - c0
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize(device)
    layer.check()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    clocks = ClockSampler(local)
    clocks.start()
    evs = []
    for _ in range(args.steps):
        flush.fill_(1.0)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(main)
        graph.replay()
        b.record(main)
        evs.append((a, b))
    torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    layer.check()
    dev_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), world, device)
    g.gptq_profile_start(1 << 17)
    for _ in range(args.steps):
        flush.fill_(1.0)
        layer.step_serial(main)
    torch.cuda.synchronize(device)
    kprof = g.gptq_profile_stop()
    peaks, src = _peaks()
    kernels = {}
    for k, (unit, amount) in work.items():
        if k not in kprof or kprof[k][1] <= 0 or amount <= 0:
            continue
        per_step_ms = kprof[k][0] / args.steps
        if unit == "TFLOP/s":
            ach = amount / (per_step_ms / 1e3) / 1e12
            bound, peak = (("tensor", peaks["bf16_tflops"]) if k == "hessian" else
                           ("alu", fp64_peak_tflops(peaks.get("sm_max_mhz", 1965.0))))
        else:
            ach = amount / (per_step_ms / 1e3) / 1e9
            bound, peak = "hbm", peaks["hbm_gbs"]
        kernels[k] = {"ms_per_step": round(per_step_ms, 4),
                      "launches_per_step": kprof[k][1] / args.steps, "bound": bound,
                      "achieved": round(ach, 2), "unit": unit, "peak": round(peak, 1),
                      "frac": round(ach / peak, 4)}
    kms = {k: round(v[0] / args.steps, 4) for k, v in kprof.items() if v[0] > 0}
    return dev_ms, launches_per_step, kernels, kms, clk


# ---------------------------------------------------------------- CPU oracle arm

def oracle_pass(probs, static_groups=False):
    """One pass of the float64 oracle over the problems (test infrastructure)."""
    from oracle import gptq as og
    from oracle import static as ost
    for p in probs:
        X = p.X.to(torch.float64).numpy()
        W = p.W.to(torch.float64).numpy()
        H = og.hessian(X)
        if static_groups:
            ost.gptq_layer_static(W, H, p.bits, p.group, p.block, p.damp, p.order)
        else:
            og.gptq_layer(W, H, p.bits, p.group, p.block, p.damp, p.order)
    return sum(p.params for p in probs)


CPU_SAMPLE_ROWS = 1024


def oracle_problem_seconds(p, static_groups=False, rows=CPU_SAMPLE_ROWS):
    """Seconds the float64 oracle takes for one whole problem, from a bounded
    sample: the Hessian and the factorisation in full, the oracle's layer pass
    on the first `rows` rows (which factorises again), and the per-row part of
    that pass scaled to all m rows (rows are independent given U).  Returns
    (seconds, rows sampled)."""
    from oracle import gptq as og
    from oracle import static as ost
    X = p.X.to(torch.float64).numpy()
    W = p.W.to(torch.float64).numpy()
    r = min(rows, p.m)
    t0 = time.perf_counter()
    H = og.hessian(X)
    t1 = time.perf_counter()
    og.prepare(H, p.damp, p.order)
    t2 = time.perf_counter()
    if static_groups:
        ost.gptq_layer_static(W[:r], H, p.bits, p.group, p.block, p.damp, p.order)
    else:
        og.gptq_layer(W[:r], H, p.bits, p.group, p.block, p.damp, p.order)
    t3 = time.perf_counter()
    per_rows = max(0.0, (t3 - t2) - (t2 - t1))
    return (t1 - t0) + (t2 - t1) + per_rows * p.m / r, r


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        if info:
            return max(int(i.get("num_threads", 1)) for i in info)
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_baseline(probs, budget_s: float = 12.0, static_groups=False):
    """The float64 oracle on the host cores over problems of the step, one after
    the other in the step's order, until ``budget_s`` has passed (at least one
    problem).  Small problems run whole; larger ones are a bounded sample
    (oracle_problem_seconds: Hessian and factorisation in full, the per-row
    pass on CPU_SAMPLE_ROWS rows scaled to all rows)."""
    done, est, count = 0, 0.0, 0
    t0 = time.perf_counter()
    samples = []
    while True:
        p = probs[count % len(probs)]
        sec, r = oracle_problem_seconds(p, static_groups)
        done += p.params
        est += sec
        samples.append(f"{p.m}x{p.n}" + ("" if r >= p.m else f" ({r} of {p.m} rows)"))
        count += 1
        if time.perf_counter() - t0 >= budget_s or count >= 50:
            break
    el = time.perf_counter() - t0
    return {"value": round(done / est, 1), "unit": "params/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": (f"{count} problems of the step ({', '.join(sorted(set(samples)))}; "
                       f"{el:.1f} s of float64 numpy): Hessian and factorisation in full, "
                       f"the per-row pass scaled from the sampled rows to all rows")}


def frontend_workload(frontend: str, cfg, bits: int, group: int, block: int) -> str:
    """The workload string of a frontend line (the GPU and the oracle arm)."""
    if frontend == "chmc":
        return (f"{cfg['name']} CHMC: per-matrix rank from the {CHMC_BPW}-bit budget, niter "
                f"{CHMC_NITER}, lambda {CHMC_LAM}, damp {CHMC_DAMP}, act-order, residual "
                f"{bits}-bit with {CHMC_GS}-row output-channel groups, block {block}")
    if frontend == "ssqr":
        return (f"{cfg['name']} SSQR: {SSQR_BITS}-bit, group {group}, act-order, target outlier "
                f"density {SSQR_TARGET} per matrix, {SSQR_ITERS} bisection steps on alpha in "
                f"[{SSQR_LO}, {SSQR_HI}], block {block}")
    return (f"{cfg['name']} HPTQ: lattice from the {HPTQ_BITS}-bit min-max step, group {group}, "
            f"act-order, budget {HPTQ_BUDGET} bits/weight per matrix, {HPTQ_ITERS} bisection "
            f"steps on alpha in [{HPTQ_LO}, {HPTQ_HI}], block {block}")


def run_reference_frontend(args, world):
    """The oracle arm of a frontend line: each step one bounded sample of the
    frontend's float64 oracle over the layer's matrices (the same function as
    the line's cpu_baseline), its metric, unit and workload."""
    cfg = CONFIGS[args.config]
    fb = {"chmc": (CHMC_METRIC, args.bits or cfg["bits"][0], chmc_cpu_baseline),
          "ssqr": (SSQR_METRIC, SSQR_BITS, ssqr_cpu_baseline),
          "hptq": (HPTQ_METRIC, HPTQ_BITS, hptq_cpu_baseline)}[args.frontend]
    metric, bits, fn = fb
    probs = problems_for(args.config, layer=0, bits=bits, order="act")
    kw = {} if args.frontend == "chmc" else {"budget_s": 0.0}
    for _ in range(args.warmup):
        fn(probs, **kw)                            # one matrix each (budget 0)
    t0 = time.perf_counter()
    vals, sample = [], ""
    for _ in range(args.steps):
        r = fn(probs)
        vals.append(r["value"])
        sample = r["sample"]
    el = time.perf_counter() - t0
    value = sum(vals) / len(vals)
    return {
        "impl": "reference", "metric": metric, "value": round(value, 1), "unit": "params/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el * 1e3 / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded cone activations, N(0,0.02^2) weights)",
        "config": {"workload": frontend_workload(args.frontend, cfg, bits, probs[0].group,
                                                 probs[0].block)},
        "cpu_baseline": {"value": round(value, 1), "unit": "params/s", "cores": blas_threads(),
                         "kind": "oracle", "sample": f"per step: {sample}"},
        "e2e": {"value": round(value, 1), "unit": "params/s",
                "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_reference(args, rank, world):
    """The oracle arm: each step one bounded sample of the same workload, the
    float64 oracle on one problem of the step (its Hessian and factorisation in
    full, the per-row pass on CPU_SAMPLE_ROWS rows scaled to all rows), taking
    the step's problems in turn."""
    if rank != 0:
        return None
    if args.frontend != "gptq":
        return run_reference_frontend(args, world)
    cfg = CONFIGS[args.config]
    bits = args.bits or cfg["bits"][0]
    nl = stack_layers(args)
    probs = problems_for(args.config, layer=0, bits=bits, order=args.order)
    for k in range(args.warmup):
        oracle_problem_seconds(probs[k % len(probs)], args.static_groups)
    t0 = time.perf_counter()
    params, est = 0, 0.0
    for k in range(args.steps):
        p = probs[k % len(probs)]
        sec, _ = oracle_problem_seconds(p, args.static_groups)
        params += p.params
        est += sec
    el = time.perf_counter() - t0
    value = params / est
    cores = blas_threads()
    shapes = ", ".join(f"{p.m}x{p.n}" for p in probs)
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": "params/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(est * 1e3 / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded cone activations, N(0,0.02^2) weights)",
        "config": {"workload": workload_name(args.config, bits, args.order, args.static_groups,
                                             nl)},
        "cpu_baseline": {"value": round(value, 1), "unit": "params/s", "cores": cores,
                         "kind": "oracle",
                         "sample": (f"per step one problem of a layer ({shapes}, in turn): "
                                    f"Hessian and factorisation in full, the per-row pass on "
                                    f"the first {CPU_SAMPLE_ROWS} rows scaled to all rows; "
                                    f"{args.steps} timed steps ({el:.1f} s) on the host cores")},
        "e2e": {"value": round(value, 1), "unit": "params/s",
                "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=None,
                    help="workload (0 single 576x576, 1 SmolLM-135M layer, 2 Qwen2.5-0.5B "
                         "x24, 3 TinyLlama-1.1B x22, 4 stress 8192^2; default 3, and 1 "
                         "for the frontends)")
    ap.add_argument("--layers", type=int, default=None,
                    help="decoder layers per step (default: every layer of the stack)")
    ap.add_argument("--lanes", type=int, default=4,
                    help="streams the Hessians and factorisations are spread over")
    ap.add_argument("--qstreams", type=int, default=8,
                    help="streams the quantize calls are spread over")
    ap.add_argument("--factor-workers", type=int, default=-1,
                    help="most worker CTAs a factorisation may use (0: every SM but one; "
                         "default: three fifths of the SMs when a step has eight or more "
                         "problems)")
    ap.add_argument("--profile-steps", type=int, default=2,
                    help="steps of the serialised per-kernel timing pass")
    ap.add_argument("--bits", type=int, default=None)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--frontend", default="gptq", choices=["gptq", "chmc", "ssqr", "hptq"],
                    help="chmc: the CHMC frontend over the layer; ssqr / hptq: SSQR / HPTQ "
                         "over the layer (separate metrics)")
    ap.add_argument("--static-groups", action="store_true",
                    help="group parameters fixed from the original weights (a variant of "
                         "the same metric)")
    ap.add_argument("--order", default=None,
                    choices=["natural", "act", "reverse", "minpivot"],
                    help="processing order for every problem (default: the workload's)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.config is None:
        args.config = 3 if args.frontend == "gptq" else 1
    rank, world, local = dist_env()

    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return 0

    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    try:
        if args.frontend == "chmc":
            out, probs = run_chmc(args, rank, world, local)
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                out["cpu_baseline"] = chmc_cpu_baseline(probs)
        elif args.frontend == "ssqr":
            out, probs = run_ssqr(args, rank, world, local)
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                out["cpu_baseline"] = ssqr_cpu_baseline(probs)
        elif args.frontend == "hptq":
            out, probs = run_hptq(args, rank, world, local)
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                out["cpu_baseline"] = hptq_cpu_baseline(probs)
        else:
            out, probs, _ = run_ours(args, rank, world, local)
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                out["cpu_baseline"] = cpu_baseline(probs, static_groups=args.static_groups)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
