"""Benchmark of the Flint int4 MoE block decode on B200.

Step: one decode token-step of a batch of B rows through the stack of 47
Flint MoE layers (RMSNorm -> MoE block -> fp32 residual add per layer), each
layer with its own seeded int4 weights (19.7 GB resident, so no layer's
weights stay in the 126 MB L2 between its uses), fresh seeded input rows per
step.  The reported value is device time per MoE layer (us/layer, lower is
better); the MoE-stack tokens/s, the batch-1 figure and the 150,144 x 2,048
int4 head GEMV are reported beside it.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--batch B] [--impl flint|reference]

N > 1 runs N independent replicas (the path is not sharded), one process per
GPU under torchrun; the time is the max over ranks.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

N_LAYERS = synth.N_MOE_LAYERS
H = synth.HIDDEN
LAYER_FIXED_BYTES = 256 * 2048 * 2 + 256 * 4 + 2048 * (1024 + 32) + 2048 * (512 + 16)
# DRAM bytes per decode layer over algorithmic bytes, from one ncu capture of
# four stacked layers of this workload at batch 4 (110.67 MB read against
# 109.89 MB algorithmic, caches flushed before every launch).  Traffic grows
# with the expert count the same way, so a full layer's traffic is reported as
# this ratio times its algorithmic bytes: a figure scaled from that capture,
# not measured in this run.
DECODE_TRAFFIC_RATIO = 110.672128 / 109.891584
TIMING_REPEATS = 20
HEAD_COPIES = 3  # copies of the head the head timing rotates over (3 x 158.6 MB > L2)
EXPERT_BYTES = 1024 * (1024 + 32) + 2048 * (256 + 8)
# group-64 affine experts: fp16 scale and offset per 64 codes
AFF_EXPERT_BYTES = 1024 * (1024 + 128) + 2048 * (256 + 32)
AFF_LAYER_FIXED_BYTES = 256 * 2048 * 2 + 256 * 4 + 2048 * (1024 + 128) + 2048 * (512 + 64)
HEAD_BYTES = synth.VOCAB * (1024 + 32)
METRIC = "us per MoE-layer decode (B=4), fraction of HBM roofline"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--batch", type=int, default=4)
    p.add_argument("--impl", default="flint", choices=["flint", "reference"])
    p.add_argument("--layers", type=int, default=N_LAYERS)
    p.add_argument("--no-head", action="store_true")
    p.add_argument("--no-cpu", action="store_true")
    p.add_argument("--no-prefill", action="store_true")
    p.add_argument("--no-affine", action="store_true")
    p.add_argument("--prefill-t", type=int, nargs="+", default=[2048, 4096, 32768],
                   help="prefill token counts timed as extra lines")
    return p.parse_args()


# router 2*256*2048 + routed 6 * 3 * 2 * 2048 * 512 + shared 3 * 2 * 2048 * 1024
PREFILL_FLOP_PER_TOKEN = 2 * 256 * 2048 + 6 * 6 * 2048 * 512 + 6 * 2048 * 1024
# grouped GEMM 1 (gate and up: 6 routed + shared), grouped GEMM 2 (down)
GEMM1_FLOP_PER_TOKEN = 6 * 2 * 2 * 2048 * 512 + 2 * 2 * 2048 * 1024
GEMM2_FLOP_PER_TOKEN = 6 * 2 * 2048 * 512 + 2 * 2048 * 1024
assert PREFILL_FLOP_PER_TOKEN == 2 * 256 * 2048 + GEMM1_FLOP_PER_TOKEN + GEMM2_FLOP_PER_TOKEN


def tensor_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""
    Q = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap,utilization.gpu")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                rows.append((ts, float(parts[0]), float(parts[1]), parts[2:6], float(parts[6])))
            except ValueError:
                continue
        inside = [r for r in rows if t0 <= r[0] <= t1] or rows
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i, v in enumerate(r[3]) if v == "Active"})
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "sm_max_mhz": max(r[2] for r in inside), "reasons": reasons,
                "samples": len(inside)}


# ------------------------------------------------------------------ workload
def decode_config(B, layers):
    """The workload both arms time (the reference arm on a bounded sample of it)."""
    return {"workload": f"flint moe decode, 47-layer stack (RMSNorm->MoE->residual), "
                        f"batch {B}, fresh rows per step",
            "batch": B, "layers": layers, "hidden": H, "experts": 256, "top_k": 6,
            "l2": "inputs larger than L2: 47 layers x 420 MB of int4 weights rotate"}


def step_inputs(steps: int, B: int) -> np.ndarray:
    """Fresh residual rows for each step: seed 10000 + 4*step + row."""
    return np.stack([synth.residual_h([10000 + 4 * s + r for r in range(B)]) for s in range(steps)])


def build_layers(n: int, device):
    import int4_expert_routing_b200 as F
    layers, structs = [], []
    for l in range(n):
        d = synth.layer_device(l, device)
        layers.append(d)
        structs.append(F.make_layer(d))
    return layers, structs


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, v: float, device: str = "cuda") -> float:
    """The largest of the ranks' values (every rank gets it); device is where
    the reduction runs: the GPU under NCCL, the CPU under gloo."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_us_per_layer(ms: float, steps: int, layers: int, world: int) -> float:
    """Whole-job figure: the slowest rank's time over every layer-step all ranks ran."""
    return ms * 1e3 / (steps * layers) / world


def host_cores() -> int:
    return os.cpu_count() or 1


def cpu_baseline(B: int, n_samples: int = 3):
    """The fp64 oracle on every host core: n_samples stack-layer calls at
    batch B (layer i on the rows of step i), timed; us per MoE layer."""
    import oracle
    cores = host_cores()
    oracle.set_threads(cores)
    hs = step_inputs(n_samples, B)
    t = 0.0
    for i in range(n_samples):
        L = oracle.Layer(synth.layer_host(i % N_LAYERS))
        t0 = time.perf_counter()
        oracle.stack_layer(L, hs[i])
        t += time.perf_counter() - t0
    return {"value": t / n_samples * 1e6, "unit": "us/layer", "cores": cores, "nproc": cores,
            "kind": "oracle",
            "sample": f"{n_samples} stack-layer calls at batch {B} (layers 0..{n_samples - 1}), "
                      f"fp64 oracle threaded over each matrix's output rows on {cores} threads"}


def cpu_baselines_other(B: int):
    """The oracle on the other workloads, each a bounded sample, all cores:
    one layer at batch 1 and at batch B (layer 0, decode rows), the output
    head at batch 1, and prefill of the first 64 tokens of the 2,048-token
    input (per-token work is the same for every token)."""
    import oracle
    cores = host_cores()
    oracle.set_threads(cores)
    out = {}
    L0 = oracle.Layer(synth.layer_host(0))
    for b, seeds in ((1, [0]), (B, list(range(1, B + 1)))):
        x = synth.decode_x(seeds)
        t0 = time.perf_counter()
        oracle.moe_layer(L0, x)
        dt = time.perf_counter() - t0
        out[f"layer_b{b}"] = {"value": dt * 1e6, "unit": "us/layer", "cores": cores,
                              "kind": "oracle", "sample": f"layer 0, batch {b}, in full"}
    head = synth.head_host()
    x = synth.head_x([0])
    t0 = time.perf_counter()
    oracle.int4_gemv(head["q"], head["s"], x)
    dt = time.perf_counter() - t0
    out["head_gemv_b1"] = {"value": dt * 1e6, "unit": "us", "cores": cores, "kind": "oracle",
                           "sample": "150,144 x 2,048 head, batch 1, in full"}
    xp = synth.prefill_x(2048, 2048)[:64]
    t0 = time.perf_counter()
    oracle.moe_layer(L0, xp)
    dt = time.perf_counter() - t0
    out["prefill_T2048"] = {"value": 64 / dt, "unit": "tokens/s", "cores": cores,
                            "kind": "oracle",
                            "sample": "first 64 of the 2,048 prefill tokens (layer 0), "
                                      "scaled per token"}
    return out


def run_reference(args):
    """Reference arm: the fp64 CPU oracle as it stands, on every host core.
    Each step is one stack-layer call at the benchmark's batch (RMSNorm ->
    block -> residual add for B rows; layers cycle through the first four of
    the stack), so the value is us per MoE layer at batch B, the arm's own
    metric, and ms_per_step is the time one such step took."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world > 1 and rank != 0:
        return
    import oracle
    cores = host_cores()
    oracle.set_threads(cores)
    B = args.batch
    hs = step_inputs(args.steps + args.warmup, B)
    cache = {}

    def layer(l):
        if l not in cache:
            cache[l] = oracle.Layer(synth.layer_host(l))
        return cache[l]

    for s in range(args.warmup):
        oracle.stack_layer(layer(s % 4), hs[s])
    t = 0.0
    for s in range(args.warmup, args.warmup + args.steps):
        L = layer(s % 4)
        t0 = time.perf_counter()
        oracle.stack_layer(L, hs[s])
        t += time.perf_counter() - t0
    per_layer_us = t / args.steps * 1e6
    line = {"impl": "reference", "metric": METRIC, "value": per_layer_us, "unit": "us/layer",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": per_layer_us / 1e3, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": decode_config(B, args.layers),
            "cpu_baseline": {"value": per_layer_us, "unit": "us/layer", "cores": cores,
                             "nproc": cores, "kind": "oracle",
                             "sample": f"{args.steps} stack-layer calls at batch {B} (layers "
                                       f"0..3 in turn), fp64 oracle on {cores} threads"},
            "e2e": {"value": per_layer_us, "unit": "us/layer", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    import torch
    import int4_expert_routing_b200 as F
    F.build()
    world, rank, local = dist_setup(args)
    dev = torch.device("cuda", torch.cuda.current_device())
    B, nl = args.batch, args.layers
    hbm, peak_kind = peaks()

    layers, structs = build_layers(nl, dev)
    layer_arr = F.layer_array(structs)
    total = args.steps + args.warmup
    h_host = torch.from_numpy(step_inputs(total, B)).pin_memory()          # [S][B][H]
    h_dev = h_host.to(dev)
    h_work = torch.empty((B, H), dtype=torch.float32, device=dev)
    nb = F.flint_workspace_bytes(F.FLINT_OP_DECODE, B)
    ws = torch.zeros(nb, dtype=torch.uint8, device=dev)
    F.flint_workspace_init(ws, nb)
    stream = torch.cuda.Stream(dev)

    def one_step(s, st, hw=h_work, b=B, w=ws, n=nb, src=None):
        hw.copy_(h_dev[s, :b] if src is None else src[s], non_blocking=True)
        F.flint_moe_decode_stack(layer_arr, nl, hw, b, None, None, None, w, n, stream=st)

    # routing of every (step, layer), outside the timed region, for the bytes count
    idx = torch.empty((nl, B, 6), dtype=torch.int32, device=dev)
    distinct = []
    with torch.cuda.stream(stream):
        for s in range(args.warmup, total):
            h_work.copy_(h_dev[s])
            F.flint_moe_decode_stack(layer_arr, nl, h_work, B, idx, None, None, ws, nb,
                                     stream=stream)
            distinct.append(idx.cpu().numpy())
    stream.synchronize()
    U = float(np.mean([len(set(a[l].ravel().tolist())) for a in distinct for l in range(nl)]))
    bytes_per_layer = LAYER_FIXED_BYTES + U * EXPERT_BYTES + 2 * B * H * 4

    def capture(step_fn):
        """CUDA graphs of the warm-up steps and of the K timed steps."""
        with torch.cuda.stream(stream):
            for s in range(args.warmup):
                step_fn(s, stream)
        stream.synchronize()
        gt = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gt, stream=stream):
            for s in range(args.warmup, total):
                step_fn(s, stream)
        gwu = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gwu, stream=stream):
            for s in range(min(args.warmup, total)):
                step_fn(s, stream)
        with torch.cuda.stream(stream):
            for _ in range(3):
                gwu.replay()
        stream.synchronize()
        return gt, gwu

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(gt):
        """TIMING_REPEATS replays of the K-step graph, each bracketed by a
        barrier and a synchronize, timed with events on the launching stream;
        per replay the max over ranks.  Returns the per-replay ms list."""
        out = []
        for _ in range(TIMING_REPEATS):
            barrier(world)
            torch.cuda.synchronize()
            with torch.cuda.stream(stream):
                e0.record(stream)
                gt.replay()
                e1.record(stream)
            e1.synchronize()
            barrier(world)
            torch.cuda.synchronize()
            out.append(max_over_ranks(world, e0.elapsed_time(e1)))
        return out

    g, gw = capture(one_step)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    # soak: replay the timed graph for ~1 s so the clock record covers a loaded GPU
    t_soak = time.time()
    while time.time() - t_soak < 1.0:
        with torch.cuda.stream(stream):
            g.replay()
        stream.synchronize()
    tw0 = time.time()
    reps = timed(g)
    tw1 = time.time()
    clocks = sampler.summary(tw0 - 0.5, tw1 + 0.5)
    ms = statistics.median(reps)

    us_per_layer = job_us_per_layer(ms, args.steps, nl, world)
    achieved = bytes_per_layer / (ms * 1e-3 / (args.steps * nl)) / 1e9
    timing = {"repeats": TIMING_REPEATS, "steps_per_repeat": args.steps,
              "us_per_layer_median": us_per_layer,
              "us_per_layer_min": job_us_per_layer(min(reps), args.steps, nl, world),
              "us_per_layer_max": job_us_per_layer(max(reps), args.steps, nl, world)}

    # ---- batch 1, same stack (context figure)
    extra = {}
    if B != 1:
        h1 = torch.empty((1, H), dtype=torch.float32, device=dev)
        nb1 = F.flint_workspace_bytes(F.FLINT_OP_DECODE, 1)
        ws1 = torch.zeros(nb1, dtype=torch.uint8, device=dev)
        F.flint_workspace_init(ws1, nb1)
        g1, gw1 = capture(lambda s, st: one_step(s, st, hw=h1, b=1, w=ws1, n=nb1))
        reps1 = timed(g1)
        ms1 = statistics.median(reps1)
        us1 = ms1 * 1e3 / (args.steps * nl)
        b1_bytes = LAYER_FIXED_BYTES + 6 * EXPERT_BYTES + 2 * H * 4
        extra["batch1"] = {"us_per_layer": us1, "us_per_layer_min": min(reps1) * 1e3 / (args.steps * nl),
                           "us_per_layer_max": max(reps1) * 1e3 / (args.steps * nl),
                           "stack_tokens_per_s": 1e6 / (us1 * nl),
                           "roofline_frac": b1_bytes / (us1 * 1e-6) / 1e9 / hbm,
                           "bytes_per_layer": b1_bytes}
        del g1, gw1

    # ---- the same stack with group-64 affine int4 experts (MLX int4 / Q4_1
    # layout) and with NVFP4 experts (weight-only, BF16 activations): 8 layers
    # of synthetic weights each (3.7 GB, larger than L2)
    aff_pf, nv_pf = [], []
    if not args.no_affine:
        naff = 8
        for fmt_name, make in (("affine", synth.affine_layer_device),
                               ("nvfp4", synth.nvfp4_layer_device)):
            fmt_structs = [F.make_layer(make(l, dev)) for l in range(naff)]
            fmt_arr = F.layer_array(fmt_structs)
            for ab in sorted({1, min(B, F.FLINT_MAX_DECODE_B_AFFINE)}):
                ha = torch.empty((ab, H), dtype=torch.float32, device=dev)
                nba = F.flint_workspace_bytes(F.FLINT_OP_DECODE, ab)
                wsa = torch.zeros(nba, dtype=torch.uint8, device=dev)
                F.flint_workspace_init(wsa, nba)

                def fmt_step(s, st, ha=ha, ab=ab, wsa=wsa, nba=nba, arr=fmt_arr):
                    ha.copy_(h_dev[s, :ab], non_blocking=True)
                    F.flint_moe_decode_stack(arr, naff, ha, ab, None, None, None, wsa, nba,
                                             stream=st)

                ga, gwa = capture(fmt_step)
                repsa = timed(ga)
                usa = statistics.median(repsa) * 1e3 / (args.steps * naff)
                rec = {"layers": naff, "us_per_layer": usa,
                       "us_per_layer_min": min(repsa) * 1e3 / (args.steps * naff),
                       "us_per_layer_max": max(repsa) * 1e3 / (args.steps * naff)}
                if ab == 1:  # six distinct experts: the bytes are known without the routing
                    # (the same for both formats: 4.5 bits per weight; NVFP4 adds
                    # 12 bytes of global scales per expert)
                    ab_bytes = AFF_LAYER_FIXED_BYTES + 6 * AFF_EXPERT_BYTES + 2 * H * 4
                    rec.update({"bytes_per_layer": ab_bytes,
                                "roofline_frac": ab_bytes / (usa * 1e-6) / 1e9 / hbm})
                extra[f"decode_{fmt_name}_b{ab}"] = rec
                del ga, gwa
            if fmt_name == "affine":
                aff_pf = fmt_structs[:3]  # prefill on affine experts rotates over three of them
            else:
                nv_pf = fmt_structs[:3]
            del fmt_structs, fmt_arr

    # ---- e2e through the C ABI with host buffers: H2D of the step's rows,
    # the stack call, D2H of the result rows, every step
    out_host = torch.empty((total, B, H), dtype=torch.float32).pin_memory()

    def e2e_step(s, st):
        h_work.copy_(h_host[s], non_blocking=True)
        F.flint_moe_decode_stack(layer_arr, nl, h_work, B, None, None, None, ws, nb, stream=st)
        out_host[s].copy_(h_work, non_blocking=True)

    ge, gwe = capture(e2e_step)
    repse = timed(ge)
    mse = statistics.median(repse)
    e2e_us = job_us_per_layer(mse, args.steps, nl, world)
    del ge, gwe

    # ---- output head int4 GEMV (B = 1 and the bench batch), context.  Timed
    # on inputs larger than L2: the launches rotate over HEAD_COPIES copies of
    # the head (158.6 MB each), so a launch never finds its weights in L2 and
    # no flush writes are left in L2 for it to write back.

    def rotating_us(calls, iters=23, skip=3, spin_cycles=400_000):
        """Median device time of single calls, call i on input copy i % len:
        a GPU spin queued ahead of each start event lets the host enqueue the
        call before the GPU reaches the event, so host launch overhead stays
        outside the timed region."""
        times = []
        for it in range(iters):
            with torch.cuda.stream(stream):
                torch.cuda._sleep(spin_cycles)
                e0.record(stream)
                calls[it % len(calls)]()
                e1.record(stream)
            e1.synchronize()
            if it >= skip:
                times.append(e0.elapsed_time(e1) * 1e3)
        return statistics.median(times)

    def head_case(name, nbytes, launch, copies):
        for hb in sorted({1, min(B, 8)}):
            xh = synth.to_device({"x": synth.head_x(list(range(hb)))}, dev)["x"]
            y = torch.empty((hb, synth.VOCAB), dtype=torch.float32, device=dev)
            am = torch.empty(hb, dtype=torch.int32, device=dev)
            nbh = F.flint_gemv_workspace_bytes(synth.VOCAB, hb)
            wsh = torch.zeros(nbh, dtype=torch.uint8, device=dev)
            F.flint_workspace_init(wsh, nbh)
            us = rotating_us([lambda c=c: launch(c, xh, hb, y, am, wsh, nbh) for c in copies])
            extra[f"{name}_b{hb}"] = {"us": us, "GBps": nbytes / (us * 1e-6) / 1e9,
                                      "roofline_frac": nbytes / (us * 1e-6) / 1e9 / hbm,
                                      "bytes": nbytes}

    if not args.no_head and rank == 0:
        hq = synth.random_bytes_torch(0, synth.T_HEAD_Q, synth.VOCAB * H // 2, dev).view(
            synth.VOCAB, H // 2)
        hs_ = synth.to_device({"s": synth.head_host(with_codes=False)["s"]}, dev)["s"]
        copies = [(hq, hs_)] + [(hq.clone(), hs_.clone()) for _ in range(HEAD_COPIES - 1)]
        head_case("head_gemv", HEAD_BYTES,
                  lambda c, xh, hb, y, am, w, n: F.flint_int4_gemv(
                      c[0], c[1], synth.VOCAB, H, xh, hb, y, am, w, n, stream=stream), copies)
        del copies, hq, hs_
        # the group-64 affine int4 format (MLX int4 / Q4_1 layout)
        wa = synth.to_device(synth.affine_head_host(), dev)
        copies = [wa] + [{k: v.clone() for k, v in wa.items()} for _ in range(HEAD_COPIES - 1)]
        head_case("head_gemv_affine", synth.VOCAB * (1024 + 2 * 64),
                  lambda c, xh, hb, y, am, w, n: F.flint_int4_gemv_affine(
                      c["q"], c["s"], c["m"], synth.VOCAB, H, xh, hb, y, am, w, n,
                      stream=stream), copies)
        del copies, wa
        # NVFP4 (E2M1 codes, E4M3 scale per 16, fp32 global scale)
        wn = synth.nvfp4_head_host()
        wnd = synth.to_device({"q": wn["q"], "s": wn["s"]}, dev)
        copies = [wnd] + [{k: v.clone() for k, v in wnd.items()} for _ in range(HEAD_COPIES - 1)]
        head_case("head_gemv_nvfp4", synth.VOCAB * (1024 + 128),
                  lambda c, xh, hb, y, am, w, n: F.flint_int4_gemv_nvfp4(
                      c["q"], c["s"], wn["g"], synth.VOCAB, H, xh, hb, y, am, w, n,
                      stream=stream), copies)
        del copies, wnd
    # ---- prefill of one MoE layer (layer 0): tokens/s and tensor-pipe roofline
    if not args.no_prefill and rank == 0:
        peak_tf, peak_kind_tf = tensor_peak()
        for T in args.prefill_t:
            xt = synth.to_device({"x": synth.prefill_x(T, T)}, dev)["x"]
            out_t = torch.empty((T, H), dtype=torch.int16, device=dev)
            nbp = F.flint_workspace_bytes(F.FLINT_OP_PREFILL, T)
            wsp = torch.zeros(nbp, dtype=torch.uint8, device=dev)
            F.flint_workspace_init(wsp, nbp)
            # inputs larger than L2: the runs rotate over layers 0..2 (420 MB of
            # weights each), so no run finds its weights in L2
            pf_layers = structs[:min(3, nl)]
            us = rotating_us([lambda l=l: F.flint_moe_prefill(l, xt, T, out_t, wsp, nbp,
                                                              stream=stream)
                              for l in pf_layers], iters=8, skip=2, spin_cycles=2_000_000)
            tflops = T * PREFILL_FLOP_PER_TOKEN / (us * 1e-6) / 1e12
            # per-stage CUDA-event times inside the call (library measurement hook)
            stage_runs = []
            F.flint_debug_prefill_events(True)
            for it in range(3):
                with torch.cuda.stream(stream):
                    F.flint_moe_prefill(pf_layers[it % len(pf_layers)], xt, T, out_t, wsp, nbp,
                                        stream=stream)
                stage_runs.append(F.flint_debug_prefill_stage_ms())
            F.flint_debug_prefill_events(False)
            stages_us = {k: 1e3 * statistics.median(r[k] for r in stage_runs) for k in stage_runs[0]}
            g1_tf = T * GEMM1_FLOP_PER_TOKEN / (stages_us["gemm1"] * 1e-6) / 1e12
            g2_tf = T * GEMM2_FLOP_PER_TOKEN / (stages_us["gemm2"] * 1e-6) / 1e12
            gg_tf = (T * (GEMM1_FLOP_PER_TOKEN + GEMM2_FLOP_PER_TOKEN)
                     / ((stages_us["gemm1"] + stages_us["gemm2"]) * 1e-6) / 1e12)
            extra[f"prefill_T{T}"] = {"us": us, "tokens_per_s": T / (us * 1e-6),
                                      "TFLOPs": tflops, "tensor_frac": tflops / peak_tf,
                                      "peak_kind": peak_kind_tf, "stages_us": stages_us,
                                      "gemm1_TFLOPs": g1_tf, "gemm1_frac": g1_tf / peak_tf,
                                      "gemm2_TFLOPs": g2_tf, "gemm2_frac": g2_tf / peak_tf,
                                      "grouped_gemms_frac": gg_tf / peak_tf}
            for fmt_name, fmt_layers in (("affine", aff_pf), ("nvfp4", nv_pf)):
                if not fmt_layers:  # the same call on group-64 affine / NVFP4 experts
                    continue
                us_a = rotating_us([lambda l=l: F.flint_moe_prefill(l, xt, T, out_t, wsp, nbp,
                                                                    stream=stream)
                                    for l in fmt_layers], iters=8, skip=2, spin_cycles=2_000_000)
                tf_a = T * PREFILL_FLOP_PER_TOKEN / (us_a * 1e-6) / 1e12
                extra[f"prefill_{fmt_name}_T{T}"] = {"us": us_a, "tokens_per_s": T / (us_a * 1e-6),
                                                     "TFLOPs": tf_a, "tensor_frac": tf_a / peak_tf,
                                                     "peak_kind": peak_kind_tf}
            del wsp, out_t, xt
    sampler.stop()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(B)
        extra["cpu_baselines"] = cpu_baselines_other(B)

    line = {
        "metric": METRIC, "value": us_per_layer, "unit": "us/layer", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms / args.steps, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; weights as the workload recipe)",
        "config": dict(decode_config(B, nl),
                       stack_tokens_per_s=B * 1e6 / (us_per_layer * nl * world) * world,
                       mean_distinct_experts=U),
        "timing": timing,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm,
                     "traffic": DECODE_TRAFFIC_RATIO * bytes_per_layer,
                     "traffic_source": "scaled: this layer's algorithmic bytes x the DRAM/"
                                       "algorithmic ratio of one ncu capture of the same "
                                       "kernels (four stacked layers, batch 4)",
                     "kernel": "decode layer (3 PDL-chained kernels)",
                     "peak_kind": peak_kind, "bytes_per_layer": bytes_per_layer},
        "e2e": {"value": e2e_us, "unit": "us/layer", "h2d_bytes_per_step": B * H * 4,
                "d2h_bytes_per_step": B * H * 4},
        "gpu_launches": 3 * nl * args.steps,
        "clocks": clocks,
        "cpu_baseline": cpu,
        "extra": extra,
    }
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        del g, gw
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
