"""Benchmark of the B200 CodeQuant LUT MoE linear layer.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME|all] [--impl ours|reference]

Default: all five workloads in one run, each a "step" of layer calls on
seeded synthetic inputs with those models' layer shapes:
  linear_m1_k2048_n2048     one linear, M=1, K=N=2048, A4W4 (rotate+quantize,
                            LUT GEMV); a step = 128 calls, each on its own
                            weight copy (> 2 x the 126 MB L2)
  qwen3_4b_ffn_decode       Qwen3-4B-shaped dense SwiGLU FFN (2560 / 9728),
                            M in {1, 4, 16} x {A4W4, A8W4}, each on two weight
                            copies: 12 layer calls, 84 tokens per step
  qwen3_30b_a3b_moe_decode  128 experts, top-8, 64 tokens, A4W4
  mixtral_8x7b_moe          8 experts (one biased), top-2, 256 tokens, A8W4
  prefill_moe_e64_s2        64 routed + 2 shared experts, top-6, 4096 tokens
The JSON line's headline (value, roofline, e2e, cpu_baseline) is the prefill
MoE layer, the largest single-GPU configuration by work (567 GFLOP, 4096
tokens); the other four are blocks under "workloads" with the same keys.

Per workload:
  value       tokens/s of the whole job (sum over ranks / max time), device
              timed with CUDA events, inputs resident in HBM, the step
              replayed from a CUDA graph
  e2e         the same metric through the C-ABI calls with host buffers: every
              step's activations (and router logits) copied from pinned host
              memory and its outputs copied back inside the timed region, the
              steps pipelined as a serving loop runs them (the next step's
              inputs and the previous step's outputs move on two copy streams
              while a step computes)
  roofline    the dominant LUT GEMM kernel, from its CUDA-event-timed
              launches: the decode kernels (mma.sync, tensor-memory decode)
              as algorithmic bytes against the measured HBM copy peak, the
              wide-token-tile tensor-memory kernel as flops against the
              measured dense bf16 peak
  cpu_baseline  (headline) the CPU oracle on the host cores, bounded sample
Multi-GPU: replicas only (each rank runs the whole workload on its own GPU);
the timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "LUT-GEMV effective GB/s & MoE-FFN tokens/s; fraction of HBM/tensor roofline"


# ---------------------------------------------------------------------------
# workloads


def workload_shapes(name):
    import synth
    if name == "qwen3_4b_ffn_decode":
        # every variant twice, each call on its own weight copy: a step streams
        # 12 x 38 MB, more than twice the 126 MB L2
        return [dataclasses.replace(synth.cfg1(M, b), name=f"{synth.cfg1(M, b).name}_w{c}")
                for c in range(2) for (M, b) in synth.CFG1_VARIANTS]
    if name == "qwen3_30b_a3b_moe_decode":
        return [synth.CFG2]
    if name == "mixtral_8x7b_moe":
        return [synth.CFG3]
    if name == "prefill_moe_e64_s2":
        return [synth.CFG4]
    raise SystemExit(f"unknown workload {name}")


LINEAR = "linear_m1_k2048_n2048"
LINEAR_COPIES = 128            # 128 x 2.2 MB of weights per step (> 2 x L2)
WORKLOADS = [LINEAR, "qwen3_4b_ffn_decode", "qwen3_30b_a3b_moe_decode", "mixtral_8x7b_moe",
             "prefill_moe_e64_s2"]
HEADLINE = "prefill_moe_e64_s2"


def load_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), "measured"
    return 6650.0, 1590.0, "fallback"


def lut_alg_bytes(M, N, K, bits):
    """Algorithmic bytes of one LUT product: packed indices + codebooks +
    activation codes + scales + fp32 output."""
    return N * K // 2 + 32 * N + M * K * bits // 8 + 4 * M + 4 * M * N


def layer_alg(shape, counts=None):
    """(algorithmic bytes, flops) of one MoE / dense FFN layer call.  Only
    experts that receive at least one token count for weights."""
    s = shape
    T, H, I = s.T, s.H, s.I
    nbytes = 2 * T * H + 4 * T * H      # x in, out
    flops = 0
    groups = []
    if s.E:
        nbytes += 4 * T * s.E            # router logits
        for c in counts:
            if c > 0:
                groups.append((int(c), I))
    for _ in range(s.n_shared):
        groups.append((T, s.I_shared))
    for (m, i) in groups:
        nbytes += 2 * (i * H // 2 + 32 * i) + (H * i // 2 + 32 * H)
        flops += 2 * m * (2 * i * H + H * i)
    return nbytes, flops


def lut_launches(shape, counts=None):
    """(algorithmic bytes, flops) of every LUT GEMM launch in one layer call,
    in launch order: gate/up routed, gate/up shared, down routed, down shared."""
    s = shape
    T, H, I, bits = s.T, s.H, s.I, s.act_bits
    gu, dn = [], []
    if s.E:
        b_gu = b_dn = f_gu = f_dn = 0
        for c in counts:
            if c > 0:
                b_gu += lut_alg_bytes(int(c), 2 * I, H, bits)
                b_dn += lut_alg_bytes(int(c), H, I, bits)
                f_gu += 2 * int(c) * 2 * I * H
                f_dn += 2 * int(c) * H * I
        gu.append((b_gu, f_gu))
        dn.append((b_dn, f_dn))
    if s.n_shared:
        Is = s.I_shared
        gu.append((s.n_shared * lut_alg_bytes(T, 2 * Is, H, bits), s.n_shared * 2 * T * 2 * Is * H))
        dn.append((s.n_shared * lut_alg_bytes(T, H, Is, bits), s.n_shared * 2 * T * H * Is))
    return gu + dn


def lut_roofline(launch_alg, timed, steps, ms_step, peak_gbs, peak_tf, peak_kind):
    """Roofline entry of the dominant LUT GEMM kernel.  launch_alg: (bytes,
    flops) of each launch of one step, in launch order; timed: (kernel, ms) of
    every timed launch over `steps` steps.  The mma.sync kernel (decode) is
    bound by HBM: its algorithmic bytes over its time, against the copy peak.
    The tensor-memory kernel (prefill) is bound by the tensor pipe: its flops
    over its time, against the measured dense bf16 peak (fp16 runs at the
    same tensor-core rate)."""
    per = {}
    for i, (kern, ms) in enumerate(timed):
        b, f = launch_alg[i % len(launch_alg)]
        e = per.setdefault(kern, [0, 0.0, 0.0, 0])
        e[0] += b
        e[1] += f
        e[2] += ms
        e[3] += 1
    kern = max(per, key=lambda k: per[k][2])
    b, f, ms, n = per[kern]
    src = {"k_lut_mma": "kernels_lut.cu", "k_lut_tc": "kernels_lut_tc.cu",
           "k_lut_ts": "lut_ts.cuh"}[kern]
    common = {"kernel": kern, "avg_launch_us": 1e3 * ms / n, "launches_timed": n,
              "share_of_step": (ms / steps) / ms_step,
              "kernels_timed": {k: {"launches": v[3], "ms": v[2]} for k, v in per.items()}}
    if kern in ("k_lut_mma", "k_lut_ts"):
        a = b / (ms / 1e3) / 1e9
        return {"bound": "hbm", "achieved": a, "peak": peak_gbs, "unit": "GB/s",
                "frac": a / peak_gbs, "peak_source": f"{peak_kind} hbm_gbs",
                "alg_bytes_per_launch": b / n, **common}, src
    a = f / (ms / 1e3) / 1e12
    return {"bound": "tensor", "achieved": a, "peak": peak_tf, "unit": "TFLOP/s",
            "frac": a / peak_tf, "peak_source": f"{peak_kind} bf16_tflops (burst; fp16 = bf16 rate)",
            "alg_flops_per_launch": f / n, **common}, src


# ---------------------------------------------------------------------------
# helpers


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix="clk", suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not self.path:
            return None
        rows = []
        for line in Path(self.path).read_text().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]),
                                 power=float(parts[3]) if parts[3] not in ("[N/A]", "") else 0.0,
                                 hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        load = [r for r in rows if r["power"] > 200] or rows
        reasons = set()
        for r in load:
            for k, nm in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                          ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[k].lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(r["sm"] for r in load),
                "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows),
                "samples_under_load": len(load)}


def profile_traffic(kernel_src: Path, profile: Path):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source (its sha256 is recorded in the summary)."""
    if not profile.exists():
        return None
    txt = profile.read_text()
    m_sha = re.search(r"source_sha256:\s*([0-9a-f]{64})", txt)
    m_b = re.search(r"dram_bytes_per_launch_full:\s*([0-9.eE+]+)", txt)
    if not (m_sha and m_b):
        return None
    sha = hashlib.sha256(kernel_src.read_bytes()).hexdigest()
    if sha != m_sha.group(1):
        return None
    return float(m_b.group(1))


# ---------------------------------------------------------------------------
# the CPU oracle (baseline leg and reference arm)

WEIGHT_FIELDS = ("gate_idx", "up_idx", "down_idx", "gate_cb", "up_cb", "down_cb", "sh_gate_idx",
                 "sh_up_idx", "sh_down_idx", "sh_gate_cb", "sh_up_cb", "sh_down_cb")


def workload_inputs(name):
    """Host inputs of every layer call of one step, keyed by shape name."""
    import synth
    shapes = workload_shapes(name)
    out = {}
    if name == "qwen3_4b_ffn_decode":
        # one k-means weight set shared by the six variants (each variant gets
        # its own device copy in the timed loop)
        base = synth.moe_inputs(synth.cfg1(16, 4))
        for s in shapes:
            x = synth.activations(s.T, s.H, seed=0, name=f"{s.name}.x")
            out[s.name] = synth.MoEInputs(s, x, None, **{k: getattr(base, k) for k in WEIGHT_FIELDS})
    else:
        for s in shapes:
            out[s.name] = synth.moe_inputs(s)
    return shapes, out


def oracle_threads():
    try:
        return int(os.environ.get("OMP_NUM_THREADS") or len(os.sched_getaffinity(0)))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_oracle_sample(shapes, inputs, budget_s):
    """Run the CPU oracle layer on single tokens, cycling through the
    workload's layer calls, until budget_s has elapsed (at least one call).
    Returns (tokens, seconds, description)."""
    import oracle
    import synth
    oracle.build()
    t0 = time.perf_counter()
    ntok, names = 0, []
    while True:
        for s in shapes:
            inp = inputs[s.name]
            one = synth.MoEShape(**{**s.__dict__, "T": 1})
            sub = synth.MoEInputs(one, inp.x[:1],
                                  inp.logits[:1] if inp.logits is not None else None,
                                  **{k: getattr(inp, k) for k in WEIGHT_FIELDS})
            oracle.moe_ffn(sub, one)
            ntok += 1
            names.append(s.name)
            if time.perf_counter() - t0 >= budget_s:
                break
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    desc = (f"{ntok} single-token layer calls ({', '.join(sorted(set(names)))}) "
            f"of the C oracle, {dt:.1f} s")
    return ntok, dt, desc


def run_reference(args):
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    shapes, inputs = workload_inputs(args.workload)
    for _ in range(args.warmup):
        cpu_oracle_sample(shapes, inputs, 0.0)
    tok = sec = 0.0
    for _ in range(args.steps):
        n, dt, desc = cpu_oracle_sample(shapes, inputs, args.ref_step_seconds)
        tok += n
        sec += dt
    v = tok / sec
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * sec / max(args.steps, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": oracle_threads(),
                         "kind": "oracle",
                         "sample": f"per step: single-token oracle layer calls for "
                                   f"~{args.ref_step_seconds:.0f} s, cycling through the "
                                   f"workload's layer calls"},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm


class DeviceLayer:
    """One layer call with every tensor resident on the device, plus pinned
    host copies of its activations / logits / output for the e2e leg."""

    def __init__(self, cq, inp, dev):
        import torch
        s = inp.shape
        self.s = s
        self.cfg = cq.MoEConfig(H=s.H, I=s.I, E=s.E, top_k=s.top_k, n_shared=s.n_shared,
                                I_shared=s.I_shared, act_bits=s.act_bits,
                                had_block_h=s.had_block_h, had_block_i=s.had_block_i,
                                had_block_i_shared=s.had_block_i_shared,
                                renormalize=s.renormalize)
        self.w = {k: torch.from_numpy(np.ascontiguousarray(getattr(inp, k))).to(dev)
                  for k in WEIGHT_FIELDS if getattr(inp, k) is not None}
        self.x = torch.from_numpy(inp.x).to(dev)
        self.lg = torch.from_numpy(inp.logits).to(dev) if s.E else None
        self.out = torch.empty((s.T, s.H), dtype=torch.float32, device=dev)
        self.call = cq.MoELayer(self.cfg, s.T, self.w, dev)
        self.x_h = torch.from_numpy(inp.x).pin_memory()
        self.lg_h = torch.from_numpy(inp.logits).pin_memory() if s.E else None
        self.out_h = torch.empty((s.T, s.H), dtype=torch.float32).pin_memory()
        self.h2d = self.x_h.numel() * 2 + (self.lg_h.numel() * 4 if s.E else 0)
        self.d2h = self.out_h.numel() * 4

    def run(self):
        self.call(self.x, self.lg, self.out)

    # e2e: two device buffer sets, so one step's copies overlap another's compute
    def e2e_buffers(self):
        import torch
        self.xb = [self.x, torch.empty_like(self.x)]
        self.lgb = [self.lg, torch.empty_like(self.lg) if self.lg is not None else None]
        self.outb = [self.out, torch.empty_like(self.out)]

    def h2d_into(self, b):
        self.xb[b].copy_(self.x_h, non_blocking=True)
        if self.lg is not None:
            self.lgb[b].copy_(self.lg_h, non_blocking=True)

    def run_buf(self, b):
        self.call(self.xb[b], self.lgb[b], self.outb[b])

    def d2h_from(self, b):
        self.out_h.copy_(self.outb[b], non_blocking=True)

    def counts(self, dev):
        """Per-expert token counts of this call (for the byte accounting)."""
        import torch
        if not self.s.E:
            return None
        c = torch.zeros((self.s.E,), dtype=torch.int32, device=dev)
        self.call(self.x, self.lg, self.out, debug={"counts": c})
        return c.cpu().numpy()


def max_over_ranks(ms, dist, world, device="cuda"):
    """The slowest rank's time: every rank gets the max (replicas are timed
    on the device and the job is as slow as its slowest GPU)."""
    if world <= 1:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_step, steps, world, ms):
    """Whole-job rate: the units all ranks processed over the max-over-ranks time."""
    return units_per_step * steps * world / (ms / 1e3)


def bf16_dense_context(shapes, dev, stream, steps, warmup, dist, world):
    """tokens/s of the same dense SwiGLU FFN calls done in bf16 by torch
    (F.linear on dense weights, one weight copy per call), replayed from a
    CUDA graph and timed like the main leg."""
    import torch
    import torch.nn.functional as F
    g = torch.Generator(device=dev).manual_seed(0)
    calls = []
    for s in shapes:
        wgu = torch.randn((2 * s.I_shared, s.H), generator=g, device=dev, dtype=torch.bfloat16)
        wd = torch.randn((s.H, s.I_shared), generator=g, device=dev, dtype=torch.bfloat16)
        x = torch.randn((s.T, s.H), generator=g, device=dev, dtype=torch.bfloat16)
        calls.append((x, wgu.mul_(0.02), wd.mul_(0.02), s.I_shared))

    def step():
        for x, wgu, wd, i in calls:
            gu = F.linear(x, wgu)
            F.linear(F.silu(gu[:, :i]) * gu[:, i:], wd)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    for _ in range(warmup):
        graph.replay()
    ms = timed(graph.replay, steps, dist, world)
    tokens = sum(s.T for s in shapes)
    return {"value": job_throughput(tokens, steps, world, ms), "unit": "tokens/s",
            "ms_per_step": ms / steps,
            "what": "torch bf16 F.linear dense SwiGLU FFN, same shapes and tokens, "
                    "own dense weight copy per call, CUDA graph"}


def timed(fn, steps, dist, world):
    """Device time (ms) of `steps` calls of fn on the current stream,
    bracketed by barrier + synchronize on both sides; max over ranks."""
    import torch
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(steps):
        fn()
    e1.record(st)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    return max_over_ranks(e0.elapsed_time(e1), dist, world)


class BatchedIO:
    """The host I/O of many small calls batched the way a caller serving them
    would: their inputs and outputs as views of one contiguous pinned host
    buffer and one device buffer per buffer set, so a step copies once each
    way.  `calls` expose x_h / y_h (host) and take device views through
    set_views(b, x, y)."""

    def __init__(self, calls):
        import torch
        self.calls = calls
        c0 = calls[0]
        n = len(calls)
        self.x_h = torch.stack([c.x_h for c in calls]).pin_memory()
        self.y_h = torch.empty((n,) + tuple(c0.y_h.shape), dtype=c0.y_h.dtype).pin_memory()
        dev = c0.x.device
        self.xd = [torch.empty(self.x_h.shape, dtype=self.x_h.dtype, device=dev) for _ in range(2)]
        self.yd = [torch.empty(self.y_h.shape, dtype=self.y_h.dtype, device=dev) for _ in range(2)]

    def e2e_buffers(self):
        for i, c in enumerate(self.calls):
            c.set_views([self.xd[0][i], self.xd[1][i]], [self.yd[0][i], self.yd[1][i]])

    def h2d_into(self, b):
        self.xd[b].copy_(self.x_h, non_blocking=True)

    def run_buf(self, b):
        for c in self.calls:
            c.run_buf(b)

    def d2h_from(self, b):
        self.y_h.copy_(self.yd[b], non_blocking=True)


def timed_e2e(calls, steps, warmup, dist, world):
    """Device time (ms) of `steps` end-to-end steps: every step copies its
    inputs from pinned host memory, runs the calls and copies its outputs back.
    Steps are pipelined the way a serving loop runs them: step s + 1's inputs
    go in on one copy stream and step s's outputs come out on another while
    step s computes (two device buffer sets).  The timed region opens before
    the first input copy and closes after the last output copy."""
    import torch
    for c in calls:
        c.e2e_buffers()
    comp = torch.cuda.current_stream()
    cin, cout = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()

    def run(n, e_start=None):
        inp = [ev(), ev()]      # inputs of buffer set b are on the device
        done = [None, None]     # compute on buffer set b finished
        outd = [None, None]     # outputs of buffer set b copied out
        if e_start is not None:
            cin.wait_event(e_start)
        for s in range(n):
            b = s & 1
            if done[b] is not None:
                cin.wait_event(done[b])         # buffer set b's inputs no longer read
            with torch.cuda.stream(cin):
                for c in calls:
                    c.h2d_into(b)
            inp[b] = ev()
            inp[b].record(cin)
            comp.wait_event(inp[b])
            if outd[b] is not None:
                comp.wait_event(outd[b])        # buffer set b's outputs copied out
            for c in calls:
                c.run_buf(b)
            done[b] = ev()
            done[b].record(comp)
            cout.wait_event(done[b])
            with torch.cuda.stream(cout):
                for c in calls:
                    c.d2h_from(b)
            outd[b] = ev()
            outd[b].record(cout)
        comp.wait_stream(cout)
        comp.wait_stream(cin)

    run(warmup)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    run(steps, e0)
    e1.record(comp)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    return max_over_ranks(e0.elapsed_time(e1), dist, world)


class LinearCall:
    """One linear call of the single-linear workload (rotate+quantize, then the
    LUT GEMV), every tensor resident, plus pinned host copies for e2e."""

    def __init__(self, cq, shape, x, w, cb, dev):
        import torch
        self.cq, self.s = cq, shape
        self.x = torch.from_numpy(x).to(dev)
        self.w, self.cb = w, cb
        self.q = torch.empty((shape.M, shape.K // 2 if shape.act_bits == 4 else shape.K),
                             dtype=torch.uint8 if shape.act_bits == 4 else torch.int8, device=dev)
        self.sx = torch.empty((shape.M,), dtype=torch.float32, device=dev)
        self.y = torch.empty((shape.M, shape.N), dtype=torch.float32, device=dev)
        nb = cq.cq_lut_gemm_workspace_size(shape.M, shape.N, shape.K, shape.act_bits)
        self.ws = torch.empty((max(nb, 1),), dtype=torch.uint8, device=dev)
        self.x_h = torch.from_numpy(x).pin_memory()
        self.y_h = torch.empty((shape.M, shape.N), dtype=torch.float32).pin_memory()
        self.h2d, self.d2h = self.x_h.numel() * 2, self.y_h.numel() * 4

    def run(self):
        s = self.s
        self.cq.cq_rotate_quantize(self.x, s.had_block, s.act_bits, q_out=self.q, s_out=self.sx)
        self.cq.cq_lut_gemm(self.q, self.sx, s.K, s.act_bits, self.w, self.cb, y=self.y,
                            workspace=self.ws)

    def set_views(self, xb, yb):
        self.xb, self.yb = xb, yb

    def run_buf(self, b):
        s = self.s
        self.cq.cq_rotate_quantize(self.xb[b], s.had_block, s.act_bits, q_out=self.q, s_out=self.sx)
        self.cq.cq_lut_gemm(self.q, self.sx, s.K, s.act_bits, self.w, self.cb, y=self.yb[b],
                            workspace=self.ws)


def lut_timed_launches(cq, step, steps, every_kernel=False):
    """Every LUT GEMM launch (every launch of the library with every_kernel)
    of `steps` eager steps, CUDA-event timed on its stream.  A spin kernel
    ahead of every step keeps the GPU busy while the host queues the step, so
    consecutive kernels run back to back and no launch's events include time
    the GPU spent waiting for the host."""
    import torch
    t_host = time.perf_counter()
    step()
    torch.cuda.synchronize()
    t_host = time.perf_counter() - t_host
    spin_cycles = int(min(50e-3, 3 * t_host + 1e-3) * 2.0e9)
    cq.cq_timing_read_launches()  # drop anything recorded before
    cq.cq_timing_enable(True, every_kernel=every_kernel)
    for _ in range(steps):
        torch.cuda._sleep(spin_cycles)
        step()
    torch.cuda.synchronize()
    cq.cq_timing_enable(False)
    return cq.cq_timing_read_launches()


def kernel_breakdown(launches, steps):
    """Device time per step of each kernel kind, every launch of the library
    event-timed (eager steps; the events cost a few microseconds per launch
    and stop consecutive kernels from overlapping, so the sum exceeds the
    graph-replayed step time)."""
    per = {}
    for k, ms in launches:
        e = per.setdefault(k, [0, 0.0])
        e[0] += 1
        e[1] += ms
    total = sum(v[1] for v in per.values()) or 1.0
    out = {k: {"launches_per_step": v[0] / steps, "us_per_step": 1e3 * v[1] / steps,
               "share": v[1] / total} for k, v in sorted(per.items(), key=lambda kv: -kv[1][1])}
    return {"kernels": out, "us_per_step_sum": 1e3 * total / steps,
            "method": "CUDA events around every launch of the library, eager steps"}


def lut_alg_bytes_bits(M, N, K, bits, idx_bits):
    """Algorithmic bytes of one LUT product with 2^idx_bits centroids per row."""
    return N * K * idx_bits // 8 + 2 * (1 << idx_bits) * N + M * K * bits // 8 + 4 * M + 4 * M * N


def measure_codebook_sizes(cq, args, dev, peaks, copies=3):
    """GB/s of the LUT GEMM per codebook size (8 / 16 / 32 centroids per row)
    on the Qwen3-4B-shaped FFN linears (gate||up 2560 -> 19456 and down
    9728 -> 2560) at M = 1 and 16, A4: every launch CUDA-event timed, each
    call on its own weight copy (copies x the shapes > the 126 MB L2).  The
    kernels' work does not depend on the values: indices are uniform random,
    codebooks sorted N(0, 0.02^2) draws."""
    import torch
    peak_gbs = peaks[0]
    g = np.random.default_rng(0)
    out = {}
    for b in (3, 4, 5):
        calls = []
        for (M, K, N) in [(1, 2560, 19456), (1, 9728, 2560), (16, 2560, 19456), (16, 9728, 2560)]:
            q = torch.from_numpy(g.integers(0, 256, (M, K // 2), dtype=np.uint8)).to(dev)
            sx = torch.full((M,), 1e-2, dtype=torch.float32, device=dev)
            for _ in range(copies):
                w = torch.from_numpy(g.integers(0, 256, (N, K * b // 8), dtype=np.uint8)).to(dev)
                cbk = torch.from_numpy(np.sort(g.standard_normal((N, 1 << b)) * 0.02, axis=1)
                                       .astype(np.float16)).to(dev)
                y = torch.empty((M, N), dtype=torch.float32, device=dev)
                nb = cq.cq_lut_gemm_ex_workspace_size(M, N, K, 4, b)
                ws = torch.empty((max(nb, 1),), dtype=torch.uint8, device=dev)
                calls.append((q, sx, K, w, cbk, y, ws, lut_alg_bytes_bits(M, N, K, 4, b)))

        def step():
            for (q, sx, K, w, cbk, y, ws, _) in calls:
                cq.cq_lut_gemm_ex(q, sx, K, 4, w, b, cbk, y=y, workspace=ws)
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        launches = lut_timed_launches(cq, step, args.steps)
        assert len(launches) == args.steps * len(calls)
        ms = sum(m for _, m in launches)
        nbytes = args.steps * sum(c[-1] for c in calls)
        gbs = nbytes / (ms / 1e3) / 1e9
        out[str(1 << b)] = {"idx_bits": b, "kernel": sorted({k for k, _ in launches}),
                            "achieved": gbs, "unit": "GB/s", "peak": peak_gbs,
                            "frac": gbs / peak_gbs, "launches_timed": len(launches),
                            "avg_launch_us": 1e3 * ms / len(launches),
                            "alg_bytes_per_step": nbytes // args.steps}
        del calls
        torch.cuda.empty_cache()
    return out


def decoder_layer_vs_bf16(cq, args, dev, stream, dist, world, ctx=1024, n_layers=4):
    """Decode step of n_layers Qwen3-4B-shaped decoder layers (hidden 2560, 32
    query / 8 key-value heads of 128, intermediate 9728, a KV cache of ctx
    tokens per sequence, M sequences decoding one token each), once with the
    linears as this library's LUT layers (QKV and O through
    cq_rotate_quantize + cq_lut_gemm, the SwiGLU FFN through cq_moe_ffn, A4W4)
    and once all in bf16 (torch F.linear).  RMSNorm, rotary embedding and
    attention (torch scaled_dot_product_attention) are the same torch code in
    both, in fp16 / bf16.  Weights are random (the work does not depend on
    their values); each of the n_layers layers has its own, so a step streams
    more than the L2.  Both steps are replayed from CUDA graphs."""
    import torch
    import torch.nn.functional as F
    H, I, nq, nkv, hd = 2560, 9728, 32, 8, 128
    g = torch.Generator(device=dev).manual_seed(0)

    def rnd_idx(n, k):
        return torch.randint(0, 256, (n, k // 2), dtype=torch.uint8, device=dev, generator=g)

    def rnd_cb(n):
        return (torch.randn((n, 16), device=dev, generator=g) * 0.02).sort(dim=1)[0].half()

    def rms(x, w):
        xf = x.float()
        return (xf * torch.rsqrt(xf.pow(2).mean(-1, keepdim=True) + 1e-6) * w).to(x.dtype)

    pos = torch.arange(hd // 2, device=dev, dtype=torch.float32)
    ang = ctx * (1e6 ** (-2 * pos / hd))
    cos, sin = torch.cos(ang), torch.sin(ang)

    def rope(t):
        a, b = t.float()[..., : hd // 2], t.float()[..., hd // 2:]
        return torch.cat([a * cos - b * sin, a * sin + b * cos], -1).to(t.dtype)

    def attention(qkv, kc, vc, M, dt):
        q = rope(qkv[:, : nq * hd].to(dt).view(M, nq, 1, hd))
        k = rope(qkv[:, nq * hd:(nq + nkv) * hd].to(dt).view(M, nkv, 1, hd))
        v = qkv[:, (nq + nkv) * hd:].to(dt).view(M, nkv, 1, hd)
        kc[:, :, ctx:ctx + 1] = k
        vc[:, :, ctx:ctx + 1] = v
        o = F.scaled_dot_product_attention(q, kc, vc, enable_gqa=True)
        return o.reshape(M, nq * hd)

    out = {}
    for M in (1, 16):
        lut_layers, bf_layers = [], []
        for _ in range(n_layers):
            nqkv = (nq + 2 * nkv) * hd
            w = {"sh_gate_idx": rnd_idx(I, H)[None], "sh_up_idx": rnd_idx(I, H)[None],
                 "sh_down_idx": rnd_idx(H, I)[None], "sh_gate_cb": rnd_cb(I)[None],
                 "sh_up_cb": rnd_cb(I)[None], "sh_down_cb": rnd_cb(H)[None]}
            cfg = cq.MoEConfig(H=H, I=I, E=0, top_k=0, n_shared=1, I_shared=I, act_bits=4,
                               had_block_h=512, had_block_i=256, had_block_i_shared=256)
            lut_layers.append(dict(
                wqkv=rnd_idx(nqkv, H), cqkv=rnd_cb(nqkv), wo=rnd_idx(H, nq * hd), co=rnd_cb(H),
                ffn=cq.MoELayer(cfg, M, w, dev), w=w,
                kc=torch.randn((M, nkv, ctx + 1, hd), device=dev, generator=g).half(),
                vc=torch.randn((M, nkv, ctx + 1, hd), device=dev, generator=g).half(),
                n1=torch.ones(H, device=dev), n2=torch.ones(H, device=dev),
                y=torch.empty((M, H), dtype=torch.float32, device=dev)))
            bf_layers.append(dict(
                wqkv=(torch.randn((nqkv, H), device=dev, generator=g) * 0.02).bfloat16(),
                wo=(torch.randn((H, nq * hd), device=dev, generator=g) * 0.02).bfloat16(),
                wgu=(torch.randn((2 * I, H), device=dev, generator=g) * 0.02).bfloat16(),
                wd=(torch.randn((H, I), device=dev, generator=g) * 0.02).bfloat16(),
                kc=torch.randn((M, nkv, ctx + 1, hd), device=dev, generator=g).bfloat16(),
                vc=torch.randn((M, nkv, ctx + 1, hd), device=dev, generator=g).bfloat16(),
                n1=torch.ones(H, device=dev), n2=torch.ones(H, device=dev)))
        x_lut = torch.randn((M, H), device=dev, generator=g).half()
        x_bf = x_lut.bfloat16()

        def lut_step():
            x = x_lut
            for L in lut_layers:
                qc, sq = cq.cq_rotate_quantize(rms(x, L["n1"]), 512, 4)
                qkv = cq.cq_lut_gemm(qc, sq, H, 4, L["wqkv"], L["cqkv"])
                a = attention(qkv, L["kc"], L["vc"], M, torch.float16)
                oc, so = cq.cq_rotate_quantize(a.contiguous(), 4096, 4)
                x1 = x + cq.cq_lut_gemm(oc, so, nq * hd, 4, L["wo"], L["co"]).half()
                L["ffn"](rms(x1, L["n2"]).contiguous(), None, L["y"])
                x = x1 + L["y"].half()
            return x

        def bf_step():
            x = x_bf
            for L in bf_layers:
                qkv = F.linear(rms(x, L["n1"]), L["wqkv"])
                a = attention(qkv, L["kc"], L["vc"], M, torch.bfloat16)
                x1 = x + F.linear(a, L["wo"])
                gu = F.linear(rms(x1, L["n2"]), L["wgu"])
                x = x1 + F.linear(F.silu(gu[:, :I]) * gu[:, I:], L["wd"])
            return x

        res = {}
        for nm, fn in (("lut", lut_step), ("bf16", bf_step)):
            for _ in range(args.warmup):
                fn()
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                fn()
            for _ in range(args.warmup):
                graph.replay()
            ms = timed(graph.replay, args.steps, dist, world)
            res[nm] = {"tokens_per_s": job_throughput(M, args.steps, world, ms),
                       "ms_per_step": ms / args.steps}
            del graph
        out[f"M{M}"] = {**res, "speedup_vs_bf16": res["lut"]["tokens_per_s"] /
                        res["bf16"]["tokens_per_s"]}
        del lut_layers, bf_layers
        torch.cuda.empty_cache()
    out["config"] = {"model": "Qwen3-4B-shaped decoder layers (random weights)",
                     "layers_per_step": n_layers, "kv_context": ctx, "heads": [nq, nkv, hd],
                     "lut": "A4W4, QKV / O / FFN through the C ABI; attention torch fp16",
                     "bf16": "torch F.linear, attention torch bf16"}
    return out


def measure(cq, name, args, dev, stream, dist, world, peaks):
    """One workload: the step resident (graph replay), the LUT kernel launch by
    launch, and the step end to end from host buffers.  Returns its block."""
    import torch
    import synth
    peak_gbs, peak_tf, peak_kind = peaks
    cpu_in = None
    if name == LINEAR:
        s = synth.CFG0
        x, w_idx, cb = synth.linear_inputs(s)
        w0 = torch.from_numpy(w_idx).to(dev)
        c0 = torch.from_numpy(cb).to(dev)
        calls = [LinearCall(cq, s, synth.activations(s.M, s.K, seed=0, name=f"{s.name}.x{i}"),
                            w0.clone(), c0.clone(), dev) for i in range(LINEAR_COPIES)]
        del w0, c0
        units_per_step = LINEAR_COPIES * s.M
        launch_alg = [(lut_alg_bytes(s.M, s.N, s.K, s.act_bits), 2 * s.M * s.N * s.K)]
        launch_alg *= LINEAR_COPIES
        alg_bytes_step = sum(b for b, _ in launch_alg) + LINEAR_COPIES * 2 * s.M * s.K
        alg_flops_step = sum(f for _, f in launch_alg)
        cfg = {"workload": name, "calls_per_step": LINEAR_COPIES, "M": s.M, "K": s.K, "N": s.N,
               "had_block": s.had_block, "act_bits": s.act_bits,
               "weights": "one k-means weight set, a device copy per call"}
    else:
        shapes, cpu_in = workload_inputs(name)
        calls = [DeviceLayer(cq, cpu_in[sh.name], dev) for sh in shapes]
        units_per_step = sum(sh.T for sh in shapes)
        counts = [L.counts(dev) for L in calls]
        launch_alg = [a for L, c in zip(calls, counts) for a in lut_launches(L.s, c)]
        alg_bytes_step = sum(layer_alg(L.s, c)[0] for L, c in zip(calls, counts))
        alg_flops_step = sum(layer_alg(L.s, c)[1] for L, c in zip(calls, counts))
        cfg = {"workload": name, "layers_per_step": [sh.name for sh in shapes]}

    def step():
        for c in calls:
            c.run()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    n0 = cq.cq_launch_count()
    step()
    torch.cuda.synchronize()
    launches_per_step = cq.cq_launch_count() - n0

    # ---- timed region: device-resident inputs, CUDA-graph replay of the step
    use_graph = not args.no_graph
    if use_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step()
        run = graph.replay
    else:
        run = step
    for _ in range(args.warmup):
        run()
    local = torch.cuda.current_device()
    with ClockSampler(local) as clk:
        ms = timed(run, args.steps, dist, world)
    clocks = clk.summary()
    ms_step = ms / args.steps
    value = job_throughput(units_per_step, args.steps, world, ms)

    # ---- the LUT GEMM kernel, launch by launch
    timed_launches = lut_timed_launches(cq, step, args.steps)
    assert len(timed_launches) == args.steps * len(launch_alg), (len(timed_launches), len(launch_alg))
    roofline, kern_src = lut_roofline(launch_alg, timed_launches, args.steps, ms_step,
                                      peak_gbs, peak_tf, peak_kind)
    roofline["traffic"] = profile_traffic(ROOT / "lut_clustered_weight_b200" / "csrc" / kern_src,
                                          ROOT / "profiles" / f"{roofline['kernel']}_{name}.md")
    breakdown = kernel_breakdown(lut_timed_launches(cq, step, args.steps, every_kernel=True),
                                 args.steps)

    # ---- e2e: host buffers through the C-ABI, copies inside the timed region
    io = [BatchedIO(calls)] if name == LINEAR else calls
    ms_e2e = timed_e2e(io, args.steps, args.warmup, dist, world)
    e2e = {"value": job_throughput(units_per_step, args.steps, world, ms_e2e), "unit": "tokens/s",
           "h2d_bytes_per_step": sum(c.h2d for c in calls),
           "d2h_bytes_per_step": sum(c.d2h for c in calls), "ms_per_step": ms_e2e / args.steps,
           "pipelining": "step s+1's inputs in and step s's outputs out on two copy streams "
                         "while step s computes (two device buffer sets)"}

    cfg.update({"tokens_per_step": units_per_step, "cuda_graph": use_graph,
                "l2": "no flush: each step streams "
                      f"{alg_bytes_step / 1e6:.0f} MB of distinct weights (> 126 MB L2)",
                "parallelism": f"replicas x{world}"})
    block = {"value": value, "unit": "tokens/s", "ms_per_step": ms_step, "config": cfg,
             "effective_gbs": alg_bytes_step / (ms_step / 1e3) / 1e9,
             "alg_bytes_per_step": alg_bytes_step, "alg_flops_per_step": alg_flops_step,
             "roofline": roofline, "kernel_breakdown": breakdown, "e2e": e2e,
             "gpu_launches": launches_per_step * args.steps, "clocks": clocks}

    # ---- context: the same dense FFN step in bf16 with torch (the pages
    # compare their decode kernel against BF16)
    if name != LINEAR and all(sh.E == 0 for sh in shapes) and not args.no_bf16:
        bf16 = bf16_dense_context(shapes, dev, stream, args.steps, args.warmup, dist, world)
        bf16["speedup_of_value"] = value / bf16["value"]
        block["bf16_context"] = bf16
    if name == "qwen3_4b_ffn_decode" and not args.no_bf16:
        block["decoder_layer_vs_bf16"] = decoder_layer_vs_bf16(cq, args, dev, stream, dist, world)
    if name == LINEAR and not args.no_codebook_sizes:
        block["codebook_sizes"] = measure_codebook_sizes(cq, args, dev, peaks)
    if use_graph:
        del graph
    del calls
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return block, cpu_in


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="all", choices=["all"] + WORKLOADS)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-graph", action="store_true", help="time eager calls, not a CUDA graph")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-step-seconds", type=float, default=4.0)
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline leg")
    ap.add_argument("--no-bf16", action="store_true", help="skip the torch bf16 context leg")
    ap.add_argument("--no-codebook-sizes", action="store_true",
                    help="skip the GB/s-per-codebook-size leg (8 / 16 / 32 centroids)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    headline = HEADLINE if args.workload == "all" else args.workload
    if args.impl == "reference":
        if headline == LINEAR:
            raise SystemExit("the reference arm times the layer workloads")
        args.workload = headline
        return run_reference(args)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    import lut_clustered_weight_b200 as cq

    peaks = load_peaks()
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)

    names = WORKLOADS if args.workload == "all" else [args.workload]
    blocks, head_inputs = {}, None
    for name in names:
        blocks[name], cpu_in = measure(cq, name, args, dev, stream, dist, world, peaks)
        if name == headline:
            head_inputs = cpu_in
    head = blocks.pop(headline)

    # ---- CPU oracle baseline of the headline workload (rank 0, one GPU only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu and headline != LINEAR:
        import oracle
        shapes = workload_shapes(headline)
        n, dt, desc = cpu_oracle_sample(shapes, head_inputs, args.cpu_seconds)
        cpu = {"value": n / dt, "unit": "tokens/s", "cores": oracle_threads(), "kind": "oracle",
               "sample": desc}
        oracle.set_threads(1)
        n1, dt1, desc1 = cpu_oracle_sample(shapes, head_inputs, args.cpu_seconds / 3)
        oracle.set_threads(oracle_threads())
        cpu["single_thread"] = {"value": n1 / dt1, "unit": "tokens/s", "cores": 1,
                                "sample": desc1}

    if world > 1:
        dist.barrier()
    if rank == 0:
        line = {
            "metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f16", "data": "synthetic", "config": head["config"],
            "effective_gbs": head["effective_gbs"],
            "alg_bytes_per_step": head["alg_bytes_per_step"],
            "alg_flops_per_step": head["alg_flops_per_step"],
            "roofline": head["roofline"], "cpu_baseline": cpu, "e2e": head["e2e"],
            "gpu_launches": head["gpu_launches"], "clocks": head["clocks"],
            "workloads": blocks,
            "dtype_note": "int4/int8 codes and 4-bit indices; looked-up weights as fp16 "
                          "into mma.sync or tcgen05 kind::f16 (tensor memory A operand) with "
                          "fp32 accumulation; rotation exact in fp64",
        }
        for extra in ("kernel_breakdown", "bf16_context", "codebook_sizes", "decoder_layer_vs_bf16"):
            if extra in head:
                line[extra] = head[extra]
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
