"""Benchmark of the W2A8 BitLinear forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline (value): decode GEMV throughput in algorithmic GB/s at M = 1 over the 2B-4T
projection shapes (N, K) in {(2560,2560), (640,2560), (6912,2560), (2560,6912)}, ternary
weights P(0) = 0.4, s_w ~ U(0.5, 2), x ~ N(0, 1). One step = bitnet_linear on every shape
for each of R weight replicas (R chosen so the step's packed weights exceed 2x L2), run
as one CUDA graph. Second number (gemm): prefill GEMM int8 TOPS at M = 2048 on the same
shapes (Student-t activations with outlier channels, ternary P(0) = 0.5).

Timing: W untimed warm-up steps, then K steps; L2 is flushed (a 256 MB write) before every
step, outside the step's CUDA-event pair; per-step event times are summed; ranks meet at a
barrier with a device synchronize on both sides and rank 0 reports the max over ranks.
Multi-GPU (torchrun): every rank runs its own replica of the workload (weak scaling, no
data-path collective).

--impl reference times the CPU oracle (plain C, one thread) on a bounded sample of the same
workload on this machine's host cores: the only reference implementation there is.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "W2A8 ternary GEMV HBM GB/s (M=1) and GEMM int8 TOPS (M>=512) vs roofline"
L2_BYTES = 126 * 1024 * 1024
DECODE_M = 1
PREFILL_M = 2048
PREFILL_M_SMALL = 512  # the prefill configuration's other token count
# nominal dense int8 : bf16 tensor-core ratio on B200 (4.5 vs 2.25 PFLOP/s)
INT8_PER_BF16 = 2.0


# DRAM bytes per decode-sweep GEMV launch, read + write, from one ncu capture of the four
# shapes with the current kernel (2560 x 2560, 640 x 2560, 6912 x 2560, 2560 x 6912 at M = 1:
# 1659648, 430592, 4455424, 4454912 bytes), averaged.
GEMV_DECODE_TRAFFIC_BYTES = 2750144
# DRAM bytes per prefill GEMM launch (tc_gemm_kernel, M = 2048), read + write, from one ncu
# capture of the four shapes (6979328, 5748736, 9764352, 18681344 bytes), averaged. The bf16
# outputs stay in L2 while the kernel runs (written back after it ends), so this is below the
# algorithmic bytes: packed weights + int8 tokens + outputs.
GEMM_PREFILL_TRAFFIC_BYTES = 10293440


def decode_bytes(M, N, K):
    """Algorithmic bytes of one BitLinear call: packed W + x + y + s_w (per tensor)."""
    return N * K // 4 + 2 * M * K + 2 * M * N + 4


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d["bf16_tflops_sustained"]), "src": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "src": "fallback"}


# ---------------------------------------------------------------------------- ranks
def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def reduce_over_ranks(local_ms: float, local_units: float, world: int):
    """Max of the per-rank time and sum of the per-rank work (the job's aggregate)."""
    if world <= 1:
        return local_ms, local_units
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([local_ms], dtype=torch.float64, device=dev)
    u = torch.tensor([local_units], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read-only) every 5 ms while
    `active` is set; timed_steps sets it around every timed region."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, index: int):
        self.index = index
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = None
        import threading
        self.active = threading.Event()

    def _run(self):
        import pynvml
        try:
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            while not self._stop.is_set():
                if self.active.is_set():
                    self.samples.append(
                        float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)))
                    bits = pynvml.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                    for name, bit in self.REASONS.items():
                        if bits & bit:
                            self.reasons.add(name)
                self._stop.wait(0.005)
        except Exception as e:  # sampling is best effort; the line says so
            self.error = repr(e)

    def __enter__(self):
        import threading
        self._stop = threading.Event()
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        self._t.join(timeout=5)
        return False

    def summary(self):
        d = {"sm_mhz": statistics.median(self.samples) if self.samples else None,
             "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
             "samples": len(self.samples)}
        if getattr(self, "error", None):
            d["error"] = self.error
        return d


# ---------------------------------------------------------------------------- workloads
def build_decode(bn, torch, replicas: int, dev):
    """Per replica and shape: packed weights, s_w, x, y (all resident in HBM)."""
    calls = []
    for r in range(replicas):
        for si in range(len(synth.SWEEP_SHAPES)):
            c = synth.decode_case(si, replica=r, M=DECODE_M)
            packed = bn.bitnet_pack_ternary(torch.from_numpy(c["t"]).to(dev))
            s_w = torch.from_numpy(c["s_w"]).to(dev)
            x = torch.from_numpy(c["x"].view(np.int16).copy()).to(dev).view(torch.bfloat16)
            y = torch.empty((DECODE_M, c["N"]), dtype=torch.bfloat16, device=dev)
            calls.append({"x": x, "packed": packed, "s_w": s_w, "y": y, "N": c["N"], "K": c["K"]})
    return calls


def build_prefill(bn, torch, dev, M):
    calls = []
    for si in range(len(synth.SWEEP_SHAPES)):
        c = synth.prefill_case(si, M)
        packed = bn.bitnet_pack_ternary(torch.from_numpy(c["t"]).to(dev))
        s_w = torch.from_numpy(c["s_w"]).to(dev)
        x = torch.from_numpy(c["x"].view(np.int16).copy()).to(dev).view(torch.bfloat16)
        y = torch.empty((M, c["N"]), dtype=torch.bfloat16, device=dev)
        ws = bn.make_workspace(M, c["K"], dev)
        calls.append({"x": x, "packed": packed, "s_w": s_w, "y": y, "N": c["N"], "K": c["K"],
                      "ws": ws})
    return calls


STACK_SPECS = {
    # name: (layers, hidden, ffn, token counts M, per_row scales)
    "2B-4T stack": (30, 2560, 6912, (1, 8, 32, 64), False),
    "8B-class stack": (32, 4096, 14336, (1, 16, 128, 4096), True),
}
BATCHED = ("q", "k", "v", "gate", "up")  # share the layer input x_h


def build_stack(bn, torch, dev, name):
    """Device weights of one stack. Layer 0 follows the recipe (2B-4T: ternary P(0)=0.4 drawn
    directly, per-tensor s_w ~ U(0.5, 2); 8B-class: latent W ~ N(0, 0.02^2) quantised per row by
    bitnet_pack_weights) and is copied into every other layer's own buffers, so each layer
    streams distinct memory; kernel time does not depend on the values, and parity of every
    projection shape is covered by the tests."""
    layers = STACK_SPECS[name][0]
    base = {}
    if name.startswith("2B"):
        for proj, d in synth.stack2b_layer(0).items():
            base[proj] = (bn.bitnet_pack_ternary(torch.from_numpy(d["t"]).to(dev)),
                          torch.from_numpy(d["s_w"]).to(dev), False)
    else:
        for proj in synth.SHAPES_8B:
            W = torch.from_numpy(synth.stack8b_latent(0, proj)).to(dev)
            packed, s_w = bn.bitnet_pack_weights(W, True)
            del W
            base[proj] = (packed, s_w, True)
    torch.cuda.synchronize()
    return [base] + [{k: (p.clone(), s_.clone(), r) for k, (p, s_, r) in base.items()}
                     for _ in range(layers - 1)]


def run_stack(bn, torch, dev, name, stack, M, steps, warmup, flush, world, peaks):
    """One pass = every layer back to back: bitnet_linear_batch(x_h -> q, k, v, gate, up),
    bitnet_linear(x_h -> o), bitnet_linear(x_f -> down), on fixed synthetic inputs."""
    layers, hidden, ffn, _, _ = STACK_SPECS[name]
    gen = synth.stack2b_x if name.startswith("2B") else synth.stack8b_x
    x_h = torch.from_numpy(gen(M, hidden, which=0).view(np.int16).copy()).to(dev).view(torch.bfloat16)
    x_f = torch.from_numpy(gen(M, ffn, which=1).view(np.int16).copy()).to(dev).view(torch.bfloat16)
    L0 = stack[0]
    ys = [torch.empty((M, L0[p][0].shape[0]), dtype=torch.bfloat16, device=dev) for p in BATCHED]
    y_o = torch.empty((M, hidden), dtype=torch.bfloat16, device=dev)
    y_d = torch.empty((M, hidden), dtype=torch.bfloat16, device=dev)
    tc = M > bn.GEMV_AUTO_M
    ws_h = bn.make_workspace(M, hidden, dev) if tc else None
    ws_f = bn.make_workspace(M, ffn, dev) if tc else None

    def one_pass():
        for L in stack:
            bn.bitnet_linear_batch(x_h, [L[p] for p in BATCHED], ys=ys, workspace=ws_h)
            bn.bitnet_linear(x_h, *L["o"], y=y_o, workspace=ws_h)
            bn.bitnet_linear(x_f, *L["down"], y=y_d, workspace=ws_f)

    g = capture(torch, one_pass)
    ms = timed_steps(torch, g.replay, steps, warmup, flush, world)
    assert bn.bitnet_check_device_errors() == 0
    ms_max, _ = reduce_over_ranks(ms, 0.0, world)
    t = ms_max * 1e-3 / steps
    shapes = [(L0[p][0].shape[0], L0[p][0].shape[1] * 4) for p in L0]
    w_bytes = layers * sum(N * K // 4 + 4 * (N if L0[p][2] else 1)
                           for p, (N, K) in zip(L0, shapes))
    act_bytes = layers * sum(2 * M * K + 2 * M * N for N, K in shapes)
    ops = layers * sum(2.0 * M * N * K for N, K in shapes)
    int8_peak = peaks["int8_tops"]
    roof = max((w_bytes + act_bytes) / (peaks["hbm_gbs"] * 1e9), ops / (int8_peak * 1e12))
    launches = layers * 3 * (2 if tc else 1)
    del g
    return {"stack": name, "M": M, "us_per_pass": t * 1e6, "tokens_per_s": M / t,
            "GB_per_s": (w_bytes + act_bytes) / t / 1e9, "TOPS": ops / t / 1e12,
            "roofline_us": roof * 1e6, "frac": roof / t,
            "bound": "hbm" if (w_bytes + act_bytes) / (peaks["hbm_gbs"] * 1e9) >= ops / (int8_peak * 1e12)
            else "tensor", "launches_per_pass": launches}, launches


MLP_SPECS = {
    # name: (layers, hidden, ffn, token counts M, per_row scales)
    "2B-4T MLP gate/up": (30, 2560, 6912, (1, 64, 2048), False),
    "8B-class MLP gate/up": (32, 4096, 14336, (1, 4096), True),
}


def build_mlp(bn, torch, dev, name):
    """Per layer: the gate and up projections packed separately (for the unfused arm) and
    interleaved (bitnet_interleave_gate_up, for the fused call). Layer 0 follows the stack
    recipe and is copied into every layer's own buffers, as in build_stack."""
    layers = MLP_SPECS[name][0]
    if name.startswith("2B"):
        d = synth.stack2b_layer(0)
        pg, sg, pu, su, per_row = (bn.bitnet_pack_ternary(torch.from_numpy(d["gate"]["t"]).to(dev)),
                                   torch.from_numpy(d["gate"]["s_w"]).to(dev),
                                   bn.bitnet_pack_ternary(torch.from_numpy(d["up"]["t"]).to(dev)),
                                   torch.from_numpy(d["up"]["s_w"]).to(dev), False)
    else:
        Wg = torch.from_numpy(synth.stack8b_latent(0, "gate")).to(dev)
        Wu = torch.from_numpy(synth.stack8b_latent(0, "up")).to(dev)
        (pg, sg), (pu, su), per_row = bn.bitnet_pack_weights(Wg, True), \
            bn.bitnet_pack_weights(Wu, True), True
        del Wg, Wu
    pgu, sgu = bn.bitnet_interleave_gate_up(pg, sg, pu, su, per_row)
    torch.cuda.synchronize()
    base = {"gate": (pg, sg, per_row), "up": (pu, su, per_row), "gu": (pgu, sgu, per_row)}
    return [base] + [{k: (a.clone(), b.clone(), r) for k, (a, b, r) in base.items()}
                     for _ in range(layers - 1)]


def run_mlp(bn, torch, dev, name, layers_w, M, steps, warmup, flush, world, peaks):
    """One pass = the gate/up + SwiGLU of every layer back to back, fused
    (bitnet_linear_swiglu) and unfused (bitnet_linear_batch of gate and up, then the
    elementwise silu(g) * u in PyTorch, for comparison). Returns the line object."""
    layers, hidden, ffn, _, per_row = MLP_SPECS[name]
    gen = synth.stack2b_x if name.startswith("2B") else synth.stack8b_x
    x = torch.from_numpy(gen(M, hidden, which=2).view(np.int16).copy()).to(dev).view(torch.bfloat16)
    h = torch.empty((M, ffn), dtype=torch.bfloat16, device=dev)
    g = torch.empty((M, ffn), dtype=torch.bfloat16, device=dev)
    u = torch.empty((M, ffn), dtype=torch.bfloat16, device=dev)
    tc = M > bn.GEMV_AUTO_M
    ws = bn.make_workspace(M, hidden, dev) if tc else None

    def fused():
        for L in layers_w:
            bn.bitnet_linear_swiglu(x, *L["gu"], h=h, workspace=ws)

    def unfused():
        for L in layers_w:
            bn.bitnet_linear_batch(x, [L["gate"], L["up"]], ys=[g, u], workspace=ws)
            torch.mul(torch.nn.functional.silu(g), u, out=h)

    res = {}
    for arm, fn in (("fused", fused), ("unfused", unfused)):
        gr = capture(torch, fn)
        ms = timed_steps(torch, gr.replay, steps, warmup, flush, world)
        ms_max, _ = reduce_over_ranks(ms, 0.0, world)
        res[arm] = ms_max * 1e-3 / steps
        del gr
    assert bn.bitnet_check_device_errors() == 0
    w_bytes = layers * (2 * ffn * hidden // 4 + 4 * (2 * ffn if per_row else 2))
    act_bytes = layers * (2 * M * hidden + 2 * M * ffn)
    ops = layers * 2.0 * M * (2 * ffn) * hidden
    int8_peak = peaks["int8_tops"]
    roof = max((w_bytes + act_bytes) / (peaks["hbm_gbs"] * 1e9), ops / (int8_peak * 1e12))
    t = res["fused"]
    launches = layers * (2 if tc else 1)
    return {"mlp": name, "M": M, "us_per_layer": t / layers * 1e6,
            "unfused_us_per_layer": res["unfused"] / layers * 1e6,
            "speedup_vs_unfused": res["unfused"] / t, "GB_per_s": (w_bytes + act_bytes) / t / 1e9,
            "TOPS": ops / t / 1e12, "roofline_us_per_layer": roof / layers * 1e6, "frac": roof / t,
            "bound": "hbm" if (w_bytes + act_bytes) / (peaks["hbm_gbs"] * 1e9) >= ops / (int8_peak * 1e12)
            else "tensor"}, launches * steps + layers * (2 if tc else 1) * steps


def run_calls(bn, calls):
    for c in calls:
        bn.bitnet_linear(c["x"], c["packed"], c["s_w"], False, y=c["y"], workspace=c.get("ws"))


def capture(torch, fn):
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # warm the launch path outside capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


_CLOCKS = None  # the run's ClockSampler; timed regions switch its sampling on


def timed_steps(torch, step_fn, steps, warmup, flush_buf, world):
    import torch.distributed as dist
    for _ in range(warmup):
        flush_buf.add_(1)
        step_fn()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    if _CLOCKS is not None:
        _CLOCKS.active.set()
    for a, b in ev:
        flush_buf.add_(1)  # evict L2 (outside the step's events)
        a.record()
        step_fn()
        b.record()
    torch.cuda.synchronize()
    if _CLOCKS is not None:
        _CLOCKS.active.clear()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in ev)


# ---------------------------------------------------------------------------- CPU oracle
def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _oracle_sweep_cases():
    import oracle
    oracle.build()
    cases = []
    for si in range(len(synth.SWEEP_SHAPES)):
        c = synth.decode_case(si, replica=0, M=DECODE_M)
        cases.append((c, oracle.pack(c["t"])))
    sweep_bytes = sum(decode_bytes(DECODE_M, c["N"], c["K"]) for c, _ in cases)

    def sweep():
        for c, packed in cases:
            oracle.bitlinear(c["x"], packed, c["s_w"], False, c["K"])

    return sweep, sweep_bytes


def _threaded_sweeps(sweep, threads: int, rounds: int):
    """`rounds` rounds of `threads` concurrent whole sweeps (the oracle's C calls release
    the GIL, so the threads run on separate cores); returns the elapsed seconds."""
    from concurrent.futures import ThreadPoolExecutor
    t0 = time.perf_counter()
    with ThreadPoolExecutor(threads) as ex:
        for _ in range(rounds):
            list(ex.map(lambda _: sweep(), range(threads)))
    return time.perf_counter() - t0


def oracle_sample(seconds: float):
    """Times the oracle (as it stands) on whole decode sweeps at M = 1: one thread for about
    half of `seconds`, then every host core running independent sweeps for the other half."""
    sweep, sweep_bytes = _oracle_sweep_cases()
    done, t0 = 0, time.perf_counter()
    while True:
        sweep()
        done += 1
        el1 = time.perf_counter() - t0
        if el1 >= seconds / 2:
            break
    one = done * sweep_bytes / el1 / 1e9
    n = os.cpu_count() or 1
    per_round = el1 / done  # one sweep per thread per round, if the cores scale
    rounds = max(1, int(seconds / 2 / per_round))
    el = _threaded_sweeps(sweep, n, rounds)
    return {"value": n * rounds * sweep_bytes / el / 1e9, "unit": "GB/s", "cores": n,
            "kind": "oracle",
            "sample": f"{n * rounds} full decode sweeps (4 shapes, M=1) on {n} threads, {el:.1f} s",
            "one_thread": {"value": one, "unit": "GB/s", "cores": 1,
                           "sample": f"{done} sweeps, {el1:.1f} s"},
            "cpu_model": cpu_model(), "nproc": n}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    sweep, sweep_bytes = _oracle_sweep_cases()
    n = os.cpu_count() or 1
    for _ in range(args.warmup):
        sweep()
    el = _threaded_sweeps(sweep, n, args.steps)  # one step = one sweep on every core
    value = args.steps * n * sweep_bytes / el / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "s8xternary->s32", "data": "synthetic",
        "config": {"workload": "decode GEMV sweep M=1, 2B-4T shapes (N,K) in "
                               "{(2560,2560),(640,2560),(6912,2560),(2560,6912)}; one sweep "
                               "(one weight replica) per host thread per step"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": n, "kind": "oracle",
                         "sample": f"{args.steps} steps of {n} concurrent sweeps of the 4 "
                                   "shapes at M=1", "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def measure_int8_peak(torch, dev, seconds: float = 1.5):
    """Dense int8 tensor-core rate of this GPU through torch._int_mm (cuBLASLt) on 8192^3:
    best of 10 single calls, and the rate of back-to-back calls for `seconds`."""
    n = 8192
    a = torch.randint(-128, 127, (n, n), dtype=torch.int8, device=dev)
    b = torch.randint(-128, 127, (n, n), dtype=torch.int8, device=dev).t()
    try:
        for _ in range(3):
            torch._int_mm(a, b)
    except RuntimeError as e:  # torch without an int8 GEMM
        return {"error": repr(e)[:200]}
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(10):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch._int_mm(a, b)
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    calls = max(1, int(seconds / (best * 1e-3)))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(calls):
        torch._int_mm(a, b)
    e1.record()
    torch.cuda.synchronize()
    ops = 2.0 * n ** 3
    return {"burst_tops": ops / (best * 1e-3) / 1e12,
            "sustained_tops": ops * calls / (e0.elapsed_time(e1) * 1e-3) / 1e12,
            "how": "torch._int_mm int8 8192^3 -> int32: best of 10, and back to back "
                   f"for {seconds} s"}


def measure_int_rates(bn, torch, dev):
    """Issue rates of the one-token GEMV's product instructions on this GPU (the library's
    probe kernels: dp4a only, legacy mma.sync m16n8k32 s8 only), 8 CTAs of 256 threads per
    SM, ~10 ms per launch, best of 3; int8 ops = 2 per multiply-add."""
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    blocks = sms * 8
    out = torch.empty(blocks, dtype=torch.int32, device=dev)
    st = torch.cuda.current_stream().cuda_stream
    res = {"how": f"bitnet_probe_int_rate, {blocks} CTAs x 256 threads, best of 3"}
    for name, kind, iters in (("dp4a", 0, 1 << 16), ("mma_sync_s8", 1, 1 << 15)):
        if bn.lib.bitnet_probe_int_rate(kind, blocks, 64, out.data_ptr(), st) != bn.OK:
            return {"error": f"probe {name} failed to launch"}
        best = float("inf")
        for _ in range(3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            bn.lib.bitnet_probe_int_rate(kind, blocks, iters, out.data_ptr(), st)
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1) * 1e-3)
        ops = bn.lib.bitnet_probe_int_ops(kind, blocks, iters)
        per_instr = 8 * 32 if kind == 0 else 2 * 16 * 8 * 32  # ops per warp instruction
        res[f"{name}_tops"] = ops / best / 1e12
        res[f"{name}_warp_instr_per_sm_per_ns"] = ops / per_instr / best / sms / 1e9
    assert bn.bitnet_check_device_errors() == 0
    return res


# ---------------------------------------------------------------------------- main arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    rank, world, local = dist_env()
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import ternary_w2a8_linear_token_b200 as bn

    peaks = load_peaks()
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    # The GEMM's denominator: the larger of the measured int8 rate (cuBLASLt through
    # torch._int_mm) and the nominal int8 : bf16 ratio times the measured bf16 peak.
    # the integer issue-rate probes first: the int8 GEMM probe leaves the GPU at its power cap
    int_rates = measure_int_rates(bn, torch, dev) if args.only == "all" else None
    int8_probe = measure_int8_peak(torch, dev) if args.only == "all" else {}
    nominal = peaks["bf16_tflops"] * INT8_PER_BF16
    measured = int8_probe.get("burst_tops", 0.0)
    peaks["int8_tops"] = max(measured, nominal)
    peaks["int8_src"] = ("measured torch._int_mm burst" if measured >= nominal else
                         f"{peaks['src']} bf16 burst x {INT8_PER_BF16} (nominal int8:bf16), above "
                         "the measured int8 rate")

    # ---------------- decode GEMV sweep
    per_replica = sum(N * K // 4 for N, K in synth.SWEEP_SHAPES)
    replicas = args.replicas or max(1, -(-2 * L2_BYTES // per_replica))
    calls = build_decode(bn, torch, replicas, dev)
    launches_per_step = len(calls)
    step_bytes = sum(decode_bytes(DECODE_M, c["N"], c["K"]) for c in calls)
    g_dec = capture(torch, lambda: run_calls(bn, calls))
    global _CLOCKS
    clk = ClockSampler(local).__enter__()  # samples inside every timed region below
    _CLOCKS = clk
    dec_ms = timed_steps(torch, g_dec.replay, args.steps, args.warmup, flush, world)
    assert bn.bitnet_check_device_errors() == 0
    dec_ms_max, total_bytes = reduce_over_ranks(dec_ms, step_bytes * args.steps, world)
    gbs = total_bytes / (dec_ms_max * 1e-3) / 1e9
    per_launch_bytes = step_bytes / launches_per_step
    avg_launch_s = dec_ms * 1e-3 / (args.steps * launches_per_step)
    achieved = per_launch_bytes / avg_launch_s / 1e9

    # ---------------- end to end: pinned host x -> device, forward, y -> pinned host
    h_x = torch.empty(sum(c["x"].numel() for c in calls), dtype=torch.bfloat16).pin_memory()
    h_y = torch.empty(sum(c["y"].numel() for c in calls), dtype=torch.bfloat16).pin_memory()
    d_x = torch.empty_like(h_x, device=dev)
    d_y = torch.empty_like(h_y, device=dev)
    off = 0
    e2e_calls = []
    for c in calls:
        n = c["x"].numel()
        xv = d_x[off:off + n].view(c["x"].shape)
        xv.copy_(c["x"])
        e2e_calls.append(dict(c, x=xv))
        off += n
    h_x.copy_(d_x)
    off = 0
    for c in e2e_calls:
        n = c["y"].numel()
        c["y"] = d_y[off:off + n].view(c["y"].shape)
        off += n
    g_e2e = capture(torch, lambda: run_calls(bn, e2e_calls))

    def e2e_step():
        d_x.copy_(h_x, non_blocking=True)
        g_e2e.replay()
        h_y.copy_(d_y, non_blocking=True)

    e2e_ms = timed_steps(torch, e2e_step, args.steps, args.warmup, flush, world)
    e2e_ms_max, _ = reduce_over_ranks(e2e_ms, 0.0, world)
    e2e_gbs = total_bytes / (e2e_ms_max * 1e-3) / 1e9

    # ---------------- prefill GEMM
    if args.only in ("decode", "mlp"):
        pcalls = []
    else:
        pcalls = build_prefill(bn, torch, dev, args.prefill_m)
    gemm = None
    g_pre = None
    if pcalls:
        g_pre = capture(torch, lambda: run_calls(bn, pcalls))
        pre_ms = timed_steps(torch, g_pre.replay, args.steps, args.warmup, flush, world)
        assert bn.bitnet_check_device_errors() == 0
        ops_step = sum(2.0 * args.prefill_m * c["N"] * c["K"] for c in pcalls)
        pre_ms_max, pre_ops = reduce_over_ranks(pre_ms, ops_step * args.steps, world)
        tops = pre_ops / (pre_ms_max * 1e-3) / 1e12
        int8_peak = peaks["int8_tops"]
        local_tops = ops_step * args.steps / (pre_ms * 1e-3) / 1e12
        gemm = {"value": tops, "unit": "TOPS", "ms_per_step": pre_ms_max / args.steps,
                "workload": f"prefill GEMM M={args.prefill_m} on the same 4 shapes, x = 0.5 t_4 "
                            "with 1% x20 outlier channels, ternary P(0)=0.5",
                "roofline": {"bound": "tensor", "achieved": local_tops, "peak": int8_peak,
                             "unit": "TOPS", "frac": local_tops / int8_peak,
                             "traffic": GEMM_PREFILL_TRAFFIC_BYTES
                             if args.prefill_m == PREFILL_M else None,
                             "traffic_src": "ncu dram__bytes_read.sum + dram__bytes_write.sum "
                                            "per tc_gemm_kernel launch at M=2048, one capture "
                                            "of the four shapes, mean",
                             "algorithmic_bytes_per_launch": sum(
                                 c["N"] * c["K"] // 4 + args.prefill_m * c["K"]
                                 + 2 * args.prefill_m * c["N"] for c in pcalls) / len(pcalls),
                             "peak_src": peaks["int8_src"],
                             "frac_vs_measured_int8": (local_tops / int8_probe["burst_tops"]
                                                       if int8_probe.get("burst_tops") else None),
                             "note": "per-call time includes the quantiser launch"}}
        # the same calls with one activation scale per tensor (partial maxima kernel added)
        def run_pt():
            for c in pcalls:
                bn.bitnet_linear_batch_act(c["x"], [(c["packed"], c["s_w"], False)],
                                           bn.ACT_PER_TENSOR, ys=[c["y"]], workspace=c["ws"])
        g_pt = capture(torch, run_pt)
        pt_ms = timed_steps(torch, g_pt.replay, args.steps, args.warmup, flush, world)
        assert bn.bitnet_check_device_errors() == 0
        pt_ms_max, pt_ops = reduce_over_ranks(pt_ms, ops_step * args.steps, world)
        gemm["act_per_tensor"] = {"value": pt_ops / (pt_ms_max * 1e-3) / 1e12, "unit": "TOPS",
                                  "ms_per_step": pt_ms_max / args.steps}
        del g_pt
        # the prefill configuration's other token count
        if args.prefill_m != PREFILL_M_SMALL:
            scalls = build_prefill(bn, torch, dev, PREFILL_M_SMALL)
            g_s = capture(torch, lambda: run_calls(bn, scalls))
            s_ms = timed_steps(torch, g_s.replay, args.steps, args.warmup, flush, world)
            assert bn.bitnet_check_device_errors() == 0
            s_ops_step = sum(2.0 * PREFILL_M_SMALL * c["N"] * c["K"] for c in scalls)
            s_ms_max, s_ops = reduce_over_ranks(s_ms, s_ops_step * args.steps, world)
            s_tops = s_ops / (s_ms_max * 1e-3) / 1e12
            gemm[f"m{PREFILL_M_SMALL}"] = {"value": s_tops, "unit": "TOPS",
                                           "ms_per_step": s_ms_max / args.steps,
                                           "frac": s_tops / int8_peak}
            del g_s, scalls

    # ---------------- layer stacks (2B-4T and 8B-class, every layer back to back)
    stacks = []
    stack_launches = 0
    if args.stacks == "all" and args.only == "all":
        for name, spec in STACK_SPECS.items():
            st = build_stack(bn, torch, dev, name)
            for M in spec[3]:
                r, nl = run_stack(bn, torch, dev, name, st, M, min(args.steps, 5), args.warmup,
                                  flush, world, peaks)
                stacks.append(r)
                stack_launches += nl * min(args.steps, 5)
            del st
            torch.cuda.empty_cache()

    # ---------------- fused MLP gate/up + SwiGLU against the unfused sequence
    mlp = []
    if args.stacks == "all" and args.only in ("all", "mlp"):
        mlp_m = [int(v) for v in args.mlp_m.split(",")] if args.mlp_m else None
        for name, spec in MLP_SPECS.items():
            ms = [M for M in spec[3] if mlp_m is None or M in mlp_m]
            if not ms:
                continue
            lw = build_mlp(bn, torch, dev, name)
            for M in ms:
                r, nl = run_mlp(bn, torch, dev, name, lw, M, min(args.steps, 5), args.warmup,
                                flush, world, peaks)
                mlp.append(r)
                stack_launches += nl
            del lw
            torch.cuda.empty_cache()

    clk.__exit__(None, None, None)
    _CLOCKS = None

    cpu = oracle_sample(args.cpu_seconds) if (rank == 0 and world == 1 and args.cpu_seconds > 0) \
        else None

    if rank == 0:
        line = {
            "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dec_ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "s8xternary->s32",
            "data": "synthetic",
            "config": {
                "workload": "decode GEMV sweep M=1, 2B-4T shapes (N,K) in {(2560,2560),"
                            "(640,2560),(6912,2560),(2560,6912)}, ternary P(0)=0.4, "
                            f"s_w~U(0.5,2), x~N(0,1); {replicas} weight replicas per step "
                            f"({per_replica * replicas / 1e6:.0f} MB packed) as one CUDA graph",
                "l2": "256 MB write before every step (outside the step's events); step "
                      "weights exceed 2x L2",
                "bytes_per_step": step_bytes, "launches_per_step": launches_per_step,
                "parallelism": f"replica x{world}",
            },
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                         "traffic": GEMV_DECODE_TRAFFIC_BYTES,
                         "traffic_src": "ncu dram__bytes_read.sum + dram__bytes_write.sum per "
                                        "launch, one capture of the four decode-sweep shapes, "
                                        "mean",
                         "algorithmic_bytes_per_launch": per_launch_bytes,
                         "peak_src": peaks["src"], "kernel": "gemv_w2a8_kernel"},
            "e2e": {"value": e2e_gbs, "unit": "GB/s",
                    "h2d_bytes_per_step": int(h_x.numel() * 2),
                    "d2h_bytes_per_step": int(h_y.numel() * 2)},
            "cpu_baseline": cpu,
            "gpu_launches": args.steps * launches_per_step * 2 + args.steps * 7 * len(pcalls)
                            + stack_launches,
            "clocks": clk.summary(),
            "gemm_tops": gemm["value"] if gemm else None,
            "gemm_frac": gemm["roofline"]["frac"] if gemm else None,
            "gemm_m512_tops": gemm[f"m{PREFILL_M_SMALL}"]["value"]
            if gemm and f"m{PREFILL_M_SMALL}" in gemm else None,
            "int8_peak": dict(int8_probe, used_tops=peaks["int8_tops"], used_src=peaks["int8_src"])
            if int8_probe else None,
            "int_rates": int_rates,
            "gemm": gemm,
            "stacks": stacks,
            "mlp": mlp,
        }
        print(json.dumps(line), flush=True)
    del g_dec, g_e2e, g_pre
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--only", choices=["all", "decode", "mlp"], default="all",
                    help="decode: skip everything after the decode sweep; mlp: decode sweep "
                         "and the MLP gate/up + SwiGLU part only (small profiling runs)")
    ap.add_argument("--mlp-m", default="",
                    help="comma-separated token counts of the MLP part (default: all listed)")
    ap.add_argument("--replicas", type=int, default=0,
                    help="weight replicas per decode step (0: enough to exceed 2x L2)")
    ap.add_argument("--prefill-m", type=int, default=PREFILL_M,
                    help="tokens of the prefill GEMM part")
    ap.add_argument("--stacks", choices=["all", "none"], default="all",
                    help="time the 2B-4T and 8B-class layer stacks and MLP gate/up + SwiGLU "
                         "(extra objects on the line)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
