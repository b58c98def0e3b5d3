"""Benchmark of the FP8 delayed-scaling linear hot path on B200.

One step = the whole hot path over one batch of the 1.2B-model linear
workload (hidden 1536, FFN 4096) at M = 8192 tokens, for both linear shapes
(W1 [1536,1536], W2 [4096,1536]):
  quantize X [M,1536] dual E4M3, W dual E4M3, G [M,N] dual E5M2 (rings
  carried across steps: delayed scaling), then
  fwd  Y  = Xq . Wq^T * sx*sw + b      (M x N x 1536)
  dX   = Gq . (W^T)q^T * sg*sw          (M x 1536 x N, A = E5M2)
  dW   = (G^T)q . (X^T)q^T * sg*sx      (N x 1536 x M, A = E5M2)
X, W and G of a linear go through fp8_quantize_multi and its dX and dW
through fp8_mm_pair (one launch each when the library fuses them), so a step
is 6 to 12 kernel launches, counted with fp8_launch_count while the step's
graph is captured.  The device-timed steps
replay a CUDA graph of the step; the end-to-end figure calls the C ABI
directly every step with host copies in and out.

Printed JSON line (rank 0): value = GEMM TFLOP/s of the whole step (GEMM
flops / step time, quantize time included), plus the GEMM-only TFLOP/s,
quantize GB/s, the roofline of the dominant kernel (the GEMM), clocks sampled
during the timed region, an end-to-end figure through the C ABI with host
buffers, and the CPU oracle baseline.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--M 8192]
Multi-GPU: one process per GPU under torch.distributed.run; the path has no
exchange step, so ranks run independent replicas (weak scaling) and only the
timing is reduced (max over ranks).
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

HIDDEN, FFN = 1536, 4096
METRIC = "mm_fp8 TFLOP/s & quantize GB/s on 1 B200, % of FP8/HBM roofline"
L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--M", type=int, default=8192)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-targets", action="store_true",
                    help="skip the 8192^3 GEMM and 12.6M-element quantize figures")
    ap.add_argument("--sweep", choices=["gemm", "quantize"], default=None,
                    help="per-shape kernel rows instead of the step line")
    ap.add_argument("--iters", type=int, default=50)
    ap.add_argument("--profile", action="store_true",
                    help="warm up, run exactly one step inside the NVTX range fp8_profile_step, exit (for ncu)")
    ap.add_argument("--shapes", default=None, help="sweep subset, e.g. 8192x8192x8192,64x8192x2048")
    ap.add_argument("--ws", action="store_true", help="gemm sweep: also time each shape with a stream-K workspace")
    ap.add_argument("--mm-out", default="bf16",
                    help="gemm sweep: output kinds to time, of bf16,e4m3,e5m2 (FP8 outputs fold an output ring)")
    ap.add_argument("--qdtypes", default="bf16,fp32", help="quantize sweep input dtypes")
    ap.add_argument("--qlayouts", default="row,T,dual", help="quantize sweep layouts")
    ap.add_argument("--qmisalign", action="store_true", help="quantize sweep: also time a base one element past 16 B")
    return ap.parse_args()


def workload_config(M, world):
    """The `config` both arms report for the 1.2B-model linear step."""
    return {"workload": f"1.2B-model linears fwd+bwd (hidden 1536, FFN 4096), M={M} tokens, "
                        "X/W/G dual quantize + fwd/dX/dW mm_fp8 for both linear shapes",
            "M": M, "linears": [[HIDDEN, HIDDEN], [FFN, HIDDEN]],
            "l2": "no flush: 2 rotating input sets, ~320 MB per set pair > 126 MB L2",
            "parallelism": f"replicas x{world}"}


def gemm_flops(M):
    return sum(3 * 2 * M * n * HIDDEN for n in (HIDDEN, FFN))


def quant_bytes(M):
    """Algorithmic bytes of the 6 dual quantizes of one step: n*2 (bf16 in) + n*2 (two fp8 outs) + ring."""
    tot = 0
    for n in (HIDDEN, FFN):
        for elems in (M * HIDDEN, n * HIDDEN, M * n):
            tot += elems * 4 + 96
    return tot


# ---------------------------------------------------------------- clocks ----

class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU, polled through NVML
    about every millisecond from a background thread (reads only; nothing is
    set).  A timed region of a few milliseconds therefore holds samples of its
    own.  Falls back to `nvidia-smi -lms 200` when NVML is not importable."""

    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index, period_s=0.001):
        self.device_index = device_index
        self.period = period_s
        self.samples = []  # (monotonic time, sm_mhz, sm_max_mhz, power_w, set of reason names)
        self._stop = threading.Event()
        self._t = None
        self._proc = None
        self.source = None

    def _nvml_handle(self):
        import pynvml

        pynvml.nvmlInit()
        try:
            import torch

            pr = torch.cuda.get_device_properties(self.device_index)
            bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:  # noqa: BLE001
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.device_index)

    def _poll_nvml(self, nv, h):
        bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
        mx = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        while not self._stop.is_set():
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((time.monotonic(), sm, mx, pw, {k for k, b in bits.items() if r & b}))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def _poll_smi(self):
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        self._proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-lms",
                                       "200", "-i", str(self.device_index)], stdout=subprocess.PIPE,
                                      stderr=subprocess.DEVNULL, text=True)
        for line in self._proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            try:
                sm, mx, pw = float(parts[0]), float(parts[1]), float(parts[2])
            except (ValueError, IndexError):
                continue
            rs = {n for n, v in zip(self.NAMES, parts[3:7]) if v.lower().startswith("active")}
            self.samples.append((time.monotonic(), sm, mx, pw, rs))

    def __enter__(self):
        try:
            nv, h = self._nvml_handle()
            self.source = "nvml, ~1 ms polling"
            self._t = threading.Thread(target=self._poll_nvml, args=(nv, h), daemon=True)
        except Exception:  # noqa: BLE001
            self.source = "nvidia-smi -lms 200"
            self._t = threading.Thread(target=self._poll_smi, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
        if self._t is not None:
            self._t.join(timeout=5)

    def summary(self, t0, t1):
        """Median SM clock and the clock-event reasons seen between t0 and t1.
        If no sample fell inside, the nearest sample on each side stands in
        (and `in_window` says so)."""
        inside = [x for x in self.samples if t0 <= x[0] <= t1]
        used = inside
        if not used:
            before = [x for x in self.samples if x[0] < t0][-1:]
            after = [x for x in self.samples if x[0] > t1][:1]
            used = before + after
        sm = [x[1] for x in used]
        reasons = sorted(set().union(*[x[4] for x in used])) if used else []
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": used[0][2] if used else None,
                "power_w_max": max(x[3] for x in used) if used else None,
                "reasons": reasons, "samples": len(used), "in_window": len(inside),
                "window_ms": round((t1 - t0) * 1e3, 2), "source": self.source}


# ----------------------------------------------------------- the workload ----

class Linear:
    """Device state of one FP8 linear: weights, bias, rings, output buffers, input sets."""

    def __init__(self, M, n_out, w, bias, inputs, torch, ops):
        self.M, self.N = M, n_out
        dev = "cuda"
        self.w = w.to(dev)
        self.bias = bias.to(dev)
        self.rx, self.rw, self.rg = ops.Ring(), ops.Ring(), ops.Ring()
        u8 = torch.uint8
        self.xq = torch.empty((M, HIDDEN), dtype=u8, device=dev)
        self.xq_t = torch.empty((HIDDEN, M), dtype=u8, device=dev)
        self.wq = torch.empty((n_out, HIDDEN), dtype=u8, device=dev)
        self.wq_t = torch.empty((HIDDEN, n_out), dtype=u8, device=dev)
        self.gq = torch.empty((M, n_out), dtype=u8, device=dev)
        self.gq_t = torch.empty((n_out, M), dtype=u8, device=dev)
        bf = torch.bfloat16
        self.y = torch.empty((M, n_out), dtype=bf, device=dev)
        self.dx = torch.empty((M, HIDDEN), dtype=bf, device=dev)
        self.dw = torch.empty((n_out, HIDDEN), dtype=bf, device=dev)
        self.inputs = [(x.to(dev), g.to(dev)) for x, g in inputs]
        self.ws = None  # stream-K workspace shared by the step's GEMMs (set by build_workload)

    def quantize(self, ops, x, g, ev=None):
        # X, W (E4M3) and G (E5M2) in one fp8_quantize_multi launch.
        ops.quantize_multi([dict(x=x, fmt=ops.E4M3, layout=ops.DUAL, ring=self.rx, out=self.xq, out_t=self.xq_t),
                            dict(x=self.w, fmt=ops.E4M3, layout=ops.DUAL, ring=self.rw, out=self.wq, out_t=self.wq_t),
                            dict(x=g, fmt=ops.E5M2, layout=ops.DUAL, ring=self.rg, out=self.gq, out_t=self.gq_t)])

    def quantize_paired(self, ops, x, g):
        # The previous schedule: X and W in one fp8_quantize_pair launch, G alone.
        ops.quantize_pair(dict(x=x, fmt=ops.E4M3, layout=ops.DUAL, ring=self.rx, out=self.xq, out_t=self.xq_t),
                          dict(x=self.w, fmt=ops.E4M3, layout=ops.DUAL, ring=self.rw, out=self.wq, out_t=self.wq_t))
        ops.quantize(g, ops.E5M2, ops.DUAL, self.rg, self.gq, self.gq_t)

    def gemms(self, ops):
        ops.mm(self.xq, self.wq, self.rx.scale_inv, self.rw.scale_inv, self.bias, out=self.y, workspace=self.ws)
        # dX and dW are independent: one fp8_mm_pair launch shares the GPU between them.
        ops.mm_pair(dict(a=self.gq, b=self.wq_t, sinv_a=self.rg.scale_inv, sinv_b=self.rw.scale_inv,
                         fmt_a=ops.E5M2, out=self.dx),
                    dict(a=self.gq_t, b=self.xq_t, sinv_a=self.rg.scale_inv, sinv_b=self.rx.scale_inv,
                         fmt_a=ops.E5M2, out=self.dw), workspace=self.ws)

    # The same step with the layout tag: row-layout quantizes only, and the
    # backward GEMMs read W, G and X as quantized through MN-major operands.
    def quantize_row(self, ops, x, g):
        ops.quantize_multi([dict(x=x, fmt=ops.E4M3, layout=ops.ROW, ring=self.rx, out=self.xq),
                            dict(x=self.w, fmt=ops.E4M3, layout=ops.ROW, ring=self.rw, out=self.wq),
                            dict(x=g, fmt=ops.E5M2, layout=ops.ROW, ring=self.rg, out=self.gq)])

    def gemms_mn(self, ops):
        ops.mm(self.xq, self.wq, self.rx.scale_inv, self.rw.scale_inv, self.bias, out=self.y, workspace=self.ws)
        ops.mm_pair(dict(a=self.gq, b=self.wq, sinv_a=self.rg.scale_inv, sinv_b=self.rw.scale_inv,
                         fmt_a=ops.E5M2, out=self.dx, b_mn_major=True),
                    dict(a=self.gq, b=self.xq, sinv_a=self.rg.scale_inv, sinv_b=self.rx.scale_inv,
                         fmt_a=ops.E5M2, out=self.dw, a_mn_major=True, b_mn_major=True), workspace=self.ws)


def build_workload(M, torch, ops, S, n_sets=2):
    (w1, b1), (w2, b2) = S.linear_1p2b_weights()
    lins = []
    for n_out, w, b in ((HIDDEN, w1, b1), (FFN, w2, b2)):
        sets = [S.linear_1p2b_step(M, n_out, s) for s in range(n_sets)]
        lins.append(Linear(M, n_out, w, b, sets, torch, ops))
    # One stream-K workspace, zeroed once, for every GEMM of the step (they run
    # one after another on one stream); sized for the largest request.
    need = 0
    for n in (HIDDEN, FFN):
        for (m, nn, k) in ((M, n, HIDDEN), (M, HIDDEN, n), (n, HIDDEN, M)):
            for amn, bmn in ((False, False), (False, True), (True, True)):
                need = max(need, ops.mm_workspace_bytes(m, nn, k, a_mn_major=amn, b_mn_major=bmn))
    ws = torch.zeros(max(need, 256), dtype=torch.uint8, device="cuda")
    for L in lins:
        L.ws = ws
    return lins


def run_step(lins, ops, i):
    for L in lins:
        x, g = L.inputs[i % len(L.inputs)]
        L.quantize(ops, x, g)
        L.gemms(ops)


def run_step_layout_tag(lins, ops, i):
    for L in lins:
        x, g = L.inputs[i % len(L.inputs)]
        L.quantize_row(ops, x, g)
        L.gemms_mn(ops)


def capture(torch, fn):
    """CUDA graph of fn() (the library allocates nothing and never syncs, so it captures)."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def time_graph(torch, g, reps):
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g.replay()
    e0.record(st)
    for _ in range(reps):
        g.replay()
    e1.record(st)
    e1.synchronize()
    return e0.elapsed_time(e1) / reps


def time_split(lins, ops, torch, reps):
    """Device time per step of the quantize phase and of the GEMM phase (graph replays)."""
    def quant():
        for i in range(2):
            for L in lins:
                x, g = L.inputs[i % len(L.inputs)]
                L.quantize(ops, x, g)

    def gemm():
        for _ in range(2):
            for L in lins:
                L.gemms(ops)

    gq, gm = capture(torch, quant), capture(torch, gemm)
    q_ms = time_graph(torch, gq, reps) / 2
    g_ms = time_graph(torch, gm, reps) / 2
    del gq, gm
    return q_ms, g_ms


# ------------------------------------------------------------- CPU oracle ----

def _oracle_sample_step(Ms, S, OR, OG, weights):
    """One pass of the oracle over a sample of the step: both linears at Ms
    tokens (6 dual quantizes + 3 GEMMs each).  Returns the sample's GEMM flops."""
    flops = 0
    for n_out, w, b in weights:
        x, g = S.linear_1p2b_step(Ms, n_out, 0)
        rx, rw, rg = OR.Ring(), OR.Ring(), OR.Ring()
        xq, xq_t, _ = OR.quantize(x, 0, OR.DUAL, rx)
        wq, wq_t, _ = OR.quantize(w, 0, OR.DUAL, rw)
        gq, gq_t, _ = OR.quantize(g, 1, OR.DUAL, rg)
        OG.mm_fp8(xq, wq, 0, 0, rx.scale_inv, rw.scale_inv, b.numpy())
        OG.mm_fp8(gq, wq_t, 1, 0, rg.scale_inv, rw.scale_inv)
        OG.mm_fp8(gq_t, xq_t, 1, 0, rg.scale_inv, rx.scale_inv)
        flops += 3 * 2 * Ms * n_out * HIDDEN
    return flops


def _oracle_threads():
    try:
        import threadpoolctl

        return max((p.get("num_threads", 1) for p in threadpoolctl.threadpool_info()), default=1)
    except Exception:  # noqa: BLE001
        return os.cpu_count()


def cpu_baseline(M_full, seconds=12.0):
    """The oracle as it stands, on a row sample of the same step, timed on host cores."""
    from fp8_delayed_scaling_02_b200 import synthetic as S
    from oracle import gemm as OG
    from oracle import recipe as OR

    Ms = 256
    (w1, b1), (w2, b2) = S.linear_1p2b_weights()
    weights = ((HIDDEN, w1, b1), (FFN, w2, b2))
    flops = 0
    t0 = time.perf_counter()
    reps = 0
    while True:
        flops += _oracle_sample_step(Ms, S, OR, OG, weights)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds or reps >= 50:
            break
    return {"value": flops / el / 1e12, "unit": "TFLOP/s", "cores": _oracle_threads(), "kind": "oracle",
            "sample": f"the same step (both linears: 6 quantizes + 3 GEMMs each) on {Ms} of {M_full} rows/tokens, "
                      f"{reps} repetitions in {el:.1f} s; numpy float64 oracle"}


def reference_arm(args, world):
    """The reference arm: the CPU oracle as it stands.  Each of the W warm-up
    and K timed steps is one bounded sample of the step (both linears at Ms of
    the M tokens); ms_per_step is the measured time of one such sample step."""
    from fp8_delayed_scaling_02_b200 import synthetic as S
    from oracle import gemm as OG
    from oracle import recipe as OR

    n = args.steps + args.warmup
    Ms = 256 if n <= 40 else (64 if n <= 200 else 16)
    (w1, b1), (w2, b2) = S.linear_1p2b_weights()
    weights = ((HIDDEN, w1, b1), (FFN, w2, b2))
    for _ in range(args.warmup):
        _oracle_sample_step(Ms, S, OR, OG, weights)
    flops = 0
    t0 = time.perf_counter()
    for _ in range(args.steps):
        flops += _oracle_sample_step(Ms, S, OR, OG, weights)
    el = time.perf_counter() - t0
    value = flops / el / 1e12
    ms = el * 1e3 / max(1, args.steps)
    sample = (f"each step: the same step (both linears: 6 dual quantizes + 3 GEMMs each) on {Ms} of {args.M} "
              f"rows/tokens; {args.steps} timed steps in {el:.1f} s; numpy float64 oracle")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(args.M, world),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": _oracle_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "ms_per_step": ms, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------ sweeps ----

GEMM_SHAPES = [(1, n, n, n) for n in (512, 1024, 1152, 2048, 3072, 4096, 8192)] + [
    (1, 64, 8192, 2048), (1, 1024, 1536, 2048), (1, 1000, 1537, 2048), (64, 512, 512, 512), (8, 1024, 2048, 2048)]
QUANT_SHAPES = [(128, 1536), (2048, 1536), (8192, 1536), (16384, 4096), (2048, 1537), (8192, 1537)]


def _kernel_ms(fn, torch, iters, flush=None):
    """Average device time of fn() from a CUDA graph of `iters` calls.  With
    `flush`, every call is preceded by a write of a buffer twice the L2 size
    and the time of a graph of the flushes alone is subtracted."""
    def body():
        for _ in range(iters):
            if flush is not None:
                flush.zero_()
            fn()
    t = time_graph(torch, capture(torch, body), 3)
    if flush is not None:
        def flush_only():
            for _ in range(iters):
                flush.zero_()
        t -= time_graph(torch, capture(torch, flush_only), 3)
    return t / iters


def pair_sweep(spec, args, torch, ops, S):
    """Time two 2-D GEMMs ("MxNxK[:lay]+MxNxK[:lay]") as one fp8_mm_pair call."""
    probs, fl = [], 0.0
    for i, part in enumerate(spec.split("+")):
        dims, _, lay = part.partition(":")
        M, N, K = (int(t) for t in dims.split("x"))
        a_mn, b_mn = lay == "mn", lay in ("mn", "bmn")
        a = S.fp8_codes((K, M) if a_mn else (M, K), seed=1 + 2 * i).cuda()
        b = S.fp8_codes((K, N) if b_mn else (N, K), seed=2 + 2 * i).cuda()
        one = torch.ones(1, device="cuda")
        out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        probs.append(dict(a=a, b=b, sinv_a=one, sinv_b=one, out=out, a_mn_major=a_mn, b_mn_major=b_mn))
        fl += 2.0 * M * N * K
    fn = lambda: ops.mm_pair(probs[0], probs[1])  # noqa: E731
    for _ in range(3):
        fn()
    ms = _kernel_ms(fn, torch, args.iters)
    print(json.dumps({"kernel": "mm_fp8_pair", "pair": spec, "us": round(ms * 1e3, 2),
                      "tflops": round(fl / ms / 1e9, 1)}))


def sweep(args):
    import torch

    from fp8_delayed_scaling_02_b200 import build as B
    from fp8_delayed_scaling_02_b200 import ops, synthetic as S

    B.build()
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    flush = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda")
    if args.sweep == "gemm":
        # A shape is [B x]M x N x K, optionally followed by ":bmn" (B read
        # MN-major) or ":mn" (A and B read MN-major), the backward layouts.
        # Two 2-D shapes joined by "+" are timed as one fp8_mm_pair call.
        shapes = []
        for spec in (args.shapes.split(",") if args.shapes else
                     ["x".join(map(str, s)) for s in GEMM_SHAPES]):
            if "+" in spec:
                pair_sweep(spec, args, torch, ops, S)
                continue
            dims, _, lay = spec.partition(":")
            v = tuple(int(t) for t in dims.split("x"))
            shapes.append(((1,) + v if len(v) == 3 else v, lay or "nt"))
        for (bt, M, N, K), lay in shapes:
            a_mn, b_mn = lay == "mn", lay in ("mn", "bmn")
            a = S.fp8_codes((bt, K, M) if a_mn else (bt, M, K), seed=1).cuda()
            nb = 1 if bt == 8 else bt
            b = S.fp8_codes((nb, K, N) if b_mn else (nb, N, K), seed=2).cuda()
            one = torch.ones(1, device="cuda")
            bias = S.uniform((N,), seed=3).cuda()
            out = torch.empty((bt, M, N), dtype=torch.bfloat16, device="cuda")
            need = ops.mm_workspace_bytes(M, N, K, batch=bt, a_mn_major=a_mn, b_mn_major=b_mn)
            ws = torch.zeros(max(need, 256), dtype=torch.uint8, device="cuda") if args.ws else None
            out8 = torch.empty((bt, M, N), dtype=torch.uint8, device="cuda")
            ring = ops.Ring()
            kinds = {"bf16": None, "e4m3": ops.E4M3, "e5m2": ops.E5M2}
            for use_ws in ((False, True) if args.ws and need > 0 else (False,)):
                for kind in args.mm_out.split(","):
                    for with_bias in (False, True):
                        bb = bias if with_bias else None
                        w = ws if use_ws else None
                        if kinds[kind] is None:
                            fn = lambda: ops.mm(a, b, one, one, bb, out=out,  # noqa: E731
                                                a_mn_major=a_mn, b_mn_major=b_mn, workspace=w)
                        else:
                            fn = lambda: ops.mm_ex(a, b, one, one, bias=bb, out_fmt=kinds[kind],  # noqa: E731
                                                   out_ring=ring, out=out8, a_mn_major=a_mn, b_mn_major=b_mn,
                                                   workspace=w)
                        for _ in range(3):
                            fn()
                        ms = _kernel_ms(fn, torch, args.iters)
                        fl = 2.0 * bt * M * N * K
                        print(json.dumps({"kernel": "mm_fp8", "batch": bt, "M": M, "N": N, "K": K, "layout": lay,
                                          "out": kind, "bias": with_bias, "stream_k_ws": need if use_ws else 0,
                                          "us": round(ms * 1e3, 2), "tflops": round(fl / ms / 1e9, 1)}))
    else:
        want = [tuple(int(v) for v in s.split("x")) for s in args.shapes.split(",")] if args.shapes else None
        for rows, cols in (QUANT_SHAPES if not want else want):
            for dt in args.qdtypes.split(","):
                x0 = S.quant_sweep_input(rows, cols, dt, 1.0).cuda()
                eb = x0.element_size()
                # The input at a 16-byte aligned base and one element past it.
                flat = torch.empty(rows * cols + 1, dtype=x0.dtype, device="cuda")
                flat[1:].copy_(x0.reshape(-1))
                for base, x in (("aligned", x0), ("+1 element", flat[1:].view(rows, cols))):
                    if base != "aligned" and not args.qmisalign:
                        continue
                    for layout, name in ((ops.ROW, "row"), (ops.TRANSPOSED, "T"), (ops.DUAL, "dual")):
                        if name not in args.qlayouts.split(","):
                            continue
                        ring = ops.Ring()
                        out = torch.empty((rows, cols), dtype=torch.uint8, device="cuda")
                        out_t = torch.empty((cols, rows), dtype=torch.uint8, device="cuda")
                        fn = lambda: ops.quantize(x, ops.E4M3, layout, ring, out, out_t)  # noqa: E731
                        for _ in range(3):
                            fn()
                        ms = _kernel_ms(fn, torch, args.iters, flush)
                        nbytes = rows * cols * (eb + (2 if layout == ops.DUAL else 1)) + 96
                        print(json.dumps({"kernel": "quantize", "dtype": dt, "layout": name, "rows": rows,
                                          "cols": cols, "base": base, "us": round(ms * 1e3, 2),
                                          "gbs": round(nbytes / ms / 1e6, 1),
                                          "frac": round(nbytes / ms / 1e6 / hbm_peak_gbs(), 3)}))
    return 0


def hbm_peak_gbs():
    """The measured HBM copy bandwidth (GB/s) of this machine, else the fallback figure."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f).get("hbm_gbs", 6650.0))
    except (OSError, ValueError):
        return 6650.0


def _time_rotating(torch, fns, reps):
    """Average device time of one call when ``reps`` calls cycle through ``fns``
    (one per buffer set) back to back inside a CUDA graph, events on the
    replay stream.  With enough sets, each call's inputs were evicted from L2
    by the calls in between."""
    def body():
        for i in range(reps):
            fns[i % len(fns)]()
    g = capture(torch, body)
    ms = time_graph(torch, g, 3) / reps
    del g
    return ms


def measure_targets(torch, ops, S, peaks, fp8_peak_burst, hbm_peak, flush):
    """The two figures the target is stated on, each on its own shape:
    the 8192^3 E4M3 GEMM (TFLOP/s, fraction of the burst FP8 peak) and the
    12.6M-element quantize (8192x1536 and its odd-width neighbour 8192x1537,
    bf16 input, E4M3, row / T / dual; GB/s and fraction of measured HBM),
    the latter timed two ways: (a) every call preceded by an L2 flush (a write
    of 2x the L2 size) with a graph of the flushes alone subtracted; (b) calls
    back to back over rotating buffer sets whose total exceeds 2x the L2 size."""
    out = {}
    n = 8192
    one = torch.ones(1, device="cuda")
    sets = [(S.fp8_codes((n, n), seed=1 + 2 * i).cuda(), S.fp8_codes((n, n), seed=2 + 2 * i).cuda()) for i in range(2)]
    y = torch.empty((n, n), dtype=torch.bfloat16, device="cuda")
    fns = [lambda a=a, b=b: ops.mm(a, b, one, one, None, out=y) for a, b in sets]
    for f in fns:
        f()
    ms = _time_rotating(torch, fns, 20)
    tf = 2.0 * n ** 3 / (ms * 1e-3) / 1e12
    out["mm_8192_cubed"] = {"us": round(ms * 1e3, 1), "tflops": round(tf, 1), "peak": round(fp8_peak_burst, 1),
                            "frac": round(tf / fp8_peak_burst, 4), "target_frac": 0.60,
                            "peak_source": "of measured (bf16 burst x 2)",
                            "l2": "two rotating operand sets (268 MB > L2)", "timing": "20 calls in a CUDA graph"}
    del sets, fns, y
    q = {"target_frac": 0.70, "peak": hbm_peak, "peak_source": "of measured hbm_gbs", "dtype": "bf16", "fmt": "E4M3",
         "flushed": {}, "rotating": {}}
    for rows, cols in ((8192, 1536), (8192, 1537)):
        el = rows * cols
        for layout, name in ((ops.ROW, "row"), (ops.TRANSPOSED, "T"), (ops.DUAL, "dual")):
            nout = 2 if layout == ops.DUAL else 1
            nbytes = el * (2 + nout) + 96
            nsets = max(2, -(-4 * L2_BYTES // (el * (2 + nout))))
            bufs = []
            for i in range(nsets):
                x = S.quant_sweep_input(rows, cols, "bf16", 1.0, seed=50 + i).cuda()
                o = torch.empty((rows, cols), dtype=torch.uint8, device="cuda") if layout != ops.TRANSPOSED else None
                ot = torch.empty((cols, rows), dtype=torch.uint8, device="cuda") if layout != ops.ROW else None
                bufs.append((x, o, ot, ops.Ring()))
            fns = [lambda b=b, lay=layout: ops.quantize(b[0], ops.E4M3, lay, b[3], b[1], b[2]) for b in bufs]
            for f in fns:
                f()
            key = f"{rows}x{cols}"
            ms_f = _kernel_ms(fns[0], torch, 20, flush)
            ms_r = _time_rotating(torch, fns, 6 * nsets)
            for tag, t in (("flushed", ms_f), ("rotating", ms_r)):
                gbs = nbytes / (t * 1e-3) / 1e9
                q[tag].setdefault(key, {})[name] = {"us": round(t * 1e3, 2), "gbs": round(gbs, 1),
                                                    "frac": round(gbs / hbm_peak, 4)}
            del bufs, fns
    q["flushed"]["how"] = "graph of 20 x (L2 flush + call) minus a graph of the 20 flushes"
    q["rotating"]["how"] = "graph of back-to-back calls over rotating buffer sets totalling > 4x L2 (no flush)"
    out["quantize_12p6M"] = q
    return out


def measured_traffic():
    """DRAM bytes per step of the 6 GEMM launches from the committed ncu summary,
    or None if the GEMM source changed since that capture."""
    import hashlib

    path = os.path.join(ROOT, "profiles", "traffic_linear_1p2b_M8192.txt")
    src = os.path.join(ROOT, "fp8_delayed_scaling_02_b200", "csrc", "mm_fp8.cu")
    try:
        kv = {}
        for line in open(path):
            line = line.split("#", 1)[0].strip()
            if "=" in line:
                k, v = line.split("=", 1)
                kv[k.strip()] = v.strip()
        sha = hashlib.sha1(open(src, "rb").read()).hexdigest()
        if kv.get("mm_fp8_cu_sha1") != sha:
            return None
        return int(kv["mm_fp8_dram_bytes_per_step"])
    except (OSError, KeyError, ValueError):
        return None


# -------------------------------------------------------------------- main ----

def main():
    args = parse()
    if args.sweep:
        return sweep(args)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(reference_arm(args, world)))
        return 0

    import torch

    from fp8_delayed_scaling_02_b200 import build as B
    from fp8_delayed_scaling_02_b200 import ops, synthetic as S

    B.build()
    torch.cuda.set_device(local)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        pg = dist

    M = args.M
    lins = build_workload(M, torch, ops, S)
    # Clocks are polled from before the warm-up until every timed region is done.
    clk = ClockSampler(local).__enter__()
    for i in range(max(3, args.warmup)):
        run_step(lins, ops, i)
    torch.cuda.synchronize()
    if args.profile:
        torch.cuda.nvtx.range_push("fp8_profile_step")
        n0 = ops.launch_count()
        run_step(lins, ops, 0)
        n1 = ops.launch_count()
        torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize()
        print(json.dumps({"profile_step": "done", "M": M, "launches": n1 - n0}))
        return 0
    q_ms, g_ms = time_split(lins, ops, torch, 50)

    # The timed steps replay a CUDA graph of two consecutive steps (one per
    # input set), so the host launch cost is off the measured device time.
    steps = args.steps + (args.steps % 2)
    n0 = ops.launch_count()
    graph = capture(torch, lambda: (run_step(lins, ops, 0), run_step(lins, ops, 1)))
    launches_per_step = (ops.launch_count() - n0) // 2
    graph.replay()
    st = torch.cuda.current_stream()
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_clk0 = time.monotonic()
    e0.record(st)
    for i in range(steps // 2):
        graph.replay()
    e1.record(st)
    torch.cuda.synchronize()
    t_clk1 = time.monotonic()
    ms = e0.elapsed_time(e1) / steps
    del graph

    # Layout-tag variant of the same step (reported beside the main line).
    for i in range(3):
        run_step_layout_tag(lins, ops, i)
    graph_lt = capture(torch, lambda: (run_step_layout_tag(lins, ops, 0), run_step_layout_tag(lins, ops, 1)))
    ms_lt = time_graph(torch, graph_lt, max(50, steps // 10)) / 2
    del graph_lt
    if pg:
        t = torch.tensor([ms_lt], device="cuda")
        pg.all_reduce(t, op=pg.ReduceOp.MAX)
        ms_lt = float(t.item())
    if pg:
        t = torch.tensor([ms], device="cuda")
        pg.all_reduce(t, op=pg.ReduceOp.MAX)
        ms = float(t.item())
        pg.barrier()
    flops = gemm_flops(M)
    value = world * flops / (ms * 1e-3) / 1e12

    # End to end through the C ABI: every step copies its X and G in from pinned
    # host memory and its Y, dX and dW out to pinned host memory.  As a
    # training loop would, it overlaps step i's compute with the copy-in of
    # step i+1 and the copy-out of step i-1 (three streams; inputs, outputs
    # and host outputs double-buffered; events order every reuse).
    e2e = None
    if not args.no_e2e:
        host_in = [[(x.cpu().pin_memory(), g.cpu().pin_memory()) for x, g in L.inputs] for L in lins]
        outs = [[(L.y, L.dx, L.dw), (torch.empty_like(L.y), torch.empty_like(L.dx), torch.empty_like(L.dw))]
                for L in lins]
        host_out = [[tuple(torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in o) for o in lo] for lo in outs]
        h2d = sum(x.numel() * x.element_size() + g.numel() * g.element_size() for x, g in (h[0] for h in host_in))
        d2h = sum(sum(t.numel() * t.element_size() for t in lo[0]) for lo in outs)
        # The same K steps as the device-timed value (at most 200), after W
        # untimed pipelined steps; the timed region still holds the pipeline's
        # fill (the first step's copy-in) and drain (the last copy-out).
        steps_e2e = max(3, min(200, args.steps))
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()  # noqa: E731
        in_ready = [ev(), ev()]      # inputs of buffer set b copied in
        in_free = [ev(), ev()]       # compute done reading buffer set b
        out_ready = [ev(), ev()]     # outputs of buffer set b computed
        out_free = [ev(), ev()]      # outputs of buffer set b copied out
        for e in in_free + out_free:
            e.record(st)
        if pg:
            pg.barrier()
        torch.cuda.synchronize()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def copy_in(i):
            b = i % 2
            with torch.cuda.stream(s_in):
                s_in.wait_event(in_free[b])
                for L, hin in zip(lins, host_in):
                    hx, hg = hin[i % len(hin)]
                    x, g = L.inputs[b]
                    x.copy_(hx, non_blocking=True)
                    g.copy_(hg, non_blocking=True)
                in_ready[b].record(s_in)

        def pipelined(nsteps):
            copy_in(0)
            for i in range(nsteps):
                b = i % 2
                if i + 1 < nsteps:
                    copy_in(i + 1)
                st.wait_event(in_ready[b])
                st.wait_event(out_free[b])
                for L, lo in zip(lins, outs):
                    x, g = L.inputs[b]
                    L.y, L.dx, L.dw = lo[b]
                    L.quantize(ops, x, g)
                    L.gemms(ops)
                in_free[b].record(st)
                out_ready[b].record(st)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(out_ready[b])
                    for lo, ho in zip(outs, host_out):
                        for t, h in zip(lo[b], ho[b]):
                            h.copy_(t, non_blocking=True)
                    out_free[b].record(s_out)
            st.wait_stream(s_out)

        pipelined(max(3, args.warmup))
        torch.cuda.synchronize()
        if pg:
            pg.barrier()
        torch.cuda.synchronize()
        a0.record(st)
        s_in.wait_stream(st)  # every timed copy starts after a0
        s_out.wait_stream(st)
        pipelined(steps_e2e)
        a1.record(st)
        torch.cuda.synchronize()
        for L, lo in zip(lins, outs):
            L.y, L.dx, L.dw = lo[0]
        ms_e2e = a0.elapsed_time(a1) / steps_e2e
        if pg:
            t = torch.tensor([ms_e2e], device="cuda")
            pg.all_reduce(t, op=pg.ReduceOp.MAX)
            ms_e2e = float(t.item())
        e2e = {"value": world * flops / (ms_e2e * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms_e2e,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "overlap": "copy-in of step i+1 and copy-out of step i-1 run beside step i's kernels"}

    peaks = {}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
    except (OSError, ValueError):
        pass
    # Every timed region here lasts milliseconds, far from the seconds-long
    # loop of the sustained figure: the burst peak is the denominator.
    if "bf16_tflops" in peaks:
        fp8_peak, peak_src = 2.0 * peaks["bf16_tflops"], "of measured (bf16 burst x 2)"
    else:
        fp8_peak, peak_src = 2.0 * 1590.0, "of fallback (1.59 PF/s bf16 burst x 2)"
    hbm_peak = peaks.get("hbm_gbs", 6650.0)
    targets, t_tg = {}, None
    if not args.no_targets:
        flush = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda")
        t_a = time.monotonic()
        targets = measure_targets(torch, ops, S, peaks, fp8_peak, hbm_peak, flush)
        t_tg = (t_a, time.monotonic())
        del flush
    clk.__exit__(None, None, None)
    traffic = measured_traffic()
    gemm_tf = flops / (g_ms * 1e-3) / 1e12
    qb = quant_bytes(M)
    quant_gbs = qb / (q_ms * 1e-3) / 1e9

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
            "steps": steps, "warmup": max(3, args.warmup), "ms_per_step": round(ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp8e4m3/e5m2->f32acc->bf16",
            "data": "synthetic",
            "config": dict(workload_config(M, world), stream_k_workspace_bytes=int(lins[0].ws.numel())),
            "mm_tflops": round(gemm_tf, 2), "quantize_gbs": round(quant_gbs, 1),
            "quantize_ms_per_step": round(q_ms, 4), "mm_ms_per_step": round(g_ms, 4),
            "layout_tag_step": {"ms_per_step": round(ms_lt, 4),
                                "value": round(world * flops / (ms_lt * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                                "what": "same step with row-only quantizes and MN-major operands for dX/dW"},
            "roofline": {"bound": "tensor", "achieved": round(gemm_tf, 2), "peak": round(fp8_peak, 1),
                         "unit": "TFLOP/s", "frac": round(gemm_tf / fp8_peak, 4),
                         "traffic": traffic if M == 8192 else None,
                         "kernel": "mm_fp8 (all GEMM launches of the step: fwd, and dX + dW through fp8_mm_pair)", "peak_source": peak_src},
            "quantize_roofline": {"bound": "hbm", "achieved": round(quant_gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                                  "frac": round(quant_gbs / hbm_peak, 4), "peak_source": "of measured hbm_gbs"},
            "clocks": clk.summary(t_clk0, t_clk1),
            **targets,
            "targets_clocks": clk.summary(*t_tg) if t_tg else None,
            "gpu_launches": launches_per_step * steps,
            "timing": f"device events around CUDA-graph replays of the step ({launches_per_step} kernels per step)",
            "e2e": e2e,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(M)
        print(json.dumps(line))
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
