"""Benchmark of the integer-only (C,e) training hot path on B200.

One step = one training step of a ViT-Ti-shaped MLP block through libict.so:
fc1 forward (12608x192 . 192x768), integer GELU, fc2 forward (12608x768 . 768x192),
fc2 backward-data and backward-weight, GELU backward, fc1 backward-data and
backward-weight, and the integer SGD-with-momentum update of both weight matrices
(per-row velocity groups).  Synthetic seeded inputs of the paper's ViT-Ti shapes
(64 images x 197 tokens; "Memory-Efficient Integer-Only Training of Deep Neural
Networks", Abstract and Table 9).

metric: (C,e) GEMM TOPS over the whole step (6 contractions = 22.31 GOP per step),
plus the int-SGD update GB/s (ResNet-50 parameter arena) and the large-shape GEMM TOPS
(ViT-B linear trio) as side measurements.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 run under torchrun: every rank runs the same single-GPU step on its own
batch (independent replicas, no data-path collective); the reported time is the max
over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from integer_only_nn_02_b200 import workloads as wl  # noqa: E402

TOKENS, D, HID, GROUP = 64 * 197, 192, 768, 32
STEP_OPS = 6 * 2 * TOKENS * D * HID  # six contractions per step
L2_FLUSH_BYTES = 512 << 20          # larger than the 126 MB L2


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-side", action="store_true", help="skip the side measurements")
    return ap.parse_args()


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        return dict(hbm=m["hbm_gbs"], bf16=m["bf16_tflops"], bf16_sust=m["bf16_tflops_sustained"],
                    source="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, source="fallback")


# --------------------------------------------------------------------- clocks


class ClockSampler:
    """SM clock and throttle reasons of one GPU, polled through NVML every ~2 ms from a
    thread while the timed region runs."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_index: int):
        self.samples, self.reason_bits, self.max_mhz = [], 0, None
        self.stop_flag = False
        self.thread = None
        self.handle = None
        try:
            import pynvml
            import torch

            pynvml.nvmlInit()
            self.nv = pynvml
            h = None
            try:
                uuid = str(torch.cuda.get_device_properties(torch_index).uuid)
                uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
                h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            except Exception:
                h = pynvml.nvmlDeviceGetHandleByIndex(torch_index)
            self.handle = h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception as exc:  # pragma: no cover
            self.error = str(exc)

    def _reasons(self):
        nv = self.nv
        f = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        return int(f(self.handle))

    def _loop(self):
        import time as _t

        while not self.stop_flag:
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.handle, self.nv.NVML_CLOCK_SM))
                self.reason_bits |= self._reasons()
            except Exception:
                pass
            _t.sleep(0.002)

    def start(self):
        import threading

        if self.handle is None:
            return
        self.thread = threading.Thread(target=self._loop, daemon=True)
        self.thread.start()

    def stop(self):
        if self.thread is None:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"], "samples": 0}
        self.stop_flag = True
        self.thread.join(timeout=5)
        reasons = sorted(n for bit, n in self.REASONS.items() if self.reason_bits & bit)
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples)}


# --------------------------------------------------------------------- the step


class MlpStep:
    """Device state of one ViT-Ti MLP block training step (all buffers preallocated)."""

    def __init__(self, ict, seed: int):
        import torch

        self.ict, self.torch = ict, torch
        cfg = wl.vit_ti_mlp(seed=seed)
        self.cfg = cfg
        E = ict.DevCE
        self.X, self.W1, self.W2, self.dY2 = (E.from_host(cfg[k]) for k in ("X", "W1", "W2", "dY2"))
        self.V1, self.V2 = E.from_host(cfg["V1"]), E.from_host(cfg["V2"])
        M = TOKENS
        self.H = E.empty(M, HID, 1, GROUP)
        self.G = E.empty(M, HID, 1, GROUP)
        self.Y = E.empty(M, D, 1, GROUP)
        self.dG = E.empty(M, HID, 1, GROUP)
        self.dH = E.empty(M, HID, 1, GROUP)
        self.dX = E.empty(M, D, 1, GROUP)
        self.dW2 = E.empty(D, HID, 1, HID)
        self.dW1 = E.empty(HID, D, 1, D)
        ws = ict.ict_linear_workspace
        need = max(ws(0, self.X, self.W1, self.H), ws(0, self.G, self.W2, self.Y),
                   ws(1, self.dY2, self.W2, self.dG), ws(2, self.dY2, self.G, self.dW2),
                   ws(1, self.dH, self.W1, self.dX), ws(2, self.dH, self.X, self.dW1))
        self.ws = torch.empty(max(need, 256), dtype=torch.uint8, device="cuda")
        self.mom, self.lr = cfg["sgd"]["mom"], cfg["sgd"]["lr"]
        self.calls = [
            ("fc1_fwd", lambda: ict.ict_linear_fwd(self.X, self.W1, self.H, self.ws)),
            ("gelu_fwd", lambda: ict.ict_gelu_fwd(self.H, self.G)),
            ("fc2_fwd", lambda: ict.ict_linear_fwd(self.G, self.W2, self.Y, self.ws)),
            ("fc2_bwd_data", lambda: ict.ict_linear_bwd_data(self.dY2, self.W2, self.dG, self.ws)),
            ("fc2_bwd_weight", lambda: ict.ict_linear_bwd_weight(self.dY2, self.G, self.dW2, self.ws)),
            ("gelu_bwd", lambda: ict.ict_gelu_bwd(self.H, self.dG, self.dH)),
            ("fc1_bwd_data", lambda: ict.ict_linear_bwd_data(self.dH, self.W1, self.dX, self.ws)),
            ("fc1_bwd_weight", lambda: ict.ict_linear_bwd_weight(self.dH, self.X, self.dW1, self.ws)),
            ("sgd_w1", lambda: ict.ict_sgd_momentum_step(self.W1, self.V1, self.dW1, self.mom, self.lr)),
            ("sgd_w2", lambda: ict.ict_sgd_momentum_step(self.W2, self.V2, self.dW2, self.mom, self.lr)),
        ]

    def run(self, events=None):
        for i, (_, fn) in enumerate(self.calls):
            if events is not None:
                events[i][0].record()
            fn()
            if events is not None:
                events[i][1].record()


def time_steps(step, K, W, flush):
    """Per-step device time (ms) with an L2 flush between steps; per-call breakdown."""
    torch = step.torch
    for _ in range(W):
        step.run()
    torch.cuda.synchronize()
    n = len(step.calls)
    per_call = np.zeros(n)
    totals = []
    for _ in range(K):
        flush.fill_(1)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        step.run(ev)
        torch.cuda.synchronize()
        ms = [a.elapsed_time(b) for a, b in ev]
        per_call += ms
        totals.append(ev[0][0].elapsed_time(ev[-1][1]))
    return float(np.mean(totals)), per_call / K


def time_e2e(step, K, W):
    """Same step through the public API with host buffers: pinned H2D of the batch
    (X, dY2 mantissas and exponents), the step, D2H of the updated weights."""
    torch, ict = step.torch, step.ict
    host_in = []
    for t in (step.X, step.dY2):
        host_in.append((t.mant.cpu().pin_memory(), t.mant))
        host_in.append((t.exp.cpu().pin_memory(), t.exp))
    host_out = []
    for t in (step.W1, step.W2):
        host_out.append((torch.empty_like(t.mant, device="cpu").pin_memory(), t.mant))
        host_out.append((torch.empty_like(t.exp, device="cpu").pin_memory(), t.exp))
    h2d = sum(h.numel() for h, _ in host_in)
    d2h = sum(h.numel() for h, _ in host_out)

    def one():
        for h, d in host_in:
            d.copy_(h, non_blocking=True)
        step.run()
        for h, d in host_out:
            h.copy_(d, non_blocking=True)

    for _ in range(W):
        one()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(K):
        one()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / K, h2d, d2h


# --------------------------------------------------------------------- side measurements


def side_measurements(ict, torch, peaks):
    out = {}
    E = ict.DevCE

    def ev_time(fn, n=10, warm=3, flush=None):
        for _ in range(warm):
            fn()
        ts = []
        for _ in range(n):
            if flush is not None:
                flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return float(np.median(ts))

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    # ViT-B linear trio: six contractions of 59.49 GOP
    c4 = wl.vit_b_linear_trio(seed=0)
    X, W1, W2, dY1, dY2 = (E.from_host(c4[k]) for k in ("X", "W1", "W2", "dY1", "dY2"))
    M = X.rows
    H1 = E.empty(M, 3072, 1, 64)
    Y2 = E.empty(M, 768, 1, 64)
    dXa = E.empty(M, 768, 1, 64)
    dHa = E.empty(M, 3072, 1, 64)
    dW1 = E.empty(3072, 768, 1, 768)
    dW2 = E.empty(768, 3072, 1, 3072)
    wsz = max(ict.ict_linear_workspace(0, X, W1, H1), ict.ict_linear_workspace(0, H1, W2, Y2),
              ict.ict_linear_workspace(1, dY2, W2, dHa), ict.ict_linear_workspace(1, dY1, W1, dXa),
              ict.ict_linear_workspace(2, dY1, X, dW1), ict.ict_linear_workspace(2, dY2, H1, dW2))
    ws = torch.empty(max(wsz, 256), dtype=torch.uint8, device="cuda")
    gop = 2 * M * 768 * 3072 / 1e9
    trio = {
        "fc1_fwd": lambda: ict.ict_linear_fwd(X, W1, H1, ws),
        "fc2_fwd": lambda: ict.ict_linear_fwd(H1, W2, Y2, ws),
        "fc2_bwd_data": lambda: ict.ict_linear_bwd_data(dY2, W2, dHa, ws),
        "fc1_bwd_data": lambda: ict.ict_linear_bwd_data(dY1, W1, dXa, ws),
        "fc1_bwd_weight": lambda: ict.ict_linear_bwd_weight(dY1, X, dW1, ws),
        "fc2_bwd_weight": lambda: ict.ict_linear_bwd_weight(dY2, H1, dW2, ws),
    }
    ms = {k: ev_time(f, flush=flush) for k, f in trio.items()}
    tot = sum(ms.values())
    out["vit_b_linear_trio"] = {
        "tops": round(6 * gop / tot, 1), "ms_total": round(tot, 4),
        "tops_each": {k: round(gop / v, 1) for k, v in ms.items()},
        "note": "each call includes its exponent-alignment passes; 357.0 GOP per trio",
    }
    del X, W1, W2, dY1, dY2, H1, Y2, dXa, dHa, dW1, dW2, ws
    # ResNet-50 SGD arena: 5 B per element + 5 B per group of 64
    c5 = wl.resnet50_sgd_arena(seed=0)
    Wd, Vd, Gd = (E.from_host(c5[k]) for k in ("W", "V", "G"))
    nbytes = 5 * c5["numel"] + 5 * Wd.rows
    t = ev_time(lambda: ict.ict_sgd_momentum_step(Wd, Vd, Gd, (230, 8), (205, 11)), n=20, flush=flush)
    out["resnet50_sgd"] = {"gbs": round(nbytes / t / 1e6, 1), "us": round(t * 1e3, 2),
                           "frac_hbm": round(nbytes / t / 1e6 / peaks["hbm"], 3),
                           "bytes_per_step": nbytes}
    del Wd, Vd, Gd
    torch.cuda.empty_cache()
    return out


# --------------------------------------------------------------------- oracle arm


def oracle_step_time(tokens: int):
    """The CPU oracle on the same step with `tokens` of the 12608 tokens."""
    import oracle

    cfg = wl.vit_ti_mlp(seed=0, tokens=tokens)
    X, W1, W2, dY2 = cfg["X"], cfg["W1"], cfg["W2"], cfg["dY2"]
    t0 = time.perf_counter()
    H = oracle.linear_fwd(X, W1, 1, GROUP)
    G = oracle.gelu_fwd(H)
    oracle.linear_fwd(G, W2, 1, GROUP)
    dG = oracle.linear_bwd_data(dY2, W2, 1, GROUP)
    dW2 = oracle.linear_bwd_weight(dY2, G, 1, HID)
    dH = oracle.gelu_bwd(H, dG, 1, GROUP)
    oracle.linear_bwd_data(dH, W1, 1, GROUP)
    dW1 = oracle.linear_bwd_weight(dH, X, 1, D)
    oracle.sgd_step(W1, cfg["V1"], dW1, *cfg["sgd"].values())
    oracle.sgd_step(W2, cfg["V2"], dW2, *cfg["sgd"].values())
    dt = time.perf_counter() - t0
    ops = 6 * 2 * tokens * D * HID
    return dt, ops, oracle.num_threads()


def base_line(args, n_gpus):
    return {
        "metric": "(C,e) GEMM TOPS fwd+bwd vs INT8 tensor peak; int-SGD update GB/s vs HBM",
        "unit": "TOPS", "n_gpus": n_gpus, "steps": args.steps, "warmup": args.warmup,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic (seeded; ViT-Ti layer shapes)",
        "config": {"workload": "vit_ti_mlp_block_step", "tokens": TOKENS, "d": D, "hidden": HID,
                   "group": GROUP, "gop_per_step": round(STEP_OPS / 1e9, 3),
                   "parallelism": f"replicas{n_gpus}" if n_gpus > 1 else "single",
                   "l2": "flushed between steps (512 MB write)"},
    }


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    tokens = TOKENS
    times = []
    for _ in range(max(1, args.warmup // 3)):
        oracle_step_time(tokens)
    for _ in range(max(1, min(args.steps, 3))):
        dt, ops, cores = oracle_step_time(tokens)
        times.append(dt)
    dt = float(np.mean(times))
    value = ops / dt / 1e12
    line = base_line(args, args.gpus)
    line.update({
        "impl": "reference", "value": value, "ms_per_step": dt * 1e3 * TOKENS / tokens,
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": cores, "kind": "oracle",
                         "sample": f"{tokens} of {TOKENS} tokens per step, {len(times)} steps"},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    })
    print(json.dumps(line))


def main():
    args = parse()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
        return
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    from integer_only_nn_02_b200 import ict

    peaks = load_peaks()
    step = MlpStep(ict, seed=rank)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    step.run()
    torch.cuda.synchronize()
    code, raw = ict.ict_get_device_status()
    if code != 0:
        raise SystemExit(f"device status {code} ({raw:#x})")

    clocks = ClockSampler(torch.cuda.current_device())
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = ict.ict_launch_count()
    clocks.start()
    t0 = time.perf_counter()
    ms, per_call = time_steps(step, args.steps, args.warmup, flush)
    wall = time.perf_counter() - t0
    clk = clocks.stop()
    launches = ict.ict_launch_count() - launches0
    launches_per_step = launches / (args.steps + args.warmup)
    torch.cuda.synchronize()
    if dist:
        t = torch.tensor([ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
        dist.barrier()
    e2e_ms, h2d, d2h = time_e2e(step, args.steps, args.warmup)
    if dist:
        t = torch.tensor([e2e_ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    code, raw = ict.ict_get_device_status()
    if code != 0:
        raise SystemExit(f"device status {code} ({raw:#x})")

    names = [n for n, _ in step.calls]
    breakdown = {n: round(float(v), 4) for n, v in zip(names, per_call)}
    # dominant kernel: fc1 forward is exactly one tensor-core launch (both operands are
    # uniform along K), so its event time is the kernel's own duration
    gemm_ms = breakdown["fc1_fwd"]
    int8_peak = 2.0 * peaks["bf16"]  # measured bf16 dense x nominal int8/bf16 ratio (2)
    achieved = (2 * TOKENS * D * HID) / (gemm_ms * 1e-3) / 1e12
    value = STEP_OPS / (ms * 1e-3) / 1e12 * world
    line = base_line(args, world)
    line.update({
        "value": round(value, 2), "ms_per_step": round(ms, 4),
        "e2e": {"value": round(STEP_OPS / (e2e_ms * 1e-3) / 1e12 * world, 2), "unit": "TOPS",
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)},
        "gpu_launches": int(round(launches_per_step * args.steps)),
        "gpu_launches_per_step": round(launches_per_step, 2),
        "breakdown_ms": breakdown,
        "roofline": {"kernel": "gemm_ce_kernel (fc1 forward, 12608x192 . 192x768)", "bound": "tensor",
                     "achieved": round(achieved, 1), "peak": round(int8_peak, 1), "unit": "TFLOP/s",
                     "frac": round(achieved / int8_peak, 4),
                     "peak_note": f"int8 = 2 x {peaks['source']} bf16 dense {peaks['bf16']} TF/s",
                     "traffic": None},
        "clocks": clk,
        "wall_s_timed": round(wall, 3),
    })
    if rank == 0 and not args.no_side:
        line["side"] = side_measurements(ict, torch, peaks)
        try:
            a = torch.randint(-127, 128, (8192, 8192), dtype=torch.int8, device="cuda")
            b = torch.randint(-127, 128, (8192, 8192), dtype=torch.int8, device="cuda")
            for _ in range(3):
                torch._int_mm(a, b)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(10):
                torch._int_mm(a, b)
            e1.record()
            torch.cuda.synchronize()
            line["side"]["torch_int_mm_8192_tops"] = round(10 * 2 * 8192 ** 3 / (e0.elapsed_time(e1) * 1e-3) / 1e12, 1)
        except Exception as exc:  # pragma: no cover
            line["side"]["torch_int_mm_8192_tops"] = f"unavailable: {exc}"
    if rank == 0:
        try:
            dt, ops, cores = oracle_step_time(TOKENS)
            line["cpu_baseline"] = {"value": round(ops / dt / 1e12, 6), "unit": "TOPS", "cores": cores,
                                    "kind": "oracle", "sample": f"one full step ({TOKENS} tokens)",
                                    "seconds": round(dt, 2)}
        except Exception as exc:  # pragma: no cover
            line["cpu_baseline"] = {"value": None, "unit": "TOPS", "cores": None, "kind": "oracle",
                                    "sample": f"failed: {exc}"}
        print(json.dumps(line))
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
