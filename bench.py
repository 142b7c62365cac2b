"""Benchmark of the integer-only (C,e) training hot path on B200.

Default step (--config vit_b_linear_trio): the six contractions of a ViT-B-shaped MLP
block through libict.so on synthetic seeded inputs (12608 tokens = 64 images x 197
tokens; d = 768, hidden 3072; (1, 64) exponent groups): fc1 forward (12608x768 .
768x3072), fc2 forward (12608x3072 . 3072x768), both backward-data Products and both
backward-weight Products ("Memory-Efficient Integer-Only Training of Deep Neural
Networks", Table 6: linear layer = Product; Figure 1a: forward and backward in integer
arithmetic).  metric: (C,e) GEMM TOPS over the step (356.95 GOP per step).

The same run measures every other configuration as a side entry with its own value,
roofline, end-to-end number and oracle baseline:
  vit_ti_mlp          ViT-Ti MLP block training step (22.31 GOP), TOPS
  resnet18_conv3x3    3x3 conv fwd, bwd-data, bwd-weight on 128x56x56x64, TOPS
  resnet50_sgd        int-SGD update of a ResNet-50-sized parameter arena, GB/s
  single_linear       64x128 linear layer fwd+bwd+SGD, microseconds per step
  resnet18_block_tail residual add fused with ReLU, ReLU backward and gradient merge on
                      the ResNet-18 stage-1 activations, GB/s

Usage:  python bench.py [--config C] [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 run under torchrun, one rank per GPU, each with its own batch of the
configuration's size (weak scaling); the reported time is the max over ranks.  The linear
configurations and the convolution train data-parallel: every backward-weight Product
exchanges exact integer sums (SUM, with the linear layers' alignment targets by MAX) and
the convolution's all-pixel output groups exchange their needs (MAX) over NCCL, so all
ranks compute what a single GPU computes on the whole batch.  resnet50_sgd and
resnet18_block_tail run as independent replicas.
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

L2_FLUSH_BYTES = 512 << 20  # larger than the 126 MB L2
METRIC = "(C,e) GEMM TOPS fwd+bwd vs INT8 tensor peak; int-SGD update GB/s vs HBM"
CLASS_NAMES = ["gemm", "sgd", "align", "requant", "gelu", "estar", "other", "pointwise"]  # ict_kernel_class order
CLASS_KERNELS = {
    "gemm": "gemm_ce_kernel (tcgen05 kind::i8, fused FIT epilogue)",
    "sgd": "sgd_rows_kernel / sgd_vec_kernel",
    "align": "align_rows_kernel / align_transpose_kernel (ALIGN_MAX shifts)",
    "requant": "requant_group_block_kernel / requant_rows_kernel",
    "gelu": "gelu_fwd_kernel / gelu_bwd_vec_kernel",
    "estar": "estar_rows_kernel / estar_cols_scratch_kernel",
    "other": "fills, weight re-layout, exponent tables",
    "pointwise": "clip_kernel / sum_rows_kernel / sum_global_*_kernel (ReLU, Sum)",
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="vit_b_linear_trio", choices=list(STEPS))
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None, help="timed steps (default 20; 100 for resnet50_sgd)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-side", action="store_true", help="skip the other configurations' side numbers")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
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
            try:
                uuid = str(torch.cuda.get_device_properties(torch_index).uuid)
                uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
                h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            except Exception:
                h = pynvml.nvmlDeviceGetHandleByIndex(torch_index)
            self.handle = h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:  # pragma: no cover
            self.handle = None

    def _reasons(self):
        f = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(self.nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        return int(f(self.handle))

    def _loop(self):
        while not self.stop_flag:
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.handle, self.nv.NVML_CLOCK_SM))
                self.reason_bits |= self._reasons()
            except Exception:
                pass
            time.sleep(0.002)

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


# --------------------------------------------------------------------- steps


class Step:
    """A configuration's step: device state, the library calls of one step, its work."""

    unit = "TOPS"
    higher_is_better = True
    sample_arg = None

    def __init__(self, ict, torch):
        self.ict, self.torch = ict, torch
        self.calls = []
        self.h2d = []  # device tensors refreshed from pinned host copies every e2e step
        self.d2h = []  # device tensors read back every e2e step

    def ws(self, nbytes):
        return self.torch.empty(max(int(nbytes), 256), dtype=self.torch.uint8, device="cuda")

    data_parallel = False  # True: with several ranks the batch is split and dW all-reduced
    gemm_bytes = 0  # algorithmic int8 bytes (operands read, results written) of the step's Products

    def bwd_weight(self, dY, X, dW, ws):
        """One linear layer's backward-weight call.  On one GPU, the library's single call;
        with several ranks (each holding its own shard of the batch), the split-batch form
        whose targets and integer sums are all-reduced over NCCL, bit-identical to one GPU
        on the whole batch."""
        from integer_only_nn_02_b200 import dp

        world = dp.world_size()
        if world == 1:
            return lambda: self.ict.ict_linear_bwd_weight(dY, X, dW, ws)
        g = dp.LinearWeightGrad(dY, X, total_rows=world * dY.rows)
        self.exchanged_bytes = getattr(self, "exchanged_bytes", 0) + g.exchanged_bytes
        return lambda: g(dY, X, dW)

    def run(self, events=None):
        for i, (_, fn) in enumerate(self.calls):
            if events is not None:
                events[i][0].record()
            fn()
            if events is not None:
                events[i][1].record()

    @classmethod
    def value_of(cls, units, seconds):
        """The metric from the step's work units and its time."""
        if cls.unit == "us":
            return seconds * 1e6
        if cls.unit == "GB/s":
            return units / seconds / 1e9
        return units / seconds / 1e12


class MlpStep(Step):
    data_parallel = True
    TOKENS, D, HID, GROUP = 64 * 197, 192, 768, 32
    sample_arg = 64 * 197
    workload = {"workload": "vit_ti_mlp_block_step", "tokens": 12608, "d": 192, "hidden": 768, "group": 32,
                "gop_per_step": 22.31}

    def __init__(self, ict, torch, seed):
        super().__init__(ict, torch)
        E = ict.DevCE
        cfg = wl.vit_ti_mlp(seed=seed)
        self.X, self.W1, self.W2, self.dY2 = (E.from_host(cfg[k]) for k in ("X", "W1", "W2", "dY2"))
        self.V1, self.V2 = E.from_host(cfg["V1"]), E.from_host(cfg["V2"])
        M, D, H, G = self.TOKENS, self.D, self.HID, self.GROUP
        self.H, self.G, self.dG, self.dH = (E.empty(M, H, 1, G) for _ in range(4))
        self.Y, self.dX = E.empty(M, D, 1, G), E.empty(M, D, 1, G)
        self.dW2, self.dW1 = E.empty(D, H, 1, H), E.empty(H, D, 1, D)
        w = ict.ict_linear_workspace
        ws = self.ws(max(w(0, self.X, self.W1, self.H), w(0, self.G, self.W2, self.Y),
                         w(1, self.dY2, self.W2, self.dG), w(2, self.dY2, self.G, self.dW2),
                         w(1, self.dH, self.W1, self.dX), w(2, self.dH, self.X, self.dW1)))
        mom, lr = cfg["sgd"]["mom"], cfg["sgd"]["lr"]
        self.calls = [
            ("fc1_fwd", lambda: ict.ict_linear_fwd(self.X, self.W1, self.H, ws)),
            ("gelu_fwd", lambda: ict.ict_gelu_fwd(self.H, self.G)),
            ("fc2_fwd", lambda: ict.ict_linear_fwd(self.G, self.W2, self.Y, ws)),
            ("fc2_bwd_data", lambda: ict.ict_linear_bwd_data(self.dY2, self.W2, self.dG, ws)),
            ("fc2_bwd_weight", self.bwd_weight(self.dY2, self.G, self.dW2, ws)),
            ("gelu_bwd", lambda: ict.ict_gelu_bwd(self.H, self.dG, self.dH)),
            ("fc1_bwd_data", lambda: ict.ict_linear_bwd_data(self.dH, self.W1, self.dX, ws)),
            ("fc1_bwd_weight", self.bwd_weight(self.dH, self.X, self.dW1, ws)),
            ("sgd_w1", lambda: ict.ict_sgd_momentum_step(self.W1, self.V1, self.dW1, mom, lr)),
            ("sgd_w2", lambda: ict.ict_sgd_momentum_step(self.W2, self.V2, self.dW2, mom, lr)),
        ]
        self.units = 6 * 2 * M * D * H
        self.gemm_bytes = 6 * (M * D + D * H + M * H)
        self.h2d = [self.X.mant, self.X.exp, self.dY2.mant, self.dY2.exp]
        self.d2h = [self.W1.mant, self.W1.exp, self.W2.mant, self.W2.exp]

    @staticmethod
    def oracle_step(tokens):
        import oracle

        cfg = wl.vit_ti_mlp(seed=0, tokens=tokens)
        X, W1, W2, dY2 = cfg["X"], cfg["W1"], cfg["W2"], cfg["dY2"]
        G = MlpStep.GROUP
        mom, lr = cfg["sgd"]["mom"], cfg["sgd"]["lr"]
        t0 = time.perf_counter()
        H = oracle.linear_fwd(X, W1, 1, G)
        Gl = oracle.gelu_fwd(H)
        oracle.linear_fwd(Gl, W2, 1, G)
        dG = oracle.linear_bwd_data(dY2, W2, 1, G)
        dW2 = oracle.linear_bwd_weight(dY2, Gl, 1, W2.cols)
        dH = oracle.gelu_bwd(H, dG, 1, G)
        oracle.linear_bwd_data(dH, W1, 1, G)
        dW1 = oracle.linear_bwd_weight(dH, X, 1, W1.cols)
        oracle.sgd_step(W1, cfg["V1"], dW1, mom, lr)
        oracle.sgd_step(W2, cfg["V2"], dW2, mom, lr)
        dt = time.perf_counter() - t0
        return dt, 6 * 2 * tokens * MlpStep.D * MlpStep.HID, f"one full step ({tokens} tokens)"


class LinearStep(Step):
    data_parallel = True
    unit = "us"
    higher_is_better = False
    workload = {"workload": "single_linear_step", "m": 64, "k": 128, "n": 64, "group": 32}

    def __init__(self, ict, torch, seed):
        super().__init__(ict, torch)
        E = ict.DevCE
        cfg = wl.single_linear(seed=seed)
        self.X, self.W, self.dY, self.V = (E.from_host(cfg[k]) for k in ("X", "W", "dY", "V"))
        G = cfg["out_group"]
        self.Y, self.dX, self.dW = E.empty(64, 64, 1, G), E.empty(64, 128, 1, G), E.empty(64, 128, 1, 128)
        w = ict.ict_linear_workspace
        ws = self.ws(max(w(0, self.X, self.W, self.Y), w(1, self.dY, self.W, self.dX),
                         w(2, self.dY, self.X, self.dW)))
        mom, lr = cfg["sgd"]["mom"], cfg["sgd"]["lr"]
        self.calls = [
            ("fwd", lambda: ict.ict_linear_fwd(self.X, self.W, self.Y, ws)),
            ("bwd_data", lambda: ict.ict_linear_bwd_data(self.dY, self.W, self.dX, ws)),
            ("bwd_weight", self.bwd_weight(self.dY, self.X, self.dW, ws)),
            ("sgd", lambda: ict.ict_sgd_momentum_step(self.W, self.V, self.dW, mom, lr)),
        ]
        self.units = 1
        self.h2d = [self.X.mant, self.X.exp, self.dY.mant, self.dY.exp]
        self.d2h = [self.W.mant, self.W.exp]

    @staticmethod
    def oracle_step(_):
        import oracle

        cfg = wl.single_linear(seed=0)
        X, W, dY, V = cfg["X"], cfg["W"], cfg["dY"], cfg["V"]
        t0 = time.perf_counter()
        oracle.linear_fwd(X, W, 1, 32)
        oracle.linear_bwd_data(dY, W, 1, 32)
        dW = oracle.linear_bwd_weight(dY, X, 1, 128)
        oracle.sgd_step(W, V, dW, cfg["sgd"]["mom"], cfg["sgd"]["lr"])
        return time.perf_counter() - t0, 1, "one full step"


class ConvStep(Step):
    data_parallel = True
    sample_arg = 32
    workload = {"workload": "resnet18_conv3x3_fwd_bwd", "n": 128, "h": 56, "w": 56, "c": 64, "k": 64,
                "group": 32, "gop_per_step": 88.785}

    def __init__(self, ict, torch, seed):
        super().__init__(ict, torch)
        E = ict.DevCE
        cfg = wl.resnet18_conv3x3(seed=seed)
        d, G = cfg["conv"], cfg["out_group"]
        self.X, self.W, self.dY = (E.from_host(cfg[k]) for k in ("X", "W", "dY"))
        npix = self.X.rows
        self.Y, self.dX = E.empty(npix, 64, npix, G), E.empty(npix, 64, npix, G)
        self.dW = E.empty(64, 576, 1, 576)
        from integer_only_nn_02_b200 import dp

        if dp.world_size() > 1:
            # data parallel: every rank holds its own 128 images; the ranks share the
            # weights and the activations' pixel-uniform exponents (those of rank 0's draw)
            c0 = wl.resnet18_conv3x3(seed=0)
            for t, k in ((self.X, "X"), (self.dY, "dY")):
                t.exp.copy_(torch.from_numpy(c0[k].exp))
            self.W = E.from_host(c0["W"])
            fwd = dp.ConvSplit(0, d, self.X, self.W, self.Y)
            bwd = dp.ConvSplit(1, d, self.dY, self.W, self.dX)
            wgt = dp.ConvWeightGrad(d)
            self.exchanged_bytes = fwd.need.numel() * 4 + bwd.need.numel() * 4 + wgt.exchanged_bytes
            self.calls = [
                ("fwd", lambda: fwd(self.X, self.W, self.Y)),
                ("bwd_data", lambda: bwd(self.dY, self.W, self.dX)),
                ("bwd_weight", lambda: wgt(self.dY, self.X, self.dW)),
            ]
        else:
            cw = ict.ict_conv_workspace
            ws = self.ws(max(cw(0, d), cw(1, d), cw(2, d)))
            self.calls = [
                ("fwd", lambda: ict.ict_conv_implicit_gemm(0, d, self.X, self.W, self.Y, ws)),
                ("bwd_data", lambda: ict.ict_conv_implicit_gemm(1, d, self.dY, self.W, self.dX, ws)),
                ("bwd_weight", lambda: ict.ict_conv_implicit_gemm(2, d, self.dY, self.X, self.dW, ws)),
            ]
        self.units = 3 * 2 * npix * 64 * 576
        self.gemm_bytes = 3 * (2 * npix * 64 + 64 * 576)
        self.h2d = [self.X.mant, self.X.exp, self.dY.mant, self.dY.exp]
        self.d2h = [self.dW.mant, self.dW.exp]

    @staticmethod
    def oracle_step(images):
        import oracle

        cfg = wl.resnet18_conv3x3(seed=0, n=images)
        X, W, dY, d = cfg["X"], cfg["W"], cfg["dY"], cfg["conv"]
        t0 = time.perf_counter()
        oracle.conv(oracle.CONV_FWD, d, X, W, X.rows, 32)
        oracle.conv(oracle.CONV_BWD_DATA, d, dY, W, X.rows, 32)
        oracle.conv(oracle.CONV_BWD_WEIGHT, d, dY, X, 1, W.cols)
        dt = time.perf_counter() - t0
        return dt, 3 * 2 * X.rows * 64 * 576, f"fwd+bwd-data+bwd-weight on {images} of the 128 images"


class TrioStep(Step):
    data_parallel = True
    sample_arg = 2048
    workload = {"workload": "vit_b_linear_trio", "tokens": 12608, "d": 768, "hidden": 3072, "group": 64,
                "gop_per_step": 356.952}

    def __init__(self, ict, torch, seed):
        super().__init__(ict, torch)
        E = ict.DevCE
        cfg = wl.vit_b_linear_trio(seed=seed)
        self.X, self.W1, self.W2, self.dY1, self.dY2 = (E.from_host(cfg[k]) for k in ("X", "W1", "W2", "dY1", "dY2"))
        M, G = self.X.rows, cfg["out_group"]
        self.H1, self.Y2 = E.empty(M, 3072, 1, G), E.empty(M, 768, 1, G)
        self.dXo, self.dHo = E.empty(M, 768, 1, G), E.empty(M, 3072, 1, G)
        self.dW1, self.dW2 = E.empty(3072, 768, 1, 768), E.empty(768, 3072, 1, 3072)
        w = ict.ict_linear_workspace
        ws = self.ws(max(w(0, self.X, self.W1, self.H1), w(0, self.H1, self.W2, self.Y2),
                         w(1, self.dY2, self.W2, self.dHo), w(1, self.dY1, self.W1, self.dXo),
                         w(2, self.dY1, self.X, self.dW1), w(2, self.dY2, self.H1, self.dW2)))
        self.calls = [
            ("fc1_fwd", lambda: ict.ict_linear_fwd(self.X, self.W1, self.H1, ws)),
            ("fc2_fwd", lambda: ict.ict_linear_fwd(self.H1, self.W2, self.Y2, ws)),
            ("fc2_bwd_data", lambda: ict.ict_linear_bwd_data(self.dY2, self.W2, self.dHo, ws)),
            ("fc1_bwd_data", lambda: ict.ict_linear_bwd_data(self.dY1, self.W1, self.dXo, ws)),
            ("fc1_bwd_weight", self.bwd_weight(self.dY1, self.X, self.dW1, ws)),
            ("fc2_bwd_weight", self.bwd_weight(self.dY2, self.H1, self.dW2, ws)),
        ]
        self.units = 6 * 2 * M * 768 * 3072
        self.gemm_bytes = 6 * (M * 768 + 768 * 3072 + M * 3072)
        self.h2d = [self.X.mant, self.X.exp, self.dY1.mant, self.dY1.exp, self.dY2.mant, self.dY2.exp]
        self.d2h = [self.dW1.mant, self.dW1.exp, self.dW2.mant, self.dW2.exp]

    @staticmethod
    def oracle_step(tokens):
        import oracle

        cfg = wl.vit_b_linear_trio(seed=0, tokens=tokens)
        X, W1, W2, dY1, dY2 = (cfg[k] for k in ("X", "W1", "W2", "dY1", "dY2"))
        t0 = time.perf_counter()
        H1 = oracle.linear_fwd(X, W1, 1, 64)
        oracle.linear_fwd(H1, W2, 1, 64)
        oracle.linear_bwd_data(dY2, W2, 1, 64)
        oracle.linear_bwd_data(dY1, W1, 1, 64)
        oracle.linear_bwd_weight(dY1, X, 1, X.cols)
        oracle.linear_bwd_weight(dY2, H1, 1, H1.cols)
        dt = time.perf_counter() - t0
        return dt, 6 * 2 * tokens * 768 * 3072, f"the six contractions on {tokens} of the 12608 tokens"


class SgdStep(Step):
    unit = "GB/s"
    workload = {"workload": "resnet50_sgd_arena", "params": 25557032, "tensors": 161, "groups": 399329,
                "group": 64, "bytes_per_step": 5 * 25557032 + 5 * 399329}

    def __init__(self, ict, torch, seed):
        super().__init__(ict, torch)
        E = ict.DevCE
        c5 = wl.resnet50_sgd_arena(seed=seed)
        self.W, self.V, self.G = (E.from_host(c5[k]) for k in ("W", "V", "G"))
        mom, lr = c5["sgd"]["mom"], c5["sgd"]["lr"]
        self.calls = [("sgd", lambda: ict.ict_sgd_momentum_step(self.W, self.V, self.G, mom, lr))]
        # algorithmic bytes: W, V, G mantissas read, W, V mantissas written (5 B per
        # parameter) and the same for the per-group exponents (5 B per group)
        self.units = 5 * c5["numel"] + 5 * self.W.rows
        self.h2d = [self.G.mant, self.G.exp]
        self.d2h = [self.W.mant, self.W.exp]

    @staticmethod
    def oracle_step(_):
        import oracle

        c5 = wl.resnet50_sgd_arena(seed=0)
        t0 = time.perf_counter()
        oracle.sgd_step(c5["W"], c5["V"], c5["G"], c5["sgd"]["mom"], c5["sgd"]["lr"])
        dt = time.perf_counter() - t0
        return dt, 5 * c5["numel"] + 5 * c5["W"].rows, "one full update of the 25.6 M-parameter arena"


class BlockTailStep(Step):
    """The pointwise steps around a ResNet-18 stage-1 basic block's convolutions, on its
    128 x 56 x 56 x 64 activations (channel groups of 32 spanning all pixels): the
    residual add and the ReLU after it in one rounding pass, A = ReLU(FIT(conv_out +
    identity)); backward dS = dA * 1[A > 0] (the same mask as 1[S > 0]) and the gradient
    merge dX = FIT(dX_conv + dS) at the block input."""

    unit = "GB/s"
    N_IMG, HW, C, GROUP = 128, 56, 64, 32
    sample_arg = 128  # images in the oracle's sample: the whole workload, about 7 s
    workload = {"workload": "resnet18_block_tail", "n": 128, "h": 56, "w": 56, "c": 64, "group": 32,
                "ops": "sum+relu (fused), relu_bwd, sum"}

    def __init__(self, ict, torch, seed):
        super().__init__(ict, torch)
        E = ict.DevCE
        cfg = wl.resnet18_block_tail(seed=seed, n=self.N_IMG)
        npix = cfg["Y"].rows
        self.Y, self.X, self.dA, self.dXc = (E.from_host(cfg[k]) for k in ("Y", "X", "dA", "dXc"))
        G = self.GROUP
        self.A = E.empty(npix, self.C, npix, G)
        self.dS, self.dX = E.empty(npix, self.C, npix, G), E.empty(npix, self.C, npix, G)
        ws = self.ws(ict.ict_sum_workspace(self.Y, self.X, self.A))
        self.calls = [
            ("residual_add_relu", lambda: ict.ict_sum_act(self.Y, self.X, self.A, ict.ACT_RELU, ws)),
            ("relu_bwd", lambda: ict.ict_relu_bwd(self.A, self.dA, False, self.dS)),
            ("grad_merge", lambda: ict.ict_sum(self.dXc, self.dS, self.dX, ws)),
        ]
        n = npix * self.C
        self.units = (3 + 3 + 3) * n  # algorithmic bytes: inputs read once, outputs written once
        self.h2d = [self.Y.mant, self.Y.exp, self.dA.mant, self.dA.exp]
        self.d2h = [self.dX.mant, self.dX.exp]

    @staticmethod
    def oracle_step(n_img):
        import oracle

        cfg = wl.resnet18_block_tail(seed=0, n=n_img)
        g = (cfg["Y"].rows, BlockTailStep.GROUP)
        t0 = time.perf_counter()
        S = oracle.sum_(cfg["Y"], cfg["X"], *g)
        A = oracle.relu_fwd(S)
        dS = oracle.relu_bwd(A, cfg["dA"])
        oracle.sum_(cfg["dXc"], dS, *g)
        dt = time.perf_counter() - t0
        n = cfg["Y"].rows * BlockTailStep.C
        return dt, 9 * n, f"one full block tail on {n_img} images"


STEPS = {"vit_ti_mlp": MlpStep, "vit_b_linear_trio": TrioStep, "resnet18_conv3x3": ConvStep,
         "resnet50_sgd": SgdStep, "single_linear": LinearStep, "resnet18_block_tail": BlockTailStep}


# --------------------------------------------------------------------- timing


def backlog(torch, ms):
    """Hold the stream with a spin kernel for about `ms` so that the host enqueues the
    launches that follow before the GPU reaches them: events between them then time the
    kernels, not the host's launch rate."""
    torch.cuda._sleep(int(ms * 2.0e6))


def time_graph(step, graph, K, W, flush):
    """Mean device time per step (ms): one graph replay per step, CUDA events on the
    replay stream, L2 flushed (512 MB write) before every step."""
    torch = step.torch
    for _ in range(W):
        flush.fill_(1)
        graph.replay()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for a, b in ev:
        flush.fill_(1)
        a.record()
        graph.replay()
        b.record()
    torch.cuda.synchronize()
    return float(np.mean([a.elapsed_time(b) for a, b in ev]))


def time_eager(step, K, W, flush, backlogged):
    """Mean device time per step (ms) with the calls launched one by one from Python,
    and the per-call breakdown.  backlogged=True holds the stream first, so the events
    time the kernels; False measures what a plain Python loop gets (host launch rate
    included)."""
    torch = step.torch
    for _ in range(W):
        step.run()
    torch.cuda.synchronize()
    n = len(step.calls)
    per_call = np.zeros(n)
    totals = []
    for _ in range(K):
        flush.fill_(1)
        if backlogged:
            backlog(torch, 1.0 + 0.1 * n)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        step.run(ev)
        torch.cuda.synchronize()
        per_call += [a.elapsed_time(b) for a, b in ev]
        totals.append(ev[0][0].elapsed_time(ev[-1][1]))
    return float(np.mean(totals)), per_call / K


def time_classes(step, K, flush):
    """Device time per kernel class inside K steps: the library brackets each of its
    kernels with CUDA events on the launch's stream while timing is enabled; the stream
    is held first so that the events time kernels, not launch gaps."""
    ict, torch = step.ict, step.torch
    torch.cuda.synchronize()
    ict.ict_timing_read(0, reset=True)
    ict.ict_timing_enable(True)
    for _ in range(K):
        flush.fill_(1)
        backlog(torch, 1.0 + 0.1 * len(step.calls))
        step.run()
    torch.cuda.synchronize()
    ict.ict_timing_enable(False)
    out = {}
    for i, name in enumerate(CLASS_NAMES):
        ms, n, work = ict.ict_timing_read(i, reset=False)
        if n:
            out[name] = {"ms_per_step": ms / K, "launches_per_step": n / K, "work_per_step": work / K}
    ict.ict_timing_read(0, reset=True)
    return out


def time_e2e(step, graph, K, W):
    """The same step through the public API with host buffers: every step's inputs are
    copied from pinned host memory and its results read back into pinned host memory,
    all inside the timed region.  The copies are pipelined with the compute, as a
    training loop's input prefetch does.  The step's inputs travel as one packed pinned
    buffer into one of two device staging buffers (one host call per step, on a copy
    stream) while the previous step computes; two CUDA graphs, one per staging buffer,
    each scatter their staging buffer into the step's input tensors, run the step and
    gather its results into a packed output staging buffer, which a second copy stream
    reads back (one host call) while the next step computes.  Returns the time per step
    and the host bytes moved each way per step."""
    torch = step.torch
    ict = step.ict

    def layout(ts):
        offs, off = [], 0
        for t in ts:
            offs.append(off)
            off += (t.numel() * t.element_size() + 255) // 256 * 256
        return offs, max(off, 256)

    def view(buf, off, t):
        n = t.numel() * t.element_size()
        return buf[off:off + n].view(t.dtype).view(t.shape)

    ins, outs = list(step.h2d), list(step.d2h)
    in_off, in_bytes = layout(ins)
    out_off, out_bytes = layout(outs)
    h2d = sum(t.numel() * t.element_size() for t in ins)
    d2h = sum(t.numel() * t.element_size() for t in outs)
    host_in = torch.empty(in_bytes, dtype=torch.uint8).pin_memory()
    host_out = torch.empty(out_bytes, dtype=torch.uint8).pin_memory()
    for t, o in zip(ins, in_off):
        view(host_in, o, t).copy_(t.cpu())
    stage_in = [torch.empty(in_bytes, dtype=torch.uint8, device="cuda") for _ in range(2)]
    stage_out = [torch.empty(out_bytes, dtype=torch.uint8, device="cuda") for _ in range(2)]

    def graph_fn(b):
        def fn():
            for t, o in zip(ins, in_off):
                t.copy_(view(stage_in[b], o, t))
            step.run()
            for t, o in zip(outs, out_off):
                view(stage_out[b], o, t).copy_(t)
        return fn

    for b in range(2):  # the staging buffers' first contents: the inputs themselves
        stage_in[b].copy_(host_in)
    graphs = [ict.StepGraph(graph_fn(b)) for b in range(2)]
    cur = torch.cuda.current_stream()
    cs_in, cs_out = torch.cuda.Stream(), torch.cuda.Stream()
    landed = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]
    read = [torch.cuda.Event() for _ in range(2)]

    def prefetch(b):  # host -> staging b, once the graph that last read it has finished
        cs_in.wait_event(done[b])
        with torch.cuda.stream(cs_in):
            stage_in[b].copy_(host_in, non_blocking=True)
            landed[b].record(cs_in)

    def run(n):
        for b in range(2):
            done[b].record(cur)
            read[b].record(cs_out)
        prefetch(0)
        for i in range(n):
            b = i & 1
            if i + 1 < n:
                prefetch(b ^ 1)  # overlaps this step's compute
            cur.wait_event(landed[b])
            cur.wait_event(read[b])  # the read-back of two steps ago has left stage_out[b]
            graphs[b].replay()
            done[b].record(cur)
            cs_out.wait_event(done[b])
            with torch.cuda.stream(cs_out):
                host_out.copy_(stage_out[b], non_blocking=True)
                read[b].record(cs_out)
        cur.wait_stream(cs_out)
        cur.wait_stream(cs_in)

    run(W)
    torch.cuda.synchronize()
    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    run(K)
    b_.record()
    torch.cuda.synchronize()
    del graphs  # released here, before any process-group teardown (they may hold collectives)
    return a.elapsed_time(b_) / K, h2d, d2h


def class_rate(name, c, peaks):
    """(achieved, peak, unit, bound) of one kernel class over its own device time."""
    if name == "gemm":
        return c["work_per_step"] / (c["ms_per_step"] * 1e-3) / 1e12, 2.0 * peaks["bf16"], "TFLOP/s", "tensor"
    return c["work_per_step"] / (c["ms_per_step"] * 1e-3) / 1e9, peaks["hbm"], "GB/s", "hbm"


# CUDA sources of each kernel class's kernels: a committed DRAM-traffic figure is used
# only while these files are unchanged since the counters were taken
CLASS_SOURCES = {
    "gemm": ["ict_gemm.cuh", "ict_device.cuh"],
    "sgd": ["ict_elementwise.cuh", "ict_device.cuh"],
    "align": ["ict_elementwise.cuh", "ict_device.cuh"],
    "requant": ["ict_elementwise.cuh", "ict_device.cuh"],
    "gelu": ["ict_elementwise.cuh", "ict_device.cuh"],
    "estar": ["ict_elementwise.cuh", "ict_device.cuh"],
    "other": ["ict_elementwise.cuh", "ict_device.cuh"],
    "pointwise": ["ict_pointwise.cuh", "ict_elementwise.cuh", "ict_device.cuh"],
}


def class_source_digest(kernel_class):
    """sha256 over the CUDA sources of one kernel class (file names and contents)."""
    import hashlib

    h = hashlib.sha256()
    src = os.path.join(ROOT, "integer_only_nn_02_b200", "csrc")
    for name in CLASS_SOURCES[kernel_class]:
        with open(os.path.join(src, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()


def measured_traffic(config, kernel_class):
    """DRAM bytes per launch (read + write) of a kernel class in a configuration, from
    the committed ncu summary, or None when the summary does not cover the class or was
    taken on other sources of that class's kernels."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    e = t.get("configs", {}).get(config, {}).get(kernel_class)
    if e is None or e.get("sources_sha256") != class_source_digest(kernel_class):
        return None
    return e["dram_bytes_per_launch"]


def roofline(classes, peaks, config, gemm_bytes=0):
    """Roofline of the kernel class with the most device time in the step: the
    memory-bound classes against the measured HBM copy rate; the tensor-core Product
    against whichever bound is binding for its shapes: the INT8 peak (measured dense
    bf16 x 2, the nominal int8/bf16 ratio) for its multiply-adds, or the HBM copy rate
    for its algorithmic bytes (int8 operands read once, int8 results written once) when
    moving those takes longer than the multiply-adds (short contractions)."""
    name = max(classes, key=lambda k: classes[k]["ms_per_step"])
    c = classes[name]
    achieved, peak, unit, bound = class_rate(name, c, peaks)
    alt = None
    if name == "gemm" and gemm_bytes:
        t_tensor = c["work_per_step"] / (2.0 * peaks["bf16"] * 1e12)
        t_hbm = gemm_bytes / (peaks["hbm"] * 1e9)
        hbm_rate = gemm_bytes / (c["ms_per_step"] * 1e-3) / 1e9
        if t_hbm > t_tensor:
            alt = {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": unit,
                   "frac": round(achieved / peak, 4)}
            achieved, peak, unit, bound = hbm_rate, peaks["hbm"], "GB/s", "hbm"
        else:
            alt = {"bound": "hbm", "achieved": round(hbm_rate, 1), "peak": round(peaks["hbm"], 1), "unit": "GB/s",
                   "frac": round(hbm_rate / peaks["hbm"], 4)}
    note = (f"INT8 = 2 x {peaks['source']} dense bf16 {peaks['bf16']} TF/s (burst)" if bound == "tensor"
            else f"{peaks['source']} HBM copy bandwidth")
    out = {"kernel": CLASS_KERNELS[name], "bound": bound, "achieved": round(achieved, 1), "peak": round(peak, 1),
           "unit": unit, "frac": round(achieved / peak, 4), "peak_note": note,
           "traffic": measured_traffic(config, name),
           "launches_per_step": c["launches_per_step"],
           "us_per_launch": round(1e3 * c["ms_per_step"] / c["launches_per_step"], 2)}
    if alt:
        out["algorithmic_bytes_per_step" if bound == "hbm" else "ops_per_step"] = (
            int(gemm_bytes) if bound == "hbm" else c["work_per_step"])
        out["other_bound"] = alt
    return out


def class_summary(classes, peaks):
    out = {}
    for name, c in classes.items():
        d = {"ms_per_step": round(c["ms_per_step"], 4), "launches_per_step": c["launches_per_step"]}
        if c["work_per_step"] > 0:
            achieved, peak, unit, _ = class_rate(name, c, peaks)
            d[unit] = round(achieved, 1)
            d["frac"] = round(achieved / peak, 4)
        out[name] = d
    return out


# --------------------------------------------------------------------- side measurements


def side_int_mm(torch):
    """torch._int_mm on 8192^3 (the library INT8 GEMM on this GPU), for context."""
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
        return round(10 * 2 * 8192 ** 3 / (e0.elapsed_time(e1) * 1e-3) / 1e12, 1)
    except Exception as exc:  # pragma: no cover
        return f"unavailable: {exc}"


def measure(step, ict, torch, peaks, flush, config, steps, warmup, dist=None):
    """Everything one configuration's line reports, for a constructed step: device time
    of one graph replay per step (max over ranks), end-to-end time through host
    buffers, host-launched time, the per-call and per-kernel-class breakdown, the
    roofline of the dominant kernel class and the SM clocks during the timed region."""
    step.run()
    torch.cuda.synchronize()
    code, raw = ict.ict_get_device_status()
    if code != 0:
        raise SystemExit(f"device status {code} ({raw:#x})")
    graph = ict.StepGraph(step.run)
    clocks = ClockSampler(torch.cuda.current_device())
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    ms = time_graph(step, graph, steps, warmup, flush)
    clk = clocks.stop()
    if dist:
        t = torch.tensor([ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
        dist.barrier()
    eager_ms, _ = time_eager(step, steps, warmup, flush, backlogged=False)
    _, per_call = time_eager(step, steps, warmup, flush, backlogged=True)
    classes = time_classes(step, steps, flush)
    e2e_ms, h2d, d2h = time_e2e(step, graph, steps, warmup)
    if dist:
        t = torch.tensor([e2e_ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    code, raw = ict.ict_get_device_status()
    if code != 0:
        raise SystemExit(f"device status {code} ({raw:#x})")
    world = dist.get_world_size() if dist else 1
    agg = world if step.higher_is_better else 1  # rates add over independent replicas
    out = {
        "value": round(step.value_of(step.units, ms * 1e-3) * agg, 3), "unit": step.unit,
        "ms_per_step": round(ms, 4),
        "e2e": {"value": round(step.value_of(step.units, e2e_ms * 1e-3) * agg, 3), "unit": step.unit,
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "copies": "one packed pinned buffer each way per step; step i+1's inputs copied in and step i's "
                          "results read back on two copy streams while step i computes (device staging buffers)"},
        "gpu_launches": int(graph.launches * steps),
        "gpu_launches_per_step": graph.launches,
        "launch": "one CUDA graph replay per step",
        "eager_ms_per_step": round(eager_ms, 4),
        "breakdown_ms": {n: round(float(v), 4) for (n, _), v in zip(step.calls, per_call)},
        "kernel_classes": class_summary(classes, peaks),
        "roofline": roofline(classes, peaks, config, step.gemm_bytes),
        "clocks": clk,
    }
    del graph
    return out


def side_measurements(ict, torch, peaks, flush, steps, warmup, skip, with_cpu):
    """The other configurations, each with its own value, roofline, e2e and oracle
    baseline (a few steps each)."""
    out = {}
    for name, cls in STEPS.items():
        if name == skip:
            continue
        st = cls(ict, torch, 0)
        k = 100 if name == "resnet50_sgd" else steps
        entry = {"config": dict(cls.workload)}
        entry.update(measure(st, ict, torch, peaks, flush, name, k, warmup))
        entry["steps"] = k
        if with_cpu:
            entry["cpu_baseline"] = safe_cpu_baseline(cls)
        out[name] = entry
        del st
        torch.cuda.empty_cache()
    out["torch_int_mm_8192_tops"] = side_int_mm(torch)
    return out


# --------------------------------------------------------------------- lines


def base_line(args, step_cls, n_gpus):
    cfg = dict(step_cls.workload)
    mode = "dp" if step_cls.data_parallel else "replicas"
    cfg.update(parallelism=f"{mode}{n_gpus}" if n_gpus > 1 else "single",
               l2="flushed between steps (512 MB write)")
    return {
        "metric": METRIC, "unit": step_cls.unit, "n_gpus": n_gpus, "steps": args.steps, "warmup": args.warmup,
        "higher_is_better": step_cls.higher_is_better, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic (seeded; layer shapes of the paper's networks)", "config": cfg,
    }


def cpu_baseline(step_cls):
    import oracle

    dt, units, sample = step_cls.oracle_step(step_cls.sample_arg)
    return {"value": step_cls.value_of(units, dt), "unit": step_cls.unit, "cores": oracle.num_threads(),
            "kind": "oracle", "sample": sample, "seconds": round(dt, 3)}


def safe_cpu_baseline(step_cls):
    try:
        return cpu_baseline(step_cls)
    except Exception as exc:  # pragma: no cover
        return {"value": None, "unit": step_cls.unit, "cores": None, "kind": "oracle", "sample": f"failed: {exc}"}


def run_reference(args):
    """The oracle as it stands, timed on the host cores on a bounded sample of the
    configuration's step (rank 0 only)."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    step_cls = STEPS[args.config]
    runs = [cpu_baseline(step_cls) for _ in range(max(1, min(args.steps, 3)))]
    value = float(np.mean([r["value"] for r in runs]))
    cb = dict(runs[-1], value=value, sample=runs[-1]["sample"] + f", mean of {len(runs)} runs")
    line = base_line(args, step_cls, args.gpus)
    line.update({
        "impl": "reference", "value": value, "cpu_baseline": cb,
        "e2e": {"value": value, "unit": step_cls.unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    })
    print(json.dumps(line))


def main():
    args = parse()
    args.warmup = max(args.warmup, 3)
    if args.steps is None:
        args.steps = 100 if args.config == "resnet50_sgd" else 20
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
    step_cls = STEPS[args.config]
    step = step_cls(ict, torch, rank)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    line = base_line(args, step_cls, world)
    line.update(measure(step, ict, torch, peaks, flush, args.config, args.steps, args.warmup, dist))
    if world > 1 and getattr(step, "exchanged_bytes", 0):
        line["allreduce_bytes_per_rank_per_step"] = int(step.exchanged_bytes)
    del step
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_side:
        line["side"] = side_measurements(ict, torch, peaks, flush, max(5, args.steps // 2), args.warmup,
                                         args.config, not args.no_cpu)
    if rank == 0:
        if not args.no_cpu and world == 1:
            line["cpu_baseline"] = safe_cpu_baseline(step_cls)
        print(json.dumps(line))
    if dist:
        torch.cuda.synchronize()  # every CUDA graph holding NCCL calls is gone by now
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
