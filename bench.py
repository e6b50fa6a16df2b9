"""Benchmark of the W4A8 Linear / MoE-expert path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode|prefill|moe_sym|moe_asym_decode|moe_asym_prefill]
                    [--m M] [--main-only] [--no-cpu-baseline]

One "step" is one pass of the hot path over one batch of synthetic input,
through the public call a user makes:
  decode / prefill:  w4a8_linear (per-token INT8 quantization of X, then the
                     W4A8 GEMM launched to overlap it);
  moe_*:             w4a8_moe_grouped_gemm (route, dispatch + quantize,
                     grouped gate_up with SiLU*up, quantize h, grouped down,
                     combine).
The default workload is the decode-shaped linear (M=32, K=4096, N=14336,
symmetric int4 group 128, 8 outlier channels x50), whose metric is the
weight bytes streamed per second; its figures form the contract line, and
the metric's other parts (prefill TOPS, MoE tokens/s for the three MoE
configurations) follow in a "workloads" object with the same figures each.

Timing: W untimed warm-up steps, then exactly K steps, bracketed by a
barrier + synchronize, timed with CUDA events on the launching stream (max
over ranks).  The timed steps are uninstrumented CUDA-graph replays of the
public call; packed weights are rotated over enough copies that every decode
step reads them from HBM, not L2 (the other workloads' operands exceed L2).
The dominant kernel's per-launch time comes from separate, untimed
instrumented replays (events around a chain of GEMM launches, or at the MoE
layer's stage boundaries).  SM clocks and throttle reasons are sampled
through NVML during the timed region.

`e2e` repeats the metric through the public API call a user makes, with the
step's input copied host->device from pinned memory and the result read back
device->host inside the timed region.

`--impl reference` times the CPU oracle (test infrastructure, the only
reference this path has) on a bounded sample of the same workload.
Multi-GPU (torchrun): every rank runs an independent replica of the workload
(the path has no exchange step); value = all ranks' work / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "W4A8 GEMM TOPS (prefill) & weight GB/s (decode) vs B200 roofline; MoE tokens/s"
L2_BYTES = 126 * 1024 * 1024

DEFAULT_STEPS = {"decode": 20000, "prefill": 1500, "moe_sym": 2000, "moe_asym_decode": 400,
                 "moe_asym_prefill": 200, "w8a8_decode": 20000, "w8a8_prefill": 1500,
                 "w4a16_decode": 20000, "w4a16_prefill": 1500, "moe_asym_prefill_e32": 400}


# ---------------------------------------------------------------- peaks ---

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sus=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), source="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


# --------------------------------------------------------------- clocks ---

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index: int):
        self.ok = False
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            pass
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()
            if not self.samples:  # region shorter than one period: take one sample now
                try:
                    self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                    self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
                except Exception:
                    pass

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"], "samples": 0}
        names = [n for b, n in self.REASONS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# ------------------------------------------------------------ workloads ---

class LinearWorkload:
    """Per-token INT8 quant + W4A8 GEMM on a [M, K] x [K, N] linear."""

    def __init__(self, name, M, K=4096, N=14336, group=128, device="cuda"):
        self.name, self.M, self.K, self.N, self.group = name, M, K, N, group
        self.dev = device
        self.decode = name.endswith("decode")
        self.w8 = name.startswith("w8a8")  # per-channel INT8 weights (the W8A8 variant)
        self.w16 = name.startswith("w4a16")  # bf16 activations, weights dequantized in the GEMM

    def setup(self):
        import torch
        import moe_linear_layers_w4a8_b200 as m
        from synth import gen_linear
        self.m = m
        M, K, N, g = self.M, self.K, self.N, self.group
        inp = gen_linear(M, K, N, seed=0, n_outliers=8, outlier_scale=50.0)
        self.X_host = inp.X
        if self.w8:
            pw = m.w8a8_pack_weights(inp.W.to(self.dev))
            self.w_bytes = N * K + N * 4
        else:
            pw = m.w4a8_pack_weights(inp.W.to(self.dev), g, True)
            self.w_bytes = N * K // 2 + (K // g) * N * 4
        # enough weight copies that the weights of consecutive steps are not in L2
        self.copies = [pw]
        if self.decode:
            n = max(2, math.ceil(2 * L2_BYTES / self.w_bytes) + 1)
            for _ in range(n - 1):
                if self.w8:
                    self.copies.append(m.PackedW8(pw.q_w.clone(), pw.s_w.clone(), pw.desc.copy()))
                else:
                    self.copies.append(m.PackedWeight(pw.packed.clone(), pw.s_w.clone(), None, pw.desc.copy()))
        self.X = inp.X.to(self.dev)
        self.q = torch.empty(M, K, dtype=torch.int8, device=self.dev)
        self.s = torch.empty(M, dtype=torch.float32, device=self.dev)
        self.Y = torch.empty(M, N, dtype=torch.bfloat16, device=self.dev)
        if self.w8:
            ws = m.w8a8_gemm_workspace_size(M, pw)
            lws = m.w8a8_linear_workspace_size(M, pw)
            self._linear, self._gemm = m.w8a8_linear, m.w8a8_gemm
        elif self.w16:
            ws = lws = m.w4a16_gemm_workspace_size(M, pw)
            self._linear = m.w4a16_gemm
            self._gemm = lambda q, s, w, out, workspace: m.w4a16_gemm(self.X, w, out=out, workspace=workspace)
        else:
            ws = m.w4a8_gemm_workspace_size(M, pw)
            lws = m.w4a8_linear_workspace_size(M, pw)
            self._linear, self._gemm = m.w4a8_linear, m.w4a8_gemm
        self.ws = torch.empty(max(ws, 16), dtype=torch.uint8, device=self.dev)
        self.lws = torch.empty(max(lws, 16), dtype=torch.uint8, device=self.dev)
        self.splitk = ws > 0
        # quantization + GEMM (split-K is summed inside the GEMM); W4A16 has no quantization
        self.launches_per_step = 1 if self.w16 else 2

    def step(self, i, ev=None):
        # the public one-call layer: the GEMM's weight streaming overlaps the quantization
        self._linear(self.X, self.copies[i % len(self.copies)], out=self.Y, workspace=self.lws)

    @property
    def kernel_timing_note(self):
        return (f"CUDA events around a graph of {self._chain} back-to-back "
                f"{'w8a8_gemm' if self.w8 else 'w4a16_gemm' if self.w16 else 'w4a8_gemm'} launches "
                f"(packed weights rotated{'' if self.w16 else ', activations quantized once'}), mean per launch")

    def kernel_time(self, torch):
        """Per-launch duration of the GEMM: events around a chain of
        back-to-back launches in a CUDA graph (separate, untimed replays)."""
        m = self.m
        if not self.w16:
            m.w4a8_quant_act(self.X, q_out=self.q, s_out=self.s)
        n = self._chain = 64 if self.decode else 8

        def chain(i, ev):
            if ev:
                ev[0].record()
            for j in range(n):
                w = self.copies[(i * n + j) % len(self.copies)]
                self._gemm(self.q, self.s, w, out=self.Y, workspace=self.ws)
            if ev:
                ev[1].record()
        g, evs = capture(torch, chain, 3, with_events=2)
        times = []
        for _ in range(2):
            g.replay()
            torch.cuda.synchronize()
            times += [e[0].elapsed_time(e[1]) / n for e in evs]
        del g
        return statistics.mean(times), None

    def release(self):
        for a in ("copies", "X", "q", "s", "Y", "ws", "lws", "X_dev2", "Y_pin", "X_pin", "Y2", "lws2"):
            if hasattr(self, a):
                delattr(self, a)

    # metric
    def units(self):
        if self.decode:
            return self.w_bytes / 1e9, "GB/s", "weight+scale bytes streamed per second"
        if self.w16:
            return 2.0 * self.M * self.N * self.K / 1e12, "TFLOPS", "2*M*N*K bf16 flops per second"
        return 2.0 * self.M * self.N * self.K / 1e12, "TOPS", "2*M*N*K int8 ops per second"

    def kernel_roofline(self, peaks):
        M, K, N, g = self.M, self.K, self.N, self.group
        kname = ("w8a8_gemm_kernel" if self.w8 else "w4a16_gemm_kernel" if self.w16 else
                 "w4a8_gemm_tc_kernel")
        if self.decode:
            # weights + scales, activations (int8 + s_x, or bf16), bf16 output
            alg = self.w_bytes + (2 * M * K if self.w16 else M * K + 4 * M) + 2 * M * N
            return dict(bound="hbm", per_launch=alg, unit="GB/s", scale=1e9, peak=peaks["hbm"],
                        peak_note=f"hbm_gbs ({peaks['source']})", kernel_name=kname)
        ops = 2.0 * M * N * K
        if self.w16:
            return dict(bound="tensor", per_launch=ops, unit="TFLOP/s", scale=1e12, peak=peaks["bf16_sus"],
                        peak_note=f"bf16_tflops_sustained ({peaks['source']})", kernel_name=kname)
        return dict(bound="tensor", per_launch=ops, unit="TOPS", scale=1e12, peak=2.0 * peaks["bf16_sus"],
                    peak_note=f"2 x bf16_tflops_sustained ({peaks['source']}; int8/bf16 nominal ratio 2)",
                    kernel_name=kname)

    def config(self):
        wfmt = ("per-channel int8 weights (W8A8)" if self.w8 else
                f"symmetric int4 g={self.group}, bf16 activations (W4A16)" if self.w16 else
                f"symmetric int4 g={self.group}")
        base = {"workload": f"{self.name} linear M={self.M} K={self.K} N={self.N} {wfmt}",
                "M": self.M, "K": self.K, "N": self.N, "group": self.K if self.w8 else self.group}
        if not hasattr(self, "copies"):
            return base
        return dict(base, **{
                "l2": (f"{len(self.copies)} packed-weight copies rotated "
                       f"({len(self.copies) * self.w_bytes / 2**20:.0f} MiB > 2x L2)" if self.decode else
                       "per-step activations+output "
                       f"{(self.M * self.K * 3 + 2 * self.M * self.N) / 2**20:.0f} MiB > L2"),
                "schedule": "split-K" if self.splitk else "data-parallel tiles"})

    def e2e_setup(self):
        import torch
        self.X_pin = self.X_host.pin_memory()
        # two steps in flight (one per stream), each with its own buffers
        self.Y_pin = [torch.empty(self.M, self.N, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        self.X_dev2 = [torch.empty_like(self.X) for _ in range(2)]
        self.Y2 = [torch.empty_like(self.Y) for _ in range(2)]
        self.lws2 = [torch.empty_like(self.lws) for _ in range(2)]
        return self.X_pin.numel() * 2, self.Y_pin[0].numel() * 2

    def e2e_step(self, i):
        b = i % 2
        self.X_dev2[b].copy_(self.X_pin, non_blocking=True)
        Y = self._linear(self.X_dev2[b], self.copies[i % len(self.copies)], out=self.Y2[b], workspace=self.lws2[b])
        self.Y_pin[b].copy_(Y, non_blocking=True)

    # CPU oracle on a bounded sample of the same workload
    def oracle_step_setup(self, n_cols):
        import numpy as np
        import oracle as O
        import torch
        W = self._W_host()
        cols = np.sort(np.random.default_rng(0).choice(self.N, n_cols, replace=False))
        Xb = self.X_host.view(torch.int16).numpy().view(np.uint16)
        if self.w8:
            qw, sw, _ = O.quant_w8(W[:, cols].copy())  # offline step, untimed
            self._orc = (O, qw, sw, Xb)
        elif self.w16:
            codes, s, _, _ = O.quant_weights(W[:, cols].copy(), self.group, True)  # offline step, untimed
            self._orc = (O, codes, s, Xb)
        else:
            codes, s, _, _ = O.quant_weights(W[:, cols].copy(), self.group, True)  # offline step, untimed
            self._orc = (O, codes, s, Xb)
        return n_cols / self.N

    def _W_host(self):
        from synth import gen_linear
        return gen_linear(self.M, self.K, self.N, seed=0, n_outliers=8, outlier_scale=50.0).W.numpy()

    def oracle_step(self):
        O, codes, s, Xb = self._orc
        if self.w8:
            qx, sx, _, _ = O.quant_act(Xb)
            O.w8a8_exact(qx, sx, codes, s)
        elif self.w16:
            O.w4a16_gemm(Xb, O.w4a16_dequant(codes, s, None, self.group))
        else:
            O.linear(Xb, codes, s, None, self.group)


class MoEWorkload:
    """One MoE expert layer."""

    def __init__(self, name, device="cuda"):
        from synth import CONFIGS
        c = CONFIGS[name]
        self.name = name
        self.T, self.H, self.E, self.topk, self.I = c["T"], c["H"], c["E"], c["topk"], c["I"]
        self.group, self.sym, self.zipf, self.wp = c["group"], c["symmetric"], c["zipf"], c["w_outlier_p"]
        self.dev = device
        # route, dispatch (one kernel, or count / scan / scatter above 256 tokens), quantize X,
        # gate_up, quantize h, down, combine
        self.launches_per_step = 7 + (2 if self.T > 256 else 0)

    def _weight(self, e, which, device):
        from synth import gen_expert_weight
        K, N = (self.H, 2 * self.I) if which == 0 else (self.I, self.H)
        return gen_expert_weight(0, e, which, K, N, outlier_p=self.wp, device=device)

    def setup(self):
        import torch
        import moe_linear_layers_w4a8_b200 as m
        from synth import gen_moe_activations
        self.m = m
        inp = gen_moe_activations(self.T, self.H, self.E, seed=0, zipf=self.zipf)
        self.X_host, self.L_host = inp.X, inp.logits
        self.X, self.L = inp.X.to(self.dev), inp.logits.to(self.dev)
        self.w1 = m.w4a8_pack_expert_weights(lambda e: self._weight(e, 0, self.dev), self.E, self.H, 2 * self.I,
                                             self.group, self.sym, self.dev)
        self.w2 = m.w4a8_pack_expert_weights(lambda e: self._weight(e, 1, self.dev), self.E, self.I, self.H,
                                             self.group, self.sym, self.dev)
        ws = m.w4a8_moe_workspace_size(self.T, self.E, self.topk, self.w1, self.w2)
        self.ws = torch.empty(ws, dtype=torch.uint8, device=self.dev)
        self.out = torch.empty(self.T, self.H, dtype=torch.bfloat16, device=self.dev)
        # Expert hit count, for the bytes of the weight-streaming roofline.
        r = m.w4a8_moe_grouped_gemm(self.X, self.L, self.topk, self.w1, self.w2, workspace=self.ws, out=self.out)
        offs = r["expert_offsets"].cpu()
        self.hit = int(((offs[1:] - offs[:-1]) > 0).sum())
        self.counts = (offs[1:] - offs[:-1]).tolist()

    STAGES = ["route", "dispatch", "quant_x", "gate_up", "quant_h", "down", "combine"]

    def step(self, i, ev=None):
        self.m.w4a8_moe_grouped_gemm(self.X, self.L, self.topk, self.w1, self.w2, workspace=self.ws, out=self.out,
                                     stage_events=ev)

    kernel_timing_note = ("CUDA events at the layer's stage boundaries (w4a8_moe_grouped_gemm_profiled) in a "
                          "separate, untimed graph replay of 4 layer steps; mean per stage")

    def kernel_time(self, torch):
        g, evs = capture(torch, self.step, 4, with_events=8)
        g.replay()
        torch.cuda.synchronize()
        stage_ms = {name: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs)
                    for i, name in enumerate(self.STAGES)}
        del g
        return stage_ms["gate_up"], stage_ms

    def release(self):
        for a in ("w1", "w2", "ws", "out", "X", "L", "X2", "L2", "out_pin", "X_pin", "L_pin", "out2", "ws2"):
            if hasattr(self, a):
                delattr(self, a)

    def units(self):
        return self.T / 1e6, "Mtokens/s", "tokens per second through the whole layer"

    def kernel_roofline(self, peaks):
        H, I, g, R = self.H, self.I, self.group, self.T * self.topk
        zb = 0 if self.sym else 1
        # the gate_up GEMM is the largest launch of the layer
        w1_expert = H * 2 * I // 2 + (H // g) * 2 * I * (4 + zb)
        act = R * H + 4 * R + R * I * 2  # q_x rows in, h rows out
        ops = 2.0 * R * H * 2 * I
        if self.name == "moe_asym_decode":
            return dict(bound="hbm", per_launch=self.hit * w1_expert + act, unit="GB/s", scale=1e9,
                        peak=peaks["hbm"], kernel="gate_up", kernel_name="w4a8_gemm_tc_kernel (gate_up)",
                        peak_note=f"hbm_gbs ({peaks['source']}); gate_up launch bytes = experts hit ({self.hit}) "
                                  f"x (packed gate_up weights + scales + zero-points) + activations in/out")
        return dict(bound="tensor", per_launch=ops, unit="TOPS", scale=1e12, peak=2.0 * peaks["bf16_sus"],
                    kernel="gate_up", kernel_name="w4a8_gemm_tc_kernel (gate_up)",
                    peak_note=f"2 x bf16_tflops_sustained ({peaks['source']}); gate_up launch ops = 2*pairs*H*2I")

    def config(self):
        return {"workload": (f"{self.name}: T={self.T} H={self.H} E={self.E} top-{self.topk} I={self.I} "
                             f"{'symmetric' if self.sym else 'asymmetric+zero-point'} int4 g={self.group}"
                             + (f", Zipf({self.zipf}) logits" if self.zipf else "")),
                "T": self.T, "H": self.H, "E": self.E, "topk": self.topk, "I": self.I, "group": self.group,
                "experts_hit": getattr(self, "hit", None),
                "l2": f"expert weights {self.E * (3 * self.H * self.I) / 2 / 2**20:.0f} MiB vs L2 126 MiB"}

    def e2e_setup(self):
        import torch
        self.X_pin = self.X_host.pin_memory()
        self.L_pin = self.L_host.pin_memory()
        # two steps in flight (one per stream), each with its own buffers
        self.out_pin = [torch.empty(self.T, self.H, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        self.X2 = [torch.empty_like(self.X) for _ in range(2)]
        self.L2 = [torch.empty_like(self.L) for _ in range(2)]
        self.out2 = [torch.empty_like(self.out) for _ in range(2)]
        self.ws2 = [torch.empty_like(self.ws) for _ in range(2)]
        return self.X_pin.numel() * 2 + self.L_pin.numel() * 4, self.out_pin[0].numel() * 2

    def e2e_step(self, i):
        b = i % 2
        self.X2[b].copy_(self.X_pin, non_blocking=True)
        self.L2[b].copy_(self.L_pin, non_blocking=True)
        r = self.m.w4a8_moe_grouped_gemm(self.X2[b], self.L2[b], self.topk, self.w1, self.w2, workspace=self.ws2[b],
                                         out=self.out2[b])
        self.out_pin[b].copy_(r["out"], non_blocking=True)

    def oracle_step_setup(self, n_tokens):
        import numpy as np
        import oracle as O
        import torch
        rng = np.random.default_rng(0)
        toks = np.sort(rng.choice(self.T, n_tokens, replace=False))
        Xb = self.X_host.view(torch.int16).numpy().view(np.uint16)[toks]
        L = self.L_host.numpy()[toks]
        idx, _, _ = O.route(L, self.topk)
        need = sorted(set(int(e) for e in idx.ravel()))
        codes1, codes2 = {}, {}
        for e in need:  # weight quantization is offline: prepared here, untimed
            codes1[e] = O.quant_weights(self._weight(e, 0, "cpu").numpy(), self.group, self.sym)[:3]
            codes2[e] = O.quant_weights(self._weight(e, 1, "cpu").numpy(), self.group, self.sym)[:3]
            if self.sym:
                codes1[e] = (codes1[e][0], codes1[e][1], None)
                codes2[e] = (codes2[e][0], codes2[e][1], None)
        self._orc = (O, Xb, L, codes1, codes2)
        return n_tokens / self.T

    def oracle_step(self):
        O, Xb, L, c1, c2 = self._orc
        idx, p, _ = O.route(L, self.topk)
        ex1 = [c1.get(e, (None, None, None)) for e in range(self.E)]
        ex2 = [c2.get(e, (None, None, None)) for e in range(self.E)]
        O.moe_forward(Xb, L, self.topk, ex1, ex2, self.group)


def make_workload(name, M):
    if name in ("decode", "prefill", "w8a8_decode", "w8a8_prefill", "w4a16_decode", "w4a16_prefill"):
        return LinearWorkload(name, M if M else (32 if name.endswith("decode") else 8192))
    return MoEWorkload(name)


# ------------------------------------------------------------- timing ---

def capture(torch, fn, n, with_events=0):
    """Captures n steps (fn(i, ev)) into one CUDA graph; with_events = number
    of timing events per step handed to fn (recorded as graph nodes)."""
    evs = [tuple(torch.cuda.Event(enable_timing=True, external=True) for _ in range(with_events))
           for _ in range(n)] if with_events else [None] * n
    for ev in evs:  # torch creates the CUDA event on its first record
        for e in ev or ():
            e.record()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn(0, None)  # one eager call on the capture stream (library state, attributes)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            for i in range(n):
                fn(i, evs[i])
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    return g, evs


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier_sync(torch, world):
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()


def max_over_ranks(torch, world, v, device="cuda"):
    """The slowest rank's time: every rank gets the max (one all-reduce)."""
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(unit_scale, steps, world, t_ms):
    """Whole-job rate: the units all ranks processed over the slowest rank's time."""
    return unit_scale * steps * world / (t_ms / 1e3)


def upload_graph(torch, g):
    """Uploads an instantiated CUDA graph to the device ahead of its first
    replay (otherwise the first replay carries the upload); best effort."""
    try:
        from cuda.bindings import runtime as rt
        rt.cudaGraphUpload(g.raw_cuda_graph_exec(), torch.cuda.current_stream().cuda_stream)
        torch.cuda.synchronize()
    except Exception:
        pass


def timed_product_steps(torch, wl, K, W, world, local):
    """W untimed warm-up steps, then exactly K steps of the public call
    (uninstrumented CUDA-graph replays of `wl.step`), bracketed by a barrier +
    synchronize and timed with CUDA events on the launching stream; returns
    (max-over-ranks ms, clock summary)."""
    Lg = max(1, min(K, 64 if wl.name == "decode" else 8))
    reps, rem = divmod(K, Lg)
    gw, _ = capture(torch, wl.step, max(W, 1))
    gt, _ = capture(torch, wl.step, Lg)
    grem = capture(torch, wl.step, rem)[0] if rem else None
    for g in (gt, grem):
        if g is not None:
            upload_graph(torch, g)
    gw.replay()
    barrier_sync(torch, world)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    with sampler:
        # An untimed ~50 us device spin ahead of the start event: the host
        # enqueues the event and the graph launches meanwhile, so the timed
        # region holds device work only, not the host's launch latency.
        torch.cuda._sleep(100_000)
        start.record()
        for _ in range(reps):
            gt.replay()
        if grem is not None:
            grem.replay()
        end.record()
        torch.cuda.synchronize()
    barrier_sync(torch, world)
    t_ms = max_over_ranks(torch, world, start.elapsed_time(end))
    del gw, gt, grem
    torch.cuda.synchronize()
    return t_ms, sampler.summary()


def measure(args, wl, K, W, peaks, world, rank, local, cpu_budget_s):
    """Every figure of one workload: product-path throughput over K timed
    steps, the dominant kernel against its roofline (from separate,
    untimed instrumented replays), end to end from host buffers, and the
    oracle on a bounded sample."""
    import torch
    wl.setup()
    unit_scale, unit, meaning = wl.units()
    roof = wl.kernel_roofline(peaks)
    t_ms, clocks = timed_product_steps(torch, wl, K, W, world, local)
    value = job_throughput(unit_scale, K, world, t_ms)

    k_ms, stage_ms = wl.kernel_time(torch)
    achieved = roof["per_launch"] / roof["scale"] / (k_ms / 1e3)
    roofline = {"bound": roof["bound"], "achieved": round(achieved, 2), "peak": round(roof["peak"], 1),
                "unit": roof["unit"], "frac": round(achieved / roof["peak"], 4),
                "traffic": traffic_from_profiles(wl.name, roof), "kernel_ms": round(k_ms, 5),
                "kernel": roof.get("kernel_name", "w4a8_gemm_tc_kernel"), "timing": wl.kernel_timing_note,
                "peak_source": roof["peak_note"], "algorithmic_per_launch": roof["per_launch"],
                "frac_note": "of measured" if peaks["source"] == "measured" else "of fallback"}
    if stage_ms is not None:
        roofline["stage_ms"] = {k: round(v, 5) for k, v in stage_ms.items()}

    # end to end through the public API with host buffers: every step copies
    # its input from pinned host memory and its result back; consecutive steps
    # alternate between two streams (own buffers and workspace each), so one
    # step's copies overlap the other's kernels, as a serving loop would run them
    h2d, d2h = wl.e2e_setup()
    Ke = max(1, min(K, 2000 if wl.name == "decode" else max(10, K // 4)))
    main = torch.cuda.current_stream()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]

    def run_e2e(first, n):
        for i in range(first, first + n):
            with torch.cuda.stream(streams[i % 2]):
                wl.e2e_step(i)

    for st in streams:
        st.wait_stream(main)
    run_e2e(0, min(W, 20))
    for st in streams:
        main.wait_stream(st)
    torch.cuda.synchronize()
    barrier_sync(torch, world)
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(main)
    for st in streams:
        st.wait_stream(main)
    run_e2e(0, Ke)
    for st in streams:
        main.wait_stream(st)
    e2.record(main)
    torch.cuda.synchronize()
    te = max_over_ranks(torch, world, s2.elapsed_time(e2))
    e2e_value = job_throughput(unit_scale, Ke, world, te)

    out = {
        "value": round(value, 3), "unit": unit, "steps": K, "warmup": W, "ms_per_step": round(t_ms / K, 6),
        "config": dict(wl.config(), quantity=meaning, parallelism=f"replicas x{world}",
                       global_batch=(getattr(wl, "M", None) or getattr(wl, "T", None)) * world),
        "roofline": roofline,
        "e2e": {"value": round(e2e_value, 3), "unit": unit, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": Ke},
        "gpu_launches": wl.launches_per_step * K,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(wl, unit_scale, unit, budget_s=cpu_budget_s)
    wl.release()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


SECONDARY = ["prefill", "moe_sym", "moe_asym_decode", "moe_asym_prefill", "w8a8_decode", "w8a8_prefill",
             "w4a16_decode", "w4a16_prefill"]


def run_ours(args, world, rank, local):
    import torch
    import moe_linear_layers_w4a8_b200 as m
    m.load_library()  # fails loudly without the CUDA library
    peaks = measured_peaks()
    K, W = args.steps, args.warmup
    main = measure(args, make_workload(args.workload, args.m), K, W, peaks, world, rank, local, 10.0)
    line = {"metric": METRIC, "value": main["value"], "unit": main["unit"], "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": main["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8", "data": "synthetic"}
    line.update({k: v for k, v in main.items() if k not in ("value", "unit", "steps", "warmup", "ms_per_step")})
    if args.workload == "decode" and args.m is None and not args.main_only:
        # the metric's other parts, each with its own figures, on the same box
        line["workloads"] = {}
        for name in SECONDARY:
            Kw = min(K, DEFAULT_STEPS[name])
            line["workloads"][name] = measure(args, make_workload(name, None), Kw, W, peaks, world, rank, local,
                                              3.0)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def kernel_sources_sha256():
    """Digest of the kernel sources; a stored ncu traffic figure is only used
    while the sources it was measured on are unchanged."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "moe_linear_layers_w4a8_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh")):
            h.update(name.encode())
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(f.read())
    return h.hexdigest()


def traffic_from_profiles(workload, roof):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary profiles/traffic.txt, or None when it was taken on other sources."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        with open(path) as f:
            lines = f.read().splitlines()
    except OSError:
        return None
    sha, table = None, {}
    for ln in lines:
        if ln.startswith("# sources-sha256:"):
            sha = ln.split(":", 1)[1].strip()
        elif ln and not ln.startswith("#"):
            parts = ln.split()
            if len(parts) >= 2:
                table[parts[0]] = int(parts[1])
    if sha != kernel_sources_sha256():
        return None
    return table.get(workload)


def cpu_baseline(wl, unit_scale, unit, budget_s=12.0):
    """The oracle, as it stands, on a bounded sample of the same workload."""
    import oracle as O
    O.build()
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    frac, sample = _oracle_sample(wl)
    t0 = time.perf_counter()
    wl.oracle_step()
    one = time.perf_counter() - t0
    reps = max(1, min(50, int(budget_s / max(one, 1e-6))))
    t0 = time.perf_counter()
    for _ in range(reps):
        wl.oracle_step()
    dt = (time.perf_counter() - t0) / reps
    return {"value": round(unit_scale * frac / dt, 6), "unit": unit, "cores": cores, "kind": "oracle",
            "sample": f"{sample}; {reps} repetitions, {dt * 1e3:.1f} ms each"}


def _oracle_sample(wl):
    if isinstance(wl, LinearWorkload):
        n = (1024 if wl.w8 else wl.N) if wl.decode else 256
        frac = wl.oracle_step_setup(n) if wl.decode else _linear_row_sample(wl, 4 if wl.w8 else 16)
        return frac, (f"{n} of {wl.N} output columns of the M={wl.M} decode step (weight quantization untimed)"
                      if wl.decode else f"{4 if wl.w8 else 16} of {wl.M} rows x all {wl.N} columns")
    n = min(wl.T, 2 if wl.E >= 256 else (8 if wl.T > 64 else 4))
    return wl.oracle_step_setup(n), f"{n} of {wl.T} tokens through the whole layer"


def _linear_row_sample(wl, rows):
    import numpy as np
    import oracle as O
    import torch
    W = wl._W_host()
    Xb = wl.X_host.view(torch.int16).numpy().view(np.uint16)[:rows].copy()
    if getattr(wl, "w8", False):
        qw, sw, _ = O.quant_w8(W)

        def step():
            qx, sx, _, _ = O.quant_act(Xb)
            O.w8a8_exact(qx, sx, qw, sw)
        wl.oracle_step = step
        return rows / wl.M
    codes, s, _, _ = O.quant_weights(W, wl.group, True)

    def step():
        O.linear(Xb, codes, s, None, wl.group)
    wl.oracle_step = step
    return rows / wl.M


def run_reference(args, world, rank):
    """Reference arm: the CPU oracle on the machine's host cores (rank 0 only)."""
    if rank != 0:
        return
    import oracle as O
    O.build()
    wl = make_workload(args.workload, args.m)
    # host-side copies of the inputs only (no GPU work on this arm)
    if isinstance(wl, LinearWorkload):
        from synth import gen_linear
        inp = gen_linear(wl.M, wl.K, wl.N, seed=0, n_outliers=8, outlier_scale=50.0)
        wl.X_host = inp.X
        wl.w_bytes = wl.N * wl.K // 2 + (wl.K // wl.group) * wl.N * 4
    else:
        from synth import gen_moe_activations
        inp = gen_moe_activations(wl.T, wl.H, wl.E, seed=0, zipf=wl.zipf)
        wl.X_host, wl.L_host = inp.X, inp.logits
    unit_scale, unit, meaning = wl.units()
    K, W = args.steps, args.warmup
    # size the per-step sample so that all K + W steps take about a minute
    budget = 60.0
    if isinstance(wl, LinearWorkload):
        n_full = wl.N if wl.decode else wl.M
        probe = max(64, n_full // 64)
        if wl.decode:
            wl.oracle_step_setup(probe)
        else:
            _linear_row_sample(wl, 1)
        t0 = time.perf_counter(); wl.oracle_step(); t_probe = time.perf_counter() - t0
        per_step = budget / (K + W)
        n = int(max(1, min(n_full, probe * per_step / max(t_probe, 1e-9))))
        if wl.decode:
            frac = wl.oracle_step_setup(max(64, n) if n >= 64 else max(1, n))
            sample = f"{max(64, n) if n >= 64 else max(1, n)} of {wl.N} output columns, all {wl.M} rows"
        else:
            frac = _linear_row_sample(wl, max(1, min(n, 64)))
            sample = f"{max(1, min(n, 64))} of {wl.M} rows x all {wl.N} columns"
    else:
        frac = wl.oracle_step_setup(1)
        sample = f"1 of {wl.T} tokens through the whole layer"
    for _ in range(W):
        wl.oracle_step()
    t0 = time.perf_counter()
    for _ in range(K):
        wl.oracle_step()
    dt = time.perf_counter() - t0
    value = unit_scale * frac * K / dt
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": unit, "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": round(dt / K * 1e3, 6), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": dict(wl.config(), quantity=meaning),
        "cpu_baseline": {"value": round(value, 6), "unit": unit, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode",
                    choices=["decode", "prefill", "moe_sym", "moe_asym_decode", "moe_asym_prefill", "w8a8_decode",
                             "w8a8_prefill", "w4a16_decode", "w4a16_prefill", "moe_asym_prefill_e32"])
    ap.add_argument("--m", type=int, default=None, help="rows of the linear workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--main-only", action="store_true",
                    help="measure only the main workload (no 'workloads' object)")
    args = ap.parse_args(argv)
    if args.steps is None:
        args.steps = DEFAULT_STEPS[args.workload]
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    world, rank, local = dist_setup(args)
    run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
