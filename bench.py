#!/usr/bin/env python
"""Benchmark of the W4A8 MoE expert FFN on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill] [--impl ours|reference]
                    [--weights asym|sym|clip999] [--group 64|128|256] [--no-cpu-baseline] [--no-extra]

Workloads: dense_gemm, toy_moe, decode, large_decode, prefill (the default: the
largest MoE layer, 384 experts, top-8, 16384 tokens, hidden 7168, expert ffn 2048,
INT8-tensor-bound) and kv_int8 (the INT8 KV cache round trip, reported in GB/s).
--weights selects the packer's scheme (asymmetric INT4, symmetric, or the
percentile range); --group the weights per scale along K (128 by default, or 64 /
256).  Decode-shaped layers with group 128 are also timed with W4A16 experts (the
same packed weights with bf16 activations), reported under "w4a16" with the ratio.  On one GPU the default run also times the two HBM-bound decode
layers (large_decode reusing the packed 384-expert weights, and decode) and reports
each under "extra" with its own step time, roofline and kernel table (--no-extra
skips them).

The INT8 tensor-core peak that tensor-bound kernels are compared with is measured
in the same run, before the timed steps: torch._int_mm (cuBLASLt) on 8192^3 INT8
operands, best of 10, CUDA events, with the SM clock sampled meanwhile.

One step = one forward of the whole hot path (routing when the workload routes
from logits, permutation, INT8 activation quant, up GEMM + SwiGLU, requant, down
GEMM, combine) over one batch of seeded synthetic input already resident in HBM.
L2 is flushed (a 256 MiB write) before every timed step, outside the timed span.
Steps are timed with CUDA events on the launching stream; per-kernel times come
from the library's event profiler over the same timed region.  With N > 1 (one
process per GPU under torchrun) every rank runs an independent replica of the
layer -- the layer has no cross-GPU exchange -- and the slowest rank's time is
reported ("scaling": "weak").  Rank 0 prints one JSON line.

--impl reference times the CPU oracle (numpy, fp64 GEMMs through BLAS) on a
bounded token sample of the same workload, on the host cores.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from w4a8_quantized_moe_token_b200 import synth  # noqa: E402

METRIC = "W4A8 MoE FFN tokens/s, TOPS and weight GB/s on 1 B200; % of HBM / INT8 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}
INT8_OVER_BF16 = 4.5 / 2.25  # nominal dense INT8 / BF16 tensor peak ratio on B200 (used only if the measurement fails)


# --------------------------------------------------------------------------- #
# accounting (algorithmic work; pages' storage format: 0.5 B/weight + 4 B per 128-group)
# --------------------------------------------------------------------------- #
def padded(k):
    return (k + 127) // 128 * 128


def packed_matrix_bytes(N, K):
    """4-bit codes + one fp16 scale and one fp16 zero point per group (the pages'
    storage: 0.5 B per weight + 4 B per group of GROUP weights)."""
    m = max(128, GROUP)
    Kp = (K + m - 1) // m * m
    return N * Kp // 2 + N * (Kp // GROUP) * 4


def moe_accounting(W, ids, w4a16=False):
    """Algorithmic ops and bytes per kernel kind.  w4a16: the comparison layer, whose
    token rows (x and h) are bf16, 2 bytes per value, and which has no requant pass."""
    T, k, H, F = W.T, W.topk, W.H, W.F
    touched = int(np.unique(ids).size)
    slots = T * k
    m = max(128, GROUP)  # token rows are padded to whole groups (and 128-wide planes)
    Hp, Fp = (H + m - 1) // m * m, (F + m - 1) // m * m
    up_w = touched * packed_matrix_bytes(2 * F, H)
    dn_w = touched * packed_matrix_bytes(H, F)
    k_ops = {
        "gemm_up": 2.0 * slots * 2 * F * H,
        "gemm_down": 2.0 * slots * H * F,
    }
    if w4a16:
        k_bytes = {
            "perm": slots * 4 * 3.0,
            "act_quant": T * H * 2.0 + slots * Hp * 2.0,
            "gemm_up": up_w + slots * Hp * 2.0 + slots * F * 2.0,
            "gemm_down": dn_w + slots * Fp * 2.0 + slots * H * 4.0,
            "combine": slots * H * 4.0 + T * H * 2.0 + slots * 8,
            "route": T * W.E * 2.0 + slots * 8,
        }
        return {"touched_experts": touched, "weight_bytes": up_w + dn_w, "ops": k_ops["gemm_up"] + k_ops["gemm_down"],
                "kernel_ops": k_ops, "kernel_bytes": k_bytes}
    k_bytes = {
        "perm": slots * 4 * 3.0,
        "act_quant": T * H * 2.0 + slots * Hp + slots * 4,
        "gemm_up": up_w + slots * Hp + slots * F * 2.0,  # h written as bf16
        "requant": slots * F * 2.0 + slots * Fp,
        "gemm_down": dn_w + slots * Fp + slots * H * 4.0,
        "combine": slots * H * 4.0 + T * H * 2.0 + slots * 8,
        "route": T * W.E * 2.0 + slots * 8,
    }
    return {"touched_experts": touched, "weight_bytes": up_w + dn_w, "ops": k_ops["gemm_up"] + k_ops["gemm_down"],
            "kernel_ops": k_ops, "kernel_bytes": k_bytes}


def gemm_accounting(W):
    M, N, K = W.M, W.N, W.K
    wb = packed_matrix_bytes(N, K)
    return {"touched_experts": 1, "weight_bytes": wb, "ops": 2.0 * M * N * K,
            "kernel_ops": {"gemm_dense": 2.0 * M * N * K},
            "kernel_bytes": {"gemm_dense": wb + M * padded(K) * 2 + M * N * 4.0, "act_quant": M * K * 2.0 + M * K}}


def load_traffic(workload: str, kernel: str):
    """DRAM bytes per launch of `kernel` on `workload` from a committed ncu capture
    (profiles/dram_traffic.json), or None when there is none or when any source file
    the kernel is built from has changed since the counters were taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
            entry = json.load(f).get(workload)
    except (OSError, ValueError):
        return None
    if not entry or entry.get("kernel") != kernel:
        return None
    for rel, digest in entry.get("sources", {}).items():
        try:
            with open(os.path.join(ROOT, rel), "rb") as f:
                if hashlib.sha256(f.read()).hexdigest() != digest:
                    return None
        except OSError:
            return None
    return float(entry["dram_bytes_per_launch"])


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


# --------------------------------------------------------------------------- #
# clocks during the timed region (NVML reads only)
# --------------------------------------------------------------------------- #
class ClockSampler:
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting", 0x1: "gpu_idle"}

    def __init__(self, index, period=0.005):
        self.index, self.period = index, period
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self._stop = threading.Event()
        self._t = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        nv = self._nv
        get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= int(get_r(self._h))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        rs = [n for b, n in self.REASONS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": rs, "samples": len(self.samples)}


# --------------------------------------------------------------------------- #
# setup on the device
# --------------------------------------------------------------------------- #
def dev_bf16(a, device):
    import torch
    return torch.from_numpy(synth.bf16_bits(a).view(np.int16)).view(torch.bfloat16).to(device)


# weight scheme of the packer: asymmetric INT4 (default), symmetric, or asymmetric on the
# 0.1th..99.9th percentile range
SCHEME = "asym"
GROUP = 128  # weights per scale along K (--group)


def weights_desc():
    return {"asym": "int4 g%d asym (fp16 scale+zp)", "sym": "int4 g%d sym (fp16 scale, zero point 8)",
            "clip999": "int4 g%d asym on the 0.1..99.9 percentile range (fp16 scale+zp)"}[SCHEME] % GROUP


def scheme_flag(B):
    return {"asym": 0, "sym": B.W4A8_PACK_SYMMETRIC, "clip999": B.W4A8_PACK_CLIP999}[SCHEME] | B.GROUP_FLAG[GROUP]


def oracle_quant(O):
    if SCHEME == "sym":
        return lambda w: O.quantize_weights_symmetric(w, GROUP)
    return lambda w: O.quantize_weights(w, clip999=SCHEME == "clip999", group=GROUP)


def pack_experts(B, torch, W, seed, device):
    """Pack every expert's up (gate|up) and down weights on the device, one expert at a time."""
    E, H, F = W.E, W.H, W.F
    flag = scheme_flag(B)
    up = B.empty_aligned(B.w4a8_packed_bytes(E, 2 * F, H, B.W4A8_LAYOUT_GATEUP | flag), device)
    dn = B.empty_aligned(B.w4a8_packed_bytes(E, H, F, B.W4A8_LAYOUT_PLAIN | flag), device)
    su = (up.numel() - 256) // E
    sd = (dn.numel() - 256) // E
    tu = B.empty_aligned(B.w4a8_packed_bytes(1, 2 * F, H, 1 | flag), device)
    td = B.empty_aligned(B.w4a8_packed_bytes(1, H, F, 0 | flag), device)
    for which, (buf, tmp, stride, rows, cols, layout) in (("up", (up, tu, su, 2 * F, H, 1)),
                                                           ("down", (dn, td, sd, H, F, 0))):
        for e, w in synth.expert_weights_parallel(seed, E, which, rows, cols):
            B.w4a8_pack_weights(dev_bf16(w, device), layout | flag, tmp)
            buf[256 + e * stride:256 + (e + 1) * stride].copy_(tmp[256:])
    torch.cuda.synchronize(device)
    return up, dn


E2E_STREAMS = 2  # end-to-end steps alternate between this many streams (MoeStep.e2e)


class MoeStep:
    """One forward of the MoE layer through w4a8_moe_forward (or, with w4a16=True,
    through the W4A16 comparison layer w4a16_moe_forward on the same packed weights)."""

    def __init__(self, B, torch, W, seed, device, packed=None, w4a16=False):
        self.B, self.torch, self.W, self.device = B, torch, W, device
        self.w4a16 = w4a16
        inp = synth.moe_inputs(W, seed)
        self.x_host = inp["x"]
        T, E, k, H, F = W.T, W.E, W.topk, W.H, W.F
        self.x = dev_bf16(inp["x"], device)
        self.ids = torch.empty((T, k), dtype=torch.int32, device=device)
        self.w = torch.empty((T, k), dtype=torch.float32, device=device)
        self.logits = None
        if "logits" in inp:
            self.logits = dev_bf16(inp["logits"], device)
            B.w4a8_route_topk(self.logits, k, self.ids, self.w)
            torch.cuda.synchronize(device)
            self.ids_host = self.ids.cpu().numpy()
            self.w_host = self.w.cpu().numpy()
        else:
            self.ids_host, self.w_host = inp["ids"], inp["wts"]
            self.ids.copy_(torch.from_numpy(inp["ids"]))
            self.w.copy_(torch.from_numpy(inp["wts"]))
        self.logits_host = inp.get("logits")
        self.packed_up, self.packed_down = packed if packed is not None else pack_experts(B, torch, W, seed, device)
        self.out = torch.empty((T, H), dtype=torch.bfloat16, device=device)
        if w4a16:
            self.ws = B.empty_aligned(B.w4a16_moe_workspace_bytes(T, E, k, H, F), device)
        else:
            self.ws = B.empty_aligned(B.w4a8_moe_workspace_bytes_g(T, E, k, H, F, GROUP), device)
        self.acct = moe_accounting(W, self.ids_host, w4a16)

    def __call__(self):
        B, W = self.B, self.W
        if self.logits is not None:
            B.w4a8_route_topk(self.logits, W.topk, self.ids, self.w)
        if self.w4a16:
            fwd = B.w4a16_moe_forward
        elif GROUP != 128:
            def fwd(*a):
                B.w4a8_moe_forward_g(*a[:5], GROUP, *a[5:])
        else:
            fwd = B.w4a8_moe_forward
        fwd(self.packed_up, self.packed_down, W.E, W.H, W.F, self.x, self.ids, self.w, self.out,
                           self.ws)

    def e2e(self, steps, warmup):
        """Same metric through the public API with HOST inputs/outputs: per step the
        pinned-host inputs are copied in and the bf16 output copied back.

        Consecutive steps alternate between two streams with their own workspace and
        output buffer (double buffering, as a server overlaps requests): step i + 1's
        input copy and step i - 1's output copy run on the copy engines while step i
        computes.  Every step's copies are inside the timed span, which runs from the
        first step's issue to the completion of the last one on both streams."""
        torch, B, W = self.torch, self.B, self.W
        T, E, k, H, F = W.T, W.E, W.topk, W.H, W.F
        pin = lambda a: torch.from_numpy(a).pin_memory()
        x_h = torch.from_numpy(synth.bf16_bits(self.x_host).view(np.int16)).view(torch.bfloat16).pin_memory()
        ids_h, w_h = pin(np.ascontiguousarray(self.ids_host)), pin(np.ascontiguousarray(self.w_host))
        lanes = []
        for _ in range(2):
            lane = {"stream": torch.cuda.Stream(self.device),
                    "out_h": torch.empty((T, H), dtype=torch.bfloat16).pin_memory()}
            if GROUP != 128:
                # the group-size entry point takes device buffers: the step's copies are
                # issued on the same stream around it
                lane["x"] = torch.empty_like(self.x)
                lane["ids"] = torch.empty_like(self.ids)
                lane["w"] = torch.empty_like(self.w)
                lane["out"] = torch.empty_like(self.out)
                lane["ws"] = B.empty_aligned(B.w4a8_moe_workspace_bytes_g(T, E, k, H, F, GROUP), self.device)
            else:
                lane["ws"] = B.empty_aligned(B.w4a8_moe_host_workspace_bytes(T, E, k, H, F), self.device)
            lanes.append(lane)
        if GROUP != 128:
            h2d = x_h.numel() * 2 + ids_h.numel() * 4 + w_h.numel() * 4

            def run(lane):
                lane["x"].copy_(x_h, non_blocking=True)
                lane["ids"].copy_(ids_h, non_blocking=True)
                lane["w"].copy_(w_h, non_blocking=True)
                B.w4a8_moe_forward_g(self.packed_up, self.packed_down, E, H, F, GROUP, lane["x"], lane["ids"],
                                     lane["w"], lane["out"], lane["ws"])
                lane["out_h"].copy_(lane["out"], non_blocking=True)
        elif self.logits is None:
            h2d = x_h.numel() * 2 + ids_h.numel() * 4 + w_h.numel() * 4

            def run(lane):
                B.w4a8_moe_forward_host(self.packed_up, self.packed_down, E, H, F, x_h, ids_h, w_h, lane["out_h"],
                                        lane["ws"])
        else:
            # routed on the device from the router logits: one C-ABI call with host buffers
            lg_h = torch.from_numpy(synth.bf16_bits(self.logits_host).view(np.int16)).view(torch.bfloat16).pin_memory()
            h2d = x_h.numel() * 2 + lg_h.numel() * 2

            def run(lane):
                B.w4a8_moe_forward_logits_host(self.packed_up, self.packed_down, E, H, F, x_h, lg_h, k,
                                               lane["out_h"], lane["ws"])

        def steps_on_lanes(n):
            main = torch.cuda.current_stream(self.device)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(main)
            for lane in lanes:
                lane["stream"].wait_event(a)
            for i in range(n):
                lane = lanes[i % 2]
                with torch.cuda.stream(lane["stream"]):
                    run(lane)
            for lane in lanes:
                main.wait_stream(lane["stream"])
            b.record(main)
            b.synchronize()
            return a.elapsed_time(b)

        steps_on_lanes(max(warmup, 2))
        torch.cuda.synchronize()
        total = steps_on_lanes(steps)
        return total / steps, h2d, T * H * 2


class GemmStep:
    """Dense W4A8 linear: per-token INT8 of x, then the W4A8 GEMM."""

    def __init__(self, B, torch, W, seed, device):
        self.B, self.torch, self.W, self.device = B, torch, W, device
        x, w = synth.dense_gemm_inputs(seed, W.M, W.K, W.N)
        self.x = dev_bf16(x, device)
        self.packed = B.empty_aligned(B.w4a8_packed_bytes(1, W.N, W.K, scheme_flag(B)), device)
        B.w4a8_pack_weights(dev_bf16(w, device), scheme_flag(B), self.packed)
        Kp = padded(W.K)
        self.q = torch.empty((W.M, Kp), dtype=torch.int8, device=device)
        self.s = torch.empty(W.M, dtype=torch.float32, device=device)
        self.y = torch.empty((W.M, W.N), dtype=torch.float32, device=device)
        self.out = self.y
        self.ws = B.empty_aligned(B.w4a8_gemm_workspace_bytes_g(W.M, W.N, W.K, GROUP), device)
        self.acct = gemm_accounting(W)

    def __call__(self):
        self.B.w4a8_quant_act(self.x, self.q, self.s)
        self.B.w4a8_gemm_g(self.q, self.s, self.packed, self.W.N, self.W.K, GROUP, self.y, self.ws)

    def e2e(self, steps, warmup):
        torch = self.torch
        x_h = self.x.cpu().pin_memory()
        y_h = torch.empty_like(self.y, device="cpu").pin_memory()

        def step():
            self.x.copy_(x_h, non_blocking=True)
            self()
            y_h.copy_(self.y, non_blocking=True)
        for _ in range(warmup):
            step()
        torch.cuda.synchronize()
        total = 0.0
        for _ in range(steps):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            step()
            b.record()
            b.synchronize()
            total += a.elapsed_time(b)
        return total / steps, x_h.numel() * 2, y_h.numel() * 4


# --------------------------------------------------------------------------- #
# CPU oracle timing (the reported CPU baseline and the reference arm)
# --------------------------------------------------------------------------- #
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


class OracleSample:
    """The oracle forward on a bounded token sample of the workload (weights
    quantised once beforehand, untimed -- the GPU step excludes packing too)."""

    def __init__(self, W, seed, target_s, max_experts=16):
        from oracle import w4a8_oracle as O
        self.O, self.W, self.seed = O, W, seed
        self.reps = 1
        if W.kind == "gemm":
            x, w = synth.dense_gemm_inputs(seed, W.M, W.K, W.N)
            self.x, self.qw = x, oracle_quant(O)(w)
            self.tokens = W.M
            self.sample_desc = f"all {W.M} rows"
            return
        inp = synth.moe_inputs(W, seed)
        self.x = inp["x"]
        if "logits" in inp:
            self.logits = inp["logits"]
            self.ids, self.w = O.route_topk(self.logits, W.topk)
        else:
            self.logits = None
            self.ids, self.w = inp["ids"], inp["wts"].astype(np.float64)
        # size the token sample: time a few tokens, scale to the target.  Every expert a
        # sampled token touches must be quantised first (about a second each for the
        # 384-expert layers), so the sample is also capped at max_experts experts; a
        # sample smaller than the target is run `reps` times per timing.
        self.experts = {}
        cap = 1
        while cap < W.T and self._touched(cap + 1) <= max_experts:
            cap += 1
        n = min(cap, 8)
        t = self._time(n)
        per_tok = t / n
        self.tokens = int(max(1, min(cap, target_s / max(per_tok, 1e-6))))
        self._ensure_experts(self.tokens)
        self.reps = int(max(1, round(target_s / max(per_tok * self.tokens, 1e-6))))
        self.sample_desc = (f"{self.tokens} of {W.T} tokens ({self._touched(self.tokens)} experts)"
                            + (f", run {self.reps} times per timing" if self.reps > 1 else ""))

    def _touched(self, n):
        return int(np.unique(self.ids[:n]).size)

    def _ensure_experts(self, n):
        for e in np.unique(self.ids[:n]):
            e = int(e)
            if e not in self.experts:
                W = self.W
                self.experts[e] = self.O.QuantExpert(synth.expert_weight(self.seed, e, "up", 2 * W.F, W.H),
                                                     synth.expert_weight(self.seed, e, "down", W.H, W.F),
                                                     symmetric=SCHEME == "sym", clip999=SCHEME == "clip999",
                                                     group=GROUP)

    def _time(self, n):
        self._ensure_experts(n)
        t0 = time.perf_counter()
        self.run(n)
        return time.perf_counter() - t0

    def run(self, n=None):
        O, W = self.O, self.W
        if W.kind == "gemm":
            qa, sa = O.quantize_act(self.x)
            return O.w4a8_linear(qa, sa, *self.qw)
        n = self.tokens if n is None else n
        self._ensure_experts(n)  # a no-op once the sample's experts are quantised
        if self.logits is not None:
            O.route_topk(self.logits[:n], W.topk)
        return O.moe_forward(self.x[:n], self.ids[:n], self.w[:n], self.experts, W.E, W.F)

    def timed(self):
        """Seconds per forward of the token sample (averaged over self.reps runs)."""
        if self.W.kind != "gemm":
            self._ensure_experts(self.tokens)
        t0 = time.perf_counter()
        for _ in range(self.reps):
            self.run()
        return (time.perf_counter() - t0) / self.reps


# --------------------------------------------------------------------------- #
def max_over_ranks(x: float, torch, device, world: int) -> float:
    """The largest of every rank's x (the job's time is its slowest rank's)."""
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / (max_ms / 1e3)


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def run_reference(args, W):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    if W.kind == "kv":
        target = max(0.5, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
        H, D = W.extra["heads"], W.extra["head_dim"]
        vals = [kv_oracle_sample(W, args.seed, target) for _ in range(args.steps)]
        value = statistics.mean(v[0] for v in vals) * 6 * H * D / 1e9
        line = {"impl": "reference", "metric": KV_METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": statistics.mean(v[2] for v in vals) * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": kv_config(W),
                "cpu_baseline": {"value": value, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
                                 "sample": vals[0][1]},
                "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0
    target = max(0.5, min(10.0, 100.0 / max(1, args.steps + args.warmup)))
    S = OracleSample(W, args.seed, target)
    for _ in range(args.warmup):
        S.run()
    t = sum(S.timed() for _ in range(args.steps)) / args.steps
    tokens = S.tokens
    value = tokens / t
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(W, "none"),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": S.sample_desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(W, l2):
    if W.kind == "gemm":
        c = {"workload": W.name, "M": W.M, "K": W.K, "N": W.N}
    else:
        c = {"workload": W.name, "T": W.T, "E": W.E, "topk": W.topk, "H": W.H, "F": W.F, "routing": W.routing}
    c.update({"weights": weights_desc(), "acts": "int8 per-token", "l2": l2,
              "parallelism": "replicas (no cross-GPU exchange)"})
    return c


KV_METRIC = "INT8 KV cache (static per-head scales): quantise + dequantise, GB/s on 1 B200; % of HBM roofline"


def kv_config(W):
    x = W.extra
    return {"workload": W.name, "T": W.T, "heads": x["heads"], "head_dim": x["head_dim"],
            "calib_tokens": x["calib_tokens"], "kv": "bf16 -> int8 (per-head static scale) -> bf16",
            "l2": "flushed before every timed step (256 MiB write, outside the timed span)",
            "parallelism": "replicas (no cross-GPU exchange)"}


def kv_oracle_sample(W, seed, target_s):
    """The oracle's quantise + dequantise on a bounded token sample (tokens/s, sample text)."""
    from oracle import w4a8_oracle as O
    H, D = W.extra["heads"], W.extra["head_dim"]
    calib = synth.kv_cache(seed, min(W.T, W.extra["calib_tokens"]), H, D)
    s = O.kv_calibrate(calib)
    n = min(W.T, 256)
    x = synth.kv_cache(seed, n, H, D)
    t0 = time.perf_counter()
    O.kv_dequantize(O.kv_quantize(x, s), s)
    per_tok = (time.perf_counter() - t0) / n
    n = int(max(1, min(W.T, target_s / max(per_tok, 1e-9))))
    x = synth.kv_cache(seed, n, H, D)
    t0 = time.perf_counter()
    O.kv_dequantize(O.kv_quantize(x, s), s)
    t = time.perf_counter() - t0
    return n / t, f"{n} of {W.T} tokens", t


def run_kv(args, W, torch, B, device, world, rank):
    """Time the INT8 KV cache round trip (w4a8_kv_quant + w4a8_kv_dequant of the whole
    cache) per step; the calibration is offline (static scales), done once before."""
    H, D, T = W.extra["heads"], W.extra["head_dim"], W.T
    x_h = synth.kv_cache(args.seed, T, H, D)
    calib = dev_bf16(x_h[:W.extra["calib_tokens"]], device)
    x = dev_bf16(x_h, device)
    scale = torch.empty(H, dtype=torch.float32, device=device)
    q = torch.empty((T, H, D), dtype=torch.int8, device=device)
    y = torch.empty((T, H, D), dtype=torch.bfloat16, device=device)
    B.w4a8_kv_calibrate(calib, scale)

    def step():
        B.w4a8_kv_quant(x, scale, q)
        B.w4a8_kv_dequant(q, scale, y)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    sampler = ClockSampler(torch.cuda.current_device())
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record()
        B.w4a8_kv_quant(x, scale, q)
        ev[i][1].record()
        B.w4a8_kv_dequant(q, scale, y)
        ev[i][2].record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    sampler.stop()
    qms = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    dms = sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps
    ms = max_over_ranks(qms + dms, torch, device, world)
    n = T * H * D
    qbytes, dbytes = 3 * n, 3 * n  # bf16 in + int8 out; int8 in + bf16 out
    # end to end: host cache in, round trip, host cache out
    xh = torch.from_numpy(synth.bf16_bits(x_h).view(np.int16)).view(torch.bfloat16).pin_memory()
    yh = torch.empty((T, H, D), dtype=torch.bfloat16).pin_memory()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(args.warmup):
        x.copy_(xh, non_blocking=True)
        step()
        yh.copy_(y, non_blocking=True)
    torch.cuda.synchronize()
    a.record()
    for _ in range(args.steps):
        x.copy_(xh, non_blocking=True)
        step()
        yh.copy_(y, non_blocking=True)
    b.record()
    torch.cuda.synchronize()
    e2e_ms = a.elapsed_time(b) / args.steps
    peaks = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    dom, dom_ms, dom_b = ("kv_dequant", dms, dbytes) if dms >= qms else ("kv_quant", qms, qbytes)
    roof = {"bound": "hbm", "achieved": dom_b / (dom_ms / 1e3) / 1e9, "peak": hbm, "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / hbm
    roof["traffic"] = load_traffic(W.name, dom)
    roof["kernel"] = dom
    roof["peak_source"] = f"{peaks['source']}: MEASURED_PEAKS hbm_gbs"
    total_bytes = (qbytes + dbytes) * world
    line = {
        "metric": KV_METRIC, "value": whole_job_rate(qbytes + dbytes, world, ms) / 1e9, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic", "config": kv_config(W),
        "tokens_per_s": T * world / (ms / 1e3),
        "roofline": roof,
        "kernels": {"kv_quant": {"launches": args.steps, "ms_per_step": qms, "gbs": qbytes / (qms / 1e3) / 1e9},
                    "kv_dequant": {"launches": args.steps, "ms_per_step": dms, "gbs": dbytes / (dms / 1e3) / 1e9}},
        "gpu_launches": 2 * args.steps,
        "e2e": {"value": total_bytes / (e2e_ms / 1e3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": 2 * n,
                "d2h_bytes_per_step": 2 * n},
        "clocks": sampler.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tps, desc, _ = kv_oracle_sample(W, args.seed, args.cpu_baseline_seconds)
        line["cpu_baseline"] = {"value": tps * 6 * H * D / 1e9, "unit": "GB/s", "cores": blas_threads(),
                                "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


def measure_int8_peak(torch, device, n=8192, reps=10):
    """Dense INT8 tensor-core throughput of a library GEMM on this GPU: torch._int_mm
    (cuBLASLt, int8 x int8 -> int32) on n^3 operands, best of `reps` CUDA-event timed
    calls after warm-up, with the SM clock sampled meanwhile.  TOPS = 2 n^3 / time."""
    info = {"method": f"torch._int_mm int8 {n}^3 (cuBLASLt), best of {reps}, CUDA events"}
    try:
        a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=device)
        b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=device).t()  # column-major operand
        for _ in range(3):
            torch._int_mm(a, b)
        torch.cuda.synchronize()
        sampler = ClockSampler(torch.cuda.current_device(), period=0.002)
        sampler.start()
        best = float("inf")
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._int_mm(a, b)
            e1.record()
            e1.synchronize()
            best = min(best, e0.elapsed_time(e1))
        sampler.stop()
        del a, b
        info.update({"tops": 2.0 * n ** 3 / (best / 1e3) / 1e12, "ms": best, "clocks": sampler.summary()})
    except Exception as ex:  # recorded, and the nominal ratio is used instead
        info.update({"tops": None, "error": f"{type(ex).__name__}: {ex}"[:200]})
    return info


def capture_step(step, torch, device):
    """The step as one CUDA graph (every launch of the forward replayed without host
    gaps, as a serving loop runs it), if it captures and its replay reproduces the
    eager output bit for bit; else the eager step.  Returns (callable, note)."""
    out = getattr(step, "out", None)
    if out is None:
        return step, "eager (no output to verify)"
    try:
        side = torch.cuda.Stream(device)
        side.wait_stream(torch.cuda.current_stream(device))
        with torch.cuda.stream(side):
            step()
        torch.cuda.current_stream(device).wait_stream(side)
        torch.cuda.synchronize(device)
        ref = out.clone()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        out.zero_()
        g.replay()
        torch.cuda.synchronize(device)
        if not torch.equal(out, ref):
            return step, "eager (graph replay differed from the eager step)"
        step.graph = g  # keep it alive
        return g.replay, "cuda graph"
    except Exception as e:  # noqa: BLE001 -- any capture failure falls back to eager launches
        torch.cuda.synchronize(device)
        return step, f"eager (capture failed: {type(e).__name__})"


def time_steps(step, B, torch, device, world, steps, warmup):
    """Warm up, then time `steps` steps with CUDA events on the launching stream (L2
    flushed before each, outside the timed span) and NVML clock samples over the same
    region; then run the same number of steps again under the library's per-kernel
    event profiler (its events between kernels would break the overlap of one kernel's
    start with the previous one's end, so the headline steps run without it).
    Returns (max-over-ranks ms per step, {kernel kind: (launches, total ms)}, clock
    summary)."""
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    run, step.graph_note = capture_step(step, torch, device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    sampler = ClockSampler(torch.cuda.current_device())
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    sampler.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    for i in range(steps):
        flush.zero_()
        starts[i].record()
        run()
        ends[i].record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    sampler.stop()
    ms = sum(a.elapsed_time(b) for a, b in zip(starts, ends)) / steps
    # the per-kernel table
    B.w4a8_profile_start()
    for _ in range(steps):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    prof = B.w4a8_profile_stop()
    assert B.w4a8_last_device_error(step.ws) == 0, "device error during the timed steps"
    return max_over_ranks(ms, torch, device, world), prof, sampler.summary()


def kernel_table(prof, acct, steps):
    kernels = {}
    for kind, (n, tot) in prof.items():
        if n:
            kernels[kind] = {"launches": n, "ms_per_step": tot / steps}
    for kind, v in kernels.items():
        kb = acct["kernel_bytes"].get(kind, 0.0)
        ko = acct["kernel_ops"].get(kind, 0.0)
        t = v["ms_per_step"] * steps / v["launches"] / 1e3
        v["gbs"] = kb / t / 1e9 if t > 0 else None
        if ko:
            v["tops"] = ko / t / 1e12 if t > 0 else None
    return kernels


def roofline_of(kernel, kernels, acct, steps, peaks, workload):
    """Roofline of one kernel: algorithmic ops (tensor-bound) or bytes (HBM-bound) per
    launch over its average event-timed launch duration, against the measured peak."""
    hbm, i8 = peaks["hbm_gbs"], peaks["int8_tops"]
    per_launch_ms = kernels[kernel]["ms_per_step"] * steps / kernels[kernel]["launches"]
    ops = acct["kernel_ops"].get(kernel, 0.0)
    byt = acct["kernel_bytes"].get(kernel, 0.0)
    ridge = i8 * 1e12 / (hbm * 1e9)
    if ops and ops / max(byt, 1) > ridge:
        roof = {"bound": "tensor", "achieved": ops / (per_launch_ms / 1e3) / 1e12, "peak": i8, "unit": "TFLOP/s",
                "peak_source": peaks["int8_source"]}
    else:
        roof = {"bound": "hbm", "achieved": byt / (per_launch_ms / 1e3) / 1e9, "peak": hbm, "unit": "GB/s",
                "peak_source": f"{peaks['source']}: MEASURED_PEAKS hbm_gbs (copy bandwidth)"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = load_traffic(workload, kernel)
    roof["kernel"] = kernel
    roof["ms_per_launch"] = per_launch_ms
    return roof


def moe_summary(W, step, ms, prof, clocks, steps, peaks, world):
    acct = step.acct
    kernels = kernel_table(prof, acct, steps)
    dom = max((k for k in kernels if k.startswith("gemm")), key=lambda k: kernels[k]["ms_per_step"])
    tokens = (W.T if W.kind == "moe" else W.M) * world
    sec = ms / 1e3
    return {
        "value": whole_job_rate(tokens // world, world, ms), "unit": "tokens/s", "ms_per_step": ms,
        "tops": acct["ops"] * world / sec / 1e12,
        "weight_gbs": acct["weight_bytes"] * world / sec / 1e9,
        "touched_experts": acct["touched_experts"],
        "roofline": roofline_of(dom, kernels, acct, steps, peaks, W.name),
        "rooflines": {k: roofline_of(k, kernels, acct, steps, peaks, W.name)
                      for k in kernels if k.startswith("gemm") and k != dom},
        "kernels": kernels,
        "gpu_launches": sum(v["launches"] for v in kernels.values()),
        "clocks": clocks,
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(synth.WORKLOADS), default="prefill")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-baseline-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="do not also time the decode layers")
    ap.add_argument("--group", type=int, choices=[64, 128, 256], default=128,
                    help="weights per scale and zero point along K (the default 128, or 64 / 256)")
    ap.add_argument("--weights", choices=["asym", "sym", "clip999"], default="asym",
                    help="packer scheme: asymmetric INT4 (default), symmetric, or asymmetric on the "
                         "0.1th..99.9th percentile range")
    args = ap.parse_args(argv)
    global SCHEME, GROUP
    SCHEME = args.weights
    GROUP = args.group
    if GROUP != 128 and SCHEME == "clip999":
        ap.error("the percentile range is defined for groups of 128")
    W = synth.WORKLOADS[args.workload]
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.impl == "reference":
        return run_reference(args, W)

    import torch
    from w4a8_quantized_moe_token_b200 import binding as B

    world, rank, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)

    if W.kind == "kv":
        return run_kv(args, W, torch, B, device, world, rank)

    peaks = load_peaks()
    i8 = measure_int8_peak(torch, device)
    if i8.get("tops"):
        peaks["int8_tops"] = i8["tops"]
        peaks["int8_source"] = "measured in this run: " + i8["method"]
    else:
        peaks["int8_tops"] = float(peaks["bf16_tflops"]) * INT8_OVER_BF16
        peaks["int8_source"] = "bf16_tflops x 2 (nominal int8/bf16 ratio; the measurement failed)"
    peaks["hbm_gbs"] = float(peaks["hbm_gbs"])

    step = (GemmStep if W.kind == "gemm" else MoeStep)(B, torch, W, args.seed, device)
    ms_max, prof, clocks = time_steps(step, B, torch, device, world, args.steps, args.warmup)
    summ = moe_summary(W, step, ms_max, prof, clocks, args.steps, peaks, world)

    e2e_ms, h2d, d2h = step.e2e(args.steps, args.warmup)
    e2e_ms = max_over_ranks(e2e_ms, torch, device, world)
    tokens = (W.T if W.kind == "moe" else W.M) * world

    line = {
        "metric": METRIC,
        "value": summ["value"],
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_max,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8",
        "data": "synthetic",
        "config": dict(config_of(W, "flushed before every timed step (256 MiB write, outside the timed span)"),
                       launch=step.graph_note),
        "tops": summ["tops"],
        "weight_gbs": summ["weight_gbs"],
        "touched_experts": summ["touched_experts"],
        "roofline": summ["roofline"],
        "rooflines": summ["rooflines"],
        "kernels": summ["kernels"],
        "gpu_launches": summ["gpu_launches"],
        "e2e": {"value": whole_job_rate(tokens // world, world, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "streams": E2E_STREAMS},
        "clocks": summ["clocks"],
        "int8_peak": i8,
    }

    # decode-shaped layers: the pages' comparison point, the same layer with W4A16
    # experts (bf16 activations, same packed weights and routing)
    if W.kind == "moe" and W.name != "prefill" and GROUP == 128:
        s16 = MoeStep(B, torch, W, args.seed, device, packed=(step.packed_up, step.packed_down), w4a16=True)
        ms16, prof16, cl16 = time_steps(s16, B, torch, device, world, args.steps, args.warmup)
        w16 = moe_summary(W, s16, ms16, prof16, cl16, args.steps, peaks, world)
        line["w4a16"] = {k: w16[k] for k in ("value", "unit", "ms_per_step", "weight_gbs", "roofline", "kernels",
                                             "gpu_launches", "clocks")}
        line["w4a16"]["launch"] = s16.graph_note
        line["w4a8_over_w4a16"] = summ["value"] / w16["value"]
        del s16

    # the HBM-bound decode layers, timed in the same run (one GPU only)
    if world == 1 and not args.no_extra and W.name == "prefill":
        extra = {}
        shared = (step.packed_up, step.packed_down)
        for name in ("large_decode", "decode"):
            Wx = synth.WORKLOADS[name]
            same = (Wx.E, Wx.H, Wx.F) == (W.E, W.H, W.F)
            sx = MoeStep(B, torch, Wx, args.seed, device, packed=shared if same else None)
            msx, profx, clx = time_steps(sx, B, torch, device, world, args.steps, args.warmup)
            ex = moe_summary(Wx, sx, msx, profx, clx, args.steps, peaks, world)
            e2x, h2x, d2x = sx.e2e(args.steps, args.warmup)
            ex["e2e"] = {"value": Wx.T / (e2x / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2x,
                         "d2h_bytes_per_step": d2x, "ms_per_step": e2x, "streams": E2E_STREAMS}
            ex["config"] = dict(config_of(Wx, "flushed before every timed step (256 MiB write, outside the timed span)"),
                                launch=sx.graph_note)
            # the pages' comparison point: the same layer with W4A16 experts (bf16
            # activations, same packed weights and routing; group 128 only)
            if GROUP != 128:
                extra[name] = ex
                del sx
                torch.cuda.empty_cache()
                continue
            s16 = MoeStep(B, torch, Wx, args.seed, device, packed=(sx.packed_up, sx.packed_down), w4a16=True)
            ms16, prof16, cl16 = time_steps(s16, B, torch, device, world, args.steps, args.warmup)
            w16 = moe_summary(Wx, s16, ms16, prof16, cl16, args.steps, peaks, world)
            ex["w4a16"] = {k: w16[k] for k in ("value", "unit", "ms_per_step", "weight_gbs", "roofline", "kernels",
                                               "gpu_launches", "clocks")}
            ex["w4a16"]["launch"] = s16.graph_note
            ex["w4a8_over_w4a16"] = ex["value"] / w16["value"]
            extra[name] = ex
            del sx, s16
            torch.cuda.empty_cache()
        line["extra"] = extra

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        S = OracleSample(W, args.seed, args.cpu_baseline_seconds)
        t = S.timed()
        line["cpu_baseline"] = {"value": S.tokens / t, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                                "sample": S.sample_desc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
