#!/usr/bin/env python
"""Throughput of the latent mixture-of-experts FFN block on B200.

One step = one pass of the whole block (router, bucketing, D_g, experts,
U_g + shared + combine) over one batch of T tokens of one layer.  The default
line is the Edge0-145B-shaped layer at T=4 (an MTP verify window); it carries
a nested "prefill" object with the same layer at T=4096 (the metric's other
half: its own steps, roofline against the tensor peak, clocks and e2e).

Timing: W untimed warm-up steps, then K steps between CUDA events on the
launching stream, barrier + synchronize on both sides, max over ranks.  Each
step runs on one of R device copies of the layer's weights (R x the bytes a
step touches > 2 x the 126 MB L2), so no step finds its weights in L2, and on
its own seeded token batch.  Multi-GPU: every rank is an independent replica
(the block shards by tokens and needs no collective): weak scaling.

`--impl reference` times the C++ fp64 CPU oracle (OpenMP) on the host cores
instead, on the same workload: each step is the whole T-token batch, or one
token of it when K + W whole batches would not finish within a few minutes."""
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

METRIC = "latent-MoE layer tokens/s (T=4 decode, T=4096 prefill); % HBM/FP4 roofline"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="edge0_145b_decode")
    ap.add_argument("--prefill-workload", default="edge0_145b_prefill",
                    help="workload of the nested prefill object ('none' to skip)")
    ap.add_argument("--T", type=int, default=None, help="override the workload's token count")
    ap.add_argument("--copies", type=int, default=0, help="weight copies to rotate (0: enough to defeat L2)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU-oracle sample budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true", help="skip the MTP verify-window sweep")
    ap.add_argument("--no-w4a4", action="store_true", help="skip the W4A4 prefill object")
    ap.add_argument("--act-fmt", choices=["fp16", "nvfp4"], default=None,
                    help="expert input format of the workload (nvfp4: W4A4); default: the workload's own")
    return ap.parse_args()


# ----------------------------------------------------------------------------
# clocks during the timed region (NVML, read only)
# ----------------------------------------------------------------------------

class ClockSampler:
    REASONS = {0x0000000000000002: "applications_clocks_setting", 0x0000000000000004: "sw_power_cap",
               0x0000000000000008: "hw_slowdown", 0x0000000000000020: "sw_thermal_slowdown",
               0x0000000000000040: "hw_thermal_slowdown", 0x0000000000000080: "hw_power_brake_slowdown",
               0x0000000000000100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.001):
        self.period = period_s
        self.samples = []
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that
            self.err = str(e)
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"error": getattr(self, "err", "nvml unavailable")}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        reasons = set()
        for _, rs in self.samples:
            for bit, name in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------------------
# algorithmic bytes of one step (from the routing actually taken)
# ----------------------------------------------------------------------------

def step_cost(shape, idx: np.ndarray, groups: np.ndarray, T: int, prefill: bool) -> dict:
    """Algorithmic bytes (few-token path) or FLOPs (tensor-core path) of each
    kernel for one step, from the routing actually taken: the weights a kernel
    must read at least once plus its activations in and out, or 2 x the
    multiply-adds of the contraction it performs for the routed pairs only."""
    H, L, E, K, G, F, Fs = (shape.hidden, shape.latent, shape.n_experts, shape.top_k, shape.n_groups, shape.ffn,
                            shape.shared_ffn)
    du = L * H // 32 * (34 if shape.du_fmt == 8 else 18)
    rec_gu = 2 * (F * L // 2 + F * L // 16)
    rec_d = F * L // 2 + F * L // 16
    rw = E * H * (2 if shape.router_dtype == "bf16" else 4)
    hit = {int(groups[e]) for e in idx.reshape(-1)}
    distinct = set(idx.reshape(-1).tolist())
    pairs_tg = sum(len({int(groups[e]) for e in idx[t]}) for t in range(idx.shape[0]))   # hit (token, group) pairs
    b = {
        "k_router_shared": rw + 2 * Fs * H * 2 + T * H * 2,
        "k_wstream_dproj": G * du + T * H * 2,     # every group (D runs before the routing is known)
        "k_wstream_gateup": len(distinct) * rec_gu,
        "k_wstream_down": len(distinct) * rec_d,
        "k_wstream_uproj": len(hit) * du + H * Fs * 2 + 2 * T * H * 2,
    }
    # the step's algorithmic bytes count only the hit groups' D
    b_total = float(sum(b.values()) - (G - len(hit)) * du)
    # the 9-63-token kernels read the same bytes per pass of 8 tokens
    for a, c in (("k_dproj_mma", "k_wstream_dproj"), ("k_gateup_mma", "k_wstream_gateup"),
                 ("k_down_mma", "k_wstream_down"), ("k_uproj_mma", "k_wstream_uproj"),
                 ("k_nvf4_gateup", "k_wstream_gateup"), ("k_nvf4_down", "k_wstream_down")):
        b[a] = b[c]
    f = {
        "x_to_fp16": 0.0,
        "router_gemm": 2.0 * T * E * H,
        "topk_bucket": 0.0,
        "shared_gateup": 2.0 * T * 2 * Fs * H,
        "dproj": 2.0 * pairs_tg * L * H,
        "gateup": 2.0 * T * K * 2 * F * L,
        "down": 2.0 * T * K * L * F,
        "combine": 0.0,
        "uproj": 2.0 * pairs_tg * H * L + 2.0 * T * H * Fs,
    }
    weight_bytes = rw + 3 * Fs * H * 2 + len(hit) * 2 * du + len(distinct) * (rec_gu + rec_d)
    out = dict(f if prefill else b)
    out["bytes_total"] = weight_bytes + 2 * T * H * 2 if prefill else b_total
    out["flops_total"] = float(sum(f.values()))
    out["n_distinct"] = len(distinct)
    out["n_groups_hit"] = len(hit)
    return out


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of a
# kernel, from one ncu capture of the kernels built from the CUDA sources
# whose hash is given (cold caches, one launch), by (workload, T, kernel).
# When the sources have changed since the capture, or the kernel has no
# capture, its traffic is reported as null.  (An edit of comments alone is
# re-keyed to the new hash by hand: the kernels it builds are unchanged.)
NCU_TRAFFIC = {
    ("edge0_145b_decode", 4, "k_router_shared"): (9282560, "1539dfd80fde"),
    ("edge0_145b_decode", 4, "k_wstream_dproj"): (39071232, "1539dfd80fde"),
    ("edge0_145b_decode", 4, "k_wstream_gateup"): (42739200, "1539dfd80fde"),
    ("edge0_145b_decode", 4, "k_wstream_down"): (21391872, "1539dfd80fde"),
    ("edge0_145b_decode", 4, "k_wstream_uproj"): (43962112, "1539dfd80fde"),
    ("edge0_145b_prefill", 4096, "gateup"): (849870250, "1539dfd80fde"),
    ("edge0_145b_prefill", 4096, "down"): (502723157, "1539dfd80fde"),
    ("edge0_145b_prefill", 4096, "dproj"): (158917376, "1539dfd80fde"),
    ("edge0_145b_prefill", 4096, "uproj"): (255054677, "1539dfd80fde"),
    ("edge0_145b_prefill+w4a4", 4096, "uproj"): (254834346, "1539dfd80fde"),
    ("edge0_145b_prefill+w4a4", 4096, "dproj"): (159186773, "1539dfd80fde"),
    ("edge0_145b_prefill+w4a4", 4096, "gateup"): (743077802, "1539dfd80fde"),
    ("edge0_145b_prefill+w4a4", 4096, "down"): (464764416, "1539dfd80fde"),
}


def cuda_source_hash() -> str:
    """First 12 hex digits of the SHA-256 of the CUDA sources and headers."""
    import glob
    import hashlib
    h = hashlib.sha256()
    pkg = os.path.join(ROOT, "latent_mixture_experts_softmax_b200", "csrc")
    for f in sorted(glob.glob(os.path.join(pkg, "*.cu*")) + [os.path.join(ROOT, "include", "lmoe.h")]):
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode())
            h.update(fh.read())
    return h.hexdigest()[:12]


def ncu_traffic(wl, T: int, kernel: str):
    """DRAM bytes per launch of `kernel` from the table above (keyed by the
    workload name, "+w4a4" for NVFP4 expert inputs), if taken of the current
    sources."""
    name = wl.name + ("+w4a4" if getattr(wl.shape, "act_fmt", "fp16") == "nvfp4" else "")
    e = NCU_TRAFFIC.get((name, T, kernel))
    if e is None or e[1] != cuda_source_hash():
        return None
    return e[0]


def tensor_core_experts(shape, T: int) -> bool:
    """Whether the library runs the few-token NVFP4 expert phases on the
    tensor cores (kind::mxf4nvf4): LMOE_FEW_TOKEN_EXPERTS=tensor_cores, at
    most 8 tokens, ffn and latent multiples of 128 up to 2048 (the rule
    stated in include/lmoe.h)."""
    L, F = shape.latent, shape.ffn
    return (shape.expert_fmt == "nvfp4" and 1 <= T <= 8 and L % 128 == 0 and F % 128 == 0 and L <= 2048
            and F <= 2048 and os.environ.get("LMOE_FEW_TOKEN_EXPERTS") == "tensor_cores")


def decode_stages(T: int, shape=None):
    """Kernels of one few-token step: the router kernel and four
    weight-streaming kernels up to 8 tokens (NVFP4 gate/up and down on the
    tensor cores where they can), the passes-of-8 kernels from 9 to 63."""
    if T <= 8:
        if shape is not None and tensor_core_experts(shape, T):
            return ["k_router_shared", "k_wstream_dproj", "k_nvf4_gateup", "k_nvf4_down", "k_wstream_uproj"]
        return ["k_router_shared", "k_wstream_dproj", "k_wstream_gateup", "k_wstream_down", "k_wstream_uproj"]
    return ["k_router_shared", "k_dproj_mma", "k_gateup_mma", "k_down_mma", "k_uproj_mma"]


PREFILL_STAGES = ["x_to_fp16", "router_gemm", "topk_bucket", "shared_gateup", "dproj", "gateup", "down", "combine",
                  "uproj"]


def workload_desc(wl, T):
    s = wl.shape
    fmt = "Q8_0" if s.du_fmt == 8 else "Q4_0"
    bias = "none" if wl.bias_sigma is None else f"N(0,{wl.bias_sigma:g})"
    return (f"{wl.name}: T={T}, hidden {s.hidden}, latent {s.latent}, {s.n_experts} experts top-{s.top_k}, "
            f"{s.n_groups} {fmt} D/U groups, NVFP4 experts ffn {s.ffn}, bf16 shared ffn {s.shared_ffn}, "
            f"{s.router_dtype} router, bias {bias}, expert_group {wl.groups}, x bf16 N(0,1), weights N(0,0.02)"
            + (", NVFP4 expert inputs (W4A4)" if getattr(s, "act_fmt", "fp16") == "nvfp4" else ""))


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
        return float(peaks["hbm_gbs"]), float(peaks["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# ----------------------------------------------------------------------------
# multi-GPU: independent replicas, max over ranks
# ----------------------------------------------------------------------------

def max_over_ranks(ms: float, device=None) -> float:
    """The slowest rank's time (every rank calls this in the same order)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(world: int, tokens_per_step: int, steps: int, ms_max: float) -> float:
    """Whole-job tokens/s: every rank processes its own batches (weak scaling)."""
    return world * tokens_per_step * steps / (ms_max / 1e3)


# ----------------------------------------------------------------------------
# the C++ oracle as a CPU baseline / reference arm
# ----------------------------------------------------------------------------

def cpu_oracle_run(wl, layer, T, budget_s=None, max_steps=None, tokens_per_step=None, draw0=10_000):
    """Runs the C++ fp64 oracle on successive seeded token batches of the
    workload (tokens_per_step of each T-token batch, default all) until the
    budget or max_steps is used.  Returns (tokens/s, tokens, seconds,
    threads, steps)."""
    from oracle import native
    from latent_mixture_experts_softmax_b200 import synth
    ntok = tokens_per_step or T
    done = steps = 0
    el = 0.0
    while True:
        xb = synth.make_x(wl, T=T, draw=draw0 + steps)[:ntok]
        t0 = time.perf_counter()
        native.latent_moe_forward(wl.shape, layer, xb)
        el += time.perf_counter() - t0
        done += ntok
        steps += 1
        if (max_steps is not None and steps >= max_steps) or (max_steps is None and el >= budget_s):
            break
    return done / el, done, el, native.threads(), steps


def cpu_baseline(wl, layer, T, budget_s, sample_tokens=None):
    rate, done, el, threads, steps = cpu_oracle_run(wl, layer, T, budget_s=budget_s, tokens_per_step=sample_tokens)
    what = f"{sample_tokens} of each T={T} batch" if sample_tokens else f"whole T={T} batches"
    return {"value": rate, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"C++ fp64 oracle, {threads} OpenMP threads: {steps} seeded batches, {what} ({done} tokens, "
                      f"{el:.1f} s), decoding the stored weights on every call"}


def run_reference(args, wl, T, rank, world):
    """The reference arm: the C++ oracle timed on the host cores (rank 0 only)."""
    if rank != 0:
        return
    from latent_mixture_experts_softmax_b200 import synth
    layer = synth.make_layer(wl)
    # one whole batch first, to size the per-step sample within a few minutes
    _, _, t_one, _, _ = cpu_oracle_run(wl, layer, T, max_steps=1, draw0=9_999)
    ntok = T if (args.steps + args.warmup) * t_one <= 150.0 else 1
    cpu_oracle_run(wl, layer, T, max_steps=args.warmup, tokens_per_step=ntok, draw0=20_000)
    rate, done, el, threads, steps = cpu_oracle_run(wl, layer, T, max_steps=args.steps, tokens_per_step=ntok)
    what = f"the whole T={T} batch" if ntok == T else f"1 token of each T={T} batch (whole batches: {t_one:.2f} s each)"
    line = {"impl": "reference", "metric": METRIC, "value": rate, "unit": "tokens/s", "n_gpus": world,
            "steps": steps, "warmup": args.warmup, "ms_per_step": 1000 * el / steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(wl, T), "T": T},
            "cpu_baseline": {"value": rate, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": f"C++ fp64 oracle, {threads} OpenMP threads; each step {what}, fresh seeded "
                                       f"x per step, weights decoded from their stored bytes on every call"},
            "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# the 48-layer stack
# ----------------------------------------------------------------------------

def run_stack(args, wl, T, rank, world, local, dev_name, n_distinct=4):
    """x <- x + block_l(RMSNorm_l(x)) over wl.n_layers layers in one call.
    n_distinct independently seeded layers are generated and copied into
    n_layers separate device buffers (layer l holds the bytes of layer
    l % n_distinct): the time depends on the bytes each layer streams and on
    its routing, which the changing residual stream drives."""
    import numpy as np
    import torch
    from latent_mixture_experts_softmax_b200 import binding as B
    from latent_mixture_experts_softmax_b200 import synth
    from latent_mixture_experts_softmax_b200.layer import DeviceLayer, to_device
    s = wl.shape
    gamma = synth.bf16_bits_from_f32(np.ones(s.hidden, np.float32))
    srcs = [synth.make_layer(wl, layer=l) for l in range(min(n_distinct, wl.n_layers))]
    devs = [DeviceLayer(s, srcs[l % len(srcs)], device=dev_name, gamma=gamma) for l in range(wl.n_layers)]
    layers = [d.as_c_layer() for d in devs]
    ws = devs[0].workspace(T)
    K, W = args.steps, args.warmup
    n_in = 8
    xs_host = [synth.make_x(wl, T=T, draw=rank * 100_003 + i) for i in range(n_in)]
    xs = [to_device(x, dev_name) for x in xs_host]
    ys = [torch.empty_like(x) for x in xs]
    eps = 1e-6

    def step(i):
        B.lmoe_stack_forward(devs[0].cfg, layers, xs[i % n_in], ys[i % n_in], T, eps, ws)

    for i in range(max(W, 1)):
        step(i)
    torch.cuda.synchronize()
    graphs = []
    if T <= 64:
        for g in range(n_in):
            cg = torch.cuda.CUDAGraph()
            with torch.cuda.graph(cg):
                step(g)
            graphs.append(cg)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start.record()
        for k in range(K):
            if graphs:
                graphs[k % n_in].replay()
            else:
                step(k)
        end.record()
        torch.cuda.synchronize()
    ms_max = max_over_ranks(start.elapsed_time(end), dev_name)
    status = B.lmoe_last_device_status(ws)
    del graphs
    # bytes per layer from the routing each layer actually takes (one untimed pass)
    idx = torch.empty((T, s.top_k), dtype=torch.int32, device=dev_name)
    wgt = torch.empty((T, s.top_k), dtype=torch.float32, device=dev_name)
    cur = xs[0].clone()
    nxt = torch.empty_like(cur)
    prefill = T >= 64 and s.router_dtype == "bf16" and s.n_experts % 128 == 0
    tot_b = tot_f = 0.0
    for l, d in enumerate(devs):
        B.lmoe_stack_forward(d.cfg, [layers[l]], cur, nxt, T, eps, ws)
        # routing of this layer's normalised input, through the block call on it
        xn = cur.view(torch.bfloat16).float()
        xn = (xn * torch.rsqrt((xn * xn).mean(dim=1, keepdim=True) + eps)).to(torch.bfloat16).view(torch.int16)
        B.lmoe_route(d.cfg, xn.contiguous(), d.router_w, d.router_b, T, idx, wgt, ws)
        c = step_cost(s, idx.cpu().numpy(), srcs[l % len(srcs)]["expert_group"], T, prefill)
        tot_b += c["bytes_total"]
        tot_f += c["flops_total"]
        cur, nxt = nxt, cur
    hbm_peak, tc_peak, src = load_peaks()
    t_step = ms_max / K / 1e3
    t_lb = max(tot_b / (hbm_peak * 1e9), tot_f / (tc_peak * 1e12))
    value = replica_throughput(world, T, K, ms_max)
    line = {"metric": "latent-MoE 48-layer stack tokens/s", "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": K, "warmup": W, "ms_per_step": ms_max / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "config": {"workload": workload_desc(wl, T), "T": T, "layers": wl.n_layers,
                       "weights": f"{len(srcs)} seeded layers copied into {wl.n_layers} device buffers",
                       "l2": f"{wl.n_layers} layers x {devs[0].weight_bytes() / 1e9:.2f} GB resident, larger than L2"},
            "layer_equivalent": {"gbs": tot_b / t_step / 1e9, "tflops": tot_f / t_step / 1e12,
                                 "roofline_time_us": t_lb * 1e6, "frac_of_roofline": t_lb / t_step,
                                 "peak_source": src},
            "clocks": clk.summary(), "device_status": status}
    if rank == 0:
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# our arm: one layer
# ----------------------------------------------------------------------------

def weight_copies(base, R):
    """R device copies of a layer's weights (copy 0 is `base`)."""
    from latent_mixture_experts_softmax_b200 import binding as B
    from latent_mixture_experts_softmax_b200.layer import DeviceLayer
    devs = [base]
    for _ in range(R - 1):
        d = DeviceLayer.__new__(DeviceLayer)
        d.__dict__.update(base.__dict__)
        for name in ("router_w", "router_b", "expert_group", "D", "U", "experts", "shared_gate", "shared_up",
                     "shared_down"):
            t = getattr(base, name)
            setattr(d, name, None if t is None else t.clone())
        d.shared = B.make_shared(d.shared_gate, d.shared_up, d.shared_down)
        devs.append(d)
    return devs


class LayerCtx:
    """One layer's weights on the device in R copies, rotated between steps so
    that R - 1 steps of at least T_min tokens touch more than twice the L2
    before a copy is reused."""

    def __init__(self, args, wl, T_min, dev_name):
        from latent_mixture_experts_softmax_b200 import binding as B
        from latent_mixture_experts_softmax_b200 import synth
        from latent_mixture_experts_softmax_b200.layer import DeviceLayer
        self.layer = synth.make_layer(wl)
        self.base = DeviceLayer(wl.shape, self.layer, device=dev_name)
        s = wl.shape
        # bytes a step of T_min tokens touches at least: every weight except
        # the experts, plus the records of its routed experts (at least top_k)
        self.touch = min(self.base.weight_bytes(), self.base.weight_bytes() - self.base.experts.numel()
                         + s.top_k * B.lmoe_expert_record_bytes(self.base.cfg))
        self.R = args.copies or (1 if self.touch > 2 * 126e6 else int(np.ceil(2 * 126e6 / self.touch)) + 1)
        self.devs = weight_copies(self.base, self.R)


def measure_layer(args, wl, T, K, W, rank, world, local, dev_name, ctx=None, light=False):
    """Times K steps of one layer at T tokens (graph replay); unless light,
    then the same steps launched one by one with events between the
    library's kernels, then K end-to-end steps through the host-buffer entry
    point.  Returns the fields of a bench line and the layer's host arrays
    (for the CPU baseline)."""
    import torch
    import torch.distributed as dist
    from latent_mixture_experts_softmax_b200 import binding as B
    from latent_mixture_experts_softmax_b200 import synth
    from latent_mixture_experts_softmax_b200.layer import to_device

    own_ctx = ctx is None
    ctx = ctx or LayerCtx(args, wl, T, dev_name)
    layer, base, devs, R = ctx.layer, ctx.base, ctx.devs, ctx.R
    s = wl.shape
    ws = base.workspace(T)
    prefill = T >= 64 and s.router_dtype == "bf16" and s.n_experts % 128 == 0
    stages = PREFILL_STAGES if prefill else decode_stages(T, s)
    # one CUDA graph per distinct step (its own token batch, weight copy and
    # output buffers); the timed loop replays them in turn
    n_graphs = min(K, 8 if prefill else 64)
    xs_host = [synth.make_x(wl, T=T, draw=rank * 100_003 + i) for i in range(n_graphs)]
    xs = [to_device(x, dev_name) for x in xs_host]
    ys = [torch.empty_like(x) for x in xs]
    idx_all = torch.empty((n_graphs, T, s.top_k), dtype=torch.int32, device=dev_name)
    w_all = torch.empty((n_graphs, T, s.top_k), dtype=torch.float32, device=dev_name)
    stream = torch.cuda.current_stream()

    def step(i, st=None):
        g = i % n_graphs
        d = devs[g % R]
        B.lmoe_forward_ex(d.cfg, xs[g], d.router_w, d.router_b, d.expert_group, d.D, d.U, d.experts, d.shared,
                          None, None, None, idx_all[g], w_all[g], ys[g], T, ws, st or torch.cuda.current_stream())

    for i in range(max(W, n_graphs)):
        step(i)
    torch.cuda.synchronize()
    graphs = []
    for g in range(n_graphs):
        cg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(cg):
            step(g)
        graphs.append(cg)
    for i in range(W):
        graphs[i % n_graphs].replay()
    torch.cuda.synchronize()

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start.record()
        for k in range(K):
            graphs[(W + k) % n_graphs].replay()
        end.record()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_max = max_over_ranks(start.elapsed_time(end), dev_name)
    status = B.lmoe_last_device_status(ws)
    del graphs

    idx_np = idx_all.cpu().numpy()
    groups = layer["expert_group"]
    per_graph = [step_cost(s, idx_np[g], groups, T, prefill) for g in range(n_graphs)]
    step_alg_bytes = float(np.mean([c["bytes_total"] for c in per_graph]))
    step_flops = float(np.mean([c["flops_total"] for c in per_graph]))
    nd = [c["n_distinct"] for c in per_graph]
    hbm_peak, tc_peak, peak_src = load_peaks()
    t_step = ms_max / K / 1e3
    t_lb = max(step_alg_bytes / (hbm_peak * 1e9), step_flops / (tc_peak * 1e12))
    if light:
        return {"T": T, "value": replica_throughput(world, T, K, ms_max), "ms_per_step": ms_max / K,
                "distinct_experts_per_step": float(np.mean(nd)), "algorithmic_bytes": step_alg_bytes,
                "gbs": step_alg_bytes / t_step / 1e9, "frac_of_roofline": t_lb / t_step,
                "clocks": clk.summary(), "device_status": status}, layer

    # per-kernel durations: the same steps launched one by one, with CUDA
    # events the library records between its kernels on the step's stream
    # (serialised: these launches lose the overlap of the graph replay)
    K2 = min(K, 200)
    n_ev = len(stages) + 1
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(K2)]
    torch.cuda.synchronize()
    for k in range(K2):
        B.lmoe_profile_stage_events(evs[k])
        step(k)
    torch.cuda.synchronize()
    B.lmoe_profile_stage_events([])
    stage_ms = np.zeros(len(stages))
    for k in range(K2):
        for j in range(len(stages)):
            stage_ms[j] += evs[k][j].elapsed_time(evs[k][j + 1])
    stage_ms /= K2

    cost = {st: float(np.mean([c[st] for c in per_graph])) for st in stages}
    dom = int(np.argmax(stage_ms))
    dom_name = stages[dom]
    dom_s = stage_ms[dom] / 1e3
    if prefill:
        dom_ach = cost[dom_name] / dom_s / 1e12
        if getattr(s, "act_fmt", "fp16") == "nvfp4" and dom_name in ("gateup", "down"):
            # W4A4 expert GEMMs run kind::mxf4nvf4: the FP4 peak, taken as the
            # measured bf16 peak times the nominal dense ratio 9 / 2.25 = 4
            peak, psrc = 4.0 * tc_peak, f"{peak_src} bf16 dense burst x 4 (nominal fp4 / bf16 dense ratio)"
        else:
            peak, psrc = tc_peak, f"{peak_src} bf16 dense burst (fp16 operands run at the bf16 rate)"
        roof = {"bound": "tensor", "kernel": dom_name, "achieved": dom_ach, "peak": peak, "unit": "TFLOP/s",
                "frac": dom_ach / peak, "peak_source": psrc, "traffic": ncu_traffic(wl, T, dom_name)}
    else:
        dom_ach = cost[dom_name] / dom_s / 1e9
        roof = {"bound": "hbm", "kernel": dom_name, "achieved": dom_ach, "peak": hbm_peak, "unit": "GB/s",
                "frac": dom_ach / hbm_peak, "peak_source": f"{peak_src} HBM copy",
                "traffic": ncu_traffic(wl, T, dom_name)}
    # e2e through the host-buffer entry point (copies inside the timed region)
    x_pin = [torch.from_numpy(x.view(np.int16)).pin_memory() for x in xs_host]
    y_pin = torch.empty((T, s.hidden), dtype=torch.int16).pin_memory()
    for i in range(max(1, min(W, K))):
        d = devs[i % R]
        B.lmoe_forward_host(d.cfg, x_pin[i % n_graphs], d.router_w, d.router_b, d.expert_group, d.D, d.U, d.experts,
                            d.shared, y_pin, T, ws, stream)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(K):
        d = devs[i % R]
        B.lmoe_forward_host(d.cfg, x_pin[i % n_graphs], d.router_w, d.router_b, d.expert_group, d.D, d.U, d.experts,
                            d.shared, y_pin, T, ws, stream)
    e1.record()
    torch.cuda.synchronize()
    e2e_rate = replica_throughput(world, T, K, max_over_ranks(e0.elapsed_time(e1), dev_name))

    out = {
        "value": replica_throughput(world, T, K, ms_max), "unit": "tokens/s", "steps": K, "warmup": W,
        "ms_per_step": ms_max / K,
        "config": {"workload": workload_desc(wl, T), "T": T, "parallelism": f"replicas x{world}",
                   "l2": (f"inputs larger than L2: {R} weight copies rotated, at least "
                          f"{(R - 1) * ctx.touch / 1e6:.0f} MB touched between reuses of one"),
                   "weights": "NVFP4 experts, Q8_0/Q4_0 D/U, bf16 router and shared expert; "
                              "bf16 activations in and out, fp32 accumulation",
                   "path": ("tensor cores (tcgen05): fp16 operands dequantised from the stored formats"
                            if prefill else
                            ("router kernel, D and U weight-streaming kernels (mma.sync, fp16 operands), NVFP4 "
                             "gate/up and down on the tensor cores as stored (tcgen05 kind::mxf4nvf4, "
                             "activations as six E2M1 terms), fp32 accumulation, programmatic dependent launch"
                             if tensor_core_experts(s, T) else
                             "router kernel + four weight-streaming kernels (mma.sync, fp16 operands, fp32 "
                             "accumulation), programmatic dependent launch")),
                   "timing": f"{n_graphs} captured CUDA graphs replayed in turn"},
        "roofline": roof,
        "layer": {"gbs": step_alg_bytes / t_step / 1e9, "tflops": step_flops / t_step / 1e12,
                  "algorithmic_bytes": step_alg_bytes, "algorithmic_flops": step_flops,
                  "roofline_time_us": t_lb * 1e6, "frac_of_roofline": t_lb / t_step,
                  "bound": "tensor" if step_flops / (tc_peak * 1e12) > step_alg_bytes / (hbm_peak * 1e9) else "hbm"},
        "distinct_experts_per_step": float(np.mean(nd)),
        "kernels": {st: {"us_avg": 1e3 * stage_ms[j], "share": stage_ms[j] / stage_ms.sum(),
                         ("tflops" if prefill else "gbs"): cost[st] / (stage_ms[j] / 1e3) / (1e12 if prefill else 1e9)}
                    for j, st in enumerate(stages)},
        "kernel_timing": (f"CUDA events recorded by the library between its kernels, {K2} steps launched one by one "
                          "(serialised: the programmatic-launch overlap of the graph replay is lost, so the shares "
                          "add up to more than a replayed step)"),
        "e2e": {"value": e2e_rate, "unit": "tokens/s", "h2d_bytes_per_step": T * s.hidden * 2,
                "d2h_bytes_per_step": T * s.hidden * 2},
        "gpu_launches": (len(stages) + (3 if prefill else 0)) * K,
        "path": "prefill" if prefill else "decode",
        "clocks": clk.summary(),
        "device_status": status,
    }
    del xs, ys
    if own_ctx:
        del devs, base, ctx
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out, layer


def dproj_ablation(ctx, wl, K, dev_name):
    """D_g alone, as the reference kernel runs it (Q8_1 activations, every
    group) and as this library needs it (fp16 activations, only the groups a
    batch hits), at 1 and 4 tokens.  Each launch reads its D from one of the
    R weight copies after an L2 flush; events bracket the kernels only."""
    import torch
    from latent_mixture_experts_softmax_b200 import binding as B
    from latent_mixture_experts_softmax_b200 import synth
    from latent_mixture_experts_softmax_b200.layer import to_device
    s = wl.shape
    G = s.n_groups
    flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev_name)
    du = B.lmoe_du_bytes(ctx.base.cfg) // G
    hbm, _, src = load_peaks()
    out = {"note": "weights read from HBM (L2 flushed before every launch); Q8_1: k_quantize_q8_1 + the D kernel",
           "peak_gbs": hbm, "peak_source": src}
    n = max(20, min(K, 100))
    for T in (1, 4):
        xs = [to_device(synth.make_x(wl, T=T, draw=700 + i), dev_name) for i in range(4)]
        ws = ctx.base.workspace(T)
        h = torch.empty((T, G, s.latent), dtype=torch.float32, device=dev_name)
        idx = torch.empty((T, s.top_k), dtype=torch.int32, device=dev_name)
        w = torch.empty((T, s.top_k), dtype=torch.float32, device=dev_name)
        masks = []
        for x in xs:
            B.lmoe_route(ctx.base.cfg, x, ctx.base.router_w, ctx.base.router_b, T, idx, w, ws)
            masks.append(sum(1 << int(g) for g in {int(ctx.layer["expert_group"][e]) for e in idx.cpu().numpy().ravel()}))
        res = {}
        for name, fmt, use_hit in (("q8_1_all_groups", 1, False), ("fp16_all_groups", 0, False),
                                   ("fp16_hit_groups", 0, True)):
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
            groups = []
            for i in range(n + 3):
                d = ctx.devs[i % ctx.R]
                mask = masks[i % 4] if use_hit else (1 << G) - 1
                flush.zero_()
                if i >= 3:
                    ev[i - 3][0].record()
                B.lmoe_dproj_ablation(d.cfg, xs[i % 4], d.D, fmt, mask, h, T, ws)
                if i >= 3:
                    ev[i - 3][1].record()
                    groups.append(bin(mask).count("1"))
            torch.cuda.synchronize()
            us = float(np.mean([a.elapsed_time(b) for a, b in ev])) * 1e3
            gb = float(np.mean(groups)) * du + T * s.hidden * 2
            res[name] = {"us": us, "groups": float(np.mean(groups)), "gbs": gb / (us * 1e-6) / 1e9,
                         "frac_of_hbm": gb / (us * 1e-6) / 1e9 / hbm}
        res["speedup_ours_vs_reference"] = res["q8_1_all_groups"]["us"] / res["fp16_hit_groups"]["us"]
        out[f"T{T}"] = res
    del flush
    return out


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    from latent_mixture_experts_softmax_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    if args.act_fmt:
        wl = wl.with_(shape=synth.replace(wl.shape, act_fmt=args.act_fmt))
    T = args.T or wl.T

    if args.impl == "reference":
        run_reference(args, wl, T, rank, world)
        return

    import torch
    import torch.distributed as dist
    from latent_mixture_experts_softmax_b200 import build

    torch.cuda.set_device(local)
    dev_name = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev_name)
    build.build_all()
    if wl.n_layers > 1:
        run_stack(args, wl, T, rank, world, local, dev_name)
        if world > 1:
            dist.destroy_process_group()
        return

    K, W = args.steps, args.warmup
    decode = T < 64
    windows = [t for t in (1, 2, 3, 8) if t != T] if decode and not args.no_sweep else []
    ctx = LayerCtx(args, wl, min([T] + windows), dev_name)
    head, layer = measure_layer(args, wl, T, K, W, rank, world, local, dev_name, ctx=ctx)
    line = {"metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W,
            "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f16", "data": "synthetic"}
    line.update({k: v for k, v in head.items() if k not in line})
    if windows:
        # MTP verify windows of other sizes on the same weights: distinct
        # experts a window routes to, against 3.05 x one token's at 4 tokens
        # (the teardown article, "The engine computes the misses where they lie")
        sweep = {T: {"T": T, "value": head["value"], "ms_per_step": head["ms_per_step"],
                     "distinct_experts_per_step": head["distinct_experts_per_step"],
                     "algorithmic_bytes": head["layer"]["algorithmic_bytes"], "gbs": head["layer"]["gbs"],
                     "frac_of_roofline": head["layer"]["frac_of_roofline"]}}
        for t in windows:
            sweep[t], _ = measure_layer(args, wl, t, K, W, rank, world, local, dev_name, ctx=ctx, light=True)
        one = sweep[1]["distinct_experts_per_step"] if 1 in sweep else float(wl.shape.top_k)
        line["mtp_window"] = {
            "windows": [sweep[t] for t in sorted(sweep)],
            "distinct_ratio_vs_one_token": {str(t): sweep[t]["distinct_experts_per_step"] / one for t in sorted(sweep)},
            "pages_ratio_at_4_tokens": 3.05,
            "note": "distinct experts per window divided by those of one token (top_k); the pages' constant is for "
                    "real routing, these windows draw independent synthetic tokens with a N(0,1) expert bias"}
    if decode and not args.no_sweep:
        line["ablation_dproj"] = dproj_ablation(ctx, wl, K, dev_name)
    del ctx
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, layer, T, args.cpu_seconds)
    pre_wl = None if args.prefill_workload == "none" or T >= 64 else synth.WORKLOADS[args.prefill_workload]
    if pre_wl is not None:
        pre, pre_layer = measure_layer(args, pre_wl, pre_wl.T, K, W, rank, world, local, dev_name)
        pre["metric"] = "latent-MoE layer tokens/s, prefill"
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            pre["cpu_baseline"] = cpu_baseline(pre_wl, pre_layer, pre_wl.T, args.cpu_seconds, sample_tokens=16)
        line["prefill"] = pre
        line["gpu_launches"] = head["gpu_launches"] + pre["gpu_launches"]
        if not args.no_w4a4 and pre_wl.shape.expert_fmt == "nvfp4":
            # the same prefill with NVFP4 expert inputs (W4A4, lmoe_cfg.act_fmt)
            w4_wl = pre_wl.with_(shape=synth.replace(pre_wl.shape, act_fmt="nvfp4"))
            w4, _ = measure_layer(args, w4_wl, w4_wl.T, K, W, rank, world, local, dev_name)
            w4["metric"] = "latent-MoE layer tokens/s, prefill, W4A4 (NVFP4 expert inputs)"
            line["prefill_w4a4"] = w4
            line["gpu_launches"] += w4["gpu_launches"]
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
