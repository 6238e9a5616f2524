#!/usr/bin/env python
"""Benchmark of one DeepSeek-V3 MoE feed-forward layer forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill]
    python bench.py --impl reference ...      # the fp64 CPU oracle, same metric

A step is one full layer forward (router, dispatch, grouped SwiGLU experts,
shared expert, combine) over one batch of synthetic tokens already resident in
HBM.  Default workload: the prefill layer, T=4096 tokens, d=7168, 256 routed
experts top-8 + 1 shared expert, inter 2048, bf16 weights and activations,
fp32 accumulation, fp32 output.  The weights (22.6 GB) are far larger than the
126 MB L2, so no flush is needed between steps.

With N > 1 (torchrun, one process per GPU) every rank runs an independent
replica of the layer on its own batch (the layer needs no exchange on one GPU's
worth of experts); time is the max over ranks and value counts all ranks'
tokens.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "MoE-layer tokens/s and TFLOPS at V3 shapes (T=4096 bf16); % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# B200 datasheet figures (dense): the second denominator every fraction is
# also reported against
DATASHEET_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0, "fp8_tflops": 4500.0}
FP8_OVER_BF16 = 2.0  # nominal dense FP8 : bf16 tensor throughput


def parse_args():
    p = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--workload", default="prefill", choices=("prefill", "decode", "skewed", "fp8", "tiny"))
    p.add_argument("--tokens", type=int, default=None, help="override T (profiling small cases)")
    p.add_argument("--experts", type=int, default=None, help="override E (profiling small cases)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-other", action="store_true",
                   help="leave out the skewed and FP8 records that the default prefill run adds")
    p.add_argument("--cpu-sample", type=int, default=16, help="tokens the CPU baseline runs through the oracle")
    p.add_argument("--ref-sample", type=int, default=2, help="tokens per step of the reference arm")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--sustain-s", type=float, default=2.5,
                   help="seconds of back-to-back layers in the sustained leg (0: skip it)")
    p.add_argument("--no-backward", action="store_true",
                   help="skip the backward-pass record that the prefill run adds to its line")
    p.add_argument("--no-decode", action="store_true",
                   help="skip the decode-batch record that the prefill run adds to its line")
    p.add_argument("--ep-size", type=int, default=1,
                   help="expert-parallel layer over this many ranks (moe_forward_ep + an all-reduce of y)")
    p.add_argument("--ep-rank", type=int, default=0,
                   help="with one process and --ep-size > 1: the rank whose share is timed")
    return p.parse_args()


# ------------------------------------------------------------------ plumbing
class Dist:
    """One process per GPU (torchrun env).  NCCL when CUDA is present, else
    gloo (host-side tests); used only for barriers and the max over ranks of
    the measured time -- the replicas exchange no data."""

    def __init__(self, backend=None, timeout_s: float = 300.0):
        self.rank = int(os.environ.get("RANK", "0"))
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        self.device = torch.device("cpu")
        if self.world > 1:
            import torch.distributed as dist
            backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
            kw = {}
            if backend == "nccl":
                torch.cuda.set_device(self.local)
                self.device = torch.device("cuda", self.local)
                kw["device_id"] = self.device
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, v: float) -> float:
        if not self.pg:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=self.device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


def load_peaks():
    """Measured peaks of this machine's B200s (MEASURED_PEAKS.json) or the
    fallback figures; FP8 tensor peaks are the bf16 ones x the nominal ratio."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        peaks, src = {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except (OSError, KeyError, ValueError):
        peaks, src = dict(FALLBACK_PEAKS), "fallback"
    peaks["fp8_tflops"] = peaks["bf16_tflops"] * FP8_OVER_BF16
    peaks["fp8_tflops_sustained"] = peaks["bf16_tflops_sustained"] * FP8_OVER_BF16
    return peaks, src


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""
    NAMES = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
             0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
             0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.ok = False
        self.samples = []
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            props = torch.cuda.get_device_properties(device_index)
            try:
                bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: report that instead of clocks
            self.err = str(e)

    def _reasons(self):
        fn = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            self.nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return fn(self.h)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append((self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM),
                                     self._reasons(), self.nv.nvmlDeviceGetUtilizationRates(self.h).gpu))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._stop = threading.Event()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok:
            return {"error": f"NVML unavailable: {self.err}"}
        busy = [s for s in self.samples if s[2] > 0] or self.samples
        if not busy:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        bits = 0
        for s in busy:
            bits |= s[1]
        reasons = [n for b, n in self.NAMES.items() if bits & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(s[0] for s in busy), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(busy)}


def captured_traffic(stage: str, args):
    """DRAM bytes per launch of `stage`'s kernel from the committed ncu capture
    of the prefill workload, or None when this run is another workload or the
    kernel sources changed since the capture."""
    import hashlib
    import re
    if args.workload != "prefill" or args.tokens or args.experts:
        return None
    path = os.path.join(ROOT, "profiles", "grouped_gemm_prefill_T4096_traffic.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    csrc = os.path.join(ROOT, "mixture_experts_ffn_17_b200", "csrc")
    h = hashlib.sha256()
    for f in ("grouped_gemm.cu", "ptx.cuh", "common.cuh", "moe_internal.h"):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    m = re.search(r"source_sha256_16:\s*([0-9a-f]{16})", text)
    t = re.search(r"traffic_bytes_per_launch\.%s:\s*(\d+)" % stage, text)
    if not m or not t or m.group(1) != h.hexdigest()[:16]:
        return None
    return int(t.group(1))


# ------------------------------------------------------------------ workload
def touched_experts(counts) -> int:
    return int((counts > 0).sum())


def layer_work(cfg, counts, y_bytes_per_el):
    """Algorithmic FLOPs and bytes of one layer forward (what the method must
    do: router + touched experts' weights read once + shared expert + Wg + x
    read + y written)."""
    wb = 1 if cfg.fp8 else 2
    flops = cfg.T * cfg.flops_per_token()
    n_touched = touched_experts(counts)
    routed_w = n_touched * 3 * cfg.d * cfg.inter * wb
    if cfg.fp8:
        routed_w += n_touched * 3 * (cfg.d // 128) * (cfg.inter // 128) * 4
    shared_w = 3 * cfg.d * cfg.shared_inter * 2
    act = cfg.T * cfg.d * 2 + cfg.T * cfg.d * y_bytes_per_el
    return flops, routed_w + shared_w + cfg.E * cfg.d * 2 + act, n_touched


def layer_roofline(cfg, counts, ms, peaks, peak_src, y_bytes_per_el=4):
    """max(FLOPs / tensor peak, bytes / HBM bandwidth) of one layer and the
    fraction of it a measured step time reaches.  The routed experts' FLOPs of
    an FP8 workload are priced at the FP8 peak and the router's and shared
    expert's at the bf16 one; `frac_bf16_rate` prices every FLOP at the bf16
    peak (the MMA runs kind::f16: the activations stay bf16).  Both against the
    measured peaks (sustained tensor peak) and against the datasheet."""
    flops, nbytes, n_touched = layer_work(cfg, counts, y_bytes_per_el)
    f_routed = cfg.T * cfg.k * 6 * cfg.d * cfg.inter
    f_fp8 = f_routed if cfg.fp8 else 0
    f_bf16 = flops - f_fp8

    def terms(bf16, fp8, hbm):
        t_tc = f_bf16 / (bf16 * 1e12) + f_fp8 / (fp8 * 1e12)
        t_tc16 = flops / (bf16 * 1e12)
        t_hbm = nbytes / (hbm * 1e9)
        return t_tc, t_tc16, t_hbm

    t_tc, t_tc16, t_hbm = terms(peaks["bf16_tflops_sustained"], peaks["fp8_tflops_sustained"], peaks["hbm_gbs"])
    d_tc, d_tc16, d_hbm = terms(DATASHEET_PEAKS["bf16_tflops"], DATASHEET_PEAKS["fp8_tflops"],
                                DATASHEET_PEAKS["hbm_gbs"])
    roof = max(t_tc, t_hbm)
    out = {"roofline_ms": 1e3 * roof, "tensor_ms": 1e3 * t_tc, "hbm_ms": 1e3 * t_hbm,
           "bound": "hbm" if t_hbm >= t_tc else "tensor", "frac": 1e3 * roof / ms,
           "frac_datasheet": 1e3 * max(d_tc, d_hbm) / ms,
           "flops": flops, "bytes": nbytes, "touched_experts": n_touched,
           "peaks": f"{peak_src}: hbm {peaks['hbm_gbs']} GB/s, bf16 {peaks['bf16_tflops_sustained']} TF/s sustained"
                    + (f", fp8 {peaks['fp8_tflops_sustained']} TF/s (bf16 x {FP8_OVER_BF16:g})" if cfg.fp8 else "")
                    + f"; datasheet: hbm {DATASHEET_PEAKS['hbm_gbs']:g} GB/s, bf16 {DATASHEET_PEAKS['bf16_tflops']:g}"
                    + (f", fp8 {DATASHEET_PEAKS['fp8_tflops']:g}" if cfg.fp8 else "") + " TF/s"}
    if cfg.fp8:
        out["frac_bf16_rate"] = 1e3 * max(t_tc16, t_hbm) / ms
        out["frac_bf16_rate_datasheet"] = 1e3 * max(d_tc16, d_hbm) / ms
    return out


def touched_weight_bytes(cfg, counts):
    """Weight bytes a layer must stream: the touched routed experts (with FP8
    block scales) and the shared expert."""
    wb = 1 if cfg.fp8 else 2
    n = touched_experts(counts)
    b = n * 3 * cfg.d * cfg.inter * wb + 3 * cfg.d * cfg.shared_inter * 2
    if cfg.fp8:
        b += n * 3 * (cfg.d // 128) * (cfg.inter // 128) * 4
    return b


def kernel_work(cfg, counts, stage):
    """Algorithmic FLOPs / bytes of one launch of an expert kernel: the
    touched experts' weight slices plus the shared expert's, the activation
    rows read once, and the rows written."""
    wb = 1 if cfg.fp8 else 2
    n_touched = touched_experts(counts)
    rows = cfg.T * cfg.k
    if stage == "experts_up":
        w = (n_touched * 2 * cfg.d * cfg.inter) * wb + 2 * cfg.d * cfg.shared_inter * 2
        flops = rows * 4 * cfg.d * cfg.inter + cfg.T * 4 * cfg.d * cfg.shared_inter
        act = cfg.T * cfg.d * 2 + rows * cfg.inter * 2 + cfg.T * cfg.shared_inter * 2
    else:  # experts_down
        w = (n_touched * cfg.d * cfg.inter) * wb + cfg.d * cfg.shared_inter * 2
        flops = rows * 2 * cfg.d * cfg.inter + cfg.T * 2 * cfg.d * cfg.shared_inter
        act = rows * cfg.inter * 2 + cfg.T * cfg.shared_inter * 2 + rows * cfg.d * 2 + cfg.T * cfg.d * 4
    return flops, w + act


# ------------------------------------------------------------------ oracle timing
def oracle_sample(w, tokens, fetch_cache=None):
    """Run the fp64 oracle on a sample of tokens of a device-resident workload.
    Returns (seconds of oracle work, outputs).  Copies device->host are not
    timed; decoding stored values and all arithmetic are."""
    import oracle
    cfg = w.cfg
    tok = torch.as_tensor(tokens, device=w.x.device)
    x_host = w.x[tok].cpu()
    wg_host = w.Wg.cpu()
    shared_host = [t.cpu() for t in (w.W1s, w.W3s, w.W2s)]
    bias = None if w.bias is None else w.bias.double().cpu().numpy()
    t0 = time.perf_counter()
    x = oracle.decode(x_host)
    lg = oracle.logits(x, oracle.decode(wg_host))
    if cfg.route == 0:
        idx, wts, _ = oracle.route_topk_softmax(lg, cfg.k)
    else:
        idx, wts, _, _ = oracle.route_sigmoid_group(lg, bias, cfg.k, cfg.n_group, cfg.topk_group, cfg.group_topn,
                                                   cfg.route_scale)
    spent = time.perf_counter() - t0
    y = np.zeros((len(tokens), cfg.d))
    for e in np.unique(idx):
        rows, slots = np.nonzero(idx == e)
        if cfg.fp8:
            host = [(w.W1[e].cpu(), w.s1[e].cpu()), (w.W3[e].cpu(), w.s3[e].cpu()), (w.W2[e].cpu(), w.s2[e].cpu())]
            t0 = time.perf_counter()
            W = [oracle.decode_e4m3_blocks(q.numpy(), s.numpy()) for q, s in host]
        else:
            host = [w.W1[e].cpu(), w.W3[e].cpu(), w.W2[e].cpu()]
            t0 = time.perf_counter()
            W = [oracle.decode(t) for t in host]
        o = oracle.swiglu_rows(x[rows], *W)
        y[rows] += wts[rows, slots][:, None] * o
        spent += time.perf_counter() - t0
    t0 = time.perf_counter()
    y += oracle.swiglu_rows(x, *[oracle.decode(t) for t in shared_host])
    spent += time.perf_counter() - t0
    return spent, y


def cpu_threads():
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


# ------------------------------------------------------------------ arms
def run_reference(args, dist):
    """The oracle as the reference arm: every step runs a bounded sample of
    the workload's tokens through the fp64 CPU oracle on the host cores."""
    from mixture_experts_ffn_17_b200 import workloads
    if dist.rank != 0:
        return
    cfg = workloads.CONFIGS[args.workload]
    if args.tokens:
        cfg = cfg.replace(T=args.tokens)
    if args.experts:
        cfg = cfg.replace(E=args.experts)
    w = workloads.make(cfg, device="cuda")
    S = args.ref_sample
    times = []
    for step in range(args.warmup + args.steps):
        toks = [(step * S + i) % cfg.T for i in range(S)]
        t, _ = oracle_sample(w, toks)
        if step >= args.warmup:
            times.append(t)
    per_tok = sum(times) / (S * len(times))
    value = 1.0 / per_tok
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(cfg, args),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
                             "sample": f"{S} tokens per step of the {cfg.name} workload through the whole layer "
                                       f"(fp64 oracle, OpenMP over rows)"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_of(cfg, args):
    return {"workload": f"{cfg.name}: MoE FFN layer T={cfg.T} d={cfg.d} E={cfg.E} top-{cfg.k} inter={cfg.inter} "
                        f"+ shared {cfg.shared_inter}, {'e4m3 experts' if cfg.fp8 else 'bf16'}",
            "T": cfg.T, "d": cfg.d, "E": cfg.E, "k": cfg.k, "inter": cfg.inter, "shared_inter": cfg.shared_inter,
            "routing": "top-k then softmax" if cfg.route == 0 else "sigmoid group-limited (8 groups, top-4)",
            "seed": cfg.seed, "l2": "inputs larger than L2 (weights 22.6 GB vs 126 MB L2); no flush",
            "parallelism": f"replicas x{args.gpus}"}


def time_loop(step, K, stream, dev, dist):
    """K calls of step(i) between events on the launching stream, with a
    barrier and a synchronize on both sides and NVML clock samples during the
    loop.  Returns (ms per step, max over ranks; clock summary)."""
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index)
    dist.barrier()
    torch.cuda.synchronize(dev)
    with sampler:
        start.record(stream)
        for i in range(K):
            step(i)
        end.record(stream)
        torch.cuda.synchronize(dev)
    dist.barrier()
    return dist.max(start.elapsed_time(end) / K), sampler.summary()


def sustained_leg(B, fwd_args, counts, cfg, K_min, ms_burst, seconds, stream, dev, dist, peaks, peak_src):
    """Back-to-back layers for about `seconds` (the power cap sets the clock
    after a few hundred ms): its own step time, clocks and roofline fraction."""
    K = max(K_min, int(math.ceil(seconds * 1e3 / ms_burst)))
    ms, clocks = time_loop(lambda i: B.forward(*fwd_args, counts=counts), K, stream, dev, dist)
    c = counts.cpu().numpy()
    roof = layer_roofline(cfg, c, ms, peaks, peak_src)
    out = {"steps": K, "seconds": K * ms / 1e3, "ms_per_step": ms, "tokens_per_s": dist.world * cfg.T / (ms / 1e3),
           "tflops": dist.world * roof["flops"] / (ms / 1e3) / 1e12, "frac": roof["frac"],
           "frac_datasheet": roof["frac_datasheet"], "clocks": clocks}
    if "frac_bf16_rate" in roof:
        out["frac_bf16_rate"] = roof["frac_bf16_rate"]
    if clocks.get("sm_mhz"):
        out["mcycles_per_step"] = ms * clocks["sm_mhz"] / 1e3   # step time x median SM clock
    return out


def decode_record(args, dist, dev, stream, peaks, peak_src):
    """The decode layer (T=64) timed in the same run: touched-expert weight
    streaming against HBM bandwidth, burst and sustained."""
    from mixture_experts_ffn_17_b200 import binding as B
    from mixture_experts_ffn_17_b200 import workloads
    cfg = workloads.CONFIGS["decode"]
    w = workloads.make(cfg, device=dev)
    shape = B.shape_of(cfg, B.MOE_F32)
    ws = B.alloc_workspace(shape, dev)
    y = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device=dev)
    counts = torch.empty(cfg.E, dtype=torch.int32, device=dev)
    fwd_args = (shape, w.x, w.Wg, w.bias, w.W1, w.W3, w.W2, w.s1, w.s3, w.s2, w.W1s, w.W3s, w.W2s, y, ws)
    for _ in range(max(args.warmup, 3)):
        B.forward(*fwd_args, counts=counts)
    rc, raw = B.check_device_status(ws)
    if rc != B.MOE_OK:
        raise B.MoeError(rc, f"decode: device status after warm-up (raw {raw})")
    K = max(args.steps, 50)
    ms, clocks = time_loop(lambda i: B.forward(*fwd_args, counts=counts), K, stream, dev, dist)
    c = counts.cpu().numpy()
    roof = layer_roofline(cfg, c, ms, peaks, peak_src)
    wbytes = touched_weight_bytes(cfg, c)
    rec = {"workload": config_of(cfg, args)["workload"], "steps": K, "ms_per_step": ms,
           "tokens_per_s": dist.world * cfg.T / (ms / 1e3), "touched_experts": roof["touched_experts"],
           "touched_weight_bytes": wbytes,
           "touched_weight_gbs": wbytes / (ms / 1e3) / 1e9,
           "hbm_frac": wbytes / (ms / 1e3) / 1e9 / peaks["hbm_gbs"],
           "hbm_frac_datasheet": wbytes / (ms / 1e3) / 1e9 / DATASHEET_PEAKS["hbm_gbs"],
           "roofline_layer": roof, "clocks": clocks}
    if args.sustain_s > 0:
        sus = sustained_leg(B, fwd_args, counts, cfg, K, ms, args.sustain_s, stream, dev, dist, peaks, peak_src)
        sus["hbm_frac"] = wbytes / (sus["ms_per_step"] / 1e3) / 1e9 / peaks["hbm_gbs"]
        rec["sustained"] = sus
    rc, raw = B.check_device_status(ws)
    if rc != B.MOE_OK:
        raise B.MoeError(rc, f"decode: device status after the timed steps (raw {raw})")
    rec["gpu_launches_per_step"] = B.forward_launches(shape)
    return rec


def workload_record(name, args, dist, dev, stream, peaks, peak_src):
    """Another workload of the layer (its own weights) timed in the same run:
    the burst and a sustained leg against its own layer roofline, with clocks,
    so that one bench line carries every config's measurement."""
    from mixture_experts_ffn_17_b200 import binding as B
    from mixture_experts_ffn_17_b200 import workloads
    cfg = workloads.CONFIGS[name]
    w = workloads.make(cfg, device=dev)
    shape = B.shape_of(cfg, B.MOE_F32)
    ws = B.alloc_workspace(shape, dev)
    y = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device=dev)
    counts = torch.empty(cfg.E, dtype=torch.int32, device=dev)
    fwd_args = (shape, w.x, w.Wg, w.bias, w.W1, w.W3, w.W2, w.s1, w.s3, w.s2, w.W1s, w.W3s, w.W2s, y, ws)
    for _ in range(max(args.warmup, 3)):
        B.forward(*fwd_args, counts=counts)
    rc, raw = B.check_device_status(ws)
    if rc != B.MOE_OK:
        raise B.MoeError(rc, f"{name}: device status after warm-up (raw {raw})")
    K = args.steps
    ms, clocks = time_loop(lambda i: B.forward(*fwd_args, counts=counts), K, stream, dev, dist)
    roof = layer_roofline(cfg, counts.cpu().numpy(), ms, peaks, peak_src)
    rec = {"workload": config_of(cfg, args)["workload"], "steps": K, "ms_per_step": ms,
           "tokens_per_s": dist.world * cfg.T / (ms / 1e3), "tflops": dist.world * roof["flops"] / (ms / 1e3) / 1e12,
           "roofline_layer": roof, "clocks": clocks}
    if args.sustain_s > 0:
        rec["sustained"] = sustained_leg(B, fwd_args, counts, cfg, K, ms, args.sustain_s, stream, dev, dist, peaks,
                                         peak_src)
    rc, raw = B.check_device_status(ws)
    if rc != B.MOE_OK:
        raise B.MoeError(rc, f"{name}: device status after the timed steps (raw {raw})")
    rec["gpu_launches_per_step"] = B.forward_launches(shape)
    if cfg.fp8:
        del ws
        rec["decode_batch"] = decode_batch_record(B, cfg, w, 64, args, dist, dev, stream, peaks, peak_src)
    return rec


def decode_batch_record(B, cfg, w, T, args, dist, dev, stream, peaks, peak_src):
    """The same weights at a decode batch (the workload's first T tokens),
    burst only: the touched experts' weight bytes over the step time against
    HBM, as the decode record measures the bf16 layer."""
    cs = cfg.replace(T=T)
    shape = B.shape_of(cs, B.MOE_F32)
    ws = B.alloc_workspace(shape, dev)
    x = w.x[:T].contiguous()
    y = torch.empty(T, cs.d, dtype=torch.float32, device=dev)
    counts = torch.empty(cs.E, dtype=torch.int32, device=dev)
    fwd_args = (shape, x, w.Wg, w.bias, w.W1, w.W3, w.W2, w.s1, w.s3, w.s2, w.W1s, w.W3s, w.W2s, y, ws)
    for _ in range(max(args.warmup, 3)):
        B.forward(*fwd_args, counts=counts)
    rc, raw = B.check_device_status(ws)
    if rc != B.MOE_OK:
        raise B.MoeError(rc, f"{cs.name} T={T}: device status after warm-up (raw {raw})")
    K = max(args.steps, 50)
    ms, clocks = time_loop(lambda i: B.forward(*fwd_args, counts=counts), K, stream, dev, dist)
    c = counts.cpu().numpy()
    wbytes = touched_weight_bytes(cs, c)
    rc, raw = B.check_device_status(ws)
    if rc != B.MOE_OK:
        raise B.MoeError(rc, f"{cs.name} T={T}: device status after the timed steps (raw {raw})")
    return {"workload": config_of(cs, args)["workload"], "steps": K, "ms_per_step": ms,
            "tokens_per_s": dist.world * T / (ms / 1e3), "touched_experts": touched_experts(c),
            "touched_weight_bytes": wbytes, "touched_weight_gbs": wbytes / (ms / 1e3) / 1e9,
            "hbm_frac": wbytes / (ms / 1e3) / 1e9 / peaks["hbm_gbs"],
            "hbm_frac_datasheet": wbytes / (ms / 1e3) / 1e9 / DATASHEET_PEAKS["hbm_gbs"],
            "roofline_layer": layer_roofline(cs, c, ms, peaks, peak_src), "clocks": clocks}


def backward_work(cfg, counts, grad_bytes):
    """Algorithmic FLOPs and bytes of one moe_backward call (the forward it
    recomputes, then the gradients): FLOPs = the forward's + per routed and
    shared row 12 d I (dH, dX, and the three weight gradients) + 4 T E d
    (dl Wg and dWg); bytes = the touched experts' and the shared expert's
    weights read twice (forward, then dH / dX), every weight gradient written
    once, Wg read twice, dWg written, x and dy read, dx written."""
    T, d, E, k, I, Is = cfg.T, cfg.d, cfg.E, cfg.k, cfg.inter, cfg.shared_inter
    flops = T * cfg.flops_per_token() + T * k * 12 * d * I + T * 12 * d * Is + 4 * T * E * d
    wbytes = touched_weight_bytes(cfg, counts)
    grads = (E * 3 * d * I + 3 * d * Is + E * d) * grad_bytes
    reads = 2 * wbytes + 2 * E * d * 2 + T * d * 2 + T * d * 4
    writes = grads + T * d * grad_bytes
    return flops, reads + writes, reads, writes


def backward_record(args, dist, dev, stream, w, cfg, peaks, peak_src):
    """moe_backward (the training pass: forward recompute and every gradient,
    bf16 gradient outputs) on the same weights, timed like the forward."""
    from mixture_experts_ffn_17_b200 import binding as B
    shape = B.shape_of(cfg, B.MOE_BF16)
    ws = B.alloc_backward_workspace(shape, dev)
    e = lambda *sz: torch.empty(sz, dtype=torch.bfloat16, device=dev)
    grads = [e(cfg.T, cfg.d), e(cfg.E, cfg.d), e(cfg.E, cfg.d, cfg.inter), e(cfg.E, cfg.d, cfg.inter),
             e(cfg.E, cfg.inter, cfg.d), e(cfg.d, cfg.shared_inter), e(cfg.d, cfg.shared_inter),
             e(cfg.shared_inter, cfg.d)]
    dy = torch.randn(cfg.T, cfg.d, generator=torch.Generator(device=dev).manual_seed(cfg.seed + 100), device=dev)
    bargs = (shape, w.x, w.Wg, w.bias, w.W1, w.W3, w.W2, w.W1s, w.W3s, w.W2s, dy, *grads, ws)
    for _ in range(max(3, args.warmup)):
        B.backward(*bargs)
    rc, raw = B.check_device_status(ws)
    if rc != B.MOE_OK:
        raise B.MoeError(rc, f"backward: device status after warm-up (raw {raw})")
    K = max(5, args.steps // 2)
    ms, clocks = time_loop(lambda i: B.backward(*bargs), K, stream, dev, dist)
    rc, raw = B.check_device_status(ws)
    if rc != B.MOE_OK:
        raise B.MoeError(rc, f"backward: device status after the timed steps (raw {raw})")
    # a training step that keeps the forward's state: moe_forward_train (the
    # layer's y) then moe_backward_saved, and the latter alone
    y_tr = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16, device=dev)
    fargs = (shape, w.x, w.Wg, w.bias, w.W1, w.W3, w.W2, w.W1s, w.W3s, w.W2s, y_tr, ws)
    sargs = (shape, w.x, w.Wg, w.W1, w.W3, w.W2, w.W1s, w.W3s, w.W2s, dy, *grads, ws)

    def train_step(i):
        B.forward_train(*fargs)
        B.backward_saved(*sargs)

    for _ in range(2):
        train_step(0)
    ms_step, clocks_step = time_loop(train_step, K, stream, dev, dist)
    ms_fwd_train, _ = time_loop(lambda i: B.forward_train(*fargs), K, stream, dev, dist)
    rc, raw = B.check_device_status(ws)
    if rc != B.MOE_OK:
        raise B.MoeError(rc, f"training step: device status after the timed steps (raw {raw})")
    counts = torch.empty(cfg.E, dtype=torch.int32, device=dev)
    y = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device=dev)
    fws = B.alloc_workspace(B.shape_of(cfg, B.MOE_F32), dev)
    B.forward(B.shape_of(cfg, B.MOE_F32), w.x, w.Wg, w.bias, w.W1, w.W3, w.W2, w.s1, w.s3, w.s2, w.W1s, w.W3s, w.W2s,
              y, fws, counts=counts)
    flops, nbytes, rbytes, wbytes = backward_work(cfg, counts.cpu().numpy(), 2)
    t_tc = flops / (peaks["bf16_tflops_sustained"] * 1e12)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    d_roof = max(flops / (DATASHEET_PEAKS["bf16_tflops"] * 1e12), nbytes / (DATASHEET_PEAKS["hbm_gbs"] * 1e9))
    roof_ms = 1e3 * max(t_tc, t_hbm)
    return {"what": "moe_backward: forward recompute + dx, dWg, dW1, dW3, dW2 and the shared expert's gradients "
                    "(bf16 gradient outputs, fp32 dy)",
            "steps": K, "ms_per_step": ms, "tokens_per_s": dist.world * cfg.T / (ms / 1e3),
            "tflops": dist.world * flops / (ms / 1e3) / 1e12, "flops": flops, "bytes": nbytes,
            "bytes_read": rbytes, "bytes_written": wbytes,
            "roofline_ms": roof_ms, "bound": "hbm" if t_hbm >= t_tc else "tensor",
            "frac": roof_ms / ms, "frac_datasheet": 1e3 * d_roof / ms,
            "train_step": {"what": "moe_forward_train (y, the forward's state kept) + moe_backward_saved",
                           "ms_per_step": ms_step, "tokens_per_s": dist.world * cfg.T / (ms_step / 1e3),
                           "forward_train_ms": ms_fwd_train, "backward_saved_ms_derived": ms_step - ms_fwd_train,
                           "roofline_ms": roof_ms, "frac": roof_ms / ms_step, "clocks": clocks_step},
            "peaks": peak_src + " (HBM copy peak for every byte read or written: plain and bulk stores reach it too)",
            "clocks": clocks}


def run_ours(args, dist):
    from mixture_experts_ffn_17_b200 import binding as B
    from mixture_experts_ffn_17_b200 import workloads

    dev = torch.device("cuda", dist.local)
    torch.cuda.set_device(dev)
    cfg = workloads.CONFIGS[args.workload]
    if args.tokens:
        cfg = cfg.replace(T=args.tokens)
    if args.experts:
        cfg = cfg.replace(E=args.experts)
    w = workloads.make(cfg, device=dev)
    shape = B.shape_of(cfg, B.MOE_F32)
    ws = B.alloc_workspace(shape, dev)
    y = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device=dev)
    counts = torch.empty(cfg.E, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    fwd_args = (shape, w.x, w.Wg, w.bias, w.W1, w.W3, w.W2, w.s1, w.s3, w.s2, w.W1s, w.W3s, w.W2s, y, ws)

    for _ in range(args.warmup):
        B.forward(*fwd_args, counts=counts)
    rc, raw = B.check_device_status(ws)
    if rc != B.MOE_OK:
        raise B.MoeError(rc, f"device status after warm-up (raw {raw})")

    # the timed steps: K layers, each with events at its stage boundaries
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(B.NUM_STAGE_EVENTS)] for _ in range(K)]
    for row in evs:
        for e in row:
            e.record(stream)
    ms_max, clocks = time_loop(lambda i: B.forward_profiled(*fwd_args, evs[i], counts=counts), K, stream, dev, dist)
    rc, raw = B.check_device_status(ws)
    if rc != B.MOE_OK:
        raise B.MoeError(rc, f"device status after the timed steps (raw {raw})")

    stage_ms = {name: statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(K))
                for j, name in enumerate(B.STAGES)}
    counts_np = counts.cpu().numpy()
    peaks, peak_src = load_peaks()
    roof_layer = layer_roofline(cfg, counts_np, ms_max, peaks, peak_src)
    flops = roof_layer["flops"]
    tokens_per_s = dist.world * cfg.T / (ms_max / 1e3)

    # the dominant kernel against its own roofline (the tensor peak of its
    # weights' dtype: FP8 routed experts at the FP8 peak)
    dom = max(("experts_up", "experts_down"), key=lambda s: stage_ms[s])
    kf, kb = kernel_work(cfg, counts_np, dom)
    k_ms = stage_ms[dom]
    tc_key = "fp8_tflops_sustained" if cfg.fp8 else "bf16_tflops_sustained"
    k_tc = kf / (peaks[tc_key] * 1e12)
    k_hbm = kb / (peaks["hbm_gbs"] * 1e9)
    if k_hbm >= k_tc:
        roof = {"bound": "hbm", "achieved": kb / (k_ms / 1e3) / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
        roof["frac_datasheet"] = roof["achieved"] / DATASHEET_PEAKS["hbm_gbs"]
    else:
        roof = {"bound": "tensor", "achieved": kf / (k_ms / 1e3) / 1e12, "peak": peaks[tc_key],
                "unit": "TFLOP/s"}
        roof["frac_datasheet"] = roof["achieved"] / DATASHEET_PEAKS["fp8_tflops" if cfg.fp8 else "bf16_tflops"]
        if cfg.fp8:
            roof["frac_bf16_rate"] = roof["achieved"] / peaks["bf16_tflops_sustained"]
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = captured_traffic(dom, args)
    roof["kernel"] = f"grouped_gemm_kernel<{'SwiGLU' if dom == 'experts_up' else 'Down'}> ({dom})"
    roof["peak_source"] = f"{peak_src} ({'hbm_gbs' if roof['bound'] == 'hbm' else tc_key})"
    roof["algorithmic_bytes_per_launch"] = kb
    roof["algorithmic_flops_per_launch"] = kf
    roof["ms_per_launch"] = k_ms

    sustained = None
    if args.sustain_s > 0:
        sustained = sustained_leg(B, fwd_args, counts, cfg, K, ms_max, args.sustain_s, stream, dev, dist, peaks,
                                  peak_src)
        if clocks.get("sm_mhz"):
            sustained["burst_mcycles_per_step"] = ms_max * clocks["sm_mhz"] / 1e3

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, B, fwd_args, w, cfg, y, dev, stream, dist)

    line = {"metric": METRIC, "value": tokens_per_s, "unit": "tokens/s", "n_gpus": dist.world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_of(cfg, args),
            "tflops": dist.world * flops / (ms_max / 1e3) / 1e12,
            "roofline_layer": roof_layer, "roofline": roof, "stage_ms": stage_ms, "clocks": clocks,
            "gpu_launches": B.forward_launches(shape) * K}
    if sustained:
        line["sustained"] = sustained
    if e2e:
        line["e2e"] = e2e
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = run_cpu_baseline(args, w, cfg)
    if args.workload == "prefill" and not args.no_backward:
        fwd_args = None
        line["backward"] = backward_record(args, dist, dev, stream, w, cfg, peaks, peak_src)
        torch.cuda.empty_cache()
    if args.workload == "prefill" and not (args.tokens or args.experts or args.no_decode):
        # the decode batch of the same layer shapes, in the same run (its own
        # weights; the prefill ones are released first)
        fwd_args = w = ws = y = None
        torch.cuda.empty_cache()
        line["decode"] = decode_record(args, dist, dev, stream, peaks, peak_src)
        line["config"]["workload"] += "; decode record: " + line["decode"]["workload"]
        if not args.no_other:
            # the two other configs of the layer, each with its own weights
            for other in ("skewed", "fp8"):
                torch.cuda.empty_cache()
                line[other] = workload_record(other, args, dist, dev, stream, peaks, peak_src)
                line["config"]["workload"] += f"; {other} record: " + line[other]["workload"]
    if dist.rank == 0:
        print(json.dumps(line), flush=True)


def run_ep(args, dist):
    """Expert-parallel layer (moe_forward_ep): rank r of --ep-size holds E/n
    experts and its slice of the shared expert's hidden features; every step
    runs the rank's share and all-reduces y over the ranks (NCCL), both inside
    the timed region.  With one process only one share can run: --ep-rank picks
    it, there is no all-reduce, and the value is that share's tokens/s."""
    from mixture_experts_ffn_17_b200 import binding as B
    from mixture_experts_ffn_17_b200 import expert_parallel as ep
    from mixture_experts_ffn_17_b200 import workloads

    n = args.ep_size
    if dist.world not in (1, n):
        raise SystemExit(f"--ep-size {n} needs {n} ranks (or one process timing one share)")
    rank = dist.rank if dist.world == n else args.ep_rank
    dev = torch.device("cuda", dist.local)
    torch.cuda.set_device(dev)
    cfg = workloads.CONFIGS[args.workload]
    if args.tokens:
        cfg = cfg.replace(T=args.tokens)
    if args.experts:
        cfg = cfg.replace(E=args.experts)
    w = workloads.make(cfg, device=dev)
    wr = ep.shard_weights(w.W1, w.W3, w.W2, w.s1, w.s3, w.s2, w.W1s, w.W3s, w.W2s, rank, n)
    sl = ep.ep_slice(cfg.E, cfg.shared_inter, rank, n)
    w.W1 = w.W3 = w.W2 = w.s1 = w.s3 = w.s2 = None  # only the rank's share stays resident
    torch.cuda.empty_cache()
    shape = B.shape_of(cfg, B.MOE_F32)
    ws = B.alloc_workspace(shape, dev)
    y = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device=dev)
    counts = torch.empty(cfg.E, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        ep.forward(shape, rank, n, w.x, w.Wg, w.bias, wr, y, ws, counts=counts)

    for _ in range(args.warmup):
        step()
    rc, raw = B.check_device_status(ws)
    if rc != B.MOE_OK:
        raise B.MoeError(rc, f"device status after warm-up (raw {raw})")
    K = args.steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index)
    dist.barrier()
    torch.cuda.synchronize(dev)
    with sampler:
        start.record(stream)
        for _ in range(K):
            step()
        end.record(stream)
        torch.cuda.synchronize(dev)
    dist.barrier()
    ms_max = dist.max(start.elapsed_time(end) / K)
    rc, raw = B.check_device_status(ws)
    if rc != B.MOE_OK:
        raise B.MoeError(rc, f"device status after the timed steps (raw {raw})")

    # the share's algorithmic work: router on every token, the rank's touched
    # experts on their rows, its shared-expert slice on every token
    c = counts.cpu().numpy()
    local_rows = int(c[sl.e_lo:sl.e_hi].sum())
    local_touched = int((c[sl.e_lo:sl.e_hi] > 0).sum())
    wb = 1 if cfg.fp8 else 2
    isl = sl.i_hi - sl.i_lo
    flops = 2 * cfg.T * cfg.d * cfg.E + local_rows * 6 * cfg.d * cfg.inter + cfg.T * 6 * cfg.d * isl
    nbytes = (local_touched * 3 * cfg.d * cfg.inter * wb + 3 * cfg.d * isl * 2 + cfg.E * cfg.d * 2
              + cfg.T * cfg.d * 2 + cfg.T * cfg.d * 4)
    if cfg.fp8:
        nbytes += local_touched * 3 * (cfg.d // 128) * (cfg.inter // 128) * 4
    peaks, peak_src = load_peaks()
    t_tc = flops / (peaks["bf16_tflops_sustained"] * 1e12)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    if t_hbm >= t_tc:
        roof = {"bound": "hbm", "achieved": nbytes / (ms_max / 1e3) / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": flops / (ms_max / 1e3) / 1e12, "peak": peaks["bf16_tflops_sustained"],
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = None
    roof["kernel"] = "whole step of the rank's share (moe_forward_ep" + (" + all-reduce)" if dist.world > 1 else ")")
    roof["peak_source"] = peak_src
    conf = config_of(cfg, args)
    conf["parallelism"] = f"ep{n}"
    conf["ep"] = {"size": n, "rank_timed": rank if dist.world == 1 else "all", "experts": [sl.e_lo, sl.e_hi],
                  "shared_features": [sl.i_lo, sl.i_hi], "all_reduce": dist.world > 1,
                  "note": ("one share on one GPU; the other ranks and the all-reduce are not run"
                           if dist.world == 1 else "all ranks, NCCL all-reduce of y every step")}
    line = {"metric": METRIC, "value": cfg.T / (ms_max / 1e3), "unit": "tokens/s", "n_gpus": dist.world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": conf,
            "tflops": flops / (ms_max / 1e3) / 1e12, "roofline": roof, "clocks": sampler.summary(),
            "gpu_launches": B.forward_launches(shape) * K}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)


def run_e2e(args, B, fwd_args, w, cfg, y, dev, stream, dist):
    """Same metric through the public call with host buffers.  Every step
    copies its own tokens from pinned host memory, runs the layer and copies
    its y back; the copies run on their own streams with double-buffered
    device x / y, so step i+1's upload and step i-1's download overlap step
    i's compute.  Timed from the first upload to the last download."""
    x_host = w.x.cpu().pin_memory()
    y_host = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(w.x) for _ in range(2)]
    y_dev = [torch.empty_like(y) for _ in range(2)]
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    comp = stream

    def run(K):
        ev_up = [torch.cuda.Event() for _ in range(K)]
        ev_comp = [torch.cuda.Event() for _ in range(K)]
        ev_down = [torch.cuda.Event() for _ in range(K)]
        for i in range(K):
            b = i % 2
            with torch.cuda.stream(s_up):
                if i >= 2:
                    s_up.wait_event(ev_comp[i - 2])          # x_dev[b] free again
                x_dev[b].copy_(x_host, non_blocking=True)
                ev_up[i].record(s_up)
            comp.wait_event(ev_up[i])
            if i >= 2:
                comp.wait_event(ev_down[i - 2])              # y_dev[b] read out
            a = list(fwd_args)
            a[1] = x_dev[b]
            a[13] = y_dev[b]
            B.forward(*a, stream=comp)
            ev_comp[i].record(comp)
            with torch.cuda.stream(s_down):
                s_down.wait_event(ev_comp[i])
                y_host[b].copy_(y_dev[b], non_blocking=True)
                ev_down[i].record(s_down)
        return ev_down[-1]

    last = run(max(2, args.warmup))
    last.synchronize()
    K = args.steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize(dev)
    start.record(s_up)
    comp.wait_event(start)
    s_down.wait_event(start)
    last = run(K)
    end.record(s_down)  # after the last download in s_down's order
    torch.cuda.synchronize(dev)
    dist.barrier()
    ms = dist.max(start.elapsed_time(end) / K)
    return {"value": dist.world * cfg.T / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
            "h2d_bytes_per_step": x_host.numel() * x_host.element_size(),
            "d2h_bytes_per_step": y_host[0].numel() * y_host[0].element_size(),
            "note": "copies of step i+1 (upload) and i-1 (download) overlap step i's compute"}


def run_cpu_baseline(args, w, cfg):
    S = min(args.cpu_sample, cfg.T)
    rng = np.random.default_rng(cfg.seed)
    toks = np.sort(rng.choice(cfg.T, size=S, replace=False))
    spent, _ = oracle_sample(w, toks)
    return {"value": S / spent, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{S} random tokens of the {cfg.name} workload through the whole layer (fp64 oracle: "
                      f"routing, every selected expert, shared expert; {spent:.1f} s)"}


def main():
    args = parse_args()
    dist = Dist()
    try:
        if args.impl == "reference":
            run_reference(args, dist)
        elif args.ep_size > 1:
            run_ep(args, dist)
        else:
            run_ours(args, dist)
    finally:
        dist.close()


if __name__ == "__main__":
    main()
