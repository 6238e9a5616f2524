"""Seeded synthetic workloads for the MoE feed-forward layer.

This module only draws inputs: shapes, seeds and value distributions of the
five workloads (tiny CPU-scale layer, DeepSeek-V3 decode / prefill / skewed /
group-routed FP8 layers).  It contains none of the layer's arithmetic (no gate,
routing, dispatch, expert or combine step), so both the fp64 oracle and the
CUDA library can consume what it produces.

Shapes follow the pages: d = 7168, moe_inter = 2048, 256 routed experts with
top-8 plus one shared expert of n_shared x moe_inter = 2048 features
("DeepSeek-V3.2-Exp / Mixture of experts / Shared expert", parameter table:
3 x 7168 x 2048 = 44,040,192 per expert; n4n.ai page, "The architecture in one
diagram": 256 routed experts, top-8, one shared expert).

Weight layout is the math orientation of the SwiGLU equations (g = x W1):
W1, W3 are [E, d, inter] and W2 is [E, inter, d], row-major.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

# Zipf bias strength of the skewed workload: the value for which the 10% most
# loaded experts receive 50% of the T*k assignments (top-8 routing over 256
# experts, popularity ranks ~ Zipf(1.1)).  Written by
# tests/golden/calibrate_zipf_beta.py, which bisects it with the fp64 oracle's
# router; tests/test_workloads.py re-checks the share at this value.
ZIPF_BETA = 0.4125
ZIPF_S = 1.1
ZIPF_X_SHIFT = 4.0  # x_t = RMSnorm(z_t + 4 u): x_t . u is about 4 for every token


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    T: int
    d: int
    E: int
    k: int
    inter: int
    shared_inter: int
    route: int            # 0: top-k then softmax over the k;  1: sigmoid group-limited
    w_std: float
    seed: int
    n_group: int = 1
    topk_group: int = 1
    group_topn: int = 2
    route_scale: float = 1.0
    fp8: bool = False     # routed expert weights stored as e4m3 + 128x128 fp32 block scales
    bias_std: float = 0.0
    zipf: bool = False
    master_f32: bool = False  # tiny: fp32 masters, bf16-rounded copies for the device

    def replace(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)

    # FLOPs the layer must do per token: router + (k routed + shared) SwiGLU experts
    def flops_per_token(self) -> int:
        return 2 * self.d * self.E + self.k * 6 * self.d * self.inter + 6 * self.d * self.shared_inter


CONFIGS = {
    "tiny": Config("tiny", T=128, d=512, E=32, k=4, inter=256, shared_inter=256, route=0,
                   w_std=0.02, seed=1701, master_f32=True),
    "decode": Config("decode", T=64, d=7168, E=256, k=8, inter=2048, shared_inter=2048, route=0,
                     w_std=0.006, seed=1702),
    "prefill": Config("prefill", T=4096, d=7168, E=256, k=8, inter=2048, shared_inter=2048, route=0,
                      w_std=0.006, seed=1703),
    "skewed": Config("skewed", T=16384, d=7168, E=256, k=8, inter=2048, shared_inter=2048, route=0,
                     w_std=0.006, seed=1704, zipf=True),
    "fp8": Config("fp8", T=8192, d=7168, E=256, k=8, inter=2048, shared_inter=2048, route=1,
                  w_std=0.006, seed=1705, n_group=8, topk_group=4, group_topn=2, route_scale=2.5,
                  fp8=True, bias_std=0.01),
}

FP8_BLOCK = 128
E4M3_MAX = 448.0


@dataclasses.dataclass
class Workload:
    cfg: Config
    x: torch.Tensor                  # [T, d] bf16
    Wg: torch.Tensor                 # [E, d] bf16
    W1: torch.Tensor                 # [E, d, I] bf16, or uint8 e4m3 codes when cfg.fp8
    W3: torch.Tensor
    W2: torch.Tensor                 # [E, I, d]
    W1s: Optional[torch.Tensor]      # [d, Is] bf16 (shared expert)
    W3s: Optional[torch.Tensor]
    W2s: Optional[torch.Tensor]      # [Is, d]
    bias: Optional[torch.Tensor] = None   # [E] fp32 selection bias (group routing)
    s1: Optional[torch.Tensor] = None     # [E, d/128, I/128] fp32 block scales (fp8)
    s3: Optional[torch.Tensor] = None
    s2: Optional[torch.Tensor] = None     # [E, I/128, d/128]
    masters: Optional[dict] = None        # fp32 masters (tiny workload only)


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _rms_normalise(z: torch.Tensor) -> torch.Tensor:
    # x_t = z_t / sqrt(mean_j z_tj^2): no epsilon, no gain (input recipe)
    return z / torch.sqrt(torch.mean(z * z, dim=1, keepdim=True))


def quantise_e4m3_blocks(w: torch.Tensor, blk: int = FP8_BLOCK):
    """Input preparation for the FP8 workload: per (blk x blk) block of a
    [rows, cols] fp32 matrix, scale = amax/448 (1 when the block is all zero),
    code = round-to-nearest-even(w / scale) in e4m3.  Returns (uint8 codes,
    fp32 scales [rows/blk, cols/blk])."""
    rows, cols = w.shape
    wb = w.reshape(rows // blk, blk, cols // blk, blk)
    amax = wb.abs().amax(dim=(1, 3))
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    q = (wb / scale[:, None, :, None]).reshape(rows, cols)
    q = q.clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
    return q.view(torch.uint8), scale.to(torch.float32)


def _zipf_parts(cfg, randn, g, dev):
    """Skewed-load recipe: x_t = RMSnorm(z_t + 4 u) for a random unit vector u,
    popularity ranks pi(e) a random permutation of 1..E with p_e ~ pi(e)^-1.1,
    and Wg = G + beta V with G ~ N(0, 1/d) and V_e = log(p_e / p_max) u / 4,
    so the logit of expert e carries a bias of about beta log(p_e / p_max)."""
    d, E = cfg.d, cfg.E
    u = randn(d)
    u = u / torch.linalg.vector_norm(u)
    x32 = _rms_normalise(randn(cfg.T, d) + ZIPF_X_SHIFT * u[None, :])
    ranks = torch.randperm(E, generator=g, device=dev).to(torch.float32) + 1.0
    logp = -ZIPF_S * torch.log(ranks)
    logp = logp - logp.max()
    G = randn(E, d) / math.sqrt(d)
    V = (logp / ZIPF_X_SHIFT)[:, None] * u[None, :]
    return x32, G, V


def zipf_parts(cfg, device="cpu"):
    """(x bf16, G fp32, V fp32) of the skewed recipe, with the same draws as make()."""
    if isinstance(cfg, str):
        cfg = CONFIGS[cfg]
    dev = torch.device(device)
    g = _gen(dev, cfg.seed)

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=dev, dtype=torch.float32)

    x32, G, V = _zipf_parts(cfg, randn, g, dev)
    return x32.to(torch.bfloat16), G, V


def make(cfg, device="cpu", T: Optional[int] = None, expert_chunk: int = 8) -> Workload:
    """Draw the workload `cfg` (a Config or a name) on `device`."""
    if isinstance(cfg, str):
        cfg = CONFIGS[cfg]
    if T is not None:
        cfg = cfg.replace(T=T)
    dev = torch.device(device)
    g = _gen(dev, cfg.seed)
    T_, d, E, I, Is = cfg.T, cfg.d, cfg.E, cfg.inter, cfg.shared_inter

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=dev, dtype=torch.float32)

    if cfg.zipf:
        x32, G, V = _zipf_parts(cfg, randn, g, dev)
        Wg32 = G + ZIPF_BETA * V
    else:
        x32 = _rms_normalise(randn(T_, d))
        Wg32 = randn(E, d) / math.sqrt(d)

    bias = None
    if cfg.bias_std > 0:
        bias = randn(E) * cfg.bias_std

    masters = None
    if cfg.master_f32:
        W1_32 = randn(E, d, I) * cfg.w_std
        W3_32 = randn(E, d, I) * cfg.w_std
        W2_32 = randn(E, I, d) * cfg.w_std
        W1s_32 = randn(d, Is) * cfg.w_std
        W3s_32 = randn(d, Is) * cfg.w_std
        W2s_32 = randn(Is, d) * cfg.w_std
        masters = dict(x=x32, Wg=Wg32, W1=W1_32, W3=W3_32, W2=W2_32, W1s=W1s_32, W3s=W3s_32, W2s=W2s_32)
        bf = lambda a: a.to(torch.bfloat16)
        return Workload(cfg, bf(x32), bf(Wg32), bf(W1_32), bf(W3_32), bf(W2_32),
                        bf(W1s_32), bf(W3s_32), bf(W2s_32), bias=bias, masters=masters)

    wdt = torch.uint8 if cfg.fp8 else torch.bfloat16
    W1 = torch.empty(E, d, I, dtype=wdt, device=dev)
    W3 = torch.empty(E, d, I, dtype=wdt, device=dev)
    W2 = torch.empty(E, I, d, dtype=wdt, device=dev)
    s1 = s3 = s2 = None
    if cfg.fp8:
        s1 = torch.empty(E, d // FP8_BLOCK, I // FP8_BLOCK, dtype=torch.float32, device=dev)
        s3 = torch.empty_like(s1)
        s2 = torch.empty(E, I // FP8_BLOCK, d // FP8_BLOCK, dtype=torch.float32, device=dev)
    for e0 in range(0, E, expert_chunk):
        e1 = min(E, e0 + expert_chunk)
        for W, S, shape in ((W1, s1, (d, I)), (W3, s3, (d, I)), (W2, s2, (I, d))):
            w = randn(e1 - e0, *shape) * cfg.w_std
            if cfg.fp8:
                for e in range(e0, e1):
                    q, sc = quantise_e4m3_blocks(w[e - e0])
                    W[e].copy_(q)
                    S[e].copy_(sc)
            else:
                W[e0:e1].copy_(w.to(torch.bfloat16))
            del w
    W1s = (randn(d, Is) * cfg.w_std).to(torch.bfloat16)
    W3s = (randn(d, Is) * cfg.w_std).to(torch.bfloat16)
    W2s = (randn(Is, d) * cfg.w_std).to(torch.bfloat16)
    return Workload(cfg, x32.to(torch.bfloat16), Wg32.to(torch.bfloat16), W1, W3, W2, W1s, W3s, W2s,
                    bias=bias, s1=s1, s3=s3, s2=s2)


def make_small(name: str, device="cpu", **shape) -> Workload:
    """A workload with the distributions of `name` but other sizes (tests)."""
    cfg = CONFIGS[name].replace(**shape)
    return make(cfg, device=device)
