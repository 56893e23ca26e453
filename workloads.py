"""Seeded synthetic inputs for the MACaQ W4A4 linear layer.

This module is the one place both the CUDA path's tests/benchmark and the CPU oracle get
their inputs from.  It holds none of the method's arithmetic (no scaling, transform or
quantisation): only random draws, outlier-channel selection and the calibration of the
per-channel scale s that the pages leave to the user.

Shapes follow the linear layers the pages' throughput claims are about ("MACaQ ...",
Abstract: Llama-3-8B perplexity, Qwen3-32B end-to-end overhead in vLLM).  There is no
dataset and no trained weight; every tensor is drawn from a seeded ``torch.Generator`` on
the CPU, so the same seed gives the same bits on any machine:

    seed = 1000 * config + 16 * layer + tensor_id,
    tensor_id: 0 = activations x, 1 = weights W, 2 = calibration batch, 3 = outlier channels.

Recipe per workload (x is drawn in fp32 and rounded to bf16, W stays fp32):

  tiny      M=16 K=256 N=128        x ~ N(0,1), channels 3 and 77 times 40;  W ~ N(0, 0.02)
  llama_up  M=2048 K=4096 N=14336   x ~ N(0,1), round(1% K) random channels times 50;  W ~ N(0, 0.02)
  qwen_up   M in {1,4,16} K=5120 N=25600
                                    x ~ Student-t(nu=4), round(0.5% K) channels times 30; W ~ N(0, 0.02)
  qwen_down M=4096 K=25600 N=5120   x = SiLU(g) * u, g, u ~ N(0,1) (heavy tail, no extra outliers);
                                    W ~ N(0, 0.014)
  qwen_stack  64 layers x {q, k, v, o, gate, up, down} with x as in llama_up, W ~ N(0, 0.02)

Calibration of s (all workloads): a separate 64-token batch x_cal from the same
distribution (same outlier channels) and s_j = sqrt(max_r |x_cal[r,j]| / max_n |W[n,j]|)
in fp64, rounded to fp32 -- the SmoothQuant alpha = 1/2 balance.
"""
from __future__ import annotations

import dataclasses
import math

import torch

CALIB_TOKENS = 64

QWEN_STACK_LAYERS = 64
# (name, in_features K, out_features N) of one Qwen3-32B-shaped decoder layer
QWEN_STACK_LINEARS = (
    ("q", 5120, 8192),
    ("k", 5120, 1024),
    ("v", 5120, 1024),
    ("o", 8192, 5120),
    ("gate", 5120, 25600),
    ("up", 5120, 25600),
    ("down", 25600, 5120),
)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    config: int
    M: int
    K: int
    N: int
    x_kind: str  # "normal" | "student_t" | "gated"
    outlier_frac: float = 0.0
    outlier_gain: float = 1.0
    fixed_outliers: tuple = ()
    w_std: float = 0.02
    layer: int = 0

    @property
    def flops(self) -> float:
        return 2.0 * self.M * self.N * self.K

    def with_m(self, M: int) -> "Workload":
        return dataclasses.replace(self, M=M)


TINY = Workload("tiny", 1, 16, 256, 128, "normal", fixed_outliers=(3, 77), outlier_gain=40.0)
LLAMA_UP = Workload("llama3_8b_up_prefill", 2, 2048, 4096, 14336, "normal", 0.01, 50.0)
QWEN_UP_DECODE = Workload("qwen3_32b_up_decode", 3, 16, 5120, 25600, "student_t", 0.005, 30.0)
QWEN_DOWN = Workload("qwen3_32b_down_prefill", 4, 4096, 25600, 5120, "gated", w_std=0.014)
QWEN_DECODE_M = (1, 4, 16)
STACK_M = (1, 32, 512, 4096)

ALL = (TINY, LLAMA_UP, QWEN_UP_DECODE, QWEN_DOWN)


def stack_layer(layer: int, linear: str, M: int) -> Workload:
    """One linear of the 64-layer Qwen3-32B-shaped stack; x drawn as in llama_up."""
    for idx, (name, K, N) in enumerate(QWEN_STACK_LINEARS):
        if name == linear:
            # one seed slot per (layer, linear): layer index 7*layer + idx
            return Workload(f"qwen3_32b_stack_L{layer}_{name}", 5, M, K, N, "normal", 0.01, 50.0,
                            layer=7 * layer + idx)
    raise KeyError(linear)


# Mixture-of-experts linears (the pages name MoE models among the method's targets but give no
# shapes): Qwen3-MoE-like experts, 128 experts of hidden 2048 / expert width 768, top-8 routing.
MOE_EXPERTS = 128
MOE_TOPK = 8
MOE_LINEARS = (("up", 2048, 768), ("down", 768, 2048))


def moe_counts(tokens: int, experts: int = MOE_EXPERTS, topk: int = MOE_TOPK, seed_: int = 6000) -> list:
    """Tokens routed to each expert: every token picks `topk` distinct experts, with popularity
    skewed like a learned router (Zipf-like weights 1/(rank+1) in a seeded random expert order)."""
    g = _gen(seed_)
    w = 1.0 / torch.arange(1, experts + 1, dtype=torch.float64)
    w = w[torch.randperm(experts, generator=g)]
    picks = torch.multinomial(w.expand(tokens, experts), topk, replacement=False, generator=g)
    return torch.bincount(picks.reshape(-1), minlength=experts).tolist()


def seed(cfg: int, layer: int, tensor_id: int) -> int:
    return 1000 * cfg + 16 * layer + tensor_id


def _gen(s: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(s)
    return g


def outlier_channels(w: Workload) -> torch.Tensor:
    """Indices of the channels whose activations carry the outlier gain."""
    if w.fixed_outliers:
        return torch.tensor(w.fixed_outliers, dtype=torch.int64)
    n = int(round(w.outlier_frac * w.K))
    if n == 0:
        return torch.zeros(0, dtype=torch.int64)
    perm = torch.randperm(w.K, generator=_gen(seed(w.config, w.layer, 3)))
    return perm[:n].sort().values


def _draw_x(w: Workload, rows: int, tensor_id: int) -> torch.Tensor:
    g = _gen(seed(w.config, w.layer, tensor_id))
    K = w.K
    if w.x_kind == "normal":
        x = torch.randn(rows, K, generator=g, dtype=torch.float32)
    elif w.x_kind == "student_t":
        # Student-t with nu = 4: Z / sqrt(V / 4), V a chi-square with 4 degrees of freedom
        z = torch.randn(rows, K, generator=g, dtype=torch.float32)
        v = torch.randn(4, rows, K, generator=g, dtype=torch.float32).square().sum(0)
        x = z / torch.sqrt(v / 4.0)
    elif w.x_kind == "gated":
        gate = torch.randn(rows, K, generator=g, dtype=torch.float32)
        up = torch.randn(rows, K, generator=g, dtype=torch.float32)
        x = torch.nn.functional.silu(gate) * up
    else:
        raise ValueError(w.x_kind)
    ch = outlier_channels(w)
    if ch.numel():
        x[:, ch] *= w.outlier_gain
    return x


def make_x(w: Workload, M: int | None = None) -> torch.Tensor:
    """Activations, bf16 [M, K] on the CPU (fp32 draw rounded to nearest-even bf16)."""
    return _draw_x(w, w.M if M is None else M, 0).to(torch.bfloat16)


def make_w(w: Workload) -> torch.Tensor:
    """Weights, fp32 [N, K] on the CPU (nn.Linear layout, y = x W^T)."""
    g = _gen(seed(w.config, w.layer, 1))
    return torch.randn(w.N, w.K, generator=g, dtype=torch.float32) * w.w_std


def _gen_device(s: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(s)
    return g


def make_w_device(w: Workload, device) -> torch.Tensor:
    """Weights drawn on the device: same seed and distribution as make_w, other values (the
    device generator's stream).  For timing stacks whose host draw would take minutes."""
    g = _gen_device(seed(w.config, w.layer, 1), device)
    return torch.randn(w.N, w.K, generator=g, dtype=torch.float32, device=device) * w.w_std


def make_x_device(w: Workload, rows: int, device, tensor_id: int = 0) -> torch.Tensor:
    """Activations drawn on the device (normal kind, the workload's outlier channels and gain),
    bf16 [rows, K]; tensor_id 2 gives the calibration batch."""
    if w.x_kind != "normal":
        raise ValueError("device draws cover the normal activation kind")
    g = _gen_device(seed(w.config, w.layer, tensor_id), device)
    x = torch.randn(rows, w.K, generator=g, dtype=torch.float32, device=device)
    ch = outlier_channels(w).to(device)
    if ch.numel():
        x[:, ch] *= w.outlier_gain
    return x.to(torch.bfloat16)


def make_xcal(w: Workload) -> torch.Tensor:
    """The separate 64-token bf16 calibration batch of a workload (same distribution as x)."""
    return _draw_x(w, CALIB_TOKENS, 2).to(torch.bfloat16)


def make_s(w: Workload, W: torch.Tensor | None = None) -> torch.Tensor:
    """Per-channel scale s (fp32 [K], > 0) from a separate 64-token calibration batch."""
    if W is None:
        W = make_w(w)
    xcal = make_xcal(w).to(torch.float64)
    xmax = xcal.abs().amax(0)
    wmax = W.to(torch.float64).abs().amax(0)
    s = torch.sqrt(xmax / wmax)
    return s.to(torch.float32)


def alg_bytes(w: Workload) -> float:
    """Bytes the fused linear must move: bf16 x, MXFP4 W (codes + E8M0), bf16 y, fp32 multiplier."""
    return 2.0 * w.M * w.K + w.N * w.K * (0.5 + 1.0 / 32.0) + 2.0 * w.M * w.N + 4.0 * w.K


def describe() -> dict:
    return {wl.name: dataclasses.asdict(wl) for wl in ALL}


if __name__ == "__main__":  # pragma: no cover
    for wl in ALL:
        print(wl.name, wl.M, wl.K, wl.N, f"{wl.flops:.3e} flop", f"{alg_bytes(wl)/1e6:.2f} MB")
    print("stack layer params:", sum(K * N for _, K, N in QWEN_STACK_LINEARS) / 1e6, "M")
    print("1/sqrt(32) =", 1 / math.sqrt(32))
