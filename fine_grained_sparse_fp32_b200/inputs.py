"""Seeded synthetic inputs for the fine-grained MoE layer.

This module only draws random numbers and lays them out; it holds none of the
layer's arithmetic. Both the CUDA path and the CPU oracle are fed from it.

Shapes follow "Inside Kolibri 1" (flozi.net), section "Routing: selection bias
and mixture weights are separate": a 2560-wide residual stream, 384 routed
micro-experts plus one shared expert, top-6, and SwiGLU experts made of two
2560->512 projections and one 512->2560 projection. The FP8 weight format
follows the same page, section "The FP8 path is explicitly mixed precision":
E4M3 values in 128x128 blocks, one FP32 scale per block.

Draw order (one torch.Generator on the target device, seeded once):
  x, router weight (drawn [d, E], stored transposed as [E, d]), correction
  bias, then the shared expert (gate, up, down), then routed experts
  e = 0..E-1 (gate, up, down).
Distributions: x ~ N(0, 1); every weight ~ N(0, 0.02); bias ~ U(-0.1, 0.1).
Weights are drawn in FP32 and then cast to BF16, or quantised to E4M3 with
scale = amax(block) / 448 (FP32, never rounded to a power of two) and
q = round-to-nearest-even(w / scale), saturated to +-448.

Layout of the returned expert tensors: index 0..E-1 are the routed experts,
index E is the shared expert, so one allocation holds all E+1 experts.
  w_gate, w_up : [E+1, I, d]   (row i of expert e is output feature i; K-major)
  w_down       : [E+1, d, I]
  s_gate, s_up : [E+1, I/128, d/128]  FP32 block scales (E4M3 only)
  s_down       : [E+1, d/128, I/128]
"""
from __future__ import annotations

from dataclasses import dataclass, replace
import torch

E4M3_MAX = 448.0
FP8_BLOCK = 128


@dataclass(frozen=True)
class LayerConfig:
    name: str
    N: int          # tokens
    d: int          # residual width
    E: int          # routed experts
    K: int          # experts selected per token
    I: int          # SwiGLU intermediate width of one expert
    x_dtype: str    # "f32" | "bf16"
    w_dtype: str    # "f32" | "bf16" | "e4m3" | "e4m3_a8" (E4M3 weights, FP8 activations in the expert GEMMs)
    skew: bool = False   # Zipf expert popularity added to the correction bias

    @property
    def fp8_weights(self) -> bool:
        """E4M3 weights with FP32 128 x 128 block scales (BF16 or FP8 activations)."""
        return self.w_dtype in ("e4m3", "e4m3_a8")

    @property
    def expert_weights(self) -> int:
        """Matrix weights of one expert: gate + up + down."""
        return 3 * self.d * self.I

    def with_tokens(self, N: int) -> "LayerConfig":
        return replace(self, N=N)


# The six workloads. "tiny" is small enough for the oracle to run every token
# in well under a second; the rest use the Kolibri-1 layer shape.
CONFIGS = {
    "tiny": LayerConfig("tiny", 128, 512, 64, 6, 128, "f32", "f32"),
    "decode": LayerConfig("decode", 32, 2560, 384, 6, 512, "bf16", "bf16"),
    "prefill": LayerConfig("prefill", 8192, 2560, 384, 6, 512, "bf16", "bf16"),
    "fp8_decode": LayerConfig("fp8_decode", 32, 2560, 384, 6, 512, "bf16", "e4m3"),
    "fp8_prefill": LayerConfig("fp8_prefill", 4096, 2560, 384, 6, 512, "bf16", "e4m3"),
    # the same layers with FP8 activations in the expert GEMMs ("Inside Kolibri 1", FP8 section)
    "fp8a8_decode": LayerConfig("fp8a8_decode", 32, 2560, 384, 6, 512, "bf16", "e4m3_a8"),
    "fp8a8_prefill": LayerConfig("fp8a8_prefill", 4096, 2560, 384, 6, 512, "bf16", "e4m3_a8"),
    "skew": LayerConfig("skew", 65536, 2560, 384, 6, 512, "bf16", "bf16", skew=True),
}

# Skewed-routing recipe: experts are ranked by a seeded permutation, and the
# correction bias of the expert of rank r (1-based) gets -SKEW_BETA * 1.1 * ln(r)
# added (a Zipf s=1.1 popularity on the logit scale); SKEW_EMPTY experts get a
# bias of -30 so that they receive no token at all. SKEW_BETA was found by
# bisection so that the 38 most popular experts (10%) receive half of all
# routed slots, on logits modelled as independent N(0, d * 0.02^2) per token
# and expert (x ~ N(0, 1) against router rows ~ N(0, 0.02), d = 2560), top-6
# of logits + bias over 40,000 tokens.
SKEW_BETA = 0.34
SKEW_EMPTY = 20


_TORCH_DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


def _quantise_e4m3(w: torch.Tensor):
    """Block-quantise a [rows, cols] FP32 matrix into E4M3 bits + FP32 scales."""
    rows, cols = w.shape
    rb, cb = rows // FP8_BLOCK, cols // FP8_BLOCK
    blocks = w.reshape(rb, FP8_BLOCK, cb, FP8_BLOCK)
    amax = blocks.abs().amax(dim=(1, 3))                      # [rb, cb]
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    q = (blocks / scale[:, None, :, None]).clamp_(-E4M3_MAX, E4M3_MAX)
    q = q.to(torch.float8_e4m3fn).view(torch.uint8).reshape(rows, cols)
    return q, scale.to(torch.float32)


def make_inputs(cfg: LayerConfig, seed: int = 0, device: str | torch.device = "cpu") -> dict:
    """Draw one layer's inputs and weights for `cfg` on `device`."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    N, d, E, I = cfg.N, cfg.d, cfg.E, cfg.I

    def normal(shape, std):
        return torch.empty(shape, device=dev, dtype=torch.float32).normal_(0.0, std, generator=gen)

    out: dict = {"cfg": cfg, "seed": seed}
    x = normal((N, d), 1.0)
    out["x"] = x.to(_TORCH_DTYPES[cfg.x_dtype])
    out["w_router"] = normal((d, E), 0.02).t().contiguous()
    bias = torch.empty(E, device=dev, dtype=torch.float32).uniform_(-0.1, 0.1, generator=gen)

    G = E + 1
    if cfg.fp8_weights:
        w_gate = torch.empty((G, I, d), device=dev, dtype=torch.uint8)
        w_up = torch.empty((G, I, d), device=dev, dtype=torch.uint8)
        w_down = torch.empty((G, d, I), device=dev, dtype=torch.uint8)
        s_gate = torch.empty((G, I // FP8_BLOCK, d // FP8_BLOCK), device=dev, dtype=torch.float32)
        s_up = torch.empty_like(s_gate)
        s_down = torch.empty((G, d // FP8_BLOCK, I // FP8_BLOCK), device=dev, dtype=torch.float32)
    else:
        wt = _TORCH_DTYPES[cfg.w_dtype]
        w_gate = torch.empty((G, I, d), device=dev, dtype=wt)
        w_up = torch.empty((G, I, d), device=dev, dtype=wt)
        w_down = torch.empty((G, d, I), device=dev, dtype=wt)

    # shared expert first (stored at index E), then routed experts 0..E-1
    for e in [E] + list(range(E)):
        g_, u_, d_ = normal((I, d), 0.02), normal((I, d), 0.02), normal((d, I), 0.02)
        if cfg.fp8_weights:
            w_gate[e], s_gate[e] = _quantise_e4m3(g_)
            w_up[e], s_up[e] = _quantise_e4m3(u_)
            w_down[e], s_down[e] = _quantise_e4m3(d_)
        else:
            w_gate[e].copy_(g_)
            w_up[e].copy_(u_)
            w_down[e].copy_(d_)
    out.update(w_gate=w_gate, w_up=w_up, w_down=w_down)
    if cfg.fp8_weights:
        out.update(s_gate=s_gate, s_up=s_up, s_down=s_down)

    if cfg.skew:
        rank = torch.randperm(E, generator=gen, device=dev).to(torch.float32) + 1.0
        bias = bias - SKEW_BETA * 1.1 * torch.log(rank)
        empty = torch.randperm(E, generator=gen, device=dev)[:SKEW_EMPTY]
        bias[empty] = -30.0
    out["bias"] = bias
    return out


def make_x(cfg: LayerConfig, seed: int, device="cpu") -> torch.Tensor:
    """A fresh token batch of the same distribution (used to rotate inputs)."""
    gen = torch.Generator(device=torch.device(device))
    gen.manual_seed(seed)
    x = torch.empty((cfg.N, cfg.d), device=device, dtype=torch.float32).normal_(0.0, 1.0, generator=gen)
    return x.to(_TORCH_DTYPES[cfg.x_dtype])


def make_block_inputs(cfg: LayerConfig, seed: int, device="cpu") -> dict:
    """Residual stream and norm gains of the sandwich block around the layer.

    One generator seeded with `seed`; draw order h, gamma_pre, gamma_post.
    h ~ N(0, 2) (a residual stream that has grown past unit scale); each gain
    ~ 1 + N(0, 0.1), the spread of trained RMSNorm gains around their
    initial value 1. All three in BF16: h [N, d], gains [d]."""
    gen = torch.Generator(device=torch.device(device))
    gen.manual_seed(seed)
    d = cfg.d
    h = torch.empty((cfg.N, d), device=device, dtype=torch.float32).normal_(0.0, 2.0, generator=gen)
    g_pre = torch.empty(d, device=device, dtype=torch.float32).normal_(1.0, 0.1, generator=gen)
    g_post = torch.empty(d, device=device, dtype=torch.float32).normal_(1.0, 0.1, generator=gen)
    return {"h": h.to(torch.bfloat16), "gamma_pre": g_pre.to(torch.bfloat16),
            "gamma_post": g_post.to(torch.bfloat16)}


def expected_distinct_experts(cfg: LayerConfig) -> float:
    """Mean number of distinct routed experts hit by N uniform top-K draws."""
    return cfg.E * (1.0 - (1.0 - cfg.K / cfg.E) ** cfg.N)


def to_host(inputs: dict) -> dict:
    """Copy every tensor to host memory (contiguous), keeping non-tensors."""
    return {k: (v.detach().to("cpu").contiguous() if torch.is_tensor(v) else v) for k, v in inputs.items()}


__all__ = ["LayerConfig", "CONFIGS", "make_inputs", "make_x", "make_block_inputs", "to_host",
           "expected_distinct_experts", "E4M3_MAX", "FP8_BLOCK", "SKEW_BETA", "SKEW_EMPTY"]
