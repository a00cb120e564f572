"""Seeded synthetic workloads for the QUADS rollout hot path.

This module only draws random numbers and arranges them into the shapes of
the five layer configurations; it holds none of the method's arithmetic and
is the one module both the CUDA path's tests/bench and the oracle's tests
read inputs from.

The pages (QUADS: gist.science/it section 4) train a 25B-parameter MoE with
2.8B active parameters; no weights, activations or datasets are available, so
every tensor here is synthetic: activations N(0,1) with a few heavy outlier
channels (the high-residual channels that Residual Activation Compensation
targets, gist.science/it section 2.2 B), router logits N(0,1) (plus a
per-expert bias for the skewed configuration) and weights N(0, 0.02).

All draws use ``torch.Generator`` seeded from (seed, tensor id); bf16 tensors
are the fp32 draws rounded to nearest bf16 by torch.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    tokens: int          # T
    hidden: int          # H
    inter: int           # I (expert intermediate); dense: output features
    experts: int         # E (1 = dense layer)
    topk: int            # k_r routed experts per token
    rac_k: int           # RAC channels per GEMM input
    outlier_channels: int
    outlier_mode: str    # "x20" or "lognormal"
    expert_bias: bool    # per-expert router logit bias N(0,1) (routing skew)
    w4a16: bool = False  # trainer-side QDQ + BF16 GEMM workload

    @property
    def dense(self) -> bool:
        return self.experts == 1 and self.topk == 1


CONFIGS = {
    # single dense layer: X [64 x 256], W [256 x 256], k = 8
    "dense_64x256": LayerConfig("dense_64x256", 64, 256, 256, 1, 1, 8, 4, "x20", False),
    # small MoE FFN: T=512, H=2048, I=768, E=8, top-2, k = 32
    "moe_t512_e8": LayerConfig("moe_t512_e8", 512, 2048, 768, 8, 2, 32,
                               round(0.01 * 2048), "lognormal", False),
    # rollout-prefill MoE layer: T=4096, H=2048, I=768, E=128, top-8, k = 64
    "moe_t4096_e128": LayerConfig("moe_t4096_e128", 4096, 2048, 768, 128, 8, 64,
                                  round(0.01 * 2048), "lognormal", False),
    # trainer-side asymmetric QAT: QDQ of 128 x (W13 [1536x2048] + W2 [2048x768]),
    # then the BF16 grouped GEMM at T=4096 top-8
    "qat_w4a16_e128": LayerConfig("qat_w4a16_e128", 4096, 2048, 768, 128, 8, 0, 0,
                                  "none", False, w4a16=True),
    # large MoE layer: T=16384, H=4096, I=1536, E=128, top-8 with skew, k = 128
    "moe_t16384_e128": LayerConfig("moe_t16384_e128", 16384, 4096, 1536, 128, 8, 128,
                                   round(0.01 * 4096), "lognormal", True),
    # the large layer's shapes per expert (H=4096, I=1536, ~1024 routed rows
    # per expert, k = 128) with 32 experts: small enough for detailed profiler
    # captures (NVFP4 weights 340 MB, a few GB on the device)
    "moe_t4096_h4096_e32": LayerConfig("moe_t4096_h4096_e32", 4096, 4096, 1536, 32, 8, 128,
                                       round(0.01 * 4096), "lognormal", True),
}

CONFIG_ORDER = ["dense_64x256", "moe_t512_e8", "moe_t4096_e128", "qat_w4a16_e128",
                "moe_t16384_e128"]


def _gen(seed: int, tensor_id: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1000003 + tensor_id * 7919) & 0x7FFFFFFFFFFFFFFF)
    return g


def activations(cfg: LayerConfig, seed: int, device="cpu", tokens: int | None = None) -> torch.Tensor:
    """X bf16 [T x H]: N(0,1) with ``outlier_channels`` channels scaled by 20
    (dense config) or by one LogNormal(mu=2, sigma=0.5) draw per channel."""
    T = cfg.tokens if tokens is None else tokens
    g = _gen(seed, 1, device)
    x = torch.randn(T, cfg.hidden, generator=g, device=device, dtype=torch.float32)
    if cfg.outlier_channels:
        gc = _gen(seed, 2, "cpu")
        ch = torch.randperm(cfg.hidden, generator=gc)[: cfg.outlier_channels]
        if cfg.outlier_mode == "x20":
            scale = torch.full((cfg.outlier_channels,), 20.0)
        else:
            scale = torch.exp(2.0 + 0.5 * torch.randn(cfg.outlier_channels, generator=gc))
        x[:, ch.to(device)] *= scale.to(device)
    return x.to(torch.bfloat16)


def router_logits(cfg: LayerConfig, seed: int, device="cpu", tokens: int | None = None) -> torch.Tensor:
    """Router logits fp32 [T x E]: N(0,1), plus a per-expert N(0,1) bias for
    the skewed configuration."""
    T = cfg.tokens if tokens is None else tokens
    g = _gen(seed, 3, device)
    logits = torch.randn(T, cfg.experts, generator=g, device=device, dtype=torch.float32)
    if cfg.expert_bias:
        gb = _gen(seed, 4, "cpu")
        logits += torch.randn(cfg.experts, generator=gb).to(device)
    return logits


def weights(cfg: LayerConfig, seed: int, device="cpu"):
    """Expert weights, bf16, N(0, 0.02), stored [out x in] (K-major rows):
    W13 [E x 2I x H] (gate rows [0, I), up rows [I, 2I)) and W2 [E x H x I].
    The dense configuration returns (W [1 x I x H], None)."""
    g = _gen(seed, 5, device)
    if cfg.dense:
        w = torch.randn(1, cfg.inter, cfg.hidden, generator=g, device=device) * 0.02
        return w.to(torch.bfloat16), None
    E, H, I = cfg.experts, cfg.hidden, cfg.inter
    w13 = torch.empty(E, 2 * I, H, dtype=torch.bfloat16, device=device)
    w2 = torch.empty(E, H, I, dtype=torch.bfloat16, device=device)
    for e in range(E):
        w13[e] = (torch.randn(2 * I, H, generator=g, device=device) * 0.02).to(torch.bfloat16)
        w2[e] = (torch.randn(H, I, generator=g, device=device) * 0.02).to(torch.bfloat16)
    return w13, w2


# Layer-error sweep (one dense layer): outlier strength alpha scales a fixed
# 1% of the input channels; RAC channel counts as percentages of K.
SWEEP = {"tokens": 4096, "channels": 4096, "out": 4096, "outlier_frac": 0.01,
         "alphas": (1.0, 5.0, 20.0, 50.0), "percents": (0, 1, 2, 5, 10, 25, 50, 100)}


def outlier_activations(tokens: int, channels: int, alpha: float, seed: int, frac: float = 0.01,
                        device="cpu") -> torch.Tensor:
    """X bf16 [tokens x channels]: N(0,1) with round(frac * channels) seeded
    channels multiplied by ``alpha`` (alpha = 1: no outliers).  The same
    channels for every alpha of a seed."""
    g = _gen(seed, 11, device)
    x = torch.randn(tokens, channels, generator=g, device=device, dtype=torch.float32)
    n = int(round(frac * channels))
    if n and alpha != 1.0:
        gc = _gen(seed, 12, "cpu")
        ch = torch.randperm(channels, generator=gc)[:n]
        x[:, ch.to(device)] *= float(alpha)
    return x.to(torch.bfloat16)


def dense_weight(n_out: int, n_in: int, seed: int, device="cpu") -> torch.Tensor:
    """W bf16 [n_out x n_in] (K-major rows), N(0, 0.02)."""
    g = _gen(seed, 13, device)
    return (torch.randn(n_out, n_in, generator=g, device=device) * 0.02).to(torch.bfloat16)


def padded_rows_bound(cfg: LayerConfig) -> int:
    """Upper bound on the expert-grouped routed rows once every expert's
    segment is padded to a multiple of 128: T*k_r + E*127, rounded up to 128."""
    rows = cfg.tokens * cfg.topk + cfg.experts * 127
    return int(math.ceil(rows / 128) * 128)


def flops(cfg: LayerConfig) -> dict:
    """Algorithmic FLOPs of one layer step (padding rows not counted)."""
    M = cfg.tokens * cfg.topk
    if cfg.dense:
        fp4 = 2.0 * cfg.tokens * cfg.inter * cfg.hidden
        rac = 2.0 * cfg.tokens * cfg.inter * cfg.rac_k
        return dict(fp4=fp4, rac=rac, gate_up_fp4=fp4, down_fp4=0.0)
    gu = 2.0 * M * (2 * cfg.inter) * cfg.hidden
    dn = 2.0 * M * cfg.hidden * cfg.inter
    rac = 2.0 * M * (2 * cfg.inter) * cfg.rac_k + 2.0 * M * cfg.hidden * cfg.rac_k
    return dict(fp4=gu + dn, rac=rac, gate_up_fp4=gu, down_fp4=dn)
