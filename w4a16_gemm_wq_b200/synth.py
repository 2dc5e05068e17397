"""Seeded synthetic inputs shaped like the Lance-Quant workloads.

This module holds no quantization arithmetic: it only draws weights and
activations. The same tensors feed both the CUDA path and the CPU oracle, so
neither side ever generates its own inputs.

Shapes come from the Qwen2.5-VL-3B-class transformer block that Lance is
built on (hidden 2048, k/v width 256, MLP width 11008, 36 layers), with a
parallel ``_moe_gen`` sibling for each of the 7 projections ("Lance-Quant",
section "校准阶段": 504 target Linear layers).

Every draw uses a ``torch.Generator`` seeded explicitly, so a (seed, shape)
pair always gives the same bytes on any machine with this torch build.
"""
from __future__ import annotations

import torch

# (name, K = in_features, N = out_features) of one Lance / Qwen2.5-VL-3B block.
PROJECTIONS = (
    ("q_proj", 2048, 2048),
    ("k_proj", 2048, 256),
    ("v_proj", 2048, 256),
    ("o_proj", 2048, 2048),
    ("gate_proj", 2048, 11008),
    ("up_proj", 2048, 11008),
    ("down_proj", 11008, 2048),
)

# The same block as an inference engine runs it: the projections that read one
# input stacked along N into one Linear (q/k/v after the attention norm,
# gate/up after the MLP norm), the layout the shared-s AWQ scale serves
# (one s per norm, folded into that norm).  Same flops as PROJECTIONS.
FUSED_PROJECTIONS = (
    ("qkv_proj", 2048, 2048 + 256 + 256),
    ("o_proj", 2048, 2048),
    ("gate_up_proj", 2048, 2 * 11008),
    ("down_proj", 11008, 2048),
)

# The four distinct decode shapes (K, N) of the block.
DECODE_SHAPES = ((2048, 2048), (2048, 256), (2048, 11008), (11008, 2048))

N_LAYERS = 36
LINEARS_PER_LAYER = 14  # 7 projections + 7 `_moe_gen` siblings
ALPHA_GRID = tuple(i / 20.0 for i in range(20))


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def outlier_channels(K: int, frac: float, seed: int) -> torch.Tensor:
    """round(frac*K) distinct input-channel indices, from a seeded permutation."""
    n = int(round(frac * K))
    perm = torch.randperm(K, generator=_gen(seed ^ 0x5A5A))
    return torch.sort(perm[:n]).values


def weight(N: int, K: int, seed: int, *, std: float = 0.02, outlier_frac: float = 0.005,
           outlier_mult: float = 20.0, device="cpu") -> torch.Tensor:
    """bf16 [N, K] ~ N(0, std^2), with round(outlier_frac*K) input channels scaled by outlier_mult."""
    g = _gen(seed, device)
    w = torch.randn(N, K, generator=g, device=device, dtype=torch.float32) * std
    ch = outlier_channels(K, outlier_frac, seed)
    if ch.numel():
        w[:, ch.to(w.device)] *= outlier_mult
    return w.to(torch.bfloat16)


def activations(M: int, K: int, seed: int, *, channels: torch.Tensor | None = None,
                mult: float = 10.0, device="cpu") -> torch.Tensor:
    """bf16 [M, K] ~ N(0, 1); the given channels are scaled by mult."""
    g = _gen(seed + 7777, device)
    x = torch.randn(M, K, generator=g, device=device, dtype=torch.float32)
    if channels is not None and channels.numel():
        x[:, channels.to(x.device)] *= mult
    return x.to(torch.bfloat16)


def activations_student_t(T: int, K: int, seed: int, *, df: int = 3, sigma: float = 1.0,
                          device="cpu") -> torch.Tensor:
    """bf16 [T, K] heavy-tailed calibration tokens: m_k * t_df with m_k = exp(sigma*Z_k).

    t_df = Z / sqrt(chi2_df / df) with chi2_df a sum of df squared normals.
    """
    g = _gen(seed + 3333, device)
    m = torch.exp(sigma * torch.randn(K, generator=g, device=device, dtype=torch.float64))
    z = torch.randn(T, K, generator=g, device=device, dtype=torch.float64)
    chi2 = torch.zeros(T, K, device=device, dtype=torch.float64)
    for _ in range(df):
        chi2 += torch.randn(T, K, generator=g, device=device, dtype=torch.float64) ** 2
    t = z / torch.sqrt(chi2 / df)
    return (m * t).to(torch.float32).to(torch.bfloat16)


def act_mean_lognormal(K: int, seed: int, *, sigma: float = 1.0, device="cpu") -> torch.Tensor:
    """fp32 [K] synthetic per-channel mean |activation| (lognormal), standing in for calibration stats."""
    g = _gen(seed + 4444, device)
    return torch.exp(sigma * torch.randn(K, generator=g, device=device, dtype=torch.float64)).to(torch.float32)


def config1(seed: int = 0):
    """Single Linear K=N=512: W with 1% outlier channels x20; X_calib [128,512], X1 [1,512], X16 [16,512]
    with the same channels x10 (all ~N(0,1) otherwise)."""
    K = N = 512
    w = weight(N, K, seed, outlier_frac=0.01)
    ch = outlier_channels(K, 0.01, seed)
    x_calib = activations(128, K, seed + 1, channels=ch)
    x1 = activations(1, K, seed + 2, channels=ch)
    x16 = activations(16, K, seed + 3, channels=ch)
    return dict(W=w, channels=ch, X_calib=x_calib, X1=x1, X16=x16, K=K, N=N)


def whole_model_layers():
    """(layer, name, K, N, seed) of the 504 target Linears of the whole-model pass:
    36 layers x (7 projections + a same-shaped `_moe_gen` sibling of each)."""
    out = []
    for layer in range(N_LAYERS):
        for p, (name, K, N) in enumerate(PROJECTIONS):
            for sib in (0, 1):
                out.append((layer, name + ("_moe_gen" if sib else ""), K, N,
                            layer_seed(5, LINEARS_PER_LAYER * layer + 2 * p + sib)))
    return out


def layer_seed(config: int, layer_index: int) -> int:
    return 1000 * config + layer_index


def awq_calib_tokens() -> int:
    return 512

