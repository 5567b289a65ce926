"""Seeded synthetic inputs for the Lighthouse layer.

This module holds no Lighthouse arithmetic: it only draws the layer's inputs
(Q, K, V and the upstream gradient dO) with the shapes and value
distribution of the workloads below, so that the CUDA path and the CPU
oracle can be fed identical bytes.

Distribution: every element is N(0, 1) times a per-token scale
exp(N(0, 0.5^2)); the scale is one scalar per (batch, token) and tensor,
shared by all heads and channels, drawn independently for Q, K and V.  dO is
plain N(0, 1).  The draw order from one ``torch.Generator`` seeded with
``seed`` is fixed: Q, K, V, scale_Q, scale_K, scale_V, dO.  Values are formed
in fp32 and cast to the storage dtype with round-to-nearest-even.

The stand-in is for the projected activations of a 530M Llama-3-style
decoder at 98,304 tokens of context (gist.science technical summary,
section 4 "Experimental Results"); no dataset or trained weight is used.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: str  # "f32" or "bf16"
    p: int
    L: int
    k: int
    backward: bool  # the configuration the pages quote includes the backward pass
    select: str = "joint"  # selection rule: "joint", "descent" or "regional"


# The workloads the layer is exercised and measured on.
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 2, 1024, 64, "f32", 4, 3, 32, False),
    "8k_bf16": Workload("8k_bf16", 1, 8, 8192, 64, "bf16", 4, 4, 256, True),
    "98k_k1536": Workload("98k_k1536", 1, 16, 98304, 64, "bf16", 4, 3, 1536, True),
    "98k_k6144": Workload("98k_k6144", 1, 16, 98304, 64, "bf16", 4, 3, 6144, True),
    "512k_k2048": Workload("512k_k2048", 1, 16, 524288, 64, "bf16", 4, 4, 2048, True),
    # the pages' best pyramid ablation (pooling factor 2) at the 98K length: S = 30720
    "98k_p2_k1536": Workload("98k_p2_k1536", 1, 16, 98304, 64, "bf16", 2, 3, 1536, True),
    # the same budget chosen by hierarchical descent (k best per level, their children kept)
    "98k_descent_k1536": Workload("98k_descent_k1536", 1, 16, 98304, 64, "bf16", 4, 3, 1536, True,
                                  "descent"),
    # the same budget with every 2048-candidate region keeping its share
    "98k_regional_k1536": Workload("98k_regional_k1536", 1, 16, 98304, 64, "bf16", 4, 3, 1536, True,
                                   "regional"),
    # head dimension 128 at the same bytes per token (8 heads x 128 channels)
    "98k_d128_k1536": Workload("98k_d128_k1536", 1, 8, 98304, 128, "bf16", 4, 3, 1536, True),
}

TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def make_inputs(B: int, H: int, N: int, d: int, dtype: str, seed: int = 0,
                device: str | torch.device = "cpu", with_grad: bool = True):
    """Return (Q, K, V, dO) as contiguous [B, H, N, d] tensors on ``device``.

    dO is None when ``with_grad`` is false (it is still drawn last, so the
    Q/K/V bytes do not depend on ``with_grad``).
    """
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    shape = (B, H, N, d)
    q = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    k = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    v = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    scales = []
    for _ in range(3):
        z = torch.randn((B, N), generator=g, device=device, dtype=torch.float32)
        scales.append(torch.exp(0.5 * z).view(B, 1, N, 1))
    q.mul_(scales[0])
    k.mul_(scales[1])
    v.mul_(scales[2])
    dt = TORCH_DTYPE[dtype]
    out = [q.to(dt).contiguous(), k.to(dt).contiguous(), v.to(dt).contiguous()]
    del q, k, v
    if with_grad:
        do = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        out.append(do.to(dt).contiguous())
    else:
        out.append(None)
    return tuple(out)


def make_workload_inputs(w: Workload, seed: int = 0, device="cpu"):
    """(Q, K, V, dO) of a workload.  dO is always drawn (after Q, K, V, so their
    bytes do not depend on it): the benchmark times forward and backward of
    every workload."""
    return make_inputs(w.B, w.H, w.N, w.d, w.dtype, seed=seed, device=device, with_grad=True)


def make_scores(B: int, H: int, M: int, seed: int = 0, distinct: int | None = None):
    """Seeded fp32 candidate-score arrays [B, H, M] for exercising selection.

    With ``distinct`` set, values are drawn from that many distinct levels so
    that exact ties are frequent.  Values are positive, like norm sums.
    """
    g = torch.Generator()
    g.manual_seed(seed)
    if distinct is None:
        s = torch.rand((B, H, M), generator=g, dtype=torch.float32) * 30.0
    else:
        s = torch.randint(0, distinct, (B, H, M), generator=g).to(torch.float32) * 0.25 + 1.0
    return s.contiguous()
