"""Seeded synthetic inputs for RWKV-7-shaped quantized projections.

Holds none of the method's arithmetic: it only draws weights and activations
and describes workload shapes.  Both the CUDA path (tests, benchmark) and the
CPU oracle receive tensors made here.

Shapes follow the RWKV-7 depth/width table in "rwkv-quant: uma matriz em bf16
elimina 39% das perdas na quantização do RWKV-7 2.9B", section "Dois presets e
seis tamanhos" (0.1B 12x768, 1.5B 24x2048, 2.9B 32x2560, 7.2B 32x4096,
13.3B 61x4096); per layer the time-mix projections R, K, V, O are D x D and the
channel-mix key/value are D -> 4D and 4D -> D.  The massive input channel of
the 2.9B model (index 517) comes from the section "Onde o 2.9B quebra" of the
same article.  Trained checkpoints are not available, so weights are
N(0, 0.02^2) fp32 and activations N(0, 1) fp16.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

W_STD = 0.02
MASSIVE_CHANNEL_2P9B = 517
MASSIVE_FACTOR = 100.0


def seed_for(workload: int, layer: int = 0, proj: int = 0) -> int:
    """Seed recipe: 1234 + 1000*workload + 10*layer + projection index."""
    return 1234 + 1000 * workload + 10 * layer + proj


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def weights(N: int, K: int, seed: int, device="cpu") -> torch.Tensor:
    """fp32 W[N, K] ~ N(0, 0.02^2), row-major (N = out features)."""
    g = _gen(seed, device)
    w = torch.randn((N, K), generator=g, device=device, dtype=torch.float32)
    return w.mul_(W_STD)


def activations(M: int, K: int, seed: int, device="cpu", massive_channel=None,
                massive_factor: float = MASSIVE_FACTOR) -> torch.Tensor:
    """fp16 x[M, K] ~ N(0, 1); optionally one channel scaled by massive_factor."""
    g = _gen(seed + 500, device)
    x = torch.randn((M, K), generator=g, device=device, dtype=torch.float32)
    if massive_channel is not None and massive_channel < K:
        x[:, massive_channel] *= massive_factor
    return x.to(torch.float16)


@dataclass(frozen=True)
class Proj:
    name: str
    N: int          # out features
    K: int          # in features


@dataclass(frozen=True)
class Workload:
    index: int
    name: str
    bits: int
    layers: int
    projs: tuple            # tuple[Proj]
    Ms: tuple
    massive_channel: int | None = None
    fused_rkv: bool = True
    notes: str = ""


def layer_projs(D: int, ffn_mult: int = 4):
    return (Proj("r", D, D), Proj("k", D, D), Proj("v", D, D), Proj("o", D, D),
            Proj("ffn_key", ffn_mult * D, D), Proj("ffn_value", D, ffn_mult * D))


WORKLOADS = {
    1: Workload(1, "int4 g64 GEMV 768x768, M=1", 4, 1, (Proj("w", 768, 768),), (1,),
                fused_rkv=False),
    2: Workload(2, "RWKV-7 1.5B-shaped decode layer, int4 g64, D=2048 (24 layers)", 4, 24,
                layer_projs(2048), (1, 4, 8, 16, 32)),
    3: Workload(3, "RWKV-7 2.9B-shaped decode layer, int8 g64, D=2560, x[:,517]*100", 8, 32,
                layer_projs(2560), (1, 8, 32), massive_channel=MASSIVE_CHANNEL_2P9B),
    4: Workload(4, "RWKV-7 7.2B-shaped prefill, int4 g64, D=4096", 4, 32,
                (Proj("d_x_d", 4096, 4096), Proj("ffn_key", 16384, 4096),
                 Proj("ffn_value", 4096, 16384)), (64, 256, 512, 2048), fused_rkv=False),
    5: Workload(5, "13.3B-shaped decode stack, int4 g64, 61 layers x D=4096", 4, 61,
                layer_projs(4096), (1, 2, 4, 8, 16, 32)),
}


def algorithmic_weight_bytes(N: int, K: int, bits: int) -> int:
    """Code bytes + fp16 scale bytes a product must stream once."""
    return N * K * bits // 8 + N * (K // 64) * 2
