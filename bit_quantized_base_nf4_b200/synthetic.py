"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module only draws random numbers; it holds none of the quantization or
linear-layer arithmetic.  Every tensor is produced on the CPU from a
``torch.Generator`` so that the CUDA path and the CPU oracle see the same
bytes.

Workload shapes follow the 7B / 70B layer shapes the source pages quote
(hidden 4096, FFN 11008; 70B: 8192 and 28672).  Distributions:

* base weight W0 ~ N(0, std) fp32 (std 0.02 for 7B shapes, 0.015 for 70B),
  optionally with a fraction of entries multiplied by 10 ("outliers"), the
  positions drawn without replacement by a seeded ``randperm``;
* activations X and upstream gradients dY ~ N(0, 1), rounded to bf16;
* LoRA A ~ N(0, 1/K) and B ~ N(0, 0.01), rounded to bf16.

N(mu, sigma): the second parameter is the standard deviation.

The 32-layer decode sweep (about 5e9 weights) is the one exception to CPU
generation: its weights are drawn on the device by torch's CUDA generator,
seeded per matrix (``decode_weight``), because drawing them on the host would
take minutes.  A check against the oracle copies the drawn rows to the host.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

# tensor index added to the per-config seed
T_W, T_X, T_A, T_B, T_DY, T_OUTLIER = 0, 1, 2, 3, 4, 5


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def normal_f32(shape, std: float, seed: int) -> torch.Tensor:
    return torch.randn(*shape, generator=_gen(seed), dtype=torch.float32) * float(std)


def normal_bf16(shape, std: float, seed: int) -> torch.Tensor:
    return normal_f32(shape, std, seed).to(torch.bfloat16)


def with_outliers(w: torch.Tensor, frac: float, factor: float, seed: int) -> torch.Tensor:
    """Multiply exactly round(frac * numel) entries, chosen by a seeded randperm, by factor."""
    n = w.numel()
    k = int(round(frac * n))
    if k == 0:
        return w
    idx = torch.randperm(n, generator=_gen(seed))[:k]
    out = w.clone().reshape(-1)
    out[idx] *= factor
    return out.reshape(w.shape)


@dataclass
class LayerCase:
    """One frozen-base LoRA linear layer problem: W0 [N,K], X [M,K], A [r,K], B [N,r], dY [M,N]."""
    name: str
    M: int
    N: int
    K: int
    r: int
    alpha: float
    w_std: float = 0.02
    outlier_frac: float = 0.0
    seed: int = 0

    @property
    def scaling(self) -> float:
        return self.alpha / self.r if self.r > 0 else 0.0

    def weight(self) -> torch.Tensor:
        w = normal_f32((self.N, self.K), self.w_std, self.seed + T_W)
        if self.outlier_frac > 0:
            w = with_outliers(w, self.outlier_frac, 10.0, self.seed + T_OUTLIER)
        return w

    def x(self) -> torch.Tensor:
        return normal_bf16((self.M, self.K), 1.0, self.seed + T_X)

    def lora_a(self) -> torch.Tensor:
        return normal_bf16((self.r, self.K), 1.0 / self.K, self.seed + T_A)

    def lora_b(self) -> torch.Tensor:
        return normal_bf16((self.N, self.r), 0.01, self.seed + T_B)

    def dy(self) -> torch.Tensor:
        return normal_bf16((self.M, self.N), 1.0, self.seed + T_DY)


def tiny_case() -> LayerCase:
    """W0 256x512, X 16x512, r=8, alpha=16 (the small correctness case)."""
    return LayerCase("tiny-256x512-m16-r8", M=16, N=256, K=512, r=8, alpha=16.0, seed=1000)


def attn7b_case() -> LayerCase:
    """7B attention projection: W0 4096x4096, 2048 tokens, r=8, alpha=16."""
    return LayerCase("7b-attn-4096x4096-m2048-r8", M=2048, N=4096, K=4096, r=8, alpha=16.0, seed=2000)


def ffn7b_cases() -> list[LayerCase]:
    """7B FFN up/down with 0.1% outliers at 10x, 4096 tokens, r=64, alpha=128."""
    return [
        LayerCase("7b-ffn-up-11008x4096-m4096-r64", M=4096, N=11008, K=4096, r=64, alpha=128.0,
                  outlier_frac=1e-3, seed=3000),
        LayerCase("7b-ffn-down-4096x11008-m4096-r64", M=4096, N=4096, K=11008, r=64, alpha=128.0,
                  outlier_frac=1e-3, seed=3100),
    ]


def l70b_cases() -> list[LayerCase]:
    """70B layer shapes, std 0.015, 4096 tokens, r=64, alpha=128."""
    return [
        LayerCase("70b-attn-8192x8192-m4096-r64", M=4096, N=8192, K=8192, r=64, alpha=128.0,
                  w_std=0.015, seed=5000),
        LayerCase("70b-ffn-up-28672x8192-m4096-r64", M=4096, N=28672, K=8192, r=64, alpha=128.0,
                  w_std=0.015, seed=5100),
        LayerCase("70b-ffn-down-8192x28672-m4096-r64", M=4096, N=8192, K=28672, r=64, alpha=128.0,
                  w_std=0.015, seed=5200),
    ]


def decode_layer_shapes(with_gate: bool = False) -> list[tuple[str, int, int, bool]]:
    """Per-layer matrices of the 7B decode sweep: (name, N_out, K_in, has_lora)."""
    shapes = [("q", 4096, 4096, True), ("k", 4096, 4096, True), ("v", 4096, 4096, True),
              ("o", 4096, 4096, True), ("up", 11008, 4096, False), ("down", 4096, 11008, False)]
    if with_gate:
        shapes.insert(4, ("gate", 11008, 4096, False))
    return shapes


def decode_weight(layer: int, index: int, n_out: int, n_in: int, device) -> torch.Tensor:
    """Weight `index` of decode layer `layer`: N(0, 0.02) fp32 [n_out, n_in] drawn on `device`."""
    g = torch.Generator(device=device)
    g.manual_seed(4000 + 16 * int(layer) + int(index))
    return torch.randn(n_out, n_in, generator=g, dtype=torch.float32, device=device) * 0.02


def decode_inputs(M: int, K: int, seed: int) -> torch.Tensor:
    """Decode activations: M tokens of width K, N(0, 1) rounded to bf16 (host)."""
    return normal_bf16((M, K), 1.0, seed)
