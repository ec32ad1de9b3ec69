"""Seeded synthetic inputs for the five RWKV-7 projection workloads.

This module only draws inputs (weights, activations, the per-channel E[x^2]
vector); it holds none of the quantization or product arithmetic, so the CPU
oracle and the CUDA path can both be fed from it.

The shapes follow the RWKV-7 sizes of the rwkv-quant article ("Two presets and
six sizes": 0.1B width 768, 1.5B width 2048 x 24 layers, 2.9B width 2560 x 32,
7.2B width 4096) and the projection shapes r/k/v/o C x C, channel-mix key
C -> 4C, value 4C -> C and the head 4096 -> 65536. The activation energy
follows the article's "massive channel" finding ("Where 2.9B breaks": channel
517 on 2.9B, channel 1202 on 1.5B, eight channels holding 98% of the energy on
2.9B and 99% on 7.2B). No trained checkpoint or calibration text exists here;
these draws stand in for them.

Weights are fp32 [N][K] (row = output feature), N(0, 0.02). Activations are
bf16 [M][K] = N(0, 1) * sqrt(a_k), so E[x_k^2] = a_k, and the same a_k is the
``act_sq`` vector handed to the quantizer.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Matrix:
    name: str
    K: int          # input features (reduction dim)
    N: int          # output features
    fmt: str        # "w4g64" | "w8g16" | "w8g64" | "w6g16" | "w4sb32" | "w5sb32" | "w6sb32"
    n_cand: int     # 1 = RTN, 64 = E[x^2]-weighted search
    outliers: bool = False


@dataclass(frozen=True)
class Workload:
    index: int
    name: str
    per_layer: tuple
    layers: int
    Ms: tuple
    massive: dict = field(default_factory=dict)   # K -> recipe key

    def matrices(self):
        """(j, layer, Matrix) for every matrix of the workload, in call order."""
        j = 0
        out = []
        for layer in range(self.layers):
            for m in self.per_layer:
                out.append((j, layer, m))
                j += 1
        return out

    def packed_bytes(self, packed_size) -> int:
        return sum(packed_size(m.fmt, m.K, m.N) for _, _, m in self.matrices())


WORKLOADS = [
    # 2048 distinct copies (642 MB, more than four times the L2): one 313 KB
    # matrix would sit in L2 and measure launch overhead, not the weight stream
    Workload(0, "w4g64-rtn-768 (RWKV-7 0.1B o_proj) x2048 distinct",
             (Matrix("o", 768, 768, "w4g64", 1),), 2048, (1,), {768: "ch5x50"}),
    Workload(1, "w8g16-aw-2048 (1.5B r/k/v/o x24, 0.1% outliers x10)",
             tuple(Matrix(n, 2048, 2048, "w8g16", 64, outliers=True) for n in "rkvo"),
             24, (1, 2, 4, 8), {}),
    Workload(2, "w4g64-aw-1.5B-layerset x24 (r/k/v/o 2048^2, ffn 2048->8192->2048)",
             tuple(Matrix(n, 2048, 2048, "w4g64", 64) for n in "rkvo")
             + (Matrix("ffn_key", 2048, 8192, "w4g64", 64),
                Matrix("ffn_value", 8192, 2048, "w4g64", 64)),
             24, (1, 4, 16, 32), {2048: "ch1202x50"}),
    Workload(3, "w4sb32-aw-2.9B x32 (o 2560^2, ffn 2560->10240->2560)",
             (Matrix("o", 2560, 2560, "w4sb32", 64),
              Matrix("ffn_key", 2560, 10240, "w4sb32", 64),
              Matrix("ffn_value", 10240, 2560, "w4sb32", 64)),
             32, (1, 8, 32), {2560: "eight98"}),
    Workload(4, "7.2B width 4096: w4g64 r/k/v/o + ffn, w8g16 head 4096->65536",
             tuple(Matrix(n, 4096, 4096, "w4g64", 64) for n in "rkvo")
             + (Matrix("ffn_key", 4096, 16384, "w4g64", 64),
                Matrix("ffn_value", 16384, 4096, "w4g64", 64),
                Matrix("head", 4096, 65536, "w8g16", 64)),
             1, (1, 32, 64, 128), {4096: "eight99"}),
]

# Preset variants: the COMPRESSION preset's wider codes at 2.9B width
# (rwkv-quant article, "Two presets and six sizes": ffn.key and head in 5 bits;
# "Where 2.9B breaks": all of o_proj in 6 bits as the alternative to one bf16
# matrix), the REDUCTION preset's 6-bit channel-mix, and the int8 g64 tier.
VARIANTS = [
    Workload(5, "w5sb32-aw-2.9B ffn.key 2560->10240 x32 (COMPRESSION)",
             (Matrix("ffn_key", 2560, 10240, "w5sb32", 64),), 32, (1, 16), {2560: "eight98"}),
    Workload(6, "w5sb32-aw-2.9B head 2560->65536 (COMPRESSION)",
             (Matrix("head", 2560, 65536, "w5sb32", 64),), 1, (1, 16), {2560: "eight98"}),
    Workload(7, "w6sb32-aw-2.9B o 2560^2 x32 (all of o_proj in 6 bits)",
             (Matrix("o", 2560, 2560, "w6sb32", 64),), 32, (1, 16), {2560: "eight98"}),
    # the REDUCTION preset's channel-mix in 6 bits (symmetric, group 16)
    Workload(8, "w6g16-aw-1.5B cmix 2048->8192->2048 x24 (REDUCTION)",
             (Matrix("ffn_key", 2048, 8192, "w6g16", 64), Matrix("ffn_value", 8192, 2048, "w6g16", 64)),
             24, (1, 16), {2048: "ch1202x50"}),
    # the model card's int8 w8g64 tier ("Accuracy warning") on the 1.5B layer set
    Workload(9, "w8g64-aw-1.5B-layerset x24 (int8 tier)",
             tuple(Matrix(n, 2048, 2048, "w8g64", 64) for n in "rkvo")
             + (Matrix("ffn_key", 2048, 8192, "w8g64", 64), Matrix("ffn_value", 8192, 2048, "w8g64", 64)),
             24, (1, 4, 16), {2048: "ch1202x50"}),
]


def weight_seed(w: Workload, j: int) -> int:
    return 1000 * w.index + j


def x_seed(w: Workload, j: int) -> int:
    return 500000 + 1000 * w.index + j


def act_sq(w: Workload, K: int) -> np.ndarray:
    """E[x_k^2] per input channel, in closed form (fp32 [K])."""
    a = np.ones(K, dtype=np.float32)
    recipe = w.massive.get(K)
    if recipe == "ch5x50":
        a[5] = 2500.0
    elif recipe == "ch1202x50":
        a[1202] = 2500.0
    elif recipe == "eight98":
        # channel 517 plus 7 others hold 98% of the energy; the other K-8 hold 2%
        g = torch.Generator().manual_seed(3998)
        rest = torch.randperm(K - 1, generator=g)[:7].numpy()
        chans = [517] + [int(c) + (1 if c >= 517 else 0) for c in rest]
        a[chans] = np.float32(0.98 * ((K - 8) / 0.02) / 8)
    elif recipe == "eight99":
        g = torch.Generator().manual_seed(4998)
        chans = torch.randperm(K, generator=g)[:8].numpy()
        a[chans] = np.float32(0.99 * ((K - 8) / 0.01) / 8)
    return a


def weights(w: Workload, j: int, m: Matrix, device: str = "cpu") -> torch.Tensor:
    """fp32 [N][K] ~ N(0, 0.02); with ``outliers``, exactly round(0.001*K*N)
    entries (chosen by randperm) are multiplied by 10."""
    dev = torch.device(device)
    g = torch.Generator(device=dev).manual_seed(weight_seed(w, j))
    W = torch.randn(m.N, m.K, generator=g, device=dev, dtype=torch.float32) * 0.02
    if m.outliers:
        cnt = int(round(0.001 * m.K * m.N))
        idx = torch.randperm(m.K * m.N, generator=g, device=dev)[:cnt]
        W.view(-1)[idx] *= 10.0
    return W


def activations(w: Workload, j: int, K: int, M: int, device: str = "cpu") -> torch.Tensor:
    """bf16 [M][K] = N(0,1) * sqrt(a_k)."""
    dev = torch.device(device)
    g = torch.Generator(device=dev).manual_seed(x_seed(w, j))
    x = torch.randn(M, K, generator=g, device=dev, dtype=torch.float32)
    scale = torch.from_numpy(np.sqrt(act_sq(w, K))).to(dev)
    return (x * scale).to(torch.bfloat16)


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    """Raw uint16 bit patterns of a bf16 tensor (on the host)."""
    return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def random_matrix(seed: int, N: int, K: int, scale: float = 0.02) -> torch.Tensor:
    g = torch.Generator().manual_seed(seed)
    return torch.randn(N, K, generator=g, dtype=torch.float32) * scale


def random_x(seed: int, M: int, K: int, a: np.ndarray | None = None) -> torch.Tensor:
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g, dtype=torch.float32)
    if a is not None:
        x = x * torch.from_numpy(np.sqrt(a))
    return x.to(torch.bfloat16)


def random_act_sq(seed: int, K: int, massive: int = 0, energy: float = 2500.0) -> np.ndarray:
    """Ones, with ``massive`` channels (randperm) set to ``energy``."""
    a = np.ones(K, dtype=np.float32)
    if massive:
        g = torch.Generator().manual_seed(seed)
        chans = torch.randperm(K, generator=g)[:massive].numpy()
        a[chans] = np.float32(energy)
    return a

