"""Seeded synthetic weights with the shapes of the Llama-2 family.

Input generation only: this module holds none of the quantiser's arithmetic
and serves the tests, the benchmark and the oracle checks alike.

Recipe (stands in for the trained Llama-2 checkpoints the pages evaluate on,
which are not available here): W = 0.02 * N(0, 1); a Bernoulli(1e-3) mask then
picks outliers, which are multiplied by 10; the result is cast to the stated
dtype.  Both draws come from one CPU ``torch.Generator`` seeded with ``seed``,
``randn`` first and ``rand`` second.  Model weight sets use
seed = 1000 * layer + matrix index (q=0, k=1, v=2, o=3, gate=4, up=5, down=6).
weight_device() draws the same recipe on the GPU (for the 70B-shaped set,
137 GB of fp16 weights).
"""
from dataclasses import dataclass

import torch

STD = 0.02
OUTLIER_FRAC = 1e-3
OUTLIER_SCALE = 10.0

MATRIX_INDEX = {"q": 0, "k": 1, "v": 2, "o": 3, "gate": 4, "up": 5, "down": 6}


def weight(rows: int, cols: int, seed: int, dtype=torch.float16, std: float = STD,
           outlier_frac: float = OUTLIER_FRAC, outlier_scale: float = OUTLIER_SCALE) -> torch.Tensor:
    """One [rows, cols] weight matrix (out x in, row-major) on the CPU."""
    g = torch.Generator("cpu").manual_seed(int(seed))
    w = torch.randn(rows, cols, generator=g, dtype=torch.float32) * std
    mask = torch.rand(rows, cols, generator=g) < outlier_frac
    w = torch.where(mask, w * outlier_scale, w)
    return w.to(dtype)


def weight_device(rows: int, cols: int, seed: int, dtype=torch.float16, device="cuda", std: float = STD,
                  outlier_frac: float = OUTLIER_FRAC, outlier_scale: float = OUTLIER_SCALE) -> torch.Tensor:
    """The same recipe drawn on the GPU (one CUDA ``torch.Generator`` seeded
    with ``seed``, ``randn`` then ``rand``), for weight sets too large to draw
    on the host in reasonable time.  The values differ from weight()'s for the
    same seed (another generator); the distribution is the same."""
    g = torch.Generator(device).manual_seed(int(seed))
    w = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32).mul_(std)
    mask = torch.rand(rows, cols, generator=g, device=device) < outlier_frac
    w = torch.where(mask, w * outlier_scale, w)
    del mask
    return w.to(dtype)


def seed_for(layer: int, matrix: str) -> int:
    return 1000 * layer + MATRIX_INDEX[matrix]


@dataclass(frozen=True)
class ModelShape:
    name: str
    layers: int
    hidden: int
    ffn: int
    kv_out: int  # output rows of k_proj / v_proj

    def matrices(self):
        """(name, rows, cols) of one decoder layer's linear weights, rows = out."""
        h, f = self.hidden, self.ffn
        return [("q", h, h), ("k", self.kv_out, h), ("v", self.kv_out, h), ("o", h, h),
                ("gate", f, h), ("up", f, h), ("down", h, f)]

    def weights_per_layer(self) -> int:
        return sum(r * c for _, r, c in self.matrices())


LLAMA2_7B = ModelShape("llama-2-7b", 32, 4096, 11008, 4096)
LLAMA2_13B = ModelShape("llama-2-13b", 40, 5120, 13824, 5120)
LLAMA2_70B = ModelShape("llama-2-70b", 80, 8192, 28672, 1024)


def scales(G: int, seed: int) -> torch.Tensor:
    """Seeded synthetic per-group scales (fp16, positive, spread like the
    dequantisation multipliers of 0.02-std weights at 2-4 bits), with a few
    constant runs: 0.004 * |N(1, 0.5)| + 1e-4, and every 977th block of 128
    set to one value."""
    gen = torch.Generator("cpu").manual_seed(seed)
    v = 0.004 * torch.randn(G, generator=gen, dtype=torch.float32).mul(0.5).add(1.0).abs() + 1e-4
    for b in range(0, G // 128, 977):
        v[b * 128:(b + 1) * 128] = v[b * 128]
    return v.to(torch.float16)
