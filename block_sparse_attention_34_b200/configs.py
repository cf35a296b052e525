"""The five seeded synthetic workloads of the block-sparse attention path.

Each workload is a per-head block-sparse attention call over a video DiT's
F x H x W latent token grid (PAROAttention, arXiv 2506.16054, review
"key_machinery": tokens of a 3D feature volume flattened to a 1D sequence;
SPADE, arXiv 2608.03335, review "referee summary": 720p Hunyuan/Wan layers).
Sizes, dtypes, densities and mask kinds are the ones the workloads are quoted
on; the inputs themselves come from :mod:`synth`.

Derived quantities follow one convention everywhere:
  N   = F*H*W tokens per head
  NB  = ceil(N / block) blocks per head (the last one may be partial)
  N_p = NB*block (the permuted sequence is zero-padded at its tail)

The kept-block budget k (from the density) is method arithmetic and is
computed by the library (``pa_k_for_density``) and, independently, by the
oracle; this module only holds the sizes.
"""

from __future__ import annotations

from dataclasses import dataclass, field

# Axis orders, listed outermost -> innermost (F = frames, H = height,
# W = width).  The id is what the C ABI takes, one int8 per head.
PERM_NAMES = ("FHW", "FWH", "HFW", "HWF", "WFH", "WHF")


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    heads: int
    d: int
    F: int
    H: int
    W: int
    block: int
    dtype: str  # "f32" | "bf16"
    density: float
    mask: str  # "static" (bitmask from pooled scores) | "topk" (online)
    perms: tuple | None = None  # fixed per-head axis orders, else drawn
    int8: bool = False  # INT8 QK^T / PV variant
    seed: int = 0
    description: str = field(default="", compare=False)

    @property
    def N(self) -> int:
        return self.F * self.H * self.W

    @property
    def NB(self) -> int:
        return -(-self.N // self.block)

    @property
    def N_p(self) -> int:
        return self.NB * self.block

    def kept_tiles(self, k: int) -> int:
        return self.B * self.heads * self.NB * k

    def flops(self, k: int) -> float:
        """Algorithmic FLOPs over kept tiles: 4*b^2*d per kept (q-block, k-block)
        tile (QK^T and PV, 2 FLOPs per multiply-add), pad rows included."""
        return 4.0 * self.block * self.block * self.d * self.kept_tiles(k)

    def with_density(self, density: float) -> "Workload":
        return Workload(self.name + f"@{density:g}", self.B, self.heads, self.d,
                        self.F, self.H, self.W, self.block, self.dtype, density,
                        self.mask, self.perms, self.int8, self.seed, self.description)


WORKLOADS = {
    "tiny_4x8x8": Workload(
        "tiny_4x8x8", B=1, heads=2, d=64, F=4, H=8, W=8, block=64, dtype="f32",
        density=0.5, mask="static", perms=(0, 5),
        description="tiny correctness case, fp32, static mask, orders FHW/WHF"),
    "small_8x16x16": Workload(
        "small_8x16x16", B=1, heads=4, d=64, F=8, H=16, W=16, block=64, dtype="bf16",
        density=0.30, mask="static",
        description="N=2048, bf16, static per-head mask from pooled scores"),
    "480p_21x30x52": Workload(
        "480p_21x30x52", B=1, heads=12, d=128, F=21, H=30, W=52, block=128, dtype="bf16",
        density=0.25, mask="topk",
        description="480p-shaped video DiT layer, online top-k"),
    "720p_21x45x80": Workload(
        "720p_21x45x80", B=1, heads=40, d=128, F=21, H=45, W=80, block=128, dtype="bf16",
        density=0.15, mask="topk",
        description="720p-shaped video DiT layer, online top-k, plus a dense run"),
    "longclip_33x45x80_int8": Workload(
        "longclip_33x45x80_int8", B=1, heads=24, d=128, F=33, H=45, W=80, block=128,
        dtype="bf16", density=0.20, mask="topk", int8=True,
        description="long clip, INT8 QK^T/PV with per-block symmetric scales"),
}

ORDER = list(WORKLOADS)
