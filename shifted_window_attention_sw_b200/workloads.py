"""The layer shapes used by the tests and the benchmark.

Shapes follow the Video Swin setting: a 32-frame 224x224 clip becomes
T/2 x H/4 x W/4 = 16 x 56 x 56 tokens ("Video Swin Transformer" summary page,
Problem and Method step 1); windows are (P, M, M) = (8, 7, 7) with the
half-window shift (4, 3, 3) by integer halving (Method steps 4-5, Pitfalls);
Swin-T uses C = 96 with heads = C / 32, Swin-B C = 128 ("Paper vs code", heads
per stage).
"""

from __future__ import annotations

from dataclasses import dataclass, field

WINDOW = (8, 7, 7)
SHIFT = (4, 3, 3)
NO_SHIFT = (0, 0, 0)


@dataclass(frozen=True)
class Layer:
    B: int
    T: int
    H: int
    W: int
    C: int
    heads: int
    window: tuple = WINDOW
    shift: tuple = SHIFT
    seed_offset: int = 0  # added to the per-tensor seed (second layer of a pair, later stages)

    @property
    def shape(self):
        return (self.B, self.T, self.H, self.W, self.C)


@dataclass(frozen=True)
class Workload:
    name: str
    index: int  # seeds are 1000 * index + k
    dtype: str  # "f32" or "bf16"
    layers: tuple = field(default_factory=tuple)
    description: str = ""


WORKLOADS = {
    "swin_t_s1_small_f32": Workload(
        "swin_t_s1_small_f32", 1, "f32",
        (Layer(1, 8, 14, 14, 96, 3, WINDOW, SHIFT), Layer(1, 8, 14, 14, 96, 3, WINDOW, NO_SHIFT)),
        "single SW-MSA layer (1,8,14,14,96), 3 heads, fp32, plus its shift-0 variant",
    ),
    "swin_t_s1_b8": Workload(
        "swin_t_s1_b8", 2, "bf16",
        (Layer(8, 16, 56, 56, 96, 3, WINDOW, NO_SHIFT), Layer(8, 16, 56, 56, 96, 3, WINDOW, SHIFT, 10)),
        "Swin-T stage 1, 32x224^2 clips, batch 8: W-MSA + SW-MSA pair, bf16",
    ),
    "swin_t_s3_b32": Workload(
        "swin_t_s3_b32", 3, "bf16",
        (Layer(32, 16, 14, 14, 384, 12, WINDOW, SHIFT),),
        "Swin-T stage 3 SW-MSA, batch 32, bf16",
    ),
    "swin_b_pad_b4": Workload(
        "swin_b_pad_b4", 4, "bf16",
        (Layer(4, 12, 40, 40, 128, 4, WINDOW, SHIFT),),
        "padding/mask stress (pads to 16x42x42), Swin-B stage-1 width, bf16",
    ),
    "swin_b_stages_b8": Workload(
        "swin_b_stages_b8", 5, "bf16",
        (
            Layer(8, 16, 56, 56, 128, 4, WINDOW, SHIFT, 0),
            Layer(8, 16, 28, 28, 256, 8, WINDOW, SHIFT, 10),
            Layer(8, 16, 14, 14, 512, 16, WINDOW, SHIFT, 20),
            Layer(8, 16, 7, 7, 1024, 32, WINDOW, (4, 0, 0), 30),
        ),
        "Swin-B SW-MSA layers of all four stages in sequence, batch 8, bf16",
    ),
}

HEADLINE = "swin_t_s1_b8"

