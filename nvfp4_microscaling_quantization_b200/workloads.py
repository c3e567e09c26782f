"""Seeded synthetic input generators for the quantization workloads.

This module holds no quantization arithmetic: it only draws bf16 tensors
with the shapes and value distributions of the linear-layer tensors that
block-scaled NVFP4 training quantizes (weights, activations, gradients), and
names the calls each workload makes.  Both the CUDA path (through bench.py and
the GPU tests) and the CPU oracle (through the tests) read the same tensors
from here.

Every tensor is drawn with a torch generator seeded by the workload seed, in
float32, then rounded to bf16 (round-to-nearest-even).  The draws happen in
the order written below, so a (workload, seed, device) triple always gives the
same bits.  Small tensors are drawn on the CPU; the full-size workloads are
drawn on the GPU (torch's CUDA generator), which takes well under a second
where the CPU takes about a minute, and are copied to the host when the
oracle needs them.

Distributions (the pages' workloads are the weight, activation and gradient
tensors of LLM linear layers, quantized forward with RTN / 4-over-6 / IF4 and
backward with SR / MS-EDEN):
  normal(std)        : std * N(0, 1)
  outlier_normal     : std * N(0, 1), then 1% of entries (Bernoulli mask) x10
  student_t3(std)    : N(0,1) / sqrt(chi2_3 / 3), chi2_3 = sum of 3 squared
                       N(0,1) draws, times std / sqrt(3) (t_3 has variance 3)
  laplace_channels   : Laplace(0, 1) (inverse CDF of U(-1/2, 1/2), tail cut
                       at |x| = 24 ln 2 so that a uniform draw of exactly 0
                       gives a finite value) times a per-column scale
                       10^U(-1, 1) (log-uniform in [0.1, 10])
"""
from dataclasses import dataclass, field
from typing import Dict, List, Tuple

import torch

ROWWISE, TRANSPOSED = 0, 1
RTN, SR, MS_EDEN, IF4, FOUR_OVER_SIX, SCALE_SEARCH, MXFP4, NVINT4 = 0, 1, 2, 3, 4, 5, 6, 7
NVFP3, NVINT3, IF3, MXFP3 = 8, 9, 10, 11
MODE_NAMES = {RTN: "rtn", SR: "sr", MS_EDEN: "ms_eden", IF4: "if4", FOUR_OVER_SIX: "4over6",
              SCALE_SEARCH: "scale_search", MXFP4: "mxfp4", NVINT4: "nvint4", NVFP3: "nvfp3",
              NVINT3: "nvint3", IF3: "if3", MXFP3: "mxfp3"}
LAYOUT_NAMES = {ROWWISE: "rowwise", TRANSPOSED: "transposed"}


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal(shape, std: float, gen: torch.Generator) -> torch.Tensor:
    return (torch.randn(shape, generator=gen, dtype=torch.float32, device=gen.device) * std).to(torch.bfloat16)


def outlier_normal(shape, std: float, frac: float, factor: float, gen: torch.Generator) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, dtype=torch.float32, device=gen.device) * std
    mask = torch.rand(shape, generator=gen, dtype=torch.float32, device=gen.device) < frac
    x = torch.where(mask, x * factor, x)
    return x.to(torch.bfloat16)


def student_t3(shape, std: float, gen: torch.Generator) -> torch.Tensor:
    z = torch.randn(shape, generator=gen, dtype=torch.float32, device=gen.device)
    chi2 = torch.zeros(shape, dtype=torch.float32, device=gen.device)
    for _ in range(3):
        n = torch.randn(shape, generator=gen, dtype=torch.float32, device=gen.device)
        chi2.addcmul_(n, n)
        del n
    t = z / torch.sqrt(chi2 / 3.0)
    return (t * (std / 3.0 ** 0.5)).to(torch.bfloat16)


def laplace_channels(shape, gen: torch.Generator) -> torch.Tensor:
    rows, cols = shape
    u = torch.rand(shape, generator=gen, dtype=torch.float32, device=gen.device) - 0.5
    # inverse CDF; torch.rand can return exactly 0 (u = -0.5), whose image is
    # -inf, so the tail is cut at 2|u| = 1 - 2^-24 (|lap| <= 24 ln 2)
    lap = -torch.sign(u) * torch.log1p(-(2.0 * u.abs()).clamp_max(1.0 - 2.0 ** -24))
    col_scale = torch.pow(10.0, torch.rand((1, cols), generator=gen, dtype=torch.float32,
                                           device=gen.device) * 2.0 - 1.0)
    return (lap * col_scale).to(torch.bfloat16)


@dataclass(frozen=True)
class Call:
    """One quantization call of a workload: which tensor, layout, mode, RHT group."""
    tensor: str
    layout: int
    mode: int
    rht_group: int

    @property
    def name(self) -> str:
        g = f"g{self.rht_group}" if self.rht_group else "norht"
        return f"{self.tensor}.{LAYOUT_NAMES[self.layout]}.{MODE_NAMES[self.mode]}.{g}"


@dataclass
class Workload:
    name: str
    seed: int
    shapes: Dict[str, Tuple[int, int]]
    calls: List[Call] = field(default_factory=list)
    description: str = ""

    def tensors(self, device="cpu") -> Dict[str, torch.Tensor]:
        """The workload's bf16 tensors, drawn on `device` ("cpu" or a CUDA device)."""
        return _GENERATORS[self.name](self, device)

    def elements(self, call: Call) -> int:
        r, c = self.shapes[call.tensor]
        return r * c


def _small(w, device):
    g = _gen(w.seed, device)
    return {"x": normal(w.shapes["x"], 1.0, g)}


def _weight(w, device):
    g = _gen(w.seed, device)
    return {"w": outlier_normal(w.shapes["w"], 0.02, 0.01, 10.0, g)}


def _gradient(w, device):
    g = _gen(w.seed, device)
    return {"g": student_t3(w.shapes["g"], 1e-3, g)}


def _activation(w, device):
    g = _gen(w.seed, device)
    return {"a": laplace_channels(w.shapes["a"], g)}


def _mlp_up(w, device):
    g = _gen(w.seed, device)
    x = normal(w.shapes["x"], 1.0, g)
    wt = normal(w.shapes["w"], 0.02, g)
    dy = student_t3(w.shapes["dy"], 1e-4, g)
    return {"x": x, "w": wt, "dy": dy}


_GENERATORS = {"small": _small, "weight": _weight, "gradient": _gradient,
               "activation": _activation, "mlp_up": _mlp_up}


def small(rows=256, cols=256) -> Workload:
    """256x256 N(0,1), seed 0: RTN and SR with and without a 128-point RHT, MS-EDEN with it."""
    calls = [Call("x", ROWWISE, RTN, 0), Call("x", ROWWISE, RTN, 128),
             Call("x", ROWWISE, SR, 0), Call("x", ROWWISE, SR, 128),
             Call("x", ROWWISE, MS_EDEN, 128)]
    return Workload("small", 0, {"x": (rows, cols)}, calls, "256x256 N(0,1)")


def weight(rows=4096, cols=4096) -> Workload:
    """Weight-like 4096x4096 N(0, 0.02^2) with 1% outliers x10, seed 1: RTN, 4/6 and scale search row-wise."""
    calls = [Call("w", ROWWISE, RTN, 0), Call("w", ROWWISE, FOUR_OVER_SIX, 0), Call("w", ROWWISE, SCALE_SEARCH, 0)]
    return Workload("weight", 1, {"w": (rows, cols)}, calls, "4096x4096 N(0,0.02) + 1% x10 outliers")


def gradient(rows=8192, cols=4096) -> Workload:
    """Gradient-like 8192x4096 Student-t3 with std 1e-3, seed 2: MS-EDEN and SR, g=128, both layouts."""
    calls = [Call("g", lay, mode, 128) for mode in (MS_EDEN, SR) for lay in (ROWWISE, TRANSPOSED)]
    return Workload("gradient", 2, {"g": (rows, cols)}, calls, "8192x4096 Student-t3 std 1e-3")


def activation(rows=16384, cols=8192) -> Workload:
    """Activation-like 16384x8192 Laplace(0,1) x per-channel 10^U(-1,1), seed 3: IF4 with and without RHT."""
    calls = [Call("a", ROWWISE, IF4, 0), Call("a", ROWWISE, IF4, 128)]
    return Workload("activation", 3, {"a": (rows, cols)}, calls, "16384x8192 Laplace x log-uniform channel scale")


def mlp_up(tokens=16384, d_model=4096, d_ff=14336, seed=4) -> Workload:
    """One Llama-style MLP up-projection training step, seed 4.

    X [tokens, d_model] N(0,1), W [d_ff, d_model] N(0, 0.02^2), dY [tokens, d_ff]
    Student-t3 std 1e-4.  Forward Y = X W^T: RTN on X and W along d_model.
    Backward dX = dY W: MS-EDEN along d_ff on dY (row-wise) and W (transposed);
    dW = dY^T X: MS-EDEN along tokens on dY (transposed) and X (transposed).
    """
    calls = [Call("x", ROWWISE, RTN, 0), Call("w", ROWWISE, RTN, 0),
             Call("dy", ROWWISE, MS_EDEN, 128), Call("w", TRANSPOSED, MS_EDEN, 128),
             Call("dy", TRANSPOSED, MS_EDEN, 128), Call("x", TRANSPOSED, MS_EDEN, 128)]
    return Workload("mlp_up", seed, {"x": (tokens, d_model), "w": (d_ff, d_model), "dy": (tokens, d_ff)},
                    calls, "MLP up-projection step: X 16384x4096, W 14336x4096, dY 16384x14336")


def gemm_operand(rows: int, k: int, seed: int, scale_codes=None, device="cpu"):
    """Random bytes standing for one quantized GEMM operand (rows x k view):
    packed E2M1 codes (rows x k/2, every byte value equally likely) and E4M3
    scale bytes (rows x k/16) drawn uniformly from `scale_codes` (default:
    every finite positive code, 0x00..0x7E).  Plain integers, no quantization:
    for checking the GEMM on operands of known structure."""
    g = _gen(seed, device)
    codes = torch.randint(0, 256, (rows, k // 2), generator=g, dtype=torch.int32, device=device).to(torch.uint8)
    if scale_codes is None:
        scale_codes = list(range(0x7F))
    table = torch.tensor(list(scale_codes), dtype=torch.uint8, device=device)
    idx = torch.randint(0, len(table), (rows, k // 16), generator=g, dtype=torch.int64, device=device)
    return codes, table[idx]


ALL = {"small": small, "weight": weight, "gradient": gradient, "activation": activation, "mlp_up": mlp_up}


def bf16_bits(t: torch.Tensor):
    """bf16 tensor (CPU) -> numpy uint16 array of its bit patterns (no copy of semantics)."""
    return t.contiguous().view(torch.int16).numpy().view("uint16")
