"""Seeded synthetic inputs for the MicroAdam step: shapes and generators only.

This module holds none of the optimizer's arithmetic. It is the one module the
tests, the benchmark and the CPU oracle's callers share: parameter vectors
~N(0, 0.02) in fp32 and bf16 gradients of the distributions the workloads name
(i.i.d. N(0, 1); Student-t with 3 degrees of freedom scaled by 1e-3, optionally
with a per-tensor scale). The model-shaped workloads stand in for the
fine-tuning runs of "MicroAdam (Sparse-Gradient Adaptive Optimization with
Quantized Error Feedback)", paragraph 4 (BERT-base, LLaMA-2 7B); no dataset or
trained weight is used.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


# ------------------------------------------------------------------ shapes
def bert_base_shapes() -> list[tuple[int, ...]]:
    """BERT-base parameter tensors in a fixed order (embeddings, 12 layers)."""
    h, f, L = 768, 3072, 12
    shapes: list[tuple[int, ...]] = [(30522, h), (512, h)]
    for _ in range(L):
        shapes += [(h, h), (h,), (h, h), (h,), (h, h), (h,), (h, h), (h,),  # q k v o
                   (h,), (h,),                                              # LayerNorm
                   (f, h), (f,), (h, f), (h,),                              # FFN
                   (h,), (h,)]                                              # LayerNorm
    return shapes


def llama2_7b_shapes() -> list[tuple[int, ...]]:
    """LLaMA-2-7B parameter tensors: embed, 32 x (q,k,v,o, gate,up,down, 2 norms), norm, head."""
    h, f, V, L = 4096, 11008, 32000, 32
    shapes: list[tuple[int, ...]] = [(V, h)]
    for _ in range(L):
        shapes += [(h, h)] * 4 + [(f, h), (f, h), (h, f)] + [(h,), (h,)]
    shapes += [(h,), (V, h)]
    return shapes


def numel(shapes) -> int:
    total = 0
    for s in shapes:
        n = 1
        for x in s:
            n *= x
        total += n
    return total


@dataclass
class Workload:
    """One optimizer workload: a flat parameter vector cut into tensors."""
    name: str
    d: int
    Bd: int
    kb: int
    m: int
    grad: str                      # "normal" | "t3" | "t3_tensor_scaled"
    steps: int
    shapes: list = field(default_factory=list)
    lr: float = 1e-3
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    wd: float = 0.0
    seed: int = 0x5EED0000
    per_tensor: bool = False       # blocks cut per tensor of ``shapes`` (else over the flat vector)
    params: str = "f32"            # parameter storage: "f32" | "bf16"

    def segments(self):
        """Tensor lengths when blocks are cut per tensor, else None."""
        return [numel([s]) for s in self.shapes] if self.per_tensor else None

    def tensor_sizes(self) -> list[int]:
        if not self.shapes:
            return [self.d]
        return [numel([s]) for s in self.shapes]


def k_for_density(Bd: int, density: float = 0.01) -> int:
    """k_b for a 1 % block density: ceil(B_d / 100) (164 at B_d = 16384)."""
    import math
    return int(math.ceil(Bd * density - 1e-9))


def flat_small() -> Workload:
    """Flat d = 2^20, N(0,1) gradients, B_d = 16384, k_b = 164, m = 10, 20 steps."""
    return Workload("flat_d2^20_normal", 1 << 20, 16384, 164, 10, "normal", 20,
                    seed=0x5EED0000)


def flat_134m() -> Workload:
    """Flat d = 2^27, 1e-3 * t(3) gradients, B_d = 16384, k_b = 164, m = 10, 50 steps."""
    return Workload("flat_d2^27_t3", 1 << 27, 16384, 164, 10, "t3", 50, seed=0x5EED0001)


def bert_base(Bd: int = 16384 // 2) -> Workload:
    """BERT-base-shaped list, t(3) gradients with per-tensor scale, 1 % density, m = 10."""
    shapes = bert_base_shapes()
    return Workload(f"bert_base_Bd{Bd}", numel(shapes), Bd, k_for_density(Bd), 10,
                    "t3_tensor_scaled", 50, shapes=shapes, seed=0x5EED0002)


def llama2_7b() -> Workload:
    """LLaMA-2-7B-shaped list (d = 6,738,415,616), t(3) per-tensor-scaled, B_d = 16384, k_b = 164, m = 10."""
    shapes = llama2_7b_shapes()
    return Workload("llama2_7b", numel(shapes), 16384, 164, 10, "t3_tensor_scaled", 10,
                    shapes=shapes, seed=0x5EED0003)


def flat_1g(m: int) -> Workload:
    """Window sweep: flat d = 2^30, N(0,1) gradients, B_d = 16384, k_b = 164, window m."""
    return Workload(f"flat_d2^30_m{m}", 1 << 30, 16384, 164, m, "normal", 30,
                    seed=0x5EED0004)


# ------------------------------------------------------------------ generators
def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & ((1 << 63) - 1))
    return g


def tensor_scale(j: int) -> float:
    """Per-tensor gradient scale 1e-3 * 2^((j mod 7) - 3)."""
    return 1e-3 * 2.0 ** ((j % 7) - 3)


def make_params(d: int, seed: int = 7, device="cpu", chunk: int = 1 << 26) -> torch.Tensor:
    """fp32 parameters ~N(0, 0.02)."""
    out = torch.empty(d, dtype=torch.float32, device=device)
    g = _gen(device, seed)
    for s in range(0, d, chunk):
        e = min(d, s + chunk)
        out[s:e].normal_(0.0, 0.02, generator=g)
    return out


def _fill_grad(dst: torch.Tensor, kind: str, scale: float, g: torch.Generator):
    n = dst.numel()
    if kind == "normal":
        x = torch.randn(n, generator=g, device=dst.device, dtype=torch.float32)
    elif kind.startswith("t3"):
        # Student-t(3) = Z / sqrt(chi2_3 / 3), chi2_3 = sum of three squared normals.
        z = torch.randn(4, n, generator=g, device=dst.device, dtype=torch.float32)
        chi = z[1].square_().add_(z[2].square_()).add_(z[3].square_()).div_(3.0)
        x = z[0].div_(chi.sqrt_())
        x.mul_(scale)
    else:
        raise ValueError(kind)
    dst.copy_(x)


def make_grads(w: Workload, step: int, device="cpu", out: torch.Tensor | None = None,
               start: int = 0, length: int | None = None, chunk: int = 1 << 24) -> torch.Tensor:
    """bf16 gradients of workload ``w`` for optimizer step ``step``.

    Element i of tensor j draws from a generator seeded by (workload, step, j,
    i // chunk), so any slice [start, start + length) of the flat vector is
    reproducible on its own (one rank's shard) and equals the same slice of
    the whole vector.
    """
    if length is None:
        length = w.d - start
    if out is None:
        out = torch.empty(length, dtype=torch.bfloat16, device=device)
    assert out.numel() == length
    end = start + length
    offset = 0
    for j, n in enumerate(w.tensor_sizes()):
        lo, hi = max(start, offset), min(end, offset + n)
        if lo < hi:
            scale = tensor_scale(j) if w.grad == "t3_tensor_scaled" else 1e-3
            for c in range((lo - offset) // chunk, (hi - offset - 1) // chunk + 1):
                c0 = offset + c * chunk
                c1 = min(offset + n, c0 + chunk)
                g = _gen(out.device, ((w.seed * 1000003 + step) * 7919 + j) * 104729 + c)
                buf = torch.empty(c1 - c0, dtype=torch.bfloat16, device=out.device)
                _fill_grad(buf, w.grad, scale, g)
                a, b = max(lo, c0), min(hi, c1)
                out[a - start: b - start].copy_(buf[a - c0: b - c0])
        offset += n
    return out


def grads_from_values(values, device="cpu") -> torch.Tensor:
    """bf16 gradient tensor from explicit values (edge-case fixtures)."""
    return torch.as_tensor(values, dtype=torch.float32, device=device).to(torch.bfloat16)


def bf16_bits(x: torch.Tensor):
    """The raw uint16 bits of a bf16 tensor, as a numpy array (CPU copy)."""
    return x.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")
