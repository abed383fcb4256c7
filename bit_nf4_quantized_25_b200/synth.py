"""Seeded synthetic inputs for the NF4 + LoRA linear layer.

Holds random draws only -- none of the method's arithmetic -- so both the CUDA
path and the CPU oracle can be fed the same tensors. There are no real model
weights or datasets here: Llama-shaped random tensors stand in for them.

Recipe (one per workload; shapes are out_features x in_features):
  * tiny      : W 256x256 ~ N(0, 0.02); A, B ~ N(0, 0.01); x, grad_h ~ N(0, 1);
                M = 8, r = 4, alpha = 8.
  * decode7b  : W 4096x4096, 11008x4096, 4096x11008 ~ N(0, 0.02); r = 16,
                alpha = 32; M in {1, 4, 16}; forward only.
  * train7b   : q/k/v/o 4096x4096, gate/up 11008x4096, down 4096x11008;
                M = 4096 (2 x 2048); r = 16, alpha = 32; fwd + bwd_x.
  * l70b      : W 8192x8192, 28672x8192, 8192x28672 ~ N(0, 0.015); r = 64,
                alpha = 16; M in {1, 16, 4096}; fwd + bwd_x.
  * bulk      : 32 layers of the 7B shapes, W ~ 0.02 * Student-t(4) with 0.1 %
                of the entries (a seeded permutation) multiplied by 20.
Seeds: workload i uses base seed 1000 * i; tensor j of a workload draws with
seed base + j, in the order W, A, B, x, grad_h.
"""
from __future__ import annotations

import dataclasses

import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    """N(0, std^2) drawn in fp32 with the seeded generator, rounded to bf16."""
    g = _gen(seed, device)
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    return (t * std).to(torch.bfloat16)


def student_t_bf16(shape, scale: float, seed: int, df: int = 4, outlier_frac: float = 1e-3,
                   outlier_mult: float = 20.0, device="cpu") -> torch.Tensor:
    """scale * z / sqrt(chi2_df / df), chi2 as a sum of df squared normals; then a
    seeded fraction of the entries is multiplied by outlier_mult."""
    g = _gen(seed, device)
    z = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    chi = torch.zeros_like(z)
    for _ in range(df):
        e = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
        chi.add_(e * e)
    t = z / torch.sqrt(chi / df)
    flat = t.view(-1)
    n_out = int(round(flat.numel() * outlier_frac))
    if n_out:
        idx = torch.randperm(flat.numel(), generator=g, device=device)[:n_out]
        flat[idx] *= outlier_mult
    return (t * scale).to(torch.bfloat16)


@dataclasses.dataclass(frozen=True)
class LayerCase:
    name: str
    n_out: int
    k_in: int
    M: int
    r: int
    alpha: float
    w_std: float
    seed: int


def tiny_case() -> LayerCase:
    return LayerCase("tiny", 256, 256, 8, 4, 8.0, 0.02, 0)


SHAPES_7B = {"q": (4096, 4096), "k": (4096, 4096), "v": (4096, 4096), "o": (4096, 4096),
             "gate": (11008, 4096), "up": (11008, 4096), "down": (4096, 11008)}
SHAPES_70B = {"attn": (8192, 8192), "up": (28672, 8192), "down": (8192, 28672)}


def decode7b_cases():
    out = []
    for j, (nm, (n, k)) in enumerate([("4096x4096", (4096, 4096)), ("11008x4096", (11008, 4096)),
                                      ("4096x11008", (4096, 11008))]):
        for M in (1, 4, 16):
            out.append(LayerCase(f"decode7b_{nm}_M{M}", n, k, M, 16, 32.0, 0.02, 1000 + 10 * j))
    return out


def train7b_cases():
    return [LayerCase(f"train7b_{nm}", n, k, 4096, 16, 32.0, 0.02, 2000 + 10 * j)
            for j, (nm, (n, k)) in enumerate(SHAPES_7B.items())]


def l70b_cases():
    out = []
    for j, (nm, (n, k)) in enumerate(SHAPES_70B.items()):
        for M in (1, 16, 4096):
            out.append(LayerCase(f"l70b_{nm}_M{M}", n, k, M, 64, 16.0, 0.015, 3000 + 10 * j))
    return out


def layer_inputs(case: LayerCase, device="cpu", need_grad=True):
    """W, A, B, x, grad_h for one layer case (bf16 tensors on `device`)."""
    s = case.seed
    W = normal_bf16((case.n_out, case.k_in), case.w_std, s + 0, device)
    A = normal_bf16((case.r, case.k_in), 0.01, s + 1, device)
    B = normal_bf16((case.n_out, case.r), 0.01, s + 2, device)
    x = normal_bf16((case.M, case.k_in), 1.0, s + 3, device)
    gh = normal_bf16((case.M, case.n_out), 1.0, s + 4, device) if need_grad else None
    return W, A, B, x, gh


def bulk_tensor(layer: int, name: str, device="cpu") -> torch.Tensor:
    """One tensor of the 32-layer 7B stack used by the bulk quantise round trip."""
    names = list(SHAPES_7B)
    j = layer * len(names) + names.index(name)
    n, k = SHAPES_7B[name]
    return student_t_bf16((n, k), 0.02, 4000 + j, device=device)


def bf16_bits(t: torch.Tensor):
    """uint16 view of a bf16 tensor as a numpy array (host copy)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")
