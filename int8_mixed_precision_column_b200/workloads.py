"""Seeded synthetic inputs for the LLM.int8() forward linear layer.

This module only draws random numbers: it holds none of the method's
arithmetic (no thresholding, no quantisation, no matmul), so both the CUDA
path and the CPU oracle may consume what it produces.

Shapes follow the workloads the method is described on: the 64->64 toy
layers of the bitsandbytes ``Linear8bitLt`` docstring example, a
Llama-7B-width prefill, and BLOOM-176B's FFN-up projection (hidden 14336,
FFN 57344) in decode and prefill form, plus an outlier-density sweep.
Outlier feature dimensions ("systematically-emergent outlier feature
dimensions", inference-research record, Activation scheme) are planted as
whole columns whose magnitude is drawn from U(lo, hi) with an independent
random sign per element.

Every generator takes ``device``: ``"cpu"`` (torch CPU generator) or
``"cuda"`` (torch CUDA generator).  The two devices give different bytes for
the same seed; a test or benchmark draws once and hands the same tensors to
both sides.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass
class LinearProblem:
    """One forward problem: X [T,K] fp16, W [N,K] fp16, bias [N] fp16 or None."""

    name: str
    X: torch.Tensor
    W: torch.Tensor
    bias: torch.Tensor | None
    threshold: float
    planted_cols: list[int] = field(default_factory=list)

    @property
    def T(self) -> int:
        return self.X.shape[0]

    @property
    def K(self) -> int:
        return self.X.shape[1]

    @property
    def N(self) -> int:
        return self.W.shape[0]


def _gen(device: str, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal(shape, std: float, g: torch.Generator, device: str) -> torch.Tensor:
    return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(torch.float16)


def _plant_columns(X: torch.Tensor, cols: list[int], lo: float, hi: float, g: torch.Generator) -> None:
    """Overwrite whole columns of X with +-U(lo, hi), sign drawn per element."""
    if not cols:
        return
    T = X.shape[0]
    c = torch.tensor(cols, dtype=torch.long, device=X.device)
    mag = lo + (hi - lo) * torch.rand((T, len(cols)), generator=g, device=X.device, dtype=torch.float32)
    sign = torch.where(
        torch.rand((T, len(cols)), generator=g, device=X.device, dtype=torch.float32) < 0.5, -1.0, 1.0
    )
    X[:, c] = (mag * sign).to(torch.float16)


def _pick_cols(K: int, n: int, g: torch.Generator, device: str) -> list[int]:
    """n distinct feature dimensions chosen by a seeded permutation, ascending."""
    if n == 0:
        return []
    perm = torch.randperm(K, generator=g, device=device)[:n]
    return sorted(int(v) for v in perm.cpu().tolist())


def make_problem(
    name: str,
    T: int,
    K: int,
    N: int,
    *,
    n_planted: int = 0,
    planted_cols: list[int] | None = None,
    lo: float = 6.0,
    hi: float = 60.0,
    w_std: float = 0.02,
    bias_std: float | None = None,
    threshold: float = 6.0,
    seed: int = 0,
    device: str = "cpu",
) -> LinearProblem:
    """Generic seeded problem: X ~ N(0,1) with planted outlier columns, W ~ N(0, w_std^2)."""
    g = _gen(device, seed)
    X = _normal((T, K), 1.0, g, device)
    cols = list(planted_cols) if planted_cols is not None else _pick_cols(K, n_planted, g, device)
    _plant_columns(X, cols, lo, hi, g)
    W = _normal((N, K), w_std, g, device)
    bias = _normal((N,), bias_std, g, device) if bias_std is not None else None
    return LinearProblem(name, X, W, bias, threshold, cols)


def toy(seed: int = 0, device: str = "cpu") -> LinearProblem:
    """64->64 toy layer with bias; columns 3 and 17 are +-U(8,20) in every row."""
    return make_problem(
        "toy_64x64", 16, 64, 64, planted_cols=[3, 17], lo=8.0, hi=20.0,
        w_std=0.05, bias_std=0.01, seed=seed, device=device,
    )


def llama7b_prefill(seed: int = 0, device: str = "cpu") -> LinearProblem:
    """Llama-7B width prefill: X [2048,4096], 6 outlier dims U(6,60); W [4096,4096]; zero bias."""
    p = make_problem(
        "llama7b_prefill_2048x4096x4096", 2048, 4096, 4096, n_planted=6, lo=6.0, hi=60.0,
        w_std=0.02, bias_std=None, seed=seed, device=device,
    )
    p.bias = torch.zeros(4096, dtype=torch.float16, device=device)
    return p


def bloom_ffn_up_decode(T: int, seed: int = 0, device: str = "cpu") -> LinearProblem:
    """BLOOM-176B FFN-up decode: X [T,14336] with 8 outlier dims +-U(6,40); W [57344,14336]."""
    return make_problem(
        f"bloom176b_ffn_up_decode_T{T}", T, 14336, 57344, n_planted=8, lo=6.0, hi=40.0,
        w_std=0.02, bias_std=0.01, seed=seed, device=device,
    )


def bloom_ffn_up_prefill(T: int = 8192, seed: int = 0, device: str = "cpu") -> LinearProblem:
    """BLOOM-176B FFN-up prefill: X [8192,14336] with 8 outlier dims +-U(6,40); W [57344,14336]."""
    return make_problem(
        f"bloom176b_ffn_up_prefill_T{T}", T, 14336, 57344, n_planted=8, lo=6.0, hi=40.0,
        w_std=0.02, bias_std=0.01, seed=seed, device=device,
    )


def density_sweep(n_dims: int, threshold: float = 6.0, seed: int = 0, device: str = "cpu") -> LinearProblem:
    """Outlier-density sweep: X [4096,8192] with n_dims columns U(6,60); W [8192,8192]; zero bias."""
    p = make_problem(
        f"density_sweep_nout{n_dims}_thr{threshold:g}", 4096, 8192, 8192, n_planted=n_dims,
        lo=6.0, hi=60.0, w_std=0.02, bias_std=None, threshold=threshold, seed=seed, device=device,
    )
    p.bias = torch.zeros(8192, dtype=torch.float16, device=device)
    return p
