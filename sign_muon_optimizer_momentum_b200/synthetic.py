"""Seeded synthetic workloads for the Sign-Muon step.

This module only describes workloads (matrix shapes, worker count, variant,
hyper-parameters) and draws their random inputs.  It contains none of the
step's arithmetic, so that both the CUDA path and the CPU oracle can be fed
from it without sharing any computation.

The workloads stand in for the ones the SignMuon summary reports on (§4:
ResNet-50 on CIFAR-10 and nanoGPT); no dataset, checkpoint or model code is
used, only the weight-matrix shapes of those networks with Gaussian weights
and gradients ``G^(m) = G* + eps^(m)`` (a shared signal plus per-worker noise).
"""
from __future__ import annotations

import dataclasses
import hashlib
from typing import List, Sequence, Tuple

import torch

Shape = Tuple[int, int]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    shapes: Tuple[Shape, ...]
    n_workers: int
    ns_iters: int
    variant: str            # "int8" (integer-sum vote) or "pack1" (1-bit packed vote)
    w_dtype: str            # "f32" or "bf16"; gradients use the same dtype
    beta: float = 0.9
    eta: float = 0.02
    w_std: float = 0.02
    g_signal_std: float = 1.0
    g_noise_std: float = 1.0
    steps: int = 1
    polar: bool = False

    @property
    def params(self) -> int:
        return sum(r * c for r, c in self.shapes)

    @property
    def units(self) -> int:
        return len(self.shapes) * self.n_workers


def resnet50_shapes() -> List[Shape]:
    """(C_out, C_in*kh*kw) of the 53 conv layers of a bottleneck ResNet-50,
    plus the 2048x1000 classifier, in network order."""
    shapes: List[Shape] = [(64, 3 * 7 * 7)]
    c_in = 64
    for blocks, width, out in ((3, 64, 256), (4, 128, 512), (6, 256, 1024), (3, 512, 2048)):
        for blk in range(blocks):
            shapes.append((width, c_in))          # 1x1 reduce
            shapes.append((width, 9 * width))     # 3x3
            shapes.append((out, width))           # 1x1 expand
            if blk == 0:
                shapes.append((out, c_in))        # 1x1 projection shortcut
            c_in = out
    shapes.append((2048, 1000))
    return shapes


def nanogpt_small_shapes(layers: int = 12, d: int = 768) -> List[Shape]:
    out: List[Shape] = []
    for _ in range(layers):
        out += [(d, 3 * d), (d, d), (d, 4 * d), (4 * d, d)]
    return out


WORKLOADS = {
    # 256x256 fp32, M=4, k=1, int8 vote, one step.
    "single256": Workload("single256", ((256, 256),), 4, 1, "int8", "f32",
                          g_noise_std=2.0, steps=1),
    # nanoGPT-small matrices, bf16 weights, M=8, k=5, 1-bit vote, 10 steps.
    "nanogpt_small": Workload("nanogpt_small", tuple(nanogpt_small_shapes()), 8, 5,
                              "pack1", "bf16", g_noise_std=3.0, steps=10),
    # ResNet-50 conv/FC matrices, fp32, M=4, k=1, int8 vote, noise ratio 1:2.
    "resnet50": Workload("resnet50", tuple(resnet50_shapes()), 4, 1, "int8", "f32",
                         g_noise_std=2.0, steps=10),
    # Majority-vote Signum baseline (k = 0: the sign of the momentum itself) on
    # the nanoGPT-small matrices, the comparison the SignMuon summary reports.
    "signum_nanogpt_small": Workload("signum_nanogpt_small", tuple(nanogpt_small_shapes()), 8, 0,
                                     "pack1", "bf16", g_noise_std=3.0, steps=10),
    # 32 square 4096^2 bf16 matrices, M=16, k=5, 1-bit vote, local polar step.
    "square4096x32": Workload("square4096x32", tuple([(4096, 4096)] * 32), 16, 5,
                              "pack1", "bf16", g_noise_std=4.0, steps=3, polar=True),
}

# Vote/update sweep: total params 2^20 .. 2^30 in x4 steps, W as (P/1024, 1024).
VOTE_SWEEP_PARAMS = tuple(2 ** e for e in range(20, 31, 2))
VOTE_SWEEP_WORKERS = (2, 3, 8, 16, 64)
VOTE_SWEEP_ETA = 0.01


def _seed(*parts) -> int:
    h = hashlib.sha256(repr(parts).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def generator(device, *parts) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(*parts))
    return g


def torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def gaussian(shape: Sequence[int], std: float, device, *parts,
             dtype: torch.dtype = torch.float32) -> torch.Tensor:
    g = generator(device, *parts)
    x = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def initial_weights(wl: Workload, seed: int = 0, device="cpu") -> List[torch.Tensor]:
    dt = torch_dtype(wl.w_dtype)
    return [gaussian(s, wl.w_std, device, "W", seed, i, dtype=dt)
            for i, s in enumerate(wl.shapes)]


def gradient_signal(wl: Workload, seed: int = 0, device="cpu") -> List[torch.Tensor]:
    """G* per matrix (fixed for the run), fp32."""
    return [gaussian(s, wl.g_signal_std, device, "Gstar", seed, i)
            for i, s in enumerate(wl.shapes)]


def worker_gradient(wl: Workload, signal: torch.Tensor, mat: int, worker: int, step: int,
                    seed: int = 0, out: torch.Tensor = None) -> torch.Tensor:
    """G^(m) = G* + eps^(m), eps fresh per (step, worker), in the workload's dtype."""
    eps = gaussian(signal.shape, wl.g_noise_std, signal.device, "eps", seed, mat, worker, step)
    eps.add_(signal)
    if out is None:
        return eps.to(torch_dtype(wl.w_dtype))
    out.copy_(eps)
    return out


def vote_sweep_signs(params: int, n_workers: int, seed: int = 0, device="cpu",
                     chunk: int = 1 << 26):
    """Random +-1 sign vectors for the vote sweep, one int8 tensor per worker.

    Per entry a probability p ~ U(0,1) is drawn once; each worker's entry is
    +1 with probability p independently.  Yields (worker, int8 tensor) so
    large sweeps can be consumed one worker at a time.
    """
    p = torch.rand(params, generator=generator(device, "p", seed, params), device=device)
    for m in range(n_workers):
        g = generator(device, "bit", seed, params, m)
        s = torch.empty(params, dtype=torch.int8, device=device)
        for lo in range(0, params, chunk):
            hi = min(params, lo + chunk)
            r = torch.rand(hi - lo, generator=g, device=device)
            s[lo:hi] = torch.where(r < p[lo:hi], 1, -1).to(torch.int8)
        yield m, s
