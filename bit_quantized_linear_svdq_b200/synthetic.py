"""Seeded synthetic SVDQuant W4A4 checkpoints and activations.

This module draws random tensors with the shapes, dtypes and value
distributions of the workloads the SVDQuant W4A4 linear is exercised on
(diffusion-transformer projection shapes).  It holds none of the method's
arithmetic: it only samples numbers and stores their raw bit patterns.  The
weight tensors follow the checkpoint contract of "SVDQuant W4A4"
(vLLM-Omni svdquant.md, section "Checkpoint contract"):

    qweight        (N, K/2)  int8, two packed FP4 (E2M1) codes per byte
    wscales        (K/16, N) float8_e4m3fn
    proj_down      (K, R)    bfloat16
    proj_up        (N, R)    bfloat16
    smooth_factor  (K,)      bfloat16
    wcscales       (N,)      bfloat16
    wtscale        (1,)      bfloat16

For the rotated workload the generator returns a dense bf16 weight instead of
(qweight, wscales); the caller quantizes it (offline, per the rotation page's
W' = R W step) with whatever quantizer it trusts.

Every array is a numpy array of raw bits: uint16 for bf16, uint8 for e4m3 and
packed E2M1.  Both the CPU oracle and the CUDA path read these same bits.

Recipe (one torch.Generator per checkpoint, seeded, fixed draw order):
  x ~ N(0,1); a seed-chosen set of input channels (randperm) is scaled x30
  (4 channels for the tiny case, round(0.01*K) otherwise); smooth_factor ~
  U[0.5, 2]; qweight = uniform random bytes (every nibble is a valid E2M1
  code); wscales = e4m3(U[0.01, 0.1]); proj_down, proj_up ~ N(0, 0.02);
  wcscales = ones or U[0.8, 1.2]; wtscale a constant.  Each float tensor is
  drawn in fp32 and rounded to bf16 (round-to-nearest-even, torch's cast).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch


@dataclasses.dataclass
class Checkpoint:
    """One SVDQuant linear layer plus one batch of activations (raw bits)."""

    name: str
    M: int
    K: int
    N: int
    R: int
    rotate_block: int                 # 0 = no online rotation, else Hadamard block size
    x: np.ndarray                     # (M, K) uint16, bf16 bits
    smooth_factor: np.ndarray         # (K,) uint16, bf16 bits
    proj_down: np.ndarray             # (K, R) uint16, bf16 bits
    proj_up: np.ndarray               # (N, R) uint16, bf16 bits
    wcscales: np.ndarray              # (N,) uint16, bf16 bits
    wtscale: np.ndarray               # (1,) uint16, bf16 bits
    qweight: Optional[np.ndarray]     # (N, K/2) uint8 or None (dense_weight given)
    wscales: Optional[np.ndarray]     # (K/16, N) uint8 (e4m3 bits) or None
    dense_weight: Optional[np.ndarray] = None  # (N, K) uint16 bf16 bits (rotated case)
    outlier_channels: Optional[np.ndarray] = None


def _bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.bfloat16).contiguous().view(torch.int16).numpy().view(np.uint16).copy()


def _e4m3_bits(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float8_e4m3fn).contiguous().view(torch.uint8).numpy().copy()


def make_checkpoint(M: int, K: int, N: int, R: int, seed: int, *,
                    rotate_block: int = 0, n_outliers: Optional[int] = None,
                    wcscales: str = "ones", wtscale: float = 1.0,
                    dense_weight: bool = False, name: str = "custom") -> Checkpoint:
    """Draw one checkpoint + activation batch with the fixed draw order."""
    if K % 16:
        raise ValueError("K must be a multiple of 16 (checkpoint contract)")
    g = torch.Generator().manual_seed(int(seed))
    x = torch.randn((M, K), generator=g, dtype=torch.float32)
    if n_outliers is None:
        n_outliers = int(round(0.01 * K))
    ch = torch.randperm(K, generator=g)[:n_outliers]
    if M > 0 and n_outliers > 0:
        x[:, ch] *= 30.0
    smooth = torch.rand((K,), generator=g, dtype=torch.float32) * 1.5 + 0.5
    qweight = wsc = dense = None
    if dense_weight:
        dense = _bf16_bits(torch.randn((N, K), generator=g, dtype=torch.float32) * 0.02)
    else:
        qweight = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8).numpy().copy()
        wsc = _e4m3_bits(torch.rand((K // 16, N), generator=g, dtype=torch.float32) * 0.09 + 0.01)
    pd = torch.randn((K, R), generator=g, dtype=torch.float32) * 0.02
    pu = torch.randn((N, R), generator=g, dtype=torch.float32) * 0.02
    if wcscales == "ones":
        wc = torch.ones((N,), dtype=torch.float32)
    elif wcscales == "uniform":
        wc = torch.rand((N,), generator=g, dtype=torch.float32) * 0.4 + 0.8
    else:
        raise ValueError(wcscales)
    return Checkpoint(
        name=name, M=M, K=K, N=N, R=R, rotate_block=rotate_block,
        x=_bf16_bits(x), smooth_factor=_bf16_bits(smooth),
        proj_down=_bf16_bits(pd), proj_up=_bf16_bits(pu),
        wcscales=_bf16_bits(wc), wtscale=_bf16_bits(torch.tensor([wtscale])),
        qweight=qweight, wscales=wsc, dense_weight=dense,
        outlier_channels=ch.numpy().copy())


# The named workloads.  Sizes are diffusion-transformer attention and MLP
# projections (hidden 3072, MLP 12288) plus a small-batch / rank sweep.
CONFIGS = {
    "tiny_16x256x256_r32": dict(M=16, K=256, N=256, R=32, seed=0, n_outliers=4),
    "attn_proj_4096x3072x3072_r32": dict(M=4096, K=3072, N=3072, R=32, seed=1),
    "mlp_up_4096x3072x12288_r32": dict(M=4096, K=3072, N=12288, R=32, seed=2,
                                        wcscales="uniform", wtscale=0.5),
    "mlp_down_rot128_4096x12288x3072_r32": dict(M=4096, K=12288, N=3072, R=32, seed=3,
                                                 rotate_block=128, dense_weight=True),
}
for _m in (1, 16, 64, 256, 1024):
    CONFIGS[f"small_batch_m{_m}_4096x4096_r32"] = dict(M=_m, K=4096, N=4096, R=32, seed=4)
for _r in (16, 32, 64, 128):
    CONFIGS[f"rank_sweep_4096x3072x3072_r{_r}"] = dict(M=4096, K=3072, N=3072, R=_r, seed=4)

# The workload the headline throughput is quoted on.
HEADLINE = "attn_proj_4096x3072x3072_r32"


def load(name: str, M: Optional[int] = None) -> Checkpoint:
    """Named workload; ``M`` optionally overrides the batch (same seed)."""
    kw = dict(CONFIGS[name])
    if M is not None:
        kw["M"] = M
    return make_checkpoint(name=name, **kw)

