"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no attention arithmetic: it only draws random numbers.
Q, K, V and dO are i.i.d. N(0, 1), drawn in that order (fp32) from one
``torch.Generator('cpu')`` seeded with ``seed``, then rounded to the working
dtype.  Both the CUDA path and the oracle receive the same rounded values
(the oracle upcasts them to fp64).
"""
import torch

DTYPES = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32, "f32": torch.float32}


def make_inputs(B, Nq, Nk, Hq, Hkv, d, seed, dtype="bf16", with_dout=True, scale_q=1.0):
    """Return a dict of CPU tensors q, k, v (and do) in ``dtype``.

    Layout: q/do ``[B, Nq, Hq, d]``, k/v ``[B, Nk, Hkv, d]``, d contiguous.
    ``scale_q`` multiplies Q before rounding (a "peaked softmax" stress variant).
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    dt = DTYPES[dtype]
    q = torch.randn((B, Nq, Hq, d), generator=g, dtype=torch.float32)
    k = torch.randn((B, Nk, Hkv, d), generator=g, dtype=torch.float32)
    v = torch.randn((B, Nk, Hkv, d), generator=g, dtype=torch.float32)
    out = {"q": (q * scale_q).to(dt), "k": k.to(dt), "v": v.to(dt)}
    if with_dout:
        out["do"] = torch.randn((B, Nq, Hq, d), generator=g, dtype=torch.float32).to(dt)
    return out


def config_seed(k: int) -> int:
    """Seed of the k-th named workload (1-based)."""
    return 1000 + k


def sweep_seed(n: int, d: int) -> int:
    """Seed of a sequence-length sweep point (N, d)."""
    return 1000 * 3 + (n // 512) * 10 + d // 64
