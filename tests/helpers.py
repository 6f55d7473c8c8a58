"""Shared helpers for the tests: seeded inputs, oracle results, comparisons."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
from gated_deltanet_chunk_02_b200.inputs import Workload, make_inputs, as_f64_numpy

# Tolerances (relative Frobenius error per output tensor).
TOL_F32 = 1e-5      # float32 data, float32 arithmetic
TOL_BF16 = 1e-2     # bf16 data, tensor-core products with fp32 accumulation


def tol_for(dtype: str) -> float:
    return TOL_F32 if dtype == "f32" else TOL_BF16


def to_dev(x: torch.Tensor) -> torch.Tensor:
    return x.to("cuda").contiguous()


def chunked(inp: dict, w: Workload) -> dict:
    """float64 numpy views of the inputs as chunk batches [nc, k, ...]."""
    return {
        "K": O.to_chunks(as_f64_numpy(inp["K"]), w.k),
        "V": O.to_chunks(as_f64_numpy(inp["V"]), w.k),
        "beta": O.to_chunks(as_f64_numpy(inp["beta"]), w.k),
        "g": O.to_chunks(as_f64_numpy(inp["g"]), w.k),
    }


def oracle_A32(inp: dict, w: Workload) -> np.ndarray:
    """The oracle's A for these inputs, rounded to float32 (the stored input of
    the standalone inversion kernels)."""
    c = chunked(inp, w)
    return O.build_A(c["K"], c["beta"], c["g"]).astype(np.float32)


def A_tensor(A32: np.ndarray, w: Workload) -> torch.Tensor:
    return torch.from_numpy(A32).reshape(w.B, w.H, w.T // w.k, w.k, w.k)


def rel(x, ref) -> float:
    if isinstance(x, torch.Tensor):
        x = x.detach().to("cpu", torch.float64).numpy()
    return O.rel_fro(np.asarray(x, np.float64).reshape(np.shape(ref)), ref)


def per_chunk_max_rel(x, ref) -> float:
    """Largest per-chunk relative Frobenius error ([nc, ...] arrays)."""
    if isinstance(x, torch.Tensor):
        x = x.detach().to("cpu", torch.float64).numpy()
    x = np.asarray(x, np.float64).reshape(ref.shape[0], -1)
    r = ref.reshape(ref.shape[0], -1)
    num = np.linalg.norm(x - r, axis=1)
    den = np.maximum(np.linalg.norm(r, axis=1), 1e-300)
    return float((num / den).max())
