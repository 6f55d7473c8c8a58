"""Seeded synthetic inputs for the chunk-wise Gated DeltaNet hot path.

This module only draws random tensors; it holds none of the method's arithmetic
(no A, no inverse, no WY factors).  Both the CUDA path (through the tests and
``bench.py``) and the CPU oracle are fed from here, so they see the same bits.

Recipe (the distributions of the workloads the method is evaluated on):

* keys ``K``: each row drawn N(0, 1), then L2-normalised over the head dim;
* values ``V``: N(0, 1);
* write strengths ``beta = sigmoid(N(0, 1))``;
* per-token log-gates ``-softplus(N(0, 1))`` (times ``gate_scale``, 1 by
  default), and ``g`` their cumulative sum restarted at every chunk of ``k``
  tokens (summed in float64, stored as float32);
* queries ``Q`` (only when asked for): drawn like ``K``;
* optionally (``key_corr = rho > 0``) keys that share one direction: each
  normalised row becomes ``sqrt(1 - rho^2) k + rho u`` (renormalised), with
  ``u`` a unit vector drawn from a second generator, so the other draws are
  unchanged.  Correlated keys make ``A`` larger and the method's residual
  correction matter more (a stress input, not one of the workloads).

Draw order from one ``torch.Generator`` seeded with ``seed``: K, V,
beta-logits, gate-logits, then Q.  K, V and Q are cast to the requested dtype
after drawing; beta, g and the log-gates stay float32.

Decode inputs (``make_decode_inputs``) use the same distributions for one or
a few tokens per sequence, with grouped heads (``Hk`` query/key heads, ``Hv``
value heads) and a carried float32 state ``S0 ~ N(0, 1/d)`` per value head.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Workload:
    """Shape of one batch of chunked sequences (head-major, chunk-contiguous)."""

    B: int
    H: int
    T: int
    k: int
    d: int = 128
    dtype: str = "bf16"

    @property
    def n_chunks(self) -> int:
        return self.B * self.H * (self.T // self.k)


def chunk_cumsum(loggate: torch.Tensor, k: int) -> torch.Tensor:
    """Cumulative sum of ``loggate`` over its last axis, restarted every ``k`` entries.

    Summed in float64 and returned as float32.
    """
    *lead, T = loggate.shape
    x = loggate.to(torch.float64).reshape(*lead, T // k, k)
    return torch.cumsum(x, dim=-1).reshape(*lead, T).to(torch.float32)


def make_inputs(w: Workload, seed: int = 0, with_q: bool = False,
                gate_scale: float = 1.0, raw_keys: bool = False, key_corr: float = 0.0) -> dict:
    """Draw one batch of inputs for workload ``w`` on the CPU.

    Returns a dict of CPU tensors: ``K``, ``V`` (``[B,H,T,d]`` in ``w.dtype``),
    ``beta``, ``loggate``, ``g`` (``[B,H,T]`` float32) and, if ``with_q``,
    ``Q`` (``[B,H,T,d]`` in ``w.dtype``).  ``raw_keys`` leaves the key rows
    un-normalised (same draws, for the kernels that normalise them);
    ``key_corr`` mixes a shared unit direction into every key row (above).
    """
    if w.T % w.k:
        raise ValueError("T must be a multiple of the chunk size k")
    gen = torch.Generator().manual_seed(seed)
    shp = (w.B, w.H, w.T, w.d)
    K = torch.randn(shp, generator=gen, dtype=torch.float32)
    if key_corr > 0.0:
        ugen = torch.Generator().manual_seed(seed * 1000003 + 424242)
        u = torch.randn(w.d, generator=ugen, dtype=torch.float32)
        norm = K.norm(dim=-1, keepdim=True)
        Kc = (1.0 - key_corr ** 2) ** 0.5 * (K / norm) + key_corr * (u / u.norm())
        K = Kc / Kc.norm(dim=-1, keepdim=True) * norm        # the raw rows keep their norms
    if not raw_keys:
        K = K / K.norm(dim=-1, keepdim=True)
    V = torch.randn(shp, generator=gen, dtype=torch.float32)
    beta = torch.sigmoid(torch.randn(shp[:3], generator=gen, dtype=torch.float32))
    loggate = -torch.nn.functional.softplus(
        torch.randn(shp[:3], generator=gen, dtype=torch.float32)) * gate_scale
    out = {
        "K": K.to(DTYPES[w.dtype]).contiguous(),
        "V": V.to(DTYPES[w.dtype]).contiguous(),
        "beta": beta.contiguous(),
        "loggate": loggate.contiguous(),
        "g": chunk_cumsum(loggate, w.k).contiguous(),
    }
    if with_q:
        Q = torch.randn(shp, generator=gen, dtype=torch.float32)
        Q = Q / Q.norm(dim=-1, keepdim=True)
        out["Q"] = Q.to(DTYPES[w.dtype]).contiguous()
    return out


def make_decode_inputs(B: int, Hk: int, Hv: int, n: int, d: int = 128, dtype: str = "bf16",
                       seed: int = 0) -> dict:
    """Draw inputs of ``n`` decode steps on the CPU.

    Draw order: K, V, beta-logits, gate-logits, Q, S0.  Returns ``Q, K``
    (``[B,Hk,n,d]``, dtype), ``V`` (``[B,Hv,n,d]``, dtype), ``beta, loggate``
    (``[B,Hv,n]`` float32, the per-token log-gates) and ``S0``
    (``[B,Hv,d,d]`` float32).
    """
    gen = torch.Generator().manual_seed(seed)
    K = torch.randn((B, Hk, n, d), generator=gen, dtype=torch.float32)
    K = K / K.norm(dim=-1, keepdim=True)
    V = torch.randn((B, Hv, n, d), generator=gen, dtype=torch.float32)
    beta = torch.sigmoid(torch.randn((B, Hv, n), generator=gen, dtype=torch.float32))
    loggate = -torch.nn.functional.softplus(
        torch.randn((B, Hv, n), generator=gen, dtype=torch.float32))
    Q = torch.randn((B, Hk, n, d), generator=gen, dtype=torch.float32)
    Q = Q / Q.norm(dim=-1, keepdim=True)
    S0 = torch.randn((B, Hv, d, d), generator=gen, dtype=torch.float32) / d ** 0.5
    return {
        "Q": Q.to(DTYPES[dtype]).contiguous(),
        "K": K.to(DTYPES[dtype]).contiguous(),
        "V": V.to(DTYPES[dtype]).contiguous(),
        "beta": beta.contiguous(),
        "loggate": loggate.contiguous(),
        "S0": S0.contiguous(),
    }


def as_f64_numpy(t: torch.Tensor):
    """Upcast a CPU tensor (any float dtype) to a float64 numpy array."""
    return t.detach().to("cpu", torch.float64).numpy()
