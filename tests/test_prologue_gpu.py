"""GPU parity of the fused step with its prologue (gdn_chunk_wy_fused_raw):
raw key rows normalised and per-token log-gates summed chunk-locally inside
the kernel, against the oracle's normalisation, cumulative sum and fused step.
"""
import numpy as np
import pytest
import torch

import oracle as O
from gated_deltanet_chunk_02_b200 import gdn
from gated_deltanet_chunk_02_b200.inputs import Workload, make_inputs, as_f64_numpy

from helpers import TOL_BF16, TOL_F32, rel, per_chunk_max_rel

pytestmark = pytest.mark.gpu


def reference(inp, w, N, mask, S, gated):
    Kn = O.l2_normalize_rows(as_f64_numpy(inp["K"]))
    g = O.chunk_cumsum(as_f64_numpy(inp["loggate"]), w.k)
    c = {"K": O.to_chunks(Kn, w.k), "V": O.to_chunks(as_f64_numpy(inp["V"]), w.k),
         "beta": O.to_chunks(as_f64_numpy(inp["beta"]), w.k), "g": O.to_chunks(g, w.k)}
    A = O.build_A(c["K"], c["beta"], c["g"])
    T = O.invert_neumann(A, N, bool(mask), S)
    W, U = O.wy(T, c["K"], c["V"], c["beta"], c["g"] if gated else None)
    return Kn, g, T, W, U


def run(inp, w, N, mask, S, gated, outputs=True):
    d = {key: v.cuda() for key, v in inp.items()}
    W = torch.empty_like(d["K"])
    U = torch.empty_like(d["V"])
    T = torch.empty(w.B, w.H, w.T // w.k, w.k, w.k, device="cuda")
    Ko = torch.full_like(d["K"], float("nan")) if outputs else None
    go = torch.full_like(d["loggate"], float("nan")) if outputs else None
    gdn.gdn_chunk_wy_fused_raw(d["K"], d["V"], d["beta"], d["loggate"], N, mask, S, int(gated),
                               W, U, T, Ko, go, k=w.k)
    assert gdn.gdn_get_status() == gdn.GDN_OK
    return W, U, T, Ko, go


@pytest.mark.parametrize("k", [32, 64, 128])
@pytest.mark.parametrize("N,mask,S,gated", [(3, 1, 0, 0), (3, 1, 8, 1), (2, 0, 3, 0)])
def test_prologue_matches_oracle(k, N, mask, S, gated):
    w = Workload(B=1, H=3, T=3 * k, k=k, dtype="bf16")      # 9 chunks, a ragged last tile
    inp = make_inputs(w, seed=51 + k, raw_keys=True)
    W, U, T, Ko, go = run(inp, w, N, mask, S, gated)
    Kn, g, Tr, Wr, Ur = reference(inp, w, N, mask, S, gated)
    assert rel(Ko, Kn) <= TOL_BF16 and torch.isfinite(Ko).all()
    assert rel(go, g) <= TOL_F32 and torch.isfinite(go).all()
    assert rel(T, Tr) <= TOL_BF16
    assert per_chunk_max_rel(T, Tr) <= TOL_BF16
    assert rel(W, Wr) <= TOL_BF16
    assert rel(U, Ur) <= TOL_BF16


def test_prologue_equals_prepared_inputs_path():
    """Feeding the kernel's own normalised keys and cumulative gates to the
    plain fused step gives the same W, U and T bits."""
    w = Workload(B=2, H=2, T=512, k=64, dtype="bf16")
    inp = make_inputs(w, seed=57, raw_keys=True)
    W1, U1, T1, Ko, go = run(inp, w, 3, 1, 8, 1)
    d = {key: v.cuda() for key, v in inp.items()}
    W2, U2 = torch.empty_like(W1), torch.empty_like(U1)
    T2 = torch.empty_like(T1)
    gdn.gdn_chunk_wy_fused(Ko, d["V"], d["beta"], go, 3, 1, 8, 1, W2, U2, T2, k=64)
    assert gdn.gdn_get_status() == gdn.GDN_OK
    assert torch.equal(W1, W2) and torch.equal(U1, U2) and torch.equal(T1, T2)


def test_prologue_scale_invariance_and_optional_outputs():
    """Scaling a key row leaves the result unchanged up to bf16 rounding of
    the scaled input; the optional outputs may be omitted."""
    w = Workload(B=1, H=2, T=256, k=64, dtype="bf16")
    inp = make_inputs(w, seed=58, raw_keys=True)
    W1, U1, _, _, _ = run(inp, w, 3, 1, 8, 0, outputs=False)
    inp2 = dict(inp)
    inp2["K"] = (inp["K"].float() * 4.0).to(torch.bfloat16)      # exact in bf16
    W2, U2, _, _, _ = run(inp2, w, 3, 1, 8, 0, outputs=False)
    assert torch.equal(W1, W2) and torch.equal(U1, U2)
