"""GPU parity of the full chunk-wise forward (gdn_forward) against the oracle's
chunk form, which is itself pinned to the token-by-token gated delta rule.

Small cases compare every output; the long-context configuration
(B=1, H=16, T=65536, k=64, bf16, zero initial state) compares two whole
heads, which the oracle recomputes chunk by chunk.
"""
import numpy as np
import pytest
import torch

import oracle as O
from gated_deltanet_chunk_02_b200 import gdn
from gated_deltanet_chunk_02_b200.inputs import Workload, make_inputs, as_f64_numpy

from helpers import TOL_BF16, TOL_F32, rel

pytestmark = pytest.mark.gpu


def oracle_forward(inp, heads, k, N, mask, S, exact, S0=None):
    """Oracle forward for the flattened heads `heads` (indices into B*H)."""
    d = inp["K"].shape[-1]
    T_len = inp["K"].shape[2]
    n = T_len // k

    def sel(x, last):
        a = as_f64_numpy(x).reshape(-1, T_len, *last)
        return a[heads]
    Q, K, V = (sel(inp[key], (d,)) for key in ("Q", "K", "V"))
    beta, g = sel(inp["beta"], ()), sel(inp["g"], ())
    BH = len(heads)
    Kc, Vc, Qc = (x.reshape(BH, n, k, d) for x in (K, V, Q))
    bc, gc = beta.reshape(BH, n, k), g.reshape(BH, n, k)
    A = O.build_A(Kc, bc, gc)
    T = O.invert_fwdsub(A) if exact else O.invert_neumann(A, N, bool(mask), S)
    S0h = None if S0 is None else S0.reshape(-1, d, d)[heads]
    Oo, Sf = O.chunk_forward(Qc, Kc, Vc, bc, gc, T, S0h)
    return Oo.reshape(BH, T_len, d), Sf


def run_forward(d, N, mask, S, exact, S0=None, k=64):
    B, H, T_len, dd = d["K"].shape
    Ot = torch.empty_like(d["Q"])
    Sf = torch.empty(B, H, dd, dd, device="cuda")
    ws = torch.empty(gdn.gdn_forward_workspace_bytes(d["K"], k), dtype=torch.uint8, device="cuda")
    gdn.gdn_forward(d["Q"], d["K"], d["V"], d["beta"], d["g"], S0, N, mask, S, exact, Ot, Sf, ws,
                    k=k)
    assert gdn.gdn_get_status() == gdn.GDN_OK
    return Ot, Sf


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,mask,S,exact", [(3, 1, 0, 0), (3, 1, 8, 0), (2, 0, 1, 0), (3, 1, 0, 1)])
@pytest.mark.parametrize("with_s0", [False, True])
def test_forward_small(dtype, N, mask, S, exact, with_s0):
    w = Workload(B=1, H=2, T=512, k=64, dtype=dtype)
    inp = make_inputs(w, seed=11, with_q=True)
    d = {key: v.cuda() for key, v in inp.items()}
    S0 = None
    if with_s0:
        S0 = torch.randn(1, 2, 128, 128, generator=torch.Generator().manual_seed(3)) * 0.1
    Ot, Sf = run_forward(d, N, mask, S, exact, None if S0 is None else S0.cuda())
    Or, Sr = oracle_forward(inp, np.arange(2), 64, N, mask, S, exact,
                            None if S0 is None else S0.double().numpy())
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    assert rel(Ot.reshape(2, 512, 128), Or) <= tol
    assert rel(Sf.reshape(2, 128, 128), Sr) <= tol


@pytest.fixture(scope="module")
def c5():
    w = Workload(B=1, H=16, T=65536, k=64, dtype="bf16")
    inp = make_inputs(w, seed=0, with_q=True)
    d = {key: v.cuda() for key, v in inp.items()}
    return inp, d


@pytest.mark.parametrize("N,mask,S,exact", [(3, 1, 0, 0), (3, 1, 8, 0), (3, 1, 0, 1)])
def test_c5_long_context(c5, N, mask, S, exact):
    inp, d = c5
    Ot, Sf = run_forward(d, N, mask, S, exact)
    assert torch.isfinite(Ot).all() and torch.isfinite(Sf).all()
    heads = np.array([0, 11])
    Or, Sr = oracle_forward(inp, heads, 64, N, mask, S, exact)
    Og = Ot.reshape(16, 65536, 128)[heads]
    Sg = Sf.reshape(16, 128, 128)[heads]
    assert rel(Og, Or) <= TOL_BF16
    assert rel(Sg, Sr) <= TOL_BF16


def test_c5_slow_gates_end_of_sequence():
    """The c5 length with slow-decay gates (log-gates scaled by 0.05), S = 8:
    two whole heads, the sequence's last 8 chunks on their own, and the final
    state against the oracle; the oracle's S = 0 forward is 0.13 away here,
    so a forward that dropped or cut short the residual would fail."""
    w = Workload(B=1, H=16, T=65536, k=64, dtype="bf16")
    inp = make_inputs(w, seed=5, with_q=True, gate_scale=0.05)
    d = {key: v.cuda() for key, v in inp.items()}
    Ot, Sf = run_forward(d, 3, 1, 8, 0)
    heads = np.array([3, 15])
    Or, Sr = oracle_forward(inp, heads, 64, 3, 1, 8, 0)
    O0, _ = oracle_forward(inp, heads, 64, 3, 1, 0, 0)
    Og = Ot.reshape(16, 65536, 128)[heads]
    last = slice(65536 - 8 * 64, 65536)
    assert rel(Og, Or) <= TOL_BF16
    assert rel(Og[:, last], Or[:, last]) <= TOL_BF16
    assert rel(Sf.reshape(16, 128, 128)[heads], Sr) <= TOL_BF16
    assert rel(Og[:, last], O0[:, last]) >= 5 * TOL_BF16


@pytest.mark.parametrize("N,mask,S", [(3, 1, 8), (3, 1, 0), (2, 0, 1)])
def test_forward_odd_chunk_count(N, mask, S):
    """21 chunks: the output pass's last 128-row tile holds a single chunk."""
    w = Workload(B=1, H=3, T=448, k=64, dtype="bf16")
    inp = make_inputs(w, seed=12, with_q=True)
    d = {key: v.cuda() for key, v in inp.items()}
    Ot, Sf = run_forward(d, N, mask, S, 0)
    Or, Sr = oracle_forward(inp, np.arange(3), 64, N, mask, S, 0)
    assert rel(Ot.reshape(3, 448, 128), Or) <= TOL_BF16
    assert rel(Sf.reshape(3, 128, 128), Sr) <= TOL_BF16


def raw_oracle(inp_raw, Q_raw, BH, T_len, N, mask, S, S0=None):
    """The oracle with its own prologue: query and key rows normalised, gates summed."""
    k, d = 64, 128
    n = T_len // k
    Qn = O.l2_normalize_rows(as_f64_numpy(Q_raw)).reshape(BH, n, k, d)
    Kn = O.l2_normalize_rows(as_f64_numpy(inp_raw["K"])).reshape(BH, n, k, d)
    V = as_f64_numpy(inp_raw["V"]).reshape(BH, n, k, d)
    b = as_f64_numpy(inp_raw["beta"]).reshape(BH, n, k)
    g = O.chunk_cumsum(as_f64_numpy(inp_raw["loggate"]), k).reshape(BH, n, k)
    T = O.invert_neumann(O.build_A(Kn, b, g), N, bool(mask), S)
    Oo, Sf = O.chunk_forward(Qn, Kn, V, b, g, T, S0)
    return Oo.reshape(BH, T_len, d), Sf


@pytest.mark.parametrize("B,H,T_len", [(1, 2, 512), (1, 3, 448)])
@pytest.mark.parametrize("N,mask,S", [(3, 1, 8), (3, 0, 0)])
@pytest.mark.parametrize("with_s0", [False, True])
def test_forward_raw_normalises_queries_and_keys(B, H, T_len, N, mask, S, with_s0):
    """gdn_forward_raw: raw key rows, query rows of any length (each row scaled
    by its own factor) and per-token log-gates, against the oracle's
    normalisation, cumulative sum and forward."""
    w = Workload(B=B, H=H, T=T_len, k=64, dtype="bf16")
    inp = make_inputs(w, seed=13, with_q=True, raw_keys=True)
    scale = 0.25 + 4.0 * torch.rand(B, H, T_len, 1, generator=torch.Generator().manual_seed(9))
    Q_raw = (inp["Q"].float() * scale).to(torch.bfloat16)
    Q_raw[0, 0, 5] = 0                                   # an all-zero query row: O row zero
    d = {key: v.cuda() for key, v in inp.items()}
    S0 = None
    if with_s0:
        S0 = torch.randn(B, H, 128, 128, generator=torch.Generator().manual_seed(4)) * 0.1
    Ot = torch.empty_like(d["K"])
    Sf = torch.empty(B, H, 128, 128, device="cuda")
    ws = torch.empty(gdn.gdn_forward_raw_workspace_bytes(d["K"], 64), dtype=torch.uint8,
                     device="cuda")
    gdn.gdn_forward_raw(Q_raw.cuda(), d["K"], d["V"], d["beta"], d["loggate"],
                        None if S0 is None else S0.cuda(), N, mask, S, Ot, Sf, ws)
    assert gdn.gdn_get_status() == gdn.GDN_OK
    Or, Sr = raw_oracle(inp, Q_raw, B * H, T_len, N, mask, S,
                        None if S0 is None else S0.double().numpy().reshape(-1, 128, 128))
    assert rel(Ot.reshape(B * H, T_len, 128), Or) <= TOL_BF16
    assert rel(Sf.reshape(B * H, 128, 128), Sr) <= TOL_BF16
    assert torch.count_nonzero(Ot[0, 0, 5]) == 0
