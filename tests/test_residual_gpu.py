"""GPU parity on inputs where the residual correction changes the answer.

On the workloads' own gates (fast decay) the truncated series is already close
to the exact inverse: T at S = 0 and at S = 8 differ by about 5e-3, under the
1e-2 contract tolerance, so a kernel that skipped or mis-scheduled the residual
rounds would still pass the contract checks.  The inputs here make the
residual sum G = sum_{s<=S} E^s (gist.science summary, Methodology section 3,
parallel residual correction) visible:

* ``slow``: per-token log-gates scaled by 0.05 (little decay inside a chunk);
* ``nodecay``: log-gates 0;
* ``corr``: gates scaled by 0.05 and key rows sharing one direction (rho = 0.5),
  which makes A and E larger; with N = 1 the oracle's T at S = 8 and S = 7
  differ by about 0.2.

Every case is checked twice: against the contract tolerance, and against a
regression bound tied to the measured floor of that path (about a third of the
bound; the floors are set by fp16 operands, bf16 outputs and, for the
prologue, the in-kernel bf16 rounding of the normalised keys).  Where the
oracle separates order S from order S - 1 (and from S = 0) by more than three
bounds, the GPU result must be within the bound of order S and at least two
bounds away from the others, so a dropped or repeated round fails.
"""
import numpy as np
import pytest
import torch

import oracle as O
from gated_deltanet_chunk_02_b200 import gdn
from gated_deltanet_chunk_02_b200.inputs import Workload, make_inputs, as_f64_numpy

from helpers import TOL_BF16, TOL_F32, A_tensor, chunked, rel, to_dev

pytestmark = pytest.mark.gpu

KINDS = {"slow": dict(gate_scale=0.05), "nodecay": dict(gate_scale=0.0),
         "corr": dict(gate_scale=0.05, key_corr=0.5)}

# regression bounds on T (relative Frobenius, against the oracle at the same
# order), per path and input kind; W and U share one bound (bf16 outputs)
BOUND_T = {
    "tc": {"slow": 2e-4, "nodecay": 5e-4, "corr": 1e-3},
    "raw": {"slow": 1e-3, "nodecay": 2e-3, "corr": 1e-3},
    "f32": {"slow": 2e-7, "nodecay": 2e-7, "corr": 2e-6},
}
BOUND_WU = 6e-3


def check_status():
    assert gdn.gdn_get_status() == gdn.GDN_OK


def separated(T, refs: dict, S: int, bound: float) -> int:
    """Checks T against the oracle's orders S, S - 1 and 0; returns 1 when the
    oracle separates order S from order S - 1 by more than three bounds (the
    case in which a dropped round would be seen), else 0."""
    err = rel(T, refs[S])
    assert err <= bound, f"order {S}: {err:.2e} > bound {bound:.1e}"
    seen = 0
    for other in sorted({S - 1, 0}):
        sep = O.rel_fro(refs[other], refs[S])
        if sep > 3 * bound:
            far = rel(T, refs[other])
            assert far >= 2 * bound, f"order {S} result within {far:.2e} of order {other}"
            seen += other == S - 1
    return seen


def fused_case(kind, k, N, mask, orders, gated, dtype="bf16"):
    w = Workload(B=1, H=3, T=3 * k, k=k, dtype=dtype)        # 9 chunks
    inp = make_inputs(w, seed=300 + k + 7 * N + mask, **KINDS[kind])
    c = chunked(inp, w)
    d = {key: to_dev(v) for key, v in inp.items()}
    A = O.build_A(c["K"], c["beta"], c["g"])
    refs = {S: O.invert_neumann(A, N, bool(mask), S) for S in set(orders) | {o - 1 for o in orders} | {0}}
    path = "f32" if dtype == "f32" else "tc"
    n_sep = 0
    for S in orders:
        W = torch.empty_like(d["K"])
        U = torch.empty_like(d["V"])
        T = torch.empty(w.B, w.H, w.T // k, k, k, device="cuda")
        gdn.gdn_chunk_wy_fused(d["K"], d["V"], d["beta"], d["g"], N, mask, S, int(gated), W, U, T, k=k)
        check_status()
        Wr, Ur = O.wy(refs[S], c["K"], c["V"], c["beta"], c["g"] if gated else None)
        tol = TOL_F32 if dtype == "f32" else TOL_BF16
        assert rel(T, refs[S]) <= tol and rel(W, Wr) <= tol and rel(U, Ur) <= tol
        if dtype != "f32":
            assert rel(W, Wr) <= BOUND_WU and rel(U, Ur) <= BOUND_WU
        n_sep += separated(T, refs, S, BOUND_T[path][kind])
    return n_sep


@pytest.mark.parametrize("kind", ["slow", "nodecay"])
@pytest.mark.parametrize("k", [32, 64, 128])
@pytest.mark.parametrize("N,mask", [(1, 1), (3, 1), (4, 1), (3, 0)])
def test_fused_residual_visible(kind, k, N, mask):
    """The fused step (tensor cores; band path at k = 64 with the mask), orders
    1-4 and 8, ungated and gated."""
    n = fused_case(kind, k, N, mask, [1, 2, 3, 4, 8], gated=False)
    n += fused_case(kind, k, N, mask, [2, 8], gated=True)
    # the inputs separate the orders this test checks (without the mask the
    # N = 3 series is already close to exact: bounds only)
    assert n >= (3 if mask else 0)


@pytest.mark.parametrize("k", [32, 64])
@pytest.mark.parametrize("N", [1, 3, 4])
def test_fused_residual_visible_correlated_keys(k, N):
    """Correlated keys, mask on: with N = 1 and k = 64 every order up to 9 is
    separated from the previous one, S = 8 (the pages' setting) included."""
    n = fused_case("corr", k, N, 1, [1, 2, 3, 4, 5, 7, 8, 9], gated=False)
    assert n >= 3
    if k == 64 and N == 1:
        assert n == 8                # every order, S = 8 included, separated from S - 1


@pytest.mark.parametrize("kind", ["slow", "corr"])
@pytest.mark.parametrize("k", [32, 64])
def test_fused_f32_residual_visible(kind, k):
    """The fp32 fused step (CUDA cores)."""
    assert fused_case(kind, k, 3, 1, [1, 2, 3, 8], gated=False, dtype="f32") >= 3


@pytest.mark.parametrize("kind", ["slow", "nodecay", "corr"])
@pytest.mark.parametrize("k", [32, 64, 128])
def test_prologue_residual_visible(kind, k):
    """The fused step with its prologue (keys normalised and log-gates summed
    in the kernel)."""
    if kind == "corr" and k == 128:
        pytest.skip("correlated keys at k = 128: the residual series diverges (see the design notes)")
    w = Workload(B=1, H=3, T=3 * k, k=k, dtype="bf16")
    inp = make_inputs(w, seed=400 + k, raw_keys=True, **KINDS[kind])
    Kn = O.l2_normalize_rows(as_f64_numpy(inp["K"]))
    g = O.chunk_cumsum(as_f64_numpy(inp["loggate"]), k)
    c = {"K": O.to_chunks(Kn, k), "V": O.to_chunks(as_f64_numpy(inp["V"]), k),
         "beta": O.to_chunks(as_f64_numpy(inp["beta"]), k), "g": O.to_chunks(g, k)}
    A = O.build_A(c["K"], c["beta"], c["g"])
    d = {key: v.cuda() for key, v in inp.items()}
    refs = {S: O.invert_neumann(A, 3, True, S) for S in range(0, 9)}
    n = 0
    for S in (1, 2, 3, 8):
        W = torch.empty_like(d["K"])
        U = torch.empty_like(d["V"])
        T = torch.empty(w.B, w.H, w.T // k, k, k, device="cuda")
        gdn.gdn_chunk_wy_fused_raw(d["K"], d["V"], d["beta"], d["loggate"], 3, 1, S, 1, W, U, T,
                                   None, None, k=k)
        check_status()
        Wr, Ur = O.wy(refs[S], c["K"], c["V"], c["beta"], c["g"])
        assert rel(W, Wr) <= BOUND_WU and rel(U, Ur) <= BOUND_WU
        n += separated(T, refs, S, BOUND_T["raw"][kind])
    assert n >= 2


@pytest.mark.parametrize("kind", ["slow", "nodecay", "corr"])
@pytest.mark.parametrize("k", [32, 64, 128, 256])
@pytest.mark.parametrize("N,mask", [(1, 1), (3, 1), (3, 0)])
def test_neumann_tc_residual_visible(kind, k, N, mask):
    """The standalone tensor-core inverse (stacked doubling at k <= 64 when
    S + 1 is 2^m or 2^m + 1, Horner otherwise, 2 x 2 blocks at k = 256)."""
    if kind == "corr" and (k >= 128 or not mask):
        pytest.skip("correlated keys: the residual series diverges at k >= 128 and without the mask")
    w = Workload(B=1, H=3 if k < 256 else 2, T=3 * k, k=k, dtype="bf16")
    inp = make_inputs(w, seed=500 + k + N + mask, **KINDS[kind])
    c = chunked(inp, w)
    A32 = O.build_A(c["K"], c["beta"], c["g"]).astype(np.float32)
    A64 = A32.astype(np.float64)
    Ad = to_dev(A_tensor(A32, w))
    orders = [1, 2, 3, 4, 7, 8, 9]
    refs = {S: O.invert_neumann(A64, N, bool(mask), S) for S in range(0, 10)}
    n = 0
    for S in orders:
        T = torch.empty(w.B, w.H, w.T // k, k, k, device="cuda")
        gdn.gdn_invert_neumann(Ad, T, N, mask, S, gdn.GDN_PREC_F16)
        check_status()
        assert rel(T, refs[S]) <= TOL_BF16
        n += separated(T, refs, S, BOUND_T["tc"][kind])
        if k <= 128 and S in (1, 3, 8):
            T32 = torch.empty_like(T)
            gdn.gdn_invert_neumann(Ad, T32, N, mask, S, gdn.GDN_PREC_F32)
            check_status()
            separated(T32, refs, S, BOUND_T["f32"][kind])
    assert n >= (3 if mask else 0)


@pytest.mark.parametrize("kind", ["slow", "nodecay", "corr"])
@pytest.mark.parametrize("k", [32, 64, 128])
def test_newton_residual_visible(kind, k):
    """The sequential correction: M steps against M - 1 and 0."""
    if kind == "corr" and k == 128:
        pytest.skip("correlated keys at k = 128: the residual series diverges")
    w = Workload(B=1, H=3, T=3 * k, k=k, dtype="bf16")
    inp = make_inputs(w, seed=600 + k, **KINDS[kind])
    c = chunked(inp, w)
    A32 = O.build_A(c["K"], c["beta"], c["g"]).astype(np.float32)
    A64 = A32.astype(np.float64)
    Ad = to_dev(A_tensor(A32, w))
    refs = {M: O.invert_newton(A64, 3, True, M) for M in range(0, 4)}
    n = 0
    for M in (1, 2, 3):
        T = torch.empty(w.B, w.H, w.T // k, k, k, device="cuda")
        gdn.gdn_invert_newton(Ad, T, 3, 1, M)
        check_status()
        n += separated(T, refs, M, BOUND_T["tc"][kind])
    assert n >= 2
