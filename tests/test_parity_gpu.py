"""GPU parity: every C-ABI entry point against the CPU oracle, element by element,
on the same seeded inputs.

Tolerances (relative Frobenius error per output tensor): 1e-5 for float32
data (float32 arithmetic), 1e-2 for bf16 data (tensor-core products with fp32
accumulation); the INT8 codes, accumulators, scales and the dequantised T are
compared bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle as O
from gated_deltanet_chunk_02_b200 import gdn
from gated_deltanet_chunk_02_b200.inputs import Workload, make_inputs

from helpers import (TOL_BF16, TOL_F32, A_tensor, chunked, oracle_A32, per_chunk_max_rel, rel, to_dev,
                     tol_for)

pytestmark = pytest.mark.gpu


def dev_inputs(inp):
    return {k: to_dev(v) for k, v in inp.items()}


def check_status():
    assert gdn.gdn_get_status() == gdn.GDN_OK


# --------------------------------------------------------------------------- #
# A
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("k", [32, 64, 128, 256])
def test_build_A(dtype, k):
    w = Workload(B=1, H=3, T=4 * k, k=k, dtype=dtype)        # 12 chunks
    inp = make_inputs(w, seed=1)
    d = dev_inputs(inp)
    A = torch.empty(w.B, w.H, w.T // k, k, k, device="cuda")
    gdn.gdn_build_A(d["K"], d["beta"], d["g"], A, k)
    check_status()
    c = chunked(inp, w)
    ref = O.build_A(c["K"], c["beta"], c["g"])
    assert rel(A, ref) <= tol_for(dtype) * (0.1 if dtype == "bf16" else 1)
    Ah = A.cpu().numpy().reshape(ref.shape)
    assert np.all(np.triu(Ah) == 0)


# --------------------------------------------------------------------------- #
# inverses
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("k", [32, 64, 128, 256])
def test_fwdsub(k):
    w = Workload(B=1, H=2, T=3 * k, k=k, dtype="f32")
    A32 = oracle_A32(make_inputs(w, seed=2), w)
    T = torch.empty(w.B, w.H, w.T // k, k, k, device="cuda")
    gdn.gdn_invert_fwdsub(to_dev(A_tensor(A32, w)), T)
    check_status()
    ref = O.invert_fwdsub(A32.astype(np.float64))
    assert rel(T, ref) <= TOL_F32
    assert per_chunk_max_rel(T, ref) <= TOL_F32


@pytest.mark.parametrize("k", [32, 64, 128])
@pytest.mark.parametrize("N", [1, 2, 3, 4])
@pytest.mark.parametrize("mask", [0, 1])
@pytest.mark.parametrize("S", [0, 1, 8])
def test_neumann_f32(k, N, mask, S):
    w = Workload(B=1, H=2, T=2 * k, k=k, dtype="f32")
    A32 = oracle_A32(make_inputs(w, seed=3), w)
    T = torch.empty(w.B, w.H, w.T // k, k, k, device="cuda")
    gdn.gdn_invert_neumann(to_dev(A_tensor(A32, w)), T, N, mask, S, gdn.GDN_PREC_F32)
    check_status()
    ref = O.invert_neumann(A32.astype(np.float64), N, bool(mask), S)
    assert rel(T, ref) <= TOL_F32


# --------------------------------------------------------------------------- #
# WY
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("k", [32, 64, 128])
@pytest.mark.parametrize("gated", [False, True])
def test_wy(dtype, k, gated):
    w = Workload(B=1, H=2, T=3 * k, k=k, dtype=dtype)
    inp = make_inputs(w, seed=4)
    d = dev_inputs(inp)
    c = chunked(inp, w)
    T32 = O.invert_fwdsub(O.build_A(c["K"], c["beta"], c["g"])).astype(np.float32)
    Td = to_dev(A_tensor(T32, w))
    W = torch.empty_like(d["K"])
    U = torch.empty_like(d["V"])
    gdn.gdn_wy(Td, d["K"], d["V"], d["beta"], d["g"] if gated else None, W, U)
    check_status()
    Wr, Ur = O.wy(T32.astype(np.float64), c["K"], c["V"], c["beta"], c["g"] if gated else None)
    assert rel(W, Wr) <= tol_for(dtype)
    assert rel(U, Ur) <= tol_for(dtype)


# --------------------------------------------------------------------------- #
# fused
# --------------------------------------------------------------------------- #
def fused_reference(c, N, mask, S, gated):
    A = O.build_A(c["K"], c["beta"], c["g"])
    T = O.invert_neumann(A, N, bool(mask), S)
    W, U = O.wy(T, c["K"], c["V"], c["beta"], c["g"] if gated else None)
    return T, W, U


@pytest.mark.parametrize("S", [0, 8])
def test_fused_c1_f32(S):
    """B=1, H=1, T=256, k=64 (4 chunks), float32, N=3 with mask, seed 0."""
    w = Workload(B=1, H=1, T=256, k=64, dtype="f32")
    inp = make_inputs(w, seed=0)
    d = dev_inputs(inp)
    W = torch.empty_like(d["K"])
    U = torch.empty_like(d["V"])
    T = torch.empty(1, 1, 4, 64, 64, device="cuda")
    gdn.gdn_chunk_wy_fused(d["K"], d["V"], d["beta"], d["g"], 3, 1, S, 0, W, U, T, k=64)
    check_status()
    Tr, Wr, Ur = fused_reference(chunked(inp, w), 3, 1, S, False)
    assert rel(T, Tr) <= TOL_F32
    assert rel(W, Wr) <= TOL_F32
    assert rel(U, Ur) <= TOL_F32


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("k", [32, 64, 128])
@pytest.mark.parametrize("N,mask,S,gated", [(3, 1, 8, False), (2, 0, 0, True), (4, 1, 1, False),
                                            (1, 1, 3, True)])
def test_fused_small(dtype, k, N, mask, S, gated):
    w = Workload(B=1, H=3, T=3 * k, k=k, dtype=dtype)       # 9 chunks: ragged vs any pairing
    inp = make_inputs(w, seed=5)
    d = dev_inputs(inp)
    W = torch.empty_like(d["K"])
    U = torch.empty_like(d["V"])
    T = torch.empty(w.B, w.H, w.T // k, k, k, device="cuda")
    gdn.gdn_chunk_wy_fused(d["K"], d["V"], d["beta"], d["g"], N, mask, S, int(gated), W, U, T, k=k)
    check_status()
    Tr, Wr, Ur = fused_reference(chunked(inp, w), N, mask, S, gated)
    tol = tol_for(dtype)
    assert rel(T, Tr) <= tol
    assert rel(W, Wr) <= tol
    assert rel(U, Ur) <= tol
    assert per_chunk_max_rel(W, Wr.reshape(Wr.shape[0], -1)) <= 2 * tol


@pytest.mark.parametrize("k", [32, 64, 128])
@pytest.mark.parametrize("N,mask", [(1, 1), (3, 1), (4, 1), (3, 0)])
@pytest.mark.parametrize("S", [0, 1, 2, 3, 4, 5, 7, 8, 9, 16])
def test_fused_residual_schedules(k, N, mask, S):
    """The residual sum G = sum E^s by doubling (S + 1 = 2^m or 2^m + 1) and by
    Horner (the other S), on 9 chunks."""
    gated = (S % 2 == 1)
    w = Workload(B=1, H=3, T=3 * k, k=k, dtype="bf16")
    inp = make_inputs(w, seed=11 + S)
    d = dev_inputs(inp)
    W = torch.empty_like(d["K"])
    U = torch.empty_like(d["V"])
    T = torch.empty(w.B, w.H, w.T // k, k, k, device="cuda")
    gdn.gdn_chunk_wy_fused(d["K"], d["V"], d["beta"], d["g"], N, mask, S, int(gated), W, U, T, k=k)
    check_status()
    Tr, Wr, Ur = fused_reference(chunked(inp, w), N, mask, S, gated)
    assert rel(T, Tr) <= TOL_BF16
    assert per_chunk_max_rel(T, Tr) <= TOL_BF16
    assert rel(W, Wr) <= TOL_BF16
    assert rel(U, Ur) <= TOL_BF16
    Th = T.cpu().numpy().reshape(Tr.shape)
    assert np.all(np.triu(Th, 1) == 0)
    if S == 0 and mask:
        dist = np.arange(k)[:, None] - np.arange(k)[None, :]
        assert np.all(Th[:, dist > N] == 0)


def test_fused_without_T_output_matches():
    w = Workload(B=2, H=2, T=256, k=64, dtype="bf16")
    inp = make_inputs(w, seed=6)
    d = dev_inputs(inp)
    W1, U1, W2, U2 = (torch.empty_like(d["K"]) for _ in range(4))
    T = torch.empty(2, 2, 4, 64, 64, device="cuda")
    gdn.gdn_chunk_wy_fused(d["K"], d["V"], d["beta"], d["g"], 3, 1, 8, 0, W1, U1, T, k=64)
    gdn.gdn_chunk_wy_fused(d["K"], d["V"], d["beta"], d["g"], 3, 1, 8, 0, W2, U2, None, k=64)
    check_status()
    assert torch.equal(W1, W2) and torch.equal(U1, U2)


# --------------------------------------------------------------------------- #
# INT8
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("N,mask", [(3, 1), (1, 1), (3, 0), (4, 1)])
@pytest.mark.parametrize("S", [1, 2, 3, 8])
def test_int8_residual_bit_exact(N, mask, S):
    """INT8 series plus the residual in int8 products: T bit for bit against
    the oracle on 67 chunks (a ragged last tile), and far closer to the exact
    inverse than the series alone."""
    w = Workload(B=1, H=1, T=67 * 64, k=64, dtype="bf16")
    A32 = oracle_A32(make_inputs(w, seed=18 + S), w)
    nc = A32.shape[0]
    Ad = to_dev(A_tensor(A32, w))
    T = torch.empty_like(Ad)
    gdn.gdn_invert_neumann_i8_residual(Ad, T, N, mask, S)
    check_status()
    ref = O.int8_residual(A32, N, bool(mask), S)
    np.testing.assert_array_equal(T.cpu().numpy().reshape(nc, 64, 64).view(np.uint32),
                                  ref.view(np.uint32))
    if N == 3 and mask:
        exact = O.invert_fwdsub(A32.astype(np.float64))
        assert O.rel_fro(ref, exact) < O.rel_fro(O.int8_neumann(A32, N, True)["T"], exact) / 10


@pytest.mark.parametrize("N", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("mask", [0, 1])
def test_int16_bit_exact(N, mask):
    """INT16 codes (byte-split products), int64 accumulators, binary64 scales
    and T, bit for bit against the oracle; 67 chunks (a ragged last tile)."""
    w = Workload(B=1, H=1, T=67 * 64, k=64, dtype="bf16")
    A32 = oracle_A32(make_inputs(w, seed=17), w)
    nc = A32.shape[0]
    Ad = to_dev(A_tensor(A32, w))
    T = torch.empty_like(Ad)
    q = torch.empty(nc, N, 64, 64, dtype=torch.int16, device="cuda")
    acc = torch.empty(nc, N, 64, 64, dtype=torch.int64, device="cuda")
    sc = torch.empty(nc, N, dtype=torch.float64, device="cuda")
    gdn.gdn_invert_neumann_i16(Ad, T, N, mask, q, acc, sc)
    check_status()
    r = O.int16_neumann(A32, N, bool(mask))
    np.testing.assert_array_equal(q.cpu().numpy(), r["q"])
    np.testing.assert_array_equal(acc.cpu().numpy(), r["acc"])
    np.testing.assert_array_equal(sc.cpu().numpy().view(np.uint64), r["scale"].view(np.uint64))
    np.testing.assert_array_equal(T.cpu().numpy().reshape(nc, 64, 64).view(np.uint32),
                                  r["T"].view(np.uint32))
    T2 = torch.empty_like(Ad)
    gdn.gdn_invert_neumann_i16(Ad, T2, N, mask)
    check_status()
    assert torch.equal(T, T2)


@pytest.mark.parametrize("N,mask", [(3, 1), (1, 1), (4, 1), (3, 0)])
@pytest.mark.parametrize("S", [1, 2, 8])
def test_int16_residual_bit_exact(N, mask, S):
    """INT16 series plus the residual in int16 products (byte-split, int64,
    binary64 scales): T bit for bit against the oracle on 67 chunks (a ragged
    last tile), and far closer to the exact inverse than the series alone."""
    w = Workload(B=1, H=1, T=67 * 64, k=64, dtype="bf16")
    A32 = oracle_A32(make_inputs(w, seed=31 + S), w)
    nc = A32.shape[0]
    Ad = to_dev(A_tensor(A32, w))
    T = torch.empty_like(Ad)
    gdn.gdn_invert_neumann_i16_residual(Ad, T, N, mask, S)
    check_status()
    ref = O.int16_residual(A32, N, bool(mask), S)
    np.testing.assert_array_equal(T.cpu().numpy().reshape(nc, 64, 64).view(np.uint32),
                                  ref.view(np.uint32))
    if N == 3 and mask:
        exact = O.invert_fwdsub(A32.astype(np.float64))
        assert O.rel_fro(ref, exact) < O.rel_fro(O.int16_neumann(A32, N, True)["T"], exact) / 10


@pytest.mark.parametrize("kind", ["slow", "corr"])
def test_int16_residual_bit_exact_where_the_residual_shows(kind):
    """Slow-decay gates (and correlated keys): E and its powers are large, so
    every residual product and requantisation moves T."""
    kw = {"slow": dict(gate_scale=0.05), "corr": dict(gate_scale=0.05, key_corr=0.5)}[kind]
    w = Workload(B=1, H=1, T=19 * 64, k=64, dtype="bf16")
    A32 = oracle_A32(make_inputs(w, seed=37, **kw), w)
    nc = A32.shape[0]
    Ad = to_dev(A_tensor(A32, w))
    for N, S in [(1, 8), (3, 8), (3, 3)]:
        T = torch.empty_like(Ad)
        gdn.gdn_invert_neumann_i16_residual(Ad, T, N, 1, S)
        check_status()
        ref = O.int16_residual(A32, N, True, S)
        np.testing.assert_array_equal(T.cpu().numpy().reshape(nc, 64, 64).view(np.uint32),
                                      ref.view(np.uint32))
        assert not np.array_equal(ref, O.int16_residual(A32, N, True, S - 1) if S > 1 else
                                  O.int16_neumann(A32, N, True)["T"])


def test_int16_residual_degenerate_chunks():
    """A zero chunk (every maximum zero: T = I), a single sub-diagonal entry
    (E = 0 exactly, so E, Gm and their codes are zero), codes at +-32767 and
    a full tile of ordinary chunks beside them."""
    rng = np.random.default_rng(41)
    A32 = np.zeros((5, 64, 64), np.float32)
    A32[1, 5, 4] = 0.75                                      # E = 0
    A32[2] = np.tril(rng.choice([-1.0, 1.0], (64, 64)), -1)  # extreme codes
    A32[3] = np.tril(rng.standard_normal((64, 64)) * 0.05, -1)
    A32[4] = np.tril(rng.standard_normal((64, 64)) * 0.2, -1)
    Ad = torch.from_numpy(A32).reshape(1, 1, 5, 64, 64).cuda()
    for N, mask, S in [(3, 1, 8), (1, 1, 2), (2, 0, 3)]:
        T = torch.empty_like(Ad)
        gdn.gdn_invert_neumann_i16_residual(Ad, T, N, mask, S)
        check_status()
        ref = O.int16_residual(A32, N, bool(mask), S)
        np.testing.assert_array_equal(T.cpu().numpy().reshape(5, 64, 64).view(np.uint32),
                                      ref.view(np.uint32))
        assert np.array_equal(ref[0], np.eye(64, dtype=np.float32))


def test_int16_extreme_codes():
    """Entries at +-amax and sign flips: the byte split must carry codes of
    +-32767 and the int64 accumulators reach ~2^36."""
    rng = np.random.default_rng(19)
    nc = 6
    A32 = np.tril(rng.choice([-1.0, 1.0], (nc, 64, 64)), -1).astype(np.float32)
    A32[:, 1:, 0] = 1.0                                      # a full column at the maximum
    Ad = torch.from_numpy(A32).reshape(1, 1, nc, 64, 64).cuda()
    for N, mask in [(2, 0), (3, 0), (3, 1)]:
        T = torch.empty_like(Ad)
        acc = torch.empty(nc, N, 64, 64, dtype=torch.int64, device="cuda")
        gdn.gdn_invert_neumann_i16(Ad, T, N, mask, None, acc, None)
        check_status()
        r = O.int16_neumann(A32, N, bool(mask))
        np.testing.assert_array_equal(acc.cpu().numpy(), r["acc"])
        np.testing.assert_array_equal(T.cpu().numpy().reshape(nc, 64, 64).view(np.uint32),
                                      r["T"].view(np.uint32))
        if not mask:
            assert np.abs(r["acc"]).max() > 2 ** 31        # beyond int32


@pytest.mark.parametrize("N", [1, 2, 3, 4])
@pytest.mark.parametrize("mask", [0, 1])
def test_int8_bit_exact(N, mask):
    w = Workload(B=1, H=4, T=1024, k=64, dtype="bf16")        # 64 chunks
    A32 = oracle_A32(make_inputs(w, seed=7), w)
    nc = A32.shape[0]
    Ad = to_dev(A_tensor(A32, w))
    T = torch.empty_like(Ad)
    q = torch.empty(nc, N, 64, 64, dtype=torch.int8, device="cuda")
    acc = torch.empty(nc, N, 64, 64, dtype=torch.int32, device="cuda")
    sc = torch.empty(nc, N, dtype=torch.float32, device="cuda")
    gdn.gdn_invert_neumann_i8(Ad, T, N, mask, q, acc, sc)
    check_status()
    r = O.int8_neumann(A32, N, bool(mask))
    np.testing.assert_array_equal(q.cpu().numpy(), r["q"])
    np.testing.assert_array_equal(acc.cpu().numpy(), r["acc"])
    np.testing.assert_array_equal(sc.cpu().numpy().view(np.uint32), r["scale"].view(np.uint32))
    np.testing.assert_array_equal(T.cpu().numpy().reshape(nc, 64, 64).view(np.uint32),
                                  r["T"].view(np.uint32))
    # without the debug outputs the same T comes out
    T2 = torch.empty_like(Ad)
    gdn.gdn_invert_neumann_i8(Ad, T2, N, mask)
    check_status()
    assert torch.equal(T, T2)


@pytest.mark.parametrize("k", [32, 64, 128])
@pytest.mark.parametrize("N", [1, 2, 3, 4])
@pytest.mark.parametrize("mask", [0, 1])
@pytest.mark.parametrize("S", [0, 1, 2, 3, 5, 8])
def test_neumann_tensor_cores(k, N, mask, S):
    """The tcgen05 chain (fp16 operands, fp32 accumulation) on 9 chunks."""
    w = Workload(B=1, H=3, T=3 * k, k=k, dtype="bf16")
    A32 = oracle_A32(make_inputs(w, seed=8), w)
    T = torch.empty(w.B, w.H, w.T // k, k, k, device="cuda")
    gdn.gdn_invert_neumann(to_dev(A_tensor(A32, w)), T, N, mask, S, gdn.GDN_PREC_F16)
    check_status()
    ref = O.invert_neumann(A32.astype(np.float64), N, bool(mask), S)
    assert rel(T, ref) <= TOL_BF16
    assert per_chunk_max_rel(T, ref) <= TOL_BF16
    Th = T.cpu().numpy().reshape(ref.shape)
    assert np.all(np.triu(Th, 1) == 0)                       # strictly lower + unit diagonal
    if mask:
        dist = np.arange(k)[:, None] - np.arange(k)[None, :]
        if S == 0:
            assert np.all(Th[:, dist > N] == 0)


@pytest.mark.parametrize("k", [32, 64, 128])
@pytest.mark.parametrize("N,mask", [(1, 1), (3, 1), (3, 0)])
@pytest.mark.parametrize("M", [0, 1, 2, 3, 4])
def test_newton_tensor_cores(k, N, mask, M):
    """The sequential correction T <- T + T (I - (I - A) T) on the tensor cores,
    9 chunks (a ragged last tile), against the oracle's literal iteration."""
    w = Workload(B=1, H=3, T=3 * k, k=k, dtype="bf16")
    A32 = oracle_A32(make_inputs(w, seed=12), w)
    T = torch.full((w.B, w.H, w.T // k, k, k), float("nan"), device="cuda")
    gdn.gdn_invert_newton(to_dev(A_tensor(A32, w)), T, N, mask, M)
    check_status()
    ref = O.invert_newton(A32.astype(np.float64), N, bool(mask), M)
    assert torch.isfinite(T).all()
    assert rel(T, ref) <= TOL_BF16
    assert per_chunk_max_rel(T, ref) <= TOL_BF16
    assert np.all(np.triu(T.cpu().numpy().reshape(ref.shape), 1) == 0)


@pytest.mark.parametrize("k", [32, 64])
@pytest.mark.parametrize("gate_scale", [1.0, 0.05])
def test_blocked_inverse_tensor_cores(k, gate_scale):
    """The exact block-decomposition inverse (fp16 operands) against the oracle
    on 9 chunks (a ragged last tile); slow gates keep far entries large."""
    w = Workload(B=1, H=3, T=3 * k, k=k, dtype="bf16")
    A32 = oracle_A32(make_inputs(w, seed=14, gate_scale=gate_scale), w)
    T = torch.full((w.B, w.H, w.T // k, k, k), float("nan"), device="cuda")
    gdn.gdn_invert_blocked(to_dev(A_tensor(A32, w)), T)
    check_status()
    A64 = A32.astype(np.float64)
    ref = O.invert_blocked(A64)
    assert np.allclose(ref, O.invert_fwdsub(A64), rtol=0, atol=1e-12)
    assert torch.isfinite(T).all()
    assert rel(T, ref) <= TOL_BF16
    assert per_chunk_max_rel(T, ref) <= TOL_BF16
    Th = T.cpu().numpy().reshape(ref.shape)
    assert np.all(np.triu(Th, 1) == 0) and np.all(np.diagonal(Th, axis1=1, axis2=2) == 1)


def test_newton_matches_parallel_residual_on_gpu():
    """M = 3 sequential steps and the parallel residual with S = 7 compute the
    same T (exactly so in exact arithmetic)."""
    k = 64
    w = Workload(B=1, H=4, T=8 * k, k=k, dtype="bf16")
    A = to_dev(A_tensor(oracle_A32(make_inputs(w, seed=13), w), w))
    T1 = torch.empty(w.B, w.H, w.T // k, k, k, device="cuda")
    T2 = torch.empty_like(T1)
    gdn.gdn_invert_newton(A, T1, 3, 1, 3)
    gdn.gdn_invert_neumann(A, T2, 3, 1, 7, gdn.GDN_PREC_F16)
    check_status()
    assert rel(T1, T2.cpu().double().numpy()) <= 1e-3


@pytest.mark.parametrize("N,mask,S", [(1, 1, 0), (2, 1, 0), (3, 1, 0), (4, 1, 0), (3, 0, 0),
                                      (8, 0, 0), (40, 1, 0), (255, 1, 0), (1, 1, 1), (3, 1, 1),
                                      (3, 1, 2), (3, 1, 8), (2, 0, 3), (40, 1, 8)])
def test_neumann_tensor_cores_k256(N, mask, S):
    """The k=256 tcgen05 chain (2 x 2 blocks of 128, Horner sums) on 6 chunks;
    N=40 puts the band across the block boundary of D10, N=255 keeps every
    power, S > 0 runs the residual through the reused operand blocks."""
    k = 256
    w = Workload(B=1, H=2, T=3 * k, k=k, dtype="bf16")
    A32 = oracle_A32(make_inputs(w, seed=9), w)
    T = torch.full((w.B, w.H, w.T // k, k, k), float("nan"), device="cuda")
    gdn.gdn_invert_neumann(to_dev(A_tensor(A32, w)), T, N, mask, S, gdn.GDN_PREC_F16)
    check_status()
    ref = O.invert_neumann(A32.astype(np.float64), N, bool(mask), S)
    assert torch.isfinite(T).all()                           # every entry written
    assert rel(T, ref) <= TOL_BF16
    assert per_chunk_max_rel(T, ref) <= TOL_BF16
    Th = T.cpu().numpy().reshape(ref.shape)
    assert np.all(np.triu(Th, 1) == 0)
    if S == 0:
        assert np.all(np.diagonal(Th, axis1=1, axis2=2) == 1)
        if mask:
            dist = np.arange(k)[:, None] - np.arange(k)[None, :]
            assert np.all(Th[:, dist > N] == 0)
        if N == 1:                                           # T = I + M.A, no products
            assert np.array_equal(Th, ref.astype(np.float32))


# --------------------------------------------------------------------------- #
# degenerate inputs
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("k", [32, 64, 128])
def test_neumann_full_order_is_exact_inverse(k):
    """N = k - 1 keeps every power (A^k = 0): the truncated series is the exact
    inverse, on the tensor-core and the fp32 chains alike."""
    w = Workload(B=1, H=2, T=2 * k, k=k, dtype="bf16")
    A32 = oracle_A32(make_inputs(w, seed=21), w)
    exact = O.invert_fwdsub(A32.astype(np.float64))
    Ad = to_dev(A_tensor(A32, w))
    for prec, tol in ((gdn.GDN_PREC_F16, TOL_BF16), (gdn.GDN_PREC_F32, TOL_F32)):
        T = torch.empty(w.B, w.H, w.T // k, k, k, device="cuda")
        gdn.gdn_invert_neumann(Ad, T, k - 1, 0, 0, prec)
        check_status()
        assert rel(T, exact) <= tol


@pytest.mark.parametrize("k", [32, 64, 128])
def test_fused_beta_zero_gives_identity(k):
    """beta = 0: A = 0, T = I and W = U = 0 exactly."""
    w = Workload(B=1, H=2, T=2 * k, k=k, dtype="bf16")
    d = dev_inputs(make_inputs(w, seed=22))
    d["beta"].zero_()
    W = torch.full_like(d["K"], 7.0)
    U = torch.full_like(d["V"], 7.0)
    T = torch.empty(w.B, w.H, w.T // k, k, k, device="cuda")
    gdn.gdn_chunk_wy_fused(d["K"], d["V"], d["beta"], d["g"], 3, 1, 8, 1, W, U, T, k=k)
    check_status()
    eye = torch.eye(k, device="cuda").expand_as(T)
    assert torch.equal(T, eye)
    assert torch.count_nonzero(W) == 0 and torch.count_nonzero(U) == 0


@pytest.mark.parametrize("gate", ["none", "strong"])
def test_fused_gate_extremes(gate):
    """No decay (g = 0) and a decay strong enough that most e^{g_i - g_j}
    underflow: both match the oracle."""
    k = 64
    w = Workload(B=1, H=3, T=3 * k, k=k, dtype="bf16")
    inp = make_inputs(w, seed=23, gate_scale=0.0 if gate == "none" else 40.0)
    d = dev_inputs(inp)
    W = torch.empty_like(d["K"])
    U = torch.empty_like(d["V"])
    T = torch.empty(w.B, w.H, w.T // k, k, k, device="cuda")
    gdn.gdn_chunk_wy_fused(d["K"], d["V"], d["beta"], d["g"], 3, 1, 8, 1, W, U, T, k=k)
    check_status()
    Tr, Wr, Ur = fused_reference(chunked(inp, w), 3, 1, 8, True)
    assert torch.isfinite(T).all() and torch.isfinite(W.float()).all()
    assert rel(T, Tr) <= TOL_BF16
    assert rel(W, Wr) <= TOL_BF16
    assert rel(U, Ur) <= TOL_BF16
