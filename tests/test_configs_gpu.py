"""The workload configurations at full size on the GPU, checked against the
oracle on sampled chunks (the oracle computes each chunk independently).

* 4 chunks, float32, N=3 with mask (B=1, H=1, T=256, k=64);
* B=4, H=16, T=4096, k=64, bf16: N in {1,2,3,4} x mask on/off x S in {0, 8};
* chunk-size sweep B=1, H=32, T=16384, k in {32, 64, 128}: Neumann + mask
  (N=3) on tensor cores and exact forward substitution;
* the INT8 scheme at B=4, H=16, T=4096: bit-exact on sampled chunks.
"""
import numpy as np
import pytest
import torch

import oracle as O
from gated_deltanet_chunk_02_b200 import gdn
from gated_deltanet_chunk_02_b200.inputs import Workload, make_inputs, as_f64_numpy

from helpers import TOL_BF16, TOL_F32, rel

pytestmark = pytest.mark.gpu


def sample_idx(nc, n=96, seed=0):
    rng = np.random.default_rng(seed)
    idx = np.unique(np.concatenate([[0, 1, nc - 2, nc - 1], rng.choice(nc, n, replace=False)]))
    return idx


def chunks_of(inp, k, idx):
    return {key: O.to_chunks(as_f64_numpy(inp[key]), k)[idx] for key in ("K", "V", "beta", "g")}


@pytest.fixture(scope="module")
def c2():
    w = Workload(B=4, H=16, T=4096, k=64, dtype="bf16")
    inp = make_inputs(w, seed=0)
    d = {key: v.cuda() for key, v in inp.items()}
    return w, inp, d


@pytest.mark.parametrize("N", [1, 2, 3, 4])
@pytest.mark.parametrize("mask", [0, 1])
@pytest.mark.parametrize("S", [0, 8])
def test_c2_fused_full_size(c2, N, mask, S):
    w, inp, d = c2
    nc = w.n_chunks
    W = torch.empty_like(d["K"])
    U = torch.empty_like(d["V"])
    T = torch.empty(nc, 64, 64, device="cuda")
    gdn.gdn_chunk_wy_fused(d["K"], d["V"], d["beta"], d["g"], N, mask, S, 0, W, U, T, k=64)
    assert gdn.gdn_get_status() == gdn.GDN_OK
    idx = sample_idx(nc, seed=N * 10 + mask + S)
    c = chunks_of(inp, 64, idx)
    A = O.build_A(c["K"], c["beta"], c["g"])
    Tr = O.invert_neumann(A, N, bool(mask), S)
    Wr, Ur = O.wy(Tr, c["K"], c["V"], c["beta"])
    Tg = T.cpu().double().numpy()[idx]
    Wg = W.cpu().double().numpy().reshape(nc, 64, 128)[idx]
    Ug = U.cpu().double().numpy().reshape(nc, 64, 128)[idx]
    assert rel(Tg, Tr) <= TOL_BF16
    assert rel(Wg, Wr) <= TOL_BF16
    assert rel(Ug, Ur) <= TOL_BF16
    assert torch.isfinite(W).all() and torch.isfinite(U).all()


def test_c1_f32_full():
    w = Workload(B=1, H=1, T=256, k=64, dtype="f32")
    inp = make_inputs(w, seed=0)
    d = {key: v.cuda() for key, v in inp.items()}
    A = torch.empty(1, 1, 4, 64, 64, device="cuda")
    T = torch.empty_like(A)
    gdn.gdn_build_A(d["K"], d["beta"], d["g"], A, 64)
    gdn.gdn_invert_neumann(A, T, 3, 1, 0, gdn.GDN_PREC_F32)
    assert gdn.gdn_get_status() == gdn.GDN_OK
    c = chunks_of(inp, 64, np.arange(4))
    Ar = O.build_A(c["K"], c["beta"], c["g"])
    assert rel(A.cpu().double().numpy().reshape(Ar.shape), Ar) <= TOL_F32
    Tr = O.invert_neumann(Ar, 3, True, 0)
    assert rel(T.cpu().double().numpy().reshape(Tr.shape), Tr) <= TOL_F32


@pytest.mark.parametrize("k", [32, 64, 128, 256])
def test_c3_chunk_sweep(k):
    w = Workload(B=1, H=32, T=16384, k=k, dtype="bf16")
    inp = make_inputs(w, seed=0)
    d = {key: v.cuda() for key, v in inp.items()}
    nc = w.n_chunks
    A = torch.empty(1, 32, 16384 // k, k, k, device="cuda")
    Tn = torch.empty_like(A)
    Tf = torch.empty_like(A)
    gdn.gdn_build_A(d["K"], d["beta"], d["g"], A, k)
    gdn.gdn_invert_neumann(A, Tn, 3, 1, 0, gdn.GDN_PREC_F16)
    gdn.gdn_invert_fwdsub(A, Tf)
    assert gdn.gdn_get_status() == gdn.GDN_OK
    idx = sample_idx(nc, seed=k)
    c = chunks_of(inp, k, idx)
    Ar = O.build_A(c["K"], c["beta"], c["g"])
    Ag = A.cpu().double().numpy().reshape(nc, k, k)[idx]
    assert rel(Ag, Ar) <= 1e-3
    # the inverses take the GPU's A as their input: compare against the oracle on that A
    assert rel(Tn.cpu().double().numpy().reshape(nc, k, k)[idx],
               O.invert_neumann(Ag, 3, True, 0)) <= TOL_BF16
    assert rel(Tf.cpu().double().numpy().reshape(nc, k, k)[idx], O.invert_fwdsub(Ag)) <= TOL_F32


@pytest.mark.parametrize("N", [1, 2, 3, 4])
@pytest.mark.parametrize("mask", [0, 1])
def test_c4_int8_full_size(N, mask):
    w = Workload(B=4, H=16, T=4096, k=64, dtype="bf16")
    inp = make_inputs(w, seed=0)
    Kc = O.to_chunks(as_f64_numpy(inp["K"]), 64)
    bc = O.to_chunks(as_f64_numpy(inp["beta"]), 64)
    gc = O.to_chunks(as_f64_numpy(inp["g"]), 64)
    A32 = O.build_A(Kc, bc, gc).astype(np.float32)
    nc = A32.shape[0]
    Ad = torch.from_numpy(A32).cuda()
    T = torch.empty_like(Ad)
    q = torch.empty(nc, N, 64, 64, dtype=torch.int8, device="cuda")
    acc = torch.empty(nc, N, 64, 64, dtype=torch.int32, device="cuda")
    sc = torch.empty(nc, N, device="cuda")
    gdn.gdn_invert_neumann_i8(Ad.view(4, 16, 64, 64, 64), T.view(4, 16, 64, 64, 64), N, mask,
                              q, acc, sc)
    assert gdn.gdn_get_status() == gdn.GDN_OK
    idx = sample_idx(nc, n=256, seed=N + 7 * mask)
    r = O.int8_neumann(A32[idx], N, bool(mask))
    np.testing.assert_array_equal(q.cpu().numpy()[idx], r["q"])
    np.testing.assert_array_equal(acc.cpu().numpy()[idx], r["acc"])
    np.testing.assert_array_equal(sc.cpu().numpy()[idx].view(np.uint32), r["scale"].view(np.uint32))
    np.testing.assert_array_equal(T.cpu().numpy()[idx].view(np.uint32), r["T"].view(np.uint32))
