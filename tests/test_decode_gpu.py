"""GPU parity of the decode steps (gdn_decode) against the oracle's plain
token-by-token definition with grouped query/key heads.

Covers float32 and bf16 data, one and several tokens per call, grouped and
ungrouped heads, both row splits (8 CTAs per value head on small grids, 4 on
grids that fill the GPU: B = 10, Hv = 8 and the batch-64 case), the state carried across calls (bit-identical to one call
over the same tokens), the batch-64 step with 32 value heads that the bench
times (sampled heads), and the degenerate inputs (n = 0, b = 0).
"""
import numpy as np
import pytest
import torch

import oracle as O
from gated_deltanet_chunk_02_b200 import gdn
from gated_deltanet_chunk_02_b200.inputs import make_decode_inputs, as_f64_numpy

from helpers import TOL_BF16, TOL_F32, rel

pytestmark = pytest.mark.gpu


def run(inp):
    d = {k: v.cuda() for k, v in inp.items()}
    S = d["S0"].clone()
    Ob = torch.empty_like(d["V"])
    gdn.gdn_decode(d["Q"], d["K"], d["V"], d["beta"], d["loggate"], S, Ob)
    assert gdn.gdn_get_status() == gdn.GDN_OK
    return Ob, S


def oracle(inp, b=slice(None), h=slice(None)):
    f = {k: as_f64_numpy(v) for k, v in inp.items()}
    Hv, Hk = f["V"].shape[1], f["K"].shape[1]
    if isinstance(h, slice):
        Q, K = f["Q"][b], f["K"][b]
        V, beta, lg, S0 = f["V"][b], f["beta"][b], f["loggate"][b], f["S0"][b]
    else:           # selected value heads, each with its own query/key head
        G = Hv // Hk
        Q, K = f["Q"][b][:, [i // G for i in h]], f["K"][b][:, [i // G for i in h]]
        V, beta, lg, S0 = (f[k][b][:, h] for k in ("V", "beta", "loggate", "S0"))
    return O.decode(Q, K, V, beta, lg, S0)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("B,Hk,Hv", [(2, 2, 4), (1, 3, 3), (3, 1, 4), (10, 4, 8)])
@pytest.mark.parametrize("n", [1, 7, 33])
def test_decode_matches_oracle(dtype, B, Hk, Hv, n):
    inp = make_decode_inputs(B, Hk, Hv, n, dtype=dtype, seed=100 + n + Hv)
    Ob, S = run(inp)
    Or, Sr = oracle(inp)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    assert rel(Ob, Or) <= tol
    assert rel(S, Sr) <= TOL_F32            # the state is float32 in both dtypes


def test_state_carried_across_calls_is_bit_identical():
    inp = make_decode_inputs(2, 2, 4, 6, dtype="bf16", seed=7)
    O_all, S_all = run(inp)
    d = {k: v.cuda() for k, v in inp.items()}
    S = d["S0"].clone()
    outs = []
    for t in range(6):
        one = {k: d[k][:, :, t:t + 1].contiguous() for k in ("Q", "K", "V", "beta", "loggate")}
        Ot = torch.empty_like(one["V"])
        gdn.gdn_decode(one["Q"], one["K"], one["V"], one["beta"], one["loggate"], S, Ot)
        outs.append(Ot)
    assert torch.equal(torch.cat(outs, dim=2), O_all)
    assert torch.equal(S, S_all)


def test_decode_batch64_sampled_heads():
    """The bench's step (batch 64, 16 query/key heads, 32 value heads, one
    token), checked on a sample of (batch, value head) pairs."""
    inp = make_decode_inputs(64, 16, 32, 1, dtype="bf16", seed=3)
    Ob, S = run(inp)
    for b, h in [(0, 0), (0, 1), (17, 30), (63, 31), (40, 15)]:
        Or, Sr = oracle(inp, b=slice(b, b + 1), h=[h])
        assert rel(Ob[b:b + 1, h:h + 1], Or) <= TOL_BF16
        assert rel(S[b:b + 1, h:h + 1], Sr) <= TOL_F32


def test_zero_tokens_and_zero_beta():
    inp = make_decode_inputs(1, 2, 2, 4, dtype="f32", seed=5)
    d = {k: v.cuda() for k, v in inp.items()}
    S = d["S0"].clone()
    n0 = gdn.gdn_launch_count()
    empty = {k: d[k][:, :, :0].contiguous() for k in ("Q", "K", "V", "beta", "loggate")}
    gdn.gdn_decode(empty["Q"], empty["K"], empty["V"], empty["beta"], empty["loggate"], S,
                   torch.empty_like(empty["V"]))
    assert gdn.gdn_launch_count() == n0 and torch.equal(S, d["S0"])
    inp["beta"] = torch.zeros_like(inp["beta"])
    Ob, S = run(inp)
    decay = torch.exp(torch.cumsum(inp["loggate"].double(), dim=-1))[..., -1]
    ref = decay[..., None, None] * inp["S0"].double()
    assert rel(S, ref.numpy()) <= TOL_F32
    Or, _ = oracle(inp)
    assert rel(Ob, Or) <= TOL_F32
