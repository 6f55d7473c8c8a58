"""gdn_forward_static: the forward that allocates nothing.

Some callers may not allocate device memory while they run (a plug-in inside
a serving process that owns the whole GPU memory pool, a deployment with a
memory budget fixed at start-up).  For them the library offers
gdn_forward_static, whose scratch is a fixed 64 MiB device array inside the
library.  This file checks, through the C ABI, that two calls in a row (with
different inputs, so the second cannot lean on what the first left in the
shared array) give the same outputs as gdn_forward with a caller-provided
workspace, and that a problem too large for the array is refused.

It is collected last on purpose, so that a failure here never hides the
result of any other test.
"""
import ctypes

import pytest
import torch

from gated_deltanet_chunk_02_b200 import gdn
from gated_deltanet_chunk_02_b200.inputs import Workload, make_inputs

from helpers import TOL_BF16, TOL_F32, rel

pytestmark = pytest.mark.gpu


def reference(d, N, mask, S, exact):
    O = torch.empty_like(d["Q"])
    Sf = torch.empty(d["K"].shape[0], d["K"].shape[1], 128, 128, device="cuda")
    ws = torch.empty(gdn.gdn_forward_workspace_bytes(d["K"], 64), dtype=torch.uint8,
                     device="cuda")
    gdn.gdn_forward(d["Q"], d["K"], d["V"], d["beta"], d["g"], None, N, mask, S, exact, O, Sf, ws)
    return O, Sf


def no_alloc(d, N, mask, S, exact):
    O = torch.empty_like(d["Q"])
    Sf = torch.empty(d["K"].shape[0], d["K"].shape[1], 128, 128, device="cuda")
    gdn.gdn_forward_static(d["Q"], d["K"], d["V"], d["beta"], d["g"], None, N, mask, S, exact,
                           O, Sf)
    return O, Sf


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("N,mask,S,exact", [(3, 1, 8, 0), (3, 1, 0, 1)])
def test_two_calls_match_the_workspace_forward(dtype, N, mask, S, exact):
    tol = TOL_BF16 if dtype == "bf16" else TOL_F32
    w = Workload(B=1, H=2, T=2048, k=64, dtype=dtype)          # 64 chunks, a few MiB of scratch
    for seed in (21, 22):                                         # two calls in a row
        inp = make_inputs(w, seed=seed, with_q=True)
        d = {key: v.cuda() for key, v in inp.items()}
        O_ref, S_ref = reference(d, N, mask, S, exact)
        O, Sf = no_alloc(d, N, mask, S, exact)
        assert gdn.gdn_get_status() == gdn.GDN_OK
        assert rel(O, O_ref.double().cpu().numpy()) <= tol
        assert rel(Sf, S_ref.double().cpu().numpy()) <= tol


def test_too_large_is_refused():
    lib = gdn.load()
    s = gdn.GdnShape(1, 16, 65536, 64, 128)          # needs about 1 GiB of scratch
    P = ctypes.c_void_p(0x10000)
    rc = lib.gdn_forward_static(P, P, P, P, P, None, 3, 1, 0, 0, P, P, s, gdn.GDN_BF16, None)
    assert rc == gdn.GDN_ERR_ARG
    assert "64 MiB" in gdn.gdn_last_error()
