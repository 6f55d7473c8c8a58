"""gdn_forward_static: the forward that allocates nothing.

Some callers may not allocate device memory while they run (a plug-in inside
a serving process that owns the whole GPU memory pool, a deployment with a
memory budget fixed at start-up).  For them the library offers
gdn_forward_static, whose scratch is a fixed 64 MiB device array inside the
library.  This file checks, through the C ABI, that two calls in a row (with
different inputs, so the second cannot lean on what the first left in the
shared array) give the same output bits as gdn_forward with a caller-provided
workspace (the same kernels on the same inputs; only the scratch differs),
that a problem needing exactly the 64 MiB runs, and that one chunk more, or a
much larger problem, is refused.

It is collected last on purpose, so that a failure here never hides the
result of any other test.
"""
import ctypes

import pytest
import torch

from gated_deltanet_chunk_02_b200 import gdn
from gated_deltanet_chunk_02_b200.inputs import Workload, make_inputs

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
    w = Workload(B=1, H=2, T=2048, k=64, dtype=dtype)          # 64 chunks, a few MiB of scratch
    for seed in (21, 22):                                         # two calls in a row
        inp = make_inputs(w, seed=seed, with_q=True)
        d = {key: v.cuda() for key, v in inp.items()}
        O_ref, S_ref = reference(d, N, mask, S, exact)
        O, Sf = no_alloc(d, N, mask, S, exact)
        assert gdn.gdn_get_status() == gdn.GDN_OK
        assert torch.equal(O, O_ref) and torch.equal(Sf, S_ref)


def test_exactly_the_array_runs():
    """1024 bf16 chunks of 64 tokens need exactly the 64 MiB array."""
    w = Workload(B=1, H=16, T=4096, k=64, dtype="bf16")
    assert gdn.gdn_forward_workspace_bytes(torch.empty(1, 16, 4096, 128, dtype=torch.bfloat16), 64) \
        == 64 << 20
    inp = make_inputs(w, seed=23, with_q=True)
    d = {key: v.cuda() for key, v in inp.items()}
    O_ref, S_ref = reference(d, 3, 1, 8, 0)
    O, Sf = no_alloc(d, 3, 1, 8, 0)
    assert gdn.gdn_get_status() == gdn.GDN_OK
    assert torch.equal(O, O_ref) and torch.equal(Sf, S_ref)


@pytest.mark.parametrize("B,H,T", [(1, 1, 1025 * 64), (1, 16, 65536)])
def test_too_large_is_refused(B, H, T):
    """One chunk more than the array holds (1025 bf16 chunks), and about
    1 GiB of scratch: refused on the host, nothing launched."""
    lib = gdn.load()
    s = gdn.GdnShape(B, H, T, 64, 128)
    P = ctypes.c_void_p(0x10000)
    rc = lib.gdn_forward_static(P, P, P, P, P, None, 3, 1, 0, 0, P, P, s, gdn.GDN_BF16, None)
    assert rc == gdn.GDN_ERR_ARG
    assert "64 MiB" in gdn.gdn_last_error()
