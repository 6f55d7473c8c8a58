"""The bounded device waits run out cleanly.

Every wait of the fused step is bounded; when one runs out the kernel sets
GDN_ERR_TIMEOUT in the status word, walks the rest of its tile's barrier
sequence without starting products, copies or stores, waits (bounded) for the
work it already started, frees its tensor memory and returns, so the context
stays usable.  The test hook ``gdn_debug_arm_wait_expiry`` makes one wait run
out on purpose: the next fused call leaves one tile's K load unissued (an
mbarrier phase that nothing completes) and bounds its waits by a few
milliseconds.  Nothing here faults, traps or hangs the GPU.

Each case checks the status, then that the next call on the same stream
succeeds and gives the same bits as a call made before the expiry.
"""
import pytest
import torch

import oracle as O
from gated_deltanet_chunk_02_b200 import gdn
from gated_deltanet_chunk_02_b200.inputs import Workload, make_inputs

from helpers import TOL_BF16, chunked, rel

pytestmark = pytest.mark.gpu


def fused(d, w, N, mask, S):
    W = torch.empty_like(d["K"])
    U = torch.empty_like(d["V"])
    T = torch.empty(w.B, w.H, w.T // w.k, w.k, w.k, device="cuda")
    gdn.gdn_chunk_wy_fused(d["K"], d["V"], d["beta"], d["g"], N, mask, S, 0, W, U, T, k=w.k)
    return W, U, T


@pytest.mark.parametrize("B,H,T,k,N,mask,S,tile,which,ms", [
    (1, 3, 192, 64, 3, 1, 8, 1, "K", 5.0),      # band path, 5 tiles: the CTA's only tile
    (1, 3, 192, 64, 3, 1, 8, 1, "V", 5.0),      # ... its V: the wait runs out inside the tile
    (1, 3, 192, 64, 3, 0, 8, 2, "V", 5.0),      # the dense chain (no mask)
    (1, 3, 384, 128, 3, 1, 8, 4, "V", 5.0),     # k = 128: one slot per CTA
    (1, 16, 4096, 64, 3, 1, 8, 0, "K", 0.02),   # 512 tiles, a 20 us bound: the other slot of
                                                # CTA 0 is inside a tile when the flag rises
])
def test_expired_wait_reports_and_the_next_call_is_clean(B, H, T, k, N, mask, S, tile, which, ms):
    w = Workload(B=B, H=H, T=T, k=k, dtype="bf16")
    inp = make_inputs(w, seed=77)
    d = {key: v.cuda() for key, v in inp.items()}
    W0, U0, T0 = fused(d, w, N, mask, S)                     # a clean call first
    assert gdn.gdn_get_status() == gdn.GDN_OK

    gdn.gdn_debug_arm_wait_expiry(tile, which, ms)
    fused(d, w, N, mask, S)
    assert gdn.gdn_get_status() == gdn.GDN_ERR_TIMEOUT
    assert "ran out" in gdn.gdn_last_error()

    W1, U1, T1 = fused(d, w, N, mask, S)                     # the same stream, no hook
    assert gdn.gdn_get_status() == gdn.GDN_OK
    assert torch.equal(W1, W0) and torch.equal(U1, U0) and torch.equal(T1, T0)
    if w.n_chunks <= 16:
        c = chunked(inp, w)
        Tr = O.invert_neumann(O.build_A(c["K"], c["beta"], c["g"]), N, bool(mask), S)
        Wr, Ur = O.wy(Tr, c["K"], c["V"], c["beta"])
        assert rel(T1, Tr) <= TOL_BF16 and rel(W1, Wr) <= TOL_BF16 and rel(U1, Ur) <= TOL_BF16
