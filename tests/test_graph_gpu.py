"""The C-ABI calls inside CUDA graphs: a serving loop captures the fused step
(or the whole forward) once and replays it.  Every launch of libgdn goes on
the caller's stream and the library allocates nothing, so a captured graph
replays to the same bits as the eager calls."""
import pytest
import torch

from gated_deltanet_chunk_02_b200 import gdn
from gated_deltanet_chunk_02_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu


def _capture(fn):
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):            # warm-up outside the capture
        fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        fn()
    return graph


def test_fused_step_graph_replay_matches_eager():
    w = Workload(B=2, H=4, T=512, k=64, dtype="bf16")
    d = {key: v.cuda() for key, v in make_inputs(w, seed=31).items()}
    W1, U1 = torch.empty_like(d["K"]), torch.empty_like(d["V"])
    gdn.gdn_chunk_wy_fused(d["K"], d["V"], d["beta"], d["g"], 3, 1, 8, 1, W1, U1, None, k=64)
    torch.cuda.synchronize()
    W2, U2 = torch.empty_like(W1), torch.empty_like(U1)
    graph = _capture(lambda: gdn.gdn_chunk_wy_fused(d["K"], d["V"], d["beta"], d["g"], 3, 1, 8, 1,
                                                    W2, U2, None, k=64))
    W2.zero_()
    U2.zero_()
    graph.replay()
    graph.replay()
    torch.cuda.synchronize()
    assert gdn.gdn_get_status() == gdn.GDN_OK
    assert torch.equal(W1, W2) and torch.equal(U1, U2)


def test_forward_graph_replay_matches_eager():
    w = Workload(B=1, H=2, T=1024, k=64, dtype="bf16")
    d = {key: v.cuda() for key, v in make_inputs(w, seed=32, with_q=True).items()}
    ws = torch.empty(gdn.gdn_forward_workspace_bytes(d["K"], 64), dtype=torch.uint8, device="cuda")
    O1 = torch.empty_like(d["Q"])
    S1 = torch.empty(1, 2, 128, 128, device="cuda")
    gdn.gdn_forward(d["Q"], d["K"], d["V"], d["beta"], d["g"], None, 3, 1, 8, 0, O1, S1, ws, k=64)
    torch.cuda.synchronize()
    O2, S2 = torch.empty_like(O1), torch.empty_like(S1)
    graph = _capture(lambda: gdn.gdn_forward(d["Q"], d["K"], d["V"], d["beta"], d["g"], None, 3, 1,
                                             8, 0, O2, S2, ws, k=64))
    O2.zero_()
    S2.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert gdn.gdn_get_status() == gdn.GDN_OK
    assert torch.equal(O1, O2) and torch.equal(S1, S2)
