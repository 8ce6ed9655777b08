"""The library's calls captured in a CUDA graph and replayed.

Everything a call launches is stream-ordered (kernels, clearing memsets), and
the split-tile arrival counters are cleared by the CTA that finishes each
tile, so a graph that replays a launch with the generation baked into its
arguments counts from zero every time.  Workload 2's MLP backward splits
its weight-gradient tiles along K (fewer tiles than SMs), so a replay that
did not start from cleared counters would finish no split tile.
"""
import pytest
import torch

from megatron_tensor_transformer_logical_b200 import binding as L
from megatron_tensor_transformer_logical_b200.inputs import WORKLOADS, make_mlp_inputs
from tests.parity import cuda, need_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()
    yield
    L.tp_device_status()


def test_mlp_step_replayed_from_a_cuda_graph():
    wl = WORKLOADS[2]
    d = {k: cuda(v) for k, v in make_mlp_inputs(wl).items()}
    X, A, B = d["X"], d["A"], d["B"]
    M, h = X.shape
    f = A.shape[1]
    t = wl.t
    e = lambda *sh: torch.empty(*sh, dtype=torch.bfloat16, device="cuda")
    out = {"Z": e(M, h), "Y": e(M, f), "dX": e(M, h), "dA": e(h, f), "dB": e(f, h),
           "dbA": e(f), "dbB": e(h)}
    wsf = L.workspace(L.TP_OP_MLP_FWD, M, h, f, 0, t, L.TP_BF16)
    wsb = L.workspace(L.TP_OP_MLP_BWD, M, h, f, 0, t, L.TP_BF16)

    def step():
        L.tp_mlp_fwd(X, A, d["bA"], B, d["bB"], out["Z"], out["Y"], t, wsf)
        L.tp_mlp_bwd(X, A, d["bA"], B, out["Y"], d["dZ"], out["dX"], out["dA"], out["dbA"],
                     out["dB"], out["dbB"], t, wsb)

    step()  # eager: one-time set-up happens outside the capture
    torch.cuda.synchronize()
    ref = {k: v.clone() for k, v in out.items()}

    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            step()
    torch.cuda.current_stream().wait_stream(s)
    for rep in range(3):
        for v in out.values():
            v.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        for k in ref:
            assert torch.equal(out[k], ref[k]), f"replay {rep}: {k} differs from the eager call"
    del g
