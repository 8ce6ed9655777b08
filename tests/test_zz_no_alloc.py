"""tp_mlp_fwd_noalloc: the MLP forward for callers that cannot allocate.

Some callers cannot give libtp a device workspace (their host owns all device
memory, or they run where an allocation is not allowed).  This entry point
keeps the forward's one intermediate in a fixed array inside libtp; its
results must match tp_mlp_fwd, which takes a caller workspace, on calls made
one after another (the array is shared and keeps the previous call's data).

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import pytest
import torch

from megatron_tensor_transformer_logical_b200 import binding as L
from megatron_tensor_transformer_logical_b200.inputs import Workload, make_mlp_inputs
from oracle import tp_oracle as O
from tests.parity import check, cuda, need_gpu

pytestmark = pytest.mark.gpu


def _run(inp, t, noalloc):
    d = {k: cuda(v) for k, v in inp.items()}
    M, h = d["X"].shape
    f = d["A"].shape[1]
    Z = torch.full((M, h), float("nan"), dtype=d["X"].dtype, device="cuda")
    Y = torch.full((M, f), float("nan"), dtype=d["X"].dtype, device="cuda")
    if noalloc:
        L.tp_mlp_fwd_noalloc(d["X"], d["A"], d["bA"], d["B"], d["bB"], Z, Y, t)
    else:
        tpd = L.TP_F32 if d["X"].dtype == torch.float32 else L.TP_BF16
        ws = L.workspace(L.TP_OP_MLP_FWD, M, h, f, 0, t, tpd)
        L.tp_mlp_fwd(d["X"], d["A"], d["bA"], d["B"], d["bB"], Z, Y, t, ws)
    torch.cuda.synchronize()
    L.tp_device_status()
    return Z, Y


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_matches_workspace_entry_point_on_consecutive_calls(dtype):
    need_gpu()
    shapes = [Workload(95, "noalloc a", b=2, s=300, h=256, f=1024, t=4, dtype=dtype,
                       w_std=0.05, bias_std=0.05),
              Workload(96, "noalloc b", b=1, s=520, h=384, f=1536, t=8, dtype=dtype,
                       w_std=0.05, bias_std=0.05)]
    for wl in shapes:  # two calls in a row, the second with other sizes and data
        inp = make_mlp_inputs(wl)
        Zr, Yr = _run(inp, wl.t, noalloc=False)
        Zn, Yn = _run(inp, wl.t, noalloc=True)
        check(Zn, Zr.double().cpu().numpy(), f"Z {wl.name}", dtype)
        check(Yn, Yr.double().cpu().numpy(), f"Ysave {wl.name}", dtype)
        # and against the CPU oracle ("图解Transformer并行计算" §2.1)
        fw = O.mlp_fwd(inp["X"], inp["A"], inp["bA"], inp["B"], inp["bB"])
        check(Zn, fw["Z"], f"Z {wl.name} vs oracle", dtype)
        check(Yn, fw["Y"], f"Ysave {wl.name} vs oracle", dtype)


def test_noalloc_accepts_exactly_its_limit():
    """H of exactly 64 MiB (M * f = 2^25 bf16 elements) is accepted and gives
    the workspace entry point's result; 8 more columns are rejected."""
    need_gpu()
    wl = Workload(99, "noalloc limit", b=1, s=4096, h=64, f=8192, t=8, dtype="bf16",
                  w_std=0.05, bias_std=0.05)
    inp = make_mlp_inputs(wl)
    Zr, Yr = _run(inp, wl.t, noalloc=False)
    Zn, Yn = _run(inp, wl.t, noalloc=True)
    check(Zn, Zr.double().cpu().numpy(), "Z at the limit", "bf16")
    check(Yn, Yr.double().cpu().numpy(), "Ysave at the limit", "bf16")
    X = torch.zeros(4096, 64, dtype=torch.bfloat16, device="cuda")
    A = torch.zeros(64, 8200, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(8200, 64, dtype=torch.bfloat16, device="cuda")
    Z = torch.zeros(4096, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.TPError) as e:
        L.tp_mlp_fwd_noalloc(X, A, None, B, None, Z, None, 8)
    assert e.value.status == L.TP_ERR_SHAPE and "64 MiB" in str(e.value)


def test_noalloc_rejects_sizes_beyond_its_array():
    need_gpu()
    M, h, f = 8192, 256, 8192 + 8  # H would need 8192 * 8200 * 2 bytes > 64 MiB
    X = torch.zeros(M, h, dtype=torch.bfloat16, device="cuda")
    A = torch.zeros(h, f, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(f, h, dtype=torch.bfloat16, device="cuda")
    Z = torch.zeros(M, h, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.TPError) as e:
        L.tp_mlp_fwd_noalloc(X, A, None, B, None, Z, None, 8)
    assert e.value.status == L.TP_ERR_SHAPE and "64 MiB" in str(e.value)
