"""GPU parity of the partitioned MLP forward and backward against the oracle.

Forward ("图解Transformer并行计算" §2.1): Y_i = X @ A_i + bA_i, H_i = GeLU(Y_i)
per column shard, Z = sum_i H_i @ B_i + bB.  Backward (same page, §2.2):
weight gradients per shard, dX = sum of the shards' partials.
"""
import numpy as np
import pytest
import torch

from megatron_tensor_transformer_logical_b200 import binding as L
from megatron_tensor_transformer_logical_b200.inputs import WORKLOADS, Workload, make_mlp_inputs
from oracle import tp_oracle as O
from tests.parity import check, cuda, need_gpu, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()
    yield
    L.tp_device_status()


def gpu_mlp(inp, t, save_y=True, dtype=torch.bfloat16):
    d = {k: cuda(v) for k, v in inp.items()}
    X, A, B = d["X"], d["A"], d["B"]
    M, h = X.shape
    f = A.shape[1]
    tpd = L.TP_F32 if dtype == torch.float32 else L.TP_BF16
    Z = torch.empty(M, h, dtype=dtype, device="cuda")
    Y = torch.empty(M, f, dtype=dtype, device="cuda") if save_y else None
    ws = L.workspace(L.TP_OP_MLP_FWD, M, h, f, 0, t, tpd)
    L.tp_mlp_fwd(X, A, d["bA"], B, d["bB"], Z, Y, t, ws)
    out = {"Z": Z, "Y": Y}
    g = {k: torch.empty_like(v) for k, v in (("dX", X), ("dA", A), ("dB", B))}
    g["dbA"] = torch.empty(f, dtype=dtype, device="cuda")
    g["dbB"] = torch.empty(h, dtype=dtype, device="cuda")
    wsb = L.workspace(L.TP_OP_MLP_BWD, M, h, f, 0, t, tpd)
    L.tp_mlp_bwd(X, A, d["bA"], B, Y, d["dZ"], g["dX"], g["dA"], g["dbA"], g["dB"], g["dbB"], t,
                 wsb)
    torch.cuda.synchronize()
    out.update(g)
    return out


def compare_full(out, inp, dtype):
    fw = O.mlp_fwd(inp["X"], inp["A"], inp["bA"], inp["B"], inp["bB"])
    bw = O.mlp_bwd(inp["X"], inp["A"], inp["bA"], inp["B"], inp["dZ"])
    check(out["Z"], fw["Z"], "Z", dtype)
    if out["Y"] is not None:
        check(out["Y"], fw["Y"], "Ysave", dtype)
    for k in ("dX", "dA", "dB", "dbA", "dbB"):
        check(out[k], bw[k], k, dtype)


def test_mlp_config1_fp32():
    wl = WORKLOADS[1]
    inp = make_mlp_inputs(wl)
    out = gpu_mlp(inp, wl.t, dtype=torch.float32)
    compare_full(out, inp, "f32")


@pytest.mark.parametrize("tile", ["auto", "192", "256", "pair"])
@pytest.mark.parametrize("save_y", [True, False], ids=["Ysave", "recompute"])
def test_mlp_ragged_bf16(monkeypatch, save_y, tile):
    if tile != "auto":
        monkeypatch.setenv("TP_GEMM_TILE", tile)
    # 200 rows (two row tiles, ragged), h=136, f=544: ragged column and K tails.
    wl = Workload(90, "ragged", b=1, s=200, h=136, f=544, t=4, w_std=0.05, bias_std=0.05)
    inp = make_mlp_inputs(wl)
    out = gpu_mlp(inp, wl.t, save_y=save_y)
    compare_full(out, inp, "bf16")


@pytest.mark.parametrize("t", [1, 2, 8])
def test_mlp_fp32_shard_counts(t):
    wl = Workload(91, "fp32 sweep", b=3, s=40, h=64, f=256, t=t, dtype="f32", bias_std=0.02)
    inp = make_mlp_inputs(wl)
    compare_full(gpu_mlp(inp, t, dtype=torch.float32), inp, "f32")


def test_mlp_bias_grads_many_row_chunks():
    """M = 8200 rows: the bias-gradient pass takes 160-row chunks (52 of them,
    the last ragged), with a ragged last column block of dZ (h = 264) and of
    the dY partials (f = 544)."""
    wl = Workload(93, "bias chunks", b=1, s=8200, h=264, f=544, t=2, w_std=0.05,
                  bias_std=0.05)
    inp = make_mlp_inputs(wl)
    out = gpu_mlp(inp, wl.t)
    compare_full(out, inp, "bf16")


@pytest.mark.parametrize("which", ["dbA", "dbB"])
@pytest.mark.parametrize("rows", [1, 3])
def test_mlp_bias_grads_one_of_two_few_rows(rows, which):
    """One bias gradient requested (the other pointer NULL) on 1 and 3 rows:
    one row chunk, one partial row of dY; the other gradient is not written."""
    wl = Workload(94, "few rows", b=1, s=rows, h=72, f=144, t=2, w_std=0.05, bias_std=0.05)
    inp = make_mlp_inputs(wl)
    d = {k: cuda(v) for k, v in inp.items()}
    X, A, B = d["X"], d["A"], d["B"]
    M, h = X.shape
    f = A.shape[1]
    Z = torch.empty(M, h, dtype=torch.bfloat16, device="cuda")
    Y = torch.empty(M, f, dtype=torch.bfloat16, device="cuda")
    L.tp_mlp_fwd(X, A, d["bA"], B, d["bB"], Z, Y, wl.t,
                 L.workspace(L.TP_OP_MLP_FWD, M, h, f, 0, wl.t, L.TP_BF16))
    g = {k: torch.empty_like(v) for k, v in (("dX", X), ("dA", A), ("dB", B))}
    sentinel = 7.0
    dbA = torch.full((f,), sentinel, dtype=torch.bfloat16, device="cuda")
    dbB = torch.full((h,), sentinel, dtype=torch.bfloat16, device="cuda")
    L.tp_mlp_bwd(X, A, d["bA"], B, Y, d["dZ"], g["dX"], g["dA"],
                 dbA if which == "dbA" else None, g["dB"], dbB if which == "dbB" else None, wl.t,
                 L.workspace(L.TP_OP_MLP_BWD, M, h, f, 0, wl.t, L.TP_BF16))
    torch.cuda.synchronize()
    bw = O.mlp_bwd(inp["X"], inp["A"], inp["bA"], inp["B"], inp["dZ"])
    got, other = (dbA, dbB) if which == "dbA" else (dbB, dbA)
    check(got, bw[which], which, "bf16")
    assert torch.all(other.float() == sentinel), "the gradient not asked for was written"
    for k in ("dX", "dA", "dB"):
        check(g[k], bw[k], k, "bf16")


def test_mlp_config2_bf16():
    wl = WORKLOADS[2]
    inp = make_mlp_inputs(wl)
    out = gpu_mlp(inp, wl.t)
    compare_full(out, inp, "bf16")


def test_mlp_cross_t_agreement_bf16():
    """t = 1/2/4/8 agree: column tiles never straddle shards, the K order is fixed."""
    wl = Workload(92, "cross-t", b=2, s=256, h=256, f=1024, t=1, w_std=0.05, bias_std=0.05)
    inp = make_mlp_inputs(wl)
    outs = [gpu_mlp(inp, t) for t in (1, 2, 4, 8)]
    for o in outs[1:]:
        for k in ("Z", "dX", "dA", "dB"):
            assert torch.equal(o[k], outs[0][k]), k


def test_mlp_config5_sampled():
    """The 175B-shaped MLP (h=12288, f=49152, t=8) at full size, sampled.

    Rows of Z and dX depend only on the same rows of X and dZ; column j of
    dA, entry j of dbA and row j of dB depend only on hidden unit j.  So the
    oracle on sampled rows / hidden units is an exact reference.
    """
    wl = WORKLOADS[5]
    inp = make_mlp_inputs(wl)
    out = gpu_mlp(inp, wl.t)
    rng = np.random.default_rng(5)
    # one row from every 128-row tile, and one hidden unit from every 256-wide
    # column tile of each shard's first and last tiles, plus the edges
    rows = np.unique(np.r_[0, wl.M - 1, [rng.integers(i, i + 128) for i in range(0, wl.M, 128)]])
    shard = wl.f // wl.t
    units = np.unique(np.r_[0, wl.f - 1, [rng.integers(i, i + 256) for i in range(0, wl.f, shard)],
                            [rng.integers(i - 256, i) for i in range(shard, wl.f + 1, shard)],
                            rng.integers(0, wl.f, 8)])
    X64, dZ64 = to64(inp["X"]), to64(inp["dZ"])
    A64, B64 = to64(inp["A"]), to64(inp["B"])
    fw = O.mlp_fwd(X64[rows], A64, None, B64, None)
    check(out["Z"][torch.as_tensor(rows, device="cuda")], fw["Z"], "Z rows", "bf16")
    check(out["Y"][torch.as_tensor(rows, device="cuda")], fw["Y"], "Y rows", "bf16")
    bw_rows = O.mlp_bwd(X64[rows], A64, None, B64, dZ64[rows])
    check(out["dX"][torch.as_tensor(rows, device="cuda")], bw_rows["dX"], "dX rows", "bf16")
    bw_units = O.mlp_bwd(X64, A64[:, units], None, B64[units], dZ64)
    u = torch.as_tensor(units, device="cuda")
    check(out["dA"][:, u], bw_units["dA"], "dA cols", "bf16")
    check(out["dbA"][u], bw_units["dbA"], "dbA", "bf16")
    check(out["dB"][u], bw_units["dB"], "dB rows", "bf16")
    check(out["dbB"], bw_units["dbB"], "dbB", "bf16")


@pytest.mark.parametrize("t", [3, 64])
def test_mlp_uncommon_shard_counts(t):
    """t = 3 (f / t = 256) and t = 64 (f / t = 8, one 8-column group per shard)."""
    wl = Workload(93, "uncommon t", b=1, s=136, h=128, f=768 if t == 3 else 512, t=t,
                  w_std=0.05, bias_std=0.05)
    inp = make_mlp_inputs(wl)
    compare_full(gpu_mlp(inp, t), inp, "bf16")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_mlp_single_token(dtype):
    """M = 1: one row in a 128-row tile (the rest of the tile is out of range)."""
    wl = Workload(94, "one token", b=1, s=1, h=256, f=1024, t=4, w_std=0.05, bias_std=0.05,
                  dtype="f32" if dtype == torch.float32 else "bf16")
    inp = make_mlp_inputs(wl)
    compare_full(gpu_mlp(inp, wl.t, dtype=dtype), inp, "f32" if dtype == torch.float32 else "bf16")


def _bf16_ulp(v):
    """The spacing of bf16 numbers at |v| (8 significant bits)."""
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def test_gelu_epilogues_against_exact_erf():
    """The GeLU of the first GEMM's epilogue, the GeLU' of the dgrad epilogue
    and the GeLU the dgrad epilogue recomputes for dB, each against the erf
    form in fp64 (the oracle's), on one token whose h = 2048 entries sweep
    [-8, 8] plus special values.  With A = B = I the MLP exposes them
    exactly: Z = bf16(GeLU(x)) (one product per output), and with dZ = 1
    the backward gives dbA = bf16(GeLU'(x)) and every column of dB =
    bf16(GeLU(x)).  The bound is half a bf16 unit of the exact value (the
    rounding) plus 1e-6 (times |x| for GeLU): the erf approximation's
    absolute error of 1.5e-7 with the approximate reciprocal, exponential
    and fp32 rounding on top, still far below a bf16 unit."""
    h = 2048
    x = np.linspace(-8.0, 8.0, h)
    x[:8] = [0.0, 1e-3, -1e-3, 1e-30, -1e-30, 0.5, -0.5, -13.0]
    X = torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).reshape(1, h)
    xb = X.double().numpy().ravel()
    eye = torch.eye(h, dtype=torch.bfloat16)
    inp = {"X": X, "A": eye, "B": eye.clone(), "bA": None, "bB": None,
           "dZ": torch.ones(1, h, dtype=torch.bfloat16)}
    out = gpu_mlp(inp, t=2)
    g_exact, gp_exact = O.gelu(xb), O.gelu_prime(xb)
    z = out["Z"].double().cpu().numpy().ravel()
    dba = out["dbA"].double().cpu().numpy().ravel()
    db0 = out["dB"][:, 0].double().cpu().numpy().ravel()
    tol_g = 0.5 * _bf16_ulp(g_exact) + np.abs(xb) * 1e-6 + 1e-30
    tol_gp = 0.5 * _bf16_ulp(gp_exact) + 1e-6
    assert np.all(np.abs(z - g_exact) <= tol_g), np.max(np.abs(z - g_exact) / tol_g)
    assert np.all(np.abs(dba - gp_exact) <= tol_gp), np.max(np.abs(dba - gp_exact) / tol_gp)
    assert np.all(np.abs(db0 - g_exact) <= tol_g)
    # The forward and the backward evaluate GeLU the same way, bit for bit.
    assert np.array_equal(z, db0)
    assert np.array_equal(out["Y"].double().cpu().numpy().ravel(), xb)
