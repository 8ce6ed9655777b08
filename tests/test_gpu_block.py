"""GPU parity of LayerNorm and the Transformer block against the oracle.

The block is the PyTorch tutorial's ParallelTransformerBlock (§3.3):
X1 = X + Attn(LN1(X)); X2 = X1 + MLP(LN2(X1)), with the attention and MLP
partitioned as in "图解Transformer并行计算" §2-§3 and the residual additions
fused into the row-split GEMMs' epilogues.
"""
import numpy as np
import pytest
import torch

from megatron_tensor_transformer_logical_b200 import binding as L
from megatron_tensor_transformer_logical_b200.inputs import WORKLOADS, normal_tensor
from oracle import tp_oracle as O
from tests.parity import check, cuda, need_gpu, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()
    yield
    L.tp_device_status()


def gpu_ln(X, g, b, dY, dR, eps=1e-5):
    M, h = X.shape
    dt = X.dtype
    Y = torch.empty_like(X)
    mean = torch.empty(M, dtype=torch.float32, device="cuda")
    rstd = torch.empty(M, dtype=torch.float32, device="cuda")
    L.tp_layernorm_fwd(X, g, b, Y, mean, rstd, eps)
    dX = torch.empty_like(X)
    dg = torch.empty(h, dtype=dt, device="cuda") if g is not None else None
    db = torch.empty(h, dtype=dt, device="cuda") if g is not None else None
    ws = L.workspace(L.TP_OP_LN_BWD, M, h, 0, 0, 1, L.TP_F32 if dt == torch.float32 else L.TP_BF16)
    L.tp_layernorm_bwd(X, g, mean, rstd, dY, dR, dX, dg, db, ws)
    torch.cuda.synchronize()
    return Y, mean, rstd, dX, dg, db


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", [(300, 264), (7, 16384), (2048, 12288)], ids=["ragged", "widest", "175b"])
def test_layernorm_fwd_bwd(dtype, shape):
    M, h = shape
    X = normal_tensor((M, h), 2.0, 1, dtype)
    X = X + normal_tensor((M, 1), 1.0, 2, dtype)  # a per-row offset the norm must remove
    g, b = normal_tensor((h,), 0.5, 3, dtype), normal_tensor((h,), 0.5, 4, dtype)
    dY, dR = normal_tensor((M, h), 1.0, 5, dtype), normal_tensor((M, h), 1.0, 6, dtype)
    Y, mean, rstd, dX, dg, db = gpu_ln(*(cuda(v) for v in (X, g, b, dY, dR)))
    fw = O.layernorm_fwd(X, g, b, 1e-5)
    bw = O.layernorm_bwd(X, g, dY, 1e-5)
    check(Y, fw["Y"], "Y", dtype)
    assert np.max(np.abs(to64(mean) - fw["mean"])) <= 1e-4 * np.max(np.abs(fw["mean"])) + 1e-5
    assert np.max(np.abs(to64(rstd) / fw["rstd"] - 1)) < 1e-4
    check(dX, bw["dX"] + to64(dR), "dX (+ residual gradient)", dtype)
    check(dg, bw["dgamma"], "dgamma", dtype)
    check(db, bw["dbeta"], "dbeta", dtype)


def make_block(b, s, h, f, heads, seed, w_std=0.05):
    t = lambda shape, std, k: normal_tensor(shape, std, seed * 100 + k)
    w = {"ln1_g": 1 + t((h,), 0.1, 1), "ln1_b": t((h,), 0.1, 2),
         "Wqkv": t((h, 3 * h), w_std, 3), "Wo": t((h, h), w_std, 4),
         "ln2_g": 1 + t((h,), 0.1, 5), "ln2_b": t((h,), 0.1, 6),
         "A": t((h, f), w_std, 7), "bA": t((f,), 0.05, 8), "B": t((f, h), w_std, 9),
         "bB": t((h,), 0.05, 10)}
    w = {k: v.to(torch.bfloat16) for k, v in w.items()}
    X = t((b * s, h), 1.0, 11)
    dX2 = t((b * s, h), 1.0, 12)
    return w, X, dX2


def gpu_block(w, X, dX2, b, s, f, heads, t, eps=1e-5):
    M, h = X.shape
    wd = {k: cuda(v) for k, v in w.items()}
    Xd, dX2d = cuda(X), cuda(dX2)
    e = lambda *sh, dt=torch.bfloat16: torch.empty(*sh, dtype=dt, device="cuda")
    sv = {"Xn1": e(M, h), "mean1": e(M, dt=torch.float32), "rstd1": e(M, dt=torch.float32),
          "QKV": e(M, 3 * h, dt=torch.float16), "O": e(M, h),
          "LSE": e(b, heads, s, dt=torch.float32), "X1": e(M, h), "Xn2": e(M, h),
          "mean2": e(M, dt=torch.float32), "rstd2": e(M, dt=torch.float32), "Y": e(M, f)}
    X2 = e(M, h)
    L.tp_block_fwd(Xd, wd, X2, sv, b, s, f, heads, t, eps,
                   L.workspace(L.TP_OP_BLOCK_FWD, M, h, f, heads, t, L.TP_BF16))
    g = {k: torch.empty_like(wd[k[1:]]) for k in ("dWqkv", "dWo", "dA", "dB")}
    for k in ("dln1_g", "dln1_b", "dln2_g", "dln2_b", "dbA", "dbB"):
        g[k] = torch.empty_like(wd[k[1:]])
    dX = e(M, h)
    L.tp_block_bwd(Xd, wd, sv, dX2d, dX, g, b, s, f, heads, t, eps,
                   L.workspace(L.TP_OP_BLOCK_BWD, M, h, f, heads, t, L.TP_BF16))
    torch.cuda.synchronize()
    return X2, sv, dX, g


@pytest.mark.parametrize("tile", ["auto", "192"])
def test_block_small_vs_oracle(monkeypatch, tile):
    """Tile 192 takes the residual epilogues through the aux rows fetched a
    chunk ahead, across a ragged column tile and from one unit to the next."""
    if tile != "auto":
        monkeypatch.setenv("TP_GEMM_TILE", tile)
    b, s, h, f, heads, t = 2, 96, 256, 1024, 2, 2
    w, X, dX2 = make_block(b, s, h, f, heads, 7)
    X2, sv, dX, g = gpu_block(w, X, dX2, b, s, f, heads, t)
    w64 = {k: to64(v) for k, v in w.items()}
    fw = O.block_fwd(X, w64, b, s, heads)
    bw = O.block_bwd(X, w64, dX2, b, s, heads)
    check(sv["X1"], fw["X1"], "X1", "bf16")
    check(X2, fw["X2"], "X2", "bf16")
    check(dX, bw["dX"], "dX", "bf16")
    for k in ("dln1_g", "dln1_b", "dWqkv", "dWo", "dln2_g", "dln2_b", "dA", "dbA", "dB", "dbB"):
        check(g[k], bw[k], k, "bf16")


def test_block_175b_forward_first_rows():
    """The 175B-shaped block at full size; under the causal mask the block's
    rows 0..255 depend only on rows 0..255, so the oracle on the first 256
    tokens is exact for them."""
    wl = WORKLOADS[5]
    w, X, dX2 = make_block(1, wl.s, wl.h, wl.f, wl.heads, 8, w_std=0.006)
    X2, sv, dX, g = gpu_block(w, X, dX2, 1, wl.s, wl.f, wl.heads, wl.t)
    r = 256
    w64 = {k: to64(v) for k, v in w.items()}
    fw = O.block_fwd(to64(X)[:r], w64, 1, r, wl.heads)
    check(X2[:r], fw["X2"], "X2 rows < 256", "bf16")
    check(sv["X1"][:r], fw["X1"], "X1 rows < 256", "bf16")
    assert torch.isfinite(dX.float()).all()
