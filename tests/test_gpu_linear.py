"""GPU parity of the column- and row-parallel linear layers against the oracle.

Column split ("图解Transformer并行计算" §1.2): Y = concat_i X @ W_i.
Row split (same page, §1.1): Z = sum_i X_i @ W_i, summed in the kernel.
Shard slicing must be bit-exact; integer-valued inputs give exact sums.
"""
import numpy as np
import pytest
import torch

from megatron_tensor_transformer_logical_b200 import binding as L
from megatron_tensor_transformer_logical_b200.inputs import (WORKLOADS, integer_tensor,
                                                             make_linear_inputs, normal_tensor)
from oracle import tp_oracle as O
from tests.parity import check, cuda, need_gpu, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu(monkeypatch):
    need_gpu()
    yield
    L.tp_device_status()


def run(mode, X, W, b, t, shard=-1, out_dtype=torch.bfloat16):
    M, K = X.shape
    N = W.shape[1]
    if mode == "col":
        Y = torch.full((M, N // t if shard >= 0 else N), float("nan"), dtype=out_dtype, device="cuda")
        L.tp_linear_col(X, W, b, Y, t, shard)
    else:
        Y = torch.full((M, N), float("nan"), dtype=out_dtype, device="cuda")
        L.tp_linear_row(X, W, b, Y, t, shard)
    torch.cuda.synchronize()
    return Y


# M spans 3 row tiles of 128 (2 pair tiles of 256) with a ragged tail, N 3
# column tiles of 256 (ragged), K 5 blocks of 64; every K/t and N/t is a
# multiple of 8.  TP_GEMM_TILE forces the 128-, 192- or 256-wide single-SM tile or
# the 256 x 256 two-SM tile.
SMALL = (300, 320, 576)


@pytest.mark.parametrize("tile", ["128", "192", "256", "pair"])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("t", [1, 2, 4, 8])
@pytest.mark.parametrize("mode", ["col", "row"])
def test_linear_random_small(monkeypatch, mode, t, out_dtype, tile):
    monkeypatch.setenv("TP_GEMM_TILE", tile)
    M, K, N = SMALL
    X, W = normal_tensor((M, K), 1.0, 1), normal_tensor((K, N), 0.05, 2)
    b = normal_tensor((N,), 0.1, 3)
    Y = run(mode, cuda(X), cuda(W), cuda(b), t, out_dtype=out_dtype)
    ref = O.linear(X, W, b)
    if out_dtype == torch.float32:
        assert O.max_rel_error(to64(Y), ref) <= 1e-5
    else:
        check(Y, ref, f"{mode} t={t}", "bf16")


@pytest.mark.parametrize("tile", ["128", "192", "256", "pair"])
@pytest.mark.parametrize("t", [1, 2, 4, 8])
@pytest.mark.parametrize("mode", ["col", "row"])
def test_linear_integer_bit_exact(monkeypatch, mode, t, tile):
    monkeypatch.setenv("TP_GEMM_TILE", tile)
    M, K, N = SMALL
    X, W = integer_tensor((M, K), -3, 3, 4), integer_tensor((K, N), -3, 3, 5)
    b = integer_tensor((N,), -8, 8, 6)
    Y = run(mode, cuda(X), cuda(W), cuda(b), t, out_dtype=torch.float32)
    assert np.array_equal(to64(Y), O.linear(X, W, b))


@pytest.mark.parametrize("tile", ["192", "256", "pair"])
@pytest.mark.parametrize("t", [2, 4, 8])
def test_column_shard_slices_bit_exact(monkeypatch, t, tile):
    monkeypatch.setenv("TP_GEMM_TILE", tile)
    M, K, N = SMALL
    X, W = cuda(normal_tensor((M, K), 1.0, 7)), cuda(normal_tensor((K, N), 0.05, 8))
    b = cuda(normal_tensor((N,), 0.1, 9))
    for out_dtype in (torch.bfloat16, torch.float32):
        full = run("col", X, W, b, t, out_dtype=out_dtype)
        w = N // t
        for i in range(t):
            part = run("col", X, W, b, t, shard=i, out_dtype=out_dtype)
            assert torch.equal(part, full[:, i * w:(i + 1) * w]), (t, i)


@pytest.mark.parametrize("tile", ["256", "pair"])
@pytest.mark.parametrize("t", [2, 4, 8])
def test_row_shard_partials_sum_to_full(monkeypatch, t, tile):
    monkeypatch.setenv("TP_GEMM_TILE", tile)
    M, K, N = SMALL
    X, W = integer_tensor((M, K), -3, 3, 10), integer_tensor((K, N), -3, 3, 11)
    b = integer_tensor((N,), -8, 8, 12)
    Xc, Wc, bc = cuda(X), cuda(W), cuda(b)
    full = run("row", Xc, Wc, bc, t, out_dtype=torch.float32)
    parts = [run("row", Xc, Wc, bc, t, shard=i, out_dtype=torch.float32) for i in range(t)]
    total = parts[0].clone()
    for p in parts[1:]:
        total += p
    assert torch.equal(total, full)
    _, ref_parts = O.linear_row_parallel(X, W, None, t, return_partials=True)
    for i, p in enumerate(parts):
        expect = ref_parts[i] + (to64(b) if i == 0 else 0.0)
        assert np.array_equal(to64(p), expect), i


def test_linear_config3_full_size_sampled():
    """Config 3 at full size (8192 x 4096 @ 4096 x 16384), t in {1,2,4,8}, both modes.

    Rows are independent, so sampled rows of the oracle are exact references.
    Results for every t must agree bitwise (same K order, same per-column work).
    """
    wl = WORKLOADS[3]
    inp = make_linear_inputs(wl)
    X, W = cuda(inp["X"]), cuda(inp["W"])
    rows = np.unique(np.r_[0, 1, 127, 128, 4095, 8191,
                           np.random.default_rng(0).integers(0, wl.M, 58)])
    ref = O.linear(inp["X"][rows], inp["W"])
    for mode in ("col", "row"):
        first = None
        for t in (1, 2, 4, 8):
            Y = run(mode, X, W, None, t)
            check(Y[torch.as_tensor(rows, device="cuda")], ref, f"config3 {mode} t={t}", "bf16")
            if first is None:
                first = Y
            else:
                assert torch.equal(Y, first), f"{mode}: t={t} differs from t=1"
            del Y


UNCOMMON = {("col", 3): (200, 320, 960), ("col", 5): (200, 320, 960), ("col", 64): (200, 320, 512),
            ("row", 3): (200, 1536, 320), ("row", 5): (200, 1280, 320), ("row", 64): (200, 4096, 320)}


@pytest.mark.parametrize("t", [3, 5, 64])
@pytest.mark.parametrize("mode", ["col", "row"])
def test_linear_uncommon_shard_counts(mode, t):
    """Shard counts that are not powers of two, and the largest allowed (64,
    8 columns per shard for the column split: the narrowest shard-aligned
    tiles).  Integer-valued inputs: exact."""
    M, K, N = UNCOMMON[(mode, t)]
    X, W = integer_tensor((M, K), -3, 3, 14), integer_tensor((K, N), -3, 3, 15)
    b = integer_tensor((N,), -8, 8, 16)
    Xc, Wc, bc = cuda(X), cuda(W), cuda(b)
    Y = run(mode, Xc, Wc, bc, t, out_dtype=torch.float32)
    assert np.array_equal(to64(Y), O.linear(X, W, b))
    if mode == "col":
        w = N // t
        for i in (0, t // 2, t - 1):
            part = run("col", Xc, Wc, bc, t, shard=i, out_dtype=torch.float32)
            assert torch.equal(part, Y[:, i * w:(i + 1) * w]), i
    else:
        parts = [run("row", Xc, Wc, bc, t, shard=i, out_dtype=torch.float32) for i in range(t)]
        total = parts[0].clone()
        for p in parts[1:]:
            total += p
        assert torch.equal(total, Y)


@pytest.mark.parametrize("mode", ["col", "row"])
def test_linear_single_row_exact(mode):
    """M = 1 with integer-valued inputs: exact for every shard count."""
    K, N = 512, 1024
    X, W = integer_tensor((1, K), -3, 3, 17), integer_tensor((K, N), -3, 3, 18)
    for t in (1, 2, 8):
        Y = run(mode, cuda(X), cuda(W), None, t, out_dtype=torch.float32)
        assert np.array_equal(to64(Y), O.linear(X, W, None)), t
