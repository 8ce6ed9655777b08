"""GPU parity of head-wise partitioned attention, forward and backward.

"图解Transformer并行计算" §3.2: Wqkv split by columns in head groups, each
group runs its heads' softmax(Q K^T / sqrt(d)) V, Wo split by rows and the
group partials summed; backward mirrors it (dWqkv, dWo per group, dX summed).
"""
import numpy as np
import pytest
import torch

from megatron_tensor_transformer_logical_b200 import binding as L
from megatron_tensor_transformer_logical_b200.inputs import WORKLOADS, Workload, make_attn_inputs
from oracle import tp_oracle as O
from tests.parity import check, cuda, need_gpu, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()
    yield
    L.tp_device_status()


def gpu_attn(inp, wl, causal=True, save_qkv=True, t=None):
    t = wl.t if t is None else t
    d = {k: cuda(v) for k, v in inp.items()}
    M, h = wl.M, wl.h
    Z = torch.empty(M, h, dtype=torch.bfloat16, device="cuda")
    QKV = torch.empty(M, 3 * h, dtype=torch.float16, device="cuda") if save_qkv else None
    Os = torch.empty(M, h, dtype=torch.bfloat16, device="cuda")
    LSE = torch.empty(wl.b, wl.heads, wl.s, dtype=torch.float32, device="cuda")
    L.tp_attn_fwd(d["X"], d["Wqkv"], d["Wo"], Z, QKV, Os, LSE, wl.b, wl.s, wl.heads, t, causal,
                  L.workspace(L.TP_OP_ATTN_FWD, M, h, 0, wl.heads, t, L.TP_BF16))
    dX, dWqkv, dWo = (torch.empty_like(d[k]) for k in ("X", "Wqkv", "Wo"))
    L.tp_attn_bwd(d["X"], d["Wqkv"], d["Wo"], QKV, Os, LSE, d["dZ"], dX, dWqkv, dWo, wl.b, wl.s,
                  wl.heads, t, causal,
                  L.workspace(L.TP_OP_ATTN_BWD, M, h, 0, wl.heads, t, L.TP_BF16))
    torch.cuda.synchronize()
    return {"Z": Z, "QKV": QKV, "O": Os, "LSE": LSE, "dX": dX, "dWqkv": dWqkv, "dWo": dWo}


def compare_full(out, inp, wl, causal):
    fw = O.attn_fwd(inp["X"], inp["Wqkv"], inp["Wo"], wl.b, wl.s, wl.heads, causal)
    bw = O.attn_bwd(inp["X"], inp["Wqkv"], inp["Wo"], inp["dZ"], wl.b, wl.s, wl.heads, causal)
    for k in ("Z", "O"):
        check(out[k], fw[k], k, "bf16")
    if out["QKV"] is not None:
        check(out["QKV"], fw["QKV"], "QKV", "bf16")
    assert np.max(np.abs(to64(out["LSE"]) - fw["LSE"])) < 2e-2
    for k in ("dX", "dWqkv", "dWo"):
        check(out[k], bw[k], k, "bf16")


@pytest.mark.parametrize("tile", ["auto", "192", "pair"])
@pytest.mark.parametrize("causal", [True, False], ids=["causal", "full"])
@pytest.mark.parametrize("save_qkv", [True, False], ids=["QKVsave", "recompute"])
def test_attention_small_ragged(monkeypatch, causal, save_qkv, tile):
    if tile != "auto":
        monkeypatch.setenv("TP_GEMM_TILE", tile)
    # s = 200: four 64-row query blocks (the last ragged), seven 32-row blocks.
    wl = Workload(80, "attn ragged", b=2, s=200, h=512, heads=4, t=2, w_std=0.05)
    inp = make_attn_inputs(wl)
    compare_full(gpu_attn(inp, wl, causal, save_qkv), inp, wl, causal)


@pytest.mark.parametrize("causal", [True, False], ids=["causal", "full"])
def test_attention_row_maximum_rising_across_blocks(causal):
    """Scores that rise by about 30 (log2 units) from one 128-key block to
    the next, so the forward raises its row maximum and rescales O and the
    row sum in tensor memory at every block ("图解Transformer并行计算" §3.2
    step 2: the softmax must not depend on when the maximum is raised).
    Column 0 of X is a ramp and feeds q[0] and k[0] of every head alone,
    through exact power-of-two weights, so the large score component is exact
    in fp16.

    The forward is compared in both masks.  The backward is compared under
    the causal mask only: with every row as sharp as this and all keys
    visible, D = rowsum(dO * O) taken from the bf16-rounded O moves the score
    gradient P (dP - D) enough that dX sits at the bf16 bar (5.9e-3
    normwise measured; a rounding-point emulation in fp64 gives the same,
    and 2.3e-3 with O unrounded)."""
    wl = Workload(86, "attn rising max", b=1, s=520, h=256, heads=2, t=2, w_std=0.05)
    inp = make_attn_inputs(wl)
    X, W = inp["X"].clone(), inp["Wqkv"].clone()
    ramp = torch.round(torch.arange(wl.s, dtype=torch.float64) * (64.0 / wl.s)) / 16.0
    X[:, 0] = ramp.to(X.dtype)  # 0 .. 4 in steps of 1/16: exact in bf16
    for head in range(wl.heads):
        for col in (head * 128, wl.h + head * 128):  # q[0] and k[0] of the head
            W[:, col] = 0.0
            W[0, col] = 8.0
    inp["X"], inp["Wqkv"] = X, W
    # The construction does what it says: for the last row, the best score of
    # each key block exceeds that of the block before by more than 8.
    x64, w64 = to64(X), to64(W)
    q, k = x64 @ w64[:, :128], x64 @ w64[:, wl.h:wl.h + 128]
    t = (q[-1] @ k.T) / np.sqrt(128.0) / np.log(2.0)
    assert all(t[128 * (i + 1):128 * (i + 2)].max() - t[128 * i:128 * (i + 1)].max() > 8.0
               for i in range(3))
    out = gpu_attn(inp, wl, causal)
    if causal:
        compare_full(out, inp, wl, causal)
        return
    fw = O.attn_fwd(inp["X"], inp["Wqkv"], inp["Wo"], wl.b, wl.s, wl.heads, causal)
    for key in ("Z", "O", "QKV"):
        check(out[key], fw[key], key, "bf16")
    assert np.max(np.abs(to64(out["LSE"]) - fw["LSE"])) < 2e-2


def test_attention_single_token_and_short():
    # s = 1 (a row that sees only itself: O = V) and s = 3.
    for s in (1, 3):
        wl = Workload(81, "attn short", b=3, s=s, h=256, heads=2, t=2, w_std=0.05)
        inp = make_attn_inputs(wl)
        out = gpu_attn(inp, wl)
        compare_full(out, inp, wl, True)
        if s == 1:
            qkv = to64(out["QKV"])
            assert np.allclose(to64(out["O"]), qkv[:, 2 * wl.h:], rtol=1e-2, atol=1e-2)


def test_attention_group_count_sweep():
    """t = 1, 2, 4: forward results and the per-group weight gradients agree
    bitwise (grouping only moves tile boundaries); dX agrees within tolerance
    (its K loop visits the groups' ranges in group order)."""
    wl = Workload(82, "attn t sweep", b=2, s=256, h=512, heads=4, t=1, w_std=0.05)
    inp = make_attn_inputs(wl)
    outs = {t: gpu_attn(inp, wl, t=t) for t in (1, 2, 4)}
    for t in (2, 4):
        for k in ("Z", "QKV", "O", "LSE", "dWqkv", "dWo"):
            assert torch.equal(outs[t][k], outs[1][k]), (t, k)
        check(outs[t]["dX"], to64(outs[1]["dX"]), f"dX t={t} vs t=1", "bf16")
    compare_full(outs[4], inp, wl, True)


def _head_slice(W, h, heads, j):
    c = O.head_columns(h, heads, j)
    return np.concatenate([c["q"], c["k"], c["v"]])


def test_attention_config4_full_size():
    """Config 4 (b=4, s=2048, h=4096, 32 heads, t=8) at full size.

    Rows of one batch element depend on that element alone, so the oracle on
    each batch element is exact for its rows (Z, O, LSE and dX are checked
    for all four); dWqkv columns and dWo rows of one head depend on that head
    alone, so a one-head oracle is exact for them.
    """
    wl = WORKLOADS[4]
    inp = make_attn_inputs(wl)
    out = gpu_attn(inp, wl)
    X, Wqkv, Wo, dZ = (to64(inp[k]) for k in ("X", "Wqkv", "Wo", "dZ"))
    for bi in range(wl.b):
        rows = slice(bi * wl.s, (bi + 1) * wl.s)
        fw = O.attn_fwd(X[rows], Wqkv, Wo, 1, wl.s, wl.heads)
        bw = O.attn_bwd(X[rows], Wqkv, Wo, dZ[rows], 1, wl.s, wl.heads)
        check(out["Z"][rows], fw["Z"], f"Z (batch {bi})", "bf16")
        check(out["O"][rows], fw["O"], f"O (batch {bi})", "bf16")
        assert np.max(np.abs(to64(out["LSE"][bi]) - fw["LSE"][0])) < 2e-2
        check(out["dX"][rows], bw["dX"], f"dX (batch {bi})", "bf16")
    for j in (0, 13, 31):  # heads in groups 0, 3 and 7
        cols = _head_slice(Wqkv, wl.h, wl.heads, j)
        d = wl.h // wl.heads
        w_rows = slice(j * d, (j + 1) * d)
        bj = O.attn_bwd(X, Wqkv[:, cols], Wo[w_rows], dZ, wl.b, wl.s, 1)
        c = torch.as_tensor(cols, device="cuda")
        check(out["dWqkv"][:, c], bj["dWqkv"], f"dWqkv head {j}", "bf16")
        check(out["dWo"][w_rows], bj["dWo"], f"dWo head {j}", "bf16")


def test_attention_config5_sampled():
    """Config 5 attention (s=2048, h=12288, 96 heads, t=8).

    With the causal mask, rows 0..255 depend only on rows 0..255, so the
    oracle on the first 256 tokens is exact for them; per-head quantities
    (O columns, LSE, dWqkv columns, dWo rows) come from a one-head oracle.
    """
    wl = WORKLOADS[5]
    inp = make_attn_inputs(wl)
    out = gpu_attn(inp, wl)
    X, Wqkv, Wo, dZ = (to64(inp[k]) for k in ("X", "Wqkv", "Wo", "dZ"))
    r = 256
    fw = O.attn_fwd(X[:r], Wqkv, Wo, 1, r, wl.heads)
    check(out["Z"][:r], fw["Z"], "Z rows < 256", "bf16")
    d = wl.h // wl.heads
    for j in (0, 50, 95):
        cols = _head_slice(Wqkv, wl.h, wl.heads, j)
        w_rows = slice(j * d, (j + 1) * d)
        fj = O.attn_fwd(X, Wqkv[:, cols], Wo[w_rows], 1, wl.s, 1)
        check(out["O"][:, j * d:(j + 1) * d], fj["O"], f"O head {j}", "bf16")
        assert np.max(np.abs(to64(out["LSE"][0, j]) - fj["LSE"][0, 0])) < 2e-2
        bj = O.attn_bwd(X, Wqkv[:, cols], Wo[w_rows], dZ, 1, wl.s, 1)
        c = torch.as_tensor(cols, device="cuda")
        check(out["dWqkv"][:, c], bj["dWqkv"], f"dWqkv head {j}", "bf16")
        check(out["dWo"][w_rows], bj["dWo"], f"dWo head {j}", "bf16")


def test_fp16_range_overflow_is_reported():
    """QKV beyond the fp16 range is saturated and reported as TP_ERR_KERNEL."""
    wl = Workload(83, "attn overflow", b=1, s=64, h=256, heads=2, t=1, w_std=0.05)
    inp = make_attn_inputs(wl)
    inp["X"] = torch.full_like(inp["X"], 256.0)
    inp["Wqkv"] = torch.full_like(inp["Wqkv"], 2.0)  # every QKV entry = 256 * 2 * 256
    d = {k: cuda(v) for k, v in inp.items()}
    M, h = wl.M, wl.h
    Z = torch.empty(M, h, dtype=torch.bfloat16, device="cuda")
    QKV = torch.empty(M, 3 * h, dtype=torch.float16, device="cuda")
    L.tp_attn_fwd(d["X"], d["Wqkv"], d["Wo"], Z, QKV, None, None, wl.b, wl.s, wl.heads, 1, True,
                  L.workspace(L.TP_OP_ATTN_FWD, M, h, 0, wl.heads, 1, L.TP_BF16))
    with pytest.raises(L.TPError) as e:
        L.tp_device_status()
    assert e.value.status == L.TP_ERR_KERNEL and "fp16" in str(e.value)
    assert torch.isfinite(QKV.float()).all() and QKV.float().max().item() == 65504.0
    L.tp_device_status()  # the word was cleared


def test_attention_with_last_wave_split():
    """b = 2, s = 2048, h = 4096 (32 heads), t = 8: the dO GEMM (fp16 output,
    single-SM tiles) and the dX GEMM (SM-pair tiles, head-group K order) both
    leave a last wave under half full, which they split along K and add back
    in a fixup kernel; the whole layer is compared with the oracle."""
    wl = Workload(97, "last-wave split", b=2, s=2048, h=4096, heads=32, t=8, w_std=0.02)
    inp = make_attn_inputs(wl)
    compare_full(gpu_attn(inp, wl), inp, wl, True)


def test_mlp_with_last_wave_split_all_epilogues():
    """M = h = f = 4096, t = 8, with biases: each of the six MLP GEMMs leaves a
    last wave of under half the SMs or SM pairs (512 single-SM or 256 pair
    tiles on 148 SMs), so the bias + GeLU, GeLU', plain and wgrad epilogues
    all run through the K split, whose last slice's CTA adds the slices;
    compared with the oracle on every output."""
    from megatron_tensor_transformer_logical_b200.inputs import make_mlp_inputs
    wl = Workload(98, "mlp last-wave split", b=2, s=2048, h=4096, f=4096, t=8, w_std=0.02,
                  bias_std=0.02)
    inp = make_mlp_inputs(wl)
    d = {k: cuda(v) for k, v in inp.items()}
    M, h, f = wl.M, wl.h, wl.f
    Z = torch.empty(M, h, dtype=torch.bfloat16, device="cuda")
    Y = torch.empty(M, f, dtype=torch.bfloat16, device="cuda")
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for kind in (256, 512):  # the plan splits the last wave whichever tile kind runs
        assert any(u["part"] >= 0 for u in L.tp_gemm_plan(M, f, h, f // wl.t, kind, sms, True))
    L.tp_mlp_fwd(d["X"], d["A"], d["bA"], d["B"], d["bB"], Z, Y, wl.t,
                 L.workspace(L.TP_OP_MLP_FWD, M, h, f, 0, wl.t, L.TP_BF16))
    g = {k: torch.empty_like(d[k]) for k in ("X", "A", "B")}
    dbA = torch.empty(f, dtype=torch.bfloat16, device="cuda")
    dbB = torch.empty(h, dtype=torch.bfloat16, device="cuda")
    L.tp_mlp_bwd(d["X"], d["A"], d["bA"], d["B"], Y, d["dZ"], g["X"], g["A"], dbA, g["B"], dbB,
                 wl.t, L.workspace(L.TP_OP_MLP_BWD, M, h, f, 0, wl.t, L.TP_BF16))
    torch.cuda.synchronize()
    fw = O.mlp_fwd(inp["X"], inp["A"], inp["bA"], inp["B"], inp["bB"])
    bw = O.mlp_bwd(inp["X"], inp["A"], inp["bA"], inp["B"], inp["dZ"])
    check(Z, fw["Z"], "Z", "bf16")
    check(Y, fw["Y"], "Y", "bf16")
    for k, v in (("dX", g["X"]), ("dA", g["A"]), ("dB", g["B"]), ("dbA", dbA), ("dbB", dbB)):
        check(v, bw[k], k, "bf16")
