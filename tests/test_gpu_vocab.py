"""GPU parity of the vocabulary-parallel embedding and cross-entropy against
the oracle ("图解Transformer并行计算：从矩阵乘法切分到Megatron架构设计" §4.1, §4.2).

Embedding: a gather and its transpose, compared bit for bit where the
arithmetic is exact (integer-valued gradients) and with the bf16 tolerance
otherwise.  Cross-entropy: the logits GEMM (bf16 in, fp32 accumulate, bf16
logits), its per-chunk reductions and the shard combination, then the
backward's softmax gradient and two GEMMs; compared with the fp64 oracle at
the bf16 tolerance.
"""
import numpy as np
import pytest
import torch

from megatron_tensor_transformer_logical_b200 import binding as L
from megatron_tensor_transformer_logical_b200.inputs import (WORKLOADS, Workload, integer_tensor,
                                                             make_vocab_inputs, normal_tensor,
                                                             zipf_ids)
from oracle import tp_oracle as O
from tests.parity import check, cuda, need_gpu, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()
    yield
    L.tp_device_status()


# ------------------------------------------------------------------ embedding

def embed_bwd(ids, dY, dE_in, dE, t):
    M = ids.numel()
    ws = (L.workspace(L.TP_OP_VOCAB_EMBED_BWD, M, dE.shape[1], dE.shape[0], 0, t, L.TP_BF16)
          if M > 0 else None)
    L.tp_vocab_embed_bwd(ids, dY, dE_in, dE, t, ws)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("t", [1, 2, 8])
def test_embed_fwd_exact(dtype, t):
    V, h, M = 1024, 264, 777
    E = normal_tensor((V, h), 1.0, 1, dtype)
    ids = zipf_ids(M, V, 2)
    ids[::97] = -1          # out of range on both sides: zero rows
    ids[5::131] = V
    Y = torch.full((M, h), float("nan"), dtype=E.dtype, device="cuda")
    L.tp_vocab_embed_fwd(cuda(ids), cuda(E), Y, t)
    torch.cuda.synchronize()
    assert np.array_equal(to64(Y), O.vocab_embed_fwd_parallel(ids.numpy(), E, t))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("accumulate", [False, True], ids=["plain", "plus_dE_in"])
def test_embed_bwd_integer_exact(dtype, accumulate):
    """Integer-valued dY: every partial sum is an exact integer below 2^8 in
    magnitude, so the scatter-add is exact in any order and in bf16."""
    V, h, M = 1000, 2056, 3000  # ragged row blocks and column slices; 2 rounds of ids
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    ids = zipf_ids(M, V, 3, exponent=0.6)
    ids[::50] = -3
    dY = integer_tensor((M, h), -1, 1, 4, tdt)
    dE_in = integer_tensor((V, h), -4, 4, 5, tdt) if accumulate else None
    dE = torch.full((V, h), float("nan"), dtype=tdt, device="cuda")
    embed_bwd(cuda(ids), cuda(dY), cuda(dE_in), dE, 4)
    torch.cuda.synchronize()
    ref = O.vocab_embed_bwd(ids.numpy(), dY, V)
    if accumulate:
        ref = ref + to64(dE_in)
    assert np.max(np.abs(ref)) < 256
    assert np.array_equal(to64(dE), ref)


def test_embed_bwd_in_place_and_hot_token():
    """dE_in aliasing dE, and one id taking every token (the longest list)."""
    V, h, M = 64, 512, 5000
    ids = torch.full((M,), 17, dtype=torch.int32)
    ids[::7] = 3
    dY = normal_tensor((M, h), 1.0, 6)
    base = normal_tensor((V, h), 1.0, 7)
    dE = cuda(base.clone())
    embed_bwd(cuda(ids), cuda(dY), dE, dE, 1)
    torch.cuda.synchronize()
    check(dE, O.vocab_embed_bwd(ids.numpy(), dY, V) + to64(base), "dE (in place)", "bf16")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_embed_bwd_many_tokens_exact(dtype):
    """More than 16384 tokens: the per-group id scan instead of the sort."""
    V, h, M = 640, 1032, 20000
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    ids = zipf_ids(M, V, 11, exponent=0.3)
    ids[::1000] = V + 5
    dY = integer_tensor((M, h), -1, 1, 12, tdt)
    dE_in = integer_tensor((V, h), -4, 4, 13, tdt)
    dE = torch.full((V, h), float("nan"), dtype=tdt, device="cuda")
    embed_bwd(cuda(ids), cuda(dY), cuda(dE_in), dE, 8)
    torch.cuda.synchronize()
    ref = O.vocab_embed_bwd(ids.numpy(), dY, V) + to64(dE_in)
    assert np.max(np.abs(ref)) < 256
    assert np.array_equal(to64(dE), ref)


def test_embed_bwd_deterministic_and_zero_tokens():
    V, h, M = 4096, 1024, 2048
    ids = zipf_ids(M, V, 8)
    dY = normal_tensor((M, h), 1.0, 9)
    outs = []
    for _ in range(2):
        dE = torch.empty((V, h), dtype=torch.bfloat16, device="cuda")
        embed_bwd(cuda(ids), cuda(dY), None, dE, 8)
        outs.append(dE)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1])
    check(outs[0], O.vocab_embed_bwd(ids.numpy(), dY, V), "dE", "bf16")
    empty = torch.full((V, h), float("nan"), dtype=torch.bfloat16, device="cuda")
    embed_bwd(torch.empty(0, dtype=torch.int32, device="cuda"),
                         torch.empty(0, h, dtype=torch.bfloat16, device="cuda"), None, empty, 8)
    torch.cuda.synchronize()
    assert not empty.float().abs().sum().item()


# -------------------------------------------------------------- cross-entropy

def gpu_ce(X, E, targets, t, dloss=None, keep_logits=True, in_place=True):
    M, h = X.shape
    V = E.shape[0]
    Xd, Ed, td = cuda(X), cuda(E), cuda(targets)
    logits = torch.empty((M, V), dtype=torch.bfloat16, device="cuda") if keep_logits else None
    lse = torch.empty(M, dtype=torch.float32, device="cuda")
    loss = torch.empty(M, dtype=torch.float32, device="cuda")
    total = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = L.workspace(L.TP_OP_VOCAB_CE_FWD, M, h, V, 0, t, L.TP_BF16)
    L.tp_vocab_ce_fwd(Xd, Ed, td, logits, lse, loss, total, t, ws)
    out = {"lse": lse, "loss": loss, "total": total}
    if keep_logits:
        out["logits"] = logits.clone()
        dlogits = logits if in_place else torch.empty_like(logits)
        dX = torch.empty_like(Xd)
        dE = torch.empty_like(Ed)
        L.tp_vocab_ce_bwd(Xd, Ed, td, logits, lse, cuda(dloss), dlogits, dX, dE, t)
        out.update(dlogits=dlogits, dX=dX, dE=dE)
    torch.cuda.synchronize()
    return out


def ce_inputs(M, h, V, seed, x_std=1.0, e_std=None, ignore=()):
    e_std = e_std if e_std is not None else 2.0 / np.sqrt(h)
    X = normal_tensor((M, h), x_std, seed)
    E = normal_tensor((V, h), e_std, seed + 1)
    targets = zipf_ids(M, V, seed + 2)
    for r, v in ignore:
        targets[r] = v
    dloss = normal_tensor((M,), 1.0, seed + 3, "f32")
    return X, E, targets, dloss


def compare_ce(out, X, E, targets, dloss, t, what="", grads=True):
    fw = O.vocab_ce_fwd_parallel(X, E, targets.numpy(), t)
    check(out["lse"], fw["lse"], f"lse{what}", "bf16")
    check(out["loss"], fw["loss"], f"loss{what}", "bf16")
    assert abs(out["total"].item() - fw["total"]) <= 2e-3 * abs(fw["total"]) + 1e-3, \
        (out["total"].item(), fw["total"])
    check(out["logits"], to64(X) @ to64(E).T, f"logits{what}", "bf16")
    if "dX" in out and grads:
        bw = O.vocab_ce_bwd(X, E, targets.numpy(), dloss.numpy() if dloss is not None else
                            np.ones(X.shape[0]))
        check(out["dlogits"], bw["dlogits"], f"dlogits{what}", "bf16")
        check(out["dX"], bw["dX"], f"dX{what}", "bf16")
        check(out["dE"], bw["dE"], f"dE{what}", "bf16")


@pytest.mark.parametrize("t", [1, 4, 8])
def test_ce_small_vs_oracle(t):
    # 300 rows (ragged), h = 264 (ragged K), V = 1536: with t = 4 a shard is
    # 384 columns, 1.5 tiles of 256; rows 7 and 8 have out-of-range targets.
    M, h, V = 300, 264, 1536
    X, E, targets, dloss = ce_inputs(M, h, V, 10, ignore=((7, -1), (8, V)))
    out = gpu_ce(X, E, targets, t, dloss)
    assert out["loss"][7].item() == 0 and out["loss"][8].item() == 0
    assert not out["dlogits"][7].float().abs().sum().item()
    compare_ce(out, X, E, targets, dloss, t)


def test_ce_shard_not_multiple_of_32():
    # V / t = 200: the last 32-column chunk of every shard has 8 columns.
    M, h, V, t = 130, 128, 800, 4
    X, E, targets, dloss = ce_inputs(M, h, V, 20)
    compare_ce(gpu_ce(X, E, targets, t, None, in_place=False), X, E, targets, None, t)


def test_ce_large_logits_stay_finite():
    """Logits of magnitude ~200: exp(z) overflows fp32 (above z = 88.7)
    without the max subtraction that every chunk, shard and combination step
    applies.  The forward is compared; at this scale the bf16 rounding of a
    logit (up to 0.5) moves its softmax weight by tens of percent, so the
    gradients are only required to be finite and to sum to zero per row."""
    M, h, V, t = 256, 256, 2048, 8
    X, E, targets, dloss = ce_inputs(M, h, V, 30, x_std=1.0, e_std=4.0)
    out = gpu_ce(X, E, targets, t, None)
    assert float(to64(out["logits"]).max()) > 150.0
    compare_ce(out, X, E, targets, None, t, " (large logits)", grads=False)
    for k in ("dlogits", "dX", "dE"):
        assert torch.isfinite(out[k].float()).all(), k
    assert float(to64(out["dlogits"]).sum(axis=1).__abs__().max()) < 0.05


@pytest.mark.parametrize("tile", ["128", "192", "256", "pair"])
def test_ce_tiles_agree_bitwise(monkeypatch, tile):
    """The chunk layout is fixed (32 columns), so every tile shape gives the
    same logits, lse and loss bit for bit."""
    M, h, V, t = 384, 256, 2560, 4
    X, E, targets, dloss = ce_inputs(M, h, V, 40)
    ref = gpu_ce(X, E, targets, t, keep_logits=True)
    monkeypatch.setenv("TP_GEMM_TILE", tile)
    got = gpu_ce(X, E, targets, t, keep_logits=True)
    for k in ("logits", "lse", "loss", "total"):
        assert torch.equal(got[k], ref[k]), k
    compare_ce(got, X, E, targets, None, t, f" tile={tile}")


def test_ce_without_saved_logits():
    M, h, V, t = 200, 128, 1024, 2
    X, E, targets, _ = ce_inputs(M, h, V, 50)
    out = gpu_ce(X, E, targets, t, keep_logits=False)
    fw = O.vocab_ce_fwd_parallel(X, E, targets.numpy(), t)
    check(out["loss"], fw["loss"], "loss", "bf16")


def test_tied_embedding_and_loss_end_to_end():
    """The tied-weight path: Y = embed(ids); loss = CE(Y @ E^T, targets);
    dE = CE's dE + the embedding's scatter of dY (dY = the CE's dX)."""
    wl = Workload(60, "tied small", b=2, s=160, h=256, vocab=2048, t=4, w_std=0.1)
    d = make_vocab_inputs(wl)
    E, ids, targets = d["E"], d["ids"], d["targets"]
    Ed = cuda(E)
    Y = torch.empty((wl.M, wl.h), dtype=torch.bfloat16, device="cuda")
    L.tp_vocab_embed_fwd(cuda(ids), Ed, Y, wl.t)
    lse = torch.empty(wl.M, dtype=torch.float32, device="cuda")
    loss = torch.empty_like(lse)
    total = torch.empty(1, dtype=torch.float32, device="cuda")
    logits = torch.empty((wl.M, wl.vocab), dtype=torch.bfloat16, device="cuda")
    ws = L.workspace(L.TP_OP_VOCAB_CE_FWD, wl.M, wl.h, wl.vocab, 0, wl.t, L.TP_BF16)
    td = cuda(targets)
    L.tp_vocab_ce_fwd(Y, Ed, td, logits, lse, loss, total, wl.t, ws)
    dY = torch.empty_like(Y)
    dE = torch.empty_like(Ed)
    L.tp_vocab_ce_bwd(Y, Ed, td, logits, lse, None, logits, dY, dE, wl.t)
    embed_bwd(cuda(ids), dY, dE, dE, wl.t)
    torch.cuda.synchronize()
    Y64 = O.vocab_embed_fwd(ids.numpy(), E)
    assert np.array_equal(to64(Y), Y64)
    fw = O.vocab_ce_fwd_parallel(Y64, E, targets.numpy(), wl.t)
    bw = O.vocab_ce_bwd(Y64, E, targets.numpy(), np.ones(wl.M))
    check(loss, fw["loss"], "loss", "bf16")
    # total gradient of E: through the output layer and through the lookup
    dE_ref = bw["dE"] + O.vocab_embed_bwd(ids.numpy(), bw["dX"], wl.vocab)
    check(dE, dE_ref, "dE (tied)", "bf16")


def test_vocab_full_size_sampled():
    """The 175B-shaped vocabulary workload (M = 2048, h = 12288, V = 51200,
    t = 8) at full size, as the bench runs it.  The embedding is exact on
    every row; the loss, lse and dX rows are exact per row, so sampled rows
    of the oracle are exact references; dE needs every token, so the oracle
    runs on all 2048 tokens and sampled rows of dE are compared."""
    wl = WORKLOADS[6]
    d = make_vocab_inputs(wl)
    E, X, ids, targets = d["E"], d["X"], d["ids"], d["targets"]
    Ed = cuda(E)
    Y = torch.empty((wl.M, wl.h), dtype=torch.bfloat16, device="cuda")
    L.tp_vocab_embed_fwd(cuda(ids), Ed, Y, wl.t)
    out = gpu_ce(X, E, targets, wl.t)
    E64, X64, tg = to64(E), to64(X), targets.numpy()
    assert np.array_equal(to64(Y), O.vocab_embed_fwd(ids.numpy(), E64))
    rng = np.random.default_rng(6)
    rows = np.unique(np.r_[0, wl.M - 1, rng.integers(0, wl.M, 10)])
    r_t = torch.as_tensor(rows, device="cuda")
    fw = O.vocab_ce_fwd_parallel(X64[rows], E64, tg[rows], wl.t)
    check(out["loss"][r_t], fw["loss"], "loss rows", "bf16")
    check(out["lse"][r_t], fw["lse"], "lse rows", "bf16")
    bw_rows = O.vocab_ce_bwd(X64[rows], E64, tg[rows], np.ones(len(rows)))
    check(out["dX"][r_t], bw_rows["dX"], "dX rows", "bf16")
    check(out["dlogits"][r_t], bw_rows["dlogits"], "dlogits rows", "bf16")
    vocab_rows = np.unique(np.r_[0, wl.vocab - 1, tg[:64], rng.integers(0, wl.vocab, 16)])
    bw = O.vocab_ce_bwd(X64, E64, tg, np.ones(wl.M))
    v_t = torch.as_tensor(vocab_rows, device="cuda")
    check(out["dE"][v_t], bw["dE"][vocab_rows], "dE rows", "bf16")
