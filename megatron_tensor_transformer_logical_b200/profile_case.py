"""Runs one libtp operation at a chosen shape a few times, for profilers.

    python -m megatron_tensor_transformer_logical_b200.profile_case CASE [--iters N]

Cases (175B-shaped layer unless noted; bf16, t = 8):
  mlp_g1      tp_linear_col  X[2048,12288] @ A[12288,49152]      (column split)
  mlp_g2      tp_linear_row  H[2048,49152] @ B[49152,12288]      (row split, sum in TMEM)
  mlp_fwd     tp_mlp_fwd     (two GEMMs)
  mlp_bwd     tp_mlp_bwd     (dgrad+GeLU', two wgrads, dgrad)
  attn_fwd    tp_attn_fwd    (QKV GEMM, attention core, Wo GEMM)
  attn_bwd    tp_attn_bwd
  small_gemm  tp_linear_col  X[1024,4096] @ W[4096,8192] (a quick case)
  block       tp_block_fwd + tp_block_bwd: LayerNorm + residual around the attention
              and the MLP of the 175B-shaped layer (gamma 1, beta 0)
  vocab_step  the tied vocabulary-parallel embedding + cross-entropy, forward and
              backward on the seeded vocabulary workload (M=2048, h=12288,
              V=51200, t=8, Zipf token ids): embedding gather, logits
              GEMM with the loss epilogue, loss combination, softmax gradient,
              dX and dE GEMMs, embedding scatter-add
  layernorm   tp_layernorm_fwd + tp_layernorm_bwd on X[8192,12288] (201 MB, larger
              than L2), gamma and beta, with a residual gradient
  mlp_bwd_bias tp_mlp_bwd with both bias gradients, M=8192, h=12288, f=1024, t=8:
              dbB = colsum(dZ [8192,12288], 201 MB) and dbA from the GeLU' epilogue's
              partials, both in one launch (mlp_bias_grads)
  mlp_small   tp_mlp_fwd + tp_mlp_bwd with biases at the GPT-2-small shape: M=8192,
              h=768, f=3072, t=4 (K = 768 and 3072 GEMMs bound by their epilogues and
              by L2 traffic; about 0.2 GB on the device)
  attn_bwd_big tp_attn_bwd at b=2, s=4096, h=6144 (48 heads; about 2.7 GB on the
              device): the D = rowsum(dO * O) kernel reads 2 x 100 MB
  linear_f32  tp_linear_col in fp32, X[4096,4096] @ W[4096,4096] (the CUDA-core path)
  mlp_bwd_quarter tp_mlp_bwd with f = 12288 (a quarter of the layer's width; about 2 GB on
              the device): the four backward GEMMs with the 175B-shaped M and h
  attn_small  tp_attn_fwd + tp_attn_bwd on two head groups of the 175B-shaped layer:
              b=1, s=2048, h=3072 (24 heads of 128, 192 forward CTAs, more than one
              per SM), t=2, causal (a small case for full ncu captures of the
              attention kernels)

Inputs are seeded N(0,1) / N(0, 0.006^2) tensors made on the device; nothing
is checked here (the tests do that).  Prints the mean device time per call.
"""
from __future__ import annotations

import argparse

import torch

from . import binding as L


def _t(shape, std, dtype=torch.bfloat16, seed=0):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return (torch.randn(*shape, generator=g, device="cuda") * std).to(dtype)


def make_case(name: str):
    M, h, f, heads, t = 2048, 12288, 49152, 96, 8
    bf = torch.bfloat16
    if name == "small_gemm":
        X, W = _t((1024, 4096), 1.0), _t((4096, 8192), 0.02, seed=1)
        Y = torch.empty(1024, 8192, dtype=bf, device="cuda")
        return lambda: L.tp_linear_col(X, W, None, Y, t)
    if name == "mlp_g1":
        X, A = _t((M, h), 1.0), _t((h, f), 0.006, seed=1)
        Y = torch.empty(M, f, dtype=bf, device="cuda")
        return lambda: L.tp_linear_col(X, A, None, Y, t)
    if name == "mlp_g2":
        H, B = _t((M, f), 0.5), _t((f, h), 0.006, seed=1)
        Z = torch.empty(M, h, dtype=bf, device="cuda")
        return lambda: L.tp_linear_row(H, B, None, Z, t)
    if name in ("mlp_fwd", "mlp_bwd"):
        X, A, B = _t((M, h), 1.0), _t((h, f), 0.006, seed=1), _t((f, h), 0.006, seed=2)
        dZ = _t((M, h), 1.0, seed=3)
        Z, Y = torch.empty(M, h, dtype=bf, device="cuda"), torch.empty(M, f, dtype=bf, device="cuda")
        wsf = L.workspace(L.TP_OP_MLP_FWD, M, h, f, 0, t, L.TP_BF16)
        L.tp_mlp_fwd(X, A, None, B, None, Z, Y, t, wsf)
        if name == "mlp_fwd":
            return lambda: L.tp_mlp_fwd(X, A, None, B, None, Z, Y, t, wsf)
        dX, dA, dB = torch.empty_like(X), torch.empty_like(A), torch.empty_like(B)
        wsb = L.workspace(L.TP_OP_MLP_BWD, M, h, f, 0, t, L.TP_BF16)
        return lambda: L.tp_mlp_bwd(X, A, None, B, Y, dZ, dX, dA, None, dB, None, t, wsb)
    if name in ("attn_fwd", "attn_bwd"):
        X, Wqkv, Wo = _t((M, h), 1.0), _t((h, 3 * h), 0.006, seed=1), _t((h, h), 0.006, seed=2)
        dZ = _t((M, h), 1.0, seed=3)
        Z = torch.empty(M, h, dtype=bf, device="cuda")
        QKV = torch.empty(M, 3 * h, dtype=torch.float16, device="cuda")
        O = torch.empty(M, h, dtype=bf, device="cuda")
        LSE = torch.empty(1, heads, M, dtype=torch.float32, device="cuda")
        wsf = L.workspace(L.TP_OP_ATTN_FWD, M, h, 0, heads, t, L.TP_BF16)
        fwd = lambda: L.tp_attn_fwd(X, Wqkv, Wo, Z, QKV, O, LSE, 1, M, heads, t, True, wsf)
        fwd()
        if name == "attn_fwd":
            return fwd
        dX, dWqkv, dWo = torch.empty_like(X), torch.empty_like(Wqkv), torch.empty_like(Wo)
        wsb = L.workspace(L.TP_OP_ATTN_BWD, M, h, 0, heads, t, L.TP_BF16)
        return lambda: L.tp_attn_bwd(X, Wqkv, Wo, QKV, O, LSE, dZ, dX, dWqkv, dWo, 1, M, heads, t,
                                     True, wsb)
    if name == "block":
        X, dX2 = _t((M, h), 1.0), _t((M, h), 1.0, seed=4)
        ones, zeros = torch.ones(h, dtype=bf, device="cuda"), torch.zeros(h, dtype=bf, device="cuda")
        w = {"ln1_g": ones, "ln1_b": zeros, "Wqkv": _t((h, 3 * h), 0.006, seed=1),
             "Wo": _t((h, h), 0.006, seed=2), "ln2_g": ones, "ln2_b": zeros,
             "A": _t((h, f), 0.006, seed=5), "B": _t((f, h), 0.006, seed=6)}
        e = lambda *sh, dt=bf: torch.empty(*sh, dtype=dt, device="cuda")
        f32 = torch.float32
        sv = {"Xn1": e(M, h), "mean1": e(M, dt=f32), "rstd1": e(M, dt=f32),
              "QKV": e(M, 3 * h, dt=torch.float16), "O": e(M, h), "LSE": e(1, heads, M, dt=f32),
              "X1": e(M, h), "Xn2": e(M, h), "mean2": e(M, dt=f32), "rstd2": e(M, dt=f32),
              "Y": e(M, f)}
        g = {"dln1_g": e(h), "dln1_b": e(h), "dWqkv": e(h, 3 * h), "dWo": e(h, h),
             "dln2_g": e(h), "dln2_b": e(h), "dA": e(h, f), "dB": e(f, h)}
        X2, dX = e(M, h), e(M, h)
        wsf = L.workspace(L.TP_OP_BLOCK_FWD, M, h, f, heads, t, L.TP_BF16)
        wsb = L.workspace(L.TP_OP_BLOCK_BWD, M, h, f, heads, t, L.TP_BF16)

        def block():
            L.tp_block_fwd(X, w, X2, sv, 1, M, f, heads, t, 1e-5, wsf)
            L.tp_block_bwd(X, w, sv, dX2, dX, g, 1, M, f, heads, t, 1e-5, wsb)
        return block
    if name == "vocab_step":
        from .inputs import WORKLOADS, make_vocab_inputs
        wl = WORKLOADS[6]
        V = wl.vocab
        d = {k: v.to("cuda") for k, v in make_vocab_inputs(wl).items()}
        ids, targets, E, X, dY = d["ids"], d["targets"], d["E"], d["X"], d["dY"]
        Y, dX = torch.empty(M, h, dtype=bf, device="cuda"), torch.empty(M, h, dtype=bf, device="cuda")
        logits = torch.empty(M, V, dtype=bf, device="cuda")
        lse, loss = (torch.empty(M, dtype=torch.float32, device="cuda") for _ in range(2))
        total = torch.empty(1, dtype=torch.float32, device="cuda")
        dE = torch.empty_like(E)
        wsc = L.workspace(L.TP_OP_VOCAB_CE_FWD, M, h, V, 0, t, L.TP_BF16)
        wse = L.workspace(L.TP_OP_VOCAB_EMBED_BWD, M, h, V, 0, t, L.TP_BF16)

        def step():
            L.tp_vocab_embed_fwd(ids, E, Y, t)
            L.tp_vocab_ce_fwd(X, E, targets, logits, lse, loss, total, t, wsc)
            L.tp_vocab_ce_bwd(X, E, targets, logits, lse, None, logits, dX, dE, t)
            L.tp_vocab_embed_bwd(ids, dY, dE, dE, t, wse)
        return step
    if name == "layernorm":
        Mb = 8192
        X, dY, dR = _t((Mb, h), 1.0), _t((Mb, h), 1.0, seed=1), _t((Mb, h), 1.0, seed=2)
        g, b = 1.0 + _t((h,), 0.1, seed=3), _t((h,), 0.1, seed=4)
        Y, dX = torch.empty_like(X), torch.empty_like(X)
        mean = torch.empty(Mb, dtype=torch.float32, device="cuda")
        rstd = torch.empty_like(mean)
        dg, db = torch.empty_like(g), torch.empty_like(b)
        ws = L.workspace(L.TP_OP_LN_BWD, Mb, h, 0, 0, 1, L.TP_BF16)

        def ln():
            L.tp_layernorm_fwd(X, g, b, Y, mean, rstd, 1e-5)
            L.tp_layernorm_bwd(X, g, mean, rstd, dY, dR, dX, dg, db, ws)
        return ln
    if name == "mlp_bwd_bias":
        Mb, fb = 8192, 1024
        X, A, B = _t((Mb, h), 1.0), _t((h, fb), 0.006, seed=1), _t((fb, h), 0.006, seed=2)
        bA, bB = _t((fb,), 0.01, seed=5), _t((h,), 0.01, seed=6)
        dZ = _t((Mb, h), 1.0, seed=3)
        Z, Y = torch.empty(Mb, h, dtype=bf, device="cuda"), torch.empty(Mb, fb, dtype=bf, device="cuda")
        L.tp_mlp_fwd(X, A, bA, B, bB, Z, Y, t, L.workspace(L.TP_OP_MLP_FWD, Mb, h, fb, 0, t, L.TP_BF16))
        dX, dA, dB = torch.empty_like(X), torch.empty_like(A), torch.empty_like(B)
        dbA, dbB = torch.empty_like(bA), torch.empty_like(bB)
        wsb = L.workspace(L.TP_OP_MLP_BWD, Mb, h, fb, 0, t, L.TP_BF16)
        return lambda: L.tp_mlp_bwd(X, A, bA, B, Y, dZ, dX, dA, dbA, dB, dbB, t, wsb)
    if name == "mlp_small":
        Ms, hs, fs, ts = 8192, 768, 3072, 4
        X, A, B = _t((Ms, hs), 1.0), _t((hs, fs), 0.02, seed=1), _t((fs, hs), 0.02, seed=2)
        bA, bB = _t((fs,), 0.01, seed=5), _t((hs,), 0.01, seed=6)
        dZ = _t((Ms, hs), 1.0, seed=3)
        Z, Y = torch.empty(Ms, hs, dtype=bf, device="cuda"), torch.empty(Ms, fs, dtype=bf, device="cuda")
        dX, dA, dB = torch.empty_like(X), torch.empty_like(A), torch.empty_like(B)
        dbA, dbB = torch.empty_like(bA), torch.empty_like(bB)
        wsf = L.workspace(L.TP_OP_MLP_FWD, Ms, hs, fs, 0, ts, L.TP_BF16)
        wsb = L.workspace(L.TP_OP_MLP_BWD, Ms, hs, fs, 0, ts, L.TP_BF16)

        def mlp_small():
            L.tp_mlp_fwd(X, A, bA, B, bB, Z, Y, ts, wsf)
            L.tp_mlp_bwd(X, A, bA, B, Y, dZ, dX, dA, dbA, dB, dbB, ts, wsb)
        return mlp_small
    if name == "attn_bwd_big":
        b2, s2 = 2, 4096
        Mb = b2 * s2
        h, heads = 6144, 48
        X, Wqkv, Wo = _t((Mb, h), 1.0), _t((h, 3 * h), 0.006, seed=1), _t((h, h), 0.006, seed=2)
        dZ = _t((Mb, h), 1.0, seed=3)
        Z = torch.empty(Mb, h, dtype=bf, device="cuda")
        QKV = torch.empty(Mb, 3 * h, dtype=torch.float16, device="cuda")
        O = torch.empty(Mb, h, dtype=bf, device="cuda")
        LSE = torch.empty(b2, heads, s2, dtype=torch.float32, device="cuda")
        L.tp_attn_fwd(X, Wqkv, Wo, Z, QKV, O, LSE, b2, s2, heads, t, True,
                      L.workspace(L.TP_OP_ATTN_FWD, Mb, h, 0, heads, t, L.TP_BF16))
        dX, dWqkv, dWo = torch.empty_like(X), torch.empty_like(Wqkv), torch.empty_like(Wo)
        wsb = L.workspace(L.TP_OP_ATTN_BWD, Mb, h, 0, heads, t, L.TP_BF16)
        return lambda: L.tp_attn_bwd(X, Wqkv, Wo, QKV, O, LSE, dZ, dX, dWqkv, dWo, b2, s2, heads,
                                     t, True, wsb)
    if name == "mlp_bwd_quarter":
        fq = 12288
        X, A, B = _t((M, h), 1.0), _t((h, fq), 0.006, seed=1), _t((fq, h), 0.006, seed=2)
        dZ = _t((M, h), 1.0, seed=3)
        Z, Y = torch.empty(M, h, dtype=bf, device="cuda"), torch.empty(M, fq, dtype=bf, device="cuda")
        L.tp_mlp_fwd(X, A, None, B, None, Z, Y, t, L.workspace(L.TP_OP_MLP_FWD, M, h, fq, 0, t, L.TP_BF16))
        dX, dA, dB = torch.empty_like(X), torch.empty_like(A), torch.empty_like(B)
        wsb = L.workspace(L.TP_OP_MLP_BWD, M, h, fq, 0, t, L.TP_BF16)
        return lambda: L.tp_mlp_bwd(X, A, None, B, Y, dZ, dX, dA, None, dB, None, t, wsb)
    if name == "attn_small":
        hs, hd = 3072, 24
        X, Wqkv, Wo = _t((M, hs), 1.0), _t((hs, 3 * hs), 0.02, seed=1), _t((hs, hs), 0.02, seed=2)
        dZ = _t((M, hs), 1.0, seed=3)
        Z = torch.empty(M, hs, dtype=bf, device="cuda")
        QKV = torch.empty(M, 3 * hs, dtype=torch.float16, device="cuda")
        O = torch.empty(M, hs, dtype=bf, device="cuda")
        LSE = torch.empty(1, hd, M, dtype=torch.float32, device="cuda")
        dX, dWqkv, dWo = torch.empty_like(X), torch.empty_like(Wqkv), torch.empty_like(Wo)
        wsf = L.workspace(L.TP_OP_ATTN_FWD, M, hs, 0, hd, 2, L.TP_BF16)
        wsb = L.workspace(L.TP_OP_ATTN_BWD, M, hs, 0, hd, 2, L.TP_BF16)

        def small():
            L.tp_attn_fwd(X, Wqkv, Wo, Z, QKV, O, LSE, 1, M, hd, 2, True, wsf)
            L.tp_attn_bwd(X, Wqkv, Wo, QKV, O, LSE, dZ, dX, dWqkv, dWo, 1, M, hd, 2, True, wsb)
        return small
    if name == "linear_f32":
        X, W = _t((4096, 4096), 1.0, torch.float32), _t((4096, 4096), 0.02, torch.float32, seed=1)
        Y = torch.empty(4096, 4096, dtype=torch.float32, device="cuda")
        return lambda: L.tp_linear_col(X, W, None, Y, 2)
    raise SystemExit(f"unknown case {name}")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case")
    ap.add_argument("--iters", type=int, default=3)
    a = ap.parse_args()
    fn = make_case(a.case)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.iters):
        fn()
    e1.record()
    torch.cuda.synchronize()
    L.tp_device_status()
    print(f"{a.case}: {e0.elapsed_time(e1) / a.iters:.3f} ms per call")


if __name__ == "__main__":
    main()
