"""CPU oracle for the Megatron-style partitioned Transformer layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` use it.  It shares no code
with the CUDA path (no kernels, headers, helpers or tables); the only thing
both sides consume is the seeded input generator module, which holds no
arithmetic of the method.

Everything here is plain fp64 numpy: a matrix product (``@``) is used as a
library primitive, ``scipy.special.erf`` gives the error function, and the
softmax is written out with its max subtraction.  No blocking, fusion or
reordering is done beyond what the definitions below state, so each
function can be checked against its page by eye.

Sources (page title, then section):

* [P3] "图解Transformer并行计算：从矩阵乘法切分到Megatron架构设计"
  - §1.1 row-wise partition: ``W = [W_0; ...; W_{t-1}]`` split on its input
    rows, ``X`` split on its last dim, ``Y = sum_i X_i @ W_i`` (AllReduce).
  - §1.2 column-wise partition: ``W = [W_0 | ... | W_{t-1}]`` split on its
    output columns, ``X`` kept whole, ``Y = concat_i X @ W_i`` (All-Gather).
  - §2.1 MLP ``Z = GeLU(X @ A) @ B`` with ``A`` split by columns and ``B``
    by rows; GeLU is taken on each shard with no exchange; ``Z = sum_i Z_i``.
  - §2.2 backward is the mirror: the weight gradients of each shard are
    computed locally, and the input-gradient partials are summed.
  - §3.1 per-head attention ``softmax(Q K^T / sqrt(d_k)) V``.
  - §3.2 Wq, Wk, Wv split by columns in head groups, ``W_o`` split by rows,
    ``Z = sum_g O_g @ Wo_g``; backward mirrors it.
* [P2] the PyTorch tensor-parallel tutorial (page title "企业官网建设流程全解析"):
  §3.3 uses ``nn.GELU()`` between the two linears (the exact erf form) and
  builds the block as x + attention(LayerNorm(x)), then x + mlp(LayerNorm(x)).
* [P4] "5.1 Tensor并行与算子拆分": ``tensor_parallel_split`` raises on a
  dimension that the partition count does not divide; the attention listing
  uses ``masked_fill(mask == 0, -inf)`` and ``1/sqrt(d_k)`` scaling.

Readings where the pages are silent (each also listed in the design notes):

* GeLU is the exact erf form (the tanh approximation is not used).
* The row-parallel bias is added once, after the sum over shards; the
  column-parallel bias is sliced with its columns.
* ``Wqkv = [Wq | Wk | Wv]`` along columns; head ``j`` owns columns
  ``[j*d, (j+1)*d)`` inside each of the three blocks; head group ``g`` owns
  heads ``[g*H/t, (g+1)*H/t)``.
* The causal mask hides key ``c`` from query ``r`` when ``c > r``.
* The saved log-sum-exp is the natural log of the softmax denominator of
  the scaled, masked scores.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(exact integer arithmetic, brute-force loops, closed forms, finite
differences); none is "parity unpinned".
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional

import numpy as np
from scipy.special import erf as _erf

__all__ = [
    "gelu", "gelu_prime", "split_cols", "split_rows", "linear",
    "linear_col_parallel", "linear_row_parallel", "mlp_fwd", "mlp_fwd_parallel",
    "mlp_bwd", "mlp_bwd_parallel", "head_columns", "group_columns",
    "attention_core", "attention_core_bwd", "attn_fwd", "attn_fwd_parallel",
    "attn_bwd", "attn_bwd_parallel", "layernorm_fwd", "layernorm_bwd", "block_fwd",
    "block_bwd", "vocab_embed_fwd", "vocab_embed_fwd_parallel", "vocab_embed_bwd",
    "vocab_ce_fwd", "vocab_ce_fwd_parallel", "vocab_ce_bwd", "max_rel_error", "normwise_error",
]

_SQRT2 = math.sqrt(2.0)
_INV_SQRT_2PI = 1.0 / math.sqrt(2.0 * math.pi)


def _f64(a) -> Optional[np.ndarray]:
    if a is None:
        return None
    if hasattr(a, "detach"):  # a torch tensor: widen exactly through fp32/fp64
        a = a.detach().cpu()
        if str(a.dtype) in ("torch.bfloat16", "torch.float16"):
            a = a.float()
        a = a.double().numpy()
    return np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------------------
# GeLU ([P2] §3.3 nn.GELU, exact form; [P3] §2.1 step 2)
# ---------------------------------------------------------------------------

def gelu(x):
    """GeLU(x) = x * Phi(x) = 0.5 * x * (1 + erf(x / sqrt(2)))."""
    x = _f64(x)
    return 0.5 * x * (1.0 + _erf(x / _SQRT2))


def gelu_prime(x):
    """d/dx GeLU(x) = Phi(x) + x * phi(x), phi(x) = exp(-x^2/2) / sqrt(2 pi)."""
    x = _f64(x)
    return 0.5 * (1.0 + _erf(x / _SQRT2)) + x * _INV_SQRT_2PI * np.exp(-0.5 * x * x)


# ---------------------------------------------------------------------------
# Partitioning ([P4] §1.1 tensor_parallel_split; [P3] §1.1, §1.2)
# ---------------------------------------------------------------------------

def _check_divisible(n: int, t: int, what: str) -> int:
    if t <= 0 or n % t != 0:
        raise ValueError(f"{what} size {n} must be divisible by {t}")
    return n // t


def split_cols(W, t: int) -> List[np.ndarray]:
    """Column shards W_i = W[:, i*n/t : (i+1)*n/t] (contiguous, equal)."""
    W = _f64(W)
    c = _check_divisible(W.shape[-1], t, "column")
    return [W[..., i * c:(i + 1) * c] for i in range(t)]


def split_rows(W, t: int) -> List[np.ndarray]:
    """Row shards W_i = W[i*k/t : (i+1)*k/t, :] (contiguous, equal)."""
    W = _f64(W)
    r = _check_divisible(W.shape[0], t, "row")
    return [W[i * r:(i + 1) * r] for i in range(t)]


# ---------------------------------------------------------------------------
# Linear layers ([P3] §1.1, §1.2)
# ---------------------------------------------------------------------------

def linear(X, W, bias=None):
    """Unpartitioned Y = X @ W (+ bias).  X [M,K], W [K,N] (weights [in, out])."""
    Y = _f64(X) @ _f64(W)
    if bias is not None:
        Y = Y + _f64(bias)
    return Y


def linear_col_parallel(X, W, bias, t: int):
    """Column-split linear ([P3] §1.2): Y = concat_i (X @ W_i + b_i)."""
    X = _f64(X)
    Ws = split_cols(W, t)
    bs = split_cols(bias, t) if bias is not None else [None] * t
    parts = [X @ Wi + (bi if bi is not None else 0.0) for Wi, bi in zip(Ws, bs)]
    return np.concatenate(parts, axis=-1)


def linear_row_parallel(X, W, bias, t: int, return_partials: bool = False):
    """Row-split linear ([P3] §1.1): X split on its last dim, Z = sum_i X_i @ W_i.

    The bias is added once, after the sum (adding it in every shard would
    add it t times).  With ``return_partials`` the list of Z_i is returned
    as well.
    """
    Xs = split_cols(X, t)
    Ws = split_rows(W, t)
    partials = [Xi @ Wi for Xi, Wi in zip(Xs, Ws)]
    Z = partials[0].copy()
    for p in partials[1:]:
        Z = Z + p
    if bias is not None:
        Z = Z + _f64(bias)
    return (Z, partials) if return_partials else Z


# ---------------------------------------------------------------------------
# MLP ([P3] §2.1 forward, §2.2 backward)
# ---------------------------------------------------------------------------

def mlp_fwd(X, A, bA, B, bB) -> Dict[str, np.ndarray]:
    """Unpartitioned MLP: Y = X@A + bA, H = GeLU(Y), Z = H@B + bB."""
    Y = linear(X, A, bA)
    H = gelu(Y)
    Z = linear(H, B, bB)
    return {"Y": Y, "H": H, "Z": Z}


def mlp_fwd_parallel(X, A, bA, B, bB, t: int) -> Dict[str, np.ndarray]:
    """The pages' partitioned MLP ([P3] §2.1 steps, §2.2 MLP_forward_TP).

    Shard i: Y_i = X @ A_i + bA_i; H_i = GeLU(Y_i) locally; Z_i = H_i @ B_i.
    Then Z = sum_i Z_i (the AllReduce), plus bB once.
    """
    X = _f64(X)
    As, Bs = split_cols(A, t), split_rows(B, t)
    bAs = split_cols(bA, t) if bA is not None else [None] * t
    Ys, Hs, Zs = [], [], []
    for Ai, bAi, Bi in zip(As, bAs, Bs):
        Yi = X @ Ai + (bAi if bAi is not None else 0.0)
        Hi = gelu(Yi)
        Ys.append(Yi)
        Hs.append(Hi)
        Zs.append(Hi @ Bi)
    Z = Zs[0].copy()
    for Zi in Zs[1:]:
        Z = Z + Zi
    if bB is not None:
        Z = Z + _f64(bB)
    return {"Y": np.concatenate(Ys, -1), "H": np.concatenate(Hs, -1), "Z": Z,
            "Z_partials": Zs}


def mlp_bwd(X, A, bA, B, dZ, Y=None) -> Dict[str, np.ndarray]:
    """Unpartitioned MLP backward by the chain rule.

    dH = dZ @ B^T; dY = dH * GeLU'(Y); dB = H^T @ dZ; dbB = colsum(dZ);
    dA = X^T @ dY; dbA = colsum(dY); dX = dY @ A^T.
    ``Y`` (the pre-activation) is recomputed when not given.
    """
    X, A, B, dZ = _f64(X), _f64(A), _f64(B), _f64(dZ)
    if Y is None:
        Y = linear(X, A, bA)
    Y = _f64(Y)
    H = gelu(Y)
    dH = dZ @ B.T
    dY = dH * gelu_prime(Y)
    return {
        "dX": dY @ A.T,
        "dA": X.T @ dY,
        "dbA": dY.sum(axis=0),
        "dB": H.T @ dZ,
        "dbB": dZ.sum(axis=0),
        "dY": dY,
    }


def mlp_bwd_parallel(X, A, bA, B, dZ, t: int) -> Dict[str, np.ndarray]:
    """The pages' mirror rule ([P3] §2.2 backward paragraph).

    dZ goes to every shard; shard i computes its own dB_i = H_i^T dZ and
    dA_i = X^T dY_i (no exchange) and a partial dX_i = dY_i @ A_i^T; the
    partials are summed (the backward AllReduce).
    """
    X, dZ = _f64(X), _f64(dZ)
    As, Bs = split_cols(A, t), split_rows(B, t)
    bAs = split_cols(bA, t) if bA is not None else [None] * t
    dA, dbA, dB, dXs = [], [], [], []
    for Ai, bAi, Bi in zip(As, bAs, Bs):
        Yi = X @ Ai + (bAi if bAi is not None else 0.0)
        Hi = gelu(Yi)
        dYi = (dZ @ Bi.T) * gelu_prime(Yi)
        dB.append(Hi.T @ dZ)
        dA.append(X.T @ dYi)
        dbA.append(dYi.sum(axis=0))
        dXs.append(dYi @ Ai.T)
    dX = dXs[0].copy()
    for p in dXs[1:]:
        dX = dX + p
    return {"dX": dX, "dA": np.concatenate(dA, -1), "dbA": np.concatenate(dbA),
            "dB": np.concatenate(dB, 0), "dbB": dZ.sum(axis=0), "dX_partials": dXs}


# ---------------------------------------------------------------------------
# Attention ([P3] §3.1, §3.2; [P4] attention listing for mask and scale)
# ---------------------------------------------------------------------------

def head_columns(h: int, heads: int, j: int) -> Dict[str, np.ndarray]:
    """Columns of head j in QKV = X @ Wqkv, Wqkv = [Wq | Wk | Wv] ([h, 3h])."""
    d = h // heads
    base = np.arange(j * d, (j + 1) * d)
    return {"q": base, "k": h + base, "v": 2 * h + base}


def group_columns(h: int, heads: int, t: int, g: int) -> np.ndarray:
    """Wqkv columns owned by head group g: its heads' q, then k, then v columns."""
    hg = _check_divisible(heads, t, "heads")
    js = range(g * hg, (g + 1) * hg)
    q = np.concatenate([head_columns(h, heads, j)["q"] for j in js])
    k = np.concatenate([head_columns(h, heads, j)["k"] for j in js])
    v = np.concatenate([head_columns(h, heads, j)["v"] for j in js])
    return np.concatenate([q, k, v])


def _masked_scores(Q, K, causal: bool):
    s_q, d = Q.shape
    S = (Q @ K.T) / math.sqrt(d)
    if causal:
        r = np.arange(s_q)[:, None]
        c = np.arange(K.shape[0])[None, :]
        S = np.where(c > r, -np.inf, S)
    return S


def attention_core(Q, K, V, causal: bool = True):
    """One head ([P3] §3.1): P = softmax(Q K^T / sqrt(d)) (masked), O = P V.

    Returns (O, P, lse) with lse the natural log of each row's softmax
    denominator of the scaled, masked scores.
    """
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    S = _masked_scores(Q, K, causal)
    m = S.max(axis=1, keepdims=True)
    E = np.exp(S - m)
    den = E.sum(axis=1, keepdims=True)
    P = E / den
    lse = (m + np.log(den))[:, 0]
    return P @ V, P, lse


def attention_core_bwd(Q, K, V, dO, causal: bool = True):
    """Backward of one head through the softmax Jacobian.

    dV = P^T dO; dP = dO V^T; dS = P * (dP - rowsum(dP * P));
    dQ = dS K / sqrt(d); dK = dS^T Q / sqrt(d).
    """
    Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
    _, P, _ = attention_core(Q, K, V, causal)
    d = Q.shape[1]
    dV = P.T @ dO
    dP = dO @ V.T
    dS = P * (dP - (dP * P).sum(axis=1, keepdims=True))
    dQ = dS @ K / math.sqrt(d)
    dK = dS.T @ Q / math.sqrt(d)
    return dQ, dK, dV


def _attn_dims(X, Wqkv, heads: int, b: int, s: int):
    """Returns (hi, d): the attention width hi = Wqkv columns / 3 (h for the
    whole layer; a head group's or one head's width for a slice of Wqkv) and
    the head dimension d = hi / heads."""
    if Wqkv.shape[1] % 3 != 0:
        raise ValueError("Wqkv must have 3 * width columns")
    hi = Wqkv.shape[1] // 3
    if hi % heads != 0:
        raise ValueError("hidden size must be divisible by the number of heads")
    if X.shape != (b * s, Wqkv.shape[0]):
        raise ValueError(f"X must be [b*s, h] = [{b * s}, {Wqkv.shape[0]}], got {X.shape}")
    return hi, hi // heads


def attn_fwd(X, Wqkv, Wo, b: int, s: int, heads: int, causal: bool = True):
    """Unpartitioned multi-head attention.

    QKV = X @ Wqkv; per batch element and head j, O_j = attention_core of
    (Q_j, K_j, V_j); the heads are concatenated in column order to O [M, h];
    Z = O @ Wo.  Returns QKV, O, LSE [b, heads, s] and Z.  Given the column
    slice of Wqkv of some heads and the matching rows of Wo (as one head
    group holds them, [P3] §3.2), it computes exactly those heads.
    """
    X, Wqkv, Wo = _f64(X), _f64(Wqkv), _f64(Wo)
    h, d = _attn_dims(X, Wqkv, heads, b, s)
    QKV = X @ Wqkv
    O = np.zeros((b * s, h))
    LSE = np.zeros((b, heads, s))
    for bi in range(b):
        rows = slice(bi * s, (bi + 1) * s)
        for j in range(heads):
            c = head_columns(h, heads, j)
            Oj, _, lse = attention_core(QKV[rows][:, c["q"]], QKV[rows][:, c["k"]],
                                        QKV[rows][:, c["v"]], causal)
            O[rows, j * d:(j + 1) * d] = Oj
            LSE[bi, j] = lse
    return {"QKV": QKV, "O": O, "LSE": LSE, "Z": O @ Wo}


def attn_fwd_parallel(X, Wqkv, Wo, b: int, s: int, heads: int, t: int, causal: bool = True):
    """The pages' head-wise partitioned attention ([P3] §3.2 forward steps 1-3).

    Group g takes Wqkv's columns of its heads (q, k and v), computes its
    heads' attention locally and Z_g = O_g @ Wo_g with Wo_g the rows of
    Wo that match its heads; Z = sum_g Z_g.
    """
    X, Wqkv, Wo = _f64(X), _f64(Wqkv), _f64(Wo)
    h, d = _attn_dims(X, Wqkv, heads, b, s)
    hg = _check_divisible(heads, t, "heads")
    Zs = []
    for g in range(t):
        cols = group_columns(h, heads, t, g)
        QKVg = X @ Wqkv[:, cols]
        w = hg * d
        Og = np.zeros((b * s, w))
        for bi in range(b):
            rows = slice(bi * s, (bi + 1) * s)
            for jl in range(hg):
                q = QKVg[rows, jl * d:(jl + 1) * d]
                k = QKVg[rows, w + jl * d:w + (jl + 1) * d]
                v = QKVg[rows, 2 * w + jl * d:2 * w + (jl + 1) * d]
                Og[rows, jl * d:(jl + 1) * d] = attention_core(q, k, v, causal)[0]
        Zs.append(Og @ Wo[g * w:(g + 1) * w])
    Z = Zs[0].copy()
    for Zg in Zs[1:]:
        Z = Z + Zg
    return {"Z": Z, "Z_partials": Zs}


def attn_bwd(X, Wqkv, Wo, dZ, b: int, s: int, heads: int, causal: bool = True):
    """Unpartitioned attention backward.

    dO = dZ @ Wo^T; dWo = O^T @ dZ; per head the core backward gives
    dQ_j, dK_j, dV_j, written to the matching columns of dQKV [M, 3h];
    dWqkv = X^T @ dQKV; dX = dQKV @ Wqkv^T.
    """
    X, Wqkv, Wo, dZ = _f64(X), _f64(Wqkv), _f64(Wo), _f64(dZ)
    h, d = _attn_dims(X, Wqkv, heads, b, s)
    fw = attn_fwd(X, Wqkv, Wo, b, s, heads, causal)
    QKV, O = fw["QKV"], fw["O"]
    dO = dZ @ Wo.T
    dQKV = np.zeros_like(QKV)
    for bi in range(b):
        rows = slice(bi * s, (bi + 1) * s)
        for j in range(heads):
            c = head_columns(h, heads, j)
            dq, dk, dv = attention_core_bwd(QKV[rows][:, c["q"]], QKV[rows][:, c["k"]],
                                            QKV[rows][:, c["v"]],
                                            dO[rows, j * d:(j + 1) * d], causal)
            dQKV[rows, c["q"]] = dq
            dQKV[rows, c["k"]] = dk
            dQKV[rows, c["v"]] = dv
    return {"dX": dQKV @ Wqkv.T, "dWqkv": X.T @ dQKV, "dWo": O.T @ dZ,
            "dQKV": dQKV, "dO": dO}


def attn_bwd_parallel(X, Wqkv, Wo, dZ, b: int, s: int, heads: int, t: int,
                      causal: bool = True):
    """The pages' mirror rule for attention ([P3] §3.2 backward steps 1-3).

    dZ goes to every group; group g computes dWo_g and dWqkv_g locally and
    a partial dX_g = dQKV_g @ Wqkv_g^T; dX = sum_g dX_g.
    """
    X, Wqkv, Wo, dZ = _f64(X), _f64(Wqkv), _f64(Wo), _f64(dZ)
    h, d = _attn_dims(X, Wqkv, heads, b, s)
    hg = _check_divisible(heads, t, "heads")
    w = hg * d
    dWqkv = np.zeros_like(Wqkv)
    dWo = np.zeros_like(Wo)
    dXs = []
    for g in range(t):
        cols = group_columns(h, heads, t, g)
        Wg = Wqkv[:, cols]
        Wog = Wo[g * w:(g + 1) * w]
        QKVg = X @ Wg
        dOg = dZ @ Wog.T
        Og = np.zeros((b * s, w))
        dQKVg = np.zeros_like(QKVg)
        for bi in range(b):
            rows = slice(bi * s, (bi + 1) * s)
            for jl in range(hg):
                sl = [slice(k * w + jl * d, k * w + (jl + 1) * d) for k in range(3)]
                q, k_, v = (QKVg[rows, sl[0]], QKVg[rows, sl[1]], QKVg[rows, sl[2]])
                Og[rows, jl * d:(jl + 1) * d] = attention_core(q, k_, v, causal)[0]
                dq, dk, dv = attention_core_bwd(q, k_, v, dOg[rows, jl * d:(jl + 1) * d],
                                                causal)
                dQKVg[rows, sl[0]], dQKVg[rows, sl[1]], dQKVg[rows, sl[2]] = dq, dk, dv
        dWqkv[:, cols] = X.T @ dQKVg
        dWo[g * w:(g + 1) * w] = Og.T @ dZ
        dXs.append(dQKVg @ Wg.T)
    dX = dXs[0].copy()
    for p in dXs[1:]:
        dX = dX + p
    return {"dX": dX, "dWqkv": dWqkv, "dWo": dWo, "dX_partials": dXs}


# ---------------------------------------------------------------------------
# LayerNorm and the Transformer block ([P2] §3.3 ParallelTransformerBlock:
# x = x + attention(norm1(x)); x = x + mlp(norm2(x)), norm = nn.LayerNorm)
# ---------------------------------------------------------------------------

def layernorm_fwd(X, gamma=None, beta=None, eps: float = 1e-5):
    """Row-wise LayerNorm: Y = (X - mean) / sqrt(var + eps) * gamma + beta,
    mean and (biased) variance over the last dimension.  Returns Y, mean and
    rstd = 1 / sqrt(var + eps) per row."""
    X = _f64(X)
    mean = X.mean(axis=-1)
    var = ((X - mean[:, None]) ** 2).mean(axis=-1)
    rstd = 1.0 / np.sqrt(var + eps)
    Y = (X - mean[:, None]) * rstd[:, None]
    if gamma is not None:
        Y = Y * _f64(gamma)
    if beta is not None:
        Y = Y + _f64(beta)
    return {"Y": Y, "mean": mean, "rstd": rstd}


def layernorm_bwd(X, gamma, dY, eps: float = 1e-5):
    """Backward of layernorm_fwd by the chain rule, with xhat = (X - mean) * rstd
    and g = dY * gamma: dX = rstd * (g - mean(g) - xhat * mean(g * xhat)),
    dgamma = sum over rows of dY * xhat, dbeta = sum over rows of dY."""
    X, dY = _f64(X), _f64(dY)
    f = layernorm_fwd(X, None, None, eps)
    xhat = (X - f["mean"][:, None]) * f["rstd"][:, None]
    g = dY * (_f64(gamma) if gamma is not None else 1.0)
    dX = f["rstd"][:, None] * (g - g.mean(axis=-1, keepdims=True)
                               - xhat * (g * xhat).mean(axis=-1, keepdims=True))
    return {"dX": dX, "dgamma": (dY * xhat).sum(axis=0), "dbeta": dY.sum(axis=0)}


def block_fwd(X, w, b: int, s: int, heads: int, eps: float = 1e-5, causal: bool = True):
    """One Transformer block: X1 = X + Attn(LN1(X)); X2 = X1 + MLP(LN2(X1)).
    `w` holds ln1_g, ln1_b, Wqkv, Wo, ln2_g, ln2_b, A, bA, B, bB."""
    X = _f64(X)
    n1 = layernorm_fwd(X, w["ln1_g"], w["ln1_b"], eps)
    at = attn_fwd(n1["Y"], w["Wqkv"], w["Wo"], b, s, heads, causal)
    X1 = X + at["Z"]
    n2 = layernorm_fwd(X1, w["ln2_g"], w["ln2_b"], eps)
    ml = mlp_fwd(n2["Y"], w["A"], w.get("bA"), w["B"], w.get("bB"))
    return {"X1": X1, "X2": X1 + ml["Z"], "Xn1": n1["Y"], "Xn2": n2["Y"]}


def block_bwd(X, w, dX2, b: int, s: int, heads: int, eps: float = 1e-5, causal: bool = True):
    """Backward of block_fwd: the residual paths pass the gradient through,
    the sublayers add theirs: dX1 = dX2 + LN2'(MLP'(dX2)); dX = dX1 + LN1'(Attn'(dX1))."""
    X, dX2 = _f64(X), _f64(dX2)
    fw = block_fwd(X, w, b, s, heads, eps, causal)
    mb = mlp_bwd(fw["Xn2"], w["A"], w.get("bA"), w["B"], dX2)
    l2 = layernorm_bwd(fw["X1"], w["ln2_g"], mb["dX"], eps)
    dX1 = dX2 + l2["dX"]
    ab = attn_bwd(fw["Xn1"], w["Wqkv"], w["Wo"], dX1, b, s, heads, causal)
    l1 = layernorm_bwd(X, w["ln1_g"], ab["dX"], eps)
    return {"dX": dX1 + l1["dX"], "dX1": dX1,
            "dln1_g": l1["dgamma"], "dln1_b": l1["dbeta"], "dWqkv": ab["dWqkv"], "dWo": ab["dWo"],
            "dln2_g": l2["dgamma"], "dln2_b": l2["dbeta"], "dA": mb["dA"], "dbA": mb["dbA"],
            "dB": mb["dB"], "dbB": mb["dbB"]}


# ---------------------------------------------------------------------------
# Vocabulary-parallel embedding and cross-entropy ([P3] §4.1, §4.2)
# ---------------------------------------------------------------------------

def vocab_embed_fwd(ids, E):
    """Unpartitioned lookup: Y[r] = E[ids[r]]; an id outside [0, V) gives 0."""
    ids = np.asarray(ids, dtype=np.int64)
    E = _f64(E)
    Y = np.zeros((len(ids), E.shape[1]))
    ok = (ids >= 0) & (ids < E.shape[0])
    Y[ok] = E[ids[ok]]
    return Y


def vocab_embed_fwd_parallel(ids, E, t: int):
    """[P3] §4.1: E split by vocabulary rows; shard i looks up the ids in its
    range [i*V/t, (i+1)*V/t) and returns a zero vector for the others; the
    partial results are summed (the AllReduce)."""
    ids = np.asarray(ids, dtype=np.int64)
    shards = split_rows(E, t)
    v = shards[0].shape[0]
    Y = np.zeros((len(ids), shards[0].shape[1]))
    for i, Ei in enumerate(shards):
        local = ids - i * v
        mine = (local >= 0) & (local < v)
        part = np.zeros_like(Y)
        part[mine] = Ei[local[mine]]
        Y = Y + part
    return Y


def vocab_embed_bwd(ids, dY, V: int):
    """dE[v] = sum of dY[r] over the rows r with ids[r] == v."""
    ids = np.asarray(ids, dtype=np.int64)
    dY = _f64(dY)
    dE = np.zeros((V, dY.shape[1]))
    ok = (ids >= 0) & (ids < V)
    np.add.at(dE, ids[ok], dY[ok])
    return dE


def _valid_targets(targets, V: int):
    """Rows whose target lies outside [0, V) are ignored: loss 0, gradient 0
    (a reading: the pages only treat in-range targets)."""
    targets = np.asarray(targets, dtype=np.int64)
    return targets, (targets >= 0) & (targets < V)


def vocab_ce_fwd(X, E, targets):
    """Unpartitioned cross-entropy of logits = X @ E^T (E [V, h], tied with the
    input embedding, [P3] §4.2): loss[r] = logsumexp(logits[r]) - logits[r, t_r],
    total = sum of loss[r] over the rows."""
    X, E = _f64(X), _f64(E)
    targets, ok = _valid_targets(targets, E.shape[0])
    z = X @ E.T
    m = z.max(axis=1)
    lse = m + np.log(np.exp(z - m[:, None]).sum(axis=1))
    rows = np.nonzero(ok)[0]
    loss = np.zeros(len(targets))
    loss[rows] = lse[rows] - z[rows, targets[rows]]
    return {"loss": loss, "lse": lse, "total": float(loss.sum())}


def vocab_ce_fwd_parallel(X, E, targets, t: int):
    """[P3] §4.2 steps 1-6 on t vocabulary shards E_i (rows of E):
    1. shard i computes its logits z_i = X @ E_i^T;
    2. its exponential sum, taken relative to the shard's own row maximum
       (a reading: the page's step 2 has no max subtraction; this is the
       same value, written so that it cannot overflow);
    3. the shards' sums are combined, rescaled to the largest maximum, into
       the global denominator (the AllReduce of b*s values), lse = log of it;
    4-5. the shard that owns a row's target takes its logit and forms that
       row's loss, lse - z_target; the shard's local loss is the sum of the
       losses of the rows whose targets it owns;
    6. the total loss is the sum of the shards' local losses (the AllReduce
       of t values)."""
    X = _f64(X)
    targets, ok = _valid_targets(targets, E.shape[0])
    shards = split_rows(E, t)
    v = shards[0].shape[0]
    M = X.shape[0]
    ms, ss = [], []
    for Ei in shards:                                    # steps 1-2
        zi = X @ Ei.T
        mi = zi.max(axis=1)
        ms.append(mi)
        ss.append(np.exp(zi - mi[:, None]).sum(axis=1))
    m = np.max(np.stack(ms), axis=0)                     # step 3
    total_exp = np.zeros(M)
    for mi, si in zip(ms, ss):
        total_exp = total_exp + si * np.exp(mi - m)
    lse = m + np.log(total_exp)
    loss = np.zeros(M)
    local_losses = []
    for i, Ei in enumerate(shards):                      # steps 4-5
        local = targets - i * v
        mine = ok & (local >= 0) & (local < v)
        rows = np.nonzero(mine)[0]
        z_t = (X[rows] * _f64(Ei)[local[rows]]).sum(axis=1)
        loss[rows] = lse[rows] - z_t
        local_losses.append(float(loss[rows].sum()))
    return {"loss": loss, "lse": lse, "total": float(sum(local_losses))}   # step 6


def vocab_ce_bwd(X, E, targets, dloss):
    """Gradient of sum_r dloss[r] * loss[r]: dlogits = (softmax - onehot) * dloss
    on the rows with a valid target (zero on ignored rows), dX = dlogits @ E,
    dE = dlogits^T @ X."""
    X, E = _f64(X), _f64(E)
    targets, ok = _valid_targets(targets, E.shape[0])
    z = X @ E.T
    p = np.exp(z - z.max(axis=1, keepdims=True))
    p = p / p.sum(axis=1, keepdims=True)
    rows = np.nonzero(ok)[0]
    p[rows, targets[rows]] -= 1.0
    p[~ok] = 0.0
    g = p * _f64(dloss)[:, None]
    return {"dX": g @ E, "dE": g.T @ X, "dlogits": g}


# ---------------------------------------------------------------------------
# Error measures used by every parity check
# ---------------------------------------------------------------------------

def max_rel_error(got, ref) -> float:
    """max_i |got_i - ref_i| / max_i |ref_i| (scaled by the tensor's max)."""
    got, ref = _f64(got), _f64(ref)
    scale = np.max(np.abs(ref))
    diff = np.max(np.abs(got - ref)) if got.size else 0.0
    return float(diff / scale) if scale > 0 else float(diff)


def normwise_error(got, ref) -> float:
    """||got - ref||_2 / ||ref||_2 over all elements."""
    got, ref = _f64(got), _f64(ref)
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((got - ref).ravel())
    return float(num / den) if den > 0 else float(num)
