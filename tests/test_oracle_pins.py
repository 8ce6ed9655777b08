"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each check relies on something the pages or mathematics fix: exact integer
arithmetic, a brute-force loop written independently on tiny inputs, textbook
values of the normal distribution, closed forms (prefix mean, identity
weights), and central finite differences for every backward.  The last group
plants plausible mistakes in a copy of the oracle and shows that some pin
fails for each of them.

Partition identities come from "图解Transformer并行计算：从矩阵乘法切分到
Megatron架构设计" (§1.1 row split = sum of partials, §1.2 column split =
concatenation, §2.1 GeLU per column shard, §2.2 and §3.2 mirror rule), and
the split-then-gather round trip and divisibility errors from "5.1 Tensor并行
与算子拆分" §1.1.
"""
import math
import os
import types

import numpy as np
import pytest

from oracle import tp_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _int_mat(shape, seed, lo=-3, hi=3):
    return _rng(seed).integers(lo, hi + 1, size=shape).astype(np.float64)


# ---------------------------------------------------------------------------
# Independent brute-force routines (pure Python loops, math module only)
# ---------------------------------------------------------------------------

def bf_matmul_int(X, W):
    """Exact integer product with Python ints."""
    M, K = len(X), len(X[0])
    N = len(W[0])
    return [[sum(int(X[i][k]) * int(W[k][j]) for k in range(K)) for j in range(N)]
            for i in range(M)]


def bf_phi_cdf(x):
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def bf_mlp(X, A, bA, B, bB):
    """Loop MLP: Z[r][c] = sum_j GeLU(sum_k X[r][k] A[k][j] + bA[j]) B[j][c] + bB[c]."""
    M, h = X.shape
    f = A.shape[1]
    Z = np.zeros((M, B.shape[1]))
    for r in range(M):
        Hrow = []
        for j in range(f):
            y = bA[j]
            for k in range(h):
                y += X[r, k] * A[k, j]
            Hrow.append(y * bf_phi_cdf(y))
        for c in range(B.shape[1]):
            z = bB[c]
            for j in range(f):
                z += Hrow[j] * B[j, c]
            Z[r, c] = z
    return Z


def bf_attention(Xb, Wqkv, Wo, heads, causal):
    """Loop multi-head attention for one sequence, indexing [Wq | Wk | Wv] by hand."""
    s, h = Xb.shape
    d = h // heads
    qkv = [[sum(Xb[r, k] * Wqkv[k, c] for k in range(h)) for c in range(3 * h)]
           for r in range(s)]
    Ocat = [[0.0] * h for _ in range(s)]
    lse = [[0.0] * s for _ in range(heads)]
    for j in range(heads):
        for r in range(s):
            scores = []
            for c in range(s):
                if causal and c > r:
                    continue
                dot = sum(qkv[r][j * d + e] * qkv[c][h + j * d + e] for e in range(d))
                scores.append((c, dot / math.sqrt(d)))
            mx = max(v for _, v in scores)
            w = [(c, math.exp(v - mx)) for c, v in scores]
            den = sum(v for _, v in w)
            lse[j][r] = mx + math.log(den)
            for e in range(d):
                Ocat[r][j * d + e] = sum(p * qkv[c][2 * h + j * d + e] for c, p in w) / den
    Z = [[sum(Ocat[r][k] * Wo[k, c] for k in range(h)) for c in range(h)] for r in range(s)]
    return np.array(Z), np.array(Ocat), np.array(lse)


# ---------------------------------------------------------------------------
# Pin checks, written as functions of an oracle module so that the planted-
# mistake tests can run them against a broken copy.
# ---------------------------------------------------------------------------

def check_gelu_table(o):
    rows = [l.split() for l in open(os.path.join(GOLDEN, "normal_cdf_pdf.txt"))
            if l.strip() and not l.startswith("#")]
    for x, cdf, pdf in ((float(a), float(b), float(c)) for a, b, c in rows):
        assert abs(float(o.gelu(np.array([x]))[0]) - x * cdf) <= 1e-15 * max(1.0, abs(x))
        assert abs(float(o.gelu_prime(np.array([x]))[0]) - (cdf + x * pdf)) <= 2e-15


def check_linear_exact(o):
    X, W = _int_mat((7, 24), 1), _int_mat((24, 16), 2)
    b = _int_mat((16,), 3)
    ref = np.array(bf_matmul_int(X.tolist(), W.tolist()), dtype=np.float64) + b
    assert np.array_equal(o.linear(X, W, b), ref)
    for t in (1, 2, 4, 8):
        assert np.array_equal(o.linear_col_parallel(X, W, b, t), ref)
        assert np.array_equal(o.linear_row_parallel(X, W, b, t), ref)
    Ws = _int_mat((24, 24), 4)  # square weight: a transposed operand would go unnoticed otherwise
    ref = np.array(bf_matmul_int(X.tolist(), Ws.tolist()), dtype=np.float64)
    assert np.array_equal(o.linear(X, Ws), ref)


def check_mlp_bruteforce(o):
    r = _rng(11)
    X = r.standard_normal((3, 4))
    A, B = r.standard_normal((4, 8)) * 0.5, r.standard_normal((8, 4)) * 0.5
    bA, bB = r.standard_normal(8) * 0.1, r.standard_normal(4) * 0.1
    ref = bf_mlp(X, A, bA, B, bB)
    got = o.mlp_fwd(X, A, bA, B, bB)["Z"]
    assert np.max(np.abs(got - ref)) < 1e-13
    for t in (1, 2, 4):
        assert np.max(np.abs(o.mlp_fwd_parallel(X, A, bA, B, bB, t)["Z"] - ref)) < 1e-13


def _fd_grad(fun, P, eps=1e-6):
    g = np.zeros_like(P)
    it = np.nditer(P, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = P[i]
        P[i] = old + eps
        up = fun()
        P[i] = old - eps
        dn = fun()
        P[i] = old
        g[i] = (up - dn) / (2 * eps)
    return g


def check_mlp_bwd_fd(o):
    r = _rng(12)
    X = r.standard_normal((3, 4))
    A, B = r.standard_normal((4, 8)) * 0.7, r.standard_normal((8, 4)) * 0.7
    bA, bB = r.standard_normal(8) * 0.1, r.standard_normal(4) * 0.1
    G = r.standard_normal((3, 4))  # L = <G, Z>, so dZ = G
    loss = lambda: float(np.sum(G * o.mlp_fwd(X, A, bA, B, bB)["Z"]))
    g = o.mlp_bwd(X, A, bA, B, G)
    for name, P in (("dX", X), ("dA", A), ("dbA", bA), ("dB", B), ("dbB", bB)):
        fd = _fd_grad(loss, P)
        assert np.max(np.abs(g[name] - fd)) < 1e-7, name
    for t in (1, 2, 4):
        gp = o.mlp_bwd_parallel(X, A, bA, B, G, t)
        for name in ("dX", "dA", "dbA", "dB", "dbB"):
            assert np.max(np.abs(gp[name] - g[name])) < 1e-12, (name, t)


def check_attention_bruteforce(o):
    r = _rng(13)
    b, s, h, heads = 2, 4, 8, 2
    X = r.standard_normal((b * s, h))
    Wqkv, Wo = r.standard_normal((h, 3 * h)) * 0.5, r.standard_normal((h, h)) * 0.5
    for causal in (True, False):
        got = o.attn_fwd(X, Wqkv, Wo, b, s, heads, causal)
        for bi in range(b):
            Z, Ocat, lse = bf_attention(X[bi * s:(bi + 1) * s], Wqkv, Wo, heads, causal)
            assert np.max(np.abs(got["Z"][bi * s:(bi + 1) * s] - Z)) < 1e-12
            assert np.max(np.abs(got["O"][bi * s:(bi + 1) * s] - Ocat)) < 1e-12
            assert np.max(np.abs(got["LSE"][bi] - lse)) < 1e-12
        for t in (1, 2):
            gp = o.attn_fwd_parallel(X, Wqkv, Wo, b, s, heads, t, causal)
            assert np.max(np.abs(gp["Z"] - got["Z"])) < 1e-12


def check_attention_closed_forms(o):
    r = _rng(14)
    s, d = 9, 8
    V = r.standard_normal((s, d))
    K = r.standard_normal((s, d))
    # Q = 0: every unmasked score is 0, so row r of O is the mean of V[0..r].
    Oq0, P, lse = o.attention_core(np.zeros((s, d)), K, V, causal=True)
    prefix_mean = np.cumsum(V, axis=0) / np.arange(1, s + 1)[:, None]
    assert np.max(np.abs(Oq0 - prefix_mean)) < 1e-14
    assert np.allclose(lse, np.log(np.arange(1, s + 1)), rtol=0, atol=1e-14)
    # Row 0 sees only key 0, so O[0] = V[0] exactly; rows of P sum to 1; masked part is 0.
    Q = r.standard_normal((s, d))
    Oc, P, _ = o.attention_core(Q, K, V, causal=True)
    assert np.array_equal(Oc[0], V[0])
    assert np.max(np.abs(P.sum(axis=1) - 1.0)) < 1e-15
    assert np.all(np.triu(P, 1) == 0.0)


def check_attention_bwd_fd(o):
    r = _rng(15)
    b, s, h, heads = 2, 4, 8, 2
    X = r.standard_normal((b * s, h))
    Wqkv, Wo = r.standard_normal((h, 3 * h)) * 0.5, r.standard_normal((h, h)) * 0.5
    G = r.standard_normal((b * s, h))
    loss = lambda: float(np.sum(G * o.attn_fwd(X, Wqkv, Wo, b, s, heads, True)["Z"]))
    g = o.attn_bwd(X, Wqkv, Wo, G, b, s, heads, True)
    for name, P in (("dX", X), ("dWqkv", Wqkv), ("dWo", Wo)):
        fd = _fd_grad(loss, P)
        assert np.max(np.abs(g[name] - fd)) < 1e-7, name
    for t in (1, 2):
        gp = o.attn_bwd_parallel(X, Wqkv, Wo, G, b, s, heads, t, True)
        for name in ("dX", "dWqkv", "dWo"):
            assert np.max(np.abs(gp[name] - g[name])) < 1e-12, (name, t)


PINS = [check_gelu_table, check_linear_exact, check_mlp_bruteforce, check_mlp_bwd_fd,
        check_attention_bruteforce, check_attention_closed_forms, check_attention_bwd_fd]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(O)


# ---------------------------------------------------------------------------
# Slicing and partition identities (bit-exact)
# ---------------------------------------------------------------------------

def test_split_gather_roundtrip_and_contiguity():
    W = _rng(20).standard_normal((32, 48))
    for t in (1, 2, 4, 8):
        cs, rs = O.split_cols(W, t), O.split_rows(W, t)
        assert np.array_equal(np.concatenate(cs, axis=1), W)
        assert np.array_equal(np.concatenate(rs, axis=0), W)
        for i in range(t):
            assert np.array_equal(cs[i], W[:, i * 48 // t:(i + 1) * 48 // t])
            assert np.array_equal(rs[i], W[i * 32 // t:(i + 1) * 32 // t])


def test_split_rejects_non_divisible():
    W = np.zeros((12, 10))
    with pytest.raises(ValueError):
        O.split_cols(W, 4)
    with pytest.raises(ValueError):
        O.split_rows(W, 5)
    with pytest.raises(ValueError):
        O.group_columns(64, 6, 4, 0)


def test_row_partials_sum_exactly_on_integers():
    X, W = _int_mat((16, 64), 21), _int_mat((64, 24), 22)
    ref = np.array(bf_matmul_int(X.tolist(), W.tolist()), dtype=np.float64)
    for t in (1, 2, 4, 8):
        Z, parts = O.linear_row_parallel(X, W, None, t, return_partials=True)
        assert np.array_equal(Z, ref)
        for i, p in enumerate(parts):
            k = 64 // t
            sub = np.array(bf_matmul_int(X[:, i * k:(i + 1) * k].tolist(),
                                         W[i * k:(i + 1) * k].tolist()), dtype=np.float64)
            assert np.array_equal(p, sub)


def test_gelu_per_shard_equals_gelu_on_full():
    X, A = _int_mat((8, 16), 23), _int_mat((16, 32), 24) / 4.0  # exact dyadic values
    full = O.mlp_fwd(X, A, None, np.zeros((32, 16)), None)
    for t in (1, 2, 4, 8):
        par = O.mlp_fwd_parallel(X, A, None, np.zeros((32, 16)), None, t)
        assert np.array_equal(par["Y"], full["Y"])
        assert np.array_equal(par["H"], full["H"])


def test_gelu_identities():
    x = np.linspace(-6, 6, 1001)
    assert np.max(np.abs(O.gelu(x) - O.gelu(-x) - x)) < 1e-14
    assert np.max(np.abs(O.gelu_prime(x) + O.gelu_prime(-x) - 1.0)) < 1e-14
    assert O.gelu(np.array([0.0]))[0] == 0.0
    assert abs(O.gelu(np.array([10.0]))[0] - 10.0) < 1e-20 * 10 + 1e-15
    fd = (O.gelu(x + 1e-6) - O.gelu(x - 1e-6)) / 2e-6
    assert np.max(np.abs(fd - O.gelu_prime(x))) < 1e-8


def test_mlp_identity_weights_closed_form():
    X = _rng(25).standard_normal((5, 6))
    I = np.eye(6)
    assert np.max(np.abs(O.mlp_fwd(X, I, None, I, None)["Z"] - X * np.vectorize(bf_phi_cdf)(X))) < 1e-15


def test_cross_t_agreement_mlp_and_attention():
    r = _rng(26)
    X = r.standard_normal((8, 16))
    A, B = r.standard_normal((16, 64)) * 0.3, r.standard_normal((64, 16)) * 0.3
    bA, bB = r.standard_normal(64) * 0.1, r.standard_normal(16) * 0.1
    ref = O.mlp_fwd(X, A, bA, B, bB)["Z"]
    for t in (1, 2, 4, 8):
        assert np.max(np.abs(O.mlp_fwd_parallel(X, A, bA, B, bB, t)["Z"] - ref)) < 1e-13
    Xa = r.standard_normal((2 * 5, 16))
    Wqkv, Wo = r.standard_normal((16, 48)) * 0.3, r.standard_normal((16, 16)) * 0.3
    ref = O.attn_fwd(Xa, Wqkv, Wo, 2, 5, 8)["Z"]
    for t in (1, 2, 4, 8):
        assert np.max(np.abs(O.attn_fwd_parallel(Xa, Wqkv, Wo, 2, 5, 8, t)["Z"] - ref)) < 1e-13


def test_group_columns_layout():
    h, heads, t = 16, 4, 2  # d = 4, two heads per group
    g1 = O.group_columns(h, heads, t, 1)
    assert g1.tolist() == [8, 9, 10, 11, 12, 13, 14, 15,
                           24, 25, 26, 27, 28, 29, 30, 31,
                           40, 41, 42, 43, 44, 45, 46, 47]


def test_error_measures():
    ref = np.array([1.0, -4.0, 2.0])
    got = np.array([1.5, -4.0, 2.0])
    assert O.max_rel_error(got, ref) == 0.5 / 4.0
    assert abs(O.normwise_error(got, ref) - 0.5 / math.sqrt(21.0)) < 1e-16


# ---------------------------------------------------------------------------
# Planted mistakes: each broken copy of the oracle must fail at least one pin
# ---------------------------------------------------------------------------

def _mutant(**overrides):
    m = types.ModuleType("oracle_mutant")
    m.__dict__.update({k: getattr(O, k) for k in dir(O) if not k.startswith("__")})
    m.__dict__.update(overrides)
    # Re-bind the module-level functions so they see the overrides.
    for name in O.__all__:
        if name in overrides:
            continue
        fn = getattr(O, name)
        if callable(fn) and hasattr(fn, "__code__"):
            m.__dict__[name] = types.FunctionType(fn.__code__, m.__dict__, fn.__name__,
                                                  fn.__defaults__, fn.__closure__)
    return m


def _tanh_gelu(x):
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1 + np.tanh(math.sqrt(2 / math.pi) * (x + 0.044715 * x ** 3)))


def _bwd_without_gelu_prime(X, A, bA, B, dZ, Y=None):
    X, A, B, dZ = (np.asarray(v, dtype=np.float64) for v in (X, A, B, dZ))
    Y = X @ A + (bA if bA is not None else 0.0)
    H = O.gelu(Y)
    dY = dZ @ B.T  # mistake: the GeLU' factor is dropped
    return {"dX": dY @ A.T, "dA": X.T @ dY, "dbA": dY.sum(0), "dB": H.T @ dZ,
            "dbB": dZ.sum(0), "dY": dY}


def _core_no_scale(Q, K, V, causal=True):
    Q, K, V = (np.asarray(v, dtype=np.float64) for v in (Q, K, V))
    S = Q @ K.T  # mistake: no 1/sqrt(d)
    if causal:
        S = np.where(np.arange(S.shape[1])[None, :] > np.arange(S.shape[0])[:, None], -np.inf, S)
    m = S.max(1, keepdims=True)
    E = np.exp(S - m)
    return (E / E.sum(1, keepdims=True)) @ V, E / E.sum(1, keepdims=True), (m + np.log(E.sum(1, keepdims=True)))[:, 0]


def _core_mask_off_by_one(Q, K, V, causal=True):
    Q, K, V = (np.asarray(v, dtype=np.float64) for v in (Q, K, V))
    S = Q @ K.T / math.sqrt(Q.shape[1])
    if causal:  # mistake: also hides the diagonal key except on row 0
        r, c = np.arange(S.shape[0])[:, None], np.arange(S.shape[1])[None, :]
        S = np.where((c >= r) & (r > 0), -np.inf, S)
    m = S.max(1, keepdims=True)
    E = np.exp(S - m)
    return (E / E.sum(1, keepdims=True)) @ V, E / E.sum(1, keepdims=True), (m + np.log(E.sum(1, keepdims=True)))[:, 0]


def _row_parallel_bias_per_shard(X, W, bias, t, return_partials=False):
    Xs, Ws = O.split_cols(X, t), O.split_rows(W, t)
    parts = [Xi @ Wi + (bias if bias is not None else 0.0) for Xi, Wi in zip(Xs, Ws)]
    Z = sum(parts[1:], parts[0].copy())
    return (Z, parts) if return_partials else Z


def _transposed_linear(X, W, bias=None):
    X, W = np.asarray(X, dtype=np.float64), np.asarray(W, dtype=np.float64)
    Y = X @ (W.T if W.shape[0] == W.shape[1] else W)  # mistake only visible for square W
    return Y + (bias if bias is not None else 0.0)


def _head_columns_swapped(h, heads, j):
    d = h // heads
    base = np.arange(j * d, (j + 1) * d)
    other = np.arange((heads - 1 - j) * d, (heads - j) * d)
    return {"q": base, "k": h + other, "v": 2 * h + base}  # mistake: k of the mirrored head


MUTANTS = {
    "wrong head columns": dict(head_columns=_head_columns_swapped),
    "tanh GeLU": dict(gelu=_tanh_gelu),
    "GeLU' dropped": dict(mlp_bwd=_bwd_without_gelu_prime),
    "no 1/sqrt(d)": dict(attention_core=_core_no_scale),
    "mask off by one": dict(attention_core=_core_mask_off_by_one),
    "row bias per shard": dict(linear_row_parallel=_row_parallel_bias_per_shard),
    "transposed square weight": dict(linear=_transposed_linear),
}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_planted_mistake_is_caught(name):
    m = _mutant(**MUTANTS[name])
    failures = 0
    for pin in PINS:
        try:
            pin(m)
        except AssertionError:
            failures += 1
    assert failures >= 1, f"no pin caught the planted mistake '{name}'"


def test_head_slice_equals_the_heads_columns():
    """[P3] §3.2: a head group computes its heads from its own column slice of
    Wq, Wk, Wv and row slice of Wo; the slice gives exactly those heads' O,
    LSE, dWqkv columns and dWo rows of the whole layer."""
    r = _rng(30)
    b, s, h, heads = 2, 5, 16, 4
    X = r.standard_normal((b * s, h))
    Wqkv, Wo = r.standard_normal((h, 3 * h)) * 0.4, r.standard_normal((h, h)) * 0.4
    dZ = r.standard_normal((b * s, h))
    full = O.attn_fwd(X, Wqkv, Wo, b, s, heads)
    gfull = O.attn_bwd(X, Wqkv, Wo, dZ, b, s, heads)
    d = h // heads
    for j in range(heads):
        c = O.head_columns(h, heads, j)
        cols = np.concatenate([c["q"], c["k"], c["v"]])
        one = O.attn_fwd(X, Wqkv[:, cols], Wo[j * d:(j + 1) * d], b, s, 1)
        assert np.max(np.abs(one["O"] - full["O"][:, j * d:(j + 1) * d])) < 1e-13
        assert np.max(np.abs(one["LSE"][:, 0] - full["LSE"][:, j])) < 1e-13
        g = O.attn_bwd(X, Wqkv[:, cols], Wo[j * d:(j + 1) * d], dZ, b, s, 1)
        assert np.max(np.abs(g["dWqkv"] - gfull["dWqkv"][:, cols])) < 1e-12
        assert np.max(np.abs(g["dWo"] - gfull["dWo"][j * d:(j + 1) * d])) < 1e-12


# ---------------------------------------------------------------------------
# LayerNorm and the block ([P2] §3.3)
# ---------------------------------------------------------------------------

def bf_layernorm_row(x, g, b, eps):
    n = len(x)
    mu = sum(x) / n
    var = sum((v - mu) ** 2 for v in x) / n
    return [(v - mu) / math.sqrt(var + eps) * gi + bi for v, gi, bi in zip(x, g, b)]


def check_layernorm(o):
    r = _rng(40)
    X = r.standard_normal((5, 12)) * 3 + 1.5
    g, b = r.standard_normal(12), r.standard_normal(12)
    out = o.layernorm_fwd(X, g, b, 1e-5)
    for i in range(5):
        ref = bf_layernorm_row(list(X[i]), list(g), list(b), 1e-5)
        assert np.max(np.abs(out["Y"][i] - ref)) < 1e-12
    plain = o.layernorm_fwd(X, None, None, 0.0)["Y"]  # closed form: zero mean, unit variance
    assert np.max(np.abs(plain.mean(axis=1))) < 1e-14
    assert np.max(np.abs((plain ** 2).mean(axis=1) - 1.0)) < 1e-13
    G = r.standard_normal((5, 12))
    loss = lambda: float(np.sum(G * o.layernorm_fwd(X, g, b, 1e-5)["Y"]))
    bw = o.layernorm_bwd(X, g, G, 1e-5)
    for name, P in (("dX", X), ("dgamma", g), ("dbeta", b)):
        assert np.max(np.abs(bw[name] - _fd_grad(loss, P))) < 1e-7, name


def _tiny_block(seed):
    r = _rng(seed)
    h, f = 8, 16
    w = {"ln1_g": 1 + 0.1 * r.standard_normal(h), "ln1_b": 0.1 * r.standard_normal(h),
         "Wqkv": r.standard_normal((h, 3 * h)) * 0.4, "Wo": r.standard_normal((h, h)) * 0.4,
         "ln2_g": 1 + 0.1 * r.standard_normal(h), "ln2_b": 0.1 * r.standard_normal(h),
         "A": r.standard_normal((h, f)) * 0.4, "bA": 0.1 * r.standard_normal(f),
         "B": r.standard_normal((f, h)) * 0.4, "bB": 0.1 * r.standard_normal(h)}
    return w, r.standard_normal((2 * 3, h)), r.standard_normal((2 * 3, h))


def check_block_bwd_fd(o):
    w, X, G = _tiny_block(41)
    loss = lambda: float(np.sum(G * o.block_fwd(X, w, 2, 3, 2)["X2"]))
    bw = o.block_bwd(X, w, G, 2, 3, 2)
    assert np.max(np.abs(bw["dX"] - _fd_grad(loss, X))) < 1e-6
    for name, key in (("dln1_g", "ln1_g"), ("dWqkv", "Wqkv"), ("dWo", "Wo"), ("dln2_b", "ln2_b"),
                      ("dA", "A"), ("dbB", "bB")):
        assert np.max(np.abs(bw[name] - _fd_grad(loss, w[key]))) < 1e-6, name


PINS += [check_layernorm, check_block_bwd_fd]


@pytest.mark.parametrize("pin", [check_layernorm, check_block_bwd_fd], ids=lambda p: p.__name__)
def test_block_pins(pin):
    pin(O)


def test_block_residual_identity():
    """With zero Wo and zero B the sublayers add nothing: X2 = X1 = X."""
    w, X, _ = _tiny_block(42)
    w["Wo"] = np.zeros_like(w["Wo"])
    w["B"], w["bB"] = np.zeros_like(w["B"]), np.zeros_like(w["bB"])
    out = O.block_fwd(X, w, 2, 3, 2)
    assert np.array_equal(out["X1"], X) and np.array_equal(out["X2"], X)


def _ln_no_centering(X, gamma=None, beta=None, eps=1e-5):
    X = np.asarray(X, dtype=np.float64)
    rstd = 1.0 / np.sqrt((X ** 2).mean(axis=-1) + eps)  # mistake: RMS norm, no mean removed
    Y = X * rstd[:, None] * (gamma if gamma is not None else 1.0) + (beta if beta is not None else 0.0)
    return {"Y": Y, "mean": X.mean(axis=-1), "rstd": rstd}


MUTANTS["LayerNorm without centering"] = dict(layernorm_fwd=_ln_no_centering)


def test_planted_layernorm_mistake_is_caught():
    m = _mutant(layernorm_fwd=_ln_no_centering)
    with pytest.raises(AssertionError):
        check_layernorm(m)


# ---------------------------------------------------------------------------
# Vocabulary-parallel embedding and cross-entropy ([P3] §4.1, §4.2)
# ---------------------------------------------------------------------------

def check_vocab(o):
    r = _rng(50)
    V, h = 24, 5
    E = r.standard_normal((V, h))
    ids = np.array([0, 23, 7, 7, -1, 24, 12, 3])
    Y = o.vocab_embed_fwd(ids, E)
    for i, v in enumerate(ids):  # exact gather; out-of-range ids give zeros
        assert np.array_equal(Y[i], E[v] if 0 <= v < V else np.zeros(h))
    for t in (1, 2, 3, 4, 8):
        assert np.array_equal(o.vocab_embed_fwd_parallel(ids, E, t), Y)
    dY = _int_mat((8, h), 51)
    dE = o.vocab_embed_bwd(ids, dY, V)
    assert np.array_equal(dE[7], dY[2] + dY[3]) and np.array_equal(dE[1], np.zeros(h))
    assert dE.sum() == dY[[0, 1, 2, 3, 6, 7]].sum()
    # cross-entropy: all-zero logits give log V; brute force on one row
    X = r.standard_normal((6, h))
    tg = np.array([0, 5, 23, 11, 11, 2])
    assert np.allclose(o.vocab_ce_fwd(X, np.zeros((V, h)), tg)["loss"], math.log(V), rtol=0, atol=1e-14)
    ce = o.vocab_ce_fwd(X, E, tg)
    for i in range(6):
        zs = [sum(X[i, k] * E[v, k] for k in range(h)) for v in range(V)]
        ref = math.log(sum(math.exp(z) for z in zs)) - zs[tg[i]]
        assert abs(ce["loss"][i] - ref) < 1e-12
    assert abs(ce["total"] - sum(ce["loss"])) < 1e-12
    for t in (1, 2, 3, 4, 8):
        cp = o.vocab_ce_fwd_parallel(X, E, tg, t)
        assert np.max(np.abs(cp["loss"] - ce["loss"])) < 1e-12
        assert np.max(np.abs(cp["lse"] - ce["lse"])) < 1e-12
        assert abs(cp["total"] - ce["total"]) < 1e-11
    # large logits: the max-subtracted form stays finite where exp overflows
    big = o.vocab_ce_fwd_parallel(X * 400.0, E, tg, 4)
    assert np.all(np.isfinite(big["loss"])) and np.all(big["loss"] >= -1e-9)
    # an ignored row (target out of range) has loss 0 and no gradient
    tg2 = tg.copy()
    tg2[3] = -1
    tg2[4] = V
    ce2 = o.vocab_ce_fwd_parallel(X, E, tg2, 3)
    assert ce2["loss"][3] == 0 and ce2["loss"][4] == 0
    assert abs(ce2["loss"][[0, 1, 2, 5]] - ce["loss"][[0, 1, 2, 5]]).max() < 1e-12
    g2 = o.vocab_ce_bwd(X, E, tg2, np.ones(6))
    assert not g2["dlogits"][3].any() and not g2["dX"][4].any()
    # softmax rows sum to one, so each valid dlogits row sums to zero
    assert np.max(np.abs(g2["dlogits"].sum(axis=1))) < 1e-12
    dl = r.standard_normal(6)
    loss = lambda: float(np.sum(dl * o.vocab_ce_fwd(X, E, tg)["loss"]))
    g = o.vocab_ce_bwd(X, E, tg, dl)
    assert np.max(np.abs(g["dX"] - _fd_grad(loss, X))) < 1e-7
    assert np.max(np.abs(g["dE"] - _fd_grad(loss, E))) < 1e-7


def test_vocab_pins():
    check_vocab(O)


def _ce_without_target(X, E, targets):
    X, E = np.asarray(X, dtype=np.float64), np.asarray(E, dtype=np.float64)
    z = X @ E.T
    m = z.max(axis=1)
    lse = m + np.log(np.exp(z - m[:, None]).sum(axis=1))
    loss = lse - z[:, 0]  # mistake: always class 0
    return {"loss": loss, "lse": lse, "total": float(loss.sum())}


def _ce_parallel_unscaled(X, E, targets, t):
    """Mistake: the shards' exponential sums are added without rescaling
    them to a common maximum."""
    X = np.asarray(X, dtype=np.float64)
    targets = np.asarray(targets, dtype=np.int64)
    shards = O.split_rows(E, t)
    tot, ms = 0.0, []
    for Ei in shards:
        zi = X @ np.asarray(Ei, dtype=np.float64).T
        mi = zi.max(axis=1)
        ms.append(mi)
        tot = tot + np.exp(zi - mi[:, None]).sum(axis=1)
    lse = np.max(np.stack(ms), axis=0) + np.log(tot)
    z = X @ np.asarray(E, dtype=np.float64).T
    loss = lse - z[np.arange(len(targets)), np.clip(targets, 0, z.shape[1] - 1)]
    return {"loss": loss, "lse": lse, "total": float(loss.sum())}


def _embed_parallel_off_by_one(ids, E, t):
    ids = np.asarray(ids)
    return O.vocab_embed_fwd_parallel(np.where(ids >= 0, ids + 1, ids), E, t)


@pytest.mark.parametrize("mutant", [dict(vocab_ce_fwd=_ce_without_target),
                                    dict(vocab_ce_fwd_parallel=_ce_parallel_unscaled),
                                    dict(vocab_embed_fwd_parallel=_embed_parallel_off_by_one)],
                         ids=["ce_target", "ce_unscaled", "embed_offset"])
def test_planted_vocab_mistake_is_caught(mutant):
    with pytest.raises(AssertionError):
        check_vocab(_mutant(**mutant))
