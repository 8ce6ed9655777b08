"""libtp's C ABI on a machine without a GPU: the library loads, exports every
entry point that include/libtp.h declares, and its host-side validation
returns the documented status before touching the device.

Divisibility rules follow "5.1 Tensor并行与算子拆分" §1.1 (tensor_parallel_split
raises on a size the partition count does not divide) and the heads rule of
the PyTorch tutorial's ParallelAttention (§2.2, num_heads // world_size).
"""
import ctypes
import os
import re

import pytest

from megatron_tensor_transformer_logical_b200 import binding as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "libtp.h")

# Fake, 16-byte aligned addresses: validation rejects the call before any use.
P = [0x10000 * (i + 1) for i in range(12)]


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(L.LIB_PATH):
        from megatron_tensor_transformer_logical_b200 import build
        build.build()
    return L.load()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"\b(tp_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert set(declared_symbols()) == set(L.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_version(lib):
    assert lib.tp_version() == 100


def _lin(lib, fn, X, W, b, Y, M, K, N, t, shard=-1, dt=L.TP_BF16, odt=L.TP_BF16):
    return getattr(lib, fn)(X, W, b, Y, M, K, N, t, shard, dt, odt, None)


@pytest.mark.parametrize("fn", ["tp_linear_col", "tp_linear_row"])
def test_linear_validation(lib, fn):
    ok = (P[0], P[1], None, P[2], 64, 128, 256, 4)
    assert _lin(lib, fn, None, P[1], None, P[2], 64, 128, 256, 4) == L.TP_ERR_NULL
    assert _lin(lib, fn, P[0], P[1], None, None, 64, 128, 256, 4) == L.TP_ERR_NULL
    assert _lin(lib, fn, *ok[:4], 0, 128, 256, 4) == L.TP_ERR_SHAPE
    assert _lin(lib, fn, *ok[:4], 64, 128, 256, 0) == L.TP_ERR_SHAPE
    assert _lin(lib, fn, *ok[:4], 64, 128, 256, 65) == L.TP_ERR_SHAPE
    assert _lin(lib, fn, *ok[:4], 64, 128, 256, 4, shard=4) == L.TP_ERR_SHAPE
    # the split dimension must be divisible by t
    if fn == "tp_linear_col":
        assert _lin(lib, fn, *ok[:4], 64, 128, 264, 16) == L.TP_ERR_SHAPE
    else:
        assert _lin(lib, fn, *ok[:4], 64, 136, 256, 16) == L.TP_ERR_SHAPE
    assert _lin(lib, fn, P[0] + 2, P[1], None, P[2], 64, 128, 256, 4) == L.TP_ERR_ALIGN
    assert _lin(lib, fn, *ok[:4], 64, 124, 256, 4) == L.TP_ERR_ALIGN
    assert _lin(lib, fn, *ok[:4], 64, 128, 256, 4, dt=7) == L.TP_ERR_DTYPE
    assert _lin(lib, fn, *ok[:4], 64, 128, 256, 4, dt=L.TP_F32, odt=L.TP_BF16) == L.TP_ERR_DTYPE
    # shard-only mode needs 8-element aligned shard widths
    assert _lin(lib, fn, *ok[:4], 64, 128, 256, 64, shard=1) == L.TP_ERR_ALIGN
    assert b"" != lib.tp_last_error()


def test_mlp_validation(lib):
    ws = P[9]
    big = 1 << 40
    args = lambda **k: dict(dict(X=P[0], A=P[1], bA=None, B=P[2], bB=None, Z=P[3], Y=None,
                                 M=64, h=128, f=512, t=4, dt=L.TP_BF16, ws=ws, wsb=big), **k)

    def fwd(a):
        return lib.tp_mlp_fwd(a["X"], a["A"], a["bA"], a["B"], a["bB"], a["Z"], a["Y"], a["M"],
                              a["h"], a["f"], a["t"], a["dt"], a["ws"], a["wsb"], None)

    assert fwd(args(X=None)) == L.TP_ERR_NULL
    assert fwd(args(f=510, t=4)) == L.TP_ERR_SHAPE
    assert fwd(args(f=516, t=8)) == L.TP_ERR_SHAPE
    assert fwd(args(h=130)) == L.TP_ERR_ALIGN
    assert fwd(args(bA=P[4] + 4)) == L.TP_ERR_ALIGN
    assert fwd(args(ws=None)) == L.TP_ERR_WORKSPACE
    assert fwd(args(wsb=16)) == L.TP_ERR_WORKSPACE
    assert fwd(args(dt=3)) == L.TP_ERR_DTYPE

    def bwd(**k):
        a = args(**k)
        return lib.tp_mlp_bwd(a["X"], a["A"], a["bA"], a["B"], None, P[5], P[6], P[7], None,
                              P[8], None, a["M"], a["h"], a["f"], a["t"], a["dt"], a["ws"],
                              a["wsb"], None)

    assert bwd(f=510) == L.TP_ERR_SHAPE
    assert bwd(ws=None) == L.TP_ERR_WORKSPACE
    assert lib.tp_mlp_bwd(P[0], P[1], None, P[2], None, None, P[6], P[7], None, P[8], None,
                          64, 128, 512, 4, L.TP_BF16, ws, big, None) == L.TP_ERR_NULL


def test_attention_validation(lib):
    big = 1 << 40

    def fwd(b=2, s=64, h=512, heads=4, t=2, dt=L.TP_BF16, X=P[0], ws=P[9]):
        return lib.tp_attn_fwd(X, P[1], P[2], P[3], None, None, None, b, s, h, heads, t, 1,
                               dt, ws, big, None)

    assert fwd(X=None) == L.TP_ERR_NULL
    assert fwd(dt=L.TP_F32) == L.TP_ERR_UNSUPPORTED
    assert fwd(heads=3) == L.TP_ERR_SHAPE          # h % heads
    assert fwd(heads=4, t=3) == L.TP_ERR_SHAPE     # heads % t
    assert fwd(h=256, heads=4) == L.TP_ERR_UNSUPPORTED  # d = 64
    assert fwd(s=0) == L.TP_ERR_SHAPE
    assert fwd(ws=None) == L.TP_ERR_WORKSPACE
    assert lib.tp_attn_bwd(P[0], P[1], P[2], None, None, P[4], P[5], P[6], P[7], P[8], 2, 64,
                           512, 4, 2, 1, L.TP_BF16, P[9], big, None) == L.TP_ERR_NULL


def test_workspace_sizes(lib):
    ws = lambda *a: lib.tp_workspace_size(*a)
    M, h, f = 2048, 12288, 49152
    assert ws(L.TP_OP_MLP_FWD, M, h, f, 0, 8, L.TP_BF16) >= M * f * 2
    assert ws(L.TP_OP_MLP_BWD, M, h, f, 0, 8, L.TP_BF16) >= 3 * M * f * 2
    assert ws(L.TP_OP_MLP_FWD, M, h, f, 0, 8, L.TP_F32) >= M * f * 4
    assert ws(L.TP_OP_ATTN_FWD, M, h, 0, 96, 8, L.TP_BF16) >= M * 4 * h * 2
    assert ws(L.TP_OP_ATTN_BWD, M, h, 0, 96, 8, L.TP_BF16) >= M * 7 * h * 2
    assert ws(L.TP_OP_MLP_FWD, 0, h, f, 0, 8, L.TP_BF16) == 0
    assert ws(L.TP_OP_ATTN_FWD, M, h, 0, 0, 8, L.TP_BF16) == 0


def test_layernorm_and_block_validation(lib):
    import ctypes as C
    big = 1 << 40
    assert lib.tp_layernorm_fwd(None, None, None, P[1], None, None, 4, 64, 1e-5, L.TP_BF16, None) == L.TP_ERR_NULL
    assert lib.tp_layernorm_fwd(P[0], None, None, P[1], None, None, 4, 60, 1e-5, L.TP_BF16, None) == L.TP_ERR_ALIGN
    assert lib.tp_layernorm_fwd(P[0], None, None, P[1], None, None, 4, 16392, 1e-5, L.TP_BF16, None) == L.TP_ERR_UNSUPPORTED
    assert lib.tp_layernorm_bwd(P[0], None, None, P[2], P[3], None, P[4], None, None, 4, 64, L.TP_BF16, P[9], big, None) == L.TP_ERR_NULL
    assert lib.tp_layernorm_bwd(P[0], None, P[1], P[2], P[3], None, P[4], None, None, 4, 64, L.TP_BF16, None, 0, None) == L.TP_ERR_WORKSPACE
    W = L.BlockWeights(*([None] * 10))
    S = L.BlockSaves(*([P[5]] * 11))
    assert lib.tp_block_fwd(P[0], C.byref(W), P[1], C.byref(S), 1, 64, 512, 2048, 4, 2, 1e-5, L.TP_BF16, P[9], big, None) == L.TP_ERR_NULL
    W = L.BlockWeights(None, None, P[2], P[3], None, None, P[4], None, P[6], None)
    assert lib.tp_block_fwd(P[0], C.byref(W), P[1], C.byref(S), 1, 64, 512, 2047, 4, 2, 1e-5, L.TP_BF16, P[9], big, None) == L.TP_ERR_SHAPE
    S0 = L.BlockSaves(*([P[5]] * 10 + [None]))
    assert lib.tp_block_fwd(P[0], C.byref(W), P[1], C.byref(S0), 1, 64, 512, 2048, 4, 2, 1e-5, L.TP_BF16, P[9], big, None) == L.TP_ERR_NULL
    assert lib.tp_block_fwd(P[0], C.byref(W), P[1], C.byref(S), 1, 64, 512, 2048, 4, 2, 1e-5, L.TP_F32, P[9], big, None) == L.TP_ERR_UNSUPPORTED
    assert lib.tp_workspace_size(L.TP_OP_BLOCK_BWD, 2048, 12288, 49152, 96, 8, L.TP_BF16) > 3 * 2048 * 12288 * 2
    assert lib.tp_workspace_size(L.TP_OP_LN_BWD, 2048, 12288, 0, 0, 1, L.TP_BF16) >= 2 * 64 * 12288 * 4


def test_vocab_validation(lib):
    """Vocabulary-parallel embedding and cross-entropy ("图解Transformer并行计算"
    §4.1, §4.2): E's rows split over t shards, so V % t must be 0."""
    big = 1 << 40
    bf, f32 = L.TP_BF16, L.TP_F32
    ef, eb = lib.tp_vocab_embed_fwd, lib.tp_vocab_embed_bwd
    assert ef(None, P[1], P[2], 16, 1024, 64, 4, bf, None) == L.TP_ERR_NULL
    assert ef(P[0], P[1], P[2], 16, 1026, 64, 4, bf, None) == L.TP_ERR_SHAPE   # V % t
    assert ef(P[0], P[1], P[2], -1, 1024, 64, 4, bf, None) == L.TP_ERR_SHAPE
    assert ef(P[0], P[1], P[2], 16, 1024, 60, 4, bf, None) == L.TP_ERR_ALIGN   # h % 8
    assert ef(P[0], P[1] + 8, P[2], 16, 1024, 64, 4, bf, None) == L.TP_ERR_ALIGN
    assert ef(P[0], P[1], P[2], 16, 1024, 64, 0, bf, None) == L.TP_ERR_SHAPE
    assert ef(P[0], P[1], P[2], 16, 1024, 64, 4, 7, None) == L.TP_ERR_DTYPE
    assert ef(P[0], P[1], P[2], 0, 1024, 64, 4, bf, None) == L.TP_OK          # nothing to do
    assert eb(P[0], None, None, P[3], 16, 1024, 64, 4, bf, P[9], big, None) == L.TP_ERR_NULL
    assert eb(P[0], P[1], None, None, 16, 1024, 64, 4, bf, P[9], big, None) == L.TP_ERR_NULL
    assert eb(P[0], P[1], None, P[3], 1 << 28, 1024, 64, 4, bf, P[9], big, None) == L.TP_ERR_SHAPE
    assert eb(P[0], P[1], None, P[3], 16, 1024, 64, 4, bf, None, 0, None) == L.TP_ERR_WORKSPACE
    need_e = lib.tp_workspace_size(L.TP_OP_VOCAB_EMBED_BWD, 16, 64, 1024, 0, 4, bf)
    assert need_e >= 3 * 16 * 4
    assert eb(P[0], P[1], None, P[3], 16, 1024, 64, 4, bf, P[9], need_e - 1, None) == L.TP_ERR_WORKSPACE
    cf, cb = lib.tp_vocab_ce_fwd, lib.tp_vocab_ce_bwd
    ok = (P[0], P[1], P[2], P[3], P[4], P[5], None)
    assert cf(None, *ok[1:], 64, 256, 1024, 4, bf, P[9], big, None) == L.TP_ERR_NULL
    assert cf(P[0], P[1], P[2], P[3], None, P[5], None, 64, 256, 1024, 4, bf, P[9], big, None) == L.TP_ERR_NULL
    assert cf(*ok, 64, 256, 1024, 4, f32, P[9], big, None) == L.TP_ERR_DTYPE  # bf16 only
    assert cf(*ok, 64, 256, 1004, 8, bf, P[9], big, None) == L.TP_ERR_SHAPE   # V % t
    assert cf(*ok, 64, 256, 1028, 4, bf, P[9], big, None) == L.TP_ERR_ALIGN   # (V/t) % 8
    assert cf(*ok, 64, 256, 1024, 4, bf, None, 0, None) == L.TP_ERR_WORKSPACE
    need = lib.tp_workspace_size(L.TP_OP_VOCAB_CE_FWD, 64, 256, 1024, 0, 4, bf)
    assert need >= 64 * 1024 // 32 * 8 + 64 * 4
    assert cf(*ok, 64, 256, 1024, 4, bf, P[9], need - 1, None) == L.TP_ERR_WORKSPACE
    assert lib.tp_workspace_size(L.TP_OP_VOCAB_CE_FWD, 64, 256, 1026, 0, 4, bf) == 0
    assert cb(P[0], P[1], P[2], None, P[4], None, P[6], P[7], P[8], 64, 256, 1024, 4, bf, None) == L.TP_ERR_NULL
    assert cb(P[0], P[1], P[2], P[3], P[4], None, None, P[7], P[8], 64, 256, 1024, 4, bf, None) == L.TP_ERR_NULL
    assert cb(P[0], P[1], P[2], P[3], P[4], None, P[6], P[7], P[8], 64, 256, 1024, 4, f32, None) == L.TP_ERR_DTYPE


def test_selftest_limit_validation(lib):
    assert lib.tp_selftest_bounded_wait(999, None) == L.TP_ERR_SHAPE
    assert lib.tp_selftest_bounded_wait(2_000_000_001, None) == L.TP_ERR_SHAPE


def test_absurd_sizes_are_rejected_before_any_product_overflows(lib):
    big = 1 << 40
    huge = 1 << 32
    assert lib.tp_workspace_size(L.TP_OP_MLP_FWD, huge, 512, huge, 0, 8, L.TP_BF16) == 0
    assert lib.tp_mlp_fwd(P[0], P[1], None, P[2], None, P[3], None, huge, 512, huge, 8,
                          L.TP_BF16, P[9], big, None) == L.TP_ERR_SHAPE
    assert lib.tp_linear_col(P[0], P[1], None, P[2], huge, 512, 512, 1, -1, L.TP_BF16,
                             L.TP_BF16, None) == L.TP_ERR_SHAPE
    assert lib.tp_attn_fwd(P[0], P[1], P[2], P[3], None, None, None, huge, huge, 512, 4, 2, 1,
                           L.TP_BF16, P[9], big, None) == L.TP_ERR_SHAPE


@pytest.mark.parametrize("M,f", [(1 << 32, 1 << 32), (4096, 8200), (1, (1 << 25) + 8)])
def test_noalloc_rejects_sizes_beyond_its_array_on_the_host(lib, M, f):
    # 2^32 x 2^32 would wrap a 64-bit byte count; the others are just past
    # the 64 MiB limit on H (bf16).  All are rejected before any CUDA call.
    assert lib.tp_mlp_fwd_noalloc(P[0], P[1], None, P[2], None, P[3], None, M, 512, f, 8,
                                  L.TP_BF16, None) == L.TP_ERR_SHAPE
    assert b"64 MiB" in lib.tp_last_error()
