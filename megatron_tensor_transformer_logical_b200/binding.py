"""Python binding of libtp: argument marshalling only.

Each function has the name of the C entry point it calls (see
include/libtp.h), takes torch CUDA tensors (PyTorch supplies device memory
and streams; nothing is computed here), derives the sizes from their shapes,
passes raw device pointers, and raises TPError on a non-OK status.  There is
no fallback: if libtp.so is missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtp.so")

TP_OK, TP_ERR_NULL, TP_ERR_SHAPE, TP_ERR_ALIGN, TP_ERR_DTYPE = 0, 1, 2, 3, 4
TP_ERR_UNSUPPORTED, TP_ERR_CUDA, TP_ERR_KERNEL, TP_ERR_WORKSPACE = 5, 6, 7, 8
TP_F32, TP_BF16 = 0, 1
TP_OP_MLP_FWD, TP_OP_MLP_BWD, TP_OP_ATTN_FWD, TP_OP_ATTN_BWD = 0, 1, 2, 3
TP_OP_LN_BWD, TP_OP_BLOCK_FWD, TP_OP_BLOCK_BWD, TP_OP_VOCAB_CE_FWD = 4, 5, 6, 7
TP_OP_VOCAB_EMBED_BWD = 8

(TP_KIND_GEMM_TCGEN05, TP_KIND_GEMM_SIMT, TP_KIND_ATTN_FWD, TP_KIND_ATTN_BWD, TP_KIND_REDUCE,
 TP_KIND_VOCAB) = range(6)
KIND_NAMES = {TP_KIND_GEMM_TCGEN05: "gemm_tcgen05", TP_KIND_GEMM_SIMT: "gemm_simt",
              TP_KIND_ATTN_FWD: "attn_fwd", TP_KIND_ATTN_BWD: "attn_bwd", TP_KIND_REDUCE: "reduce",
              TP_KIND_VOCAB: "vocab"}

EXPORTS = ("tp_linear_col", "tp_linear_row", "tp_mlp_fwd", "tp_mlp_bwd", "tp_attn_fwd",
           "tp_attn_bwd", "tp_workspace_size", "tp_last_error", "tp_device_status",
           "tp_version", "tp_profile_enable", "tp_profile_read", "tp_launch_count",
           "tp_mlp_fwd_noalloc", "tp_profile_count", "tp_profile_record", "tp_layernorm_fwd",
           "tp_layernorm_bwd", "tp_block_fwd", "tp_block_bwd", "tp_vocab_embed_fwd",
           "tp_vocab_embed_bwd", "tp_vocab_ce_fwd", "tp_vocab_ce_bwd", "tp_gemm_plan",
           "tp_selftest_bounded_wait")

_W_FIELDS = ("ln1_g", "ln1_b", "Wqkv", "Wo", "ln2_g", "ln2_b", "A", "bA", "B", "bB")
_S_FIELDS = ("Xn1", "mean1", "rstd1", "QKV", "O", "LSE", "X1", "Xn2", "mean2", "rstd2", "Y")
_G_FIELDS = ("dln1_g", "dln1_b", "dWqkv", "dWo", "dln2_g", "dln2_b", "dA", "dbA", "dB", "dbB")


class BlockWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _W_FIELDS]


class BlockSaves(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _S_FIELDS]


class BlockGrads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _G_FIELDS]


class LaunchRecord(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("tile", ctypes.c_int), ("m", ctypes.c_int64),
                ("n", ctypes.c_int64), ("k", ctypes.c_int64), ("ms", ctypes.c_double),
                ("flops", ctypes.c_double), ("bytes", ctypes.c_double)]


class GemmUnit(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("m0", "rows", "n0", "n_end", "kb0", "kb1", "part",
                                              "tile")]


class ProfileStats(ctypes.Structure):
    _fields_ = [("launches", ctypes.c_int64), ("total_ms", ctypes.c_double),
                ("flops", ctypes.c_double), ("bytes", ctypes.c_double)]


class TPError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"libtp status {status}: {msg}")
        self.status = status


_lib = None


def load() -> ctypes.CDLL:
    """Loads libtp.so once and declares its signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is not built: run "
                           "`python -m megatron_tensor_transformer_logical_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    L.tp_linear_col.argtypes = [vp, vp, vp, vp, i64, i64, i64, i32, i32, i32, i32, vp]
    L.tp_linear_row.argtypes = [vp, vp, vp, vp, i64, i64, i64, i32, i32, i32, i32, vp]
    L.tp_mlp_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i32, i32, vp, sz, vp]
    L.tp_mlp_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i32, i32, vp]
    L.tp_mlp_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i32,
                             i32, vp, sz, vp]
    L.tp_attn_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i32, i32, i32, i32,
                              vp, sz, vp]
    L.tp_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i32, i32,
                              i32, i32, vp, sz, vp]
    f32 = ctypes.c_float
    L.tp_layernorm_fwd.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, f32, i32, vp]
    L.tp_layernorm_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i32, vp, sz, vp]
    L.tp_block_fwd.argtypes = [vp, ctypes.POINTER(BlockWeights), vp, ctypes.POINTER(BlockSaves),
                               i64, i64, i64, i64, i32, i32, f32, i32, vp, sz, vp]
    L.tp_block_bwd.argtypes = [vp, ctypes.POINTER(BlockWeights), ctypes.POINTER(BlockSaves), vp,
                               vp, ctypes.POINTER(BlockGrads), i64, i64, i64, i64, i32, i32, f32,
                               i32, vp, sz, vp]
    L.tp_vocab_embed_fwd.argtypes = [vp, vp, vp, i64, i64, i64, i32, i32, vp]
    L.tp_vocab_embed_bwd.argtypes = [vp, vp, vp, vp, i64, i64, i64, i32, i32, vp, sz, vp]
    L.tp_vocab_ce_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i32, i32, vp, sz, vp]
    L.tp_vocab_ce_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i32, i32,
                                  vp]
    L.tp_workspace_size.argtypes = [i32, i64, i64, i64, i32, i32, i32]
    L.tp_workspace_size.restype = sz
    L.tp_last_error.argtypes = []
    L.tp_last_error.restype = ctypes.c_char_p
    L.tp_device_status.argtypes = [vp]
    L.tp_selftest_bounded_wait.argtypes = [i64, vp]
    L.tp_version.argtypes = []
    L.tp_profile_enable.argtypes = [i32]
    L.tp_profile_read.argtypes = [i32, ctypes.POINTER(ProfileStats)]
    L.tp_launch_count.argtypes = []
    L.tp_profile_count.argtypes = []
    L.tp_profile_count.restype = ctypes.c_int64
    L.tp_profile_record.argtypes = [ctypes.c_int64, ctypes.POINTER(LaunchRecord)]
    L.tp_gemm_plan.argtypes = [i64, i64, i64, i64, i32, i32, i32, ctypes.POINTER(GemmUnit), i64]
    for name in EXPORTS:
        if name not in ("tp_workspace_size", "tp_last_error", "tp_launch_count",
                        "tp_profile_count", "tp_gemm_plan"):
            getattr(L, name).restype = ctypes.c_int
    L.tp_launch_count.restype = ctypes.c_int64
    L.tp_gemm_plan.restype = ctypes.c_int64
    _lib = L
    return L


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("libtp takes dense row-major (contiguous) tensors")
    return t.data_ptr()


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return TP_BF16
    if t.dtype == torch.float32:
        return TP_F32
    raise ValueError(f"unsupported dtype {t.dtype}")


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _check(status: int) -> None:
    if status != TP_OK:
        raise TPError(status, load().tp_last_error().decode(errors="replace"))


def tp_linear_col(X, W, bias, Y, t: int, shard: int = -1, stream=None) -> None:
    M, K = X.shape
    N = W.shape[1]
    _check(load().tp_linear_col(_ptr(X), _ptr(W), _ptr(bias), _ptr(Y), M, K, N, t, shard,
                                _dtype(X), _dtype(Y), _stream(stream)))


def tp_linear_row(X, W, bias, Z, t: int, shard: int = -1, stream=None) -> None:
    M, K = X.shape
    N = W.shape[1]
    _check(load().tp_linear_row(_ptr(X), _ptr(W), _ptr(bias), _ptr(Z), M, K, N, t, shard,
                                _dtype(X), _dtype(Z), _stream(stream)))


def tp_workspace_size(op: int, M: int, h: int, f: int, heads: int, t: int, dtype: int) -> int:
    return int(load().tp_workspace_size(op, M, h, f, heads, t, dtype))


def tp_mlp_fwd(X, A, bA, B, bB, Z, Ysave, t: int, ws, stream=None) -> None:
    M, h = X.shape
    f = A.shape[1]
    _check(load().tp_mlp_fwd(_ptr(X), _ptr(A), _ptr(bA), _ptr(B), _ptr(bB), _ptr(Z),
                             _ptr(Ysave), M, h, f, t, _dtype(X), _ptr(ws),
                             ws.numel() * ws.element_size(), _stream(stream)))


def tp_mlp_fwd_noalloc(X, A, bA, B, bB, Z, Ysave, t: int, stream=None) -> None:
    """tp_mlp_fwd with its intermediate in libtp's fixed 64 MiB device array:
    for callers that cannot allocate a workspace (see include/libtp.h)."""
    M, h = X.shape
    f = A.shape[1]
    _check(load().tp_mlp_fwd_noalloc(_ptr(X), _ptr(A), _ptr(bA), _ptr(B), _ptr(bB), _ptr(Z),
                                     _ptr(Ysave), M, h, f, t, _dtype(X), _stream(stream)))


def tp_mlp_bwd(X, A, bA, B, Ysave, dZ, dX, dA, dbA, dB, dbB, t: int, ws, stream=None) -> None:
    M, h = X.shape
    f = A.shape[1]
    _check(load().tp_mlp_bwd(_ptr(X), _ptr(A), _ptr(bA), _ptr(B), _ptr(Ysave), _ptr(dZ),
                             _ptr(dX), _ptr(dA), _ptr(dbA), _ptr(dB), _ptr(dbB), M, h, f, t,
                             _dtype(X), _ptr(ws), ws.numel() * ws.element_size(),
                             _stream(stream)))


def tp_attn_fwd(X, Wqkv, Wo, Z, QKVsave, Osave, LSEsave, b: int, s: int, heads: int, t: int,
                causal: bool, ws, stream=None) -> None:
    h = X.shape[1]
    _check(load().tp_attn_fwd(_ptr(X), _ptr(Wqkv), _ptr(Wo), _ptr(Z), _ptr(QKVsave),
                              _ptr(Osave), _ptr(LSEsave), b, s, h, heads, t, int(causal),
                              _dtype(X), _ptr(ws), ws.numel() * ws.element_size(),
                              _stream(stream)))


def tp_attn_bwd(X, Wqkv, Wo, QKVsave, Osave, LSEsave, dZ, dX, dWqkv, dWo, b: int, s: int,
                heads: int, t: int, causal: bool, ws, stream=None) -> None:
    h = X.shape[1]
    _check(load().tp_attn_bwd(_ptr(X), _ptr(Wqkv), _ptr(Wo), _ptr(QKVsave), _ptr(Osave),
                              _ptr(LSEsave), _ptr(dZ), _ptr(dX), _ptr(dWqkv), _ptr(dWo), b, s,
                              h, heads, t, int(causal), _dtype(X), _ptr(ws),
                              ws.numel() * ws.element_size(), _stream(stream)))


def tp_layernorm_fwd(X, gamma, beta, Y, mean, rstd, eps: float = 1e-5, stream=None) -> None:
    M, h = X.shape
    _check(load().tp_layernorm_fwd(_ptr(X), _ptr(gamma), _ptr(beta), _ptr(Y), _ptr(mean),
                                   _ptr(rstd), M, h, eps, _dtype(X), _stream(stream)))


def tp_layernorm_bwd(X, gamma, mean, rstd, dY, dR, dX, dgamma, dbeta, ws, stream=None) -> None:
    M, h = X.shape
    _check(load().tp_layernorm_bwd(_ptr(X), _ptr(gamma), _ptr(mean), _ptr(rstd), _ptr(dY),
                                   _ptr(dR), _ptr(dX), _ptr(dgamma), _ptr(dbeta), M, h, _dtype(X),
                                   _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def _struct(cls, fields, d):
    return cls(*[_ptr(d.get(n)) for n in fields])


def tp_block_fwd(X, w: dict, X2, saves: dict, b: int, s: int, f: int, heads: int, t: int,
                 eps: float, ws, stream=None) -> None:
    """w: dict of the tp_block_weights fields; saves: dict of tp_block_saves fields."""
    h = X.shape[1]
    W, S = _struct(BlockWeights, _W_FIELDS, w), _struct(BlockSaves, _S_FIELDS, saves)
    _check(load().tp_block_fwd(_ptr(X), ctypes.byref(W), _ptr(X2), ctypes.byref(S), b, s, h, f,
                               heads, t, eps, _dtype(X), _ptr(ws), ws.numel() * ws.element_size(),
                               _stream(stream)))


def tp_block_bwd(X, w: dict, saves: dict, dX2, dX, grads: dict, b: int, s: int, f: int,
                 heads: int, t: int, eps: float, ws, stream=None) -> None:
    h = X.shape[1]
    W, S = _struct(BlockWeights, _W_FIELDS, w), _struct(BlockSaves, _S_FIELDS, saves)
    G = _struct(BlockGrads, _G_FIELDS, grads)
    _check(load().tp_block_bwd(_ptr(X), ctypes.byref(W), ctypes.byref(S), _ptr(dX2), _ptr(dX),
                               ctypes.byref(G), b, s, h, f, heads, t, eps, _dtype(X), _ptr(ws),
                               ws.numel() * ws.element_size(), _stream(stream)))


def _ids(t: torch.Tensor) -> int:
    if t.dtype != torch.int32:
        raise ValueError("token ids and targets are int32")
    return _ptr(t)


def tp_vocab_embed_fwd(ids, E, Y, t: int, stream=None) -> None:
    """Y[r] = E[ids[r]] (zero for ids outside [0, V)); ids int32 [M]."""
    V, h = E.shape
    _check(load().tp_vocab_embed_fwd(_ids(ids), _ptr(E), _ptr(Y), ids.numel(), V, h, t,
                                     _dtype(E), _stream(stream)))


def tp_vocab_embed_bwd(ids, dY, dE_in, dE, t: int, ws, stream=None) -> None:
    """dE = scatter-add of dY rows by id (+ dE_in, which may be dE)."""
    V, h = dE.shape
    _check(load().tp_vocab_embed_bwd(_ids(ids), _ptr(dY), _ptr(dE_in), _ptr(dE), ids.numel(), V,
                                     h, t, _dtype(dE), _ptr(ws),
                                     0 if ws is None else ws.numel() * ws.element_size(),
                                     _stream(stream)))


def tp_vocab_ce_fwd(X, E, targets, logits, lse, loss, total, t: int, ws, stream=None) -> None:
    M, h = X.shape
    V = E.shape[0]
    _check(load().tp_vocab_ce_fwd(_ptr(X), _ptr(E), _ids(targets), _ptr(logits), _ptr(lse),
                                  _ptr(loss), _ptr(total), M, h, V, t, _dtype(X), _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream(stream)))


def tp_vocab_ce_bwd(X, E, targets, logits, lse, dloss, dlogits, dX, dE, t: int,
                    stream=None) -> None:
    M, h = X.shape
    V = E.shape[0]
    _check(load().tp_vocab_ce_bwd(_ptr(X), _ptr(E), _ids(targets), _ptr(logits), _ptr(lse),
                                  _ptr(dloss), _ptr(dlogits), _ptr(dX), _ptr(dE), M, h, V, t,
                                  _dtype(X), _stream(stream)))


def tp_device_status(stream=None) -> None:
    _check(load().tp_device_status(_stream(stream)))


def tp_selftest_bounded_wait(limit_ns: int, stream=None) -> None:
    _check(load().tp_selftest_bounded_wait(int(limit_ns), _stream(stream)))


def tp_version() -> int:
    return int(load().tp_version())


def tp_profile_enable(on: bool) -> None:
    _check(load().tp_profile_enable(1 if on else 0))


def tp_profile_read(kind: int) -> dict:
    st = ProfileStats()
    _check(load().tp_profile_read(kind, ctypes.byref(st)))
    return {"launches": st.launches, "total_ms": st.total_ms, "flops": st.flops, "bytes": st.bytes}


def tp_launch_count() -> int:
    return int(load().tp_launch_count())


def tp_profile_records() -> list:
    """Every launch recorded since profiling was turned on, as dicts."""
    L = load()
    out = []
    for i in range(int(L.tp_profile_count())):
        r = LaunchRecord()
        _check(L.tp_profile_record(i, ctypes.byref(r)))
        out.append({"kind": KIND_NAMES.get(r.kind, str(r.kind)), "tile": r.tile, "m": r.m,
                    "n": r.n, "k": r.k, "ms": r.ms, "flops": r.flops, "bytes": r.bytes})
    return out


def tp_gemm_plan(M: int, N: int, K: int, n_shard: int, kind: int, sms: int,
                 tail_scratch: bool) -> list:
    """The tensor-core GEMM's work units for one shape (host only), as dicts
    with m0, rows, n0, n_end, kb0, kb1, part, tile; raises on bad sizes."""
    L = load()
    n = int(L.tp_gemm_plan(M, N, K, n_shard, kind, sms, int(tail_scratch), None, 0))
    if n < 0:
        raise TPError(TP_ERR_SHAPE, "invalid GEMM plan request")
    buf = (GemmUnit * max(n, 1))()
    got = int(L.tp_gemm_plan(M, N, K, n_shard, kind, sms, int(tail_scratch), buf, n))
    assert got == n
    return [{f: getattr(buf[i], f) for f, _ in GemmUnit._fields_} for i in range(n)]


def workspace(op: int, M: int, h: int, f: int, heads: int, t: int, dtype: int,
              device="cuda") -> torch.Tensor:
    """A byte tensor of tp_workspace_size() bytes on `device`."""
    n = tp_workspace_size(op, M, h, f, heads, t, dtype)
    if n == 0:
        raise TPError(TP_ERR_SHAPE, "invalid sizes for the workspace query")
    return torch.empty(n, dtype=torch.uint8, device=device)
