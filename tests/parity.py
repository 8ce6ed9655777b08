"""Shared helpers for the GPU parity tests: tolerances and comparisons.

Tolerances (max-rel is scaled by the reference tensor's largest magnitude,
normwise is the ratio of 2-norms):
  fp32 path:  max-rel <= 1e-5
  bf16 path:  max-rel <= 2e-2 and normwise <= 5e-3 (bf16 inputs, fp32 accumulation)
"""
import numpy as np
import pytest
import torch

from oracle import tp_oracle as O

F32_MAX_REL = 1e-5
BF16_MAX_REL = 2e-2
BF16_NORMWISE = 5e-3


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def to64(t) -> np.ndarray:
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().float().cpu().double().numpy()


def check(got, ref, what: str, dtype: str):
    got, ref = to64(got), to64(ref)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    mr = O.max_rel_error(got, ref)
    if dtype == "f32":
        assert mr <= F32_MAX_REL, f"{what}: max-rel {mr:.3e} > {F32_MAX_REL}"
    else:
        nw = O.normwise_error(got, ref)
        assert mr <= BF16_MAX_REL and nw <= BF16_NORMWISE, \
            f"{what}: max-rel {mr:.3e} (<= {BF16_MAX_REL}), normwise {nw:.3e} (<= {BF16_NORMWISE})"
    return mr


def cuda(t, dtype=None):
    if t is None:
        return None
    t = t.to("cuda")
    return t.to(dtype) if dtype is not None else t
