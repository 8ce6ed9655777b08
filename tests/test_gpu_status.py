"""The device status: a flag or a timeout recorded by one launch must not
change the results of later launches, and a bounded wait that runs out must
be reported, with the kernel returning normally.

Failure detection here makes no GPU fault: the bounded-wait self-test kernel
waits on an mbarrier that nothing completes, with a 1 ms limit, and returns.

Pages: "图解Transformer并行计算" §2.1-§2.2 (the MLP) and §3.2 (attention
forward steps 1-3 and the backward), which the parity checks after each event
compare against.
"""
import time

import pytest
import torch

from megatron_tensor_transformer_logical_b200 import binding as L
from megatron_tensor_transformer_logical_b200.inputs import (Workload, make_attn_inputs,
                                                             make_mlp_inputs)
from tests.parity import cuda, need_gpu
from tests.test_gpu_attention import compare_full as compare_attn
from tests.test_gpu_attention import gpu_attn
from tests.test_gpu_mlp import compare_full as compare_mlp
from tests.test_gpu_mlp import gpu_mlp

pytestmark = pytest.mark.gpu

ATTN = Workload(84, "attn after event", b=2, s=520, h=512, heads=4, t=2, w_std=0.05)
MLP = Workload(85, "mlp after event", b=2, s=300, h=512, f=2048, t=4, w_std=0.05, bias_std=0.05)


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()
    try:
        L.tp_device_status()  # start from a clear status
    except L.TPError:
        pass
    yield
    try:
        L.tp_device_status()
    except L.TPError:
        pass


def _saturating_attention():
    """An attention forward whose QKV (256 * 2 * 256 per entry) exceeds the
    fp16 range: its epilogue saturates and sets the fp16 flag."""
    wl = Workload(83, "attn overflow", b=1, s=64, h=256, heads=2, t=1, w_std=0.05)
    inp = make_attn_inputs(wl)
    inp["X"] = torch.full_like(inp["X"], 256.0)
    inp["Wqkv"] = torch.full_like(inp["Wqkv"], 2.0)
    d = {k: cuda(v) for k, v in inp.items()}
    M, h = wl.M, wl.h
    Z = torch.empty(M, h, dtype=torch.bfloat16, device="cuda")
    QKV = torch.empty(M, 3 * h, dtype=torch.float16, device="cuda")
    L.tp_attn_fwd(d["X"], d["Wqkv"], d["Wo"], Z, QKV, None, None, wl.b, wl.s, wl.heads, 1, True,
                  L.workspace(L.TP_OP_ATTN_FWD, M, h, 0, wl.heads, 1, L.TP_BF16))
    torch.cuda.synchronize()
    assert QKV.float().max().item() == 65504.0


def _layer_parity_without_reading_status():
    """Attention fwd+bwd and MLP fwd+bwd against the oracle, with the status
    left as it is (nothing reads or clears it in between)."""
    ai = make_attn_inputs(ATTN)
    compare_attn(gpu_attn(ai, ATTN), ai, ATTN, True)
    mi = make_mlp_inputs(MLP)
    compare_mlp(gpu_mlp(mi, MLP.t), mi, "bf16")


def test_saturation_flag_does_not_stop_later_calls():
    _saturating_attention()
    _layer_parity_without_reading_status()
    with pytest.raises(L.TPError) as e:
        L.tp_device_status()
    assert e.value.status == L.TP_ERR_KERNEL and "fp16" in str(e.value)
    L.tp_device_status()  # read once, then clear


def test_bounded_wait_expires_and_is_reported():
    t0 = time.perf_counter()
    L.tp_selftest_bounded_wait(1_000_000)  # 1 ms
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    # The second warp's wait has the default 2 s limit; it returns this soon
    # only because the first warp's timeout aborts the launch's other waits.
    assert elapsed < 1.0, elapsed
    with pytest.raises(L.TPError) as e:
        L.tp_device_status()
    assert e.value.status == L.TP_ERR_KERNEL and "self-test" in str(e.value)
    L.tp_device_status()  # cleared by the read


def test_stale_timeout_does_not_stop_later_calls():
    L.tp_selftest_bounded_wait(1_000_000)
    _layer_parity_without_reading_status()
    with pytest.raises(L.TPError) as e:
        L.tp_device_status()
    assert e.value.status == L.TP_ERR_KERNEL and "self-test" in str(e.value)
    L.tp_device_status()


def test_timeout_and_flag_reported_together():
    L.tp_selftest_bounded_wait(1_000_000)
    _saturating_attention()
    with pytest.raises(L.TPError) as e:
        L.tp_device_status()
    msg = str(e.value)
    assert e.value.status == L.TP_ERR_KERNEL and "self-test" in msg and "fp16" in msg
    L.tp_device_status()
