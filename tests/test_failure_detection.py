"""Failure detection without a GPU fault: the tensor-core kernels' waits are bounded and report
through the device status word. A self-test kernel runs the same bounded wait on a barrier that
nothing arrives at; the status must read MOEQ_ERR_DEVICE_TIMEOUT, clear on request, and the
context must stay usable (a layer forward still matches the oracle afterwards)."""
import numpy as np
import pytest
import torch

import quantized_mixture_experts_align_b200 as moeq
import workloads as W
from tests._util import TOL_W4A16, assert_layer_close, bf16_to_f64, oracle_layer

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    assert torch.cuda.is_available()
    assert moeq.moe_device_status(clear=True) == moeq.MOEQ_OK
    moeq.moe_selftest_bounded_wait()
    torch.cuda.synchronize()
    assert moeq.moe_device_status() == moeq.MOEQ_ERR_DEVICE_TIMEOUT
    assert moeq.moe_device_status(clear=True) == moeq.MOEQ_ERR_DEVICE_TIMEOUT   # read, then cleared
    assert moeq.moe_device_status() == moeq.MOEQ_OK
    d = W.make_moe(W.WORKLOADS["tiny_w4a16"], device="cuda:0")
    out = moeq.moe_w4a16_forward(d["x"], d["logits"], d["k"], d["w13q"], d["w13s"], d["w2q"], d["w2s"])
    torch.cuda.synchronize()
    assert_layer_close(bf16_to_f64(out), oracle_layer(d, np.arange(d["T"], dtype=np.int32)), TOL_W4A16, "after")
    assert moeq.moe_device_status() == moeq.MOEQ_OK
