"""The scratch-free W4A16 entry point, moe_w4a16_forward_noalloc.

Some callers cannot allocate device memory where they run the layer (a plugin or custom-op host
that only hands over its input and output buffers, a serving runtime that plans all device memory
at start-up). For them the library keeps the layer's scratch in a built-in static device array.
These tests call that entry point through the C ABI and check it bit for bit against
moe_w4a16_forward (which takes a caller workspace) on the same inputs, for two calls in a row with
different inputs, so a call cannot lean on what the previous one left in the shared array; the
first call is also checked against the oracle. Both schedules run: the register-fed decode
schedule and the tensor-core schedule. This file is collected last
and needs nothing from the other test files."""
import numpy as np
import pytest
import torch

import quantized_mixture_experts_align_b200 as moeq
import workloads as W
from tests._util import TOL_W4A16, assert_layer_close, bf16_to_f64, oracle_layer

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _two_calls(d, want_oracle_tokens):
    """Two calls in a row with different inputs through the scratch-free entry point, each equal
    bit for bit to moe_w4a16_forward with a caller workspace (the same kernels on the same inputs),
    the first also checked against the oracle. The output buffers are allocated up front, so the
    calls themselves must not change the device memory torch has allocated."""
    T, E, k, H = d["T"], d["E"], d["k"], d["H"]
    weights = (d["w13q"], d["w13s"], d["w2q"], d["w2s"])
    g = torch.Generator(device=DEV).manual_seed(1234)
    inputs = [(d["x"], d["logits"]),
              (torch.randn(d["x"].shape, device=DEV, generator=g).to(torch.bfloat16),
               torch.randn(d["logits"].shape, device=DEV, generator=g))]
    for call, (x, logits) in enumerate(inputs):
        ref_ids = torch.empty((T, k), dtype=torch.int32, device=DEV)
        ref = moeq.moe_w4a16_forward(x, logits, k, *weights, topk_ids_out=ref_ids)
        ids = torch.full((T, k), -1, dtype=torch.int32, device=DEV)
        out = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device=DEV)
        torch.cuda.synchronize()
        before = torch.cuda.memory_allocated(DEV)
        moeq.moe_w4a16_forward_noalloc(x, logits, k, *weights, out=out, topk_ids_out=ids)
        torch.cuda.synchronize()
        assert torch.cuda.memory_allocated(DEV) == before, f"call {call}: device memory was allocated"
        assert torch.equal(ids, ref_ids), f"call {call}: routing differs"
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), f"call {call}: output differs"
        if call == 0:
            toks = np.asarray(want_oracle_tokens, np.int32)
            assert_layer_close(bf16_to_f64(out[torch.as_tensor(toks, device=DEV).long()]), oracle_layer(d, toks),
                               TOL_W4A16, "noalloc vs oracle")
    assert moeq.moe_device_status() == 0


def test_noalloc_forward_decode_schedule_two_calls():
    """Decode shapes (T = 32, E = 384): the register-fed schedule."""
    d = W.make_moe(W.WORKLOADS["decode_w4a16"], device=DEV)
    _two_calls(d, np.arange(d["T"], dtype=np.int32))


def test_noalloc_forward_tensor_core_schedule_two_calls():
    """T * k / E >= 16 rows per expert: the tensor-core schedule (256-row expert blocks, the
    activation gather, the few-row blocks on the register-fed kernel, the device status word),
    at a size whose workspace fits the built-in scratch."""
    d = W.make_moe(W.WORKLOADS["tiny_w4a16"], device=DEV, T=300, E=8, k=2, H=512, I=256)
    assert moeq.moe_w4a16_workspace_size(300, 512, 256, 8, 2) <= 16 << 20
    _two_calls(d, np.arange(d["T"], dtype=np.int32))


def test_noalloc_rejects_shapes_beyond_its_scratch():
    H, I, E, k = 7168, 2048, 384, 8
    assert moeq.moe_w4a16_workspace_size(103, H, I, E, k) <= 16 << 20 < moeq.moe_w4a16_workspace_size(104, H, I, E, k)
    x = torch.zeros((104, H), dtype=torch.bfloat16, device=DEV)
    logits = torch.zeros((104, E), device=DEV)
    # rejected before any device work, so the weight contents do not matter
    w13q = torch.empty((E, 2 * I, H // 8), dtype=torch.int32, device=DEV)
    w13s = torch.empty((E, 2 * I, H // 32), dtype=torch.bfloat16, device=DEV)
    w2q = torch.empty((E, H, I // 8), dtype=torch.int32, device=DEV)
    w2s = torch.empty((E, H, I // 32), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(moeq.MoeqError) as ei:
        moeq.moe_w4a16_forward_noalloc(x, logits, k, w13q, w13s, w2q, w2s)
    assert ei.value.code == moeq.MOEQ_ERR_WORKSPACE
    assert "built-in" in str(ei.value)
