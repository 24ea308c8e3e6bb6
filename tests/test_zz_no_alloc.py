"""The scratch-free W4A16 entry point, moe_w4a16_forward_noalloc.

Some callers cannot allocate device memory where they run the layer (a plugin or custom-op host
that only hands over its input and output buffers, a serving runtime that plans all device memory
at start-up). For them the library keeps the layer's scratch in a built-in static device array.
These tests call that entry point through the C ABI and check it against moe_w4a16_forward (which
takes a caller workspace) on the same inputs, for two calls in a row with different inputs, so a
call cannot lean on what the previous one left in the shared array. This file is collected last
and needs nothing from the other test files."""
import numpy as np
import pytest
import torch

import quantized_mixture_experts_align_b200 as moeq
import workloads as W
from tests._util import TOL_W4A16, assert_layer_close, bf16_to_f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def test_noalloc_forward_matches_workspace_forward_on_two_calls():
    d = W.make_moe(W.WORKLOADS["decode_w4a16"], device=DEV)
    T, E, k = d["T"], d["E"], d["k"]
    weights = (d["w13q"], d["w13s"], d["w2q"], d["w2s"])
    g = torch.Generator(device=DEV).manual_seed(1234)
    inputs = [(d["x"], d["logits"]),
              (torch.randn(d["x"].shape, device=DEV, generator=g).to(torch.bfloat16),
               torch.randn(d["logits"].shape, device=DEV, generator=g))]
    for call, (x, logits) in enumerate(inputs):
        ref_ids = torch.empty((T, k), dtype=torch.int32, device=DEV)
        ref = moeq.moe_w4a16_forward(x, logits, k, *weights, topk_ids_out=ref_ids)
        ids = torch.full((T, k), -1, dtype=torch.int32, device=DEV)
        out = moeq.moe_w4a16_forward_noalloc(x, logits, k, *weights, topk_ids_out=ids)
        torch.cuda.synchronize()
        assert torch.equal(ids, ref_ids), f"call {call}: routing differs"
        assert_layer_close(bf16_to_f64(out), bf16_to_f64(ref), TOL_W4A16, f"noalloc call {call}")


def test_noalloc_rejects_shapes_beyond_its_scratch():
    H, I, E, k = 7168, 2048, 384, 8
    assert moeq.moe_w4a16_workspace_size(113, H, I, E, k) <= 16 << 20 < moeq.moe_w4a16_workspace_size(114, H, I, E, k)
    x = torch.zeros((114, H), dtype=torch.bfloat16, device=DEV)
    logits = torch.zeros((114, E), device=DEV)
    # rejected before any device work, so the weight contents do not matter
    w13q = torch.empty((E, 2 * I, H // 8), dtype=torch.int32, device=DEV)
    w13s = torch.empty((E, 2 * I, H // 32), dtype=torch.bfloat16, device=DEV)
    w2q = torch.empty((E, H, I // 8), dtype=torch.int32, device=DEV)
    w2s = torch.empty((E, H, I // 32), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(moeq.MoeqError) as ei:
        moeq.moe_w4a16_forward_noalloc(x, logits, k, w13q, w13s, w2q, w2s)
    assert ei.value.code == moeq.MOEQ_ERR_WORKSPACE
    assert "built-in" in str(ei.value)
