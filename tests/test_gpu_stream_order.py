"""Stream order toward the caller with programmatic dependent launches inside the library: layers
chained on one stream with no synchronization (each reading the previous one's output), followed
by an ordinary torch kernel, give the same bytes as the same calls with a synchronize between
each."""
import pytest
import torch

import quantized_mixture_experts_align_b200 as moeq
import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.mark.parametrize("T", [32, 600])   # register-fed chain (programmatic launches) / tensor-core schedule
def test_chained_layers_keep_stream_order(T):
    d = W.make_moe(W.WORKLOADS["decode_w4a16"], device=DEV, T=T, E=64)
    w = (d["w13q"], d["w13s"], d["w2q"], d["w2s"])
    k = d["k"]
    # the layer maps [T, H] to [T, H], so its output can feed the next call
    y = d["x"]
    for _ in range(3):
        y = moeq.moe_w4a16_forward(y, d["logits"], k, *w)
    total = y.float().sum(dim=1)            # an ordinary launch right after the chain
    torch.cuda.synchronize()
    r = d["x"]
    for _ in range(3):
        r = moeq.moe_w4a16_forward(r, d["logits"], k, *w)
        torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), r.view(torch.int16))
    assert torch.equal(total, r.float().sum(dim=1))
    assert moeq.moe_device_status() == 0


def test_ep_share_then_reduce_keeps_stream_order():
    """Two expert-parallel shares on one stream into separate outputs, summed by an ordinary torch
    kernel without synchronization: the same as summing after a synchronize."""
    from quantized_mixture_experts_align_b200 import sharding as S
    d = W.make_moe(W.WORKLOADS["decode_w4a16"], device=DEV, T=32, E=64)
    full = {n: d[n] for n in ("w13q", "w13s", "w2q", "w2s")}
    outs = []
    for r in range(2):
        wd, base, _ = S.shard_experts(full, "w4a16", r, 2)
        outs.append(S.forward_ep_partial("w4a16", d["x"], d["logits"], d["k"], wd, base))
    s_async = outs[0].float() + outs[1].float()
    torch.cuda.synchronize()
    assert torch.equal(s_async, outs[0].float() + outs[1].float())
    assert moeq.moe_device_status() == 0
