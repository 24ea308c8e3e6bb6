"""Whole-layer CUDA-graph capture through the C ABI: every entry point is asynchronous on the
caller's stream and makes no host synchronization, so a forward captured into a CUDA graph must
replay to exactly the bytes an eager call writes (the kernels are deterministic), also after the
inputs are overwritten in place between replays; the replay on the new inputs is also checked
against the oracle."""
import numpy as np
import pytest
import torch

import quantized_mixture_experts_align_b200 as moeq
import workloads as W
from tests._util import TOL_FP8, TOL_W4A16, assert_layer_close, bf16_to_f64, oracle_layer

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _capture(fn):
    """Warm up on a side stream (tensor maps, function attributes, lazily loaded kernels), then
    capture one call."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def _layer_case(case):
    if case == "w4a16_decode":  # register-fed schedule (few rows per expert)
        d = W.make_moe(W.WORKLOADS["decode_w4a16"], device=DEV, E=64)
    elif case == "w4a16_tensor_core":  # tcgen05 schedule with a Zipf tail on the register-fed kernel
        d = W.make_moe(W.WORKLOADS["tiny_w4a16"], device=DEV, T=512, E=16, k=4, H=512, I=256)
        d["logits"] = W.router_logits(W.WORKLOADS["prefill_w4a16"], 512, 16, device=DEV)
    else:  # block-FP8 tensor-core schedule
        d = W.make_moe(W.WORKLOADS["moe_fp8"], device=DEV, T=512, E=16, k=4, H=512, I=256)
    return d


@pytest.mark.parametrize("case", ["w4a16_decode", "w4a16_tensor_core", "fp8_tensor_core"])
def test_layer_graph_replay_matches_eager(case):
    d = _layer_case(case)
    T, H = d["x"].shape
    E, k = d["logits"].shape[1], d["k"]
    w4 = d["kind"] == "w4a16"
    I = d["w2q"].shape[2] * 8 if w4 else d["w2"].shape[2]
    need = (moeq.moe_w4a16_workspace_size if w4 else moeq.moe_w8a8_block_fp8_workspace_size)(T, H, I, E, k)
    ws = moeq.workspace(need, DEV)
    out_eager = torch.empty((T, H), dtype=torch.bfloat16, device=DEV)
    out_graph = torch.empty_like(out_eager)
    x_in = d["x"].clone()
    lg_in = d["logits"].clone()

    def fwd(out):
        if w4:
            moeq.moe_w4a16_forward(x_in, lg_in, k, d["w13q"], d["w13s"], d["w2q"], d["w2s"], out=out, ws=ws)
        else:
            moeq.moe_w8a8_block_fp8_forward(x_in, lg_in, k, d["w13"], d["w13s"], d["w2"], d["w2s"], out=out, ws=ws)

    g = _capture(lambda: fwd(out_graph))
    for trial in range(2):
        if trial == 1:  # new inputs in place: the graph reads whatever the buffers hold
            gen = torch.Generator(device=DEV).manual_seed(11)
            x_in.copy_(torch.randn(x_in.shape, device=DEV, generator=gen).to(torch.bfloat16))
            lg_in.copy_(lg_in.flip(0))
        out_graph.zero_()
        g.replay()
        fwd(out_eager)
        torch.cuda.synchronize()
        assert torch.equal(out_graph.view(torch.int16), out_eager.view(torch.int16)), f"{case} trial {trial}"
    # the replay on the inputs written in place, against the oracle on those inputs (tokens
    # sampled from the decode workload, all tokens of the small ones)
    d_new = dict(d, x=x_in, logits=lg_in)
    toks = np.arange(T, dtype=np.int32) if T <= 512 else np.arange(0, T, max(1, T // 16), dtype=np.int32)
    assert_layer_close(bf16_to_f64(out_graph[torch.as_tensor(toks, device=DEV).long()]), oracle_layer(d_new, toks),
                       TOL_W4A16 if w4 else TOL_FP8, f"{case} graph replay vs oracle")
    assert moeq.moe_device_status() == 0


@pytest.mark.parametrize("kind,M,N,K", [
    ("block", 8, 512, 1024),       # swap-AB tiles, K split over a cluster of 8
    ("block", 24, 512, 1024),      # swap-AB tiles, three CTAs per SM, K split over a cluster of 8
    ("block", 100, 512, 1024),     # 128-row tiles, K split over a cluster of 4
    ("block", 512, 8192, 1024),    # 128-row tiles, no split
    ("channel", 40, 512, 1024),    # channelwise swap-AB
    ("channel", 2400, 4096, 256),  # channelwise CTA pairs
])
def test_dense_fp8_graph_replay_matches_eager(kind, M, N, K):
    if kind == "block":
        dd = W.make_dense_fp8(W.WORKLOADS["dense_fp8"], M, device=DEV, N=N, K=K)
        mm = moeq.w8a8_block_fp8_matmul
    else:
        dd = W.make_dense_fp8_channel(W.WORKLOADS["dense_fp8_channel"], M, device=DEV, N=N, K=K)
        mm = moeq.w8a8_channel_fp8_matmul
    c_eager = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    c_graph = torch.empty_like(c_eager)
    g = _capture(lambda: mm(dd["A"], dd["As"], dd["B"], dd["Bs"], out=c_graph))
    c_graph.zero_()
    g.replay()
    mm(dd["A"], dd["As"], dd["B"], dd["Bs"], out=c_eager)
    torch.cuda.synchronize()
    assert torch.equal(c_graph.view(torch.int16), c_eager.view(torch.int16))
    assert moeq.moe_device_status() == 0
