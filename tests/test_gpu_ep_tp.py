"""GPU parity of the expert-parallel entry points (moe_*_forward_ep) and of tensor-parallel weight
slices against the oracle, through the C ABI, for every weight format. The ranks of a group are
run one after another on one GPU (independent calls, nothing waits on another rank): each rank's
share is compared with the oracle's share, and the shares' sum with the whole layer."""
import numpy as np
import pytest
import torch

import oracle
import quantized_mixture_experts_align_b200 as moeq
import workloads as W
from quantized_mixture_experts_align_b200 import sharding as S
from tests._util import TOL_FP8, TOL_W4A16, assert_layer_close, bf16_to_f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
RECIPE = {"w4a16": "tiny_w4a16", "mxfp4": "decode_mxfp4", "nvfp4": "decode_nvfp4", "fp8": "moe_fp8"}
TOL = {"w4a16": TOL_W4A16, "mxfp4": TOL_W4A16, "nvfp4": TOL_W4A16, "fp8": TOL_FP8}


def _make(kind, T, E, k, H, I):
    d = W.make_moe(W.WORKLOADS[RECIPE[kind]], device=DEV, T=T, E=E, k=k, H=H, I=I)
    if kind == "fp8":
        dev = {n: d[n] for n in ("w13", "w13s", "w2", "w2s")}
        host = {n: W.np_bits(d[n]) for n in dev}
    else:
        f13, f2 = ("w13s", "w2s") if kind == "w4a16" else ("w13f", "w2f")
        prep = {"mxfp4": moeq.moe_mxfp4_prepack_scales, "nvfp4": moeq.moe_nvfp4_prepack_scales}.get(kind)
        dev = {"w13q": d["w13q"], "w2q": d["w2q"], f13: prep(d["w13s"]) if prep else d["w13s"],
               f2: prep(d["w2s"]) if prep else d["w2s"]}
        host = {"w13q": W.np_bits(d["w13q"]), "w2q": W.np_bits(d["w2q"]), f13: W.np_bits(d["w13s"]),
                f2: W.np_bits(d["w2s"])}
        if kind == "nvfp4":
            dev.update(g13=d["g13"], g2=d["g2"])
            host.update(g13=W.np_bits(d["g13"]), g2=W.np_bits(d["g2"]))
    return d, dev, host


def _host_shard(host, kind, fn, *a):
    r = fn({n: torch.from_numpy(np.ascontiguousarray(v)) for n, v in host.items()}, kind, *a)
    w = r[0] if isinstance(r, tuple) else r
    return {n: v.numpy() for n, v in w.items()}


def _oracle(d, kind, hw, tokens, base=None):
    """The oracle's layer on the given (host) weights; with base, the expert-parallel share of
    experts [base, base + len(weights))."""
    x, lg, k = W.np_bits(d["x"]), W.np_bits(d["logits"]), d["k"]
    if kind == "fp8":
        if base is None:
            return oracle.moe_fp8(x, lg, k, hw["w13"], hw["w13s"], hw["w2"], hw["w2s"], tokens=tokens)
        return oracle.moe_fp8_ep(x, lg, k, base, hw["w13"], hw["w13s"], hw["w2"], hw["w2s"], tokens=tokens)
    s13, s2 = (hw["w13s"], hw["w2s"]) if kind == "w4a16" else (hw["w13f"], hw["w2f"])
    if base is None:
        base = 0
    return oracle.moe_q4_ep(kind, x, lg, k, base, hw["w13q"], s13, hw["w2q"], s2, hw.get("g13"), hw.get("g2"),
                            tokens=tokens)


@pytest.mark.parametrize("kind", ["w4a16", "mxfp4", "nvfp4", "fp8"])
@pytest.mark.parametrize("T", [16, 600])   # register-fed schedule / tensor-core schedule
def test_ep_shares_match_oracle_and_sum_to_the_layer(kind, T):
    E, k, H, I, world = 8, 2, 384, 256, 3              # uneven ranges: 2, 3, 3 experts
    d, dev, host = _make(kind, T, E, k, H, I)
    tokens = np.arange(T, dtype=np.int32)
    rid, _ = oracle.route_topk(W.np_bits(d["logits"]), k)
    full = _oracle(d, kind, host, tokens)
    total = np.zeros((T, H))
    for r in range(world):
        wd, base, local = S.shard_experts(dev, kind, r, world)
        ids = torch.empty((T, k), dtype=torch.int32, device=DEV)
        out = S.forward_ep_partial(kind, d["x"], d["logits"], k, wd, base, topk_ids_out=ids)
        torch.cuda.synchronize()
        got = bf16_to_f64(out)
        ref = _oracle(d, kind, _host_shard(host, kind, S.shard_experts, r, world), tokens, base)
        # rows with a slot on this rank: the layer tolerance, scaled by the layer's output on those
        # rows; the other rows are exact zeros
        mine = ((rid >= base) & (rid < base + local)).any(1)
        if mine.any():
            assert_layer_close(got[mine], ref[mine], TOL[kind], f"{kind} T={T} EP rank {r} of {world}",
                               rms=np.sqrt(np.mean(full[mine] ** 2)))
        assert np.all(got[~mine] == 0.0) and np.all(ref[~mine] == 0.0), \
            "tokens with no slot on this rank must get zero rows"
        assert np.array_equal(ids.cpu().numpy(), rid), "topk_ids_out holds the global expert ids"
        total += got
    assert_layer_close(total, full, TOL[kind], f"{kind} T={T} EP sum over {world} ranks")
    assert moeq.moe_device_status() == 0


@pytest.mark.parametrize("kind", ["w4a16", "nvfp4", "fp8"])
@pytest.mark.parametrize("T", [16, 600])
def test_tp_slices_match_oracle_and_sum_to_the_layer(kind, T):
    E, k, H, I, world = 8, 2, 384, 256, 2              # 128 features per rank
    d, dev, host = _make(kind, T, E, k, H, I)
    tokens = np.arange(T, dtype=np.int32)
    total = np.zeros((T, H))
    for r in range(world):
        out = S.forward_tp_partial(kind, d["x"], d["logits"], k, S.shard_intermediate(dev, kind, I, r, world))
        torch.cuda.synchronize()
        got = bf16_to_f64(out)
        ref = _oracle(d, kind, _host_shard(host, kind, S.shard_intermediate, I, r, world), tokens)
        assert_layer_close(got, ref, TOL[kind], f"{kind} T={T} TP rank {r} of {world}")
        total += got
    assert_layer_close(total, _oracle(d, kind, host, tokens), TOL[kind], f"{kind} T={T} TP sum")
    assert moeq.moe_device_status() == 0


def test_ep_rank_with_no_routed_slot_writes_zeros():
    d, dev, host = _make("w4a16", 64, 8, 2, 256, 128)
    lg = torch.full((64, 8), -5.0, device=DEV)
    lg[:, 0], lg[:, 1] = 3.0, 2.0                      # every token on experts 0 and 1
    d["logits"] = lg
    wd, base, _ = S.shard_experts(dev, "w4a16", 1, 2)  # experts 4..7
    out = torch.full((64, 256), 7.0, dtype=torch.bfloat16, device=DEV)
    S.forward_ep_partial("w4a16", d["x"], d["logits"], 2, wd, base, out=out)
    torch.cuda.synchronize()
    assert torch.all(out == 0)


def test_ep_decode_kimi_shapes_one_rank_of_eight():
    """Decode shapes (T = 32, H = 7168, I = 2048, k = 8) over 64 experts, rank 3 of an EP8 group
    (8 experts), every token; the share against the oracle's."""
    d, dev, host = _make("w4a16", 32, 64, 8, 7168, 2048)
    wd, base, local = S.shard_experts(dev, "w4a16", 3, 8)
    out = S.forward_ep_partial("w4a16", d["x"], d["logits"], 8, wd, base)
    torch.cuda.synchronize()
    hw = {n: W.np_bits(v) for n, v in wd.items()}
    ref = _oracle(d, "w4a16", hw, np.arange(32, dtype=np.int32), base)
    rid, _ = oracle.route_topk(W.np_bits(d["logits"]), 8)
    mine = ((rid >= base) & (rid < base + local)).any(1)
    got = bf16_to_f64(out)
    assert_layer_close(got[mine], ref[mine], TOL_W4A16, "EP8 rank 3 decode Kimi shapes")
    assert np.all(got[~mine] == 0.0)
    assert moeq.moe_device_status() == 0


def test_forward_ep_alone_is_the_layer():
    """Without a process group, forward_ep (share + reduce) over the whole expert range is the
    single-GPU layer, bit for bit."""
    d, dev, host = _make("w4a16", 200, 8, 2, 384, 256)
    ep = S.forward_ep("w4a16", d["x"], d["logits"], 2, dev, 0)
    one = moeq.moe_w4a16_forward(d["x"], d["logits"], 2, dev["w13q"], dev["w13s"], dev["w2q"], dev["w2s"])
    torch.cuda.synchronize()
    assert torch.equal(ep.view(torch.int16), one.view(torch.int16))
