"""GPU parity of the routed layer with NVFP4 weights (E2M1 codes, E4M3 group-16 scales, f32 tensor
scale per expert matrix) against the oracle's NVFP4 layer, through the C ABI: the scale prepack bit
for bit, the layer on the register-fed schedule, on the tensor-core schedule and at the Kimi-K2
decode shapes."""
import numpy as np
import pytest
import torch

import oracle
import quantized_mixture_experts_align_b200 as moeq
import workloads as W
from tests._util import TOL_W4A16, assert_layer_close, bf16_to_f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def test_nvfp4_prepack_every_scale_code():
    """Factor E4M3(s) * 2^118 as bf16 for every code, exact (torch's E4M3 decoder); NaN codes stay
    NaN."""
    s = torch.arange(256, dtype=torch.uint8, device=DEV)
    f = moeq.moe_nvfp4_prepack_scales(s)
    torch.cuda.synchronize()
    got = f.double().cpu().numpy()
    want = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy() * 2.0 ** 118
    nan = np.isnan(want)
    assert nan.sum() == 2 and np.all(np.isnan(got[nan]))
    assert np.array_equal(got[~nan], want[~nan])


def _layer(T, E, k, H, I, logit_mode="normal"):
    d = W.make_moe(W.WORKLOADS["decode_nvfp4"], device=DEV, T=T, E=E, k=k, H=H, I=I)
    if logit_mode == "split":
        lg = torch.full((T, E), -30.0, device=DEV)
        lg[torch.arange(T), torch.arange(T) % E] = 5.0
        lg[torch.arange(T), (torch.arange(T) * 7 + 3) % E] = 4.0
        d["logits"] = lg
    return d


def _parity(d, tokens, what):
    T, k = d["T"], d["k"]
    f13 = moeq.moe_nvfp4_prepack_scales(d["w13s"])
    f2 = moeq.moe_nvfp4_prepack_scales(d["w2s"])
    ids = torch.empty((T, k), dtype=torch.int32, device=DEV)
    out = moeq.moe_nvfp4_forward(d["x"], d["logits"], k, d["w13q"], f13, d["g13"], d["w2q"], f2, d["g2"],
                                 topk_ids_out=ids)
    torch.cuda.synchronize()
    ref = oracle.moe_nvfp4(W.np_bits(d["x"]), W.np_bits(d["logits"]), k, W.np_bits(d["w13q"]), W.np_bits(d["w13s"]),
                           W.np_bits(d["g13"]), W.np_bits(d["w2q"]), W.np_bits(d["w2s"]), W.np_bits(d["g2"]),
                           tokens=tokens)
    assert_layer_close(bf16_to_f64(out[torch.as_tensor(tokens, device=DEV).long()]), ref, TOL_W4A16, what)
    rid, _ = oracle.route_topk(W.np_bits(d["logits"]), k)
    assert np.array_equal(ids.cpu().numpy(), rid)
    assert moeq.moe_device_status() == 0


@pytest.mark.parametrize("T,E,k,H,I,mode", [
    (16, 8, 2, 512, 256, "normal"),      # register-fed schedule
    (1, 8, 2, 256, 128, "normal"),       # one token
    (400, 32, 2, 256, 128, "split"),     # tensor-core schedule, blocks of <= 8 rows on the register-fed kernel
    (600, 8, 2, 384, 256, "normal"),     # tensor-core schedule, ragged 256-row blocks
])
def test_nvfp4_layer_all_tokens(T, E, k, H, I, mode):
    d = _layer(T, E, k, H, I, mode)
    _parity(d, np.arange(T, dtype=np.int32), f"nvfp4 T={T} E={E} k={k} H={H} I={I} {mode}")


def test_nvfp4_decode_kimi_shapes():
    """The decode workload (T = 32, H = 7168, I = 2048, k = 8) with 64 experts, every token."""
    d = W.make_moe(W.WORKLOADS["decode_nvfp4"], device=DEV, E=64)
    _parity(d, np.arange(d["T"], dtype=np.int32), "nvfp4 decode Kimi shapes")
