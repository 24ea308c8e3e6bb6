"""Seeded synthetic inputs for the quantized routed-MoE layer, shared by the CUDA path's tests and
benchmark and by the CPU oracle. This module holds none of the layer's arithmetic: it draws
random numbers and encodes synthetic checkpoints with torch's own dtype casts.

Workloads (all seed 0, one independent random stream per (workload, tensor, expert)):

  tiny_w4a16     T=16, H=512, I=256, E=8, top-2; router logits N(0,1)
  decode_w4a16   T=32, H=7168, I=2048 (gate+up N=4096), E=384, top-8; router logits U[0,1)
  prefill_w4a16  the decode shapes with T=8192; logits N(0,1) plus a per-expert Zipf bias
  dense_fp8      A [M, 7168] (M = 1, 2, 4, ..., 4096), B [24576, 7168], E4M3 block-FP8
  moe_fp8        T=4096, H=7168, I=2048, E=256, top-8, E4M3 block-FP8, Zipf-biased logits

Recipes:
  * x: bf16 of N(0,1) f32 draws.
  * W4A16 weights: f32 N(0, 0.02) draws quantized per 32 consecutive inputs to unsigned INT4 with
    scale = bf16(max|w| / 7) and code = clamp(round_half_even(w / scale) + 8, 0, 15) (code 8 for
    an all-zero group), packed 8 codes per int32, code j of a word in bits [4j, 4j+4).
  * FP8 weights: f32 N(0, 0.02) draws, one f32 scale max(amax, 1e-10)/448 per [128, 128] block,
    codes = E4M3(w / scale) (torch's float8_e4m3fn cast).
  * dense_fp8 activations: bf16 N(0,1) draws quantized per row and 128-column group the same way.
  * Zipf bias: bias_e = -1.1 * ln(rank_e) with rank a seeded permutation of 1..E, added (f32) to
    N(0,1) logits, so routed rows per expert are skewed: many experts get no rows, a few get
    more than a thousand.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

SEED = 0


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str              # "w4a16", "mxfp4", "nvfp4", "fp8" (MoE layers) or "dense_fp8"
    wid: int               # stream id of the workload
    T: int = 0
    H: int = 0
    I: int = 0
    E: int = 0
    k: int = 0
    logits: str = "normal"  # "normal", "uniform" or "zipf"
    M_list: tuple = field(default_factory=tuple)
    N: int = 0
    K: int = 0


WORKLOADS = {
    "tiny_w4a16": Workload("tiny_w4a16", "w4a16", 0, T=16, H=512, I=256, E=8, k=2, logits="normal"),
    "decode_w4a16": Workload("decode_w4a16", "w4a16", 1, T=32, H=7168, I=2048, E=384, k=8, logits="uniform"),
    "prefill_w4a16": Workload("prefill_w4a16", "w4a16", 2, T=8192, H=7168, I=2048, E=384, k=8, logits="zipf"),
    "dense_fp8": Workload("dense_fp8", "dense_fp8", 3, M_list=tuple(2 ** i for i in range(13)), N=24576, K=7168),
    "moe_fp8": Workload("moe_fp8", "fp8", 4, T=4096, H=7168, I=2048, E=256, k=8, logits="zipf"),
    # the decode and prefill layers with MXFP4 weights (E2M1 codes, UE8M0 group-32 scales)
    "decode_mxfp4": Workload("decode_mxfp4", "mxfp4", 6, T=32, H=7168, I=2048, E=384, k=8, logits="uniform"),
    "prefill_mxfp4": Workload("prefill_mxfp4", "mxfp4", 7, T=8192, H=7168, I=2048, E=384, k=8, logits="zipf"),
    # ... and with NVFP4 weights (E2M1 codes, E4M3 group-16 scales, one f32 scale per expert matrix)
    "decode_nvfp4": Workload("decode_nvfp4", "nvfp4", 8, T=32, H=7168, I=2048, E=384, k=8, logits="uniform"),
    # channelwise W8A8 FP8 GEMM at the N = K = 4096 shape the SGLang config page gives as its example
    "dense_fp8_channel": Workload("dense_fp8_channel", "dense_fp8_channel", 5,
                                  M_list=(1, 16, 64, 128, 256, 1024, 4096), N=4096, K=4096),
}

# tensor stream ids
_X, _LOGITS, _RANKS, _W13, _W2, _A, _B = range(7)


def generator(wid: int, tensor: int, expert: int = 0, device="cpu", seed: int = SEED) -> torch.Generator:
    state = np.random.SeedSequence([seed, wid, tensor, expert]).generate_state(2, dtype=np.uint32)
    g = torch.Generator(device=device)
    g.manual_seed(int(state[0]) << 32 | int(state[1]))
    return g


def bf16_normal(shape, g, device) -> torch.Tensor:
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def router_logits(wl: Workload, T: int, E: int, device="cpu", wid=None) -> torch.Tensor:
    wid = wl.wid if wid is None else wid
    g = generator(wid, _LOGITS, device=device)
    if wl.logits == "uniform":
        return torch.rand((T, E), generator=g, device=device, dtype=torch.float32)
    z = torch.randn((T, E), generator=g, device=device, dtype=torch.float32)
    if wl.logits == "zipf":
        gr = generator(wid, _RANKS, device="cpu")
        rank = torch.randperm(E, generator=gr).to(torch.float64) + 1.0
        bias = (-1.1 * torch.log(rank)).to(torch.float32).to(device)
        z = z + bias[None, :]
    return z


def quantize_w4_group32(w: torch.Tensor):
    """f32 [N, K] -> (codes packed int32 [N, K/8], bf16 scales [N, K/32])."""
    N, K = w.shape
    wg = w.view(N, K // 32, 32)
    scale = (wg.abs().amax(-1) / 7.0).to(torch.bfloat16)
    sf = scale.float()[..., None]
    safe = torch.where(sf > 0, sf, torch.ones_like(sf))
    q = torch.where(sf > 0, torch.round(wg / safe) + 8.0, torch.full_like(wg, 8.0)).clamp(0, 15)
    q = q.to(torch.int64).view(N, K // 8, 8)
    shifts = torch.arange(0, 32, 4, device=w.device, dtype=torch.int64)
    packed = (q << shifts).sum(-1)
    packed = packed - ((packed >> 31) & 1) * (1 << 32)       # uint32 bit pattern as int32
    return packed.to(torch.int32).contiguous(), scale.contiguous()


# midpoints between consecutive E2M1 magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; a value on a midpoint
# goes to the even code (the lower one for midpoints 0, 2, 4, 6, the upper one for 1, 3, 5)
_E2M1_MIDS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)


def quantize_mxfp4_group32(w: torch.Tensor):
    """f32 [N, K] -> (E2M1 codes packed int32 [N, K/8] in the INT4 nibble order, UE8M0 scales
    uint8 [N, K/32]). Per group: the smallest power of two 2^(s-127) with amax / 2^(s-127) <= 6,
    codes rounded to nearest (ties to the even code); an all-zero group gets s = 0 and code 0."""
    N, K = w.shape
    wg = w.float().view(N, K // 32, 32)
    amax = wg.abs().amax(-1)
    pos = amax > 0
    e = torch.ceil(torch.log2(torch.where(pos, amax, torch.ones_like(amax)) / 6.0))
    # exact power-of-two boundary: keep the smallest exponent whose scaled amax is <= 6
    e = torch.where(amax / torch.pow(2.0, e) > 6.0, e + 1, e)
    e = torch.where(amax / torch.pow(2.0, e - 1) <= 6.0, e - 1, e)
    s = torch.where(pos, (e + 127).clamp(0, 254), torch.zeros_like(e))
    a = (wg / torch.pow(2.0, s - 127)[..., None]).abs().clamp(max=6.0)
    mids = torch.tensor(_E2M1_MIDS, dtype=torch.float32, device=w.device)
    code = torch.bucketize(a, mids)                     # a <= mid -> lower code
    on_mid = torch.zeros_like(a, dtype=torch.bool)
    lower = code.clamp(max=6)
    on_mid = (a == mids[lower]) & (lower % 2 == 1)      # ties at odd midpoints go up
    code = code + on_mid.to(code.dtype)
    code = code + 8 * ((wg < 0) & (code > 0)).to(code.dtype)
    q = code.to(torch.int64).view(N, K // 8, 8)
    shifts = torch.arange(0, 32, 4, device=w.device, dtype=torch.int64)
    packed = (q << shifts).sum(-1)
    packed = packed - ((packed >> 31) & 1) * (1 << 32)
    return packed.to(torch.int32).contiguous(), s.to(torch.uint8).contiguous()


def _e2m1_codes(a: torch.Tensor, neg: torch.Tensor) -> torch.Tensor:
    """|values| already scaled into [0, 6] -> E2M1 codes (nearest, ties to the even code)."""
    mids = torch.tensor(_E2M1_MIDS, dtype=torch.float32, device=a.device)
    code = torch.bucketize(a, mids)
    lower = code.clamp(max=6)
    code = code + ((a == mids[lower]) & (lower % 2 == 1)).to(code.dtype)
    return code + 8 * (neg & (code > 0)).to(code.dtype)


def _pack_nibbles(code: torch.Tensor, N: int, K: int) -> torch.Tensor:
    q = code.to(torch.int64).reshape(N, K // 8, 8)
    shifts = torch.arange(0, 32, 4, device=code.device, dtype=torch.int64)
    packed = (q << shifts).sum(-1)
    packed = packed - ((packed >> 31) & 1) * (1 << 32)
    return packed.to(torch.int32).contiguous()


def quantize_nvfp4_group16(w: torch.Tensor):
    """f32 [N, K] -> (E2M1 codes packed int32 [N, K/8], E4M3 scales uint8 [N, K/16], f32 tensor
    scale g). g = amax / (6 * 448); a 16-group's scale is E4M3(amax_group / (6 g)) (torch's
    rounding); codes are the group's values over E4M3(scale) * g, nearest with ties to even."""
    N, K = w.shape
    wf = w.float()
    amax = wf.abs().max()
    g = (amax / (6.0 * 448.0)).clamp(min=1e-30)
    wg = wf.view(N, K // 16, 16)
    sg = (wg.abs().amax(-1) / (6.0 * g)).to(torch.float8_e4m3fn)
    sv = sg.float()
    denom = (sv * g)[..., None]
    a = torch.where(denom > 0, wg.abs() / torch.where(denom > 0, denom, torch.ones_like(denom)),
                    torch.zeros_like(wg)).clamp(max=6.0)
    code = _e2m1_codes(a, wg < 0)
    return _pack_nibbles(code, N, K), sg.view(torch.uint8).contiguous(), g.reshape(1)


def quantize_fp8_blocks(w: torch.Tensor, bn: int = 128, bk: int = 128):
    """f32 [N, K] -> (E4M3 codes uint8 [N, K], f32 scales [N/bn, K/bk])."""
    N, K = w.shape
    wb = w.view(N // bn, bn, K // bk, bk)
    amax = wb.abs().amax(dim=(1, 3))
    scale = torch.clamp(amax, min=1e-10) / 448.0
    q = (wb / scale[:, None, :, None]).to(torch.float8_e4m3fn)
    return q.view(N, K).view(torch.uint8).contiguous(), scale.contiguous()


def quantize_fp8_rows(a: torch.Tensor, group: int = 128):
    """f32 [M, K] -> (E4M3 codes uint8 [M, K], f32 scales [M, K/group])."""
    M, K = a.shape
    ag = a.view(M, K // group, group)
    scale = torch.clamp(ag.abs().amax(-1), min=1e-10) / 448.0
    q = (ag / scale[..., None]).to(torch.float8_e4m3fn)
    return q.view(M, K).view(torch.uint8).contiguous(), scale.contiguous()


def make_moe(wl: Workload, device="cpu", T=None, E=None, k=None, H=None, I=None):
    """Inputs of a routed MoE workload. Overrides let tests reuse a recipe at other sizes."""
    T = wl.T if T is None else T
    E = wl.E if E is None else E
    k = wl.k if k is None else k
    H = wl.H if H is None else H
    I = wl.I if I is None else I
    x = bf16_normal((T, H), generator(wl.wid, _X, device=device), device)
    logits = router_logits(wl, T, E, device)
    d = dict(x=x, logits=logits, T=T, H=H, I=I, E=E, k=k, kind=wl.kind)
    if wl.kind in ("w4a16", "mxfp4"):
        quant = quantize_w4_group32 if wl.kind == "w4a16" else quantize_mxfp4_group32
        sdt = torch.bfloat16 if wl.kind == "w4a16" else torch.uint8
        w13q = torch.empty((E, 2 * I, H // 8), dtype=torch.int32, device=device)
        w13s = torch.empty((E, 2 * I, H // 32), dtype=sdt, device=device)
        w2q = torch.empty((E, H, I // 8), dtype=torch.int32, device=device)
        w2s = torch.empty((E, H, I // 32), dtype=sdt, device=device)
        for e in range(E):
            g = generator(wl.wid, _W13, e, device=device)
            w13q[e], w13s[e] = quant(torch.randn((2 * I, H), generator=g, device=device) * 0.02)
            g = generator(wl.wid, _W2, e, device=device)
            w2q[e], w2s[e] = quant(torch.randn((H, I), generator=g, device=device) * 0.02)
        d.update(w13q=w13q, w13s=w13s, w2q=w2q, w2s=w2s)
    elif wl.kind == "nvfp4":
        w13q = torch.empty((E, 2 * I, H // 8), dtype=torch.int32, device=device)
        w13s = torch.empty((E, 2 * I, H // 16), dtype=torch.uint8, device=device)
        w2q = torch.empty((E, H, I // 8), dtype=torch.int32, device=device)
        w2s = torch.empty((E, H, I // 16), dtype=torch.uint8, device=device)
        g13 = torch.empty((E,), dtype=torch.float32, device=device)
        g2 = torch.empty((E,), dtype=torch.float32, device=device)
        for e in range(E):
            g = generator(wl.wid, _W13, e, device=device)
            w13q[e], w13s[e], g13[e:e + 1] = quantize_nvfp4_group16(torch.randn((2 * I, H), generator=g, device=device) * 0.02)
            g = generator(wl.wid, _W2, e, device=device)
            w2q[e], w2s[e], g2[e:e + 1] = quantize_nvfp4_group16(torch.randn((H, I), generator=g, device=device) * 0.02)
        d.update(w13q=w13q, w13s=w13s, w2q=w2q, w2s=w2s, g13=g13, g2=g2)
    elif wl.kind == "fp8":
        w13 = torch.empty((E, 2 * I, H), dtype=torch.uint8, device=device)
        w13s = torch.empty((E, 2 * I // 128, H // 128), dtype=torch.float32, device=device)
        w2 = torch.empty((E, H, I), dtype=torch.uint8, device=device)
        w2s = torch.empty((E, H // 128, I // 128), dtype=torch.float32, device=device)
        for e in range(E):
            g = generator(wl.wid, _W13, e, device=device)
            w13[e], w13s[e] = quantize_fp8_blocks(torch.randn((2 * I, H), generator=g, device=device) * 0.02)
            g = generator(wl.wid, _W2, e, device=device)
            w2[e], w2s[e] = quantize_fp8_blocks(torch.randn((H, I), generator=g, device=device) * 0.02)
        d.update(w13=w13, w13s=w13s, w2=w2, w2s=w2s)
    else:
        raise ValueError(wl.kind)
    return d


def make_dense_fp8(wl: Workload, M: int, device="cpu", N=None, K=None):
    """A (quantized per row and 128-group) [M, K] and B (block-quantized) [N, K]. Rows of A do not
    depend on M: A for M rows is the first M rows of the largest draw."""
    N = wl.N if N is None else N
    K = wl.K if K is None else K
    Mmax = max(M, max(wl.M_list) if wl.M_list else M)
    a = bf16_normal((Mmax, K), generator(wl.wid, _A, device=device), device)[:M].float()
    Aq, As = quantize_fp8_rows(a)
    gb = generator(wl.wid, _B, device=device)
    Bq, Bs = quantize_fp8_blocks(torch.randn((N, K), generator=gb, device=device) * 0.02)
    return dict(A=Aq, As=As, B=Bq, Bs=Bs, M=M, N=N, K=K)


def make_dense_fp8_channel(wl: Workload, M: int, device="cpu", N=None, K=None):
    """A quantized per token (one scale per row, As [M]) and B per channel (Bs [N]), E4M3."""
    N = wl.N if N is None else N
    K = wl.K if K is None else K
    Mmax = max(M, max(wl.M_list) if wl.M_list else M)
    a = bf16_normal((Mmax, K), generator(wl.wid, _A, device=device), device)[:M].float()
    Aq, As = quantize_fp8_rows(a, group=K)
    gb = generator(wl.wid, _B, device=device)
    Bq, Bs = quantize_fp8_rows(torch.randn((N, K), generator=gb, device=device) * 0.02, group=K)
    return dict(A=Aq, As=As.reshape(M).contiguous(), B=Bq, Bs=Bs.reshape(N).contiguous(), M=M, N=N, K=K)


def np_bits(t: torch.Tensor) -> np.ndarray:
    """Host numpy view of a tensor's raw storage: bf16 -> uint16, everything else as is."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def moe_flops(T: int, k: int, H: int, I: int) -> float:
    """Algorithmic FLOPs of the layer: 2 per multiply-add of gate/up (N=2I, K=H) and of down
    (N=H, K=I), over the T*k routed rows (padding excluded)."""
    return 2.0 * T * k * (2 * I * H + H * I)


def w4a16_expert_bytes(H: int, I: int) -> int:
    """Packed codes + bf16 scales of one expert's gate/up and down matrices."""
    return (2 * I * H) // 2 + (2 * I * H // 32) * 2 + (H * I) // 2 + (H * I // 32) * 2


def fp8_expert_bytes(H: int, I: int) -> int:
    return 2 * I * H + (2 * I // 128) * (H // 128) * 4 + H * I + (H // 128) * (I // 128) * 4


def cdiv(a: int, b: int) -> int:
    return -(-a // b)


__all__ = ["WORKLOADS", "Workload", "make_moe", "make_dense_fp8", "make_dense_fp8_channel", "np_bits", "moe_flops",
           "w4a16_expert_bytes", "fp8_expert_bytes", "router_logits", "cdiv", "math"]
