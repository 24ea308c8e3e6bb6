"""Python driver of the plain CPU oracle (``moe_oracle.c``), over numpy buffers.

TEST INFRASTRUCTURE: only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package. It shares no code with the CUDA library under
``quantized_mixture_experts_align_b200/`` and never imports it.

Every function here only marshals arguments; the arithmetic is in ``moe_oracle.c``, whose
comments cite the pages each step follows:
  * "vLLM x Novita AI: Chord W4A16 INT4 MoE Kernel for Kimi K2.x" (routing buffers, alignment,
    INT4 group-32 format, gate/up, down);
  * "SGLang W8A8 Block FP8 quantized kernel config files" (E4M3, [128, 128] weight blocks,
    per-token group-128 activation scales, ``w8a8_block_fp8_matmul``).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build as _build, LIB_PATH

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH) or os.path.getmtime(LIB_PATH) < os.path.getmtime(
            os.path.join(os.path.dirname(LIB_PATH), "moe_oracle.c")
        ):
            _build()
        _lib = ctypes.CDLL(LIB_PATH)
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle buffers must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


def _check(rc: int, name: str):
    if rc != 0:
        raise ValueError(f"oracle {name} rejected its arguments (status {rc})")


def route_topk(logits: np.ndarray, k: int):
    """logits f32 [T, E] -> (ids i32 [T, k], w f32 [T, k])."""
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    ids = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float32)
    _check(lib().orc_route_topk(_p(logits), T, E, k, _p(ids), _p(w)), "route_topk")
    return ids, w


def align(ids: np.ndarray, E: int, block_m: int):
    """ids i32 [T, k] -> (sorted_ids [T*k + E*(B-1)], expert_ids [cdiv(., B)], num_tokens_padded)."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, k = ids.shape
    cap = T * k + E * (block_m - 1)
    sorted_ids = np.zeros(cap, np.int32)
    expert_ids = np.zeros((cap + block_m - 1) // block_m, np.int32)
    ntp = np.zeros(1, np.int32)
    _check(lib().orc_align(_p(ids), T, k, E, block_m, _p(sorted_ids), _p(expert_ids), _p(ntp)), "align")
    return sorted_ids, expert_ids, int(ntp[0])


def fp8_act_quant(x_bf16: np.ndarray):
    """x bf16 bits (uint16) [R, C] -> (q uint8 [R, C], s f32 [R, C/128])."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    R, C = x.shape
    q = np.zeros((R, C), np.uint8)
    s = np.zeros((R, C // 128), np.float32)
    _check(lib().orc_fp8_act_quant(_p(x), R, C, _p(q), _p(s)), "fp8_act_quant")
    return q, s


def _tokens(tokens, T):
    if tokens is None:
        tokens = np.arange(T, dtype=np.int32)
    return np.ascontiguousarray(tokens, dtype=np.int32)


def moe_w4a16(x, logits, k, w13q, w13s, w2q, w2s, tokens=None, want_h=False):
    """Layer output (float64 [len(tokens), H]) for the chosen tokens; optionally the bf16 bits of
    each slot's intermediate [len(tokens), k, I]."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, H = x.shape
    E = logits.shape[1]
    I = w2q.shape[2] * 8
    tok = _tokens(tokens, T)
    out = np.zeros((len(tok), H), np.float64)
    h = np.zeros((len(tok), k, I), np.uint16) if want_h else None
    args = [np.ascontiguousarray(a) for a in (w13q, w13s, w2q, w2s)]
    assert args[0].dtype == np.int32 and args[1].dtype == np.uint16
    rc = lib().orc_moe_w4a16(_p(x), _p(logits), T, H, I, E, k, *[_p(a) for a in args], _p(tok), len(tok),
                             _p(out), _p(h) if h is not None else None)
    _check(rc, "moe_w4a16")
    return (out, h) if want_h else out


def moe_mxfp4(x, logits, k, w13q, w13s, w2q, w2s, tokens=None, want_h=False):
    """As moe_w4a16 with MXFP4 weights: E2M1 codes int32 [E, rows, K/8] (INT4 nibble order) and
    UE8M0 group-32 scales uint8 [E, rows, K/32]."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, H = x.shape
    E = logits.shape[1]
    I = w2q.shape[2] * 8
    tok = _tokens(tokens, T)
    out = np.zeros((len(tok), H), np.float64)
    h = np.zeros((len(tok), k, I), np.uint16) if want_h else None
    args = [np.ascontiguousarray(a) for a in (w13q, w13s, w2q, w2s)]
    assert args[0].dtype == np.int32 and args[1].dtype == np.uint8 and args[3].dtype == np.uint8
    rc = lib().orc_moe_mxfp4(_p(x), _p(logits), T, H, I, E, k, *[_p(a) for a in args], _p(tok), len(tok),
                             _p(out), _p(h) if h is not None else None)
    _check(rc, "moe_mxfp4")
    return (out, h) if want_h else out


def moe_nvfp4(x, logits, k, w13q, w13s, g13, w2q, w2s, g2, tokens=None, want_h=False):
    """As moe_w4a16 with NVFP4 weights: E2M1 codes int32 [E, rows, K/8], E4M3 group-16 scales
    uint8 [E, rows, K/16] and f32 tensor scales g13 [E] (gate/up) and g2 [E] (down)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, H = x.shape
    E = logits.shape[1]
    I = w2q.shape[2] * 8
    tok = _tokens(tokens, T)
    out = np.zeros((len(tok), H), np.float64)
    h = np.zeros((len(tok), k, I), np.uint16) if want_h else None
    q13, s13, q2, s2 = (np.ascontiguousarray(a) for a in (w13q, w13s, w2q, w2s))
    assert q13.dtype == np.int32 and s13.dtype == np.uint8 and s2.dtype == np.uint8
    assert s13.shape[-1] * 16 == H and s2.shape[-1] * 16 == I
    g13 = np.ascontiguousarray(g13, dtype=np.float32).reshape(E)
    g2 = np.ascontiguousarray(g2, dtype=np.float32).reshape(E)
    rc = lib().orc_moe_nvfp4(_p(x), _p(logits), T, H, I, E, k, _p(q13), _p(s13), _p(g13), _p(q2), _p(s2), _p(g2),
                             _p(tok), len(tok), _p(out), _p(h) if h is not None else None)
    _check(rc, "moe_nvfp4")
    return (out, h) if want_h else out


def moe_fp8(x, logits, k, w13, w13s, w2, w2s, tokens=None, want_h=False):
    """W8A8 block-FP8 layer output (float64 [len(tokens), H]); optionally the quantized
    intermediate (uint8 [len(tokens), k, I], f32 [len(tokens), k, I/128])."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, H = x.shape
    E = logits.shape[1]
    I = w2.shape[2]
    tok = _tokens(tokens, T)
    out = np.zeros((len(tok), H), np.float64)
    hq = np.zeros((len(tok), k, I), np.uint8) if want_h else None
    hs = np.zeros((len(tok), k, I // 128), np.float32) if want_h else None
    args = [np.ascontiguousarray(a) for a in (w13, w13s, w2, w2s)]
    rc = lib().orc_moe_fp8(_p(x), _p(logits), T, H, I, E, k, *[_p(a) for a in args], _p(tok), len(tok),
                           _p(out), _p(hq) if hq is not None else None, _p(hs) if hs is not None else None)
    _check(rc, "moe_fp8")
    return (out, hq, hs) if want_h else out


_Q4_FORMATS = {"w4a16": (0, np.uint16), "mxfp4": (1, np.uint8), "nvfp4": (2, np.uint8)}


def moe_q4_ep(fmt, x, logits, k, ep_base, w13q, w13s, w2q, w2s, g13=None, g2=None, tokens=None):
    """One expert-parallel rank's share of the 4-bit layer (float64 [len(tokens), H]): the slots
    whose expert lies in [ep_base, ep_base + ep_local), ep_local = len(w13q), the weights given
    being those experts'. fmt "w4a16" (bf16 scale bits), "mxfp4" (UE8M0 bytes) or "nvfp4" (E4M3
    bytes, with the tensor scales g13 / g2 [ep_local])."""
    code, sdt = _Q4_FORMATS[fmt]
    x = np.ascontiguousarray(x, dtype=np.uint16)
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, H = x.shape
    E = logits.shape[1]
    I = w2q.shape[2] * 8
    ep_local = w13q.shape[0]
    tok = _tokens(tokens, T)
    out = np.zeros((len(tok), H), np.float64)
    q13, q2 = np.ascontiguousarray(w13q, dtype=np.int32), np.ascontiguousarray(w2q, dtype=np.int32)
    s13, s2 = np.ascontiguousarray(w13s), np.ascontiguousarray(w2s)
    assert s13.dtype == sdt and s2.dtype == sdt
    gp = [None, None]
    if code == 2:
        g13 = np.ascontiguousarray(g13, dtype=np.float32).reshape(ep_local)
        g2 = np.ascontiguousarray(g2, dtype=np.float32).reshape(ep_local)
        gp = [_p(g13), _p(g2)]
    rc = lib().orc_moe_q4_ep(code, _p(x), _p(logits), T, H, I, E, k, int(ep_base), ep_local, _p(q13), _p(s13), gp[0],
                             _p(q2), _p(s2), gp[1], _p(tok), len(tok), _p(out))
    _check(rc, "moe_q4_ep")
    return out


def moe_fp8_ep(x, logits, k, ep_base, w13, w13s, w2, w2s, tokens=None):
    """One expert-parallel rank's share of the block-FP8 layer (float64 [len(tokens), H]), the
    weights given being those of experts [ep_base, ep_base + len(w13))."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, H = x.shape
    E = logits.shape[1]
    I = w2.shape[2]
    tok = _tokens(tokens, T)
    out = np.zeros((len(tok), H), np.float64)
    args = [np.ascontiguousarray(a) for a in (w13, w13s, w2, w2s)]
    rc = lib().orc_moe_fp8_ep(_p(x), _p(logits), T, H, I, E, k, int(ep_base), args[0].shape[0],
                              *[_p(a) for a in args], _p(tok), len(tok), _p(out))
    _check(rc, "moe_fp8_ep")
    return out


def fp8_block_matmul(A, As, B, Bs, rows=None):
    """C rows (float64 [len(rows), N]) of the dense block-FP8 product."""
    A = np.ascontiguousarray(A, dtype=np.uint8)
    B = np.ascontiguousarray(B, dtype=np.uint8)
    As = np.ascontiguousarray(As, dtype=np.float32)
    Bs = np.ascontiguousarray(Bs, dtype=np.float32)
    M, K = A.shape
    N = B.shape[0]
    r = _tokens(rows, M)
    C = np.zeros((len(r), N), np.float64)
    _check(lib().orc_fp8_block_matmul(_p(A), _p(As), _p(B), _p(Bs), M, N, K, _p(r), len(r), _p(C)),
           "fp8_block_matmul")
    return C


def fp8_channel_matmul(A, As, B, Bs, rows=None):
    """C rows (float64 [len(rows), N]) of the channelwise FP8 product As[m] Bs[n] (A_q B_q^T)[m, n].
    A uint8 E4M3 [M, K], As f32 [M], B uint8 E4M3 [N, K], Bs f32 [N]."""
    A = np.ascontiguousarray(A, dtype=np.uint8)
    B = np.ascontiguousarray(B, dtype=np.uint8)
    As = np.ascontiguousarray(As, dtype=np.float32).reshape(-1)
    Bs = np.ascontiguousarray(Bs, dtype=np.float32).reshape(-1)
    M, K = A.shape
    N = B.shape[0]
    if As.size != M or Bs.size != N or B.shape[1] != K:
        raise ValueError("fp8_channel_matmul: shapes")
    r = _tokens(rows, M)
    C = np.zeros((len(r), N), np.float64)
    _check(lib().orc_fp8_channel_matmul(_p(A), _p(As), _p(B), _p(Bs), M, N, K, _p(r), len(r), _p(C)),
           "fp8_channel_matmul")
    return C


def grouped_w4a16(A, wq, ws, expert_of_row, rows=None):
    """C rows (float64 [len(rows), N]) of the grouped W4A16 GEMM: row m times the dequantized
    weights of expert expert_of_row[m] (zeros where it is -1). A bf16 bits [M, K]; wq int32
    [G, N, K/8]; ws bf16 bits [G, N, K/32]."""
    A = np.ascontiguousarray(A, dtype=np.uint16)
    wq = np.ascontiguousarray(wq, dtype=np.int32)
    ws = np.ascontiguousarray(ws, dtype=np.uint16)
    eor = np.ascontiguousarray(expert_of_row, dtype=np.int32)
    M, K = A.shape
    G, N = wq.shape[0], wq.shape[1]
    r = _tokens(rows, M)
    C = np.zeros((len(r), N), np.float64)
    _check(lib().orc_grouped_w4a16(_p(A), M, K, _p(wq), _p(ws), G, N, _p(eor), _p(r), len(r), _p(C)),
           "grouped_w4a16")
    return C


# ---- format primitives (for the pins) ------------------------------------------------------

def bf16_round(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.zeros(v.shape, np.uint16)
    lib().orc_bf16_round(_p(v), _p(out), ctypes.c_long(v.size))
    return out


def bf16_value(b: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    out = np.zeros(b.shape, np.float64)
    lib().orc_bf16_value(_p(b), _p(out), ctypes.c_long(b.size))
    return out


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.zeros(v.shape, np.uint8)
    lib().orc_e4m3_encode(_p(v), _p(out), ctypes.c_long(v.size))
    return out


def e4m3_value(c: np.ndarray) -> np.ndarray:
    c = np.ascontiguousarray(c, dtype=np.uint8)
    out = np.zeros(c.shape, np.float64)
    lib().orc_e4m3_value(_p(c), _p(out), ctypes.c_long(c.size))
    return out


def w4a16_dequant(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.int32)
    s = np.ascontiguousarray(s, dtype=np.uint16)
    N, K8 = q.shape
    out = np.zeros((N, K8 * 8), np.float64)
    _check(lib().orc_w4a16_dequant(_p(q), _p(s), N, K8 * 8, _p(out)), "w4a16_dequant")
    return out


def mxfp4_dequant(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.int32)
    s = np.ascontiguousarray(s, dtype=np.uint8)
    N, K8 = q.shape
    out = np.zeros((N, K8 * 8), np.float64)
    _check(lib().orc_mxfp4_dequant(_p(q), _p(s), N, K8 * 8, _p(out)), "mxfp4_dequant")
    return out


def nvfp4_dequant(q: np.ndarray, s: np.ndarray, g: float) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.int32)
    s = np.ascontiguousarray(s, dtype=np.uint8)
    N, K8 = q.shape
    out = np.zeros((N, K8 * 8), np.float64)
    _check(lib().orc_nvfp4_dequant(_p(q), _p(s), ctypes.c_float(g), N, K8 * 8, _p(out)), "nvfp4_dequant")
    return out


def e2m1_value(c: np.ndarray) -> np.ndarray:
    c = np.ascontiguousarray(c, dtype=np.uint8)
    out = np.zeros(c.shape, np.float64)
    lib().orc_e2m1_value(_p(c), _p(out), ctypes.c_long(c.size))
    return out


def threads() -> int:
    """OpenMP threads the oracle will use (OMP_NUM_THREADS, else the host's cores)."""
    v = os.environ.get("OMP_NUM_THREADS")
    return int(v) if v else (os.cpu_count() or 1)
