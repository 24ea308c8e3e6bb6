"""Python binding of libmoeq.so, the sm_100a library for the routed, weight-quantized
Mixture-of-Experts expert layer. Every function has the name of the C entry point it calls
(declared in include/moeq.h) and only marshals arguments: torch CUDA tensors in, their device
pointers and sizes to the C ABI, the status checked. All computation runs in the library's CUDA
kernels; there is no CPU or PyTorch fallback - a missing library or a non-CUDA tensor raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoeq.so")

MOEQ_OK, MOEQ_ERR_INVALID_ARG, MOEQ_ERR_UNSUPPORTED, MOEQ_ERR_WORKSPACE, MOEQ_ERR_CUDA, MOEQ_ERR_DEVICE_TIMEOUT = range(6)


class MoeqError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"moeq error {code}: {msg}")
        self.code = code


_lib = None

_V, _I, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_SIGNATURES = {
    "moe_last_error": ([], ctypes.c_char_p),
    "moe_version": ([], ctypes.c_char_p),
    "moe_route_topk": ([_V, _I, _I, _I, _V, _V, _V], _I),
    "moe_align": ([_V, _I, _I, _I, _I, _V, _V, _V, _V, _Z, _V], _I),
    "moe_align_workspace_size": ([_I, _I, _I], _Z),
    "moe_fp8_act_quant": ([_V, _I, _I, _V, _V, _V], _I),
    "moe_w4a16_workspace_size": ([_I, _I, _I, _I, _I], _Z),
    "moe_w4a16_forward": ([_V, _V, _I, _I, _I, _I, _I, _V, _V, _V, _V, _V, _V, _V, _V, _Z, _V], _I),
    "moe_w4a16_forward_noalloc": ([_V, _V, _I, _I, _I, _I, _I, _V, _V, _V, _V, _V, _V, _V, _V], _I),
    "moe_mxfp4_prepack_scales": ([_V, ctypes.c_longlong, _V, _V], _I),
    "moe_nvfp4_prepack_scales": ([_V, ctypes.c_longlong, _V, _V], _I),
    "moe_nvfp4_workspace_size": ([_I, _I, _I, _I, _I], _Z),
    "moe_nvfp4_forward": ([_V, _V, _I, _I, _I, _I, _I, _V, _V, _V, _V, _V, _V, _V, _V, _V, _V, _Z, _V], _I),
    "moe_mxfp4_workspace_size": ([_I, _I, _I, _I, _I], _Z),
    "moe_mxfp4_forward": ([_V, _V, _I, _I, _I, _I, _I, _V, _V, _V, _V, _V, _V, _V, _V, _Z, _V], _I),
    "moe_w8a8_block_fp8_workspace_size": ([_I, _I, _I, _I, _I], _Z),
    "moe_w8a8_block_fp8_forward": ([_V, _V, _I, _I, _I, _I, _I, _V, _V, _V, _V, _V, _V, _V, _V, _Z, _V], _I),
    "moe_w4a16_ep_workspace_size": ([_I, _I, _I, _I, _I, _I], _Z),
    "moe_w4a16_forward_ep": ([_V, _V] + [_I] * 7 + [_V] * 8 + [_Z, _V], _I),
    "moe_mxfp4_forward_ep": ([_V, _V] + [_I] * 7 + [_V] * 8 + [_Z, _V], _I),
    "moe_nvfp4_forward_ep": ([_V, _V] + [_I] * 7 + [_V] * 10 + [_Z, _V], _I),
    "moe_w8a8_block_fp8_ep_workspace_size": ([_I, _I, _I, _I, _I, _I], _Z),
    "moe_w8a8_block_fp8_forward_ep": ([_V, _V] + [_I] * 7 + [_V] * 8 + [_Z, _V], _I),
    "w8a8_block_fp8_matmul": ([_V, _V, _V, _V, _I, _I, _I, _I, _I, _V, _V], _I),
    "w8a8_channel_fp8_matmul": ([_V, _V, _V, _V, _I, _I, _I, _V, _V], _I),
    "moe_w4a16_grouped_contiguous_workspace_size": ([_I, _I, _I, _I], _Z),
    "moe_w4a16_grouped_contiguous": ([_V, _I, _I, _V, _V, _I, _I, _V, _V, _V, _Z, _V], _I),
    "moe_w4a16_grouped_masked_workspace_size": ([_I, _I, _I, _I, _I], _Z),
    "moe_w4a16_grouped_masked": ([_V, _I, _I, _I, _V, _V, _I, _V, _I, _V, _V, _Z, _V], _I),
    "moe_trace_enable": ([_I], _I),
    "moe_trace_read": ([_V, _V, _I, _I], _I),
    "moe_host_stats": ([_V, _V, _V, _V, _I], _I),
    "moe_device_status": ([_I], _I),
    "moe_selftest_bounded_wait": ([_V], _I),
}


def lib() -> ctypes.CDLL:
    """Load libmoeq.so (built in-tree by build.py). Raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run quantized_mixture_experts_align_b200/build.py")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def exported_symbols() -> list[str]:
    return list(_SIGNATURES)


def _check(rc: int):
    if rc != MOEQ_OK:
        raise MoeqError(rc, lib().moe_last_error().decode())


def _dev(t: torch.Tensor | None, name: str, dtype=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise ValueError(f"{name} must have dtype {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _shape(t, want, name: str):
    """Raise unless tensor t has shape `want` (checked before any pointer is taken)."""
    if tuple(t.shape) != tuple(want):
        raise ValueError(f"{name} must have shape {tuple(want)}, got {tuple(t.shape)}")


def _layer_shapes(x, logits, w13, s13, w2, s2, E_w, I, w_div, s_div, fmt="w4a16"):
    """Shapes of a layer call: x [T, H], logits [T, E], and the weights of E_w experts: gate/up
    [E_w, 2I, H / w_div] with scales [E_w, 2I / s_row, H / s_div], down [E_w, H, I / w_div] with
    scales [E_w, H / s_row, I / s_div] (s_row = 128 for block FP8, else 1)."""
    T, H = x.shape
    if logits.dim() != 2 or logits.shape[0] != T:
        raise ValueError(f"logits must be [T={T}, E], got {tuple(logits.shape)}")
    if H % s_div or I % s_div:
        raise ValueError(f"H={H} and I={I} must be multiples of {s_div}")
    r = 128 if fmt == "fp8" else 1
    _shape(w13, (E_w, 2 * I, H // w_div), "w13")
    _shape(s13, (E_w, 2 * I // r, H // s_div), "w13 scales")
    _shape(w2, (E_w, H, I // w_div), "w2")
    _shape(s2, (E_w, H // r, I // s_div), "w2 scales")


def _layer_outputs(x, k, out, topk_ids_out, topk_w_out):
    """The layer's output buffers: out [T, H] (allocated when None) and the optional routing
    outputs topk_ids_out / topk_w_out [T, k]. A caller-passed buffer of another shape raises before
    any pointer is taken: the kernels write T x H and T x k elements through the raw pointers."""
    T, H = x.shape
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    _shape(out, (T, H), "out")
    if topk_ids_out is not None:
        _shape(topk_ids_out, (T, k), "topk_ids_out")
    if topk_w_out is not None:
        _shape(topk_w_out, (T, k), "topk_w_out")
    return out


_BF16 = (torch.bfloat16, torch.int16, torch.uint16)
_U8 = (torch.uint8, torch.float8_e4m3fn)


def version() -> str:
    return lib().moe_version().decode()


def moe_route_topk(logits: torch.Tensor, k: int, topk_ids=None, topk_w=None, stream=None):
    T, E = logits.shape
    topk_ids = torch.empty((T, k), dtype=torch.int32, device=logits.device) if topk_ids is None else topk_ids
    topk_w = torch.empty((T, k), dtype=torch.float32, device=logits.device) if topk_w is None else topk_w
    _shape(topk_ids, (T, k), "topk_ids")
    _shape(topk_w, (T, k), "topk_w")
    _check(lib().moe_route_topk(_dev(logits, "logits", torch.float32), T, E, k, _dev(topk_ids, "topk_ids", torch.int32),
                                _dev(topk_w, "topk_w", torch.float32), _stream(stream)))
    return topk_ids, topk_w


def moe_align_workspace_size(T: int, k: int, E: int) -> int:
    return int(lib().moe_align_workspace_size(T, k, E))


def moe_align(topk_ids: torch.Tensor, E: int, block_m: int, ws=None, stream=None):
    """ws: None allocates the scratch moe_align_workspace_size asks for; pass an empty tensor to
    run without scratch (the one-CTA kernel)."""
    T, k = topk_ids.shape
    cap = T * k + E * (block_m - 1)
    dev = topk_ids.device
    sorted_ids = torch.empty(cap, dtype=torch.int32, device=dev)
    expert_ids = torch.empty(-(-cap // block_m), dtype=torch.int32, device=dev)
    ntp = torch.empty(1, dtype=torch.int32, device=dev)
    if ws is None:
        ws = workspace(moe_align_workspace_size(T, k, E), dev)
    nbytes = ws.numel() * ws.element_size()
    _check(lib().moe_align(_dev(topk_ids, "topk_ids", torch.int32), T, k, E, block_m, _dev(sorted_ids, "sorted_ids"),
                           _dev(expert_ids, "expert_ids"), _dev(ntp, "ntp"), _dev(ws, "ws") if nbytes else None,
                           nbytes, _stream(stream)))
    return sorted_ids, expert_ids, ntp


def moe_fp8_act_quant(x: torch.Tensor, stream=None):
    rows, cols = x.shape
    q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    s = torch.empty((rows, cols // 128), dtype=torch.float32, device=x.device)
    _check(lib().moe_fp8_act_quant(_dev(x, "x", _BF16), rows, cols, _dev(q, "q"), _dev(s, "s"), _stream(stream)))
    return q, s


def moe_w4a16_workspace_size(T: int, H: int, I: int, E: int, k: int) -> int:
    return int(lib().moe_w4a16_workspace_size(T, H, I, E, k))


def moe_w8a8_block_fp8_workspace_size(T: int, H: int, I: int, E: int, k: int) -> int:
    return int(lib().moe_w8a8_block_fp8_workspace_size(T, H, I, E, k))


def workspace(nbytes: int, device) -> torch.Tensor:
    """A device scratch buffer for the *_forward calls (torch allocations are 256-byte aligned)."""
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def moe_w4a16_forward(x, logits, k, w13_q, w13_s, w2_q, w2_s, out=None, ws=None, topk_ids_out=None,
                      topk_w_out=None, stream=None):
    T, H = x.shape
    E = logits.shape[1]
    I = w2_q.shape[2] * 8
    _layer_shapes(x, logits, w13_q, w13_s, w2_q, w2_s, E, I, 8, 32)
    out = _layer_outputs(x, k, out, topk_ids_out, topk_w_out)
    need = moe_w4a16_workspace_size(T, H, I, E, k)
    ws = workspace(need, x.device) if ws is None else ws
    _check(lib().moe_w4a16_forward(
        _dev(x, "x", _BF16), _dev(logits, "logits", torch.float32), T, H, I, E, k,
        _dev(w13_q, "w13_q", torch.int32), _dev(w13_s, "w13_s", _BF16), _dev(w2_q, "w2_q", torch.int32),
        _dev(w2_s, "w2_s", _BF16), _dev(out, "out", _BF16), _dev(topk_ids_out, "topk_ids_out", torch.int32),
        _dev(topk_w_out, "topk_w_out", torch.float32), _dev(ws, "ws"), ws.numel() * ws.element_size(),
        _stream(stream)))
    return out


def moe_mxfp4_prepack_scales(s_ue8m0, out=None, stream=None):
    """UE8M0 group scales (uint8, any shape) -> the bf16 group factors 2^(s - 1) moe_mxfp4_forward
    takes (same shape)."""
    out = torch.empty(s_ue8m0.shape, dtype=torch.bfloat16, device=s_ue8m0.device) if out is None else out
    _shape(out, s_ue8m0.shape, "out")
    _check(lib().moe_mxfp4_prepack_scales(_dev(s_ue8m0, "s_ue8m0", _U8), s_ue8m0.numel(), _dev(out, "out", _BF16),
                                          _stream(stream)))
    return out


def moe_mxfp4_forward(x, logits, k, w13_q, w13_f, w2_q, w2_f, out=None, ws=None, topk_ids_out=None,
                      topk_w_out=None, stream=None):
    """The routed layer with MXFP4 weights: E2M1 codes w13_q / w2_q (int32, the INT4 packing) and
    the prepacked bf16 group factors w13_f / w2_f from moe_mxfp4_prepack_scales."""
    T, H = x.shape
    E = logits.shape[1]
    I = w2_q.shape[2] * 8
    _layer_shapes(x, logits, w13_q, w13_f, w2_q, w2_f, E, I, 8, 32)
    out = _layer_outputs(x, k, out, topk_ids_out, topk_w_out)
    need = lib().moe_mxfp4_workspace_size(T, H, I, E, k)
    ws = workspace(need, x.device) if ws is None else ws
    _check(lib().moe_mxfp4_forward(
        _dev(x, "x", _BF16), _dev(logits, "logits", torch.float32), T, H, I, E, k,
        _dev(w13_q, "w13_q", torch.int32), _dev(w13_f, "w13_f", _BF16), _dev(w2_q, "w2_q", torch.int32),
        _dev(w2_f, "w2_f", _BF16), _dev(out, "out", _BF16), _dev(topk_ids_out, "topk_ids_out", torch.int32),
        _dev(topk_w_out, "topk_w_out", torch.float32), _dev(ws, "ws"), ws.numel() * ws.element_size(),
        _stream(stream)))
    return out


def moe_nvfp4_prepack_scales(s_e4m3, out=None, stream=None):
    """E4M3 group scales (uint8, any shape) -> the bf16 factors E4M3(s) * 2^118 moe_nvfp4_forward
    takes (same shape)."""
    out = torch.empty(s_e4m3.shape, dtype=torch.bfloat16, device=s_e4m3.device) if out is None else out
    _shape(out, s_e4m3.shape, "out")
    _check(lib().moe_nvfp4_prepack_scales(_dev(s_e4m3, "s_e4m3", _U8), s_e4m3.numel(), _dev(out, "out", _BF16),
                                          _stream(stream)))
    return out


def moe_nvfp4_forward(x, logits, k, w13_q, w13_f, w13_g, w2_q, w2_f, w2_g, out=None, ws=None, topk_ids_out=None,
                      topk_w_out=None, stream=None):
    """The routed layer with NVFP4 weights: E2M1 codes (int32, the INT4 packing), the prepacked
    bf16 group-16 factors of moe_nvfp4_prepack_scales and the f32 tensor scales [E] per matrix."""
    T, H = x.shape
    E = logits.shape[1]
    I = w2_q.shape[2] * 8
    _layer_shapes(x, logits, w13_q, w13_f, w2_q, w2_f, E, I, 8, 16)
    _shape(w13_g, (E,), "w13_g")
    _shape(w2_g, (E,), "w2_g")
    out = _layer_outputs(x, k, out, topk_ids_out, topk_w_out)
    need = lib().moe_nvfp4_workspace_size(T, H, I, E, k)
    ws = workspace(need, x.device) if ws is None else ws
    _check(lib().moe_nvfp4_forward(
        _dev(x, "x", _BF16), _dev(logits, "logits", torch.float32), T, H, I, E, k,
        _dev(w13_q, "w13_q", torch.int32), _dev(w13_f, "w13_f", _BF16), _dev(w13_g, "w13_g", torch.float32),
        _dev(w2_q, "w2_q", torch.int32), _dev(w2_f, "w2_f", _BF16), _dev(w2_g, "w2_g", torch.float32),
        _dev(out, "out", _BF16), _dev(topk_ids_out, "topk_ids_out", torch.int32),
        _dev(topk_w_out, "topk_w_out", torch.float32), _dev(ws, "ws"), ws.numel() * ws.element_size(),
        _stream(stream)))
    return out


def moe_w4a16_forward_noalloc(x, logits, k, w13_q, w13_s, w2_q, w2_s, out=None, topk_ids_out=None,
                              topk_w_out=None, stream=None):
    """moe_w4a16_forward without a caller workspace: the library's built-in static device scratch
    is used (for callers that cannot allocate device memory; shapes up to a fixed size)."""
    T, H = x.shape
    E = logits.shape[1]
    I = w2_q.shape[2] * 8
    _layer_shapes(x, logits, w13_q, w13_s, w2_q, w2_s, E, I, 8, 32)
    out = _layer_outputs(x, k, out, topk_ids_out, topk_w_out)
    _check(lib().moe_w4a16_forward_noalloc(
        _dev(x, "x", _BF16), _dev(logits, "logits", torch.float32), T, H, I, E, k,
        _dev(w13_q, "w13_q", torch.int32), _dev(w13_s, "w13_s", _BF16), _dev(w2_q, "w2_q", torch.int32),
        _dev(w2_s, "w2_s", _BF16), _dev(out, "out", _BF16), _dev(topk_ids_out, "topk_ids_out", torch.int32),
        _dev(topk_w_out, "topk_w_out", torch.float32), _stream(stream)))
    return out


def moe_w8a8_block_fp8_forward(x, logits, k, w13, w13_s, w2, w2_s, out=None, ws=None, topk_ids_out=None,
                               topk_w_out=None, stream=None):
    T, H = x.shape
    E = logits.shape[1]
    I = w2.shape[2]
    _layer_shapes(x, logits, w13, w13_s, w2, w2_s, E, I, 1, 128, fmt="fp8")
    out = _layer_outputs(x, k, out, topk_ids_out, topk_w_out)
    need = moe_w8a8_block_fp8_workspace_size(T, H, I, E, k)
    ws = workspace(need, x.device) if ws is None else ws
    _check(lib().moe_w8a8_block_fp8_forward(
        _dev(x, "x", _BF16), _dev(logits, "logits", torch.float32), T, H, I, E, k,
        _dev(w13, "w13", _U8), _dev(w13_s, "w13_s", torch.float32), _dev(w2, "w2", _U8),
        _dev(w2_s, "w2_s", torch.float32), _dev(out, "out", _BF16), _dev(topk_ids_out, "topk_ids_out", torch.int32),
        _dev(topk_w_out, "topk_w_out", torch.float32), _dev(ws, "ws"), ws.numel() * ws.element_size(),
        _stream(stream)))
    return out


def moe_w4a16_ep_workspace_size(T: int, H: int, I: int, E: int, k: int, ep_local: int) -> int:
    return int(lib().moe_w4a16_ep_workspace_size(T, H, I, E, k, ep_local))


def moe_w8a8_block_fp8_ep_workspace_size(T: int, H: int, I: int, E: int, k: int, ep_local: int) -> int:
    return int(lib().moe_w8a8_block_fp8_ep_workspace_size(T, H, I, E, k, ep_local))


def _ep_call(name, x, logits, k, ep_base, weights, out, ws, topk_ids_out, topk_w_out, stream, I, ws_fn):
    """Shared marshalling of the *_forward_ep entry points: weights = [(tensor, name, dtype), ...] of
    ep_local experts, in the entry point's order."""
    T, H = x.shape
    E = logits.shape[1]
    ep_local = weights[0][0].shape[0]
    mats = [t for t, n, _ in weights if not n.endswith("_g")]  # codes / scales in the layer order
    if name == "moe_w8a8_block_fp8_forward_ep":
        _layer_shapes(x, logits, *mats, ep_local, I, 1, 128, fmt="fp8")
    else:
        _layer_shapes(x, logits, *mats, ep_local, I, 8, 16 if name == "moe_nvfp4_forward_ep" else 32)
    for t, n, _ in weights:
        if n.endswith("_g"):
            _shape(t, (ep_local,), n)
    out = _layer_outputs(x, k, out, topk_ids_out, topk_w_out)
    ws = workspace(ws_fn(T, H, I, E, k, ep_local), x.device) if ws is None else ws
    _check(getattr(lib(), name)(
        _dev(x, "x", _BF16), _dev(logits, "logits", torch.float32), T, H, I, E, k, int(ep_base), ep_local,
        *[_dev(t, n, dt) for t, n, dt in weights], _dev(out, "out", _BF16),
        _dev(topk_ids_out, "topk_ids_out", torch.int32), _dev(topk_w_out, "topk_w_out", torch.float32),
        _dev(ws, "ws"), ws.numel() * ws.element_size(), _stream(stream)))
    return out


def moe_w4a16_forward_ep(x, logits, k, ep_base, w13_q, w13_s, w2_q, w2_s, out=None, ws=None, topk_ids_out=None,
                         topk_w_out=None, stream=None):
    """One expert-parallel rank's share of the W4A16 layer: the weights of experts
    [ep_base, ep_base + len(w13_q)) only; the ranks' outputs sum to the layer's."""
    return _ep_call("moe_w4a16_forward_ep", x, logits, k, ep_base,
                    [(w13_q, "w13_q", torch.int32), (w13_s, "w13_s", _BF16), (w2_q, "w2_q", torch.int32),
                     (w2_s, "w2_s", _BF16)], out, ws, topk_ids_out, topk_w_out, stream, w2_q.shape[2] * 8,
                    moe_w4a16_ep_workspace_size)


def moe_mxfp4_forward_ep(x, logits, k, ep_base, w13_q, w13_f, w2_q, w2_f, out=None, ws=None, topk_ids_out=None,
                         topk_w_out=None, stream=None):
    """One expert-parallel rank's share of the MXFP4 layer (prepacked factors)."""
    return _ep_call("moe_mxfp4_forward_ep", x, logits, k, ep_base,
                    [(w13_q, "w13_q", torch.int32), (w13_f, "w13_f", _BF16), (w2_q, "w2_q", torch.int32),
                     (w2_f, "w2_f", _BF16)], out, ws, topk_ids_out, topk_w_out, stream, w2_q.shape[2] * 8,
                    moe_w4a16_ep_workspace_size)


def moe_nvfp4_forward_ep(x, logits, k, ep_base, w13_q, w13_f, w13_g, w2_q, w2_f, w2_g, out=None, ws=None,
                         topk_ids_out=None, topk_w_out=None, stream=None):
    """One expert-parallel rank's share of the NVFP4 layer (prepacked factors, tensor scales of the
    rank's experts)."""
    return _ep_call("moe_nvfp4_forward_ep", x, logits, k, ep_base,
                    [(w13_q, "w13_q", torch.int32), (w13_f, "w13_f", _BF16), (w13_g, "w13_g", torch.float32),
                     (w2_q, "w2_q", torch.int32), (w2_f, "w2_f", _BF16), (w2_g, "w2_g", torch.float32)],
                    out, ws, topk_ids_out, topk_w_out, stream, w2_q.shape[2] * 8, moe_w4a16_ep_workspace_size)


def moe_w8a8_block_fp8_forward_ep(x, logits, k, ep_base, w13, w13_s, w2, w2_s, out=None, ws=None, topk_ids_out=None,
                                  topk_w_out=None, stream=None):
    """One expert-parallel rank's share of the block-FP8 layer."""
    return _ep_call("moe_w8a8_block_fp8_forward_ep", x, logits, k, ep_base,
                    [(w13, "w13", _U8), (w13_s, "w13_s", torch.float32), (w2, "w2", _U8),
                     (w2_s, "w2_s", torch.float32)], out, ws, topk_ids_out, topk_w_out, stream, w2.shape[2],
                    moe_w8a8_block_fp8_ep_workspace_size)


def w8a8_block_fp8_matmul(A, As, B, Bs, block_size=(128, 128), out=None, stream=None):
    """C = block-scaled A B^T in bf16: A E4M3 [M, K], As f32 [M, K/128] (per token and 128-column
    group), B E4M3 [N, K], Bs f32 [cdiv(N, 128), cdiv(K, 128)] (per [128, 128] block)."""
    M, K = A.shape
    N = B.shape[0]
    _shape(B, (N, K), "B")
    _shape(As, (M, -(-K // 128)), "As")
    _shape(Bs, (-(-N // 128), -(-K // 128)), "Bs")
    out = torch.empty((M, N), dtype=torch.bfloat16, device=A.device) if out is None else out
    _shape(out, (M, N), "out")
    _check(lib().w8a8_block_fp8_matmul(
        _dev(A, "A", _U8), _dev(As, "As", torch.float32), _dev(B, "B", _U8), _dev(Bs, "Bs", torch.float32),
        M, N, K, int(block_size[0]), int(block_size[1]), _dev(out, "out", _BF16), _stream(stream)))
    return out


def w8a8_channel_fp8_matmul(A, As, B, Bs, out=None, stream=None):
    """Channelwise FP8 product C = As[m] Bs[n] (A B^T)[m, n] in bf16. A uint8 E4M3 [M, K], As f32
    [M], B uint8 E4M3 [N, K], Bs f32 [N]."""
    M, K = A.shape
    N = B.shape[0]
    if As.numel() != M or Bs.numel() != N:
        raise ValueError("w8a8_channel_fp8_matmul: As must hold M and Bs N scales")
    out = torch.empty((M, N), dtype=torch.bfloat16, device=A.device) if out is None else out
    _shape(out, (M, N), "out")
    _check(lib().w8a8_channel_fp8_matmul(
        _dev(A, "A", _U8), _dev(As, "As", torch.float32), _dev(B, "B", _U8), _dev(Bs, "Bs", torch.float32),
        M, N, K, _dev(out, "out", _BF16), _stream(stream)))
    return out


def moe_w4a16_grouped_contiguous(A, w_q, w_s, m_indices, out=None, ws=None, stream=None):
    """Grouped W4A16 GEMM, contiguous layout: C[m] = A[m] . dequant(W[m_indices[m]]) for rows with
    m_indices >= 0 (other rows of out are left as they are). A bf16 [M, K]; w_q int32 [G, N, K/8];
    w_s bf16 [G, N, K/32]; m_indices int32 [M]."""
    M, K = A.shape
    G, N = w_q.shape[0], w_q.shape[1]
    _shape(w_q, (G, N, K // 8), "w_q")
    _shape(w_s, (G, N, K // 32), "w_s")
    _shape(m_indices, (M,), "m_indices")
    out = torch.empty((M, N), dtype=torch.bfloat16, device=A.device) if out is None else out
    _shape(out, (M, N), "out")
    ws = workspace(lib().moe_w4a16_grouped_contiguous_workspace_size(M, K, N, G), A.device) if ws is None else ws
    _check(lib().moe_w4a16_grouped_contiguous(
        _dev(A, "A", _BF16), M, K, _dev(w_q, "w_q", torch.int32), _dev(w_s, "w_s", _BF16), G, N,
        _dev(m_indices, "m_indices", torch.int32), _dev(out, "out", _BF16), _dev(ws, "ws"),
        ws.numel() * ws.element_size(), _stream(stream)))
    return out


def moe_w4a16_grouped_masked(A, w_q, w_s, masked_m, expected_m, out=None, ws=None, stream=None):
    """Grouped W4A16 GEMM, masked layout: A bf16 [G, max_m, K] (or [G * max_m, K]); the first
    masked_m[e] rows of expert e's budget are computed, the rest of out is left as it is.
    expected_m: host-side rows-per-expert hint for the launch. Returns out [G * max_m, N]."""
    G, N = w_q.shape[0], w_q.shape[1]
    K = A.shape[-1]
    max_m = A.numel() // (G * K)
    if A.numel() != G * max_m * K:
        raise ValueError(f"A must hold G={G} budgets of max_m rows of K={K}, got {tuple(A.shape)}")
    _shape(w_q, (G, N, K // 8), "w_q")
    _shape(w_s, (G, N, K // 32), "w_s")
    _shape(masked_m, (G,), "masked_m")
    out = torch.empty((G * max_m, N), dtype=torch.bfloat16, device=A.device) if out is None else out
    _shape(out, (G * max_m, N), "out")
    ws = workspace(lib().moe_w4a16_grouped_masked_workspace_size(G, max_m, K, N, expected_m), A.device) \
        if ws is None else ws
    _check(lib().moe_w4a16_grouped_masked(
        _dev(A, "A", _BF16), G, max_m, K, _dev(w_q, "w_q", torch.int32), _dev(w_s, "w_s", _BF16), N,
        _dev(masked_m, "masked_m", torch.int32), int(expected_m), _dev(out, "out", _BF16), _dev(ws, "ws"),
        ws.numel() * ws.element_size(), _stream(stream)))
    return out


TRACE_STAGES = ("route_topk", "align", "fp8_act_quant", "gate_up", "down", "combine", "dense_fp8", "gather",
                "few_rows")


def moe_trace_enable(enable: bool = True):
    _check(lib().moe_trace_enable(1 if enable else 0))


def moe_trace_read(reset: bool = False) -> dict:
    """{stage name: (total ms, calls)} of the kernel stages recorded since the last reset."""
    n = len(TRACE_STAGES)
    ms = (ctypes.c_double * n)()
    calls = (ctypes.c_longlong * n)()
    rc = lib().moe_trace_read(ctypes.cast(ms, ctypes.c_void_p), ctypes.cast(calls, ctypes.c_void_p), n,
                              1 if reset else 0)
    if rc != n:
        _check(rc)
    return {name: (ms[i], calls[i]) for i, name in enumerate(TRACE_STAGES)}


def moe_host_stats(reset: bool = False) -> dict:
    """Host time the library's entry points spent (microseconds, summed), their call count, and
    tensor maps encoded / reused from the library's memo."""
    us = ctypes.c_double()
    calls, enc, reu = ctypes.c_longlong(), ctypes.c_longlong(), ctypes.c_longlong()
    _check(lib().moe_host_stats(ctypes.byref(us), ctypes.byref(calls), ctypes.byref(enc), ctypes.byref(reu),
                                1 if reset else 0))
    return {"host_us": us.value, "calls": calls.value, "tmap_encoded": enc.value, "tmap_reused": reu.value}


def moe_selftest_bounded_wait(stream=None):
    _check(lib().moe_selftest_bounded_wait(_stream(stream)))


def moe_device_status(clear: bool = False) -> int:
    return int(lib().moe_device_status(1 if clear else 0))
