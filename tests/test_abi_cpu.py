"""CPU-side checks of the C ABI: the library builds, loads and exports every entry point that
include/moeq.h declares, and host-side validation rejects bad arguments before any device work
(no GPU is touched: every call here fails validation before the first CUDA call)."""
import ctypes
import os
import re

import pytest

import quantized_mixture_experts_align_b200 as moeq
from quantized_mixture_experts_align_b200 import build as moeq_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    moeq_build.build()
    return moeq.lib()


def _declared():
    text = open(os.path.join(ROOT, "include", "moeq.h")).read()
    return re.findall(r"^MOEQ_API\s+[\w\s\*]*?\b(\w+)\s*\(", text, flags=re.M)


def test_header_declares_the_boundary():
    names = set(_declared())
    for need in ("moe_route_topk", "moe_align", "moe_w4a16_forward", "moe_w8a8_block_fp8_forward",
                 "w8a8_block_fp8_matmul", "w8a8_channel_fp8_matmul", "moe_fp8_act_quant", "moe_last_error"):
        assert need in names


def test_library_exports_every_declared_symbol(L):
    for name in _declared():
        assert hasattr(L, name), name
    assert set(_declared()) <= set(moeq.exported_symbols())


def test_version(L):
    assert "sm_100a" in moeq.version()


def test_workspace_sizes(L):
    a = moeq.moe_w4a16_workspace_size(32, 7168, 2048, 384, 8)
    n = 32 * 8
    assert a >= n * 2048 * 2 + n * 7168 * 2                   # h + weighted slot outputs (both bf16)
    assert moeq.moe_w4a16_workspace_size(8192, 7168, 2048, 384, 8) > a
    assert moeq.moe_w8a8_block_fp8_workspace_size(4096, 7168, 2048, 256, 8) > 0
    assert moeq.moe_w4a16_workspace_size(32, 100, 2048, 384, 8) == 0      # unsupported H
    assert moeq.moe_w4a16_workspace_size(32, 7168, 2048, 4, 8) == 0       # k > E


def _rc(L, name, *args):
    fn = getattr(L, name)
    return fn(*args)


def test_validation_rejects_before_device_work(L):
    N = None
    # route: k > E, E too large, k > 32
    assert _rc(L, "moe_route_topk", N, 4, 8, 9, N, N, N) == moeq.MOEQ_ERR_UNSUPPORTED
    assert _rc(L, "moe_route_topk", N, 4, 2000, 8, N, N, N) == moeq.MOEQ_ERR_UNSUPPORTED
    assert _rc(L, "moe_route_topk", N, 4, 64, 33, N, N, N) == moeq.MOEQ_ERR_UNSUPPORTED
    assert _rc(L, "moe_route_topk", N, 4, 64, 8, N, N, N) == moeq.MOEQ_ERR_INVALID_ARG   # NULL logits
    assert b"logits" in L.moe_last_error()
    # align: bad block size, negative T, NULL outputs
    assert _rc(L, "moe_align", N, 3, 2, 3, 0, N, N, N, N, 0, N) == moeq.MOEQ_ERR_UNSUPPORTED
    assert _rc(L, "moe_align", N, -1, 2, 3, 4, N, N, N, N, 0, N) == moeq.MOEQ_ERR_INVALID_ARG
    assert _rc(L, "moe_align", N, 3, 2, 3, 4, N, N, N, N, 0, N) == moeq.MOEQ_ERR_INVALID_ARG
    # act quant: ragged columns
    assert _rc(L, "moe_fp8_act_quant", N, 4, 100, N, N, N) == moeq.MOEQ_ERR_UNSUPPORTED
    # forward: unsupported H / I, workspace too small, misaligned workspace
    fwd = (N, N, 32, 7000, 2048, 384, 8, N, N, N, N, N, N, N, N, 0, N)
    assert _rc(L, "moe_w4a16_forward", *fwd) == moeq.MOEQ_ERR_UNSUPPORTED
    fwd = (N, N, 32, 7168, 2000, 384, 8, N, N, N, N, N, N, N, N, 0, N)
    assert _rc(L, "moe_w8a8_block_fp8_forward", *fwd) == moeq.MOEQ_ERR_UNSUPPORTED
    p = ctypes.c_void_p(256)
    fwd = (p, p, 32, 7168, 2048, 384, 8, p, p, p, p, p, N, N, p, 10, N)
    assert _rc(L, "moe_w4a16_forward", *fwd) == moeq.MOEQ_ERR_WORKSPACE
    assert b"workspace" in L.moe_last_error()
    q = ctypes.c_void_p(257)
    fwd = (p, p, 32, 7168, 2048, 384, 8, p, p, p, p, p, N, N, q, 1 << 40, N)
    assert _rc(L, "moe_w4a16_forward", *fwd) == moeq.MOEQ_ERR_INVALID_ARG
    # dense matmul: block size must be [128, 128]; K, N multiples of 128
    assert _rc(L, "w8a8_block_fp8_matmul", N, N, N, N, 4, 256, 256, 64, 128, N, N) == moeq.MOEQ_ERR_UNSUPPORTED
    assert _rc(L, "w8a8_block_fp8_matmul", N, N, N, N, 4, 256, 200, 128, 128, N, N) == moeq.MOEQ_ERR_UNSUPPORTED
    assert _rc(L, "w8a8_block_fp8_matmul", N, N, N, N, 4, 200, 256, 128, 128, N, N) == moeq.MOEQ_ERR_UNSUPPORTED
    # MXFP4 layer: the W4A16 validation; prepack: NULL / negative n
    mx = (p, p, 32, 7168, 2048, 384, 8, p, p, p, p, p, N, N, p, 10, N)
    assert _rc(L, "moe_mxfp4_forward", *mx) == moeq.MOEQ_ERR_WORKSPACE
    assert _rc(L, "moe_mxfp4_forward", p, p, 32, 100, 2048, 384, 8, p, p, p, p, p, N, N, p, 1 << 40, N) == \
        moeq.MOEQ_ERR_UNSUPPORTED
    assert moeq.lib().moe_mxfp4_workspace_size(32, 7168, 2048, 384, 8) == \
        moeq.lib().moe_w4a16_workspace_size(32, 7168, 2048, 384, 8) > 0
    assert _rc(L, "moe_mxfp4_prepack_scales", N, 16, p, N) == moeq.MOEQ_ERR_INVALID_ARG
    assert _rc(L, "moe_mxfp4_prepack_scales", p, -1, p, N) == moeq.MOEQ_ERR_INVALID_ARG
    assert _rc(L, "moe_mxfp4_prepack_scales", N, 0, N, N) == moeq.MOEQ_OK
    # NVFP4 layer: tensor scales required; prepack like MXFP4's
    nv = lambda g13, g2: _rc(L, "moe_nvfp4_forward", p, p, 32, 7168, 2048, 384, 8, p, p, g13, p, p, g2, p, N, N, p,
                             1 << 40, N)
    assert nv(N, p) == moeq.MOEQ_ERR_INVALID_ARG and nv(p, N) == moeq.MOEQ_ERR_INVALID_ARG
    assert _rc(L, "moe_nvfp4_prepack_scales", N, 16, p, N) == moeq.MOEQ_ERR_INVALID_ARG
    assert moeq.lib().moe_nvfp4_workspace_size(32, 7168, 2048, 384, 8) == \
        moeq.lib().moe_w4a16_workspace_size(32, 7168, 2048, 384, 8)
    # channelwise dense matmul: K, N multiples of 128; aligned A, B, C; NULL scales
    cw = lambda A_, As_, C_, M, Nn, K: _rc(L, "w8a8_channel_fp8_matmul", A_, As_, p, p, M, Nn, K, C_, N)
    assert cw(p, p, p, 4, 256, 200) == moeq.MOEQ_ERR_UNSUPPORTED
    assert cw(p, p, p, 4, 200, 256) == moeq.MOEQ_ERR_UNSUPPORTED
    assert cw(p, N, p, 4, 256, 256) == moeq.MOEQ_ERR_INVALID_ARG
    assert cw(p, p, p, -1, 256, 256) == moeq.MOEQ_ERR_INVALID_ARG
    assert cw(p, p, ctypes.c_void_p(p.value + 8), 4, 256, 256) == moeq.MOEQ_ERR_UNSUPPORTED
    assert cw(ctypes.c_void_p(p.value + 4), p, p, 4, 256, 256) == moeq.MOEQ_ERR_UNSUPPORTED
    assert cw(N, N, N, 0, 256, 256) == moeq.MOEQ_OK
    assert _rc(L, "w8a8_block_fp8_matmul", p, p, p, p, 4, 256, 256, 128, 128, ctypes.c_void_p(p.value + 2), N) == \
        moeq.MOEQ_ERR_UNSUPPORTED
    # grouped W4A16 GEMM: shapes, row map, workspace
    gc = lambda M, K, Nn, G, idx, ws, wsb: _rc(L, "moe_w4a16_grouped_contiguous", p, M, K, p, p, G, Nn, idx, p, ws, wsb, N)
    assert gc(64, 100, 256, 4, p, p, 1 << 40) == moeq.MOEQ_ERR_UNSUPPORTED       # K % 128
    assert gc(64, 256, 200, 4, p, p, 1 << 40) == moeq.MOEQ_ERR_UNSUPPORTED       # N % 128
    assert gc(64, 256, 256, 0, p, p, 1 << 40) == moeq.MOEQ_ERR_UNSUPPORTED       # G
    assert gc(64, 256, 256, 4, N, p, 1 << 40) == moeq.MOEQ_ERR_INVALID_ARG       # NULL m_indices
    assert gc(64, 256, 256, 4, p, p, 10) == moeq.MOEQ_ERR_WORKSPACE
    assert gc(0, 256, 256, 4, N, N, 0) == moeq.MOEQ_OK                           # no rows: no-op
    assert moeq.lib().moe_w4a16_grouped_contiguous_workspace_size(64, 100, 256, 4) == 0
    gm = lambda G, mm, K, Nn, masked, em: _rc(L, "moe_w4a16_grouped_masked", p, G, mm, K, p, p, Nn, masked, em, p, p,
                                              1 << 40, N)
    assert gm(4, 16, 256, 256, N, 4) == moeq.MOEQ_ERR_INVALID_ARG                # NULL masked_m
    assert gm(4, -1, 256, 256, p, 4) == moeq.MOEQ_ERR_INVALID_ARG                # max_m < 0
    assert gm(4, 16, 256, 256, p, -2) == moeq.MOEQ_ERR_INVALID_ARG               # expected_m < 0
    assert gm(2000, 16, 256, 256, p, 4) == moeq.MOEQ_ERR_UNSUPPORTED             # G > 1024
    assert moeq.lib().moe_w4a16_grouped_masked_workspace_size(8, 64, 256, 384, 48) > \
        moeq.lib().moe_w4a16_grouped_masked_workspace_size(8, 64, 256, 384, 4)   # tensor-core gather buffer
    # expert-parallel layers: the range must be non-empty and inside [0, E); workspace by ep_local
    ep = lambda name, base, local, wsb: _rc(L, name, p, p, 32, 7168, 2048, 384, 8, base, local, p, p, p, p, p, N, N,
                                            p, wsb, N)
    for name in ("moe_w4a16_forward_ep", "moe_mxfp4_forward_ep", "moe_w8a8_block_fp8_forward_ep"):
        assert ep(name, 0, 0, 1 << 40) == moeq.MOEQ_ERR_INVALID_ARG             # empty range
        assert ep(name, -1, 48, 1 << 40) == moeq.MOEQ_ERR_INVALID_ARG           # negative base
        assert ep(name, 340, 48, 1 << 40) == moeq.MOEQ_ERR_INVALID_ARG          # past E
        assert b"expert range" in L.moe_last_error()
        assert ep(name, 336, 48, 10) == moeq.MOEQ_ERR_WORKSPACE
    nvep = lambda g13, g2: _rc(L, "moe_nvfp4_forward_ep", p, p, 32, 7168, 2048, 384, 8, 0, 48, p, p, g13, p, p, g2,
                               p, N, N, p, 1 << 40, N)
    assert nvep(N, p) == moeq.MOEQ_ERR_INVALID_ARG and nvep(p, N) == moeq.MOEQ_ERR_INVALID_ARG
    w4_full = moeq.moe_w4a16_workspace_size(32, 7168, 2048, 384, 8)
    w4_ep = moeq.moe_w4a16_ep_workspace_size(32, 7168, 2048, 384, 8, 48)
    assert 0 < w4_ep < w4_full                     # the alignment's capacity follows ep_local
    assert moeq.moe_w4a16_ep_workspace_size(32, 7168, 2048, 384, 8, 384) == w4_full
    assert moeq.moe_w4a16_ep_workspace_size(32, 7168, 2048, 384, 8, 0) == 0
    assert moeq.moe_w8a8_block_fp8_ep_workspace_size(4096, 7168, 2048, 256, 8, 256) == \
        moeq.moe_w8a8_block_fp8_workspace_size(4096, 7168, 2048, 256, 8)
    assert moeq.moe_w8a8_block_fp8_ep_workspace_size(4096, 7168, 2048, 256, 8, 32) > 0
    # T == 0 / M == 0 are valid no-ops
    assert _rc(L, "moe_route_topk", N, 0, 8, 2, N, N, N) == 0
    assert _rc(L, "w8a8_block_fp8_matmul", N, N, N, N, 0, 256, 256, 128, 128, N, N) == 0


def test_binding_refuses_cpu_tensors(L):
    import torch
    with pytest.raises(ValueError):
        moeq.moe_route_topk(torch.zeros(4, 8), 2)


def test_binding_rejects_mismatched_shapes(L):
    """The binding checks every tensor's shape against the sizes it passes to the C ABI (which
    sees pointers only) and raises before taking any pointer (meta tensors: no memory, no GPU)."""
    import torch
    m = lambda *sh, dt=torch.uint8: torch.empty(sh, dtype=dt, device="meta")
    f32, i32, bf = torch.float32, torch.int32, torch.bfloat16
    # dense block FP8: As [M, cdiv(K,128)], Bs [cdiv(N,128), cdiv(K,128)], B [N, K]
    A, B = m(4, 256), m(384, 256)
    with pytest.raises(ValueError, match="Bs"):
        moeq.w8a8_block_fp8_matmul(A, m(4, 2, dt=f32), B, m(2, 2, dt=f32))
    with pytest.raises(ValueError, match="As"):
        moeq.w8a8_block_fp8_matmul(A, m(4, 3, dt=f32), B, m(3, 2, dt=f32))
    with pytest.raises(ValueError, match="B must"):
        moeq.w8a8_block_fp8_matmul(A, m(4, 2, dt=f32), m(384, 128), m(3, 2, dt=f32))
    # W4A16 layer (T=2, H=256, I=128, E=4): every weight tensor and the logits
    x, lg = m(2, 256, dt=bf), m(2, 4, dt=f32)
    good = [m(4, 256, 32, dt=i32), m(4, 256, 8, dt=bf), m(4, 256, 16, dt=i32), m(4, 256, 4, dt=bf)]
    for i, bad in enumerate([m(3, 256, 32, dt=i32), m(4, 256, 4, dt=bf), m(4, 128, 16, dt=i32), m(4, 256, 8, dt=bf)]):
        w = list(good)
        w[i] = bad
        with pytest.raises(ValueError, match="w13|w2"):
            moeq.moe_w4a16_forward(x, lg, 2, *w)
    with pytest.raises(ValueError, match="logits"):
        moeq.moe_w4a16_forward(x, m(3, 4, dt=f32), 2, *good)
    # NVFP4 group-16 scales and per-expert tensor scales
    nv = [m(4, 256, 32, dt=i32), m(4, 256, 16, dt=bf), m(4, dt=f32), m(4, 256, 16, dt=i32), m(4, 256, 8, dt=bf),
          m(4, dt=f32)]
    bad = list(nv)
    bad[2] = m(3, dt=f32)
    with pytest.raises(ValueError, match="w13_g"):
        moeq.moe_nvfp4_forward(x, lg, 2, *bad)
    bad = list(nv)
    bad[1] = m(4, 256, 8, dt=bf)                                  # group-32 scales given
    with pytest.raises(ValueError, match="w13 scales"):
        moeq.moe_nvfp4_forward(x, lg, 2, *bad)
    # block-FP8 layer: scales per [128, 128] block
    fp = [m(4, 256, 256), m(4, 2, 2, dt=f32), m(4, 256, 128), m(4, 2, 1, dt=f32)]
    bad = list(fp)
    bad[3] = m(4, 2, 2, dt=f32)
    with pytest.raises(ValueError, match="w2 scales"):
        moeq.moe_w8a8_block_fp8_forward(m(2, 256, dt=bf), lg, 2, *bad)
    # expert-parallel share: every tensor holds the same ep_local experts
    with pytest.raises(ValueError, match="w2"):
        moeq.moe_w4a16_forward_ep(x, lg, 2, 2, m(2, 256, 32, dt=i32), m(2, 256, 8, dt=bf), m(3, 256, 16, dt=i32),
                                  m(2, 256, 4, dt=bf))


def test_grouped_binding_rejects_mismatched_shapes(L):
    import torch
    m = lambda *sh, dt=torch.uint8: torch.empty(sh, dtype=dt, device="meta")
    i32, bf = torch.int32, torch.bfloat16
    A, wq, ws = m(256, 256, dt=bf), m(4, 128, 32, dt=i32), m(4, 128, 8, dt=bf)
    with pytest.raises(ValueError, match="w_s"):
        moeq.moe_w4a16_grouped_contiguous(A, wq, m(4, 128, 4, dt=bf), m(256, dt=i32))
    with pytest.raises(ValueError, match="m_indices"):
        moeq.moe_w4a16_grouped_contiguous(A, wq, ws, m(255, dt=i32))
    with pytest.raises(ValueError, match="masked_m"):
        moeq.moe_w4a16_grouped_masked(m(4, 16, 256, dt=bf), wq, ws, m(3, dt=i32), 4)
    with pytest.raises(ValueError, match="budgets"):
        moeq.moe_w4a16_grouped_masked(m(4, 15, 256, dt=bf).view(60, 256)[:58], wq, ws, m(4, dt=i32), 4)


def test_binding_rejects_output_buffers_of_the_wrong_shape(L):
    """Caller-passed outputs (out [T, H], topk_ids_out / topk_w_out [T, k], dense C [M, N]) are
    checked before any pointer is taken: a smaller buffer would be written past its end."""
    import torch
    m = lambda *sh, dt=torch.uint8: torch.empty(sh, dtype=dt, device="meta")
    f32, i32, bf = torch.float32, torch.int32, torch.bfloat16
    x, lg = m(2, 256, dt=bf), m(2, 4, dt=f32)
    w = [m(4, 256, 32, dt=i32), m(4, 256, 8, dt=bf), m(4, 256, 16, dt=i32), m(4, 256, 4, dt=bf)]
    with pytest.raises(ValueError, match="out"):
        moeq.moe_w4a16_forward(x, lg, 2, *w, out=m(1, 256, dt=bf))
    with pytest.raises(ValueError, match="topk_ids_out"):
        moeq.moe_w4a16_forward(x, lg, 2, *w, topk_ids_out=m(2, 1, dt=i32))
    with pytest.raises(ValueError, match="topk_w_out"):
        moeq.moe_mxfp4_forward(x, lg, 2, *w, topk_w_out=m(2, 3, dt=f32))
    fp = [m(4, 256, 256), m(4, 2, 2, dt=f32), m(4, 256, 128), m(4, 2, 1, dt=f32)]
    with pytest.raises(ValueError, match="out"):
        moeq.moe_w8a8_block_fp8_forward(x, lg, 2, *fp, out=m(2, 128, dt=bf))
    with pytest.raises(ValueError, match="out"):
        moeq.moe_w4a16_forward_ep(x, lg, 2, 0, *w, out=m(2, 255, dt=bf))
    with pytest.raises(ValueError, match="out"):
        moeq.w8a8_block_fp8_matmul(m(4, 256), m(4, 2, dt=f32), m(384, 256), m(3, 2, dt=f32), out=m(4, 256, dt=bf))
    with pytest.raises(ValueError, match="topk_ids"):
        moeq.moe_route_topk(lg, 2, topk_ids=m(2, 3, dt=i32))


def test_noalloc_binding_checks_shapes(L):
    """The scratch-free forward checks its tensors like moe_w4a16_forward before any pointer."""
    import torch
    m = lambda *sh, dt=torch.uint8: torch.empty(sh, dtype=dt, device="meta")
    f32, i32, bf = torch.float32, torch.int32, torch.bfloat16
    x, lg = m(2, 256, dt=bf), m(2, 4, dt=f32)
    good = [m(4, 256, 32, dt=i32), m(4, 256, 8, dt=bf), m(4, 256, 16, dt=i32), m(4, 256, 4, dt=bf)]
    for i, bad in enumerate([m(3, 256, 32, dt=i32), m(4, 256, 4, dt=bf), m(4, 128, 16, dt=i32), m(4, 256, 8, dt=bf)]):
        w = list(good)
        w[i] = bad
        with pytest.raises(ValueError, match="w13|w2"):
            moeq.moe_w4a16_forward_noalloc(x, lg, 2, *w)
    with pytest.raises(ValueError, match="logits"):
        moeq.moe_w4a16_forward_noalloc(x, m(3, 4, dt=f32), 2, *good)
    with pytest.raises(ValueError, match="out"):
        moeq.moe_w4a16_forward_noalloc(x, lg, 2, *good, out=m(2, 128, dt=bf))


def test_host_stats_counts_calls_without_a_device(L):
    """moe_host_stats reads host-side counters only. A call rejected during validation still
    counts its (host) time."""
    s0 = moeq.moe_host_stats(reset=True)
    assert s0["host_us"] >= 0 and s0["calls"] >= 0
    N = None
    rc = L.moe_w4a16_forward(N, N, 4, 7168, 2048, 384, 0, N, N, N, N, N, N, N, N, 0, N)  # k = 0: rejected
    assert rc != 0
    s1 = moeq.moe_host_stats()
    assert s1["calls"] == 1 and s1["host_us"] >= 0
