"""GPU parity of the grouped W4A16 GEMM entry points (contiguous and masked layouts) against the
oracle's grouped product, through the C ABI: every computed row within the W4A16 tolerance, and
rows the layout marks as padding / masked out left untouched."""
import numpy as np
import pytest
import torch

import oracle
import quantized_mixture_experts_align_b200 as moeq
import workloads as W
from tests._util import TOL_W4A16, assert_layer_close, bf16_to_f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
SENTINEL = 0x7FC1  # a bf16 NaN pattern no computed row can produce here


def _weights(G, N, K, seed_E=None):
    """INT4 group-32 weights [G, N, K/8] / [G, N, K/32] from the W4A16 recipe (W13 of the layer
    recipe with N = 2I, K = H)."""
    d = W.make_moe(W.WORKLOADS["tiny_w4a16"], device=DEV, T=1, E=G, k=1, H=K, I=N // 2)
    return d["w13q"], d["w13s"]


def _activations(M, K, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randn((M, K), generator=g).to(torch.bfloat16).to(DEV)


def _check(A, wq, ws, expert_of_row, out, rows, what):
    torch.cuda.synchronize()
    eor = np.asarray(expert_of_row, np.int32)
    ref = oracle.grouped_w4a16(W.np_bits(A), W.np_bits(wq), W.np_bits(ws), eor, rows=rows)
    got = out[torch.as_tensor(rows, device=DEV).long()]
    live = eor[rows] >= 0
    assert_layer_close(bf16_to_f64(got[torch.as_tensor(live, device=DEV)]), ref[live], TOL_W4A16, what)
    dead = got[torch.as_tensor(~live, device=DEV)]
    assert torch.all(dead.view(torch.int16) == SENTINEL), f"{what}: padding rows were written"


def _contiguous_layout(counts, pad=128):
    """m_indices of the pages' contiguous layout: each expert's rows, padded to a multiple of pad."""
    idx = []
    for e, c in enumerate(counts):
        idx += [e] * c + [-1] * ((-c) % pad)
    return np.array(idx, np.int32)


@pytest.mark.parametrize("counts,K,N", [
    ([300, 0, 7, 128, 1, 9, 64, 200], 256, 256),   # tensor-core schedule (>= 16 rows per expert on average)
    ([3, 1, 0, 2, 5, 4, 1, 1] * 4, 384, 128),     # register-fed schedule (few rows per expert)
])
def test_grouped_contiguous_matches_oracle(counts, K, N):
    G = len(counts)
    m_idx = _contiguous_layout(counts)
    M = len(m_idx)
    wq, ws = _weights(G, N, K)
    A = _activations(M, K, seed=M)
    out = torch.full((M, N), SENTINEL, dtype=torch.int16, device=DEV).view(torch.bfloat16)
    moeq.moe_w4a16_grouped_contiguous(A, wq, ws, torch.as_tensor(m_idx, device=DEV), out=out)
    _check(A, wq, ws, m_idx, out, np.arange(M, dtype=np.int32), f"contiguous G={G} M={M}")


def test_grouped_contiguous_any_row_order():
    """The implementation takes any row-to-expert map, not only sorted segments."""
    G, K, N = 6, 256, 256
    g = np.random.default_rng(8)
    m_idx = g.integers(-1, G, size=700).astype(np.int32)
    wq, ws = _weights(G, N, K)
    A = _activations(700, K, seed=5)
    out = torch.full((700, N), SENTINEL, dtype=torch.int16, device=DEV).view(torch.bfloat16)
    moeq.moe_w4a16_grouped_contiguous(A, wq, ws, torch.as_tensor(m_idx, device=DEV), out=out)
    _check(A, wq, ws, m_idx, out, np.arange(700, dtype=np.int32), "contiguous shuffled")


@pytest.mark.parametrize("expected_m", [4, 48])  # register-fed / tensor-core launch
def test_grouped_masked_matches_oracle(expected_m):
    G, max_m, K, N = 8, 64, 256, 384
    masked = np.array([0, 1, 5, 8, 9, 33, 64, 70], np.int32)  # 70 > max_m counts as max_m
    wq, ws = _weights(G, N, K)
    A = _activations(G * max_m, K, seed=17).view(G, max_m, K)
    out = torch.full((G * max_m, N), SENTINEL, dtype=torch.int16, device=DEV).view(torch.bfloat16)
    moeq.moe_w4a16_grouped_masked(A, wq, ws, torch.as_tensor(masked, device=DEV), expected_m, out=out)
    eor = np.array([e if r < min(masked[e], max_m) else -1 for e in range(G) for r in range(max_m)], np.int32)
    _check(A.view(G * max_m, K), wq, ws, eor, out, np.arange(G * max_m, dtype=np.int32), f"masked e_m={expected_m}")


def test_grouped_contiguous_kimi_shapes_sampled():
    """Kimi-K2 expert shapes (N = 2I = 4096, K = H = 7168), 16 experts with Zipf-like row counts;
    rows sampled for the oracle."""
    counts = [2000, 700, 300, 129, 128, 50, 17, 9, 8, 5, 3, 1, 1, 0, 0, 260]
    m_idx = _contiguous_layout(counts)
    M, G, K, N = len(m_idx), len(counts), 7168, 4096
    wq, ws = _weights(G, N, K)
    A = _activations(M, K, seed=3)
    out = torch.full((M, N), SENTINEL, dtype=torch.int16, device=DEV).view(torch.bfloat16)
    moeq.moe_w4a16_grouped_contiguous(A, wq, ws, torch.as_tensor(m_idx, device=DEV), out=out)
    g = np.random.default_rng(0)
    starts = np.concatenate([[0], np.cumsum([c + (-c) % 128 for c in counts])])
    rows = sorted(set([int(starts[e]) for e in range(G) if counts[e]] +
                      [int(starts[e] + counts[e] - 1) for e in range(G) if counts[e]] +
                      [int(starts[e] + counts[e]) for e in range(G) if counts[e] % 128] +
                      g.integers(0, M, size=12).tolist()))
    _check(A, wq, ws, m_idx, out, np.array(rows, np.int32), "contiguous Kimi shapes")
    assert moeq.moe_device_status() == 0
