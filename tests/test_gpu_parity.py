"""GPU parity of the CUDA path (called through the C ABI binding) against the CPU oracle, on
seeded synthetic inputs: bit-exact for routing ids and alignment, bit-exact for the FP8
activation quantizer, within the layer tolerance for outputs. Full-size workloads are checked on
sampled tokens / rows, which the oracle computes one by one."""
import numpy as np
import pytest
import torch

import oracle
import quantized_mixture_experts_align_b200 as moeq
import workloads as W
from tests._util import (TOL_FP8, TOL_W4A16, assert_layer_close, bf16_to_f64, block_tokens, oracle_layer,
                         sample_tokens)

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    moeq.lib()
    yield
    assert moeq.moe_device_status() == 0


_cache = {}


def workload(name, **kw):
    key = (name, tuple(sorted(kw.items())))
    if key not in _cache:
        wl = W.WORKLOADS[name]
        _cache[key] = W.make_moe(wl, device=DEV, **kw)
    return _cache[key]


def _forward(d, **kw):
    if d["kind"] == "w4a16":
        return moeq.moe_w4a16_forward(d["x"], d["logits"], d["k"], d["w13q"], d["w13s"], d["w2q"], d["w2s"], **kw)
    return moeq.moe_w8a8_block_fp8_forward(d["x"], d["logits"], d["k"], d["w13"], d["w13s"], d["w2"], d["w2s"], **kw)


# --------------------------------------------------------------------------------------------
# routing and alignment
# --------------------------------------------------------------------------------------------

def _check_route(logits_t, k):
    ids, w = moeq.moe_route_topk(logits_t, k)
    torch.cuda.synchronize()
    rid, rw = oracle.route_topk(W.np_bits(logits_t), k)
    assert np.array_equal(ids.cpu().numpy(), rid)
    gw = w.cpu().numpy()
    assert np.all(np.abs(gw.astype(np.float64) - rw) <= 2.5e-7 * np.abs(rw) + 1e-30)
    return ids


@pytest.mark.parametrize("name", ["tiny_w4a16", "decode_w4a16", "prefill_w4a16", "moe_fp8"])
def test_route_matches_oracle(name):
    wl = W.WORKLOADS[name]
    logits = W.router_logits(wl, wl.T, wl.E, device=DEV)
    _check_route(logits, wl.k)


def test_route_ties_and_edges():
    # ties go to the lower index; k = E; k = 1; E = 1024, k = 32
    _check_route(torch.zeros((5, 8), device=DEV), 8)
    lg = torch.tensor([[0.5, 2.0, 2.0, -1.0, 2.0, 0.0]], device=DEV)
    ids = _check_route(lg, 3)
    assert ids.tolist() == [[1, 2, 4]]
    _check_route(torch.randn((3, 7), device=DEV), 1)
    g = torch.Generator(device=DEV).manual_seed(5)
    _check_route(torch.randn((64, 1024), device=DEV, generator=g), 32)
    _check_route(torch.round(torch.randn((64, 97), device=DEV, generator=g) * 2) / 2, 9)


def _check_align(ids_t, E, B):
    s, e, n = moeq.moe_align(ids_t, E, B)
    torch.cuda.synchronize()
    rs, re_, rn = oracle.align(ids_t.cpu().numpy(), E, B)
    assert int(n.item()) == rn
    assert np.array_equal(s.cpu().numpy(), rs)
    assert np.array_equal(e.cpu().numpy(), re_)


@pytest.mark.parametrize("name", ["tiny_w4a16", "decode_w4a16", "prefill_w4a16", "moe_fp8"])
@pytest.mark.parametrize("B", [1, 8, 16, 32, 64, 128, 256])
def test_align_matches_oracle(name, B):
    wl = W.WORKLOADS[name]
    logits = W.router_logits(wl, wl.T, wl.E, device=DEV)
    ids, _ = moeq.moe_route_topk(logits, wl.k)
    _check_align(ids, wl.E, B)


def test_align_edges():
    g = torch.Generator(device="cpu").manual_seed(7)
    # T = 1; all slots on one expert; one expert of many; E = 1024 random; long input (many tiles)
    _check_align(torch.tensor([[3, 0]], dtype=torch.int32, device=DEV), 5, 4)
    _check_align(torch.full((3000, 1), 6, dtype=torch.int32, device=DEV), 8, 64)
    _check_align(torch.zeros((1, 1), dtype=torch.int32, device=DEV), 1, 1)
    ids = torch.stack([torch.randperm(1024, generator=g)[:4] for _ in range(700)]).to(torch.int32).to(DEV)
    _check_align(ids, 1024, 16)
    ids = torch.stack([torch.randperm(64, generator=g)[:8] for _ in range(40000)]).to(torch.int32).to(DEV)
    _check_align(ids, 64, 128)
    _check_align(torch.zeros((0, 2), dtype=torch.int32, device=DEV), 4, 8)


@pytest.mark.parametrize("B", [1, 8, 64, 128, 256])
def test_align_many_cta_matches_one_cta_and_oracle(B):
    """Past 8192 slots the alignment runs over many CTAs (per-chunk counts, scan, per-chunk stable
    scatter); it must equal the oracle and the one-CTA kernel (run without scratch) exactly:
    ragged chunk tails, one expert taking most slots (Zipf), E = 1024."""
    g = torch.Generator(device="cpu").manual_seed(31)
    cases = [
        (W.router_logits(W.WORKLOADS["prefill_w4a16"], 3001, 384, device=DEV), 384, 8),   # 24008 slots
        (torch.randn((2500, 1024), generator=g).to(DEV), 1024, 4),                        # 10000 slots
    ]
    for logits, E, k in cases:
        ids, _ = moeq.moe_route_topk(logits, k)
        assert moeq.moe_align_workspace_size(ids.shape[0], k, E) > 0
        _check_align(ids, E, B)
        s0, e0, n0 = moeq.moe_align(ids, E, B, ws=torch.empty(0, dtype=torch.uint8, device=DEV))
        s1, e1, n1 = moeq.moe_align(ids, E, B)
        torch.cuda.synchronize()
        assert torch.equal(s0, s1) and torch.equal(e0, e1) and torch.equal(n0, n1)
    skew = torch.zeros((9000, 1), dtype=torch.int32)
    skew[::7] = 5
    _check_align(skew.to(DEV), 8, B)


# --------------------------------------------------------------------------------------------
# FP8 activation quantizer (bit-exact: same IEEE division and RNE rounding)
# --------------------------------------------------------------------------------------------

def test_fp8_act_quant_bit_exact():
    g = torch.Generator(device=DEV).manual_seed(11)
    x = torch.randn((300, 1024), device=DEV, generator=g).to(torch.bfloat16)
    x[1, :128] = 0
    x[2, 128:256] = 1e4
    x[3, 256:384] = -3e-3
    x[4, 384:512] = torch.randn(128, device=DEV, generator=g).to(torch.bfloat16) * 1e-8
    q, s = moeq.moe_fp8_act_quant(x)
    torch.cuda.synchronize()
    rq, rs = oracle.fp8_act_quant(W.np_bits(x))
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(s.cpu().numpy(), rs)
    d = workload("moe_fp8")
    q, s = moeq.moe_fp8_act_quant(d["x"])
    rq, rs = oracle.fp8_act_quant(W.np_bits(d["x"]))
    assert np.array_equal(q.cpu().numpy(), rq) and np.array_equal(s.cpu().numpy(), rs)


# --------------------------------------------------------------------------------------------
# W4A16 layer
# --------------------------------------------------------------------------------------------

def _layer_parity(d, tokens, tol, what):
    T, k = d["T"], d["k"]
    ids = torch.empty((T, k), dtype=torch.int32, device=DEV)
    tw = torch.empty((T, k), dtype=torch.float32, device=DEV)
    out = _forward(d, topk_ids_out=ids, topk_w_out=tw)
    torch.cuda.synchronize()
    ref = oracle_layer(d, tokens)
    assert_layer_close(bf16_to_f64(out[torch.as_tensor(tokens, device=DEV).long()]), ref, tol, what)
    rid, rw = oracle.route_topk(W.np_bits(d["logits"]), k)
    assert np.array_equal(ids.cpu().numpy(), rid)
    return out


def test_w4a16_tiny_all_tokens():
    d = workload("tiny_w4a16")
    _layer_parity(d, np.arange(d["T"], dtype=np.int32), TOL_W4A16, "tiny_w4a16")


def test_w4a16_tiny_hand_worked_golden(golden_dir):
    """The hand-worked fixture of the oracle pins, run through the CUDA path."""
    import json, os
    from tests.test_oracle_pins import _hand_case
    g = json.load(open(os.path.join(golden_dir, "w4a16_hand.json")))
    # the library needs H, I multiples of 128: embed the 64x32 case into 128x128 with zero codes
    for case in g["cases"]:
        xb, logits, w13q, w13s, w2q, w2s = _hand_case(g, case)
        E, T = g["E"], g["T"]
        H, I, H2, I2 = g["H"], g["I"], 128, 128
        X = np.zeros((T, H2), np.uint16); X[:, :H] = xb
        zero = np.uint32(0x88888888).view(np.int32)
        Q13 = np.full((E, 2 * I2, H2 // 8), zero, np.int32)
        S13 = np.zeros((E, 2 * I2, H2 // 32), np.uint16)
        Q13[:, :I, :H // 8] = w13q[:, :I]; Q13[:, I2:I2 + I, :H // 8] = w13q[:, I:]
        S13[:, :I, :H // 32] = w13s[:, :I]; S13[:, I2:I2 + I, :H // 32] = w13s[:, I:]
        Q2 = np.full((E, H2, I2 // 8), zero, np.int32)
        S2 = np.zeros((E, H2, I2 // 32), np.uint16)
        Q2[:, :H, :I // 8] = w2q; S2[:, :H, :I // 32] = w2s
        t = lambda a, dt: torch.from_numpy(a.view(dt) if a.dtype == np.uint16 else a).to(DEV)
        out = moeq.moe_w4a16_forward(t(X, np.int16).view(torch.bfloat16), torch.from_numpy(logits).to(DEV),
                                     case["k"], t(Q13, None), t(S13, np.int16).view(torch.bfloat16), t(Q2, None),
                                     t(S2, np.int16).view(torch.bfloat16))
        got = bf16_to_f64(out)[:, :H]
        ref = np.zeros((T, H))
        for tt, m, v in case["out_nonzero"]:
            ref[tt, m] = v
        assert_layer_close(got, ref, TOL_W4A16, "hand-worked")


def test_w4a16_decode_all_tokens():
    d = workload("decode_w4a16")
    _layer_parity(d, np.arange(d["T"], dtype=np.int32), TOL_W4A16, "decode_w4a16")


@pytest.mark.parametrize("seed", [7, 9])
def test_w4a16_decode_peaked_routing_all_tokens(seed):
    """Decode shapes with peaked routing (N(0,1) logits times 3: one expert often carries most of a
    token's weight), so a token's output is dominated by one expert's rounding; the seeds are
    batches whose worst element exceeded the bound when the INT4 weights were rounded to bf16."""
    d = dict(workload("decode_w4a16"))
    g = torch.Generator(device=DEV).manual_seed(100 + seed)
    d["x"] = torch.randn(d["x"].shape, device=DEV, generator=g).to(torch.bfloat16)
    d["logits"] = torch.randn(d["logits"].shape, device=DEV, generator=g) * 3.0
    _layer_parity(d, np.arange(d["T"], dtype=np.int32), TOL_W4A16, f"decode_w4a16 peaked seed {seed}")


def test_w4a16_prefill_sampled():
    d = workload("prefill_w4a16")
    _layer_parity(d, sample_tokens(d, 10), TOL_W4A16, "prefill_w4a16")


def test_w4a16_prefill_heavy_and_tail_blocks():
    """Full prefill shapes (T = 8192, Zipf routing): every token of the most loaded expert's first
    and last 256-row tensor-core block, and every token of one block with at most 8 real rows (the
    register-fed side of the schedule)."""
    d = workload("prefill_w4a16")
    toks = block_tokens(d, 256, small_rows=8)
    assert toks.size > 256
    _layer_parity(d, toks, TOL_W4A16, "prefill_w4a16 heavy/tail blocks")


@pytest.mark.parametrize("T,E,k,H,I,logit_mode", [
    (1, 8, 2, 512, 256, "normal"),        # one token
    (200, 8, 1, 512, 256, "one"),         # every token on one expert (block_m 64, ragged tail)
    (37, 16, 16, 256, 128, "equal"),      # k = E, uniform weights 1/E
    (5, 1024, 32, 256, 128, "normal"),    # largest E and k
    (300, 64, 6, 384, 256, "zipf"),       # skewed, empty experts, ragged blocks
    (400, 32, 2, 256, 128, "split"),      # tensor-core schedule with blocks of exactly 8 and 9 rows
])
def test_w4a16_edge_cases(T, E, k, H, I, logit_mode):
    wl = W.WORKLOADS["tiny_w4a16"]
    d = W.make_moe(wl, device=DEV, T=T, E=E, k=k, H=H, I=I)
    if logit_mode == "one":
        d["logits"] = torch.zeros((T, E), device=DEV)
        d["logits"][:, 3] = 5.0
    elif logit_mode == "equal":
        d["logits"] = torch.zeros((T, E), device=DEV)
    elif logit_mode == "zipf":
        d["logits"] = W.router_logits(W.WORKLOADS["prefill_w4a16"], T, E, device=DEV)
    elif logit_mode == "split":
        # experts 0/1 take 300 tokens (full 256-row blocks + a tail), 2/3 exactly 8 (the register-fed
        # side of the small-block threshold), 4/5 exactly 9 (the tensor-core side), the rest 1-5
        first = np.zeros(T, np.int64)
        first[:300] = 0
        first[300:308] = 2
        first[308:317] = 4
        first[317:] = 6 + (np.arange(T - 317) % 20)
        lg = torch.zeros((T, E), device=DEV)
        idx = torch.as_tensor(first, device=DEV)
        lg[torch.arange(T, device=DEV), idx] = 5.0
        lg[torch.arange(T, device=DEV), idx + 1] = 4.0
        d["logits"] = lg
    _layer_parity(d, np.arange(T, dtype=np.int32), TOL_W4A16, f"w4a16 T={T} E={E} k={k}")


# --------------------------------------------------------------------------------------------
# W8A8 block-FP8 layer and dense matmul
# --------------------------------------------------------------------------------------------

def test_fp8_moe_small_all_tokens():
    d = W.make_moe(W.WORKLOADS["moe_fp8"], device=DEV, T=64, E=16, k=4, H=512, I=256)
    _layer_parity(d, np.arange(64, dtype=np.int32), TOL_FP8, "fp8 small")


def test_fp8_moe_full_sampled():
    d = workload("moe_fp8")
    _layer_parity(d, sample_tokens(d, 8), TOL_FP8, "moe_fp8")


def test_fp8_moe_full_heavy_tail_blocks_and_sampled():
    """Full block-FP8 MoE shapes (T = 4096, E = 256, Zipf routing): every token of the most loaded
    expert's first and last 128-row block, every token of one block with at most 8 real rows, and
    64 sampled tokens."""
    d = workload("moe_fp8")
    toks = block_tokens(d, 128, small_rows=8, n_sampled=64, seed=3)
    assert toks.size > 192
    _layer_parity(d, toks, TOL_FP8, "moe_fp8 heavy/tail blocks + sampled")


@pytest.mark.parametrize("T,E,k,H,logit_mode", [
    (1, 8, 2, 256, "normal"),      # register-fed path (few rows per expert)
    (150, 4, 1, 256, "one"),       # tensor-core path, one expert takes every token
    (33, 8, 8, 256, "equal"),      # k = E
    (100, 4, 2, 384, "zipf"),      # H not a multiple of 256: 128-column down tiles; empty experts
    (517, 24, 6, 512, "zipf"),     # many expert blocks, ragged tails
])
def test_fp8_moe_edge_cases(T, E, k, H, logit_mode):
    d = W.make_moe(W.WORKLOADS["moe_fp8"], device=DEV, T=T, E=E, k=k, H=H, I=256)
    if logit_mode == "one":
        d["logits"] = torch.zeros((T, E), device=DEV)
        d["logits"][:, 2] = 5.0
    elif logit_mode == "equal":
        d["logits"] = torch.zeros((T, E), device=DEV)
    elif logit_mode == "zipf":
        d["logits"] = W.router_logits(W.WORKLOADS["moe_fp8"], T, E, device=DEV)
    _layer_parity(d, np.arange(T, dtype=np.int32), TOL_FP8, f"fp8 T={T} E={E} k={k}")


def _dense_parity(M, N, K, rows):
    dd = W.make_dense_fp8(W.WORKLOADS["dense_fp8"], M, device=DEV, N=N, K=K)
    C = moeq.w8a8_block_fp8_matmul(dd["A"], dd["As"], dd["B"], dd["Bs"])
    torch.cuda.synchronize()
    ref = oracle.fp8_block_matmul(W.np_bits(dd["A"]), W.np_bits(dd["As"]), W.np_bits(dd["B"]), W.np_bits(dd["Bs"]),
                                  rows=rows)
    assert_layer_close(bf16_to_f64(C[torch.as_tensor(rows, device=DEV).long()]), ref, TOL_FP8, f"dense M={M}")


@pytest.mark.parametrize("M", [1, 2, 3, 8, 13, 16, 33, 64, 100])
def test_dense_fp8_small_shapes_all_rows(M):
    _dense_parity(M, 512, 1024, np.arange(M, dtype=np.int32))


@pytest.mark.parametrize("M,N,K", [(5, 256, 896), (70, 1280, 2944), (17, 384, 384), (128, 384, 1024),
                                   (120, 128, 7168), (33, 24576 // 16, 7168), (24, 24576 // 8, 7168),
                                   (32, 24576, 1152), (20, 640, 7168)])
def test_dense_fp8_skinny_split_shapes_all_rows(M, N, K):
    """The few-row path splits K over a cluster of CTAs: cluster sizes that do not divide the K
    blocks (7 CTAs over 7 blocks, 8 CTAs over 23), every padded row count (16 .. 128), one tile;
    17-32 rows on the three-CTAs-per-SM form with K splits of 2 (full N) and 8 (fewer tiles)."""
    _dense_parity(M, N, K, np.arange(M, dtype=np.int32))


@pytest.mark.parametrize("M,N,K", [(128, 256, 1024), (200, 512, 512), (300, 384, 896), (1000, 256, 7168),
                                   (256, 512, 384), (257, 768, 640), (640, 256, 1152), (2048, 2048, 1024),
                                   (2200, 2048, 1024)])
def test_dense_fp8_tensor_core_shapes_all_rows(M, N, K):
    """Row counts past the few-row kernel: 128- and 256-column tiles, the K range split over
    clusters of 2 to 4 CTAs where the tiles are few (uneven K ranges), ragged M tails, N not a
    multiple of 256."""
    _dense_parity(M, N, K, np.arange(M, dtype=np.int32))


@pytest.mark.parametrize("M", [1, 16, 32, 64, 128, 1000, 4096])
def test_dense_fp8_full_shape_sampled(M):
    rows = np.unique(np.array([0, M - 1, M // 2, M // 3], np.int32))
    _dense_parity(M, 24576, 7168, rows)


def _channel_parity(M, N, K, rows, what=""):
    d = W.make_dense_fp8_channel(W.WORKLOADS["dense_fp8_channel"], M, device=DEV, N=N, K=K)
    C = moeq.w8a8_channel_fp8_matmul(d["A"], d["As"], d["B"], d["Bs"])
    torch.cuda.synchronize()
    ref = oracle.fp8_channel_matmul(W.np_bits(d["A"]), W.np_bits(d["As"]), W.np_bits(d["B"]), W.np_bits(d["Bs"]),
                                    rows=rows)
    assert_layer_close(bf16_to_f64(C[torch.as_tensor(rows, device=DEV).long()]), ref, TOL_FP8,
                       f"channelwise M={M} N={N} K={K} {what}")
    assert moeq.moe_device_status() == 0


@pytest.mark.parametrize("M,N,K", [(1, 256, 1024), (5, 256, 896), (16, 128, 384), (33, 1280, 2944),
                                   (64, 384, 128), (65, 256, 1024), (128, 384, 640), (200, 512, 512),
                                   (256, 512, 384), (257, 768, 640), (640, 256, 1152), (2200, 2048, 1024),
                                   (2400, 4096, 256)])
def test_dense_fp8_channel_shapes_all_rows(M, N, K):
    """Every schedule of the channelwise GEMM: the few-row swap-AB kernel (cluster K split, 16 /
    32 / 64 padded rows), 128- and 256-column tiles with and without a cluster K split, CTA pairs
    (2400 rows: two waves of tiles, a ragged 256-row pair tile), ragged row tails."""
    _channel_parity(M, N, K, np.arange(M, dtype=np.int32))


@pytest.mark.parametrize("M", [1, 64, 4096])
def test_dense_fp8_channel_page_shape_sampled(M):
    """The N = K = 4096 shape of the SGLang channelwise config example, rows sampled."""
    rows = np.unique(np.array([0, M - 1, M // 2, M // 3], np.int32))
    _channel_parity(M, 4096, 4096, rows)


def test_dense_fp8_channel_closed_form():
    """All codes 448 with As[m] = 2^(m % 4) / 448 and Bs[n] = (1 + n % 3) / 448: C[m, n] =
    K 2^(m % 4) (1 + n % 3), exact in bf16 for K = 1024 (row and column scale indexing)."""
    for M in (3, 300):
        N, K = 384, 1024
        A = torch.full((M, K), 0x7E, dtype=torch.uint8, device=DEV)
        B = torch.full((N, K), 0x7E, dtype=torch.uint8, device=DEV)
        As = torch.tensor([2.0 ** (m % 4) / 448.0 for m in range(M)], device=DEV)
        Bs = torch.tensor([(1 + n % 3) / 448.0 for n in range(N)], device=DEV)
        C = moeq.w8a8_channel_fp8_matmul(A, As, B, Bs).double().cpu().numpy()
        want = K * np.array([2.0 ** (m % 4) for m in range(M)])[:, None] * np.array([1 + n % 3 for n in range(N)])[None, :]
        assert np.allclose(C, want, rtol=2 ** -8), f"M={M}"


def test_dense_fp8_closed_form_ones():
    M, N, K = 4, 256, 7168
    A = torch.full((M, K), 0x7E, dtype=torch.uint8, device=DEV)
    As = torch.full((M, K // 128), 1.0 / 448.0, device=DEV)
    B = torch.full((N, K), 0x7E, dtype=torch.uint8, device=DEV)
    Bs = torch.full((N // 128, K // 128), 0.5 / 448.0, device=DEV)
    C = moeq.w8a8_block_fp8_matmul(A, As, B, Bs).float().cpu().numpy()
    assert np.all(np.abs(C - 0.5 * K) <= 0.5 * K * 2 ** -8)


def test_tensor_map_memo_reuses_encodings():
    """A repeated tensor-core call on the same buffers reuses its encoded tensor maps (no driver
    encode), and a call on other buffers encodes new ones; the results are unchanged."""
    d = W.make_moe(W.WORKLOADS["moe_fp8"], device=DEV, T=256, E=8, k=2, H=512, I=256)
    ws = moeq.workspace(moeq.moe_w8a8_block_fp8_workspace_size(256, 512, 256, 8, 2), DEV)
    out1 = _forward(d, ws=ws)
    s0 = moeq.moe_host_stats()
    out2 = _forward(d, ws=ws)
    s1 = moeq.moe_host_stats()
    torch.cuda.synchronize()
    assert s1["tmap_encoded"] == s0["tmap_encoded"] and s1["tmap_reused"] >= s0["tmap_reused"] + 4
    assert s1["calls"] == s0["calls"] + 1 and s1["host_us"] > s0["host_us"]
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    ws2 = moeq.workspace(ws.numel() + 4096, DEV)
    _forward(d, ws=ws2)
    assert moeq.moe_host_stats()["tmap_encoded"] > s1["tmap_encoded"]
