"""Pins of the CPU oracle to facts that do not come from the oracle itself: hand-worked cases,
closed forms, invariants, brute force on tiny inputs and library routines (torch dtype casts,
numpy float64 matmul). Each test names the oracle function it pins."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads as W


def _bf16_bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


# --------------------------------------------------------------------------------------------
# number formats
# --------------------------------------------------------------------------------------------

def test_bf16_value_all_patterns_match_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = oracle.bf16_value(bits)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_bf16_round_matches_torch_on_f32_values_and_ties():
    rng = np.random.default_rng(1)
    u = rng.integers(0, 2 ** 32, 200000, dtype=np.uint64).astype(np.uint32)
    u = u[((u >> 23) & 0xFF) != 0xFF]                       # finite only
    ties = (u & 0xFFFF0000) | 0x8000                        # exact halfway cases
    f = np.concatenate([u, ties]).view(np.float32)
    ref = _bf16_bits(torch.from_numpy(f).to(torch.bfloat16))
    got = oracle.bf16_round(f.astype(np.float64))
    assert np.array_equal(got, ref)


def test_bf16_round_is_a_single_rounding_of_the_double():
    # 1 + 2^-8 + 2^-40 lies just above the halfway point between 1 and 1 + 2^-7: the nearest bf16
    # is 1 + 2^-7. Rounding to f32 first would land exactly on the tie and go to even (1.0).
    v = np.array([1 + 2.0 ** -8 + 2.0 ** -40, -(1 + 2.0 ** -8 + 2.0 ** -40), 1 + 2.0 ** -8], np.float64)
    got = oracle.bf16_value(oracle.bf16_round(v))
    assert list(got) == [1 + 2.0 ** -7, -(1 + 2.0 ** -7), 1.0]


def test_e4m3_value_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    got = oracle.e4m3_value(codes)
    nan = np.isnan(ref)
    assert nan.sum() == 2 and np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6


def test_e4m3_encode_matches_torch_in_range_and_saturates():
    rng = np.random.default_rng(2)
    vals = np.concatenate([
        rng.uniform(-448, 448, 100000), rng.normal(0, 1, 100000), rng.normal(0, 0.01, 50000),
    ]).astype(np.float32)
    grid = oracle.e4m3_value(np.arange(0, 0x7F, dtype=np.uint8))   # all finite non-negative values
    mids = ((grid[1:] + grid[:-1]) / 2).astype(np.float32)           # exact ties (representable in f32)
    vals = np.concatenate([vals, mids, -mids, grid.astype(np.float32)])
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(vals)
    assert np.array_equal(got, ref)
    sat = oracle.e4m3_encode(np.array([448.0, 460.0, 470.0, 1e6, -500.0], np.float32))
    assert list(sat) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE]


# --------------------------------------------------------------------------------------------
# routing
# --------------------------------------------------------------------------------------------

def test_route_closed_forms():
    ids, w = oracle.route_topk(np.array([[0.0, math.log(3.0)]], np.float32), 2)
    assert ids.tolist() == [[1, 0]]
    assert abs(w[0, 0] - 0.75) < 2e-7 and abs(w[0, 1] - 0.25) < 2e-7
    # all logits equal, k = E: ties go to the lower index, weights exactly 1/E
    ids, w = oracle.route_topk(np.zeros((3, 8), np.float32), 8)
    assert ids.tolist() == [list(range(8))] * 3
    assert np.all(w == np.float32(0.125))
    # k = 1: weight exactly 1
    ids, w = oracle.route_topk(np.array([[0.3, -2.0, 5.0, 5.0]], np.float32), 1)
    assert ids.tolist() == [[2]] and w[0, 0] == 1.0


def test_route_brute_force_against_numpy():
    rng = np.random.default_rng(3)
    for trial in range(200):
        T, E = int(rng.integers(1, 9)), int(rng.integers(1, 40))
        k = int(rng.integers(1, E + 1))
        lg = rng.normal(size=(T, E)).astype(np.float32)
        if trial % 3 == 0:                                 # force ties
            lg = np.round(lg * 2) / 2
        ids, w = oracle.route_topk(lg, k)
        for t in range(T):
            order = sorted(range(E), key=lambda e: (-float(lg[t, e]), e))[:k]
            assert ids[t].tolist() == order
            ex = np.exp(lg[t, order].astype(np.float64) - lg[t, order[0]])
            ref = (ex / ex.sum()).astype(np.float32)
            assert np.array_equal(w[t], ref)
            assert abs(float(w[t].astype(np.float64).sum()) - 1.0) <= 1e-6


# --------------------------------------------------------------------------------------------
# alignment
# --------------------------------------------------------------------------------------------

def test_align_hand_worked(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "align_hand.json")))
    s, e, n = oracle.align(np.array(g["topk_ids"], np.int32), g["E"], g["block_m"])
    assert s.tolist() == g["sorted_ids"]
    assert e.tolist() == g["expert_ids"]
    assert n == g["num_tokens_padded"]


def _align_numpy(ids, E, B):
    flat = ids.reshape(-1)
    n = flat.size
    cap = n + E * (B - 1)
    sorted_ids = np.full(cap, n, np.int32)
    expert_ids = np.full(-(-cap // B), -1, np.int32)
    order = np.argsort(flat, kind="stable")            # by expert, ties by slot
    counts = np.bincount(flat, minlength=E)
    pos, src = 0, 0
    for e in range(E):
        c = int(counts[e])
        sorted_ids[pos:pos + c] = order[src:src + c]
        p = -(-c // B) * B
        expert_ids[pos // B:(pos + p) // B] = e
        pos += p
        src += c
    return sorted_ids, expert_ids, pos


def test_align_brute_force_and_invariants():
    rng = np.random.default_rng(4)
    for _ in range(300):
        T, E = int(rng.integers(0, 9)), int(rng.integers(1, 7))
        k = int(rng.integers(1, min(3, E) + 1))
        B = int(rng.choice([1, 2, 3, 4, 8, 16]))
        ids = np.array([rng.permutation(E)[:k] for _ in range(T)], np.int32).reshape(T, k)
        s, e, n = oracle.align(ids, E, B)
        rs, re_, rn = _align_numpy(ids, E, B)
        assert np.array_equal(s, rs) and np.array_equal(e, re_) and n == rn
        flat = ids.reshape(-1)
        real = s[:n][s[:n] < T * k]
        assert sorted(real.tolist()) == list(range(T * k))      # every slot exactly once
        for b in range(n // B):                                  # one expert per block
            blk = s[b * B:(b + 1) * B]
            assert all(flat[f] == e[b] for f in blk if f < T * k)
        assert n == sum(-(-int(c) // B) * B for c in np.bincount(flat, minlength=E))


# --------------------------------------------------------------------------------------------
# W4A16 layer
# --------------------------------------------------------------------------------------------

def _hand_case(g, case):
    H, I, E, T = g["H"], g["I"], g["E"], g["T"]
    x = np.zeros((T, H), np.float32)
    for t, c, v in g["x_nonzero"]:
        x[t, c] = v
    dw = np.uint32(int(g["default_word"], 16)).view(np.int32)
    w13q = np.full((E, 2 * I, H // 8), dw, np.int32)
    w2q = np.full((E, H, I // 8), dw, np.int32)
    w13s = np.full((E, 2 * I, H // 32), g["default_scale_w13"], np.float32)
    w2s = np.full((E, H, I // 32), g["default_scale_w2"], np.float32)
    for e, r, wi, word in g["w13_words"]:
        w13q[e, r, wi] = np.uint32(int(word, 16)).view(np.int32)
    for e, r, wi, word in g["w2_words"]:
        w2q[e, r, wi] = np.uint32(int(word, 16)).view(np.int32)
    for e, r, gi, s in g["w13_scales"]:
        w13s[e, r, gi] = s
    for e, r, gi, s in g["w2_scales"]:
        w2s[e, r, gi] = s
    xb = _bf16_bits(torch.from_numpy(x).to(torch.bfloat16))
    w13sb = _bf16_bits(torch.from_numpy(w13s).to(torch.bfloat16))
    w2sb = _bf16_bits(torch.from_numpy(w2s).to(torch.bfloat16))
    logits = np.array(case["logits"], np.float32)
    return xb, logits, w13q, w13sb, w2q, w2sb


def test_w4a16_hand_worked(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "w4a16_hand.json")))
    for case in g["cases"]:
        xb, logits, w13q, w13s, w2q, w2s = _hand_case(g, case)
        out = oracle.moe_w4a16(xb, logits, case["k"], w13q, w13s, w2q, w2s)
        ref = np.zeros_like(out)
        for t, m, v in case["out_nonzero"]:
            ref[t, m] = v
        tol = case["rel_tol"] * np.abs(ref) + 1e-300
        assert np.all(np.abs(out - ref) <= tol), (out[np.nonzero(ref)], ref[np.nonzero(ref)])


def _np_unpack_w4(q, s):
    """Independent numpy restatement of the INT4 group-32 format (for library-matmul pins)."""
    q = q.view(np.uint32)
    N, K8 = q.shape
    codes = np.stack([(q >> (4 * j)) & 15 for j in range(8)], axis=-1).reshape(N, K8 * 8)
    scale = torch.from_numpy(s.view(np.int16)).view(torch.bfloat16).double().numpy()
    return (codes.astype(np.float64) - 8.0) * np.repeat(scale, 32, axis=1)


def _np_bf16(v):
    """bf16 rounding via torch (library); exact on these inputs (values come from f32 math below)."""
    return torch.from_numpy(np.ascontiguousarray(v)).to(torch.bfloat16).double().numpy()


def _np_ffn_w4(xd, w13, w2, I):
    g = xd @ w13[:I].T
    u = xd @ w13[I:].T
    a = g / (1.0 + np.exp(-g)) * u
    return a, w2


def test_w4a16_dense_equivalence_with_uniform_routing():
    """k = E and equal logits: every expert is selected with weight exactly 1/E, so the layer is
    (1/E) * sum_e FFN_e(x); FFN_e evaluated with numpy float64 matmul on the unpacked weights."""
    wl = W.WORKLOADS["tiny_w4a16"]
    d = W.make_moe(wl, T=4, E=8, k=8, H=128, I=64)
    x = W.np_bits(d["x"])
    logits = np.zeros((4, 8), np.float32)
    w13q, w13s, w2q, w2s = (W.np_bits(d[n]) for n in ("w13q", "w13s", "w2q", "w2s"))
    out, h = oracle.moe_w4a16(x, logits, 8, w13q, w13s, w2q, w2s, want_h=True)
    xd = oracle.bf16_value(x)  # exact
    ref = np.zeros_like(out)
    for e in range(8):
        w13 = _np_unpack_w4(w13q[e], w13s[e])
        w2 = _np_unpack_w4(w2q[e], w2s[e])
        a, _ = _np_ffn_w4(xd, w13, w2, 64)
        # h must be bf16(a): compare the oracle's intermediate to the rounding of numpy's a
        hv = oracle.bf16_value(h[:, e, :])
        assert np.all(np.abs(hv - a) <= np.abs(a) * 2.0 ** -8 + 1e-30)
        ref += (1.0 / 8.0) * (hv @ w2.T)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-15)


def test_w4a16_single_expert_is_dense_gemm():
    """k = 1 and one dominant logit: every token goes to expert 5 with weight 1."""
    wl = W.WORKLOADS["tiny_w4a16"]
    d = W.make_moe(wl, T=6, E=8, k=1, H=256, I=128)
    x = W.np_bits(d["x"])
    logits = np.zeros((6, 8), np.float32)
    logits[:, 5] = 10.0
    w13q, w13s, w2q, w2s = (W.np_bits(d[n]) for n in ("w13q", "w13s", "w2q", "w2s"))
    out = oracle.moe_w4a16(x, logits, 1, w13q, w13s, w2q, w2s)
    xd = oracle.bf16_value(x)
    w13 = _np_unpack_w4(w13q[5], w13s[5])
    w2 = _np_unpack_w4(w2q[5], w2s[5])
    a, _ = _np_ffn_w4(xd, w13, w2, 128)
    ref = _np_bf16(a) @ w2.T
    # a from numpy and from the oracle may differ in the last double bit, which can flip a bf16
    # rounding of h; bound that by one bf16 ulp of h per term
    bound = (np.abs(a) * 2.0 ** -8) @ np.abs(w2.T) + 1e-12
    assert np.all(np.abs(out - ref) <= bound)
    assert np.allclose(out, ref, rtol=1e-6, atol=1e-9)


def test_w4a16_dequant_matches_numpy_unpack():
    d = W.make_moe(W.WORKLOADS["tiny_w4a16"], T=1, E=1, k=1, H=128, I=64)
    q, s = W.np_bits(d["w13q"])[0], W.np_bits(d["w13s"])[0]
    assert np.array_equal(oracle.w4a16_dequant(q, s), _np_unpack_w4(q, s))


def test_grouped_w4a16_matches_numpy_on_numpy_unpacked_weights():
    """Library special case: each row times its expert's weights, unpacked by numpy (not by the
    oracle) and multiplied with float64 matmul; -1 rows are not computed (zeros)."""
    d = W.make_moe(W.WORKLOADS["tiny_w4a16"], T=1, E=3, k=1, H=128, I=64)
    wq, ws = W.np_bits(d["w13q"]), W.np_bits(d["w13s"])          # [3, 128, 16], [3, 128, 4]
    g = np.random.default_rng(3)
    A = _bf16_bits(torch.from_numpy(g.standard_normal((9, 128)).astype(np.float32)).to(torch.bfloat16))
    eor = np.array([0, 0, 2, -1, 1, 2, -1, 0, 1], np.int32)
    got = oracle.grouped_w4a16(A, wq, ws, eor)
    Ad = torch.from_numpy(A.view(np.int16)).view(torch.bfloat16).double().numpy()   # bits -> values (torch)
    for m in range(9):
        if eor[m] < 0:
            assert np.all(got[m] == 0.0)
            continue
        ref = _np_unpack_w4(wq[eor[m]], ws[eor[m]]) @ Ad[m]
        assert np.allclose(got[m], ref, rtol=1e-12, atol=1e-12)


def test_grouped_w4a16_closed_form_and_nibble_order():
    """Codes all 9 with scale 0.5 and A of ones give K * 0.5; one code 10 at input column 37 (word
    4, nibble 5) of row 3 of expert 1 adds exactly A[m, 37] * 0.5 there."""
    G, N, K = 2, 4, 64
    wq = np.full((G, N, K // 8), np.int32(np.uint32(0x99999999).view(np.int32)), np.int32)
    ws = np.full((G, N, K // 32), 0x3F00, np.uint16)                        # bf16 0.5
    A = np.full((3, K), 0x3F80, np.uint16)                                  # bf16 1.0
    C = oracle.grouped_w4a16(A, wq, ws, np.array([0, 1, -1], np.int32))
    assert np.all(C[0] == K * 0.5) and np.all(C[1] == K * 0.5) and np.all(C[2] == 0.0)
    word = np.uint32(0x99999999) & ~np.uint32(0xF << 20) | np.uint32(0xA << 20)
    wq[1, 3, 4] = np.int32(word.view(np.int32))
    A[1, 37] = 0x4040                                                       # bf16 3.0
    C = oracle.grouped_w4a16(A, wq, ws, np.array([0, 1, -1], np.int32))
    # row 3: 63 columns of 1.0 * 0.5, column 37 of 3.0 * (10 - 8) * 0.5; row 2: column 37 at 0.5
    assert C[1, 3] == (K - 1) * 0.5 + 3.0 * 1.0 and C[1, 2] == (K - 1) * 0.5 + 3.0 * 0.5
    assert np.all(C[0] == K * 0.5)


def test_w4a16_combine_weights_sum_to_one_on_workload_logits():
    for name in ("tiny_w4a16", "decode_w4a16", "prefill_w4a16", "moe_fp8"):
        wl = W.WORKLOADS[name]
        lg = W.router_logits(wl, min(wl.T, 512), wl.E).numpy()
        ids, w = oracle.route_topk(lg, wl.k)
        assert np.all(np.abs(w.astype(np.float64).sum(1) - 1.0) <= 1e-6)
        assert all(len(set(r)) == wl.k for r in ids.tolist())


# --------------------------------------------------------------------------------------------
# FP8
# --------------------------------------------------------------------------------------------

def test_fp8_act_quant_matches_torch_quantizer():
    rng = np.random.default_rng(5)
    x = torch.from_numpy(rng.normal(size=(37, 512)).astype(np.float32)).to(torch.bfloat16)
    x[3, :128] = 0.0                                  # all-zero group: scale 1e-10/448
    x[4, 128:256] = 1000.0
    q, s = oracle.fp8_act_quant(_bf16_bits(x))
    rq, rs = W.quantize_fp8_rows(x.float())
    assert np.array_equal(q, rq.numpy()) and np.array_equal(s, rs.numpy())


def test_fp8_closed_form_ones():
    K, N = 7168, 256
    a = np.full((2, K), 1.0, np.float32)
    q, s = oracle.fp8_act_quant(_bf16_bits(torch.from_numpy(a).to(torch.bfloat16)))
    assert np.all(q == 0x7E) and np.all(s == np.float32(1.0) / np.float32(448.0))
    B = np.full((N, K), 0x7E, np.uint8)
    Bs = np.full((N // 128, K // 128), np.float32(0.5) / np.float32(448.0), np.float32)
    C = oracle.fp8_block_matmul(q, s, B, Bs)
    assert np.all(np.abs(C - 0.5 * K) <= 1e-6 * 0.5 * K)


def test_fp8_block_scale_indexing():
    """One nonzero element per K block with power-of-two scales: C[m, n] = sum_kb
    As[m, kb] * Bs[n // 128, kb] exactly, which fails for any transposed or shifted scale index."""
    M, N, K = 3, 384, 512
    one = 0x38                                                   # E4M3 code of 1.0
    A = np.zeros((M, K), np.uint8)
    B = np.zeros((N, K), np.uint8)
    A[:, ::128] = one
    B[:, 5::128] = 0
    B[:, ::128] = one
    As = np.array([[2.0 ** (kb + 4 * m) for kb in range(K // 128)] for m in range(M)], np.float32)
    Bs = np.array([[2.0 ** (-2 * kb - 8 * nb) for kb in range(K // 128)] for nb in range(N // 128)], np.float32)
    C = oracle.fp8_block_matmul(A, As, B, Bs)
    for m in range(M):
        for n in (0, 127, 128, 300, 383):
            assert C[m, n] == sum(2.0 ** (kb + 4 * m) * 2.0 ** (-2 * kb - 8 * (n // 128)) for kb in range(K // 128))


def test_fp8_dense_matches_numpy_matmul():
    d = W.make_dense_fp8(W.WORKLOADS["dense_fp8"], 16, N=256, K=1024)
    A, As, B, Bs = (d[n].numpy() for n in ("A", "As", "B", "Bs"))
    C = oracle.fp8_block_matmul(A, As, B, Bs)
    Ad = torch.from_numpy(A).view(torch.float8_e4m3fn).double().numpy() * np.repeat(As, 128, 1)
    Bd = torch.from_numpy(B).view(torch.float8_e4m3fn).double().numpy() * np.repeat(np.repeat(Bs, 128, 0), 128, 1)
    ref = Ad @ Bd.T
    assert np.allclose(C, ref, rtol=1e-12, atol=1e-12)


def test_fp8_channel_matches_numpy_matmul():
    """Channelwise product against numpy float64 matmul of the torch-decoded E4M3 operands, the
    per-token scale on the rows and the per-channel scale on the columns."""
    d = W.make_dense_fp8_channel(W.WORKLOADS["dense_fp8_channel"], 24, N=384, K=640)
    A, As, B, Bs = (d[n].numpy() for n in ("A", "As", "B", "Bs"))
    assert As.shape == (24,) and Bs.shape == (384,)
    C = oracle.fp8_channel_matmul(A, As, B, Bs)
    Ad = torch.from_numpy(A).view(torch.float8_e4m3fn).double().numpy()
    Bd = torch.from_numpy(B).view(torch.float8_e4m3fn).double().numpy()
    ref = (Ad @ Bd.T) * As.astype(np.float64)[:, None] * Bs.astype(np.float64)[None, :]
    assert np.allclose(C, ref, rtol=1e-12, atol=1e-12)
    rows = np.array([23, 0, 7], np.int32)
    assert np.array_equal(oracle.fp8_channel_matmul(A, As, B, Bs, rows=rows), C[rows])


def test_fp8_channel_closed_form_and_scale_indexing():
    """All codes 448 (0x7E) with As[m] = 2^m / 448 and Bs[n] = 3^(n % 5) / 448: C[m, n] =
    K * 2^m * 3^(n % 5) exactly (M != N, so a transposed scale index cannot pass)."""
    M, N, K = 3, 10, 96
    A = np.full((M, K), 0x7E, np.uint8)
    B = np.full((N, K), 0x7E, np.uint8)
    As = np.array([2.0 ** m / 448.0 for m in range(M)], np.float32)
    Bs = np.array([3.0 ** (n % 5) / 448.0 for n in range(N)], np.float32)
    C = oracle.fp8_channel_matmul(A, As, B, Bs)
    for m in range(M):
        for n in range(N):
            assert C[m, n] == pytest.approx(K * 2.0 ** m * 3.0 ** (n % 5), rel=1e-6)
    # one code of -1.5 (0xBC) in row 1 of A at column 5 against 2.0 (0x40) in channel 7
    A2 = np.zeros((M, K), np.uint8)
    B2 = np.zeros((N, K), np.uint8)
    A2[1, 5], B2[7, 5] = 0xBC, 0x40
    ones = np.ones(M, np.float32), np.ones(N, np.float32)
    C2 = oracle.fp8_channel_matmul(A2, ones[0], B2, ones[1])
    assert C2[1, 7] == -3.0 and np.count_nonzero(C2) == 1


def test_fp8_channel_equals_block_when_scales_are_constant_per_block():
    """With As constant along K and Bs constant over each 128-row block, the channelwise and the
    block-scaled definitions describe the same product: the two oracle functions agree."""
    d = W.make_dense_fp8_channel(W.WORKLOADS["dense_fp8_channel"], 5, N=256, K=384)
    A, As, B = d["A"].numpy(), d["As"].numpy(), d["B"].numpy()
    Bs_blk = np.array([0.25, 3.0], np.float32)
    Bs = np.repeat(Bs_blk, 128)
    C = oracle.fp8_channel_matmul(A, As, B, Bs)
    Cb = oracle.fp8_block_matmul(A, np.repeat(As[:, None], 3, 1), B, np.repeat(Bs_blk[:, None], 3, 1))
    assert np.allclose(C, Cb, rtol=1e-12, atol=1e-12)


# ---- MXFP4 (E2M1 codes, UE8M0 group-32 scales) ------------------------------------------------

def _e2m1_via_e4m3(codes):
    """E2M1 code -> value through torch's E4M3 decoder: every E2M1 value is an E4M3 value with the
    same sign, exponent + 6 (bias 1 -> 7) and the mantissa bit moved to the top of three; the
    E2M1 subnormal 0.5 is the E4M3 normal 2^-1 (code 0x30) and 0 is 0."""
    codes = np.asarray(codes, np.uint8) & 15
    e, m, sg = (codes >> 1) & 3, codes & 1, codes >> 3
    e4 = np.where(e > 0, (sg << 7) | ((e + 6) << 3) | (m << 2), np.where(m == 1, (sg << 7) | 0x30, sg << 7))
    return torch.from_numpy(e4.astype(np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def _mxfp4_numpy_dequant(q, s):
    """numpy unpack of int32 words (nibble j = input 8w + j) times 2^(s - 127) per 32 inputs."""
    q = np.asarray(q).view(np.uint32)
    N, K8 = q.shape
    codes = ((q[:, :, None] >> (4 * np.arange(8, dtype=np.uint32))) & 15).reshape(N, K8 * 8)
    return _e2m1_via_e4m3(codes) * np.ldexp(1.0, np.repeat(s.astype(np.int64), 32, 1) - 127)


def test_e2m1_all_codes_match_e4m3_route():
    c = np.arange(16, dtype=np.uint8)
    assert np.array_equal(oracle.e2m1_value(c), _e2m1_via_e4m3(c))
    assert list(oracle.e2m1_value(c[:8])) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]


def test_mxfp4_dequant_hand_worked_and_numpy():
    """Row 0: input 0 code 0x1 (0.5), input 9 code 0xF (-6), input 33 code 0x3 (1.5) with group
    scales 2^(125-127) and 2^(130-127): -> 0.125, -1.5, 12.0; everything else code 0 -> 0."""
    q = np.zeros((2, 8), np.uint32)
    q[0, 0] = 0x1                      # input 0, nibble 0
    q[0, 1] = 0xF << 4                 # input 9 = word 1, nibble 1
    q[0, 4] = 0x3 << 4                 # input 33 = word 4, nibble 1
    s = np.array([[125, 130], [0, 254]], np.uint8)
    deq = oracle.mxfp4_dequant(q.view(np.int32), s)
    want = np.zeros((2, 64))
    want[0, 0], want[0, 9], want[0, 33] = 0.125, -1.5, 12.0
    assert np.array_equal(deq, want)
    d = W.make_moe(W.WORKLOADS["decode_mxfp4"], T=2, E=2, k=1, H=256, I=128)
    for e in range(2):
        qq, ss = W.np_bits(d["w13q"][e]), W.np_bits(d["w13s"][e])
        assert np.array_equal(oracle.mxfp4_dequant(qq, ss), _mxfp4_numpy_dequant(qq, ss))


def test_mxfp4_layer_equals_int4_layer_on_integer_weights():
    """Weights whose MXFP4 values are the integers -6..6 (scale 2^0) written also as INT4 codes
    q = value + 8 with bf16 scale 1: the MXFP4 and the INT4 layer oracles agree exactly."""
    T, E, k, H, I = 3, 3, 2, 64, 32
    rng = np.random.default_rng(5)
    vals = np.array([0, 1, 2, 3, 4, 6, -1, -2, -3, -4, -6])
    code_of = {0: 0, 1: 2, 2: 4, 3: 5, 4: 6, 6: 7, -1: 10, -2: 12, -3: 13, -4: 14, -6: 15}

    def pack(v, table):
        c = np.vectorize(table.__getitem__)(v).astype(np.uint32)
        N, K = c.shape
        return (c.reshape(N, K // 8, 8) << (4 * np.arange(8, dtype=np.uint32))).sum(-1).astype(np.uint32).view(np.int32)

    v13 = rng.choice(vals, size=(E, 2 * I, H))
    v2 = rng.choice(vals, size=(E, H, I))
    fp4 = lambda v: np.stack([pack(x, code_of) for x in v])
    int4 = lambda v: np.stack([pack(x, {u: u + 8 for u in vals}) for x in v])
    one = 0x3F80
    x = torch.randn(T, H).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    a = oracle.moe_mxfp4(x, logits, k, fp4(v13), np.full((E, 2 * I, H // 32), 127, np.uint8), fp4(v2),
                         np.full((E, H, I // 32), 127, np.uint8))
    b = oracle.moe_w4a16(x, logits, k, int4(v13), np.full((E, 2 * I, H // 32), one, np.uint16), int4(v2),
                         np.full((E, H, I // 32), one, np.uint16))
    assert np.array_equal(a, b)


def test_mxfp4_layer_dense_equivalence_with_uniform_routing():
    """k = E, equal logits: out = (1/E) sum_e FFN_e(x), FFN_e from numpy float64 matmul on the
    torch/numpy-decoded weights and a torch-rounded bf16 intermediate."""
    T, E, H, I = 3, 4, 128, 64
    d = W.make_moe(W.WORKLOADS["decode_mxfp4"], T=T, E=E, k=E, H=H, I=I)
    x = W.np_bits(d["x"])
    w13q, w13s, w2q, w2s = (W.np_bits(d[n]) for n in ("w13q", "w13s", "w2q", "w2s"))
    logits = np.zeros((T, E), np.float32)
    out = oracle.moe_mxfp4(x, logits, E, w13q, w13s, w2q, w2s)
    xd = d["x"].double().numpy()
    ref = np.zeros_like(out)
    for e in range(E):
        w13 = _mxfp4_numpy_dequant(w13q[e], w13s[e])
        g, u = xd @ w13[:I].T, xd @ w13[I:].T
        h = torch.from_numpy(g / (1 + np.exp(-g)) * u).to(torch.bfloat16).double().numpy()
        ref += 0.25 * (h @ _mxfp4_numpy_dequant(w2q[e], w2s[e]).T)
    assert np.allclose(out, ref, rtol=1e-9, atol=1e-12)


# ---- NVFP4 (E2M1 codes, E4M3 group-16 scales, f32 tensor scale) -------------------------------

def _nvfp4_numpy_dequant(q, s, g):
    q = np.asarray(q).view(np.uint32)
    N, K8 = q.shape
    codes = ((q[:, :, None] >> (4 * np.arange(8, dtype=np.uint32))) & 15).reshape(N, K8 * 8)
    sv = torch.from_numpy(np.ascontiguousarray(s)).view(torch.float8_e4m3fn).double().numpy()
    return _e2m1_via_e4m3(codes) * np.repeat(sv, 16, 1) * float(g)


def test_nvfp4_dequant_hand_worked_and_numpy():
    """Input 0 code 0x2 (1.0) with scale 0x40 (2.0), input 17 code 0xB (-1.5) with 0x30 (0.5), input
    40 code 0x7 (6.0) with 0x2C (0.375), tensor scale 0.5: 1.0, -0.375, 1.125 (group = input / 16)."""
    q = np.zeros((1, 8), np.uint32)
    q[0, 0] = 0x2
    q[0, 2] = 0xB << 4                 # input 17 = word 2, nibble 1
    q[0, 5] = 0x7                      # input 40 = word 5, nibble 0
    s = np.array([[0x40, 0x30, 0x2C, 0x38]], np.uint8)
    deq = oracle.nvfp4_dequant(q.view(np.int32), s, 0.5)
    want = np.zeros((1, 64))
    want[0, 0], want[0, 17], want[0, 40] = 1.0, -0.375, 1.125
    assert np.array_equal(deq, want)
    d = W.make_moe(W.WORKLOADS["decode_nvfp4"], T=2, E=2, k=1, H=256, I=128)
    for e in range(2):
        qq, ss, gg = W.np_bits(d["w13q"][e]), W.np_bits(d["w13s"][e]), float(d["g13"][e])
        assert np.array_equal(oracle.nvfp4_dequant(qq, ss, gg), _nvfp4_numpy_dequant(qq, ss, gg))


def test_nvfp4_layer_equals_mxfp4_layer_on_power_of_two_scales():
    """E4M3 scales that are powers of two, equal over each 32 inputs, and tensor scales of 1: the
    NVFP4 layer is the MXFP4 layer with UE8M0 codes log2(scale) + 127."""
    T, E, k, H, I = 3, 3, 2, 64, 32
    rng = np.random.default_rng(9)
    q13 = rng.integers(0, 2 ** 31, size=(E, 2 * I, H // 8), dtype=np.int64).astype(np.uint32).view(np.int32)
    q2 = rng.integers(0, 2 ** 31, size=(E, H, I // 8), dtype=np.int64).astype(np.uint32).view(np.int32)
    p13 = rng.integers(-4, 3, size=(E, 2 * I, H // 32))
    p2 = rng.integers(-4, 3, size=(E, H, I // 32))
    e4m3_of = lambda p: ((p + 7) << 3).astype(np.uint8)           # 2^p, p in [-6, 8]
    n13, n2 = np.repeat(e4m3_of(p13), 2, -1), np.repeat(e4m3_of(p2), 2, -1)
    m13, m2 = (p13 + 127).astype(np.uint8), (p2 + 127).astype(np.uint8)
    x = torch.randn(T, H).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    ones = np.ones(E, np.float32)
    a = oracle.moe_nvfp4(x, logits, k, q13, n13, ones, q2, n2, ones)
    b = oracle.moe_mxfp4(x, logits, k, q13, m13, q2, m2)
    assert np.array_equal(a, b)


def test_nvfp4_layer_dense_equivalence_with_uniform_routing():
    T, E, H, I = 3, 4, 128, 64
    d = W.make_moe(W.WORKLOADS["decode_nvfp4"], T=T, E=E, k=E, H=H, I=I)
    x = W.np_bits(d["x"])
    q13, s13, q2, s2 = (W.np_bits(d[n]) for n in ("w13q", "w13s", "w2q", "w2s"))
    g13, g2 = d["g13"].numpy(), d["g2"].numpy()
    out = oracle.moe_nvfp4(x, np.zeros((T, E), np.float32), E, q13, s13, g13, q2, s2, g2)
    xd = d["x"].double().numpy()
    ref = np.zeros_like(out)
    for e in range(E):
        w13 = _nvfp4_numpy_dequant(q13[e], s13[e], g13[e])
        g, u = xd @ w13[:I].T, xd @ w13[I:].T
        h = torch.from_numpy(g / (1 + np.exp(-g)) * u).to(torch.bfloat16).double().numpy()
        ref += 0.25 * (h @ _nvfp4_numpy_dequant(q2[e], s2[e], g2[e]).T)
    assert np.allclose(out, ref, rtol=1e-9, atol=1e-12)


def _torch_fp8_rows(v32):
    q, s = W.quantize_fp8_rows(torch.from_numpy(np.ascontiguousarray(v32)))
    return q.numpy(), s.numpy()


def test_fp8_moe_dense_equivalence_with_uniform_routing():
    """k = E, equal logits: out = (1/E) sum_e FFN_e(x) with FFN_e from numpy float64 matmul on
    decoded E4M3 weights and a torch-quantized intermediate."""
    T, E, H, I = 3, 4, 256, 256
    d = W.make_moe(W.WORKLOADS["moe_fp8"], T=T, E=E, k=E, H=H, I=I)
    x = W.np_bits(d["x"])
    w13, w13s, w2, w2s = (W.np_bits(d[n]) for n in ("w13", "w13s", "w2", "w2s"))
    logits = np.zeros((T, E), np.float32)
    out, hq, hs = oracle.moe_fp8(x, logits, E, w13, w13s, w2, w2s, want_h=True)
    xq, xs = _torch_fp8_rows(d["x"].float().numpy())

    def deq(q, s, bn=128):
        v = torch.from_numpy(q).view(torch.float8_e4m3fn).double().numpy()
        return v * np.repeat(np.repeat(s, bn, 0), 128, 1)

    xd = torch.from_numpy(xq).view(torch.float8_e4m3fn).double().numpy() * np.repeat(xs, 128, 1)
    ref = np.zeros_like(out)
    for e in range(E):
        g = xd @ deq(w13[e, :I], w13s[e, :I // 128]).T
        u = xd @ deq(w13[e, I:], w13s[e, I // 128:]).T
        a = (g / (1 + np.exp(-g)) * u).astype(np.float32)
        q2, s2 = _torch_fp8_rows(a)
        # g and u agree with the oracle's to a few double ulps, so the f32 intermediate and its
        # codes and scales agree exactly (a flip would need a double within ~1e-16 of an f32
        # rounding boundary)
        assert np.array_equal(hq[:, e, :], q2) and np.array_equal(hs[:, e, :], s2)
        hd = torch.from_numpy(hq[:, e, :].copy()).view(torch.float8_e4m3fn).double().numpy() * np.repeat(hs[:, e, :], 128, 1)
        ref += 0.25 * (hd @ deq(w2[e], w2s[e]).T)
    assert np.allclose(out, ref, rtol=1e-10, atol=1e-12)
