"""Helpers shared by the GPU parity tests: input synthesis on the device, host copies for the
oracle, and the layer tolerance check."""
from __future__ import annotations

import numpy as np
import torch

import workloads as W

# Layer-output tolerances: |gpu - ref| <= tol * (|ref| + rms(ref)), element-wise.
TOL_W4A16 = 2e-2
TOL_FP8 = 3e-2


def assert_layer_close(gpu: np.ndarray, ref: np.ndarray, tol: float, what: str = "", rms: float | None = None):
    """rms: the output scale of the bound (default: rms of ref). A share of the layer (one rank's
    experts) passes the layer's own output rms on the same rows: its errors are those of its slots,
    and its value may be a small part of the layer's."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite GPU output"
    rms = float(np.sqrt(np.mean(ref ** 2))) if rms is None else float(rms)
    err = np.abs(gpu - ref)
    bound = tol * (np.abs(ref) + rms)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err / bound), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} elements out of tolerance; worst at {i}: "
                             f"gpu={gpu[i]!r} ref={ref[i]!r} bound={bound[i]!r} (rms {rms:.3g})")


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def host_moe_weights(d: dict, experts) -> dict:
    """Host numpy copies of the weights of the given experts, laid out full-size (untouched
    experts stay zero pages) so the oracle can index them by expert id."""
    out = {}
    names = ("w13q", "w13s", "w2q", "w2s") if d["kind"] == "w4a16" else ("w13", "w13s", "w2", "w2s")
    for n in names:
        t = d[n]
        np_dtype = {torch.int32: np.int32, torch.bfloat16: np.uint16, torch.uint8: np.uint8,
                    torch.float32: np.float32}[t.dtype]
        arr = np.zeros(tuple(t.shape), np_dtype)
        for e in sorted(set(int(v) for v in experts)):
            arr[e] = W.np_bits(t[e])
        out[n] = arr
    return out


def oracle_layer(d: dict, tokens, want_h=False):
    """Oracle output rows for `tokens` of a generated MoE workload (float64 [len(tokens), H])."""
    import oracle
    x = W.np_bits(d["x"])
    logits = W.np_bits(d["logits"])
    ids, _ = oracle.route_topk(logits[np.asarray(tokens)], d["k"])
    hw = host_moe_weights(d, ids.ravel())
    if d["kind"] == "w4a16":
        return oracle.moe_w4a16(x, logits, d["k"], hw["w13q"], hw["w13s"], hw["w2q"], hw["w2s"], tokens=tokens,
                                want_h=want_h)
    return oracle.moe_fp8(x, logits, d["k"], hw["w13"], hw["w13s"], hw["w2"], hw["w2s"], tokens=tokens,
                          want_h=want_h)


def sample_tokens(d: dict, n: int, seed: int = 0) -> np.ndarray:
    """Seeded token sample that includes the first and last token and tokens routed to the most
    and least loaded experts."""
    import oracle
    T = d["T"]
    if T <= n:
        return np.arange(T, dtype=np.int32)
    logits = W.np_bits(d["logits"])
    ids, _ = oracle.route_topk(logits, d["k"])
    counts = np.bincount(ids.ravel(), minlength=d["E"])
    heavy = int(np.argmax(counts))
    light = int(np.argmin(np.where(counts > 0, counts, 1 << 30)))
    pick = {0, T - 1}
    pick.add(int(np.nonzero((ids == heavy).any(1))[0][0]))
    pick.add(int(np.nonzero((ids == light).any(1))[0][0]))
    rng = np.random.default_rng(seed)
    while len(pick) < n:
        pick.add(int(rng.integers(0, T)))
    return np.array(sorted(pick), dtype=np.int32)


def block_tokens(d: dict, block_m: int, small_rows: int = 0, n_sampled: int = 0, seed: int = 0) -> np.ndarray:
    """Tokens whose outputs run through chosen blocks of the aligned routing (the oracle's routing
    and alignment): every token of the most loaded expert's first and last block_m-row block, every
    token of one block with at most `small_rows` real rows (the few-row tail), and n_sampled more
    tokens from the seeded sample."""
    import oracle
    logits = W.np_bits(d["logits"])
    ids, _ = oracle.route_topk(logits, d["k"])
    sorted_ids, expert_ids, ntp = oracle.align(ids, d["E"], block_m)
    n_slots = ids.size
    counts = np.bincount(ids.ravel(), minlength=d["E"])
    heavy = int(np.argmax(counts))
    blocks = [b for b in range(ntp // block_m) if expert_ids[b] == heavy]
    pick = set()
    for b in (blocks[0], blocks[-1]):
        rows = sorted_ids[b * block_m:(b + 1) * block_m]
        pick.update(int(s) // d["k"] for s in rows if s < n_slots)
    if small_rows:
        for b in range(ntp // block_m):
            rows = sorted_ids[b * block_m:(b + 1) * block_m]
            real = rows[rows < n_slots]
            if 0 < real.size <= small_rows:
                pick.update(int(s) // d["k"] for s in real)
                break
    if n_sampled:
        pick.update(int(t) for t in sample_tokens(d, n_sampled, seed))
    return np.array(sorted(pick), dtype=np.int32)
