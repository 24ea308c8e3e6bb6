"""Expert- and tensor-parallel sharding on the CPU: the oracle's expert-parallel share pinned to its
whole layer, the weight slicing of the sharding module checked through the oracle (the ranks'
shares must sum to the unsharded layer), and the sum over ranks run as a world_size-2 gloo group."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import workloads as W
from quantized_mixture_experts_align_b200 import sharding as S

KINDS = {"w4a16": "tiny_w4a16", "mxfp4": "decode_mxfp4", "nvfp4": "decode_nvfp4", "fp8": "moe_fp8"}


def _layer(kind, T=6, E=6, k=2, H=128, I=256):
    return W.make_moe(W.WORKLOADS[KINDS[kind]], T=T, E=E, k=k, H=H, I=I)


def _host(d, kind):
    """The weights as the oracle takes them, keyed as the sharding module names them (the oracle
    reads the raw MXFP4 / NVFP4 scale bytes where the GPU path reads prepacked factors: same layout)."""
    if kind == "fp8":
        return {n: W.np_bits(d[n]) for n in ("w13", "w13s", "w2", "w2s")}
    w = {"w13q": W.np_bits(d["w13q"]), "w2q": W.np_bits(d["w2q"])}
    f = "w13s" if kind == "w4a16" else "w13f"
    w[f] = W.np_bits(d["w13s"])
    w[f.replace("13", "2")] = W.np_bits(d["w2s"])
    if kind == "nvfp4":
        w.update(g13=W.np_bits(d["g13"]), g2=W.np_bits(d["g2"]))
    return w


def _oracle_full(d, kind, w):
    x, lg, k = W.np_bits(d["x"]), W.np_bits(d["logits"]), d["k"]
    if kind == "fp8":
        return oracle.moe_fp8(x, lg, k, w["w13"], w["w13s"], w["w2"], w["w2s"])
    if kind == "nvfp4":
        return oracle.moe_nvfp4(x, lg, k, w["w13q"], w["w13f"], w["g13"], w["w2q"], w["w2f"], w["g2"])
    if kind == "mxfp4":
        return oracle.moe_mxfp4(x, lg, k, w["w13q"], w["w13f"], w["w2q"], w["w2f"])
    return oracle.moe_w4a16(x, lg, k, w["w13q"], w["w13s"], w["w2q"], w["w2s"])


def _oracle_ep(d, kind, w, base):
    x, lg, k = W.np_bits(d["x"]), W.np_bits(d["logits"]), d["k"]
    if kind == "fp8":
        return oracle.moe_fp8_ep(x, lg, k, base, w["w13"], w["w13s"], w["w2"], w["w2s"])
    if kind == "nvfp4":
        return oracle.moe_q4_ep("nvfp4", x, lg, k, base, w["w13q"], w["w13f"], w["w2q"], w["w2f"], w["g13"], w["g2"])
    if kind == "mxfp4":
        return oracle.moe_q4_ep("mxfp4", x, lg, k, base, w["w13q"], w["w13f"], w["w2q"], w["w2f"])
    return oracle.moe_q4_ep("w4a16", x, lg, k, base, w["w13q"], w["w13s"], w["w2q"], w["w2s"])


def _shard_np(w, kind, fn, *a):
    t = {n: torch.from_numpy(np.ascontiguousarray(v)) for n, v in w.items()}
    r = fn(t, kind, *a)
    if isinstance(r, tuple):
        return ({n: v.numpy() for n, v in r[0].items()},) + r[1:]
    return {n: v.numpy() for n, v in r.items()}


def test_expert_range_tiles_experts():
    for E, N in [(384, 8), (384, 16), (10, 3), (7, 7), (256, 32)]:
        ranges = [S.expert_range(E, r, N) for r in range(N)]
        assert ranges[0][0] == 0 and sum(n for _, n in ranges) == E
        assert all(b1 == b0 + n0 for (b0, n0), (b1, _) in zip(ranges, ranges[1:]))
        assert max(n for _, n in ranges) - min(n for _, n in ranges) <= 1
    with pytest.raises(ValueError):
        S.expert_range(4, 0, 5)


@pytest.mark.parametrize("kind", list(KINDS))
def test_oracle_ep_whole_range_is_the_layer(kind):
    """orc_moe_q4_ep / orc_moe_fp8_ep with every expert held are the layer, bit for bit."""
    d = _layer(kind)
    w = _host(d, kind)
    assert np.array_equal(_oracle_ep(d, kind, w, 0), _oracle_full(d, kind, w))


@pytest.mark.parametrize("kind", list(KINDS))
@pytest.mark.parametrize("world", [2, 4])
def test_oracle_ep_shares_sum_to_the_layer(kind, world):
    """The ranks' shares (uneven ranges at world 4 over 6 experts) add up to the whole layer; each
    share holds only its experts' slots (a share over experts no token picked is zero)."""
    d = _layer(kind)
    w = _host(d, kind)
    full = _oracle_full(d, kind, w)
    ids, _ = oracle.route_topk(W.np_bits(d["logits"]), d["k"])
    total = np.zeros_like(full)
    for r in range(world):
        ws, base, local = _shard_np(w, kind, S.shard_experts, r, world)
        part = _oracle_ep(d, kind, ws, base)
        mine = ((ids >= base) & (ids < base + local)).any(1)
        assert np.all(part[~mine] == 0.0)
        total += part
    np.testing.assert_allclose(total, full, rtol=1e-12, atol=1e-12 * np.abs(full).max())


def test_oracle_ep_share_with_no_routed_slot_is_zero():
    d = _layer("w4a16")
    lg = torch.full((d["T"], d["E"]), -5.0)
    lg[:, 0], lg[:, 1] = 3.0, 2.0                    # every token picks experts 0 and 1
    d["logits"] = lg
    w = _host(d, "w4a16")
    ws, base, _ = _shard_np(w, "w4a16", S.shard_experts, 1, 2)   # experts 3..5
    assert np.all(_oracle_ep(d, "w4a16", ws, base) == 0.0)


@pytest.mark.parametrize("kind", list(KINDS))
def test_tp_slices_sum_to_the_layer(kind):
    """shard_intermediate's gate / up / down slices: the oracle on each rank's slice, summed over
    ranks, is the unsharded layer (SiLU(gate) * up is per feature, the down product sums over
    features)."""
    d = _layer(kind, I=256)
    w = _host(d, kind)
    full = _oracle_full(d, kind, w)
    total = np.zeros_like(full)
    for r in range(2):
        total += _oracle_full(d, kind, _shard_np(w, kind, S.shard_intermediate, 256, r, 2))
    np.testing.assert_allclose(total, full, rtol=1e-12, atol=1e-12 * np.abs(full).max())


def test_tp_slice_rejects_unaligned_split():
    d = _layer("w4a16", I=256)
    w = {n: d[n] for n in ("w13q", "w13s", "w2q", "w2s")}
    with pytest.raises(ValueError):
        S.shard_intermediate(w, "w4a16", 256, 0, 4)      # 64 features per rank


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    d = _layer("w4a16")
    w = _host(d, "w4a16")
    ws, base, _ = _shard_np(w, "w4a16", S.shard_experts, rank, world)
    ep = torch.from_numpy(_oracle_ep(d, "w4a16", ws, base))
    tp = torch.from_numpy(_oracle_full(d, "w4a16", _shard_np(w, "w4a16", S.shard_intermediate, 256, rank, world)))
    S.reduce_partial(ep)
    S.reduce_partial(tp)
    q.put((rank, ep.numpy(), tp.numpy()))
    dist.destroy_process_group()


def test_ep_and_tp_sum_over_a_gloo_group():
    """Each rank of a world_size-2 gloo group computes its EP share and its TP share; after
    reduce_partial every rank holds the whole layer."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    d = _layer("w4a16")
    full = _oracle_full(d, "w4a16", _host(d, "w4a16"))
    for _, ep, tp in res:
        np.testing.assert_allclose(ep, full, rtol=1e-12, atol=1e-12 * np.abs(full).max())
        np.testing.assert_allclose(tp, full, rtol=1e-12, atol=1e-12 * np.abs(full).max())
