"""Expert- and tensor-parallel execution of the routed layer, one process per GPU.

"vLLM x Novita AI: Chord W4A16 INT4 MoE Kernel for Kimi K2.x", "Other deployment details" and the
measured results, runs the layer as EP8 / EP16 / EP32 (each GPU holds E / N of the experts) and as
TP8 (each GPU holds a slice of every expert's intermediate features). This layer's output is
linear in both the experts' contributions and the intermediate features:

  * EP: out = sum over ranks of out_r, out_r summing only the slots routed to rank r's experts
    (``moe_*_forward_ep``: the routing still ranks all E experts, on every rank);
  * TP: rank r holds features [r I/N, (r+1) I/N) of every expert: those gate rows, those up rows,
    those down columns and their scales; SiLU(gate) * up is per feature, so the single-GPU forward
    on the slice gives out_r, and out = sum over ranks of out_r.

Each rank therefore runs one library call on its own weights, then one all-reduce (sum) of the
[T, H] bf16 output over the process group (NCCL over NVLink on GPUs). The sharding helpers only
slice tensors; every step of the layer runs in the library's kernels.
"""
from __future__ import annotations

import torch

import quantized_mixture_experts_align_b200 as M

# weight tensors of each format: (gate/up tensors [E, 2I * r, ...], down tensors [E, H * r, I * c])
_W13 = {"w4a16": ("w13q", "w13s"), "mxfp4": ("w13q", "w13f"), "nvfp4": ("w13q", "w13f"), "fp8": ("w13", "w13s")}
_W2 = {"w4a16": ("w2q", "w2s"), "mxfp4": ("w2q", "w2f"), "nvfp4": ("w2q", "w2f"), "fp8": ("w2", "w2s")}
_PER_EXPERT = {"nvfp4": ("g13", "g2")}  # per-expert scalars, unchanged by a feature slice


def expert_range(E: int, rank: int, world: int) -> tuple[int, int]:
    """(ep_base, ep_local) of rank `rank`: contiguous ranges that tile [0, E), sizes differing by at
    most one."""
    if not 0 <= rank < world or world > E:
        raise ValueError(f"expert_range: need 0 <= rank < world <= E (rank={rank}, world={world}, E={E})")
    lo, hi = rank * E // world, (rank + 1) * E // world
    return lo, hi - lo


def shard_experts(weights: dict, kind: str, rank: int, world: int) -> tuple[dict, int, int]:
    """Rank `rank`'s experts of the layer weights (every tensor sliced along its expert axis).
    Returns (weights of experts [ep_base, ep_base + ep_local), ep_base, ep_local)."""
    names = _W13[kind] + _W2[kind] + _PER_EXPERT.get(kind, ())
    E = weights[names[0]].shape[0]
    base, local = expert_range(E, rank, world)
    return {n: weights[n][base:base + local].contiguous() for n in names}, base, local


def _feature_slice_rows(t: torch.Tensor, rank: int, world: int) -> torch.Tensor:
    """Gate/up tensor [E, 2R, ...]: rows [r R/N, (r+1) R/N) of the gate half and of the up half,
    gate first (the fused layout the kernels read)."""
    R = t.shape[1] // 2
    if t.shape[1] != 2 * R or R % world:
        raise ValueError(f"gate/up tensor of {t.shape[1]} rows does not split over {world} ranks")
    n = R // world
    return torch.cat([t[:, rank * n:(rank + 1) * n], t[:, R + rank * n:R + (rank + 1) * n]], dim=1).contiguous()


def _feature_slice_cols(t: torch.Tensor, rank: int, world: int) -> torch.Tensor:
    """Down tensor [E, rows, C]: columns [r C/N, (r+1) C/N) (codes, scales or factors: each is laid
    out along I in the same order, so one fraction of its columns is one feature range)."""
    C = t.shape[-1]
    if C % world:
        raise ValueError(f"down tensor of {C} columns does not split over {world} ranks")
    n = C // world
    return t[..., rank * n:(rank + 1) * n].contiguous()


def shard_intermediate(weights: dict, kind: str, I: int, rank: int, world: int) -> dict:
    """Rank `rank`'s intermediate features [r I/N, (r+1) I/N) of every expert. I / N must be a
    multiple of 128 (the kernels' feature tile and the FP8 scale block)."""
    if I % world or (I // world) % 128:
        raise ValueError(f"I / world must be a multiple of 128 (I={I}, world={world})")
    out = {n: _feature_slice_rows(weights[n], rank, world) for n in _W13[kind]}
    out.update({n: _feature_slice_cols(weights[n], rank, world) for n in _W2[kind]})
    out.update({n: weights[n] for n in _PER_EXPERT.get(kind, ())})
    return out


def reduce_partial(out: torch.Tensor, group=None) -> torch.Tensor:
    """Sum of the ranks' partial outputs, in place (all-reduce over `group`; a no-op alone)."""
    if torch.distributed.is_available() and torch.distributed.is_initialized() and \
            torch.distributed.get_world_size(group) > 1:
        torch.distributed.all_reduce(out, op=torch.distributed.ReduceOp.SUM, group=group)
    return out


def forward_ep_partial(kind: str, x, logits, k: int, w: dict, ep_base: int, **kw):
    """This rank's share out_r of the layer (no reduction): `w` holds the weights of experts
    [ep_base, ep_base + ep_local) in the layout of the single-GPU forward of format `kind`
    ("w4a16", "mxfp4" with prepacked factors w13f / w2f, "nvfp4" with w13f / w2f / g13 / g2, "fp8")."""
    if kind == "fp8":
        return M.moe_w8a8_block_fp8_forward_ep(x, logits, k, ep_base, w["w13"], w["w13s"], w["w2"], w["w2s"], **kw)
    if kind == "nvfp4":
        return M.moe_nvfp4_forward_ep(x, logits, k, ep_base, w["w13q"], w["w13f"], w["g13"], w["w2q"], w["w2f"],
                                      w["g2"], **kw)
    if kind == "mxfp4":
        return M.moe_mxfp4_forward_ep(x, logits, k, ep_base, w["w13q"], w["w13f"], w["w2q"], w["w2f"], **kw)
    return M.moe_w4a16_forward_ep(x, logits, k, ep_base, w["w13q"], w["w13s"], w["w2q"], w["w2s"], **kw)


def forward_ep(kind: str, x, logits, k: int, w: dict, ep_base: int, group=None, **kw):
    """The layer's output on every rank of an expert-parallel group: this rank's share, then the
    all-reduce (sum) over the group."""
    return reduce_partial(forward_ep_partial(kind, x, logits, k, w, ep_base, **kw), group)


def forward_tp_partial(kind: str, x, logits, k: int, w: dict, **kw):
    """This rank's share out_r under tensor parallelism: the single-GPU forward on the rank's
    feature slice (from shard_intermediate)."""
    if kind == "fp8":
        return M.moe_w8a8_block_fp8_forward(x, logits, k, w["w13"], w["w13s"], w["w2"], w["w2s"], **kw)
    if kind == "nvfp4":
        return M.moe_nvfp4_forward(x, logits, k, w["w13q"], w["w13f"], w["g13"], w["w2q"], w["w2f"], w["g2"], **kw)
    if kind == "mxfp4":
        return M.moe_mxfp4_forward(x, logits, k, w["w13q"], w["w13f"], w["w2q"], w["w2f"], **kw)
    return M.moe_w4a16_forward(x, logits, k, w["w13q"], w["w13s"], w["w2q"], w["w2s"], **kw)


def forward_tp(kind: str, x, logits, k: int, w: dict, group=None, **kw):
    """The layer's output on every rank of a tensor-parallel group."""
    return reduce_partial(forward_tp_partial(kind, x, logits, k, w, **kw), group)
