"""Expert parallelism: the layer's routed experts split over the ranks of a process group.

One process per GPU, ``torch.distributed`` for the exchanges (NCCL between GPUs). Rank r
of ``world`` owns the routed experts ``owned_experts(E_r, world, r)`` plus a copy of the
shared expert, which serves its own rank's tokens. A forward on this rank's tokens:

  1. route its tokens (the library's route kernel);
  2. dispatch (``moe_ep_dispatch``): the (token, slot) pairs sorted stably by owner rank,
     each owner's segment padded to 16 rows, packed as hidden rows + owner-local expert id
     + routing weight;
  3. exchange segment sizes, then the rows, ids and weights (all-to-all);
  4. the owners run their experts on what they received: the routed forward with one slot
     per row, which returns each row times its weight (bf16);
  5. the reverse all-to-all brings the weighted rows back in send order;
  6. combine (``moe_ep_combine``): each token's k' rows summed in slot order in fp32,
     rounded once to bf16.

Only the exchanges (and the host copy of the segment sizes they need) are in Python; every
other step is a library kernel. The exchanges go through ``all_to_all_single`` on byte views
of the rows, so any backend that moves uint8, int32 and fp32 tensors carries them.

The steps that compute are methods of a backend object; :class:`GpuBackend` runs the
library. A test may pass its own backend to run the same orchestration elsewhere.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import List, Optional, Tuple

import torch

from . import (_ptr, _stream, check, lib, make_problem, moe_forward_routed, prepare_weights, read_workspace,
               stage_route)

__all__ = ["owned_experts", "local_expert_weights", "prepare_local_weights", "EpDispatch", "GpuBackend",
           "ep_moe_forward"]


def owned_experts(num_routed: int, world: int, rank: int) -> range:
    """Routed experts of ``rank``: a contiguous range of ``num_routed / world``."""
    if world < 1 or num_routed % world != 0 or not 0 <= rank < world:
        raise ValueError("the routed experts must split evenly over the ranks")
    n = num_routed // world
    return range(rank * n, (rank + 1) * n)


def local_expert_weights(w13: torch.Tensor, w2: torch.Tensor, num_routed: int, num_shared: int, world: int,
                         rank: int) -> Tuple[torch.Tensor, torch.Tensor]:
    """This rank's experts out of checkpoint-layout [E, ...] weights: its routed range, then
    the shared expert (local id num_routed / world)."""
    idx = list(owned_experts(num_routed, world, rank)) + list(range(num_routed, num_routed + num_shared))
    sel = torch.tensor(idx, device=w13.device)
    return w13.index_select(0, sel).contiguous(), w2.index_select(0, sel.to(w2.device)).contiguous()


@dataclass
class EpDispatch:
    send_rows: torch.Tensor         # [max_send, H] bf16
    send_expert: torch.Tensor       # [max_send] int32, owner-local ids
    send_weight: torch.Tensor       # [max_send] fp32
    send_counts: List[int]          # rows of each destination rank's segment
    pair_to_send_row: torch.Tensor  # [T * k'] int32


class GpuBackend:
    """The library's kernels on the current CUDA device."""

    def __init__(self):
        self._ws = {}

    @property
    def comm_device(self):
        return torch.device("cuda", torch.cuda.current_device())

    def _workspace(self, key, nbytes: int) -> torch.Tensor:
        ws = self._ws.get(key)
        if ws is None or ws.numel() < nbytes:
            ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.comm_device)
            self._ws[key] = ws
        return ws

    def route(self, prob, hidden, router_logits):
        ws = self._workspace("layer", lib().moe_workspace_size(ctypes.byref(prob)))
        stage_route(prob, router_logits, ws)
        parts = read_workspace(prob, ws)
        return parts["topk_ids"], parts["topk_w"]

    def dispatch(self, prob, world: int, rank: int, hidden, ids, weights) -> EpDispatch:
        L = lib()
        max_rows = L.moe_ep_max_send_rows(ctypes.byref(prob), world)
        if max_rows < 0:
            raise ValueError("invalid problem or world for expert parallelism")
        dev = hidden.device
        rows = torch.empty((max_rows, prob.hidden), dtype=torch.bfloat16, device=dev)
        expert = torch.empty(max_rows, dtype=torch.int32, device=dev)
        weight = torch.empty(max_rows, dtype=torch.float32, device=dev)
        offsets = torch.empty(world + 1, dtype=torch.int32, device=dev)
        p2r = torch.empty(max(prob.num_tokens * (prob.topk + prob.num_shared), 1), dtype=torch.int32, device=dev)
        ws = self._workspace("dispatch", L.moe_ep_workspace_size(ctypes.byref(prob), world))
        check(L.moe_ep_dispatch(ctypes.byref(prob), world, rank, _ptr(hidden), _ptr(ids), _ptr(weights), _ptr(rows),
                                _ptr(expert), _ptr(weight), _ptr(offsets), _ptr(p2r), _ptr(ws), ws.numel(),
                                _stream()), "moe_ep_dispatch")
        off = offsets.tolist()  # the exchange needs the segment sizes on the host
        return EpDispatch(rows, expert, weight, [off[r + 1] - off[r] for r in range(world)], p2r)

    def local_forward(self, rows, expert, weight, w13_local, w2_local, num_local: int, activation):
        return moe_forward_routed(rows, expert.view(-1, 1), weight.view(-1, 1), w13_local, w2_local, num_local,
                                  activation)

    def combine(self, prob, world: int, returned, pair_to_send_row):
        out = torch.empty((prob.num_tokens, prob.hidden), dtype=torch.bfloat16, device=returned.device)
        check(lib().moe_ep_combine(ctypes.byref(prob), world, _ptr(returned), _ptr(pair_to_send_row), _ptr(out),
                                   _stream()), "moe_ep_combine")
        return out


def _exchange(x: torch.Tensor, recv_counts: List[int], send_counts: List[int], group) -> torch.Tensor:
    """all_to_all_single of the first sum(send_counts) rows of x; 2-D rows travel as bytes."""
    import torch.distributed as dist
    n = sum(send_counts)
    src = x[:n].contiguous()
    if src.dim() == 2:
        width = src.shape[1] * src.element_size()
        out = torch.empty((sum(recv_counts), width), dtype=torch.uint8, device=src.device)
        dist.all_to_all_single(out, src.view(torch.uint8).view(n, width), recv_counts, send_counts, group=group)
        return out.view(src.dtype).view(sum(recv_counts), src.shape[1])
    out = torch.empty(sum(recv_counts), dtype=src.dtype, device=src.device)
    dist.all_to_all_single(out, src, recv_counts, send_counts, group=group)
    return out


def ep_moe_forward(hidden: torch.Tensor, router_logits: torch.Tensor, w13_local, w2_local, topk: int,
                   renormalize: bool, activation_type, *, num_shared: int = 0, group=None,
                   backend: Optional[GpuBackend] = None) -> torch.Tensor:
    """The layer forward for this rank's tokens with the experts split over the group.

    ``hidden`` bf16 [T, H] and ``router_logits`` fp32 [T, E_r] are this rank's tokens;
    ``w13_local`` / ``w2_local`` hold this rank's experts (``local_expert_weights``), prepared
    for a problem of E_r / world + num_shared routed experts. Every rank of the group calls
    this once per step (T may differ between ranks). Returns bf16 [T, H].
    """
    import torch.distributed as dist
    be = backend if backend is not None else GpuBackend()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    T, H = hidden.shape
    E_r = router_logits.shape[1]
    I = getattr(w2_local, "moe_intermediate", None) or w2_local.shape[-1]
    prob = make_problem(T, H, E_r, topk, I, renormalize=renormalize, activation=activation_type,
                        num_shared=num_shared)
    ids, weights = be.route(prob, hidden, router_logits)
    d = be.dispatch(prob, world, rank, hidden, ids, weights)
    # segment sizes first (every rank learns what it will receive), then the segments
    sc = torch.tensor(d.send_counts, dtype=torch.int64, device=be.comm_device)
    rc = torch.empty_like(sc)
    dist.all_to_all_single(rc, sc, group=group)
    recv_counts = [int(v) for v in rc.tolist()]
    rows = _exchange(d.send_rows, recv_counts, d.send_counts, group)
    expert = _exchange(d.send_expert, recv_counts, d.send_counts, group)
    weight = _exchange(d.send_weight, recv_counts, d.send_counts, group)
    y = be.local_forward(rows, expert, weight, w13_local, w2_local, E_r // world + num_shared, activation_type)
    back = _exchange(y, d.send_counts, recv_counts, group)
    return be.combine(prob, world, back, d.pair_to_send_row)


def prepare_local_weights(w13_local: torch.Tensor, w2_local: torch.Tensor, num_local: int, topk_local: int,
                          intermediate_in: int, activation_type):
    """Prepare this rank's experts for the routed forward (bf16; tiled layout)."""
    T, H = 1, w13_local.shape[-1]
    from . import padded_intermediate
    I = padded_intermediate(intermediate_in, activation_type)
    prob = make_problem(T, H, num_local, topk_local, I, renormalize=False, activation=activation_type)
    return prepare_weights(prob, w13_local, w2_local, intermediate_in)
