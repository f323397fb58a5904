"""A CPU stand-in for the expert-parallel backend, for running the orchestration of
``mixture_experts_expert_topk_b200.ep`` under gloo without a GPU. Routing and each owner's
experts come from the oracle; dispatch and combine restate the kernels' contract (stable
sort by owner rank with 16-row padding per owner; slot-order fp32 sum rounded once to bf16);
the owners' outputs are rounded to bf16 as the routed forward returns them."""
import numpy as np
import torch

from oracle import moe_oracle as O


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.asarray(a, np.float64).astype(np.float32)).to(torch.bfloat16)


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


class CpuBackend:
    comm_device = torch.device("cpu")

    def __init__(self, w13_local_bits, w2_local_bits):
        self.w13 = w13_local_bits   # checkpoint layout, this rank's experts (routed range, then shared)
        self.w2 = w2_local_bits

    def route(self, prob, hidden, router_logits):
        ids, w = O.route(router_logits.numpy(), prob.topk, bool(prob.renormalize), prob.num_shared)
        return torch.from_numpy(ids.astype(np.int32)), torch.from_numpy(w.astype(np.float32))

    def dispatch(self, prob, world, rank, hidden, ids, weights):
        from mixture_experts_expert_topk_b200.ep import EpDispatch
        E_r, k = prob.num_routed, prob.topk + prob.num_shared
        per = E_r // world
        idn = ids.numpy().reshape(-1)
        owner = np.where(idn < E_r, idn // per, rank)
        order = np.argsort(owner, kind="stable")
        counts = [int(np.sum(owner == r)) for r in range(world)]
        padded = [-(-c // 16) * 16 for c in counts]
        H = prob.hidden
        rows = torch.zeros((sum(padded), H), dtype=torch.bfloat16)
        expert = torch.zeros(sum(padded), dtype=torch.int32)
        weight = torch.zeros(sum(padded), dtype=torch.float32)
        p2r = torch.zeros(idn.size, dtype=torch.int32)
        at, src = 0, 0
        for r in range(world):
            for p in order[src:src + counts[r]]:
                e = int(idn[p])
                rows[at] = hidden[p // k]
                expert[at] = e % per if e < E_r else per
                weight[at] = float(weights.numpy().reshape(-1)[p])
                p2r[p] = at
                at += 1
            at += padded[r] - counts[r]
            src += counts[r]
        return EpDispatch(rows, expert, weight, padded, p2r)

    def local_forward(self, rows, expert, weight, w13_local, w2_local, num_local, activation):
        if rows.shape[0] == 0:
            return torch.zeros((0, rows.shape[1]), dtype=torch.bfloat16)
        out = O.moe_forward(_bits(rows), None, self.w13, self.w2, topk=1, renormalize=False, activation=activation,
                            routing=(expert.numpy()[:, None], weight.numpy()[:, None]))
        return _bf16(out)

    def combine(self, prob, world, returned, pair_to_send_row):
        T, k = prob.num_tokens, prob.topk + prob.num_shared
        r = returned.to(torch.float32).numpy()
        acc = np.zeros((T, prob.hidden), np.float32)
        for j in range(k):
            acc += r[pair_to_send_row.numpy().reshape(T, k)[:, j]]
        return torch.from_numpy(acc).to(torch.bfloat16)
