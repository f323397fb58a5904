"""Expert-parallel kernels on the GPU: dispatch and combine against restatements of their
contract (bit for bit), and the whole expert-parallel forward on a one-rank NCCL group
against the oracle. Several ranks need several GPUs; their exchange logic runs on CPU in
test_ep.py."""
import os
import socket

import numpy as np
import pytest
import torch

import mixture_experts_expert_topk_b200 as moe
from mixture_experts_expert_topk_b200 import ep
from mixture_experts_expert_topk_b200.synth import MoeConfig, make_inputs
from oracle import moe_oracle as O

from _cases import bits, err_beyond_rounding, report

pytestmark = pytest.mark.gpu


def _cfg(**kw) -> MoeConfig:
    base = dict(name="ep", T=300, H=256, E=16, topk=4, I=128, renormalize=True, activation="swiglu")
    base.update(kw)
    return MoeConfig(**base)


@pytest.mark.parametrize("world,rank,shared", [(4, 1, 1), (2, 0, 0), (1, 0, 0)])
def test_ep_dispatch_and_combine_kernels(world, rank, shared):
    cfg = _cfg(num_shared=shared)
    inp = make_inputs(cfg, 0, weights=False)
    dev = torch.device("cuda:0")
    hidden, logits = inp["hidden"].to(dev), inp["logits"].to(dev)
    prob = moe.make_problem(cfg.T, cfg.H, cfg.E, cfg.topk, cfg.I, renormalize=cfg.renormalize, num_shared=shared)
    be = ep.GpuBackend()
    ids, w = be.route(prob, hidden, logits)
    d = be.dispatch(prob, world, rank, hidden, ids, w)
    torch.cuda.synchronize()
    # restatement: owner = id / (E_r / world) for routed ids, this rank for the shared slot;
    # stable sort by owner, each owner's segment padded to 16 rows
    idn = ids.cpu().numpy().reshape(-1)
    wn = w.cpu().numpy().reshape(-1)
    k = cfg.topk + shared
    per = cfg.E // world
    owner = np.where(idn < cfg.E, idn // per, rank)
    order = np.argsort(owner, kind="stable")
    counts = np.bincount(owner, minlength=world)
    assert d.send_counts == [int(-(-c // 16) * 16) for c in counts]
    starts = np.concatenate([[0], np.cumsum(d.send_counts)])
    rows = d.send_rows.cpu().view(torch.int16).numpy()
    hid = hidden.cpu().view(torch.int16).numpy()
    exp_ = d.send_expert.cpu().numpy()
    wt = d.send_weight.cpu().numpy()
    p2r = d.pair_to_send_row.cpu().numpy()
    src = 0
    for r in range(world):
        seg = order[src:src + counts[r]]
        at = np.arange(starts[r], starts[r] + counts[r])
        np.testing.assert_array_equal(p2r[seg], at)
        np.testing.assert_array_equal(rows[at], hid[seg // k])
        np.testing.assert_array_equal(exp_[at], np.where(idn[seg] < cfg.E, idn[seg] % per, per))
        np.testing.assert_array_equal(wt[at], wn[seg])
        pad = np.arange(starts[r] + counts[r], starts[r + 1])
        assert np.all(rows[pad] == 0) and np.all(exp_[pad] == 0) and np.all(wt[pad] == 0)
        src += counts[r]
    # combine: slot-order fp32 sum of the returned bf16 rows, one rounding, bit for bit
    S = int(starts[-1])
    ret = torch.randn(S, cfg.H, device=dev).to(torch.bfloat16)
    out = be.combine(prob, world, ret, d.pair_to_send_row)
    r32 = ret.float().cpu().numpy()
    acc = np.zeros((cfg.T, cfg.H), np.float32)
    for j in range(k):
        acc += r32[p2r.reshape(cfg.T, k)[:, j]]
    np.testing.assert_array_equal(bits(out.cpu()), bits(torch.from_numpy(acc).to(torch.bfloat16)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("shared,act", [(0, "swiglu"), (1, "relu2")])
def test_ep_forward_one_rank_matches_oracle(shared, act):
    import torch.distributed as dist
    cfg = _cfg(num_shared=shared, activation=act, renormalize=act != "relu2", I=256 if act == "relu2" else 128)
    inp = make_inputs(cfg, 0)
    dev = torch.device("cuda:0")
    import datetime
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            device_id=dev, timeout=datetime.timedelta(seconds=60))
    try:
        w13_l, w2_l = ep.local_expert_weights(inp["w13"].to(dev), inp["w2"].to(dev), cfg.E, shared, 1, 0)
        w13p, w2p = ep.prepare_local_weights(w13_l, w2_l, cfg.E + shared, 1, cfg.I, act)
        out = ep.ep_moe_forward(inp["hidden"].to(dev), inp["logits"].to(dev), w13p, w2p, cfg.topk, cfg.renormalize,
                                act, num_shared=shared)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ref = O.moe_forward(bits(inp["hidden"]), inp["logits"].numpy(), bits(inp["w13"]), bits(inp["w2"]), topk=cfg.topk,
                        renormalize=cfg.renormalize, activation=act, num_shared=shared)
    e = err_beyond_rounding(out.cpu().float().numpy().astype(np.float64), ref)
    report(f"ep one rank {act} shared={shared}: beyond-rounding {e:.4f}")
    assert e <= 2e-2, e
