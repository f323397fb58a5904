"""Expert parallelism: the orchestration of mixture_experts_expert_topk_b200.ep on CPU with
gloo ranks (a CPU stand-in computes each step, see _ep_backend.py), and the host-side checks
of the expert-parallel entry points. The kernels themselves run in test_gpu_parity.py."""
import ctypes
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import mixture_experts_expert_topk_b200 as moe
from mixture_experts_expert_topk_b200 import ep
from mixture_experts_expert_topk_b200.synth import MoeConfig, make_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cfg(**kw) -> MoeConfig:
    base = dict(name="ep", T=40, H=128, E=8, topk=3, I=32, renormalize=True, activation="swiglu")
    base.update(kw)
    return MoeConfig(**base)


def _worker(rank, world, port, cfg, splits, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch.distributed as dist
    from _ep_backend import CpuBackend, _bits
    dist.init_process_group("gloo", rank=rank, world_size=world)
    inp = make_inputs(cfg, 0)
    lo, hi = splits[rank], splits[rank + 1]
    w13_l, w2_l = ep.local_expert_weights(inp["w13"], inp["w2"], cfg.E, cfg.num_shared, world, rank)
    be = CpuBackend(_bits(w13_l), _bits(w2_l))
    out = ep.ep_moe_forward(inp["hidden"][lo:hi], inp["logits"][lo:hi], w13_l, w2_l, cfg.topk, cfg.renormalize,
                            cfg.activation, num_shared=cfg.num_shared, backend=be)
    q.put((rank, out.to(torch.float32).numpy()))
    dist.barrier()
    dist.destroy_process_group()


def _run(cfg, world, splits):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, cfg, splits, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=240) for _ in range(world))
    for p in procs:
        p.join(60)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    return np.concatenate([res[r] for r in range(world)])


@pytest.mark.parametrize("shared,world,splits", [(0, 2, [0, 23, 40]), (1, 2, [0, 40, 40]), (0, 4, [0, 5, 17, 30, 40])])
def test_ep_gloo_ranks_match_the_layer(shared, world, splits):
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from _cases import err_beyond_rounding
    from oracle import moe_oracle as O
    cfg = _cfg(num_shared=shared)
    got = _run(cfg, world, splits)
    inp = make_inputs(cfg, 0)
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    ref = O.moe_forward(bits(inp["hidden"]), inp["logits"].numpy(), bits(inp["w13"]), bits(inp["w2"]),
                        topk=cfg.topk, renormalize=cfg.renormalize, activation=cfg.activation, num_shared=shared)
    # the owners return bf16 rows (one rounding per pair) before the fp32 combine
    assert err_beyond_rounding(got.astype(np.float64), ref) <= 2e-2


def test_owned_experts_and_local_weights():
    assert list(ep.owned_experts(8, 4, 2)) == [4, 5]
    with pytest.raises(ValueError):
        ep.owned_experts(10, 4, 0)
    w13 = torch.arange(9 * 2 * 3, dtype=torch.float32).view(9, 2, 3)
    w2 = -w13.clone()
    a, b = ep.local_expert_weights(w13, w2, 8, 1, 2, 1)
    assert torch.equal(a, w13[[4, 5, 6, 7, 8]]) and torch.equal(b, w2[[4, 5, 6, 7, 8]])


def test_ep_entry_points_host_checks():
    L = moe.lib()
    p = moe.make_problem(40, 128, 8, 3, 32)
    P = 40 * 3
    assert L.moe_ep_max_send_rows(ctypes.byref(p), 2) == -(-(P + 2 * 15) // 16) * 16
    assert L.moe_ep_workspace_size(ctypes.byref(p), 2) > 0
    assert L.moe_ep_max_send_rows(ctypes.byref(p), 3) == -1          # 8 experts do not split over 3 ranks
    assert L.moe_ep_workspace_size(ctypes.byref(p), 0) == 0
    fake = ctypes.c_void_p(1 << 20)
    s = ctypes.c_void_p(0)
    n = L.moe_ep_workspace_size(ctypes.byref(p), 2)
    args = [fake] * 8
    assert L.moe_ep_dispatch(ctypes.byref(p), 2, 2, *args, fake, n, s) == 1      # rank out of range
    assert L.moe_ep_dispatch(ctypes.byref(p), 2, 0, *args, ctypes.c_void_p((1 << 20) + 16), n, s) == 1
    assert L.moe_ep_dispatch(ctypes.byref(p), 2, 0, *args, fake, n - 1, s) == 3  # workspace too small
    assert L.moe_ep_combine(ctypes.byref(p), 2, None, fake, fake, s) == 1
