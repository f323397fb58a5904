"""The workspace-free align entry point (moe_align_noalloc), checked against the
workspace-based one (moe_stage_align) through the C ABI.

moe_align_noalloc exists for callers that cannot allocate device memory (a plugin handed
only its input and output tensors, code under stream capture, paths where an allocation
could synchronise the device); it keeps its scratch in a fixed device array owned by the
library. Its outputs are integers, so they must match the workspace version bit for bit,
on two calls in a row with different routings (the shared scratch keeps the previous
call's contents, which must not leak into the next result).

This file is collected last so that a run stopping at the first failure has already run
every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import mixture_experts_expert_topk_b200 as moe
from mixture_experts_expert_topk_b200.synth import MoeConfig, make_inputs

pytestmark = pytest.mark.gpu


def _i32(n):
    return torch.full((max(n, 1),), -7, dtype=torch.int32, device="cuda")


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("T,E,topk,shared", [(1024, 64, 8, 0), (2048, 40, 6, 1)])
def test_align_noalloc_matches_workspace_align_twice(T, E, topk, shared):
    L = moe.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, seed in enumerate((11, 12)):          # two calls in a row, different routings
        cfg = MoeConfig("noalloc", T=T, H=256, E=E, topk=topk, I=256, renormalize=True,
                        activation="swiglu", num_shared=shared, logit_bias_std=1.0)
        inp = make_inputs(cfg, seed, weights=False)
        prob = moe.make_problem(T, 256, E, topk, 256, num_shared=shared)
        lay = moe.workspace_layout(prob)
        assert lay["num_chunks"] > 1            # the case that uses the scratch array
        ws = moe.new_workspace(prob)
        moe.stage_route(prob, inp["logits"].cuda(), ws)
        moe.stage_align(prob, ws)               # the existing, workspace-based entry point
        ref = moe.read_workspace(prob, ws)
        P = T * (topk + shared)
        rows = lay["max_rows"]
        Et = E + shared
        out = {"sorted_pair_ids": _i32(rows), "expert_offsets": _i32(Et + 1),
               "block_expert": _i32(rows // lay["block_m"]), "pair_to_row": _i32(P), "num_blocks": _i32(1)}
        ids = ref["topk_ids"].contiguous()
        st = L.moe_align_noalloc(ctypes.byref(prob), _ptr(ids), _ptr(out["sorted_pair_ids"]),
                                 _ptr(out["expert_offsets"]), _ptr(out["block_expert"]),
                                 _ptr(out["pair_to_row"]), _ptr(out["num_blocks"]), stream)
        assert st == 0, (call, moe._capi.status_string(st))
        torch.cuda.synchronize()
        nb = int(ref["num_blocks"][0])
        assert int(out["num_blocks"][0]) == nb
        p_pad = nb * lay["block_m"]
        assert torch.equal(out["expert_offsets"], ref["expert_offsets"])
        assert torch.equal(out["sorted_pair_ids"][:p_pad], ref["sorted_pair_ids"][:p_pad])
        assert torch.equal(out["block_expert"][:nb], ref["block_expert"][:nb])
        assert torch.equal(out["pair_to_row"], ref["pair_to_row"])


def test_align_noalloc_rejects_oversized_problem():
    L = moe.lib()
    # 300 chunks of 1024 experts exceed the fixed 262144-int scratch
    prob = moe.make_problem(300 * 2048 // 16, 256, 1024, 16, 256)
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    p = _ptr(dummy)
    st = L.moe_align_noalloc(ctypes.byref(prob), p, p, p, p, p, p,
                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == moe._capi.MOE_ERR_UNSUPPORTED
