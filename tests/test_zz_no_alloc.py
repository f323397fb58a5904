"""The workspace-free align entry point (moe_align_noalloc), checked through the C ABI
against the CPU oracle's align and against the workspace-based entry point
(moe_stage_align).

moe_align_noalloc exists for callers that cannot allocate device memory (a plugin handed
only its input and output tensors, code under stream capture, paths where an allocation
could synchronise the device); it keeps its scratch in a fixed device array owned by the
library. Its outputs are integers, so they must match bit for bit, on two calls in a row
with different routings (the shared scratch keeps the previous call's contents, which
must not leak into the next result). Every output buffer is sized exactly as the header
states and followed by a guard region that must come back untouched.

This file is collected last so that a run stopping at the first failure has already run
every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import mixture_experts_expert_topk_b200 as moe
from mixture_experts_expert_topk_b200.synth import MoeConfig, make_inputs
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu

GUARD = 64          # int32 guard words after every output buffer
FILL = -7


def _buffers(lay, P, E):
    """One device allocation per output: the header's size, then GUARD words of FILL."""
    sizes = {"sorted_pair_ids": lay["max_rows"], "expert_offsets": E + 1,
             "block_expert": lay["max_rows"] // lay["block_m"], "pair_to_row": P, "num_blocks": 1}
    return sizes, {k: torch.full((n + GUARD,), FILL, dtype=torch.int32, device="cuda") for k, n in sizes.items()}


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _call(L, prob, ids, out):
    return L.moe_align_noalloc(ctypes.byref(prob), _ptr(ids), _ptr(out["sorted_pair_ids"]),
                               _ptr(out["expert_offsets"]), _ptr(out["block_expert"]), _ptr(out["pair_to_row"]),
                               _ptr(out["num_blocks"]), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _check_guards(sizes, out):
    for k, n in sizes.items():
        tail = out[k][n:].cpu().numpy()
        assert np.all(tail == FILL), f"{k}: write past the documented size"


@pytest.mark.parametrize("T,E,topk,shared,block_m", [(1024, 64, 8, 0, 0), (2048, 40, 6, 1, 0),
                                                     (1500, 24, 4, 0, 128)])
def test_align_noalloc_matches_oracle_and_workspace_align_twice(T, E, topk, shared, block_m):
    L = moe.lib()
    for call, seed in enumerate((11, 12)):          # two calls in a row, different routings
        cfg = MoeConfig("noalloc", T=T, H=256, E=E, topk=topk, I=256, renormalize=True,
                        activation="swiglu", num_shared=shared, logit_bias_std=1.0)
        inp = make_inputs(cfg, seed, weights=False)
        prob = moe.make_problem(T, 256, E, topk, 256, num_shared=shared, block_m=block_m)
        lay = moe.workspace_layout(prob)
        assert lay["num_chunks"] > 1            # the case that uses the scratch array
        ws = moe.new_workspace(prob)
        moe.stage_route(prob, inp["logits"].cuda(), ws)
        moe.stage_align(prob, ws)               # the existing, workspace-based entry point
        ref = moe.read_workspace(prob, ws)
        P = T * (topk + shared)
        Et = E + shared
        sizes, out = _buffers(lay, P, Et)
        ids = ref["topk_ids"].contiguous()
        st = _call(L, prob, ids, out)
        assert st == 0, (call, moe._capi.status_string(st))
        torch.cuda.synchronize()
        _check_guards(sizes, out)
        bm = lay["block_m"]
        nb = int(out["num_blocks"][0])
        p_pad = nb * bm
        # the oracle's align of the same ids, bit for bit
        a = O.align(ids.cpu().numpy(), Et, bm)
        assert p_pad == int(a["P_pad"])
        np.testing.assert_array_equal(out["expert_offsets"][:Et + 1].cpu().numpy(), a["expert_offsets"])
        np.testing.assert_array_equal(out["sorted_pair_ids"][:p_pad].cpu().numpy(), a["sorted_pair_ids"])
        np.testing.assert_array_equal(out["block_expert"][:nb].cpu().numpy(), a["block_expert"])
        np.testing.assert_array_equal(out["pair_to_row"][:P].cpu().numpy(), a["pair_to_row"])
        # and the workspace entry point's outputs
        assert int(ref["num_blocks"][0]) == nb
        assert torch.equal(out["expert_offsets"][:Et + 1], ref["expert_offsets"])
        assert torch.equal(out["sorted_pair_ids"][:p_pad], ref["sorted_pair_ids"][:p_pad])
        assert torch.equal(out["block_expert"][:nb], ref["block_expert"][:nb])
        assert torch.equal(out["pair_to_row"][:P], ref["pair_to_row"])


def test_align_noalloc_skips_out_of_range_ids():
    # ids outside [0, E) are skipped by the kernels' own range check: those pairs get
    # pair_to_row -1 and the others are aligned as if the bad pairs were absent
    L = moe.lib()
    T, E, topk = 1200, 16, 4
    prob = moe.make_problem(T, 256, E, topk, 256)
    lay = moe.workspace_layout(prob)
    assert lay["num_chunks"] > 1
    g = torch.Generator().manual_seed(5)
    ids = torch.randint(0, E, (T, topk), generator=g, dtype=torch.int32)
    bad = [(0, 0), (7, 3), (1199, 1), (600, 2)]
    for (t, j), v in zip(bad, (-1, E, 1 << 30, -(1 << 30))):
        ids[t, j] = v
    P = T * topk
    sizes, out = _buffers(lay, P, E)
    st = _call(L, prob, ids.cuda(), out)
    assert st == 0
    torch.cuda.synchronize()
    _check_guards(sizes, out)
    flat = ids.numpy().reshape(-1)
    keep = (flat >= 0) & (flat < E)
    p2r = out["pair_to_row"][:P].cpu().numpy()
    assert np.all(p2r[~keep] == -1)
    # the valid pairs: the oracle's align over them alone (same stable order, same padding)
    cnt = np.bincount(flat[keep], minlength=E)
    off = np.concatenate([[0], np.cumsum(-(-cnt // lay["block_m"]) * lay["block_m"])])
    np.testing.assert_array_equal(out["expert_offsets"][:E + 1].cpu().numpy(), off)
    spi = out["sorted_pair_ids"][:int(off[-1])].cpu().numpy()
    for e in range(E):
        seg = spi[off[e]:off[e + 1]]
        pairs = np.nonzero(keep & (flat == e))[0]
        np.testing.assert_array_equal(seg[:len(pairs)], pairs)
        assert np.all(seg[len(pairs):] == P)
        np.testing.assert_array_equal(p2r[pairs], off[e] + np.arange(len(pairs)))


def test_align_noalloc_rejects_oversized_problem():
    L = moe.lib()
    # 300 chunks of 1024 experts exceed the fixed 262144-int scratch
    prob = moe.make_problem(300 * 2048 // 16, 256, 1024, 16, 256)
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    p = _ptr(dummy)
    st = L.moe_align_noalloc(ctypes.byref(prob), p, p, p, p, p, p,
                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == moe._capi.MOE_ERR_UNSUPPORTED
