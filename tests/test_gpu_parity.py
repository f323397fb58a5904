"""Parity of the CUDA path (through the C ABI) against the CPU oracle.

Integer outputs (routing ids, permutation, expert_offsets, block map) must match
bit for bit. Floating-point outputs: routing weights within 1e-5 relative (fp32
exponentials against float64); the layer output within 2e-2 * RMS(ref) beyond the
rounding of the exact result to bf16 (``err_beyond_rounding``: the output format is
bf16, and on the prefill workload rounding the exact float64 result to bf16 alone
gives max|err| = 2.2e-2 * RMS); the GEMM1 activation elementwise within 2^-8 relative
(its bf16 store) plus 1e-3 * RMS (fp32 accumulation).
"""
import dataclasses

import numpy as np
import pytest
import torch

import mixture_experts_expert_topk_b200 as moe
from mixture_experts_expert_topk_b200.synth import CONFIGS, MoeConfig, make_inputs
from oracle import moe_oracle as O

from _cases import (act_rows_f64, bf16_act_bound, bf16_to_f64, bits, check_act_pairs, cover_tokens,
                    cpu_inputs, dirty_workspace, err_beyond_rounding, GpuForward, max_err_over_rms,
                    oracle_fp8_block_weights, oracle_mxfp8_weights, oracle_out, report, untile_b128,
                    untile_groups, untile_u8, untile_weights)

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2
FP8_TOL = 5e-2


def _small(name, **kw) -> MoeConfig:
    base = dict(T=64, H=256, E=8, topk=2, I=512, renormalize=True, activation="swiglu")
    base.update(kw)
    return MoeConfig(name, **base)


SMALL = {
    "tiny": CONFIGS["tiny"],
    # several row tiles per expert, ragged tails, BN=160 for N1=640, GEMM2 K=320
    "ragged": _small("ragged", T=300, H=512, E=16, topk=4, I=320),
    "relu2_small": _small("relu2_small", T=200, H=384, E=8, topk=3, I=384, activation="relu2",
                          renormalize=False),
    # unaligned intermediate: padded 200 -> 208 (gated), K tail in GEMM2
    "pad_gated": _small("pad_gated", T=96, H=256, E=6, topk=2, I=200),
    "pad_relu2": _small("pad_relu2", T=96, H=256, E=6, topk=2, I=300, activation="relu2",
                        renormalize=False),
    "shared_bf16": _small("shared_bf16", T=130, H=256, E=12, topk=3, I=256, num_shared=1),
    "k_equals_E": _small("k_equals_E", T=40, H=256, E=8, topk=8, I=128),
    "skewed": _small("skewed", T=512, H=256, E=32, topk=4, I=256, logit_bias_std=3.0),
    # more than 1024 pairs (row groups of up to 256, permuted rows by TMA) with a partial
    # last weight tile (N1 = 416) and a K tail in GEMM2 (K = 208)
    "pad_gated_big": _small("pad_gated_big", T=600, H=256, E=6, topk=2, I=200),
    "relu2_big": _small("relu2_big", T=600, H=384, E=8, topk=3, I=300, activation="relu2",
                        renormalize=False),
    # three align chunks (the single-launch align with its grid barrier) and more experts
    # than the align CTA has threads
    "many_experts": _small("many_experts", T=700, H=256, E=300, topk=8, I=128),
    # the gelu_tanh gated activation, both GEMM paths (with an unaligned intermediate)
    "gelu_small": _small("gelu_small", T=300, H=256, E=8, topk=2, I=200, activation="gelu_tanh"),
    "gelu_big": _small("gelu_big", T=600, H=256, E=6, topk=2, I=256, activation="gelu_tanh"),
    # swigluoai; weights large enough (z ~ N(0, 8^2)) that both of its clamps are active
    "oai_small": _small("oai_small", T=300, H=256, E=8, topk=2, I=200, activation="swigluoai", weight_std=0.5),
    "oai_big": _small("oai_big", T=600, H=256, E=6, topk=2, I=256, activation="swigluoai", weight_std=0.5,
                      num_shared=1),
}


def _check_route_align(cfg, parts, logits, bm=None):
    ids, w = O.route(logits.numpy(), cfg.topk, cfg.renormalize, cfg.num_shared)
    np.testing.assert_array_equal(parts["topk_ids"], ids)
    np.testing.assert_allclose(parts["topk_w"], w, rtol=1e-5, atol=1e-7)
    bm = bm or parts["block_m"]
    a = O.align(ids, cfg.E_total, bm)
    P_pad = int(a["P_pad"])
    assert int(parts["num_blocks"][0]) == P_pad // bm
    np.testing.assert_array_equal(parts["expert_offsets"], a["expert_offsets"])
    np.testing.assert_array_equal(parts["sorted_pair_ids"][:P_pad], a["sorted_pair_ids"])
    np.testing.assert_array_equal(parts["block_expert"][:P_pad // bm], a["block_expert"])
    np.testing.assert_array_equal(parts["pair_to_row"], a["pair_to_row"])
    if bm == 16:
        _check_groups(cfg, parts, a)
    return ids, a


def _check_groups(cfg, parts, a):
    """Row groups of the swapped-operand GEMMs: each expert's padded segment cut into
    ceil(rows / G) groups of whole 16-row blocks, sizes as even as possible, larger first
    (G = 256; 128 for FP8 block-128), the word expert | rows << 16 | padding << 25 (the
    segment's padding rows, all in its last group); and, for bf16, the permuted hidden rows."""
    P = cfg.T * cfg.k_total
    G = 128 if cfg.block128 else 256
    off = a["expert_offsets"]
    expect = []
    for e in range(cfg.E_total):
        seg = int(off[e + 1] - off[e])
        if seg == 0:
            continue
        count = int(np.sum(a["sorted_pair_ids"][int(off[e]):int(off[e + 1])] < P))
        assert 0 <= seg - count < 16
        ng = -(-seg // G)
        base, extra = divmod(seg // 16, ng)
        row = int(off[e])
        for i in range(ng):
            n = 16 * (base + (1 if i < extra else 0))
            assert 16 <= n <= G
            expect.append((row, e | (n << 16) | ((seg - count if i == ng - 1 else 0) << 25)))
            row += n
        assert row == off[e + 1]
    assert int(parts["num_blocks"][1]) == len(expect)
    np.testing.assert_array_equal(parts["group_info"][:len(expect)], np.array(expect, dtype=np.int32).reshape(-1, 2))
    if cfg.fp8:
        return
    # the permuted hidden rows, in row-group order
    rows = int(a["P_pad"])
    xs = untile_groups(parts["xs"], parts["group_info"], len(expect), rows, cfg.H // 64)
    pids = a["sorted_pair_ids"][:rows]
    hb = parts["hidden_bits"]
    real = pids < P
    np.testing.assert_array_equal(xs[real], hb[pids[real] // cfg.k_total])  # padding rows: unwritten


def _check_act(cfg, run, parts, ids, a):
    """GEMM1 + activation per sorted row against the oracle's expert FFN first half."""
    x = bf16_to_f64(run.inp["hidden"])
    w13 = run.inp["w13"]
    kk = cfg.k_total
    P = cfg.T * kk
    if parts["block_m"] == 16:   # row-group order: back to sorted rows
        rows = parts["sorted_pair_ids"].shape[0]
        act_bits = untile_groups(parts["act"], parts["group_info"], int(parts["num_blocks"][1]), rows,
                                 -(-run.I_pad // 64))[:, :run.I_pad]
    else:
        act_bits = parts["act"]
    act_gpu = bf16_to_f64(act_bits)
    if parts["block_m"] == 16:   # a group's padding rows: zero activation whatever X held
        P_pad = int(a["expert_offsets"][-1])
        pad = a["sorted_pair_ids"][:P_pad] >= P
        assert np.all(act_bits[:P_pad][pad] == 0)
    worst = 0.0
    for e in np.unique(ids):
        rows = np.arange(a["expert_offsets"][e], a["expert_offsets"][e + 1])
        pids = a["sorted_pair_ids"][rows]
        keep = pids < P
        rows, pids = rows[keep], pids[keep]
        W = bf16_to_f64(w13[e])
        ref = O.activation_fn(x[pids // kk] @ W.T, cfg.activation, cfg.I)
        got = act_gpu[rows, :cfg.I]
        err = np.abs(got - ref)
        bound = 2.0 ** -8 * np.abs(ref) + 1e-3 * O.rms(ref) + 1e-30
        worst = max(worst, float(np.max(err / bound)))
        if run.I_pad > cfg.I:   # padded columns are exact zeros
            assert np.all(act_gpu[rows, cfg.I:] == 0)
    assert worst <= 1.0, worst


@pytest.mark.parametrize("name,bm", [(n, 0) for n in SMALL] +
                         [(n, 128) for n in ("ragged", "skewed", "pad_gated", "relu2_small", "gelu_small",
                                             "oai_small")])
def test_layer_parity_small(name, bm):
    # bm 0: the default (bf16: 16-row alignment, weights on the MMA's M); 128: token tiles
    cfg = SMALL[name]
    run = GpuForward(cfg, block_m=bm)
    out = run.forward()
    parts = run.parts()
    ids, a = _check_route_align(cfg, parts, run.inp["logits"])
    _check_act(cfg, run, parts, ids, a)
    ref = oracle_out(cfg, run.inp)
    got = bf16_to_f64(out)
    assert np.all(np.isfinite(got))
    e = err_beyond_rounding(got, ref)
    report(f"{name}: beyond-rounding {e:.4f}, raw max|err|/RMS {max_err_over_rms(got, ref):.4f}")
    assert e <= BF16_TOL, e
    st, word = moe.device_status(run.ws)
    assert st == 0 and word == 0


def test_forward_is_bitwise_deterministic_and_pdl_invariant():
    cfg = SMALL["ragged"]
    run = GpuForward(cfg)
    a = bits(run.forward()).copy()
    b = bits(run.forward()).copy()
    np.testing.assert_array_equal(a, b)
    run2 = GpuForward(cfg, pdl=False)
    np.testing.assert_array_equal(bits(run2.forward()), a)


def test_stage_entry_points_match_forward():
    cfg = SMALL["ragged"]
    run = GpuForward(cfg)
    ref = bits(run.forward()).copy()
    ws = moe.new_workspace(run.prob)
    out = torch.empty_like(run.hidden)
    moe.stage_route(run.prob, run.logits, ws)
    moe.stage_align(run.prob, ws)
    moe.stage_permute(run.prob, run.hidden, ws)
    moe.stage_gemm1(run.prob, run.hidden, run.w13p, ws)
    moe.stage_gemm2(run.prob, run.w2p, ws)
    moe.stage_combine(run.prob, out, ws)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bits(out), ref)


def test_tied_logits_pick_lowest_indices():
    cfg = _small("ties", T=33, H=256, E=16, topk=4, I=128)
    inp = make_inputs(cfg, 3)
    inp["logits"][:] = 0.5
    inp["logits"][5, 9] = 0.5   # still tied
    run = GpuForward(cfg, inputs=inp)
    run.forward()
    parts = run.parts()
    assert (parts["topk_ids"] == np.arange(4)).all()
    ids, a = _check_route_align(cfg, parts, inp["logits"])
    ref = oracle_out(cfg, inp)
    assert err_beyond_rounding(bf16_to_f64(run.out), ref) <= BF16_TOL


@pytest.mark.parametrize("T", [700, 1500])   # row groups of 16, and of up to 256 (uneven)
def test_all_tokens_one_expert_and_empty_experts(T):
    cfg = _small("one_expert", T=T, H=256, E=8, topk=1, I=256)
    inp = make_inputs(cfg, 4)
    inp["logits"][:, 5] += 100.0   # every token picks expert 5; 7 experts empty
    run = GpuForward(cfg, inputs=inp)
    run.forward()
    parts = run.parts()
    ids, a = _check_route_align(cfg, parts, inp["logits"])
    bm = parts["block_m"]
    seg = -(-T // bm) * bm                        # T pairs padded to the row tile
    assert list(a["expert_offsets"]) == [0] * 6 + [seg] * 3
    ref = oracle_out(cfg, inp)
    assert err_beyond_rounding(bf16_to_f64(run.out), ref) <= BF16_TOL


def test_zero_tokens_is_a_no_op():
    cfg = _small("empty", T=0)
    prob = moe.make_problem(0, 256, 8, 2, 512)
    ws = moe.new_workspace(prob) if moe.workspace_size(prob) else torch.empty(256, dtype=torch.uint8, device="cuda")
    h = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    l = torch.empty((0, 8), dtype=torch.float32, device="cuda")
    w13 = torch.zeros((8, 1024, 256), dtype=torch.bfloat16, device="cuda")
    w2 = torch.zeros((8, 256, 512), dtype=torch.bfloat16, device="cuda")
    out = moe.moe_forward(h, l, w13, w2, 2, True, "swiglu", workspace=ws)
    assert out.shape == (0, 256)


@pytest.mark.parametrize("bm", [16, 128])
def test_prepare_weights_matches_oracle_layout(bm):
    # bm 128: row-major; bm 16: tiled (128 x 64 tiles, swizzled, zero past the matrix)
    for act, I in (("swiglu", 200), ("swiglu", 512), ("relu2", 300)):
        cfg = _small("prep", T=4, H=256, E=3, topk=1, I=I, activation=act)
        inp = make_inputs(cfg, 1)
        I_pad = moe.padded_intermediate(I, act)
        prob = moe.make_problem(4, 256, 3, 1, I_pad, activation=act, block_m=bm)
        w13p, w2p = moe.prepare_weights(prob, inp["w13"].cuda(), inp["w2"].cuda(), I)
        torch.cuda.synchronize()
        p13, p2, ip = O.pad_weights(bits(inp["w13"]), bits(inp["w2"]), I, act == "swiglu")
        assert ip == I_pad
        if act == "swiglu":
            p13 = O.interleave_gate_up(p13, I_pad)
        g13, g2 = bits(w13p), bits(w2p)
        if bm == 16:
            N1 = p13.shape[1]
            t13 = untile_weights(g13, 3, N1, 256)
            t2 = untile_weights(g2, 3, 256, I_pad)
            assert np.all(t13[:, N1:] == 0) and np.all(t2[:, :, I_pad:] == 0)
            g13, g2 = t13[:, :N1, :256], t2[:, :256, :I_pad]
        np.testing.assert_array_equal(g13, p13)
        np.testing.assert_array_equal(g2, p2)


def test_fp8_quantizers_bit_exact():
    g = torch.Generator().manual_seed(7)
    x = torch.randn((37, 512), generator=g).to(torch.bfloat16)
    x[3, 128:256] = 0
    x[5, :5] = 1000.0
    prob = moe.make_problem(37, 512, 8, 2, 512, fp8=True, block_m=128)   # the token-tile path quantises [T, H]
    ws = moe.new_workspace(prob)
    moe.stage_quant_act(prob, x.cuda(), ws)
    torch.cuda.synchronize()
    v = moe.read_workspace(prob, ws)
    q, s = O.quant_groups_1x128(O.bf16_bits_to_f32(bits(x)))
    np.testing.assert_array_equal(v["xq"].cpu().numpy(), q)
    np.testing.assert_array_equal(v["xq_scale"].cpu().numpy(), s)
    w = (0.02 * torch.randn((3, 256, 384), generator=g)).to(torch.bfloat16)
    w[1, :128, :128] = 0
    codes, scales = moe.quantize_weights_fp8(w.cuda())
    torch.cuda.synchronize()
    for m in range(3):
        qm, sm = O.quant_blocks_128x128(O.bf16_bits_to_f32(bits(w[m])))
        np.testing.assert_array_equal(codes[m].cpu().numpy(), qm)
        np.testing.assert_array_equal(scales[m].cpu().numpy(), sm)


# ---- the workloads at full size ------------------------------------------------------

def _full_size(cfg, n_sample=48, seed=0):
    run = GpuForward(cfg, seed)
    out = run.forward()
    parts = run.parts()
    ids, a = _check_route_align(cfg, parts, run.inp["logits"])
    rng = np.random.default_rng(123)
    tokens = np.sort(rng.choice(cfg.T, size=min(n_sample, cfg.T), replace=False))
    fp8w = None
    if cfg.fp8:
        # the oracle quantises only the experts the sampled tokens use
        fp8w = O.quantize_weights_fp8(bits(run.inp["w13"]), bits(run.inp["w2"]),
                                      experts=np.unique(ids[tokens]))
    ref = oracle_out(cfg, run.inp, tokens=tokens, fp8_weights=fp8w)
    got = bf16_to_f64(out)[tokens]
    assert np.all(np.isfinite(bf16_to_f64(out)))
    report(f"{cfg.name}: beyond-rounding {err_beyond_rounding(got, ref):.4f}, raw {max_err_over_rms(got, ref):.4f}")
    return err_beyond_rounding(got, ref), run


@pytest.mark.parametrize("name,n_sample", [("prefill", 4096), ("relu2", 512)])
def test_workload_full_size(name, n_sample):
    # prefill: every token; relu2 (541 GFLOP in float64): a quarter of the tokens
    cfg = CONFIGS[name]
    e, run = _full_size(cfg, n_sample=n_sample)
    assert e <= (FP8_TOL if cfg.fp8 else BF16_TOL), e
    assert moe.device_status(run.ws)[0] == 0


@pytest.mark.parametrize("T", [1, 4, 16, 64])
def test_decode_full(T):
    cfg = CONFIGS[f"decode_T{T}"]
    run = GpuForward(cfg)
    out = run.forward()
    parts = run.parts()
    _check_route_align(cfg, parts, run.inp["logits"])
    ref = oracle_out(cfg, run.inp)
    got = bf16_to_f64(out)
    report(f"{cfg.name}: beyond-rounding {err_beyond_rounding(got, ref):.4f}, raw {max_err_over_rms(got, ref):.4f}")
    assert err_beyond_rounding(got, ref) <= BF16_TOL


# ---- FP8 E4M3 W8A8 block-128 ---------------------------------------------------------

FP8_SMALL = {
    "fp8_tiny": _small("fp8_tiny", T=64, H=256, E=8, topk=2, I=256, fp8=True),
    # several row tiles per expert, shared slot, H and I not multiples of 256
    "fp8_shared_small": _small("fp8_shared_small", T=300, H=384, E=16, topk=3, I=384, num_shared=1, fp8=True),
    "fp8_relu2": _small("fp8_relu2", T=96, H=256, E=6, topk=2, I=256, activation="relu2", renormalize=False,
                        fp8=True),
    "fp8_gelu": _small("fp8_gelu", T=64, H=256, E=8, topk=2, I=256, activation="gelu_tanh", fp8=True),
    "fp8_oai": _small("fp8_oai", T=200, H=256, E=8, topk=2, I=256, activation="swigluoai", fp8=True, weight_std=0.5),
}


def _check_b128_operands(cfg, parts, a, hidden_bits):
    """FP8 block-128 on the swapped-operand GEMMs: the permuted hidden rows and GEMM2's
    input (GEMM1's own bf16 activation) quantised per 1x128, codes and scales bit for bit
    against the oracle's quantiser (padding rows of X are not written; GEMM1 stores zero
    activation rows for them)."""
    kk = cfg.k_total
    P = cfg.T * kk
    P_pad = int(a["P_pad"])
    gi, ng = parts["group_info"], int(parts["num_blocks"][1])
    pids = a["sorted_pair_ids"][:P_pad]
    real = pids < P
    qx, sx = O.quant_groups_1x128(O.bf16_bits_to_f32(hidden_bits))
    np.testing.assert_array_equal(parts["xq"], qx)          # once per token
    np.testing.assert_array_equal(parts["xq_scale"], sx)
    xs_c, xs_s = untile_b128(parts["xs"], gi, ng, P_pad, cfg.H // 128)
    np.testing.assert_array_equal(xs_c[real], qx[pids[real] // kk])
    np.testing.assert_array_equal(xs_s[real], sx[pids[real] // kk])
    act_bits = untile_groups(parts["act"], gi, ng, P_pad, -(-cfg.I // 64))[:, :cfg.I]
    assert np.all(act_bits[~real] == 0)
    qa, sa = O.quant_groups_1x128(O.bf16_bits_to_f32(act_bits[real]))
    aq_c, aq_s = untile_b128(parts["actq"], gi, ng, P_pad, cfg.I // 128)
    np.testing.assert_array_equal(aq_c[real], qa)
    np.testing.assert_array_equal(aq_s[real], sa)
    return qx, sx


@pytest.mark.parametrize("name,bm", [(n, 0) for n in FP8_SMALL] +
                         [(n, 128) for n in ("fp8_tiny", "fp8_shared_small", "fp8_relu2", "fp8_oai")])
def test_fp8_layer_parity_small(name, bm):
    # bm 0: the default (16-row alignment, weights on the MMA's M, per-chunk partials
    # promoted in the epilogue); 128: 128-row token tiles
    cfg = FP8_SMALL[name]
    run = GpuForward(cfg, block_m=bm)
    out = run.forward()
    parts = run.parts()
    ids, a = _check_route_align(cfg, parts, run.inp["logits"])
    if parts["block_m"] == 16:
        qx, sx = _check_b128_operands(cfg, parts, a, bits(run.inp["hidden"]))
    else:
        # the GPU quantises its own bf16 activation per 1x128 group: codes and scales must be
        # what the oracle's quantiser gives for those same bf16 values
        rows = np.nonzero(a["sorted_pair_ids"] < cfg.T * cfg.k_total)[0]
        act32 = O.bf16_bits_to_f32(parts["act"][rows])
        q, sc = O.quant_groups_1x128(act32)
        np.testing.assert_array_equal(parts["actq"][rows], q)
        np.testing.assert_array_equal(parts["act_scale"][rows], sc)
        # the hidden quantisation too
        qx, sx = O.quant_groups_1x128(O.bf16_bits_to_f32(bits(run.inp["hidden"])))
        np.testing.assert_array_equal(parts["xq"], qx)
        np.testing.assert_array_equal(parts["xq_scale"], sx)
    fp8w = O.quantize_weights_fp8(bits(run.inp["w13"]), bits(run.inp["w2"]))
    np.testing.assert_array_equal(run.w13_q.cpu().numpy(), fp8w[0])
    np.testing.assert_array_equal(run.w13_scale.cpu().numpy(), fp8w[1])
    # GEMM1's bf16 activation element by element against the oracle's activation of the
    # same quantised operands (before its 1x128 re-quantisation)
    xd = O.dequant_groups_1x128(qx, sx)
    check_act_pairs(
        lambda e, t: O.activation_fn(xd[t] @ O.dequant_blocks_128x128(fp8w[0][e], fp8w[1][e]).T, cfg.activation,
                                     cfg.I),
        act_rows_f64(parts, run.I_pad), ids, np.arange(cfg.T), a["pair_to_row"], bf16_act_bound)
    ref = oracle_out(cfg, run.inp, fp8_weights=fp8w)
    got = bf16_to_f64(out)
    assert np.all(np.isfinite(got))
    e = err_beyond_rounding(got, ref)
    report(f"{name}/bm{parts['block_m']}: beyond-rounding {e:.4f}, raw {max_err_over_rms(got, ref):.4f}")
    assert e <= FP8_TOL, e
    assert moe.device_status(run.ws)[0] == 0


@pytest.mark.parametrize("T,bm", [(16, 128), (64, 128), (4, 16)])
def test_decode_both_row_tilings(T, bm):
    # the same decode batch through 16-row token blocks (weights as the MMA's M operand)
    # and through 128-row tiles must both match the oracle
    cfg = CONFIGS[f"decode_T{T}"]
    run = GpuForward(cfg, block_m=bm)
    out = run.forward()
    parts = run.parts()
    assert parts["block_m"] == bm
    _check_route_align(cfg, parts, run.inp["logits"])
    ref = oracle_out(cfg, run.inp)
    assert err_beyond_rounding(bf16_to_f64(out), ref) <= BF16_TOL


FUSED_ROUTE_ALIGN = {
    "tiny": CONFIGS["tiny"],
    "decode_T1": CONFIGS["decode_T1"],
    "decode_T16": CONFIGS["decode_T16"],
    "shared_t12": _small("shared_t12", T=12, H=256, E=12, topk=3, I=256, num_shared=1),
}


@pytest.mark.parametrize("name", sorted(FUSED_ROUTE_ALIGN))
def test_fused_route_align_matches_the_separate_steps(name):
    # batches of at most 16 tokens route and align in one kernel inside the forward; its
    # routing, permutation, offsets and row groups must be those of the separate route and
    # align steps, bit for bit
    cfg = FUSED_ROUTE_ALIGN[name]
    assert cfg.T <= 16
    run = GpuForward(cfg)
    run.forward()
    keys = ["topk_ids", "topk_w", "sorted_pair_ids", "expert_offsets", "pair_to_row", "num_blocks", "group_info"]
    fused = {k: v.clone() for k, v in moe.read_workspace(run.prob, run.ws).items() if k in keys + ["xs"]}
    run.ws.zero_()
    moe.stage_route(run.prob, run.logits, run.ws)
    moe.stage_align(run.prob, run.ws)
    moe.stage_permute(run.prob, run.hidden, run.ws)
    torch.cuda.synchronize()
    staged = moe.read_workspace(run.prob, run.ws)
    # the permuted token rows (fused into the same kernel for at most 64 bf16 pairs)
    P = cfg.T * cfg.k_total
    ng = int(staged["num_blocks"][1])
    P_pad = int(staged["expert_offsets"][-1])
    pids = staged["sorted_pair_ids"][:P_pad].cpu().numpy()
    real = pids < P
    gi = staged["group_info"].cpu().numpy()
    xs_f = untile_groups(bits(fused["xs"]), gi, ng, P_pad, cfg.H // 64)
    xs_s = untile_groups(bits(staged["xs"]), gi, ng, P_pad, cfg.H // 64)
    np.testing.assert_array_equal(xs_f[real], xs_s[real])
    np.testing.assert_array_equal(xs_s[real], bits(run.inp["hidden"])[pids[real] // cfg.k_total])
    # only the written prefixes: the padded rows and the row groups that align produced
    rows = int(staged["expert_offsets"][-1])
    groups = int(staged["num_blocks"][1])
    assert int(fused["expert_offsets"][-1]) == rows and int(fused["num_blocks"][1]) == groups
    fused["sorted_pair_ids"], staged["sorted_pair_ids"] = fused["sorted_pair_ids"][:rows], staged["sorted_pair_ids"][:rows]
    fused["group_info"], staged["group_info"] = fused["group_info"][:groups], staged["group_info"][:groups]
    for k in keys:
        assert torch.equal(fused[k].cpu(), staged[k].cpu()), k


# ---- caller-supplied routing (the routed variant) -------------------------------------

def _routed_call(run, ids, w, cfg):
    out = torch.empty_like(run.hidden)
    moe.moe_forward_routed(run.hidden, ids.cuda().contiguous(), w.cuda().contiguous(), run.w13p, run.w2p, cfg.E,
                           cfg.activation, run.w13_scale, run.w2_scale, num_shared=cfg.num_shared,
                           workspace=run.ws, out=out)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("name", ["ragged", "shared_bf16", "tiny"])
def test_routed_with_own_routing_is_bitwise_the_forward(name):
    # the routed entry point given the route step's own choice runs the same kernels on
    # the same routing, so its output is the forward's, bit for bit
    cfg = SMALL[name]
    run = GpuForward(cfg)
    ref = bits(run.forward()).copy()
    parts = run.parts()
    ids = torch.from_numpy(parts["topk_ids"][:, :cfg.topk].copy())
    w = torch.from_numpy(parts["topk_w"][:, :cfg.topk].copy())
    np.testing.assert_array_equal(bits(_routed_call(run, ids, w, cfg)), ref)
    assert moe.device_status(run.ws)[0] == 0


@pytest.mark.parametrize("name", ["skewed", "shared_bf16", "fp8_tiny"])
def test_routed_arbitrary_routing_matches_oracle(name):
    # repeated experts within a token and weights that are not a softmax
    cfg = SMALL.get(name) or FP8_SMALL[name]
    run = GpuForward(cfg)
    g = torch.Generator().manual_seed(21)
    ids = torch.randint(0, cfg.E, (cfg.T, cfg.topk), generator=g, dtype=torch.int32)
    ids[::5, 0] = ids[::5, -1]                      # repeats
    w = torch.rand((cfg.T, cfg.topk), generator=g) * 2.0
    got = bf16_to_f64(_routed_call(run, ids, w, cfg))
    routing = O.append_shared_slot(ids.numpy(), w.numpy(), cfg.E, cfg.num_shared)
    if cfg.fp8:
        ref = O.moe_forward_fp8(bits(run.inp["hidden"]), None, *O.quantize_weights_fp8(
            bits(run.inp["w13"]), bits(run.inp["w2"])), topk=cfg.topk, renormalize=False,
            activation=cfg.activation, num_shared=cfg.num_shared, routing=routing)
    else:
        ref = O.moe_forward(bits(run.inp["hidden"]), None, bits(run.inp["w13"]), bits(run.inp["w2"]),
                            topk=cfg.topk, renormalize=False, activation=cfg.activation,
                            num_shared=cfg.num_shared, routing=routing)
    e = err_beyond_rounding(got, ref)
    assert e <= (FP8_TOL if cfg.fp8 else BF16_TOL), e
    assert moe.device_status(run.ws)[0] == 0


def test_routed_out_of_range_ids_are_dropped_and_reported():
    cfg = SMALL["ragged"]
    run = GpuForward(cfg)
    g = torch.Generator().manual_seed(22)
    ids = torch.randint(0, cfg.E, (cfg.T, cfg.topk), generator=g, dtype=torch.int32)
    w = torch.rand((cfg.T, cfg.topk), generator=g)
    ids[3, 1] = -1
    ids[10, 0] = cfg.E            # one past the last routed expert
    got = bf16_to_f64(_routed_call(run, ids, w, cfg))
    st, word = moe.device_status(run.ws)
    assert st == 1 and word == 0x20000            # MOE_ERR_INVALID_ARG, bad routing
    assert moe.device_status(run.ws)[0] == 0      # the query cleared it
    # the dropped pairs contribute nothing: the oracle with their weights set to zero
    ids_ok, w_ok = ids.clone(), w.clone()
    for t, j in ((3, 1), (10, 0)):
        ids_ok[t, j] = 0
        w_ok[t, j] = 0.0
    ref = O.moe_forward(bits(run.inp["hidden"]), None, bits(run.inp["w13"]), bits(run.inp["w2"]),
                        topk=cfg.topk, renormalize=False, activation=cfg.activation,
                        routing=O.append_shared_slot(ids_ok.numpy(), w_ok.numpy(), cfg.E, 0))
    assert err_beyond_rounding(got, ref) <= BF16_TOL


# ---- per-tensor FP8 -------------------------------------------------------------------

PT_SMALL = {
    "pt_swiglu": _small("pt_swiglu", T=300, H=256, E=8, topk=2, I=256),
    "pt_relu2": _small("pt_relu2", T=200, H=384, E=6, topk=3, I=384, activation="relu2", renormalize=False),
    "pt_gelu_shared": _small("pt_gelu_shared", T=130, H=256, E=12, topk=3, I=256, num_shared=1,
                             activation="gelu_tanh"),
    # groups of more than 128 rows (one K chunk per step) and three align chunks
    "pt_big_groups": _small("pt_big_groups", T=1500, H=256, E=4, topk=2, I=128),
    "pt_decode": _small("pt_decode", T=4, H=512, E=32, topk=4, I=256),
    "pt_oai": _small("pt_oai", T=200, H=256, E=8, topk=2, I=256, activation="swigluoai", weight_std=0.5),
}


@pytest.mark.parametrize("name", list(PT_SMALL))
def test_fp8_per_tensor_layer_parity(name):
    cfg = PT_SMALL[name]
    inp = make_inputs(cfg, 0)
    dev = torch.device("cuda:0")
    hidden, logits = inp["hidden"].to(dev), inp["logits"].to(dev)
    w13, w2 = inp["w13"].to(dev), inp["w2"].to(dev)
    # device quantiser, bit-exact against the oracle's
    q13, s13 = moe.quantize_weights_fp8_per_tensor(w13)
    q2, s2 = moe.quantize_weights_fp8_per_tensor(w2)
    o13, os13, o2, os2 = O.quantize_weights_fp8_per_tensor(bits(inp["w13"]), bits(inp["w2"]))
    np.testing.assert_array_equal(q13.cpu().numpy(), o13)
    np.testing.assert_array_equal(q2.cpu().numpy(), o2)
    np.testing.assert_array_equal(s13.cpu().numpy(), os13)
    np.testing.assert_array_equal(s2.cpu().numpy(), os2)
    # static scales: the hidden amax, and an activation calibration from the bf16 oracle's
    # GEMM1 output on these inputs (values beyond it saturate, in the kernel and the oracle)
    s_in = float(np.float32(np.abs(bf16_to_f64(inp["hidden"])).max() / 448))
    x = bf16_to_f64(inp["hidden"])
    W13 = bf16_to_f64(inp["w13"])
    ids0, _ = O.route(inp["logits"].numpy(), cfg.topk, cfg.renormalize, cfg.num_shared)
    amax = max(float(np.abs(O.activation_fn(x[np.nonzero(ids0 == e)[0]] @ W13[e].T, cfg.activation, cfg.I)).max())
               for e in np.unique(ids0))
    s_act = float(np.float32(amax / 448 * 0.8))
    prob = moe.make_problem(cfg.T, cfg.H, cfg.E, cfg.topk, cfg.I, renormalize=cfg.renormalize,
                            activation=cfg.activation, num_shared=cfg.num_shared, fp8="per_tensor",
                            input_scale=s_in, activation_scale=s_act)
    w13p, w2p = moe.prepare_weights(prob, q13, q2, cfg.I)
    ws = dirty_workspace(prob)
    out = moe.moe_forward(hidden, logits, w13p, w2p, cfg.topk, cfg.renormalize, cfg.activation, s13, s2,
                          num_shared=cfg.num_shared, workspace=ws, input_scale=s_in, activation_scale=s_act)
    torch.cuda.synchronize()
    assert moe.device_status(ws)[0] == 0
    parts = {k: v.cpu().numpy() for k, v in moe.read_workspace(prob, ws).items()}
    # routing and permutation, bit for bit
    ids_o, w_o = O.route(inp["logits"].numpy(), cfg.topk, cfg.renormalize, cfg.num_shared)
    np.testing.assert_array_equal(parts["topk_ids"], ids_o)
    al = O.align(ids_o, cfg.E_total, 16)
    P_pad = int(al["P_pad"])
    np.testing.assert_array_equal(parts["sorted_pair_ids"][:P_pad], al["sorted_pair_ids"])
    # the permuted, quantised hidden rows: e4m3(hidden * fp32(1 / input_scale)), bit for bit
    ng = int(parts["num_blocks"][1])
    xs = untile_u8(parts["xs"], parts["group_info"], ng, P_pad, cfg.H // 128)
    pids = al["sorted_pair_ids"][:P_pad]
    real = pids < cfg.T * cfg.k_total
    xq = O.quant_per_tensor_inv(O.bf16_bits_to_f32(bits(inp["hidden"])), s_in)
    np.testing.assert_array_equal(xs[real], xq[pids[real] // cfg.k_total])
    # the layer
    ref = O.moe_forward_fp8_per_tensor(bits(inp["hidden"]), inp["logits"].numpy(), o13, os13, o2, os2, s_in, s_act,
                                       topk=cfg.topk, renormalize=cfg.renormalize, activation=cfg.activation,
                                       num_shared=cfg.num_shared)
    got = bf16_to_f64(out)
    assert np.all(np.isfinite(got))
    e = err_beyond_rounding(got, ref)
    report(f"{name}: beyond-rounding {e:.4f}, raw {max_err_over_rms(got, ref):.4f}")
    assert e <= FP8_TOL, e


# ---- MXFP8 ------------------------------------------------------------------------------

MX_SMALL = {
    "mx_swiglu": _small("mx_swiglu", T=300, H=256, E=8, topk=2, I=256, fp8="mxfp8"),
    "mx_relu2": _small("mx_relu2", T=200, H=384, E=6, topk=3, I=384, activation="relu2", renormalize=False,
                       fp8="mxfp8"),
    "mx_gelu_shared": _small("mx_gelu_shared", T=130, H=256, E=12, topk=3, I=256, num_shared=1,
                             activation="gelu_tanh", fp8="mxfp8"),
    # row groups of 129-192 rows (two 128-row scale blocks per chunk, one K chunk per step)
    # and three align chunks
    "mx_big_groups": _small("mx_big_groups", T=1500, H=256, E=4, topk=2, I=128, fp8="mxfp8"),
    "mx_decode": _small("mx_decode", T=4, H=512, E=32, topk=4, I=256, fp8="mxfp8"),
    "mx_oai": _small("mx_oai", T=200, H=256, E=8, topk=2, I=256, activation="swigluoai", fp8="mxfp8",
                     weight_std=0.5),
}


def _mx_group_scales(sf_flat, group_info, num_groups, rows, kchunks):
    """[rows, 4 * kchunks] scale bytes from the row-group scale blocks: the group at x_row
    owns the 1024-byte block ((x_row / 16) * kchunks + c) * 1024 of chunk c, whose byte
    512 h + 16 l + 4 j + k is the scale of group row 128 h + 32 j + l for K block 4 c + k."""
    flat = np.asarray(sf_flat).reshape(-1)
    out = np.zeros((rows, 4 * kchunks), dtype=np.uint8)
    for g in range(num_groups):
        x_row, meta = int(group_info[g][0]), int(group_info[g][1])
        n = (meta >> 16) & 0x1FF
        for r in range(n):
            for c in range(kchunks):
                base = ((x_row // 16) * kchunks + c) * 1024 + (r // 128) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4
                out[x_row + r, 4 * c:4 * c + 4] = flat[base:base + 4]
    return out


def _mx_weight_scales(flat, E, rows, K, gated):
    """The tiled weight scale blocks back to the checkpoint layout [E, rows, K/32] (gated w13
    rows un-interleaved)."""
    MT, KC = -(-rows // 128), -(-K // 128)
    t = np.asarray(flat).reshape(E, MT, KC, 32, 4, 4)            # [e, m, c, l, j, k]
    s = t.transpose(0, 1, 4, 3, 2, 5).reshape(E, MT * 128, KC * 4)  # row 128 m + 32 j + l, block 4 c + k
    s = s[:, :rows, :K // 32]
    if gated:
        I = rows // 2
        s = np.concatenate([s[:, 0::2], s[:, 1::2]], axis=1)      # [gate0, up0, ...] -> gate rows, up rows
        assert s.shape[1] == 2 * I
    return s


@pytest.mark.parametrize("name", list(MX_SMALL))
def test_mxfp8_layer_parity(name):
    cfg = MX_SMALL[name]
    _mx_parity(cfg, make_inputs(cfg, 0), name)


def test_mxfp8_zero_blocks_and_rows():
    """All-zero 32-column blocks (scale byte 0, codes 0) and all-zero hidden rows."""
    cfg = MX_SMALL["mx_swiglu"]
    inp = make_inputs(cfg, 0)
    h = inp["hidden"].clone()
    h[::7] = 0                       # whole rows
    h[1::5, 32:96] = 0               # two 32-column blocks of other rows
    h[2::9, 224:256] = 0             # the last block
    inp["hidden"] = h
    _mx_parity(cfg, inp, "mx_zero_blocks")


def _mx_parity(cfg, inp, name):
    dev = torch.device("cuda:0")
    hidden, logits = inp["hidden"].to(dev), inp["logits"].to(dev)
    # device quantiser, bit-exact against the oracle's (OCP MX conversion decided in fp32)
    q13, s13 = moe.quantize_weights_mxfp8(inp["w13"].to(dev))
    q2, s2 = moe.quantize_weights_mxfp8(inp["w2"].to(dev))
    o13, os13, o2, os2 = O.quantize_weights_mxfp8(bits(inp["w13"]), bits(inp["w2"]))
    np.testing.assert_array_equal(q13.cpu().numpy(), o13)
    np.testing.assert_array_equal(s13.cpu().numpy(), os13)
    np.testing.assert_array_equal(q2.cpu().numpy(), o2)
    np.testing.assert_array_equal(s2.cpu().numpy(), os2)
    prob = moe.make_problem(cfg.T, cfg.H, cfg.E, cfg.topk, cfg.I, renormalize=cfg.renormalize,
                            activation=cfg.activation, num_shared=cfg.num_shared, fp8="mxfp8")
    w13p, w2p = moe.prepare_weights(prob, q13, q2, cfg.I, w13_scale=s13, w2_scale=s2)
    # prepared layout: the codes as the per-tensor tiles, then one scale block per tile
    E, N1 = cfg.E_total, cfg.N1
    c13 = 16384 * E * (-(-N1 // 128)) * (cfg.H // 128)
    c2 = 16384 * E * (cfg.H // 128) * (cfg.I // 128)
    np.testing.assert_array_equal(_mx_weight_scales(w13p[c13:].cpu().numpy(), E, N1, cfg.H, cfg.gated), os13)
    np.testing.assert_array_equal(_mx_weight_scales(w2p[c2:].cpu().numpy(), E, cfg.H, cfg.I, False), os2)
    ws = dirty_workspace(prob)
    out = moe.moe_forward(hidden, logits, w13p, w2p, cfg.topk, cfg.renormalize, cfg.activation,
                          num_shared=cfg.num_shared, workspace=ws)
    torch.cuda.synchronize()
    assert moe.device_status(ws)[0] == 0
    raw = moe.read_workspace(prob, ws)
    act_bits = raw.pop("act").view(torch.int16).cpu().numpy().view(np.uint16)
    parts = {k: v.cpu().numpy() for k, v in raw.items()}
    ids_o, _ = O.route(inp["logits"].numpy(), cfg.topk, cfg.renormalize, cfg.num_shared)
    np.testing.assert_array_equal(parts["topk_ids"], ids_o)
    al = O.align(ids_o, cfg.E_total, 16)
    P_pad = int(al["P_pad"])
    np.testing.assert_array_equal(parts["sorted_pair_ids"][:P_pad], al["sorted_pair_ids"])
    ng = int(parts["num_blocks"][1])
    gi = parts["group_info"]
    assert max((int(gi[g][1]) >> 16) & 0x1FF for g in range(ng)) <= 192
    # the permuted hidden rows: MXFP8 codes and scale bytes, bit for bit
    pids = al["sorted_pair_ids"][:P_pad]
    real = pids < cfg.T * cfg.k_total
    xq, xsc = O.quant_mx(O.bf16_bits_to_f32(bits(inp["hidden"])))
    xs = untile_u8(parts["xs"], gi, ng, P_pad, cfg.H // 128)
    np.testing.assert_array_equal(xs[real], xq[pids[real] // cfg.k_total])
    xss = _mx_group_scales(parts["xs_scale"], gi, ng, P_pad, cfg.H // 128)
    np.testing.assert_array_equal(xss[real], xsc[pids[real] // cfg.k_total])
    # GEMM2's input: the kernel's own bf16 activation quantised per 32, bit for bit
    act = untile_groups(act_bits, gi, ng, P_pad, -(-cfg.I // 64))[:, :cfg.I]
    aq, asc = O.quant_mx(O.bf16_bits_to_f32(act))
    np.testing.assert_array_equal(untile_u8(parts["actq"], gi, ng, P_pad, cfg.I // 128), aq)
    np.testing.assert_array_equal(_mx_group_scales(parts["act_scale"], gi, ng, P_pad, cfg.I // 128), asc)
    # the layer
    ref = O.moe_forward_mxfp8(bits(inp["hidden"]), inp["logits"].numpy(), o13, os13, o2, os2, topk=cfg.topk,
                              renormalize=cfg.renormalize, activation=cfg.activation, num_shared=cfg.num_shared)
    got = bf16_to_f64(out)
    assert np.all(np.isfinite(got))
    e = err_beyond_rounding(got, ref)
    report(f"{name}: beyond-rounding {e:.4f}, raw {max_err_over_rms(got, ref):.4f}")
    assert e <= FP8_TOL, e


def test_mxfp8_full_size_every_expert():
    """The MXFP8 prefill workload at full size: routing and align over all tokens, the
    layer output and GEMM1's stored activation on a token sample that covers every
    routed expert."""
    cfg = CONFIGS["mxfp8_prefill"]
    inp = make_inputs(cfg, 0)
    dev = torch.device("cuda:0")
    q13, s13 = moe.quantize_weights_mxfp8(inp["w13"].to(dev))
    q2, s2 = moe.quantize_weights_mxfp8(inp["w2"].to(dev))
    prob = moe.make_problem(cfg.T, cfg.H, cfg.E, cfg.topk, cfg.I, renormalize=cfg.renormalize,
                            activation=cfg.activation, fp8="mxfp8")
    w13p, w2p = moe.prepare_weights(prob, q13, q2, cfg.I, w13_scale=s13, w2_scale=s2)
    del q13, q2, s13, s2
    ws = dirty_workspace(prob)
    out = moe.moe_forward(inp["hidden"].to(dev), inp["logits"].to(dev), w13p, w2p, cfg.topk, cfg.renormalize,
                          cfg.activation, workspace=ws)
    torch.cuda.synchronize()
    assert moe.device_status(ws)[0] == 0
    raw = moe.read_workspace(prob, ws)
    act_bits = raw.pop("act").view(torch.int16).cpu().numpy().view(np.uint16)
    parts = {k: v.cpu().numpy() for k, v in raw.items()}
    ids, _ = O.route(inp["logits"].numpy(), cfg.topk, cfg.renormalize)
    np.testing.assert_array_equal(parts["topk_ids"], ids)
    al = O.align(ids, cfg.E_total, 16)
    P_pad = int(al["P_pad"])
    np.testing.assert_array_equal(parts["sorted_pair_ids"][:P_pad], al["sorted_pair_ids"])
    np.testing.assert_array_equal(parts["pair_to_row"], al["pair_to_row"])
    tokens = cover_tokens(ids, cfg.E, extra=16)
    experts = np.unique(ids[tokens])
    assert len(experts) == len(np.unique(ids))
    o13, os13, o2, os2 = oracle_mxfp8_weights(bits(inp["w13"]), bits(inp["w2"]), experts)
    # GEMM1's bf16 activation of every sampled pair against the oracle's (same MXFP8 inputs)
    gi, ng = parts["group_info"], int(parts["num_blocks"][1])
    act = bf16_to_f64(untile_groups(act_bits, gi, ng, P_pad, -(-cfg.I // 64))[:, :cfg.I])
    x = O.dequant_mx(*O.quant_mx(O.bf16_bits_to_f32(bits(inp["hidden"]))))
    n = check_act_pairs(lambda e, t: O.activation_fn(x[t] @ O.dequant_mx(o13[e], os13[e]).T, cfg.activation, cfg.I),
                        act, ids, tokens, al["pair_to_row"], bf16_act_bound)
    ref = O.moe_forward_mxfp8(bits(inp["hidden"]), inp["logits"].numpy(), o13, os13, o2, os2, topk=cfg.topk,
                              renormalize=cfg.renormalize, activation=cfg.activation, tokens=tokens)
    got = bf16_to_f64(out.cpu()[torch.from_numpy(tokens)])
    e = err_beyond_rounding(got, ref)
    report(f"mxfp8_prefill: {len(tokens)} tokens over {len(experts)} experts, {n} activation values; "
          f"beyond-rounding {e:.4f}, raw {max_err_over_rms(got, ref):.4f}")
    assert e <= FP8_TOL, e


def test_fp8_block128_full_size_every_expert():
    """FP8 block-128 with the fused shared slot at full size (T=8192, 512+1 experts,
    top-10+1): routing and align over all tokens; the quantised hidden rows bit for bit;
    GEMM1's stored activation and the layer output on a token sample that covers every
    routed expert."""
    cfg = CONFIGS["fp8_shared"]
    run = GpuForward(cfg)
    out = run.forward()
    parts = run.parts()
    ids, a = _check_route_align(cfg, parts, run.inp["logits"])
    assert parts["block_m"] == 16
    qx, sx = _check_b128_operands(cfg, parts, a, bits(run.inp["hidden"]))
    tokens = cover_tokens(ids, cfg.E, extra=16)
    experts = np.unique(ids[tokens])
    assert len(experts) == cfg.E_total
    fp8w = oracle_fp8_block_weights(bits(run.inp["w13"]), bits(run.inp["w2"]), experts)
    xd = O.dequant_groups_1x128(qx, sx)
    act = act_rows_f64(parts, run.I_pad)
    n = check_act_pairs(
        lambda e, t: O.activation_fn(xd[t] @ O.dequant_blocks_128x128(fp8w[0][e], fp8w[1][e]).T, cfg.activation,
                                     cfg.I),
        act, ids, tokens, a["pair_to_row"], bf16_act_bound)
    ref = oracle_out(cfg, run.inp, tokens=tokens, fp8_weights=fp8w)
    got = bf16_to_f64(out)[tokens]
    assert np.all(np.isfinite(bf16_to_f64(out)))
    e = err_beyond_rounding(got, ref)
    report(f"fp8_shared: {len(tokens)} tokens over {len(experts)} experts, {n} activation values; "
          f"beyond-rounding {e:.4f}, raw {max_err_over_rms(got, ref):.4f}")
    assert e <= FP8_TOL, e
    assert moe.device_status(run.ws)[0] == 0


def _e4m3_within_one_step(ref_scaled: np.ndarray, got_codes: np.ndarray) -> np.ndarray:
    """True where the code is the e4m3 rounding of ref_scaled (saturated at 448) or the
    neighbouring value: fp32 accumulation against float64 may flip a rounding decision."""
    r = np.clip(ref_scaled, -448.0, 448.0)
    step = np.ldexp(1.0, np.maximum(np.floor(np.log2(np.maximum(np.abs(r), 2.0 ** -9))), -6).astype(np.int64) - 3)
    return np.abs(O.e4m3_decode(got_codes) - r) <= step * (1 + 1e-9)


def test_fp8_per_tensor_full_size_every_expert():
    """Per-tensor FP8 with the fused shared slot at its full benchmarked shape (T=8192,
    512+1 experts, top-10+1), with the static scales calibrated as the benchmark does
    (input scale = amax(hidden) / 448, activation scale 0.03): weights, routing, align
    and the quantised permuted hidden rows bit for bit; GEMM1's e4m3 activation codes
    within one step of the oracle's and the layer output on a token sample that covers
    every routed expert."""
    cfg = CONFIGS["fp8pt_shared"]
    inp = make_inputs(cfg, 0)
    dev = torch.device("cuda:0")
    s_in = float(inp["hidden"].float().abs().max() / 448)
    s_act = cfg.activation_scale
    q13, s13 = moe.quantize_weights_fp8_per_tensor(inp["w13"].to(dev))
    q2, s2 = moe.quantize_weights_fp8_per_tensor(inp["w2"].to(dev))
    o13, os13, o2, os2 = O.quantize_weights_fp8_per_tensor(bits(inp["w13"]), bits(inp["w2"]))
    np.testing.assert_array_equal(s13.cpu().numpy(), os13)
    np.testing.assert_array_equal(s2.cpu().numpy(), os2)
    np.testing.assert_array_equal(q13.cpu().numpy(), o13)
    np.testing.assert_array_equal(q2.cpu().numpy(), o2)
    prob = moe.make_problem(cfg.T, cfg.H, cfg.E, cfg.topk, cfg.I, renormalize=cfg.renormalize,
                            activation=cfg.activation, num_shared=cfg.num_shared, fp8="per_tensor",
                            input_scale=s_in, activation_scale=s_act)
    w13p, w2p = moe.prepare_weights(prob, q13, q2, cfg.I)
    del q13, q2
    ws = dirty_workspace(prob)
    out = moe.moe_forward(inp["hidden"].to(dev), inp["logits"].to(dev), w13p, w2p, cfg.topk, cfg.renormalize,
                          cfg.activation, s13, s2, num_shared=cfg.num_shared, workspace=ws, input_scale=s_in,
                          activation_scale=s_act)
    torch.cuda.synchronize()
    assert moe.device_status(ws)[0] == 0
    parts = {k: v.cpu().numpy() for k, v in moe.read_workspace(prob, ws).items()}
    ids, w = O.route(inp["logits"].numpy(), cfg.topk, cfg.renormalize, cfg.num_shared)
    np.testing.assert_array_equal(parts["topk_ids"], ids)
    np.testing.assert_allclose(parts["topk_w"], w, rtol=1e-5, atol=1e-7)
    al = O.align(ids, cfg.E_total, 16)
    P_pad = int(al["P_pad"])
    np.testing.assert_array_equal(parts["sorted_pair_ids"][:P_pad], al["sorted_pair_ids"])
    np.testing.assert_array_equal(parts["pair_to_row"], al["pair_to_row"])
    gi, ng = parts["group_info"], int(parts["num_blocks"][1])
    pids = al["sorted_pair_ids"][:P_pad]
    real = pids < cfg.T * cfg.k_total
    xq = O.quant_per_tensor_inv(O.bf16_bits_to_f32(bits(inp["hidden"])), s_in)
    xs = untile_u8(parts["xs"], gi, ng, P_pad, cfg.H // 128)
    np.testing.assert_array_equal(xs[real], xq[pids[real] // cfg.k_total])
    tokens = cover_tokens(ids, cfg.E, extra=16)
    assert len(np.unique(ids[tokens])) == cfg.E_total
    # GEMM1's e4m3 activation codes: the oracle's activation / activation_scale, one step
    x = O.e4m3_decode(xq) * np.float64(np.float32(s_in))
    codes = untile_u8(parts["act"], gi, ng, P_pad, cfg.I // 128)
    inv = np.float64(np.float32(1.0) / np.float32(s_act))
    n = check_act_pairs(
        lambda e, t: O.activation_fn(x[t] @ (O.e4m3_decode(o13[e]) * np.float64(os13[e])).T, cfg.activation,
                                     cfg.I) * inv,
        codes, ids, tokens, al["pair_to_row"], lambda ref, got: _e4m3_within_one_step(ref, got.astype(np.uint8)))
    ref = O.moe_forward_fp8_per_tensor(bits(inp["hidden"]), inp["logits"].numpy(), o13, os13, o2, os2, s_in, s_act,
                                       topk=cfg.topk, renormalize=cfg.renormalize, activation=cfg.activation,
                                       num_shared=cfg.num_shared, tokens=tokens)
    got = bf16_to_f64(out.cpu()[torch.from_numpy(tokens)])
    e = err_beyond_rounding(got, ref)
    report(f"fp8pt_shared: {len(tokens)} tokens, {n} activation codes; beyond-rounding {e:.4f}, "
          f"raw {max_err_over_rms(got, ref):.4f}")
    assert e <= FP8_TOL, e
