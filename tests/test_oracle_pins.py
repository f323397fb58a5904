"""Pins for the CPU oracle: brute force, closed forms, library routines, invariants.

Each test checks the oracle against something other than itself, chosen so
that a plausible mistake (dropped term, wrong sign or index, transposed
operand, wrong tie-break or padding) fails at least one of them. The last
tests plant such mistakes in copies of oracle functions and check that the
pins catch them.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def _bf16_bits(x: torch.Tensor) -> np.ndarray:
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# --------------------------------------------------------------------------
# routing
# --------------------------------------------------------------------------


def _route_brute(logits, topk, renorm, num_shared=0):
    """Per-token brute force: Python sort on (-logit, index), math.exp softmax."""
    T, E = logits.shape
    ids, ws = [], []
    for t in range(T):
        row = [float(v) for v in logits[t]]
        sel = sorted(range(E), key=lambda e: (-row[e], e))[:topk]
        m = max(row)
        den = sum(math.exp(v - m) for v in row)
        p = [math.exp(row[e] - m) / den for e in sel]
        if renorm:
            s = sum(p)
            p = [v / s for v in p]
        ids.append(sel + [E] * num_shared)
        ws.append(p + [1.0] * num_shared)
    return np.array(ids, dtype=np.int64).reshape(T, topk + num_shared), np.array(ws).reshape(T, -1)


@pytest.mark.parametrize("E,topk,renorm,shared", [(8, 2, True, 0), (16, 5, False, 0),
                                                  (33, 7, True, 1), (5, 5, False, 0)])
def test_route_matches_brute_force(E, topk, renorm, shared):
    rng = np.random.default_rng(E * 100 + topk)
    logits = rng.standard_normal((40, E)).astype(np.float32)
    # plant exact ties: copy some entries onto others
    logits[3, 1] = logits[3, 0]
    logits[7, :] = 0.25
    ids, w = O.route(logits, topk, renorm, shared)
    bi, bw = _route_brute(logits, topk, renorm, shared)
    np.testing.assert_array_equal(ids, bi)
    np.testing.assert_allclose(w, bw, rtol=2e-7, atol=0)


def test_route_two_expert_closed_form():
    # k = 1 of 2 experts, no renormalisation: w = sigmoid(l_sel - l_other)
    l = np.array([[1.5, -0.25], [-2.0, 0.75]], dtype=np.float32)
    ids, w = O.route(l, 1, False)
    assert ids[:, 0].tolist() == [0, 1]
    exp0 = 1.0 / (1.0 + math.exp(-(1.5 + 0.25)))
    exp1 = 1.0 / (1.0 + math.exp(-(0.75 + 2.0)))
    np.testing.assert_allclose(w[:, 0], [exp0, exp1], rtol=1e-7)
    # renormalised single choice is exactly 1
    _, wr = O.route(l, 1, True)
    assert np.all(wr == 1.0)


def test_route_ties_and_one_hot():
    E, k = 12, 4
    ids, w = O.route(np.zeros((3, E), np.float32), k, False)
    assert ids.tolist() == [[0, 1, 2, 3]] * 3            # lower index wins ties
    np.testing.assert_allclose(w, 1.0 / E, rtol=1e-7)
    _, wr = O.route(np.zeros((3, E), np.float32), k, True)
    np.testing.assert_allclose(wr, 1.0 / k, rtol=1e-7)
    oh = np.full((2, E), -50.0, np.float32)
    oh[0, 7] = 5.0
    oh[1, 11] = 5.0
    ids, _ = O.route(oh, 1, False)
    assert ids[:, 0].tolist() == [7, 11]


def test_route_renormalized_weights_sum_to_one_and_shared_slot():
    rng = np.random.default_rng(3)
    l = rng.standard_normal((50, 64)).astype(np.float32)
    ids, w = O.route(l, 10, True, num_shared=1)
    np.testing.assert_allclose(w[:, :10].astype(np.float64).sum(1), 1.0, atol=1e-6)
    assert np.all(ids[:, 10] == 64) and np.all(w[:, 10] == 1.0)
    # weights are non-increasing along the slots (ordered by logit)
    assert np.all(np.diff(w[:, :10], axis=1) <= 0)


# --------------------------------------------------------------------------
# align
# --------------------------------------------------------------------------


def _align_brute(ids, E, bm):
    flat = [int(v) for v in np.asarray(ids).reshape(-1)]
    P = len(flat)
    order = sorted(range(P), key=lambda p: (flat[p], p))
    sorted_ids, offsets, block_expert = [], [0], []
    pos = 0
    for e in range(E):
        seg = [p for p in order if flat[p] == e]
        n = (len(seg) + bm - 1) // bm * bm
        sorted_ids += seg + [P] * (n - len(seg))
        block_expert += [e] * (n // bm)
        pos += n
        offsets.append(pos)
    p2r = [0] * P
    for r, p in enumerate(sorted_ids):
        if p < P:
            p2r[p] = r
    return sorted_ids, offsets, block_expert, p2r


@pytest.mark.parametrize("T,E,k,bm", [(16, 8, 2, 128), (37, 5, 3, 4), (1, 9, 9, 16), (64, 40, 6, 8)])
def test_align_matches_brute_force(T, E, k, bm):
    rng = np.random.default_rng(T + E)
    l = rng.standard_normal((T, E)).astype(np.float32)
    l[:, 0] += 2.0  # expert 0 overloaded, some experts empty
    ids, _ = O.route(l, k, True)
    a = O.align(ids, E, bm)
    s, off, be, p2r = _align_brute(ids, E, bm)
    assert a["sorted_pair_ids"].tolist() == s
    assert a["expert_offsets"].tolist() == off
    assert a["block_expert"].tolist() == be
    assert a["pair_to_row"].tolist() == p2r
    assert int(a["P_pad"]) == off[-1] and off[-1] % bm == 0


def test_align_empty_and_single_expert():
    a = O.align(np.zeros((0, 2), np.int32), 4, 16)
    assert a["expert_offsets"].tolist() == [0, 0, 0, 0, 0] and a["sorted_pair_ids"].size == 0
    ids = np.full((10, 1), 2, np.int32)
    a = O.align(ids, 4, 8)
    assert a["expert_offsets"].tolist() == [0, 0, 0, 16, 16]
    assert a["sorted_pair_ids"].tolist() == list(range(10)) + [10] * 6
    assert a["block_expert"].tolist() == [2, 2]


# --------------------------------------------------------------------------
# activations and weight preparation (golden fixtures from the pages / closed forms)
# --------------------------------------------------------------------------


def test_activation_closed_forms():
    for fn, x, v in _rows("activation_points.txt"):
        f = O.silu if fn == "silu" else O.relu2
        got = float(f(np.array([float(x)]))[0])
        assert got == pytest.approx(float(v), rel=1e-15, abs=1e-300), (fn, x)
    # limits: silu(x) -> x for large x, -> 0 for very negative x, no NaN at overflow
    assert float(O.silu(np.array([1000.0]))[0]) == 1000.0
    assert float(O.silu(np.array([-1000.0]))[0]) == 0.0


def test_gelu_tanh_against_torch_and_limits():
    # the library routine with the same (tanh) approximation, on a grid and random points
    x = np.concatenate([np.linspace(-12.0, 12.0, 2001), np.random.default_rng(5).standard_normal(4000) * 3])
    want = torch.nn.functional.gelu(torch.from_numpy(x), approximate="tanh").numpy()
    np.testing.assert_allclose(O.gelu_tanh(x), want, rtol=1e-13, atol=1e-15)
    # closed forms: odd part and limits; gelu_tanh(0) = 0, -> x for large x, -> 0 for very negative x
    assert float(O.gelu_tanh(np.array([0.0]))[0]) == 0.0
    assert float(O.gelu_tanh(np.array([30.0]))[0]) == 30.0
    assert abs(float(O.gelu_tanh(np.array([-30.0]))[0])) < 1e-300 or float(O.gelu_tanh(np.array([-30.0]))[0]) == 0.0
    y = np.linspace(0.1, 5.0, 50)
    np.testing.assert_allclose(O.gelu_tanh(y) - O.gelu_tanh(-y), y, rtol=1e-12)   # gelu(x) - gelu(-x) = x
    # the gated form is act(gate) * up on the gate-first halves
    z = np.random.default_rng(6).standard_normal((5, 8))
    np.testing.assert_array_equal(O.activation_fn(z, "gelu_tanh", 4), O.gelu_tanh(z[:, :4]) * z[:, 4:8])
    assert O.is_gated("gelu_tanh") and O.is_gated("swiglu") and not O.is_gated("relu2")


def _swigluoai_decimal(g: float, u: float) -> float:
    """The gpt-oss SwiGLU at one point in 40-digit decimal arithmetic (independent of
    NumPy): g clamped to <= 7, u to [-7, 7], g / (1 + e^(-1.702 g)) * (u + 1)."""
    from decimal import Decimal, getcontext
    getcontext().prec = 40
    gd = min(Decimal(repr(g)), Decimal(7))
    ud = max(min(Decimal(repr(u)), Decimal(7)), Decimal(-7))
    return float(gd / (1 + (-Decimal("1.702") * gd).exp()) * (ud + 1))


def test_swigluoai_closed_forms():
    pts = [(0.0, 5.0), (1.0, 0.0), (2.0, -1.0), (10.0, 10.0), (-3.0, 2.0), (7.0, -9.0), (-20.0, 0.5),
           (6.5, -6.5), (7.5, 3.0), (-0.25, 100.0)]
    for g, u in pts:
        got = float(O.swigluoai(np.array([g]), np.array([u]))[0])
        assert got == pytest.approx(_swigluoai_decimal(g, u), rel=1e-14, abs=1e-300), (g, u)
    # special cases: a zero gate or an up value of -1 gives exactly 0; beyond the limits the
    # value no longer depends on the input (the clamps)
    assert float(O.swigluoai(np.array([0.0]), np.array([3.0]))[0]) == 0.0
    assert float(O.swigluoai(np.array([4.0]), np.array([-1.0]))[0]) == 0.0
    a = O.swigluoai(np.array([7.0, 9.0, 100.0]), np.array([7.0, 8.0, 1e6]))
    assert a[0] == a[1] == a[2]
    assert float(O.swigluoai(np.array([-1000.0]), np.array([1.0]))[0]) == 0.0   # no NaN at overflow
    # inside the limits it is silu(1.702 g) / 1.702 * (u + 1), through the separately pinned silu
    rng = np.random.default_rng(8)
    g = rng.uniform(-7, 7, 500)
    u = rng.uniform(-7, 7, 500)
    np.testing.assert_allclose(O.swigluoai(g, u), O.silu(1.702 * g) / 1.702 * (u + 1.0), rtol=1e-12, atol=1e-15)
    # the gated form takes the gate-first (un-interleaved) halves
    z = rng.standard_normal((5, 8)) * 4
    np.testing.assert_array_equal(O.activation_fn(z, "swigluoai", 4), O.swigluoai(z[:, :4], z[:, 4:8]))
    assert O.is_gated("swigluoai")


def test_routed_variant_equals_logit_routing():
    # the forward with caller-supplied routing, given route()'s routed choice, is the
    # logit-routed forward; append_shared_slot adds the shared slot exactly as route()
    rng = np.random.default_rng(13)
    T, H, E, k, I = 7, 32, 5, 2, 16
    x = _bf16_bits(torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)))
    l = rng.standard_normal((T, E)).astype(np.float32)
    for shared in (0, 1):
        Et = E + shared
        w13 = _bf16_bits(torch.from_numpy(0.2 * rng.standard_normal((Et, 2 * I, H)).astype(np.float32)))
        w2 = _bf16_bits(torch.from_numpy(0.2 * rng.standard_normal((Et, H, I)).astype(np.float32)))
        ids, w = O.route(l, k, True, shared)
        rid, rw = O.append_shared_slot(ids[:, :k], w[:, :k], E, shared)
        np.testing.assert_array_equal(rid, ids)
        np.testing.assert_array_equal(rw, w)
        a = O.moe_forward(x, l, w13, w2, topk=k, renormalize=True, activation="swiglu", num_shared=shared)
        b = O.moe_forward(x, None, w13, w2, topk=k, renormalize=True, activation="swiglu", num_shared=shared,
                          routing=(rid, rw))
        np.testing.assert_array_equal(a, b)
        # arbitrary routing (repeated experts, unnormalised weights) against the dense form
        rid2 = rng.integers(0, E, size=(T, k)).astype(np.int32)
        rw2 = rng.uniform(0.1, 2.0, size=(T, k)).astype(np.float32)
        rid2, rw2 = O.append_shared_slot(rid2, rw2, E, shared)
        got = O.moe_forward(x, None, w13, w2, topk=k, renormalize=True, activation="swiglu", num_shared=shared,
                            routing=(rid2, rw2))
        X, W13, W2 = O.bf16_bits_to_f64(x), O.bf16_bits_to_f64(w13), O.bf16_bits_to_f64(w2)
        want = np.zeros((T, H))
        for t in range(T):
            for j in range(rid2.shape[1]):
                e = rid2[t, j]
                z = W13[e] @ X[t]
                want[t] += float(rw2[t, j]) * (W2[e] @ (z[:I] / (1 + np.exp(-z[:I])) * z[I:]))
        np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)


def test_padding_rules_from_page():
    for i_in, gated, i_pad in _rows("padding_rules.txt"):
        assert O.padded_intermediate(int(i_in), gated == "1") == int(i_pad)


def test_interleave_order_from_page():
    rows = _rows("interleave_order.txt")
    I = int(rows[0][1])
    want = rows[1]
    labels = [f"g{j}" for j in range(I)] + [f"u{j}" for j in range(I)]
    w = np.arange(2 * I, dtype=np.float64).reshape(1, 2 * I, 1)
    got = O.interleave_gate_up(w, I)[0, :, 0].astype(int)
    assert [labels[i] for i in got] == want


def test_padding_leaves_layer_unchanged():
    # zero-padding the intermediate size adds exact zeros: silu(0)*0 = relu2(0) =
    # swigluoai(0, 0) = 0
    rng = np.random.default_rng(5)
    for act, I in (("swiglu", 40), ("relu2", 100), ("swigluoai", 40)):
        gated = act != "relu2"
        T, H, E, k = 6, 128, 3, 2
        x = _bf16_bits(torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)))
        l = rng.standard_normal((T, E)).astype(np.float32)
        w13 = _bf16_bits(torch.from_numpy(0.1 * rng.standard_normal((E, (2 if gated else 1) * I, H)).astype(np.float32)))
        w2 = _bf16_bits(torch.from_numpy(0.1 * rng.standard_normal((E, H, I)).astype(np.float32)))
        p13, p2, I_pad = O.pad_weights(w13, w2, I, gated)
        assert I_pad == O.padded_intermediate(I, gated) and I_pad > I
        a = O.moe_forward(x, l, w13, w2, topk=k, renormalize=True, activation=act)
        b = O.moe_forward(x, l, p13, p2, topk=k, renormalize=True, activation=act)
        np.testing.assert_allclose(b, a, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# whole layer: dense-FFN invariant and scalar brute force
# --------------------------------------------------------------------------


def _dense_layer(x, logits, w13, w2, topk, renorm, act, num_shared=0):
    """out_t = sum_e g_te * FFN_e(x_t) with every expert evaluated densely.

    The gate vector g is zero outside the brute-force top-k; FFN_e uses
    einsum over all experts at once (a different route through the math
    than the oracle's per-expert grouping).
    """
    ids, wts = _route_brute(logits, topk, renorm, num_shared)
    wts = wts.astype(np.float32).astype(np.float64)   # routing weights are stored as fp32
    T = x.shape[0]
    E = w13.shape[0]
    I = w2.shape[2]
    g = np.zeros((T, E))
    for t in range(T):
        for j in range(ids.shape[1]):
            g[t, ids[t, j]] += wts[t, j]
    z = np.einsum("th,enh->ten", x, w13)
    if act == "swiglu":
        a = z[:, :, :I] / (1.0 + np.exp(-z[:, :, :I])) * z[:, :, I:]
    elif act == "gelu_tanh":
        g0 = z[:, :, :I]
        a = 0.5 * g0 * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (g0 + 0.044715 * g0 ** 3))) * z[:, :, I:]
    elif act == "swigluoai":
        g0 = np.minimum(z[:, :, :I], 7.0)
        a = g0 * (1.0 / (1.0 + np.exp(-1.702 * g0))) * (np.clip(z[:, :, I:], -7.0, 7.0) + 1.0)
    else:
        a = np.maximum(z, 0.0) ** 2
    ffn = np.einsum("tei,ehi->teh", a, w2)
    return np.einsum("te,teh->th", g, ffn)


@pytest.mark.parametrize("act,renorm,shared", [("swiglu", True, 0), ("relu2", False, 0), ("swiglu", True, 1),
                                                ("gelu_tanh", True, 0), ("swigluoai", True, 0)])
def test_layer_dense_ffn_invariant(act, renorm, shared):
    rng = np.random.default_rng(11)
    T, H, E, k, I = 9, 64, 6, 3, 24
    N1 = 2 * I if act != "relu2" else I
    x = _bf16_bits(torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)))
    l = rng.standard_normal((T, E)).astype(np.float32)
    Et = E + shared
    w13 = _bf16_bits(torch.from_numpy(0.2 * rng.standard_normal((Et, N1, H)).astype(np.float32)))
    w2 = _bf16_bits(torch.from_numpy(0.2 * rng.standard_normal((Et, H, I)).astype(np.float32)))
    got = O.moe_forward(x, l, w13, w2, topk=k, renormalize=renorm, activation=act, num_shared=shared)
    want = _dense_layer(O.bf16_bits_to_f64(x), l, O.bf16_bits_to_f64(w13), O.bf16_bits_to_f64(w2),
                        k, renorm, act, shared)
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)


def test_layer_scalar_brute_force_tiny():
    # pure-Python scalar loops on a 2-token, 3-expert, H=4, I=2 layer
    rng = np.random.default_rng(2)
    T, H, E, k, I = 2, 4, 3, 2, 2
    x = _bf16_bits(torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)))
    l = rng.standard_normal((T, E)).astype(np.float32)
    w13 = _bf16_bits(torch.from_numpy(rng.standard_normal((E, 2 * I, H)).astype(np.float32)))
    w2 = _bf16_bits(torch.from_numpy(rng.standard_normal((E, H, I)).astype(np.float32)))
    X, W13, W2 = O.bf16_bits_to_f64(x), O.bf16_bits_to_f64(w13), O.bf16_bits_to_f64(w2)
    ids, wts = _route_brute(l, k, True)
    wts = wts.astype(np.float32).astype(np.float64)   # routing weights are stored as fp32
    want = [[0.0] * H for _ in range(T)]
    for t in range(T):
        for j in range(k):
            e = ids[t, j]
            a = []
            for n in range(I):
                g = sum(X[t, h] * W13[e, n, h] for h in range(H))
                u = sum(X[t, h] * W13[e, I + n, h] for h in range(H))
                a.append(g / (1.0 + math.exp(-g)) * u)
            for h in range(H):
                want[t][h] += wts[t, j] * sum(a[n] * W2[e, h, n] for n in range(I))
    got = O.moe_forward(x, l, w13, w2, topk=k, renormalize=True, activation="swiglu")
    np.testing.assert_allclose(got, np.array(want), rtol=1e-12, atol=1e-14)


def test_layer_subset_of_tokens_equals_full_rows():
    rng = np.random.default_rng(8)
    T, H, E, k, I = 12, 128, 5, 2, 16
    x = _bf16_bits(torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)))
    l = rng.standard_normal((T, E)).astype(np.float32)
    w13 = _bf16_bits(torch.from_numpy(0.1 * rng.standard_normal((E, 2 * I, H)).astype(np.float32)))
    w2 = _bf16_bits(torch.from_numpy(0.1 * rng.standard_normal((E, H, I)).astype(np.float32)))
    full = O.moe_forward(x, l, w13, w2, topk=k, renormalize=True, activation="swiglu")
    sub = O.moe_forward(x, l, w13, w2, topk=k, renormalize=True, activation="swiglu", tokens=[3, 0, 11])
    np.testing.assert_allclose(sub, full[[3, 0, 11]], rtol=1e-13, atol=0)


# --------------------------------------------------------------------------
# FP8 E4M3 codec and quantisers (library routine: torch.float8_e4m3fn casts)
# --------------------------------------------------------------------------


def test_e4m3_golden_points():
    for v, code in _rows("e4m3_points.txt"):
        x = np.array([float(v)], dtype=np.float32)
        assert int(O.e4m3_encode(x)[0]) == int(code, 16), v


def test_e4m3_encode_matches_torch_cast_on_all_bf16_values():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    x = O.bf16_bits_to_f32(bits)
    keep = np.isfinite(x) & (np.abs(x) <= 448.0)
    x = x[keep]
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(O.e4m3_encode(x), want)


def test_e4m3_encode_matches_torch_cast_on_random_and_midpoints():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(200000) * rng.choice([1e-3, 0.1, 1.0, 30.0, 200.0], 200000)).astype(np.float32)
    x = np.clip(x, -448, 448)
    # exact midpoints between neighbouring codes (ties-to-even cases)
    vals = O.e4m3_decode(np.arange(0, 0x7E, dtype=np.uint8))
    mids = ((vals[1:] + vals[:-1]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids])
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(O.e4m3_encode(x), want)


def test_e4m3_decode_roundtrip_and_monotone():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    v = O.e4m3_decode(codes)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(v, want)
    np.testing.assert_array_equal(O.e4m3_encode(v.astype(np.float32)), codes)
    pos = O.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    assert np.all(np.diff(pos) > 0) and pos[-1] == 448.0


def test_e4m3_saturates():
    x = np.array([449.0, 463.9, 464.0, 500.0, 1e30, -1e30], dtype=np.float32)
    assert O.e4m3_encode(x).tolist() == [0x7E] * 4 + [0x7E, 0xFE]


def test_quant_groups_definition():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((3, 256)).astype(np.float32)
    x[1, 128:] = 0.0                      # all-zero group -> scale 1, codes 0
    q, s = O.quant_groups_1x128(x)
    assert s.dtype == np.float32 and s.shape == (3, 2)
    assert s[1, 1] == 1.0 and np.all(q[1, 128:] == 0)
    for r in range(3):
        for g in range(2):
            blk = x[r, g * 128:(g + 1) * 128]
            amax = np.float32(np.abs(blk).max())
            if amax == 0:
                continue
            sc = np.float32(amax / np.float32(448.0))
            assert s[r, g] == sc
            want = torch.from_numpy((blk / sc).astype(np.float32)).to(torch.float8_e4m3fn)
            np.testing.assert_array_equal(q[r, g * 128:(g + 1) * 128], want.view(torch.uint8).numpy())
    # the group's largest magnitude maps to +-448 (code 0x7E / 0xFE)
    i = int(np.argmax(np.abs(x[0, :128])))
    assert (q[0, i] & 0x7F) == 0x7E
    # dequantisation error is within half an e4m3 step (relative 2^-4) per element
    d = O.dequant_groups_1x128(q, s)
    assert np.all(np.abs(d - x) <= np.abs(x) * 2.0 ** -4 + np.repeat(s, 128, 1) * 2.0 ** -10)


def test_quant_blocks_definition():
    rng = np.random.default_rng(6)
    w = (0.02 * rng.standard_normal((256, 384))).astype(np.float32)
    q, s = O.quant_blocks_128x128(w)
    assert s.shape == (2, 3)
    for bi in range(2):
        for bj in range(3):
            blk = w[bi * 128:(bi + 1) * 128, bj * 128:(bj + 1) * 128]
            sc = np.float32(np.float32(np.abs(blk).max()) / np.float32(448.0))
            assert s[bi, bj] == sc
            want = torch.from_numpy((blk / sc).astype(np.float32)).to(torch.float8_e4m3fn)
            np.testing.assert_array_equal(q[bi * 128:(bi + 1) * 128, bj * 128:(bj + 1) * 128],
                                          want.view(torch.uint8).numpy())


def test_fp8_layer_equals_bf16_layer_on_dequantised_inputs():
    # moe_forward_fp8 == dense invariant evaluated on the dequantised operands
    rng = np.random.default_rng(9)
    T, H, E, k, I = 5, 256, 3, 2, 128
    x = _bf16_bits(torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)))
    l = rng.standard_normal((T, E)).astype(np.float32)
    w13 = _bf16_bits(torch.from_numpy(0.02 * rng.standard_normal((E, 2 * I, H)).astype(np.float32)))
    w2 = _bf16_bits(torch.from_numpy(0.02 * rng.standard_normal((E, H, I)).astype(np.float32)))
    q13, s13, q2, s2 = O.quantize_weights_fp8(w13, w2)
    got = O.moe_forward_fp8(x, l, q13, s13, q2, s2, topk=k, renormalize=True, activation="swiglu")
    # independent restatement: dequantise with torch casts, dense evaluation
    X = O.bf16_bits_to_f32(x)
    xs = np.abs(X.reshape(T, 2, 128)).max(2) / np.float32(448)
    Xq = torch.from_numpy((X.reshape(T, 2, 128) / xs[:, :, None]).astype(np.float32)).to(torch.float8_e4m3fn)
    Xd = (Xq.to(torch.float64).numpy() * xs[:, :, None]).reshape(T, H)
    W13d = np.stack([np.kron(s13[e].astype(np.float64), np.ones((128, 128))) *
                     torch.from_numpy(q13[e]).view(torch.float8_e4m3fn).to(torch.float64).numpy() for e in range(E)])
    W2d = np.stack([np.kron(s2[e].astype(np.float64), np.ones((128, 128))) *
                    torch.from_numpy(q2[e]).view(torch.float8_e4m3fn).to(torch.float64).numpy() for e in range(E)])
    ids, wts = _route_brute(l, k, True)
    wts = wts.astype(np.float32).astype(np.float64)
    want = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            e = ids[t, j]
            z = W13d[e] @ Xd[t]
            # the activation is stored as bf16 before its 1x128 quantisation
            a = torch.from_numpy((z[:I] / (1 + np.exp(-z[:I])) * z[I:]).astype(np.float32)).to(
                torch.bfloat16).to(torch.float32).numpy()
            asc = np.float32(np.abs(a).max() / np.float32(448))
            aq = torch.from_numpy((a / asc).astype(np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()
            want[t] += wts[t, j] * (W2d[e] @ (aq * asc))
    np.testing.assert_allclose(got, want, rtol=1e-9, atol=1e-12)


def test_quant_per_tensor_matches_torch_cast():
    rng = np.random.default_rng(31)
    x = (rng.standard_normal(20000) * 3).astype(np.float32)
    scale = np.float32(np.abs(x).max() / 448)
    want = torch.from_numpy(x / scale).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(O.quant_per_tensor(x, scale), want)
    # beyond 448 saturates (the torch cast would give NaN there)
    assert O.quant_per_tensor(np.array([1000.0, -1000.0], np.float32), 1.0).tolist() == [0x7E, 0xFE]
    # the reciprocal form for GEMM inputs: the torch cast of x * fp32(1 / scale)
    inv = np.float32(1.0) / scale
    want_inv = torch.from_numpy((x * inv).astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(O.quant_per_tensor_inv(x, scale), want_inv)


@pytest.mark.parametrize("act", ["swiglu", "relu2", "gelu_tanh"])
def test_fp8_per_tensor_layer_against_torch_casts(act):
    # independent restatement with torch float8 casts and a dense per-token loop
    rng = np.random.default_rng(17)
    T, H, E, k, I = 6, 256, 3, 2, 128
    N1 = I if act == "relu2" else 2 * I
    x = _bf16_bits(torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)))
    l = rng.standard_normal((T, E)).astype(np.float32)
    w13 = _bf16_bits(torch.from_numpy(0.02 * rng.standard_normal((E, N1, H)).astype(np.float32)))
    w2 = _bf16_bits(torch.from_numpy(0.02 * rng.standard_normal((E, H, I)).astype(np.float32)))
    q13, s13, q2, s2 = O.quantize_weights_fp8_per_tensor(w13, w2)
    X = O.bf16_bits_to_f32(x)
    s_in = np.float32(np.abs(X).max() / 448)
    s_act = np.float32(0.05)
    got = O.moe_forward_fp8_per_tensor(x, l, q13, s13, q2, s2, s_in, s_act, topk=k, renormalize=True,
                                       activation=act)

    def f8(a, s):  # weights: quantise x / s with the torch cast, dequantise to float64
        q = torch.from_numpy(np.clip(a / s, -448, 448).astype(np.float32)).to(torch.float8_e4m3fn)
        return q.to(torch.float64).numpy() * np.float64(s)

    def f8i(a, s):  # GEMM inputs: x * fp32(1 / s)
        inv = np.float32(1.0) / np.float32(s)
        q = torch.from_numpy(np.clip(a.astype(np.float32) * inv, -448, 448).astype(np.float32)).to(
            torch.float8_e4m3fn)
        return q.to(torch.float64).numpy() * np.float64(s)

    W13 = [f8(O.bf16_bits_to_f32(w13[e]), s13[e]) for e in range(E)]
    W2 = [f8(O.bf16_bits_to_f32(w2[e]), s2[e]) for e in range(E)]
    Xd = f8i(X, s_in)
    ids, wts = _route_brute(l, k, True)
    want = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            e = ids[t, j]
            z = W13[e] @ Xd[t]
            if act == "relu2":
                a = np.maximum(z, 0) ** 2
            else:
                g, u = z[:I], z[I:]
                a = (g / (1 + np.exp(-g)) if act == "swiglu" else
                     0.5 * g * (1 + np.tanh(np.sqrt(2 / np.pi) * (g + 0.044715 * g ** 3)))) * u
            want[t] += np.float64(np.float32(wts[t, j])) * (W2[e] @ f8i(a.astype(np.float32), s_act))
    np.testing.assert_allclose(got, want, rtol=1e-9, atol=1e-12)
    # per-expert weight scales are amax / 448
    np.testing.assert_array_equal(s13, (np.abs(O.bf16_bits_to_f32(w13).reshape(E, -1)).max(1) / np.float32(448))
                                  .astype(np.float32))


# --------------------------------------------------------------------------
# MXFP8 (OCP MX v1.0 conversion, block 32, E8M0 scales)
# --------------------------------------------------------------------------


def test_quant_mx_golden_points():
    # hand-derived: all ones -> floor(log2 1) - 8 = -8 (byte 119), 1 * 2^8 = 256 -> 0x78
    q, s = O.quant_mx(np.ones(32, np.float32))
    assert s.tolist() == [119] and np.all(q == 0x78)
    # amax 3 -> s = 1 - 8 = -7 (byte 120); 3 * 128 = 384 = 1.5 * 2^8 -> 0x7C;
    # -0.375 * 128 = -48 = -1.5 * 2^5 -> sign | exponent field 12 | mantissa 4 = 0xE4
    x = np.zeros(32, np.float32)
    x[0], x[31] = 3.0, -0.375
    q, s = O.quant_mx(x)
    assert s.tolist() == [120] and q[0] == 0x7C and q[31] == 0xE4 and np.all(q[1:31] == 0)
    # 255/128 -> s = -8, scaled 510 saturates to 448 (0x7E)
    q, s = O.quant_mx(np.full(32, 255.0 / 128.0, np.float32))
    assert s.tolist() == [119] and np.all(q == 0x7E)
    # all-zero block: byte 0, codes 0
    q, s = O.quant_mx(np.zeros(32, np.float32))
    assert s.tolist() == [0] and np.all(q == 0)
    # exponent clamps: amax 2^-130 wants s = -138 -> -127 (byte 0), 2^-130 * 2^127 = 2^-3 -> 0x20;
    # amax 2^120 -> s = 112 (byte 239) -> 2^8 -> 0x78
    q, s = O.quant_mx(np.array([2.0 ** -130] + [0.0] * 31 + [2.0 ** 120] + [0.0] * 31, np.float32))
    assert s.tolist() == [0, 239] and q[0] == 0x20 and q[32] == 0x78


def test_quant_mx_against_math_frexp_and_torch_cast():
    rng = np.random.default_rng(41)
    x = (rng.standard_normal((6, 256)) * np.exp2(rng.integers(-12, 12, (6, 1)))).astype(np.float32)
    x[2, 64:96] = 0.0
    x[3, 5] = 1e30                               # one huge value dominates its block
    q, s = O.quant_mx(x)
    assert q.shape == x.shape and s.shape == (6, 8) and s.dtype == np.uint8
    for r in range(6):
        for b in range(8):
            blk = x[r, 32 * b:32 * b + 32].astype(np.float64)
            amax = float(np.abs(blk).max())
            e = (math.frexp(amax)[1] - 1 - 8) if amax > 0 else -127
            e = max(-127, min(127, e))
            assert int(s[r, b]) == e + 127
            scaled = torch.from_numpy(np.clip(blk * 2.0 ** -e, -448, 448).astype(np.float32))
            want = scaled.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            np.testing.assert_array_equal(q[r, 32 * b:32 * b + 32], want)
            if amax > 0:                          # the block maximum lands in [256, 512)
                assert 256.0 <= amax * 2.0 ** -e < 512.0
    # dequantisation: exact for E4M3 values times a power of two, else within half a step
    d = O.dequant_mx(q, s)
    step = np.repeat(np.ldexp(1.0, s.astype(np.int32) - 127), 32, 1)
    sat = np.abs(x) * np.repeat(np.ldexp(1.0, 127 - s.astype(np.int32)), 32, 1) > 448
    assert np.all(np.abs(d - x)[~sat] <= (np.abs(x) * 2.0 ** -4 + step * 2.0 ** -10)[~sat])
    # a block of E4M3 values whose largest is 448 keeps scale 2^0 (times any power of two)
    codes = np.concatenate([rng.integers(0, 0x7E, (3, 31)), np.full((3, 1), 0x7E)], 1).astype(np.uint8)
    codes[1] |= 0x80
    v = (O.e4m3_decode(codes) * np.ldexp(1.0, np.array([-5, 0, 7]))[:, None]).reshape(1, 96)
    q2, s2 = O.quant_mx(v.astype(np.float32))
    assert s2.tolist() == [[122, 127, 134]]
    np.testing.assert_array_equal(O.dequant_mx(q2, s2), v)


def test_mxfp8_padding_rule_from_page():
    # the page's rule: I rounded up to min_alignment (16 gated, 128 non-gated), codes and
    # scales zero-filled after the original values, unchanged when already aligned
    rng = np.random.default_rng(61)
    for gated, I, align, I_pad in ((True, 96, 128, 128), (False, 160, 128, 256), (True, 64, 16, 64)):
        E, H = 2, 64
        N1 = (2 if gated else 1) * I
        w13 = rng.integers(1, 255, (E, N1, H)).astype(np.uint8)
        s13 = rng.integers(100, 140, (E, N1, H // 32)).astype(np.uint8)
        w2 = rng.integers(1, 255, (E, H, I)).astype(np.uint8)
        s2 = rng.integers(100, 140, (E, H, I // 32)).astype(np.uint8)
        p13, ps13, p2, ps2, got = O.pad_weights_mxfp8(w13, s13, w2, s2, I, gated, align)
        assert got == I_pad
        if I_pad == I:
            assert p13 is w13 and ps2 is s2
            continue
        assert p13.shape == (E, (2 if gated else 1) * I_pad, H) and ps13.shape == (E, p13.shape[1], H // 32)
        assert p2.shape == (E, H, I_pad) and ps2.shape == (E, H, I_pad // 32)
        for h in range(2 if gated else 1):
            np.testing.assert_array_equal(p13[:, h * I_pad:h * I_pad + I], w13[:, h * I:(h + 1) * I])
            np.testing.assert_array_equal(ps13[:, h * I_pad:h * I_pad + I], s13[:, h * I:(h + 1) * I])
            assert np.all(p13[:, h * I_pad + I:(h + 1) * I_pad] == 0) and np.all(ps13[:, h * I_pad + I:(h + 1) * I_pad] == 0)
        np.testing.assert_array_equal(p2[:, :, :I], w2)
        np.testing.assert_array_equal(ps2[:, :, :I // 32], s2)
        assert np.all(p2[:, :, I:] == 0) and np.all(ps2[:, :, I // 32:] == 0)


def test_mxfp8_padding_leaves_layer_unchanged():
    rng = np.random.default_rng(67)
    for act, I in (("swiglu", 96), ("relu2", 160)):
        gated = act == "swiglu"
        T, H, E, k = 5, 128, 3, 2
        x = _bf16_bits(torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)))
        l = rng.standard_normal((T, E)).astype(np.float32)
        w13 = _bf16_bits(torch.from_numpy(0.05 * rng.standard_normal((E, (2 if gated else 1) * I, H)).astype(np.float32)))
        w2 = _bf16_bits(torch.from_numpy(0.05 * rng.standard_normal((E, H, I)).astype(np.float32)))
        q = O.quantize_weights_mxfp8(w13, w2)
        padded = O.pad_weights_mxfp8(*q, I, gated, 128)
        a = O.moe_forward_mxfp8(x, l, *q, topk=k, renormalize=True, activation=act)
        b = O.moe_forward_mxfp8(x, l, *padded[:4], topk=k, renormalize=True, activation=act)
        # the padded activation columns are exact zeros, and an all-zero 32-block quantises to zero
        np.testing.assert_allclose(b, a, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("act", ["swiglu", "relu2"])
def test_mxfp8_layer_against_torch_casts(act):
    # independent restatement: math.frexp exponents, torch float8 casts, a dense per-token loop
    rng = np.random.default_rng(43)
    T, H, E, k, I = 5, 128, 3, 2, 64
    N1 = I if act == "relu2" else 2 * I
    x = _bf16_bits(torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)))
    l = rng.standard_normal((T, E)).astype(np.float32)
    w13 = _bf16_bits(torch.from_numpy(0.02 * rng.standard_normal((E, N1, H)).astype(np.float32)))
    w2 = _bf16_bits(torch.from_numpy(0.02 * rng.standard_normal((E, H, I)).astype(np.float32)))
    q13, s13, q2, s2 = O.quantize_weights_mxfp8(w13, w2)
    got = O.moe_forward_mxfp8(x, l, q13, s13, q2, s2, topk=k, renormalize=True, activation=act)

    def mx(a):  # quantise + dequantise rows of a (float32) in blocks of 32
        a = np.asarray(a, np.float32)
        out = np.zeros(a.shape)
        for idx in np.ndindex(a.shape[:-1]):
            for b in range(a.shape[-1] // 32):
                blk = a[idx][32 * b:32 * b + 32].astype(np.float64)
                amax = float(np.abs(blk).max())
                e = max(-127, min(127, (math.frexp(amax)[1] - 9) if amax > 0 else -127))
                c = torch.from_numpy(np.clip(blk * 2.0 ** -e, -448, 448).astype(np.float32)).to(torch.float8_e4m3fn)
                out[idx][32 * b:32 * b + 32] = c.to(torch.float64).numpy() * 2.0 ** e
        return out

    W13 = [mx(O.bf16_bits_to_f32(w13[e])) for e in range(E)]
    W2 = [mx(O.bf16_bits_to_f32(w2[e])) for e in range(E)]
    Xd = mx(O.bf16_bits_to_f32(x))
    ids, wts = _route_brute(l, k, True)
    want = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            e = ids[t, j]
            z = W13[e] @ Xd[t]
            a = np.maximum(z, 0) ** 2 if act == "relu2" else z[:I] / (1 + np.exp(-z[:I])) * z[I:]
            a16 = torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16).to(torch.float32).numpy()
            want[t] += np.float64(np.float32(wts[t, j])) * (W2[e] @ mx(a16[None])[0])
    np.testing.assert_allclose(got, want, rtol=1e-9, atol=1e-12)
    # the MX layer stays near the bf16 layer (three E4M3 roundings of about 4% RMS each)
    ref = O.moe_forward(x, l, w13, w2, topk=k, renormalize=True, activation=act)
    assert O.rms(got - ref) < 0.15 * O.rms(ref)


# --------------------------------------------------------------------------
# NVFP4 (E2M1 values, E4M3 scale per 16, fp32 scale per tensor)
# --------------------------------------------------------------------------

# the E2M1 grid (sign bit 3, exponent bias 1, one mantissa bit): code -> value
E2M1_TABLE = {0: 0.0, 1: 0.5, 2: 1.0, 3: 1.5, 4: 2.0, 5: 3.0, 6: 4.0, 7: 6.0}


def _e2m1_brute(v: float) -> int:
    """Nearest grid magnitude by exhaustive search; on a tie the code with mantissa bit 0."""
    a = min(abs(v), 6.0)
    best = min(E2M1_TABLE, key=lambda c: (abs(a - E2M1_TABLE[c]), c & 1))
    return best | (8 if math.copysign(1.0, v) < 0 else 0)


def test_e2m1_decode_table_and_brute_force_encode():
    np.testing.assert_array_equal(O.e2m1_decode(np.arange(16, dtype=np.uint8)),
                                  [0, .5, 1, 1.5, 2, 3, 4, 6, -0.0, -.5, -1, -1.5, -2, -3, -4, -6])
    # every tie point, every grid point, values around them and beyond the range
    pts = sorted(set(E2M1_TABLE.values()))
    mids = [(a + b) / 2 for a, b in zip(pts, pts[1:])]
    vals = pts + mids + [m + d for m in mids for d in (-1e-3, 1e-3)] + [6.5, 7.0, 100.0, 1e-30]
    vals = np.array(vals + [-v for v in vals] + [-0.0], dtype=np.float32)
    rng = np.random.default_rng(47)
    vals = np.concatenate([vals, (rng.standard_normal(4000) * 3).astype(np.float32)])
    got = O.e2m1_encode(vals)
    want = np.array([_e2m1_brute(float(v)) for v in vals], dtype=np.uint8)
    np.testing.assert_array_equal(got, want)
    # hand-picked ties: 0.25 -> 0, 0.75 -> 1.0, 1.25 -> 1.0, 1.75 -> 2, 2.5 -> 2, 3.5 -> 4, 5 -> 4
    t = O.e2m1_encode(np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32))
    assert t.tolist() == [0, 2, 2, 4, 4, 6, 6]


def test_quant_nvfp4_definition():
    rng = np.random.default_rng(53)
    x = (rng.standard_normal((4, 64)) * np.exp2(rng.integers(-6, 6, (4, 1)))).astype(np.float32)
    x[1, 16:32] = 0.0
    g = O.nvfp4_global_scale(np.abs(x).max())
    assert g == np.float32(np.float32(np.abs(x).max()) / np.float32(2688.0))
    q, s = O.quant_nvfp4(x, g)
    assert q.shape == x.shape and s.shape == (4, 4)
    for r in range(4):
        for b in range(4):
            blk = x[r, 16 * b:16 * b + 16]
            amax = np.float32(np.abs(blk).max())
            sc = torch.tensor([float(np.float32(np.float32(amax / np.float32(6.0)) / g))]).to(torch.float8_e4m3fn)
            assert int(s[r, b]) == int(sc.view(torch.uint8).item())
            den = np.float32(np.float32(sc.to(torch.float32).item()) * g)
            want = [(_e2m1_brute(float(np.float32(v / den))) if den > 0 else 0) for v in blk]
            assert q[r, 16 * b:16 * b + 16].tolist() == want
    assert np.all(q[1, 16:32] == 0) and s[1, 1] == 0
    # dequantisation stays within half an E2M1 step of the scaled value plus the block-scale error
    d = O.dequant_nvfp4(q, s, g)
    assert np.all(np.abs(d - x) <= 0.25 * np.abs(x) + np.repeat(O.e4m3_decode(s), 16, 1) * g * 0.26 + 1e-30)
    # the tensor's largest value keeps its block at E2M1's top: code 6.0 (7) when 6 * s * g reaches it
    i = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    assert (q[i] & 7) in (6, 7)


@pytest.mark.parametrize("act", ["swiglu", "relu2"])
def test_nvfp4_layer_against_dense_restatement(act):
    rng = np.random.default_rng(59)
    T, H, E, k, I = 5, 128, 3, 2, 64
    N1 = I if act == "relu2" else 2 * I
    x = _bf16_bits(torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)))
    l = rng.standard_normal((T, E)).astype(np.float32)
    w13 = _bf16_bits(torch.from_numpy(0.02 * rng.standard_normal((E, N1, H)).astype(np.float32)))
    w2 = _bf16_bits(torch.from_numpy(0.02 * rng.standard_normal((E, H, I)).astype(np.float32)))
    q13, s13, g13, q2, s2, g2 = O.quantize_weights_nvfp4(w13, w2)
    g_in, g_act = np.float32(0.002), np.float32(0.0004)
    got = O.moe_forward_nvfp4(x, l, q13, s13, g13, q2, s2, g2, g_in, g_act, topk=k, renormalize=True,
                              activation=act)

    def fp4(a, g):  # per row, per 16: torch E4M3 block scale, brute-force E2M1 values
        a = np.asarray(a, np.float32)
        out = np.zeros(a.shape)
        for idx in np.ndindex(a.shape[:-1]):
            row = a[idx]
            for b in range(row.shape[0] // 16):
                blk = row[16 * b:16 * b + 16]
                sc = torch.tensor([float(np.float32(np.float32(np.abs(blk).max() / np.float32(6)) / g))]).to(
                    torch.float8_e4m3fn).to(torch.float32).item()
                den = np.float32(np.float32(sc) * g)
                for i, v in enumerate(blk):
                    c = _e2m1_brute(float(np.float32(v / den))) if den > 0 else 0
                    # the value is exact: code * block scale * global scale, in float64
                    out[idx][16 * b + i] = (-1 if c & 8 else 1) * E2M1_TABLE[c & 7] * sc * float(g)
        return out

    W13 = [fp4(O.bf16_bits_to_f32(w13[e]), g13[e]) for e in range(E)]
    W2 = [fp4(O.bf16_bits_to_f32(w2[e]), g2[e]) for e in range(E)]
    Xd = fp4(O.bf16_bits_to_f32(x), g_in)
    ids, wts = _route_brute(l, k, True)
    want = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            e = ids[t, j]
            z = W13[e] @ Xd[t]
            a = np.maximum(z, 0) ** 2 if act == "relu2" else z[:I] / (1 + np.exp(-z[:I])) * z[I:]
            a16 = torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16).to(torch.float32).numpy()
            want[t] += np.float64(np.float32(wts[t, j])) * (W2[e] @ fp4(a16[None], g_act)[0])
    np.testing.assert_allclose(got, want, rtol=1e-9, atol=1e-12)
    # per-expert global scales: amax / (6 * 448)
    np.testing.assert_array_equal(g13, (np.abs(O.bf16_bits_to_f32(w13).reshape(E, -1)).max(1) / np.float32(2688))
                                  .astype(np.float32))


# --------------------------------------------------------------------------
# planted mistakes: each mutated oracle must fail a pin above
# --------------------------------------------------------------------------


def _tiny_layer_inputs(act):
    rng = np.random.default_rng(21)
    T, H, E, k, I = 7, 32, 5, 2, 8
    N1 = 2 * I if act == "swiglu" else I
    x = _bf16_bits(torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)))
    l = rng.standard_normal((T, E)).astype(np.float32)
    w13 = _bf16_bits(torch.from_numpy(0.3 * rng.standard_normal((E, N1, H)).astype(np.float32)))
    w2 = _bf16_bits(torch.from_numpy(0.3 * rng.standard_normal((E, H, I)).astype(np.float32)))
    return x, l, w13, w2, k


@pytest.mark.parametrize("mutation", ["silu_sign", "swap_gate_up", "no_renorm", "tie_high_index",
                                      "transpose_w2_slice", "drop_last_slot"])
def test_planted_mistakes_are_caught(monkeypatch, mutation):
    act = "swiglu"
    x, l, w13, w2, k = _tiny_layer_inputs(act)
    want = _dense_layer(O.bf16_bits_to_f64(x), l, O.bf16_bits_to_f64(w13), O.bf16_bits_to_f64(w2),
                        k, True, act)
    real_route = O.route
    if mutation == "silu_sign":
        monkeypatch.setattr(O, "silu", lambda z: z / (1.0 + np.exp(z)))
    elif mutation == "swap_gate_up":
        monkeypatch.setattr(O, "activation_fn", lambda z, a, I: O.silu(z[:, I:2 * I]) * z[:, :I])
    elif mutation == "no_renorm":
        monkeypatch.setattr(O, "route", lambda lg, kk, r, s=0: real_route(lg, kk, False, s))
    elif mutation == "tie_high_index":
        l = l.copy()
        l[:, :3] = [1.0, 1.0, 2.0]   # experts 0 and 1 tie at the top-2 cut
        l[:, 3:] = -1.0
        want = _dense_layer(O.bf16_bits_to_f64(x), l, O.bf16_bits_to_f64(w13), O.bf16_bits_to_f64(w2),
                            k, True, act)

        def bad_route(lg, kk, r, s=0):
            E = lg.shape[1]
            ids, w = real_route(lg[:, ::-1].copy(), kk, r, s)
            return (E - 1 - ids).astype(np.int32), w
        monkeypatch.setattr(O, "route", bad_route)
    elif mutation == "transpose_w2_slice":
        w2 = w2.copy()
        w2_t = w2.copy()
        w2_t[:, :8, :] = np.swapaxes(w2[:, :8, :8], 1, 2)
        got = O.moe_forward(x, l, w13, w2_t, topk=k, renormalize=True, activation=act)
        assert np.max(np.abs(got - want)) > 1e-6
        return
    elif mutation == "drop_last_slot":
        monkeypatch.setattr(O, "route", lambda lg, kk, r, s=0: real_route(lg, max(kk - 1, 1), r, s))
    got = O.moe_forward(x, l, w13, w2, topk=k, renormalize=True, activation=act)
    assert np.max(np.abs(got - want)) > 1e-6, mutation


def test_half_ulp_bf16_helper():
    # the tolerance helper used by the parity tests: half the bf16 spacing at |x|
    import sys
    sys.path.insert(0, os.path.dirname(__file__))
    from _cases import half_ulp_bf16
    assert half_ulp_bf16(np.array([1.0]))[0] == 2.0 ** -8
    assert half_ulp_bf16(np.array([1.99]))[0] == 2.0 ** -8
    assert half_ulp_bf16(np.array([-2.0]))[0] == 2.0 ** -7
    assert half_ulp_bf16(np.array([0.75]))[0] == 2.0 ** -9
    x = np.random.default_rng(0).standard_normal(100000) * 10.0
    r = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.all(np.abs(r - x.astype(np.float32)) <= half_ulp_bf16(x) * (1 + 1e-7))


def test_round_to_bf16_matches_torch_cast():
    rng = np.random.default_rng(12)
    x = np.concatenate([rng.standard_normal(200000) * 10.0 ** rng.integers(-6, 6, 200000),
                        np.float64([0.0, -0.0, 1.0, 448.0, 3.0e38, -1e-30])])
    want = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(O.round_to_bf16(x), want)
    # exact ties: halfway between neighbouring bf16 values round to the even one
    a = np.float32([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8])
    assert O.round_to_bf16(a).tolist() == [1.0, 1.0 + 2 * 2.0 ** -7]
