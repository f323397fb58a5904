"""NVFP4 (E2M1 values, an E4M3 scale per 16 values of K, an fp32 scale per tensor) through the
C ABI against the CPU oracle: the weight and input quantisers bit for bit, the prepared
(tiled) weights and scale blocks bit for bit, the permuted quantised rows and GEMM2's input
(the kernel's own bf16 activation quantised) bit for bit, GEMM1's activation element by
element, and the layer output.

Tolerance: the oracle quantises the same bf16 values with the same decisions, so the layer
differs only by the fp32 accumulation order and by E2M1 codes of GEMM2's input that land on
the other side of a rounding boundary when the kernel's bf16 activation and the oracle's
differ by one ulp; both are far inside the FP8 bound (5e-2 * RMS beyond the output rounding),
which is applied here too.
"""
import numpy as np
import pytest
import torch

import mixture_experts_expert_topk_b200 as moe
from mixture_experts_expert_topk_b200.synth import CONFIGS, MoeConfig, make_inputs
from oracle import moe_oracle as O

from _cases import (bf16_act_bound, bf16_to_f64, bits, check_act_pairs, cover_tokens, dirty_workspace,
                    err_beyond_rounding, max_err_over_rms, per_expert_threaded, report, untile_groups,
                    untile_u8)

pytestmark = pytest.mark.gpu

TOL = 5e-2


def _small(name, **kw) -> MoeConfig:
    base = dict(T=64, H=256, E=8, topk=2, I=256, renormalize=True, activation="swiglu", fp8="nvfp4")
    base.update(kw)
    return MoeConfig(name, **base)


NV_SMALL = {
    "nv_swiglu": _small("nv_swiglu", T=300),
    "nv_relu2": _small("nv_relu2", T=200, H=512, E=6, topk=3, activation="relu2", renormalize=False),
    "nv_gelu_shared": _small("nv_gelu_shared", T=130, E=12, topk=3, num_shared=1, activation="gelu_tanh"),
    "nv_oai": _small("nv_oai", T=200, activation="swigluoai", weight_std=0.5),
    # groups of up to 128 rows and three align chunks
    "nv_big_groups": _small("nv_big_groups", T=1500, E=4),
    "nv_decode": _small("nv_decode", T=4, H=512, E=32, topk=4),
    # an odd number of 256-value chunks (the last K step holds one) and I = 512
    "nv_odd_chunks": _small("nv_odd_chunks", T=100, H=768, I=512),
}


def pack(codes: np.ndarray) -> np.ndarray:
    """One E2M1 code per byte -> two per byte, the lower K index in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def untile_w_bytes(flat: np.ndarray, E: int, rows: int, kbytes: int) -> np.ndarray:
    """[E, MT*128, KC*128] bytes from 128-row x 128-byte tiles at ((e*MT + m)*KC + c)*16384,
    row r's 16-byte piece q stored at q ^ (r % 8)."""
    MT, KC = -(-rows // 128), -(-kbytes // 128)
    t = np.asarray(flat)[:E * MT * KC * 16384].reshape(E, MT, KC, 128, 8, 16)
    r = np.arange(128)
    phys = np.arange(8)[None, :] ^ (r[:, None] & 7)
    u = t[:, :, :, r[:, None], phys, :]
    return u.transpose(0, 1, 3, 2, 4, 5).reshape(E, MT * 128, KC * 128)


def untile_w_scales(flat: np.ndarray, E: int, rows: int, K: int) -> np.ndarray:
    """[E, MT*128, KC*16] scale codes from 2048-byte blocks per tile: byte 512 mm + 16 l +
    4 j + k = row 32 j + l, block 16 c + 4 mm + k."""
    MT, KC = -(-rows // 128), -(-K // 256)
    t = np.asarray(flat).reshape(E, MT, KC, 4, 32, 4, 4)       # [e, m, c, mm, l, j, k]
    return t.transpose(0, 1, 5, 4, 2, 3, 6).reshape(E, MT * 128, KC * 16)


def group_scales(flat, group_info, num_groups, rows, KC) -> np.ndarray:
    """[rows, 16*KC] scale codes from the row groups' 2048-byte blocks at ((x_row / 16) * KC +
    c) * 2048: byte 512 mm + 16 (j % 32) + 4 (j / 32) + k = group row j, block 16 c + 4 mm + k."""
    flat = np.asarray(flat).reshape(-1)
    out = np.zeros((rows, 16 * KC), dtype=np.uint8)
    for g in range(num_groups):
        x_row, meta = int(group_info[g][0]), int(group_info[g][1])
        n = (meta >> 16) & 0x1FF
        j = np.arange(n)
        for c in range(KC):
            base = ((x_row // 16) * KC + c) * 2048
            for mm in range(4):
                for k in range(4):
                    out[x_row + j, 16 * c + 4 * mm + k] = flat[base + 512 * mm + 16 * (j % 32) + 4 * (j // 32) + k]
    return out


def deinterleave(rows_tiled: np.ndarray, I: int) -> np.ndarray:
    """Interleaved [gate0, up0, gate1, up1, ...] rows ([2I, cols]) -> gate rows then up rows."""
    return np.concatenate([rows_tiled[0:2 * I:2], rows_tiled[1:2 * I:2]], axis=0)


def _act_scale(cfg, inp, s_in) -> float:
    """The activation's tensor scale: the oracle's GEMM1 activation amax / (6 * 448) on these
    inputs (NVFP4 operands), times 1.25."""
    x = O.dequant_nvfp4(*O.quant_nvfp4(O.bf16_bits_to_f32(bits(inp["hidden"])), s_in), s_in)
    ids, _ = O.route(inp["logits"].numpy(), cfg.topk, cfg.renormalize, cfg.num_shared)
    w13 = bits(inp["w13"])
    amax = 0.0
    for e in np.unique(ids):
        t = np.nonzero((ids == e).any(axis=1))[0]
        W = O.bf16_bits_to_f64(w13[e])
        amax = max(amax, float(np.abs(O.activation_fn(x[t] @ W.T, cfg.activation, cfg.I)).max()))
    return float(np.float32(amax * 1.25 / 2688))


def _run(cfg, inp, s_act=None, experts=None, tokens=None):
    dev = torch.device("cuda:0")
    s_in = float(inp["hidden"].float().abs().max() / 2688)
    if s_act is None:
        s_act = _act_scale(cfg, inp, s_in)
    q13, sc13, g13 = moe.quantize_weights_nvfp4(inp["w13"].to(dev))
    q2, sc2, g2 = moe.quantize_weights_nvfp4(inp["w2"].to(dev))
    prob = moe.make_problem(cfg.T, cfg.H, cfg.E, cfg.topk, cfg.I, renormalize=cfg.renormalize,
                            activation=cfg.activation, num_shared=cfg.num_shared, fp8="nvfp4",
                            input_scale=s_in, activation_scale=s_act)
    w13p, w2p = moe.prepare_weights(prob, q13, q2, cfg.I, w13_scale=sc13, w2_scale=sc2)
    ws = dirty_workspace(prob)
    out = moe.moe_forward(inp["hidden"].to(dev), inp["logits"].to(dev), w13p, w2p, cfg.topk, cfg.renormalize,
                          cfg.activation, g13, g2, num_shared=cfg.num_shared, workspace=ws, input_scale=s_in,
                          activation_scale=s_act)
    torch.cuda.synchronize()
    assert moe.device_status(ws)[0] == 0
    raw = moe.read_workspace(prob, ws)
    act_bits = raw.pop("act").view(torch.int16).cpu().numpy().view(np.uint16)
    parts = {k: v.cpu().numpy() for k, v in raw.items()}
    return dict(out=out, parts=parts, act_bits=act_bits, s_in=s_in, s_act=s_act, q13=q13, sc13=sc13, g13=g13,
                q2=q2, sc2=sc2, g2=g2, w13p=w13p, w2p=w2p)


def _check(cfg, inp, r, oracle_w, tokens=None):
    """Everything the forward left in the workspace, then the layer on ``tokens`` (all if None)."""
    o13, os13, og13, o2, os2, og2 = oracle_w
    parts, s_in, s_act = r["parts"], r["s_in"], r["s_act"]
    kk = cfg.k_total
    P = cfg.T * kk
    ids, w = O.route(inp["logits"].numpy(), cfg.topk, cfg.renormalize, cfg.num_shared)
    np.testing.assert_array_equal(parts["topk_ids"], ids)
    al = O.align(ids, cfg.E_total, 16)
    P_pad = int(al["P_pad"])
    np.testing.assert_array_equal(parts["sorted_pair_ids"][:P_pad], al["sorted_pair_ids"])
    np.testing.assert_array_equal(parts["pair_to_row"], al["pair_to_row"])
    gi, ng = parts["group_info"], int(parts["num_blocks"][1])
    assert max((int(gi[g][1]) >> 16) & 0x1FF for g in range(ng)) <= 128
    # the hidden rows quantised once per token with the input scale, then permuted
    hq, hs = O.quant_nvfp4(O.bf16_bits_to_f32(bits(inp["hidden"])), s_in)
    np.testing.assert_array_equal(parts["xq"], pack(hq))
    np.testing.assert_array_equal(parts["xq_scale"], hs)
    pids = al["sorted_pair_ids"][:P_pad]
    real = pids < P
    KC1 = cfg.H // 256
    xs = untile_u8(parts["xs"], gi, ng, P_pad, KC1)
    np.testing.assert_array_equal(xs[real], pack(hq)[pids[real] // kk])
    xss = group_scales(parts["xs_scale"], gi, ng, P_pad, KC1)
    np.testing.assert_array_equal(xss[real], hs[pids[real] // kk])
    # GEMM2's input: the kernel's own bf16 activation quantised with the activation scale
    act = untile_groups(r["act_bits"], gi, ng, P_pad, -(-cfg.I // 64))[:, :cfg.I]
    aq, asc = O.quant_nvfp4(O.bf16_bits_to_f32(act[real]), s_act)
    KC2 = cfg.I // 256
    np.testing.assert_array_equal(untile_u8(parts["actq"], gi, ng, P_pad, KC2)[real], pack(aq))
    np.testing.assert_array_equal(group_scales(parts["act_scale"], gi, ng, P_pad, KC2)[real], asc)
    # GEMM1's bf16 activation against the oracle's on the same NVFP4 operands
    x = O.dequant_nvfp4(hq, hs, s_in)
    toks = np.arange(cfg.T) if tokens is None else tokens
    n_act = check_act_pairs(
        lambda e, t: O.activation_fn(x[t] @ O.dequant_nvfp4(o13[e], os13[e], og13[e]).T, cfg.activation, cfg.I),
        bf16_to_f64(act), ids, toks, al["pair_to_row"], bf16_act_bound)
    # the layer
    ref = O.moe_forward_nvfp4(bits(inp["hidden"]), inp["logits"].numpy(), o13, os13, og13, o2, os2, og2, s_in,
                              np.float32(s_act), topk=cfg.topk, renormalize=cfg.renormalize,
                              activation=cfg.activation, num_shared=cfg.num_shared, tokens=tokens)
    got = bf16_to_f64(r["out"].cpu()[torch.from_numpy(toks)])
    assert np.all(np.isfinite(got))
    e = err_beyond_rounding(got, ref)
    report(f"{cfg.name}: {len(toks)} tokens, {n_act} activation values; beyond-rounding {e:.4f}, "
          f"raw {max_err_over_rms(got, ref):.4f}")
    assert e <= TOL, e


@pytest.mark.parametrize("name", list(NV_SMALL))
def test_nvfp4_layer_parity(name):
    cfg = NV_SMALL[name]
    inp = make_inputs(cfg, 0)
    r = _run(cfg, inp)
    # the device quantiser, bit for bit against the oracle's
    ow = O.quantize_weights_nvfp4(bits(inp["w13"]), bits(inp["w2"]))
    o13, os13, og13, o2, os2, og2 = ow
    np.testing.assert_array_equal(r["q13"].cpu().numpy(), pack(o13))
    np.testing.assert_array_equal(r["sc13"].cpu().numpy(), os13)
    np.testing.assert_array_equal(r["g13"].cpu().numpy(), og13)
    np.testing.assert_array_equal(r["q2"].cpu().numpy(), pack(o2))
    np.testing.assert_array_equal(r["sc2"].cpu().numpy(), os2)
    np.testing.assert_array_equal(r["g2"].cpu().numpy(), og2)
    # the prepared weights: codes tiled (gated rows interleaved), then the scale blocks
    E, N1 = cfg.E_total, cfg.N1
    n13 = E * (-(-N1 // 128)) * (cfg.H // 256) * 16384
    n2 = E * (cfg.H // 128) * (cfg.I // 256) * 16384
    w13p, w2p = r["w13p"].cpu().numpy(), r["w2p"].cpu().numpy()
    t13 = untile_w_bytes(w13p[:n13], E, N1, cfg.H // 2)[:, :N1, :cfg.H // 2]
    s13 = untile_w_scales(w13p[n13:], E, N1, cfg.H)[:, :N1, :cfg.H // 16]
    if cfg.gated:
        t13 = np.stack([deinterleave(t13[e], cfg.I) for e in range(E)])
        s13 = np.stack([deinterleave(s13[e], cfg.I) for e in range(E)])
    np.testing.assert_array_equal(t13, pack(o13))
    np.testing.assert_array_equal(s13, os13)
    np.testing.assert_array_equal(untile_w_bytes(w2p[:n2], E, cfg.H, cfg.I // 2)[:, :, :cfg.I // 2], pack(o2))
    np.testing.assert_array_equal(untile_w_scales(w2p[n2:], E, cfg.H, cfg.I)[:, :, :cfg.I // 16], os2)
    _check(cfg, inp, r, ow)


def test_nvfp4_full_size_every_expert():
    """The NVFP4 prefill workload at full size (T=4096, 256 experts, top-8): all of the
    workspace checks over every token and the layer on a token sample that covers every
    routed expert."""
    cfg = CONFIGS["nvfp4_prefill"]
    inp = make_inputs(cfg, 0)
    r = _run(cfg, inp, s_act=cfg.activation_scale)
    ids, _ = O.route(inp["logits"].numpy(), cfg.topk, cfg.renormalize)
    tokens = cover_tokens(ids, cfg.E, extra=16)
    experts = np.unique(ids[tokens])
    assert len(experts) == len(np.unique(ids))
    E = cfg.E_total
    w13b, w2b = bits(inp["w13"]), bits(inp["w2"])
    o13 = np.zeros(w13b.shape, np.uint8)
    os13 = np.zeros(w13b.shape[:2] + (cfg.H // 16,), np.uint8)
    o2 = np.zeros(w2b.shape, np.uint8)
    os2 = np.zeros(w2b.shape[:2] + (cfg.I // 16,), np.uint8)
    og13, og2 = np.ones(E, np.float32), np.ones(E, np.float32)

    def one(e):
        return O.quantize_weights_nvfp4(w13b[e:e + 1], w2b[e:e + 1])

    for e, (a13, b13, c13, a2, b2, c2) in per_expert_threaded(one, experts).items():
        o13[e], os13[e], og13[e], o2[e], os2[e], og2[e] = a13[0], b13[0], c13[0], a2[0], b2[0], c2[0]
    ow = (o13, os13, og13, o2, os2, og2)
    np.testing.assert_array_equal(r["g13"].cpu().numpy()[experts], og13[experts])
    _check(cfg, inp, r, ow, tokens=tokens)
