"""CPU oracle for the fused Mixture-of-Experts layer forward.

TEST INFRASTRUCTURE. This module is a plain, slow, obviously-correct NumPy
restatement of what the layer computes, in float64. It exists only to check
the CUDA library. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import it; the library and
its Python binding never do, and it imports nothing from them.

The layer (one forward call) computes, for every token t with hidden row x_t:

  1. route:   pick the top-k experts of the router logits, softmax weights,
              optional renormalisation, optional fused shared-expert slot;
  2. align:   stable sort of the (token, slot) pairs by expert, each expert's
              segment padded to the GEMM row tile ``block_m``;
  3. GEMM1:   z = W13[e] x_t, then a gated activation act(gate)*up (SwiGLU: silu;
              gelu_tanh), swigluoai(gate, up), or relu2 max(z,0)^2;
  4. GEMM2:   y = w_tj * (W2[e] a);
  5. combine: out_t = sum_j y_tj in slot order j = 0..k'-1.

Citations name the source pages by title and section:
  [TRTLLM]  "FlashInfer TRTLLM-Gen MoE kernel optimisation: NemotronH support"
            (sglang PR 21321)
  [GATED]   "FlashInfer gated MoE kernel optimisation for Blackwell"
            (flashinfer PR 4329)
  [SHARED]  "Qwen3-Next FP8 MoE optimisation: shared-expert fusion for H200"
            (sglang PR 26204)
  [SWIGLU]  "[MoE] SwiGLU fusion into the MoE up-GEMM epilogue"
            (sglang PR 32944)
  [W4A8]    "W4A8 grouped GEMM optimisation for GLM-5.2 MoE on H200"
            (sglang PR 38220)

Where the pages leave a step open, the reading taken is stated at the
function. Every function here is pinned by tests in ``tests/`` against
brute force, closed forms or library routines (none is "parity unpinned").
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Sequence

import numpy as np

E4M3_MAX = 448.0

# --------------------------------------------------------------------------
# Number formats
# --------------------------------------------------------------------------


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Decode bf16 bit patterns (uint16) to float64 exactly.

    A bf16 value is the upper 16 bits of an IEEE binary32 value.
    """
    b = np.ascontiguousarray(bits).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(bits).astype(np.uint32) << 16
    return b.view(np.float32)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round to bf16 (8 significant bits, round to nearest even) via float32.

    The value is first rounded to float32 (the precision the activation is computed
    in) and then to bf16, returned as float32. Finite inputs only.
    """
    b = np.ascontiguousarray(np.asarray(x, dtype=np.float32)).view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    r = ((b + 0x7FFF + lsb) >> 16) << 16
    return r.astype(np.uint32).view(np.float32)


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Encode float32 values as FP8 E4M3 (the OCP "fn" variant) codes.

    Format: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; no
    infinities; the largest finite magnitude is 448 (exponent field 15,
    mantissa 6); exponent field 0 holds subnormals m * 2^-9.
    Rounding is to nearest, ties to even; magnitudes beyond 448 saturate to
    448 ("satfinite"). Inputs must be finite. The sign of zero is kept.
    Used for the FP8 W8A8 128x128 block-scale configuration of [SHARED],
    section 1 (dtype=fp8_w8a8, block_shape=[128, 128]).
    """
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x).astype(np.float64)
    sign = (np.signbit(x)).astype(np.uint8) << 7
    # quantum (spacing of representable values) at the magnitude of a
    _, ex = np.frexp(a)                     # a = m * 2^ex, m in [0.5, 1)
    e_unb = ex.astype(np.int64) - 1         # a in [2^e_unb, 2^(e_unb+1))
    e_unb = np.maximum(e_unb, -6)           # below 2^-6: subnormal spacing 2^-9
    quantum = np.ldexp(1.0, (e_unb - 3).astype(np.int32))
    r = np.rint(a / quantum) * quantum      # exact in float64; rint is ties-to-even
    r = np.minimum(r, E4M3_MAX)
    # r -> bits
    codes = np.zeros(x.shape, dtype=np.uint8)
    nz = r > 0
    _, ex2 = np.frexp(r)
    e2 = ex2.astype(np.int64) - 1
    normal = nz & (e2 >= -6)
    sub = nz & (e2 < -6)
    mant_n = np.where(normal, r / np.ldexp(1.0, e2.astype(np.int32)) - 1.0, 0.0) * 8.0
    exp_field = np.where(normal, e2 + 7, 0)
    codes = np.where(normal, (exp_field.astype(np.uint8) << 3) | mant_n.astype(np.uint8), codes)
    codes = np.where(sub, (r / 2.0 ** -9).astype(np.uint8), codes)
    return (codes | sign).astype(np.uint8)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Decode FP8 E4M3 codes to float64 (code 0x7F/0xFF, NaN, never occurs here)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.ldexp(1.0, (e - 7).astype(np.int32)))
    return s * val


def quant_groups_1x128(x: np.ndarray):
    """Dynamic per-row, per-128-column quantisation to E4M3.

    For each row and each group of 128 consecutive columns:
    scale = amax / 448 (IEEE fp32 division), q = e4m3(x / scale) with the
    fp32 division rounded to nearest. An all-zero group takes scale 1 (the
    pages do not say; with scale 1 every code is 0 and dequantisation is
    exact). Both the division and the encoding run in fp32, the precision the
    kernel uses, so the codes are a bit-exact reference.
    Returns (codes uint8 [R, C], scales float32 [R, C/128]).
    """
    x = np.asarray(x, dtype=np.float32)
    R, C = x.shape
    assert C % 128 == 0
    g = x.reshape(R, C // 128, 128)
    amax = np.abs(g).max(axis=2)
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    scale = np.where(amax == 0, np.float32(1.0), scale).astype(np.float32)
    q = e4m3_encode((g / scale[:, :, None]).astype(np.float32))
    return q.reshape(R, C), scale


def quant_blocks_128x128(w: np.ndarray):
    """Static per-128x128-block quantisation of a weight matrix to E4M3.

    ``w`` is [R, C] (fp32 values of the bf16 masters), R and C multiples of
    128. scale = amax(block) / 448 in fp32, q = e4m3(w / scale); an all-zero
    block takes scale 1. Returns (codes uint8 [R, C], scales float32
    [R/128, C/128]).
    """
    w = np.asarray(w, dtype=np.float32)
    R, C = w.shape
    assert R % 128 == 0 and C % 128 == 0
    b = w.reshape(R // 128, 128, C // 128, 128)
    amax = np.abs(b).max(axis=(1, 3))
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    scale = np.where(amax == 0, np.float32(1.0), scale).astype(np.float32)
    q = e4m3_encode((b / scale[:, None, :, None]).astype(np.float32))
    return q.reshape(R, C), scale


def dequant_groups_1x128(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    return e4m3_decode(codes) * np.repeat(scales.astype(np.float64), 128, axis=1)


def dequant_blocks_128x128(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    s = np.repeat(np.repeat(scales.astype(np.float64), 128, axis=0), 128, axis=1)
    return e4m3_decode(codes) * s


# --------------------------------------------------------------------------
# Step 1: routing
# --------------------------------------------------------------------------


def route(logits: np.ndarray, topk: int, renormalize: bool, num_shared: int = 0):
    """Top-k expert selection with softmax routing weights.

    [TRTLLM] section 1 gives the fused op's arguments ``topk: int`` and
    ``renormalize: bool`` but not the formula. Reading taken (the plainest
    one consistent with an optional renormalisation and no bias or expert
    grouping on the page):
      * the k experts with the largest raw fp32 logits are selected, ordered
        by logit descending, ties broken towards the lower expert index;
      * p_e = softmax over all routed experts, in float64;
      * w_j = p_{id_j}, or p_{id_j} / sum_j' p_{id_j'} when renormalize.
    [SHARED] section 2 fuses a shared expert as an extra expert slot that
    every token selects: with ``num_shared`` = 1 the slot id is E (the
    routed expert count) with weight exactly 1, placed after the k routed
    slots and never renormalised.
    Returns ids int32 [T, k + num_shared] and weights float32 (same shape).
    """
    logits = np.asarray(logits, dtype=np.float32)
    T, E = logits.shape
    kk = topk + num_shared
    ids = np.empty((T, kk), dtype=np.int32)
    w = np.empty((T, kk), dtype=np.float32)
    if T == 0:
        return ids, w
    # a stable sort of the negated logits keeps equal logits in index order
    order = np.argsort(-logits, axis=1, kind="stable")[:, :topk]
    l64 = logits.astype(np.float64)
    m = l64.max(axis=1, keepdims=True)
    ex = np.exp(l64 - m)
    p = ex / ex.sum(axis=1, keepdims=True)
    sel = np.take_along_axis(p, order, axis=1)
    if renormalize:
        sel = sel / sel.sum(axis=1, keepdims=True)
    ids[:, :topk] = order
    w[:, :topk] = sel
    if num_shared:
        ids[:, topk:] = E
        w[:, topk:] = 1.0
    return ids, w


# --------------------------------------------------------------------------
# Step 2: align / permute
# --------------------------------------------------------------------------


def align(ids: np.ndarray, num_experts: int, block_m: int) -> Dict[str, np.ndarray]:
    """Sort (token, slot) pairs by expert and pad each expert to ``block_m``.

    Pair p = t * k' + j. The grouped GEMM contract of [W4A8] section 1
    (``expert_offsets``, ``problem_sizes``) gives each expert a contiguous
    row range. Reading taken: the expert's segment lists its pairs in
    ascending pair order (stable), followed by the sentinel P (= number of
    pairs) up to the next multiple of ``block_m``; an expert with no pairs
    gets no rows.
      expert_offsets[e+1] = expert_offsets[e] + round_up(count_e, block_m)
      block_expert[b]     = expert owning rows [b*block_m, (b+1)*block_m)
      pair_to_row[p]      = row of pair p in the sorted order
    """
    flat = np.asarray(ids, dtype=np.int64).reshape(-1)
    P = flat.size
    counts = np.bincount(flat, minlength=num_experts)[:num_experts]
    padded = (counts + block_m - 1) // block_m * block_m
    offsets = np.zeros(num_experts + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(padded)
    P_pad = int(offsets[-1])
    sorted_pair_ids = np.full(P_pad, P, dtype=np.int32)
    pair_to_row = np.empty(P, dtype=np.int32)
    block_expert = np.empty(P_pad // block_m, dtype=np.int32)
    for e in range(num_experts):
        pairs = np.nonzero(flat == e)[0]
        rows = offsets[e] + np.arange(pairs.size)
        sorted_pair_ids[rows] = pairs
        pair_to_row[pairs] = rows
        block_expert[offsets[e] // block_m: offsets[e + 1] // block_m] = e
    return {
        "sorted_pair_ids": sorted_pair_ids,
        "expert_offsets": offsets.astype(np.int32),
        "block_expert": block_expert,
        "pair_to_row": pair_to_row,
        "P_pad": np.int64(P_pad),
    }


# --------------------------------------------------------------------------
# Load-time weight preparation
# --------------------------------------------------------------------------


def padded_intermediate(I: int, gated: bool) -> int:
    """Intermediate size after alignment padding.

    [TRTLLM] section 2 (``_align_fp8_moe_weights`` and its caller): the
    intermediate size is rounded up to a multiple of 16 for gated
    activations and 128 for non-gated ones, and left unchanged when it is
    already aligned.
    """
    a = 16 if gated else 128
    return (I + a - 1) // a * a


def pad_weights(w13: np.ndarray, w2: np.ndarray, I: int, gated: bool):
    """Zero-pad w13 [E, up_mult*I, H] and w2 [E, H, I] to the padded I.

    [TRTLLM] section 2: the gate/up block becomes up_mult * I_pad rows (up_mult
    2 gated, 1 non-gated) with the original rows copied to the front and
    zeros after, and w2's last axis is zero-padded to I_pad. Note that the
    page copies the whole original w13 block to the front, so for a gated
    layer the up rows move only if I changes; this oracle keeps gate rows
    [0, I) and up rows [I_pad, I_pad + I) so that the padded matrix still
    reads as [Gate, Up] with the zero rows at the end of each half.
    """
    I_pad = padded_intermediate(I, gated)
    E, R, H = w13.shape
    if I_pad == I:
        return w13, w2, I
    if gated:
        out13 = np.zeros((E, 2 * I_pad, H), dtype=w13.dtype)
        out13[:, :I] = w13[:, :I]
        out13[:, I_pad:I_pad + I] = w13[:, I:2 * I]
    else:
        out13 = np.zeros((E, I_pad, H), dtype=w13.dtype)
        out13[:, :I] = w13
    out2 = np.zeros((E, w2.shape[1], I_pad), dtype=w2.dtype)
    out2[:, :, :I] = w2
    return out13, out2, I_pad


def interleave_gate_up(w13: np.ndarray, I: int) -> np.ndarray:
    """Row-interleave gate and up: [gate0, up0, gate1, up1, ...].

    [SWIGLU] section 3 (load-time interleave) so that the gate and up rows of
    one intermediate index sit in the same GEMM tile; [TRTLLM] section 2
    applies the same idea (``reorder_rows_for_gated_act_gemm``) to gated
    layers only.
    """
    E, R, H = w13.shape
    assert R == 2 * I
    out = np.empty_like(w13)
    out[:, 0::2] = w13[:, :I]
    out[:, 1::2] = w13[:, I:]
    return out


# --------------------------------------------------------------------------
# Step 3-5: expert FFNs and combine
# --------------------------------------------------------------------------


def silu(x: np.ndarray) -> np.ndarray:
    """silu(x) = x / (1 + e^-x), the gate activation of SwiGLU ([SWIGLU] section 1)."""
    with np.errstate(over="ignore"):
        return x / (1.0 + np.exp(-x))


def relu2(x: np.ndarray) -> np.ndarray:
    """relu2(x) = max(x, 0)^2, the non-gated activation of [TRTLLM] section 1."""
    r = np.maximum(x, 0.0)
    return r * r


def gelu_tanh(x: np.ndarray) -> np.ndarray:
    """GELU with the tanh approximation, one of the gated activations of [GATED]
    section 2 (named there as the Gaussian error linear unit with the tanh
    approximation; the pages print no formula, so the standard one is taken):
    0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))."""
    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x * x * x)))


SWIGLUOAI_ALPHA = 1.702   # sigmoid slope of the gpt-oss SwiGLU
SWIGLUOAI_LIMIT = 7.0     # its clamp on the gate (from above) and on the up value


def swigluoai(gate: np.ndarray, up: np.ndarray) -> np.ndarray:
    """``swigluoai_uninterleave``, a SwiGLU variant among the gated activations of [GATED]
    section 2, which reuses the standard formula without printing it. Reading taken: the
    SwiGLU published with OpenAI's gpt-oss models, on gate and up halves that are not
    interleaved (the gate-first checkpoint layout of SwiGLU here):
      g = min(gate, 7),  u = clamp(up, -7, 7),  a = g * sigmoid(1.702 g) * (u + 1)."""
    g = np.minimum(gate, SWIGLUOAI_LIMIT)
    u = np.clip(up, -SWIGLUOAI_LIMIT, SWIGLUOAI_LIMIT)
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-SWIGLUOAI_ALPHA * g)) * (u + 1.0)


GATED_ACTIVATIONS = ("swiglu", "gelu_tanh", "swigluoai")


def is_gated(activation: str) -> bool:
    return activation in GATED_ACTIVATIONS


def activation_fn(z: np.ndarray, activation: str, I: int) -> np.ndarray:
    """Apply the layer activation to GEMM1 rows z [n, N1] (gate-first layout).

    Gated: a = act(z[:, :I]) * z[:, I:2I] with act = silu for SwiGLU ([SWIGLU]
    section 1, ``silu(gate) * up``) or gelu_tanh ([GATED] section 2; [GATED]
    section 1: activation(gate) * up); swigluoai(z[:, :I], z[:, I:2I]) ([GATED]
    section 2).
    relu2: a = relu2(z) over the I columns.
    """
    if activation == "swigluoai":
        return swigluoai(z[:, :I], z[:, I:2 * I])
    if is_gated(activation):
        act = silu if activation == "swiglu" else gelu_tanh
        return act(z[:, :I]) * z[:, I:2 * I]
    if activation == "relu2":
        return relu2(z[:, :I])
    raise ValueError(activation)


def append_shared_slot(ids: np.ndarray, w: np.ndarray, num_routed: int, num_shared: int):
    """Caller-supplied routing ([TRTLLM] section 1 names a routed variant of the fused
    op, ``trtllm_fp8_block_scale_routed_moe``, that takes the top-k choice instead of
    router logits): routed ids [T, k] and weights [T, k] as given, then, with
    num_shared = 1, the fused shared slot after them (id E_r, weight 1, the same rule
    as ``route``)."""
    ids = np.asarray(ids, dtype=np.int32)
    w = np.asarray(w, dtype=np.float32)
    if num_shared:
        T = ids.shape[0]
        ids = np.concatenate([ids, np.full((T, 1), num_routed, dtype=np.int32)], axis=1)
        w = np.concatenate([w, np.ones((T, 1), dtype=np.float32)], axis=1)
    return ids, w


def moe_forward(hidden_bits: np.ndarray, logits: Optional[np.ndarray], w13_bits, w2_bits, *,
                topk: int, renormalize: bool, activation: str, num_shared: int = 0,
                tokens: Optional[Sequence[int]] = None, return_parts: bool = False,
                routing=None):
    """bf16 layer forward in float64.

    ``hidden_bits`` uint16 [T, H] (bf16), ``logits`` float32 [T, E_r],
    ``w13_bits`` uint16 [E, N1, H] and ``w2_bits`` uint16 [E, H, I] in the
    checkpoint layout (gate rows first). No intermediate rounding: GEMM
    products and sums are float64, the activation is applied to the exact
    GEMM1 result, the routing weight multiplies the exact GEMM2 result and
    the k' slot contributions are summed in slot order j = 0..k'-1.
    ``tokens`` restricts the computation to a subset of tokens (routing is
    per token, so the subset's outputs equal the full call's rows).
    ``routing`` = (ids [T, k'], weights [T, k']) replaces step 1 (the routed
    variant, see ``append_shared_slot``); ``logits`` is then unused.
    Returns out float64 [len(tokens) or T, H].
    """
    if routing is not None:
        ids, w = (np.asarray(routing[0], dtype=np.int32), np.asarray(routing[1], dtype=np.float32))
        if tokens is not None:
            tokens = np.asarray(tokens, dtype=np.int64)
            hidden_bits = np.asarray(hidden_bits)[tokens]
            ids, w = ids[tokens], w[tokens]
    else:
        logits = np.asarray(logits, dtype=np.float32)
        if tokens is not None:
            tokens = np.asarray(tokens, dtype=np.int64)
            hidden_bits = np.asarray(hidden_bits)[tokens]
            logits = logits[tokens]
        ids, w = route(logits, topk, renormalize, num_shared)
    x = bf16_bits_to_f64(hidden_bits)
    T, kk = ids.shape
    H = x.shape[1]
    I = w2_bits.shape[2]
    y = np.zeros((T, kk, H), dtype=np.float64)
    for e in np.unique(ids):
        t_idx, j_idx = np.nonzero(ids == e)
        W13 = bf16_bits_to_f64(np.asarray(w13_bits[e]))
        W2 = bf16_bits_to_f64(np.asarray(w2_bits[e]))
        z = x[t_idx] @ W13.T
        a = activation_fn(z, activation, I)
        y[t_idx, j_idx] = w[t_idx, j_idx].astype(np.float64)[:, None] * (a @ W2.T)
    out = np.zeros((T, H), dtype=np.float64)
    for j in range(kk):
        out += y[:, j]
    if return_parts:
        return out, {"ids": ids, "w": w}
    return out


def moe_forward_fp8(hidden_bits: np.ndarray, logits: Optional[np.ndarray], w13_q, w13_s, w2_q, w2_s, *,
                    topk: int, renormalize: bool, activation: str, num_shared: int = 0,
                    tokens: Optional[Sequence[int]] = None, routing=None):
    """FP8 E4M3 W8A8 layer forward with 128x128 weight blocks, in float64.

    [SHARED] section 1 names the configuration (fp8_w8a8, block_shape
    [128, 128]); [TRTLLM] section 1 the fused op that takes per-block weight
    scales. Reading taken (the pages print no formula):
      * weights: e4m3 codes with one fp32 scale per 128x128 block of the
        checkpoint-layout matrices w13 [E, N1, H] and w2 [E, H, I];
      * activations: the bf16 hidden rows are quantised per token per 128
        columns (``quant_groups_1x128``) before GEMM1, and the GEMM1
        activation output is quantised the same way before GEMM2 (W8A8 means
        both GEMM inputs are 8-bit). The activation is first stored in the
        compute dtype, bf16 ([SWIGLU] section 1: the fused epilogue casts
        silu(gate)*up ``.to(compute_type)`` before the store), so its 1x128
        codes are decided on the bf16 value;
      * every product uses the exactly dequantised values q * s in float64.
    ``w13_q``/``w2_q`` are uint8 codes, ``w13_s`` [E, N1/128, H/128] and
    ``w2_s`` [E, H/128, I/128] float32 scales. ``routing`` as in ``moe_forward``.
    """
    if routing is not None:
        ids, w = (np.asarray(routing[0], dtype=np.int32), np.asarray(routing[1], dtype=np.float32))
        if tokens is not None:
            tokens = np.asarray(tokens, dtype=np.int64)
            hidden_bits = np.asarray(hidden_bits)[tokens]
            ids, w = ids[tokens], w[tokens]
    else:
        logits = np.asarray(logits, dtype=np.float32)
        if tokens is not None:
            tokens = np.asarray(tokens, dtype=np.int64)
            hidden_bits = np.asarray(hidden_bits)[tokens]
            logits = logits[tokens]
        ids, w = route(logits, topk, renormalize, num_shared)
    xq, xs = quant_groups_1x128(bf16_bits_to_f32(hidden_bits))
    x = dequant_groups_1x128(xq, xs)
    T, kk = ids.shape
    H = x.shape[1]
    I = w2_q.shape[2]
    y = np.zeros((T, kk, H), dtype=np.float64)
    for e in np.unique(ids):
        t_idx, j_idx = np.nonzero(ids == e)
        W13 = dequant_blocks_128x128(np.asarray(w13_q[e]), np.asarray(w13_s[e]))
        W2 = dequant_blocks_128x128(np.asarray(w2_q[e]), np.asarray(w2_s[e]))
        a = activation_fn(x[t_idx] @ W13.T, activation, I)
        aq, as_ = quant_groups_1x128(round_to_bf16(a))
        ad = dequant_groups_1x128(aq, as_)
        y[t_idx, j_idx] = w[t_idx, j_idx].astype(np.float64)[:, None] * (ad @ W2.T)
    out = np.zeros((T, H), dtype=np.float64)
    for j in range(kk):
        out += y[:, j]
    return out


def quant_per_tensor(x: np.ndarray, scale) -> np.ndarray:
    """Static per-tensor quantisation to E4M3: q = e4m3(x / scale), the division in
    fp32 rounded to nearest, saturating at 448. The per-tensor FP8 variant of the
    fused op (``trtllm_fp8_per_tensor_scale_moe``, [TRTLLM] sections 1 and 2) takes
    one fp32 scale per tensor: per expert for the weights, one static input scale and
    one static activation scale for the two GEMM inputs."""
    x = np.asarray(x, dtype=np.float32)
    return e4m3_encode((x / np.float32(scale)).astype(np.float32))


def quant_per_tensor_inv(x: np.ndarray, scale) -> np.ndarray:
    """Static per-tensor quantisation of a GEMM input as the per-tensor variant writes it:
    [TRTLLM] section 2 scales by the reciprocal, ``* (1.0 / activation_scale)``, so
    q = e4m3(x * inv) with inv = fp32(1 / scale) and the product rounded to fp32,
    saturating at 448. Used for the hidden rows (input_scale) and for GEMM1's activation
    (activation_scale)."""
    x = np.asarray(x, dtype=np.float32)
    inv = np.float32(1.0) / np.float32(scale)
    return e4m3_encode((x * inv).astype(np.float32))


def quantize_weights_fp8_per_tensor(w13_bits, w2_bits):
    """Per-expert E4M3 weights for the per-tensor variant: scale = amax / 448 of the
    expert's matrix in fp32 (1 for an all-zero matrix), codes = quant_per_tensor.
    Returns (w13 codes, w13 scales [E], w2 codes, w2 scales [E])."""
    out = []
    for wb in (w13_bits, w2_bits):
        w = bf16_bits_to_f32(np.asarray(wb))
        amax = np.abs(w.reshape(w.shape[0], -1)).max(axis=1)
        sc = (amax / np.float32(E4M3_MAX)).astype(np.float32)
        sc = np.where(amax == 0, np.float32(1.0), sc).astype(np.float32)
        q = np.stack([quant_per_tensor(w[e], sc[e]) for e in range(w.shape[0])])
        out += [q, sc]
    return tuple(out)


def moe_forward_fp8_per_tensor(hidden_bits: np.ndarray, logits: Optional[np.ndarray], w13_q, w13_s, w2_q, w2_s,
                               input_scale, activation_scale, *, topk: int, renormalize: bool, activation: str,
                               num_shared: int = 0, tokens: Optional[Sequence[int]] = None, routing=None):
    """Per-tensor FP8 layer forward in float64.

    [TRTLLM] section 2 gives the scale algebra of the per-tensor variant: the GEMM1
    output is dequantised by g1_alphas = w13_scale * input_scale and, after the
    activation, requantised for GEMM2 by 1 / activation_scale; for a gated layer the
    two fold into g1_scale_c = g1_alphas / activation_scale, for relu2 (no gate
    dequantisation term) into 1 / activation_scale. Reading taken (the kernel itself is
    not printed): the activation acts on the dequantised GEMM1 output, and
      * x_q = quant_per_tensor_inv(hidden, input_scale);
      * z = (x_q * input_scale) (W13_q[e] * w13_scale[e])^T, a = activation(z);
      * a_q = quant_per_tensor_inv(a, activation_scale) (decided in fp32 on a);
      * y = w_tj * (a_q * activation_scale) (W2_q[e] * w2_scale[e])^T;
    ``w13_s``/``w2_s`` are float32 [E]; the two static scales are float32 scalars.
    ``routing`` as in ``moe_forward``.
    """
    if routing is not None:
        ids, w = (np.asarray(routing[0], dtype=np.int32), np.asarray(routing[1], dtype=np.float32))
        if tokens is not None:
            tokens = np.asarray(tokens, dtype=np.int64)
            hidden_bits = np.asarray(hidden_bits)[tokens]
            ids, w = ids[tokens], w[tokens]
    else:
        logits = np.asarray(logits, dtype=np.float32)
        if tokens is not None:
            tokens = np.asarray(tokens, dtype=np.int64)
            hidden_bits = np.asarray(hidden_bits)[tokens]
            logits = logits[tokens]
        ids, w = route(logits, topk, renormalize, num_shared)
    s_in, s_act = np.float32(input_scale), np.float32(activation_scale)
    x = e4m3_decode(quant_per_tensor_inv(bf16_bits_to_f32(hidden_bits), s_in)) * np.float64(s_in)
    T, kk = ids.shape
    H = x.shape[1]
    I = w2_q.shape[2]
    y = np.zeros((T, kk, H), dtype=np.float64)
    for e in np.unique(ids):
        t_idx, j_idx = np.nonzero(ids == e)
        W13 = e4m3_decode(np.asarray(w13_q[e])) * np.float64(w13_s[e])
        W2 = e4m3_decode(np.asarray(w2_q[e])) * np.float64(w2_s[e])
        a = activation_fn(x[t_idx] @ W13.T, activation, I)
        ad = e4m3_decode(quant_per_tensor_inv(a, s_act)) * np.float64(s_act)
        y[t_idx, j_idx] = w[t_idx, j_idx].astype(np.float64)[:, None] * (ad @ W2.T)
    out = np.zeros((T, H), dtype=np.float64)
    for j in range(kk):
        out += y[:, j]
    return out


def quantize_weights_fp8(w13_bits, w2_bits, experts=None):
    """Quantise bf16 master weights per 128x128 block (``quant_blocks_128x128``).

    Returns (w13_q, w13_s, w2_q, w2_s) in the checkpoint layout. ``experts`` limits the
    work to the listed experts (the others are left zero), for evaluating a few tokens
    of a large layer.
    """
    E = w13_bits.shape[0]
    w13_q = np.zeros(w13_bits.shape, dtype=np.uint8)
    w2_q = np.zeros(w2_bits.shape, dtype=np.uint8)
    w13_s = np.zeros((E, w13_bits.shape[1] // 128, w13_bits.shape[2] // 128), dtype=np.float32)
    w2_s = np.zeros((E, w2_bits.shape[1] // 128, w2_bits.shape[2] // 128), dtype=np.float32)
    for e in (range(E) if experts is None else experts):
        w13_q[e], w13_s[e] = quant_blocks_128x128(bf16_bits_to_f32(np.asarray(w13_bits[e])))
        w2_q[e], w2_s[e] = quant_blocks_128x128(bf16_bits_to_f32(np.asarray(w2_bits[e])))
    return w13_q, w13_s, w2_q, w2_s


# --------------------------------------------------------------------------
# MXFP8: E4M3 values sharing one power-of-two scale per block of 32
# --------------------------------------------------------------------------

MX_BLOCK = 32        # values per scale ([TRTLLM] section 2, ``_align_mxfp8_moe_weights``)
E4M3_EMAX = 8        # exponent of the largest power of two E4M3 holds (2^8 = 256 <= 448)


def quant_mx(x: np.ndarray):
    """MXFP8 quantisation along the last axis (the GEMM's reduction dimension).

    [TRTLLM] section 2 (``_align_mxfp8_moe_weights``) fixes the block: one scale per 32
    consecutive values of K (the scale tensors' last dimension is K / 32) and pads the
    scales with the weights. The pages print no conversion rule; reading taken: the OCP
    Microscaling Formats (MX) v1.0 conversion for MXFP8 E4M3, i.e. per block
      shared exponent  s = floor(log2(amax)) - 8  (8 = E4M3's largest exponent),
                       clamped to [-127, 127]; an all-zero block takes -127;
      scale            2^s, stored as the E8M0 byte s + 127;
      elements         e4m3(x * 2^-s), round to nearest even, saturating at 448.
    The product x * 2^-s is exact (a power-of-two scaling of an fp32 value), so the codes
    are decided exactly; the block's largest value lands in [256, 512).
    Returns (codes uint8 [..., K], scale bytes uint8 [..., K / 32]).
    """
    x = np.asarray(x, dtype=np.float32)
    K = x.shape[-1]
    assert K % MX_BLOCK == 0
    b = x.reshape(x.shape[:-1] + (K // MX_BLOCK, MX_BLOCK)).astype(np.float64)
    amax = np.abs(b).max(axis=-1)
    _, ex = np.frexp(amax)                                  # amax = m * 2^ex, m in [0.5, 1)
    s = np.where(amax > 0, ex.astype(np.int64) - 1 - E4M3_EMAX, -127)
    s = np.clip(s, -127, 127)
    scaled = (b * np.ldexp(1.0, (-s)[..., None].astype(np.int32))).astype(np.float32)
    codes = e4m3_encode(scaled).reshape(x.shape)
    return codes, (s + 127).astype(np.uint8)


def dequant_mx(codes: np.ndarray, scale_bytes: np.ndarray) -> np.ndarray:
    """codes * 2^(byte - 127) per block of 32 along the last axis, in float64."""
    s = np.repeat(scale_bytes.astype(np.int64) - 127, MX_BLOCK, axis=-1)
    return e4m3_decode(codes) * np.ldexp(1.0, s.astype(np.int32))


def quantize_weights_mxfp8(w13_bits, w2_bits, experts=None):
    """MXFP8 weights (``quant_mx`` along each matrix's K: H for w13, I for w2).

    Returns (w13 codes [E, N1, H], w13 scale bytes [E, N1, H/32], w2 codes [E, H, I],
    w2 scale bytes [E, H, I/32]) in the checkpoint layout. ``experts`` limits the work to
    the listed experts (the others stay zero).
    """
    out = []
    for wb in (w13_bits, w2_bits):
        wb = np.asarray(wb)
        E, R, C = wb.shape
        q = np.zeros((E, R, C), dtype=np.uint8)
        sc = np.zeros((E, R, C // MX_BLOCK), dtype=np.uint8)
        for e in (range(E) if experts is None else experts):
            q[e], sc[e] = quant_mx(bf16_bits_to_f32(wb[e]))
        out += [q, sc]
    return tuple(out)


def pad_weights_mxfp8(w13_q, w13_sc, w2_q, w2_sc, I: int, gated: bool, min_alignment: int):
    """Zero-pad MXFP8 weights and their scales to I_pad = round_up(I, min_alignment).

    [TRTLLM] section 2, ``_align_mxfp8_moe_weights``: the codes are padded like the FP8
    weights (w13 to up_mult * I_pad rows, w2's last axis to I_pad, zeros after the
    original values), and the scales with them: w13's scales gain the new rows, w2's scales
    (one per 32 values of I) grow to I_pad / 32 columns, all zero. As in ``pad_weights``,
    a gated w13 keeps gate rows [0, I) and up rows [I_pad, I_pad + I), each half padded on
    its own. Zero codes make the padded rows and columns contribute exact zeros whatever
    their (zero-byte) scales. Returns (w13_q, w13_sc, w2_q, w2_sc, I_pad); the inputs
    themselves when I is already aligned.
    """
    I_pad = (I + min_alignment - 1) // min_alignment * min_alignment
    if I_pad == I:
        return w13_q, w13_sc, w2_q, w2_sc, I
    assert I_pad % MX_BLOCK == 0 and I % MX_BLOCK == 0
    E = w13_q.shape[0]
    halves = 2 if gated else 1
    out13 = np.zeros((E, halves * I_pad, w13_q.shape[2]), dtype=w13_q.dtype)
    out13s = np.zeros((E, halves * I_pad, w13_sc.shape[2]), dtype=w13_sc.dtype)
    for h in range(halves):
        out13[:, h * I_pad:h * I_pad + I] = w13_q[:, h * I:(h + 1) * I]
        out13s[:, h * I_pad:h * I_pad + I] = w13_sc[:, h * I:(h + 1) * I]
    out2 = np.zeros((E, w2_q.shape[1], I_pad), dtype=w2_q.dtype)
    out2[:, :, :I] = w2_q
    out2s = np.zeros((E, w2_sc.shape[1], I_pad // MX_BLOCK), dtype=w2_sc.dtype)
    out2s[:, :, :I // MX_BLOCK] = w2_sc
    return out13, out13s, out2, out2s, I_pad


def moe_forward_mxfp8(hidden_bits: np.ndarray, logits: Optional[np.ndarray], w13_q, w13_sc, w2_q, w2_sc, *,
                      topk: int, renormalize: bool, activation: str, num_shared: int = 0,
                      tokens: Optional[Sequence[int]] = None, routing=None):
    """MXFP8 W8A8 layer forward in float64.

    [TRTLLM] section 2 adds MXFP8 MoE weights with per-32 scales beside the FP8 ones.
    Reading taken for what the pages leave open: both GEMM inputs are MXFP8 (the
    block-scaled MMA takes one scale per 32 values of K on each operand), so
      * the bf16 hidden rows are quantised per token (``quant_mx``) before GEMM1;
      * GEMM1's activation is stored in bf16 (as in the bf16 and 128x128 FP8 paths) and
        quantised per pair row the same way before GEMM2;
      * every product uses the exactly dequantised values in float64.
    ``w13_q``/``w2_q`` uint8 codes, ``w13_sc`` [E, N1, H/32] and ``w2_sc`` [E, H, I/32]
    uint8 E8M0 scale bytes. ``routing`` as in ``moe_forward``.
    """
    if routing is not None:
        ids, w = (np.asarray(routing[0], dtype=np.int32), np.asarray(routing[1], dtype=np.float32))
        if tokens is not None:
            tokens = np.asarray(tokens, dtype=np.int64)
            hidden_bits = np.asarray(hidden_bits)[tokens]
            ids, w = ids[tokens], w[tokens]
    else:
        logits = np.asarray(logits, dtype=np.float32)
        if tokens is not None:
            tokens = np.asarray(tokens, dtype=np.int64)
            hidden_bits = np.asarray(hidden_bits)[tokens]
            logits = logits[tokens]
        ids, w = route(logits, topk, renormalize, num_shared)
    x = dequant_mx(*quant_mx(bf16_bits_to_f32(hidden_bits)))
    T, kk = ids.shape
    H = x.shape[1]
    I = w2_q.shape[2]
    y = np.zeros((T, kk, H), dtype=np.float64)
    for e in np.unique(ids):
        t_idx, j_idx = np.nonzero(ids == e)
        W13 = dequant_mx(np.asarray(w13_q[e]), np.asarray(w13_sc[e]))
        W2 = dequant_mx(np.asarray(w2_q[e]), np.asarray(w2_sc[e]))
        a = activation_fn(x[t_idx] @ W13.T, activation, I)
        ad = dequant_mx(*quant_mx(round_to_bf16(a)))
        y[t_idx, j_idx] = w[t_idx, j_idx].astype(np.float64)[:, None] * (ad @ W2.T)
    out = np.zeros((T, H), dtype=np.float64)
    for j in range(kk):
        out += y[:, j]
    return out


# --------------------------------------------------------------------------
# NVFP4: E2M1 values, an E4M3 scale per 16, an fp32 scale per tensor
# --------------------------------------------------------------------------

NVFP4_BLOCK = 16
E2M1_MAX = 6.0


def e2m1_encode(x: np.ndarray) -> np.ndarray:
    """Encode float32 values as FP4 E2M1 codes (uint8 0..15).

    Format: 1 sign bit (bit 3), 2 exponent bits with bias 1, 1 mantissa bit; magnitudes
    0, 0.5 (exponent field 0: subnormal), 1, 1.5, 2, 3, 4, 6. Round to nearest, ties to the
    even code (the one whose mantissa bit is 0); magnitudes beyond 6 saturate to 6. The sign
    of zero is kept. Finite inputs only.
    """
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x).astype(np.float64)
    _, ex = np.frexp(a)
    e = np.maximum(ex.astype(np.int64) - 1, 0)        # exponent of a, subnormal range below 1
    quantum = np.ldexp(1.0, (e - 1).astype(np.int32))  # spacing: 0.5 below 2, then 1, then 2
    r = np.minimum(np.rint(a / quantum) * quantum, E2M1_MAX)
    # r -> code: 0 -> 0, 0.5 -> 1, then 2 codes per power of two
    _, ex2 = np.frexp(r)
    e2 = ex2.astype(np.int64) - 1
    code = np.where(r == 0, 0, np.where(r == 0.5, 1, 2 * (e2 + 1) + (r / np.ldexp(1.0, e2.astype(np.int32)) > 1)))
    return (code.astype(np.uint8) | (np.signbit(x).astype(np.uint8) << 3)).astype(np.uint8)


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    mag = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])[c & 7]
    return np.where(c & 8, -mag, mag)


def nvfp4_global_scale(amax) -> np.float32:
    """Per-tensor decode scale: amax / (6 * 448), so that every block scale fits E4M3; 1 for
    an all-zero tensor. fp32."""
    amax = np.float32(amax)
    return np.float32(1.0) if amax == 0 else np.float32(amax / np.float32(E2M1_MAX * E4M3_MAX))


def quant_nvfp4(x: np.ndarray, global_scale):
    """NVFP4 quantisation along the last axis with the tensor's fp32 decode scale g.

    The pages name NVFP4 weights ("FlashInfer gated MoE kernel optimisation for
    Blackwell", section 4; the NVFP4 results of [TRTLLM]) without printing the format.
    Reading taken: NVIDIA's published NVFP4 — E2M1 values, one E4M3 scale per 16 consecutive
    values of K and one fp32 scale per tensor — with, per block, in fp32:
      block scale  s = e4m3(amax / 6 / g)            (round to nearest even, saturating);
      elements     q = e2m1(x / (decode(s) * g))     (0 when the block scale decodes to 0);
      value        decode(q) * decode(s) * g.
    Returns (codes uint8 [..., K] holding one E2M1 code each, scale codes uint8 [..., K/16]).
    """
    x = np.asarray(x, dtype=np.float32)
    K = x.shape[-1]
    assert K % NVFP4_BLOCK == 0
    g = np.float32(global_scale)
    b = x.reshape(x.shape[:-1] + (K // NVFP4_BLOCK, NVFP4_BLOCK))
    amax = np.abs(b).max(axis=-1).astype(np.float32)
    s_code = e4m3_encode((amax / np.float32(E2M1_MAX) / g).astype(np.float32))
    denom = (e4m3_decode(s_code).astype(np.float32) * g).astype(np.float32)
    safe = np.where(denom > 0, denom, np.float32(1.0)).astype(np.float32)
    scaled = np.where(denom[..., None] > 0, (b / safe[..., None]).astype(np.float32), np.float32(0.0))
    codes = e2m1_encode(scaled.astype(np.float32)).reshape(x.shape)
    return codes, s_code


def dequant_nvfp4(codes: np.ndarray, scale_codes: np.ndarray, global_scale) -> np.ndarray:
    s = np.repeat(e4m3_decode(scale_codes), NVFP4_BLOCK, axis=-1)
    return e2m1_decode(codes) * s * np.float64(np.float32(global_scale))


def quantize_weights_nvfp4(w13_bits, w2_bits, experts=None):
    """NVFP4 weights: per expert matrix a global scale from its amax, then ``quant_nvfp4``
    along K. Returns (w13 codes, w13 block scales, w13 global scales [E], the same for w2)."""
    out = []
    for wb in (w13_bits, w2_bits):
        wb = np.asarray(wb)
        E, R, C = wb.shape
        q = np.zeros((E, R, C), dtype=np.uint8)
        sc = np.zeros((E, R, C // NVFP4_BLOCK), dtype=np.uint8)
        gs = np.ones(E, dtype=np.float32)
        for e in (range(E) if experts is None else experts):
            w = bf16_bits_to_f32(wb[e])
            gs[e] = nvfp4_global_scale(np.abs(w).max())
            q[e], sc[e] = quant_nvfp4(w, gs[e])
        out += [q, sc, gs]
    return tuple(out)


def moe_forward_nvfp4(hidden_bits: np.ndarray, logits: Optional[np.ndarray], w13_q, w13_sc, w13_g, w2_q, w2_sc,
                      w2_g, input_scale, activation_scale, *, topk: int, renormalize: bool, activation: str,
                      num_shared: int = 0, tokens: Optional[Sequence[int]] = None, routing=None):
    """NVFP4 W4A4 layer forward in float64.

    Reading taken (see ``quant_nvfp4``): the weights carry their own global scales; the two
    GEMM inputs are quantised with the static per-tensor global scales ``input_scale`` (the
    hidden rows) and ``activation_scale`` (GEMM1's activation, stored in bf16 first), the
    static input / activation scales of the per-tensor algebra of [TRTLLM] section 2, and
    dynamic E4M3 block scales per 16. Products use the exactly dequantised values.
    """
    if routing is not None:
        ids, w = (np.asarray(routing[0], dtype=np.int32), np.asarray(routing[1], dtype=np.float32))
        if tokens is not None:
            tokens = np.asarray(tokens, dtype=np.int64)
            hidden_bits = np.asarray(hidden_bits)[tokens]
            ids, w = ids[tokens], w[tokens]
    else:
        logits = np.asarray(logits, dtype=np.float32)
        if tokens is not None:
            tokens = np.asarray(tokens, dtype=np.int64)
            hidden_bits = np.asarray(hidden_bits)[tokens]
            logits = logits[tokens]
        ids, w = route(logits, topk, renormalize, num_shared)
    x = dequant_nvfp4(*quant_nvfp4(bf16_bits_to_f32(hidden_bits), input_scale), input_scale)
    T, kk = ids.shape
    H = x.shape[1]
    I = w2_q.shape[2]
    y = np.zeros((T, kk, H), dtype=np.float64)
    for e in np.unique(ids):
        t_idx, j_idx = np.nonzero(ids == e)
        W13 = dequant_nvfp4(np.asarray(w13_q[e]), np.asarray(w13_sc[e]), w13_g[e])
        W2 = dequant_nvfp4(np.asarray(w2_q[e]), np.asarray(w2_sc[e]), w2_g[e])
        a = activation_fn(x[t_idx] @ W13.T, activation, I)
        ad = dequant_nvfp4(*quant_nvfp4(round_to_bf16(a), activation_scale), activation_scale)
        y[t_idx, j_idx] = w[t_idx, j_idx].astype(np.float64)[:, None] * (ad @ W2.T)
    out = np.zeros((T, H), dtype=np.float64)
    for j in range(kk):
        out += y[:, j]
    return out


def rms(x: np.ndarray) -> float:
    x = np.asarray(x, dtype=np.float64)
    return math.sqrt(float(np.mean(x * x))) if x.size else 0.0
