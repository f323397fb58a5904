"""Shared helpers for the GPU parity tests: build a case, run the CUDA path through the
Python binding (C ABI), and evaluate the CPU oracle on the same seeded inputs."""
from __future__ import annotations

import functools
from typing import Dict, Optional

import numpy as np
import torch

import mixture_experts_expert_topk_b200 as moe
from mixture_experts_expert_topk_b200.synth import CONFIGS, MoeConfig, make_inputs
from oracle import moe_oracle as O


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 bit patterns (numpy, CPU)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


@functools.lru_cache(maxsize=4)
def cpu_inputs(cfg: MoeConfig, seed: int = 0) -> Dict[str, torch.Tensor]:
    return make_inputs(cfg, seed)


# Parity figures reported by the GPU tests (one line per configuration), printed again in the
# session's terminal summary (conftest.py) so that a quiet run still shows them.
PARITY_REPORT: list = []


def report(line: str) -> None:
    """Print a parity figure and keep it for the session summary."""
    print(line)
    PARITY_REPORT.append(line)


def dirty_workspace(prob) -> torch.Tensor:
    """A workspace whose every byte is 0xFF (NaN as bf16, fp16, fp32, e4m3 and E8M0): the
    forward must read nothing it has not written (X padding rows are never written)."""
    ws = moe.new_workspace(prob)
    ws.fill_(0xFF)
    return ws


class GpuForward:
    """One forward of ``cfg`` on cuda:0 with every intermediate kept in the workspace."""

    def __init__(self, cfg: MoeConfig, seed: int = 0, inputs: Optional[dict] = None, pdl: bool = True,
                 block_m: int = 0):
        self.cfg = cfg
        inp = inputs if inputs is not None else cpu_inputs(cfg, seed)
        self.inp = inp
        self.I_pad = moe.padded_intermediate(cfg.I, cfg.activation, cfg.fp8)
        self.prob = moe.make_problem(cfg.T, cfg.H, cfg.E, cfg.topk, self.I_pad,
                                     renormalize=cfg.renormalize, activation=cfg.activation,
                                     num_shared=cfg.num_shared, fp8=cfg.fp8, pdl=pdl, block_m=block_m)
        dev = torch.device("cuda:0")
        self.hidden = inp["hidden"].to(dev)
        self.logits = inp["logits"].to(dev)
        w13 = inp["w13"].to(dev)
        w2 = inp["w2"].to(dev)
        self.w13_scale = self.w2_scale = None
        if cfg.fp8:
            self.w13_q, self.w13_scale = moe.quantize_weights_fp8(w13)
            self.w2_q, self.w2_scale = moe.quantize_weights_fp8(w2)
            self.w13p, self.w2p = moe.prepare_weights(self.prob, self.w13_q, self.w2_q, cfg.I)
        else:
            self.w13p, self.w2p = moe.prepare_weights(self.prob, w13, w2, cfg.I)
        del w13, w2
        self.ws = dirty_workspace(self.prob)
        self.out = torch.empty_like(self.hidden)

    def forward(self) -> torch.Tensor:
        # through the C ABI with this run's problem (block_m included)
        import ctypes
        L = moe.lib()
        st = L.moe_forward(ctypes.byref(self.prob), ctypes.c_void_p(self.hidden.data_ptr()),
                           ctypes.c_void_p(self.logits.data_ptr()), ctypes.c_void_p(self.w13p.data_ptr()),
                           ctypes.c_void_p(self.w2p.data_ptr()),
                           None if self.w13_scale is None else ctypes.c_void_p(self.w13_scale.data_ptr()),
                           None if self.w2_scale is None else ctypes.c_void_p(self.w2_scale.data_ptr()),
                           ctypes.c_void_p(self.out.data_ptr()), ctypes.c_void_p(self.ws.data_ptr()),
                           self.ws.numel(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        moe.check(st, "moe_forward")
        torch.cuda.synchronize()
        return self.out

    def parts(self) -> Dict[str, np.ndarray]:
        v = moe.read_workspace(self.prob, self.ws)
        out = {"block_m": moe.workspace_layout(self.prob)["block_m"], "hidden_bits": bits(self.inp["hidden"])}
        for k, t in v.items():
            if t.dtype == torch.bfloat16:
                out[k] = bits(t)
            else:
                out[k] = t.cpu().numpy()
        return out


def oracle_out(cfg: MoeConfig, inp, tokens=None, fp8_weights=None) -> np.ndarray:
    if cfg.fp8:
        q13, s13, q2, s2 = fp8_weights
        return O.moe_forward_fp8(bits(inp["hidden"]), inp["logits"].numpy(), q13, s13, q2, s2,
                                 topk=cfg.topk, renormalize=cfg.renormalize,
                                 activation=cfg.activation, num_shared=cfg.num_shared,
                                 tokens=tokens)
    # the oracle takes the checkpoint (unpadded, gate-first) weights
    w13, w2 = bits(inp["w13"]), bits(inp["w2"])
    return O.moe_forward(bits(inp["hidden"]), inp["logits"].numpy(), w13, w2, topk=cfg.topk,
                         renormalize=cfg.renormalize, activation=cfg.activation,
                         num_shared=cfg.num_shared, tokens=tokens)


def bf16_to_f64(t_or_bits) -> np.ndarray:
    b = bits(t_or_bits) if isinstance(t_or_bits, torch.Tensor) else t_or_bits
    return O.bf16_bits_to_f64(b)


def max_err_over_rms(got: np.ndarray, ref: np.ndarray) -> float:
    """max|got - ref| / RMS(ref) (the raw figure, reported for information)."""
    r = O.rms(ref)
    return float(np.max(np.abs(got - ref)) / r) if r > 0 else float(np.max(np.abs(got - ref)))


def half_ulp_bf16(x: np.ndarray) -> np.ndarray:
    """Half the bf16 spacing at |x| (8 significant bits): 2^(floor(log2|x|) - 8)."""
    a = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -126)
    return np.ldexp(1.0, (np.floor(np.log2(a)) - 8).astype(np.int64))


def err_beyond_rounding(got: np.ndarray, ref: np.ndarray) -> float:
    """max(|got - ref| - half_ulp_bf16(ref)) / RMS(ref).

    The layer's output is bf16, so every implementation pays the rounding of the exact
    result to bf16; on the prefill workload that rounding alone reaches 2.2e-2 * RMS.
    The stated bounds (2e-2 bf16, 5e-2 FP8) apply to the error beyond it.
    """
    r = O.rms(ref)
    return float(np.max(np.abs(got - ref) - half_ulp_bf16(ref)) / r)


__all__ = ["CONFIGS", "GpuForward", "bits", "cpu_inputs", "oracle_out", "bf16_to_f64", "max_err_over_rms",
           "half_ulp_bf16", "err_beyond_rounding"]


def untile_groups(flat_bits: np.ndarray, group_info: np.ndarray, num_groups: int, rows: int,
                  kchunks: int) -> np.ndarray:
    """Row-major [rows, 64 * kchunks] from a buffer in the row-group order of the
    swapped-operand GEMMs: the group of n rows at x_row starts at element x_row * 64 *
    kchunks; its chunk c is n rows of 64 elements; row j's 16-byte piece q is stored at
    position q ^ (j % 8). Rows outside every group stay zero."""
    flat = np.asarray(flat_bits).reshape(-1)
    out = np.zeros((rows, 64 * kchunks), dtype=flat.dtype)
    for g in range(num_groups):
        x_row, meta = int(group_info[g][0]), int(group_info[g][1])
        n = (meta >> 16) & 0x1FF  # rows (bits 16-24; padding count above)
        base = x_row * 64 * kchunks
        grp = flat[base:base + n * 64 * kchunks].reshape(kchunks, n, 8, 8)
        j = np.arange(n)
        phys = np.arange(8)[None, :] ^ (j[:, None] & 7)       # where logical piece q is stored
        logical = grp[:, j[:, None], phys, :]                  # [kchunks, n, 8, 8]
        out[x_row:x_row + n] = logical.transpose(1, 0, 2, 3).reshape(n, 64 * kchunks)
    return out


def untile_weights(flat_bits: np.ndarray, E: int, rows: int, K: int) -> np.ndarray:
    """[E, MT*128, KC*64] from the tiled weight layout: tile (e, m, c) of 128 x 64 at
    ((e * MT + m) * KC + c) * 8192 elements, row r's 16-byte piece q at q ^ (r % 8)."""
    MT, KC = -(-rows // 128), -(-K // 64)
    t = np.asarray(flat_bits).reshape(E, MT, KC, 128, 8, 8)
    r = np.arange(128)
    phys = np.arange(8)[None, :] ^ (r[:, None] & 7)
    u = t[:, :, :, r[:, None], phys, :]                          # [E, MT, KC, 128, 8, 8]
    return u.transpose(0, 1, 3, 2, 4, 5).reshape(E, MT * 128, KC * 64)


def cover_tokens(ids: np.ndarray, num_routed: int, extra: int = 0, seed: int = 0) -> np.ndarray:
    """A token sample in which every routed expert that receives any pair appears at
    least once: tokens taken greedily (most still-uncovered routed experts first, lowest
    index on ties), plus ``extra`` more drawn at random. Ids >= num_routed (the shared
    slot) count as covered. Returns sorted token indices."""
    clipped = np.minimum(np.asarray(ids), num_routed)
    covered = np.ones(num_routed + 1, dtype=bool)
    covered[np.unique(clipped[clipped < num_routed])] = False
    chosen = []
    while not covered.all():
        t = int(np.argmax((~covered[clipped]).sum(axis=1)))
        chosen.append(t)
        covered[clipped[t]] = True
    rest = np.setdiff1d(np.arange(clipped.shape[0]), chosen)
    if extra > 0 and rest.size:
        chosen += list(np.random.default_rng(seed).choice(rest, size=min(extra, rest.size), replace=False))
    return np.sort(np.asarray(chosen, dtype=np.int64))


def per_expert_threaded(fn, experts, workers: int = 8) -> dict:
    """{e: fn(e)} for every listed expert, evaluated on a thread pool (the oracle's
    NumPy routines release the interpreter lock inside their array operations)."""
    from concurrent.futures import ThreadPoolExecutor
    experts = [int(e) for e in experts]
    with ThreadPoolExecutor(max_workers=workers) as ex:
        return dict(zip(experts, ex.map(fn, experts)))


def oracle_fp8_block_weights(w13_bits, w2_bits, experts):
    """O.quantize_weights_fp8 for the listed experts (others zero), expert by expert on
    a thread pool."""
    E = w13_bits.shape[0]
    w13_q = np.zeros(w13_bits.shape, dtype=np.uint8)
    w2_q = np.zeros(w2_bits.shape, dtype=np.uint8)
    w13_s = np.zeros((E, w13_bits.shape[1] // 128, w13_bits.shape[2] // 128), dtype=np.float32)
    w2_s = np.zeros((E, w2_bits.shape[1] // 128, w2_bits.shape[2] // 128), dtype=np.float32)

    def one(e):
        return (O.quant_blocks_128x128(O.bf16_bits_to_f32(np.asarray(w13_bits[e]))),
                O.quant_blocks_128x128(O.bf16_bits_to_f32(np.asarray(w2_bits[e]))))

    for e, ((q13, s13), (q2, s2)) in per_expert_threaded(one, experts).items():
        w13_q[e], w13_s[e], w2_q[e], w2_s[e] = q13, s13, q2, s2
    return w13_q, w13_s, w2_q, w2_s


def oracle_mxfp8_weights(w13_bits, w2_bits, experts):
    """O.quantize_weights_mxfp8 for the listed experts (others zero), on a thread pool."""
    E, N1, H = w13_bits.shape
    I = w2_bits.shape[2]
    out = [np.zeros((E, N1, H), np.uint8), np.zeros((E, N1, H // 32), np.uint8),
           np.zeros((E, H, I), np.uint8), np.zeros((E, H, I // 32), np.uint8)]

    def one(e):
        return (O.quant_mx(O.bf16_bits_to_f32(np.asarray(w13_bits[e]))),
                O.quant_mx(O.bf16_bits_to_f32(np.asarray(w2_bits[e]))))

    for e, ((q13, s13), (q2, s2)) in per_expert_threaded(one, experts).items():
        out[0][e], out[1][e], out[2][e], out[3][e] = q13, s13, q2, s2
    return tuple(out)


def sampled_pairs(ids: np.ndarray, tokens: np.ndarray):
    """(token, slot, expert) of every pair of the sampled tokens."""
    t = np.repeat(np.asarray(tokens, dtype=np.int64), ids.shape[1])
    j = np.tile(np.arange(ids.shape[1]), len(tokens))
    return t, j, ids[t, j]


def check_act_pairs(ref_fn, got_rows: np.ndarray, ids: np.ndarray, tokens: np.ndarray, pair_to_row: np.ndarray,
                    bound_fn) -> float:
    """GEMM1's stored activation of every pair of the sampled tokens against the oracle's.
    ref_fn(e, token_indices) -> reference activation rows [n, I] (float64); got_rows[r] is
    the kernel's activation of sorted row r (float64, [rows, I]); bound_fn(ref, got) ->
    True where the element is within its bound. Returns the number of elements checked."""
    kk = ids.shape[1]
    t, j, e = sampled_pairs(ids, tokens)
    n = 0
    for ex in np.unique(e):
        sel = e == ex
        ref = ref_fn(int(ex), t[sel])
        got = got_rows[pair_to_row[t[sel] * kk + j[sel]], :ref.shape[1]]
        ok = bound_fn(ref, got)
        if not np.all(ok):
            bad = np.argwhere(~ok)[0]
            raise AssertionError(f"activation of expert {ex}, pair {bad}: got {got[tuple(bad)]}, ref {ref[tuple(bad)]}")
        n += ref.size
    return n


def bf16_act_bound(ref: np.ndarray, got: np.ndarray) -> np.ndarray:
    """A bf16-stored activation: its rounding (2^-8 relative, with room for fp32
    accumulation order) plus 1e-3 of the RMS of the checked rows."""
    return np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-3 * O.rms(ref) + 1e-30


def act_rows_f64(parts: Dict[str, np.ndarray], I_pad: int) -> np.ndarray:
    """GEMM1's bf16 activation as float64 [rows, I_pad] in sorted row order, from the
    row-group layout (block_m 16) or the row-major one (block_m 128)."""
    if parts["block_m"] == 16:
        rows = parts["sorted_pair_ids"].shape[0]
        b = untile_groups(parts["act"], parts["group_info"], int(parts["num_blocks"][1]), rows, -(-I_pad // 64))
        return bf16_to_f64(b[:, :I_pad])
    return bf16_to_f64(parts["act"])


def untile_u8(flat, group_info, num_groups, rows, kchunks):
    """Row-major [rows, 128 * kchunks] bytes from row-group order with 128-byte chunks of
    e4m3 codes (row j's 16-byte piece q stored at position q ^ (j % 8))."""
    flat = np.asarray(flat).reshape(-1)
    out = np.zeros((rows, 128 * kchunks), dtype=np.uint8)
    for g in range(num_groups):
        x_row, meta = int(group_info[g][0]), int(group_info[g][1])
        n = (meta >> 16) & 0x1FF  # rows (bits 16-24; padding count above)
        grp = flat[x_row * 128 * kchunks:(x_row + n) * 128 * kchunks].reshape(kchunks, n, 8, 16)
        j = np.arange(n)
        phys = np.arange(8)[None, :] ^ (j[:, None] & 7)
        out[x_row:x_row + n] = grp[:, j[:, None], phys, :].transpose(1, 0, 2, 3).reshape(n, 128 * kchunks)
    return out


def untile_b128(flat, group_info, num_groups, rows, kchunks):
    """(codes uint8 [rows, 128 * kchunks], scales float32 [rows, kchunks]) from the FP8
    block-128 X layout of the swapped-operand GEMMs: the group of n rows at x_row owns
    bytes from x_row * kchunks * 132; its K step of chunks [c0, c0 + kcs) (kcs chunks per
    step as the GEMM takes them for n rows: 4 up to 32 rows, 3 up to 64, 2 up to 128)
    starts at c0 * n * 132 with kcs chunks of n swizzled 128-byte code rows, then the
    step's fp32 scales, chunk-major. Rows outside every group stay zero."""
    flat = np.asarray(flat).reshape(-1)
    codes = np.zeros((rows, 128 * kchunks), dtype=np.uint8)
    scales = np.zeros((rows, kchunks), dtype=np.float32)
    for g in range(num_groups):
        x_row, meta = int(group_info[g][0]), int(group_info[g][1])
        n = (meta >> 16) & 0x1FF  # rows (bits 16-24; padding count above)
        kc = 4 if n <= 32 else (3 if n <= 64 else (2 if n <= 128 else 1))
        base = x_row * kchunks * 132
        j = np.arange(n)
        phys = np.arange(8)[None, :] ^ (j[:, None] & 7)
        for c0 in range(0, kchunks, kc):
            kcs = min(kc, kchunks - c0)
            step = base + c0 * n * 132
            cod = flat[step:step + kcs * n * 128].reshape(kcs, n, 8, 16)
            codes[x_row:x_row + n, 128 * c0:128 * (c0 + kcs)] = \
                cod[:, j[:, None], phys, :].transpose(1, 0, 2, 3).reshape(n, 128 * kcs)
            sc = flat[step + kcs * n * 128:step + kcs * n * 132].copy().view(np.float32).reshape(kcs, n)
            scales[x_row:x_row + n, c0:c0 + kcs] = sc.T
    return codes, scales
