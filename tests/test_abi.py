"""Host-side checks of the C ABI: the library loads, exports every declared entry
point, and validates arguments before touching the GPU (no kernel runs here)."""
import ctypes
import os
import re

import pytest

import mixture_experts_expert_topk_b200 as moe
from mixture_experts_expert_topk_b200 import _capi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(_capi.LIB_PATH):
        from mixture_experts_expert_topk_b200 import build
        build.build()
    return moe.lib()


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_header_functions_exported_and_bound(L):
    names = _declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(L, n), n            # exported by the .so
        assert n in _capi.SIGNATURES, n    # bound by the Python layer
    assert set(_capi.SIGNATURES) == set(names)


def _prob(**kw):
    base = dict(T=16, H=256, num_routed=8, topk=2, intermediate=512, renormalize=True,
                activation="swiglu")
    base.update(kw)
    T, H, E, k, I = base.pop("T"), base.pop("H"), base.pop("num_routed"), base.pop("topk"), base.pop("intermediate")
    return moe.make_problem(T, H, E, k, I, **base)


def test_check_problem_accepts_the_workloads(L):
    from mixture_experts_expert_topk_b200.synth import CONFIGS
    for cfg in CONFIGS.values():
        p = moe.make_problem(cfg.T, cfg.H, cfg.E, cfg.topk, cfg.I, renormalize=cfg.renormalize,
                             activation=cfg.activation, num_shared=cfg.num_shared, fp8=cfg.fp8,
                             input_scale=0.01, activation_scale=cfg.activation_scale)
        assert L.moe_check_problem(ctypes.byref(p)) == 0, cfg.name


@pytest.mark.parametrize("kw,status", [
    (dict(T=-1), 1), (dict(H=0), 1), (dict(H=200), 2), (dict(num_routed=0), 1),
    (dict(topk=9), 1), (dict(topk=0), 1), (dict(intermediate=500), 1),
    (dict(intermediate=512, activation="relu2"), 0), (dict(intermediate=528, activation="relu2"), 1),
    (dict(num_routed=1100, topk=2), 2), (dict(num_routed=32, topk=17), 2),
    (dict(block_m=64), 2), (dict(intermediate=528, fp8=True), 1), (dict(block_m=16, fp8=True), 0),
    (dict(block_m=128, fp8="mxfp8"), 2), (dict(block_m=128, fp8="per_tensor", input_scale=0.1, activation_scale=0.1), 2),
    (dict(H=4224, fp8=True), 2),
])
def test_check_problem_rejects(L, kw, status):
    p = _prob(**kw)
    assert L.moe_check_problem(ctypes.byref(p)) == status


def test_check_problem_flags_and_shared(L):
    p = _prob()
    p.flags = 0x10
    assert L.moe_check_problem(ctypes.byref(p)) == 1
    p = _prob(num_shared=2)
    assert L.moe_check_problem(ctypes.byref(p)) == 1
    p = _prob(num_shared=1, topk=8)   # E_r = 8, topk 8 + shared slot
    assert L.moe_check_problem(ctypes.byref(p)) == 0
    assert L.moe_check_problem(None) == 1


def test_padded_intermediate_follows_page_rule(L):
    with open(os.path.join(GOLDEN, "padding_rules.txt")) as f:
        rows = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    for i_in, gated, i_pad in rows:
        act = _capi.MOE_ACT_SWIGLU if gated == "1" else _capi.MOE_ACT_RELU2
        assert L.moe_padded_intermediate(int(i_in), act, 0) == int(i_pad)
    assert L.moe_padded_intermediate(500, _capi.MOE_ACT_SWIGLU, 1) == 512   # FP8: 128
    assert L.moe_padded_intermediate(0, 0, 0) == -1
    assert L.moe_padded_intermediate(200, _capi.MOE_ACT_SWIGLU, _capi.MOE_DTYPE_FP8_PER_TENSOR) == 256
    assert L.moe_padded_intermediate(200, _capi.MOE_ACT_GELU_TANH, 0) == 208
    assert L.moe_padded_intermediate(200, _capi.MOE_ACT_SWIGLUOAI, 0) == 208   # gated: 16
    assert L.moe_padded_intermediate(200, 4, 0) == -1                          # no such activation
    assert L.moe_padded_intermediate(200, 0, _capi.MOE_DTYPE_MXFP8) == 256   # MXFP8: 128
    assert L.moe_padded_intermediate(200, 0, _capi.MOE_DTYPE_NVFP4) == 256   # NVFP4: 256-value chunks
    assert L.moe_padded_intermediate(200, 0, 5) == -1
    assert L.moe_padded_intermediate(16, 7, 0) == -1


def test_workspace_layout(L):
    from mixture_experts_expert_topk_b200.synth import CONFIGS
    for cfg in CONFIGS.values():
        p = moe.make_problem(cfg.T, cfg.H, cfg.E, cfg.topk, cfg.I, renormalize=cfg.renormalize,
                             activation=cfg.activation, num_shared=cfg.num_shared, fp8=cfg.fp8,
                             input_scale=0.01, activation_scale=cfg.activation_scale)
        lay = moe.workspace_layout(p)
        P = cfg.T * cfg.k_total
        E = cfg.E_total
        assert lay["status"] == 0
        bm = lay["block_m"]
        # every format aligns each expert to 16 rows by default (token rows on the MMA's N)
        assert bm == 16
        # the permuted hidden rows (row-group order): bf16, e4m3 codes, or (FP8 block-128)
        # e4m3 codes with a 4-byte scale per row per 128 columns
        xs_bytes = lay["xs_scale"] - lay["xs"]
        row_bytes = (cfg.H * 132 // 128 if cfg.block128 else
                     (cfg.H // 2 if cfg.nv else cfg.H * (1 if (cfg.per_tensor or cfg.mx) else 2)))
        assert xs_bytes == -(-lay["max_rows"] * row_bytes // 1024) * 1024
        assert lay["max_rows"] == -(-(P + min(E, P) * (bm - 1)) // bm) * bm
        assert lay["num_chunks"] == -(-P // 2048)
        offs = sorted(v for k, v in lay.items() if k not in ("total_bytes", "max_rows", "num_chunks", "block_m"))
        assert all(o % 1024 == 0 for o in offs)
        assert lay["y"] + lay["max_rows"] * cfg.H * 4 <= lay["total_bytes"]
        assert moe.workspace_size(p) == lay["total_bytes"]
    bad = _prob(H=0)
    assert L.moe_workspace_size(ctypes.byref(bad)) == 0


def test_entry_points_validate_before_any_cuda_call(L):
    p = _prob()
    n = moe.workspace_size(p)
    fake = ctypes.c_void_p(1 << 20)      # aligned, never dereferenced
    mis = ctypes.c_void_p((1 << 20) + 4)
    s = ctypes.c_void_p(0)
    f = L.moe_forward
    # null / misaligned pointers
    assert f(ctypes.byref(p), None, fake, fake, fake, None, None, fake, fake, n, s) == 1
    assert f(ctypes.byref(p), mis, fake, fake, fake, None, None, fake, fake, n, s) == 1
    # output aliasing the input
    assert f(ctypes.byref(p), fake, fake, fake, fake, None, None, fake, ctypes.c_void_p(2 << 20), n, s) == 1
    # workspace too small / misaligned
    ws = ctypes.c_void_p(4 << 20)
    assert f(ctypes.byref(p), fake, fake, fake, fake, None, None, ctypes.c_void_p(3 << 20), ws, n - 1, s) == 3
    assert f(ctypes.byref(p), fake, fake, fake, fake, None, None, ctypes.c_void_p(3 << 20),
             ctypes.c_void_p((4 << 20) + 16), n, s) == 1
    # FP8 without scales
    p8 = _prob(fp8=True)
    n8 = moe.workspace_size(p8)
    assert f(ctypes.byref(p8), fake, fake, fake, fake, None, None, ctypes.c_void_p(3 << 20), ws, n8, s) == 1
    # T == 0: valid, nothing enqueued, no device needed
    p0 = _prob(T=0)
    n0 = moe.workspace_size(p0)
    assert f(ctypes.byref(p0), fake, fake, fake, fake, None, None, ctypes.c_void_p(3 << 20), ws, n0, s) == 0
    # invalid problem
    pb = _prob(topk=0)
    assert f(ctypes.byref(pb), fake, fake, fake, fake, None, None, ctypes.c_void_p(3 << 20), ws, n, s) == 1
    # stages and helpers
    assert L.moe_stage_route(ctypes.byref(p), None, ws, n, s) == 1
    assert L.moe_stage_align(ctypes.byref(p), ws, n - 1, s) == 3
    assert L.moe_stage_quant_act(ctypes.byref(p), fake, ws, n, s) == 1          # bf16 problem
    assert L.moe_stage_gemm1(ctypes.byref(p), None, fake, None, ws, n, s) == 1
    assert L.moe_stage_gemm2(ctypes.byref(p8), fake, None, ws, n8, s) == 1       # FP8 needs scales
    assert L.moe_stage_combine(ctypes.byref(p), None, ws, n, s) == 1
    assert L.moe_forward_host(ctypes.byref(p), None, fake, fake, fake, None, None, fake, ws, n, s) == 1
    assert L.moe_prepare_weights(ctypes.byref(p), 300, fake, fake, fake, fake, s) == 1   # pads to 304 != 512
    assert L.moe_quantize_weights_fp8(fake, 1, 100, 128, fake, fake, s) == 1
    assert L.moe_quantize_weights_fp8(fake, 0, 128, 128, fake, fake, s) == 0
    assert L.moe_get_device_status(None, s, None) == 1


def test_status_strings(L):
    for code, name in [(0, "MOE_OK"), (1, "MOE_ERR_INVALID_ARG"), (2, "MOE_ERR_UNSUPPORTED"),
                       (3, "MOE_ERR_WORKSPACE_TOO_SMALL"), (4, "MOE_ERR_CUDA"),
                       (5, "MOE_ERR_DEVICE_TIMEOUT")]:
        assert L.moe_status_string(code).decode() == name


def test_python_layer_fails_loudly_without_a_gpu_tensor():
    import torch
    with pytest.raises(ValueError):
        moe.moe_forward(torch.zeros(4, 256, dtype=torch.bfloat16), torch.zeros(4, 8),
                        torch.zeros(1), torch.zeros(1), 2, True, "swiglu")


def test_per_tensor_fp8_problem_rules(L):
    ok = moe.make_problem(64, 256, 8, 2, 256, fp8="per_tensor", input_scale=0.01, activation_scale=0.05)
    assert L.moe_check_problem(ctypes.byref(ok)) == 0
    lay = moe.workspace_layout(ok)
    assert lay["block_m"] == 16
    # e4m3 tiles of 128 x 128: w13 [8, 512, 256] and w2 [8, 256, 256]
    assert L.moe_prepared_weights_bytes(ctypes.byref(ok), 0) == 8 * 4 * 2 * 16384
    assert L.moe_prepared_weights_bytes(ctypes.byref(ok), 1) == 8 * 2 * 2 * 16384
    # the activation (e4m3, rows x I) and permuted rows (rows x H) are one byte per element
    assert lay["y"] - lay["act"] >= lay["max_rows"] * 256
    for bad in (dict(input_scale=0.0), dict(activation_scale=-1.0), dict(input_scale=float("nan")),
                dict(activation_scale=float("inf"))):
        kw = dict(input_scale=0.01, activation_scale=0.05)
        kw.update(bad)
        p = moe.make_problem(64, 256, 8, 2, 256, fp8="per_tensor", **kw)
        assert L.moe_check_problem(ctypes.byref(p)) == 1, bad
    p = moe.make_problem(64, 256, 8, 2, 256, fp8="per_tensor", input_scale=0.01, activation_scale=0.05,
                         block_m=128)
    assert L.moe_check_problem(ctypes.byref(p)) == 2          # 128-row tiles: not for per-tensor
    p = moe.make_problem(64, 256, 8, 2, 200, fp8="per_tensor", input_scale=0.01, activation_scale=0.05)
    assert L.moe_check_problem(ctypes.byref(p)) == 1          # I must be padded to 128


def test_mxfp8_problem_rules(L):
    ok = moe.make_problem(64, 256, 8, 2, 256, fp8="mxfp8")
    assert L.moe_check_problem(ctypes.byref(ok)) == 0
    lay = moe.workspace_layout(ok)
    assert lay["block_m"] == 16
    # e4m3 tiles of 128 x 128 plus one 512-byte scale block per tile: w13 [8, 512, 256], w2 [8, 256, 256]
    assert L.moe_prepared_weights_bytes(ctypes.byref(ok), 0) == 8 * 4 * 2 * (16384 + 512)
    assert L.moe_prepared_weights_bytes(ctypes.byref(ok), 1) == 8 * 2 * 2 * (16384 + 512)
    # scale blocks of the permuted hidden rows and of the activation: 1024 bytes per 16 rows
    # per 128 columns
    assert lay["group_info"] - lay["xs_scale"] >= lay["max_rows"] // 16 * 2 * 1024
    assert lay["y"] - lay["act_scale"] >= lay["max_rows"] // 16 * 2 * 1024
    assert lay["act_scale"] - lay["actq"] >= lay["max_rows"] * 256
    p = moe.make_problem(64, 256, 8, 2, 256, fp8="mxfp8", block_m=128)
    assert L.moe_check_problem(ctypes.byref(p)) == 2          # 128-row tiles: not for MXFP8
    p = moe.make_problem(64, 256, 8, 2, 200, fp8="mxfp8")
    assert L.moe_check_problem(ctypes.byref(p)) == 1          # I must be padded to 128
    fake = ctypes.c_void_p(1 << 20)
    s = ctypes.c_void_p(0)
    n = moe.workspace_size(ok)
    # the scales travel inside the prepared weights: scale pointers must be NULL
    assert L.moe_forward(ctypes.byref(ok), fake, fake, fake, fake, fake, None, ctypes.c_void_p(3 << 20),
                         ctypes.c_void_p(4 << 20), n, s) == 1
    # the generic preparation refuses MXFP8; the MXFP8 one refuses other formats and missing scales
    assert L.moe_prepare_weights(ctypes.byref(ok), 256, fake, fake, fake, fake, s) == 1
    assert L.moe_prepare_weights_mxfp8(ctypes.byref(_prob()), fake, fake, fake, fake, fake, fake, s) == 1
    assert L.moe_prepare_weights_mxfp8(ctypes.byref(ok), fake, None, fake, fake, fake, fake, s) == 1
    assert L.moe_quantize_weights_mxfp8(fake, 1, 4, 48, fake, fake, s) == 1   # 32-column blocks
    assert L.moe_quantize_weights_mxfp8(fake, 0, 4, 64, fake, fake, s) == 0
