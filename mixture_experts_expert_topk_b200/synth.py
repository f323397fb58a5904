"""Seeded synthetic inputs for the fused MoE layer forward.

This module only draws random numbers and arranges them into the tensors a
caller hands to the layer: hidden states, router logits and bf16 master
weights. It holds none of the layer's arithmetic (no routing, no
quantisation, no GEMM), so both the CUDA path and the CPU oracle can take
their inputs from here without sharing any of the method.

All tensors are drawn on the CPU from one ``torch.Generator`` seeded with
``seed``, in the fixed order hidden, logits, [logit bias], w13, w2, so that
every consumer sees identical bytes. Values are drawn in fp32 and rounded to
bf16 where the layer consumes bf16.

Weight layout is the checkpoint layout: ``w13[e]`` holds the gate rows
``[0, I)`` followed by the up rows ``[I, 2I)`` for gated activations (the
"[Gate, Up]" order of the sglang #21321 page, section 2, after its
``swap_w13_halves`` step), or just ``I`` rows for relu2; ``w2[e]`` is
``[H, I]``. A fused shared expert, when present, is the last expert slot.
"""
from __future__ import annotations

import dataclasses
from typing import Dict

import torch

__all__ = ["MoeConfig", "CONFIGS", "decode_config", "make_inputs", "make_logits"]


@dataclasses.dataclass(frozen=True)
class MoeConfig:
    name: str
    T: int                 # tokens
    H: int                 # hidden size
    E: int                 # routed experts (columns of router_logits)
    topk: int              # routed experts per token
    I: int                 # intermediate size (unpadded)
    renormalize: bool
    activation: str        # "swiglu" | "relu2" | "gelu_tanh" | "swigluoai"
    num_shared: int = 0    # fused shared-expert slots appended after the routed experts
    # False: bf16. True: e4m3 with 128-wide block scales. "per_tensor": e4m3 with one scale
    # per expert matrix and static input / activation scales (activation_scale below; the
    # input scale is the hidden rows' amax / 448). "mxfp8": e4m3 with a power-of-two scale
    # per 32 values of K on both GEMM inputs. "nvfp4": E2M1 with an E4M3 scale per 16 values
    # of K and tensor scales (the input's: the hidden rows' amax / (6 * 448); the
    # activation's: activation_scale below)
    fp8: object = False
    activation_scale: float = 0.03
    hidden_std: float = 1.0
    weight_std: float = 0.02
    logit_bias_std: float = 0.0   # per-expert bias added to the logits (skewed load)
    block_m: int = 128

    @property
    def per_tensor(self) -> bool:
        return self.fp8 == "per_tensor"

    @property
    def block128(self) -> bool:
        return self.fp8 is True

    @property
    def mx(self) -> bool:
        return self.fp8 == "mxfp8"

    @property
    def nv(self) -> bool:
        return self.fp8 == "nvfp4"

    @property
    def gated(self) -> bool:
        return self.activation != "relu2"

    @property
    def E_total(self) -> int:
        return self.E + self.num_shared

    @property
    def k_total(self) -> int:
        return self.topk + self.num_shared

    @property
    def N1(self) -> int:
        return 2 * self.I if self.gated else self.I

    def replace(self, **kw) -> "MoeConfig":
        return dataclasses.replace(self, **kw)

    def flops(self) -> float:
        """Algorithmic FLOPs of one layer call (both GEMMs, 2 flops per MAC)."""
        P = self.T * self.k_total
        return 2.0 * P * self.H * self.N1 + 2.0 * P * self.I * self.H


# The five workloads of the layer (tiny parity case, prefill, relu2, FP8 with a
# fused shared expert, decode sweep).
CONFIGS: Dict[str, MoeConfig] = {
    "tiny": MoeConfig("tiny", T=16, H=256, E=8, topk=2, I=512, renormalize=True,
                      activation="swiglu"),
    "prefill": MoeConfig("prefill", T=4096, H=2048, E=256, topk=8, I=512, renormalize=True,
                         activation="swiglu", logit_bias_std=0.5),
    "relu2": MoeConfig("relu2", T=2048, H=4096, E=128, topk=6, I=2688, renormalize=False,
                       activation="relu2"),
    "fp8_shared": MoeConfig("fp8_shared", T=8192, H=2048, E=512, topk=10, I=512,
                            renormalize=True, activation="swiglu", num_shared=1, fp8=True),
    # the same shape with per-tensor FP8 scales
    "fp8pt_shared": MoeConfig("fp8pt_shared", T=8192, H=2048, E=512, topk=10, I=512,
                              renormalize=True, activation="swiglu", num_shared=1, fp8="per_tensor"),
}


# The prefill shape with MXFP8 weights and GEMM inputs.
CONFIGS["mxfp8_prefill"] = MoeConfig("mxfp8_prefill", T=4096, H=2048, E=256, topk=8, I=512, renormalize=True,
                                     activation="swiglu", logit_bias_std=0.5, fp8="mxfp8")


# A smaller case of the prefill workload for profiler captures: the same shapes per
# expert (H, I, top-8, about 128 pairs per expert) with 64 experts, so the weights
# (400 MB) still exceed L2 but a capture holds well under a gigabyte.
CONFIGS["prefill_e64"] = MoeConfig("prefill_e64", T=1024, H=2048, E=64, topk=8, I=512,
                                   renormalize=True, activation="swiglu", logit_bias_std=0.5)
CONFIGS["mxfp8_e64"] = CONFIGS["prefill_e64"].replace(name="mxfp8_e64", fp8="mxfp8")
CONFIGS["fp8_e64"] = CONFIGS["prefill_e64"].replace(name="fp8_e64", fp8=True)


# The prefill shape with NVFP4 weights and GEMM inputs (W4A4). The activation's tensor scale
# is 12 / (6 * 448): GEMM1's activation on this workload stays below about 10 in magnitude
# (the float64 activation over an eighth of the tokens peaks at 10.06), so no block scale
# saturates.
CONFIGS["nvfp4_prefill"] = CONFIGS["prefill"].replace(name="nvfp4_prefill", fp8="nvfp4", activation_scale=12.0 / 2688)
CONFIGS["nvfp4_e64"] = CONFIGS["prefill_e64"].replace(name="nvfp4_e64", fp8="nvfp4", activation_scale=12.0 / 2688)


# A compute-bound case of the prefill kernels: the prefill shapes (H=2048, I=512, SwiGLU,
# top-8) with 8 experts and 16384 tokens, so every expert receives 16384 rows (about 16k
# tokens per expert, far above the ~250 flop/byte ridge) and the grouped GEMMs are bound
# by the tensor cores rather than by the weight stream.
CONFIGS["compute_diag"] = MoeConfig("compute_diag", T=16384, H=2048, E=8, topk=8, I=512, renormalize=True,
                                    activation="swiglu")


def decode_config(T: int) -> MoeConfig:
    """Decode-sweep workload: T in {1, 4, 16, 64} tokens, uniform logits."""
    return MoeConfig(f"decode_T{T}", T=T, H=2048, E=256, topk=8, I=512, renormalize=True,
                     activation="swiglu")


for _t in (1, 4, 16, 64):
    CONFIGS[f"decode_T{_t}"] = decode_config(_t)


def _normal(gen: torch.Generator, shape, std: float) -> torch.Tensor:
    x = torch.empty(shape, dtype=torch.float32)
    x.normal_(mean=0.0, std=std, generator=gen)
    return x


def make_logits(cfg: MoeConfig, gen: torch.Generator) -> torch.Tensor:
    logits = _normal(gen, (cfg.T, cfg.E), 1.0)
    if cfg.logit_bias_std > 0:
        bias = _normal(gen, (cfg.E,), cfg.logit_bias_std)
        logits += bias[None, :]
    return logits


def make_inputs(cfg: MoeConfig, seed: int = 0, weights: bool = True) -> Dict[str, torch.Tensor]:
    """Draw the layer inputs of ``cfg`` on the CPU.

    Returns ``hidden`` (bf16 [T,H]), ``logits`` (fp32 [T,E]) and, when
    ``weights`` is true, ``w13`` (bf16 [E_total, N1, H]) and ``w2`` (bf16
    [E_total, H, I]). Weights are drawn expert by expert so the fp32
    temporaries stay small.
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    out: Dict[str, torch.Tensor] = {}
    out["hidden"] = _normal(gen, (cfg.T, cfg.H), cfg.hidden_std).to(torch.bfloat16)
    out["logits"] = make_logits(cfg, gen)
    if not weights:
        return out
    E_tot = cfg.E_total
    w13 = torch.empty((E_tot, cfg.N1, cfg.H), dtype=torch.bfloat16)
    for e in range(E_tot):
        w13[e] = _normal(gen, (cfg.N1, cfg.H), cfg.weight_std).to(torch.bfloat16)
    w2 = torch.empty((E_tot, cfg.H, cfg.I), dtype=torch.bfloat16)
    for e in range(E_tot):
        w2[e] = _normal(gen, (cfg.H, cfg.I), cfg.weight_std).to(torch.bfloat16)
    out["w13"] = w13
    out["w2"] = w2
    return out
