// Top-k expert routing of one token by one warp (the arithmetic of route.cu's step 1),
// shared by the routing kernel and the fused routing + align kernel of small batches.
//
// "FlashInfer TRTLLM-Gen MoE kernel optimisation: NemotronH support" (sglang PR 21321),
// section 1: the fused op takes router logits, `topk` and `renormalize`. Reading: select the
// k largest raw fp32 logits (ties towards the lower expert index, slots ordered by logit
// descending), weight each by its softmax probability over all routed experts, optionally
// divided by the selected sum. "Qwen3-Next FP8 MoE optimisation: shared-expert fusion for
// H200" (sglang PR 26204), section 2: a fused shared expert is one more slot, id E_r,
// weight 1, after the routed slots.
#pragma once

#include "moe_device.cuh"

namespace moe {

// Order-preserving map of finite floats to unsigned integers (larger float -> larger
// key; -0 is folded onto +0 so the two compare equal, as floats do). Key 0 is below every
// finite float's key and marks absent or already selected entries.
__device__ __forceinline__ uint32_t order_key(float x) {
  const uint32_t b = __float_as_uint(x == 0.f ? 0.f : x);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Token t's routing by the calling warp (all 32 lanes): row = its E logits; writes its
// k' = topk + num_shared slots at topk_ids / topk_w [t * k']. A lane holds logits lane,
// lane+32, ... as order-preserving integer keys; each of the k selection rounds is a
// register scan plus two warp reductions (redux.sync max of the key, then min of the
// expert index among the lanes holding it). Selection runs on the raw logits, so the ids
// never depend on the exponential's rounding.
template <int VPL>
__device__ __forceinline__ void route_token(const float* __restrict__ logits, int t, int E, int topk,
                                            int num_shared, int renormalize, int lane, int* topk_ids,
                                            float* topk_w) {
  const float* row = logits + static_cast<size_t>(t) * E;

  // lane holds experts lane, lane + 32, ...; an expert's index is lane + 32 * i
  uint32_t key[VPL];
  uint32_t lmax = 0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane + 32 * i;
    key[i] = e < E ? order_key(__ldg(row + e)) : 0u;
    lmax = max(lmax, key[i]);
  }
  // softmax shift: the largest logit
  const float m = key_value(__reduce_max_sync(0xffffffffu, lmax));
  // with renormalisation the full softmax denominator cancels and is not needed
  float s = 0.f;
  if (!renormalize) {
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      if (key[i] != 0u) s += expf(key_value(key[i]) - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  }

  // k rounds: the largest remaining key, ties to the lowest expert index. Lane j keeps
  // slot j's expert and exp(l - m).
  float my_e = 0.f;
  int my_id = 0;
  float sel_sum = 0.f;
  for (int j = 0; j < topk; ++j) {
    uint32_t bk = 0u;
    int bi = 0;
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      if (key[i] > bk) {  // strict: the lowest i among equal keys
        bk = key[i];
        bi = i;
      }
    const uint32_t wk = __reduce_max_sync(0xffffffffu, bk);
    const uint32_t widx = __reduce_min_sync(0xffffffffu, bk == wk ? static_cast<uint32_t>(lane + 32 * bi) : 0xffffffffu);
    if (static_cast<uint32_t>(lane) == (widx & 31u)) {
#pragma unroll
      for (int i = 0; i < VPL; ++i)
        if (i == bi) key[i] = 0u;
    }
    const float ej = expf(key_value(wk) - m);
    sel_sum += ej;
    if (lane == j) {
      my_e = ej;
      my_id = static_cast<int>(widx);
    }
  }
  const int kk = topk + num_shared;
  if (lane < topk) {
    const float w = renormalize ? my_e / sel_sum : my_e / s;
    topk_ids[static_cast<size_t>(t) * kk + lane] = my_id;
    topk_w[static_cast<size_t>(t) * kk + lane] = w;
  } else if (lane < kk) {
    topk_ids[static_cast<size_t>(t) * kk + lane] = E;
    topk_w[static_cast<size_t>(t) * kk + lane] = 1.0f;
  }
}

}  // namespace moe
