// Step 1 of the layer: top-k expert routing with softmax weights.
//
// "FlashInfer TRTLLM-Gen MoE kernel optimisation: NemotronH support" (sglang PR 21321),
// section 1: the fused op takes router logits, `topk` and `renormalize`. Reading (the
// page prints no formula): select the k largest raw fp32 logits (ties towards the lower
// expert index, slots ordered by logit descending), weight each by its softmax
// probability over all routed experts, optionally divided by the selected sum.
// "Qwen3-Next FP8 MoE optimisation: shared-expert fusion for H200" (sglang PR 26204),
// section 2: a fused shared expert is one more slot, id E_r, weight 1, after the routed
// slots.
//
// One warp per token. A lane holds logits lane, lane+32, ... in registers; each of the
// k selection rounds is a register scan plus a 5-step butterfly arg-max. Selection runs
// on the raw logits, so the ids never depend on the exponential's rounding.
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kRouteWarps = 8;

struct Cand {
  float v;
  int i;
};

// a beats b: larger logit, or equal logit and lower expert index.
__device__ __forceinline__ bool beats(const Cand& a, const Cand& b) {
  return a.v > b.v || (a.v == b.v && a.i < b.i);
}

template <int VPL>
__global__ void __launch_bounds__(kRouteWarps * 32)
    route_kernel(const float* __restrict__ logits, int T, int E, int topk, int num_shared,
                 int renormalize, int* __restrict__ topk_ids, float* __restrict__ topk_w,
                 int* __restrict__ status) {
  griddep_wait();
  // routing starts every forward: clear the device status word of the workspace
  if (blockIdx.x == 0 && threadIdx.x == 0) *status = 0;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kRouteWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  const float* row = logits + static_cast<size_t>(t) * E;

  float v[VPL];
  uint32_t taken = 0;  // bit i: value i of this lane selected or absent
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      v[i] = __ldg(row + e);
    } else {
      v[i] = -INFINITY;
      taken |= 1u << i;
    }
  }

  // softmax denominator over all routed experts (max subtracted)
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < VPL; ++i)
    if (!(taken >> i & 1u)) m = fmaxf(m, v[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i)
    if (!(taken >> i & 1u)) s += expf(v[i] - m);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);

  // k rounds of arg-max; slot j's exp(l - m) is kept by lane j
  float my_e = 0.f;
  int my_id = 0;
  float sel_sum = 0.f;
  for (int j = 0; j < topk; ++j) {
    Cand best{-INFINITY, 0x7fffffff};
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      Cand c{v[i], lane + 32 * i};
      if (!(taken >> i & 1u) && beats(c, best)) best = c;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      Cand other{__shfl_xor_sync(0xffffffffu, best.v, o), __shfl_xor_sync(0xffffffffu, best.i, o)};
      if (beats(other, best)) best = other;
    }
    if ((best.i & 31) == lane) taken |= 1u << (best.i >> 5);
    const float ej = expf(best.v - m);
    sel_sum += ej;
    if (lane == j) {
      my_e = ej;
      my_id = best.i;
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

template <int VPL>
cudaError_t launch_vpl(const Launch& l, const float* logits, int T, int E, int topk,
                       int num_shared, int renormalize, int* ids, float* w, int* status) {
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3((T + kRouteWarps - 1) / kRouteWarps),
                     dim3(kRouteWarps * 32), 0);
  return cudaLaunchKernelEx(&cfg, route_kernel<VPL>, logits, T, E, topk, num_shared, renormalize,
                            ids, w, status);
}

}  // namespace

cudaError_t launch_route(const Launch& l, const float* logits, int T, int E_routed, int topk,
                         int num_shared, int renormalize, int* topk_ids, float* topk_w,
                         int* status) {
  const int vpl = (E_routed + 31) / 32;
  if (vpl <= 1) return launch_vpl<1>(l, logits, T, E_routed, topk, num_shared, renormalize, topk_ids, topk_w, status);
  if (vpl <= 2) return launch_vpl<2>(l, logits, T, E_routed, topk, num_shared, renormalize, topk_ids, topk_w, status);
  if (vpl <= 4) return launch_vpl<4>(l, logits, T, E_routed, topk, num_shared, renormalize, topk_ids, topk_w, status);
  if (vpl <= 8) return launch_vpl<8>(l, logits, T, E_routed, topk, num_shared, renormalize, topk_ids, topk_w, status);
  if (vpl <= 16) return launch_vpl<16>(l, logits, T, E_routed, topk, num_shared, renormalize, topk_ids, topk_w, status);
  return launch_vpl<32>(l, logits, T, E_routed, topk, num_shared, renormalize, topk_ids, topk_w, status);
}

}  // namespace moe
