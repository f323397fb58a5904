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
// One warp per token; the per-token arithmetic is route_token (route_device.cuh).
#include "moe_device.cuh"
#include "moe_internal.h"
#include "route_device.cuh"

namespace moe {
namespace {

constexpr int kRouteWarps = 8;

template <int VPL>
__global__ void __launch_bounds__(kRouteWarps * 32)
    route_kernel(const float* __restrict__ logits, int T, int E, int topk, int num_shared,
                 int renormalize, int* __restrict__ topk_ids, float* __restrict__ topk_w,
                 int* __restrict__ status, const uint8_t* __restrict__ hidden, int hidden_row_bytes) {
  griddep_wait();
  griddep_launch_dependents();
  // routing starts every forward: clear the workspace's status word ([0]) and the GEMMs'
  // work counters ([4..7])
  if (blockIdx.x == 0 && threadIdx.x < 8) status[threadIdx.x] = 0;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kRouteWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  // start pulling this token's hidden row into L2: GEMM1 gathers it k times right after
  if (hidden != nullptr && lane == 0)
    prefetch_l2_bulk(hidden + static_cast<size_t>(t) * hidden_row_bytes, static_cast<uint32_t>(hidden_row_bytes));
  route_token<VPL>(logits, t, E, topk, num_shared, renormalize, lane, topk_ids, topk_w);
}

// The routed variant ("FlashInfer TRTLLM-Gen MoE kernel optimisation: NemotronH support",
// section 1, names a routed form of the fused op that takes the top-k choice): the
// caller's ids and weights [T, topk] into the workspace's [T, k'] layout, the shared slot
// (id E_r, weight 1) after them as in route_kernel. An id outside [0, E_r) cannot be
// routed: the pair becomes expert 0 with weight 0 (contributing nothing) and the status
// word records kStatusBadRouting.
__global__ void load_routing_kernel(const int* __restrict__ ids_in, const float* __restrict__ w_in, int T, int E,
                                    int topk, int num_shared, int* __restrict__ topk_ids, float* __restrict__ topk_w,
                                    int* __restrict__ status) {
  griddep_wait();
  griddep_launch_dependents();
  const int kk = topk + num_shared;
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long long>(T) * kk) return;
  const long long t = idx / kk;
  const int j = static_cast<int>(idx - t * kk);
  int e = E;
  float w = 1.0f;
  if (j < topk) {
    e = __ldg(ids_in + t * topk + j);
    w = __ldg(w_in + t * topk + j);
    if (e < 0 || e >= E) {
      e = 0;
      w = 0.0f;
      atomicCAS(status, 0, kStatusBadRouting);
    }
  }
  topk_ids[idx] = e;
  topk_w[idx] = w;
}

template <int VPL>
cudaError_t launch_vpl(const Launch& l, const float* logits, int T, int E, int topk,
                       int num_shared, int renormalize, int* ids, float* w, int* status,
                       const void* hidden, int hidden_row_bytes) {
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3((T + kRouteWarps - 1) / kRouteWarps),
                     dim3(kRouteWarps * 32), 0);
  return cudaLaunchKernelEx(&cfg, route_kernel<VPL>, logits, T, E, topk, num_shared, renormalize,
                            ids, w, status, static_cast<const uint8_t*>(hidden), hidden_row_bytes);
}

}  // namespace

cudaError_t launch_load_routing(const Launch& l, const int* ids_in, const float* w_in, int T, int E_routed,
                                int topk, int num_shared, int* topk_ids, float* topk_w, int* status) {
  const long long n = static_cast<long long>(T) * (topk + num_shared);
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0);
  return cudaLaunchKernelEx(&cfg, load_routing_kernel, ids_in, w_in, T, E_routed, topk, num_shared, topk_ids, topk_w,
                            status);
}

cudaError_t launch_route(const Launch& l, const float* logits, int T, int E_routed, int topk,
                         int num_shared, int renormalize, int* topk_ids, float* topk_w,
                         int* status, const void* hidden, int hidden_row_bytes) {
  const int vpl = (E_routed + 31) / 32;
  if (vpl <= 1) return launch_vpl<1>(l, logits, T, E_routed, topk, num_shared, renormalize, topk_ids, topk_w, status, hidden, hidden_row_bytes);
  if (vpl <= 2) return launch_vpl<2>(l, logits, T, E_routed, topk, num_shared, renormalize, topk_ids, topk_w, status, hidden, hidden_row_bytes);
  if (vpl <= 4) return launch_vpl<4>(l, logits, T, E_routed, topk, num_shared, renormalize, topk_ids, topk_w, status, hidden, hidden_row_bytes);
  if (vpl <= 8) return launch_vpl<8>(l, logits, T, E_routed, topk, num_shared, renormalize, topk_ids, topk_w, status, hidden, hidden_row_bytes);
  if (vpl <= 16) return launch_vpl<16>(l, logits, T, E_routed, topk, num_shared, renormalize, topk_ids, topk_w, status, hidden, hidden_row_bytes);
  return launch_vpl<32>(l, logits, T, E_routed, topk, num_shared, renormalize, topk_ids, topk_w, status, hidden, hidden_row_bytes);
}

}  // namespace moe
