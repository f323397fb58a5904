// Step 5 of the layer: deterministic combine back to token order.
//
// out[t, h] = sum_{j=0}^{k'-1} y[t*k' + j, h], where y already carries the routing
// weight (GEMM2 epilogue). The sum runs in slot order j = 0, 1, ..., k'-1 in fp32 and is
// rounded once to bf16, so the result does not depend on scheduling. The output is bf16
// of the hidden shape ("FlashInfer TRTLLM-Gen MoE kernel optimisation: NemotronH
// support", sglang PR 21321, section 1: the fused op returns a bf16 tensor shaped like
// hidden_states).
//
// HBM-bound: each thread owns 8 consecutive columns of one token, reads k' 16-byte
// vectors and writes one.
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kCombineThreads = 256;

__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(const uint4* __restrict__ y, int T, int k_total, int H8, uint4* __restrict__ out) {
  griddep_wait();
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long long>(T) * H8) return;
  const long long t = idx / H8;
  const int c = static_cast<int>(idx - t * H8);
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  const uint4* src = y + t * k_total * H8 + c;
  for (int j = 0; j < k_total; ++j) {
    const uint4 v = __ldcs(src + static_cast<long long>(j) * H8);  // read once: streaming
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(b[i]);
      acc[2 * i] += f.x;
      acc[2 * i + 1] += f.y;
    }
  }
  uint4 o;
  o.x = pack_bf16x2(acc[0], acc[1]);
  o.y = pack_bf16x2(acc[2], acc[3]);
  o.z = pack_bf16x2(acc[4], acc[5]);
  o.w = pack_bf16x2(acc[6], acc[7]);
  out[idx] = o;
}

}  // namespace

cudaError_t launch_combine(const Launch& l, const void* y, int T, int k_total, int H, void* out) {
  const int H8 = H / 8;
  const long long n = static_cast<long long>(T) * H8;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(static_cast<unsigned>((n + kCombineThreads - 1) / kCombineThreads)),
                     dim3(kCombineThreads), 0);
  return cudaLaunchKernelEx(&cfg, combine_kernel, static_cast<const uint4*>(y), T, k_total, H8,
                            static_cast<uint4*>(out));
}

}  // namespace moe
