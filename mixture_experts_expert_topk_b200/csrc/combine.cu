// Step 5 of the layer: deterministic combine back to token order.
//
// out[t, h] = sum_{j=0}^{k'-1} w_tj * y[pair_to_row[t*k' + j], h], y in sorted row order
// (GEMM2's output). The sum runs in slot order j = 0, 1, ..., k'-1 in fp32 and is rounded
// once to bf16, so the result does not depend on scheduling. The output is bf16 of the hidden shape ("FlashInfer TRTLLM-Gen MoE kernel
// optimisation: NemotronH support", sglang PR 21321, section 1: the fused op returns a
// bf16 tensor shaped like hidden_states).
//
// y comes in one of two formats: fp32 rows already weighted (the 128-row token-tile GEMMs),
// or unweighted fp16 rows with one power-of-two exponent per 32 columns of each row (the
// swapped-operand GEMMs), for which the combine applies the routing weight:
// out[t] = sum_j w_tj * y16_j * 2^exp_j, each product exact in fp32 but the one by w. The
// fp16 form halves the bytes of this HBM-bound pass.
//
// Each thread owns 8 consecutive columns of one token and reads k' x 32 (fp32) or k' x 17
// (fp16 + exponent) bytes, writing 16.
#include <cuda_fp16.h>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kCombineThreads = 256;

__global__ void __launch_bounds__(kCombineThreads)
    combine_f32_kernel(const float4* __restrict__ y, const int* __restrict__ pair_to_row, int T, int k_total, int H8,
                       uint4* __restrict__ out) {
  griddep_wait();
  griddep_launch_dependents();
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long long>(T) * H8) return;
  const long long t = idx / H8;
  const int c = static_cast<int>(idx - t * H8);
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  const int* rows = pair_to_row + t * k_total;
  for (int j = 0; j < k_total; ++j) {
    // columns 8c..8c+7 of y row pair_to_row[t*k' + j] = float4 pair 2c, 2c+1 of that row
    const float4* src = y + (static_cast<long long>(__ldg(rows + j)) * H8 + c) * 2;
    const float4 a = __ldcs(src);  // read once: streaming
    const float4 b = __ldcs(src + 1);
    acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
    acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
  }
  uint4 o;
  o.x = pack_bf16x2(acc[0], acc[1]);
  o.y = pack_bf16x2(acc[2], acc[3]);
  o.z = pack_bf16x2(acc[4], acc[5]);
  o.w = pack_bf16x2(acc[6], acc[7]);
  out[idx] = o;
}

__global__ void __launch_bounds__(kCombineThreads)
    combine_f16_kernel(const uint4* __restrict__ y, const int8_t* __restrict__ y_exp, const float* __restrict__ topk_w,
                       const int* __restrict__ pair_to_row, int T, int k_total, int H8, uint4* __restrict__ out) {
  griddep_wait();
  griddep_launch_dependents();
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long long>(T) * H8) return;
  const long long t = idx / H8;
  const int c = static_cast<int>(idx - t * H8);
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  const int* rows = pair_to_row + t * k_total;
  const float* w = topk_w + t * k_total;
  const int H32 = H8 >> 2;  // exponents per row
  for (int j = 0; j < k_total; ++j) {
    const long long r = __ldg(rows + j);
    const uint4 v = __ldcs(y + r * H8 + c);  // columns 8c..8c+7, read once: streaming
    const int s = __ldg(y_exp + r * H32 + (c >> 2));
    const float scale = __ldg(w + j) * __int_as_float((127 + s) << 23);  // w * 2^s, s in [-100, 113]
    const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(h[i]);
      acc[2 * i] += f.x * scale;
      acc[2 * i + 1] += f.y * scale;
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

cudaError_t launch_combine(const Launch& l, const void* y, const int8_t* y_exp, const float* topk_w,
                           const int* pair_to_row, int T, int k_total, int H, void* out) {
  const int H8 = H / 8;
  const long long n = static_cast<long long>(T) * H8;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(static_cast<unsigned>((n + kCombineThreads - 1) / kCombineThreads)),
                     dim3(kCombineThreads), 0);
  if (y_exp != nullptr) {
    if (H % 32 != 0 || topk_w == nullptr) return cudaErrorInvalidValue;
    return cudaLaunchKernelEx(&cfg, combine_f16_kernel, static_cast<const uint4*>(y), y_exp, topk_w, pair_to_row, T,
                              k_total, H8, static_cast<uint4*>(out));
  }
  return cudaLaunchKernelEx(&cfg, combine_f32_kernel, static_cast<const float4*>(y), pair_to_row, T, k_total, H8,
                            static_cast<uint4*>(out));
}

}  // namespace moe
