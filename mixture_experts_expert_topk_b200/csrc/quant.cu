// FP8 E4M3 quantisers for the W8A8 block-128 configuration ("Qwen3-Next FP8 MoE
// optimisation: shared-expert fusion for H200", sglang PR 26204, section 1:
// dtype=fp8_w8a8, block_shape=[128, 128]).
//
//   activations: one fp32 scale per token per 128 consecutive columns (1x128 groups);
//   weights:     one fp32 scale per 128x128 block.
// In both, scale = amax / 448 (IEEE fp32 division), or 1 for an all-zero group, and
// code = e4m3(x / scale) with IEEE fp32 division, round to nearest even, saturating at
// +-448 (cvt ... .satfinite). The oracle takes the same decisions in the same
// precision, so the codes and scales are compared bit for bit.
#include <cuda_fp8.h>

#include <algorithm>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// One warp per (row, 128-column group): lane l quantises columns 4l..4l+3. When
// `num_blocks` is given, only the first num_blocks[0] * block_m rows are processed.
__global__ void __launch_bounds__(256)
    quant_act_kernel(const uint2* __restrict__ x, int T, int G, uint32_t* __restrict__ q,
                     float* __restrict__ scale, const int* __restrict__ num_blocks, int block_m) {
  griddep_wait();
  griddep_launch_dependents();
  const long long g = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const long long rows = num_blocks != nullptr ? static_cast<long long>(*num_blocks) * block_m : T;
  if (g >= rows * G) return;
  const int lane = threadIdx.x & 31;
  const uint2 raw = x[g * 32 + lane];
  const float2 f01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
  const float2 f23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
  float amax = fmaxf(fmaxf(fabsf(f01.x), fabsf(f01.y)), fmaxf(fabsf(f23.x), fabsf(f23.y)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
  q[g * 32 + lane] = e4m3x4(__fdiv_rn(f01.x, s), __fdiv_rn(f01.y, s), __fdiv_rn(f23.x, s),
                            __fdiv_rn(f23.y, s));
  if (lane == 0) scale[g] = s;
}

// One CTA of 256 threads per 128x128 block: thread t covers 64 columns of row t/2.
__global__ void __launch_bounds__(256)
    quant_weights_kernel(const uint4* __restrict__ w, int rows, int cols, uint2* __restrict__ q,
                         float* __restrict__ scale) {
  __shared__ float red[8];
  griddep_wait();
  const int rb = rows / 128, cb = cols / 128;
  const long long blk = blockIdx.x;
  const long long mat = blk / (static_cast<long long>(rb) * cb);
  const int rem = static_cast<int>(blk - mat * rb * cb);
  const int bi = rem / cb, bj = rem - (rem / cb) * cb;
  const int r = bi * 128 + (threadIdx.x >> 1);
  const int c0 = bj * 128 + (threadIdx.x & 1) * 64;
  const long long base = (mat * rows + r) * static_cast<long long>(cols) + c0;  // element index
  float v[64];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint4 u = w[base / 8 + i];
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(b[k]);
      v[8 * i + 2 * k] = f.x;
      v[8 * i + 2 * k + 1] = f.y;
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 64; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
  const float s = amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint2 o;
    o.x = e4m3x4(__fdiv_rn(v[8 * i + 0], s), __fdiv_rn(v[8 * i + 1], s), __fdiv_rn(v[8 * i + 2], s),
                 __fdiv_rn(v[8 * i + 3], s));
    o.y = e4m3x4(__fdiv_rn(v[8 * i + 4], s), __fdiv_rn(v[8 * i + 5], s), __fdiv_rn(v[8 * i + 6], s),
                 __fdiv_rn(v[8 * i + 7], s));
    q[base / 8 + i] = o;
  }
  if (threadIdx.x == 0) scale[blk] = s;
}

// Per-tensor weights ("FlashInfer TRTLLM-Gen MoE kernel optimisation: NemotronH support",
// section 1: the per-tensor FP8 variant, one fp32 scale per weight tensor). Pass 1: amax
// of each matrix into amax_bits[mat] (non-negative floats order like their bit patterns,
// so an integer max is a float max); pass 2: scale = amax / 448 (1 for all zeros) and
// codes; pass 3: the scales replace the amax bits.
__global__ void amax_per_matrix_kernel(const uint4* __restrict__ w, long long mat_vecs, int* __restrict__ amax_bits) {
  griddep_wait();
  const long long mat = blockIdx.y;
  float amax = 0.f;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < mat_vecs;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint4 u = w[mat * mat_vecs + i];
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(b[k]);
      amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits + mat, __float_as_int(amax));
}

__device__ __forceinline__ float scale_of(int amax_bits) {
  const float amax = __int_as_float(amax_bits);
  return amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
}

__global__ void quant_per_matrix_kernel(const uint4* __restrict__ w, long long mat_vecs, const int* __restrict__ amax_bits,
                                        uint2* __restrict__ q) {
  const long long mat = blockIdx.y;
  const float s = scale_of(amax_bits[mat]);
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < mat_vecs;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint4 u = w[mat * mat_vecs + i];
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
    float v[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(b[k]);
      v[2 * k] = f.x;
      v[2 * k + 1] = f.y;
    }
    uint2 o;
    o.x = e4m3x4(__fdiv_rn(v[0], s), __fdiv_rn(v[1], s), __fdiv_rn(v[2], s), __fdiv_rn(v[3], s));
    o.y = e4m3x4(__fdiv_rn(v[4], s), __fdiv_rn(v[5], s), __fdiv_rn(v[6], s), __fdiv_rn(v[7], s));
    q[mat * mat_vecs + i] = o;
  }
}

__global__ void scales_from_amax_kernel(int* __restrict__ amax_bits, long long num_mats) {
  const long long m = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (m < num_mats) amax_bits[m] = __float_as_int(scale_of(amax_bits[m]));
}

// MXFP8 weights (OCP Microscaling v1.0, block 32 along the row): one thread per block,
// 64 bytes of bf16 in, 32 code bytes and one E8M0 scale byte out. The MXFP8 weight
// scales of "FlashInfer TRTLLM-Gen MoE kernel optimisation: NemotronH support" (section 2,
// the MXFP8 alignment helper) hold one scale per 32 values of K.
__global__ void __launch_bounds__(256)
    quant_mx_rows_kernel(const uint4* __restrict__ w, long long blocks, uint4* __restrict__ codes,
                         uint8_t* __restrict__ scales) {
  griddep_wait();
  for (long long b = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; b < blocks;
       b += static_cast<long long>(gridDim.x) * blockDim.x) {
    float v[32];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 raw = w[b * 4 + i];
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __bfloat1622float2(h[k]);
        v[8 * i + 2 * k] = f.x;
        v[8 * i + 2 * k + 1] = f.y;
      }
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const int e = mx_exponent(amax);
    const float inv = mx_inv(e);
    uint32_t c[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) c[i] = mx_e4m3x4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3], inv);
    codes[b * 2] = make_uint4(c[0], c[1], c[2], c[3]);
    codes[b * 2 + 1] = make_uint4(c[4], c[5], c[6], c[7]);
    scales[b] = static_cast<uint8_t>(e + 127);
  }
}

// NVFP4 ("FlashInfer gated MoE kernel optimisation for Blackwell", section 4, names NVFP4
// weights; the format is NVIDIA's: E2M1 values, an E4M3 scale per 16 values, an fp32 scale
// per tensor). One thread per block of 16 values along a row: 32 bytes of bf16 in, 8 code
// bytes (two values per byte, the lower K index in the low nibble) and one scale byte out.
// The tensor scale is g_static, or (amax_bits != nullptr) amax / (6 * 448) of the block's
// matrix, from pass 1 of the per-tensor path (amax_per_matrix_kernel).
__global__ void __launch_bounds__(256)
    quant_nvfp4_rows_kernel(const uint4* __restrict__ w, long long blocks, long long blocks_per_mat,
                            const int* __restrict__ amax_bits, float g_static, uint2* __restrict__ codes,
                            uint8_t* __restrict__ scales) {
  griddep_wait();
  griddep_launch_dependents();
  for (long long b = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; b < blocks;
       b += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float g = amax_bits != nullptr ? nvfp4_tensor_scale(__int_as_float(amax_bits[b / blocks_per_mat])) : g_static;
    float v[16];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint4 raw = w[b * 2 + i];
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __bfloat1622float2(h[k]);
        v[8 * i + 2 * k] = f.x;
        v[8 * i + 2 * k + 1] = f.y;
      }
    }
    uint2 packed;
    scales[b] = nvfp4_block(v, g, packed);
    codes[b] = packed;
  }
}

__global__ void nvfp4_scales_from_amax_kernel(int* __restrict__ amax_bits, long long num_mats) {
  const long long m = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (m < num_mats) amax_bits[m] = __float_as_int(nvfp4_tensor_scale(__int_as_float(amax_bits[m])));
}

}  // namespace

cudaError_t launch_quant_weights_nvfp4(const Launch& l, const void* w, int64_t num_mats, int64_t mat_elems,
                                       void* codes, void* scales, float* global_scales) {
  if (mat_elems % 16 != 0 || num_mats <= 0 || num_mats > 65535) return cudaErrorInvalidValue;
  const long long vecs = mat_elems / 8;
  int* bits = reinterpret_cast<int*>(global_scales);
  cudaError_t err = cudaMemsetAsync(bits, 0, static_cast<size_t>(num_mats) * sizeof(int), l.stream);
  if (err != cudaSuccess) return err;
  const unsigned bx = static_cast<unsigned>(std::min<long long>((vecs + 255) / 256, 1024));
  amax_per_matrix_kernel<<<dim3(bx, static_cast<unsigned>(num_mats)), 256, 0, l.stream>>>(
      static_cast<const uint4*>(w), vecs, bits);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  const long long blocks = num_mats * (mat_elems / 16);
  quant_nvfp4_rows_kernel<<<static_cast<unsigned>(std::min<long long>((blocks + 255) / 256, 8192)), 256, 0,
                            l.stream>>>(static_cast<const uint4*>(w), blocks, mat_elems / 16, bits, 1.0f,
                                        static_cast<uint2*>(codes), static_cast<uint8_t*>(scales));
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  nvfp4_scales_from_amax_kernel<<<static_cast<unsigned>((num_mats + 255) / 256), 256, 0, l.stream>>>(bits, num_mats);
  return cudaGetLastError();
}

cudaError_t launch_quant_rows_nvfp4(const Launch& l, const void* x, long long rows, int cols, float g, void* codes,
                                    void* scales) {
  if (cols % 16 != 0 || rows < 0) return cudaErrorInvalidValue;
  const long long blocks = rows * (cols / 16);
  if (blocks == 0) return cudaSuccess;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(static_cast<unsigned>(std::min<long long>((blocks + 255) / 256, 8192))),
                     dim3(256), 0);
  return cudaLaunchKernelEx(&cfg, quant_nvfp4_rows_kernel, static_cast<const uint4*>(x), blocks, blocks,
                            static_cast<const int*>(nullptr), g, static_cast<uint2*>(codes),
                            static_cast<uint8_t*>(scales));
}

cudaError_t launch_quant_weights_per_tensor(const Launch& l, const void* w, int64_t num_mats, int64_t mat_elems,
                                            void* codes, float* scales) {
  if (mat_elems % 8 != 0 || num_mats <= 0 || num_mats > 65535) return cudaErrorInvalidValue;
  const long long vecs = mat_elems / 8;
  int* bits = reinterpret_cast<int*>(scales);
  cudaError_t err = cudaMemsetAsync(bits, 0, static_cast<size_t>(num_mats) * sizeof(int), l.stream);
  if (err != cudaSuccess) return err;
  const unsigned bx = static_cast<unsigned>(std::min<long long>((vecs + 255) / 256, 1024));
  amax_per_matrix_kernel<<<dim3(bx, static_cast<unsigned>(num_mats)), 256, 0, l.stream>>>(
      static_cast<const uint4*>(w), vecs, bits);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  quant_per_matrix_kernel<<<dim3(bx, static_cast<unsigned>(num_mats)), 256, 0, l.stream>>>(
      static_cast<const uint4*>(w), vecs, bits, static_cast<uint2*>(codes));
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  scales_from_amax_kernel<<<static_cast<unsigned>((num_mats + 255) / 256), 256, 0, l.stream>>>(bits, num_mats);
  return cudaGetLastError();
}

cudaError_t launch_quant_act(const Launch& l, const void* x, int T, int H, void* q, float* scale) {
  const int G = H / 128;
  const long long groups = static_cast<long long>(T) * G;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(static_cast<unsigned>((groups + 7) / 8)), dim3(256), 0);
  return cudaLaunchKernelEx(&cfg, quant_act_kernel, static_cast<const uint2*>(x), T, G,
                            static_cast<uint32_t*>(q), scale, static_cast<const int*>(nullptr), 1);
}

cudaError_t launch_quant_rows(const Launch& l, const void* x, int max_rows, int cols, const int* num_blocks,
                              int block_m, void* q, float* scale) {
  const int G = cols / 128;
  const long long groups = static_cast<long long>(max_rows) * G;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(static_cast<unsigned>((groups + 7) / 8)), dim3(256), 0);
  return cudaLaunchKernelEx(&cfg, quant_act_kernel, static_cast<const uint2*>(x), max_rows, G,
                            static_cast<uint32_t*>(q), scale, num_blocks, block_m);
}

cudaError_t launch_quant_weights(const Launch& l, const void* w, int64_t num_mats, int rows, int cols,
                                 void* q, float* scale) {
  const long long blocks = num_mats * static_cast<long long>(rows / 128) * (cols / 128);
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(static_cast<unsigned>(blocks)), dim3(256), 0);
  return cudaLaunchKernelEx(&cfg, quant_weights_kernel, static_cast<const uint4*>(w), rows, cols,
                            static_cast<uint2*>(q), scale);
}

cudaError_t launch_quant_weights_mx(const Launch& l, const void* w, long long rows, int cols, void* codes,
                                    void* scales) {
  if (cols % 32 != 0 || rows < 0) return cudaErrorInvalidValue;
  const long long blocks = rows * (cols / 32);
  if (blocks == 0) return cudaSuccess;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(static_cast<unsigned>(std::min<long long>((blocks + 255) / 256, 8192))),
                     dim3(256), 0);
  return cudaLaunchKernelEx(&cfg, quant_mx_rows_kernel, static_cast<const uint4*>(w), blocks,
                            static_cast<uint4*>(codes), static_cast<uint8_t*>(scales));
}

}  // namespace moe
