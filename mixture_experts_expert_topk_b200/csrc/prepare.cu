// Load-time weight preparation (not part of the timed forward).
//
// "FlashInfer TRTLLM-Gen MoE kernel optimisation: NemotronH support" (sglang PR 21321),
// section 2: the intermediate size is zero-padded up to a multiple of 16 (gated) or 128
// (non-gated), and for gated layers the gate/up rows of w13 are reordered for the fused
// activation GEMM. "[MoE] SwiGLU fusion into the MoE up-GEMM epilogue" (sglang PR 32944),
// section 3, fixes the order: [gate0, up0, gate1, up1, ...].
//
// Reading of the padding for gated layers: each half is padded on its own (gate rows
// [0, I_in) then zeros, up rows then zeros), so the interleaved row 2j holds gate j and
// row 2j+1 holds up j for every j < I_pad, with zeros for j >= I_in.
//
// Input w13 [E, up_mult*I_in, H] (gate rows first), output [E, N1, H]; input w2
// [E, H, I_in], output [E, H, I_pad]. Elements are 1 (e4m3) or 2 (bf16) bytes.
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

// One CTA per output row of w13; 16-byte vectors (H * elt_bytes is a multiple of 256).
__global__ void prepare_w13_kernel(const uint4* __restrict__ in, uint4* __restrict__ out, int I_in,
                                   int I_pad, int N1, int row_vecs, int gated) {
  griddep_wait();
  const long long orow = blockIdx.x;  // e * N1 + n
  const long long e = orow / N1;
  const int n = static_cast<int>(orow - e * N1);
  long long src = -1;
  if (gated) {
    const int j = n >> 1, half = n & 1;
    if (j < I_in) src = e * 2LL * I_in + static_cast<long long>(half) * I_in + j;
  } else if (n < I_in) {
    src = e * static_cast<long long>(I_in) + n;
  }
  uint4* dst = out + orow * row_vecs;
  for (int c = threadIdx.x; c < row_vecs; c += blockDim.x)
    dst[c] = src >= 0 ? in[src * row_vecs + c] : make_uint4(0, 0, 0, 0);
}

// One thread per output element (the row length I_in need not be vector aligned).
template <typename T>
__global__ void prepare_w2_kernel(const T* __restrict__ in, T* __restrict__ out, long long rows,
                                  int I_in, int I_pad) {
  griddep_wait();
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= rows * I_pad) return;
  const long long r = idx / I_pad;
  const int i = static_cast<int>(idx - r * I_pad);
  out[idx] = i < I_in ? in[r * I_in + i] : T(0);
}

}  // namespace

cudaError_t launch_prepare_w13(const Launch& l, const void* in, void* out, int E, int I_in, int I_pad,
                               int H, int gated, int elt_bytes) {
  const int N1 = gated ? 2 * I_pad : I_pad;
  const int row_vecs = H * elt_bytes / 16;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(static_cast<unsigned>(static_cast<long long>(E) * N1)),
                     dim3(128), 0);
  return cudaLaunchKernelEx(&cfg, prepare_w13_kernel, static_cast<const uint4*>(in),
                            static_cast<uint4*>(out), I_in, I_pad, N1, row_vecs, gated);
}

cudaError_t launch_prepare_w2(const Launch& l, const void* in, void* out, int E, int H, int I_in,
                              int I_pad, int elt_bytes) {
  const long long rows = static_cast<long long>(E) * H;
  const long long n = rows * I_pad;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0);
  if (elt_bytes == 2)
    return cudaLaunchKernelEx(&cfg, prepare_w2_kernel<uint16_t>, static_cast<const uint16_t*>(in),
                              static_cast<uint16_t*>(out), rows, I_in, I_pad);
  return cudaLaunchKernelEx(&cfg, prepare_w2_kernel<uint8_t>, static_cast<const uint8_t*>(in),
                            static_cast<uint8_t*>(out), rows, I_in, I_pad);
}

}  // namespace moe
