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
//
// For the bf16 GEMMs that take the weights as the MMA's M operand (gemm_swap.cu) the same
// padded, interleaved matrices are stored tiled instead: tile (expert e, 128-row block m,
// 64-column chunk c) of 16 KB at ((e * MT + m) * KC + c) * 16 KB, MT = ceil(rows / 128),
// KC = ceil(K / 64); row r of a tile is 128 contiguous bytes whose 16-byte piece q sits at
// position q ^ (r % 8) (the 128-byte swizzle of the MMA's shared-memory operand); rows and
// columns past the matrix are zero.
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

// One thread per 16-byte piece of the tiled output. which = 0: w13 (rows N1, K = H; row n
// from the checkpoint row of gate/up index n / 2 (gated) or n); which = 1: w2 (rows H,
// K = I_pad; columns >= I_in zero).
__global__ void tile_weights_kernel(const uint16_t* __restrict__ in, uint4* __restrict__ out, long long pieces,
                                    int which, int rows, int MT, int KC, int H, int I_in, int gated) {
  griddep_wait();
  for (long long o = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; o < pieces;
       o += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long t = o >> 10;  // 1024 pieces per 16 KB tile
    const int rr = static_cast<int>((o >> 3) & 127);
    const int q = static_cast<int>(o & 7) ^ (rr & 7);  // logical piece stored at this position
    const int c = static_cast<int>(t % KC);
    const long long tm = t / KC;
    const int m = static_cast<int>(tm % MT);
    const long long e = tm / MT;
    const int r = m * 128 + rr;
    const int k0 = c * 64 + q * 8;
    long long src = -1;  // source row
    int ld = H, kvalid = H;
    if (r < rows) {
      if (which == 0) {
        if (gated) {
          const int j = r >> 1, half = r & 1;
          if (j < I_in) src = e * 2LL * I_in + static_cast<long long>(half) * I_in + j;
        } else if (r < I_in) {
          src = e * static_cast<long long>(I_in) + r;
        }
      } else {
        src = e * static_cast<long long>(H) + r;
        ld = I_in;
        kvalid = I_in;
      }
    }
    uint16_t v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = (src >= 0 && k0 + i < kvalid) ? in[src * ld + k0 + i] : uint16_t(0);
    uint4 w;
    w.x = v[0] | (static_cast<uint32_t>(v[1]) << 16);
    w.y = v[2] | (static_cast<uint32_t>(v[3]) << 16);
    w.z = v[4] | (static_cast<uint32_t>(v[5]) << 16);
    w.w = v[6] | (static_cast<uint32_t>(v[7]) << 16);
    out[o] = w;
  }
}

// The tiled layout for e4m3 codes: a 128-byte chunk row holds 128 elements, so tile
// (e, m, c) covers rows [128m, 128m + 128) and columns [128c, 128c + 128). FP8 requires
// I == I_in (a multiple of 128): only the gate/up interleave of w13 moves rows.
__global__ void tile_weights_u8_kernel(const uint4* __restrict__ in, uint4* __restrict__ out, long long pieces,
                                       int which, int rows, int MT, int KC, int K, int I, int gated) {
  griddep_wait();
  for (long long o = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; o < pieces;
       o += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long t = o >> 10;
    const int rr = static_cast<int>((o >> 3) & 127);
    const int q = static_cast<int>(o & 7) ^ (rr & 7);
    const int c = static_cast<int>(t % KC);
    const long long tm = t / KC;
    const int m = static_cast<int>(tm % MT);
    const long long e = tm / MT;
    const int r = m * 128 + rr;
    const int k0 = c * 128 + q * 16;
    long long src = -1;
    if (r < rows) {
      if (which == 0 && gated) {
        const int j = r >> 1, half = r & 1;
        src = e * 2LL * I + static_cast<long long>(half) * I + j;
      } else {
        src = e * static_cast<long long>(rows) + r;
      }
    }
    out[o] = (src >= 0 && k0 < K) ? in[(src * K + k0) / 16] : make_uint4(0u, 0u, 0u, 0u);
  }
}

// MXFP8 weight scales beside the tiled codes: tile (e, m, c) (128 rows, 128 columns of K)
// has a 512-byte block whose byte 16 l + 4 j + k is the E8M0 scale of tile row 32 j + l for
// K block 4 c + k, the order in which tcgen05.cp (32 lanes x 16 bytes, replicated to the
// four lane quadrants) leaves row r's scale for K block k in TMEM lane r % 32, column
// r / 32, byte k: where the block-scaled MMA reads it. Rows follow the code tiles (gate
// and up interleaved for w13 of a gated layer); rows or K blocks past the matrix take 0.
__global__ void tile_scales_mx_kernel(const uint8_t* __restrict__ in, uint8_t* __restrict__ out, long long bytes,
                                      int which, int rows, int MT, int KC, int KB, int I, int gated) {
  griddep_wait();
  for (long long o = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; o < bytes;
       o += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long t = o >> 9;
    const int b = static_cast<int>(o & 511);
    const int l = b >> 4, j = (b >> 2) & 3, k = b & 3;
    const int c = static_cast<int>(t % KC);
    const long long tm = t / KC;
    const int m = static_cast<int>(tm % MT);
    const long long e = tm / MT;
    const int r = m * 128 + 32 * j + l;
    const int kb = 4 * c + k;
    long long src = -1;
    if (r < rows) {
      if (which == 0 && gated) {
        src = e * 2LL * I + static_cast<long long>(r & 1) * I + (r >> 1);
      } else {
        src = e * static_cast<long long>(rows) + r;
      }
    }
    out[o] = (src >= 0 && kb < KB) ? in[src * KB + kb] : static_cast<uint8_t>(0);
  }
}

// NVFP4 weight scales beside the tiled codes: tile (e, m, c) (128 rows, 256 values of K in
// one 128-byte chunk row) has a 2048-byte block of four 512-byte blocks, one per MMA of
// K = 64: byte 512 mm + 16 l + 4 j + k is the E4M3 scale of tile row 32 j + l for the
// 16-value block 16 c + 4 mm + k. tcgen05.cp (32 lanes x 16 bytes, replicated to the four
// lane quadrants) leaves MMA mm's scales of row r in TMEM lane r % 32, column r / 32 of its
// four columns, byte k = the row's block k of that MMA's 64 values: where the block-scaled
// MMA with scale_vec::4X reads them. Rows follow the code tiles (gate and up interleaved for
// w13 of a gated layer); rows or blocks past the matrix take 0.
__global__ void tile_scales_nvfp4_kernel(const uint8_t* __restrict__ in, uint8_t* __restrict__ out, long long bytes,
                                         int which, int rows, int MT, int KC, int KB, int I, int gated) {
  griddep_wait();
  for (long long o = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; o < bytes;
       o += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long t = o >> 11;
    const int b = static_cast<int>(o & 2047);
    const int mm = b >> 9, l = (b >> 4) & 31, j = (b >> 2) & 3, k = b & 3;
    const int c = static_cast<int>(t % KC);
    const long long tm = t / KC;
    const int m = static_cast<int>(tm % MT);
    const long long e = tm / MT;
    const int r = m * 128 + 32 * j + l;
    const int kb = 16 * c + 4 * mm + k;
    long long src = -1;
    if (r < rows) {
      if (which == 0 && gated) {
        src = e * 2LL * I + static_cast<long long>(r & 1) * I + (r >> 1);
      } else {
        src = e * static_cast<long long>(rows) + r;
      }
    }
    out[o] = (src >= 0 && kb < KB) ? in[src * KB + kb] : static_cast<uint8_t>(0);
  }
}

}  // namespace

size_t tiled_scale_bytes_nvfp4(int E, int rows, int K) {
  return static_cast<size_t>(E) * ((rows + 127) / 128) * ((K + 255) / 256) * kNvChunkScaleBytes;
}

cudaError_t launch_tile_scales_nvfp4(const Launch& l, int which, const void* in, void* out, int E, int H, int I,
                                     int gated) {
  const int rows = which == 0 ? (gated ? 2 * I : I) : H;
  const int K = which == 0 ? H : I;
  if (K % 16 != 0) return cudaErrorInvalidValue;
  const int MT = (rows + 127) / 128, KC = (K + 255) / 256;
  const long long bytes = static_cast<long long>(tiled_scale_bytes_nvfp4(E, rows, K));
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(4096), dim3(256), 0);
  return cudaLaunchKernelEx(&cfg, tile_scales_nvfp4_kernel, static_cast<const uint8_t*>(in),
                            static_cast<uint8_t*>(out), bytes, which, rows, MT, KC, K / 16, I, gated);
}

size_t tiled_weight_bytes_u8(int E, int rows, int K) {
  return static_cast<size_t>(E) * ((rows + 127) / 128) * ((K + 127) / 128) * 16384;
}

cudaError_t launch_tile_weights_u8(const Launch& l, int which, const void* in, void* out, int E, int H, int I,
                                   int gated, int k_div) {
  const int rows = which == 0 ? (gated ? 2 * I : I) : H;
  const int K = (which == 0 ? H : I) / k_div;  // bytes per row: packed E2M1 holds two values per byte
  if (K % 16 != 0) return cudaErrorInvalidValue;
  const int MT = (rows + 127) / 128, KC = (K + 127) / 128;
  const long long pieces = static_cast<long long>(tiled_weight_bytes_u8(E, rows, K) / 16);
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(4096), dim3(256), 0);
  return cudaLaunchKernelEx(&cfg, tile_weights_u8_kernel, static_cast<const uint4*>(in), static_cast<uint4*>(out),
                            pieces, which, rows, MT, KC, K, I, gated);
}

size_t tiled_weight_bytes(int E, int rows, int K) {
  return static_cast<size_t>(E) * ((rows + 127) / 128) * ((K + 63) / 64) * 16384;
}

cudaError_t launch_tile_weights(const Launch& l, int which, const void* in, void* out, int E, int H, int I_in,
                                int I_pad, int gated) {
  const int rows = which == 0 ? (gated ? 2 * I_pad : I_pad) : H;
  const int K = which == 0 ? H : I_pad;
  const int MT = (rows + 127) / 128, KC = (K + 63) / 64;
  const long long pieces = static_cast<long long>(tiled_weight_bytes(E, rows, K) / 16);
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(4096), dim3(256), 0);
  return cudaLaunchKernelEx(&cfg, tile_weights_kernel, static_cast<const uint16_t*>(in), static_cast<uint4*>(out),
                            pieces, which, rows, MT, KC, H, I_in, gated);
}

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

size_t tiled_scale_bytes_mx(int E, int rows, int K) {
  return static_cast<size_t>(E) * ((rows + 127) / 128) * ((K + 127) / 128) * 512;
}

cudaError_t launch_tile_scales_mx(const Launch& l, int which, const void* in, void* out, int E, int H, int I,
                                  int gated) {
  const int rows = which == 0 ? (gated ? 2 * I : I) : H;
  const int K = which == 0 ? H : I;
  if (K % 32 != 0) return cudaErrorInvalidValue;
  const int MT = (rows + 127) / 128, KC = (K + 127) / 128;
  const long long bytes = static_cast<long long>(tiled_scale_bytes_mx(E, rows, K));
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(2048), dim3(256), 0);
  return cudaLaunchKernelEx(&cfg, tile_scales_mx_kernel, static_cast<const uint8_t*>(in),
                            static_cast<uint8_t*>(out), bytes, which, rows, MT, KC, K / 32, I, gated);
}

}  // namespace moe
