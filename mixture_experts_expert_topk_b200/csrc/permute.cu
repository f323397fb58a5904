// GEMM1's token rows in the row-group order of the swapped-operand GEMM (gemm_swap.cu).
//
// For each row group (x_row, n) of align's output, row j of the group is the hidden row of
// its pair's token, hidden[sorted_pair_ids[x_row + j] / k']; padding rows are not written
// (GEMM1 stores zeros for them whatever they hold, since an MMA output column depends only on
// its own X column).
// The group occupies bytes [x_row * H * 2, (x_row + n) * H * 2) of xs; 64-column chunk c of
// it is n rows of 128 bytes at offset c * n * 128, the 16-byte piece q of row j stored at
// position q ^ (j % 8) (the 128-byte swizzle the MMA reads). The GEMM then loads each K
// step of a group with one contiguous bulk copy.
//
// A CTA copies a 32-row slice of a row group; each warp two rows at a time, each lane with
// sixteen 16-byte loads of the hidden rows in flight (coalesced) before writing them to
// their chunk rows.
#include <cuda_fp8.h>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kRowsPerStep = 2;    // rows a warp copies at once
constexpr int kPiecesPerLane = 8;  // 16-byte pieces per lane per row and step
constexpr int kRowsPerCta = 32;    // rows of a group per CTA (grid.y covers 256 / 32 slices)

__global__ void __launch_bounds__(kThreads)
    permute_rows_kernel(const uint4* __restrict__ hidden, int row_pieces, const int* __restrict__ sorted_pair_ids,
                        const int* __restrict__ num_groups, const int2* __restrict__ group_info, int P, int k_total,
                        uint8_t* __restrict__ xs) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int G = *num_groups;
  // CTA (x, y) copies rows [kRowsPerCta * y, kRowsPerCta * (y + 1)) of groups x, x + gridDim.x, ...
  for (int g = blockIdx.x; g < G; g += gridDim.x) {
    const int2 gi = group_info[g];
    const int x_row = gi.x, n = group_word_rows(gi.y);
    uint8_t* base = xs + static_cast<size_t>(x_row) * row_pieces * 16;
    for (int j0 = kRowsPerCta * blockIdx.y + kRowsPerStep * warp; j0 < min(n, kRowsPerCta * (blockIdx.y + 1));
         j0 += kRowsPerStep * (kThreads / 32)) {
      const uint4* src[kRowsPerStep];
#pragma unroll
      for (int r = 0; r < kRowsPerStep; ++r) {
        const int pid = j0 + r < n ? sorted_pair_ids[x_row + j0 + r] : P;
        src[r] = pid < P ? hidden + static_cast<size_t>(pid / k_total) * row_pieces : nullptr;
      }
      for (int p0 = lane; p0 < row_pieces; p0 += 32 * kPiecesPerLane) {
        // kRowsPerStep x kPiecesPerLane 16-byte loads in flight per lane before the stores
        uint4 v[kRowsPerStep][kPiecesPerLane];
#pragma unroll
        for (int r = 0; r < kRowsPerStep; ++r)
#pragma unroll
          for (int i = 0; i < kPiecesPerLane; ++i) {
            const int p = p0 + 32 * i;
            v[r][i] = (src[r] != nullptr && p < row_pieces) ? __ldg(src[r] + p) : make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
        for (int r = 0; r < kRowsPerStep; ++r) {
          const int j = j0 + r;
          if (j >= n || src[r] == nullptr) continue;  // padding rows are not written
#pragma unroll
          for (int i = 0; i < kPiecesPerLane; ++i) {
            const int p = p0 + 32 * i;
            if (p < row_pieces) {
              const int c = p >> 3, q = p & 7;
              *reinterpret_cast<uint4*>(base + static_cast<size_t>(c) * n * 128 + j * 128 + ((q ^ (j & 7)) << 4)) =
                  v[r][i];
            }
          }
        }
      }
    }
  }
}


// Per-tensor FP8: the same row-group order with each element quantised on the way,
// e4m3(x * inv_scale), inv_scale = fp32(1 / input_scale) (the per-tensor variant scales
// by the reciprocal: "FlashInfer TRTLLM-Gen MoE kernel optimisation: NemotronH support",
// section 2), round to nearest, saturating at 448; a chunk is 128 elements (128 bytes).
// Piece p of a row is elements [16p, 16p + 16); a warp converts two rows at a time, each
// lane four pieces per row, all loads issued before the conversions.
constexpr int kQPieces = 4;
__global__ void __launch_bounds__(kThreads)
    permute_quant_rows_kernel(const uint4* __restrict__ hidden, int H, const int* __restrict__ sorted_pair_ids,
                              const int* __restrict__ num_groups, const int2* __restrict__ group_info, int P,
                              int k_total, float inv_scale, uint8_t* __restrict__ xs) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int G = *num_groups;
  const int pieces = H / 16;  // 16 elements: 32 bytes in, 16 bytes out
  for (int g = blockIdx.x; g < G; g += gridDim.x) {
    const int2 gi = group_info[g];
    const int x_row = gi.x, n = group_word_rows(gi.y);
    uint8_t* base = xs + static_cast<size_t>(x_row) * H;
    for (int j0 = kRowsPerCta * blockIdx.y + kRowsPerStep * warp; j0 < min(n, kRowsPerCta * (blockIdx.y + 1));
         j0 += kRowsPerStep * (kThreads / 32)) {
      const uint4* src[kRowsPerStep];
#pragma unroll
      for (int r = 0; r < kRowsPerStep; ++r) {
        const int pid = j0 + r < n ? sorted_pair_ids[x_row + j0 + r] : P;
        src[r] = pid < P ? hidden + static_cast<size_t>(pid / k_total) * (H / 8) : nullptr;
      }
      for (int p0 = lane; p0 < pieces; p0 += 32 * kQPieces) {
        uint4 in[kRowsPerStep][kQPieces][2];
#pragma unroll
        for (int r = 0; r < kRowsPerStep; ++r)
#pragma unroll
          for (int i = 0; i < kQPieces; ++i) {
            const int p = p0 + 32 * i;
            const bool ok = src[r] != nullptr && p < pieces;
            in[r][i][0] = ok ? __ldg(src[r] + 2 * p) : make_uint4(0u, 0u, 0u, 0u);
            in[r][i][1] = ok ? __ldg(src[r] + 2 * p + 1) : make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
        for (int r = 0; r < kRowsPerStep; ++r) {
          const int j = j0 + r;
          if (j >= n || src[r] == nullptr) continue;  // padding rows are not written
#pragma unroll
          for (int i = 0; i < kQPieces; ++i) {
            const int p = p0 + 32 * i;
            if (p >= pieces) continue;
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(in[r][i]);
            uint32_t o[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float2 a = __bfloat1622float2(h2[2 * k]);
              const float2 b = __bfloat1622float2(h2[2 * k + 1]);
              const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a.x * inv_scale, a.y * inv_scale),
                                                           __NV_SATFINITE, __NV_E4M3);
              const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(b.x * inv_scale, b.y * inv_scale),
                                                           __NV_SATFINITE, __NV_E4M3);
              o[k] = lo | (hi << 16);
            }
            const int c = p >> 3, q = p & 7;
            *reinterpret_cast<uint4*>(base + static_cast<size_t>(c) * n * 128 + j * 128 + ((q ^ (j & 7)) << 4)) =
                make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
      }
    }
  }
}

// MXFP8: the same row-group order, each row quantised per 32 columns (OCP Microscaling
// v1.0: E8M0 exponent floor(log2(amax)) - 8, e4m3 codes of x * 2^-exponent, saturating),
// with the scale bytes laid out for the block-scaled MMA: the group starting at x_row owns
// the 1024-byte block ((x_row / 16) * H/128 + c) * 1024 of column chunk c, whose byte
// 512 h + 16 l + 4 j + k is the scale of group row 128 h + 32 j + l for K block 4 c + k.
// Lanes 2m and 2m+1 hold the two 16-column pieces of one 32-column block and exchange
// their maxima with one shuffle; every lane runs every iteration so the shuffles are
// warp-wide.
__global__ void __launch_bounds__(kThreads)
    permute_mx_rows_kernel(const uint4* __restrict__ hidden, int H, const int* __restrict__ sorted_pair_ids,
                           const int* __restrict__ num_groups, const int2* __restrict__ group_info, int P,
                           int k_total, uint8_t* __restrict__ xs, uint8_t* __restrict__ xs_sf) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int G = *num_groups;
  const int pieces = H / 16, KC = H / 128;
  for (int g = blockIdx.x; g < G; g += gridDim.x) {
    const int2 gi = group_info[g];
    const int x_row = gi.x, n = group_word_rows(gi.y);
    uint8_t* base = xs + static_cast<size_t>(x_row) * H;
    uint8_t* sf = xs_sf + static_cast<size_t>(x_row >> 4) * KC * 1024;
    for (int j0 = kRowsPerCta * blockIdx.y + kRowsPerStep * warp; j0 < min(n, kRowsPerCta * (blockIdx.y + 1));
         j0 += kRowsPerStep * (kThreads / 32)) {
      const uint4* src[kRowsPerStep];
#pragma unroll
      for (int r = 0; r < kRowsPerStep; ++r) {
        const int pid = j0 + r < n ? sorted_pair_ids[x_row + j0 + r] : P;
        src[r] = pid < P ? hidden + static_cast<size_t>(pid / k_total) * (H / 8) : nullptr;
      }
      for (int p0 = 0; p0 < pieces; p0 += 32 * kQPieces) {
        uint4 in[kRowsPerStep][kQPieces][2];
#pragma unroll
        for (int r = 0; r < kRowsPerStep; ++r)
#pragma unroll
          for (int i = 0; i < kQPieces; ++i) {
            const int p = p0 + lane + 32 * i;
            const bool ok = src[r] != nullptr && p < pieces;
            in[r][i][0] = ok ? __ldg(src[r] + 2 * p) : make_uint4(0u, 0u, 0u, 0u);
            in[r][i][1] = ok ? __ldg(src[r] + 2 * p + 1) : make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
        for (int r = 0; r < kRowsPerStep; ++r) {
          const int j = j0 + r;  // warp-uniform
#pragma unroll
          for (int i = 0; i < kQPieces; ++i) {
            const int p = p0 + lane + 32 * i;  // p and p ^ 1 are both inside the row or both past it
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(in[r][i]);
            float v[16];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const float2 f = __bfloat1622float2(h2[k]);
              v[2 * k] = f.x;
              v[2 * k + 1] = f.y;
            }
            float amax = 0.f;
#pragma unroll
            for (int k = 0; k < 16; ++k) amax = fmaxf(amax, fabsf(v[k]));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            const int e = mx_exponent(amax);
            const float inv = mx_inv(e);
            if (p < pieces && j < n && src[r] != nullptr) {  // padding rows are not written
              const int c = p >> 3, q = p & 7;
              *reinterpret_cast<uint4*>(base + static_cast<size_t>(c) * n * 128 + j * 128 + ((q ^ (j & 7)) << 4)) =
                  make_uint4(mx_e4m3x4(v[0], v[1], v[2], v[3], inv), mx_e4m3x4(v[4], v[5], v[6], v[7], inv),
                             mx_e4m3x4(v[8], v[9], v[10], v[11], inv), mx_e4m3x4(v[12], v[13], v[14], v[15], inv));
              if ((lane & 1) == 0) {
                const int b = p >> 1;  // 32-column block
                sf[static_cast<size_t>(b >> 2) * 1024 + (j >> 7) * 512 + (j & 31) * 16 + ((j >> 5) & 3) * 4 + (b & 3)] =
                    static_cast<uint8_t>(e + 127);
              }
            }
          }
        }
      }
    }
  }
}

// GEMM1's bf16 activation (row-group order, 64-column chunks of 128-byte rows) to MXFP8
// codes (128-column chunks) and scales, in the layout of permute_mx_rows_kernel, for
// GEMM2. A warp converts one row, four 128-column chunks at a time (their loads first):
// lane l takes columns 4l..4l+3 of each (8 bytes of bf16 chunk 2c + l/16), eight lanes form
// a 32-column block.
constexpr int kActChunksPerPass = 4;
__global__ void __launch_bounds__(kThreads)
    act_quant_mx_kernel(const uint8_t* __restrict__ act, int I, const int* __restrict__ num_groups,
                        const int2* __restrict__ group_info, uint8_t* __restrict__ actq,
                        uint8_t* __restrict__ act_sf) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int G = *num_groups;
  const int KCb = I / 64, KCq = I / 128;
  const int ib = 8 * (lane & 15);  // byte of the bf16 chunk row
  const int ob = 4 * lane;         // byte of the e4m3 chunk row
  for (int g = blockIdx.x; g < G; g += gridDim.x) {
    const int2 gi = group_info[g];
    const int x_row = gi.x, n = group_word_rows(gi.y);
    const uint8_t* in = act + static_cast<size_t>(x_row) * KCb * 128;
    uint8_t* out = actq + static_cast<size_t>(x_row) * KCq * 128;
    uint8_t* sf = act_sf + static_cast<size_t>(x_row >> 4) * KCq * 1024;
    for (int j = blockIdx.y * (kThreads / 32) + warp; j < n; j += gridDim.y * (kThreads / 32)) {
      for (int c0 = 0; c0 < KCq; c0 += kActChunksPerPass) {
        uint2 raw[kActChunksPerPass];
#pragma unroll
        for (int i = 0; i < kActChunksPerPass; ++i) {
          const int c = c0 + i;
          raw[i] = c < KCq ? *reinterpret_cast<const uint2*>(in + static_cast<size_t>(2 * c + (lane >> 4)) * n * 128 +
                                                             j * 128 + ((((ib >> 4) ^ j) & 7) << 4) + (ib & 15))
                           : make_uint2(0u, 0u);
        }
#pragma unroll
        for (int i = 0; i < kActChunksPerPass; ++i) {
          const int c = c0 + i;
          if (c >= KCq) break;  // warp-uniform
          const float2 f01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[i].x));
          const float2 f23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[i].y));
          float amax = fmaxf(fmaxf(fabsf(f01.x), fabsf(f01.y)), fmaxf(fabsf(f23.x), fabsf(f23.y)));
#pragma unroll
          for (int o = 1; o < 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
          const int e = mx_exponent(amax);
          *reinterpret_cast<uint32_t*>(out + static_cast<size_t>(c) * n * 128 + j * 128 +
                                       ((((ob >> 4) ^ j) & 7) << 4) + (ob & 15)) =
              mx_e4m3x4(f01.x, f01.y, f23.x, f23.y, mx_inv(e));
          if ((lane & 7) == 0)
            sf[static_cast<size_t>(c) * 1024 + (j >> 7) * 512 + (j & 31) * 16 + ((j >> 5) & 3) * 4 + (lane >> 3)] =
                static_cast<uint8_t>(e + 127);
        }
      }
    }
  }
}

// Byte offsets, inside a row group of n rows and KC chunks, of row j's codes in chunk c
// (unswizzled start of the 128-byte chunk row) and of its fp32 scale: the FP8 block-128
// X layout (moe_internal.h).
__device__ __forceinline__ void b128_offsets(int n, int KC, int c, int j, size_t& code, size_t& scale) {
  const int kc = chunks_per_step(n);
  const int c0 = c - c % kc;
  const int kcs = min(kc, KC - c0);
  const size_t step = static_cast<size_t>(c0) * n * kB128RowBytesPerChunk;
  code = step + static_cast<size_t>(c - c0) * n * 128 + static_cast<size_t>(j) * 128;
  scale = step + static_cast<size_t>(kcs) * n * 128 + (static_cast<size_t>(c - c0) * n + j) * 4;
}

// One 1x128 group held as four values per lane: scale = amax / 448 (1 for all zeros) and
// the lane's four codes e4m3(x / scale), IEEE divisions. Every lane takes part.
__device__ __forceinline__ uint32_t quant_group_1x128(float x0, float x1, float x2, float x3, float& s) {
  float amax = fmaxf(fmaxf(fabsf(x0), fabsf(x1)), fmaxf(fabsf(x2), fabsf(x3)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  s = amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(x0, s), __fdiv_rn(x1, s)), __NV_SATFINITE,
                                               __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(x2, s), __fdiv_rn(x3, s)), __NV_SATFINITE,
                                               __NV_E4M3);
  return lo | (hi << 16);
}

// FP8 block-128: the token rows, already quantised once per token (quant_act_kernel: e4m3
// codes [T, H] and fp32 1x128 scales [T, H/128]), copied into the X layout of their row
// groups. A warp copies one row: lane l moves 16-byte pieces l, l + 32, ... of the row's
// codes (all loads first) and lanes 0..KC-1 its scales. Padding rows are not written (GEMM1
// stores zeros for them whatever they hold).
constexpr int kB128Pieces = 4;  // 16-byte pieces per lane per pass (a 2 KB row in one pass)
__global__ void __launch_bounds__(kThreads)
    permute_b128_rows_kernel(const uint4* __restrict__ xq, const float* __restrict__ xq_scale, int H,
                             const int* __restrict__ sorted_pair_ids, const int* __restrict__ num_groups,
                             const int2* __restrict__ group_info, int P, int k_total, uint8_t* __restrict__ xs) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int G = *num_groups;
  const int KC = H / 128, pieces = H / 16;
  for (int g = blockIdx.x; g < G; g += gridDim.x) {
    const int2 gi = group_info[g];
    const int x_row = gi.x, n = group_word_rows(gi.y);
    uint8_t* base = xs + static_cast<size_t>(x_row) * KC * kB128RowBytesPerChunk;
    for (int j = blockIdx.y * (kThreads / 32) + warp; j < n; j += gridDim.y * (kThreads / 32)) {
      const int pid = sorted_pair_ids[x_row + j];
      if (pid >= P) continue;  // a padding row (warp-uniform)
      const long long tok = pid / k_total;
      for (int p0 = 0; p0 < pieces; p0 += 32 * kB128Pieces) {
        uint4 v[kB128Pieces];
#pragma unroll
        for (int i = 0; i < kB128Pieces; ++i) {
          const int p = p0 + lane + 32 * i;
          v[i] = p < pieces ? __ldg(xq + tok * pieces + p) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int i = 0; i < kB128Pieces; ++i) {
          const int p = p0 + lane + 32 * i;
          if (p < pieces) {
            size_t co, so;
            b128_offsets(n, KC, p >> 3, j, co, so);
            *reinterpret_cast<uint4*>(base + co + ((((p & 7) ^ j) & 7) << 4)) = v[i];
          }
        }
      }
      for (int c = lane; c < KC; c += 32) {
        size_t co, so;
        b128_offsets(n, KC, c, j, co, so);
        *reinterpret_cast<float*>(base + so) = __ldg(xq_scale + tok * KC + c);
      }
    }
  }
}

// FP8 block-128: GEMM1's bf16 activation (64-column chunks of 128-byte rows, row-group
// order) quantised per 1x128 group into the X layout; a warp takes one row, four chunks at
// a time (their loads first), lane l columns 4l..4l+3 of each 128-column chunk (8 bytes of
// bf16 chunk 2c + l / 16).
__global__ void __launch_bounds__(kThreads)
    act_quant_b128_kernel(const uint8_t* __restrict__ act, int I, const int* __restrict__ num_groups,
                          const int2* __restrict__ group_info, uint8_t* __restrict__ actq) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int G = *num_groups;
  const int KCb = I / 64, KC = I / 128;
  for (int g = blockIdx.x; g < G; g += gridDim.x) {
    const int2 gi = group_info[g];
    const int x_row = gi.x, n = group_word_rows(gi.y);
    const uint8_t* in = act + static_cast<size_t>(x_row) * KCb * 128;
    uint8_t* base = actq + static_cast<size_t>(x_row) * KC * kB128RowBytesPerChunk;
    for (int j = blockIdx.y * (kThreads / 32) + warp; j < n; j += gridDim.y * (kThreads / 32)) {
      const int ib = 8 * (lane & 15);  // byte of the bf16 chunk row
      for (int c0 = 0; c0 < KC; c0 += kActChunksPerPass) {
        uint2 raw[kActChunksPerPass];
#pragma unroll
        for (int i = 0; i < kActChunksPerPass; ++i) {
          const int c = c0 + i;
          raw[i] = c < KC ? *reinterpret_cast<const uint2*>(in + static_cast<size_t>(2 * c + (lane >> 4)) * n * 128 +
                                                            j * 128 + ((((ib >> 4) ^ j) & 7) << 4) + (ib & 15))
                          : make_uint2(0u, 0u);
        }
#pragma unroll
        for (int i = 0; i < kActChunksPerPass; ++i) {
          const int c = c0 + i;
          if (c >= KC) break;  // warp-uniform
          const float2 f01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[i].x));
          const float2 f23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[i].y));
          float sc;
          const uint32_t codes = quant_group_1x128(f01.x, f01.y, f23.x, f23.y, sc);
          size_t co, so;
          b128_offsets(n, KC, c, j, co, so);
          const int ob = 4 * lane;
          *reinterpret_cast<uint32_t*>(base + co + ((((ob >> 4) ^ j) & 7) << 4) + (ob & 15)) = codes;
          if (lane == 0) *reinterpret_cast<float*>(base + so) = sc;
        }
      }
    }
  }
}

// NVFP4: the token rows, quantised once per token (codes [T, H/2], scales [T, H/16]),
// copied into their row groups: codes as 128-byte chunk rows (256 values, swizzled like the
// other 8-bit layouts), scales into the group's 2048-byte block per chunk (byte 512 mm +
// 16 (j % 32) + 4 (j / 32) + k: group row j, 16-value block 16 c + 4 mm + k). A warp copies
// one row; lane l moves 16-byte code pieces l, l + 32, ... and the row's scale bytes 4l..4l+3
// (blocks 4l..4l+3: one MMA's four). Padding rows are not written (GEMM1 stores zeros for
// them whatever they hold).
__global__ void __launch_bounds__(kThreads)
    permute_nvfp4_rows_kernel(const uint4* __restrict__ xq, const uint8_t* __restrict__ xq_scale, int H,
                              const int* __restrict__ sorted_pair_ids, const int* __restrict__ num_groups,
                              const int2* __restrict__ group_info, int P, int k_total, uint8_t* __restrict__ xs,
                              uint8_t* __restrict__ xs_sf) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int G = *num_groups;
  const int KC = H / 256, pieces = H / 32, sbytes = H / 16;
  for (int g = blockIdx.x; g < G; g += gridDim.x) {
    const int2 gi = group_info[g];
    const int x_row = gi.x, n = group_word_rows(gi.y);
    uint8_t* base = xs + static_cast<size_t>(x_row) * KC * 128;
    uint8_t* sfb = xs_sf + static_cast<size_t>(x_row >> 4) * KC * kNvChunkScaleBytes;
    for (int j = blockIdx.y * (kThreads / 32) + warp; j < n; j += gridDim.y * (kThreads / 32)) {
      const int pid = sorted_pair_ids[x_row + j];
      if (pid >= P) continue;  // a padding row (warp-uniform)
      const long long tok = pid / k_total;
      for (int p0 = 0; p0 < pieces; p0 += 32 * kB128Pieces) {
        uint4 v[kB128Pieces];
#pragma unroll
        for (int i = 0; i < kB128Pieces; ++i) {
          const int p = p0 + lane + 32 * i;
          v[i] = p < pieces ? __ldg(xq + tok * pieces + p) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int i = 0; i < kB128Pieces; ++i) {
          const int p = p0 + lane + 32 * i;
          if (p < pieces)
            *reinterpret_cast<uint4*>(base + static_cast<size_t>(p >> 3) * n * 128 + j * 128 +
                                      ((((p & 7) ^ j) & 7) << 4)) = v[i];
        }
      }
      for (int b0 = 4 * lane; b0 < sbytes; b0 += 128) {
        const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(xq_scale + tok * sbytes + b0));
        const int c = b0 >> 4, mm = (b0 >> 2) & 3;
        *reinterpret_cast<uint32_t*>(sfb + static_cast<size_t>(c) * kNvChunkScaleBytes + mm * 512 + 16 * (j & 31) +
                                     4 * (j >> 5)) = w;
      }
    }
  }
}

// NVFP4: GEMM1's bf16 activation (64-column chunks of 128-byte rows, row-group order)
// quantised with tensor scale g into the layout of permute_nvfp4_rows_kernel. A warp takes
// one row, four 256-column chunks at a time (their loads first): lane l converts columns
// 8l..8l+7 of each (16 bytes of bf16 chunk 4c + l / 8); lanes 2b and 2b+1 share 16-value
// block b and exchange their maxima.
__global__ void __launch_bounds__(kThreads)
    act_quant_nvfp4_kernel(const uint8_t* __restrict__ act, int I, float g, const int* __restrict__ num_groups,
                           const int2* __restrict__ group_info, uint8_t* __restrict__ actq, uint8_t* __restrict__ act_sf) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int G = *num_groups;
  const int KCb = I / 64, KC = I / 256;
  const int ib = 16 * (lane & 7);  // byte of the bf16 chunk row
  const int ob = 4 * lane;         // byte of the code chunk row
  for (int gr = blockIdx.x; gr < G; gr += gridDim.x) {
    const int2 gi = group_info[gr];
    const int x_row = gi.x, n = group_word_rows(gi.y);
    const uint8_t* in = act + static_cast<size_t>(x_row) * KCb * 128;
    uint8_t* out = actq + static_cast<size_t>(x_row) * KC * 128;
    uint8_t* sf = act_sf + static_cast<size_t>(x_row >> 4) * KC * kNvChunkScaleBytes;
    for (int j = blockIdx.y * (kThreads / 32) + warp; j < n; j += gridDim.y * (kThreads / 32)) {
      for (int c0 = 0; c0 < KC; c0 += kActChunksPerPass) {
        uint4 raw[kActChunksPerPass];
#pragma unroll
        for (int i = 0; i < kActChunksPerPass; ++i) {
          const int c = c0 + i;
          raw[i] = c < KC ? *reinterpret_cast<const uint4*>(in + static_cast<size_t>(4 * c + (lane >> 3)) * n * 128 +
                                                            j * 128 + ((((ib >> 4) ^ j) & 7) << 4))
                          : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int i = 0; i < kActChunksPerPass; ++i) {
          const int c = c0 + i;
          if (c >= KC) break;  // warp-uniform
          const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw[i]);
          float v[8];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 f = __bfloat1622float2(h[k]);
            v[2 * k] = f.x;
            v[2 * k + 1] = f.y;
          }
          float amax = 0.f;
#pragma unroll
          for (int k = 0; k < 8; ++k) amax = fmaxf(amax, fabsf(v[k]));
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
          const uint8_t s = nvfp4_block_scale(amax, g);
          const float d = e4m3_value(s) * g;
          const uint32_t codes = nvfp4_pair(v[0], v[1], d) | (nvfp4_pair(v[2], v[3], d) << 8) |
                                 (nvfp4_pair(v[4], v[5], d) << 16) | (nvfp4_pair(v[6], v[7], d) << 24);
          *reinterpret_cast<uint32_t*>(out + static_cast<size_t>(c) * n * 128 + j * 128 +
                                       ((((ob >> 4) ^ j) & 7) << 4) + (ob & 15)) = codes;
          if ((lane & 1) == 0) {
            const int b = lane >> 1;
            sf[static_cast<size_t>(c) * kNvChunkScaleBytes + (b >> 2) * 512 + 16 * (j & 31) + 4 * (j >> 5) + (b & 3)] =
                s;
          }
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_permute_nvfp4_rows(const Launch& l, const void* xq, const void* xq_scale, int H,
                                      const int* sorted_pair_ids, const int* num_groups, const int2* group_info, int P,
                                      int k_total, void* xs, void* xs_sf, int num_sms) {
  if (H % 256 != 0) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(2 * num_sms, kNvGroupRows / (kThreads / 32)), dim3(kThreads), 0);
  return cudaLaunchKernelEx(&cfg, permute_nvfp4_rows_kernel, static_cast<const uint4*>(xq),
                            static_cast<const uint8_t*>(xq_scale), H, sorted_pair_ids, num_groups, group_info, P,
                            k_total, static_cast<uint8_t*>(xs), static_cast<uint8_t*>(xs_sf));
}

cudaError_t launch_act_quant_nvfp4(const Launch& l, const void* act, int I, float g, const int* num_groups,
                                   const int2* group_info, void* actq, void* act_sf, int num_sms) {
  if (I % 256 != 0) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(2 * num_sms, kNvGroupRows / (kThreads / 32)), dim3(kThreads), 0);
  return cudaLaunchKernelEx(&cfg, act_quant_nvfp4_kernel, static_cast<const uint8_t*>(act), I, g, num_groups,
                            group_info, static_cast<uint8_t*>(actq), static_cast<uint8_t*>(act_sf));
}

cudaError_t launch_permute_b128_rows(const Launch& l, const void* xq, const float* xq_scale, int H,
                                     const int* sorted_pair_ids, const int* num_groups, const int2* group_info, int P,
                                     int k_total, void* xs, int num_sms) {
  if (H % 128 != 0) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(2 * num_sms, kB128GroupRows / (kThreads / 32)), dim3(kThreads), 0);
  return cudaLaunchKernelEx(&cfg, permute_b128_rows_kernel, static_cast<const uint4*>(xq), xq_scale, H,
                            sorted_pair_ids, num_groups, group_info, P, k_total, static_cast<uint8_t*>(xs));
}

cudaError_t launch_act_quant_b128(const Launch& l, const void* act, int I, const int* num_groups,
                                  const int2* group_info, void* actq, int num_sms) {
  if (I % 128 != 0) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(2 * num_sms, kB128GroupRows / (kThreads / 32)), dim3(kThreads), 0);
  return cudaLaunchKernelEx(&cfg, act_quant_b128_kernel, static_cast<const uint8_t*>(act), I, num_groups,
                            group_info, static_cast<uint8_t*>(actq));
}

cudaError_t launch_permute_quant_rows(const Launch& l, const void* hidden, int H, const int* sorted_pair_ids,
                                      const int* num_groups, const int2* group_info, int P, int k_total,
                                      float input_scale, void* xs, int num_sms) {
  if (H % 128 != 0) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(2 * num_sms, 256 / kRowsPerCta), dim3(kThreads), 0);
  const float inv_scale = 1.0f / input_scale;  // IEEE fp32 division on the host
  return cudaLaunchKernelEx(&cfg, permute_quant_rows_kernel, static_cast<const uint4*>(hidden), H, sorted_pair_ids,
                            num_groups, group_info, P, k_total, inv_scale, static_cast<uint8_t*>(xs));
}

cudaError_t launch_permute_rows(const Launch& l, const void* hidden, int H, const int* sorted_pair_ids,
                                const int* num_groups, const int2* group_info, int P, int k_total, void* xs,
                                int num_sms) {
  if (H % 64 != 0) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(2 * num_sms, 256 / kRowsPerCta), dim3(kThreads), 0);
  return cudaLaunchKernelEx(&cfg, permute_rows_kernel, static_cast<const uint4*>(hidden), H / 8, sorted_pair_ids,
                            num_groups, group_info, P, k_total, static_cast<uint8_t*>(xs));
}

cudaError_t launch_permute_mx_rows(const Launch& l, const void* hidden, int H, const int* sorted_pair_ids,
                                   const int* num_groups, const int2* group_info, int P, int k_total, void* xs,
                                   void* xs_sf, int num_sms) {
  if (H % 128 != 0) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(2 * num_sms, (kMxGroupRows + kRowsPerCta - 1) / kRowsPerCta),
                     dim3(kThreads), 0);
  return cudaLaunchKernelEx(&cfg, permute_mx_rows_kernel, static_cast<const uint4*>(hidden), H, sorted_pair_ids,
                            num_groups, group_info, P, k_total, static_cast<uint8_t*>(xs),
                            static_cast<uint8_t*>(xs_sf));
}

cudaError_t launch_act_quant_mx(const Launch& l, const void* act, int I, const int* num_groups,
                                const int2* group_info, void* actq, void* act_sf, int num_sms) {
  if (I % 128 != 0) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(2 * num_sms, kMxGroupRows / (kThreads / 32)), dim3(kThreads), 0);
  return cudaLaunchKernelEx(&cfg, act_quant_mx_kernel, static_cast<const uint8_t*>(act), I, num_groups,
                            group_info, static_cast<uint8_t*>(actq), static_cast<uint8_t*>(act_sf));
}

}  // namespace moe
