// GEMM1's token rows in the row-group order of the swapped-operand GEMM (gemm_swap.cu).
//
// For each row group (x_row, n) of align's output, row j of the group is the hidden row of
// its pair's token, hidden[sorted_pair_ids[x_row + j] / k'], or zero for a padding row.
// The group occupies bytes [x_row * H * 2, (x_row + n) * H * 2) of xs; 64-column chunk c of
// it is n rows of 128 bytes at offset c * n * 128, the 16-byte piece q of row j stored at
// position q ^ (j % 8) (the 128-byte swizzle the MMA reads). The GEMM then loads each K
// step of a group with one contiguous bulk copy.
//
// A CTA copies a 32-row slice of a row group; each warp two rows at a time, each lane with
// sixteen 16-byte loads of the hidden rows in flight (coalesced) before writing them to
// their chunk rows.
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
    const int x_row = gi.x, n = gi.y >> 16;
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
          if (j >= n) continue;
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

}  // namespace

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

}  // namespace moe
