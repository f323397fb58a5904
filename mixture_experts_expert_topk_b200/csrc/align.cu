// Step 2 of the layer: stable sort of the (token, slot) pairs by expert, each expert's
// segment padded to the GEMM row tile.
//
// The grouped GEMM contract of "W4A8 grouped GEMM optimisation for GLM-5.2 MoE on H200"
// (sglang PR 38220), section 1, gives each expert a contiguous row range
// (expert_offsets). Reading: an expert's segment lists its pair ids p = t*k' + j in
// ascending order, then the sentinel P up to the next multiple of block_m; an expert
// with no pairs has no rows.
//
// Deterministic three-pass counting sort, no atomics on positions:
//   count   one CTA per chunk of 1024 pairs: per-expert histogram of the chunk;
//   scan    one CTA: per-expert prefix over chunks, padded segment sizes, exclusive
//           scan over experts -> expert_offsets, block_expert, sentinel padding;
//   scatter one warp per chunk: walks its chunk in order, 32 pairs at a time; lanes with
//           the same expert find each other with __match_any_sync and take consecutive
//           ranks, so the in-chunk order is the pair order.
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kCountThreads = 256;
constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kCountThreads)
    align_count_kernel(const int* __restrict__ ids, int P, int E, int* __restrict__ chunk_hist) {
  __shared__ int hist[kMaxExperts];
  griddep_wait();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int base = blockIdx.x * kAlignChunk;
  const int end = min(base + kAlignChunk, P);
  for (int p = base + threadIdx.x; p < end; p += blockDim.x) atomicAdd(&hist[ids[p]], 1);
  __syncthreads();
  int* out = chunk_hist + static_cast<size_t>(blockIdx.x) * E;
  for (int e = threadIdx.x; e < E; e += blockDim.x) out[e] = hist[e];
}

__global__ void __launch_bounds__(kScanThreads)
    align_scan_kernel(int* __restrict__ chunk_hist, int num_chunks, int E, int P, int block_m,
                      int* __restrict__ sorted_pair_ids, int* __restrict__ expert_offsets,
                      int* __restrict__ block_expert, int* __restrict__ num_blocks) {
  __shared__ int warp_sums[kScanThreads / 32];
  griddep_wait();
  const int e = threadIdx.x;  // E <= 1024: one expert per thread
  int count = 0;
  if (e < E) {
    for (int c = 0; c < num_chunks; ++c) {
      int* h = chunk_hist + static_cast<size_t>(c) * E + e;
      const int x = *h;
      *h = count;  // exclusive prefix of expert e over chunks
      count += x;
    }
  }
  const int padded = (count + block_m - 1) / block_m * block_m;
  // block-wide exclusive scan of `padded` over experts
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = padded;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const int off = incl - padded + (warp > 0 ? warp_sums[warp - 1] : 0);
  if (e < E) {
    expert_offsets[e] = off;
    for (int r = off + count; r < off + padded; ++r) sorted_pair_ids[r] = P;
    for (int b = off / block_m; b < (off + padded) / block_m; ++b) block_expert[b] = e;
    if (e == E - 1) {
      expert_offsets[E] = off + padded;
      *num_blocks = (off + padded) / block_m;
    }
  }
}

__global__ void __launch_bounds__(32)
    align_scatter_kernel(const int* __restrict__ ids, int P, int E,
                         const int* __restrict__ chunk_hist, const int* __restrict__ expert_offsets,
                         int* __restrict__ sorted_pair_ids, int* __restrict__ pair_to_row) {
  __shared__ int next[kMaxExperts];
  griddep_wait();
  const int lane = threadIdx.x;
  const int* h = chunk_hist + static_cast<size_t>(blockIdx.x) * E;
  for (int e = lane; e < E; e += 32) next[e] = expert_offsets[e] + h[e];
  __syncwarp();
  const unsigned lt_mask = (1u << lane) - 1u;
  const int base = blockIdx.x * kAlignChunk;
  const int end = min(base + kAlignChunk, P);
  for (int s = base; s < end; s += 32) {
    const int p = s + lane;
    const bool valid = p < end;
    const int e = valid ? ids[p] : E;  // E never matches a real expert
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & lt_mask);
    int pos = 0;
    if (valid) {
      pos = next[e] + rank;
      sorted_pair_ids[pos] = p;
      pair_to_row[p] = pos;
    }
    __syncwarp();
    if (valid && lane == 31 - __clz(peers)) next[e] += __popc(peers);
    __syncwarp();
  }
}

}  // namespace

cudaError_t launch_align(const Launch& l, const int* topk_ids, int P, int E, int block_m,
                         int num_chunks, int* chunk_hist, int* sorted_pair_ids,
                         int* expert_offsets, int* block_expert, int* pair_to_row,
                         int* num_blocks) {
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(num_chunks), dim3(kCountThreads), 0);
  cudaError_t err = cudaLaunchKernelEx(&cfg, align_count_kernel, topk_ids, P, E, chunk_hist);
  if (err != cudaSuccess) return err;
  make_launch_config(&cfg, attr, l, dim3(1), dim3(kScanThreads), 0);
  err = cudaLaunchKernelEx(&cfg, align_scan_kernel, chunk_hist, num_chunks, E, P, block_m,
                           sorted_pair_ids, expert_offsets, block_expert, num_blocks);
  if (err != cudaSuccess) return err;
  make_launch_config(&cfg, attr, l, dim3(num_chunks), dim3(32), 0);
  return cudaLaunchKernelEx(&cfg, align_scatter_kernel, (const int*)topk_ids, P, E,
                            (const int*)chunk_hist, (const int*)expert_offsets, sorted_pair_ids,
                            pair_to_row);
}

}  // namespace moe
