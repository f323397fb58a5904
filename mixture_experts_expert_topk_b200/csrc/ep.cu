// Expert parallelism: the dispatch and combine steps around the layer when the experts
// are split over several GPUs (one process per GPU).
//
// Rank r of `world` owns the routed experts [r * E_r / world, (r + 1) * E_r / world) and a
// copy of the shared expert (slot id E_r), which stays on the token's own rank. Dispatch
// sorts this rank's (token, slot) pairs stably by owner rank (the align kernels with the
// owner as the key, each owner's segment padded to 16 rows) and packs, in that order, the
// token's hidden row, the owner-local expert id and the routing weight of each pair; the
// caller exchanges the segments (one all-to-all), runs the owners' experts on what they
// received (the routed forward with one slot per row) and sends the weighted rows back
// (the reverse all-to-all). Combine then sums each token's k' returned rows in slot order
// in fp32 and rounds once to bf16, so the result does not depend on which rank computed
// what or in which order the rows arrived.
#include <algorithm>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;

// Owner rank of every pair: a routed id's range, the shared slot's own rank.
__global__ void __launch_bounds__(kThreads)
    ep_owner_kernel(const int* __restrict__ ids, long long P, int E_r, int per_rank, int rank, int* __restrict__ owner) {
  griddep_wait();
  griddep_launch_dependents();
  for (long long p = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; p < P;
       p += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int e = ids[p];
    owner[p] = e < E_r ? e / per_rank : rank;
  }
}

// Row i of the send buffer (i < send_offsets[world]): the pair sorted_pair_ids[i]'s hidden
// row, owner-local expert id and weight; padding rows (sentinel P) are zero rows with
// expert 0 and weight 0. One warp per row, 16-byte pieces.
__global__ void __launch_bounds__(kThreads)
    ep_pack_kernel(const uint4* __restrict__ hidden, int H8, const int* __restrict__ sorted_pair_ids,
                   const int* __restrict__ send_offsets, int world, int P, int k_total, const int* __restrict__ ids,
                   const float* __restrict__ weights, int E_r, int per_rank, uint4* __restrict__ send_rows,
                   int* __restrict__ send_expert, float* __restrict__ send_weight) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const long long rows = send_offsets[world];
  for (long long i = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; i < rows;
       i += (static_cast<long long>(gridDim.x) * blockDim.x) >> 5) {
    const int pid = sorted_pair_ids[i];
    const bool real = pid < P;
    const uint4* src = real ? hidden + static_cast<long long>(pid / k_total) * H8 : nullptr;
    uint4* dst = send_rows + i * H8;
    for (int c = lane; c < H8; c += 32) dst[c] = real ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
    if (lane == 0) {
      int local = 0;
      float w = 0.f;
      if (real) {
        const int e = ids[pid];
        local = e < E_r ? e - (e / per_rank) * per_rank : per_rank;  // the shared copy follows the range
        w = weights[pid];
      }
      send_expert[i] = local;
      send_weight[i] = w;
    }
  }
}

// out[t] = sum_j returned[pair_to_row[t * k' + j]] over j = 0..k'-1 in fp32, rounded once
// to bf16. One thread per 8 columns of a token.
__global__ void __launch_bounds__(kThreads)
    ep_combine_kernel(const uint4* __restrict__ returned, const int* __restrict__ pair_to_row, int T, int k_total,
                      int H8, uint4* __restrict__ out) {
  griddep_wait();
  griddep_launch_dependents();
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long long>(T) * H8) return;
  const long long t = idx / H8;
  const int c = static_cast<int>(idx - t * H8);
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  for (int j = 0; j < k_total; ++j) {
    const uint4 v = __ldg(returned + static_cast<long long>(__ldg(pair_to_row + t * k_total + j)) * H8 + c);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(h[k]);
      acc[2 * k] += f.x;
      acc[2 * k + 1] += f.y;
    }
  }
  out[idx] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                        pack_bf16x2(acc[6], acc[7]));
}

}  // namespace

cudaError_t launch_ep_owner(const Launch& l, const int* ids, long long P, int E_r, int per_rank, int rank,
                            int* owner) {
  if (P == 0) return cudaSuccess;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(static_cast<unsigned>(std::min<long long>((P + kThreads - 1) / kThreads, 1024))),
                     dim3(kThreads), 0);
  return cudaLaunchKernelEx(&cfg, ep_owner_kernel, ids, P, E_r, per_rank, rank, owner);
}

cudaError_t launch_ep_pack(const Launch& l, const void* hidden, int H, const int* sorted_pair_ids,
                           const int* send_offsets, int world, int P, int k_total, const int* ids, const float* weights,
                           int E_r, int per_rank, long long max_rows, void* send_rows, int* send_expert,
                           float* send_weight, int num_sms) {
  if (H % 8 != 0) return cudaErrorInvalidValue;
  const long long blocks = std::min<long long>((max_rows * 32 + kThreads - 1) / kThreads, 8LL * num_sms);
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(static_cast<unsigned>(std::max<long long>(blocks, 1))), dim3(kThreads), 0);
  return cudaLaunchKernelEx(&cfg, ep_pack_kernel, static_cast<const uint4*>(hidden), H / 8, sorted_pair_ids,
                            send_offsets, world, P, k_total, ids, weights, E_r, per_rank,
                            static_cast<uint4*>(send_rows), send_expert, send_weight);
}

cudaError_t launch_ep_combine(const Launch& l, const void* returned, const int* pair_to_row, int T, int k_total, int H,
                              void* out) {
  const int H8 = H / 8;
  const long long n = static_cast<long long>(T) * H8;
  if (n == 0) return cudaSuccess;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(static_cast<unsigned>((n + kThreads - 1) / kThreads)), dim3(kThreads), 0);
  return cudaLaunchKernelEx(&cfg, ep_combine_kernel, static_cast<const uint4*>(returned), pair_to_row, T, k_total,
                            H8, static_cast<uint4*>(out));
}

}  // namespace moe
