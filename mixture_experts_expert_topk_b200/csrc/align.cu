// Step 2 of the layer: stable sort of the (token, slot) pairs by expert, each expert's
// segment padded to the GEMM row tile.
//
// The grouped GEMM contract of "W4A8 grouped GEMM optimisation for GLM-5.2 MoE on H200"
// (sglang PR 38220), section 1, gives each expert a contiguous row range
// (expert_offsets). Reading: an expert's segment lists its pair ids p = t*k' + j in
// ascending order, then the sentinel P up to the next multiple of block_m; an expert
// with no pairs has no rows.
//
// Deterministic counting sort (no atomics decide any position). Pairs are cut into
// chunks of kAlignChunk; a chunk is handled by 8 warps of 256 consecutive pairs each:
//   count   per chunk: per-expert histogram (shared-memory atomics; counts only);
//   scan    one CTA: per-expert exclusive prefix over chunks (chunk histograms staged in
//           shared memory batch by batch, so no thread walks global memory serially),
//           padded segment sizes, exclusive scan over experts -> expert_offsets,
//           block_expert, sentinel padding;
//   scatter per chunk: each warp counts its 256 pairs per expert, the 8 warp counts are
//           prefix-summed per expert, then each warp places its pairs 32 at a time; lanes
//           with the same expert find each other with __match_any_sync and take
//           consecutive ranks, so the order within an expert is the pair order.
// With a single chunk (decode-sized batches) the three phases run in one CTA.
//
// For the GEMMs that put the tokens on the MMA's N operand (block_m 16), the scan also
// cuts every expert's padded segment into row groups of at most group_rows rows, in
// multiples of 16 and as even in size as possible, and lists them in expert order.
#include <algorithm>

#include "moe_device.cuh"
#include "moe_internal.h"
#include "route_device.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;                        // warps per chunk
constexpr int kPairsPerWarp = kAlignChunk / kWarps;  // 256
constexpr int kIdsPerLane = kPairsPerWarp / 32;  // 8
constexpr int kScanThreads = 1024;
constexpr int kScanSmemInts = 40960;             // 160 KB of chunk-histogram staging

static_assert(kPairsPerWarp % 32 == 0, "warp slices are whole 32-pair steps");

// Load this warp's pair ids (p = base + 32 i + lane); -1 marks pairs past the end and
// kBadId a pair whose expert id lies outside [0, E): such a pair is neither counted nor
// placed, and its pair_to_row entry becomes -1.
constexpr int kBadId = -2;
__device__ __forceinline__ void load_ids(const int* ids, int base, int end, int E, int lane,
                                         int (&e)[kIdsPerLane]) {
#pragma unroll
  for (int i = 0; i < kIdsPerLane; ++i) {
    const int p = base + 32 * i + lane;
    const int id = p < end ? __ldcg(ids + p) : -1;  // L2: the ids may come from this CTA
    e[i] = p >= end ? -1 : (static_cast<unsigned>(id) < static_cast<unsigned>(E) ? id : kBadId);
  }
}

// Per-expert counts of this warp's pairs into cnt[] (shared; one writer per expert per step).
__device__ __forceinline__ void warp_count(const int (&e)[kIdsPerLane], int lane, int* cnt) {
#pragma unroll
  for (int i = 0; i < kIdsPerLane; ++i) {
    const unsigned peers = __match_any_sync(0xffffffffu, e[i]);
    if (e[i] >= 0 && lane == 31 - __clz(peers)) cnt[e[i]] += __popc(peers);
    __syncwarp();
  }
}

// Place this warp's pairs: next[] holds each expert's next free row for this warp.
__device__ __forceinline__ void warp_place(const int (&e)[kIdsPerLane], int base, int lane, int* next,
                                           int* sorted_pair_ids, int* pair_to_row) {
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int i = 0; i < kIdsPerLane; ++i) {
    const unsigned peers = __match_any_sync(0xffffffffu, e[i]);
    if (e[i] >= 0) {
      const int p = base + 32 * i + lane;
      const int pos = next[e[i]] + __popc(peers & lt);
      sorted_pair_ids[pos] = p;
      pair_to_row[p] = pos;
    } else if (e[i] == kBadId) {
      pair_to_row[base + 32 * i + lane] = -1;
    }
    __syncwarp();
    if (e[i] >= 0 && lane == 31 - __clz(peers)) next[e[i]] += __popc(peers);
    __syncwarp();
  }
}

// Exclusive scan of one value per thread over a CTA of up to 1024 threads.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = (blockDim.x + 31) >> 5;
    int w = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const int excl = incl - v + (warp > 0 ? warp_sums[warp - 1] : 0);
  if (total) *total = warp_sums[((blockDim.x + 31) >> 5) - 1];
  __syncthreads();
  return excl;
}

// Padded segments of experts [0, E): sentinel rows after each expert's pairs and the
// expert id of each row tile. One thread per expert (at most block_m - 1 sentinels and
// padded / block_m tile ids each), so no warp walks the experts one after another; most
// experts of a small batch have no rows at all. seg_off/seg_cnt/seg_pad are shared-memory
// arrays; off and pad are multiples of block_m.
__device__ __forceinline__ void write_segments(int E, const int* seg_off, const int* seg_cnt, const int* seg_pad,
                                               int block_m, int P, int* sorted_pair_ids, int* block_expert) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int off = seg_off[e], cnt = seg_cnt[e], pad = seg_pad[e];
    if (pad == 0) continue;
    for (int r = off + cnt; r < off + pad; ++r) sorted_pair_ids[r] = P;
    const int b0 = off / block_m, b1 = (off + pad) / block_m;
    for (int b = b0; b < b1; ++b) block_expert[b] = e;
  }
}

__device__ __forceinline__ int num_groups_of(int padded, int group_rows) {
  return group_rows > 0 && padded > 0 ? (padded + group_rows - 1) / group_rows : 0;
}

// Row groups of expert e's padded segment [off, off + padded) holding `count` pairs, written
// from index g0; the last group carries the segment's padding rows.
__device__ __forceinline__ void write_groups(int e, int off, int count, int padded, int group_rows, int g0,
                                             int2* group_info) {
  const int ng = num_groups_of(padded, group_rows);
  if (ng == 0) return;
  const int blocks = padded / 16;
  const int base = blocks / ng, extra = blocks - base * ng;
  int row = off;
  for (int i = 0; i < ng; ++i) {
    const int rows = 16 * (base + (i < extra ? 1 : 0));
    group_info[g0 + i] = make_int2(row, group_word(e, rows, i == ng - 1 ? padded - count : 0));
    row += rows;
  }
}

__global__ void __launch_bounds__(kWarps * 32)
    align_count_kernel(const int* __restrict__ ids, int P, int E, int* __restrict__ chunk_hist) {
  __shared__ int hist[kMaxExperts];
  griddep_wait();
  griddep_launch_dependents();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int base = blockIdx.x * kAlignChunk;
  const int end = min(base + kAlignChunk, P);
  for (int p = base + threadIdx.x; p < end; p += blockDim.x) {
    const int id = ids[p];
    if (static_cast<unsigned>(id) < static_cast<unsigned>(E)) atomicAdd(&hist[id], 1);
  }
  __syncthreads();
  int* out = chunk_hist + static_cast<size_t>(blockIdx.x) * E;
  for (int e = threadIdx.x; e < E; e += blockDim.x) out[e] = hist[e];
}

__global__ void __launch_bounds__(kScanThreads)
    align_scan_kernel(int* __restrict__ chunk_hist, int num_chunks, int E, int P, int block_m,
                      int* __restrict__ sorted_pair_ids, int* __restrict__ expert_offsets,
                      int* __restrict__ block_expert, int* __restrict__ num_blocks, int group_rows,
                      int2* __restrict__ group_info) {
  extern __shared__ int stage[];  // [batch chunks][E]
  __shared__ int warp_sums[32];
  __shared__ int seg_off[kMaxExperts], seg_cnt[kMaxExperts], seg_pad[kMaxExperts];
  griddep_wait();
  griddep_launch_dependents();
  const int e = threadIdx.x;  // E <= 1024: one expert per thread
  const int batch = max(1, kScanSmemInts / E);
  int count = 0;
  for (int c0 = 0; c0 < num_chunks; c0 += batch) {
    const int nc = min(batch, num_chunks - c0);
    int* g = chunk_hist + static_cast<size_t>(c0) * E;
    for (int i = threadIdx.x; i < nc * E; i += blockDim.x) stage[i] = g[i];
    __syncthreads();
    if (e < E) {
      for (int c = 0; c < nc; ++c) {
        const int x = stage[c * E + e];
        g[c * E + e] = count;  // exclusive prefix of expert e over chunks
        count += x;
      }
    }
    __syncthreads();
  }
  const int padded = e < E ? (count + block_m - 1) / block_m * block_m : 0;
  int total = 0;
  const int off = block_exclusive_scan(padded, warp_sums, &total);
  if (e < E) {
    expert_offsets[e] = off;
    seg_off[e] = off;
    seg_cnt[e] = count;
    seg_pad[e] = padded;
  }
  int gtotal = 0;
  const int g0 = block_exclusive_scan(e < E ? num_groups_of(padded, group_rows) : 0, warp_sums, &gtotal);
  if (e < E) write_groups(e, off, count, padded, group_rows, g0, group_info);
  if (threadIdx.x == 0) {
    expert_offsets[E] = total;
    num_blocks[0] = total / block_m;
    if (group_rows > 0) num_blocks[1] = gtotal;
  }
  __syncthreads();
  write_segments(E, seg_off, seg_cnt, seg_pad, block_m, P, sorted_pair_ids, block_expert);
}

__global__ void __launch_bounds__(kWarps * 32)
    align_scatter_kernel(const int* __restrict__ ids, int P, int E, const int* __restrict__ chunk_hist,
                         const int* __restrict__ expert_offsets, int* __restrict__ sorted_pair_ids,
                         int* __restrict__ pair_to_row) {
  __shared__ int cnt[kWarps][kMaxExperts];
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int x = threadIdx.x; x < E; x += blockDim.x)
#pragma unroll
    for (int w = 0; w < kWarps; ++w) cnt[w][x] = 0;
  const int base = blockIdx.x * kAlignChunk + warp * kPairsPerWarp;
  int e[kIdsPerLane];
  load_ids(ids, base, P, E, lane, e);
  __syncthreads();
  warp_count(e, lane, cnt[warp]);
  __syncthreads();
  const int* h = chunk_hist + static_cast<size_t>(blockIdx.x) * E;
  for (int x = threadIdx.x; x < E; x += blockDim.x) {
    int run = expert_offsets[x] + h[x];
    for (int w = 0; w < kWarps; ++w) {
      const int c = cnt[w][x];
      cnt[w][x] = run;
      run += c;
    }
  }
  __syncthreads();
  warp_place(e, base, lane, cnt[warp], sorted_pair_ids, pair_to_row);
}

// All of align for P <= kAlignChunk by one CTA of kWarps warps (every thread calls it).
struct AlignSingleSmem {
  int cnt[kWarps][kMaxExperts];
  int warp_sums[32];
  int seg_off[kMaxExperts], seg_cnt[kMaxExperts], seg_pad[kMaxExperts];
};
__device__ __forceinline__ void align_single_cta(AlignSingleSmem& sm, const int* ids, int P, int E, int block_m,
                                                 int* sorted_pair_ids, int* expert_offsets, int* block_expert,
                                                 int* pair_to_row, int* num_blocks, int group_rows,
                                                 int2* group_info) {
  auto& cnt = sm.cnt;
  int* warp_sums = sm.warp_sums;
  int* seg_off = sm.seg_off;
  int* seg_cnt = sm.seg_cnt;
  int* seg_pad = sm.seg_pad;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int x = threadIdx.x; x < E; x += blockDim.x)
#pragma unroll
    for (int w = 0; w < kWarps; ++w) cnt[w][x] = 0;
  const int base = warp * kPairsPerWarp;
  int e[kIdsPerLane];
  load_ids(ids, base, P, E, lane, e);
  __syncthreads();
  warp_count(e, lane, cnt[warp]);
  __syncthreads();
  // experts in groups of blockDim.x: totals, padded sizes, exclusive scan, warp prefixes
  int carry = 0, gcarry = 0;
  for (int x0 = 0; x0 < E; x0 += blockDim.x) {
    const int x = x0 + threadIdx.x;
    int count = 0;
    if (x < E)
      for (int w = 0; w < kWarps; ++w) count += cnt[w][x];
    const int padded = x < E ? (count + block_m - 1) / block_m * block_m : 0;
    int total = 0;
    const int off = carry + block_exclusive_scan(padded, warp_sums, &total);
    if (x < E) {
      expert_offsets[x] = off;
      seg_off[x] = off;
      seg_cnt[x] = count;
      seg_pad[x] = padded;
      int run = off;
      for (int w = 0; w < kWarps; ++w) {
        const int c = cnt[w][x];
        cnt[w][x] = run;
        run += c;
      }
    }
    int gtotal = 0;
    const int g0 = gcarry + block_exclusive_scan(x < E ? num_groups_of(padded, group_rows) : 0, warp_sums, &gtotal);
    if (x < E) write_groups(x, off, count, padded, group_rows, g0, group_info);
    carry += total;
    gcarry += gtotal;
  }
  if (threadIdx.x == 0) {
    expert_offsets[E] = carry;
    num_blocks[0] = carry / block_m;
    if (group_rows > 0) num_blocks[1] = gcarry;
  }
  __syncthreads();
  write_segments(E, seg_off, seg_cnt, seg_pad, block_m, P, sorted_pair_ids, block_expert);
  warp_place(e, base, lane, cnt[warp], sorted_pair_ids, pair_to_row);
}

__global__ void __launch_bounds__(kWarps * 32)
    align_single_kernel(const int* __restrict__ ids, int P, int E, int block_m, int* __restrict__ sorted_pair_ids,
                        int* __restrict__ expert_offsets, int* __restrict__ block_expert,
                        int* __restrict__ pair_to_row, int* __restrict__ num_blocks, int group_rows,
                        int2* __restrict__ group_info) {
  __shared__ AlignSingleSmem sm;
  griddep_wait();
  griddep_launch_dependents();
  align_single_cta(sm, ids, P, E, block_m, sorted_pair_ids, expert_offsets, block_expert, pair_to_row, num_blocks,
                   group_rows, group_info);
}

// Routing and align of a small batch (T <= kWarps * kRouteAlignTokensPerWarp tokens, one
// align chunk) in one CTA, one kernel boundary fewer: each warp routes its tokens
// (route_token, as the routing kernel), the CTA synchronises, then aligns the pairs it just
// wrote (read back through L2). Like the routing kernel it starts the forward: it clears the
// status word and the GEMMs' work counters, and prefetches the token rows into L2. With xs
// (bf16, at most kFusedPermutePairs pairs) it also copies each pair's token row into its
// row group (the permute step's layout; padding rows are not written), a warp per pair: the
// group is found by binary search over the row groups just written.
template <int VPL>
__global__ void __launch_bounds__(kWarps * 32)
    route_align_kernel(const float* __restrict__ logits, int T, int E_r, int topk, int num_shared, int renormalize,
                       int* topk_ids, float* topk_w, int* status, const uint8_t* __restrict__ hidden,
                       int hidden_row_bytes, int E, int block_m, int* sorted_pair_ids, int* expert_offsets,
                       int* block_expert, int* pair_to_row, int* num_blocks, int group_rows, int2* group_info,
                       uint8_t* xs) {
  __shared__ AlignSingleSmem sm;
  griddep_wait();
  griddep_launch_dependents();
  if (threadIdx.x < 8) status[threadIdx.x] = 0;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int t = warp; t < T; t += kWarps) {
    if (hidden != nullptr && lane == 0)
      prefetch_l2_bulk(hidden + static_cast<size_t>(t) * hidden_row_bytes, static_cast<uint32_t>(hidden_row_bytes));
    route_token<VPL>(logits, t, E_r, topk, num_shared, renormalize, lane, topk_ids, topk_w);
  }
  __syncthreads();  // every token's slots are written (global memory, visible to the CTA)
  const int P = T * (topk + num_shared);
  align_single_cta(sm, topk_ids, P, E, block_m, sorted_pair_ids, expert_offsets, block_expert, pair_to_row,
                   num_blocks, group_rows, group_info);
  if (xs == nullptr) return;
  __syncthreads();  // pair_to_row, the row groups and their count are written
  const int G = __ldcg(num_blocks + 1);
  const int pieces = hidden_row_bytes >> 4;  // 16-byte pieces of a row: 8 per 128-byte chunk
  for (int p = warp; p < P; p += kWarps) {
    const int pos = __ldcg(pair_to_row + p);
    if (pos < 0) continue;  // an unroutable id (warp-uniform)
    int lo = 0, hi = G - 1;  // the last group starting at or before pos
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldcg(&group_info[mid].x) <= pos) lo = mid; else hi = mid - 1;
    }
    const int2 gi = __ldcg(group_info + lo);
    const int n = group_word_rows(gi.y), j = pos - gi.x;
    const uint4* src = reinterpret_cast<const uint4*>(hidden + static_cast<size_t>(p / (topk + num_shared)) * hidden_row_bytes);
    uint8_t* base = xs + static_cast<size_t>(gi.x) * hidden_row_bytes;
    for (int q = lane; q < pieces; q += 32) {
      const int c = q >> 3;
      *reinterpret_cast<uint4*>(base + static_cast<size_t>(c) * n * 128 + j * 128 + (((q & 7) ^ (j & 7)) << 4)) =
          __ldg(src + q);
    }
  }
}

template <int VPL>
cudaError_t launch_route_align_vpl(const Launch& l, const float* logits, int T, int E_r, int topk, int num_shared,
                                   int renormalize, int* topk_ids, float* topk_w, int* status, const void* hidden,
                                   int hidden_row_bytes, int E, int block_m, int* sorted_pair_ids,
                                   int* expert_offsets, int* block_expert, int* pair_to_row, int* num_blocks,
                                   int group_rows, int2* group_info, void* xs) {
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(1), dim3(kWarps * 32), 0);
  return cudaLaunchKernelEx(&cfg, route_align_kernel<VPL>, logits, T, E_r, topk, num_shared, renormalize, topk_ids,
                            topk_w, status, static_cast<const uint8_t*>(hidden), hidden_row_bytes, E, block_m,
                            sorted_pair_ids, expert_offsets, block_expert, pair_to_row, num_blocks, group_rows,
                            group_info, static_cast<uint8_t*>(xs));
}

bool g_scan_attr[64] = {};

}  // namespace

cudaError_t launch_align(const Launch& l, const int* topk_ids, int P, int E, int block_m, int num_chunks,
                         int* chunk_hist, int* sorted_pair_ids, int* expert_offsets, int* block_expert,
                         int* pair_to_row, int* num_blocks, int group_rows, int2* group_info) {
  if (group_rows != 0 && (block_m != 16 || group_rows % 16 != 0 || group_rows > 256)) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  if (num_chunks == 1) {
    make_launch_config(&cfg, attr, l, dim3(1), dim3(kWarps * 32), 0);
    return cudaLaunchKernelEx(&cfg, align_single_kernel, topk_ids, P, E, block_m, sorted_pair_ids,
                              expert_offsets, block_expert, pair_to_row, num_blocks, group_rows, group_info);
  }
  make_launch_config(&cfg, attr, l, dim3(num_chunks), dim3(kWarps * 32), 0);
  cudaError_t err = cudaLaunchKernelEx(&cfg, align_count_kernel, topk_ids, P, E, chunk_hist);
  if (err != cudaSuccess) return err;
  const int batch = std::max(1, kScanSmemInts / E);
  const size_t smem = static_cast<size_t>(std::min(batch, num_chunks)) * E * sizeof(int);
  int dev = 0;
  if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
  if (dev < 64 && !g_scan_attr[dev]) {
    err = cudaFuncSetAttribute(align_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kScanSmemInts * static_cast<int>(sizeof(int)));
    if (err != cudaSuccess) return err;
    g_scan_attr[dev] = true;
  }
  make_launch_config(&cfg, attr, l, dim3(1), dim3(kScanThreads), smem);
  err = cudaLaunchKernelEx(&cfg, align_scan_kernel, chunk_hist, num_chunks, E, P, block_m, sorted_pair_ids,
                           expert_offsets, block_expert, num_blocks, group_rows, group_info);
  if (err != cudaSuccess) return err;
  make_launch_config(&cfg, attr, l, dim3(num_chunks), dim3(kWarps * 32), 0);
  return cudaLaunchKernelEx(&cfg, align_scatter_kernel, (const int*)topk_ids, P, E, (const int*)chunk_hist,
                            (const int*)expert_offsets, sorted_pair_ids, pair_to_row);
}

cudaError_t launch_route_align(const Launch& l, const float* logits, int T, int E_routed, int topk, int num_shared,
                               int renormalize, int* topk_ids, float* topk_w, int* status, const void* hidden,
                               int hidden_row_bytes, int E, int block_m, int* sorted_pair_ids, int* expert_offsets,
                               int* block_expert, int* pair_to_row, int* num_blocks, int group_rows,
                               int2* group_info, void* xs) {
  if (T > kWarps * kRouteAlignTokensPerWarp || T * (topk + num_shared) > kAlignChunk || E > kMaxExperts ||
      (group_rows != 0 && (block_m != 16 || group_rows % 16 != 0 || group_rows > 256)))
    return cudaErrorInvalidValue;
  if (xs != nullptr && (group_rows == 0 || hidden == nullptr || T * (topk + num_shared) > kFusedPermutePairs ||
                        hidden_row_bytes % 128 != 0))
    return cudaErrorInvalidValue;
  const int vpl = (E_routed + 31) / 32;
#define MOE_RA(V)                                                                                              \
  return launch_route_align_vpl<V>(l, logits, T, E_routed, topk, num_shared, renormalize, topk_ids, topk_w, status, \
                                   hidden, hidden_row_bytes, E, block_m, sorted_pair_ids, expert_offsets,         \
                                   block_expert, pair_to_row, num_blocks, group_rows, group_info, xs)
  if (vpl <= 1) MOE_RA(1);
  if (vpl <= 2) MOE_RA(2);
  if (vpl <= 4) MOE_RA(4);
  if (vpl <= 8) MOE_RA(8);
  if (vpl <= 16) MOE_RA(16);
  MOE_RA(32);
#undef MOE_RA
}

}  // namespace moe
