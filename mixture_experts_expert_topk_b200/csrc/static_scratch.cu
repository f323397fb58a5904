// moe_align_noalloc: the align step (stable sort of (token, slot) pairs by expert, padded
// to the GEMM row tile) for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc or hand this library a workspace: an inference
// engine plugin that only receives its input and output tensors, code that runs while a
// stream is being captured (allocation is not allowed there), or a latency-critical path
// where an allocation could synchronise the device. This entry point gives them the align
// step without any allocation: its scratch (the per-chunk expert histograms) lives in a
// fixed-size array in device global memory that belongs to this library and is loaded
// with it. Every GPU that loads the library holds the array until the process exits.
//
// The kernels are the same ones moe_stage_align runs; only the scratch pointer differs.
#include <atomic>
#include <mutex>

#include "moe_b200.h"
#include "moe_internal.h"

namespace {

// Scratch: align chunk histograms, one int per (chunk of 2048 pairs, expert). 1 MiB
// covers e.g. 256 chunks (524288 pairs) of 1024 experts.
constexpr size_t kStaticScratchInts = 262144;
static __device__ __align__(256) int g_align_scratch[kStaticScratchInts];

// In host code `g_align_scratch` names a host-side stand-in, not device memory: its device
// address comes from cudaGetSymbolAddress, once per device with that device current.
std::mutex g_scratch_mutex;
int* g_scratch_ptr[64] = {};

moe_status_t scratch_for_current_device(int** ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= 64) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_align_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
    g_scratch_ptr[dev] = static_cast<int*>(p);
  }
  *ptr = g_scratch_ptr[dev];
  return MOE_OK;
}

bool aligned4(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace

extern "C" __attribute__((visibility("default"))) moe_status_t moe_align_noalloc(
    const moe_problem_t* problem, const int32_t* topk_ids, int32_t* sorted_pair_ids, int32_t* expert_offsets,
    int32_t* block_expert, int32_t* pair_to_row, int32_t* num_blocks, moe_stream_t stream) {
  moe_workspace_layout_t lay;
  moe_status_t st = moe_workspace_layout(problem, &lay);
  if (st != MOE_OK) return st;
  if (problem->num_tokens == 0) return MOE_OK;
  if (!aligned4(topk_ids) || !aligned4(sorted_pair_ids) || !aligned4(expert_offsets) || !aligned4(block_expert) ||
      !aligned4(pair_to_row) || !aligned4(num_blocks))
    return MOE_ERR_INVALID_ARG;
  const int E = problem->num_routed + problem->num_shared;
  const long long P = static_cast<long long>(problem->num_tokens) * (problem->topk + problem->num_shared);
  // the chunk histograms must fit the fixed scratch array
  if (static_cast<size_t>(lay.num_chunks) * static_cast<size_t>(E) > kStaticScratchInts) return MOE_ERR_UNSUPPORTED;
  int major = 0, minor = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (major != 10 || minor != 0) return MOE_ERR_UNSUPPORTED;  // sm_100 kernels only
  int* scratch = nullptr;
  st = scratch_for_current_device(&scratch);
  if (st != MOE_OK) return st;
  moe::Launch l;
  l.stream = reinterpret_cast<cudaStream_t>(stream);
  l.pdl = (problem->flags & MOE_FLAG_PDL) != 0;
  const cudaError_t e = moe::launch_align(l, topk_ids, static_cast<int>(P), E, lay.block_m, lay.num_chunks, scratch,
                                          sorted_pair_ids, expert_offsets, block_expert, pair_to_row, num_blocks, 0,
                                          nullptr);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
