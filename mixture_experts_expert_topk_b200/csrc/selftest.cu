// moe_selftest_bounded_wait: exercises the device-side timeout path of the kernels without
// faulting, trapping or hanging the GPU.
//
// Every wait inside this library's kernels (mbarrier phases of the copy rings, the
// accumulator hand-offs and the tile queues) goes through mbar_wait_bounded: after its
// limit it raises the CTA's abort flag, records kStatusTimeout | site in the workspace
// status word and returns, so the host can read MOE_ERR_DEVICE_TIMEOUT from
// moe_get_device_status while the context stays usable. The kernel below waits, through
// that same routine, on an mbarrier that expects one arrival; with arrive = 0 nothing
// arrives and the wait must run out after the caller's (short) limit.
#include "moe_b200.h"
#include "moe_device.cuh"
#include "moe_internal.h"

namespace {

constexpr int kSiteSelftest = 0x7F;

__global__ void bounded_wait_kernel(int* status, unsigned long long limit_ns, int arrive) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    moe::mbar_init(moe::smem_u32(&bar), 1);
    abort_flag = 0;
    moe::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (arrive) moe::mbar_arrive(moe::smem_u32(&bar));
    moe::mbar_wait_bounded(moe::smem_u32(&bar), 0, &abort_flag, status, kSiteSelftest, limit_ns);
  }
}

}  // namespace

extern "C" __attribute__((visibility("default"))) moe_status_t moe_selftest_bounded_wait(
    void* workspace, uint32_t limit_us, int32_t arrive, moe_stream_t stream) {
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MOE_ERR_INVALID_ARG;
  if (limit_us < 1 || limit_us > 1000000 || (arrive != 0 && arrive != 1)) return MOE_ERR_INVALID_ARG;
  bounded_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<int*>(workspace), static_cast<unsigned long long>(limit_us) * 1000ull, arrive);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
