// Steps 3 and 4 of the layer for decode-sized batches (bf16): the grouped GEMMs with the
// operands swapped.
//
// With a few tokens per expert, a 128-row token tile would be almost all padding while
// the expert's weights still stream in full. Here the expert's weight rows are the MMA's
// M operand (128 rows per tile) and the expert's token rows, padded to blocks of 16, are
// its N operand: D^T[n, r] = sum_k W[e][n, k] * X[r, k], tcgen05.mma kind::f16 with M=128,
// N=16, K=16, fp32 accumulators in TMEM (16 columns per tile, double-buffered). A TMEM lane
// is then one weight row: for GEMM1 the gate and up rows of an intermediate index
// ([gate0, up0, gate1, up1, ...] after the load-time interleave of "[MoE] SwiGLU fusion
// into the MoE up-GEMM epilogue", sglang PR 32944, section 3) sit in adjacent lanes and are
// paired with one shuffle before silu(gate)*up (or relu2) is applied.
//
// GEMM1: W = w13 tile (TMA), X = the block's 16 token rows gathered from hidden
// (cp.async); output act [rows, I] bf16 in sorted row order.
// GEMM2: W = w2 tile (TMA), X = the block's 16 activation rows (TMA); output y [rows, H]
// fp32 = topk_w[p] * D, sorted row order, as in the 128-row path.
//
// One persistent CTA per SM, 6 warps: warp 0 producer (weights by TMA, token rows by TMA or
// cp.async), warp 1 TMEM allocator and MMA issuer, warps 2-5 epilogue (lane quadrant = warp
// % 4). A deep ring (10 stages of 18 KB) keeps ~180 KB of weights in flight per SM.
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kMW = 128;                 // weight rows per tile (MMA M)
constexpr int kNT = 16;                  // token rows per block (MMA N)
constexpr int kBKBytes = 128;            // 64 bf16 of K per stage
constexpr int kStageW = kMW * kBKBytes;  // 16 KB
constexpr int kStageX = 2048;            // 16 rows x 128 B, padded to a 1 KB multiple
constexpr int kStageBytes = kStageW + kStageX;
constexpr int kStages = 10;
constexpr int kThreads = 192;
constexpr int kTmemCols = 32;  // two 16-column accumulators
constexpr int kBarOffset = kStages * kStageBytes;
constexpr int kSmemBytes = kBarOffset + 256 + 1024;

enum : int { kSiteEmpty = 1, kSiteFull = 2, kSiteTmemEmpty = 3, kSiteTmemFull = 4 };

struct Args {
  int mode;        // 0 = GEMM1, 1 = GEMM2
  int n_tiles;     // weight-row tiles per expert (N1/128 or H/128)
  int k_blocks;    // ceil(K / 64)
  int w_rows_per_expert;
  int k_total, num_pairs, activation;
  int block_m;     // token rows per block (16)
  const uint8_t* x_rows;  // GEMM1: hidden [T, H] bf16
  int x_row_bytes;        // GEMM1: H * 2
  const int* num_blocks;
  const int* block_expert;
  const int* sorted_pair_ids;
  const float* topk_w;
  void* out;       // GEMM1: act bf16 [rows, I]; GEMM2: y fp32 [rows, H]
  int out_cols;    // I or H
  int* status;
};

__global__ void __launch_bounds__(kThreads, 1)
    gemm_decode_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                       const Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t s0 = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOffset);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * kStages;
  const uint32_t tfull0 = empty0 + 8 * kStages;
  const uint32_t tempty0 = tfull0 + 16;
  const uint32_t drain_bar = tempty0 + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool gather_x = a.mode == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      // GEMM1: the weight copy's expect-tx arrival + one cp.async arrival per producer lane
      mbar_init(full0 + 8 * s, gather_x ? 33 : 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, 128);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmW);
    if (!gather_x) prefetch_tmap(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  griddep_wait();
  griddep_launch_dependents();
  const int num_tiles = *a.num_blocks * a.n_tiles;

  if (warp == 0) {
    // ---------------- producer ----------------
    const uint64_t pol_w = policy_evict_first();
    const uint64_t pol_x = policy_evict_last();
    const uint32_t bytes = kStageW + (gather_x ? 0u : static_cast<uint32_t>(a.block_m) * kBKBytes);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      const int b = tile / a.n_tiles;
      const int nt = tile - b * a.n_tiles;
      const int wrow = a.block_expert[b] * a.w_rows_per_expert + nt * kMW;
      // GEMM1: lane l copies 16-byte chunk (l & 7) of token rows (l >> 3) + 4 i
      const uint8_t* src[4];
      if (gather_x) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = (lane >> 3) + 4 * i;
          const int pid = a.sorted_pair_ids[b * a.block_m + r];
          const int tok = pid < a.num_pairs ? pid / a.k_total : 0;
          src[i] = a.x_rows + static_cast<size_t>(tok) * a.x_row_bytes + (lane & 7) * 16;
        }
      }
      for (int kb = 0; kb < a.k_blocks; ++kb) {
        int got = 0;
        if (lane == 0) got = mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag, a.status, kSiteEmpty);
        if (!__shfl_sync(0xffffffffu, got, 0)) {
          ok = false;
          break;
        }
        const uint32_t full = full0 + 8 * stage;
        const uint32_t w_dst = s0 + stage * kStageBytes;
        const uint32_t x_dst = w_dst + kStageW;
        if (lane == 0) {
          mbar_arrive_expect_tx(full, bytes);
          tma_load_2d(w_dst, &tmW, full, kb * 64, wrow, pol_w);
          if (!gather_x) tma_load_2d(x_dst, &tmX, full, kb * 64, b * a.block_m, pol_x);
        }
        if (gather_x) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int r = (lane >> 3) + 4 * i;
            cp_async16(x_dst + r * kBKBytes + (((lane & 7) ^ (r & 7)) << 4), src[i] + kb * kBKBytes);
          }
          cp_async_mbar_arrive(full);
        }
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (gather_x) cp_async_wait_all();
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kMW, kNT);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        if (!mbar_wait(tempty0 + 8 * acc, ((it >> 1) & 1) ^ 1u, abort_flag, a.status, kSiteTmemEmpty)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kNT;
        for (int kb = 0; kb < a.k_blocks; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag, a.status, kSiteFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t w_addr = s0 + stage * kStageBytes;
          const uint64_t adesc = umma_desc_sw128(w_addr);
          const uint64_t bdesc = umma_desc_sw128(w_addr + kStageW);
#pragma unroll
          for (int k = 0; k < 4; ++k) umma_bf16(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0);
          umma_commit(empty0 + 8 * stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) umma_commit(tfull0 + 8 * acc);
      }
      umma_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0);
    }
  } else {
    // ---------------- epilogue (warps 2..5): lane = weight row ----------------
    const int q = warp & 3;
    const bool gated = a.activation == 0;
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      const bool got = mbar_wait(tfull0 + 8 * acc, (it >> 1) & 1, abort_flag, a.status, kSiteTmemFull);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int b = tile / a.n_tiles;
      const int nt = tile - b * a.n_tiles;
      // lanes 0..15 hold the block's pair ids
      const int my_pid = lane < a.block_m ? a.sorted_pair_ids[b * a.block_m + lane] : a.num_pairs;
      const float my_w = (a.mode != 0 && my_pid < a.num_pairs) ? a.topk_w[my_pid] : 0.f;
      uint32_t v[16];
      __syncwarp();
      tmem_ld16(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * kNT, v);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(tempty0 + 8 * acc);  // the accumulator is in registers now
      const int n = nt * kMW + q * 32 + lane;  // weight row of this lane
      if (a.mode == 0) {
        __nv_bfloat16* act = static_cast<__nv_bfloat16*>(a.out);
#pragma unroll
        for (int r = 0; r < kNT; ++r) {
          const int pid = __shfl_sync(0xffffffffu, my_pid, r);
          const float z = __uint_as_float(v[r]);
          const float up = __shfl_down_sync(0xffffffffu, z, 1);  // odd lane: the up row
          if (pid < a.num_pairs) {
            const size_t row = static_cast<size_t>(b) * a.block_m + r;
            if (gated) {
              if ((lane & 1) == 0) act[row * a.out_cols + (n >> 1)] = __float2bfloat16_rn(silu_f32(z) * up);
            } else {
              const float zr = fmaxf(z, 0.f);
              act[row * a.out_cols + n] = __float2bfloat16_rn(zr * zr);
            }
          }
        }
      } else {
        float* y = static_cast<float*>(a.out);
#pragma unroll
        for (int r = 0; r < kNT; ++r) {
          const int pid = __shfl_sync(0xffffffffu, my_pid, r);
          const float w = __shfl_sync(0xffffffffu, my_w, r);
          if (pid < a.num_pairs)
            y[(static_cast<size_t>(b) * a.block_m + r) * a.out_cols + n] = __uint_as_float(v[r]) * w;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

bool g_attr_set[64] = {};

}  // namespace

cudaError_t launch_gemm_decode(const Launch& l, int mode, const CUtensorMap& tm_w, const CUtensorMap& tm_x,
                               const void* x_rows, const GemmShape& s, const GemmBuffers& b) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 64 && !g_attr_set[dev]) {
    err = cudaFuncSetAttribute(gemm_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return err;
    g_attr_set[dev] = true;
  }
  Args a;
  a.mode = mode;
  a.n_tiles = s.N / kMW;
  a.k_blocks = (s.K + 63) / 64;
  a.w_rows_per_expert = s.w_rows_per_expert;
  a.k_total = s.k_total;
  a.num_pairs = s.num_pairs;
  a.activation = s.activation;
  a.block_m = kNT;
  a.x_rows = static_cast<const uint8_t*>(x_rows);
  a.x_row_bytes = s.K * 2;
  a.num_blocks = b.num_blocks;
  a.block_expert = b.block_expert;
  a.sorted_pair_ids = b.sorted_pair_ids;
  a.topk_w = b.topk_w;
  a.out = b.out;
  a.out_cols = s.out_cols;
  a.status = b.status;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(s.num_sms), dim3(kThreads), kSmemBytes);
  return cudaLaunchKernelEx(&cfg, gemm_decode_kernel, tm_w, tm_x, a);
}

}  // namespace moe
