// Steps 3 and 4 of the layer in bf16: the two grouped GEMMs over the expert-sorted rows.
//
// GEMM1 (up-GEMM with fused activation; "[MoE] SwiGLU fusion into the MoE up-GEMM
// epilogue", sglang PR 32944, sections 1 and 3): row r of the sorted order belongs to
// pair p = sorted_pair_ids[r] and expert e = block_expert[r / 128]; its A row is
// hidden[p / k'], gathered straight from the token-order hidden tensor with TMA
// gather4. B is the prepared w13 of expert e, whose gate and up rows are interleaved
// ([gate0, up0, gate1, up1, ...]), so accumulator columns (2j, 2j+1) of a tile hold
// gate_j and up_j. The epilogue applies silu(gate)*up (or relu2) to the fp32
// accumulators in registers and writes only the I-wide bf16 activation.
//
// GEMM2 (down-GEMM with routing weight): A is the activation in sorted row order, B is
// w2 of the row tile's expert; the epilogue multiplies row r by topk_w[p] and writes it
// in fp32 to row p of y (pair order), ready for the fixed-order combine.
//
// Kernel structure (one persistent CTA per SM, 6 warps):
//   warp 0      TMA producer: B tile (weights, 2-D tiled load) + A tile (gather4 or 2-D)
//               into a 4-stage shared-memory ring, 128-byte swizzle, 64 bf16 of K per
//               stage;
//   warp 1      TMEM allocator and MMA issuer: tcgen05.mma kind::f16, M=128, N=BN,
//               K=16, fp32 accumulators in TMEM, double-buffered (2 x 256 columns) so
//               the epilogue of tile i overlaps the main loop of tile i+1;
//   warps 2-5   epilogue: tcgen05.ld 32 columns at a time, activation / weighting in
//               registers, 16-byte global stores.
// Tiles are (row tile, N tile) pairs, row-tile-major, so the CTAs running at the same
// time work on neighbouring row tiles of the same experts and share weight tiles in L2.
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kBM = 128;
constexpr int kBKBytes = 128;               // one 128-byte swizzle atom of K per stage
constexpr int kStages = 4;
constexpr int kMaxBN = 256;
constexpr int kStageA = kBM * kBKBytes;     // 16 KB
constexpr int kStageB = kMaxBN * kBKBytes;  // 32 KB
constexpr int kStageBytes = kStageA + kStageB;
constexpr int kThreads = 192;
constexpr int kAccCols = 256;               // TMEM columns per accumulator buffer
constexpr int kTmemCols = 512;
constexpr int kBarOffset = kStages * kStageBytes;
constexpr int kSmemBytes = kBarOffset + 256 + 1024;  // barriers + 1024-byte alignment slack

// wait sites (device status detail)
enum : int { kSiteEmpty = 1, kSiteFull = 2, kSiteTmemEmpty = 3, kSiteTmemFull = 4, kSiteDrain = 5 };

struct Args {
  int mode;  // 0 = GEMM1 (gather + activation), 1 = GEMM2 (weighted scatter)
  int K, BN, n_tiles, k_blocks;
  int w_rows_per_expert;
  int k_total, num_pairs, activation, out_cols;
  const int* num_blocks;
  const int* block_expert;
  const int* sorted_pair_ids;
  const float* topk_w;
  void* out;  // GEMM1: bf16 act [rows, I]; GEMM2: fp32 y [P, H]
  int* status;
};

__global__ void __launch_bounds__(kThreads, 1)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOffset);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = smem_u32(bars + kStages);
  const uint32_t tfull0 = smem_u32(bars + 2 * kStages);
  const uint32_t tempty0 = smem_u32(bars + 2 * kStages + 2);
  const uint32_t drain_bar = smem_u32(bars + 2 * kStages + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
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
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // everything above overlaps the previous kernel; inputs are read only after this
  griddep_wait();
  const int num_tiles = *a.num_blocks * a.n_tiles;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    const uint64_t pol_w = policy_evict_first();  // weights: streamed once
    const uint64_t pol_a = policy_evict_last();   // activations: reused across N tiles
    const uint32_t b_bytes = static_cast<uint32_t>(a.BN) * kBKBytes;
    int stage = 0;
    uint32_t phase = 0;
    long long issued = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      const int mb = tile / a.n_tiles;
      const int nt = tile - mb * a.n_tiles;
      const int e = a.block_expert[mb];
      const int brow = e * a.w_rows_per_expert + nt * a.BN;
      int r[4] = {0, 0, 0, 0};
      if (a.mode == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int pid = a.sorted_pair_ids[mb * kBM + lane * 4 + i];
          r[i] = pid < a.num_pairs ? pid / a.k_total : 0;  // padding rows read token 0
        }
      }
      for (int kb = 0; kb < a.k_blocks; ++kb) {
        int got = 0;
        if (lane == 0) got = mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag, a.status, kSiteEmpty);
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) {
          ok = false;
          break;
        }
        const uint32_t full = full0 + 8 * stage;
        const uint32_t a_dst = smem_u32(smem + stage * kStageBytes);
        const uint32_t b_dst = a_dst + kStageA;
        if (lane == 0) {
          mbar_arrive_expect_tx(full, kStageA + b_bytes);
          tma_load_2d(b_dst, &tmB, full, kb * 64, brow, pol_w);
          if (a.mode != 0) tma_load_2d(a_dst, &tmA, full, kb * 64, mb * kBM, pol_a);
        }
        __syncwarp();
        if (a.mode == 0)
          tma_gather4(a_dst + lane * 4 * kBKBytes, &tmA, full, kb * 64, r[0], r[1], r[2], r[3], pol_a);
        ++issued;
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok && lane == 0) {
      // make sure no copy lands in shared memory after the CTA exits
      for (int s = 0; s < kStages; ++s) {
        if (issued <= s) break;
        const long long last = issued - 1 - ((issued - 1 - s) % kStages);
        mbar_wait_drain(full0 + 8 * s, static_cast<uint32_t>((last / kStages) & 1));
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kBM, a.BN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t aphase = (it >> 1) & 1;
        if (!mbar_wait(tempty0 + 8 * acc, aphase ^ 1u, abort_flag, a.status, kSiteTmemEmpty)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kAccCols;
        for (int kb = 0; kb < a.k_blocks; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag, a.status, kSiteFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * kStageBytes);
          const uint64_t adesc = umma_desc_sw128(a_addr);
          const uint64_t bdesc = umma_desc_sw128(a_addr + kStageA);
#pragma unroll
          for (int k = 0; k < 4; ++k)  // 4 x K=16 bf16 = 128 bytes; +32 bytes = +2 encoded
            umma_bf16(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0);
          umma_commit(empty0 + 8 * stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) umma_commit(tfull0 + 8 * acc);
      }
      // all MMAs of this thread complete before TMEM is released
      umma_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0);
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const int row = q * 32 + lane;
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      const uint32_t aphase = (it >> 1) & 1;
      const bool got = mbar_wait(tfull0 + 8 * acc, aphase, abort_flag, a.status, kSiteTmemFull);
      if (!__all_sync(0xffffffffu, got)) break;  // leave warp-uniformly (tcgen05.ld is .aligned)
      tc_fence_after();
      const int mb = tile / a.n_tiles;
      const int nt = tile - mb * a.n_tiles;
      const int grow = mb * kBM + row;
      const int pid = a.sorted_pair_ids[grow];
      const bool valid = pid < a.num_pairs;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * kAccCols;
      if (a.mode == 0) {
        const bool gated = a.activation == 0;
        const int ncol = gated ? a.BN / 2 : a.BN;
        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.out) + static_cast<size_t>(grow) * a.out_cols + nt * ncol;
        for (int c = 0; c < a.BN / 32; ++c) {
          uint32_t v[32];
          __syncwarp();  // tcgen05.ld is .sync.aligned
          tmem_ld32(taddr + c * 32, v);
          tmem_wait_ld();
          if (gated) {
            uint32_t o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float g0 = __uint_as_float(v[4 * i + 0]), u0 = __uint_as_float(v[4 * i + 1]);
              const float g1 = __uint_as_float(v[4 * i + 2]), u1 = __uint_as_float(v[4 * i + 3]);
              o[i] = pack_bf16x2(silu_f32(g0) * u0, silu_f32(g1) * u1);
            }
            if (valid) {
              uint4* dst = reinterpret_cast<uint4*>(orow + c * 16);
              dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
              dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
            }
          } else {
            uint32_t o[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float z0 = fmaxf(__uint_as_float(v[2 * i + 0]), 0.f);
              float z1 = fmaxf(__uint_as_float(v[2 * i + 1]), 0.f);
              o[i] = pack_bf16x2(z0 * z0, z1 * z1);
            }
            if (valid) {
              uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
              for (int i = 0; i < 4; ++i) dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
            }
          }
        }
      } else {
        // y is kept in fp32: rounding it to bf16 before the combine would cost about as
        // much accuracy as the final bf16 output rounding itself
        const float w = valid ? a.topk_w[pid] : 0.f;
        float* orow = reinterpret_cast<float*>(a.out) + static_cast<size_t>(valid ? pid : 0) * a.out_cols + nt * a.BN;
        for (int c = 0; c < a.BN / 32; ++c) {
          uint32_t v[32];
          __syncwarp();  // tcgen05.ld is .sync.aligned
          tmem_ld32(taddr + c * 32, v);
          tmem_wait_ld();
          if (valid) {
            float4* dst = reinterpret_cast<float4*>(orow + c * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(v[4 * i]) * w, __uint_as_float(v[4 * i + 1]) * w,
                                   __uint_as_float(v[4 * i + 2]) * w, __uint_as_float(v[4 * i + 3]) * w);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(tempty0 + 8 * acc);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();  // tcgen05.dealloc is .sync.aligned: the whole warp, converged
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

bool g_attr_set[64] = {};

cudaError_t launch(const Launch& l, const CUtensorMap& tmA, const CUtensorMap& tmB, const Args& args,
                   int num_sms) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 64 && !g_attr_set[dev]) {
    err = cudaFuncSetAttribute(gemm_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return err;
    g_attr_set[dev] = true;
  }
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(num_sms), dim3(kThreads), kSmemBytes);
  return cudaLaunchKernelEx(&cfg, gemm_bf16_kernel, tmA, tmB, args);
}

Args make_args(int mode, const GemmShape& s, const GemmBuffers& b) {
  Args a;
  a.mode = mode;
  a.K = s.K;
  a.BN = s.BN;
  a.n_tiles = s.N / s.BN;
  a.k_blocks = (s.K + 63) / 64;
  a.w_rows_per_expert = s.w_rows_per_expert;
  a.k_total = s.k_total;
  a.num_pairs = s.num_pairs;
  a.activation = s.activation;
  a.out_cols = s.out_cols;
  a.num_blocks = b.num_blocks;
  a.block_expert = b.block_expert;
  a.sorted_pair_ids = b.sorted_pair_ids;
  a.topk_w = b.topk_w;
  a.out = b.out;
  a.status = b.status;
  return a;
}

}  // namespace

int pick_bn(int N, bool gated) {
  (void)gated;
  for (int bn = kMaxBN; bn >= 32; bn -= 32)
    if (N % bn == 0) return bn;
  return 0;
}

size_t gemm_bf16_smem_bytes() { return kSmemBytes; }

cudaError_t launch_gemm1_bf16(const Launch& l, const CUtensorMap& tm_hidden, const CUtensorMap& tm_w13,
                              const GemmShape& s, const GemmBuffers& b) {
  return launch(l, tm_hidden, tm_w13, make_args(0, s, b), s.num_sms);
}

cudaError_t launch_gemm2_bf16(const Launch& l, const CUtensorMap& tm_act, const CUtensorMap& tm_w2,
                              const GemmShape& s, const GemmBuffers& b) {
  return launch(l, tm_act, tm_w2, make_args(1, s, b), s.num_sms);
}

}  // namespace moe
