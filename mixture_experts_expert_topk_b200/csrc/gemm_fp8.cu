// Steps 3 and 4 of the layer for FP8 E4M3 W8A8 with 128x128 weight blocks and 1x128
// activation groups ("Qwen3-Next FP8 MoE optimisation: shared-expert fusion for H200",
// sglang PR 26204, section 1: dtype=fp8_w8a8, block_shape=[128, 128]).
//
// The operands are e4m3 codes with one fp32 scale per 128-element K group (activations,
// per row) and per 128x128 block (weights). The scales are arbitrary fp32 (amax/448), so
// they cannot ride on the tensor core's power-of-two block scaling; instead every
// 128-wide K block is its own tcgen05.mma (kind::f8f6f4, 4 x K=32) into a fresh fp32
// partial in TMEM, and the epilogue warps "promote" it: acc += partial * (s_a * s_w), in
// registers. Partials are double-buffered in TMEM so the MMAs of K block kb+1 run while
// block kb is promoted.
//
// GEMM1: A = quantised hidden rows gathered per sorted row (cp.async), B = the prepared
// (gate/up-interleaved) w13 codes; an N tile of 128 interleaved rows is 64 gate/up pairs,
// whose weight scales are the gate block and the up block of the checkpoint layout. The
// epilogue applies silu(gate)*up (or relu2) and writes bf16 activations; a separate pass
// quantises them per 1x128 group for GEMM2.
// GEMM2: A = the quantised activations (TMA), B = w2 codes; one N tile is one 128-row
// weight-scale block. The epilogue multiplies by the routing weight and writes fp32 y in
// sorted row order, like the bf16 path.
//
// Warp roles, rings, tile scheduling and TMA-store epilogue follow gemm_bf16.cu.
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kBKBytes = 128;           // 128 e4m3 of K per stage: one quantisation group
constexpr int kStageA = kBM * kBKBytes;  // 16 KB
constexpr int kStageB = kBN * kBKBytes;  // 16 KB
constexpr int kStagesA = 4;
constexpr int kStagesB = 6;
constexpr int kNumAWarps = 2;  // 8 warps in all, so the promotion warps may use up to 255 registers
constexpr int kWarpSched = 2;
constexpr int kWarpMma = 3;
constexpr int kWarpEpi = 4;
constexpr int kThreads = 256;
constexpr int kRowsPerAThread = kBM / (kNumAWarps * 32 / 8);  // 16
constexpr int kTmemCols = 256;  // two 128-column partial buffers
constexpr int kTileRing = 4;
constexpr int kStagingBuf = 32 * 128;
constexpr int kStagingOffset = kStagesA * kStageA + kStagesB * kStageB;
constexpr int kBarOffset = kStagingOffset + 4 * 2 * kStagingBuf;
constexpr int kSmemBytes = kBarOffset + 512 + 1024;

enum : int {
  kSiteEmptyB = 1, kSiteFullA = 2, kSitePartEmpty = 3, kSitePartFull = 4, kSiteFullB = 5, kSiteEmptyA = 6,
  kSiteTileFull = 7, kSiteTileEmpty = 8
};

struct Args {
  int mode;  // 0 = GEMM1, 1 = GEMM2
  int n_tiles, k_blocks;
  int w_rows_per_expert;
  int k_total, num_pairs, activation;
  const uint8_t* a_rows;        // GEMM1: quantised hidden [T, H] e4m3
  int a_row_bytes;              // GEMM1: H
  const float* a_scale;         // GEMM1: [T, H/128] per token; GEMM2: [rows, I/128] per sorted row
  int a_scale_cols;             // K / 128
  const float* w_scale;         // [E, w_scale_rows, w_scale_cols]
  int w_scale_rows, w_scale_cols;
  int up_block_offset;          // GEMM1 gated: scale-block row of up row 0 (I / 128)
  const int* num_blocks;
  const int* block_expert;
  const int* sorted_pair_ids;
  const float* topk_w;
  int* tile_counter;
  int* status;
};

__device__ __forceinline__ int token_of(const Args& a, int row) {
  const int pid = a.sorted_pair_ids[row];
  return pid < a.num_pairs ? pid / a.k_total : 0;
}

__device__ __forceinline__ int ring_take(uint32_t tfull0, uint32_t tempty0, volatile int* ring, int& slot,
                                         uint32_t& ph, volatile int* abort, int* status) {
  int tile = -2;
  if (mbar_wait(tfull0 + 8 * slot, ph, abort, status, kSiteTileFull)) tile = ring[slot];
  mbar_arrive(tempty0 + 8 * slot);
  if (++slot == kTileRing) {
    slot = 0;
    ph ^= 1u;
  }
  return tile;
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_fp8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmC, const Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + kStagesA * kStageA;
  const uint32_t sStage = sA + kStagingOffset;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOffset);
  const uint32_t fullA0 = smem_u32(bars);
  const uint32_t emptyA0 = fullA0 + 8 * kStagesA;
  const uint32_t fullB0 = emptyA0 + 8 * kStagesA;
  const uint32_t emptyB0 = fullB0 + 8 * kStagesB;
  const uint32_t pfull0 = emptyB0 + 8 * kStagesB;
  const uint32_t pempty0 = pfull0 + 16;
  const uint32_t ringfull0 = pempty0 + 16;
  const uint32_t ringempty0 = ringfull0 + 8 * kTileRing;
  const uint32_t drain_bar = ringempty0 + 8 * kTileRing;
  volatile int* ring = reinterpret_cast<volatile int*>(bars + 2 * kStagesA + 2 * kStagesB + 4 + 2 * kTileRing + 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(const_cast<int*>(ring) + kTileRing);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool gather_a = a.mode == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesA; ++s) {
      mbar_init(fullA0 + 8 * s, gather_a ? 32 * kNumAWarps : 1);
      mbar_init(emptyA0 + 8 * s, 1);
    }
    for (int s = 0; s < kStagesB; ++s) {
      mbar_init(fullB0 + 8 * s, 1);
      mbar_init(emptyB0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(pfull0 + 8 * b, 1);
      mbar_init(pempty0 + 8 * b, 4);  // one arrival per epilogue warp
    }
    const uint32_t readers = (gather_a ? kNumAWarps : 1) + 1 + 4;
    for (int s = 0; s < kTileRing; ++s) {
      mbar_init(ringfull0 + 8 * s, 1);
      mbar_init(ringempty0 + 8 * s, readers);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpSched && lane == 0) prefetch_tmap(&tmB);
  if (warp == 0 && lane == 0 && !gather_a) prefetch_tmap(&tmA);
  if (warp == kWarpEpi && lane == 0) prefetch_tmap(&tmC);
  if (warp == kWarpMma) {
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

  if (warp < kNumAWarps) {
    if (gather_a) {
      // ---------------- A gather (cp.async), both A warps ----------------
      const int t = threadIdx.x;  // 0..63
      const int c = t & 7;        // 16-byte chunk of the 128-byte K slice
      const int r0 = t >> 3;      // rows r0 + 8 i, i = 0..15
      int rslot = 0, sa = 0;
      uint32_t rph = 0, pha = 0;
      while (true) {
        int tile = 0;
        if (lane == 0) tile = ring_take(ringfull0, ringempty0, ring, rslot, rph, abort_flag, a.status);
        tile = __shfl_sync(0xffffffffu, tile, 0);
        if (tile < 0) break;
        const int mb = tile / a.n_tiles;
        const uint8_t* src[kRowsPerAThread];
#pragma unroll
        for (int i = 0; i < kRowsPerAThread; ++i)
          src[i] = a.a_rows + static_cast<size_t>(token_of(a, mb * kBM + r0 + 8 * i)) * a.a_row_bytes + c * 16;
        bool ok = true;
        for (int kb = 0; kb < a.k_blocks; ++kb) {
          int got = 0;
          if (lane == 0) got = mbar_wait(emptyA0 + 8 * sa, pha ^ 1u, abort_flag, a.status, kSiteEmptyA);
          if (!__shfl_sync(0xffffffffu, got, 0)) {
            ok = false;
            break;
          }
          const uint32_t base = sA + sa * kStageA;
#pragma unroll
          for (int i = 0; i < kRowsPerAThread; ++i) {
            const int r = r0 + 8 * i;
            cp_async16(base + r * kBKBytes + ((c ^ (r & 7)) << 4), src[i] + kb * kBKBytes);
          }
          cp_async_mbar_arrive(fullA0 + 8 * sa);
          if (++sa == kStagesA) {
            sa = 0;
            pha ^= 1u;
          }
        }
        if (!ok) break;
      }
      cp_async_wait_all();
    } else if (warp == 0 && lane == 0) {
      // ---------------- A tile (TMA), GEMM2 ----------------
      const uint64_t pol_a = policy_evict_last();
      int rslot = 0, sa = 0;
      uint32_t rph = 0, pha = 0;
      uint32_t fills = 0;
      bool ok = true;
      while (ok) {
        const int tile = ring_take(ringfull0, ringempty0, ring, rslot, rph, abort_flag, a.status);
        if (tile < 0) break;
        const int mb = tile / a.n_tiles;
        for (int kb = 0; kb < a.k_blocks; ++kb) {
          if (!mbar_wait(emptyA0 + 8 * sa, pha ^ 1u, abort_flag, a.status, kSiteEmptyA)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(fullA0 + 8 * sa, kStageA);
          tma_load_2d(sA + sa * kStageA, &tmA, fullA0 + 8 * sa, kb * kBKBytes, mb * kBM, pol_a);
          ++fills;
          if (++sa == kStagesA) {
            sa = 0;
            pha ^= 1u;
          }
        }
      }
      drain_fills(fullA0, kStagesA, fills);  // no A copy may land after the CTA exits
    }
  } else if (warp == kWarpSched) {
    // ---------------- tile scheduler + B producer ----------------
    if (lane == 0) {
      const uint64_t pol_b = gather_a ? policy_evict_first() : policy_evict_last();
      int wslot = 0, sb = 0;
      uint32_t wph = 0, phb = 0;
      uint32_t fills = 0;
      // the first tile is the CTA index; later ones come from the counter, after the grid's first tiles
      int tile = static_cast<int>(blockIdx.x);
      while (true) {
        if (!mbar_wait(ringempty0 + 8 * wslot, wph ^ 1u, abort_flag, a.status, kSiteTileEmpty)) break;
        const bool done = tile >= num_tiles;
        ring[wslot] = done ? -1 : tile;
        mbar_arrive(ringfull0 + 8 * wslot);
        if (++wslot == kTileRing) {
          wslot = 0;
          wph ^= 1u;
        }
        if (done) break;
        const int next = static_cast<int>(gridDim.x) + atomicAdd(a.tile_counter, 1);
        const int mb = tile / a.n_tiles;
        const int nt = tile - mb * a.n_tiles;
        const int brow = a.block_expert[mb] * a.w_rows_per_expert + nt * kBN;
        bool ok = true;
        for (int kb = 0; kb < a.k_blocks; ++kb) {
          if (!mbar_wait(emptyB0 + 8 * sb, phb ^ 1u, abort_flag, a.status, kSiteEmptyB)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(fullB0 + 8 * sb, kStageB);
          tma_load_2d(sB + sb * kStageB, &tmB, fullB0 + 8 * sb, kb * kBKBytes, brow, pol_b);
          ++fills;
          if (++sb == kStagesB) {
            sb = 0;
            phb ^= 1u;
          }
        }
        if (!ok) break;
        tile = next;
      }
      drain_fills(fullB0, kStagesB, fills);  // no B copy may land after the CTA exits
    }
  } else if (warp == kWarpMma) {
    // ---------------- MMA issuer: one partial per K block ----------------
    if (lane == 0) {
      const uint32_t idesc = idesc_e4m3(kBM, kBN);
      int rslot = 0, sa = 0, sb = 0;
      uint32_t rph = 0, pha = 0, phb = 0;
      int np = 0;  // partials issued
      bool ok = true;
      while (ok) {
        const int tile = ring_take(ringfull0, ringempty0, ring, rslot, rph, abort_flag, a.status);
        if (tile < 0) break;
        for (int kb = 0; kb < a.k_blocks; ++kb, ++np) {
          const int pb = np & 1;
          const uint32_t pph = (np >> 1) & 1;
          if (!mbar_wait(pempty0 + 8 * pb, pph ^ 1u, abort_flag, a.status, kSitePartEmpty) ||
              !mbar_wait(fullA0 + 8 * sa, pha, abort_flag, a.status, kSiteFullA) ||
              !mbar_wait(fullB0 + 8 * sb, phb, abort_flag, a.status, kSiteFullB)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + pb * kBN;
          const uint64_t adesc = umma_desc_sw128(sA + sa * kStageA);
          const uint64_t bdesc = umma_desc_sw128(sB + sb * kStageB);
#pragma unroll
          for (int k = 0; k < 4; ++k)  // 4 x K=32 e4m3 = 128 bytes; +32 bytes = +2 encoded
            umma_e4m3(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, k != 0);
          umma_commit(emptyA0 + 8 * sa);
          umma_commit(emptyB0 + 8 * sb);
          umma_commit(pfull0 + 8 * pb);
          if (++sa == kStagesA) {
            sa = 0;
            pha ^= 1u;
          }
          if (++sb == kStagesB) {
            sb = 0;
            phb ^= 1u;
          }
        }
      }
      umma_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0);
    }
  } else {
    // ---------------- promotion + epilogue (warps 6..9) ----------------
    const int q = warp & 3;
    const uint32_t staging = sStage + (warp - kWarpEpi) * 2 * kStagingBuf;
    const bool gated = a.activation != 1;  // 0 SwiGLU, 2 gelu_tanh, 3 swigluoai; 1 relu2
    int nst = 0;
    int np = 0;
    int rslot = 0;
    uint32_t rph = 0;
    while (true) {
      int tile = 0;
      if (lane == 0) tile = ring_take(ringfull0, ringempty0, ring, rslot, rph, abort_flag, a.status);
      tile = __shfl_sync(0xffffffffu, tile, 0);
      if (tile < 0) break;
      const int mb = tile / a.n_tiles;
      const int nt = tile - mb * a.n_tiles;
      const int grow0 = mb * kBM + q * 32;
      const int row = grow0 + lane;
      const int pid = a.sorted_pair_ids[row];
      const bool valid = pid < a.num_pairs;
      const int e = a.block_expert[mb];
      // activation scale row: GEMM1 per token, GEMM2 per sorted row
      const float* sa_row = a.a_scale + static_cast<size_t>(gather_a ? (valid ? pid / a.k_total : 0) : row) *
                                            a.a_scale_cols;
      // weight scale rows of this N tile: gated GEMM1 pairs a gate block and an up block
      const float* sw_base = a.w_scale + static_cast<size_t>(e) * a.w_scale_rows * a.w_scale_cols;
      const float* sw_even;
      const float* sw_odd;
      if (gather_a && gated) {
        sw_even = sw_base + static_cast<size_t>(nt / 2) * a.w_scale_cols;
        sw_odd = sw_base + static_cast<size_t>(a.up_block_offset + nt / 2) * a.w_scale_cols;
      } else {
        sw_even = sw_odd = sw_base + static_cast<size_t>(nt) * a.w_scale_cols;
      }
      // the tile's weight scales, lane k holding K block k (k_blocks <= 32), read once;
      // the row's activation scale is fetched one K block ahead
      const float sw_even_l = lane < a.k_blocks ? __ldg(sw_even + lane) : 0.f;
      const float sw_odd_l = lane < a.k_blocks ? __ldg(sw_odd + lane) : 0.f;
      float sa_next = __ldg(sa_row);
      float acc[kBN];
#pragma unroll
      for (int i = 0; i < kBN; ++i) acc[i] = 0.f;
      bool ok = true;
      for (int kb = 0; kb < a.k_blocks; ++kb, ++np) {
        const int pb = np & 1;
        const uint32_t pph = (np >> 1) & 1;
        const float s_a = sa_next;
        if (kb + 1 < a.k_blocks) sa_next = __ldg(sa_row + kb + 1);
        const float s_even = s_a * __shfl_sync(0xffffffffu, sw_even_l, kb);
        const float s_odd = s_a * __shfl_sync(0xffffffffu, sw_odd_l, kb);
        const bool got = mbar_wait(pfull0 + 8 * pb, pph, abort_flag, a.status, kSitePartFull);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + pb * kBN;
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) {
          uint32_t v[32];
          __syncwarp();
          tmem_ld32(taddr + c * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            acc[c * 32 + i] = fmaf(__uint_as_float(v[i]), s_even, acc[c * 32 + i]);
            acc[c * 32 + i + 1] = fmaf(__uint_as_float(v[i + 1]), s_odd, acc[c * 32 + i + 1]);
          }
        }
        tc_fence_before();
        __syncwarp();  // every lane's loads of the partial are complete
        if (lane == 0) mbar_arrive(pempty0 + 8 * pb);
      }
      if (!ok) break;
      const bool any_valid = __ballot_sync(0xffffffffu, valid) != 0u;
      if (gather_a) {
        // activation -> bf16, boxes of 32 rows x 64 columns (128 B rows, 128-byte swizzle)
        const int nbox = gated ? 1 : 2;
        const int col0 = nt * (gated ? kBN / 2 : kBN);
#pragma unroll
        for (int bx = 0; bx < 2; ++bx) {
          if (bx >= nbox) break;
          const uint32_t buf = staging + (nst & 1) * kStagingBuf;
          if (nst >= 2 && lane == 0) bulk_wait_group_read<1>();
          __syncwarp();
          uint32_t o[32];
          if (gated) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              o[i] = pack_bf16x2(gated_act(acc[4 * i], acc[4 * i + 1], a.activation),
                                 gated_act(acc[4 * i + 2], acc[4 * i + 3], a.activation));
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float z0 = fmaxf(acc[bx * 64 + 2 * i], 0.f), z1 = fmaxf(acc[bx * 64 + 2 * i + 1], 0.f);
              o[i] = pack_bf16x2(z0 * z0, z1 * z1);
            }
          }
          const uint32_t dst = buf + lane * 128;
#pragma unroll
          for (int s8 = 0; s8 < 8; ++s8)
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst + ((s8 ^ (lane & 7)) << 4)),
                         "r"(o[4 * s8]), "r"(o[4 * s8 + 1]), "r"(o[4 * s8 + 2]), "r"(o[4 * s8 + 3]) : "memory");
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && any_valid) {
            tma_store_2d(&tmC, buf, col0 + bx * 64, grow0);
            bulk_commit_group();
          }
          ++nst;
        }
      } else {
        // y = w * acc in fp32, boxes of 32 rows x 32 columns (128-byte swizzle)
        const float w = valid ? a.topk_w[pid] : 0.f;
#pragma unroll
        for (int bx = 0; bx < kBN / 32; ++bx) {
          const uint32_t buf = staging + (nst & 1) * kStagingBuf;
          if (nst >= 2 && lane == 0) bulk_wait_group_read<1>();
          __syncwarp();
          const uint32_t dst = buf + lane * 128;
#pragma unroll
          for (int s8 = 0; s8 < 8; ++s8)
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst + ((s8 ^ (lane & 7)) << 4)),
                         "f"(acc[bx * 32 + 4 * s8] * w), "f"(acc[bx * 32 + 4 * s8 + 1] * w),
                         "f"(acc[bx * 32 + 4 * s8 + 2] * w), "f"(acc[bx * 32 + 4 * s8 + 3] * w) : "memory");
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && any_valid) {
            tma_store_2d(&tmC, buf, nt * kBN + bx * 32, grow0);
            bulk_commit_group();
          }
          ++nst;
        }
      }
    }
    if (lane == 0) bulk_wait_group<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(a.tile_counter + 1, 1) == static_cast<int>(gridDim.x) - 1) {
      a.tile_counter[0] = 0;
      a.tile_counter[1] = 0;
    }
  }
}

bool g_attr_set[64] = {};

cudaError_t launch(const Launch& l, const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmC,
                   const Args& args, int num_sms) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 64 && !g_attr_set[dev]) {
    err = cudaFuncSetAttribute(gemm_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return err;
    g_attr_set[dev] = true;
  }
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(num_sms), dim3(kThreads), kSmemBytes);
  return cudaLaunchKernelEx(&cfg, gemm_fp8_kernel, tmA, tmB, tmC, args);
}

Args make_args(int mode, const GemmShape& s, const GemmBuffers& b, const void* a_rows) {
  Args a;
  a.mode = mode;
  a.n_tiles = s.N / kBN;
  a.k_blocks = s.K / 128;
  a.w_rows_per_expert = s.w_rows_per_expert;
  a.k_total = s.k_total;
  a.num_pairs = s.num_pairs;
  a.activation = s.activation;
  a.a_rows = static_cast<const uint8_t*>(a_rows);
  a.a_row_bytes = s.K;
  a.a_scale = b.a_scale;
  a.a_scale_cols = b.a_scale_cols;
  a.w_scale = b.w_scale;
  a.w_scale_rows = b.w_scale_rows;
  a.w_scale_cols = b.w_scale_cols;
  a.up_block_offset = b.up_block_offset;
  a.num_blocks = b.num_blocks;
  a.block_expert = b.block_expert;
  a.sorted_pair_ids = b.sorted_pair_ids;
  a.topk_w = b.topk_w;
  a.tile_counter = b.tile_counter;
  a.status = b.status;
  return a;
}

}  // namespace

size_t gemm_fp8_smem_bytes() { return kSmemBytes; }

cudaError_t launch_gemm1_fp8(const Launch& l, const void* xq, const CUtensorMap& tm_w13,
                             const CUtensorMap& tm_act_store, const GemmShape& s, const GemmBuffers& b) {
  return launch(l, tm_w13, tm_w13, tm_act_store, make_args(0, s, b, xq), s.num_sms);
}

cudaError_t launch_gemm2_fp8(const Launch& l, const CUtensorMap& tm_actq, const CUtensorMap& tm_w2,
                             const CUtensorMap& tm_y_store, const GemmShape& s, const GemmBuffers& b) {
  return launch(l, tm_actq, tm_w2, tm_y_store, make_args(1, s, b, nullptr), s.num_sms);
}

}  // namespace moe
