// Steps 3 and 4 of the layer in bf16: the two grouped GEMMs over the expert-sorted rows.
//
// GEMM1 (up-GEMM with fused activation; "[MoE] SwiGLU fusion into the MoE up-GEMM
// epilogue", sglang PR 32944, sections 1 and 3): row r of the sorted order belongs to
// pair p = sorted_pair_ids[r] and expert e = block_expert[r / 128]; its A row is
// hidden[p / k'], gathered straight from the token-order hidden tensor. B is the
// prepared w13 of expert e, whose gate and up rows are interleaved ([gate0, up0, gate1,
// up1, ...]), so accumulator columns (2j, 2j+1) of a tile hold gate_j and up_j. The
// epilogue applies silu(gate)*up (or relu2) to the fp32 accumulators in registers and
// writes only the I-wide bf16 activation.
//
// GEMM2 (down-GEMM with routing weight): A is the activation in sorted row order, B is
// w2 of the row tile's expert; the epilogue multiplies row r by topk_w[p] and writes it
// in fp32 to row r of y (sorted order); the fixed-order combine gathers it back through
// pair_to_row.
//
// Kernel structure (one persistent CTA per SM, 10 warps):
//   warps 0-3   GEMM1 A gather: 128 threads copy the tile's 128 token rows, 128 bytes of
//               K each per stage, with 16-byte cp.async into the 128-byte-swizzled layout
//               the MMA reads; each thread's copies arrive on the stage's barrier when they
//               land (cp.async.mbarrier.arrive). A TMA gather4 per 4 rows was measured to
//               cap the producer at one stage per ~1.3 us; cp.async keeps up with HBM.
//   warp 4      TMA: B tile (weights, 2-D tiled load, 128-byte swizzle) and, for GEMM2,
//               the contiguous A tile; 4-stage ring of 48 KB stages;
//   warp 5      TMEM allocator and MMA issuer: tcgen05.mma kind::f16, M=128, N=BN, K=16,
//               fp32 accumulators in TMEM, double-buffered (2 x 256 columns) so the
//               epilogue of tile i overlaps the main loop of tile i+1;
//   warps 6-9   epilogue: tcgen05.ld 32 columns at a time, activation / weighting in
//               registers, 32-row boxes staged in shared memory and written with TMA
//               tensor stores (double-buffered per warp).
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
constexpr int kNumAWarps = 4;
constexpr int kWarpTma = 4;
constexpr int kWarpMma = 5;
constexpr int kWarpEpi = 6;
constexpr int kThreads = 320;
constexpr int kAccCols = 256;               // TMEM columns per accumulator buffer
constexpr int kTmemCols = 512;
constexpr int kStagingBuf = 32 * 128;       // one 32-row epilogue box (<= 128 B per row)
constexpr int kStagingBytes = 2 * kStagingBuf;  // double-buffered per epilogue warp
constexpr int kStagingOffset = kStages * kStageBytes;
constexpr int kBarOffset = kStagingOffset + 4 * kStagingBytes;
constexpr int kSmemBytes = kBarOffset + 256 + 1024;  // barriers + 1024-byte alignment slack

// wait sites (device status detail)
enum : int { kSiteEmpty = 1, kSiteFull = 2, kSiteTmemEmpty = 3, kSiteTmemFull = 4, kSiteEmptyA = 6 };

struct Args {
  int mode;  // 0 = GEMM1 (gather + activation), 1 = GEMM2 (weighted scatter)
  int K, BN, n_tiles, k_blocks;
  int w_rows_per_expert;
  int k_total, num_pairs, activation, out_cols;
  const uint8_t* a_rows;  // GEMM1: hidden [T, H] bf16
  int a_row_bytes;        // GEMM1: H * 2
  const int* num_blocks;
  const int* block_expert;
  const int* sorted_pair_ids;
  const float* topk_w;
  void* out;  // unused by the kernel: outputs go through the store tensor map
  int* status;
};

__device__ __forceinline__ int token_of(const Args& a, int row) {
  const int pid = a.sorted_pair_ids[row];
  return pid < a.num_pairs ? pid / a.k_total : 0;  // padding rows read token 0
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, const Args a) {
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
  const bool gather_a = a.mode == 0;

  if (threadIdx.x == 0) {
    // GEMM1: the B copy's expect-tx arrival plus one cp.async arrival per gather thread
    const uint32_t full_count = gather_a ? 1 + 32 * kNumAWarps : 1;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full0 + 8 * s, full_count);
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
  if (warp == kWarpTma && lane == 0) {
    prefetch_tmap(&tmB);
    if (!gather_a) prefetch_tmap(&tmA);
  }
  if (warp == kWarpEpi && lane == 0) prefetch_tmap(&tmC);
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // everything above overlaps the previous kernel; inputs are read only after this
  griddep_wait();
  griddep_launch_dependents();
  const int num_tiles = *a.num_blocks * a.n_tiles;

  if (warp < kNumAWarps) {
    if (gather_a) {
      // ---------------- A gather (cp.async) ----------------
      const int t = threadIdx.x;  // 0..127
      const int c = t & 7;        // 16-byte chunk of the 128-byte K slice
      const int r0 = t >> 3;      // rows r0 + 16 i, i = 0..7
      int stage = 0;
      uint32_t phase = 0;
      int tok_next[8];
      if (static_cast<int>(blockIdx.x) < num_tiles) {
        const int mb = blockIdx.x / a.n_tiles;
#pragma unroll
        for (int i = 0; i < 8; ++i) tok_next[i] = token_of(a, mb * kBM + r0 + 16 * i);
      }
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const uint8_t* src[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          src[i] = a.a_rows + static_cast<size_t>(tok_next[i]) * a.a_row_bytes + c * 16;
        const int next = tile + gridDim.x;
        if (next < num_tiles) {  // prefetch the next tile's token rows
          const int mb = next / a.n_tiles;
#pragma unroll
          for (int i = 0; i < 8; ++i) tok_next[i] = token_of(a, mb * kBM + r0 + 16 * i);
        }
        for (int kb = 0; kb < a.k_blocks; ++kb) {
          int got = 0;
          if (lane == 0) got = mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag, a.status, kSiteEmptyA);
          got = __shfl_sync(0xffffffffu, got, 0);
          if (!got) {
            ok = false;
            break;
          }
          const uint32_t base = smem_u32(smem + stage * kStageBytes);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int r = r0 + 16 * i;
            cp_async16(base + r * kBKBytes + ((c ^ (r & 7)) << 4), src[i] + kb * kBKBytes);
          }
          cp_async_mbar_arrive(full0 + 8 * stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      cp_async_wait_all();  // no copy may land after the CTA exits
    }
  } else if (warp == kWarpTma) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();  // weights: streamed once
      const uint64_t pol_a = policy_evict_last();   // activations: reused across N tiles
      const uint32_t bytes = static_cast<uint32_t>(a.BN) * kBKBytes + (gather_a ? 0u : kStageA);
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      int e_next = static_cast<int>(blockIdx.x) < num_tiles ? a.block_expert[blockIdx.x / a.n_tiles] : 0;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int mb = tile / a.n_tiles;
        const int nt = tile - mb * a.n_tiles;
        const int e = e_next;
        const int next = tile + gridDim.x;
        if (next < num_tiles) e_next = a.block_expert[next / a.n_tiles];
        const int brow = e * a.w_rows_per_expert + nt * a.BN;
        for (int kb = 0; kb < a.k_blocks; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag, a.status, kSiteEmpty)) {
            ok = false;
            break;
          }
          const uint32_t full = full0 + 8 * stage;
          const uint32_t a_dst = smem_u32(smem + stage * kStageBytes);
          mbar_arrive_expect_tx(full, bytes);
          // GEMM1 streams each weight tile once; GEMM2's weight tiles are short rows
          // re-read at the next K step, so they keep the normal eviction priority
          tma_load_2d(a_dst + kStageA, &tmB, full, kb * 64, brow, gather_a ? pol_w : pol_a);
          if (!gather_a) tma_load_2d(a_dst, &tmA, full, kb * 64, mb * kBM, pol_a);
          ++issued;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // wait (bounded) for the last copy issued into each stage
        for (int s = 0; s < kStages; ++s) {
          if (issued <= s) break;
          const long long last = issued - 1 - ((issued - 1 - s) % kStages);
          mbar_wait_drain(full0 + 8 * s, static_cast<uint32_t>((last / kStages) & 1));
        }
      }
    }
  } else if (warp == kWarpMma) {
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
    // ---------------- epilogue (warps 6..9) ----------------
    // Each warp owns 32 accumulator rows (its TMEM lane quadrant). Per 32 accumulator
    // columns it writes one box of 32 output rows to shared memory and stores it with a
    // TMA tensor store; two staging buffers let the next box be written while the
    // previous store drains.
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const uint32_t staging = smem_u32(smem + kStagingOffset + (warp - kWarpEpi) * kStagingBytes);
    const bool gated = a.activation == 0;
    // GEMM1: act bf16 rows of 16 (gated) or 32 (relu2) columns per box, no swizzle;
    // GEMM2: y fp32 rows of 32 columns (128 B), 128-byte swizzle
    const int box_cols = a.mode == 0 ? (gated ? 16 : 32) : 32;
    int nst = 0;  // boxes this warp has staged (selects the staging buffer)
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      const uint32_t aphase = (it >> 1) & 1;
      const bool got = mbar_wait(tfull0 + 8 * acc, aphase, abort_flag, a.status, kSiteTmemFull);
      if (!__all_sync(0xffffffffu, got)) break;  // leave warp-uniformly (tcgen05.ld is .aligned)
      tc_fence_after();
      const int mb = tile / a.n_tiles;
      const int nt = tile - mb * a.n_tiles;
      const int grow0 = mb * kBM + q * 32;
      const int pid = a.sorted_pair_ids[grow0 + lane];
      const bool valid = pid < a.num_pairs;
      const bool any_valid = __ballot_sync(0xffffffffu, valid) != 0u;  // skip all-padding boxes
      const float w = (a.mode != 0 && valid) ? a.topk_w[pid] : 0.f;
      const int col0 = nt * (a.mode == 0 && gated ? a.BN / 2 : a.BN);
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * kAccCols;
      for (int c = 0; c < a.BN / 32; ++c, ++nst) {
        const uint32_t buf = staging + (nst & 1) * kStagingBuf;
        if (nst >= 2) {
          if (lane == 0) bulk_wait_group_read<1>();  // the store that last used `buf` has read it
        }
        __syncwarp();  // also: tcgen05.ld below is .sync.aligned
        uint32_t v[32];
        tmem_ld32(taddr + c * 32, v);
        tmem_wait_ld();
        if (a.mode == 0) {
          if (gated) {
            uint32_t o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float g0 = __uint_as_float(v[4 * i + 0]), u0 = __uint_as_float(v[4 * i + 1]);
              const float g1 = __uint_as_float(v[4 * i + 2]), u1 = __uint_as_float(v[4 * i + 3]);
              o[i] = pack_bf16x2(silu_f32(g0) * u0, silu_f32(g1) * u1);
            }
            const uint32_t dst = buf + lane * 32;
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(o[0]), "r"(o[1]), "r"(o[2]),
                         "r"(o[3]) : "memory");
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst + 16), "r"(o[4]), "r"(o[5]),
                         "r"(o[6]), "r"(o[7]) : "memory");
          } else {
            uint32_t o[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float z0 = fmaxf(__uint_as_float(v[2 * i + 0]), 0.f);
              const float z1 = fmaxf(__uint_as_float(v[2 * i + 1]), 0.f);
              o[i] = pack_bf16x2(z0 * z0, z1 * z1);
            }
            const uint32_t dst = buf + lane * 64;
#pragma unroll
            for (int s4 = 0; s4 < 4; ++s4)
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst + 16 * s4), "r"(o[4 * s4]),
                           "r"(o[4 * s4 + 1]), "r"(o[4 * s4 + 2]), "r"(o[4 * s4 + 3]) : "memory");
          }
        } else {
          // 128-byte swizzle: 16-byte chunk s of row r lives at chunk (s ^ (r & 7))
          const uint32_t dst = buf + lane * 128;
#pragma unroll
          for (int s8 = 0; s8 < 8; ++s8)
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst + ((s8 ^ (lane & 7)) << 4)),
                         "f"(__uint_as_float(v[4 * s8]) * w), "f"(__uint_as_float(v[4 * s8 + 1]) * w),
                         "f"(__uint_as_float(v[4 * s8 + 2]) * w), "f"(__uint_as_float(v[4 * s8 + 3]) * w)
                         : "memory");
        }
        fence_proxy_async_smem();  // the generic-proxy writes above feed an async-proxy store
        __syncwarp();
        if (lane == 0 && any_valid) {
          tma_store_2d(&tmC, buf, col0 + c * box_cols, grow0);
          bulk_commit_group();
        }
      }
      tc_fence_before();
      mbar_arrive(tempty0 + 8 * acc);
    }
    if (lane == 0) bulk_wait_group<0>();  // stores complete before the CTA retires
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    __syncwarp();  // tcgen05.dealloc is .sync.aligned: the whole warp, converged
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

bool g_attr_set[64] = {};

cudaError_t launch(const Launch& l, const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmC,
                   const Args& args, int num_sms) {
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
  return cudaLaunchKernelEx(&cfg, gemm_bf16_kernel, tmA, tmB, tmC, args);
}

Args make_args(int mode, const GemmShape& s, const GemmBuffers& b, const void* a_rows) {
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
  a.a_rows = static_cast<const uint8_t*>(a_rows);
  a.a_row_bytes = s.K * 2;
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

cudaError_t launch_gemm1_bf16(const Launch& l, const void* hidden, const CUtensorMap& tm_w13,
                              const CUtensorMap& tm_act_store, const GemmShape& s, const GemmBuffers& b) {
  // the A operand is gathered with cp.async; tmA is not read in this mode
  return launch(l, tm_w13, tm_w13, tm_act_store, make_args(0, s, b, hidden), s.num_sms);
}

cudaError_t launch_gemm2_bf16(const Launch& l, const CUtensorMap& tm_act, const CUtensorMap& tm_w2,
                              const CUtensorMap& tm_y_store, const GemmShape& s, const GemmBuffers& b) {
  return launch(l, tm_act, tm_w2, tm_y_store, make_args(1, s, b, nullptr), s.num_sms);
}

}  // namespace moe
