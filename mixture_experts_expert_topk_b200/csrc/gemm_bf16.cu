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
//   warps 0-3   A producer. GEMM1: 128 threads gather the tile's 128 token rows, 128 bytes
//               of K each per stage, with 16-byte cp.async into the 128-byte-swizzled
//               layout the MMA reads; each thread's copies arrive on the stage barrier when
//               they land (cp.async.mbarrier.arrive). (A TMA gather4 per 4 rows was measured
//               to cap the producer at one stage per ~1.3 us.) GEMM2: warp 0 loads the
//               contiguous A tile with TMA.
//   warp 4      tile scheduler and B producer: takes tiles from a global atomic counter,
//               publishes them to the other roles through a small shared-memory ring, and
//               streams the weight tiles with TMA (2-D tiled loads, 128-byte swizzle).
//   warp 5      TMEM allocator and MMA issuer: tcgen05.mma kind::f16, M=128, N=BN, K=16,
//               fp32 accumulators in TMEM, double-buffered (2 x 256 columns) so the
//               epilogue of tile i overlaps the main loop of tile i+1.
//   warps 6-9   epilogue: tcgen05.ld 32 columns at a time, activation / weighting in
//               registers, 32-row boxes staged in shared memory and written with TMA
//               tensor stores.
// A and B have rings of their own: the weights (from HBM) keep more stages in flight
// than the activation rows (mostly L2 hits). Tiles are (row tile, N tile) pairs handed out
// in row-tile-major order, so CTAs running at the same time work on neighbouring row tiles
// of the same experts and share weight tiles in L2; taking them from a counter rather
// than a fixed stride lets CTAs whose tiles hit in L2 take more of them.
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kBM = 128;
constexpr int kBKBytes = 128;  // one 128-byte swizzle atom of K per stage
constexpr int kMaxBN = 256;
constexpr int kStageA = kBM * kBKBytes;     // 16 KB
constexpr int kStageB = kMaxBN * kBKBytes;  // 32 KB
constexpr int kNumAWarps = 4;
constexpr int kWarpSched = 4;
constexpr int kWarpMma = 5;
constexpr int kWarpEpi = 6;
constexpr int kThreads = 320;
constexpr int kAccCols = 256;  // TMEM columns per accumulator buffer
constexpr int kTmemCols = 512;
constexpr int kTileRing = 4;
constexpr int kBarBytes = 512;
constexpr int kSmemCap = 232448;  // opt-in shared memory per CTA on sm_100

// wait sites (device status detail)
enum : int {
  kSiteEmptyB = 1, kSiteFullA = 2, kSiteTmemEmpty = 3, kSiteTmemFull = 4, kSiteFullB = 5, kSiteEmptyA = 6,
  kSiteTileFull = 7, kSiteTileEmpty = 8
};

struct Args {
  int mode;  // 0 = GEMM1 (gather + activation), 1 = GEMM2 (weighted rows)
  int BN, n_tiles, k_blocks;
  int w_rows_per_expert;
  int k_total, num_pairs, activation;
  int stages_a, stages_b;            // ring depths
  int staging_bufs, staging_bytes;   // per epilogue warp: buffers and bytes per buffer
  const uint8_t* a_rows;  // GEMM1: hidden [T, H] bf16
  int a_row_bytes;        // GEMM1: H * 2
  const int* num_blocks;
  const int* block_expert;
  const int* sorted_pair_ids;
  const float* topk_w;
  int* tile_counter;  // [2]: next tile, CTAs finished; both 0 between launches
  int* status;
};

__host__ __device__ constexpr int smem_bytes(int sa, int sb, int bufs, int buf_bytes) {
  return sa * kStageA + sb * kStageB + 4 * bufs * buf_bytes + kBarBytes + 1024;
}

__device__ __forceinline__ int token_of(const Args& a, int row) {
  const int pid = a.sorted_pair_ids[row];
  return pid < a.num_pairs ? pid / a.k_total : 0;  // padding rows read token 0
}

// Reader side of the tile ring: the next tile id (or -1 when done, -2 on abort). Called
// by one thread; it releases the slot as soon as it has read it.
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
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, const Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int SA = a.stages_a, SB = a.stages_b;
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + SA * kStageA;
  const uint32_t sStage = sB + SB * kStageB;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SA * kStageA + SB * kStageB + 4 * a.staging_bufs * a.staging_bytes);
  const uint32_t fullA0 = smem_u32(bars);
  const uint32_t emptyA0 = fullA0 + 8 * SA;
  const uint32_t fullB0 = emptyA0 + 8 * SA;
  const uint32_t emptyB0 = fullB0 + 8 * SB;
  const uint32_t tfull0 = emptyB0 + 8 * SB;
  const uint32_t tempty0 = tfull0 + 16;
  const uint32_t ringfull0 = tempty0 + 16;
  const uint32_t ringempty0 = ringfull0 + 8 * kTileRing;
  const uint32_t drain_bar = ringempty0 + 8 * kTileRing;
  volatile int* ring = reinterpret_cast<volatile int*>(bars + 2 * SA + 2 * SB + 4 + 2 * kTileRing + 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(const_cast<int*>(ring) + kTileRing);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool gather_a = a.mode == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SA; ++s) {
      // GEMM1: one cp.async arrival per gather thread; GEMM2: the TMA expect-tx arrival
      mbar_init(fullA0 + 8 * s, gather_a ? 32 * kNumAWarps : 1);
      mbar_init(emptyA0 + 8 * s, 1);
    }
    for (int s = 0; s < SB; ++s) {
      mbar_init(fullB0 + 8 * s, 1);
      mbar_init(emptyB0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, 4);  // one arrival per epilogue warp
    }
    // tile-ring readers: the A warps (4 gathering, or the one TMA warp), MMA, 4 epilogue warps
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

  // everything above overlaps the previous kernel; inputs are read only after this
  griddep_wait();
  griddep_launch_dependents();
  const int num_tiles = *a.num_blocks * a.n_tiles;

  if (warp < kNumAWarps) {
    if (gather_a) {
      // ---------------- A gather (cp.async), all 4 warps ----------------
      const int t = threadIdx.x;  // 0..127
      const int c = t & 7;        // 16-byte chunk of the 128-byte K slice
      const int r0 = t >> 3;      // rows r0 + 16 i, i = 0..7
      int rslot = 0, sa = 0;
      uint32_t rph = 0, pha = 0;
      while (true) {
        int tile = 0;
        if (lane == 0) tile = ring_take(ringfull0, ringempty0, ring, rslot, rph, abort_flag, a.status);
        tile = __shfl_sync(0xffffffffu, tile, 0);
        if (tile < 0) break;
        const int mb = tile / a.n_tiles;
        const uint8_t* src[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          src[i] = a.a_rows + static_cast<size_t>(token_of(a, mb * kBM + r0 + 16 * i)) * a.a_row_bytes + c * 16;
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
          for (int i = 0; i < 8; ++i) {
            const int r = r0 + 16 * i;
            cp_async16(base + r * kBKBytes + ((c ^ (r & 7)) << 4), src[i] + kb * kBKBytes);
          }
          cp_async_mbar_arrive(fullA0 + 8 * sa);
          if (++sa == SA) {
            sa = 0;
            pha ^= 1u;
          }
        }
        if (!ok) break;
      }
      cp_async_wait_all();  // no copy may land after the CTA exits
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
          tma_load_2d(sA + sa * kStageA, &tmA, fullA0 + 8 * sa, kb * 64, mb * kBM, pol_a);
          ++fills;
          if (++sa == SA) {
            sa = 0;
            pha ^= 1u;
          }
        }
      }
      drain_fills(fullA0, SA, fills);  // no A copy may land after the CTA exits
    }
  } else if (warp == kWarpSched) {
    // ---------------- tile scheduler + B producer ----------------
    if (lane == 0) {
      // GEMM1 streams each weight tile once; GEMM2's weight rows are short and re-read at
      // the next K step, so they keep the normal eviction priority
      const uint64_t pol_b = gather_a ? policy_evict_first() : policy_evict_last();
      const uint32_t b_bytes = static_cast<uint32_t>(a.BN) * kBKBytes;
      int wslot = 0, sb = 0;
      uint32_t wph = 0, phb = 0;
      uint32_t fills = 0;
      // the first tile is the CTA index; later ones come from the counter, after the grid's first tiles
      int tile = static_cast<int>(blockIdx.x);
      while (true) {
        if (!mbar_wait(ringempty0 + 8 * wslot, wph ^ 1u, abort_flag, a.status, kSiteTileEmpty)) break;
        const bool done = tile >= num_tiles;
        ring[wslot] = done ? -1 : tile;
        mbar_arrive(ringfull0 + 8 * wslot);  // release: the ring entry is visible to its readers
        if (++wslot == kTileRing) {
          wslot = 0;
          wph ^= 1u;
        }
        if (done) break;
        const int next = static_cast<int>(gridDim.x) + atomicAdd(a.tile_counter, 1);  // its latency overlaps this tile's loads
        const int mb = tile / a.n_tiles;
        const int nt = tile - mb * a.n_tiles;
        const int brow = a.block_expert[mb] * a.w_rows_per_expert + nt * a.BN;
        bool ok = true;
        for (int kb = 0; kb < a.k_blocks; ++kb) {
          if (!mbar_wait(emptyB0 + 8 * sb, phb ^ 1u, abort_flag, a.status, kSiteEmptyB)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(fullB0 + 8 * sb, b_bytes);
          tma_load_2d(sB + sb * kStageB, &tmB, fullB0 + 8 * sb, kb * 64, brow, pol_b);
          ++fills;
          if (++sb == SB) {
            sb = 0;
            phb ^= 1u;
          }
        }
        if (!ok) break;
        tile = next;
      }
      drain_fills(fullB0, SB, fills);  // no B copy may land after the CTA exits
    }
  } else if (warp == kWarpMma) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kBM, a.BN);
      int rslot = 0, sa = 0, sb = 0;
      uint32_t rph = 0, pha = 0, phb = 0;
      int it = 0;
      bool ok = true;
      while (ok) {
        const int tile = ring_take(ringfull0, ringempty0, ring, rslot, rph, abort_flag, a.status);
        if (tile < 0) break;
        const int acc = it & 1;
        const uint32_t aphase = (it >> 1) & 1;
        if (!mbar_wait(tempty0 + 8 * acc, aphase ^ 1u, abort_flag, a.status, kSiteTmemEmpty)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kAccCols;
        for (int kb = 0; kb < a.k_blocks; ++kb) {
          if (!mbar_wait(fullA0 + 8 * sa, pha, abort_flag, a.status, kSiteFullA) ||
              !mbar_wait(fullB0 + 8 * sb, phb, abort_flag, a.status, kSiteFullB)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = umma_desc_sw128(sA + sa * kStageA);
          const uint64_t bdesc = umma_desc_sw128(sB + sb * kStageB);
#pragma unroll
          for (int k = 0; k < 4; ++k)  // 4 x K=16 bf16 = 128 bytes; +32 bytes = +2 encoded
            umma_bf16(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0);
          umma_commit(emptyA0 + 8 * sa);  // each arrives once these MMAs have read the stage
          umma_commit(emptyB0 + 8 * sb);
          if (++sa == SA) {
            sa = 0;
            pha ^= 1u;
          }
          if (++sb == SB) {
            sb = 0;
            phb ^= 1u;
          }
        }
        if (ok) umma_commit(tfull0 + 8 * acc);
        ++it;
      }
      // all MMAs of this thread complete before TMEM is released
      umma_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0);
    }
  } else {
    // ---------------- epilogue (warps 6..9) ----------------
    // Each warp owns 32 accumulator rows (its TMEM lane quadrant). Per 32 accumulator
    // columns it writes one box of 32 output rows to shared memory and stores it with a
    // TMA tensor store; with two staging buffers the next box is written while the
    // previous store drains.
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const uint32_t staging = sStage + (warp - kWarpEpi) * a.staging_bufs * a.staging_bytes;
    const bool gated = a.activation != 1;  // 0 SwiGLU, 2 gelu_tanh, 3 swigluoai; 1 relu2
    // GEMM1: act bf16 rows of 16 (gated) or 32 (relu2) columns per box, no swizzle;
    // GEMM2: y fp32 rows of 32 columns (128 B), 128-byte swizzle
    const int box_cols = a.mode == 0 ? (gated ? 16 : 32) : 32;
    int nst = 0;  // boxes this warp has staged (selects the staging buffer)
    int it = 0;
    int rslot = 0;
    uint32_t rph = 0;
    while (true) {
      int tile = 0;
      if (lane == 0) tile = ring_take(ringfull0, ringempty0, ring, rslot, rph, abort_flag, a.status);
      tile = __shfl_sync(0xffffffffu, tile, 0);
      if (tile < 0) break;
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
        const uint32_t buf = staging + (nst % a.staging_bufs) * a.staging_bytes;
        if (nst >= a.staging_bufs && lane == 0) {
          // the store that last used `buf` has finished reading it
          if (a.staging_bufs == 2)
            bulk_wait_group_read<1>();
          else
            bulk_wait_group_read<0>();
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
              o[i] = pack_bf16x2(gated_act(g0, u0, a.activation), gated_act(g1, u1, a.activation));
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
      __syncwarp();  // every lane's loads of the accumulator are complete
      if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
      ++it;
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
  if (threadIdx.x == 0) {
    // the last CTA to finish resets the tile counter for the next launch (every CTA's
    // scheduler has taken its last tile before its CTA gets here)
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
    err = cudaFuncSetAttribute(gemm_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemCap);
    if (err != cudaSuccess) return err;
    g_attr_set[dev] = true;
  }
  const int smem = smem_bytes(args.stages_a, args.stages_b, args.staging_bufs, args.staging_bytes);
  if (smem > kSmemCap) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(num_sms), dim3(kThreads), smem);
  return cudaLaunchKernelEx(&cfg, gemm_bf16_kernel, tmA, tmB, tmC, args);
}

Args make_args(int mode, const GemmShape& s, const GemmBuffers& b, const void* a_rows) {
  Args a;
  a.mode = mode;
  a.BN = s.BN;
  a.n_tiles = s.N / s.BN;
  a.k_blocks = (s.K + 63) / 64;
  a.w_rows_per_expert = s.w_rows_per_expert;
  a.k_total = s.k_total;
  a.num_pairs = s.num_pairs;
  a.activation = s.activation;
  // 224 KB of rings and staging either way; GEMM1 boxes are at most 64 B x 32 rows
  a.stages_a = 3;
  a.stages_b = 5;
  a.staging_bufs = mode == 0 ? 2 : 1;
  a.staging_bytes = mode == 0 ? 2048 : 4096;
  a.a_rows = static_cast<const uint8_t*>(a_rows);
  a.a_row_bytes = s.K * 2;
  a.num_blocks = b.num_blocks;
  a.block_expert = b.block_expert;
  a.sorted_pair_ids = b.sorted_pair_ids;
  a.topk_w = b.topk_w;
  a.tile_counter = b.tile_counter;
  a.status = b.status;
  return a;
}

}  // namespace

int pick_bn(int N, long long est_row_tiles, int num_sms) {
  // the widest N tile (multiple of 32 dividing N) that still gives every SM a tile;
  // decode-sized batches have a handful of row tiles and need narrow N tiles to spread
  // the weight stream over all SMs
  int best = 0;
  for (int bn = kMaxBN; bn >= 32; bn -= 32) {
    if (N % bn != 0) continue;
    best = bn;
    if (est_row_tiles * (N / bn) >= num_sms) return bn;
  }
  return best;
}

size_t gemm_bf16_smem_bytes() { return kSmemCap; }

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
