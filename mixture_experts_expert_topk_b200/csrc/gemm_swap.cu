// Steps 3 and 4 of the layer in bf16: the grouped GEMMs with the expert's weight rows as
// the MMA's M operand and its token rows as N.
//
// Each expert's rows in the sorted order are padded to a multiple of 16 only (not to a
// 128-row tile) and cut into row groups of at most 256 rows (align writes the groups). A
// tile is (row group, 128 weight rows): D^T[n, j] = sum_k W[e][n, k] * X[j, k] with
// tcgen05.mma kind::f16, M = 128, N = the group's rows (16..256, a multiple of 16), K = 16,
// fp32 accumulators in TMEM (double-buffered). Putting the tokens on N keeps the padding
// per expert below 16 rows, where 128-row token tiles pad the skewed routing of a large
// batch by about half.
//
// A TMEM lane is one weight row. GEMM1: the gate and up rows of an intermediate index sit
// in adjacent lanes (the [gate0, up0, gate1, up1, ...] interleave prepared at load time,
// "[MoE] SwiGLU fusion into the MoE up-GEMM epilogue", sglang PR 32944, section 3) and are
// paired with one shuffle before the gated activation (silu(gate)*up, gelu_tanh(gate)*up or
// swigluoai; or relu2 without a gate); the kernel writes only the
// bf16 activation. GEMM2: the epilogue multiplies token column j by topk_w of its pair and
// writes fp32 y rows (sorted order) for the fixed-order combine.
//
// Operand layout: both operands are stored in HBM already in the shared-memory layout the
// MMA reads (K-major, 128-byte rows of 64 bf16, the 16-byte pieces of row r permuted by
// r mod 8: the 128-byte swizzle), so every load is one plain bulk copy (cp.async.bulk)
// rather than a tiled tensor copy. Measured on B200, one thread's copies are served one
// after another, at roughly 600 cycles each for bulk copies and 1300 for tiled boxes,
// nearly independent of their size up to 32 KB; so each step is a few large copies,
// issued by two threads.
//   W (prepared weights): tile (expert e, 128-row block m, K chunk c of 64) of 16 KB at
//     ((e * MT + m) * KC + c) * 16 KB; rows and K past the matrix are zero.
//   X (row-group order): the group of n rows starting at sorted row x_row occupies bytes
//     [x_row * KC * 128, (x_row + n) * KC * 128); chunk c of the group is n rows of 128 B
//     at offset c * n * 128 inside it. The token-row permutation writes GEMM1's X in this
//     order, and GEMM1's epilogue writes the activation (GEMM2's X) in it.
// One K step of a tile moves kc chunks of W (kc * 16 KB, one copy) and of X (kc * n * 128
// bytes, one copy), kc = 1..4 chosen from n so that a step holds 48 to 72 KB.
//
// Per-tensor FP8 (e4m3 operands, one fp32 scale per tensor): the same tiles and copies
// with tcgen05.mma kind::f8f6f4 (a 128-byte chunk is 128 elements of K, four K=32 MMAs).
// GEMM1's epilogue dequantises with w13_scale[e] * input_scale before the activation and
// writes e4m3(activation * (1 / activation_scale)); GEMM2's multiplies by activation_scale
// * w2_scale[e] and the routing weight ("FlashInfer TRTLLM-Gen MoE kernel optimisation:
// NemotronH support", section 2: g1_alphas = w13_scale * input_scale, requantised by
// 1.0 / activation_scale). The kernel is compiled once per operand type.
//
// MXFP8 (e4m3 operands, one E8M0 power-of-two scale per 32 values of K on both operands,
// the block size of the MXFP8 weights of the same page, section 2): tcgen05.mma
// kind::mxf8f6f4.block_scale applies the scales inside the MMA. Each K step also carries
// the scale bytes (512 per W chunk, 1024 per X chunk) in the ring; the MMA thread copies
// them to TMEM with tcgen05.cp (row r's scale for K block k in lane r % 32, column r / 32,
// byte k) and MMA k of a chunk selects byte k. Row groups have at most 192 rows so that
// the two accumulators leave 128 TMEM columns for four scale buffers. GEMM1's epilogue
// writes the bf16 activation, which a separate pass quantises for GEMM2.
//
// FP8 E4M3 W8A8 with 128x128 weight blocks and 1x128 activation groups ("Qwen3-Next FP8
// MoE optimisation: shared-expert fusion for H200", sglang PR 26204, section 1): the same
// tiles with kind::f8f6f4, but the scales are arbitrary fp32 (amax / 448), which the tensor
// core's power-of-two block scaling cannot carry. Every 128-element K chunk is therefore
// its own partial product in TMEM (four 128-column buffers, so the MMAs run up to four
// chunks ahead), and the epilogue warps promote it in registers:
// acc[j] += partial[j] * s_w(row block, chunk) * s_x(token j, chunk). A 128-row weight tile
// is exactly one scale block row (gated: its even lanes are gate rows, its odd lanes up
// rows, two block rows of the checkpoint layout), so s_w is one value per lane per chunk;
// s_x varies along N: each K step of X stores, right behind its codes, the fp32 scales of
// its rows (chunk-major), and the X producer copies them into a small ring of their own
// (8 slots of 1 KB) that the epilogue reads as shared-memory broadcasts and frees after
// the step's last chunk; the operand ring is released by the MMAs as in the other kinds.
// Row groups have at most 128 rows (kB128GroupRows) so the accumulator fits the epilogue
// threads' registers.
// GEMM1 writes the bf16 activation, which a separate pass quantises per 1x128 for GEMM2.
//
// NVFP4 (packed E2M1 operands, one E4M3 scale per 16 values of K on both operands, an fp32
// scale per tensor; NVIDIA's NVFP4, named by "FlashInfer gated MoE kernel optimisation for
// Blackwell", section 4): tcgen05.mma kind::mxf4nvf4.block_scale.scale_vec::4X applies the
// block scales inside the MMA. A 128-byte chunk row holds 256 values: four MMAs of K = 64,
// each reading four TMEM scale columns per operand (row r's four block scales in lane
// r % 32, column r / 32, one byte per block). Each K step (at most two chunks) carries the
// W and X scale blocks (2 KB per chunk each) after its codes; the MMA thread copies them to
// TMEM with tcgen05.cp. The epilogue multiplies by the two tensor scales (the expert's
// weight scale and the static input / activation scale). Row groups have at most 128 rows.
//
// One persistent CTA per SM, 7 warps:
//   warp 0      scheduler (tiles from a global atomic counter, published to the other
//               roles through a shared-memory ring) and W copies;
//   warp 6      X copies;
//   warp 1      TMEM allocator and MMA issuer;
//   warps 2-5   epilogue (TMEM lane quadrant = warp % 4).
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kMW = 128;                   // weight rows per tile (MMA M)
constexpr int kChunkBytes = 128;           // one K chunk of a row: 64 bf16
constexpr int kTileW = kMW * kChunkBytes;  // 16 KB: one W chunk
constexpr int kNMax = 256;                 // rows of a row group at most (MMA N)
constexpr int kThreads = 224;
constexpr int kWarpX = 6;
// FP8 block-128 adds twelve epilogue warps (7..18): four per TMEM lane quadrant in all, each
// promoting 32 of a tile's token columns (warps 2..5 columns 0..31, warps 3 + 4 p .. 6 + 4 p
// columns 32 p .. 32 p + 31 for p = 1, 2, 3)
constexpr int kB128EpiWarps = 16;
template <int kKind>
__host__ __device__ constexpr int threads_for() { return kKind == 3 ? kThreads + 32 * (kB128EpiWarps - 4) : kThreads; }
constexpr int kTileRing = 4;
constexpr int kRingReaders = 6;  // MMA, 4 epilogue warps, X producer (FP8 block-128: 16 epilogue warps)
constexpr int kSmemCap = 232448;
constexpr uint32_t kTmemCols = 2 * kNMax;
// MXFP8: scale bytes per chunk in the ring, TMEM columns of the accumulators and of the
// scale buffers (a step of kcs chunks needs 4 kcs columns for W and 4 or 8 per chunk for X)
constexpr int kSfW = 512;
constexpr int kSfX = 1024;
constexpr int kMxAccCols = kMxGroupRows;
constexpr int kSfBufs = 4;
constexpr int kSfBufCols = 32;
constexpr int kSfCol0 = 2 * kMxAccCols;
static_assert(kSfCol0 + kSfBufs * kSfBufCols <= static_cast<int>(kTmemCols), "TMEM columns");
// NVFP4: the same four scale buffers, 64 columns each (two chunks of 16 W and 16 X columns)
constexpr int kNvSfCol0 = 2 * kNvGroupRows;
constexpr int kNvSfBufCols = 64;
static_assert(kNvSfCol0 + kSfBufs * kNvSfBufCols <= static_cast<int>(kTmemCols), "TMEM columns");
// FP8 block-128: partial-product buffers in TMEM (one per K chunk in flight)
constexpr int kPartBufs = 4;
constexpr int kPartCols = kB128GroupRows;
static_assert(kPartBufs * kPartCols <= static_cast<int>(kTmemCols), "TMEM columns");

// Operand ring: a K step takes kc * (16 KB + n * 128) contiguous bytes (W chunks, then X
// chunks); a step that would cross the end of the ring starts again at its beginning.
// Offsets stay multiples of 1024 bytes, the period of the 128-byte swizzle.
constexpr int kRingBytes = 225 * 1024;
// FP8 block-128: a shorter operand ring, then kSxSlots slots of the X scale ring
constexpr int kSxSlots = 8;
constexpr int kSxSlotBytes = 1024;  // a step's scales: kcs * n * 4 <= 4 * 32 * 4 = 3 * 64 * 4 < 2 * 128 * 4 + 1
constexpr int kRingBytesB128 = kRingBytes - kSxSlots * kSxSlotBytes - 1024;
static_assert(4 * 32 * 4 <= kSxSlotBytes && 3 * 64 * 4 <= kSxSlotBytes && 2 * kB128GroupRows * 4 <= kSxSlotBytes,
              "a step's X scales fit a slot");
template <int kKind>
__host__ __device__ constexpr int ring_bytes() { return kKind == 3 ? kRingBytesB128 : kRingBytes; }
constexpr int kSlots = 16;  // barrier pairs: at most this many K steps in flight
constexpr int kBarOff = kRingBytes;
constexpr int kBarBytes = 1024;  // barriers, step ends, tile ring, TMEM address, abort flag
static_assert((3 * kSlots + 4 + 2 * kTileRing + 1 + 2 * 4 + 8) * 8 + 2 * kSlots * 8 + 16 * kTileRing + 8 <= kBarBytes,
              "barrier region");
constexpr int kSmemBytes = kBarOff + kBarBytes + 1024;
static_assert(kSmemBytes <= kSmemCap, "shared memory");

enum : int {
  kSiteEmpty = 1, kSiteFull = 2, kSiteTmemEmpty = 3, kSiteTmemFull = 4, kSiteTileFull = 5, kSiteTileEmpty = 6,
  kSiteEmptyX = 7, kSiteSfFree = 8, kSiteFullX = 9, kSitePartEmpty = 10, kSitePartFull = 11, kSiteSxFree = 12
};

struct Args {
  int mode;                // 0 = GEMM1 (activation), 1 = GEMM2 (routing weight)
  int m_tiles;             // MT: 128-row weight blocks per expert
  int k_chunks;            // KC: K chunks of 64 (weights and X)
  int k_total, num_pairs, activation;
  const uint8_t* w;        // tiled weights
  const uint8_t* x;        // X in row-group order
  void* out;               // GEMM1: activation in row-group order; GEMM2: y fp32 [rows, H]
  int out_chunks;          // GEMM1: K chunks of the activation (GEMM2's KC)
  int out_cols;            // GEMM2: H
  const int* num_groups;
  const int2* group_info;  // {first sorted row, expert | rows << 16}
  const int* sorted_pair_ids;
  const float* topk_w;
  int* tile_counter;       // [2]: next tile, CTAs finished; both 0 between launches
  int* status;
  const float* w_scale;    // FP8: per-expert weight scales [E]
  float in_scale;          // FP8 GEMM1: input scale; GEMM2: activation scale (the X scale)
  float act_inv;           // FP8 GEMM1: 1 / activation scale (requantisation of the output)
  const uint8_t* w_sf;     // MXFP8: tiled weight scales, 512 bytes per (expert, 128-row block, K chunk)
  const uint8_t* x_sf;     // MXFP8: X scales, 1024 bytes per (16 rows of the group's first row, K chunk)
  // FP8 block-128: w_scale is fp32 [E, ws_rows, k_chunks] (checkpoint block layout); gated
  // GEMM1 tiles take the gate block row mt / 2 and the up block row up_block + mt / 2
  int ws_rows;             // 128-row scale blocks per expert
  int up_block;            // gated GEMM1: I / 128; 0 otherwise
  int8_t* y_exp;           // GEMM2: the power-of-two exponent of each 32 columns of y
  int w_early;             // 1: the previous kernel does not write the row groups (see below)
};

// Ring bytes of one K step of kcs chunks for a group of n rows. MXFP8 steps add the scale
// blocks of W and X and round up to the 1024-byte period of the swizzle.
template <int kKind>
__device__ __forceinline__ uint32_t step_bytes(int kcs, int n) {
  const uint32_t b = static_cast<uint32_t>(kcs) * (kTileW + n * kChunkBytes);
  if (kKind == 2) return (b + static_cast<uint32_t>(kcs) * (kSfW + kSfX) + 1023u) & ~1023u;
  if (kKind == 4) return b + static_cast<uint32_t>(kcs) * 2u * kNvChunkScaleBytes;
  return b;
}
// K chunks per step: NVFP4 steps take at most two (their scale buffers hold two chunks);
// per-tensor FP8 and MXFP8 groups of more than 128 rows take two (one 16 KB weight copy per
// step measured slower for these kinds, while bf16 keeps one: its GEMMs ran slower with
// two, from the fewer steps in flight)
template <int kKind>
__device__ __forceinline__ int step_chunks(int n) {
  if (kKind == 4) return min(chunks_per_step(n), 2);
  if ((kKind == 1 || kKind == 2) && n > 128) return 2;
  return chunks_per_step(n);
}
static_assert(4 * (kTileW + 32 * kChunkBytes + kSfW + kSfX) <= kRingBytes / 2 &&
                  2 * (kTileW + kMxGroupRows * kChunkBytes + kSfW + kSfX) + 1023 <= kRingBytes / 2,
              "at least two MXFP8 steps fit the ring");
static_assert(2 * (kTileW + kNMax * kChunkBytes) <= kRingBytes / 2, "at least two per-tensor FP8 steps fit the ring");
static_assert(4 * (kTileW + 32 * kChunkBytes) <= kRingBytes / 2 && 2 * (kTileW + 128 * kChunkBytes) <= kRingBytes / 2 &&
                  kTileW + kNMax * kChunkBytes <= kRingBytes / 2,
              "at least two steps fit the ring");
static_assert(4 * (kTileW + 32 * kChunkBytes) <= kRingBytesB128 / 2 &&
                  2 * (kTileW + kB128GroupRows * kChunkBytes) <= kRingBytesB128 / 2,
              "at least two FP8 block-128 steps fit the ring");

// Byte offset in the ring of the next step of `bytes`. pos: offset of the next free byte;
// head: running count of the bytes used, skipped ring tails included.
template <int kBytes>
__device__ __forceinline__ uint32_t ring_alloc(uint32_t& pos, uint64_t& head, uint32_t bytes) {
  if (pos + bytes > static_cast<uint32_t>(kBytes)) {
    head += kBytes - pos;
    pos = 0;
  }
  const uint32_t off = pos;
  pos += bytes;
  head += bytes;
  return off;
}

// Waits, oldest step first, until the step just allocated (its end is `head`, its index
// ks) fits the ring and has a free slot. Each producer keeps its own copy of this state;
// both allocate the same sequence of steps.
template <int kBytes>
__device__ __forceinline__ bool ring_reserve(uint64_t head, uint64_t& freed, uint32_t ks, uint32_t& oldest,
                                             uint64_t* step_end, uint32_t empty0, volatile int* abort, int* status,
                                             int site) {
  while (head - freed > static_cast<uint64_t>(kBytes) || ks - oldest >= static_cast<uint32_t>(kSlots)) {
    if (!mbar_wait(empty0 + 8 * (oldest % kSlots), (oldest / kSlots) & 1u, abort, status, site)) return false;
    freed = step_end[oldest % kSlots];
    ++oldest;
  }
  step_end[ks % kSlots] = head;
  return true;
}

// Reader side of the tile ring: {x_row, n (0 = no more tiles), expert, mt}.
__device__ __forceinline__ bool ring_read(uint32_t rfull0, uint32_t rempty0, volatile int* ring, int& slot,
                                          uint32_t& ph, volatile int* abort, int* status, int4& t) {
  const bool ok = mbar_wait(rfull0 + 8 * slot, ph, abort, status, kSiteTileFull);
  if (ok) t = make_int4(ring[4 * slot + 0], ring[4 * slot + 1], ring[4 * slot + 2], ring[4 * slot + 3]);
  mbar_arrive(rempty0 + 8 * slot);
  if (++slot == kTileRing) {
    slot = 0;
    ph ^= 1u;
  }
  return ok;
}

// One contiguous global -> shared copy completing on `bar` (16-byte aligned addresses,
// size a multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar,
                                          uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}

// kKind: 0 bf16, 1 per-tensor e4m3, 2 MXFP8, 3 FP8 block-128, 4 NVFP4.
template <int kKind>
__global__ void __launch_bounds__(threads_for<kKind>(), 1) gemm_swap_kernel(const Args a) {
  constexpr bool kFp8 = kKind == 1;  // scales applied in the epilogue
  constexpr bool kMx = kKind == 2;   // scales applied by the MMA
  constexpr bool kB128 = kKind == 3; // a partial per K chunk, promoted in the epilogue
  constexpr bool kE4m3 = kFp8 || kB128;
  constexpr bool kNv = kKind == 4;   // block scales applied by the MMA, tensor scales in the epilogue
  constexpr int kAccCols = kMx ? kMxAccCols : (kNv ? kNvGroupRows : kNMax);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t s0 = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * kSlots;
  const uint32_t tfull0 = empty0 + 8 * kSlots;
  const uint32_t tempty0 = tfull0 + 16;
  const uint32_t rfull0 = tempty0 + 16;
  const uint32_t rempty0 = rfull0 + 8 * kTileRing;
  const uint32_t drain_bar = rempty0 + 8 * kTileRing;
  const uint32_t fullx0 = drain_bar + 8;                                      // [kSlots]
  const uint32_t pfull0 = fullx0 + 8 * kSlots;                                // [kPartBufs]
  const uint32_t pempty0 = pfull0 + 8 * kPartBufs;                            // [kPartBufs]
  const uint32_t sxfree0 = pempty0 + 8 * kPartBufs;                           // [kSxSlots]
  const uint32_t sx0 = s0 + kRingBytesB128;                                   // FP8 block-128 X scale ring
  uint64_t* step_end_w = bars + 3 * kSlots + 4 + 2 * kTileRing + 1 + 2 * kPartBufs + kSxSlots;  // [kSlots]
  uint64_t* step_end_x = step_end_w + kSlots;                                 // [kSlots]
  volatile int* ring = reinterpret_cast<volatile int*>(step_end_x + kSlots);  // [kTileRing][4]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(const_cast<int*>(ring) + 4 * kTileRing);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(full0 + 8 * s, 1);   // the W copies of a step
      mbar_init(fullx0 + 8 * s, 1);  // the X copies of a step
      mbar_init(empty0 + 8 * s, 1);  // released by the MMAs' commit
    }
    for (int b = 0; b < kPartBufs; ++b) {
      mbar_init(pfull0 + 8 * b, 1);
      mbar_init(pempty0 + 8 * b, kB128EpiWarps);  // one arrival per epilogue warp
    }
    for (int b = 0; b < kSxSlots; ++b) mbar_init(sxfree0 + 8 * b, kB128EpiWarps);  // every epilogue warp
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, 4);  // one arrival per epilogue warp
    }
    for (int s = 0; s < kTileRing; ++s) {
      mbar_init(rfull0 + 8 * s, 1);
      mbar_init(rempty0 + 8 * s, kB128 ? kRingReaders + kB128EpiWarps - 4 : kRingReaders);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // Everything above overlaps the previous kernel. With w_early the scheduler + W producer
  // (warp 0) starts right away: it reads only the weights, align's row groups and the work
  // counter, which the launcher vouches were complete before the previous kernel (itself
  // behind its own wait) could launch this one, so the first weight copies overlap that
  // kernel's tail. Every other role waits for the previous kernel's output (X) first.
  if (warp != 0 || !a.w_early) {
    griddep_wait();
    griddep_launch_dependents();
  }

  // bytes of X per row: a 128-byte chunk row per K chunk (FP8 block-128: and its fp32 scale)
  const size_t x_row_bytes = static_cast<size_t>(a.k_chunks) * (kB128 ? kB128RowBytesPerChunk : kChunkBytes);

  if (warp == 0) {
    // ---------------- scheduler + W producer ----------------
    if (lane == 0) {
      const int num_tiles = *a.num_groups * a.m_tiles;
      const uint64_t pol = policy_evict_first();  // each weight tile is streamed by one group
      int wslot = 0;
      uint32_t wph = 0, pos = 0, ks = 0, oldest = 0;
      uint64_t head = 0, freed = 0;
      // the first tile is the CTA index; later ones come from the counter, after the grid's first tiles
      int tile = static_cast<int>(blockIdx.x);
      bool ok = true;
      while (ok) {
        if (!mbar_wait(rempty0 + 8 * wslot, wph ^ 1u, abort_flag, a.status, kSiteTileEmpty)) break;
        int x_row = 0, n = 0, e = 0, mt = 0, n_real = 0;
        if (tile < num_tiles) {
          const int g = tile / a.m_tiles;
          mt = tile - g * a.m_tiles;
          const int2 gi = a.group_info[g];
          x_row = gi.x;
          n = group_word_rows(gi.y);
          e = group_word_expert(gi.y);
          n_real = n - group_word_pad(gi.y);  // the group's padding rows are its last
        }
        ring[4 * wslot + 0] = x_row;
        ring[4 * wslot + 1] = n | (n_real << 16);  // the group's real rows beside n; n == 0: stop
        ring[4 * wslot + 2] = e;
        ring[4 * wslot + 3] = mt;
        mbar_arrive(rfull0 + 8 * wslot);  // release: the entry is visible to its readers
        if (++wslot == kTileRing) {
          wslot = 0;
          wph ^= 1u;
        }
        if (n == 0) break;
        const int next = static_cast<int>(gridDim.x) + atomicAdd(a.tile_counter, 1);  // its latency overlaps the loads
        const int kc = step_chunks<kKind>(n);
        const uint8_t* wsrc = a.w + (static_cast<size_t>(e) * a.m_tiles + mt) * a.k_chunks * kTileW;
        for (int c0 = 0; c0 < a.k_chunks; c0 += kc, ++ks) {
          const int kcs = min(kc, a.k_chunks - c0);
          const uint32_t off = ring_alloc<ring_bytes<kKind>()>(pos, head, step_bytes<kKind>(kcs, n));
          if (!ring_reserve<ring_bytes<kKind>()>(head, freed, ks, oldest, step_end_w, empty0, abort_flag, a.status, kSiteEmpty)) {
            ok = false;
            break;
          }
          const uint32_t full = full0 + 8 * (ks % kSlots);
          const uint32_t bytes = static_cast<uint32_t>(kcs) * kTileW;
          constexpr uint32_t kWsf = kMx ? kSfW : (kNv ? kNvChunkScaleBytes : 0u);  // W scale bytes per chunk
          const uint32_t sf_bytes = static_cast<uint32_t>(kcs) * kWsf;
          mbar_arrive_expect_tx(full, bytes + sf_bytes);
          bulk_load(s0 + off, wsrc + static_cast<size_t>(c0) * kTileW, bytes, full, pol);
          if constexpr (kMx || kNv)
            bulk_load(s0 + off + static_cast<uint32_t>(kcs) * (kTileW + n * kChunkBytes),
                      a.w_sf + ((static_cast<size_t>(e) * a.m_tiles + mt) * a.k_chunks + c0) * kWsf, sf_bytes, full,
                      pol);
        }
        tile = next;
      }
      drain_fills(full0, kSlots, ks);  // no W copy may land after the CTA exits
    }
  } else if (warp == kWarpX) {
    // ---------------- X producer ----------------
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();  // a group's rows are read by m_tiles tiles
      int rslot = 0;
      uint32_t rph = 0, pos = 0, ks = 0, oldest = 0;
      uint64_t head = 0, freed = 0;
      bool ok = true;
      while (ok) {
        int4 t;
        if (!ring_read(rfull0, rempty0, ring, rslot, rph, abort_flag, a.status, t) || t.y == 0) break;
        const int x_row = t.x, n = t.y & 0xffff;
        const int kc = step_chunks<kKind>(n);
        const uint8_t* xsrc = a.x + static_cast<size_t>(x_row) * x_row_bytes;
        for (int c0 = 0; c0 < a.k_chunks; c0 += kc, ++ks) {
          const int kcs = min(kc, a.k_chunks - c0);
          const uint32_t off = ring_alloc<ring_bytes<kKind>()>(pos, head, step_bytes<kKind>(kcs, n));
          if (!ring_reserve<ring_bytes<kKind>()>(head, freed, ks, oldest, step_end_x, empty0, abort_flag, a.status, kSiteEmptyX)) {
            ok = false;
            break;
          }
          const uint32_t full = fullx0 + 8 * (ks % kSlots);
          const uint32_t bytes = static_cast<uint32_t>(kcs * n) * kChunkBytes;
          // MXFP8: the scale blocks; FP8 block-128: the rows' scales, stored right behind
          // the step's codes, into a slot of the X scale ring once the epilogue freed it
          const uint32_t sf_bytes = kMx ? static_cast<uint32_t>(kcs) * kSfX
                                        : (kNv ? static_cast<uint32_t>(kcs) * kNvChunkScaleBytes
                                               : (kB128 ? static_cast<uint32_t>(kcs * n) * 4u : 0u));
          if (kB128 && !mbar_wait(sxfree0 + 8 * (ks % kSxSlots), ((ks / kSxSlots) & 1u) ^ 1u, abort_flag, a.status,
                                  kSiteSxFree)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full, bytes + sf_bytes);
          const uint8_t* step_src = xsrc + static_cast<size_t>(c0) * n * (kB128 ? kB128RowBytesPerChunk : kChunkBytes);
          bulk_load(s0 + off + kcs * kTileW, step_src, bytes, full, pol);
          if constexpr (kB128) bulk_load(sx0 + (ks % kSxSlots) * kSxSlotBytes, step_src + bytes, sf_bytes, full, pol);
          if constexpr (kMx)
            bulk_load(s0 + off + static_cast<uint32_t>(kcs) * (kTileW + n * kChunkBytes + kSfW),
                      a.x_sf + (static_cast<size_t>(x_row >> 4) * a.k_chunks + c0) * kSfX, sf_bytes, full, pol);
          if constexpr (kNv)
            bulk_load(s0 + off + static_cast<uint32_t>(kcs) * (kTileW + n * kChunkBytes + kNvChunkScaleBytes),
                      a.x_sf + (static_cast<size_t>(x_row >> 4) * a.k_chunks + c0) * kNvChunkScaleBytes, sf_bytes,
                      full, pol);
        }
      }
      drain_fills(fullx0, kSlots, ks);  // no X copy may land after the CTA exits
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int rslot = 0, it = 0;
      uint32_t rph = 0, ks = 0, pos = 0, pc = 0;  // pc: FP8 block-128 partials issued
      uint64_t head = 0;  // the producers' ring allocation, replayed
      while (true) {
        int4 t;
        if (!ring_read(rfull0, rempty0, ring, rslot, rph, abort_flag, a.status, t) || t.y == 0) break;
        const int n = t.y & 0xffff;
        const int kc = step_chunks<kKind>(n);
        const int acc = it & 1;
        if (!kB128 && !mbar_wait(tempty0 + 8 * acc, ((it >> 1) & 1) ^ 1u, abort_flag, a.status, kSiteTmemEmpty)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kAccCols;
        const uint32_t idesc =
            kMx ? idesc_mx(kMW, n) : (kNv ? idesc_nvf4(kMW, n) : (kE4m3 ? idesc_e4m3(kMW, n) : idesc_bf16(kMW, n)));
        bool ok = true;
        for (int c0 = 0; c0 < a.k_chunks; c0 += kc, ++ks) {
          const int kcs = min(kc, a.k_chunks - c0);
          const uint32_t base = s0 + ring_alloc<ring_bytes<kKind>()>(pos, head, step_bytes<kKind>(kcs, n));
          if (!mbar_wait(full0 + 8 * (ks % kSlots), (ks / kSlots) & 1u, abort_flag, a.status, kSiteFull) ||
              !mbar_wait(fullx0 + 8 * (ks % kSlots), (ks / kSlots) & 1u, abort_flag, a.status, kSiteFullX)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // descriptor low words: W chunk c at base + c * 16 KB, X chunk c at base + kcs * 16 KB
          // + c * n * 128 (the encoded address counts 16-byte units)
          const uint32_t a_lo = umma_desc_lo(base);
          const uint32_t b_lo = a_lo + static_cast<uint32_t>(kcs) * (kTileW >> 4);
          const uint32_t b_step = static_cast<uint32_t>(n) * (kChunkBytes >> 4);
          if constexpr (kMx) {
            // the scale buffer of this step was last read by the MMAs of step ks - kSfBufs
            if (ks >= static_cast<uint32_t>(kSfBufs) &&
                !mbar_wait(empty0 + 8 * ((ks - kSfBufs) % kSlots), ((ks - kSfBufs) / kSlots) & 1u, abort_flag,
                           a.status, kSiteSfFree)) {
              ok = false;
              break;
            }
            const uint32_t sf_s = base + static_cast<uint32_t>(kcs) * (kTileW + n * kChunkBytes);
            const uint32_t sf_t = tmem_base + kSfCol0 + (ks % kSfBufs) * kSfBufCols;
            const int nb = n > 128 ? 2 : 1;  // 128-row scale blocks of X
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              if (c < kcs) {
                tmem_cp_sf(sf_t + 4 * c, sf_s + c * kSfW);
                tmem_cp_sf(sf_t + 4 * kcs + 4 * nb * c, sf_s + kcs * kSfW + c * kSfX);
                if (nb == 2) tmem_cp_sf(sf_t + 4 * kcs + 4 * nb * c + 4, sf_s + kcs * kSfW + c * kSfX + 512);
              }
            }
#pragma unroll
            for (int c = 0; c < 4; ++c)
              if (c < kcs)
                umma_mx_chunk(d_tmem, a_lo + c * (kTileW >> 4), b_lo + c * b_step, idesc, sf_t + 4 * c,
                              sf_t + 4 * kcs + 4 * nb * c, (c0 != 0 || c != 0) ? 1u : 0u);
          } else if (kNv) {
            // the scale buffer of this step was last read by the MMAs of step ks - kSfBufs
            if (ks >= static_cast<uint32_t>(kSfBufs) &&
                !mbar_wait(empty0 + 8 * ((ks - kSfBufs) % kSlots), ((ks - kSfBufs) / kSlots) & 1u, abort_flag,
                           a.status, kSiteSfFree)) {
              ok = false;
              break;
            }
            const uint32_t sf_s = base + static_cast<uint32_t>(kcs) * (kTileW + n * kChunkBytes);
            const uint32_t sf_t = tmem_base + kNvSfCol0 + (ks % kSfBufs) * kNvSfBufCols;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              if (c < kcs) {
#pragma unroll
                for (int mm = 0; mm < 4; ++mm) {
                  tmem_cp_sf(sf_t + 16 * c + 4 * mm, sf_s + c * kNvChunkScaleBytes + mm * 512);
                  tmem_cp_sf(sf_t + 32 + 16 * c + 4 * mm,
                             sf_s + (kcs + c) * kNvChunkScaleBytes + mm * 512);
                }
              }
            }
#pragma unroll
            for (int c = 0; c < 2; ++c)
              if (c < kcs)
                umma_nvf4_chunk(d_tmem, a_lo + c * (kTileW >> 4), b_lo + c * b_step, idesc, sf_t + 16 * c,
                                sf_t + 32 + 16 * c, (c0 != 0 || c != 0) ? 1u : 0u);
          } else if (kB128) {
            // one fresh partial per K chunk, into the next free buffer
            for (int c = 0; c < kcs; ++c, ++pc) {
              const uint32_t pb = pc % kPartBufs;
              if (!mbar_wait(pempty0 + 8 * pb, ((pc / kPartBufs) & 1u) ^ 1u, abort_flag, a.status, kSitePartEmpty)) {
                ok = false;
                break;
              }
              tc_fence_after();
              umma_e4m3_chunk(tmem_base + pb * kPartCols, a_lo + c * (kTileW >> 4), b_lo + c * b_step, idesc, 0u);
              umma_commit(pfull0 + 8 * pb);
            }
            if (!ok) break;
          } else if (kFp8) {
            umma_e4m3_chunk(d_tmem, a_lo, b_lo, idesc, c0 != 0);
#pragma unroll
            for (int c = 1; c < 4; ++c)
              if (c < kcs) umma_e4m3_chunk(d_tmem, a_lo + c * (kTileW >> 4), b_lo + c * b_step, idesc, 1u);
          } else {
            umma_bf16_chunk(d_tmem, a_lo, b_lo, idesc, c0 != 0);
#pragma unroll
            for (int c = 1; c < 4; ++c)
              if (c < kcs) umma_bf16_chunk(d_tmem, a_lo + c * (kTileW >> 4), b_lo + c * b_step, idesc, 1u);
          }
          umma_commit(empty0 + 8 * (ks % kSlots));  // arrives once these MMAs have read the step
        }
        if (!ok) break;
        if (!kB128) umma_commit(tfull0 + 8 * acc);
        ++it;
      }
      // all MMAs of this thread complete before TMEM is released
      umma_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0);
    }
  } else {
    // ---------------- epilogue (warps 2..5; FP8 block-128 also 7..10): lane = weight row ----
    // 32 token columns at a time. For a given token the warp's 32 lanes hold neighbouring
    // output columns, so each store writes one contiguous piece of an output row (GEMM2:
    // 64 B of fp16; GEMM1: 64 or 32 B of a 128-byte activation chunk row).
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    // FP8 block-128: this warp's token columns [32 part, 32 part + 32)
    const int part = kB128 && warp > kWarpX ? 1 + (warp - kWarpX - 1) / 4 : 0;
    const bool gated = a.activation != 1;  // 0 SwiGLU, 2 gelu_tanh, 3 swigluoai; 1 relu2
    const bool odd = (lane & 1) != 0;
    int rslot = 0, it = 0;
    uint32_t rph = 0;
    uint32_t ks = 0, pc = 0;  // FP8 block-128: K steps and partials consumed
    while (true) {
      int4 t = make_int4(0, 0, 0, 0);
      int ok = 0;
      if (lane == 0) ok = ring_read(rfull0, rempty0, ring, rslot, rph, abort_flag, a.status, t);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      const int ny = __shfl_sync(0xffffffffu, t.y, 0);
      const int n = ny & 0xffff, n_real = ny >> 16;  // GEMM1: the group's rows that are not padding
      if (!ok || n == 0) break;
      const int x_row = __shfl_sync(0xffffffffu, t.x, 0);
      const int expert = __shfl_sync(0xffffffffu, t.z, 0);
      const int mt = __shfl_sync(0xffffffffu, t.w, 0);
      // FP8 per-tensor, NVFP4: the accumulator's dequantisation scale (the weight's and the
      // X operand's tensor scales; GEMM1: before the activation)
      const float dq = (kFp8 || kNv) ? __ldg(a.w_scale + expert) * a.in_scale : 1.0f;
      // GEMM1: this lane's activation feature f lies in K chunk f / 64 (bf16) or f / 128
      // (e4m3) of the activation; byte b of a 128-byte chunk row sits in 16-byte piece
      // (b / 16) ^ (row % 8)
      const int f = gated ? mt * (kMW / 2) + q * 16 + (lane >> 1) : mt * kMW + q * 32 + lane;
      const int fc = kFp8 ? f >> 7 : f >> 6;
      const int fo = kFp8 ? f & 127 : (f & 63) * 2;  // byte offset in the chunk row
      uint8_t* act_grp = static_cast<uint8_t*>(a.out) + static_cast<size_t>(x_row) * a.out_chunks * kChunkBytes +
                         static_cast<size_t>(fc) * n * kChunkBytes;

      // Output of token columns c0 .. c0 + 31 (c0 .. c0 + 15 unless `full`) of this lane's
      // weight row, from v[j] = accumulator of column c0 + j.
      auto store_block = [&](const uint32_t(&v)[32], int c0, bool full) {
        if (a.mode != 0) {
          // GEMM2: y = acc * dq (the routing weight is applied by the combine), stored as fp16
          // scaled by a power of two shared by this block of 32 tokens x 32 columns (the
          // warp's lanes): 2^-s brings the block's largest magnitude into [2^14, 2^15), so no
          // value overflows fp16, and every value within 2^-28 of that maximum keeps 11
          // significant bits. s (at least -100) is stored for each of the block's token rows.
          float m = 0.f;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < 16 || full) m = fmaxf(m, fabsf(__uint_as_float(v[j])));
          const uint32_t amax = __reduce_max_sync(0xffffffffu, __float_as_uint(m * dq));
          const int s = amax == 0u ? 0 : max(static_cast<int>(amax >> 23) - 127 - 14, -100);
          const float f = dq * __int_as_float((127 - s) << 23);
          const int col = mt * kMW + q * 32 + lane;
          __half* y = static_cast<__half*>(a.out) + static_cast<size_t>(x_row + c0) * a.out_cols + col;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (j == 16 && !full) break;
            y[static_cast<size_t>(j) * a.out_cols] = __float2half_rn(__uint_as_float(v[j]) * f);
          }
          if (lane < 16 || full)
            a.y_exp[static_cast<size_t>(x_row + c0 + lane) * (a.out_cols >> 5) + (col >> 5)] = static_cast<int8_t>(s);
        } else if (!gated) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (j == 16 && !full) break;
            const int row = c0 + j;
            const float z = fmaxf(__uint_as_float(v[j]) * dq, 0.f);
            uint8_t* dst = act_grp + row * kChunkBytes + ((((fo >> 4) ^ row) & 7) << 4) + (fo & 15);
            if (kFp8)
              *dst = __nv_cvt_float_to_fp8(z * z * a.act_inv, __NV_SATFINITE, __NV_E4M3);
            else
              *reinterpret_cast<__nv_bfloat16*>(dst) = __float2bfloat16_rn(z * z);
          }
        } else {
          // lane pair (2m, 2m+1) = (gate, up) of feature m. The even lane finishes tokens
          // 0..15 of the batch, the odd lane tokens 16..31: each passes the other the half
          // it needs, so every lane evaluates the activation on 16 tokens.
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float mine_lo = __uint_as_float(v[j]) * dq;       // even: gate_j; odd: up_j
            const float mine_hi = __uint_as_float(v[16 + j]) * dq;  // even: gate_{16+j}; odd: up_{16+j}
            const float other = __shfl_xor_sync(0xffffffffu, odd ? mine_lo : mine_hi, 1);
            const float g = odd ? other : mine_lo;
            const float u = odd ? mine_hi : other;
            const int row = c0 + (odd ? 16 + j : j);
            if (!odd || full) {
              const float h = gated_act(g, u, a.activation);
              uint8_t* dst = act_grp + row * kChunkBytes + ((((fo >> 4) ^ row) & 7) << 4) + (fo & 15);
              if (kFp8)
                *dst = __nv_cvt_float_to_fp8(h * a.act_inv, __NV_SATFINITE, __NV_E4M3);
              else
                *reinterpret_cast<__nv_bfloat16*>(dst) = __float2bfloat16_rn(h);
            }
          }
        }
        // GEMM1: a group's padding rows (a suffix, from n_real on) hold whatever X held there
        // (the permute does not write them); zeros over them, so GEMM2 sees zero rows. Only
        // the block that holds them takes this branch (block-uniform), each thread rewriting
        // the rows it stored above, in program order.
        const int c1 = c0 + (full ? 32 : 16);
        if (a.mode == 0 && c1 > n_real) {
          const int r0 = gated ? c0 + (odd ? 16 : 0) : c0;
          const int r1 = gated ? (odd ? (full ? c1 : r0) : min(c1, c0 + 16)) : c1;
          for (int row = max(r0, n_real); row < r1; ++row) {
            uint8_t* dst = act_grp + row * kChunkBytes + ((((fo >> 4) ^ row) & 7) << 4) + (fo & 15);
            if (kFp8)
              *dst = 0;
            else
              *reinterpret_cast<__nv_bfloat16*>(dst) = __float2bfloat16_rn(0.f);
          }
        }
      };

      if constexpr (kB128) {
        // promote each K chunk's partial: acc[j] += partial[j] * s_w * s_x[j]
        const int kc = step_chunks<kKind>(n);
        // the tile's weight scales, lane k holding K chunk k (k_chunks <= 32): gated GEMM1's
        // even lanes are gate rows (block row mt / 2), its odd lanes up rows
        const float* sw_e = a.w_scale + static_cast<size_t>(expert) * a.ws_rows * a.k_chunks;
        const int rb_even = a.up_block > 0 ? mt >> 1 : mt;
        const int rb_odd = a.up_block > 0 ? a.up_block + (mt >> 1) : mt;
        const float swl_even = lane < a.k_chunks ? __ldg(sw_e + static_cast<size_t>(rb_even) * a.k_chunks + lane) : 0.f;
        const float swl_odd = lane < a.k_chunks ? __ldg(sw_e + static_cast<size_t>(rb_odd) * a.k_chunks + lane) : 0.f;
        // this warp's token columns [32 part, 32 part + 32)
        const int nb = n - 32 * part;  // columns left from this warp's first
        const bool has = nb > 0, full = nb >= 32;
        float2 acc[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] = make_float2(0.f, 0.f);
        bool good = true;
        for (int c0 = 0; c0 < a.k_chunks && good; c0 += kc, ++ks) {
          const int kcs = min(kc, a.k_chunks - c0);
          // the X scales of this step, [chunk][row] fp32, in its slot of the X scale ring (the
          // full barrier the partials' MMAs waited on also covered this copy)
          const uint32_t sf = (ks % kSxSlots) * kSxSlotBytes + kRingBytesB128;
          for (int c = 0; c < kcs; ++c, ++pc) {
            const uint32_t pb = pc % kPartBufs;
            const bool got = mbar_wait(pfull0 + 8 * pb, (pc / kPartBufs) & 1u, abort_flag, a.status, kSitePartFull);
            if (!__all_sync(0xffffffffu, got)) {  // leave warp-uniformly (tcgen05.ld is .aligned)
              good = false;
              break;
            }
            tc_fence_after();
            // lane k holds chunk k's weight scales (even and odd rows)
            const float sw_e_k = __shfl_sync(0xffffffffu, swl_even, c0 + c);
            const float sw_o_k = __shfl_sync(0xffffffffu, swl_odd, c0 + c);
            const float sw = odd ? sw_o_k : sw_e_k;
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + pb * kPartCols + 32 * part;
            // the partial in two halves of 16 columns (fewer live registers than one load of 32)
            const float4* sx4 = reinterpret_cast<const float4*>(smem + sf + static_cast<uint32_t>(c * n + 32 * part) * 4u);
            const float2 sw2 = make_float2(sw, sw);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              if (16 * h < nb) {  // warp-uniform
                uint32_t v[16];
                tmem_ld16(taddr + 16 * h, v);
                tmem_wait_ld();
#pragma unroll
                for (int j4 = 0; j4 < 4; ++j4) {
                  // columns 16 h + 4 j4 .. + 3 of this warp's 32: acc pairs 8 h + 2 j4, + 1; the
                  // same scales for every lane (shared-memory broadcasts)
                  const int j = 4 * j4, a2 = 8 * h + 2 * j4;
                  const float4 sx = sx4[4 * h + j4];
                  acc[a2] = __ffma2_rn(make_float2(__uint_as_float(v[j]), __uint_as_float(v[j + 1])),
                                       __fmul2_rn(make_float2(sx.x, sx.y), sw2), acc[a2]);
                  acc[a2 + 1] = __ffma2_rn(make_float2(__uint_as_float(v[j + 2]), __uint_as_float(v[j + 3])),
                                           __fmul2_rn(make_float2(sx.z, sx.w), sw2), acc[a2 + 1]);
                }
              }
            }
            tc_fence_before();
            __syncwarp();  // every lane's loads of the partial are complete
            if (lane == 0) mbar_arrive(pempty0 + 8 * pb);  // the partial is in registers now
          }
          if (!good) break;
          __syncwarp();  // every lane has read the step's scales
          if (lane == 0) mbar_arrive(sxfree0 + 8 * (ks % kSxSlots));
        }
        if (!__all_sync(0xffffffffu, good)) break;
        if (has) store_block(*reinterpret_cast<const uint32_t(*)[32]>(&acc[0]), 32 * part, full);
      } else {
        const int acc = it & 1;
        const bool got = mbar_wait(tfull0 + 8 * acc, (it >> 1) & 1, abort_flag, a.status, kSiteTmemFull);
        if (!__all_sync(0xffffffffu, got)) break;  // leave warp-uniformly (tcgen05.ld is .aligned)
        tc_fence_after();
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * kAccCols;
        for (int c0 = 0; c0 < n; c0 += 32) {
          const bool full = n - c0 >= 32;  // else 16 columns remain
          uint32_t v[32];
          if (full) {
            tmem_ld32(taddr + c0, v);
          } else {
            uint32_t(&v16)[16] = *reinterpret_cast<uint32_t(*)[16]>(&v[0]);
            tmem_ld16(taddr + c0, v16);
#pragma unroll
            for (int j = 16; j < 32; ++j) v[j] = 0u;
          }
          tmem_wait_ld();
          if (c0 + 32 >= n) {
            tc_fence_before();
            __syncwarp();  // every lane's loads of the accumulator are complete
            if (lane == 0) mbar_arrive(tempty0 + 8 * acc);  // the accumulator is in registers now
          }
          store_block(v, c0, full);
        }
      }
      ++it;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
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

bool g_attr_set[5][64] = {};

}  // namespace

cudaError_t launch_gemm_swap(const Launch& l, int mode, const SwapOperands& o, const GemmShape& s,
                             const GemmBuffers& b) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const int kind = o.nv ? 4 : (o.b128 ? 3 : (o.mx ? 2 : (o.fp8 ? 1 : 0)));
  void (*const kernel)(const Args) =
      kind == 4 ? gemm_swap_kernel<4>
                : (kind == 3 ? gemm_swap_kernel<3>
                             : (kind == 2 ? gemm_swap_kernel<2> : (kind == 1 ? gemm_swap_kernel<1> : gemm_swap_kernel<0>)));
  if (!g_attr_set[kind][dev]) {
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return err;
    g_attr_set[kind][dev] = true;
  }
  if ((reinterpret_cast<uintptr_t>(o.w) | reinterpret_cast<uintptr_t>(o.x)) & 15u) return cudaErrorInvalidValue;
  if ((kind == 2 || kind == 4) && (o.w_sf == nullptr || o.x_sf == nullptr ||
                    ((reinterpret_cast<uintptr_t>(o.w_sf) | reinterpret_cast<uintptr_t>(o.x_sf)) & 15u)))
    return cudaErrorInvalidValue;
  // FP8 block-128: K and the weight rows whole 128-blocks, the K chunks' weight scales held
  // one per lane of a warp
  if (kind == 3 && (o.w_scale == nullptr || s.K % 128 != 0 || s.N % 128 != 0 || s.K / 128 > 32))
    return cudaErrorInvalidValue;
  Args a;
  a.mode = mode;
  a.m_tiles = (s.N + kMW - 1) / kMW;
  if (kind == 4 && (o.w_scale == nullptr || s.K % 256 != 0)) return cudaErrorInvalidValue;
  const int chunk_elems = kind == 4 ? 256 : (kind != 0 ? 128 : 64);  // elements of K in a 128-byte chunk
  a.k_chunks = (s.K + chunk_elems - 1) / chunk_elems;
  a.k_total = s.k_total;
  a.num_pairs = s.num_pairs;
  a.activation = s.activation;
  a.w = static_cast<const uint8_t*>(o.w);
  a.x = static_cast<const uint8_t*>(o.x);
  a.out = b.out;
  a.out_chunks = o.out_chunks;
  a.out_cols = s.out_cols;
  a.num_groups = b.num_groups;
  a.group_info = b.group_info;
  a.sorted_pair_ids = b.sorted_pair_ids;
  a.topk_w = b.topk_w;
  a.tile_counter = b.tile_counter;
  a.status = b.status;
  a.w_scale = o.w_scale;
  a.in_scale = o.in_scale;
  a.act_inv = o.act_scale > 0.f ? 1.0f / o.act_scale : 0.f;
  a.w_sf = static_cast<const uint8_t*>(o.w_sf);
  a.x_sf = static_cast<const uint8_t*>(o.x_sf);
  a.ws_rows = s.N / 128;
  a.up_block = o.up_block;
  a.y_exp = b.out_exp;
  if (mode == 1 && (a.y_exp == nullptr || s.out_cols % 32 != 0)) return cudaErrorInvalidValue;
  a.w_early = o.w_early;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  make_launch_config(&cfg, attr, l, dim3(s.num_sms), dim3(kind == 3 ? threads_for<3>() : kThreads), kSmemBytes);
  return cudaLaunchKernelEx(&cfg, kernel, a);
}

}  // namespace moe
