// Host-side declarations shared by the kernel files and the C-ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

constexpr int kMaxExperts = 1024;  // routed + shared
constexpr int kMaxSlots = 16;      // k' = topk + num_shared
constexpr int kAlignChunk = 2048;  // pairs per align chunk
// A row group's second int32 (group_info[g].y): expert | rows << 16 | padding rows << 25. rows
// is a multiple of 16, at most 256; the padding rows (sentinels, fewer than 16) are the
// group's last rows and only an expert's last group has any.
__host__ __device__ constexpr int group_word(int e, int rows, int pad) { return e | (rows << 16) | (pad << 25); }
__host__ __device__ constexpr int group_word_rows(int y) { return (y >> 16) & 0x1ff; }
__host__ __device__ constexpr int group_word_pad(int y) { return (y >> 25) & 0xf; }
__host__ __device__ constexpr int group_word_expert(int y) { return y & 0xffff; }
constexpr int kRouteAlignTokensPerWarp = 2;  // fused routing + align: tokens per warp (8 warps)
constexpr int kFusedPermutePairs = 64;       // fused routing + align also permutes (bf16) up to this many pairs
// Status word value (beyond the wait timeouts 0x10000 | site): caller-supplied routing held
// an expert id outside [0, E_r) (the pair was dropped: id 0, weight 0).
constexpr int kStatusBadRouting = 0x20000;

// Launch configuration shared by all launchers.
struct Launch {
  cudaStream_t stream;
  bool pdl;
};

// Fill `cfg` (grid, block, smem, stream) and the PDL attribute in `attr`.
void make_launch_config(cudaLaunchConfig_t* cfg, cudaLaunchAttribute* attr, const Launch& l,
                        dim3 grid, dim3 block, size_t smem);

// ---- route (route.cu) ----
cudaError_t launch_route(const Launch& l, const float* logits, int T, int E_routed, int topk,
                         int num_shared, int renormalize, int* topk_ids, float* topk_w,
                         int* status, const void* hidden, int hidden_row_bytes);

// Caller-supplied routing ids/weights [T, topk] into topk_ids/topk_w [T, k'] (route.cu).
// The caller clears the status words first.
cudaError_t launch_load_routing(const Launch& l, const int* ids_in, const float* w_in, int T, int E_routed,
                                int topk, int num_shared, int* topk_ids, float* topk_w, int* status);

// ---- align (align.cu) ----
// num_blocks[0] = P_pad / block_m. With group_rows > 0 (block_m 16), each expert's rows
// are also cut into row groups of at most group_rows rows (multiples of 16, sizes as even
// as possible): group_info[g] = {first row, expert | rows << 16}, num_blocks[1] = count
// (num_blocks[1] is not touched when group_rows is 0).
cudaError_t launch_align(const Launch& l, const int* topk_ids, int P, int E, int block_m,
                         int num_chunks, int* chunk_hist, int* sorted_pair_ids,
                         int* expert_offsets, int* block_expert, int* pair_to_row,
                         int* num_blocks, int group_rows, int2* group_info);
// Routing (as launch_route) and align (as launch_align with one chunk) of a batch of at most
// 8 * kRouteAlignTokensPerWarp tokens and kAlignChunk pairs in one single-CTA kernel; with xs
// (bf16 hidden rows of hidden_row_bytes, row groups, at most kFusedPermutePairs pairs) also
// the permute step into xs.
cudaError_t launch_route_align(const Launch& l, const float* logits, int T, int E_routed, int topk, int num_shared,
                               int renormalize, int* topk_ids, float* topk_w, int* status, const void* hidden,
                               int hidden_row_bytes, int E, int block_m, int* sorted_pair_ids, int* expert_offsets,
                               int* block_expert, int* pair_to_row, int* num_blocks, int group_rows,
                               int2* group_info, void* xs);
// The token rows of every row group in the row-group order of the swapped-operand GEMM
// (gemm_swap.cu): row j of the group starting at x_row is hidden[sorted_pair_ids[x_row +
// j] / k_total] (zero for padding), H / 64 chunks of 128 bytes, swizzled.
cudaError_t launch_permute_rows(const Launch& l, const void* hidden, int H, const int* sorted_pair_ids,
                                const int* num_groups, const int2* group_info, int P, int k_total, void* xs,
                                int num_sms);
// As launch_permute_rows with every element quantised to e4m3(x * fp32(1 / input_scale)):
// H bytes per row, 128-byte chunks of 128 elements.
cudaError_t launch_permute_quant_rows(const Launch& l, const void* hidden, int H, const int* sorted_pair_ids,
                                      const int* num_groups, const int2* group_info, int P, int k_total,
                                      float input_scale, void* xs, int num_sms);
// FP8 block-128: the token rows of every row group, quantised per 1x128 group once per token
// by launch_quant_act (xq e4m3 [T, H], xq_scale fp32 [T, H/128]), copied into the X layout
// above with KC = H / 128. Padding rows are zero codes with scale 1.
cudaError_t launch_permute_b128_rows(const Launch& l, const void* xq, const float* xq_scale, int H,
                                     const int* sorted_pair_ids, const int* num_groups, const int2* group_info, int P,
                                     int k_total, void* xs, int num_sms);
// FP8 block-128: GEMM1's bf16 activation (row-group order, 64-column chunks) quantised per
// 1x128 group the same way into the X layout above with KC = I / 128, for GEMM2.
cudaError_t launch_act_quant_b128(const Launch& l, const void* act, int I, const int* num_groups,
                                  const int2* group_info, void* actq, int num_sms);

// ---- GEMMs (gemm_bf16.cu, gemm_fp8.cu) ----
struct GemmShape {
  int K;                  // reduction length
  int N;                  // output columns of the GEMM (N1 or H)
  int BN;                 // N tile
  int w_rows_per_expert;  // rows per expert in the 2-D weight tensor map
  int k_total;            // slots per token (k')
  int num_pairs;          // P
  int activation;         // moe_activation_t (GEMM1)
  int out_cols;           // leading dimension of the output (I for act, H for y)
  int num_sms;
};
struct GemmBuffers {
  const int* num_blocks;
  const int* block_expert;
  const int* sorted_pair_ids;
  const float* topk_w;
  void* out;
  float* out_scale;         // FP8 GEMM1: act scales [max_rows, I/128]
  const float* a_scale;     // FP8: activation scales of the A operand
  const float* w_scale;     // FP8: weight block scales
  int a_scale_cols;         // FP8: columns of a_scale (K/128)
  int w_scale_rows;         // FP8: rows of w_scale per expert
  int w_scale_cols;         // FP8: columns of w_scale (K/128)
  int up_block_offset;      // FP8 GEMM1: row-block offset of the up half (I/128)
  int* tile_counter;        // [2] work counter of the persistent kernel; 0 between launches
  int* status;
  const int* num_groups;    // row groups (gemm_swap)
  const int2* group_info;
  // GEMM2 of the swapped-operand GEMMs: unweighted y as fp16 [rows, H] (out) with one
  // power-of-two exponent per 32 columns of each row here, int8 [rows, H/32]: y = y16 * 2^exp
  int8_t* out_exp;
};
// Operands of the swapped-operand GEMM: tiled weights, X in row-group order, and (GEMM1)
// the number of 64-column chunks of the activation it writes in row-group order.
struct SwapOperands {
  const void* w;
  const void* x;
  int out_chunks;
  // per-tensor FP8 (e4m3 operands): fp8 = 1, w_scale [E]; in_scale = the X operand's scale
  // (GEMM1: the input scale; GEMM2: the activation scale); act_scale = GEMM1's output
  // requantisation scale (the activation scale)
  int fp8;
  const float* w_scale;
  float in_scale, act_scale;
  // MXFP8 (e4m3 operands with E8M0 scales per 32 values of K, applied by the MMA): mx = 1;
  // w_sf = the tiled weight scales (512 bytes per 128-row x 128-column tile), x_sf = the X
  // operand's scales (1024 bytes per 128-column chunk per 16 rows of the group's first row)
  int mx;
  const void* w_sf;
  const void* x_sf;
  // FP8 block-128 (e4m3 operands, fp32 scales per 128x128 weight block and per 1x128 group
  // of X, promoted in the epilogue): b128 = 1; w_scale [E, rows/128, K/128] in the
  // checkpoint block layout; gated GEMM1 sets up_block = I / 128 (the up half's first block
  // row). X is in row-group order with each K step's codes followed by the fp32 scales of
  // its rows (launch_permute_b128_rows, launch_act_quant_b128).
  int b128;
  int up_block;
  // NVFP4 (packed E2M1 operands, E4M3 scales per 16 values of K applied by the MMA): nv = 1;
  // w_sf / x_sf = the tiled weight scales / the X scale blocks (kNvChunkScaleBytes per 128-row
  // block per chunk); w_scale [E] and in_scale the tensor scales (dequantised in the epilogue)
  int nv;
  // 1: the kernel launched before this GEMM does not write the row groups (they were complete
  // before it could launch this one), so the weight stream may start before the dependency
  // wait; 0: everything waits
  int w_early;
};
// Row groups of the MXFP8 swapped-operand GEMMs: at most this many rows, so that two
// accumulators leave a quarter of TMEM for the block scales.
constexpr int kMxGroupRows = 192;
// Row groups of the FP8 block-128 swapped-operand GEMMs: at most this many rows, so that a
// group's fp32 accumulator fits the epilogue threads' registers.
constexpr int kB128GroupRows = 128;
// K chunks (128-byte chunk rows) per K step of the swapped-operand GEMMs for a row group
// of n rows: steps of 48 to 72 KB of operands.
__host__ __device__ constexpr int chunks_per_step(int n) {
  return n <= 32 ? 4 : (n <= 64 ? 3 : (n <= 128 ? 2 : 1));
}
// FP8 block-128 X layout (row-group order with each K step's fp32 row scales behind its
// codes): the group of n rows at sorted row x_row owns bytes [x_row * KC * 132, (x_row + n)
// * KC * 132); its step of chunks [c0, c0 + kcs), kcs = min(chunks_per_step(n), KC - c0),
// starts at c0 * n * 132 and holds kcs chunks of n rows x 128 bytes of e4m3 codes (row j
// of chunk c at (c - c0) * n * 128 + j * 128, its 16-byte pieces swizzled by j % 8), then
// the fp32 scales of chunk c, row j at kcs * n * 128 + ((c - c0) * n + j) * 4.
constexpr int kB128RowBytesPerChunk = 132;
// N tile for a GEMM with N output columns, given an estimate of the number of 128-row
// tiles and the SM count (0 if no multiple of 32 divides N).
int pick_bn(int N, long long est_row_tiles, int num_sms);
size_t gemm_bf16_smem_bytes();
cudaError_t launch_gemm1_bf16(const Launch& l, const void* hidden, const CUtensorMap& tm_w13,
                              const CUtensorMap& tm_act_store, const GemmShape& s, const GemmBuffers& b);
cudaError_t launch_gemm2_bf16(const Launch& l, const CUtensorMap& tm_act, const CUtensorMap& tm_w2,
                              const CUtensorMap& tm_y_store, const GemmShape& s, const GemmBuffers& b);
// Row groups of at most 256 token rows as the MMA's N operand, 128 weight rows as M.
// mode 0 = GEMM1 (b.out: activation in row-group order), mode 1 = GEMM2 (b.out: y fp32).
cudaError_t launch_gemm_swap(const Launch& l, int mode, const SwapOperands& o, const GemmShape& s,
                             const GemmBuffers& b);
size_t gemm_fp8_smem_bytes();
cudaError_t launch_gemm1_fp8(const Launch& l, const void* xq, const CUtensorMap& tm_w13,
                             const CUtensorMap& tm_act_store, const GemmShape& s, const GemmBuffers& b);
cudaError_t launch_gemm2_fp8(const Launch& l, const CUtensorMap& tm_actq, const CUtensorMap& tm_w2,
                             const CUtensorMap& tm_y_store, const GemmShape& s, const GemmBuffers& b);

// ---- MXFP8 (quant.cu, permute.cu, prepare.cu) ----
// Codes and E8M0 scale bytes of rows of bf16 values, one scale per 32 columns.
cudaError_t launch_quant_weights_mx(const Launch& l, const void* w, long long rows, int cols, void* codes,
                                    void* scales);
// Hidden rows in row-group order as MXFP8 codes (128-column chunks, like the per-tensor
// layout) plus their scales: for the group starting at sorted row x_row, chunk c, a
// 1024-byte block at ((x_row / 16) * H/128 + c) * 1024 holding two 512-byte blocks of 128
// rows each (byte 16 l + 4 j + k: row 32 j + l, K block 4 c + k).
cudaError_t launch_permute_mx_rows(const Launch& l, const void* hidden, int H, const int* sorted_pair_ids,
                                   const int* num_groups, const int2* group_info, int P, int k_total, void* xs,
                                   void* xs_sf, int num_sms);
// GEMM1's bf16 activation (row-group order, 64-column chunks) to MXFP8 codes (128-column
// chunks) and scales in the layout above, for GEMM2.
cudaError_t launch_act_quant_mx(const Launch& l, const void* act, int I, const int* num_groups,
                                const int2* group_info, void* actq, void* act_sf, int num_sms);
size_t tiled_scale_bytes_mx(int E, int rows, int K);

// ---- NVFP4 (quant.cu, permute.cu, prepare.cu) ----
// Row groups of the NVFP4 swapped-operand GEMMs: at most this many rows (two accumulators
// leave half of TMEM for four buffers of block scales).
constexpr int kNvGroupRows = 128;
// Bytes of one K chunk's block scales for 128 rows: four 512-byte blocks, one per MMA of
// K = 64 (a 128-byte chunk row holds 256 E2M1 values, sixteen 16-value blocks): byte
// 512 m + 16 l + 4 j + k of a chunk's blocks is the scale of row 32 j + l for block 4 m + k.
constexpr int kNvChunkScaleBytes = 2048;
// NVFP4 weights: per matrix g = amax / (6 * 448) (1 if all zero) into global_scales[m],
// then per block of 16 values of a row: scale e4m3(amax / 6 / g) and E2M1 codes of
// x / (scale * g), two per byte (lower K index in the low nibble). w bf16 [num_mats,
// mat_elems]; codes [num_mats, mat_elems / 2]; scales [num_mats, mat_elems / 16].
cudaError_t launch_quant_weights_nvfp4(const Launch& l, const void* w, int64_t num_mats, int64_t mat_elems,
                                       void* codes, void* scales, float* global_scales);
// The same for rows of bf16 values with a fixed tensor scale g (the hidden rows: the input
// scale; GEMM1's activation: the activation scale).
cudaError_t launch_quant_rows_nvfp4(const Launch& l, const void* x, long long rows, int cols, float g, void* codes,
                                    void* scales);
// The token rows of every row group (quantised per token by launch_quant_rows_nvfp4: codes
// [T, H/2], scales [T, H/16]) in row-group order: codes in 128-byte chunk rows (256 values)
// as the per-tensor FP8 layout, scales in kNvChunkScaleBytes blocks at ((x_row / 16) *
// (H / 256) + c) * kNvChunkScaleBytes for the group starting at sorted row x_row.
cudaError_t launch_permute_nvfp4_rows(const Launch& l, const void* xq, const void* xq_scale, int H,
                                      const int* sorted_pair_ids, const int* num_groups, const int2* group_info, int P,
                                      int k_total, void* xs, void* xs_sf, int num_sms);
// GEMM1's bf16 activation (row-group order, 64-column chunks) to NVFP4 under tensor scale g,
// in the layout of launch_permute_nvfp4_rows with H = I, for GEMM2.
cudaError_t launch_act_quant_nvfp4(const Launch& l, const void* act, int I, float g, const int* num_groups,
                                   const int2* group_info, void* actq, void* act_sf, int num_sms);
// Tiled NVFP4 weight scales beside the tiled codes: per (expert, 128-row block, 256-value
// chunk) one kNvChunkScaleBytes block (rows interleaved like the codes for gated w13).
size_t tiled_scale_bytes_nvfp4(int E, int rows, int K);
cudaError_t launch_tile_scales_nvfp4(const Launch& l, int which, const void* in, void* out, int E, int H, int I,
                                     int gated);
cudaError_t launch_tile_scales_mx(const Launch& l, int which, const void* in, void* out, int E, int H, int I,
                                  int gated);

// ---- expert parallelism (ep.cu) ----
// owner[p] = ids[p] / per_rank for a routed id (< E_r), `rank` for the shared slot.
cudaError_t launch_ep_owner(const Launch& l, const int* ids, long long P, int E_r, int per_rank, int rank,
                            int* owner);
// Send rows in the order of sorted_pair_ids (rows < send_offsets[world], at most max_rows):
// hidden row, owner-local expert id and weight of each pair; zero for padding rows.
cudaError_t launch_ep_pack(const Launch& l, const void* hidden, int H, const int* sorted_pair_ids,
                           const int* send_offsets, int world, int P, int k_total, const int* ids, const float* weights,
                           int E_r, int per_rank, long long max_rows, void* send_rows, int* send_expert,
                           float* send_weight, int num_sms);
// out[t] = bf16(sum_j returned[pair_to_row[t k' + j]]) in slot order, fp32 accumulation.
cudaError_t launch_ep_combine(const Launch& l, const void* returned, const int* pair_to_row, int T, int k_total, int H,
                              void* out);

// ---- elementwise (combine.cu, quant.cu, prepare.cu) ----
// y: fp32 [rows, H] already weighted (y_exp == nullptr), or unweighted fp16 [rows, H] scaled by
// 2^y_exp[row][col / 32], weighted here by topk_w [T, k'].
cudaError_t launch_combine(const Launch& l, const void* y, const int8_t* y_exp, const float* topk_w,
                           const int* pair_to_row, int T, int k_total, int H, void* out);
cudaError_t launch_quant_act(const Launch& l, const void* x, int T, int H, void* q, float* scale);
// As launch_quant_act over the first num_blocks[0] * block_m of max_rows rows.
cudaError_t launch_quant_rows(const Launch& l, const void* x, int max_rows, int cols, const int* num_blocks,
                              int block_m, void* q, float* scale);
cudaError_t launch_quant_weights(const Launch& l, const void* w, int64_t num_mats, int rows,
                                 int cols, void* q, float* scale);
cudaError_t launch_prepare_w13(const Launch& l, const void* in, void* out, int E, int I_in,
                               int I_pad, int H, int gated, int elt_bytes);
cudaError_t launch_prepare_w2(const Launch& l, const void* in, void* out, int E, int H, int I_in,
                              int I_pad, int elt_bytes);
// bf16 weights in the tiled layout of gemm_swap.cu: which = 0 for w13 (rows N1, K = H),
// 1 for w2 (rows H, K = I_pad), from the checkpoint layout (moe_prepare_weights).
size_t tiled_weight_bytes(int E, int rows, int K);
cudaError_t launch_tile_weights(const Launch& l, int which, const void* in, void* out, int E, int H, int I_in,
                                int I_pad, int gated);
// The same for e4m3 codes (1 byte, 128 elements per 128-byte chunk row): tiles of 128 rows x
// 128 bytes; tiled_weight_bytes_u8 gives the size (rows, K bytes). k_div = 2 tiles packed
// E2M1 codes (two values per byte: 256 values per chunk row, K bytes = K / 2).
size_t tiled_weight_bytes_u8(int E, int rows, int K);
cudaError_t launch_tile_weights_u8(const Launch& l, int which, const void* in, void* out, int E, int H, int I,
                                   int gated, int k_div = 1);
// Per-tensor FP8 weight quantisation of num_mats bf16 [rows, cols] matrices: scale = amax
// / 448 per matrix (1 for all zeros), codes = e4m3(w / scale).
cudaError_t launch_quant_weights_per_tensor(const Launch& l, const void* w, int64_t num_mats, int64_t mat_elems,
                                            void* codes, float* scales);

}  // namespace moe
