/*
 * moe_b200.h -- C ABI of the B200 (sm_100a) fused Mixture-of-Experts layer forward.
 *
 * One call computes, for T tokens with hidden rows x_t (bf16, H wide):
 *   1. route    top-k experts per token from fp32 router logits, softmax weights,
 *               optional renormalisation, optional fused shared-expert slot;
 *   2. align    stable sort of the T*k' (token, slot) pairs by expert, each expert's
 *               segment padded to the GEMM row tile (block_m);
 *   3. GEMM1    z = W13[e] x_t with the SwiGLU (silu(gate)*up) or relu2 (max(z,0)^2)
 *               activation applied in the GEMM epilogue, so only the I-wide result
 *               reaches memory;
 *   4. GEMM2    y = w_tj * (W2[e] a);
 *   5. combine  out_t = sum_j y_tj, in slot order j = 0..k'-1 (deterministic).
 * k' = topk + num_shared. Pair p = t*k' + j.
 *
 * Sources, by page title and section:
 *   "FlashInfer TRTLLM-Gen MoE kernel optimisation: NemotronH support" (sglang PR 21321):
 *       section 1, the fused op trtllm_fp8_block_scale_moe(hidden_states, w13, w2, scales,
 *       expert_weights, topk, renormalize, ..., activation_type) returning a bf16 tensor
 *       of the hidden shape; section 2, intermediate padding (16 gated / 128 non-gated)
 *       and the gated-only gate/up row reordering.
 *   "[MoE] SwiGLU fusion into the MoE up-GEMM epilogue" (sglang PR 32944): section 1, the
 *       activation in the GEMM1 epilogue writing N/2 columns; section 3, the load-time
 *       [gate0, up0, gate1, up1, ...] interleave.
 *   "Qwen3-Next FP8 MoE optimisation: shared-expert fusion for H200" (sglang PR 26204):
 *       sections 1-2, FP8 W8A8 with 128x128 block scales and the shared expert fused as
 *       an extra, always-selected expert slot.
 *   "W4A8 grouped GEMM optimisation for GLM-5.2 MoE on H200" (sglang PR 38220): section 1,
 *       the grouped-GEMM contract (expert_offsets, problem sizes).
 *
 * Conventions for every entry point:
 *   - Pointers named d_* or documented as "device" are CUDA device pointers; "host"
 *     pointers are CPU memory. All buffers are owned by the caller; the library
 *     allocates no memory and keeps no per-call state outside the caller's workspace.
 *   - Device pointers must be 16-byte aligned. Tensors are dense, row-major, with the
 *     layouts stated at each argument.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default stream)
 *     and runs asynchronously unless stated otherwise. No entry point synchronises
 *     except moe_forward_host and moe_get_device_status.
 *   - All argument checks run on the host before any launch; a failing check returns an
 *     error status and enqueues nothing. No C++ exception crosses this interface.
 *   - A launch failure returns MOE_ERR_CUDA (the CUDA error is left for
 *     cudaGetLastError). A device without sm_100 support returns MOE_ERR_UNSUPPORTED:
 *     there is no fallback path.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* == cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,         /* null/misaligned pointer, inconsistent sizes */
  MOE_ERR_UNSUPPORTED = 2,         /* valid but not implemented (shape, dtype, device) */
  MOE_ERR_WORKSPACE_TOO_SMALL = 3, /* workspace_bytes < moe_workspace_size() */
  MOE_ERR_CUDA = 4,                /* a CUDA runtime call or launch failed */
  MOE_ERR_DEVICE_TIMEOUT = 5       /* a kernel gave up a bounded wait (see moe_get_device_status) */
} moe_status_t;

/* Activation of GEMM1 ("activation_type", sglang PR 21321 section 1). The numeric
 * values are this library's own; the page does not print FlashInfer's enum values. */
typedef enum {
  MOE_ACT_SWIGLU = 0, /* gated: a_n = silu(gate_n) * up_n, silu(x) = x / (1 + e^-x) */
  MOE_ACT_RELU2 = 1,  /* non-gated: a_n = max(z_n, 0)^2 */
  MOE_ACT_GELU_TANH = 2, /* gated: a_n = gelu_tanh(gate_n) * up_n, gelu_tanh(x) = 0.5 x (1 +
                            tanh(sqrt(2/pi) (x + 0.044715 x^3))) ("FlashInfer gated MoE kernel
                            optimisation for Blackwell", section 2; padded like SWIGLU) */
  MOE_ACT_SWIGLUOAI = 3  /* gated, "swigluoai_uninterleave" of the same page, section 2: the
                            SwiGLU variant published with OpenAI's gpt-oss models, on gate and
                            up halves that are not interleaved (the w13 checkpoint layout of
                            SWIGLU): g = min(gate_n, 7), u = clamp(up_n, -7, 7),
                            a_n = g / (1 + e^(-1.702 g)) * (u + 1); padded like SWIGLU */
} moe_activation_t;

/* Weight / activation number format. */
typedef enum {
  MOE_DTYPE_BF16 = 0,         /* bf16 weights and activations, fp32 accumulation */
  MOE_DTYPE_FP8_BLOCK128 = 1, /* e4m3 weights with one fp32 scale per 128x128 block and
                                 e4m3 activations with one fp32 scale per 1x128 group
                                 (FP8 W8A8, block_shape [128, 128]; sglang PR 26204
                                 section 1) */
  MOE_DTYPE_FP8_PER_TENSOR = 2, /* e4m3 weights with one fp32 scale per expert matrix, e4m3
                                   GEMM inputs with the static problem->input_scale and
                                   problem->activation_scale (the per-tensor FP8 variant,
                                   sglang PR 21321 sections 1-2); I and H multiples of 128 */
  MOE_DTYPE_MXFP8 = 3,          /* MXFP8: e4m3 weights and GEMM inputs, each with one E8M0
                                   (power-of-two) scale per 32 values of K (the MXFP8 weights
                                   of sglang PR 21321 section 2), applied by the tensor core's
                                   block-scaled MMA. Conversion (weights, hidden rows and
                                   GEMM1's bf16 activation): OCP Microscaling v1.0, shared
                                   exponent floor(log2(amax)) - 8 clamped to [-127, 127]
                                   (-127 for an all-zero block), byte = exponent + 127, codes
                                   e4m3(x * 2^-exponent) round to nearest even, saturating.
                                   I and H multiples of 128. */
  MOE_DTYPE_NVFP4 = 4           /* NVFP4 W4A4 ("FlashInfer gated MoE kernel optimisation for
                                   Blackwell", section 4, names NVFP4 weights; the format is
                                   NVIDIA's): E2M1 values packed two per byte (lower K index in
                                   the low nibble), one E4M3 scale per 16 values of K and one
                                   fp32 scale g per tensor, value = e2m1 * e4m3 * g, with block
                                   scale e4m3(amax / 6 / g) and codes e2m1(x / (scale * g)), round
                                   to nearest even, saturating. The weights carry g per expert
                                   matrix (moe_quantize_weights_nvfp4: amax / (6 * 448)); the GEMM
                                   inputs use the static problem->input_scale (hidden rows) and
                                   problem->activation_scale (GEMM1's activation) as their g, with
                                   block scales per 16 values. The block-scaled MMA applies the
                                   block scales. I and H multiples of 256. */
} moe_wdtype_t;

/* Bit flags of moe_problem_t.flags. */
#define MOE_FLAG_PDL 1u /* launch with programmatic dependent launch between kernels */

/* Problem description shared by all entry points. */
typedef struct {
  int32_t num_tokens;   /* T >= 0 */
  int32_t hidden;       /* H > 0, multiple of 128 (FP8: H <= 4096 and I <= 4096) */
  int32_t num_routed;   /* E_r >= 1: columns of router_logits */
  int32_t num_shared;   /* 0 or 1: shared-expert slots; slot id E_r, weight 1, after the
                           routed slots (sglang PR 26204 section 2). Experts in the
                           weights: E = E_r + num_shared <= 1024. */
  int32_t intermediate; /* I after padding (moe_padded_intermediate): multiple of 16 for the
                           gated activations, of 128 for RELU2 and the 8-bit formats, of 256
                           for NVFP4 */
  int32_t topk;         /* 1 <= topk <= E_r; topk + num_shared <= 16 */
  int32_t renormalize;  /* 0/1: divide the selected softmax weights by their sum */
  int32_t activation;   /* moe_activation_t */
  int32_t wdtype;       /* moe_wdtype_t */
  int32_t block_m;      /* row alignment of each expert's segment: 0 = default (16), 16 (the
                           expert's weight rows are the MMA's M operand and its token rows
                           N) or 128 (BF16 and FP8 block-128 only: 128-row token tiles) */
  uint32_t flags;       /* MOE_FLAG_* */
  float input_scale;      /* MOE_DTYPE_FP8_PER_TENSOR: static scale of the hidden rows,
                             x_q = e4m3(x / input_scale); MOE_DTYPE_NVFP4: the hidden rows'
                             tensor scale g; finite, > 0 (ignored otherwise) */
  float activation_scale; /* MOE_DTYPE_FP8_PER_TENSOR: static scale of GEMM1's activation,
                             a_q = e4m3(a / activation_scale); MOE_DTYPE_NVFP4: the
                             activation's tensor scale g; finite, > 0 (ignored otherwise) */
} moe_problem_t;

/* Byte offsets of the intermediates inside the caller's workspace (for inspection by
 * tests and tools; the contents are this library's private format otherwise). */
typedef struct {
  size_t total_bytes;
  size_t status;          /* int32 device status word (0 = ok); the 256-byte region also
                             holds the GEMM kernels' work counters */
  size_t num_blocks;      /* int32 [2]: block_m row blocks after align (= P_pad/block_m), row
                             groups (block_m 16) */
  size_t topk_ids;        /* int32 [T, k'] selected expert ids, slot order */
  size_t topk_w;          /* fp32  [T, k'] routing weights */
  size_t sorted_pair_ids; /* int32 [max_rows]: pair ids sorted by expert, sentinel P in padding */
  size_t expert_offsets;  /* int32 [E+1]: first row of each expert segment; [E] = P_pad */
  size_t block_expert;    /* int32 [max_rows/block_m]: expert of each row tile */
  size_t pair_to_row;     /* int32 [T*k']: sorted row of each pair */
  size_t chunk_hist;      /* int32 [num_chunks, E]: align scratch */
  size_t xq;              /* FP8 block-128: e4m3 [T, H] quantised hidden */
  size_t xq_scale;        /* FP8 block-128: fp32 [T, H/128] */
  size_t act;             /* GEMM1 output: bf16 [max_rows, I] (block_m 128) or bf16 in
                             row-group order (block_m 16; per-tensor FP8: e4m3 codes) */
  size_t actq;            /* FP8 block-128: the activation quantised per 1x128 group, e4m3
                             [max_rows, I] (block_m 128) or codes and fp32 scales in the
                             layout of xs (block_m 16); MXFP8: e4m3 codes in row-group order */
  size_t act_scale;       /* FP8 block-128, block_m 128: fp32 [max_rows, I/128]; MXFP8: E8M0
                             scale blocks */
  size_t y;               /* GEMM2 rows in sorted order: block_m 128: fp32 [max_rows, H], times
                             the routing weight; block_m 16: fp16 [max_rows, H] followed by
                             int8 [max_rows, H/32], row r's columns [32b, 32b+32) scaled by
                             2^(int8 [r, b]), without the routing weight (the combine applies
                             it) */
  size_t xs;              /* block_m 16: the hidden rows of every row group in row-group order
                             (bf16; e4m3 codes for the 8-bit formats; FP8 block-128: each K
                             step's e4m3 codes followed by its rows' fp32 1x128 scales, 132
                             bytes per row per 128 columns); the padding rows are not written
                             (GEMM1 stores zero activation rows for them); size 0 otherwise */
  size_t xs_scale;        /* MXFP8: E8M0 scale bytes of xs: per row group, 1024 bytes per
                             128 columns at ((first row / 16) * H/128 + chunk) * 1024 */
  size_t group_info;      /* int32 pairs [max_rows/16 + 1]: row groups {first row, expert |
                             rows << 16 | padding rows << 25} of the GEMMs (block_m 16): rows
                             a multiple of 16 (at most 256); the padding rows (fewer than 16,
                             the sentinels of an expert's segment) are the last rows of the
                             expert's last group; the count is the second int32 of the
                             num_blocks region */
  size_t io_hidden;       /* staging for moe_forward_host: bf16 [T, H] */
  size_t io_logits;       /* staging for moe_forward_host: fp32 [T, E_r] */
  size_t io_out;          /* staging for moe_forward_host: bf16 [T, H] */
  int64_t max_rows;       /* upper bound of P_pad: round_up(P + min(E,P)*(block_m-1), block_m) */
  int32_t num_chunks;     /* align chunks of 2048 pairs */
  int32_t block_m;
} moe_workspace_layout_t;

/* Human-readable name of a status code (static string). */
const char* moe_status_string(moe_status_t status);

/* Host-only validation of a problem description. No CUDA call. */
moe_status_t moe_check_problem(const moe_problem_t* problem);

/* Intermediate size after alignment padding: round up to 16 (SWIGLU) or 128 (RELU2),
 * as in sglang PR 21321 section 2 (_align_fp8_moe_weights); FP8 requires 128. Returns
 * -1 for invalid arguments. Host only. */
int32_t moe_padded_intermediate(int32_t intermediate, int32_t activation, int32_t wdtype);

/* Workspace layout and size for `problem` (host only). On error `*layout` is zeroed. */
moe_status_t moe_workspace_layout(const moe_problem_t* problem, moe_workspace_layout_t* layout);

/* Workspace bytes for `problem`, or 0 if the problem is invalid. Host only. */
size_t moe_workspace_size(const moe_problem_t* problem);

/* Load-time weight preparation (sglang PR 21321 section 2; PR 32944 section 3).
 *   w13_in  device [E, up_mult*intermediate_in, H], checkpoint order: gate rows [0, I_in)
 *           then up rows [I_in, 2*I_in) for SWIGLU (up_mult 2), I_in rows for RELU2.
 *   w2_in   device [E, H, intermediate_in].
 * The prepared matrices are w13 [E, N1, H] with N1 = 2*I (SWIGLU) or I (RELU2), I =
 * problem->intermediate = moe_padded_intermediate(intermediate_in, ...), SWIGLU rows
 * interleaved [gate0, up0, gate1, up1, ...] and rows of padded indices zero; and w2
 * [E, H, I] with columns >= intermediate_in zero. They are stored
 *   - block_m 128 (FP8 block-128 or BF16 with block_m = 128): row-major as above;
 *   - block_m 16 (the default): tiled for the GEMMs that take the weights as the MMA's M
 *     operand: tile (e, m, c) of rows [128m, 128m+128) and the 128 bytes of columns of
 *     chunk c (64 bf16 or 128 e4m3 columns) at byte ((e*MT + m)*KC + c) * 16384, MT =
 *     ceil(rows/128), KC = the number of such chunks; each tile row is 128 contiguous
 *     bytes whose 16-byte piece q sits at position q ^ (r % 8); rows and columns past the
 *     matrix are zero.
 *   w13_out, w2_out  device, moe_prepared_weights_bytes(problem, 0 / 1) bytes each,
 *                    16-byte aligned, not overlapping the inputs.
 * Elements are bf16 (2 bytes) or e4m3 codes (1 byte) per problem->wdtype. For FP8 the
 * block scales need no change (FP8 requires intermediate_in == I, a multiple of 128);
 * pass them to moe_forward in the checkpoint layout. Asynchronous on `stream`. */
moe_status_t moe_prepare_weights(const moe_problem_t* problem, int32_t intermediate_in,
                                 const void* w13_in, const void* w2_in, void* w13_out,
                                 void* w2_out, moe_stream_t stream);

/* Per-tensor FP8 quantisation of bf16 weights (MOE_DTYPE_FP8_PER_TENSOR):
 *   w        device bf16 [num_mats, rows, cols], rows * cols a multiple of 8, num_mats <= 65535;
 *   codes    device e4m3 [num_mats, rows, cols];
 *   scales   device fp32 [num_mats]: amax / 448 of each matrix (IEEE division; 1 if amax == 0).
 * code = e4m3(w / scale), round to nearest even, saturating at 448. */
moe_status_t moe_quantize_weights_fp8_per_tensor(const void* w, int64_t num_mats, int32_t rows,
                                                 int32_t cols, void* codes, float* scales,
                                                 moe_stream_t stream);

/* MXFP8 quantisation of bf16 weights (MOE_DTYPE_MXFP8), along each row:
 *   w        device bf16 [num_mats, rows, cols], cols a multiple of 32;
 *   codes    device e4m3 [num_mats, rows, cols];
 *   scales   device uint8 [num_mats, rows, cols/32]: E8M0 bytes (exponent + 127).
 * Per block of 32 values of a row: the OCP Microscaling v1.0 conversion (see
 * MOE_DTYPE_MXFP8). Asynchronous on `stream`. */
moe_status_t moe_quantize_weights_mxfp8(const void* w, int64_t num_mats, int32_t rows, int32_t cols,
                                        void* codes, void* scales, moe_stream_t stream);

/* Load-time preparation of MXFP8 weights (problem->wdtype == MOE_DTYPE_MXFP8, default
 * block_m 16):
 *   w13_codes [E, N1, H] e4m3 and w13_scales [E, N1, H/32] E8M0 bytes, checkpoint order
 *             (gate rows then up rows for a gated activation);
 *   w2_codes  [E, H, I] and w2_scales [E, H, I/32]; I = problem->intermediate (a multiple
 *             of 128: the weights come already padded, as for FP8).
 * Each output (moe_prepared_weights_bytes(problem, 0 / 1) bytes, 16-byte aligned) holds the
 * codes tiled as for per-tensor FP8 (tile (e, m, c): rows [128m, 128m+128), columns
 * [128c, 128c+128), 16384 bytes at ((e*MT + m)*KC + c) * 16384, gated rows interleaved
 * [gate0, up0, ...], 16-byte pieces of row r at position q ^ (r % 8)), followed by the
 * scales: a 512-byte block per tile at the same tile index, byte 16 l + 4 j + k = scale of
 * tile row 32 j + l for K block 4 c + k (zero past the matrix). moe_forward takes the
 * prepared buffers and NULL scale pointers. Asynchronous on `stream`. */
moe_status_t moe_prepare_weights_mxfp8(const moe_problem_t* problem, const void* w13_codes,
                                       const void* w13_scales, const void* w2_codes,
                                       const void* w2_scales, void* w13_out, void* w2_out,
                                       moe_stream_t stream);

/* NVFP4 quantisation of bf16 weights (MOE_DTYPE_NVFP4), along each row:
 *   w              device bf16 [num_mats, rows, cols], cols a multiple of 16, num_mats <= 65535;
 *   codes          device uint8 [num_mats, rows, cols/2]: E2M1 pairs, lower column in the low nibble;
 *   scales         device uint8 [num_mats, rows, cols/16]: E4M3 block scales;
 *   global_scales  device fp32 [num_mats]: g = amax / (6 * 448) of each matrix (1 if all zero).
 * Per block of 16 values: scale = e4m3(amax / 6 / g), codes = e2m1(x / (scale * g)) (IEEE
 * divisions; round to nearest even, saturating). Asynchronous on `stream`. */
moe_status_t moe_quantize_weights_nvfp4(const void* w, int64_t num_mats, int32_t rows, int32_t cols,
                                        void* codes, void* scales, float* global_scales,
                                        moe_stream_t stream);

/* Load-time preparation of NVFP4 weights (problem->wdtype == MOE_DTYPE_NVFP4):
 *   w13_codes [E, N1, H/2] and w13_scales [E, N1, H/16] (checkpoint order: gate rows then up
 *             rows for a gated activation), w2_codes [E, H, I/2] and w2_scales [E, H, I/16],
 *             as moe_quantize_weights_nvfp4 writes them; I = problem->intermediate (a multiple
 *             of 256: the weights come padded).
 * Each output (moe_prepared_weights_bytes(problem, 0 / 1) bytes, 16-byte aligned) holds the
 * codes tiled as 128 rows x 128 bytes (256 values of K) per tile at ((e*MT + m)*KC + c) *
 * 16384 (gated rows interleaved [gate0, up0, ...], 16-byte pieces of row r at position
 * q ^ (r % 8)), followed by the scales: a 2048-byte block per tile at the same tile index,
 * byte 512 mm + 16 l + 4 j + k = scale of tile row 32 j + l for block 16 c + 4 mm + k (zero
 * past the matrix). moe_forward takes the prepared buffers with w13_scale / w2_scale = the
 * global scales [E]. Asynchronous on `stream`. */
moe_status_t moe_prepare_weights_nvfp4(const moe_problem_t* problem, const void* w13_codes,
                                       const void* w13_scales, const void* w2_codes,
                                       const void* w2_scales, void* w13_out, void* w2_out,
                                       moe_stream_t stream);

/* Bytes of the prepared w13 (which = 0) or w2 (which = 1) for `problem` (host only), or
 * 0 for an invalid problem or `which`. */
size_t moe_prepared_weights_bytes(const moe_problem_t* problem, int32_t which);

/* Block quantisation of bf16 weights to e4m3 (FP8 W8A8 block-128 weights):
 *   w        device bf16 [num_mats, rows, cols], rows and cols multiples of 128;
 *   codes    device e4m3 [num_mats, rows, cols];
 *   scales   device fp32 [num_mats, rows/128, cols/128].
 * Per 128x128 block: scale = amax/448 (fp32, IEEE division; 1 if amax == 0),
 * code = e4m3(w/scale), round to nearest even, saturating at 448. */
moe_status_t moe_quantize_weights_fp8(const void* w, int64_t num_mats, int32_t rows,
                                      int32_t cols, void* codes, float* scales,
                                      moe_stream_t stream);

/* The layer forward (all five steps), asynchronous on `stream`.
 *   hidden         device bf16 [T, H]
 *   router_logits  device fp32 [T, E_r] (finite values; NaN/Inf are not supported)
 *   w13, w2        device, prepared by moe_prepare_weights for this problem's layout
 *   w13_scale      FP8 block-128: device fp32 [E, N1/128, H/128], checkpoint (gate-first,
 *                  un-interleaved) block order; FP8 per-tensor and NVFP4: device fp32 [E]
 *                  (NVFP4: the global scales); else NULL
 *   w2_scale       FP8 block-128: device fp32 [E, H/128, I/128]; per-tensor, NVFP4: [E]; else
 *                  NULL (MXFP8: both NULL, the scales are part of the prepared weights)
 *   out            device bf16 [T, H] (must not alias hidden)
 *   workspace      device, >= moe_workspace_size(problem) bytes, 256-byte aligned; one
 *                  workspace must not be used by two calls in flight at once.
 * T == 0 returns MOE_OK and enqueues nothing. Routing ids, the permutation and
 * expert_offsets are deterministic; the output is bitwise reproducible run to run. */
moe_status_t moe_forward(const moe_problem_t* problem, const void* hidden,
                         const float* router_logits, const void* w13, const void* w2,
                         const float* w13_scale, const float* w2_scale, void* out,
                         void* workspace, size_t workspace_bytes, moe_stream_t stream);

/* The routed variant of moe_forward: the caller supplies the expert choice instead of
 * router logits ("FlashInfer TRTLLM-Gen MoE kernel optimisation: NemotronH support",
 * section 1, names such a routed form of the fused op), and steps 2-5 run as in
 * moe_forward.
 *   topk_ids       device int32 [T, topk]: routed expert ids in [0, E_r), slot order;
 *                  repeats allowed
 *   topk_weights   device fp32 [T, topk]: their weights, used as given
 * With num_shared = 1 the shared slot (id E_r, weight 1) follows the routed slots. An id
 * outside [0, E_r) is dropped (weight 0) and reported by moe_get_device_status as
 * MOE_ERR_INVALID_ARG (status word bit 0x20000); the other pairs are unaffected. */
moe_status_t moe_forward_routed(const moe_problem_t* problem, const void* hidden,
                                const int32_t* topk_ids, const float* topk_weights,
                                const void* w13, const void* w2, const float* w13_scale,
                                const float* w2_scale, void* out, void* workspace,
                                size_t workspace_bytes, moe_stream_t stream);

/* moe_forward with HOST hidden [T,H] bf16, router_logits [T,E_r] fp32 and out [T,H] bf16
 * (pinned memory gives asynchronous copies; pageable memory works too). The inputs are
 * copied into the workspace staging areas, the forward runs, the output is copied back
 * and the stream is synchronised before returning. Weights and workspace are device
 * memory as in moe_forward. */
moe_status_t moe_forward_host(const moe_problem_t* problem, const void* h_hidden,
                              const float* h_router_logits, const void* w13, const void* w2,
                              const float* w13_scale, const float* w2_scale, void* h_out,
                              void* workspace, size_t workspace_bytes, moe_stream_t stream);

/* The steps as separate calls on the same workspace: route, align, quant_act (FP8
 * block-128, NVFP4), permute (block_m 16), gemm1, gemm2, combine; moe_forward runs exactly
 * these, in this order. They exist so tests can check each intermediate and tools can time each kernel;
 * each requires the previous steps to have been enqueued. */
moe_status_t moe_stage_route(const moe_problem_t* problem, const float* router_logits,
                             void* workspace, size_t workspace_bytes, moe_stream_t stream);
moe_status_t moe_stage_align(const moe_problem_t* problem, void* workspace,
                             size_t workspace_bytes, moe_stream_t stream);
/* FP8 block-128 and NVFP4 only (else MOE_ERR_INVALID_ARG): quantise hidden once per token
 * into the workspace (xq, xq_scale): per 128 columns (FP8 block-128) or to NVFP4 with the
 * input scale (NVFP4). */
moe_status_t moe_stage_quant_act(const moe_problem_t* problem, const void* hidden,
                                 void* workspace, size_t workspace_bytes, moe_stream_t stream);
/* block_m 16 (the default): copy the token rows of every row group into the workspace in
 * the order GEMM1 reads them (xs), quantised on the way for per-tensor FP8 and MXFP8 (FP8
 * block-128 copies the codes and scales of the quant_act step); hidden device bf16 [T, H].
 * block_m 128: nothing to do, MOE_OK. */
moe_status_t moe_stage_permute(const moe_problem_t* problem, const void* hidden, void* workspace,
                               size_t workspace_bytes, moe_stream_t stream);
moe_status_t moe_stage_gemm1(const moe_problem_t* problem, const void* hidden, const void* w13,
                             const float* w13_scale, void* workspace, size_t workspace_bytes,
                             moe_stream_t stream);
moe_status_t moe_stage_gemm2(const moe_problem_t* problem, const void* w2, const float* w2_scale,
                             void* workspace, size_t workspace_bytes, moe_stream_t stream);
moe_status_t moe_stage_combine(const moe_problem_t* problem, void* out, void* workspace,
                               size_t workspace_bytes, moe_stream_t stream);

/* The align step without a workspace, for callers that cannot allocate device memory
 * (an engine plugin that is handed only its input and output tensors, code running under
 * stream capture, or a path where an allocation could synchronise the device). The pages
 * have no counterpart of this entry point; it runs the same kernels as moe_stage_align.
 * Sizes below use max_rows and block_m from moe_workspace_layout(problem) (block_m is 16
 * for the BF16 default, 128 for FP8 block-128 or an explicit problem->block_m of 128):
 *   topk_ids        device int32 [T, k'] expert ids (e.g. from moe_stage_route); read only.
 *                   An id outside [0, E) is skipped: its pair is not placed in any segment
 *                   and its pair_to_row entry is -1 (nothing outside the buffers below is
 *                   written).
 *   sorted_pair_ids device int32 [max_rows]: pair ids sorted by expert, sentinel T*k' in
 *                   the padding (entries past P_pad = num_blocks[0]*block_m are not written)
 *   expert_offsets  device int32 [E+1]
 *   block_expert    device int32 [max_rows/block_m]: expert of each block_m-row tile
 *                   (entries past num_blocks[0] are not written)
 *   pair_to_row     device int32 [T*k']
 *   num_blocks      device int32 [1]: P_pad / block_m
 * These are the workspace fields of the same names. The row groups that moe_stage_align
 * also writes for block_m 16 (group_info and the second num_blocks entry) are not
 * produced, so these outputs do not drive the block_m-16 GEMM stages by themselves.
 * Its scratch is a fixed array of 262144 int32 (1 MiB) in device memory owned by the
 * library: every GPU that loads the library holds it until the process exits. A problem
 * needing more (ceil(T*k'/2048) * E > 262144) returns MOE_ERR_UNSUPPORTED. The first call
 * on a device looks the array up for that device (cudaGetSymbolAddress), so make that
 * first call before any stream capture. All calls on a device share its one array, whose
 * contents persist from call to call: calls that may overlap on the GPU (for example on
 * two streams of one device) race, so the caller must order them. No memory is allocated
 * and nothing is synchronised. */
moe_status_t moe_align_noalloc(const moe_problem_t* problem, const int32_t* topk_ids,
                               int32_t* sorted_pair_ids, int32_t* expert_offsets,
                               int32_t* block_expert, int32_t* pair_to_row, int32_t* num_blocks,
                               moe_stream_t stream);

/* Expert parallelism over `world` ranks (one process per GPU): rank r owns the routed
 * experts [r*E_r/world, (r+1)*E_r/world) (E_r a multiple of world) and a copy of the shared
 * expert, which serves its own rank's tokens. ("W4A8 grouped GEMM optimisation for GLM-5.2
 * MoE on H200", sglang PR 38220, introduction, tunes for EP-8 layouts; the contiguous split and
 * the replicated shared expert are this library's reading.) A forward is: route this rank's T tokens
 * (moe_stage_route), moe_ep_dispatch, an all-to-all of the send segments, the routed forward
 * on the received rows (moe_forward_routed with topk 1 and the rank's E_r/world routed experts
 * plus the shared copy as local experts 0..E_r/world), the reverse all-to-all of the weighted
 * output rows, and moe_ep_combine. `problem` describes the layer on this rank's tokens.
 *
 * Bytes of the dispatch workspace (0 for an invalid problem or world) and the largest
 * number of send rows (-1 if invalid): round_up(T*k' + min(T*k', world)*15, 16). Host only. */
size_t moe_ep_workspace_size(const moe_problem_t* problem, int32_t world);
int64_t moe_ep_max_send_rows(const moe_problem_t* problem, int32_t world);

/* Dispatch: this rank's (token, slot) pairs sorted stably by owner rank, each owner's
 * segment padded to a multiple of 16 rows.
 *   topk_ids, topk_weights  device int32 / fp32 [T, k']: the route step's output (the shared
 *                           slot, id E_r, included)
 *   send_rows     device bf16 [max_send_rows, H]: row i = hidden row of the i-th sorted pair
 *   send_expert   device int32 [max_send_rows]: the pair's expert id on its owner (id mod
 *                 E_r/world; E_r/world for the shared slot)
 *   send_weight   device fp32 [max_send_rows]: its routing weight
 *   send_offsets  device int32 [world+1]: the owner-r segment is rows [offsets[r], offsets[r+1])
 *   pair_to_send_row device int32 [T*k']: send row of pair t*k' + j
 * Padding rows are zero rows with expert 0 and weight 0. workspace: device,
 * moe_ep_workspace_size bytes, 256-byte aligned. T == 0 writes zero offsets. */
moe_status_t moe_ep_dispatch(const moe_problem_t* problem, int32_t world, int32_t rank, const void* hidden,
                             const int32_t* topk_ids, const float* topk_weights, void* send_rows,
                             int32_t* send_expert, float* send_weight, int32_t* send_offsets,
                             int32_t* pair_to_send_row, void* workspace, size_t workspace_bytes,
                             moe_stream_t stream);

/* Combine: out[t] = sum over j = 0..k'-1 of returned_rows[pair_to_send_row[t*k' + j]], in slot
 * order in fp32, rounded once to bf16.
 *   returned_rows  device bf16 [max_send_rows, H]: the owners' weighted outputs, in send order
 *   out            device bf16 [T, H] */
moe_status_t moe_ep_combine(const moe_problem_t* problem, int32_t world, const void* returned_rows,
                            const int32_t* pair_to_send_row, void* out, moe_stream_t stream);

/* Synchronises `stream`, reads and clears the workspace status word. Returns MOE_OK,
 * MOE_ERR_DEVICE_TIMEOUT if a kernel abandoned a bounded wait since the last query
 * (word 0x10000 | site; its outputs are then undefined), MOE_ERR_INVALID_ARG if
 * moe_forward_routed met an expert id out of range (word 0x20000), or MOE_ERR_CUDA.
 * `*detail` (may be NULL) receives the raw word. */
moe_status_t moe_get_device_status(void* workspace, moe_stream_t stream, int32_t* detail);

/* Test of the device-side timeout path (failure detection without a GPU fault). Every
 * wait inside this library's kernels is bounded: when its limit passes, the kernel records
 * 0x10000 | site in the workspace status word and returns, and moe_get_device_status then
 * reports MOE_ERR_DEVICE_TIMEOUT. This call launches one small kernel that waits, through
 * that same bounded wait, on an mbarrier expecting one arrival:
 *   workspace  device, 256-byte aligned; only its status word (offset 0) is written
 *   limit_us   the wait's limit, 1 .. 1000000 microseconds
 *   arrive     1: the kernel arrives first, so the wait completes and the status word is
 *              untouched; 0: nothing arrives, the wait gives up after limit_us and the
 *              status word becomes 0x1007F (site 0x7F)
 * Asynchronous on `stream`; MOE_ERR_INVALID_ARG for a bad pointer or limit. */
moe_status_t moe_selftest_bounded_wait(void* workspace, uint32_t limit_us, int32_t arrive,
                                       moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
