// C ABI of the fused MoE layer forward: argument checks, workspace carving, tensor-map
// encoding and the launch sequence route -> align -> [quant] -> GEMM1 -> GEMM2 -> combine
// on the caller's stream. See include/moe_b200.h for the contract of each entry point.
#include <cudaTypedefs.h>

#include <atomic>
#include <cstring>
#include <mutex>

#include "moe_b200.h"
#include "moe_internal.h"

#define MOE_API extern "C" __attribute__((visibility("default")))

namespace moe {

void make_launch_config(cudaLaunchConfig_t* cfg, cudaLaunchAttribute* attr, const Launch& l, dim3 grid,
                        dim3 block, size_t smem) {
  std::memset(cfg, 0, sizeof(*cfg));
  cfg->gridDim = grid;
  cfg->blockDim = block;
  cfg->dynamicSmemBytes = smem;
  cfg->stream = l.stream;
  if (l.pdl) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg->attrs = attr;
    cfg->numAttrs = 1;
  } else {
    cfg->attrs = nullptr;
    cfg->numAttrs = 0;
  }
}

}  // namespace moe

namespace {

using moe::GemmBuffers;
using moe::GemmShape;
using moe::Launch;

constexpr size_t kAlign = 1024;
constexpr int kGroupRows = 256;  // row groups of the swapped-operand GEMMs: at most this many rows

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

struct Plan {
  int T, H, Er, Es, E, I, topk, kk, bm, grp, N1, gated, fp8, pt, mx, nv, q8, renorm, act;
  float in_scale, act_scale;  // static scales of the GEMM inputs (per-tensor FP8, NVFP4)
  long long P;
  int bn1, bn2;
  moe_workspace_layout_t lay;
};

moe_status_t make_plan(const moe_problem_t* p, Plan* pl) {
  if (p == nullptr || pl == nullptr) return MOE_ERR_INVALID_ARG;
  Plan q;
  std::memset(&q, 0, sizeof(q));
  if (p->num_tokens < 0 || p->hidden <= 0 || p->num_routed < 1 || p->topk < 1 || p->intermediate <= 0)
    return MOE_ERR_INVALID_ARG;
  if (p->num_shared != 0 && p->num_shared != 1) return MOE_ERR_INVALID_ARG;
  if (p->topk > p->num_routed) return MOE_ERR_INVALID_ARG;
  if (p->renormalize != 0 && p->renormalize != 1) return MOE_ERR_INVALID_ARG;
  if (p->activation != MOE_ACT_SWIGLU && p->activation != MOE_ACT_RELU2 && p->activation != MOE_ACT_GELU_TANH &&
      p->activation != MOE_ACT_SWIGLUOAI)
    return MOE_ERR_INVALID_ARG;
  if (p->wdtype != MOE_DTYPE_BF16 && p->wdtype != MOE_DTYPE_FP8_BLOCK128 && p->wdtype != MOE_DTYPE_FP8_PER_TENSOR &&
      p->wdtype != MOE_DTYPE_MXFP8 && p->wdtype != MOE_DTYPE_NVFP4)
    return MOE_ERR_INVALID_ARG;
  if (p->flags & ~MOE_FLAG_PDL) return MOE_ERR_INVALID_ARG;
  q.gated = p->activation != MOE_ACT_RELU2;
  q.fp8 = p->wdtype == MOE_DTYPE_FP8_BLOCK128;
  q.pt = p->wdtype == MOE_DTYPE_FP8_PER_TENSOR;
  q.mx = p->wdtype == MOE_DTYPE_MXFP8;
  q.nv = p->wdtype == MOE_DTYPE_NVFP4;
  q.q8 = q.fp8 || q.pt || q.mx || q.nv;  // quantised weights: I must come padded (128; NVFP4 256)
  if (q.pt || q.nv) {
    // static scales: finite and positive
    if (!(p->input_scale > 0.0f && p->input_scale < 3.0e38f) ||
        !(p->activation_scale > 0.0f && p->activation_scale < 3.0e38f))
      return MOE_ERR_INVALID_ARG;
    q.in_scale = p->input_scale;
    q.act_scale = p->activation_scale;
  }
  // the intermediate size must already be padded (moe_padded_intermediate)
  const int ialign = q.nv ? 256 : ((q.q8 || !q.gated) ? 128 : 16);
  if (p->intermediate % ialign != 0) return MOE_ERR_INVALID_ARG;
  if (p->hidden % (q.nv ? 256 : 128) != 0) return MOE_ERR_UNSUPPORTED;
  if (p->num_routed + p->num_shared > moe::kMaxExperts) return MOE_ERR_UNSUPPORTED;
  if (p->topk + p->num_shared > moe::kMaxSlots) return MOE_ERR_UNSUPPORTED;
  if (p->block_m != 0 && p->block_m != 16 && p->block_m != 128) return MOE_ERR_UNSUPPORTED;
  if (p->hidden > (1 << 20) || p->intermediate > (1 << 20)) return MOE_ERR_UNSUPPORTED;
  // FP8: a GEMM's K blocks (H/128 and I/128) are held one per lane of a warp
  if (q.fp8 && (p->hidden > 4096 || p->intermediate > 4096)) return MOE_ERR_UNSUPPORTED;

  q.T = p->num_tokens;
  q.H = p->hidden;
  q.Er = p->num_routed;
  q.Es = p->num_shared;
  q.E = q.Er + q.Es;
  q.I = p->intermediate;
  q.topk = p->topk;
  q.kk = q.topk + q.Es;
  q.N1 = q.gated ? 2 * q.I : q.I;
  // Row alignment. Default: 16-row blocks, the expert's weights as the MMA's M operand and
  // row groups of token rows as N (up to 256 rows; 192 for MXFP8, 128 for FP8 block-128).
  // block_m = 128 (BF16 and FP8 block-128 only): 128-row token tiles.
  if (p->block_m == 128 && (q.pt || q.mx || q.nv)) return MOE_ERR_UNSUPPORTED;
  q.bm = p->block_m != 0 ? p->block_m : 16;
  q.grp = q.bm == 16 ? (q.mx ? moe::kMxGroupRows
                             : (q.fp8 ? moe::kB128GroupRows : (q.nv ? moe::kNvGroupRows : kGroupRows)))
                     : 0;
  q.renorm = p->renormalize;
  q.act = p->activation;
  q.P = static_cast<long long>(q.T) * q.kk;
  if (q.P >= (1LL << 31) - (1LL << 20)) return MOE_ERR_UNSUPPORTED;
  // N tiles for a full device; the launches refine them for the actual SM count
  q.bn1 = moe::pick_bn(q.N1, 1, 1);
  q.bn2 = moe::pick_bn(q.H, 1, 1);
  if (q.bn1 == 0 || q.bn2 == 0) return MOE_ERR_UNSUPPORTED;

  moe_workspace_layout_t& L = q.lay;
  const long long active = q.P < q.E ? q.P : q.E;
  L.block_m = q.bm;
  L.max_rows = static_cast<int64_t>(align_up(static_cast<size_t>(q.P + active * (q.bm - 1)), q.bm));
  L.num_chunks = static_cast<int32_t>(q.P == 0 ? 1 : (q.P + moe::kAlignChunk - 1) / moe::kAlignChunk);
  const size_t T = static_cast<size_t>(q.T), H = q.H, I = q.I, P = static_cast<size_t>(q.P);
  const size_t rows = static_cast<size_t>(L.max_rows);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, kAlign);
    return at;
  };
  L.status = take(256);  // always offset 0 (moe_get_device_status relies on it)
  L.num_blocks = take(256);
  L.topk_ids = take(P * 4);
  L.topk_w = take(P * 4);
  L.sorted_pair_ids = take(rows * 4);
  L.expert_offsets = take((static_cast<size_t>(q.E) + 1) * 4);
  L.block_expert = take(rows / q.bm * 4 + 4);
  L.pair_to_row = take(P * 4);
  L.chunk_hist = take(static_cast<size_t>(L.num_chunks) * q.E * 4);
  const bool fp8_tiles = q.fp8 && q.bm == 128;  // FP8 block-128 with 128-row token tiles
  const bool b128 = q.fp8 && q.bm == 16;        // FP8 block-128 on the swapped-operand GEMMs
  // the hidden rows quantised once per token: FP8 block-128 e4m3 [T, H] + fp32 [T, H/128];
  // NVFP4 packed E2M1 [T, H/2] + E4M3 [T, H/16]
  L.xq = take(q.fp8 ? T * H : (q.nv ? T * H / 2 : 0));
  L.xq_scale = take(q.fp8 ? T * (H / 128) * 4 : (q.nv ? T * H / 16 : 0));
  // the swapped-operand GEMMs keep the activation in row-group order, 128-byte chunks (64
  // bf16 or 128 e4m3 columns)
  const size_t act_bytes = q.pt ? rows * I : rows * (q.bm == 16 ? align_up(I, 64) : I) * 2;
  L.act = take(act_bytes);
  // the activation quantised for GEMM2: FP8 block-128 with token tiles: e4m3 [rows, I] and
  // fp32 [rows, I/128]; on the swapped-operand GEMMs: codes and scales together (132 bytes
  // per row per 128 columns); MXFP8: codes (128-column chunks) and scales, 1024 bytes per 16
  // rows per 128 columns (a group's scale blocks sit at its first row / 16)
  // NVFP4: packed codes (256-value chunks) and scale blocks, 2048 bytes per 16 rows per 256
  // columns (a group's blocks sit at its first row / 16)
  L.actq = take(fp8_tiles || q.mx ? rows * I
                                  : (b128 ? rows * (I / 128) * moe::kB128RowBytesPerChunk : (q.nv ? rows * I / 2 : 0)));
  L.act_scale = take(fp8_tiles ? rows * (I / 128) * 4
                               : (q.mx ? rows / 16 * (I / 128) * 1024
                                       : (q.nv ? rows / 16 * (I / 256) * moe::kNvChunkScaleBytes : 0)));
  L.y = take(rows * H * 4);
  L.xs = take(q.bm == 16 ? (b128 ? rows * (H / 128) * moe::kB128RowBytesPerChunk
                                : (q.nv ? rows * H / 2 : rows * H * (q.pt || q.mx ? 1 : 2)))
                         : 0);
  L.xs_scale = take(q.mx ? rows / 16 * (H / 128) * 1024 : (q.nv ? rows / 16 * (H / 256) * moe::kNvChunkScaleBytes : 0));
  L.group_info = take(q.bm == 16 ? (rows / 16 + 1) * 8 : 0);
  L.io_hidden = take(T * H * 2);
  L.io_logits = take(T * static_cast<size_t>(q.Er) * 4);
  L.io_out = take(T * H * 2);
  L.total_bytes = off;
  *pl = q;
  return MOE_OK;
}

// Device support: sm_100 (compute capability 10.0) only. Caches the SM count.
std::atomic<int> g_dev_sms[64];

moe_status_t device_sms(int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev >= 0 && dev < 64) {
    const int c = g_dev_sms[dev].load(std::memory_order_relaxed);
    if (c > 0) {
      *num_sms = c;
      return MOE_OK;
    }
    if (c < 0) return MOE_ERR_UNSUPPORTED;
  }
  int major = 0, minor = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  const bool ok = major == 10 && minor == 0;
  if (dev >= 0 && dev < 64) g_dev_sms[dev].store(ok ? sms : -1, std::memory_order_relaxed);
  if (!ok) return MOE_ERR_UNSUPPORTED;
  *num_sms = sms;
  return MOE_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &qres) ==
            cudaSuccess &&
        qres == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

// 2-D tensor map over a row-major [outer, inner] matrix with a {box_inner, box_outer}
// box (128-byte swizzle unless stated), zero fill out of bounds.
bool make_tmap_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elt_bytes, uint64_t inner,
                  uint64_t outer, uint32_t box_inner, uint32_t box_outer,
                  CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * static_cast<uint64_t>(elt_bytes)};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T>
T* ws_ptr(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

moe_status_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return MOE_OK;
  if (e == cudaErrorNotSupported) return MOE_ERR_UNSUPPORTED;
  return MOE_ERR_CUDA;
}

moe_status_t check_ws(const Plan& pl, const void* ws, size_t ws_bytes) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < pl.lay.total_bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  return MOE_OK;
}

// ---- the steps (arguments already checked) ----------------------------------------

// `hidden` (may be NULL) is prefetched into L2 for GEMM1's row gather
moe_status_t run_route(const Plan& pl, const float* logits, void* ws, const Launch& l, const void* hidden) {
  const auto& L = pl.lay;
  // the route kernel also resets the device status word: it starts every forward
  return cuda_status(moe::launch_route(l, logits, pl.T, pl.Er, pl.topk, pl.Es, pl.renorm,
                                       ws_ptr<int>(ws, L.topk_ids), ws_ptr<float>(ws, L.topk_w),
                                       ws_ptr<int>(ws, L.status), pl.fp8 ? nullptr : hidden,
                                       pl.H * 2));
}

// Routing and align of a small batch in one kernel (the same results as run_route, run_align);
// with `permute` also the bf16 permute step (the same xs as run_permute).
moe_status_t run_route_align(const Plan& pl, const float* logits, void* ws, const Launch& l, const void* hidden,
                             bool permute) {
  const auto& L = pl.lay;
  return cuda_status(moe::launch_route_align(
      l, logits, pl.T, pl.Er, pl.topk, pl.Es, pl.renorm, ws_ptr<int>(ws, L.topk_ids), ws_ptr<float>(ws, L.topk_w),
      ws_ptr<int>(ws, L.status), pl.fp8 ? nullptr : hidden, pl.H * 2, pl.E, pl.bm, ws_ptr<int>(ws, L.sorted_pair_ids),
      ws_ptr<int>(ws, L.expert_offsets), ws_ptr<int>(ws, L.block_expert), ws_ptr<int>(ws, L.pair_to_row),
      ws_ptr<int>(ws, L.num_blocks), pl.grp, pl.grp != 0 ? ws_ptr<int2>(ws, L.group_info) : nullptr,
      permute ? ws_ptr<void>(ws, L.xs) : nullptr));
}

moe_status_t run_align(const Plan& pl, void* ws, const Launch& l) {
  const auto& L = pl.lay;
  return cuda_status(moe::launch_align(l, ws_ptr<int>(ws, L.topk_ids), static_cast<int>(pl.P), pl.E, pl.bm,
                                       L.num_chunks, ws_ptr<int>(ws, L.chunk_hist),
                                       ws_ptr<int>(ws, L.sorted_pair_ids), ws_ptr<int>(ws, L.expert_offsets),
                                       ws_ptr<int>(ws, L.block_expert), ws_ptr<int>(ws, L.pair_to_row),
                                       ws_ptr<int>(ws, L.num_blocks), pl.grp,
                                       pl.grp != 0 ? ws_ptr<int2>(ws, L.group_info) : nullptr));
}

moe_status_t run_quant_act(const Plan& pl, const void* hidden, void* ws, const Launch& l) {
  const auto& L = pl.lay;
  if (pl.nv)
    return cuda_status(moe::launch_quant_rows_nvfp4(l, hidden, pl.T, pl.H, pl.in_scale, ws_ptr<void>(ws, L.xq),
                                                    ws_ptr<void>(ws, L.xq_scale)));
  return cuda_status(moe::launch_quant_act(l, hidden, pl.T, pl.H, ws_ptr<void>(ws, L.xq),
                                           ws_ptr<float>(ws, L.xq_scale)));
}

GemmBuffers common_buffers(const Plan& pl, void* ws) {
  const auto& L = pl.lay;
  GemmBuffers b;
  std::memset(&b, 0, sizeof(b));
  b.num_blocks = ws_ptr<int>(ws, L.num_blocks);
  b.block_expert = ws_ptr<int>(ws, L.block_expert);
  b.sorted_pair_ids = ws_ptr<int>(ws, L.sorted_pair_ids);
  b.topk_w = ws_ptr<float>(ws, L.topk_w);
  b.status = ws_ptr<int>(ws, L.status);
  b.num_groups = ws_ptr<int>(ws, L.num_blocks) + 1;
  b.group_info = ws_ptr<int2>(ws, L.group_info);
  return b;
}


// The swapped-operand GEMMs (block_m 16) store unweighted y as fp16 [max_rows, H] followed
// by its int8 exponents [max_rows, H/32] (y = y16 * 2^exp; the combine applies the routing
// weight); the 128-row token-tile GEMMs store weighted fp32 [max_rows, H] (no exponents).
int8_t* y_exp_ptr(const Plan& pl, void* ws) {
  if (pl.bm != 16) return nullptr;
  return ws_ptr<int8_t>(ws, pl.lay.y + static_cast<size_t>(pl.lay.max_rows) * pl.H * 2);
}

// Lower bound on the number of 128-row tiles align produces: every expert that receives
// a pair gets at least one, and there are at least ceil(P / 128).
long long est_row_tiles(const Plan& pl) {
  const long long by_rows = (pl.P + 127) / 128;
  const long long by_experts = pl.P < pl.E ? pl.P : pl.E;
  return by_rows > by_experts ? by_rows : by_experts;
}

moe_status_t run_gemm1(const Plan& pl_in, const void* hidden, const void* w13, const float* w13_scale, void* ws,
                       const Launch& l, int num_sms,
                       bool w_early = true) {
  Plan pl = pl_in;
  if (!pl.fp8) pl.bn1 = moe::pick_bn(pl.N1, est_row_tiles(pl), num_sms);
  const auto& L = pl.lay;
  GemmShape s;
  s.K = pl.H;
  s.N = pl.N1;
  s.BN = pl.bn1;
  s.w_rows_per_expert = pl.N1;
  s.k_total = pl.kk;
  s.num_pairs = static_cast<int>(pl.P);
  s.activation = pl.act;
  s.out_cols = pl.I;
  s.num_sms = num_sms;
  GemmBuffers b = common_buffers(pl, ws);
  b.out = ws_ptr<void>(ws, L.act);
  b.tile_counter = ws_ptr<int>(ws, L.status) + 4;
  CUtensorMap ta, tb;
  if (pl.bm == 16) {
    // tiled weights as the MMA's M operand, the token rows in row-group order (run_permute):
    // both operands load with bulk copies
    moe::SwapOperands o{};
    o.w = w13;
    // the kernel before GEMM1 (the permute) does not write the row groups, unless the
    // permute ran inside the routing + align kernel
    o.w_early = w_early ? 1 : 0;
    o.x = ws_ptr<void>(ws, L.xs);
    o.out_chunks = pl.pt ? pl.I / 128 : (pl.I + 63) / 64;
    o.fp8 = pl.pt;
    o.w_scale = w13_scale;
    o.in_scale = pl.in_scale;
    o.act_scale = pl.act_scale;
    if (pl.nv) {
      // NVFP4: the codes and then the scale blocks in the prepared weights; GEMM1 writes the
      // bf16 activation, quantised with the activation scale for GEMM2
      o.nv = 1;
      o.w_sf = static_cast<const uint8_t*>(w13) + moe::tiled_weight_bytes_u8(pl.E, pl.N1, pl.H / 2);
      o.x_sf = ws_ptr<void>(ws, L.xs_scale);
      moe_status_t st = cuda_status(moe::launch_gemm_swap(l, 0, o, s, b));
      if (st != MOE_OK) return st;
      return cuda_status(moe::launch_act_quant_nvfp4(l, ws_ptr<void>(ws, L.act), pl.I, pl.act_scale,
                                                     ws_ptr<int>(ws, L.num_blocks) + 1, ws_ptr<int2>(ws, L.group_info),
                                                     ws_ptr<void>(ws, L.actq), ws_ptr<void>(ws, L.act_scale), num_sms));
    }
    if (pl.fp8) {
      // FP8 block-128: GEMM1 writes the bf16 activation, then quantised per 1x128 for GEMM2
      o.b128 = 1;
      o.up_block = pl.gated ? pl.I / 128 : 0;
      moe_status_t st = cuda_status(moe::launch_gemm_swap(l, 0, o, s, b));
      if (st != MOE_OK) return st;
      return cuda_status(moe::launch_act_quant_b128(l, ws_ptr<void>(ws, L.act), pl.I, ws_ptr<int>(ws, L.num_blocks) + 1,
                                                    ws_ptr<int2>(ws, L.group_info), ws_ptr<void>(ws, L.actq), num_sms));
    }
    if (pl.mx) {
      // the weight scales follow the tiled codes; GEMM1 writes the bf16 activation, which is
      // then quantised for GEMM2
      o.mx = 1;
      o.w_sf = static_cast<const uint8_t*>(w13) + moe::tiled_weight_bytes_u8(pl.E, pl.N1, pl.H);
      o.x_sf = ws_ptr<void>(ws, L.xs_scale);
      moe_status_t st = cuda_status(moe::launch_gemm_swap(l, 0, o, s, b));
      if (st != MOE_OK) return st;
      return cuda_status(moe::launch_act_quant_mx(l, ws_ptr<void>(ws, L.act), pl.I, ws_ptr<int>(ws, L.num_blocks) + 1,
                                                  ws_ptr<int2>(ws, L.group_info), ws_ptr<void>(ws, L.actq),
                                                  ws_ptr<void>(ws, L.act_scale), num_sms));
    }
    return cuda_status(moe::launch_gemm_swap(l, 0, o, s, b));
  }
  if (!pl.fp8) {
    // the token rows of hidden are gathered by the kernel itself (no tensor map); the
    // activation is written in boxes of 32 rows x 16 (SwiGLU) or 32 (relu2) columns
    CUtensorMap tc;
    if (!make_tmap_2d(&tb, w13, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, pl.H, static_cast<uint64_t>(pl.E) * pl.N1,
                      64, pl.bn1) ||
        !make_tmap_2d(&tc, ws_ptr<void>(ws, L.act), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, pl.I,
                      static_cast<uint64_t>(L.max_rows), pl.gated ? 16 : 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE))
      return MOE_ERR_CUDA;
    return cuda_status(moe::launch_gemm1_bf16(l, hidden, tb, tc, s, b));
  }
  // FP8: quantised hidden rows gathered by the kernel; weight codes in 128 x 128 boxes;
  // bf16 activation written in boxes of 32 rows x 64 columns, then quantised per 1x128
  (void)ta;
  CUtensorMap tc;
  if (!make_tmap_2d(&tb, w13, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, pl.H, static_cast<uint64_t>(pl.E) * pl.N1, 128,
                    128) ||
      !make_tmap_2d(&tc, ws_ptr<void>(ws, L.act), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, pl.I,
                    static_cast<uint64_t>(L.max_rows), 64, 32))
    return MOE_ERR_CUDA;
  b.a_scale = ws_ptr<float>(ws, L.xq_scale);
  b.w_scale = w13_scale;
  b.a_scale_cols = pl.H / 128;
  b.w_scale_rows = pl.N1 / 128;
  b.w_scale_cols = pl.H / 128;
  b.up_block_offset = pl.I / 128;
  s.BN = 128;
  moe_status_t st = cuda_status(moe::launch_gemm1_fp8(l, ws_ptr<void>(ws, L.xq), tb, tc, s, b));
  if (st != MOE_OK) return st;
  return cuda_status(moe::launch_quant_rows(l, ws_ptr<void>(ws, L.act), static_cast<int>(L.max_rows), pl.I,
                                            ws_ptr<int>(ws, L.num_blocks), pl.bm, ws_ptr<void>(ws, L.actq),
                                            ws_ptr<float>(ws, L.act_scale)));
}

// The token rows of each row group in row-group order (block_m 16 only).
moe_status_t run_permute(const Plan& pl, const void* hidden, void* ws, const Launch& l, int num_sms) {
  if (pl.bm != 16) return MOE_OK;
  const auto& L = pl.lay;
  if (pl.fp8)
    return cuda_status(moe::launch_permute_b128_rows(
        l, ws_ptr<void>(ws, L.xq), ws_ptr<float>(ws, L.xq_scale), pl.H, ws_ptr<int>(ws, L.sorted_pair_ids),
        ws_ptr<int>(ws, L.num_blocks) + 1, ws_ptr<int2>(ws, L.group_info), static_cast<int>(pl.P), pl.kk,
        ws_ptr<void>(ws, L.xs), num_sms));
  if (pl.nv)
    return cuda_status(moe::launch_permute_nvfp4_rows(
        l, ws_ptr<void>(ws, L.xq), ws_ptr<void>(ws, L.xq_scale), pl.H, ws_ptr<int>(ws, L.sorted_pair_ids),
        ws_ptr<int>(ws, L.num_blocks) + 1, ws_ptr<int2>(ws, L.group_info), static_cast<int>(pl.P), pl.kk,
        ws_ptr<void>(ws, L.xs), ws_ptr<void>(ws, L.xs_scale), num_sms));
  if (pl.mx)
    return cuda_status(moe::launch_permute_mx_rows(
        l, hidden, pl.H, ws_ptr<int>(ws, L.sorted_pair_ids), ws_ptr<int>(ws, L.num_blocks) + 1,
        ws_ptr<int2>(ws, L.group_info), static_cast<int>(pl.P), pl.kk, ws_ptr<void>(ws, L.xs),
        ws_ptr<void>(ws, L.xs_scale), num_sms));
  if (pl.pt)
    return cuda_status(moe::launch_permute_quant_rows(
        l, hidden, pl.H, ws_ptr<int>(ws, L.sorted_pair_ids), ws_ptr<int>(ws, L.num_blocks) + 1,
        ws_ptr<int2>(ws, L.group_info), static_cast<int>(pl.P), pl.kk, pl.in_scale, ws_ptr<void>(ws, L.xs), num_sms));
  return cuda_status(moe::launch_permute_rows(l, hidden, pl.H, ws_ptr<int>(ws, L.sorted_pair_ids),
                                              ws_ptr<int>(ws, L.num_blocks) + 1, ws_ptr<int2>(ws, L.group_info),
                                              static_cast<int>(pl.P), pl.kk, ws_ptr<void>(ws, L.xs), num_sms));
}

moe_status_t run_gemm2(const Plan& pl_in, const void* w2, const float* w2_scale, void* ws, const Launch& l,
                       int num_sms) {
  Plan pl = pl_in;
  if (!pl.fp8) pl.bn2 = moe::pick_bn(pl.H, est_row_tiles(pl), num_sms);
  const auto& L = pl.lay;
  GemmShape s;
  s.K = pl.I;
  s.N = pl.H;
  s.BN = pl.bn2;
  s.w_rows_per_expert = pl.H;
  s.k_total = pl.kk;
  s.num_pairs = static_cast<int>(pl.P);
  s.activation = pl.act;
  s.out_cols = pl.H;
  s.num_sms = num_sms;
  GemmBuffers b = common_buffers(pl, ws);
  b.out = ws_ptr<void>(ws, L.y);
  b.out_exp = y_exp_ptr(pl, ws);
  b.tile_counter = ws_ptr<int>(ws, L.status) + 6;
  CUtensorMap ta, tb;
  const uint64_t rows = static_cast<uint64_t>(L.max_rows);
  if (pl.bm == 16) {
    moe::SwapOperands o{};
    o.w = w2;
    o.w_early = 1;  // the kernel before GEMM2 (GEMM1 or the activation quantiser) writes no row groups
    o.x = ws_ptr<void>(ws, L.act);
    o.out_chunks = 0;
    o.fp8 = pl.pt;
    o.w_scale = w2_scale;
    o.in_scale = pl.act_scale;
    if (pl.fp8) {
      o.b128 = 1;
      o.x = ws_ptr<void>(ws, L.actq);
    }
    if (pl.nv) {
      o.nv = 1;
      o.x = ws_ptr<void>(ws, L.actq);
      o.w_sf = static_cast<const uint8_t*>(w2) + moe::tiled_weight_bytes_u8(pl.E, pl.H, pl.I / 2);
      o.x_sf = ws_ptr<void>(ws, L.act_scale);
    }
    if (pl.mx) {
      o.mx = 1;
      o.x = ws_ptr<void>(ws, L.actq);
      o.w_sf = static_cast<const uint8_t*>(w2) + moe::tiled_weight_bytes_u8(pl.E, pl.H, pl.I);
      o.x_sf = ws_ptr<void>(ws, L.act_scale);
    }
    return cuda_status(moe::launch_gemm_swap(l, 1, o, s, b));
  }
  if (!pl.fp8) {
    CUtensorMap tc;  // y [max_rows, H] fp32 in sorted row order, boxes of 32 x 32
    if (!make_tmap_2d(&ta, ws_ptr<void>(ws, L.act), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, pl.I, rows, 64, 128) ||
        !make_tmap_2d(&tb, w2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, pl.I, static_cast<uint64_t>(pl.E) * pl.H, 64,
                      pl.bn2) ||
        !make_tmap_2d(&tc, ws_ptr<void>(ws, L.y), CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, pl.H, rows, 32, 32))
      return MOE_ERR_CUDA;
    return cuda_status(moe::launch_gemm2_bf16(l, ta, tb, tc, s, b));
  }
  CUtensorMap tc;
  if (!make_tmap_2d(&ta, ws_ptr<void>(ws, L.actq), CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, pl.I, rows, 128, 128) ||
      !make_tmap_2d(&tb, w2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, pl.I, static_cast<uint64_t>(pl.E) * pl.H, 128, 128) ||
      !make_tmap_2d(&tc, ws_ptr<void>(ws, L.y), CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, pl.H, rows, 32, 32))
    return MOE_ERR_CUDA;
  b.a_scale = ws_ptr<float>(ws, L.act_scale);
  b.w_scale = w2_scale;
  b.a_scale_cols = pl.I / 128;
  b.w_scale_rows = pl.H / 128;
  b.w_scale_cols = pl.I / 128;
  s.BN = 128;
  return cuda_status(moe::launch_gemm2_fp8(l, ta, tb, tc, s, b));
}

moe_status_t run_combine(const Plan& pl, void* out, void* ws, const Launch& l) {
  return cuda_status(moe::launch_combine(l, ws_ptr<void>(ws, pl.lay.y), y_exp_ptr(pl, ws),
                                         ws_ptr<float>(ws, pl.lay.topk_w), ws_ptr<int>(ws, pl.lay.pair_to_row), pl.T,
                                         pl.kk, pl.H, out));
}

// Common preamble of the entry points that launch: plan, workspace, device.
moe_status_t prologue(const moe_problem_t* p, const void* ws, size_t ws_bytes, Plan* pl, int* num_sms) {
  moe_status_t st = make_plan(p, pl);
  if (st != MOE_OK) return st;
  st = check_ws(*pl, ws, ws_bytes);
  if (st != MOE_OK) return st;
  if (pl->T == 0) return MOE_OK;
  return device_sms(num_sms);
}

Launch launch_of(const moe_problem_t* p, moe_stream_t stream) {
  Launch l;
  l.stream = reinterpret_cast<cudaStream_t>(stream);
  l.pdl = (p->flags & MOE_FLAG_PDL) != 0;
  return l;
}

// Steps 2-5 (everything after the routing step) on routing already in the workspace; with
// `aligned` the align step has run too, with `permuted` also the permute step.
moe_status_t forward_after_route(const Plan& pl, const Launch& l, const void* hidden, const void* w13, const void* w2,
                                 const float* s13, const float* s2, void* out, void* ws, int num_sms,
                                 bool aligned = false, bool permuted = false) {
  moe_status_t st = aligned ? MOE_OK : run_align(pl, ws, l);
  if (st == MOE_OK && (pl.fp8 || pl.nv)) st = run_quant_act(pl, hidden, ws, l);
  if (st == MOE_OK && !permuted) st = run_permute(pl, hidden, ws, l, num_sms);
  if (st == MOE_OK) st = run_gemm1(pl, hidden, w13, s13, ws, l, num_sms, !permuted);
  if (st == MOE_OK) st = run_gemm2(pl, w2, s2, ws, l, num_sms);
  if (st == MOE_OK) st = run_combine(pl, out, ws, l);
  return st;
}

moe_status_t forward_device(const Plan& pl, const moe_problem_t* p, const void* hidden, const float* logits,
                            const void* w13, const void* w2, const float* s13, const float* s2, void* out,
                            void* ws, moe_stream_t stream, int num_sms) {
  const Launch l = launch_of(p, stream);
  // a small batch (one align chunk, at most 16 tokens): routing and align in one kernel, and
  // for bf16 row groups of at most kFusedPermutePairs pairs the permute too
  const bool fused = pl.T <= 8 * moe::kRouteAlignTokensPerWarp && pl.lay.num_chunks == 1;
  const bool bf16 = !(pl.fp8 || pl.pt || pl.mx || pl.nv);
  const bool permute = fused && bf16 && pl.bm == 16 && pl.P <= moe::kFusedPermutePairs;
  const moe_status_t st =
      fused ? run_route_align(pl, logits, ws, l, hidden, permute) : run_route(pl, logits, ws, l, hidden);
  if (st != MOE_OK) return st;
  return forward_after_route(pl, l, hidden, w13, w2, s13, s2, out, ws, num_sms, fused, permute);
}

// A weight-scale pointer as the problem's format wants it: fp32 (4-byte aligned) for the
// FP8 formats, NULL for bf16 (ignored) and for MXFP8 (its scales are in the prepared weights).
bool scale_ok(const Plan& pl, const float* s) {
  if (pl.mx) return s == nullptr;
  return !pl.q8 || aligned4(s);
}

moe_status_t check_weights(const Plan& pl, const void* w13, const void* w2, const float* s13, const float* s2) {
  if (!aligned16(w13) || !aligned16(w2)) return MOE_ERR_INVALID_ARG;
  if (!scale_ok(pl, s13) || !scale_ok(pl, s2)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

}  // namespace

MOE_API const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "MOE_ERR_WORKSPACE_TOO_SMALL";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT";
  }
  return "MOE_ERR_UNKNOWN";
}

MOE_API moe_status_t moe_check_problem(const moe_problem_t* problem) {
  Plan pl;
  return make_plan(problem, &pl);
}

MOE_API int32_t moe_padded_intermediate(int32_t intermediate, int32_t activation, int32_t wdtype) {
  if (intermediate <= 0 || intermediate > (1 << 20)) return -1;
  if (activation != MOE_ACT_SWIGLU && activation != MOE_ACT_RELU2 && activation != MOE_ACT_GELU_TANH &&
      activation != MOE_ACT_SWIGLUOAI)
    return -1;
  if (wdtype != MOE_DTYPE_BF16 && wdtype != MOE_DTYPE_FP8_BLOCK128 && wdtype != MOE_DTYPE_FP8_PER_TENSOR &&
      wdtype != MOE_DTYPE_MXFP8 && wdtype != MOE_DTYPE_NVFP4)
    return -1;
  const int a = wdtype == MOE_DTYPE_NVFP4 ? 256 : ((wdtype != MOE_DTYPE_BF16 || activation == MOE_ACT_RELU2) ? 128 : 16);
  return (intermediate + a - 1) / a * a;
}

MOE_API moe_status_t moe_workspace_layout(const moe_problem_t* problem, moe_workspace_layout_t* layout) {
  if (layout == nullptr) return MOE_ERR_INVALID_ARG;
  std::memset(layout, 0, sizeof(*layout));
  Plan pl;
  const moe_status_t st = make_plan(problem, &pl);
  if (st == MOE_OK) *layout = pl.lay;
  return st;
}

MOE_API size_t moe_workspace_size(const moe_problem_t* problem) {
  Plan pl;
  return make_plan(problem, &pl) == MOE_OK ? pl.lay.total_bytes : 0;
}

MOE_API moe_status_t moe_prepare_weights(const moe_problem_t* problem, int32_t intermediate_in, const void* w13_in,
                                         const void* w2_in, void* w13_out, void* w2_out, moe_stream_t stream) {
  Plan pl;
  moe_status_t st = make_plan(problem, &pl);  // num_tokens plays no part in weight preparation
  if (st != MOE_OK) return st;
  if (pl.mx || pl.nv) return MOE_ERR_INVALID_ARG;  // block-scaled weights: moe_prepare_weights_mxfp8 / _nvfp4
  if (moe_padded_intermediate(intermediate_in, pl.act, problem->wdtype) != pl.I) return MOE_ERR_INVALID_ARG;
  if (pl.q8 && intermediate_in != pl.I) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w13_in) || !aligned16(w13_out) || w2_in == nullptr || w2_out == nullptr)
    return MOE_ERR_INVALID_ARG;
  const int elt = pl.q8 ? 1 : 2;
  if ((reinterpret_cast<uintptr_t>(w2_in) | reinterpret_cast<uintptr_t>(w2_out)) & (elt - 1))
    return MOE_ERR_INVALID_ARG;
  int sms = 0;
  st = device_sms(&sms);
  if (st != MOE_OK) return st;
  const Launch l = launch_of(problem, stream);
  cudaError_t e;
  if (pl.pt || (pl.fp8 && pl.bm == 16)) {
    // e4m3 codes, tiled for the swapped-operand GEMMs
    e = moe::launch_tile_weights_u8(l, 0, w13_in, w13_out, pl.E, pl.H, pl.I, pl.gated);
    if (e == cudaSuccess) e = moe::launch_tile_weights_u8(l, 1, w2_in, w2_out, pl.E, pl.H, pl.I, pl.gated);
    return cuda_status(e);
  }
  if (pl.bm == 16) {
    // the swapped-operand GEMMs read the weights tiled
    e = moe::launch_tile_weights(l, 0, w13_in, w13_out, pl.E, pl.H, intermediate_in, pl.I, pl.gated);
    if (e == cudaSuccess) e = moe::launch_tile_weights(l, 1, w2_in, w2_out, pl.E, pl.H, intermediate_in, pl.I, pl.gated);
    return cuda_status(e);
  }
  e = moe::launch_prepare_w13(l, w13_in, w13_out, pl.E, intermediate_in, pl.I, pl.H, pl.gated, elt);
  if (e == cudaSuccess) e = moe::launch_prepare_w2(l, w2_in, w2_out, pl.E, pl.H, intermediate_in, pl.I, elt);
  return cuda_status(e);
}

MOE_API size_t moe_prepared_weights_bytes(const moe_problem_t* problem, int32_t which) {
  Plan pl;
  if (make_plan(problem, &pl) != MOE_OK || (which != 0 && which != 1)) return 0;
  if (pl.mx)
    return which == 0 ? moe::tiled_weight_bytes_u8(pl.E, pl.N1, pl.H) + moe::tiled_scale_bytes_mx(pl.E, pl.N1, pl.H)
                      : moe::tiled_weight_bytes_u8(pl.E, pl.H, pl.I) + moe::tiled_scale_bytes_mx(pl.E, pl.H, pl.I);
  if (pl.nv)
    return which == 0
               ? moe::tiled_weight_bytes_u8(pl.E, pl.N1, pl.H / 2) + moe::tiled_scale_bytes_nvfp4(pl.E, pl.N1, pl.H)
               : moe::tiled_weight_bytes_u8(pl.E, pl.H, pl.I / 2) + moe::tiled_scale_bytes_nvfp4(pl.E, pl.H, pl.I);
  if (pl.pt || (pl.fp8 && pl.bm == 16))
    return which == 0 ? moe::tiled_weight_bytes_u8(pl.E, pl.N1, pl.H) : moe::tiled_weight_bytes_u8(pl.E, pl.H, pl.I);
  if (pl.bm == 16)
    return which == 0 ? moe::tiled_weight_bytes(pl.E, pl.N1, pl.H) : moe::tiled_weight_bytes(pl.E, pl.H, pl.I);
  const size_t elt = pl.fp8 ? 1 : 2;
  return which == 0 ? static_cast<size_t>(pl.E) * pl.N1 * pl.H * elt : static_cast<size_t>(pl.E) * pl.H * pl.I * elt;
}

MOE_API moe_status_t moe_prepare_weights_mxfp8(const moe_problem_t* problem, const void* w13_codes,
                                               const void* w13_scales, const void* w2_codes, const void* w2_scales,
                                               void* w13_out, void* w2_out, moe_stream_t stream) {
  Plan pl;
  moe_status_t st = make_plan(problem, &pl);  // num_tokens plays no part in weight preparation
  if (st != MOE_OK) return st;
  if (!pl.mx) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w13_codes) || !aligned16(w2_codes) || !aligned16(w13_out) || !aligned16(w2_out) ||
      w13_scales == nullptr || w2_scales == nullptr)
    return MOE_ERR_INVALID_ARG;
  int sms = 0;
  st = device_sms(&sms);
  if (st != MOE_OK) return st;
  const Launch l = launch_of(problem, stream);
  uint8_t* o13 = static_cast<uint8_t*>(w13_out);
  uint8_t* o2 = static_cast<uint8_t*>(w2_out);
  cudaError_t e = moe::launch_tile_weights_u8(l, 0, w13_codes, o13, pl.E, pl.H, pl.I, pl.gated);
  if (e == cudaSuccess) e = moe::launch_tile_weights_u8(l, 1, w2_codes, o2, pl.E, pl.H, pl.I, pl.gated);
  if (e == cudaSuccess)
    e = moe::launch_tile_scales_mx(l, 0, w13_scales, o13 + moe::tiled_weight_bytes_u8(pl.E, pl.N1, pl.H), pl.E, pl.H,
                                   pl.I, pl.gated);
  if (e == cudaSuccess)
    e = moe::launch_tile_scales_mx(l, 1, w2_scales, o2 + moe::tiled_weight_bytes_u8(pl.E, pl.H, pl.I), pl.E, pl.H,
                                   pl.I, pl.gated);
  return cuda_status(e);
}

MOE_API moe_status_t moe_prepare_weights_nvfp4(const moe_problem_t* problem, const void* w13_codes,
                                               const void* w13_scales, const void* w2_codes, const void* w2_scales,
                                               void* w13_out, void* w2_out, moe_stream_t stream) {
  Plan pl;
  moe_status_t st = make_plan(problem, &pl);  // num_tokens plays no part in weight preparation
  if (st != MOE_OK) return st;
  if (!pl.nv) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w13_codes) || !aligned16(w2_codes) || !aligned16(w13_out) || !aligned16(w2_out) ||
      w13_scales == nullptr || w2_scales == nullptr)
    return MOE_ERR_INVALID_ARG;
  int sms = 0;
  st = device_sms(&sms);
  if (st != MOE_OK) return st;
  const Launch l = launch_of(problem, stream);
  uint8_t* o13 = static_cast<uint8_t*>(w13_out);
  uint8_t* o2 = static_cast<uint8_t*>(w2_out);
  cudaError_t e = moe::launch_tile_weights_u8(l, 0, w13_codes, o13, pl.E, pl.H, pl.I, pl.gated, 2);
  if (e == cudaSuccess) e = moe::launch_tile_weights_u8(l, 1, w2_codes, o2, pl.E, pl.H, pl.I, pl.gated, 2);
  if (e == cudaSuccess)
    e = moe::launch_tile_scales_nvfp4(l, 0, w13_scales, o13 + moe::tiled_weight_bytes_u8(pl.E, pl.N1, pl.H / 2), pl.E,
                                      pl.H, pl.I, pl.gated);
  if (e == cudaSuccess)
    e = moe::launch_tile_scales_nvfp4(l, 1, w2_scales, o2 + moe::tiled_weight_bytes_u8(pl.E, pl.H, pl.I / 2), pl.E,
                                      pl.H, pl.I, pl.gated);
  return cuda_status(e);
}

MOE_API moe_status_t moe_quantize_weights_nvfp4(const void* w, int64_t num_mats, int32_t rows, int32_t cols,
                                                void* codes, void* scales, float* global_scales, moe_stream_t stream) {
  if (num_mats < 0 || num_mats > 65535 || rows <= 0 || cols <= 0 || cols % 16 != 0) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(codes) || scales == nullptr || !aligned4(global_scales)) return MOE_ERR_INVALID_ARG;
  if (num_mats == 0) return MOE_OK;
  int sms = 0;
  moe_status_t st = device_sms(&sms);
  if (st != MOE_OK) return st;
  Launch l;
  l.stream = reinterpret_cast<cudaStream_t>(stream);
  l.pdl = false;
  return cuda_status(moe::launch_quant_weights_nvfp4(l, w, num_mats, static_cast<int64_t>(rows) * cols, codes, scales,
                                                     global_scales));
}

MOE_API moe_status_t moe_quantize_weights_mxfp8(const void* w, int64_t num_mats, int32_t rows, int32_t cols,
                                                void* codes, void* scales, moe_stream_t stream) {
  if (num_mats < 0 || rows <= 0 || cols <= 0 || cols % 32 != 0) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(codes) || scales == nullptr) return MOE_ERR_INVALID_ARG;
  if (num_mats == 0) return MOE_OK;
  int sms = 0;
  moe_status_t st = device_sms(&sms);
  if (st != MOE_OK) return st;
  Launch l;
  l.stream = reinterpret_cast<cudaStream_t>(stream);
  l.pdl = false;
  return cuda_status(moe::launch_quant_weights_mx(l, w, num_mats * rows, cols, codes, scales));
}

MOE_API moe_status_t moe_quantize_weights_fp8(const void* w, int64_t num_mats, int32_t rows, int32_t cols,
                                              void* codes, float* scales, moe_stream_t stream) {
  if (num_mats < 0 || rows <= 0 || cols <= 0 || rows % 128 != 0 || cols % 128 != 0) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(codes) || !aligned4(scales)) return MOE_ERR_INVALID_ARG;
  if (num_mats * static_cast<int64_t>(rows / 128) * (cols / 128) >= (1LL << 31)) return MOE_ERR_UNSUPPORTED;
  if (num_mats == 0) return MOE_OK;
  int sms = 0;
  const moe_status_t st = device_sms(&sms);
  if (st != MOE_OK) return st;
  Launch l;
  l.stream = reinterpret_cast<cudaStream_t>(stream);
  l.pdl = false;
  return cuda_status(moe::launch_quant_weights(l, w, num_mats, rows, cols, codes, scales));
}

MOE_API moe_status_t moe_quantize_weights_fp8_per_tensor(const void* w, int64_t num_mats, int32_t rows, int32_t cols,
                                                         void* codes, float* scales, moe_stream_t stream) {
  if (num_mats < 0 || num_mats > 65535 || rows <= 0 || cols <= 0) return MOE_ERR_INVALID_ARG;
  const int64_t elems = static_cast<int64_t>(rows) * cols;
  if (elems % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(codes) || !aligned4(scales)) return MOE_ERR_INVALID_ARG;
  if (num_mats == 0) return MOE_OK;
  int sms = 0;
  const moe_status_t st = device_sms(&sms);
  if (st != MOE_OK) return st;
  Launch l;
  l.stream = reinterpret_cast<cudaStream_t>(stream);
  l.pdl = false;
  return cuda_status(moe::launch_quant_weights_per_tensor(l, w, num_mats, elems, codes, scales));
}

MOE_API moe_status_t moe_forward(const moe_problem_t* problem, const void* hidden, const float* router_logits,
                                 const void* w13, const void* w2, const float* w13_scale, const float* w2_scale,
                                 void* out, void* workspace, size_t workspace_bytes, moe_stream_t stream) {
  Plan pl;
  int sms = 0;
  moe_status_t st = make_plan(problem, &pl);
  if (st != MOE_OK || pl.T == 0) return st;  // T == 0: nothing to do, pointers unused
  if (!aligned16(hidden) || !aligned16(router_logits) || !aligned16(out) || hidden == out)
    return MOE_ERR_INVALID_ARG;
  st = check_weights(pl, w13, w2, w13_scale, w2_scale);
  if (st != MOE_OK) return st;
  st = prologue(problem, workspace, workspace_bytes, &pl, &sms);
  if (st != MOE_OK || pl.T == 0) return st;
  return forward_device(pl, problem, hidden, router_logits, w13, w2, w13_scale, w2_scale, out, workspace, stream,
                        sms);
}

MOE_API moe_status_t moe_forward_routed(const moe_problem_t* problem, const void* hidden, const int32_t* topk_ids,
                                        const float* topk_weights, const void* w13, const void* w2,
                                        const float* w13_scale, const float* w2_scale, void* out, void* workspace,
                                        size_t workspace_bytes, moe_stream_t stream) {
  Plan pl;
  int sms = 0;
  moe_status_t st = make_plan(problem, &pl);
  if (st != MOE_OK || pl.T == 0) return st;  // T == 0: nothing to do, pointers unused
  if (!aligned16(hidden) || !aligned4(topk_ids) || !aligned4(topk_weights) || !aligned16(out) || hidden == out)
    return MOE_ERR_INVALID_ARG;
  st = check_weights(pl, w13, w2, w13_scale, w2_scale);
  if (st != MOE_OK) return st;
  st = prologue(problem, workspace, workspace_bytes, &pl, &sms);
  if (st != MOE_OK || pl.T == 0) return st;
  const Launch l = launch_of(problem, stream);
  const auto& L = pl.lay;
  // the status word and work counters start at zero, as after the routing kernel
  if (cudaMemsetAsync(ws_ptr<int>(workspace, L.status), 0, 16 * sizeof(int), l.stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  st = cuda_status(moe::launch_load_routing(l, topk_ids, topk_weights, pl.T, pl.Er, pl.topk, pl.Es,
                                            ws_ptr<int>(workspace, L.topk_ids), ws_ptr<float>(workspace, L.topk_w),
                                            ws_ptr<int>(workspace, L.status)));
  if (st != MOE_OK) return st;
  return forward_after_route(pl, l, hidden, w13, w2, w13_scale, w2_scale, out, workspace, sms);
}

MOE_API moe_status_t moe_forward_host(const moe_problem_t* problem, const void* h_hidden,
                                      const float* h_router_logits, const void* w13, const void* w2,
                                      const float* w13_scale, const float* w2_scale, void* h_out, void* workspace,
                                      size_t workspace_bytes, moe_stream_t stream) {
  Plan pl;
  int sms = 0;
  moe_status_t st = make_plan(problem, &pl);
  if (st != MOE_OK || pl.T == 0) return st;  // T == 0: nothing to do, pointers unused
  if (h_hidden == nullptr || h_router_logits == nullptr || h_out == nullptr) return MOE_ERR_INVALID_ARG;
  st = check_weights(pl, w13, w2, w13_scale, w2_scale);
  if (st != MOE_OK) return st;
  st = prologue(problem, workspace, workspace_bytes, &pl, &sms);
  if (st != MOE_OK || pl.T == 0) return st;
  const auto& L = pl.lay;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  void* d_hidden = ws_ptr<void>(workspace, L.io_hidden);
  float* d_logits = ws_ptr<float>(workspace, L.io_logits);
  void* d_out = ws_ptr<void>(workspace, L.io_out);
  const size_t hbytes = static_cast<size_t>(pl.T) * pl.H * 2;
  if (cudaMemcpyAsync(d_hidden, h_hidden, hbytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(d_logits, h_router_logits, static_cast<size_t>(pl.T) * pl.Er * 4, cudaMemcpyHostToDevice,
                      s) != cudaSuccess)
    return MOE_ERR_CUDA;
  st = forward_device(pl, problem, d_hidden, d_logits, w13, w2, w13_scale, w2_scale, d_out, workspace, stream, sms);
  if (st != MOE_OK) return st;
  if (cudaMemcpyAsync(h_out, d_out, hbytes, cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ERR_CUDA;
  return cudaStreamSynchronize(s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

MOE_API moe_status_t moe_stage_route(const moe_problem_t* problem, const float* router_logits, void* workspace,
                                     size_t workspace_bytes, moe_stream_t stream) {
  Plan pl;
  int sms = 0;
  moe_status_t st = make_plan(problem, &pl);
  if (st != MOE_OK || pl.T == 0) return st;  // T == 0: nothing to do, pointers unused
  if (!aligned16(router_logits)) return MOE_ERR_INVALID_ARG;
  st = prologue(problem, workspace, workspace_bytes, &pl, &sms);
  if (st != MOE_OK || pl.T == 0) return st;
  return run_route(pl, router_logits, workspace, launch_of(problem, stream), nullptr);
}

MOE_API moe_status_t moe_stage_align(const moe_problem_t* problem, void* workspace, size_t workspace_bytes,
                                     moe_stream_t stream) {
  Plan pl;
  int sms = 0;
  moe_status_t st = prologue(problem, workspace, workspace_bytes, &pl, &sms);
  if (st != MOE_OK || pl.T == 0) return st;
  return run_align(pl, workspace, launch_of(problem, stream));
}

MOE_API moe_status_t moe_stage_quant_act(const moe_problem_t* problem, const void* hidden, void* workspace,
                                         size_t workspace_bytes, moe_stream_t stream) {
  Plan pl;
  int sms = 0;
  moe_status_t st = make_plan(problem, &pl);
  if (st != MOE_OK || pl.T == 0) return st;  // T == 0: nothing to do, pointers unused
  if (!(pl.fp8 || pl.nv) || !aligned16(hidden)) return MOE_ERR_INVALID_ARG;
  st = prologue(problem, workspace, workspace_bytes, &pl, &sms);
  if (st != MOE_OK || pl.T == 0) return st;
  return run_quant_act(pl, hidden, workspace, launch_of(problem, stream));
}

MOE_API moe_status_t moe_stage_permute(const moe_problem_t* problem, const void* hidden, void* workspace,
                                       size_t workspace_bytes, moe_stream_t stream) {
  Plan pl;
  int sms = 0;
  moe_status_t st = make_plan(problem, &pl);
  if (st != MOE_OK || pl.T == 0) return st;  // T == 0: nothing to do, pointers unused
  if (pl.bm == 16 && !aligned16(hidden)) return MOE_ERR_INVALID_ARG;
  st = prologue(problem, workspace, workspace_bytes, &pl, &sms);
  if (st != MOE_OK || pl.T == 0) return st;
  return run_permute(pl, hidden, workspace, launch_of(problem, stream), sms);
}

MOE_API moe_status_t moe_stage_gemm1(const moe_problem_t* problem, const void* hidden, const void* w13,
                                     const float* w13_scale, void* workspace, size_t workspace_bytes,
                                     moe_stream_t stream) {
  Plan pl;
  int sms = 0;
  moe_status_t st = make_plan(problem, &pl);
  if (st != MOE_OK || pl.T == 0) return st;  // T == 0: nothing to do, pointers unused
  if (!aligned16(hidden) || !aligned16(w13) || !scale_ok(pl, w13_scale)) return MOE_ERR_INVALID_ARG;
  st = prologue(problem, workspace, workspace_bytes, &pl, &sms);
  if (st != MOE_OK || pl.T == 0) return st;
  return run_gemm1(pl, hidden, w13, w13_scale, workspace, launch_of(problem, stream), sms);
}

MOE_API moe_status_t moe_stage_gemm2(const moe_problem_t* problem, const void* w2, const float* w2_scale,
                                     void* workspace, size_t workspace_bytes, moe_stream_t stream) {
  Plan pl;
  int sms = 0;
  moe_status_t st = make_plan(problem, &pl);
  if (st != MOE_OK || pl.T == 0) return st;  // T == 0: nothing to do, pointers unused
  if (!aligned16(w2) || !scale_ok(pl, w2_scale)) return MOE_ERR_INVALID_ARG;
  st = prologue(problem, workspace, workspace_bytes, &pl, &sms);
  if (st != MOE_OK || pl.T == 0) return st;
  return run_gemm2(pl, w2, w2_scale, workspace, launch_of(problem, stream), sms);
}

MOE_API moe_status_t moe_stage_combine(const moe_problem_t* problem, void* out, void* workspace,
                                       size_t workspace_bytes, moe_stream_t stream) {
  Plan pl;
  int sms = 0;
  moe_status_t st = make_plan(problem, &pl);
  if (st != MOE_OK || pl.T == 0) return st;  // T == 0: nothing to do, pointers unused
  if (!aligned16(out)) return MOE_ERR_INVALID_ARG;
  st = prologue(problem, workspace, workspace_bytes, &pl, &sms);
  if (st != MOE_OK || pl.T == 0) return st;
  return run_combine(pl, out, workspace, launch_of(problem, stream));
}

// ---- expert parallelism ----------------------------------------------------------

namespace {

// Workspace of the dispatch sort: this rank's pairs keyed by owner rank (the align kernels
// with `world` keys and 16-row padding per key).
struct EpLayout {
  size_t owner, sorted, block_expert, num_blocks, chunk_hist, total;
  long long max_rows;
  int num_chunks;
};

moe_status_t ep_plan(const moe_problem_t* p, int32_t world, Plan* pl, EpLayout* o) {
  moe_status_t st = make_plan(p, pl);
  if (st != MOE_OK) return st;
  if (world < 1 || world > moe::kMaxExperts || pl->Er % world != 0) return MOE_ERR_INVALID_ARG;
  const long long P = pl->P;
  const long long active = P < world ? P : world;
  o->max_rows = static_cast<long long>(align_up(static_cast<size_t>(P + active * 15), 16));
  o->num_chunks = static_cast<int>(P == 0 ? 1 : (P + moe::kAlignChunk - 1) / moe::kAlignChunk);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, kAlign);
    return at;
  };
  o->owner = take(static_cast<size_t>(P) * 4);
  o->sorted = take(static_cast<size_t>(o->max_rows) * 4);
  o->block_expert = take(static_cast<size_t>(o->max_rows) / 16 * 4 + 4);
  o->num_blocks = take(256);
  o->chunk_hist = take(static_cast<size_t>(o->num_chunks) * world * 4);
  o->total = off;
  return MOE_OK;
}

}  // namespace

MOE_API size_t moe_ep_workspace_size(const moe_problem_t* problem, int32_t world) {
  Plan pl;
  EpLayout el;
  return ep_plan(problem, world, &pl, &el) == MOE_OK ? el.total : 0;
}

MOE_API int64_t moe_ep_max_send_rows(const moe_problem_t* problem, int32_t world) {
  Plan pl;
  EpLayout el;
  return ep_plan(problem, world, &pl, &el) == MOE_OK ? el.max_rows : -1;
}

MOE_API moe_status_t moe_ep_dispatch(const moe_problem_t* problem, int32_t world, int32_t rank, const void* hidden,
                                     const int32_t* topk_ids, const float* topk_weights, void* send_rows,
                                     int32_t* send_expert, float* send_weight, int32_t* send_offsets,
                                     int32_t* pair_to_send_row, void* workspace, size_t workspace_bytes,
                                     moe_stream_t stream) {
  Plan pl;
  EpLayout el;
  moe_status_t st = ep_plan(problem, world, &pl, &el);
  if (st != MOE_OK) return st;
  if (rank < 0 || rank >= world) return MOE_ERR_INVALID_ARG;
  if (!aligned4(send_offsets)) return MOE_ERR_INVALID_ARG;
  if (pl.T == 0) {  // nothing to send: the offsets are all zero
    return cuda_status(cudaMemsetAsync(send_offsets, 0, (static_cast<size_t>(world) + 1) * 4,
                                       reinterpret_cast<cudaStream_t>(stream)));
  }
  if (!aligned16(hidden) || !aligned4(topk_ids) || !aligned4(topk_weights) || !aligned16(send_rows) ||
      !aligned4(send_expert) || !aligned4(send_weight) || !aligned4(pair_to_send_row))
    return MOE_ERR_INVALID_ARG;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MOE_ERR_INVALID_ARG;
  if (workspace_bytes < el.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  int sms = 0;
  st = device_sms(&sms);
  if (st != MOE_OK) return st;
  const Launch l = launch_of(problem, stream);
  const int per_rank = pl.Er / world;
  int* owner = ws_ptr<int>(workspace, el.owner);
  int* sorted = ws_ptr<int>(workspace, el.sorted);
  cudaError_t e = moe::launch_ep_owner(l, topk_ids, pl.P, pl.Er, per_rank, rank, owner);
  if (e == cudaSuccess)
    e = moe::launch_align(l, owner, static_cast<int>(pl.P), world, 16, el.num_chunks, ws_ptr<int>(workspace, el.chunk_hist),
                          sorted, send_offsets, ws_ptr<int>(workspace, el.block_expert), pair_to_send_row,
                          ws_ptr<int>(workspace, el.num_blocks), 0, nullptr);
  if (e == cudaSuccess)
    e = moe::launch_ep_pack(l, hidden, pl.H, sorted, send_offsets, world, static_cast<int>(pl.P), pl.kk, topk_ids,
                            topk_weights, pl.Er, per_rank, el.max_rows, send_rows, send_expert, send_weight, sms);
  return cuda_status(e);
}

MOE_API moe_status_t moe_ep_combine(const moe_problem_t* problem, int32_t world, const void* returned_rows,
                                    const int32_t* pair_to_send_row, void* out, moe_stream_t stream) {
  Plan pl;
  EpLayout el;
  moe_status_t st = ep_plan(problem, world, &pl, &el);
  if (st != MOE_OK || pl.T == 0) return st;
  if (!aligned16(returned_rows) || !aligned4(pair_to_send_row) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  int sms = 0;
  st = device_sms(&sms);
  if (st != MOE_OK) return st;
  return cuda_status(
      moe::launch_ep_combine(launch_of(problem, stream), returned_rows, pair_to_send_row, pl.T, pl.kk, pl.H, out));
}

MOE_API moe_status_t moe_get_device_status(void* workspace, moe_stream_t stream, int32_t* detail) {
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MOE_ERR_INVALID_ARG;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int32_t word = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (word != 0 && cudaMemset(workspace, 0, sizeof(word)) != cudaSuccess) return MOE_ERR_CUDA;
  if (detail != nullptr) *detail = word;
  if (word == 0) return MOE_OK;
  return (word & moe::kStatusBadRouting) ? MOE_ERR_INVALID_ARG : MOE_ERR_DEVICE_TIMEOUT;
}
