// Device-side building blocks for the sm_100a MoE kernels: mbarriers with bounded
// waits, TMA tile / gather4 loads, tcgen05 (UMMA) descriptors, MMA, commit and TMEM
// loads, written as inline PTX.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Device status word values (workspace "status"). Bits 0-15: the wait site.
constexpr int kStatusTimeout = 0x10000;

// Bounded waits give up after this long (the longest legitimate wait inside one of
// these kernels is well under a millisecond).
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---- programmatic dependent launch -------------------------------------------------
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- mbarrier ------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
          bar),
      "r"(bytes)
      : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase of parity `parity` of barrier `bar` to complete. Gives up when
// another thread of the CTA has raised `*abort` or after `limit_ns`; a timeout raises
// `*abort` and records `kStatusTimeout | site` in the device status word. Returns true
// when the phase completed.
static __device__ __noinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort,
                                                      int* status, int site, unsigned long long limit_ns) {
  const unsigned long long t0 = globaltimer_ns();
  for (uint32_t i = 0;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 31u) == 31u) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        *abort = 1;
        atomicCAS(status, 0, kStatusTimeout | site);
        return false;
      }
    }
  }
}
static __device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, volatile int* abort,
                                                   int* status, int site) {
  return mbar_wait_bounded(bar, parity, abort, status, site, kWaitTimeoutNs);
}
// The common case stays inline: one try_wait (which suspends the thread in hardware for a
// while when the phase is not complete), then the bounded loop. Retrying inline measured
// slower on the prefill forward (475 vs 459 us).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          int* status, int site) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, abort, status, site);
}
// Bounded wait that ignores the abort flag (used to drain in-flight copies on exit).
static __device__ __noinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity) {
  const unsigned long long t0 = globaltimer_ns();
  for (uint32_t i = 0;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 31u) == 31u && globaltimer_ns() - t0 > kWaitTimeoutNs) return false;
  }
}

// Before a producer thread leaves (normally or after an abort): wait, bounded, until the
// copies it issued into a ring of `stages` full barriers (one arrival each, from this
// thread only, stage s at full0 + 8 s) have landed, so that no copy writes shared memory
// after the CTA exits. `fills` counts the stages this thread filled, in order from
// stage 0; fill i used stage i % stages with phase parity (i / stages) & 1. On the
// normal path every fill was consumed long ago and each wait returns at once.
__device__ __forceinline__ void drain_fills(uint32_t full0, uint32_t stages, uint32_t fills) {
  const uint32_t first = fills > stages ? fills - stages : 0u;
  for (uint32_t i = first; i < fills; ++i) mbar_wait_drain(full0 + 8 * (i % stages), (i / stages) & 1u);
}

// ---- TMA -----------------------------------------------------------------------------
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
// 2-D tiled load of the tensor map's box at (c0 = innermost, c1) into shared memory.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}
// Gather four rows r0..r3 (box one row high, c0 innermost) into four consecutive box
// rows of shared memory.
__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int r0, int r1, int r2, int r3,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4, %5, %6, %7}], [%2], %8;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(r0), "r"(r1), "r"(r2),
      "r"(r3), "l"(policy)
      : "memory");
}
// 16-byte asynchronous global -> shared copy (L2 only, bypassing L1).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
// Arrive on `bar` once all cp.async copies issued so far by this thread have landed; the
// arrival counts against the barrier's expected count (.noinc).
__device__ __forceinline__ void cp_async_mbar_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}
// 2-D tiled store of a shared-memory box to the tensor map at (c0 = innermost, c1), as
// part of this thread's current bulk async-group.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until at most N of this thread's bulk groups are incomplete.
template <int N>
__device__ __forceinline__ void bulk_wait_group() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}
// Make this thread's generic-proxy shared-memory writes visible to the async proxy (TMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Prefetch `bytes` (multiple of 16) at a 16-byte aligned global address into L2.
__device__ __forceinline__ void prefetch_l2_bulk(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ---- tcgen05 / TMEM ------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor of a K-major operand tile stored with the 128-byte
// swizzle: rows of 128 bytes, groups of 8 rows 1024 bytes apart (stride byte offset),
// tile base 1024-byte aligned. The leading byte offset is unused for this layout.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);  // start address      [0,14)
  d |= static_cast<uint64_t>(1) << 16;                   // leading byte off.  [16,30)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;           // stride byte off.   [32,46)
  d |= static_cast<uint64_t>(1) << 46;                   // descriptor version [46,48)
  d |= static_cast<uint64_t>(2) << 61;                   // 128-byte swizzle   [61,64)
  return d;
}

// Instruction descriptor for kind::f16 with bf16 A/B, fp32 D, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4)                                   // D format: f32
         | (1u << 7)                                 // A format: bf16
         | (1u << 10)                                // B format: bf16
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}
// Instruction descriptor for kind::f8f6f4 with e4m3 A/B, fp32 D, both K-major.
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N) {
  return (1u << 4)                                   // D format: f32
         | (0u << 7)                                 // A format: e4m3
         | (0u << 10)                                // B format: e4m3
         | (static_cast<uint32_t>(N >> 3) << 17)
         | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_e4m3(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// The two 32-bit halves of umma_desc_sw128: the low word carries the start address (and
// the unused leading byte offset), the high word is the same for every tile.
__device__ __forceinline__ uint32_t umma_desc_lo(uint32_t saddr) { return ((saddr & 0x3FFFFu) >> 4) | (1u << 16); }
constexpr uint32_t kUmmaDescHi = (1024u >> 4) | (1u << (46 - 32)) | (2u << (61 - 32));

// One 128-byte K chunk of operands: four MMAs (kind::f16: bf16, K=16; kind::f8f6f4:
// e4m3, K=32), each step advancing both
// descriptors by 32 bytes (+2 in the encoded start address). The first MMA accumulates
// into D when `accumulate` is nonzero, the other three always do. The descriptors are
// assembled inside the asm block from their low words, so the issuing thread spends a few
// integer adds per MMA: a single thread's instruction stream between MMAs limits how fast
// they can be issued.
__device__ __forceinline__ void umma_bf16_chunk(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t idesc,
                                                uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t.reg .b32 al, bl;\n\t.reg .b64 a, b;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 q, %4, %4;\n\t"
      "mov.b64 a, {%1, %5};\n\tmov.b64 b, {%2, %5};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, p;\n\t"
      "add.u32 al, %1, 2;\n\tadd.u32 bl, %2, 2;\n\tmov.b64 a, {al, %5};\n\tmov.b64 b, {bl, %5};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, q;\n\t"
      "add.u32 al, %1, 4;\n\tadd.u32 bl, %2, 4;\n\tmov.b64 a, {al, %5};\n\tmov.b64 b, {bl, %5};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, q;\n\t"
      "add.u32 al, %1, 6;\n\tadd.u32 bl, %2, 6;\n\tmov.b64 a, {al, %5};\n\tmov.b64 b, {bl, %5};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, q;\n\t}" ::"r"(d_tmem),
      "r"(a_lo), "r"(b_lo), "r"(idesc), "r"(accumulate), "n"(kUmmaDescHi)
      : "memory");
}

__device__ __forceinline__ void umma_e4m3_chunk(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t idesc,
                                                uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t.reg .b32 al, bl;\n\t.reg .b64 a, b;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 q, %4, %4;\n\t"
      "mov.b64 a, {%1, %5};\n\tmov.b64 b, {%2, %5};\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a, b, %3, p;\n\t"
      "add.u32 al, %1, 2;\n\tadd.u32 bl, %2, 2;\n\tmov.b64 a, {al, %5};\n\tmov.b64 b, {bl, %5};\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a, b, %3, q;\n\t"
      "add.u32 al, %1, 4;\n\tadd.u32 bl, %2, 4;\n\tmov.b64 a, {al, %5};\n\tmov.b64 b, {bl, %5};\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a, b, %3, q;\n\t"
      "add.u32 al, %1, 6;\n\tadd.u32 bl, %2, 6;\n\tmov.b64 a, {al, %5};\n\tmov.b64 b, {bl, %5};\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a, b, %3, q;\n\t}" ::"r"(d_tmem),
      "r"(a_lo), "r"(b_lo), "r"(idesc), "r"(accumulate), "n"(kUmmaDescHi)
      : "memory");
}

// Arrive once on `bar` when all previously issued tcgen05 operations of this thread
// have completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// Load 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
// Load 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---- small helpers -------------------------------------------------------------------
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// silu(g) = g / (1 + e^-g). The result is rounded to bf16 right after, so the fast
// division (__fdividef, which returns 0 once the divisor exceeds 2^126, the right limit
// for very negative g) costs no visible accuracy.
__device__ __forceinline__ float silu_f32(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// gelu_tanh(g) = 0.5 g (1 + tanh(sqrt(2/pi) (g + 0.044715 g^3))), with CUDA's tanhf.
__device__ __forceinline__ float gelu_tanh_f32(float g) {
  return 0.5f * g * (1.0f + tanhf(0.7978845608028654f * (g + 0.044715f * g * g * g)));
}

// Gate activation of a gated layer: act 0 = SwiGLU (silu), 2 = gelu_tanh.
__device__ __forceinline__ float gate_act(float g, int act) { return act == 2 ? gelu_tanh_f32(g) : silu_f32(g); }

// The SwiGLU variant published with OpenAI's gpt-oss models (alpha 1.702, limit 7): the gate
// clamped from above and the up value to [-7, 7], then g sigmoid(1.702 g) (u + 1). The
// division is the fast one, as in silu_f32 (a very negative g gives 0).
__device__ __forceinline__ float swigluoai_f32(float g, float u) {
  const float gc = fminf(g, 7.0f);
  const float uc = fminf(fmaxf(u, -7.0f), 7.0f);
  return __fdividef(gc, 1.0f + __expf(-1.702f * gc)) * (uc + 1.0f);
}

// Activation of a gated layer from its gate and up values: act 0 = SwiGLU, 2 = gelu_tanh
// (act(gate) * up), 3 = swigluoai.
__device__ __forceinline__ float gated_act(float g, float u, int act) {
  return act == 3 ? swigluoai_f32(g, u) : gate_act(g, act) * u;
}

// ---- MXFP8 (OCP Microscaling v1.0: E4M3 values, one E8M0 power-of-two scale per 32) ----

// Shared exponent of a block whose largest magnitude is amax: floor(log2(amax)) - 8 (8 is
// the exponent of E4M3's largest power of two), clamped to [-127, 127]; -127 for an
// all-zero block. The scale byte is the exponent + 127.
__device__ __forceinline__ int mx_exponent(float amax) {
  if (!(amax > 0.f)) return -127;
  return max(-127, min(127, ilogbf(amax) - 8));
}
// 2^-e as an fp32 (e in [-127, 119] for finite bf16 or fp32 inputs: always a normal number),
// so that x * mx_inv(e) is exact unless the product falls below the normal range.
__device__ __forceinline__ float mx_inv(int e) { return __int_as_float((127 - min(e, 126)) << 23); }
// Four values scaled by inv, to E4M3 (round to nearest even, saturating), packed low first.
__device__ __forceinline__ uint32_t mx_e4m3x4(float a, float b, float c, float d, float inv) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a * inv, b * inv), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c * inv, d * inv), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

// Instruction descriptor for kind::mxf8f6f4.block_scale with e4m3 A/B (both K-major), fp32
// D and E8M0 scales. The scale-factor byte of A (bits 29-30) and B (bits 4-5) selects which
// byte of the scale columns this MMA reads: the K block within a 128-element chunk.
__host__ __device__ constexpr uint32_t idesc_mx(int M, int N) {
  return (0u << 7)                                   // A format: e4m3
         | (0u << 10)                                // B format: e4m3
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (1u << 23)                                // scale format: E8M0
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

// Shared-memory descriptor of a 32-row x 16-byte block (no swizzle, K-major, rows 16
// bytes apart: core matrices of 8 rows 128 bytes apart) for tcgen05.cp.
__device__ __forceinline__ uint64_t sf_block_desc(uint32_t saddr) {
  uint64_t d = static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(128 >> 4) << 16;  // leading byte offset (one core matrix wide: unused)
  d |= static_cast<uint64_t>(128 >> 4) << 32;  // stride byte offset: next 8 rows
  d |= static_cast<uint64_t>(1) << 46;         // descriptor version
  return d;
}

// Copy a 32 x 16-byte block of scale bytes to TMEM columns [col, col + 4) of lanes 0-31,
// replicated to the four lane quadrants: byte 16 l + 4 j + k lands in lane l (+ 32 q),
// column col + j, byte k. With row r's scales at l = r % 32, j = r / 32 and byte k = its
// K block, this is where a block-scaled MMA of M (or N) <= 128 rows reads them.
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint32_t saddr) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sf_block_desc(saddr))
               : "memory");
}

// One 128-byte K chunk of e4m3 operands with block scales: four MMAs of K = 32; MMA k reads
// scale byte k of the A columns at sfa and the B columns at sfb. The first accumulates into
// D when `accumulate` is nonzero, the others always do.
__device__ __forceinline__ void umma_mx_chunk(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t idesc,
                                              uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t.reg .b32 al, bl, id;\n\t.reg .b64 a, b;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 q, %4, %4;\n\t"
      "mov.b64 a, {%1, %5};\n\tmov.b64 b, {%2, %5};\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], a, b, %3, [%6], [%7], p;\n\t"
      "add.u32 al, %1, 2;\n\tadd.u32 bl, %2, 2;\n\tmov.b64 a, {al, %5};\n\tmov.b64 b, {bl, %5};\n\t"
      "or.b32 id, %3, 0x20000010;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], a, b, id, [%6], [%7], q;\n\t"
      "add.u32 al, %1, 4;\n\tadd.u32 bl, %2, 4;\n\tmov.b64 a, {al, %5};\n\tmov.b64 b, {bl, %5};\n\t"
      "or.b32 id, %3, 0x40000020;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], a, b, id, [%6], [%7], q;\n\t"
      "add.u32 al, %1, 6;\n\tadd.u32 bl, %2, 6;\n\tmov.b64 a, {al, %5};\n\tmov.b64 b, {bl, %5};\n\t"
      "or.b32 id, %3, 0x60000030;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], a, b, id, [%6], [%7], q;\n\t}" ::"r"(d_tmem),
      "r"(a_lo), "r"(b_lo), "r"(idesc), "r"(accumulate), "n"(kUmmaDescHi), "r"(sfa), "r"(sfb)
      : "memory");
}

// ---- NVFP4 (E2M1 values, one E4M3 scale per 16 values, one fp32 scale per tensor) ----

// Per-tensor decode scale from the tensor's largest magnitude: amax / (6 * 448), so that
// every block scale fits E4M3 (IEEE division); 1 for an all-zero tensor.
__device__ __forceinline__ float nvfp4_tensor_scale(float amax) { return amax == 0.f ? 1.f : __fdiv_rn(amax, 2688.f); }
// E4M3 code of the block scale of 16 values with largest magnitude amax under the tensor
// scale g: e4m3(amax / 6 / g), two IEEE divisions, round to nearest even, saturating.
__device__ __forceinline__ uint8_t nvfp4_block_scale(float amax, float g) {
  return __nv_cvt_float_to_fp8(__fdiv_rn(__fdiv_rn(amax, 6.0f), g), __NV_SATFINITE, __NV_E4M3);
}
__device__ __forceinline__ float e4m3_value(uint8_t code) {
  return __half2float(__half(__nv_cvt_fp8_to_halfraw(code, __NV_E4M3)));
}
// Two values a, b (K order) divided by d (IEEE) to E2M1, round to nearest even, saturating,
// packed into one byte with a in the low nibble; both 0 when d is not positive.
__device__ __forceinline__ uint32_t nvfp4_pair(float a, float b, float d) {
  if (!(d > 0.f)) return 0u;
  return __nv_cvt_float2_to_fp4x2(make_float2(__fdiv_rn(a, d), __fdiv_rn(b, d)), __NV_E2M1, cudaRoundNearest);
}
// Sixteen values (one block) to NVFP4 under tensor scale g: the block's E4M3 scale code and
// its eight code bytes packed as two words (value 2i in the low nibble of byte i).
__device__ __forceinline__ uint8_t nvfp4_block(const float (&v)[16], float g, uint2& packed) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint8_t s = nvfp4_block_scale(amax, g);
  const float d = e4m3_value(s) * g;
  uint32_t w[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 8; ++i) w[i >> 2] |= nvfp4_pair(v[2 * i], v[2 * i + 1], d) << (8 * (i & 3));
  packed = make_uint2(w[0], w[1]);
  return s;
}

// Instruction descriptor for kind::mxf4nvf4.block_scale with E2M1 A/B (both K-major), fp32
// D and UE4M3 scales (one per 16 values, scale_vec::4X: the scale-factor byte selectors are
// 0, each MMA reads all four bytes of its scale columns).
__host__ __device__ constexpr uint32_t idesc_nvf4(int M, int N) {
  return (1u << 7)                                   // A format: E2M1
         | (1u << 10)                                // B format: E2M1
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16; bit 23 clear: UE4M3 scales
}

// One 128-byte K chunk of packed E2M1 operands (256 values): four MMAs of K = 64, MMA m
// reading the four scale columns sfa + 4 m (A) and sfb + 4 m (B). The first accumulates
// into D when `accumulate` is nonzero, the others always do.
__device__ __forceinline__ void umma_nvf4_chunk(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t idesc,
                                                uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t.reg .b32 al, bl, sa, sb;\n\t.reg .b64 a, b;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 q, %4, %4;\n\t"
      "mov.b64 a, {%1, %5};\n\tmov.b64 b, {%2, %5};\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], a, b, %3, [%6], [%7], p;\n\t"
      "add.u32 al, %1, 2;\n\tadd.u32 bl, %2, 2;\n\tmov.b64 a, {al, %5};\n\tmov.b64 b, {bl, %5};\n\t"
      "add.u32 sa, %6, 4;\n\tadd.u32 sb, %7, 4;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], a, b, %3, [sa], [sb], q;\n\t"
      "add.u32 al, %1, 4;\n\tadd.u32 bl, %2, 4;\n\tmov.b64 a, {al, %5};\n\tmov.b64 b, {bl, %5};\n\t"
      "add.u32 sa, %6, 8;\n\tadd.u32 sb, %7, 8;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], a, b, %3, [sa], [sb], q;\n\t"
      "add.u32 al, %1, 6;\n\tadd.u32 bl, %2, 6;\n\tmov.b64 a, {al, %5};\n\tmov.b64 b, {bl, %5};\n\t"
      "add.u32 sa, %6, 12;\n\tadd.u32 sb, %7, 12;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], a, b, %3, [sa], [sb], q;\n\t}" ::"r"(d_tmem),
      "r"(a_lo), "r"(b_lo), "r"(idesc), "r"(accumulate), "n"(kUmmaDescHi), "r"(sfa), "r"(sfb)
      : "memory");
}

}  // namespace moe
