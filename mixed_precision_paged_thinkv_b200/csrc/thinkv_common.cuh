// thinkv_common.cuh -- shared device helpers of libthinkv (sm_100a).
//
// Layout arithmetic for the page-head blocks declared in include/thinkv.h,
// the sticky status word, and thin wrappers over the PTX this library uses:
// mbarrier + cp.async.bulk (the TMA bulk-copy engine) and mma.sync m16n8k16.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "thinkv.h"

namespace thinkv {

constexpr int kPage = 16;

// ---------------------------------------------------------------------------
// geometry
// ---------------------------------------------------------------------------
__host__ __device__ inline int64_t page_head_bytes(int d, int G, int b) {
  // K codes + V codes (2*d*b each) + K/V params (64 bytes per group each)
  if (b == 16) return 64LL * d;
  return 4LL * d * b + 128LL * (d / G);
}

// Code regions of a page-head block hold 32 lanes x lane_bytes bytes; the
// lanes' portions are interleaved in chunks of min(16, lane_bytes) bytes, so
// that 32 lanes reading the same chunk read one contiguous span of shared
// memory (no bank conflicts).  Offset of byte o of lane l's portion:
__host__ __device__ inline int chunk_bytes(int lane_bytes) { return lane_bytes < 16 ? lane_bytes : 16; }
__host__ __device__ inline int lane_off(int lane, int o, int lane_bytes) {
  const int u = chunk_bytes(lane_bytes);
  return (o / u) * 32 * u + lane * u + (o % u);
}

// Table entry fields.
__host__ __device__ inline uint32_t entry_page(uint64_t e) { return (uint32_t)(e & 0xFFFFFFFFull); }
__host__ __device__ inline int entry_class(uint64_t e) { return (int)((e >> 32) & 0xFF); }
__host__ __device__ inline uint32_t entry_mask(uint64_t e) { return (uint32_t)(e >> 48); }
__host__ __device__ inline uint64_t make_entry(uint32_t page, int cls, uint32_t mask) {
  return (uint64_t)page | ((uint64_t)cls << 32) | ((uint64_t)mask << 48);
}
// Live-list descriptor: page | class << 32 | table entry << 40.
__host__ __device__ inline uint64_t make_live_desc(uint32_t page, int cls, int entry) {
  return (uint64_t)page | ((uint64_t)cls << 32) | ((uint64_t)entry << 40);
}
__host__ __device__ inline int live_desc_entry(uint64_t x) { return (int)(x >> 40); }

// ---------------------------------------------------------------------------
// sticky status: the first error wins
// ---------------------------------------------------------------------------
__device__ inline void set_status(int32_t* status, int32_t code) {
  atomicCAS(status, 0, code);
}

// ---------------------------------------------------------------------------
// programmatic dependent launch: a kernel launched with the programmatic
// stream-serialisation attribute may start while the previous kernel of the
// stream still runs, once every CTA of that kernel has called
// pdl_launch_dependents() (or exited).  Before pdl_wait() returns -- when the
// previous kernel has completed and its writes are visible -- it may only
// read its own inputs, never cache state.  Without the attribute both are
// no-ops.
// ---------------------------------------------------------------------------
__device__ inline void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ inline void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

#ifdef __CUDACC__
// Launches kernel k with the programmatic stream-serialisation attribute.
template <typename... Params, typename... Args>
inline cudaError_t launch_pdl(void (*k)(Params...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, std::forward<Args>(args)...);
}
#endif

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ inline uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ inline void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ inline void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ inline void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Orders this thread's view of global memory (generic proxy) before its
// later bulk copies (async proxy) that read it.
__device__ inline void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ inline void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
      "r"(bytes)
      : "memory");
}

// One bounded probe of phase `parity`; true once the phase has completed.
__device__ inline bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking probe of phase `parity`.
__device__ inline bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for phase `parity` with an iteration bound; false if the bound ran out.
// The non-blocking probe answers at once when the data has already landed.
constexpr uint32_t kWaitLimit = 1u << 22;
__device__ inline bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  if (mbar_test_wait(bar, parity)) return true;
  for (uint32_t it = 0; it < kWaitLimit; ++it)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// Bulk copy (TMA engine, no tensor map, no multicast) global -> shared,
// completing `bytes` of transaction count on `bar`.  dst, src 16-byte
// aligned; bytes a multiple of 16.
__device__ inline void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// D = A * B + C, m16n8k16, fp16 inputs, fp32 accumulate.
__device__ inline void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 2^x on the SFU (PTX ex2.approx; relative error about 2^-22).
__device__ inline float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// half2 bit pattern of (lo, hi) fp32 values, each rounded to nearest.
__device__ inline uint32_t pack_half2_rn(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ inline uint32_t hsub2_bits(uint32_t a, uint32_t b) {
  __half2 r = __hsub2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

// ---------------------------------------------------------------------------
// code unpacking: element k of the low and of the high half-word of `w`
// (b-bit codes, element k at bits [b*k, b*k+b) of its half) as the half2
// (1024 + code_lo, 1024 + code_hi) -- exact, since fp16 has 10 mantissa bits.
// ---------------------------------------------------------------------------
template <int B>
__device__ inline uint32_t unpack_pair(uint32_t w, int k) {
  constexpr uint32_t m = (1u << B) - 1u;
  return ((w >> (B * k)) & (m | (m << 16))) | 0x64006400u;
}
// 8-bit codes: one byte permute places bytes k and k+2 under the 0x64 exponent byte.
template <>
__device__ inline uint32_t unpack_pair<8>(uint32_t w, int k) {
  return __byte_perm(w, 0x64646464u, k == 0 ? 0x4240u : 0x4341u);
}

// fp16 pair (1024 + 2^(b-1), same): subtracted from an unpacked pair it gives
// the centred codes (code - 2^(b-1)), exactly.
template <int B>
__device__ inline uint32_t centre_bits() {
  constexpr uint32_t h = 0x6400u + (1u << (B - 1));
  return h | (h << 16);
}

// fp16 pair (-(1024 + 2^(b-1)), same), exact in fp16: the constant A operand
// that turns the products of (1024 + code) into products of the centred code.
template <int B>
__device__ inline uint32_t neg_centre_bits() {
  constexpr uint32_t h = 0xE400u + (1u << (B - 1));  // sign | 1024 + 2^(b-1)
  return h | (h << 16);
}

// ---------------------------------------------------------------------------
// the float code formats (a class with fmt 1): FP8 E4M3 and FP4 E2M1, converted
// by the hardware's cvt (round to nearest even, saturating to the largest
// finite value); both are exact in fp16.
// ---------------------------------------------------------------------------
// E4M3 code of x.
__device__ inline uint32_t e4m3_code(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(r) : "f"(x));
  return r & 0xFFu;
}
// E2M1 code of x (4 bits).
__device__ inline uint32_t e2m1_code(float x) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %1;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(r)
      : "f"(x));
  return r & 0xFu;
}
// Two E4M3 codes (lo: bits 0-7, hi: bits 8-15) as the half2 (value(lo), value(hi)).
__device__ inline uint32_t e4m3x2_to_half2(uint32_t pair) {
  uint32_t r;
  asm("{\n\t.reg .b16 t;\n\t"
      "cvt.u16.u32 t, %1;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
      : "=r"(r)
      : "r"(pair));
  return r;
}
// Two E2M1 codes (lo: bits 0-3, hi: bits 4-7) as the half2 (value(lo), value(hi)).
__device__ inline uint32_t e2m1x2_to_half2(uint32_t pair) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.u8.u32 t, %1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
      : "=r"(r)
      : "r"(pair));
  return r;
}
// Float-format operand pair k of word w, laid out like unpack_pair: element k
// of the low half-word (even channel / first token) in the low fp16 half,
// element k of the high half-word in the high half.
template <int B>
__device__ inline uint32_t unpack_float_pair(uint32_t w, int k) {
  if constexpr (B == 8) {
    return e4m3x2_to_half2(__byte_perm(w, 0u, k == 0 ? 0x0020u : 0x0031u));
  } else {
    const uint32_t t = w >> (4 * k);
    return e2m1x2_to_half2((t & 0xFu) | ((t >> 12) & 0xF0u));
  }
}

}  // namespace thinkv
