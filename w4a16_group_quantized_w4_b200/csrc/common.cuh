// Device helpers shared by the libw4a16 kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/w4a16.h"

namespace w4 {

constexpr int kGroup = 32;            // weights per scale along the input dimension

// Every wait on an mbarrier gives up after this many nanoseconds of %globaltimer (then the
// kernel reports W4_ERR_TIMEOUT instead of hanging).
constexpr uint64_t kWaitLimitNs = 2000000000ull;
// Suspend-time hint for mbarrier.try_wait: a waiting thread sleeps up to this long (it wakes as
// soon as the phase completes) instead of spinning.
constexpr uint32_t kSuspendHintNs = 20000;

// ------------------------------------------------------------------------------------------
// scalar conversions
// ------------------------------------------------------------------------------------------

__device__ __forceinline__ float bf16_lo_to_f32(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi_to_f32(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return (uint32_t)f32_to_bf16_bits(lo) | ((uint32_t)f32_to_bf16_bits(hi) << 16);
}

// ------------------------------------------------------------------------------------------
// shared-memory addresses, mbarriers, bulk copies (PTX ISA: mbarrier, cp.async.bulk)
// ------------------------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_inval(uint64_t* bar) {
  asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
               ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendHintNs) : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// try_wait without a suspend-time hint (the hardware's own time limit per try)
__device__ __forceinline__ bool mbar_try_wait_nohint(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}

// Bounded wait of the streaming kernel's rings (no suspend hint: a waiting warp resumes sooner
// once the phase completes); returns false once limit_ns have passed.
__device__ __forceinline__ bool mbar_wait_ring(uint64_t* bar, uint32_t parity,
                                               uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait_nohint(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_nohint(bar, parity)) return true;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// Bounded wait: returns false once kWaitLimitNs have passed (the caller reports W4_ERR_TIMEOUT).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
}

// 1-D bulk copy global -> shared, completion counted in bytes on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// 2-D tiled tensor copy global -> shared (coordinates: x = innermost element, y = row).
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, int32_t x, int32_t y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_u32(dst)), "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// L2 prefetch of one 2-D tensor tile (no shared-memory destination, nothing to wait for).  The
// innermost coordinate obeys the same 16-byte rule as a tile load.
__device__ __forceinline__ void tma_prefetch_2d(const void* tmap, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];"
               ::"l"(tmap), "r"(x), "r"(y) : "memory");
}

// L2 prefetch of a contiguous range: src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// ------------------------------------------------------------------------------------------
// loads
// ------------------------------------------------------------------------------------------

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint4 ldg_stream128(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ uint16_t ldg_u16(const uint16_t* p) {
  unsigned short v;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

// ------------------------------------------------------------------------------------------
// power-of-two row exponents, int4 -> fp16 nibble extraction and the warp-level fp16 MMA
// ------------------------------------------------------------------------------------------

__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }   // |e| <= 126

// Power-of-two exponent that brings a finite magnitude with bf16 bit pattern m (sign cleared) to
// [2^(top), 2^(top+1)); 0 for m == 0.  Clamped to +-100 so that 2^e and 2^-e stay normal floats.
__device__ __forceinline__ int shift_for(uint32_t m, int top) {
  if (m == 0) return 0;
  int E = static_cast<int>(m >> 7);
  if (E == 0) E = 1;                                   // subnormal: below 2^-126
  int e = top + 127 - E;
  return e < -100 ? -100 : (e > 100 ? 100 : e);
}


// Nibble fields of a layout-L1 code word as exact fp16 pairs, without a subtraction: OR-ing a
// field into the mantissa of 1024 (0x6400, unit in the last place 1) gives 1024 + u when the field
// sits at bits 0..3 of each half, 1024 + 16 u at bits 4..7.  The bias (1024, or 1024 / 16 once the
// matching activation is pre-divided by 16) and the -8 of q = u - 8 are removed by a per-group
// correction that enters the MMA as its C operand.
__device__ __forceinline__ uint32_t nib_f16x2_lo(uint32_t v) {   // bits 0..3 | 16..19 -> 1024 + u
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(v), "r"(0x000F000Fu), "r"(0x64006400u));
  return r;
}
__device__ __forceinline__ uint32_t nib_f16x2_hi(uint32_t v) {   // bits 4..7 | 20..23 -> 1024 + 16u
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(v), "r"(0x00F000F0u), "r"(0x64006400u));
  return r;
}

// k order of the kernels' extracted fp16 pairs.  Both GEMMs split a layout-L1 code word (nibble j =
// element j of eight) into the pairs (0, 4), (1, 5), (2, 6), (3, 7): one mask takes the nibbles at
// bits 4j and 16 + 4j together.  The activation side is written in the same order, so a pair of
// weights always meets its own pair of activations: eight bf16 values (x0..x7, two per word of w)
// become four fp16 pairs (x0, x4), (x1, x5), (x2, x6), (x3, x7); the first and third pair are
// multiplied by m_even, the second and fourth by m_odd.
__device__ __forceinline__ void f16_pairs_l1(const uint32_t (&w)[4], float m_even, float m_odd,
                                             uint32_t (&o)[4]) {
  const __half2 h0 = __floats2half2_rn(bf16_lo_to_f32(w[0]) * m_even, bf16_lo_to_f32(w[2]) * m_even);
  const __half2 h1 = __floats2half2_rn(bf16_hi_to_f32(w[0]) * m_odd, bf16_hi_to_f32(w[2]) * m_odd);
  const __half2 h2 = __floats2half2_rn(bf16_lo_to_f32(w[1]) * m_even, bf16_lo_to_f32(w[3]) * m_even);
  const __half2 h3 = __floats2half2_rn(bf16_hi_to_f32(w[1]) * m_odd, bf16_hi_to_f32(w[3]) * m_odd);
  o[0] = *reinterpret_cast<const uint32_t*>(&h0);
  o[1] = *reinterpret_cast<const uint32_t*>(&h1);
  o[2] = *reinterpret_cast<const uint32_t*>(&h2);
  o[3] = *reinterpret_cast<const uint32_t*>(&h3);
}

// D = A(16x16 fp16, row) * B(16x8 fp16, col) + C, float32 accumulators.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                              uint32_t b1, const float (&c)[4]) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%10, %11, %12, %13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1),
        "f"(c[0]), "f"(c[1]), "f"(c[2]), "f"(c[3]));
}

__device__ __forceinline__ float gelu_tanh(float z) {
  const float c = 0.7978845608028654f;  // sqrt(2/pi)
  return 0.5f * z * (1.0f + tanhf(c * (z + 0.044715f * z * z * z)));
}

// Programmatic dependent launch.  pdl_trigger lets the next kernel on the stream (launched with
// launch_pdl) start launching while this one runs; pdl_wait blocks until the previous kernel on
// the stream has completed and its memory operations are visible.  A kernel touches no global
// memory before its pdl_wait (the previous kernel may still read or write it).  Both are no-ops
// in a kernel launched without the attribute.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void set_status(int32_t* dev_status, int32_t code) {
  if (dev_status) atomicCAS(dev_status, 0, code);
}

// ------------------------------------------------------------------------------------------
// hand-over between CTAs of one kernel: counters in global memory
// ------------------------------------------------------------------------------------------

__device__ __forceinline__ int ld_acquire_gpu(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// orders this thread's generic-proxy global accesses with later async-proxy ones (bulk copies)
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// orders this thread's generic-proxy shared-memory accesses with later async-proxy ones
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Bounded wait until *p >= need (acquire at GPU scope); false once limit_ns have passed.
__device__ __forceinline__ bool wait_count(const int32_t* p, int need, uint64_t limit_ns) {
  if (ld_acquire_gpu(p) >= need) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    __nanosleep(32);
    if (ld_acquire_gpu(p) >= need) return true;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

}  // namespace w4

// Host: launch a kernel that may begin while the previous kernel on `stream` finishes
// (programmatic stream serialization; the kernel synchronises with pdl_wait).
template <typename... KArgs, typename... Args>
static inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                     cudaStream_t stream, Args... args) {
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
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}
