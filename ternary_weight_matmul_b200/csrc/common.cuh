// common.cuh -- shared device helpers of libmmf: dtype access, reductions, the device error
// flag, bounded mbarrier waits and the sm_100a (tcgen05 / TMA) PTX wrappers.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mmf.h"

namespace mmf {

// ---------------------------------------------------------------------------------------------
// device error flag: kernels OR a code in; mmf_sync_status() reads and clears it
// ---------------------------------------------------------------------------------------------
enum : unsigned { kErrNone = 0u, kErrTimeout = 1u };
__device__ unsigned g_device_error = 0u;

__device__ __forceinline__ void raise_device_error(unsigned code) { atomicOr(&g_device_error, code); }

// ---------------------------------------------------------------------------------------------
// dtype access
// ---------------------------------------------------------------------------------------------
template <mmf_dtype DT> struct Elem;
template <> struct Elem<MMF_F32> {
  using T = float;
  static __device__ __forceinline__ float to_float(T v) { return v; }
  static __device__ __forceinline__ float load(const T* p) { return *p; }
  static __device__ __forceinline__ void store(T* p, float v) { *p = v; }
};
template <> struct Elem<MMF_BF16> {
  using T = __nv_bfloat16;
  static __device__ __forceinline__ float to_float(T v) { return __bfloat162float(v); }
  static __device__ __forceinline__ float load(const T* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ void store(T* p, float v) { *p = __float2bfloat16_rn(v); }
};

__device__ __forceinline__ float load_as_float(const void* base, int64_t idx, mmf_dtype dt) {
  return dt == MMF_F32 ? reinterpret_cast<const float*>(base)[idx]
                       : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[idx]);
}
__device__ __forceinline__ void store_from_float(void* base, int64_t idx, mmf_dtype dt, float v) {
  if (dt == MMF_F32) reinterpret_cast<float*>(base)[idx] = v;
  else reinterpret_cast<__nv_bfloat16*>(base)[idx] = __float2bfloat16_rn(v);
}

// sigmoid and SiLU from their definitions, 1 / (1 + e^-z) and z * sigmoid(z), with the CUDA
// fast-math intrinsics __expf and __fdividef (a few ulp; e^-z overflowing to +inf gives 0).
__device__ __forceinline__ float sigmoidf_(float z) { return __fdividef(1.0f, 1.0f + __expf(-z)); }
__device__ __forceinline__ float siluf_(float z) { return z * sigmoidf_(z); }
// HGRN gates: f = sigmoid(zf) and 1 - f = sigmoid(-zf) = e^-zf * f, formed from one exponential so
// 1 - f keeps full relative accuracy when f is close to 1; zf is clamped at -80 (e^80 is finite,
// and sigmoid(-80) is below 2e-35) so the product never meets inf * 0.
__device__ __forceinline__ void hgrn_forget(float zf, float& f, float& one_minus_f) {
  const float e = __expf(-fmaxf(zf, -80.0f));
  f = __fdividef(1.0f, 1.0f + e);
  one_minus_f = e * f;
}

// ---------------------------------------------------------------------------------------------
// reductions
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
// Block-wide sum / max; `red` is shared scratch of >= 32 floats. All threads get the result.
__device__ __forceinline__ float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float r = lane < nw ? red[lane] : 0.0f;
  return warp_sum(r);
}
__device__ __forceinline__ float block_max(float v, float* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float r = lane < nw ? red[lane] : 0.0f;
  return warp_max(r);
}

// ---------------------------------------------------------------------------------------------
// ternary code expansion
// ---------------------------------------------------------------------------------------------
// A packed word holds 16 codes; quad q (columns 4q..4q+3) sits in the low two bits of the four
// nibbles of half (q >> 1), shifted by 2*(q & 1). Byte-permuting the constant 0xFF000100
// (bytes: 0x00, 0x01, 0x00, 0xFF) by those nibbles maps field 00 -> 0, 01 -> +1, 11 -> -1
// (the unused 10 -> 0) and yields the quad as four int8 lanes, lowest column in byte 0.
__device__ __forceinline__ void expand_word(uint32_t w, uint32_t out[4]) {
  const uint32_t lo = w & 0x33333333u;          // quads 0 (low half) and 2 (high half)
  const uint32_t hi = (w >> 2) & 0x33333333u;   // quads 1 and 3
  out[0] = __byte_perm(0xFF000100u, 0u, lo & 0xFFFFu);
  out[1] = __byte_perm(0xFF000100u, 0u, hi & 0xFFFFu);
  out[2] = __byte_perm(0xFF000100u, 0u, lo >> 16);
  out[3] = __byte_perm(0xFF000100u, 0u, hi >> 16);
}

// ---------------------------------------------------------------------------------------------
// mbarrier, TMA and tcgen05 wrappers (sm_100a)
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0u;
}
__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// SM cycles per microsecond used to turn the wait cap into a cycle budget. The SM clock never
// exceeds 1.965 GHz on B200, so the real cap is at least the requested time.
constexpr int64_t kCyclesPerUs = 2000;

// Bounded wait for the phase with the given parity. Gives up after `limit_us` microseconds
// (counted in SM cycles, checked every 16 polls) or as soon as another role of the CTA has set
// *abort; on giving up it raises the timeout flag, sets *abort and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint32_t limit_us,
                                                  volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const int64_t t0 = clock64();
  const int64_t lim = (int64_t)limit_us * kCyclesPerUs;
  uint32_t polls = 0;
  while (!mbar_try_wait(bar, parity)) {
    if ((++polls & 15u) == 0u) {
      if (*abort) return false;
      if (clock64() - t0 >= lim) {
        raise_device_error(kErrTimeout);
        *abort = 1;
        return false;
      }
    }
  }
  return true;
}

// Wait without an abort check, used only while draining after an abort. Its own cap (1 s) does
// not follow the (possibly lowered) wait limit: copies and MMAs already issued complete within
// microseconds, and the CTA must not release shared or tensor memory before they have.
constexpr int64_t kDrainCycles = 1000000ll * kCyclesPerUs;
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const int64_t t0 = clock64();
  while (!mbar_try_wait(bar, parity) && clock64() - t0 < kDrainCycles) {
  }
}

// 2-D tiled TMA load global -> shared, completion counted on `bar` (no multicast).
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, int32_t c0,
                                            int32_t c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Whole-warp TMEM allocation; the column base is written to *dst (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// Arrive once on `bar` when every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
// D(tmem) (+)= A(tmem) x B(smem), int8 x int8 -> int32.
__device__ __forceinline__ void tc_mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D(tmem) (+)= A(smem) x B(smem), bf16 x bf16 -> float32 (kind::f16, both operands by descriptor).
__device__ __forceinline__ void tc_mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Shared-memory matrix descriptor of a K-major, 128-byte-swizzled operand tile: start address
// >> 4 (bits 0-13), leading byte offset 16 B (unused for this layout, bits 16-29), stride byte
// offset 1024 B = 8 rows x 128 B (bits 32-45), descriptor version 1 (bits 46-47), layout type
// SWIZZLE_128B = 2 (bits 61-63). The tile starts on a 1024-byte boundary; K steps inside the
// 128-byte atom advance the start address.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr) {
  return (uint64_t)((smem_addr & 0x3FFFFu) >> 4) | ((uint64_t)1u << 16) | ((uint64_t)64u << 32) |
         ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

#define MMF_R32(i) "r"(v[i])
// 32 lanes x 32 consecutive 32-bit columns, one column per register.
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32};" ::"r"(taddr),
      MMF_R32(0), MMF_R32(1), MMF_R32(2), MMF_R32(3), MMF_R32(4), MMF_R32(5), MMF_R32(6),
      MMF_R32(7), MMF_R32(8), MMF_R32(9), MMF_R32(10), MMF_R32(11), MMF_R32(12), MMF_R32(13),
      MMF_R32(14), MMF_R32(15), MMF_R32(16), MMF_R32(17), MMF_R32(18), MMF_R32(19), MMF_R32(20),
      MMF_R32(21), MMF_R32(22), MMF_R32(23), MMF_R32(24), MMF_R32(25), MMF_R32(26), MMF_R32(27),
      MMF_R32(28), MMF_R32(29), MMF_R32(30), MMF_R32(31)
      : "memory");
}
#undef MMF_R32
#define MMF_W32(i) "=r"(v[i])
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31}, [%32];"
      : MMF_W32(0), MMF_W32(1), MMF_W32(2), MMF_W32(3), MMF_W32(4), MMF_W32(5), MMF_W32(6),
        MMF_W32(7), MMF_W32(8), MMF_W32(9), MMF_W32(10), MMF_W32(11), MMF_W32(12), MMF_W32(13),
        MMF_W32(14), MMF_W32(15), MMF_W32(16), MMF_W32(17), MMF_W32(18), MMF_W32(19),
        MMF_W32(20), MMF_W32(21), MMF_W32(22), MMF_W32(23), MMF_W32(24), MMF_W32(25),
        MMF_W32(26), MMF_W32(27), MMF_W32(28), MMF_W32(29), MMF_W32(30), MMF_W32(31)
      : "r"(taddr)
      : "memory");
}
#undef MMF_W32
#define MMF_W16(i) "=r"(v[i])
// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : MMF_W16(0), MMF_W16(1), MMF_W16(2), MMF_W16(3), MMF_W16(4), MMF_W16(5), MMF_W16(6),
        MMF_W16(7), MMF_W16(8), MMF_W16(9), MMF_W16(10), MMF_W16(11), MMF_W16(12), MMF_W16(13),
        MMF_W16(14), MMF_W16(15)
      : "r"(taddr)
      : "memory");
}
#undef MMF_W16
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

}  // namespace mmf
