// Small device helpers (inline PTX for sm_100a).
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

#include "dictproj_internal.h"

namespace dictproj {

// ---- programmatic dependent launch -------------------------------------------
// Wait until the preceding grid on the stream has completed and its memory is
// visible. Must precede every read of data a previous kernel may have written.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
// Allow the next grid on the stream to start launching its CTAs.
__device__ __forceinline__ void trigger_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" :::);
}

// ---- loads --------------------------------------------------------------------
// Streaming read-only 16-byte load (weights: read once per call).
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}
__device__ __forceinline__ uint2 ld_stream_v2(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
               : "=r"(r.x), "=r"(r.y)
               : "l"(p));
  return r;
}
__device__ __forceinline__ uint32_t ld_stream_u16(const void* p) {
  unsigned short r;
  asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(r) : "l"(p));
  return r;
}
__device__ __forceinline__ uint32_t ld_stream_u8(const void* p) {
  unsigned short r;
  asm volatile("ld.global.nc.L1::no_allocate.u8 %0, [%1];" : "=h"(r) : "l"(p));
  return r;
}
// Load of data another grid wrote (served by L2, never a stale L1 line).
__device__ __forceinline__ float4 ld_cg_v4f(const float* p) {
  float4 r;
  asm volatile("ld.global.cg.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
               : "l"(p)
               : "memory");
  return r;
}
// Read-only load that may stay in L1 (small operands reused across a CTA).
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Bulk prefetch of [p, p+bytes) into L2; p 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
// Prefetch the 16-byte chunks that lie wholly inside [begin, end) of a 16-byte
// aligned array (rounded inward, so no address outside the range is named; the
// partial chunks at the two ends are simply not prefetched).
__device__ __forceinline__ void prefetch_l2_range(const void* base, size_t begin, size_t end) {
  const char* b = static_cast<const char*>(base);
  size_t a = (begin + 15) & ~size_t(15);
  size_t e = end & ~size_t(15);
  while (a < e) {
    size_t n = e - a;
    if (n > 65536) n = 65536;
    prefetch_l2_bulk(b + a, (uint32_t)n);
    a += n;
  }
}

// ---- NVFP4 element / scale conversion ------------------------------------------
// Two E2M1 codes in one byte (low nibble = first element) -> f16x2 (first in .x).
// E2M1 values are exact in fp16.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte_in_low8) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t}"
      : "=r"(out)
      : "r"(byte_in_low8));
  return out;
}
// All four bytes of a word: out[i] holds elements 2i, 2i+1.
__device__ __forceinline__ void e2m1x8_to_f16x2x4(uint32_t w, uint32_t out[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(out[0]), "=r"(out[1]), "=r"(out[2]), "=r"(out[3])
      : "r"(w));
}
// Two E4M3 codes (low byte first) -> f16x2. E4M3 values are exact in fp16.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_bytes) {
  uint32_t out;
  unsigned short h = (unsigned short)(two_bytes & 0xFFFF);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(out) : "h"(h));
  return out;
}
__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) {
  uint32_t h2 = e4m3x2_to_f16x2(byte & 0xFF);
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFF)));
}

// One E4M3 byte -> f32 with integer operations and one multiply (no conversion
// unit): the 7 magnitude bits placed at bit 20 read as an fp32 whose exponent is
// the E4M3 exponent field (subnormals read as fp32 subnormals), so scaling by
// 2^(127-7) gives the E4M3 value exactly; the sign bit moves to bit 31.
__device__ __forceinline__ float e4m3_to_f32_int(uint32_t byte) {
  const uint32_t bits = ((byte & 0x7Fu) << 20) | ((byte & 0x80u) << 24);
  return __uint_as_float(bits) * 0x1p120f;
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
// Broadcast the low / high half of an f16x2 to both halves.
__device__ __forceinline__ uint32_t dup_lo(uint32_t h2) { return __byte_perm(h2, 0, 0x1010); }
__device__ __forceinline__ uint32_t dup_hi(uint32_t h2) { return __byte_perm(h2, 0, 0x3232); }

// ---- legacy warp MMA (16x8x16, fp16 in, fp32 accumulate) ------------------------
__device__ __forceinline__ void mma_16816(float c[4], const uint32_t a[4], const uint32_t b[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

}  // namespace dictproj

namespace dictproj {

// ---- shared-memory addresses, mbarriers and bulk async copies ------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t phase) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(phase)
      : "memory");
  return ok != 0;
}
// Global -> shared bulk copy completing on `bar`; addresses 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ---- 32-bit shared-memory loads (explicit shared state space) -------------------
__device__ __forceinline__ float lds_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ float2 lds_f32x2(uint32_t a) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ float4 lds_f32x4(uint32_t a) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 lds_u32x2(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint4 lds_u32x4(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
// 8- and 16-bit loads zero-extended straight into a 32-bit register.
__device__ __forceinline__ uint32_t lds_u8(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds_u16(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}

// x << n with the PTX rule for n >= 32 (the result is 0).
__device__ __forceinline__ uint32_t shl_clamped(uint32_t x, uint32_t n) {
  uint32_t r;
  asm("shl.b32 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(n));
  return r;
}
// prmt.b32 in its default mode: result byte i is byte (sel nibble i & 7) of
// {b:a}, replaced by copies of that byte's top bit when nibble bit 3 is set.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// ---- fp16 Z rows: one mixed-precision FMA per token ---------------------------
// acc += z * v with z and v fp16 and acc fp32 (fma.rn.f32.f16: the product of two
// fp16 values is exact in fp32, so only the accumulation rounds). v is half H of
// an f16x2 register.
__device__ __forceinline__ unsigned short lds_h16(uint32_t a) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}
template <int H>
__device__ __forceinline__ void ffma_h(float& acc, unsigned short z, uint32_t v2) {
  if constexpr (H == 0)
    asm("{\n\t.reg .f16 vl, vh;\n\tmov.b32 {vl, vh}, %2;\n\tfma.rn.f32.f16 %0, %1, vl, %0;\n\t}"
        : "+f"(acc) : "h"(z), "r"(v2));
  else
    asm("{\n\t.reg .f16 vl, vh;\n\tmov.b32 {vl, vh}, %2;\n\tfma.rn.f32.f16 %0, %1, vh, %0;\n\t}"
        : "+f"(acc) : "h"(z), "r"(v2));
}
// Both halves of an f16x2 word z2 (two tokens) times half H of v2.
template <int H>
__device__ __forceinline__ void ffma_h2(float& a0, float& a1, uint32_t z2, uint32_t v2) {
  if constexpr (H == 0)
    asm("{\n\t.reg .f16 z0, z1, vl, vh;\n\tmov.b32 {z0, z1}, %2;\n\tmov.b32 {vl, vh}, %3;\n\t"
        "fma.rn.f32.f16 %0, z0, vl, %0;\n\tfma.rn.f32.f16 %1, z1, vl, %1;\n\t}"
        : "+f"(a0), "+f"(a1) : "r"(z2), "r"(v2));
  else
    asm("{\n\t.reg .f16 z0, z1, vl, vh;\n\tmov.b32 {z0, z1}, %2;\n\tmov.b32 {vl, vh}, %3;\n\t"
        "fma.rn.f32.f16 %0, z0, vh, %0;\n\tfma.rn.f32.f16 %1, z1, vh, %1;\n\t}"
        : "+f"(a0), "+f"(a1) : "r"(z2), "r"(v2));
}
// Z rows of MP fp16 tokens at byte address a; acc[m] += Z[m] * (half H of v2).
template <int MP, int H>
__device__ __forceinline__ void fma_zh(float acc[MP], uint32_t a, uint32_t v2) {
  if constexpr (MP == 1) {
    ffma_h<H>(acc[0], lds_h16(a), v2);
  } else if constexpr (MP == 2) {
    ffma_h2<H>(acc[0], acc[1], lds_u32(a), v2);
  } else if constexpr (MP == 4) {
    const uint2 z = lds_u32x2(a);
    ffma_h2<H>(acc[0], acc[1], z.x, v2);
    ffma_h2<H>(acc[2], acc[3], z.y, v2);
  } else {
    const uint4 z = lds_u32x4(a);
    ffma_h2<H>(acc[0], acc[1], z.x, v2);
    ffma_h2<H>(acc[2], acc[3], z.y, v2);
    ffma_h2<H>(acc[4], acc[5], z.z, v2);
    ffma_h2<H>(acc[6], acc[7], z.w, v2);
  }
}

// Z rows live in shared memory at byte address zaddr + atom * MP * 4.
template <int MP>
__device__ __forceinline__ void fma_z(float blk[MP], uint32_t a, float v) {
  if constexpr (MP == 1) {
    blk[0] = fmaf(lds_f32(a), v, blk[0]);
  } else if constexpr (MP == 2) {
    const float2 t = lds_f32x2(a);
    blk[0] = fmaf(t.x, v, blk[0]);
    blk[1] = fmaf(t.y, v, blk[1]);
  } else {
#pragma unroll
    for (int m = 0; m < MP; m += 4) {
      const float4 t = lds_f32x4(a + 4 * m);
      blk[m] = fmaf(t.x, v, blk[m]);
      blk[m + 1] = fmaf(t.y, v, blk[m + 1]);
      blk[m + 2] = fmaf(t.z, v, blk[m + 2]);
      blk[m + 3] = fmaf(t.w, v, blk[m + 3]);
    }
  }
}

// Device error word of the translation unit that includes this header (bit 0:
// a bounded wait gave up). Each kernel file exposes a host reader for it.
static __device__ unsigned int g_dictproj_error;

// Wait for `phase` of `bar` for at most `limit` SM clocks; on time-out record the
// error and return false (the caller then leaves its loop).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t phase,
                                                  long long limit = kWaitLimitCycles) {
  if (mbar_try_wait(bar, phase)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, phase)) {
    if (clock64() - t0 > limit) {
      atomicOr(&g_dictproj_error, 1u);
      return false;
    }
  }
  return true;
}

}  // namespace dictproj
