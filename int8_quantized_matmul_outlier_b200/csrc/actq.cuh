// Device helpers shared by the activation and weight passes: binary16
// magnitude maxima, the scale c = 127/absmax, round-to-nearest-even int8
// codes, programmatic-dependent-launch controls, and the few memory
// operations the single-launch activation pass needs (bulk copies into shared
// memory, release stores; the acquire load and the release add are in
// ptx.cuh).
//
// Method: "LLM.int8() — 大模型激活值里藏着几个超大异常通道", 方法1 (one scale
// per row of X and per column of W, c = 127/absmax, codes rounded to int8).
//
// |x| is handled as the binary16 magnitude bits (h & 0x7fff), whose unsigned
// order equals the order of |x|, so maxima are exact and two lanes are
// compared per instruction (vmax2).
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

namespace i8mm {

// fp32 product rounded once, then round-to-nearest-even, clamped to +-127.
__device__ __forceinline__ int8_t quant_rne(float x, float c) {
  int q = __float2int_rn(__fmul_rn(x, c));
  q = max(-127, min(127, q));
  return static_cast<int8_t>(q);
}

// c = 127 / absmax for an absmax given as binary16 magnitude bits; 0 when
// the absmax is 0 (an all-zero vector keeps all-zero codes).
__device__ __forceinline__ float scale_from_absmax_bits(uint32_t bits) {
  const float a = __half2float(__ushort_as_half(static_cast<unsigned short>(bits)));
  return a == 0.0f ? 0.0f : __fdiv_rn(127.0f, a);
}

__device__ __forceinline__ uint32_t max_pair(uint32_t m) { return max(m & 0xffffu, m >> 16); }

// rne(x * c) as int8 in the low byte.  |x| <= absmax and c = 127/absmax
// bound |x * c| by 127 (1 + 2^-24), which rounds to at most 127, so the
// saturating conversion equals the clamp to [-127, 127] exactly.
__device__ __forceinline__ uint32_t q8(float x, float c) {
  int32_t q;
  asm("cvt.rni.sat.s8.f32 %0, %1;" : "=r"(q) : "f"(__fmul_rn(x, c)));
  return static_cast<uint32_t>(q);
}

// Eight halves -> eight int8 codes, as two little-endian words.
__device__ __forceinline__ uint2 quant8(const uint4& v, float c) {
  const __half2* h = reinterpret_cast<const __half2*>(&v);
  const float2 f0 = __half22float2(h[0]), f1 = __half22float2(h[1]);
  const float2 f2 = __half22float2(h[2]), f3 = __half22float2(h[3]);
  const uint32_t a01 = __byte_perm(q8(f0.x, c), q8(f0.y, c), 0x0040);
  const uint32_t a23 = __byte_perm(q8(f1.x, c), q8(f1.y, c), 0x0040);
  const uint32_t b01 = __byte_perm(q8(f2.x, c), q8(f2.y, c), 0x0040);
  const uint32_t b23 = __byte_perm(q8(f3.x, c), q8(f3.y, c), 0x0040);
  return make_uint2(__byte_perm(a01, a23, 0x5410), __byte_perm(b01, b23, 0x5410));
}

// The same codes without conversion instructions (which issue at a fraction
// of the FMA rate), by the textbook "magic number" rounding of a float to an
// integer: y = fl(x c) as above, then fl(y + 1.5 2^23), whose ulp is 1 for
// |y| <= 2^22, rounds y to the nearest integer, ties to even (the FPU's
// rounding of the addition), and the sum's low mantissa byte is that integer
// in two's complement.  For |y| <= 127 (every non-outlier entry) the byte is
// the code; other entries are masked or overwritten by the caller.
__device__ __forceinline__ uint32_t rne_low_byte(float x, float c) {
  return __float_as_uint(__fadd_rn(__fmul_rn(x, c), 12582912.0f));
}
__device__ __forceinline__ uint32_t quant4_fma(uint32_t w01, uint32_t w23, float c) {
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w01));
  const float2 g = __half22float2(*reinterpret_cast<const __half2*>(&w23));
  const uint32_t a = __byte_perm(rne_low_byte(f.x, c), rne_low_byte(f.y, c), 0x0040);
  const uint32_t b = __byte_perm(rne_low_byte(g.x, c), rne_low_byte(g.y, c), 0x0040);
  return __byte_perm(a, b, 0x5410);
}
__device__ __forceinline__ uint2 quant8_fma(const uint4& v, float c) {
  return make_uint2(quant4_fma(v.x, v.y, c), quant4_fma(v.z, v.w, c));
}

// Bits 0..3 of n -> 0xff in bytes 0..3 of the result.
__device__ __forceinline__ uint32_t expand_nibble(uint32_t n) {
  return ((n * 0x00204081u) & 0x01010101u) * 0xffu;
}

// Max of the magnitudes of the halves of v whose flag bit is clear.
__device__ __forceinline__ uint32_t masked_absmax2(uint32_t m, const uint4& v, uint32_t fl) {
  if (fl == 0) {
    m = __vmaxu2(m, v.x & 0x7fff7fffu);
    m = __vmaxu2(m, v.y & 0x7fff7fffu);
    m = __vmaxu2(m, v.z & 0x7fff7fffu);
    return __vmaxu2(m, v.w & 0x7fff7fffu);
  }
  const uint32_t* w = reinterpret_cast<const uint32_t*>(&v);
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const uint32_t keep = (((fl >> (2 * p)) & 1u) ? 0u : 0x0000ffffu) | (((fl >> (2 * p + 1)) & 1u) ? 0u : 0xffff0000u);
    m = __vmaxu2(m, w[p] & 0x7fff7fffu & keep);
  }
  return m;
}

// Programmatic dependent launch: let the next kernel of the stream start its
// prologue, and wait until the previous kernel's results are visible.  Both
// are no-ops for a kernel launched without the programmatic attribute.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Contiguous bulk copy global -> this CTA's shared memory, completing on the
// mbarrier `bar` with `bytes` transaction bytes.  Both addresses 16-byte
// aligned, `bytes` a multiple of 16.
__device__ __forceinline__ void bulk_load_1d(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
               "l"(gsrc), "r"(bytes), "r"(static_cast<uint32_t>(__cvta_generic_to_shared(bar)))
               : "memory");
}

__device__ __forceinline__ void st_release_gpu(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

}  // namespace i8mm
