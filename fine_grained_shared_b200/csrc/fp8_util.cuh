// fp8_util.cuh -- E4M3 / UE8M0 helpers of the fine-grained FP8 path, and
// the tcgen05 forms that take block-scaled FP8 operands.
//
// DeepSeek-V3 technical report, section 3.3 "FP8 Training": GEMM inputs in
// FP8, each small group of values carrying its own scale (fine-grained
// scaling), the scales powers of two.  Per group, e = the smallest integer
// with max|x| <= 448 * 2^e, clamped to [-127, 127]; code = E4M3(x * 2^-e),
// round to nearest even; the scale is stored as the byte e + 127 (UE8M0).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace fgs {

// Smallest e with amax <= 448 * 2^e, from the bits of amax (>= 0, finite).
// amax = (1 + m / 2^23) * 2^(E - 127) for a normal float; 448 = 1.75 * 2^8, so
// e = E - 127 - 8 when the significand is <= 1.75 and one more above it.
// Zero and subnormal maxima need e below -127 and take the clamp.
__device__ __forceinline__ int scale_exponent(float amax) {
  const uint32_t b = __float_as_uint(amax);
  const int E = int(b >> 23);
  const uint32_t m = b & 0x7FFFFFu;
  const int e = E == 0 ? -127 : E - 135 + (m > 0x600000u ? 1 : 0);
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

__device__ __forceinline__ float pow2_neg(int e) {  // 2^-e for e in [-127, 127) as a normal float
  return __uint_as_float(uint32_t(127 - e) << 23);
}

// max |x| of 8 bf16 values (exact: abs and max do not round)
__device__ __forceinline__ float amax8(const uint4& v) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
  __nv_bfloat162 m = __hmax2(__habs2(h[0]), __habs2(h[1]));
  m = __hmax2(m, __hmax2(__habs2(h[2]), __habs2(h[3])));
  return fmaxf(__low2float(m), __high2float(m));
}

// E4M3 codes of 8 bf16 values times 2^-e, in memory order.  The product is
// exact in fp32, so the paired conversion rounds once.
__device__ __forceinline__ uint2 encode8(const uint4& v, float inv) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
  uint32_t c[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 p = __bfloat1622float2(h[i]);
    p.x *= inv;
    p.y *= inv;
    c[i] = uint32_t(__nv_cvt_float2_to_fp8x2(p, __NV_SATFINITE, __NV_E4M3)) & 0xFFFFu;  // .x in the low byte
  }
  return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}


// ---------------------------------------------------------------------------
// Block-scaled MMA (tcgen05.mma.kind::mxf8f6f4.block_scale, E4M3 operands,
// UE8M0 scales, one scale per 32 consecutive K of a row).  The scales live in
// tensor memory: row m of an operand at lane m % 32 (of every 32-lane
// quadrant) and column m / 32 of its scale block, the byte within the 32-bit
// cell selecting the 32-wide K block.  They get there with tcgen05.cp from a
// 512-byte shared-memory atom per 128 rows, where byte 16 (m % 32) + 4 (m / 32)
// + k holds row m's scale of K block k.  The layer's scales cover 128 K (a
// 1 x 128 activation group or a 128 x 128 weight block), so all four bytes of
// a row's cell are equal and every MMA may read byte 0.
// ---------------------------------------------------------------------------
constexpr uint32_t kSfAtomBytes = 512;

// byte offset of row m (0..127) in a scale atom
__host__ __device__ constexpr uint32_t sf_atom_offset(int m) {
  return 16u * static_cast<uint32_t>(m & 31) + 4u * static_cast<uint32_t>(m >> 5);
}

// Shared-memory descriptor of a scale atom for tcgen05.cp: no swizzle,
// K-major, 32 rows of 16 bytes, 8-row groups 128 bytes apart.
__device__ __forceinline__ uint64_t sf_atom_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(128u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  return d;
}

// Copy a scale atom (32 rows x 128 bits) into TMEM lanes 0-31, columns
// taddr .. +3, and broadcast it to the other three lane quadrants.
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Instruction descriptor of the block-scaled MMA: E4M3 A and B (K-major),
// UE8M0 scales, fp32 accumulator, shape M x N, K = 32.  Bits: [7,10) A format
// (0 = E4M3), [10,13) B format, [17,23) N >> 3, 23 scale format (1 = UE8M0),
// [24,29) M >> 4; the scale-byte selectors ([4,6) B, [29,31) A) stay 0.
__host__ __device__ constexpr uint32_t idesc_mxf8_e4m3(int M, int N) {
  return (static_cast<uint32_t>(N >> 3) << 17) | (1u << 23) | (static_cast<uint32_t>(M >> 4) << 24);
}

// D[tmem] (+)= (A * 2^sfa) (B * 2^sfb)^T over K = 32.  One thread.
__device__ __forceinline__ void umma_mxf8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Generic-proxy writes to shared memory become visible to the async proxy
// (TMA, tcgen05.cp, tcgen05.mma) after this fence.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

}  // namespace fgs
