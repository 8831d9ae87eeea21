// Internal definitions shared by the kernels and the C ABI layer of libmoemx.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "../../include/moemx.h"

namespace moemx {

typedef __nv_bfloat16 bf16;

// Bits of the device status word (moe_ctx's first int).
constexpr int kStatusDevice = 1;   // bad expert index / split_sizes mismatch
constexpr int kStatusTimeout = 2;  // a bounded wait expired

// Bounded-wait limit in SM clock cycles (about one second at the B200's clocks).
constexpr long long kWaitLimitCycles = 2000000000LL;

__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ inline int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

// Byte offset of scale S[r][kb] of a matrix with KB scale columns (K/32) in the tensor-core tile
// layout: 512-byte tiles of 128 rows x 4 scale columns, row-block major; inside a tile
// row r sits in 16-byte line r%32 at word (r/32)%4, and the scale column picks the byte.
__host__ __device__ inline int64_t sf_mma_offset(int64_t r, int64_t kb, int64_t KB) {
  return ((r >> 7) * (KB >> 2) + (kb >> 2)) * 512 + ((r & 31) << 4) + (((r >> 5) & 3) << 2) + (kb & 3);
}

// E8M0 exponent e = the smallest integer with amax <= 448 * 2^e, from the fp32 bits of amax
// (amax = (1 + m/2^23) * 2^E: e = E - 8, plus one when the mantissa exceeds 0.75), clamped to
// [-127, 127].  With ``floor_rule`` (the OCP MX v1.0 variant) e = E - 8 = floor(log2 amax) - 8,
// and the block's largest elements may exceed 448 after scaling (the conversion saturates them).
// For E5M2 elements (``e5m2``) the largest finite value is 57344 = 1.75 * 2^15: 15 replaces 8.
// Returns the biased byte e + 127.
__device__ __forceinline__ uint32_t e8m0_from_amax_bits(uint32_t abits, int floor_rule = 0, int e5m2 = 0) {
  const int E = static_cast<int>((abits >> 23) & 0xFFu) - 127;
  int e = E - (e5m2 ? 15 : 8) + ((!floor_rule && (abits & 0x7FFFFFu) > 0x600000u) ? 1 : 0);
  e = e < -127 ? -127 : (e > 127 ? 127 : e);
  return static_cast<uint32_t>(e + 127);
}
// Two fp32 values -> two 8-bit codes (low byte first), round to nearest even, saturating: E4M3, or
// E5M2 when ``e5m2``.
__device__ __forceinline__ uint32_t fp8x2(float lo, float hi, int e5m2) {
  return static_cast<uint32_t>(
      __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, e5m2 ? __NV_E5M2 : __NV_E4M3));
}
// Per-tensor FP8 scale (current scaling): s = vmax / amax rounded to nearest in fp32 (vmax 448 for
// E4M3, 57344 for E5M2); 1 for an all-zero tensor; the largest finite fp32 when the quotient
// overflows.  ``amax_bits``: the fp32 bits of the tensor's largest magnitude.
__device__ __forceinline__ float fp8_tensor_scale(uint32_t amax_bits, int e5m2) {
  const float amax = __uint_as_float(amax_bits);
  if (!(amax > 0.f)) return 1.f;
  const float s = __fdiv_rn(e5m2 ? 57344.f : 448.f, amax);
  return isinf(s) ? __uint_as_float(0x7F7FFFFFu) : s;
}
// 2^-(byte-127) as an fp32 (byte <= 253 for every finite input).
__device__ __forceinline__ float e8m0_inv_scale(uint32_t byte) {
  return __uint_as_float((254u - byte) << 23);
}

}  // namespace moemx
