// Tensor-core peak loop: the dense rate of this GPU's tcgen05 tensor cores for the three operand
// kinds the grouped GEMMs use (block-scaled MXFP8, kind::mxf8f6f4 with one E8M0 scale per 32 K;
// per-tensor FP8, kind::f8f6f4; and BF16, kind::f16), measured with every operand resident in
// shared memory so that no memory traffic bounds it.  It is the denominator of the GEMMs' roofline
// fractions (ai4snews, paragraph 2: MXFP8 runs on Blackwell's tensor-core instructions).
//
// One CTA per SM.  Warp 2 allocates all 512 TMEM columns; one thread of warp 1 issues ``iters``
// groups of four M=128, N=256 MMAs (K = 4 x 32 E4M3 or 4 x 16 bf16: one 128-byte K step, the
// shape of the grouped GEMM's mainloop) into one TMEM accumulator, then commits and waits
// (bounded) for them.  With ``scale_refresh`` the MXFP8 loop also copies its A and B scale tiles
// shared memory -> TMEM before every group, into four rotating slots, as the GEMM mainloop does.
#include "common.cuh"
#include "ptx_sm100.cuh"

namespace moemx {
namespace {
constexpr int PK_A = 128 * 128;   // A tile: 128 rows x 128 bytes, 128B-swizzled
constexpr int PK_B = 256 * 128;   // B tile: 256 rows x 128 bytes
constexpr int PK_SF = 512 + 1024; // scale tiles of A (128 rows) and B (256 rows)
// Dynamic shared memory requested per CTA: more than half of an SM's, so that exactly one CTA
// runs per SM (only the first PK_A + PK_B + PK_SF bytes are used).
constexpr int PK_SMEM = 120 * 1024;
static_assert(PK_A + PK_B + PK_SF + 1024 <= PK_SMEM, "peak loop shared memory");
constexpr long long PK_MAX_ITERS = 1000000;  // one launch stays well inside the bounded final wait
constexpr uint32_t PK_SF_COL = 256;  // TMEM columns after the 128 x 256 fp32 accumulator
}  // namespace

// KIND: 0 BF16, 1 MXFP8, 2 per-tensor FP8
template <int KIND>
__global__ void __launch_bounds__(128, 1) tensor_peak_kernel(long long iters, int scale_refresh, int* status) {
  constexpr bool MX = KIND == 1, Q8 = KIND != 0;
  extern __shared__ uint8_t pk_raw[];
  uint8_t* smem = pk_raw + ((1024u - (ptx::smem_u32(pk_raw) & 1023u)) & 1023u);
  __shared__ uint64_t done;
  __shared__ uint32_t tmem_base;
  const int tid = threadIdx.x;

  // operands: hashed bit patterns restricted to finite values (E4M3 exponent field <= 14, so no
  // NaN code; bf16 magnitudes in [0.5, 1)), scale bytes 127 (a scale of 1)
  uint32_t* w = reinterpret_cast<uint32_t*>(smem);
  for (int i = tid; i < (PK_A + PK_B) / 4; i += blockDim.x) {
    uint32_t h = (static_cast<uint32_t>(i) + 1u) * 2654435761u ^ (blockIdx.x * 40503u);
    h ^= h >> 15;
    h *= 2246822519u;
    h ^= h >> 13;
    w[i] = Q8 ? (h & 0xF7F7F7F7u) : ((h & 0x807F807Fu) | 0x3F003F00u);
  }
  for (int i = tid; i < PK_SF / 4; i += blockDim.x) w[(PK_A + PK_B) / 4 + i] = 0x7F7F7F7Fu;
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic writes -> tensor-core reads
  if (tid == 0) {
    ptx::mbar_init(&done, 1);
    ptx::fence_mbar_init();
  }
  if ((tid >> 5) == 2) {
    ptx::tmem_alloc(&tmem_base, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (tid == 32) {
    const uint32_t s0 = ptx::smem_u32(smem);
    const uint64_t adesc = ptx::smem_desc(s0, 16, 1024, ptx::kSwizzle128B);
    const uint64_t bdesc = ptx::smem_desc(s0 + PK_A, 16, 1024, ptx::kSwizzle128B);
    const uint64_t sfadesc = ptx::smem_desc(s0 + PK_A + PK_B, 0, 128, ptx::kSwizzleNone);
    const uint64_t sfbdesc = ptx::smem_desc(s0 + PK_A + PK_B + 512, 0, 128, ptx::kSwizzleNone);
    const uint32_t sf0 = tmem + PK_SF_COL;
    if (MX) {
      ptx::tc_cp_32x128b_warpx4(sf0, sfadesc);
      ptx::tc_cp_32x128b_warpx4(sf0 + 4, sfbdesc);
      ptx::tc_cp_32x128b_warpx4(sf0 + 8, sfbdesc + 32);
    }
    for (long long it = 0; it < iters; ++it) {
      if (MX) {
        uint32_t sfa = sf0;
        if (scale_refresh) {
          sfa = sf0 + 12u * static_cast<uint32_t>(it & 3);
          ptx::tc_cp_32x128b_warpx4(sfa, sfadesc);
          ptx::tc_cp_32x128b_warpx4(sfa + 4, sfbdesc);
          ptx::tc_cp_32x128b_warpx4(sfa + 8, sfbdesc + 32);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k)
          ptx::tc_mma_mxf8(tmem, adesc + 2 * k, bdesc + 2 * k, ptx::idesc_mxf8(128, 256, k, k), sfa, sfa + 4,
                           (it | k) != 0);
      } else if (Q8) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          ptx::tc_mma_f8(tmem, adesc + 2 * k, bdesc + 2 * k, ptx::idesc_f8(128, 256), (it | k) != 0);
      } else {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          ptx::tc_mma_bf16(tmem, adesc + 2 * k, bdesc + 2 * k, ptx::idesc_bf16(128, 256), (it | k) != 0);
      }
    }
    ptx::tc_commit(&done);
    volatile int never = 0;
    if (!ptx::mbar_wait(&done, 0, &never, kWaitLimitCycles)) atomicOr(status, kStatusTimeout);
  }
  __syncthreads();
  if ((tid >> 5) == 2) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

double tensor_peak_flops(int kind, int num_sms, long long iters) {
  return static_cast<double>(num_sms) * static_cast<double>(iters) * 4.0 * 2.0 * 128.0 * 256.0 * (kind ? 32.0 : 16.0);
}

cudaError_t launch_tensor_peak(int kind, long long iters, int scale_refresh, int num_sms, int* status,
                               cudaStream_t st) {
  if (iters > PK_MAX_ITERS || kind < 0 || kind > 2) return cudaErrorInvalidValue;
  auto kern = kind == 1 ? tensor_peak_kernel<1> : (kind == 2 ? tensor_peak_kernel<2> : tensor_peak_kernel<0>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PK_SMEM);
  if (e != cudaSuccess) return e;
  kern<<<num_sms, 128, PK_SMEM, st>>>(iters, scale_refresh, status);
  return cudaGetLastError();
}

}  // namespace moemx
