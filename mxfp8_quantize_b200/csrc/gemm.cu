// Persistent grouped GEMM for sm_100a.
//
// C[m, n] = sum_k A[m, k] * B[n, k] with both operands K-major, tiles of 128 x 256 outputs,
// over a device-side list of (expert, m-tile, n-tile) built from the padded expert offsets:
//  * M-grouped (forward and dgrad GEMMs): A's rows are the expert-sorted tokens, expert e
//    owning rows [poffsets[e], poffsets[e+1]); B is expert e's weight matrix.
//  * K-grouped (wgrad GEMMs): the reduction runs over expert e's tokens, K = [poffsets[e],
//    poffsets[e+1]); every expert has the same M x N output tiles (zeros when it has no tokens).
// The operands are MXFP8 (tcgen05 kind::mxf8f6f4 block-scaled MMA, one E8M0 scale per 32 K in
// TMEM) or BF16 (kind::f16).  The pages' requirement that the grouped call equal the per-expert
// loop while handling uneven counts in one launch (andresseo.expert, "Fragmented Expert
// Kernels") is what the tile list provides.
//
// One CTA per SM, 12 warps:
//   warp 0  TMA producer (one thread): operand tiles + scale tiles into a 4-stage smem ring
//   warp 1  MMA issuer (one thread): scale tiles smem->TMEM, 4 MMAs per stage, commits
//   warp 2  TMEM allocator
//   warps 4-11 epilogue: TMEM -> registers -> fused math -> global stores
// Every wait is bounded: on expiry the kernel records MOE_ERR_TIMEOUT and all roles stop.
#include <cuda_fp8.h>

#include "gemm.cuh"
#include "ptx_sm100.cuh"

namespace moemx {
namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * 128;  // 128 rows x 128 bytes of K
constexpr int B_BYTES = BN * 128;
constexpr int OFF_B = A_BYTES;
constexpr int OFF_SFA = A_BYTES + B_BYTES;
constexpr int OFF_SFB = OFF_SFA + 512;
constexpr int STAGE_BYTES = 51200;  // 1024-aligned
constexpr int EPI_WARPS = 8;
constexpr int NUM_THREADS = 32 * (4 + EPI_WARPS);
constexpr int STAGING_PER_WARP = 2048;
constexpr int SMEM_DYN = STAGES * STAGE_BYTES + EPI_WARPS * STAGING_PER_WARP + 1024;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_TMEM_COL = 256;  // scale tiles live after the 256 accumulator columns

struct SharedState {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int total_tiles;
  int tile_prefix[MOE_MAX_EXPERTS + 1];
  int poff[MOE_MAX_EXPERTS + 1];
};

struct Tile {
  int e, mb, nb, nk;
  int a_row;  // first row of A (M-grouped: token row; K-grouped: row of the M dimension)
  int k0;     // first K coordinate (K-grouped: the expert's first token row)
};

__device__ __forceinline__ void decode_tile(int t, const SharedState& s, const GemmArgs& g, bool mx, Tile& o) {
  int lo = 0, hi = g.E;  // find e with prefix[e] <= t < prefix[e+1]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s.tile_prefix[mid] <= t) lo = mid; else hi = mid;
  }
  const int e = lo;
  const int local = t - s.tile_prefix[e];
  const int P = s.poff[e + 1] - s.poff[e];
  const int bk = mx ? 128 : 64;  // K elements per stage (128 bytes)
  o.e = e;
  if (!g.kgrouped) {
    const int mt = P / BM;
    o.nb = local / mt;
    o.mb = local - o.nb * mt;
    o.a_row = s.poff[e] + o.mb * BM;
    o.k0 = 0;
    o.nk = g.K / bk;
  } else {
    o.mb = local / g.n_tiles;
    o.nb = local - o.mb * g.n_tiles;
    o.a_row = o.mb * BM;
    o.k0 = s.poff[e];
    o.nk = P / bk;
  }
}

__device__ __forceinline__ void tma_load_3d(void* smem_dst, const void* tmap, int32_t x, int32_t y, int32_t z,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(ptx::smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(ptx::smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

// Pack 8 floats as bf16 (round to nearest even) into a uint4.
__device__ __forceinline__ uint4 pack_bf16x8(const float* v) {
  uint4 o;
  uint32_t* w = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  return o;
}
__device__ __forceinline__ void unpack_bf16x8(uint4 v, float* o) {
  const bf16* h = reinterpret_cast<const bf16*>(&v);
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = __bfloat162float(h[i]);
}
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

// Row-wise MXFP8 of 32 consecutive values of this thread's row: 32 codes + 1 scale byte.
__device__ __forceinline__ void quant_row32(const float* v, uint8_t* q, uint8_t* sbyte) {
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) m = max(m, __float_as_uint(v[i]) & 0x7FFFFFFFu);
  const uint32_t sb = e8m0_from_amax_bits(m);
  const float inv = e8m0_inv_scale(sb);
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    w[i] = e4m3x2(v[4 * i] * inv, v[4 * i + 1] * inv) | (e4m3x2(v[4 * i + 2] * inv, v[4 * i + 3] * inv) << 16);
  reinterpret_cast<uint4*>(q)[0] = make_uint4(w[0], w[1], w[2], w[3]);
  reinterpret_cast<uint4*>(q)[1] = make_uint4(w[4], w[5], w[6], w[7]);
  *sbyte = static_cast<uint8_t>(sb);
}

// Column-wise MXFP8 of a 32 x 32 block held one row per lane (v = this lane's row): per column
// the amax is taken over the 32 lanes; codes are transposed through ``stage`` so that lane l
// stores column l's 32 codes contiguously at colT + l * ld, and its scale byte at sf[l].
__device__ __forceinline__ void quant_col32(const float* v, uint8_t* stage, uint8_t* colT, int64_t ld,
                                            uint8_t* sf_base, int64_t sf_row0, int64_t sf_kb, int64_t sf_KB) {
  const int lane = threadIdx.x & 31;
  uint32_t my_sb = 0;
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const uint32_t m0 = __reduce_max_sync(0xffffffffu, __float_as_uint(v[i]) & 0x7FFFFFFFu);
    const uint32_t m1 = __reduce_max_sync(0xffffffffu, __float_as_uint(v[i + 1]) & 0x7FFFFFFFu);
    const uint32_t s0 = e8m0_from_amax_bits(m0), s1 = e8m0_from_amax_bits(m1);
    if (lane == i) my_sb = s0;
    if (lane == i + 1) my_sb = s1;
    const uint32_t c = e4m3x2(v[i] * e8m0_inv_scale(s0), v[i + 1] * e8m0_inv_scale(s1));
    if ((i & 3) == 0) w[i >> 2] = c; else w[i >> 2] |= c << 16;
  }
  // stage row ``lane`` (32 bytes, two 16-byte chunks swizzled by bit 2 of the row)
  const int sw = (lane >> 2) & 1;
  reinterpret_cast<uint4*>(stage + lane * 32)[0 ^ sw] = make_uint4(w[0], w[1], w[2], w[3]);
  reinterpret_cast<uint4*>(stage + lane * 32)[1 ^ sw] = make_uint4(w[4], w[5], w[6], w[7]);
  __syncwarp();
  uint32_t o[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    uint32_t acc = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int r = 4 * j + b;
      const int ch = (lane >> 4) ^ ((r >> 2) & 1);
      acc |= static_cast<uint32_t>(stage[r * 32 + ch * 16 + (lane & 15)]) << (8 * b);
    }
    o[j] = acc;
  }
  __syncwarp();
  uint8_t* dst = colT + lane * ld;
  reinterpret_cast<uint4*>(dst)[0] = make_uint4(o[0], o[1], o[2], o[3]);
  reinterpret_cast<uint4*>(dst)[1] = make_uint4(o[4], o[5], o[6], o[7]);
  sf_base[sf_mma_offset(sf_row0 + lane, sf_kb, sf_KB)] = static_cast<uint8_t>(my_sb);
}

// Column-wise bf16 transpose of a 32 x 32 block held one row per lane: lane l stores column l.
__device__ __forceinline__ void transpose_col32_bf16(const float* v, uint8_t* stage, bf16* colT, int64_t ld) {
  const int lane = threadIdx.x & 31;
  const int sw = (lane >> 1) & 3;
#pragma unroll
  for (int c = 0; c < 4; ++c)
    reinterpret_cast<uint4*>(stage + lane * 64)[c ^ sw] = pack_bf16x8(v + 8 * c);
  __syncwarp();
  uint32_t o[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    uint32_t acc = 0;
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const int r = 2 * j + b;
      const int ch = (lane >> 3) ^ ((r >> 1) & 3);
      const uint16_t hv = *reinterpret_cast<const uint16_t*>(stage + r * 64 + ch * 16 + (lane & 7) * 2);
      acc |= static_cast<uint32_t>(hv) << (16 * b);
    }
    o[j] = acc;
  }
  __syncwarp();
  uint4* dst = reinterpret_cast<uint4*>(colT + lane * ld);
#pragma unroll
  for (int c = 0; c < 4; ++c) dst[c] = make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
}

__device__ __forceinline__ void load_acc32(uint32_t taddr, float* v) {
  uint32_t r[32];
  ptx::tmem_ld_32(taddr, r);
  ptx::tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

}  // namespace

template <bool MX, int EPI>
__global__ void __launch_bounds__(NUM_THREADS, 1) grouped_gemm_kernel(const __grid_constant__ GemmArgs g) {
  __shared__ SharedState s;
  extern __shared__ uint8_t dyn_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dyn_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging_base = smem + STAGES * STAGE_BYTES;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- set-up: tile prefix over experts, barriers, TMEM
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int e = 0; e < g.E; ++e) {
      const int p0 = g.poffsets[e], p1 = g.poffsets[e + 1];
      s.poff[e] = p0;
      s.tile_prefix[e] = acc;
      acc += g.kgrouped ? g.m_tiles * g.n_tiles : ((p1 - p0) / BM) * g.n_tiles;
    }
    s.poff[g.E] = g.poffsets[g.E];
    s.tile_prefix[g.E] = acc;
    s.total_tiles = acc;
    s.abort_flag = 0;
    for (int i = 0; i < STAGES; ++i) {
      ptx::mbar_init(&s.full[i], 1);
      ptx::mbar_init(&s.empty[i], 1);
    }
    ptx::mbar_init(&s.acc_full, 1);
    ptx::mbar_init(&s.acc_empty, EPI_WARPS);
    ptx::mbar_init(&s.drain, 1);
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&g.tmap_a);
    ptx::prefetch_tmap(&g.tmap_b);
  }
  if (warp == 2) {
    ptx::tmem_alloc(&s.tmem_base, TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  const int total = s.total_tiles;
  volatile int* abort_flag = &s.abort_flag;
  const long long lim = kWaitLimitCycles;

  if (warp == 0 && lane == 0) {
    // ================= TMA producer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_mask = 0, last_parity = 0;
    const uint32_t tx = A_BYTES + B_BYTES + (MX ? 512 + 1024 : 0);
    for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x) {
      Tile tl;
      decode_tile(t, s, g, MX, tl);
      const int bk = MX ? 128 : 64;
      for (int kb = 0; kb < tl.nk; ++kb) {
        if (!ptx::mbar_wait(&s.empty[stage], phase ^ 1, abort_flag, lim)) break;
        uint8_t* st = smem + stage * STAGE_BYTES;
        ptx::mbar_arrive_expect_tx(&s.full[stage], tx);
        const int kx = tl.k0 + kb * bk;
        ptx::tma_load_2d(st, &g.tmap_a, kx, tl.a_row, &s.full[stage]);
        int b_r0, b_r1;
        if (!g.kgrouped) {
          if (g.gate_up_half) {
            b_r0 = tl.nb * 128;
            b_r1 = g.gate_up_half + tl.nb * 128;
          } else {
            b_r0 = tl.nb * BN;
            b_r1 = b_r0 + 128;
          }
          tma_load_3d(st + OFF_B, &g.tmap_b, kx, b_r0, tl.e, &s.full[stage]);
          tma_load_3d(st + OFF_B + B_BYTES / 2, &g.tmap_b, kx, b_r1, tl.e, &s.full[stage]);
        } else {
          b_r0 = tl.nb * BN;
          b_r1 = b_r0 + 128;
          ptx::tma_load_2d(st + OFF_B, &g.tmap_b, kx, b_r0, &s.full[stage]);
          ptx::tma_load_2d(st + OFF_B + B_BYTES / 2, &g.tmap_b, kx, b_r1, &s.full[stage]);
        }
        if (MX) {
          const int64_t kq = kx / 128;
          const uint8_t* sa = g.sfa + ((static_cast<int64_t>(tl.a_row) / 128) * g.sfa_kb4 + kq) * 512;
          ptx::bulk_load(st + OFF_SFA, sa, 512, &s.full[stage]);
          const int64_t eb = g.kgrouped ? 0 : static_cast<int64_t>(tl.e) * g.sfb_expert_rows;
          const uint8_t* sb0 = g.sfb + (((eb + b_r0) / 128) * g.sfb_kb4 + kq) * 512;
          const uint8_t* sb1 = g.sfb + (((eb + b_r1) / 128) * g.sfb_kb4 + kq) * 512;
          ptx::bulk_load(st + OFF_SFB, sb0, 512, &s.full[stage]);
          ptx::bulk_load(st + OFF_SFB + 512, sb1, 512, &s.full[stage]);
        }
        issued_mask |= 1u << stage;
        last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    // wait for the loads still in flight (only possible after an abort)
    for (int i = 0; i < STAGES; ++i)
      if (issued_mask & (1u << i)) {
        volatile int never = 0;
        ptx::mbar_wait(&s.full[i], (last_parity >> i) & 1u, &never, lim);
      }
  } else if (warp == 1 && lane == 0) {
    // ================= MMA issuer
    int stage = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool issued_any = false;
    const uint32_t d_tmem = tmem;
    for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x) {
      Tile tl;
      decode_tile(t, s, g, MX, tl);
      if (tl.nk == 0) continue;
      if (!ptx::mbar_wait(&s.acc_empty, acc_phase ^ 1, abort_flag, lim)) break;
      ptx::tc_fence_after();
      bool ok = true;
      for (int kb = 0; kb < tl.nk; ++kb) {
        if (!ptx::mbar_wait(&s.full[stage], phase, abort_flag, lim)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t st = ptx::smem_u32(smem + stage * STAGE_BYTES);
        const uint64_t adesc = ptx::smem_desc(st, 16, 1024, ptx::kSwizzle128B);
        const uint64_t bdesc = ptx::smem_desc(st + OFF_B, 16, 1024, ptx::kSwizzle128B);
        if (MX) {
          const uint32_t sfa_t = tmem + SF_TMEM_COL + 12 * stage;
          const uint32_t sfb_t = sfa_t + 4;
          ptx::tc_cp_32x128b_warpx4(sfa_t, ptx::smem_desc(st + OFF_SFA, 0, 128, ptx::kSwizzleNone));
          ptx::tc_cp_32x128b_warpx4(sfb_t, ptx::smem_desc(st + OFF_SFB, 0, 128, ptx::kSwizzleNone));
          ptx::tc_cp_32x128b_warpx4(sfb_t + 4, ptx::smem_desc(st + OFF_SFB + 512, 0, 128, ptx::kSwizzleNone));
#pragma unroll
          for (int k = 0; k < 4; ++k)
            ptx::tc_mma_mxf8(d_tmem, adesc + 2 * k, bdesc + 2 * k, ptx::idesc_mxf8(BM, BN, k, k), sfa_t, sfb_t,
                             (kb | k) != 0);
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            ptx::tc_mma_bf16(d_tmem, adesc + 2 * k, bdesc + 2 * k, ptx::idesc_bf16(BM, BN), (kb | k) != 0);
        }
        ptx::tc_commit(&s.empty[stage]);
        issued_any = true;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      ptx::tc_commit(&s.acc_full);
      acc_phase ^= 1;
    }
    if (issued_any) {  // all MMAs of this CTA complete before TMEM can be released
      ptx::tc_commit(&s.drain);
      volatile int never = 0;
      ptx::mbar_wait(&s.drain, 0, &never, lim);
    }
  } else if (warp >= 4) {
    // ================= epilogue
    const int q = warp & 3;          // TMEM lane quadrant this warp may read
    const int ch = (warp - 4) >> 2;  // column half of the tile
    uint8_t* stage_buf = staging_base + (warp - 4) * STAGING_PER_WARP;
    const EpiArgs& ep = g.epi;
    uint32_t acc_phase = 0;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(32 * q) << 16);
    for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x) {
      Tile tl;
      decode_tile(t, s, g, MX, tl);
      const int64_t row_w = tl.a_row + 32 * q;  // first row of this warp
      const int64_t row = row_w + lane;
      if (tl.nk == 0) {
        // K-grouped expert without tokens: its weight gradient is zero
        if (EPI == EPI_STORE) {
          bf16* out = static_cast<bf16*>(const_cast<void*>(ep.out_ptrs.p[tl.e]));
          const int64_t c0 = static_cast<int64_t>(tl.nb) * BN + 128 * ch;
          uint4* dst = reinterpret_cast<uint4*>(out + row * ep.ldo + c0);
#pragma unroll 4
          for (int i = 0; i < 16; ++i) dst[i] = make_uint4(0, 0, 0, 0);
        }
        continue;
      }
      if (!ptx::mbar_wait(&s.acc_full, acc_phase, abort_flag, lim)) break;
      ptx::tc_fence_after();

      if (EPI == EPI_STORE) {
        bf16* out = g.kgrouped ? static_cast<bf16*>(const_cast<void*>(ep.out_ptrs.p[tl.e])) : ep.out;
        const int64_t c0 = static_cast<int64_t>(tl.nb) * BN + 128 * ch;
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          float v[32];
          load_acc32(t_lane + 128 * ch + 32 * cc, v);
          uint4* dst = reinterpret_cast<uint4*>(out + row * ep.ldo + c0 + 32 * cc);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = pack_bf16x8(v + 8 * i);
        }
      } else if (EPI == EPI_SWIGLU) {
        const float p = ep.p_perm[row];
        const int64_t f = ep.f;
#pragma unroll 1
        for (int cc = 0; cc < 2; ++cc) {
          const int64_t j = static_cast<int64_t>(tl.nb) * 128 + 64 * ch + 32 * cc;  // output column
          float gv[32], uv[32];
          load_acc32(t_lane + 64 * ch + 32 * cc, gv);
          load_acc32(t_lane + 128 + 64 * ch + 32 * cc, uv);
          if (ep.h) {
            uint4* hg = reinterpret_cast<uint4*>(ep.h + row * 2 * f + j);
            uint4* hu = reinterpret_cast<uint4*>(ep.h + row * 2 * f + f + j);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              hg[i] = pack_bf16x8(gv + 8 * i);
              hu[i] = pack_bf16x8(uv + 8 * i);
            }
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) gv[i] = silu_f(gv[i]) * uv[i] * p;  // a, in place
          if (ep.dump) {
            float4* dd = reinterpret_cast<float4*>(ep.dump + row * f + j);
#pragma unroll
            for (int i = 0; i < 8; ++i) dd[i] = make_float4(gv[4 * i], gv[4 * i + 1], gv[4 * i + 2], gv[4 * i + 3]);
          }
          if (MX) {
            uint8_t sb;
            quant_row32(gv, ep.q_row + row * f + j, &sb);
            ep.s_row[sf_mma_offset(row, j / 32, f / 32)] = sb;
            if (ep.q_colT)
              quant_col32(gv, stage_buf, ep.q_colT + j * ep.cap + row_w, ep.cap, ep.s_colT, j, row_w / 32,
                          ep.cap / 32);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(ep.o_row + row * f + j);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = pack_bf16x8(gv + 8 * i);
            if (ep.o_colT) transpose_col32_bf16(gv, stage_buf, ep.o_colT + j * ep.cap + row_w, ep.cap);
          }
        }
      } else {  // EPI_DSWIGLU
        const float p = ep.p_perm[row];
        const int64_t f = ep.f, f2 = 2 * ep.f;
        float dp = 0.f;
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          const int64_t j = static_cast<int64_t>(tl.nb) * BN + 128 * ch + 32 * cc;  // f column
          float da[32];
          load_acc32(t_lane + 128 * ch + 32 * cc, da);
          float dg[32], du[32];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float gg[8], uu[8];
            unpack_bf16x8(reinterpret_cast<const uint4*>(ep.h + row * f2 + j)[i], gg);
            unpack_bf16x8(reinterpret_cast<const uint4*>(ep.h + row * f2 + f + j)[i], uu);
#pragma unroll
            for (int q8 = 0; q8 < 8; ++q8) {
              const float gx = gg[q8], ux = uu[q8], d = da[8 * i + q8];
              const float sg = 1.0f / (1.0f + __expf(-gx));
              const float sl = gx * sg;
              dg[8 * i + q8] = d * p * ux * sg * (1.0f + gx * (1.0f - sg));
              du[8 * i + q8] = d * p * sl;
              dp += d * sl * ux;
            }
          }
          if (ep.dump) {
            float4* d0 = reinterpret_cast<float4*>(ep.dump + row * f2 + j);
            float4* d1 = reinterpret_cast<float4*>(ep.dump + row * f2 + f + j);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              d0[i] = make_float4(dg[4 * i], dg[4 * i + 1], dg[4 * i + 2], dg[4 * i + 3]);
              d1[i] = make_float4(du[4 * i], du[4 * i + 1], du[4 * i + 2], du[4 * i + 3]);
            }
          }
          if (MX) {
            uint8_t sb;
            quant_row32(dg, ep.q_row + row * f2 + j, &sb);
            ep.s_row[sf_mma_offset(row, j / 32, f2 / 32)] = sb;
            quant_row32(du, ep.q_row + row * f2 + f + j, &sb);
            ep.s_row[sf_mma_offset(row, (f + j) / 32, f2 / 32)] = sb;
            quant_col32(dg, stage_buf, ep.q_colT + j * ep.cap + row_w, ep.cap, ep.s_colT, j, row_w / 32, ep.cap / 32);
            quant_col32(du, stage_buf, ep.q_colT + (f + j) * ep.cap + row_w, ep.cap, ep.s_colT, f + j, row_w / 32,
                        ep.cap / 32);
          } else {
            uint4* d0 = reinterpret_cast<uint4*>(ep.o_row + row * f2 + j);
            uint4* d1 = reinterpret_cast<uint4*>(ep.o_row + row * f2 + f + j);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              d0[i] = pack_bf16x8(dg + 8 * i);
              d1[i] = pack_bf16x8(du + 8 * i);
            }
            transpose_col32_bf16(dg, stage_buf, ep.o_colT + j * ep.cap + row_w, ep.cap);
            transpose_col32_bf16(du, stage_buf, ep.o_colT + (f + j) * ep.cap + row_w, ep.cap);
          }
        }
        ep.dp_part[(static_cast<int64_t>(tl.nb) * 2 + ch) * ep.cap + row] = dp;
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&s.acc_empty);
      acc_phase ^= 1;
    }
  }

  __syncthreads();
  if (threadIdx.x == 0 && s.abort_flag) atomicOr(g.status, kStatusTimeout);
  if (warp == 2) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, TMEM_COLS);
  }
}

namespace {
template <bool MX, int EPI>
cudaError_t launch_t(const GemmArgs& args, int num_sms, cudaStream_t st) {
  auto kern = grouped_gemm_kernel<MX, EPI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_DYN);
  if (e != cudaSuccess) return e;
  kern<<<num_sms, NUM_THREADS, SMEM_DYN, st>>>(args);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_grouped_gemm(const GemmArgs& args, bool mx, int epi, int num_sms, cudaStream_t st) {
  if (mx) {
    if (epi == EPI_STORE) return launch_t<true, EPI_STORE>(args, num_sms, st);
    if (epi == EPI_SWIGLU) return launch_t<true, EPI_SWIGLU>(args, num_sms, st);
    return launch_t<true, EPI_DSWIGLU>(args, num_sms, st);
  }
  if (epi == EPI_STORE) return launch_t<false, EPI_STORE>(args, num_sms, st);
  if (epi == EPI_SWIGLU) return launch_t<false, EPI_SWIGLU>(args, num_sms, st);
  return launch_t<false, EPI_DSWIGLU>(args, num_sms, st);
}

}  // namespace moemx
