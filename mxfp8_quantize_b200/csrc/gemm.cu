// Persistent grouped GEMM for sm_100a.
//
// C[m, n] = sum_k A[m, k] * B[n, k] with both operands K-major, tiles of 128 x BN outputs,
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
// One CTA per SM, LEAD + EPI_WARPS warps:
//   warp 0  TMA producer (one thread): operand tiles + scale tiles into a STAGES-deep smem ring
//           (scale tiles as 3-D tensor-map boxes over the tile-layout scale buffers)
//   warp 1  MMA issuer (one thread): scale tiles smem->TMEM, 4 MMAs per stage, commits
//   warp 2  TMEM allocator (warp 0 when LEAD = 2)
//   warps LEAD.. epilogue: TMEM -> registers -> fused math -> global stores
// The bf16-store and gate_up kernels use 128 x 256 tiles with one TMEM accumulator (two
// 256-column accumulators would leave no room for the per-stage scale tiles); the dSwiGLU kernel
// uses 128 x 128 tiles with two, so that its heavy epilogue overlaps the next tile's MMAs.  Plain
// bf16-store epilogues drain the accumulator into packed registers and release it before storing;
// the fused ScaledSwiGLU / dSwiGLU epilogues release it after their last TMEM load and requantise
// column-wise through a small padded smem transpose (one scale per column per lane).  Row-strided
// outputs leave in 256-bit stores (a whole 32-byte sector per lane).
// Every wait is bounded: on expiry the kernel records MOE_ERR_TIMEOUT and all roles stop; copies
// and MMAs already issued are waited for before TMEM is freed.
#include <cuda_fp16.h>
#include <algorithm>
#include <type_traits>
#include <cuda_fp8.h>

#include "gemm.cuh"
#include "ptx_sm100.cuh"

namespace moemx {
namespace {

constexpr int BM = 128;
constexpr uint32_t TMEM_COLS = 512;

// Tile shape and thread layout of one kernel instance.
//   EPI_WARPS epilogue warps (a multiple of 4: each TMEM lane quadrant gets EPI_WARPS/4 warps that
//   split the tile's columns); PASS columns per pass of the column-wise transpose buffer.
//   LEAD warps before the epilogue warps: 4 (producer, MMA issuer, TMEM allocator, idle) or 2 (the
//   producer's warp also allocates TMEM), the latter leaving more registers per thread.
//   PAIR: two CTAs of a cluster compute one 256 x BN tile with tcgen05 cta_group::2 MMAs; each CTA
//   loads its 128 rows of A, half of the tile's B rows and all of the tile's B scales, and keeps its
//   128 rows of the accumulator (MXFP8 store and SwiGLU epilogues).
//   KSUB: 128-byte K blocks per pipeline stage (more than one halves the barrier round trips per
//   MMA).
template <int BN_, int NBUF_, int STAGES_, bool STAGING_, int EPI_WARPS_, int PASS_, bool HTILE_ = false, int LEAD_ = 4,
          bool PAIR_ = false, int KSUB_ = 1>
struct Shape {
  static constexpr bool PAIR = PAIR_;
  static constexpr int KSUB = KSUB_;
  static constexpr int BN = BN_;
  static constexpr int NBUF = NBUF_;
  static constexpr int STAGES = STAGES_;
  static constexpr int EPI_WARPS = EPI_WARPS_;
  static constexpr int LEAD = LEAD_;
  static constexpr int ALLOC_WARP = LEAD == 4 ? 2 : 0;
  static constexpr int NUM_THREADS = 32 * (LEAD + EPI_WARPS);
  static constexpr int PASS = PASS_;
  static constexpr int PITCH = PASS + 1;  // odd pitch: conflict-free row writes and column reads
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_BYTES = (PAIR ? BN / 2 : BN) * 128;  // this CTA's B rows
  static constexpr int SFB_BYTES = (BN / 128) * 512;
  static constexpr int OFF_B = A_BYTES;
  static constexpr int OFF_SFA = A_BYTES + B_BYTES;
  static constexpr int OFF_SFB = OFF_SFA + 512;
  static constexpr int BLOCK_BYTES = (OFF_SFB + SFB_BYTES + 1023) / 1024 * 1024;  // one K block
  static constexpr int STAGE_BYTES = KSUB * BLOCK_BYTES;
  static constexpr int SF_COLS = 4 + 4 * (BN / 128);
  static constexpr uint32_t SF_TMEM_COL = NBUF * BN;
  static constexpr int STAGING_PER_WARP = STAGING_ ? (32 * PITCH * 4 + 15) / 16 * 16 : 0;
  static constexpr bool HTILE = HTILE_;  // dSwiGLU: the tile's saved gate/up values staged in smem by TMA
  static constexpr int H_BYTES = HTILE ? BM * 2 * BN * 2 : 0;
  static constexpr int OFF_H = STAGES * STAGE_BYTES;
  static constexpr int OFF_STAGING = OFF_H + H_BYTES;
  static constexpr int SMEM_DYN = OFF_STAGING + EPI_WARPS * STAGING_PER_WARP + 1024;
  static_assert(NBUF * BN + STAGES * KSUB * SF_COLS <= (int)TMEM_COLS, "TMEM budget");
  static_assert(SMEM_DYN + 6144 <= 232448, "shared memory budget");  // + the static SharedState
  static_assert(EPI_WARPS % 4 == 0 && 32 % PASS == 0 && (LEAD == 4 || LEAD == 2), "thread layout");
  static_assert(!PAIR || (NBUF == 1 && !HTILE && LEAD == 4), "pair instances: one accumulator, no h tile");
};
// the store GEMMs (all precisions) on CTA pairs: 256 x 256 tiles, each CTA streaming 128 rows of A
// and 128 of B per K block (two thirds of the single-CTA bytes per MMA), three stages of two K
// blocks (one barrier round trip per two blocks)
using ShapeStorePair = Shape<256, 1, 3, false, 8, 16, false, 4, true, 2>;
// (the gate_up + ScaledSwiGLU kernel stays on single CTAs: on pairs each tile waits for the slower
// of two heavy epilogues, and it measured 5% slower)
using ShapeSwiglu = Shape<256, 1, 4, true, 16, 8>;    // gate_up + ScaledSwiGLU: one 32-column group per thread
// dgrad of down + dSwiGLU: two accumulators, so the epilogue overlaps the next tile; stages of two K
// blocks (one barrier round trip per two blocks)
using ShapeDswiglu = Shape<128, 2, 2, true, 8, 16, true, 4, false, 2>;
using ShapeDswigluG = Shape<128, 2, 4, true, 8, 16, false>;  // ... reading the saved h from global memory (MXFP8 h)

struct SharedState {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint64_t h_full;
  uint64_t h_empty;
  uint32_t tmem_base;
  int abort_flag;
  int total_tiles;
  int total1;                            // EPI_FUSED_FWD: gate_up tiles (the down tiles follow)
  int tile_prefix[MOE_MAX_EXPERTS + 1];  // tiles before the i-th expert of ``order``
  int tile_prefix2[MOE_MAX_EXPERTS + 1]; // EPI_FUSED_FWD: down tiles before expert e
  int poff[MOE_MAX_EXPERTS + 1];         // padded row offsets, by expert id
  int order[MOE_MAX_EXPERTS];            // expert ids in tile-list order
};

struct Tile {
  int e, mb, nb, nk;
  int a_row;  // first row of A (M-grouped: token row; K-grouped: row of the M dimension); for a CTA
              // pair the first row of the pair's 256-row tile
  int k0;     // first K coordinate (K-grouped: the expert's first token row)
  bool down;  // EPI_FUSED_FWD: a tile of the down GEMM
  bool hi_ok; // CTA pair: the tile's second 128 rows exist (an expert may end after the first half)
};

// The i-th tile of this CTA (or CTA pair): tiles are dealt out in rounds of G workers, in
// boustrophedon order (even rounds to workers 0, 1, ..., odd rounds in reverse), so that with the
// tile list sorted from the most to the least work every worker gets a similar total.
__device__ __forceinline__ int tile_of(int i, int G, int b) { return i * G + ((i & 1) ? G - 1 - b : b); }

// Rows of A per tile: 128, or 256 for a CTA pair.
__device__ __forceinline__ void decode_tile(int t, const SharedState& s, const GemmArgs& g, bool mx, Tile& o,
                                            int rows = BM) {
  o.down = false;
  o.hi_ok = true;
  if (g.mblock_done && t >= s.total1) {  // fused forward: a down tile (experts in id order)
    const int t2 = t - s.total1;
    int lo = 0, hi = g.E;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s.tile_prefix2[mid] <= t2) lo = mid; else hi = mid;
    }
    const int e = lo, local = t2 - s.tile_prefix2[e];
    const int mt = (s.poff[e + 1] - s.poff[e]) / BM;
    o.down = true;
    o.e = e;
    o.nb = local / mt;
    o.mb = local - o.nb * mt;
    o.a_row = s.poff[e] + o.mb * BM;
    o.k0 = 0;
    o.nk = g.K2 / (mx ? 128 : 64);
    return;
  }
  int lo = 0, hi = g.E;  // largest i with prefix[i] <= t (experts without tiles are skipped)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s.tile_prefix[mid] <= t) lo = mid; else hi = mid;
  }
  const int e = s.order[lo];
  const int local = t - s.tile_prefix[lo];
  const int P = s.poff[e + 1] - s.poff[e];
  const int bk = mx ? 128 : 64;  // K elements per stage (128 bytes)
  o.e = e;
  if (!g.kgrouped) {
    const int mt = (P + rows - 1) / rows;
    o.nb = local / mt;
    o.mb = local - o.nb * mt;
    o.a_row = s.poff[e] + o.mb * rows;
    o.hi_ok = o.mb * rows + BM < P;
    o.k0 = 0;
    o.nk = g.K / bk;
  } else {
    o.mb = local / g.n_tiles;
    o.nb = local - o.mb * g.n_tiles;
    o.a_row = o.mb * rows;
    o.k0 = s.poff[e];
    o.nk = P / bk;
  }
}


// silu(g) = g * sigmoid(g); sigmoid from the hardware exp2 and a fast reciprocal-multiply
__device__ __forceinline__ float sigmoid_f(float g) { return __fdividef(1.0f, 1.0f + __expf(-g)); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
// Pack 8 floats as bf16 (round to nearest even) into a uint4.
__device__ __forceinline__ uint4 pack_bf16x8(const float* v) {
  return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                    pack_bf16x2(v[6], v[7]));
}
__device__ __forceinline__ void unpack_bf16x8(uint4 v, float* o) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    o[2 * i] = __uint_as_float(w[i] << 16);
    o[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
// Eight E4M3 codes (bytes of lo then hi) -> fp32 values times ``scale`` (exact: every E4M3 value
// is an fp16 value, and the scale is a power of two).
__device__ __forceinline__ void e4m3x8_to_float(uint32_t lo, uint32_t hi, float scale, float* o) {
  const uint32_t w[2] = {lo, hi};
#pragma unroll
  for (int k = 0; k < 2; ++k)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const __half2_raw r =
          __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>((w[k] >> (16 * h)) & 0xFFFFu), __NV_E4M3);
      const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&r));
      o[4 * k + 2 * h] = v.x * scale;
      o[4 * k + 2 * h + 1] = v.y * scale;
    }
}
// Largest magnitude of eight packed bf16 values, as bf16 bits (bits & 0x7FFF grows with |x|).
__device__ __forceinline__ uint32_t absmax_bf16x8_bits(uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t m = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) m = max(m, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
  return m;
}
// 2^(byte - 127) as an fp32 (byte 0: 2^-127, a subnormal).
__device__ __forceinline__ float e8m0_scale(uint32_t byte) {
  return byte ? __uint_as_float(byte << 23) : __uint_as_float(0x00400000u);
}

// MXFP8 of 32 values with the scale of their own amax: 32 codes (E4M3, or E5M2 when ``e5m2``)
// stored at q (32-byte aligned); returns the E8M0 byte.
__device__ __forceinline__ uint32_t quant32_store(const float* v, uint8_t* q, int floor_rule, int e5m2) {
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) m = max(m, __float_as_uint(v[i]) & 0x7FFFFFFFu);
  const uint32_t sb = e8m0_from_amax_bits(m, floor_rule, e5m2);
  const float inv = e8m0_inv_scale(sb);
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    w[i] = fp8x2(v[4 * i] * inv, v[4 * i + 1] * inv, e5m2) | (fp8x2(v[4 * i + 2] * inv, v[4 * i + 3] * inv, e5m2) << 16);
  ptx::st_global_v8(q, make_uint4(w[0], w[1], w[2], w[3]), make_uint4(w[4], w[5], w[6], w[7]));
  return sb;
}

// Column-wise outputs of a 32 x 32 block held one row per lane (v = this lane's 32 values), in
// 32/P passes of P columns through the warp's padded smem buffer: after a pass lane l holds column
// c = l % P of the pass, rows P*(l/P) .. +P.
template <int P, class F>
__device__ __forceinline__ void column_passes(const float* v, float* stage, F&& emit) {
  const int lane = threadIdx.x & 31;
  constexpr int PITCH = P + 1;
#pragma unroll
  for (int h = 0; h < 32 / P; ++h) {
#pragma unroll
    for (int c = 0; c < P; ++c) stage[lane * PITCH + c] = v[P * h + c];
    __syncwarp();
    float col[P];
    const int cl = lane % P, rg = lane / P;
#pragma unroll
    for (int i = 0; i < P; ++i) col[i] = stage[(P * rg + i) * PITCH + cl];
    __syncwarp();
    emit(h, cl, rg, col);
  }
}

// Column-wise MXFP8 of a 32 x 32 block (rows = lanes): each column is quantised with the scale of
// its 32 values; column c's 32 codes go to colT + c * ld, its scale to S[sf_row0 + c][sf_kb] of a
// tile-layout scale matrix with sf_KB columns.
template <int P>
__device__ __forceinline__ void colwise_mx(const float* v, float* stage, uint8_t* colT, int64_t ld, uint8_t* sf,
                                           int64_t sf_row0, int64_t sf_kb, int64_t sf_KB, int floor_rule, int e5m2) {
  column_passes<P>(v, stage, [&](int h, int cl, int rg, const float* col) {
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < P; ++i) m = max(m, __float_as_uint(col[i]) & 0x7FFFFFFFu);
#pragma unroll
    for (int s = P; s < 32; s <<= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, s));
    const uint32_t sb = e8m0_from_amax_bits(m, floor_rule, e5m2);
    const float inv = e8m0_inv_scale(sb);
    uint32_t w[P / 4];
#pragma unroll
    for (int i = 0; i < P / 4; ++i)
      w[i] = fp8x2(col[4 * i] * inv, col[4 * i + 1] * inv, e5m2) |
             (fp8x2(col[4 * i + 2] * inv, col[4 * i + 3] * inv, e5m2) << 16);
    const int c = P * h + cl;
    uint8_t* dst = colT + c * ld + P * rg;
    if constexpr (P == 16) {
      *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
    } else {
      static_assert(P == 8, "pass width");
      *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
    }
    if (rg == 0) sf[sf_mma_offset(sf_row0 + c, sf_kb, sf_KB)] = static_cast<uint8_t>(sb);
  });
}

// Column-wise bf16 of a 32 x 32 block: column c (32 bf16) goes to colT + c * ld.
template <int P>
__device__ __forceinline__ void colwise_bf16(const float* v, float* stage, bf16* colT, int64_t ld) {
  column_passes<P>(v, stage, [&](int h, int cl, int rg, const float* col) {
    uint4* dst = reinterpret_cast<uint4*>(colT + (P * h + cl) * ld + P * rg);
#pragma unroll
    for (int i = 0; i < P / 8; ++i) dst[i] = pack_bf16x8(col + 8 * i);
  });
}

__device__ __forceinline__ void load_acc32(uint32_t taddr, float* v) {
  uint32_t r[32];
  ptx::tmem_ld_32(taddr, r);
  ptx::tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

}  // namespace

template <bool MX, int EPI, class S>
__global__ void __launch_bounds__(S::NUM_THREADS, 1) grouped_gemm_kernel(const __grid_constant__ GemmArgs g) {
  __shared__ SharedState s;
  extern __shared__ uint8_t dyn_raw[];
  // 1024-byte aligned start, derived from the shared array itself (not through an integer) so
  // that the compiler keeps every access below in the shared state space
  uint8_t* smem = dyn_raw + ((1024u - (ptx::smem_u32(dyn_raw) & 1023u)) & 1023u);
  float* staging_base = reinterpret_cast<float*>(smem + S::OFF_STAGING);
  uint8_t* hbuf = smem + S::OFF_H;
  constexpr int BN = S::BN;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool K128 = MX || g.fp8;  // 8-bit operands: 128 K elements per 128-byte stage row
  // CTA pair: this CTA's rank (rank 0 issues the MMAs), the tile walkers are the pairs
  const uint32_t rank = S::PAIR ? ptx::cluster_ctarank() : 0u;
  const int NW = S::PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  const int WID = S::PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  constexpr int TILE_ROWS = S::PAIR ? 2 * BM : BM;

  // ---- set-up: tile prefix over experts, barriers, TMEM
  if (threadIdx.x == 0) {
    for (int e = 0; e <= g.E; ++e) s.poff[e] = g.poffsets[e];
    // tile list order: experts in id order, except for K-grouped GEMMs, whose tiles cost in
    // proportion to the expert's token count: there the experts go from most to fewest tokens
    // (stable insertion sort), so that skewed routing does not leave a tail of long tiles
    for (int i = 0; i < g.E; ++i) {
      int j = i;
      if (g.kgrouped) {
        const int P = s.poff[i + 1] - s.poff[i];
        while (j > 0 && s.poff[s.order[j - 1] + 1] - s.poff[s.order[j - 1]] < P) {
          s.order[j] = s.order[j - 1];
          --j;
        }
      }
      s.order[j] = i;
    }
    int acc = 0;
    for (int i = 0; i < g.E; ++i) {
      const int e = s.order[i];
      s.tile_prefix[i] = acc;
      acc += g.kgrouped ? (g.m_tiles * BM / TILE_ROWS) * g.n_tiles
                        : ((s.poff[e + 1] - s.poff[e] + TILE_ROWS - 1) / TILE_ROWS) * g.n_tiles;
    }
    s.tile_prefix[g.E] = acc;
    s.total1 = acc;
    if (EPI == EPI_FUSED_FWD) {  // the down tiles after all gate_up tiles
      int acc2 = 0;
      for (int e = 0; e < g.E; ++e) {
        s.tile_prefix2[e] = acc2;
        acc2 += ((s.poff[e + 1] - s.poff[e]) / BM) * g.n_tiles2;
      }
      s.tile_prefix2[g.E] = acc2;
      acc += acc2;
    }
    s.total_tiles = acc;
    s.abort_flag = 0;
    for (int i = 0; i < S::STAGES; ++i) {
      ptx::mbar_init(&s.full[i], 1);
      ptx::mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < S::NBUF; ++i) {
      ptx::mbar_init(&s.acc_full[i], 1);
      ptx::mbar_init(&s.acc_empty[i], S::EPI_WARPS * (S::PAIR ? 2 : 1));  // pair: both CTAs' epilogues
    }
    ptx::mbar_init(&s.drain, 1);
    ptx::mbar_init(&s.h_full, 1);
    ptx::mbar_init(&s.h_empty, S::EPI_WARPS);
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&g.tmap_a);
    ptx::prefetch_tmap(&g.tmap_b);
    if (EPI == EPI_FUSED_FWD) {
      ptx::prefetch_tmap(&g.tmap_a2);
      ptx::prefetch_tmap(&g.tmap_b2);
    }
    if (MX) {
      ptx::prefetch_tmap(&g.tmap_sfa);
      ptx::prefetch_tmap(&g.tmap_sfb);
    }
    if (S::HTILE) ptx::prefetch_tmap(&g.tmap_h);
  }
  if (warp == S::ALLOC_WARP) {
    if (S::PAIR) {
      ptx::tmem_alloc_pair(&s.tmem_base, TMEM_COLS);
      ptx::tmem_relinquish_pair();
    } else {
      ptx::tmem_alloc(&s.tmem_base, TMEM_COLS);
      ptx::tmem_relinquish();
    }
  }
  ptx::tc_fence_before();
  if (S::PAIR)
    ptx::cluster_sync();  // both CTAs' barriers initialised before any load or commit reaches them
  else
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
    uint32_t h_count = 0;
    bool h_issued = false;
    bool stalled = false;
    // bytes per stage; for a CTA pair rank 0's barrier counts both CTAs' loads
    const uint32_t tx = (S::A_BYTES + S::B_BYTES + (MX ? 512 + S::SFB_BYTES : 0)) * (S::PAIR ? 2 : 1);
    for (int i = 0, t = tile_of(0, NW, WID); t < total && !*abort_flag; t = tile_of(++i, NW, WID)) {
      Tile tl;
      decode_tile(t, s, g, K128, tl, TILE_ROWS);
      const int bk = K128 ? 128 : 64;
      if (EPI == EPI_FUSED_FWD && tl.down) {
        // the tile's 128 rows of a are complete once every gate_up tile of its row block has released them
        if (!ptx::wait_counter(g.mblock_done + tl.a_row / BM, g.n_tiles * S::EPI_WARPS, abort_flag, lim)) break;
        ptx::fence_proxy_async_global();  // TMA reads of what other CTAs wrote with ordinary stores
      }
      const CUtensorMap* map_a = tl.down ? &g.tmap_a2 : &g.tmap_a;
      const CUtensorMap* map_b = tl.down ? &g.tmap_b2 : &g.tmap_b;
      const CUtensorMap* map_sfa = tl.down ? &g.tmap_sfa2 : &g.tmap_sfa;
      const CUtensorMap* map_sfb = tl.down ? &g.tmap_sfb2 : &g.tmap_sfb;
      const int64_t sfb_rows = tl.down ? g.sfb_expert_rows2 : g.sfb_expert_rows;
      for (int kb = 0; kb < tl.nk; kb += S::KSUB) {
        if (g.stall_flag && !stalled && kb + S::KSUB > min(2, tl.nk - 1)) {  // test hook: a wait that can only expire
          stalled = true;
          if (!ptx::wait_flag(g.stall_flag, abort_flag, g.stall_limit)) break;
        }
        if (!ptx::mbar_wait(&s.empty[stage], phase ^ 1, abort_flag, lim)) break;
        uint8_t* st = smem + stage * S::STAGE_BYTES;
        const int kx = tl.k0 + kb * bk;
        if (S::PAIR) {
          // this CTA's 128 rows of A and half of the tile's B rows, all of its B scales, for the stage's
          // K blocks; completion counted on rank 0's barrier, which expects both CTAs' bytes
          const int nsub = min(S::KSUB, tl.nk - kb);
          if (rank == 0) ptx::mbar_arrive_expect_tx(&s.full[stage], tx * nsub);
          const int32_t arow = tl.a_row + static_cast<int32_t>(rank) * BM;
          const int32_t brow = tl.nb * BN + static_cast<int32_t>(rank) * (BN / 2);
          for (int j = 0; j < nsub; ++j) {
            uint8_t* blk = st + j * S::BLOCK_BYTES;
            const int kxj = kx + j * bk;
            ptx::tma_load_2d_pair(blk, map_a, kxj, arow, &s.full[stage]);
            if (!g.kgrouped)
              ptx::tma_load_3d_pair(blk + S::OFF_B, map_b, kxj, brow, tl.e, &s.full[stage]);
            else
              ptx::tma_load_2d_pair(blk + S::OFF_B, map_b, kxj, brow, &s.full[stage]);
            if (MX) {
              const int32_t kq = kxj / 128;
              const int64_t eb = g.kgrouped ? 0 : static_cast<int64_t>(tl.e) * sfb_rows;
              ptx::tma_load_3d_pair(blk + S::OFF_SFA, map_sfa, 0, kq, arow / 128, &s.full[stage]);
              ptx::tma_load_3d_pair(blk + S::OFF_SFB, map_sfb, 0, kq,
                                    static_cast<int32_t>((eb + static_cast<int64_t>(tl.nb) * BN) / 128),
                                    &s.full[stage]);
            }
          }
        } else {
          const int nsub = min(S::KSUB, tl.nk - kb);
          ptx::mbar_arrive_expect_tx(&s.full[stage], tx * nsub);
          for (int j = 0; j < nsub; ++j) {
            uint8_t* blk = st + j * S::BLOCK_BYTES;
            const int kxj = kx + j * bk;
            ptx::tma_load_2d(blk, map_a, kxj, tl.a_row, &s.full[stage]);
            if (!g.kgrouped && g.gate_up_half && !tl.down) {
              // bf16 gate_up: BN/2 gate rows then the matching BN/2 up rows of expert e
              ptx::tma_load_3d(blk + S::OFF_B, map_b, kxj, tl.nb * (BN / 2), tl.e, &s.full[stage]);
              ptx::tma_load_3d(blk + S::OFF_B + S::B_BYTES / 2, map_b, kxj, g.gate_up_half + tl.nb * (BN / 2), tl.e,
                               &s.full[stage]);
            } else if (!g.kgrouped) {  // one box of BN rows
              ptx::tma_load_3d(blk + S::OFF_B, map_b, kxj, tl.nb * BN, tl.e, &s.full[stage]);
            } else {
              ptx::tma_load_2d(blk + S::OFF_B, map_b, kxj, tl.nb * BN, &s.full[stage]);
            }
            if (MX) {  // this block's scale tiles: one of A, BN/128 consecutive ones of B
              const int32_t kq = kxj / 128;
              const int64_t eb = g.kgrouped ? 0 : static_cast<int64_t>(tl.e) * sfb_rows;
              ptx::tma_load_3d(blk + S::OFF_SFA, map_sfa, 0, kq, tl.a_row / 128, &s.full[stage]);
              ptx::tma_load_3d(blk + S::OFF_SFB, map_sfb, 0, kq,
                               static_cast<int32_t>((eb + static_cast<int64_t>(tl.nb) * BN) / 128), &s.full[stage]);
            }
          }
        }
        issued_mask |= 1u << stage;
        last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == S::STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (S::HTILE && !*abort_flag) {
        // the tile's saved gate/up columns, once the epilogue has finished with the previous tile's
        if (!ptx::mbar_wait(&s.h_empty, (h_count & 1) ^ 1, abort_flag, lim)) break;
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        ptx::mbar_arrive_expect_tx(&s.h_full, S::H_BYTES);
        const int32_t hr = tl.a_row, gc = tl.nb * BN;
#pragma unroll
        for (int i = 0; i < BN / 64; ++i) {
          ptx::tma_load_2d(hbuf + i * 16384, &g.tmap_h, gc + 64 * i, hr, &s.h_full);
          ptx::tma_load_2d(hbuf + (BN / 64 + i) * 16384, &g.tmap_h, static_cast<int32_t>(g.epi.f) + gc + 64 * i, hr,
                           &s.h_full);
        }
        h_issued = true;
        ++h_count;
      }
    }
    if (S::HTILE && h_issued) {  // the last h tile must have landed before the CTA exits
      volatile int never = 0;
      ptx::mbar_wait(&s.h_full, (h_count - 1) & 1, &never, lim);
    }
    // wait for the loads still in flight (only possible after an abort; a pair's rank 1 has no
    // barrier of its own to wait on: rank 0's waits and the final cluster barrier cover it)
    for (int i = 0; i < S::STAGES; ++i)
      if ((!S::PAIR || rank == 0) && (issued_mask & (1u << i))) {
        volatile int never = 0;
        ptx::mbar_wait(&s.full[i], (last_parity >> i) & 1u, &never, lim);
      }
  } else if (S::PAIR && rank != 0 && warp == 1 && lane == 0) {
    // pair rank 1: rank 0 issues the MMAs for both CTAs; its final commit arrives here once they have
    // all completed, before this CTA's TMEM is freed
    volatile int never = 0;
    ptx::mbar_wait(&s.drain, 0, &never, lim);
  } else if (warp == 1 && lane == 0) {
    // ================= MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    int local = 0;  // tiles with MMAs issued by this CTA
    bool issued_any = false;
    // descriptors of stage 0; stage s adds s * STAGE_BYTES / 16 to the 14-bit start-address field
    // (shared addresses stay below 2^18, so the sum never carries out of it)
    const uint32_t smem0 = ptx::smem_u32(smem);
    const uint64_t adesc0 = ptx::smem_desc(smem0, 16, 1024, ptx::kSwizzle128B);
    const uint64_t bdesc0 = ptx::smem_desc(smem0 + S::OFF_B, 16, 1024, ptx::kSwizzle128B);
    const uint64_t sfadesc0 = ptx::smem_desc(smem0 + S::OFF_SFA, 0, 128, ptx::kSwizzleNone);
    const uint64_t sfbdesc0 = ptx::smem_desc(smem0 + S::OFF_SFB, 0, 128, ptx::kSwizzleNone);
    const uint32_t a_fmt = ptx::idesc_a_format(g.a_e5m2 ? ptx::kFmtE5M2 : ptx::kFmtE4M3);  // A's element format
    for (int i = 0, t = tile_of(0, NW, WID); t < total && !*abort_flag; t = tile_of(++i, NW, WID)) {
      Tile tl;
      decode_tile(t, s, g, K128, tl, TILE_ROWS);
      if (tl.nk == 0) continue;
      const int buf = S::NBUF == 2 ? (local & 1) : 0;
      const uint32_t acc_par = static_cast<uint32_t>((S::NBUF == 2 ? (local >> 1) : local) & 1);
      if (!ptx::mbar_wait(&s.acc_empty[buf], acc_par ^ 1, abort_flag, lim)) break;
      ptx::tc_fence_after();
      const uint32_t d_tmem = tmem + static_cast<uint32_t>(buf * BN);
      bool ok = true;
      for (int kb = 0; kb < tl.nk; kb += S::KSUB) {
        if (!ptx::mbar_wait(&s.full[stage], phase, abort_flag, lim)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint64_t soff = static_cast<uint64_t>(stage * (S::STAGE_BYTES >> 4));
        const uint64_t adesc = adesc0 + soff;
        const uint64_t bdesc = bdesc0 + soff;
        if (S::PAIR) {
          // per K block of the stage: both CTAs' scale tiles into their own TMEM, then M = 256 MMAs
          // over both CTAs' operands
          const int nsub = min(S::KSUB, tl.nk - kb);
          for (int j = 0; j < nsub; ++j) {
            const uint64_t boff = soff + static_cast<uint64_t>(j * (S::BLOCK_BYTES >> 4));
            const uint32_t acc = ((kb + j) != 0) ? 1u : 0u;  // the tile's first block overwrites D
            if (MX) {
              const uint32_t sfa_t = tmem + S::SF_TMEM_COL + S::SF_COLS * (stage * S::KSUB + j);
              const uint32_t sfb_t = sfa_t + 4;
              ptx::tc_cp_32x128b_warpx4_pair(sfa_t, sfadesc0 + boff);
#pragma unroll
              for (int i = 0; i < BN / 128; ++i)
                ptx::tc_cp_32x128b_warpx4_pair(sfb_t + 4 * i, sfbdesc0 + boff + 32 * i);
#pragma unroll
              for (int k = 0; k < 4; ++k)
                ptx::tc_mma_mxf8_pair(d_tmem, adesc0 + boff + 2 * k, bdesc0 + boff + 2 * k,
                                      ptx::idesc_mxf8(2 * BM, BN, k, k) | a_fmt, sfa_t, sfb_t, acc | k);
            } else if (g.fp8) {
#pragma unroll
              for (int k = 0; k < 4; ++k)
                ptx::tc_mma_f8_pair(d_tmem, adesc0 + boff + 2 * k, bdesc0 + boff + 2 * k,
                                    ptx::idesc_f8(2 * BM, BN) | a_fmt, acc | k);
            } else {
#pragma unroll
              for (int k = 0; k < 4; ++k)
                ptx::tc_mma_bf16_pair(d_tmem, adesc0 + boff + 2 * k, bdesc0 + boff + 2 * k, ptx::idesc_bf16(2 * BM, BN),
                                      acc | k);
            }
          }
        } else {
          const int nsub = min(S::KSUB, tl.nk - kb);
          for (int j = 0; j < nsub; ++j) {
            const uint64_t boff = static_cast<uint64_t>(j * (S::BLOCK_BYTES >> 4));
            const uint32_t acc = ((kb + j) != 0) ? 1u : 0u;  // the tile's first block overwrites D
            if (MX) {
              const uint32_t sfa_t = tmem + S::SF_TMEM_COL + S::SF_COLS * (stage * S::KSUB + j);
              const uint32_t sfb_t = sfa_t + 4;
              ptx::tc_cp_32x128b_warpx4(sfa_t, sfadesc0 + soff + boff);
#pragma unroll
              for (int i = 0; i < BN / 128; ++i)
                ptx::tc_cp_32x128b_warpx4(sfb_t + 4 * i, sfbdesc0 + soff + boff + 32 * i);
#pragma unroll
              for (int k = 0; k < 4; ++k)
                ptx::tc_mma_mxf8(d_tmem, adesc + boff + 2 * k, bdesc + boff + 2 * k,
                                 ptx::idesc_mxf8(BM, BN, k, k) | a_fmt, sfa_t, sfb_t, acc | k);
            } else if (g.fp8) {
#pragma unroll
              for (int k = 0; k < 4; ++k)
                ptx::tc_mma_f8(d_tmem, adesc + boff + 2 * k, bdesc + boff + 2 * k, ptx::idesc_f8(BM, BN) | a_fmt,
                               acc | k);
            } else {
#pragma unroll
              for (int k = 0; k < 4; ++k)
                ptx::tc_mma_bf16(d_tmem, adesc + boff + 2 * k, bdesc + boff + 2 * k, ptx::idesc_bf16(BM, BN), acc | k);
            }
          }
        }
        if (S::PAIR)
          ptx::tc_commit_pair(&s.empty[stage]);  // frees the stage in both CTAs
        else
          ptx::tc_commit(&s.empty[stage]);
        issued_any = true;
        if (++stage == S::STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      if (S::PAIR)
        ptx::tc_commit_pair(&s.acc_full[buf]);  // both CTAs' epilogues
      else
        ptx::tc_commit(&s.acc_full[buf]);
      ++local;
    }
    if (S::PAIR) {  // always, so that rank 1's wait for it ends
      ptx::tc_commit_pair(&s.drain);
      volatile int never = 0;
      ptx::mbar_wait(&s.drain, 0, &never, lim);
    } else if (issued_any) {  // all MMAs of this CTA complete before TMEM can be released
      ptx::tc_commit(&s.drain);
      volatile int never = 0;
      ptx::mbar_wait(&s.drain, 0, &never, lim);
    }
  } else if (warp >= S::LEAD) {
    // ================= epilogue
    const int q = warp & 3;               // TMEM lane quadrant this warp may read
    const int ch = (warp - S::LEAD) >> 2;  // which of the quadrant's EPI_WARPS/4 column parts this warp owns
    constexpr int NPART = S::EPI_WARPS / 4;
    float* stage_buf = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(staging_base) +
                                                (warp - S::LEAD) * S::STAGING_PER_WARP);
    const EpiArgs& ep = g.epi;
    int local = 0;
    // hand the accumulator back to the MMA issuer (a pair's issuer is rank 0: its barrier counts the
    // epilogue warps of both CTAs)
    auto release_acc = [&](int b) {
      if (S::PAIR)
        ptx::mbar_arrive_leader(&s.acc_empty[b]);
      else
        ptx::mbar_arrive(&s.acc_empty[b]);
    };
    // per-tensor FP8: this warp's largest magnitude written for expert amax_e so far (bf16 bits),
    // added to ep.amax_out[amax_e] when the expert changes and at the end
    uint32_t amax_run = 0;
    int amax_e = -1;
    auto amax_flush = [&]() {
      if (MX || !ep.amax_out || amax_e < 0) return;
      const unsigned mask = __activemask();
      const uint32_t m = __reduce_max_sync(mask, amax_run);
      if (lane == __ffs(mask) - 1 && m) atomicMax(ep.amax_out + amax_e, m << 16);
    };
    for (int i = 0, t = tile_of(0, NW, WID); t < total && !*abort_flag; t = tile_of(++i, NW, WID)) {
      Tile tl;
      decode_tile(t, s, g, K128, tl, TILE_ROWS);
      const int64_t row_w = tl.a_row + (S::PAIR ? static_cast<int>(rank) * BM : 0) + 32 * q;  // first row of this warp
      const int64_t row = row_w + lane;
      // per-tensor FP8: the accumulator times 1/s_a * 1/s_b of the tile's expert
      float fac = 1.f;
      if (!MX && g.pt_amax_a)
        fac = __frcp_rn(fp8_tensor_scale(g.pt_amax_a[tl.e], g.a_e5m2)) * __frcp_rn(fp8_tensor_scale(g.pt_amax_b[tl.e], 0));
      if (!MX && ep.amax_out && tl.e != amax_e) {
        amax_flush();
        amax_e = tl.e;
        amax_run = 0;
      }
      if (tl.nk == 0) {
        // K-grouped expert without tokens: its weight gradient is zero
        if (EPI == EPI_STORE) {
          bf16* out = static_cast<bf16*>(const_cast<void*>(ep.out_ptrs.p[tl.e]));
          const int64_t c0 = static_cast<int64_t>(tl.nb) * BN + (BN / NPART) * ch;
          uint4* dst = reinterpret_cast<uint4*>(out + row * ep.ldo + c0);
#pragma unroll 4
          for (int i = 0; i < BN / NPART / 8; ++i) dst[i] = make_uint4(0, 0, 0, 0);
        }
        continue;
      }
      const int buf = S::NBUF == 2 ? (local & 1) : 0;
      const uint32_t acc_par = static_cast<uint32_t>((S::NBUF == 2 ? (local >> 1) : local) & 1);
      ++local;

      if (EPI == EPI_STORE || (EPI == EPI_FUSED_FWD && tl.down)) {
        // drain the accumulator into packed bf16, release it, then store
        if (!ptx::mbar_wait(&s.acc_full[buf], acc_par, abort_flag, lim)) break;
        ptx::tc_fence_after();
        const uint32_t t_lane = tmem + static_cast<uint32_t>(buf * BN) + (static_cast<uint32_t>(32 * q) << 16);
        constexpr int CPT = BN / NPART;  // columns per thread
        uint32_t pk[CPT / 2];
#pragma unroll
        for (int cc = 0; cc < CPT / 32; ++cc) {
          float v[32];
          load_acc32(t_lane + CPT * ch + 32 * cc, v);
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[16 * cc + i] = pack_bf16x2(v[2 * i] * fac, v[2 * i + 1] * fac);
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) release_acc(buf);
        if (S::PAIR && rank != 0 && !tl.hi_ok) continue;  // the expert ends in the pair tile's first half
        bf16* out = g.kgrouped ? static_cast<bf16*>(const_cast<void*>(ep.out_ptrs.p[tl.e])) : ep.out;
        bf16* orow = out + row * ep.ldo + static_cast<int64_t>(tl.nb) * BN + CPT * ch;
        if ((reinterpret_cast<uintptr_t>(out) & 31u) == 0 && (ep.ldo & 15) == 0) {  // whole 32-byte sectors
#pragma unroll
          for (int i = 0; i < CPT / 16; ++i)
            ptx::st_global_v8(orow + 16 * i, make_uint4(pk[8 * i], pk[8 * i + 1], pk[8 * i + 2], pk[8 * i + 3]),
                              make_uint4(pk[8 * i + 4], pk[8 * i + 5], pk[8 * i + 6], pk[8 * i + 7]));
        } else {
          uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
          for (int i = 0; i < CPT / 8; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      } else if (EPI == EPI_SWIGLU || EPI == EPI_FUSED_FWD) {
        // tile = BN/2 output columns; accumulator columns [0,BN/2) gate, [BN/2,BN) up
        constexpr int OPT = BN / 2 / NPART;  // output columns per thread
        constexpr int G = OPT / 32;          // groups of 32 output columns per thread
        if (!ptx::mbar_wait(&s.acc_full[buf], acc_par, abort_flag, lim)) break;
        if (S::PAIR && rank != 0 && !tl.hi_ok) {  // the expert ends in the pair tile's first half
          ptx::tc_fence_after();
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) release_acc(buf);
          continue;
        }
        const float p = ep.p_perm[row];
        const int64_t f = ep.f;
        ptx::tc_fence_after();
        const uint32_t t_lane = tmem + static_cast<uint32_t>(buf * BN) + (static_cast<uint32_t>(32 * q) << 16);
#pragma unroll 1
        for (int cc = 0; cc < G; ++cc) {
          const int64_t j = static_cast<int64_t>(tl.nb) * (BN / 2) + OPT * ch + 32 * cc;  // 32 output columns
          float gv[32], uv[32];
          load_acc32(t_lane + OPT * ch + 32 * cc, gv);
          load_acc32(t_lane + BN / 2 + OPT * ch + 32 * cc, uv);
          if (!MX) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              gv[i] *= fac;
              uv[i] *= fac;
            }
          }
          if (cc == G - 1) {
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) release_acc(buf);
          }
          if (ep.h_q) {  // saved as MXFP8: 32 codes and one scale per 32 gate (and up) values
            const uint32_t sbg = quant32_store(gv, ep.h_q + row * 2 * f + j, ep.scale_floor, 0);
            const uint32_t sbu = quant32_store(uv, ep.h_q + row * 2 * f + f + j, ep.scale_floor, 0);
            ep.h_s[row * (2 * f / 32) + j / 32] = static_cast<uint8_t>(sbg);
            ep.h_s[row * (2 * f / 32) + (f + j) / 32] = static_cast<uint8_t>(sbu);
          } else if (ep.h) {  // saved gate/up pre-activations: 64 bytes of each per row, in 32-byte stores
            bf16* hg = ep.h + row * 2 * f + j;
            bf16* hu = hg + f;
#pragma unroll
            for (int i = 0; i < 2; ++i) ptx::st_global_v8(hg + 16 * i, pack_bf16x8(gv + 16 * i), pack_bf16x8(gv + 16 * i + 8));
#pragma unroll
            for (int i = 0; i < 2; ++i) ptx::st_global_v8(hu + 16 * i, pack_bf16x8(uv + 16 * i), pack_bf16x8(uv + 16 * i + 8));
          }
          if (!ep.q_row && !ep.o_row) continue;  // h only (the backward recomputing h)
#pragma unroll
          for (int i = 0; i < 32; ++i) gv[i] = gv[i] * sigmoid_f(gv[i]) * uv[i] * p;  // a, in place
          if (ep.dump) {
            float4* dd = reinterpret_cast<float4*>(ep.dump + row * f + j);
#pragma unroll
            for (int i = 0; i < 8; ++i) dd[i] = make_float4(gv[4 * i], gv[4 * i + 1], gv[4 * i + 2], gv[4 * i + 3]);
          }
          if (MX) {
            const uint32_t sb = quant32_store(gv, ep.q_row + row * f + j, ep.scale_floor, 0);
            ep.s_row[sf_mma_offset(row, j / 32, f / 32)] = static_cast<uint8_t>(sb);
            if (ep.q_colT)
              colwise_mx<S::PASS>(gv, stage_buf, ep.q_colT + j * ep.cap + row_w, ep.cap, ep.s_colT, j, row_w / 32,
                                  ep.cap / 32, ep.scale_floor, 0);
          } else {
            bf16* dst = ep.o_row + row * f + j;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const uint4 lo = pack_bf16x8(gv + 16 * i), hi = pack_bf16x8(gv + 16 * i + 8);
              ptx::st_global_v8(dst + 16 * i, lo, hi);
              if (ep.amax_out) amax_run = max(amax_run, max(absmax_bf16x8_bits(lo), absmax_bf16x8_bits(hi)));
            }
            if (ep.o_colT) colwise_bf16<S::PASS>(gv, stage_buf, ep.o_colT + j * ep.cap + row_w, ep.cap);
          }
        }
        if (EPI == EPI_FUSED_FWD) {
          // this warp's share of the tile's rows of a (codes and scales) is written: release it to the
          // down tiles of the row block (every lane's stores, then one GPU-scope fence and count)
          __syncwarp();
          if (lane == 0) {
            __threadfence();
            atomicAdd(g.mblock_done + tl.a_row / BM, 1);
          }
        }
      } else {  // EPI_DSWIGLU: tile = BN f-columns of da; this thread owns BN/2 of them
        constexpr int CPT = BN / NPART;  // da columns per thread
        constexpr int G = CPT / 32;      // groups of 32 columns per thread
        const float p = ep.p_perm[row];
        const int64_t f = ep.f, f2 = 2 * ep.f;
        const int64_t j0 = static_cast<int64_t>(tl.nb) * BN + CPT * ch;
        const bool mxh = !S::HTILE && ep.h_q != nullptr;  // h saved as MXFP8
        const bf16* hrow = ep.h + row * f2;
        // saved gate/up values: 16-byte chunk c (of this thread's 32-column group cc) of the gate part
        // and of the up part, from the TMA-staged tile in smem (128B-swizzled rows) or from global.
        // MXFP8 h: chunks 0 and 1 are the group's 32 codes, chunk 2 holds its scale byte.
        const int rl = 32 * q + lane;  // row within the tile
        auto h_chunk = [&](int up, int cc, int c) -> uint4 {
          if (S::HTILE) {
            const int col = CPT * ch + 32 * cc + 8 * c;  // column within the tile's gate (or up) part
            const uint8_t* box = hbuf + (up * (BN / 64) + col / 64) * 16384;
            const int chunk = ((col % 64) / 8) ^ (rl & 7);
            return *reinterpret_cast<const uint4*>(box + rl * 128 + chunk * 16);
          }
          if (mxh) {
            const int64_t col = (up ? f : 0) + j0 + 32 * cc;
            if (c < 2) return reinterpret_cast<const uint4*>(ep.h_q + row * f2 + col)[c];
            if (c == 2) return make_uint4(ep.h_s[row * (f2 / 32) + col / 32], 0u, 0u, 0u);
            return make_uint4(0u, 0u, 0u, 0u);
          }
          return reinterpret_cast<const uint4*>(hrow + (up ? f : 0) + j0 + 32 * cc)[c];
        };
        // eight gate (or up) values of chunk i from the group's raw chunks
        auto h_values = [&](const uint4 (&hv)[4], int i, float* o) {
          if (mxh) {
            const uint4 c = hv[i >> 1];
            e4m3x8_to_float((i & 1) ? c.z : c.x, (i & 1) ? c.w : c.y, e8m0_scale(hv[2].x), o);
          } else {
            unpack_bf16x8(hv[i], o);
          }
        };
        uint4 hg[4], hu[4];
        if (!S::HTILE) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {  // saved gate/up values of the first group, before the wait
            hg[i] = h_chunk(0, 0, i);
            hu[i] = h_chunk(1, 0, i);
          }
        }
        if (!ptx::mbar_wait(&s.acc_full[buf], acc_par, abort_flag, lim)) break;
        if (S::HTILE) {
          if (!ptx::mbar_wait(&s.h_full, static_cast<uint32_t>((local - 1) & 1), abort_flag, lim)) break;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            hg[i] = h_chunk(0, 0, i);
            hu[i] = h_chunk(1, 0, i);
          }
        }
        ptx::tc_fence_after();
        const uint32_t t_lane = tmem + static_cast<uint32_t>(buf * BN) + (static_cast<uint32_t>(32 * q) << 16);
        float dp = 0.f;
#pragma unroll 1
        for (int cc = 0; cc < G; ++cc) {
          const int64_t j = j0 + 32 * cc;
          float da[32];
          load_acc32(t_lane + CPT * ch + 32 * cc, da);
          if (!MX) {
#pragma unroll
            for (int i = 0; i < 32; ++i) da[i] *= fac;
          }
          if (cc == G - 1) {
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) release_acc(buf);
          }
          float dg[32], du[32];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float gg[8], uu[8];
            h_values(hg, i, gg);
            h_values(hu, i, uu);
#pragma unroll
            for (int q8 = 0; q8 < 8; ++q8) {
              const float gx = gg[q8], ux = uu[q8], d = da[8 * i + q8];
              const float sg = sigmoid_f(gx);
              const float sl = gx * sg;
              dg[8 * i + q8] = d * p * ux * sg * (1.0f + gx * (1.0f - sg));
              du[8 * i + q8] = d * p * sl;
              dp += d * sl * ux;
            }
          }
          if (cc < G - 1) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {  // next group's saved values
              hg[i] = h_chunk(0, cc + 1, i);
              hu[i] = h_chunk(1, cc + 1, i);
            }
          } else if (S::HTILE) {  // done with the staged h tile: the producer may refill it
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&s.h_empty);
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
            // the gradient's element format as a constant inside each branch: one conversion
            // instruction per pair of values instead of both formats' and a select
            auto requant = [&](auto e5) {
              constexpr int E5 = decltype(e5)::value;
              uint32_t sb = quant32_store(dg, ep.q_row + row * f2 + j, ep.scale_floor, E5);
              ep.s_row[sf_mma_offset(row, j / 32, f2 / 32)] = static_cast<uint8_t>(sb);
              sb = quant32_store(du, ep.q_row + row * f2 + f + j, ep.scale_floor, E5);
              ep.s_row[sf_mma_offset(row, (f + j) / 32, f2 / 32)] = static_cast<uint8_t>(sb);
              colwise_mx<S::PASS>(dg, stage_buf, ep.q_colT + j * ep.cap + row_w, ep.cap, ep.s_colT, j, row_w / 32,
                                  ep.cap / 32, ep.scale_floor, E5);
              colwise_mx<S::PASS>(du, stage_buf, ep.q_colT + (f + j) * ep.cap + row_w, ep.cap, ep.s_colT, f + j,
                                  row_w / 32, ep.cap / 32, ep.scale_floor, E5);
            };
            if (ep.grad_e5m2)
              requant(std::integral_constant<int, 1>{});
            else
              requant(std::integral_constant<int, 0>{});
          } else {
            bf16* d0 = ep.o_row + row * f2 + j;
            bf16* d1 = d0 + f;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const uint4 g0 = pack_bf16x8(dg + 16 * i), g1 = pack_bf16x8(dg + 16 * i + 8);
              const uint4 u0 = pack_bf16x8(du + 16 * i), u1 = pack_bf16x8(du + 16 * i + 8);
              ptx::st_global_v8(d0 + 16 * i, g0, g1);
              ptx::st_global_v8(d1 + 16 * i, u0, u1);
              if (ep.amax_out)
                amax_run = max(amax_run, max(max(absmax_bf16x8_bits(g0), absmax_bf16x8_bits(g1)),
                                             max(absmax_bf16x8_bits(u0), absmax_bf16x8_bits(u1))));
            }
            if (ep.o_colT) {
              colwise_bf16<S::PASS>(dg, stage_buf, ep.o_colT + j * ep.cap + row_w, ep.cap);
              colwise_bf16<S::PASS>(du, stage_buf, ep.o_colT + (f + j) * ep.cap + row_w, ep.cap);
            }
          }
        }
        ep.dp_part[(static_cast<int64_t>(tl.nb) * NPART + ch) * ep.cap + row] = dp;
      }
    }
    amax_flush();
  }

  __syncthreads();
  if (threadIdx.x == 0 && s.abort_flag) atomicOr(g.status, kStatusTimeout);
  if (S::PAIR) ptx::cluster_sync();  // no arrival from the other CTA can still be on its way here
  if (warp == S::ALLOC_WARP) {
    ptx::tc_fence_after();
    if (S::PAIR)
      ptx::tmem_dealloc_pair(tmem, TMEM_COLS);
    else
      ptx::tmem_dealloc(tmem, TMEM_COLS);
  }
}

namespace {
template <bool MX, int EPI, class S>
cudaError_t launch_t(const GemmArgs& args, int num_sms, cudaStream_t st) {
  auto kern = grouped_gemm_kernel<MX, EPI, S>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM_DYN);
  if (e != cudaSuccess) return e;
  if (S::PAIR) {
    // clusters of two CTAs, as many pairs as can be resident at once (one CTA per SM)
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(num_sms & ~1));
    cfg.blockDim = dim3(S::NUM_THREADS);
    cfg.dynamicSmemBytes = S::SMEM_DYN;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // the occupancy query once per device (a host call of some microseconds)
    static int resident[64] = {};
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int clusters = (dev >= 0 && dev < 64) ? resident[dev] : 0;
    if (clusters < 1) {
      e = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg);
      if (e != cudaSuccess) return e;
      if (clusters < 1) return cudaErrorInvalidConfiguration;
      if (dev >= 0 && dev < 64) resident[dev] = clusters;
    }
    cfg.gridDim = dim3(static_cast<unsigned>(2 * std::min(clusters, num_sms / 2)));
    return cudaLaunchKernelEx(&cfg, kern, args);
  }
  kern<<<num_sms, S::NUM_THREADS, S::SMEM_DYN, st>>>(args);
  return cudaGetLastError();
}
}  // namespace

// Rows of B one CTA loads per stage (its tensor-map box): the tile's N, or half of it for CTA pairs.
int gemm_b_box_rows(bool mx, int epi) {
  if (epi == EPI_STORE) return ShapeStorePair::BN / 2;
  return gemm_tile_n(epi);
}

int gemm_tile_n(int epi) {
  return epi == EPI_STORE ? ShapeStorePair::BN
                          : ((epi == EPI_SWIGLU || epi == EPI_FUSED_FWD) ? ShapeSwiglu::BN : ShapeDswiglu::BN);
}

int gemm_dswiglu_parts() { return ShapeDswiglu::EPI_WARPS / 4; }

cudaError_t launch_grouped_gemm(const GemmArgs& args, bool mx, int epi, int num_sms, cudaStream_t st) {
  if (mx) {
    if (epi == EPI_STORE) return launch_t<true, EPI_STORE, ShapeStorePair>(args, num_sms, st);
    if (epi == EPI_SWIGLU) return launch_t<true, EPI_SWIGLU, ShapeSwiglu>(args, num_sms, st);
    if (epi == EPI_FUSED_FWD) return launch_t<true, EPI_FUSED_FWD, ShapeSwiglu>(args, num_sms, st);
    if (args.epi.h_q) return launch_t<true, EPI_DSWIGLU, ShapeDswigluG>(args, num_sms, st);
    return launch_t<true, EPI_DSWIGLU, ShapeDswiglu>(args, num_sms, st);
  }
  if (epi == EPI_STORE) return launch_t<false, EPI_STORE, ShapeStorePair>(args, num_sms, st);
  if (epi == EPI_SWIGLU) return launch_t<false, EPI_SWIGLU, ShapeSwiglu>(args, num_sms, st);
  if (epi == EPI_FUSED_FWD) return launch_t<false, EPI_FUSED_FWD, ShapeSwiglu>(args, num_sms, st);
  return launch_t<false, EPI_DSWIGLU, ShapeDswiglu>(args, num_sms, st);
}

}  // namespace moemx
