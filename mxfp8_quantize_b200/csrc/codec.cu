// HBM-bound kernels of the grouped MoE MLP: routing bookkeeping, MXFP8 quantisation (with the
// token gather fused in), the bf16 gather/transpose used by the BF16 path, the combine of
// expert rows back to tokens, and the reduction of the routing-probability gradient.
#include <cuda_fp8.h>

#include "codec.cuh"
#include "ptx_sm100.cuh"

namespace moemx {

// ------------------------------------------------------------------------------------------
// Routing: stable counting sort of the T*k slots by expert (sitech.ge "Grouped experts instead
// of a Python loop": per-expert token counts drive one grouped call).  One CTA of 1024 threads;
// warp w owns a contiguous run of slots, so counting per (warp, expert) and an exclusive scan
// over warps gives every slot its stable position without atomics.
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(1024, 1)
route_kernel(const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_prob, int Tk, int E,
             int capacity, const int32_t* __restrict__ split_in, int32_t* __restrict__ split_out,
             int32_t* __restrict__ poffsets, int32_t* __restrict__ sorted_to_src, int32_t* __restrict__ src_to_sorted,
             float* __restrict__ prob_perm, int* __restrict__ status) {
  extern __shared__ int32_t sm[];      // [32][E] per-warp counts, then running bases
  __shared__ int32_t s_poff[MOE_MAX_EXPERTS + 1];
  __shared__ int s_bad;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int32_t* wcnt = sm;

  for (int i = tid; i < 32 * E; i += blockDim.x) wcnt[i] = 0;
  if (tid == 0) s_bad = 0;
  for (int i = tid; i < capacity; i += blockDim.x) {
    sorted_to_src[i] = -1;
    if (prob_perm) prob_perm[i] = 0.f;
  }
  __syncthreads();

  const int per_warp = static_cast<int>(round_up(ceil_div(Tk, 32), 32));
  const int lo = warp * per_warp;
  const int hi = min(Tk, lo + per_warp);
  const unsigned lt_mask = (1u << lane) - 1u;

  // pass 1: per-warp histograms (each lane loads RB slots of a chunk before using any)
  constexpr int RB = 16;
  for (int base = lo; base < hi; base += 32 * RB) {
    int ev[RB];
#pragma unroll
    for (int i = 0; i < RB; ++i) {
      const int s = base + 32 * i + lane;
      ev[i] = s < hi ? topk_idx[s] : -1;
    }
#pragma unroll
    for (int i = 0; i < RB; ++i) {
      const int s = base + 32 * i + lane;
      int e = ev[i];
      if (s < hi && (e < 0 || e >= E)) {
        s_bad = 1;
        e = -1;
      }
      const unsigned peers = __match_any_sync(0xffffffffu, e);
      if (e >= 0 && (peers & lt_mask) == 0) wcnt[warp * E + e] += __popc(peers);
      __syncwarp();
    }
  }
  __syncthreads();

  // exclusive scan over warps per expert; totals
  for (int e = tid; e < E; e += blockDim.x) {
    int run = 0;
    for (int w = 0; w < 32; ++w) {
      const int c = wcnt[w * E + e];
      wcnt[w * E + e] = run;
      run += c;
    }
    split_out[e] = run;
    if (split_in && split_in[e] != run) s_bad = 1;
  }
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int e = 0; e < E; ++e) {
      s_poff[e] = acc;
      acc += static_cast<int>(round_up(split_out[e], MOE_ROW_ALIGN));
    }
    s_poff[E] = acc;
  }
  __syncthreads();
  for (int e = tid; e <= E; e += blockDim.x) poffsets[e] = s_poff[e];
  if (tid == 0 && s_bad) atomicOr(status, kStatusDevice);

  // pass 2: positions (same chunking)
  for (int base = lo; base < hi; base += 32 * RB) {
    int ev[RB];
#pragma unroll
    for (int i = 0; i < RB; ++i) {
      const int s = base + 32 * i + lane;
      ev[i] = s < hi ? topk_idx[s] : -1;
    }
#pragma unroll
    for (int i = 0; i < RB; ++i) {
      const int s = base + 32 * i + lane;
      int e = ev[i];
      if (e < 0 || e >= E) e = -1;
      const unsigned peers = __match_any_sync(0xffffffffu, e);
      int pos = -1;
      if (e >= 0) pos = s_poff[e] + wcnt[warp * E + e] + __popc(peers & lt_mask);
      __syncwarp();
      if (e >= 0 && (peers & lt_mask) == 0) wcnt[warp * E + e] += __popc(peers);
      __syncwarp();
      if (e >= 0) {
        sorted_to_src[pos] = s;
        src_to_sorted[s] = pos;
        if (prob_perm) prob_perm[pos] = topk_prob[s];
      } else if (s < hi) {
        src_to_sorted[s] = -1;
      }
    }
  }
}

// ------------------------------------------------------------------------------------------
// Quantise / gather / transpose tiles of 128 rows x 128 columns (256 threads).
//   MXFP8 mode: row-wise codes + scales (blocks of 32 along a row) and column-wise codes +
//               scales (blocks of 32 down a column) written transposed, from one read of x.
//   BF16 mode:  the gathered rows copied, and/or written transposed.
// The source row of output row r is r itself, or, when ``sorted_to_src`` is given, token
// sorted_to_src[r] / k (padding rows, -1, read as zeros).  Every thread issues its 8 loads before
// using any; the column pass writes whole 128-byte lines of the transposed output.
// ------------------------------------------------------------------------------------------
namespace {
constexpr int QT_ROWS = 128;
constexpr int QT_COLS = 128;
constexpr int QT_PITCH = QT_COLS + 8;  // bf16 elements per smem row (padding against bank conflicts)
constexpr int QT_LOADS = QT_ROWS * QT_COLS / 8 / 256;

// |a| and |b| of two bf16 pairs, max per half (max.bf16x2); inputs are finite.
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b) {
  a &= 0x7FFF7FFFu;
  b &= 0x7FFF7FFFu;
  __nv_bfloat162 r = __hmax2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
// fp32 bits of the larger half of a bf16 pair of non-negative values
__device__ __forceinline__ uint32_t fold_halves(uint32_t m2) { return max(m2 << 16, m2 & 0xFFFF0000u); }

}  // namespace

// Column-wise outputs of one thread: columns (2p, 2p+1) of the tile and 32-row block rb (each smem
// word holds one row of both columns).  Scales go to the block's 512-byte scale tile in smem when
// the tensor-core layout is requested, else straight to the row-major scale matrix.
__device__ __forceinline__ void column_pass(const QuantArgs& a, const uint32_t* tile, int p, int rb, int64_t gc,
                                            int64_t gr, int b, uint8_t* satom_col, uint8_t* qcol_tile) {
  const int64_t R = a.rows, C = a.cols, KBc = R / 32;
  uint32_t wv[32];
  uint32_t m2 = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    wv[i] = tile[(rb * 32 + i) * (QT_PITCH / 2) + p];
    m2 = absmax_bf16x2(m2, wv[i]);
  }
  if (a.mx) {
    const uint32_t sb0 = e8m0_from_amax_bits(m2 << 16, a.scale_floor, a.e5m2);
    const uint32_t sb1 = e8m0_from_amax_bits(m2 & 0xFFFF0000u, a.scale_floor, a.e5m2);
    const float inv0 = e8m0_inv_scale(sb0), inv1 = e8m0_inv_scale(sb1);
    uint32_t q0[8], q1[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t lo0 = fp8x2(__uint_as_float(wv[4 * i] << 16) * inv0, __uint_as_float(wv[4 * i + 1] << 16) * inv0, a.e5m2);
      const uint32_t hi0 =
          fp8x2(__uint_as_float(wv[4 * i + 2] << 16) * inv0, __uint_as_float(wv[4 * i + 3] << 16) * inv0, a.e5m2);
      const uint32_t lo1 = fp8x2(__uint_as_float(wv[4 * i] & 0xFFFF0000u) * inv1,
                                  __uint_as_float(wv[4 * i + 1] & 0xFFFF0000u) * inv1, a.e5m2);
      const uint32_t hi1 = fp8x2(__uint_as_float(wv[4 * i + 2] & 0xFFFF0000u) * inv1,
                                  __uint_as_float(wv[4 * i + 3] & 0xFFFF0000u) * inv1, a.e5m2);
      q0[i] = lo0 | (hi0 << 16);
      q1[i] = lo1 | (hi1 << 16);
    }
    if (a.tma_store) {  // transposed code tile: 128-byte row per column, 32-byte run per row block
      uint8_t* ct = qcol_tile;
      const int r0 = 2 * p, r1 = 2 * p + 1;
      uint8_t* row0p = ct + r0 * 128;
      uint8_t* row1p = ct + r1 * 128;
      *reinterpret_cast<uint4*>(row0p + (((2 * rb) ^ (r0 & 7)) << 4)) = make_uint4(q0[0], q0[1], q0[2], q0[3]);
      *reinterpret_cast<uint4*>(row0p + (((2 * rb + 1) ^ (r0 & 7)) << 4)) = make_uint4(q0[4], q0[5], q0[6], q0[7]);
      *reinterpret_cast<uint4*>(row1p + (((2 * rb) ^ (r1 & 7)) << 4)) = make_uint4(q1[0], q1[1], q1[2], q1[3]);
      *reinterpret_cast<uint4*>(row1p + (((2 * rb + 1) ^ (r1 & 7)) << 4)) = make_uint4(q1[4], q1[5], q1[6], q1[7]);
    } else {
      uint8_t* qc = a.q_colT + (static_cast<int64_t>(b) * C + gc) * R + gr;
      reinterpret_cast<uint4*>(qc)[0] = make_uint4(q0[0], q0[1], q0[2], q0[3]);
      reinterpret_cast<uint4*>(qc)[1] = make_uint4(q0[4], q0[5], q0[6], q0[7]);
      reinterpret_cast<uint4*>(qc + R)[0] = make_uint4(q1[0], q1[1], q1[2], q1[3]);
      reinterpret_cast<uint4*>(qc + R)[1] = make_uint4(q1[4], q1[5], q1[6], q1[7]);
    }
    if (a.sf_mma) {
      satom_col[sf_mma_offset(2 * p, rb, 4)] = static_cast<uint8_t>(sb0);
      satom_col[sf_mma_offset(2 * p + 1, rb, 4)] = static_cast<uint8_t>(sb1);
    } else {
      const int64_t kb = gr / 32;
      uint8_t* sc = a.s_colT + static_cast<int64_t>(b) * C * KBc;
      sc[gc * KBc + kb] = static_cast<uint8_t>(sb0);
      sc[(gc + 1) * KBc + kb] = static_cast<uint8_t>(sb1);
    }
  } else {
    uint32_t c0[16], c1[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      c0[i] = __byte_perm(wv[2 * i], wv[2 * i + 1], 0x5410);  // low halves: column 2p
      c1[i] = __byte_perm(wv[2 * i], wv[2 * i + 1], 0x7632);  // high halves: column 2p+1
    }
    bf16* oc = a.o_colT + (static_cast<int64_t>(b) * C + gc) * R + gr;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      reinterpret_cast<uint4*>(oc)[i] = make_uint4(c0[4 * i], c0[4 * i + 1], c0[4 * i + 2], c0[4 * i + 3]);
      reinterpret_cast<uint4*>(oc + R)[i] = make_uint4(c1[4 * i], c1[4 * i + 1], c1[4 * i + 2], c1[4 * i + 3]);
    }
  }
}

__global__ void __launch_bounds__(256)
quant_tile_kernel(const __grid_constant__ QuantArgs a) {
  __shared__ __align__(16) uint32_t tile[QT_ROWS * QT_PITCH / 2];  // bf16 pairs
  // code tiles for the TMA stores (128B-swizzled rows of 128 bytes)
  extern __shared__ uint8_t qdyn_raw[];
  // 1024-byte aligned, derived from the shared array (keeps the accesses in the shared state space)
  uint8_t* qdyn = qdyn_raw + ((1024u - (static_cast<uint32_t>(__cvta_generic_to_shared(qdyn_raw)) & 1023u)) & 1023u);
  // In the tensor-core scale layout a 128 x 128 tile's row-wise scales and its column-wise scales
  // are each exactly one 512-byte scale tile: they are assembled here and stored with one write
  // each (single-byte scale stores scattered over the scale matrix cost more than the codes).
  __shared__ __align__(16) uint8_t satom_row[512], satom_col[512];
  const int tid = threadIdx.x;
  // column tiles vary fastest so that CTAs running together read whole contiguous rows
  const int64_t row0 = static_cast<int64_t>(blockIdx.y) * QT_ROWS;
  const int64_t col0 = static_cast<int64_t>(blockIdx.x) * QT_COLS;
  const int b = blockIdx.z;
  const int64_t R = a.rows, C = a.cols, KBr = C / 32, KBc = R / 32;
  const bool sf_atoms = a.mx && a.sf_mma;

  const bf16* src = a.src_ptrs.p[0] ? static_cast<const bf16*>(a.src_ptrs.p[b])
                                    : static_cast<const bf16*>(a.src) + static_cast<int64_t>(b) * a.src_batch_stride;

  // ---- load 128 x 128: 8 chunks of 8 bf16 per thread, all issued before any use
  const int cchunk = tid & 15;
  const int64_t col = col0 + cchunk * 8;
  const bool col_ok = col < C;
  uint4 v[QT_LOADS];
#pragma unroll
  for (int i = 0; i < QT_LOADS; ++i) {
    const int64_t r = row0 + (tid >> 4) + 16 * i;
    v[i] = make_uint4(0, 0, 0, 0);
    if (r < R && col_ok) {
      int64_t sr = r;
      bool zero = false;
      if (a.sorted_to_src) {
        const int32_t s = a.sorted_to_src[r];
        zero = s < 0;
        sr = zero ? 0 : static_cast<int64_t>(s / a.k);
      }
      if (!zero) v[i] = __ldg(reinterpret_cast<const uint4*>(src + sr * a.src_ld + col));
    }
  }
  // destination rows: identity, or the gate/up interleaving (128 rows from each half per 256-row group)
  auto dst_row = [&](int64_t r) -> int64_t {
    if (!a.gate_up_half) return r;
    const int64_t hf = a.gate_up_half;
    return r < hf ? (r / 128) * 256 + (r % 128) : ((r - hf) / 128) * 256 + 128 + ((r - hf) % 128);
  };
  // ---- row-wise outputs (and the smem copy for the column pass)
  uint8_t* qbase = a.q_row + static_cast<int64_t>(b) * R * C + col;
  uint8_t* sbase = a.s_row + static_cast<int64_t>(b) * R * KBr;
  bf16* obase = a.o_row + static_cast<int64_t>(b) * R * C + col;
#pragma unroll
  for (int i = 0; i < QT_LOADS; ++i) {
    const int lr = (tid >> 4) + 16 * i;
    const int64_t r = row0 + lr;
    const bool valid = r < R && col_ok;
    const int64_t dr = dst_row(r);
    if (a.do_col) *reinterpret_cast<uint4*>(&tile[lr * (QT_PITCH / 2) + cchunk * 4]) = v[i];
    if (!a.do_row) continue;
    if (a.mx) {
      uint32_t m = fold_halves(absmax_bf16x2(absmax_bf16x2(v[i].x, v[i].y), absmax_bf16x2(v[i].z, v[i].w)));
      m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
      const uint32_t sb = e8m0_from_amax_bits(m, a.scale_floor, a.e5m2);
      const float inv = e8m0_inv_scale(sb);
      if (valid) {
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
        uint32_t q[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          q[j] = fp8x2(__uint_as_float(w[j] << 16) * inv, __uint_as_float(w[j] & 0xFFFF0000u) * inv, a.e5m2);
        const uint2 qq = make_uint2(q[0] | (q[1] << 16), q[2] | (q[3] << 16));
        if (a.tma_store) {  // row lr, bytes 8*cchunk.. of the swizzled 128-byte row
          uint8_t* rowp = qdyn + lr * 128;
          *reinterpret_cast<uint2*>(rowp + (((cchunk >> 1) ^ (lr & 7)) << 4) + ((cchunk & 1) << 3)) = qq;
        } else {
          *reinterpret_cast<uint2*>(qbase + dr * C) = qq;
        }
        if ((cchunk & 3) == 0) {
          const int64_t kb = col / 32;
          if (sf_atoms)
            satom_row[sf_mma_offset(lr, kb & 3, 4)] = static_cast<uint8_t>(sb);
          else
            sbase[dr * KBr + kb] = static_cast<uint8_t>(sb);
        }
      }
    } else if (valid) {
      *reinterpret_cast<uint4*>(obase + dr * C) = v[i];
    }
  }

  // ---- column-wise: thread -> columns (2p, 2p+1) of the tile, 32-row block rb
  if (a.do_col) {
    __syncthreads();
    const int p = tid & 63;
    const int rb = tid >> 6;
    const int64_t gc = col0 + 2 * p;
    const int64_t gr = row0 + rb * 32;
    if (gc < C && gr < R) column_pass(a, tile, p, rb, gc, gr, b, satom_col, qdyn + 16384);
  }

  // ---- code tiles through TMA tensor stores; scales as one 512-byte store per scale tile (this
  //      layout needs rows and columns in multiples of 128)
  if (a.tma_store) {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // smem writes -> visible to the copy engine
    __syncthreads();
    if (tid == 0) {
      if (a.do_row)
        asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                         reinterpret_cast<uint64_t>(&a.tmap_qrow)),
                     "r"(static_cast<int32_t>(col0)), "r"(static_cast<int32_t>(b * R + dst_row(row0))),
                     "r"(static_cast<uint32_t>(__cvta_generic_to_shared(qdyn)))
                     : "memory");
      if (a.do_col)
        asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                         reinterpret_cast<uint64_t>(&a.tmap_qcol)),
                     "r"(static_cast<int32_t>(row0)), "r"(static_cast<int32_t>(b * C + col0)),
                     "r"(static_cast<uint32_t>(__cvta_generic_to_shared(qdyn + 16384)))
                     : "memory");
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    }
  }
  if (sf_atoms) {
    if (!a.tma_store) __syncthreads();
    if (tid < 32) {
      if (a.do_row)
        reinterpret_cast<uint4*>(sbase + ((dst_row(row0) / 128) * (KBr / 4) + col0 / 128) * 512)[tid] =
            reinterpret_cast<const uint4*>(satom_row)[tid];
    } else if (tid < 64) {
      if (a.do_col) {
        uint8_t* sc = a.s_colT + static_cast<int64_t>(b) * C * KBc;
        reinterpret_cast<uint4*>(sc + ((col0 / 128) * (KBc / 4) + row0 / 128) * 512)[tid - 32] =
            reinterpret_cast<const uint4*>(satom_col)[tid - 32];
      }
    }
  }
  if (a.tma_store && tid == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// ------------------------------------------------------------------------------------------
// The same MXFP8 quantisation (tensor-core scale layout, row-wise and optionally column-wise) for a
// uniformly strided [batch, rows, cols] source whose rows and cols are multiples of 128, as a
// persistent kernel: the CTAs walk the 128 x 128 tiles (column tiles fastest); each source tile
// arrives by a TMA tensor load (or, for a gather, by tile::gather4 row fetches) into a QW_NIN-deep
// ring issued QW_NIN tiles ahead.  Two ways out for the codes, chosen per use by measurement:
//  * staged (weights, bf16 transposes): code tiles in 128B-swizzled shared memory leave through TMA
//    tensor stores as whole 128-byte lines; two CTAs per SM;
//  * direct (the x / dy gathers): codes leave straight from registers in whole sectors (8-byte row
//    chunks, 16 threads per 128-byte row; 32-byte column runs), no output staging, three CTAs per
//    SM.
// Same arithmetic, bit for bit, as quant_tile_kernel.
// ------------------------------------------------------------------------------------------
namespace {
constexpr int QW_NIN = 2;                           // source tiles in flight per CTA
constexpr int QW_IN_BYTES = QT_ROWS * QT_COLS * 2;  // one bf16 source tile, rows of 256 bytes
constexpr int QW_OUT_BYTES = 2 * QT_ROWS * QT_COLS;  // staged: row-wise + column-wise code tiles
static_assert(QW_OUT_BYTES >= QT_ROWS * QT_COLS * 2, "an output buffer also holds one transposed bf16 tile");
template <bool DIRECT>
struct QwShape {
  static constexpr int CTAS_PER_SM = DIRECT ? 3 : 2;
  static constexpr int OUT_BYTES = DIRECT ? 0 : QW_OUT_BYTES;
  static constexpr int SMEM = QW_NIN * QW_IN_BYTES + OUT_BYTES + 1024 + 1024;  // + 2 scale tiles, + alignment
};
}  // namespace

template <bool DIRECT, int FMT>
__global__ void __launch_bounds__(256, QwShape<DIRECT>::CTAS_PER_SM)
    quant_w_tma_kernel(const __grid_constant__ QuantArgs a, int tiles) {
  // the element format and the shared-exponent rule as constants (FMT bit 0: E5M2, bit 1: the floor
  // rule), so that each conversion is a single instruction of the one format
  constexpr int E5 = FMT & 1, FLOOR = (FMT >> 1) & 1;
  extern __shared__ uint8_t qw_raw[];
  uint8_t* sm = qw_raw + ((1024u - (static_cast<uint32_t>(__cvta_generic_to_shared(qw_raw)) & 1023u)) & 1023u);
  uint8_t* in_base = sm;                                        // QW_NIN source tiles
  uint8_t* qrow = sm + QW_NIN * QW_IN_BYTES;                    // staged: row-wise code tile (16 KB)
  uint8_t* qcol = qrow + QT_ROWS * QT_COLS;                     //         column-wise code tile (16 KB)
  uint8_t* satom_row = qrow + QwShape<DIRECT>::OUT_BYTES;       // the tile's row-wise scale tile (512 B)
  uint8_t* satom_col = satom_row + 512;                         // and its column-wise one
  __shared__ uint64_t full[QW_NIN];
  __shared__ int stop;
  __shared__ float pt_sc[MOE_MAX_EXPERTS];       // per-tensor FP8: the scale of each tensor
  __shared__ int32_t pt_off[MOE_MAX_EXPERTS + 1];  // ... and the expert segments' first rows
  const int tid = threadIdx.x;
  const int64_t R = a.rows, C = a.cols, KBr = C / 32, KBc = R / 32;
  const int CT = static_cast<int>(C / QT_COLS), RT = static_cast<int>(R / QT_ROWS);
  const bool pt = a.pt_amax != nullptr;
  auto coords = [&](int t, int& b, int& rt, int& ct) {
    b = t / (RT * CT);
    const int rem = t - b * RT * CT;
    rt = rem / CT;
    ct = rem - rt * CT;
  };
  auto dst_row = [&](int64_t r) -> int64_t {
    if (!a.gate_up_half) return r;
    const int64_t hf = a.gate_up_half;
    return r < hf ? (r / 128) * 256 + (r % 128) : ((r - hf) / 128) * 256 + 128 + ((r - hf) % 128);
  };
  // gather: the four source rows lane ``tid`` of warp 0 fetches for tile t (padding rows point past
  // the last source row, where the copy reads zeros)
  auto gather_rows = [&](int t, int32_t (&y)[4]) {
    int b, rt, ct;
    coords(t, b, rt, ct);
    const int64_t r0 = static_cast<int64_t>(rt) * QT_ROWS + 4 * (tid & 31);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int32_t s = a.sorted_to_src[r0 + j];
      y[j] = s < 0 ? static_cast<int32_t>(a.src_rows) : s / a.k;
    }
  };
  // source tile t into ring slot ``slot``: one 3-D box (thread 0), or, for a gather, 32 gather4
  // loads of four rows each (one per lane of warp 0, rows ``y``)
  auto issue = [&](int t, int slot, const int32_t (&y)[4]) {
    int b, rt, ct;
    coords(t, b, rt, ct);
    if (!a.tma_gather) {
      ptx::mbar_arrive_expect_tx(&full[slot], QW_IN_BYTES);
      ptx::tma_load_3d(in_base + slot * QW_IN_BYTES, &a.tmap_src, ct * QT_COLS, rt * QT_ROWS, b, &full[slot]);
      return;
    }
    const int lane = tid & 31;
    if (lane == 0) ptx::mbar_arrive_expect_tx(&full[slot], QW_IN_BYTES);
    ptx::tma_gather4(in_base + slot * QW_IN_BYTES + lane * 4 * 256, &a.tmap_src, ct * QT_COLS, y[0], y[1], y[2], y[3],
                     &full[slot]);
  };
  const bool issuer = a.tma_gather ? tid < 32 : tid == 0;
  if (pt) {
    const int n = a.pt_poff ? a.pt_E : tiles / (RT * CT);
    for (int i = tid; i < n; i += blockDim.x) pt_sc[i] = fp8_tensor_scale(a.pt_amax[i], E5);
    if (a.pt_poff)
      for (int i = tid; i <= a.pt_E; i += blockDim.x) pt_off[i] = a.pt_poff[i];
  }
  if (tid == 0) {
    for (int i = 0; i < QW_NIN; ++i) ptx::mbar_init(&full[i], 1);
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&a.tmap_src);
    stop = 0;
  }
  __syncthreads();
  int issued_last = 0;  // last tile whose load was issued (waited for at exit only after an abort)
  // gather: rows of the next tile to be issued, loaded one refill ahead so that the index loads'
  // latency overlaps a tile's work instead of delaying the refill
  int32_t y_next[4] = {0, 0, 0, 0};
  if (issuer) {
    for (int j = 0; j < QW_NIN; ++j) {
      const int t = blockIdx.x + j * gridDim.x;
      if (t < tiles) {
        if (a.tma_gather) gather_rows(t, y_next);
        issue(t, j, y_next);
        issued_last = t;
      }
    }
    const int tn = blockIdx.x + QW_NIN * gridDim.x;
    if (a.tma_gather && tn < tiles) gather_rows(tn, y_next);
  }
  // direct: 32-byte aligned column-wise output leaves in single 256-bit stores
  const bool col32 = ((reinterpret_cast<uintptr_t>(a.mx ? static_cast<void*>(a.q_colT) : static_cast<void*>(a.o_colT)) &
                       31u) == 0);
  int it = 0;
  for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++it) {
    const int slot = it % QW_NIN;
    if (tid == 0) {
      // this tile's source has landed (staged: and the stores that read the code tiles are done)
      volatile int* flag = &stop;  // raised by an expired wait
      bool ok = true;
      if (a.stall_flag && it == 0)  // test hook: a wait that can only expire, first source tiles in flight
        ok = ptx::wait_flag(a.stall_flag, flag, a.stall_limit);
      if (ok && !ptx::mbar_wait(&full[slot], static_cast<uint32_t>((it / QW_NIN) & 1), flag, kWaitLimitCycles))
        ok = false;
      if (!ok) {
        stop = 1;
        if (a.status) atomicOr(a.status, kStatusTimeout);
      }
      if (!DIRECT) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    }
    __syncthreads();
    if (stop) break;
    int b, rt, ct;
    coords(t, b, rt, ct);
    const int64_t row0 = static_cast<int64_t>(rt) * QT_ROWS, col0 = static_cast<int64_t>(ct) * QT_COLS;
    const uint8_t* in = in_base + slot * QW_IN_BYTES;
    float pts = 0.f;  // per-tensor FP8: the tile's tensor scale
    if (pt) {
      int e = b;
      if (a.pt_poff) {  // the expert segment holding row0 (largest e with pt_off[e] <= row0)
        int lo = 0, hi = a.pt_E;
        while (hi - lo > 1) {
          const int mid = (lo + hi) >> 1;
          if (pt_off[mid] <= row0) lo = mid; else hi = mid;
        }
        e = lo;
      }
      pts = pt_sc[e];
    }

    if (!a.mx) {
      // bf16 transpose only: thread -> columns (2p, 2p+1) = rows of the transposed tile, source rows
      // 32 rb .. +31
      const int p = tid & 63, rb = tid >> 6;
      const uint32_t* words = reinterpret_cast<const uint32_t*>(in);  // 64 bf16 pairs per row
      uint32_t c0[16], c1[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const uint32_t w0 = words[(rb * 32 + 2 * i) * 64 + p], w1 = words[(rb * 32 + 2 * i + 1) * 64 + p];
        c0[i] = __byte_perm(w0, w1, 0x5410);  // low halves: column 2p
        c1[i] = __byte_perm(w0, w1, 0x7632);  // high halves: column 2p+1
      }
      if (!DIRECT) {
        // the transposed tile (32 KB: the whole output buffer) as two 64-column halves of 128-byte
        // rows, 128B-swizzled
        uint8_t* half = qrow + (rb >> 1) * (QT_ROWS * 128);
        const int r0 = 2 * p, r1 = 2 * p + 1;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int chunk = (rb & 1) * 4 + j;
          *reinterpret_cast<uint4*>(half + r0 * 128 + ((chunk ^ (r0 & 7)) << 4)) =
              make_uint4(c0[4 * j], c0[4 * j + 1], c0[4 * j + 2], c0[4 * j + 3]);
          *reinterpret_cast<uint4*>(half + r1 * 128 + ((chunk ^ (r1 & 7)) << 4)) =
              make_uint4(c1[4 * j], c1[4 * j + 1], c1[4 * j + 2], c1[4 * j + 3]);
        }
      } else {
        // columns 2p and 2p+1 of the source are rows of the transposed output: 64 bytes each
        bf16* o0 = a.o_colT + (static_cast<int64_t>(b) * C + col0 + 2 * p) * R + row0 + rb * 32;
        bf16* o1 = o0 + R;
        if (col32) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            ptx::st_global_v8(o0 + 16 * j, make_uint4(c0[8 * j], c0[8 * j + 1], c0[8 * j + 2], c0[8 * j + 3]),
                              make_uint4(c0[8 * j + 4], c0[8 * j + 5], c0[8 * j + 6], c0[8 * j + 7]));
            ptx::st_global_v8(o1 + 16 * j, make_uint4(c1[8 * j], c1[8 * j + 1], c1[8 * j + 2], c1[8 * j + 3]),
                              make_uint4(c1[8 * j + 4], c1[8 * j + 5], c1[8 * j + 6], c1[8 * j + 7]));
          }
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            reinterpret_cast<uint4*>(o0)[j] = make_uint4(c0[4 * j], c0[4 * j + 1], c0[4 * j + 2], c0[4 * j + 3]);
            reinterpret_cast<uint4*>(o1)[j] = make_uint4(c1[4 * j], c1[4 * j + 1], c1[4 * j + 2], c1[4 * j + 3]);
          }
        }
      }
    } else {
      // ---- row-wise: thread -> 8-column chunk ``cchunk`` of rows tid/16 + 16 i
      const int cchunk = tid & 15;
#pragma unroll
      for (int i = 0; i < QT_LOADS; ++i) {
        const int lr = (tid >> 4) + 16 * i;
        const uint4 v = *reinterpret_cast<const uint4*>(in + lr * 256 + cchunk * 16);
        uint32_t m = fold_halves(absmax_bf16x2(absmax_bf16x2(v.x, v.y), absmax_bf16x2(v.z, v.w)));
        m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
        const uint32_t sb = e8m0_from_amax_bits(m, FLOOR, E5);
        const float inv = pt ? pts : e8m0_inv_scale(sb);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t q[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          q[j] = fp8x2(__uint_as_float(w[j] << 16) * inv, __uint_as_float(w[j] & 0xFFFF0000u) * inv, E5);
        const uint2 qq = make_uint2(q[0] | (q[1] << 16), q[2] | (q[3] << 16));
        if (!DIRECT)
          *reinterpret_cast<uint2*>(qrow + lr * 128 + (((cchunk >> 1) ^ (lr & 7)) << 4) + ((cchunk & 1) << 3)) = qq;
        else
          *reinterpret_cast<uint2*>(a.q_row + (static_cast<int64_t>(b) * R + dst_row(row0 + lr)) * C + col0 +
                                    cchunk * 8) = qq;
        if ((cchunk & 3) == 0 && !pt) satom_row[sf_mma_offset(lr, (cchunk >> 2) & 3, 4)] = static_cast<uint8_t>(sb);
      }

      // ---- column-wise: thread -> columns (2p, 2p+1), 32-row block rb
      if (a.do_col) {
        const int p = tid & 63, rb = tid >> 6;
        const uint32_t* words = reinterpret_cast<const uint32_t*>(in);  // 64 bf16 pairs per row
        uint32_t wv[32];
        uint32_t m2 = 0;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          wv[i] = words[(rb * 32 + i) * 64 + p];
          m2 = absmax_bf16x2(m2, wv[i]);
        }
        const uint32_t sb0 = e8m0_from_amax_bits(m2 << 16, FLOOR, E5);
        const uint32_t sb1 = e8m0_from_amax_bits(m2 & 0xFFFF0000u, FLOOR, E5);
        const float inv0 = pt ? pts : e8m0_inv_scale(sb0), inv1 = pt ? pts : e8m0_inv_scale(sb1);
        uint32_t q0[8], q1[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t lo0 =
              fp8x2(__uint_as_float(wv[4 * i] << 16) * inv0, __uint_as_float(wv[4 * i + 1] << 16) * inv0, E5);
          const uint32_t hi0 =
              fp8x2(__uint_as_float(wv[4 * i + 2] << 16) * inv0, __uint_as_float(wv[4 * i + 3] << 16) * inv0, E5);
          const uint32_t lo1 = fp8x2(__uint_as_float(wv[4 * i] & 0xFFFF0000u) * inv1,
                                      __uint_as_float(wv[4 * i + 1] & 0xFFFF0000u) * inv1, E5);
          const uint32_t hi1 = fp8x2(__uint_as_float(wv[4 * i + 2] & 0xFFFF0000u) * inv1,
                                      __uint_as_float(wv[4 * i + 3] & 0xFFFF0000u) * inv1, E5);
          q0[i] = lo0 | (hi0 << 16);
          q1[i] = lo1 | (hi1 << 16);
        }
        if (!DIRECT) {
          const int r0 = 2 * p, r1 = 2 * p + 1;  // rows of the transposed code tile
          uint8_t* row0p = qcol + r0 * 128;
          uint8_t* row1p = qcol + r1 * 128;
          *reinterpret_cast<uint4*>(row0p + (((2 * rb) ^ (r0 & 7)) << 4)) = make_uint4(q0[0], q0[1], q0[2], q0[3]);
          *reinterpret_cast<uint4*>(row0p + (((2 * rb + 1) ^ (r0 & 7)) << 4)) = make_uint4(q0[4], q0[5], q0[6], q0[7]);
          *reinterpret_cast<uint4*>(row1p + (((2 * rb) ^ (r1 & 7)) << 4)) = make_uint4(q1[0], q1[1], q1[2], q1[3]);
          *reinterpret_cast<uint4*>(row1p + (((2 * rb + 1) ^ (r1 & 7)) << 4)) = make_uint4(q1[4], q1[5], q1[6], q1[7]);
        } else {
          // columns 2p and 2p+1 are rows of the transposed codes: one 32-byte run each
          uint8_t* c0p = a.q_colT + (static_cast<int64_t>(b) * C + col0 + 2 * p) * R + row0 + rb * 32;
          uint8_t* c1p = c0p + R;
          if (col32) {
            ptx::st_global_v8(c0p, make_uint4(q0[0], q0[1], q0[2], q0[3]), make_uint4(q0[4], q0[5], q0[6], q0[7]));
            ptx::st_global_v8(c1p, make_uint4(q1[0], q1[1], q1[2], q1[3]), make_uint4(q1[4], q1[5], q1[6], q1[7]));
          } else {
            reinterpret_cast<uint4*>(c0p)[0] = make_uint4(q0[0], q0[1], q0[2], q0[3]);
            reinterpret_cast<uint4*>(c0p)[1] = make_uint4(q0[4], q0[5], q0[6], q0[7]);
            reinterpret_cast<uint4*>(c1p)[0] = make_uint4(q1[0], q1[1], q1[2], q1[3]);
            reinterpret_cast<uint4*>(c1p)[1] = make_uint4(q1[4], q1[5], q1[6], q1[7]);
          }
        }
        if (!pt) {
          satom_col[sf_mma_offset(2 * p, rb, 4)] = static_cast<uint8_t>(sb0);
          satom_col[sf_mma_offset(2 * p + 1, rb, 4)] = static_cast<uint8_t>(sb1);
        }
      }
    }

    if (!DIRECT) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // code tiles -> the copy engine
    __syncthreads();  // the source tile is consumed; code tiles (staged) and scale tiles are complete
    if (!DIRECT && tid == 0) {
      if (a.mx) {
        asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                         reinterpret_cast<uint64_t>(&a.tmap_qrow)),
                     "r"(static_cast<int32_t>(col0)), "r"(static_cast<int32_t>(b * R + dst_row(row0))),
                     "r"(static_cast<uint32_t>(__cvta_generic_to_shared(qrow)))
                     : "memory");
        if (a.do_col)
          asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                           reinterpret_cast<uint64_t>(&a.tmap_qcol)),
                       "r"(static_cast<int32_t>(row0)), "r"(static_cast<int32_t>(b * C + col0)),
                       "r"(static_cast<uint32_t>(__cvta_generic_to_shared(qcol)))
                       : "memory");
      } else {  // the transposed bf16 tile: two boxes of 64 columns x 128 rows
#pragma unroll
        for (int h = 0; h < 2; ++h)
          asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                           reinterpret_cast<uint64_t>(&a.tmap_qcol)),
                       "r"(static_cast<int32_t>(row0 + 64 * h)), "r"(static_cast<int32_t>(b * C + col0)),
                       "r"(static_cast<uint32_t>(__cvta_generic_to_shared(qrow + h * QT_ROWS * 128)))
                       : "memory");
      }
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    }
    if (issuer) {
      const int tn = t + QW_NIN * gridDim.x;  // refill the slot just consumed
      if (tn < tiles) {
        issue(tn, slot, y_next);
        issued_last = tn;
        if (a.tma_gather && tn + static_cast<int>(gridDim.x) < tiles) gather_rows(tn + gridDim.x, y_next);
      }
    } else if (a.mx && !pt && tid >= 32 && tid < 64) {  // warp 1: the two 512-byte scale tiles, 16 bytes per lane
      const int l = tid - 32;
      uint8_t* sr = a.s_row + static_cast<int64_t>(b) * R * KBr;
      reinterpret_cast<uint4*>(sr + ((dst_row(row0) / 128) * (KBr / 4) + col0 / 128) * 512)[l] =
          reinterpret_cast<const uint4*>(satom_row)[l];
      if (a.do_col) {
        uint8_t* sc = a.s_colT + static_cast<int64_t>(b) * C * KBc;
        reinterpret_cast<uint4*>(sc + ((col0 / 128) * (KBc / 4) + row0 / 128) * 512)[l] =
            reinterpret_cast<const uint4*>(satom_col)[l];
      }
    }
  }
  if (tid == 0) {
    if (stop) {  // after an abort: the source tiles still in flight land before the CTA exits
      volatile int never = 0;
      for (int j = 0; j < QW_NIN; ++j) {
        const int t = issued_last - j * static_cast<int>(gridDim.x);
        if (t < static_cast<int>(blockIdx.x)) break;
        const int k = (t - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x);
        ptx::mbar_wait(&full[k % QW_NIN], static_cast<uint32_t>((k / QW_NIN) & 1), &never, kWaitLimitCycles);
      }
    }
    if (!DIRECT) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
  }
}

// ------------------------------------------------------------------------------------------
// Combine: y[t] = bf16(sum_j w_j * fp32(rows[row(t, j)])), j ascending, fp32 products and sums;
// slots whose row is -1 are skipped.
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
unpermute_kernel(const bf16* __restrict__ rows, const int32_t* __restrict__ src_to_sorted,
                 const float* __restrict__ probs, int64_t T, int k, int64_t d, bf16* __restrict__ y) {
  const int64_t chunks = d / 8;
  const int64_t total = T * chunks;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / chunks;
    const int64_t c = (i - t * chunks) * 8;
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.f;
    auto add = [&](const uint4& v, int j) {
      const bf16* h = reinterpret_cast<const bf16*>(&v);
      if (probs) {
        const float w = probs[t * k + j];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = __fadd_rn(acc[q], __fmul_rn(w, __bfloat162float(h[q])));
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = __fadd_rn(acc[q], __bfloat162float(h[q]));
      }
    };
    if (k == 2) {  // top-2: both rows' loads in flight before either is used
      const int64_t r0 = src_to_sorted[t * 2], r1 = src_to_sorted[t * 2 + 1];
      uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
      if (r0 >= 0) v0 = __ldg(reinterpret_cast<const uint4*>(rows + r0 * d + c));
      if (r1 >= 0) v1 = __ldg(reinterpret_cast<const uint4*>(rows + r1 * d + c));
      if (r0 >= 0) add(v0, 0);
      if (r1 >= 0) add(v1, 1);
    } else {
      for (int j = 0; j < k; ++j) {
        const int64_t r = src_to_sorted[t * k + j];
        if (r < 0) continue;  // a slot the routing rejected (expert index out of range): contributes nothing
        add(__ldg(reinterpret_cast<const uint4*>(rows + r * d + c)), j);
      }
    }
    uint4 o;
    bf16* ho = reinterpret_cast<bf16*>(&o);
#pragma unroll
    for (int q = 0; q < 8; ++q) ho[q] = __float2bfloat16_rn(acc[q]);
    *reinterpret_cast<uint4*>(y + t * d + c) = o;
  }
}

// d_topk_prob[t][j] = the sum of the partial row sums of the ScaledSwiGLU probability gradient at
// row(t, j), over all n-tiles.  Four consecutive threads share a row: thread q sums the q-th quarter
// of the partials in ascending order (eight independent loads in flight; consecutive rows are
// consecutive words of every partial), then the four quarter sums are added in order q = 0..3.  The
// sum is written to the row's slot; slots the routing rejected (no row) get zero.
__global__ void dprob_reduce_kernel(const float* __restrict__ part, int n_parts, int64_t part_stride,
                                    const int32_t* __restrict__ sorted_to_src, int64_t rows,
                                    const int32_t* __restrict__ src_to_sorted, int64_t Tk,
                                    float* __restrict__ d_prob) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t i0 = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  const int lane = threadIdx.x & 31, q = lane & 3;
  const int per = (n_parts + 3) / 4;
  const int n0 = min(n_parts, q * per), n1 = min(n_parts, n0 + per);
  // the loop bound is the same for the whole warp, so every lane reaches the shuffles below
  for (int64_t wbase = i0 - lane; wbase < 4 * rows; wbase += stride) {
    const int64_t r = (wbase + lane) / 4;
    const int32_t s = r < rows ? sorted_to_src[r] : -1;
    float acc = 0.f;
    if (s >= 0) {
      int n = n0;
      for (; n + 8 <= n1; n += 8) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = __ldg(part + (n + u) * part_stride + r);
#pragma unroll
        for (int u = 0; u < 8; ++u) acc = __fadd_rn(acc, v[u]);
      }
      for (; n < n1; ++n) acc = __fadd_rn(acc, __ldg(part + n * part_stride + r));
    }
    // quarter sums in order 0..3 (the four lanes of a row are adjacent)
    const float a1 = __shfl_down_sync(0xffffffffu, acc, 1, 4);
    const float a2 = __shfl_down_sync(0xffffffffu, acc, 2, 4);
    const float a3 = __shfl_down_sync(0xffffffffu, acc, 3, 4);
    if (q == 0 && s >= 0) d_prob[s] = __fadd_rn(__fadd_rn(__fadd_rn(acc, a1), a2), a3);
  }
  for (int64_t s = i0; s < Tk; s += stride)
    if (src_to_sorted[s] < 0) d_prob[s] = 0.f;
}

// Row-wise MXFP8 -> fp32 (tests).
__global__ void dequant_kernel(const uint8_t* __restrict__ q, const uint8_t* __restrict__ s, int64_t R, int64_t C,
                               int sf_mma, float* __restrict__ out) {
  const int64_t KB = C / 32;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < R * C;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / C, c = i - r * C;
    const int64_t kb = c / 32;
    const uint8_t sb = s[sf_mma ? sf_mma_offset(r, kb, KB) : r * KB + kb];
    const __nv_fp8_e4m3 v = *reinterpret_cast<const __nv_fp8_e4m3*>(q + i);
    const float scale = sb == 255 ? __uint_as_float(0x7FC00000u) : (sb == 0 ? 0x1p-127f : __uint_as_float(static_cast<uint32_t>(sb) << 23));
    out[i] = static_cast<float>(v) * scale;
  }
}

// ------------------------------------------------------------------------------------------
// launchers
// ------------------------------------------------------------------------------------------
cudaError_t launch_route(const int32_t* topk_idx, const float* topk_prob, int Tk, int E, int capacity,
                         const int32_t* split_in, int32_t* split_out, int32_t* poffsets, int32_t* sorted_to_src,
                         int32_t* src_to_sorted, float* prob_perm, int* status, cudaStream_t st) {
  const size_t smem = static_cast<size_t>(32) * E * sizeof(int32_t);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  route_kernel<<<1, 1024, smem, st>>>(topk_idx, topk_prob, Tk, E, capacity, split_in, split_out, poffsets,
                                       sorted_to_src, src_to_sorted, prob_perm, status);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// Per-tensor FP8 maxima: current scaling needs each tensor's largest magnitude before any of it is
// quantised.  Magnitudes compare as bf16 bit patterns (bits & 0x7FFF grows with |x| for finite
// values) and are kept as fp32 bits, so that atomicMax on unsigned words orders them.
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t absmax8_bf16(uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t m = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) m = max(m, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
  return m;
}

// grid (row slices, batch): block x of batch b takes rows x, x + gridDim.x, ...
__global__ void __launch_bounds__(256) amax_batched_kernel(const __grid_constant__ PtrArray ptrs, const bf16* src,
                                                           int64_t batch_stride, int64_t rows, int64_t cols,
                                                           int64_t ld, uint32_t* __restrict__ amax) {
  __shared__ uint32_t wmax[8];
  const int b = blockIdx.y;
  const bf16* base = ptrs.p[b] ? static_cast<const bf16*>(ptrs.p[b]) : src + b * batch_stride;
  const int64_t cv = cols / 8;
  uint32_t m = 0;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const uint4* row = reinterpret_cast<const uint4*>(base + r * ld);
    for (int64_t c = threadIdx.x; c < cv; c += blockDim.x) m = max(m, absmax8_bf16(__ldcs(row + c)));
  }
  m = __reduce_max_sync(0xffffffffu, m);
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < 8; ++w) m = max(m, wmax[w]);
    if (m) atomicMax(amax + b, m << 16);
  }
}

// One warp per row of the expert-sorted order (rows without a slot are skipped): the row reads token
// sorted_to_src[r] / k and belongs to the expert whose padded segment poffsets[e] .. poffsets[e+1]
// holds r; per-CTA maxima in shared memory first.
__global__ void __launch_bounds__(256) amax_routed_kernel(const bf16* __restrict__ x, int64_t ld, int64_t d,
                                                          const int32_t* __restrict__ sorted_to_src,
                                                          const int32_t* __restrict__ poffsets, int64_t rows, int k,
                                                          int E, uint32_t* __restrict__ amax) {
  __shared__ uint32_t sm[MOE_MAX_EXPERTS];
  __shared__ int32_t off[MOE_MAX_EXPERTS + 1];
  for (int i = threadIdx.x; i < E; i += blockDim.x) sm[i] = 0;
  for (int i = threadIdx.x; i <= E; i += blockDim.x) off[i] = poffsets[i];
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += nwarps) {
    const int32_t slot = sorted_to_src[r];
    if (slot < 0 || r >= off[E]) continue;  // padding row
    int lo = 0, hi = E;                     // largest e with off[e] <= r
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (off[mid] <= r) lo = mid; else hi = mid;
    }
    const uint4* row = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(slot / k) * ld);
    uint32_t m = 0;
    for (int64_t c = lane; c < d / 8; c += 32) m = max(m, absmax8_bf16(row[c]));
    m = __reduce_max_sync(0xffffffffu, m);
    if (lane == 0 && m) atomicMax(&sm[lo], m);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < E; i += blockDim.x)
    if (sm[i]) atomicMax(amax + i, sm[i] << 16);
}

cudaError_t launch_amax_batched(const PtrArray& src_ptrs, const bf16* src, int64_t batch_stride, int batch,
                                int64_t rows, int64_t cols, int64_t ld, uint32_t* amax, int num_sms,
                                cudaStream_t st) {
  if (batch <= 0 || rows <= 0 || cols <= 0) return cudaSuccess;
  if (cols % 8 || ld % 8 || batch > 65535) return cudaErrorInvalidValue;
  const int64_t per_batch = std::max<int64_t>(1, static_cast<int64_t>(num_sms) * 8 / batch);
  dim3 grid(static_cast<unsigned>(std::min<int64_t>(rows, per_batch)), static_cast<unsigned>(batch));
  amax_batched_kernel<<<grid, 256, 0, st>>>(src_ptrs, src, batch_stride, rows, cols, ld, amax);
  return cudaGetLastError();
}

cudaError_t launch_amax_routed(const bf16* x, int64_t ld, int64_t d, const int32_t* sorted_to_src,
                               const int32_t* poffsets, int64_t rows, int k, int E, uint32_t* amax, int num_sms,
                               cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  if (d % 8 || ld % 8 || E > MOE_MAX_EXPERTS) return cudaErrorInvalidValue;
  const int64_t blocks = std::min<int64_t>(ceil_div(rows, 8), static_cast<int64_t>(num_sms) * 4);
  amax_routed_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(x, ld, d, sorted_to_src, poffsets, rows, k, E,
                                                                     amax);
  return cudaGetLastError();
}

__global__ void fp8_scales_kernel(uint32_t* v, int n, int e5m2) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) v[i] = __float_as_uint(fp8_tensor_scale(v[i], e5m2));
}

cudaError_t launch_fp8_scales(uint32_t* amax_to_scale, int n, int e5m2, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  fp8_scales_kernel<<<(n + 255) / 256, 256, 0, st>>>(amax_to_scale, n, e5m2);
  return cudaGetLastError();
}

cudaError_t launch_quant(const QuantArgs& a, int batch, int num_sms, cudaStream_t st) {
  if (a.rows == 0 || a.cols == 0 || batch == 0) return cudaSuccess;
  const bool persistent = a.tma_load && a.tma_store && (a.mx ? a.do_row : (a.do_col && !a.do_row));
  if (a.pt_amax && (!persistent || !a.mx || (a.pt_poff ? a.pt_E : batch) > MOE_MAX_EXPERTS))
    return cudaErrorInvalidValue;  // per-tensor FP8 exists only in the TMA-fed kernel
  if (persistent) {
    const int64_t tiles = (a.rows / QT_ROWS) * (a.cols / QT_COLS) * batch;
    // direct stores for the gathers, staged TMA stores otherwise (measured: the gathers run 13% faster
    // direct, the weight quantisation 10% faster staged)
    const int fmt = (a.e5m2 ? 1 : 0) | (a.scale_floor ? 2 : 0);
    void (*const kerns[2][4])(QuantArgs, int) = {
        {quant_w_tma_kernel<false, 0>, quant_w_tma_kernel<false, 1>, quant_w_tma_kernel<false, 2>,
         quant_w_tma_kernel<false, 3>},
        {quant_w_tma_kernel<true, 0>, quant_w_tma_kernel<true, 1>, quant_w_tma_kernel<true, 2>,
         quant_w_tma_kernel<true, 3>}};
    auto kern = kerns[a.tma_gather ? 1 : 0][fmt];
    const int smem = a.tma_gather ? QwShape<true>::SMEM : QwShape<false>::SMEM;
    const int per_sm = a.tma_gather ? QwShape<true>::CTAS_PER_SM : QwShape<false>::CTAS_PER_SM;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int grid = static_cast<int>(std::min<int64_t>(tiles, static_cast<int64_t>(num_sms) * per_sm));
    kern<<<grid, 256, smem, st>>>(a, static_cast<int>(tiles));
    return cudaGetLastError();
  }
  dim3 grid(static_cast<unsigned>(ceil_div(a.cols, QT_COLS)), static_cast<unsigned>(ceil_div(a.rows, QT_ROWS)),
            static_cast<unsigned>(batch));
  const int dyn = a.tma_store ? 32768 + 1024 : 0;
  if (dyn) {
    cudaError_t e = cudaFuncSetAttribute(quant_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
    if (e != cudaSuccess) return e;
  }
  quant_tile_kernel<<<grid, 256, dyn, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_unpermute(const bf16* rows, const int32_t* src_to_sorted, const float* probs, int64_t T, int k,
                             int64_t d, bf16* y, int num_sms, cudaStream_t st) {
  const int64_t total = T * (d / 8);
  if (total == 0) return cudaSuccess;
  const int64_t blocks = std::min<int64_t>(ceil_div(total, 256), static_cast<int64_t>(num_sms) * 16);
  unpermute_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(rows, src_to_sorted, probs, T, k, d, y);
  return cudaGetLastError();
}

cudaError_t launch_dprob_reduce(const float* part, int n_parts, int64_t part_stride, const int32_t* sorted_to_src,
                                int64_t rows, const int32_t* src_to_sorted, int64_t Tk, float* d_prob,
                                cudaStream_t st) {
  if (Tk == 0) return cudaSuccess;
  const int64_t blocks = std::min<int64_t>(ceil_div(std::max(4 * rows, Tk), 256), 4096);
  dprob_reduce_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(part, n_parts, part_stride, sorted_to_src, rows,
                                                                      src_to_sorted, Tk, d_prob);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const uint8_t* q, const uint8_t* s, int64_t R, int64_t C, int sf_mma, float* out,
                           int num_sms, cudaStream_t st) {
  if (R * C == 0) return cudaSuccess;
  const int64_t blocks = std::min<int64_t>(ceil_div(R * C, 256), static_cast<int64_t>(num_sms) * 16);
  dequant_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(q, s, R, C, sf_mma, out);
  return cudaGetLastError();
}

}  // namespace moemx
