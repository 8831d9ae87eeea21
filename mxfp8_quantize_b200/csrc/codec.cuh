// Declarations of the HBM-bound kernels' launchers (codec.cu).
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace moemx {

struct PtrArray {
  const void* p[MOE_MAX_EXPERTS];
};

// One quantise / gather / transpose pass over a [batch, rows, cols] bf16 source.
struct QuantArgs {
  const bf16* src;             // batch 0 source (when src_ptrs.p[0] is null)
  int64_t src_batch_stride;    // elements between batches of ``src``
  int64_t src_ld;              // elements between source rows
  PtrArray src_ptrs;           // per-batch sources (expert weights), or all null
  const int32_t* sorted_to_src;  // gather: output row r reads token sorted_to_src[r] / k (-1: zeros)
  int k;
  int64_t rows, cols;          // output rows and columns per batch
  int mx;                      // 1: MXFP8 codes + scales; 0: bf16 copies
  int64_t gate_up_half;        // >0: row-wise outputs in 256-row groups [128 rows < half | 128 rows >= half]
  int do_row, do_col, sf_mma;
  int scale_floor;             // MXFP8 shared exponent: 0 round-up rule, 1 OCP floor rule
  int e5m2;                    // MXFP8 element format: 0 E4M3, 1 E5M2
  uint8_t* q_row;
  uint8_t* s_row;
  uint8_t* q_colT;
  uint8_t* s_colT;
  bf16* o_row;
  bf16* o_colT;
  // MXFP8 with the tensor-core scale layout: code tiles leave through TMA tensor stores
  // (uint8 maps over [batch*rows, cols] and [batch*cols, rows], 128 x 128 boxes, 128B swizzle)
  int tma_store;
  CUtensorMap tmap_qrow;
  CUtensorMap tmap_qcol;
  // ... and, when the source is one uniformly strided [batch, rows, cols] tensor with rows and
  // cols multiples of 128, it arrives through TMA tensor loads (bf16 map over [batch, rows, cols],
  // 128 x 128 boxes) into a persistent kernel's ring of tiles
  int tma_load;
  CUtensorMap tmap_src;
  // ... or, for a gather (``sorted_to_src``), a 2-D bf16 map over the [src_rows, cols] source
  // whose boxes are single rows, four of them per tile::gather4 load (padding rows read past
  // src_rows, which the copy fills with zeros)
  int tma_gather;
  int64_t src_rows;
  // per-tensor FP8 (with mx = 1: codes only, no scale bytes): a tile's codes are E4M3 / E5M2 of
  // v * s with s = vmax / amax of its tensor (fp8_tensor_scale); amax as fp32 bits from
  // pt_amax[b] for batch b, or, with pt_poff, from pt_amax[e] for the expert e whose padded rows
  // pt_poff[e] .. pt_poff[e+1] hold the tile (one [rows, cols] source of expert segments)
  const uint32_t* pt_amax;
  const int32_t* pt_poff;
  int pt_E;
  int* status;                 // device status word (a bounded wait that expired)
  const int* stall_flag;       // test hook: waited on once per CTA (TMA-fed kernel) for stall_limit cycles
  long long stall_limit;
};

cudaError_t launch_route(const int32_t* topk_idx, const float* topk_prob, int Tk, int E, int capacity,
                         const int32_t* split_in, int32_t* split_out, int32_t* poffsets, int32_t* sorted_to_src,
                         int32_t* src_to_sorted, float* prob_perm, int* status, cudaStream_t st);
cudaError_t launch_quant(const QuantArgs& a, int batch, int num_sms, cudaStream_t st);
cudaError_t launch_unpermute(const bf16* rows, const int32_t* src_to_sorted, const float* probs, int64_t T, int k,
                             int64_t d, bf16* y, int num_sms, cudaStream_t st);
cudaError_t launch_dprob_reduce(const float* part, int n_parts, int64_t part_stride, const int32_t* sorted_to_src,
                                int64_t rows, const int32_t* src_to_sorted, int64_t Tk, float* d_prob,
                                cudaStream_t st);
// Per-tensor maxima (fp32 bits, atomicMax into ``amax`` which the caller zeroes first):
// amax[b] = max |x| over batch b of a [batch, rows, cols] bf16 source (per-batch pointers in
// ``src_ptrs``, or ``src`` with ``batch_stride`` elements between batches; rows ``ld`` apart) ...
cudaError_t launch_amax_batched(const PtrArray& src_ptrs, const bf16* src, int64_t batch_stride, int batch,
                                int64_t rows, int64_t cols, int64_t ld, uint32_t* amax, int num_sms,
                                cudaStream_t st);
// ... and amax[e] = max |x[t]| over the tokens t routed to expert e: the rows r of the expert-sorted
// order (``rows`` of them) with a slot sorted_to_src[r] >= 0 read token sorted_to_src[r] / k and
// belong to the expert e with poffsets[e] <= r < poffsets[e+1]; x is [T, d] with rows ``ld`` apart.
cudaError_t launch_amax_routed(const bf16* x, int64_t ld, int64_t d, const int32_t* sorted_to_src,
                               const int32_t* poffsets, int64_t rows, int k, int E, uint32_t* amax, int num_sms,
                               cudaStream_t st);
// In place: the fp32 bits of each of n tensor maxima become that tensor's per-tensor FP8 scale.
cudaError_t launch_fp8_scales(uint32_t* amax_to_scale, int n, int e5m2, cudaStream_t st);
cudaError_t launch_dequant(const uint8_t* q, const uint8_t* s, int64_t R, int64_t C, int sf_mma, float* out,
                           int num_sms, cudaStream_t st);

}  // namespace moemx
