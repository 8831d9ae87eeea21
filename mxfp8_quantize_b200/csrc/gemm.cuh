// Grouped GEMM on the sm_100a tensor cores (tcgen05) with fused epilogues.
#pragma once
#include <cuda.h>

#include "codec.cuh"

namespace moemx {

enum EpiKind : int {
  EPI_STORE = 0,    // fp32 accumulator -> bf16 rows
  EPI_SWIGLU = 1,   // gate/up accumulator -> a = silu(g)*u*p, requantised (ScaledSwiGLU)
  EPI_DSWIGLU = 2,  // da accumulator + saved h -> dh = [dg, du] requantised, dp partial sums
  EPI_FUSED_FWD = 3,  // the whole forward in one launch: gate_up tiles (EPI_SWIGLU epilogue), then
                      // down tiles (bf16 rows), each waiting for its rows of a
};

struct EpiArgs {
  // EPI_STORE
  bf16* out;          // M-grouped: [rows, ldo]
  int64_t ldo;
  PtrArray out_ptrs;  // K-grouped: per-expert outputs [M, ldo]
  // EPI_SWIGLU / EPI_DSWIGLU
  int64_t f;          // ffn width
  int64_t cap;        // padded row capacity (token axis of the transposed outputs)
  const float* p_perm;
  bf16* h;            // [cap, 2f] saved gate/up pre-activations (written by SWIGLU, read by DSWIGLU)
  uint8_t* h_q;       // ... or saved as MXFP8 (E4M3 codes [cap, 2f], blocks of 32 along 2f)
  uint8_t* h_s;       //     with their E8M0 scales, row-major [cap, 2f/32]
  uint8_t* q_row;     // MXFP8 row-wise codes ([cap, f] for a, [cap, 2f] for dh)
  uint8_t* s_row;     // their scales, tensor-core tile layout
  uint8_t* q_colT;    // MXFP8 codes transposed ([f, cap] / [2f, cap])
  uint8_t* s_colT;
  bf16* o_row;        // BF16 path equivalents
  bf16* o_colT;
  float* dump;        // debug: fp32 values before quantisation
  int scale_floor;    // MXFP8 shared exponent of the requantisations: 0 round-up rule, 1 OCP floor rule
  int grad_e5m2;      // DSWIGLU: dh requantised with E5M2 elements (gradient-format variant)
  float* dp_part;     // DSWIGLU: [parts * n_tiles, cap] partial sums of the probability gradient
  uint32_t* amax_out; // per-tensor FP8 (bf16 o_row outputs): per expert, the largest magnitude written,
                      // as fp32 bits (atomicMax; the caller zeroes it)
};

struct GemmArgs {
  CUtensorMap tmap_a;  // A: 2-D [rows, K] K-contiguous, box 128 rows x 128 bytes, 128B swizzle
  CUtensorMap tmap_b;  // B: 3-D [E, rows, K] (M-grouped) or 2-D [rows, K] (K-grouped); box BN rows (bf16
                       // gate_up: BN/2, one box of gate rows and one of up rows)
  CUtensorMap tmap_h;  // dSwiGLU: saved h [cap, 2f] bf16, box 128 rows x 64 columns, 128B swizzle
  // MXFP8 scales of A and B in the tile layout, as 3-D u32 arrays [row tiles][kb4][128]: one box is
  // the 512-byte tile of one 128-K step for one (A) or BN/128 (B) consecutive 128-row blocks
  CUtensorMap tmap_sfa;
  CUtensorMap tmap_sfb;
  int kgrouped;        // 0: M grouped by expert (rows of A = expert segments); 1: K grouped (wgrad)
  int E;
  int K;               // M-grouped reduction length
  int n_tiles;         // output tiles along N per expert
  int m_tiles;         // K-grouped: M / 128
  int gate_up_half;    // B tile made of two 128-row boxes: gate rows nb*128, up rows gate_up_half + nb*128
                       // (bf16 gate_up GEMM reading the unpermuted weights); 0 = BN/128 boxes of 128 rows
  const int32_t* poffsets;
  const uint8_t* sfa;  // MXFP8 scales of A / B in the tile layout
  int64_t sfa_kb4;     // 128-wide K blocks per 128-row block of A's scales
  const uint8_t* sfb;
  int64_t sfb_kb4;
  int64_t sfb_expert_rows;  // rows of B per expert (M-grouped), for the scale tile index
  int a_e5m2;          // MXFP8 / FP8: A's elements are E5M2 (B's stay E4M3)
  // per-tensor FP8 (with mx = false): 8-bit operands without block scales, kind::f8f6f4 MMAs over
  // 128-element K steps; the epilogue multiplies the accumulator of expert e by
  // 1/s_a(e) * 1/s_b(e), s = fp8_tensor_scale of pt_amax_a[e] (A's format) and pt_amax_b[e] (E4M3)
  int fp8;
  const uint32_t* pt_amax_a;
  const uint32_t* pt_amax_b;
  // EPI_FUSED_FWD: the down GEMM that follows the gate_up tiles (A = a [rows, f], B = W2 [E, d, f]),
  // its output rows go to epi.out / epi.ldo
  CUtensorMap tmap_a2;
  CUtensorMap tmap_b2;
  CUtensorMap tmap_sfa2;
  CUtensorMap tmap_sfb2;
  int K2;              // the down GEMM's reduction length (f)
  int n_tiles2;        // its output tiles per 128-row block (d / BN)
  int64_t sfb_expert_rows2;
  int* mblock_done;    // per 128-row block: epilogue-warp completions of its gate_up tiles (zeroed by the
                       // caller before the launch); a down tile starts once all n_tiles x warps arrived
  int* status;
  // test hook: a device flag nothing sets; when non-null the producer of each CTA waits on it once,
  // for at most stall_limit cycles, after issuing the first stages of its first tile
  const int* stall_flag;
  long long stall_limit;
  EpiArgs epi;
};

// Output tile width (N) of the kernel used for an epilogue kind.
int gemm_tile_n(int epi);
// Rows of B per tensor-map box of the kernel used for an epilogue kind (half the tile's N for the
// CTA-pair instances).
int gemm_b_box_rows(bool mx, int epi);
// Partial sums of the probability gradient the dSwiGLU epilogue writes per output tile and row.
int gemm_dswiglu_parts();

// Launch one grouped GEMM.  ``mx``: MXFP8 (kind::mxf8f6f4); otherwise BF16 (kind::f16), or per-tensor
// FP8 (kind::f8f6f4) when args.fp8 is set.
cudaError_t launch_grouped_gemm(const GemmArgs& args, bool mx, int epi, int num_sms, cudaStream_t st);

// Tensor-core peak loop (peak.cu): one CTA per SM issuing iters x 4 MMAs of 128 x 256 on operands
// resident in shared memory (kind 0 BF16, 1 MXFP8, 2 per-tensor FP8); its FLOPs per launch.
cudaError_t launch_tensor_peak(int kind, long long iters, int scale_refresh, int num_sms, int* status,
                               cudaStream_t st);
double tensor_peak_flops(int kind, int num_sms, long long iters);

}  // namespace moemx
