// C ABI of libmoemx (declared in include/moemx.h): argument checks, buffer layout of the
// saved / workspace regions, TMA tensor maps, and the launch sequence of the fused layer.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "codec.cuh"
#include "common.cuh"
#include "gemm.cuh"

using namespace moemx;

struct moe_ctx_s {
  int device;
  int num_sms;
  int* d_status;  // [0] status bits
  float* dbg_a;
  float* dbg_dh;
  moe_launch_hook_t hook;
  void* hook_user;
  int scale_floor;          // MXFP8 shared-exponent rule of the fused layer (moe_ctx_set_scale_rule)
  int grad_e5m2;            // MXFP8 gradient operands in E5M2 (moe_ctx_set_grad_format)
  int saved_h;              // format of the h a training forward saves (moe_ctx_set_saved_h)
  int fused_fwd;            // both forward GEMMs in one launch (moe_ctx_set_fused_forward)
  int stall;                // test hook for the bounded waits (moe_ctx_set_test_stall)
  long long stall_limit;
};

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

// 2-D map over [rows, inner] (inner contiguous), box ``box_rows`` rows x 128 bytes, 128-byte swizzle.
bool map_2d(CUtensorMap* m, const void* base, bool fp8, uint64_t inner, uint64_t rows, uint64_t row_bytes,
            uint32_t box_rows = 128) {
  const CUtensorMapDataType dt = fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {fp8 ? 128u : 64u, box_rows};
  cuuint32_t es[2] = {1, 1};
  return g_encode(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// 3-D map over [E, rows, inner] with an arbitrary (16-byte multiple) stride between experts.
bool map_3d(CUtensorMap* m, const void* base, bool fp8, uint64_t inner, uint64_t rows, uint64_t E,
            uint64_t row_bytes, uint64_t expert_bytes, uint32_t box_rows = 128) {
  const CUtensorMapDataType dt = fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  cuuint64_t dims[3] = {inner, rows, E};
  cuuint64_t strides[2] = {row_bytes, expert_bytes};
  cuuint32_t box[3] = {fp8 ? 128u : 64u, box_rows, 1u};
  cuuint32_t es[3] = {1, 1, 1};
  return g_encode(m, dt, 3, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A scale buffer in the tensor-core tile layout (512-byte tiles, [rows/128][kb4]) as a 3-D u32
// array [rows/128][kb4][128]; a box is ``box_tiles`` tiles of consecutive 128-row blocks at one kb4.
bool map_sf(CUtensorMap* m, const void* base, uint64_t rows, int64_t kb4, uint32_t box_tiles) {
  cuuint64_t dims[3] = {128, static_cast<uint64_t>(kb4), rows / 128};
  cuuint64_t strides[2] = {512, static_cast<uint64_t>(kb4) * 512};
  cuuint32_t box[3] = {128, 1, box_tiles};
  cuuint32_t es[3] = {1, 1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// Scale maps of a GEMM's A (``a_rows`` rows) and B (``b_rows`` rows over all experts) operands, for
// the kernel whose tiles are ``bn`` wide.
bool sf_maps(GemmArgs& g, uint64_t a_rows, uint64_t b_rows, int bn) {
  return map_sf(&g.tmap_sfa, g.sfa, a_rows, g.sfa_kb4, 1) &&
         map_sf(&g.tmap_sfb, g.sfb, b_rows, g.sfb_kb4, static_cast<uint32_t>(bn / 128));
}

// MXFP8 with the tensor-core scale layout: code tiles are written by TMA tensor stores (uint8 maps
// over [batch*rows, cols] and [batch*cols, rows], 128 x 128 boxes, 128-byte swizzle).
int64_t uniform_stride(const void* const* p, int E, int64_t min_bytes);

// TMA source map of a quantisation pass when the persistent kernel can take it: one uniformly
// strided [batch, rows, cols] bf16 source with 16-byte aligned rows, rows and cols multiples of 128.
void quant_load_map(QuantArgs& a, int batch) {
  a.tma_load = 0;
  a.tma_gather = 0;
  const bool outputs_ok = a.mx ? a.do_row : (a.do_col && !a.do_row);  // the kernel's modes
  if (a.rows % 128 || a.cols % 128 || !outputs_ok) return;
  if (a.sorted_to_src) {
    // MXFP8 gather of one [src_rows, cols] source: rows fetched four at a time by tile::gather4
    // through a map whose box is one row of 128 columns
    if (!a.mx || batch != 1 || a.src_ptrs.p[0] || !a.src || !aligned16(a.src) || ((a.src_ld * 2) & 15) ||
        a.src_rows <= 0 || a.src_rows >= (int64_t(1) << 31))
      return;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.cols), static_cast<cuuint64_t>(a.src_rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.src_ld) * 2};
    cuuint32_t box[2] = {128, 1};
    cuuint32_t es[2] = {1, 1};
    if (g_encode(&a.tmap_src, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<bf16*>(a.src), dims, strides, box, es,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS) {
      a.tma_load = 1;
      a.tma_gather = 1;
    }
    return;
  }
  const void* base = a.src_ptrs.p[0] ? a.src_ptrs.p[0] : a.src;
  const int64_t row_bytes = a.src_ld * 2, tile_bytes = a.rows * row_bytes;
  int64_t stride = a.src_ptrs.p[0] ? uniform_stride(a.src_ptrs.p, batch, tile_bytes) : a.src_batch_stride * 2;
  if (batch == 1) stride = tile_bytes;
  if (!base || !aligned16(base) || (row_bytes & 15) || stride <= 0 || (stride & 15) || stride < tile_bytes) return;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(a.cols), static_cast<cuuint64_t>(a.rows), static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(stride)};
  cuuint32_t box[3] = {128, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  if (g_encode(&a.tmap_src, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
    a.tma_load = 1;
}

bool quant_store_maps(QuantArgs& a, int batch) {
  a.tma_store = 0;
  a.tma_load = 0;
  if (!a.mx) {
    // bf16 transpose of a strided source: the TMA-fed kernel writes the transposed tiles through
    // a bf16 map over [batch*cols, rows] (boxes of 64 columns x 128 rows); otherwise the tile kernel
    quant_load_map(a, batch);
    if (!a.tma_load) return true;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.rows), static_cast<cuuint64_t>(batch) * a.cols};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.rows) * 2};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t es[2] = {1, 1};
    if (!aligned16(a.o_colT) ||
        g_encode(&a.tmap_qcol, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.o_colT, dims, strides, box, es,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
      a.tma_load = 0;
      return true;
    }
    a.tma_store = 1;
    return true;
  }
  if (!a.sf_mma) return true;
  const uint64_t R = a.rows, C = a.cols, B = batch;
  cuuint32_t box[2] = {128, 128};
  cuuint32_t es[2] = {1, 1};
  if (a.do_row) {
    cuuint64_t dims[2] = {C, B * R};
    cuuint64_t strides[1] = {C};
    if (g_encode(&a.tmap_qrow, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, a.q_row, dims, strides, box, es,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  if (a.do_col) {
    cuuint64_t dims[2] = {R, B * C};
    cuuint64_t strides[1] = {R};
    if (g_encode(&a.tmap_qcol, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, a.q_colT, dims, strides, box, es,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  a.tma_store = 1;
  quant_load_map(a, batch);
  return true;
}

// Bump allocator over a caller buffer (1 KiB granules); with base == nullptr it only measures.
struct Carve {
  uint8_t* base;
  size_t off = 0;
  explicit Carve(void* b) : base(static_cast<uint8_t*>(b)) {}
  template <class T>
  T* take(size_t bytes) {
    off = (off + 1023) & ~size_t(1023);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += bytes;
    return p;
  }
};

struct Dims {
  int64_t T, d, f, cap, Tk;
  int E, k;
  bool mx;      // MXFP8
  bool fp8;     // per-tensor FP8
  bool q8;      // 8-bit GEMM operands (either of the two)
  int saved_h;  // MOE_SAVED_H_BF16 or MOE_SAVED_H_MXFP8
};

// Everything a training forward leaves for the backward.
struct Saved {
  int32_t *split, *poff, *s2src, *src2s;
  float* pperm;
  uint8_t *w1c_q, *w1c_s, *w2c_q, *w2c_s;  // MXFP8: weights quantised down the columns, transposed
  uint8_t *xT_q, *xT_s, *aT_q, *aT_s;      // MXFP8: token-axis quantised x and a, transposed
  bf16 *xT, *aT;                           // BF16: transposed copies
  bf16* h;                                 // [cap, 2f] gate/up pre-activations (bf16) ...
  uint8_t *h_q, *h_s;                      // ... or as MXFP8: codes [cap, 2f], scales [cap, 2f/32] ...
  uint8_t *xr_q, *xr_s;                    // ... or not at all (recompute): x's gate_up operand instead,
  bf16* xr;                                //     MXFP8 row-wise codes + scales, or the BF16 gathered rows
  uint32_t* pt_amax;                       // per-tensor FP8: [4][E] tensor maxima (fp32 bits) of x, W1, W2, a
};
void carve_saved(Carve& c, const Dims& D, Saved& s, bool full = true) {
  s.split = c.take<int32_t>(D.E * 4);
  s.poff = c.take<int32_t>((D.E + 1) * 4);
  s.s2src = c.take<int32_t>(D.cap * 4);
  s.src2s = c.take<int32_t>(D.Tk * 4);
  s.pperm = c.take<float>(D.cap * 4);
  s.w1c_q = s.w1c_s = s.w2c_q = s.w2c_s = s.xT_q = s.xT_s = s.aT_q = s.aT_s = nullptr;
  s.xT = s.aT = nullptr;
  s.h = nullptr;
  s.h_q = s.h_s = nullptr;
  s.xr_q = s.xr_s = nullptr;
  s.xr = nullptr;
  s.pt_amax = nullptr;
  if (!full) return;  // inference: routing bookkeeping only
  if (D.fp8) {  // per-tensor FP8: codes only (one quantisation serves both of a tensor's GEMMs)
    s.w1c_q = c.take<uint8_t>(D.E * D.d * 2 * D.f);
    s.w2c_q = c.take<uint8_t>(D.E * D.f * D.d);
    s.xT_q = c.take<uint8_t>(D.d * D.cap);
    s.aT_q = c.take<uint8_t>(D.f * D.cap);
    s.pt_amax = c.take<uint32_t>(4 * D.E * 4);
  } else if (D.mx) {
    s.w1c_q = c.take<uint8_t>(D.E * D.d * 2 * D.f);
    s.w1c_s = c.take<uint8_t>(D.E * D.d * 2 * D.f / 32);
    s.w2c_q = c.take<uint8_t>(D.E * D.f * D.d);
    s.w2c_s = c.take<uint8_t>(D.E * D.f * D.d / 32);
    s.xT_q = c.take<uint8_t>(D.d * D.cap);
    s.xT_s = c.take<uint8_t>(D.d * D.cap / 32);
    s.aT_q = c.take<uint8_t>(D.f * D.cap);
    s.aT_s = c.take<uint8_t>(D.f * D.cap / 32);
  } else {
    s.xT = c.take<bf16>(D.d * D.cap * 2);
    s.aT = c.take<bf16>(D.f * D.cap * 2);
  }
  if (D.saved_h == MOE_SAVED_H_MXFP8) {
    s.h_q = c.take<uint8_t>(D.cap * 2 * D.f);
    s.h_s = c.take<uint8_t>(D.cap * 2 * D.f / 32);
  } else if (D.saved_h == MOE_SAVED_H_RECOMPUTE) {
    if (D.mx) {
      s.xr_q = c.take<uint8_t>(D.cap * D.d);
      s.xr_s = c.take<uint8_t>(D.cap * D.d / 32);
    } else {
      s.xr = c.take<bf16>(D.cap * D.d * 2);
    }
  } else {
    s.h = c.take<bf16>(D.cap * 2 * D.f * 2);
  }
}

struct FwdWs {
  uint8_t *w1_q, *w1_s, *w2_q, *w2_s, *x_q, *x_s, *a_q, *a_s;
  bf16 *x_perm, *a, *w1_copy, *w2_copy;
  bf16* y_perm;
  int* mblk;          // fused forward: completion counters per 128-row block
  uint32_t* pt_amax;  // per-tensor FP8 inference: [4][E] tensor maxima of x, W1, W2, a
};
void carve_fwd(Carve& c, const Dims& D, FwdWs& w) {
  std::memset(&w, 0, sizeof(w));
  if (D.fp8) {  // codes of W1 [E, 2f, d], W2 [E, d, f], x [cap, d]; a in bf16 [cap, f] and its codes
    w.w1_q = c.take<uint8_t>(D.E * 2 * D.f * D.d);
    w.w2_q = c.take<uint8_t>(D.E * D.d * D.f);
    w.x_q = c.take<uint8_t>(D.cap * D.d);
    w.a = c.take<bf16>(D.cap * D.f * 2);
    w.a_q = c.take<uint8_t>(D.cap * D.f);
    w.pt_amax = c.take<uint32_t>(4 * D.E * 4);
  } else if (D.mx) {
    w.w1_q = c.take<uint8_t>(D.E * 2 * D.f * D.d);
    w.w1_s = c.take<uint8_t>(D.E * 2 * D.f * D.d / 32);
    w.w2_q = c.take<uint8_t>(D.E * D.d * D.f);
    w.w2_s = c.take<uint8_t>(D.E * D.d * D.f / 32);
    w.x_q = c.take<uint8_t>(D.cap * D.d);
    w.x_s = c.take<uint8_t>(D.cap * D.d / 32);
    w.a_q = c.take<uint8_t>(D.cap * D.f);
    w.a_s = c.take<uint8_t>(D.cap * D.f / 32);
  } else {
    w.x_perm = c.take<bf16>(D.cap * D.d * 2);
    w.a = c.take<bf16>(D.cap * D.f * 2);
    w.w1_copy = c.take<bf16>(D.E * 2 * D.f * D.d * 2);
    w.w2_copy = c.take<bf16>(D.E * D.d * D.f * 2);
  }
  w.y_perm = c.take<bf16>(D.cap * D.d * 2);
  w.mblk = c.take<int>(D.cap / 128 * sizeof(int));
}

struct BwdWs {
  uint32_t* pt_amax;  // per-tensor FP8: [2][E] tensor maxima (fp32 bits) of dy, dh
  uint8_t *dy_q, *dy_s, *dyT_q, *dyT_s, *dh_q, *dh_s, *dhT_q, *dhT_s;
  bf16 *dy_perm, *dyT, *dh, *dhT, *w1T, *w2T;
  bf16* dx_perm;
  float* dp_part;
  bf16* hr;               // recompute: h regenerated by the gate_up GEMM
  uint8_t *w1r_q, *w1r_s;  // recompute, MXFP8: W1 quantised again (row-wise, gate/up interleaved)
  bf16* w1r_copy;          // recompute, BF16: W1 gathered when the experts are not evenly spaced
};
void carve_bwd(Carve& c, const Dims& D, BwdWs& w) {
  std::memset(&w, 0, sizeof(w));
  if (D.fp8) {  // codes of dy both ways; dh in bf16 [cap, 2f] and its codes both ways
    w.dy_q = c.take<uint8_t>(D.cap * D.d);
    w.dyT_q = c.take<uint8_t>(D.d * D.cap);
    w.dh = c.take<bf16>(D.cap * 2 * D.f * 2);
    w.dh_q = c.take<uint8_t>(D.cap * 2 * D.f);
    w.dhT_q = c.take<uint8_t>(2 * D.f * D.cap);
    w.pt_amax = c.take<uint32_t>(2 * D.E * 4);
  } else if (D.mx) {
    w.dy_q = c.take<uint8_t>(D.cap * D.d);
    w.dy_s = c.take<uint8_t>(D.cap * D.d / 32);
    w.dyT_q = c.take<uint8_t>(D.d * D.cap);
    w.dyT_s = c.take<uint8_t>(D.d * D.cap / 32);
    w.dh_q = c.take<uint8_t>(D.cap * 2 * D.f);
    w.dh_s = c.take<uint8_t>(D.cap * 2 * D.f / 32);
    w.dhT_q = c.take<uint8_t>(2 * D.f * D.cap);
    w.dhT_s = c.take<uint8_t>(2 * D.f * D.cap / 32);
  } else {
    w.dy_perm = c.take<bf16>(D.cap * D.d * 2);
    w.dyT = c.take<bf16>(D.d * D.cap * 2);
    w.dh = c.take<bf16>(D.cap * 2 * D.f * 2);
    w.dhT = c.take<bf16>(2 * D.f * D.cap * 2);
    w.w1T = c.take<bf16>(D.E * D.d * 2 * D.f * 2);
    w.w2T = c.take<bf16>(D.E * D.f * D.d * 2);
  }
  w.dx_perm = c.take<bf16>(D.cap * D.d * 2);
  w.dp_part = c.take<float>(gemm_dswiglu_parts() * (D.f / gemm_tile_n(EPI_DSWIGLU)) * D.cap * 4);
  if (D.saved_h == MOE_SAVED_H_RECOMPUTE) {
    w.hr = c.take<bf16>(D.cap * 2 * D.f * 2);
    if (D.mx) {
      w.w1r_q = c.take<uint8_t>(D.E * 2 * D.f * D.d);
      w.w1r_s = c.take<uint8_t>(D.E * 2 * D.f * D.d / 32);
    } else {
      w.w1r_copy = c.take<bf16>(D.E * 2 * D.f * D.d * 2);
    }
  }
}

int64_t capacity_rows(int64_t T, int k, int E) {
  return round_up(T * k + static_cast<int64_t>(E) * (MOE_ROW_ALIGN - 1), MOE_ROW_ALIGN);
}

moe_status_t check_dims(int64_t T, int64_t d, int64_t f, int E, int k) {
  if (T <= 0 || d <= 0 || f <= 0) return MOE_ERR_INVALID_ARG;
  if (E < 1 || E > MOE_MAX_EXPERTS || k < 1 || k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
  if (d % 256 || f % 256) return MOE_ERR_SHAPE;
  if (capacity_rows(T, k, E) >= (int64_t(1) << 31) / 2) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

Dims make_dims(int64_t T, int64_t d, int64_t f, int E, int k, moe_precision_t prec, int saved_h = 0) {
  Dims D;
  D.saved_h = saved_h;
  D.T = T;
  D.d = d;
  D.f = f;
  D.E = E;
  D.k = k;
  D.Tk = T * k;
  D.cap = capacity_rows(T, k, E);
  D.mx = prec == MOE_PREC_MXFP8;
  D.fp8 = prec == MOE_PREC_FP8;
  D.q8 = D.mx || D.fp8;
  return D;
}

struct DeviceGuard {
  int prev = -1;
  explicit DeviceGuard(int dev) {
    cudaGetDevice(&prev);
    if (prev != dev) cudaSetDevice(dev);
  }
  ~DeviceGuard() {
    int cur = -1;
    cudaGetDevice(&cur);
    if (prev >= 0 && cur != prev) cudaSetDevice(prev);
  }
};

#define MOE_CUDA(x)                       \
  do {                                    \
    if ((x) != cudaSuccess) return MOE_ERR_CUDA; \
  } while (0)

// Enqueue one kernel, calling the context's launch hook around it.
#define MOE_LAUNCH(ctx, name, st, x)                                          \
  do {                                                                        \
    if ((ctx)->hook) (ctx)->hook((ctx)->hook_user, name, 0, (void*)(st));     \
    const cudaError_t moe_launch_err_ = (x);                                  \
    if ((ctx)->hook) (ctx)->hook((ctx)->hook_user, name, 1, (void*)(st));     \
    if (moe_launch_err_ != cudaSuccess) return MOE_ERR_CUDA;                  \
  } while (0)

// Uniform byte stride between consecutive expert pointers (0 if not uniform / not usable by TMA).
int64_t uniform_stride(const void* const* p, int E, int64_t min_bytes) {
  if (E == 1) return min_bytes;
  const int64_t s = reinterpret_cast<const uint8_t*>(p[1]) - reinterpret_cast<const uint8_t*>(p[0]);
  if (s < min_bytes || (s & 15)) return 0;
  for (int e = 2; e < E; ++e)
    if (reinterpret_cast<const uint8_t*>(p[e]) - reinterpret_cast<const uint8_t*>(p[e - 1]) != s) return 0;
  return s;
}

// Word of the context's status block that nothing ever writes (zeroed at creation): the flag the
// test hook's waits can only give up on.
constexpr int kNeverSetWord = 32;

QuantArgs quant_args(moe_ctx_t ctx) {
  QuantArgs a;
  std::memset(&a, 0, sizeof(a));
  a.status = ctx->d_status;
  a.scale_floor = ctx->scale_floor;
  if (ctx->stall) {
    a.stall_flag = ctx->d_status + kNeverSetWord;
    a.stall_limit = ctx->stall_limit;
  }
  return a;
}

GemmArgs gemm_args(moe_ctx_t ctx) {
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  g.status = ctx->d_status;
  g.epi.scale_floor = ctx->scale_floor;
  if (ctx->stall) {
    g.stall_flag = ctx->d_status + kNeverSetWord;
    g.stall_limit = ctx->stall_limit;
  }
  return g;
}

// Per-tensor FP8 codes of E expert matrices [rows, cols] (bf16 at ptrs[e], rows contiguous): row-wise
// into q_row [E, rows, cols] and, when q_colT is set, transposed into q_colT [E, cols, rows], each
// expert with the scale of amax[e].  One launch over all experts when they are evenly spaced, else
// one launch per expert.
moe_status_t quant_experts_fp8(moe_ctx_t ctx, const char* name, const void* const* ptrs, int E, int64_t rows,
                               int64_t cols, const uint32_t* amax, uint8_t* q_row, uint8_t* q_colT, cudaStream_t st) {
  QuantArgs a = quant_args(ctx);
  a.src_ld = cols;
  a.rows = rows;
  a.cols = cols;
  a.mx = 1;
  a.sf_mma = 1;
  a.scale_floor = 0;
  a.do_row = 1;
  a.do_col = q_colT != nullptr;
  if (uniform_stride(ptrs, E, rows * cols * 2)) {
    for (int e = 0; e < E; ++e) a.src_ptrs.p[e] = ptrs[e];
    a.pt_amax = amax;
    a.q_row = q_row;
    a.q_colT = q_colT;
    if (!quant_store_maps(a, E)) return MOE_ERR_CUDA;
    MOE_LAUNCH(ctx, name, st, launch_quant(a, E, ctx->num_sms, st));
    return MOE_OK;
  }
  for (int e = 0; e < E; ++e) {
    a.src = static_cast<const bf16*>(ptrs[e]);
    a.pt_amax = amax + e;
    a.q_row = q_row + e * rows * cols;
    a.q_colT = q_colT ? q_colT + e * cols * rows : nullptr;
    if (!quant_store_maps(a, 1)) return MOE_ERR_CUDA;
    MOE_LAUNCH(ctx, name, st, launch_quant(a, 1, ctx->num_sms, st));
  }
  return MOE_OK;
}

// Per-tensor FP8 codes of one [cap, cols] bf16 tensor of expert segments (a, dh): row-wise into
// q_row and, when q_colT is set, transposed into q_colT [cols, cap], each 128-row block with the scale
// of its expert's amax.
moe_status_t quant_segments_fp8(moe_ctx_t ctx, const char* name, const bf16* src, int64_t cap, int64_t cols,
                                const int32_t* poff, int E, const uint32_t* amax, int e5m2, uint8_t* q_row,
                                uint8_t* q_colT, cudaStream_t st) {
  QuantArgs a = quant_args(ctx);
  a.src = src;
  a.src_ld = cols;
  a.rows = cap;
  a.cols = cols;
  a.mx = 1;
  a.sf_mma = 1;
  a.scale_floor = 0;
  a.e5m2 = e5m2;
  a.do_row = 1;
  a.q_row = q_row;
  a.do_col = q_colT != nullptr;
  a.q_colT = q_colT;
  a.pt_amax = amax;
  a.pt_poff = poff;
  a.pt_E = E;
  if (!quant_store_maps(a, 1)) return MOE_ERR_CUDA;
  MOE_LAUNCH(ctx, name, st, launch_quant(a, 1, ctx->num_sms, st));
  return MOE_OK;
}

}  // namespace

// ====================================================================================== ABI

extern "C" {

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_SHAPE: return "shape breaks an alignment rule";
    case MOE_ERR_UNSUPPORTED: return "unsupported device or size";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE: return "device-detected error (bad expert index or split_sizes mismatch)";
    case MOE_ERR_TIMEOUT: return "bounded in-kernel wait expired";
    case MOE_ERR_WORKSPACE: return "workspace or saved buffer too small";
  }
  return "unknown status";
}

moe_status_t moe_ctx_create(moe_ctx_t* out, int device) {
  if (!out) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, device) != cudaSuccess) return MOE_ERR_CUDA;
  if (prop.major != 10 || prop.minor != 0) return MOE_ERR_UNSUPPORTED;
  if (!encoder()) return MOE_ERR_CUDA;
  DeviceGuard guard(device);
  moe_ctx_s* c = new moe_ctx_s();
  c->device = device;
  c->num_sms = prop.multiProcessorCount;
  c->dbg_a = c->dbg_dh = nullptr;
  c->hook = nullptr;
  c->hook_user = nullptr;
  c->scale_floor = 0;
  c->grad_e5m2 = 0;
  c->saved_h = MOE_SAVED_H_BF16;
  c->fused_fwd = 0;
  c->stall = 0;
  c->stall_limit = 0;
  if (cudaMalloc(&c->d_status, 256) != cudaSuccess) {
    delete c;
    return MOE_ERR_CUDA;
  }
  if (cudaMemset(c->d_status, 0, 256) != cudaSuccess) {
    cudaFree(c->d_status);
    delete c;
    return MOE_ERR_CUDA;
  }
  *out = c;
  return MOE_OK;
}

moe_status_t moe_ctx_destroy(moe_ctx_t ctx) {
  if (!ctx) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(ctx->device);
  cudaFree(ctx->d_status);
  delete ctx;
  return MOE_OK;
}

moe_status_t moe_ctx_set_debug_dump(moe_ctx_t ctx, float* a_f32, float* dh_f32) {
  if (!ctx) return MOE_ERR_INVALID_ARG;
  ctx->dbg_a = a_f32;
  ctx->dbg_dh = dh_f32;
  return MOE_OK;
}

moe_status_t moe_ctx_set_launch_hook(moe_ctx_t ctx, moe_launch_hook_t hook, void* user) {
  if (!ctx) return MOE_ERR_INVALID_ARG;
  ctx->hook = hook;
  ctx->hook_user = user;
  return MOE_OK;
}

moe_status_t moe_ctx_set_test_stall(moe_ctx_t ctx, int stall, int64_t limit_cycles) {
  if (!ctx || (stall && (limit_cycles <= 0 || limit_cycles > kWaitLimitCycles))) return MOE_ERR_INVALID_ARG;
  ctx->stall = stall ? 1 : 0;
  ctx->stall_limit = stall ? limit_cycles : 0;
  return MOE_OK;
}

moe_status_t moe_ctx_set_scale_rule(moe_ctx_t ctx, int rule) {
  if (!ctx || (rule != MXFP8_SCALE_ROUND_UP && rule != MXFP8_SCALE_FLOOR)) return MOE_ERR_INVALID_ARG;
  ctx->scale_floor = rule == MXFP8_SCALE_FLOOR ? 1 : 0;
  return MOE_OK;
}

moe_status_t moe_ctx_set_grad_format(moe_ctx_t ctx, int fmt) {
  if (!ctx || (fmt != MOE_GRAD_E4M3 && fmt != MOE_GRAD_E5M2)) return MOE_ERR_INVALID_ARG;
  ctx->grad_e5m2 = fmt == MOE_GRAD_E5M2 ? 1 : 0;
  return MOE_OK;
}

moe_status_t moe_ctx_set_saved_h(moe_ctx_t ctx, int mode) {
  if (!ctx || mode < MOE_SAVED_H_BF16 || mode > MOE_SAVED_H_RECOMPUTE) return MOE_ERR_INVALID_ARG;
  ctx->saved_h = mode;
  return MOE_OK;
}

moe_status_t moe_ctx_set_fused_forward(moe_ctx_t ctx, int on) {
  if (!ctx) return MOE_ERR_INVALID_ARG;
  ctx->fused_fwd = on ? 1 : 0;
  return MOE_OK;
}

moe_status_t moe_get_status(moe_ctx_t ctx, void* stream) {
  if (!ctx) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(ctx->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  int word = 0;
  if (cudaMemcpy(&word, ctx->d_status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (word && cudaMemset(ctx->d_status, 0, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  if (word & kStatusTimeout) return MOE_ERR_TIMEOUT;
  if (word & kStatusDevice) return MOE_ERR_DEVICE;
  return MOE_OK;
}

int64_t moe_capacity_rows(int64_t T, int k, int E) {
  if (T < 0 || k < 1 || E < 1) return 0;
  return capacity_rows(T, k, E);
}

moe_status_t mxfp8_quantize(moe_ctx_t ctx, const void* x, int64_t batch, int64_t rows, int64_t cols, int flags,
                            uint8_t* q_row, uint8_t* s_row, uint8_t* q_colT, uint8_t* s_colT, void* stream) {
  if (!ctx || !x || batch <= 0 || rows <= 0 || cols <= 0) return MOE_ERR_INVALID_ARG;
  const bool row = flags & MXFP8_ROWWISE, col = flags & MXFP8_COLWISE_T, mma = flags & MXFP8_SF_MMA_LAYOUT;
  if ((flags & ~31) || !(row || col)) return MOE_ERR_INVALID_ARG;
  if (row && (!q_row || !s_row)) return MOE_ERR_INVALID_ARG;
  if (col && (!q_colT || !s_colT)) return MOE_ERR_INVALID_ARG;
  if (cols % 32) return MOE_ERR_SHAPE;
  if (col && rows % 32) return MOE_ERR_SHAPE;
  if (mma && (rows % 128 || cols % 128)) return MOE_ERR_SHAPE;
  if (batch > 65535 || ceil_div(rows, 128) > 65535 || ceil_div(cols, 128) > (int64_t(1) << 31) - 1)
    return MOE_ERR_UNSUPPORTED;
  if (!aligned16(x) || (row && !aligned16(q_row)) || (col && !aligned16(q_colT))) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(ctx->device);
  QuantArgs a = quant_args(ctx);
  a.src = static_cast<const bf16*>(x);
  a.src_batch_stride = rows * cols;
  a.src_ld = cols;
  a.rows = rows;
  a.cols = cols;
  a.mx = 1;
  a.do_row = row;
  a.do_col = col;
  a.sf_mma = mma;
  a.scale_floor = (flags & MXFP8_FLAG_SCALE_FLOOR) ? 1 : 0;
  a.e5m2 = (flags & MXFP8_FLAG_E5M2) ? 1 : 0;
  a.q_row = q_row;
  a.s_row = s_row;
  a.q_colT = q_colT;
  a.s_colT = s_colT;
  if (!quant_store_maps(a, static_cast<int>(batch))) return MOE_ERR_CUDA;
  MOE_LAUNCH(ctx, "mxfp8_quantize", stream, launch_quant(a, static_cast<int>(batch), ctx->num_sms, static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status_t mxfp8_dequantize(moe_ctx_t ctx, const uint8_t* q, const uint8_t* s, int64_t rows, int64_t cols,
                              int sf_mma_layout, float* out, void* stream) {
  if (!ctx || !q || !s || !out || rows <= 0 || cols <= 0) return MOE_ERR_INVALID_ARG;
  if (cols % 32) return MOE_ERR_SHAPE;
  if (sf_mma_layout && (rows % 128 || cols % 128)) return MOE_ERR_SHAPE;
  DeviceGuard guard(ctx->device);
  MOE_LAUNCH(ctx, "mxfp8_dequantize", stream, launch_dequant(q, s, rows, cols, sf_mma_layout, out, ctx->num_sms, static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status_t fp8_quantize(moe_ctx_t ctx, const void* x, int64_t batch, int64_t rows, int64_t cols, int flags,
                          uint8_t* q_row, uint8_t* q_colT, float* scale, void* stream) {
  if (!ctx || !x || !scale || batch <= 0 || rows <= 0 || cols <= 0) return MOE_ERR_INVALID_ARG;
  const bool col = flags & FP8_COLWISE_T;
  if ((flags & ~(FP8_ROWWISE | FP8_COLWISE_T | FP8_FLAG_E5M2)) || !(flags & FP8_ROWWISE) || !q_row ||
      (col && !q_colT))
    return MOE_ERR_INVALID_ARG;
  if (rows % 128 || cols % 128) return MOE_ERR_SHAPE;
  if (batch > MOE_MAX_EXPERTS || rows * cols >= (int64_t(1) << 40)) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(q_row) || (col && !aligned16(q_colT))) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(ctx->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int e5m2 = (flags & FP8_FLAG_E5M2) ? 1 : 0;
  uint32_t* amax = reinterpret_cast<uint32_t*>(scale);  // the maxima first; the scales replace them at the end
  MOE_CUDA(cudaMemsetAsync(amax, 0, static_cast<size_t>(batch) * sizeof(uint32_t), st));
  PtrArray none;
  std::memset(&none, 0, sizeof(none));
  MOE_LAUNCH(ctx, "fp8_amax", st,
             launch_amax_batched(none, static_cast<const bf16*>(x), rows * cols, static_cast<int>(batch), rows, cols,
                                 cols, amax, ctx->num_sms, st));
  QuantArgs a = quant_args(ctx);
  a.src = static_cast<const bf16*>(x);
  a.src_batch_stride = rows * cols;
  a.src_ld = cols;
  a.rows = rows;
  a.cols = cols;
  a.mx = 1;
  a.sf_mma = 1;
  a.scale_floor = 0;
  a.e5m2 = e5m2;
  a.do_row = 1;
  a.q_row = q_row;
  a.do_col = col;
  a.q_colT = q_colT;
  a.pt_amax = amax;
  if (!quant_store_maps(a, static_cast<int>(batch))) return MOE_ERR_CUDA;
  MOE_LAUNCH(ctx, "fp8_quantize", st, launch_quant(a, static_cast<int>(batch), ctx->num_sms, st));
  MOE_LAUNCH(ctx, "fp8_scales", st, launch_fp8_scales(amax, static_cast<int>(batch), e5m2, st));
  return MOE_OK;
}

moe_status_t moe_permute(moe_ctx_t ctx, const void* x, const int32_t* topk_idx, const float* topk_prob, int64_t T,
                         int k, int E, int64_t d, const int32_t* split_sizes_in, int32_t* split_sizes,
                         int32_t* poffsets, int32_t* sorted_to_src, int32_t* src_to_sorted, float* prob_perm,
                         void* x_perm, void* stream) {
  if (!ctx || !topk_idx || !split_sizes || !poffsets || !sorted_to_src || !src_to_sorted) return MOE_ERR_INVALID_ARG;
  if (T <= 0) return MOE_ERR_INVALID_ARG;
  if (E < 1 || E > MOE_MAX_EXPERTS || k < 1 || k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
  if (prob_perm && !topk_prob) return MOE_ERR_INVALID_ARG;
  if ((x_perm != nullptr) != (x != nullptr)) return MOE_ERR_INVALID_ARG;
  if (x && (d <= 0 || d % 32 || !aligned16(x) || !aligned16(x_perm))) return x && d % 32 ? MOE_ERR_SHAPE : MOE_ERR_INVALID_ARG;
  const int64_t cap = capacity_rows(T, k, E);
  if (cap >= (int64_t(1) << 31) / 2) return MOE_ERR_UNSUPPORTED;
  DeviceGuard guard(ctx->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MOE_LAUNCH(ctx, "route", st, launch_route(topk_idx, topk_prob, static_cast<int>(T * k), E, static_cast<int>(cap), split_sizes_in,
                        split_sizes, poffsets, sorted_to_src, src_to_sorted, prob_perm, ctx->d_status, st));
  if (x) {
    QuantArgs a = quant_args(ctx);
    a.src = static_cast<const bf16*>(x);
    a.src_ld = d;
    a.sorted_to_src = sorted_to_src;
    a.k = k;
    a.rows = cap;
    a.cols = d;
    a.mx = 0;
    a.do_row = 1;
    a.o_row = static_cast<bf16*>(x_perm);
    if (!quant_store_maps(a, static_cast<int>(1))) return MOE_ERR_CUDA;
    MOE_LAUNCH(ctx, "permute_x", st, launch_quant(a, 1, ctx->num_sms, st));
  }
  return MOE_OK;
}

moe_status_t moe_unpermute(moe_ctx_t ctx, const void* y_perm, const int32_t* src_to_sorted, const float* probs,
                           int64_t T, int k, int64_t d, void* y, void* stream) {
  if (!ctx || !y_perm || !src_to_sorted || !y || T <= 0 || d <= 0) return MOE_ERR_INVALID_ARG;
  if (k < 1 || k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
  if (d % 8) return MOE_ERR_SHAPE;
  if (!aligned16(y_perm) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(ctx->device);
  MOE_LAUNCH(ctx, "unpermute", stream, launch_unpermute(static_cast<const bf16*>(y_perm), src_to_sorted, probs, T, k, d, static_cast<bf16*>(y),
                            ctx->num_sms, static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

size_t moe_saved_size_ex(int64_t T, int k, int E, int64_t d, int64_t f, moe_precision_t prec, int saved_h) {
  if (check_dims(T, d, f, E, k) != MOE_OK) return 0;
  if (saved_h != MOE_SAVED_H_BF16 && saved_h != MOE_SAVED_H_RECOMPUTE &&
      (saved_h != MOE_SAVED_H_MXFP8 || prec != MOE_PREC_MXFP8))
    return 0;
  if (prec == MOE_PREC_FP8 && saved_h != MOE_SAVED_H_BF16) return 0;
  Dims D = make_dims(T, d, f, E, k, prec, saved_h);
  Carve c(nullptr);
  Saved s;
  carve_saved(c, D, s);
  return c.off + 1024;
}

size_t moe_saved_size(int64_t T, int k, int E, int64_t d, int64_t f, moe_precision_t prec) {
  return moe_saved_size_ex(T, k, E, d, f, prec, MOE_SAVED_H_BF16);
}

size_t moe_fwd_workspace_size(int64_t T, int k, int E, int64_t d, int64_t f, moe_precision_t prec, int training) {
  if (check_dims(T, d, f, E, k) != MOE_OK) return 0;
  Dims D = make_dims(T, d, f, E, k, prec);
  Carve c(nullptr);
  FwdWs w;
  carve_fwd(c, D, w);
  if (!training) {  // routing bookkeeping lives in the workspace when nothing is saved
    Saved s;
    carve_saved(c, D, s, false);
  }
  return c.off + 1024;
}

size_t moe_bwd_workspace_size_ex(int64_t T, int k, int E, int64_t d, int64_t f, moe_precision_t prec, int saved_h) {
  if (check_dims(T, d, f, E, k) != MOE_OK) return 0;
  if (saved_h < MOE_SAVED_H_BF16 || saved_h > MOE_SAVED_H_RECOMPUTE) return 0;
  if (prec == MOE_PREC_FP8 && saved_h != MOE_SAVED_H_BF16) return 0;
  Dims D = make_dims(T, d, f, E, k, prec, saved_h);
  Carve c(nullptr);
  BwdWs w;
  carve_bwd(c, D, w);
  return c.off + 1024;
}

size_t moe_bwd_workspace_size(int64_t T, int k, int E, int64_t d, int64_t f, moe_precision_t prec) {
  return moe_bwd_workspace_size_ex(T, k, E, d, f, prec, MOE_SAVED_H_BF16);
}

moe_status_t moe_grouped_mlp_fwd(moe_ctx_t ctx, const void* x, const int32_t* topk_idx, const float* topk_prob,
                                 const int32_t* split_sizes, const void* const* w_gate_up,
                                 const void* const* w_down, int64_t T, int64_t d, int64_t f, int E, int k,
                                 moe_precision_t prec, int training, void* y, void* saved, size_t saved_bytes,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  if (!ctx || !x || !topk_idx || !topk_prob || !w_gate_up || !w_down || !y || !workspace) return MOE_ERR_INVALID_ARG;
  if (prec != MOE_PREC_BF16 && prec != MOE_PREC_MXFP8 && prec != MOE_PREC_FP8) return MOE_ERR_INVALID_ARG;
  const moe_status_t dc = check_dims(T, d, f, E, k);
  if (dc != MOE_OK) return dc;
  if (training && !saved) return MOE_ERR_INVALID_ARG;
  for (int e = 0; e < E; ++e)
    if (!w_gate_up[e] || !w_down[e] || !aligned16(w_gate_up[e]) || !aligned16(w_down[e])) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  const int saved_h = training ? ctx->saved_h : MOE_SAVED_H_BF16;
  if (saved_h == MOE_SAVED_H_MXFP8 && prec != MOE_PREC_MXFP8) return MOE_ERR_UNSUPPORTED;
  if (prec == MOE_PREC_FP8 && saved_h != MOE_SAVED_H_BF16) return MOE_ERR_UNSUPPORTED;
  if (workspace_bytes < moe_fwd_workspace_size(T, k, E, d, f, prec, training)) return MOE_ERR_WORKSPACE;
  if (training && saved_bytes < moe_saved_size_ex(T, k, E, d, f, prec, saved_h)) return MOE_ERR_WORKSPACE;

  DeviceGuard guard(ctx->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Dims D = make_dims(T, d, f, E, k, prec, saved_h);
  Carve cw(reinterpret_cast<void*>(round_up(reinterpret_cast<uintptr_t>(workspace), 1024)));
  FwdWs w;
  carve_fwd(cw, D, w);
  Saved s;
  if (training) {
    Carve cs(reinterpret_cast<void*>(round_up(reinterpret_cast<uintptr_t>(saved), 1024)));
    carve_saved(cs, D, s);
  } else {
    carve_saved(cw, D, s, false);
  }

  // x's gate_up operand: in the workspace, or in the saved buffer when the backward recomputes h
  uint8_t* x_q = s.xr_q ? s.xr_q : w.x_q;
  uint8_t* x_s = s.xr_s ? s.xr_s : w.x_s;
  bf16* x_perm = s.xr ? s.xr : w.x_perm;

  // per-tensor FP8: the maxima of x, W1, W2 and a (per expert), kept for the backward when training
  uint32_t* amax = D.fp8 ? (training ? s.pt_amax : w.pt_amax) : nullptr;
  uint32_t* amax_x = amax;
  uint32_t* amax_w1 = amax ? amax + E : nullptr;
  uint32_t* amax_w2 = amax ? amax + 2 * E : nullptr;
  uint32_t* amax_a = amax ? amax + 3 * E : nullptr;
  if (D.fp8) MOE_CUDA(cudaMemsetAsync(amax, 0, 4 * static_cast<size_t>(E) * sizeof(uint32_t), st));

  // 1. routing: counts, padded offsets, stable permutation, per-row probabilities
  MOE_LAUNCH(ctx, "route", st, launch_route(topk_idx, topk_prob, static_cast<int>(D.Tk), E, static_cast<int>(D.cap), split_sizes, s.split,
                        s.poff, s.s2src, s.src2s, s.pperm, ctx->d_status, st));

  // 2. operands of the gate_up GEMM
  const void* w1_base;
  const void* w2_base;
  int64_t w1_stride, w2_stride;  // bytes between experts
  if (D.fp8) {
    // per-tensor FP8 with current scaling: every expert's W1, W2 and rows of x get one scale from their
    // own maximum, so the maxima come first; one quantisation serves both GEMMs of each tensor
    PtrArray p1, p2;
    for (int e = 0; e < E; ++e) {
      p1.p[e] = w_gate_up[e];
      p2.p[e] = w_down[e];
    }
    MOE_LAUNCH(ctx, "amax_w_gate_up", st, launch_amax_batched(p1, nullptr, 0, E, 2 * f, d, d, amax_w1, ctx->num_sms, st));
    MOE_LAUNCH(ctx, "amax_w_down", st, launch_amax_batched(p2, nullptr, 0, E, d, f, f, amax_w2, ctx->num_sms, st));
    MOE_LAUNCH(ctx, "amax_x", st,
               launch_amax_routed(static_cast<const bf16*>(x), d, d, s.s2src, s.poff, D.cap, k, E, amax_x, ctx->num_sms, st));
    moe_status_t r = quant_experts_fp8(ctx, "quantize_w_gate_up", w_gate_up, E, 2 * f, d, amax_w1, w.w1_q,
                                       training ? s.w1c_q : nullptr, st);
    if (r != MOE_OK) return r;
    r = quant_experts_fp8(ctx, "quantize_w_down", w_down, E, d, f, amax_w2, w.w2_q, training ? s.w2c_q : nullptr, st);
    if (r != MOE_OK) return r;
    w1_base = w.w1_q;
    w1_stride = 2 * f * d;
    w2_base = w.w2_q;
    w2_stride = d * f;
    QuantArgs xa = quant_args(ctx);
    xa.src = static_cast<const bf16*>(x);
    xa.src_ld = d;
    xa.sorted_to_src = s.s2src;
    xa.src_rows = T;
    xa.k = k;
    xa.rows = D.cap;
    xa.cols = d;
    xa.mx = 1;
    xa.sf_mma = 1;
    xa.scale_floor = 0;
    xa.do_row = 1;
    xa.q_row = w.x_q;
    xa.do_col = training;
    xa.q_colT = s.xT_q;
    xa.pt_amax = amax_x;
    xa.pt_poff = s.poff;
    xa.pt_E = E;
    if (!quant_store_maps(xa, 1)) return MOE_ERR_CUDA;
    MOE_LAUNCH(ctx, "permute_quantize_x", st, launch_quant(xa, 1, ctx->num_sms, st));
  } else if (D.mx) {
    // 16-bit masters -> MXFP8 every step: row-wise (K = d / f of the forward GEMMs) and, for the
    // backward, down the columns (K = 2f / d of the dgrad GEMMs), from one read of each weight.
    QuantArgs a = quant_args(ctx);
    for (int e = 0; e < E; ++e) a.src_ptrs.p[e] = w_gate_up[e];
    a.src_ld = d;
    a.rows = 2 * f;
    a.cols = d;
    a.mx = 1;
    a.sf_mma = 1;
    a.do_row = 1;
    a.q_row = w.w1_q;
    a.s_row = w.w1_s;
    a.do_col = training;
    a.q_colT = s.w1c_q;
    a.s_colT = s.w1c_s;
    a.gate_up_half = f;  // row-wise copy in 256-row groups of 128 gate + 128 up rows (one B tile each)
    if (!quant_store_maps(a, static_cast<int>(E))) return MOE_ERR_CUDA;
    MOE_LAUNCH(ctx, "quantize_w_gate_up", st, launch_quant(a, E, ctx->num_sms, st));
    a.gate_up_half = 0;
    for (int e = 0; e < E; ++e) a.src_ptrs.p[e] = w_down[e];
    a.src_ld = f;
    a.rows = d;
    a.cols = f;
    a.q_row = w.w2_q;
    a.s_row = w.w2_s;
    a.q_colT = s.w2c_q;
    a.s_colT = s.w2c_s;
    if (!quant_store_maps(a, static_cast<int>(E))) return MOE_ERR_CUDA;
    MOE_LAUNCH(ctx, "quantize_w_down", st, launch_quant(a, E, ctx->num_sms, st));
    w1_base = w.w1_q;
    w1_stride = 2 * f * d;
    w2_base = w.w2_q;
    w2_stride = d * f;

    // x: gather by expert + row-wise MXFP8 (K = d) and, for wgrad, token-axis MXFP8 transposed
    QuantArgs xa = quant_args(ctx);
    xa.src = static_cast<const bf16*>(x);
    xa.src_ld = d;
    xa.sorted_to_src = s.s2src;
    xa.src_rows = T;
    xa.k = k;
    xa.rows = D.cap;
    xa.cols = d;
    xa.mx = 1;
    xa.sf_mma = 1;
    xa.do_row = 1;
    xa.q_row = x_q;
    xa.s_row = x_s;
    xa.do_col = training;
    xa.q_colT = s.xT_q;
    xa.s_colT = s.xT_s;
    if (!quant_store_maps(xa, static_cast<int>(1))) return MOE_ERR_CUDA;
    MOE_LAUNCH(ctx, "permute_quantize_x", st, launch_quant(xa, 1, ctx->num_sms, st));
  } else {
    w1_stride = uniform_stride(w_gate_up, E, 2 * f * d * 2);
    w2_stride = uniform_stride(w_down, E, d * f * 2);
    w1_base = w_gate_up[0];
    w2_base = w_down[0];
    QuantArgs a = quant_args(ctx);
    a.mx = 0;
    a.do_row = 1;
    if (!w1_stride) {  // experts not evenly spaced: gather into one [E, 2f, d] tensor
      for (int e = 0; e < E; ++e) a.src_ptrs.p[e] = w_gate_up[e];
      a.src_ld = d;
      a.rows = 2 * f;
      a.cols = d;
      a.o_row = w.w1_copy;
      if (!quant_store_maps(a, static_cast<int>(E))) return MOE_ERR_CUDA;
    MOE_LAUNCH(ctx, "gather_w_gate_up", st, launch_quant(a, E, ctx->num_sms, st));
      w1_base = w.w1_copy;
      w1_stride = 2 * f * d * 2;
    }
    if (!w2_stride) {
      for (int e = 0; e < E; ++e) a.src_ptrs.p[e] = w_down[e];
      a.src_ld = f;
      a.rows = d;
      a.cols = f;
      a.o_row = w.w2_copy;
      if (!quant_store_maps(a, static_cast<int>(E))) return MOE_ERR_CUDA;
    MOE_LAUNCH(ctx, "gather_w_down", st, launch_quant(a, E, ctx->num_sms, st));
      w2_base = w.w2_copy;
      w2_stride = d * f * 2;
    }
    QuantArgs xa = quant_args(ctx);
    xa.src = static_cast<const bf16*>(x);
    xa.src_ld = d;
    xa.sorted_to_src = s.s2src;
    xa.src_rows = T;
    xa.k = k;
    xa.rows = D.cap;
    xa.cols = d;
    xa.mx = 0;
    xa.do_row = 1;
    xa.o_row = x_perm;
    xa.do_col = training;
    xa.o_colT = s.xT;
    if (!quant_store_maps(xa, static_cast<int>(1))) return MOE_ERR_CUDA;
    MOE_LAUNCH(ctx, "permute_x", st, launch_quant(xa, 1, ctx->num_sms, st));
  }

  // 3. gate_up GEMM + ScaledSwiGLU + requantisation of a
  {
    GemmArgs g = gemm_args(ctx);
    // MXFP8: the quantised copy is gate/up interleaved, two 128-row boxes per tile; BF16 reads the
    // unpermuted weights as a 128-row gate box plus the matching 128-row up box.
    const bool ok = map_2d(&g.tmap_a, D.q8 ? static_cast<const void*>(x_q) : x_perm, D.q8, d, D.cap,
                           d * (D.q8 ? 1 : 2)) &&
                    map_3d(&g.tmap_b, w1_base, D.q8, d, 2 * f, E, d * (D.q8 ? 1 : 2), w1_stride,
                           !D.mx ? gemm_tile_n(EPI_SWIGLU) / 2
                                 : (ctx->fused_fwd ? gemm_tile_n(EPI_SWIGLU) : gemm_b_box_rows(true, EPI_SWIGLU)));
    if (!ok) return MOE_ERR_CUDA;
    g.kgrouped = 0;
    g.E = E;
    g.K = static_cast<int>(d);
    g.n_tiles = static_cast<int>(f / 128);
    g.gate_up_half = D.mx ? 0 : static_cast<int>(f);
    g.fp8 = D.fp8;
    g.pt_amax_a = amax_x;
    g.pt_amax_b = amax_w1;
    g.poffsets = s.poff;
    g.sfa = x_s;
    g.sfa_kb4 = d / 128;
    g.sfb = w.w1_s;
    g.sfb_kb4 = d / 128;
    g.sfb_expert_rows = 2 * f;
    if (D.mx && !sf_maps(g, D.cap, E * 2 * f, gemm_tile_n(EPI_SWIGLU))) return MOE_ERR_CUDA;
    EpiArgs& ep = g.epi;
    ep.f = f;
    ep.cap = D.cap;
    ep.p_perm = s.pperm;
    ep.h = training ? s.h : nullptr;  // (null when h is saved as MXFP8)
    ep.h_q = training ? s.h_q : nullptr;
    ep.h_s = training ? s.h_s : nullptr;
    ep.dump = ctx->dbg_a;
    if (D.mx) {
      ep.q_row = w.a_q;
      ep.s_row = w.a_s;
      ep.q_colT = training ? s.aT_q : nullptr;
      ep.s_colT = training ? s.aT_s : nullptr;
    } else {
      // BF16: a in bf16 both ways; per-tensor FP8: a in bf16 rows and its per-expert maximum, then
      // quantised once its maximum is complete
      ep.o_row = w.a;
      ep.o_colT = (training && !D.fp8) ? s.aT : nullptr;
      ep.amax_out = D.fp8 ? amax_a : nullptr;
    }
    // 4. down GEMM: its own launch, or (fused forward) the tiles that follow in the same launch
    GemmArgs g2 = gemm_args(ctx);
    const bool ok2 = map_2d(&g2.tmap_a, D.q8 ? static_cast<const void*>(w.a_q) : w.a, D.q8, f, D.cap,
                            f * (D.q8 ? 1 : 2)) &&
                     map_3d(&g2.tmap_b, w2_base, D.q8, f, d, E, f * (D.q8 ? 1 : 2), w2_stride,
                            ctx->fused_fwd ? gemm_tile_n(EPI_STORE) : gemm_b_box_rows(D.mx, EPI_STORE));
    if (!ok2) return MOE_ERR_CUDA;
    g2.kgrouped = 0;
    g2.E = E;
    g2.K = static_cast<int>(f);
    g2.n_tiles = static_cast<int>(d / 256);
    g2.fp8 = D.fp8;
    g2.pt_amax_a = amax_a;
    g2.pt_amax_b = amax_w2;
    g2.poffsets = s.poff;
    g2.sfa = w.a_s;
    g2.sfa_kb4 = f / 128;
    g2.sfb = w.w2_s;
    g2.sfb_kb4 = f / 128;
    g2.sfb_expert_rows = d;
    if (D.mx && !sf_maps(g2, D.cap, E * d, gemm_tile_n(EPI_STORE))) return MOE_ERR_CUDA;
    g2.epi.out = w.y_perm;
    g2.epi.ldo = d;
    if (ctx->fused_fwd && !D.fp8) {
      // one persistent launch: gate_up tiles, then down tiles that wait for their 128-row blocks of a
      // (per-tensor FP8 cannot: a is quantised only once all of its expert's tiles are done)
      g.tmap_a2 = g2.tmap_a;
      g.tmap_b2 = g2.tmap_b;
      g.tmap_sfa2 = g2.tmap_sfa;
      g.tmap_sfb2 = g2.tmap_sfb;
      g.K2 = g2.K;
      g.n_tiles2 = g2.n_tiles;
      g.sfb_expert_rows2 = g2.sfb_expert_rows;
      g.epi.out = g2.epi.out;
      g.epi.ldo = g2.epi.ldo;
      g.mblock_done = w.mblk;
      MOE_CUDA(cudaMemsetAsync(w.mblk, 0, static_cast<size_t>(D.cap / 128) * sizeof(int), st));
      MOE_LAUNCH(ctx, "gemm_fused_forward", st, launch_grouped_gemm(g, D.mx, EPI_FUSED_FWD, ctx->num_sms, st));
    } else {
      MOE_LAUNCH(ctx, "gemm_gate_up_swiglu", st, launch_grouped_gemm(g, D.mx, EPI_SWIGLU, ctx->num_sms, st));
      if (D.fp8) {
        const moe_status_t r = quant_segments_fp8(ctx, "quantize_a", w.a, D.cap, f, s.poff, E, amax_a, 0, w.a_q,
                                                  training ? s.aT_q : nullptr, st);
        if (r != MOE_OK) return r;
      }
      MOE_LAUNCH(ctx, "gemm_down", st, launch_grouped_gemm(g2, D.mx, EPI_STORE, ctx->num_sms, st));
    }
  }
  // 5. combine (probabilities were applied in ScaledSwiGLU)
  MOE_LAUNCH(ctx, "unpermute_y", st, launch_unpermute(w.y_perm, s.src2s, nullptr, T, k, d, static_cast<bf16*>(y), ctx->num_sms, st));
  return MOE_OK;
}

moe_status_t moe_grouped_mlp_bwd(moe_ctx_t ctx, const void* dy, const void* saved, size_t saved_bytes,
                                 const void* const* w_gate_up, const void* const* w_down, int64_t T, int64_t d,
                                 int64_t f, int E, int k, moe_precision_t prec, void* dx, void* const* dw_gate_up,
                                 void* const* dw_down, float* d_topk_prob, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  if (!ctx || !dy || !saved || !w_gate_up || !w_down || !dx || !dw_gate_up || !dw_down || !d_topk_prob || !workspace)
    return MOE_ERR_INVALID_ARG;
  if (prec != MOE_PREC_BF16 && prec != MOE_PREC_MXFP8 && prec != MOE_PREC_FP8) return MOE_ERR_INVALID_ARG;
  const moe_status_t dc = check_dims(T, d, f, E, k);
  if (dc != MOE_OK) return dc;
  for (int e = 0; e < E; ++e)
    if (!w_gate_up[e] || !w_down[e] || !dw_gate_up[e] || !dw_down[e] || !aligned16(dw_gate_up[e]) ||
        !aligned16(dw_down[e]) || !aligned16(w_gate_up[e]) || !aligned16(w_down[e]))
      return MOE_ERR_INVALID_ARG;
  if (!aligned16(dy) || !aligned16(dx)) return MOE_ERR_INVALID_ARG;
  const int saved_h = ctx->saved_h;
  if (saved_h == MOE_SAVED_H_MXFP8 && prec != MOE_PREC_MXFP8) return MOE_ERR_UNSUPPORTED;
  if (prec == MOE_PREC_FP8 && saved_h != MOE_SAVED_H_BF16) return MOE_ERR_UNSUPPORTED;
  if (saved_bytes < moe_saved_size_ex(T, k, E, d, f, prec, saved_h)) return MOE_ERR_WORKSPACE;
  if (workspace_bytes < moe_bwd_workspace_size_ex(T, k, E, d, f, prec, saved_h)) return MOE_ERR_WORKSPACE;

  DeviceGuard guard(ctx->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Dims D = make_dims(T, d, f, E, k, prec, saved_h);
  Saved s;
  Carve cs(reinterpret_cast<void*>(round_up(reinterpret_cast<uintptr_t>(saved), 1024)));
  carve_saved(cs, D, s);
  BwdWs w;
  Carve cw(reinterpret_cast<void*>(round_up(reinterpret_cast<uintptr_t>(workspace), 1024)));
  carve_bwd(cw, D, w);
  // per-tensor FP8: the forward's maxima of x, W1, W2, a, and this pass's of dy and dh
  const uint32_t* amax_x = s.pt_amax;
  const uint32_t* amax_w1 = s.pt_amax ? s.pt_amax + E : nullptr;
  const uint32_t* amax_w2 = s.pt_amax ? s.pt_amax + 2 * E : nullptr;
  const uint32_t* amax_a = s.pt_amax ? s.pt_amax + 3 * E : nullptr;
  uint32_t* amax_dy = w.pt_amax;
  uint32_t* amax_dh = w.pt_amax ? w.pt_amax + E : nullptr;
  if (D.fp8) {
    MOE_CUDA(cudaMemsetAsync(w.pt_amax, 0, 2 * static_cast<size_t>(E) * sizeof(uint32_t), st));
    MOE_LAUNCH(ctx, "amax_dy", st,
               launch_amax_routed(static_cast<const bf16*>(dy), d, d, s.s2src, s.poff, D.cap, k, E, amax_dy, ctx->num_sms, st));
  }

  // 0. recompute mode: h again, from x's saved gate_up operand and W1 (quantised again for MXFP8),
  //    through the gate_up GEMM with an epilogue that only writes h
  bf16* h_src = s.h;
  if (D.saved_h == MOE_SAVED_H_RECOMPUTE) {
    const void* w1_base;
    int64_t w1_stride;
    if (D.mx) {
      QuantArgs a = quant_args(ctx);
      for (int e = 0; e < E; ++e) a.src_ptrs.p[e] = w_gate_up[e];
      a.src_ld = d;
      a.rows = 2 * f;
      a.cols = d;
      a.mx = 1;
      a.sf_mma = 1;
      a.do_row = 1;
      a.q_row = w.w1r_q;
      a.s_row = w.w1r_s;
      a.gate_up_half = f;
      if (!quant_store_maps(a, static_cast<int>(E))) return MOE_ERR_CUDA;
      MOE_LAUNCH(ctx, "requantize_w_gate_up", st, launch_quant(a, E, ctx->num_sms, st));
      w1_base = w.w1r_q;
      w1_stride = 2 * f * d;
    } else {
      w1_stride = uniform_stride(w_gate_up, E, 2 * f * d * 2);
      w1_base = w_gate_up[0];
      if (!w1_stride) {
        QuantArgs a = quant_args(ctx);
        for (int e = 0; e < E; ++e) a.src_ptrs.p[e] = w_gate_up[e];
        a.src_ld = d;
        a.rows = 2 * f;
        a.cols = d;
        a.mx = 0;
        a.do_row = 1;
        a.o_row = w.w1r_copy;
        if (!quant_store_maps(a, static_cast<int>(E))) return MOE_ERR_CUDA;
        MOE_LAUNCH(ctx, "gather_w_gate_up", st, launch_quant(a, E, ctx->num_sms, st));
        w1_base = w.w1r_copy;
        w1_stride = 2 * f * d * 2;
      }
    }
    GemmArgs g = gemm_args(ctx);
    const bool ok = map_2d(&g.tmap_a, D.mx ? static_cast<const void*>(s.xr_q) : s.xr, D.mx, d, D.cap,
                           d * (D.mx ? 1 : 2)) &&
                    map_3d(&g.tmap_b, w1_base, D.mx, d, 2 * f, E, d * (D.mx ? 1 : 2), w1_stride,
                           D.mx ? gemm_b_box_rows(true, EPI_SWIGLU) : gemm_tile_n(EPI_SWIGLU) / 2);
    if (!ok) return MOE_ERR_CUDA;
    g.kgrouped = 0;
    g.E = E;
    g.K = static_cast<int>(d);
    g.n_tiles = static_cast<int>(f / 128);
    g.gate_up_half = D.mx ? 0 : static_cast<int>(f);
    g.poffsets = s.poff;
    g.sfa = s.xr_s;
    g.sfa_kb4 = d / 128;
    g.sfb = w.w1r_s;
    g.sfb_kb4 = d / 128;
    g.sfb_expert_rows = 2 * f;
    if (D.mx && !sf_maps(g, D.cap, E * 2 * f, gemm_tile_n(EPI_SWIGLU))) return MOE_ERR_CUDA;
    g.epi.f = f;
    g.epi.cap = D.cap;
    g.epi.p_perm = s.pperm;
    g.epi.h = w.hr;  // no a outputs: the epilogue stops after saving h
    MOE_LAUNCH(ctx, "gemm_recompute_h", st, launch_grouped_gemm(g, D.mx, EPI_SWIGLU, ctx->num_sms, st));
    h_src = w.hr;
  }

  // 1. dy gathered by expert: row-wise (K = d, dgrad of down) and token-axis transposed (wgrad of down)
  {
    QuantArgs a = quant_args(ctx);
    a.src = static_cast<const bf16*>(dy);
    a.src_ld = d;
    a.sorted_to_src = s.s2src;
    a.src_rows = T;
    a.k = k;
    a.rows = D.cap;
    a.cols = d;
    a.do_row = 1;
    a.do_col = 1;
    if (D.fp8) {  // per-tensor FP8 with each expert's maximum
      a.mx = 1;
      a.sf_mma = 1;
      a.scale_floor = 0;
      a.e5m2 = ctx->grad_e5m2;
      a.q_row = w.dy_q;
      a.q_colT = w.dyT_q;
      a.pt_amax = amax_dy;
      a.pt_poff = s.poff;
      a.pt_E = E;
    } else if (D.mx) {
      a.mx = 1;
      a.sf_mma = 1;
      a.e5m2 = ctx->grad_e5m2;  // dy is a gradient operand
      a.q_row = w.dy_q;
      a.s_row = w.dy_s;
      a.q_colT = w.dyT_q;
      a.s_colT = w.dyT_s;
    } else {
      a.o_row = w.dy_perm;
      a.o_colT = w.dyT;
    }
    if (!quant_store_maps(a, static_cast<int>(1))) return MOE_ERR_CUDA;
    MOE_LAUNCH(ctx, "gather_quantize_dy", st, launch_quant(a, 1, ctx->num_sms, st));
  }
  const void* w1c;  // B of dgrad of gate_up: [E, d, 2f]
  const void* w2c;  // B of dgrad of down:    [E, f, d]
  if (D.q8) {
    w1c = s.w1c_q;
    w2c = s.w2c_q;
  } else {
    QuantArgs a = quant_args(ctx);
    a.mx = 0;
    a.do_col = 1;
    for (int e = 0; e < E; ++e) a.src_ptrs.p[e] = w_gate_up[e];
    a.src_ld = d;
    a.rows = 2 * f;
    a.cols = d;
    a.o_colT = w.w1T;
    if (!quant_store_maps(a, static_cast<int>(E))) return MOE_ERR_CUDA;
    MOE_LAUNCH(ctx, "transpose_w_gate_up", st, launch_quant(a, E, ctx->num_sms, st));
    for (int e = 0; e < E; ++e) a.src_ptrs.p[e] = w_down[e];
    a.src_ld = f;
    a.rows = d;
    a.cols = f;
    a.o_colT = w.w2T;
    if (!quant_store_maps(a, static_cast<int>(E))) return MOE_ERR_CUDA;
    MOE_LAUNCH(ctx, "transpose_w_down", st, launch_quant(a, E, ctx->num_sms, st));
    w1c = w.w1T;
    w2c = w.w2T;
  }
  const int es = D.q8 ? 1 : 2;
  // 2. dgrad of down + ScaledSwiGLU backward: dh = [dg, du] requantised both ways, dp partials
  {
    GemmArgs g = gemm_args(ctx);
    const bool ok = map_2d(&g.tmap_a, D.q8 ? static_cast<const void*>(w.dy_q) : w.dy_perm, D.q8, d, D.cap, d * es) &&
                    map_3d(&g.tmap_b, w2c, D.q8, d, f, E, d * es, f * d * es, gemm_tile_n(EPI_DSWIGLU)) &&
                    (s.h_q || map_2d(&g.tmap_h, h_src, false, 2 * f, D.cap, 2 * f * 2));  // bf16 boxes, 128 x 64
    if (!ok) return MOE_ERR_CUDA;
    g.kgrouped = 0;
    g.E = E;
    g.K = static_cast<int>(d);
    g.n_tiles = static_cast<int>(f / gemm_tile_n(EPI_DSWIGLU));
    g.fp8 = D.fp8;
    g.pt_amax_a = amax_dy;
    g.pt_amax_b = amax_w2;
    g.poffsets = s.poff;
    g.sfa = w.dy_s;
    g.sfa_kb4 = d / 128;
    g.sfb = s.w2c_s;
    g.sfb_kb4 = d / 128;
    g.sfb_expert_rows = f;
    if (D.mx && !sf_maps(g, D.cap, E * f, gemm_tile_n(EPI_DSWIGLU))) return MOE_ERR_CUDA;
    EpiArgs& ep = g.epi;
    ep.f = f;
    ep.cap = D.cap;
    ep.p_perm = s.pperm;
    ep.h = h_src;    // bf16 h (saved or recomputed) staged by TMA, or
    ep.h_q = s.h_q;  // MXFP8 h read by the epilogue (the kernel instance without h staging)
    ep.h_s = s.h_s;
    ep.dump = ctx->dbg_dh;
    ep.dp_part = w.dp_part;
    ep.grad_e5m2 = ctx->grad_e5m2;  // dh is the gradient operand of both gate_up backward GEMMs
    g.a_e5m2 = ctx->grad_e5m2;      // A = dy
    if (D.mx) {
      ep.q_row = w.dh_q;
      ep.s_row = w.dh_s;
      ep.q_colT = w.dhT_q;
      ep.s_colT = w.dhT_s;
    } else {
      // BF16: dh in bf16 both ways; per-tensor FP8: dh in bf16 rows and its per-expert maximum, then
      // quantised once its maximum is complete
      ep.o_row = w.dh;
      ep.o_colT = D.fp8 ? nullptr : w.dhT;
      ep.amax_out = amax_dh;
    }
    MOE_LAUNCH(ctx, "gemm_dgrad_down_dswiglu", st, launch_grouped_gemm(g, D.mx, EPI_DSWIGLU, ctx->num_sms, st));
    if (D.fp8) {
      const moe_status_t r = quant_segments_fp8(ctx, "quantize_dh", w.dh, D.cap, 2 * f, s.poff, E, amax_dh,
                                                ctx->grad_e5m2, w.dh_q, w.dhT_q, st);
      if (r != MOE_OK) return r;
    }
  }
  // 3. wgrad of down: dW2_e [d, f] = dy_e^T a_e (K = the expert's tokens)
  {
    GemmArgs g = gemm_args(ctx);
    const bool ok =
        map_2d(&g.tmap_a, D.q8 ? static_cast<const void*>(w.dyT_q) : w.dyT, D.q8, D.cap, d, D.cap * es) &&
        map_2d(&g.tmap_b, D.q8 ? static_cast<const void*>(s.aT_q) : s.aT, D.q8, D.cap, f, D.cap * es,
               gemm_b_box_rows(D.mx, EPI_STORE));
    if (!ok) return MOE_ERR_CUDA;
    g.kgrouped = 1;
    g.E = E;
    g.m_tiles = static_cast<int>(d / 128);
    g.n_tiles = static_cast<int>(f / 256);
    g.fp8 = D.fp8;
    g.pt_amax_a = amax_dy;
    g.pt_amax_b = amax_a;
    g.poffsets = s.poff;
    g.sfa = w.dyT_s;
    g.sfa_kb4 = D.cap / 128;
    g.sfb = s.aT_s;
    g.sfb_kb4 = D.cap / 128;
    if (D.mx && !sf_maps(g, d, f, gemm_tile_n(EPI_STORE))) return MOE_ERR_CUDA;
    g.epi.ldo = f;
    for (int e = 0; e < E; ++e) g.epi.out_ptrs.p[e] = dw_down[e];
    g.a_e5m2 = ctx->grad_e5m2;  // A is a gradient operand (dy or dh)
    MOE_LAUNCH(ctx, "gemm_wgrad_down", st, launch_grouped_gemm(g, D.mx, EPI_STORE, ctx->num_sms, st));
  }
  // 4. dgrad of gate_up: dx_perm = dh W1 (K = 2f)
  {
    GemmArgs g = gemm_args(ctx);
    const bool ok =
        map_2d(&g.tmap_a, D.q8 ? static_cast<const void*>(w.dh_q) : w.dh, D.q8, 2 * f, D.cap, 2 * f * es) &&
        map_3d(&g.tmap_b, w1c, D.q8, 2 * f, d, E, 2 * f * es, 2 * f * d * es, gemm_b_box_rows(D.mx, EPI_STORE));
    if (!ok) return MOE_ERR_CUDA;
    g.kgrouped = 0;
    g.E = E;
    g.K = static_cast<int>(2 * f);
    g.n_tiles = static_cast<int>(d / 256);
    g.fp8 = D.fp8;
    g.pt_amax_a = amax_dh;
    g.pt_amax_b = amax_w1;
    g.poffsets = s.poff;
    g.sfa = w.dh_s;
    g.sfa_kb4 = 2 * f / 128;
    g.sfb = s.w1c_s;
    g.sfb_kb4 = 2 * f / 128;
    g.sfb_expert_rows = d;
    if (D.mx && !sf_maps(g, D.cap, E * d, gemm_tile_n(EPI_STORE))) return MOE_ERR_CUDA;
    g.epi.out = w.dx_perm;
    g.epi.ldo = d;
    g.a_e5m2 = ctx->grad_e5m2;  // A is a gradient operand (dy or dh)
    MOE_LAUNCH(ctx, "gemm_dgrad_gate_up", st, launch_grouped_gemm(g, D.mx, EPI_STORE, ctx->num_sms, st));
  }
  // 5. wgrad of gate_up: dW1_e [2f, d] = dh_e^T x_e
  {
    GemmArgs g = gemm_args(ctx);
    const bool ok =
        map_2d(&g.tmap_a, D.q8 ? static_cast<const void*>(w.dhT_q) : w.dhT, D.q8, D.cap, 2 * f, D.cap * es) &&
        map_2d(&g.tmap_b, D.q8 ? static_cast<const void*>(s.xT_q) : s.xT, D.q8, D.cap, d, D.cap * es,
               gemm_b_box_rows(D.mx, EPI_STORE));
    if (!ok) return MOE_ERR_CUDA;
    g.kgrouped = 1;
    g.E = E;
    g.m_tiles = static_cast<int>(2 * f / 128);
    g.n_tiles = static_cast<int>(d / 256);
    g.fp8 = D.fp8;
    g.pt_amax_a = amax_dh;
    g.pt_amax_b = amax_x;
    g.poffsets = s.poff;
    g.sfa = w.dhT_s;
    g.sfa_kb4 = D.cap / 128;
    g.sfb = s.xT_s;
    g.sfb_kb4 = D.cap / 128;
    if (D.mx && !sf_maps(g, 2 * f, d, gemm_tile_n(EPI_STORE))) return MOE_ERR_CUDA;
    g.epi.ldo = d;
    for (int e = 0; e < E; ++e) g.epi.out_ptrs.p[e] = dw_gate_up[e];
    g.a_e5m2 = ctx->grad_e5m2;  // A is a gradient operand (dy or dh)
    MOE_LAUNCH(ctx, "gemm_wgrad_gate_up", st, launch_grouped_gemm(g, D.mx, EPI_STORE, ctx->num_sms, st));
  }
  // 6. combine dx, reduce the probability gradient
  MOE_LAUNCH(ctx, "unpermute_dx", st, launch_unpermute(w.dx_perm, s.src2s, nullptr, T, k, d, static_cast<bf16*>(dx), ctx->num_sms, st));
  MOE_LAUNCH(ctx, "dprob_reduce", st,
             launch_dprob_reduce(w.dp_part, static_cast<int>(gemm_dswiglu_parts() * (f / gemm_tile_n(EPI_DSWIGLU))),
                                 D.cap, s.s2src, D.cap, s.src2s, D.Tk, d_topk_prob, st));
  return MOE_OK;
}

moe_status_t moe_tensor_peak_loop(moe_ctx_t ctx, moe_precision_t prec, int64_t iters, int scale_refresh,
                                  void* stream) {
  if (!ctx || iters <= 0 || iters > 1000000 ||
      (prec != MOE_PREC_BF16 && prec != MOE_PREC_MXFP8 && prec != MOE_PREC_FP8))
    return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(ctx->device);
  MOE_LAUNCH(ctx, "tensor_peak_loop", stream,
             launch_tensor_peak(static_cast<int>(prec), iters, scale_refresh ? 1 : 0, ctx->num_sms, ctx->d_status,
                                static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

double moe_tensor_peak_flops(moe_ctx_t ctx, moe_precision_t prec, int64_t iters) {
  if (!ctx || iters <= 0) return 0.0;
  if (prec != MOE_PREC_BF16 && prec != MOE_PREC_MXFP8 && prec != MOE_PREC_FP8) return 0.0;
  return tensor_peak_flops(static_cast<int>(prec), ctx->num_sms, iters);
}

void* moe_buffer_address_ex(int64_t T, int k, int E, int64_t d, int64_t f, moe_precision_t prec, int training,
                            int saved_h, int which, void* base, const char* name) {
  if (!base || !name || check_dims(T, d, f, E, k) != MOE_OK) return nullptr;
  const Dims D = make_dims(T, d, f, E, k, prec, saved_h);
  Carve c(reinterpret_cast<void*>(round_up(reinterpret_cast<uintptr_t>(base), 1024)));
  struct Named {
    const char* n;
    void* p;
  };
  if (which == 0 || (which == 1 && !training)) {
    Saved s;
    if (which == 1) {
      FwdWs w;
      carve_fwd(c, D, w);
    }
    carve_saved(c, D, s, which == 0);
    const Named tab[] = {{"split_sizes", s.split}, {"poffsets", s.poff}, {"sorted_to_src", s.s2src},
                         {"src_to_sorted", s.src2s}, {"prob_perm", s.pperm}, {"w1c_q", s.w1c_q},
                         {"w1c_s", s.w1c_s}, {"w2c_q", s.w2c_q}, {"w2c_s", s.w2c_s}, {"xT_q", s.xT_q},
                         {"xT_s", s.xT_s}, {"aT_q", s.aT_q}, {"aT_s", s.aT_s}, {"xT", s.xT}, {"aT", s.aT},
                         {"h", s.h},       {"h_q", s.h_q},     {"h_s", s.h_s},   {"xr_q", s.xr_q},
                         {"xr_s", s.xr_s}, {"xr", s.xr},   {"pt_amax", s.pt_amax}};
    for (const Named& e : tab)
      if (!std::strcmp(e.n, name) && e.p) return e.p;
    if (which == 0) return nullptr;
    c = Carve(reinterpret_cast<void*>(round_up(reinterpret_cast<uintptr_t>(base), 1024)));
  }
  if (which == 1) {
    FwdWs w;
    carve_fwd(c, D, w);
    const Named tab[] = {{"w1_q", w.w1_q}, {"w1_s", w.w1_s}, {"w2_q", w.w2_q}, {"w2_s", w.w2_s},
                         {"x_q", w.x_q},   {"x_s", w.x_s},   {"a_q", w.a_q},   {"a_s", w.a_s},
                         {"x_perm", w.x_perm}, {"a", w.a}, {"y_perm", w.y_perm}, {"pt_amax", w.pt_amax}};
    for (const Named& e : tab)
      if (!std::strcmp(e.n, name) && e.p) return e.p;
    return nullptr;
  }
  if (which == 2) {
    BwdWs w;
    carve_bwd(c, D, w);
    const Named tab[] = {{"dy_q", w.dy_q},   {"dy_s", w.dy_s},     {"dyT_q", w.dyT_q}, {"dyT_s", w.dyT_s},
                         {"dh_q", w.dh_q},   {"dh_s", w.dh_s},     {"dhT_q", w.dhT_q}, {"dhT_s", w.dhT_s},
                         {"dy_perm", w.dy_perm}, {"dyT", w.dyT},   {"dh", w.dh},       {"dhT", w.dhT},
                         {"w1T", w.w1T},     {"w2T", w.w2T},       {"dx_perm", w.dx_perm},
                         {"dp_part", w.dp_part}, {"hr", w.hr},     {"w1r_q", w.w1r_q}, {"w1r_s", w.w1r_s},
                         {"pt_amax", w.pt_amax}};
    for (const Named& e : tab)
      if (!std::strcmp(e.n, name) && e.p) return e.p;
  }
  return nullptr;
}

void* moe_buffer_address(int64_t T, int k, int E, int64_t d, int64_t f, moe_precision_t prec, int training,
                         int which, void* base, const char* name) {
  return moe_buffer_address_ex(T, k, E, d, f, prec, training, MOE_SAVED_H_BF16, which, base, name);
}

// ---- forward without allocation: file-scope scratch, looked up once per device
static __device__ __align__(256) uint8_t g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];
static __device__ __align__(256) int g_noalloc_status[64];

namespace {
constexpr int kNoAllocMaxDevices = 64;
struct NoAllocDevice {
  bool ready;
  int num_sms;
  void* scratch;  // device address of g_noalloc_scratch on this device
  int* status;    // device address of g_noalloc_status on this device
};
NoAllocDevice g_noalloc_dev[kNoAllocMaxDevices];
std::mutex g_noalloc_mu;

moe_status_t noalloc_setup(int dev, NoAllocDevice& out) {
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoAllocDevice& nd = g_noalloc_dev[dev];
  if (!nd.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (major != 10 || minor != 0) return MOE_ERR_UNSUPPORTED;
    if (!encoder()) return MOE_ERR_CUDA;
    void* scratch = nullptr;
    void* status = nullptr;
    // host code must not use the arrays' names as device addresses: ask the runtime, with ``dev`` current
    if (cudaGetSymbolAddress(&scratch, g_noalloc_scratch) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaGetSymbolAddress(&status, g_noalloc_status) != cudaSuccess) return MOE_ERR_CUDA;
    nd.num_sms = sms;
    nd.scratch = scratch;
    nd.status = static_cast<int*>(status);
    nd.ready = true;
  }
  out = nd;
  return MOE_OK;
}
}  // namespace

moe_status_t moe_grouped_mlp_fwd_noalloc(const void* x, const int32_t* topk_idx, const float* topk_prob,
                                         const int32_t* split_sizes, const void* const* w_gate_up,
                                         const void* const* w_down, int64_t T, int64_t d, int64_t f, int E, int k,
                                         moe_precision_t prec, void* y, int* device_status, void* stream) {
  const moe_status_t dc = check_dims(T, d, f, E, k);
  if (dc != MOE_OK) return dc;
  if (moe_fwd_workspace_size(T, k, E, d, f, prec, 0) > MOE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_WORKSPACE;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) return MOE_ERR_CUDA;
  NoAllocDevice nd;
  const moe_status_t st = noalloc_setup(dev, nd);
  if (st != MOE_OK) return st;
  // a context on the stack: no debug hooks, status into the caller's word (or the static one)
  moe_ctx_s c;
  c.device = dev;
  c.num_sms = nd.num_sms;
  c.d_status = device_status ? device_status : nd.status;
  c.dbg_a = c.dbg_dh = nullptr;
  c.hook = nullptr;
  c.hook_user = nullptr;
  c.scale_floor = 0;
  c.grad_e5m2 = 0;
  c.saved_h = MOE_SAVED_H_BF16;
  c.fused_fwd = 0;
  c.stall = 0;
  c.stall_limit = 0;
  // the scratch base is 256-aligned; the workspace carving aligns to 1 KiB inside the size bound
  return moe_grouped_mlp_fwd(&c, x, topk_idx, topk_prob, split_sizes, w_gate_up, w_down, T, d, f, E, k, prec, 0, y,
                             nullptr, 0, nd.scratch, MOE_NOALLOC_SCRATCH_BYTES, stream);
}

}  // extern "C"
