// Host side of the libminf C ABI: argument validation, workspace carving,
// TMA descriptor set-up and kernel dispatch.  See include/minf.h for the
// contract of every entry point.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>

#include "minf_device.cuh"
#include "minf_internal.h"

using namespace minf;

namespace {

constexpr size_t kStatusBytes = 256;

size_t align_up(size_t x, size_t a = 256) { return (x + a - 1) / a * a; }

bool shape_ok(const minf_shape* s) {
  if (!s) return false;
  if (s->B < 1 || s->Hq < 1 || s->Hkv < 1 || s->N < 128) return false;
  if (s->Hq % s->Hkv != 0) return false;
  if (s->N % 128 != 0) return false;
  if ((long long)s->B * s->Hq * s->N >= (1ll << 31)) return false;
  return true;
}

minf_status check_shape(const minf_shape* s) {
  if (!shape_ok(s)) return MINF_ERR_INVALID_ARG;
  if (s->d != 64 && s->d != 128) return MINF_ERR_UNSUPPORTED;
  return MINF_OK;
}

float eff_scale(const minf_shape* s) { return s->scale > 0.f ? s->scale : 1.0f / std::sqrt((float)s->d); }

// Carves consecutive 256-byte-aligned buffers out of a workspace.
struct Carver {
  char* base;
  size_t off;
  template <class T>
  T* take(size_t count) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off = align_up(off + count * sizeof(T));
    return p;
  }
};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// 2-D bf16 view [rows, d] with a box of 64 columns x box_rows rows, 128B swizzle.
bool make_map(CUtensorMap* m, const void* ptr, long long rows, int d, int box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D bf16 view of a row-major [rows, d] matrix: x = column within a 64-column
// region, y = row, z = region (global stride 128 B).  A box of 64 x box_rows x
// d/64 lands region z at z * box_rows * 128 B in shared memory, each region
// 128B-swizzled: the same layout as d/64 separate 2-D copies.
bool make_map3(CUtensorMap* m, const void* ptr, long long rows, int d, int box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)rows, (cuuint64_t)(d / 64)};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, 128};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, (cuuint32_t)(d / 64)};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

minf_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MINF_OK : MINF_ERR_CUDA; }

// ----------------------------------------------------------- workspace plans
struct VsEstWs {
  DevStatus* status;
  float *part_ml, *row_ml, *v_score, *s_score, *dpart;
  uint32_t* topk;
};
size_t plan_vs_est(const minf_shape* s, int nh, char* ws, VsEstWs* out) {
  Carver c{ws, 0};
  const size_t bh = (size_t)s->B * nh;
  const size_t ntiles = (s->N + 127) / 128;
  VsEstWs w;
  w.status = c.take<DevStatus>(kStatusBytes / sizeof(DevStatus));
  w.part_ml = c.take<float>(bh * ntiles * 64 * 2);
  w.row_ml = c.take<float>(bh * 64 * 2);
  w.v_score = c.take<float>(bh * s->N);
  w.s_score = c.take<float>(bh * s->N);
  w.dpart = c.take<float>(bh * ntiles * 192);
  w.topk = c.take<uint32_t>(topk_scratch_words((int)bh));
  if (out) *out = w;
  return c.off;
}

struct BsEstWs {
  DevStatus* status;
  float *qbar, *kbar, *scores;
  __nv_bfloat16 *qs, *ks;
};
// The pooled means and the pooled score matrix; with a budget k_b that the
// tensor-core path takes (k_b = 0 never), also the means' bf16 parts.
size_t plan_bs_est(const minf_shape* s, int nh, int k_b, char* ws, BsEstWs* out) {
  Carver c{ws, 0};
  const size_t bh = (size_t)s->B * nh;
  const size_t nb = s->N / 64;
  BsEstWs w;
  w.status = c.take<DevStatus>(kStatusBytes / sizeof(DevStatus));
  w.qbar = c.take<float>(bh * nb * s->d);
  w.kbar = c.take<float>(bh * nb * s->d);
  w.scores = c.take<float>(bh * nb * nb);
  w.qs = w.ks = nullptr;
  if (bs_select_supported(s->N, s->d, k_b)) {
    w.qs = c.take<__nv_bfloat16>(3 * bh * nb * s->d);
    w.ks = c.take<__nv_bfloat16>(3 * bh * nb * s->d);
  }
  if (out) *out = w;
  return c.off;
}

// 3-D bf16 view of the split key means [3 * bh, nb, d]: x = d, y = key block,
// z = part * bh + slot, with 64 x 128 x 1 boxes (128-byte swizzled); rows
// past nb read as zero.
// The Grid workspace: the Block-Sparse estimation's workspace of the permuted
// shape first (its status block is the call's), then the permuted Q, K, V
// and O, the permuted LSE and the selection (when the caller passes none).
struct GridWs {
  char* est;
  size_t est_bytes;
  __nv_bfloat16 *qp, *kp, *vp, *op;
  float* lsep;
  int32_t *bi, *bc;
};
minf_shape grid_shape(const minf_shape* s, int P) {
  minf_shape g = *s;
  g.B = s->B * P;
  g.N = s->N / P;
  return g;
}
size_t plan_grid(const minf_shape* s, int nh, int k_b, int P, char* ws, GridWs* out) {
  const minf_shape g = grid_shape(s, P);
  GridWs w;
  w.est = ws;
  w.est_bytes = plan_bs_est(&g, nh, k_b, nullptr, nullptr);
  Carver c{ws, w.est_bytes};
  const size_t rows_q = (size_t)s->B * s->Hq * s->N, rows_kv = (size_t)s->B * s->Hkv * s->N;
  w.qp = c.take<__nv_bfloat16>(rows_q * s->d);
  w.kp = c.take<__nv_bfloat16>(rows_kv * s->d);
  w.vp = c.take<__nv_bfloat16>(rows_kv * s->d);
  w.op = c.take<__nv_bfloat16>(rows_q * s->d);
  w.lsep = c.take<float>(rows_q);
  const size_t blocks = (size_t)g.B * nh * (g.N / 64);
  w.bi = c.take<int32_t>(blocks * (size_t)std::max(k_b, 1));
  w.bc = c.take<int32_t>(blocks);
  if (out) *out = w;
  return c.off;
}

// 3-D fp32 view of the pooled score matrices [bh, nb, nb]: x = key block,
// y = query block, z = slot, with 32 x 128 x 1 boxes (128-byte swizzled).
bool make_scores_map(CUtensorMap* m, const void* ptr, long long bh, int nb) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)nb, (cuuint64_t)nb, (cuuint64_t)bh};
  cuuint64_t strides[2] = {(cuuint64_t)nb * 4, (cuuint64_t)nb * nb * 4};
  cuuint32_t box[3] = {32, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(ptr), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_parts_map(CUtensorMap* m, const void* ptr, long long bh, int nb, int d) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)nb, (cuuint64_t)(3 * bh)};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)nb * d * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Checks the arguments every attention call shares and fills the common
// part of the launch parameters (no segment yet).
minf_status attn_common(const minf_shape* s, const minf_bf16* Q, const minf_bf16* K, const minf_bf16* V,
                        minf_bf16* O, float* lse, void* ws, size_t ws_bytes, AttnParams& p) {
  minf_status st = check_shape(s);
  if (st != MINF_OK) return st;
  if (!Q || !K || !V || !O || !ws) return MINF_ERR_INVALID_ARG;
  if (ws_bytes < kStatusBytes) return MINF_ERR_WORKSPACE_TOO_SMALL;
  if (((uintptr_t)Q | (uintptr_t)K | (uintptr_t)V | (uintptr_t)O) & 15) return MINF_ERR_INVALID_ARG;
  std::memset(&p, 0, sizeof(p));
  p.Q = reinterpret_cast<const __nv_bfloat16*>(Q);
  p.K = reinterpret_cast<const __nv_bfloat16*>(K);
  p.V = reinterpret_cast<const __nv_bfloat16*>(V);
  p.O = reinterpret_cast<__nv_bfloat16*>(O);
  p.lse = lse;
  p.B = s->B;
  p.Hq = s->Hq;
  p.Hkv = s->Hkv;
  p.N = s->N;
  p.group = s->Hq / s->Hkv;
  p.scale_log2 = eff_scale(s) * 1.4426950408889634f;
  p.status = reinterpret_cast<DevStatus*>(ws);
  return MINF_OK;
}

// Appends a pattern's heads (heads == NULL means heads 0 .. nh-1).
minf_status add_seg(AttnParams& p, int pol, const int32_t* heads, int nh) {
  if (nh < 1 || nh > p.Hq || p.nseg >= 3) return MINF_ERR_INVALID_ARG;
  p.seg[p.nseg].pol = pol;
  p.seg[p.nseg].heads = heads;
  p.seg[p.nseg].nh = nh;
  ++p.nseg;
  p.nh_total += nh;
  return p.nh_total <= p.Hq ? MINF_OK : MINF_ERR_INVALID_ARG;
}

minf_status attn_launch(const minf_shape* s, AttnParams& p, void* stream) {
  if (p.nseg < 1) return MINF_ERR_INVALID_ARG;
  p.nqt = s->N / 128;
  const long long items = (long long)p.nqt * s->B * p.nh_total;
  if (items >= (1ll << 31)) return MINF_ERR_UNSUPPORTED;
  p.nitems = (int)items;
  CUtensorMap tq, tk, tv, tk2, tv2;
  const long long kv_rows = (long long)s->B * s->Hkv * s->N;
  if (!make_map(&tq, p.Q, (long long)s->B * s->Hq * s->N, s->d, 128) || !make_map(&tk, p.K, kv_rows, s->d, 64) ||
      !make_map(&tv, p.V, kv_rows, s->d, 64) || !make_map3(&tk2, p.K, kv_rows, s->d, 128) ||
      !make_map3(&tv2, p.V, kv_rows, s->d, 128))
    return MINF_ERR_CUDA;
  return cuda_status(attn_dispatch(s->d, tq, tk, tv, tk2, tv2, p, (cudaStream_t)stream));
}

bool vs_index_ok(const minf_vs_index* idx) {
  return idx && idx->tgrp && idx->tgrp_cnt && idx->wmap && idx->vcnt && idx->vidx && idx->tvcnt && idx->tvidx;
}

void set_vs_index(AttnParams& p, const minf_shape* s, const minf_vs_index* idx, int k_v, int k_s) {
  p.tgrp = idx->tgrp;
  p.tgrp_cnt = idx->tgrp_cnt;
  p.wmap = idx->wmap;
  p.vcnt = idx->vcnt;
  p.vidx = idx->vidx;
  p.tvcnt = idx->tvcnt;
  p.tvidx = idx->tvidx;
  p.k_s = k_s;
  p.k_v = k_v;
  p.wmap_words = (int)minf_vs_wmap_words(s->N);
}

}  // namespace

extern "C" {

size_t minf_vs_wmap_words(int N) { return N > 0 ? (size_t)(N + 64) / 32 + 2 : 0; }
size_t minf_vs_bits_words(int N) { return N > 0 ? (size_t)N / 32 + 8 : 0; }
size_t minf_vs_twmap_words(int N) { return N > 0 ? (size_t)(N + 128) / 32 + 2 : 0; }

size_t minf_workspace_size(int op, const minf_shape* s, int nh, int k_v, int k_s, int k_b) {
  (void)k_v;
  (void)k_s;
  (void)k_b;
  if (!shape_ok(s) || nh < 1) return 0;
  switch (op) {
    case MINF_OP_ESTIMATE_VS:
      return plan_vs_est(s, nh, nullptr, nullptr);
    case MINF_OP_ESTIMATE_BS:
      return plan_bs_est(s, nh, k_b, nullptr, nullptr);
    case MINF_OP_BUILD_INDEX:
    case MINF_OP_BUILD_INDEX_EXACT:
    case MINF_OP_SPARSE_ATTN_VS_EXACT:
    case MINF_OP_SPARSE_ATTN_VS:
    case MINF_OP_SPARSE_ATTN_BS:
    case MINF_OP_ATTN_ASHAPE:
    case MINF_OP_DENSE_ATTN:
    case MINF_OP_SPARSE_ATTN_LAYER:
      return kStatusBytes;
    case MINF_OP_ATTN_GRID:
      return plan_grid(s, nh, k_b, 1, nullptr, nullptr);  // one token per frame needs the most
    default:
      return 0;
  }
}

minf_status minf_estimate_vs(const minf_shape* s, const minf_bf16* Q, const minf_bf16* K, const int32_t* heads,
                             int nh, int last_q, int k_v, int k_s, int32_t* v_idx, int32_t* s_idx, float* v_score,
                             float* s_score, void* ws, size_t ws_bytes, void* stream) {
  minf_status st = check_shape(s);
  if (st != MINF_OK) return st;
  if (!Q || !K || !heads || !v_idx || !s_idx || !ws) return MINF_ERR_INVALID_ARG;
  if (nh < 1 || nh > s->Hq || last_q < 1 || last_q > 64) return MINF_ERR_INVALID_ARG;
  if (k_v < 1 || k_s < 1 || k_v > s->N || k_s > s->N) return MINF_ERR_INVALID_ARG;
  if (ws_bytes < plan_vs_est(s, nh, nullptr, nullptr)) return MINF_ERR_WORKSPACE_TOO_SMALL;
  VsEstWs w;
  plan_vs_est(s, nh, (char*)ws, &w);
  VsEstParams p;
  p.Q = reinterpret_cast<const __nv_bfloat16*>(Q);
  p.K = reinterpret_cast<const __nv_bfloat16*>(K);
  p.heads = heads;
  p.nh = nh;
  p.B = s->B;
  p.Hq = s->Hq;
  p.Hkv = s->Hkv;
  p.N = s->N;
  p.d = s->d;
  p.group = s->Hq / s->Hkv;
  p.last_q = last_q;
  p.scale_log2 = eff_scale(s) * 1.4426950408889634f;
  p.part_ml = w.part_ml;
  p.row_ml = w.row_ml;
  p.v_score = v_score ? v_score : w.v_score;
  p.s_score = s_score ? s_score : w.s_score;
  p.dpart = w.dpart;
  p.status = w.status;
  cudaStream_t cs = (cudaStream_t)stream;
  CUtensorMap tq, tk;
  if (((uintptr_t)Q | (uintptr_t)K) & 15) return MINF_ERR_INVALID_ARG;
  if (!make_map(&tq, Q, (long long)s->B * s->Hq * s->N, s->d, 64) ||
      !make_map(&tk, K, (long long)s->B * s->Hkv * s->N, s->d, 64))
    return MINF_ERR_CUDA;
  cudaError_t e = vs_estimate_tc_launch(tq, tk, p, cs);
  if (e != cudaSuccess) return MINF_ERR_CUDA;
  TopkRows t;
  t.scores = p.v_score;
  t.row_stride = s->N;
  t.rows = s->B * nh;
  t.len_mode = 0;
  t.len = s->N;
  t.rows_per_group = 1;
  t.forced_mode = 0;
  t.k = k_v;
  t.out_idx = v_idx;
  t.out_cnt = nullptr;
  t.status = w.status;
  t.scratch = w.topk;
  e = topk_rows_launch(t, cs);
  if (e != cudaSuccess) return MINF_ERR_CUDA;
  t.scores = p.s_score;
  t.forced_mode = 1;
  t.k = k_s;
  t.out_idx = s_idx;
  return cuda_status(topk_rows_launch(t, cs));
}

minf_status minf_estimate_bs(const minf_shape* s, const minf_bf16* Q, const minf_bf16* K, const int32_t* heads,
                             int nh, int block, int k_b, int32_t* blk_idx, int32_t* blk_cnt, float* blk_score,
                             void* ws, size_t ws_bytes, void* stream) {
  minf_status st = check_shape(s);
  if (st != MINF_OK) return st;
  if (!Q || !K || !heads || !blk_idx || !blk_cnt || !ws) return MINF_ERR_INVALID_ARG;
  if (nh < 1 || nh > s->Hq || k_b < 1) return MINF_ERR_INVALID_ARG;
  if (block != 64) return MINF_ERR_UNSUPPORTED;
  // the tensor-core path, unless the workspace was sized without it (k_b = 0)
  const bool fused = bs_select_supported(s->N, s->d, k_b) && ws_bytes >= plan_bs_est(s, nh, k_b, nullptr, nullptr);
  if (!fused && ws_bytes < plan_bs_est(s, nh, 0, nullptr, nullptr)) return MINF_ERR_WORKSPACE_TOO_SMALL;
  BsEstWs w;
  plan_bs_est(s, nh, fused ? k_b : 0, (char*)ws, &w);
  BsEstParams p;
  p.Q = reinterpret_cast<const __nv_bfloat16*>(Q);
  p.K = reinterpret_cast<const __nv_bfloat16*>(K);
  p.heads = heads;
  p.nh = nh;
  p.B = s->B;
  p.Hq = s->Hq;
  p.Hkv = s->Hkv;
  p.N = s->N;
  p.d = s->d;
  p.group = s->Hq / s->Hkv;
  p.scale = eff_scale(s);
  p.qbar = w.qbar;
  p.kbar = w.kbar;
  p.scores = blk_score ? blk_score : w.scores;
  p.qs = fused ? w.qs : nullptr;
  p.ks = fused ? w.ks : nullptr;
  p.status = w.status;
  cudaStream_t cs = (cudaStream_t)stream;
  const int nb = s->N / 64;
  if (fused) {
    CUtensorMap tm, tms;
    if (!make_parts_map(&tm, w.ks, (long long)s->B * nh, nb, s->d) ||
        !make_scores_map(&tms, p.scores, (long long)s->B * nh, nb))
      return MINF_ERR_CUDA;
    BsEstParams pool = p;
    pool.scores = nullptr;  // pooling and split only
    cudaError_t e = bs_pool_score_launch(pool, cs);
    if (e != cudaSuccess) return MINF_ERR_CUDA;
    return cuda_status(bs_select_launch(tm, tms, p, k_b, blk_idx, blk_cnt, cs));
  }
  cudaError_t e = bs_pool_score_launch(p, cs);
  if (e != cudaSuccess) return MINF_ERR_CUDA;
  TopkRows t;
  t.scores = p.scores;
  t.row_stride = nb;
  t.rows = s->B * nh * nb;
  t.len_mode = 1;
  t.len = nb;
  t.rows_per_group = nb;
  t.forced_mode = 2;
  t.k = k_b;
  t.out_idx = blk_idx;
  t.out_cnt = blk_cnt;
  t.status = w.status;
  t.scratch = nullptr;
  return cuda_status(topk_rows_launch(t, cs));
}

minf_status minf_attn_grid(const minf_shape* s, const minf_bf16* Q, const minf_bf16* K, const minf_bf16* V,
                           const int32_t* heads, int nh, int frame_tokens, int k_b, int32_t* blk_idx,
                           int32_t* blk_cnt, minf_bf16* O, float* lse, void* ws, size_t ws_bytes, void* stream) {
  minf_status st = check_shape(s);
  if (st != MINF_OK) return st;
  if (!Q || !K || !V || !heads || !O || !ws || nh < 1 || nh > s->Hq || k_b < 1) return MINF_ERR_INVALID_ARG;
  const int P = frame_tokens;
  if (P < 1 || s->N % P != 0 || (s->N / P) % 128 != 0) return MINF_ERR_INVALID_ARG;
  if (((uintptr_t)Q | (uintptr_t)K | (uintptr_t)V | (uintptr_t)O) & 15) return MINF_ERR_INVALID_ARG;
  if (ws_bytes < plan_grid(s, nh, k_b, P, nullptr, nullptr)) return MINF_ERR_WORKSPACE_TOO_SMALL;
  GridWs w;
  plan_grid(s, nh, k_b, P, (char*)ws, &w);
  const minf_shape g = grid_shape(s, P);
  int32_t* bi = blk_idx ? blk_idx : w.bi;
  int32_t* bc = blk_cnt ? blk_cnt : w.bc;
  cudaStream_t cs = (cudaStream_t)stream;
  GridPermParams gp;
  gp.B = s->B;
  gp.N = s->N;
  gp.F = s->N / P;
  gp.P = P;
  gp.d = s->d;
  gp.status = reinterpret_cast<DevStatus*>(ws);
  gp.dir = 0;
  gp.lse_src = nullptr;
  gp.lse_dst = nullptr;
  // the listed heads' Q rows and every KV head's K and V rows, position-major
  gp.src = reinterpret_cast<const __nv_bfloat16*>(Q);
  gp.dst = w.qp;
  gp.heads = heads;
  gp.nh = nh;
  gp.H = s->Hq;
  if (grid_permute_launch(gp, cs) != cudaSuccess) return MINF_ERR_CUDA;
  gp.heads = nullptr;
  gp.nh = s->Hkv;
  gp.H = s->Hkv;
  gp.src = reinterpret_cast<const __nv_bfloat16*>(K);
  gp.dst = w.kp;
  if (grid_permute_launch(gp, cs) != cudaSuccess) return MINF_ERR_CUDA;
  gp.src = reinterpret_cast<const __nv_bfloat16*>(V);
  gp.dst = w.vp;
  if (grid_permute_launch(gp, cs) != cudaSuccess) return MINF_ERR_CUDA;
  // Block-Sparse estimation and attention on the B * P position sequences;
  // both share the call's status block (at the workspace's start)
  const minf_bf16* qp = reinterpret_cast<const minf_bf16*>(w.qp);
  const minf_bf16* kp = reinterpret_cast<const minf_bf16*>(w.kp);
  const minf_bf16* vp = reinterpret_cast<const minf_bf16*>(w.vp);
  st = minf_estimate_bs(&g, qp, kp, heads, nh, 64, k_b, bi, bc, nullptr, w.est, w.est_bytes, stream);
  if (st != MINF_OK) return st;
  st = minf_sparse_attn_bs(&g, qp, kp, vp, heads, nh, bi, bc, k_b, reinterpret_cast<minf_bf16*>(w.op),
                           lse ? w.lsep : nullptr, ws, kStatusBytes, stream);
  if (st != MINF_OK) return st;
  // the output (and LSE) rows back to frame-major order
  gp.dir = 1;
  gp.src = w.op;
  gp.dst = reinterpret_cast<__nv_bfloat16*>(O);
  gp.heads = heads;
  gp.nh = nh;
  gp.H = s->Hq;
  gp.lse_src = lse ? w.lsep : nullptr;
  gp.lse_dst = lse;
  return cuda_status(grid_permute_launch(gp, cs));
}

minf_status minf_build_index(const minf_shape* s, int nh, const int32_t* v_idx, int k_v, const int32_t* s_idx,
                             int k_s, const minf_vs_index* idx, void* ws, size_t ws_bytes, void* stream) {
  minf_status st = check_shape(s);
  if (st != MINF_OK) return st;
  if (!v_idx || !s_idx || !idx || !ws || nh < 1) return MINF_ERR_INVALID_ARG;
  if (!idx->grp || !idx->grp_cnt || !idx->tgrp || !idx->tgrp_cnt || !idx->wmap || !idx->vcnt || !idx->vidx ||
      !idx->tvcnt || !idx->tvidx)
    return MINF_ERR_INVALID_ARG;
  if (k_v < 1 || k_s < 1 || k_v > s->N || k_s > s->N) return MINF_ERR_INVALID_ARG;
  if (s->N > (1 << 30)) return MINF_ERR_UNSUPPORTED;  // tvidx keeps the key in 30 bits
  if (ws_bytes < kStatusBytes) return MINF_ERR_WORKSPACE_TOO_SMALL;
  VsIndexParams p;
  p.v_idx = v_idx;
  p.s_idx = s_idx;
  p.nh = nh;
  p.B = s->B;
  p.N = s->N;
  p.k_v = k_v;
  p.k_s = k_s;
  p.wmap_words = (int)minf_vs_wmap_words(s->N);
  p.idx = *idx;
  p.status = reinterpret_cast<DevStatus*>(ws);
  return cuda_status(vs_index_launch(p, (cudaStream_t)stream));
}

minf_status minf_build_index_exact(const minf_shape* s, int nh, const int32_t* v_idx, int k_v,
                                   const int32_t* s_idx, int k_s, const minf_vs_exact_index* idx, void* ws,
                                   size_t ws_bytes, void* stream) {
  minf_status st = check_shape(s);
  if (st != MINF_OK) return st;
  if (!v_idx || !s_idx || !idx || !ws || nh < 1) return MINF_ERR_INVALID_ARG;
  if (!idx->tgrp || !idx->tgrp_cnt || !idx->sbits || !idx->vbits || !idx->twmap || !idx->vcnt || !idx->vidx)
    return MINF_ERR_INVALID_ARG;
  if (k_v < 1 || k_s < 1 || k_v > s->N || k_s > s->N) return MINF_ERR_INVALID_ARG;
  if (ws_bytes < kStatusBytes) return MINF_ERR_WORKSPACE_TOO_SMALL;
  VsIndexParams p;
  std::memset(&p, 0, sizeof(p));
  p.v_idx = v_idx;
  p.s_idx = s_idx;
  p.nh = nh;
  p.B = s->B;
  p.N = s->N;
  p.k_v = k_v;
  p.k_s = k_s;
  p.status = reinterpret_cast<DevStatus*>(ws);
  return cuda_status(vs_exact_index_launch(p, *idx, (int)minf_vs_bits_words(s->N), (int)minf_vs_twmap_words(s->N),
                                           (cudaStream_t)stream));
}

minf_status minf_sparse_attn_vs_exact(const minf_shape* s, const minf_bf16* Q, const minf_bf16* K,
                                      const minf_bf16* V, const int32_t* heads, int nh,
                                      const minf_vs_exact_index* idx, int k_v, int k_s, minf_bf16* O, float* lse,
                                      void* ws, size_t ws_bytes, void* stream) {
  AttnParams p;
  minf_status st = attn_common(s, Q, K, V, O, lse, ws, ws_bytes, p);
  if (st != MINF_OK) return st;
  if (!heads || (st = add_seg(p, POL_VS_EXACT, heads, nh)) != MINF_OK) return MINF_ERR_INVALID_ARG;
  if (!idx || !idx->tgrp || !idx->tgrp_cnt || !idx->sbits || !idx->vbits || !idx->twmap || !idx->vcnt ||
      !idx->vidx)
    return MINF_ERR_INVALID_ARG;
  if (k_v < 1 || k_s < 1 || k_v > s->N || k_s > s->N) return MINF_ERR_INVALID_ARG;
  p.tgrp = idx->tgrp;
  p.tgrp_cnt = idx->tgrp_cnt;
  p.sbits = idx->sbits;
  p.vbits = idx->vbits;
  p.twmap = idx->twmap;
  p.bits_words = (int)minf_vs_bits_words(s->N);
  p.twmap_words = (int)minf_vs_twmap_words(s->N);  // unused by the kernel; kept with the index
  p.vcnt = idx->vcnt;
  p.vidx = idx->vidx;
  p.k_s = k_s;
  p.k_v = k_v;
  return attn_launch(s, p, stream);
}

minf_status minf_sparse_attn_vs(const minf_shape* s, const minf_bf16* Q, const minf_bf16* K, const minf_bf16* V,
                                const int32_t* heads, int nh, const minf_vs_index* idx, int k_v, int k_s,
                                minf_bf16* O, float* lse, void* ws, size_t ws_bytes, void* stream) {
  AttnParams p;
  minf_status st = attn_common(s, Q, K, V, O, lse, ws, ws_bytes, p);
  if (st != MINF_OK) return st;
  if (!heads || add_seg(p, POL_VS, heads, nh) != MINF_OK) return MINF_ERR_INVALID_ARG;
  if (!vs_index_ok(idx)) return MINF_ERR_INVALID_ARG;
  if (k_v < 1 || k_s < 1 || k_v > s->N || k_s > s->N) return MINF_ERR_INVALID_ARG;
  set_vs_index(p, s, idx, k_v, k_s);
  return attn_launch(s, p, stream);
}

minf_status minf_sparse_attn_bs(const minf_shape* s, const minf_bf16* Q, const minf_bf16* K, const minf_bf16* V,
                                const int32_t* heads, int nh, const int32_t* blk_idx, const int32_t* blk_cnt,
                                int k_b, minf_bf16* O, float* lse, void* ws, size_t ws_bytes, void* stream) {
  AttnParams p;
  minf_status st = attn_common(s, Q, K, V, O, lse, ws, ws_bytes, p);
  if (st != MINF_OK) return st;
  if (!heads || add_seg(p, POL_BS, heads, nh) != MINF_OK) return MINF_ERR_INVALID_ARG;
  if (!blk_idx || !blk_cnt || k_b < 1) return MINF_ERR_INVALID_ARG;
  p.blk_idx = blk_idx;
  p.blk_cnt = blk_cnt;
  p.k_b = k_b;
  return attn_launch(s, p, stream);
}

minf_status minf_attn_ashape(const minf_shape* s, const minf_bf16* Q, const minf_bf16* K, const minf_bf16* V,
                             const int32_t* heads, int nh, int n_sink, int n_local, minf_bf16* O, float* lse,
                             void* ws, size_t ws_bytes, void* stream) {
  AttnParams p;
  minf_status st = attn_common(s, Q, K, V, O, lse, ws, ws_bytes, p);
  if (st != MINF_OK) return st;
  if (!heads || add_seg(p, POL_ASHAPE, heads, nh) != MINF_OK) return MINF_ERR_INVALID_ARG;
  if (n_sink < 0 || n_local < 1) return MINF_ERR_INVALID_ARG;
  p.n_sink = n_sink;
  p.n_local = n_local;
  return attn_launch(s, p, stream);
}

minf_status minf_dense_attn(const minf_shape* s, const minf_bf16* Q, const minf_bf16* K, const minf_bf16* V,
                            const int32_t* heads, int nh, minf_bf16* O, float* lse, void* ws, size_t ws_bytes,
                            void* stream) {
  AttnParams p;
  minf_status st = attn_common(s, Q, K, V, O, lse, ws, ws_bytes, p);
  if (st != MINF_OK) return st;
  if (!heads) nh = s->Hq;
  if (add_seg(p, POL_DENSE, heads, nh) != MINF_OK) return MINF_ERR_INVALID_ARG;
  return attn_launch(s, p, stream);
}

minf_status minf_sparse_attn_layer(const minf_shape* s, const minf_bf16* Q, const minf_bf16* K,
                                   const minf_bf16* V, const int32_t* vs_heads, int n_vs,
                                   const minf_vs_index* vs_idx, int k_v, int k_s, const int32_t* bs_heads,
                                   int n_bs, const int32_t* blk_idx, const int32_t* blk_cnt, int k_b,
                                   const int32_t* a_heads, int n_a, int n_sink, int n_local, minf_bf16* O,
                                   float* lse, void* ws, size_t ws_bytes, void* stream) {
  AttnParams p;
  minf_status st = attn_common(s, Q, K, V, O, lse, ws, ws_bytes, p);
  if (st != MINF_OK) return st;
  if (n_vs < 0 || n_bs < 0 || n_a < 0 || n_vs + n_bs + n_a < 1) return MINF_ERR_INVALID_ARG;
  if (n_vs > 0) {
    if (!vs_heads || add_seg(p, POL_VS, vs_heads, n_vs) != MINF_OK || !vs_index_ok(vs_idx))
      return MINF_ERR_INVALID_ARG;
    if (k_v < 1 || k_s < 1 || k_v > s->N || k_s > s->N) return MINF_ERR_INVALID_ARG;
    set_vs_index(p, s, vs_idx, k_v, k_s);
  }
  if (n_bs > 0) {
    if (!bs_heads || add_seg(p, POL_BS, bs_heads, n_bs) != MINF_OK || !blk_idx || !blk_cnt || k_b < 1)
      return MINF_ERR_INVALID_ARG;
    p.blk_idx = blk_idx;
    p.blk_cnt = blk_cnt;
    p.k_b = k_b;
  }
  if (n_a > 0) {
    if (!a_heads || add_seg(p, POL_ASHAPE, a_heads, n_a) != MINF_OK || n_sink < 0 || n_local < 1)
      return MINF_ERR_INVALID_ARG;
    p.n_sink = n_sink;
    p.n_local = n_local;
  }
  return attn_launch(s, p, stream);
}

minf_status minf_get_device_status(void* ws, void* stream) {
  if (!ws) return MINF_ERR_INVALID_ARG;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MINF_ERR_CUDA;
  DevStatus h{0, 0};
  if (cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return MINF_ERR_CUDA;
  if (h.code != 0 && cudaMemset(ws, 0, sizeof(h)) != cudaSuccess) return MINF_ERR_CUDA;
  if (h.code == 0) return MINF_OK;
  return (minf_status)h.code;
}

const char* minf_status_string(minf_status s) {
  switch (s) {
    case MINF_OK: return "ok";
    case MINF_ERR_INVALID_ARG: return "invalid argument";
    case MINF_ERR_UNSUPPORTED: return "unsupported configuration";
    case MINF_ERR_CUDA: return "CUDA error";
    case MINF_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MINF_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case MINF_ERR_DEVICE_BOUNDS: return "device index out of range";
  }
  return "unknown status";
}

}  // extern "C"
