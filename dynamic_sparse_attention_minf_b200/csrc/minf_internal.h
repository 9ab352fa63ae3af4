// Internal declarations shared by the host launcher (api.cu) and the kernel
// translation units of libminf.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/minf.h"

namespace minf {

struct DevStatus;

enum { POL_DENSE = 0, POL_ASHAPE = 1, POL_VS = 2, POL_BS = 3, POL_VS_EXACT = 4 };

// One pattern's heads in an attention launch.  Work items are 128-row query
// tiles of one (batch, head); a launch may hold up to three segments (one per
// pattern), whose items interleave.
struct AttnSeg {
  int pol;
  const int32_t* heads;  // nh query-head ids, or NULL for heads 0 .. nh-1
  int nh;
};

struct AttnParams {
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  __nv_bfloat16* O;
  float* lse;
  AttnSeg seg[3];
  int nseg, nh_total;
  int nqt, nitems;      // query tiles N / 128; items = nqt * B * nh_total
  int B, Hq, Hkv, N, group;
  float scale_log2;  // softmax scale * log2(e)
  // A-shape
  int n_sink, n_local;
  // Vertical-Slash index (band reading: tgrp, wmap, per-128-row-tile gather
  // lists tvcnt / tvidx; exact reading: tgrp, twmap, sbits, vbits,
  // per-128-row-tile lists vcnt / vidx)
  const int32_t* tgrp;
  const int32_t* tgrp_cnt;
  const uint32_t* wmap;
  const uint32_t* twmap;
  const int32_t* vcnt;
  const int32_t* vidx;
  const int32_t* tvcnt;
  const int32_t* tvidx;
  int k_s, k_v, wmap_words, twmap_words;
  const uint32_t* sbits;
  const uint32_t* vbits;
  int bits_words;
  // Block-Sparse index
  const int32_t* blk_idx;
  const int32_t* blk_cnt;
  int k_b;
  DevStatus* status;
};

// tq: Q with 128-row boxes; tk/tv: K and V with 64-row boxes; tk2/tv2: K and V
// with 128-row boxes (all 128-byte swizzled, 64 columns wide).  One CTA per
// work item.
cudaError_t attn_dispatch(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          const CUtensorMap& tk2, const CUtensorMap& tv2, const AttnParams& p, cudaStream_t stream);

// ---- estimation / index kernels (estimate.cu, index.cu)
struct VsEstParams {
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  const int32_t* heads;
  int nh, B, Hq, Hkv, N, d, group, last_q;
  float scale_log2;
  float* part_ml;     // [B, nh, ntiles, 64, 2] per-tile (max, sum) of each row
  float* row_ml;      // [B, nh, 64, 2] combined (max, 1/sum)
  float* v_score;     // [B, nh, N]
  float* dpart;       // [B, nh, ntiles, 192] per-tile diagonal partial sums
  float* s_score;     // [B, nh, N]
  DevStatus* status;
};
cudaError_t vs_combine_launch(const VsEstParams& p, int nparts, cudaStream_t stream);
cudaError_t vs_slash_launch(const VsEstParams& p, cudaStream_t stream);
// tensor-core estimation: tq and tk view Q and K as [rows, d] with 64-row
// boxes (128-byte swizzled)
cudaError_t vs_estimate_tc_launch(const CUtensorMap& tq, const CUtensorMap& tk, const VsEstParams& p,
                                  cudaStream_t stream);

struct TopkRows {
  const float* scores;   // row r's scores start at scores + r * row_stride (+ offset)
  long long row_stride;
  int rows;              // total rows
  int len_mode;          // 0: every row has length `len`; 1: row r has length (r % rows_per_group) + 1
  int len;
  int rows_per_group;
  int forced_mode;       // 0: none; 1: index 0; 2: index (r % rows_per_group)
  int k;
  int32_t* out_idx;      // [rows, k] ascending, -1 padded
  int32_t* out_cnt;      // [rows] or NULL
  DevStatus* status;
  uint32_t* scratch;     // rows * kTopkScratchWords words for rows longer than kTopkLongRow, or NULL
};
// Rows longer than this (with len_mode 0) are split over many CTAs, given
// topk_scratch_words(rows) words of scratch; shorter rows take one CTA each.
constexpr int kTopkLongRow = 32768;
constexpr int kTopkScratchWords = 2048 + 8 + 2 * 1024;
inline size_t topk_scratch_words(int rows) { return (size_t)rows * kTopkScratchWords; }
cudaError_t topk_rows_launch(const TopkRows& t, cudaStream_t stream);

struct BsEstParams {
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  const int32_t* heads;
  int nh, B, Hq, Hkv, N, d, group;
  float scale;
  float* qbar;     // [B, nh, nb, d]
  float* kbar;     // [B, nh, nb, d]
  float* scores;   // [B, nh, nb, nb]
  __nv_bfloat16* qs;  // [3, B, nh, nb, d]: qbar = qs[0] + qs[1] + qs[2] (bf16 parts), or NULL
  __nv_bfloat16* ks;  // [3, B, nh, nb, d], the same for kbar
  DevStatus* status;
};
// Pools Q and K per 64-row block (and splits the means into bf16 parts when
// qs / ks are set); when `scores` is set, also writes the pooled score matrix.
cudaError_t bs_pool_score_launch(const BsEstParams& p, cudaStream_t stream);

// Block-Sparse selection fused with the pooled scores on the tensor cores
// (bs_select.cu): from the split means, the k best key blocks of every query
// block, diagonal forced, in ascending order.
// tmKs: the key parts as a 3-D bf16 view (x = d, y = key block, z = part *
// B * nh + batch * nh + head slot) with 64 x 128 x 1 boxes; tmS: the score
// matrices as a 3-D fp32 view (x = key block, y = query block, z = batch * nh
// + head slot) with 32 x 128 x 1 boxes; both 128-byte swizzled.
bool bs_select_supported(int N, int d, int k);
cudaError_t bs_select_launch(const CUtensorMap& tmKs, const CUtensorMap& tmS, const BsEstParams& p, int k,
                             int32_t* blk_idx, int32_t* blk_cnt, cudaStream_t stream);

// Grid pattern row permutation (grid.cu): dir 0 gathers frame-major rows
// [B, H, F * P, d] into position-major [B * P, H, F, d], dir 1 scatters back;
// only the listed heads' rows (heads NULL: 0 .. nh-1); lse rows follow when set.
struct GridPermParams {
  const __nv_bfloat16* src;
  __nv_bfloat16* dst;
  const float* lse_src;
  float* lse_dst;
  const int32_t* heads;
  int nh, B, H, N, F, P, d, dir;
  DevStatus* status;
};
cudaError_t grid_permute_launch(const GridPermParams& p, cudaStream_t stream);

struct VsIndexParams {
  const int32_t* v_idx;
  const int32_t* s_idx;
  int nh, B, N, k_v, k_s, wmap_words;
  minf_vs_index idx;
  DevStatus* status;
};
cudaError_t vs_index_launch(const VsIndexParams& p, cudaStream_t stream);
cudaError_t vs_exact_index_launch(const VsIndexParams& p, const minf_vs_exact_index& x, int bits_words,
                                  int twmap_words, cudaStream_t stream);

}  // namespace minf
