// Vertical-Slash index build.  A slash offset o sweeps, through a 64-row
// query block with first row r0, the keys r0 - o .. r0 + 63 - o; offsets
// closer than 64 therefore merge into one contiguous band per block (a
// "group"), and offsets closer than 128 into one band per 128-row tile.
// Written from the summary page of "MInference 1.0" ("Key points": vertical
// and slash lines estimated from the last queries), with the band reading of
// a slash documented in the design notes.
//
//  1. groups:   scan of the ascending offsets -> (a_g, b_g) at gap 64 and 128
//  2. bitmap:   bit x <=> block offset u = x - 63 lies in some [a_g - 63, b_g]
//  3. verticals: per query block, the vertical columns off every band
#include "minf_device.cuh"
#include "minf_internal.h"

namespace minf {

__device__ __forceinline__ int block_excl_scan_int(int v, int* wsum, int& total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[w] = x;
  __syncthreads();
  if (w == 0) {
    int s = (lane < nw) ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, s, o);
      if (lane >= o) s += y;
    }
    wsum[lane] = s;
  }
  __syncthreads();
  const int before = (w > 0) ? wsum[w - 1] : 0;
  total = wsum[nw - 1];
  __syncthreads();
  return x - v + before;
}

// One CTA per (batch, head): validates both index lists and writes the groups.
__global__ void __launch_bounds__(1024) vs_groups_kernel(const VsIndexParams p) {
  const int hi = blockIdx.x, b = blockIdx.y;
  const size_t bh = (size_t)b * p.nh + hi;
  const int* s = p.s_idx + bh * p.k_s;
  const int* v = p.v_idx + bh * p.k_v;
  __shared__ int wsum[32];
  // validation: ascending, in range
  for (int x = threadIdx.x; x < p.k_v; x += blockDim.x) {
    const int j = v[x];
    if (j < 0 || j >= p.N || (x > 0 && v[x - 1] >= j)) report(p.status, MINF_ERR_DEVICE_BOUNDS, 50);
  }
  for (int x = threadIdx.x; x < p.k_s; x += blockDim.x) {
    const int o = s[x];
    if (o < 0 || o >= p.N || (x > 0 && s[x - 1] >= o)) report(p.status, MINF_ERR_DEVICE_BOUNDS, 51);
  }
  int32_t* grp = p.idx.grp ? p.idx.grp + bh * p.k_s * 2 : nullptr;  // null: tile groups only
  int32_t* tgrp = p.idx.tgrp + bh * p.k_s * 2;
  int run_g = 0, run_t = 0;
  for (int base = 0; base < p.k_s; base += blockDim.x) {
    const int x = base + threadIdx.x;
    const bool valid = x < p.k_s;
    const int o = valid ? s[x] : 0;
    const int prev = (valid && x > 0) ? s[x - 1] : 0;
    const int next = (valid && x + 1 < p.k_s) ? s[x + 1] : 0;
    const bool start_g = valid && (x == 0 || o - prev > 64);
    const bool end_g = valid && (x + 1 == p.k_s || next - o > 64);
    const bool start_t = valid && (x == 0 || o - prev > 128);
    const bool end_t = valid && (x + 1 == p.k_s || next - o > 128);
    int tot_g, tot_t;
    const int eg = block_excl_scan_int(start_g ? 1 : 0, wsum, tot_g);
    const int et = block_excl_scan_int(start_t ? 1 : 0, wsum, tot_t);
    // group index of element x = (#starts up to and including x) - 1
    const int gi = run_g + eg + (start_g ? 1 : 0) - 1;
    const int ti = run_t + et + (start_t ? 1 : 0) - 1;
    if (grp && start_g) grp[2 * gi] = o;
    if (grp && end_g) grp[2 * gi + 1] = o;
    if (start_t) tgrp[2 * ti] = o;
    if (end_t) tgrp[2 * ti + 1] = o;
    run_g += tot_g;
    run_t += tot_t;
  }
  if (threadIdx.x == 0) {
    if (p.idx.grp_cnt) p.idx.grp_cnt[bh] = run_g;
    p.idx.tgrp_cnt[bh] = run_t;
  }
}

// One thread per bitmap word: bit x set iff x - (BLK - 1) lies in some
// [a_g - (BLK - 1), b_g] of the given groups (the groups of gap BLK).
template <int BLK>
__global__ void __launch_bounds__(256) vs_wmap_kernel(const VsIndexParams p, const int32_t* grps,
                                                      const int32_t* gcnt, uint32_t* wmap, int words) {
  const int w = blockIdx.x * 256 + threadIdx.x;
  const int hi = blockIdx.y, b = blockIdx.z;
  if (w >= words) return;
  const size_t bh = (size_t)b * p.nh + hi;
  const int* grp = grps + bh * p.k_s * 2;
  const int G = gcnt[bh];
  const int u_lo = 32 * w - (BLK - 1), u_hi = u_lo + 31;
  // first group with b_g >= u_lo
  int lo = 0, hi2 = G;
  while (lo < hi2) {
    const int mid = (lo + hi2) >> 1;
    if (grp[2 * mid + 1] < u_lo) lo = mid + 1; else hi2 = mid;
  }
  uint32_t word = 0;
  for (int g = lo; g < G; ++g) {
    const int a = grp[2 * g] - (BLK - 1), bb = grp[2 * g + 1];
    if (a > u_hi) break;
    const int s0 = max(a, u_lo) - u_lo, s1 = min(bb, u_hi) - u_lo;
    if (s0 <= s1) {
      const int n = s1 - s0 + 1;
      const uint32_t m = (n >= 32) ? 0xFFFFFFFFu : (((1u << n) - 1u) << s0);
      word |= m;
    }
  }
  wmap[bh * words + w] = word;
}

// One warp per BLK-row query block: the ascending vertical columns j <= the
// block's last row whose bit (r0 - j + BLK - 1) of the group bitmap is clear.
template <int BLK>
__global__ void __launch_bounds__(256) vs_vlist_kernel(const VsIndexParams p, const uint32_t* wmap, int words,
                                                       int32_t* vcnt, int32_t* vidx) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = p.N / BLK;
  const int qb = blockIdx.x * 8 + warp;
  const int hi = blockIdx.y, b = blockIdx.z;
  if (qb >= nb) return;
  const size_t bh = (size_t)b * p.nh + hi;
  const int* v = p.v_idx + bh * p.k_v;
  const uint32_t* W = wmap + bh * words;
  int32_t* out = vidx + (bh * nb + qb) * (size_t)p.k_v;
  const int r0 = qb * BLK;
  int n = 0;
  for (int base = 0; base < p.k_v; base += 32) {
    const int x = base + lane;
    const int j = (x < p.k_v) ? v[x] : 0x7FFFFFFF;
    const bool inr = (j >= 0) && (j <= r0 + BLK - 1);
    bool keep = false;
    if (inr) {
      const int bit = r0 - j + BLK - 1;
      keep = !((__ldg(W + (bit >> 5)) >> (bit & 31)) & 1u);
    }
    const uint32_t bal = __ballot_sync(0xFFFFFFFFu, keep);
    if (keep) out[n + __popc(bal & ((1u << lane) - 1u))] = j;
    n += __popc(bal);
    if (!__all_sync(0xFFFFFFFFu, inr || x >= p.k_v)) break;  // list is ascending
  }
  if (lane == 0) vcnt[bh * nb + qb] = n;
}

// One warp per 128-row query tile t (blocks b0 = 2t, b1 = 2t + 1, first row
// R): the vertical lists of both blocks and the columns the tile gathers.
// Column j is listed for block b (first row r0) when j <= r0 + 63 and bit
// (r0 - j + 63) of the group bitmap is clear.  The tile's entries: first every
// column of block b1's list (bit 31; bit 30 too if block b0 lists it), then
// the columns of block b0's list that block b1 does not list (bit 30 only).
// The first pass over the ascending verticals writes both block lists and the
// first part; a second, up to row R + 63, the second part after it.
__global__ void __launch_bounds__(256) vs_tile_lists_kernel(const VsIndexParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt = p.N / 128, nb = p.N / 64;
  const int qt = blockIdx.x * 8 + warp;
  const int hi = blockIdx.y, b = blockIdx.z;
  if (qt >= nt) return;
  const size_t bh = (size_t)b * p.nh + hi;
  const int* v = p.v_idx + bh * p.k_v;
  const uint32_t* W = p.idx.wmap + bh * p.wmap_words;
  int32_t* out = p.idx.tvidx + (bh * nt + qt) * (size_t)p.k_v;
  int32_t* list0 = p.idx.vidx + (bh * nb + 2 * qt) * (size_t)p.k_v;
  int32_t* list1 = list0 + p.k_v;
  const int R = qt * 128;
  const uint32_t lt = (1u << lane) - 1u;
  auto covered = [&](int bit) -> bool { return (__ldg(W + (bit >> 5)) >> (bit & 31)) & 1u; };
  int n = 0, n0 = 0;
  for (int pass = 0; pass < 2; ++pass) {
    const int last = R + (pass == 0 ? 127 : 63);
    for (int base = 0; base < p.k_v; base += 32) {
      const int x = base + lane;
      const int j = (x < p.k_v) ? v[x] : 0x7FFFFFFF;
      const bool inr = (j >= 0) && (j <= last);
      bool in0 = false, in1 = false;
      if (inr) {
        in0 = (j <= R + 63) && !covered(R - j + 63);  // block b0 lists j
        in1 = !covered(R + 127 - j);                   // block b1 lists j
      }
      const bool keep = (pass == 0) ? in1 : (in0 && !in1);
      const uint32_t e = (uint32_t)j | (in0 ? (1u << 30) : 0u) | (in1 ? (1u << 31) : 0u);
      const uint32_t bal = __ballot_sync(0xFFFFFFFFu, keep);
      if (keep) out[n + __popc(bal & lt)] = (int32_t)e;
      n += __popc(bal);
      if (pass == 0) {
        const uint32_t b0 = __ballot_sync(0xFFFFFFFFu, in0);
        if (in0) list0[n0 + __popc(b0 & lt)] = j;
        if (in1) list1[__popc(bal & lt) + (n - __popc(bal))] = j;
        n0 += __popc(b0);
      }
      if (!__all_sync(0xFFFFFFFFu, inr || x >= p.k_v)) break;  // list is ascending
    }
    if (pass == 0 && lane == 0) {
      p.idx.vcnt[bh * nb + 2 * qt] = n0;
      p.idx.vcnt[bh * nb + 2 * qt + 1] = n;
    }
  }
  if (lane == 0) p.idx.tvcnt[bh * nt + qt] = n;
}

// One thread per word of the offset and key bitmaps: bit o of sbits set iff
// o is in S, bit j of vbits iff j is in V (both lists ascending).
__global__ void __launch_bounds__(256) vs_bits_kernel(const VsIndexParams p, uint32_t* sbits, uint32_t* vbits,
                                                      int words) {
  const int w = blockIdx.x * 256 + threadIdx.x;
  const int hi = blockIdx.y, b = blockIdx.z;
  if (w >= words) return;
  const size_t bh = (size_t)b * p.nh + hi;
  auto word_of = [&](const int* lst, int n) -> uint32_t {
    int lo = 0, hi2 = n;  // first element >= 32 w
    while (lo < hi2) {
      const int mid = (lo + hi2) >> 1;
      if (lst[mid] < 32 * w) lo = mid + 1; else hi2 = mid;
    }
    uint32_t word = 0;
    for (int x = lo; x < n && lst[x] < 32 * w + 32; ++x) word |= 1u << (lst[x] - 32 * w);
    return word;
  };
  sbits[bh * words + w] = word_of(p.s_idx + bh * p.k_s, p.k_s);
  vbits[bh * words + w] = word_of(p.v_idx + bh * p.k_v, p.k_v);
}

cudaError_t vs_index_launch(const VsIndexParams& p, cudaStream_t stream) {
  vs_groups_kernel<<<dim3(p.nh, p.B), 1024, 0, stream>>>(p);
  vs_wmap_kernel<64><<<dim3((p.wmap_words + 255) / 256, p.nh, p.B), 256, 0, stream>>>(
      p, p.idx.grp, p.idx.grp_cnt, p.idx.wmap, p.wmap_words);
  const int nt = p.N / 128;
  vs_tile_lists_kernel<<<dim3((nt + 7) / 8, p.nh, p.B), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t vs_exact_index_launch(const VsIndexParams& p, const minf_vs_exact_index& x, int bits_words,
                                  int twmap_words, cudaStream_t stream) {
  VsIndexParams q = p;  // tile groups only
  q.idx.grp = nullptr;
  q.idx.grp_cnt = nullptr;
  q.idx.tgrp = x.tgrp;
  q.idx.tgrp_cnt = x.tgrp_cnt;
  vs_groups_kernel<<<dim3(q.nh, q.B), 1024, 0, stream>>>(q);
  vs_bits_kernel<<<dim3((bits_words + 255) / 256, q.nh, q.B), 256, 0, stream>>>(q, x.sbits, x.vbits, bits_words);
  vs_wmap_kernel<128><<<dim3((twmap_words + 255) / 256, q.nh, q.B), 256, 0, stream>>>(q, x.tgrp, x.tgrp_cnt,
                                                                                     x.twmap, twmap_words);
  const int nt = q.N / 128;
  vs_vlist_kernel<128><<<dim3((nt + 7) / 8, q.nh, q.B), 256, 0, stream>>>(q, x.twmap, twmap_words, x.vcnt, x.vidx);
  return cudaGetLastError();
}

}  // namespace minf
