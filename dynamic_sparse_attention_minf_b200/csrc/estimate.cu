// Online sparse-index estimation ("MInference 1.0" summary, "Key points",
// second item):
//  * Vertical-Slash: the last query rows are scored against all keys; a
//    softmax over each row gives p_ij, summed per key column (vertical score)
//    and per diagonal offset i - j (slash score).
//  * Block-Sparse: queries and keys are mean-pooled over 64-token blocks and
//    the pooled query of each block is scored against the pooled keys.
//  * Top-k per score row by radix select, ties to the lower index, output
//    ascending.
// All reductions run in a fixed order, so results are bit-reproducible.
#include "minf_device.cuh"
#include "minf_internal.h"

namespace minf {

// ===================================================== Vertical-Slash scores
// Row combine and slash sums of the tensor-core estimation (estimate_tc.cu):
// score tiles of 128 keys, 192 diagonal partials per tile (191 used).
constexpr int kVsKeys = 128;
constexpr int kVsDiag = 192;  // diagonals of a 64 x 128 tile (191 used)

// Combines the per-tile (max, sum) of each row in a fixed order.
__global__ void __launch_bounds__(256) vs_combine_kernel(const VsEstParams p, int ntiles) {
  const int r = blockIdx.x, hi = blockIdx.y, b = blockIdx.z;
  const float* part = p.part_ml + ((size_t)(b * p.nh + hi) * ntiles) * 64 * 2;
  __shared__ float red[256];
  float m = -INFINITY;
  for (int t = threadIdx.x; t < ntiles; t += 256) m = fmaxf(m, part[((size_t)t * 64 + r) * 2]);
  red[threadIdx.x] = m;
  __syncthreads();
  for (int s = 128; s > 0; s >>= 1) {
    if (threadIdx.x < s) red[threadIdx.x] = fmaxf(red[threadIdx.x], red[threadIdx.x + s]);
    __syncthreads();
  }
  const float M = red[0];
  __syncthreads();
  float l = 0.f;
  if (M != -INFINITY) {
    for (int t = threadIdx.x; t < ntiles; t += 256) {
      const float mt = part[((size_t)t * 64 + r) * 2], lt = part[((size_t)t * 64 + r) * 2 + 1];
      if (mt != -INFINITY) l += lt * exp2f(mt - M);
    }
  }
  red[threadIdx.x] = l;
  __syncthreads();
  for (int s = 128; s > 0; s >>= 1) {
    if (threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    float* o = p.row_ml + ((size_t)(b * p.nh + hi) * 64 + r) * 2;
    o[0] = M;
    o[1] = (red[0] > 0.f) ? 1.f / red[0] : 0.f;
  }
}

// sigma_o = sum of the (at most two) tiles' diagonal partials holding offset o.
__global__ void __launch_bounds__(256) vs_slash_kernel(const VsEstParams p, int ntiles) {
  const int o = blockIdx.x * 256 + threadIdx.x;
  const int hi = blockIdx.y, b = blockIdx.z;
  if (o >= p.N) return;
  const size_t bh = (size_t)(b * p.nh + hi);
  const int L = p.last_q;
  // tile t holds offset o at k = o - (N - L - 128 t) + 127 in [0, 190]
  const int base = p.N - L - o;
  int tlo = base - 127;  // 128 t >= base - 127
  tlo = (tlo <= 0) ? 0 : (tlo + 127) / 128;
  const int thi = min(ntiles - 1, (base + 63) >= 0 ? (base + 63) / 128 : -1);
  float s = 0.f;
  for (int t = tlo; t <= thi; ++t) {
    const int k = 128 * t + 127 - base;
    if (k >= 0 && k <= 190) s += p.dpart[(bh * ntiles + t) * kVsDiag + k];
  }
  p.s_score[bh * p.N + o] = s;
}

cudaError_t vs_combine_launch(const VsEstParams& p, int nparts, cudaStream_t stream) {
  vs_combine_kernel<<<dim3(64, p.nh, p.B), 256, 0, stream>>>(p, nparts);
  return cudaGetLastError();
}

cudaError_t vs_slash_launch(const VsEstParams& p, cudaStream_t stream) {
  const int ntiles = (p.N + kVsKeys - 1) / kVsKeys;
  vs_slash_kernel<<<dim3((p.N + 255) / 256, p.nh, p.B), 256, 0, stream>>>(p, ntiles);
  return cudaGetLastError();
}

// ================================================================ top-k rows
constexpr int kTopkThreads = 1024;
constexpr int kTopkItems = 16;
constexpr int kTopkLoads = 16;

__device__ __forceinline__ uint32_t order_key(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inclusive block scan of 64-bit values; returns the inclusive prefix and
// writes the block total.
__device__ __forceinline__ unsigned long long block_scan_u64(unsigned long long v, unsigned long long* wsum,
                                                             unsigned long long& total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xFFFFFFFFu, v, o);
    if (lane >= o) v += y;
  }
  if (lane == 31) wsum[w] = v;
  __syncthreads();
  if (w == 0) {
    unsigned long long s = (lane < (int)(blockDim.x >> 5)) ? wsum[lane] : 0ull;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_up_sync(0xFFFFFFFFu, s, o);
      if (lane >= o) s += y;
    }
    wsum[lane] = s;  // inclusive warp-total prefix
  }
  __syncthreads();
  const unsigned long long before = (w > 0) ? wsum[w - 1] : 0ull;
  total = wsum[(blockDim.x >> 5) - 1];
  __syncthreads();
  return v + before;
}

// The digit of the rem-th largest key from an NB-bin histogram (all threads
// of the block take part): returns the digit and the count of keys in higher
// digits (through shared memory).
__device__ void topk_find_digit(const unsigned* h, int NB, uint32_t rem, unsigned long long* wsum,
                                uint32_t* sh_digit, uint32_t* sh_above) {
  const int per = NB / blockDim.x;  // bins per thread, descending
  uint32_t sum = 0;
  for (int e = 0; e < per; ++e) sum += h[NB - 1 - per * threadIdx.x - e];
  unsigned long long tot;
  const unsigned long long inc = block_scan_u64(sum, wsum, tot);
  const unsigned long long before = inc - sum;
  if (before < rem && inc >= rem) {
    uint32_t cum = (uint32_t)before;
    for (int e = 0; e < per; ++e) {
      const uint32_t c = h[NB - 1 - per * threadIdx.x - e];
      if (cum + c >= rem) {
        *sh_digit = (uint32_t)(NB - 1 - per * threadIdx.x - e);
        *sh_above = cum;
        break;
      }
      cum += c;
    }
  }
  __syncthreads();
}

constexpr int kTopkCap = 1024;  // candidate buffer of the short-row path

template <bool SHORT>
__device__ __forceinline__ void topk_rows_body(const TopkRows& t) {
  const int row = blockIdx.x;
  const int len = (t.len_mode == 0) ? t.len : (row % t.rows_per_group) + 1;
  const int forced = (t.forced_mode == 0) ? -1 : (t.forced_mode == 1) ? 0 : (row % t.rows_per_group);
  const float* sc = t.scores + (long long)row * t.row_stride;
  const int k = min(t.k, len);
  // long rows: one 256-bin histogram per warp (1024 threads); short rows: one
  // 2048-bin histogram (8 KB), so that more rows' CTAs fit on an SM
  __shared__ unsigned hist[SHORT ? 8 : kTopkThreads / 32][256];
  __shared__ unsigned long long wsum[32];
  __shared__ uint32_t sh_sel, sh_rem;
  __shared__ uint32_t ck[kTopkCap];
  __shared__ int32_t ci[kTopkCap];
  auto key_of = [&](int j) -> uint32_t { return (j == forced) ? 0xFFFFFFFFu : order_key(sc[j]); };

  // Short rows: two passes over the row.  (1) a histogram of the top 11 key
  // bits gives the bin of the k-th largest key; (2) every key in that bin or
  // above (fewer than k above, plus the bin) is copied in index order to
  // shared memory.  The threshold is then resolved within those candidates
  // and they are compacted in order.  Rows whose candidates do not fit take
  // the general path below.
  if (SHORT && k > 0) {
    unsigned* h = &hist[0][0];  // 2048 bins
    for (int x = threadIdx.x; x < 2048; x += blockDim.x) h[x] = 0;
    __syncthreads();
    {
      uint32_t last = 2048;
      unsigned run = 0;
      for (int base = 0; base < len; base += blockDim.x * kTopkLoads) {
        uint32_t dg[kTopkLoads];
#pragma unroll
        for (int e = 0; e < kTopkLoads; ++e) {
          const int j = base + e * blockDim.x + threadIdx.x;
          dg[e] = (j < len) ? (key_of(j) >> 21) : 2048u;
        }
#pragma unroll
        for (int e = 0; e < kTopkLoads; ++e) {
          if (dg[e] != last) {
            if (last < 2048) atomicAdd(&h[last], run);
            last = dg[e];
            run = 0;
          }
          ++run;
        }
      }
      if (last < 2048) atomicAdd(&h[last], run);
    }
    __syncthreads();
    topk_find_digit(h, 2048, (uint32_t)k, wsum, &sh_sel, &sh_rem);
    const uint32_t b1 = sh_sel, above = sh_rem;
    const uint32_t M = above + h[b1];
    __syncthreads();
    if (M <= (uint32_t)kTopkCap) {
      // (2) ordered copy of the keys with top bits >= b1
      unsigned long long taken = 0;
      const int chunk = blockDim.x * kTopkItems;
      for (int base = 0; base < len; base += chunk) {
        uint32_t keys[kTopkItems];
        unsigned c = 0;
#pragma unroll
        for (int e = 0; e < kTopkItems; ++e) {
          const int j = base + threadIdx.x * kTopkItems + e;
          keys[e] = (j < len) ? key_of(j) : 0u;
          c += (j < len && (keys[e] >> 21) >= b1);
        }
        unsigned long long tot;
        const unsigned long long inc = block_scan_u64(c, wsum, tot);
        unsigned long long pos = taken + inc - c;
#pragma unroll
        for (int e = 0; e < kTopkItems; ++e) {
          const int j = base + threadIdx.x * kTopkItems + e;
          if (j < len && (keys[e] >> 21) >= b1) {
            ck[pos] = keys[e];
            ci[pos] = j;
            ++pos;
          }
        }
        taken += tot;
      }
      __syncthreads();
      // the exact threshold among the bin's keys: 11 more bits, then 10
      uint32_t prefix = b1 << 21, pmask = 0xFFE00000u, rem = (uint32_t)k - above;
      for (int pass = 0; pass < 2; ++pass) {
        const int shift = pass == 0 ? 10 : 0, nb = pass == 0 ? 2048 : 1024;
        for (int x = threadIdx.x; x < nb; x += blockDim.x) h[x] = 0;
        __syncthreads();
        for (uint32_t x = threadIdx.x; x < M; x += blockDim.x)
          if ((ck[x] & pmask) == prefix) atomicAdd(&h[(ck[x] >> shift) & (nb - 1)], 1u);
        __syncthreads();
        topk_find_digit(h, nb, rem, wsum, &sh_sel, &sh_rem);
        prefix |= sh_sel << shift;
        pmask |= (uint32_t)(nb - 1) << shift;
        rem -= sh_rem;
        __syncthreads();
      }
      const uint32_t T = prefix;
      const uint32_t need = rem;  // keys equal to T that are taken (lowest indices)
      // ordered compaction of the candidates
      int32_t* out = t.out_idx + (long long)row * t.k;
      unsigned long long gt_before = 0, eq_before = 0;
      for (uint32_t base = 0; base < M; base += blockDim.x) {
        const uint32_t x = base + threadIdx.x;
        const uint32_t key = (x < M) ? ck[x] : 0u;
        const unsigned cg = (x < M && key > T), ce = (x < M && key == T);
        unsigned long long tot;
        const unsigned long long inc = block_scan_u64(((unsigned long long)cg << 32) | ce, wsum, tot);
        const unsigned long long exc = inc - (((unsigned long long)cg << 32) | ce);
        const unsigned long long g = gt_before + (exc >> 32), q = eq_before + (exc & 0xFFFFFFFFull);
        if (cg) out[g + min(q, (unsigned long long)need)] = ci[x];
        else if (ce && q < need) out[g + q] = ci[x];
        gt_before += tot >> 32;
        eq_before += tot & 0xFFFFFFFFull;
      }
      for (int x = k + threadIdx.x; x < t.k; x += blockDim.x) out[x] = -1;
      if (t.out_cnt && threadIdx.x == 0) t.out_cnt[row] = k;
      return;
    }
  }

  // radix select of the k-th largest key, 8 bits at a time from the top
  uint32_t prefix = 0, pmask = 0, rem = (uint32_t)k;
  for (int shift = 24; shift >= 0 && k > 0; shift -= 8) {
    // long rows: one histogram per warp; short rows: one for the block
    const int nh = (blockDim.x >= 1024) ? (blockDim.x >> 5) : 1;
    unsigned* my_hist = hist[(blockDim.x >= 1024) ? (threadIdx.x >> 5) : 0];
    for (int x = threadIdx.x; x < nh * 256; x += blockDim.x) hist[x >> 8][x & 255] = 0;
    __syncthreads();
    // each thread counts runs of equal digits in registers and adds a run
    // when its digit changes
    uint32_t last = 256;
    unsigned run = 0;
    // kTopkLoads independent coalesced loads per thread in flight per step
    for (int base = 0; base < len; base += blockDim.x * kTopkLoads) {
      uint32_t digit[kTopkLoads];
#pragma unroll
      for (int e = 0; e < kTopkLoads; ++e) {
        const int j = base + e * blockDim.x + threadIdx.x;
        digit[e] = 256;
        if (j < len) {
          const uint32_t key = key_of(j);
          if ((key & pmask) == prefix) digit[e] = (key >> shift) & 255u;
        }
      }
#pragma unroll
      for (int e = 0; e < kTopkLoads; ++e) {
        if (digit[e] != last) {
          if (last < 256) atomicAdd(&my_hist[last], run);
          last = digit[e];
          run = 0;
        }
        ++run;
      }
    }
    if (last < 256) atomicAdd(&my_hist[last], run);
    __syncthreads();
    // sum the warps' histograms into the first, in a fixed order
    for (int x = threadIdx.x; x < 256 && nh > 1; x += blockDim.x) {
      unsigned c = hist[0][x];
      for (int w = 1; w < nh; ++w) c += hist[w][x];
      hist[0][x] = c;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // the digit holding the rem-th largest key: lane l owns digits
      // 255 - 8l down to 248 - 8l; a scan over lanes finds the crossing
      const int lane = threadIdx.x;
      uint32_t h[8], sum = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        h[e] = hist[0][255 - 8 * lane - e];
        sum += h[e];
      }
      uint32_t inc = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, inc, o);
        if (lane >= o) inc += y;
      }
      const unsigned ball = __ballot_sync(0xFFFFFFFFu, inc >= rem);
      const int owner = ball ? __ffs(ball) - 1 : 0;
      if (lane == owner) {
        uint32_t cum = inc - sum, sel = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (cum + h[e] >= rem) {
            sel = (uint32_t)(255 - 8 * lane - e);
            break;
          }
          cum += h[e];
        }
        sh_sel = sel;
        sh_rem = rem - cum;
      }
    }
    __syncthreads();
    prefix |= sh_sel << shift;
    pmask |= 255u << shift;
    rem = sh_rem;
    __syncthreads();
  }
  const uint32_t T = prefix;
  const unsigned long long need = rem;  // how many keys equal to T are taken (lowest indices)
  int32_t* out = t.out_idx + (long long)row * t.k;
  // ordered compaction: element j is taken when key > T, or key == T and
  // fewer than `need` equal keys precede it
  unsigned long long gt_before = 0, eq_before = 0;
  const int chunk = blockDim.x * kTopkItems;
  for (int base = 0; base < len && k > 0; base += chunk) {
    uint32_t keys[kTopkItems];
    unsigned cgt = 0, ceq = 0;
#pragma unroll
    for (int e = 0; e < kTopkItems; ++e) {
      const int j = base + threadIdx.x * kTopkItems + e;
      keys[e] = (j < len) ? key_of(j) : 0u;
      const bool valid = j < len;
      cgt += (valid && keys[e] > T);
      ceq += (valid && keys[e] == T);
    }
    unsigned long long tot;
    const unsigned long long inc = block_scan_u64(((unsigned long long)cgt << 32) | ceq, wsum, tot);
    const unsigned long long exc = inc - (((unsigned long long)cgt << 32) | ceq);
    unsigned long long g = gt_before + (exc >> 32), q = eq_before + (exc & 0xFFFFFFFFull);
#pragma unroll
    for (int e = 0; e < kTopkItems; ++e) {
      const int j = base + threadIdx.x * kTopkItems + e;
      if (j < len) {
        if (keys[e] > T) {
          out[g + min(q, need)] = j;
          ++g;
        } else if (keys[e] == T) {
          if (q < need) out[g + q] = j;
          ++q;
        }
      }
    }
    gt_before += tot >> 32;
    eq_before += tot & 0xFFFFFFFFull;
  }
  for (int x = k + threadIdx.x; x < t.k; x += blockDim.x) out[x] = -1;
  if (t.out_cnt && threadIdx.x == 0) t.out_cnt[row] = k;
}

// One CTA per row: 1024 threads for rows too long for the short-row path
// (only when no scratch is given), 256 for the rest.
__global__ void __launch_bounds__(kTopkThreads, 1) topk_rows_kernel(const TopkRows t) { topk_rows_body<false>(t); }
__global__ void __launch_bounds__(256, 4) topk_short_rows_kernel(const TopkRows t) { topk_rows_body<true>(t); }

// ---------------------------------------------- top-k of long rows, many CTAs
// The same selection as topk_rows_kernel, for rows too long for one CTA: the
// threshold key T is found by three radix passes (11, 11 and 10 bits) whose
// histograms are gathered from (segment, row) CTAs into a per-row histogram
// and resolved by one CTA per row; then every segment counts its keys above
// and equal to T, and writes its selected indices at the offset given by the
// counts of the segments before it (ascending order, lowest-index ties).
// Per-row scratch: [0, 2048) histogram, [2048, 2051) prefix / mask / rem,
// [2056, 2056 + 2 * 1024) per-segment (above, equal) counts.
constexpr int kMsState = 2048;
constexpr int kMsCounts = 2056;
constexpr int kMsThreads = 512;

struct TopkRowView {
  const float* sc;
  int len, forced, k;
  __device__ TopkRowView(const TopkRows& t, int row) {
    sc = t.scores + (long long)row * t.row_stride;
    len = t.len;
    forced = (t.forced_mode == 1) ? 0 : -1;
    k = min(t.k, len);
  }
  __device__ uint32_t key(int j) const { return (j == forced) ? 0xFFFFFFFFu : order_key(sc[j]); }
};

__global__ void __launch_bounds__(256) topk_ms_init_kernel(const TopkRows t) {
  uint32_t* ws = t.scratch + (size_t)blockIdx.x * kTopkScratchWords;
  for (int x = threadIdx.x; x < kMsState; x += blockDim.x) ws[x] = 0;
  if (threadIdx.x == 0) {
    ws[kMsState] = 0;
    ws[kMsState + 1] = 0;
    ws[kMsState + 2] = (uint32_t)min(t.k, t.len);
  }
}

template <int SHIFT, int BITS>
__global__ void __launch_bounds__(kMsThreads) topk_ms_hist_kernel(const TopkRows t, int seg) {
  constexpr int NB = 1 << BITS;
  __shared__ unsigned h[NB];
  const int row = blockIdx.y;
  const TopkRowView r(t, row);
  uint32_t* ws = t.scratch + (size_t)row * kTopkScratchWords;
  const uint32_t prefix = ws[kMsState], pmask = ws[kMsState + 1];
  for (int x = threadIdx.x; x < NB; x += blockDim.x) h[x] = 0;
  __syncthreads();
  const int j0 = blockIdx.x * seg, j1 = min(r.len, j0 + seg);
  for (int base = j0; base < j1; base += blockDim.x * kTopkLoads) {
    uint32_t kk[kTopkLoads];
#pragma unroll
    for (int e = 0; e < kTopkLoads; ++e) {
      const int j = base + e * blockDim.x + threadIdx.x;
      kk[e] = (j < j1) ? r.key(j) : 0u;
    }
#pragma unroll
    for (int e = 0; e < kTopkLoads; ++e) {
      const int j = base + e * blockDim.x + threadIdx.x;
      if (j < j1 && (kk[e] & pmask) == prefix) atomicAdd(&h[(kk[e] >> SHIFT) & (NB - 1)], 1u);
    }
  }
  __syncthreads();
  for (int x = threadIdx.x; x < NB; x += blockDim.x)
    if (h[x]) atomicAdd(&ws[x], h[x]);
}

// Resolves one pass: the digit holding the rem-th largest remaining key, and
// clears the histogram for the next pass.
template <int SHIFT, int BITS>
__global__ void __launch_bounds__(1024) topk_ms_select_kernel(const TopkRows t) {
  constexpr int NB = 1 << BITS;
  constexpr int PER = NB / 1024;  // bins per thread, descending
  __shared__ unsigned long long wsum[32];
  uint32_t* ws = t.scratch + (size_t)blockIdx.x * kTopkScratchWords;
  const uint32_t rem = ws[kMsState + 2];
  uint32_t c[PER], sum = 0;
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    c[e] = ws[NB - 1 - PER * threadIdx.x - e];
    sum += c[e];
  }
  unsigned long long tot;
  const unsigned long long inc = block_scan_u64(sum, wsum, tot);
  const unsigned long long before = inc - sum;
  if (before < rem && inc >= rem) {
    uint32_t cum = (uint32_t)before, d = 0;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      if (cum + c[e] >= rem) {
        d = (uint32_t)(NB - 1 - PER * threadIdx.x - e);
        break;
      }
      cum += c[e];
    }
    ws[kMsState] |= d << SHIFT;
    ws[kMsState + 1] |= (uint32_t)(NB - 1) << SHIFT;
    ws[kMsState + 2] = rem - cum;
  }
  __syncthreads();
  for (int x = threadIdx.x; x < NB; x += blockDim.x) ws[x] = 0;
}

// Keys above and equal to the threshold, per segment.
__global__ void __launch_bounds__(kMsThreads) topk_ms_count_kernel(const TopkRows t, int seg) {
  __shared__ unsigned long long wsum[32];
  const int row = blockIdx.y;
  const TopkRowView r(t, row);
  uint32_t* ws = t.scratch + (size_t)row * kTopkScratchWords;
  const uint32_t T = ws[kMsState];
  const int j0 = blockIdx.x * seg, j1 = min(r.len, j0 + seg);
  unsigned gt = 0, eq = 0;
  for (int base = j0; base < j1; base += blockDim.x * kTopkLoads) {
#pragma unroll
    for (int e = 0; e < kTopkLoads; ++e) {
      const int j = base + e * blockDim.x + threadIdx.x;
      if (j < j1) {
        const uint32_t kk = r.key(j);
        gt += kk > T;
        eq += kk == T;
      }
    }
  }
  unsigned long long tot;
  block_scan_u64(((unsigned long long)gt << 32) | eq, wsum, tot);
  if (threadIdx.x == 0) {
    ws[kMsCounts + 2 * blockIdx.x] = (uint32_t)(tot >> 32);
    ws[kMsCounts + 2 * blockIdx.x + 1] = (uint32_t)tot;
  }
}

// Writes each segment's selected indices after those of the segments before it.
__global__ void __launch_bounds__(kMsThreads) topk_ms_write_kernel(const TopkRows t, int seg) {
  __shared__ unsigned long long wsum[32];
  const int row = blockIdx.y, sgi = blockIdx.x;
  const TopkRowView r(t, row);
  const uint32_t* ws = t.scratch + (size_t)row * kTopkScratchWords;
  const uint32_t T = ws[kMsState];
  const unsigned long long need = ws[kMsState + 2];
  unsigned long long pre = 0;
  for (int s2 = threadIdx.x; s2 < sgi; s2 += blockDim.x)
    pre += ((unsigned long long)ws[kMsCounts + 2 * s2] << 32) | ws[kMsCounts + 2 * s2 + 1];
  unsigned long long tot;
  block_scan_u64(pre, wsum, tot);
  unsigned long long gt_before = tot >> 32, eq_before = tot & 0xFFFFFFFFull;
  int32_t* out = t.out_idx + (long long)row * t.k;
  const int j0 = sgi * seg, j1 = min(r.len, j0 + seg);
  const int chunk = blockDim.x * kTopkItems;
  for (int base = j0; base < j1; base += chunk) {
    uint32_t keys[kTopkItems];
    unsigned cgt = 0, ceq = 0;
#pragma unroll
    for (int e = 0; e < kTopkItems; ++e) {
      const int j = base + threadIdx.x * kTopkItems + e;
      const bool valid = j < j1;
      keys[e] = valid ? r.key(j) : 0u;
      cgt += (valid && keys[e] > T);
      ceq += (valid && keys[e] == T);
    }
    unsigned long long ctot;
    const unsigned long long inc = block_scan_u64(((unsigned long long)cgt << 32) | ceq, wsum, ctot);
    const unsigned long long exc = inc - (((unsigned long long)cgt << 32) | ceq);
    unsigned long long g = gt_before + (exc >> 32), q = eq_before + (exc & 0xFFFFFFFFull);
#pragma unroll
    for (int e = 0; e < kTopkItems; ++e) {
      const int j = base + threadIdx.x * kTopkItems + e;
      if (j < j1) {
        if (keys[e] > T) {
          out[g + min(q, need)] = j;
          ++g;
        } else if (keys[e] == T) {
          if (q < need) out[g + q] = j;
          ++q;
        }
      }
    }
    gt_before += ctot >> 32;
    eq_before += ctot & 0xFFFFFFFFull;
  }
  if (sgi == 0) {
    for (int x = r.k + threadIdx.x; x < t.k; x += blockDim.x) out[x] = -1;
    if (t.out_cnt && threadIdx.x == 0) t.out_cnt[row] = r.k;
  }
}

static cudaError_t topk_long_rows_launch(const TopkRows& t, cudaStream_t stream) {
  const int seg = max(16384, (t.len + 1023) / 1024);
  const int nseg = (t.len + seg - 1) / seg;
  const dim3 g2(nseg, t.rows);
  topk_ms_init_kernel<<<t.rows, 256, 0, stream>>>(t);
  topk_ms_hist_kernel<21, 11><<<g2, kMsThreads, 0, stream>>>(t, seg);
  topk_ms_select_kernel<21, 11><<<t.rows, 1024, 0, stream>>>(t);
  topk_ms_hist_kernel<10, 11><<<g2, kMsThreads, 0, stream>>>(t, seg);
  topk_ms_select_kernel<10, 11><<<t.rows, 1024, 0, stream>>>(t);
  topk_ms_hist_kernel<0, 10><<<g2, kMsThreads, 0, stream>>>(t, seg);
  topk_ms_select_kernel<0, 10><<<t.rows, 1024, 0, stream>>>(t);
  topk_ms_count_kernel<<<g2, kMsThreads, 0, stream>>>(t, seg);
  topk_ms_write_kernel<<<g2, kMsThreads, 0, stream>>>(t, seg);
  return cudaGetLastError();
}

cudaError_t topk_rows_launch(const TopkRows& t, cudaStream_t stream) {
  if (t.rows <= 0) return cudaSuccess;
  if (t.len_mode == 0 && t.len > kTopkLongRow && t.scratch && t.forced_mode != 2)
    return topk_long_rows_launch(t, stream);
  // long rows (Vertical-Slash: one per head) take a whole SM each; short
  // rows (Block-Sparse: one per query block) run several CTAs per SM
  if (t.len > 32768)
    topk_rows_kernel<<<t.rows, kTopkThreads, 0, stream>>>(t);
  else
    topk_short_rows_kernel<<<t.rows, 256, 0, stream>>>(t);
  return cudaGetLastError();
}

// ====================================================== Block-Sparse scores
// Mean of every 64-row block of Q (listed heads) and K (their KV heads), fp32.
// One CTA of 256 threads per (64-row block, head slot): threads 0-127 pool Q,
// 128-255 K.  Within a matrix a thread sums 8 adjacent columns (16-byte
// loads) over every (128 / (d / 8))-th row of the block; the row phases are
// then added in a fixed order, one thread per column.
__global__ void __launch_bounds__(256) bs_pool_kernel(const BsEstParams p) {
  __shared__ float red[2][16][128];  // [matrix][row phase][column]
  const int qb = blockIdx.x, hi = blockIdx.y, b = blockIdx.z;
  const int head = p.heads[hi];
  if (head < 0 || head >= p.Hq) {
    if (threadIdx.x == 0) report(p.status, MINF_ERR_DEVICE_BOUNDS, 40);
    return;
  }
  const int nb = p.N / 64;
  const int kvh = head / p.group;
  const int nc = p.d / 8;     // 16-byte column groups of a row
  const int per = 128 / nc;   // row phases
  {
    const int isk = threadIdx.x >> 7, t = threadIdx.x & 127;
    const int cg = t % nc, rp = t / nc;
    const __nv_bfloat16* src = isk ? p.K + ((size_t)(b * p.Hkv + kvh) * p.N + qb * 64) * p.d
                                   : p.Q + ((size_t)(b * p.Hq + head) * p.N + qb * 64) * p.d;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int r = rp; r < 64; r += per) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + (size_t)r * p.d + 8 * cg));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * e] += __uint_as_float(w[e] << 16);
        acc[2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red[isk][rp][8 * cg + e] = acc[e];
  }
  __syncthreads();
  if (threadIdx.x >= 2 * p.d) return;
  const int isk = threadIdx.x / p.d, dd = threadIdx.x % p.d;
  float s = 0.f;
  for (int rp = 0; rp < per; ++rp) s += red[isk][rp][dd];
  const size_t at = (((size_t)(b * p.nh + hi) * nb) + qb) * p.d + dd;
  const float m = s * (1.0f / 64.0f);
  (isk ? p.kbar : p.qbar)[at] = m;
  __nv_bfloat16* parts = isk ? p.ks : p.qs;
  if (parts) {
    // m = x0 + x1 + x2 up to 2^-24 relative: each part is the bf16 rounding
    // of what the earlier parts leave, and every difference is exact in fp32
    const size_t stride = (size_t)p.B * p.nh * nb * p.d;
    const __nv_bfloat16 x0 = __float2bfloat16_rn(m);
    const float r1 = m - __bfloat162float(x0);
    const __nv_bfloat16 x1 = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(x1);
    parts[at] = x0;
    parts[stride + at] = x1;
    parts[2 * stride + at] = __float2bfloat16_rn(r2);
  }
}

// t[b, c] = scale * qbar_b . kbar_c over 64 x 64 tiles with c-tile <= b-tile.
__global__ void __launch_bounds__(256) bs_score_kernel(const BsEstParams p) {
  const int ct = blockIdx.x, bt = blockIdx.y, bhz = blockIdx.z;
  if (ct > bt) return;
  const int nb = p.N / 64;
  const float* qb = p.qbar + (size_t)bhz * nb * p.d;
  const float* kb = p.kbar + (size_t)bhz * nb * p.d;
  __shared__ float As[32][64 + 4];
  __shared__ float Bs[32][64 + 4];
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < p.d; k0 += 32) {
    for (int e = tid; e < 64 * 32; e += 256) {
      const int r = e / 32, kk = e % 32;
      const int gr = bt * 64 + r, gc = ct * 64 + r;
      As[kk][r] = (gr < nb) ? qb[(size_t)gr * p.d + k0 + kk] : 0.f;
      Bs[kk][r] = (gc < nb) ? kb[(size_t)gc * p.d + k0 + kk] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < 32; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
      const float4 bb = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float bv[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
  float* out = p.scores + (size_t)bhz * nb * nb;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = bt * 64 + ty * 4 + i;
    if (r >= nb) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = ct * 64 + tx * 4 + j;
      if (c < nb) out[(size_t)r * nb + c] = acc[i][j] * p.scale;
    }
  }
}

// t[b, c] = scale * qbar_b . kbar_c over 128 x 128 tiles of the lower
// triangle (c-tile <= b-tile), one CTA per tile: 256 threads with 8 x 8
// outputs each, packed two-lane fp32 FMAs, k in chunks of 16 staged
// transposed in shared memory.
constexpr int kBsT = 128, kBsK = 16, kBsPad = 4;
__global__ void __launch_bounds__(256) bs_score_tri_kernel(const BsEstParams p, int nt) {
  // lower-triangle tile x -> (bt, ct), ct <= bt
  const int x = blockIdx.x;
  int bt = (int)((sqrtf(8.f * (float)x + 1.f) - 1.f) * 0.5f);
  while ((bt + 1) * (bt + 2) / 2 <= x) ++bt;
  while (bt * (bt + 1) / 2 > x) --bt;
  const int ct = x - bt * (bt + 1) / 2;
  const int bhz = blockIdx.y;
  const int nb = p.N / 64;
  const float* qb = p.qbar + (size_t)bhz * nb * p.d;
  const float* kb = p.kbar + (size_t)bhz * nb * p.d;
  __shared__ __align__(16) float As[kBsK][kBsT + kBsPad];
  __shared__ __align__(16) float Bs[kBsK][kBsT + kBsPad];
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  uint64_t acc[8][4];  // row ty*8+i, columns tx*8 + 2j, 2j+1
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0ull;
  for (int k0 = 0; k0 < p.d; k0 += kBsK) {
    // 128 rows x 16 k of each operand: 512 float4 per operand, 2 per thread
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int f = tid + 256 * u;
      const int r = f >> 2, kq = f & 3;
      const int gr = bt * kBsT + r, gc = ct * kBsT + r;
      const float4 av = (gr < nb) ? *reinterpret_cast<const float4*>(qb + (size_t)gr * p.d + k0 + 4 * kq)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 bv = (gc < nb) ? *reinterpret_cast<const float4*>(kb + (size_t)gc * p.d + k0 + 4 * kq)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
      As[4 * kq + 0][r] = av.x; As[4 * kq + 1][r] = av.y; As[4 * kq + 2][r] = av.z; As[4 * kq + 3][r] = av.w;
      Bs[4 * kq + 0][r] = bv.x; Bs[4 * kq + 1][r] = bv.y; Bs[4 * kq + 2][r] = bv.z; Bs[4 * kq + 3][r] = bv.w;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kBsK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[kk][ty * 8]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[kk][ty * 8 + 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[kk][tx * 8]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[kk][tx * 8 + 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const uint64_t bp[4] = {f32x2_pack(b0.x, b0.y), f32x2_pack(b0.z, b0.w), f32x2_pack(b1.x, b1.y),
                              f32x2_pack(b1.z, b1.w)};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint64_t a2 = f32x2_pack(av[i], av[i]);
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = f32x2_fma(a2, bp[j], acc[i][j]);
      }
    }
    __syncthreads();
  }
  float* out = p.scores + (size_t)bhz * nb * nb;
  const int c0 = ct * kBsT + tx * 8;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = bt * kBsT + ty * 8 + i;
    if (r >= nb) continue;
    float v[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      f32x2_unpack(acc[i][j], v[2 * j], v[2 * j + 1]);
      v[2 * j] *= p.scale;
      v[2 * j + 1] *= p.scale;
    }
    if (c0 + 8 <= nb) {
      float4* dst = reinterpret_cast<float4*>(out + (size_t)r * nb + c0);
      dst[0] = make_float4(v[0], v[1], v[2], v[3]);
      dst[1] = make_float4(v[4], v[5], v[6], v[7]);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (c0 + j < nb) out[(size_t)r * nb + c0 + j] = v[j];
    }
  }
}

cudaError_t bs_pool_score_launch(const BsEstParams& p, cudaStream_t stream) {
  const int nb = p.N / 64;
  bs_pool_kernel<<<dim3(nb, p.nh, p.B), 256, 0, stream>>>(p);
  if (!p.scores) return cudaGetLastError();
  if (nb % 8 == 0 && p.d % kBsK == 0) {
    const int nt = (nb + kBsT - 1) / kBsT;
    bs_score_tri_kernel<<<dim3(nt * (nt + 1) / 2, p.B * p.nh), 256, 0, stream>>>(p, nt);
  } else {
    const int nt = (nb + 63) / 64;
    bs_score_kernel<<<dim3(nt, nt, p.B * p.nh), 256, 0, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace minf
