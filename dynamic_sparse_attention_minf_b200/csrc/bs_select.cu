// Block-Sparse index estimation on the tensor cores ("MInference 1.0"
// summary, "Key points": Block-Sparse heads mean-pool queries and keys in
// 64-token blocks; each query block keeps its k best key blocks).
//
// Two kernels:
//
// bs_score_tc_kernel: t[b, c] = scale * qbar_b . kbar_c for key blocks
// c <= b, into the row-major [nb, nb] matrix of each head.  The fp32 means
// arrive split into three bf16 parts each (x = x0 + x1 + x2 up to 2^-24
// relative), and the tensor cores form
//     q0 k0 + q0 k1 + q1 k0 + q0 k2 + q1 k1 + q2 k0
// in fp32: the score to about fp32 accuracy (the dropped terms are below
// 2^-24 of |qbar| |kbar|), six bf16 MMAs per K step.  One CTA per (batch,
// head, 128 query blocks), heaviest row tiles first:
//   warps 0-3  epilogue: thread = query block; the 128 x 128 score tile from
//              TMEM, scaled, through two 32-column staging boxes in shared
//              memory to the row-major score matrix by TMA stores (columns
//              past the diagonal are written too: the matrix leaves them
//              undefined)
//   warp 4     tcgen05 issuer and TMEM owner: A = the query parts, resident in
//              TMEM (written once by the epilogue warps); B = the key parts
//              from shared memory; D = two 128 x 128 fp32 score buffers
//   warp 5     producer: TMA loads of the key parts, one 64-column half of d
//              (three parts, 48 KB) per ring slot
//
// bs_topk_warp_kernel: one warp per query block, many warps per SM.  The row
// is read from the diagonal down, 128 columns at a time; columns whose key
// reaches the row's threshold go to a shared-memory list, which a warp-wide
// binary search on the order-preserving keys compacts to the k best (ties to
// the lowest column) when the next chunk could overflow it; that sets the
// threshold.  Scores that grow toward the diagonal (a local bias) raise the
// threshold early this way.
//
// Every wait is bounded and records MINF_ERR_DEVICE_TIMEOUT when it runs out.
#include "minf_device.cuh"
#include "minf_internal.h"

namespace minf {

namespace {

constexpr int kSelThreads = 192;
constexpr int kStages = 4;              // ring slots (64-column halves of d)
constexpr int kPartBytes = 128 * 128;   // 128 key blocks x 64 d (bf16)
constexpr int kStageBytes = 3 * kPartBytes;
constexpr int kOffB = 0;
constexpr int kStageOut = 128 * 128;    // 128 rows x 32 fp32 columns
constexpr int kOffOut = kOffB + kStages * kStageBytes;
constexpr int kOffBars = kOffOut + 2 * kStageOut;
// barriers: b_full[kStages], b_empty[kStages], d_full[2], d_empty[2], a_full, done
constexpr int kNumBars = 2 * kStages + 6;
constexpr int kOffMisc = kOffBars + kNumBars * 8;
constexpr int kSmem = kOffMisc + 16;
static_assert(kSmem <= 232448, "shared memory budget");

// TMEM columns: D buffers at 0 and 128, the query parts at 256 + 64 p
constexpr uint32_t kColA = 256;
constexpr uint32_t kIdesc = idesc_bf16(128, 128, 0, 0);

struct ScoreParams {
  const __nv_bfloat16* qs;
  float* scores;  // [bh_total, nb, nb]
  float scale;
  int nb, nrt, bh_total;
  DevStatus* status;
};

__device__ __forceinline__ uint32_t sel_order_key(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ bool sel_wait(uint64_t* bar, uint32_t parity, volatile int* abort, DevStatus* st,
                                         int where) {
  const bool ok = mbar_wait(bar, parity, abort, st, where);
  return __all_sync(0xFFFFFFFFu, ok);
}

__device__ __forceinline__ bool sel_elect() {
  uint32_t e;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(e));
  return e != 0;
}

// the six products of the split: (query part, key part)
__constant__ int kPa[6] = {0, 0, 1, 0, 1, 2};
__constant__ int kPb[6] = {0, 1, 0, 2, 1, 0};

__global__ void __launch_bounds__(kSelThreads, 1)
    bs_score_tc_kernel(const __grid_constant__ CUtensorMap tmKs, const __grid_constant__ CUtensorMap tmS,
                       const ScoreParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rt = p.nrt - 1 - (int)blockIdx.x;  // heaviest row tiles first
  const int bh = blockIdx.y;                    // batch * nh + head slot
  const int ntiles = rt + 1;                    // key tiles 0 .. rt (causal)
  const int nchunks = 2 * ntiles;               // (key tile, half of d)

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBars);
  uint64_t* b_full = bars;              // a ring slot's three key parts have landed
  uint64_t* b_empty = bars + kStages;   // the MMAs that read a ring slot are done
  uint64_t* d_full = bars + 2 * kStages;  // a score buffer is complete
  uint64_t* d_empty = d_full + 2;       // the epilogue warps have read a score buffer
  uint64_t* a_full = d_empty + 2;       // the query parts are in TMEM
  uint64_t* done = a_full + 1;          // every MMA issued has completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  if ((smem_u32(smem) & 1023u) != 0u) {
    if (threadIdx.x == 0) report(p.status, MINF_ERR_DEVICE_BOUNDS, 60);
    return;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&d_full[s], 1);
      mbar_init(&d_empty[s], 128);
    }
    mbar_init(a_full, 4);
    mbar_init(done, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 5) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tmKs);
      prefetch_tmap(&tmS);
      int issued = 0;
      for (int u = 0; u < nchunks; ++u) {
        const int s = u % kStages;
        if (u >= kStages && !mbar_wait(&b_empty[s], ((u / kStages) - 1) & 1, abort, p.status, 61)) break;
        mbar_arrive_expect_tx(&b_full[s], kStageBytes);
        uint8_t* dst = smem + kOffB + s * kStageBytes;
        const int j = u >> 1, h = u & 1;
#pragma unroll
        for (int pb = 0; pb < 3; ++pb)
          tma_load_3d(dst + pb * kPartBytes, &tmKs, &b_full[s], 64 * h, 128 * j, pb * p.bh_total + bh);
        ++issued;
      }
      // no copy may be in flight when the CTA exits: wait (bounded, ignoring
      // the abort flag) for the last load of each slot
      int dummy = 0;
      for (int u = max(0, issued - kStages); u < issued; ++u)
        mbar_wait(&b_full[u % kStages], (u / kStages) & 1, &dummy, p.status, 62);
    }
    __syncwarp();
  } else if (warp == 4) {
    // ---------------------------------------------------------- MMA issuer
    bool ok = sel_wait(a_full, 0, abort, p.status, 63);
    tc_fence_after();
    for (int j = 0; j < ntiles && ok; ++j) {
      const int db = j & 1;
      if (j >= 2) {
        if (!sel_wait(&d_empty[db], ((j >> 1) - 1) & 1, abort, p.status, 64)) { ok = false; break; }
        tc_fence_after();
      }
      for (int h = 0; h < 2; ++h) {
        const int u = 2 * j + h, s = u % kStages;
        if (!sel_wait(&b_full[s], (u / kStages) & 1, abort, p.status, 65)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sbase = smem_u32(smem + kOffB + s * kStageBytes);
        if (sel_elect()) {
#pragma unroll
          for (int pr = 0; pr < 6; ++pr) {
            const uint64_t bd = sdesc_sw128(sbase + kPb[pr] * kPartBytes, 16, 1024);
            const uint32_t ad = tmem + kColA + 64 * kPa[pr] + 32 * h;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_ts(tmem + 128 * db, ad + 8 * kk, bd + (uint64_t)(2 * kk), kIdesc,
                      (h == 0 && pr == 0 && kk == 0) ? 0u : 1u);
          }
          umma_commit(&b_empty[s]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (sel_elect()) umma_commit(&d_full[db]);
      __syncwarp();
    }
    if (sel_elect()) umma_commit(done);
    __syncwarp();
    if (lane == 0) {
      int dummy = 0;
      mbar_wait(done, 0, &dummy, p.status, 66);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ epilogue warps
    const int r = warp * 32 + lane;  // TMEM lane and row of the tile
    const int b = rt * 128 + r;      // this thread's query block
    const bool vrow = b < p.nb;
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    // A: the row's three query parts, bf16 pairs in consecutive TMEM columns
    {
      const size_t pstride = (size_t)p.bh_total * p.nb * 128;
      const __nv_bfloat16* q = p.qs + ((size_t)bh * p.nb + (vrow ? b : 0)) * 128;
#pragma unroll 1
      for (int pa = 0; pa < 3; ++pa) {
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          uint32_t w[32];
          const uint4* src = reinterpret_cast<const uint4*>(q + pa * pstride + half * 64);
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const uint4 x = vrow ? __ldg(src + v) : make_uint4(0u, 0u, 0u, 0u);
            w[4 * v] = x.x;
            w[4 * v + 1] = x.y;
            w[4 * v + 2] = x.z;
            w[4 * v + 3] = x.w;
          }
          tmem_st32(tl + kColA + 64 * pa + 32 * half, w);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(a_full);
    }
    // Every chunk: TMEM to registers, wait until the staging box it takes was
    // read by the store two chunks back, write the scaled row 128B-swizzled,
    // and one thread stores the box.  The break on a failed wait is agreed by
    // all 128 threads, since the named barriers below need every one of them.
    for (int j = 0; j < ntiles; ++j) {
      const int db = j & 1;
      const bool okw = sel_wait(&d_full[db], (j >> 1) & 1, abort, p.status, 67);
      if (!bar_and(2, 128, okw)) break;
      tc_fence_after();
#pragma unroll 1
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t sr[32];
        tmem_ld32(tl + 128 * db + 32 * q4, sr);
        tmem_wait_ld();
        reg_fence(sr);
        const int sb = q4 & 1;
        if (threadIdx.x == 0) bulk_wait_read<1>();
        named_bar_sync(1, 128);
        uint8_t* stg = smem + kOffOut + sb * kStageOut + r * 128;
#pragma unroll
        for (int qq = 0; qq < 8; ++qq)
          *reinterpret_cast<float4*>(stg + ((qq ^ (r & 7)) << 4)) =
              make_float4(__uint_as_float(sr[4 * qq]) * p.scale, __uint_as_float(sr[4 * qq + 1]) * p.scale,
                          __uint_as_float(sr[4 * qq + 2]) * p.scale, __uint_as_float(sr[4 * qq + 3]) * p.scale);
        fence_proxy_async();
        named_bar_sync(1, 128);
        if (threadIdx.x == 0) {
          tma_store_3d(&tmS, smem + kOffOut + sb * kStageOut, 128 * j + 32 * q4, 128 * rt, bh);
          bulk_commit();
        }
      }
      tc_fence_before();
      mbar_arrive(&d_empty[db]);
    }
    if (threadIdx.x == 0) bulk_wait_all<0>();  // every store has landed before the CTA exits
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

constexpr int kTkWarps = 8;
constexpr int kTkChunk = 128;           // columns a warp takes at a time (4 per lane)
constexpr int kTkCap = 256;             // list entries per warp
constexpr int kTkPer = kTkCap / 32;     // list entries per lane in a compaction

// Keeps, in list order, the k best of the n > k entries of a warp's list
// (largest key first; among equal keys the later entries, whose columns are
// lower: the list runs in descending column order) and returns the k-th best
// key.  The warp finds that key bit by bit: the largest T with at least k
// keys >= T, searching only the bits below the common prefix of the smallest
// listed key and the largest one other than the forced diagonal's.
__device__ uint32_t tk_compact(uint32_t* keys, int32_t* cols, int n, int k, int lane) {
  uint32_t kv[kTkPer];
  int32_t cv[kTkPer];
#pragma unroll
  for (int i = 0; i < kTkPer; ++i) {
    const int x = 32 * i + lane;
    kv[i] = (x < n) ? keys[x] : 0u;  // key 0 (below every listed key) marks no entry
    cv[i] = (x < n) ? cols[x] : 0;
  }
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
#pragma unroll
  for (int i = 0; i < kTkPer; ++i) {
    if (kv[i] != 0u) lo = min(lo, kv[i]);
    if (kv[i] != 0xFFFFFFFFu) hi = max(hi, kv[i]);
  }
  lo = __reduce_min_sync(0xFFFFFFFFu, lo);
  hi = __reduce_max_sync(0xFFFFFFFFu, hi);
  uint32_t T;
  if (k == 1 || hi == 0u) {
    T = 0xFFFFFFFFu;  // only the forced diagonal stays
  } else {
    // lo <= T <= hi: T shares their common high bits
    const uint32_t dif = lo ^ hi;
    const int top = dif ? 31 - __clz(dif) : -1;
    T = (top < 0) ? lo : (hi & ~((top == 31) ? 0xFFFFFFFFu : ((2u << top) - 1u)));
    for (int bit = top; bit >= 0; --bit) {
      const uint32_t trial = T | (1u << bit);
      uint32_t c = 0;
#pragma unroll
      for (int i = 0; i < kTkPer; ++i) c += (kv[i] >= trial);
      if (__reduce_add_sync(0xFFFFFFFFu, c) >= (uint32_t)k) T = trial;
    }
  }
  uint32_t g = 0, e = 0;
#pragma unroll
  for (int i = 0; i < kTkPer; ++i) {
    g += (kv[i] > T);
    e += (kv[i] == T);
  }
  const uint32_t n_gt = __reduce_add_sync(0xFFFFFFFFu, g), n_eq = __reduce_add_sync(0xFFFFFFFFu, e);
  const uint32_t need = (uint32_t)k - n_gt;  // entries equal to T that stay: the last `need`
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t wpos = 0, eq_seen = 0;
  __syncwarp();
#pragma unroll
  for (int i = 0; i < kTkPer; ++i) {
    const bool eq = kv[i] == T;
    const uint32_t eqb = __ballot_sync(0xFFFFFFFFu, eq);
    const bool keep = kv[i] > T || (eq && eq_seen + __popc(eqb & lt) >= n_eq - need);
    const uint32_t kb = __ballot_sync(0xFFFFFFFFu, keep);
    if (keep) {
      keys[wpos + __popc(kb & lt)] = kv[i];
      cols[wpos + __popc(kb & lt)] = cv[i];
    }
    wpos += __popc(kb);
    eq_seen += __popc(eqb);
  }
  __syncwarp();
  return T;
}

__device__ __forceinline__ float tk_key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key ^ 0x80000000u) : ~key);
}

// One warp per query block b: the k best key blocks c <= b of its score row
// (b itself forced), written ascending and padded with -1.  Rows are taken
// longest first.  Lane l holds the four consecutive columns hi - 4l - u,
// u = 0..3, of a 128-column chunk, so that lane-major order is descending
// column order; a chunk's loads are issued while the chunk before is
// filtered.  Columns are compared with the threshold as floats (the order
// keys order them alike; the threshold is -inf until the first compaction,
// columns before 0 load as NaN, which no comparison keeps, and the forced
// diagonal loads as +inf); only the survivors get their keys.
__global__ void __launch_bounds__(32 * kTkWarps, 4) bs_topk_warp_kernel(const float* __restrict__ scores, int nb,
                                                                       int bh_total, int k, int32_t* blk_idx,
                                                                       int32_t* blk_cnt) {
  __shared__ uint32_t skeys[kTkWarps][kTkCap];
  __shared__ int32_t scols[kTkWarps][kTkCap];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long x = (long long)blockIdx.x * kTkWarps + warp;
  if (x >= (long long)nb * bh_total) return;
  const int b = nb - 1 - (int)(x / bh_total);
  const int bh = (int)(x % bh_total);
  const size_t row = (size_t)bh * nb + b;
  const float* sr = scores + row * nb;
  uint32_t* keys = skeys[warp];
  int32_t* cols = scols[warp];
  auto load = [&](int hi, float (&v)[4]) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = hi - 4 * lane - u;
      v[u] = (c >= 0) ? __ldg(sr + c) : __int_as_float(0x7FC00000);  // NaN
    }
  };
  int cnt = 0;
  float tauf = -INFINITY;  // the threshold as a value: -inf until the first compaction
  float cur[4];
  load(b, cur);
  if (lane == 0) cur[0] = INFINITY;  // column b: the forced diagonal
  for (int hi = b; hi >= 0; hi -= kTkChunk) {
    float nxt[4];
    if (hi - kTkChunk >= 0) load(hi - kTkChunk, nxt);
    // survivors: columns at or above the threshold (a value equal to it has
    // a lower column than the list's entries of that key, so it ranks above
    // them)
    auto survivors = [&]() {
      uint32_t m = 0;
#pragma unroll
      for (int u = 0; u < 4; ++u) m |= (uint32_t)(cur[u] >= tauf) << u;
      return m;
    };
    uint32_t m = survivors();
    int tot = (int)__reduce_add_sync(0xFFFFFFFFu, (uint32_t)__popc(m));
    if (cnt + tot > kTkCap) {
      tauf = tk_key_value(tk_compact(keys, cols, cnt, k, lane));
      cnt = k;
      m = survivors();
      tot = (int)__reduce_add_sync(0xFFFFFFFFu, (uint32_t)__popc(m));
    }
    if (tot) {
      const int n = __popc(m);
      int incl = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
      }
      int pos = cnt + incl - n;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if ((m >> u) & 1u) {
          const int c = hi - 4 * lane - u;
          keys[pos] = (c == b) ? 0xFFFFFFFFu : sel_order_key(cur[u]);
          cols[pos] = c;
          ++pos;
        }
      }
      cnt += tot;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) cur[u] = nxt[u];
  }
  __syncwarp();
  if (cnt > k) {
    tk_compact(keys, cols, cnt, k, lane);
    cnt = k;
  }
  int32_t* out = blk_idx + row * k;
  for (int i = lane; i < k; i += 32) out[i] = (i < cnt) ? cols[cnt - 1 - i] : -1;
  if (lane == 0) blk_cnt[row] = cnt;
}

}  // namespace

// d = 128; budgets up to 128 (a compacted list keeps room for a chunk); N a
// multiple of 256, so that score rows start 16-byte aligned for the TMA stores
bool bs_select_supported(int N, int d, int k) {
  return d == 128 && k >= 1 && k <= kTkCap - kTkChunk && N % 256 == 0 && N / 64 <= 65536;
}

cudaError_t bs_select_launch(const CUtensorMap& tmKs, const CUtensorMap& tmS, const BsEstParams& bp, int k,
                             int32_t* blk_idx, int32_t* blk_cnt, cudaStream_t stream) {
  ScoreParams sp;
  sp.qs = bp.qs;
  sp.scores = bp.scores;
  sp.scale = bp.scale;
  sp.nb = bp.N / 64;
  sp.nrt = (sp.nb + 127) / 128;
  sp.bh_total = bp.B * bp.nh;
  sp.status = bp.status;
  cudaError_t e = cudaFuncSetAttribute(bs_score_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  bs_score_tc_kernel<<<dim3(sp.nrt, sp.bh_total), kSelThreads, kSmem, stream>>>(tmKs, tmS, sp);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long rows = (long long)sp.nb * sp.bh_total;
  bs_topk_warp_kernel<<<(unsigned)((rows + kTkWarps - 1) / kTkWarps), 32 * kTkWarps, 0, stream>>>(
      bp.scores, sp.nb, sp.bh_total, k, blk_idx, blk_cnt);
  return cudaGetLastError();
}

}  // namespace minf
