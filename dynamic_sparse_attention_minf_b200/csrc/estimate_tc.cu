// Vertical-Slash index estimation on the tensor cores ("MInference 1.0"
// summary, "Key points": the last query vectors are scored against all keys).
//
// One CTA takes one head and a run of 128-key tiles, and scores the last 64
// query rows against each tile with one tcgen05 GEMM (bf16 inputs, exact
// products, fp32 accumulation in TMEM).  The real rows are the last
// `last_q` <= 64; the others are masked.  Two passes:
//
//  pass 1 (vs_rowstat_tc_kernel): S = Q_last K^T with the 64 rows as TMEM
//          lanes.  The A operand holds Q's last 64 rows twice (rows 0-63 and
//          64-127), so that every lane quarter holds real scores: lanes 0-63
//          serve key columns 0-63 and lanes 64-127 key columns 64-127, and
//          eight score warps (two per SM sub-partition) each keep an online
//          (max, sum) of 2^(s * scale * log2 e) over 32 columns of their row.
//          The four column groups of a row are merged and written as the
//          CTA's partial of that row; a fixed-order kernel combines the CTAs.
//  pass 2 (vs_colsum_tc_kernel): S^T = K Q_last^T with the tile's 128 keys
//          as TMEM lanes and the 64 rows as columns, so that each thread owns
//          one key.  It forms p = 2^(x - m) / l for its 64 rows with the
//          combined row statistics; the key's vertical score is a sum over
//          its own registers, and the diagonal sums come from a rotation of
//          the warp's 32 x 64 block through lane shuffles (below).  Two
//          groups of four score warps take alternate tiles, each with its own
//          64-column TMEM buffer, and two CTAs share each SM.
//
// Both passes end with one warp whose lane 0 is the TMA producer and one
// TMEM-owning MMA issuer warp.  Every sum runs in a fixed order and nothing
// is added atomically, so results are bit-reproducible.
#include <algorithm>
#include <type_traits>

#include "minf_device.cuh"
#include "minf_internal.h"

namespace minf {

// ------------------------------------------------------------------ pass 1
// Two K stages keep the CTA under half of an SM's shared memory, so that two
// CTAs share each SM and hide each other's waits.
template <int D>
struct RowCfg {
  static constexpr int kScoreWarps = 8;
  static constexpr int kThreads = 32 * (kScoreWarps + 2);
  static constexpr int kScoreThreads = 256;
  static constexpr int kRegion = 128 * 128;
  static constexpr int kTileBytes = 128 * D * 2;  // 128 rows (Q twice) or 128 keys (K)
  static constexpr int kStages = 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kTileBytes;
  static constexpr int kOffBars = kOffK + kStages * kTileBytes;
  // barriers: q_full, k_full[kStages], k_empty[kStages], s_full[2], s_free[2], mma_done
  static constexpr int kNumBars = 1 + 2 * kStages + 4 + 1;
  static constexpr int kOffMisc = kOffBars + kNumBars * 8;
  static constexpr int kOffXch = kOffMisc + 16;  // [4][64][2] fp32
  static constexpr int kSmem = kOffXch + 4 * 64 * 2 * 4;
  static_assert(kSmem <= 232448 / 2, "two CTAs per SM");
  static constexpr uint32_t kIdescS = idesc_bf16(128, 128, 0, 0);
};

template <int D>
__global__ void __launch_bounds__(RowCfg<D>::kThreads, 2)
    vs_rowstat_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const VsEstParams p, int tiles_per_cta, int nchunks) {
  using C = RowCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // heads vary fastest: the CTAs resident together take the same key tiles
  // for every listed head, so that the heads of one KV group read each K tile
  // from L2 after the first one brought it in
  const int hi = blockIdx.x, chunk = blockIdx.y, b = blockIdx.z;
  const int head = p.heads[hi];
  if ((smem_u32(smem) & 1023u) != 0u || head < 0 || head >= p.Hq) {
    if (threadIdx.x == 0) report(p.status, MINF_ERR_DEVICE_BOUNDS, 60);
    return;
  }
  const int kvh = head / p.group;
  const int ntiles = (p.N + 127) / 128;
  const int t0 = chunk * tiles_per_cta;
  const int nt = min(ntiles, t0 + tiles_per_cta) - t0;
  const size_t bh = (size_t)b * p.nh + hi;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + C::kStages;
  uint64_t* s_full = k_empty + C::kStages;
  uint64_t* s_free = s_full + 2;
  uint64_t* mma_done = s_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&s_full[w], 1);
      mbar_init(&s_free[w], C::kScoreThreads);
    }
    mbar_init(mma_done, 1);
    *abort = 0;
    fence_mbar_init();
  }
  const int w_prod = C::kScoreWarps, w_mma = C::kScoreWarps + 1;
  if (warp == w_mma) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == w_prod) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // Q's last 64 rows into rows 0-63 and again into rows 64-127
      mbar_arrive_expect_tx(q_full, C::kTileBytes);
      const int qrow0 = (b * p.Hq + head) * p.N + p.N - 64;
#pragma unroll
      for (int h = 0; h < D / 64; ++h) {
        tma_load_2d(smem + C::kOffQ + h * C::kRegion, &tmQ, q_full, 64 * h, qrow0);
        tma_load_2d(smem + C::kOffQ + h * C::kRegion + 8192, &tmQ, q_full, 64 * h, qrow0);
      }
      const int kv_row0 = (b * p.Hkv + kvh) * p.N;
      int issued = 0;
      for (int k = 0; k < nt; ++k) {
        const int st = k % C::kStages;
        if (k >= C::kStages && !mbar_wait(&k_empty[st], ((k / C::kStages) - 1) & 1, abort, p.status, 61)) break;
        const int j0 = (t0 + k) * 128;
        uint8_t* kb = smem + C::kOffK + st * C::kTileBytes;
        mbar_arrive_expect_tx(&k_full[st], C::kTileBytes);
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
          tma_load_2d(kb + h * C::kRegion, &tmK, &k_full[st], 64 * h, kv_row0 + j0);
          tma_load_2d(kb + h * C::kRegion + 8192, &tmK, &k_full[st], 64 * h, kv_row0 + j0 + 64);
        }
        issued = k + 1;
      }
      int dummy = 0;  // never exit with copies in flight
      for (int k = max(0, issued - C::kStages); k < issued; ++k)
        mbar_wait(&k_full[k % C::kStages], (k / C::kStages) & 1, &dummy, p.status, 62);
      mbar_wait(q_full, 0, &dummy, p.status, 63);
    }
  } else if (warp == w_mma) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(q_full, 0, abort, p.status, 64);
      const uint32_t qaddr = smem_u32(smem + C::kOffQ);
      for (int k = 0; k < nt && ok; ++k) {
        const int st = k % C::kStages, buf = k & 1;
        ok = mbar_wait(&k_full[st], (k / C::kStages) & 1, abort, p.status, 65);
        if (ok && k >= 2) ok = mbar_wait(&s_free[buf], ((k >> 1) - 1) & 1, abort, p.status, 66);
        if (!ok) break;
        tc_fence_after();
        const uint32_t kaddr = smem_u32(smem + C::kOffK + st * C::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kRegion + (kk & 3) * 32;
          umma_ss(tmem + buf * 128, sdesc_sw128(qaddr + off, 16, 1024), sdesc_sw128(kaddr + off, 16, 1024),
                  C::kIdescS, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[buf]);
        umma_commit(&k_empty[st]);
      }
      umma_commit(mma_done);
      int dummy = 0;
      mbar_wait(mma_done, 0, &dummy, p.status, 67);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------- score warps
    const int qq = warp & 3;                       // TMEM lane quarter (warp & 3)
    const int grp = (qq >> 1) * 2 + (warp >> 2);  // column group: key columns 32 grp .. 32 grp + 31
    const int bar_sync = 1, bar_vote = 2;
    const int qrow = (qq & 1) * 32 + lane;         // query row N - 64 + qrow
    const int i = p.N - 64 + qrow;
    const bool real = qrow >= 64 - p.last_q;
    const uint32_t taddr = tmem + ((uint32_t)(qq * 32) << 16) + grp * 32;
    const float sl2 = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    for (int k = 0; k < nt; ++k) {
      const int buf = k & 1;
      // all score warps agree before going on (the exchange below meets at a
      // barrier, which a warp that gave up would never reach)
      const bool got = __all_sync(0xFFFFFFFFu, mbar_wait(&s_full[buf], (k >> 1) & 1, abort, p.status, 68));
      if (!bar_and(bar_vote, C::kScoreThreads, got)) break;
      tc_fence_after();
      uint32_t v0[32];
      tmem_ld32(taddr + buf * 128, v0);
      tmem_wait_ld();
      reg_fence(v0);
      tc_fence_before();
      mbar_arrive(&s_free[buf]);
      const int j0 = (t0 + k) * 128 + grp * 32;
      float x[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) x[c] = (real && j0 + c <= i) ? __uint_as_float(v0[c]) * sl2 : -INFINITY;
      float m4[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) m4[q] = -INFINITY;
#pragma unroll
      for (int c = 0; c < 32; ++c) m4[c & 3] = fmaxf(m4[c & 3], x[c]);
      const float tm = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      if (tm > m) {
        if (m != -INFINITY) l *= fast_exp2(m - tm);
        m = tm;
      }
      if (m != -INFINITY) {
        float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 32; ++c) a4[c & 3] += fast_exp2(x[c] - m);
        l += (a4[0] + a4[1]) + (a4[2] + a4[3]);
      }
    }
    float* xch = reinterpret_cast<float*>(smem + C::kOffXch);
    xch[(grp * 64 + qrow) * 2] = m;
    xch[(grp * 64 + qrow) * 2 + 1] = l;
    named_bar_sync(bar_sync, C::kScoreThreads);
    if (grp == 0) {
      float M = -INFINITY;
#pragma unroll
      for (int g = 0; g < 4; ++g) M = fmaxf(M, xch[(g * 64 + qrow) * 2]);
      float L = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const float mg = xch[(g * 64 + qrow) * 2], lg = xch[(g * 64 + qrow) * 2 + 1];
          if (mg != -INFINITY) L += lg * fast_exp2(mg - M);
        }
      }
      float* out = p.part_ml + ((bh * nchunks + chunk) * 64 + qrow) * 2;
      out[0] = M;
      out[1] = L;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == w_mma) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ------------------------------------------------------------------ pass 2
// Diagonal sums by rotation.  Warp w of a group holds the keys 32 w + L of
// the tile (lane L) and, in register q, the entry of query row q.  At step q
// every lane L reads register q of lane (q - L) mod 32, whose entry lies on
// the warp-local diagonal (row - key) = q - ((q - L) mod 32), which is L - 32,
// L or L + 32.  Each lane therefore adds the 64 values it receives into three
// sums, the warp-local diagonals L - 32, L and L + 32, taking each entry of
// the warp's 32 x 64 block exactly once; only 64 shuffles per warp and tile
// are needed.  The tile diagonal kd (entries (q, key q - kd + 127)) is the
// warp-local diagonal kd - 127 + 32 w, so the four warps' sums are combined
// in a fixed order through 96 shared-memory slots per warp.
template <int D>
struct ColCfg {
  static constexpr int kGroups = 2;          // score groups, on alternate key tiles
  static constexpr int kGroupThreads = 128; // one warp per TMEM lane quarter
  static constexpr int kScoreWarps = 4 * kGroups;
  static constexpr int kThreads = 32 * (kScoreWarps + 2);
  static constexpr int kQHalf = 64 * 128;   // a 64-column half of Q's 64 rows (bytes)
  static constexpr int kKHalf = 128 * 128;  // a 64-column half of a 128-key tile
  static constexpr int kQBytes = 64 * D * 2;
  static constexpr int kKBytes = 128 * D * 2;
  static constexpr int kStages = 2;          // two CTAs per SM: four K tiles in flight
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;               // 1024-aligned
  static constexpr int kOffPart = kOffK + kStages * kKBytes;  // [kGroups][4][96] fp32
  static constexpr int kOffRow = kOffPart + kGroups * 4 * 96 * 4;  // [32] row-pair statistics
  static constexpr int kOffBars = kOffRow + 64 * 8;
  // barriers: q_full, k_full[kStages], k_empty[kStages], s_full[kGroups], s_free[kGroups], mma_done
  static constexpr int kNumBars = 1 + 2 * kStages + 2 * kGroups + 1;
  static constexpr int kOffMisc = kOffBars + kNumBars * 8;
  static constexpr int kSmem = kOffMisc + 16;
  static_assert(kSmem <= 232448 / 2, "two CTAs per SM");
  static_assert(kOffK % 1024 == 0, "swizzled K stages");
  static_assert(kOffRow % 16 == 0, "row statistics read as float4");
  static constexpr int kTmemCols = 64 * kGroups;
  static constexpr uint32_t kIdescT = idesc_bf16(128, 64, 0, 0);  // M = 128 keys, N = 64 rows
};

template <int D>
__global__ void __launch_bounds__(ColCfg<D>::kThreads, 2)
    vs_colsum_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const VsEstParams p, int tiles_per_cta) {
  using C = ColCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hi = blockIdx.x, chunk = blockIdx.y, b = blockIdx.z;  // heads fastest, as in pass 1
  const int head = p.heads[hi];
  if ((smem_u32(smem) & 1023u) != 0u || head < 0 || head >= p.Hq) {
    if (threadIdx.x == 0) report(p.status, MINF_ERR_DEVICE_BOUNDS, 60);
    return;
  }
  const int kvh = head / p.group;
  const int ntiles = (p.N + 127) / 128;
  const int t0 = chunk * tiles_per_cta;
  const int nt = min(ntiles, t0 + tiles_per_cta) - t0;
  const size_t bh = (size_t)b * p.nh + hi;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + C::kStages;
  uint64_t* s_full = k_empty + C::kStages;
  uint64_t* s_free = s_full + C::kGroups;
  uint64_t* mma_done = s_free + C::kGroups;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  float* rowst = reinterpret_cast<float*>(smem + C::kOffRow);
  const float4* row4 = reinterpret_cast<const float4*>(smem + C::kOffRow);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int g = 0; g < C::kGroups; ++g) {
      mbar_init(&s_full[g], 1);
      mbar_init(&s_free[g], C::kGroupThreads);
    }
    mbar_init(mma_done, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 64) {
    // combined statistics of row q, stored by pairs of rows as
    // (-max[2h], -max[2h+1], 1/sum[2h], 1/sum[2h+1]); rows that are not real
    // stay 0 and are masked below
    const int q = threadIdx.x;
    float nm = 0.f, il = 0.f;
    if (q >= 64 - p.last_q) {
      nm = -p.row_ml[(bh * 64 + q) * 2];
      il = p.row_ml[(bh * 64 + q) * 2 + 1];
    }
    rowst[(q >> 1) * 4 + (q & 1)] = nm;
    rowst[(q >> 1) * 4 + 2 + (q & 1)] = il;
  }
  const int w_prod = C::kScoreWarps, w_mma = C::kScoreWarps + 1;
  if (warp == w_mma) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == w_prod) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, C::kQBytes);
      const int qrow0 = (b * p.Hq + head) * p.N + p.N - 64;
#pragma unroll
      for (int h = 0; h < D / 64; ++h) tma_load_2d(smem + C::kOffQ + h * C::kQHalf, &tmQ, q_full, 64 * h, qrow0);
      const int kv_row0 = (b * p.Hkv + kvh) * p.N;
      int issued = 0;
      for (int k = 0; k < nt; ++k) {
        const int st = k % C::kStages;
        if (k >= C::kStages && !mbar_wait(&k_empty[st], ((k / C::kStages) - 1) & 1, abort, p.status, 81)) break;
        const int j0 = (t0 + k) * 128;
        uint8_t* kb = smem + C::kOffK + st * C::kKBytes;
        mbar_arrive_expect_tx(&k_full[st], C::kKBytes);
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
          tma_load_2d(kb + h * C::kKHalf, &tmK, &k_full[st], 64 * h, kv_row0 + j0);
          tma_load_2d(kb + h * C::kKHalf + 8192, &tmK, &k_full[st], 64 * h, kv_row0 + j0 + 64);
        }
        issued = k + 1;
      }
      int dummy = 0;  // never exit with copies in flight
      for (int k = max(0, issued - C::kStages); k < issued; ++k)
        mbar_wait(&k_full[k % C::kStages], (k / C::kStages) & 1, &dummy, p.status, 82);
      mbar_wait(q_full, 0, &dummy, p.status, 83);
    }
  } else if (warp == w_mma) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(q_full, 0, abort, p.status, 84);
      const uint32_t qaddr = smem_u32(smem + C::kOffQ);
      for (int k = 0; k < nt && ok; ++k) {
        const int st = k % C::kStages, g = k % C::kGroups, use = k / C::kGroups;
        ok = mbar_wait(&k_full[st], (k / C::kStages) & 1, abort, p.status, 85);
        if (ok && use > 0) ok = mbar_wait(&s_free[g], (use - 1) & 1, abort, p.status, 86);
        if (!ok) break;
        tc_fence_after();
        const uint32_t kaddr = smem_u32(smem + C::kOffK + st * C::kKBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ka = kaddr + (kk >> 2) * C::kKHalf + (kk & 3) * 32;
          const uint32_t qa = qaddr + (kk >> 2) * C::kQHalf + (kk & 3) * 32;
          umma_ss(tmem + g * 64, sdesc_sw128(ka, 16, 1024), sdesc_sw128(qa, 16, 1024), C::kIdescT,
                  kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[g]);
        umma_commit(&k_empty[st]);
      }
      umma_commit(mma_done);
      int dummy = 0;
      mbar_wait(mma_done, 0, &dummy, p.status, 87);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------- score warps
    const int g = warp >> 2;                         // group: key tiles g, g + kGroups, ...
    const int qq = warp & 3;                         // TMEM lane quarter: keys 32 qq .. 32 qq + 31
    const int bar_vote = 1 + 2 * g, bar_sync = 2 + 2 * g;
    const int tid = threadIdx.x & (C::kGroupThreads - 1);
    const uint32_t taddr = tmem + ((uint32_t)(qq * 32) << 16) + g * 64;
    float* part = reinterpret_cast<float*>(smem + C::kOffPart) + g * 4 * 96;
    const uint64_t sl2x2 = f32x2_pack(p.scale_log2, p.scale_log2);
    const int qfirst = 64 - p.last_q;  // rows below are not real
    for (int k = g; k < nt; k += C::kGroups) {
      // the group's four warps agree before going on (they meet at a barrier
      // below, which a warp that gave up would never reach); the vote also
      // tells every thread that the previous tile's slots have been read
      const bool got =
          __all_sync(0xFFFFFFFFu, mbar_wait(&s_full[g], (k / C::kGroups) & 1, abort, p.status, 88));
      if (!bar_and(bar_vote, C::kGroupThreads, got)) break;
      tc_fence_after();
      const int j = (t0 + k) * 128 + qq * 32 + lane;  // this thread's key
      // row q (position N - 64 + q) sees key j when it is real and j <= N - 64 + q
      const int qmin = max(qfirst, j - (p.N - 64));
      // vertical score of key j as four interleaved partial sums (rows q mod
      // 4), and the warp-local diagonals lane - 32 (dlo), lane (dmid) and
      // lane + 32 (dhi); rows 0-31 are finished before rows 32-63
      uint64_t a01 = 0ull, a23 = 0ull;  // partial sums of rows 0, 1 and 2, 3 mod 4, paired
      float dlo = 0.f, dmid = 0.f, dhi = 0.f;
      // `masked` (a std::bool_constant) compiles the row mask in or out.  The
      // TMEM buffer is the group's alone until its next tile, so the rows are
      // read 32 at a time and the buffer is released after the second read.
      auto rows32 = [&](const int q0, float& d_up, float& d_lo, auto masked) {
        uint32_t r[32];
        tmem_ld32(taddr + q0, r);
        tmem_wait_ld();
        reg_fence(r);
        if (q0 == 32) {
          tc_fence_before();
          mbar_arrive(&s_free[g]);
        }
        float pv[32];
        // rows 2 h and 2 h + 1 share one broadcast load of their statistics
        // and go through the paired fp32 FMA (each half an ordinary fma)
#pragma unroll
        for (int h = 0; h < 16; ++h) {
          const float4 ml = row4[q0 / 2 + h];
          float x0, x1, p0, p1;
          f32x2_unpack(f32x2_fma(f32x2_pack(__uint_as_float(r[2 * h]), __uint_as_float(r[2 * h + 1])), sl2x2,
                                 f32x2_pack(ml.x, ml.y)),
                       x0, x1);
          // e * (1/sum) + 0 rounds exactly as the product does
          f32x2_unpack(f32x2_fma(f32x2_pack(fast_exp2(x0), fast_exp2(x1)), f32x2_pack(ml.z, ml.w), 0ull), p0, p1);
          if constexpr (decltype(masked)::value) {
            pv[2 * h] = q0 + 2 * h >= qmin ? p0 : 0.f;
            pv[2 * h + 1] = q0 + 2 * h + 1 >= qmin ? p1 : 0.f;
          } else {
            pv[2 * h] = p0;
            pv[2 * h + 1] = p1;
          }
        }
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          a01 = f32x2_add(a01, f32x2_pack(pv[c], pv[c + 1]));
          a23 = f32x2_add(a23, f32x2_pack(pv[c + 2], pv[c + 3]));
        }
        // row q0 + c of lane (c - lane) mod 32 lies on the warp-local diagonal
        // q0 + lane (c >= lane) or q0 + lane - 32
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float v = __shfl_sync(0xFFFFFFFFu, pv[c], (c - lane) & 31);
          if (c >= lane) d_up += v; else d_lo += v;
        }
      };
      if (__all_sync(0xFFFFFFFFu, qmin <= 0)) {
        rows32(0, dmid, dlo, std::false_type{});
        rows32(32, dhi, dmid, std::false_type{});
      } else {
        rows32(0, dmid, dlo, std::true_type{});
        rows32(32, dhi, dmid, std::true_type{});
      }
      float a0, a1, a2, a3;
      f32x2_unpack(a01, a0, a1);
      f32x2_unpack(a23, a2, a3);
      if (j < p.N) p.v_score[bh * p.N + j] = (a0 + a1) + (a2 + a3);
      float* pw = part + qq * 96;  // slot s holds the warp-local diagonal s - 32
      pw[lane] = dlo;
      pw[32 + lane] = dmid;
      pw[64 + lane] = dhi;
      named_bar_sync(bar_sync, C::kGroupThreads);
      float* dp = p.dpart + (bh * ntiles + t0 + k) * 192;
      auto combine = [&](int kd) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const int sl = kd - 95 + 32 * w;
          if (sl >= 0 && sl < 96) s += part[w * 96 + sl];
        }
        dp[kd] = s;
      };
      combine(tid);
      if (tid < 63) combine(128 + tid);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == w_mma) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int D>
static cudaError_t launch_est_tc(const CUtensorMap& tq, const CUtensorMap& tk, const VsEstParams& p,
                                 cudaStream_t stream) {
  using C1 = RowCfg<D>;
  using C2 = ColCfg<D>;
  const int ntiles = (p.N + 127) / 128;
  const long long units = (long long)ntiles * p.nh * p.B;
  // pass 1: about four CTAs per SM in all, at most 32 key tiles each
  const int tpc = (int)std::max<long long>(1, std::min<long long>(32, (units + 591) / 592));
  const int nchunks = (ntiles + tpc - 1) / tpc;
  // pass 2 (two CTAs per SM): runs of 2 to 64 tiles, so that both score groups
  // have work, and about four waves when there are enough tiles
  const int tpc2 = (int)std::max<long long>(ColCfg<D>::kGroups, std::min<long long>(64, (units + 1183) / 1184));
  const int nchunks2 = (ntiles + tpc2 - 1) / tpc2;
  if (nchunks > 65535 || nchunks2 > 65535 || p.nh > 65535 || p.B > 65535) return cudaErrorInvalidConfiguration;
  cudaError_t e =
      cudaFuncSetAttribute(vs_rowstat_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C1::kSmem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(vs_colsum_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C2::kSmem);
  if (e != cudaSuccess) return e;
  vs_rowstat_tc_kernel<D><<<dim3(p.nh, nchunks, p.B), C1::kThreads, C1::kSmem, stream>>>(tq, tk, p, tpc, nchunks);
  e = vs_combine_launch(p, nchunks, stream);
  if (e != cudaSuccess) return e;
  vs_colsum_tc_kernel<D><<<dim3(p.nh, nchunks2, p.B), C2::kThreads, C2::kSmem, stream>>>(tq, tk, p, tpc2);
  // the tile's score rows are the last 64 query rows (rows beyond last_q are
  // zero), so the diagonal partials use the 64-row geometry
  VsEstParams q64 = p;
  q64.last_q = 64;
  return vs_slash_launch(q64, stream);
}

cudaError_t vs_estimate_tc_launch(const CUtensorMap& tq, const CUtensorMap& tk, const VsEstParams& p,
                                  cudaStream_t stream) {
  if (p.d == 128) return launch_est_tc<128>(tq, tk, p, stream);
  if (p.d == 64) return launch_est_tc<64>(tq, tk, p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace minf
