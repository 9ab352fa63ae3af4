// Vertical-Slash index estimation on the tensor cores ("MInference 1.0"
// summary, "Key points": the last query vectors are scored against all keys).
//
// One CTA takes one head and a run of 128-key tiles.  The scores of the last
// query rows against a key tile, S = Q_last K^T, are one tcgen05 GEMM (bf16
// inputs, exact products, fp32 accumulation in TMEM).  The A operand holds
// Q's last 64 rows twice (rows 0-63 and 64-127), so that every TMEM lane
// quarter holds real scores: lanes 0-63 serve key columns 0-63 and lanes
// 64-127 key columns 64-127, and all eight score warps (two per SM
// sub-partition) work on each tile, 32 rows x 32 columns each.  The real rows
// are the last `last_q` <= 64.  K tiles stream through a TMA ring of 2 stages
// (pass 1, two CTAs per SM) or 3 (pass 2).
//
//  pass 1: each thread keeps an online (max, sum) of 2^(s * scale * log2 e)
//          over its columns of the CTA's tiles; the four column groups of a
//          row are merged and written as the CTA's partial of that row.
//  pass 2: p = 2^(x - m) / l with the combined row statistics is written to
//          shared memory, and the CTA forms, in a fixed order, the column
//          sums (vertical scores) and the tile's 191 diagonal partials.
//
// Score warps: 8 (pass 1) or 16 (pass 2: two groups of 8 on alternate key
// tiles, each with its own P buffer); then one warp whose lane 0 is the TMA
// producer, and one TMEM-owning MMA issuer warp.
#include <algorithm>

#include "minf_device.cuh"
#include "minf_internal.h"

namespace minf {

// Pass 1 needs no P buffer: two K stages keep its CTA under half of an SM's
// shared memory, so that two CTAs share each SM and hide each other's waits.
// Pass 2 runs two groups of eight score warps, on the even and the odd key
// tiles, so that one group's shared-memory sums overlap the other's scores.
template <int D, int PASS>
struct EstCfg {
  static constexpr int kGroups = (PASS == 1) ? 1 : 2;
  static constexpr int kScoreWarps = 8 * kGroups;
  static constexpr int kThreads = 32 * (kScoreWarps + 2);
  static constexpr int kScoreThreads = 256;  // per group
  static constexpr int kRegion = 128 * 128;
  static constexpr int kTileBytes = 128 * D * 2;  // 128 rows (Q twice) or 128 keys (K)
  static constexpr int kStages = (PASS == 1) ? 2 : 3;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kTileBytes;
  static constexpr int kOffP = kOffK + kStages * kTileBytes;  // pass 2: 2 x [64][129] fp32
  static constexpr int kPStride = 129;
  static constexpr int kPBytes = 64 * kPStride * 4;
  static constexpr int kOffBars = kOffP + (PASS == 2 ? 2 * kPBytes : 0);
  // barriers: q_full, k_full[kStages], k_empty[kStages], s_full[2], s_free[2], mma_done
  static constexpr int kNumBars = 1 + 2 * kStages + 4 + 1;
  static constexpr int kOffMisc = kOffBars + kNumBars * 8;
  static constexpr int kOffXch = kOffMisc + 16;             // pass 1: [4][64][2] fp32
  static constexpr int kSmem = kOffXch + 4 * 64 * 2 * 4;
  static_assert(kSmem <= 232448, "shared memory budget");
  static constexpr uint32_t kIdescS = idesc_bf16(128, 128, 0, 0);
};

template <int D, int PASS>
__global__ void __launch_bounds__(EstCfg<D, PASS>::kThreads, PASS == 1 ? 2 : 1)
    vs_est_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const VsEstParams p, int tiles_per_cta, int nchunks) {
  using C = EstCfg<D, PASS>;
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
    const int sg = warp >> 3;                     // warp group: key tiles sg, sg + kGroups, ...
    const int ww = warp & 7;
    const int qq = ww & 3;                        // TMEM lane quarter (warp & 3)
    const int grp = (qq >> 1) * 2 + (ww >> 2);    // column group: key columns 32 grp .. 32 grp + 31
    const int bar_sync = 1 + 2 * sg, bar_vote = 2 + 2 * sg;  // this group's named barriers
    const int qrow = (qq & 1) * 32 + lane;        // query row N - 64 + qrow
    const int i = p.N - 64 + qrow;
    const bool real = qrow >= 64 - p.last_q;
    const uint32_t taddr = tmem + ((uint32_t)(qq * 32) << 16) + grp * 32;
    const float sl2 = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    float mr = 0.f, il = 0.f;
    if (PASS == 2 && real) {
      mr = p.row_ml[(bh * 64 + qrow) * 2];
      il = p.row_ml[(bh * 64 + qrow) * 2 + 1];
    }
    for (int k = sg; k < nt; k += C::kGroups) {
      const int buf = k & 1;
      // all score warps of the group agree before going on (pass 2 meets at a
      // barrier below, which a warp that gave up would never reach)
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
      if (PASS == 1) {
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
      } else {
        float* P = reinterpret_cast<float*>(smem + C::kOffP + buf * C::kPBytes);
#pragma unroll
        for (int c = 0; c < 32; ++c)
          P[qrow * C::kPStride + grp * 32 + c] = (x[c] == -INFINITY) ? 0.f : fast_exp2(x[c] - mr) * il;
        named_bar_sync(bar_sync, C::kScoreThreads);
        const int tid = threadIdx.x & 255;  // 0 .. 255 within the group
        // Fixed-order sums over the tile's 64 rows, each as four interleaved
        // partial sums (rows q = 0, 1, 2, 3 mod 4) added in a fixed order.
        // Threads 0-127: vertical score of key column tid, then (0-62) the
        // diagonal 128 + tid; threads 128-255: the diagonal tid - 128.
        // Diagonal kd holds the entries (q, q - kd + 127).
        auto diag = [&](int kd) {
          float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
          const int qhi = min(63, kd);
          // entry (q, q - kd + 127) sits at q * (stride + 1) + 127 - kd
          constexpr int kStep = C::kPStride + 1;
          int q = max(0, kd - 127);
          int x = q * kStep + 127 - kd;
          for (; q + 3 <= qhi; q += 4, x += 4 * kStep) {
            a0 += P[x];
            a1 += P[x + kStep];
            a2 += P[x + 2 * kStep];
            a3 += P[x + 3 * kStep];
          }
          for (; q <= qhi; ++q, x += kStep) a0 += P[x];
          p.dpart[(bh * ntiles + t0 + k) * 192 + kd] = (a0 + a1) + (a2 + a3);
        };
        if (tid < 128) {
          float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 16
          for (int q = 0; q < 64; ++q) a4[q & 3] += P[q * C::kPStride + tid];
          const int jj = (t0 + k) * 128 + tid;
          if (jj < p.N) p.v_score[bh * p.N + jj] = (a4[0] + a4[1]) + (a4[2] + a4[3]);
          if (tid < 63) diag(128 + tid);
        } else {
          diag(tid - 128);
        }
      }
    }
    if (PASS == 1) {
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
  }
  tc_fence_before();
  __syncthreads();
  if (warp == w_mma) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int D>
static cudaError_t launch_est_tc(const CUtensorMap& tq, const CUtensorMap& tk, const VsEstParams& p,
                                 cudaStream_t stream) {
  using C1 = EstCfg<D, 1>;
  using C2 = EstCfg<D, 2>;
  const int ntiles = (p.N + 127) / 128;
  // about four CTAs per SM in all, at most 32 key tiles each
  const long long units = (long long)ntiles * p.nh * p.B;
  const int tpc = (int)std::max<long long>(1, std::min<long long>(32, (units + 591) / 592));
  const int nchunks = (ntiles + tpc - 1) / tpc;
  cudaError_t e = cudaFuncSetAttribute(vs_est_tc_kernel<D, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, C1::kSmem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(vs_est_tc_kernel<D, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, C2::kSmem);
  if (e != cudaSuccess) return e;
  const dim3 grid(p.nh, nchunks, p.B);
  vs_est_tc_kernel<D, 1><<<grid, C1::kThreads, C1::kSmem, stream>>>(tq, tk, p, tpc, nchunks);
  e = vs_combine_launch(p, nchunks, stream);
  if (e != cudaSuccess) return e;
  vs_est_tc_kernel<D, 2><<<grid, C2::kThreads, C2::kSmem, stream>>>(tq, tk, p, tpc, nchunks);
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
