// Causal (sparse) attention mainloop for sm_100a: one CTA per work item, a
// (batch, head, 128-row query tile), warp-specialized.  One launch can hold
// the heads of up to three patterns, so that a whole layer of mixed patterns
// is one grid ("MInference 1.0" summary, "Summary": a pattern per head,
// attention over the indices only).  The grid takes the patterns in turn and
// within a pattern one head after the other, each head's query tiles from
// the bottom of the causal triangle up: the CTAs resident at a time share
// one head's K and V in L2, and the light items (a head's first tiles, and
// the Block-Sparse and A-shape heads after the Vertical-Slash ones) fill the
// end of the launch.
//
//   warps 0-3  softmax warpgroup 0: key columns 0-63 of every tile  (thread = query row)
//   warps 4-7  softmax warpgroup 1: key columns 64-127 of every tile
//   warp  8    tcgen05 issuer (the whole warp runs the loop, one elected lane
//              issues) and TMEM owner
//   warp  9    producer: enumerates the key tiles of the query tile for the
//              head's pattern, writes each tile's descriptor (column ids and
//              per-64-row-half membership masks) and stages K and V into two
//              rings of shared-memory slots: by TMA for contiguous 64-key
//              chunks (one 3-D copy of all column regions when the two chunks
//              are adjacent), by cp.async for gathered columns.  A K slot frees
//              when S of its tile is done and the softmax has released its
//              descriptor, a V slot when P V is done; the V of a range tile is
//              loaded after the next tile's K.
//
// Per key tile t (128 keys) the issuer computes S = Q K^T into TMEM buffer
// t&1.  Warpgroup w masks and exponentiates its 64 columns of S and writes P
// (bf16) back over them in TMEM; the issuer then accumulates
// O_w += P[:, 64w:64w+64] V[64w:64w+64, :] with P read from TMEM.  Each
// warpgroup keeps its own running max / sum and O accumulator over its column
// half of every tile, and the two are merged in the epilogue, so both
// warpgroups work on every tile with no exchange between them, while the
// issuer computes the next tile's scores into the other buffer.
//
// The four key sources ("MInference 1.0" summary, "Summary": A-shape,
// Vertical-Slash, Block-Sparse; and dense causal attention as the baseline):
//   dense   : keys [0, R+128) in 128-key tiles, causal mask on the last
//   A-shape : [0, n_sink) and the local band [R - n_local + 1, R + 128),
//             per element j < n_sink or i - j < n_local
//   VS      : the union over slash groups of the bands swept by the tile's
//             rows, then the verticals of both 64-row halves, gathered
//   BS      : the selected 64-key blocks of both halves, two per tile
//   VS exact: the same ranges at 128-row granularity, masked per element
//             from offset and key bitmaps, then the tile's vertical list
//
// The softmax runs one pair of exponentials in four through a polynomial on
// the FMA pipe (the rest on the MUFU).  Every wait is bounded: a wait that
// runs out records MINF_ERR_DEVICE_TIMEOUT, and all roles stop, drain their
// copies and MMAs, free TMEM and return.
#include "minf_device.cuh"
#include "minf_internal.h"

namespace minf {

enum { KIND_END = 0, KIND_RANGE = 1, KIND_GATHER = 2 };
enum { F_MASK = 1, F_CAUSAL = 2, F_ASHAPE = 4, F_EXACT = 8 };

struct TileDesc {
  int kind;
  int flags;
  int j0[2];             // RANGE: first key of the two 64-key chunks
  uint32_t mask[2][4];   // per 64-row half: key-column membership bits
  int cols[128];         // GATHER: key id of every column
};

template <int D>
struct AttnCfg {
  static constexpr int kThreads = 320;
  static constexpr int kRegion = 128 * 128;                 // bytes: 128 rows x 128 B
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kKVBytes = 128 * D * 2;
  static constexpr int kKStages = (D == 128) ? 3 : 4;  // K slots (with their descriptors)
  static constexpr int kVStages = (D == 128) ? 3 : 4;  // V slots
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kKStages * kKVBytes;
  static constexpr int kOffDesc = kOffV + kVStages * kKVBytes;
  static constexpr int kOffSCols = kOffDesc + kKStages * (int)sizeof(TileDesc);
  static constexpr int kOffSBits = kOffSCols + 160 * 4;
  static constexpr int kOffBars = kOffSBits + 160;
  // barriers: k_full, k_empty, d_empty [kKStages]; v_full, v_empty [kVStages];
  // s_full[2], p_full[2], q_full, mma_done
  static constexpr int kNumBars = 3 * kKStages + 2 * kVStages + 6;
  static constexpr int kOffMisc = kOffBars + kNumBars * 8;
  static constexpr int kSmem = kOffMisc + 16;
  static_assert(kSmem <= 232448, "shared memory budget");
  static constexpr uint32_t kIdescS = idesc_bf16(128, 128, 0, 0);
  static constexpr uint32_t kIdescPV = idesc_bf16(128, D, 0, 1);
  static constexpr int kColO0 = 256;
  static constexpr int kColO1 = 256 + D;
};

__device__ __forceinline__ uint32_t count_mask(int cnt, int wd) {
  int n = cnt - 32 * wd;
  if (n >= 32) return 0xFFFFFFFFu;
  if (n <= 0) return 0u;
  return (1u << n) - 1u;
}

// 32 bits of the slash-band bitmap starting at bit position p (bits below 0
// read as zero).
__device__ __forceinline__ uint32_t wmap_window(const uint32_t* W, int p) {
  if (p <= -32) return 0u;
  if (p < 0) return __ldg(W) << (-p);
  const int wi = p >> 5;
  return __funnelshift_r(__ldg(W + wi), __ldg(W + wi + 1), p & 31);
}
__device__ __forceinline__ uint32_t wmap_bit(const uint32_t* W, int x) {
  return (__ldg(W + (x >> 5)) >> (x & 31)) & 1u;
}

// Bits p .. p + 63 of a bitmap as one 64-bit value, bit k = bit p + k (bits
// below 0 read as zero), from the three words starting at word max(p, 0) / 32
// (loaded separately, so that the loads can be issued early).
struct Window64 {
  uint32_t w0, w1, w2;
  int p;
  __device__ __forceinline__ void load(const uint32_t* W, int p_) {
    p = p_;
    const int wi = max(p, 0) >> 5;
    w0 = __ldg(W + wi);
    w1 = __ldg(W + wi + 1);
    w2 = __ldg(W + wi + 2);
  }
  __device__ __forceinline__ uint64_t bits() const {
    if (p <= -64) return 0ull;
    const int sh = max(p, 0) & 31;
    uint64_t v = ((uint64_t)__funnelshift_r(w1, w2, sh) << 32) | __funnelshift_r(w0, w1, sh);
    if (p < 0) v <<= -p;
    return v;
  }
};
__device__ __forceinline__ uint64_t brev64(uint64_t x) {
  return ((uint64_t)__brev((uint32_t)x) << 32) | __brev((uint32_t)(x >> 32));
}

// A wait whose outcome is the same for every lane of the warp (the TMEM
// accesses that follow are warp-collective).
// True in exactly one lane of a fully active warp, the same lane every time.
__device__ __forceinline__ bool elect_one() {
  uint32_t e;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(e));
  return e != 0;
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, DevStatus* st,
                                          int where) {
  const bool ok = mbar_wait(bar, parity, abort, st, where);
  return __all_sync(0xFFFFFFFFu, ok);
}

template <int D>
struct Producer {
  using C = AttnCfg<D>;
  uint8_t* smem;
  TileDesc* desc;
  int* scols;
  uint8_t* sbits;
  uint64_t* k_full;
  uint64_t* v_full;
  uint64_t* k_empty;
  uint64_t* v_empty;
  uint64_t* d_empty;
  const CUtensorMap* tmK;   // 64-row boxes
  const CUtensorMap* tmV;
  const CUtensorMap* tmK2;  // 128-row boxes over all d/64 column regions (3-D view)
  const CUtensorMap* tmV2;
  const __nv_bfloat16* Kh;  // this (batch, kv head)'s K rows
  const __nv_bfloat16* Vh;
  int kv_row0;
  int R;
  int N;
  int lane;
  int t;        // tiles whose K side (and descriptor) has been emitted
  int tv;       // tiles whose V side has been emitted: t - 1 (a range tile's V lags) or t
  int vj0[2];   // key chunks of tile tv while its V lags
  volatile int* abort;
  DevStatus* st;
  bool ok;

  // Claims the K slot and the descriptor of tile t: S = Q K^T of tile t - S
  // is done and the softmax warps have read its descriptor.  False on abort.
  __device__ bool acquire_k(int& stage) {
    stage = t % C::kKStages;
    if (t >= C::kKStages) {
      const uint32_t par = ((t / C::kKStages) - 1) & 1;
      if (!warp_wait(&k_empty[stage], par, abort, st, 1) || !warp_wait(&d_empty[stage], par, abort, st, 14)) {
        ok = false;
        return false;
      }
    }
    return true;
  }

  // Claims the V slot of tile u: P V of tile u - S is done.
  __device__ bool acquire_v(int u, int& stage) {
    stage = u % C::kVStages;
    if (u >= C::kVStages) {
      if (!warp_wait(&v_empty[stage], ((u / C::kVStages) - 1) & 1, abort, st, 15)) {
        ok = false;
        return false;
      }
    }
    return true;
  }

  // Issues the V loads of the range tile whose V lags behind its K.
  __device__ void emit_v_lag() {
    if (!ok || tv == t) return;
    int stage;
    if (!acquire_v(tv, stage)) return;
    if (lane == 0) {
      uint8_t* vb = smem + C::kOffV + stage * C::kKVBytes;
      mbar_arrive_expect_tx(&v_full[stage], C::kKVBytes);
      if (vj0[1] == vj0[0] + 64) {
        tma_load_3d(vb, tmV2, &v_full[stage], 0, kv_row0 + vj0[0], 0);
      } else {
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
          tma_load_2d(vb + h * C::kRegion, tmV, &v_full[stage], 64 * h, kv_row0 + vj0[0]);
          tma_load_2d(vb + h * C::kRegion + 8192, tmV, &v_full[stage], 64 * h, kv_row0 + vj0[1]);
        }
      }
    }
    ++tv;
  }

  // A tile of two 64-key chunks at keys j0a, j0b with per-half mask words
  // (lane l < 8 holds word (l >> 2, l & 3)).  K is loaded now; V after the
  // next tile's K, so that K loads run ahead of the V slots' release.
  __device__ void emit_range(int j0a, int j0b, uint32_t word, int flags) {
    if (!ok) return;
    int stage;
    if (!acquire_k(stage)) return;
    TileDesc& dd = desc[stage];
    const bool full = __all_sync(0xFFFFFFFFu, lane >= 8 || word == 0xFFFFFFFFu);
    if (lane < 8) dd.mask[lane >> 2][lane & 3] = word;
    if (lane == 0) {
      dd.kind = KIND_RANGE;
      dd.flags = flags | (full ? 0 : F_MASK);
      dd.j0[0] = j0a;
      dd.j0[1] = j0b;
    }
    // __syncwarp orders the lanes' descriptor writes before lane 0's
    // release-arrive on k_full; no further fence is needed
    __syncwarp();
    if (lane == 0) {
      uint8_t* kb = smem + C::kOffK + stage * C::kKVBytes;
      mbar_arrive_expect_tx(&k_full[stage], C::kKVBytes);
      if (j0b == j0a + 64) {
        tma_load_3d(kb, tmK2, &k_full[stage], 0, kv_row0 + j0a, 0);
      } else {
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
          tma_load_2d(kb + h * C::kRegion, tmK, &k_full[stage], 64 * h, kv_row0 + j0a);
          tma_load_2d(kb + h * C::kRegion + 8192, tmK, &k_full[stage], 64 * h, kv_row0 + j0b);
        }
      }
    }
    emit_v_lag();  // V of the previous tile
    ++t;
    vj0[0] = j0a;
    vj0[1] = j0b;
  }

  // A gathered tile of the first cnt staged columns (1 <= cnt <= 128); its K
  // and V rows are copied together.
  __device__ void emit_gather(int cnt) {
    if (!ok) return;
    int stage;
    if (!acquire_k(stage)) return;
    TileDesc& dd = desc[stage];
    int any_late = 0;
#pragma unroll
    for (int wd = 0; wd < 4; ++wd) {
      const int c = 32 * wd + lane;
      const int j = (c < cnt) ? scols[c] : scols[0];
      dd.cols[c] = j;
      any_late |= (c < cnt && j > R);
      const uint32_t b = (c < cnt) ? sbits[c] : 0u;
      const uint32_t w0 = __ballot_sync(0xFFFFFFFFu, b & 1u);
      const uint32_t w1 = __ballot_sync(0xFFFFFFFFu, b & 2u);
      if (lane == 0) {
        dd.mask[0][wd] = w0;
        dd.mask[1][wd] = w1;
      }
    }
    any_late = __any_sync(0xFFFFFFFFu, any_late);
    if (lane == 0) {
      dd.kind = KIND_GATHER;
      dd.flags = F_MASK | (any_late ? F_CAUSAL : 0);
    }
    __syncwarp();
    // 128 K rows, then 128 V rows, by cp.async into the 128B-swizzled layout.
    // Every lane's copies lower the slot barrier's count when they land
    // (cp.async.mbarrier.arrive), and lane 0's plain arrival completes the
    // phase, so the producer never waits for a gather; the issuer adds the
    // proxy fence that the generic-proxy writes need before the MMAs.
    constexpr int CH = D * 2 / 16;  // 16-byte chunks per row
    {
      const uint32_t kb = smem_u32(smem + C::kOffK + stage * C::kKVBytes);
#pragma unroll 8
      for (int it = 0; it < 128 * CH / 32; ++it) {
        const int idx = it * 32 + lane;
        const int c = idx / CH, q = idx % CH;
        const uint32_t off = (q >> 3) * C::kRegion + c * 128 + (((q & 7) ^ (c & 7)) << 4);
        cp_async16(kb + off, Kh + (size_t)dd.cols[c] * D + q * 8);
      }
      cp_async_mbar_arrive(&k_full[stage]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&k_full[stage]);
    }
    emit_v_lag();  // V of the previous tile
    int vstage;
    if (!acquire_v(t, vstage)) return;
    {
      const uint32_t vb = smem_u32(smem + C::kOffV + vstage * C::kKVBytes);
#pragma unroll 8
      for (int it = 0; it < 128 * CH / 32; ++it) {
        const int idx = it * 32 + lane;
        const int c = idx / CH, q = idx % CH;
        const uint32_t off = (q >> 3) * C::kRegion + c * 128 + (((q & 7) ^ (c & 7)) << 4);
        cp_async16(vb + off, Vh + (size_t)dd.cols[c] * D + q * 8);
      }
      cp_async_mbar_arrive(&v_full[vstage]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&v_full[vstage]);
    }
    ++t;
    ++tv;
  }

  __device__ void emit_end() {
    emit_v_lag();
    if (!ok) return;
    int stage;
    if (!acquire_k(stage)) return;
    if (lane == 0) {
      desc[stage].kind = KIND_END;
      desc[stage].flags = 0;
      mbar_arrive(&k_full[stage]);
    }
    __syncwarp();
    ++t;  // the END tile has no V side: tv stays at the last real tile
  }

  // Appends a warp-wide batch of candidate columns to the staging list,
  // emitting gathered tiles whenever 128 are ready.  n_staged is warp-uniform.
  __device__ void append(bool keep, int j, uint32_t bits, int& n_staged) {
    const uint32_t bal = __ballot_sync(0xFFFFFFFFu, keep);
    const int pos = n_staged + __popc(bal & ((1u << lane) - 1u));
    if (keep) {
      scols[pos] = j;
      sbits[pos] = (uint8_t)bits;
    }
    n_staged += __popc(bal);
    __syncwarp();
    if (n_staged >= 128) {
      emit_gather(128);
      __syncwarp();
      const int rest = n_staged - 128;
      int mj = 0;
      uint8_t mb = 0;
      if (lane < rest) {
        mj = scols[128 + lane];
        mb = sbits[128 + lane];
      }
      __syncwarp();
      if (lane < rest) {
        scols[lane] = mj;
        sbits[lane] = mb;
      }
      n_staged = rest;
      __syncwarp();
    }
  }

  // Waits (bounded, ignoring the abort flag) until every copy this producer
  // started has landed, so that the CTA never exits with copies in flight:
  // the last tiles of each ring (older ones were waited for when
  // their slots were reused).  The slots carry no per-stage bookkeeping
  // (an array indexed by stage would move the producer's state to local
  // memory).
  __device__ void drain() {
    cp_async_wait<0>();
    __syncwarp();
    if (lane == 0) {
      int dummy = 0;
      for (int u = max(0, t - C::kKStages); u < t; ++u)
        mbar_wait(&k_full[u % C::kKStages], (u / C::kKStages) & 1, &dummy, st, 9);
      for (int u = max(0, tv - C::kVStages); u < tv; ++u)
        mbar_wait(&v_full[u % C::kVStages], (u / C::kVStages) & 1, &dummy, st, 9);
    }
    __syncwarp();
  }
};

// batches of 32 vertical-list entries whose loads are issued together
constexpr int kVB = 8;
// band tiles between two gathered tiles of a Vertical-Slash query tile
constexpr int kGatherGap = 24;

template <int D>
__device__ void produce_tiles(Producer<D>& P, const AttnParams& p, int POL, int nh, int b, int hi, int qt) {
  const int R = qt * 128;
  const int lane = P.lane;
  if (POL == POL_DENSE) {
    for (int m = 0; m <= qt && P.ok; ++m) {
      P.emit_range(128 * m, 128 * m + 64, 0xFFFFFFFFu, m == qt ? F_CAUSAL : 0);
    }
  } else if (POL == POL_ASHAPE) {
    const int lloc = max(0, R - p.n_local + 1);
    const int far_edge = R + 127 - p.n_local;   // keys <= this may leave some row's window
    auto interval = [&](int lo, int hi_) {
      for (int j0 = lo; j0 <= hi_ && P.ok; j0 += 128) {
        const int cnt = min(128, hi_ - j0 + 1);
        const uint32_t word = (lane < 8) ? count_mask(cnt, lane & 3) : 0xFFFFFFFFu;
        int flags = (j0 + cnt - 1 > R) ? F_CAUSAL : 0;
        if (max(j0, p.n_sink) <= min(j0 + cnt - 1, far_edge)) flags |= F_ASHAPE;
        P.emit_range(j0, j0 + 64, word, flags);
      }
    };
    if (p.n_sink >= lloc) {
      interval(0, R + 127);  // sinks and window touch: one interval
    } else {
      if (p.n_sink > 0) interval(0, p.n_sink - 1);
      interval(lloc, R + 127);
    }
  } else if (POL == POL_VS) {
    const size_t hrow = (size_t)b * nh + hi;
    const int* tg = p.tgrp + hrow * p.k_s * 2;
    const int G = p.tgrp_cnt[hrow];
    const uint32_t* W = p.wmap + hrow * p.wmap_words;
    // The tile's gathered columns come from its gather list, 128 per tile,
    // one gathered tile after every kGatherGap band tiles (their copies take
    // the producer several band tiles' time) and the rest after the bands.
    // Each tile's list entries are loaded while the tile before is emitted.
    const int nt = p.N / 128;
    const int32_t* gl = p.tvidx + (hrow * nt + qt) * (size_t)p.k_v;
    const int gcnt = min(__ldg(p.tvcnt + hrow * nt + qt), p.k_v);
    int gpos = 0, since = 0;
    uint32_t gbuf[4];
    auto gload = [&]() {
#pragma unroll
      for (int wd = 0; wd < 4; ++wd) {
        const int c = gpos + 32 * wd + lane;
        gbuf[wd] = (c < gcnt) ? (uint32_t)__ldg(gl + c) : 0u;
      }
    };
    auto gemit = [&]() {
      const int cnt = min(128, gcnt - gpos);
#pragma unroll
      for (int wd = 0; wd < 4; ++wd) {
        const int c = 32 * wd + lane;
        if (c < cnt) {
          int j = (int)(gbuf[wd] & 0x3FFFFFFFu);
          if (j > R + 127) { report(P.st, MINF_ERR_DEVICE_BOUNDS, 20); j = 0; }
          P.scols[c] = j;
          P.sbits[c] = (uint8_t)(gbuf[wd] >> 30);
        }
      }
      __syncwarp();
      P.emit_gather(cnt);
      __syncwarp();
      gpos += cnt;
      gload();
    };
    auto band = [&](int j0, uint32_t word, int flags) {
      P.emit_range(j0, j0 + 64, word, flags);
      if (++since == kGatherGap) {
        since = 0;
        if (gpos < gcnt && P.ok) gemit();
      }
    };
    gload();
    // Slash bands, in ascending keys = descending offsets.  Only tile groups
    // with a_G <= R + 127 reach this query tile: binary-search the last one,
    // then walk down 32 groups at a time, one group per lane, each lane
    // fetching its group's first-tile mask words so that the loads of a batch
    // overlap instead of costing a round trip per group.
    int top = 0;
    {
      int lo = 0, hi2 = G;
      while (lo < hi2) {
        const int mid = (lo + hi2) >> 1;
        if (__ldg(tg + 2 * mid) <= R + 127) lo = mid + 1; else hi2 = mid;
      }
      top = lo - 1;
    }
    auto tile_word = [&](int j0, int cnt, int hh, int wd) -> uint32_t {
      const int x0 = R + 64 * hh - j0 + 63 - 32 * wd;
      return __brev(wmap_window(W, x0 - 31)) & count_mask(cnt, wd);
    };
    // The words of a group's later tiles are fetched four tiles at a time,
    // one word per lane, and the next four are requested while the current
    // ones are emitted, so that no tile waits for a bitmap load.
    for (int base = top; base >= 0 && P.ok; base -= 32) {
      const int gl = base - lane;
      int lo_l = 0, hi_l = -1;
      uint32_t w8[8];
      if (gl >= 0) {
        const int A = __ldg(tg + 2 * gl), Bo = __ldg(tg + 2 * gl + 1);
        hi_l = min(R + 127 - A, p.N - 1);
        lo_l = max(0, R - Bo);
        const int cnt = min(128, hi_l - lo_l + 1);
#pragma unroll
        for (int q = 0; q < 8; ++q) w8[q] = tile_word(lo_l, cnt, q >> 2, q & 3);
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) w8[q] = 0u;
      }
      const int nbatch = min(32, base + 1);
      for (int k = 0; k < nbatch && P.ok; ++k) {
        const int lo_key = __shfl_sync(0xFFFFFFFFu, lo_l, k);
        const int hi_key = __shfl_sync(0xFFFFFFFFu, hi_l, k);
        uint32_t wf = 0xFFFFFFFFu;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint32_t v = __shfl_sync(0xFFFFFFFFu, w8[q], k);
          if (lane == q) wf = v;
        }
        const int ntile = (hi_key - lo_key) / 128 + 1;
        // word (lane & 7) of tile 1 + 4c + (lane >> 3)
        auto chunk_word = [&](int c) -> uint32_t {
          const int tt = 1 + 4 * c + (lane >> 3);
          if (tt >= ntile) return 0xFFFFFFFFu;
          const int j0 = lo_key + 128 * tt;
          return tile_word(j0, min(128, hi_key - j0 + 1), (lane >> 2) & 1, lane & 3);
        };
        uint32_t wcur = (ntile > 1) ? chunk_word(0) : 0xFFFFFFFFu;
        uint32_t wnext = (ntile > 5) ? chunk_word(1) : 0xFFFFFFFFu;
        {
          const int cnt = min(128, hi_key - lo_key + 1);
          band(lo_key, wf, (lo_key + cnt - 1 > R) ? F_CAUSAL : 0);
        }
        for (int tt = 1; tt < ntile && P.ok; ++tt) {
          const int slot = (tt - 1) & 3;
          if (slot == 0 && tt > 1) {
            wcur = wnext;
            const int c = (tt - 1) >> 2;
            wnext = (1 + 4 * (c + 1) < ntile) ? chunk_word(c + 1) : 0xFFFFFFFFu;
          }
          const uint32_t wv = __shfl_sync(0xFFFFFFFFu, wcur, slot * 8 + (lane & 7));
          const int j0 = lo_key + 128 * tt;
          const int cnt = min(128, hi_key - j0 + 1);
          band(j0, lane < 8 ? wv : 0xFFFFFFFFu, (j0 + cnt - 1 > R) ? F_CAUSAL : 0);
        }
      }
    }
    while (gpos < gcnt && P.ok) gemit();
  } else if (POL == POL_VS_EXACT) {
    // The same key ranges as the band variant at 128-row granularity (one per
    // offset group of gap 128), masked element by element by the softmax from
    // the offset and key bitmaps; then the tile's own vertical list.
    const size_t hrow = (size_t)b * nh + hi;
    const int* tg = p.tgrp + hrow * p.k_s * 2;
    const int G = p.tgrp_cnt[hrow];
    int top = 0;
    {
      int lo = 0, hi2 = G;
      while (lo < hi2) {
        const int mid = (lo + hi2) >> 1;
        if (__ldg(tg + 2 * mid) <= R + 127) lo = mid + 1; else hi2 = mid;
      }
      top = lo - 1;
    }
    for (int base = top; base >= 0 && P.ok; base -= 32) {
      const int gl = base - lane;
      int lo_l = 0, hi_l = -1;
      if (gl >= 0) {
        hi_l = min(R + 127 - __ldg(tg + 2 * gl), p.N - 1);
        lo_l = max(0, R - __ldg(tg + 2 * gl + 1));
      }
      const int nbatch = min(32, base + 1);
      for (int k = 0; k < nbatch && P.ok; ++k) {
        const int lo_key = __shfl_sync(0xFFFFFFFFu, lo_l, k);
        const int hi_key = __shfl_sync(0xFFFFFFFFu, hi_l, k);
        for (int j0 = lo_key; j0 <= hi_key && P.ok; j0 += 128) {
          const int cnt = min(128, hi_key - j0 + 1);
          const uint32_t word = (lane < 8) ? count_mask(cnt, lane & 3) : 0xFFFFFFFFu;
          P.emit_range(j0, j0 + 64, word, F_EXACT | ((j0 + cnt - 1 > R) ? F_CAUSAL : 0));
        }
      }
    }
    const int nt = p.N / 128;
    const int* vl = p.vidx + (hrow * nt + qt) * (size_t)p.k_v;
    const int c = min(p.vcnt[hrow * nt + qt], p.k_v);
    int n_staged = 0;
    for (int base = 0; base < c && P.ok; base += 32 * kVB) {
      int jv[kVB];
#pragma unroll
      for (int k = 0; k < kVB; ++k) {
        const int idx = base + 32 * k + lane;
        jv[k] = (idx < c) ? __ldg(vl + idx) : 0;
      }
#pragma unroll
      for (int k = 0; k < kVB; ++k) {
        if (base + 32 * k >= c || !P.ok) break;
        const int idx = base + 32 * k + lane;
        int j = jv[k];
        if (j < 0 || j > R + 127) { if (idx < c) report(P.st, MINF_ERR_DEVICE_BOUNDS, 24); j = 0; }
        P.append(idx < c, j, (j <= R + 63 ? 1u : 0u) | 2u, n_staged);
      }
    }
    if (n_staged > 0 && P.ok) P.emit_gather(n_staged);
  } else if (POL == POL_BS) {
    const size_t hrow = (size_t)b * nh + hi;
    const int nb = p.N / 64;
    const int b0 = R / 64, b1 = b0 + 1;
    const int* s0 = p.blk_idx + (hrow * nb + b0) * (size_t)p.k_b;
    const int* s1 = p.blk_idx + (hrow * nb + b1) * (size_t)p.k_b;
    const int n0 = min(p.blk_cnt[hrow * nb + b0], p.k_b);
    const int n1 = min(p.blk_cnt[hrow * nb + b1], p.k_b);
    int n_staged = 0;
    // staging of whole key blocks; a tile takes two
    auto flush_pairs = [&](bool final_) {
      while (n_staged >= 2 || (final_ && n_staged == 1)) {
        const int ca = P.scols[0];
        const uint32_t ba = P.sbits[0];
        const bool two = n_staged >= 2;
        const int cb = two ? P.scols[1] : ca;
        const uint32_t bb = two ? P.sbits[1] : 0u;
        uint32_t word = 0xFFFFFFFFu;
        if (lane < 8) {
          const int hh = lane >> 2, wd = lane & 3;
          const uint32_t bits = (wd < 2) ? ba : bb;
          word = ((bits >> hh) & 1u) ? 0xFFFFFFFFu : 0u;
        }
        const int flags = (max(ca, cb) >= b0) ? F_CAUSAL : 0;
        P.emit_range(64 * ca, 64 * cb, word, flags);
        __syncwarp();
        const int used = two ? 2 : 1;
        int mj = 0;
        uint8_t mb = 0;
        const int rest = n_staged - used;
        if (lane < rest) { mj = P.scols[used + lane]; mb = P.sbits[used + lane]; }
        __syncwarp();
        if (lane < rest) { P.scols[lane] = mj; P.sbits[lane] = mb; }
        n_staged = rest;
        __syncwarp();
        if (!P.ok) return;
      }
    };
    for (int base = 0; base < n1 && P.ok; base += 32) {
      const int idx = base + lane;
      int c = (idx < n1) ? s1[idx] : 0;
      if (c < 0 || c > b1) { if (idx < n1) report(P.st, MINF_ERR_DEVICE_BOUNDS, 22); c = 0; }
      // member of half 0's list?  (binary search in s0)
      int lo = 0, hi2 = n0;
      while (lo < hi2) { const int mid = (lo + hi2) >> 1; if (s0[mid] < c) lo = mid + 1; else hi2 = mid; }
      const uint32_t h0 = (lo < n0 && s0[lo] == c) ? 1u : 0u;
      const bool keep = idx < n1;
      const uint32_t bal = __ballot_sync(0xFFFFFFFFu, keep);
      // append one at a time through the shared staging list in order
      const int pos = n_staged + __popc(bal & ((1u << lane) - 1u));
      if (keep) { P.scols[pos] = c; P.sbits[pos] = (uint8_t)(h0 | 2u); }
      n_staged += __popc(bal);
      __syncwarp();
      flush_pairs(false);
    }
    for (int base = 0; base < n0 && P.ok; base += 32) {
      const int idx = base + lane;
      int c = (idx < n0) ? s0[idx] : 0;
      if (c < 0 || c > b0) { if (idx < n0) report(P.st, MINF_ERR_DEVICE_BOUNDS, 23); c = 0; }
      int lo = 0, hi2 = n1;
      while (lo < hi2) { const int mid = (lo + hi2) >> 1; if (s1[mid] < c) lo = mid + 1; else hi2 = mid; }
      const bool in1 = (lo < n1 && s1[lo] == c);
      const bool keep = idx < n0 && !in1;
      const uint32_t bal = __ballot_sync(0xFFFFFFFFu, keep);
      const int pos = n_staged + __popc(bal & ((1u << lane) - 1u));
      if (keep) { P.scols[pos] = c; P.sbits[pos] = 1u; }
      n_staged += __popc(bal);
      __syncwarp();
      flush_pairs(false);
    }
    if (P.ok) flush_pairs(true);
  }
}

template <int D, bool EXACT>
__global__ void __launch_bounds__(320, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmK2,
                const __grid_constant__ CUtensorMap tmV2, const AttnParams p) {
  using C = AttnCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // work item: the segment (pattern), then (batch, head), then the query
  // tile from the heaviest down
  int x = (int)blockIdx.x;
  int seg = 0;
  while (seg < p.nseg - 1 && x >= p.B * p.seg[seg].nh * p.nqt) {
    x -= p.B * p.seg[seg].nh * p.nqt;
    ++seg;
  }
  const int qt = p.nqt - 1 - x % p.nqt;
  const int bh = x / p.nqt;
  const int b = bh / p.seg[seg].nh;
  const int hi = bh % p.seg[seg].nh;
  const int pol = p.seg[seg].pol;
  const int nh = p.seg[seg].nh;
  const int head = p.seg[seg].heads ? __ldg(p.seg[seg].heads + hi) : hi;
  const int kvh = head / p.group;
  const int R = qt * 128;

  TileDesc* desc = reinterpret_cast<TileDesc*>(smem + C::kOffDesc);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint64_t* k_full = bars;
  uint64_t* k_empty = bars + C::kKStages;      // S = Q K^T of the slot's tile is done
  uint64_t* d_empty = bars + 2 * C::kKStages;  // the softmax warps have read the descriptor
  uint64_t* v_full = bars + 3 * C::kKStages;
  uint64_t* v_empty = v_full + C::kVStages;    // P V of the slot's tile is done
  uint64_t* s_full = v_empty + C::kVStages;
  uint64_t* p_full = s_full + 2;
  uint64_t* q_full = p_full + 2;
  uint64_t* mma_done = q_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  if ((smem_u32(smem) & 1023u) != 0u) {  // the swizzled layouts need 1 KiB alignment
    if (threadIdx.x == 0) report(p.status, MINF_ERR_DEVICE_BOUNDS, 99);
    return;
  }
  if (head < 0 || head >= p.Hq) {
    if (threadIdx.x == 0) report(p.status, MINF_ERR_DEVICE_BOUNDS, 98);
    return;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kKStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&d_empty[s], 256);
    }
    for (int s = 0; s < C::kVStages; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&s_full[w], 1);
      mbar_init(&p_full[w], 256);
    }
    mbar_init(q_full, 1);
    mbar_init(mma_done, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 9) {
    // ------------------------------------------------------------ producer
    Producer<D> P;
    P.smem = smem;
    P.desc = desc;
    P.scols = reinterpret_cast<int*>(smem + C::kOffSCols);
    P.sbits = smem + C::kOffSBits;
    P.k_full = k_full;
    P.v_full = v_full;
    P.k_empty = k_empty;
    P.v_empty = v_empty;
    P.d_empty = d_empty;
    P.tmK = &tmK;
    P.tmV = &tmV;
    P.tmK2 = &tmK2;
    P.tmV2 = &tmV2;
    P.kv_row0 = (b * p.Hkv + kvh) * p.N;
    P.Kh = p.K + (size_t)P.kv_row0 * D;
    P.Vh = p.V + (size_t)P.kv_row0 * D;
    P.R = R;
    P.N = p.N;
    P.lane = lane;
    P.t = 0;
    P.tv = 0;
    P.vj0[0] = P.vj0[1] = 0;
    P.abort = abort;
    P.st = p.status;
    P.ok = true;
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmK2);
      prefetch_tmap(&tmV2);
      mbar_arrive_expect_tx(q_full, C::kQBytes);
      const int qrow = (b * p.Hq + head) * p.N + R;
#pragma unroll
      for (int h = 0; h < D / 64; ++h) tma_load_2d(smem + C::kOffQ + h * C::kRegion, &tmQ, q_full, 64 * h, qrow);
    }
    __syncwarp();
    // Failure-detection test hook: the first CTA withholds every key tile,
    // so its consumers' bounded waits run out and the call reports a timeout.
    const bool withhold = p.status->withhold != 0 && blockIdx.x == 0;
    if (!withhold) {
      produce_tiles<D>(P, p, pol, nh, b, hi, qt);
      if (lane == 0 && P.ok) atomicAdd(&p.status->tiles, (unsigned long long)P.t);
      P.emit_end();
    }
    P.drain();
    if (lane == 0) {
      int dummy = 0;
      mbar_wait(q_full, 0, &dummy, p.status, 8);
    }
  } else if (warp == 8) {
    // --------------------------------------------------------- MMA issuer
    // The whole warp runs the loop, so that stage indices and descriptors are
    // warp-uniform; one elected lane issues the MMAs and their commits.
    const uint32_t qaddr = smem_u32(smem + C::kOffQ);
    // O_0 += P[:, 0:64] V[0:64, :] and O_1 += P[:, 64:128] V[64:128, :];
    // warpgroup w's bf16 P occupies TMEM columns 64w .. 64w+31 of the buffer
    auto issue_pv = [&](int tp, bool gathered) -> bool {
      const int bp = tp & 1;
      const int sp = tp % C::kVStages;
      if (!warp_wait(&p_full[bp], (tp >> 1) & 1, abort, p.status, 3)) return false;
      if (!warp_wait(&v_full[sp], (tp / C::kVStages) & 1, abort, p.status, 4)) return false;
      if (gathered) fence_proxy_async();  // V rows written by cp.async
      tc_fence_after();
      // descriptors of the K-steps: the stage's base plus a constant (the
      // start-address field holds address / 16 and never carries out)
      const uint64_t vd0 = sdesc_sw128(smem_u32(smem + C::kOffV + sp * C::kKVBytes), C::kRegion, 1024);
      const uint32_t a0 = tmem + bp * 128;
      const uint32_t acc0 = tp > 0 ? 1u : 0u;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t d_tmem = tmem + (kk < 4 ? C::kColO0 : C::kColO1);
          umma_ts(d_tmem, a0 + (kk >> 2) * 64 + (kk & 3) * 8, vd0 + (uint64_t)(kk * 2048 / 16), C::kIdescPV,
                  (kk & 3) > 0 ? 1u : acc0);
        }
        umma_commit(&v_empty[sp]);
      }
      __syncwarp();
      return true;
    };
    bool ok = warp_wait(q_full, 0, abort, p.status, 2);
    const uint64_t qd0 = sdesc_sw128(qaddr, 16, 1024);
    int t = 0, pend = -1;
    bool pend_gathered = false;
    while (ok) {
      const int st = t % C::kKStages;
      if (!warp_wait(&k_full[st], (t / C::kKStages) & 1, abort, p.status, 5)) { ok = false; break; }
      const int kd = desc[st].kind;
      if (__all_sync(0xFFFFFFFFu, kd == KIND_END)) break;
      // Q and range K tiles were written by TMA, and the barrier alone orders
      // them before the MMA (no tcgen05 fence here: it would stall the issue
      // of every tile); gathered rows were written by cp.async, whose
      // generic-proxy writes need a proxy fence first.
      const bool gathered = __all_sync(0xFFFFFFFFu, kd == KIND_GATHER);
      if (gathered) fence_proxy_async();
      const int w = t & 1;  // S buffer
      const uint64_t kd0 = sdesc_sw128(smem_u32(smem + C::kOffK + st * C::kKVBytes), 16, 1024);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off16 = (uint64_t)(((kk >> 2) * C::kRegion + (kk & 3) * 32) / 16);
          umma_ss(tmem + w * 128, qd0 + off16, kd0 + off16, C::kIdescS, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[w]);
        umma_commit(&k_empty[st]);
      }
      __syncwarp();
      if (pend >= 0 && !issue_pv(pend, pend_gathered)) { ok = false; pend = -1; break; }
      pend = t;
      pend_gathered = gathered;
      ++t;
    }
    if (ok && pend >= 0) issue_pv(pend, pend_gathered);
    if (elect_one()) umma_commit(mma_done);
    __syncwarp();
    if (lane == 0) {
      int dummy = 0;
      mbar_wait(mma_done, 0, &dummy, p.status, 7);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- softmax
    const int wg = warp >> 2;  // column half of every tile
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const int i = R + r;
    const int half = r >> 6;
    const float sl2 = p.scale_log2;
    const uint32_t srow = tmem + ((uint32_t)(q4 * 32) << 16);
    float m_run = -INFINITY, l_run = 0.f;
    int n = 0;
    unsigned nnz = 0;
    for (int t = 0;; ++t) {
      const int st = t % C::kKStages;
      if (!warp_wait(&k_full[st], (t / C::kKStages) & 1, abort, p.status, 10)) break;
      const TileDesc& dd = desc[st];
      // kind and flags, rebuilt through one vote so that every test on them
      // is warp-uniform for the compiler too (bit l of the word is lane l's)
      const uint32_t kf = __ballot_sync(
          0xFFFFFFFFu, ((((uint32_t)dd.kind & 0xFFu) << 8 | ((uint32_t)dd.flags & 0xFFu)) >> lane) & 1u);
      const int kind = (int)(kf >> 8);
      const int flags = (int)(kf & 0xFFu);
      if (kind == KIND_END) break;
      // element-exact tiles: the bitmap words of this row's window are
      // requested before waiting for the scores
      Window64 xs, xv;
      const bool exact = EXACT && (flags & F_EXACT);
      const int jw = dd.j0[wg];  // RANGE tiles: first key of this warpgroup's chunk
      if (exact) {
        const size_t hb = ((size_t)b * nh + hi) * p.bits_words;
        xs.load(p.sbits + hb, i - jw - 63);
        xv.load(p.vbits + hb, jw);
      }
      // Membership words of this warp's 64-row half for the warpgroup's two
      // 32-column chunks.  All rows of a warp lie in one half, so the chunk
      // tests are warp-uniform: full chunks need no masking, empty chunks are
      // not exponentiated.
      uint32_t mw[2] = {0xFFFFFFFFu, 0xFFFFFFFFu};
      if (flags & F_MASK) {
        const uint2 m2 = *reinterpret_cast<const uint2*>(&dd.mask[half][2 * wg]);
        mw[0] = m2.x;
        mw[1] = m2.y;
      }
      // a RANGE descriptor is fully read: release it (and with it the K slot)
      // before waiting for the scores; a GATHER one is read until the causal test
      if (kind != KIND_GATHER) mbar_arrive(&d_empty[st]);
      if (!warp_wait(&s_full[t & 1], (t >> 1) & 1, abort, p.status, 11)) break;
      tc_fence_after();
      const uint32_t scol = srow + (t & 1) * 128 + wg * 64;
      if (exact) {
        // bit c: (i - j in S) or (j in V) for key j = j0 + c; these words
        // differ between rows, so a chunk is skipped only if empty in all
        uint64_t em = brev64(xs.bits()) | xv.bits();
        // causal as bits: key j0 + c is allowed for c <= i - j0
        const int lim = i - jw;
        em &= (lim >= 63) ? ~0ull : (lim < 0 ? 0ull : ((2ull << lim) - 1ull));
        mw[0] &= (uint32_t)em;
        mw[1] &= (uint32_t)(em >> 32);
      }
      // chunk c2 needs no masking if full in every row, and no exponentials
      // if empty in every row
      bool cfull[2], cany[2];
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        cfull[c2] = __all_sync(0xFFFFFFFFu, mw[c2] == 0xFFFFFFFFu);
        cany[c2] = __any_sync(0xFFFFFFFFu, mw[c2] != 0u);
      }
      uint32_t sr[2][32];
      tmem_ld32(scol, sr[0]);
      tmem_ld32(scol + 32, sr[1]);
      tmem_wait_ld();
      reg_fence(sr[0]);
      reg_fence(sr[1]);
      float s[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(sr[c >> 5][c & 31]);
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        if (!cfull[c2] && cany[c2]) {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (!((mw[c2] >> e) & 1u)) s[c2 * 32 + e] = -INFINITY;
        }
      }
      if (!exact && (flags & (F_CAUSAL | F_ASHAPE))) {
        const bool causal = flags & F_CAUSAL;
        const bool ash = flags & F_ASHAPE;
        if (kind == KIND_RANGE) {
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const int j = jw + c;
            bool drop = causal && (j > i);
            drop |= ash && (j >= p.n_sink) && (i - j >= p.n_local);
            if (drop) s[c] = -INFINITY;
          }
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const int j = dd.cols[wg * 64 + c];
            if (causal && j > i) s[c] = -INFINITY;
          }
        }
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          if (cany[c2]) {
#pragma unroll
            for (int e = 0; e < 32; ++e) nnz += (s[c2 * 32 + e] != -INFINITY);
          }
        }
      } else {
        nnz += __popc(mw[0]) + __popc(mw[1]);
      }
      if (kind == KIND_GATHER) mbar_arrive(&d_empty[st]);  // descriptor no longer read
      // row max: eight independent chains over the non-empty chunks
      float mx8[8];
#pragma unroll
      for (int k8 = 0; k8 < 8; ++k8) mx8[k8] = -INFINITY;
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        if (cany[c2]) {
#pragma unroll
          for (int e = 0; e < 32; ++e) mx8[e & 7] = fmaxf(mx8[e & 7], s[c2 * 32 + e]);
        }
      }
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      const float m_new = fmaxf(m_run, mx * sl2);
      float alpha = 1.f;
      const bool resc = m_new > m_run + 8.f;
      if (resc) {
        alpha = fast_exp2(m_run - m_new);
        m_run = m_new;
      }
      const float msub = (m_run == -INFINITY) ? 0.f : m_run;
      // P = 2^(s * scale * log2 e - m) as bf16 pairs; the argument and the
      // row sum use packed two-lane fp32 instructions.
      const uint64_t sl2x2 = f32x2_pack(sl2, sl2), nm2 = f32x2_pack(-msub, -msub);
      uint64_t acc2[2] = {0ull, 0ull};
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        uint32_t pk[16];
        if (cany[c2]) {
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float x0, x1;
            f32x2_unpack(f32x2_fma(f32x2_pack(s[c2 * 32 + e], s[c2 * 32 + e + 1]), sl2x2, nm2), x0, x1);
            // one pair in four on the FMA pipe, the rest on the MUFU
            float p0, p1;
            if ((e & 6) == 6) {
              exp2_poly_x2(x0, x1, p0, p1);
            } else {
              p0 = fast_exp2(x0);
              p1 = fast_exp2(x1);
            }
            acc2[(e >> 1) & 1] = f32x2_add(acc2[(e >> 1) & 1], f32x2_pack(p0, p1));
            pk[e >> 1] = pack_bf16x2(p0, p1);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = 0u;
        }
        tmem_st16(scol + c2 * 16, pk);
      }
      float a0, a1, b0, b1;
      f32x2_unpack(acc2[0], a0, a1);
      f32x2_unpack(acc2[1], b0, b1);
      l_run = l_run * alpha + ((a0 + a1) + (b0 + b1));
      // lazy correction of the running output (rare after the first tiles),
      // done after the P stores so that the scores are no longer live
      if (__any_sync(0xFFFFFFFFu, resc && n > 0)) {
        // P V of the previous tile must be complete before O is rescaled
        if (!warp_wait(&v_empty[(n - 1) % C::kVStages], ((n - 1) / C::kVStages) & 1, abort, p.status, 12)) break;
        tc_fence_after();
        const uint32_t orow = srow + (wg ? C::kColO1 : C::kColO0);
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(orow + c0, o);
          tmem_wait_ld();
          reg_fence(o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(orow + c0, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[t & 1]);
      ++n;
    }
    // ----------------------------------------------------------- epilogue
    {
      unsigned long long c = nnz;
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) c += __shfl_xor_sync(0xFFFFFFFFu, c, o);
      if (lane == 0) atomicAdd(&p.status->nnz, c);
    }
    bool ok = !*abort;
    if (ok && n > 0) ok = warp_wait(&v_empty[(n - 1) % C::kVStages], ((n - 1) / C::kVStages) & 1, abort, p.status, 13);
    named_bar_sync(1, 256);
    float* xch = reinterpret_cast<float*>(smem + C::kOffK);  // all S MMAs are done: K stage 0 is free
    xch[(wg * 128 + r) * 4 + 0] = m_run;
    xch[(wg * 128 + r) * 4 + 1] = l_run;
    xch[(wg * 128 + r) * 4 + 2] = __int_as_float(n);
    named_bar_sync(1, 256);
    const float m0 = xch[r * 4 + 0], l0 = xch[r * 4 + 1];
    const float m1 = xch[(128 + r) * 4 + 0], l1 = xch[(128 + r) * 4 + 1];
    const int n0 = __float_as_int(xch[r * 4 + 2]);
    const int n1 = __float_as_int(xch[(128 + r) * 4 + 2]);
    ok = ok && !*abort;
    if (ok) {
      const float mt = fmaxf(m0, m1);
      const float a0 = (l0 > 0.f) ? fast_exp2(m0 - mt) : 0.f;
      const float a1 = (l1 > 0.f) ? fast_exp2(m1 - mt) : 0.f;
      const float L = l0 * a0 + l1 * a1;
      const float inv = (L > 0.f) ? 1.f / L : 0.f;
      const float c0f = a0 * inv, c1f = a1 * inv;
      tc_fence_after();
      __nv_bfloat16* orow_g = p.O + ((size_t)(b * p.Hq + head) * p.N + i) * D;
#pragma unroll
      for (int cc = 0; cc < D / 2; cc += 32) {
        const int col = wg * (D / 2) + cc;
        uint32_t x0[32], x1[32];
        if (n0 > 0) tmem_ld32(srow + C::kColO0 + col, x0);
        if (n1 > 0) tmem_ld32(srow + C::kColO1 + col, x1);
        tmem_wait_ld();
        reg_fence(x0);
        reg_fence(x1);
        uint32_t outw[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float v0 = 0.f, v1 = 0.f;
          if (n0 > 0) { v0 += __uint_as_float(x0[e]) * c0f; v1 += __uint_as_float(x0[e + 1]) * c0f; }
          if (n1 > 0) { v0 += __uint_as_float(x1[e]) * c1f; v1 += __uint_as_float(x1[e + 1]) * c1f; }
          outw[e >> 1] = pack_bf16x2(v0, v1);
        }
        if (i < p.N) {
          uint4* dst = reinterpret_cast<uint4*>(orow_g + col);
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[v] = make_uint4(outw[4 * v], outw[4 * v + 1], outw[4 * v + 2], outw[4 * v + 3]);
        }
      }
      if (wg == 0 && p.lse != nullptr && i < p.N) {
        p.lse[(size_t)(b * p.Hq + head) * p.N + i] = (L > 0.f) ? (mt + __log2f(L)) * 0.69314718055994531f : -INFINITY;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ launch
template <int D, bool EXACT>
static cudaError_t launch_attn(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                               const CUtensorMap& tk2, const CUtensorMap& tv2, const AttnParams& p,
                               cudaStream_t stream) {
  using C = AttnCfg<D>;
  auto kfn = attn_kernel<D, EXACT>;
  cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  kfn<<<p.nitems, C::kThreads, C::kSmem, stream>>>(tq, tk, tv, tk2, tv2, p);
  return cudaGetLastError();
}

cudaError_t attn_dispatch(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          const CUtensorMap& tk2, const CUtensorMap& tv2, const AttnParams& p, cudaStream_t stream) {
  // the element-exact reading has a kernel of its own (its bitmap windows
  // need registers in the softmax); it is never mixed with other patterns
  const bool exact = p.nseg == 1 && p.seg[0].pol == POL_VS_EXACT;
  if (d == 64) return exact ? launch_attn<64, true>(tq, tk, tv, tk2, tv2, p, stream)
                            : launch_attn<64, false>(tq, tk, tv, tk2, tv2, p, stream);
  if (d == 128) return exact ? launch_attn<128, true>(tq, tk, tv, tk2, tv2, p, stream)
                             : launch_attn<128, false>(tq, tk, tv, tk2, tv2, p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace minf
