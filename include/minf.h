/*
 * minf.h -- C ABI of libminf.so: the pre-fill hot path of dynamic sparse
 * attention ("MInference 1.0: Accelerating Pre-filling for Long-Context LLMs
 * via Dynamic Sparse Attention"), built for NVIDIA B200 (sm_100a).
 *
 * The method (abstract; summary page, "Summary" and "Key points"): every
 * attention head follows one of three patterns -- A-shape, Vertical-Slash or
 * Block-Sparse.  At inference time the sparse indices of a Vertical-Slash
 * head are estimated by scoring the last query vectors against all keys, and
 * those of a Block-Sparse head from queries and keys mean-pooled in 64-token
 * blocks; attention is then computed over those indices only.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are dense, row-major, on the device, owned by the caller:
 *      Q, O : [B, Hq,  N, d]  bf16 (raw bits, minf_bf16)
 *      K, V : [B, Hkv, N, d]  bf16
 *      LSE  : [B, Hq,  N]     fp32, natural-log log-sum-exp of each row
 *    Query head h reads KV head h / (Hq / Hkv) (grouped-query attention).
 *  - `heads` is a device array of `nh` query-head ids (int32, each in
 *    [0, Hq), no duplicates).  Per-head index arrays are laid out [B, nh, ...]
 *    in the order of that list.  Attention calls write O (and LSE) only for
 *    the listed heads, so calls for different patterns fill disjoint heads of
 *    one O.  Where documented, heads == NULL means all Hq heads (nh = Hq).
 *  - Requirements: N % 128 == 0, d in {64, 128}, Hq % Hkv == 0, B >= 1.  Violations return MINF_ERR_INVALID_ARG or MINF_ERR_UNSUPPORTED
 *    before anything is launched.
 *  - The library allocates no device memory.  Scratch space comes from the
 *    caller's workspace `ws` of `ws_bytes` bytes, sized by
 *    minf_workspace_size(); its first 256 bytes hold a device status word
 *    that kernels set on a device-side error (a bounded wait that ran out,
 *    an index out of range).  Zero the workspace once before first use;
 *    read and clear the status with minf_get_device_status().  The attention
 *    calls also add two work counters there, as uint64 at byte offsets 8 and
 *    16: the 128 x 128 key tiles they executed and the score entries their
 *    masks kept (the useful entries); they are never reset by the library.
 *    The int32 at byte offset 24 is a failure-detection test hook: while it
 *    is non-zero, the first CTA of every attention call withholds its key
 *    tiles, its bounded waits (2 s) run out, and the call's status becomes
 *    MINF_ERR_DEVICE_TIMEOUT without faulting or hanging the GPU.  Keep it
 *    zero in normal use.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream) and returns a host-side status: launch errors
 *    come back as MINF_ERR_CUDA.
 *  - Selection ties go to the lower index; selected index lists are sorted
 *    ascending.  A requested k larger than the number of candidates is
 *    clamped to it.
 */
#ifndef MINF_H
#define MINF_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t minf_bf16; /* raw bfloat16 bits */

typedef enum {
  MINF_OK = 0,
  MINF_ERR_INVALID_ARG = 1,
  MINF_ERR_UNSUPPORTED = 2,
  MINF_ERR_CUDA = 3,
  MINF_ERR_WORKSPACE_TOO_SMALL = 4,
  MINF_ERR_DEVICE_TIMEOUT = 5,   /* a kernel's bounded wait expired; outputs are invalid */
  MINF_ERR_DEVICE_BOUNDS = 6     /* a kernel found an index outside its range; outputs are invalid */
} minf_status;

/* Problem geometry.  scale <= 0 selects the softmax temperature 1/sqrt(d). */
typedef struct {
  int B, Hq, Hkv, N, d;
  float scale;
} minf_shape;

/* Operation ids for minf_workspace_size(). */
enum {
  MINF_OP_ESTIMATE_VS = 0,
  MINF_OP_ESTIMATE_BS = 1,
  MINF_OP_BUILD_INDEX = 2,
  MINF_OP_SPARSE_ATTN_VS = 3,
  MINF_OP_SPARSE_ATTN_BS = 4,
  MINF_OP_ATTN_ASHAPE = 5,
  MINF_OP_DENSE_ATTN = 6
};

/*
 * Compact Vertical-Slash index of nh heads, written by minf_build_index and
 * read by minf_sparse_attn_vs.  All buffers are caller-owned device memory;
 * nb = N / 64, W = minf_vs_wmap_words(N).
 *   grp      [B, nh, k_s, 2] slash groups (a_g, b_g): ascending offsets merged
 *                            while consecutive offsets differ by <= 64
 *   grp_cnt  [B, nh]         number of groups
 *   tgrp     [B, nh, k_s, 2] the same offsets merged while they differ by
 *                            <= 128 (the bands of a 128-row query tile)
 *   tgrp_cnt [B, nh]
 *   wmap     [B, nh, W]      bit x set iff block offset u = x - 63 lies in
 *                            some [a_g - 63, b_g]: key j is on a slash band of
 *                            the query block whose first row is r0 exactly
 *                            when bit (r0 - j + 63) is set
 *   vcnt     [B, nh, nb]     per 64-row query block, the number of vertical
 *                            columns not already covered by a slash band
 *   vidx     [B, nh, nb, k_v] those columns, ascending (j <= last row of the block)
 *   tvcnt    [B, nh, nt]      per 128-row query tile (nt = N / 128, blocks 2t and
 *                            2t + 1), the number of entries of tvidx
 *   tvidx    [B, nh, nt, k_v] the columns the tile gathers, each with its rows:
 *                            key j in bits 0-29, bit 30 set iff block 2t lists
 *                            j, bit 31 iff block 2t + 1 does.  First block
 *                            2t + 1's list in order, then the columns of block
 *                            2t's list that block 2t + 1 does not list.  Every
 *                            column of V appears at most once per tile, so k_v
 *                            entries suffice.  Requires N <= 2^30.
 */
typedef struct {
  int32_t* grp;
  int32_t* grp_cnt;
  int32_t* tgrp;
  int32_t* tgrp_cnt;
  uint32_t* wmap;
  int32_t* vcnt;
  int32_t* vidx;
  int32_t* tvcnt;
  int32_t* tvidx;
} minf_vs_index;

/* Number of 32-bit words of one head's slash-band bitmap (wmap). */
size_t minf_vs_wmap_words(int N);

/*
 * Bytes of workspace that operation `op` needs for this shape, head count and
 * budgets (k_v, k_s, k_b are ignored where the operation has none).  Always at
 * least 256 (the status word).  Returns 0 for an unknown op or a bad shape.
 * MINF_OP_ESTIMATE_BS: the size for the fused selection when k_b allows it,
 * else (k_b = 0 included) for the pooled score matrix.
 */
size_t minf_workspace_size(int op, const minf_shape* shape, int nh, int k_v, int k_s, int k_b);

/*
 * Vertical-Slash index estimation (summary, "Key points": the last query
 * vectors are scored against all keys).  For each listed head and each of
 * the last `last_q` query rows i (1 <= last_q <= 64; the pages' reading is
 * 64), the causal scores s_ij = scale * q_i . k_j (j <= i) are softmax-ed
 * over j in fp32; then
 *     v_j     = sum_i p_ij           (vertical score of key column j)
 *     sigma_o = sum_i p_{i, i-o}     (slash score of diagonal offset o >= 0)
 * v_idx gets the k_v best columns, s_idx the k_s best offsets with offset 0
 * always kept; both ascending.  v_score / s_score ([B, nh, N] fp32) receive
 * the scores when non-NULL.  Outputs: v_idx [B, nh, k_v], s_idx [B, nh, k_s].
 */
minf_status minf_estimate_vs(const minf_shape* shape, const minf_bf16* Q, const minf_bf16* K,
                             const int32_t* heads, int nh, int last_q, int k_v, int k_s,
                             int32_t* v_idx, int32_t* s_idx, float* v_score, float* s_score,
                             void* ws, size_t ws_bytes, void* stream);

/*
 * Allocation-free variant of minf_estimate_vs.  MInference has no counterpart:
 * this exists for callers that cannot allocate device memory where they run
 * the estimation (for example code inside a CUDA-graph capture that forbids
 * allocation, or an engine plugin whose memory was planned up front), so they
 * cannot provide a workspace.  Arguments and results are those of
 * minf_estimate_vs without ws / ws_bytes; the scratch space is a 64 MiB array
 * built into the library, held on every GPU that loads it until the process
 * exits.  Problems that need more scratch than that (minf_workspace_size for
 * MINF_OP_ESTIMATE_VS above 64 MiB, about 3.5M (batch x heads x tokens))
 * are rejected with MINF_ERR_WORKSPACE_TOO_SMALL before anything runs.  The
 * call allocates nothing.  Every call looks up the array's device address
 * (which follows a module reloaded after cudaDeviceReset); the first call on
 * a device loads the library's device code, so make it before any stream
 * capture begins.  All calls share the one array: calls that overlap on the
 * GPU race, so serialise them.  Device-side errors are latched in the
 * array's status word: read them with minf_noalloc_device_status.
 */
minf_status minf_estimate_vs_noalloc(const minf_shape* shape, const minf_bf16* Q, const minf_bf16* K,
                                     const int32_t* heads, int nh, int last_q, int k_v, int k_s,
                                     int32_t* v_idx, int32_t* s_idx, float* v_score, float* s_score,
                                     void* stream);

/*
 * Synchronizes `stream` and returns the device status word of the built-in
 * scratch array of minf_estimate_vs_noalloc (MINF_OK when no kernel reported
 * an error since the last read), then clears it.  Copies to and from host
 * memory only: it allocates nothing.  Not for use during a stream capture.
 */
minf_status minf_noalloc_device_status(void* stream);

/*
 * Block-Sparse index estimation (summary, "Key points": queries and keys are
 * mean-pooled in 64-token blocks).  Pooled means are taken in fp32; per query
 * block b the k_b best key blocks c <= b by the pooled score
 * t[b, c] = scale * Qbar_b . Kbar_c are kept (ties to the lower c), block b
 * itself always.  block must be 64.  Outputs: blk_idx [B, nh, N/64, k_b]
 * ascending, padded with -1; blk_cnt [B, nh, N/64] = min(b + 1, k_b).
 *
 * For d = 128 and k_b <= 128, t is formed on the tensor cores from the means
 * split into three bf16 parts each (six products per K step: fp32
 * accuracy), and each row is selected by one warp from the diagonal down;
 * this needs the workspace minf_workspace_size gives for this k_b.  Otherwise
 * (or with a workspace sized for k_b = 0) t is formed with fp32 FMAs.  Either
 * way t is stored as a [N/64, N/64] matrix per head; blk_score, when
 * non-NULL, receives it as [B, nh, N/64, N/64] (entries with c > b
 * undefined).
 */
minf_status minf_estimate_bs(const minf_shape* shape, const minf_bf16* Q, const minf_bf16* K,
                             const int32_t* heads, int nh, int block, int k_b,
                             int32_t* blk_idx, int32_t* blk_cnt, float* blk_score,
                             void* ws, size_t ws_bytes, void* stream);

/*
 * Vertical-Slash index build: compacts v_idx [B, nh, k_v] and s_idx
 * [B, nh, k_s] (both ascending, as minf_estimate_vs writes them) into the
 * minf_vs_index above.  A slash offset o covers, in a 64-row query block with
 * first row r0, the keys r0 - o .. r0 + 63 - o; verticals already on such a
 * band are dropped from that block's list so that every key is counted once.
 * Unsorted or out-of-range input indices set MINF_ERR_DEVICE_BOUNDS.
 */
minf_status minf_build_index(const minf_shape* shape, int nh, const int32_t* v_idx, int k_v,
                             const int32_t* s_idx, int k_s, const minf_vs_index* idx,
                             void* ws, size_t ws_bytes, void* stream);

/*
 * Vertical-Slash sparse attention (summary, "Summary", stage 3: attention
 * over the estimated indices only).  Row i of query block b attends to the
 * keys j <= i that lie on a slash band of block b or in block b's vertical
 * list; softmax in fp32, P.V in bf16 with fp32 accumulation, on tcgen05
 * tensor cores.  lse may be NULL.
 */
minf_status minf_sparse_attn_vs(const minf_shape* shape, const minf_bf16* Q, const minf_bf16* K,
                                const minf_bf16* V, const int32_t* heads, int nh,
                                const minf_vs_index* idx, int k_v, int k_s,
                                minf_bf16* O, float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * Block-Sparse sparse attention: row i attends to keys j <= i whose 64-key
 * block is listed for i's query block in blk_idx / blk_cnt (as written by
 * minf_estimate_bs).  lse may be NULL.
 */
minf_status minf_sparse_attn_bs(const minf_shape* shape, const minf_bf16* Q, const minf_bf16* K,
                                const minf_bf16* V, const int32_t* heads, int nh,
                                const int32_t* blk_idx, const int32_t* blk_cnt, int k_b,
                                minf_bf16* O, float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * A-shape attention (abstract; summary, "Summary": the A-shape pattern):
 * row i attends to keys j <= i with j < n_sink or i - j < n_local.  lse may be
 * NULL.  n_sink >= 0, n_local >= 1.
 */
minf_status minf_attn_ashape(const minf_shape* shape, const minf_bf16* Q, const minf_bf16* K,
                             const minf_bf16* V, const int32_t* heads, int nh, int n_sink,
                             int n_local, minf_bf16* O, float* lse, void* ws, size_t ws_bytes,
                             void* stream);

/*
 * Dense causal attention (the baseline the pages' speed-ups are measured
 * against; summary, "Key points": the kernels build on FlashAttention), on
 * the same tcgen05 mainloop.  heads may be NULL (all heads).  lse may be NULL.
 */
minf_status minf_dense_attn(const minf_shape* shape, const minf_bf16* Q, const minf_bf16* K,
                            const minf_bf16* V, const int32_t* heads, int nh, minf_bf16* O,
                            float* lse, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Element-exact Vertical-Slash variant.  The slash lines of the summary page
 * ("Key points": vertical and slash lines), read as the diagonals themselves
 * rather than as the 64-key bands they sweep through a 64-row query block:
 * row i attends to the keys j <= i with j in V or i - j in S.  This set is
 * contained in the band set of minf_sparse_attn_vs.
 * ------------------------------------------------------------------------- */
enum { MINF_OP_BUILD_INDEX_EXACT = 7, MINF_OP_SPARSE_ATTN_VS_EXACT = 8 };

/*
 * Index of the exact variant, written by minf_build_index_exact and read by
 * minf_sparse_attn_vs_exact.  Caller-owned device buffers; nt = N / 128,
 * Wb = minf_vs_bits_words(N), Wt = minf_vs_twmap_words(N):
 *   tgrp     [B, nh, k_s, 2] offsets merged while they differ by <= 128; the
 *                            diagonals of group g cross the 128-row query tile
 *                            with first row R in the keys [R - b_g, R + 127 - a_g]
 *   tgrp_cnt [B, nh]
 *   sbits    [B, nh, Wb]     bit o set iff offset o is in S (padding bits zero)
 *   vbits    [B, nh, Wb]     bit j set iff key j is in V (padding bits zero)
 *   twmap    [B, nh, Wt]     bit x set iff x lies in some [a_g, b_g + 127]; key j
 *                            lies in one of the ranges of tile R exactly when
 *                            bit (R + 127 - j) is set
 *   vcnt     [B, nh, nt]     per 128-row query tile, the number of vertical
 *                            columns outside every range of that tile
 *   vidx     [B, nh, nt, k_v] those columns, ascending (j <= R + 127)
 */
typedef struct {
  int32_t* tgrp;
  int32_t* tgrp_cnt;
  uint32_t* sbits;
  uint32_t* vbits;
  uint32_t* twmap;
  int32_t* vcnt;
  int32_t* vidx;
} minf_vs_exact_index;

/* Words of one head's sbits / vbits (N / 32 + 8) and of its twmap. */
size_t minf_vs_bits_words(int N);
size_t minf_vs_twmap_words(int N);

/*
 * Builds minf_vs_exact_index from ascending v_idx [B, nh, k_v] and s_idx
 * [B, nh, k_s] (as minf_estimate_vs writes them).  Unsorted or out-of-range
 * input indices set MINF_ERR_DEVICE_BOUNDS.  N must be a multiple of 128.
 */
minf_status minf_build_index_exact(const minf_shape* shape, int nh, const int32_t* v_idx, int k_v,
                                   const int32_t* s_idx, int k_s, const minf_vs_exact_index* idx,
                                   void* ws, size_t ws_bytes, void* stream);

/*
 * Element-exact Vertical-Slash sparse attention: row i attends to the keys
 * j <= i with j in V or i - j in S (see above).  The key tiles are those of
 * minf_sparse_attn_vs at 128-row granularity (the ranges of the offset groups,
 * then the tile's vertical list); inside a range the membership of each
 * element is read from sbits and vbits.  lse may be NULL.
 */
minf_status minf_sparse_attn_vs_exact(const minf_shape* shape, const minf_bf16* Q, const minf_bf16* K,
                                      const minf_bf16* V, const int32_t* heads, int nh,
                                      const minf_vs_exact_index* idx, int k_v, int k_s, minf_bf16* O,
                                      float* lse, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * One launch for a whole layer of mixed patterns.
 * ------------------------------------------------------------------------- */
enum { MINF_OP_SPARSE_ATTN_LAYER = 9 };

/*
 * Attention of every head of a layer whose heads follow different patterns
 * (summary page, "Summary": a pattern per head, chosen offline; attention over
 * the estimated indices only), in one launch: the Vertical-Slash
 * heads vs_heads[n_vs] with the index vs_idx (as minf_sparse_attn_vs), the
 * Block-Sparse heads bs_heads[n_bs] with blk_idx / blk_cnt (as
 * minf_sparse_attn_bs) and the A-shape heads a_heads[n_a] (as
 * minf_attn_ashape).  Per-head index arrays are laid out [B, n, ...] in the
 * order of their own head list.  Any of the three groups may be empty (n = 0,
 * pointers ignored); the head lists must be disjoint and hold at most Hq
 * heads together.  The results equal those of the three separate calls; the
 * work items of all heads are interleaved heaviest first, so the light
 * Block-Sparse and A-shape heads fill the end of the launch instead of
 * running launches of their own.  lse may be NULL.
 */
minf_status minf_sparse_attn_layer(const minf_shape* shape, const minf_bf16* Q, const minf_bf16* K,
                                   const minf_bf16* V, const int32_t* vs_heads, int n_vs,
                                   const minf_vs_index* vs_idx, int k_v, int k_s, const int32_t* bs_heads,
                                   int n_bs, const int32_t* blk_idx, const int32_t* blk_cnt, int k_b,
                                   const int32_t* a_heads, int n_a, int n_sink, int n_local, minf_bf16* O,
                                   float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * Synchronizes `stream`, returns the device status word of `ws` (MINF_OK when
 * no kernel reported an error since the last call) and clears it.
 */
minf_status minf_get_device_status(void* ws, void* stream);

/*
 * Diagnostic, not part of the method: evaluates on the device the two
 * exponentials the attention softmax uses for P = 2^(s * scale * log2 e - m),
 * for n caller-given arguments x (device arrays of n floats each):
 *   y_poly = the FMA-pipe routine that takes one pair of exponentials in four
 *            (2^x = 2^round(x) * p(x - round(x)) with p the degree-3 minimax
 *            fit of 2^f on [-1/2, 1/2] for relative error, at most 7.5e-5;
 *            arguments below -126 are clamped to -126)
 *   y_mufu = ex2.approx.ftz.f32 (the MUFU unit)
 * so that a caller can check their accuracy on the GPU that runs them.
 * Asynchronous on `stream`.
 */
minf_status minf_selftest_exp2(const float* x, float* y_poly, float* y_mufu, int n, void* stream);

/* Static description of a status code. */
const char* minf_status_string(minf_status s);

/* ---------------------------------------------------------------------------
 * Grid pattern (MMInference abstract: the temporal and spatial locality of
 * video gives a Grid pattern, handled through a permutation).
 * ------------------------------------------------------------------------- */
enum { MINF_OP_ATTN_GRID = 10 };

/*
 * Grid-pattern attention of the listed heads over a video segment of
 * N / frame_tokens frames of frame_tokens tokens each, stored frame-major
 * (token i = f * frame_tokens + p).  Reading (the abstract defines no more):
 * a query attends to keys at its own in-frame position p; the tokens of one
 * position, in frame order, form a sequence of their own, and each such
 * sequence gets the Block-Sparse treatment of minf_estimate_bs and
 * minf_sparse_attn_bs (64-frame mean-pooled blocks, the k_b best key blocks
 * per query block, the diagonal block forced, causal in frame order, which
 * is causal in token order).  Implemented as that permutation: the rows are
 * gathered position-major into the workspace, the two Block-Sparse calls run
 * on the shape (B * frame_tokens, Hq, Hkv, N / frame_tokens, d), and O (and
 * lse) are scattered back to the listed heads' rows.  N / frame_tokens must
 * be a multiple of 128.  blk_idx [B, frame_tokens, nh, N / frame_tokens / 64,
 * k_b] and blk_cnt [B, frame_tokens, nh, N / frame_tokens / 64] receive the
 * per-position selections when non-NULL (the workspace holds them
 * otherwise).  Workspace: minf_workspace_size(MINF_OP_ATTN_GRID, shape, nh,
 * 0, 0, k_b), which covers every frame_tokens.
 */
minf_status minf_attn_grid(const minf_shape* shape, const minf_bf16* Q, const minf_bf16* K, const minf_bf16* V,
                           const int32_t* heads, int nh, int frame_tokens, int k_b, int32_t* blk_idx,
                           int32_t* blk_cnt, minf_bf16* O, float* lse, void* ws, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MINF_H */
