/*
 * lbsa.h -- C ABI of liblbsa, block-sparse self-attention over 3D video token
 * grids on NVIDIA B200 (sm_100a).
 *
 * The path has three stages, each one call below:
 *   1. lbsa_score  -- per (head, query block) block scores: the exact block
 *      attention mass of one dense softmax pass (LoSA abstract, scholarbro.com
 *      author page of C. Sun) or the block-mean proxy (VMoBA review on
 *      pith.science, arXiv 2506.23858, "What carries the argument").
 *   2. lbsa_select -- mass-threshold selection: sort the scores, accumulate,
 *      keep the smallest key-block set whose retained mass reaches p (LoSA
 *      abstract; VMoBA review, circularity check: the least count k' of pairs
 *      whose running sum of normalised similarity gets to tau), per
 *      query-block row (LoSA) or over
 *      all block pairs of a head (VMoBA global selection).  The result is a
 *      blockset that can be frozen and reused by later calls (LoSA abstract:
 *      the frozen block indices are reused for all remaining steps).
 *      Further rules: lbsa_select_rule (Local + TopK; top-p with a per-head
 *      floor), lbsa_select_tokens (per-token pairs), lbsa_select_routed
 *      (entropy-routed cross-head pools).
 *   3. lbsa_attend -- block-sparse flash attention that visits only the kept
 *      key blocks (VMoBA review: attention runs on the true keys and values of
 *      the kept blocks and nothing else).
 * plus lbsa_permute / lbsa_partition_perm for the 1D / 2D / 3D block
 * partitions of the token grid (VMoBA review: layer-wise cyclic 1D-2D-3D
 * partition).
 *
 * Conventions shared by every call
 *   - Pointers named q, k, v, out, scores, lse, perm, x, y are DEVICE pointers
 *     owned by the caller; the library never frees them.  All work is
 *     enqueued on the caller's CUDA stream (`stream`, a cudaStream_t; NULL is
 *     the legacy default stream) and returns without synchronising unless a
 *     function says otherwise.
 *   - A return value is an lbsa_status.  Host-side validation failures return
 *     LBSA_ERR_INVALID_ARG / LBSA_ERR_UNSUPPORTED before anything is launched;
 *     lbsa_last_error() then holds a one-line reason (thread-local).
 *   - Errors found on the device (an out-of-range block index, invalid scores,
 *     a wait that ran out) are recorded in the blockset's device status word
 *     (lbsa_get_status) or in the library's per-device status word
 *     (lbsa_device_status); kernels never trap.
 *   - Tensors are [B, H, rows, d] with d contiguous (stride 1) and element
 *     strides stride_b, stride_h, stride_n given in lbsa_qkv_desc; rows
 *     0..N_valid-1 are tokens in block order (block i = rows i*block ..
 *     i*block+block-1).  A partial last block is allowed: rows >= N_valid are
 *     never read and never written.  Base pointers and the byte sizes of
 *     stride_b, stride_h, stride_n must be multiples of 16.
 */
#ifndef LBSA_H
#define LBSA_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LBSA_OK = 0,
  LBSA_ERR_INVALID_ARG = 1,     /* bad pointer, shape, stride or parameter        */
  LBSA_ERR_UNSUPPORTED = 2,     /* valid but not built (e.g. d not in {64,128})   */
  LBSA_ERR_CUDA = 3,            /* a CUDA runtime/driver call failed               */
  LBSA_ERR_OOM = 4,             /* device allocation failed                        */
  LBSA_ERR_BAD_INDEX = 5,       /* device: a block index outside [0, nB)           */
  LBSA_ERR_INVALID_SCORES = 6,  /* device: a score NaN, negative or >= 2           */
  LBSA_ERR_TIMEOUT = 7          /* device: a bounded wait ran out                  */
} lbsa_status;

typedef enum { LBSA_BF16 = 0, LBSA_F32 = 1 } lbsa_dtype;
typedef enum { LBSA_SCORE_EXACT_MASS = 0, LBSA_SCORE_MEANPOOL = 1, LBSA_SCORE_MEANPOOL_TOKEN = 2 } lbsa_score_mode;
typedef enum { LBSA_SCOPE_ROW = 0, LBSA_SCOPE_HEAD = 1, LBSA_SCOPE_TOKEN = 2, LBSA_SCOPE_ROUTED = 3 } lbsa_scope;
typedef enum {
  LBSA_PART_RASTER = 0,         /* identity                                        */
  LBSA_PART_1D = 1,             /* temporal rows: t fastest                        */
  LBSA_PART_2D = 2,             /* per-frame th x tw spatial tiles                 */
  LBSA_PART_3D = 3              /* tt x th x tw spatio-temporal tiles              */
} lbsa_partition;

typedef struct {
  int32_t B, H;                 /* batch, heads                                    */
  int32_t N_valid;              /* tokens per (batch, head); rows >= N_valid are padding */
  int32_t d;                    /* head dim: 64 or 128                             */
  int32_t dtype;                /* lbsa_dtype of q, k, v and out                   */
  int32_t reserved;
  int64_t stride_b, stride_h, stride_n;   /* element strides; the d stride is 1   */
} lbsa_qkv_desc;

/* Opaque, library-owned selection result: per query-block row r =
 * (b*H + h)*nB + i the ascending list of kept key-block ids, plus a device
 * status word.  Read-only once built; safe to reuse across any number of
 * lbsa_attend calls (the frozen indices of LoSA). */
typedef struct lbsa_blockset lbsa_blockset;

/* Stage 1: block scores.
 * LoSA abstract (exact mass) / VMoBA review "What carries the argument"
 * (block-mean proxy; per-token queries: referee report major comment 1, every
 * query token against every key-block mean).
 *   q, k    [B, H, N_valid, d] per desc (bf16 or fp32)
 *   block   tokens per block, 64 or 128 (same for queries and keys)
 *   mode    LBSA_SCORE_EXACT_MASS: scores[b,h,i,j] = mean over the valid
 *           query rows r of block i of sum over valid keys c of block j of
 *           softmax_c(q_r . k_c / sqrt(d)); every row of a head sums to 1.
 *           LBSA_SCORE_MEANPOOL: qbar_i, kbar_j = means of the valid tokens of
 *           the blocks (fp32), s_ij = qbar_i . kbar_j / sqrt(d),
 *           scores[b,h,:,:] = softmax over all nB*nB pairs of the head.
 *           LBSA_SCORE_MEANPOOL_TOKEN: every valid query token scores the
 *           key-block means, s_rj = q_r . kbar_j / sqrt(d), and
 *           scores[b,h,:,:] = softmax over all N_valid*nB pairs of the head.
 *   scores  out: fp32 [B, H, nB, nB] contiguous, nB = ceil(N_valid / block)
 *           (LBSA_SCORE_MEANPOOL_TOKEN: [B, H, N_valid, nB])
 *   lse     optional out (exact mode only; NULL to skip): fp32 [B, H, N_valid]
 *           contiguous, natural-log log-sum-exp of each query row of the dense
 *           pass.
 * The exact mode is one dense sweep (tensor cores for bf16) that keeps each
 * row's per-chunk log-sum-exp and turns it into masses once the row's lse is
 * known. */
int lbsa_score(const void* q, const void* k, const lbsa_qkv_desc* desc, int32_t block,
               int32_t mode, float* scores, float* lse, void* stream);

/* Stages 1 and 3 fused for a dense step: dense attention that also returns
 * the exact block masses of lbsa_score (LoSA abstract: the masses are measured
 * at one early dense step; that step's attention output is needed anyway).
 * One sweep over the keys: per 64-key chunk each row keeps its chunk
 * log-sum-exp in a strip, the row's lse then turns the strip into masses.
 *   q, k, v  bf16 [B, H, N_valid, d] per desc (fp32 returns LBSA_ERR_UNSUPPORTED)
 *   block    64 or 128 (the mass granularity)
 *   scores   out: fp32 [B, H, nB, nB] contiguous, as lbsa_score (exact mode)
 *   out      out: dense attention output, same dtype and strides as q
 *   lse      optional out: fp32 [B, H, N_valid] natural-log row log-sum-exp
 * Scratch, from the library pool: one slot per SM of 2 x 128 x
 * ceil(N_valid / 64) floats (a strip for each row of the two 128-row query
 * tiles a CTA holds), plus one int32 flag per slot.  nB = ceil(N_valid / block) <= 4096
 * (LBSA_ERR_UNSUPPORTED beyond). */
int lbsa_score_attend(const void* q, const void* k, const void* v, const lbsa_qkv_desc* desc, int32_t block,
                      float* scores, void* out, float* lse, void* stream);

/* Stage 2: mass-threshold selection into a new blockset.
 * LoSA abstract (per head and query block, smallest set meeting the
 * threshold); VMoBA review (global selection over a head; threshold tau;
 * rows may come out empty).
 *   scores  fp32 [B, H, nB, nB] contiguous device array, 0 <= x < 2
 *   block   tokens per block the scores were computed with (64 or 128)
 *   p       threshold in (0, 1]; p = 1 keeps every block (dense)
 *   scope   LBSA_SCOPE_ROW: one decision per (b, h, query block), at least
 *           one block kept per row.  LBSA_SCOPE_HEAD: one decision over the
 *           nB*nB pairs of each (b, h), at least one pair per head; rows may
 *           be empty.
 *   out     receives a new blockset (free with lbsa_free).
 * Rule, exact and order-independent: w = floor(x * 2^32), W = sum w,
 * P = round_half_even(p * 2^24), T = ceil(P * W / 2^24); order by score
 * descending, then flat index ascending; keep the shortest prefix whose sum
 * of w is >= T (at least one element).  A segment holding a NaN, negative or
 * >= 2 score keeps all its blocks and sets LBSA_ERR_INVALID_SCORES in the
 * blockset's status word.  The blockset's device memory is allocated
 * stream-ordered at worst-case size (B*H*nB*(nB+1) int32); no host sync.
 * Limits: nB <= 4096 and B*H*nB < 2^31 (LBSA_ERR_UNSUPPORTED beyond). */
int lbsa_select(const float* scores, int32_t B, int32_t H, int32_t nB, int32_t block, double p,
                int32_t scope, lbsa_blockset** out, void* stream);

/* Stage 2, two further rules of the pages, into a new blockset (row scope).
 *   LBSA_RULE_LOCAL_TOPK  VMoBA review (referee report major comment 2: the
 *       training-free experiments select blocks by "Local + TopK", with
 *       k = 2, 6 or 18).  Row (b, h, i) keeps its own key block i plus the k
 *       top-ranked other key blocks: min(k + 1, nB) blocks.  p, n_valid unused.
 *   LBSA_RULE_TOPP_FLOOR  SCOPE abstract (a per-head Top-k set to the mean
 *       of the key counts the first pass kept, weighted by query-cluster size;
 *       more keys only where a count is below it).  The
 *       LBSA_SCOPE_ROW threshold rule with p gives counts c_i; the head's
 *       floor is K = ceil(sum_i v_i c_i / sum_i v_i) with v_i the valid tokens
 *       of query block i, min(block, n_valid - i * block); row i keeps the
 *       first max(c_i, min(K, nB)) blocks of its ranked order.  k unused.
 * Ranked order: score descending, then key-block id ascending.  nB <= 4096.
 * Invalid scores are handled as by lbsa_select.
 *   n_valid  valid tokens: (nB - 1) * block < n_valid <= nB * block
 *   p        in (0, 1] (LBSA_RULE_TOPP_FLOOR)
 *   k        >= 0 (LBSA_RULE_LOCAL_TOPK)
 *   out      receives a new blockset (free with lbsa_free). */
typedef enum { LBSA_RULE_LOCAL_TOPK = 0, LBSA_RULE_TOPP_FLOOR = 1 } lbsa_rule;
int lbsa_select_rule(const float* scores, int32_t B, int32_t H, int32_t nB, int32_t block, int32_t n_valid,
                     int32_t rule, double p, int32_t k, lbsa_blockset** out, void* stream);

/* Stage 2 at token granularity (VMoBA review: global selection over a head,
 * here over its (query token, key block) pairs, the pairs of the
 * LBSA_SCORE_MEANPOOL_TOKEN scores; threshold tau; tokens may keep nothing).
 *   scores   fp32 [B, H, n_valid, nB] contiguous device array, 0 <= x < 2
 *   n_valid  valid tokens; nB = ceil(n_valid / 64) <= 4096
 *   block    must be 64 (a query block's tokens fit one 64-bit mask)
 *   p        in (0, 1]
 *   out      receives a new blockset (scope LBSA_SCOPE_TOKEN, free with
 *            lbsa_free): query block i lists, ascending, every key block that
 *            at least one of its tokens keeps, each with the 64-bit set of
 *            those tokens (lbsa_blockset_masks); lbsa_attend then lets token
 *            r attend to its own kept blocks only.
 * Rule: as lbsa_select with LBSA_SCOPE_HEAD over the head's n_valid*nB pairs
 * (flat index r*nB + j, exact fixed-point sums, score descending then flat
 * index ascending, at least one pair per head).  Invalid scores keep every
 * pair of the head and set LBSA_ERR_INVALID_SCORES.  Scratch: the radix
 * histograms and per-token tie counts of B*H heads, from the library pool. */
int lbsa_select_tokens(const float* scores, int32_t B, int32_t H, int32_t n_valid, int32_t block, double p,
                       lbsa_blockset** out, void* stream);

/* Stage 2 with entropy-routed competition domains (EG-Sparse abstract,
 * readsearch.ai page of arXiv 2610.14672, "Competition Domains Matter:
 * Selective Head Globalization for Training-Free Sparse Attention in Video
 * Diffusion Transformers": heads whose scores have low entropy select jointly
 * with a group of other heads, the rest per row, from the block scores the
 * path computes anyway).  Into a new blockset (scope LBSA_SCOPE_ROUTED, row lists as
 * LBSA_SCOPE_ROW).
 *   scores   fp32 [B, H, nB, nB] contiguous device array, 0 <= x < 2
 *   block    tokens per block the scores were computed with (64 or 128)
 *   p        threshold in (0, 1]; p = 1 keeps every block
 *   entropy_threshold  head (b, h) is routed when its entropy E < this value
 *            (any non-NaN value; <= 0 routes none, > 1 routes all)
 *   group    >= 1: routed heads of one batch element, in ascending head
 *            order, form consecutive pools of `group` heads (the last may be
 *            smaller); group >= H makes one pool of all routed heads
 *   head_entropy  optional out (NULL to skip): device fp64 [B, H], E of
 *            every head
 *   head_domain   optional out (NULL to skip): device int32 [B, H], -1 for a
 *            head selected per row, else its pool's index within b
 *   out      receives a new blockset (free with lbsa_free).
 * E = (1 / (nB ln nB)) sum_i H_i with H_i = ln S_i - (sum_j x_ij ln x_ij) / S_i,
 * S_i = sum_j x_ij, the entropy of row i's normalised scores (0 ln 0 = 0; a
 * zero row gives 0; nB = 1 gives E = 0), computed from fp32 logarithms in fp64
 * (absolute error a few 1e-7).  Domains: a high-entropy head's row i, or a
 * pool's member rows i, flat index m*nB + j with m the member's rank in the
 * pool.  Every domain takes the lbsa_select rule (exact fixed-point sums,
 * score descending then flat index ascending, at least one pair); a member's
 * row keeps the pairs of the prefix that are its own and may be empty (its
 * attention output is then 0).  A domain holding a NaN, negative or >= 2
 * score keeps every block of its rows and sets LBSA_ERR_INVALID_SCORES (a
 * head with a NaN or negative score has a NaN entropy and is never routed).
 * Scratch: B*H*ceil(nB/8) fp64 partial entropy sums and the domain tables,
 * from the library pool; nB <= 4096, H <= 4096 and B*H <= 65535; a pool's
 * min(group, H) * nB scores must fit 200 KiB of shared memory, else
 * LBSA_ERR_UNSUPPORTED. */
int lbsa_select_routed(const float* scores, int32_t B, int32_t H, int32_t nB, int32_t block, double p,
                       double entropy_threshold, int32_t group, double* head_entropy, int32_t* head_domain,
                       lbsa_blockset** out, void* stream);

/* Stage 3: block-sparse attention over a (frozen) blockset.
 * VMoBA review "What carries the argument" (only selected blocks contribute
 * their key-value pairs); LoSA abstract (frozen indices reused).
 *   q, k, v  [B, H, N_valid, d] per desc; bf16 runs on tcgen05 tensor cores,
 *            fp32 on CUDA cores in true fp32
 *   bs       blockset from lbsa_select (or lbsa_blockset_from_csr) with the
 *            same B, H and nB = ceil(N_valid / block)
 *   out      [B, H, N_valid, d], same dtype and strides as q:
 *            out_r = sum_{c in K_i} softmax_{c in K_i}(q_r . k_c / sqrt(d)) v_c
 *            where K_i are the valid keys of the kept blocks of r's block
 *            (per-token blockset: of the blocks that token r itself keeps).
 *            A row whose list is empty gets 0.
 *   lse      optional fp32 [B, H, N_valid] (natural log; -inf for empty rows).
 * An out-of-range block id in bs is skipped and flags LBSA_ERR_BAD_INDEX in
 * bs's status word. */
int lbsa_attend(const void* q, const void* k, const void* v, const lbsa_qkv_desc* desc,
                const lbsa_blockset* bs, void* out, float* lse, void* stream);

/* Release a blockset (stream-ordered on the stream it was created on).  NULL is a no-op. */
void lbsa_free(lbsa_blockset* bs);

/* Describe a blockset: any output pointer may be NULL. */
int lbsa_blockset_info(const lbsa_blockset* bs, int32_t* B, int32_t* H, int32_t* nB,
                       int32_t* block, int32_t* scope);

/* Device views of the blockset's storage (read-only; valid until lbsa_free):
 * counts[r] = kept blocks of row r (R = B*H*nB rows); cols[r*nB + t], t <
 * counts[r], ascending key-block ids. */
int lbsa_blockset_views(const lbsa_blockset* bs, const int32_t** counts, const int32_t** cols);

/* Device view of a per-token blockset's token sets (read-only; valid until
 * lbsa_free): masks[r*nB + t], t < counts[r], bit u set when token
 * i*64 + u of query block i keeps the t-th listed key block.  *masks is NULL
 * for blocksets of the other scopes. */
int lbsa_blockset_masks(const lbsa_blockset* bs, const uint64_t** masks);

/* Compact CSR export (a helper, not on the per-call path).  row_ptr: device
 * int32 [R + 1]; col: device int32 with room for R*nB entries; *nnz (host)
 * receives the total.  Synchronises the stream. */
int lbsa_blockset_export(const lbsa_blockset* bs, int32_t* row_ptr, int32_t* col, int64_t* nnz,
                         void* stream);

/* Build a blockset from a caller CSR (device int32 row_ptr [R+1], col [nnz];
 * lists must be ascending), e.g. frozen indices saved by an earlier run.
 * Copies the data; ids are validated on the device (status word).  row_ptr
 * must be a valid CSR offset array (row_ptr[0] = 0, non-decreasing, row_ptr[R]
 * <= the length of col): the copy reads col through it unchecked, and a row
 * longer than nB is rejected (LBSA_ERR_BAD_INDEX, row left empty). */
int lbsa_blockset_from_csr(const int32_t* row_ptr, const int32_t* col, int32_t B, int32_t H,
                           int32_t nB, int32_t block, lbsa_blockset** out, void* stream);

/* Block bitmask export (the next-row fused dense step's companion format;
 * ScalingAttention abstract on the mlsift.com sparse-attention listing: a
 * bit-wise block-sparse mask drives its kernel).  bits: device uint32
 * [R][W], W = ceil(nB / 32), R = B*H*nB rows as in the blockset; bit (j % 32)
 * of word j / 32 of row r is set when key block j is kept for row r.  The
 * caller owns bits.  Asynchronous on `stream`.  Per-token blocksets (whose
 * entries carry token sets) return LBSA_ERR_UNSUPPORTED. */
int lbsa_blockset_export_bitmask(const lbsa_blockset* bs, uint32_t* bits, void* stream);

/* Build a blockset from a block bitmask in the layout above (device uint32
 * [B*H*nB][ceil(nB/32)]), e.g. a static prior mask computed offline.  Copies
 * the data; the kept ids of each row come out ascending.  Bits past nB in a
 * row's last word are ignored and raise LBSA_ERR_BAD_INDEX in the status
 * word. */
int lbsa_blockset_from_bitmask(const uint32_t* bits, int32_t B, int32_t H, int32_t nB, int32_t block,
                               lbsa_blockset** out, void* stream);

/* Read (and with clear != 0 reset) the blockset's device status word: 0 or an
 * lbsa_status of the first device error.  Synchronises the stream. */
int lbsa_get_status(const lbsa_blockset* bs, int32_t* device_status, int32_t clear, void* stream);

/* Per-device status word of calls that have no blockset (lbsa_score,
 * lbsa_permute).  Synchronises the stream. */
int lbsa_device_status(int32_t* device_status, int32_t clear, void* stream);

/* Token order of a (T, Hg, Wg) grid for one block partition (VMoBA review:
 * 1D-2D-3D partition; raster index (t*Hg + h)*Wg + w):
 *   blocked[slot] = raster[perm[slot]], slot in [0, T*Hg*Wg).
 * LBSA_PART_1D: t fastest.  LBSA_PART_2D: per frame, th x tw tiles in raster
 * tile order, raster inside a tile.  LBSA_PART_3D: tt x th x tw tiles in
 * raster tile order, raster inside a tile.  Edge tiles are truncated.
 * on_device != 0: perm is a device pointer, filled by a kernel on stream;
 * otherwise a host pointer, filled synchronously on the CPU. */
int lbsa_partition_perm(int32_t T, int32_t Hg, int32_t Wg, int32_t kind, int32_t tt, int32_t th,
                        int32_t tw, int32_t* perm, int32_t on_device, void* stream);

/* Row gather / scatter of up to 3 tensors that share desc and perm:
 *   inverse == 0:  ys[t][b,h,slot,:] = xs[t][b,h,perm[slot],:]
 *   inverse != 0:  ys[t][b,h,perm[slot],:] = xs[t][b,h,slot,:]
 * for slot < desc->N_valid; perm (device int32 [N_valid]) must be a
 * permutation of [0, N_valid).  An entry outside [0, N_valid) skips its row
 * and records LBSA_ERR_BAD_INDEX in the per-device status word
 * (lbsa_device_status); a repeated entry leaves rows unwritten (gather) or
 * written twice (scatter).  x and y may not alias. */
int lbsa_permute(const void* const* xs, void* const* ys, int32_t count, const int32_t* perm,
                 const lbsa_qkv_desc* desc, int32_t inverse, void* stream);

/* Self-test of the bounded-wait machinery: one kernel waits on an mbarrier
 * that nothing completes, gives up after `limit_us` microseconds of wall time
 * (the same check every device wait of the library makes, with a 2 s limit)
 * and writes LBSA_ERR_TIMEOUT to *device_out (device int32).  Never hangs. */
int lbsa_selftest_wait(int64_t limit_us, int32_t* device_out, void* stream);

/* Self-test of the FMA-pipe exponential the exact scorer uses for a quarter
 * of its exponentials: out[i] = 2^v[i] for n device floats v[i] <= 0, by
 * round-to-nearest range reduction and a degree-4 polynomial on [-1/2, 1/2]
 * (relative error below 3e-6 for v in [-125, 0]; inputs below -125 give
 * 2^-125).  v and out are device float arrays of n elements (n >= 0); they
 * may alias.  Returns LBSA_ERR_INVALID_ARG on a NULL pointer with n > 0. */
int lbsa_selftest_exp2(const float* v, float* out, int64_t n, void* stream);

/* Head-scope selection that allocates nothing (the pages have no
 * counterpart).  It serves callers that cannot call cudaMalloc: a host
 * framework whose own caching allocator owns the device's memory (a
 * cudaMalloc behind its back can fail once that pool has grown to the
 * device's capacity), or a latency-bound serving loop that cannot accept the
 * device-wide synchronisation a cudaMalloc may bring.  Same rule and results
 * as lbsa_select(..., LBSA_SCOPE_HEAD, ...), written to caller buffers:
 *   counts  device int32 [B*H*nB]: kept key blocks of row r = (b*H + h)*nB + i
 *   cols    device int32 [B*H*nB*nB]: row r's ascending ids at cols[r*nB ...]
 *   status  device int32 [1]: set to 0, then to the first device error
 * Its scratch (radix histograms, per-head state, tie counts) lives in a
 * 1 MiB file-scope device array that every GPU loading the library holds
 * until the process exits; B*H <= 64 heads with nB <= 1024 always fit, larger
 * sizes return LBSA_ERR_UNSUPPORTED with no launch.  The first call on a
 * device looks up the array's device address (cudaGetSymbolAddress), so make
 * that first call before any stream capture.  All calls on one GPU share that
 * GPU's array and clear what they need at the start: calls that overlap on
 * the same GPU (e.g. issued to different streams) race on it and must be
 * serialised by the caller. */
int lbsa_select_head_noalloc(const float* scores, int32_t B, int32_t H, int32_t nB, double p,
                             int32_t* counts, int32_t* cols, int32_t* status, void* stream);

/* Thread-local one-line reason for the last non-OK return of this thread.
 * With the environment variable LBSA_LOG set (to anything but "" or "0") when
 * the library first checks it, every entry point and every non-OK return
 * also writes one line to stderr ("[lbsa] ..."): arguments, shapes, reasons. */
const char* lbsa_last_error(void);

/* Library ABI version (major * 100 + minor). */
int lbsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LBSA_H */
