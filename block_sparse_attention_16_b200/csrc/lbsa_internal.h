// Internal declarations shared by the C ABI layer and the kernel files.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "lbsa.h"   // include/ is on the include path

// Library-owned selection result.  Row r = (b*H + h)*nB + i owns the slot
// cols[r*nB .. r*nB + nB); counts[r] entries of it are valid, ascending.
struct lbsa_blockset {
  int32_t B, H, nB, block, scope;
  double p;
  int32_t* counts;      // device [R]
  int32_t* cols;        // device [R * nB]
  uint64_t* masks;      // device [R * nB] or NULL: per-token scope, bit t = token t of the query block keeps the entry
  int32_t* status;      // device [1]
  void* base;           // single stream-ordered allocation holding the three arrays
  cudaStream_t stream;  // stream it was created on (freed on it)
  int device;
};

namespace lbsa {

constexpr long long kDefaultWaitLimit = 2000000000ll;   // ns a device wait may take before it gives up (2 s)

struct AttendArgs {
  int B, H, N_valid, d, block, nB;
  const int32_t* counts;
  const int32_t* cols;
  int32_t* status;
  void* out;
  int64_t ostride_b, ostride_h, ostride_n;   // elements
  float* lse;
  long long wait_limit;
  // fused dense step only (launch_score_attend_pp_bf16): exact block masses out
  float* scores;          // [B, H, nB, nB]
  float* fscratch;        // n_slots * 2 * 128 * n_chunks floats: per-CTA strips
  int32_t* slots;         // n_slots flags, zero at launch
  int n_slots;
  // per-token scope (64-token blocks): masks[row * nB + t] is the 64-bit set of
  // the query block's tokens that keep its t-th listed key block; NULL otherwise
  const uint64_t* masks = nullptr;
};

struct ScoreArgs {
  int B, H, N_valid, d, block, nB;
  float* scores;
  float* lse;
  int32_t* status;
  long long wait_limit;
  float* scratch;       // bf16 exact mode: score_exact_bf16_workspace_bytes() of scratch
};

// bf16 tcgen05 kernels (attend_tc.cu, score_tc.cu)
cudaError_t launch_attend_bf16(const CUtensorMap* tq, const CUtensorMap* tk, const CUtensorMap* tv,
                               const AttendArgs& a, cudaStream_t s);
// two query tiles per CTA in ping-pong, 128-key steps (attend_pp.cu): any blockset
// without per-token masks (lbsa_attend gives it the dense ones); the Q map's box is
// 128 rows, the K and V maps' 64 rows
bool attend_pp_supported(const AttendArgs& a);
cudaError_t launch_attend_pp_bf16(const CUtensorMap* tq, const CUtensorMap* tk, const CUtensorMap* tv,
                                  const AttendArgs& a, cudaStream_t s);
// the fused dense step on the two-tile kernel: dense attention and the exact block
// masses (a.scores); workspace: n_slots int32 flags (flag_bytes, 256-aligned), then
// per slot 2 x 128 x ceil(N_valid / 64) floats of strips
size_t score_attend_pp_workspace_bytes(int N_valid, int* n_slots, size_t* flag_bytes);
cudaError_t launch_score_attend_pp_bf16(const CUtensorMap* tq, const CUtensorMap* tk, const CUtensorMap* tv,
                                        const AttendArgs& a, cudaStream_t s);
cudaError_t launch_score_exact_bf16(const CUtensorMap* tq, const CUtensorMap* tk, const ScoreArgs& a,
                                    cudaStream_t s);
size_t score_exact_bf16_workspace_bytes(int B, int H, int N_valid);
int score_exact_bf16_key_rows();   // rows of the K tensor map box the exact scorer loads per step

// fp32 SIMT kernels (simt_f32.cu)
cudaError_t launch_attend_f32(const float* q, const float* k, const float* v, const lbsa_qkv_desc& d,
                              const AttendArgs& a, cudaStream_t s);
cudaError_t launch_score_exact_f32(const float* q, const float* k, const lbsa_qkv_desc& d,
                                   const ScoreArgs& a, cudaStream_t s);

// block-mean proxy (meanpool.cu); workspace holds 2*B*H*nB*d floats + partials
// nQ: rows of the score matrix, nB (query-block means) or n_valid (query tokens)
// Per-token proxy logits on the tensor cores (token_logits_tc.cu).
struct TokenLogitsArgs {
  int G, H, nQ, nB, d;
  float scale;            // 1 / sqrt(d)
  float* scores;          // [G][nQ][nB] fp32 logits out
  float2* part;           // [G][token_logits_parts(nQ, nB)] (max, sum of exp) per 32 tokens and 128 key blocks
  int32_t* status;
  long long wait_limit;
  int cpi = 0;            // 128-column chunks a work item takes (set by the launcher)
};
int token_logits_parts(int nQ, int nB);
// tq: bf16 Q as lbsa_attend's Q map (box 64 x 128); tkb: the hi / lo terms as a 4D
// bf16 map (d, nB, G, 2) with box 64 x 128 x 1 x 1, 128-byte swizzle
// ts: the logits [G][nQ][nB] as a 3D fp32 map (nB, nQ, G), box 32 x 128 x 1, or NULL
// (direct stores; required when nB is not a multiple of 4)
// q_split: tq is instead the query-block means' hi / lo terms as a 4D bf16 map
// (d, nQ, G, 2) like tkb (the block-mean proxy); then ts must be given
cudaError_t launch_token_logits_bf16(const CUtensorMap* tq, const CUtensorMap* tkb, const CUtensorMap* ts,
                                     const TokenLogitsArgs& a, cudaStream_t s, bool q_split = false);
size_t meanpool_workspace_bytes(int B, int H, int nB, int d, int nQ);
// where, in the mean-pool workspace, the per-token path keeps the bf16 hi / lo
// terms of the key-block means (2 x G x nB x d bf16)
void* meanpool_split_ptr(void* ws);
// the block-mean proxy's hi / lo terms of the query-block and key-block means
// (each 2 x G x nB x d bf16), after the fp32 means and the partials
void meanpool_block_split_ptrs(void* ws, int B, int H, int nB, int d, void** qs, void** ks);
// tq / tkb: non-NULL for bf16 per-token mode, which then takes the tensor-core logits
cudaError_t launch_meanpool(const void* q, const void* k, const lbsa_qkv_desc& d, int block, int nB, bool tokens,
                            float* scores, void* ws, cudaStream_t s, const CUtensorMap* tq = nullptr,
                            const CUtensorMap* tkb = nullptr, int32_t* status = nullptr, long long wait_limit = 0,
                            const CUtensorMap* ts = nullptr, const CUtensorMap* tqs = nullptr);

// selection (select.cu)
cudaError_t launch_select_row(const float* scores, int R, int nB, double p, lbsa_blockset* bs,
                              cudaStream_t s);
cudaError_t launch_select_rank(const float* scores, int R, int nB, int mode, int k, const int32_t* head_floor,
                               lbsa_blockset* bs, cudaStream_t s);
cudaError_t launch_head_floor(const int32_t* counts, int G, int nB, int block, int n_valid, int32_t* head_floor,
                              cudaStream_t s);
// nQ: rows of each head's pairs (nB query blocks, or n_valid query tokens); 0 means nB
size_t select_head_workspace_bytes(int B, int H, int nB, int nQ = 0);
// block-scope head selection runs as one cluster launch without workspace for
// heads whose nB x nB scores fit the cluster's shared memory
bool select_head_one_launch(int nB);
cudaError_t launch_select_head(const float* scores, int B, int H, int nB, double p, lbsa_blockset* bs,
                               void* workspace, cudaStream_t s);
// per-token scope: nQ = n_valid token rows of nB key blocks, 64-token blocks; writes
// bs->counts / cols / masks per query block
cudaError_t launch_select_tokens(const float* scores, int B, int H, int nQ, int nB, double p, lbsa_blockset* bs,
                                 void* workspace, cudaStream_t s);
cudaError_t launch_export_csr(const lbsa_blockset* bs, int32_t* row_ptr, int32_t* col,
                              int32_t* nnz_dev, cudaStream_t s);
cudaError_t launch_export_bitmask(const lbsa_blockset* bs, uint32_t* bits, cudaStream_t s);
cudaError_t launch_from_bitmask(const uint32_t* bits, lbsa_blockset* bs, cudaStream_t s);
cudaError_t launch_from_csr(const int32_t* row_ptr, const int32_t* col, lbsa_blockset* bs,
                            cudaStream_t s);

// permutation (permute.cu)
void partition_perm_host(int T, int Hg, int Wg, int kind, int tt, int th, int tw, int32_t* perm);
cudaError_t launch_partition_perm(int T, int Hg, int Wg, int kind, int tt, int th, int tw,
                                  int32_t* perm, cudaStream_t s);
cudaError_t launch_permute(const void* const* xs, void* const* ys, int count, const int32_t* perm,
                           const lbsa_qkv_desc& d, int inverse, int32_t* status, cudaStream_t s);

cudaError_t launch_selftest_wait(long long limit_ns, int32_t* out, cudaStream_t s);
cudaError_t launch_selftest_exp2(const float* v, float* out, long long n, cudaStream_t s);

// Records `msg` as this thread's lbsa_last_error() text and returns `code`.
int set_error(int code, const char* msg);

}  // namespace lbsa
