// C ABI of liblbsa: argument validation, TMA tensor maps, blockset ownership,
// status words, and dispatch to the kernels.  No torch types cross this
// boundary: plain pointers, sizes and a cudaStream_t passed as void*.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include <cudaTypedefs.h>

#include "lbsa_device.cuh"
#include "lbsa_routed.h"

namespace {

thread_local std::string g_err;

// Host-side call log: with LBSA_LOG set to a non-empty value other than "0",
// every entry point and every non-OK return writes one line to stderr.
bool log_on() {
  static const bool on = [] {
    const char* v = std::getenv("LBSA_LOG");
    return v && *v && std::strcmp(v, "0") != 0;
  }();
  return on;
}
void log_line(const char* fmt, ...) {
  if (!log_on()) return;
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  std::fprintf(stderr, "[lbsa] %s\n", buf);
}

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  log_line("error %d: %s", code, buf);
  return code;
}

int cuda_fail(cudaError_t e, const char* where) {
  return fail(e == cudaErrorMemoryAllocation ? LBSA_ERR_OOM : LBSA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int validate_desc(const lbsa_qkv_desc* d) {
  if (!d) return fail(LBSA_ERR_INVALID_ARG, "desc is NULL");
  if (d->B < 1 || d->H < 1 || d->N_valid < 1)
    return fail(LBSA_ERR_INVALID_ARG, "B, H and N_valid must be >= 1 (got %d, %d, %d)", d->B, d->H, d->N_valid);
  if (d->dtype != LBSA_BF16 && d->dtype != LBSA_F32) return fail(LBSA_ERR_INVALID_ARG, "dtype %d unknown", d->dtype);
  if (d->d != 64 && d->d != 128) return fail(LBSA_ERR_UNSUPPORTED, "head dim %d: only 64 and 128 are built", d->d);
  const int es = d->dtype == LBSA_BF16 ? 2 : 4;
  if (d->stride_n < d->d || d->stride_h < 1 || d->stride_b < 1)
    return fail(LBSA_ERR_INVALID_ARG, "strides (%lld, %lld, %lld) smaller than a row", (long long)d->stride_b,
                (long long)d->stride_h, (long long)d->stride_n);
  if ((d->stride_n * es) % 16 || (d->stride_h * es) % 16 || (d->stride_b * es) % 16)
    return fail(LBSA_ERR_INVALID_ARG, "byte strides must be multiples of 16");
  if (static_cast<long long>(d->N_valid) >= (1ll << 31)) return fail(LBSA_ERR_INVALID_ARG, "N_valid too large");
  return LBSA_OK;
}

int validate_ptr(const void* p, const char* name) {
  if (!p) return fail(LBSA_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned16(p)) return fail(LBSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return LBSA_OK;
}

int n_blocks(int n_valid, int block) { return static_cast<int>((static_cast<long long>(n_valid) + block - 1) / block); }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// bf16 [B, H, N_valid, d] as a 4D tensor map (d, N, H, B); box = 64 x box_rows,
// 128-byte swizzle (each box row is one 128-byte swizzle line).
int make_tmap(CUtensorMap* map, const void* ptr, const lbsa_qkv_desc* d, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(LBSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d->d), static_cast<cuuint64_t>(d->N_valid),
                        static_cast<cuuint64_t>(d->H), static_cast<cuuint64_t>(d->B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(d->stride_n) * 2, static_cast<cuuint64_t>(d->stride_h) * 2,
                           static_cast<cuuint64_t>(d->stride_b) * 2};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(box_rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LBSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return LBSA_OK;
}

// A dense bf16 [n3][n2][n1][n0] array (n0 innermost, contiguous) as a 4D tensor
// map with box 64 x box_rows x 1 x 1 and 128-byte swizzle.
int make_tmap_4d(CUtensorMap* map, const void* ptr, long long n0, long long n1, long long n2, long long n3,
                 int box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(LBSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(n0), static_cast<cuuint64_t>(n1), static_cast<cuuint64_t>(n2),
                        static_cast<cuuint64_t>(n3)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(n0) * 2, static_cast<cuuint64_t>(n0 * n1) * 2,
                           static_cast<cuuint64_t>(n0 * n1 * n2) * 2};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(box_rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LBSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return LBSA_OK;
}

// A dense fp32 [n2][n1][n0] array as a 3D tensor map with box 32 x box_rows x 1
// (one 128-byte swizzle line a box row); n0 * 4 must be a multiple of 16.
int make_tmap_f32_3d(CUtensorMap* map, void* ptr, long long n0, long long n1, long long n2, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(LBSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(n0), static_cast<cuuint64_t>(n1), static_cast<cuuint64_t>(n2)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(n0) * 4, static_cast<cuuint64_t>(n0 * n1) * 4};
  cuuint32_t box[3] = {32, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, ptr, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LBSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return LBSA_OK;
}

// Per-device state: a status word for calls without a blockset, and a memory
// pool that serves blocksets and per-call scratch stream-ordered
// (cudaMallocFromPoolAsync / cudaFreeAsync).  The pool keeps freed memory
// cached, so after the first call of a given size nothing reaches the driver.
struct DeviceState {
  int32_t* status = nullptr;
  cudaMemPool_t pool = nullptr;
};
std::mutex g_mu;
DeviceState g_dev[64];

int device_state(DeviceState** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(LBSA_ERR_UNSUPPORTED, "device %d", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState& s = g_dev[dev];
  if (!s.pool) {
    cudaMemPoolProps props{};
    props.allocType = cudaMemAllocationTypePinned;
    props.handleTypes = cudaMemHandleTypeNone;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    e = cudaMemPoolCreate(&s.pool, &props);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemPoolCreate");
    uint64_t keep = ~0ull;
    cudaMemPoolSetAttribute(s.pool, cudaMemPoolAttrReleaseThreshold, &keep);
  }
  if (!s.status) {
    e = cudaMalloc(&s.status, sizeof(int32_t));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(status)");
    e = cudaMemset(s.status, 0, sizeof(int32_t));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(status)");
  }
  *out = &s;
  return LBSA_OK;
}

// Stream-ordered scratch for one call: freed on the same stream after the
// call's kernels, so concurrent calls on different streams never share it.
struct Scratch {
  void* ptr = nullptr;
  cudaStream_t s = nullptr;
  ~Scratch() {
    if (ptr) cudaFreeAsync(ptr, s);
  }
};

int scratch_alloc(DeviceState* ds, size_t bytes, cudaStream_t s, Scratch* out) {
  cudaError_t e = cudaMallocFromPoolAsync(&out->ptr, bytes, ds->pool, s);
  if (e != cudaSuccess) {
    out->ptr = nullptr;
    return cuda_fail(e, "cudaMallocFromPoolAsync(scratch)");
  }
  out->s = s;
  return LBSA_OK;
}

long long wait_limit() { return lbsa::kDefaultWaitLimit; }

int new_blockset(int B, int H, int nB, int block, int scope, double p, cudaStream_t s, lbsa_blockset** out) {
  // the kernels take the row count as an int
  if (static_cast<long long>(B) * H * nB > 2147483647ll)
    return fail(LBSA_ERR_UNSUPPORTED, "B*H*nB = %lld rows exceed 2^31 - 1", static_cast<long long>(B) * H * nB);
  const size_t R = static_cast<size_t>(B) * H * nB;
  const size_t cols_bytes = ((R * nB * sizeof(int32_t)) + 255) & ~size_t(255);
  const size_t counts_bytes = ((R * sizeof(int32_t)) + 255) & ~size_t(255);
  const size_t mask_bytes = (scope == LBSA_SCOPE_TOKEN) ? R * nB * sizeof(uint64_t) : 0;   // per-token scope only
  const size_t bytes = counts_bytes + cols_bytes + 256 + mask_bytes;
  void* base = nullptr;
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != LBSA_OK) return rc;
  cudaError_t e = cudaMallocFromPoolAsync(&base, bytes, ds->pool, s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMallocFromPoolAsync(blockset)");
  auto* bs = new lbsa_blockset;
  bs->B = B;
  bs->H = H;
  bs->nB = nB;
  bs->block = block;
  bs->scope = scope;
  bs->p = p;
  bs->base = base;
  bs->counts = static_cast<int32_t*>(base);
  bs->cols = reinterpret_cast<int32_t*>(static_cast<char*>(base) + counts_bytes);
  bs->status = reinterpret_cast<int32_t*>(static_cast<char*>(base) + counts_bytes + cols_bytes);
  bs->masks = mask_bytes ? reinterpret_cast<uint64_t*>(static_cast<char*>(base) + counts_bytes + cols_bytes + 256)
                         : nullptr;
  bs->stream = s;
  cudaGetDevice(&bs->device);
  e = cudaMemsetAsync(bs->status, 0, sizeof(int32_t), s);
  if (e != cudaSuccess) {
    cudaFreeAsync(base, s);
    delete bs;
    return cuda_fail(e, "cudaMemsetAsync");
  }
  *out = bs;
  return LBSA_OK;
}

}  // namespace

extern "C" {

int lbsa_version(void) { return 101; }

const char* lbsa_last_error(void) { return g_err.c_str(); }

int lbsa_score(const void* q, const void* k, const lbsa_qkv_desc* desc, int32_t block, int32_t mode, float* scores,
               float* lse, void* stream) {
  int rc;
  if (desc)
    log_line("lbsa_score mode=%d B=%d H=%d N=%d d=%d dtype=%d block=%d lse=%d", mode, desc->B, desc->H, desc->N_valid,
             desc->d, desc->dtype, block, lse != nullptr);
  if ((rc = validate_desc(desc)) != LBSA_OK) return rc;
  if ((rc = validate_ptr(q, "q")) != LBSA_OK) return rc;
  if ((rc = validate_ptr(k, "k")) != LBSA_OK) return rc;
  if ((rc = validate_ptr(scores, "scores")) != LBSA_OK) return rc;
  if (block != 64 && block != 128) return fail(LBSA_ERR_UNSUPPORTED, "block %d: only 64 and 128 are built", block);
  if (mode != LBSA_SCORE_EXACT_MASS && mode != LBSA_SCORE_MEANPOOL && mode != LBSA_SCORE_MEANPOOL_TOKEN)
    return fail(LBSA_ERR_INVALID_ARG, "mode %d", mode);
  if (lse && mode != LBSA_SCORE_EXACT_MASS) return fail(LBSA_ERR_INVALID_ARG, "lse is only produced in exact mode");
  const int nB = n_blocks(desc->N_valid, block);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DeviceState* ds = nullptr;
  if ((rc = device_state(&ds)) != LBSA_OK) return rc;
  cudaError_t e;
  Scratch ws;
  if (mode == LBSA_SCORE_EXACT_MASS) {
    lbsa::ScoreArgs a{desc->B, desc->H, desc->N_valid, desc->d, block, nB, scores, lse, ds->status, wait_limit(),
                      nullptr};
    if (desc->dtype == LBSA_BF16) {
      CUtensorMap tq, tk;
      if ((rc = make_tmap(&tq, q, desc, 128)) != LBSA_OK) return rc;
      if ((rc = make_tmap(&tk, k, desc, lbsa::score_exact_bf16_key_rows())) != LBSA_OK) return rc;
      if ((rc = scratch_alloc(ds, lbsa::score_exact_bf16_workspace_bytes(desc->B, desc->H, desc->N_valid), s, &ws)) !=
          LBSA_OK)
        return rc;
      a.scratch = static_cast<float*>(ws.ptr);
      e = lbsa::launch_score_exact_bf16(&tq, &tk, a, s);
    } else {
      e = lbsa::launch_score_exact_f32(static_cast<const float*>(q), static_cast<const float*>(k), *desc, a, s);
    }
  } else {
    const bool tokens = mode == LBSA_SCORE_MEANPOOL_TOKEN;
    const int nQ = tokens ? desc->N_valid : nB;
    if ((rc = scratch_alloc(ds, lbsa::meanpool_workspace_bytes(desc->B, desc->H, nB, desc->d, nQ), s, &ws)) != LBSA_OK)
      return rc;
    if (tokens && desc->dtype == LBSA_BF16) {
      // the logits on the tensor cores: Q as the attention reads it, and the bf16
      // hi / lo terms of the key-block means as a (d, nB, G, 2) map
      CUtensorMap tq, tkb;
      if ((rc = make_tmap(&tq, q, desc, 128)) != LBSA_OK) return rc;
      const long long G = static_cast<long long>(desc->B) * desc->H;
      if ((rc = make_tmap_4d(&tkb, lbsa::meanpool_split_ptr(ws.ptr), desc->d, nB, G, 2, 128)) != LBSA_OK) return rc;
      // the logits leave through TMA stores when a score row is a whole number of 16-byte units
      CUtensorMap ts;
      const bool tma_out = (nB % 4) == 0;
      if (tma_out && (rc = make_tmap_f32_3d(&ts, scores, nB, nQ, G, 128)) != LBSA_OK) return rc;
      e = lbsa::launch_meanpool(q, k, *desc, block, nB, tokens, scores, ws.ptr, s, &tq, &tkb, ds->status,
                                wait_limit(), tma_out ? &ts : nullptr);
    } else if (!tokens && desc->dtype == LBSA_BF16 && nB % 4 == 0) {
      // the block-mean logits on the tensor cores: both means as bf16 hi / lo terms
      const long long G = static_cast<long long>(desc->B) * desc->H;
      void *qs, *ks;
      lbsa::meanpool_block_split_ptrs(ws.ptr, desc->B, desc->H, nB, desc->d, &qs, &ks);
      CUtensorMap tqs, tks, ts;
      if ((rc = make_tmap_4d(&tqs, qs, desc->d, nB, G, 2, 128)) != LBSA_OK) return rc;
      if ((rc = make_tmap_4d(&tks, ks, desc->d, nB, G, 2, 128)) != LBSA_OK) return rc;
      if ((rc = make_tmap_f32_3d(&ts, scores, nB, nB, G, 128)) != LBSA_OK) return rc;
      e = lbsa::launch_meanpool(q, k, *desc, block, nB, tokens, scores, ws.ptr, s, nullptr, &tks, ds->status,
                                wait_limit(), &ts, &tqs);
    } else {
      e = lbsa::launch_meanpool(q, k, *desc, block, nB, tokens, scores, ws.ptr, s);
    }
  }
  if (e != cudaSuccess) return cuda_fail(e, "lbsa_score launch");
  return LBSA_OK;
}

int lbsa_score_attend(const void* q, const void* k, const void* v, const lbsa_qkv_desc* desc, int32_t block,
                      float* scores, void* out, float* lse, void* stream) {
  int rc;
  if (desc)
    log_line("lbsa_score_attend B=%d H=%d N=%d d=%d dtype=%d block=%d lse=%d", desc->B, desc->H, desc->N_valid,
             desc->d, desc->dtype, block, lse != nullptr);
  if ((rc = validate_desc(desc)) != LBSA_OK) return rc;
  if ((rc = validate_ptr(q, "q")) != LBSA_OK) return rc;
  if ((rc = validate_ptr(k, "k")) != LBSA_OK) return rc;
  if ((rc = validate_ptr(v, "v")) != LBSA_OK) return rc;
  if ((rc = validate_ptr(scores, "scores")) != LBSA_OK) return rc;
  if ((rc = validate_ptr(out, "out")) != LBSA_OK) return rc;
  if (block != 64 && block != 128) return fail(LBSA_ERR_UNSUPPORTED, "block %d: only 64 and 128 are built", block);
  if (desc->dtype != LBSA_BF16) return fail(LBSA_ERR_UNSUPPORTED, "the fused dense step is built for bf16");
  const int nB = n_blocks(desc->N_valid, block);
  if (nB > 4096) return fail(LBSA_ERR_UNSUPPORTED, "nB %d > 4096", nB);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DeviceState* ds = nullptr;
  if ((rc = device_state(&ds)) != LBSA_OK) return rc;
  int n_slots = 0;
  size_t flag_bytes = 0;
  const size_t bytes = lbsa::score_attend_pp_workspace_bytes(desc->N_valid, &n_slots, &flag_bytes);
  Scratch ws;
  if ((rc = scratch_alloc(ds, bytes, s, &ws)) != LBSA_OK) return rc;
  lbsa::AttendArgs a{desc->B, desc->H, desc->N_valid, desc->d, block, nB, nullptr, nullptr, ds->status,
                     out, desc->stride_b, desc->stride_h, desc->stride_n, lse, wait_limit(),
                     scores, reinterpret_cast<float*>(static_cast<char*>(ws.ptr) + flag_bytes),
                     static_cast<int32_t*>(ws.ptr), n_slots};
  CUtensorMap tq, tk, tv;
  if ((rc = make_tmap(&tq, q, desc, 128)) != LBSA_OK) return rc;
  if ((rc = make_tmap(&tk, k, desc, 64)) != LBSA_OK) return rc;
  if ((rc = make_tmap(&tv, v, desc, 64)) != LBSA_OK) return rc;
  cudaError_t e = cudaMemsetAsync(ws.ptr, 0, flag_bytes, s);     // every strip slot free
  if (e == cudaSuccess) e = lbsa::launch_score_attend_pp_bf16(&tq, &tk, &tv, a, s);
  if (e != cudaSuccess) return cuda_fail(e, "lbsa_score_attend launch");
  return LBSA_OK;
}

int lbsa_select(const float* scores, int32_t B, int32_t H, int32_t nB, int32_t block, double p, int32_t scope,
                lbsa_blockset** out, void* stream) {
  int rc;
  log_line("lbsa_select B=%d H=%d nB=%d block=%d p=%.9g scope=%d", B, H, nB, block, p, scope);
  if (!out) return fail(LBSA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if ((rc = validate_ptr(scores, "scores")) != LBSA_OK) return rc;
  if (B < 1 || H < 1 || nB < 1) return fail(LBSA_ERR_INVALID_ARG, "B, H, nB must be >= 1");
  if (block != 64 && block != 128) return fail(LBSA_ERR_UNSUPPORTED, "block %d: only 64 and 128 are built", block);
  if (!(p > 0.0) || !(p <= 1.0) || std::isnan(p)) return fail(LBSA_ERR_INVALID_ARG, "p = %g not in (0, 1]", p);
  if (scope != LBSA_SCOPE_ROW && scope != LBSA_SCOPE_HEAD) return fail(LBSA_ERR_INVALID_ARG, "scope %d", scope);
  if (nB > 4096) return fail(LBSA_ERR_UNSUPPORTED, "nB %d > 4096", nB);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  lbsa_blockset* bs = nullptr;
  if ((rc = new_blockset(B, H, nB, block, scope, p, s, &bs)) != LBSA_OK) return rc;
  cudaError_t e;
  if (scope == LBSA_SCOPE_ROW) {
    e = lbsa::launch_select_row(scores, B * H * nB, nB, p, bs, s);
  } else {
    DeviceState* ds = nullptr;
    Scratch ws;
    if ((rc = device_state(&ds)) != LBSA_OK ||
        (!lbsa::select_head_one_launch(nB) &&
         (rc = scratch_alloc(ds, lbsa::select_head_workspace_bytes(B, H, nB), s, &ws)) != LBSA_OK)) {
      lbsa_free(bs);
      return rc;
    }
    e = lbsa::launch_select_head(scores, B, H, nB, p, bs, ws.ptr, s);
  }
  if (e != cudaSuccess) {
    lbsa_free(bs);
    return cuda_fail(e, "lbsa_select launch");
  }
  *out = bs;
  return LBSA_OK;
}

int lbsa_select_rule(const float* scores, int32_t B, int32_t H, int32_t nB, int32_t block, int32_t n_valid,
                     int32_t rule, double p, int32_t k, lbsa_blockset** out, void* stream) {
  int rc;
  log_line("lbsa_select_rule B=%d H=%d nB=%d block=%d n_valid=%d rule=%d p=%.9g k=%d", B, H, nB, block, n_valid, rule,
           p, k);
  if (!out) return fail(LBSA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if ((rc = validate_ptr(scores, "scores")) != LBSA_OK) return rc;
  if (B < 1 || H < 1 || nB < 1) return fail(LBSA_ERR_INVALID_ARG, "B, H, nB must be >= 1");
  if (block != 64 && block != 128) return fail(LBSA_ERR_UNSUPPORTED, "block %d: only 64 and 128 are built", block);
  if (nB > 4096) return fail(LBSA_ERR_UNSUPPORTED, "the rank rules are built for nB <= 4096");
  if (static_cast<long long>(nB - 1) * block >= n_valid || n_valid > static_cast<long long>(nB) * block)
    return fail(LBSA_ERR_INVALID_ARG, "n_valid %d does not match nB %d x block %d", n_valid, nB, block);
  if (rule == LBSA_RULE_LOCAL_TOPK) {
    if (k < 0) return fail(LBSA_ERR_INVALID_ARG, "k = %d < 0", k);
  } else if (rule == LBSA_RULE_TOPP_FLOOR) {
    if (!(p > 0.0) || !(p <= 1.0) || std::isnan(p)) return fail(LBSA_ERR_INVALID_ARG, "p = %g not in (0, 1]", p);
  } else {
    return fail(LBSA_ERR_INVALID_ARG, "rule %d", rule);
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  lbsa_blockset* bs = nullptr;
  if ((rc = new_blockset(B, H, nB, block, LBSA_SCOPE_ROW, rule == LBSA_RULE_TOPP_FLOOR ? p : 0.0, s, &bs)) != LBSA_OK)
    return rc;
  const int R = B * H * nB;
  cudaError_t e;
  if (rule == LBSA_RULE_LOCAL_TOPK) {
    e = lbsa::launch_select_rank(scores, R, nB, 0, k, nullptr, bs, s);
  } else {
    DeviceState* ds = nullptr;
    Scratch ws;
    if ((rc = device_state(&ds)) != LBSA_OK ||
        (rc = scratch_alloc(ds, static_cast<size_t>(B) * H * sizeof(int32_t) + 256, s, &ws)) != LBSA_OK) {
      lbsa_free(bs);
      return rc;
    }
    int32_t* floor_dev = static_cast<int32_t*>(ws.ptr);
    e = lbsa::launch_select_row(scores, R, nB, p, bs, s);
    if (e == cudaSuccess) e = lbsa::launch_head_floor(bs->counts, B * H, nB, block, n_valid, floor_dev, s);
    if (e == cudaSuccess) e = lbsa::launch_select_rank(scores, R, nB, 1, 0, floor_dev, bs, s);
  }
  if (e != cudaSuccess) {
    lbsa_free(bs);
    return cuda_fail(e, "lbsa_select_rule launch");
  }
  *out = bs;
  return LBSA_OK;
}

int lbsa_select_tokens(const float* scores, int32_t B, int32_t H, int32_t n_valid, int32_t block, double p,
                       lbsa_blockset** out, void* stream) {
  int rc;
  log_line("lbsa_select_tokens B=%d H=%d n_valid=%d block=%d p=%.9g", B, H, n_valid, block, p);
  if (!out) return fail(LBSA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if ((rc = validate_ptr(scores, "scores")) != LBSA_OK) return rc;
  if (B < 1 || H < 1 || n_valid < 1) return fail(LBSA_ERR_INVALID_ARG, "B, H, n_valid must be >= 1");
  if (block != 64) return fail(LBSA_ERR_UNSUPPORTED, "per-token scope is built for 64-token blocks (block %d)", block);
  if (!(p > 0.0) || !(p <= 1.0) || std::isnan(p)) return fail(LBSA_ERR_INVALID_ARG, "p = %g not in (0, 1]", p);
  const int nB = n_blocks(n_valid, block);
  if (nB > 4096) return fail(LBSA_ERR_UNSUPPORTED, "per-token scope is built for nB <= 4096 (nB %d)", nB);
  if (static_cast<long long>(n_valid) * nB > 65535ll * 4096)
    return fail(LBSA_ERR_UNSUPPORTED, "%d tokens x %d blocks per head exceed the histogram grid", n_valid, nB);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  lbsa_blockset* bs = nullptr;
  if ((rc = new_blockset(B, H, nB, block, LBSA_SCOPE_TOKEN, p, s, &bs)) != LBSA_OK) return rc;
  DeviceState* ds = nullptr;
  Scratch ws;
  if ((rc = device_state(&ds)) != LBSA_OK ||
      (rc = scratch_alloc(ds, lbsa::select_head_workspace_bytes(B, H, nB, n_valid), s, &ws)) != LBSA_OK) {
    lbsa_free(bs);
    return rc;
  }
  cudaError_t e = lbsa::launch_select_tokens(scores, B, H, n_valid, nB, p, bs, ws.ptr, s);
  if (e != cudaSuccess) {
    lbsa_free(bs);
    return cuda_fail(e, "lbsa_select_tokens launch");
  }
  *out = bs;
  return LBSA_OK;
}

int lbsa_select_routed(const float* scores, int32_t B, int32_t H, int32_t nB, int32_t block, double p,
                       double entropy_threshold, int32_t group, double* head_entropy, int32_t* head_domain,
                       lbsa_blockset** out, void* stream) {
  int rc;
  log_line("lbsa_select_routed B=%d H=%d nB=%d block=%d p=%.9g threshold=%.9g group=%d", B, H, nB, block, p,
           entropy_threshold, group);
  if (!out) return fail(LBSA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if ((rc = validate_ptr(scores, "scores")) != LBSA_OK) return rc;
  if (B < 1 || H < 1 || nB < 1) return fail(LBSA_ERR_INVALID_ARG, "B, H, nB must be >= 1");
  if (block != 64 && block != 128) return fail(LBSA_ERR_UNSUPPORTED, "block %d: only 64 and 128 are built", block);
  if (!(p > 0.0) || !(p <= 1.0) || std::isnan(p)) return fail(LBSA_ERR_INVALID_ARG, "p = %g not in (0, 1]", p);
  if (std::isnan(entropy_threshold)) return fail(LBSA_ERR_INVALID_ARG, "entropy threshold is NaN");
  if (group < 1) return fail(LBSA_ERR_INVALID_ARG, "group = %d < 1", group);
  if (H > 4096) return fail(LBSA_ERR_UNSUPPORTED, "routed scope is built for H <= 4096 (H %d)", H);
  if (nB > 4096) return fail(LBSA_ERR_UNSUPPORTED, "routed scope is built for nB <= 4096 (nB %d)", nB);
  if (static_cast<long long>(B) * H > 65535)
    return fail(LBSA_ERR_UNSUPPORTED, "routed scope is built for B*H <= 65535 heads (%d x %d)", B, H);
  const size_t smem = lbsa::select_routed_smem_bytes(H, nB, group);
  if (smem > 200 * 1024)
    return fail(LBSA_ERR_UNSUPPORTED, "a pool of %d heads x %d key blocks needs %zu bytes of shared memory (> 200 KiB)",
                group < H ? group : H, nB, smem);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  lbsa_blockset* bs = nullptr;
  if ((rc = new_blockset(B, H, nB, block, LBSA_SCOPE_ROUTED, p, s, &bs)) != LBSA_OK) return rc;
  DeviceState* ds = nullptr;
  Scratch ws;
  if ((rc = device_state(&ds)) != LBSA_OK ||
      (rc = scratch_alloc(ds, lbsa::select_routed_workspace_bytes(B, H, nB), s, &ws)) != LBSA_OK) {
    lbsa_free(bs);
    return rc;
  }
  cudaError_t e = lbsa::launch_select_routed(scores, B, H, nB, p, entropy_threshold, group, head_entropy, head_domain,
                                             bs, ws.ptr, s);
  if (e != cudaSuccess) {
    lbsa_free(bs);
    return cuda_fail(e, "lbsa_select_routed launch");
  }
  *out = bs;
  return LBSA_OK;
}

int lbsa_attend(const void* q, const void* k, const void* v, const lbsa_qkv_desc* desc, const lbsa_blockset* bs,
                void* out, float* lse, void* stream) {
  int rc;
  if (desc)
    log_line("lbsa_attend B=%d H=%d N=%d d=%d dtype=%d blockset=%p (scope %d) lse=%d", desc->B, desc->H, desc->N_valid,
             desc->d, desc->dtype, static_cast<const void*>(bs), bs ? bs->scope : -1, lse != nullptr);
  if ((rc = validate_desc(desc)) != LBSA_OK) return rc;
  if ((rc = validate_ptr(q, "q")) != LBSA_OK) return rc;
  if ((rc = validate_ptr(k, "k")) != LBSA_OK) return rc;
  if ((rc = validate_ptr(v, "v")) != LBSA_OK) return rc;
  if ((rc = validate_ptr(out, "out")) != LBSA_OK) return rc;
  if (!bs) return fail(LBSA_ERR_INVALID_ARG, "blockset is NULL");
  if (bs->B != desc->B || bs->H != desc->H || bs->nB != n_blocks(desc->N_valid, bs->block))
    return fail(LBSA_ERR_INVALID_ARG, "blockset (B=%d, H=%d, nB=%d, block=%d) does not match q (B=%d, H=%d, N=%d)",
                bs->B, bs->H, bs->nB, bs->block, desc->B, desc->H, desc->N_valid);
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev != bs->device) return fail(LBSA_ERR_INVALID_ARG, "blockset lives on device %d, current is %d", bs->device, dev);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  lbsa::AttendArgs a{desc->B, desc->H, desc->N_valid, desc->d, bs->block, bs->nB, bs->counts, bs->cols, bs->status,
                     out, desc->stride_b, desc->stride_h, desc->stride_n, lse, wait_limit()};
  a.masks = bs->masks;
  cudaError_t e;
  if (desc->dtype == LBSA_BF16) {
    CUtensorMap tq, tk, tv;
    if ((rc = make_tmap(&tq, q, desc, 128)) != LBSA_OK) return rc;
    if ((rc = make_tmap(&tk, k, desc, 64)) != LBSA_OK) return rc;
    if ((rc = make_tmap(&tv, v, desc, 64)) != LBSA_OK) return rc;
    // a dense row-scope blockset (p = 1) takes the two-tile kernel (128-key
    // steps, measured a few percent faster on dense layers); every sparse one
    // the 64-key kernel (measured 5-40% faster across the sparse workloads)
    const bool dense = bs->scope == LBSA_SCOPE_ROW && bs->p >= 1.0;
    e = (dense && lbsa::attend_pp_supported(a)) ? lbsa::launch_attend_pp_bf16(&tq, &tk, &tv, a, s)
                                                : lbsa::launch_attend_bf16(&tq, &tk, &tv, a, s);
  } else {
    e = lbsa::launch_attend_f32(static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
                                *desc, a, s);
  }
  if (e != cudaSuccess) return cuda_fail(e, "lbsa_attend launch");
  return LBSA_OK;
}

void lbsa_free(lbsa_blockset* bs) {
  if (!bs) return;
  if (bs->base) cudaFreeAsync(bs->base, bs->stream);
  delete bs;
}

int lbsa_blockset_info(const lbsa_blockset* bs, int32_t* B, int32_t* H, int32_t* nB, int32_t* block, int32_t* scope) {
  if (!bs) return fail(LBSA_ERR_INVALID_ARG, "blockset is NULL");
  if (B) *B = bs->B;
  if (H) *H = bs->H;
  if (nB) *nB = bs->nB;
  if (block) *block = bs->block;
  if (scope) *scope = bs->scope;
  return LBSA_OK;
}

int lbsa_blockset_masks(const lbsa_blockset* bs, const uint64_t** masks) {
  if (!bs) return fail(LBSA_ERR_INVALID_ARG, "blockset is NULL");
  if (masks) *masks = bs->masks;
  return LBSA_OK;
}

int lbsa_blockset_views(const lbsa_blockset* bs, const int32_t** counts, const int32_t** cols) {
  if (!bs) return fail(LBSA_ERR_INVALID_ARG, "blockset is NULL");
  if (counts) *counts = bs->counts;
  if (cols) *cols = bs->cols;
  return LBSA_OK;
}

int lbsa_blockset_export(const lbsa_blockset* bs, int32_t* row_ptr, int32_t* col, int64_t* nnz, void* stream) {
  if (!bs) return fail(LBSA_ERR_INVALID_ARG, "blockset is NULL");
  if (!row_ptr || !col || !nnz) return fail(LBSA_ERR_INVALID_ARG, "row_ptr, col and nnz must be non-NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* d_nnz = row_ptr + static_cast<long long>(bs->B) * bs->H * bs->nB;   // row_ptr[R] holds the total
  cudaError_t e = lbsa::launch_export_csr(bs, row_ptr, col, d_nnz, s);
  if (e != cudaSuccess) return cuda_fail(e, "lbsa_blockset_export launch");
  int32_t h = 0;
  e = cudaMemcpyAsync(&h, d_nnz, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "lbsa_blockset_export copy");
  *nnz = h;
  return LBSA_OK;
}

int lbsa_blockset_from_csr(const int32_t* row_ptr, const int32_t* col, int32_t B, int32_t H, int32_t nB, int32_t block,
                           lbsa_blockset** out, void* stream) {
  if (!out) return fail(LBSA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (!row_ptr || !col) return fail(LBSA_ERR_INVALID_ARG, "row_ptr and col must be non-NULL");
  if (B < 1 || H < 1 || nB < 1 || nB > 4096) return fail(LBSA_ERR_INVALID_ARG, "bad B/H/nB");
  if (block != 64 && block != 128) return fail(LBSA_ERR_UNSUPPORTED, "block %d", block);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  lbsa_blockset* bs = nullptr;
  int rc = new_blockset(B, H, nB, block, LBSA_SCOPE_ROW, -1.0, s, &bs);
  if (rc != LBSA_OK) return rc;
  cudaError_t e = lbsa::launch_from_csr(row_ptr, col, bs, s);
  if (e != cudaSuccess) {
    lbsa_free(bs);
    return cuda_fail(e, "lbsa_blockset_from_csr launch");
  }
  *out = bs;
  return LBSA_OK;
}

int lbsa_blockset_export_bitmask(const lbsa_blockset* bs, uint32_t* bits, void* stream) {
  if (!bs) return fail(LBSA_ERR_INVALID_ARG, "blockset is NULL");
  if (!bits) return fail(LBSA_ERR_INVALID_ARG, "bits is NULL");
  if (bs->masks) return fail(LBSA_ERR_UNSUPPORTED, "per-token blocksets have no block bitmask (use lbsa_blockset_masks)");
  cudaError_t e = lbsa::launch_export_bitmask(bs, bits, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lbsa_blockset_export_bitmask launch");
  return LBSA_OK;
}

int lbsa_blockset_from_bitmask(const uint32_t* bits, int32_t B, int32_t H, int32_t nB, int32_t block,
                               lbsa_blockset** out, void* stream) {
  if (!out) return fail(LBSA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (!bits) return fail(LBSA_ERR_INVALID_ARG, "bits is NULL");
  if (B < 1 || H < 1 || nB < 1 || nB > 4096) return fail(LBSA_ERR_INVALID_ARG, "bad B/H/nB");
  if (block != 64 && block != 128) return fail(LBSA_ERR_UNSUPPORTED, "block %d", block);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  lbsa_blockset* bs = nullptr;
  int rc = new_blockset(B, H, nB, block, LBSA_SCOPE_ROW, -1.0, s, &bs);
  if (rc != LBSA_OK) return rc;
  cudaError_t e = lbsa::launch_from_bitmask(bits, bs, s);
  if (e != cudaSuccess) {
    lbsa_free(bs);
    return cuda_fail(e, "lbsa_blockset_from_bitmask launch");
  }
  *out = bs;
  return LBSA_OK;
}

int lbsa_get_status(const lbsa_blockset* bs, int32_t* device_status, int32_t clear, void* stream) {
  if (!bs || !device_status) return fail(LBSA_ERR_INVALID_ARG, "NULL argument");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(device_status, bs->status, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess && clear) e = cudaMemsetAsync(bs->status, 0, sizeof(int32_t), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "lbsa_get_status");
  return LBSA_OK;
}

int lbsa_device_status(int32_t* device_status, int32_t clear, void* stream) {
  if (!device_status) return fail(LBSA_ERR_INVALID_ARG, "NULL argument");
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != LBSA_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(device_status, ds->status, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess && clear) e = cudaMemsetAsync(ds->status, 0, sizeof(int32_t), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "lbsa_device_status");
  return LBSA_OK;
}

int lbsa_partition_perm(int32_t T, int32_t Hg, int32_t Wg, int32_t kind, int32_t tt, int32_t th, int32_t tw,
                        int32_t* perm, int32_t on_device, void* stream) {
  if (!perm) return fail(LBSA_ERR_INVALID_ARG, "perm is NULL");
  if (T < 1 || Hg < 1 || Wg < 1) return fail(LBSA_ERR_INVALID_ARG, "grid must be >= 1 in every axis");
  if (static_cast<long long>(T) * Hg * Wg >= (1ll << 31)) return fail(LBSA_ERR_INVALID_ARG, "grid too large");
  if (kind < LBSA_PART_RASTER || kind > LBSA_PART_3D) return fail(LBSA_ERR_INVALID_ARG, "partition kind %d", kind);
  if ((kind == LBSA_PART_2D && (th < 1 || tw < 1)) || (kind == LBSA_PART_3D && (tt < 1 || th < 1 || tw < 1)))
    return fail(LBSA_ERR_INVALID_ARG, "tile sizes must be >= 1");
  if (!on_device) {
    lbsa::partition_perm_host(T, Hg, Wg, kind, tt, th, tw, perm);
    return LBSA_OK;
  }
  cudaError_t e = lbsa::launch_partition_perm(T, Hg, Wg, kind, tt, th, tw, perm, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lbsa_partition_perm launch");
  return LBSA_OK;
}

int lbsa_permute(const void* const* xs, void* const* ys, int32_t count, const int32_t* perm, const lbsa_qkv_desc* desc,
                 int32_t inverse, void* stream) {
  int rc;
  if (desc) log_line("lbsa_permute count=%d B=%d H=%d N=%d d=%d inverse=%d", count, desc->B, desc->H, desc->N_valid,
                     desc->d, inverse);
  if ((rc = validate_desc(desc)) != LBSA_OK) return rc;
  if (!xs || !ys || count < 1 || count > 3) return fail(LBSA_ERR_INVALID_ARG, "need 1..3 tensors");
  if (!perm) return fail(LBSA_ERR_INVALID_ARG, "perm is NULL");
  for (int t = 0; t < count; ++t) {
    if ((rc = validate_ptr(xs[t], "x")) != LBSA_OK) return rc;
    if ((rc = validate_ptr(ys[t], "y")) != LBSA_OK) return rc;
    if (xs[t] == ys[t]) return fail(LBSA_ERR_INVALID_ARG, "x and y may not alias");
  }
  DeviceState* ds = nullptr;
  if ((rc = device_state(&ds)) != LBSA_OK) return rc;
  cudaError_t e =
      lbsa::launch_permute(xs, ys, count, perm, *desc, inverse, ds->status, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lbsa_permute launch");
  return LBSA_OK;
}

int lbsa_selftest_wait(int64_t limit_us, int32_t* device_out, void* stream) {
  if (!device_out) return fail(LBSA_ERR_INVALID_ARG, "device_out is NULL");
  if (limit_us < 1 || limit_us > 10000000) return fail(LBSA_ERR_INVALID_ARG, "limit_us must lie in [1, 1e7]");
  cudaError_t e = lbsa::launch_selftest_wait(limit_us * 1000, device_out, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lbsa_selftest_wait launch");
  return LBSA_OK;
}

int lbsa_selftest_exp2(const float* v, float* out, int64_t n, void* stream) {
  if (n < 0) return fail(LBSA_ERR_INVALID_ARG, "n < 0");
  if (n == 0) return LBSA_OK;
  if (!v || !out) return fail(LBSA_ERR_INVALID_ARG, "v or out is NULL");
  cudaError_t e = lbsa::launch_selftest_exp2(v, out, n, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lbsa_selftest_exp2 launch");
  return LBSA_OK;
}

}  // extern "C"

namespace lbsa {
int set_error(int code, const char* msg) { return fail(code, "%s", msg); }

namespace {
// One thread waits on an mbarrier that nothing ever completes.
__global__ void selftest_wait_kernel(long long limit_ns, int32_t* out) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  __shared__ int32_t st;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    st = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = mbar_wait(&bar, 0, limit_ns, &st, &abort_flag);
    *out = ok ? LBSA_OK : st;
  }
}
}  // namespace

cudaError_t launch_selftest_wait(long long limit_ns, int32_t* out, cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>(limit_ns, out);
  return cudaGetLastError();
}

namespace {
// pairs through exp2_poly2; an odd tail element is paired with itself
__global__ void selftest_exp2_kernel(const float* __restrict__ v, float* __restrict__ out, long long n) {
  for (long long i = 2 * (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x); i < n;
       i += 2ll * gridDim.x * blockDim.x) {
    const float a = v[i], b = (i + 1 < n) ? v[i + 1] : a;
    float ra, rb;
    u64_as_f2(exp2_poly2(f2_as_u64(a, b)), ra, rb);
    out[i] = ra;
    if (i + 1 < n) out[i + 1] = rb;
  }
}
}  // namespace

cudaError_t launch_selftest_exp2(const float* v, float* out, long long n, cudaStream_t s) {
  const long long pairs = (n + 1) / 2;
  const unsigned blocks = static_cast<unsigned>(std::min<long long>((pairs + 255) / 256, 4096));
  selftest_exp2_kernel<<<blocks, 256, 0, s>>>(v, out, n);
  return cudaGetLastError();
}
}  // namespace lbsa
