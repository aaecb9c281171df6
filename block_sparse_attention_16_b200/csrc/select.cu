// Mass-threshold block selection (LoSA abstract: per head and query block, as
// few key/value blocks as retain the threshold share of the mass; VMoBA
// review on pith.science, circularity check: the least count k' of pairs whose
// running sum of normalised similarity gets to tau, with VMoBA's global
// selection over all block pairs of a head, where query rows may come out
// empty).
//
// The cumulative sum is exact so that the kept set does not depend on the
// order of a parallel reduction:
//   w = floor(x * 2^32)  (x fp32 in [0, 2): w < 2^33, computed from the bits)
//   W = sum w,  P = round_half_even(p * 2^24),  T = ceil(P * W / 2^24)
//   order by x descending, then flat index ascending; keep the shortest
//   prefix whose sum of w reaches T (at least one element); p >= 1 keeps all.
// Instead of sorting, both scopes search for the threshold value tb: the
// largest bit pattern whose "weight at or above" S(tb) = sum_{bits >= tb} w
// still reaches T.  Every element above tb is kept; of the elements equal to
// tb (all of weight w(tb)), the ceil((T - S(tb+1)) / w(tb)) with the lowest
// flat indices are kept.  This is exactly the sorted-prefix rule.
#include <cooperative_groups.h>
#include <cstdio>
#include <mutex>

#include "lbsa_device.cuh"
#include "lbsa_routed.h"

namespace lbsa {
namespace {

constexpr uint32_t kInvalidBits = 0x40000000u;    // bits >= this: NaN, inf, negative, or >= 2.0

// floor(x * 2^32) for a valid fp32 bit pattern (0 <= x < 2), in integers.
__device__ __forceinline__ uint64_t fixed_weight(uint32_t bits) {
  const uint32_t e = bits >> 23;
  if (e == 0) return 0;                       // zero / subnormal: x * 2^32 < 1
  const uint64_t M = (bits & 0x7FFFFFu) | 0x800000u;
  if (e >= 118) return M << (e - 118);
  const uint32_t sh = 118 - e;
  return sh >= 24 ? 0 : (M >> sh);
}

// Exact warp sum of per-lane values below 2^54: the low 27 bits and the rest
// are summed separately by two redux.sync adds (each total fits 32 bits),
// a shorter dependent chain than five rounds of 64-bit shuffles.
__device__ __forceinline__ uint64_t warp_sum_u64(uint64_t v) {
  const uint32_t lo = static_cast<uint32_t>(v) & ((1u << 27) - 1u);
  const uint32_t hi = static_cast<uint32_t>(v >> 27);
  const uint32_t slo = __reduce_add_sync(0xffffffffu, lo);
  const uint32_t shi = __reduce_add_sync(0xffffffffu, hi);
  return (static_cast<uint64_t>(shi) << 27) + slo;
}

__device__ __forceinline__ uint64_t threshold_T(uint64_t W, uint32_t Pfix) {
  const unsigned __int128 num = static_cast<unsigned __int128>(W) * Pfix + ((1u << 24) - 1);
  return static_cast<uint64_t>(num >> 24);
}

// ---------------------------------------------------------------- row scope
// One warp per row of nB scores; lane l holds elements l, l+32, ...
// skip_head (NULL for plain row scope): rows of heads with skip_head[h] >= 0
// (pooled heads of the routed scope) are left to the domain kernel.
// The bisection runs in two phases.  While more than 32 weighted elements lie
// in the bracket [lo, hi), every step sums all of the row's weights at or
// above mid; each weight carries the element count in its low 11 bits, so the
// same exact sum also gives the bracket's population.  Then the bracket's
// elements are compacted to one a lane and the remaining steps sum only
// those, on top of S at the bracket's upper end.  The result is the bisection's.
constexpr int kRowThreads = 64;
template <int EPL>
__global__ void __launch_bounds__(kRowThreads) select_row_kernel(
    const float* __restrict__ scores, int R, int nB, uint32_t Pfix, int keep_all, int32_t* __restrict__ counts,
    int32_t* __restrict__ cols, int32_t* __restrict__ status, const int32_t* __restrict__ skip_head) {
  __shared__ uint32_t cbits[kRowThreads / 32][32];
  __shared__ unsigned long long cw[kRowThreads / 32][32];
  const int lane = threadIdx.x & 31;
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (row >= R) return;
  if (skip_head && skip_head[row / nB] >= 0) return;      // warp-uniform
  const uint32_t* x = reinterpret_cast<const uint32_t*>(scores) + row * nB;
  int32_t* out = cols + row * nB;
  uint32_t bits[EPL];
  uint64_t wc[EPL];            // (w << 11) | 1 for an element of weight w > 0, else 0 (w < 2^33)
  bool bad = false;
  uint64_t wsum = 0;
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    const int idx = e * 32 + lane;
    const uint32_t b = (idx < nB) ? __ldg(x + idx) : 0u;
    bad |= (idx < nB) && (b >= kInvalidBits);
    bits[e] = b;
    const uint64_t w = (idx < nB && b < kInvalidBits) ? fixed_weight(b) : 0;
    wc[e] = w ? ((w << 11) | 1ull) : 0ull;
    wsum += wc[e];
  }
  const bool any_bad = __any_sync(0xffffffffu, bad);
  if (any_bad || keep_all) {
    if (any_bad && lane == 0) raise_status(status, LBSA_ERR_INVALID_SCORES);
    for (int idx = lane; idx < nB; idx += 32) out[idx] = idx;
    if (lane == 0) counts[row] = nB;
    return;
  }
  // at most 1024 elements of weight < 2^33: every sum below stays under 2^54
  const uint64_t Wc = warp_sum_u64(wsum);
  const uint64_t W = Wc >> 11;
  const uint64_t T = threshold_T(W, Pfix);
  uint32_t tb;
  uint32_t need;
  if (T == 0) {
    // nothing to reach: keep one block, the highest score with the lowest index
    uint32_t mb = 0;
#pragma unroll
    for (int e = 0; e < EPL; ++e)
      if (e * 32 + lane < nB) mb = max(mb, bits[e]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, o));
    tb = mb;
    need = 1;
  } else {
    // the bracket starts at the weighted scores' range: S(min) = W >= T and S(max + 1) = 0 < T
    uint32_t bmin = 0xFFFFFFFFu, bmax = 0u;
#pragma unroll
    for (int e = 0; e < EPL; ++e)
      if (wc[e]) {
        bmin = min(bmin, bits[e]);
        bmax = max(bmax, bits[e]);
      }
    uint32_t lo = __reduce_min_sync(0xffffffffu, bmin);   // invariant: S(lo) >= T > S(hi)
    uint32_t hi = __reduce_max_sync(0xffffffffu, bmax) + 1u;
    uint64_t S_hi = 0;                        // S(hi)
    uint32_t c_lo = static_cast<uint32_t>(Wc & 2047u), c_hi = 0;   // weighted elements at or above lo / hi
    const uint64_t Tc = T << 11;              // S(mid) >= T  <=>  (S(mid) << 11) + count >= Tc
    while (hi - lo > 1 && c_lo - c_hi > 32) {
      const uint32_t mid = lo + ((hi - lo) >> 1);
      // four independent partial sums: the 64-bit adds do not form one long chain
      uint64_t s4[4] = {0, 0, 0, 0};
#pragma unroll
      for (int e = 0; e < EPL; ++e) s4[e & 3] += (bits[e] >= mid) ? wc[e] : 0;
      const uint64_t s = warp_sum_u64((s4[0] + s4[1]) + (s4[2] + s4[3]));
      if (s >= Tc) {
        lo = mid;
        c_lo = static_cast<uint32_t>(s & 2047u);
      } else {
        hi = mid;
        c_hi = static_cast<uint32_t>(s & 2047u);
        S_hi = s >> 11;
      }
    }
    if (hi - lo > 1) {
      // at most 32 weighted elements left in [lo, hi): one a lane
      const int wi = threadIdx.x >> 5;
      const uint32_t lt = (1u << lane) - 1u;
      uint32_t n = 0;
      const uint32_t span = hi - lo;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        const bool act = wc[e] != 0 && bits[e] - lo < span;
        const uint32_t m = __ballot_sync(0xffffffffu, act);
        if (act) {
          const uint32_t pos = n + __popc(m & lt);
          cbits[wi][pos] = bits[e];
          cw[wi][pos] = wc[e];
        }
        n += __popc(m);
      }
      __syncwarp();
      const uint32_t b1 = (lane < static_cast<int>(n)) ? cbits[wi][lane] : 0u;
      const uint64_t w1 = (lane < static_cast<int>(n)) ? (cw[wi][lane] >> 11) : 0ull;
      const uint64_t base = S_hi;             // S at the bracket's upper end when compacted
      while (hi - lo > 1) {
        const uint32_t mid = lo + ((hi - lo) >> 1);
        const uint64_t s = base + warp_sum_u64((b1 >= mid) ? w1 : 0ull);
        if (s >= T) lo = mid;
        else {
          hi = mid;
          S_hi = s;
        }
      }
    }
    tb = lo;
    const uint64_t above = S_hi;              // S(tb + 1)
    const uint64_t ww = fixed_weight(tb);     // > 0 because S(tb) > S(tb + 1)
    const uint64_t rest = T - above;
    need = static_cast<uint32_t>((rest + ww - 1) / ww);
  }
  // emit in ascending index order
  int base = 0;
  uint32_t ties_before = 0;
  const uint32_t lt_mask = (1u << lane) - 1u;
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    const int idx = e * 32 + lane;
    const bool present = idx < nB;
    const bool tie = present && bits[e] == tb;
    const uint32_t tmask = __ballot_sync(0xffffffffu, tie);
    const uint32_t rank = ties_before + __popc(tmask & lt_mask);
    const bool keep = present && (bits[e] > tb || (tie && rank < need));
    const uint32_t kmask = __ballot_sync(0xffffffffu, keep);
    if (keep) out[base + __popc(kmask & lt_mask)] = idx;
    base += __popc(kmask);
    ties_before += __popc(tmask);
  }
  if (lane == 0) counts[row] = base;
}

// ---------------------------------------------------------------- wide rows
// Rows of more than 1024 blocks (up to 4096): one 256-thread CTA per row,
// thread t holding elements t, t + 256, ...; the same threshold search as the
// one-warp kernels above with CTA-wide exact sums, then an ascending emit by
// CTA-wide prefix counts.  kind 0: the threshold rule on fixed-point weights
// (skip_head as in select_row_kernel); kind 1: the row's own block plus the k
// top-ranked others (Local + TopK); kind 2: the first max(c, min(K, nB)) of the
// ranked order (per-head floor), rows with n == c left as they are.
constexpr int kWideThreads = 256;

// Exact CTA sum of per-thread values below 2^54 (< 2^62 in total); buf is one
// of two [8] slots used alternately, so one barrier per call suffices.
__device__ __forceinline__ uint64_t cta_sum_u64(uint64_t v, unsigned long long* buf) {
  v = warp_sum_u64(v);
  if ((threadIdx.x & 31) == 0) buf[threadIdx.x >> 5] = v;
  __syncthreads();
  uint64_t t = 0;
#pragma unroll
  for (int w = 0; w < kWideThreads / 32; ++w) t += buf[w];
  return t;
}

// Exclusive CTA prefix count of a per-thread flag in thread order, and the total.
__device__ __forceinline__ uint32_t cta_prefix(bool f, uint32_t* buf, uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t m = __ballot_sync(0xffffffffu, f);
  if (lane == 0) buf[warp] = __popc(m);
  __syncthreads();
  uint32_t before = 0;
  total = 0;
#pragma unroll
  for (int w = 0; w < kWideThreads / 32; ++w) {
    const uint32_t c = buf[w];
    before += (w < warp) ? c : 0u;
    total += c;
  }
  return before + __popc(m & ((1u << lane) - 1u));
}

template <int EPT>
__global__ void __launch_bounds__(kWideThreads) select_wide_kernel(
    const float* __restrict__ scores, int R, int nB, int kind, uint32_t Pfix, int keep_all, int k,
    const int32_t* __restrict__ head_floor, int32_t* __restrict__ counts, int32_t* __restrict__ cols,
    int32_t* __restrict__ status, const int32_t* __restrict__ skip_head) {
  __shared__ unsigned long long red[2][kWideThreads / 32];
  __shared__ uint32_t cnt[4][kWideThreads / 32];
  const long long row = blockIdx.x;
  if (row >= R) return;                                     // CTA-uniform
  if (kind == 0 && skip_head && skip_head[row / nB] >= 0) return;
  const int t = threadIdx.x;
  const int diag = (kind == 1) ? static_cast<int>(row % nB) : -1;
  int n = 0;
  if (kind == 1) {
    n = min(k, nB - 1);
  } else if (kind == 2) {
    const int c = counts[row];
    n = max(c, min(head_floor[row / nB], nB));
    if (n == c) return;
  }
  const uint32_t* x = reinterpret_cast<const uint32_t*>(scores) + row * nB;
  int32_t* out = cols + row * nB;
  uint32_t bits[EPT];
  bool bad = false;
#pragma unroll
  for (int e = 0; e < EPT; ++e) {
    const int idx = e * kWideThreads + t;
    bits[e] = (idx < nB) ? __ldg(x + idx) : 0u;
    bad |= (idx < nB) && (bits[e] >= kInvalidBits);
  }
  int step = 0;                                             // alternates the two reduction slots
  if (__syncthreads_or(bad)) {
    if (t == 0) raise_status(status, LBSA_ERR_INVALID_SCORES);
    for (int idx = t; idx < nB; idx += kWideThreads) out[idx] = idx;
    if (t == 0) counts[row] = nB;
    return;
  }
  if (kind == 0 && keep_all) {
    for (int idx = t; idx < nB; idx += kWideThreads) out[idx] = idx;
    if (t == 0) counts[row] = nB;
    return;
  }
  // weight of element e: its fixed-point mass (kind 0) or 1 (ranked kinds)
  auto weight = [&](int e) -> uint64_t {
    const int idx = e * kWideThreads + t;
    if (idx >= nB || idx == diag) return 0;
    return kind == 0 ? fixed_weight(bits[e]) : 1ull;
  };
  uint64_t T;
  if (kind == 0) {
    uint64_t ws = 0;
#pragma unroll
    for (int e = 0; e < EPT; ++e) ws += weight(e);
    T = threshold_T(cta_sum_u64(ws, red[step++ & 1]), Pfix);
  } else {
    T = static_cast<uint64_t>(n);
  }
  uint32_t tb = 0u, need = 0u;
  bool none = kind != 0 && n == 0;                          // ranked kinds with nothing ranked in
  if (!none && T == 0) {
    // nothing to reach (kind 0): keep one block, the highest score with the lowest index
    uint32_t mb = 0;
#pragma unroll
    for (int e = 0; e < EPT; ++e)
      if (e * kWideThreads + t < nB) mb = max(mb, bits[e]);
    mb = __reduce_max_sync(0xffffffffu, mb);
    if ((t & 31) == 0) cnt[0][t >> 5] = mb;
    __syncthreads();
    for (int w = 0; w < kWideThreads / 32; ++w) tb = max(tb, cnt[0][w]);
    need = 1;
    __syncthreads();
  } else if (!none) {
    uint32_t lo = 0, hi = kInvalidBits;                     // invariant: S(lo) >= T > S(hi)
    while (hi - lo > 1) {
      const uint32_t mid = lo + ((hi - lo) >> 1);
      uint64_t s4[4] = {0, 0, 0, 0};
#pragma unroll
      for (int e = 0; e < EPT; ++e) s4[e & 3] += (bits[e] >= mid) ? weight(e) : 0;
      const uint64_t sum = cta_sum_u64((s4[0] + s4[1]) + (s4[2] + s4[3]), red[step++ & 1]);
      if (sum >= T) lo = mid;
      else hi = mid;
    }
    tb = lo;
    uint64_t above = 0;
#pragma unroll
    for (int e = 0; e < EPT; ++e) above += (bits[e] > tb) ? weight(e) : 0;
    above = cta_sum_u64(above, red[step++ & 1]);
    const uint64_t ww = kind == 0 ? fixed_weight(tb) : 1ull;
    need = static_cast<uint32_t>((T - above + ww - 1) / ww);
  }
  // emit in ascending index order: chunk e holds indices e*256 .. e*256 + 255
  uint32_t base = 0, ties_before = 0;
#pragma unroll
  for (int e = 0; e < EPT; ++e) {
    const int idx = e * kWideThreads + t;
    const bool elig = idx < nB && idx != diag;
    const bool tie = !none && elig && bits[e] == tb;
    uint32_t ttot, ktot;
    const uint32_t rank = ties_before + cta_prefix(tie, cnt[e & 1], ttot);
    const bool keep = (idx == diag && idx < nB) || (!none && elig && (bits[e] > tb || (tie && rank < need)));
    const uint32_t pos = base + cta_prefix(keep, cnt[2 + (e & 1)], ktot);
    if (keep) out[pos] = idx;
    base += ktot;
    ties_before += ttot;
  }
  if (t == 0) counts[row] = static_cast<int32_t>(base);
}

// ---------------------------------------------------------------- head scope
// Weighted MSD radix select over 30 significant bits in three 10-bit digits.
struct HeadState {
  unsigned long long W, T, above;
  unsigned int prefix;      // resolved high digits so far
  unsigned int maxbits;
  int bad;
  int resolved;             // 1: tb/need final (T == 0 case)
  int keep_all;
  unsigned int tb;
  unsigned int need;
  unsigned int arrived;      // histogram CTAs of the current pass that have finished
};

constexpr int kDigitBits = 10;
constexpr int kBins = 1 << kDigitBits;
constexpr long long kHistPerCta = 16384;    // most elements a histogram CTA sees (256 threads x 64)
constexpr int kLoBits = 18;                  // weight split for the 32-bit shared sums (see head_hist_kernel)

// After pass k, run by the last histogram CTA of the head (256 threads, bins
// 4t .. 4t+3 per thread): pick the digit where the weight at or above crosses
// T, and clear the histogram for the next pass.
__device__ void find_digit(int pass, uint32_t Pfix, int keep_all, unsigned long long* __restrict__ gh,
                           HeadState* __restrict__ s, int32_t* __restrict__ status) {
  __shared__ unsigned long long warp_tot[8];
  __shared__ int done;
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  unsigned long long v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[i] = __ldcg(gh + 4 * t + i);           // summed by other CTAs' atomics: read from L2
    gh[4 * t + i] = 0ull;
  }
  // suffix sums: thread total, inclusive suffix over the warp's lanes, then over the warps
  unsigned long long x = (v[0] + v[1]) + (v[2] + v[3]);
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_down_sync(0xffffffffu, x, o);
    if (lane + o < 32) x += y;
  }
  if (lane == 0) warp_tot[w] = x;
  if (t == 0) done = 0;
  __syncthreads();
  unsigned long long later = 0;
  for (int u = w + 1; u < 8; ++u) later += warp_tot[u];
  unsigned long long S[5];                    // S[i] = weight of bins >= 4t + i
  S[0] = x + later;
#pragma unroll
  for (int i = 0; i < 4; ++i) S[i + 1] = S[i] - v[i];
  if (t == 0 && pass == 0) {
    s->W = S[0];
    if (__ldcg(&s->bad)) {                  // set by other CTAs' atomics this pass
      raise_status(status, LBSA_ERR_INVALID_SCORES);
      s->keep_all = 1;
      done = 1;
    } else if (keep_all) {
      s->keep_all = 1;
      done = 1;
    } else {
      s->T = threshold_T(S[0], Pfix);
      s->above = 0;
      s->prefix = 0;
      if (s->T == 0) {
        s->resolved = 1;
        s->tb = __ldcg(&s->maxbits);
        s->need = 1;
        done = 1;
      }
    }
  }
  __syncthreads();
  if (done) return;
  const unsigned long long T = s->T;
  const unsigned long long above = s->above;
  const unsigned int prefix = s->prefix;
  __syncthreads();                            // every thread has read the state before it changes
  // the largest bin b with above + S(b) >= T (exists: S(0) covers everything not above)
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (above + S[i] >= T && above + S[i + 1] < T) {
      const unsigned int b = static_cast<unsigned int>(4 * t + i);
      s->above = above + S[i + 1];
      s->prefix = (prefix << kDigitBits) | b;
      if (pass == 2) {
        const unsigned int tb = (prefix << kDigitBits) | b;
        s->tb = tb;
        const unsigned long long ww = fixed_weight(tb);
        s->need = static_cast<unsigned int>((T - (above + S[i + 1]) + ww - 1) / ww);
        s->resolved = 1;
      }
    }
  }
}

// pass 0..2: histogram of weights by digit among elements whose higher digits
// match the resolved prefix.  grid (chunks, G), 256 threads.
__global__ void __launch_bounds__(256) head_hist_kernel(const float* __restrict__ scores, long long seg_len, int pass,
                                                        uint32_t Pfix, int keep_all,
                                                        unsigned long long* __restrict__ hist,
                                                        HeadState* __restrict__ st, int32_t* __restrict__ status) {
  __shared__ int is_last;
  // weights (< 2^33) split into 18 low and 15 high bits, summed with 32-bit
  // shared atomics: a CTA sees at most kHistPerCta = 2^14 elements, so the low
  // sums stay below 2^32 and the high ones below 2^29
  __shared__ uint32_t sh_lo[kBins], sh_hi[kBins];
  __shared__ unsigned int smax;
  __shared__ int sbad;
  const int g = blockIdx.y;
  HeadState* s = st + g;
  if (pass > 0 && (s->resolved || s->keep_all)) return;
  for (int i = threadIdx.x; i < kBins; i += blockDim.x) {
    sh_lo[i] = 0u;
    sh_hi[i] = 0u;
  }
  if (threadIdx.x == 0) {
    smax = 0;
    sbad = 0;
  }
  __syncthreads();
  const int shift = 20 - kDigitBits * pass;
  const unsigned int prefix = (pass > 0) ? s->prefix : 0u;
  const uint32_t* x = reinterpret_cast<const uint32_t*>(scores) + static_cast<long long>(g) * seg_len;
  unsigned int lmax = 0;
  int lbad = 0;
  // a thread's elements come in batches of 16, all loaded before any is
  // binned, so their DRAM round trips overlap
  constexpr int kBatch = 16;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i0 = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i0 < seg_len;
       i0 += kBatch * stride) {
    uint32_t v[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const long long i = i0 + u * stride;
      v[u] = (i < seg_len) ? __ldg(x + i) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      if (i0 + u * stride >= seg_len) break;
      const uint32_t b = v[u];
      if (b >= kInvalidBits) {
        lbad = 1;
        continue;
      }
      if (pass == 0) lmax = max(lmax, b);
      if (pass > 0 && (b >> (shift + kDigitBits)) != prefix) continue;
      const uint64_t w = fixed_weight(b);
      if (w) {
        const uint32_t bin = (b >> shift) & (kBins - 1);
        atomicAdd(&sh_lo[bin], static_cast<uint32_t>(w & ((1ull << kLoBits) - 1)));
        atomicAdd(&sh_hi[bin], static_cast<uint32_t>(w >> kLoBits));
      }
    }
  }
  if (pass == 0) {
    atomicMax(&smax, lmax);
    if (lbad) sbad = 1;
  }
  __syncthreads();
  unsigned long long* gh = hist + static_cast<long long>(g) * kBins;
  for (int i = threadIdx.x; i < kBins; i += blockDim.x) {
    const unsigned long long v = (static_cast<unsigned long long>(sh_hi[i]) << kLoBits) + sh_lo[i];
    if (v) atomicAdd(gh + i, v);
  }
  if (threadIdx.x == 0 && pass == 0) {
    atomicMax(&s->maxbits, smax);
    if (sbad) atomicExch(&s->bad, 1);
  }
  // the last CTA of this head to finish resolves the digit (no CTA waits for another)
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(&s->arrived, 1u) == gridDim.x - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  if (threadIdx.x == 0) s->arrived = 0;       // for the next pass
  find_digit(pass, Pfix, keep_all, gh, s, status);
}

// Ties (bits == tb) per row of a head's nQ x nB pairs (rows: query blocks, or
// query tokens in per-token scope).  One warp per row.
__global__ void head_tiecount_kernel(const float* __restrict__ scores, int G, int nQ, int nB,
                                     const HeadState* __restrict__ st, int32_t* __restrict__ tiecnt) {
  const int lane = threadIdx.x & 31;
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (row >= static_cast<long long>(G) * nQ) return;
  const HeadState* s = st + row / nQ;
  if (s->keep_all) return;
  const uint32_t* x = reinterpret_cast<const uint32_t*>(scores) + row * nB;
  int c = 0;
  for (int j = lane; j < nB; j += 32) c += (__ldg(x + j) == s->tb);
  c = __reduce_add_sync(0xffffffffu, static_cast<unsigned>(c));
  if (lane == 0) tiecnt[row] = c;
}

// Exclusive scan of the nQ rows' tie counts within each head.  grid G, 1024 threads.
__global__ void head_tiescan_kernel(int nQ, const HeadState* __restrict__ st, int32_t* __restrict__ tiecnt) {
  __shared__ int buf[1024];
  __shared__ int carry;
  const int g = blockIdx.x;
  if (st[g].keep_all) return;
  int32_t* c = tiecnt + static_cast<long long>(g) * nQ;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < nQ; base += 1024) {
    const int i = base + threadIdx.x;
    const int v = (i < nQ) ? c[i] : 0;
    buf[threadIdx.x] = v;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
      const int add = (threadIdx.x >= o) ? buf[threadIdx.x - o] : 0;
      __syncthreads();
      buf[threadIdx.x] += add;
      __syncthreads();
    }
    if (i < nQ) c[i] = carry + buf[threadIdx.x] - v;
    __syncthreads();
    if (threadIdx.x == 1023) carry += buf[1023];
    __syncthreads();
  }
}

// Emit kept pairs per query-block row (ascending key block).  One warp per row.
__global__ void head_emit_kernel(const float* __restrict__ scores, int G, int nB, const HeadState* __restrict__ st,
                                 const int32_t* __restrict__ tiebase, int32_t* __restrict__ counts,
                                 int32_t* __restrict__ cols) {
  const int lane = threadIdx.x & 31;
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (row >= static_cast<long long>(G) * nB) return;
  const HeadState* s = st + row / nB;
  const uint32_t* x = reinterpret_cast<const uint32_t*>(scores) + row * nB;
  int32_t* out = cols + row * nB;
  if (s->keep_all) {
    for (int j = lane; j < nB; j += 32) out[j] = j;
    if (lane == 0) counts[row] = nB;
    return;
  }
  const uint32_t tb = s->tb, need = s->need;
  uint32_t ties_before = static_cast<uint32_t>(tiebase[row]);
  const uint32_t lt_mask = (1u << lane) - 1u;
  int base = 0;
  for (int j0 = 0; j0 < nB; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t b = (j < nB) ? __ldg(x + j) : 0u;
    const bool tie = (j < nB) && b == tb;
    const uint32_t tmask = __ballot_sync(0xffffffffu, tie);
    const uint32_t rank = ties_before + __popc(tmask & lt_mask);
    const bool keep = (j < nB) && (b > tb || (tie && rank < need));
    const uint32_t kmask = __ballot_sync(0xffffffffu, keep);
    if (keep) out[base + __popc(kmask & lt_mask)] = j;
    base += __popc(kmask);
    ties_before += __popc(tmask);
  }
  if (lane == 0) counts[row] = base;
}

// Head scope in one launch, for segments that fit the cluster's shared memory:
// a cluster of kHC CTAs per (batch, head) segment of nQ x nB scores (rows of
// nB; flat index i*nB + j).  CTA r owns rows [r*rpc, (r+1)*rpc), rpc =
// ceil(nQ / kHC), and keeps them in shared memory after the first pass.  Each
// of the three 10-bit digit passes builds the CTA's exact histogram of
// fixed-point weights (16/17-bit split 32-bit shared atomics, folded into
// 64-bit bins every 2^15 scores, so the 32-bit sums stay exact); the cluster
// sums the bins through distributed shared memory (CTA r reduces bins
// [128r, 128r + 128)) and every CTA takes the same digit decision from the
// same sums.  Ties (scores equal to the threshold value) are ranked in flat
// order from per-row counts and the CTAs' totals; then each warp emits rows.
// All control flow that spans cluster barriers is uniform over the cluster.
constexpr int kHC = 8;
constexpr int kHCT = 1024;                    // threads a CTA (one histogram bin each)
static_assert(kHCT == kBins, "the digit decision gives each thread one bin");
constexpr int kHCMaxRows = 2 * kHCT;          // rows a CTA can own
constexpr int kHCMaxSlice = 40960;            // scores a CTA keeps in shared memory (160 KB)

// S[i] = weight of bins >= t + i over the CTA's 1024 bins (one a thread)
__device__ __forceinline__ void hc_suffix(const unsigned long long (&v)[1], unsigned long long (&S)[2],
                                          unsigned long long* warp_tot) {
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  unsigned long long x = v[0];
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_down_sync(0xffffffffu, x, o);
    if (lane + o < 32) x += y;
  }
  if (lane == 0) warp_tot[w] = x;
  __syncthreads();
  unsigned long long later = 0;
  for (int u = w + 1; u < kHCT / 32; ++u) later += warp_tot[u];
  S[0] = x + later;
  S[1] = S[0] - v[0];
  __syncthreads();                            // warp_tot is reused by the next call
}

__global__ void __cluster_dims__(kHC, 1, 1) __launch_bounds__(kHCT)
head_select_cluster_kernel(const float* __restrict__ scores, int nQ, int nB, uint32_t Pfix, int keep_all_p,
                           int32_t* __restrict__ counts, int32_t* __restrict__ cols, int32_t* __restrict__ status) {
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  extern __shared__ __align__(16) uint32_t slice[];   // this CTA's rows, [row][nB] score bits
  __shared__ uint32_t h_lo[kBins], h_hi[kBins];
  __shared__ unsigned long long h64[kBins];    // this CTA's histogram of the pass
  __shared__ unsigned long long red[kBins / kHC];   // bins [r*128, r*128 + 128) summed over the cluster
  __shared__ unsigned long long warp_tot[kHCT / 32];
  __shared__ int tiecnt[kHCMaxRows];
  __shared__ unsigned int s_max, s_ties;
  __shared__ int s_bad;
  __shared__ unsigned long long s_state[2];    // T, above
  __shared__ unsigned int s_dec[4];            // prefix, tb, need, mode (0 search, 1 resolved, 2 keep all)
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int r = static_cast<int>(cl.block_rank());
  const long long g = blockIdx.x / kHC;
  const int rpc = (nQ + kHC - 1) / kHC;
  const int r0 = min(nQ, r * rpc), r1 = min(nQ, r0 + rpc);
  const uint32_t* x = reinterpret_cast<const uint32_t*>(scores) + (g * nQ + r0) * static_cast<long long>(nB);
  const int n = (r1 - r0) * nB;                // this CTA's scores (<= kHCMaxSlice)
  if (t == 0) {
    s_max = 0;
    s_bad = 0;
    s_dec[0] = 0;
    s_dec[3] = keep_all_p ? 2u : 0u;
    s_state[1] = 0;
  }
  __syncthreads();
  for (int pass = 0; pass < 3; ++pass) {
    const bool search = s_dec[3] == 0 || pass == 0;   // uniform: every CTA holds the same decision
    if (search) {
      const int shift = 20 - kDigitBits * pass;
      const unsigned int prefix = s_dec[0];
      for (int i = t; i < kBins; i += kHCT) {
        h_lo[i] = 0u;
        h_hi[i] = 0u;
        h64[i] = 0ull;
      }
      __syncthreads();
      unsigned int lmax = 0;
      int lbad = 0;
      auto bin_one = [&](uint32_t b) {
        if (b >= kInvalidBits) {
          lbad = 1;
          return;
        }
        if (pass == 0) lmax = max(lmax, b);
        if (pass > 0 && (b >> (shift + kDigitBits)) != prefix) return;
        const uint64_t w = fixed_weight(b);
        if (w) {
          const uint32_t bin = (b >> shift) & (kBins - 1);
          atomicAdd(&h_lo[bin], static_cast<uint32_t>(w & 0xFFFFull));
          atomicAdd(&h_hi[bin], static_cast<uint32_t>(w >> 16));
        }
      };
      // rounds of at most 2^15 scores: 16-bit low parts sum below 2^31, 17-bit high parts below 2^32
      for (int q0 = 0; q0 < n; q0 += 32768) {
        const int q1 = min(n, q0 + 32768);
        if (pass == 0) {
          // from global memory (16-byte loads when rows are whole 16-byte units), kept in shared memory
          if ((nB & 3) == 0) {
            for (int i0 = q0 + 4 * t; i0 < q1; i0 += 4 * kHCT * 4) {
              uint4 v[4];
#pragma unroll
              for (int u = 0; u < 4; ++u)
                v[u] = (i0 + 4 * kHCT * u < q1) ? __ldg(reinterpret_cast<const uint4*>(x + i0 + 4 * kHCT * u))
                                                 : make_uint4(0, 0, 0, 0);
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const int i = i0 + 4 * kHCT * u;
                if (i >= q1) break;
                *reinterpret_cast<uint4*>(slice + i) = v[u];
                bin_one(v[u].x);
                bin_one(v[u].y);
                bin_one(v[u].z);
                bin_one(v[u].w);
              }
            }
          } else {
            for (int i = q0 + t; i < q1; i += kHCT) {
              const uint32_t b = __ldg(x + i);
              slice[i] = b;
              bin_one(b);
            }
          }
        } else {
          for (int i = q0 + t; i < q1; i += kHCT) bin_one(slice[i]);
        }
        __syncthreads();
        for (int i = t; i < kBins; i += kHCT) {
          h64[i] += (static_cast<unsigned long long>(h_hi[i]) << 16) + h_lo[i];
          h_lo[i] = 0u;
          h_hi[i] = 0u;
        }
        __syncthreads();
      }
      if (pass == 0) {
        atomicMax(&s_max, lmax);
        if (lbad) atomicOr(&s_bad, 1);
      }
    }
    cl.sync();                                 // every CTA's h64, s_max, s_bad are final
    if (search) {
      if (t < kBins / kHC) {
        unsigned long long acc = 0;
        for (int q = 0; q < kHC; ++q) acc += cl.map_shared_rank(h64, q)[r * (kBins / kHC) + t];
        red[t] = acc;
      }
      if (pass == 0 && t == kHCT - 1) {
        unsigned int mx = 0;
        int bad = 0;
        for (int q = 0; q < kHC; ++q) {
          mx = max(mx, *cl.map_shared_rank(&s_max, q));
          bad |= *cl.map_shared_rank(&s_bad, q);
        }
        s_dec[1] = mx;                         // the threshold value if T turns out 0
        s_dec[2] = static_cast<unsigned int>(bad);
      }
    }
    cl.sync();                                 // every CTA's red is final
    if (search) {
      unsigned long long v[1];
      v[0] = cl.map_shared_rank(red, t / (kBins / kHC))[t % (kBins / kHC)];
      unsigned long long S[2];
      hc_suffix(v, S, warp_tot);               // (its barriers also publish s_dec[1..2])
      if (pass == 0 && t == 0) {
        if (s_dec[2]) {
          if (r == 0) raise_status(status, LBSA_ERR_INVALID_SCORES);
          s_dec[3] = 2u;
        } else if (s_dec[3] != 2u) {
          s_state[0] = threshold_T(S[0], Pfix);
          s_state[1] = 0;
          if (s_state[0] == 0) {
            s_dec[2] = 1u;                     // keep one: the highest score (tb = the max), lowest index
            s_dec[3] = 1u;
          }
        }
      }
      __syncthreads();
      if (s_dec[3] == 0) {
        const unsigned long long T = s_state[0], above = s_state[1];
        const unsigned int prefix = s_dec[0];
        __syncthreads();
#pragma unroll
        for (int i = 0; i < 1; ++i) {
          if (above + S[i] >= T && above + S[i + 1] < T) {
            const unsigned int b = static_cast<unsigned int>(t + i);
            s_state[1] = above + S[i + 1];
            s_dec[0] = (prefix << kDigitBits) | b;
            if (pass == 2) {
              const unsigned int tb = (prefix << kDigitBits) | b;
              const unsigned long long ww = fixed_weight(tb);
              s_dec[1] = tb;
              s_dec[2] = static_cast<unsigned int>((T - (above + S[i + 1]) + ww - 1) / ww);
              s_dec[3] = 1u;
            }
          }
        }
      }
      __syncthreads();
    }
  }
  const bool all = s_dec[3] == 2u;
  const uint32_t tb = s_dec[1], need = s_dec[2];
  // ties per row of this CTA, the CTA's total, and the cluster's totals before it
  if (t == 0) s_ties = 0;
  __syncthreads();
  for (int i = warp; i < r1 - r0; i += kHCT / 32) {
    int c = 0;
    if (!all)
      for (int j = lane; j < nB; j += 32) c += (slice[i * nB + j] == tb);
    c = __reduce_add_sync(0xffffffffu, static_cast<unsigned>(c));
    if (lane == 0) {
      tiecnt[i] = c;
      atomicAdd(&s_ties, static_cast<unsigned>(c));
    }
  }
  __syncthreads();
  cl.sync();
  unsigned int base = 0;
  for (int q = 0; q < r; ++q) base += *cl.map_shared_rank(&s_ties, q);
  cl.sync();                                   // no CTA leaves while another reads its total
  {
    // exclusive scan of the rows' tie counts (at most kHCMaxRows = 2 x kHCT rows)
    const int nr = r1 - r0;
    const int a = (2 * t < nr) ? tiecnt[2 * t] : 0, b = (2 * t + 1 < nr) ? tiecnt[2 * t + 1] : 0;
    unsigned int incl = static_cast<unsigned int>(a + b);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    unsigned int before = base + incl - static_cast<unsigned int>(a + b);
    for (int u = 0; u < warp; ++u) before += static_cast<unsigned int>(warp_tot[u]);
    __syncthreads();
    if (2 * t < nr) tiecnt[2 * t] = static_cast<int>(before);
    if (2 * t + 1 < nr) tiecnt[2 * t + 1] = static_cast<int>(before + a);
  }
  __syncthreads();
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int i = warp; i < r1 - r0; i += kHCT / 32) {
    const long long row = g * nQ + r0 + i;
    int32_t* out = cols + row * nB;
    if (all) {
      for (int j = lane; j < nB; j += 32) out[j] = j;
      if (lane == 0) counts[row] = nB;
      continue;
    }
    const uint32_t* xr = slice + i * nB;
    uint32_t ties_before = static_cast<uint32_t>(tiecnt[i]);
    int cnt = 0;
    for (int j0 = 0; j0 < nB; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t b = (j < nB) ? xr[j] : 0u;
      const bool tie = (j < nB) && b == tb;
      const uint32_t tmask = __ballot_sync(0xffffffffu, tie);
      const uint32_t rank = ties_before + __popc(tmask & lt_mask);
      const bool keep = (j < nB) && (b > tb || (tie && rank < need));
      const uint32_t kmask = __ballot_sync(0xffffffffu, keep);
      if (keep) out[cnt + __popc(kmask & lt_mask)] = j;
      cnt += __popc(kmask);
      ties_before += __popc(tmask);
    }
    if (lane == 0) counts[row] = cnt;
  }
}

// Per-token scope: emit, for each query block, the key blocks kept by at
// least one of its (up to 64) tokens, ascending, each with the 64-bit mask of
// the tokens that keep it.  One CTA (256 threads) per (head, query block):
// every warp decides 8 token rows in flat order (ties ranked across the head
// by the scanned per-row tie counts), the keep bits are transposed in shared
// memory, then the non-empty entries are compacted in ascending order.
constexpr int kTokMaxB = 4096;                // nB bound of per-token scope
__global__ void __launch_bounds__(256) token_emit_kernel(const float* __restrict__ scores, int G, int nQ, int nB,
                                                         const HeadState* __restrict__ st,
                                                         const int32_t* __restrict__ tiebase,
                                                         int32_t* __restrict__ counts, int32_t* __restrict__ cols,
                                                         uint64_t* __restrict__ masks) {
  __shared__ uint32_t keep[64][kTokMaxB / 32];   // [token][word of key blocks]
  __shared__ int wsum[8];
  const int nQB = (nQ + 63) >> 6;
  const int qb = blockIdx.x % nQB, g = blockIdx.x / nQB;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const HeadState* s = st + g;
  const int nW = (nB + 31) >> 5;
  const uint32_t lt_mask = (1u << lane) - 1u;
  const bool all = s->keep_all;
  const uint32_t tb = s->tb, need = s->need;
  for (int tt = warp; tt < 64; tt += 8) {
    const int r = qb * 64 + tt;
    if (r >= nQ) {
      for (int w = lane; w < nW; w += 32) keep[tt][w] = 0u;
      continue;
    }
    const uint32_t* x = reinterpret_cast<const uint32_t*>(scores) + (static_cast<long long>(g) * nQ + r) * nB;
    uint32_t ties_before = all ? 0u : static_cast<uint32_t>(tiebase[static_cast<long long>(g) * nQ + r]);
    // sixteen 32-column loads in flight before the first is used
    for (int j1 = 0; j1 < nB; j1 += 512) {
      uint32_t bv[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int j = j1 + 32 * u + lane;
        bv[u] = (j < nB) ? __ldg(x + j) : 0u;
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int j0 = j1 + 32 * u;
        if (j0 >= nB) break;
        const int j = j0 + lane;
        const uint32_t b = bv[u];
        const bool tie = (j < nB) && b == tb;
        const uint32_t tmask = __ballot_sync(0xffffffffu, tie);
        const uint32_t rank = ties_before + __popc(tmask & lt_mask);
        const bool k = (j < nB) && (all || b > tb || (tie && rank < need));
        const uint32_t kmask = __ballot_sync(0xffffffffu, k);
        if (lane == 0) keep[tt][j0 >> 5] = kmask;
        ties_before += __popc(tmask);
      }
    }
  }
  __syncthreads();
  // thread t owns key blocks [t*per, t*per + per): masks, then an ordered compaction
  const int per = (nB + 255) / 256;
  const int j_lo = threadIdx.x * per, j_hi = min(nB, j_lo + per);
  uint64_t m[(kTokMaxB + 255) / 256];
  int cnt = 0;
#pragma unroll
  for (int u = 0; u < (kTokMaxB + 255) / 256; ++u) {
    m[u] = 0ull;
    const int j = j_lo + u;
    if (u < per && j < j_hi) {
      for (int tt = 0; tt < 64; ++tt) m[u] |= static_cast<uint64_t>((keep[tt][j >> 5] >> (j & 31)) & 1u) << tt;
      cnt += (m[u] != 0ull);
    }
  }
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int pos = incl - cnt;
  for (int w = 0; w < warp; ++w) pos += wsum[w];
  const long long row = static_cast<long long>(g) * nQB + qb;
#pragma unroll
  for (int u = 0; u < (kTokMaxB + 255) / 256; ++u) {
    const int j = j_lo + u;
    if (u < per && j < j_hi && m[u]) {
      cols[row * nB + pos] = j;
      masks[row * nB + pos] = m[u];
      ++pos;
    }
  }
  if (threadIdx.x == 255) counts[row] = pos;
}

// ---------------------------------------------------------------- CSR export / import
__global__ void export_scan_kernel(const int32_t* __restrict__ counts, long long R, int32_t* __restrict__ row_ptr,
                                   int32_t* __restrict__ nnz) {
  __shared__ int buf[1024];
  __shared__ int carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (long long base = 0; base < R; base += 1024) {
    const long long i = base + threadIdx.x;
    const int v = (i < R) ? counts[i] : 0;
    buf[threadIdx.x] = v;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
      const int add = (threadIdx.x >= o) ? buf[threadIdx.x - o] : 0;
      __syncthreads();
      buf[threadIdx.x] += add;
      __syncthreads();
    }
    if (i < R) row_ptr[i] = carry + buf[threadIdx.x] - v;
    __syncthreads();
    if (threadIdx.x == 1023) carry += buf[1023];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    row_ptr[R] = carry;
    *nnz = carry;
  }
}

__global__ void export_copy_kernel(const int32_t* __restrict__ counts, const int32_t* __restrict__ cols, long long R,
                                   int nB, const int32_t* __restrict__ row_ptr, int32_t* __restrict__ col) {
  const int lane = threadIdx.x & 31;
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (row >= R) return;
  const int n = counts[row];
  const int32_t* src = cols + row * nB;
  int32_t* dst = col + row_ptr[row];
  for (int t = lane; t < n; t += 32) dst[t] = src[t];
}

__global__ void from_csr_kernel(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col, long long R,
                                int nB, int32_t* __restrict__ counts, int32_t* __restrict__ cols,
                                int32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (row >= R) return;
  const int a = row_ptr[row], n = row_ptr[row + 1] - a;
  if (n < 0 || n > nB) {
    if (lane == 0) {
      raise_status(status, LBSA_ERR_BAD_INDEX);
      counts[row] = 0;
    }
    return;
  }
  bool bad = false;
  for (int t = lane; t < n; t += 32) {
    const int c = col[a + t];
    bad |= (c < 0 || c >= nB);
    cols[row * nB + t] = c;
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) raise_status(status, LBSA_ERR_BAD_INDEX);
  if (lane == 0) counts[row] = n;
}

// Block bitmask of a blockset: row r's W = ceil(nB / 32) words, bit j % 32 of
// word j / 32 set when key block j is kept.  One warp per row: each lane builds
// its words from the row's ascending ids (a word's ids are a contiguous run).
__global__ void export_bitmask_kernel(const int32_t* __restrict__ counts, const int32_t* __restrict__ cols, long long R,
                                      int nB, uint32_t* __restrict__ bits) {
  const int lane = threadIdx.x & 31;
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (row >= R) return;
  const int W = (nB + 31) >> 5;
  const int n = counts[row];
  const int32_t* ids = cols + row * nB;
  uint32_t* out = bits + row * W;
  for (int w = lane; w < W; w += 32) out[w] = 0u;
  __syncwarp();
  for (int t = lane; t < n; t += 32) {
    const int j = ids[t];
    if (j >= 0 && j < nB) atomicOr(out + (j >> 5), 1u << (j & 31));
  }
}

// The inverse: ascending ids of the set bits, one warp per row (words in lane
// order, each lane's ids placed after the lower lanes' by a warp prefix count).
__global__ void from_bitmask_kernel(const uint32_t* __restrict__ bits, long long R, int nB,
                                    int32_t* __restrict__ counts, int32_t* __restrict__ cols,
                                    int32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (row >= R) return;
  const int W = (nB + 31) >> 5;
  const uint32_t* in = bits + row * W;
  int32_t* dst = cols + row * nB;
  const uint32_t tail = (nB & 31) ? ((1u << (nB & 31)) - 1u) : 0xffffffffu;
  int base = 0;
  bool bad = false;
  for (int w0 = 0; w0 < W; w0 += 32) {
    const int w = w0 + lane;
    uint32_t x = (w < W) ? in[w] : 0u;
    if (w == W - 1) {
      bad |= (x & ~tail) != 0u;                 // bits past nB
      x &= tail;
    }
    const int c = __popc(x);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int pos = base + incl - c;
    while (x) {
      const int b = __ffs(x) - 1;
      x &= x - 1;
      dst[pos++] = w * 32 + b;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) raise_status(status, LBSA_ERR_BAD_INDEX);
  if (lane == 0) counts[row] = base;
}

inline uint32_t fixed_p(double p) {
  return static_cast<uint32_t>(std::nearbyint(p * 16777216.0));   // ties to even in the default mode
}

// ---------------------------------------------------------------- rank rules
// Top-n of a row by rank (score bits descending, then lower id): one warp per
// row, lane l holds ids l, l+32, ...; a 30-step bisection on the bits with
// element counts finds the bits tb of the n-th ranked eligible element.
//   mode 0 (Local + TopK, VMoBA review, referee report major comment 2): the
//           row's own key block i = row % nB is kept and not ranked; n = k.
//   mode 1 (top-p with a per-head floor, SCOPE abstract): n = max(c, min(K, nB))
//           with c the threshold rule's count (already in the blockset) and K
//           the head's floor; rows with n == c are left as they are.
template <int EPL>
__global__ void __launch_bounds__(256) select_rank_kernel(const float* __restrict__ scores, int R, int nB, int mode,
                                                          int k, const int32_t* __restrict__ head_floor,
                                                          int32_t* __restrict__ counts, int32_t* __restrict__ cols,
                                                          int32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (row >= R) return;                       // warp-uniform
  const int diag = (mode == 0) ? static_cast<int>(row % nB) : -1;
  int n;
  if (mode == 0) {
    n = min(k, nB - 1);
  } else {
    const int c = counts[row];
    n = max(c, min(head_floor[row / nB], nB));
    if (n == c) return;
  }
  const uint32_t* x = reinterpret_cast<const uint32_t*>(scores) + row * nB;
  int32_t* out = cols + row * nB;
  uint32_t bits[EPL];
  bool bad = false;
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    const int idx = e * 32 + lane;
    bits[e] = (idx < nB) ? __ldg(x + idx) : 0u;
    bad |= (idx < nB) && (bits[e] >= kInvalidBits);
  }
  if (__any_sync(0xffffffffu, bad)) {
    if (lane == 0) raise_status(status, LBSA_ERR_INVALID_SCORES);
    for (int idx = lane; idx < nB; idx += 32) out[idx] = idx;
    if (lane == 0) counts[row] = nB;
    return;
  }
  uint32_t tb = 0u;                           // with n == 0 nothing is ranked in
  uint32_t need = 0u;
  if (n > 0) {
    // the bracket starts at the eligible scores' range: cnt(>= min) = all eligible >= n
    // and cnt(>= max + 1) = 0 < n; cnt(bits >= hi) is kept as hi moves
    uint32_t bmin = 0xFFFFFFFFu, bmax = 0u;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const int idx = e * 32 + lane;
      if (idx < nB && idx != diag) {
        bmin = min(bmin, bits[e]);
        bmax = max(bmax, bits[e]);
      }
    }
    uint32_t lo = __reduce_min_sync(0xffffffffu, bmin);   // invariant: cnt(bits >= lo) >= n > cnt(bits >= hi)
    uint32_t hi = __reduce_max_sync(0xffffffffu, bmax) + 1u;
    uint32_t c_hi = 0;
    while (hi - lo > 1) {
      const uint32_t mid = lo + ((hi - lo) >> 1);
      uint32_t c = 0;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        const int idx = e * 32 + lane;
        c += (idx < nB && idx != diag && bits[e] >= mid) ? 1u : 0u;
      }
      c = __reduce_add_sync(0xffffffffu, c);
      if (c >= static_cast<uint32_t>(n)) {
        lo = mid;
      } else {
        hi = mid;
        c_hi = c;
      }
    }
    tb = lo;
    need = static_cast<uint32_t>(n) - c_hi;   // c_hi = cnt(bits > tb)
  }
  // emit in ascending id order: the own block (mode 0), the ids ranked above tb,
  // and the first `need` ties at tb in id order
  int base = 0;
  uint32_t ties_before = 0;
  const uint32_t lt_mask = (1u << lane) - 1u;
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    const int idx = e * 32 + lane;
    const bool elig = idx < nB && idx != diag;
    const bool tie = n > 0 && elig && bits[e] == tb;
    const uint32_t tmask = __ballot_sync(0xffffffffu, tie);
    const uint32_t rank = ties_before + __popc(tmask & lt_mask);
    const bool keep = (idx == diag) || (n > 0 && elig && (bits[e] > tb || (tie && rank < need)));
    const uint32_t kmask = __ballot_sync(0xffffffffu, keep);
    if (keep) out[base + __popc(kmask & lt_mask)] = idx;
    base += __popc(kmask);
    ties_before += __popc(tmask);
  }
  if (lane == 0) counts[row] = base;
}

// One CTA of 256 threads per head: floor K = ceil(sum_i v_i c_i / sum_i v_i),
// v_i = valid tokens of query block i, in exact integers.
__global__ void __launch_bounds__(256) head_floor_kernel(const int32_t* __restrict__ counts, int nB, int block,
                                                         int n_valid, int32_t* __restrict__ head_floor) {
  __shared__ unsigned long long red[2][8];
  const int g = blockIdx.x, lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  unsigned long long num = 0, den = 0;
  for (int i = threadIdx.x; i < nB; i += blockDim.x) {
    const unsigned long long v = static_cast<unsigned long long>(min(block, n_valid - i * block));
    num += v * static_cast<unsigned long long>(counts[static_cast<long long>(g) * nB + i]);
    den += v;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    num += __shfl_xor_sync(0xffffffffu, num, o);
    den += __shfl_xor_sync(0xffffffffu, den, o);
  }
  if (lane == 0) {
    red[0][w] = num;
    red[1][w] = den;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long N = 0, D = 0;
    for (int u = 0; u < 8; ++u) {
      N += red[0][u];
      D += red[1][u];
    }
    head_floor[g] = static_cast<int32_t>((N + D - 1) / D);
  }
}

// ---------------------------------------------------------------- routed scope
// EG-Sparse abstract (readsearch.ai page of arXiv 2610.14672, "Competition
// Domains Matter"): heads whose scores have low entropy compete in a pool
// shared by a group of heads, the others keep per-row selection.
//   head entropy  mean over the head's rows of the entropy of the row's
//                 normalised scores, divided by ln(nB); a head is routed when
//                 it is below the threshold; routed heads form consecutive
//                 groups of `group` in head order
//   domain        a pool's members' row i (flat index m*nB + j, m the member's
//                 rank), or one high-entropy head's row i; each domain takes
//                 the fixed-point threshold rule above.
// High-entropy heads go through the row kernel (a one-head domain is a row);
// the pools go through domain_select_kernel.  Pool table of batch element b
// (int32, 2H + 2 entries): [0] = pool count np, [1 .. np + 1] = member
// offsets, [H + 2 ..] = member heads.

// Row entropy ln S - (sum_j x_j ln x_j) / S, S = sum_j x_j, in fp64 from fp32
// logarithms (0 ln 0 = 0; a zero row gives 0; invalid scores give NaN or a
// value the domain kernel rejects).  One warp per row, 8 rows per CTA; the CTA
// writes the sum of its rows' entropies (fixed reduction order throughout, so
// the result does not vary from run to run).  grid (ceil(nQ / 8), B*H).
constexpr int kEntRowsPerCta = 8;
__global__ void __launch_bounds__(256) row_entropy_kernel(const float* __restrict__ scores, int nQ, int nB,
                                                          double* __restrict__ part) {
  __shared__ double wsum[8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = blockIdx.y, i = blockIdx.x * kEntRowsPerCta + warp;
  double h = 0.0;
  if (i < nQ) {                               // warp-uniform
    const float* x = scores + (static_cast<long long>(g) * nQ + i) * nB;
    double S = 0.0, L = 0.0;
    for (int j = lane; j < nB; j += 32) {
      const float v = __ldg(x + j);
      if (v != 0.0f) {
        S += v;
        L += static_cast<double>(v) * static_cast<double>(logf(v));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      S += __shfl_xor_sync(0xffffffffu, S, o);
      L += __shfl_xor_sync(0xffffffffu, L, o);
    }
    h = (S == 0.0) ? 0.0 : log(S) - L / S;   // lane 0's value is the one used
  }
  if (lane == 0) wsum[warp] = h;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
#pragma unroll
    for (int u = 0; u < 8; ++u) s += wsum[u];
    part[static_cast<long long>(g) * gridDim.x + blockIdx.x] = s;
  }
}

// One CTA (256 threads) per batch element: head entropies (warp per head,
// fixed order over the row-entropy partials), then the domain table; optional
// caller copies of both.
__global__ void __launch_bounds__(256) route_kernel(const double* __restrict__ part, int n_part, int H, int nQ, int nB,
                                                    double threshold, int group, int32_t* __restrict__ dom,
                                                    int32_t* __restrict__ head_dom, double* __restrict__ ent_out,
                                                    int32_t* __restrict__ dom_out) {
  extern __shared__ double sh_ent[];          // [H]
  const int b = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const double inv = (nB > 1) ? 1.0 / (static_cast<double>(nQ) * log(static_cast<double>(nB))) : 0.0;
  for (int h = warp; h < H; h += 8) {
    const double* r = part + (static_cast<long long>(b) * H + h) * n_part;
    double s = 0.0;
    for (int c = lane; c < n_part; c += 32) s += r[c];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) {
      const double e = s * inv;
      sh_ent[h] = e;
      if (ent_out) ent_out[static_cast<long long>(b) * H + h] = e;
    }
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  int32_t* D = dom + static_cast<long long>(b) * (2 * H + 2);
  int32_t* off = D + 1;
  int32_t* mem = D + H + 2;
  int nd = 0, nm = 0, rank = 0;
  for (int h = 0; h < H; ++h) {               // routed heads, `group` to a pool, in head order (NaN is not below)
    const bool routed = sh_ent[h] < threshold;
    const int32_t id = routed ? rank / group : -1;
    if (routed) {
      if (rank % group == 0) off[nd++] = nm;
      mem[nm++] = h;
      ++rank;
    }
    head_dom[static_cast<long long>(b) * H + h] = id;
    if (dom_out) dom_out[static_cast<long long>(b) * H + h] = id;
  }
  off[nd] = nm;
  D[0] = nd;
}

// Sum over the CTA's 8 warps of a per-thread value below 2^54; uniform result.
__device__ __forceinline__ unsigned long long cta_sum_u64(unsigned long long v, unsigned long long (*red)[8],
                                                          int& parity) {
  const unsigned long long ws = warp_sum_u64(v);
  if ((threadIdx.x & 31) == 0) red[parity][threadIdx.x >> 5] = ws;
  __syncthreads();
  unsigned long long s = 0;
#pragma unroll
  for (int u = 0; u < 8; ++u) s += red[parity][u];
  parity ^= 1;                                // the next sum writes the other buffer
  return s;
}

// One CTA (256 threads) per (query block i, pool d, batch element b): the
// pool's M*nB scores are staged in shared memory, the threshold bits tb are
// found by a weighted radix select over the 30 significant bits in three
// 10-bit digits (exact 64-bit bin sums in shared memory), then every member
// row is emitted with the ties at tb ranked across the domain in flat order.
__global__ void __launch_bounds__(256) domain_select_kernel(const float* __restrict__ scores, int H, int nQ, int nB,
                                                            const int32_t* __restrict__ dom, uint32_t Pfix,
                                                            int keep_all, int32_t* __restrict__ counts,
                                                            int32_t* __restrict__ cols, int32_t* __restrict__ status) {
  extern __shared__ uint32_t sbits[];         // [M * nB], then M + 1 tie offsets
  __shared__ unsigned long long hist[kBins];
  __shared__ uint32_t h_lo[kBins], h_hi[kBins];
  __shared__ unsigned long long red[2][8];
  __shared__ uint32_t red_max[8];
  __shared__ unsigned long long s_above;
  __shared__ uint32_t s_prefix;
  const int i = blockIdx.x, d = blockIdx.y, b = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int32_t* D = dom + static_cast<long long>(b) * (2 * H + 2);
  if (d >= D[0]) return;                      // CTA-uniform
  const int m0 = D[1 + d], M = D[2 + d] - m0;
  const int32_t* mem = D + H + 2 + m0;
  const int n = M * nB;
  int32_t* tie_off = reinterpret_cast<int32_t*>(sbits + n);
  unsigned long long wsum = 0;
  uint32_t mx = 0;
  int bad = 0;
  for (int m = 0; m < M; ++m) {
    const uint32_t* x =
        reinterpret_cast<const uint32_t*>(scores) + ((static_cast<long long>(b) * H + mem[m]) * nQ + i) * nB;
    for (int j = threadIdx.x; j < nB; j += blockDim.x) {
      const uint32_t v = __ldg(x + j);
      sbits[m * nB + j] = v;
      if (v >= kInvalidBits) {
        bad = 1;
      } else {
        wsum += fixed_weight(v);
        mx = max(mx, v);
      }
    }
  }
  int parity = 0;
  mx = __reduce_max_sync(0xffffffffu, mx);
  if (lane == 0) red_max[warp] = mx;
  const int any_bad = __syncthreads_or(bad);
  const unsigned long long W = cta_sum_u64(wsum, red, parity);
  mx = 0;
#pragma unroll
  for (int u = 0; u < 8; ++u) mx = max(mx, red_max[u]);
  if (any_bad || keep_all) {
    if (any_bad && threadIdx.x == 0) raise_status(status, LBSA_ERR_INVALID_SCORES);
    for (int m = warp; m < M; m += 8) {
      const long long r = (static_cast<long long>(b) * H + mem[m]) * nQ + i;
      for (int j = lane; j < nB; j += 32) cols[r * nB + j] = j;
      if (lane == 0) counts[r] = nB;
    }
    return;
  }
  const unsigned long long T = threshold_T(W, Pfix);
  uint32_t tb, need;
  if (T == 0) {
    tb = mx;                                  // keep one pair: the highest score, lowest flat index
    need = 1;
  } else {
    if (threadIdx.x == 0) {
      s_above = 0;
      s_prefix = 0;
    }
    for (int pass = 0; pass < 3; ++pass) {
      const int shift = 20 - kDigitBits * pass;
#pragma unroll
      for (int u = 0; u < kBins / 256; ++u) {
        hist[threadIdx.x + 256 * u] = 0ull;
        h_lo[threadIdx.x + 256 * u] = 0u;
        h_hi[threadIdx.x + 256 * u] = 0u;
      }
      __syncthreads();                        // bins cleared; s_prefix / s_above of the last pass visible
      const uint32_t prefix = s_prefix;
      const unsigned long long above = s_above;
      // exact bins: 16 low and 17 high bits of each weight (< 2^33) summed with
      // 32-bit shared atomics, folded into the 64-bit bins every 2^15 scores so
      // that neither 32-bit sum can wrap
      for (int q0 = 0; q0 < n; q0 += 32768) {
        const int q1 = min(n, q0 + 32768);
        for (int e = q0 + threadIdx.x; e < q1; e += blockDim.x) {
          const uint32_t v = sbits[e];
          if (pass > 0 && (v >> (shift + kDigitBits)) != prefix) continue;
          const unsigned long long w = fixed_weight(v);
          if (w) {
            const uint32_t bin = (v >> shift) & (kBins - 1);
            atomicAdd(&h_lo[bin], static_cast<uint32_t>(w & 0xFFFFull));
            atomicAdd(&h_hi[bin], static_cast<uint32_t>(w >> 16));
          }
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < kBins / 256; ++u) {
          const int t = threadIdx.x + 256 * u;
          hist[t] += (static_cast<unsigned long long>(h_hi[t]) << 16) + h_lo[t];
          h_lo[t] = 0u;
          h_hi[t] = 0u;
        }
        __syncthreads();
      }
      // thread t owns bins 4t .. 4t+3: suffix sums S[k] = weight of bins >= 4t + k
      unsigned long long hv[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) hv[k] = hist[4 * threadIdx.x + k];
      unsigned long long x = (hv[0] + hv[1]) + (hv[2] + hv[3]);
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long y = __shfl_down_sync(0xffffffffu, x, o);
        if (lane + o < 32) x += y;
      }
      if (lane == 0) red[parity][warp] = x;
      __syncthreads();
      unsigned long long later = 0;
      for (int u = warp + 1; u < 8; ++u) later += red[parity][u];
      parity ^= 1;
      unsigned long long S[5];
      S[0] = x + later;
#pragma unroll
      for (int k = 0; k < 4; ++k) S[k + 1] = S[k] - hv[k];
      // the largest bin with above + S(bin) >= T (it exists: the prefix's elements reach T - above);
      // every thread read prefix / above before the binning barrier, so they may change now
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (above + S[k] >= T && above + S[k + 1] < T) {
          s_prefix = (prefix << kDigitBits) | static_cast<uint32_t>(4 * threadIdx.x + k);
          s_above = above + S[k + 1];
        }
      }
    }
    __syncthreads();
    tb = s_prefix;
    const unsigned long long ww = fixed_weight(tb);   // > 0: the chosen bin holds weight
    need = static_cast<uint32_t>((T - s_above + ww - 1) / ww);
  }
  // ties at tb per member, then their exclusive offsets in flat order
  for (int m = warp; m < M; m += 8) {
    int c = 0;
    for (int j = lane; j < nB; j += 32) c += (sbits[m * nB + j] == tb);
    c = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(c)));
    if (lane == 0) tie_off[m + 1] = c;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    tie_off[0] = 0;
    for (int m = 0; m < M; ++m) tie_off[m + 1] += tie_off[m];
  }
  __syncthreads();
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int m = warp; m < M; m += 8) {
    const long long r = (static_cast<long long>(b) * H + mem[m]) * nQ + i;
    int32_t* out = cols + r * nB;
    uint32_t ties_before = static_cast<uint32_t>(tie_off[m]);
    int base = 0;
    for (int j0 = 0; j0 < nB; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t v = (j < nB) ? sbits[m * nB + j] : 0u;
      const bool tie = (j < nB) && v == tb;
      const uint32_t tmask = __ballot_sync(0xffffffffu, tie);
      const uint32_t rank = ties_before + __popc(tmask & lt_mask);
      const bool keep = (j < nB) && (v > tb || (tie && rank < need));
      const uint32_t kmask = __ballot_sync(0xffffffffu, keep);
      if (keep) out[base + __popc(kmask & lt_mask)] = j;
      base += __popc(kmask);
      ties_before += __popc(tmask);
    }
    if (lane == 0) counts[r] = base;
  }
}

}  // namespace

// skip_head: see select_row_kernel (NULL for plain row scope)
static cudaError_t launch_select_wide(const float* scores, int R, int nB, int kind, uint32_t P, int keep_all, int k,
                                      const int32_t* head_floor, lbsa_blockset* bs, const int32_t* skip_head,
                                      cudaStream_t s) {
  if (nB > 4096) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(R));
#define LBSA_WIDE(EPT)                                                                                             \
  select_wide_kernel<EPT><<<grid, kWideThreads, 0, s>>>(scores, R, nB, kind, P, keep_all, k, head_floor, bs->counts, \
                                                         bs->cols, bs->status, skip_head)
  if (nB <= 2048) LBSA_WIDE(8);
  else LBSA_WIDE(16);
#undef LBSA_WIDE
  return cudaGetLastError();
}

static cudaError_t launch_select_row_skip(const float* scores, int R, int nB, double p, lbsa_blockset* bs, cudaStream_t s,
                                   const int32_t* skip_head) {
  const uint32_t P = fixed_p(p);
  const int keep_all = p >= 1.0 ? 1 : 0;
  // two warps (rows) per block: residency is then bounded by registers, not by
  // the block granularity of the register-heavy wide-row instantiations
  const int threads = kRowThreads;
  const long long blocks = (static_cast<long long>(R) * 32 + threads - 1) / threads;
  dim3 grid(static_cast<unsigned>(blocks));
#define LBSA_SEL(EPL)                                                                                       \
  select_row_kernel<EPL><<<grid, threads, 0, s>>>(scores, R, nB, P, keep_all, bs->counts, bs->cols, bs->status, \
                                                  skip_head)
  if (nB <= 32) LBSA_SEL(1);
  else if (nB <= 64) LBSA_SEL(2);
  else if (nB <= 128) LBSA_SEL(4);
  else if (nB <= 256) LBSA_SEL(8);
  else if (nB <= 512) LBSA_SEL(16);
  else if (nB <= 1024) LBSA_SEL(32);
  else return launch_select_wide(scores, R, nB, 0, P, keep_all, 0, nullptr, bs, skip_head, s);
#undef LBSA_SEL
  return cudaGetLastError();
}

cudaError_t launch_select_row(const float* scores, int R, int nB, double p, lbsa_blockset* bs, cudaStream_t s) {
  return launch_select_row_skip(scores, R, nB, p, bs, s, nullptr);
}

cudaError_t launch_select_rank(const float* scores, int R, int nB, int mode, int k, const int32_t* head_floor,
                               lbsa_blockset* bs, cudaStream_t s) {
  const int threads = 256;
  dim3 grid(static_cast<unsigned>((static_cast<long long>(R) * 32 + threads - 1) / threads));
#define LBSA_RANK(EPL)                                                                                     \
  select_rank_kernel<EPL><<<grid, threads, 0, s>>>(scores, R, nB, mode, k, head_floor, bs->counts, bs->cols, \
                                                   bs->status)
  if (nB <= 32) LBSA_RANK(1);
  else if (nB <= 64) LBSA_RANK(2);
  else if (nB <= 128) LBSA_RANK(4);
  else if (nB <= 256) LBSA_RANK(8);
  else if (nB <= 512) LBSA_RANK(16);
  else if (nB <= 1024) LBSA_RANK(32);
  else return launch_select_wide(scores, R, nB, mode == 0 ? 1 : 2, 0u, 0, k, head_floor, bs, nullptr, s);
#undef LBSA_RANK
  return cudaGetLastError();
}

cudaError_t launch_head_floor(const int32_t* counts, int G, int nB, int block, int n_valid, int32_t* head_floor,
                              cudaStream_t s) {
  head_floor_kernel<<<G, 256, 0, s>>>(counts, nB, block, n_valid, head_floor);
  return cudaGetLastError();
}

// Histogram CTAs per head: at most kHistPerCta elements each (the 32-bit shared
// sums rely on that bound); fewer per CTA, down to 4,096, while the launch would
// otherwise hold fewer than four CTAs per SM.
static long long hist_chunks(long long seg, int G) {
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  long long per = kHistPerCta;
  while (per > 4096 && static_cast<long long>(G) * ((seg + per - 1) / per) < 4ll * sms) per >>= 1;
  return (seg + per - 1) / per;
}

bool select_head_one_launch(int nB) {
  return static_cast<long long>((nB + kHC - 1) / kHC) * nB <= kHCMaxSlice;
}

size_t select_head_workspace_bytes(int B, int H, int nB, int nQ) {
  const size_t G = static_cast<size_t>(B) * H;
  if (nQ <= 0) nQ = nB;
  return G * kBins * sizeof(unsigned long long) + G * sizeof(HeadState) + G * nQ * sizeof(int32_t) + 256;
}

cudaError_t launch_select_head(const float* scores, int B, int H, int nB, double p, lbsa_blockset* bs, void* ws,
                               cudaStream_t s) {
  const int G = B * H;
  if (select_head_one_launch(nB)) {
    const long long slice = static_cast<long long>((nB + kHC - 1) / kHC) * nB;
    // one launch: a cluster of kHC CTAs per head, each keeping its rows in shared memory
    const int smem = static_cast<int>(slice * sizeof(uint32_t));
    cudaError_t e = cudaFuncSetAttribute(head_select_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    head_select_cluster_kernel<<<static_cast<unsigned>(G) * kHC, kHCT, smem, s>>>(scores, nB, nB, fixed_p(p),
                                                                                 p >= 1.0 ? 1 : 0, bs->counts,
                                                                                 bs->cols, bs->status);
    return cudaGetLastError();
  }
  const long long seg = static_cast<long long>(nB) * nB;
  unsigned long long* hist = reinterpret_cast<unsigned long long*>(ws);
  HeadState* st = reinterpret_cast<HeadState*>(hist + static_cast<size_t>(G) * kBins);
  int32_t* tie = reinterpret_cast<int32_t*>(st + G);
  cudaError_t e = cudaMemsetAsync(ws, 0, static_cast<size_t>(G) * kBins * sizeof(unsigned long long) +
                                             static_cast<size_t>(G) * sizeof(HeadState), s);
  if (e != cudaSuccess) return e;
  const uint32_t P = fixed_p(p);
  const int keep_all = p >= 1.0 ? 1 : 0;
  const int chunks = static_cast<int>(hist_chunks(seg, G));
  for (int pass = 0; pass < 3; ++pass) {
    head_hist_kernel<<<dim3(chunks, G), 256, 0, s>>>(scores, seg, pass, P, keep_all, hist, st, bs->status);
  }
  const long long rows = static_cast<long long>(G) * nB;
  const unsigned wblocks = static_cast<unsigned>((rows * 32 + 255) / 256);
  head_tiecount_kernel<<<wblocks, 256, 0, s>>>(scores, G, nB, nB, st, tie);
  head_tiescan_kernel<<<G, 1024, 0, s>>>(nB, st, tie);
  head_emit_kernel<<<wblocks, 256, 0, s>>>(scores, G, nB, st, tie, bs->counts, bs->cols);
  return cudaGetLastError();
}

cudaError_t launch_select_tokens(const float* scores, int B, int H, int nQ, int nB, double p, lbsa_blockset* bs,
                                 void* ws, cudaStream_t s) {
  if (nB > kTokMaxB) return cudaErrorInvalidValue;
  const int G = B * H;
  const long long seg = static_cast<long long>(nQ) * nB;
  unsigned long long* hist = reinterpret_cast<unsigned long long*>(ws);
  HeadState* st = reinterpret_cast<HeadState*>(hist + static_cast<size_t>(G) * kBins);
  int32_t* tie = reinterpret_cast<int32_t*>(st + G);
  cudaError_t e = cudaMemsetAsync(ws, 0, static_cast<size_t>(G) * kBins * sizeof(unsigned long long) +
                                             static_cast<size_t>(G) * sizeof(HeadState), s);
  if (e != cudaSuccess) return e;
  const uint32_t P = fixed_p(p);
  const int keep_all = p >= 1.0 ? 1 : 0;
  const long long chunks = hist_chunks(seg, G);
  if (chunks > 65535) return cudaErrorInvalidValue;
  const unsigned hc = static_cast<unsigned>(chunks);
  for (int pass = 0; pass < 3; ++pass) {
    head_hist_kernel<<<dim3(hc, G), 256, 0, s>>>(scores, seg, pass, P, keep_all, hist, st, bs->status);
  }
  const long long rows = static_cast<long long>(G) * nQ;
  const unsigned wblocks = static_cast<unsigned>((rows * 32 + 255) / 256);
  head_tiecount_kernel<<<wblocks, 256, 0, s>>>(scores, G, nQ, nB, st, tie);
  head_tiescan_kernel<<<G, 1024, 0, s>>>(nQ, st, tie);
  const int nQB = (nQ + 63) / 64;
  token_emit_kernel<<<static_cast<unsigned>(G) * nQB, 256, 0, s>>>(scores, G, nQ, nB, st, tie, bs->counts, bs->cols,
                                                                  bs->masks);
  return cudaGetLastError();
}

size_t select_routed_workspace_bytes(int B, int H, int nB) {
  const size_t parts = static_cast<size_t>(B) * H * ((nB + kEntRowsPerCta - 1) / kEntRowsPerCta);
  return parts * sizeof(double) + static_cast<size_t>(B) * (3 * H + 2) * sizeof(int32_t) + 256;
}

size_t select_routed_smem_bytes(int H, int nB, int group) {
  const int M = group < H ? group : H;
  return static_cast<size_t>(M) * nB * sizeof(uint32_t) + static_cast<size_t>(M + 1) * sizeof(int32_t);
}

cudaError_t launch_select_routed(const float* scores, int B, int H, int nB, double p, double threshold, int group,
                                 double* ent_out, int32_t* dom_out, lbsa_blockset* bs, void* ws, cudaStream_t s) {
  const int n_part = (nB + kEntRowsPerCta - 1) / kEntRowsPerCta;
  double* part = reinterpret_cast<double*>(ws);
  int32_t* head_dom = reinterpret_cast<int32_t*>(part + static_cast<size_t>(B) * H * n_part);
  int32_t* dom = head_dom + static_cast<size_t>(B) * H;
  row_entropy_kernel<<<dim3(n_part, B * H), 256, 0, s>>>(scores, nB, nB, part);
  route_kernel<<<B, 256, static_cast<size_t>(H) * sizeof(double), s>>>(part, n_part, H, nB, nB, threshold, group, dom,
                                                                      head_dom, ent_out, dom_out);
  cudaError_t e = launch_select_row_skip(scores, B * H * nB, nB, p, bs, s, head_dom);
  if (e != cudaSuccess) return e;
  const size_t smem = select_routed_smem_bytes(H, nB, group);
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(domain_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  const int max_pools = (H + group - 1) / group;
  domain_select_kernel<<<dim3(nB, max_pools, B), 256, smem, s>>>(scores, H, nB, nB, dom, fixed_p(p),
                                                                 p >= 1.0 ? 1 : 0, bs->counts, bs->cols, bs->status);
  return cudaGetLastError();
}

cudaError_t launch_export_csr(const lbsa_blockset* bs, int32_t* row_ptr, int32_t* col, int32_t* nnz_dev,
                              cudaStream_t s) {
  const long long R = static_cast<long long>(bs->B) * bs->H * bs->nB;
  export_scan_kernel<<<1, 1024, 0, s>>>(bs->counts, R, row_ptr, nnz_dev);
  export_copy_kernel<<<static_cast<unsigned>((R * 32 + 255) / 256), 256, 0, s>>>(bs->counts, bs->cols, R, bs->nB,
                                                                               row_ptr, col);
  return cudaGetLastError();
}

cudaError_t launch_export_bitmask(const lbsa_blockset* bs, uint32_t* bits, cudaStream_t s) {
  const long long R = static_cast<long long>(bs->B) * bs->H * bs->nB;
  export_bitmask_kernel<<<static_cast<unsigned>((R * 32 + 255) / 256), 256, 0, s>>>(bs->counts, bs->cols, R, bs->nB,
                                                                                     bits);
  return cudaGetLastError();
}

cudaError_t launch_from_bitmask(const uint32_t* bits, lbsa_blockset* bs, cudaStream_t s) {
  const long long R = static_cast<long long>(bs->B) * bs->H * bs->nB;
  from_bitmask_kernel<<<static_cast<unsigned>((R * 32 + 255) / 256), 256, 0, s>>>(bits, R, bs->nB, bs->counts,
                                                                                   bs->cols, bs->status);
  return cudaGetLastError();
}

cudaError_t launch_from_csr(const int32_t* row_ptr, const int32_t* col, lbsa_blockset* bs, cudaStream_t s) {
  const long long R = static_cast<long long>(bs->B) * bs->H * bs->nB;
  from_csr_kernel<<<static_cast<unsigned>((R * 32 + 255) / 256), 256, 0, s>>>(row_ptr, col, R, bs->nB, bs->counts,
                                                                             bs->cols, bs->status);
  return cudaGetLastError();
}

}  // namespace lbsa

// ---------------------------------------------------------------- allocation-free head-scope selection
// lbsa_select_head_noalloc runs the same head-scope kernels as lbsa_select,
// but its scratch (radix histograms, per-head state, per-row tie counts) lives
// in the file-scope device array below instead of memory obtained at run time,
// and its outputs go to caller buffers.  The array is part of the loaded
// module: every GPU that loads the library holds it until the process exits.
namespace lbsa {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;   // 1 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_addr[64] = {};

// Device address of g_noalloc_scratch on the current device, looked up once
// per device.  In host code the array's name is only a host-side stand-in,
// never a device address, so kernels are always given this pointer.
cudaError_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace lbsa

extern "C" int lbsa_select_head_noalloc(const float* scores, int32_t B, int32_t H, int32_t nB, double p,
                                        int32_t* counts, int32_t* cols, int32_t* status, void* stream) {
  using namespace lbsa;
  if (!scores || (reinterpret_cast<uintptr_t>(scores) & 15u))
    return set_error(LBSA_ERR_INVALID_ARG, "scores must be a non-NULL, 16-byte aligned device pointer");
  if (!counts || !cols || !status) return set_error(LBSA_ERR_INVALID_ARG, "counts, cols and status must be non-NULL");
  if (B < 1 || H < 1 || nB < 1) return set_error(LBSA_ERR_INVALID_ARG, "B, H, nB must be >= 1");
  if (!(p > 0.0) || !(p <= 1.0)) return set_error(LBSA_ERR_INVALID_ARG, "p must lie in (0, 1]");
  // the same bound as lbsa_select's head scope (32-bit per-head counters need nB*nB < 2^32)
  if (nB > 4096) return set_error(LBSA_ERR_UNSUPPORTED, "head scope is built for nB <= 4096");
  const size_t need = select_head_workspace_bytes(B, H, nB);
  if (need > kNoAllocScratchBytes) {
    char msg[200];
    std::snprintf(msg, sizeof(msg),
                  "B*H=%lld heads with nB=%d need %zu bytes of scratch; the static array holds %zu "
                  "(B*H <= 64 with nB <= 1024 always fits)",
                  static_cast<long long>(B) * H, nB, need, kNoAllocScratchBytes);
    return set_error(LBSA_ERR_UNSUPPORTED, msg);
  }
  void* ws = nullptr;
  cudaError_t e = noalloc_scratch(&ws);
  if (e != cudaSuccess) return set_error(LBSA_ERR_CUDA, cudaGetErrorString(e));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int G = B * H;
  const long long seg = static_cast<long long>(nB) * nB;
  unsigned long long* hist = reinterpret_cast<unsigned long long*>(ws);
  HeadState* st = reinterpret_cast<HeadState*>(hist + static_cast<size_t>(G) * kBins);
  int32_t* tie = reinterpret_cast<int32_t*>(st + G);
  // the array keeps the previous call's contents: clear the histograms, the
  // per-head state and the caller's status word before the passes
  e = cudaMemsetAsync(ws, 0, static_cast<size_t>(G) * kBins * sizeof(unsigned long long) +
                                 static_cast<size_t>(G) * sizeof(HeadState), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(status, 0, sizeof(int32_t), s);
  if (e != cudaSuccess) return set_error(LBSA_ERR_CUDA, cudaGetErrorString(e));
  const uint32_t P = fixed_p(p);
  const int keep_all = p >= 1.0 ? 1 : 0;
  const int chunks = static_cast<int>(hist_chunks(seg, G));
  for (int pass = 0; pass < 3; ++pass) {
    head_hist_kernel<<<dim3(chunks, G), 256, 0, s>>>(scores, seg, pass, P, keep_all, hist, st, status);
  }
  const long long rows = static_cast<long long>(G) * nB;
  const unsigned wblocks = static_cast<unsigned>((rows * 32 + 255) / 256);
  head_tiecount_kernel<<<wblocks, 256, 0, s>>>(scores, G, nB, nB, st, tie);
  head_tiescan_kernel<<<G, 1024, 0, s>>>(nB, st, tie);
  head_emit_kernel<<<wblocks, 256, 0, s>>>(scores, G, nB, st, tie, counts, cols);
  e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(LBSA_ERR_CUDA, cudaGetErrorString(e));
  return LBSA_OK;
}
