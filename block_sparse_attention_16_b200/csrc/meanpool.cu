// Block-mean proxy scores (VMoBA review on pith.science, arXiv 2506.23858,
// "What carries the argument": each key block stands in as the mean of its
// keys, and queries score those means).  Block-granular reading: the query
// side is pooled the same way, and the similarities of one head are
// normalised by a softmax over all of its query-block x key-block pairs:
//   qbar_i = mean_{r in I_i} q_r,  kbar_j = mean_{c in J_j} k_c   (fp32)
//   s_ij = qbar_i . kbar_j / sqrt(d)
//   score[b,h,i,j] = exp(s_ij - M) / sum_{i',j'} exp(s_i'j' - M),  M = max s
// Three kernels: block means (reads Q and K once, 16-byte loads), the 64x64
// tiles of s with per-tile (max, sum of exp), and the normalisation.
//
// Per-token mode (the same review, referee report major comment 1: every
// query token against every key-block mean):
//   s_rj = q_r . kbar_j / sqrt(d),   score[b,h,r,j] = exp(s_rj - M) / Z
// over the head's n_valid x nB (token, key block) pairs; the logits kernel
// then reads its rows straight from Q instead of from the query-block means.
#include "lbsa_device.cuh"

#include <cuda_bf16.h>

namespace lbsa {
namespace {


int g_sms = 0;
int num_sms() {
  if (!g_sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_sms <= 0) g_sms = 148;
  }
  return g_sms;
}

// Eight consecutive columns of one row as raw 16-byte vectors (one for bf16,
// two for fp32), so that a thread's loads for a whole block can be issued
// before any of them is used.
template <typename T>
struct Raw8;
template <>
struct Raw8<__nv_bfloat16> {
  uint4 a;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { a = __ldg(reinterpret_cast<const uint4*>(p)); }
  __device__ __forceinline__ void add_to(float (&f)[8]) const {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&a);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 t = __bfloat1622float2(h[i]);
      f[2 * i] += t.x;
      f[2 * i + 1] += t.y;
    }
  }
};
template <>
struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = __ldg(reinterpret_cast<const float4*>(p));
    b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  }
  __device__ __forceinline__ void add_to(float (&f)[8]) const {
    f[0] += a.x; f[1] += a.y; f[2] += a.z; f[3] += a.w;
    f[4] += b.x; f[5] += b.y; f[6] += b.z; f[7] += b.w;
  }
};

// Persistent grid over the (b, h, block) items (blocks of at most MAXR
// tokens), 256 threads: thread = (row group g, 8-column vector v).  The loads of a thread's next item are issued
// before the current item's sums are reduced, so DRAM traffic continues
// through the reduction.  Reduction: lanes of a warp that share v by
// shuffles, then the eight warps through double-buffered shared memory (one
// barrier per item).  qs / ks (optional): the means' bf16 hi / lo terms for the
// tensor-core logits, hi = bf16(m) at [item*D + c], lo = bf16(m - hi) at n + that.
template <typename T, int D, int MAXR>
__global__ void __launch_bounds__(256) block_mean_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                         lbsa_qkv_desc desc, int block, int nB, long long items,
                                                         float* __restrict__ qbar, float* __restrict__ kbar,
                                                         __nv_bfloat16* __restrict__ qs, __nv_bfloat16* __restrict__ ks) {
  const long long nsplit = items * D;
  constexpr int V = D / 8;               // vectors per row
  constexpr int G = 256 / V;             // row groups
  constexpr int kMaxIt = MAXR / G;       // rows per thread at block = MAXR
  __shared__ float red[2][8][2 * D];
  const int v = threadIdx.x % V, g = threadIdx.x / V;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  Raw8<T> rq[kMaxIt], rk[kMaxIt];
  auto issue = [&](long long item) {
    const int i = static_cast<int>(item % nB);
    const long long bh = item / nB;
    const int h = static_cast<int>(bh % desc.H), bb = static_cast<int>(bh / desc.H);
    const int r0 = i * block, r1 = min(r0 + block, desc.N_valid);
    const long long base = bb * desc.stride_b + h * desc.stride_h + v * 8;
#pragma unroll
    for (int it = 0; it < kMaxIt; ++it) {
      const int r = r0 + g + it * G;
      if (r < r1) {
        rq[it].load(q + base + r * desc.stride_n);
        rk[it].load(k + base + r * desc.stride_n);
      }
    }
  };
  long long item = blockIdx.x;
  if (item < items) issue(item);
  for (int buf = 0; item < items; item += gridDim.x, buf ^= 1) {
    const int i = static_cast<int>(item % nB);
    const int r0 = i * block, r1 = min(r0 + block, desc.N_valid);
    float aq[8] = {0, 0, 0, 0, 0, 0, 0, 0}, ak[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int it = 0; it < kMaxIt; ++it) {
      if (r0 + g + it * G < r1) {
        rq[it].add_to(aq);
        rk[it].add_to(ak);
      }
    }
    if (item + gridDim.x < items) issue(item + gridDim.x);
#pragma unroll
    for (int o = V; o < 32; o <<= 1)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        aq[e] += __shfl_xor_sync(0xffffffffu, aq[e], o);
        ak[e] += __shfl_xor_sync(0xffffffffu, ak[e], o);
      }
    if (lane < V) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        red[buf][warp][v * 8 + e] = aq[e];
        red[buf][warp][D + v * 8 + e] = ak[e];
      }
    }
    __syncthreads();
    const float inv = 1.0f / static_cast<float>(r1 - r0);
    for (int c = threadIdx.x; c < 2 * D; c += blockDim.x) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) s += red[buf][w][c];
      const float m = s * inv;
      float* dst = c < D ? qbar : kbar;        // qbar is NULL when only the terms are wanted
      if (dst) dst[item * D + (c % D)] = m;
      __nv_bfloat16* sp = c < D ? qs : ks;
      if (sp) {
        const __nv_bfloat16 hi = __float2bfloat16_rn(m);
        sp[item * D + (c % D)] = hi;
        sp[nsplit + item * D + (c % D)] = __float2bfloat16_rn(m - __bfloat162float(hi));
      }
    }
  }
}

// Query tokens as logits rows: Q in its own dtype and strides, four columns at a time.
template <typename T>
struct TokenRows {
  const T* p;
  long long sb, sh, sn;
  int H;
  __device__ __forceinline__ float4 load(int g, int r, int c) const;
};
template <>
__device__ __forceinline__ float4 TokenRows<float>::load(int g, int r, int c) const {
  return __ldg(reinterpret_cast<const float4*>(p + (g / H) * sb + (g % H) * sh + r * sn + c));
}
template <>
__device__ __forceinline__ float4 TokenRows<__nv_bfloat16>::load(int g, int r, int c) const {
  const uint2 u = __ldg(reinterpret_cast<const uint2*>(p + (g / H) * sb + (g % H) * sh + r * sn + c));
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}

// grid (nTk, nTq, B*H) with nTk = ceil(nB/128), nTq = ceil(nQ/64); 128 threads.
// A CTA computes a 64 x 128 tile of s: rows are the nQ query blocks (qbar,
// fp32) or, in per-token mode, the nQ = n_valid query tokens read from Q;
// columns are key blocks (kbar).  Thread (y, x) of the 8 x 16 thread grid owns
// rows {4y..4y+3, 32+4y..32+4y+3} and columns {4x..4x+3, 64+4x..64+4x+3}, so
// that each 16-byte shared load of a warp (8 x 4 threads) touches distinct
// bank groups: 4 loads feed 64 FMAs.  Column chunks of 16 of d are staged
// transposed ([c][row], rows padded by 4) through registers, the next chunk's
// global loads in flight while the current one is used.  Every s_ij is summed
// over d in ascending order.
constexpr int kTq = 64, kTk = 128;
template <int D, typename TQ, bool TOK>
__global__ void __launch_bounds__(128) logits_kernel(const TQ* __restrict__ qsrc, long long q_sb, long long q_sh,
                                                     long long q_sn, int H, const float* __restrict__ kbar, int nQ,
                                                     int nB, float scale, float* __restrict__ scores,
                                                     float2* __restrict__ part) {
  constexpr int KC = 16;                 // columns of d staged per round
  constexpr int LQ = kTq + 4, LK = kTk + 4;
  __shared__ __align__(16) float sq[KC][LQ];
  __shared__ __align__(16) float sk[KC][LK];
  __shared__ float red_m[4], red_s[4];
  const int ti = blockIdx.y, tj = blockIdx.x, g = blockIdx.z;
  const int nTk = gridDim.x, nTq = gridDim.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float* kb = kbar + static_cast<long long>(g) * nB * D;
  const int y = lane >> 2, x = warp * 4 + (lane & 3);
  // accumulators as packed pairs of adjacent columns: acc2[u][v] = (s[u][2v], s[u][2v+1])
  unsigned long long acc2[8][4];
#pragma unroll
  for (int u = 0; u < 8; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) acc2[u][v] = 0ull;
  // staging: the q tile is 64 rows x 4 float4 (2 per thread), the kbar tile
  // 128 rows x 4 float4 (4 per thread); element e -> row e >> 2, columns 4*(e & 3)
  float4 na[2], nb[4];
  auto fetch = [&](int c0) {
#pragma unroll
    for (int it = 0; it < 2; ++it) {
      const int e = threadIdx.x + it * 128;
      const int r = e >> 2, c4 = (e & 3) * 4;
      const int qi = ti * kTq + r;
      if (qi < nQ) {
        if constexpr (TOK) {
          na[it] = (TokenRows<TQ>{qsrc, q_sb, q_sh, q_sn, H}).load(g, qi, c0 + c4);
        } else {
          na[it] = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(qsrc) +
                                                    (static_cast<long long>(g) * nQ + qi) * D + c0 + c4);
        }
      } else {
        na[it] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int e = threadIdx.x + it * 128;
      const int r = e >> 2, c4 = (e & 3) * 4;
      const int kj = tj * kTk + r;
      nb[it] = (kj < nB) ? *reinterpret_cast<const float4*>(kb + static_cast<long long>(kj) * D + c0 + c4)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  fetch(0);
  for (int c0 = 0; c0 < D; c0 += KC) {
#pragma unroll
    for (int it = 0; it < 2; ++it) {
      const int e = threadIdx.x + it * 128;
      const int r = e >> 2, c4 = (e & 3) * 4;
      sq[c4][r] = na[it].x; sq[c4 + 1][r] = na[it].y; sq[c4 + 2][r] = na[it].z; sq[c4 + 3][r] = na[it].w;
    }
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int e = threadIdx.x + it * 128;
      const int r = e >> 2, c4 = (e & 3) * 4;
      sk[c4][r] = nb[it].x; sk[c4 + 1][r] = nb[it].y; sk[c4 + 2][r] = nb[it].z; sk[c4 + 3][r] = nb[it].w;
    }
    __syncthreads();
    if (c0 + KC < D) fetch(c0 + KC);
#pragma unroll
    for (int c = 0; c < KC; ++c) {
      const float4 a0 = *reinterpret_cast<const float4*>(&sq[c][4 * y]);
      const float4 a1 = *reinterpret_cast<const float4*>(&sq[c][32 + 4 * y]);
      const float4 b0 = *reinterpret_cast<const float4*>(&sk[c][4 * x]);
      const float4 b1 = *reinterpret_cast<const float4*>(&sk[c][64 + 4 * x]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const unsigned long long bp[4] = {f2_as_u64(b0.x, b0.y), f2_as_u64(b0.z, b0.w), f2_as_u64(b1.x, b1.y),
                                        f2_as_u64(b1.z, b1.w)};
      // packed fp32x2 FMAs (each half an ordinary fp32 FMA: the same sums as scalar FMAs)
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const unsigned long long ap = f2_as_u64(av[u], av[u]);
#pragma unroll
        for (int v = 0; v < 4; ++v) acc2[u][v] = ffma2(ap, bp[v], acc2[u][v]);
      }
    }
    __syncthreads();
  }
  // epilogue: scale, store (16-byte vectors where the 4 columns are in range), tile (max, sum of exp)
  float acc[8][8];
#pragma unroll
  for (int u = 0; u < 8; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) u64_as_f2(acc2[u][v], acc[u][2 * v], acc[u][2 * v + 1]);
  float mx = -INFINITY;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int qi = ti * kTq + (u < 4 ? 4 * y + u : 32 + 4 * y + u - 4);
#pragma unroll
    for (int w = 0; w < 8; ++w) acc[u][w] *= scale;
    if (qi >= nQ) continue;
#pragma unroll
    for (int hx = 0; hx < 2; ++hx) {
      const int kj0 = tj * kTk + hx * 64 + 4 * x;
      float* dst = scores + (static_cast<long long>(g) * nQ + qi) * nB + kj0;
      const float* a = &acc[u][4 * hx];
      if ((nB & 3) == 0 && kj0 + 3 < nB) {
        *reinterpret_cast<float4*>(dst) = make_float4(a[0], a[1], a[2], a[3]);
        mx = fmaxf(mx, fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3])));
      } else {
#pragma unroll
        for (int w = 0; w < 4; ++w)
          if (kj0 + w < nB) {
            dst[w] = a[w];
            mx = fmaxf(mx, a[w]);
          }
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) red_m[warp] = mx;
  __syncthreads();
  const float tm = fmaxf(fmaxf(red_m[0], red_m[1]), fmaxf(red_m[2], red_m[3]));
  float sm = 0.f;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int qi = ti * kTq + (u < 4 ? 4 * y + u : 32 + 4 * y + u - 4);
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      const int kj = tj * kTk + (w < 4 ? 4 * x + w : 64 + 4 * x + w - 4);
      if (qi < nQ && kj < nB) sm += expf(acc[u][w] - tm);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
  if (lane == 0) red_s[warp] = sm;
  __syncthreads();
  if (threadIdx.x == 0)
    part[(static_cast<long long>(g) * nTq + ti) * nTk + tj] = make_float2(tm, (red_s[0] + red_s[1]) + (red_s[2] + red_s[3]));
}

// grid (chunks, B*H), 256 threads: warp 0 combines the head's tile partials
// (fixed order per lane, then a fixed shuffle tree), then the block
// normalises a chunk of the head's scores in place.
__global__ void normalize_kernel(float* __restrict__ scores, const float2* __restrict__ part, long long n,
                                 int n_part) {
  __shared__ float sM, sZ;
  const int g = blockIdx.y;
  const float2* pp = part + static_cast<long long>(g) * n_part;
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    float M = -INFINITY;
    for (int t = lane; t < n_part; t += 32) M = fmaxf(M, pp[t].x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float Z = 0.f;
    for (int t = lane; t < n_part; t += 32) Z += pp[t].y * expf(pp[t].x - M);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Z += __shfl_xor_sync(0xffffffffu, Z, o);
    if (lane == 0) {
      sM = M;
      sZ = Z;
    }
  }
  __syncthreads();
  const float M = sM, invZ = 1.0f / sZ;
  float* s = scores + static_cast<long long>(g) * n;
  // 16-byte vectors (when n is a multiple of 4), four in flight per thread
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if ((n & 3) == 0 && (reinterpret_cast<uintptr_t>(s) & 15) == 0) {
    float4* s4 = reinterpret_cast<float4*>(s);
    const long long n4 = n >> 2;
    for (; i + 3 * stride < n4; i += 4 * stride) {
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = s4[i + u * stride];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        v[u].x = expf(v[u].x - M) * invZ;
        v[u].y = expf(v[u].y - M) * invZ;
        v[u].z = expf(v[u].z - M) * invZ;
        v[u].w = expf(v[u].w - M) * invZ;
        s4[i + u * stride] = v[u];
      }
    }
    for (; i < n4; i += stride) {
      float4 v = s4[i];
      v.x = expf(v.x - M) * invZ;
      v.y = expf(v.y - M) * invZ;
      v.z = expf(v.z - M) * invZ;
      v.w = expf(v.w - M) * invZ;
      s4[i] = v;
    }
  } else {
    for (; i < n; i += stride) s[i] = expf(s[i] - M) * invZ;
  }
}

// Per-token mode: a head has thousands of logits tiles; one CTA per head folds
// their (max, sum of exp) partials into one (M, Z) first (fixed order per
// thread, then a fixed tree), so that the normalising CTAs read one pair.
__global__ void __launch_bounds__(256) combine_partials_kernel(const float2* __restrict__ part, int n_part,
                                                               float2* __restrict__ out) {
  __shared__ float red[256];
  const int g = blockIdx.x;
  const float2* pp = part + static_cast<long long>(g) * n_part;
  float M = -INFINITY;
  for (int t = threadIdx.x; t < n_part; t += 256) M = fmaxf(M, pp[t].x);
  red[threadIdx.x] = M;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) red[threadIdx.x] = fmaxf(red[threadIdx.x], red[threadIdx.x + o]);
    __syncthreads();
  }
  M = red[0];
  __syncthreads();
  float Z = 0.f;
  for (int t = threadIdx.x; t < n_part; t += 256) Z += pp[t].y * expf(pp[t].x - M);
  red[threadIdx.x] = Z;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) out[g] = make_float2(M, red[0]);
}

// One CTA per resident slot (persistent), from the occupancy of this instantiation.
template <typename T, int D, int MAXR>
void launch_mean(const void* q, const void* k, const lbsa_qkv_desc& d, int block, int nB, long long items,
                 float* qbar, float* kbar, cudaStream_t s, void* qs, void* ks) {
  static int per_sm = 0;
  if (!per_sm) {
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, block_mean_kernel<T, D, MAXR>, 256, 0);
    if (per_sm <= 0) per_sm = 1;
  }
  const unsigned grid = static_cast<unsigned>(std::min<long long>(items, static_cast<long long>(per_sm) * num_sms()));
  block_mean_kernel<T, D, MAXR><<<grid, 256, 0, s>>>(static_cast<const T*>(q), static_cast<const T*>(k), d, block,
                                                     nB, items, qbar, kbar, static_cast<__nv_bfloat16*>(qs),
                                                     static_cast<__nv_bfloat16*>(ks));
}

template <int D>
cudaError_t run(const void* q, const void* k, const lbsa_qkv_desc& d, int block, int nB, bool tokens, float* scores,
                void* ws, cudaStream_t s, const CUtensorMap* tq, const CUtensorMap* tkb, int32_t* status,
                long long wait_limit, const CUtensorMap* ts, const CUtensorMap* tqs) {
  const long long G = static_cast<long long>(d.B) * d.H;
  float* qbar = static_cast<float*>(ws);
  float* kbar = qbar + G * nB * D;
  float2* part = reinterpret_cast<float2*>(kbar + G * nB * D);
  const int nQ = tokens ? d.N_valid : nB;
  const int nTk = (nB + kTk - 1) / kTk, nTq = (nQ + kTq - 1) / kTq;
  const long long items = G * nB;
  // the tensor-core logits take the means as bf16 hi / lo terms, written with the means
  void *qs = nullptr, *ks = nullptr;
  const bool tc_tok = tokens && tq && tkb, tc_blk = !tokens && tqs && tkb && ts;
  if (tc_tok) ks = qbar;                     // the query-block means' slot, unused in this mode
  if (tc_blk) meanpool_block_split_ptrs(ws, d.B, d.H, nB, D, &qs, &ks);
  if (d.dtype == LBSA_BF16) {
    if (block <= 64)
      launch_mean<__nv_bfloat16, D, 64>(q, k, d, block, nB, items, tc_tok ? nullptr : qbar, kbar, s, qs, ks);
    else
      launch_mean<__nv_bfloat16, D, 128>(q, k, d, block, nB, items, tc_tok ? nullptr : qbar, kbar, s, qs, ks);
  } else {
    if (block <= 64)
      launch_mean<float, D, 64>(q, k, d, block, nB, items, qbar, kbar, s, qs, ks);
    else
      launch_mean<float, D, 128>(q, k, d, block, nB, items, qbar, kbar, s, qs, ks);
  }
  const float scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  const dim3 lgrid(nTk, nTq, static_cast<unsigned>(G));
  const long long n = static_cast<long long>(nQ) * nB;
  const int chunks = static_cast<int>(std::min<long long>(tokens ? 256 : 64, (n + 2047) / 2048));
  if (tc_tok) {
    // bf16 token rows: the logits on the tensor cores, from the key means' hi / lo
    // terms (in the query-block means' slot, which this mode does not use)
    cudaError_t e;
    const int np = token_logits_parts(nQ, nB);
    TokenLogitsArgs a{static_cast<int>(G), d.H, nQ, nB, D, scale, scores, part, status, wait_limit};
    e = launch_token_logits_bf16(tq, tkb, ts, a, s);
    if (e != cudaSuccess) return e;
    float2* head = part + G * np;
    combine_partials_kernel<<<static_cast<unsigned>(G), 256, 0, s>>>(part, np, head);
    normalize_kernel<<<dim3(chunks, static_cast<unsigned>(G)), 256, 0, s>>>(scores, head, n, 1);
    return cudaGetLastError();
  }
  if (tc_blk) {
    // both sides are fp32 means: hi / lo terms of each, three chains on the tensor cores
    cudaError_t e;
    const int np = token_logits_parts(nQ, nB);
    TokenLogitsArgs a{static_cast<int>(G), d.H, nQ, nB, D, scale, scores, part, status, wait_limit};
    e = launch_token_logits_bf16(tqs, tkb, ts, a, s, true);
    if (e != cudaSuccess) return e;
    normalize_kernel<<<dim3(chunks, static_cast<unsigned>(G)), 256, 0, s>>>(scores, part, n, np);
    return cudaGetLastError();
  }
  if (!tokens) {
    logits_kernel<D, float, false><<<lgrid, 128, 0, s>>>(qbar, 0, 0, 0, d.H, kbar, nQ, nB, scale, scores, part);
  } else if (d.dtype == LBSA_BF16) {
    logits_kernel<D, __nv_bfloat16, true><<<lgrid, 128, 0, s>>>(static_cast<const __nv_bfloat16*>(q), d.stride_b,
                                                                 d.stride_h, d.stride_n, d.H, kbar, nQ, nB, scale,
                                                                 scores, part);
  } else {
    logits_kernel<D, float, true><<<lgrid, 128, 0, s>>>(static_cast<const float*>(q), d.stride_b, d.stride_h,
                                                         d.stride_n, d.H, kbar, nQ, nB, scale, scores, part);
  }
  if (tokens) {
    float2* head = part + G * nTq * nTk;
    combine_partials_kernel<<<static_cast<unsigned>(G), 256, 0, s>>>(part, nTq * nTk, head);
    normalize_kernel<<<dim3(chunks, static_cast<unsigned>(G)), 256, 0, s>>>(scores, head, n, 1);
  } else {
    normalize_kernel<<<dim3(chunks, static_cast<unsigned>(G)), 256, 0, s>>>(scores, part, n, nTq * nTk);
  }
  return cudaGetLastError();
}

}  // namespace

size_t meanpool_workspace_bytes(int B, int H, int nB, int d, int nQ) {
  const size_t G = static_cast<size_t>(B) * H;
  const size_t nTk = (nB + kTk - 1) / kTk, nTq = (nQ + kTq - 1) / kTq;
  const size_t parts = std::max<size_t>(nTq * nTk, static_cast<size_t>(token_logits_parts(nQ, nB)));
  const size_t base = (2 * G * nB * d * sizeof(float) + (G * parts + G) * sizeof(float2) + 255) / 256 * 256;
  return base + (nQ == nB ? 2 * G * nB * d * sizeof(float) : 0) + 256;   // + the block proxy's hi / lo terms
}

void meanpool_block_split_ptrs(void* ws, int B, int H, int nB, int d, void** qs, void** ks) {
  const size_t G = static_cast<size_t>(B) * H;
  const size_t nTk = (nB + kTk - 1) / kTk, nTq = (nB + kTq - 1) / kTq;
  const size_t parts = std::max<size_t>(nTq * nTk, static_cast<size_t>(token_logits_parts(nB, nB)));
  const size_t base = (2 * G * nB * d * sizeof(float) + (G * parts + G) * sizeof(float2) + 255) / 256 * 256;
  *qs = static_cast<char*>(ws) + base;
  *ks = static_cast<char*>(ws) + base + G * nB * d * 2 * sizeof(uint16_t);
}

void* meanpool_split_ptr(void* ws) { return ws; }   // the query-block means' slot: G x nB x d fp32

cudaError_t launch_meanpool(const void* q, const void* k, const lbsa_qkv_desc& d, int block, int nB, bool tokens,
                            float* scores, void* ws, cudaStream_t s, const CUtensorMap* tq, const CUtensorMap* tkb,
                            int32_t* status, long long wait_limit, const CUtensorMap* ts, const CUtensorMap* tqs) {
  return d.d == 128 ? run<128>(q, k, d, block, nB, tokens, scores, ws, s, tq, tkb, status, wait_limit, ts, tqs)
                    : run<64>(q, k, d, block, nB, tokens, scores, ws, s, tq, tkb, status, wait_limit, ts, tqs);
}

}  // namespace lbsa
