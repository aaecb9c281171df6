// True-fp32 exact block mass and block-sparse attention on CUDA cores.
//
// Same definitions as the tensor-core path (LoSA abstract: exact block mass at
// a dense step; VMoBA review: attention over the kept blocks only), computed
// with fp32 FMAs and expf/logf so that fp32 inputs meet a 1e-5 bound.  One
// warp owns one query row at a time (a CTA of up to 32 warps takes a query
// block); lane l holds q[l + 32e], e < d/32; each key's dot product is a
// butterfly shuffle reduction (fixed order, so results are deterministic).
#include "lbsa_device.cuh"

namespace lbsa {
namespace {

constexpr int kMaxWarps = 32;

// Warps a CTA runs: one per row of the block, at most 32, and (scorer) within
// the shared memory that holds one partial row of nB sums per warp.
int f32_warps(int block, int nB, bool scorer) {
  int w = block < kMaxWarps ? block : kMaxWarps;
  if (scorer)
    while (w > 1 && static_cast<size_t>(w) * nB * sizeof(float) > 200 * 1024) w >>= 1;
  return w;
}

template <int D>
__device__ __forceinline__ float warp_dot(const float (&q)[D / 32], const float* krow, int lane) {
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < D / 32; ++e) s = fmaf(q[e], krow[lane + 32 * e], s);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}

// grid (nB, H, B), 32 x warps threads.  part: dynamic smem [warps][nB].
template <int D>
__global__ void score_exact_f32_kernel(const float* __restrict__ q, const float* __restrict__ k, lbsa_qkv_desc desc,
                                       ScoreArgs a) {
  extern __shared__ float part[];
  const int i = blockIdx.x, h = blockIdx.y, bb = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = a.N_valid, nB = a.nB, blk = a.block;
  const float scale = 1.0f / sqrtf(static_cast<float>(D));
  const int nw = blockDim.x >> 5;
  for (int t = threadIdx.x; t < nw * nB; t += blockDim.x) part[t] = 0.f;
  __syncthreads();
  const float* qh = q + bb * desc.stride_b + h * desc.stride_h;
  const float* kh = k + bb * desc.stride_b + h * desc.stride_h;
  const int r0 = i * blk, r1 = min(r0 + blk, N);
  for (int r = r0 + warp; r < r1; r += nw) {
    float qr[D / 32];
#pragma unroll
    for (int e = 0; e < D / 32; ++e) qr[e] = qh[r * desc.stride_n + lane + 32 * e];
    float m = -INFINITY, l = 0.f;
    for (int c = 0; c < N; ++c) {
      const float s = warp_dot<D>(qr, kh + c * desc.stride_n, lane) * scale;
      const float mn = fmaxf(m, s);
      l = l * expf(m - mn) + expf(s - mn);
      m = mn;
    }
    const float lse = m + logf(l);
    if (a.lse && lane == 0) a.lse[(static_cast<long long>(bb) * a.H + h) * N + r] = lse;
    for (int j = 0; j < nB; ++j) {
      float acc = 0.f;
      const int c1 = min((j + 1) * blk, N);
      for (int c = j * blk; c < c1; ++c) acc += expf(warp_dot<D>(qr, kh + c * desc.stride_n, lane) * scale - lse);
      if (lane == 0) part[warp * nB + j] += acc;
    }
  }
  __syncthreads();
  const float rv = static_cast<float>(r1 - r0);
  const long long orow = ((static_cast<long long>(bb) * a.H + h) * nB + i) * nB;
  for (int j = threadIdx.x; j < nB; j += blockDim.x) {
    float v = 0.f;
    for (int w = 0; w < nw; ++w) v += part[w * nB + j];
    a.scores[orow + j] = v / rv;
  }
}

// grid (nB, H, B), 32 x warps threads.
template <int D>
__global__ void attend_f32_kernel(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
                                  lbsa_qkv_desc desc, AttendArgs a) {
  const int i = blockIdx.x, h = blockIdx.y, bb = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = a.N_valid, nB = a.nB, blk = a.block;
  const float scale = 1.0f / sqrtf(static_cast<float>(D));
  const long long row = (static_cast<long long>(bb) * a.H + h) * nB + i;
  const int cnt = a.counts[row];
  const int32_t* list = a.cols + row * nB;
  const float* qh = q + bb * desc.stride_b + h * desc.stride_h;
  const float* kh = k + bb * desc.stride_b + h * desc.stride_h;
  const float* vh = v + bb * desc.stride_b + h * desc.stride_h;
  float* oh = reinterpret_cast<float*>(a.out) + bb * a.ostride_b + h * a.ostride_h;
  const int r0 = i * blk, r1 = min(r0 + blk, N);
  for (int r = r0 + warp; r < r1; r += static_cast<int>(blockDim.x >> 5)) {
    float qr[D / 32], o[D / 32];
#pragma unroll
    for (int e = 0; e < D / 32; ++e) {
      qr[e] = qh[r * desc.stride_n + lane + 32 * e];
      o[e] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    for (int t = 0; t < cnt; ++t) {
      const int j = list[t];
      if (j < 0 || j >= nB) {
        if (lane == 0) raise_status(a.status, LBSA_ERR_BAD_INDEX);
        continue;
      }
      // per-token lists (64-token blocks): skip entries this token does not keep
      if (a.masks && !((a.masks[row * nB + t] >> (r - r0)) & 1ull)) continue;
      const int c1 = min((j + 1) * blk, N);
      for (int c = j * blk; c < c1; ++c) {
        const float s = warp_dot<D>(qr, kh + c * desc.stride_n, lane) * scale;
        const float mn = fmaxf(m, s);
        const float f = expf(m - mn);
        const float p = expf(s - mn);
        l = l * f + p;
#pragma unroll
        for (int e = 0; e < D / 32; ++e) o[e] = fmaf(p, vh[c * desc.stride_n + lane + 32 * e], o[e] * f);
        m = mn;
      }
    }
    const float inv = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll
    for (int e = 0; e < D / 32; ++e) oh[r * a.ostride_n + lane + 32 * e] = o[e] * inv;
    if (a.lse && lane == 0)
      a.lse[(static_cast<long long>(bb) * a.H + h) * N + r] = (l > 0.f) ? m + logf(l) : -INFINITY;
  }
}

}  // namespace

cudaError_t launch_attend_f32(const float* q, const float* k, const float* v, const lbsa_qkv_desc& d,
                              const AttendArgs& a, cudaStream_t s) {
  dim3 grid(a.nB, a.H, a.B);
  const int threads = 32 * f32_warps(a.block, a.nB, false);
  if (a.d == 128) attend_f32_kernel<128><<<grid, threads, 0, s>>>(q, k, v, d, a);
  else attend_f32_kernel<64><<<grid, threads, 0, s>>>(q, k, v, d, a);
  return cudaGetLastError();
}

cudaError_t launch_score_exact_f32(const float* q, const float* k, const lbsa_qkv_desc& d, const ScoreArgs& a,
                                   cudaStream_t s) {
  dim3 grid(a.nB, a.H, a.B);
  const int warps = f32_warps(a.block, a.nB, true);
  const size_t smem = static_cast<size_t>(warps) * a.nB * sizeof(float);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(a.d == 128 ? score_exact_f32_kernel<128> : score_exact_f32_kernel<64>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  if (a.d == 128) score_exact_f32_kernel<128><<<grid, 32 * warps, smem, s>>>(q, k, d, a);
  else score_exact_f32_kernel<64><<<grid, 32 * warps, smem, s>>>(q, k, d, a);
  return cudaGetLastError();
}

}  // namespace lbsa
