// Token orders for VMoBA's 1D / 2D / 3D block partitions (pith.science review
// of arXiv 2506.23858: layer-wise cyclic 1D-2D-3D partition) and the row
// gather / scatter that puts Q, K, V into block order and O back.
//
// slot_of(t, h, w) gives the blocked position of the raster token (t, h, w) in
// closed form: tiles are visited in raster tile order and tokens in raster
// order inside a tile, with edge tiles truncated, so every tile before the
// token's tile in its tile-row / tile-slab is full-sized along the axes that
// are already passed.
#include "lbsa_device.cuh"

namespace lbsa {
namespace {

__host__ __device__ inline long long slot_of(int t, int h, int w, int T, int Hg, int Wg, int kind, int tt, int th,
                                             int tw) {
  switch (kind) {
    case LBSA_PART_1D:
      return (static_cast<long long>(h) * Wg + w) * T + t;
    case LBSA_PART_2D: {
      const int a = h / th, c = w / tw;
      const int sh = min(th, Hg - a * th), sw = min(tw, Wg - c * tw);
      const long long frame = static_cast<long long>(t) * Hg * Wg;
      return frame + static_cast<long long>(a) * th * Wg + static_cast<long long>(sh) * c * tw +
             static_cast<long long>(h - a * th) * sw + (w - c * tw);
    }
    case LBSA_PART_3D: {
      const int at = t / tt, a = h / th, c = w / tw;
      const int st = min(tt, T - at * tt), sh = min(th, Hg - a * th), sw = min(tw, Wg - c * tw);
      return static_cast<long long>(at) * tt * Hg * Wg + static_cast<long long>(st) * a * th * Wg +
             static_cast<long long>(st) * sh * c * tw +
             (static_cast<long long>(t - at * tt) * sh + (h - a * th)) * sw + (w - c * tw);
    }
    default:
      return (static_cast<long long>(t) * Hg + h) * Wg + w;
  }
}

__global__ void partition_perm_kernel(int T, int Hg, int Wg, int kind, int tt, int th, int tw, int32_t* perm) {
  const long long n = static_cast<long long>(T) * Hg * Wg;
  for (long long tok = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; tok < n;
       tok += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int w = static_cast<int>(tok % Wg);
    const int h = static_cast<int>((tok / Wg) % Hg);
    const int t = static_cast<int>(tok / (static_cast<long long>(Wg) * Hg));
    perm[slot_of(t, h, w, T, Hg, Wg, kind, tt, th, tw)] = static_cast<int32_t>(tok);
  }
}

// One thread per 16-byte vector of a row; vec_per_row = d * esize / 16 and the
// strides are in 16-byte vectors.  Up to three tensors share perm.
struct PtrPack {
  const uint4* x[3];
  uint4* y[3];
};

// grid (ceil(N / kPermRows), count * B * H), 256 threads: thread (row r of the
// CTA's iteration, 16-byte vector v) copies row slots r0 + r, r0 + r + rpi, ...
// (32-bit row indices; every thread keeps several independent loads in flight).
constexpr int kPermRows = 64;
// A perm entry outside [0, N) skips its row and records LBSA_ERR_BAD_INDEX.
__global__ void __launch_bounds__(256) permute_kernel_packed(PtrPack pk, const int32_t* __restrict__ perm, int B,
                                                             int H, int N, int vec_per_row, long long sb,
                                                             long long sh, long long sn, int inverse,
                                                             int32_t* status) {
  const int tbh = blockIdx.y;                       // tensor * (B*H) + b*H + h
  const int t = tbh / (B * H);
  const int bh = tbh - t * (B * H);
  const int b = bh / H, h = bh - b * H;
  const long long base = b * sb + h * sh;
  const uint4* __restrict__ x = pk.x[t];
  uint4* __restrict__ y = pk.y[t];
  const int rpi = blockDim.x / vec_per_row;         // rows per iteration
  const int lr = threadIdx.x / vec_per_row;
  const int v = threadIdx.x - lr * vec_per_row;
  const int r0 = blockIdx.x * kPermRows;
  const int r1 = min(r0 + kPermRows, N);
#pragma unroll 4
  for (int slot = r0 + lr; slot < r1; slot += rpi) {
    const int src = __ldg(perm + slot);
    if (src < 0 || src >= N) {
      if (v == 0) raise_status(status, LBSA_ERR_BAD_INDEX);
      continue;
    }
    if (!inverse) y[base + slot * sn + v] = __ldg(x + base + src * sn + v);
    else y[base + src * sn + v] = __ldg(x + base + slot * sn + v);
  }
}

}  // namespace

void partition_perm_host(int T, int Hg, int Wg, int kind, int tt, int th, int tw, int32_t* perm) {
  for (int t = 0; t < T; ++t)
    for (int h = 0; h < Hg; ++h)
      for (int w = 0; w < Wg; ++w)
        perm[slot_of(t, h, w, T, Hg, Wg, kind, tt, th, tw)] = (t * Hg + h) * Wg + w;
}

cudaError_t launch_partition_perm(int T, int Hg, int Wg, int kind, int tt, int th, int tw, int32_t* perm,
                                  cudaStream_t s) {
  const long long n = static_cast<long long>(T) * Hg * Wg;
  const int blocks = static_cast<int>(std::min<long long>((n + 255) / 256, 148 * 8));
  partition_perm_kernel<<<blocks, 256, 0, s>>>(T, Hg, Wg, kind, tt, th, tw, perm);
  return cudaGetLastError();
}

cudaError_t launch_permute(const void* const* xs, void* const* ys, int count, const int32_t* perm,
                           const lbsa_qkv_desc& d, int inverse, int32_t* status, cudaStream_t s) {
  const int esize = d.dtype == LBSA_BF16 ? 2 : 4;
  const int vec_per_row = d.d * esize / 16;
  const long long k = 16 / esize;   // elements per vector
  PtrPack pk{};
  for (int t = 0; t < count; ++t) {
    pk.x[t] = static_cast<const uint4*>(xs[t]);
    pk.y[t] = static_cast<uint4*>(ys[t]);
  }
  // vec_per_row is d * esize / 16 in {8, 16, 32}: it divides the 256 threads
  if (vec_per_row <= 0 || 256 % vec_per_row != 0) return cudaErrorInvalidValue;
  const long long ybh = static_cast<long long>(count) * d.B * d.H;
  if (ybh > 65535) return cudaErrorInvalidValue;
  dim3 grid((d.N_valid + kPermRows - 1) / kPermRows, static_cast<unsigned>(ybh));
  permute_kernel_packed<<<grid, 256, 0, s>>>(pk, perm, d.B, d.H, d.N_valid, vec_per_row, d.stride_b / k, d.stride_h / k,
                                             d.stride_n / k, inverse, status);
  return cudaGetLastError();
}

}  // namespace lbsa
