// Per-token proxy logits on sm_100a tensor cores (VMoBA review on pith.science,
// referee report major comment 1: every query token scores every key-block
// mean).  For one head g:
//   s_rj = q_r . kbar_j / sqrt(d)      (q_r bf16 token rows, kbar_j fp32 block means)
// The block means enter the tensor cores as two bf16 terms, hi = bf16(kbar)
// and lo = bf16(kbar - hi), so kbar - hi - lo is below 2^-17 |kbar| and
//   q . kbar = q . hi + q . lo   (both products exact in the fp32 accumulator)
// is within about 2^-17 |q| |kbar| of the fp32 dot product: far below the
// scores' tolerance once normalised.  Each (128-token tile, 128-key-block
// chunk) is 2 x d/16 UMMAs of 128 x 128 x 16 into one TMEM accumulator.
//
// The block-mean proxy (query-block means against key-block means) runs the
// same kernel with the query side split the same way (A_SPLIT): then
//   qbar . kbar = qh . kh + qh . kl + ql . kh   (ql . kl is below 2^-17 of it)
// three chains into the accumulator, the query rows loaded as two terms.
//
// Outputs, as the CUDA-core logits kernel writes them: the scaled logits
// s_rj into the scores buffer ([g][r][j], fp32) and, per warp of 32 tokens and
// chunk, the (max, sum of exp(s - max)) of its valid logits, so that the
// normalisation can form the head's softmax.
//
// Persistent grid, one CTA per SM (192 threads):
//   warps 0-3  epilogue: thread t = token row t of the tile = TMEM lane t; reads
//              a chunk's 128 logits from TMEM, frees the accumulator, stores and
//              reduces them
//   warp 4     TMA producer: the Q tile once per item, then per chunk the hi
//              and lo tiles of 128 block means into a 2-stage ring
//   warp 5     UMMA issuer and TMEM owner: two 128-column accumulators, so the
//              UMMAs of chunk c+1 run while the epilogue drains chunk c
#include <algorithm>

#include "lbsa_device.cuh"

namespace lbsa {
namespace {

constexpr int kRows = 128;       // tokens per tile
constexpr int kCols = 128;       // key blocks per chunk
constexpr int kTLThreads = 192;

template <int D, bool A_SPLIT>
struct TLLayout {
  static constexpr int Q_BYTES = kRows * D * 2;            // one term of the query tile
  static constexpr int NQT = A_SPLIT ? 2 : 1;              // query terms
  static constexpr int TILE_BYTES = kCols * D * 2;        // one term (hi or lo) of one chunk
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RING = NQT * Q_BYTES;           // [stage][term] tiles
  static constexpr int OFF_OUT = OFF_RING + 4 * TILE_BYTES;  // two 128 x 32 fp32 store boxes (16 KB each)
  static constexpr int OUT_BYTES = kRows * 32 * 4;
  static constexpr int OFF_BAR = OFF_OUT + 2 * OUT_BYTES;
  // q_full, q_empty, kv_full[2], kv_empty[2], acc_full[2], acc_empty[2], drain
  static constexpr int NBAR = 11;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;      // [0] tmem base [1] abort
  static constexpr int BYTES = OFF_MISC + 16 + 1024;       // + alignment slack
};

template <int D, bool TMA_OUT, bool A_SPLIT>
__global__ void __launch_bounds__(kTLThreads, 1)
token_logits_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_kb,
                       const __grid_constant__ CUtensorMap tmap_s, const TokenLogitsArgs args) {
  using L = TLLayout<D, A_SPLIT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* q_full = bar;
  uint64_t* q_empty = bar + 1;
  uint64_t* kv_full = bar + 2;
  uint64_t* kv_empty = bar + 4;
  uint64_t* acc_full = bar + 6;
  uint64_t* acc_empty = bar + 8;
  uint64_t* drain = bar + 10;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  if (*reinterpret_cast<volatile int32_t*>(args.status) == LBSA_ERR_TIMEOUT) return;

  const int nTq = (args.nQ + kRows - 1) / kRows;
  const int nC = (args.nB + kCols - 1) / kCols;
  // work items: (head, 128-row tile, group of args.cpi chunks); a small launch
  // splits a tile's chunks over several CTAs (each loads the tile's query rows)
  const int nCG = (nC + args.cpi - 1) / args.cpi;
  const long long items = static_cast<long long>(args.G) * nTq * nCG;
  const long long wl = args.wait_limit;

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(kv_full + i, 1);
      mbar_init(kv_empty + i, 1);
      mbar_init(acc_full + i, 1);
      mbar_init(acc_empty + i, 4);           // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    misc[1] = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(misc, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tmap_q);
      prefetch_tmap(&tmap_kb);
      long long step = 0;
      int it = 0, q_loads = 0;
      bool ok = true;
      for (long long item = blockIdx.x; ok && item < items; item += gridDim.x, ++it) {
        const long long tile = item / nCG;
        const int g = static_cast<int>(tile / nTq), tq = static_cast<int>(tile % nTq);
        const int c_lo = static_cast<int>(item % nCG) * args.cpi, c_hi = min(nC, c_lo + args.cpi);
        const int b = g / args.H, h = g % args.H;
        if (it > 0 && !(ok = mbar_wait(q_empty, (it - 1) & 1, wl, args.status, abort_flag))) break;
        ++q_loads;
        mbar_arrive_expect_tx(q_full, L::NQT * L::Q_BYTES);
        for (int u = 0; u < L::NQT; ++u)
          for (int dc = 0; dc < D / 64; ++dc) {
            uint8_t* dst = smem + L::OFF_Q + u * L::Q_BYTES + dc * kRows * 128;
            if (A_SPLIT) tma_load_4d(dst, &tmap_q, q_full, dc * 64, tq * kRows, g, u);   // (d, nQ, G, term)
            else tma_load_4d(dst, &tmap_q, q_full, dc * 64, tq * kRows, h, b);          // (d, N, H, B)
          }
        for (int c = c_lo; c < c_hi; ++c, ++step) {
          const int st = static_cast<int>(step & 1);
          if (step >= 2 && !(ok = mbar_wait(kv_empty + st, ((step >> 1) - 1) & 1, wl, args.status, abort_flag)))
            break;
          mbar_arrive_expect_tx(kv_full + st, 2 * L::TILE_BYTES);
          for (int u = 0; u < 2; ++u)
            for (int dc = 0; dc < D / 64; ++dc)
              tma_load_4d(smem + L::OFF_RING + (st * 2 + u) * L::TILE_BYTES + dc * kCols * 128, &tmap_kb,
                          kv_full + st, dc * 64, c * kCols, g, u);
        }
      }
      // every copy issued has landed before the CTA can exit
      if (q_loads > 0) mbar_wait(q_full, (q_loads - 1) & 1, wl, args.status, nullptr);
      for (long long s = (step > 2 ? step - 2 : 0); s < step; ++s)
        mbar_wait(kv_full + (s & 1), (s >> 1) & 1, wl, args.status, nullptr);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ UMMA issuer
    const uint32_t idesc = idesc_bf16_f32(kRows, kCols, 0);
    const uint64_t dQ = smem_desc_sw128(smem_u32(smem + L::OFF_Q), 16, 1024);
    const uint64_t dR = smem_desc_sw128(smem_u32(smem + L::OFF_RING), 16, 1024);
    auto wait0 = [&](uint64_t* b, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(b, parity, wl, args.status, abort_flag));
    };
    long long step = 0;
    int it = 0;
    bool ok = true;
    for (long long item = blockIdx.x; ok && item < items; item += gridDim.x, ++it) {
      const int c_lo = static_cast<int>(item % nCG) * args.cpi, c_hi = min(nC, c_lo + args.cpi);
      if (!(ok = wait0(q_full, it & 1))) break;
      for (int c = c_lo; c < c_hi; ++c, ++step) {
        const int st = static_cast<int>(step & 1);
        if (!(ok = wait0(kv_full + st, (step >> 1) & 1))) break;
        if (step >= 2 && !(ok = wait0(acc_empty + st, ((step >> 1) - 1) & 1))) break;
        tc_fence_after();
        if (elect_one()) {
          // chains (query term, mean term): (0, 0), (0, 1) and, split, (1, 0)
#pragma unroll
          for (int ch = 0; ch < (A_SPLIT ? 3 : 2); ++ch) {
            const int ua = ch == 2 ? 1 : 0, ub = ch == 1 ? 1 : 0;
            const uint64_t a0 = dQ + static_cast<uint64_t>((ua * L::Q_BYTES) >> 4);
            const uint64_t b0 = dR + static_cast<uint64_t>(((st * 2 + ub) * L::TILE_BYTES) >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = ((kk >> 2) * (kRows * 128) + (kk & 3) * 32) >> 4;
              umma_ss(tmem + st * kCols, a0 + off, b0 + off, idesc, (ch > 0 || kk > 0) ? 1u : 0u);
            }
          }
          umma_commit(kv_empty + st);
          umma_commit(acc_full + st);
          if (c == c_hi - 1) umma_commit(q_empty);
        }
        __syncwarp();
      }
    }
    if (elect_one()) umma_commit(drain);
    __syncwarp();
    mbar_wait(drain, 0, wl, args.status, nullptr);
  } else {
    // ------------------------------------------------------------ epilogue (warps 0-3)
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    long long step = 0;
    long long boxes = 0;                     // TMA store boxes issued (alternating staging buffers)
    bool ok = true;
    for (long long item = blockIdx.x; ok && item < items; item += gridDim.x) {
      const long long tile = item / nCG;
      const int g = static_cast<int>(tile / nTq), tq = static_cast<int>(tile % nTq);
      const int c_lo = static_cast<int>(item % nCG) * args.cpi, c_hi = min(nC, c_lo + args.cpi);
      const int row = tq * kRows + warp * 32 + lane;
      const bool rvalid = row < args.nQ;
      float* srow = args.scores + (static_cast<long long>(g) * args.nQ + (rvalid ? row : 0)) * args.nB;
      for (int c = c_lo; c < c_hi; ++c, ++step) {
        const int st = static_cast<int>(step & 1);
        // the four warps decide together (they share named barriers below)
        if (!(ok = named_bar_and(2, 128, mbar_wait(acc_full + st, (step >> 1) & 1, wl, args.status, abort_flag))))
          break;
        tc_fence_after();
        uint32_t v[128];
#pragma unroll
        for (int k = 0; k < 4; ++k) tmem_ld32(t_lane + st * kCols + k * 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * k]));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty + st);   // the accumulator may take chunk c + 2
        const int col0 = c * kCols;
        const int ncol = min(kCols, args.nB - col0);
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < 128; ++j) {
          const float x = __uint_as_float(v[j]) * args.scale;
          v[j] = __float_as_uint(x);
          if (rvalid && j < ncol) mx = fmaxf(mx, x);
        }
        if (TMA_OUT) {
          // four 128 x 32 boxes through two swizzled staging buffers: row t's
          // 16-byte unit u sits at unit u ^ (t & 7) of its 128-byte line; one
          // thread issues each TMA store (clipped at nQ rows and nB columns)
          const int t = warp * 32 + lane;
#pragma unroll
          for (int k = 0; k < 4; ++k, ++boxes) {
            uint8_t* box = smem + L::OFF_OUT + (boxes & 1) * L::OUT_BYTES;
            if (boxes >= 2) {
              if (t == 0) tma_store_wait_read<1>();       // the store that last read this box is done with it
              named_bar_sync(1, 128);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u)
              *reinterpret_cast<uint4*>(box + t * 128 + ((u ^ (t & 7)) << 4)) =
                  make_uint4(v[32 * k + 4 * u], v[32 * k + 4 * u + 1], v[32 * k + 4 * u + 2], v[32 * k + 4 * u + 3]);
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            if (t == 0) {
              tma_store_3d(&tmap_s, box, col0 + 32 * k, tq * kRows, g);
              tma_store_commit();
            }
          }
        } else if (rvalid) {
          float* dst = srow + col0;
#pragma unroll
          for (int j = 0; j < 128; ++j)
            if (j < ncol) dst[j] = __uint_as_float(v[j]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float sm = 0.f;
        if (rvalid && mx != -INFINITY) {
          const float mxl = mx * 1.4426950408889634f;
#pragma unroll
          for (int j = 0; j < 128; ++j)
            if (j < ncol) sm += ex2(fmaf(__uint_as_float(v[j]), 1.4426950408889634f, -mxl));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
        if (lane == 0)
          args.part[((static_cast<long long>(g) * nTq + tq) * nC + c) * 4 + warp] = make_float2(mx, sm);
      }
    }
    if (TMA_OUT && warp == 0 && lane == 0) tma_store_wait<0>();   // the logits are in global memory
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

int tl_sms() {
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  return sms;
}

}  // namespace

int token_logits_parts(int nQ, int nB) { return ((nQ + kRows - 1) / kRows) * ((nB + kCols - 1) / kCols) * 4; }

cudaError_t launch_token_logits_bf16(const CUtensorMap* tq, const CUtensorMap* tkb, const CUtensorMap* ts,
                                     const TokenLogitsArgs& a, cudaStream_t s, bool q_split) {
  if (!(a.d == 64 || a.d == 128) || a.nB < 1 || a.nQ < 1 || a.G < 1) return cudaErrorInvalidValue;
  const long long tiles = static_cast<long long>(a.G) * ((a.nQ + kRows - 1) / kRows);
  const int nC = (a.nB + kCols - 1) / kCols;
  // whole tiles per item, unless that leaves SMs idle: then groups of fewer chunks
  TokenLogitsArgs b = a;
  b.cpi = nC;
  while (b.cpi > 1 && tiles * ((nC + b.cpi - 1) / b.cpi) < tl_sms()) b.cpi = (b.cpi + 1) / 2;
  const long long items = tiles * ((nC + b.cpi - 1) / b.cpi);
  const unsigned grid = static_cast<unsigned>(std::min<long long>(items, tl_sms()));
  auto go = [&](auto kern, int smem) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kTLThreads, smem, s>>>(*tq, *tkb, ts ? *ts : *tq, b);
    return cudaGetLastError();
  };
  if (q_split) {
    if (!ts) return cudaErrorInvalidValue;
    return a.d == 128 ? go(token_logits_tc_kernel<128, true, true>, TLLayout<128, true>::BYTES)
                      : go(token_logits_tc_kernel<64, true, true>, TLLayout<64, true>::BYTES);
  }
  if (ts)
    return a.d == 128 ? go(token_logits_tc_kernel<128, true, false>, TLLayout<128, false>::BYTES)
                      : go(token_logits_tc_kernel<64, true, false>, TLLayout<64, false>::BYTES);
  return a.d == 128 ? go(token_logits_tc_kernel<128, false, false>, TLLayout<128, false>::BYTES)
                    : go(token_logits_tc_kernel<64, false, false>, TLLayout<64, false>::BYTES);
}

}  // namespace lbsa
