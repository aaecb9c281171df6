// Exact block attention mass on sm_100a tensor cores (bf16 in, fp32 out).
//
// LoSA (abstract, scholarbro.com author page of C. Sun) takes the block masses
// exactly, from a single dense step.  Reading used for how the rows of a
// query block combine: the mean over the block's valid rows, so
//   mass[b,h,i,j] = (1/|I_i|) sum_{r in I_i} sum_{c in J_j} softmax_c(q_r.k_c/sqrt(d)).
//
// One sweep over the keys per 128-row query tile.  For every row and 64-key
// chunk the softmax warps keep the online max m and sum l, and store the
// chunk's log-sum-exp  L[r,c] = m + log2(sum_{k in chunk} 2^(x_k - m))  (base
// 2, x = q.k * log2(e)/sqrt(d)) to a per-CTA scratch strip.  After the sweep
// each row knows its lse, and  2^(L[r,c] - lse_r)  is the row's exact mass on
// the chunk; warp shuffles sum it over the rows of a warp, and per-warp
// partials are combined in a fixed order (deterministic).  Every Q K^T product
// and every exponential of the dense pass is computed once.
//
// Persistent grid (three CTAs per SM, each walking tiles with a grid stride),
// so the scratch is bounded: gridDim.x * (128 + 4) * n_chunks floats.  Each
// thread reads back only the strip values it wrote itself.
//
// Warp roles (192 threads): warps 0-3 softmax (thread t = tile row t = TMEM
// lane t), warp 4 TMA producer (Q per tile, K 64-key tiles through a 2-stage
// ring), warp 5 UMMA issuer (S = Q K^T, M=128, N=64, K=d, double-buffered in
// TMEM columns [0,64) and [64,128)).  About 67 KB of shared memory, 128 TMEM
// columns and at most 112 registers a thread let three CTAs (three softmax
// warps per SM sub-partition) share an SM, which hides more of the softmax's
// dependent latency than two CTAs with 128-key steps.  The step width is a
// build-time choice (LBSA_SCORE_BK = 64 or 128, LBSA_SCORE_CTAS = 3 or 2).
#include "lbsa_device.cuh"

namespace lbsa {
namespace {

constexpr int BM = 128;
#ifndef LBSA_SCORE_BK
#define LBSA_SCORE_BK 64
#endif
#ifndef LBSA_SCORE_CTAS
#define LBSA_SCORE_CTAS 3
#endif
constexpr int BK = LBSA_SCORE_BK;  // keys per UMMA step
constexpr int CH = 64;            // keys per chunk (one mass entry per 64-key chunk)
#ifndef LBSA_SCORE_NS
#define LBSA_SCORE_NS 2
#endif
constexpr int NS = LBSA_SCORE_NS;  // K ring depth
// Of every 8 exponential pairs of a full chunk, those whose bit is set take
// the FMA-pipe exponential (exp2_poly2) instead of MUFU ex2: a quarter of the
// exponentials moves off the MUFU, which otherwise bounds the softmax warps.
#ifndef LBSA_SCORE_POLY_MASK
#define LBSA_SCORE_POLY_MASK 0x88
#endif
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 2 * BK;     // S double-buffered
constexpr int kCtasPerSm = LBSA_SCORE_CTAS;
template <int D>
struct Layout {
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int K_BYTES = BK * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_BAR = OFF_K + NS * K_BYTES;
  // q_full, q_empty, k_full[NS], k_empty[NS], s_full[2], s_free[2], drain
  static constexpr int NBAR = 2 + 2 * NS + 5;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static size_t bytes() { return OFF_MISC + 16 + 1024; }
};

struct TileIdx {
  int tile, h, bb;
};
__device__ __forceinline__ TileIdx tile_of(int g, int tiles_per_bh, int H) {
  TileIdx t;
  t.tile = g % tiles_per_bh;
  const int bh = g / tiles_per_bh;
  t.h = bh % H;
  t.bb = bh / H;
  return t;
}

template <int D>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
score_exact_bf16_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                        const ScoreArgs args, float scale_log2) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int N = args.N_valid;
  const int n_chunks = (N + CH - 1) / CH;
  const int n_steps = (N + BK - 1) / BK;
  const int tiles_per_bh = (N + BM - 1) / BM;
  const int total_tiles = tiles_per_bh * args.H * args.B;
  const long long wl = args.wait_limit;
  if (*reinterpret_cast<volatile int32_t*>(args.status) == LBSA_ERR_TIMEOUT) return;

  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* q_full = bar;
  uint64_t* q_empty = bar + 1;
  uint64_t* k_full = bar + 2;
  uint64_t* k_empty = bar + 2 + NS;
  uint64_t* s_full = bar + 2 + 2 * NS;
  uint64_t* s_free = s_full + 2;
  uint64_t* drain = s_free + 2;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  // per-warp chunk partials of the current tile: [4][n_chunks] after the strips
  float* part = args.scratch + static_cast<long long>(gridDim.x) * n_chunks * BM +
                static_cast<long long>(blockIdx.x) * 4 * n_chunks;

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(k_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(s_free + i, 128);
    }
    mbar_init(drain, 1);
    misc[1] = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(misc, kTmemCols);
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
      prefetch_tmap(&tmap_k);
      uint8_t* sQ = smem + L::OFF_Q;
      long long s = 0;       // global step counter (ring position)
      int st = 0;            // s % NS
      uint32_t ph = 0;       // (s / NS) & 1
      int it = 0;            // tiles handled by this CTA
      bool ok = true;
      for (int g = blockIdx.x; ok && g < total_tiles; g += gridDim.x, ++it) {
        const TileIdx t = tile_of(g, tiles_per_bh, args.H);
        if (it >= 1 && !mbar_wait(q_empty, (it - 1) & 1, wl, args.status, abort_flag)) break;
        mbar_arrive_expect_tx(q_full, L::Q_BYTES);
        for (int c = 0; c < D / 64; ++c) tma_load_4d(sQ + c * BM * 128, &tmap_q, q_full, c * 64, t.tile * BM, t.h, t.bb);
        for (int j = 0; j < n_steps; ++j, ++s) {
          if (s >= NS && !mbar_wait(k_empty + st, ph ^ 1u, wl, args.status, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* sK = smem + L::OFF_K + st * L::K_BYTES;
          mbar_arrive_expect_tx(k_full + st, L::K_BYTES);
          for (int c = 0; c < D / 64; ++c) tma_load_4d(sK + c * BK * 128, &tmap_k, k_full + st, c * 64, j * BK, t.h, t.bb);
          if (++st == NS) {
            st = 0;
            ph ^= 1u;
          }
        }
      }
      if (*abort_flag) {
        // let copies still in flight land before the CTA can exit
        for (long long r = (s > NS ? s - NS : 0); r < s; ++r)
          mbar_wait(k_full + r % NS, static_cast<uint32_t>((r / NS) & 1), wl, args.status, nullptr);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(BM, BK, 0);
      const uint32_t sQ = smem_u32(smem + L::OFF_Q);
      const uint32_t sK0 = smem_u32(smem + L::OFF_K);
      long long s = 0;
      int st = 0;            // s % NS
      uint32_t ph = 0;       // (s / NS) & 1
      int it = 0;
      bool ok = true;
      for (int g = blockIdx.x; ok && g < total_tiles; g += gridDim.x, ++it) {
        if (!mbar_wait(q_full, it & 1, wl, args.status, abort_flag)) break;
        for (int j = 0; j < n_steps; ++j, ++s) {
          const int sb = static_cast<int>(s & 1);
          if (!mbar_wait(k_full + st, ph, wl, args.status, abort_flag) ||
              (s >= 2 && !mbar_wait(s_free + sb, static_cast<uint32_t>(((s - 2) >> 1) & 1), wl, args.status, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t kbase = sK0 + st * L::K_BYTES;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk & 3) * 32;
            const uint64_t a = smem_desc_sw128(sQ + (kk >> 2) * (BM * 128) + off, 16, 1024);
            const uint64_t b = smem_desc_sw128(kbase + (kk >> 2) * (BK * 128) + off, 16, 1024);
            umma_ss(tmem + sb * BK, a, b, idesc, kk > 0 ? 1u : 0u);
          }
          umma_commit(s_full + sb);
          umma_commit(k_empty + st);
          if (++st == NS) {
            st = 0;
            ph ^= 1u;
          }
        }
        umma_commit(q_empty);          // Q may be replaced once this tile's UMMAs are done
      }
      umma_commit(drain);
      mbar_wait(drain, 0, wl, args.status, nullptr);
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 0-3)
    const int row = tid;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float* strip = args.scratch + static_cast<long long>(blockIdx.x) * n_chunks * BM;   // [n_chunks][128]
    long long s = 0;
    bool alive = true;
    for (int g = blockIdx.x; alive && g < total_tiles; g += gridDim.x) {
      const TileIdx t = tile_of(g, tiles_per_bh, args.H);
      const int grow = t.tile * BM + row;
      const bool valid_row = grow < N;
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < n_steps && alive; ++j, ++s) {
        const int sb = static_cast<int>(s & 1);
        if (!mbar_wait(s_full + sb, static_cast<uint32_t>((s >> 1) & 1), wl, args.status, abort_flag)) {
          alive = false;
          break;
        }
        tc_fence_after();
        const int nh = min(BK / CH, n_chunks - (BK / CH) * j);   // chunks in this step (block-uniform)
        for (int hf = 0; hf < nh; ++hf) {
          const int ch = (BK / CH) * j + hf;
          uint32_t r[64];
          tmem_ld32(t_lane + sb * BK + hf * CH, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
          tmem_ld32(t_lane + sb * BK + hf * CH + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
          tmem_wait_ld();
          if (hf == nh - 1) {
            // the whole S buffer is in registers: the UMMA may overwrite it
            tc_fence_before();
            mbar_arrive(s_free + sb);
          }
          const int nvk = N - ch * CH;
          // row max of the raw logits (the scale is positive), 4 independent chains
          float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
          if (nvk >= 64) {
#pragma unroll
            for (int c = 0; c < 64; c += 2)
              mx4[(c >> 1) & 3] = fmax3(mx4[(c >> 1) & 3], __uint_as_float(r[c]), __uint_as_float(r[c + 1]));
          } else {
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (c < nvk) mx4[c & 3] = fmaxf(mx4[c & 3], __uint_as_float(r[c]));
          }
          const float m_new = fmaxf(m, fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * scale_log2);
          // sum of 2^(s*scale - m_new): packed FMA per pair, MUFU ex2 (or the
          // FMA-pipe exponential for the pairs LBSA_SCORE_POLY_MASK picks), packed adds
          const unsigned long long sc2 = f2_as_u64(scale_log2, scale_log2);
          const unsigned long long nm2 = f2_as_u64(-m_new, -m_new);
          unsigned long long acc4[4] = {0ull, 0ull, 0ull, 0ull};
          if (nvk >= 64) {
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              float v0, v1;
              const unsigned long long v2 = ffma2(f2_as_u64(__uint_as_float(r[2 * c]), __uint_as_float(r[2 * c + 1])), sc2, nm2);
              if ((LBSA_SCORE_POLY_MASK >> (c & 7)) & 1) {
                acc4[c & 3] = fadd2(acc4[c & 3], exp2_poly2(v2));
              } else {
                u64_as_f2(v2, v0, v1);
                acc4[c & 3] = fadd2(acc4[c & 3], f2_as_u64(ex2(v0), ex2(v1)));
              }
            }
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              float v0, v1;
              u64_as_f2(ffma2(f2_as_u64(__uint_as_float(r[2 * c]), __uint_as_float(r[2 * c + 1])), sc2, nm2), v0, v1);
              acc4[c & 3] = fadd2(acc4[c & 3], f2_as_u64(2 * c < nvk ? ex2(v0) : 0.f, 2 * c + 1 < nvk ? ex2(v1) : 0.f));
            }
          }
          float a8[8];
#pragma unroll
          for (int i = 0; i < 4; ++i) u64_as_f2(acc4[i], a8[2 * i], a8[2 * i + 1]);
          const float bsum = ((a8[0] + a8[1]) + (a8[2] + a8[3])) + ((a8[4] + a8[5]) + (a8[6] + a8[7]));
          l = (m == -INFINITY) ? bsum : fmaf(l, ex2(m - m_new), bsum);
          m = m_new;
          strip[static_cast<long long>(ch) * BM + row] = m + __log2f(bsum);
        }
      }
      if (!alive) break;
      const float lse2 = m + __log2f(l);
      // mass of each chunk, summed over this warp's rows.  The strip is read
      // back 16 chunks at a time so that 16 loads are in flight per thread.
      for (int ch0 = 0; ch0 < n_chunks; ch0 += 16) {
        float Lv[16];
#pragma unroll
        for (int u = 0; u < 16; ++u)
          Lv[u] = (ch0 + u < n_chunks) ? strip[static_cast<long long>(ch0 + u) * BM + row] : -INFINITY;
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          if (ch0 + u >= n_chunks) break;
          float v = valid_row ? ex2(Lv[u] - lse2) : 0.f;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          if (lane == 0) part[warp * n_chunks + ch0 + u] = v;
        }
      }
      named_bar_sync(1, 128);
      const int nB = args.nB;
      const long long hrow = (static_cast<long long>(t.bb) * args.H + t.h) * nB;
      if (args.block == 64) {
        for (int o = tid; o < 2 * nB; o += 128) {
          const int half = o / nB, kb = o % nB;
          const int qb = 2 * t.tile + half;
          if (qb >= nB) continue;
          const int rv = min(64, N - qb * 64);
          const float v = (part[(2 * half) * n_chunks + kb] + part[(2 * half + 1) * n_chunks + kb]) /
                          static_cast<float>(rv);
          args.scores[(hrow + qb) * nB + kb] = v;
        }
      } else {
        const int qb = t.tile;
        const int rv = min(128, N - qb * 128);
        for (int kb = tid; kb < nB; kb += 128) {
          float v = 0.f;
          for (int half = 0; half < 2; ++half) {
            const int c = 2 * kb + half;
            if (c < n_chunks)
              v += (part[c] + part[n_chunks + c]) + (part[2 * n_chunks + c] + part[3 * n_chunks + c]);
          }
          args.scores[(hrow + qb) * nB + kb] = v / static_cast<float>(rv);
        }
      }
      if (args.lse && valid_row)
        args.lse[(static_cast<long long>(t.bb) * args.H + t.h) * N + grow] = lse2 * 0.69314718055994531f;
      named_bar_sync(1, 128);           // part[] is reused by the next tile
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

int g_num_sms = 0;

int num_sms() {
  if (!g_num_sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_num_sms <= 0) g_num_sms = 148;
  }
  return g_num_sms;
}

int score_grid(int N, int H, int B) {
  const long long tiles = static_cast<long long>((N + BM - 1) / BM) * H * B;
  return static_cast<int>(std::min<long long>(tiles, static_cast<long long>(kCtasPerSm) * num_sms()));
}

}  // namespace

int score_exact_bf16_key_rows() { return BK; }

size_t score_exact_bf16_workspace_bytes(int B, int H, int N_valid) {
  const int n_chunks = (N_valid + CH - 1) / CH;
  return static_cast<size_t>(score_grid(N_valid, H, B)) * (BM + 4) * n_chunks * sizeof(float) + 256;
}

cudaError_t launch_score_exact_bf16(const CUtensorMap* tq, const CUtensorMap* tk, const ScoreArgs& a,
                                    cudaStream_t s) {
  dim3 grid(score_grid(a.N_valid, a.H, a.B));
  const float scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(a.d)));
  if (a.d == 128) {
    const size_t smem = Layout<128>::bytes();
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(score_exact_bf16_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    score_exact_bf16_kernel<128><<<grid, kThreads, smem, s>>>(*tq, *tk, a, scale_log2);
  } else {
    const size_t smem = Layout<64>::bytes();
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(score_exact_bf16_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    score_exact_bf16_kernel<64><<<grid, kThreads, smem, s>>>(*tq, *tk, a, scale_log2);
  }
  return cudaGetLastError();
}

}  // namespace lbsa
