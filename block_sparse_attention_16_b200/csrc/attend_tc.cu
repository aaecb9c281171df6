// Block-sparse flash attention on sm_100a tensor cores (bf16 in, fp32 accumulate).
//
// What it computes (VMoBA review on pith.science, "What carries the argument":
// attention runs on the true keys and values of the kept blocks and on nothing
// else; LoSA abstract: the frozen block indices are reused at every later step):
//   out_r = sum_{c in K_i} softmax_{c in K_i}(q_r . k_c / sqrt(d)) v_c
// where K_i is the set of valid keys of the blocks kept for query block i.
// An empty list gives out_r = 0 and lse_r = -inf.
//
// Tiling.  A CTA owns a 128-row query tile (one 128-token block, or two
// 64-token blocks that share the tile).  It walks the ascending union of the
// tile's kept key blocks in 64-key steps; a row whose own block did not keep
// the current key block gives it zero probability.
//
// Warp roles (192 threads):
//   warps 0-3  softmax: thread t owns tile row t = TMEM lane t.  Reads S from
//              TMEM, keeps the running max / sum, writes P (bf16, packed two
//              per column) back over the first 32 columns of the same S
//              buffer, rescales O in TMEM when the running max grows by more
//              than 2^8, and writes the output.
//   warp 4     TMA producer: Q once, then K and V 64-key tiles through two
//              separate 2-stage rings, each refilled as soon as its slot frees.
//   warp 5     UMMA issuer: S = Q K^T (M=128, N=64, K=d, both operands in
//              smem) into one of two TMEM S buffers, then O += P V (M=128,
//              N=d, K=64, P read from TMEM) into TMEM.
// TMEM columns: [0,64) S0/P0, [64,128) S1/P1, [128,128+d) O.  About 100 KB of
// shared memory per CTA, so two CTAs (two softmax warpgroups) share an SM.
//
// Per-token lists (MASKED, 64-token blocks; VMoBA's per-token selection): an
// entry of a query block's list also carries the 64-bit set of its tokens that
// keep the key block; the tile keeps both blocks' sets per key block in shared
// memory, and a row outside the set gives that block zero probability.
#include "lbsa_device.cuh"

namespace lbsa {
namespace {

constexpr int BM = 128;           // query rows per tile
constexpr int BK = 64;            // keys per step
constexpr int NS = 2;             // K/V ring depth
constexpr int kThreads = 192;
constexpr int kMaxBlocks = 4096;  // nB bound (bitmap size)
constexpr int kMaxWords = kMaxBlocks / 32;
constexpr uint32_t kTmemCols = 256;
// kPoly8 of every 8 pairs of logits of a step without masked keys take their
// exponentials on the FMA pipe (scalar cubic, relative error < 8e-5, far below
// bf16's rounding of P), which unloads the MUFU; 0 keeps every one on the MUFU
#ifndef LBSA_ATT_POLY8
#define LBSA_ATT_POLY8 0
#endif
constexpr int kPoly8 = LBSA_ATT_POLY8;
template <int D>
struct Layout {
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BK * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NS * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + NS * KV_BYTES;
  // q_full, k_full[NS], k_empty[NS], v_full[NS], v_empty[NS], s_full[2], p_full[2], o_done[2], drain
  static constexpr int NBAR = 1 + 4 * NS + 7;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;        // tmem base, abort, n_entries, pad
  static constexpr int OFF_BITMAP = OFF_MISC + 16;
  static constexpr int OFF_SCHED = OFF_BITMAP + 2 * kMaxWords * 4;
  // per-token mask tables (MASKED): two uint64 per key block after the schedule
  __host__ __device__ static size_t mask_off(int nB) { return (OFF_SCHED + static_cast<size_t>(nB) * 4 + 7) & ~size_t(7); }
  static size_t bytes(int nB, bool masked = false) {
    return (masked ? mask_off(nB) + static_cast<size_t>(nB) * 16 : OFF_SCHED + static_cast<size_t>(nB) * 4) + 1024;
  }
};

struct Bars {
  uint64_t* q_full;
  uint64_t* k_full;
  uint64_t* k_empty;
  uint64_t* v_full;
  uint64_t* v_empty;
  uint64_t* s_full;
  uint64_t* p_full;
  uint64_t* o_done;
  uint64_t* drain;
};

__device__ __forceinline__ Bars make_bars(uint8_t* base) {
  uint64_t* b = reinterpret_cast<uint64_t*>(base);
  Bars r;
  r.q_full = b;
  r.k_full = b + 1;
  r.k_empty = b + 1 + NS;
  r.v_full = b + 1 + 2 * NS;
  r.v_empty = b + 1 + 3 * NS;
  r.s_full = b + 1 + 4 * NS;
  r.p_full = r.s_full + 2;
  r.o_done = r.p_full + 2;
  r.drain = r.o_done + 2;
  return r;
}

template <int D, bool MASKED>
__global__ void __launch_bounds__(kThreads, 2)
attend_bf16_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_v, const AttendArgs args, float scale_log2) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int tile = blockIdx.x;
  const int h = blockIdx.y;
  const int bb = blockIdx.z;
  const int nB = args.nB;
  const int blk = args.block;               // 64 or 128
  const int spb_log = (blk == 128) ? 1 : 0;  // log2 of the steps per kept key block (no division in the loops)
  const int spb = 1 << spb_log;

  Bars bars = make_bars(smem + L::OFF_BAR);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  uint32_t* bm0 = reinterpret_cast<uint32_t*>(smem + L::OFF_BITMAP);
  uint32_t* bm1 = bm0 + kMaxWords;
  uint32_t* sched = reinterpret_cast<uint32_t*>(smem + L::OFF_SCHED);
  uint64_t* maskA = reinterpret_cast<uint64_t*>(smem + L::mask_off(nB));   // MASKED: rows 0-63 of the tile
  uint64_t* maskB = maskA + nB;                                            // MASKED: rows 64-127
  const int nwords = (nB + 31) >> 5;
  // a CTA of this launch already gave up on a wait: skip the work, the call has failed
  if (*reinterpret_cast<volatile int32_t*>(args.status) == LBSA_ERR_TIMEOUT) return;

  // ---- set-up: barriers, TMEM, schedule (union of the tile's block lists)
  if (tid == 0) {
    mbar_init(bars.q_full, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(bars.k_full + i, 1);
      mbar_init(bars.k_empty + i, 1);
      mbar_init(bars.v_full + i, 1);
      mbar_init(bars.v_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bars.s_full + i, 1);
      mbar_init(bars.p_full + i, 128);
      mbar_init(bars.o_done + i, 1);
    }
    mbar_init(bars.drain, 1);
    misc[1] = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(misc, kTmemCols);
    tmem_relinquish();
  }
  for (int i = tid; i < nwords; i += kThreads) {
    bm0[i] = 0;
    bm1[i] = 0;
  }
  if (MASKED)
    for (int i = tid; i < 2 * nB; i += kThreads) maskA[i] = 0ull;
  __syncthreads();
  if (warp == 4 && lane == 0) {
    // the Q tile does not depend on the schedule: its load overlaps the build
    prefetch_tmap(&tmap_q);
    prefetch_tmap(&tmap_k);
    prefetch_tmap(&tmap_v);
    mbar_arrive_expect_tx(bars.q_full, L::Q_BYTES);
    for (int c = 0; c < D / 64; ++c)
      tma_load_4d(smem + L::OFF_Q + c * BM * 128, &tmap_q, bars.q_full, c * 64, tile * BM, h, bb);
  }

  const int qb0 = (blk == 64) ? 2 * tile : tile;
  const int qb1 = (blk == 64 && 2 * tile + 1 < nB) ? 2 * tile + 1 : -1;
  {
    // both rows' counts, then both lists, with their loads in flight together
    const long long row0 = (static_cast<long long>(bb) * args.H + h) * nB + qb0;
    const long long row1 = row0 + 1;
    const int c0 = args.counts[row0];
    const int c1 = (qb1 >= 0) ? args.counts[row1] : 0;
    const int32_t* l0 = args.cols + row0 * nB;
    const int32_t* l1 = args.cols + row1 * nB;
    for (int i = tid; i < max(c0, c1); i += kThreads) {
      const bool h0 = i < c0, h1 = i < c1;
      const int a = h0 ? l0[i] : 0;
      const int b = h1 ? l1[i] : 0;
      const uint64_t ma = (MASKED && h0) ? args.masks[row0 * nB + i] : 0ull;
      const uint64_t mb = (MASKED && h1) ? args.masks[row1 * nB + i] : 0ull;
      if (h0) {
        if (a < 0 || a >= nB) raise_status(args.status, LBSA_ERR_BAD_INDEX);
        else {
          atomicOr(&bm0[a >> 5], 1u << (a & 31));
          if (MASKED) maskA[a] = ma;
        }
      }
      if (h1) {
        if (b < 0 || b >= nB) raise_status(args.status, LBSA_ERR_BAD_INDEX);
        else {
          atomicOr(&bm1[b >> 5], 1u << (b & 31));
          if (MASKED) maskB[b] = mb;
        }
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    // each lane owns a contiguous run of bitmap words; exclusive scan of popcounts
    const int per = (nwords + 31) / 32;
    const int w0 = lane * per;
    int cnt = 0;
    for (int w = w0; w < w0 + per && w < nwords; ++w) cnt += __popc(bm0[w] | bm1[w]);
    int incl = cnt;
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int pos = incl - cnt;
    for (int w = w0; w < w0 + per && w < nwords; ++w) {
      const uint32_t a = bm0[w], b = bm1[w];
      uint32_t u = a | b;
      while (u) {
        const int bit = __ffs(u) - 1;
        u &= u - 1;
        uint32_t mask = (blk == 64) ? (((a >> bit) & 1u) | (((b >> bit) & 1u) << 1)) : 3u;
        sched[pos++] = static_cast<uint32_t>(w * 32 + bit) | (mask << 30);
      }
    }
    if (lane == 31) misc[2] = static_cast<uint32_t>(incl);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = misc[0];
  const int n_steps = static_cast<int>(misc[2]) * spb;
  const long long wl = args.wait_limit;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // a tile without steps never waits for Q: let the copy land before exit
      if (n_steps == 0) mbar_wait(bars.q_full, 0, wl, args.status, nullptr);
      // K and V stream through separate rings: K stage s is free once S = Q K^T
      // of step s - NS has completed, V stage s once O += P V of step s - NS
      // has.  Both slots are probed without blocking so that a K load never
      // queues behind a V stage that the softmax still holds.
      int sk = 0, sv = 0;
      uint64_t t_last = globaltimer_ns();
      while (sv < n_steps) {
        const bool k_free = sk < n_steps && (sk < NS || mbar_test_wait(bars.k_empty + sk % NS, ((sk / NS) & 1) ^ 1));
        const bool v_free = sv < sk && (sv < NS || mbar_test_wait(bars.v_empty + sv % NS, ((sv / NS) & 1) ^ 1));
        // K of step s+1 is consumed before V of step s: prefer it while it is at most one step ahead
        const bool do_k = k_free && (sk <= sv + 1 || !v_free);
        if (do_k || v_free) {
          const int s = do_k ? sk : sv;
          const int st = s % NS;
          const uint32_t e = sched[s >> spb_log];
          const int key0 = static_cast<int>(e & 0xFFFFu) * blk + (s & (spb - 1)) * BK;
          if (do_k) {
            uint8_t* sK = smem + L::OFF_K + st * L::KV_BYTES;
            mbar_arrive_expect_tx(bars.k_full + st, L::KV_BYTES);
            for (int c = 0; c < D / 64; ++c) tma_load_4d(sK + c * BK * 128, &tmap_k, bars.k_full + st, c * 64, key0, h, bb);
            ++sk;
          } else {
            uint8_t* sV = smem + L::OFF_V + st * L::KV_BYTES;
            mbar_arrive_expect_tx(bars.v_full + st, L::KV_BYTES);
            for (int c = 0; c < D / 64; ++c) tma_load_4d(sV + c * BK * 128, &tmap_v, bars.v_full + st, c * 64, key0, h, bb);
            ++sv;
          }
          t_last = globaltimer_ns();
          continue;
        }
        if (*abort_flag) break;
        if (globaltimer_ns() - t_last > static_cast<uint64_t>(wl)) {
          raise_status(args.status, LBSA_ERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
      }
      if (*abort_flag) {
        // let copies still in flight land before the CTA can exit
        mbar_wait(bars.q_full, 0, wl, args.status, nullptr);
        for (int s = (sk > NS ? sk - NS : 0); s < sk; ++s) mbar_wait(bars.k_full + s % NS, (s / NS) & 1, wl, args.status, nullptr);
        for (int s = (sv > NS ? sv - NS : 0); s < sv; ++s) mbar_wait(bars.v_full + s % NS, (s / NS) & 1, wl, args.status, nullptr);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(BM, BK, 0);
      const uint32_t idesc_o = idesc_bf16_f32(BM, D, 1);
      const uint32_t sQ = smem_u32(smem + L::OFF_Q);
      const uint32_t sK0 = smem_u32(smem + L::OFF_K);
      const uint32_t sV0 = smem_u32(smem + L::OFF_V);
      bool ok = n_steps == 0 || mbar_wait(bars.q_full, 0, wl, args.status, abort_flag);
      for (int s = 0; ok && s <= n_steps; ++s) {
        if (s < n_steps) {
          const int st = s % NS;
          if (!mbar_wait(bars.k_full + st, (s / NS) & 1, wl, args.status, abort_flag)) break;
          tc_fence_after();
          const uint32_t d_s = tmem + (s & 1) * BK;
          const uint32_t kbase = sK0 + st * L::KV_BYTES;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk & 3) * 32;
            const uint64_t a = smem_desc_sw128(sQ + (kk >> 2) * (BM * 128) + off, 16, 1024);
            const uint64_t b = smem_desc_sw128(kbase + (kk >> 2) * (BK * 128) + off, 16, 1024);
            umma_ss(d_s, a, b, idesc_s, kk > 0 ? 1u : 0u);
          }
          umma_commit(bars.s_full + (s & 1));
          umma_commit(bars.k_empty + st);
        }
        if (s >= 1) {
          const int j = s - 1;
          const int st = j % NS;
          if (!mbar_wait(bars.p_full + (j & 1), (j >> 1) & 1, wl, args.status, abort_flag)) break;
          if (!mbar_wait(bars.v_full + st, (j / NS) & 1, wl, args.status, abort_flag)) break;
          tc_fence_after();
          const uint32_t pcol = tmem + (j & 1) * BK;
          const uint32_t vbase = sV0 + st * L::KV_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t b = smem_desc_sw128(vbase + kk * 2048, BK * 128, 1024);
            umma_ts(tmem + 128, pcol + kk * 8, b, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(bars.o_done + (j & 1));
          umma_commit(bars.v_empty + st);
        }
      }
      // drain: every UMMA this thread issued has completed before TMEM is released
      umma_commit(bars.drain);
      mbar_wait(bars.drain, 0, wl, args.status, nullptr);
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 0-3)
    const int row = tid;                       // tile row == TMEM lane
    const int grow = tile * BM + row;          // token row
    const int half = row >> 6;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float m = -INFINITY;                       // running max (log2 units), possibly stale by < 8
    float l = 0.f;
    bool alive = true;
    for (int s = 0; s < n_steps && alive; ++s) {
      const int sb = s & 1;
      if (!mbar_wait(bars.s_full + sb, (s >> 1) & 1, wl, args.status, abort_flag)) { alive = false; break; }
      tc_fence_after();
      const uint32_t e = sched[s >> spb_log];
      const int key0 = static_cast<int>(e & 0xFFFFu) * blk + (s & (spb - 1)) * BK;
      const int nvk = args.N_valid - key0;     // valid keys in this step (may exceed 64)
      // warp-uniform: rows 0-63 (warps 0,1) and 64-127 (warps 2,3) are the two halves
      const bool take = (((e >> 30) >> half) & 1u) && nvk > 0;
      const bool full = take && nvk >= 64;
      // per-token lists: this row's own bit for the key block (not warp-uniform)
      bool mine = true;
      if (MASKED) mine = ((half ? maskB : maskA)[e & 0xFFFFu] >> (row & 63)) & 1ull;
      uint32_t r[64];
      tmem_ld32(t_lane + sb * BK, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
      tmem_ld32(t_lane + sb * BK + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
      tmem_wait_ld();
      // row max of the raw logits (the scale is positive), 4 independent chains
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (full) {
#pragma unroll
        for (int c = 0; c < 64; c += 2)
          mx4[(c >> 1) & 3] = fmax3(mx4[(c >> 1) & 3], __uint_as_float(r[c]), __uint_as_float(r[c + 1]));
      } else if (take) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c < nvk) mx4[c & 3] = fmaxf(mx4[c & 3], __uint_as_float(r[c]));
      }
      const float mx = (MASKED && !mine) ? -INFINITY : fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * scale_log2;
      const float m_new = fmaxf(m, mx);
      const bool need = (m != -INFINITY) && (m_new > m + 8.0f);
      if (m == -INFINITY) m = m_new;
      if (__any_sync(0xffffffffu, need)) {
        if (s >= 1 && !mbar_wait(bars.o_done + ((s - 1) & 1), ((s - 1) >> 1) & 1, wl, args.status, abort_flag)) {
          alive = false;
          break;
        }
        tc_fence_after();
        const float f = need ? ex2(m - m_new) : 1.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(t_lane + 128 + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
          tmem_st32(t_lane + 128 + c * 32, o);
        }
        tmem_wait_st();
        if (need) {
          l *= f;
          m = m_new;
        }
      }
      // p = 2^(s*scale - m): one packed FMA per pair, MUFU ex2, packed row-sum adds
      uint32_t pk[32];
      unsigned long long sum4[4] = {0ull, 0ull, 0ull, 0ull};
      const unsigned long long sc2 = f2_as_u64(scale_log2, scale_log2);
      const unsigned long long nm2 = f2_as_u64(-m, -m);
      if (full) {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          float v0, v1;
          u64_as_f2(ffma2(f2_as_u64(__uint_as_float(r[2 * c]), __uint_as_float(r[2 * c + 1])), sc2, nm2), v0, v1);
          const bool poly = ((c * kPoly8) & 7) < kPoly8;
          const float p0 = poly ? exp2_poly3(v0) : ex2(v0), p1 = poly ? exp2_poly3(v1) : ex2(v1);
          sum4[c & 3] = fadd2(sum4[c & 3], f2_as_u64(p0, p1));
          pk[c] = pack_bf16x2(p0, p1);
        }
      } else if (take) {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          float v0, v1;
          u64_as_f2(ffma2(f2_as_u64(__uint_as_float(r[2 * c]), __uint_as_float(r[2 * c + 1])), sc2, nm2), v0, v1);
          const float p0 = (2 * c < nvk) ? ex2(v0) : 0.f;
          const float p1 = (2 * c + 1 < nvk) ? ex2(v1) : 0.f;
          sum4[c & 3] = fadd2(sum4[c & 3], f2_as_u64(p0, p1));
          pk[c] = pack_bf16x2(p0, p1);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = 0u;
      }
      float sum8[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) u64_as_f2(sum4[i], sum8[2 * i], sum8[2 * i + 1]);
      float bsum = ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7]));
      if (MASKED && !mine) {
        // outside this row's own list: zero probability (values computed above are discarded)
        bsum = 0.f;
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = 0u;
      }
      l += bsum;
      if (s >= 2 && !mbar_wait(bars.o_done + sb, ((s - 2) >> 1) & 1, wl, args.status, abort_flag)) {
        alive = false;
        break;
      }
      // P row -> TMEM lane `row`, columns [sb*64, sb*64 + 32) of the S buffer just read
      tmem_st32(t_lane + sb * BK, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bars.p_full + sb);
    }
    // ---- epilogue: O / l  -> out, lse
    bool ok_o = alive && n_steps > 0 && !*abort_flag;
    if (ok_o) {
      ok_o = mbar_wait(bars.o_done + ((n_steps - 1) & 1), ((n_steps - 1) >> 1) & 1, wl, args.status, abort_flag);
      tc_fence_after();
    }
    const bool valid = grow < args.N_valid;
    const float inv = (l > 0.f) ? 1.f / l : 0.f;
    __nv_bfloat16* outp = reinterpret_cast<__nv_bfloat16*>(args.out);
    const long long obase = static_cast<long long>(bb) * args.ostride_b + static_cast<long long>(h) * args.ostride_h +
                            static_cast<long long>(grow) * args.ostride_n;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      if (__all_sync(0xffffffffu, ok_o)) {
        tmem_ld32(t_lane + 128 + c * 32, o);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0u;
      }
      if (valid) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
        uint4* dst = reinterpret_cast<uint4*>(outp + obase + c * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
      }
    }
    if (args.lse && valid) {
      const float v = (l > 0.f) ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      args.lse[(static_cast<long long>(bb) * args.H + h) * args.N_valid + grow] = v;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_attend_bf16(const CUtensorMap* tq, const CUtensorMap* tk, const CUtensorMap* tv,
                               const AttendArgs& a, cudaStream_t s) {
  const int tiles = (a.N_valid + BM - 1) / BM;
  dim3 grid(tiles, a.H, a.B);
  const float scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(a.d)));
  if (a.nB > kMaxBlocks) return cudaErrorInvalidValue;
  if (a.masks && a.block != 64) return cudaErrorInvalidValue;
  const bool masked = a.masks != nullptr;
  auto go = [&](auto kern, size_t smem) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, s>>>(*tq, *tk, *tv, a, scale_log2);
    return cudaGetLastError();
  };
  if (a.d == 128)
    return masked ? go(attend_bf16_kernel<128, true>, Layout<128>::bytes(a.nB, true))
                  : go(attend_bf16_kernel<128, false>, Layout<128>::bytes(a.nB));
  return masked ? go(attend_bf16_kernel<64, true>, Layout<64>::bytes(a.nB, true))
                : go(attend_bf16_kernel<64, false>, Layout<64>::bytes(a.nB));
}

}  // namespace lbsa
