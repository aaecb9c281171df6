// Block-sparse flash attention on sm_100a tensor cores, two query tiles per CTA
// in ping-pong (bf16 in, fp32 accumulate).
//
// What it computes (VMoBA review on pith.science, "What carries the argument":
// attention runs on the true keys and values of the kept blocks and on nothing
// else; LoSA abstract: the frozen block indices are reused at every later step):
//   out_r = sum_{c in K_i} softmax_{c in K_i}(q_r . k_c / sqrt(d)) v_c
// where K_i is the set of valid keys of the blocks kept for query block i.
// An empty list gives out_r = 0 and lse_r = -inf.
//
// Tiling.  A CTA owns two 128-row query tiles, A and B (tiles 2u and 2u+1 of
// its head).  A tile is one 128-token query block, or two 64-token blocks.  The
// CTA merges the kept lists of its query blocks into one list of key blocks,
// ordered: blocks kept by both tiles, then blocks only A keeps, then blocks
// only B keeps (ascending inside each group; each entry carries which query
// blocks keep it).  The list is walked in 128-key steps: one 128-token key
// block, or two consecutive 64-token entries (the halves of a step need not be
// adjacent in the sequence; each half is its own TMA box).  A tile takes part
// in the steps that hold an entry of its own, so the blocks both tiles keep are
// loaded once and feed both tiles' UMMAs, and a tile computes the blocks only
// it keeps alone.  A row gives zero probability to a key block its own query
// block did not keep.
//
// Why two tiles: S = Q K^T of one tile runs on the tensor pipe while the other
// tile's softmax runs on the CUDA cores.  Per tile t and step k, one "round" of
// UMMAs is O_t += P_t(k) V(k) followed by S_t(k+1) = Q_t K(k+1)^T (16 UMMAs of
// 128 x 128 x 16 at d = 128), and the issue order is
//   S_A(0) S_B(0) | round A(0) | round B(0) | round A(1) | round B(1) | ...
// so each tile's softmax of step k has the other tile's round to hide behind.
// 128-key S tiles keep every UMMA at N = 128, which the tensor pipe runs at its
// full rate; N = 64 does not.  A round needs two waits: its K/V slot pair (V(k)
// and K(k+1) land on one barrier) and its tile's P; the issuing warp has about
// as much queued UMMA work as a few hundred cycles, so per-round bookkeeping
// stays short.
//
// Warp roles (384 threads):
//   warps 0-3   softmax of tile A (thread t = tile row t = TMEM lane t)
//   warps 4-7   softmax of tile B
//   warp 8      TMA producer: Q_A, Q_B once, then per round the V and K tiles
//               into a pair of ring slots, in the order the UMMAs consume them
//               (a round both tiles share is loaded once)
//   warp 9      UMMA issuer (and TMEM owner): the whole warp walks the rounds
//               and waits, one elected lane issues
//   warps 10-11 idle after set-up
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A [256,256+d),
// O_B [384,384+d).  P (bf16, two per column) is written over the first 64
// columns of its tile's S buffer and read from there by O += P V.
//
// Ordering facts the kernel relies on: a tcgen05.commit arrives only when every
// UMMA the issuing thread launched before it has completed.  So when a softmax
// sees S_t(k) complete, O += P V of step k-1 is complete too: O_t may be
// rescaled and P_t(k) may overwrite P_t(k-1) without another wait, and nothing
// touches O_t or S_t until this softmax publishes P_t(k).
#include "lbsa_device.cuh"

namespace lbsa {
namespace {

constexpr int kBM = 128;           // query rows per tile
constexpr int kBN = 128;           // keys per step
constexpr int kThreads = 384;
constexpr int kMaxBlocks = 4096;   // nB bound (12-bit ids in the schedule)
constexpr uint32_t kTmemCols = 512;
// register split after set-up: 256 softmax threads x RegSplit::high + 128 others
// x RegSplit::low must not exceed what the CTA was launched with (384 x registers
// per thread); the launcher checks the kernel's count before the first launch
template <int D> struct RegSplit;                 // chosen by ptxas spill reports: none in the loops
template <> struct RegSplit<128> { static constexpr int high = 208, low = 72; };
template <> struct RegSplit<64> { static constexpr int high = 216, low = 56; };
template <int D>
constexpr int regs_launch_min() { return (256 * RegSplit<D>::high + 128 * RegSplit<D>::low + kThreads - 1) / kThreads; }
// kPoly8 of every 8 pairs of logits of a step without masked keys take their
// exponentials on the FMA pipe (scalar cubic, relative error < 8e-5, far below
// bf16's rounding of P), which unloads the MUFU; 0 keeps every exponential on
// the MUFU
#ifndef LBSA_PP_POLY8
#define LBSA_PP_POLY8 0
#endif
constexpr int kPoly8 = LBSA_PP_POLY8;

template <int D>
struct PPLayout {
  static constexpr int Q_BYTES = kBM * D * 2;            // one query tile
  static constexpr int SLOT_BYTES = kBN * D * 2;         // one K or V tile of 128 keys
  static constexpr int CHUNK_BYTES = kBN * 128;          // 64 d-columns of a slot (128-byte rows)
  static constexpr int NPAIR = (D == 128) ? 2 : 4;       // ring of slot pairs (V slot, K slot): 128 KB
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RING = 2 * Q_BYTES;
  static constexpr int OFF_BAR = OFF_RING + 2 * NPAIR * SLOT_BYTES;
  // q_full[2], pair_full[NPAIR], pair_empty[NPAIR], s_full[2], p_full[2], o_final[2], drain
  static constexpr int NBAR = 2 + 2 * NPAIR + 7;
  // [0] tmem base [1] abort [2] entries kept by both tiles [3] by A only [4] by B only
  // [5] the fused dense step's strip slot (-1: none)
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_LSE = (OFF_MISC + 32 + 15) / 16 * 16;   // fused dense step: [2 tiles][128 rows] row lse (log2)
  static constexpr int OFF_BITMAP = OFF_LSE + 2 * kBM * 4;  // 4 bitmaps of nB bits (A0, A1, B0, B1)
  __host__ __device__ static int words(int nB) { return (nB + 31) >> 5; }
  __host__ __device__ static int sched_off(int nB) { return OFF_BITMAP + 4 * words(nB) * 4; }
  // merged list: nB uint16 entries (bits 0-11 key block; bit 12 + 2*tile + half: that
  // query block keeps it, with half the 64-row half of the tile)
  static size_t bytes(int nB) { return static_cast<size_t>(sched_off(nB)) + 2 * static_cast<size_t>(nB) + 1024; }
};

struct PPBars {
  uint64_t* q_full;      // [2]
  uint64_t* pair_full;   // [NPAIR]  both tiles of the slot pair landed
  uint64_t* pair_empty;  // [NPAIR]  the last round that reads the pair has completed
  uint64_t* s_full;      // [2]
  uint64_t* p_full;      // [2]      all of P_t(k) is in TMEM
  uint64_t* o_final;     // [2]
  uint64_t* drain;
};

template <int NPAIR>
__device__ __forceinline__ PPBars pp_bars(uint8_t* base) {
  uint64_t* b = reinterpret_cast<uint64_t*>(base);
  PPBars r;
  r.q_full = b;
  r.pair_full = b + 2;
  r.pair_empty = b + 2 + NPAIR;
  r.s_full = b + 2 + 2 * NPAIR;
  r.p_full = r.s_full + 2;
  r.o_final = r.p_full + 2;
  r.drain = r.o_final + 2;
  return r;
}

// Key rows of the two 64-key halves of step `u` of the merged list, and the
// entries behind them (a 64-token list of odd length leaves the last step's
// second half empty: it repeats the first half's rows, which every row masks).
struct StepKeys {
  int row0, row1;
  uint32_t e0, e1;     // list entries (keep bits 12-15); e1 = 0 if the half is empty
};
__device__ __forceinline__ StepKeys step_keys(const uint16_t* list, int n_entries, int u, int blk) {
  StepKeys k;
  if (blk == 128) {
    const uint32_t e = list[u];
    k.e0 = k.e1 = e;
    k.row0 = static_cast<int>(e & 0xFFFu) * 128;
    k.row1 = k.row0 + 64;
  } else {
    k.e0 = list[2 * u];
    k.row0 = static_cast<int>(k.e0 & 0xFFFu) * 64;
    if (2 * u + 1 < n_entries) {
      k.e1 = list[2 * u + 1];
      k.row1 = static_cast<int>(k.e1 & 0xFFFu) * 64;
    } else {
      k.e1 = 0;
      k.row1 = k.row0;
    }
  }
  return k;
}

// Which steps of the merged list each tile takes.  With e entries per step
// (2 for 64-token blocks, 1 for 128), nb entries kept by both tiles, na by A
// only and nc by B only: A takes steps [0, ceil((nb+na)/e)); B takes
// [0, ceil(nb/e)) and, when nc > 0, [lo2, ceil((nb+na+nc)/e)) with
// lo2 = max(floor((nb+na)/e), ceil(nb/e)).  Tile A's k-th step is step k; tile
// B's is step_b(k).  Step k is shared when both tiles' k-th step is step k.
struct TileSteps {
  int nA, nB1, lo2, nB;
  __device__ __forceinline__ void init(int nb, int na, int nc, int e) {
    const int nU = nb + na + nc;
    nA = (nb + na + e - 1) / e;
    nB1 = (nb + e - 1) / e;
    lo2 = max((nb + na) / e, nB1);
    nB = nB1 + (nc > 0 ? (nU + e - 1) / e - lo2 : 0);
  }
  __device__ __forceinline__ int step_b(int k) const { return k < nB1 ? k : lo2 + (k - nB1); }
  __device__ __forceinline__ bool shared(int k) const { return k < nA && k < nB && step_b(k) == k; }
  __device__ __forceinline__ int step(int t, int k) const { return t ? step_b(k) : k; }
  // tile B's round k reads the very slot pair tile A's round k loaded: the same
  // V(k), and the same K(k+1) or none for both
  __device__ __forceinline__ bool pair_shared(int k) const {
    if (!shared(k)) return false;
    const bool na = k + 1 < nA, nb = k + 1 < nB;
    return na == nb && (!na || shared(k + 1));
  }
};

// The slot pairs both the producer and the UMMA issuer walk, in the order the
// UMMAs consume them: tile A's first S, tile B's first S (unless it shares A's
// step 0), then per step k: tile A's round k, tile B's round k (unless it
// shares A's pair).  A pair holds the round's V(k) in its first slot and its
// K(k+1) in the second (the first S of a tile holds only K(0)).
struct PairItem {
  int tile, k;      // k = -1: the tile's first S
  bool has_v, has_k;
};
struct PairSeq {
  const TileSteps* ts;
  int k, t;         // next round (k = -1: first S)
  __device__ __forceinline__ void init(const TileSteps* s) { ts = s; k = -1; t = 0; }
  // next pair that needs a load; false when done
  __device__ __forceinline__ bool next(PairItem& it) {
    for (;;) {
      if (k >= ts->nA && k >= ts->nB) return false;
      const int tt = t, kk = k;
      if (++t == 2) { t = 0; ++k; }
      const int n = tt ? ts->nB : ts->nA;
      if (kk < 0) {
        if (n == 0 || (tt == 1 && ts->shared(0))) continue;
        it = {tt, -1, false, true};
        return true;
      }
      if (kk >= n || (tt == 1 && ts->pair_shared(kk))) continue;
      it = {tt, kk, true, kk + 1 < n};
      return true;
    }
  }
};

// One half (64 logits, r[64*HF .. 64*HF + 63]) of a row: p = 2^(s*scale - m)
// as one packed FMA per pair then two MUFU ex2 (or, for POLY8 of every 8
// pairs, spread out, the FMA-pipe cubic), the packed row-sum adds, and P packed
// to bf16 into pk.  With MAX the pairs of the OTHER half also feed the 8 row-max
// chains (independent work that overlaps the exponentials).
template <int POLY8, int HF, bool MAX>
__device__ __forceinline__ void exp_half(const uint32_t (&r)[128], unsigned long long sc2, unsigned long long nm2,
                                         unsigned long long (&sum4)[4], uint32_t (&pk)[32], float (&mx8)[8]) {
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    const int j = HF * 64 + 2 * c;
    if (MAX) {
      const int o = (1 - HF) * 64 + 2 * c;
      mx8[c & 7] = fmax3(mx8[c & 7], __uint_as_float(r[o]), __uint_as_float(r[o + 1]));
    }
    const unsigned long long v = ffma2(f2_as_u64(__uint_as_float(r[j]), __uint_as_float(r[j + 1])), sc2, nm2);
    float p0, p1;
    if (((c * POLY8) & 7) < POLY8) {
      float v0, v1;
      u64_as_f2(v, v0, v1);
      p0 = exp2_poly3(v0);
      p1 = exp2_poly3(v1);
    } else {
      float v0, v1;
      u64_as_f2(v, v0, v1);
      p0 = ex2(v0);
      p1 = ex2(v1);
    }
    sum4[c & 3] = fadd2(sum4[c & 3], f2_as_u64(p0, p1));
    pk[c] = pack_bf16x2(p0, p1);
  }
}

// The row max over the first half's 64 logits alone, 8 chains.
__device__ __forceinline__ void max_half0(const uint32_t (&r)[128], float (&mx8)[8]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) mx8[j] = fmaxf(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
#pragma unroll
  for (int c = 16; c < 64; c += 2)
    mx8[(c >> 1) & 7] = fmax3(mx8[(c >> 1) & 7], __uint_as_float(r[c]), __uint_as_float(r[c + 1]));
}

// Warp transpose-reduce: lane l holds x[0..31] (one partial per key block);
// afterwards x[0] of lane l is the sum over the 32 lanes of x[l].  Five levels;
// at the level of width w a lane keeps the half of its values that its lane bit w
// selects, sends the other half to lane ^ w and adds what it receives.
__device__ __forceinline__ void warp_transpose_reduce32(float (&x)[32], int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool upper = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float send = upper ? x[i] : x[i + w];
      const float keep = upper ? x[i + w] : x[i];
      x[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
    }
  }
}

// The row sum of the packed partial sums (a fixed order).
__device__ __forceinline__ float hsum4(const unsigned long long (&sum4)[4]) {
  float s8[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) u64_as_f2(sum4[i], s8[2 * i], s8[2 * i + 1]);
  return ((s8[0] + s8[1]) + (s8[2] + s8[3])) + ((s8[4] + s8[5]) + (s8[6] + s8[7]));
}

__device__ __forceinline__ float max8(const float (&mx8)[8]) {
  return fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])), fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
}

// The running max after seeing a new (scaled) max mx: an integer, raised only
// when mx passes it by more than 8 (so every p it gives stays <= 2^8), and set
// at the first finite max.
__device__ __forceinline__ float raise_max(float m, float mx) {
  if (m == -INFINITY) return mx == -INFINITY ? m : ceilf(mx);
  return mx > m + 8.0f ? ceilf(mx) : m;
}

template <int D, bool FUSED>
__global__ void __launch_bounds__(kThreads, 1)
attend_pp_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                 const __grid_constant__ CUtensorMap tmap_v, const AttendArgs args, float scale_log2) {
  using L = PPLayout<D>;
  constexpr int NPAIR = L::NPAIR;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int h = blockIdx.y;
  const int bb = blockIdx.z;
  const int nB = args.nB;
  const int blk = args.block;
  const int n_tiles = (args.N_valid + kBM - 1) / kBM;
  const int tileA = 2 * blockIdx.x;
  const bool hasB = tileA + 1 < n_tiles;

  PPBars bars = pp_bars<NPAIR>(smem + L::OFF_BAR);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  const int nwords = L::words(nB);
  uint32_t* bm = reinterpret_cast<uint32_t*>(smem + L::OFF_BITMAP);     // [4][nwords]
  uint16_t* sched = reinterpret_cast<uint16_t*>(smem + L::sched_off(nB));   // merged list [nB]
  // a CTA of this launch already gave up on a wait: skip the work, the call has failed
  if (*reinterpret_cast<volatile int32_t*>(args.status) == LBSA_ERR_TIMEOUT) return;

  // ---- set-up: barriers, TMEM, the two tiles' schedules
  if (tid == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(bars.q_full + t, 1);
      mbar_init(bars.s_full + t, 1);
      mbar_init(bars.p_full + t, 4);            // one arrival per softmax warp of the tile
      mbar_init(bars.o_final + t, 1);
    }
    for (int i = 0; i < NPAIR; ++i) {
      mbar_init(bars.pair_full + i, 1);
      mbar_init(bars.pair_empty + i, 1);
    }
    mbar_init(bars.drain, 1);
    misc[1] = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(misc, kTmemCols);
    tmem_relinquish();
  }
  for (int i = tid; i < 4 * nwords; i += kThreads) bm[i] = 0;
  __syncthreads();
  if (warp == 8 && lane == 0) {
    // the Q tiles do not depend on the schedules: their loads overlap the build
    prefetch_tmap(&tmap_q);
    prefetch_tmap(&tmap_k);
    prefetch_tmap(&tmap_v);
    for (int t = 0; t < (hasB ? 2 : 1); ++t) {
      mbar_arrive_expect_tx(bars.q_full + t, L::Q_BYTES);
      for (int c = 0; c < D / 64; ++c)
        tma_load_4d(smem + L::OFF_Q + t * L::Q_BYTES + c * kBM * 128, &tmap_q, bars.q_full + t, c * 64,
                    (tileA + t) * kBM, h, bb);
    }
  }
  if (FUSED) {
    // dense step: every key block for every query block of the CTA
    for (int i = tid; i < nwords; i += kThreads) {
      const uint32_t all = (i == nwords - 1 && (nB & 31)) ? ((1u << (nB & 31)) - 1u) : 0xffffffffu;
      bm[i] = all;
      bm[nwords + i] = all;
      bm[2 * nwords + i] = hasB ? all : 0u;
      bm[3 * nwords + i] = hasB ? all : 0u;
    }
    if (tid == 0) {
      // a strip slot: at most one CTA per SM holds TMEM at a time and each holds one
      // slot, so a free one exists; the probe is bounded all the same
      int slot = -1;
      const uint64_t t0 = globaltimer_ns();
      for (int i = (blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z)) % args.n_slots;;
           i = (i + 1) % args.n_slots) {
        if (atomicCAS(args.slots + i, 0, 1) == 0) {
          slot = i;
          break;
        }
        if (globaltimer_ns() - t0 > static_cast<uint64_t>(args.wait_limit)) {
          raise_status(args.status, LBSA_ERR_TIMEOUT);
          break;
        }
      }
      __threadfence();
      misc[5] = static_cast<uint32_t>(slot);
    }
  } else {
    // query blocks: b = 64: A0 = 4u, A1 = 4u+1, B0 = 4u+2, B1 = 4u+3; b = 128: A = 2u, B = 2u+1
    const long long hrow = (static_cast<long long>(bb) * args.H + h) * nB;
    const int per_tile = (blk == 64) ? 2 : 1;
    for (int q = 0; q < 4; ++q) {
      const int t = q >> 1, sub = q & 1;
      if (sub >= per_tile) continue;
      if (t == 1 && !hasB) continue;
      const int qb = (tileA + t) * per_tile + sub;
      if (qb >= nB) continue;
      const int cnt = args.counts[hrow + qb];
      const int32_t* lst = args.cols + (hrow + qb) * nB;
      uint32_t* map = bm + q * nwords;
      for (int i = tid; i < cnt; i += kThreads) {
        const int a = lst[i];
        if (a < 0 || a >= nB) raise_status(args.status, LBSA_ERR_BAD_INDEX);
        else atomicOr(&map[a >> 5], 1u << (a & 31));
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    // the merged list: both tiles' blocks, then A's only, then B's only; each
    // lane owns a run of bitmap words and scans the three group counts
    const uint32_t* a0 = bm;
    const uint32_t* a1 = bm + nwords;
    const uint32_t* b0 = bm + 2 * nwords;
    const uint32_t* b1 = bm + 3 * nwords;
    const int per = (nwords + 31) / 32;
    const int w0 = lane * per;
    int cnt[3] = {0, 0, 0};
    for (int w = w0; w < w0 + per && w < nwords; ++w) {
      const uint32_t ta = a0[w] | a1[w], tb = b0[w] | b1[w];
      cnt[0] += __popc(ta & tb);
      cnt[1] += __popc(ta & ~tb);
      cnt[2] += __popc(tb & ~ta);
    }
    int pos[3], tot[3];
#pragma unroll
    for (int g = 0; g < 3; ++g) {
      int incl = cnt[g];
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      tot[g] = __shfl_sync(0xffffffffu, incl, 31);
      pos[g] = incl - cnt[g];
    }
    int p0 = pos[0], p1 = pos[1] + tot[0], p2 = pos[2] + tot[0] + tot[1];
    for (int w = w0; w < w0 + per && w < nwords; ++w) {
      const uint32_t x0 = a0[w], x1 = a1[w], x2 = b0[w], x3 = b1[w];
      const uint32_t ta = x0 | x1, tb = x2 | x3;
      uint32_t u = ta | tb;
      while (u) {
        const int bit = __ffs(u) - 1;
        u &= u - 1;
        uint32_t keep;
        if (blk == 64)
          keep = ((x0 >> bit) & 1u) | (((x1 >> bit) & 1u) << 1) | (((x2 >> bit) & 1u) << 2) | (((x3 >> bit) & 1u) << 3);
        else
          keep = (((ta >> bit) & 1u) ? 3u : 0u) | (((tb >> bit) & 1u) ? 12u : 0u);
        const int g = (keep & 3u) ? ((keep & 12u) ? 0 : 1) : 2;
        const int at = g == 0 ? p0 : (g == 1 ? p1 : p2);
        sched[at] = static_cast<uint16_t>((w * 32 + bit) | (keep << 12));
        p0 += g == 0;
        p1 += g == 1;
        p2 += g == 2;
      }
    }
    if (lane == 0) {
      // fused step without a strip slot: no steps (the call has failed)
      const bool none = FUSED && static_cast<int>(misc[5]) < 0;
      misc[2] = none ? 0u : static_cast<uint32_t>(tot[0]);
      misc[3] = none ? 0u : static_cast<uint32_t>(tot[1]);
      misc[4] = none ? 0u : static_cast<uint32_t>(tot[2]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const long long wl = args.wait_limit;
  // each role reads the list shape from shared memory itself (nothing computed
  // here stays live across the register split below)
#define PP_LIST_SHAPE                                                                                      \
  const uint32_t tmem = misc[0];                                                                           \
  const int nU = static_cast<int>(misc[2] + misc[3] + misc[4]);                                            \
  TileSteps ts;                                                                                            \
  ts.init(static_cast<int>(misc[2]), static_cast<int>(misc[3]), static_cast<int>(misc[4]), blk == 64 ? 2 : 1); \
  const int nSA = ts.nA, nSB = ts.nB;                                                                      \
  (void)tmem;                                                                                              \
  (void)nU

  // registers: the producer / UMMA warpgroup gives up most of its share to the
  // two softmax warpgroups (each thread of those holds a full 128-column S row)
  if (warp >= 8) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(RegSplit<D>::low));
  PP_LIST_SHAPE;
  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      PairSeq seq;
      seq.init(&ts);
      PairItem it;
      int cnt = 0;
      bool ok = true;
      while (seq.next(it)) {
        const int pr = cnt % NPAIR;
        if (cnt >= NPAIR && !mbar_wait(bars.pair_empty + pr, ((cnt / NPAIR) & 1) ^ 1, wl, args.status, abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* dst = smem + L::OFF_RING + pr * 2 * L::SLOT_BYTES;
        mbar_arrive_expect_tx(bars.pair_full + pr, (it.has_v + it.has_k) * L::SLOT_BYTES);
        for (int part = 0; part < 2; ++part) {
          if (part == 0 ? !it.has_v : !it.has_k) continue;
          const StepKeys kk = step_keys(sched, nU, ts.step(it.tile, part == 0 ? it.k : it.k + 1), blk);
          const CUtensorMap* map = part == 0 ? &tmap_v : &tmap_k;
          uint8_t* slot = dst + part * L::SLOT_BYTES;
          for (int c = 0; c < D / 64; ++c) {
            tma_load_4d(slot + c * L::CHUNK_BYTES, map, bars.pair_full + pr, c * 64, kk.row0, h, bb);
            tma_load_4d(slot + c * L::CHUNK_BYTES + 64 * 128, map, bars.pair_full + pr, c * 64, kk.row1, h, bb);
          }
        }
        ++cnt;
      }
      (void)ok;
      // every copy this thread issued has landed before the CTA can exit (on the
      // normal path these phases completed long ago: the waits return at once)
      for (int t = 0; t < (hasB ? 2 : 1); ++t) mbar_wait(bars.q_full + t, 0, wl, args.status, nullptr);
      for (int c = (cnt > NPAIR ? cnt - NPAIR : 0); c < cnt; ++c)
        mbar_wait(bars.pair_full + c % NPAIR, (c / NPAIR) & 1, wl, args.status, nullptr);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ UMMA issuer
    // The whole warp walks the rounds and waits (its values stay warp-uniform);
    // one elected lane issues.  Shared-memory descriptors are built
    // once and moved by adding 16-byte units to their start-address field (every
    // operand lies below 256 KB, so the 14-bit field never carries).
    const uint32_t idesc_s = idesc_bf16_f32(kBM, kBN, 0);
    const uint32_t idesc_o = idesc_bf16_f32(kBM, D, 1);
    const uint64_t dQ = smem_desc_sw128(smem_u32(smem + L::OFF_Q), 16, 1024);
    const uint64_t dK = smem_desc_sw128(smem_u32(smem + L::OFF_RING + L::SLOT_BYTES), 16, 1024);
    const uint64_t dV = smem_desc_sw128(smem_u32(smem + L::OFF_RING), L::CHUNK_BYTES, 1024);
    // every lane waits; the outcome is made warp-uniform so the lanes leave together
    auto wait0 = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, wl, args.status, abort_flag));
    };
    auto issue_s = [&](int t, int pr, bool release) {
      const uint64_t a0 = dQ + static_cast<uint64_t>((t * L::Q_BYTES) >> 4);
      const uint64_t b0 = dK + static_cast<uint64_t>((pr * 2 * L::SLOT_BYTES) >> 4);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t a_off = ((kk >> 2) * (kBM * 128) + (kk & 3) * 32) >> 4;
        const uint32_t b_off = ((kk >> 2) * L::CHUNK_BYTES + (kk & 3) * 32) >> 4;
        umma_ss(tmem + t * 128, a0 + a_off, b0 + b_off, idesc_s, kk > 0 ? 1u : 0u);
      }
      umma_commit(bars.s_full + t);
      if (release) umma_commit(bars.pair_empty + pr);
    };
    bool ok = true;
    for (int t = 0; t < 2 && ok; ++t)
      if ((t ? nSB : nSA) > 0) ok = wait0(bars.q_full + t, 0);
    int cnt = 0;                   // pairs consumed so far (ring position)
    int pr_a = 0;                  // tile A's latest pair (tile B may share it)
    // the pair of tile t's next round (k = -1: first S); waits for it unless shared
    auto take = [&](int t, int k, int& pr, bool& release) {
      const bool sh = t == 1 && (k < 0 ? ts.shared(0) : ts.pair_shared(k));
      const bool a_shares = t == 0 && (k < 0 ? (nSB > 0 && ts.shared(0)) : ts.pair_shared(k));
      release = !a_shares;
      if (sh) {
        pr = pr_a;
        return true;
      }
      pr = cnt % NPAIR;
      if (!wait0(bars.pair_full + pr, (cnt / NPAIR) & 1)) return false;
      ++cnt;
      if (t == 0) pr_a = pr;
      return true;
    };
    // first S of each tile
    for (int t = 0; t < 2 && ok; ++t) {
      if ((t ? nSB : nSA) == 0) continue;
      int pr;
      bool rel;
      if (!(ok = take(t, -1, pr, rel))) break;
      tc_fence_after();
      if (elect_one()) issue_s(t, pr, rel);
      __syncwarp();
    }
    // rounds: per tile, O_t += P_t(k) V(k) then S_t(k+1) = Q_t K(k+1)^T
    for (int k = 0; ok && (k < nSA || k < nSB); ++k) {
      for (int t = 0; t < 2; ++t) {
        const int n = t ? nSB : nSA;
        if (k >= n) continue;
        int pr;
        bool rel;
        if (!(ok = take(t, k, pr, rel))) break;
        if (!(ok = wait0(bars.p_full + t, k & 1))) break;
        tc_fence_after();
        const uint64_t b0 = dV + static_cast<uint64_t>((pr * 2 * L::SLOT_BYTES) >> 4);
        if (elect_one()) {
          // P from TMEM (S_t's first 64 columns), V MN-major in smem
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            umma_ts(tmem + 256 + t * 128, tmem + t * 128 + kk * 8, b0 + kk * (2048 >> 4), idesc_o,
                    (k > 0 || kk > 0) ? 1u : 0u);
          if (k + 1 < n) {
            issue_s(t, pr, rel);
          } else {
            umma_commit(bars.o_final + t);
            if (rel) umma_commit(bars.pair_empty + pr);
          }
        }
        __syncwarp();
      }
    }
    // drain: every UMMA this warp issued has completed before TMEM is released
    if (elect_one()) umma_commit(bars.drain);
    __syncwarp();
    mbar_wait(bars.drain, 0, wl, args.status, nullptr);
  }
  } else {
    // ------------------------------------------------------------ softmax (warps 0-7)
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(RegSplit<D>::high));
    PP_LIST_SHAPE;
    const int t = warp >> 2;                   // tile
    const int row = tid & 127;                 // tile row == TMEM lane
    const int grow = (tileA + t) * kBM + row;  // token row
    const int rh = row >> 6;                   // row half (64-token blocks: which query block)
    const uint32_t t_lane = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t s_col = t * 128;
    const uint32_t o_col = 256 + t * 128;
    const int n_steps = t ? nSB : nSA;
    const int kbit = 12 + 2 * t + rh;          // this row's keep bit in a list entry
    // fused dense step: this CTA's strip, [tile][64-key chunk][row] log-sum-exp (log2 units)
    const int n_chunks = (args.N_valid + 63) / 64;
    const int slot = FUSED ? static_cast<int>(misc[5]) : -1;
    // this row's column of its tile's strip: an element offset into the scratch
    // (below 2^31: at most 2 x SM count x 128 x 8192 floats), -1 without a slot
    const int soff = (FUSED && slot >= 0) ? ((slot * 2 + t) * n_chunks * kBM + row) : -1;
    float m = -INFINITY;                       // running max (log2 units, an integer), possibly stale by < 8
    float l = 0.f;
    bool alive = true;
    const unsigned long long sc2 = f2_as_u64(scale_log2, scale_log2);
    for (int s = 0; s < n_steps; ++s) {
      if (!mbar_wait(bars.s_full + t, s & 1, wl, args.status, abort_flag)) {
        alive = false;
        break;
      }
      tc_fence_after();
      const StepKeys kk = step_keys(sched, nU, ts.step(t, s), blk);
      // valid keys of each half for this row (warp-uniform: rh is uniform per warp)
      const int nv0 = ((kk.e0 >> kbit) & 1u) ? min(64, max(0, args.N_valid - kk.row0)) : 0;
      const int nv1 = ((kk.e1 >> kbit) & 1u) ? min(64, max(0, args.N_valid - kk.row1)) : 0;
      const bool full = nv0 == 64 && nv1 == 64;   // every key of the step counts for this row
      // S row: the second half's load is in flight while the first half's max runs
      uint32_t r[128];
      tmem_ld32(t_lane + s_col, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
      tmem_ld32(t_lane + s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
      tmem_wait_ld_dep(*reinterpret_cast<uint32_t(*)[32]>(&r[0]));
      reg_dep(*reinterpret_cast<uint32_t(*)[32]>(&r[32]));
      tmem_ld32(t_lane + s_col + 64, *reinterpret_cast<uint32_t(*)[32]>(&r[64]));
      tmem_ld32(t_lane + s_col + 96, *reinterpret_cast<uint32_t(*)[32]>(&r[96]));
      if (!full) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c >= nv0) r[c] = __float_as_uint(-INFINITY);
      }
      // The running max m is an integer (log2 units), so rescaling by 2^(m_old -
      // m_new) is exact.  The first half's max is found first and m raised if
      // needed; the first half's exponentials run fused with the second half's
      // max; if the full max raises m further, the first half's P (still in
      // registers) and its sum are scaled down to it, exactly; then the second
      // half.  Every p stays <= 2^8.
      const float m_start = m;
      float mx8[8];
      max_half0(r, mx8);
      const float mx0 = max8(mx8) * scale_log2;
      m = raise_max(m, mx0);
      tmem_wait_ld_dep(*reinterpret_cast<uint32_t(*)[32]>(&r[64]));
      reg_dep(*reinterpret_cast<uint32_t(*)[32]>(&r[96]));
      if (!full) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c >= nv1) r[64 + c] = __float_as_uint(-INFINITY);
      }
      const float m_h0 = m;
#pragma unroll
      for (int j = 0; j < 8; ++j) mx8[j] = -INFINITY;
      unsigned long long sum4[4] = {0ull, 0ull, 0ull, 0ull};
      uint32_t pk[32];
      {
        const float mu = (m == -INFINITY) ? 0.f : m;      // nothing valid so far: every p is 0
        const unsigned long long nm2 = f2_as_u64(-mu, -mu);
        if (kPoly8 > 0 && full) exp_half<kPoly8, 0, true>(r, sc2, nm2, sum4, pk, mx8);
        else exp_half<0, 0, true>(r, sc2, nm2, sum4, pk, mx8);
      }
      m = raise_max(m, fmaxf(mx0, max8(mx8) * scale_log2));
      if (__any_sync(0xffffffffu, m != m_h0)) {
        // a power of two (0 when the first half had nothing valid: its p are 0)
        const float f = (m == m_h0) ? 1.f : (m_h0 == -INFINITY ? 0.f : ex2(m_h0 - m));
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float lo = __uint_as_float(pk[i] << 16), hi = __uint_as_float(pk[i] & 0xFFFF0000u);
          pk[i] = pack_bf16x2(lo * f, hi * f);
        }
        const unsigned long long f2 = f2_as_u64(f, f);
#pragma unroll
        for (int i = 0; i < 4; ++i) sum4[i] = ffma2(sum4[i], f2, 0ull);
      }
      tmem_st32(t_lane + s_col, pk);
      float sum_h0 = 0.f;
      if (FUSED) {
        // the fused step keeps the two 64-key halves' sums apart
        sum_h0 = hsum4(sum4);
#pragma unroll
        for (int i = 0; i < 4; ++i) sum4[i] = 0ull;
      }
      {
        const float mu = (m == -INFINITY) ? 0.f : m;
        const unsigned long long nm2 = f2_as_u64(-mu, -mu);
        if (kPoly8 > 0 && full) exp_half<kPoly8, 1, false>(r, sc2, nm2, sum4, pk, mx8);
        else exp_half<0, 1, false>(r, sc2, nm2, sum4, pk, mx8);
      }
      tmem_st32(t_lane + s_col + 32, pk);
      float sum_step = hsum4(sum4);
      // fused step: each 64-key chunk's log-sum-exp (log2 units), chunks 2u and 2u + 1
      // of merged-list step u (the dense list walks every key block in order); stored
      // once P is published, so the stores never hold up the arrival
      float lse_c0 = 0.f, lse_c1 = 0.f;
      if (FUSED) {
        lse_c0 = m + __log2f(sum_h0);
        lse_c1 = m + __log2f(sum_step);
        sum_step += sum_h0;
      }
      // O and the row sum of earlier steps, rescaled to the new max (exactly)
      const bool need = m_start != -INFINITY && m != m_start;
      if (__any_sync(0xffffffffu, need)) {
        // O_t is quiescent here (see the ordering facts at the top): rescale it in
        // place before O_t += P_t(k) V(k) may start (it waits for P_t(k))
        const float f = need ? ex2(m_start - m) : 1.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(t_lane + o_col + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
          tmem_st32(t_lane + o_col + c * 32, o);
        }
        l *= f;
      }
      l += sum_step;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.p_full + t);
      if (FUSED && soff >= 0) {
        const int c0 = 2 * ts.step(t, s);
        if (c0 < n_chunks) args.fscratch[soff + c0 * kBM] = lse_c0;
        if (c0 + 1 < n_chunks) args.fscratch[soff + (c0 + 1) * kBM] = lse_c1;
      }
    }
    // ---- epilogue: O / l -> out, lse
    bool ok_o = alive && n_steps > 0 && !*abort_flag;
    if (ok_o) {
      ok_o = mbar_wait(bars.o_final + t, 0, wl, args.status, abort_flag);
      tc_fence_after();
    }
    const bool valid = grow < args.N_valid && (t == 0 || hasB);
    const float inv = (l > 0.f) ? 1.f / l : 0.f;
    __nv_bfloat16* outp = reinterpret_cast<__nv_bfloat16*>(args.out);
    const long long obase = static_cast<long long>(bb) * args.ostride_b + static_cast<long long>(h) * args.ostride_h +
                            static_cast<long long>(grow) * args.ostride_n;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      if (__all_sync(0xffffffffu, ok_o)) {
        tmem_ld32(t_lane + o_col + c * 32, o);
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
    if (FUSED) {
      // exact block masses (LoSA abstract): 2^(L[r,c] - lse_r) is row r's share on
      // chunk c.  Each warp of the tile takes groups of 32 key blocks; lane l reads
      // rows l, l+32, l+64, l+96 of each chunk (coalesced), sums per query block, and
      // a transpose-reduce leaves key block 32g + l's sums in lane l.  Invalid rows
      // have lse = +inf and add nothing.
      float* lse_s = reinterpret_cast<float*>(smem + L::OFF_LSE) + t * kBM;
      lse_s[row] = (valid && l > 0.f) ? m + __log2f(l) : INFINITY;
      named_bar_sync(1 + t, kBM);
      if (soff >= 0 && (t == 0 || hasB) && __all_sync(0xffffffffu, ok_o)) {
        const float* st = args.fscratch + (soff - row) + lane;     // the tile's strip, this lane's row
        const long long hrow = (static_cast<long long>(bb) * args.H + h) * nB;
        float ls[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) ls[j] = lse_s[lane + 32 * j];
        for (int g = warp & 3; g * 32 < nB; g += 4) {
          float x0[32], x1[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int kb = g * 32 + j;
            float a0 = 0.f, a1 = 0.f;
            if (blk == 64) {
              if (kb < nB) {
                const float* sc = st + static_cast<long long>(kb) * kBM;
                a0 = ex2(sc[0] - ls[0]) + ex2(sc[32] - ls[1]);
                a1 = ex2(sc[64] - ls[2]) + ex2(sc[96] - ls[3]);
              }
            } else {
#pragma unroll
              for (int cc = 0; cc < 2; ++cc) {
                if (2 * kb + cc < n_chunks) {
                  const float* sc = st + static_cast<long long>(2 * kb + cc) * kBM;
                  a0 += (ex2(sc[0] - ls[0]) + ex2(sc[32] - ls[1])) + (ex2(sc[64] - ls[2]) + ex2(sc[96] - ls[3]));
                }
              }
            }
            x0[j] = a0;
            x1[j] = a1;
          }
          warp_transpose_reduce32(x0, lane);
          if (blk == 64) warp_transpose_reduce32(x1, lane);
          const int kb = g * 32 + lane;
          if (kb < nB) {
            for (int q = 0; q < (blk == 64 ? 2 : 1); ++q) {
              const int qb = (blk == 64) ? 2 * (tileA + t) + q : tileA + t;
              if (qb >= nB) continue;
              const int rv = min(blk, args.N_valid - qb * blk);
              args.scores[(hrow + qb) * nB + kb] = (q ? x1[0] : x0[0]) / static_cast<float>(rv);
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (FUSED && tid == 0 && static_cast<int>(misc[5]) >= 0) {
    __threadfence();                          // the strip's last readers are done
    atomicExch(args.slots + misc[5], 0);
  }
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(misc[0], kTmemCols);
  }
#undef PP_LIST_SHAPE
}

}  // namespace

bool attend_pp_supported(const AttendArgs& a) {
  return a.masks == nullptr && a.nB <= kMaxBlocks && (a.d == 64 || a.d == 128) && (a.block == 64 || a.block == 128);
}

namespace {
template <bool FUSED>
cudaError_t launch_pp(const CUtensorMap* tq, const CUtensorMap* tk, const CUtensorMap* tv, const AttendArgs& a,
                      cudaStream_t s) {
  const int tiles = (a.N_valid + kBM - 1) / kBM;
  dim3 grid((tiles + 1) / 2, a.H, a.B);
  const float scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(a.d)));
  auto go = [&](auto kern, size_t smem, int regs_min) {
    // the register split after set-up waits forever unless the launch holds enough registers
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if (fa.numRegs < regs_min) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, s>>>(*tq, *tk, *tv, a, scale_log2);
    return cudaGetLastError();
  };
  if (a.d == 128) return go(attend_pp_kernel<128, FUSED>, PPLayout<128>::bytes(a.nB), regs_launch_min<128>());
  return go(attend_pp_kernel<64, FUSED>, PPLayout<64>::bytes(a.nB), regs_launch_min<64>());
}

int sm_count() {
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

cudaError_t launch_attend_pp_bf16(const CUtensorMap* tq, const CUtensorMap* tk, const CUtensorMap* tv,
                                  const AttendArgs& a, cudaStream_t s) {
  if (!attend_pp_supported(a)) return cudaErrorInvalidValue;
  return launch_pp<false>(tq, tk, tv, a, s);
}

size_t score_attend_pp_workspace_bytes(int N_valid, int* n_slots, size_t* flag_bytes) {
  // one CTA per SM holds TMEM at a time, and a CTA takes its slot while it holds TMEM
  const int slots = sm_count();
  if (n_slots) *n_slots = slots;
  const size_t flags = (static_cast<size_t>(slots) * sizeof(int32_t) + 255) / 256 * 256;   // slot flags first
  if (flag_bytes) *flag_bytes = flags;
  const size_t n_chunks = (N_valid + 63) / 64;
  return flags + static_cast<size_t>(slots) * 2 * kBM * n_chunks * sizeof(float);
}

cudaError_t launch_score_attend_pp_bf16(const CUtensorMap* tq, const CUtensorMap* tk, const CUtensorMap* tv,
                                        const AttendArgs& a, cudaStream_t s) {
  if (a.masks != nullptr || a.nB > kMaxBlocks || a.n_slots < 1 || !a.slots || !a.fscratch || !a.scores ||
      !(a.d == 64 || a.d == 128) || !(a.block == 64 || a.block == 128))
    return cudaErrorInvalidValue;
  return launch_pp<true>(tq, tk, tv, a, s);
}

}  // namespace lbsa
