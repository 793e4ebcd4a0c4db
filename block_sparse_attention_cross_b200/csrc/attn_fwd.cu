// attn_fwd.cu -- persistent block-sparse flash-attention forward for sm_100a.
//
// CalibAtt (arXiv 2603.05503, paper page, Abstract and Figure 5(b) top): the
// kept blocks of the calibrated mask are computed densely and the others are
// skipped.  Each query tile (128 rows of one batch/head) walks its compiled
// kept-block list; only the kept K/V tiles are loaded (TMA) and multiplied
// (tcgen05), so a skipped block costs neither bytes nor FLOPs.
//
// Two kernels, both templated on the head dim D (128 or 64) and the
// key-block size BK (64, 80, 96, 128 or 144; query blocks are always 128
// rows; the paper page's Table S6 compares these key-block sizes):
//   k_attn_fwd_pp  two query tiles per CTA, one thread per query row (see
//                  the section that defines it); used wherever its two tiles'
//                  scores and accumulators fit in TMEM: every shape but
//                  D = 128 with 144-key blocks.
//   k_attn_fwd     one query tile per CTA, each block's keys split between
//                  two warps of the same rows (described here); used for
//                  D = 128 with 144-key blocks.
// The text below describes k_attn_fwd at BK = 128.  In general its two
// softmax halves take W0 = BK / 2 rounded up to a multiple of 16 key columns
// and BK - W0 (80 = 48 + 32, 144 = 80 + 64), so that each half's
// probabilities feed whole PV K steps of 16 keys; score buffers are 128 TMEM
// columns apart (160 for BK = 144) and O follows them.
//
// Persistent CTA (one per SM, one query tile at a time), 12 warps:
//   warps 0-3   softmax, key columns 0-63 of each block (warp w: rows 32w..32w+31)
//   warps 4-7   softmax, key columns 64-127 of the same rows
//   warp 8      TMA producer: the Q tile, then K and V tiles of the kept blocks
//               into one shared ring, in exactly the order the MMA warp uses them
//   warp 9      TMEM allocator and MMA issuer
//   warps 10-11 idle (they complete the control warpgroup)
// The block is launched with 168 registers per thread; inside its own branch
// the control warpgroup (two walk cursors per role) lowers its limit to 120
// and the softmax warpgroups raise theirs to 192 (a 64-column half row of
// scores in registers): 2 * 128 * 192 + 128 * 120 = 384 * 168.
//
// TMEM (512 columns): two score buffers S0 = [0, 128) and S1 = [128, 256) and
// the O accumulator [256, 256 + d).  Block g of the CTA's walk uses buffer
// g % 2.  The softmax half h overwrites the first 32 columns of its own 64
// score columns with its probabilities as bf16 pairs, so P of one block sits
// at columns [0, 32) and [64, 96) of its buffer: the A operand of the PV MMA
// (tcgen05.mma with A in TMEM), issued as two K = 64 groups.
// MMA issue order: S(0), S(1), then PV(g), S(g + 2) for g = 0, 1, ...: the
// tensor core computes the scores of block g + 1 and PV of block g - 1 while
// the softmax works on block g, and S(g + 2) may overwrite P(g) because the
// in-order tensor pipe has consumed it.
//
// Softmax: exp2 of the scaled scores against a reference max m shared by the
// two halves of a row.  The first block of a tile takes the exact row max
// (the halves exchange their maxima through shared memory); later blocks are
// exponentiated against the current m while their max is found, and the
// halves exchange their block maxima after their stores are in flight.  Only
// when a row's block max exceeds m by more than kRescaleThreshold is the
// block redone with the raised m and O rescaled (after the previous PV has
// completed).  Each tile walks its list from the first kept block at or after
// its own (diagonal) block, wrapping around, so the first block usually holds
// the row max.  The epilogue moves the bf16 rounding error of each half's
// largest probability into the normaliser (see the epilogue).
// Query rows (N, Np) and key rows (Nk, Npk) may differ: gathered anchor
// queries attend to the whole sequence.
// Every wait is bounded; on expiry the CTA reports CALIBATT_E_TIMEOUT, drains
// its own copies and MMAs, frees TMEM and exits.
#include <atomic>
#include <cmath>
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace calibatt {
namespace {

constexpr int TILE = 128;
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;
constexpr uint32_t kSoftmaxRegs = 192;
constexpr uint32_t kControlRegs = 120;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kControlRegs == kThreads * kLaunchRegs, "register split");
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint32_t kTmemCols = 512;
// The reference max is raised (and O rescaled) only when a block's row max
// exceeds it by more than this many log2 units, so every P <= 2^64; row sums
// and O stay far below the fp32 range for |v| < 2^47.
constexpr float kRescaleThreshold = 64.0f;

// D: head dim; BK: key-block size (64, 80, 96, 128 or 144; query blocks are always 128).
template <int D, int BK>
struct FwdLayout {
  static constexpr uint32_t QBOX_BYTES = TILE * 64 * 2;  // 128 rows x 64 bf16 (one 128-byte swizzle span)
  static constexpr uint32_t KBOX_BYTES = BK * 64 * 2;    // BK rows x 64 bf16
  static constexpr uint32_t Q_BYTES = TILE * D * 2;
  static constexpr uint32_t KV_BYTES = BK * D * 2;
  static constexpr int RING = 163840 / KV_BYTES;               // 160 KB of K/V tiles
  // Key columns of the two softmax halves: the first a multiple of 16 (one
  // PV K step), the second the rest; and the TMEM stride of a score buffer.
  static constexpr int W0 = (BK / 2 + 15) / 16 * 16;
  static constexpr int W1 = BK - W0;
  static constexpr uint32_t SB = BK <= 128 ? 128 : (BK + 31) / 32 * 32;
  static_assert(W1 >= 32 && W1 % 16 == 0 && 2 * SB + 128 <= 512, "key-block size");
  static_assert(KV_BYTES % 1024 == 0 && KBOX_BYTES % 1024 == 0, "128-byte swizzle needs 1 KB aligned tiles");
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_RING = Q_BYTES;
  static constexpr uint32_t OFF_XCHG = OFF_RING + RING * KV_BYTES;   // float2 [2 slots][2 halves][128 rows]
  static constexpr uint32_t XCHG_BYTES = 2 * 2 * 128 * 8;
  static constexpr uint32_t OFF_CTRL = OFF_XCHG + XCHG_BYTES;
  static constexpr uint32_t CTRL_BYTES = 1024;
  static constexpr uint32_t SMEM_BYTES = OFF_CTRL + CTRL_BYTES + 1024;  // + alignment slack
};

template <int RING>
struct FwdCtrl {
  uint64_t ring_full[RING], ring_empty[RING];
  uint64_t q_full, q_empty;
  uint64_t s_full[2], p_full[2];
  uint64_t pv_done;
  uint64_t o_full, o_free;
  uint64_t xchg[4];   // per row quarter: the two softmax warps of those rows
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

template <int V>
using IntC = std::integral_constant<int, V>;


__device__ __forceinline__ float u2f(uint32_t x) { return __uint_as_float(x); }
__device__ __forceinline__ uint32_t f2u(float x) { return __float_as_uint(x); }

struct TileList {
  int bh, h, qb;
  int n;      // kept blocks (0 for an empty or rejected list)
  int base;   // first kept block
  int p0;     // start of the pattern in pat_off
  int rot;    // blocks are walked from list index rot (first kept block >= qb), wrapping around
};

// Reads and checks the kept-block list of work tile t.  Warp-collective: every
// lane returns the same result, and every role evaluates the same data, so
// all roles agree on n.
__device__ __forceinline__ TileList tile_list(const TcArgs& a, int t, bool report) {
  TileList tl;
  tl.bh = t / a.nqb;
  tl.qb = t - tl.bh * a.nqb;
  tl.h = tl.bh % a.H;
  const long long r = static_cast<long long>(a.map_offset + tl.h) * a.nqb + tl.qb;
  tl.base = a.row_base[r];
  const int pat = a.row_pat[r];
  bool bad = false;
  int p0 = 0, p1 = 0;
  if (pat < 0 || pat >= a.n_pat) {
    bad = true;
  } else {
    p0 = a.pat_ptr[pat];
    p1 = a.pat_ptr[pat + 1];
    if (p0 < 0 || p1 < p0 || p1 > a.nnz_pat || p1 - p0 > a.nkb) bad = true;
  }
  const int n = bad ? 0 : p1 - p0;
  const int lane = threadIdx.x & 31;
  for (int i = lane; i < n; i += 32) {
    const int off = a.pat_off[p0 + i];
    const int kb = tl.base + off;
    bool ok = kb >= 0 && kb < a.nkb;
    if (i > 0) ok = ok && off > a.pat_off[p0 + i - 1];
    bad |= !ok;
  }
  bad = __any_sync(0xffffffffu, bad);
  if (bad && report && lane == 0) report_status(a.status, CALIBATT_E_CORRUPT);
  tl.n = bad ? 0 : n;
  tl.p0 = p0;
  // Walk order: start at the query tile's own (diagonal) block -- the key
  // block holding its first token -- or the first kept block after it, and
  // wrap around.  For video attention the query's own block usually holds
  // the row maximum, so later blocks rarely raise it.
  const int kb_diag = tl.qb * TILE / a.block_k;
  int below = 0;
  for (int i0 = 0; i0 < tl.n; i0 += 32) {
    const int i = i0 + lane;
    below += __popc(__ballot_sync(0xffffffffu, i < tl.n && tl.base + a.pat_off[p0 + i] < kb_diag));
  }
  tl.rot = (below < tl.n) ? below : 0;
  return tl;
}

// Walk over the kept blocks of this CTA's non-empty work tiles c, c + G,
// c + 2G, ... (G = gridDim.x), shared by the producer and the MMA warp.
struct Cursor {
  int t, n, base, p0, bh, qb, rot, j;
  bool done;
};

__device__ __forceinline__ void cursor_seek(const TcArgs& a, Cursor& cu, int T, int G) {
  while (cu.t < T) {
    const TileList tl = tile_list(a, cu.t, false);
    if (tl.n > 0) {
      cu.n = tl.n;
      cu.base = tl.base;
      cu.p0 = tl.p0;
      cu.bh = tl.bh;
      cu.qb = tl.qb;
      cu.rot = tl.rot;
      cu.j = 0;
      return;
    }
    cu.t += G;
  }
  cu.done = true;
}

__device__ __forceinline__ void cursor_init(const TcArgs& a, Cursor& cu, int T, int G) {
  cu.t = blockIdx.x;
  cu.done = false;
  cursor_seek(a, cu, T, G);
}

__device__ __forceinline__ void cursor_next(const TcArgs& a, Cursor& cu, int T, int G) {
  if (++cu.j == cu.n) {
    cu.t += G;
    cursor_seek(a, cu, T, G);
  }
}

__device__ __forceinline__ int cursor_kb(const TcArgs& a, const Cursor& cu) {
  return cu.base + a.pat_off[cu.p0 + (cu.j + cu.rot) % cu.n];
}

// The score stream (S, K tiles) runs up to two blocks ahead of the PV stream
// (PV, V tiles): S(gs) reuses the buffer of block gs - 2, whose PV must have
// been issued.  Producer and MMA warp take the same decision from their own
// counters, so the ring is filled in exactly the order it is consumed.
__device__ __forceinline__ bool take_score(const Cursor& cs, uint32_t gs, uint32_t gp) {
  return !cs.done && gs <= gp + 1;
}

template <int D, int BK>
__global__ void __launch_bounds__(kThreads, 1)
    k_attn_fwd(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const TcArgs a) {
  using L = FwdLayout<D, BK>;
  constexpr int R = L::RING;
  constexpr int W0 = L::W0;    // key columns of softmax half 0 (half 1: BK - W0)
  constexpr uint32_t SB = L::SB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  FwdCtrl<R>* c = reinterpret_cast<FwdCtrl<R>*>(smem + L::OFF_CTRL);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int G = gridDim.x;
  const int T = a.B * a.H * a.nqb;

  if (tid == 0) {
    for (int e = 0; e < R; ++e) {
      mbar_init(&c->ring_full[e], 1);
      mbar_init(&c->ring_empty[e], 1);
    }
    mbar_init(&c->q_full, 1);
    mbar_init(&c->q_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&c->s_full[b], 1);
      mbar_init(&c->p_full[b], 256);
    }
    mbar_init(&c->pv_done, 1);
    mbar_init(&c->o_full, 1);
    mbar_init(&c->o_free, 256);
    for (int w = 0; w < 4; ++w) mbar_init(&c->xchg[w], 64);
    mbar_init(&c->drain, 1);
    c->abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&c->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = c->tmem_base;

  if (warp >= 8) regs_dec<kControlRegs>();
  if (warp == kProducerWarp) {
    // ===================== TMA producer =======================================
    Cursor cs, cp;
    cursor_init(a, cs, T, G);
    cursor_init(a, cp, T, G);
    uint32_t g = 0, gs = 0, gp = 0;   // ring fills, K tiles, V tiles issued
    int qfills = 0;
    bool ok = true;
    const uint64_t pol = l2_policy_evict_last();
    const uint64_t pol_q = l2_policy_evict_first();
    while (ok && !(cs.done && cp.done)) {
      const bool score = take_score(cs, gs, gp);
      if (score && cs.j == 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(&c->q_empty, (qfills & 1) ^ 1, &c->abort, a.spin_ns));
        if (!ok) break;
        mbar_arrive_expect_tx_w(&c->q_full, L::Q_BYTES);
#pragma unroll
        for (int x = 0; x < D / 64; ++x)
          tma_load_2d_w(smem + L::OFF_Q + x * L::QBOX_BYTES, &tmQ, x * 64, cs.bh * a.Np + cs.qb * TILE, &c->q_full,
                        pol_q);
        ++qfills;
      }
      const int row = score ? cs.bh * a.Npk + cursor_kb(a, cs) * BK : cp.bh * a.Npk + cursor_kb(a, cp) * BK;
      const int e = g % R;
      ok = __all_sync(0xffffffffu, mbar_wait(&c->ring_empty[e], ((g / R) & 1) ^ 1, &c->abort, a.spin_ns));
      if (!ok) break;
      mbar_arrive_expect_tx_w(&c->ring_full[e], L::KV_BYTES);
      const CUtensorMap* tm = score ? &tmK : &tmV;
#pragma unroll
      for (int x = 0; x < D / 64; ++x)
        tma_load_2d_w(smem + L::OFF_RING + e * L::KV_BYTES + x * L::KBOX_BYTES, tm, x * 64, row, &c->ring_full[e],
                      pol);
      ++g;
      if (score) {
        ++gs;
        cursor_next(a, cs, T, G);
      } else {
        ++gp;
        cursor_next(a, cp, T, G);
      }
    }
    if (lane == 0) {
      if (!ok) {
        c->abort = 1;
        report_status(a.status, CALIBATT_E_TIMEOUT);
      }
      // Drain: every copy issued must have landed before the CTA may exit.
      for (int e = 0; e < R; ++e) {
        const uint32_t fills = (g > static_cast<uint32_t>(e)) ? (g - 1 - e) / R + 1 : 0;
        if (fills > 0) mbar_wait(&c->ring_full[e], (fills - 1) & 1, nullptr, a.spin_ns);
      }
      if (qfills > 0) mbar_wait(&c->q_full, (qfills - 1) & 1, nullptr, a.spin_ns);
    }
  } else if (warp == kMmaWarp) {
    // ===================== MMA issuer =========================================
    Cursor cs, cp;
    cursor_init(a, cs, T, G);
    cursor_init(a, cp, T, G);
    constexpr uint32_t IDESC_S = idesc_bf16_f32(TILE, BK, false);
    constexpr uint32_t IDESC_O = idesc_bf16_f32(TILE, D, true);
    const uint32_t sQ = smem_u32(smem + L::OFF_Q);
    const uint32_t sRing = smem_u32(smem + L::OFF_RING);
    const uint32_t tO = tmem + 2 * SB;
    uint32_t g = 0, gs = 0, gp = 0;
    int qtiles = 0;   // tiles whose first S was issued
    int otiles = 0;   // tiles whose first PV was issued
    bool ok = true;
    while (ok && !(cs.done && cp.done)) {
      const int e = g % R;
      if (take_score(cs, gs, gp)) {
        const uint32_t tS = tmem + (gs & 1) * SB;
        ok = (cs.j > 0 || mbar_wait(&c->q_full, qtiles & 1, &c->abort, a.spin_ns)) &&
             mbar_wait(&c->ring_full[e], (g / R) & 1, &c->abort, a.spin_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const uint32_t sK = sRing + e * L::KV_BYTES;
        if (D == 128 && BK == TILE) {
          mma_ss_k128_w(tS, sdesc_sw128(sQ, 16, 1024), sdesc_sw128(sK, 16, 1024), IDESC_S, L::QBOX_BYTES >> 4);
        } else {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t ad = sdesc_sw128(sQ + (kk >> 2) * L::QBOX_BYTES + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(sK + (kk >> 2) * L::KBOX_BYTES + (kk & 3) * 32, 16, 1024);
            mma_bf16_ss_w(tS, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
          }
        }
        mma_commit_w(&c->s_full[gs & 1]);
        mma_commit_w(&c->ring_empty[e]);
        if (cs.j == 0) ++qtiles;
        if (cs.j == cs.n - 1) mma_commit_w(&c->q_empty);
        ++gs;
        cursor_next(a, cs, T, G);
      } else {
        const uint32_t tP = tmem + (gp & 1) * SB;
        ok = mbar_wait(&c->p_full[gp & 1], (gp >> 1) & 1, &c->abort, a.spin_ns) &&
             mbar_wait(&c->ring_full[e], (g / R) & 1, &c->abort, a.spin_ns) &&
             (cp.j > 0 || mbar_wait(&c->o_free, (otiles & 1) ^ 1, &c->abort, a.spin_ns));
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const uint64_t vd = sdesc_sw128(sRing + e * L::KV_BYTES, L::KBOX_BYTES, 1024);
        if (BK == TILE) {
          // keys 0-63 (P columns [0, 32)), then keys 64-127 (P columns [64, 96))
          mma_ts_k64_w(tO, tP, vd, IDESC_O, cp.j > 0 ? 1u : 0u);
          mma_ts_k64_w(tO, tP + 64, vd + 512, IDESC_O, 1u);
        } else {
          // 16 keys (8 P columns, 16 V rows = 2048 bytes) per step; the P of
          // half 0 starts at column 0, that of half 1 at its first score
          // column W0
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const int acol = kk < W0 / 16 ? kk * 8 : W0 + (kk - W0 / 16) * 8;
            mma_bf16_ts_w(tO, tP + acol, vd + kk * 128, IDESC_O, (cp.j > 0 || kk > 0) ? 1u : 0u);
          }
        }
        mma_commit_w(&c->ring_empty[e]);
        mma_commit_w(&c->pv_done);
        if (cp.j == 0) ++otiles;
        if (cp.j == cp.n - 1) mma_commit_w(&c->o_full);
        ++gp;
        cursor_next(a, cp, T, G);
      }
      ++g;
    }
    if (!ok && lane == 0) {
      c->abort = 1;
      report_status(a.status, CALIBATT_E_TIMEOUT);
    }
    __syncwarp();
    mma_commit_w(&c->drain);
    mbar_wait(&c->drain, 0, nullptr, a.spin_ns);
  } else if (warp < 8) {
    // ===================== softmax warpgroups =================================
    regs_inc<kSoftmaxRegs>();
    // One softmax half: HB key columns starting at column c0 of every block
    // (one instantiation serves both halves when they are equal).
    auto softmax = [&](auto hb_c) {
    constexpr int HB = decltype(hb_c)::value;
    const int h = warp >> 2;                  // key-column half of every block
    const int c0 = h * W0;
    const int w = warp & 3;                   // TMEM lane quarter
    const int row = w * 32 + lane;
    const uint32_t t_row = tmem + (static_cast<uint32_t>(w * 32) << 16);
    const float c2 = a.scale_log2;
    float2* xbuf = reinterpret_cast<float2*>(smem + L::OFF_XCHG);
    uint32_t xc = 0;   // exchanges with the partner warp (same rows, other half)
    uint32_t gb = 0;   // blocks of non-empty tiles consumed by this CTA
    int tiles = 0;     // non-empty tiles finished
    bool ok = true;
    // Posts this thread's value for its row, then (finish) waits for the
    // partner's; the two steps may be split to overlap other work.
    auto xpost = [&](float2 v) {
      xbuf[((xc & 1) * 2 + h) * 128 + row] = v;
      mbar_arrive(&c->xchg[w]);
    };
    auto xfinish = [&]() -> float2 {
      const bool got = mbar_wait(&c->xchg[w], xc & 1, &c->abort, a.spin_ns);
      ok = __all_sync(0xffffffffu, got) && ok;
      const float2 v = xbuf[((xc & 1) * 2 + (h ^ 1)) * 128 + row];
      ++xc;
      return v;
    };
    for (int t = blockIdx.x; ok && t < T; t += G) {
      const TileList tl = tile_list(a, t, true);
      const int grow = tl.qb * TILE + row;
      const size_t orow_idx = static_cast<size_t>(tl.bh) * a.Np + grow;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.o) + orow_idx * D + h * (D / 2);
      if (tl.n == 0) {
        uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int i = 0; i < D / 16; ++i) reinterpret_cast<uint4*>(orow)[i] = z;
        if (a.lse != nullptr && h == 0) a.lse[orow_idx] = -INFINITY;
        continue;
      }
      const int kb_last = tl.base + a.pat_off[tl.p0 + tl.n - 1];
      const int valid_last = (kb_last == a.nkb - 1) ? (a.Nk - kb_last * BK) : BK;
      const int j_last = (tl.n - 1 - tl.rot + tl.n) % tl.n;   // walk position of the highest kept block
      float m = -INFINITY;
      float l = 0.f;
      // Largest raw score of this half-row so far (for the normalisation
      // fix-up in the epilogue).
      float s_best = -INFINITY;
      for (int j = 0; j < tl.n; ++j, ++gb) {
        const uint32_t b = gb & 1;
        const bool got = mbar_wait(&c->s_full[b], (gb >> 1) & 1, &c->abort, a.spin_ns);
        ok = __all_sync(0xffffffffu, got);
        if (!ok) break;
        tc_fence_after();
        const uint32_t t_s = t_row + b * SB + c0;   // this half's HB score columns
        uint32_t r[HB];
#pragma unroll
        for (int q4 = 0; q4 < HB / 32; ++q4)
          tmem_ld32(t_s + q4 * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[q4 * 32]));
        if constexpr (HB % 32 == 16) tmem_ld16(t_s + HB / 32 * 32, *reinterpret_cast<uint32_t(*)[16]>(&r[HB / 32 * 32]));
        tmem_ld_wait();
        reg_fence(r);
        if (j == j_last && valid_last < BK) {
          // Key columns past the sequence end exist only in the last block.
#pragma unroll
          for (int i = 0; i < HB; ++i)
            if (c0 + i >= valid_last) r[i] = f2u(-INFINITY);
        }
        // p = 2^(s c2 - mref) two columns at a time on the MUFU unit, as
        // bf16 pairs into the first 32 columns of this half's score columns,
        // 16 columns (32 probabilities) per store.  Returns the half-row sum;
        // with `track` it also returns the half-row maximum of the raw scores.
        const uint64_t c2x2 = f2pack(c2, c2);
        auto emit_p = [&](float mref, bool track, float& mx_out) -> float {
          const uint64_t negm = f2pack(-mref, -mref);
          uint64_t acc0 = f2pack(0.f, 0.f), acc1 = acc0;
          float mxa = -INFINITY, mxb = -INFINITY;
          // NP pairs of columns from column e0: bf16 pairs stored from P column e0 / 2
          auto chunk = [&](auto np_c, int e0, uint32_t (&pk)[decltype(np_c)::value]) {
            constexpr int NP = decltype(np_c)::value;
#pragma unroll
            for (int i = 0; i < NP; ++i) {
              const int e = e0 + 2 * i;
              if (track) {
                if (i & 1) mxb = fmax3(mxb, u2f(r[e]), u2f(r[e + 1]));
                else mxa = fmax3(mxa, u2f(r[e]), u2f(r[e + 1]));
              }
              const uint64_t x = ffma2(f2pack(u2f(r[e]), u2f(r[e + 1])), c2x2, negm);
              float xl, xh;
              f2unpack(x, xl, xh);
              const uint64_t pv = f2pack(ex2_approx(xl), ex2_approx(xh));
              if (i & 1) acc1 = fadd2(acc1, pv); else acc0 = fadd2(acc0, pv);
              float pl, ph;
              f2unpack(pv, pl, ph);
              pk[i] = pack_bf16x2(pl, ph);
            }
          };
#pragma unroll
          for (int c16 = 0; c16 < HB / 32; ++c16) {
            uint32_t pk[16];
            chunk(IntC<16>{}, c16 * 32, pk);
            tmem_st16(t_s + c16 * 16, pk);
          }
          if constexpr (HB % 32 == 16) {
            uint32_t pk[8];
            chunk(IntC<8>{}, HB / 32 * 32, pk);
            tmem_st8(t_s + HB / 32 * 16, pk);
          }
          mx_out = fmaxf(mxa, mxb);
          float a0, a1, b0, b1;
          f2unpack(acc0, a0, a1);
          f2unpack(acc1, b0, b1);
          return (a0 + a1) + (b0 + b1);
        };
        float alpha = 1.f;
        float rs;
        if (j == 0) {
          // First block of the tile: the exact row maximum (both halves) sets
          // the reference.
          float mx0 = u2f(r[0]), mx1 = u2f(r[1]), mx2 = u2f(r[2]), mx3 = u2f(r[3]);
#pragma unroll
          for (int i = 4; i + 8 <= HB; i += 8) {
            mx0 = fmax3(mx0, u2f(r[i + 0]), u2f(r[i + 1]));
            mx1 = fmax3(mx1, u2f(r[i + 2]), u2f(r[i + 3]));
            mx2 = fmax3(mx2, u2f(r[i + 4]), u2f(r[i + 5]));
            mx3 = fmax3(mx3, u2f(r[i + 6]), u2f(r[i + 7]));
          }
          static_assert(HB % 8 == 0, "the loop above leaves exactly the last 4 columns");
          mx0 = fmax3(mx0, u2f(r[HB - 4]), u2f(r[HB - 3]));
          mx1 = fmax3(mx1, u2f(r[HB - 2]), u2f(r[HB - 1]));
          s_best = fmax3(mx0, mx1, fmaxf(mx2, mx3));
          xpost(make_float2(s_best, 0.f));
          const float2 other = xfinish();
          m = fmaxf(s_best, other.x) * c2;
          float unused;
          rs = emit_p(m, false, unused);
        } else {
          // Later blocks: exponentiate against the current reference while
          // finding the block maximum; the halves exchange their maxima while
          // the stores are in flight.  Only if a row's maximum exceeds the
          // reference by more than the threshold (rare) is the block redone
          // with the raised reference and O rescaled.
          float mx;
          rs = emit_p(m, true, mx);
          xpost(make_float2(mx, 0.f));
          s_best = fmaxf(s_best, mx);
          const float m_cand = fmaxf(mx, xfinish().x) * c2;
          const bool raise = m_cand > m + kRescaleThreshold;
          if (__any_sync(0xffffffffu, raise)) {
            // O must hold PV of every earlier block of the tile: wait for the
            // previous block's PV (the commit that signalled S(j) covers the
            // ones before it).
            const bool pv = mbar_wait(&c->pv_done, (gb - 1) & 1, &c->abort, a.spin_ns);
            ok = __all_sync(0xffffffffu, pv) && ok;
            tc_fence_after();
            if (raise) {
              alpha = ex2_approx(m - m_cand);
              m = m_cand;
            }
            tmem_st_wait();   // the speculative P stores land before they are overwritten
            float unused;
            rs = emit_p(m, false, unused);
#pragma unroll
            for (int q4 = 0; q4 < D / 64; ++q4) {
              uint32_t ro[32];
              const uint32_t t_o = t_row + 2 * SB + h * (D / 2) + q4 * 32;
              tmem_ld32(t_o, ro);
              tmem_ld_wait();
              reg_fence(ro);
#pragma unroll
              for (int i = 0; i < 32; ++i) ro[i] = f2u(u2f(ro[i]) * alpha);
              tmem_st32(t_o, ro);
            }
          }
        }
        l = l * alpha + rs;
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&c->p_full[b]);
        if (!ok) break;
      }
      if (!ok) break;
      // ---- epilogue: O / l, LSE -------------------------------------------
      // O holds sums of bf16-rounded probabilities while l sums the fp32 ones.
      // Their mismatch is negligible except for a dominant probability, which
      // is not exactly representable once the reference lags the row maximum
      // (threshold above): the rounding error of each half's largest
      // probability, re-formed here exactly as the softmax formed it, is moved
      // into the normaliser, so that a row with one dominant key returns that
      // key's value.  The largest score was always exponentiated against the
      // final reference m: a raise after its block would need a larger score,
      // and a raise in its block redoes the block against a reference at or
      // above it.  The LSE keeps the fp32 sum.
      const float p_best = ex2_approx(fmaf(s_best, c2, -m));
      const float corr = __uint_as_float(pack_bf16x2(p_best, 0.f) << 16) - p_best;
      xpost(make_float2(l, corr));
      const float2 other = xfinish();
      const float l_row = l + other.x;
      const float l_o = l_row + (corr + other.y);
      const bool got = mbar_wait(&c->o_full, tiles & 1, &c->abort, a.spin_ns);
      ok = __all_sync(0xffffffffu, got) && ok;
      if (!ok) break;
      ++tiles;
      tc_fence_after();
      const bool pad_row = grow >= a.N;
      const float inv_l = pad_row ? 0.f : 1.f / l_o;
#pragma unroll
      for (int q4 = 0; q4 < D / 64; ++q4) {
        uint32_t r[32];
        tmem_ld32(t_row + 2 * SB + h * (D / 2) + q4 * 32, r);
        tmem_ld_wait();
        reg_fence(r);
        uint4* dst = reinterpret_cast<uint4*>(orow + q4 * 32);
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          uint4 pk;
          pk.x = pack_bf16x2(u2f(r[8 * v4 + 0]) * inv_l, u2f(r[8 * v4 + 1]) * inv_l);
          pk.y = pack_bf16x2(u2f(r[8 * v4 + 2]) * inv_l, u2f(r[8 * v4 + 3]) * inv_l);
          pk.z = pack_bf16x2(u2f(r[8 * v4 + 4]) * inv_l, u2f(r[8 * v4 + 5]) * inv_l);
          pk.w = pack_bf16x2(u2f(r[8 * v4 + 6]) * inv_l, u2f(r[8 * v4 + 7]) * inv_l);
          dst[v4] = pk;
        }
      }
      tc_fence_before();
      mbar_arrive(&c->o_free);
      if (a.lse != nullptr && h == 0)
        a.lse[orow_idx] = pad_row ? -INFINITY : (m + log2f(l_row)) * 0.69314718055994531f;
    }
    if (!ok) {
      c->abort = 1;
      report_status(a.status, CALIBATT_E_TIMEOUT);
    }
    };
    if constexpr (2 * W0 == BK) softmax(IntC<W0>{});
    else if ((warp >> 2) == 0) softmax(IntC<W0>{});
    else softmax(IntC<BK - W0>{});
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

// ===========================================================================
// Two query tiles per CTA ("slots" 0 and 1), one thread per query row.
//
// Each slot has its own softmax warpgroup (warps 0-3: slot 0, warps 4-7:
// slot 1; warp w's rows are TMEM lanes 32 (w % 4) ...), its own Q buffer,
// score buffer S_s, accumulator O_s, TMA producer (warps 8 and 11) and K/V
// ring; warp 9 issues every MMA, warp 10 is idle.  A thread holds its row's
// whole block of scores in registers, so the row maximum needs no exchange
// between warps: the block maximum is taken first and the exponentials use
// the reference that follows from it.  The two warps that share an SM
// sub-partition belong to different slots; the tensor core alternates
// between the slots (PV_0, S_0, PV_1, S_1, ...), so while one slot's scores
// are being computed the other slot's warps exponentiate, and one slot's
// TMEM loads, stores and waits overlap the other slot's exponentials.
//
// TMEM (512 columns): slot s owns [256 s, 256 s + 256): S_s at
// [256 s, 256 s + SK) and O_s at [256 s + OC, 256 s + OC + D), where a step
// holds SK keys (128 for BK = 64, 96, 128; the block for 80 and 144) and
// OC = 128 (160 for SK = 144).  P overwrites the first SK / 2 columns of S_s
// as bf16 pairs: the A operand of the PV MMA.  With one score buffer per slot
// the order per slot is S(j), softmax(j), PV(j), S(j + 1): S(j + 1) may
// overwrite P(j) because the in-order tensor pipe has consumed it, and the
// commit that signals S(j + 1) also covers PV(j), so O_s can be rescaled as
// soon as the scores of step j + 1 are visible.
// ===========================================================================

constexpr int cgcd(int x, int y) { return y == 0 ? x : cgcd(y, x % y); }

template <int D, int BK>
struct PpLayout {
  static constexpr uint32_t QBOX_BYTES = TILE * 64 * 2;
  static constexpr uint32_t KBOX_BYTES = BK * 64 * 2;
  static constexpr uint32_t Q_BYTES = TILE * D * 2;
  // Steps of 128 keys where gcd(BK, 128) >= 32 (BK = 64, 96, 128): the keys
  // come in pieces of PK = gcd(BK, 128), taken in walk order from the kept
  // blocks (a block is BK / PK pieces, a step 128 / PK: one block at 128, two
  // at 64, parts of two at 96), one TMA box per piece and 64 columns; the last
  // step of a tile repeats its last real piece where the walk has ended, and
  // the softmax masks those columns.  So each step pays its fixed costs once
  // per 128 keys.  With 16-key pieces (BK = 80, 144) the many small copies
  // cost more than they save (measured: -8% and -12%), so there a step is one
  // block.
  static constexpr int PG = cgcd(BK, TILE);
  static constexpr bool PACK = PG >= 32;
  static constexpr int PK = PACK ? PG : BK;               // keys per piece
  static constexpr int SK = PACK ? TILE : BK;             // keys per step
  static constexpr int PPB = BK / PK;                     // pieces per key block
  static constexpr int PPS = SK / PK;                     // pieces per step
  static constexpr uint32_t PBOX_BYTES = PK * 64 * 2;     // one 64-column box of a piece (one TMA copy)
  static constexpr uint32_t SBOX_BYTES = SK * 64 * 2;     // one 64-column box of a step's K or V tile
  static constexpr uint32_t STEP_BYTES = SK * D * 2;      // a step's K (or V) tile
  static constexpr uint32_t OC = SK <= 128 ? 128 : 160;   // O_s column offset inside the slot
  static_assert(BK % 16 == 0 && BK >= 64 && OC + D <= 256 && SK <= OC, "key-block size / head dim");
  static_assert(PBOX_BYTES % 1024 == 0 && STEP_BYTES % 1024 == 0, "128-byte swizzle needs 1 KB aligned boxes");
  static constexpr uint32_t OFF_Q = 0;   // Q tiles of slots 0 and 1
  static constexpr uint32_t OFF_RING = 2 * Q_BYTES;
  static constexpr uint32_t CTRL_BYTES = 1024;
  static constexpr uint32_t BUDGET = 232448 - OFF_RING - CTRL_BYTES - 1024;
  // K/V step tiles per slot ring (each slot's producer fills its own ring)
  static constexpr int RING = (BUDGET / (2 * STEP_BYTES)) > 4 ? 4 : static_cast<int>(BUDGET / (2 * STEP_BYTES));
  static_assert(RING >= 2, "ring");
  static constexpr uint32_t OFF_CTRL = OFF_RING + 2 * RING * STEP_BYTES;
  static constexpr uint32_t SMEM_BYTES = OFF_CTRL + CTRL_BYTES + 1024;  // + alignment slack
};

template <int RING>
struct PpCtrl {
  uint64_t ring_full[2][RING], ring_empty[2][RING];
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full[2], p_full[2];
  uint64_t o_full[2], o_free[2];
  uint64_t drain[2];
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void pp_cursor_init(const TcArgs& a, Cursor& cu, int slot, int T, int G) {
  cu.t = blockIdx.x + slot * G;
  cu.done = false;
  cursor_seek(a, cu, T, 2 * G);
}

constexpr int kPpProducer0 = 8, kPpMma = 9, kPpProducer1 = 11;   // warp 10 idle

// Moves a piece cursor (cu.j counts pieces, ppb per kept block) by `per`
// pieces (one step), to the next non-empty tile of the walk when the current
// one is done.
__device__ __forceinline__ void cursor_step(const TcArgs& a, Cursor& cu, int T, int stride, int per, int ppb) {
  cu.j += per;
  if (cu.j >= cu.n * ppb) {
    cu.t += stride;
    cursor_seek(a, cu, T, stride);
  }
}

// Key block at walk position j of the cursor's tile.
__device__ __forceinline__ int cursor_kb_at(const TcArgs& a, const Cursor& cu, int j) {
  return cu.base + a.pat_off[cu.p0 + (j + cu.rot) % cu.n];
}

template <int D, int BK>
__global__ void __launch_bounds__(kThreads, 1)
    k_attn_fwd_pp(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const TcArgs a) {
  using L = PpLayout<D, BK>;
  constexpr int R = L::RING;
  constexpr uint32_t OC = L::OC;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  PpCtrl<R>* c = reinterpret_cast<PpCtrl<R>*>(smem + L::OFF_CTRL);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int G = gridDim.x;
  const int T = a.B * a.H * a.nqb;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      for (int e = 0; e < R; ++e) {
        mbar_init(&c->ring_full[s][e], 1);
        mbar_init(&c->ring_empty[s][e], 1);
      }
      mbar_init(&c->q_full[s], 1);
      mbar_init(&c->q_empty[s], 1);
      mbar_init(&c->s_full[s], 1);
      mbar_init(&c->p_full[s], 128);
      mbar_init(&c->o_full[s], 1);
      mbar_init(&c->o_free[s], 128);
      mbar_init(&c->drain[s], 1);
    }
    c->abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == kPpMma) {
    tmem_alloc(&c->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = c->tmem_base;

  if (warp >= 8) regs_dec<kControlRegs>();
  if (warp == kPpProducer0 || warp == kPpProducer1) {
    // ===================== TMA producer of one slot ===========================
    // Per step of the slot's walk (128 keys in pieces from the kept blocks):
    // its K tile, then its V tile, into the slot's own ring (the order the
    // slot's MMA warp consumes them).
    const int s = warp == kPpProducer1;
    Cursor cu;
    pp_cursor_init(a, cu, s, T, G);
    uint32_t g = 0;   // ring fills
    int qf = 0;
    bool ok = true;
    const uint64_t pol = l2_policy_evict_last();
    const uint64_t pol_q = l2_policy_evict_first();
    uint8_t* ring = smem + L::OFF_RING + s * R * L::STEP_BYTES;
    while (ok && !cu.done) {
      if (cu.j == 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(&c->q_empty[s], (qf & 1) ^ 1, &c->abort, a.spin_ns));
        if (!ok) break;
        mbar_arrive_expect_tx_w(&c->q_full[s], L::Q_BYTES);
#pragma unroll
        for (int x = 0; x < D / 64; ++x)
          tma_load_2d_w(smem + L::OFF_Q + s * L::Q_BYTES + x * L::QBOX_BYTES, &tmQ, x * 64,
                        cu.bh * a.Np + cu.qb * TILE, &c->q_full[s], pol_q);
        ++qf;
      }
      // first key row of each piece of the step (past the walk's end: the last
      // real piece again, masked by the softmax)
      int prow[L::PPS];
      const int np = cu.n * L::PPB;
#pragma unroll
      for (int p = 0; p < L::PPS; ++p) {
        const int gp = min(cu.j + p, np - 1);
        prow[p] = cu.bh * a.Npk + cursor_kb_at(a, cu, gp / L::PPB) * BK + (gp % L::PPB) * L::PK;
      }
#pragma unroll 1
      for (int kv = 0; kv < 2; ++kv) {
        const int e = g % R;
        ok = __all_sync(0xffffffffu, mbar_wait(&c->ring_empty[s][e], ((g / R) & 1) ^ 1, &c->abort, a.spin_ns));
        if (!ok) break;
        mbar_arrive_expect_tx_w(&c->ring_full[s][e], L::STEP_BYTES);
        const CUtensorMap* tm = kv ? &tmV : &tmK;
#pragma unroll
        for (int x = 0; x < D / 64; ++x)
#pragma unroll
          for (int p = 0; p < L::PPS; ++p)
            tma_load_2d_w(ring + e * L::STEP_BYTES + x * L::SBOX_BYTES + p * L::PBOX_BYTES, tm, x * 64, prow[p],
                          &c->ring_full[s][e], pol);
        ++g;
      }
      cursor_step(a, cu, T, 2 * G, L::PPS, L::PPB);
    }
    if (lane == 0) {
      if (!ok) {
        c->abort = 1;
        report_status(a.status, CALIBATT_E_TIMEOUT);
      }
      // Drain: every copy issued must have landed before the CTA may exit.
      for (int e = 0; e < R; ++e) {
        const uint32_t fills = (g > static_cast<uint32_t>(e)) ? (g - 1 - e) / R + 1 : 0;
        if (fills > 0) mbar_wait(&c->ring_full[s][e], (fills - 1) & 1, nullptr, a.spin_ns);
      }
      if (qf > 0) mbar_wait(&c->q_full[s], (qf - 1) & 1, nullptr, a.spin_ns);
    }
  } else if (warp == kPpMma) {
    // ===================== MMA issuer =========================================
    // Per kept block b of a slot's walk: S(b), then (once the slot's softmax
    // has stored P(b)) PV(b) followed by S(b + 1).  The slots are served in
    // turn.  Both slots start together, but the second slot's next scores
    // queue behind the first slot's PV and S, so from the second block on the
    // slots run half a period apart: one slot exponentiates while the other
    // slot's products run, and each slot's MMA wait is another's softmax.
    // (Measured: serving the slot whose P arrives first, polling both
    // barriers, was slower; so were PV(b) and S(b + 1) issued as one burst
    // and P signalled in two key halves.)
    Cursor cu0, cu1;
    pp_cursor_init(a, cu0, 0, T, G);
    pp_cursor_init(a, cu1, 1, T, G);
    constexpr uint32_t IDESC_S = idesc_bf16_f32(TILE, L::SK, false);
    constexpr uint32_t IDESC_O = idesc_bf16_f32(TILE, D, true);
    uint32_t g0 = 0, g1 = 0;     // ring tiles consumed per slot
    uint32_t gb0 = 0, gb1 = 0;   // blocks whose PV was issued per slot
    int qt0 = 0, qt1 = 0;        // tiles whose first S was issued per slot
    int ot0 = 0, ot1 = 0;        // tiles whose first PV was issued per slot
    bool ok = true;
    // The slot is a compile-time constant in both steps, so every slot's
    // state stays in registers.
    auto issue_s = [&](auto s_c) {
      constexpr int s = decltype(s_c)::value;
      Cursor& cu = s ? cu1 : cu0;
      uint32_t& g = s ? g1 : g0;
      int& qt = s ? qt1 : qt0;
      const uint32_t sRing = smem_u32(smem + L::OFF_RING + s * R * L::STEP_BYTES);
      const uint32_t sQ = smem_u32(smem + L::OFF_Q + s * L::Q_BYTES);
      const uint32_t tS = tmem + s * 256;
      const int e = g % R;
      bool w = (cu.j > 0 || mbar_wait(&c->q_full[s], qt & 1, &c->abort, a.spin_ns)) &&
               mbar_wait(&c->ring_full[s][e], (g / R) & 1, &c->abort, a.spin_ns);
      if (!__all_sync(0xffffffffu, w)) return false;
      tc_fence_after();
      const uint32_t sK = sRing + e * L::STEP_BYTES;
      if (D == 128 && L::SK == TILE) {
        mma_ss_k128_w(tS, sdesc_sw128(sQ, 16, 1024), sdesc_sw128(sK, 16, 1024), IDESC_S, L::QBOX_BYTES >> 4);
      } else {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(sQ + (kk >> 2) * L::QBOX_BYTES + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(sK + (kk >> 2) * L::SBOX_BYTES + (kk & 3) * 32, 16, 1024);
          mma_bf16_ss_w(tS, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
        }
      }
      mma_commit_w(&c->s_full[s]);
      mma_commit_w(&c->ring_empty[s][e]);
      if (cu.j == 0) ++qt;
      if (cu.j + L::PPS >= cu.n * L::PPB) mma_commit_w(&c->q_empty[s]);
      ++g;
      return true;
    };
    // PV(b) of slot s (its P is stored), then the slot's next S.
    auto issue_pv = [&](auto s_c) {
      constexpr int s = decltype(s_c)::value;
      Cursor& cu = s ? cu1 : cu0;
      uint32_t& g = s ? g1 : g0;
      uint32_t& gb = s ? gb1 : gb0;
      int& ot = s ? ot1 : ot0;
      const uint32_t sRing = smem_u32(smem + L::OFF_RING + s * R * L::STEP_BYTES);
      const uint32_t tS = tmem + s * 256;
      const uint32_t tO = tS + OC;
      const int e = g % R;
      // P: SK / 2 columns of bf16 pairs at the start of S_s; 16 keys (8
      // columns, 16 V rows = 2048 bytes) per K step.
      const uint64_t vd = sdesc_sw128(sRing + e * L::STEP_BYTES, L::SBOX_BYTES, 1024);
      if (L::SK == TILE) {
        mma_ts_k128_w(tO, tS, vd, IDESC_O, cu.j > 0 ? 1u : 0u);
      } else {
#pragma unroll
        for (int kk = 0; kk < L::SK / 16; ++kk)
          mma_bf16_ts_w(tO, tS + kk * 8, vd + kk * 128, IDESC_O, (cu.j > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit_w(&c->ring_empty[s][e]);
      if (cu.j == 0) ++ot;
      if (cu.j + L::PPS >= cu.n * L::PPB) mma_commit_w(&c->o_full[s]);
      ++g;
      ++gb;
      cursor_step(a, cu, T, 2 * G, L::PPS, L::PPB);
      return cu.done ? true : issue_s(s_c);
    };
    bool due0 = false, due1 = false;   // an S was issued whose PV is outstanding
    if (!cu0.done) ok = due0 = issue_s(IntC<0>{});
    if (ok && !cu1.done) ok = due1 = issue_s(IntC<1>{});
    int turn = 0;
    while (ok && (due0 || due1)) {
      // the slots in turn (suspending waits)
      const int s = (due0 && (turn == 0 || !due1)) ? 0 : 1;
      // The PV's V tile and (first block of a tile) the free O are usually
      // ready long before P: wait for them first, so that only P stands
      // between the softmax's last store and the PV issue.
      {
        const Cursor& cu = s ? cu1 : cu0;
        const uint32_t g = s ? g1 : g0;
        const int ot = s ? ot1 : ot0;
        const bool w = mbar_wait(&c->ring_full[s][g % R], (g / R) & 1, &c->abort, a.spin_ns) &&
                       (cu.j > 0 || mbar_wait(&c->o_free[s], (ot & 1) ^ 1, &c->abort, a.spin_ns)) &&
                       mbar_wait(&c->p_full[s], (s ? gb1 : gb0) & 1, &c->abort, a.spin_ns);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
      }
      tc_fence_after();
      if (s == 0) {
        ok = issue_pv(IntC<0>{});
        due0 = !cu0.done;
      } else {
        ok = issue_pv(IntC<1>{});
        due1 = !cu1.done;
      }
      turn = s ^ 1;
    }
    if (!ok && lane == 0) {
      c->abort = 1;
      report_status(a.status, CALIBATT_E_TIMEOUT);
    }
    __syncwarp();
    mma_commit_w(&c->drain[0]);
    mbar_wait(&c->drain[0], 0, nullptr, a.spin_ns);
  } else if (warp < 8) {
    // ===================== softmax warpgroups =================================
    regs_inc<kSoftmaxRegs>();
    const int slot = warp >> 2;
    const int w = warp & 3;                   // TMEM lane quarter
    const int row = w * 32 + lane;
    const uint32_t t_s = tmem + (static_cast<uint32_t>(w * 32) << 16) + slot * 256;   // this row of S_slot
    const uint32_t t_o = t_s + OC;                                                      // and of O_slot
    const float c2 = a.scale_log2;
    const uint64_t c2x2 = f2pack(c2, c2);
    uint32_t gb = 0;   // blocks of non-empty tiles consumed by this slot
    int tiles = 0;     // non-empty tiles finished
    bool ok = true;
    for (int t = blockIdx.x + slot * G; ok && t < T; t += 2 * G) {
      const TileList tl = tile_list(a, t, true);
      const int grow = tl.qb * TILE + row;
      const size_t orow_idx = static_cast<size_t>(tl.bh) * a.Np + grow;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.o) + orow_idx * D;
      if (tl.n == 0) {
        uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int i = 0; i < D / 8; ++i) reinterpret_cast<uint4*>(orow)[i] = z;
        if (a.lse != nullptr) a.lse[orow_idx] = -INFINITY;
        continue;
      }
      const int kb_last = tl.base + a.pat_off[tl.p0 + tl.n - 1];
      const int valid_last = (kb_last == a.nkb - 1) ? (a.Nk - kb_last * BK) : BK;
      const int j_last = (tl.n - 1 - tl.rot + tl.n) % tl.n;   // walk position of the highest kept block
      float m = -INFINITY;
      float l = 0.f;
      float s_best = -INFINITY;   // largest raw score of the row (normalisation fix-up)
      constexpr int SK = L::SK;
      const int np = tl.n * L::PPB;   // pieces of this tile's walk
      for (int j = 0; j < np; j += L::PPS, ++gb) {
        const bool got = mbar_wait(&c->s_full[slot], gb & 1, &c->abort, a.spin_ns);
        ok = __all_sync(0xffffffffu, got);
        if (!ok) break;
        tc_fence_after();
        // The row's SK scores of this step, loaded at once.
        uint32_t r[SK];
#pragma unroll
        for (int q4 = 0; q4 < SK / 32; ++q4)
          tmem_ld32(t_s + q4 * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[q4 * 32]));
        if constexpr (SK % 32 == 16) tmem_ld16(t_s + SK / 32 * 32, *reinterpret_cast<uint32_t(*)[16]>(&r[SK / 32 * 32]));
        tmem_ld_wait();
        reg_fence(r);
        // Valid keys of each piece: key columns past the sequence end exist
        // only in the highest kept block; pieces past the walk's end (the last
        // real piece repeated) are masked entirely.
        int lim[L::PPS];
        bool partial = false;
#pragma unroll
        for (int p = 0; p < L::PPS; ++p) {
          const int gp = j + p;
          lim[p] = gp >= np ? 0
                 : gp / L::PPB == j_last ? max(0, min(L::PK, valid_last - (gp % L::PPB) * L::PK))
                                         : L::PK;
          partial |= lim[p] < L::PK;
        }
        if (partial) {
#pragma unroll
          for (int i = 0; i < SK; ++i)
            if (i % L::PK >= lim[i / L::PK]) r[i] = f2u(-INFINITY);
        }
        float mx0 = u2f(r[0]), mx1 = u2f(r[1]), mx2 = u2f(r[2]), mx3 = u2f(r[3]);
#pragma unroll
        for (int i = 4; i + 8 <= SK; i += 8) {
          mx0 = fmax3(mx0, u2f(r[i + 0]), u2f(r[i + 1]));
          mx1 = fmax3(mx1, u2f(r[i + 2]), u2f(r[i + 3]));
          mx2 = fmax3(mx2, u2f(r[i + 4]), u2f(r[i + 5]));
          mx3 = fmax3(mx3, u2f(r[i + 6]), u2f(r[i + 7]));
        }
        mx0 = fmax3(mx0, u2f(r[SK - 4]), u2f(r[SK - 3]));
        mx1 = fmax3(mx1, u2f(r[SK - 2]), u2f(r[SK - 1]));
        const float bmax = fmax3(mx0, mx1, fmaxf(mx2, mx3));
        s_best = fmaxf(s_best, bmax);
        // The reference: the exact maximum on the first block; later it is
        // raised only when the block's maximum exceeds it by more than the
        // threshold (rare), and then O and l are rescaled (after the
        // exponentials, with the scores no longer live; PV of the previous
        // block is complete: its commit preceded this block's S, and this
        // block's PV waits for the arrival below).
        float alpha = 1.f;
        bool rescale = false;
        if (j == 0) {
          m = bmax * c2;
        } else {
          const float m_cand = bmax * c2;
          const bool raise = m_cand > m + kRescaleThreshold;
          rescale = __any_sync(0xffffffffu, raise);
          if (raise) {
            alpha = ex2_approx(m - m_cand);
            m = m_cand;
          }
        }
        // p = 2^(s c2 - m) two columns at a time on the MUFU unit, stored as
        // bf16 pairs over the first SK / 2 columns of S (already read).
        const uint64_t negm = f2pack(-m, -m);
        uint64_t acc0 = f2pack(0.f, 0.f), acc1 = acc0;
        auto chunk = [&](auto np_c, int e0, uint32_t (&pk)[decltype(np_c)::value]) {
          constexpr int NP = decltype(np_c)::value;
#pragma unroll
          for (int i = 0; i < NP; ++i) {
            const int e = e0 + 2 * i;
            const uint64_t x = ffma2(f2pack(u2f(r[e]), u2f(r[e + 1])), c2x2, negm);
            float xl, xh;
            f2unpack(x, xl, xh);
            const uint64_t pv = f2pack(ex2_approx(xl), ex2_approx(xh));
            if (i & 1) acc1 = fadd2(acc1, pv); else acc0 = fadd2(acc0, pv);
            float pl, ph;
            f2unpack(pv, pl, ph);
            pk[i] = pack_bf16x2(pl, ph);
          }
        };
#pragma unroll
        for (int c16 = 0; c16 < SK / 32; ++c16) {
          uint32_t pk[16];
          chunk(IntC<16>{}, c16 * 32, pk);
          tmem_st16(t_s + c16 * 16, pk);
        }
        if constexpr (SK % 32 == 16) {
          uint32_t pk[8];
          chunk(IntC<8>{}, SK / 32 * 32, pk);
          tmem_st8(t_s + SK / 32 * 16, pk);
        }
        if (rescale) {
#pragma unroll
          for (int q4 = 0; q4 < D / 32; ++q4) {
            uint32_t ro[32];
            tmem_ld32(t_o + q4 * 32, ro);
            tmem_ld_wait();
            reg_fence(ro);
#pragma unroll
            for (int i = 0; i < 32; ++i) ro[i] = f2u(u2f(ro[i]) * alpha);
            tmem_st32(t_o + q4 * 32, ro);
          }
        }
        float a0, a1, b0, b1;
        f2unpack(acc0, a0, a1);
        f2unpack(acc1, b0, b1);
        l = l * alpha + ((a0 + a1) + (b0 + b1));
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&c->p_full[slot]);
      }
      if (!ok) break;
      // ---- epilogue: O / l, LSE -------------------------------------------
      // O holds sums of bf16-rounded probabilities while l sums the fp32 ones.
      // Their mismatch is negligible except for a dominant probability, which
      // is not exactly representable once the reference lags the row maximum
      // (threshold above): the rounding error of the row's largest
      // probability, re-formed here exactly as the softmax formed it, is moved
      // into the normaliser, so that a row with one dominant key returns that
      // key's value.  The largest score was exponentiated against the final
      // reference m: a raise after its block needs a larger score.  The LSE
      // keeps the fp32 sum.
      const float p_best = ex2_approx(fmaf(s_best, c2, -m));
      const float corr = __uint_as_float(pack_bf16x2(p_best, 0.f) << 16) - p_best;
      const float l_o = l + corr;
      const bool got = mbar_wait(&c->o_full[slot], tiles & 1, &c->abort, a.spin_ns);
      ok = __all_sync(0xffffffffu, got) && ok;
      if (!ok) break;
      ++tiles;
      tc_fence_after();
      const bool pad_row = grow >= a.N;
      const float inv_l = pad_row ? 0.f : 1.f / l_o;
#pragma unroll
      for (int q4 = 0; q4 < D / 32; ++q4) {
        uint32_t ro[32];
        tmem_ld32(t_o + q4 * 32, ro);
        tmem_ld_wait();
        reg_fence(ro);
        uint4* dst = reinterpret_cast<uint4*>(orow + q4 * 32);
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          uint4 pk;
          pk.x = pack_bf16x2(u2f(ro[8 * v4 + 0]) * inv_l, u2f(ro[8 * v4 + 1]) * inv_l);
          pk.y = pack_bf16x2(u2f(ro[8 * v4 + 2]) * inv_l, u2f(ro[8 * v4 + 3]) * inv_l);
          pk.z = pack_bf16x2(u2f(ro[8 * v4 + 4]) * inv_l, u2f(ro[8 * v4 + 5]) * inv_l);
          pk.w = pack_bf16x2(u2f(ro[8 * v4 + 6]) * inv_l, u2f(ro[8 * v4 + 7]) * inv_l);
          dst[v4] = pk;
        }
      }
      tc_fence_before();
      mbar_arrive(&c->o_free[slot]);
      if (a.lse != nullptr)
        a.lse[orow_idx] = pad_row ? -INFINITY : (m + log2f(l)) * 0.69314718055994531f;
    }
    if (!ok) {
      c->abort = 1;
      report_status(a.status, CALIBATT_E_TIMEOUT);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kPpMma) tmem_dealloc(tmem, kTmemCols);
}

// SM count of every device, looked up on its first launch there.
std::atomic<int> g_num_sms[kMaxDevices];

// The two-slot kernel wherever its two slots fit in TMEM (all but d = 128 with
// 144-key blocks); there the kernel that splits each block's keys between two
// warps of the same rows.
template <int D, int BK>
constexpr bool kUsePp = ((cgcd(BK, TILE) >= 32 ? TILE : BK) <= 128 ? 128 : 160) + D <= 256;

template <int D, int BK>
int launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const TcArgs& a,
               cudaStream_t s) {
  constexpr bool pp = kUsePp<D, BK>;
  auto kern = [] {
    if constexpr (kUsePp<D, BK>) return k_attn_fwd_pp<D, BK>;
    else return k_attn_fwd<D, BK>;
  }();
  constexpr uint32_t smem_bytes = [] {
    if constexpr (kUsePp<D, BK>) return PpLayout<D, BK>::SMEM_BYTES;
    else return FwdLayout<D, BK>::SMEM_BYTES;
  }();
  (void)pp;
  int dev = 0;
  if (int rc = current_device(&dev)) return rc;
  // One-time set-up per instantiation and device (the shared-memory limit is
  // a per-device function attribute); atomics keep concurrent first calls
  // from several host threads race-free (the set-up itself is idempotent).
  static std::atomic<bool> configured[kMaxDevices];
  if (!configured[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) != cudaSuccess)
      return check_launch("cudaFuncSetAttribute(k_attn_fwd)");
    configured[dev].store(true, std::memory_order_release);
  }
  static std::atomic<int> launch_regs{-1};
  int regs = launch_regs.load(std::memory_order_acquire);
  if (regs < 0) {
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return check_launch("cudaFuncGetAttributes(k_attn_fwd)");
    regs = fa.numRegs;
    launch_regs.store(regs, std::memory_order_release);
  }
  // The register re-split inside the kernel is sized for exactly kLaunchRegs
  // per thread at launch; refuse to launch a build with any other count.
  if (regs != kLaunchRegs)
    return set_error(CALIBATT_E_UNSUPPORTED, "k_attn_fwd was built with %d registers per thread, expected %d", regs,
                     kLaunchRegs);
  int sms = g_num_sms[dev].load(std::memory_order_acquire);
  if (sms == 0) {
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return check_launch("cudaDeviceGetAttribute(SM count)");
    g_num_sms[dev].store(sms, std::memory_order_release);
  }
  const long long T = static_cast<long long>(a.B) * a.H * a.nqb;
  const int grid = static_cast<int>(std::min<long long>(sms, T));
  kern<<<grid, kThreads, smem_bytes, s>>>(tq, tk, tv, a);
  count_launch();
  return check_launch("k_attn_fwd");
}

}  // namespace

int launch_tc_fwd(const void* q, const void* k, const void* v, int d, const TcArgs& a, cudaStream_t s) {
  CUtensorMap tq, tk, tv;
  const uint64_t qrows = static_cast<uint64_t>(a.B) * a.H * a.Np;
  const uint64_t krows = static_cast<uint64_t>(a.B) * a.H * a.Npk;
  const uint32_t bk = static_cast<uint32_t>(a.block_k);
  int rc;
  if ((rc = make_tmap_bf16(&tq, q, qrows, d, TILE)) != CALIBATT_OK) return rc;
  // K and V are copied in pieces of gcd(bk, 128) rows where that is at least
  // 32 (two-slot kernel, 128-key steps), else in whole blocks
  const int pg = cgcd(static_cast<int>(bk), TILE);
  const uint32_t box = pg >= 32 ? static_cast<uint32_t>(pg) : bk;
  if ((rc = make_tmap_bf16(&tk, k, krows, d, box)) != CALIBATT_OK) return rc;
  if ((rc = make_tmap_bf16(&tv, v, krows, d, box)) != CALIBATT_OK) return rc;
  switch (bk) {
    case 64: return d == 128 ? launch_fwd<128, 64>(tq, tk, tv, a, s) : launch_fwd<64, 64>(tq, tk, tv, a, s);
    case 80: return d == 128 ? launch_fwd<128, 80>(tq, tk, tv, a, s) : launch_fwd<64, 80>(tq, tk, tv, a, s);
    case 96: return d == 128 ? launch_fwd<128, 96>(tq, tk, tv, a, s) : launch_fwd<64, 96>(tq, tk, tv, a, s);
    case 144: return d == 128 ? launch_fwd<128, 144>(tq, tk, tv, a, s) : launch_fwd<64, 144>(tq, tk, tv, a, s);
    default: return d == 128 ? launch_fwd<128, 128>(tq, tk, tv, a, s) : launch_fwd<64, 128>(tq, tk, tv, a, s);
  }
}

}  // namespace calibatt
