// attn_tc.cu -- the two dense passes of the block-energy calibration on
// Blackwell tensor cores (tcgen05 + TMEM + TMA).
//
// CalibAtt (arXiv 2603.05503, paper page) scores key blocks by their
// post-softmax mass (Figure 2 block-level maps; Table S5 "block energies").
// STATS computes each query row's dense log-sum-exp (log2 domain) over all
// real keys; ENERGY recomputes the scores, sums exp2(s - LSE) inside every key
// block and reduces the 128 rows of the query block in a fixed order, so the
// result is deterministic.  Scores are always produced in 128-key tiles; for a
// key-block size BK other than 128 (Table S6: 64, 80, 96, 144) a tile covers up
// to three key blocks, whose boundaries fall on 16-column chunks, so every
// chunk's sum goes to exactly one block.
//
// CTA = one 128-row query tile of one head, 12 warps:
//   warp 0      TMA producer: the Q tile once, then every K tile into a
//               4-deep ring.
//   warp 1      TMEM allocator and MMA issuer: S = Q K^T into one of two TMEM
//               S buffers (columns [0,128) and [128,256)), so the next block's
//               product overlaps the current block's exponentials.
//   warps 4..7  score warpgroup 0: key columns [0, 64) of every tile; thread t
//               owns query row t (TMEM lane t).
//   warps 8..11 score warpgroup 1: key columns [64, 128) of the same rows.
// Both passes are MUFU-bound (one exponential per score); two score warps per
// SM sub-partition keep that unit busy.  The energy pass needs no exchange
// between the halves (row sums per key block are reduced over rows anyway);
// the statistics pass merges the halves' (max, sum) once per tile.
// Both control warps run their loops warp-uniformly and issue through one
// elected lane.  Every wait is bounded; on expiry the CTA records
// CALIBATT_E_TIMEOUT, waits (bounded) for its own copies and MMAs, frees TMEM
// and exits.
#include <atomic>
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace calibatt {
namespace {

enum { MODE_STATS = 1, MODE_ENERGY = 2 };

constexpr int TILE = 128;
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 256;
constexpr int kRing = 4;
constexpr int kMaxBlocks = 2048;  // key blocks per row (partials buffer)

template <int D>
struct EnergyLayout {
  static constexpr uint32_t BOX_BYTES = TILE * 64 * 2;  // one 128 x 64 bf16 TMA box
  static constexpr uint32_t TILE_BYTES = TILE * D * 2;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + TILE_BYTES;
  // ENERGY: per-warp block sums, 8 per key block; STATS: the halves' (max, sum) per row
  static constexpr uint32_t OFF_PART = OFF_K + kRing * TILE_BYTES;
  static constexpr uint32_t OFF_CTRL = OFF_PART + kMaxBlocks * 8 * 4;
  static constexpr uint32_t CTRL_BYTES = 1024;
  static constexpr uint32_t SMEM_BYTES = OFF_CTRL + CTRL_BYTES + 1024;  // + alignment slack
};

struct EnergyCtrl {
  uint64_t q_full;
  uint64_t k_full[kRing], k_empty[kRing];
  uint64_t s_full[2], s_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void give_up(EnergyCtrl* c, int32_t* status) {
  c->abort = 1;
  report_status(status, CALIBATT_E_TIMEOUT);
}

template <int D, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    k_energy_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK, const TcArgs a) {
  using L = EnergyLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  EnergyCtrl* c = reinterpret_cast<EnergyCtrl*>(smem + L::OFF_CTRL);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int qb = blockIdx.x;
  const int h = blockIdx.y;
  const int n = a.nkb;   // dense: every key block, in order

  if (tid == 0) {
    mbar_init(&c->q_full, 1);
    for (int e = 0; e < kRing; ++e) {
      mbar_init(&c->k_full[e], 1);
      mbar_init(&c->k_empty[e], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&c->s_full[s], 1);
      mbar_init(&c->s_empty[s], 256);
    }
    mbar_init(&c->drain, 1);
    c->abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
  }
  if (warp == 1) {
    tmem_alloc(&c->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = c->tmem_base;

  if (warp == 0) {
    // ===================== TMA producer ======================================
    const uint64_t pol_k = l2_policy_evict_last();
    const uint64_t pol_q = l2_policy_evict_first();
    int kf = 0;
    bool ok = true;
    mbar_arrive_expect_tx_w(&c->q_full, L::TILE_BYTES);
#pragma unroll
    for (int x = 0; x < D / 64; ++x)
      tma_load_2d_w(smem + L::OFF_Q + x * L::BOX_BYTES, &tmQ, x * 64, h * a.Np + qb * TILE, &c->q_full, pol_q);
    for (int j = 0; j < n; ++j) {
      const int e = j % kRing;
      ok = __all_sync(0xffffffffu, mbar_wait(&c->k_empty[e], ((j / kRing) & 1) ^ 1, &c->abort, a.spin_ns));
      if (!ok) break;
      mbar_arrive_expect_tx_w(&c->k_full[e], L::TILE_BYTES);
#pragma unroll
      for (int x = 0; x < D / 64; ++x)
        tma_load_2d_w(smem + L::OFF_K + e * L::TILE_BYTES + x * L::BOX_BYTES, &tmK, x * 64, h * a.Np + j * TILE,
                      &c->k_full[e], pol_k);
      ++kf;
    }
    if (lane == 0) {
      if (!ok) give_up(c, a.status);
      // Drain: every issued copy must have landed before the CTA may exit.
      mbar_wait(&c->q_full, 0, nullptr, a.spin_ns);
      for (int e = 0; e < kRing; ++e) {
        const int fills = (kf > e) ? (kf - 1 - e) / kRing + 1 : 0;
        if (fills > 0) mbar_wait(&c->k_full[e], (fills - 1) & 1, nullptr, a.spin_ns);
      }
    }
  } else if (warp == 1) {
    // ===================== MMA issuer ========================================
    const uint32_t sQ = smem_u32(smem + L::OFF_Q);
    const uint32_t sK = smem_u32(smem + L::OFF_K);
    constexpr uint32_t IDESC_S = idesc_bf16_f32(TILE, TILE, false);
    bool ok = __all_sync(0xffffffffu, mbar_wait(&c->q_full, 0, &c->abort, a.spin_ns));
    for (int j = 0; ok && j < n; ++j) {
      const int e = j % kRing;
      const int sb = j & 1;
      ok = mbar_wait(&c->k_full[e], (j / kRing) & 1, &c->abort, a.spin_ns) &&
           (j < 2 || mbar_wait(&c->s_empty[sb], ((j >> 1) & 1) ^ 1, &c->abort, a.spin_ns));
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t ad = sdesc_sw128(sQ + (kk >> 2) * L::BOX_BYTES + (kk & 3) * 32, 16, 1024);
        const uint64_t bd =
            sdesc_sw128(sK + e * L::TILE_BYTES + (kk >> 2) * L::BOX_BYTES + (kk & 3) * 32, 16, 1024);
        mma_bf16_ss_w(tmem + sb * TILE, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
      }
      mma_commit_w(&c->s_full[sb]);
      mma_commit_w(&c->k_empty[e]);
    }
    if (!ok && lane == 0) give_up(c, a.status);
    __syncwarp();
    // Drain: all issued MMAs complete before TMEM can be released.
    mma_commit_w(&c->drain);
    mbar_wait(&c->drain, 0, nullptr, a.spin_ns);
  } else if (warp >= 4) {
    // ===================== score warpgroups ==================================
    const int w = warp & 3;                   // TMEM lane quarter
    const int hh = (warp - 4) >> 2;           // key-column half of every tile
    const int c0 = hh * 64;
    const int w8 = hh * 4 + w;                // this warp's partial slot
    const int row = w * 32 + lane;
    const int grow = qb * TILE + row;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(w * 32) << 16);
    const float c2 = a.scale_log2;
    float* part = reinterpret_cast<float*>(smem + L::OFF_PART);
    const int bk = a.block_k;
    if (MODE == MODE_ENERGY && bk != TILE) {
      // Each warp owns the slots part[8 * kb + w8]; they accumulate across tiles.
      for (int kb = lane; kb < a.nke; kb += 32) part[8 * kb + w8] = 0.f;
      __syncwarp();
    }
    const float lse2_row =
        (MODE == MODE_ENERGY && grow < a.N) ? a.lse2[static_cast<size_t>(h) * a.Np + grow] : 0.f;
    float m = -INFINITY;
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int sb = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&c->s_full[sb], (j >> 1) & 1, &c->abort, a.spin_ns));
      if (!ok) break;
      tc_fence_after();
      float s[64];
      {
        uint32_t r[64];
#pragma unroll
        for (int q4 = 0; q4 < 2; ++q4)
          tmem_ld32(t_lane + sb * TILE + c0 + q4 * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[q4 * 32]));
        tmem_ld_wait();
        reg_fence(r);
#pragma unroll
        for (int i = 0; i < 64; ++i) s[i] = __uint_as_float(r[i]);
      }
      tc_fence_before();
      mbar_arrive(&c->s_empty[sb]);
      // Key columns past the sequence end exist only in the last block.
      const int valid = (j == a.nkb - 1) ? (a.N - j * TILE) : TILE;
      if (valid < TILE) {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (c0 + i >= valid) s[i] = -INFINITY;
      }
      // sum of 2^(s c2 - ref) over columns [i0, i0 + 2 np): packed pairs, two
      // accumulators (independent chains for the MUFU pipe)
      const uint64_t c2x2 = f2pack(c2, c2);
      auto exp_sum = [&](int i0, int np, float ref) {
        const uint64_t negr = f2pack(-ref, -ref);
        uint64_t acc0 = f2pack(0.f, 0.f), acc1 = acc0;
#pragma unroll
        for (int i = 0; i < np; ++i) {
          const uint64_t x = ffma2(f2pack(s[i0 + 2 * i], s[i0 + 2 * i + 1]), c2x2, negr);
          float xl, xh;
          f2unpack(x, xl, xh);
          const uint64_t pv = f2pack(ex2_approx(xl), ex2_approx(xh));
          if (i & 1) acc1 = fadd2(acc1, pv); else acc0 = fadd2(acc0, pv);
        }
        float a0, a1, b0, b1;
        f2unpack(acc0, a0, a1);
        f2unpack(acc1, b0, b1);
        return (a0 + a1) + (b0 + b1);
      };
      if (MODE == MODE_ENERGY && bk == TILE) {
        float rs = 0.f;
        if (grow < a.N) rs = exp_sum(0, 32, lse2_row);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, o);
        if (lane == 0) part[j * 8 + w8] = rs;
      } else if (MODE == MODE_ENERGY) {
        // Key blocks kb0, kb0+1, kb0+2 meet this tile at columns [0,b1),
        // [b1,b2), [b2,128); b1 and b2 are multiples of 16.
        const int kb0 = (j * TILE) / bk;
        const int b1 = (kb0 + 1) * bk - j * TILE;
        const int b2 = b1 + bk;
        float r0 = 0.f, r1 = 0.f, r2 = 0.f;
        if (grow < a.N) {
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const float cs = exp_sum(cc * 16, 8, lse2_row);
            const int col = c0 + cc * 16;
            if (col < b1) r0 += cs;
            else if (col < b2) r1 += cs;
            else r2 += cs;
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          r0 += __shfl_xor_sync(0xffffffffu, r0, o);
          r1 += __shfl_xor_sync(0xffffffffu, r1, o);
          r2 += __shfl_xor_sync(0xffffffffu, r2, o);
        }
        if (lane == 0) {
          part[8 * kb0 + w8] += r0;
          if (b1 < TILE && kb0 + 1 < a.nke) part[8 * (kb0 + 1) + w8] += r1;
          if (b2 < TILE && kb0 + 2 < a.nke) part[8 * (kb0 + 2) + w8] += r2;
        }
        __syncwarp();
      } else {
        float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
        for (int i = 4; i < 60; i += 8) {
          mx0 = fmax3(mx0, s[i], s[i + 1]);
          mx1 = fmax3(mx1, s[i + 2], s[i + 3]);
          mx2 = fmax3(mx2, s[i + 4], s[i + 5]);
          mx3 = fmax3(mx3, s[i + 6], s[i + 7]);
        }
        mx0 = fmax3(mx0, s[60], s[61]);
        mx1 = fmax3(mx1, s[62], s[63]);
        const float mx = fmax3(mx0, mx1, fmaxf(mx2, mx3));
        const float m_new = fmaxf(m, mx * c2);
        // (a half whose columns are all past the sequence end so far keeps m = -inf)
        if (m_new != -INFINITY) {
          const float alpha = ex2_approx(m - m_new);
          l = l * alpha + exp_sum(0, 32, m_new);
          m = m_new;
        }
      }
    }
    if (!ok) give_up(c, a.status);
    if (MODE == MODE_STATS) {
      // The two halves of each row: (max, sum) merged in half 0.
      float2* xb = reinterpret_cast<float2*>(smem + L::OFF_PART);
      xb[hh * 128 + row] = make_float2(m, l);
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (hh == 0) {
        const float2 o = xb[128 + row];
        const float mm = fmaxf(m, o.x);
        float ll = 0.f;
        if (mm != -INFINITY) ll = l * ex2_approx(m - mm) + o.y * ex2_approx(o.x - mm);
        a.lse2[static_cast<size_t>(h) * a.Np + grow] = (ok && grow < a.N && mm != -INFINITY) ? mm + log2f(ll) : -INFINITY;
      }
    } else {
      // ENERGY: per key block, the eight warp partials in a fixed order.
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (ok) {
        const int rows = min(TILE, a.N - qb * TILE);
        const float inv_rows = 1.f / static_cast<float>(rows);
        const int ne = (bk == TILE) ? n : a.nke;
        float* erow = a.energy + (static_cast<size_t>(h) * a.nqb + qb) * ne;
        for (int jj = hh * 128 + row; jj < ne; jj += 256) {
          const float* pp = part + 8 * jj;
          const float tot = ((pp[0] + pp[1]) + (pp[2] + pp[3])) + ((pp[4] + pp[5]) + (pp[6] + pp[7]));
          erow[jj] = tot * inv_rows;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

template <int D, int MODE>
int launch_one(const CUtensorMap& tq, const CUtensorMap& tk, const TcArgs& a, dim3 grid, cudaStream_t s) {
  auto kern = k_energy_tc<D, MODE>;
  int dev = 0;
  if (int rc = current_device(&dev)) return rc;
  // One-time, idempotent set-up per device (the shared-memory limit is a
  // per-device function attribute); race-free across host threads.
  static std::atomic<bool> configured[kMaxDevices];
  if (!configured[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, EnergyLayout<D>::SMEM_BYTES) !=
        cudaSuccess)
      return check_launch("cudaFuncSetAttribute(k_energy_tc)");
    configured[dev].store(true, std::memory_order_release);
  }
  kern<<<grid, kThreads, EnergyLayout<D>::SMEM_BYTES, s>>>(tq, tk, a);
  count_launch();
  return check_launch("k_energy_tc");
}

}  // namespace

int launch_tc_stats(const void* q, const void* k, int d, const TcArgs& a, cudaStream_t s) {
  CUtensorMap tq, tk;
  const uint64_t rows = static_cast<uint64_t>(a.H) * a.Np;
  int rc;
  if ((rc = make_tmap_bf16(&tq, q, rows, d)) != CALIBATT_OK) return rc;
  if ((rc = make_tmap_bf16(&tk, k, rows, d)) != CALIBATT_OK) return rc;
  dim3 grid(a.nqb, a.H, 1);
  return d == 128 ? launch_one<128, MODE_STATS>(tq, tk, a, grid, s) : launch_one<64, MODE_STATS>(tq, tk, a, grid, s);
}

int launch_tc_energy(const void* q, const void* k, int d, const TcArgs& a, cudaStream_t s) {
  CUtensorMap tq, tk;
  const uint64_t rows = static_cast<uint64_t>(a.H) * a.Np;
  int rc;
  if ((rc = make_tmap_bf16(&tq, q, rows, d)) != CALIBATT_OK) return rc;
  if ((rc = make_tmap_bf16(&tk, k, rows, d)) != CALIBATT_OK) return rc;
  dim3 grid(a.nqb, a.H, 1);
  if (d == 128) {
    if ((rc = launch_one<128, MODE_STATS>(tq, tk, a, grid, s)) != CALIBATT_OK) return rc;
    return launch_one<128, MODE_ENERGY>(tq, tk, a, grid, s);
  }
  if ((rc = launch_one<64, MODE_STATS>(tq, tk, a, grid, s)) != CALIBATT_OK) return rc;
  return launch_one<64, MODE_ENERGY>(tq, tk, a, grid, s);
}

}  // namespace calibatt
