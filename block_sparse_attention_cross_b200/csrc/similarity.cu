// similarity.cu -- the spatial-similarity score of an attention map and the
// repetition dictionary built from it.
//
// CalibAtt (arXiv 2603.05503, paper page): Figure 4 shows attention maps
// whose pattern repeats across the spatial rows of each query frame; Figure
// 5(a) flags the heads that show this repetition and stores them in a
// dictionary; Figure 6(a) plots each map's "spatial similarity", Figure 6(b)
// its low spread across calibration prompts, and Figure S13 counts the heads
// whose score exceeds tau = 0.87.  The pages name the score but do not define
// it.  Reading taken here: the mean, over the query tokens (f, r, c) whose
// spatial row r has a next row in the same frame, of the cosine similarity of
// the dense attention rows of (f, r, c) and (f, r + 1, c) -- the two rows the
// anchor broadcast of Figure 5(b) bottom treats as one.  Rows of P are
// non-negative, so the score lies in [0, 1] and is 1 exactly when neighbouring
// rows attend identically.
//
// Per input and head, on the tensor cores: the log-sum-exp of every query row
// (the STATS pass of the block energies), then one pass over all key blocks
// in which a CTA holds the query tile Q (rows i) and the tile Q' shifted by
// one spatial row (rows i + cols), computes S = Q K^T and S' = Q' K^T into
// TMEM and accumulates, per row, <p_i, p_i'>, |p_i|^2 and |p_i'|^2 with
// p = 2^(s c2 - lse2).  The tile's cosines are reduced in a fixed order and a
// second kernel sums the tiles of each head in a fixed order, so the score is
// deterministic.
//
// CTA = one 128-row query tile of one head, 8 warps:
//   warp 0      TMA producer: Q and Q' once, then every K tile into a 4-deep ring
//   warp 1      TMEM allocator and MMA issuer: S, S' into one of two buffer
//               pairs (columns [0, 256) and [256, 512))
//   warps 4..7  thread t owns query row t (TMEM lane t)
// Every wait is bounded; on expiry the CTA records CALIBATT_E_TIMEOUT, waits
// (bounded) for its own copies and MMAs, frees TMEM and exits.
#include <atomic>
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace calibatt {
namespace {

constexpr int TILE = 128;
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;
constexpr int kRing = 4;

template <int D>
struct SimLayout {
  static constexpr uint32_t BOX_BYTES = TILE * 64 * 2;
  static constexpr uint32_t TILE_BYTES = TILE * D * 2;
  static constexpr uint32_t OFF_Q = 0;                          // Q, then Q'
  static constexpr uint32_t OFF_K = OFF_Q + 2 * TILE_BYTES;
  static constexpr uint32_t OFF_RED = OFF_K + kRing * TILE_BYTES;   // 4 warp partial sums + counts
  static constexpr uint32_t OFF_HALF = OFF_RED + 64;   // column half 1's (dot, |a|^2, |b|^2) per row
  static constexpr uint32_t OFF_CTRL = OFF_HALF + TILE * 3 * 4;
  static constexpr uint32_t CTRL_BYTES = 512;
  static constexpr uint32_t SMEM_BYTES = OFF_CTRL + CTRL_BYTES + 1024;
};

struct SimCtrl {
  uint64_t q_full;
  uint64_t k_full[kRing], k_empty[kRing];
  uint64_t s_full[2], s_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

struct SimArgs {
  int H, N, Np, nqb, nkb;
  int n_video, rows, cols;   // query tokens with a next spatial row: t < n_video and (t / cols) % rows < rows - 1
  float scale_log2;
  const float* lse2;         // [H * Np] log2-domain LSE of every row (STATS pass)
  float* tile_sum;           // [H * nqb] sum of the tile's cosines
  int32_t* tile_cnt;         // [H * nqb] rows counted
  int32_t* status;
  unsigned long long spin_ns;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    k_spatial_sim(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK, const SimArgs a) {
  using L = SimLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  SimCtrl* c = reinterpret_cast<SimCtrl*>(smem + L::OFF_CTRL);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int qb = blockIdx.x;
  const int h = blockIdx.y;
  const int n = a.nkb;

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
    mbar_arrive_expect_tx_w(&c->q_full, 2 * L::TILE_BYTES);
    // Q: rows qb * 128 ...; Q': the same rows one spatial row later.  Rows past
    // the tensor read as zeros; rows of the next head are never counted.
    const int row0 = h * a.Np + qb * TILE;
#pragma unroll
    for (int x = 0; x < D / 64; ++x) {
      tma_load_2d_w(smem + L::OFF_Q + x * L::BOX_BYTES, &tmQ, x * 64, row0, &c->q_full, pol_q);
      tma_load_2d_w(smem + L::OFF_Q + L::TILE_BYTES + x * L::BOX_BYTES, &tmQ, x * 64, row0 + a.cols, &c->q_full,
                    pol_q);
    }
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
      if (!ok) {
        c->abort = 1;
        report_status(a.status, CALIBATT_E_TIMEOUT);
      }
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
      for (int qq = 0; qq < 2; ++qq) {   // S = Q K^T, then S' = Q' K^T
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad =
              sdesc_sw128(sQ + qq * L::TILE_BYTES + (kk >> 2) * L::BOX_BYTES + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(sK + e * L::TILE_BYTES + (kk >> 2) * L::BOX_BYTES + (kk & 3) * 32, 16, 1024);
          mma_bf16_ss_w(tmem + sb * 256 + qq * TILE, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
        }
      }
      mma_commit_w(&c->s_full[sb]);
      mma_commit_w(&c->k_empty[e]);
    }
    if (!ok && lane == 0) {
      c->abort = 1;
      report_status(a.status, CALIBATT_E_TIMEOUT);
    }
    __syncwarp();
    mma_commit_w(&c->drain);
    mbar_wait(&c->drain, 0, nullptr, a.spin_ns);
  } else if (warp >= 4) {
    // ===================== row warpgroups ====================================
    // Warps 4-7 take key columns [0, 64) of every block, warps 8-11 [64, 128)
    // (two warps per SM sub-partition for the MUFU unit); half 1 hands its
    // row sums to half 0, which forms the cosine.
    const int w = warp & 3;
    const int hh = (warp - 4) >> 2;
    const int c0 = hh * 64;
    const int row = w * 32 + lane;
    const int grow = qb * TILE + row;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(w * 32) << 16);
    const float c2 = a.scale_log2;
    const bool counted = grow < a.n_video && (grow / a.cols) % a.rows < a.rows - 1;
    const float lse_a = counted ? a.lse2[static_cast<size_t>(h) * a.Np + grow] : 0.f;
    const float lse_b = counted ? a.lse2[static_cast<size_t>(h) * a.Np + grow + a.cols] : 0.f;
    float dot = 0.f, na = 0.f, nb = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int sb = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&c->s_full[sb], (j >> 1) & 1, &c->abort, a.spin_ns));
      if (!ok) break;
      tc_fence_after();
      const int valid = (j == a.nkb - 1) ? (a.N - j * TILE) : TILE;   // real keys of this block
      // this block's sums (two accumulators each), added to the row's totals after it
      float dot0 = 0.f, na0 = 0.f, nb0 = 0.f, dot1 = 0.f, na1 = 0.f, nb1 = 0.f;
#pragma unroll
      for (int q4 = 0; q4 < 2; ++q4) {
        uint32_t ra[32], rb[32];
        tmem_ld32(t_lane + sb * 256 + c0 + q4 * 32, ra);
        tmem_ld32(t_lane + sb * 256 + TILE + c0 + q4 * 32, rb);
        tmem_ld_wait();
        reg_fence(ra);
        reg_fence(rb);
        if (counted) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (c0 + q4 * 32 + i < valid) {
              const float pa = ex2_approx(fmaf(__uint_as_float(ra[i]), c2, -lse_a));
              const float pb = ex2_approx(fmaf(__uint_as_float(rb[i]), c2, -lse_b));
              if (i & 1) {
                dot1 = fmaf(pa, pb, dot1);
                na1 = fmaf(pa, pa, na1);
                nb1 = fmaf(pb, pb, nb1);
              } else {
                dot0 = fmaf(pa, pb, dot0);
                na0 = fmaf(pa, pa, na0);
                nb0 = fmaf(pb, pb, nb0);
              }
            }
          }
        }
      }
      dot += dot0 + dot1;
      na += na0 + na1;
      nb += nb0 + nb1;
      tc_fence_before();
      mbar_arrive(&c->s_empty[sb]);
    }
    if (!ok) {
      c->abort = 1;
      report_status(a.status, CALIBATT_E_TIMEOUT);
    }
    // The row's sums: half 0's plus half 1's, in that order.
    float* half = reinterpret_cast<float*>(smem + L::OFF_HALF);
    if (hh == 1) {
      half[row] = dot;
      half[TILE + row] = na;
      half[2 * TILE + row] = nb;
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (hh == 0) {
      dot += half[row];
      na += half[TILE + row];
      nb += half[2 * TILE + row];
      // Fixed-order reduction of the tile: lanes by shuffle, then the 4 warps.
      float cs = (counted && na > 0.f && nb > 0.f) ? dot * rsqrtf(na * nb) : 0.f;
      int cnt = counted ? 1 : 0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        cs += __shfl_xor_sync(0xffffffffu, cs, o);
        cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
      }
      float* red = reinterpret_cast<float*>(smem + L::OFF_RED);
      int* redc = reinterpret_cast<int*>(smem + L::OFF_RED + 32);
      if (lane == 0) {
        red[w] = cs;
        redc[w] = cnt;
      }
      asm volatile("bar.sync 2, 128;" ::: "memory");
      if (row == 0 && ok) {
        a.tile_sum[h * a.nqb + qb] = ((red[0] + red[1]) + red[2]) + red[3];
        a.tile_cnt[h * a.nqb + qb] = redc[0] + redc[1] + redc[2] + redc[3];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// score[h] = (sum of the tile sums of head h, in tile order, in double) /
// (rows counted); one warp per head, lanes take tiles in a fixed stride and
// the partials are combined in a fixed order.
__global__ void k_sim_finalize(const float* tile_sum, const int32_t* tile_cnt, int H, int nqb, float* score) {
  const int h = blockIdx.x;
  const int lane = threadIdx.x;
  double s = 0.0;
  long long cnt = 0;
  for (int t = lane; t < nqb; t += 32) {
    s += static_cast<double>(tile_sum[h * nqb + t]);
    cnt += tile_cnt[h * nqb + t];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, o);
    cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  }
  if (lane == 0) score[h] = cnt > 0 ? static_cast<float>(s / static_cast<double>(cnt)) : 0.f;
}

// mean[m] = (sum over inputs, in input order, of scores[i, m]) / n_inputs in
// float32; flags[m] = mean[m] >= tau.
__global__ void k_repetition_flags(const float* scores, int n_inputs, int n_maps, float tau, float* mean,
                                   uint8_t* flags) {
  for (int m = blockIdx.x * blockDim.x + threadIdx.x; m < n_maps; m += gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int i = 0; i < n_inputs; ++i) s += scores[static_cast<long long>(i) * n_maps + m];
    const float mu = s / static_cast<float>(n_inputs);
    if (mean != nullptr) mean[m] = mu;
    flags[m] = mu >= tau ? 1 : 0;
  }
}

template <int D>
int launch_sim(const CUtensorMap& tq, const CUtensorMap& tk, const SimArgs& a, cudaStream_t s) {
  auto kern = k_spatial_sim<D>;
  int dev = 0;
  if (int rc = current_device(&dev)) return rc;
  static std::atomic<bool> configured[kMaxDevices];
  if (!configured[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SimLayout<D>::SMEM_BYTES) !=
        cudaSuccess)
      return check_launch("cudaFuncSetAttribute(k_spatial_sim)");
    configured[dev].store(true, std::memory_order_release);
  }
  kern<<<dim3(a.nqb, a.H), kThreads, SimLayout<D>::SMEM_BYTES, s>>>(tq, tk, a);
  count_launch();
  return check_launch("k_spatial_sim");
}

size_t sim_ws_bytes(int H, int Np) {
  const size_t nqb = static_cast<size_t>(Np) / TILE;
  auto up = [](size_t b) { return (b + 255) & ~size_t(255); };
  return 256 + up(static_cast<size_t>(H) * Np * 4) + 2 * up(static_cast<size_t>(H) * nqb * 4);
}

}  // namespace
}  // namespace calibatt

using namespace calibatt;

extern "C" {

int calibatt_spatial_similarity_workspace_size(int H, int Np, size_t* bytes) {
  if (bytes == nullptr) return set_error(CALIBATT_E_INVALID, "bytes is NULL");
  if (H <= 0 || Np <= 0 || Np % TILE) return set_error(CALIBATT_E_INVALID, "bad sizes");
  *bytes = sim_ws_bytes(H, Np);
  return CALIBATT_OK;
}

int calibatt_spatial_similarity(const void* q, const void* k, int H, int N, int Np, int d, int dtype, int frames,
                                int rows, int cols, float scale, float* score_out, void* workspace,
                                size_t workspace_bytes, int32_t* dev_status, calibatt_stream_t stream) {
  int rc = check_energy_args(q, k, H, N, Np, d, dtype, TILE, TILE, scale);
  if (rc) return rc;
  if (dtype != CALIBATT_BF16) return set_error(CALIBATT_E_UNSUPPORTED, "the spatial similarity is bf16 only");
  if (score_out == nullptr) return set_error(CALIBATT_E_INVALID, "score_out is NULL");
  if (frames <= 0 || rows < 2 || cols <= 0 || static_cast<long long>(frames) * rows * cols > N)
    return set_error(CALIBATT_E_INVALID, "video geometry %dx%dx%d does not fit N=%d (and rows >= 2)", frames, rows,
                     cols, N);
  if (workspace == nullptr || workspace_bytes < sim_ws_bytes(H, Np))
    return set_error(CALIBATT_E_WORKSPACE, "workspace too small: need %zu bytes", sim_ws_bytes(H, Np));
  const int nqb = Np / TILE;
  auto up = [](size_t b) { return (b + 255) & ~size_t(255); };
  char* base = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(workspace) + 255) & ~uintptr_t(255));
  float* lse2 = reinterpret_cast<float*>(base);
  float* tile_sum = reinterpret_cast<float*>(base + up(static_cast<size_t>(H) * Np * 4));
  int32_t* tile_cnt = reinterpret_cast<int32_t*>(base + up(static_cast<size_t>(H) * Np * 4) +
                                                 up(static_cast<size_t>(H) * nqb * 4));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // Pass 1: every row's log-sum-exp (the block energies' STATS pass).
  TcArgs ta{};
  ta.B = 1; ta.H = H; ta.N = N; ta.Np = Np; ta.nqb = nqb; ta.nkb = nqb;
  ta.scale_log2 = scale * 1.4426950408889634f;
  ta.lse2 = lse2; ta.status = dev_status; ta.spin_ns = spin_limit_ns();
  if ((rc = launch_tc_stats(q, k, d, ta, s))) return rc;
  // Pass 2: the row-pair cosines, then the per-head means.
  CUtensorMap tq, tk;
  const uint64_t qrows = static_cast<uint64_t>(H) * Np;
  if ((rc = make_tmap_bf16(&tq, q, qrows, d, TILE)) != CALIBATT_OK) return rc;
  if ((rc = make_tmap_bf16(&tk, k, qrows, d, TILE)) != CALIBATT_OK) return rc;
  SimArgs sa{};
  sa.H = H; sa.N = N; sa.Np = Np; sa.nqb = nqb; sa.nkb = nqb;
  sa.n_video = frames * rows * cols; sa.rows = rows; sa.cols = cols;
  sa.scale_log2 = ta.scale_log2; sa.lse2 = lse2; sa.tile_sum = tile_sum; sa.tile_cnt = tile_cnt;
  sa.status = dev_status; sa.spin_ns = spin_limit_ns();
  if ((rc = d == 128 ? launch_sim<128>(tq, tk, sa, s) : launch_sim<64>(tq, tk, sa, s))) return rc;
  k_sim_finalize<<<H, 32, 0, s>>>(tile_sum, tile_cnt, H, nqb, score_out);
  count_launch();
  return check_launch("k_sim_finalize");
}

int calibatt_repetition_flags(const float* scores, int n_inputs, int n_maps, float tau, float* mean_out,
                              uint8_t* flags_out, calibatt_stream_t stream) {
  if (scores == nullptr || flags_out == nullptr) return set_error(CALIBATT_E_INVALID, "scores and flags are NULL");
  if (n_inputs <= 0 || n_maps <= 0) return set_error(CALIBATT_E_INVALID, "bad sizes");
  if (!std::isfinite(tau)) return set_error(CALIBATT_E_INVALID, "tau must be finite");
  const unsigned grid = static_cast<unsigned>(std::min(148 * 4, (n_maps + 255) / 256));
  k_repetition_flags<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(scores, n_inputs, n_maps, tau,
                                                                               mean_out, flags_out);
  count_launch();
  return check_launch("k_repetition_flags");
}

}  // extern "C"
