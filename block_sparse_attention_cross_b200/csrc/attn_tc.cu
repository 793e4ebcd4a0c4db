// attn_tc.cu -- block-sparse flash-attention forward on Blackwell tensor cores
// (tcgen05 + TMEM + TMA), plus the two dense passes of the block-energy
// calibration that reuse the same pipeline.
//
// CalibAtt (arXiv 2603.05503, paper page): at inference the selected blocks
// are computed densely and the unselected ones are skipped (Abstract;
// Figure 5(b) top).  Here a CTA owns one 128-row query tile of one (batch,
// head) and walks that tile's compiled kept-block list: only the kept K/V
// tiles are fetched (TMA) and multiplied (tcgen05), so a skipped block costs
// neither bytes nor FLOPs.  Calibration scores blocks by their post-softmax
// mass (Figure 2 block-level maps, Table S5 "block energies"): STATS computes
// each row's dense log-sum-exp, ENERGY recomputes the scores and sums the
// probabilities falling in each key block.
//
// CTA = 8 warps:
//   warp 0      TMA producer (one lane): Q tile once, then K (and V) tiles of
//               the kept blocks into 2-deep rings.
//   warp 1      TMEM allocator and MMA issuer (one lane): S = Q K^T into one of
//               two TMEM S buffers, then O += P V into the TMEM O accumulator.
//   warps 4..7  softmax warpgroup: thread t owns query row t (TMEM lane t);
//               online softmax in registers, P (bf16) written to shared memory
//               in the 128-byte-swizzled K-major layout the MMA reads, O
//               rescaled in TMEM when the running max grows, final O / l and
//               LSE written out.
// TMEM columns: [0,128) S0, [128,256) S1, [256,256+d) O.
// Every wait is bounded; on expiry the CTA records CALIBATT_E_TIMEOUT, waits
// (bounded) for its own copies and MMAs, frees TMEM and exits.
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace calibatt {
namespace {

enum { MODE_FWD = 0, MODE_STATS = 1, MODE_ENERGY = 2 };

constexpr int TILE = 128;
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxBlocks = 1024;  // longest kept-block list (key blocks per row)

template <int D>
struct Layout {
  static constexpr uint32_t BOX_BYTES = TILE * 64 * 2;   // one 128 x 64 bf16 TMA box
  static constexpr uint32_t Q_BYTES = TILE * D * 2;
  static constexpr uint32_t KV_BYTES = TILE * D * 2;
  static constexpr uint32_t P_BYTES = TILE * TILE * 2;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + 2 * KV_BYTES;
  static constexpr uint32_t OFF_P = OFF_V + 2 * KV_BYTES;
  static constexpr uint32_t OFF_CTRL = OFF_P + P_BYTES;
  static constexpr uint32_t CTRL_BYTES = 8192;
  static constexpr uint32_t SMEM_BYTES = OFF_CTRL + CTRL_BYTES + 1024;  // + alignment slack
};

struct Ctrl {
  uint64_t q_full;
  uint64_t k_full[2], k_empty[2];
  uint64_t v_full[2], v_empty[2];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full;
  uint64_t o_done;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int list[kMaxBlocks];
};
static_assert(sizeof(Ctrl) <= 8192, "control block too large");

__device__ __forceinline__ void give_up(Ctrl* c, int32_t* status) {
  c->abort = 1;
  report_status(status, CALIBATT_E_TIMEOUT);
}

__device__ __forceinline__ float u2f(uint32_t x) { return __uint_as_float(x); }
__device__ __forceinline__ uint32_t f2u(float x) { return __float_as_uint(x); }

template <int D, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    k_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const TcArgs a) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctrl* c = reinterpret_cast<Ctrl*>(smem + L::OFF_CTRL);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int qb = blockIdx.x;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int bh = b * a.H + h;

  if (tid == 0) {
    mbar_init(&c->q_full, 1);
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      mbar_init(&c->k_full[s], 1);
      mbar_init(&c->k_empty[s], 1);
      mbar_init(&c->v_full[s], 1);
      mbar_init(&c->v_empty[s], 1);
      mbar_init(&c->s_full[s], 1);
      mbar_init(&c->s_empty[s], 128);
    }
    mbar_init(&c->p_full, 128);
    mbar_init(&c->o_done, 1);
    mbar_init(&c->drain, 1);
    c->abort = 0;
    fence_barrier_init();
  }
  if (tid == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    if (MODE == MODE_FWD) tma_prefetch_desc(&tmV);
  }

  // ---- the kept-block list of this query tile (validated) ----------------
  int n;
  bool bad = false;
  if (MODE == MODE_FWD) {
    const long long r = static_cast<long long>(a.map_offset + h) * a.nqb + qb;
    const int base = a.row_base[r];
    const int pat = a.row_pat[r];
    int p0 = 0, p1 = 0;
    if (pat < 0 || pat >= a.n_pat) {
      bad = true;
    } else {
      p0 = a.pat_ptr[pat];
      p1 = a.pat_ptr[pat + 1];
      if (p0 < 0 || p1 < p0 || p1 > a.nnz_pat || p1 - p0 > a.nkb) bad = true;
    }
    n = bad ? 0 : p1 - p0;
    for (int i = tid; i < n; i += kThreads) {
      const int off = a.pat_off[p0 + i];
      const int kb = base + off;
      bool ok = (kb >= 0) && (kb < a.nkb);
      if (i > 0) ok = ok && (off > a.pat_off[p0 + i - 1]);
      if (!ok) bad = true;
      c->list[i] = kb;
    }
  } else {
    n = a.nkb;
    for (int i = tid; i < n; i += kThreads) c->list[i] = i;
  }
  bad = __syncthreads_or(bad) != 0;
  if (bad) {
    n = 0;
    if (tid == 0) report_status(a.status, CALIBATT_E_CORRUPT);
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
    if (lane == 0 && n > 0) {
      const int qrow = bh * a.Np + qb * TILE;
      int kf = 0, vf = 0;  // loads issued
      bool ok = true;
      mbar_arrive_expect_tx(&c->q_full, L::Q_BYTES);
#pragma unroll
      for (int x = 0; x < D / 64; ++x)
        tma_load_2d(smem + L::OFF_Q + x * L::BOX_BYTES, &tmQ, x * 64, qrow, &c->q_full);
      for (int j = 0; j < n; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        const int krow = bh * a.Np + c->list[j] * TILE;
        if (!mbar_wait(&c->k_empty[st], ph ^ 1, &c->abort, a.spin_ns)) { ok = false; break; }
        mbar_arrive_expect_tx(&c->k_full[st], L::KV_BYTES);
#pragma unroll
        for (int x = 0; x < D / 64; ++x)
          tma_load_2d(smem + L::OFF_K + st * L::KV_BYTES + x * L::BOX_BYTES, &tmK, x * 64, krow, &c->k_full[st]);
        ++kf;
        if (MODE == MODE_FWD) {
          if (!mbar_wait(&c->v_empty[st], ph ^ 1, &c->abort, a.spin_ns)) { ok = false; break; }
          mbar_arrive_expect_tx(&c->v_full[st], L::KV_BYTES);
#pragma unroll
          for (int x = 0; x < D / 64; ++x)
            tma_load_2d(smem + L::OFF_V + st * L::KV_BYTES + x * L::BOX_BYTES, &tmV, x * 64, krow,
                        &c->v_full[st]);
          ++vf;
        }
      }
      if (!ok) give_up(c, a.status);
      // Drain: every issued copy must have landed before the CTA may exit.
      mbar_wait(&c->q_full, 0, nullptr, a.spin_ns);
#pragma unroll
      for (int st = 0; st < 2; ++st) {
        const int fk = (kf - st + 1) / 2;
        if (fk > 0) mbar_wait(&c->k_full[st], (fk - 1) & 1, nullptr, a.spin_ns);
        const int fv = (vf - st + 1) / 2;
        if (fv > 0) mbar_wait(&c->v_full[st], (fv - 1) & 1, nullptr, a.spin_ns);
      }
    }
  } else if (warp == 1) {
    // ===================== MMA issuer ========================================
    if (lane == 0 && n > 0) {
      const uint32_t sQ = smem_u32(smem + L::OFF_Q);
      const uint32_t sK = smem_u32(smem + L::OFF_K);
      const uint32_t sV = smem_u32(smem + L::OFF_V);
      const uint32_t sP = smem_u32(smem + L::OFF_P);
      constexpr uint32_t IDESC_S = idesc_bf16_f32(TILE, TILE, false);
      constexpr uint32_t IDESC_O = idesc_bf16_f32(TILE, D, true);
      bool ok = mbar_wait(&c->q_full, 0, &c->abort, a.spin_ns);

      auto issue_pv = [&](int i) -> bool {
        const int st = i & 1;
        const uint32_t ph = (i >> 1) & 1;
        if (!mbar_wait(&c->v_full[st], ph, &c->abort, a.spin_ns)) return false;
        if (!mbar_wait(&c->p_full, i & 1, &c->abort, a.spin_ns)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < TILE / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(sP + (kk >> 2) * L::BOX_BYTES + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(sV + st * L::KV_BYTES + kk * 2048, L::BOX_BYTES, 1024);
          mma_bf16_ss(tmem + 256, ad, bd, IDESC_O, (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&c->v_empty[st]);
        mma_commit(&c->o_done);
        return true;
      };

      for (int j = 0; ok && j < n; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait(&c->k_full[st], ph, &c->abort, a.spin_ns)) { ok = false; break; }
        if (j >= 2 && !mbar_wait(&c->s_empty[st], ph ^ 1, &c->abort, a.spin_ns)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(sQ + (kk >> 2) * L::BOX_BYTES + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(sK + st * L::KV_BYTES + (kk >> 2) * L::BOX_BYTES + (kk & 3) * 32, 16, 1024);
          mma_bf16_ss(tmem + st * TILE, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
        }
        mma_commit(&c->s_full[st]);
        mma_commit(&c->k_empty[st]);
        if (MODE == MODE_FWD && j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok && MODE == MODE_FWD) ok = issue_pv(n - 1);
      if (!ok) give_up(c, a.status);
      // Drain: all issued MMAs complete before TMEM can be released.
      mma_commit(&c->drain);
      mbar_wait(&c->drain, 0, nullptr, a.spin_ns);
    }
  } else if (warp >= 4) {
    // ===================== softmax warpgroup =================================
    const int w = warp - 4;
    const int row = w * 32 + lane;
    const int grow = qb * TILE + row;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(w * 32) << 16);
    const float c2 = a.scale_log2;
    float m = -INFINITY;
    float l = 0.f;
    float lse2_row = 0.f;
    float* part = reinterpret_cast<float*>(smem + L::OFF_P);  // ENERGY: per-warp block partials
    if (MODE == MODE_ENERGY) lse2_row = (grow < a.N) ? a.lse2[static_cast<size_t>(h) * a.Np + grow] : 0.f;
    const uint32_t sP = smem_u32(smem + L::OFF_P);
    bool ok = true;

    for (int j = 0; j < n; ++j) {
      const int sb = j & 1;
      const uint32_t ph = (j >> 1) & 1;
      ok = mbar_wait(&c->s_full[sb], ph, &c->abort, a.spin_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      float s[TILE];
#pragma unroll
      for (int q4 = 0; q4 < TILE / 32; ++q4) {
        uint32_t r[32];
        tmem_ld32(t_lane + sb * TILE + q4 * 32, r);
        tmem_ld_wait();
        reg_fence(r);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[q4 * 32 + i] = u2f(r[i]);
      }
      tc_fence_before();
      mbar_arrive(&c->s_empty[sb]);

      const int kb = c->list[j];
      const int valid = (kb == a.nkb - 1) ? (a.N - kb * TILE) : TILE;
      if (valid < TILE) {
#pragma unroll
        for (int i = 0; i < TILE; ++i)
          if (i >= valid) s[i] = -INFINITY;
      }

      if (MODE == MODE_ENERGY) {
        float rs = 0.f;
        if (grow < a.N) {
#pragma unroll
          for (int i = 0; i < TILE; ++i) rs += ex2_approx(fmaf(s[i], c2, -lse2_row));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, o);
        if (lane == 0) part[j * 4 + w] = rs;
        continue;
      }

      float mx = s[0];
#pragma unroll
      for (int i = 1; i < TILE; ++i) mx = fmaxf(mx, s[i]);
      const float m_new = fmaxf(m, mx * c2);
      const float alpha = ex2_approx(m - m_new);
      const float neg = -m_new;
      float rs = 0.f;
#pragma unroll
      for (int i = 0; i < TILE; ++i) {
        s[i] = ex2_approx(fmaf(s[i], c2, neg));
        rs += s[i];
      }
      l = l * alpha + rs;
      m = m_new;

      if (MODE == MODE_FWD) {
        if (j > 0) {
          // PV(j-1) done: the P buffer is free and O holds the sum so far.
          ok = mbar_wait(&c->o_done, (j - 1) & 1, &c->abort, a.spin_ns);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          if (__any_sync(0xffffffffu, alpha < 1.f)) {
#pragma unroll
            for (int q4 = 0; q4 < D / 32; ++q4) {
              uint32_t r[32];
              tmem_ld32(t_lane + 256 + q4 * 32, r);
              tmem_ld_wait();
              reg_fence(r);
#pragma unroll
              for (int i = 0; i < 32; ++i) r[i] = f2u(u2f(r[i]) * alpha);
              tmem_st32(t_lane + 256 + q4 * 32, r);
            }
            tmem_st_wait();
          }
        }
        // P row -> shared memory, 128-byte swizzle, two 64-column boxes.
#pragma unroll
        for (int cc = 0; cc < TILE / 8; ++cc) {
          const uint32_t addr = sP + (cc >> 3) * L::BOX_BYTES + row * 128 + (((cc & 7) ^ (row & 7)) << 4);
          st_shared_v4(addr, pack_bf16x2(s[8 * cc + 0], s[8 * cc + 1]), pack_bf16x2(s[8 * cc + 2], s[8 * cc + 3]),
                       pack_bf16x2(s[8 * cc + 4], s[8 * cc + 5]), pack_bf16x2(s[8 * cc + 6], s[8 * cc + 7]));
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&c->p_full);
      }
    }
    if (!ok) give_up(c, a.status);

    if (MODE == MODE_FWD) {
      bool have = ok && n > 0;
      if (have) {
        have = mbar_wait(&c->o_done, (n - 1) & 1, &c->abort, a.spin_ns);
        have = __all_sync(0xffffffffu, have);
        if (!have) give_up(c, a.status);
        tc_fence_after();
      }
      const bool zero = !have || grow >= a.N;
      const float inv_l = zero ? 0.f : 1.f / l;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.o) + (static_cast<size_t>(bh) * a.Np + grow) * D;
#pragma unroll
      for (int q4 = 0; q4 < D / 32; ++q4) {
        uint32_t r[32];
        if (have) {
          tmem_ld32(t_lane + 256 + q4 * 32, r);
          tmem_ld_wait();
          reg_fence(r);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = 0u;
        }
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
      if (a.lse != nullptr)
        a.lse[static_cast<size_t>(bh) * a.Np + grow] = zero ? -INFINITY : (m + log2f(l)) * 0.69314718055994531f;
    } else if (MODE == MODE_STATS) {
      a.lse2[static_cast<size_t>(h) * a.Np + grow] = (ok && grow < a.N) ? m + log2f(l) : -INFINITY;
    } else {
      // ENERGY: per key block, the four warp partials in a fixed order.
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (ok) {
        const int rows = min(TILE, a.N - qb * TILE);
        const float inv_rows = 1.f / static_cast<float>(rows);
        float* erow = a.energy + (static_cast<size_t>(h) * a.nqb + qb) * a.nkb;
        for (int j = row; j < n; j += TILE) {
          const float tot = ((part[4 * j + 0] + part[4 * j + 1]) + part[4 * j + 2]) + part[4 * j + 3];
          erow[j] = tot * inv_rows;
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
int launch_one(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const TcArgs& a, dim3 grid,
               cudaStream_t s) {
  auto kern = k_attn_tc<D, MODE>;
  static bool configured = false;
  if (!configured) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Layout<D>::SMEM_BYTES) !=
        cudaSuccess)
      return check_launch("cudaFuncSetAttribute(k_attn_tc)");
    configured = true;
  }
  kern<<<grid, kThreads, Layout<D>::SMEM_BYTES, s>>>(tq, tk, tv, a);
  count_launch();
  return check_launch("k_attn_tc");
}

}  // namespace

int launch_tc_fwd(const void* q, const void* k, const void* v, int d, const TcArgs& a, cudaStream_t s) {
  CUtensorMap tq, tk, tv;
  const uint64_t rows = static_cast<uint64_t>(a.B) * a.H * a.Np;
  int rc;
  if ((rc = make_tmap_bf16(&tq, q, rows, d)) != CALIBATT_OK) return rc;
  if ((rc = make_tmap_bf16(&tk, k, rows, d)) != CALIBATT_OK) return rc;
  if ((rc = make_tmap_bf16(&tv, v, rows, d)) != CALIBATT_OK) return rc;
  dim3 grid(a.nqb, a.H, a.B);
  if (d == 128) return launch_one<128, MODE_FWD>(tq, tk, tv, a, grid, s);
  return launch_one<64, MODE_FWD>(tq, tk, tv, a, grid, s);
}

int launch_tc_energy(const void* q, const void* k, int d, const TcArgs& a, cudaStream_t s) {
  CUtensorMap tq, tk;
  const uint64_t rows = static_cast<uint64_t>(a.H) * a.Np;
  int rc;
  if ((rc = make_tmap_bf16(&tq, q, rows, d)) != CALIBATT_OK) return rc;
  if ((rc = make_tmap_bf16(&tk, k, rows, d)) != CALIBATT_OK) return rc;
  dim3 grid(a.nqb, a.H, 1);
  if (d == 128) {
    if ((rc = launch_one<128, MODE_STATS>(tq, tk, tk, a, grid, s)) != CALIBATT_OK) return rc;
    return launch_one<128, MODE_ENERGY>(tq, tk, tk, a, grid, s);
  }
  if ((rc = launch_one<64, MODE_STATS>(tq, tk, tk, a, grid, s)) != CALIBATT_OK) return rc;
  return launch_one<64, MODE_ENERGY>(tq, tk, tk, a, grid, s);
}

}  // namespace calibatt
