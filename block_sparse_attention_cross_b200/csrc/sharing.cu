// sharing.cu -- timestep sharing of calibrated masks.
//
// CalibAtt calibrates one block mask per (layer, head, timestep).  Its paper
// page notes that masks of consecutive late denoising steps are alike
// (Figure S11: intersection-over-union of the skipped-block masks of two
// timesteps, averaged over layers and heads) and shares masks across
// timesteps whose pair-wise IoU is at least tau (Table S3), which shrinks the
// stored dictionary.  Here, per layer, the similarity of two timesteps is
// the mean over heads of the IoU of their skipped-block sets; consecutive
// timesteps are grouped greedily in time order while every pair of a group
// stays at or above tau; each group stores the union of its members' kept
// blocks, so nothing any member keeps is skipped.
//
// Mask layout: [L, T, H, nqb, nkb] uint8 (nonzero = kept), the dictionary
// order map = (l T + t) H + h.  The pair counts are integers, so the
// clustering is exact and independent of summation order.
#include <algorithm>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace calibatt {
namespace {

constexpr int kThreadsPair = 256;
constexpr int kMaxSteps = 1024;

// Counts of blocks skipped in both / in either of the masks of (l, t1, h) and
// (l, t2, h), for every t2 > t1 (and the skipped count on the diagonal).
// One CTA per (l, h, t1).  Output [L][H][T][T] int64, both triangles.
__global__ void __launch_bounds__(kThreadsPair) k_pair_counts(const uint8_t* __restrict__ masks, int T, int H,
                                                             long long nb, long long* inter, long long* uni) {
  const int t1 = blockIdx.x % T;
  const int lh = blockIdx.x / T;
  const int h = lh % H;
  const int l = lh / H;
  const uint8_t* m1 = masks + (static_cast<size_t>(l * T + t1) * H + h) * nb;
  __shared__ long long red[2][kThreadsPair / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  long long* base_i = inter + static_cast<size_t>(lh) * T * T;
  long long* base_u = uni + static_cast<size_t>(lh) * T * T;
  for (int t2 = t1; t2 < T; ++t2) {
    const uint8_t* m2 = masks + (static_cast<size_t>(l * T + t2) * H + h) * nb;
    long long ci = 0, cu = 0;
    for (long long p = threadIdx.x; p < nb; p += blockDim.x) {
      const bool s1 = m1[p] == 0, s2 = m2[p] == 0;
      ci += (s1 && s2) ? 1 : 0;
      cu += (s1 || s2) ? 1 : 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      ci += __shfl_xor_sync(0xffffffffu, ci, o);
      cu += __shfl_xor_sync(0xffffffffu, cu, o);
    }
    if (lane == 0) {
      red[0][warp] = ci;
      red[1][warp] = cu;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      long long si = 0, su = 0;
      for (int w = 0; w < kThreadsPair / 32; ++w) {
        si += red[0][w];
        su += red[1][w];
      }
      base_i[t1 * T + t2] = si;
      base_u[t1 * T + t2] = su;
      base_i[t2 * T + t1] = si;
      base_u[t2 * T + t1] = su;
    }
    __syncthreads();
  }
}

// Union of the kept blocks of every member of a run: one CTA per (run, head)
// and chunk of positions.  run_of[l T + t] is the global run index; the
// members of run r are the (l, t) with run_of == r.
__global__ void k_share_masks(const uint8_t* __restrict__ masks, int L, int T, int H, long long nb,
                              const int32_t* __restrict__ run_of, uint8_t* shared) {
  const int r = blockIdx.y / H;
  const int h = blockIdx.y % H;
  __shared__ int first, last;
  if (threadIdx.x == 0) {
    first = -1;
    last = -1;
    for (int i = 0; i < L * T; ++i) {
      if (run_of[i] == r) {
        if (first < 0) first = i;
        last = i;
      }
    }
  }
  __syncthreads();
  uint8_t* out = shared + (static_cast<size_t>(r) * H + h) * nb;
  for (long long p = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; p < nb;
       p += static_cast<long long>(gridDim.x) * blockDim.x) {
    uint8_t v = 0;
    for (int i = first; i >= 0 && i <= last; ++i)
      if (run_of[i] == r && masks[(static_cast<size_t>(i) * H + h) * nb + p] != 0) v = 1;
    out[p] = v;
  }
}

size_t counts_bytes(int L, int T, int H) { return 2 * static_cast<size_t>(L) * H * T * T * sizeof(long long); }

int check_dims(const uint8_t* masks, int L, int T, int H, int nqb, int nkb) {
  if (masks == nullptr) return set_error(CALIBATT_E_INVALID, "masks is NULL");
  if (L <= 0 || T <= 0 || H <= 0 || nqb <= 0 || nkb <= 0)
    return set_error(CALIBATT_E_INVALID, "bad sizes L=%d T=%d H=%d nqb=%d nkb=%d", L, T, H, nqb, nkb);
  if (T > kMaxSteps) return set_error(CALIBATT_E_UNSUPPORTED, "at most %d timesteps", kMaxSteps);
  if (static_cast<long long>(L) * T > (1ll << 20)) return set_error(CALIBATT_E_UNSUPPORTED, "L*T too large");
  return CALIBATT_OK;
}

}  // namespace
}  // namespace calibatt

using namespace calibatt;

extern "C" {

int calibatt_timestep_clusters_workspace_size(int L, int T, int H, size_t* bytes) {
  if (bytes == nullptr) return set_error(CALIBATT_E_INVALID, "bytes is NULL");
  if (L <= 0 || T <= 0 || H <= 0) return set_error(CALIBATT_E_INVALID, "bad sizes");
  *bytes = counts_bytes(L, T, H);
  return CALIBATT_OK;
}

int calibatt_timestep_clusters(const uint8_t* masks, int L, int T, int H, int nqb, int nkb, double tau,
                               int32_t* run_of, int32_t* n_runs, void* workspace, size_t workspace_bytes,
                               calibatt_stream_t stream) {
  int rc = check_dims(masks, L, T, H, nqb, nkb);
  if (rc) return rc;
  if (run_of == nullptr || n_runs == nullptr) return set_error(CALIBATT_E_INVALID, "run_of and n_runs must be non-NULL");
  if (!(tau == tau)) return set_error(CALIBATT_E_INVALID, "tau is NaN");
  const size_t need = counts_bytes(L, T, H);
  if (workspace == nullptr || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return set_error(CALIBATT_E_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned", need);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  long long* inter = static_cast<long long*>(workspace);
  long long* uni = inter + static_cast<size_t>(L) * H * T * T;
  const long long nb = static_cast<long long>(nqb) * nkb;
  k_pair_counts<<<static_cast<unsigned>(static_cast<long long>(L) * H * T), kThreadsPair, 0, s>>>(masks, T, H, nb,
                                                                                                   inter, uni);
  count_launch();
  if ((rc = check_launch("k_pair_counts"))) return rc;
  std::vector<long long> hi(static_cast<size_t>(L) * H * T * T), hu(hi.size());
  if (cudaMemcpyAsync(hi.data(), inter, hi.size() * sizeof(long long), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaMemcpyAsync(hu.data(), uni, hu.size() * sizeof(long long), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return check_launch("copying the pair counts");
  // Mean over heads of the skipped-block IoU; both masks skipping nothing
  // count as identical (IoU 1).
  auto sim = [&](int l, int t1, int t2) {
    double acc = 0.0;
    for (int h = 0; h < H; ++h) {
      const size_t i = ((static_cast<size_t>(l) * H + h) * T + t1) * T + t2;
      acc += hu[i] == 0 ? 1.0 : static_cast<double>(hi[i]) / static_cast<double>(hu[i]);
    }
    return acc / H;
  };
  int next = 0;
  for (int l = 0; l < L; ++l) {
    int start = 0;
    run_of[l * T] = next;
    for (int t = 1; t < T; ++t) {
      bool join = true;
      for (int u = start; u < t && join; ++u) join = sim(l, t, u) >= tau;
      if (!join) {
        ++next;
        start = t;
      }
      run_of[l * T + t] = next;
    }
    ++next;
  }
  *n_runs = next;
  return CALIBATT_OK;
}

int calibatt_share_masks(const uint8_t* masks, int L, int T, int H, int nqb, int nkb, const int32_t* run_of_dev,
                         int n_runs, uint8_t* shared, calibatt_stream_t stream) {
  int rc = check_dims(masks, L, T, H, nqb, nkb);
  if (rc) return rc;
  if (run_of_dev == nullptr || shared == nullptr) return set_error(CALIBATT_E_INVALID, "run_of and shared must be non-NULL");
  if (n_runs <= 0 || n_runs > L * T) return set_error(CALIBATT_E_INVALID, "n_runs %d out of range", n_runs);
  if (static_cast<long long>(n_runs) * H > 65535) return set_error(CALIBATT_E_UNSUPPORTED, "n_runs * H too large");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long nb = static_cast<long long>(nqb) * nkb;
  const unsigned chunks = static_cast<unsigned>(std::min<long long>((nb + 255) / 256, 64));
  k_share_masks<<<dim3(chunks, static_cast<unsigned>(n_runs * H)), 256, 0, s>>>(masks, L, T, H, nb, run_of_dev, shared);
  count_launch();
  return check_launch("k_share_masks");
}

}  // extern "C"
