// plan.cu -- index plans and storage sizes of the NEXT-row paths.
//
// Spatial repetition (paper page, Figure 4: attention repeats across the
// spatial rows of a frame; Figure 5(b) bottom and Table S4: attention is
// computed for k anchor rows per frame and broadcast to the other rows):
// which rows are anchors, which anchor every row takes its output from, and
// the two gather index lists of a video geometry.
//
// Interval skip lists (paper page, Figure S9, Figure S10 and Table S3): the
// per-layer widths of the padded interval arrays -- full (ceil(nkb / 2)
// intervals per row), trimmed to the layer's widest row, and merged to a
// nearest-rank percentile of the layer's interval counts -- and their bytes
// (one interval = an int32 pair).
#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace calibatt {
namespace {

// Anchor row i of k in a frame of `rows` spatial rows: floor((i + 1/2) rows / k),
// evenly spaced and centred, in exact integer arithmetic.
__host__ __device__ __forceinline__ int anchor_row(int i, int rows, int k) {
  return static_cast<int>((static_cast<long long>(2 * i + 1) * rows) / (2ll * k));
}

// The anchor slot a spatial row takes its output from: the nearest anchor,
// the lower one on a tie (anchors ascend with the slot, so the first slot at
// the smallest distance wins).
__host__ __device__ __forceinline__ int nearest_slot(int r, int rows, int k) {
  int best = 0, best_d = abs(anchor_row(0, rows, k) - r);
  for (int i = 1; i < k; ++i) {
    const int dd = abs(anchor_row(i, rows, k) - r);
    if (dd < best_d) {
      best = i;
      best_d = dd;
    }
  }
  return best;
}

// idx_q[i] (i < npq): source token of gathered query i (anchor rows of every
// frame, frame-major, then slot, then column), -1 for padding.
// idx_o[t] (t < Np): gathered row whose output token t takes, -1 for padding.
__global__ void k_anchor_plan(int frames, int rows, int cols, int k, int Np, int nq, int npq, int32_t* idx_q,
                              int32_t* idx_o) {
  const int N = frames * rows * cols;
  const int per_frame = k * cols;
  const int total = npq > Np ? npq : Np;
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < total; t += gridDim.x * blockDim.x) {
    if (t < npq) {
      int v = -1;
      if (t < nq) {
        const int f = t / per_frame, rem = t - f * per_frame;
        const int slot = rem / cols, c = rem - slot * cols;
        v = (f * rows + anchor_row(slot, rows, k)) * cols + c;
      }
      idx_q[t] = v;
    }
    if (t < Np) {
      int v = -1;
      if (t < N) {
        const int f = t / (rows * cols), rem = t - f * rows * cols;
        const int r = rem / cols, c = rem - r * cols;
        v = f * per_frame + nearest_slot(r, rows, k) * cols + c;
      }
      idx_o[t] = v;
    }
  }
}

// One CTA per layer: a histogram of the layer's interval counts in shared
// memory (integer atomics: exact), then the largest count and, for every
// requested rank, the smallest count with at least that many counts at or
// below it (nearest rank).  Per-map widths are written for the merge.
__global__ void k_skiplist_widths(const int32_t* __restrict__ counts, int rows_per_layer, int maps_per_layer,
                                  int n_layers, int nbins, const long long* __restrict__ ranks, int n_pcts,
                                  int32_t* layer_max, int32_t* layer_width, int32_t* map_width, int n_maps) {
  extern __shared__ int hist[];
  __shared__ int widths[64];
  const int l = blockIdx.x;
  for (int b = threadIdx.x; b < nbins; b += blockDim.x) hist[b] = 0;
  __syncthreads();
  const int32_t* c = counts + static_cast<long long>(l) * rows_per_layer;
  for (int i = threadIdx.x; i < rows_per_layer; i += blockDim.x) {
    const int v = c[i];
    atomicAdd(&hist[v < 0 ? 0 : (v >= nbins ? nbins - 1 : v)], 1);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int mx = 0;
    for (int b = nbins - 1; b >= 0; --b)
      if (hist[b] > 0) {
        mx = b;
        break;
      }
    layer_max[l] = mx;
    for (int p = 0; p < n_pcts; ++p) {
      long long cum = 0;
      int w = mx;
      for (int b = 0; b < nbins; ++b) {
        cum += hist[b];
        if (cum >= ranks[p]) {
          w = b;
          break;
        }
      }
      widths[p] = w;
      layer_width[p * n_layers + l] = w;
    }
  }
  __syncthreads();
  if (map_width != nullptr) {
    for (int i = threadIdx.x; i < n_pcts * maps_per_layer; i += blockDim.x) {
      const int p = i / maps_per_layer, m = i - p * maps_per_layer;
      map_width[static_cast<long long>(p) * n_maps + l * maps_per_layer + m] = widths[p];
    }
  }
}

// Sum of the pattern lengths of rows [r0, r1): the kept blocks of those rows.
__global__ void k_rows_kept(const int32_t* __restrict__ row_pat, const int32_t* __restrict__ pat_ptr, long long r0,
                            long long r1, unsigned long long* out) {
  __shared__ unsigned long long part[8];
  unsigned long long acc = 0;
  for (long long r = r0 + static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; r < r1;
       r += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int p = row_pat[r];
    acc += static_cast<unsigned long long>(pat_ptr[p + 1] - pat_ptr[p]);
  }
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long t = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t += part[w];
    atomicAdd(out, t);
  }
}

constexpr int kMaxPcts = 64;
constexpr int kMaxSkipKeyBlocks = 16384;   // histogram of <= 8193 bins in shared memory

int cuda_ok(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return CALIBATT_OK;
  return set_error(CALIBATT_E_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

size_t skiplist_ws_bytes(int n_layers, int n_pcts) {
  return 256 + ((static_cast<size_t>(n_layers) * (1 + n_pcts) * 4 + 255) & ~size_t(255)) + 8 * kMaxPcts;
}

}  // namespace
}  // namespace calibatt

using namespace calibatt;

extern "C" {

int calibatt_anchor_rows(int rows, int k, int32_t* anchors, int32_t* nearest) {
  if (anchors == nullptr || nearest == nullptr) return set_error(CALIBATT_E_INVALID, "anchors and nearest are NULL");
  if (rows <= 0 || k <= 0 || k > rows) return set_error(CALIBATT_E_INVALID, "need 1 <= k <= rows (rows=%d k=%d)", rows, k);
  for (int i = 0; i < k; ++i) anchors[i] = anchor_row(i, rows, k);
  for (int r = 0; r < rows; ++r) nearest[r] = anchor_row(nearest_slot(r, rows, k), rows, k);
  return CALIBATT_OK;
}

int calibatt_anchor_plan_size(int frames, int rows, int cols, int k, int* nq, int* npq) {
  if (nq == nullptr || npq == nullptr) return set_error(CALIBATT_E_INVALID, "nq and npq are NULL");
  if (frames <= 0 || rows <= 0 || cols <= 0 || k <= 0 || k > rows)
    return set_error(CALIBATT_E_INVALID, "bad geometry frames=%d rows=%d cols=%d k=%d", frames, rows, cols, k);
  const long long n = static_cast<long long>(frames) * k * cols;
  const long long np = (n + 127) / 128 * 128;
  if (np >= (1ll << 31)) return set_error(CALIBATT_E_UNSUPPORTED, "too many anchor tokens");
  *nq = static_cast<int>(n);
  *npq = static_cast<int>(np);
  return CALIBATT_OK;
}

int calibatt_anchor_plan(int frames, int rows, int cols, int k, int Np, int32_t* idx_q, int32_t* idx_o,
                         calibatt_stream_t stream) {
  int nq = 0, npq = 0;
  int rc = calibatt_anchor_plan_size(frames, rows, cols, k, &nq, &npq);
  if (rc) return rc;
  if (idx_q == nullptr || idx_o == nullptr) return set_error(CALIBATT_E_INVALID, "idx_q and idx_o are NULL");
  const long long N = static_cast<long long>(frames) * rows * cols;
  if (Np < N || N >= (1ll << 31)) return set_error(CALIBATT_E_INVALID, "Np=%d is below the %lld video tokens", Np, N);
  const int total = std::max(npq, Np);
  const unsigned grid = static_cast<unsigned>(std::min<long long>((total + 255) / 256, 148ll * 8));
  k_anchor_plan<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(frames, rows, cols, k, Np, nq, npq, idx_q,
                                                                          idx_o);
  count_launch();
  return check_launch("k_anchor_plan");
}

int calibatt_skiplist_sizes_workspace_size(int n_maps, int maps_per_layer, int n_pcts, size_t* bytes) {
  if (bytes == nullptr) return set_error(CALIBATT_E_INVALID, "bytes is NULL");
  if (n_maps <= 0 || maps_per_layer <= 0 || n_maps % maps_per_layer || n_pcts < 0 || n_pcts > kMaxPcts)
    return set_error(CALIBATT_E_INVALID, "bad sizes");
  *bytes = skiplist_ws_bytes(n_maps / maps_per_layer, n_pcts);
  return CALIBATT_OK;
}

int calibatt_skiplist_sizes(const int32_t* counts, int n_maps, int nqb, int nkb, int maps_per_layer,
                            const double* pcts, int n_pcts, int32_t* layer_max, int32_t* layer_width,
                            int32_t* map_width, int64_t* bytes, void* workspace, size_t workspace_bytes,
                            calibatt_stream_t stream) {
  if (counts == nullptr || layer_max == nullptr || bytes == nullptr || (n_pcts > 0 && (pcts == nullptr || layer_width == nullptr)))
    return set_error(CALIBATT_E_INVALID, "NULL argument");
  if (n_maps <= 0 || nqb <= 0 || nkb <= 0 || nkb > kMaxSkipKeyBlocks || maps_per_layer <= 0 ||
      n_maps % maps_per_layer || n_pcts < 0 || n_pcts > kMaxPcts)
    return set_error(CALIBATT_E_INVALID, "bad sizes (n_maps a multiple of maps_per_layer, nkb <= %d, <= %d pcts)",
                     kMaxSkipKeyBlocks, kMaxPcts);
  const int n_layers = n_maps / maps_per_layer;
  const long long rows_per_layer = static_cast<long long>(maps_per_layer) * nqb;
  if (rows_per_layer >= (1ll << 31)) return set_error(CALIBATT_E_UNSUPPORTED, "too many rows per layer");
  if (workspace == nullptr || workspace_bytes < skiplist_ws_bytes(n_layers, n_pcts))
    return set_error(CALIBATT_E_WORKSPACE, "workspace too small: need %zu bytes", skiplist_ws_bytes(n_layers, n_pcts));
  // Nearest rank of every percentile: ceil(pct / 100 * n), at least 1.
  long long ranks[kMaxPcts];
  for (int p = 0; p < n_pcts; ++p) {
    if (!(pcts[p] > 0.0) || pcts[p] > 100.0) return set_error(CALIBATT_E_INVALID, "percentiles must be in (0, 100]");
    ranks[p] = std::max(1ll, static_cast<long long>(std::ceil(pcts[p] / 100.0 * static_cast<double>(rows_per_layer))));
  }
  char* base = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(workspace) + 255) & ~uintptr_t(255));
  int32_t* d_max = reinterpret_cast<int32_t*>(base);
  int32_t* d_width = d_max + n_layers;
  long long* d_ranks = reinterpret_cast<long long*>(base + ((static_cast<size_t>(n_layers) * (1 + n_pcts) * 4 + 255) & ~size_t(255)));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int rc;
  if (n_pcts > 0 &&
      (rc = cuda_ok(cudaMemcpyAsync(d_ranks, ranks, sizeof(long long) * n_pcts, cudaMemcpyHostToDevice, s), "ranks")))
    return rc;
  const int nbins = (nkb + 1) / 2 + 1;
  const size_t smem = static_cast<size_t>(nbins) * sizeof(int);
  k_skiplist_widths<<<n_layers, 256, smem, s>>>(counts, static_cast<int>(rows_per_layer), maps_per_layer, n_layers, nbins,
                                                d_ranks, n_pcts, d_max, d_width, map_width, n_maps);
  count_launch();
  if ((rc = check_launch("k_skiplist_widths"))) return rc;
  if ((rc = cuda_ok(cudaMemcpyAsync(layer_max, d_max, sizeof(int32_t) * n_layers, cudaMemcpyDeviceToHost, s), "max")))
    return rc;
  if (n_pcts > 0 && (rc = cuda_ok(cudaMemcpyAsync(layer_width, d_width, sizeof(int32_t) * n_layers * n_pcts,
                                                 cudaMemcpyDeviceToHost, s), "widths")))
    return rc;
  if ((rc = cuda_ok(cudaStreamSynchronize(s), "cudaStreamSynchronize"))) return rc;
  // Bytes: one interval = two int32 (8 bytes) per slot, rows_per_layer rows per layer.
  const long long row_bytes = 8;
  bytes[0] = static_cast<long long>(n_layers) * rows_per_layer * ((nkb + 1) / 2) * row_bytes;
  long long trimmed = 0;
  for (int l = 0; l < n_layers; ++l) trimmed += static_cast<long long>(layer_max[l]) * rows_per_layer * row_bytes;
  bytes[1] = trimmed;
  for (int p = 0; p < n_pcts; ++p) {
    long long merged = 0;
    for (int l = 0; l < n_layers; ++l) merged += static_cast<long long>(layer_width[p * n_layers + l]) * rows_per_layer * row_bytes;
    bytes[2 + p] = merged;
  }
  return CALIBATT_OK;
}

int calibatt_min_votes(double rho, int n_inputs, int32_t* min_votes) {
  if (min_votes == nullptr) return set_error(CALIBATT_E_INVALID, "min_votes is NULL");
  if (n_inputs <= 0 || !std::isfinite(rho)) return set_error(CALIBATT_E_INVALID, "bad rho or input count");
  // ceil(rho I), after rounding rho I to 9 decimals so that a product such as
  // 0.3 * 10 = 3.0000000000000004 counts as 3
  const double v = std::nearbyint(rho * n_inputs * 1e9) / 1e9;
  double c = std::ceil(v);
  if (c < 0) c = 0;
  if (c > n_inputs) c = n_inputs;
  *min_votes = static_cast<int32_t>(c);
  return CALIBATT_OK;
}

int calibatt_topk_count(double frac, int nkb, int32_t* k) {
  if (k == nullptr) return set_error(CALIBATT_E_INVALID, "k is NULL");
  if (nkb <= 0 || !(frac > 0.0) || frac > 1.0) return set_error(CALIBATT_E_INVALID, "need 0 < frac <= 1, nkb > 0");
  double v = std::ceil(frac * nkb);
  if (v < 1) v = 1;
  if (v > nkb) v = nkb;
  *k = static_cast<int32_t>(v);
  return CALIBATT_OK;
}

int calibatt_blocklist_bytes(int n_maps, int nqb, int64_t nnz, int32_t n_pat, int32_t nnz_pat, int64_t* csr_bytes,
                             int64_t* pool_bytes) {
  if (csr_bytes == nullptr || pool_bytes == nullptr) return set_error(CALIBATT_E_INVALID, "NULL outputs");
  if (n_maps <= 0 || nqb <= 0 || nnz < 0 || n_pat <= 0 || nnz_pat < 0) return set_error(CALIBATT_E_INVALID, "bad sizes");
  const long long rows = static_cast<long long>(n_maps) * nqb;
  *csr_bytes = (rows + 1) * 8 + nnz * 2;                             // int64 row_ptr + int16 col
  *pool_bytes = rows * 8 + (static_cast<long long>(n_pat) + 1) * 4 + static_cast<long long>(nnz_pat) * 2;
  return CALIBATT_OK;
}

int calibatt_blocklist_kept(const calibatt_blocklist* bl, int map_offset, int n_maps, int64_t* kept, void* workspace,
                            size_t workspace_bytes, calibatt_stream_t stream) {
  if (bl == nullptr || kept == nullptr || bl->row_pat == nullptr || bl->pat_ptr == nullptr)
    return set_error(CALIBATT_E_INVALID, "NULL argument");
  if (map_offset < 0 || n_maps <= 0 || static_cast<long long>(map_offset) + n_maps > bl->n_maps)
    return set_error(CALIBATT_E_INVALID, "maps [%d, %d) outside the list's %d maps", map_offset, map_offset + n_maps,
                     bl->n_maps);
  if (workspace == nullptr || workspace_bytes < 8) return set_error(CALIBATT_E_WORKSPACE, "need 8 bytes of workspace");
  if (reinterpret_cast<uintptr_t>(workspace) & 7u) return set_error(CALIBATT_E_INVALID, "workspace must be 8-byte aligned");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned long long* d = static_cast<unsigned long long*>(workspace);
  int rc;
  if ((rc = cuda_ok(cudaMemsetAsync(d, 0, 8, s), "cudaMemsetAsync"))) return rc;
  const long long r0 = static_cast<long long>(map_offset) * bl->n_q_blocks;
  const long long r1 = r0 + static_cast<long long>(n_maps) * bl->n_q_blocks;
  const unsigned grid = static_cast<unsigned>(std::min<long long>((r1 - r0 + 255) / 256, 148ll * 4));
  k_rows_kept<<<grid, 256, 0, s>>>(bl->row_pat, bl->pat_ptr, r0, r1, d);
  count_launch();
  if ((rc = check_launch("k_rows_kept"))) return rc;
  unsigned long long h = 0;
  if ((rc = cuda_ok(cudaMemcpyAsync(&h, d, 8, cudaMemcpyDeviceToHost, s), "cudaMemcpyAsync")) ||
      (rc = cuda_ok(cudaStreamSynchronize(s), "cudaStreamSynchronize")))
    return rc;
  *kept = static_cast<int64_t>(h);
  return CALIBATT_OK;
}

}  // extern "C"
