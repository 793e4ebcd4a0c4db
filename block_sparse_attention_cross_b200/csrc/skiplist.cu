// skiplist.cu -- the paper page's interval skip-list view of a mask dictionary.
//
// The paper page stores each layer's masks as a padded 2-D array with one row
// per (timestep, head, query block) holding interval pairs (Figure S10);
// Figure S9 counts intervals per row, and Figure S10 / Table S3 shrink a
// layer's padded width by trimming it to the widest row and by merging
// outlier rows.  This build computes attention from its own CSR / pattern
// pool; these kernels give the interval counts of every row (maximal runs of
// consecutive kept key blocks) and perform the merge: a row with more than
// the layer's width of intervals gets its smallest gaps (runs of skipped
// blocks between two kept blocks; ties to the leftmost) filled -- those
// blocks are then computed too -- until the width is met.
#include "common.cuh"
#include "internal.h"

namespace calibatt {
namespace {

constexpr int kMaxKeyBlocks = 2048;
constexpr int kMergeWarps = 4;

// One warp per row: ballot the kept bits 32 blocks at a time; a run starts
// where a kept block follows a skipped one (or the row start).
__global__ void k_interval_counts(const uint8_t* __restrict__ masks, long long rows, int nkb, int32_t* counts) {
  const long long row = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint8_t* m = masks + row * nkb;
  uint32_t prev_top = 0;
  int count = 0;
  for (int k0 = 0; k0 < nkb; k0 += 32) {
    const int kb = k0 + lane;
    const uint32_t v = __ballot_sync(0xffffffffu, kb < nkb && m[kb] != 0);
    const uint32_t starts = v & ~((v << 1) | prev_top);
    count += __popc(starts);
    prev_top = v >> 31;
  }
  if (lane == 0) counts[row] = count;
}

// One warp per row.  Lane 0 lists the row's gaps in shared memory; then, as
// many times as the row has intervals beyond its width, the warp finds the
// smallest unfilled gap (key = length, start) and fills it.
__global__ void k_merge_intervals(uint8_t* masks, long long rows, int nqb, int nkb, const int32_t* __restrict__ width,
                                  unsigned long long* filled) {
  __shared__ int g_start[kMergeWarps][kMaxKeyBlocks / 2];
  __shared__ int g_len[kMergeWarps][kMaxKeyBlocks / 2];
  const int w = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * kMergeWarps + w;
  if (row >= rows) return;
  uint8_t* m = masks + row * nkb;
  int n_gaps = 0, any = 0;
  if (lane == 0) {
    int last_kept = -1;
    for (int kb = 0; kb < nkb; ++kb) {
      if (m[kb] != 0) {
        if (last_kept >= 0 && kb > last_kept + 1) {
          g_start[w][n_gaps] = last_kept + 1;
          g_len[w][n_gaps] = kb - last_kept - 1;
          ++n_gaps;
        }
        last_kept = kb;
      }
    }
    any = last_kept >= 0;
  }
  n_gaps = __shfl_sync(0xffffffffu, n_gaps, 0);
  any = __shfl_sync(0xffffffffu, any, 0);
  __syncwarp();
  const int map = static_cast<int>(row / nqb);
  const int wd = width[map] < 1 ? 1 : width[map];
  const int excess = any ? n_gaps + 1 - wd : 0;
  unsigned long long done = 0;
  for (int e = 0; e < excess; ++e) {
    unsigned long long best = ~0ull;
    for (int i = lane; i < n_gaps; i += 32) {
      const int len = g_len[w][i];
      if (len > 0) {
        const unsigned long long key = (static_cast<unsigned long long>(len) << 32) | static_cast<unsigned>(g_start[w][i]);
        best = key < best ? key : best;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
      best = other < best ? other : best;
    }
    const int start = static_cast<int>(best & 0xffffffffu);
    const int len = static_cast<int>(best >> 32);
    for (int p = start + lane; p < start + len; p += 32) m[p] = 1;
    // retire the gap (its start is unique among the row's gaps)
    for (int i = lane; i < n_gaps; i += 32)
      if (g_start[w][i] == start) g_len[w][i] = 0;
    __syncwarp();
    done += static_cast<unsigned long long>(len);
  }
  if (lane == 0 && done > 0) atomicAdd(filled, done);
}

}  // namespace
}  // namespace calibatt

using namespace calibatt;

extern "C" {

int calibatt_interval_counts(const uint8_t* masks, int n_maps, int nqb, int nkb, int32_t* counts,
                             calibatt_stream_t stream) {
  if (masks == nullptr || counts == nullptr) return set_error(CALIBATT_E_INVALID, "masks and counts must be non-NULL");
  if (n_maps <= 0 || nqb <= 0 || nkb <= 0) return set_error(CALIBATT_E_INVALID, "bad sizes");
  const long long rows = static_cast<long long>(n_maps) * nqb;
  const unsigned grid = static_cast<unsigned>((rows + 7) / 8);
  k_interval_counts<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(masks, rows, nkb, counts);
  count_launch();
  return check_launch("k_interval_counts");
}

int calibatt_merge_intervals(uint8_t* masks, int n_maps, int nqb, int nkb, const int32_t* width,
                             unsigned long long* filled, calibatt_stream_t stream) {
  if (masks == nullptr || width == nullptr || filled == nullptr)
    return set_error(CALIBATT_E_INVALID, "masks, width and filled must be non-NULL");
  if (n_maps <= 0 || nqb <= 0 || nkb <= 0) return set_error(CALIBATT_E_INVALID, "bad sizes");
  if (nkb > kMaxKeyBlocks) return set_error(CALIBATT_E_UNSUPPORTED, "at most %d key blocks per row", kMaxKeyBlocks);
  const long long rows = static_cast<long long>(n_maps) * nqb;
  const unsigned grid = static_cast<unsigned>((rows + kMergeWarps - 1) / kMergeWarps);
  k_merge_intervals<<<grid, kMergeWarps * 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(masks, rows, nqb, nkb,
                                                                                           width, filled);
  count_launch();
  return check_launch("k_merge_intervals");
}

}  // extern "C"
