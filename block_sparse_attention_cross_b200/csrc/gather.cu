// gather.cu -- row gather between sequence layouts.
//
// The spatial-repetition path of the paper page (Figure 4: attention patterns
// repeat across the spatial rows of a frame; Figure 5(b) bottom and Table S4:
// attention is computed for k anchor query rows per frame and its outputs are
// broadcast to the other rows) moves rows of [planes, rows, d] tensors: the
// anchor queries are gathered into a compact query tensor, and every token's
// output row is taken from its anchor's output row.  Both are
// dst[p, i, :] = src[p, idx[i], :]; an index outside [0, rows_src) gives a zero
// row (padding).
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace calibatt {
namespace {

__global__ void k_gather_rows(const uint4* __restrict__ src, uint4* __restrict__ dst, const int32_t* __restrict__ idx,
                              long long n_planes, int rows_src, int rows_dst, int vec_per_row) {
  const long long total = n_planes * rows_dst * static_cast<long long>(vec_per_row);
  for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int v = static_cast<int>(t % vec_per_row);
    const long long r = t / vec_per_row;
    const int i = static_cast<int>(r % rows_dst);
    const long long p = r / rows_dst;
    const int j = idx[i];
    uint4 x = make_uint4(0, 0, 0, 0);
    if (j >= 0 && j < rows_src) x = src[(p * rows_src + j) * vec_per_row + v];
    dst[r * vec_per_row + v] = x;
  }
}

}  // namespace
}  // namespace calibatt

using namespace calibatt;

extern "C" {

int calibatt_gather_rows(const void* src, void* dst, const int32_t* idx, int n_planes, int rows_src, int rows_dst,
                         int row_bytes, calibatt_stream_t stream) {
  if (src == nullptr || dst == nullptr || idx == nullptr)
    return set_error(CALIBATT_E_INVALID, "src, dst and idx must be non-NULL");
  if (n_planes <= 0 || rows_src <= 0 || rows_dst <= 0 || row_bytes <= 0 || row_bytes % 16 != 0)
    return set_error(CALIBATT_E_INVALID, "bad sizes (row_bytes must be a positive multiple of 16)");
  if ((reinterpret_cast<uintptr_t>(src) & 15u) || (reinterpret_cast<uintptr_t>(dst) & 15u))
    return set_error(CALIBATT_E_INVALID, "src and dst must be 16-byte aligned");
  const long long total = static_cast<long long>(n_planes) * rows_dst * (row_bytes / 16);
  const unsigned grid = static_cast<unsigned>(std::min<long long>((total + 255) / 256, 148ll * 16));
  k_gather_rows<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), idx, n_planes, rows_src, rows_dst, row_bytes / 16);
  count_launch();
  return check_launch("k_gather_rows");
}

}  // extern "C"
