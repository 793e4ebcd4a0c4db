// noalloc.cu -- block energies for callers that cannot allocate device memory.
//
// calibatt_block_energy needs a per-row log-sum-exp scratch buffer between
// its two passes, which the caller normally provides as workspace.  Some
// callers have no way to provide it: a plugin that its host engine hands
// only input and output buffers, or a service that reserved all of the GPU's
// memory for its own pool at start-up and allows no allocation afterwards.
// For them this file keeps that scratch in a fixed-size array in the
// library's own device memory, so the call needs nothing but q, k and the
// energy output.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds it (kNoallocScratchFloats floats, 16 MiB) until the process
// exits.  All calls share it, so calls that overlap on the GPU (different
// streams, or different host threads on the same device) race on it; calls
// on one stream are ordered and safe.  The first pass of every call writes
// each scratch entry it later reads, so nothing needs clearing between calls.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace calibatt {
namespace {

constexpr long long kNoallocScratchFloats = 4ll * 1024 * 1024;  // 16 MiB: H * Np <= 4 Mi rows

static __device__ __align__(256) float g_noalloc_scratch[kNoallocScratchFloats];

std::mutex g_noalloc_mutex;
float* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  Host code may
// not use the array's name as an address (it is a host-side stand-in), so the
// address is looked up once per device, with that device current.
int scratch_for_current_device(float** out) {
  int dev = -1;
  if (int rc = current_device(&dev)) return rc;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return set_error(CALIBATT_E_CUDA, "cudaGetSymbolAddress(scratch) failed: %s", cudaGetErrorString(e));
    }
    g_noalloc_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return CALIBATT_OK;
}

}  // namespace
}  // namespace calibatt

using namespace calibatt;

// Same validation and launch path as calibatt_block_energy; only the source
// of the per-row scratch differs.
extern "C" int calibatt_block_energy_noalloc(const void* q, const void* k, int H, int N, int Np, int d, int dtype,
                                             int block_q, int block_k, float scale, float* energy_out,
                                             int32_t* dev_status, calibatt_stream_t stream) {
  int rc = check_energy_args(q, k, H, N, Np, d, dtype, block_q, block_k, scale);
  if (rc) return rc;
  if (energy_out == nullptr) return set_error(CALIBATT_E_INVALID, "energy_out is NULL");
  if (static_cast<long long>(H) * Np > kNoallocScratchFloats)
    return set_error(CALIBATT_E_WORKSPACE,
                     "H * Np = %lld rows exceeds the built-in scratch of %lld rows; use calibatt_block_energy "
                     "with a workspace",
                     static_cast<long long>(H) * Np, kNoallocScratchFloats);
  float* scratch = nullptr;
  if ((rc = scratch_for_current_device(&scratch))) return rc;
  return energy_impl(q, k, H, N, Np, d, dtype, block_q, block_k, scale, energy_out, scratch, dev_status,
                     reinterpret_cast<cudaStream_t>(stream));
}
