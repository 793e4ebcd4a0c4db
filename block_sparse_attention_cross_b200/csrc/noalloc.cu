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
#include <cmath>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace calibatt {
namespace {

constexpr long long kNoallocScratchFloats = 4ll * 1024 * 1024;  // 16 MiB: H * Np <= 4 Mi rows
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_noalloc_scratch[kNoallocScratchFloats];

std::mutex g_noalloc_mutex;
float* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  Host code may
// not use the array's name as an address (it is a host-side stand-in), so the
// address is looked up once per device, with that device current.
int scratch_for_current_device(float** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return check_launch("cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return set_error(CALIBATT_E_UNSUPPORTED, "device ordinal %d out of range", dev);
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

extern "C" int calibatt_block_energy_noalloc(const void* q, const void* k, int H, int N, int Np, int d, int dtype,
                                             int block_q, int block_k, float scale, float* energy_out,
                                             int32_t* dev_status, calibatt_stream_t stream) {
  if (q == nullptr || k == nullptr || energy_out == nullptr)
    return set_error(CALIBATT_E_INVALID, "q, k and energy_out must be non-NULL");
  if (H <= 0 || N <= 0 || Np < N || d <= 0 || block_q <= 0 || block_k <= 0 || Np % block_q || Np % block_k)
    return set_error(CALIBATT_E_INVALID, "bad sizes H=%d N=%d Np=%d d=%d", H, N, Np, d);
  if ((Np - N) >= block_k || (Np - N) >= block_q)
    return set_error(CALIBATT_E_INVALID, "Np - N must be smaller than one block");
  if (!(scale > 0.f) || !std::isfinite(scale)) return set_error(CALIBATT_E_INVALID, "scale must be finite and > 0");
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k)) & 15u)
    return set_error(CALIBATT_E_INVALID, "q and k must be 16-byte aligned");
  if (static_cast<long long>(H) * Np > kNoallocScratchFloats)
    return set_error(CALIBATT_E_WORKSPACE,
                     "H * Np = %lld rows exceeds the built-in scratch of %lld rows; use calibatt_block_energy "
                     "with a workspace",
                     static_cast<long long>(H) * Np, kNoallocScratchFloats);
  const int nqb = Np / block_q, nkb = Np / block_k;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == CALIBATT_BF16) {
    if (!(d == 64 || d == 128) || block_q != 128 || block_k != 128)
      return set_error(CALIBATT_E_UNSUPPORTED, "bf16 energies support d in {64,128} with 128x128 blocks");
    if (nkb > 1024) return set_error(CALIBATT_E_UNSUPPORTED, "at most 1024 key blocks");
  } else if (dtype == CALIBATT_FP32) {
    if (!(d == 64 || d == 128) || !(block_q == 64 || block_q == 128) || !(block_k == 64 || block_k == 128))
      return set_error(CALIBATT_E_UNSUPPORTED, "fp32 energies support d in {64,128}, blocks in {64,128}");
  } else {
    return set_error(CALIBATT_E_UNSUPPORTED, "unknown dtype %d", dtype);
  }
  float* scratch = nullptr;
  int rc = scratch_for_current_device(&scratch);
  if (rc) return rc;
  if (dtype == CALIBATT_BF16) {
    TcArgs a{};
    a.B = 1; a.H = H; a.N = N; a.Np = Np; a.nqb = nqb; a.nkb = nkb;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.lse2 = scratch; a.energy = energy_out; a.status = dev_status; a.spin_ns = spin_limit_ns();
    return launch_tc_energy(q, k, d, a, s);
  }
  SimtArgs a{};
  a.B = 1; a.H = H; a.N = N; a.Np = Np; a.block_q = block_q; a.block_k = block_k; a.nqb = nqb; a.nkb = nkb;
  a.scale = scale; a.lse = scratch; a.energy = energy_out; a.status = dev_status;
  return launch_simt_energy(q, k, d, a, s);
}
