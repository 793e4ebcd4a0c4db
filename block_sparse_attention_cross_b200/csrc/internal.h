// internal.h -- host-side declarations shared by the calibatt translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "calibatt.h"

namespace calibatt {

// Error reporting (thread-local text behind calibatt_last_error).
int set_error(int code, const char* fmt, ...);
int check_launch(const char* what);   // cudaGetLastError -> status
void count_launch(int n = 1);
uint64_t spin_limit_ns();

// One-time launch set-up (dynamic shared-memory limits, SM counts, symbol
// addresses) is a per-device property: it is kept per device ordinal.
constexpr int kMaxDevices = 64;
// The current device's ordinal, checked against kMaxDevices.
int current_device(int* dev);

// Kernel arguments of the tensor-core attention kernels.
struct TcArgs {
  int B, H, N, Np, nqb, nkb;   // N, Np: query rows (real, padded)
  int Nk, Npk;                 // forward: key rows (real, padded); equal to N, Np unless queries are gathered
  float scale_log2;
  const int32_t* row_base;
  const int32_t* row_pat;
  const int32_t* pat_ptr;
  const int16_t* pat_off;
  int n_pat, nnz_pat, map_offset;
  int block_k;             // key-block size (64, 80, 96, 128 or 144)
  int nke;                 // energies: key blocks of block_k keys, ceil(N / block_k)
  void* o;                 // bf16 [B, H, Np, d]
  float* lse;              // [B, H, Np] natural-log LSE or nullptr
  float* lse2;             // calibration: per-row log2-domain LSE [H * Np]
  float* energy;           // calibration: [H, nqb, nkb]
  int32_t* status;
  unsigned long long spin_ns;
};

struct SimtArgs {
  int B, H, N, Np, block_q, block_k, nqb, nkb;
  float scale;
  const int32_t* row_base;
  const int32_t* row_pat;
  const int32_t* pat_ptr;
  const int16_t* pat_off;
  int n_pat, nnz_pat, map_offset;
  float* lse;        // fwd: [B,H,Np] or nullptr; calibration: per-row LSE [H*Np]
  float* energy;     // calibration: [H, nqb, nkb]
  int32_t* status;
};

// Argument checks and launch of the block energies, shared by
// calibatt_block_energy, calibatt_calibrate and calibatt_block_energy_noalloc
// (api.cu).  lse_ws: per-row scratch of H * Np floats.
int check_energy_args(const void* q, const void* k, int H, int N, int Np, int d, int dtype, int block_q,
                      int block_k, float scale);
int energy_impl(const void* q, const void* k, int H, int N, int Np, int d, int dtype, int block_q, int block_k,
                float scale, float* energy_out, float* lse_ws, int32_t* dev_status, cudaStream_t s);

// attn_tc.cu (bf16, tcgen05)
int launch_tc_fwd(const void* q, const void* k, const void* v, int d, const TcArgs& a, cudaStream_t s);
int launch_tc_energy(const void* q, const void* k, int d, const TcArgs& a, cudaStream_t s);
// The STATS pass alone: a.lse2[h * Np + row] = log2-domain LSE of every row over the real keys.
int launch_tc_stats(const void* q, const void* k, int d, const TcArgs& a, cudaStream_t s);

// attn_simt.cu (fp32, FFMA)
int launch_simt_fwd(const void* q, const void* k, const void* v, void* o, int d, const SimtArgs& a,
                    cudaStream_t s);
int launch_simt_energy(const void* q, const void* k, int d, const SimtArgs& a, cudaStream_t s);

// select_vote.cu
int launch_select_vote(const float* energy, int rows, int nkb, int mode, int topk, double eps,
                       int32_t* votes, float* esum, cudaStream_t s);
int launch_finalize(const int32_t* votes, const float* esum, int rows, int nkb, int min_votes,
                    uint8_t* mask, cudaStream_t s);

// compile.cu
size_t compile_workspace_bytes(long long rows, int nkb);
int run_compile(const uint8_t* masks, int n_maps, int nqb, int nkb, int dedup, void* ws, size_t ws_bytes,
                calibatt_blocklist* out, int64_t totals[3], cudaStream_t s);

// selftest
int launch_selftest_timeout(uint64_t limit_ns, int32_t* status, cudaStream_t s);

// TMA descriptor for a row-major bf16 matrix [rows, cols]; box 64 cols x box_rows rows, 128-byte swizzle.
int make_tmap_bf16(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows = 128);

}  // namespace calibatt
