// attn_simt.cu -- float32 block-sparse attention and block energies on CUDA
// cores (FFMA), for inputs whose tolerance tensor-core arithmetic cannot meet.
//
// Same method as attn_tc.cu (CalibAtt paper page, Abstract and Figure 5(b):
// kept blocks computed exactly, skipped blocks never touched; Figure 2 /
// Table S5: block-level post-softmax energies), but in plain fp32: scores are
// fp32 dot products, probabilities use expf, and the output keeps fp32.
// One CTA owns one query block (one thread per query row); the K and V
// blocks of each kept key block are staged in shared memory and broadcast to
// all rows.
#include <cfloat>
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace calibatt {
namespace {

template <typename T>
__device__ __forceinline__ float ld_f(const T* p);
template <>
__device__ __forceinline__ float ld_f<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }

template <typename T>
__device__ __forceinline__ void st_f(T* p, float v);
template <>
__device__ __forceinline__ void st_f<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void st_f<__nv_bfloat16>(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// Loads `rows` rows (from token r0) of a [.., D] tensor into s[rows][ld]; rows >= N read as 0.
template <typename T, int D>
__device__ __forceinline__ void stage_rows(float* s, int ld, const T* src, int r0, int rows, int N) {
  for (int e = threadIdx.x; e < rows * D; e += blockDim.x) {
    const int r = e / D, cidx = e % D;
    const int tok = r0 + r;
    s[r * ld + cidx] = (tok < N) ? ld_f(src + static_cast<size_t>(tok) * D + cidx) : 0.f;
  }
}

template <int D>
__device__ __forceinline__ float dot_row(const float* q, const float* k) {
  float acc = 0.f;
#pragma unroll 16
  for (int i = 0; i < D; ++i) acc = fmaf(q[i], k[i], acc);
  return acc;
}

// Reads and checks the kept-block list of row (map_offset + h, qb) into list[];
// returns its length, or 0 (with E_CORRUPT) when the list fails the checks.
__device__ int load_list(const SimtArgs& a, int h, int qb, int* list) {
  const long long r = static_cast<long long>(a.map_offset + h) * a.nqb + qb;
  const int base = a.row_base[r];
  const int pat = a.row_pat[r];
  bool bad = false;
  int p0 = 0, p1 = 0;
  if (pat < 0 || pat >= a.n_pat) {
    bad = true;
  } else {
    p0 = a.pat_ptr[pat];
    p1 = a.pat_ptr[pat + 1];
    if (p0 < 0 || p1 < p0 || p1 > a.nnz_pat || p1 - p0 > a.nkb) bad = true;
  }
  int n = bad ? 0 : p1 - p0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int off = a.pat_off[p0 + i];
    const int kb = base + off;
    bool ok = kb >= 0 && kb < a.nkb;
    if (i > 0) ok = ok && off > a.pat_off[p0 + i - 1];
    if (!ok) bad = true;
    list[i] = kb;
  }
  bad = __syncthreads_or(bad) != 0;
  if (bad) {
    if (threadIdx.x == 0) report_status(a.status, CALIBATT_E_CORRUPT);
    return 0;
  }
  return n;
}

constexpr int kMaxList = 2048;

// Sparse forward.  grid (nqb, H, B), block = block_q threads.
template <typename T, int D>
__global__ void __launch_bounds__(128) k_fwd_simt(const T* __restrict__ q, const T* __restrict__ k,
                                                  const T* __restrict__ v, T* __restrict__ o, const SimtArgs a) {
  extern __shared__ float sm[];
  __shared__ int list[kMaxList];
  const int BQ = a.block_q, BK = a.block_k;
  float* Qs = sm;                       // [BQ][D+1]
  float* Ks = Qs + BQ * (D + 1);        // [BK][D+1]
  float* Vs = Ks + BK * (D + 1);        // [BK][D]
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const size_t bh_off = (static_cast<size_t>(b) * a.H + h) * a.Np;
  const T* qh = q + bh_off * D;
  const T* kh = k + bh_off * D;
  const T* vh = v + bh_off * D;
  const int row = threadIdx.x;
  const int tok = qb * BQ + row;

  const int n = load_list(a, h, qb, list);
  stage_rows<T, D>(Qs, D + 1, qh, qb * BQ, BQ, a.N);

  float acc[D];
#pragma unroll
  for (int i = 0; i < D; ++i) acc[i] = 0.f;
  float m = -INFINITY, l = 0.f;
  const float* qrow = Qs + row * (D + 1);

  for (int j = 0; j < n; ++j) {
    const int kb = list[j];
    const int k0 = kb * BK;
    const int valid = min(BK, a.N - k0);
    __syncthreads();
    stage_rows<T, D>(Ks, D + 1, kh, k0, BK, a.N);
    stage_rows<T, D>(Vs, D, vh, k0, BK, a.N);
    __syncthreads();
    float mx = -INFINITY;
    for (int t = 0; t < valid; ++t) mx = fmaxf(mx, dot_row<D>(qrow, Ks + t * (D + 1)) * a.scale);
    const float m_new = fmaxf(m, mx);
    const float alpha = expf(m - m_new);
    l *= alpha;
#pragma unroll
    for (int i = 0; i < D; ++i) acc[i] *= alpha;
    for (int t = 0; t < valid; ++t) {
      const float p = expf(dot_row<D>(qrow, Ks + t * (D + 1)) * a.scale - m_new);
      l += p;
      const float* vr = Vs + t * D;
#pragma unroll
      for (int i = 0; i < D; ++i) acc[i] = fmaf(p, vr[i], acc[i]);
    }
    m = m_new;
  }

  const bool zero = (n == 0) || tok >= a.N;
  const float inv_l = zero ? 0.f : 1.f / l;
  T* orow = o + (bh_off + tok) * D;
#pragma unroll
  for (int i = 0; i < D; ++i) st_f<T>(orow + i, acc[i] * inv_l);
  if (a.lse != nullptr) a.lse[bh_off + tok] = zero ? -INFINITY : m + logf(l);
}

// Dense row LSE (natural log) of one calibration input.  grid (nqb, H).
template <typename T, int D>
__global__ void __launch_bounds__(128) k_stats_simt(const T* __restrict__ q, const T* __restrict__ k, const SimtArgs a) {
  extern __shared__ float sm[];
  const int BQ = a.block_q, BK = a.block_k;
  float* Qs = sm;
  float* Ks = Qs + BQ * (D + 1);
  const int qb = blockIdx.x, h = blockIdx.y;
  const T* qh = q + static_cast<size_t>(h) * a.Np * D;
  const T* kh = k + static_cast<size_t>(h) * a.Np * D;
  const int row = threadIdx.x;
  const int tok = qb * BQ + row;
  stage_rows<T, D>(Qs, D + 1, qh, qb * BQ, BQ, a.N);
  const float* qrow = Qs + row * (D + 1);
  float m = -INFINITY, l = 0.f;
  for (int kb = 0; kb < a.nkb; ++kb) {
    const int k0 = kb * BK;
    const int valid = min(BK, a.N - k0);
    __syncthreads();
    stage_rows<T, D>(Ks, D + 1, kh, k0, BK, a.N);
    __syncthreads();
    float mx = -INFINITY;
    for (int t = 0; t < valid; ++t) mx = fmaxf(mx, dot_row<D>(qrow, Ks + t * (D + 1)) * a.scale);
    const float m_new = fmaxf(m, mx);
    l *= expf(m - m_new);
    for (int t = 0; t < valid; ++t) l += expf(dot_row<D>(qrow, Ks + t * (D + 1)) * a.scale - m_new);
    m = m_new;
  }
  a.lse[static_cast<size_t>(h) * a.Np + tok] = (tok < a.N) ? m + logf(l) : -INFINITY;
}

// Block energies from the dense row LSE.  grid (nqb, H).  The per-row block
// sums are reduced over the rows by a fixed-order tree (deterministic).
template <typename T, int D>
__global__ void __launch_bounds__(128) k_energy_simt(const T* __restrict__ q, const T* __restrict__ k, const SimtArgs a) {
  extern __shared__ float sm[];
  __shared__ float red[128];
  const int BQ = a.block_q, BK = a.block_k;
  float* Qs = sm;
  float* Ks = Qs + BQ * (D + 1);
  const int qb = blockIdx.x, h = blockIdx.y;
  const T* qh = q + static_cast<size_t>(h) * a.Np * D;
  const T* kh = k + static_cast<size_t>(h) * a.Np * D;
  const int row = threadIdx.x;
  const int tok = qb * BQ + row;
  stage_rows<T, D>(Qs, D + 1, qh, qb * BQ, BQ, a.N);
  const float* qrow = Qs + row * (D + 1);
  const float lse = (tok < a.N) ? a.lse[static_cast<size_t>(h) * a.Np + tok] : 0.f;
  const int rows = min(BQ, a.N - qb * BQ);
  float* erow = a.energy + (static_cast<size_t>(h) * a.nqb + qb) * a.nkb;
  for (int kb = 0; kb < a.nkb; ++kb) {
    const int k0 = kb * BK;
    const int valid = min(BK, a.N - k0);
    __syncthreads();
    stage_rows<T, D>(Ks, D + 1, kh, k0, BK, a.N);
    __syncthreads();
    float rs = 0.f;
    if (tok < a.N)
      for (int t = 0; t < valid; ++t) rs += expf(dot_row<D>(qrow, Ks + t * (D + 1)) * a.scale - lse);
    red[row] = rs;
    __syncthreads();
    for (int w = BQ / 2; w > 0; w >>= 1) {
      if (row < w) red[row] += red[row + w];
      __syncthreads();
    }
    if (row == 0) erow[kb] = red[0] / static_cast<float>(rows);
  }
}

template <typename Kern>
int set_smem(Kern kern, size_t bytes) {
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)) !=
      cudaSuccess)
    return check_launch("cudaFuncSetAttribute(simt)");
  return CALIBATT_OK;
}

template <int D>
int fwd_d(const void* q, const void* k, const void* v, void* o, const SimtArgs& a, cudaStream_t s) {
  const size_t bytes = sizeof(float) * (a.block_q * (D + 1) + a.block_k * (D + 1) + a.block_k * D);
  auto kern = k_fwd_simt<float, D>;
  int rc = set_smem(kern, bytes);
  if (rc) return rc;
  kern<<<dim3(a.nqb, a.H, a.B), a.block_q, bytes, s>>>(static_cast<const float*>(q), static_cast<const float*>(k),
                                                         static_cast<const float*>(v), static_cast<float*>(o), a);
  count_launch();
  return check_launch("k_fwd_simt");
}

template <int D>
int energy_d(const void* q, const void* k, const SimtArgs& a, cudaStream_t s) {
  const size_t bytes = sizeof(float) * (a.block_q * (D + 1) + a.block_k * (D + 1));
  auto ks = k_stats_simt<float, D>;
  auto ke = k_energy_simt<float, D>;
  int rc = set_smem(ks, bytes);
  if (rc) return rc;
  rc = set_smem(ke, bytes);
  if (rc) return rc;
  ks<<<dim3(a.nqb, a.H), a.block_q, bytes, s>>>(static_cast<const float*>(q), static_cast<const float*>(k), a);
  count_launch();
  if ((rc = check_launch("k_stats_simt"))) return rc;
  ke<<<dim3(a.nqb, a.H), a.block_q, bytes, s>>>(static_cast<const float*>(q), static_cast<const float*>(k), a);
  count_launch();
  return check_launch("k_energy_simt");
}

}  // namespace

int launch_simt_fwd(const void* q, const void* k, const void* v, void* o, int d, const SimtArgs& a,
                    cudaStream_t s) {
  if (d == 64) return fwd_d<64>(q, k, v, o, a, s);
  return fwd_d<128>(q, k, v, o, a, s);
}

int launch_simt_energy(const void* q, const void* k, int d, const SimtArgs& a, cudaStream_t s) {
  if (d == 64) return energy_d<64>(q, k, a, s);
  return energy_d<128>(q, k, a, s);
}

}  // namespace calibatt
