// api.cu -- the extern "C" entry points declared in include/calibatt.h:
// argument validation, status codes, TMA descriptor encoding and dispatch to
// the kernels.  Nothing here allocates device memory.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <mutex>
#include <string>

#include "common.cuh"
#include "internal.h"

namespace calibatt {

namespace {
thread_local std::string g_last_error = "no error";
std::atomic<uint64_t> g_launches{0};
std::atomic<uint64_t> g_spin_ns{0};
std::once_flag g_spin_once;

void init_spin() {
  uint64_t v = 2000000000ull;
  if (const char* e = std::getenv("CALIBATT_SPIN_LIMIT_NS")) {
    char* end = nullptr;
    const unsigned long long x = std::strtoull(e, &end, 10);
    if (end != e && x > 0) v = x;
  }
  uint64_t expected = 0;
  g_spin_ns.compare_exchange_strong(expected, v);
}
}  // namespace

int set_error(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(CALIBATT_E_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return CALIBATT_OK;
}

void count_launch(int n) { g_launches.fetch_add(static_cast<uint64_t>(n)); }

uint64_t spin_limit_ns() {
  std::call_once(g_spin_once, init_spin);
  return g_spin_ns.load();
}

int current_device(int* dev) {
  int d = -1;
  if (cudaGetDevice(&d) != cudaSuccess) return check_launch("cudaGetDevice");
  if (d < 0 || d >= kMaxDevices) return set_error(CALIBATT_E_UNSUPPORTED, "device ordinal %d out of range", d);
  *dev = d;
  return CALIBATT_OK;
}

// ---- TMA descriptors --------------------------------------------------------

namespace {
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

void load_encode() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q{};
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
}
}  // namespace

int make_tmap_bf16(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  std::call_once(g_encode_once, load_encode);
  if (g_encode == nullptr) return set_error(CALIBATT_E_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(CALIBATT_E_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return CALIBATT_OK;
}

// ---- self-test kernel: a wait that can only run out -------------------------

namespace {
__global__ void k_selftest_timeout(uint64_t limit_ns, int32_t* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Nothing ever arrives on `bar`: the bounded wait must give up.
    if (!mbar_wait(&bar, 0, &abort_flag, limit_ns)) report_status(status, CALIBATT_E_TIMEOUT);
    // Complete the pending phase so the barrier is left in a clean state.
    mbar_arrive(&bar);
  }
}
}  // namespace

int launch_selftest_timeout(uint64_t limit_ns, int32_t* status, cudaStream_t s) {
  k_selftest_timeout<<<1, 32, 0, s>>>(limit_ns, status);
  count_launch();
  return check_launch("k_selftest_timeout");
}

}  // namespace calibatt

using namespace calibatt;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int validate_blocklist(const calibatt_blocklist* bl) {
  if (bl == nullptr) return set_error(CALIBATT_E_INVALID, "block list is NULL");
  if (bl->row_base == nullptr || bl->row_pat == nullptr || bl->pat_ptr == nullptr)
    return set_error(CALIBATT_E_INVALID, "block list arrays are NULL");
  if (bl->nnz_pat > 0 && bl->pat_off == nullptr) return set_error(CALIBATT_E_INVALID, "pat_off is NULL");
  if (bl->n_maps <= 0 || bl->n_q_blocks <= 0 || bl->n_k_blocks <= 0 || bl->n_pat <= 0 || bl->nnz_pat < 0)
    return set_error(CALIBATT_E_INVALID, "block list sizes are invalid");
  return CALIBATT_OK;
}

}  // namespace

namespace {

// Argument checks of the forward, shared by the plain, the streamed and the
// gathered-query entry points so that none enqueues anything for a call it
// would reject.  Queries have Nq real rows padded to Npq, keys Nk padded to Npk.
int check_fwd(const void* q, const void* k, const void* v, const void* o, int B, int H, int Nq, int Npq, int Nk,
              int Npk, int d, int dtype, float scale, const calibatt_blocklist* bl, int map_offset) {
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr)
    return set_error(CALIBATT_E_INVALID, "q, k, v and o must be non-NULL");
  if (B <= 0 || H <= 0 || Nq <= 0 || Npq < Nq || Nk <= 0 || Npk < Nk || d <= 0)
    return set_error(CALIBATT_E_INVALID, "bad sizes B=%d H=%d Nq=%d Npq=%d Nk=%d Npk=%d d=%d", B, H, Nq, Npq, Nk, Npk,
                     d);
  if (!(scale > 0.f) || !std::isfinite(scale)) return set_error(CALIBATT_E_INVALID, "scale must be finite and > 0");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return set_error(CALIBATT_E_INVALID, "q, k, v, o must be 16-byte aligned");
  int rc = validate_blocklist(bl);
  if (rc) return rc;
  if (bl->block_q <= 0 || bl->block_k <= 0 || Npq % bl->block_q != 0 || Npk % bl->block_k != 0)
    return set_error(CALIBATT_E_INVALID, "Np=%d/%d is not a multiple of the block sizes", Npq, Npk);
  const int nqb = Npq / bl->block_q, nkb = Npk / bl->block_k;
  if (bl->n_q_blocks != nqb || bl->n_k_blocks != nkb)
    return set_error(CALIBATT_E_INVALID, "block list grid %dx%d does not match Np/block = %dx%d", bl->n_q_blocks,
                     bl->n_k_blocks, nqb, nkb);
  if ((Npk - Nk) >= bl->block_k || (Npq - Nq) >= bl->block_q)
    return set_error(CALIBATT_E_INVALID, "Np - N must be smaller than one block");
  if (map_offset < 0 || static_cast<long long>(map_offset) + H > bl->n_maps)
    return set_error(CALIBATT_E_INVALID, "map_offset %d + H %d exceeds n_maps %d", map_offset, H, bl->n_maps);
  if (static_cast<long long>(B) * H * (Npq > Npk ? Npq : Npk) >= (1ll << 31))
    return set_error(CALIBATT_E_UNSUPPORTED, "B*H*Np must be below 2^31 rows");
  if (dtype == CALIBATT_BF16) {
    const int bk = bl->block_k;
    if (!(d == 64 || d == 128) || bl->block_q != 128 || !(bk == 64 || bk == 80 || bk == 96 || bk == 128 || bk == 144))
      return set_error(CALIBATT_E_UNSUPPORTED,
                       "bf16 path supports d in {64,128}, 128-row query blocks and key blocks of 64, 80, 96, 128 "
                       "or 144");
    if (nkb > 2048) return set_error(CALIBATT_E_UNSUPPORTED, "at most 2048 key blocks per row");
    return CALIBATT_OK;
  }
  if (dtype == CALIBATT_FP32) {
    if (Nq != Nk || Npq != Npk) return set_error(CALIBATT_E_UNSUPPORTED, "fp32 path needs equal query and key lengths");
    if (!(d == 64 || d == 128) || !(bl->block_q == 64 || bl->block_q == 128) ||
        !(bl->block_k == 64 || bl->block_k == 128))
      return set_error(CALIBATT_E_UNSUPPORTED, "fp32 path supports d in {64,128}, blocks in {64,128}");
    if (nkb > 2048) return set_error(CALIBATT_E_UNSUPPORTED, "at most 2048 key blocks per row");
    return CALIBATT_OK;
  }
  return set_error(CALIBATT_E_UNSUPPORTED, "unknown dtype %d", dtype);
}

int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq, int Npq, int Nk,
             int Npk, int d, int dtype, float scale, const calibatt_blocklist* bl, int map_offset, int32_t* dev_status,
             calibatt_stream_t stream) {
  int rc = check_fwd(q, k, v, o, B, H, Nq, Npq, Nk, Npk, d, dtype, scale, bl, map_offset);
  if (rc) return rc;
  const int nqb = Npq / bl->block_q, nkb = Npk / bl->block_k;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == CALIBATT_BF16) {
    TcArgs a{};
    a.B = B; a.H = H; a.N = Nq; a.Np = Npq; a.Nk = Nk; a.Npk = Npk; a.nqb = nqb; a.nkb = nkb;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.row_base = bl->row_base; a.row_pat = bl->row_pat; a.pat_ptr = bl->pat_ptr; a.pat_off = bl->pat_off;
    a.n_pat = bl->n_pat; a.nnz_pat = bl->nnz_pat; a.map_offset = map_offset;
    a.block_k = bl->block_k;
    a.o = o; a.lse = lse; a.status = dev_status; a.spin_ns = spin_limit_ns();
    return launch_tc_fwd(q, k, v, d, a, s);
  }
  SimtArgs a{};
  a.B = B; a.H = H; a.N = Nq; a.Np = Npq; a.block_q = bl->block_q; a.block_k = bl->block_k;
  a.nqb = nqb; a.nkb = nkb; a.scale = scale;
  a.row_base = bl->row_base; a.row_pat = bl->row_pat; a.pat_ptr = bl->pat_ptr; a.pat_off = bl->pat_off;
  a.n_pat = bl->n_pat; a.nnz_pat = bl->nnz_pat; a.map_offset = map_offset;
  a.lse = lse; a.status = dev_status;
  return launch_simt_fwd(q, k, v, o, d, a, s);
}

}  // namespace

namespace {

// Copy streams and events of the streamed forward, one set per device,
// created on first use and kept for the life of the process.  The mutex makes
// each call's record/wait sequence atomic, so concurrent callers never see
// each other's event records.
struct StreamSet {
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, in = nullptr, out = nullptr, done = nullptr;
};
std::mutex g_stream_mu;
StreamSet g_streams[kMaxDevices];

int stream_set(StreamSet** out) {
  int dev = 0;
  if (int rc = current_device(&dev)) return rc;
  StreamSet& ss = g_streams[dev];
  if (ss.h2d == nullptr) {
    if (cudaStreamCreateWithFlags(&ss.h2d, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&ss.d2h, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.start, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.in, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.out, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.done, cudaEventDisableTiming) != cudaSuccess) {
      ss = StreamSet{};
      return check_launch("creating the copy streams");
    }
  }
  *out = &ss;
  return CALIBATT_OK;
}

int cuda_ok(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return CALIBATT_OK;
  return set_error(CALIBATT_E_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

}  // namespace

extern "C" {

const char* calibatt_last_error(void) { return g_last_error.c_str(); }

int calibatt_version(void) { return 1 * 10000 + 0 * 100 + 0; }

uint64_t calibatt_launch_count(void) { return g_launches.load(); }

void calibatt_set_spin_limit_ns(uint64_t ns) {
  spin_limit_ns();
  g_spin_ns.store(ns > 0 ? ns : 1);
}

uint64_t calibatt_get_spin_limit_ns(void) { return spin_limit_ns(); }

int calibatt_sparse_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
                             int Np, int d, int dtype, float scale, const calibatt_blocklist* bl, int map_offset,
                             int32_t* dev_status, calibatt_stream_t stream) {
  return fwd_impl(q, k, v, o, lse, B, H, N, Np, N, Np, d, dtype, scale, bl, map_offset, dev_status, stream);
}

int calibatt_sparse_attn_fwd_qk(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                                int Nq, int Npq, int Nk, int Npk, int d, int dtype, float scale,
                                const calibatt_blocklist* bl, int map_offset, int32_t* dev_status,
                                calibatt_stream_t stream) {
  if (dtype != CALIBATT_BF16)
    return set_error(CALIBATT_E_UNSUPPORTED, "separate query and key lengths are supported for bf16 only");
  return fwd_impl(q, k, v, o, lse, B, H, Nq, Npq, Nk, Npk, d, dtype, scale, bl, map_offset, dev_status, stream);
}

int calibatt_sparse_attn_fwd_streamed(const void* q_host, const void* k_host, const void* v_host, void* o_host,
                                      float* lse_host, void* q_dev, void* k_dev, void* v_dev, void* o_dev,
                                      float* lse_dev, int B, int H, int N, int Np, int d, int dtype, float scale,
                                      const calibatt_blocklist* bl, int map_offset, int heads_per_chunk,
                                      int32_t* dev_status, calibatt_stream_t stream) {
  if (q_host == nullptr || k_host == nullptr || v_host == nullptr || o_host == nullptr)
    return set_error(CALIBATT_E_INVALID, "q_host, k_host, v_host and o_host must be non-NULL");
  if (q_dev == nullptr || k_dev == nullptr || v_dev == nullptr || o_dev == nullptr)
    return set_error(CALIBATT_E_INVALID, "q_dev, k_dev, v_dev and o_dev must be non-NULL");
  if ((lse_host == nullptr) != (lse_dev == nullptr))
    return set_error(CALIBATT_E_INVALID, "lse_host and lse_dev must both be given or both be NULL");
  if (heads_per_chunk <= 0) return set_error(CALIBATT_E_INVALID, "heads_per_chunk must be >= 1");
  int rc = check_fwd(q_dev, k_dev, v_dev, o_dev, B, H, N, Np, N, Np, d, dtype, scale, bl, map_offset);
  if (rc) return rc;
  const size_t esize = dtype == CALIBATT_BF16 ? 2 : 4;
  const size_t plane = static_cast<size_t>(Np) * d * esize;   // bytes of one (b, h) slice
  const int hc = heads_per_chunk < H ? heads_per_chunk : H;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  std::lock_guard<std::mutex> lock(g_stream_mu);
  StreamSet* ss = nullptr;
  rc = stream_set(&ss);
  if (rc) return rc;
  // The staging buffers may still be in use by work already on `stream`.
  if ((rc = cuda_ok(cudaEventRecord(ss->start, s), "cudaEventRecord")) ||
      (rc = cuda_ok(cudaStreamWaitEvent(ss->h2d, ss->start, 0), "cudaStreamWaitEvent")) ||
      (rc = cuda_ok(cudaStreamWaitEvent(ss->d2h, ss->start, 0), "cudaStreamWaitEvent")))
    return rc;
  for (int b = 0; b < B; ++b) {
    for (int h0 = 0; h0 < H; h0 += hc) {
      const int hn = (H - h0) < hc ? (H - h0) : hc;
      const size_t first = static_cast<size_t>(b) * H + h0;      // first (b, h) slice of the chunk
      const size_t off = first * plane, bytes = static_cast<size_t>(hn) * plane;
      const size_t loff = first * Np, lbytes = static_cast<size_t>(hn) * Np * sizeof(float);
      auto at = [](const void* p, size_t o) { return static_cast<const char*>(p) + o; };
      auto atw = [](void* p, size_t o) { return static_cast<char*>(p) + o; };
      if ((rc = cuda_ok(cudaMemcpyAsync(atw(q_dev, off), at(q_host, off), bytes, cudaMemcpyHostToDevice, ss->h2d),
                        "cudaMemcpyAsync(q)")) ||
          (rc = cuda_ok(cudaMemcpyAsync(atw(k_dev, off), at(k_host, off), bytes, cudaMemcpyHostToDevice, ss->h2d),
                        "cudaMemcpyAsync(k)")) ||
          (rc = cuda_ok(cudaMemcpyAsync(atw(v_dev, off), at(v_host, off), bytes, cudaMemcpyHostToDevice, ss->h2d),
                        "cudaMemcpyAsync(v)")) ||
          (rc = cuda_ok(cudaEventRecord(ss->in, ss->h2d), "cudaEventRecord")) ||
          (rc = cuda_ok(cudaStreamWaitEvent(s, ss->in, 0), "cudaStreamWaitEvent")))
        return rc;
      rc = calibatt_sparse_attn_fwd(atw(q_dev, off), atw(k_dev, off), atw(v_dev, off), atw(o_dev, off),
                                    lse_dev ? lse_dev + loff : nullptr, 1, hn, N, Np, d, dtype, scale, bl,
                                    map_offset + h0, dev_status, stream);
      if (rc) return rc;
      if ((rc = cuda_ok(cudaEventRecord(ss->out, s), "cudaEventRecord")) ||
          (rc = cuda_ok(cudaStreamWaitEvent(ss->d2h, ss->out, 0), "cudaStreamWaitEvent")) ||
          (rc = cuda_ok(cudaMemcpyAsync(atw(o_host, off), at(o_dev, off), bytes, cudaMemcpyDeviceToHost, ss->d2h),
                        "cudaMemcpyAsync(o)")))
        return rc;
      if (lse_host != nullptr &&
          (rc = cuda_ok(cudaMemcpyAsync(lse_host + loff, lse_dev + loff, lbytes, cudaMemcpyDeviceToHost, ss->d2h),
                        "cudaMemcpyAsync(lse)")))
        return rc;
    }
  }
  if ((rc = cuda_ok(cudaEventRecord(ss->done, ss->d2h), "cudaEventRecord")) ||
      (rc = cuda_ok(cudaStreamWaitEvent(s, ss->done, 0), "cudaStreamWaitEvent")))
    return rc;
  return CALIBATT_OK;
}

int calibatt_calibrate_workspace_size(int H, int N, int Np, int d, int block_q, int block_k, size_t* bytes) {
  if (bytes == nullptr) return set_error(CALIBATT_E_INVALID, "bytes is NULL");
  if (H <= 0 || N <= 0 || Np < N || d <= 0 || block_q <= 0 || block_k <= 0 || Np % block_q)
    return set_error(CALIBATT_E_INVALID, "bad sizes");
  const size_t nqb = Np / block_q, nkb = (static_cast<size_t>(N) + block_k - 1) / block_k;
  // per-row LSE [H*Np] + energies [H*nqb*nkb], each 256-byte aligned
  *bytes = ((static_cast<size_t>(H) * Np * 4 + 255) & ~size_t(255)) + ((H * nqb * nkb * 4 + 255) & ~size_t(255)) + 256;
  return CALIBATT_OK;
}

}  // extern "C"

namespace calibatt {

int energy_impl(const void* q, const void* k, int H, int N, int Np, int d, int dtype, int block_q, int block_k,
                float scale, float* energy_out, float* lse_ws, int32_t* dev_status, cudaStream_t s) {
  const int nqb = Np / block_q, nkb = (N + block_k - 1) / block_k;
  if (dtype == CALIBATT_BF16) {
    TcArgs a{};
    // nkb: 128-key tiles walked; the energies use nke blocks of block_k keys
    a.B = 1; a.H = H; a.N = N; a.Np = Np; a.nqb = nqb; a.nkb = Np / 128; a.block_k = block_k; a.nke = nkb;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.lse2 = lse_ws; a.energy = energy_out; a.status = dev_status; a.spin_ns = spin_limit_ns();
    return launch_tc_energy(q, k, d, a, s);
  }
  SimtArgs a{};
  a.B = 1; a.H = H; a.N = N; a.Np = Np; a.block_q = block_q; a.block_k = block_k; a.nqb = nqb; a.nkb = nkb;
  a.scale = scale; a.lse = lse_ws; a.energy = energy_out; a.status = dev_status;
  return launch_simt_energy(q, k, d, a, s);
}

int check_energy_args(const void* q, const void* k, int H, int N, int Np, int d, int dtype, int block_q,
                      int block_k, float scale) {
  if (q == nullptr || k == nullptr) return set_error(CALIBATT_E_INVALID, "q and k must be non-NULL");
  if (H <= 0 || N <= 0 || Np < N || d <= 0 || block_q <= 0 || block_k <= 0 || Np % block_q)
    return set_error(CALIBATT_E_INVALID, "bad sizes H=%d N=%d Np=%d d=%d", H, N, Np, d);
  if ((Np - N) >= block_q) return set_error(CALIBATT_E_INVALID, "Np - N must be smaller than one query block");
  if (!(scale > 0.f) || !std::isfinite(scale)) return set_error(CALIBATT_E_INVALID, "scale must be finite and > 0");
  if (!aligned16(q) || !aligned16(k)) return set_error(CALIBATT_E_INVALID, "q and k must be 16-byte aligned");
  if (static_cast<long long>(H) * Np >= (1ll << 31)) return set_error(CALIBATT_E_UNSUPPORTED, "H*Np too large");
  if (dtype == CALIBATT_BF16) {
    if (!(d == 64 || d == 128) || block_q != 128 ||
        !(block_k == 64 || block_k == 80 || block_k == 96 || block_k == 128 || block_k == 144))
      return set_error(CALIBATT_E_UNSUPPORTED,
                       "bf16 energies support d in {64,128}, 128-row query blocks and key blocks of 64, 80, 96, 128 or "
                       "144");
    if (Np / 128 > 2048 || (N + block_k - 1) / block_k > 2048)
      return set_error(CALIBATT_E_UNSUPPORTED, "at most 2048 key blocks");
    return CALIBATT_OK;
  }
  if (dtype == CALIBATT_FP32) {
    if (!(d == 64 || d == 128) || !(block_q == 64 || block_q == 128) || !(block_k == 64 || block_k == 128))
      return set_error(CALIBATT_E_UNSUPPORTED, "fp32 energies support d in {64,128}, blocks in {64,128}");
    if (Np % block_k || (Np - N) >= block_k)
      return set_error(CALIBATT_E_INVALID, "fp32 energies need Np a multiple of block_k and Np - N below it");
    return CALIBATT_OK;
  }
  return set_error(CALIBATT_E_UNSUPPORTED, "unknown dtype %d", dtype);
}

}  // namespace calibatt

extern "C" {

namespace {

int carve_energy_ws(void* ws, size_t ws_bytes, int H, int N, int Np, int d, int bq, int bk, float** lse,
                    float** energy) {
  size_t need = 0;
  calibatt_calibrate_workspace_size(H, N, Np, d, bq, bk, &need);
  if (ws == nullptr || ws_bytes < need)
    return set_error(CALIBATT_E_WORKSPACE, "workspace too small: need %zu bytes, got %zu", need, ws_bytes);
  char* base = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255));
  *lse = reinterpret_cast<float*>(base);
  const size_t lse_bytes = (static_cast<size_t>(H) * Np * 4 + 255) & ~size_t(255);
  *energy = reinterpret_cast<float*>(base + lse_bytes);
  return CALIBATT_OK;
}

int topk_of(double frac, int nkb) {
  double k = std::ceil(frac * nkb);
  if (k < 1) k = 1;
  if (k > nkb) k = nkb;
  return static_cast<int>(k);
}

}  // namespace

int calibatt_block_energy(const void* q, const void* k, int H, int N, int Np, int d, int dtype, int block_q,
                          int block_k, float scale, float* energy_out, void* workspace, size_t workspace_bytes,
                          int32_t* dev_status, calibatt_stream_t stream) {
  int rc = check_energy_args(q, k, H, N, Np, d, dtype, block_q, block_k, scale);
  if (rc) return rc;
  if (energy_out == nullptr) return set_error(CALIBATT_E_INVALID, "energy_out is NULL");
  float *lse = nullptr, *scratch_e = nullptr;
  if ((rc = carve_energy_ws(workspace, workspace_bytes, H, N, Np, d, block_q, block_k, &lse, &scratch_e))) return rc;
  return energy_impl(q, k, H, N, Np, d, dtype, block_q, block_k, scale, energy_out, lse, dev_status,
                     reinterpret_cast<cudaStream_t>(stream));
}

int calibatt_select_vote(const float* energy, int H, int nqb, int nkb, int select_mode, double select_param,
                         int32_t* votes_inout, float* energy_sum_inout, calibatt_stream_t stream) {
  if (energy == nullptr || votes_inout == nullptr || energy_sum_inout == nullptr)
    return set_error(CALIBATT_E_INVALID, "energy, votes and energy_sum must be non-NULL");
  if (H <= 0 || nqb <= 0 || nkb <= 0) return set_error(CALIBATT_E_INVALID, "bad sizes");
  if (nkb > 2048) return set_error(CALIBATT_E_UNSUPPORTED, "at most 2048 key blocks per row");
  if (static_cast<long long>(H) * nqb >= (1ll << 31)) return set_error(CALIBATT_E_UNSUPPORTED, "H*nqb too large");
  int topk = 0;
  double eps = 0.0;
  if (select_mode == CALIBATT_SELECT_TOPK) {
    if (!(select_param > 0.0) || select_param > 1.0) return set_error(CALIBATT_E_INVALID, "top-k fraction must be in (0,1]");
    topk = topk_of(select_param, nkb);
  } else if (select_mode == CALIBATT_SELECT_ENERGY) {
    if (!(select_param >= 0.0) || !(select_param < 1.0)) return set_error(CALIBATT_E_INVALID, "eps must be in [0,1)");
    eps = select_param;
  } else {
    return set_error(CALIBATT_E_INVALID, "unknown select mode %d", select_mode);
  }
  return launch_select_vote(energy, H * nqb, nkb, select_mode, topk, eps, votes_inout, energy_sum_inout,
                            reinterpret_cast<cudaStream_t>(stream));
}

int calibatt_finalize_mask(const int32_t* votes, const float* energy_sum, int H, int nqb, int nkb, int min_votes,
                           uint8_t* mask_out, calibatt_stream_t stream) {
  if (votes == nullptr || energy_sum == nullptr || mask_out == nullptr)
    return set_error(CALIBATT_E_INVALID, "votes, energy_sum and mask must be non-NULL");
  if (H <= 0 || nqb <= 0 || nkb <= 0) return set_error(CALIBATT_E_INVALID, "bad sizes");
  if (static_cast<long long>(H) * nqb >= (1ll << 31)) return set_error(CALIBATT_E_UNSUPPORTED, "H*nqb too large");
  if (min_votes < 0) return set_error(CALIBATT_E_INVALID, "min_votes must be >= 0");
  return launch_finalize(votes, energy_sum, H * nqb, nkb, min_votes, mask_out,
                         reinterpret_cast<cudaStream_t>(stream));
}

int calibatt_calibrate(const void* const* q_list, const void* const* k_list, int n_inputs, int H, int N, int Np,
                       int d, int dtype, int block_q, int block_k, float scale, int select_mode, double select_param,
                       int32_t* votes_inout, float* energy_sum_inout, int min_votes, uint8_t* mask_out,
                       void* workspace, size_t workspace_bytes, int32_t* dev_status, calibatt_stream_t stream) {
  if (n_inputs < 0 || (n_inputs > 0 && (q_list == nullptr || k_list == nullptr)))
    return set_error(CALIBATT_E_INVALID, "bad input lists");
  if (votes_inout == nullptr || energy_sum_inout == nullptr)
    return set_error(CALIBATT_E_INVALID, "votes and energy_sum must be non-NULL");
  int rc;
  for (int n = 0; n < n_inputs; ++n)
    if ((rc = check_energy_args(q_list[n], k_list[n], H, N, Np, d, dtype, block_q, block_k, scale))) return rc;
  const int nqb = Np / block_q, nkb = (N + block_k - 1) / block_k;
  if (nkb > 2048) return set_error(CALIBATT_E_UNSUPPORTED, "at most 2048 key blocks per row");
  if (select_mode == CALIBATT_SELECT_TOPK) {
    if (!(select_param > 0.0) || select_param > 1.0) return set_error(CALIBATT_E_INVALID, "top-k fraction must be in (0,1]");
  } else if (select_mode == CALIBATT_SELECT_ENERGY) {
    if (!(select_param >= 0.0) || !(select_param < 1.0)) return set_error(CALIBATT_E_INVALID, "eps must be in [0,1)");
  } else {
    return set_error(CALIBATT_E_INVALID, "unknown select mode %d", select_mode);
  }
  if (mask_out != nullptr && min_votes < 0) return set_error(CALIBATT_E_INVALID, "min_votes must be >= 0");
  float *lse = nullptr, *energy = nullptr;
  if ((rc = carve_energy_ws(workspace, workspace_bytes, H, N, Np, d, block_q, block_k, &lse, &energy))) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  for (int n = 0; n < n_inputs; ++n) {
    if ((rc = energy_impl(q_list[n], k_list[n], H, N, Np, d, dtype, block_q, block_k, scale, energy, lse, dev_status, s)))
      return rc;
    if ((rc = calibatt_select_vote(energy, H, nqb, nkb, select_mode, select_param, votes_inout, energy_sum_inout,
                                   stream)))
      return rc;
  }
  if (mask_out != nullptr)
    return calibatt_finalize_mask(votes_inout, energy_sum_inout, H, nqb, nkb, min_votes, mask_out, stream);
  return CALIBATT_OK;
}

int calibatt_compile_workspace_size(int n_maps, int nqb, int nkb, size_t* bytes) {
  if (bytes == nullptr) return set_error(CALIBATT_E_INVALID, "bytes is NULL");
  if (n_maps <= 0 || nqb <= 0 || nkb <= 0) return set_error(CALIBATT_E_INVALID, "bad sizes");
  *bytes = compile_workspace_bytes(static_cast<long long>(n_maps) * nqb, nkb);
  return CALIBATT_OK;
}

namespace {
int check_compile_args(const uint8_t* masks, int n_maps, int nqb, int nkb, int dedup) {
  if (masks == nullptr) return set_error(CALIBATT_E_INVALID, "masks is NULL");
  if (n_maps <= 0 || nqb <= 0 || nkb <= 0) return set_error(CALIBATT_E_INVALID, "bad sizes");
  if (nkb > 32767) return set_error(CALIBATT_E_UNSUPPORTED, "nkb must be <= 32767");
  if (static_cast<long long>(n_maps) * nqb >= (1ll << 31)) return set_error(CALIBATT_E_UNSUPPORTED, "too many rows");
  if (dedup < CALIBATT_DEDUP_NONE || dedup > CALIBATT_DEDUP_HASH_WEAK)
    return set_error(CALIBATT_E_INVALID, "unknown dedup mode %d", dedup);
  return CALIBATT_OK;
}
}  // namespace

int calibatt_compile_size(const uint8_t* masks, int n_maps, int nqb, int nkb, int dedup, int64_t* nnz,
                          int32_t* n_pat, int32_t* nnz_pat, void* workspace, size_t workspace_bytes,
                          calibatt_stream_t stream) {
  int rc = check_compile_args(masks, n_maps, nqb, nkb, dedup);
  if (rc) return rc;
  if (nnz == nullptr || n_pat == nullptr || nnz_pat == nullptr) return set_error(CALIBATT_E_INVALID, "NULL outputs");
  if (workspace == nullptr) return set_error(CALIBATT_E_WORKSPACE, "workspace is NULL");
  int64_t totals[3];
  if ((rc = run_compile(masks, n_maps, nqb, nkb, dedup, workspace, workspace_bytes, nullptr, totals,
                        reinterpret_cast<cudaStream_t>(stream))))
    return rc;
  if (totals[1] >= (1ll << 31) || totals[2] >= (1ll << 31))
    return set_error(CALIBATT_E_UNSUPPORTED, "pattern pool exceeds int32 indexing");
  *nnz = totals[0];
  *n_pat = static_cast<int32_t>(totals[1]);
  *nnz_pat = static_cast<int32_t>(totals[2]);
  return CALIBATT_OK;
}

int calibatt_compile(const uint8_t* masks, int n_maps, int nqb, int nkb, int dedup, int block_q, int block_k,
                     calibatt_blocklist* out, void* workspace, size_t workspace_bytes, calibatt_stream_t stream) {
  int rc = check_compile_args(masks, n_maps, nqb, nkb, dedup);
  if (rc) return rc;
  if (out == nullptr || out->row_base == nullptr || out->row_pat == nullptr || out->pat_ptr == nullptr)
    return set_error(CALIBATT_E_INVALID, "output block list arrays are NULL");
  if (out->n_pat <= 0 || out->nnz_pat < 0 || (out->nnz_pat > 0 && out->pat_off == nullptr))
    return set_error(CALIBATT_E_INVALID, "output capacities invalid");
  if ((out->csr_row_ptr == nullptr) != (out->csr_col == nullptr) && out->nnz > 0)
    return set_error(CALIBATT_E_INVALID, "csr_row_ptr and csr_col must be given together");
  if (block_q <= 0 || block_k <= 0) return set_error(CALIBATT_E_INVALID, "block sizes must be positive");
  if (workspace == nullptr) return set_error(CALIBATT_E_WORKSPACE, "workspace is NULL");
  int64_t totals[3];
  if ((rc = run_compile(masks, n_maps, nqb, nkb, dedup, workspace, workspace_bytes, out, totals,
                        reinterpret_cast<cudaStream_t>(stream))))
    return rc;
  if (totals[1] > out->n_pat || totals[2] > out->nnz_pat || (out->csr_col != nullptr && totals[0] > out->nnz))
    return set_error(CALIBATT_E_INVALID, "capacities too small: need n_pat=%lld nnz_pat=%lld nnz=%lld",
                     static_cast<long long>(totals[1]), static_cast<long long>(totals[2]),
                     static_cast<long long>(totals[0]));
  out->n_maps = n_maps;
  out->n_q_blocks = nqb;
  out->n_k_blocks = nkb;
  out->block_q = block_q;
  out->block_k = block_k;
  out->n_pat = static_cast<int32_t>(totals[1]);
  out->nnz_pat = static_cast<int32_t>(totals[2]);
  out->nnz = totals[0];
  return CALIBATT_OK;
}

int calibatt_selftest_wait_timeout(uint64_t limit_ns, int32_t* dev_status, calibatt_stream_t stream) {
  if (dev_status == nullptr) return set_error(CALIBATT_E_INVALID, "dev_status is NULL");
  if (limit_ns == 0 || limit_ns > 10000000000ull) return set_error(CALIBATT_E_INVALID, "limit must be in (0, 10 s]");
  return launch_selftest_timeout(limit_ns, dev_status, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
