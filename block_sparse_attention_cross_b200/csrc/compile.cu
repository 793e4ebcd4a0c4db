// compile.cu -- compile block masks into per-row kept-block lists with
// translation-relative row-pattern dedup.
//
// CalibAtt paper page, Abstract: the calibrated patterns are compiled into
// attention operations per layer, head and diffusion timestep; Figure 4(b):
// the attention pattern repeats across spatial rows within a frame.  A row
// (map, query block) is stored as base = first kept key block plus the
// offsets kb - base; rows with identical offset lists (translates) share one
// entry of the pattern pool.  Patterns are numbered by first occurrence in
// ascending row order, pattern 0 being the empty pattern, so the result is
// unique and independent of thread scheduling.
//
// Steps (all integer work):
//  1. per row: popcount, first kept block, 64-bit hash of the offset set;
//  2. hash table (open addressing) keyed by the hash, value = smallest row;
//  3. each row checks its pattern against that row; a mismatch (a hash
//     collision) is resolved exactly by a brute-force search for the
//     smallest row with an identical pattern;
//  4. exclusive scans: pattern ids, pattern-pool offsets, CSR row pointers;
//  5. fill row_base / row_pat / pat_ptr / pat_off (and the optional CSR).
#include <climits>
#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace calibatt {
namespace {

constexpr unsigned long long kEmptyKey = ~0ull;
constexpr int kScanItems = 1024;   // items per scan block (256 threads x 4)

__device__ __forceinline__ unsigned long long mix64(unsigned long long x) {
  // splitmix64 finalizer
  x += 0x9E3779B97F4A7C15ull;
  x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
  x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
  return x ^ (x >> 31);
}

__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ int warp_min(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

struct Work {
  int32_t* cnt;
  int32_t* first;
  unsigned long long* hash;
  int32_t* focc;           // first-occurrence row; -2 empty row
  long long* pid;          // exclusive scan of "is first occurrence"
  long long* pstart;       // exclusive scan of unique-pattern lengths
  long long* rowptr;       // exclusive scan of counts
  unsigned long long* tkeys;
  int32_t* tvals;
  int32_t* coll;           // collided rows
  long long* misc;         // [0] collisions, [1] unique patterns, [2] pool length, [3] nnz
  long long* partials;
  unsigned long long cap;  // hash table capacity (power of two)
};

// 1. row statistics; one warp per row.
__global__ void k_row_info(const uint8_t* __restrict__ masks, long long R, int nkb, int weak, Work w) {
  const long long r = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= R) return;
  const uint8_t* row = masks + r * nkb;
  int c = 0, f = INT_MAX;
  for (int j = lane; j < nkb; j += 32) {
    if (row[j]) {
      ++c;
      f = min(f, j);
    }
  }
  c = warp_sum(c);
  f = warp_min(f);
  unsigned long long hs = 0;
  if (c > 0 && !weak) {
    for (int j = lane; j < nkb; j += 32)
      if (row[j]) hs += mix64(static_cast<unsigned long long>(j - f));
    hs = warp_sum_u64(hs);
  }
  if (lane == 0) {
    w.cnt[r] = c;
    w.first[r] = c > 0 ? f : 0;
    unsigned long long hv = weak ? static_cast<unsigned long long>(c) : mix64(hs ^ (0xD6E8FEB86659FD93ull * c));
    w.hash[r] = hv & 0x7FFFFFFFFFFFFFFFull;
  }
}

// 2. insert: smallest row index per hash.
__global__ void k_hash_insert(long long R, Work w) {
  const long long r = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (r >= R || w.cnt[r] == 0) return;
  const unsigned long long key = w.hash[r];
  const unsigned long long mask = w.cap - 1;
  unsigned long long slot = mix64(key) & mask;
  for (unsigned long long probe = 0; probe < w.cap; ++probe) {
    const unsigned long long prev = atomicCAS(&w.tkeys[slot], kEmptyKey, key);
    if (prev == kEmptyKey || prev == key) {
      atomicMin(&w.tvals[slot], static_cast<int>(r));
      return;
    }
    slot = (slot + 1) & mask;
  }
}

__device__ bool same_pattern(const uint8_t* masks, int nkb, long long ra, int fa, long long rb, int fb) {
  const uint8_t* a = masks + ra * nkb;
  const uint8_t* b = masks + rb * nkb;
  bool diff = false;
  const int lane = threadIdx.x & 31;
  for (int t = lane; t < nkb; t += 32) {
    const int ba = (fa + t < nkb) ? (a[fa + t] != 0) : 0;
    const int bb = (fb + t < nkb) ? (b[fb + t] != 0) : 0;
    diff |= (ba != bb);
  }
  return !__any_sync(0xffffffffu, diff);
}

// 3a. verify against the hash representative; one warp per row.
__global__ void k_hash_verify(const uint8_t* __restrict__ masks, long long R, int nkb, Work w) {
  const long long r = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= R) return;
  const int c = w.cnt[r];
  if (c == 0) {
    if (lane == 0) w.focc[r] = -2;
    return;
  }
  const unsigned long long key = w.hash[r];
  const unsigned long long mask = w.cap - 1;
  unsigned long long slot = mix64(key) & mask;
  for (unsigned long long probe = 0; probe < w.cap; ++probe) {
    if (w.tkeys[slot] == key) break;
    slot = (slot + 1) & mask;
  }
  const long long rep = w.tvals[slot];
  if (rep == r) {
    if (lane == 0) w.focc[r] = static_cast<int>(r);
    return;
  }
  bool eq = (rep >= 0 && rep < R) && (w.cnt[rep] == c);
  if (eq) eq = same_pattern(masks, nkb, r, w.first[r], rep, w.first[rep]);
  if (lane == 0) {
    if (eq) {
      w.focc[r] = static_cast<int>(rep);
    } else {
      w.focc[r] = -1;
      const long long idx = atomicAdd(reinterpret_cast<unsigned long long*>(&w.misc[0]), 1ull);
      w.coll[idx] = static_cast<int>(r);
    }
  }
}

// 3b. exact resolution of collided rows: smallest row with the same pattern.
__global__ void k_collisions(const uint8_t* __restrict__ masks, long long R, int nkb, Work w) {
  __shared__ int best;
  const long long ncoll = w.misc[0];
  const int warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (long long idx = blockIdx.x; idx < ncoll; idx += gridDim.x) {
    const long long r = w.coll[idx];
    if (threadIdx.x == 0) best = static_cast<int>(r);
    __syncthreads();
    const int c = w.cnt[r];
    const unsigned long long key = w.hash[r];
    for (long long cand = warp; cand < r; cand += nwarps) {
      if (cand >= best) break;
      if (w.cnt[cand] != c || w.hash[cand] != key) continue;
      if (same_pattern(masks, nkb, r, w.first[r], cand, w.first[cand])) {
        if ((threadIdx.x & 31) == 0) atomicMin(&best, static_cast<int>(cand));
        break;
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) w.focc[r] = best;
    __syncthreads();
  }
}

__global__ void k_focc_identity(long long R, Work w) {
  const long long r = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (r < R) w.focc[r] = w.cnt[r] > 0 ? static_cast<int>(r) : -2;
}

// ---- exclusive scan (int64) over a generated sequence -----------------------
enum { SEQ_FIRST = 0, SEQ_ULEN = 1, SEQ_CNT = 2 };

__device__ __forceinline__ long long seq_item(const Work& w, int seq, long long i) {
  if (seq == SEQ_CNT) return w.cnt[i];
  const bool fo = w.focc[i] == i;
  if (seq == SEQ_FIRST) return fo ? 1 : 0;
  return fo ? w.cnt[i] : 0;
}

__device__ long long block_excl_scan(long long v, long long* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  long long inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  if (threadIdx.x == 0) {
    long long run = 0;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) {
      const long long t = warp_tot[i];
      warp_tot[i] = run;
      run += t;
    }
    warp_tot[32] = run;
  }
  __syncthreads();
  return warp_tot[warp] + inc - v;
}

__global__ void __launch_bounds__(256) k_scan_reduce(long long R, int seq, Work w) {
  __shared__ long long wt[33];
  const long long b0 = static_cast<long long>(blockIdx.x) * kScanItems;
  long long s = 0;
  for (int k = 0; k < 4; ++k) {
    const long long i = b0 + threadIdx.x * 4 + k;
    if (i < R) s += seq_item(w, seq, i);
  }
  block_excl_scan(s, wt);
  if (threadIdx.x == 0) w.partials[blockIdx.x] = wt[32];
}

__global__ void __launch_bounds__(1024) k_scan_top(long long P, long long* total_out, Work w) {
  __shared__ long long wt[33];
  long long carry = 0;
  for (long long base = 0; base < P; base += blockDim.x) {
    const long long i = base + threadIdx.x;
    const long long v = i < P ? w.partials[i] : 0;
    const long long ex = block_excl_scan(v, wt);
    if (i < P) w.partials[i] = carry + ex;
    const long long tot = wt[32];
    __syncthreads();
    carry += tot;
  }
  if (threadIdx.x == 0) *total_out = carry;
}

__global__ void __launch_bounds__(256) k_scan_apply(long long R, int seq, long long* out, Work w) {
  __shared__ long long wt[33];
  const long long b0 = static_cast<long long>(blockIdx.x) * kScanItems;
  long long v[4], s = 0;
  for (int k = 0; k < 4; ++k) {
    const long long i = b0 + threadIdx.x * 4 + k;
    v[k] = i < R ? seq_item(w, seq, i) : 0;
    s += v[k];
  }
  long long run = block_excl_scan(s, wt) + w.partials[blockIdx.x];
  for (int k = 0; k < 4; ++k) {
    const long long i = b0 + threadIdx.x * 4 + k;
    if (i < R) out[i] = run;
    run += v[k];
  }
}

// 5. fill the outputs; one warp per row.  Writes are bounded by the caller's capacities.
__global__ void k_fill(const uint8_t* __restrict__ masks, long long R, int nkb, Work w, calibatt_blocklist out) {
  const long long r = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= R) return;
  const long long n_pat = 1 + w.misc[1];
  const long long nnz_pat = w.misc[2];
  const long long nnz = w.misc[3];
  if (r == 0 && lane == 0) {
    if (out.pat_ptr != nullptr) {
      out.pat_ptr[0] = 0;
      if (n_pat <= out.n_pat) out.pat_ptr[n_pat] = static_cast<int32_t>(nnz_pat);
    }
    if (out.csr_row_ptr != nullptr) out.csr_row_ptr[R] = nnz;
  }
  const int c = w.cnt[r];
  const int f = w.first[r];
  const int fo = w.focc[r];
  if (lane == 0) {
    out.row_base[r] = c > 0 ? f : 0;
    long long p = 0;
    if (c > 0) p = 1 + w.pid[fo];
    out.row_pat[r] = static_cast<int32_t>(p < out.n_pat ? p : 0);
    if (fo == r && p < out.n_pat) out.pat_ptr[p] = static_cast<int32_t>(w.pstart[r]);
    if (out.csr_row_ptr != nullptr) out.csr_row_ptr[r] = w.rowptr[r];
  }
  if (c == 0) return;
  const uint8_t* row = masks + r * nkb;
  const bool uniq = (fo == r);
  const long long pbase = w.pstart[r];
  const long long cbase = w.rowptr[r];
  int done = 0;
  for (int j0 = 0; j0 < nkb; j0 += 32) {
    const int j = j0 + lane;
    const bool b = j < nkb && row[j] != 0;
    const unsigned bal = __ballot_sync(0xffffffffu, b);
    if (b) {
      const int i = done + __popc(bal & ((1u << lane) - 1u));
      if (uniq && pbase + i < out.nnz_pat) out.pat_off[pbase + i] = static_cast<int16_t>(j - f);
      if (out.csr_col != nullptr && cbase + i < out.nnz) out.csr_col[cbase + i] = static_cast<int16_t>(j);
    }
    done += __popc(bal);
  }
}

size_t align_up(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

unsigned long long table_cap(long long R) {
  unsigned long long cap = 2;
  while (cap < 2ull * static_cast<unsigned long long>(R)) cap <<= 1;
  return cap;
}

struct Carve {
  char* base;
  size_t off = 0;
  template <typename T>
  T* take(size_t count) {
    T* p = reinterpret_cast<T*>(base + off);
    off = align_up(off + count * sizeof(T));
    return p;
  }
};

size_t carve_all(Work* w, char* base, long long R) {
  Carve cv{base};
  const long long P = (R + kScanItems - 1) / kScanItems;
  const unsigned long long cap = table_cap(R);
  Work t;
  t.cnt = cv.take<int32_t>(R);
  t.first = cv.take<int32_t>(R);
  t.hash = cv.take<unsigned long long>(R);
  t.focc = cv.take<int32_t>(R);
  t.pid = cv.take<long long>(R);
  t.pstart = cv.take<long long>(R);
  t.rowptr = cv.take<long long>(R + 1);
  t.tkeys = cv.take<unsigned long long>(cap);
  t.tvals = cv.take<int32_t>(cap);
  t.coll = cv.take<int32_t>(R);
  t.misc = cv.take<long long>(8);
  t.partials = cv.take<long long>(P + 1);
  t.cap = cap;
  if (w) *w = t;
  return cv.off;
}

int scan(long long R, int seq, long long* out, long long* total, const Work& w, cudaStream_t s) {
  const long long P = (R + kScanItems - 1) / kScanItems;
  k_scan_reduce<<<static_cast<unsigned>(P), 256, 0, s>>>(R, seq, w);
  k_scan_top<<<1, 1024, 0, s>>>(P, total, w);
  k_scan_apply<<<static_cast<unsigned>(P), 256, 0, s>>>(R, seq, out, w);
  count_launch(3);
  return check_launch("compile scan");
}

}  // namespace

size_t compile_workspace_bytes(long long rows, int /*nkb*/) { return carve_all(nullptr, nullptr, rows) + 256; }

int run_compile(const uint8_t* masks, int n_maps, int nqb, int nkb, int dedup, void* ws, size_t ws_bytes,
                calibatt_blocklist* out, int64_t totals[3], cudaStream_t s) {
  const long long R = static_cast<long long>(n_maps) * nqb;
  char* base = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~static_cast<uintptr_t>(255));
  Work w;
  const size_t need = carve_all(&w, base, R);
  if (need + static_cast<size_t>(base - static_cast<char*>(ws)) > ws_bytes)
    return set_error(CALIBATT_E_WORKSPACE, "compile workspace too small: need %zu bytes", need + 256);
  int rc;
  if (cudaMemsetAsync(w.misc, 0, 8 * sizeof(long long), s) != cudaSuccess) return check_launch("memset misc");
  const unsigned warp_blocks = static_cast<unsigned>((R * 32 + 255) / 256);
  const unsigned thr_blocks = static_cast<unsigned>((R + 255) / 256);
  const int weak = dedup == CALIBATT_DEDUP_HASH_WEAK ? 1 : 0;
  k_row_info<<<warp_blocks, 256, 0, s>>>(masks, R, nkb, weak, w);
  count_launch();
  if ((rc = check_launch("k_row_info"))) return rc;
  if (dedup == CALIBATT_DEDUP_NONE) {
    k_focc_identity<<<thr_blocks, 256, 0, s>>>(R, w);
    count_launch();
    if ((rc = check_launch("k_focc_identity"))) return rc;
  } else {
    if (cudaMemsetAsync(w.tkeys, 0xFF, w.cap * sizeof(unsigned long long), s) != cudaSuccess ||
        cudaMemsetAsync(w.tvals, 0x7F, w.cap * sizeof(int32_t), s) != cudaSuccess)
      return check_launch("memset table");
    k_hash_insert<<<thr_blocks, 256, 0, s>>>(R, w);
    k_hash_verify<<<warp_blocks, 256, 0, s>>>(masks, R, nkb, w);
    const unsigned cb = static_cast<unsigned>(R < 1024 ? (R > 0 ? R : 1) : 1024);
    k_collisions<<<cb, 256, 0, s>>>(masks, R, nkb, w);
    count_launch(3);
    if ((rc = check_launch("compile dedup"))) return rc;
  }
  if ((rc = scan(R, SEQ_FIRST, w.pid, &w.misc[1], w, s))) return rc;
  if ((rc = scan(R, SEQ_ULEN, w.pstart, &w.misc[2], w, s))) return rc;
  long long* rowptr = w.rowptr;
  if (out != nullptr && out->csr_row_ptr != nullptr) rowptr = reinterpret_cast<long long*>(out->csr_row_ptr);
  Work wf = w;
  wf.rowptr = rowptr;
  if ((rc = scan(R, SEQ_CNT, rowptr, &w.misc[3], wf, s))) return rc;
  if (out != nullptr) {
    k_fill<<<warp_blocks, 256, 0, s>>>(masks, R, nkb, wf, *out);
    count_launch();
    if ((rc = check_launch("k_fill"))) return rc;
  }
  long long host_misc[8];
  if (cudaMemcpyAsync(host_misc, w.misc, sizeof(host_misc), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return check_launch("copy compile sizes");
  if (cudaStreamSynchronize(s) != cudaSuccess) return check_launch("compile sync");
  totals[0] = host_misc[3];         // nnz
  totals[1] = 1 + host_misc[1];     // patterns incl. the empty one
  totals[2] = host_misc[2];         // pattern-pool length
  return CALIBATT_OK;
}

}  // namespace calibatt
