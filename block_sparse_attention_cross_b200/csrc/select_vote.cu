// select_vote.cu -- per-query-block selection of key blocks and agreement voting.
//
// CalibAtt paper page, Figure 5(a): the top key blocks of every query block
// are thresholded, and the masks of the calibration prompts are aggregated;
// Figure 3(b): the keep frequency of a block across prompts; Figure 7: the
// agreement threshold rho.  Order used for "top": energy descending, then key
// block index ascending (a strict total order, so the selection is unique).
// TOPK keeps the first k blocks of that order.  ENERGY keeps the shortest
// prefix whose float64 running sum (in selection order) reaches
// (1 - eps) * (float64 sum of the row in index order), the crossing block
// included (Figure S8 energy threshold).
#include "common.cuh"
#include "internal.h"

namespace calibatt {
namespace {

constexpr int kSelThreads = 256;
constexpr int kSelMax = 2048;

// One CTA per (head, query block) row.
__global__ void __launch_bounds__(kSelThreads) k_select_vote(const float* __restrict__ energy, int nkb, int mode,
                                                             int topk, double eps, int32_t* __restrict__ votes,
                                                             float* __restrict__ esum) {
  __shared__ float e[kSelMax];
  __shared__ short order[kSelMax];
  __shared__ unsigned char keep[kSelMax];
  const size_t row = blockIdx.x;
  const float* er = energy + row * nkb;
  for (int j = threadIdx.x; j < nkb; j += kSelThreads) {
    e[j] = er[j];
    keep[j] = 0;
  }
  __syncthreads();
  for (int j = threadIdx.x; j < nkb; j += kSelThreads) {
    const float ej = e[j];
    int rank = 0;
    for (int i = 0; i < nkb; ++i) {
      const float ei = e[i];
      rank += (ei > ej) || (ei == ej && i < j);
    }
    if (mode == CALIBATT_SELECT_TOPK) {
      keep[j] = rank < topk ? 1 : 0;
    } else {
      order[rank] = static_cast<short>(j);
    }
  }
  __syncthreads();
  if (mode == CALIBATT_SELECT_ENERGY && threadIdx.x == 0) {
    double total = 0.0;
    for (int j = 0; j < nkb; ++j) total += static_cast<double>(e[j]);
    const double target = (1.0 - eps) * total;
    double run = 0.0;
    for (int r = 0; r < nkb; ++r) {
      const int j = order[r];
      keep[j] = 1;
      run += static_cast<double>(e[j]);
      if (run >= target) break;
    }
  }
  __syncthreads();
  int32_t* vr = votes + row * nkb;
  float* sr = esum + row * nkb;
  for (int j = threadIdx.x; j < nkb; j += kSelThreads) {
    vr[j] += keep[j];
    sr[j] = sr[j] + e[j];
  }
}

// mask = votes >= min_votes; an empty row keeps its best block by
// (votes desc, energy sum desc, index asc).
__global__ void __launch_bounds__(kSelThreads) k_finalize(const int32_t* __restrict__ votes,
                                                          const float* __restrict__ esum, int nkb, int min_votes,
                                                          uint8_t* __restrict__ mask) {
  __shared__ int bv[kSelThreads];
  __shared__ float be[kSelThreads];
  __shared__ int bj[kSelThreads];
  const size_t row = blockIdx.x;
  const int32_t* vr = votes + row * nkb;
  const float* sr = esum + row * nkb;
  uint8_t* mr = mask + row * nkb;
  int any = 0;
  int cv = -1, cj = 0x7fffffff;
  float ce = -INFINITY;
  for (int j = threadIdx.x; j < nkb; j += kSelThreads) {
    const int vv = vr[j];
    const float ee = sr[j];
    const uint8_t kk = vv >= min_votes ? 1 : 0;
    mr[j] = kk;
    any |= kk;
    const bool better = (vv > cv) || (vv == cv && (ee > ce || (ee == ce && j < cj)));
    if (better) {
      cv = vv;
      ce = ee;
      cj = j;
    }
  }
  if (__syncthreads_or(any)) return;
  bv[threadIdx.x] = cv;
  be[threadIdx.x] = ce;
  bj[threadIdx.x] = cj;
  __syncthreads();
  for (int w = kSelThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) {
      const int ov = bv[threadIdx.x + w], oj = bj[threadIdx.x + w];
      const float oe = be[threadIdx.x + w];
      const int mv = bv[threadIdx.x], mj = bj[threadIdx.x];
      const float me = be[threadIdx.x];
      if ((ov > mv) || (ov == mv && (oe > me || (oe == me && oj < mj)))) {
        bv[threadIdx.x] = ov;
        be[threadIdx.x] = oe;
        bj[threadIdx.x] = oj;
      }
    }
    __syncthreads();
  }
  if (threadIdx.x == 0 && bj[0] >= 0 && bj[0] < nkb) mr[bj[0]] = 1;
}

}  // namespace

int launch_select_vote(const float* energy, int rows, int nkb, int mode, int topk, double eps, int32_t* votes,
                       float* esum, cudaStream_t s) {
  if (rows == 0) return CALIBATT_OK;
  k_select_vote<<<rows, kSelThreads, 0, s>>>(energy, nkb, mode, topk, eps, votes, esum);
  count_launch();
  return check_launch("k_select_vote");
}

int launch_finalize(const int32_t* votes, const float* esum, int rows, int nkb, int min_votes, uint8_t* mask,
                    cudaStream_t s) {
  if (rows == 0) return CALIBATT_OK;
  k_finalize<<<rows, kSelThreads, 0, s>>>(votes, esum, nkb, min_votes, mask);
  count_launch();
  return check_launch("k_finalize");
}

}  // namespace calibatt
