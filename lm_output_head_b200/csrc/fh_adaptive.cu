// Adaptive probe count (write-up section 1.2.2, "dynamic adjustment"; section
// 4.2: fewer probes for frequent tokens): for each row of centroid scores,
// the smallest p in [p_min, p_max] whose top-p clusters hold at least a
// fraction tau of softmax(s / T) over all c clusters.
//
// One CTA per row: the row's scores are sorted in shared memory (bitonic,
// descending, padded to a power of two with -inf), their softmax weights are
// scanned in that order, and the first prefix reaching tau * total gives p.
// The mass of the top p depends only on the p largest values, so the order
// of equal scores does not matter.
#include <climits>

#include "fh_device.cuh"

namespace fh {
namespace {

constexpr int kAdaptThreads = 1024;

struct AdaptParams {
  const float* scores;  // [B, c]
  int32_t* out_p;       // [B]
  int c, npow2, p_min, p_max;
  float tau, T;
};

__global__ void __launch_bounds__(kAdaptThreads) adaptive_probes_kernel(const AdaptParams P) {
  extern __shared__ float ks[];  // [npow2]
  __shared__ float scr[kAdaptThreads / 32 + 1];
  __shared__ int first;
  const int tid = threadIdx.x, r = blockIdx.x, n = P.npow2;
  const float* s = P.scores + static_cast<size_t>(r) * P.c;
  for (int i = tid; i < n; i += kAdaptThreads) ks[i] = i < P.c ? s[i] : -INFINITY;
  if (tid == 0) first = INT_MAX;
  __syncthreads();
  // bitonic sort, descending
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < n; i += kAdaptThreads) {
        const int l = i ^ j;
        if (l > i) {
          const float a = ks[i], b = ks[l];
          const bool desc = (i & k) == 0;
          if (desc ? a < b : a > b) {
            ks[i] = b;
            ks[l] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  // softmax weights in sorted order: contiguous ranges per thread, block scan
  const float m = ks[0];
  const float invT = 1.f / P.T;
  const int per = (P.c + kAdaptThreads - 1) / kAdaptThreads;
  const int i0 = min(P.c, tid * per), i1 = min(P.c, i0 + per);
  float loc = 0.f;
  for (int i = i0; i < i1; ++i) loc += expf((ks[i] - m) * invT);
  float total;
  const float before = block_exclusive_scan<kAdaptThreads, float>(loc, scr, &total);
  const float target = P.tau * total;
  float run = before;
  for (int i = i0; i < i1; ++i) {
    run += expf((ks[i] - m) * invT);
    if (run >= target) {
      atomicMin(&first, i);
      break;
    }
  }
  __syncthreads();
  if (tid == 0) {
    const int p = first == INT_MAX ? P.c : first + 1;  // rounding at tau = 1: all clusters
    P.out_p[r] = min(max(p, P.p_min), P.p_max);
  }
}

}  // namespace

cudaError_t launch_adaptive_probes(const float* scores, int B, int c, float tau, int p_min, int p_max, float T,
                                   int32_t* out_p, cudaStream_t st) {
  int npow2 = 1;
  while (npow2 < c) npow2 <<= 1;
  const size_t smem = static_cast<size_t>(npow2) * 4;
  if (smem > 200 * 1024) return cudaErrorInvalidValue;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(adaptive_probes_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  AdaptParams P{scores, out_p, c, npow2, p_min, p_max, tau, T};
  adaptive_probes_kernel<<<B, kAdaptThreads, smem, st>>>(P);
  return cudaGetLastError();
}

}  // namespace fh
