// Speculative drafting with FlashHead (write-up section 4.2): a token drafted
// from FlashHead's candidates is checked against the dense head.
//
// Standard speculative sampling with the draft law taken given the chosen
// clusters: q = softmax(z/T) over the draft's candidate tokens (zero
// elsewhere), p = softmax(z/T) over the whole vocabulary. The draft x is kept
// when u_accept < p(x) / q(x); otherwise the token is drawn by inverse CDF in
// token order from max(0, p - q). For every cluster set the result follows p
// exactly.
//
// One CTA per row: a bitmap of the candidates in shared memory, block
// reductions for the two normalisers, and when the draft is rejected a
// block scan of the residual over contiguous token ranges.
#include <climits>

#include "fh_device.cuh"

namespace fh {
namespace {

constexpr int kSpecThreads = 1024;

struct SpecParams {
  const float* logits;     // [B, v]
  const int32_t* cand;     // [B, n]
  const int32_t* draft;    // [B]
  const float* u_accept;   // [B]
  const float* u_resample; // [B]
  int32_t* out;            // [B]
  int* status;
  int v, n;
  float T;
};

__device__ __forceinline__ float block_max(float x, float* scr) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xFFFFFFFFu, x, o));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) scr[threadIdx.x >> 5] = x;
  __syncthreads();
  float m = scr[0];
  for (int i = 1; i < kSpecThreads / 32; ++i) m = fmaxf(m, scr[i]);
  return m;
}

__device__ __forceinline__ float block_sum(float x, float* scr) {
  x = warp_sum(x);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) scr[threadIdx.x >> 5] = x;
  __syncthreads();
  float s = 0.f;
  for (int i = 0; i < kSpecThreads / 32; ++i) s += scr[i];
  return s;
}

__global__ void __launch_bounds__(kSpecThreads) spec_verify_kernel(const SpecParams P) {
  extern __shared__ uint32_t in_cand[];  // [ceil(v / 32)] candidate bitmap
  __shared__ float scr[kSpecThreads / 32 + 1];
  __shared__ int pick, fallback, bad;
  const int tid = threadIdx.x, r = blockIdx.x;
  const float* z = P.logits + static_cast<size_t>(r) * P.v;
  const int32_t* cand = P.cand + static_cast<size_t>(r) * P.n;
  const int words = (P.v + 31) / 32;
  const float invT = 1.f / P.T;
  for (int i = tid; i < words; i += kSpecThreads) in_cand[i] = 0u;
  if (tid == 0) {
    pick = INT_MAX;
    fallback = -1;
    bad = 0;
  }
  __syncthreads();
  float mq = -INFINITY;
  for (int i = tid; i < P.n; i += kSpecThreads) {
    const int t = cand[i];
    if (t < 0 || t >= P.v) {
      bad = 1;
      continue;
    }
    atomicOr(&in_cand[t >> 5], 1u << (t & 31));
    mq = fmaxf(mq, z[t]);
  }
  float m = -INFINITY;
  for (int t = tid; t < P.v; t += kSpecThreads) m = fmaxf(m, z[t]);
  m = block_max(m, scr);
  mq = block_max(mq, scr);
  const int x = P.draft[r];
  if (bad || x < 0 || x >= P.v || !((in_cand[x >> 5] >> (x & 31)) & 1u)) {
    if (tid == 0) {
      record_error(P.status, FH_ERR_OUT_OF_RANGE);
      P.out[r] = -1;
    }
    return;
  }
  // normalisers of p (vocabulary) and q (candidates)
  float zp = 0.f, zq = 0.f;
  for (int t = tid; t < P.v; t += kSpecThreads) zp += expf((z[t] - m) * invT);
  for (int i = tid; i < P.n; i += kSpecThreads) zq += expf((z[cand[i]] - mq) * invT);
  zp = block_sum(zp, scr);
  zq = block_sum(zq, scr);
  const float px = expf((z[x] - m) * invT) / zp;
  const float qx = expf((z[x] - mq) * invT) / zq;
  if (P.u_accept[r] < px / qx) {
    if (tid == 0) P.out[r] = x;
    return;
  }
  // rejected: inverse CDF of max(0, p - q) over contiguous token ranges
  const int per = (P.v + kSpecThreads - 1) / kSpecThreads;
  const int t0 = min(P.v, tid * per), t1 = min(P.v, t0 + per);
  auto resid = [&](int t) {
    const float pt = expf((z[t] - m) * invT) / zp;
    const bool c = (in_cand[t >> 5] >> (t & 31)) & 1u;
    const float qt = c ? expf((z[t] - mq) * invT) / zq : 0.f;
    return fmaxf(pt - qt, 0.f);
  };
  float loc = 0.f;
  for (int t = t0; t < t1; ++t) loc += resid(t);
  __syncthreads();  // every thread has read the reduction scratch the scan reuses
  float total;
  const float before = block_exclusive_scan<kSpecThreads, float>(loc, scr, &total);
  const float u = fminf(fmaxf(P.u_resample[r], 0.f), 0.99999994f);
  const float target = u * total;
  float run = before;
  int claim = INT_MAX, last = -1;
  for (int t = t0; t < t1; ++t) {
    const float w = resid(t);
    if (w > 0.f) last = t;
    run += w;
    if (run > target && w > 0.f) {
      claim = t;
      break;
    }
  }
  if (claim != INT_MAX) atomicMin(&pick, claim);
  if (last >= 0) atomicMax(&fallback, last);
  __syncthreads();
  if (tid == 0) P.out[r] = pick != INT_MAX ? pick : (fallback >= 0 ? fallback : x);
}

}  // namespace

cudaError_t launch_spec_verify(const float* logits, int v, const int32_t* cand, int n, int B, const int32_t* draft,
                               float T, const float* u_accept, const float* u_resample, int32_t* out, int* status,
                               cudaStream_t st) {
  const size_t smem = static_cast<size_t>((v + 31) / 32) * 4;
  if (smem > 200 * 1024) return cudaErrorInvalidValue;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(spec_verify_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  SpecParams P{logits, cand, draft, u_accept, u_resample, out, status, v, n, T};
  spec_verify_kernel<<<B, kSpecThreads, smem, st>>>(P);
  return cudaGetLastError();
}

}  // namespace fh
