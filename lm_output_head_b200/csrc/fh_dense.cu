// Dense comparison head z = E h with a fused argmax (FlashHead write-up,
// section 1.1: the classification head as one v x d matrix product).
//
// One persistent launch, two 512-thread CTAs per SM: the v token rows are
// spread round-robin over all warps; a warp streams a row HBM -> registers
// with non-allocating 16-byte loads and dots it with every hidden row of the
// launch, staged once per CTA in shared memory as fp32. Per-row maxima are
// packed (logit, token) words, merged per CTA and then with one 64-bit
// atomicMax; the last CTA to finish writes the argmax and clears the
// accumulators.
#include "fh_device.cuh"

namespace fh {
namespace {

constexpr int kDenseMaxRows = 8;

template <int NCH>
__global__ void __launch_bounds__(kThreads, 2) dense_kernel(const DenseParams P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ unsigned long long wbest[kWarps][kDenseMaxRows];
  __shared__ int s_last;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = gridDim.x, W = G * kWarps, gw = blockIdx.x * kWarps + warp;
  const int d = P.d, R = P.rows;
  float* hs = reinterpret_cast<float*>(smem);  // [R][d]

  uint4 w[NCH];
  if (gw < P.v) row_load_bf16<NCH>(P.E + static_cast<size_t>(gw) * d, d, w);  // first row goes out first
  for (int r = 0; r < R; ++r) stage_h_f32(P.hidden + static_cast<size_t>(P.row0 + r) * d, d, hs + r * d);
  for (int i = tid; i < kWarps * kDenseMaxRows; i += kThreads) (&wbest[0][0])[i] = 0ull;
  __syncthreads();

  unsigned long long best[kDenseMaxRows];
#pragma unroll
  for (int r = 0; r < kDenseMaxRows; ++r) best[r] = 0ull;
  for (int t = gw; t < P.v; t += W) {
    if (t != gw) row_load_bf16<NCH>(P.E + static_cast<size_t>(t) * d, d, w);
#pragma unroll
    for (int r = 0; r < kDenseMaxRows; ++r) {
      if (r < R) {
        const float z = row_dot_bf16_hs<NCH>(w, hs + r * d, d);
        const unsigned long long pk = pack_best(z, t);
        best[r] = pk > best[r] ? pk : best[r];
        if (lane == 0 && P.logits) P.logits[static_cast<size_t>(P.row0 + r) * P.v + t] = z;
      }
    }
  }
  if (lane == 0)
#pragma unroll
    for (int r = 0; r < kDenseMaxRows; ++r) wbest[warp][r] = best[r];
  __syncthreads();
  for (int r = tid; r < R; r += kThreads) {
    unsigned long long m = 0ull;
    for (int i = 0; i < kWarps; ++i) m = wbest[i][r] > m ? wbest[i][r] : m;
    if (m) atomicMax(P.best + P.row0 + r, m);
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    s_last = atomicAdd(&P.sync->ticket, 1u) == static_cast<uint32_t>(G - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int r = tid; r < R; r += kThreads) {
    const unsigned long long bw = atomicExch(P.best + P.row0 + r, 0ull);
    P.out_argmax[P.row0 + r] = best_token(bw);
  }
  if (tid == 0) P.sync->ticket = 0u;
}

}  // namespace

cudaError_t launch_dense(const DenseParams& P, int grid, size_t smem, int nch, cudaStream_t st) {
  if (P.rows > kDenseMaxRows) return cudaErrorInvalidValue;
#define FH_L(N)                                                    \
  dense_kernel<N><<<grid, kThreads, smem, st>>>(P);                \
  return cudaGetLastError();
  switch (nch) {
    case 1: FH_L(1)
    case 2: FH_L(2)
    case 3: FH_L(3)
    case 4: FH_L(4)
    case 5: FH_L(5)
    case 6: FH_L(6)
    case 8: FH_L(8)
    case 10: FH_L(10)
    default: return cudaErrorInvalidValue;
  }
#undef FH_L
}

int dense_max_rows() { return kDenseMaxRows; }

cudaError_t occupancy_dense(int nch, size_t smem, int* blocks) {
  switch (nch) {
    case 1: return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks, dense_kernel<1>, kThreads, smem);
    case 2: return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks, dense_kernel<2>, kThreads, smem);
    case 3: return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks, dense_kernel<3>, kThreads, smem);
    case 4: return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks, dense_kernel<4>, kThreads, smem);
    case 5: return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks, dense_kernel<5>, kThreads, smem);
    case 6: return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks, dense_kernel<6>, kThreads, smem);
    case 8: return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks, dense_kernel<8>, kThreads, smem);
    case 10: return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks, dense_kernel<10>, kThreads, smem);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t set_attrs_dense(int max_smem) {
  cudaError_t e = cudaSuccess;
  auto set = [&](const void* f) {
    if (e == cudaSuccess) e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
  };
  set(reinterpret_cast<const void*>(dense_kernel<1>));
  set(reinterpret_cast<const void*>(dense_kernel<2>));
  set(reinterpret_cast<const void*>(dense_kernel<3>));
  set(reinterpret_cast<const void*>(dense_kernel<4>));
  set(reinterpret_cast<const void*>(dense_kernel<5>));
  set(reinterpret_cast<const void*>(dense_kernel<6>));
  set(reinterpret_cast<const void*>(dense_kernel<8>));
  set(reinterpret_cast<const void*>(dense_kernel<10>));
  return e;
}

// ----------------------------------------------------------------------------
// create-time utilities
// ----------------------------------------------------------------------------
namespace {

__global__ void c2t_count_kernel(const C2TCheckParams P) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < P.n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int t = P.C2T.at(static_cast<size_t>(i));
    if (t < 0 || t >= P.v) atomicExch(P.bad, 1);
    else atomicAdd(P.counts + t, 1u);
  }
}

__global__ void c2t_verify_kernel(const C2TCheckParams P) {
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < P.v; t += gridDim.x * blockDim.x)
    if (P.counts[t] != 1u) atomicExch(P.bad, 1);
}

// Packed row k: [qb code bytes][d/16 scale bytes][zero pad to rs] (INT4: qb = d/2, INT8: qb = d).
__global__ void repack_kernel(const RepackParams P) {
  const long long total = static_cast<long long>(P.c) * P.rs;
  const int qb = P.qb, sb = P.d / 16;
  const uint8_t* scales = reinterpret_cast<const uint8_t*>(P.C_scales);
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long k = i / P.rs;
    const int o = static_cast<int>(i - k * P.rs);
    uint8_t v = 0;
    if (o < qb) v = P.C_q[k * qb + o];
    else if (o < qb + sb) v = scales[k * sb + (o - qb)];
    P.out[i] = v;
  }
}

// Cluster-major copy of E: row r = k*b + j holds E[C2T[k][j]] (C2T already
// verified to be a permutation of 0..v-1), 16 bytes per thread step.
__global__ void gather_cluster_major_kernel(const uint16_t* E, const C2TView C2T, uint16_t* out, int v, int d) {
  const int chunks = d / 8;
  const long long total = static_cast<long long>(v) * chunks;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / chunks;
    const int q = static_cast<int>(i - r * chunks);
    const int t = C2T.at(static_cast<size_t>(r));
    reinterpret_cast<uint4*>(out + r * d)[q] = __ldg(reinterpret_cast<const uint4*>(E + static_cast<size_t>(t) * d) + q);
  }
}

}  // namespace

cudaError_t launch_gather_cluster_major(const uint16_t* E, C2TView C2T, uint16_t* out, int v, int d,
                                        cudaStream_t st) {
  gather_cluster_major_kernel<<<2048, 256, 0, st>>>(E, C2T, out, v, d);
  return cudaGetLastError();
}

cudaError_t launch_c2t_check(const C2TCheckParams& P, cudaStream_t st) {
  c2t_count_kernel<<<1024, 256, 0, st>>>(P);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  c2t_verify_kernel<<<1024, 256, 0, st>>>(P);
  return cudaGetLastError();
}

cudaError_t launch_repack(const RepackParams& P, cudaStream_t st) {
  repack_kernel<<<1024, 256, 0, st>>>(P);
  return cudaGetLastError();
}

}  // namespace fh
