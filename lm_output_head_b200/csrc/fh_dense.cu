// Dense comparison head z = E h with a fused argmax (FlashHead write-up,
// section 1.1: the classification head as one v x d matrix product).
//
// One persistent launch of one 512-thread CTA per SM: the v token rows are
// spread round-robin over all warps, each streamed HBM -> shared memory once
// with cp.async.bulk through a per-warp ring and dotted with every hidden row
// of the launch. For B = 1 the hidden state lives in registers; otherwise the
// block of hidden rows lives in shared memory. Per-row maxima are packed
// (logit, token) words, merged per CTA and then with one 64-bit atomicMax;
// the last CTA to finish writes the argmax and clears the accumulators.
#include "fh_device.cuh"

namespace fh {
namespace {

constexpr int kDenseMaxRows = 32;

template <int NCH, bool ONE>
__global__ void __launch_bounds__(kThreads, 1) dense_kernel(const DenseParams P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ unsigned long long wbest[kWarps][kDenseMaxRows];
  __shared__ int s_last;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = gridDim.x, W = G * kWarps, gw = blockIdx.x * kWarps + warp;
  const int d = P.d, R = P.rows;
  uint16_t* sh = reinterpret_cast<uint16_t*>(smem + P.off_h);
  const uint32_t sh_a = smem_addr(sh);
  const uint32_t ring_w = smem_addr(smem + P.off_ring) + static_cast<uint32_t>(warp * P.nslot * P.slot_bytes);
  const uint32_t bar_w = smem_addr(smem + P.off_bar) + static_cast<uint32_t>(warp * P.nslot * 8);

  const int n = gw < P.v ? (P.v - 1 - gw) / W + 1 : 0;
  uint32_t phase_bits = 0;
  auto src = [&](int i, const void*& ptr, uint32_t& bytes) {
    ptr = P.E + static_cast<size_t>(gw + i * W) * d;
    bytes = static_cast<uint32_t>(d * 2);
  };
  // first copies go out before the hidden rows are staged
  warp_ring_init(bar_w, P.nslot);
  warp_stream_prologue(n, P.nslot, ring_w, P.slot_bytes, bar_w, src);
  const uint4* hsrc = reinterpret_cast<const uint4*>(P.hidden + static_cast<size_t>(P.row0) * d);
  for (int i = tid; i < R * d / 8; i += kThreads) reinterpret_cast<uint4*>(sh)[i] = hsrc[i];
  for (int i = tid; i < kWarps * kDenseMaxRows; i += kThreads) (&wbest[0][0])[i] = 0ull;
  __syncthreads();
  bool ok;
  if constexpr (ONE) {
    float hr[NCH * 8];
    load_h_chunks<NCH>(sh, d, hr);
    unsigned long long best = 0ull;
    auto use = [&](int i, uint32_t slot) {
      const int t = gw + i * W;
      const float z = row_dot_bf16<NCH>(slot, d, hr);
      const unsigned long long pk = pack_best(z, t);
      best = pk > best ? pk : best;
      if (lane == 0 && P.logits) P.logits[static_cast<size_t>(P.row0) * P.v + t] = z;
    };
    ok = warp_stream_run(n, P.nslot, ring_w, P.slot_bytes, bar_w, phase_bits, kWaitBudget, src, use);
    if (lane == 0) wbest[warp][0] = best;
  } else {
    auto use = [&](int i, uint32_t slot) {
      const int t = gw + i * W;
      uint4 ew[NCH];
#pragma unroll
      for (int m = 0; m < NCH; ++m) {
        const int e = (lane + 32 * m) * 8;
        ew[m] = e < d ? lds128(slot + 2u * e) : make_uint4(0, 0, 0, 0);
      }
      for (int r = 0; r < R; ++r) {
        const uint32_t hrow = sh_a + static_cast<uint32_t>(r * d * 2);
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < NCH; ++m) {
          const int e = (lane + 32 * m) * 8;
          if (e < d) {
            const uint4 hv = lds128(hrow + 2u * e);
            acc = fmaf(bf16lo(ew[m].x), bf16lo(hv.x), acc);
            acc = fmaf(bf16hi(ew[m].x), bf16hi(hv.x), acc);
            acc = fmaf(bf16lo(ew[m].y), bf16lo(hv.y), acc);
            acc = fmaf(bf16hi(ew[m].y), bf16hi(hv.y), acc);
            acc = fmaf(bf16lo(ew[m].z), bf16lo(hv.z), acc);
            acc = fmaf(bf16hi(ew[m].z), bf16hi(hv.z), acc);
            acc = fmaf(bf16lo(ew[m].w), bf16lo(hv.w), acc);
            acc = fmaf(bf16hi(ew[m].w), bf16hi(hv.w), acc);
          }
        }
        const float z = warp_sum(acc);
        if (lane == 0) {
          const unsigned long long pk = pack_best(z, t);
          if (pk > wbest[warp][r]) wbest[warp][r] = pk;
          if (P.logits) P.logits[static_cast<size_t>(P.row0 + r) * P.v + t] = z;
        }
      }
    };
    ok = warp_stream_run(n, P.nslot, ring_w, P.slot_bytes, bar_w, phase_bits, kWaitBudget, src, use);
  }
  if (!ok && lane == 0) record_error(&P.sync->status, FH_ERR_TIMEOUT);
  __syncthreads();
  for (int r = tid; r < R; r += kThreads) {
    unsigned long long m = 0ull;
    for (int w = 0; w < kWarps; ++w) m = wbest[w][r] > m ? wbest[w][r] : m;
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
  const bool one = P.rows == 1;
#define FH_L(N)                                                       \
  if (one) dense_kernel<N, true><<<grid, kThreads, smem, st>>>(P);    \
  else dense_kernel<N, false><<<grid, kThreads, smem, st>>>(P);       \
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

cudaError_t set_attrs_dense(int max_smem) {
  cudaError_t e = cudaSuccess;
  auto set = [&](const void* f) {
    if (e == cudaSuccess) e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
  };
#define FH_S(N)                                                   \
  set(reinterpret_cast<const void*>(dense_kernel<N, true>));      \
  set(reinterpret_cast<const void*>(dense_kernel<N, false>));
  FH_S(1) FH_S(2) FH_S(3) FH_S(4) FH_S(5) FH_S(6) FH_S(8) FH_S(10)
#undef FH_S
  return e;
}

// ----------------------------------------------------------------------------
// create-time utilities
// ----------------------------------------------------------------------------
namespace {

__global__ void c2t_count_kernel(const C2TCheckParams P) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < P.n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int t = P.C2T[i];
    if (t < 0 || t >= P.v) atomicExch(P.bad, 1);
    else atomicAdd(P.counts + t, 1u);
  }
}

__global__ void c2t_verify_kernel(const C2TCheckParams P) {
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < P.v; t += gridDim.x * blockDim.x)
    if (P.counts[t] != 1u) atomicExch(P.bad, 1);
}

// Packed INT4 row k: [d/2 code bytes][d/16 scale bytes][zero pad to rs].
__global__ void repack_int4_kernel(const RepackParams P) {
  const long long total = static_cast<long long>(P.c) * P.rs;
  const int qb = P.d / 2, sb = P.d / 16;
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

}  // namespace

cudaError_t launch_c2t_check(const C2TCheckParams& P, cudaStream_t st) {
  c2t_count_kernel<<<1024, 256, 0, st>>>(P);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  c2t_verify_kernel<<<1024, 256, 0, st>>>(P);
  return cudaGetLastError();
}

cudaError_t launch_repack_int4(const RepackParams& P, cudaStream_t st) {
  repack_int4_kernel<<<1024, 256, 0, st>>>(P);
  return cudaGetLastError();
}

}  // namespace fh
