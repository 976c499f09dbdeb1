// Cross-row de-duplication of the gathered clusters for batched decodes
// (FlashHead write-up, section 4.2: rows of a batch share cluster
// selections; balanced clusters and the C2T map, section 1.2.1; stage-2
// logits in full precision, section 1.2.4).
//
// After the per-row selection, the B x p chosen (row, cluster) pairs are
// grouped by cluster (CSR: counts, one scan that also lists the union U of
// chosen clusters, fill). Then every cluster k of U is handled once: its b
// token rows are read from HBM once, however many rows chose it, and
// multiplied with the hidden rows R_k that chose it on the tensor cores
// (mma.sync m16n8k16, bf16 in, fp32 accumulate: 16 token slots x 8 hidden
// rows per tile, K = d). A cluster's tile is a handful of hidden rows, far
// below the 64- or 128-row minimum of a tcgen05 MMA, so the warp-level MMA
// keeps the work exact instead of padding it 4-8x. Fragments are loaded
// straight from global memory (token rows once, hidden rows from L2).
// Outputs: the packed (logit, token) maximum of every row (64-bit
// atomicMax), and, when sampling, every logit at its canonical position in
// the row (rank of k among the row's ascending clusters, then slot).
#include <algorithm>

#include "fh_device.cuh"

namespace fh {
namespace {

// ---------------------------------------------------------------------------
// CSR of the selections
// ---------------------------------------------------------------------------
__global__ void csr_count_kernel(const GroupParams P) {
  const long long n = static_cast<long long>(P.B) * P.p;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int k = P.sel[i];
    if (static_cast<unsigned>(k) < static_cast<unsigned>(P.c)) atomicAdd(P.cnt + k, 1u);
  }
}

// One CTA: exclusive scan of the c counts into off[0..c], the union list
// (clusters with a nonzero count, ascending) and its length. Thread t owns
// 32 consecutive ids, read and written as 16-byte vectors (c % 4 == 0), or
// one by one otherwise.
__global__ void __launch_bounds__(kThreads, 1) csr_scan_kernel(const GroupParams P) {
  __shared__ uint32_t wsum[kWarps], wsum2[kWarps];
  const int tid = threadIdx.x;
  constexpr int kPer = 32;
  uint32_t all_tot = 0, all_nz = 0, carry_o = 0, carry_u = 0;
  const bool vec = (P.c & 3) == 0;
  for (int base = 0; base < P.c; base += kPer * kThreads) {  // one pass for c <= 16384
    const int k0 = base + tid * kPer;
    uint32_t v[kPer];
    if (vec && k0 + kPer <= P.c) {
#pragma unroll
      for (int j = 0; j < kPer; j += 4) {
        const uint4 x = *reinterpret_cast<const uint4*>(P.cnt + k0 + j);
        v[j] = x.x; v[j + 1] = x.y; v[j + 2] = x.z; v[j + 3] = x.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < kPer; ++j) v[j] = k0 + j < P.c ? P.cnt[k0 + j] : 0u;
    }
    uint32_t tot = 0, nz = 0;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      tot += v[j];
      nz += v[j] ? 1u : 0u;
    }
    uint32_t ptot, pnz;
    uint32_t o = carry_o + block_scan_excl_u32(tot, wsum, &ptot);
    uint32_t u = carry_u + block_scan_excl_u32(nz, wsum2, &pnz);
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int k = k0 + j;
      if (k < P.c) {
        P.off[k] = o;
        if (v[j]) P.ulist[u++] = k;
      }
      o += v[j];
    }
    carry_o += ptot;
    carry_u += pnz;
    __syncthreads();
  }
  all_tot = carry_o;
  all_nz = carry_u;
  for (int k = tid; k < P.c; k += kThreads) P.cur[k] = 0u;
  if (tid == 0) {
    P.off[P.c] = all_tot;
    *P.union_count = all_nz;
    *P.next = 0u;
  }
}

__global__ void csr_fill_kernel(const GroupParams P) {
  const long long n = static_cast<long long>(P.B) * P.p;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int k = P.sel[i];
    if (static_cast<unsigned>(k) >= static_cast<unsigned>(P.c)) continue;
    const uint32_t at = P.off[k] + atomicAdd(P.cur + k, 1u);
    P.rows_of[at] = static_cast<int32_t>(i / P.p);
  }
}

// ---------------------------------------------------------------------------
// grouped candidate logits
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Eight consecutive bf16 of a row from element k (k % 8 == 0, d % 8 == 0: a
// chunk never straddles d); zeros past the row's end.
__device__ __forceinline__ uint4 ld_chunk(const uint16_t* p, int k, int d) {
  return k < d ? __ldg(reinterpret_cast<const uint4*>(p + k)) : make_uint4(0, 0, 0, 0);
}

// Position of cluster k among the row's ascending clusters (binary search).
__device__ __forceinline__ int rank_in_row(const int32_t* sel, int p, int k) {
  int lo = 0, hi = p - 1;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (sel[mid] < k) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

constexpr int kChunks = 4;  // 8-row chunks of R_k per pass (32 hidden rows)

__global__ void __launch_bounds__(256) group_kernel(const GroupParams P) {
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;  // mma fragment coordinates
  const int d = P.d, b = P.b;
  const uint32_t nu = *P.union_count;
  for (;;) {
    uint32_t ui = 0;
    if (lane == 0) ui = atomicAdd(P.next, 1u);
    ui = __shfl_sync(0xFFFFFFFFu, ui, 0);
    if (ui >= nu) break;
    const int k = P.ulist[ui];
    const int r0 = static_cast<int>(P.off[k]), r1 = static_cast<int>(P.off[k + 1]);
    // token slots g and g + 8 of cluster k (b == 16: one m16 tile)
    const int tok_a = __ldg(P.C2T + static_cast<size_t>(k) * b + g);
    const int tok_b = __ldg(P.C2T + static_cast<size_t>(k) * b + g + 8);
    const uint16_t* ea = P.E + static_cast<size_t>(tok_a) * d;
    const uint16_t* eb = P.E + static_cast<size_t>(tok_b) * d;
    for (int rb = r0; rb < r1; rb += 8 * kChunks) {
      const int nch = min(kChunks, (r1 - rb + 7) / 8);
      // hidden row of fragment column g in each chunk (rows past the cluster's list repeat a valid row)
      const uint16_t* hrow[kChunks];
#pragma unroll
      for (int ch = 0; ch < kChunks; ++ch) {
        const int idx = min(rb + ch * 8 + g, r1 - 1);
        hrow[ch] = P.H + static_cast<size_t>(P.rows_of[idx]) * d;
      }
      float acc[kChunks][4];
#pragma unroll
      for (int ch = 0; ch < kChunks; ++ch) acc[ch][0] = acc[ch][1] = acc[ch][2] = acc[ch][3] = 0.f;
      // The dot product over K is order-free, so two MMA K-steps take 32
      // elements in a lane-friendly order: lane t of a fragment row loads the
      // 8 contiguous elements [k0 + 8t, k0 + 8t + 8); the first K-step uses
      // elements 8t..8t+3 (as its columns 2t, 2t+1, 2t+8, 2t+9), the second
      // 8t+4..8t+7. A and B use the same order, so the sums are unchanged.
#pragma unroll 2
      for (int k0 = 0; k0 < d; k0 += 32) {
        const int kk = k0 + 8 * t;
        const uint4 xa = ld_chunk(ea, kk, d), xb = ld_chunk(eb, kk, d);
        uint4 xh[kChunks];
#pragma unroll
        for (int ch = 0; ch < kChunks; ++ch) xh[ch] = ch < nch ? ld_chunk(hrow[ch], kk, d) : make_uint4(0, 0, 0, 0);
        const uint32_t a0[4] = {xa.x, xb.x, xa.y, xb.y};
        const uint32_t a1[4] = {xa.z, xb.z, xa.w, xb.w};
#pragma unroll
        for (int ch = 0; ch < kChunks; ++ch) {
          if (ch < nch) {
            mma_16816(acc[ch], a0, xh[ch].x, xh[ch].y);
            mma_16816(acc[ch], a1, xh[ch].z, xh[ch].w);
          }
        }
      }
      // acc[ch]: (slot g, col 2t), (slot g, col 2t+1), (slot g+8, col 2t), (slot g+8, col 2t+1)
#pragma unroll
      for (int ch = 0; ch < kChunks; ++ch) {
        if (ch >= nch) break;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int ri = rb + ch * 8 + 2 * t + cc;  // position in the cluster's row list
          const bool rv = ri < r1;
          const int row = rv ? P.rows_of[ri] : 0;
          const float za = acc[ch][cc], zb = acc[ch][2 + cc];
          if (rv && P.logits) {
            const int pos = rank_in_row(P.sel + static_cast<size_t>(row) * P.p, P.p, k) * b;
            float* zr = P.logits + static_cast<size_t>(row) * P.p * b + pos;
            zr[g] = za;
            zr[g + 8] = zb;
          }
          unsigned long long pa = pack_best(za, tok_a), pb = pack_best(zb, tok_b);
          unsigned long long m = pa > pb ? pa : pb;
#pragma unroll
          for (int o = 4; o < 32; o <<= 1) {  // across the 8 slots g of this column
            const unsigned long long y = __shfl_xor_sync(0xFFFFFFFFu, m, o);
            m = y > m ? y : m;
          }
          if (g == 0 && rv) atomicMax(P.best + row, m);
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_group(const GroupParams& P, int num_sms, cudaStream_t st) {
  const long long n = static_cast<long long>(P.B) * P.p;
  const int gsz = static_cast<int>(std::min<long long>((n + 255) / 256, 4LL * num_sms));
  cudaError_t e = cudaMemsetAsync(P.cnt, 0, static_cast<size_t>(P.c) * 4, st);
  if (e != cudaSuccess) return e;
  csr_count_kernel<<<gsz, 256, 0, st>>>(P);
  csr_scan_kernel<<<1, kThreads, 0, st>>>(P);
  csr_fill_kernel<<<gsz, 256, 0, st>>>(P);
  group_kernel<<<num_sms * 8, 256, 0, st>>>(P);
  return cudaGetLastError();
}

}  // namespace fh
