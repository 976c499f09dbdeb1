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
// (clusters with a nonzero count, ascending) and its length.
__global__ void __launch_bounds__(kThreads, 1) csr_scan_kernel(const GroupParams P) {
  __shared__ uint32_t wsum[kWarps], wsum2[kWarps];
  const int tid = threadIdx.x;
  const int per = (P.c + kThreads - 1) / kThreads;
  const int k0 = min(P.c, tid * per), k1 = min(P.c, k0 + per);
  uint32_t tot = 0, nz = 0;
  for (int k = k0; k < k1; ++k) {
    const uint32_t v = P.cnt[k];
    tot += v;
    nz += v ? 1u : 0u;
  }
  uint32_t all_tot, all_nz;
  uint32_t o = block_scan_excl_u32(tot, wsum, &all_tot);
  uint32_t u = block_scan_excl_u32(nz, wsum2, &all_nz);
  for (int k = k0; k < k1; ++k) {
    const uint32_t v = P.cnt[k];
    P.off[k] = o;
    P.cur[k] = 0u;
    o += v;
    if (v) P.ulist[u++] = k;
  }
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

__device__ __forceinline__ uint32_t ld_pair(const uint16_t* p, int k, int d) {
  return k < d ? __ldg(reinterpret_cast<const uint32_t*>(p + k)) : 0u;  // k even, d even: pairs never straddle d
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
#pragma unroll 4
      for (int k0 = 0; k0 < d; k0 += 16) {
        const int ka = k0 + 2 * t, kb = k0 + 8 + 2 * t;
        const uint32_t a[4] = {ld_pair(ea, ka, d), ld_pair(eb, ka, d), ld_pair(ea, kb, d), ld_pair(eb, kb, d)};
#pragma unroll
        for (int ch = 0; ch < kChunks; ++ch) {
          if (ch < nch) mma_16816(acc[ch], a, ld_pair(hrow[ch], ka, d), ld_pair(hrow[ch], kb, d));
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
