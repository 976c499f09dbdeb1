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
// keeps the work exact instead of padding it 4-8x. Token rows are read once,
// from the head's cluster-major copy (a cluster's 16 rows are one contiguous
// block); hidden rows come from L2; both are staged through a per-warp
// cp.async ring in shared memory.
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

constexpr int kChunks = 4;          // 8-row chunks of R_k per pass (32 hidden rows)
constexpr int kRing = 4;            // cp.async stages per warp
constexpr int kSlice = 32;          // K elements per stage: 64 bytes of every row
constexpr int kStageBytes = (16 + 8 * kChunks) * kSlice * 2;  // 16 token rows + 32 hidden rows: 3 KB
constexpr int kGroupWarps = 16;     // warps per CTA (one CTA per SM)
constexpr int kGroupSmem = kGroupWarps * kRing * kStageBytes;  // 192 KB

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// One warp per distinct cluster (dynamic). For each pass over up to 32 of the
// hidden rows that chose it, K is streamed in slices of 32 elements through a
// per-warp ring of kRing shared-memory stages filled with 16-byte cp.async
// copies (the cluster's 16 token rows, contiguous in the cluster-major copy,
// and the pass's hidden rows, zero-filled past the row list): every warp keeps
// several KB in flight without holding them in registers. Fragments are read
// back with 16-byte shared loads (conflict-free: 64-byte rows) in the permuted
// K order described below and fed to mma.sync m16n8k16.
__global__ void __launch_bounds__(kGroupWarps * 32, 1) group_kernel(const GroupParams P) {
  extern __shared__ __align__(128) uint8_t gsm[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;  // mma fragment coordinates
  const int d = P.d, b = P.b;
  const int nsl = (d + kSlice - 1) / kSlice;
  const uint32_t ring = static_cast<uint32_t>(__cvta_generic_to_shared(gsm)) +
                        static_cast<uint32_t>(warp * kRing * kStageBytes);
  const uint32_t nu = *P.union_count;
  for (;;) {
    uint32_t ui = 0;
    if (lane == 0) ui = atomicAdd(P.next, 1u);
    ui = __shfl_sync(0xFFFFFFFFu, ui, 0);
    if (ui >= nu) break;
    const int k = P.ulist[ui];
    const int r0 = static_cast<int>(P.off[k]), r1 = static_cast<int>(P.off[k + 1]);
    const uint16_t* ek = P.Ecm + static_cast<size_t>(k) * b * d;  // the cluster's 16 rows, contiguous
    const int tok_a = P.C2T.at(static_cast<size_t>(k) * b + g);
    const int tok_b = P.C2T.at(static_cast<size_t>(k) * b + g + 8);
    for (int rb = r0; rb < r1; rb += 8 * kChunks) {
      const int nrows = min(8 * kChunks, r1 - rb);
      const int nch = (nrows + 7) / 8;
      const int hl = P.rows_of[rb + min(lane, nrows - 1)];  // hidden row of pass row `lane`
      auto issue = [&](int sl) {
        const uint32_t st = ring + static_cast<uint32_t>((sl % kRing) * kStageBytes);
        const int e0 = sl * kSlice;
#pragma unroll
        for (int i = 0; i < 2; ++i) {  // token rows: 16 rows x 4 chunks
          const int c = lane + 32 * i, row = c >> 2, ch = c & 3;
          const bool ok = e0 + 8 * ch < d;
          cp_async16(st + static_cast<uint32_t>(row * 64 + ch * 16), ek + static_cast<size_t>(row) * d + (ok ? e0 + 8 * ch : 0), ok);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {  // hidden rows: 32 rows x 4 chunks
          const int c = lane + 32 * i, row = c >> 2, ch = c & 3;
          const int hr = __shfl_sync(0xFFFFFFFFu, hl, row);
          const bool ok = row < nrows && e0 + 8 * ch < d;
          cp_async16(st + static_cast<uint32_t>((16 + row) * 64 + ch * 16),
                     P.H + static_cast<size_t>(hr) * d + (ok ? e0 + 8 * ch : 0), ok);
        }
        cp_async_commit();
      };
#pragma unroll
      for (int sl = 0; sl < kRing - 1; ++sl) {
        if (sl < nsl) issue(sl);
        else cp_async_commit();  // empty group: keeps the group count uniform
      }
      float acc[kChunks][4];
#pragma unroll
      for (int ch = 0; ch < kChunks; ++ch) acc[ch][0] = acc[ch][1] = acc[ch][2] = acc[ch][3] = 0.f;
      for (int sl = 0; sl < nsl; ++sl) {
        cp_async_wait<kRing - 2>();
        __syncwarp();
        const uint32_t st = ring + static_cast<uint32_t>((sl % kRing) * kStageBytes);
        // The dot product over K is order-free, so the slice's 32 elements feed
        // two MMA K-steps in a lane-friendly order: lane t of a fragment row
        // takes the 8 contiguous elements 8t..8t+7 of the slice; the first
        // K-step uses 8t..8t+3 (as its columns 2t, 2t+1, 2t+8, 2t+9), the second
        // 8t+4..8t+7. A and B use the same order, so the sums are unchanged.
        const uint4 xa = lds128(st + static_cast<uint32_t>(g * 64 + t * 16));
        const uint4 xb = lds128(st + static_cast<uint32_t>((g + 8) * 64 + t * 16));
        const uint32_t a0[4] = {xa.x, xb.x, xa.y, xb.y};
        const uint32_t a1[4] = {xa.z, xb.z, xa.w, xb.w};
#pragma unroll
        for (int ch = 0; ch < kChunks; ++ch) {
          if (ch < nch) {
            const uint4 xh = lds128(st + static_cast<uint32_t>((16 + 8 * ch + g) * 64 + t * 16));
            mma_16816(acc[ch], a0, xh.x, xh.y);
            mma_16816(acc[ch], a1, xh.z, xh.w);
          }
        }
        __syncwarp();  // the stage is read before it is refilled
        if (sl + kRing - 1 < nsl) issue(sl + kRing - 1);
        else cp_async_commit();
      }
      cp_async_wait<0>();
      __syncwarp();
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

cudaError_t set_attrs_group() {
  return cudaFuncSetAttribute(group_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGroupSmem);
}

cudaError_t launch_group(const GroupParams& P, int num_sms, cudaStream_t st) {
  const long long n = static_cast<long long>(P.B) * P.p;
  const int gsz = static_cast<int>(std::min<long long>((n + 255) / 256, 4LL * num_sms));
  cudaError_t e = cudaMemsetAsync(P.cnt, 0, static_cast<size_t>(P.c) * 4, st);
  if (e != cudaSuccess) return e;
  csr_count_kernel<<<gsz, 256, 0, st>>>(P);
  csr_scan_kernel<<<1, kThreads, 0, st>>>(P);
  csr_fill_kernel<<<gsz, 256, 0, st>>>(P);
  group_kernel<<<num_sms, kGroupWarps * 32, kGroupSmem, st>>>(P);
  return cudaGetLastError();
}

}  // namespace fh
