// Offline balanced spherical k-means that produces a FlashHead head (C, C2T).
//
// FlashHead write-up (www.framerc.cn/news/2430929), section 2.1 (offline
// clustering: normalised embeddings, k-means++ seeding, a loop of cosine
// similarities -> balanced assignment -> normalised cluster means) with the
// balance rule of section 1.2.1 (every cluster holds exactly b = v/c tokens).
//
// Kernels:
//  - normalize_kernel: one warp per token row, fp32 norm, bf16 output.
//  - seed_dist_kernel / seed_pick_kernel: one k-means++ draw per pair of
//    launches; squared distances to the newest centre folded into a running
//    minimum, fp64 block sums, inverse CDF in token order by one CTA.
//  - the v x c similarity product runs on the tcgen05 GEMM (fh_gemm.cu), the
//    centres as the M operand in chunks of 256, the token rows streamed.
//  - the balanced assignment in rounds of proposals: propose_kernel (every
//    unassigned token picks its best cluster among those whose b-th held
//    pair it beats, from a per-token shortlist of its 16 best clusters kept
//    by the first round, else from its whole column), a CSR of the
//    proposals by cluster, accept_kernel (one
//    warp per cluster keeps the best b of its held tokens and proposers with
//    a 32-lane bitonic merge). Under one strict order of all (token,
//    cluster) pairs -- similarity desc, token asc, cluster asc -- the
//    balanced assignment without a blocking pair is unique and equals the
//    global greedy, and the rounds reach it.
//  - update_kernel: one CTA per cluster sums its b rows in fp32 and writes
//    the normalised mean as bf16.
#include <cuda_bf16.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstring>
#include <new>

#include "fh_cluster.h"
#include "fh_device.cuh"
#include "fh_internal.h"

namespace fh {
namespace {

constexpr int kCT = 256;          // threads of the builder's streaming kernels
constexpr int kPickThreads = 1024;
constexpr int kSeedBlocks = 1024;  // row blocks of the seeding sums (one per pick thread)
constexpr int kMaxB = 32;          // a cluster's held list lives in one warp
constexpr int kMaxDC = 8192;       // update_kernel keeps d / 256 chunks of 8 per thread
constexpr int kUpdChunks = kMaxDC / (kCT * 8);
constexpr int kShort = 16;         // per-token shortlist of its best clusters

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(a));
  const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(b));
  return lo | (hi << 16);
}

__device__ __forceinline__ void widen8(const uint4 w, float (&x)[8]) {
  x[0] = bf16lo(w.x); x[1] = bf16hi(w.x);
  x[2] = bf16lo(w.y); x[3] = bf16hi(w.y);
  x[4] = bf16lo(w.z); x[5] = bf16hi(w.z);
  x[6] = bf16lo(w.w); x[7] = bf16hi(w.w);
}

// ---------------------------------------------------------------------------
// step 1: row normalisation
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kCT) normalize_kernel(const uint16_t* __restrict__ E, uint16_t* __restrict__ En,
                                                        int v, int d) {
  const int lane = threadIdx.x & 31;
  const long long nw = static_cast<long long>(gridDim.x) * (kCT / 32);
  for (long long t = static_cast<long long>(blockIdx.x) * (kCT / 32) + (threadIdx.x >> 5); t < v; t += nw) {
    const uint16_t* row = E + t * d;
    float ss = 0.f;
    for (int i = lane * 8; i < d; i += 256) {
      float x[8];
      widen8(*reinterpret_cast<const uint4*>(row + i), x);
#pragma unroll
      for (int j = 0; j < 8; ++j) ss = fmaf(x[j], x[j], ss);
    }
    ss = warp_sum(ss);
    const float n = sqrtf(ss);
    uint16_t* out = En + t * d;
    for (int i = lane * 8; i < d; i += 256) {
      float x[8];
      widen8(*reinterpret_cast<const uint4*>(row + i), x);
      uint4 o;
      if (ss > 0.f) {
        o.x = pack_bf16x2(__fdiv_rn(x[0], n), __fdiv_rn(x[1], n));
        o.y = pack_bf16x2(__fdiv_rn(x[2], n), __fdiv_rn(x[3], n));
        o.z = pack_bf16x2(__fdiv_rn(x[4], n), __fdiv_rn(x[5], n));
        o.w = pack_bf16x2(__fdiv_rn(x[6], n), __fdiv_rn(x[7], n));
      } else {
        o = make_uint4(0u, 0u, 0u, 0u);
      }
      *reinterpret_cast<uint4*>(out + i) = o;
    }
  }
}

// ---------------------------------------------------------------------------
// step 2: k-means++ seeding
// ---------------------------------------------------------------------------
struct SeedParams {
  const uint16_t* En;
  const float* u;
  int32_t* seed_ids;
  float* d2;        // [v] squared distance to the nearest chosen centre
  double* part;     // [kSeedBlocks] sums of d2 over each block's rows
  uint8_t* taken;   // [v]
  int32_t* cur;     // the newest centre
  int* status;
  int v, d, rows_per_blk;
};

// d2[t] = min(d2[t], |En[t] - En[cur]|^2) (or the distance itself on the first
// draw); block g covers rows [g*R, (g+1)*R) and writes their fp64 sum.
__global__ void __launch_bounds__(kCT) seed_dist_kernel(SeedParams P, int first) {
  extern __shared__ float ys[];  // the newest centre, fp32 [d]
  __shared__ double wsum[kCT / 32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int y = *P.cur;
  for (int i = threadIdx.x; i < P.d; i += kCT) ys[i] = bf16f(P.En[static_cast<size_t>(y) * P.d + i]);
  __syncthreads();
  const int r0 = blockIdx.x * P.rows_per_blk;
  const int r1 = min(P.v, r0 + P.rows_per_blk);
  double acc = 0.0;
  for (int t = r0 + w; t < r1; t += kCT / 32) {
    const uint16_t* row = P.En + static_cast<size_t>(t) * P.d;
    float s = 0.f;
    for (int i = lane * 8; i < P.d; i += 256) {
      float x[8];
      widen8(*reinterpret_cast<const uint4*>(row + i), x);
      const float4 y0 = *reinterpret_cast<const float4*>(ys + i);
      const float4 y1 = *reinterpret_cast<const float4*>(ys + i + 4);
      const float y[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float e = x[j] - y[j];
        s = fmaf(e, e, s);
      }
    }
    s = warp_sum(s);
    const float nd = first ? s : fminf(P.d2[t], s);
    if (lane == 0) P.d2[t] = nd;
    acc += static_cast<double>(nd);
  }
  if (lane == 0) wsum[w] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int i = 0; i < kCT / 32; ++i) s += wsum[i];
    P.part[blockIdx.x] = s;
  }
}

// Draw j: the first token whose running weight exceeds u[j] * total (token
// order), or the lowest unchosen token when every weight is zero. Draw 0 is
// token floor(u[0] * v).
__global__ void __launch_bounds__(kPickThreads) seed_pick_kernel(SeedParams P, int j) {
  __shared__ double scr[kPickThreads / 32 + 1];
  __shared__ double incl_s[kPickThreads];
  __shared__ int gsel, pick, lowest;
  const int tid = threadIdx.x;
  if (j == 0) {
    if (tid == 0) {
      const double f = floor(static_cast<double>(P.u[0]) * P.v);
      const int t = static_cast<int>(fmin(fmax(f, 0.0), static_cast<double>(P.v - 1)));
      P.seed_ids[0] = t;
      P.taken[t] = 1;
      *P.cur = t;
    }
    return;
  }
  if (tid == 0) {
    gsel = INT_MAX;
    pick = -1;
    lowest = INT_MAX;
  }
  const int nblk = (P.v + P.rows_per_blk - 1) / P.rows_per_blk;  // <= kPickThreads
  const double mine = tid < nblk ? P.part[tid] : 0.0;
  double total;
  const double incl = block_exclusive_scan<kPickThreads, double>(mine, scr, &total) + mine;
  incl_s[tid] = incl;
  __syncthreads();  // also orders the initialisation above
  const double all = incl_s[nblk - 1];
  if (all > 0.0) {
    const double target = static_cast<double>(P.u[j]) * all;
    // the first row block whose inclusive sum exceeds the target
    if (tid < nblk && incl > target) atomicMin(&gsel, tid);
    __syncthreads();
    const int g = gsel;
    if (g != INT_MAX && tid == 0) {
      const int r0 = g * P.rows_per_blk;
      const int r1 = min(P.v, r0 + P.rows_per_blk);
      double run = g == 0 ? 0.0 : incl_s[g - 1];
      int t = -1, last = -1;
      for (int r = r0; r < r1; ++r) {
        const float w = P.d2[r];
        if (w > 0.f) last = r;
        run += static_cast<double>(w);
        if (run > target && w > 0.f) { t = r; break; }
      }
      pick = t >= 0 ? t : last;  // rounding between the two sums: the block's last weighted row
    }
    __syncthreads();
    const bool need = pick < 0;  // no crossing (target at the very top): the last weighted token
    __syncthreads();
    if (need) {
      int best = -1;
      for (int r = tid; r < P.v; r += kPickThreads)
        if (P.d2[r] > 0.f) best = r;
      atomicMax(&pick, best);
    }
  } else {
    for (int r = tid; r < P.v; r += kPickThreads)
      if (!P.taken[r]) { atomicMin(&lowest, r); break; }
    __syncthreads();
    if (tid == 0) pick = lowest == INT_MAX ? -1 : lowest;
  }
  __syncthreads();
  if (tid == 0) {
    const int t = pick;
    if (t < 0 || t >= P.v) {
      record_error(P.status, FH_ERR_OUT_OF_RANGE);
      return;
    }
    P.seed_ids[j] = t;
    P.taken[t] = 1;
    *P.cur = t;
  }
}

// ---------------------------------------------------------------------------
// centres from token ids: C[k] = En[ids[k]]
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kCT) gather_rows_kernel(const uint16_t* __restrict__ En, const int32_t* __restrict__ ids,
                                                          uint16_t* __restrict__ C, int v, int d, int c, int* status) {
  const int lane = threadIdx.x & 31;
  const int nw = gridDim.x * (kCT / 32);
  for (int k = blockIdx.x * (kCT / 32) + (threadIdx.x >> 5); k < c; k += nw) {
    const int t = ids[k];
    if (t < 0 || t >= v) {
      if (lane == 0) record_error(status, FH_ERR_OUT_OF_RANGE);
      continue;
    }
    for (int i = lane * 8; i < d; i += 256)
      *reinterpret_cast<uint4*>(C + static_cast<size_t>(k) * d + i) =
          *reinterpret_cast<const uint4*>(En + static_cast<size_t>(t) * d + i);
  }
}

// ---------------------------------------------------------------------------
// step 3b: balanced assignment by rounds of proposals
// ---------------------------------------------------------------------------
struct AssignParams {
  const float* S;       // [c, v]
  float* held_s;        // [c, 32] held pairs of every cluster, best first
  int32_t* held_t;
  int32_t* held_n;      // [c]
  int2* thr;            // [c] (similarity bits, token) of the b-th held pair; (-inf, INT_MAX) while not full
  int32_t* tok;         // [v] cluster of every token, -1 while unassigned
  int32_t* prop_k;      // [v] this round's proposal of every unassigned token
  float* prop_s;
  uint32_t* cnt;        // [c] proposals per cluster
  uint32_t* off;        // [c + 1]
  uint32_t* cur;        // [c]
  int32_t* list;        // [v] proposers grouped by cluster
  int32_t* unassigned;
  float* sl_s;          // [kShort, v] every token's best clusters (similarity desc, cluster asc)
  int32_t* sl_k;        //   INT_MAX past the end when c < kShort
  int32_t* sl_pos;      // [v] first shortlist entry not yet ruled out
  int* status;
  int v, c, b;
};

// (s, t) ranks above (s2, t2): similarity descending, then token ascending.
__device__ __forceinline__ bool better(float s, int t, float s2, int t2) {
  return s > s2 || (s == s2 && t < t2);
}

__global__ void __launch_bounds__(kCT) assign_init_kernel(AssignParams P) {
  const int i = blockIdx.x * kCT + threadIdx.x;
  if (i < P.c) {
    P.held_n[i] = 0;
    P.thr[i] = make_int2(__float_as_int(-INFINITY), INT_MAX);
  }
  if (i < P.v) P.tok[i] = -1;
  if (i == 0) *P.unassigned = P.v;
}

// First round (every cluster has room): every token proposes to its best
// cluster and keeps its kShort best (similarity desc, cluster asc) as a
// shortlist, so that later rounds rarely read its whole column again.
__global__ void __launch_bounds__(kCT) propose_first_kernel(AssignParams P) {
  const int lane = threadIdx.x & 31;
  const int nw = gridDim.x * (kCT / 32);
  const int ngroups = (P.v + 31) / 32;
  for (int g = blockIdx.x * (kCT / 32) + (threadIdx.x >> 5); g < ngroups; g += nw) {
    const int t = g * 32 + lane;
    const bool valid = t < P.v;
    const int tc = valid ? t : P.v - 1;  // keep the loads in bounds
    float ls[kShort];
    int lk[kShort];
#pragma unroll
    for (int i = 0; i < kShort; ++i) {
      ls[i] = -INFINITY;
      lk[i] = INT_MAX;
    }
    for (int k = 0; k < P.c; ++k) {
      const float s = __ldg(P.S + static_cast<size_t>(k) * P.v + tc);
      if (s > ls[kShort - 1]) {  // k ascending: an equal similarity stays below the earlier cluster
#pragma unroll
        for (int i = kShort - 1; i > 0; --i) {
          if (s > ls[i - 1]) {
            ls[i] = ls[i - 1];
            lk[i] = lk[i - 1];
          } else if (s > ls[i]) {
            ls[i] = s;
            lk[i] = k;
          }
        }
        if (s > ls[0]) {
          ls[0] = s;
          lk[0] = k;
        }
      }
    }
    if (valid) {
#pragma unroll
      for (int i = 0; i < kShort; ++i) {
        P.sl_s[static_cast<size_t>(i) * P.v + t] = ls[i];
        P.sl_k[static_cast<size_t>(i) * P.v + t] = lk[i];
      }
      P.sl_pos[t] = 0;
      if (lk[0] == INT_MAX) {
        record_error(P.status, FH_ERR_OUT_OF_RANGE);  // only non-finite similarities get here
        P.prop_k[t] = -1;
      } else {
        P.prop_k[t] = lk[0];
        P.prop_s[t] = ls[0];
        atomicAdd(P.cnt + lk[0], 1u);
      }
    }
  }
}

// Every unassigned token proposes to its best cluster (similarity desc,
// cluster asc) among those that would not reject it at the round's start:
// the first shortlist entry still eligible (clusters only ever raise their
// bar, so an entry ruled out once stays out, and every cluster outside the
// shortlist ranks below all of it), else the best of its whole column.
__global__ void __launch_bounds__(kCT) propose_kernel(AssignParams P) {
  const int lane = threadIdx.x & 31;
  const int nw = gridDim.x * (kCT / 32);
  const int ngroups = (P.v + 31) / 32;
  for (int g = blockIdx.x * (kCT / 32) + (threadIdx.x >> 5); g < ngroups; g += nw) {
    const int t = g * 32 + lane;
    const bool valid = t < P.v;
    const bool active = valid && P.tok[t] < 0;
    if (!__any_sync(0xFFFFFFFFu, active)) continue;
    const int tc = valid ? t : P.v - 1;  // keep the loads in bounds
    float bs = -INFINITY;
    int bk = -1;
    if (active) {
      int j = P.sl_pos[t];
      for (; j < kShort; ++j) {
        const int k = P.sl_k[static_cast<size_t>(j) * P.v + t];
        if (k == INT_MAX) {
          j = kShort;
          break;
        }
        const float s = P.sl_s[static_cast<size_t>(j) * P.v + t];
        const int2 th = __ldg(P.thr + k);
        if (better(s, t, __int_as_float(th.x), th.y)) {
          bs = s;
          bk = k;
          break;
        }
      }
      P.sl_pos[t] = j;
    }
    const bool scan = active && bk < 0;  // shortlist exhausted: the whole column
    if (__any_sync(0xFFFFFFFFu, scan)) {
      int k = 0;
      for (; k + 4 <= P.c; k += 4) {
        float s[4];
        int2 th[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          s[q] = __ldg(P.S + static_cast<size_t>(k + q) * P.v + tc);
          th[q] = __ldg(P.thr + k + q);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const bool elig = better(s[q], t, __int_as_float(th[q].x), th[q].y);
          if (scan && elig && (bk < 0 || s[q] > bs)) { bs = s[q]; bk = k + q; }
        }
      }
      for (; k < P.c; ++k) {
        const float s = __ldg(P.S + static_cast<size_t>(k) * P.v + tc);
        const int2 th = __ldg(P.thr + k);
        if (scan && better(s, t, __int_as_float(th.x), th.y) && (bk < 0 || s > bs)) { bs = s; bk = k; }
      }
    }
    if (active) {
      if (bk < 0) {
        record_error(P.status, FH_ERR_OUT_OF_RANGE);  // only non-finite similarities get here
        P.prop_k[t] = -1;
      } else {
        P.prop_k[t] = bk;
        P.prop_s[t] = bs;
        atomicAdd(P.cnt + bk, 1u);
      }
    }
  }
}

// off = exclusive scan of cnt (one CTA); cur = 0.
__global__ void __launch_bounds__(kPickThreads) assign_scan_kernel(AssignParams P) {
  __shared__ uint32_t scr[kPickThreads / 32 + 1];
  const int per = (P.c + kPickThreads - 1) / kPickThreads;
  const int k0 = threadIdx.x * per;
  uint32_t s = 0;
  for (int k = k0; k < min(P.c, k0 + per); ++k) s += P.cnt[k];
  uint32_t total;
  uint32_t run = block_exclusive_scan<kPickThreads, uint32_t>(s, scr, &total);
  for (int k = k0; k < min(P.c, k0 + per); ++k) {
    P.off[k] = run;
    run += P.cnt[k];
    P.cur[k] = 0;
  }
  if (threadIdx.x == 0) P.off[P.c] = total;
}

__global__ void __launch_bounds__(kCT) assign_fill_kernel(AssignParams P) {
  for (int t = blockIdx.x * kCT + threadIdx.x; t < P.v; t += gridDim.x * kCT) {
    if (P.tok[t] >= 0) continue;
    const int k = P.prop_k[t];
    if (k < 0) continue;
    const uint32_t pos = P.off[k] + atomicAdd(P.cur + k, 1u);
    P.list[pos] = t;
  }
}

// Bitonic sort of one (s, t) pair per lane: lane 0 ends with the best.
__device__ __forceinline__ void warp_sort_desc(float& s, int& t) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const float os = __shfl_xor_sync(0xFFFFFFFFu, s, j);
      const int ot = __shfl_xor_sync(0xFFFFFFFFu, t, j);
      const bool keep_better = ((lane & j) == 0) == ((lane & k) == 0);
      const bool take = keep_better ? better(os, ot, s, t) : better(s, t, os, ot);
      if (take) { s = os; t = ot; }
    }
  }
}

// Merge a sorted batch into the sorted running list: the best 32 of both, sorted.
__device__ __forceinline__ void warp_merge_desc(float& s, int& t, float bs, int bt) {
  const int lane = threadIdx.x & 31;
  const float rs = __shfl_sync(0xFFFFFFFFu, bs, 31 - lane);
  const int rt = __shfl_sync(0xFFFFFFFFu, bt, 31 - lane);
  if (better(rs, rt, s, t)) { s = rs; t = rt; }
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) {
    const float os = __shfl_xor_sync(0xFFFFFFFFu, s, j);
    const int ot = __shfl_xor_sync(0xFFFFFFFFu, t, j);
    const bool lower = (lane & j) == 0;
    const bool take = lower ? better(os, ot, s, t) : better(s, t, os, ot);
    if (take) { s = os; t = ot; }
  }
}

// Every cluster with proposals keeps the best b of its held pairs and its proposers.
__global__ void __launch_bounds__(kCT) accept_kernel(AssignParams P) {
  const int lane = threadIdx.x & 31;
  const int nw = gridDim.x * (kCT / 32);
  for (int k = blockIdx.x * (kCT / 32) + (threadIdx.x >> 5); k < P.c; k += nw) {
    const uint32_t o0 = P.off[k], o1 = P.off[k + 1];
    if (o0 == o1) continue;
    const int n_old = P.held_n[k];
    float s = -INFINITY;
    int t = INT_MAX;
    if (lane < n_old) {
      s = P.held_s[k * kMaxB + lane];
      t = P.held_t[k * kMaxB + lane];
    }
    const int old_t = lane < n_old ? t : -1;
    for (uint32_t base = o0; base < o1; base += 32) {
      float ps = -INFINITY;
      int pt = INT_MAX;
      if (base + lane < o1) {
        pt = P.list[base + lane];
        ps = P.prop_s[pt];
      }
      warp_sort_desc(ps, pt);
      warp_merge_desc(s, t, ps, pt);
    }
    const bool kept = lane < P.b && t != INT_MAX;
    const int n_new = __popc(__ballot_sync(0xFFFFFFFFu, kept));
    if (lane < P.b) {
      P.held_s[k * kMaxB + lane] = s;
      P.held_t[k * kMaxB + lane] = t;
    }
    // old members that lost their place become unassigned
    bool stays = false;
    for (int j = 0; j < n_new; ++j) stays |= __shfl_sync(0xFFFFFFFFu, t, j) == old_t;
    const bool kicked = old_t >= 0 && !stays;
    if (kicked) P.tok[old_t] = -1;
    if (kept) P.tok[t] = k;
    const int n_kicked = __popc(__ballot_sync(0xFFFFFFFFu, kicked));
    const float ws = __shfl_sync(0xFFFFFFFFu, s, P.b - 1);
    const int wt = __shfl_sync(0xFFFFFFFFu, t, P.b - 1);
    if (lane == 0) {
      P.held_n[k] = n_new;
      P.thr[k] = n_new == P.b ? make_int2(__float_as_int(ws), wt) : make_int2(__float_as_int(-INFINITY), INT_MAX);
      // accepted proposers = n_new - (n_old - n_kicked)
      const int accepted = n_new - (n_old - n_kicked);
      atomicSub(P.unassigned, accepted - n_kicked);
    }
  }
}

// Final map: every cluster's tokens in ascending id, and the token -> cluster map.
__global__ void __launch_bounds__(kCT) assign_final_kernel(AssignParams P, int32_t* assign, int32_t* C2T) {
  const int lane = threadIdx.x & 31;
  const int nw = gridDim.x * (kCT / 32);
  for (int k = blockIdx.x * (kCT / 32) + (threadIdx.x >> 5); k < P.c; k += nw) {
    if (P.held_n[k] != P.b) {
      if (lane == 0) record_error(P.status, FH_ERR_OUT_OF_RANGE);
      continue;
    }
    // ascending token id: sort (-t) descending with equal similarity keys
    float s = 0.f;
    int t = lane < P.b ? P.held_t[k * kMaxB + lane] : INT_MAX;
    warp_sort_desc(s, t);
    if (lane < P.b) {
      C2T[static_cast<size_t>(k) * P.b + lane] = t;
      assign[t] = k;
    }
  }
}

// Number of positions where two maps differ.
__global__ void __launch_bounds__(kCT) count_diff_kernel(const int32_t* a, const int32_t* b, long long n, uint32_t* out) {
  uint32_t m = 0;
  for (long long i = blockIdx.x * static_cast<long long>(kCT) + threadIdx.x; i < n; i += gridDim.x * static_cast<long long>(kCT))
    m += a[i] != b[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m += __shfl_xor_sync(0xFFFFFFFFu, m, o);
  if ((threadIdx.x & 31) == 0 && m) atomicAdd(out, m);
}

// ---------------------------------------------------------------------------
// step 3c: centres = normalised means of their tokens
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kCT) update_kernel(const uint16_t* __restrict__ En, const int32_t* __restrict__ C2T,
                                                     uint16_t* __restrict__ C, int v, int d, int b, int* status) {
  __shared__ int toks[kMaxB];
  __shared__ float wss[kCT / 32];
  __shared__ int bad;
  const int k = blockIdx.x;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  if (threadIdx.x < b) {
    const int t = C2T[static_cast<size_t>(k) * b + threadIdx.x];
    toks[threadIdx.x] = t;
    if (t < 0 || t >= v) bad = 1;
  }
  __syncthreads();
  if (bad) {
    if (threadIdx.x == 0) record_error(status, FH_ERR_OUT_OF_RANGE);
    return;
  }
  float acc[kUpdChunks][8];
  float ss = 0.f;
#pragma unroll
  for (int q = 0; q < kUpdChunks; ++q) {
    const int i = (q * kCT + threadIdx.x) * 8;
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[q][j] = 0.f;
    if (i < d) {
      for (int r = 0; r < b; ++r) {
        float x[8];
        widen8(*reinterpret_cast<const uint4*>(En + static_cast<size_t>(toks[r]) * d + i), x);
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[q][j] += x[j];
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) ss = fmaf(acc[q][j], acc[q][j], ss);
    }
  }
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) wss[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < kCT / 32; ++w) tot += wss[w];
  if (!(tot > 0.f)) return;  // zero mean: the centre stays
  const float n = sqrtf(tot);
#pragma unroll
  for (int q = 0; q < kUpdChunks; ++q) {
    const int i = (q * kCT + threadIdx.x) * 8;
    if (i < d) {
      uint4 o;
      o.x = pack_bf16x2(__fdiv_rn(acc[q][0], n), __fdiv_rn(acc[q][1], n));
      o.y = pack_bf16x2(__fdiv_rn(acc[q][2], n), __fdiv_rn(acc[q][3], n));
      o.z = pack_bf16x2(__fdiv_rn(acc[q][4], n), __fdiv_rn(acc[q][5], n));
      o.w = pack_bf16x2(__fdiv_rn(acc[q][6], n), __fdiv_rn(acc[q][7], n));
      *reinterpret_cast<uint4*>(C + static_cast<size_t>(k) * d + i) = o;
    }
  }
}

inline size_t up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

fh_status fail(cudaError_t e) {
  (void)cudaGetLastError();
  return e == cudaErrorMemoryAllocation ? FH_ERR_OOM : FH_ERR_CUDA;
}

}  // namespace
}  // namespace fh

using namespace fh;

struct fh_cluster {
  int v = 0, d = 0, c = 0, b = 0;
  int device = 0, num_sms = 0;
  uint8_t* ws = nullptr;
  size_t ws_bytes = 0;
  uint16_t* En = nullptr;   // [v, d] normalised rows (fh_cluster_build)
  float* S = nullptr;       // [c, v]
  uint16_t* C = nullptr;    // [c, d] working centres
  int32_t* c2t[2] = {nullptr, nullptr};
  int32_t* assign = nullptr;
  int32_t* ids = nullptr;   // [c] seeds
  AssignParams A{};
  SeedParams Sd{};
  uint32_t* diff = nullptr;
  int* status = nullptr;
};

namespace {

int grid_for(const fh_cluster* cl, long long items, int per_cta) {
  const long long g = (items + per_cta - 1) / per_cta;
  return static_cast<int>(std::max<long long>(1, std::min<long long>(g, 8LL * cl->num_sms)));
}

fh_status read_word(const void* dev, void* host, size_t n, cudaStream_t st) {
  cudaError_t e = cudaMemcpyAsync(host, dev, n, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  return e == cudaSuccess ? FH_OK : fail(e);
}

fh_status run_assign(fh_cluster* cl, const float* S, int32_t* assign, int32_t* C2T, int32_t* rounds, cudaStream_t st) {
  AssignParams P = cl->A;
  P.S = S;
  const int gv = grid_for(cl, cl->v, kCT);
  const int gw = grid_for(cl, (cl->v + 31) / 32, kCT / 32);
  const int gc = grid_for(cl, cl->c, kCT / 32);
  assign_init_kernel<<<static_cast<int>((std::max(cl->v, cl->c) + kCT - 1) / kCT), kCT, 0, st>>>(P);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(e);
  // Every round ends with all tokens placed or rules out at least one (token, cluster)
  // pair for good (a rejected or displaced token never beats that cluster again),
  // so v*c rounds bound the loop.
  const long long max_rounds = static_cast<long long>(cl->v) * cl->c + 2;
  long long r = 0;
  for (;;) {
    if (++r > max_rounds) return FH_ERR_TIMEOUT;
    e = cudaMemsetAsync(P.cnt, 0, sizeof(uint32_t) * cl->c, st);
    if (e != cudaSuccess) return fail(e);
    if (r == 1) propose_first_kernel<<<gw, kCT, 0, st>>>(P);
    else propose_kernel<<<gw, kCT, 0, st>>>(P);
    assign_scan_kernel<<<1, kPickThreads, 0, st>>>(P);
    assign_fill_kernel<<<gv, kCT, 0, st>>>(P);
    accept_kernel<<<gc, kCT, 0, st>>>(P);
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail(e);
    int32_t left = 0;
    int dev_status = 0;
    fh_status s = read_word(P.unassigned, &left, sizeof(left), st);
    if (s == FH_OK) s = read_word(P.status, &dev_status, sizeof(dev_status), st);
    if (s != FH_OK) return s;
    if (dev_status) return static_cast<fh_status>(dev_status);
    if (left <= 0) break;
  }
  assign_final_kernel<<<gc, kCT, 0, st>>>(P, assign, C2T);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail(e);
  if (rounds) *rounds = static_cast<int32_t>(std::min<long long>(r, INT_MAX));
  return FH_OK;
}

fh_status run_similarities(fh_cluster* cl, const void* En, const void* C, float* S, cudaStream_t st) {
  for (int k0 = 0; k0 < cl->c; k0 += 256) {
    GemmParams P{};
    P.rows = cl->v;
    P.d = cl->d;
    P.nb = std::min(256, cl->c - k0);
    P.epi = 0;
    P.mode = 0;
    P.T = 1.f;
    P.out = S + static_cast<size_t>(k0) * cl->v;
    P.ldo = cl->v;
    P.status = cl->status;
    cudaError_t e = launch_gemm(P, En, static_cast<const uint16_t*>(C) + static_cast<size_t>(k0) * cl->d,
                                cl->num_sms, st);
    if (e != cudaSuccess) return fail(e);
  }
  return FH_OK;
}

fh_status run_seed(fh_cluster* cl, const void* En, const float* u, int32_t* seed_ids, cudaStream_t st) {
  SeedParams P = cl->Sd;
  P.En = static_cast<const uint16_t*>(En);
  P.u = u;
  P.seed_ids = seed_ids;
  cudaError_t e = cudaMemsetAsync(P.taken, 0, cl->v, st);
  if (e != cudaSuccess) return fail(e);
  const int nblk = (cl->v + P.rows_per_blk - 1) / P.rows_per_blk;
  const size_t smem = static_cast<size_t>(cl->d) * sizeof(float);
  seed_pick_kernel<<<1, kPickThreads, 0, st>>>(P, 0);
  for (int j = 1; j < cl->c; ++j) {
    seed_dist_kernel<<<nblk, kCT, smem, st>>>(P, j == 1);
    seed_pick_kernel<<<1, kPickThreads, 0, st>>>(P, j);
  }
  e = cudaGetLastError();
  return e == cudaSuccess ? FH_OK : fail(e);
}

fh_status check_rows(const fh_cluster* cl, const void* p) {
  return p && aligned(p, 16) ? FH_OK : FH_ERR_INVALID_ARG;
}

}  // namespace

extern "C" {

fh_status fh_cluster_create(int32_t v, int32_t d, int32_t c, fh_stream_t stream, fh_cluster** out) {
  if (!out) return FH_ERR_INVALID_ARG;
  *out = nullptr;
  if (v < 1 || c < 1 || d < 8 || v % c) return FH_ERR_INVALID_ARG;
  if (d % 8) return FH_ERR_INVALID_ARG;
  const int b = v / c;
  if (b > kMaxB || d > kMaxDC) return FH_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(e);
  cudaDeviceProp prop;
  e = cudaGetDeviceProperties(&prop, dev);
  if (e != cudaSuccess) return fail(e);
  if (prop.major != 10) return FH_ERR_UNSUPPORTED;
  e = set_attrs_gemm();  // the seeding kernel's centre (d fp32 <= 32 KB) fits the default limit
  if (e != cudaSuccess) return fail(e);

  fh_cluster* cl = new (std::nothrow) fh_cluster();
  if (!cl) return FH_ERR_OOM;
  cl->v = v; cl->d = d; cl->c = c; cl->b = b;
  cl->device = dev;
  cl->num_sms = prop.multiProcessorCount;

  const size_t V = v, D = d, Cn = c;
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t o = off; off = up(off + bytes, 256); return o; };
  const size_t o_words = take(64);
  const size_t o_en = take(V * D * 2);
  const size_t o_s = take(Cn * V * 4);
  const size_t o_c = take(Cn * D * 2);
  const size_t o_m0 = take(Cn * b * 4);
  const size_t o_m1 = take(Cn * b * 4);
  const size_t o_asg = take(V * 4);
  const size_t o_ids = take(Cn * 4);
  const size_t o_hs = take(Cn * kMaxB * 4);
  const size_t o_ht = take(Cn * kMaxB * 4);
  const size_t o_hn = take(Cn * 4);
  const size_t o_thr = take(Cn * 8);
  const size_t o_tok = take(V * 4);
  const size_t o_pk = take(V * 4);
  const size_t o_ps = take(V * 4);
  const size_t o_cnt = take(Cn * 4);
  const size_t o_off = take((Cn + 1) * 4);
  const size_t o_cur = take(Cn * 4);
  const size_t o_list = take(V * 4);
  const size_t o_d2 = take(V * 4);
  const size_t o_part = take(kSeedBlocks * 8);
  const size_t o_taken = take(V);
  const size_t o_sls = take(V * kShort * 4);
  const size_t o_slk = take(V * kShort * 4);
  const size_t o_slp = take(V * 4);
  cl->ws_bytes = off;
  e = cudaMalloc(&cl->ws, cl->ws_bytes);
  if (e != cudaSuccess) {
    delete cl;
    return fail(e);
  }
  uint8_t* w = cl->ws;
  int32_t* words = reinterpret_cast<int32_t*>(w + o_words);
  cl->status = words;
  cl->diff = reinterpret_cast<uint32_t*>(words + 1);
  cl->En = reinterpret_cast<uint16_t*>(w + o_en);
  cl->S = reinterpret_cast<float*>(w + o_s);
  cl->C = reinterpret_cast<uint16_t*>(w + o_c);
  cl->c2t[0] = reinterpret_cast<int32_t*>(w + o_m0);
  cl->c2t[1] = reinterpret_cast<int32_t*>(w + o_m1);
  cl->assign = reinterpret_cast<int32_t*>(w + o_asg);
  cl->ids = reinterpret_cast<int32_t*>(w + o_ids);
  AssignParams& A = cl->A;
  A.held_s = reinterpret_cast<float*>(w + o_hs);
  A.held_t = reinterpret_cast<int32_t*>(w + o_ht);
  A.held_n = reinterpret_cast<int32_t*>(w + o_hn);
  A.thr = reinterpret_cast<int2*>(w + o_thr);
  A.tok = reinterpret_cast<int32_t*>(w + o_tok);
  A.prop_k = reinterpret_cast<int32_t*>(w + o_pk);
  A.prop_s = reinterpret_cast<float*>(w + o_ps);
  A.cnt = reinterpret_cast<uint32_t*>(w + o_cnt);
  A.off = reinterpret_cast<uint32_t*>(w + o_off);
  A.cur = reinterpret_cast<uint32_t*>(w + o_cur);
  A.list = reinterpret_cast<int32_t*>(w + o_list);
  A.unassigned = words + 2;
  A.sl_s = reinterpret_cast<float*>(w + o_sls);
  A.sl_k = reinterpret_cast<int32_t*>(w + o_slk);
  A.sl_pos = reinterpret_cast<int32_t*>(w + o_slp);
  A.status = cl->status;
  A.v = v; A.c = c; A.b = b;
  SeedParams& Sd = cl->Sd;
  Sd.d2 = reinterpret_cast<float*>(w + o_d2);
  Sd.part = reinterpret_cast<double*>(w + o_part);
  Sd.taken = w + o_taken;
  Sd.cur = words + 3;
  Sd.status = cl->status;
  Sd.v = v; Sd.d = d;
  Sd.rows_per_blk = (v + kSeedBlocks - 1) / kSeedBlocks;
  e = cudaMemsetAsync(words, 0, 64, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) {
    cudaFree(cl->ws);
    delete cl;
    return fail(e);
  }
  *out = cl;
  return FH_OK;
}

void fh_cluster_destroy(fh_cluster* cl) {
  if (!cl) return;
  cudaDeviceSynchronize();
  cudaFree(cl->ws);
  delete cl;
}

fh_status fh_cluster_normalize(fh_cluster* cl, const void* E, void* En, fh_stream_t stream) {
  if (!cl || check_rows(cl, E) != FH_OK || check_rows(cl, En) != FH_OK || E == En) return FH_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  normalize_kernel<<<grid_for(cl, cl->v, kCT / 32), kCT, 0, st>>>(static_cast<const uint16_t*>(E),
                                                                 static_cast<uint16_t*>(En), cl->v, cl->d);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FH_OK : fail(e);
}

fh_status fh_cluster_seed(fh_cluster* cl, const void* En, const float* u, int32_t* seed_ids, fh_stream_t stream) {
  if (!cl || check_rows(cl, En) != FH_OK || !u || !seed_ids) return FH_ERR_INVALID_ARG;
  return run_seed(cl, En, u, seed_ids, reinterpret_cast<cudaStream_t>(stream));
}

fh_status fh_cluster_gather(fh_cluster* cl, const void* En, const int32_t* ids, void* C, fh_stream_t stream) {
  if (!cl || check_rows(cl, En) != FH_OK || check_rows(cl, C) != FH_OK || !ids) return FH_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  gather_rows_kernel<<<grid_for(cl, cl->c, kCT / 32), kCT, 0, st>>>(
      static_cast<const uint16_t*>(En), ids, static_cast<uint16_t*>(C), cl->v, cl->d, cl->c, cl->status);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FH_OK : fail(e);
}

fh_status fh_cluster_similarities(fh_cluster* cl, const void* En, const void* C, float* S, fh_stream_t stream) {
  if (!cl || check_rows(cl, En) != FH_OK || check_rows(cl, C) != FH_OK || !S || !aligned(S, 16))
    return FH_ERR_INVALID_ARG;
  return run_similarities(cl, En, C, S, reinterpret_cast<cudaStream_t>(stream));
}

fh_status fh_cluster_assign(fh_cluster* cl, const float* S, int32_t* assign, int32_t* C2T, int32_t* rounds,
                            fh_stream_t stream) {
  if (!cl || !S || !assign || !C2T) return FH_ERR_INVALID_ARG;
  return run_assign(cl, S, assign, C2T, rounds, reinterpret_cast<cudaStream_t>(stream));
}

fh_status fh_cluster_update(fh_cluster* cl, const void* En, const int32_t* C2T, void* C, fh_stream_t stream) {
  if (!cl || check_rows(cl, En) != FH_OK || check_rows(cl, C) != FH_OK || !C2T) return FH_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  update_kernel<<<cl->c, kCT, 0, st>>>(static_cast<const uint16_t*>(En), C2T, static_cast<uint16_t*>(C), cl->v,
                                       cl->d, cl->b, cl->status);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FH_OK : fail(e);
}

fh_status fh_cluster_build(fh_cluster* cl, const void* E, const int32_t* init_ids, const float* u_init,
                           int32_t max_iter, void* C_out, int32_t* C2T_out, int32_t* iterations,
                           fh_stream_t stream) {
  if (!cl || check_rows(cl, E) != FH_OK || check_rows(cl, C_out) != FH_OK || !C2T_out) return FH_ERR_INVALID_ARG;
  if (!init_ids && !u_init) return FH_ERR_INVALID_ARG;
  if (max_iter < 1) return FH_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  fh_status s = fh_cluster_normalize(cl, E, cl->En, stream);
  if (s != FH_OK) return s;
  const int32_t* ids = init_ids;
  if (!ids) {
    s = run_seed(cl, cl->En, u_init, cl->ids, st);
    if (s != FH_OK) return s;
    ids = cl->ids;
  }
  s = fh_cluster_gather(cl, cl->En, ids, cl->C, stream);
  if (s != FH_OK) return s;
  int prev = -1, cur = 0, it = 0, last = 0;
  const long long nmap = static_cast<long long>(cl->c) * cl->b;
  for (it = 1; it <= max_iter; ++it) {
    s = run_similarities(cl, cl->En, cl->C, cl->S, st);
    if (s == FH_OK) s = run_assign(cl, cl->S, cl->assign, cl->c2t[cur], nullptr, st);
    if (s != FH_OK) return s;
    last = cur;
    if (prev >= 0) {
      cudaError_t e = cudaMemsetAsync(cl->diff, 0, sizeof(uint32_t), st);
      if (e != cudaSuccess) return fail(e);
      count_diff_kernel<<<grid_for(cl, nmap, kCT), kCT, 0, st>>>(cl->c2t[cur], cl->c2t[prev], nmap, cl->diff);
      uint32_t nd = 0;
      s = read_word(cl->diff, &nd, sizeof(nd), st);
      if (s != FH_OK) return s;
      if (nd == 0) break;
    }
    s = fh_cluster_update(cl, cl->En, cl->c2t[cur], cl->C, stream);
    if (s != FH_OK) return s;
    prev = cur;
    cur ^= 1;
  }
  if (it > max_iter) it = max_iter;
  cudaError_t e = cudaMemcpyAsync(C_out, cl->C, static_cast<size_t>(cl->c) * cl->d * 2, cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(C2T_out, cl->c2t[last], static_cast<size_t>(nmap) * 4, cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return fail(e);
  if (iterations) *iterations = it;
  return fh_cluster_get_device_status(cl, stream);
}

fh_status fh_cluster_get_device_status(fh_cluster* cl, fh_stream_t stream) {
  if (!cl) return FH_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int s = 0;
  fh_status r = read_word(cl->status, &s, sizeof(s), st);
  if (r != FH_OK) return r;
  if (s) {
    cudaError_t e = cudaMemsetAsync(cl->status, 0, sizeof(int), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return fail(e);
  }
  return static_cast<fh_status>(s);
}

}  // extern "C"
