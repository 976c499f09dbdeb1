// Fused FlashHead decode for one hidden state (B = 1): one persistent
// cooperative launch, two 512-thread CTAs per SM, every row streamed HBM ->
// registers with non-allocating 16-byte loads and dotted with h staged once
// per CTA in shared memory (fp32).
//
// The pages' pipeline (FlashHead write-up, section 2.2.2: h -> centroid_scores
// -> top_p_clusters -> token_scores) runs as phases of one kernel:
//
//  1. centroid scores (section 1.2.2; INT4 centroids per section 1.2.4):
//     cluster k belongs to CTA k mod G (warp (k / G) mod 16), so every CTA
//     owns c/G clusters; the owning warp streams the centroid row and
//     computes the key -- the score, or when sampling the Gumbel key
//     s/T - ln(-ln u) (section 1.2.3). The key stays in a lane register of the
//     owning warp and is counted into a device-wide histogram of its top 12
//     bits (fire-and-forget atomics).
//  2. device-wide barrier; each CTA scans the histogram once and finds the
//     bin t1 holding the p-th largest key. Keys above t1 are selected; keys
//     inside t1 form the boundary. Owners publish the b token ids of each
//     selected cluster (its C2T row, section 1.2.1: slot k*b + j holds token
//     C2T[k][j]) into a device-wide row queue, and the boundary keys into a
//     small list.
//  3. candidate rows are spread over every warp of the grid the same way
//     (row r to CTA r mod G): a warp polls its queue slot for the token id, streams the token row and
//     keeps a packed (logit, token) maximum (section 1.2.4, stage 2).
//  4. when the boundary bin is split (some but not all of its keys needed),
//     a warp that owns boundary keys ranks them exactly (key desc, id asc)
//     against the list as soon as a second barrier says the list is
//     complete -- checked inside its polling loop, so no wait can deadlock --
//     and queues the chosen clusters, whose rows the consumers pick up as in
//     step 3.
//  5. CTA maxima meet in one 64-bit atomicMax; the last CTA to finish (exit
//     ticket) writes the token: the argmax, or, when sampling, the inverse-CDF
//     draw over softmax(z/T) in canonical order (cluster asc, slot asc),
//     walking a bitmap of the selected clusters.
//
// No CTA ever reads all c keys, and HBM traffic is the algorithmic minimum:
// each centroid row once, each selected token row once, plus C2T rows and h.
// Device-wide counters are spread over 8 cache lines so that arrivals do not
// serialise on one address.
#include <climits>

#include "fh_device.cuh"

namespace fh {
namespace {

constexpr int kBarLanes = 8;       // counters per device-wide barrier
constexpr int kBarStride = 32;     // words between counters (one 128-byte line each)

struct B1Misc {
  unsigned long long hbar;
  unsigned long long wbar[kWarps];
  unsigned long long wbest[kWarps];
  float scan[kWarps + 1];
  uint32_t uscan[kWarps + 1];
  int claim, lastpos, ok, last;
  uint32_t t1, need, split, fallback, n_sure;
  uint32_t cta_sure, qbase;
};

__device__ __forceinline__ void bar_arrive(uint32_t* bar) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(bar + (blockIdx.x % kBarLanes) * kBarStride, 1u);
  }
}

// Sum of the counters: relaxed loads, all in flight together (the waiter
// fences once after seeing the target).
__device__ __forceinline__ uint32_t bar_count(const uint32_t* bar) {
  uint32_t v[kBarLanes], s = 0;
#pragma unroll
  for (int i = 0; i < kBarLanes; ++i) v[i] = ld_relaxed_u32(bar + i * kBarStride);
#pragma unroll
  for (int i = 0; i < kBarLanes; ++i) s += v[i];
  return s;
}

// All CTAs wait until `target` arrivals; false if `budget` cycles pass first.
__device__ bool bar_wait(const uint32_t* bar, uint32_t target, long long budget, int* flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    if (bar_count(bar) < target) {
      const long long t0 = clock64();
      while (bar_count(bar) < target) {
        if (clock64() - t0 > budget) {
          ok = 0;
          break;
        }
      }
    }
    __threadfence();
    *flag = ok;
  }
  __syncthreads();
  return *flag != 0;
}

// Queue the b token ids of cluster k at row-queue position pos (one warp).
__device__ __forceinline__ void queue_cluster(const B1Params& P, int32_t* rq, uint32_t* bitmap, uint32_t pos,
                                              int k) {
  const int lane = threadIdx.x & 31;
  if (lane == 0) atomicOr(bitmap + (k >> 5), 1u << (k & 31));
  if (pos >= static_cast<uint32_t>(P.p)) return;  // only an inconsistent histogram could overfill the queue
  for (int j = lane; j < P.b; j += 32)
    rq[static_cast<size_t>(pos) * P.b + j] = __ldg(P.C2T + static_cast<size_t>(k) * P.b + j);
}

// Exact rank of each of this warp's boundary keys (lanes set in `mine`)
// against the published boundary list; the chosen clusters are queued.
__device__ void rank_boundary(const B1Params& P, int32_t* rq, uint32_t* bitmap, uint32_t* qcount,
                              const unsigned long long* bnd_list, const uint32_t* bnd_count, uint32_t mine,
                              uint32_t own_key, int cw, int cstride, uint32_t need) {
  const int lane = threadIdx.x & 31;
  const uint32_t nb = min(__ldcg(bnd_count), static_cast<uint32_t>(kBoundaryMax));
  while (mine) {
    const int j = __ffs(mine) - 1;
    mine &= mine - 1;
    const uint32_t kq = __shfl_sync(0xFFFFFFFFu, own_key, j);
    const int idq = cw + j * cstride;
    uint32_t r = 0;
    for (uint32_t e0 = 0; e0 < nb; e0 += 128) {
      unsigned long long v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t e = e0 + lane + 32 * u;
        v[u] = e < nb ? __ldcg(bnd_list + e) : 0ull;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t e = e0 + lane + 32 * u;
        const uint32_t ke = static_cast<uint32_t>(v[u] >> 32);
        r += e < nb && ((ke > kq) || (ke == kq && static_cast<int>(v[u] & 0xFFFFFFFFu) < idq));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(0xFFFFFFFFu, r, o);
    if (r < need) {
      uint32_t pos = 0;
      if (lane == 0) pos = atomicAdd(qcount, 1u);
      pos = __shfl_sync(0xFFFFFFFFu, pos, 0);
      queue_cluster(P, rq, bitmap, pos, idq);
    }
  }
}

// Ascending list of the clusters set in `bitmap` into `sel` (at most cap).
__device__ void bitmap_to_list(const uint32_t* bitmap, int words, int32_t* sel, int cap, B1Misc* misc) {
  const int tid = threadIdx.x;
  uint32_t base = 0;
  for (int w0 = 0; w0 < words; w0 += kThreads) {
    const int w = w0 + tid;
    const uint32_t bits = w < words ? __ldcg(bitmap + w) : 0u;
    uint32_t total;
    const uint32_t before = block_exclusive_scan<kThreads, uint32_t>(static_cast<uint32_t>(__popc(bits)),
                                                                     misc->uscan, &total);
    uint32_t at = base + before, wb = bits;
    while (wb) {
      const int bit = __ffs(wb) - 1;
      wb &= wb - 1;
      if (at < static_cast<uint32_t>(cap)) sel[at] = w * 32 + bit;
      ++at;
    }
    base += total;
  }
  __syncthreads();
}

template <int NCH, bool INT4>
__global__ void __launch_bounds__(kThreads, 2) decode_b1_kernel(const B1Params P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = gridDim.x;
  const int d = P.d, b = P.b;
  const bool gumbel = P.mode == 1;

  float* hs = reinterpret_cast<float*>(smem + P.off_h);
  int32_t* ssel = reinterpret_cast<int32_t*>(smem + P.off_sel);
  B1Misc* misc = reinterpret_cast<B1Misc*>(smem + P.off_misc);
  uint8_t* scratch = smem + P.off_scratch;  // fallback select state

  // per-call state: two buffers used by alternate calls; this call clears the other one
  const uint32_t epoch = P.sync->epoch;
  const uint32_t par = epoch & 1u, nxt = par ^ 1u;
  uint32_t* hist = P.hist + par * kHistBins;
  uint32_t* bitmap = P.bitmap + par * P.words;
  unsigned long long* bnd_list = P.bnd_list + par * kBoundaryMax;
  uint32_t* bnd_count = P.counts + 2 * par;
  uint32_t* qcount = P.counts + 2 * par + 1;
  int32_t* rq = P.row_queue + static_cast<size_t>(par) * P.nc_max;
  uint32_t* bar1 = P.bars;
  uint32_t* bar2 = P.bars + kBarLanes * kBarStride;

  // ---------------- phase 1: centroid scores ----------------
  // Cluster k is owned by CTA k mod G, warp (k / G) mod 16, item k / (16 G):
  // every CTA owns c/G clusters, so phase 1 ends at the same time everywhere.
  // h goes out first, as one bulk copy per CTA (bf16, into the upper half of
  // the fp32 buffer); then the warp's first centroid row.
  const uint32_t hbar = smem_addr(&misc->hbar);
  uint16_t* hraw = reinterpret_cast<uint16_t*>(hs + d / 2);
  if (tid == 0) {
    mbar_init(hbar, 1);
    fence_mbar_init();
    mbar_expect_tx(hbar, static_cast<uint32_t>(d * 2));
    bulk_g2s(smem_addr(hraw), P.hidden, static_cast<uint32_t>(d * 2), hbar);
  }
  const int cw = static_cast<int>(blockIdx.x) + G * warp;  // first cluster of this warp
  const int n1 = cw < P.c ? (P.c - 1 - cw) / (G * kWarps) + 1 : 0;  // <= 32 (host-checked)
  auto cluster_of = [&](int i) { return cw + i * G * kWarps; };
  constexpr int NQ = (NCH + 1) / 2;
  uint4 w[NCH];
  uint2 q[NQ];
  uint32_t sc[NQ];
  // the warp's second row (if any) is requested at once into its shared-memory slot
  const uint32_t wbar = smem_addr(&misc->wbar[warp]);
  const uint32_t slot = smem_addr(smem + P.off_slots) + static_cast<uint32_t>(warp * P.slot_bytes);
  if (lane == 0) {
    mbar_init(wbar, 1);
    fence_mbar_init();
    if (n1 >= 2) {
      mbar_expect_tx(wbar, static_cast<uint32_t>(P.crow_bytes));
      bulk_g2s(slot, P.Crows + static_cast<size_t>(cluster_of(1)) * P.crow_bytes, static_cast<uint32_t>(P.crow_bytes),
               wbar);
    }
  }
  if (n1 > 0) {
    if constexpr (INT4) row_load_int4<NQ>(P.Crows + static_cast<size_t>(cw) * P.crow_bytes, d, q, sc);
    else row_load_bf16<NCH>(reinterpret_cast<const uint16_t*>(P.Crows + static_cast<size_t>(cw) * P.crow_bytes), d, w);
  }
  float ureg = 0.f;  // lane j holds u of item j
  if (gumbel && lane < n1) ureg = __ldg(P.u_clusters + cluster_of(lane));
  {
    const int nz = kHistBins + P.words + 2 + P.nc_max;
    const int per = (nz + G - 1) / G;
    for (int i = tid; i < per; i += kThreads) {
      int z = blockIdx.x * per + i;
      if (z < kHistBins) { P.hist[nxt * kHistBins + z] = 0u; continue; }
      z -= kHistBins;
      if (z < P.words) { P.bitmap[nxt * P.words + z] = 0u; continue; }
      z -= P.words;
      if (z < 2) { P.counts[2 * nxt + z] = 0u; continue; }
      z -= 2;
      if (z < P.nc_max) P.row_queue[static_cast<size_t>(nxt) * P.nc_max + z] = -1;
    }
  }
  if (tid == 0) misc->cta_sure = 0u;
  __syncthreads();  // hbar initialised before anyone waits on it
  if (!mbar_wait_bounded(hbar, 0u, kWaitBudget)) {
    if (lane == 0) record_error(&P.sync->status, FH_ERR_TIMEOUT);
  }
  // widen h in place (d <= 4 * kThreads, so one round: every chunk is read
  // before any is written): element e moves from hraw[e] to hs[e]
  {
    float hv[8];
    const int i = tid;
    if (i < d / 8) {
      const uint4 x = *reinterpret_cast<const uint4*>(hraw + 8 * i);
      hv[0] = bf16lo(x.x); hv[1] = bf16hi(x.x); hv[2] = bf16lo(x.y); hv[3] = bf16hi(x.y);
      hv[4] = bf16lo(x.z); hv[5] = bf16hi(x.z); hv[6] = bf16lo(x.w); hv[7] = bf16hi(x.w);
    }
    __syncthreads();
    if (i < d / 8) {
      reinterpret_cast<float4*>(hs)[2 * i] = make_float4(hv[0], hv[1], hv[2], hv[3]);
      reinterpret_cast<float4*>(hs)[2 * i + 1] = make_float4(hv[4], hv[5], hv[6], hv[7]);
    }
    __syncthreads();
  }

  uint32_t own_key = 0u;  // lane j: key of the warp's item j
  for (int i = 0; i < n1; ++i) {
    const int k = cluster_of(i);
    float s;
    if (i == 1) {  // the row that landed in the slot
      if (!mbar_wait_bounded(wbar, 0u, kWaitBudget) && lane == 0) record_error(&P.sync->status, FH_ERR_TIMEOUT);
      if constexpr (INT4) s = srow_dot_int4_hs<NQ>(slot, hs, d);
      else s = srow_dot_bf16_hs<NCH>(slot, hs, d);
    } else if constexpr (INT4) {
      if (i > 0) row_load_int4<NQ>(P.Crows + static_cast<size_t>(k) * P.crow_bytes, d, q, sc);
      s = row_dot_int4_hs<NQ>(q, sc, hs, d);
    } else {
      if (i > 0) row_load_bf16<NCH>(reinterpret_cast<const uint16_t*>(P.Crows + static_cast<size_t>(k) * P.crow_bytes), d, w);
      s = row_dot_bf16_hs<NCH>(w, hs, d);
    }
    const float u = __shfl_sync(0xFFFFFFFFu, ureg, i & 31);
    const float key = gumbel ? gumbel_key(s, P.T, u) : s;
    const uint32_t kk = f2key(key);
    if (lane == (i & 31)) own_key = kk;
    if (lane == 0) {
      P.keys[k] = kk;
      atomicAdd(hist + (kk >> kHistShift), 1u);
      prefetch_l2(P.C2T + static_cast<size_t>(k) * b);
    }
  }

  // ---------------- phase 2: barrier, boundary bin, owners publish ----------------
  bar_arrive(bar1);
  const bool passed = bar_wait(bar1, static_cast<uint32_t>(G), P.spin_budget, &misc->ok);
  unsigned long long best = 0ull;
  bool ok = true;
  if (!passed) {
    if (tid == 0) record_error(&P.sync->status, FH_ERR_TIMEOUT);
  } else {
    const uint32_t p = static_cast<uint32_t>(P.p);
    {
      // bin t1 of the p-th largest key: thread t owns bins 4095-8t .. 4088-8t
      constexpr int kBpt = kHistBins / kThreads;
      uint32_t hv[kBpt], loc = 0;
#pragma unroll
      for (int i = 0; i < kBpt; ++i) {
        hv[i] = __ldcg(hist + kHistBins - 1 - kBpt * tid - i);
        loc += hv[i];
      }
      const uint32_t above = block_exclusive_scan<kThreads, uint32_t>(loc, misc->uscan, nullptr);
      uint32_t run = above;
#pragma unroll
      for (int i = 0; i < kBpt; ++i) {
        if (run < p && run + hv[i] >= p) {
          const uint32_t need = p - run;
          misc->t1 = static_cast<uint32_t>(kHistBins - 1 - kBpt * tid - i);
          misc->need = need;
          misc->split = hv[i] != need ? 1u : 0u;
          misc->fallback = (hv[i] != need && hv[i] > static_cast<uint32_t>(kBoundaryMax)) ? 1u : 0u;
          misc->n_sure = hv[i] != need ? run : p;
        }
        run += hv[i];
      }
    }
    __syncthreads();
    const uint32_t t1 = misc->t1, need = misc->need;
    const bool split = misc->split != 0, fallback = misc->fallback != 0;
    const int r_all = P.p * b;
    const uint32_t dg = own_key >> kHistShift;
    const bool mine = lane < n1;
    uint32_t bnd_mine = 0u;

    if (!fallback) {
      // one queue reservation per CTA for its surely selected clusters
      const uint32_t sure = __ballot_sync(0xFFFFFFFFu, mine && (dg > t1 || (dg == t1 && !split)));
      uint32_t off = 0;
      if (lane == 0 && sure) off = atomicAdd(&misc->cta_sure, static_cast<uint32_t>(__popc(sure)));
      off = __shfl_sync(0xFFFFFFFFu, off, 0);
      __syncthreads();
      if (tid == 0) misc->qbase = misc->cta_sure ? atomicAdd(qcount, misc->cta_sure) : 0u;
      __syncthreads();
      uint32_t pos = misc->qbase + off, sm = sure;
      while (sm) {
        const int j = __ffs(sm) - 1;
        sm &= sm - 1;
        queue_cluster(P, rq, bitmap, pos++, cluster_of(j));
      }
      bnd_mine = __ballot_sync(0xFFFFFFFFu, mine && split && dg == t1);
      if (bnd_mine & (1u << lane)) {
        const uint32_t at = atomicAdd(bnd_count, 1u);
        if (at < static_cast<uint32_t>(kBoundaryMax))
          bnd_list[at] = (static_cast<unsigned long long>(own_key) << 32) | static_cast<uint32_t>(cluster_of(lane));
      }
      __threadfence();
      if (split) bar_arrive(bar2);
    } else {
      // pathological ties (a boundary bin larger than the exact-rank list):
      // every CTA selects over all keys and reads its rows' tokens directly
      block_select_top_p(P.keys, P.c, P.p, ssel, *reinterpret_cast<SelectSmem*>(scratch));
      if (blockIdx.x == 0)
        for (int i = tid; i < P.p; i += kThreads) atomicOr(bitmap + (ssel[i] >> 5), 1u << (ssel[i] & 31));
    }

    // ---------------- phases 3-4: consume candidate rows ----------------
    bool ranked = bnd_mine == 0u;
    const long long budget = P.spin_budget;
    // candidate row r goes to CTA r mod G, warp (r / G) mod 16: balanced like phase 1
    for (int r = static_cast<int>(blockIdx.x) + G * warp; r < r_all; r += G * kWarps) {
      int t;
      if (fallback) {
        t = __ldg(P.C2T + static_cast<size_t>(ssel[r / b]) * b + r % b);
      } else {
        long long t0 = 0;
        for (;;) {
          if (!ranked) {  // publish this warp's boundary choices once the list is complete
            uint32_t ready = 0;
            if (lane == 0) ready = bar_count(bar2) >= static_cast<uint32_t>(G);
            if (__shfl_sync(0xFFFFFFFFu, ready, 0)) {
              __threadfence();
              rank_boundary(P, rq, bitmap, qcount, bnd_list, bnd_count, bnd_mine, own_key, cw, G * kWarps, need);
              ranked = true;
            }
          }
          int v = 0;
          if (lane == 0) v = static_cast<int>(ld_acquire_u32(reinterpret_cast<const unsigned*>(rq + r)));
          t = __shfl_sync(0xFFFFFFFFu, v, 0);
          if (t >= 0) break;
          if (t0 == 0) t0 = clock64();
          else if (clock64() - t0 > budget) break;
        }
        if (t < 0) {
          ok = false;
          continue;
        }
      }
      uint4 e[NCH];
      row_load_bf16<NCH>(P.E + static_cast<size_t>(t) * d, d, e);
      const float z = row_dot_bf16_hs<NCH>(e, hs, d);
      const unsigned long long pk = pack_best(z, t);
      best = pk > best ? pk : best;
      if (gumbel && lane == 0) P.z_tok[t] = z;
    }
    if (!ranked) {  // no rows left to poll on: wait for the list, then publish
      long long t0 = clock64();
      uint32_t ready = 0;
      for (;;) {
        if (lane == 0) ready = bar_count(bar2) >= static_cast<uint32_t>(G);
        if (__shfl_sync(0xFFFFFFFFu, ready, 0)) break;
        if (clock64() - t0 > budget) break;
      }
      if (__shfl_sync(0xFFFFFFFFu, ready, 0)) {
        __threadfence();
        rank_boundary(P, rq, bitmap, qcount, bnd_list, bnd_count, bnd_mine, own_key, cw, G * kWarps, need);
      }
      else {
        ok = false;
      }
    }
    if (!ok && lane == 0) record_error(&P.sync->status, FH_ERR_TIMEOUT);
  }
  best = warp_max_u64(best);
  if (lane == 0) misc->wbest[warp] = best;
  __syncthreads();
  if (tid == 0) {
    unsigned long long m = 0ull;
    for (int i = 0; i < kWarps; ++i) m = misc->wbest[i] > m ? misc->wbest[i] : m;
    if (m) atomicMax(P.best, m);
  }

  // ---------------- exit: the last CTA writes the token ----------------
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const uint32_t t = atomicAdd(&P.sync->ticket, 1u);
    misc->last = (t == static_cast<uint32_t>(G - 1));
  }
  __syncthreads();
  if (!misc->last) return;
  __threadfence();

  const unsigned long long bw = *reinterpret_cast<volatile unsigned long long*>(P.best);
  if (passed && (gumbel || P.out_cluster_ids)) {
    bitmap_to_list(bitmap, P.words, ssel, P.p, misc);
    if (P.out_cluster_ids)
      for (int i = tid; i < P.p; i += kThreads) P.out_cluster_ids[i] = ssel[i];
  }
  if (!gumbel || !passed) {
    if (tid == 0) {
      P.out_tokens[0] = best_token(bw);
      if (P.out_max_logit) P.out_max_logit[0] = best_logit(bw);
    }
  } else {
    // inverse CDF over softmax(z/T), canonical order (cluster asc, slot asc)
    const int nc = P.p * b;
    const float ym = best_logit(bw) / P.T;
    const int qn = (nc + kThreads - 1) / kThreads;
    const int i0 = min(nc, tid * qn), i1 = min(nc, i0 + qn);
    auto tok_at = [&](int i) { return __ldg(P.C2T + static_cast<size_t>(ssel[i / b]) * b + i % b); };
    float loc = 0.f;
    for (int i = i0; i < i1; ++i) loc += expf(__ldcg(P.z_tok + tok_at(i)) / P.T - ym);
    if (tid == 0) {
      misc->claim = INT_MAX;
      misc->lastpos = 0;
    }
    float total;
    const float before = block_exclusive_scan<kThreads, float>(loc, misc->scan, &total);
    const float u = fminf(fmaxf(__ldg(P.u_token), 0.f), 0.99999994f);
    const float target = u * total;
    float run = before;
    int claim = INT_MAX, lastpos = -1;
    for (int i = i0; i < i1; ++i) {
      const float wgt = expf(__ldcg(P.z_tok + tok_at(i)) / P.T - ym);
      if (wgt > 0.f) lastpos = i;
      run += wgt;
      if (run > target) {
        claim = i;
        break;
      }
    }
    if (claim != INT_MAX) atomicMin(&misc->claim, claim);
    if (lastpos >= 0) atomicMax(&misc->lastpos, lastpos);
    __syncthreads();
    if (tid == 0) {
      const int idx = misc->claim != INT_MAX ? misc->claim : misc->lastpos;
      P.out_tokens[0] = tok_at(idx);
      if (P.out_max_logit) P.out_max_logit[0] = best_logit(bw);
    }
  }
  if (tid < 2 * kBarLanes) P.bars[tid * kBarStride] = 0u;
  if (tid == 0) {
    *P.best = 0ull;
    P.sync->ticket = 0u;
    P.sync->epoch = epoch + 1u;
  }
  __threadfence();
}

template <int NCH>
cudaError_t launch_nch(const B1Params& P, int grid, size_t smem, int int4, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (int4) return cudaLaunchKernelEx(&cfg, decode_b1_kernel<NCH, true>, P);
  return cudaLaunchKernelEx(&cfg, decode_b1_kernel<NCH, false>, P);
}

}  // namespace

size_t decode_b1_misc_bytes() { return sizeof(B1Misc); }
size_t decode_b1_bar_words() { return 2 * kBarLanes * kBarStride; }

cudaError_t launch_decode_b1(const B1Params& P, int grid, size_t smem, int int4, int nch, cudaStream_t st) {
  switch (nch) {
    case 1: return launch_nch<1>(P, grid, smem, int4, st);
    case 2: return launch_nch<2>(P, grid, smem, int4, st);
    case 3: return launch_nch<3>(P, grid, smem, int4, st);
    case 4: return launch_nch<4>(P, grid, smem, int4, st);
    case 5: return launch_nch<5>(P, grid, smem, int4, st);
    case 6: return launch_nch<6>(P, grid, smem, int4, st);
    case 8: return launch_nch<8>(P, grid, smem, int4, st);
    case 10: return launch_nch<10>(P, grid, smem, int4, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t occupancy_decode_b1(int int4, int nch, size_t smem, int* blocks) {
#define FH_O(N)                                                                                      \
  return int4 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks, decode_b1_kernel<N, true>, kThreads, smem) \
              : cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks, decode_b1_kernel<N, false>, kThreads, smem);
  switch (nch) {
    case 1: FH_O(1)
    case 2: FH_O(2)
    case 3: FH_O(3)
    case 4: FH_O(4)
    case 5: FH_O(5)
    case 6: FH_O(6)
    case 8: FH_O(8)
    case 10: FH_O(10)
    default: return cudaErrorInvalidValue;
  }
#undef FH_O
}

cudaError_t set_attrs_decode_b1(int max_smem) {
  cudaError_t e = cudaSuccess;
#define FH_SET(N)                                                                                         \
  if (e == cudaSuccess)                                                                                   \
    e = cudaFuncSetAttribute(decode_b1_kernel<N, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem); \
  if (e == cudaSuccess)                                                                                   \
    e = cudaFuncSetAttribute(decode_b1_kernel<N, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
  FH_SET(1) FH_SET(2) FH_SET(3) FH_SET(4) FH_SET(5) FH_SET(6) FH_SET(8) FH_SET(10)
#undef FH_SET
  return e;
}

}  // namespace fh
