// Fused FlashHead decode for one hidden state (B = 1): one persistent
// cooperative launch of one 512-thread CTA per SM.
//
// The pages' pipeline (FlashHead write-up, section 2.2.2: h -> centroid_scores
// -> top_p_clusters -> token_scores) runs as phases of one kernel:
//
//  1. centroid scores (section 1.2.2; INT4 centroids per section 1.2.4): the
//     c centroid rows are spread round-robin over every warp of the grid
//     (cluster k belongs to global warp k mod W); each warp streams its rows
//     HBM -> shared memory with cp.async.bulk into a private ring of slots and
//     dots them with h held in registers. The key (the score, or when sampling
//     the Gumbel key s/T - ln(-ln u), section 1.2.3) stays in a lane register
//     of the owning warp and is counted into two device-wide histograms of its
//     top 8 and top 12 bits (fire-and-forget atomics).
//  2. device-wide barrier; one warp per CTA reads the two small histograms and
//     finds the 12-bit bin t1 holding the p-th largest key. Every key above t1
//     is selected; the keys inside t1 are the boundary. Each CTA classifies
//     only the clusters it owns -- no CTA ever reads all c keys.
//  3. each CTA streams the token rows of its own surely-selected clusters
//     (gather through C2T, section 1.2.1: slot k*b + j holds token C2T[k][j]),
//     dots them with h and keeps a packed (logit, token) maximum.
//  4. only when the boundary bin is split (some but not all of its keys are
//     needed): the boundary keys were published to a small global list, a
//     second barrier (whose wait overlaps step 3) completes it, and each CTA
//     ranks its own boundary keys exactly (key desc, id asc) and streams the
//     ones that are in.
//  5. the CTA maxima meet in one 64-bit atomicMax; the last CTA to finish
//     (exit ticket) writes the token: the argmax, or, when sampling, the
//     inverse-CDF draw over softmax(z/T) in canonical order (cluster asc, slot
//     asc), walking a bitmap of the selected clusters.
//
// HBM traffic is the algorithmic minimum: each centroid row once, each
// selected token row once, plus the C2T rows and h.
#include <climits>

#include "fh_device.cuh"

namespace fh {
namespace {

constexpr int kHiBins = 256;
constexpr int kMaxOwn = kWarps * 32;  // clusters a CTA can own (32 per warp)

struct B1Misc {
  unsigned long long hbar;
  unsigned long long wbest[kWarps];
  float scan[kWarps + 1];
  uint32_t uscan[kWarps + 1];
  int claim, lastpos, ok, last;
  uint32_t t1, need, split, fallback;
  uint32_t n_sure, n_bnd, n_bsel;
  int32_t sure[kMaxOwn];
  int32_t bnd[kMaxOwn];
  uint32_t bnd_key[kMaxOwn];
};

// Device-wide barrier over the cooperative grid; false if `budget` cycles pass first.
__device__ bool grid_barrier(uint32_t* arrive, uint32_t G, long long budget, B1Misc* misc) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(arrive, 1u);
    int ok = 1;
    if (ld_acquire_u32(arrive) < G) {
      const long long t0 = clock64();
      while (ld_acquire_u32(arrive) < G) {
        if (clock64() - t0 > budget) {
          ok = 0;
          break;
        }
      }
    }
    __threadfence();
    misc->ok = ok;
  }
  __syncthreads();
  return misc->ok != 0;
}

// Warp-inclusive prefix sum over lanes.
__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t x) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  return x;
}

// Stream the rows of `n_items` candidate slots of this CTA (item q -> cluster
// list[q / b], slot q % b) through the warp rings; items go round-robin over
// the CTA's warps. Updates `best` and, when sampling, the per-slot logits.
template <int NCH>
__device__ __forceinline__ bool stream_candidates(const B1Params& P, const int32_t* list, int n_items,
                                                  const float* hr, uint32_t ring_w, uint32_t bar_w,
                                                  uint32_t& phase_bits, unsigned long long& best,
                                                  bool gumbel) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n = warp < n_items ? (n_items - 1 - warp) / kWarps + 1 : 0;
  const int b = P.b;
  auto slot_of = [&](int i) -> int {  // flat index k*b + j of the warp's item i
    const int q = warp + i * kWarps;
    return list[q / b] * b + q % b;
  };
  int tok0 = 0, tok1 = 0;  // lane j: tokens of items j and 32 + j
  if (lane < n) tok0 = __ldg(P.C2T + slot_of(lane));
  if (32 + lane < n) tok1 = __ldg(P.C2T + slot_of(32 + lane));
  auto token_of = [&](int i) -> int {
    const int a = __shfl_sync(0xFFFFFFFFu, tok0, i & 31);
    const int c1 = __shfl_sync(0xFFFFFFFFu, tok1, i & 31);
    if (i < 32) return a;
    if (i < 64) return c1;
    return __ldg(P.C2T + slot_of(i));
  };
  auto src = [&](int i, const void*& ptr, uint32_t& bytes) {
    ptr = P.E + static_cast<size_t>(token_of(i)) * P.d;
    bytes = static_cast<uint32_t>(P.d * 2);
  };
  auto use = [&](int i, uint32_t slot) {
    const int t = token_of(i);
    const float z = row_dot_bf16<NCH>(slot, P.d, hr);
    const unsigned long long pk = pack_best(z, t);
    best = pk > best ? pk : best;
    if (gumbel && lane == 0) P.z_slot[slot_of(i)] = z;
  };
  return warp_stream(n, P.nslot, ring_w, P.slot_bytes, bar_w, phase_bits, kWaitBudget, src, use);
}

// Ascending list of the clusters set in `bitmap` (words of 32 ids) into `sel`.
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
__global__ void __launch_bounds__(kThreads, 1) decode_b1_kernel(const B1Params P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = gridDim.x;
  const int W = G * kWarps;
  const int gw = blockIdx.x * kWarps + warp;
  const int d = P.d;

  uint16_t* sh = reinterpret_cast<uint16_t*>(smem + P.off_h);
  int32_t* ssel = reinterpret_cast<int32_t*>(smem + P.off_sel);
  B1Misc* misc = reinterpret_cast<B1Misc*>(smem + P.off_misc);
  uint8_t* ring = smem + P.off_ring;
  const uint32_t ring_w = smem_addr(ring) + static_cast<uint32_t>(warp * P.nslot * P.slot_bytes);
  const uint32_t bar_w = smem_addr(smem + P.off_bar) + static_cast<uint32_t>(warp * P.nslot * 8);

  uint32_t phase_bits = 0;
  bool ok = true;
  const bool gumbel = P.mode == 1;
  // per-call state lives in two buffers used by alternate calls; this call
  // clears the other buffer for the next one
  const uint32_t epoch = P.sync->epoch;
  const uint32_t par = epoch & 1u, nxt = par ^ 1u;
  uint32_t* hist_hi = P.hist_hi + par * kHiBins;
  uint32_t* hist_lo = P.hist_lo + par * kHistBins;
  uint32_t* bitmap = P.bitmap + par * P.words;
  unsigned long long* bnd_list = P.bnd_list + par * kBoundaryMax;
  uint32_t* bnd_count = P.bnd_count + par;

  // ---------------- phase 1: centroid scores ----------------
  // h is staged by the first bulk copy of the CTA; the centroid rows follow
  // at once (they do not depend on h).
  const uint32_t hbar = smem_addr(&misc->hbar);
  if (tid == 0) {
    mbar_init(hbar, 1);
    fence_mbar_init();
    mbar_expect_tx(hbar, static_cast<uint32_t>(d * 2));
    bulk_g2s(smem_addr(sh), P.hidden, static_cast<uint32_t>(d * 2), hbar);
  }
  warp_ring_init(bar_w, P.nslot);
  const int n1 = gw < P.c ? (P.c - 1 - gw) / W + 1 : 0;  // <= 32 (host-checked)
  auto src1 = [&](int i, const void*& ptr, uint32_t& bytes) {
    ptr = P.Crows + static_cast<size_t>(gw + i * W) * P.crow_bytes;
    bytes = static_cast<uint32_t>(P.crow_bytes);
  };
  warp_stream_prologue(n1, P.nslot, ring_w, P.slot_bytes, bar_w, src1);
  float ureg = 0.f;  // lane j holds u of item j
  if (gumbel && lane < n1) ureg = __ldg(P.u_clusters + gw + lane * W);
  {
    const int nz = kHiBins + kHistBins + P.words + 1;
    const int per = (nz + G - 1) / G;
    for (int i = tid; i < per; i += kThreads) {
      const int z = blockIdx.x * per + i;
      if (z < kHiBins) P.hist_hi[nxt * kHiBins + z] = 0u;
      else if (z < kHiBins + kHistBins) P.hist_lo[nxt * kHistBins + (z - kHiBins)] = 0u;
      else if (z < kHiBins + kHistBins + P.words) P.bitmap[nxt * P.words + (z - kHiBins - kHistBins)] = 0u;
      else if (z == nz - 1) P.bnd_count[nxt] = 0u;
    }
  }
  if (tid == 0) {
    misc->n_sure = 0u;
    misc->n_bnd = 0u;
    misc->n_bsel = 0u;
  }
  __syncthreads();  // hbar initialised before anyone waits on it
  if (!mbar_wait_bounded(hbar, 0u, kWaitBudget)) {
    ok = false;
    if (lane == 0) record_error(&P.sync->status, FH_ERR_TIMEOUT);
  }
  uint32_t own_key = 0u;  // lane j: key of the warp's item j
  {
    auto finish = [&](int i, float s) {
      const int k = gw + i * W;
      const float u = __shfl_sync(0xFFFFFFFFu, ureg, i & 31);
      const float key = gumbel ? gumbel_key(s, P.T, u) : s;
      const uint32_t kk = f2key(key);
      if (lane == (i & 31)) own_key = kk;
      if (lane == 0) {
        P.scores[k] = key;
        atomicAdd(hist_hi + (kk >> 24), 1u);
        atomicAdd(hist_lo + (kk >> kHistShift), 1u);
        prefetch_l2(P.C2T + static_cast<size_t>(k) * P.b);
      }
    };
    if constexpr (INT4) {
      constexpr int NQ = (NCH + 1) / 2;
      float hq[NQ * 16];
      load_h_halfgroups<NQ>(sh, d, hq);
      auto use = [&](int i, uint32_t slot) { finish(i, row_dot_int4<NQ>(slot, d, hq)); };
      ok = warp_stream_run(n1, P.nslot, ring_w, P.slot_bytes, bar_w, phase_bits, kWaitBudget, src1, use) && ok;
    } else {
      float hr[NCH * 8];
      load_h_chunks<NCH>(sh, d, hr);
      auto use = [&](int i, uint32_t slot) { finish(i, row_dot_bf16<NCH>(slot, d, hr)); };
      ok = warp_stream_run(n1, P.nslot, ring_w, P.slot_bytes, bar_w, phase_bits, kWaitBudget, src1, use) && ok;
    }
    if (!ok && lane == 0) record_error(&P.sync->status, FH_ERR_TIMEOUT);
  }

  // ---------------- phase 2: barrier, boundary bin, own classification ----------------
  const bool passed = grid_barrier(&P.sync->arrive, static_cast<uint32_t>(G), P.spin_budget, misc);
  unsigned long long best = 0ull;
  if (!passed) {
    if (tid == 0) record_error(&P.sync->status, FH_ERR_TIMEOUT);
  } else {
    const uint32_t p = static_cast<uint32_t>(P.p);
    if (warp == 0) {
      // top-8-bit bins, descending: lane l owns bins 255-8l .. 248-8l
      uint32_t hv[8], s = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        hv[i] = __ldcg(hist_hi + kHiBins - 1 - 8 * lane - i);
        s += hv[i];
      }
      const uint32_t incl = warp_incl_scan(s), excl = incl - s;
      const int L = __ffs(__ballot_sync(0xFFFFFFFFu, excl < p && p <= incl)) - 1;
      uint32_t thi = 0, above_hi = 0, run = excl;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (run < p && run + hv[i] >= p) {
          thi = kHiBins - 1 - 8 * lane - i;
          above_hi = run;
        }
        run += hv[i];
      }
      thi = __shfl_sync(0xFFFFFFFFu, thi, L);
      above_hi = __shfl_sync(0xFFFFFFFFu, above_hi, L);
      // its 16 sub-bins of 12 bits, descending
      const uint32_t x = lane < 16 ? __ldcg(hist_lo + thi * 16 + 15 - lane) : 0u;
      const uint32_t incl2 = warp_incl_scan(x), excl2 = incl2 - x;
      const uint32_t target = p - above_hi;
      const int L2 = __ffs(__ballot_sync(0xFFFFFFFFu, lane < 16 && excl2 < target && target <= incl2)) - 1;
      const uint32_t ex2 = __shfl_sync(0xFFFFFFFFu, excl2, L2);
      const uint32_t m1 = __shfl_sync(0xFFFFFFFFu, x, L2);
      if (lane == 0) {
        misc->t1 = thi * 16 + 15 - L2;
        misc->need = target - ex2;
        misc->split = (m1 != target - ex2) ? 1u : 0u;
        misc->fallback = (m1 != target - ex2 && m1 > static_cast<uint32_t>(kBoundaryMax)) ? 1u : 0u;
      }
    }
    __syncthreads();
    const uint32_t t1 = misc->t1;
    const bool split = misc->split != 0, fallback = misc->fallback != 0;

    if (!fallback) {
      if (lane < n1) {
        const int k = gw + lane * W;
        const uint32_t dg = own_key >> kHistShift;
        if (dg > t1 || (dg == t1 && !split)) {
          misc->sure[atomicAdd(&misc->n_sure, 1u)] = k;
          atomicOr(bitmap + (k >> 5), 1u << (k & 31));
        } else if (dg == t1) {
          const uint32_t q = atomicAdd(&misc->n_bnd, 1u);
          misc->bnd[q] = k;
          misc->bnd_key[q] = own_key;
          const uint32_t at = atomicAdd(bnd_count, 1u);
          if (at < static_cast<uint32_t>(kBoundaryMax))
            bnd_list[at] = (static_cast<unsigned long long>(own_key) << 32) | static_cast<uint32_t>(k);
        }
      }
      __syncthreads();
      if (split && tid == 0) {  // boundary keys published: arrive at the second barrier
        __threadfence();
        atomicAdd(&P.sync->arrive2, 1u);
      }
    } else {
      // pathological ties (huge boundary bin): every CTA selects over all keys
      select_top_p_hist(P.scores, nullptr, 1.f, P.c, P.p, hist_lo, ssel, ring);
      for (int q = tid; q < P.p; q += kThreads) {
        const int k = ssel[q];
        if ((k % W) / kWarps == static_cast<int>(blockIdx.x)) {
          misc->sure[atomicAdd(&misc->n_sure, 1u)] = k;
          atomicOr(bitmap + (k >> 5), 1u << (k & 31));
        }
      }
      __syncthreads();
    }
    fence_proxy_async_smem();
    __syncthreads();

    // ---------------- phase 3: stream own selected clusters ----------------
    float hr[NCH * 8];
    load_h_chunks<NCH>(sh, d, hr);
    ok = stream_candidates<NCH>(P, misc->sure, static_cast<int>(misc->n_sure) * P.b, hr, ring_w, bar_w,
                                phase_bits, best, gumbel);
    if (!ok && lane == 0) record_error(&P.sync->status, FH_ERR_TIMEOUT);

    if (split && !fallback) {
      // ---------------- phase 4: exact rank of own boundary keys ----------------
      __syncthreads();
      if (tid == 0) {
        int bok = 1;
        if (ld_acquire_u32(&P.sync->arrive2) < static_cast<uint32_t>(G)) {
          const long long t0 = clock64();
          while (ld_acquire_u32(&P.sync->arrive2) < static_cast<uint32_t>(G)) {
            if (clock64() - t0 > P.spin_budget) {
              bok = 0;
              break;
            }
          }
        }
        __threadfence();
        misc->ok = bok;
      }
      __syncthreads();
      if (!misc->ok) {
        if (tid == 0) record_error(&P.sync->status, FH_ERR_TIMEOUT);
      } else {
        const uint32_t nb = min(__ldcg(bnd_count), static_cast<uint32_t>(kBoundaryMax));
        unsigned long long* sl = reinterpret_cast<unsigned long long*>(ring);
        for (uint32_t i = tid; i < nb; i += kThreads) sl[i] = __ldcg(bnd_list + i);
        __syncthreads();
        const uint32_t need = misc->need;
        for (uint32_t q = warp; q < misc->n_bnd; q += kWarps) {
          const uint32_t kq = misc->bnd_key[q];
          const int idq = misc->bnd[q];
          uint32_t r = 0;
          for (uint32_t e = lane; e < nb; e += 32) {
            const unsigned long long v = sl[e];
            const uint32_t ke = static_cast<uint32_t>(v >> 32);
            const int ide = static_cast<int>(v & 0xFFFFFFFFu);
            r += (ke > kq) || (ke == kq && ide < idq);
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(0xFFFFFFFFu, r, o);
          if (lane == 0 && r < need) {
            misc->sure[atomicAdd(&misc->n_bsel, 1u)] = idq;  // sure[] was consumed by phase 3
            atomicOr(bitmap + (idq >> 5), 1u << (idq & 31));
          }
        }
        fence_proxy_async_smem();
        __syncthreads();
        const int nbs = static_cast<int>(misc->n_bsel);
        ok = stream_candidates<NCH>(P, misc->sure, nbs * P.b, hr, ring_w, bar_w, phase_bits, best, gumbel);
        if (!ok && lane == 0) record_error(&P.sync->status, FH_ERR_TIMEOUT);
      }
    }
  }
  best = warp_max_u64(best);
  if (lane == 0) misc->wbest[warp] = best;
  __syncthreads();
  if (tid == 0) {
    unsigned long long m = 0ull;
    for (int w = 0; w < kWarps; ++w) m = misc->wbest[w] > m ? misc->wbest[w] : m;
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
    const int nc = P.p * P.b, b = P.b;
    const float ym = best_logit(bw) / P.T;
    const int q = (nc + kThreads - 1) / kThreads;
    const int i0 = min(nc, tid * q), i1 = min(nc, i0 + q);
    auto zc = [&](int i) { return __ldcg(P.z_slot + static_cast<size_t>(ssel[i / b]) * b + i % b); };
    float loc = 0.f;
    for (int i = i0; i < i1; ++i) loc += expf(zc(i) / P.T - ym);
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
      const float w = expf(zc(i) / P.T - ym);
      if (w > 0.f) lastpos = i;
      run += w;
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
      P.out_tokens[0] = __ldg(P.C2T + static_cast<size_t>(ssel[idx / b]) * b + idx % b);
      if (P.out_max_logit) P.out_max_logit[0] = best_logit(bw);
    }
  }
  if (tid == 0) {
    *P.best = 0ull;
    P.sync->arrive = 0u;
    P.sync->arrive2 = 0u;
    P.sync->ticket = 0u;
    P.sync->epoch = epoch + 1u;
    __threadfence();
  }
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
