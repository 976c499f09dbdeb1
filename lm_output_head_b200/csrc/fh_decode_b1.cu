// Fused FlashHead decode for one hidden state (B = 1): one persistent
// cooperative launch, two 512-thread CTAs per SM, every row streamed from
// HBM with non-allocating loads and dotted with h staged once per CTA in
// shared memory (fp32).
//
// The pages' pipeline (FlashHead write-up, section 2.2.2: h -> centroid_scores
// -> top_p_clusters -> token_scores) runs as phases of one kernel:
//
//  1. centroid scores (section 1.2.2; INT4 or INT8 centroids per section 1.2.4):
//     cluster k belongs to CTA k mod G (warp (k / G) mod 16), so every CTA
//     owns c/G clusters. A warp's first row streams into registers, its
//     second into a shared-memory slot by one bulk copy, both requested at
//     kernel start. The key -- the score, or when sampling the Gumbel key
//     s/T - ln(-ln u) (section 1.2.3) -- goes to global memory. A key that
//     falls in the region where the p-th key is expected (predicted from the
//     previous call: from its rank-2p key up to its rank-p key plus twice
//     their distance, relative to |h| when greedy) also counts in a global
//     histogram of that region (kB1Bins equal bins; keys above it count in the
//     top bin) and is appended, (key, id), to a short candidate list (one
//     reservation per CTA).
//  2. one grid-wide arrival count (release / acquire); then every CTA
//     selects the same boundary redundantly from the histogram and the list:
//     the bin holding the p-th largest key, and an exact rank (key desc, id
//     asc) of that bin's few entries. Cluster k is chosen iff its (key, id)
//     reaches the boundary entry, so the chosen set is the list entries that
//     reach it -- no CTA waits for a published selection. If the region holds
//     fewer than p keys or the boundary bin is crowded (the first call, a poor
//     prediction, heavy ties), the CTA runs the general exact selector over
//     all c keys instead.
//  3. the chosen clusters in a fixed order (list order, or ascending ids after
//     the general selector) give the candidate rows: row r is slot r % b of
//     the (r / b)-th chosen cluster and belongs to CTA r mod G, warp
//     (r / G) mod 16; it is read from the head's cluster-major copy of E (row
//     k*b + j holds token C2T[k][j], so no C2T lookup precedes the row load)
//     and dotted with h (section 1.2.4, stage 2), keeping a packed (logit,
//     token) maximum.
//  4. CTA maxima meet in one 64-bit atomicMax; the last CTA to finish (exit
//     ticket) writes the token: the argmax, or, when sampling, the inverse-CDF
//     draw over softmax(z/T) in canonical order (cluster asc, slot asc)
//     through the per-slot logit buffer. It also stores this call's rank-p
//     and rank-2p keys for the next call and clears the histogram.
//
// The result does not depend on the prediction: it only decides whether the
// short list or the general selector finds the boundary.
#include <algorithm>
#include <climits>

#include "fh_device.cuh"

namespace fh {
namespace {


static_assert(kB1Bins == 4 * kThreads, "each thread scans four histogram bins");

constexpr int kNoteMax = kThreads;  // list entries one CTA stages (it owns at most 16 * 32 clusters)

struct B1Misc {
  unsigned long long hbar;
  unsigned long long wbar[kWarps];
  unsigned long long wbest[kWarps];
  float scan[kWarps + 1];
  uint32_t uscan[kWarps + 1];
  int claim, lastpos, last, full;
  uint32_t t1, above, m1, t2, total;
  uint32_t bkey;
  int32_t bid;
  float edge_2p;
  uint32_t nnote, base, nlist;
  int32_t note_k[kNoteMax];
  uint32_t note_key[kNoteMax];
};

__device__ __forceinline__ bool chosen(uint32_t key, int32_t id, uint32_t bkey, int32_t bid) {
  return key > bkey || (key == bkey && id <= bid);
}

__device__ __forceinline__ size_t up128(size_t x) { return (x + 127) & ~size_t(127); }

// Histogram bin of a key in the predicted region [L, L + kB1Bins / S): -1
// below it, the top bin above it. Every CTA evaluates it with the same L, S
// and the same rounding, so all agree on every key's bin.
__device__ __forceinline__ int region_bin(float key, float L, float S) {
  if (!(key >= L)) return -1;
  const float x = __fmul_rn(__fsub_rn(key, L), S);
  return x >= static_cast<float>(kB1Bins - 1) ? kB1Bins - 1 : static_cast<int>(x);
}

template <int NCH, int FMT>
__global__ void __launch_bounds__(kThreads, 2) decode_b1_kernel(const B1Params P) {
  constexpr bool INT4 = FMT == kFmtInt4, INT8 = FMT == kFmtInt8;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = gridDim.x;
  const int d = P.d, b = P.b;
  const bool gumbel = P.mode == 1;

  float* hs = reinterpret_cast<float*>(smem + P.off_h);
  int32_t* ssel = reinterpret_cast<int32_t*>(smem + P.off_sel);  // the chosen clusters, ascending
  B1Misc* misc = reinterpret_cast<B1Misc*>(smem + P.off_misc);
  uint8_t* slots = smem + P.off_slots;  // per-warp row slots; the selection's scratch between phases


  // ---------------- phase 1: centroid scores ----------------
  const uint32_t hbar = smem_addr(&misc->hbar);
  const uint32_t wbar = smem_addr(&misc->wbar[warp]);
  const uint32_t slot = smem_addr(slots) + static_cast<uint32_t>(warp * P.slot_bytes);
  uint16_t* hraw = reinterpret_cast<uint16_t*>(hs + d / 2);
  const int cw = static_cast<int>(blockIdx.x) + G * warp;  // first cluster of this warp
  const int cstride = G * kWarps;
  const int n1 = cw < P.c ? (P.c - 1 - cw) / cstride + 1 : 0;  // <= 32 (host-checked)
  uint32_t wphase = 0;  // parity of this warp's slot barrier
  // h is requested first, then every warp's first two centroid rows: one into
  // registers, one into its slot by a bulk copy
  if (tid == 0) {
    mbar_init(hbar, 1);
    fence_mbar_init();
    mbar_expect_tx(hbar, static_cast<uint32_t>(d * 2));
    bulk_g2s(smem_addr(hraw), P.hidden, static_cast<uint32_t>(d * 2), hbar);
    misc->nnote = 0u;
  }
  if (lane == 0) {
    mbar_init(wbar, 1);
    fence_mbar_init();
    if (n1 >= 2) {
      mbar_expect_tx(wbar, static_cast<uint32_t>(P.crow_bytes));
      bulk_g2s(slot, P.Crows + static_cast<size_t>(cw + cstride) * P.crow_bytes, static_cast<uint32_t>(P.crow_bytes),
               wbar);
    }
  }
  uint4 w[NCH];
  uint32_t q[NCH], sc[NCH];
  uint2 q8[NCH];
  uint32_t sw8[int8_scale_words<NCH>()];
  if (n1 > 0) {
    if constexpr (INT4) row_load_int4<NCH>(P.Crows + static_cast<size_t>(cw) * P.crow_bytes, d, q, sc);
    else if constexpr (INT8) row_load_int8<NCH>(P.Crows + static_cast<size_t>(cw) * P.crow_bytes, d, q8, sw8);
    else row_load_bf16<NCH>(reinterpret_cast<const uint16_t*>(P.Crows + static_cast<size_t>(cw) * P.crow_bytes), d, w);
  }
  float ureg = 0.f;  // lane j holds u of item j
  if (gumbel && lane < n1) ureg = __ldg(P.u_clusters + cw + lane * cstride);
  const int mi = gumbel ? 1 : 0;
  const uint32_t prior_ok = P.sync->prior_ok[mi];
  const float prior_p = P.sync->prior_p[mi];
  const float prior_2p = P.sync->prior_2p[mi];
  __syncthreads();  // hbar initialised before anyone waits on it
  if (!mbar_wait_bounded(hbar, 0u, kWaitBudget) && lane == 0) record_error(&P.sync->status, FH_ERR_TIMEOUT);
  float hnorm;
  {
    // widen h in place (d <= 4 * kThreads: one round, every chunk read before any is written)
    float hv[8];
    float ss = 0.f;
    if (tid < d / 8) {
      const uint4 x = *reinterpret_cast<const uint4*>(hraw + 8 * tid);
      hv[0] = bf16lo(x.x); hv[1] = bf16hi(x.x); hv[2] = bf16lo(x.y); hv[3] = bf16hi(x.y);
      hv[4] = bf16lo(x.z); hv[5] = bf16hi(x.z); hv[6] = bf16lo(x.w); hv[7] = bf16hi(x.w);
#pragma unroll
      for (int i = 0; i < 8; ++i) ss = fmaf(hv[i], hv[i], ss);
    }
    ss = warp_sum(ss);
    if (lane == 0) misc->scan[warp] = ss;
    __syncthreads();
    if (tid < d / 8) {
      reinterpret_cast<float4*>(hs)[2 * tid] = make_float4(hv[0], hv[1], hv[2], hv[3]);
      reinterpret_cast<float4*>(hs)[2 * tid + 1] = make_float4(hv[4], hv[5], hv[6], hv[7]);
    }
    float tot = 0.f;
#pragma unroll
    for (int i = 0; i < kWarps; ++i) tot += misc->scan[i];
    hnorm = sqrtf(tot);
    __syncthreads();
  }
  // the predicted region [L, U): from the last call's rank-2p key up to its
  // rank-p key plus twice their distance (identical arithmetic in every CTA)
  const float unit = gumbel ? 1.f : hnorm;
  float L = 0.f, S = 0.f;
  bool region = prior_ok != 0u && unit > 0.f;
  if (region) {
    const float kp = prior_p * unit, k2 = prior_2p * unit;
    float span = 3.f * (kp - k2);
    if (!(span > 0.f)) span = fmaxf(fabsf(kp), 1e-30f) * 0.25f;
    L = k2;
    S = static_cast<float>(kB1Bins) / span;
    region = fabsf(L) < 3.0e38f && S > 0.f && S < 3.0e38f;
  }
  for (int i = 0; i < n1; ++i) {
    const int k = cw + i * cstride;
    float s;
    if (i == 1) {  // the row that landed in the slot
      if (!mbar_wait_bounded(wbar, wphase, kWaitBudget) && lane == 0) record_error(&P.sync->status, FH_ERR_TIMEOUT);
      wphase ^= 1u;
      if constexpr (INT4) s = srow_dot_int4_hs<NCH>(slot, hs, d);
      else if constexpr (INT8) s = srow_dot_int8_hs<NCH>(slot, hs, d);
      else s = srow_dot_bf16_hs<NCH>(slot, hs, d);
    } else if constexpr (INT4) {
      if (i > 0) row_load_int4<NCH>(P.Crows + static_cast<size_t>(k) * P.crow_bytes, d, q, sc);
      s = row_dot_int4_hs<NCH>(q, sc, hs, d);
    } else if constexpr (INT8) {
      if (i > 0) row_load_int8<NCH>(P.Crows + static_cast<size_t>(k) * P.crow_bytes, d, q8, sw8);
      s = row_dot_int8_hs<NCH>(q8, sw8, hs, d);
    } else {
      if (i > 0) row_load_bf16<NCH>(reinterpret_cast<const uint16_t*>(P.Crows + static_cast<size_t>(k) * P.crow_bytes), d, w);
      s = row_dot_bf16_hs<NCH>(w, hs, d);
    }
    const float u = __shfl_sync(0xFFFFFFFFu, ureg, i & 31);
    const float key = gumbel ? gumbel_key(s, P.T, u) : s;
    if (lane == 0) {
      const uint32_t kk = f2key(key);
      P.keys[k] = kk;
      const int bn = region ? region_bin(key, L, S) : -1;
      if (bn >= 0) {
        red_relaxed_add_u32(P.hist + bn, 1u);
        // in the region's upper half, i.e. above the predicted rank-p key by half
        // the predicted gap to rank 2p: almost surely chosen, so its token rows
        // start towards L2 now (the post-barrier prefetch covers the rest)
        if (bn >= kB1Bins / 2 && k < P.c)
          bulk_prefetch_l2(P.Ecm + static_cast<size_t>(k) * P.b * P.d, static_cast<uint32_t>(P.b * P.d * 2));
        const uint32_t at = atomicAdd(&misc->nnote, 1u);
        if (at < static_cast<uint32_t>(kNoteMax)) {
          misc->note_k[at] = k;
          misc->note_key[at] = kk;
        }
      }
    }
  }
  __syncthreads();
  // append this CTA's region keys to the candidate list
  const int nnote = min(static_cast<int>(misc->nnote), kNoteMax);
  if (tid == 0)
    misc->base = nnote ? static_cast<uint32_t>(atomicAdd(&P.hot->arrive_list, static_cast<unsigned long long>(nnote)))
                       : 0u;
  __syncthreads();
  for (int i = tid; i < nnote; i += kThreads) {
    const uint32_t at = misc->base + static_cast<uint32_t>(i);
    if (at < static_cast<uint32_t>(P.list_cap)) {
      P.list_key[at] = misc->note_key[i];
      P.list_id[at] = misc->note_k[i];
    }
  }
  __syncthreads();
  if (tid == 0) {
    red_release_add_u64(&P.hot->arrive_list, 1ull << 32);  // keys, counts and list entries of this CTA are published
    // wait (bounded, with backoff) until every CTA has arrived
    int okw = 1;
    const long long t0 = clock64();
    unsigned long long av;
    while (((av = ld_acquire_u64(&P.hot->arrive_list)) >> 32) < static_cast<unsigned long long>(G)) {
      __nanosleep(32);
      if (clock64() - t0 > P.spin_budget) {
        okw = 0;
        break;
      }
    }
    misc->claim = okw;
    misc->nlist = static_cast<uint32_t>(av);
  }
  __syncthreads();
  bool ok = misc->claim != 0;

  // ---------------- phase 2: the boundary of the top p ----------------
  // scratch (the slot area): the list's keys and ids, or all c keys; then the selection state
  const int p = P.p, c = P.c;
  const int r_2p = min(c, 2 * p);
  uint32_t* skey = reinterpret_cast<uint32_t*>(slots);
  int32_t* sid = reinterpret_cast<int32_t*>(slots + up128(static_cast<size_t>(P.list_cap) * 4));
  const uint32_t nlist = misc->nlist;
  const bool use_list = region && nlist >= static_cast<uint32_t>(p) && nlist <= static_cast<uint32_t>(P.list_cap);
  const int nl = use_list ? static_cast<int>(nlist) : 0;
  const uint32_t bs_off =
      static_cast<uint32_t>(P.off_slots) +
      static_cast<uint32_t>(std::max(2 * up128(static_cast<size_t>(P.list_cap) * 4), up128(static_cast<size_t>(c) * 4)));
  BoundSmem& bs = *reinterpret_cast<BoundSmem*>(smem + bs_off);
  bool full = true;
  if (tid == 0) {
    misc->total = nlist;
    misc->t2 = 0xFFFFFFFFu;
  }
  if (ok) {
    if (use_list) {
      const uint4 hq = __ldcg(reinterpret_cast<const uint4*>(P.hist) + (kB1Bins / 4 - 1 - tid));
      for (int i = tid; i < nl; i += kThreads) {
        skey[i] = __ldcg(P.list_key + i);
        sid[i] = __ldcg(P.list_id + i);
      }
      // bins from the top: thread t owns kB1Bins-1-4t (first) .. kB1Bins-4-4t
      const uint32_t hv[4] = {hq.w, hq.z, hq.y, hq.x};
      uint32_t total;
      uint32_t run = block_scan_excl_u32(hv[0] + hv[1] + hv[2] + hv[3], misc->uscan, &total);
      if (tid == 0) {
        misc->total = total;
        misc->m1 = 0xFFFFFFFFu;
        misc->t2 = 0xFFFFFFFFu;
        bs.nc = 0u;
      }
      __syncthreads();
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t bin = static_cast<uint32_t>(kB1Bins - 1 - 4 * tid - j);
        if (run < static_cast<uint32_t>(p) && run + hv[j] >= static_cast<uint32_t>(p)) {
          misc->t1 = bin;
          misc->above = run;
          misc->m1 = hv[j];
        }
        if (run < static_cast<uint32_t>(r_2p) && run + hv[j] >= static_cast<uint32_t>(r_2p)) misc->t2 = bin;
        run += hv[j];
      }
      __syncthreads();
      // the list holds every key the histogram counted; a crowded boundary bin takes the general path
      full = misc->m1 > static_cast<uint32_t>(kBoundEntries) || misc->total != nlist;
      if (!full) {
        // the clusters above the boundary bin are certain: start reading their
        // token rows into L2 now, under the rest of the selection
        const int t1 = static_cast<int>(misc->t1);
        for (int i = static_cast<int>(blockIdx.x) + G * tid; i < nl; i += G * kThreads) {
          const int k = sid[i];
          if (k >= 0 && k < c && region_bin(key2f(skey[i]), L, S) > t1)
            bulk_prefetch_l2(P.Ecm + static_cast<size_t>(k) * b * d, static_cast<uint32_t>(b * d * 2));
        }
      }
      if (!full) {
        // gather the boundary bin's entries (their bins agree with phase 1), rank them exactly
        const int t1 = static_cast<int>(misc->t1);
        for (int i = tid; i < nl; i += kThreads) {
          const uint32_t kk = skey[i];
          if (region_bin(key2f(kk), L, S) == t1) {
            const uint32_t at = atomicAdd(&bs.nc, 1u);
            if (at < static_cast<uint32_t>(kBoundEntries)) {
              bs.ckey[at] = kk;
              bs.cid[at] = sid[i];
            }
          }
        }
        __syncthreads();
        const uint32_t m1 = min(bs.nc, static_cast<uint32_t>(kBoundEntries));  // == misc->m1
        const uint32_t need = static_cast<uint32_t>(p) - misc->above;
        for (uint32_t a = tid; a < m1; a += kThreads) {
          const uint32_t ka = bs.ckey[a];
          const int32_t ia = bs.cid[a];
          uint32_t r = 0;
          for (uint32_t bb = 0; bb < m1; ++bb) {
            const uint32_t kb = bs.ckey[bb];
            r += (kb > ka || (kb == ka && bs.cid[bb] < ia)) ? 1u : 0u;
          }
          if (r + 1u == need) {
            misc->bkey = ka;
            misc->bid = ia;
          }
        }
        if (tid == 0) {
          misc->edge_2p = misc->t2 != 0xFFFFFFFFu ? L + static_cast<float>(misc->t2) / S
                                                  : __int_as_float(0x7FC00000);
          if (m1 != misc->m1) misc->m1 = 0xFFFFFFFFu;  // inconsistent counts: take the general path
        }
        __syncthreads();
        full = misc->m1 == 0xFFFFFFFFu;
      }
    }
    if (full) {
      // the general exact selector over all c keys
      __syncthreads();  // every thread is done with the list scratch before the keys overwrite it
      for (int i = tid; i < c / 4; i += kThreads)
        reinterpret_cast<uint4*>(skey)[i] = __ldcg(reinterpret_cast<const uint4*>(P.keys) + i);
      for (int i = (c / 4) * 4 + tid; i < c; i += kThreads) skey[i] = __ldcg(P.keys + i);
      __syncthreads();
      select_boundary(c, p, p, r_2p, static_cast<uint32_t>(P.off_slots), kImplicitIds, bs_off);
      if (bs.heavy) {
        // heavy ties: radix select (ties to the lower id) into ssel, then its worst entry
        __syncthreads();
        SelectSmem& rs = *reinterpret_cast<SelectSmem*>(smem + bs_off);
        block_select_top_p(skey, c, p, ssel, rs);
        unsigned long long worst = ~0ull;
        for (int i = tid; i < p; i += kThreads) {
          const int k = ssel[i];
          const unsigned long long cmp = (static_cast<unsigned long long>(skey[k]) << 32) |
                                         static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<uint32_t>(k));
          worst = cmp < worst ? cmp : worst;
        }
        for (int o = 16; o > 0; o >>= 1) {
          const unsigned long long y = __shfl_xor_sync(0xFFFFFFFFu, worst, o);
          worst = y < worst ? y : worst;
        }
        if (lane == 0) misc->wbest[warp] = worst;
        __syncthreads();
        if (tid == 0) {
          unsigned long long m = ~0ull;
          for (int i = 0; i < kWarps; ++i) m = misc->wbest[i] < m ? misc->wbest[i] : m;
          misc->bkey = static_cast<uint32_t>(m >> 32);
          misc->bid = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(m & 0xFFFFFFFFull));
          misc->edge_2p = __int_as_float(0x7FC00000);
        }
      } else if (tid == 0) {
        misc->bkey = bs.bkey;
        misc->bid = bs.bid;
        misc->edge_2p = bs.edge_b;
      }
      __syncthreads();
    }
    if (tid == 0) misc->full = full;
    // the chosen clusters in row order (list order, or ascending ids): warp w
    // owns entries [w * span, w * span + span), 32 consecutive per step (one per
    // lane: no bank conflicts), one ballot each
    const uint32_t bkey = misc->bkey;
    const int32_t bid = misc->bid;
    const int n = full ? c : nl;
    const int wspan = ((n + kWarps - 1) / kWarps + 31) & ~31;
    const int w0 = min(n, warp * wspan), w1 = min(n, w0 + wspan);
    uint32_t cnt = 0;
    for (int base = w0; base < w1; base += 32) {
      const int i = base + lane;
      const bool ch = i < w1 && chosen(skey[i], full ? i : sid[i], bkey, bid);
      cnt += __popc(__ballot_sync(0xFFFFFFFFu, ch));
    }
    if (lane == 0) misc->uscan[warp] = cnt;
    __syncthreads();
    uint32_t pos = 0;
    for (int i = 0; i < warp; ++i) pos += misc->uscan[i];
    const uint32_t lt = (1u << lane) - 1u;
    for (int base = w0; base < w1; base += 32) {
      const int i = base + lane;
      const int32_t k = i < w1 ? (full ? i : sid[i]) : 0;
      const bool ch = i < w1 && chosen(skey[i], k, bkey, bid);
      const uint32_t m = __ballot_sync(0xFFFFFFFFu, ch);
      const uint32_t at = pos + __popc(m & lt);
      if (ch && at < static_cast<uint32_t>(p)) ssel[at] = k;
      pos += __popc(m);
    }
    fence_proxy_async_smem();  // the slots were generic scratch; bulk copies follow
    __syncthreads();
  }

  // ---------------- phase 3: candidate rows ----------------
  // row r is slot r % b of the (r / b)-th chosen cluster; rows
  // blockIdx + G * warp + 16 G i belong to this warp, two at a time
  unsigned long long best = 0ull;
  const int r_all = p * b;
  for (int r0 = cw; ok && r0 < r_all; r0 += 2 * cstride) {
    const int r1 = r0 + cstride;
    const bool two = r1 < r_all;
    // the rows sit at k*b + j of the cluster-major copy: their loads do not wait for C2T,
    // whose entries (the token ids of the output) are read alongside
    const int k0 = ssel[r0 / b], k1 = two ? ssel[r1 / b] : k0;
    if (k0 < 0 || k0 >= c || k1 < 0 || k1 >= c) {  // only an inconsistent selection; never read outside E
      ok = false;
      break;
    }
    const size_t q0 = static_cast<size_t>(k0) * b + r0 % b, q1 = static_cast<size_t>(k1) * b + r1 % b;
    if (two && lane == 0) {
      mbar_expect_tx(wbar, static_cast<uint32_t>(d * 2));
      bulk_g2s(slot, P.Ecm + q1 * d, static_cast<uint32_t>(d * 2), wbar);
    }
    uint4 e[NCH];
    row_load_bf16<NCH>(P.Ecm + q0 * d, d, e);
    int t = 0;
    if (lane == 0) t = P.C2T.at(q0);
    else if (lane == 1 && two) t = P.C2T.at(q1);
    const int t0 = __shfl_sync(0xFFFFFFFFu, t, 0);
    const int t1 = two ? __shfl_sync(0xFFFFFFFFu, t, 1) : 0;
    const float z0 = row_dot_bf16_hs<NCH>(e, hs, d);
    unsigned long long pk = pack_best(z0, t0);
    best = pk > best ? pk : best;
    if (gumbel && lane == 0) P.z_buf[static_cast<size_t>(ssel[r0 / b]) * b + r0 % b] = z0;
    if (two) {
      const bool got = mbar_wait_bounded(wbar, wphase, kWaitBudget);
      wphase ^= 1u;
      if (!__all_sync(0xFFFFFFFFu, got)) {
        mbar_wait_bounded(wbar, wphase ^ 1u, kWaitBudget);  // drain before the slot is released
        ok = false;
        break;
      }
      const float z1 = srow_dot_bf16_hs<NCH>(slot, hs, d);
      pk = pack_best(z1, t1);
      best = pk > best ? pk : best;
      if (gumbel && lane == 0) P.z_buf[static_cast<size_t>(ssel[r1 / b]) * b + r1 % b] = z1;
      __syncwarp();
      if (lane == 0) fence_proxy_async_smem();
    }
  }
  if (!ok && lane == 0) record_error(&P.sync->status, FH_ERR_TIMEOUT);
  best = warp_max_u64(best);
  if (lane == 0) misc->wbest[warp] = best;
  __syncthreads();

  // ---------------- exit: the last CTA writes the token ----------------
  if (tid == 0) {
    unsigned long long m = 0ull;
    for (int i = 0; i < kWarps; ++i) m = misc->wbest[i] > m ? misc->wbest[i] : m;
    if (m) atomicMax(&P.hot->best, m);
    // acq_rel: this CTA's maximum and logits are published; the last CTA sees everyone's
    misc->last = atom_acq_rel_add_u32(&P.hot->ticket, 1u) == static_cast<uint32_t>(G - 1);
  }
  __syncthreads();
  if (!misc->last) return;

  const unsigned long long bw = __ldcg(&P.hot->best);
  if (tid == 0) {
    if (!gumbel) P.out_tokens[0] = best_token(bw);
    if (P.out_max_logit) P.out_max_logit[0] = best_logit(bw);
  }
  if (ok && (gumbel || P.out_cluster_ids) && !misc->full) {
    // list order -> ascending ids (canonical order): membership bitmap over the c ids, then a scan
    const int words = (c + 31) >> 5;
    uint32_t* bits = reinterpret_cast<uint32_t*>(slots);
    for (int i = tid; i < words; i += kThreads) bits[i] = 0u;
    __syncthreads();
    for (int i = tid; i < p; i += kThreads) atomicOr(&bits[ssel[i] >> 5], 1u << (ssel[i] & 31));
    __syncthreads();
    const int wpt = (words + kThreads - 1) / kThreads;
    const int v0 = min(words, tid * wpt), v1 = min(words, v0 + wpt);
    uint32_t cnt = 0;
    for (int wi = v0; wi < v1; ++wi) cnt += __popc(bits[wi]);
    uint32_t pos = block_scan_excl_u32(cnt, misc->uscan, nullptr);
    __syncthreads();  // every ssel entry is in the bitmap before any is overwritten
    for (int wi = v0; wi < v1; ++wi)
      for (uint32_t m = bits[wi]; m; m &= m - 1u) {
        if (pos < static_cast<uint32_t>(p)) ssel[pos] = wi * 32 + __ffs(m) - 1;
        ++pos;
      }
    __syncthreads();
  }
  if (ok && P.out_cluster_ids)
    for (int i = tid; i < p; i += kThreads) P.out_cluster_ids[i] = ssel[i];
  if (ok && gumbel) {
    // inverse CDF over softmax(z/T) in canonical order (cluster asc, slot asc)
    auto zc = [&](int i) -> float { return __ldcg(P.z_buf + static_cast<size_t>(ssel[i / b]) * b + i % b); };
    const float ym = best_logit(bw) / P.T;
    const int qn = (r_all + kThreads - 1) / kThreads;
    const int i0 = min(r_all, tid * qn), i1 = min(r_all, i0 + qn);
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
      const float wgt = expf(zc(i) / P.T - ym);
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
      P.out_tokens[0] = P.C2T.at(static_cast<size_t>(ssel[idx / b]) * b + idx % b);
    }
  }
  // clear the histogram for the next call (every CTA has read it)
  if (region) reinterpret_cast<uint4*>(P.hist)[tid] = make_uint4(0, 0, 0, 0);
  if (tid == 0) {
    // this call's keys of rank p and 2p for the next call; past the region's
    // count the rank-2p key is extrapolated linearly from the region's edge
    if (ok) {
      const float kp = key2f(misc->bkey);
      float k2 = misc->edge_2p;
      if (!misc->full && misc->t2 == 0xFFFFFFFFu) {
        const float tot = static_cast<float>(misc->total);
        k2 = L - (kp - L) * (static_cast<float>(r_2p) - tot) / fmaxf(1.f, tot - static_cast<float>(p));
      }
      const float pp = kp / unit, p2 = fminf(k2, kp) / unit;
      if (pp == pp && p2 == p2 && fabsf(pp) < 3.0e38f && fabsf(p2) < 3.0e38f && unit > 0.f) {
        P.sync->prior_p[mi] = pp;
        P.sync->prior_2p[mi] = p2;
        P.sync->prior_ok[mi] = 1u;
      }
      P.sync->last_in_range = region ? misc->total : 0u;
      P.sync->last_full = misc->full;
    }
    P.hot->best = 0ull;
    P.hot->arrive_list = 0ull;
    P.hot->ticket = 0u;
    red_relaxed_add_u32(&P.sync->epoch, 1u);  // a count of calls; nothing waits for it
  }
}

template <int NCH>
cudaError_t launch_nch(const B1Params& P, int grid, size_t smem, int cfmt, cudaStream_t st) {
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
  if (cfmt == kFmtInt4) return cudaLaunchKernelEx(&cfg, decode_b1_kernel<NCH, kFmtInt4>, P);
  if (cfmt == kFmtInt8) return cudaLaunchKernelEx(&cfg, decode_b1_kernel<NCH, kFmtInt8>, P);
  return cudaLaunchKernelEx(&cfg, decode_b1_kernel<NCH, kFmtBf16>, P);
}

}  // namespace

size_t decode_b1_misc_bytes() { return sizeof(B1Misc); }

// Scratch of the selection phase (in the slot area): the candidate list's
// keys and ids, or all c keys, then the selection's shared state.
size_t decode_b1_scratch_bytes(int c, int list_cap) {
  auto r128 = [](size_t x) { return (x + 127) & ~size_t(127); };
  const size_t keys = std::max(2 * r128(static_cast<size_t>(list_cap) * 4), r128(static_cast<size_t>(c) * 4));
  return keys + std::max(sizeof(BoundSmem), sizeof(SelectSmem));
}


cudaError_t launch_decode_b1(const B1Params& P, int grid, size_t smem, int cfmt, int nch, cudaStream_t st) {
  switch (nch) {
    case 1: return launch_nch<1>(P, grid, smem, cfmt, st);
    case 2: return launch_nch<2>(P, grid, smem, cfmt, st);
    case 3: return launch_nch<3>(P, grid, smem, cfmt, st);
    case 4: return launch_nch<4>(P, grid, smem, cfmt, st);
    case 5: return launch_nch<5>(P, grid, smem, cfmt, st);
    case 6: return launch_nch<6>(P, grid, smem, cfmt, st);
    case 8: return launch_nch<8>(P, grid, smem, cfmt, st);
    case 10: return launch_nch<10>(P, grid, smem, cfmt, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t occupancy_decode_b1(int cfmt, int nch, size_t smem, int* blocks) {
#define FH_O(N)                                                                                           \
  return cfmt == kFmtInt4                                                                                 \
             ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks, decode_b1_kernel<N, kFmtInt4>, kThreads, smem) \
         : cfmt == kFmtInt8                                                                               \
             ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks, decode_b1_kernel<N, kFmtInt8>, kThreads, smem) \
             : cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks, decode_b1_kernel<N, kFmtBf16>, kThreads, smem);
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
    e = cudaFuncSetAttribute(decode_b1_kernel<N, kFmtBf16>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem); \
  if (e == cudaSuccess)                                                                                   \
    e = cudaFuncSetAttribute(decode_b1_kernel<N, kFmtInt4>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem); \
  if (e == cudaSuccess)                                                                                   \
    e = cudaFuncSetAttribute(decode_b1_kernel<N, kFmtInt8>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
  FH_SET(1) FH_SET(2) FH_SET(3) FH_SET(4) FH_SET(5) FH_SET(6) FH_SET(8) FH_SET(10)
#undef FH_SET
  return e;
}

}  // namespace fh
