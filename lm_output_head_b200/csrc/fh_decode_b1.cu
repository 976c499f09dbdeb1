// Fused FlashHead decode for one hidden state (B = 1), one persistent
// cooperative launch of one 512-thread CTA per SM.
//
// The pages' pipeline (FlashHead write-up, section 2.2.2: h -> centroid_scores
// -> top_p_clusters -> token_scores) runs as three phases of one kernel:
//
//  1. centroid scores (section 1.2.2; INT4 centroids per section 1.2.4): the
//     c centroid rows are spread round-robin over every warp of the grid;
//     each warp streams its rows HBM -> shared memory with cp.async.bulk into
//     a private ring of slots, dots them with h held in registers, and
//     writes the score (or, when sampling, the Gumbel key s/T - ln(-ln u),
//     section 1.2.3) to the workspace;
//  2. one device-wide barrier (bounded spin), then every CTA reads all c
//     keys back from L2 and runs the same block radix select, so each CTA
//     knows the same p clusters in ascending id order without a second
//     barrier;
//  3. the p*b candidate slots (slot q*b + j = token C2T[sel_q][j], the slot
//     arithmetic of section 1.2.1) are spread over every warp; each streams
//     its E rows, dots them with h and keeps a packed (logit, token) max;
//     the CTA maxima meet in one 64-bit atomicMax. The last CTA to finish
//     (exit ticket) writes the token: the argmax, or, when sampling, the
//     inverse-CDF draw over softmax(z/T) in canonical candidate order.
//
// HBM traffic is the algorithmic minimum: each centroid row once, each
// selected token row once, plus the C2T rows and h.
#include <climits>

#include "fh_device.cuh"

namespace fh {
namespace {

struct B1Misc {
  unsigned long long hbar;
  unsigned long long wbest[kWarps];
  float scan[kWarps + 1];
  int claim, lastpos, ok, last;
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
  // histogram of this call's keys, and the other buffer to clear for the next call
  const uint32_t epoch = P.sync->epoch;
  uint32_t* hist_cur = P.ghist + (epoch & 1u) * kHistBins;
  uint32_t* hist_next = P.ghist + ((epoch + 1u) & 1u) * kHistBins;

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
  const int n1 = gw < P.c ? (P.c - 1 - gw) / W + 1 : 0;
  auto src1 = [&](int i, const void*& ptr, uint32_t& bytes) {
    ptr = P.Crows + static_cast<size_t>(gw + i * W) * P.crow_bytes;
    bytes = static_cast<uint32_t>(P.crow_bytes);
  };
  warp_stream_prologue(n1, P.nslot, ring_w, P.slot_bytes, bar_w, src1);
  float ureg = 0.f;  // lane j holds u of item j (j < 32)
  if (gumbel && lane < n1) ureg = __ldg(P.u_clusters + gw + lane * W);
  {
    const int per = (kHistBins + G - 1) / G;
    for (int i = tid; i < per; i += kThreads) {
      const int b = blockIdx.x * per + i;
      if (b < kHistBins) hist_next[b] = 0u;
    }
  }
  __syncthreads();  // hbar initialised before anyone waits on it
  if (!mbar_wait_bounded(hbar, 0u, kWaitBudget)) {
    ok = false;
    if (lane == 0) record_error(&P.sync->status, FH_ERR_TIMEOUT);
  }
  {
    if constexpr (INT4) {
      constexpr int NQ = (NCH + 1) / 2;
      float hq[NQ * 16];
      load_h_halfgroups<NQ>(sh, d, hq);
      auto use = [&](int i, uint32_t slot) {
        const int k = gw + i * W;
        const float u = __shfl_sync(0xFFFFFFFFu, ureg, i & 31);
        const float s = row_dot_int4<NQ>(slot, d, hq);
        if (lane == 0) {
          float key = s;
          if (gumbel) key = gumbel_key(s, P.T, i < 32 ? u : __ldg(P.u_clusters + k));
          P.scores[k] = key;
          atomicAdd(hist_cur + (f2key(key) >> kHistShift), 1u);
          prefetch_l2(P.C2T + static_cast<size_t>(k) * P.b);
        }
      };
      ok = warp_stream_run(n1, P.nslot, ring_w, P.slot_bytes, bar_w, phase_bits, kWaitBudget, src1, use);
    } else {
      float hr[NCH * 8];
      load_h_chunks<NCH>(sh, d, hr);
      auto use = [&](int i, uint32_t slot) {
        const int k = gw + i * W;
        const float u = __shfl_sync(0xFFFFFFFFu, ureg, i & 31);
        const float s = row_dot_bf16<NCH>(slot, d, hr);
        if (lane == 0) {
          float key = s;
          if (gumbel) key = gumbel_key(s, P.T, i < 32 ? u : __ldg(P.u_clusters + k));
          P.scores[k] = key;
          atomicAdd(hist_cur + (f2key(key) >> kHistShift), 1u);
          prefetch_l2(P.C2T + static_cast<size_t>(k) * P.b);
        }
      };
      ok = warp_stream_run(n1, P.nslot, ring_w, P.slot_bytes, bar_w, phase_bits, kWaitBudget, src1, use);
    }
    if (!ok && lane == 0) record_error(&P.sync->status, FH_ERR_TIMEOUT);
  }

  // ---------------- phase 2: barrier + redundant top-p select ----------------
  const bool passed = grid_barrier(&P.sync->arrive, static_cast<uint32_t>(G), P.spin_budget, misc);
  if (!passed) {
    if (tid == 0) record_error(&P.sync->status, FH_ERR_TIMEOUT);
  } else {
    select_top_p_hist(P.scores, nullptr, 1.f, P.c, P.p, hist_cur, ssel, ring);
    if (blockIdx.x == 0 && P.out_cluster_ids)
      for (int i = tid; i < P.p; i += kThreads) P.out_cluster_ids[i] = ssel[i];
    fence_proxy_async_smem();  // generic writes to the ring before the next bulk copies
    __syncthreads();

    // ---------------- phase 3: gather + candidate logits ----------------
    const int nc = P.p * P.b;
    const int n3 = gw < nc ? (nc - 1 - gw) / W + 1 : 0;
    int tok0 = 0, tok1 = 0;  // lane j: token of item j and of item 32 + j
    if (lane < n3) {
      const int r = gw + lane * W;
      tok0 = __ldg(P.C2T + static_cast<size_t>(ssel[r / P.b]) * P.b + r % P.b);
    }
    if (32 + lane < n3) {
      const int r = gw + (32 + lane) * W;
      tok1 = __ldg(P.C2T + static_cast<size_t>(ssel[r / P.b]) * P.b + r % P.b);
    }
    auto token_of = [&](int i) -> int {
      const int a = __shfl_sync(0xFFFFFFFFu, tok0, i & 31);
      const int b1 = __shfl_sync(0xFFFFFFFFu, tok1, i & 31);
      if (i < 32) return a;
      if (i < 64) return b1;
      const int r = gw + i * W;
      return __ldg(P.C2T + static_cast<size_t>(ssel[r / P.b]) * P.b + r % P.b);
    };
    float hr[NCH * 8];
    load_h_chunks<NCH>(sh, d, hr);
    unsigned long long best = 0ull;
    auto src = [&](int i, const void*& ptr, uint32_t& bytes) {
      ptr = P.E + static_cast<size_t>(token_of(i)) * d;
      bytes = static_cast<uint32_t>(d * 2);
    };
    auto use = [&](int i, uint32_t slot) {
      const int t = token_of(i);
      const float z = row_dot_bf16<NCH>(slot, d, hr);
      const unsigned long long pk = pack_best(z, t);
      best = pk > best ? pk : best;
      if (gumbel && lane == 0) P.cand_logits[gw + i * W] = z;
    };
    ok = warp_stream(n3, P.nslot, ring_w, P.slot_bytes, bar_w, phase_bits, kWaitBudget, src, use);
    if (!ok && lane == 0) record_error(&P.sync->status, FH_ERR_TIMEOUT);
    if (lane == 0) misc->wbest[warp] = best;
    __syncthreads();
    if (tid == 0) {
      unsigned long long m = 0ull;
      for (int w = 0; w < kWarps; ++w) m = misc->wbest[w] > m ? misc->wbest[w] : m;
      if (m) atomicMax(P.best, m);
    }
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
  if (!gumbel || !passed) {
    if (tid == 0) {
      P.out_tokens[0] = best_token(bw);
      if (P.out_max_logit) P.out_max_logit[0] = best_logit(bw);
    }
  } else {
    // inverse CDF over softmax(z/T), canonical order (cluster asc, slot asc)
    const int nc = P.p * P.b;
    const float ym = best_logit(bw) / P.T;
    const int q = (nc + kThreads - 1) / kThreads;
    const int i0 = min(nc, tid * q), i1 = min(nc, i0 + q);
    float loc = 0.f;
    for (int i = i0; i < i1; ++i) loc += expf(__ldcg(P.cand_logits + i) / P.T - ym);
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
      const float w = expf(__ldcg(P.cand_logits + i) / P.T - ym);
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
      P.out_tokens[0] = __ldg(P.C2T + static_cast<size_t>(ssel[idx / P.b]) * P.b + idx % P.b);
      if (P.out_max_logit) P.out_max_logit[0] = best_logit(bw);
    }
  }
  if (tid == 0) {
    *P.best = 0ull;
    P.sync->arrive = 0u;
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
