// Fused FlashHead decode for one hidden state (B = 1): one persistent
// cooperative launch, two 512-thread CTAs per SM, every row streamed from
// HBM with non-allocating loads and dotted with h staged once per CTA in
// shared memory (fp32).
//
// The pages' pipeline (FlashHead write-up, section 2.2.2: h -> centroid_scores
// -> top_p_clusters -> token_scores) runs as phases of one kernel:
//
//  1. centroid scores (section 1.2.2; INT4 centroids per section 1.2.4):
//     cluster k belongs to CTA k mod G (warp (k / G) mod 16), so every CTA
//     owns c/G clusters. A warp's first row streams into registers, its
//     second into a shared-memory slot by one bulk copy, both requested at
//     kernel start. The key -- the score, or when sampling the Gumbel key
//     s/T - ln(-ln u) (section 1.2.3) -- goes to global memory.
//  2. the last CTA to finish phase 1 (one atomic ticket) becomes the
//     selector: it reads the c keys once, selects the p largest exactly
//     (key desc, id asc; histogram + exact rank of the boundary bin in shared
//     memory), publishes the chosen ids in ascending order and raises a
//     ready flag. Candidate row r is then slot r % b of the (r / b)-th chosen
//     cluster: the canonical candidate order (section 1.2.1).
//  3. one thread per CTA polls the flag with backoff; candidate row r belongs
//     to CTA r mod G, warp (r / G) mod 16, which maps it through C2T (rows
//     prefetched to L2 in phase 1), streams it (first row in registers,
//     second into its slot) and keeps a packed (logit, token) maximum
//     (section 1.2.4, stage 2).
//  4. CTA maxima meet in one 64-bit atomicMax; the last CTA to finish (exit
//     ticket) writes the token: the argmax, or, when sampling, the inverse-CDF
//     draw over softmax(z/T) walking the candidates in canonical order.
//
// Device-wide coordination is two atomic tickets and one flag; no
// device-wide barrier, no histogram atomics on hot lines, and no CTA but the
// selector reads all c keys. HBM traffic is the algorithmic
// minimum: each centroid row once, each selected token row once, plus C2T
// rows and h.
#include <climits>

#include "fh_device.cuh"

namespace fh {
namespace {

struct B1Misc {
  unsigned long long hbar;
  unsigned long long wbar[kWarps];
  unsigned long long wbest[kWarps];
  float scan[kWarps + 1];
  uint32_t uscan[kWarps + 1];
  int claim, lastpos, last, selector;
};

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
  uint8_t* slots = smem + P.off_slots;  // per-warp row slots; the selector's scratch after phase 1

  const uint32_t epoch = P.sync->epoch;  // calls on one head are stream-ordered

  // ---------------- phase 1: centroid scores ----------------
  const uint32_t hbar = smem_addr(&misc->hbar);
  const uint32_t wbar = smem_addr(&misc->wbar[warp]);
  const uint32_t slot = smem_addr(slots) + static_cast<uint32_t>(warp * P.slot_bytes);
  uint16_t* hraw = reinterpret_cast<uint16_t*>(hs + d / 2);
  if (tid == 0) {
    mbar_init(hbar, 1);
    fence_mbar_init();
    mbar_expect_tx(hbar, static_cast<uint32_t>(d * 2));
    bulk_g2s(smem_addr(hraw), P.hidden, static_cast<uint32_t>(d * 2), hbar);
  }
  const int cw = static_cast<int>(blockIdx.x) + G * warp;  // first cluster of this warp
  const int cstride = G * kWarps;
  const int n1 = cw < P.c ? (P.c - 1 - cw) / cstride + 1 : 0;  // <= 32 (host-checked)
  uint32_t wphase = 0;  // parity of this warp's slot barrier
  if (lane == 0) {
    mbar_init(wbar, 1);
    fence_mbar_init();
    if (n1 >= 2) {
      mbar_expect_tx(wbar, static_cast<uint32_t>(P.crow_bytes));
      bulk_g2s(slot, P.Crows + static_cast<size_t>(cw + cstride) * P.crow_bytes, static_cast<uint32_t>(P.crow_bytes),
               wbar);
    }
  }
  constexpr int NQ = (NCH + 1) / 2;
  uint4 w[NCH];
  uint2 q[NQ];
  uint32_t sc[NQ];
  if (n1 > 0) {
    if constexpr (INT4) row_load_int4<NQ>(P.Crows + static_cast<size_t>(cw) * P.crow_bytes, d, q, sc);
    else row_load_bf16<NCH>(reinterpret_cast<const uint16_t*>(P.Crows + static_cast<size_t>(cw) * P.crow_bytes), d, w);
  }
  float ureg = 0.f;  // lane j holds u of item j
  if (gumbel && lane < n1) ureg = __ldg(P.u_clusters + cw + lane * cstride);
  if (lane < n1) prefetch_l2(P.C2T + static_cast<size_t>(cw + lane * cstride) * b);  // read in phase 3 if chosen
  __syncthreads();  // hbar initialised before anyone waits on it
  if (!mbar_wait_bounded(hbar, 0u, kWaitBudget) && lane == 0) record_error(&P.sync->status, FH_ERR_TIMEOUT);
  {
    // widen h in place (d <= 4 * kThreads: one round, every chunk read before any is written)
    float hv[8];
    if (tid < d / 8) {
      const uint4 x = *reinterpret_cast<const uint4*>(hraw + 8 * tid);
      hv[0] = bf16lo(x.x); hv[1] = bf16hi(x.x); hv[2] = bf16lo(x.y); hv[3] = bf16hi(x.y);
      hv[4] = bf16lo(x.z); hv[5] = bf16hi(x.z); hv[6] = bf16lo(x.w); hv[7] = bf16hi(x.w);
    }
    __syncthreads();
    if (tid < d / 8) {
      reinterpret_cast<float4*>(hs)[2 * tid] = make_float4(hv[0], hv[1], hv[2], hv[3]);
      reinterpret_cast<float4*>(hs)[2 * tid + 1] = make_float4(hv[4], hv[5], hv[6], hv[7]);
    }
    __syncthreads();
  }
  for (int i = 0; i < n1; ++i) {
    const int k = cw + i * cstride;
    float s;
    if (i == 1) {  // the row that landed in the slot
      if (!mbar_wait_bounded(wbar, wphase, kWaitBudget) && lane == 0) record_error(&P.sync->status, FH_ERR_TIMEOUT);
      wphase ^= 1u;
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
    if (lane == 0) P.keys[k] = f2key(key);
  }

  // ---------------- phase 2: the last CTA to finish selects ----------------
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    misc->selector = atomicAdd(&P.sync->arrive, 1u) == static_cast<uint32_t>(G - 1);
  }
  __syncthreads();
  const int r_all = P.p * b;
  if (misc->selector) {
    __threadfence();
    if (P.c <= kThreads * 16) {
      select_reg<16>(P.keys, P.c, P.p, P.off_sel, P.off_slots);
    } else if (P.c <= kThreads * 32) {
      select_reg<32>(P.keys, P.c, P.p, P.off_sel, P.off_slots);
    } else {
      select_stage_gkeys(P.keys, P.c, slots);
      select_top_p_staged(P.c, P.p, P.off_sel, P.off_slots);
    }
    for (int i = tid; i < P.p; i += kThreads) {
      P.sel_list[i] = ssel[i];
      if (P.out_cluster_ids) P.out_cluster_ids[i] = ssel[i];
    }
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      st_release_u32(&P.sync->ready, epoch + 1u);  // the selection of this call is published
    }
    fence_proxy_async_smem();  // the slots were generic scratch; bulk copies follow
  } else {
    // one thread per CTA waits (bounded, with backoff) for the selector's flag
    if (tid == 0) {
      int okw = 1;
      const long long t0 = clock64();
      while (ld_acquire_u32(&P.sync->ready) != epoch + 1u) {
        __nanosleep(200);
        if (clock64() - t0 > P.spin_budget) {
          okw = 0;
          break;
        }
      }
      misc->claim = okw;
    }
  }
  __syncthreads();
  const bool sel_ok = misc->selector || misc->claim;

  // ---------------- phase 3: candidate rows ----------------
  // rows r0 = blockIdx + G * warp, r0 + 16 G, ...: two at a time are polled
  // together and streamed together (registers, slot).
  unsigned long long best = 0ull;
  bool ok = true;
  if (!sel_ok) ok = false;
  for (int r0 = cw; sel_ok && r0 < r_all; r0 += 2 * cstride) {
    const int r1 = r0 + cstride;
    const bool two = r1 < r_all;
    // candidate row r is slot r % b of the (r / b)-th chosen cluster (canonical order)
    int t = 0;
    if (lane == 0 || (lane == 1 && two)) {
      const int r = lane == 0 ? r0 : r1;
      const int k = __ldcg(P.sel_list + r / b);
      t = (k >= 0 && k < P.c) ? __ldg(P.C2T + static_cast<size_t>(k) * b + r % b) : -1;
    }
    const int t0 = __shfl_sync(0xFFFFFFFFu, t, 0);
    const int t1 = two ? __shfl_sync(0xFFFFFFFFu, t, 1) : 0;
    if (t0 < 0 || t1 < 0) {  // only an inconsistent selection; never read outside E
      ok = false;
      break;
    }
    if (two && lane == 0) {
      fence_proxy_async_smem();
      mbar_expect_tx(wbar, static_cast<uint32_t>(d * 2));
      bulk_g2s(slot, P.E + static_cast<size_t>(t1) * d, static_cast<uint32_t>(d * 2), wbar);
    }
    uint4 e[NCH];
    row_load_bf16<NCH>(P.E + static_cast<size_t>(t0) * d, d, e);
    const float z0 = row_dot_bf16_hs<NCH>(e, hs, d);
    unsigned long long pk = pack_best(z0, t0);
    best = pk > best ? pk : best;
    if (gumbel && lane == 0) P.z_row[r0] = z0;
    if (two) {
      if (!mbar_wait_bounded(wbar, wphase, kWaitBudget)) ok = false;
      wphase ^= 1u;
      const float z1 = srow_dot_bf16_hs<NCH>(slot, hs, d);
      pk = pack_best(z1, t1);
      best = pk > best ? pk : best;
      if (gumbel && lane == 0) P.z_row[r1] = z1;
      __syncwarp();
    }
  }
  if (!ok && lane == 0) record_error(&P.sync->status, FH_ERR_TIMEOUT);
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
    const uint32_t tk = atomicAdd(&P.sync->ticket, 1u);
    misc->last = (tk == static_cast<uint32_t>(G - 1));
  }
  __syncthreads();
  if (!misc->last) return;
  __threadfence();

  const unsigned long long bw = *reinterpret_cast<volatile unsigned long long*>(P.best);
  if (!gumbel) {
    if (tid == 0) {
      P.out_tokens[0] = best_token(bw);
      if (P.out_max_logit) P.out_max_logit[0] = best_logit(bw);
    }
  } else {
    // inverse CDF over softmax(z/T) in canonical order (cluster asc, slot asc)
    const float ym = best_logit(bw) / P.T;
    const int qn = (r_all + kThreads - 1) / kThreads;
    const int i0 = min(r_all, tid * qn), i1 = min(r_all, i0 + qn);
    float loc = 0.f;
    for (int i = i0; i < i1; ++i) loc += expf(__ldcg(P.z_row + i) / P.T - ym);
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
      const float wgt = expf(__ldcg(P.z_row + i) / P.T - ym);
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
      P.out_tokens[0] = __ldg(P.C2T + static_cast<size_t>(__ldcg(P.sel_list + idx / b)) * b + idx % b);
      if (P.out_max_logit) P.out_max_logit[0] = best_logit(bw);
    }
  }
  if (tid == 0) {
    *P.best = 0ull;
    P.sync->arrive = 0u;
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
