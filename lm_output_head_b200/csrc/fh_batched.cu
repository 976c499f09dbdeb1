// FlashHead for a batch of hidden states (B > 1), and the stage-by-stage
// entry points. Stages (FlashHead write-up, section 2.2.2):
//
//  scores_kernel      stage 1, s = C h for a block of rows (section 1.2.2),
//                     optionally turned into Gumbel keys s/T - ln(-ln u)
//                     (section 1.2.3). Every centroid row is streamed from HBM
//                     once per launch and dotted with all rows held in smem.
//  select_kernel      per-row top-p of the keys (block radix select), ids in
//                     ascending order, plus the candidate token list of the
//                     row in canonical order through C2T (section 1.2.1).
//  sort_ids_kernel    the same candidate list for caller-given cluster ids
//                     (validated: in range and distinct).
//  candidates_kernel  stage 2, z_t = E_t . h for every candidate (section
//                     1.2.4), streaming E rows through per-warp smem rings,
//                     with a packed per-row (logit, token) max.
//  epilogue_kernel    per row: argmax token, or the inverse-CDF draw from
//                     softmax(z/T) in canonical order (section 1.2.3).
#include <climits>

#include "fh_device.cuh"

namespace fh {
namespace {

// ----------------------------------------------------------------------------
// stage 1 for a block of rows
// ----------------------------------------------------------------------------
template <int NCH, int FMT>
__global__ void __launch_bounds__(kThreads, 1) scores_kernel(const ScoresParams P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int W = gridDim.x * kWarps, gw = blockIdx.x * kWarps + warp;
  const int d = P.d, R = P.rows;
  uint16_t* sh = reinterpret_cast<uint16_t*>(smem + P.off_h);
  const uint32_t sh_a = smem_addr(sh);
  const uint32_t ring_w = smem_addr(smem + P.off_ring) + static_cast<uint32_t>(warp * P.nslot * P.slot_bytes);
  const uint32_t bar_w = smem_addr(smem + P.off_bar) + static_cast<uint32_t>(warp * P.nslot * 8);

  const uint4* hsrc = reinterpret_cast<const uint4*>(P.hidden + static_cast<size_t>(P.row0) * d);
  for (int i = tid; i < R * d / 8; i += kThreads) reinterpret_cast<uint4*>(sh)[i] = hsrc[i];
  warp_ring_init(bar_w, P.nslot);
  __syncthreads();

  const int n = gw < P.c ? (P.c - 1 - gw) / W + 1 : 0;
  uint32_t phase_bits = 0;
  auto src = [&](int i, const void*& ptr, uint32_t& bytes) {
    ptr = P.Crows + static_cast<size_t>(gw + i * W) * P.crow_bytes;
    bytes = static_cast<uint32_t>(P.crow_bytes);
  };
  auto emit = [&](int r, int k, float s) {
    const size_t o = static_cast<size_t>(P.row0 + r) * P.c + k;
    const float key = P.mode == 1 ? gumbel_key(s, P.T, __ldg(P.u_clusters + o)) : s;
    P.out[o] = key;
  };
  bool ok;
  if constexpr (FMT == kFmtInt8) {
    // packed INT8 row: chunk m of lane l = the 8 codes of elements (l + 32 m) * 8 .. + 8
    auto use = [&](int i, uint32_t slot) {
      const int k = gw + i * W;
      uint2 q[NCH];
      float sc[NCH];
#pragma unroll
      for (int m = 0; m < NCH; ++m) {
        const int e = (lane + 32 * m) * 8;
        q[m] = make_uint2(0u, 0u);
        sc[m] = 0.f;
        if (e < d) {
          q[m] = lds64(slot + static_cast<uint32_t>(e));
          sc[m] = bf16f(lds16(slot + static_cast<uint32_t>(d + 2 * (e >> 5))));
        }
      }
      for (int r = 0; r < R; ++r) {
        const uint32_t hrow = sh_a + static_cast<uint32_t>(r * d * 2);
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < NCH; ++m) {
          const int e = (lane + 32 * m) * 8;
          if (e < d) {
            const uint4 hv = lds128(hrow + 2u * e);
            float part = sbyte(q[m].x, 0) * bf16lo(hv.x);
            part = fmaf(sbyte(q[m].x, 1), bf16hi(hv.x), part);
            part = fmaf(sbyte(q[m].x, 2), bf16lo(hv.y), part);
            part = fmaf(sbyte(q[m].x, 3), bf16hi(hv.y), part);
            part = fmaf(sbyte(q[m].y, 0), bf16lo(hv.z), part);
            part = fmaf(sbyte(q[m].y, 1), bf16hi(hv.z), part);
            part = fmaf(sbyte(q[m].y, 2), bf16lo(hv.w), part);
            part = fmaf(sbyte(q[m].y, 3), bf16hi(hv.w), part);
            acc = fmaf(sc[m], part, acc);
          }
        }
        acc = warp_sum(acc);
        if (lane == 0) emit(r, k, acc);
      }
    };
    ok = warp_stream(n, P.nslot, ring_w, P.slot_bytes, bar_w, phase_bits, kWaitBudget, src, use);
  } else if constexpr (FMT == kFmtInt4) {
    constexpr int NQ = (NCH + 1) / 2;
    auto use = [&](int i, uint32_t slot) {
      const int k = gw + i * W;
      float qf[NQ * 16];
      float sc[NQ];
#pragma unroll
      for (int m = 0; m < NQ; ++m) {
        const int g = lane + 32 * m;
        uint2 q = make_uint2(0u, 0u);  // padding half-groups decode to code 0 with scale 0
        sc[m] = 0.f;
        if (g * 16 < d) {
          q = lds64(slot + 8u * g);
          sc[m] = bf16f(lds16(slot + d / 2 + 2u * (g >> 1)));
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          qf[16 * m + j] = nib(q.x, j);
          qf[16 * m + 8 + j] = nib(q.y, j);
        }
      }
      for (int r = 0; r < R; ++r) {
        const uint32_t hrow = sh_a + static_cast<uint32_t>(r * d * 2);
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < NQ; ++m) {
          const int g = lane + 32 * m;
          if (g * 16 < d) {
            const uint4 a = lds128(hrow + 32u * g), b2 = lds128(hrow + 32u * g + 16u);
            float part = 0.f;
            const uint32_t hw[8] = {a.x, a.y, a.z, a.w, b2.x, b2.y, b2.z, b2.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              part = fmaf(qf[16 * m + 2 * j], bf16lo(hw[j]), part);
              part = fmaf(qf[16 * m + 2 * j + 1], bf16hi(hw[j]), part);
            }
            acc = fmaf(sc[m], part, acc);
          }
        }
        acc = warp_sum(acc);
        if (lane == 0) emit(r, k, acc);
      }
    };
    ok = warp_stream(n, P.nslot, ring_w, P.slot_bytes, bar_w, phase_bits, kWaitBudget, src, use);
  } else {
    auto use = [&](int i, uint32_t slot) {
      const int k = gw + i * W;
      uint4 cw[NCH];
#pragma unroll
      for (int m = 0; m < NCH; ++m) {
        const int e = (lane + 32 * m) * 8;
        cw[m] = e < d ? lds128(slot + 2u * e) : make_uint4(0, 0, 0, 0);
      }
      for (int r = 0; r < R; ++r) {
        const uint32_t hrow = sh_a + static_cast<uint32_t>(r * d * 2);
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < NCH; ++m) {
          const int e = (lane + 32 * m) * 8;
          if (e < d) {
            const uint4 hv = lds128(hrow + 2u * e);
            acc = fmaf(bf16lo(cw[m].x), bf16lo(hv.x), acc);
            acc = fmaf(bf16hi(cw[m].x), bf16hi(hv.x), acc);
            acc = fmaf(bf16lo(cw[m].y), bf16lo(hv.y), acc);
            acc = fmaf(bf16hi(cw[m].y), bf16hi(hv.y), acc);
            acc = fmaf(bf16lo(cw[m].z), bf16lo(hv.z), acc);
            acc = fmaf(bf16hi(cw[m].z), bf16hi(hv.z), acc);
            acc = fmaf(bf16lo(cw[m].w), bf16lo(hv.w), acc);
            acc = fmaf(bf16hi(cw[m].w), bf16hi(hv.w), acc);
          }
        }
        acc = warp_sum(acc);
        if (lane == 0) emit(r, k, acc);
      }
    };
    ok = warp_stream(n, P.nslot, ring_w, P.slot_bytes, bar_w, phase_bits, kWaitBudget, src, use);
  }
  if (!ok && lane == 0) record_error(P.status, FH_ERR_TIMEOUT);
}

// ----------------------------------------------------------------------------
// per-row top-p select + candidate token list
// ----------------------------------------------------------------------------
__device__ void write_candidates(const SelectParams& P, const int32_t* ssel, int row) {
  if (!P.cand_tok) return;
  const int nc = P.p * P.b;
  int32_t* out = P.cand_tok + static_cast<size_t>(row) * nc;
  for (int r = threadIdx.x; r < nc; r += kThreads)
    out[r] = P.C2T.at(static_cast<size_t>(ssel[r / P.b]) * P.b + r % P.b);
}

__global__ void __launch_bounds__(kThreads, 1) select_kernel(const SelectParams P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int row = blockIdx.x;
  int32_t* ssel = reinterpret_cast<int32_t*>(smem);
  const uint32_t scratch_off = static_cast<uint32_t>((static_cast<size_t>(P.p) * 4 + 127) & ~size_t(127));
  uint8_t* scratch = smem + scratch_off;
  const float* in = P.in + static_cast<size_t>(row) * P.c;
  const float* u = P.perturb ? P.u_clusters + static_cast<size_t>(row) * P.c : nullptr;
  select_stage_scores(in, u, P.T, P.c, scratch);
  select_top_p_staged(P.c, P.p, 0u, scratch_off);
  int32_t* gsel = P.sel + static_cast<size_t>(row) * P.p;
  for (int i = threadIdx.x; i < P.p; i += kThreads) gsel[i] = ssel[i];
  write_candidates(P, ssel, row);
}

// Caller-given ids: validate (in range, distinct), sort ascending through a
// c-bit membership mask, then emit the canonical candidate list.
__global__ void __launch_bounds__(kThreads, 1) sort_ids_kernel(const SelectParams P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int words = (P.c + 31) / 32;
  uint32_t* bits = reinterpret_cast<uint32_t*>(smem);
  const size_t bit_bytes = (static_cast<size_t>(words) * 4 + 127) & ~size_t(127);
  int32_t* ssel = reinterpret_cast<int32_t*>(smem + bit_bytes);
  const size_t sel_bytes = (static_cast<size_t>(P.p) * 4 + 127) & ~size_t(127);
  uint32_t* wcount = reinterpret_cast<uint32_t*>(smem + bit_bytes + sel_bytes);
  __shared__ int bad;
  if (tid == 0) bad = 0;
  for (int i = tid; i < words; i += kThreads) bits[i] = 0u;
  __syncthreads();
  const int32_t* ids = P.ids_in + static_cast<size_t>(row) * P.p;
  for (int i = tid; i < P.p; i += kThreads) {
    const int k = ids[i];
    if (k < 0 || k >= P.c) {
      bad = 1;
    } else {
      const uint32_t old = atomicOr(&bits[k >> 5], 1u << (k & 31));
      if (old & (1u << (k & 31))) bad = 1;
    }
  }
  __syncthreads();
  if (bad) {
    if (tid == 0) {
      record_error(P.status, FH_ERR_OUT_OF_RANGE);
      P.row_ok[row] = 0;
    }
    // token 0 is a valid row address: the skipped row is streamed but never written out
    if (P.cand_tok) {
      int32_t* out = P.cand_tok + static_cast<size_t>(row) * P.p * P.b;
      for (int r = tid; r < P.p * P.b; r += kThreads) out[r] = 0;
    }
    return;
  }
  // compaction of set bits in id order: warp w owns a contiguous word range
  const int per_warp = (words + kWarps - 1) / kWarps;
  const int w0 = warp * per_warp, w1 = min(words, w0 + per_warp);
  uint32_t cnt = 0;
  for (int wi = w0 + lane; wi < w1; wi += 32) cnt += __popc(bits[wi]);
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xFFFFFFFFu, cnt, o);
  if (lane == 0) wcount[warp] = cnt;
  __syncthreads();
  uint32_t pos = 0;
  for (int w = 0; w < warp; ++w) pos += wcount[w];
  for (int base = w0; base < w1; base += 32) {
    const int wi = base + lane;
    const uint32_t word = wi < w1 ? bits[wi] : 0u;
    const uint32_t c = __popc(word);
    // exclusive prefix of popcounts across lanes
    uint32_t x = c;
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
      if (lane >= o) x += y;
    }
    uint32_t p0 = pos + x - c;
    uint32_t wb = word;
    while (wb) {
      const int bit = __ffs(wb) - 1;
      wb &= wb - 1;
      ssel[p0++] = wi * 32 + bit;
    }
    pos += __shfl_sync(0xFFFFFFFFu, x, 31);
  }
    __syncthreads();
  if (tid == 0) P.row_ok[row] = 1;
  int32_t* gsel = P.sel + static_cast<size_t>(row) * P.p;
  for (int i = tid; i < P.p; i += kThreads) gsel[i] = ssel[i];
  write_candidates(P, ssel, row);
}

// ----------------------------------------------------------------------------
// stage 2: candidate logits
// ----------------------------------------------------------------------------
template <int NCH>
__global__ void __launch_bounds__(kThreads, 1) candidates_kernel(const CandParams P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int W = gridDim.x * kWarps, gw = blockIdx.x * kWarps + warp;
  const int d = P.d;
  const uint32_t ring_w = smem_addr(smem + P.off_ring) + static_cast<uint32_t>(warp * P.nslot * P.slot_bytes);
  const uint32_t bar_w = smem_addr(smem + P.off_bar) + static_cast<uint32_t>(warp * P.nslot * 8);
  warp_ring_init(bar_w, P.nslot);
  __syncthreads();

  // contiguous item range per warp: item = row * nc + r
  const long long total = static_cast<long long>(P.B) * P.nc;
  const long long per = (total + W - 1) / W;
  const long long i0 = static_cast<long long>(gw) * per;
  const long long i1 = i0 + per < total ? i0 + per : total;
  const int n = i0 < total ? static_cast<int>(i1 - i0) : 0;

  // tokens of items [32*q, 32*q + 32) of this warp live in lane registers
  int tq = -2, tcur = 0, tnext = 0;  // -2: no batch loaded yet
  auto tok_batch = [&](int q) -> int {
    const long long it = i0 + 32LL * q + lane;
    return it < i1 ? __ldg(P.cand_tok + it) : 0;
  };
  auto token_of = [&](int i) -> int {
    const int q = i >> 5;
    if (q != tq && q != tq + 1) {  // first use or a jump: reload both batches
      tq = q;
      tcur = tok_batch(q);
      tnext = tok_batch(q + 1);
    } else if (q == tq + 1) {
      tq = q;
      tcur = tnext;
      tnext = tok_batch(q + 1);
    }
    return __shfl_sync(0xFFFFFFFFu, tcur, i & 31);
  };
  // src runs ahead of use by nslot (< 32) items, so keep a separate cursor for it
  int sq = -2, scur = 0, snext = 0;
  auto src_token = [&](int i) -> int {
    const int q = i >> 5;
    if (q != sq && q != sq + 1) {
      sq = q;
      scur = tok_batch(q);
      snext = tok_batch(q + 1);
    } else if (q == sq + 1) {
      sq = q;
      scur = snext;
      snext = tok_batch(q + 1);
    }
    return __shfl_sync(0xFFFFFFFFu, scur, i & 31);
  };

  float hr[NCH * 8];
  int cur_row = -1;
  bool row_valid = true;
  unsigned long long best = 0ull;
  auto flush = [&]() {
    if (cur_row >= 0 && lane == 0 && best && P.best) atomicMax(P.best + cur_row, best);
  };
  uint32_t phase_bits = 0;
  auto src = [&](int i, const void*& ptr, uint32_t& bytes) {
    int t = src_token(i);
    t = static_cast<unsigned>(t) < static_cast<unsigned>(P.v) ? t : 0;  // never address outside E
    ptr = P.E + static_cast<size_t>(t) * d;
    bytes = static_cast<uint32_t>(d * 2);
  };
  auto use = [&](int i, uint32_t slot) {
    const long long it = i0 + i;
    const int row = static_cast<int>(it / P.nc);
    const int t = token_of(i);
    if (row != cur_row) {
      flush();
      cur_row = row;
      best = 0ull;
      row_valid = P.row_ok ? (__ldg(P.row_ok + row) != 0) : true;
      load_h_chunks<NCH>(P.hidden + static_cast<size_t>(row) * d, d, hr);
    }
    const float z = row_dot_bf16<NCH>(slot, d, hr);
    if (row_valid) {
      const unsigned long long pk = pack_best(z, t);
      best = pk > best ? pk : best;
      if (lane == 0) {
        if (P.logits) P.logits[it] = z;
        if (P.token_out) P.token_out[it] = t;
      }
    }
  };
  const bool ok = warp_stream(n, P.nslot, ring_w, P.slot_bytes, bar_w, phase_bits, kWaitBudget, src, use);
  flush();
  if (!ok && lane == 0) record_error(P.status, FH_ERR_TIMEOUT);
}

// ----------------------------------------------------------------------------
// per-row output token
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1) epilogue_kernel(const EpilogueParams P) {
  __shared__ float scan[kWarps + 1];
  __shared__ int s_claim, s_last;
  const int row = blockIdx.x, tid = threadIdx.x;
  const unsigned long long bw = P.best[row];
  if (P.mode == 0) {
    if (tid == 0) {
      P.out_tokens[row] = best_token(bw);
      if (P.out_max_logit) P.out_max_logit[row] = best_logit(bw);
      P.best[row] = 0ull;
    }
    return;
  }
  const float* z = P.logits + static_cast<size_t>(row) * P.nc;
  const int nc = P.nc;
  const float ym = best_logit(bw) / P.T;
  const int q = (nc + kThreads - 1) / kThreads;
  const int i0 = min(nc, tid * q), i1 = min(nc, i0 + q);
  float loc = 0.f;
  for (int i = i0; i < i1; ++i) loc += expf(z[i] / P.T - ym);
  if (tid == 0) {
    s_claim = INT_MAX;
    s_last = 0;
  }
  float total;
  const float before = block_exclusive_scan<kThreads, float>(loc, scan, &total);
  const float u = fminf(fmaxf(P.u_token[row], 0.f), 0.99999994f);
  const float target = u * total;
  float run = before;
  int claim = INT_MAX, lastpos = -1;
  for (int i = i0; i < i1; ++i) {
    const float w = expf(z[i] / P.T - ym);
    if (w > 0.f) lastpos = i;
    run += w;
    if (run > target) {
      claim = i;
      break;
    }
  }
  if (claim != INT_MAX) atomicMin(&s_claim, claim);
  if (lastpos >= 0) atomicMax(&s_last, lastpos);
  __syncthreads();
  if (tid == 0) {
    const int idx = s_claim != INT_MAX ? s_claim : s_last;
    P.out_tokens[row] = P.cand_tok[static_cast<size_t>(row) * nc + idx];
    if (P.out_max_logit) P.out_max_logit[row] = best_logit(bw);
    P.best[row] = 0ull;
  }
}

}  // namespace

#define FH_DISPATCH_NCH(nch, CALL) \
  switch (nch) {                   \
    case 1: CALL(1);               \
    case 2: CALL(2);               \
    case 3: CALL(3);               \
    case 4: CALL(4);               \
    case 5: CALL(5);               \
    case 6: CALL(6);               \
    case 8: CALL(8);               \
    case 10: CALL(10);             \
    default: return cudaErrorInvalidValue; \
  }

cudaError_t launch_scores(const ScoresParams& P, int grid, size_t smem, int cfmt, int nch, cudaStream_t st) {
#define FH_L(N)                                                                          \
  if (cfmt == kFmtInt4) scores_kernel<N, kFmtInt4><<<grid, kThreads, smem, st>>>(P);      \
  else if (cfmt == kFmtInt8) scores_kernel<N, kFmtInt8><<<grid, kThreads, smem, st>>>(P); \
  else scores_kernel<N, kFmtBf16><<<grid, kThreads, smem, st>>>(P);                       \
  return cudaGetLastError();
  FH_DISPATCH_NCH(nch, FH_L)
#undef FH_L
}

cudaError_t launch_select(const SelectParams& P, int B, size_t smem, cudaStream_t st) {
  select_kernel<<<B, kThreads, smem, st>>>(P);
  return cudaGetLastError();
}

cudaError_t launch_sort_ids(const SelectParams& P, int B, size_t smem, cudaStream_t st) {
  sort_ids_kernel<<<B, kThreads, smem, st>>>(P);
  return cudaGetLastError();
}

cudaError_t launch_candidates(const CandParams& P, int grid, size_t smem, int nch, cudaStream_t st) {
#define FH_L(N)                                                    \
  candidates_kernel<N><<<grid, kThreads, smem, st>>>(P);           \
  return cudaGetLastError();
  FH_DISPATCH_NCH(nch, FH_L)
#undef FH_L
}

cudaError_t launch_epilogue(const EpilogueParams& P, int B, cudaStream_t st) {
  epilogue_kernel<<<B, kThreads, 0, st>>>(P);
  return cudaGetLastError();
}

cudaError_t set_attrs_batched(int max_smem) {
  cudaError_t e = cudaSuccess;
  auto set = [&](const void* f) {
    if (e == cudaSuccess) e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
  };
#define FH_S(N)                                                   \
  set(reinterpret_cast<const void*>(scores_kernel<N, kFmtBf16>)); \
  set(reinterpret_cast<const void*>(scores_kernel<N, kFmtInt4>)); \
  set(reinterpret_cast<const void*>(scores_kernel<N, kFmtInt8>)); \
  set(reinterpret_cast<const void*>(candidates_kernel<N>));
  FH_S(1) FH_S(2) FH_S(3) FH_S(4) FH_S(5) FH_S(6) FH_S(8) FH_S(10)
#undef FH_S
  set(reinterpret_cast<const void*>(select_kernel));
  set(reinterpret_cast<const void*>(sort_ids_kernel));
  return e;
}

}  // namespace fh
