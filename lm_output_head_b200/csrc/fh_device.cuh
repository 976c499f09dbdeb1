// Device building blocks shared by the FlashHead kernels (sm_100a).
//
//  * bulk global->shared copies (cp.async.bulk) completed on mbarriers, with
//    bounded waits;
//  * order-preserving float <-> uint32 keys and packed (logit, token) argmax
//    words;
//  * bf16 / INT4 unpacking into fp32;
//  * block-wide scans and the block radix select that picks the p largest
//    keys (ties to the lower id), used for probe selection (multi-probe
//    retrieval, FlashHead write-up section 1.2.2).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "fh_internal.h"

namespace fh {

constexpr int kThreads = 512;           // threads per CTA of the streaming kernels
constexpr int kWarps = kThreads / 32;

// ---------------------------------------------------------------------------
// status word
// ---------------------------------------------------------------------------
__device__ __forceinline__ void record_error(int* status, int code) {
  atomicCAS(status, 0, code);
}

// ---------------------------------------------------------------------------
// shared-memory addresses, mbarriers, bulk copies
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

// One contiguous global->shared copy; both addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of `bar` for at most `budget` SM clock cycles.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, long long budget) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > budget) return false;
  }
  return true;
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Bring `bytes` (multiple of 16, 16-byte aligned) into L2 without waiting.
__device__ __forceinline__ void bulk_prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const unsigned* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_u32(unsigned* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Release add without a result (orders this thread's earlier memory operations, and
// those made visible to it by a CTA barrier, before the add).
__device__ __forceinline__ void red_release_add_u32(unsigned* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void red_relaxed_add_u32(unsigned* p, uint32_t v) {
  asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t atom_acq_rel_add_u32(unsigned* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("red.release.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_relaxed_u32(const unsigned* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint16_t lds16(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}

// ---------------------------------------------------------------------------
// number formats
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ float bf16f(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

// Signed 4-bit code (two's complement) in bits [4i, 4i+4) of w, as an exact float.
// (n ^ 8) maps -8..7 to 0..15; OR-ing it into the mantissa of 2^23 gives 2^23 + (n ^ 8)
// exactly, and subtracting 2^23 + 8 leaves the signed code.
__device__ __forceinline__ float nib(uint32_t w, int i) {
  const uint32_t u = ((w >> (4 * i)) & 0xFu) ^ 0x8u;
  return __uint_as_float(0x4B000000u | u) - 8388616.0f;
}

// Signed byte i (two's complement) of w as an exact float, by the same trick:
// (byte ^ 0x80) maps -128..127 to 0..255 inside the mantissa of 2^23.
__device__ __forceinline__ float sbyte(uint32_t w, int i) {
  const uint32_t u = ((w >> (8 * i)) & 0xFFu) ^ 0x80u;
  return __uint_as_float(0x4B000000u | u) - 8388736.0f;
}

// Dot of 8 bf16 (one 16-byte chunk) with 8 fp32 values.
__device__ __forceinline__ float dot8(const uint4 w, const float* h, float acc) {
  acc = fmaf(bf16lo(w.x), h[0], acc);
  acc = fmaf(bf16hi(w.x), h[1], acc);
  acc = fmaf(bf16lo(w.y), h[2], acc);
  acc = fmaf(bf16hi(w.y), h[3], acc);
  acc = fmaf(bf16lo(w.z), h[4], acc);
  acc = fmaf(bf16hi(w.z), h[5], acc);
  acc = fmaf(bf16lo(w.w), h[6], acc);
  acc = fmaf(bf16hi(w.w), h[7], acc);
  return acc;
}

// Dot of 16 INT4 codes (8 bytes) with 16 fp32 values; the group scale is applied by the caller.
__device__ __forceinline__ float dot16q(const uint2 q, const float* h) {
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) a = fmaf(nib(q.x, i), h[i], a);
#pragma unroll
  for (int i = 0; i < 8; ++i) a = fmaf(nib(q.y, i), h[8 + i], a);
  return a;
}

// ---------------------------------------------------------------------------
// keys
// ---------------------------------------------------------------------------
// Monotone map float -> uint32 (larger float => larger key).
__device__ __forceinline__ uint32_t f2key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key2f(uint32_t k) {
  const uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(u);
}
// (logit, token) packed so that a larger word = larger logit, then lower token id.
__device__ __forceinline__ unsigned long long pack_best(float z, int32_t token) {
  return (static_cast<unsigned long long>(f2key(z)) << 32) |
         static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<uint32_t>(token));
}
__device__ __forceinline__ int32_t best_token(unsigned long long w) {
  return static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(w & 0xFFFFFFFFull));
}
__device__ __forceinline__ float best_logit(unsigned long long w) {
  return key2f(static_cast<uint32_t>(w >> 32));
}

// Gumbel-perturbed key s/T - ln(-ln u), u clamped to [2^-126, 1 - 2^-24].
__device__ __forceinline__ float gumbel_key(float s, float T, float u) {
  u = fminf(fmaxf(u, 1.17549435e-38f), 0.99999994f);
  return s / T - logf(-logf(u));
}

// ---------------------------------------------------------------------------
// warp / block reductions and scans
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long w = __shfl_xor_sync(0xFFFFFFFFu, v, o);
    v = w > v ? w : v;
  }
  return v;
}

// Exclusive scan of one value per thread over the block (NT threads);
// `scratch` holds NT/32 + 1 words. Returns the exclusive prefix; *total gets the sum.
template <int NT, typename T>
__device__ __forceinline__ T block_exclusive_scan(T v, T* scratch, T* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  T x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const T y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[w] = x;
  __syncthreads();
  if (w == 0) {
    const T t = lane < NT / 32 ? scratch[lane] : T(0);
    T s = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const T y = __shfl_up_sync(0xFFFFFFFFu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < NT / 32) scratch[lane] = s - t;
    if (lane == NT / 32 - 1) scratch[NT / 32] = s;
  }
  __syncthreads();
  const T r = scratch[w] + x - v;
  if (total) *total = scratch[NT / 32];
  __syncthreads();
  return r;
}

// ---------------------------------------------------------------------------
// block top-p select
// ---------------------------------------------------------------------------
struct SelectSmem {
  uint32_t hist[2048];
  uint32_t scan[kWarps + 1];
  uint32_t warp_gt[kWarps];
  uint32_t warp_eq[kWarps];
  uint32_t digit, above, bincount;
};

// Selects the p largest of n keys (order-preserving uint32) held in shared
// memory; equal keys go to the lower id. Writes the chosen ids to `sel`
// (shared or global) in ascending id order. All kThreads threads must call it.
//
// MSB-first radix select with 11/11/10-bit digits: each pass histograms the
// keys that still agree with the decided prefix, finds the digit where the
// count from the top reaches the remaining need, and stops early once that
// digit's bin holds exactly the keys still needed.
__device__ inline void block_select_top_p(const uint32_t* skey, int n, int p, int32_t* sel,
                                          SelectSmem& sm) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t prefix = 0, mask = 0;
  int need = p;
  const int shifts[3] = {21, 10, 0};
  const uint32_t digit_mask[3] = {0x7FFu, 0x7FFu, 0x3FFu};
  const int iters = (n + kThreads - 1) / kThreads;

  for (int pass = 0; pass < 3; ++pass) {
    const int sh = shifts[pass];
    const uint32_t dm = digit_mask[pass];
    for (int i = tid; i < 2048; i += kThreads) sm.hist[i] = 0;
    __syncthreads();
    for (int it = 0; it < iters; ++it) {
      const int k = it * kThreads + tid;
      bool act = k < n;
      const uint32_t key = act ? skey[k] : 0u;
      act = act && ((key & mask) == prefix);
      const uint32_t bin = (key >> sh) & dm;
      const uint32_t grp = __match_any_sync(0xFFFFFFFFu, act ? bin : (0x10000u | lane));
      if (act && lane == __ffs(grp) - 1) atomicAdd(&sm.hist[bin], static_cast<uint32_t>(__popc(grp)));
    }
    __syncthreads();
    // thread t owns bins 2047-4t .. 2044-4t (descending), so the exclusive
    // scan gives the number of keys in higher bins
    constexpr int kBpt = 2048 / kThreads;
    uint32_t loc = 0;
#pragma unroll
    for (int i = 0; i < kBpt; ++i) loc += sm.hist[2047 - kBpt * tid - i];
    const uint32_t above = block_exclusive_scan<kThreads, uint32_t>(loc, sm.scan, nullptr);
    uint32_t run = above;
#pragma unroll
    for (int i = 0; i < kBpt; ++i) {
      const int dg = 2047 - kBpt * tid - i;
      const uint32_t h = sm.hist[dg];
      if (run < static_cast<uint32_t>(need) && run + h >= static_cast<uint32_t>(need)) {
        sm.digit = static_cast<uint32_t>(dg);
        sm.above = run;
        sm.bincount = h;
      }
      run += h;
    }
    __syncthreads();
    need -= static_cast<int>(sm.above);
    prefix |= sm.digit << sh;
    mask |= dm << sh;
    const bool done = sm.bincount == static_cast<uint32_t>(need);
    __syncthreads();
    if (done) break;
  }

  // Compaction in ascending id order. Keys with (key & mask) > prefix are
  // taken; of those equal to prefix under the mask, the first `need` ids.
  const int per_warp = ((n + kWarps - 1) / kWarps + 31) & ~31;
  const int w0 = warp * per_warp, w1 = min(n, w0 + per_warp);
  uint32_t cgt = 0, ceq = 0;
  for (int k0 = w0; k0 < w1; k0 += 32) {
    const int k = k0 + lane;
    const uint32_t mk = k < w1 ? (skey[k] & mask) : 0u;
    const bool in = k < w1;
    cgt += __popc(__ballot_sync(0xFFFFFFFFu, in && mk > prefix));
    ceq += __popc(__ballot_sync(0xFFFFFFFFu, in && mk == prefix));
  }
  if (lane == 0) {
    sm.warp_gt[warp] = cgt;
    sm.warp_eq[warp] = ceq;
  }
  __syncthreads();
  uint32_t gt_before = 0, eq_before = 0;
  for (int w = 0; w < warp; ++w) {
    gt_before += sm.warp_gt[w];
    eq_before += sm.warp_eq[w];
  }
  uint32_t pos = gt_before + min(eq_before, static_cast<uint32_t>(need));
  uint32_t eq_seen = eq_before;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int k0 = w0; k0 < w1; k0 += 32) {
    const int k = k0 + lane;
    const bool in = k < w1;
    const uint32_t mk = in ? (skey[k] & mask) : 0u;
    const bool gt = in && mk > prefix;
    const bool eq = in && mk == prefix;
    const uint32_t eqm = __ballot_sync(0xFFFFFFFFu, eq);
    const bool take = gt || (eq && eq_seen + __popc(eqm & lt_mask) < static_cast<uint32_t>(need));
    const uint32_t tm = __ballot_sync(0xFFFFFFFFu, take);
    const uint32_t at = pos + __popc(tm & lt_mask);
    if (take && at < static_cast<uint32_t>(p)) sel[at] = k;
    pos += __popc(tm);
    eq_seen += __popc(eqm);
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// histogram-driven top-p select (compact code: it runs once per call)
// ---------------------------------------------------------------------------
// The keys' value range [lo, hi] is split into 4096 equal-width bins (linear
// in the key's float value, so even a concentrated score distribution puts
// only a few dozen keys in any bin and the shared-memory atomics that build
// the histogram rarely collide). A scan locates the bin holding the p-th
// largest key; every key above that bin is taken, and the keys inside it are
// ranked exactly (key desc, id asc) against each other. Keys live in shared
// memory and every loop stays a loop: the code runs once per call.
constexpr int kHistBins = 4096;
constexpr int kBoundaryMax = 2048;  // exact all-pairs ranking up to this many keys in the boundary bin

struct HistSelectSmem {
  uint32_t hist[kHistBins];
  uint32_t ckey[kBoundaryMax];
  int32_t cid[kBoundaryMax];
  uint32_t scan[kWarps + 1];
  uint32_t wmin[kWarps], wmax[kWarps];
  uint32_t t1, above, m1, ncand;
  float lo, scale;
  SelectSmem radix;
};

// Shared scratch for c keys: the struct, the keys, a c-byte flag array.
__host__ __device__ inline size_t hist_select_smem_bytes(int c) {
  return ((sizeof(HistSelectSmem) + 127) & ~size_t(127)) + ((static_cast<size_t>(c) * 4 + 127) & ~size_t(127)) +
         ((static_cast<size_t>(c) + 127) & ~size_t(127));
}

__device__ __forceinline__ uint32_t* select_keys_area(uint8_t* scratch) {
  return reinterpret_cast<uint32_t*>(scratch + ((sizeof(HistSelectSmem) + 127) & ~size_t(127)));
}

// Monotone bin of an order-preserving key: linear in its float value over [lo, lo + 4096/scale].
__device__ __forceinline__ uint32_t value_bin(uint32_t key, float lo, float scale) {
  const float x = (key2f(key) - lo) * scale;
  return static_cast<uint32_t>(fminf(fmaxf(x, 0.f), static_cast<float>(kHistBins - 1)));
}

// The launching kernel's dynamic shared memory. The out-of-line selectors
// below take byte offsets into it rather than pointers: a pointer argument of
// a non-inlined function is generic, and generic loads, stores and atomics
// into shared memory measured 2-3x slower than shared-space ones here.
extern __shared__ __align__(1024) uint8_t fh_dyn_smem[];

// Top-p of the c keys already staged in select_keys_area(scratch); writes the
// chosen ids ascending to `sel` (both byte offsets into the dynamic shared
// memory). All kThreads threads must call it.
static __device__ __noinline__ void select_top_p_staged(int c, int p, uint32_t sel_off, uint32_t scratch_off) {
  int32_t* sel = reinterpret_cast<int32_t*>(fh_dyn_smem + sel_off);
  uint8_t* scratch = fh_dyn_smem + scratch_off;
  HistSelectSmem& sm = *reinterpret_cast<HistSelectSmem*>(scratch);
  const uint32_t* key = select_keys_area(scratch);
  uint8_t* flag = reinterpret_cast<uint8_t*>(select_keys_area(scratch)) + ((static_cast<size_t>(c) * 4 + 127) & ~size_t(127));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // value range of the keys
  uint32_t mn = 0xFFFFFFFFu, mx = 0u;
  for (int k = tid; k < c; k += kThreads) {
    mn = min(mn, key[k]);
    mx = max(mx, key[k]);
  }
  for (int o = 16; o > 0; o >>= 1) {
    mn = min(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, o));
    mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
  }
  if (lane == 0) {
    sm.wmin[warp] = mn;
    sm.wmax[warp] = mx;
  }
  for (int i = tid; i < kHistBins; i += kThreads) sm.hist[i] = 0u;
  for (int i = tid; i < (c + 15) / 16; i += kThreads) reinterpret_cast<uint4*>(flag)[i] = make_uint4(0, 0, 0, 0);
  __syncthreads();
  if (tid == 0) {
    for (int w = 0; w < kWarps; ++w) {
      mn = min(mn, sm.wmin[w]);
      mx = max(mx, sm.wmax[w]);
    }
    const float flo = key2f(mn), fhi = key2f(mx);
    const float span = fhi - flo;
    sm.lo = flo;
    sm.scale = span > 0.f ? static_cast<float>(kHistBins) / span : 0.f;
    sm.ncand = 0u;
  }
  __syncthreads();
  const float lo = sm.lo, scale = sm.scale;
#pragma unroll 4
  for (int k = tid; k < c; k += kThreads) atomicAdd(&sm.hist[value_bin(key[k], lo, scale)], 1u);
  __syncthreads();

  // bin t1 holding the p-th largest key: thread t owns bins 4095-8t .. 4088-8t
  constexpr int kBpt = kHistBins / kThreads;
  uint32_t loc = 0;
  for (int i = 0; i < kBpt; ++i) loc += sm.hist[kHistBins - 1 - kBpt * tid - i];
  uint32_t run = block_exclusive_scan<kThreads, uint32_t>(loc, sm.scan, nullptr);
  for (int i = 0; i < kBpt; ++i) {
    const uint32_t h = sm.hist[kHistBins - 1 - kBpt * tid - i];
    if (run < static_cast<uint32_t>(p) && run + h >= static_cast<uint32_t>(p)) {
      sm.t1 = static_cast<uint32_t>(kHistBins - 1 - kBpt * tid - i);
      sm.above = run;
      sm.m1 = h;
    }
    run += h;
  }
  __syncthreads();
  const uint32_t t1 = sm.t1, m1 = sm.m1;
  const uint32_t need = static_cast<uint32_t>(p) - sm.above;
  const bool all_in_bin = (m1 == need);

  if (!all_in_bin && m1 > static_cast<uint32_t>(kBoundaryMax)) {  // pathological ties: radix fallback
    block_select_top_p(key, c, p, sel, sm.radix);
    return;
  }
  if (!all_in_bin) {
    // gather the boundary bin, rank it exactly (key desc, id asc), flag the chosen ids
    for (int k = tid; k < c; k += kThreads) {
      const uint32_t kk = key[k];
      if (value_bin(kk, lo, scale) == t1) {
        const uint32_t at = atomicAdd(&sm.ncand, 1u);
        if (at < static_cast<uint32_t>(kBoundaryMax)) {
          sm.ckey[at] = kk;
          sm.cid[at] = k;
        }
      }
    }
    __syncthreads();
    const uint32_t nb = min(sm.ncand, static_cast<uint32_t>(kBoundaryMax));  // == m1 for a consistent histogram
    for (uint32_t a = tid; a < nb; a += kThreads) {
      const uint32_t ka = sm.ckey[a];
      const int ia = sm.cid[a];
      uint32_t r = 0;
#pragma unroll 8
      for (uint32_t bb = 0; bb < nb; ++bb) {
        const uint32_t kb = sm.ckey[bb];
        r += (kb > ka) || (kb == ka && sm.cid[bb] < ia);
      }
      if (r < need) flag[ia] = 1;
    }
    __syncthreads();
  }

  // ascending-id compaction: warp w owns ids [w * span, w * span + span), 32
  // consecutive ids per step (one per lane: no shared-memory bank conflicts)
  const int span = ((c + kWarps - 1) / kWarps + 31) & ~31;
  const int w0 = min(c, warp * span), w1 = min(c, w0 + span);
  auto taken = [&](int k) {
    const uint32_t bn = value_bin(key[k], lo, scale);
    return bn > t1 || (bn == t1 && (all_in_bin || flag[k]));
  };
  uint32_t cnt = 0;
  for (int base = w0; base < w1; base += 32) {
    const int k = base + lane;
    cnt += __popc(__ballot_sync(0xFFFFFFFFu, k < w1 && taken(k)));
  }
  if (lane == 0) sm.scan[warp] = cnt;
  __syncthreads();
  uint32_t pos = 0;
  for (int w = 0; w < warp; ++w) pos += sm.scan[w];
  const uint32_t lt = (1u << lane) - 1u;
  for (int base = w0; base < w1; base += 32) {
    const int k = base + lane;
    const bool tk = k < w1 && taken(k);
    const uint32_t m = __ballot_sync(0xFFFFFFFFu, tk);
    const uint32_t at = pos + __popc(m & lt);
    if (tk && at < static_cast<uint32_t>(p)) sel[at] = k;
    pos += __popc(m);
  }
  __syncthreads();
}


// Exclusive block scan of one u32 per thread: warp scans by shuffles, one
// barrier, then every thread adds the totals of the warps before it.
// `wsum` (kWarps words) must not be reused before the next barrier.
__device__ __forceinline__ uint32_t block_scan_excl_u32(uint32_t v, uint32_t* wsum, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  uint32_t before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const uint32_t t = wsum[w];
    before += w < warp ? t : 0u;
    all += t;
  }
  if (total) *total = all;
  return before + x - v;
}

// ---------------------------------------------------------------------------
// boundary of a top-p set
// ---------------------------------------------------------------------------
// For n keys (order-preserving u32) in shared memory with their cluster ids
// (a shared array, or the key's index when ids_off == kImplicitIds), finds the
// p-th entry in the order (key desc, id asc): cluster k with key x is among
// the p best iff x > bkey, or x == bkey and k <= bid. Also returns the lower
// value edges of the histogram bins holding the ra-th and rb-th largest keys
// (NaN where the rank exceeds n), used to predict the next call's
// thresholds. Steps: value range, a value-linear 4096-bin histogram, a
// two-level search from the top for the bins of ranks p, ra, rb, and an
// exact rank (key desc, id asc) of the entries of the boundary bin. More than
// kBoundEntries entries in that bin (heavy ties) sets `heavy` and returns
// without a boundary. All kThreads threads must call it; every thread sees
// the result in the struct after it returns.
constexpr uint32_t kImplicitIds = 0xFFFFFFFFu;
constexpr int kBoundEntries = 1024;

struct BoundSmem {
  uint32_t hist[kHistBins];
  uint32_t ckey[kBoundEntries];
  int32_t cid[kBoundEntries];
  uint32_t wmin[kWarps], wmax[kWarps], wtot[kWarps];
  uint32_t t[3], above, m1, nc;
  uint32_t bkey;
  int32_t bid;
  float lo, scale, edge_a, edge_b;
  int heavy;
};

static __device__ __noinline__ void select_boundary(int n, int p, int ra, int rb, uint32_t keys_off,
                                                    uint32_t ids_off, uint32_t sm_off) {
  const uint32_t* key = reinterpret_cast<const uint32_t*>(fh_dyn_smem + keys_off);
  const int32_t* ids = reinterpret_cast<const int32_t*>(fh_dyn_smem + (ids_off == kImplicitIds ? 0u : ids_off));
  BoundSmem& sm = *reinterpret_cast<BoundSmem*>(fh_dyn_smem + sm_off);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool implicit = ids_off == kImplicitIds;

  uint32_t mn = 0xFFFFFFFFu, mx = 0u;
  for (int i = tid; i < n; i += kThreads) {
    mn = min(mn, key[i]);
    mx = max(mx, key[i]);
  }
  mn = __reduce_min_sync(0xFFFFFFFFu, mn);
  mx = __reduce_max_sync(0xFFFFFFFFu, mx);
  if (lane == 0) {
    sm.wmin[warp] = mn;
    sm.wmax[warp] = mx;
  }
  for (int i = tid; i < kHistBins / 4; i += kThreads) reinterpret_cast<uint4*>(sm.hist)[i] = make_uint4(0, 0, 0, 0);
  if (tid == 0) sm.nc = 0u;
  __syncthreads();
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    mn = min(mn, sm.wmin[w]);
    mx = max(mx, sm.wmax[w]);
  }
  const float lo = key2f(mn), span = key2f(mx) - lo;
  const float scale = span > 0.f ? static_cast<float>(kHistBins) / span : 0.f;
  for (int i = tid; i < n; i += kThreads) atomicAdd(&sm.hist[value_bin(key[i], lo, scale)], 1u);
  __syncthreads();
  {
    uint32_t s = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) s += sm.hist[kHistBins - 1 - 256 * warp - (lane + 32 * i)];
    s = __reduce_add_sync(0xFFFFFFFFu, s);
    if (lane == 0) sm.wtot[warp] = s;
  }
  __syncthreads();
  {
    uint32_t above_w = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) above_w += w < warp ? sm.wtot[w] : 0u;
    const uint32_t rk[3] = {static_cast<uint32_t>(p), static_cast<uint32_t>(ra), static_cast<uint32_t>(rb)};
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const uint32_t rr = rk[j];
      if (rr >= 1u && above_w < rr && above_w + sm.wtot[warp] >= rr) {
        uint32_t hv[8], s = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          hv[i] = sm.hist[kHistBins - 1 - 256 * warp - 8 * lane - i];
          s += hv[i];
        }
        uint32_t incl = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (lane >= o) incl += y;
        }
        uint32_t run = above_w + incl - s;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (run < rr && run + hv[i] >= rr) {
            sm.t[j] = static_cast<uint32_t>(kHistBins - 1 - 256 * warp - 8 * lane - i);
            if (j == 0) {
              sm.above = run;
              sm.m1 = hv[i];
            }
          }
          run += hv[i];
        }
      }
    }
  }
  __syncthreads();
  const uint32_t t1 = sm.t[0], m1 = sm.m1, need = static_cast<uint32_t>(p) - sm.above;
  if (tid == 0) {
    sm.lo = lo;
    sm.scale = scale;
    sm.edge_a = ra <= n ? (scale > 0.f ? lo + static_cast<float>(sm.t[1]) / scale : lo) : __int_as_float(0x7FC00000);
    sm.edge_b = rb <= n ? (scale > 0.f ? lo + static_cast<float>(sm.t[2]) / scale : lo) : __int_as_float(0x7FC00000);
    sm.heavy = m1 > static_cast<uint32_t>(kBoundEntries) ? 1 : 0;
  }
  if (m1 > static_cast<uint32_t>(kBoundEntries)) {
    __syncthreads();
    return;
  }
  for (int i = tid; i < n; i += kThreads) {
    const uint32_t x = key[i];
    if (value_bin(x, lo, scale) == t1) {
      const uint32_t at = atomicAdd(&sm.nc, 1u);
      sm.ckey[at] = x;
      sm.cid[at] = implicit ? i : (ids[i] & 0x7FFFFFFF);
    }
  }
  __syncthreads();
  for (uint32_t a = tid; a < m1; a += kThreads) {
    const uint32_t ka = sm.ckey[a];
    const int32_t ia = sm.cid[a];
    uint32_t r = 0;
    for (uint32_t bb = 0; bb < m1; ++bb) {
      const uint32_t kb = sm.ckey[bb];
      r += (kb > ka || (kb == ka && sm.cid[bb] < ia)) ? 1u : 0u;
    }
    if (r + 1u == need) {
      sm.bkey = ka;
      sm.bid = ia;
    }
  }
  __syncthreads();
}

// Stage keys from fp32 scores, optionally Gumbel-perturbed: scores/T - ln(-ln u).
__device__ __forceinline__ void select_stage_scores(const float* scores, const float* u, float T, int c,
                                                    uint8_t* scratch) {
  uint32_t* key = select_keys_area(scratch);
#pragma unroll 4
  for (int k = threadIdx.x; k < c; k += kThreads) {
    float v = __ldcg(scores + k);
    if (u) v = gumbel_key(v, T, __ldcg(u + k));
    key[k] = f2key(v);
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// register streaming of rows
// ---------------------------------------------------------------------------
// A warp reads a row with plain non-allocating 16-byte loads straight into
// registers (lane l holds chunks l, l+32, ...) and dots it with h staged once
// per CTA in shared memory as fp32. With two 512-thread CTAs per SM this keeps
// ~128 KB per SM in flight and measured 6.3 TB/s on a 1 GiB read sweep, above
// the cp.async.bulk rings tried for the same job.
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// bf16 row: chunk m of lane l covers elements (l + 32 m) * 8 .. + 8.
template <int NCH>
__device__ __forceinline__ void row_load_bf16(const uint16_t* row, int d, uint4 (&w)[NCH]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int m = 0; m < NCH; ++m) {
    const int e = (lane + 32 * m) * 8;
    w[m] = e < d ? ldg_stream(row + e) : make_uint4(0, 0, 0, 0);
  }
}

template <int NCH>
__device__ __forceinline__ float row_dot_bf16_hs(const uint4 (&w)[NCH], const float* hs, int d) {
  const int lane = threadIdx.x & 31;
  float acc = 0.f;
#pragma unroll
  for (int m = 0; m < NCH; ++m) {
    const int e = (lane + 32 * m) * 8;
    if (e < d) {
      const float4 a = *reinterpret_cast<const float4*>(hs + e);
      const float4 b = *reinterpret_cast<const float4*>(hs + e + 4);
      acc = fmaf(bf16lo(w[m].x), a.x, acc);
      acc = fmaf(bf16hi(w[m].x), a.y, acc);
      acc = fmaf(bf16lo(w[m].y), a.z, acc);
      acc = fmaf(bf16hi(w[m].y), a.w, acc);
      acc = fmaf(bf16lo(w[m].z), b.x, acc);
      acc = fmaf(bf16hi(w[m].z), b.y, acc);
      acc = fmaf(bf16lo(w[m].w), b.z, acc);
      acc = fmaf(bf16hi(w[m].w), b.w, acc);
    }
  }
  return warp_sum(acc);
}

// Packed INT4 row ([d/2 code bytes][d/16 scale bytes]) in the same chunk
// layout as a bf16 row: for chunk m, lane l holds the 4 code bytes of
// elements (l + 32 m) * 8 .. + 8 (one 32-bit word) and the bf16 scale of their
// group of 32, so the codes load coalesced and h is read as two float4 per
// chunk at a 32-byte lane stride (no shared-memory bank conflicts).
__device__ __forceinline__ uint32_t ldg_stream32(const void* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

template <int NCH>
__device__ __forceinline__ void row_load_int4(const uint8_t* row, int d, uint32_t (&q)[NCH], uint32_t (&sc)[NCH]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int m = 0; m < NCH; ++m) {
    const int e = (lane + 32 * m) * 8;
    if (e < d) {
      q[m] = ldg_stream32(row + e / 2);
      sc[m] = __ldg(reinterpret_cast<const unsigned short*>(row + d / 2) + (e >> 5));
    } else {
      q[m] = 0u;
      sc[m] = 0u;
    }
  }
}

template <int NCH>
__device__ __forceinline__ float row_dot_int4_hs(const uint32_t (&q)[NCH], const uint32_t (&sc)[NCH], const float* hs,
                                                 int d) {
  const int lane = threadIdx.x & 31;
  float acc = 0.f;
#pragma unroll
  for (int m = 0; m < NCH; ++m) {
    const int e = (lane + 32 * m) * 8;
    if (e < d) {
      const float4 a = *reinterpret_cast<const float4*>(hs + e);
      const float4 b = *reinterpret_cast<const float4*>(hs + e + 4);
      float part = nib(q[m], 0) * a.x;
      part = fmaf(nib(q[m], 1), a.y, part);
      part = fmaf(nib(q[m], 2), a.z, part);
      part = fmaf(nib(q[m], 3), a.w, part);
      part = fmaf(nib(q[m], 4), b.x, part);
      part = fmaf(nib(q[m], 5), b.y, part);
      part = fmaf(nib(q[m], 6), b.z, part);
      part = fmaf(nib(q[m], 7), b.w, part);
      acc = fmaf(__uint_as_float(sc[m] << 16), part, acc);
    }
  }
  return warp_sum(acc);
}

// Packed INT8 row ([d code bytes][d/16 scale bytes]) in the bf16 chunk layout:
// for chunk m, lane l holds the 8 codes of elements (l + 32 m) * 8 .. + 8 (one
// 8-byte load) and the bf16 scale of their group of 32.
__device__ __forceinline__ uint2 ldg_stream64(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}

// The row's bf16 scales travel as 32-bit words (word w = the scales of groups
// 2w and 2w + 1), NW words per lane (lane l holds words l, l + 32, ...): one
// register per 2048 elements instead of one per chunk. Chunk m of lane l
// needs group (l >> 2) + 8 m, i.e. word (l >> 3) + 4 m, which sits in lane
// ((l >> 3) + 4 m) % 32, register m / 8 -- the same register for the whole warp.
template <int NCH>
constexpr int int8_scale_words() { return (NCH + 7) / 8; }

template <int NCH>
__device__ __forceinline__ void row_load_int8(const uint8_t* row, int d, uint2 (&q)[NCH],
                                              uint32_t (&scw)[int8_scale_words<NCH>()]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int m = 0; m < NCH; ++m) {
    const int e = (lane + 32 * m) * 8;
    q[m] = e < d ? ldg_stream64(row + e) : make_uint2(0u, 0u);
  }
  const int nw = (d / 32 + 1) / 2;  // scale words of the row
#pragma unroll
  for (int j = 0; j < int8_scale_words<NCH>(); ++j) {
    const int wi = lane + 32 * j;
    uint32_t v = 0u;
    if (wi < nw) {
      const unsigned short* sp = reinterpret_cast<const unsigned short*>(row + d) + 2 * wi;
      v = __ldg(sp);
      if (2 * wi + 1 < d / 32) v |= static_cast<uint32_t>(__ldg(sp + 1)) << 16;
    }
    scw[j] = v;
  }
}

template <int NCH>
__device__ __forceinline__ float row_dot_int8_hs(const uint2 (&q)[NCH], const uint32_t (&scw)[int8_scale_words<NCH>()],
                                                 const float* hs, int d) {
  const int lane = threadIdx.x & 31;
  float acc = 0.f;
#pragma unroll
  for (int m = 0; m < NCH; ++m) {
    const int wi = (lane >> 3) + 4 * m;
    const uint32_t word = __shfl_sync(0xFFFFFFFFu, scw[m / 8], wi & 31);
    const int e = (lane + 32 * m) * 8;
    if (e < d) {
      const float4 a = *reinterpret_cast<const float4*>(hs + e);
      const float4 b = *reinterpret_cast<const float4*>(hs + e + 4);
      float part = sbyte(q[m].x, 0) * a.x;
      part = fmaf(sbyte(q[m].x, 1), a.y, part);
      part = fmaf(sbyte(q[m].x, 2), a.z, part);
      part = fmaf(sbyte(q[m].x, 3), a.w, part);
      part = fmaf(sbyte(q[m].y, 0), b.x, part);
      part = fmaf(sbyte(q[m].y, 1), b.y, part);
      part = fmaf(sbyte(q[m].y, 2), b.z, part);
      part = fmaf(sbyte(q[m].y, 3), b.w, part);
      const uint32_t bits = ((lane >> 2) & 1) ? (word & 0xFFFF0000u) : (word << 16);  // group parity
      acc = fmaf(__uint_as_float(bits), part, acc);
    }
  }
  return warp_sum(acc);
}

// The same dots for a row held in shared memory (landed by a bulk copy).
template <int NCH>
__device__ __forceinline__ float srow_dot_bf16_hs(uint32_t row, const float* hs, int d) {
  const int lane = threadIdx.x & 31;
  float acc = 0.f;
#pragma unroll
  for (int m = 0; m < NCH; ++m) {
    const int e = (lane + 32 * m) * 8;
    if (e < d) {
      const uint4 w = lds128(row + 2u * e);
      const float4 a = *reinterpret_cast<const float4*>(hs + e);
      const float4 b = *reinterpret_cast<const float4*>(hs + e + 4);
      acc = fmaf(bf16lo(w.x), a.x, acc);
      acc = fmaf(bf16hi(w.x), a.y, acc);
      acc = fmaf(bf16lo(w.y), a.z, acc);
      acc = fmaf(bf16hi(w.y), a.w, acc);
      acc = fmaf(bf16lo(w.z), b.x, acc);
      acc = fmaf(bf16hi(w.z), b.y, acc);
      acc = fmaf(bf16lo(w.w), b.z, acc);
      acc = fmaf(bf16hi(w.w), b.w, acc);
    }
  }
  return warp_sum(acc);
}

template <int NCH>
__device__ __forceinline__ float srow_dot_int4_hs(uint32_t row, const float* hs, int d) {
  uint32_t q[NCH], sc[NCH];
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int m = 0; m < NCH; ++m) {
    const int e = (lane + 32 * m) * 8;
    if (e < d) {
      uint32_t w;
      asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w) : "r"(row + static_cast<uint32_t>(e / 2)));
      q[m] = w;
      sc[m] = lds16(row + static_cast<uint32_t>(d / 2 + 2 * (e >> 5)));
    } else {
      q[m] = 0u;
      sc[m] = 0u;
    }
  }
  return row_dot_int4_hs<NCH>(q, sc, hs, d);
}

template <int NCH>
__device__ __forceinline__ float srow_dot_int8_hs(uint32_t row, const float* hs, int d) {
  const int lane = threadIdx.x & 31;
  float acc = 0.f;
#pragma unroll
  for (int m = 0; m < NCH; ++m) {
    const int e = (lane + 32 * m) * 8;
    if (e < d) {
      const uint2 q = lds64(row + static_cast<uint32_t>(e));
      const float scl = bf16f(lds16(row + static_cast<uint32_t>(d + 2 * (e >> 5))));
      const float4 a = *reinterpret_cast<const float4*>(hs + e);
      const float4 b = *reinterpret_cast<const float4*>(hs + e + 4);
      float part = sbyte(q.x, 0) * a.x;
      part = fmaf(sbyte(q.x, 1), a.y, part);
      part = fmaf(sbyte(q.x, 2), a.z, part);
      part = fmaf(sbyte(q.x, 3), a.w, part);
      part = fmaf(sbyte(q.y, 0), b.x, part);
      part = fmaf(sbyte(q.y, 1), b.y, part);
      part = fmaf(sbyte(q.y, 2), b.z, part);
      part = fmaf(sbyte(q.y, 3), b.w, part);
      acc = fmaf(scl, part, acc);
    }
  }
  return warp_sum(acc);
}

// Stage a bf16 vector of d elements (d % 8 == 0) into shared memory as fp32.
__device__ __forceinline__ void stage_h_f32(const uint16_t* h, int d, float* hs) {
  for (int i = threadIdx.x; i < d / 8; i += blockDim.x) {
    const uint4 w = *reinterpret_cast<const uint4*>(h + 8 * i);
    float4 a, b;
    a.x = bf16lo(w.x); a.y = bf16hi(w.x); a.z = bf16lo(w.y); a.w = bf16hi(w.y);
    b.x = bf16lo(w.z); b.y = bf16hi(w.z); b.z = bf16lo(w.w); b.w = bf16hi(w.w);
    reinterpret_cast<float4*>(hs)[2 * i] = a;
    reinterpret_cast<float4*>(hs)[2 * i + 1] = b;
  }
}

// ---------------------------------------------------------------------------
// per-warp streaming of rows through a ring of shared-memory slots
// ---------------------------------------------------------------------------
// Each warp owns `nslot` slots of `slot_bytes` and one mbarrier per slot.
// Item i of the warp's n items is copied by one cp.async.bulk into slot
// i % nslot; lane 0 issues, all lanes wait, `use(i, slot_addr)` consumes, and
// the slot is refilled with item i + nslot. `src(i, ptr, bytes)` is evaluated
// by all lanes (it may shuffle prefetched ids). The first min(n, nslot)
// copies can be issued early (warp_stream_prologue) so that they overlap
// whatever the warp does before consuming. A wait that exceeds `budget`
// cycles makes the warp wait (bounded) for its copies still in flight and
// return false.
__device__ __forceinline__ void warp_ring_init(uint32_t bars, int nslot) {
  if ((threadIdx.x & 31) == 0) {
    for (int s = 0; s < nslot; ++s) mbar_init(bars + 8u * s, 1);
    fence_mbar_init();
  }
  __syncwarp();
}

template <class Src>
__device__ __forceinline__ void warp_stream_prologue(int n, int nslot, uint32_t ring, uint32_t slot_bytes,
                                                     uint32_t bars, Src src) {
  const int lane = threadIdx.x & 31;
  const int pre = n < nslot ? n : nslot;
  for (int s = 0; s < pre; ++s) {
    const void* ptr;
    uint32_t bytes;
    src(s, ptr, bytes);
    if (lane == 0) {
      mbar_expect_tx(bars + 8u * s, bytes);
      bulk_g2s(ring + s * slot_bytes, ptr, bytes, bars + 8u * s);
    }
  }
}

template <class Src, class Use>
__device__ __forceinline__ bool warp_stream_run(int n, int nslot, uint32_t ring, uint32_t slot_bytes,
                                                uint32_t bars, uint32_t& phase_bits, long long budget,
                                                Src src, Use use) {
  const int lane = threadIdx.x & 31;
  for (int i = 0; i < n; ++i) {
    const int s = i % nslot;
    const uint32_t bar = bars + 8u * s;
    const bool got = mbar_wait_bounded(bar, (phase_bits >> s) & 1u, budget);
    if (!__all_sync(0xFFFFFFFFu, got)) {
      const int last = (i + nslot < n) ? i + nslot : n;
      for (int j = i; j < last; ++j) {
        const int sj = j % nslot;
        mbar_wait_bounded(bars + 8u * sj, (phase_bits >> sj) & 1u, budget);
      }
      __syncwarp();
      return false;
    }
    phase_bits ^= 1u << s;
    use(i, ring + s * slot_bytes);
    __syncwarp();
    if (i + nslot < n) {
      const void* ptr;
      uint32_t bytes;
      src(i + nslot, ptr, bytes);
      if (lane == 0) {
        fence_proxy_async_smem();
        mbar_expect_tx(bar, bytes);
        bulk_g2s(ring + s * slot_bytes, ptr, bytes, bar);
      }
    }
  }
  return true;
}

template <class Src, class Use>
__device__ __forceinline__ bool warp_stream(int n, int nslot, uint32_t ring, uint32_t slot_bytes,
                                            uint32_t bars, uint32_t& phase_bits, long long budget,
                                            Src src, Use use) {
  warp_stream_prologue(n, nslot, ring, slot_bytes, bars, src);
  return warp_stream_run(n, nslot, ring, slot_bytes, bars, phase_bits, budget, src, use);
}


// Load this lane's slice of a bf16 vector into fp32 registers in the layout
// of 16-byte chunks: chunk m covers elements (lane + 32 m) * 8 .. + 8.
template <int NCH>
__device__ __forceinline__ void load_h_chunks(const uint16_t* h, int d, float* hr) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int m = 0; m < NCH; ++m) {
    const int e = (lane + 32 * m) * 8;
    uint4 w = make_uint4(0, 0, 0, 0);
    if (e < d) w = *reinterpret_cast<const uint4*>(h + e);
    hr[8 * m + 0] = bf16lo(w.x); hr[8 * m + 1] = bf16hi(w.x);
    hr[8 * m + 2] = bf16lo(w.y); hr[8 * m + 3] = bf16hi(w.y);
    hr[8 * m + 4] = bf16lo(w.z); hr[8 * m + 5] = bf16hi(w.z);
    hr[8 * m + 6] = bf16lo(w.w); hr[8 * m + 7] = bf16hi(w.w);
  }
}


// Dot of a bf16 row in shared memory with register-resident h (chunk layout), warp-reduced.
template <int NCH>
__device__ __forceinline__ float row_dot_bf16(uint32_t row, int d, const float* hr) {
  const int lane = threadIdx.x & 31;
  float acc = 0.f;
#pragma unroll
  for (int m = 0; m < NCH; ++m) {
    const int e = (lane + 32 * m) * 8;
    if (e < d) acc = dot8(lds128(row + 2u * e), hr + 8 * m, acc);
  }
  return warp_sum(acc);
}


}  // namespace fh
