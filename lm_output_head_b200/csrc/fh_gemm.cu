// Tensor-core (tcgen05) tile GEMM for batches of hidden states (B >= 64),
// where the head's contractions are dense enough for the 5th-generation
// tensor cores: centroid scores S = H C^T (FlashHead write-up, section
// 1.2.2; INT4 centroids per section 1.2.4) and the dense comparison head
// z = H E^T with a fused argmax (section 1.1).
//
// The hidden rows are the MMA's M side (one or two blocks of 128; up to 256
// rows per launch) and the streamed centroid / token rows its N side, tn =
// 256 (or 128) per tile, so every epilogue thread owns one hidden row: the
// argmax is a register-local running maximum and score rows are stored as
// contiguous runs. One persistent CTA per SM loops over tiles of the
// streamed rows:
//   - warp 5 (one lane) loads H blocks, and the streamed rows when they are
//     bf16, with TMA (cp.async.bulk.tensor, 128-byte swizzle, no multicast)
//     into a ring of shared-memory stages of 64 K-elements;
//   - INT4 or INT8 centroids: warps 8..15 read the packed codes and bf16
//     scales and write code * scale into the stage as an exact pair of bf16
//     tiles hi + lo (hi = bf16(code * scale), lo = the rest, exact in bf16:
//     code * scale has at most 7 + 8 significant bits), in the same swizzled
//     layout, so two MMAs give the exact products;
//   - warp 4 (one lane) issues tcgen05.mma kind::f16 (M 128, N tn, K 16; bf16
//     in, fp32 accumulators in tensor memory, double-buffered when they fit so
//     the epilogue of one tile overlaps the MMAs of the next) and commits stage
//     releases to mbarriers;
//   - warps 0..3 read the accumulators (tcgen05.ld, one TMEM lane = one hidden
//     row per thread) and either store scores (or Gumbel keys
//     s/T - ln(-ln u)), or keep a packed (logit, token) maximum per hidden row
//     (one atomicMax per row and CTA at the end), optionally storing logits.
// Every wait is bounded; one that runs out records FH_ERR_TIMEOUT, the CTA
// drains its copies and MMAs, frees its tensor memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "fh_device.cuh"

namespace fh {
namespace {

constexpr int kGemmThreads = 512;  // 16 warps
constexpr int kTileM = 128;
constexpr int kTileK = 64;         // bf16 elements per stage row: 128 bytes, one swizzle span
constexpr int kMaxN = 256;
constexpr long long kGemmBudget = 4000000000LL;

constexpr int kDequantThreads = 256;  // warps 8..15

struct GemmSmem {  // after the stages
  unsigned long long full[4], empty[4], tfull[2], tempty[2], done;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ bool wait_parity(uint32_t bar, uint32_t parity, const volatile int* abort_flag,
                                            long long budget) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > budget) return false;
  }
  return true;
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(dst),
      "l"(map), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// Shared-memory matrix descriptor: K-major operand, rows of 128 bytes with the
// 128-byte swizzle, 8-row groups 1024 bytes apart (tile base 1024-aligned).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);          // start address
  d |= static_cast<uint64_t>(1u) << 16;                        // leading byte offset (unused when swizzled)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;                // stride byte offset: 8 rows x 128 B
  d |= static_cast<uint64_t>(1u) << 46;                        // descriptor version
  d |= static_cast<uint64_t>(2u) << 61;                        // 128-byte swizzle
  return d;
}

// Instruction descriptor, kind::f16: bf16 A and B (K-major), fp32 D, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t dtmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(dtmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}


template <int FMT>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmR, const GemmParams P) {
  constexpr bool B_Q = FMT != kFmtBf16;  // streamed rows dequantised in the kernel
  extern __shared__ __align__(1024) uint8_t gsm[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = P.stages, hm = P.hm, tn = P.tn, nbuf = P.nbuf;
  const uint32_t a_bytes = kTileM * kTileK * 2;                     // one 128-row block of H: 16 KB
  const uint32_t b_bytes = static_cast<uint32_t>(tn) * kTileK * 2;  // tn streamed rows x 128 B
  const uint32_t stage_bytes = static_cast<uint32_t>(hm) * a_bytes + (B_Q ? 2u : 1u) * b_bytes;
  // stages start at the first 1024-byte boundary (the 128-byte swizzle repeats every 1024 bytes)
  const uint32_t raw = smem_addr(gsm);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = gsm + (base - raw);
  GemmSmem& sm = *reinterpret_cast<GemmSmem*>(gbase + static_cast<size_t>(S) * stage_bytes);
  auto a_at = [&](int s, int m) { return base + static_cast<uint32_t>(s) * stage_bytes + static_cast<uint32_t>(m) * a_bytes; };
  auto b_hi = [&](int s) { return base + static_cast<uint32_t>(s) * stage_bytes + static_cast<uint32_t>(hm) * a_bytes; };
  auto b_lo = [&](int s) { return b_hi(s) + b_bytes; };
  auto bar = [&](unsigned long long& x) { return smem_addr(&x); };

  const int ntiles = (P.rows + tn - 1) / tn;
  const int kst = (P.d + kTileK - 1) / kTileK;
  const volatile int* abort_flag = &sm.abort_flag;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(bar(sm.full[s]), B_Q ? 1 + kDequantThreads : 1);
      mbar_init(bar(sm.empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar(sm.tfull[a]), 1);
      mbar_init(bar(sm.tempty[a]), kTileM);
    }
    mbar_init(bar(sm.done), 1);
    fence_mbar_init();
    sm.abort_flag = 0;
  }
  if (warp == 4) {  // tensor memory: nbuf x hm accumulators of tn fp32 columns
    const uint32_t dst = smem_addr(&sm.tmem_base);
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst), "r"(P.tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  auto fail = [&]() {
    record_error(P.status, FH_ERR_TIMEOUT);
    sm.abort_flag = 1;
  };

  if (warp == 5) {
    // ---------------- TMA producer: H blocks, and the streamed rows when bf16 ----------------
    if (lane == 0) {
      int g = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
        for (int ks = 0; ks < kst; ++ks, ++g) {
          const int s = g % S;
          const uint32_t ph = static_cast<uint32_t>(g / S) & 1u;
          if (!wait_parity(bar(sm.empty[s]), ph ^ 1u, abort_flag, kGemmBudget)) {
            ok = false;
            break;
          }
          mbar_expect_tx(bar(sm.full[s]), static_cast<uint32_t>(hm) * a_bytes + (B_Q ? 0u : b_bytes));
          for (int m = 0; m < hm; ++m) tma_load_2d(a_at(s, m), &tmH, ks * kTileK, m * kTileM, bar(sm.full[s]));
          if (!B_Q) tma_load_2d(b_hi(s), &tmR, ks * kTileK, t * tn, bar(sm.full[s]));
        }
      }
      if (!ok) fail();
      // drain: the last stages issued have landed before the CTA can exit
      for (int j = std::max(0, g - S); j < g; ++j)
        wait_parity(bar(sm.full[j % S]), static_cast<uint32_t>(j / S) & 1u, abort_flag, kGemmBudget / 4);
    }
  } else if (B_Q && warp >= 8) {
    // ---------------- INT4 / INT8 dequantisation of the streamed rows (hi + lo bf16) ----------------
    // thread pair (2r, 2r + 1) handles row r of the tile, 32 elements each; the
    // codes of a stage are loaded before its slot is free
    const int dt = tid - 8 * 32;  // 0 .. kDequantThreads-1
    const int half = dt & 1;
    int g = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
      for (int ks = 0; ks < kst; ++ks, ++g) {
        const int s = g % S;
        const uint32_t ph = static_cast<uint32_t>(g / S) & 1u;
        const int e0 = ks * kTileK + 32 * half;  // this thread's 32 elements (one scale group)
        constexpr int kRowsPerPass = kDequantThreads / 2;
        const int nrow = tn / kRowsPerPass;  // 2 (tn 128) or 4 (tn 256)
        uint4 q[4], q2[4];  // q2: INT8 codes 16..31 of the group
        uint32_t scw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          q[i] = make_uint4(0, 0, 0, 0);
          q2[i] = make_uint4(0, 0, 0, 0);
          scw[i] = 0u;
          const int r = (dt >> 1) + i * kRowsPerPass;
          const int row = t * tn + r;
          if (i < nrow && row < P.rows && e0 < P.d) {
            const uint8_t* src = P.crows + static_cast<size_t>(row) * P.crow_bytes;
            if constexpr (FMT == kFmtInt4) {
              q[i] = *reinterpret_cast<const uint4*>(src + e0 / 2);
              scw[i] = *reinterpret_cast<const unsigned short*>(src + P.d / 2 + 2 * (e0 / 32));
            } else {
              q[i] = *reinterpret_cast<const uint4*>(src + e0);
              q2[i] = *reinterpret_cast<const uint4*>(src + e0 + 16);
              scw[i] = *reinterpret_cast<const unsigned short*>(src + P.d + 2 * (e0 / 32));
            }
          }
        }
        if (!wait_parity(bar(sm.empty[s]), ph ^ 1u, abort_flag, kGemmBudget)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (i >= nrow) break;
          const int r = (dt >> 1) + i * kRowsPerPass;
          const float scl = __uint_as_float(scw[i] << 16);
          const uint32_t qw[8] = {q[i].x, q[i].y, q[i].z, q[i].w, q2[i].x, q2[i].y, q2[i].z, q2[i].w};
          uint8_t* hi = gbase + (b_hi(s) - base) + r * 128;
          uint8_t* lo = gbase + (b_lo(s) - base) + r * 128;
#pragma unroll
          for (int j = 0; j < 4; ++j) {  // 16-byte chunk 4 half + j: elements 8j .. 8j+7 of the half
            uint32_t h[4], l[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float v0, v1;
              if constexpr (FMT == kFmtInt4) {
                v0 = nib(qw[j], 2 * e) * scl;
                v1 = nib(qw[j], 2 * e + 1) * scl;
              } else {  // elements 8j + 2e, 8j + 2e + 1: word 2j + e/2, bytes 2(e&1), 2(e&1) + 1
                const uint32_t wd = qw[2 * j + (e >> 1)];
                v0 = sbyte(wd, 2 * (e & 1)) * scl;
                v1 = sbyte(wd, 2 * (e & 1) + 1) * scl;
              }
              const __nv_bfloat162 hb = __floats2bfloat162_rn(v0, v1);
              const float2 hf = __bfloat1622float2(hb);
              const __nv_bfloat162 lb = __floats2bfloat162_rn(v0 - hf.x, v1 - hf.y);  // exact rest
              h[e] = *reinterpret_cast<const uint32_t*>(&hb);
              l[e] = *reinterpret_cast<const uint32_t*>(&lb);
            }
            const int pc = ((4 * half + j) ^ (r & 7)) * 16;  // 128-byte swizzle of the chunk in row r
            *reinterpret_cast<uint4*>(hi + pc) = make_uint4(h[0], h[1], h[2], h[3]);
            *reinterpret_cast<uint4*>(lo + pc) = make_uint4(l[0], l[1], l[2], l[3]);
          }
        }
        fence_proxy_async_smem();  // generic writes -> tensor core reads
        mbar_arrive(bar(sm.full[s]));
      }
    }
    if (!ok) fail();
  } else if (warp == 4) {
    // ---------------- MMA issuer ----------------
    const uint32_t idesc = idesc_bf16(kTileM, tn);
    int g = 0, lt = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x, ++lt) {
      const int buf = nbuf == 2 ? (lt & 1) : 0;
      const uint32_t aph = static_cast<uint32_t>(nbuf == 2 ? (lt >> 1) : lt) & 1u;
      if (!wait_parity(bar(sm.tempty[buf]), aph ^ 1u, abort_flag, kGemmBudget)) {
        ok = false;
        break;
      }
      tc_fence_after();
      for (int ks = 0; ks < kst; ++ks, ++g) {
        const int s = g % S;
        const uint32_t ph = static_cast<uint32_t>(g / S) & 1u;
        if (!wait_parity(bar(sm.full[s]), ph, abort_flag, kGemmBudget)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
#pragma unroll
          for (int k = 0; k < kTileK / 16; ++k) {  // 16 elements = 32 bytes per MMA along K
            const uint64_t bh = smem_desc_sw128(b_hi(s) + 32u * k);
            const uint64_t bl = smem_desc_sw128(b_lo(s) + 32u * k);
            for (int m = 0; m < hm; ++m) {
              const uint32_t dcol = tmem + static_cast<uint32_t>((buf * hm + m) * tn);
              const uint64_t ad = smem_desc_sw128(a_at(s, m) + 32u * k);
              mma_bf16(dcol, ad, bh, idesc, (ks | k) != 0);
              if (B_Q) mma_bf16(dcol, ad, bl, idesc, 1u);
            }
          }
          mma_commit(bar(sm.empty[s]));  // the stage is free once these MMAs have read it
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) mma_commit(bar(sm.tfull[buf]));  // the accumulators are complete
      __syncwarp();
    }
    if (!ok) fail();
    // every MMA this warp issued has finished before tensor memory is released
    if (lane == 0) mma_commit(bar(sm.done));
    __syncwarp();
    wait_parity(bar(sm.done), 0u, abort_flag, kGemmBudget / 4);
  } else if (warp < 4) {
    // ---------------- epilogue: one hidden row (TMEM lane) per thread ----------------
    const int q = warp;  // lanes 32q .. 32q+31 of every accumulator
    unsigned long long best[2] = {0ull, 0ull};
    int lt = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x, ++lt) {
      const int buf = nbuf == 2 ? (lt & 1) : 0;
      const uint32_t aph = static_cast<uint32_t>(nbuf == 2 ? (lt >> 1) : lt) & 1u;
      if (!wait_parity(bar(sm.tfull[buf]), aph, abort_flag, kGemmBudget)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        if (m >= hm) break;
        const int r = m * kTileM + q * 32 + lane;  // hidden row
        const bool rv = r < P.nb;
        for (int c0 = 0; c0 < tn; c0 += 16) {
          uint32_t v[16];
          tmem_ld16(tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>((buf * hm + m) * tn + c0), v);
          const int n0 = t * tn + c0;  // streamed row of v[0]
          if (!rv || n0 >= P.rows) continue;
          float* o = P.out ? P.out + static_cast<size_t>(r) * P.ldo + n0 : nullptr;
          const int nv = min(16, P.rows - n0);
          if (P.epi == 0) {
            if (P.mode == 1) {
              const float* u = P.u + static_cast<size_t>(r) * P.ldo + n0;
#pragma unroll
              for (int j = 0; j < 16; ++j)
                if (j < nv) o[j] = gumbel_key(__uint_as_float(v[j]), P.T, __ldg(u + j));
            } else if (nv == 16 && (reinterpret_cast<uintptr_t>(o) & 15) == 0) {
              float4* o4 = reinterpret_cast<float4*>(o);
#pragma unroll
              for (int j = 0; j < 4; ++j)
                o4[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                    __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j)
                if (j < nv) o[j] = __uint_as_float(v[j]);
            }
          } else {
            unsigned long long bm = best[m];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              if (j < nv) {
                const unsigned long long pk =
                    (static_cast<unsigned long long>(f2key(__uint_as_float(v[j]))) << 32) |
                    static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<uint32_t>(n0 + j));
                bm = pk > bm ? pk : bm;
              }
            }
            best[m] = bm;
            if (o) {
#pragma unroll
              for (int j = 0; j < 16; ++j)
                if (j < nv) o[j] = __uint_as_float(v[j]);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar(sm.tempty[buf]));
    }
    if (!ok) fail();
    if (P.epi == 1)
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        if (m >= hm) break;
        const int r = m * kTileM + q * 32 + lane;
        if (r < P.nb && best[m]) atomicMax(P.best + r, best[m]);
      }
  }

  __syncthreads();
  tc_fence_after();
  if (warp == 4)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(P.tmem_cols) : "memory");
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 tensor [rows, d] row-major; boxes of 64 x box_rows, 128-byte swizzle,
// zero fill outside the tensor.
bool make_map(CUtensorMap* map, const void* ptr, int rows, int d, int box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kTileK), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Stage plan: hm H blocks (16 KB each) + tn streamed rows (x2 for dequantised hi/lo) per stage.
size_t gemm_smem_bytes(int hm, int tn, int dequant, int* stages) {
  const size_t st = static_cast<size_t>(hm) * kTileM * kTileK * 2 + (dequant ? 2 : 1) * static_cast<size_t>(tn) * kTileK * 2;
  const size_t extra = sizeof(GemmSmem) + 1024;  // + alignment slack
  int s = 4;
  while (s > 2 && static_cast<size_t>(s) * st + extra > 227 * 1024) --s;
  *stages = s;
  return static_cast<size_t>(s) * st + extra;
}

cudaError_t launch_gemm(const GemmParams& P0, const void* rows_bf16, const void* H, int num_sms, cudaStream_t st) {
  GemmParams P = P0;
  if (P.nb < 1 || P.nb > kMaxN || P.d < 8 || P.rows < 1) return cudaErrorInvalidValue;
  P.hm = (P.nb + kTileM - 1) / kTileM;
  // 256 streamed rows per tile, or 128 when that leaves SMs idle
  P.tn = (P.rows + 255) / 256 >= num_sms ? 256 : 128;
  P.nbuf = P.hm * P.tn * 2 <= 512 ? 2 : 1;  // double-buffered accumulators when tensor memory allows
  P.tmem_cols = 32;
  while (P.tmem_cols < P.nbuf * P.hm * P.tn) P.tmem_cols *= 2;  // a power of two >= 32
  const size_t smem = gemm_smem_bytes(P.hm, P.tn, P.cfmt != kFmtBf16, &P.stages);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  CUtensorMap mh{}, mr{};
  if (!make_map(&mh, H, P.nb, P.d, kTileM)) return cudaErrorInvalidValue;
  if (P.cfmt != kFmtBf16) {
    mr = mh;  // unused: the streamed rows are read and dequantised by the kernel
  } else if (!make_map(&mr, rows_bf16, P.rows, P.d, P.tn)) {
    return cudaErrorInvalidValue;
  }
  const int ntiles = (P.rows + P.tn - 1) / P.tn;
  const int grid = std::min(num_sms, ntiles);
  if (P.cfmt == kFmtInt4) gemm_kernel<kFmtInt4><<<grid, kGemmThreads, smem, st>>>(mh, mr, P);
  else if (P.cfmt == kFmtInt8) gemm_kernel<kFmtInt8><<<grid, kGemmThreads, smem, st>>>(mh, mr, P);
  else gemm_kernel<kFmtBf16><<<grid, kGemmThreads, smem, st>>>(mh, mr, P);
  return cudaGetLastError();
}

cudaError_t set_attrs_gemm() {
  cudaError_t e = cudaFuncSetAttribute(gemm_kernel<kFmtInt4>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gemm_kernel<kFmtInt8>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gemm_kernel<kFmtBf16>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  return e;
}

}  // namespace fh
