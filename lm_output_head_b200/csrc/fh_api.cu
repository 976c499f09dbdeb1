// Host layer of the C ABI declared in include/fh.h: argument validation,
// workspace planning, shared-memory planning of each kernel, and dispatch.
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>

#include "fh_device.cuh"

namespace fh {
cudaError_t set_attrs_decode_b1(int max_smem);
cudaError_t set_attrs_batched(int max_smem);
cudaError_t set_attrs_dense(int max_smem);
int dense_max_rows();
cudaError_t occupancy_decode_b1(int cfmt, int nch, size_t smem, int* blocks);
size_t decode_b1_misc_bytes();
size_t decode_b1_scratch_bytes(int c, int list_cap);
cudaError_t occupancy_dense(int nch, size_t smem, int* blocks);

}  // namespace fh

using namespace fh;

struct fh_head {
  fh_head_desc desc;
  int device = 0;
  int num_sms = 0;
  size_t smem_budget = 0;  // dynamic shared memory the kernels may use
  uint8_t* ws = nullptr;
  size_t ws_bytes = 0;
  SyncWords* sync = nullptr;
  unsigned long long* best = nullptr;  // [max_batch]
  float* keys = nullptr;               // [max_batch, c]
  int32_t* sel = nullptr;              // [max_batch, max_probes]
  int32_t* cand_tok = nullptr;         // [max_batch, max_probes * b]
  float* cand_logits = nullptr;        // [max_batch, max_probes * b]
  int32_t* row_ok = nullptr;           // [max_batch]
  uint32_t* c2t_counts = nullptr;      // [v]
  uint16_t* Ecm = nullptr;             // [v, d] cluster-major copy of the token rows
  uint32_t* g_cnt = nullptr;           // de-duplication: [c] counts, [c] cursors, [c + 1] offsets
  uint32_t* g_cur = nullptr;
  uint32_t* g_off = nullptr;
  int32_t* g_ulist = nullptr;          // [c]
  int32_t* g_rows = nullptr;           // [max_batch * max_probes]
  uint32_t* g_next = nullptr;
  uint32_t* b1_keys = nullptr;         // fused B = 1 state
  float* b1_z_buf = nullptr;           // [c * b]
  uint32_t* b1_hist = nullptr;         // [kB1Bins]
  uint32_t* b1_list_key = nullptr;     // [b1_list_cap]
  int32_t* b1_list_id = nullptr;       // [b1_list_cap]
  int b1_list_cap = 0;
  B1Hot* b1_hot = nullptr;             // the fused call's shared counters
  C2TView c2t{};                       // the caller's C2T, int32 or uint16
  int words = 0;
  int b1_grid = 0;
  int dense_grid = 0;
  const uint8_t* crows = nullptr;      // centroid rows (bf16 borrowed, or packed INT4 / INT8 in ws)
  int crow_bytes = 0;
  int nch = 0;
  long long spin_budget = kDefaultSpinBudget;
  // fused B = 1 plan
  bool fused_ok = false;
  int b1_off_h = 0, b1_off_sel = 0, b1_off_misc = 0, b1_off_slots = 0, b1_slot_bytes = 0;
  size_t b1_smem = 0;
};

namespace {

constexpr size_t kAlign = 256;
inline size_t up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }


std::mutex g_attr_mu;
bool g_attr_done[64] = {};

fh_status cuda_fail(cudaError_t e) {
  (void)cudaGetLastError();
  return e == cudaErrorMemoryAllocation ? FH_ERR_OOM : FH_ERR_CUDA;
}

bool valid_mode(int32_t m) { return m == FH_GREEDY || m == FH_SAMPLE_GUMBEL; }

fh_status check_call(const fh_head* h, const void* hidden, int32_t B) {
  if (!h || !hidden) return FH_ERR_INVALID_ARG;
  if (!aligned(hidden, 16)) return FH_ERR_INVALID_ARG;
  if (B < 1 || B > h->desc.max_batch) return FH_ERR_INVALID_ARG;
  return FH_OK;
}

fh_status check_probe_args(const fh_head* h, int32_t p, int32_t mode, float T) {
  if (p < 1 || p > h->desc.max_probes || p > h->desc.c) return FH_ERR_INVALID_ARG;
  if (!valid_mode(mode)) return FH_ERR_INVALID_ARG;
  if (mode == FH_SAMPLE_GUMBEL && !(T > 0.f && T < 3.0e38f)) return FH_ERR_INVALID_ARG;
  return FH_OK;
}

// Per-warp ring plan: as many slots (<= 8) of `slot` bytes as fit after `fixed` bytes.
int ring_slots(size_t budget, size_t fixed, size_t slot) {
  if (fixed >= budget) return 0;
  const size_t n = (budget - fixed) / (static_cast<size_t>(kWarps) * slot);
  return static_cast<int>(n > 8 ? 8 : n);
}

fh_status launch_scores_rows(fh_head* h, const void* hidden, int32_t B, int mode, float T,
                             const float* u, float* out, cudaStream_t st) {
  const fh_head_desc& D = h->desc;
  const size_t slot = up(static_cast<size_t>(h->crow_bytes), 128);
  const int nslot = 2;
  const size_t ring = static_cast<size_t>(kWarps) * nslot * slot;
  const size_t off_bar = 0, off_ring = 1024;
  const size_t row_bytes = static_cast<size_t>(D.d) * 2;
  if (off_ring + ring + row_bytes > h->smem_budget) return FH_ERR_UNSUPPORTED;
  const int rmax = static_cast<int>((h->smem_budget - off_ring - ring) / row_bytes);
  for (int r0 = 0; r0 < B; r0 += rmax) {
    const int rows = B - r0 < rmax ? B - r0 : rmax;
    ScoresParams P{};
    P.Crows = h->crows;
    P.hidden = static_cast<const uint16_t*>(hidden);
    P.u_clusters = u;
    P.out = out;
    P.status = &h->sync->status;
    P.d = D.d;
    P.c = D.c;
    P.crow_bytes = h->crow_bytes;
    P.row0 = r0;
    P.rows = rows;
    P.mode = mode;
    P.T = T;
    P.nslot = nslot;
    P.slot_bytes = static_cast<int>(slot);
    P.off_bar = static_cast<int>(off_bar);
    P.off_ring = static_cast<int>(off_ring);
    P.off_h = static_cast<int>(off_ring + ring);
    const size_t smem = off_ring + ring + up(rows * row_bytes, 128);
    cudaError_t e = launch_scores(P, h->num_sms, smem, D.fmt, h->nch, st);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return FH_OK;
}

fh_status launch_candidates_rows(fh_head* h, const void* hidden, int32_t B, int32_t p,
                                 float* logits, int32_t* token_out, bool use_best,
                                 bool use_row_ok, cudaStream_t st) {
  const fh_head_desc& D = h->desc;
  const size_t slot = up(static_cast<size_t>(D.d) * 2, 128);
  const int nslot = ring_slots(h->smem_budget, 1024, slot);
  if (nslot < 1) return FH_ERR_UNSUPPORTED;
  CandParams P{};
  P.E = static_cast<const uint16_t*>(D.E);
  P.hidden = static_cast<const uint16_t*>(hidden);
  P.cand_tok = h->cand_tok;
  P.row_ok = use_row_ok ? h->row_ok : nullptr;
  P.logits = logits;
  P.token_out = token_out;
  P.best = use_best ? h->best : nullptr;
  P.status = &h->sync->status;
  P.v = D.v;
  P.d = D.d;
  P.nc = p * D.b;
  P.B = B;
  P.nslot = nslot;
  P.slot_bytes = static_cast<int>(slot);
  P.off_bar = 0;
  P.off_ring = 1024;
  const size_t smem = 1024 + static_cast<size_t>(kWarps) * nslot * slot;
  cudaError_t e = launch_candidates(P, h->num_sms, smem, h->nch, st);
  return e == cudaSuccess ? FH_OK : cuda_fail(e);
}

// Batches of at least this many hidden rows run the dense head on the tensor
// cores; smaller ones stream E on CUDA cores.
constexpr int kGemmMinBatch = 64;

// Centroid scores move to the tensor cores at a smaller batch: the CUDA-core
// kernel's time grows with B (one FMA per element and row) while the GEMM's is
// flat below 128 rows. Crossovers measured on B200 with a cold L2 (c 8016-9496,
// d 2048-2560): bf16 centroids 45 vs 34 us at B = 8; INT4 / INT8 centroids,
// dequantised to hi + lo pairs for the MMA, 32-36 vs 46 us at B = 8 and 54-58
// vs 46 us at B = 16.
int scores_gemm_min_batch(int fmt) { return fmt == FH_CENTROID_BF16 ? 8 : 16; }

// tcgen05 GEMM over blocks of up to 256 hidden rows. epi 0: out[r][k] =
// scores (mode 0) or Gumbel keys (mode 1) of A = the centroids; epi 1: packed
// (logit, token) maxima of A = E into h->best[r] (+ optional logits out[r][t]).
fh_status launch_gemm_rows(fh_head* h, const void* hidden, int32_t B, int epi, int mode, float T, const float* u,
                           float* out, cudaStream_t st) {
  const fh_head_desc& D = h->desc;
  const bool centroids = epi == 0;
  const int cfmt = centroids ? D.fmt : kFmtBf16;  // packed INT4 / INT8 centroid rows, or bf16 rows
  const int rows = centroids ? D.c : D.v;
  const long long ldo = rows;
  for (int r0 = 0; r0 < B; r0 += 256) {
    GemmParams P{};
    P.rows = rows;
    P.d = D.d;
    P.nb = std::min(256, B - r0);
    P.cfmt = cfmt;
    P.epi = epi;
    P.mode = mode;
    P.T = T;
    P.crows = h->crows;
    P.crow_bytes = h->crow_bytes;
    P.out = out ? out + static_cast<size_t>(r0) * ldo : nullptr;
    P.ldo = ldo;
    P.u = u ? u + static_cast<size_t>(r0) * ldo : nullptr;
    P.best = h->best + r0;
    P.status = &h->sync->status;
    const void* A = centroids ? (cfmt != kFmtBf16 ? nullptr : D.C) : D.E;
    const void* H = static_cast<const uint16_t*>(hidden) + static_cast<size_t>(r0) * D.d;
    cudaError_t e = launch_gemm(P, A, H, h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return FH_OK;
}

size_t select_smem(const fh_head* h, int32_t p) {
  return up(static_cast<size_t>(p) * 4, 128) + hist_select_smem_bytes(h->desc.c);
}

}  // namespace

extern "C" {

const char* fh_status_string(fh_status s) {
  switch (s) {
    case FH_OK: return "ok";
    case FH_ERR_INVALID_ARG: return "invalid argument";
    case FH_ERR_INVALID_C2T: return "C2T is not a permutation of 0..v-1";
    case FH_ERR_UNSUPPORTED: return "unsupported device or shape";
    case FH_ERR_OOM: return "out of device memory";
    case FH_ERR_CUDA: return "CUDA runtime error";
    case FH_ERR_OUT_OF_RANGE: return "cluster id out of range or repeated";
    case FH_ERR_TIMEOUT: return "bounded device wait ran out";
  }
  return "unknown status";
}

fh_status fh_create(const fh_head_desc* desc, fh_stream_t stream, fh_head** out) {
  if (!desc || !out) return FH_ERR_INVALID_ARG;
  *out = nullptr;
  const fh_head_desc D = *desc;
  if (D.v < 1 || D.d < 8 || D.c < 1 || D.b < 1) return FH_ERR_INVALID_ARG;
  if (static_cast<long long>(D.c) * D.b != D.v) return FH_ERR_INVALID_ARG;
  if (D.d % 8) return FH_ERR_INVALID_ARG;
  if (D.max_batch < 1 || D.max_probes < 1 || D.max_probes > D.c) return FH_ERR_INVALID_ARG;
  if (D.c2t_format != FH_C2T_INT32 && D.c2t_format != FH_C2T_UINT16) return FH_ERR_INVALID_ARG;
  const bool c2t16 = D.c2t_format == FH_C2T_UINT16;
  if (c2t16 && D.v > 65536) return FH_ERR_INVALID_ARG;  // token ids 0..v-1 must fit in 16 bits
  if (!D.E || !aligned(D.E, 16) || !D.C2T || !aligned(D.C2T, c2t16 ? 2 : 4)) return FH_ERR_INVALID_ARG;
  if (D.fmt == FH_CENTROID_BF16) {
    if (!D.C || !aligned(D.C, 16)) return FH_ERR_INVALID_ARG;
  } else if (D.fmt == FH_CENTROID_INT4_G32 || D.fmt == FH_CENTROID_INT8_G32) {
    if (D.d % 32 || !D.C_q || !D.C_scales || !aligned(D.C_scales, 2)) return FH_ERR_INVALID_ARG;
  } else {
    return FH_ERR_INVALID_ARG;
  }
  if (D.d > kMaxD) return FH_ERR_UNSUPPORTED;  // kMaxD <= 4 * kThreads: h widens in one round

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaDeviceProp prop;
  e = cudaGetDeviceProperties(&prop, dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (prop.major != 10) return FH_ERR_UNSUPPORTED;

  fh_head* h = new (std::nothrow) fh_head();
  if (!h) return FH_ERR_OOM;
  h->desc = D;
  h->c2t = C2TView::make(D.C2T, c2t16);
  h->device = dev;
  h->num_sms = prop.multiProcessorCount;
  // leave room for the kernels' static shared memory
  h->smem_budget = static_cast<size_t>(prop.sharedMemPerBlockOptin) - 8192;
  h->nch = nch_for(D.d);
  if (D.fmt == FH_CENTROID_INT4_G32) {
    h->crow_bytes = static_cast<int>(up(static_cast<size_t>(D.d) / 2 + static_cast<size_t>(D.d) / 16, 16));
  } else if (D.fmt == FH_CENTROID_INT8_G32) {
    h->crow_bytes = static_cast<int>(up(static_cast<size_t>(D.d) + static_cast<size_t>(D.d) / 16, 16));
  } else {
    h->crow_bytes = D.d * 2;
  }

  // ---- workspace plan ----
  const size_t mb = D.max_batch, mp = D.max_probes, nc = mp * D.b;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = up(off + bytes, kAlign);
    return o;
  };
  const size_t o_sync = take(sizeof(SyncWords));
  const size_t o_best = take(mb * 8);
  const size_t o_keys = take(mb * D.c * 4);
  const size_t o_sel = take(mb * mp * 4);
  const size_t o_tok = take(mb * nc * 4);
  const size_t o_log = take(mb * nc * 4);
  const size_t o_rok = take(mb * 4);
  const size_t o_cnt = take(static_cast<size_t>(D.v) * 4);
  const size_t o_ecm = take(static_cast<size_t>(D.v) * D.d * 2);
  const size_t o_gcnt = take(static_cast<size_t>(D.c) * 4);
  const size_t o_gcur = take(static_cast<size_t>(D.c) * 4);
  const size_t o_goff = take(static_cast<size_t>(D.c + 1) * 4);
  const size_t o_gul = take(static_cast<size_t>(D.c) * 4);
  const size_t o_grows = take(mb * mp * 4);
  const size_t o_gnext = take(16);
  const int words = (D.c + 31) / 32;
  const size_t o_keys1 = take(static_cast<size_t>(D.c) * 4);
  const size_t o_zbuf = take(static_cast<size_t>(D.v) * 4);
  // predicted-region histogram of the fused decode
  const size_t o_hist1 = take(static_cast<size_t>(kB1Bins) * 4);
  // candidate list of the fused decode: up to 4 p entries (the region aims at ~2 p keys)
  const int list_cap = static_cast<int>(std::min<size_t>(4 * mp, D.c));
  const size_t o_lkey = take(static_cast<size_t>(list_cap) * 4);
  const size_t o_lid = take(static_cast<size_t>(list_cap) * 4);
  const size_t o_hot = take(sizeof(B1Hot));
  const bool packed = D.fmt != FH_CENTROID_BF16;
  const size_t o_crow = packed ? take(static_cast<size_t>(D.c) * h->crow_bytes) : 0;
  h->ws_bytes = off;

  const char* cap = std::getenv("FH_TEST_WORKSPACE_LIMIT");
  if (cap && static_cast<size_t>(std::strtoull(cap, nullptr, 10)) < h->ws_bytes) {
    delete h;
    return FH_ERR_OOM;
  }
  e = cudaMalloc(reinterpret_cast<void**>(&h->ws), h->ws_bytes);
  if (e != cudaSuccess) {
    delete h;
    return cuda_fail(e);
  }
  h->sync = reinterpret_cast<SyncWords*>(h->ws + o_sync);
  h->best = reinterpret_cast<unsigned long long*>(h->ws + o_best);
  h->keys = reinterpret_cast<float*>(h->ws + o_keys);
  h->sel = reinterpret_cast<int32_t*>(h->ws + o_sel);
  h->cand_tok = reinterpret_cast<int32_t*>(h->ws + o_tok);
  h->cand_logits = reinterpret_cast<float*>(h->ws + o_log);
  h->row_ok = reinterpret_cast<int32_t*>(h->ws + o_rok);
  h->c2t_counts = reinterpret_cast<uint32_t*>(h->ws + o_cnt);
  h->Ecm = reinterpret_cast<uint16_t*>(h->ws + o_ecm);
  h->g_cnt = reinterpret_cast<uint32_t*>(h->ws + o_gcnt);
  h->g_cur = reinterpret_cast<uint32_t*>(h->ws + o_gcur);
  h->g_off = reinterpret_cast<uint32_t*>(h->ws + o_goff);
  h->g_ulist = reinterpret_cast<int32_t*>(h->ws + o_gul);
  h->g_rows = reinterpret_cast<int32_t*>(h->ws + o_grows);
  h->g_next = reinterpret_cast<uint32_t*>(h->ws + o_gnext);
  h->b1_keys = reinterpret_cast<uint32_t*>(h->ws + o_keys1);
  h->b1_z_buf = reinterpret_cast<float*>(h->ws + o_zbuf);
  h->b1_hist = reinterpret_cast<uint32_t*>(h->ws + o_hist1);
  h->b1_list_key = reinterpret_cast<uint32_t*>(h->ws + o_lkey);
  h->b1_list_id = reinterpret_cast<int32_t*>(h->ws + o_lid);
  h->b1_list_cap = list_cap;
  h->b1_hot = reinterpret_cast<B1Hot*>(h->ws + o_hot);
  h->words = words;
  h->crows = packed ? h->ws + o_crow : static_cast<const uint8_t*>(D.C);

  fh_status status = FH_OK;
  do {
    {
      std::lock_guard<std::mutex> lk(g_attr_mu);
      if (dev < 64 && !g_attr_done[dev]) {
        const int ms = static_cast<int>(h->smem_budget);
        e = set_attrs_decode_b1(ms);
        if (e == cudaSuccess) e = set_attrs_batched(ms);
        if (e == cudaSuccess) e = set_attrs_dense(ms);
        if (e == cudaSuccess) e = set_attrs_gemm();
        if (e == cudaSuccess) e = set_attrs_group();
        if (e != cudaSuccess) {
          status = cuda_fail(e);
          break;
        }
        g_attr_done[dev] = true;
      }
    }
    e = cudaMemsetAsync(h->ws, 0, h->ws_bytes, st);
    if (e != cudaSuccess) { status = cuda_fail(e); break; }
    C2TCheckParams cp{h->c2t, h->c2t_counts, &h->sync->status, static_cast<long long>(D.v), D.v};
    e = launch_c2t_check(cp, st);
    if (e != cudaSuccess) { status = cuda_fail(e); break; }
    if (packed) {
      RepackParams rp{D.C_q, static_cast<const uint16_t*>(D.C_scales), h->ws + o_crow, D.c, D.d, h->crow_bytes,
                      D.fmt == FH_CENTROID_INT8_G32 ? D.d : D.d / 2};
      e = launch_repack(rp, st);
      if (e != cudaSuccess) { status = cuda_fail(e); break; }
    }
    int bad = 0;
    e = cudaMemcpyAsync(&bad, &h->sync->status, sizeof(int), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) { status = cuda_fail(e); break; }
    if (bad) { status = FH_ERR_INVALID_C2T; break; }
    // token rows in cluster-major order (C2T is a permutation: every read is in range)
    e = launch_gather_cluster_major(static_cast<const uint16_t*>(D.E), h->c2t, h->Ecm, D.v, D.d, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) { status = cuda_fail(e); break; }
  } while (false);
  if (status != FH_OK) {
    cudaFree(h->ws);
    delete h;
    return status;
  }

  // ---- fused B = 1 plan: h (fp32), selection list, misc, per-warp row slots ----
  {
    size_t o = 0;
    h->b1_off_h = static_cast<int>(o);
    o += up(static_cast<size_t>(D.d) * 4, 128);
    h->b1_off_sel = static_cast<int>(o);
    o += up(static_cast<size_t>(D.max_probes) * 4, 128);
    h->b1_off_misc = static_cast<int>(o);
    o += up(decode_b1_misc_bytes(), 128);
    h->b1_off_slots = static_cast<int>(o);
    h->b1_slot_bytes = static_cast<int>(up(std::max(static_cast<size_t>(h->crow_bytes), static_cast<size_t>(D.d) * 2), 128));
    // the slots double as the selection's scratch between the phases
    o += std::max(static_cast<size_t>(kWarps) * h->b1_slot_bytes, decode_b1_scratch_bytes(D.c, h->b1_list_cap));
    h->b1_smem = o;
    int blocks = 0;
    e = occupancy_decode_b1(D.fmt, h->nch, h->b1_smem, &blocks);
    (void)cudaGetLastError();
    const int per_sm = e == cudaSuccess ? std::min(blocks, 2) : 0;
    h->b1_grid = per_sm * h->num_sms;
    // each warp owns at most 32 clusters (one key per lane register)
    h->fused_ok = per_sm >= 1 && D.c <= 32LL * h->b1_grid * kWarps;
  }
  {
    int blocks = 0;
    e = occupancy_dense(h->nch, static_cast<size_t>(dense_max_rows()) * D.d * 4, &blocks);
    (void)cudaGetLastError();
    h->dense_grid = (e == cudaSuccess && blocks >= 1 ? std::min(blocks, 2) : 1) * h->num_sms;
  }
  *out = h;
  return FH_OK;
}

void fh_destroy(fh_head* h) {
  if (!h) return;
  cudaDeviceSynchronize();
  cudaFree(h->ws);
  delete h;
}

fh_status fh_set_spin_budget(fh_head* h, int64_t cycles) {
  if (!h || cycles < 0) return FH_ERR_INVALID_ARG;
  h->spin_budget = cycles;
  return FH_OK;
}

fh_status fh_query(fh_head* h, int32_t key, int64_t* value) {
  if (!h || !value) return FH_ERR_INVALID_ARG;
  switch (key) {
    case FH_QUERY_WORKSPACE_BYTES: *value = static_cast<int64_t>(h->ws_bytes); return FH_OK;
    case FH_QUERY_LAST_UNION: {
      uint32_t u = 0;
      cudaError_t e = cudaMemcpy(&u, &h->sync->union_count, 4, cudaMemcpyDeviceToHost);
      if (e != cudaSuccess) return cuda_fail(e);
      *value = u;
      return FH_OK;
    }
    case FH_QUERY_LAST_LIST:
    case FH_QUERY_LAST_FULL: {
      uint32_t u = 0;
      const uint32_t* src = key == FH_QUERY_LAST_LIST ? &h->sync->last_in_range : &h->sync->last_full;
      cudaError_t e = cudaMemcpy(&u, src, 4, cudaMemcpyDeviceToHost);
      if (e != cudaSuccess) return cuda_fail(e);
      *value = u;
      return FH_OK;
    }
    case FH_QUERY_NUM_SMS: *value = h->num_sms; return FH_OK;
    case FH_QUERY_FUSED_B1: *value = h->fused_ok ? 1 : 0; return FH_OK;
  }
  return FH_ERR_INVALID_ARG;
}

fh_status fh_get_device_status(fh_head* h, fh_stream_t stream) {
  if (!h) return FH_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int s = 0;
  cudaError_t e = cudaMemcpyAsync(&s, &h->sync->status, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e);
  if (s) {
    e = cudaMemsetAsync(&h->sync->status, 0, sizeof(int), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return static_cast<fh_status>(s);
}

fh_status fh_centroid_scores(fh_head* h, const void* hidden, int32_t B, float* scores, fh_stream_t stream) {
  fh_status s = check_call(h, hidden, B);
  if (s != FH_OK) return s;
  if (!scores || !aligned(scores, 4)) return FH_ERR_INVALID_ARG;
  if (B >= scores_gemm_min_batch(h->desc.fmt))
    return launch_gemm_rows(h, hidden, B, 0, 0, 1.f, nullptr, scores, reinterpret_cast<cudaStream_t>(stream));
  return launch_scores_rows(h, hidden, B, 0, 1.f, nullptr, scores, reinterpret_cast<cudaStream_t>(stream));
}

fh_status fh_select_clusters(fh_head* h, const float* scores, int32_t B, int32_t p, int32_t mode, float T,
                             const float* u_clusters, int32_t* cluster_ids, fh_stream_t stream) {
  if (!h || !scores || !cluster_ids) return FH_ERR_INVALID_ARG;
  if (B < 1 || B > h->desc.max_batch) return FH_ERR_INVALID_ARG;
  fh_status s = check_probe_args(h, p, mode, T);
  if (s != FH_OK) return s;
  if (mode == FH_SAMPLE_GUMBEL && !u_clusters) return FH_ERR_INVALID_ARG;
  SelectParams P{};
  P.in = scores;
  P.u_clusters = mode == FH_SAMPLE_GUMBEL ? u_clusters : nullptr;
  P.C2T = h->c2t;
  P.sel = cluster_ids;
  P.status = &h->sync->status;
  P.c = h->desc.c;
  P.b = h->desc.b;
  P.p = p;
  P.perturb = mode == FH_SAMPLE_GUMBEL;
  P.T = T;
  const size_t smem = select_smem(h, p);
  if (smem > h->smem_budget) return FH_ERR_UNSUPPORTED;
  cudaError_t e = launch_select(P, B, smem, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FH_OK : cuda_fail(e);
}

fh_status fh_candidate_logits(fh_head* h, const void* hidden, int32_t B, int32_t p, const int32_t* cluster_ids,
                              int32_t* token_ids, float* logits, fh_stream_t stream) {
  fh_status s = check_call(h, hidden, B);
  if (s != FH_OK) return s;
  if (p < 1 || p > h->desc.max_probes) return FH_ERR_INVALID_ARG;
  if (!cluster_ids || !token_ids || !logits) return FH_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  SelectParams P{};
  P.ids_in = cluster_ids;
  P.C2T = h->c2t;
  P.sel = h->sel;
  P.cand_tok = h->cand_tok;
  P.row_ok = h->row_ok;
  P.status = &h->sync->status;
  P.c = h->desc.c;
  P.b = h->desc.b;
  P.p = p;
  const size_t smem = up(static_cast<size_t>((h->desc.c + 31) / 32) * 4, 128) + up(static_cast<size_t>(p) * 4, 128) +
                      kWarps * 4;
  if (smem > h->smem_budget) return FH_ERR_UNSUPPORTED;
  cudaError_t e = launch_sort_ids(P, B, smem, st);
  if (e != cudaSuccess) return cuda_fail(e);
  return launch_candidates_rows(h, hidden, B, p, logits, token_ids, false, true, st);
}

fh_status fh_decode(fh_head* h, const void* hidden, int32_t B, int32_t p, int32_t mode, float T,
                    const float* u_clusters, const float* u_token, int32_t* out_tokens, int32_t* out_cluster_ids,
                    float* out_max_logit, fh_stream_t stream) {
  fh_status s = check_call(h, hidden, B);
  if (s != FH_OK) return s;
  s = check_probe_args(h, p, mode, T);
  if (s != FH_OK) return s;
  if (!out_tokens) return FH_ERR_INVALID_ARG;
  if (mode == FH_SAMPLE_GUMBEL && (!u_clusters || !u_token)) return FH_ERR_INVALID_ARG;
  const fh_head_desc& D = h->desc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool gumbel = mode == FH_SAMPLE_GUMBEL;

  if (B == 1 && h->fused_ok) {
    B1Params P{};
    P.E = static_cast<const uint16_t*>(D.E);
    P.Ecm = h->Ecm;
    P.Crows = h->crows;
    P.C2T = h->c2t;
    P.hidden = static_cast<const uint16_t*>(hidden);
    P.u_clusters = gumbel ? u_clusters : nullptr;
    P.u_token = gumbel ? u_token : nullptr;
    P.out_tokens = out_tokens;
    P.out_cluster_ids = out_cluster_ids;
    P.out_max_logit = out_max_logit;
    P.keys = h->b1_keys;
    P.z_buf = h->b1_z_buf;
    P.hist = h->b1_hist;
    P.list_key = h->b1_list_key;
    P.list_id = h->b1_list_id;
    P.list_cap = h->b1_list_cap;
    P.hot = h->b1_hot;
    P.sync = h->sync;
    P.v = D.v;
    P.d = D.d;
    P.c = D.c;
    P.b = D.b;
    P.p = p;
    P.crow_bytes = h->crow_bytes;
    P.mode = mode;
    P.T = gumbel ? T : 1.f;
    P.off_h = h->b1_off_h;
    P.off_sel = h->b1_off_sel;
    P.off_misc = h->b1_off_misc;
    P.off_slots = h->b1_off_slots;
    P.slot_bytes = h->b1_slot_bytes;
    P.spin_budget = h->spin_budget;
    cudaError_t e = launch_decode_b1(P, h->b1_grid, h->b1_smem, D.fmt, h->nch, st);
    return e == cudaSuccess ? FH_OK : cuda_fail(e);
  }

  // batched path: keys -> per-row select -> candidates -> epilogue
  s = B >= scores_gemm_min_batch(D.fmt)
          ? launch_gemm_rows(h, hidden, B, 0, gumbel ? 1 : 0, gumbel ? T : 1.f, u_clusters, h->keys, st)
          : launch_scores_rows(h, hidden, B, gumbel ? 1 : 0, gumbel ? T : 1.f, u_clusters, h->keys, st);
  if (s != FH_OK) return s;
  SelectParams SP{};
  SP.in = h->keys;
  SP.C2T = h->c2t;
  SP.sel = h->sel;
  SP.cand_tok = h->cand_tok;
  SP.status = &h->sync->status;
  SP.c = D.c;
  SP.b = D.b;
  SP.p = p;
  SP.perturb = 0;
  const size_t ssm = select_smem(h, p);
  if (ssm > h->smem_budget) return FH_ERR_UNSUPPORTED;
  cudaError_t e = launch_select(SP, B, ssm, st);
  if (e != cudaSuccess) return cuda_fail(e);
  if (D.b == 16) {
    // de-duplicated across the batch: every chosen cluster's token rows are read once
    GroupParams GP{};
    GP.sel = h->sel;
    GP.C2T = h->c2t;
    GP.Ecm = h->Ecm;
    GP.H = static_cast<const uint16_t*>(hidden);
    GP.cnt = h->g_cnt;
    GP.cur = h->g_cur;
    GP.off = h->g_off;
    GP.ulist = h->g_ulist;
    GP.rows_of = h->g_rows;
    GP.union_count = &h->sync->union_count;
    GP.next = h->g_next;
    GP.best = h->best;
    GP.logits = gumbel ? h->cand_logits : nullptr;
    GP.B = B;
    GP.p = p;
    GP.c = D.c;
    GP.b = D.b;
    GP.d = D.d;
    e = launch_group(GP, h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e);
  } else {
    s = launch_candidates_rows(h, hidden, B, p, gumbel ? h->cand_logits : nullptr, nullptr, true, false, st);
    if (s != FH_OK) return s;
  }
  EpilogueParams EP{};
  EP.logits = h->cand_logits;
  EP.cand_tok = h->cand_tok;
  EP.u_token = u_token;
  EP.best = h->best;
  EP.out_tokens = out_tokens;
  EP.out_max_logit = out_max_logit;
  EP.nc = p * D.b;
  EP.mode = mode;
  EP.T = gumbel ? T : 1.f;
  e = launch_epilogue(EP, B, st);
  if (e != cudaSuccess) return cuda_fail(e);
  if (out_cluster_ids) {
    e = cudaMemcpyAsync(out_cluster_ids, h->sel, static_cast<size_t>(B) * p * 4, cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return FH_OK;
}

fh_status fh_dense_head(fh_head* h, const void* hidden, int32_t B, float* logits, int32_t* out_argmax,
                        fh_stream_t stream) {
  fh_status s = check_call(h, hidden, B);
  if (s != FH_OK) return s;
  if (!out_argmax) return FH_ERR_INVALID_ARG;
  const fh_head_desc& D = h->desc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (B >= kGemmMinBatch) {
    // tensor cores: fused column argmax into h->best, then one word per row out
    s = launch_gemm_rows(h, hidden, B, 1, 0, 1.f, nullptr, logits, st);
    if (s != FH_OK) return s;
    EpilogueParams EP{};
    EP.best = h->best;
    EP.out_tokens = out_argmax;
    EP.mode = 0;
    EP.T = 1.f;
    cudaError_t e = launch_epilogue(EP, B, st);
    return e == cudaSuccess ? FH_OK : cuda_fail(e);
  }
  const int rmax = dense_max_rows();
  for (int r0 = 0; r0 < B; r0 += rmax) {
    const int rows = B - r0 < rmax ? B - r0 : rmax;
    DenseParams P{};
    P.E = static_cast<const uint16_t*>(D.E);
    P.hidden = static_cast<const uint16_t*>(hidden);
    P.logits = logits;
    P.out_argmax = out_argmax;
    P.best = h->best;
    P.sync = h->sync;
    P.v = D.v;
    P.d = D.d;
    P.row0 = r0;
    P.rows = rows;
    const size_t smem = static_cast<size_t>(rows) * D.d * 4;
    cudaError_t e = launch_dense(P, h->dense_grid, smem, h->nch, st);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return FH_OK;
}

fh_status fh_speculative_verify(fh_head* h, const float* logits, const int32_t* cand_tokens, int32_t n, int32_t B,
                                const int32_t* draft, float T, const float* u_accept, const float* u_resample,
                                int32_t* out_tokens, fh_stream_t stream) {
  if (!h || !logits || !cand_tokens || !draft || !u_accept || !u_resample || !out_tokens) return FH_ERR_INVALID_ARG;
  if (B < 1 || n < 1 || n > h->desc.v || !(T > 0.f && T < 3.0e38f)) return FH_ERR_INVALID_ARG;
  cudaError_t e = launch_spec_verify(logits, h->desc.v, cand_tokens, n, B, draft, T, u_accept, u_resample, out_tokens,
                                     &h->sync->status, reinterpret_cast<cudaStream_t>(stream));
  if (e == cudaErrorInvalidValue) {
    (void)cudaGetLastError();
    return FH_ERR_UNSUPPORTED;
  }
  return e == cudaSuccess ? FH_OK : cuda_fail(e);
}

fh_status fh_adaptive_probes(fh_head* h, const float* scores, int32_t B, float tau, int32_t p_min, int32_t p_max,
                             float T, int32_t* out_p, fh_stream_t stream) {
  if (!h || !scores || !out_p || B < 1) return FH_ERR_INVALID_ARG;
  if (!(tau > 0.f && tau <= 1.f) || p_min < 1 || p_min > p_max || p_max > h->desc.c) return FH_ERR_INVALID_ARG;
  if (!(T > 0.f && T < 3.0e38f)) return FH_ERR_INVALID_ARG;
  cudaError_t e = launch_adaptive_probes(scores, B, h->desc.c, tau, p_min, p_max, T, out_p,
                                         reinterpret_cast<cudaStream_t>(stream));
  if (e == cudaErrorInvalidValue) {
    (void)cudaGetLastError();
    return FH_ERR_UNSUPPORTED;
  }
  return e == cudaSuccess ? FH_OK : cuda_fail(e);
}

fh_status fh_prefetch_clusters(fh_head* h, const int32_t* cluster_ids, int32_t n, fh_stream_t stream) {
  if (!h || n < 0 || (n > 0 && !cluster_ids)) return FH_ERR_INVALID_ARG;
  cudaError_t e = launch_prefetch_clusters(h->Ecm, h->c2t, h->desc.c, h->desc.b, h->desc.d, cluster_ids, n,
                                           &h->sync->status, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FH_OK : cuda_fail(e);
}

}  // extern "C"
