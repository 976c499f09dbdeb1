// Internal declarations shared by the host layer and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "fh.h"

namespace fh {

// Largest hidden size the register-resident kernels handle: each lane keeps
// ceil(d/256) 16-byte chunks of h (8 fp32 each) in registers.
constexpr int kMaxD = 2560;
constexpr long long kWaitBudget = 4000000000LL;      // bulk-copy waits (~2 s)
constexpr long long kDefaultSpinBudget = 2000000000LL;  // device-wide waits (~1 s)
constexpr int kB1Bins = 2048;  // histogram bins of the fused B = 1 selection's predicted region

// Centroid row formats as the kernels see them (the same values as fh_centroid_format):
// bf16 rows; packed INT4 g32 rows [d/2 codes][d/16 scale bytes]; packed INT8 g32 rows
// [d codes][d/16 scale bytes] (packed rows padded to 16 bytes).
constexpr int kFmtBf16 = 0, kFmtInt4 = 1, kFmtInt8 = 2;

// The caller's cluster-to-token map C2T [c, b] (write-up section 1.2.1):
// int32 entries, or uint16 entries when v <= 65536 (the compact map). One
// word: the map's address, with bit 0 set for uint16 entries (every map is at
// least 2-byte aligned), so a kernel holds it in one register pair.
struct C2TView {
  uintptr_t bits;
  static C2TView make(const void* ptr, bool u16) {
    return C2TView{reinterpret_cast<uintptr_t>(ptr) | (u16 ? 1u : 0u)};
  }
#ifdef __CUDACC__
  __device__ __forceinline__ int32_t at(size_t q) const {
    const uintptr_t a = bits & ~static_cast<uintptr_t>(1);
    return (bits & 1u) ? static_cast<int32_t>(__ldg(reinterpret_cast<const unsigned short*>(a) + q))
                       : __ldg(reinterpret_cast<const int32_t*>(a) + q);
  }
  __device__ __forceinline__ const void* ptr() const {
    return reinterpret_cast<const void*>(bits & ~static_cast<uintptr_t>(1));
  }
  __device__ __forceinline__ size_t elem_bytes() const { return (bits & 1u) ? 2u : 4u; }
#endif
};

// Workspace words at the start of the workspace.
struct SyncWords {
  int32_t status;
  uint32_t arrive;        // batched decode: grid barrier arrivals (unused by the fused call)
  uint32_t ticket;        // kernel exit tickets (last CTA finalises)
  uint32_t union_count;   // distinct clusters of the last batched decode
  uint32_t epoch;         // fused B = 1 calls so far
  uint32_t last_full;     // 1 if the last fused call selected without its histogram
  float prior_p[2];       // fused call: keys of rank p and 2p in the last call of each mode
  float prior_2p[2];      //   [greedy: key / |h|, sampling: key]
  uint32_t prior_ok[2];   // the predictions of a mode hold values
  float prior_T[2];       // the temperature and probe count they were taken at
  int32_t prior_pc[2];
  uint32_t last_in_range; // keys the last fused call counted in its histogram
};

// Counters that every CTA of a fused B = 1 call updates or polls, each on a
// 128-byte line of its own (workspace; zero between calls). The arrival count
// and the candidate list's length share one 64-bit word: a CTA reserves its
// list entries (low half) before it arrives (high half), so the poll that sees
// the last arrival also reads the final length.
struct B1Hot {
  alignas(128) unsigned long long arrive_list;  // CTAs arrived << 32 | list entries reserved
  alignas(128) uint32_t ticket;          // exit tickets (the last CTA finalises)
  alignas(128) unsigned long long best;  // packed (logit, token) maximum over the candidates
};

struct B1Params {
  const uint16_t* E;
  const uint16_t* Ecm;    // cluster-major token rows: row k*b + j = E[C2T[k][j]]
  const uint8_t* Crows;   // bf16 rows (d*2 bytes) or packed INT4 / INT8 rows (crow_bytes)
  C2TView C2T;
  const uint16_t* hidden;
  const float* u_clusters;
  const float* u_token;
  int32_t* out_tokens;
  int32_t* out_cluster_ids;
  float* out_max_logit;
  uint32_t* keys;         // workspace [c]: order-preserving keys of the clusters
  float* z_buf;           // workspace [c*b]: logit of slot k*b + j of the scored clusters (sampling)
  uint32_t* hist;         // workspace [kB1Bins]: counts of keys per bin of the predicted region
  uint32_t* list_key;     // workspace [list_cap]: keys in the predicted region (candidate list)
  int32_t* list_id;       // workspace [list_cap]: their cluster ids
  int list_cap;
  B1Hot* hot;
  SyncWords* sync;
  int v, d, c, b, p;
  int crow_bytes;
  int mode;
  float T;
  int off_h, off_sel, off_misc, off_slots, slot_bytes;
  long long spin_budget;
};

struct ScoresParams {
  const uint8_t* Crows;
  const uint16_t* hidden;  // [B, d]
  const float* u_clusters; // [B, c] (gumbel)
  float* out;              // [B, c]
  int*  status;
  int d, c, crow_bytes;
  int row0, rows;          // hidden rows [row0, row0+rows) in this launch
  int mode;                // 0 raw scores, 1 Gumbel keys
  float T;
  int nslot, slot_bytes;
  int off_h, off_bar, off_ring;
};

struct SelectParams {
  const float* in;         // [B, c] scores or keys
  const float* u_clusters; // [B, c] when perturb
  const int32_t* ids_in;   // [B, p] explicit ids (sort mode) or null
  C2TView C2T;
  int32_t* sel;            // [B, p] ascending
  int32_t* cand_tok;       // [B, p*b] canonical token ids, or null
  int32_t* row_ok;         // [B] (sort mode) or null
  int*  status;
  int c, b, p;
  int perturb;             // compute Gumbel keys from scores + u
  float T;
};

struct CandParams {
  const uint16_t* E;
  const uint16_t* hidden;   // [B, d]
  const int32_t* cand_tok;  // [B, p*b]
  const int32_t* row_ok;    // [B] or null
  float* logits;            // [B, p*b] or null
  int32_t* token_out;       // [B, p*b] or null
  unsigned long long* best; // [B] or null
  int*  status;
  int v, d, nc, B;
  int nslot, slot_bytes;
  int off_bar, off_ring;
};

struct EpilogueParams {
  const float* logits;      // [B, nc]
  const int32_t* cand_tok;  // [B, nc]
  const float* u_token;
  unsigned long long* best; // [B]
  int32_t* out_tokens;
  float* out_max_logit;
  int nc, mode;
  float T;
};

struct DenseParams {
  const uint16_t* E;
  const uint16_t* hidden;   // [B, d]
  float* logits;            // [B, v] or null
  int32_t* out_argmax;      // [B]
  unsigned long long* best; // [B]
  SyncWords* sync;
  int v, d;
  int row0, rows;
  int nslot, slot_bytes;
  int off_h, off_bar, off_ring;
};

struct GemmParams {
  int rows, d;              // streamed operand: rows x d (centroid or token rows), K = d
  int nb;                   // hidden rows of this launch, 1..256 (two M blocks of 128)
  int hm, tn, nbuf, stages, tmem_cols;  // set by the launcher
  int cfmt;                 // streamed operand: kFmtBf16 rows through TMA, or packed INT4 / INT8 rows (crows)
  int epi;                  // 0: store scores / keys, 1: per-hidden-row argmax
  int mode;                 // epi 0: 0 raw scores, 1 Gumbel keys
  float T;
  const uint8_t* crows;
  int crow_bytes;
  float* out;               // [nb, ldo]: scores/keys (epi 0) or logits (epi 1, may be null)
  long long ldo;
  const float* u;           // [nb, ldo] Gumbel uniforms (epi 0, mode 1)
  unsigned long long* best; // [nb] packed (logit, token) maxima (epi 1)
  int* status;
};

struct GroupParams {
  const int32_t* sel;       // [B, p] chosen clusters per row, ascending
  C2TView C2T;              // [c, b]
  const uint16_t* Ecm;      // [v, d] cluster-major token rows: row k*b + j = E[C2T[k][j]]
  const uint16_t* H;        // [B, d]
  uint32_t* cnt;            // [c] workspace: rows per cluster
  uint32_t* cur;            // [c] workspace: fill cursors
  uint32_t* off;            // [c + 1] workspace: CSR offsets
  int32_t* ulist;           // [c] workspace: the union of chosen clusters, ascending
  int32_t* rows_of;         // [B * p] workspace: rows of each cluster, grouped by cluster
  uint32_t* union_count;    // |union|
  uint32_t* next;           // work counter of the grouped kernel
  unsigned long long* best; // [B] packed (logit, token) maxima
  float* logits;            // [B, p*b] canonical candidate logits (sampling), or null
  int B, p, c, b, d;
};

struct C2TCheckParams {
  C2TView C2T;
  uint32_t* counts;         // [v]
  int* bad;
  long long n;
  int v;
};

struct RepackParams {
  const uint8_t* C_q;
  const uint16_t* C_scales;
  uint8_t* out;
  int c, d, rs;
  int qb;                   // code bytes per row: d / 2 (INT4) or d (INT8)
};

// Launchers (defined in the .cu files). Each returns the CUDA error of the launch.
cudaError_t launch_decode_b1(const B1Params& P, int grid, size_t smem, int cfmt, int nch,
                             cudaStream_t st);
cudaError_t launch_scores(const ScoresParams& P, int grid, size_t smem, int cfmt, int nch,
                          cudaStream_t st);
cudaError_t launch_select(const SelectParams& P, int B, size_t smem, cudaStream_t st);
cudaError_t launch_sort_ids(const SelectParams& P, int B, size_t smem, cudaStream_t st);
cudaError_t launch_candidates(const CandParams& P, int grid, size_t smem, int nch, cudaStream_t st);
cudaError_t launch_epilogue(const EpilogueParams& P, int B, cudaStream_t st);
cudaError_t launch_dense(const DenseParams& P, int grid, size_t smem, int nch, cudaStream_t st);
cudaError_t launch_c2t_check(const C2TCheckParams& P, cudaStream_t st);
cudaError_t launch_repack(const RepackParams& P, cudaStream_t st);
// Cluster-major copy of the token rows: out[k*b + j] = E[C2T[k][j]].
cudaError_t launch_gather_cluster_major(const uint16_t* E, C2TView C2T, uint16_t* out, int v, int d,
                                        cudaStream_t st);
// tcgen05 GEMM (B >= 64): streamed rows bf16 [rows, d] through TMA, or packed INT4 / INT8 rows; H bf16 [nb, d].
cudaError_t launch_gemm(const GemmParams& P, const void* rows_bf16, const void* H, int num_sms, cudaStream_t st);
cudaError_t set_attrs_gemm();
// De-duplicated candidate logits of a batch (b == 16): CSR of the selections by cluster, then one
// pass per distinct cluster on the tensor cores.
cudaError_t launch_group(const GroupParams& P, int num_sms, cudaStream_t st);
cudaError_t set_attrs_group();
// Speculative verification of draft tokens against dense logits (one CTA per row).
cudaError_t launch_spec_verify(const float* logits, int v, const int32_t* cand, int n, int B, const int32_t* draft,
                               float T, const float* u_accept, const float* u_resample, int32_t* out, int* status,
                               cudaStream_t st);
// Adaptive probe count per row of centroid scores (one CTA per row).
cudaError_t launch_adaptive_probes(const float* scores, int B, int c, float tau, int p_min, int p_max, float T,
                                   int32_t* out_p, cudaStream_t st);

// L2 prefetch of the token rows (cluster-major copy) and C2T rows of n clusters.
cudaError_t launch_prefetch_clusters(const uint16_t* Ecm, C2TView C2T, int c, int b, int d, const int32_t* ids, int n,
                                     int* status, cudaStream_t st);

// Opt-in shared memory attribute for every instantiation (called once per device).
cudaError_t set_kernel_attributes(int max_smem);

// Register-array width for a hidden size: chunks of 8 elements per lane.
inline int nch_for(int d) {
  const int n = (d + 255) / 256;
  const int sizes[] = {1, 2, 3, 4, 5, 6, 8, 10};
  for (int s : sizes)
    if (n <= s) return s;
  return -1;
}

}  // namespace fh
