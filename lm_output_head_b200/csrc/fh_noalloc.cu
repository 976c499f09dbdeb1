// Allocation-free dense head (fh_dense_head_noalloc): the dense comparison
// head z = E h and its argmax (FlashHead write-up, section 1.1) launched with
// no handle and no device allocation. It runs the same dense kernel as
// fh_dense_head; only the kernel's per-call scratch -- one packed (logit,
// token) word per hidden row and the exit ticket -- lives in a fixed
// file-scope device array instead of an fh_create workspace.
//
// The write-up has no counterpart. It is plumbing for callers that must not
// allocate device memory while they run: a serving process whose caching
// allocator already holds the free HBM for its KV cache (a late cudaMalloc
// fails, or forces that cache to shrink), and latency-critical loops, where a
// cudaMalloc / cudaFree may synchronise the whole device.
//
// Scratch contract. The array is zero when the module is loaded. Every launch
// leaves it zero again: the kernel's last CTA takes each best word with
// atomicExch(., 0) and clears the ticket. All calls on one device share the
// array, so calls whose launches can overlap in time (unordered streams, host
// threads racing on one device) corrupt each other's results: order them,
// e.g. on one stream.
//
// First call per device: resolves the array's device address with
// cudaGetSymbolAddress (which may load this module onto the device) and sets
// the dense kernels' shared-memory attribute. Make that first call before any
// stream capture begins.
#include <mutex>

#include "fh.h"
#include "fh_internal.h"

namespace fh {

// defined with the dense kernel
cudaError_t set_attrs_dense(int max_smem);
int dense_max_rows();
cudaError_t occupancy_dense(int nch, size_t smem, int* blocks);

// one best word per row (FH_NOALLOC_MAX_ROWS of them) and the sync words
constexpr size_t kNoAllocScratchBytes = 1024;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

struct NoAllocScratch {
  unsigned long long best[FH_NOALLOC_MAX_ROWS];
  SyncWords sync;
};
static_assert(sizeof(NoAllocScratch) <= kNoAllocScratchBytes, "scratch layout exceeds the fixed array");

struct NoAllocDevice {
  bool ready = false;
  NoAllocScratch* scratch = nullptr;
  int num_sms = 0;
};

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
NoAllocDevice g_noalloc_dev[kMaxDevices];

fh_status fail(cudaError_t e) {
  (void)cudaGetLastError();
  return e == cudaErrorNoDevice || e == cudaErrorInsufficientDriver ? FH_ERR_UNSUPPORTED : FH_ERR_CUDA;
}

// Once per device, with that device current: scratch address, SM count,
// kernel attributes. Nothing here allocates device memory (module loading
// aside, which places the array itself).
fh_status setup_device(int dev, NoAllocDevice** out) {
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  NoAllocDevice& s = g_noalloc_dev[dev];
  if (!s.ready) {
    int major = 0, sms = 0, optin = 0;
    cudaError_t e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return fail(e);
    if (major != 10) return FH_ERR_UNSUPPORTED;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return fail(e);
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) return fail(e);
    e = set_attrs_dense(optin - 8192);
    if (e != cudaSuccess) return fail(e);
    s.scratch = static_cast<NoAllocScratch*>(p);
    s.num_sms = sms;
    s.ready = true;
  }
  *out = &s;
  return FH_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace
}  // namespace fh

using namespace fh;

extern "C" {

fh_status fh_dense_head_noalloc(const void* E, int32_t v, int32_t d, const void* hidden, int32_t B,
                                float* logits, int32_t* out_argmax, fh_stream_t stream) {
  if (!E || !hidden || !out_argmax) return FH_ERR_INVALID_ARG;
  if (!aligned16(E) || !aligned16(hidden)) return FH_ERR_INVALID_ARG;
  if (v < 1 || d < 8 || d % 8) return FH_ERR_INVALID_ARG;
  if (B < 1 || B > FH_NOALLOC_MAX_ROWS) return FH_ERR_INVALID_ARG;  // the fixed scratch holds 64 rows
  if (d > kMaxD) return FH_ERR_UNSUPPORTED;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(e);
  if (dev < 0 || dev >= kMaxDevices) return FH_ERR_UNSUPPORTED;
  NoAllocDevice* s = nullptr;
  fh_status st = setup_device(dev, &s);
  if (st != FH_OK) return st;

  const int nch = nch_for(d);
  const int rmax = dense_max_rows();
  int blocks = 0;
  e = occupancy_dense(nch, static_cast<size_t>(rmax) * d * 4, &blocks);
  if (e != cudaSuccess) return fail(e);
  const int grid = (blocks >= 1 ? (blocks < 2 ? blocks : 2) : 1) * s->num_sms;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  for (int r0 = 0; r0 < B; r0 += rmax) {
    const int rows = B - r0 < rmax ? B - r0 : rmax;
    DenseParams P{};
    P.E = static_cast<const uint16_t*>(E);
    P.hidden = static_cast<const uint16_t*>(hidden);
    P.logits = logits;
    P.out_argmax = out_argmax;
    P.best = s->scratch->best;  // row r0 + r uses best[r0 + r] < FH_NOALLOC_MAX_ROWS
    P.sync = &s->scratch->sync;
    P.v = v;
    P.d = d;
    P.row0 = r0;
    P.rows = rows;
    e = launch_dense(P, grid, static_cast<size_t>(rows) * d * 4, nch, cs);
    if (e != cudaSuccess) return fail(e);
  }
  return FH_OK;
}

}  // extern "C"
