// Hot-cluster residency (write-up section 2.2.1: the token rows of frequently
// chosen clusters kept close to the compute units). On B200 the on-chip level
// that every SM shares is the 126 MB L2, so residency here means: the token rows
// of the clusters a caller expects to be chosen are requested into L2 ahead of
// the decode that reads them. One thread per cluster issues one bulk L2
// prefetch of the cluster's block in the cluster-major copy of E (b rows of d
// bf16, contiguous) and one of its C2T row; nothing waits for the data.
#include "fh_device.cuh"

namespace fh {
namespace {

__global__ void __launch_bounds__(128) prefetch_clusters_kernel(const uint16_t* Ecm, C2TView C2T, int c, int b, int d,
                                                                const int32_t* ids, int n, int* status) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int k = __ldg(ids + i);
  if (k < 0 || k >= c) {
    record_error(status, FH_ERR_OUT_OF_RANGE);
    return;
  }
  const size_t row0 = static_cast<size_t>(k) * b;
  bulk_prefetch_l2(Ecm + row0 * d, static_cast<uint32_t>(b) * static_cast<uint32_t>(d) * 2u);
  // the C2T row: one line prefetch per 128 bytes (its size need not be a multiple of 16)
  const uint8_t* t = reinterpret_cast<const uint8_t*>(C2T.ptr()) + row0 * C2T.elem_bytes();
  const size_t tb = static_cast<size_t>(b) * C2T.elem_bytes();
  for (size_t o = 0; o < tb; o += 128) prefetch_l2(t + o);
}

}  // namespace

cudaError_t launch_prefetch_clusters(const uint16_t* Ecm, C2TView C2T, int c, int b, int d, const int32_t* ids, int n,
                                     int* status, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  prefetch_clusters_kernel<<<(n + 127) / 128, 128, 0, st>>>(Ecm, C2T, c, b, d, ids, n, status);
  return cudaGetLastError();
}

}  // namespace fh
