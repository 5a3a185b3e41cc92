// dsa_sparse_mla_fwd_noalloc: sparse MLA attention for callers that cannot
// allocate device memory (see include/dsa.h).  The scratch that
// dsa_sparse_mla_fwd takes from the caller lives here in a fixed array of the
// library's device image instead; everything else is the regular entry point.
#include <atomic>

#include "dsa_internal.cuh"

namespace {

// The scratch every call of the entry point shares.  Zero-initialised when the
// library's device image is loaded; kept by each GPU that loads it until exit.
__device__ __align__(256) unsigned char g_noalloc_scratch[DSA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_addr[kMaxDevices];  // device address of the array, per device

}  // namespace

extern "C" dsa_status_t dsa_sparse_mla_fwd_noalloc(const dsa_seqs_t* seqs, const void* q, const void* kv,
                                                   const int32_t* idx, int K, int H, float scale, void* out,
                                                   dsa_out_dtype_t out_dtype, float* lse, dsa_stream_t stream) {
  // Size check first: host arithmetic only, nothing launched on rejection.
  if (!seqs) return DSA_ERR_INVALID_ARG;
  const size_t need = dsa_workspace_size(DSA_OP_SPARSE_MLA, seqs, K, H);
  if (need > (size_t)DSA_NOALLOC_SCRATCH_BYTES) return DSA_ERR_WORKSPACE;
  // need == 0 means invalid sizes; the regular entry point reports which.

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DSA_ERR_CUDA;
  void* scratch = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (!scratch) {
    // One-time set-up on this device (the device is current): the host-side
    // name of the array is not a device address, so ask the runtime for it.
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return DSA_ERR_CUDA;
    g_scratch_addr[dev].store(p, std::memory_order_release);
    scratch = p;
  }
  // The error word at the head of the scratch is the only part that has to
  // start at zero; earlier calls may have left bits in it.
  if (cudaMemsetAsync(scratch, 0, 256, (cudaStream_t)stream) != cudaSuccess) return DSA_ERR_CUDA;
  return dsa_sparse_mla_fwd(seqs, q, kv, idx, K, H, scale, out, out_dtype, lse, scratch,
                            (size_t)DSA_NOALLOC_SCRATCH_BYTES, stream);
}
