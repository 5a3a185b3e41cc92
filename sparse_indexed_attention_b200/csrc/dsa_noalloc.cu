// dsa_sparse_mla_fwd_noalloc: sparse MLA attention for callers that cannot
// allocate device memory (see include/dsa.h).  The scratch that
// dsa_sparse_mla_fwd takes from the caller lives here in a fixed array of the
// library's device image instead; everything else is the regular entry point.
#include "dsa_internal.cuh"

namespace {

// The scratch every call of the entry point shares.  Zero-initialised when the
// library's device image is loaded; kept by each GPU that loads it until exit.
__device__ __align__(256) unsigned char g_noalloc_scratch[DSA_NOALLOC_SCRATCH_BYTES];

// Device address of the array in the current context.  Looked up on every
// call (a cheap host-side query): a cached address would go stale if the
// library's module were reloaded in a new primary context.
dsa_status_t scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return DSA_ERR_CUDA;
  *out = p;
  return DSA_OK;
}

}  // namespace

extern "C" dsa_status_t dsa_sparse_mla_fwd_noalloc(const dsa_seqs_t* seqs, const void* q, const void* kv,
                                                   const int32_t* idx, int K, int H, float scale, void* out,
                                                   dsa_out_dtype_t out_dtype, float* lse, dsa_stream_t stream) {
  // Size check first: host arithmetic only, nothing launched on rejection.
  if (!seqs) return DSA_ERR_INVALID_ARG;
  const size_t need = dsa_workspace_size(DSA_OP_SPARSE_MLA, seqs, K, H);
  if (need > (size_t)DSA_NOALLOC_SCRATCH_BYTES) return DSA_ERR_WORKSPACE;
  // need == 0 means invalid sizes; the regular entry point reports which.
  void* scratch = nullptr;
  const dsa_status_t st = scratch_address(&scratch);
  if (st != DSA_OK) return st;
  // The error word at the head of the scratch is the only part that has to
  // start at zero: the previous call may have left bits in it.
  if (cudaMemsetAsync(scratch, 0, 256, (cudaStream_t)stream) != cudaSuccess) return DSA_ERR_CUDA;
  return dsa_sparse_mla_fwd(seqs, q, kv, idx, K, H, scale, out, out_dtype, lse, scratch,
                            (size_t)DSA_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" dsa_status_t dsa_check_error_noalloc(dsa_stream_t stream) {
  void* scratch = nullptr;
  const dsa_status_t st = scratch_address(&scratch);
  if (st != DSA_OK) return st;
  return dsa_check_error(scratch, stream);
}
