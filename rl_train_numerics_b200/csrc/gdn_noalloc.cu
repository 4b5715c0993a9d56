// gdn_noalloc.cu -- gdn_cpr_forward_noalloc: the CPR forward for callers that
// cannot allocate device memory.
//
// Some callers of this library cannot call cudaMalloc: for example a host
// runtime that owns the device memory pool and does not lend it out, a plugin
// host that gives a C library no allocator, or code that must not allocate on
// its hot path.  This entry point runs exactly gdn_cpr_forward, with its
// scratch space taken from a fixed-size array compiled into the library
// instead of a caller-provided workspace.  It calls no cudaMalloc, cudaFree or
// other allocating routine.
//
// The array holds GDN_NOALLOC_SCRATCH_BYTES (32 MiB).  Every GPU on which the
// library's device code for this file is loaded keeps that much memory until
// the process exits (with CUDA's default lazy module loading, from the first
// call of this entry point on that device).  In host code the array's name is
// only a host-side stand-in, not a device address, so the device address is
// looked up once per device with cudaGetSymbolAddress (with that device
// current) and cached; that set-up happens in the first call on each device,
// which should therefore come before any stream capture.  The cached address
// belongs to the device's primary context: after cudaDeviceReset (or anything
// else that destroys that context) the cache is stale and this entry point
// must not be called again in the process.
//
// Every call shares the one array per device and leaves its contents behind
// for the next call.  The forward writes every part of the scratch it reads
// before reading it, except the device error word, which this entry point
// clears at the start of each call.  Calls whose work can overlap on the GPU
// (for instance on two streams without an ordering between them) race on the
// array: callers must order them.
#include <cuda_runtime.h>

#include "../../include/gdn_cpr.h"
#include "gdn_layout.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[GDN_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch in the current context, looked up on
// every call (a host-side lookup; a cached address would outlive a reset or
// re-created primary context).
int scratch_on_current_device(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || p == nullptr) return GDN_ERR_CUDA;
  *out = p;
  return GDN_OK;
}

}  // namespace

extern "C" int gdn_cpr_forward_noalloc(const void* q, const void* k, const void* v, int in_dtype,
                                       const float* beta, const float* g,
                                       const int32_t* cu_seqlens, int n_seqs,
                                       int64_t total_tokens, int H, int dk, int dv, int C,
                                       float scale, const float* h0, void* o, int out_dtype,
                                       float* s_run_final, float* s_run_scale,
                                       float* s_bnd_final, int32_t* error_word,
                                       void* stream) {
  // Every argument check comes before any device work.
  const int chk = gdn::forward_check_args(q, k, v, in_dtype, beta, g, cu_seqlens, n_seqs,
                                          total_tokens, H, dk, dv, C, scale, h0, o, out_dtype,
                                          s_run_final, s_run_scale, s_bnd_final);
  if (chk != GDN_OK && chk != gdn::kFwdEmpty) return chk;
  if (error_word && (reinterpret_cast<uintptr_t>(error_word) & 3u) != 0)
    return GDN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (chk == gdn::kFwdEmpty) {
    // An empty batch launches nothing; the caller's error word still reports
    // this call (no error) rather than keeping an earlier call's bits.
    if (error_word && cudaMemsetAsync(error_word, 0, sizeof(int32_t), st) != cudaSuccess)
      return GDN_ERR_CUDA;
    return GDN_OK;
  }
  const size_t need = gdn_cpr_forward_workspace_bytes(n_seqs, total_tokens, H, dk, dv, C,
                                                      in_dtype);
  if (need == 0 || need > GDN_NOALLOC_SCRATCH_BYTES) return GDN_ERR_WORKSPACE;
  void* scratch = nullptr;
  int rc = scratch_on_current_device(&scratch);
  if (rc != GDN_OK) return rc;
  if (cudaMemsetAsync(scratch, 0, sizeof(int32_t), st) != cudaSuccess) return GDN_ERR_CUDA;
  rc = gdn_cpr_forward_ex(q, k, v, in_dtype, beta, g, cu_seqlens, n_seqs, total_tokens, H, dk,
                          dv, C, scale, h0, o, out_dtype, s_run_final, s_run_scale, s_bnd_final,
                          scratch, GDN_NOALLOC_SCRATCH_BYTES, nullptr, stream);
  if (rc != GDN_OK || error_word == nullptr) return rc;
  if (cudaMemcpyAsync(error_word, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice, st) !=
      cudaSuccess)
    return GDN_ERR_CUDA;
  return GDN_OK;
}
