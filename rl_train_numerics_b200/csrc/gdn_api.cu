// gdn_api.cu -- extern "C" entry points of libgdn_cpr.so (declared in
// include/gdn_cpr.h).  Host-side argument validation happens here, before any
// CUDA call, so that argument errors are reported synchronously and without
// touching the device; the kernels are in gdn_kernels.cu.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "../../include/gdn_cpr.h"
#include "gdn_layout.h"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool valid_dtype(int d) { return d == GDN_BF16 || d == GDN_F32; }

// Shape check shared by every entry point: returns GDN_OK, INVALID_ARG or UNSUPPORTED.
int check_shape(int H, int dk, int dv, int C, int in_dtype) {
  if (H <= 0 || dk <= 0 || dv <= 0 || C <= 0) return GDN_ERR_INVALID_ARG;
  if (!valid_dtype(in_dtype)) return GDN_ERR_INVALID_ARG;
  if (dk != dv || (dk != 64 && dk != 128) || C != 64) return GDN_ERR_UNSUPPORTED;
  if (in_dtype == GDN_F32 && dk != 64) return GDN_ERR_UNSUPPORTED;  // fp32 inputs: d = 64
  if (H > 65535) return GDN_ERR_UNSUPPORTED;  // grid.y
  return GDN_OK;
}

int from_cuda(cudaError_t e) { return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA; }

}  // namespace

extern "C" {

int gdn_cpr_abi_version(void) { return GDN_CPR_ABI_VERSION; }

const char* gdn_status_string(int status) {
  switch (status) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG: invalid argument";
    case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED: unsupported shape or dtype";
    case GDN_ERR_WORKSPACE: return "GDN_ERR_WORKSPACE: workspace missing or too small";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA: CUDA launch or runtime error";
    case GDN_ERR_DEVICE_DATA: return "GDN_ERR_DEVICE_DATA: device-side validation failed";
    case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT: bounded device wait gave up";
    case GDN_ERR_CONTRACT: return "GDN_ERR_CONTRACT: numerical policies differ";
    default: return "unknown gdn_status";
  }
}

size_t gdn_cpr_forward_workspace_bytes(int n_seqs, int64_t total_tokens, int H, int dk, int dv,
                                       int C, int in_dtype) {
  if (n_seqs < 0 || total_tokens < 0 || total_tokens > INT32_MAX) return 0;
  if (check_shape(H, dk, dv, C, in_dtype) != GDN_OK) return 0;
  return gdn::fwd_layout(n_seqs, total_tokens, H, dk, dv, C, in_dtype == GDN_BF16).total;
}

int gdn_cpr_forward(const void* q, const void* k, const void* v, int in_dtype, const float* beta,
                    const float* g, const int32_t* cu_seqlens, int n_seqs, int64_t total_tokens,
                    int H, int dk, int dv, int C, float scale, const float* h0, void* o,
                    int out_dtype, float* s_run_final, float* s_run_scale, float* s_bnd_final,
                    void* workspace, size_t workspace_bytes, void* stream) {
  return gdn_cpr_forward_ex(q, k, v, in_dtype, beta, g, cu_seqlens, n_seqs, total_tokens, H, dk,
                            dv, C, scale, h0, o, out_dtype, s_run_final, s_run_scale, s_bnd_final,
                            workspace, workspace_bytes, nullptr, stream);
}

}  // extern "C"

// Every host-side check of a forward call except the workspace's: returns
// GDN_OK, an error status, or kFwdEmpty for a valid empty batch (nothing
// to launch).
int gdn::forward_check_args(const void* q, const void* k, const void* v, int in_dtype,
                            const float* beta, const float* g, const int32_t* cu_seqlens,
                            int n_seqs, int64_t total_tokens, int H, int dk, int dv, int C,
                            float scale, const float* h0, const void* o, int out_dtype,
                            const float* s_run_final, const float* s_run_scale,
                            const float* s_bnd_final) {
  if (n_seqs < 0 || total_tokens < 0 || !valid_dtype(out_dtype) || !isfinite(scale))
    return GDN_ERR_INVALID_ARG;
  int rc = check_shape(H, dk, dv, C, in_dtype);
  if (rc != GDN_OK) return rc;
  if (total_tokens > INT32_MAX) return GDN_ERR_UNSUPPORTED;
  if (n_seqs == 0) return total_tokens == 0 ? kFwdEmpty : GDN_ERR_INVALID_ARG;
  if (!cu_seqlens || !aligned4(cu_seqlens)) return GDN_ERR_INVALID_ARG;
  if (total_tokens > 0) {
    if (!q || !k || !v || !beta || !g || !o) return GDN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return GDN_ERR_INVALID_ARG;
    if (!aligned4(beta) || !aligned4(g)) return GDN_ERR_INVALID_ARG;
  }
  if ((h0 && !aligned16(h0)) || (s_run_final && !aligned16(s_run_final)) ||
      (s_bnd_final && !aligned16(s_bnd_final)) || (s_run_scale && !aligned4(s_run_scale)))
    return GDN_ERR_INVALID_ARG;
  if (s_run_scale && !s_run_final) return GDN_ERR_INVALID_ARG;
  return GDN_OK;
}

extern "C" {

int gdn_cpr_forward_ex(const void* q, const void* k, const void* v, int in_dtype,
                       const float* beta, const float* g, const int32_t* cu_seqlens, int n_seqs,
                       int64_t total_tokens, int H, int dk, int dv, int C, float scale,
                       const float* h0, void* o, int out_dtype, float* s_run_final,
                       float* s_run_scale, float* s_bnd_final, void* workspace,
                       size_t workspace_bytes, void* const* kernel_events, void* stream) {
  const int rc = gdn::forward_check_args(q, k, v, in_dtype, beta, g, cu_seqlens, n_seqs,
                                         total_tokens, H, dk, dv, C, scale, h0, o, out_dtype,
                                         s_run_final, s_run_scale, s_bnd_final);
  if (rc == gdn::kFwdEmpty) return GDN_OK;
  if (rc != GDN_OK) return rc;
  const gdn::FwdLayout lay =
      gdn::fwd_layout(n_seqs, total_tokens, H, dk, dv, C, in_dtype == GDN_BF16);
  if (!workspace || workspace_bytes < lay.total) return GDN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return GDN_ERR_INVALID_ARG;
  gdn::FwdArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.in_bf16 = in_dtype == GDN_BF16;
  a.beta = beta;
  a.g = g;
  a.cu_seqlens = cu_seqlens;
  a.n_seqs = n_seqs;
  a.T = total_tokens;
  a.H = H;
  a.D = dk;
  a.scale = scale;
  a.h0 = h0;
  a.o = o;
  a.out_bf16 = out_dtype == GDN_BF16;
  a.s_run_final = s_run_final;
  a.s_run_scale = s_run_scale;
  a.s_bnd_final = s_bnd_final;
  a.ws = static_cast<char*>(workspace);
  a.lay = lay;
  a.events = kernel_events;
  return from_cuda(gdn::launch_forward(a, static_cast<cudaStream_t>(stream)));
}

int gdn_native_forward(const void* q, const void* k, const void* v, int in_dtype,
                       const float* beta, const float* g, const int32_t* cu_seqlens, int n_seqs,
                       int64_t total_tokens, int H, int dk, int dv, int C, float scale,
                       const float* h0, void* o, int out_dtype, float* s_final,
                       float* s_bnd_final, void* workspace, size_t workspace_bytes,
                       void* const* kernel_events, void* stream) {
  const int rc = gdn::forward_check_args(q, k, v, in_dtype, beta, g, cu_seqlens, n_seqs,
                                         total_tokens, H, dk, dv, C, scale, h0, o, out_dtype,
                                         s_final, nullptr, s_bnd_final);
  if (rc != GDN_OK && rc != gdn::kFwdEmpty) return rc;
  if (in_dtype != GDN_BF16 || dk != 128) return GDN_ERR_UNSUPPORTED;
  if (rc == gdn::kFwdEmpty) return GDN_OK;
  const gdn::FwdLayout lay = gdn::fwd_layout(n_seqs, total_tokens, H, dk, dv, C, true);
  if (!workspace || workspace_bytes < lay.total) return GDN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return GDN_ERR_INVALID_ARG;
  gdn::FwdArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.in_bf16 = 1;
  a.beta = beta;
  a.g = g;
  a.cu_seqlens = cu_seqlens;
  a.n_seqs = n_seqs;
  a.T = total_tokens;
  a.H = H;
  a.D = dk;
  a.scale = scale;
  a.h0 = h0;
  a.o = o;
  a.out_bf16 = out_dtype == GDN_BF16;
  a.s_run_final = s_final;
  a.s_bnd_final = s_bnd_final;
  a.ws = static_cast<char*>(workspace);
  a.lay = lay;
  a.events = kernel_events;
  return from_cuda(gdn::launch_native_forward(a, static_cast<cudaStream_t>(stream)));
}

size_t gdn_cpr_backward_workspace_bytes(int n_seqs, int64_t total_tokens, int H, int dk, int dv,
                                        int C, int in_dtype) {
  if (n_seqs < 0 || total_tokens < 0 || total_tokens > INT32_MAX) return 0;
  if (check_shape(H, dk, dv, C, in_dtype) != GDN_OK) return 0;
  return gdn::bwd_layout(n_seqs, total_tokens, H, dk, dv, C, in_dtype == GDN_BF16).total;
}

int gdn_cpr_backward(const void* q, const void* k, const void* v, int in_dtype,
                     const float* beta, const float* g, const int32_t* cu_seqlens, int n_seqs,
                     int64_t total_tokens, int H, int dk, int dv, int C, float scale,
                     const float* h0, const void* d_o, const float* ds_final, float* d_q,
                     float* d_k, float* d_v, float* d_beta, float* d_g, float* d_h0,
                     void* workspace, size_t workspace_bytes, int flags, void* stream) {
  return gdn_cpr_backward_ex(q, k, v, in_dtype, beta, g, cu_seqlens, n_seqs, total_tokens, H, dk,
                             dv, C, scale, h0, d_o, ds_final, d_q, d_k, d_v, d_beta, d_g, d_h0,
                             workspace, workspace_bytes, flags, nullptr, stream);
}

int gdn_cpr_backward_ex(const void* q, const void* k, const void* v, int in_dtype,
                        const float* beta, const float* g, const int32_t* cu_seqlens,
                        int n_seqs, int64_t total_tokens, int H, int dk, int dv, int C,
                        float scale, const float* h0, const void* d_o, const float* ds_final,
                        float* d_q, float* d_k, float* d_v, float* d_beta, float* d_g,
                        float* d_h0, void* workspace, size_t workspace_bytes, int flags,
                        void* const* kernel_events, void* stream) {
  if (n_seqs < 0 || total_tokens < 0 || !isfinite(scale)) return GDN_ERR_INVALID_ARG;
  if ((flags & ~GDN_BWD_REUSE_FORWARD) != 0) return GDN_ERR_INVALID_ARG;
  int rc = check_shape(H, dk, dv, C, in_dtype);
  if (rc != GDN_OK) return rc;
  if (total_tokens > INT32_MAX) return GDN_ERR_UNSUPPORTED;
  if (n_seqs == 0) return total_tokens == 0 ? GDN_OK : GDN_ERR_INVALID_ARG;
  if (!cu_seqlens || !aligned4(cu_seqlens)) return GDN_ERR_INVALID_ARG;
  if (total_tokens > 0) {
    if (!q || !k || !v || !beta || !g || !d_o || !d_q || !d_k || !d_v || !d_beta || !d_g)
      return GDN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(d_o) || !aligned16(d_q) ||
        !aligned16(d_k) || !aligned16(d_v))
      return GDN_ERR_INVALID_ARG;
    if (!aligned4(beta) || !aligned4(g) || !aligned4(d_beta) || !aligned4(d_g))
      return GDN_ERR_INVALID_ARG;
  }
  if ((h0 && !aligned16(h0)) || (ds_final && !aligned16(ds_final)) || (d_h0 && !aligned16(d_h0)))
    return GDN_ERR_INVALID_ARG;
  const gdn::BwdLayout lay =
      gdn::bwd_layout(n_seqs, total_tokens, H, dk, dv, C, in_dtype == GDN_BF16);
  if (!workspace || workspace_bytes < lay.total) return GDN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return GDN_ERR_INVALID_ARG;
  gdn::BwdArgs a{};
  a.fwd.q = q;
  a.fwd.k = k;
  a.fwd.v = v;
  a.fwd.in_bf16 = in_dtype == GDN_BF16;
  a.fwd.beta = beta;
  a.fwd.g = g;
  a.fwd.cu_seqlens = cu_seqlens;
  a.fwd.n_seqs = n_seqs;
  a.fwd.T = total_tokens;
  a.fwd.H = H;
  a.fwd.D = dk;
  a.fwd.scale = scale;
  a.fwd.h0 = h0;
  a.fwd.ws = static_cast<char*>(workspace);
  a.fwd.lay = lay.fwd;
  a.d_o = d_o;
  a.ds_final = ds_final;
  a.d_q = d_q;
  a.d_k = d_k;
  a.d_v = d_v;
  a.d_beta = d_beta;
  a.d_g = d_g;
  a.d_h0 = d_h0;
  a.reuse_forward = (flags & GDN_BWD_REUSE_FORWARD) ? 1 : 0;
  a.lay = lay;
  a.events = kernel_events;
  return from_cuda(gdn::launch_backward(a, static_cast<cudaStream_t>(stream)));
}

static int check_state(const gdn_decode_state& st) {
  if (st.n_slots <= 0 || !st.s_run || !st.s_scale || !st.s_bnd || !st.buf_k || !st.buf_v ||
      !st.buf_beta || !st.buf_g || !st.pos || !st.error || !st.resync)
    return GDN_ERR_INVALID_ARG;
  if (!aligned16(st.s_run) || !aligned16(st.s_bnd) || !aligned16(st.buf_k) ||
      !aligned16(st.buf_v) || !aligned4(st.buf_beta) || !aligned4(st.buf_g) ||
      !aligned4(st.pos) || !aligned4(st.error) || !aligned4(st.s_scale) || !aligned4(st.resync))
    return GDN_ERR_INVALID_ARG;
  return GDN_OK;
}

int gdn_cpr_decode_state_from_prefill(const void* k, const void* v, int in_dtype,
                                      const float* beta, const float* g,
                                      const int32_t* cu_seqlens, int n_seqs,
                                      int64_t total_tokens, int H, int dk, int dv, int C,
                                      const float* s_run_final, const float* s_run_scale,
                                      const float* s_bnd_final, const int32_t* slot_idx,
                                      gdn_decode_state st, void* stream) {
  if (n_seqs < 0 || total_tokens < 0) return GDN_ERR_INVALID_ARG;
  int rc = check_shape(H, dk, dv, C, in_dtype);
  if (rc != GDN_OK) return rc;
  if (total_tokens > INT32_MAX) return GDN_ERR_UNSUPPORTED;
  if (n_seqs == 0) return GDN_OK;
  if ((rc = check_state(st)) != GDN_OK) return rc;
  if (!cu_seqlens || !s_run_final || !s_bnd_final) return GDN_ERR_INVALID_ARG;
  if (total_tokens > 0 && (!k || !v || !beta || !g)) return GDN_ERR_INVALID_ARG;
  if (!aligned16(s_run_final) || !aligned16(s_bnd_final)) return GDN_ERR_INVALID_ARG;
  if (s_run_scale && !aligned4(s_run_scale)) return GDN_ERR_INVALID_ARG;
  if (!slot_idx && n_seqs > st.n_slots) return GDN_ERR_INVALID_ARG;
  gdn::HandoffArgs a{};
  a.k = k;
  a.v = v;
  a.in_bf16 = in_dtype == GDN_BF16;
  a.beta = beta;
  a.g = g;
  a.cu_seqlens = cu_seqlens;
  a.n_seqs = n_seqs;
  a.T = total_tokens;
  a.H = H;
  a.D = dk;
  a.s_run_final = s_run_final;
  a.s_run_scale = s_run_scale;
  a.s_bnd_final = s_bnd_final;
  a.slot_idx = slot_idx;
  a.s_run = st.s_run;
  a.s_scale = st.s_scale;
  a.s_bnd = st.s_bnd;
  a.buf_k = st.buf_k;
  a.buf_v = st.buf_v;
  a.buf_beta = st.buf_beta;
  a.buf_g = st.buf_g;
  a.pos = st.pos;
  a.error = st.error;
  a.n_slots = st.n_slots;
  return from_cuda(gdn::launch_handoff(a, static_cast<cudaStream_t>(stream)));
}

int gdn_cpr_decode_step(const void* q, const void* k, const void* v, int in_dtype,
                        const float* beta, const float* g, const int32_t* slot_idx, int B, int H,
                        int dk, int dv, int C, float scale, gdn_decode_state st, void* o,
                        int out_dtype, void* stream) {
  if (B < 0 || !valid_dtype(out_dtype) || !isfinite(scale)) return GDN_ERR_INVALID_ARG;
  int rc = check_shape(H, dk, dv, C, in_dtype);
  if (rc != GDN_OK) return rc;
  if (B == 0) return GDN_OK;
  if ((rc = check_state(st)) != GDN_OK) return rc;
  if (!q || !k || !v || !beta || !g || !o) return GDN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(beta) ||
      !aligned4(g))
    return GDN_ERR_INVALID_ARG;
  if (!slot_idx && B > st.n_slots) return GDN_ERR_INVALID_ARG;
  gdn::DecArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.in_bf16 = in_dtype == GDN_BF16;
  a.beta = beta;
  a.g = g;
  a.slot_idx = slot_idx;
  a.B = B;
  a.H = H;
  a.D = dk;
  a.scale = scale;
  a.s_run = st.s_run;
  a.s_scale = st.s_scale;
  a.s_bnd = st.s_bnd;
  a.buf_k = st.buf_k;
  a.buf_v = st.buf_v;
  a.buf_beta = st.buf_beta;
  a.buf_g = st.buf_g;
  a.pos = st.pos;
  a.error = st.error;
  a.resync = st.resync;
  a.n_slots = st.n_slots;
  a.o = o;
  a.out_bf16 = out_dtype == GDN_BF16;
  return from_cuda(gdn::launch_decode_step(a, static_cast<cudaStream_t>(stream)));
}

int gdn_chunk_boundary(const float* s_start, const void* k, const void* v, int in_dtype,
                       const float* beta, const float* g, int B, int H, int dk, int dv, int C,
                       float* s_end, void* stream) {
  if (B < 0) return GDN_ERR_INVALID_ARG;
  int rc = check_shape(H, dk, dv, C, in_dtype);
  if (rc != GDN_OK) return rc;
  if (B == 0) return GDN_OK;
  if (!s_start || !k || !v || !beta || !g || !s_end) return GDN_ERR_INVALID_ARG;
  if (!aligned16(s_start) || !aligned16(s_end) || !aligned16(k) || !aligned16(v) ||
      !aligned4(beta) || !aligned4(g))
    return GDN_ERR_INVALID_ARG;
  gdn::BndArgs a{};
  a.s_start = s_start;
  a.k = k;
  a.v = v;
  a.in_bf16 = in_dtype == GDN_BF16;
  a.beta = beta;
  a.g = g;
  a.B = B;
  a.H = H;
  a.D = dk;
  a.s_end = s_end;
  return from_cuda(gdn::launch_chunk_boundary(a, static_cast<cudaStream_t>(stream)));
}

int gdn_check_error(void* error_word, int32_t* bits_out, void* stream) {
  if (!error_word || !aligned4(error_word)) return GDN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t bits = 0;
  if (cudaStreamSynchronize(st) != cudaSuccess) return GDN_ERR_CUDA;
  if (cudaMemcpy(&bits, error_word, sizeof(bits), cudaMemcpyDeviceToHost) != cudaSuccess)
    return GDN_ERR_CUDA;
  if (bits != 0 && cudaMemset(error_word, 0, sizeof(int32_t)) != cudaSuccess) return GDN_ERR_CUDA;
  if (bits_out) *bits_out = bits;
  return bits ? GDN_ERR_DEVICE_DATA : GDN_OK;
}

}  // extern "C"
