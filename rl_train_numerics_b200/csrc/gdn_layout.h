// gdn_layout.h -- host-side layout of the forward workspace and the launch
// interface between the C ABI (gdn_api.cu) and the kernels (gdn_kernels.cu).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace gdn {

// Bytes of one walk pack (mirrors pack_size<D, IN>() in gdn_boundary.cuh; a
// static_assert there keeps the two equal): Tb and Tv as bf16 term planes of
// C x C, the decay vector [C] and 4 floats, then the chunk's keys and values
// as bf16 term planes of C x D.
constexpr size_t pack_bytes(int D, bool in_bf16) {
  const size_t NW = in_bf16 ? 2 : 3, NK = in_bf16 ? 1 : 3, C = 64;
  const size_t b = 2 * NW * C * C * 2 + C * 4 + 16 + 2 * NK * C * (size_t)D * 2;
  return (b + 127) / 128 * 128;
}

// Workspace of gdn_cpr_forward.  Offsets are 256-byte aligned.
//   hdr        int32[64]: [0] device error word, [1] number of chunks,
//                         [2] 1 when this call's chunk table is valid
//   chunk_off  int32[N+1]   first global chunk index of each sequence
//   chunk_seq  int32[MC]    sequence of each global chunk
//   walk_done  int32[N,H]   nonzero once the walk has stored a unit's boundary states
//   fill_off   int32[N]     each sequence's first entry in fill_order
//   fill_order int32[MC]    the chunks after each sequence's first, fewest-chunk
//                           sequences first (the fill's order for them)
//   bstate     f32[MC,H,dv,dk]  state at the start of every chunk
//   pack       [MC,H] walk packs (boundary prep of full chunks; the chunked
//                     forward also prepares trailing partial chunks, zero-padded)
// MC = floor(T/C) + N + 1 bounds the number of chunks for any valid
// cu_seqlens (each sequence adds at most one partial chunk).
struct FwdLayout {
  int64_t max_chunks;
  size_t pack_bytes;
  size_t hdr, chunk_off, seq_order, chunk_seq, walk_done, fill_off, fill_order, bstate, pack,
      total;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline FwdLayout fwd_layout(int n_seqs, int64_t T, int H, int dk, int dv, int C, bool in_bf16) {
  FwdLayout L{};
  L.max_chunks = T / C + n_seqs + 1;
  L.pack_bytes = pack_bytes(dk, in_bf16);
  const size_t mc = (size_t)L.max_chunks;
  size_t off = 0;
  L.hdr = off;
  off += align256(64 * sizeof(int32_t));
  L.chunk_off = off;
  off += align256((size_t)(n_seqs + 1) * sizeof(int32_t));
  L.seq_order = off;
  off += align256((size_t)n_seqs * sizeof(int32_t));
  L.chunk_seq = off;
  off += align256(mc * sizeof(int32_t));
  L.walk_done = off;
  off += align256((size_t)n_seqs * H * sizeof(int32_t));
  L.fill_off = off;
  off += align256((size_t)n_seqs * sizeof(int32_t));
  L.fill_order = off;
  off += align256(mc * sizeof(int32_t));
  L.bstate = off;
  off += align256(mc * H * dv * dk * sizeof(float));
  L.pack = off;
  off += align256(mc * H * L.pack_bytes);
  L.total = off;
  return L;
}

struct FwdArgs {
  const void* q;
  const void* k;
  const void* v;
  int in_bf16;
  const float* beta;
  const float* g;
  const int32_t* cu_seqlens;
  int n_seqs;
  int64_t T;
  int H, D;
  float scale;
  const float* h0;
  void* o;
  int out_bf16;
  float* s_run_final;
  float* s_run_scale;
  float* s_bnd_final;
  char* ws;
  FwdLayout lay;
  void* const* events;  // 5 cudaEvent_t recorded around the kernels, or null
  int pass1_only;       // 1: chunk table and boundary states only (no fill, o unused)
};

struct DecArgs {
  const void* q;
  const void* k;
  const void* v;
  int in_bf16;
  const float* beta;
  const float* g;
  const int32_t* slot_idx;
  int B, H, D;
  float scale;
  float* s_run;
  float* s_scale;
  float* s_bnd;
  void* buf_k;
  void* buf_v;
  float* buf_beta;
  float* buf_g;
  int32_t* pos;
  int32_t* error;
  int32_t* resync;
  int n_slots;
  void* o;
  int out_bf16;
};

struct HandoffArgs {
  const void* k;
  const void* v;
  int in_bf16;
  const float* beta;
  const float* g;
  const int32_t* cu_seqlens;
  int n_seqs;
  int64_t T;
  int H, D;
  const float* s_run_final;
  const float* s_run_scale;
  const float* s_bnd_final;
  const int32_t* slot_idx;
  float* s_run;
  float* s_scale;
  float* s_bnd;
  void* buf_k;
  void* buf_v;
  float* buf_beta;
  float* buf_g;
  int32_t* pos;
  int32_t* error;
  int n_slots;
};

struct BndArgs {
  const float* s_start;
  const void* k;
  const void* v;
  int in_bf16;
  const float* beta;
  const float* g;
  int B, H, D;
  float* s_end;
};

// Workspace of gdn_cpr_backward: the forward's (its first pass runs again
// inside the backward) followed by
//   mu_end  f32[MC,H,dv,dk]  adjoint flowing into the state at the end of
//                            every chunk (from the tokens after it)
//   wbuf    f32[T,H,dv]      w_t = Lambda_t k_t, one value per state row
//   ubuf    f32[T,H,dv]      u_t = beta_t (v_t - alpha_t S_{t-1} k_t) per row
//   with bf16 inputs (the adjoint in chunk form, gdn_adjoint.cuh), also
//   apack   [MC,H] adjoint packs (mirrors adj_pack_bytes<D>(): head of
//                  2C + 4 floats, keys as a bf16 plane C x D, X as three
//                  bf16 term planes C x D, Tb, T and Pm as three term planes
//                  C x C each)
//   ydv     f32[MC,H,dv,C]  (mu_e K^T) diag(dvec) per chunk (the walk's output)
constexpr size_t adj_pack_bytes_host(int D) {
  const size_t C = 64;
  const size_t b = (2 * C + 4) * 4 + C * (size_t)D * 2 + 3 * C * (size_t)D * 2 + 9 * C * C * 2;
  return (b + 127) / 128 * 128;
}

struct BwdLayout {
  FwdLayout fwd;
  size_t mu_end, wbuf, ubuf, apack, ydv, total;
};

inline BwdLayout bwd_layout(int n_seqs, int64_t T, int H, int dk, int dv, int C, bool in_bf16) {
  BwdLayout L{};
  L.fwd = fwd_layout(n_seqs, T, H, dk, dv, C, in_bf16);
  size_t off = L.fwd.total;
  L.mu_end = off;
  off += align256((size_t)L.fwd.max_chunks * H * dv * dk * sizeof(float));
  L.wbuf = off;
  off += align256((size_t)T * H * dv * sizeof(float));
  L.ubuf = off;
  off += align256((size_t)T * H * dv * sizeof(float));
  L.apack = L.ydv = off;
  if (in_bf16) {
    off += align256((size_t)L.fwd.max_chunks * H * adj_pack_bytes_host(dk));
    L.ydv = off;
    off += align256((size_t)L.fwd.max_chunks * H * dv * C * sizeof(float));
  }
  L.total = off;
  return L;
}

struct BwdArgs {
  FwdArgs fwd;  // inputs, shapes, scale, h0 and the workspace (first pass only)
  const void* d_o;
  const float* ds_final;
  float* d_q;
  float* d_k;
  float* d_v;
  float* d_beta;
  float* d_g;
  float* d_h0;
  int reuse_forward;  // 1: the workspace already holds this batch's first pass
  BwdLayout lay;
  void* const* events;  // 5 cudaEvent_t recorded around the kernels, or null
};

cudaError_t launch_forward(const FwdArgs& a, cudaStream_t stream);
// The chunked ("native mixed") forward (d = 128, bf16 inputs): the forward
// workspace, s_run_final as the state itself (s_run_scale unused).
cudaError_t launch_native_forward(const FwdArgs& a, cudaStream_t stream);

// Host-side argument checks of gdn_cpr_forward (all but the workspace);
// kFwdEmpty marks a valid call with nothing to launch.
constexpr int kFwdEmpty = 1;
int forward_check_args(const void* q, const void* k, const void* v, int in_dtype,
                       const float* beta, const float* g, const int32_t* cu_seqlens, int n_seqs,
                       int64_t total_tokens, int H, int dk, int dv, int C, float scale,
                       const float* h0, const void* o, int out_dtype, const float* s_run_final,
                       const float* s_run_scale, const float* s_bnd_final);
cudaError_t launch_backward(const BwdArgs& a, cudaStream_t stream);
cudaError_t launch_decode_step(const DecArgs& a, cudaStream_t stream);
cudaError_t launch_handoff(const HandoffArgs& a, cudaStream_t stream);
cudaError_t launch_chunk_boundary(const BndArgs& a, cudaStream_t stream);

}  // namespace gdn
