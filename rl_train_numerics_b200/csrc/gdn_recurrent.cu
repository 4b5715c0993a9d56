// gdn_recurrent.cu -- the "recurrent everywhere" Gated DeltaNet layer: the
// per-token recurrence for prefill and training as well as for decode, with
// no chunk boundaries and no resync.
//
// "NovaSky's IsoExec Fixes the Hidden Math Bug Corrupting AI Training Runs",
// section "Solving the linear-attention headache": one of the two layouts the
// per-layer table compares CPR with runs the recurrent form for training,
// prefill and decode alike, so that all three share one rounding schedule by
// construction, at the price of a serial sweep over every token.  Here that
// layout is built from the same pinned step as the CPR fill and decode
// (gdn_common.cuh): S = c M with the per-(sequence, head) scale c, the row dot
// order, the renormalisation rule.  Consequences, both checked by the tests:
//   * the first chunk of every sequence is bitwise the CPR forward's (both
//     start from h0 with c = 1 and run the same step);
//   * a forward over P tokens that returns the mantissa and scale, followed by
//     recurrent decode steps, gives bitwise the forward over all the tokens.
//
// Rows of the state evolve independently (the step's only coupling between
// rows is the shared scale c, which depends on the gates alone), so a
// (sequence, head) unit is split over D / (32 RT) blocks of 32 quads, each
// quad holding RT rows; how rows are spread does not change any row's bits.
// Tokens arrive in tiles of 32, double-buffered with cp.async while the
// previous tile's tokens run.
#include <cuda_runtime.h>
#include <math.h>

#include "../../include/gdn_cpr.h"
#include "gdn_fill.cuh"
#include "gdn_layout.h"

namespace gdn {

constexpr int kRecurThreads = 128;  // 32 quads
constexpr int kRecurTile = 32;      // tokens per tile

template <int D, class IN, int RB>
struct RecurTile {
  IN k[kRecurTile][D];
  IN q[kRecurTile][D];
  IN v[kRecurTile][RB];  // the block's rows of v
  float g[kRecurTile];
  float b[kRecurTile];
};

template <int D, class IN, int RB>
struct RecurSmem {
  RecurTile<D, IN, RB> buf[2];
  float kf[kRecurTile][D];  // keys of the running tile, widened to fp32
  float a[kRecurTile];      // exp(g) of the running tile
};

__device__ __forceinline__ void cp_async4b(void* smem, const void* gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(smem)), "l"(gmem));
}

// Issue the copies of one tile (tokens t0 .. t0 + len - 1 of head h); rows
// past len are zero-filled with plain stores.
template <int D, class IN, int RB>
__device__ __forceinline__ void recur_issue(RecurTile<D, IN, RB>& tl, const IN* q, const IN* k,
                                            const IN* v, const float* beta, const float* g,
                                            size_t tb, int H, int rbase, int len) {
  constexpr int P = (int)(D * sizeof(IN) / 16), E = (int)(16 / sizeof(IN));
  constexpr int PV = (int)(RB * sizeof(IN) / 16), EV = E;
  const int tid = threadIdx.x;
  for (int e = tid; e < 2 * kRecurTile * P; e += kRecurThreads) {
    const int rr = e / P, pc = (e % P) * E;
    const bool isk = rr < kRecurTile;
    const int t = isk ? rr : rr - kRecurTile;
    IN* dst = isk ? &tl.k[t][pc] : &tl.q[t][pc];
    if (t < len) cp_async16(dst, (isk ? k : q) + (tb + (size_t)t * H) * D + pc);
    else *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
  }
  for (int e = tid; e < kRecurTile * PV; e += kRecurThreads) {
    const int t = e / PV, pc = (e % PV) * EV;
    if (t < len) cp_async16(&tl.v[t][pc], v + (tb + (size_t)t * H) * D + rbase + pc);
    else *reinterpret_cast<uint4*>(&tl.v[t][pc]) = make_uint4(0u, 0u, 0u, 0u);
  }
  for (int t = tid; t < kRecurTile; t += kRecurThreads) {
    if (t < len) {
      cp_async4b(&tl.g[t], g + tb + (size_t)t * H);
      cp_async4b(&tl.b[t], beta + tb + (size_t)t * H);
    } else {
      tl.g[t] = 0.f;
      tl.b[t] = 0.f;
    }
  }
  cp_async_commit();
}

// Sequence bounds check shared by the recurrent forward's blocks: cu_seqlens
// must start at 0, end at T and not decrease at this block's sequence.
__device__ __forceinline__ bool recur_seq_ok(const int32_t* cu, int N, int64_t T, int n) {
  return cu[0] == 0 && (int64_t)cu[N] == T && cu[n] >= 0 && cu[n + 1] >= cu[n] &&
         (int64_t)cu[n + 1] <= T;
}

// One block per (sequence, head, block of RB = 32 RT state rows).
template <int D, class IN, class OUT, int RT>
__global__ void __launch_bounds__(kRecurThreads)
    k_recur(const IN* __restrict__ q, const IN* __restrict__ k, const IN* __restrict__ v,
            const float* __restrict__ beta, const float* __restrict__ g,
            const int32_t* __restrict__ cu, int N, int64_t T, int H, float scale,
            const float* __restrict__ h0, OUT* __restrict__ o, float* __restrict__ s_final,
            float* __restrict__ s_final_scale, int32_t* __restrict__ error) {
  constexpr int M4 = D / 16, RB = 32 * RT;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  RecurSmem<D, IN, RB>& sm = *reinterpret_cast<RecurSmem<D, IN, RB>*>(smem_raw);
  const int n = blockIdx.x, h = blockIdx.y, rb = blockIdx.z;
  if (!recur_seq_ok(cu, N, T, n)) {
    if (threadIdx.x == 0 && error) atomicOr(error, kErrCuSeqlens);
    return;
  }
  const int tid = threadIdx.x, l = tid & 3;
  const int rbase = rb * RB, r0 = rbase + (tid >> 2) * RT;
  const int64_t L = (int64_t)cu[n + 1] - cu[n];
  const size_t DD = (size_t)D * D;
  const size_t tb0 = (size_t)cu[n] * H + h;
  const int64_t ntiles = (L + kRecurTile - 1) / kRecurTile;

  Slice<RT, M4> S;
  if (h0) {
    slice_load<RT, M4>(S, h0 + ((size_t)n * H + h) * DD, D, r0, l);
  } else {
#pragma unroll
    for (int i = 0; i < RT; i++)
#pragma unroll
      for (int m = 0; m < M4; m++) S.s[i][m][0] = S.s[i][m][1] = f2(0.f, 0.f);
  }
  float c = 1.f;
  auto tile_len = [&](int64_t j) { return (int)min((int64_t)kRecurTile, L - j * kRecurTile); };
  if (ntiles > 0)
    recur_issue<D, IN, RB>(sm.buf[0], q, k, v, beta, g, tb0, H, rbase, tile_len(0));
  for (int64_t j = 0; j < ntiles; j++) {
    const int len = tile_len(j);
    if (j + 1 < ntiles) {
      recur_issue<D, IN, RB>(sm.buf[(j + 1) & 1], q, k, v, beta, g,
                             tb0 + (size_t)(j + 1) * kRecurTile * H, H, rbase, tile_len(j + 1));
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const RecurTile<D, IN, RB>& tl = sm.buf[j & 1];
    for (int e = tid; e < kRecurTile * (D / 4); e += kRecurThreads) {
      const int t = e / (D / 4), cc = (e % (D / 4)) * 4;
      *reinterpret_cast<float4*>(&sm.kf[t][cc]) = sld4(&tl.k[t][cc]);
    }
    for (int t = tid; t < kRecurTile; t += kRecurThreads)
      sm.a[t] = t < len ? step_decay(tl.g[t]) : 0.f;
    __syncthreads();

    // The first token's dot (a separate sweep carries the fused dot's bits).
    float p[RT];
    slice_dot<RT, M4>(S, [&](int m) { return sld4(&sm.kf[0][group_col(l, m)]); }, p);
#pragma unroll
    for (int i = 0; i < RT; i++) p[i] = quad_sum(p[i]);
    OUT* ob = o + (tb0 + (size_t)j * kRecurTile * H) * D + r0 + l;
    const int rl = (tid >> 2) * RT;  // the quad's first row within the block
    for (int t = 0; t < len; t++) {
      float ov[RT];
      auto fv = [&](int i) { return to_f(tl.v[t][rl + i]); };
      auto fk = [&](int m) { return sld4(&sm.kf[t][group_col(l, m)]); };
      auto fq = [&](int m) { return sld4(&tl.q[t][group_col(l, m)]); };
      auto fn = [&](int m) { return sld4(&sm.kf[t + 1][group_col(l, m)]); };
      if (t + 1 < len)
        slice_token<true, RT, M4>(S, c, sm.a[t], tl.b[t], fv, fk, fq, fn, p, ov);
      else
        slice_token<false, RT, M4>(S, c, sm.a[t], tl.b[t], fv, fk, fq, fk, p, ov);
#pragma unroll
      for (int i = 0; i < RT; i++) ov[i] = __fmul_rn(scale, ov[i]);
      if (l < RT) st1(ob + (size_t)t * H * D, pick<RT>(ov, l));
    }
    __syncthreads();  // this buffer is refilled with tile j + 2
  }
  if (s_final) {
    float* dst = s_final + ((size_t)n * H + h) * DD;
    if (s_final_scale) {
      slice_store<RT, M4>(S, dst, D, r0, l);
      if (rb == 0 && tid == 0) s_final_scale[(size_t)n * H + h] = c;
    } else {
      slice_store_scaled<RT, M4>(S, c, dst, D, r0, l);
    }
  }
}

// One recurrent decode step per (row b, head): the CPR decode step's
// arithmetic on the running pair (mantissa s, scale s_scale), in place, with
// no chunk buffer and no resync.
constexpr int kRecurStepThreads = 128;

template <int D, class IN, class OUT>
__global__ void __launch_bounds__(kRecurStepThreads)
    k_recur_step(const IN* __restrict__ q, const IN* __restrict__ k, const IN* __restrict__ v,
                 const float* __restrict__ beta, const float* __restrict__ g, int H, float scale,
                 float* __restrict__ s, float* __restrict__ s_scale, OUT* __restrict__ o) {
  constexpr int RT = D / 32, M4 = D / 16;
  const int b = blockIdx.x, h = blockIdx.y;
  const int tid = threadIdx.x, l = tid & 3, r0 = (tid >> 2) * RT;
  const size_t unit = (size_t)b * H + h, DD = (size_t)D * D;
  Slice<RT, M4> S;
  slice_load<RT, M4>(S, s + unit * DD, D, r0, l);
  const IN* kp = k + unit * D;
  const IN* qp = q + unit * D;
  const float a = step_decay(g[unit]);
  const float bt = beta[unit];
  float c = s_scale[unit];
  float p[RT], ov[RT];
  auto kf = [&](int m) { return ld4(kp + group_col(l, m)); };
  slice_dot<RT, M4>(S, kf, p);
#pragma unroll
  for (int i = 0; i < RT; i++) p[i] = quad_sum(p[i]);
  slice_token<false, RT, M4>(
      S, c, a, bt, [&](int i) { return ld1(v + unit * D + r0 + i); }, kf,
      [&](int m) { return ld4(qp + group_col(l, m)); }, kf, p, ov);
#pragma unroll
  for (int i = 0; i < RT; i++) ov[i] = __fmul_rn(scale, ov[i]);
  if (l < RT) st1(o + unit * D + r0 + l, pick<RT>(ov, l));
  slice_store<RT, M4>(S, s + unit * DD, D, r0, l);
  if (tid == 0) s_scale[unit] = c;
}

// ----------------------------------------------------------------------------
// Launchers
// ----------------------------------------------------------------------------
// Rows per quad of the recurrent forward (at most D / 32).  Four rows (one
// block per unit at d = 128) ran the 5 x 2048 prefill in 1.11 ms against
// 1.24 ms with two and 1.38 ms with one: the per-token chain of dependent
// steps, not the number of blocks, sets the time, and more rows per thread
// give it more independent work.
constexpr int kRecurRT = 4;

template <int D, class IN, class OUT>
static cudaError_t recur_forward_impl(const void* q, const void* k, const void* v,
                                      const float* beta, const float* g, const int32_t* cu,
                                      int N, int64_t T, int H, float scale, const float* h0,
                                      void* o, float* s_final, float* s_final_scale,
                                      int32_t* error, cudaStream_t st) {
  constexpr int RT = 32 * kRecurRT <= D ? kRecurRT : D / 32, RB = 32 * RT;
  static_assert(D % RB == 0, "whole row blocks");
  auto kern = k_recur<D, IN, OUT, RT>;
  const size_t smem = sizeof(RecurSmem<D, IN, RB>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3((unsigned)N, (unsigned)H, (unsigned)(D / RB)), kRecurThreads, smem, st>>>(
      static_cast<const IN*>(q), static_cast<const IN*>(k), static_cast<const IN*>(v), beta, g,
      cu, N, T, H, scale, h0, static_cast<OUT*>(o), s_final, s_final_scale, error);
  return cudaGetLastError();
}

template <int D, class IN, class OUT>
static cudaError_t recur_step_impl(const void* q, const void* k, const void* v,
                                   const float* beta, const float* g, int B, int H, float scale,
                                   float* s, float* s_scale, void* o, cudaStream_t st) {
  k_recur_step<D, IN, OUT><<<dim3((unsigned)B, (unsigned)H), kRecurStepThreads, 0, st>>>(
      static_cast<const IN*>(q), static_cast<const IN*>(k), static_cast<const IN*>(v), beta, g,
      H, scale, s, s_scale, static_cast<OUT*>(o));
  return cudaGetLastError();
}

using bf16 = __nv_bfloat16;

}  // namespace gdn

namespace {

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool al4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace

extern "C" int gdn_recurrent_forward(const void* q, const void* k, const void* v, int in_dtype,
                                     const float* beta, const float* g,
                                     const int32_t* cu_seqlens, int n_seqs, int64_t total_tokens,
                                     int H, int dk, int dv, float scale, const float* h0,
                                     void* o, int out_dtype, float* s_final,
                                     float* s_final_scale, int32_t* error_word, void* stream) {
  using namespace gdn;
  const int chk = forward_check_args(q, k, v, in_dtype, beta, g, cu_seqlens, n_seqs,
                                     total_tokens, H, dk, dv, kChunk, scale, h0, o, out_dtype,
                                     s_final, s_final_scale, nullptr);
  if (chk != GDN_OK && chk != kFwdEmpty) return chk;
  if (error_word && !al4(error_word)) return GDN_ERR_INVALID_ARG;
  if (s_final && !al16(s_final)) return GDN_ERR_INVALID_ARG;
  if (s_final_scale && (!s_final || !al4(s_final_scale))) return GDN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (error_word && cudaMemsetAsync(error_word, 0, sizeof(int32_t), st) != cudaSuccess)
    return GDN_ERR_CUDA;
  if (chk == kFwdEmpty) return GDN_OK;
  const bool ib = in_dtype == GDN_BF16, ob = out_dtype == GDN_BF16;
  cudaError_t e;
  const int N = n_seqs;
  const int64_t T = total_tokens;
  if (dk == 64) {
    if (ib)
      e = ob ? recur_forward_impl<64, bf16, bf16>(q, k, v, beta, g, cu_seqlens, N, T, H, scale,
                                                  h0, o, s_final, s_final_scale, error_word, st)
             : recur_forward_impl<64, bf16, float>(q, k, v, beta, g, cu_seqlens, N, T, H, scale,
                                                   h0, o, s_final, s_final_scale, error_word, st);
    else
      e = ob ? recur_forward_impl<64, float, bf16>(q, k, v, beta, g, cu_seqlens, N, T, H, scale,
                                                   h0, o, s_final, s_final_scale, error_word, st)
             : recur_forward_impl<64, float, float>(q, k, v, beta, g, cu_seqlens, N, T, H,
                                                    scale, h0, o, s_final, s_final_scale,
                                                    error_word, st);
  } else {
    e = ob ? recur_forward_impl<128, bf16, bf16>(q, k, v, beta, g, cu_seqlens, N, T, H, scale,
                                                 h0, o, s_final, s_final_scale, error_word, st)
           : recur_forward_impl<128, bf16, float>(q, k, v, beta, g, cu_seqlens, N, T, H, scale,
                                                  h0, o, s_final, s_final_scale, error_word, st);
  }
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

extern "C" int gdn_recurrent_decode_step(const void* q, const void* k, const void* v,
                                         int in_dtype, const float* beta, const float* g, int B,
                                         int H, int dk, int dv, float scale, float* s,
                                         float* s_scale, void* o, int out_dtype, void* stream) {
  using namespace gdn;
  if (B < 0 || H <= 0 || dk != dv || (dk != 64 && dk != 128)) {
    if (B < 0 || H <= 0 || dk <= 0 || dv <= 0) return GDN_ERR_INVALID_ARG;
    return GDN_ERR_UNSUPPORTED;
  }
  if ((in_dtype != GDN_BF16 && in_dtype != GDN_F32) ||
      (out_dtype != GDN_BF16 && out_dtype != GDN_F32) || !isfinite(scale))
    return GDN_ERR_INVALID_ARG;
  if (in_dtype == GDN_F32 && dk != 64) return GDN_ERR_UNSUPPORTED;
  if (H > 65535) return GDN_ERR_UNSUPPORTED;
  if (B == 0) return GDN_OK;
  if (!q || !k || !v || !beta || !g || !s || !s_scale || !o) return GDN_ERR_INVALID_ARG;
  if (!al16(q) || !al16(k) || !al16(v) || !al16(s) || !al16(o) || !al4(beta) || !al4(g) ||
      !al4(s_scale))
    return GDN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool ib = in_dtype == GDN_BF16, ob = out_dtype == GDN_BF16;
  cudaError_t e;
  if (dk == 64) {
    if (ib)
      e = ob ? recur_step_impl<64, bf16, bf16>(q, k, v, beta, g, B, H, scale, s, s_scale, o, st)
             : recur_step_impl<64, bf16, float>(q, k, v, beta, g, B, H, scale, s, s_scale, o, st);
    else
      e = ob ? recur_step_impl<64, float, bf16>(q, k, v, beta, g, B, H, scale, s, s_scale, o, st)
             : recur_step_impl<64, float, float>(q, k, v, beta, g, B, H, scale, s, s_scale, o,
                                                 st);
  } else {
    e = ob ? recur_step_impl<128, bf16, bf16>(q, k, v, beta, g, B, H, scale, s, s_scale, o, st)
           : recur_step_impl<128, bf16, float>(q, k, v, beta, g, B, H, scale, s, s_scale, o, st);
  }
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}
