// gdn_common.cuh -- shared device code of the CPR Gated DeltaNet kernels.
//
// The per-token step below is the one piece of arithmetic that the
// intra-chunk fill (second CPR pass) and the decode step both run.  The
// section "Solving the linear-attention headache" of "NovaSky's IsoExec Fixes
// the Hidden Math Bug Corrupting AI Training Runs" asks that prefill,
// training and decode share one rounding schedule; here that schedule is
// fixed instruction by instruction.
//
// Scaled running state.  Inside a chunk the state is kept as S = c * M: a
// per-(sequence, head) scale c and a d_v x d_k mantissa M.  At a chunk
// boundary M is the boundary state and c = 1.  One token (a = expf(g)):
//
//   p_r = c * dot(M_r, k)                 (dot order below)
//   u_r = beta * fma(-a, p_r, v_r)
//   c'  = a * c
//   if c' >= 2^-64:   M_r[j] <- fma(u_r * (1/c'), k_j, M_r[j]),  c <- c'
//   else (renormalise, also when a underflows to 0):
//                     M_r[j] <- fma(c', M_r[j], u_r * k_j),      c <- 1
//   o_r = scale * (c * dot(M_r, q))
//
// which is S_t = a S_{t-1} + u k^T, o_t = scale * S_t q_t with
// u = beta (v - a S_{t-1} k) -- the recurrence
// S_t = a S_{t-1} (I - beta k k^T) + beta v k^T -- with one fused
// multiply-add per state element for the update instead of a multiply and an
// add.  1/c' is the correctly rounded reciprocal.
//
// Row-dot order.  Rows of M evolve independently.  A row of d_k values is
// split over the 4 lanes of a quad; lane l holds the column groups l, l+4,
// l+8, ... (columns 4(l+4m) .. 4(l+4m)+3).  Each lane keeps two partial sums
// (a packed fp32 pair): columns 4c and 4c+2 of each group go to the first,
// 4c+1 and 4c+3 to the second, groups in ascending m, one fused multiply-add
// per element starting from +0; the lane partial is first + second; the quad
// then adds x += shfl_xor(x,1); x += shfl_xor(x,2).  IEEE addition is
// commutative, so all four lanes end with identical bits.  How many rows a
// thread holds, and how the kernels interleave rows, does not change any
// row's bits.  Packed fp32 operations (fma.rn.f32x2 / mul.rn.f32x2) are two
// independent IEEE round-to-nearest operations.
//
// Every operation is written with an explicit round-to-nearest intrinsic so
// that the compiler cannot contract or reorder it (the library is also built
// with --fmad=false).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

constexpr int kChunk = 64;        // chunk size C supported by the kernels
constexpr int kQuad = 4;          // lanes per state row
constexpr unsigned kFull = 0xffffffffu;

constexpr int kErrCuSeqlens = 1;  // GDN_DEVERR_CU_SEQLENS
constexpr int kErrPos = 2;        // GDN_DEVERR_POS
constexpr int kErrTimeout = 4;    // GDN_DEVERR_TIMEOUT

// ----------------------------------------------------------------------------
// Loads / stores with conversion to fp32
// ----------------------------------------------------------------------------
__device__ __forceinline__ float4 ld4(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}
__device__ __forceinline__ float4 ld4(const __nv_bfloat16* p) {
  uint2 raw = *reinterpret_cast<const uint2*>(p);
  __nv_bfloat162 lo = *reinterpret_cast<__nv_bfloat162*>(&raw.x);
  __nv_bfloat162 hi = *reinterpret_cast<__nv_bfloat162*>(&raw.y);
  float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ float ld1(const float* p) { return *p; }
__device__ __forceinline__ float ld1(const __nv_bfloat16* p) { return __bfloat162float(*p); }

__device__ __forceinline__ void st1(float* p, float x) { *p = x; }
__device__ __forceinline__ void st1(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// Four consecutive elements of a shared-memory row as fp32 (bf16 widening is
// a bit shift, exact).
__device__ __forceinline__ float4 sld4(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}
__device__ __forceinline__ float4 sld4(const __nv_bfloat16* p) {
  const uint2 r = *reinterpret_cast<const uint2*>(p);
  return make_float4(__uint_as_float(r.x << 16), __uint_as_float(r.x & 0xffff0000u),
                     __uint_as_float(r.y << 16), __uint_as_float(r.y & 0xffff0000u));
}

// ----------------------------------------------------------------------------
// The pinned step arithmetic
// ----------------------------------------------------------------------------
__device__ __forceinline__ float quad_sum(float x) {
  x = __fadd_rn(x, __shfl_xor_sync(kFull, x, 1));
  x = __fadd_rn(x, __shfl_xor_sync(kFull, x, 2));
  return x;
}

__device__ __forceinline__ float step_decay(float g) { return expf(g); }

__device__ __forceinline__ float step_u(float a, float beta, float p, float v) {
  return __fmul_rn(beta, __fmaf_rn(-a, p, v));
}

// Smallest scale kept without renormalising: 2^-64.
__device__ __forceinline__ bool scale_ok(float c) { return c >= 5.42101086242752217e-20f; }

__device__ __forceinline__ float2 f2(float x, float y) { return make_float2(x, y); }

// State slice of one thread: RT rows x M4 groups of 4 columns, each group held
// as two float2 (columns 4c, 4c+1 and 4c+2, 4c+3).
template <int RT, int M4>
struct Slice {
  float2 s[RT][M4][2];
};

// out[i] = lane-partial dot of row i with x (x fetched per group m as a
// float4).  Columns 4c and 4c+2 of every group accumulate into the .x half,
// 4c+1 and 4c+3 into the .y half (packed fp32 FMA, groups ascending); the
// lane partial is .x + .y.
template <int RT, int M4, class Fetch>
__device__ __forceinline__ void slice_dot(const Slice<RT, M4>& S, Fetch fx, float (&out)[RT]) {
  float2 acc[RT];
#pragma unroll
  for (int i = 0; i < RT; i++) acc[i] = f2(0.f, 0.f);
#pragma unroll
  for (int m = 0; m < M4; m++) {
    const float4 x = fx(m);
    const float2 x01 = f2(x.x, x.y), x23 = f2(x.z, x.w);
#pragma unroll
    for (int i = 0; i < RT; i++) {
      acc[i] = __ffma2_rn(S.s[i][m][0], x01, acc[i]);
      acc[i] = __ffma2_rn(S.s[i][m][1], x23, acc[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < RT; i++) out[i] = __fadd_rn(acc[i].x, acc[i].y);
}

// Update every mantissa element and, in the same sweep, accumulate the
// lane-partial dots with q (the output) and, when NEXT, with the next
// token's key (the next step's dot), in the slice_dot order, so the fused
// dots carry the same bits as separate slice_dot sweeps.
//   RENORM = false:  M <- fma(w_r, k_j, M)          (w = u / c')
//   RENORM = true:   M <- fma(c', M, u_r * k_j)     (w holds u, cn = c')
template <bool NEXT, bool RENORM, int RT, int M4, class FK, class FQ, class FN>
__device__ __forceinline__ void slice_update(Slice<RT, M4>& S, float cn, const float (&w)[RT],
                                             FK fk, FQ fq, FN fn, float (&oout)[RT],
                                             float (&pout)[RT]) {
  float2 oacc[RT], pacc[RT];
#pragma unroll
  for (int i = 0; i < RT; i++) oacc[i] = pacc[i] = f2(0.f, 0.f);
  const float2 cc = f2(cn, cn);
#pragma unroll
  for (int m = 0; m < M4; m++) {
    const float4 k4 = fk(m);
    const float4 q4 = fq(m);
    float4 n4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (NEXT) n4 = fn(m);
    const float2 k01 = f2(k4.x, k4.y), k23 = f2(k4.z, k4.w);
    const float2 q01 = f2(q4.x, q4.y), q23 = f2(q4.z, q4.w);
    const float2 n01 = f2(n4.x, n4.y), n23 = f2(n4.z, n4.w);
#pragma unroll
    for (int i = 0; i < RT; i++) {
      const float2 ww = f2(w[i], w[i]);
      float2 s01, s23;
      if (RENORM) {
        s01 = __ffma2_rn(cc, S.s[i][m][0], __fmul2_rn(ww, k01));
        s23 = __ffma2_rn(cc, S.s[i][m][1], __fmul2_rn(ww, k23));
      } else {
        s01 = __ffma2_rn(ww, k01, S.s[i][m][0]);
        s23 = __ffma2_rn(ww, k23, S.s[i][m][1]);
      }
      S.s[i][m][0] = s01;
      S.s[i][m][1] = s23;
      oacc[i] = __ffma2_rn(s01, q01, oacc[i]);
      oacc[i] = __ffma2_rn(s23, q23, oacc[i]);
      if (NEXT) {
        pacc[i] = __ffma2_rn(s01, n01, pacc[i]);
        pacc[i] = __ffma2_rn(s23, n23, pacc[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < RT; i++) {
    oout[i] = __fadd_rn(oacc[i].x, oacc[i].y);
    pout[i] = __fadd_rn(pacc[i].x, pacc[i].y);
  }
}

// One token on a slice: given the quad-reduced dot pd = dot(M_r, k) of each
// row and the scale c, apply the step (with NEXT, also return the next
// token's dot in pd), write o (before `scale`) to ov and update c.
template <bool NEXT, int RT, int M4, class FK, class FQ, class FN, class FV>
__device__ __forceinline__ void slice_token(Slice<RT, M4>& S, float& c, float a, float beta,
                                            FV fv, FK fk, FQ fq, FN fn, float (&pd)[RT],
                                            float (&ov)[RT]) {
  float u[RT], oacc[RT], pacc[RT];
#pragma unroll
  for (int i = 0; i < RT; i++) u[i] = step_u(a, beta, __fmul_rn(c, pd[i]), fv(i));
  const float cn = __fmul_rn(a, c);
  float cnew;
  if (scale_ok(cn)) {
    const float d = __frcp_rn(cn);
    float w[RT];
#pragma unroll
    for (int i = 0; i < RT; i++) w[i] = __fmul_rn(u[i], d);
    slice_update<NEXT, false, RT, M4>(S, cn, w, fk, fq, fn, oacc, pacc);
    cnew = cn;
  } else {
    slice_update<NEXT, true, RT, M4>(S, cn, u, fk, fq, fn, oacc, pacc);
    cnew = 1.f;
  }
  c = cnew;
#pragma unroll
  for (int i = 0; i < RT; i++) {
    ov[i] = __fmul_rn(cnew, quad_sum(oacc[i]));
    if (NEXT) pd[i] = quad_sum(pacc[i]);
  }
}

// Column offset (in floats) of group m for quad lane l.
__device__ __forceinline__ int group_col(int l, int m) { return 4 * (l + kQuad * m); }

template <int RT, int M4>
__device__ __forceinline__ void slice_load(Slice<RT, M4>& S, const float* rows, int ld, int r0,
                                           int l) {
#pragma unroll
  for (int i = 0; i < RT; i++)
#pragma unroll
    for (int m = 0; m < M4; m++) {
      const float4 x = ld4(rows + (size_t)(r0 + i) * ld + group_col(l, m));
      S.s[i][m][0] = f2(x.x, x.y);
      S.s[i][m][1] = f2(x.z, x.w);
    }
}

// Boundary-state rows in the forward workspace keep their 16-byte pieces
// permuted inside every 128-byte line: piece g of row r is stored at piece
// (g & ~7) | ((g ^ r) & 7), so that rows written one per thread through
// shared memory hit distinct banks.  Column c (a multiple of 4) of row r:
__device__ __forceinline__ int bst_col(int r, int c) {
  const int g = c >> 2;
  return ((g & ~7) | ((g ^ r) & 7)) << 2;
}

// slice_load from the permuted boundary-state layout.
template <int RT, int M4>
__device__ __forceinline__ void slice_load_bst(Slice<RT, M4>& S, const float* rows, int ld,
                                               int r0, int l) {
#pragma unroll
  for (int i = 0; i < RT; i++)
#pragma unroll
    for (int m = 0; m < M4; m++) {
      const int r = r0 + i;
      const float4 x = ld4(rows + (size_t)r * ld + bst_col(r, group_col(l, m)));
      S.s[i][m][0] = f2(x.x, x.y);
      S.s[i][m][1] = f2(x.z, x.w);
    }
}

template <int RT, int M4>
__device__ __forceinline__ void slice_store(const Slice<RT, M4>& S, float* rows, int ld, int r0,
                                            int l) {
#pragma unroll
  for (int i = 0; i < RT; i++)
#pragma unroll
    for (int m = 0; m < M4; m++) {
      const float4 x = make_float4(S.s[i][m][0].x, S.s[i][m][0].y, S.s[i][m][1].x,
                                   S.s[i][m][1].y);
      *reinterpret_cast<float4*>(rows + (size_t)(r0 + i) * ld + group_col(l, m)) = x;
    }
}

// Store c * M (the state itself) instead of the mantissa.
template <int RT, int M4>
__device__ __forceinline__ void slice_store_scaled(const Slice<RT, M4>& S, float c, float* rows,
                                                   int ld, int r0, int l) {
  const float2 cc = f2(c, c);
#pragma unroll
  for (int i = 0; i < RT; i++)
#pragma unroll
    for (int m = 0; m < M4; m++) {
      const float2 a = __fmul2_rn(cc, S.s[i][m][0]), b = __fmul2_rn(cc, S.s[i][m][1]);
      *reinterpret_cast<float4*>(rows + (size_t)(r0 + i) * ld + group_col(l, m)) =
          make_float4(a.x, a.y, b.x, b.y);
    }
}

}  // namespace gdn
