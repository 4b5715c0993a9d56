// gdn_common.cuh -- shared device code of the CPR Gated DeltaNet kernels.
//
// The per-token step below is the one piece of arithmetic that the
// intra-chunk fill (second CPR pass) and the decode step both run.  The
// section "Solving the linear-attention headache" of "NovaSky's IsoExec Fixes
// the Hidden Math Bug Corrupting AI Training Runs" asks that prefill,
// training and decode share one rounding schedule; here that schedule is
// fixed instruction by instruction:
//
//   a   = expf(g_t)
//   p_r = sum_j S[r][j] k_j              per-row dot (order below)
//   u_r = beta * fma(-a, p_r, v_r)
//   S[r][j] <- fma(a, S[r][j], u_r * k_j)
//   o_r = scale * sum_j S[r][j] q_j      same dot order
//
// Row-dot order.  Rows of S evolve independently.  A row of d_k values is
// split over the 4 lanes of a quad; lane l holds the float4 column groups
// l, l+4, l+8, ... (columns 4(l+4m) .. 4(l+4m)+3).  Each lane accumulates its
// groups in ascending m and, within a group, ascending column, starting from
// +0 with one fused multiply-add per element; the quad then adds
// x += shfl_xor(x,1); x += shfl_xor(x,2).  IEEE addition is commutative, so
// all four lanes end with identical bits.  How many rows a thread holds, and
// how the kernels interleave rows, does not change any row's bits.
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

__device__ __forceinline__ float step_s(float a, float s, float u, float k) {
  return __fmaf_rn(a, s, __fmul_rn(u, k));
}

// State slice of one thread: RT rows x M4 float4 groups.
template <int RT, int M4>
struct Slice {
  float s[RT][M4][4];
};

// acc[i] = lane-partial dot of row i with x (x fetched per group m).
template <int RT, int M4, class Fetch>
__device__ __forceinline__ void slice_dot(const Slice<RT, M4>& S, Fetch fx, float (&acc)[RT]) {
#pragma unroll
  for (int i = 0; i < RT; i++) acc[i] = 0.f;
#pragma unroll
  for (int m = 0; m < M4; m++) {
    const float4 x = fx(m);
#pragma unroll
    for (int i = 0; i < RT; i++) {
      acc[i] = __fmaf_rn(S.s[i][m][0], x.x, acc[i]);
      acc[i] = __fmaf_rn(S.s[i][m][1], x.y, acc[i]);
      acc[i] = __fmaf_rn(S.s[i][m][2], x.z, acc[i]);
      acc[i] = __fmaf_rn(S.s[i][m][3], x.w, acc[i]);
    }
  }
}

// Update every element with step_s, and in the same sweep accumulate the
// lane-partial dots with q (output) and, when NEXT, with the next token's key
// (the next step's p).  Accumulation order per row is the slice_dot order, so
// the fused dots carry the same bits as separate slice_dot sweeps.
template <bool NEXT, int RT, int M4, class FK, class FQ, class FN>
__device__ __forceinline__ void slice_update(Slice<RT, M4>& S, float a, const float (&u)[RT],
                                             FK fk, FQ fq, FN fn, float (&oacc)[RT],
                                             float (&pacc)[RT]) {
#pragma unroll
  for (int i = 0; i < RT; i++) {
    oacc[i] = 0.f;
    pacc[i] = 0.f;
  }
#pragma unroll
  for (int m = 0; m < M4; m++) {
    const float4 k4 = fk(m);
    const float4 q4 = fq(m);
    float4 n4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (NEXT) n4 = fn(m);
#pragma unroll
    for (int i = 0; i < RT; i++) {
      float s0 = step_s(a, S.s[i][m][0], u[i], k4.x);
      float s1 = step_s(a, S.s[i][m][1], u[i], k4.y);
      float s2 = step_s(a, S.s[i][m][2], u[i], k4.z);
      float s3 = step_s(a, S.s[i][m][3], u[i], k4.w);
      S.s[i][m][0] = s0;
      S.s[i][m][1] = s1;
      S.s[i][m][2] = s2;
      S.s[i][m][3] = s3;
      oacc[i] = __fmaf_rn(s0, q4.x, oacc[i]);
      oacc[i] = __fmaf_rn(s1, q4.y, oacc[i]);
      oacc[i] = __fmaf_rn(s2, q4.z, oacc[i]);
      oacc[i] = __fmaf_rn(s3, q4.w, oacc[i]);
      if (NEXT) {
        pacc[i] = __fmaf_rn(s0, n4.x, pacc[i]);
        pacc[i] = __fmaf_rn(s1, n4.y, pacc[i]);
        pacc[i] = __fmaf_rn(s2, n4.z, pacc[i]);
        pacc[i] = __fmaf_rn(s3, n4.w, pacc[i]);
      }
    }
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
      float4 x = ld4(rows + (size_t)(r0 + i) * ld + group_col(l, m));
      S.s[i][m][0] = x.x;
      S.s[i][m][1] = x.y;
      S.s[i][m][2] = x.z;
      S.s[i][m][3] = x.w;
    }
}

template <int RT, int M4>
__device__ __forceinline__ void slice_store(const Slice<RT, M4>& S, float* rows, int ld, int r0,
                                            int l) {
#pragma unroll
  for (int i = 0; i < RT; i++)
#pragma unroll
    for (int m = 0; m < M4; m++) {
      float4 x = make_float4(S.s[i][m][0], S.s[i][m][1], S.s[i][m][2], S.s[i][m][3]);
      *reinterpret_cast<float4*>(rows + (size_t)(r0 + i) * ld + group_col(l, m)) = x;
    }
}

}  // namespace gdn
