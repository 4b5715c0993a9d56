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

// State slice of one thread: RT rows x M4 groups of 4 columns, each group held
// as two float2 (columns 4c, 4c+1 and 4c+2, 4c+3).
template <int RT, int M4>
struct Slice {
  float2 s[RT][M4][2];
};

__device__ __forceinline__ float2 f2(float x, float y) { return make_float2(x, y); }

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

// Update every element with s <- fma(a, s, u*k), and in the same sweep
// accumulate the lane-partial dots with q (the output) and, when NEXT, with
// the next token's key (the next step's p), in the slice_dot order, so the
// fused dots carry the same bits as separate slice_dot sweeps.
template <bool NEXT, int RT, int M4, class FK, class FQ, class FN>
__device__ __forceinline__ void slice_update(Slice<RT, M4>& S, float a, const float (&u)[RT],
                                             FK fk, FQ fq, FN fn, float (&oout)[RT],
                                             float (&pout)[RT]) {
  float2 oacc[RT], pacc[RT];
#pragma unroll
  for (int i = 0; i < RT; i++) oacc[i] = pacc[i] = f2(0.f, 0.f);
  const float2 aa = f2(a, a);
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
      const float2 uu = f2(u[i], u[i]);
      const float2 s01 = __ffma2_rn(aa, S.s[i][m][0], __fmul2_rn(uu, k01));
      const float2 s23 = __ffma2_rn(aa, S.s[i][m][1], __fmul2_rn(uu, k23));
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

}  // namespace gdn
