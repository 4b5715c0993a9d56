// gdn_boundary.cuh -- the chunk boundary function (first CPR pass and the
// decode resync).
//
// "NovaSky's IsoExec Fixes the Hidden Math Bug Corrupting AI Training Runs",
// section "Solving the linear-attention headache": a first pass computes the
// recurrent state at chunk boundaries; decode re-synchronises its state every
// chunk-size tokens with the same computation.  The pages do not write the
// boundary formula; it is derived here from the recurrence
// S_i = alpha_i S_{i-1} (I - beta_i k_i k_i^T) + beta_i v_i k_i^T
// (the UT / WY form of a product of generalised Householder updates):
//
//   G_i   = g_1 + ... + g_i                 (cumulative log-decay, in double)
//   A_ij  = beta_i exp(G_i - G_j) (k_i . k_j)       j < i
//   T     = (I + A)^{-1}                    unit lower triangular
//   W     = T diag(beta_m exp(G_m)) K       C x d_k
//   U~    = T diag(beta_m) V                C x d_v
//   U     = U~ - W S0^T                     C x d_v
//   S_C   = exp(G_C) S0 + U^T diag(exp(G_C - G_i)) K
//
// The first five lines depend only on the chunk's tokens ("prep"); the last
// two are the serial "walk" from one boundary state to the next.  Both CPR
// passes and the decode resync call exactly these device functions, with the
// same block size, so boundary states are bitwise identical wherever they are
// computed.  A row of S0 maps to the same row of S_C, so the walk runs one
// row per thread.
//
// Fixed evaluation order (fp32 unless stated):
//   G        double, ascending i
//   dots     fma chains from +0, ascending index
//   T        right-looking substitution: T_ij accumulates -A_im T_mj for
//            m = j, j+1, ..., i-1 (one fma each)
//   W, U~    T_im * (beta_m exp(G_m)) rounded, then fma over m = 0..i
//   U        Ud_i = exp(G_C - G_i) * (U~_ir - dot(S0_r, W_i))
//   S_C      start from exp(G_C) * S0_rj, then fma over i ascending
#pragma once

#include "gdn_common.cuh"

namespace gdn {

constexpr int kBndThreads = 128;  // block size of every kernel that calls these

template <int D>
struct BndSmem {
  float K[kChunk][D];
  float V[kChunk][D];
  float W[kChunk][D];
  float Ut[kChunk][D];
  union {
    struct {
      float A[kChunk][kChunk];
      float T[kChunk][kChunk];
    } at;
    float Ud[kChunk][D];
  } u;
  double G[kChunk];
  float beta[kChunk];
  float g[kChunk];
  float bg[kChunk];
  float dvec[kChunk];
  float gammaC;
};

// Walk-only shared memory (forward pass 1 stages prep results from global).
template <int D>
struct WalkSmem {
  float K[kChunk][D];
  float W[kChunk][D];
  float Ut[kChunk][D];
  float Ud[kChunk][D];
  float dvec[kChunk];
  float gammaC;
};

// Stage one chunk's keys/values/beta/g (rows at stride `ld` elements) into
// fp32 shared memory.  Bit-exact widening.
template <int D, class IN>
__device__ __forceinline__ void stage_chunk_kv(float (*K)[D], float (*V)[D], float* beta,
                                               float* g, const IN* k, const IN* v, size_t ld,
                                               const float* bsrc, const float* gsrc,
                                               size_t ldbg) {
  constexpr int G4 = D / 4;
  for (int e = threadIdx.x; e < kChunk * G4; e += kBndThreads) {
    int i = e / G4, c = (e % G4) * 4;
    float4 kk = ld4(k + i * ld + c);
    float4 vv = ld4(v + i * ld + c);
    *reinterpret_cast<float4*>(&K[i][c]) = kk;
    *reinterpret_cast<float4*>(&V[i][c]) = vv;
  }
  for (int i = threadIdx.x; i < kChunk; i += kBndThreads) {
    beta[i] = bsrc[i * ldbg];
    g[i] = gsrc[i * ldbg];
  }
}

// Chunk prep: everything in the boundary that does not depend on S0.
// Inputs sm.K, sm.V, sm.beta, sm.g; outputs sm.W, sm.Ut, sm.dvec, sm.gammaC.
// Must be called by all kBndThreads threads.
template <int D>
__device__ void bnd_prep(BndSmem<D>& sm) {
  const int tid = threadIdx.x;
  if (tid == 0) {
    double acc = 0.0;
    for (int i = 0; i < kChunk; i++) {
      acc += (double)sm.g[i];
      sm.G[i] = acc;
    }
  }
  __syncthreads();
  // A (strictly lower), T = I.
  for (int e = tid; e < kChunk * kChunk; e += kBndThreads) {
    const int i = e / kChunk, j = e % kChunk;
    float a = 0.f;
    if (j < i) {
      float dot = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; c++) dot = __fmaf_rn(sm.K[i][c], sm.K[j][c], dot);
      const float decay = expf(__double2float_rn(sm.G[i] - sm.G[j]));
      a = __fmul_rn(__fmul_rn(sm.beta[i], decay), dot);
    }
    sm.u.at.A[i][j] = a;
    sm.u.at.T[i][j] = (i == j) ? 1.f : 0.f;
  }
  for (int i = tid; i < kChunk; i += kBndThreads) {
    sm.bg[i] = __fmul_rn(sm.beta[i], expf(__double2float_rn(sm.G[i])));
    sm.dvec[i] = expf(__double2float_rn(sm.G[kChunk - 1] - sm.G[i]));
  }
  if (tid == 0) sm.gammaC = expf(__double2float_rn(sm.G[kChunk - 1]));
  __syncthreads();
  // T = (I + A)^{-1}, right-looking: step m finalises row m.
  for (int m = 0; m < kChunk - 1; m++) {
    const int ni = kChunk - 1 - m, nj = m + 1;
    for (int e = tid; e < ni * nj; e += kBndThreads) {
      const int i = m + 1 + e / nj, j = e % nj;
      sm.u.at.T[i][j] = __fmaf_rn(-sm.u.at.A[i][m], sm.u.at.T[m][j], sm.u.at.T[i][j]);
    }
    __syncthreads();
  }
  // A <- T diag(beta*gamma), T <- T diag(beta)   (element-wise, own element)
  for (int e = tid; e < kChunk * kChunk; e += kBndThreads) {
    const int i = e / kChunk, m = e % kChunk;
    const float t = sm.u.at.T[i][m];
    sm.u.at.A[i][m] = __fmul_rn(t, sm.bg[m]);
    sm.u.at.T[i][m] = __fmul_rn(t, sm.beta[m]);
  }
  __syncthreads();
  for (int e = tid; e < kChunk * D; e += kBndThreads) {
    const int i = e / D, c = e % D;
    float w = 0.f, ut = 0.f;
    for (int m = 0; m <= i; m++) {
      w = __fmaf_rn(sm.u.at.A[i][m], sm.K[m][c], w);
      ut = __fmaf_rn(sm.u.at.T[i][m], sm.V[m][c], ut);
    }
    sm.W[i][c] = w;
    sm.Ut[i][c] = ut;
  }
  __syncthreads();
}

// Walk one state row r (held in registers by thread r) across one chunk.
// W, Ut, K: [kChunk][D] (shared); Ud: [kChunk][D] scratch (shared), column r
// is private to thread r.
template <int D>
__device__ __forceinline__ void bnd_walk_row(float (&s)[D], int r, const float* W,
                                             const float* Ut, const float* K, float* Ud,
                                             const float* dvec, float gammaC) {
  constexpr int IB = 8;
  for (int i0 = 0; i0 < kChunk; i0 += IB) {
    float acc[IB];
#pragma unroll
    for (int ii = 0; ii < IB; ii++) acc[ii] = 0.f;
#pragma unroll
    for (int j = 0; j < D; j += 4) {
#pragma unroll
      for (int ii = 0; ii < IB; ii++) {
        const float4 w = *reinterpret_cast<const float4*>(W + (i0 + ii) * D + j);
        acc[ii] = __fmaf_rn(s[j + 0], w.x, acc[ii]);
        acc[ii] = __fmaf_rn(s[j + 1], w.y, acc[ii]);
        acc[ii] = __fmaf_rn(s[j + 2], w.z, acc[ii]);
        acc[ii] = __fmaf_rn(s[j + 3], w.w, acc[ii]);
      }
    }
#pragma unroll
    for (int ii = 0; ii < IB; ii++) {
      const int i = i0 + ii;
      Ud[i * D + r] = __fmul_rn(dvec[i], __fsub_rn(Ut[i * D + r], acc[ii]));
    }
  }
#pragma unroll
  for (int j = 0; j < D; j++) s[j] = __fmul_rn(gammaC, s[j]);
  for (int i = 0; i < kChunk; i++) {
    const float ud = Ud[i * D + r];
#pragma unroll
    for (int j = 0; j < D; j += 4) {
      const float4 kk = *reinterpret_cast<const float4*>(K + i * D + j);
      s[j + 0] = __fmaf_rn(ud, kk.x, s[j + 0]);
      s[j + 1] = __fmaf_rn(ud, kk.y, s[j + 1]);
      s[j + 2] = __fmaf_rn(ud, kk.z, s[j + 2]);
      s[j + 3] = __fmaf_rn(ud, kk.w, s[j + 3]);
    }
  }
}

template <int D>
__device__ __forceinline__ void row_load(float (&s)[D], const float* src) {
#pragma unroll
  for (int j = 0; j < D; j += 4) {
    const float4 x = *reinterpret_cast<const float4*>(src + j);
    s[j] = x.x;
    s[j + 1] = x.y;
    s[j + 2] = x.z;
    s[j + 3] = x.w;
  }
}

template <int D>
__device__ __forceinline__ void row_store(const float (&s)[D], float* dst) {
#pragma unroll
  for (int j = 0; j < D; j += 4)
    *reinterpret_cast<float4*>(dst + j) = make_float4(s[j], s[j + 1], s[j + 2], s[j + 3]);
}

template <int D>
__device__ __forceinline__ void row_zero(float (&s)[D]) {
#pragma unroll
  for (int j = 0; j < D; j++) s[j] = 0.f;
}

}  // namespace gdn
