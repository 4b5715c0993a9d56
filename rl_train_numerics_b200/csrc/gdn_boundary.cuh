// gdn_boundary.cuh -- the chunk boundary function (first CPR pass and the
// decode resync), on tensor cores.
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
//   Tb    = T diag(beta_m exp(G_m)),  Tv = T diag(beta_m)
//   U     = Tv V - Tb (K S0^T)              C x d_v
//   S_C   = exp(G_C) S0 + U^T diag(exp(G_C - G_i)) K
//
// "Prep" (G, A, T, Tb, Tv) depends only on the chunk's tokens and runs for all
// chunks in parallel; the "walk" (last two lines) is the serial step from one
// boundary state to the next.  The forward's first pass and the decode resync
// call exactly these device functions, so boundary states are bitwise
// identical wherever they are computed.
//
// Contractions run on the tensor cores (mma.sync m16n8k16, bf16 operands,
// fp32 accumulation).  Operands that are not exactly bf16 (the fp32 state,
// Tb, Tv, the intermediate K S0^T and U, and fp32 inputs) are split exactly
// into bf16 terms (gdn_mma.cuh); the products of all term pairs down to the
// finer split's precision are accumulated in a fixed order.  That keeps the
// boundary at about fp32 accuracy: two terms (16 significant bits) for bf16
// inputs, whose K and V are exact in bf16, and three terms (24 bits) for fp32
// inputs.
//
// Fixed evaluation order (part of the rounding schedule):
//   G        double, ascending i
//   P=KK^T   k16 steps ascending; split pairs in SplitPairs order
//   A_ij     (beta_i * expf((float)(G_i - G_j))) * P_ij
//   T        right-looking substitution: T_ij accumulates -A_im T_mj over
//            m = j .. i-1 (one fma each)
//   Tb, Tv   T_im * (beta_m expf(G_m)) and T_im * beta_m, then split
//   Y        (S0 K^T): k16 steps over the key channel ascending
//   U^T      one accumulator: per k16 step over m (ascending, up to the
//            diagonal block), first + V^T Tv^T then - Y Tb^T
//   Ud       exp(G_C - G_i) * U^T
//   S_C      accumulator starts at exp(G_C) * S0, then k16 steps over i
#pragma once

#include "gdn_common.cuh"
#include "gdn_mma.cuh"

namespace gdn {

constexpr int kBndThreads = 128;  // block size of every kernel that runs the prep

// Split counts per input dtype (see the header comment).
template <class IN>
struct Splits;
template <>
struct Splits<__nv_bfloat16> {
  static constexpr int S = 2;  // state, K S0^T, U (walk A operands)
  static constexpr int W = 2;  // Tb, Tv
  static constexpr int K = 1;  // keys and values
};
template <>
struct Splits<float> {
  static constexpr int S = 3;
  static constexpr int W = 3;
  static constexpr int K = 3;
};

constexpr size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// What the walk needs from the prep of one (chunk, head): the walk pack.  It
// is copied as raw bytes (global <-> shared), so its layout is the shared
// memory layout: bf16 planes with padded rows (bank-conflict-free ldmatrix).
template <int D, class IN>
struct PackHead {
  static constexpr int NW = Splits<IN>::W;
  static constexpr int LDT = kChunk + 8;
  __nv_bfloat16 Tb[NW][kChunk][LDT];
  __nv_bfloat16 Tv[NW][kChunk][LDT];
  float dvec[kChunk];
  float gamma[4];  // [0] = exp(G_C)
};

// Keys and values of one chunk as bf16 term planes (padded rows).
template <int D, class IN>
struct KVPlanes {
  static constexpr int NK = Splits<IN>::K;
  static constexpr int LDB = D + 8;
  __nv_bfloat16 K[NK][kChunk][LDB];
  __nv_bfloat16 V[NK][kChunk][LDB];
};

template <int D, class IN>
constexpr size_t pack_size() {
  return round_up(sizeof(PackHead<D, IN>), 128);
}

// Shared memory of the prep.  AT holds A transposed with padded columns:
// AT[m][i] = A_im for i > m (zero elsewhere), so a column of A is contiguous.
template <int D, class IN>
struct PrepSmem {
  static constexpr int NW = Splits<IN>::W, NK = Splits<IN>::K;
  static constexpr int LDB = D + 8;
  PackHead<D, IN> head;
  __nv_bfloat16 K[NK][kChunk][LDB];
  float AT[kChunk][kChunk];
  double G[kChunk];
  float beta[kChunk];
  float g[kChunk];
  float bg[kChunk];
};

// Stage the rows of a [C][D] block (row stride ld elements) into bf16 term
// planes: bf16 inputs are copied with cp.async (the caller commits and waits),
// fp32 inputs are split into three bf16 terms with plain loads and stores.
template <int D, class IN>
__device__ __forceinline__ void stage_planes(__nv_bfloat16 (*dst)[kChunk][D + 8], const IN* src,
                                             size_t ld, int nthreads) {
  constexpr int NK = Splits<IN>::K;
  if constexpr (NK == 1) {
    constexpr int P = D / 8;  // 16-byte pieces per row
    for (int e = threadIdx.x; e < kChunk * P; e += nthreads) {
      const int r = e / P, c = (e % P) * 8;
      cp_async16(&dst[0][r][c], src + (size_t)r * ld + c);
    }
  } else {
    constexpr int G4 = D / 4;
    for (int e = threadIdx.x; e < kChunk * G4; e += nthreads) {
      const int r = e / G4, c = (e % G4) * 4;
      const float4 x4 = ld4(src + (size_t)r * ld + c);
      const float xs[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
      for (int q = 0; q < 4; q++) {
        __nv_bfloat16 s[NK];
        split_bf16<NK>(xs[q], s);
#pragma unroll
        for (int t = 0; t < NK; t++) dst[t][r][c + q] = s[t];
      }
    }
  }
}

// ldmatrix address of the A fragment (x4) of rows r0.., columns c0.. in a
// row-major bf16 matrix with row stride ld.
__device__ __forceinline__ const __nv_bfloat16* afrag_addr(const __nv_bfloat16* base, int ld,
                                                           int r0, int c0) {
  const int lane = threadIdx.x & 31, mi = lane >> 3;
  return base + (size_t)(r0 + (mi & 1) * 8 + (lane & 7)) * ld + c0 + (mi >> 1) * 8;
}
// A fragment (x4.trans) of A[r][c] = M[c][r] (M row-major, rows = the k index).
__device__ __forceinline__ const __nv_bfloat16* afrag_t_addr(const __nv_bfloat16* base, int ld,
                                                             int r0, int c0) {
  const int lane = threadIdx.x & 31, mi = lane >> 3;
  return base + (size_t)(c0 + (mi >> 1) * 8 + (lane & 7)) * ld + r0 + (mi & 1) * 8;
}
// B fragments (x4 = two n8 tiles) of B[k][n] = M[n][k] (M row-major, rows = n).
__device__ __forceinline__ const __nv_bfloat16* bfrag_nk_addr(const __nv_bfloat16* base, int ld,
                                                              int n0, int k0) {
  const int lane = threadIdx.x & 31, mi = lane >> 3;
  return base + (size_t)(n0 + (mi >> 1) * 8 + (lane & 7)) * ld + k0 + (mi & 1) * 8;
}
// B fragments (x4.trans = two n8 tiles) of B[k][n] = M[k][n] (M row-major, rows = k).
__device__ __forceinline__ const __nv_bfloat16* bfrag_kn_addr(const __nv_bfloat16* base, int ld,
                                                              int k0, int n0) {
  const int lane = threadIdx.x & 31, mi = lane >> 3;
  return base + (size_t)(k0 + (mi & 1) * 8 + (lane & 7)) * ld + n0 + (mi >> 1) * 8;
}

// Stage one chunk for the prep: keys (rows at stride ld), beta and g
// (stride ldbg).  Ends with the data landed and a block barrier.
template <int D, class IN>
__device__ __forceinline__ void prep_stage(PrepSmem<D, IN>& sm, const IN* k, size_t ld,
                                           const float* bsrc, const float* gsrc, size_t ldbg) {
  stage_planes<D, IN>(sm.K, k, ld, kBndThreads);
  cp_async_commit();
  for (int i = threadIdx.x; i < kChunk; i += kBndThreads) {
    sm.beta[i] = bsrc[i * ldbg];
    sm.g[i] = gsrc[i * ldbg];
  }
  cp_async_wait<0>();
  __syncthreads();
}

// Prep of one chunk: sm.K, sm.beta, sm.g staged -> sm.head (Tb, Tv, dvec,
// gamma).  All kBndThreads threads; ends with a block barrier.
template <int D, class IN>
__device__ void bnd_prep(PrepSmem<D, IN>& sm) {
  constexpr int NW = Splits<IN>::W, NK = Splits<IN>::K;
  constexpr int LDB = PrepSmem<D, IN>::LDB;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;

  // P = K K^T on the tensor cores; warp w owns rows 16w..16w+15 (m-tile w)
  // and the n8 tiles that reach below the diagonal.
  float acc[8][4];
  {
    using PP = SplitPairs<NK, NK>;
    const int m0 = 16 * warp;
#pragma unroll
    for (int n = 0; n < 8; n++)
#pragma unroll
      for (int e = 0; e < 4; e++) acc[n][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ks++) {
      uint32_t a[NK][4];
#pragma unroll
      for (int t = 0; t < NK; t++) ldsm_x4(a[t], afrag_addr(&sm.K[t][0][0], LDB, m0, 16 * ks));
#pragma unroll
      for (int np = 0; np < 4; np++) {
        if (np <= warp) {
          uint32_t b[NK][4];
#pragma unroll
          for (int t = 0; t < NK; t++)
            ldsm_x4(b[t], bfrag_nk_addr(&sm.K[t][0][0], LDB, 16 * np, 16 * ks));
#pragma unroll
          for (int p = 0; p < PP::kCount; p++) {
            mma16816(acc[2 * np], a[PP::a(p)], b[PP::b(p)][0], b[PP::b(p)][1]);
            mma16816(acc[2 * np + 1], a[PP::a(p)], b[PP::b(p)][2], b[PP::b(p)][3]);
          }
        }
      }
    }
  }
  if (tid == 0) {
    double s = 0.0;
    for (int i = 0; i < kChunk; i++) {
      s += (double)sm.g[i];
      sm.G[i] = s;
    }
  }
  for (int e = tid; e < kChunk * kChunk / 4; e += kBndThreads)
    reinterpret_cast<float4*>(&sm.AT[0][0])[e] = make_float4(0.f, 0.f, 0.f, 0.f);
  __syncthreads();
  {
    const int m0 = 16 * warp;
#pragma unroll
    for (int n = 0; n < 8; n++) {
      if (n < 2 * warp + 2) {
#pragma unroll
        for (int e = 0; e < 4; e++) {
          const int i = m0 + gq + (e >> 1) * 8, j = 8 * n + 2 * tq + (e & 1);
          if (j < i) {
            const float decay = expf(__double2float_rn(sm.G[i] - sm.G[j]));
            sm.AT[j][i] = __fmul_rn(__fmul_rn(sm.beta[i], decay), acc[n][e]);
          }
        }
      }
    }
  }
  for (int i = tid; i < kChunk; i += kBndThreads) {
    sm.bg[i] = __fmul_rn(sm.beta[i], expf(__double2float_rn(sm.G[i])));
    sm.head.dvec[i] = expf(__double2float_rn(sm.G[kChunk - 1] - sm.G[i]));
  }
  if (tid == 0) {
    sm.head.gamma[0] = expf(__double2float_rn(sm.G[kChunk - 1]));
    sm.head.gamma[1] = sm.head.gamma[2] = sm.head.gamma[3] = 0.f;
  }
  __syncthreads();

  // T = (I + A)^{-1}, column j held in registers by thread j: right-looking
  // over m, so T_ij accumulates -A_im T_mj in ascending m.  Steps m < j only
  // add signed zeros to zeros (T_mj = 0 there), leaving the bits unchanged.
  // Then Tb = T diag(beta*gamma), Tv = T diag(beta), split into bf16 terms.
  if (tid < kChunk) {
    const int j = tid;
    float t[kChunk];
#pragma unroll
    for (int i = 0; i < kChunk; i++) t[i] = (i == j) ? 1.f : 0.f;
#pragma unroll
    for (int m = 0; m < kChunk - 1; m++) {
      const float tm = t[m];
      const float* col = &sm.AT[m][0];
#pragma unroll
      for (int i4 = (m + 1) & ~3; i4 < kChunk; i4 += 4) {
        const float4 a4 = *reinterpret_cast<const float4*>(col + i4);
        const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
        for (int q = 0; q < 4; q++)
          if (i4 + q > m) t[i4 + q] = __fmaf_rn(-av[q], tm, t[i4 + q]);
      }
    }
    const float bgj = sm.bg[j], bj = sm.beta[j];
#pragma unroll
    for (int i = 0; i < kChunk; i++) {
      __nv_bfloat16 sb[NW], sv[NW];
      split_bf16<NW>(__fmul_rn(t[i], bgj), sb);
      split_bf16<NW>(__fmul_rn(t[i], bj), sv);
#pragma unroll
      for (int q = 0; q < NW; q++) {
        sm.head.Tb[q][i][j] = sb[q];
        sm.head.Tv[q][i][j] = sv[q];
      }
    }
  }
  __syncthreads();
}

// ----------------------------------------------------------------------------
// Walk step: 16 state rows per warp, held in accumulator layout
// (sacc[n][e]: row r0 + g + 8*(e>>1), column 8n + 2t + (e&1)).
// ----------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ void sacc_load(float (&sacc)[D / 8][4], const float* S, int r0) {
  const int lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
#pragma unroll
  for (int n = 0; n < D / 8; n++)
#pragma unroll
    for (int hf = 0; hf < 2; hf++) {
      const float2 x =
          *reinterpret_cast<const float2*>(S + (size_t)(r0 + gq + 8 * hf) * D + 8 * n + 2 * tq);
      sacc[n][2 * hf] = x.x;
      sacc[n][2 * hf + 1] = x.y;
    }
}

// Store 16 rows; lanes t and t^1 swap halves so that every lane writes one
// 16-byte run of one row.
template <int D>
__device__ __forceinline__ void sacc_store(const float (&sacc)[D / 8][4], float* S, int r0) {
  const int lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3, odd = tq & 1;
#pragma unroll
  for (int n = 0; n < D / 8; n++) {
    // even t keeps row g and receives its partner's row-g pair; odd t keeps
    // row g+8 and receives its partner's row-(g+8) pair.
    const float s0 = odd ? sacc[n][0] : sacc[n][2];
    const float s1 = odd ? sacc[n][1] : sacc[n][3];
    const float r0v = __shfl_xor_sync(kFull, s0, 1);
    const float r1v = __shfl_xor_sync(kFull, s1, 1);
    float4 out;
    if (!odd) out = make_float4(sacc[n][0], sacc[n][1], r0v, r1v);
    else out = make_float4(r0v, r1v, sacc[n][2], sacc[n][3]);
    const int row = r0 + gq + 8 * odd, col = 8 * n + 2 * (tq & 2);
    *reinterpret_cast<float4*>(S + (size_t)row * D + col) = out;
  }
}

template <int D>
__device__ __forceinline__ void sacc_zero(float (&sacc)[D / 8][4]) {
#pragma unroll
  for (int n = 0; n < D / 8; n++)
#pragma unroll
    for (int e = 0; e < 4; e++) sacc[n][e] = 0.f;
}

// One boundary step for the warp's 16 rows (r0 = first row within the head):
//   Y  = S K^T                      (16 x C)
//   Z  = (V^T Tv^T) - Y Tb^T        (= U^T for these rows)
//   S <- exp(G_C) S + (dvec * Z) K
// hd (Tb, Tv, dvec, gamma) and the K, V planes are in shared memory.
template <int D, class IN>
__device__ __forceinline__ void bnd_walk_warp(float (&sacc)[D / 8][4], const PackHead<D, IN>& hd,
                                              const __nv_bfloat16* Kp, const __nv_bfloat16* Vp,
                                              int r0) {
  constexpr int NS = Splits<IN>::S, NW = Splits<IN>::W, NK = Splits<IN>::K;
  constexpr int LDB = D + 8, LDT = kChunk + 8;
  constexpr size_t PL = (size_t)kChunk * LDB;  // elements per K/V plane
  const int lane = threadIdx.x & 31, tq = lane & 3;
  // Y = S K^T
  float y[kChunk / 8][4];
#pragma unroll
  for (int n = 0; n < kChunk / 8; n++)
#pragma unroll
    for (int e = 0; e < 4; e++) y[n][e] = 0.f;
  {
    using PP = SplitPairs<NS, NK>;
#pragma unroll
    for (int ks = 0; ks < D / 16; ks++) {
      uint32_t a[NS][4];
      acc_to_afrag<NS>(sacc[2 * ks], sacc[2 * ks + 1], a);
#pragma unroll
      for (int np = 0; np < kChunk / 16; np++) {
        uint32_t b[NK][4];
#pragma unroll
        for (int q = 0; q < NK; q++) ldsm_x4(b[q], bfrag_nk_addr(Kp + q * PL, LDB, 16 * np, 16 * ks));
#pragma unroll
        for (int p = 0; p < PP::kCount; p++) {
          mma16816(y[2 * np], a[PP::a(p)], b[PP::b(p)][0], b[PP::b(p)][1]);
          mma16816(y[2 * np + 1], a[PP::a(p)], b[PP::b(p)][2], b[PP::b(p)][3]);
        }
      }
    }
  }
  // Z = V^T Tv^T - Y Tb^T  (Tb, Tv vanish above the diagonal block)
  float z[kChunk / 8][4];
#pragma unroll
  for (int n = 0; n < kChunk / 8; n++)
#pragma unroll
    for (int e = 0; e < 4; e++) z[n][e] = 0.f;
  {
    using PV = SplitPairs<NK, NW>;
    using PY = SplitPairs<NS, NW>;
#pragma unroll
    for (int ks = 0; ks < kChunk / 16; ks++) {
      uint32_t av[NK][4], ay[NS][4];
#pragma unroll
      for (int q = 0; q < NK; q++) ldsm_x4_t(av[q], afrag_t_addr(Vp + q * PL, LDB, r0, 16 * ks));
      float ny0[4], ny1[4];
#pragma unroll
      for (int e = 0; e < 4; e++) {
        ny0[e] = -y[2 * ks][e];
        ny1[e] = -y[2 * ks + 1][e];
      }
      acc_to_afrag<NS>(ny0, ny1, ay);
#pragma unroll
      for (int np = ks; np < kChunk / 16; np++) {
        uint32_t bv[NW][4], bb[NW][4];
#pragma unroll
        for (int q = 0; q < NW; q++) {
          ldsm_x4(bv[q], bfrag_nk_addr(&hd.Tv[q][0][0], LDT, 16 * np, 16 * ks));
          ldsm_x4(bb[q], bfrag_nk_addr(&hd.Tb[q][0][0], LDT, 16 * np, 16 * ks));
        }
#pragma unroll
        for (int p = 0; p < PV::kCount; p++) {
          mma16816(z[2 * np], av[PV::a(p)], bv[PV::b(p)][0], bv[PV::b(p)][1]);
          mma16816(z[2 * np + 1], av[PV::a(p)], bv[PV::b(p)][2], bv[PV::b(p)][3]);
        }
#pragma unroll
        for (int p = 0; p < PY::kCount; p++) {
          mma16816(z[2 * np], ay[PY::a(p)], bb[PY::b(p)][0], bb[PY::b(p)][1]);
          mma16816(z[2 * np + 1], ay[PY::a(p)], bb[PY::b(p)][2], bb[PY::b(p)][3]);
        }
      }
    }
  }
  // Ud = dvec * Z
#pragma unroll
  for (int n = 0; n < kChunk / 8; n++)
#pragma unroll
    for (int e = 0; e < 4; e++) z[n][e] = __fmul_rn(hd.dvec[8 * n + 2 * tq + (e & 1)], z[n][e]);
  // S' = gamma S + Ud^T K
  {
    const float gam = hd.gamma[0];
#pragma unroll
    for (int n = 0; n < D / 8; n++)
#pragma unroll
      for (int e = 0; e < 4; e++) sacc[n][e] = __fmul_rn(gam, sacc[n][e]);
    using PP = SplitPairs<NS, NK>;
#pragma unroll
    for (int ks = 0; ks < kChunk / 16; ks++) {
      uint32_t a[NS][4];
      acc_to_afrag<NS>(z[2 * ks], z[2 * ks + 1], a);
#pragma unroll
      for (int np = 0; np < D / 16; np++) {
        uint32_t b[NK][4];
#pragma unroll
        for (int q = 0; q < NK; q++) ldsm_x4_t(b[q], bfrag_kn_addr(Kp + q * PL, LDB, 16 * ks, 16 * np));
#pragma unroll
        for (int p = 0; p < PP::kCount; p++) {
          mma16816(sacc[2 * np], a[PP::a(p)], b[PP::b(p)][0], b[PP::b(p)][1]);
          mma16816(sacc[2 * np + 1], a[PP::a(p)], b[PP::b(p)][2], b[PP::b(p)][3]);
        }
      }
    }
  }
}

}  // namespace gdn
