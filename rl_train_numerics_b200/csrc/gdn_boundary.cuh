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
//   W     = T diag(beta_m exp(G_m)) K       C x d_k
//   U~    = T diag(beta_m) V                C x d_v
//   U     = U~ - W S0^T                     C x d_v
//   S_C   = exp(G_C) S0 + U^T diag(exp(G_C - G_i)) K
//
// "Prep" (everything but the last two lines) depends only on the chunk's
// tokens and runs for all chunks in parallel; the "walk" (last two lines) is
// the serial step from one boundary state to the next.  The forward's first
// pass and the decode resync call exactly these device functions, so boundary
// states are bitwise identical wherever they are computed.
//
// Contractions run on the tensor cores (mma.sync m16n8k16, bf16 operands,
// fp32 accumulation).  Operands that are not exactly bf16 (the fp32 state,
// T, the intermediate U, and fp32 inputs) are split exactly into bf16 terms
// (gdn_mma.cuh); the products of all term pairs down to the finer split's
// precision are accumulated in a fixed order, which keeps the boundary at
// about fp32 accuracy: two terms (16 significant bits) for bf16 inputs, whose
// K and V are exact in bf16, and three terms (24 bits) for fp32 inputs.
//
// Fixed evaluation order (part of the rounding schedule):
//   G        double, ascending i
//   P=KK^T   k16 steps ascending; split pairs in SplitPairs order
//   A_ij     (beta_i * expf((float)(G_i - G_j))) * P_ij
//   T        right-looking substitution: T_ij accumulates -A_im T_mj over
//            m = j .. i-1 (one fma each)
//   W, U~    (T_im * (beta_m expf(G_m))) and (T_im * beta_m), split, then
//            k16 steps m ascending up to the diagonal block (U~ is formed
//            transposed, as V^T Tv^T)
//   U        Ud_i = exp(G_C - G_i) * (U~_ir - (S0 W^T)_ri)
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
  static constexpr int S = 2;  // state and U (walk A operands)
  static constexpr int W = 2;  // T-derived operands and W
  static constexpr int K = 1;  // keys and values
};
template <>
struct Splits<float> {
  static constexpr int S = 3;
  static constexpr int W = 3;
  static constexpr int K = 3;
};

constexpr size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// The walk pack: everything the walk needs from one (chunk, head), in the
// padded shared-memory layout (bank-conflict-free ldmatrix rows).
template <int D, class IN>
struct Pack {
  static constexpr int NW = Splits<IN>::W, NK = Splits<IN>::K;
  static constexpr int LDB = D + 8;       // bf16 row stride of W and K planes
  static constexpr int LDU = kChunk + 8;  // fp32 row stride of U~^T
  static constexpr size_t kW = 0;                                        // NW x [C][LDB] bf16
  static constexpr size_t kK = kW + (size_t)NW * kChunk * LDB * 2;       // NK x [C][LDB] bf16
  static constexpr size_t kU = kK + (size_t)NK * kChunk * LDB * 2;       // [D][LDU] fp32
  static constexpr size_t kDvec = kU + (size_t)D * LDU * 4;              // [C] fp32
  static constexpr size_t kGamma = kDvec + (size_t)kChunk * 4;           // fp32
  static constexpr size_t kBytes = round_up(kGamma + 16, 128);

  static __device__ __forceinline__ __nv_bfloat16* W(char* p, int t) {
    return reinterpret_cast<__nv_bfloat16*>(p + kW) + (size_t)t * kChunk * LDB;
  }
  static __device__ __forceinline__ __nv_bfloat16* K(char* p, int t) {
    return reinterpret_cast<__nv_bfloat16*>(p + kK) + (size_t)t * kChunk * LDB;
  }
  static __device__ __forceinline__ float* U(char* p) { return reinterpret_cast<float*>(p + kU); }
  static __device__ __forceinline__ float* dvec(char* p) {
    return reinterpret_cast<float*>(p + kDvec);
  }
  static __device__ __forceinline__ float* gamma(char* p) {
    return reinterpret_cast<float*>(p + kGamma);
  }
};

// Shared memory of the prep.  A is stored packed (strictly lower triangle,
// row-major: element (i, j), j < i, at i(i-1)/2 + j).
template <int D, class IN>
struct PrepSmem {
  static constexpr int NW = Splits<IN>::W, NK = Splits<IN>::K;
  static constexpr int LDB = D + 8, LDT = kChunk + 8;
  __nv_bfloat16 K[NK][kChunk][LDB];
  __nv_bfloat16 V[NK][kChunk][LDB];
  __nv_bfloat16 Tb[NW][kChunk][LDT];
  __nv_bfloat16 Tv[NW][kChunk][LDT];
  float A[kChunk * (kChunk - 1) / 2];
  double G[kChunk];
  float beta[kChunk];
  float g[kChunk];
  float bg[kChunk];
  float dvec[kChunk];
  float gammaC;
};

__device__ __forceinline__ constexpr int tri(int i, int j) { return i * (i - 1) / 2 + j; }

// Stage one chunk's k, v (rows at stride `ld` elements), beta, g (stride ldbg)
// into the prep's shared memory.  bf16 inputs are copied as is (cp.async);
// fp32 inputs are split into three bf16 terms.  Ends with the copies landed
// and a block barrier.
template <int D, class IN>
__device__ __forceinline__ void prep_stage(PrepSmem<D, IN>& sm, const IN* k, const IN* v,
                                           size_t ld, const float* bsrc, const float* gsrc,
                                           size_t ldbg) {
  constexpr int NK = Splits<IN>::K;
  if constexpr (NK == 1) {
    constexpr int P = D / 8;  // 16-byte pieces per row
    for (int e = threadIdx.x; e < 2 * kChunk * P; e += kBndThreads) {
      const int r = (e / P) % kChunk, c = (e % P) * 8;
      if (e < kChunk * P) cp_async16(&sm.K[0][r][c], k + (size_t)r * ld + c);
      else cp_async16(&sm.V[0][r][c], v + (size_t)r * ld + c);
    }
    cp_async_commit();
  } else {
    constexpr int G4 = D / 4;
    for (int e = threadIdx.x; e < kChunk * G4; e += kBndThreads) {
      const int i = e / G4, c = (e % G4) * 4;
      const float4 kk = ld4(k + i * ld + c);
      const float4 vv = ld4(v + i * ld + c);
      const float kx[4] = {kk.x, kk.y, kk.z, kk.w}, vx[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
      for (int q = 0; q < 4; q++) {
        __nv_bfloat16 ks[NK], vs[NK];
        split_bf16<NK>(kx[q], ks);
        split_bf16<NK>(vx[q], vs);
#pragma unroll
        for (int t = 0; t < NK; t++) {
          sm.K[t][i][c + q] = ks[t];
          sm.V[t][i][c + q] = vs[t];
        }
      }
    }
  }
  for (int i = threadIdx.x; i < kChunk; i += kBndThreads) {
    sm.beta[i] = bsrc[i * ldbg];
    sm.g[i] = gsrc[i * ldbg];
  }
  if constexpr (NK == 1) cp_async_wait<0>();
  __syncthreads();
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

// Prep of one chunk: sm.K, sm.V, sm.beta, sm.g staged (prep_stage) -> the
// walk pack at `pack` (global or shared; generic addressing).  All
// kBndThreads threads.
template <int D, class IN>
__device__ void bnd_prep(PrepSmem<D, IN>& sm, char* pack) {
  using PK = Pack<D, IN>;
  constexpr int NW = Splits<IN>::W, NK = Splits<IN>::K;
  constexpr int LDB = PrepSmem<D, IN>::LDB, LDT = PrepSmem<D, IN>::LDT;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;

  // P = K K^T on the tensor cores; warp w owns rows 16w..16w+15 (m-tile w)
  // and the n8 tiles that reach below the diagonal.  Warp 0, which has the
  // fewest tiles, then accumulates G.
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
            sm.A[tri(i, j)] = __fmul_rn(__fmul_rn(sm.beta[i], decay), acc[n][e]);
          }
        }
      }
    }
  }
  for (int i = tid; i < kChunk; i += kBndThreads) {
    sm.bg[i] = __fmul_rn(sm.beta[i], expf(__double2float_rn(sm.G[i])));
    sm.dvec[i] = expf(__double2float_rn(sm.G[kChunk - 1] - sm.G[i]));
  }
  if (tid == 0) sm.gammaC = expf(__double2float_rn(sm.G[kChunk - 1]));
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
#pragma unroll
      for (int i = m + 1; i < kChunk; i++) t[i] = __fmaf_rn(-sm.A[tri(i, m)], tm, t[i]);
    }
    const float bgj = sm.bg[j], bj = sm.beta[j];
#pragma unroll
    for (int i = 0; i < kChunk; i++) {
      __nv_bfloat16 sb[NW], sv[NW];
      split_bf16<NW>(__fmul_rn(t[i], bgj), sb);
      split_bf16<NW>(__fmul_rn(t[i], bj), sv);
#pragma unroll
      for (int q = 0; q < NW; q++) {
        sm.Tb[q][i][j] = sb[q];
        sm.Tv[q][i][j] = sv[q];
      }
    }
  }
  __syncthreads();

  // W = Tb K (rows i; warp w owns columns [D/4 w, D/4 (w+1))), and
  // U~^T = V^T Tv^T (rows c; warp w owns rows [D/4 w, D/4 (w+1))).
  {
    using PW = SplitPairs<NW, NK>;
    constexpr int NT = D / 32;  // n8 tiles of W per warp (D/4 columns)
    const int c0 = (D / 4) * warp;
#pragma unroll 1
    for (int mt = 0; mt < 4; mt++) {
      float w[NT][4];
#pragma unroll
      for (int n = 0; n < NT; n++)
#pragma unroll
        for (int e = 0; e < 4; e++) w[n][e] = 0.f;
      for (int ks = 0; ks <= mt; ks++) {
        uint32_t ab[NW][4];
#pragma unroll
        for (int q = 0; q < NW; q++) ldsm_x4(ab[q], afrag_addr(&sm.Tb[q][0][0], LDT, 16 * mt, 16 * ks));
#pragma unroll
        for (int np = 0; np < NT / 2; np++) {
          uint32_t bk[NK][4];
#pragma unroll
          for (int t = 0; t < NK; t++)
            ldsm_x4_t(bk[t], bfrag_kn_addr(&sm.K[t][0][0], LDB, 16 * ks, c0 + 16 * np));
#pragma unroll
          for (int p = 0; p < PW::kCount; p++) {
            mma16816(w[2 * np], ab[PW::a(p)], bk[PW::b(p)][0], bk[PW::b(p)][1]);
            mma16816(w[2 * np + 1], ab[PW::a(p)], bk[PW::b(p)][2], bk[PW::b(p)][3]);
          }
        }
      }
#pragma unroll
      for (int n = 0; n < NT; n++) {
#pragma unroll
        for (int hf = 0; hf < 2; hf++) {
          const int i = 16 * mt + gq + 8 * hf, c = c0 + 8 * n + 2 * tq;
          __nv_bfloat16 s0[NW], s1[NW];
          split_bf16<NW>(w[n][2 * hf], s0);
          split_bf16<NW>(w[n][2 * hf + 1], s1);
#pragma unroll
          for (int q = 0; q < NW; q++)
            *reinterpret_cast<uint32_t*>(PK::W(pack, q) + (size_t)i * PK::LDB + c) =
                pack_bf16(s0[q], s1[q]);
        }
      }
    }
    using PU = SplitPairs<NK, NW>;
    float* Up = PK::U(pack);
#pragma unroll 1
    for (int mt = 0; mt < D / 64; mt++) {
      const int r0 = c0 + 16 * mt;  // rows c of U~^T
      float u[8][4];
#pragma unroll
      for (int n = 0; n < 8; n++)
#pragma unroll
        for (int e = 0; e < 4; e++) u[n][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 4; ks++) {
        uint32_t av[NK][4];
#pragma unroll
        for (int t = 0; t < NK; t++) ldsm_x4_t(av[t], afrag_t_addr(&sm.V[t][0][0], LDB, r0, 16 * ks));
#pragma unroll
        for (int np = 0; np < 4; np++) {
          if (np >= ks) {  // Tv^T is zero above the diagonal block (m > i)
            uint32_t bt[NW][4];
#pragma unroll
            for (int q = 0; q < NW; q++)
              ldsm_x4(bt[q], bfrag_nk_addr(&sm.Tv[q][0][0], LDT, 16 * np, 16 * ks));
#pragma unroll
            for (int p = 0; p < PU::kCount; p++) {
              mma16816(u[2 * np], av[PU::a(p)], bt[PU::b(p)][0], bt[PU::b(p)][1]);
              mma16816(u[2 * np + 1], av[PU::a(p)], bt[PU::b(p)][2], bt[PU::b(p)][3]);
            }
          }
        }
      }
#pragma unroll
      for (int n = 0; n < 8; n++)
#pragma unroll
        for (int hf = 0; hf < 2; hf++)
          *reinterpret_cast<float2*>(Up + (size_t)(r0 + gq + 8 * hf) * PK::LDU + 8 * n + 2 * tq) =
              make_float2(u[n][2 * hf], u[n][2 * hf + 1]);
    }
  }
  // Keys (bf16 terms), decay vector and chunk decay into the pack.
  for (int e = tid; e < NK * kChunk * (D / 8); e += kBndThreads) {
    const int t = e / (kChunk * (D / 8)), r = (e / (D / 8)) % kChunk, c = (e % (D / 8)) * 8;
    *reinterpret_cast<uint4*>(PK::K(pack, t) + (size_t)r * PK::LDB + c) =
        *reinterpret_cast<const uint4*>(&sm.K[t][r][c]);
  }
  for (int i = tid; i < kChunk; i += kBndThreads) PK::dvec(pack)[i] = sm.dvec[i];
  if (tid == 0) *PK::gamma(pack) = sm.gammaC;
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

template <int D>
__device__ __forceinline__ void sacc_store(const float (&sacc)[D / 8][4], float* S, int r0) {
  const int lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
#pragma unroll
  for (int n = 0; n < D / 8; n++)
#pragma unroll
    for (int hf = 0; hf < 2; hf++)
      *reinterpret_cast<float2*>(S + (size_t)(r0 + gq + 8 * hf) * D + 8 * n + 2 * tq) =
          make_float2(sacc[n][2 * hf], sacc[n][2 * hf + 1]);
}

template <int D>
__device__ __forceinline__ void sacc_zero(float (&sacc)[D / 8][4]) {
#pragma unroll
  for (int n = 0; n < D / 8; n++)
#pragma unroll
    for (int e = 0; e < 4; e++) sacc[n][e] = 0.f;
}

// One boundary step for the warp's 16 rows (r0 = first row within the head):
// sacc <- exp(G_C) sacc + Ud^T K with Ud = dvec * (U~ - W sacc^T).  `pack` is
// in shared memory.
template <int D, class IN>
__device__ __forceinline__ void bnd_walk_warp(float (&sacc)[D / 8][4], char* pack, int r0) {
  using PK = Pack<D, IN>;
  constexpr int NS = Splits<IN>::S, NW = Splits<IN>::W, NK = Splits<IN>::K;
  const int lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
  // X = S W^T  (16 x C)
  float x[kChunk / 8][4];
#pragma unroll
  for (int n = 0; n < kChunk / 8; n++)
#pragma unroll
    for (int e = 0; e < 4; e++) x[n][e] = 0.f;
  {
    using PP = SplitPairs<NS, NW>;
#pragma unroll
    for (int ks = 0; ks < D / 16; ks++) {
      uint32_t a[NS][4];
      acc_to_afrag<NS>(sacc[2 * ks], sacc[2 * ks + 1], a);
#pragma unroll
      for (int np = 0; np < kChunk / 16; np++) {
        uint32_t b[NW][4];
#pragma unroll
        for (int q = 0; q < NW; q++)
          ldsm_x4(b[q], bfrag_nk_addr(PK::W(pack, q), PK::LDB, 16 * np, 16 * ks));
#pragma unroll
        for (int p = 0; p < PP::kCount; p++) {
          mma16816(x[2 * np], a[PP::a(p)], b[PP::b(p)][0], b[PP::b(p)][1]);
          mma16816(x[2 * np + 1], a[PP::a(p)], b[PP::b(p)][2], b[PP::b(p)][3]);
        }
      }
    }
  }
  // Ud = dvec * (U~^T - X)
  {
    const float* U = PK::U(pack);
    const float* dv = PK::dvec(pack);
#pragma unroll
    for (int n = 0; n < kChunk / 8; n++)
#pragma unroll
      for (int e = 0; e < 4; e++) {
        const int r = r0 + gq + 8 * (e >> 1), i = 8 * n + 2 * tq + (e & 1);
        x[n][e] = __fmul_rn(dv[i], __fsub_rn(U[(size_t)r * PK::LDU + i], x[n][e]));
      }
  }
  // S' = gamma S + Ud^T K  (16 x D)
  {
    const float gam = *PK::gamma(pack);
#pragma unroll
    for (int n = 0; n < D / 8; n++)
#pragma unroll
      for (int e = 0; e < 4; e++) sacc[n][e] = __fmul_rn(gam, sacc[n][e]);
    using PP = SplitPairs<NS, NK>;
#pragma unroll
    for (int ks = 0; ks < kChunk / 16; ks++) {
      uint32_t a[NS][4];
      acc_to_afrag<NS>(x[2 * ks], x[2 * ks + 1], a);
#pragma unroll
      for (int np = 0; np < D / 16; np++) {
        uint32_t b[NK][4];
#pragma unroll
        for (int q = 0; q < NK; q++)
          ldsm_x4_t(b[q], bfrag_kn_addr(PK::K(pack, q), PK::LDB, 16 * ks, 16 * np));
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
