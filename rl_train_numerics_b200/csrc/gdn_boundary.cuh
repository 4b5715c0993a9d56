// gdn_boundary.cuh -- the chunk boundary function (first CPR pass and the
// decode resync), on tensor cores.
//
// "NovaSky's IsoExec Fixes the Hidden Math Bug Corrupting AI Training Runs",
// section "Solving the linear-attention headache": CPR's serial sweep yields
// the state entering every chunk, and decode, after each chunk's worth of
// tokens, swaps its state for the result of that same computation.  The pages
// do not write the
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
//   G        double: pair sums, then a Kogge-Stone scan (bnd_prep)
//   P=KK^T   k16 steps ascending; split pairs in SplitPairs order
//   A_ij     (beta_i * expf((float)(G_i - G_j))) * P_ij
//   T        blocked forward substitution over 16 x 16 blocks (bnd_prep
//            states the order of every sum)
//   Tb, Tv   T_im * (beta_m expf(G_m)) and T_im * beta_m, then split
//   Y        (S0 K^T): k16 steps over the key channel ascending
//   U^T      one accumulator: per k16 step over m (ascending, up to the
//            diagonal block), first + V^T Tv^T then - Y Tb^T
//   Ud       exp(G_C - G_i) * U^T
//   S_C      accumulator starts at exp(G_C) * S0, then k16 steps over i
#pragma once

#include "gdn_common.cuh"
#include "gdn_mma.cuh"
#include "gdn_umma.cuh"

#include <type_traits>

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
// memory layout.  Tb and Tv are stored transposed, in the core-matrix layout
// of gdn_umma.cuh with 64 rows: TbT[q][core_off<64>(j, i)] is split term q of
// Tb_ij (zero above the diagonal, j > i).
template <int D, class IN>
struct PackHead {
  static constexpr int NW = Splits<IN>::W;
  __nv_bfloat16 TbT[NW][kChunk * kChunk];
  __nv_bfloat16 TvT[NW][kChunk * kChunk];
  float dvec[kChunk];
  float gamma[32];  // [0] = exp(G_C), the rest zero (the head is whole 128-byte lines)
};

// Keys and values of one chunk as bf16 term planes, core-matrix layout with
// 64 rows (token i) and D columns (channel): plane[core_off<64>(i, c)].
template <int D, class IN>
struct KVPlanes {
  static constexpr int NK = Splits<IN>::K;
  __nv_bfloat16 K[NK][kChunk * D];
  __nv_bfloat16 V[NK][kChunk * D];
};

// The walk's input for one (chunk, head), written by the prep and read back
// with one bulk copy: the pack head and the chunk's key and value planes.
template <int D, class IN>
struct WalkPack {
  PackHead<D, IN> head;
  KVPlanes<D, IN> kv;
};

template <int D, class IN>
constexpr size_t pack_size() {
  return round_up(sizeof(WalkPack<D, IN>), 128);
}

// Shared memory of the prep, apart from its scratch matrix AT (PrepAT), which
// callers place where it can share space with later work.
template <int D, class IN>
struct PrepSmem {
  static constexpr int NW = Splits<IN>::W, NK = Splits<IN>::K;
  PackHead<D, IN> head;
  __nv_bfloat16 K[NK][kChunk * D];
  double G[kChunk];
  float beta[kChunk];
  float g[kChunk];
  float bg[kChunk];
};
// AT[m][i] = A_im for i > m (zero elsewhere): a column of A is contiguous.
using PrepAT = float[kChunk][kChunk];

// The rows of a [C][D] block (row stride ld elements) as bf16 term planes
// (core-matrix layout) written with plain loads and stores: bf16 inputs are
// copied, fp32 inputs split into three bf16 terms.  A warp takes 8 rows x 4
// column groups of bf16 input: 64 contiguous bytes of each row, 128
// contiguous destination bytes per quarter warp.  Rows at or past `rows`
// are written as zeros (a chunk's padding past its length).
template <int D, class IN>
__device__ __forceinline__ void copy_planes(__nv_bfloat16 (*dst)[kChunk * D], const IN* src,
                                            size_t ld, int nthreads, int rows = kChunk) {
  constexpr int NK = Splits<IN>::K;
  if constexpr (NK == 1) {
    constexpr int P = D / 8;  // 16-byte pieces per row
    static_assert(P % 4 == 0, "column groups come in fours");
    for (int e = threadIdx.x; e < kChunk * P; e += nthreads) {
      const int w = e >> 5, l = e & 31;
      const int cg = (w % (P / 4)) * 4 + (l >> 3), r = (w / (P / 4)) * 8 + (l & 7);
      *reinterpret_cast<uint4*>(&dst[0][core_off<kChunk>(r, 8 * cg)]) =
          r < rows ? *reinterpret_cast<const uint4*>(src + (size_t)r * ld + 8 * cg)
                   : make_uint4(0u, 0u, 0u, 0u);
    }
  } else {
    constexpr int G4 = D / 4;
    for (int e = threadIdx.x; e < kChunk * G4; e += nthreads) {
      const int r = e / G4, c = (e % G4) * 4;
      const float4 x4 = r < rows ? ld4(src + (size_t)r * ld + c) : make_float4(0.f, 0.f, 0.f, 0.f);
      const float xs[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
      for (int q = 0; q < 4; q++) {
        __nv_bfloat16 s[NK];
        split_bf16<NK>(xs[q], s);
#pragma unroll
        for (int t = 0; t < NK; t++) dst[t][core_off<kChunk>(r, c + q)] = s[t];
      }
    }
  }
}

// One thread's share (NT threads) of a [C][D] block held in registers: loaded
// early, written out as bf16 term planes (core-matrix layout) later, so the
// load latency hides behind other work.  Same piece mapping as copy_planes.
template <int D, class IN, int NT>
struct PlaneRows {
  static constexpr bool kBf16 = Splits<IN>::K == 1;
  static constexpr int kPerRow = kBf16 ? D / 8 : D / 4;  // 16-byte pieces of a row
  static constexpr int kPieces = kChunk * kPerRow / NT;
  static_assert(kChunk * kPerRow % NT == 0, "whole pieces per thread");
  uint4 x[kPieces];
  __device__ __forceinline__ static void where(int e, int& r, int& c) {
    if constexpr (kBf16) {
      const int w = e >> 5, l = e & 31;
      c = 8 * ((w % (kPerRow / 4)) * 4 + (l >> 3));
      r = (w / (kPerRow / 4)) * 8 + (l & 7);
    } else {
      r = e / kPerRow;
      c = (e % kPerRow) * 4;
    }
  }
  // Rows at or past `rows` load as zeros.
  __device__ __forceinline__ void load(const IN* src, size_t ld, int rows = kChunk) {
#pragma unroll
    for (int j = 0; j < kPieces; j++) {
      int r, c;
      where((int)threadIdx.x + j * NT, r, c);
      x[j] = r < rows ? *reinterpret_cast<const uint4*>(src + (size_t)r * ld + c)
                      : make_uint4(0u, 0u, 0u, 0u);
    }
  }
  __device__ __forceinline__ void store(__nv_bfloat16 (*dst)[kChunk * D]) const {
#pragma unroll
    for (int j = 0; j < kPieces; j++) {
      int r, c;
      where((int)threadIdx.x + j * NT, r, c);
      if constexpr (kBf16) {
        *reinterpret_cast<uint4*>(&dst[0][core_off<kChunk>(r, c)]) = x[j];
      } else {
        const float xs[4] = {__uint_as_float(x[j].x), __uint_as_float(x[j].y),
                             __uint_as_float(x[j].z), __uint_as_float(x[j].w)};
#pragma unroll
        for (int q = 0; q < 4; q++) {
          __nv_bfloat16 t3[Splits<IN>::K];
          split_bf16<Splits<IN>::K>(xs[q], t3);
#pragma unroll
          for (int tt = 0; tt < Splits<IN>::K; tt++) dst[tt][core_off<kChunk>(r, c + q)] = t3[tt];
        }
      }
    }
  }
};

// The same into shared memory; bf16 inputs go with cp.async (the caller
// commits and waits).  Rows at or past `rows` are written as zeros.
template <int D, class IN>
__device__ __forceinline__ void stage_planes(__nv_bfloat16 (*dst)[kChunk * D], const IN* src,
                                             size_t ld, int nthreads, int rows = kChunk) {
  if constexpr (Splits<IN>::K == 1) {
    constexpr int P = D / 8;
    for (int e = threadIdx.x; e < kChunk * P; e += nthreads) {
      const int w = e >> 5, l = e & 31;
      const int cg = (w % (P / 4)) * 4 + (l >> 3), r = (w / (P / 4)) * 8 + (l & 7);
      if (r < rows)
        cp_async16(&dst[0][core_off<kChunk>(r, 8 * cg)], src + (size_t)r * ld + 8 * cg);
      else
        *reinterpret_cast<uint4*>(&dst[0][core_off<kChunk>(r, 8 * cg)]) = make_uint4(0u, 0u, 0u, 0u);
    }
  } else {
    copy_planes<D, IN>(dst, src, ld, nthreads, rows);
  }
}

// ldmatrix row addresses (x4) in 64-row core-layout tiles.  A fragment of
// rows r0.., columns c0.. of the tile:
__device__ __forceinline__ const __nv_bfloat16* afrag_addr(const __nv_bfloat16* base, int r0,
                                                           int c0) {
  const int lane = threadIdx.x & 31, mi = lane >> 3;
  return base + core_off<kChunk>(r0 + (mi & 1) * 8 + (lane & 7), c0 + (mi >> 1) * 8);
}
// A fragment (x4.trans) of A[r][c] = M[c][r] (the tile's rows are the k index).
__device__ __forceinline__ const __nv_bfloat16* afrag_t_addr(const __nv_bfloat16* base, int r0,
                                                             int c0) {
  const int lane = threadIdx.x & 31, mi = lane >> 3;
  return base + core_off<kChunk>(c0 + (mi >> 1) * 8 + (lane & 7), r0 + (mi & 1) * 8);
}
// B fragments (x4 = two n8 tiles) of B[k][n] = M[n][k] (the tile's rows are n).
__device__ __forceinline__ const __nv_bfloat16* bfrag_nk_addr(const __nv_bfloat16* base, int n0,
                                                              int k0) {
  const int lane = threadIdx.x & 31, mi = lane >> 3;
  return base + core_off<kChunk>(n0 + (mi >> 1) * 8 + (lane & 7), k0 + (mi & 1) * 8);
}
// B fragments (x4.trans = two n8 tiles) of B[k][n] = M[k][n] (the tile's rows are k).
__device__ __forceinline__ const __nv_bfloat16* bfrag_kn_addr(const __nv_bfloat16* base, int k0,
                                                              int n0) {
  const int lane = threadIdx.x & 31, mi = lane >> 3;
  return base + core_off<kChunk>(k0 + (mi & 1) * 8 + (lane & 7), n0 + (mi >> 1) * 8);
}

// Stage one chunk for the prep: keys (rows at stride ld), beta and g
// (stride ldbg).  Tokens at or past `rows` (the padding of a chunk shorter
// than C) stage as zeros: beta = g = 0 and a zero key make them identity
// steps.  Ends with the data landed and a block barrier.
template <int D, class IN>
__device__ __forceinline__ void prep_stage(PrepSmem<D, IN>& sm, const IN* k, size_t ld,
                                           const float* bsrc, const float* gsrc, size_t ldbg,
                                           int rows = kChunk) {
  stage_planes<D, IN>(sm.K, k, ld, (int)blockDim.x, rows);
  cp_async_commit();
  for (int i = threadIdx.x; i < kChunk; i += kBndThreads) {
    sm.beta[i] = i < rows ? bsrc[i * ldbg] : 0.f;
    sm.g[i] = i < rows ? gsrc[i * ldbg] : 0.f;
  }
  cp_async_wait<0>();
  __syncthreads();
}

// Prep of one chunk: sm.K, sm.beta, sm.g staged -> sm.head (Tb, Tv, dvec,
// gamma), with AT as scratch.  The first kBndThreads threads do the work;
// every thread of the block takes the barriers.  Ends with a block barrier.
// CPT consecutive floats of a row of AT (16-byte loads where CPT allows).
template <int CPT>
__device__ __forceinline__ void at_row(float (&x)[CPT], const float* src) {
  if constexpr (CPT % 4 == 0) {
#pragma unroll
    for (int e = 0; e < CPT; e += 4) {
      const float4 u = *reinterpret_cast<const float4*>(src + e);
      x[e] = u.x, x[e + 1] = u.y, x[e + 2] = u.z, x[e + 3] = u.w;
    }
  } else {
#pragma unroll
    for (int e = 0; e < CPT; e += 2) {
      const float2 u = *reinterpret_cast<const float2*>(src + e);
      x[e] = u.x, x[e + 1] = u.y;
    }
  }
}
template <int CPT>
__device__ __forceinline__ void at_row_store(float* dst, const float2 (&x)[CPT / 2], float sgn) {
#pragma unroll
  for (int e = 0; e < CPT / 2; e++)
    *reinterpret_cast<float2*>(dst + 2 * e) = f2(sgn * x[e].x, sgn * x[e].y);
}

// Stage ST of the blocked inverse (see bnd_prep): the blocks (b, c) of T with
// b - c = ST, thread (block, row i, columns j0 .. j0 + CPT - 1).  X = the sum
// over k = c .. b-1 of A_bk T_kc (one fma chain per element, ascending inner
// index), then T_bc = -(D_b X) (from X_ij, D_b[i][k] X_kj in ascending k < i).
// Packed pairs of fmas: each element's arithmetic is the scalar fma chain.
template <int ST, int CPT>
__device__ __forceinline__ void t_stage(PrepAT& AT, float* X, int tid) {
  constexpr int NB = 16, NBLK = kChunk / NB - ST, TPB = NB * NB / CPT;
  const int blk = tid / TPB, rem = tid % TPB;
  const int i = rem / (NB / CPT), j0 = (rem % (NB / CPT)) * CPT;
  const int c0 = blk * NB, b0 = c0 + ST * NB;
  float* Xr = X + blk * NB * NB;
  const bool active = blk < NBLK;
  if (active) {
    float2 acc[CPT / 2];
#pragma unroll
    for (int e = 0; e < CPT / 2; e++) acc[e] = f2(0.f, 0.f);
#pragma unroll
    for (int kb = 0; kb < ST; kb++) {
      const int k0 = c0 + kb * NB;
#pragma unroll
      for (int q = 0; q < NB; q++) {
        const float a = AT[k0 + q][b0 + i];  // A_{b0+i, k0+q}
        float tv[CPT];
        at_row<CPT>(tv, &AT[k0 + q][c0 + j0]);
        if (kb == 0) {
#pragma unroll
          for (int e = 0; e < CPT; e++)
            if (q < j0 + e) tv[e] = 0.f;  // above T's diagonal (A lives there)
        }
#pragma unroll
        for (int e = 0; e < CPT / 2; e++) acc[e] = __ffma2_rn(f2(a, a), f2(tv[2 * e], tv[2 * e + 1]), acc[e]);
      }
    }
    at_row_store<CPT>(Xr + i * NB + j0, acc, 1.f);
  }
  __syncthreads();
  if (active) {
    float2 acc[CPT / 2];
    {
      float x[CPT];
      at_row<CPT>(x, Xr + i * NB + j0);
#pragma unroll
      for (int e = 0; e < CPT / 2; e++) acc[e] = f2(x[2 * e], x[2 * e + 1]);
    }
#pragma unroll
    for (int k = 0; k < NB - 1; k++) {
      if (k < i) {
        const float d = AT[b0 + k][b0 + i];  // D_b[i][k]
        float y[CPT];
        at_row<CPT>(y, Xr + k * NB + j0);
#pragma unroll
        for (int e = 0; e < CPT / 2; e++) acc[e] = __ffma2_rn(f2(d, d), f2(y[2 * e], y[2 * e + 1]), acc[e]);
      }
    }
    at_row_store<CPT>(&AT[b0 + i][c0 + j0], acc, -1.f);
  }
  __syncthreads();
}

// G = cumulative sum of a chunk's g in double, by one warp: lane l sums
// g_2l + g_2l+1, then an inclusive Kogge-Stone scan over the 32 pair sums
// (offsets 1, 2, 4, 8, 16); G_2l+1 = scan_l, G_2l = scan_(l-1) + g_2l
// (scan_(-1) = 0).
__device__ __forceinline__ void chunk_cumsum_g(const float* g, double* G) {
  const int lane = threadIdx.x & 31;
  const double g0 = (double)g[2 * lane], g1 = (double)g[2 * lane + 1];
  double x = g0 + g1;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const double y = __shfl_up_sync(kFull, x, off);
    if (lane >= off) x += y;
  }
  const double e = __shfl_up_sync(kFull, x, 1);
  G[2 * lane + 1] = x;
  G[2 * lane] = lane > 0 ? e + g0 : g0;
}

struct PrepNoHook {
  __device__ void operator()() const {}
};

// after_p(): all threads, once P = K K^T is in registers and before AT is
// first written (a caller whose AT shares memory with K saves K there).
template <int D, class IN, class AfterP = PrepNoHook>
__device__ void bnd_prep(PrepSmem<D, IN>& sm, PrepAT& AT, const AfterP& after_p = AfterP{}) {
  constexpr int NW = Splits<IN>::W, NK = Splits<IN>::K;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;

  // P = K K^T on the tensor cores; warp w owns rows 16w..16w+15 (m-tile w)
  // and the n8 tiles that reach below the diagonal.
  float acc[8][4];
  if (warp < kBndThreads / 32) {
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
      for (int t = 0; t < NK; t++) ldsm_x4(a[t], afrag_addr(sm.K[t], m0, 16 * ks));
#pragma unroll
      for (int np = 0; np < 4; np++) {
        if (np <= warp) {
          uint32_t b[NK][4];
#pragma unroll
          for (int t = 0; t < NK; t++)
            ldsm_x4(b[t], bfrag_nk_addr(sm.K[t], 16 * np, 16 * ks));
#pragma unroll
          for (int p = 0; p < PP::kCount; p++) {
            mma16816(acc[2 * np], a[PP::a(p)], b[PP::b(p)][0], b[PP::b(p)][1]);
            mma16816(acc[2 * np + 1], a[PP::a(p)], b[PP::b(p)][2], b[PP::b(p)][3]);
          }
        }
      }
    }
  }
  // G = cumulative sum of g in double: warp 0, lane l sums g_2l + g_2l+1,
  // then an inclusive Kogge-Stone scan over the 32 pair sums (offsets 1, 2,
  // 4, 8, 16); G_2l+1 = scan_l, G_2l = scan_(l-1) + g_2l (scan_(-1) = 0).
  if (warp == 0) chunk_cumsum_g(sm.g, sm.G);
  after_p();
  if (tid < kBndThreads)
    for (int e = tid; e < kChunk * kChunk / 4; e += kBndThreads)
      reinterpret_cast<float4*>(&AT[0][0])[e] = make_float4(0.f, 0.f, 0.f, 0.f);
  __syncthreads();
  if (warp < kBndThreads / 32) {
    const int m0 = 16 * warp;
#pragma unroll
    for (int n = 0; n < 8; n++) {
      if (n < 2 * warp + 2) {
#pragma unroll
        for (int e = 0; e < 4; e++) {
          const int i = m0 + gq + (e >> 1) * 8, j = 8 * n + 2 * tq + (e & 1);
          if (j < i) {
            const float decay = expf(__double2float_rn(sm.G[i] - sm.G[j]));
            AT[j][i] = __fmul_rn(__fmul_rn(sm.beta[i], decay), acc[n][e]);
          }
        }
      }
    }
  }
  for (int i = tid; i < kChunk; i += kBndThreads) {
    sm.bg[i] = __fmul_rn(sm.beta[i], expf(__double2float_rn(sm.G[i])));
    sm.head.dvec[i] = expf(__double2float_rn(sm.G[kChunk - 1] - sm.G[i]));
  }
  if (tid < 32) sm.head.gamma[tid] = tid == 0 ? expf(__double2float_rn(sm.G[kChunk - 1])) : 0.f;
  __syncthreads();

  // T = (I + A)^{-1} (unit lower triangular) by blocked forward substitution
  // over 16 x 16 blocks, kept in AT's free lower triangle: AT[i][j] = T_ij for
  // i >= j (A stays above the diagonal, AT[m][i] = A_im for i > m).
  //  1. diagonal blocks D_b = (I + A_bb)^{-1}, column j of block b held by
  //     one thread: right-looking, T_ij accumulates -A_im T_mj in ascending m;
  //  2. for s = 1, 2, 3 and every block (b, c) with b - c = s:
  //     X = sum over k = c .. b-1 (ascending) of A_bk T_kc, one fma chain per
  //     element in ascending inner index; then T_bc = -(D_b X), accumulated
  //     from X_ij with D_b[i][k] X_kj in ascending k < i.
  {
    constexpr int NB = 16;
    if (tid < kChunk) {
      const int b0 = (tid / NB) * NB, j = tid % NB;
      float t[NB];
#pragma unroll
      for (int i = 0; i < NB; i++) t[i] = (i == j) ? 1.f : 0.f;
#pragma unroll
      for (int m = 0; m < NB - 1; m++) {
        const float tm = t[m];
        const float* col = &AT[b0 + m][b0];
#pragma unroll
        for (int i4 = (m + 1) & ~3; i4 < NB; i4 += 4) {
          const float4 a4 = *reinterpret_cast<const float4*>(col + i4);
          const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
          for (int q = 0; q < 4; q++)
            if (i4 + q > m) t[i4 + q] = __fmaf_rn(-av[q], tm, t[i4 + q]);
        }
      }
#pragma unroll
      for (int i = 0; i < NB; i++)
        if (i >= j) AT[b0 + i][b0 + j] = t[i];
    }
    __syncthreads();
    // A_bb is no longer needed: its place above the diagonal takes D_b
    // transposed, AT[b0 + k][b0 + i] = D_b[i][k] for i > k, so that the
    // products below read D_b by rows of AT.
    if (tid < kChunk) {
      const int b0 = (tid / NB) * NB, j = tid % NB;
#pragma unroll
      for (int i = 0; i < NB; i++)
        if (i > j) AT[b0 + j][b0 + i] = AT[b0 + i][b0 + j];
    }
    __syncthreads();
    // Stages s = 1, 2, 3: thread (block, row i, CPT columns), CPT = 8, 4, 2
    // so that every stage but the first keeps all 128 threads busy.
    float* X = reinterpret_cast<float*>(sm.head.TbT[0]);  // scratch until the splits below
    t_stage<1, 8>(AT, X, tid);
    t_stage<2, 4>(AT, X, tid);
    t_stage<3, 2>(AT, X, tid);
  }

  // Tb = T diag(beta*gamma), Tv = T diag(beta), split into bf16 terms; thread
  // (j, half) takes rows 32 half .. 32 half + 31 of column j of T, which is
  // row j of the transposed tiles: 16-byte stores.
  if (tid < 2 * kChunk) {
    const int j = tid % kChunk, i0 = (tid / kChunk) * (kChunk / 2);
    const float bgj = sm.bg[j], bj = sm.beta[j];
#pragma unroll
    for (int i8 = i0; i8 < i0 + kChunk / 2; i8 += 8) {
      __nv_bfloat16 sb[8][NW], sv[8][NW];
#pragma unroll
      for (int e = 0; e < 8; e++) {
        const float tij = (i8 + e >= j) ? AT[i8 + e][j] : 0.f;
        split_bf16<NW>(__fmul_rn(tij, bgj), sb[e]);
        split_bf16<NW>(__fmul_rn(tij, bj), sv[e]);
      }
#pragma unroll
      for (int q = 0; q < NW; q++) {
        const uint4 pb = make_uint4(pack_bf16(sb[0][q], sb[1][q]), pack_bf16(sb[2][q], sb[3][q]),
                                    pack_bf16(sb[4][q], sb[5][q]), pack_bf16(sb[6][q], sb[7][q]));
        const uint4 pv = make_uint4(pack_bf16(sv[0][q], sv[1][q]), pack_bf16(sv[2][q], sv[3][q]),
                                    pack_bf16(sv[4][q], sv[5][q]), pack_bf16(sv[6][q], sv[7][q]));
        *reinterpret_cast<uint4*>(&sm.head.TbT[q][core_off<kChunk>(j, i8)]) = pb;
        *reinterpret_cast<uint4*>(&sm.head.TvT[q][core_off<kChunk>(j, i8)]) = pv;
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

// sacc_store into the permuted boundary-state layout of the forward workspace.
template <int D>
__device__ __forceinline__ void sacc_store_bst(const float (&sacc)[D / 8][4], float* S, int r0) {
  const int lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3, odd = tq & 1;
#pragma unroll
  for (int n = 0; n < D / 8; n++) {
    const float s0 = odd ? sacc[n][0] : sacc[n][2];
    const float s1 = odd ? sacc[n][1] : sacc[n][3];
    const float r0v = __shfl_xor_sync(kFull, s0, 1);
    const float r1v = __shfl_xor_sync(kFull, s1, 1);
    float4 out;
    if (!odd) out = make_float4(sacc[n][0], sacc[n][1], r0v, r1v);
    else out = make_float4(r0v, r1v, sacc[n][2], sacc[n][3]);
    const int row = r0 + gq + 8 * odd, col = 8 * n + 2 * (tq & 2);
    *reinterpret_cast<float4*>(S + (size_t)row * D + bst_col(row, col)) = out;
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
  constexpr size_t PL = (size_t)kChunk * D;  // elements per K/V plane
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
        for (int q = 0; q < NK; q++) ldsm_x4(b[q], bfrag_nk_addr(Kp + q * PL, 16 * np, 16 * ks));
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
      for (int q = 0; q < NK; q++) ldsm_x4_t(av[q], afrag_t_addr(Vp + q * PL, r0, 16 * ks));
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
          ldsm_x4_t(bv[q], bfrag_kn_addr(hd.TvT[q], 16 * ks, 16 * np));
          ldsm_x4_t(bb[q], bfrag_kn_addr(hd.TbT[q], 16 * ks, 16 * np));
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
        for (int q = 0; q < NK; q++) ldsm_x4_t(b[q], bfrag_kn_addr(Kp + q * PL, 16 * ks, 16 * np));
#pragma unroll
        for (int p = 0; p < PP::kCount; p++) {
          mma16816(sacc[2 * np], a[PP::a(p)], b[PP::b(p)][0], b[PP::b(p)][1]);
          mma16816(sacc[2 * np + 1], a[PP::a(p)], b[PP::b(p)][2], b[PP::b(p)][3]);
        }
      }
    }
  }
}

// ----------------------------------------------------------------------------
// Walk step on the fifth-generation tensor cores (tcgen05), for
// d_k = d_v = 128 with bf16 inputs.  128 * NCS threads: warp w works on the
// state rows of its tensor-memory lane quadrant, 32 (w % 4) .. 32 (w % 4) + 31,
// and on column slice w / 4 of NCS; each thread holds its row's slice of S in
// registers.  Warp 0 issues every product (M = 128) into tensor memory and
// one mbarrier signals their completion.  Tensor-memory columns (fp32
// accumulators; bf16 terms packed two per column):
//   [  0,128)  S terms (hi [0,64), lo [64,128)), the A operand of Y; then P
//   [128,192)  Y; then the -Y terms, then the Ud terms (hi [128,160), lo [160,192))
//   [192,256)  Z
// Products:
//   Y = S K^T              A: S terms          B: K (K-major)
//   Z = V^T Tv^T - Y Tb^T  A: V (MN-major), then the -Y terms
//                          B: TvT, TbT (MN-major); k16 step ks only reaches
//                          the columns >= 16 ks (Tb, Tv are lower triangular)
//   P = Ud K               A: Ud terms         B: K (MN-major)
//   S <- fma(exp(G_C), S, P)   per element
// Fixed evaluation order (the rounding schedule of this path):
//   Y   k16 steps over the key channel ascending; per step S hi, then S lo
//   Z   first V^T Tv^T (k16 steps ascending; Tv hi, then lo), then -Y Tb^T
//       (k16 steps ascending; pairs (hi,hi), (hi,lo), (lo,hi))
//   Ud  dvec_i * Z, split into two bf16 terms
//   P   k16 steps over i ascending; per step Ud hi, then Ud lo
// Which thread does an element's elementwise work does not change its bits,
// so every NCS gives the same results.  Every wait is bounded; a step that
// gives up returns false on all threads.
// ----------------------------------------------------------------------------
constexpr int kTcRows = 128;
constexpr uint32_t kTmSA = 0, kTmP = 0, kTmY = 128, kTmYA = 128, kTmZ = 192;
constexpr uint32_t kTmemCols = 256;
constexpr int kTcWaitPolls = 1 << 22;

template <int D, class IN>
constexpr bool use_tc() {
  return D == 128 && std::is_same<IN, __nv_bfloat16>::value;
}

struct TcCtx {
  uint32_t tmem;   // first of the kTmemCols allocated columns
  uint32_t mbar;   // completion mbarrier (shared address)
  uint32_t phase;  // parity of the phase waited for next
};

// Allocate tensor memory (warp 0) and initialise the mbarrier; all threads.
__device__ __forceinline__ void tc_setup(TcCtx& cx, uint64_t* mbar, uint32_t* tmem_slot,
                                         uint32_t cols = kTmemCols) {
  if (threadIdx.x < 32) tmem_alloc(smem_u32(tmem_slot), cols);
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(mbar), 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cx.tmem = *tmem_slot;
  cx.mbar = smem_u32(mbar);
  cx.phase = 0;
}

// Wait (bounded) for the products committed last.  After a timeout the phase
// is not advanced, so tc_drain waits for the same completion.
__device__ __forceinline__ bool tc_wait(TcCtx& cx) {
  const bool ok = mbar_wait(cx.mbar, cx.phase, kTcWaitPolls);
  if (ok) cx.phase ^= 1;
  tc_fence_after();
  return ok;
}

// After a failed step: wait once more (bounded) for the products in flight.
__device__ __forceinline__ void tc_drain(TcCtx& cx) { (void)tc_wait(cx); }

// Release tensor memory (warp 0) once every thread's tensor-memory accesses
// are done; all threads.
__device__ __forceinline__ void tc_teardown(const TcCtx& cx, uint32_t cols = kTmemCols) {
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x < 32) tmem_dealloc(cx.tmem, cols);
  if (threadIdx.x == 0) mbar_inval(cx.mbar);
}

// Two-term bf16 split of (x0, x1), packed as bf16 pairs (x0 in the low half).
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const __nv_bfloat162 l =
      __floats2bfloat162_rn(__fsub_rn(x0, __low2float(h)), __fsub_rn(x1, __high2float(h)));
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// N consecutive tensor-memory columns of this thread's lane, loaded and waited.
template <int N>
__device__ __forceinline__ void tmem_load(uint32_t taddr, float (&x)[N]) {
  static_assert(N == 16 || N == 32, "16 or 32 columns");
  if constexpr (N == 16) tmem_ld16(taddr, x);
  else tmem_ld32(taddr, x);
  tmem_wait_ld(x);
}
template <int N>
__device__ __forceinline__ void tmem_store(uint32_t taddr, const uint32_t (&r)[N]) {
  static_assert(N == 8 || N == 16 || N == 32, "8, 16 or 32 columns");
  if constexpr (N == 8) tmem_st8(taddr, r);
  else if constexpr (N == 16) tmem_st16(taddr, r);
  else tmem_st32(taddr, r);
}

// Writes n = 2 NP values as two bf16 term blocks (hi at taddr, lo at
// taddr + lo_off), optionally negated.
template <int NP, bool NEG>
__device__ __forceinline__ void store_terms(uint32_t taddr, uint32_t lo_off, const float* x) {
  uint32_t hi[NP], lo[NP];
#pragma unroll
  for (int j = 0; j < NP; j++) split2(NEG ? -x[2 * j] : x[2 * j], NEG ? -x[2 * j + 1] : x[2 * j + 1], hi[j], lo[j]);
  tmem_store<NP>(taddr, hi);
  tmem_store<NP>(taddr + lo_off, lo);
}

// Hooks of a step, for work that overlaps it:
//   inputs_ready()  all threads, before the first barrier: false gives up
//   after_first()   warp 0, once the first round of products is committed
//   during_first(s) all threads, while the first round runs (s: the state
//                   the step starts from)
//   after_second()  warp 0, once the second round is committed
//   after_last()    warp 0, once the last round is committed (the step's
//                   final barrier follows)
struct TcNoHooks {
  __device__ bool inputs_ready() const { return true; }
  __device__ void after_first() const {}
  __device__ void during_first(const float*) const {}
  __device__ void after_second() const {}
  __device__ void after_last() const {}
};

// Outcome of a step: done, gave up before issuing any product, or gave up
// after (products may still be in flight: tc_drain).
enum TcStep { kStepDone = 0, kStepNoInputs = 1, kStepFailed = 2 };

// One boundary step S <- S_C for the block's 128 rows (see above).  Kp, Vp:
// the chunk's key and value planes; hd: its pack.  Returns a TcStep.
template <int NCS, class Hooks>
__device__ __forceinline__ int tc_walk_step(float (&s)[128 / NCS],
                                             const PackHead<128, __nv_bfloat16>& hd,
                                             const __nv_bfloat16* Kp, const __nv_bfloat16* Vp,
                                             TcCtx& cx, const Hooks& hooks) {
  constexpr int D = 128, SC = D / NCS, YC = kChunk / NCS, YP = YC < 32 ? YC : 32;
  static_assert(SC % 32 == 0, "state slices are whole 32-column pieces");
  constexpr uint32_t TPLANE = kChunk * kChunk * 2;
  constexpr uint32_t IY = idesc_bf16(kTcRows, kChunk, false, false);
  constexpr uint32_t IP = idesc_bf16(kTcRows, D, false, true);
  const int t = threadIdx.x, w = t >> 5, cs = w >> 2;
  const uint32_t tl = cx.tmem + ((uint32_t)(32 * (w & 3)) << 16);  // this warp's lanes
  const uint32_t kb = smem_u32(Kp), vb = smem_u32(Vp);
  const uint32_t tbb = smem_u32(hd.TbT[0]), tvb = smem_u32(hd.TvT[0]);
  bool ok = true;

  // S terms -> tensor memory; Y = S K^T and V^T Tv^T into Z
  tc_fence_after();
#pragma unroll
  for (int pc = 0; pc < SC / 32; pc++)
    store_terms<16, false>(tl + kTmSA + (cs * SC + 32 * pc) / 2, 64, &s[32 * pc]);
  tmem_wait_st();
  const bool in_ok = hooks.inputs_ready();
  tc_fence_before();
  if (__syncthreads_or(!in_ok)) return kStepNoInputs;
  if (w == 0) {
    tc_fence_after();
#pragma unroll
    for (int ks = 0; ks < D / 16; ks++)
#pragma unroll
      for (int a = 0; a < 2; a++)
        umma_bf16_ts(cx.tmem + kTmY, cx.tmem + kTmSA + 64 * a + 8 * ks,
                     desc_kmajor<kChunk>(kb + ks * 2 * kChunk * 16), IY, (ks > 0 || a > 0));
#pragma unroll
    for (int ks = 0; ks < kChunk / 16; ks++)
#pragma unroll
      for (int q = 0; q < 2; q++)
        umma_bf16(cx.tmem + kTmZ + 16 * ks, desc_mnmajor<kChunk>(vb + ks * 256),
                  desc_mnmajor<kChunk>(tvb + q * TPLANE + ks * 256 + ks * 2 * kChunk * 16),
                  idesc_bf16(kTcRows, kChunk - 16 * ks, true, true), (ks > 0 || q > 0));
    umma_commit(cx.mbar);
    hooks.after_first();
  }
  hooks.during_first(s);
  ok = tc_wait(cx);

  // -Y terms over Y's columns (once every thread has its slice of Y); Z -= Y Tb^T
  {
    float y[YC];
#pragma unroll
    for (int pc = 0; pc < YC / YP; pc++)
      tmem_load<YP>(tl + kTmY + cs * YC + YP * pc, *reinterpret_cast<float(*)[YP]>(&y[YP * pc]));
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
#pragma unroll
    for (int pc = 0; pc < YC / YP; pc++)
      store_terms<YP / 2, true>(tl + kTmYA + (cs * YC + YP * pc) / 2, 32, &y[YP * pc]);
    tmem_wait_st();
  }
  tc_fence_before();
  if (__syncthreads_or(!ok)) return kStepFailed;
  if (w == 0) {
    tc_fence_after();
    using PY = SplitPairs<2, 2>;
#pragma unroll
    for (int ks = 0; ks < kChunk / 16; ks++)
#pragma unroll
      for (int p = 0; p < PY::kCount; p++)
        umma_bf16_ts(cx.tmem + kTmZ + 16 * ks, cx.tmem + kTmYA + 32 * PY::a(p) + 8 * ks,
                     desc_mnmajor<kChunk>(tbb + PY::b(p) * TPLANE + ks * 256 + ks * 2 * kChunk * 16),
                     idesc_bf16(kTcRows, kChunk - 16 * ks, false, true), 1u);
    umma_commit(cx.mbar);
    hooks.after_second();
  }
  ok = tc_wait(cx);

  // Ud = dvec * Z -> terms; P = Ud K
#pragma unroll
  for (int pc = 0; pc < YC / YP; pc++) {
    float z[YP];
    tmem_load<YP>(tl + kTmZ + cs * YC + YP * pc, z);
#pragma unroll
    for (int i = 0; i < YP; i++) z[i] = __fmul_rn(hd.dvec[cs * YC + YP * pc + i], z[i]);
    store_terms<YP / 2, false>(tl + kTmYA + (cs * YC + YP * pc) / 2, 32, z);
  }
  tmem_wait_st();
  tc_fence_before();
  if (__syncthreads_or(!ok)) return kStepFailed;
  if (w == 0) {
    tc_fence_after();
#pragma unroll
    for (int ks = 0; ks < kChunk / 16; ks++)
#pragma unroll
      for (int a = 0; a < 2; a++)
        umma_bf16_ts(cx.tmem + kTmP, cx.tmem + kTmYA + 32 * a + 8 * ks,
                     desc_mnmajor<kChunk>(kb + ks * 256), IP, (ks > 0 || a > 0));
    umma_commit(cx.mbar);
    hooks.after_last();
  }
  ok = tc_wait(cx);

  // S <- exp(G_C) S + P
  const float gam = hd.gamma[0];
#pragma unroll
  for (int pc = 0; pc < SC / 32; pc++) {
    float p[32];
    tmem_load<32>(tl + kTmP + cs * SC + 32 * pc, p);
#pragma unroll
    for (int i = 0; i < 32; i++) s[32 * pc + i] = __fmaf_rn(gam, s[32 * pc + i], p[i]);
  }
  tc_fence_before();
  return __syncthreads_or(!ok) ? kStepFailed : kStepDone;
}

// Pack arrival: thread 0 issues one bulk copy per chunk into a buffer whose
// mbarrier counts the bytes; every thread waits (bounded) on that barrier.
// Buffer b's j-th use completes phase j, so chunk c waits for parity
// (c >> 1) & 1 on buffer c & 1.
template <int D, class IN>
__device__ __forceinline__ void pack_fetch(WalkPack<D, IN>& dst, const char* src, uint64_t* bar) {
  const uint32_t mb = smem_u32(bar);
  mbar_expect_tx(mb, (uint32_t)sizeof(WalkPack<D, IN>));
  bulk_load(smem_u32(&dst), src, (uint32_t)sizeof(WalkPack<D, IN>), mb);
}
__device__ __forceinline__ bool pack_wait(uint64_t* bars, int64_t c) {
  return mbar_wait(smem_u32(&bars[c & 1]), (uint32_t)((c >> 1) & 1), kTcWaitPolls);
}
// After a failed wait: wait (bounded) for every pack copy still in flight,
// chunks c .. issued - 1.
__device__ __forceinline__ void pack_drain(uint64_t* bars, int64_t c, int64_t issued) {
  for (int64_t j = c; j < issued; j++) (void)pack_wait(bars, j);
}
__device__ __forceinline__ void pack_bars_init(uint64_t* bars) {
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars[0]), 1);
    mbar_init(smem_u32(&bars[1]), 1);
    fence_mbar_init();
  }
  __syncthreads();
}

// A state row of D fp32 values (16-byte pieces).
template <int D>
__device__ __forceinline__ void row_load(float (&s)[D], const float* src) {
#pragma unroll
  for (int c = 0; c < D; c += 4) {
    const float4 x = *reinterpret_cast<const float4*>(src + c);
    s[c] = x.x;
    s[c + 1] = x.y;
    s[c + 2] = x.z;
    s[c + 3] = x.w;
  }
}
template <int D>
__device__ __forceinline__ void row_store(const float (&s)[D], float* dst) {
#pragma unroll
  for (int c = 0; c < D; c += 4)
    *reinterpret_cast<float4*>(dst + c) = make_float4(s[c], s[c + 1], s[c + 2], s[c + 3]);
}

}  // namespace gdn
